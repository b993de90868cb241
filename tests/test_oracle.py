"""Pins of the fp64 oracle against what the pages and the mathematics fix (CPU only).

Each pin is chosen so that a plausible mistake in the oracle (a dropped term, a wrong
sign, index or scale, a transposed operand) fails at least one of them; the planted-
mistake tests at the end check exactly that by patching the oracle on the CPU.
"""
import math
import os

import numpy as np
import pytest
import torch

import oracle
from oracle import rope_attention as ra
from workloads import WORKLOADS, make_inputs, score_bound

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _tiny(n, d, H=1, B=1, seed=0, dist="uniform"):
    rng = np.random.default_rng(seed)
    f = (lambda *s: rng.uniform(-1, 1, s)) if dist == "uniform" else (lambda *s: rng.standard_normal(s))
    return {
        "A1": f(B, H, n, d), "A2": f(B, H, n, d), "A3": f(B, H, n, d), "E": f(B, H, n, d),
        "WQ": rng.standard_normal((H, d, d)) / math.sqrt(d),
        "WK": rng.standard_normal((H, d, d)) / math.sqrt(d),
        "WV": rng.standard_normal((H, d, d)) / math.sqrt(d),
        "pos": np.arange(n, dtype=np.int32),
    }


def _rel(a, b):
    a, b = np.asarray(a, float), np.asarray(b, float)
    nb = np.linalg.norm(b)
    return np.linalg.norm(a - b) / (nb if nb > 0 else 1.0)


# ---------------------------------------------------------------------------------------
# Pin helpers (each returns an error measure; the planted-mistake tests reuse them)
# ---------------------------------------------------------------------------------------

def fd_gradient_error(inp, causal, base, h_rel=1e-5):
    """max over WQ, WK, WV of ||g_fd - g|| / ||g|| with central differences of Loss."""
    g = oracle.forward_backward(inp, causal, base)
    worst = 0.0
    for wname, gname in (("WQ", "dWQ"), ("WK", "dWK"), ("WV", "dWV")):
        W = inp[wname]
        fd = np.zeros_like(W, dtype=float)
        for idx in np.ndindex(W.shape):
            w0 = W[idx]
            step = h_rel * max(1.0, abs(w0))
            W[idx] = w0 + step
            lp = oracle.loss_only(inp, causal, base)
            W[idx] = w0 - step
            lm = oracle.loss_only(inp, causal, base)
            W[idx] = w0
            fd[idx] = (lp - lm) / (2 * step)
        worst = max(worst, _rel(g[gname], fd))
    return worst


def fd_input_gradient_error(inp, causal, base, h_rel=1e-5):
    """max over A1, A2, A3 of ||g_fd - g|| / ||g|| with central differences of Loss
    (every entry of every instance)."""
    g = oracle.forward_backward(inp, causal, base)
    worst = 0.0
    for aname, gname in (("A1", "dA1"), ("A2", "dA2"), ("A3", "dA3")):
        A = inp[aname]
        fd = np.zeros_like(A, dtype=float)
        for idx in np.ndindex(A.shape):
            a0 = A[idx]
            step = h_rel * max(1.0, abs(a0))
            A[idx] = a0 + step
            lp = oracle.loss_only(inp, causal, base)
            A[idx] = a0 - step
            lm = oracle.loss_only(inp, causal, base)
            A[idx] = a0
            fd[idx] = (lp - lm) / (2 * step)
        worst = max(worst, _rel(g[gname], fd))
    return worst


def sdpa_error(inp, causal):
    """Positions all zero: compare O, lse, loss and dW with torch's SDPA + autograd (fp64).

    With every angle zero RoPE is the identity, so the problem reduces to plain softmax
    attention (the one-layer attention of Alman and Song, and D^-1 A V of the
    HyperAttention article); torch's scaled_dot_product_attention is a library
    implementation of it with scale 1/sqrt(d), and autograd differentiates it.
    """
    inp = dict(inp)
    inp["pos"] = np.zeros_like(inp["pos"])
    r = oracle.forward_backward(inp, causal, 10000.0)
    t = {k: torch.tensor(np.asarray(inp[k], float), dtype=torch.float64) for k in
         ("A1", "A2", "A3", "E")}
    W = {k: torch.tensor(np.asarray(inp[k], float), dtype=torch.float64, requires_grad=True)
         for k in ("WQ", "WK", "WV")}
    Q = torch.einsum("bhnd,hde->bhne", t["A1"], W["WQ"])
    K = torch.einsum("bhnd,hde->bhne", t["A2"], W["WK"])
    V = torch.einsum("bhnd,hde->bhne", t["A3"], W["WV"])
    O = torch.nn.functional.scaled_dot_product_attention(Q, K, V, is_causal=causal)
    loss = 0.5 * ((O - t["E"]) ** 2).sum()
    loss.backward()
    d = Q.shape[-1]
    Z = Q @ K.transpose(-1, -2) / math.sqrt(d)
    if causal:
        n = Q.shape[-2]
        Z = Z.masked_fill(torch.ones(n, n, dtype=torch.bool).triu(1), float("-inf"))
    lse = torch.logsumexp(Z, dim=-1)
    errs = [
        _rel(r["O"], O.detach().numpy()),
        _rel(r["lse"], lse.detach().numpy()),
        abs(r["loss"] - loss.item()) / abs(loss.item()),
        _rel(r["dWQ"], W["WQ"].grad.numpy()),
        _rel(r["dWK"], W["WK"].grad.numpy()),
        _rel(r["dWV"], W["WV"].grad.numpy()),
    ]
    return max(errs)


def golden_error():
    """Max abs deviation from the hand-worked n=2, d=2 example in tests/golden."""
    vals = {}
    with open(os.path.join(GOLDEN, "worked_n2_d2.txt")) as f:
        for line in f:
            if line.startswith("#") or not line.strip():
                continue
            k, *v = line.split()
            vals[k] = np.array([float(x) for x in v])
    I = np.eye(2)[None, None]
    inp = {"A1": I.copy(), "A2": I.copy(), "A3": I.copy(), "E": np.zeros((1, 1, 2, 2)),
           "WQ": np.eye(2)[None], "WK": np.eye(2)[None], "WV": np.eye(2)[None],
           "pos": np.array([0, 1], dtype=np.int32)}
    worst = 0.0
    for tag, causal in (("noncausal", False), ("causal", True)):
        r = oracle.forward_backward(inp, causal, 10000.0, want_grad=False)
        worst = max(worst, np.max(np.abs(r["O"].ravel() - vals[f"{tag}.O"])),
                    np.max(np.abs(r["lse"].ravel() - vals[f"{tag}.lse"])),
                    abs(r["loss"] - vals[f"{tag}.loss"][0]))
    return worst


def gamma_jacobian_error(n=6, seed=3):
    """gamma_i against J_i beta_i with the softmax Jacobian J_i = diag(s_i) - s_i s_i^T formed."""
    rng = np.random.default_rng(seed)
    Z = rng.standard_normal((4, n))
    s, _ = ra.softmax_rows(Z)
    beta = rng.standard_normal((4, n))
    g = ra.gamma_closed_form(s, beta)
    ref = np.stack([(np.diag(s[i]) - np.outer(s[i], s[i])) @ beta[i] for i in range(4)])
    return _rel(g, ref)


# ---------------------------------------------------------------------------------------
# RoPE
# ---------------------------------------------------------------------------------------

def test_theta_closed_form():
    # base^(-2k/d) with d=8, base=1e4 is 10^-k exactly in real arithmetic
    np.testing.assert_allclose(ra.rope_theta(8, 1e4), [1.0, 0.1, 0.01, 0.001], rtol=1e-15)
    np.testing.assert_allclose(ra.rope_theta(2, 5e5), [1.0], rtol=0)


def test_rope_d2_is_plain_rotation():
    # d = 2: one pair rotated counter-clockwise by pos radians (theta_0 = 1)
    x = np.array([[1.0, 0.0], [1.0, 0.0], [0.0, 1.0]])
    pos = np.array([0, 1, 3])
    y = ra.rope_rotate(x, ra.rope_angles(pos, 2, 10000.0))
    np.testing.assert_allclose(y[0], [1, 0], atol=1e-15)
    np.testing.assert_allclose(y[1], [math.cos(1), math.sin(1)], atol=1e-15)
    np.testing.assert_allclose(y[2], [-math.sin(3), math.cos(3)], atol=1e-15)


def test_rope_pairs_are_adjacent():
    # a vector with only component 2 set moves only within the pair (2, 3), by theta_1
    x = np.zeros((1, 8)); x[0, 2] = 1.0
    th = ra.rope_theta(8, 1e4)
    y = ra.rope_rotate(x, ra.rope_angles(np.array([7]), 8, 1e4))
    want = np.zeros(8); want[2] = math.cos(7 * th[1]); want[3] = math.sin(7 * th[1])
    np.testing.assert_allclose(y[0], want, atol=1e-15)


def test_rope_norm_and_inverse():
    rng = np.random.default_rng(1)
    X = rng.standard_normal((50, 16))
    phi = ra.rope_angles(np.arange(50) * 37, 16, 1e4)
    Y = ra.rope_rotate(X, phi)
    np.testing.assert_allclose(np.linalg.norm(Y, axis=1), np.linalg.norm(X, axis=1), rtol=1e-13)
    np.testing.assert_allclose(ra.rope_rotate(Y, -phi), X, atol=1e-13)


@pytest.mark.parametrize("base", [1e4, 5e5, 10.0])
def test_scores_depend_on_relative_position_only(base):
    rng = np.random.default_rng(2)
    n, d = 24, 16
    Q, K = rng.standard_normal((n, d)), rng.standard_normal((n, d))
    pos = np.arange(n)
    z0 = ra.rope_rotate(Q, ra.rope_angles(pos, d, base)) @ ra.rope_rotate(K, ra.rope_angles(pos, d, base)).T
    z1 = (ra.rope_rotate(Q, ra.rope_angles(pos + 1000, d, base))
          @ ra.rope_rotate(K, ra.rope_angles(pos + 1000, d, base)).T)
    np.testing.assert_allclose(z1, z0, atol=1e-10 * np.abs(z0).max())


# ---------------------------------------------------------------------------------------
# softmax, gamma, delta identity
# ---------------------------------------------------------------------------------------

def test_softmax_rows_sum_to_one_and_causal_zeros():
    inp = _tiny(17, 8)
    r = ra.instance_forward_backward(*(inp[k][0, 0] for k in ("A1", "A2", "A3", "E")),
                                     inp["WQ"][0], inp["WK"][0], inp["WV"][0], inp["pos"],
                                     True, 1e4, want_grad=False)
    Z = ra.scores_rows(r["Qt"], r["Kt"], np.arange(17), True)
    s, lse = ra.softmax_rows(Z)
    assert np.max(np.abs(s.sum(1) - 1)) <= 1e-14
    assert np.all(s[np.triu_indices(17, 1)] == 0.0)
    np.testing.assert_allclose(lse, r["lse"], rtol=1e-14)


def test_gamma_matches_explicit_jacobian():
    assert gamma_jacobian_error() <= 1e-13


def test_gamma_matches_brute_force_derivative():
    # gamma_i = d(1/2 ||s_i V - e_i||^2)/dZ_i, checked by central differences in Z
    rng = np.random.default_rng(4)
    n, d = 7, 3
    Z = rng.standard_normal((1, n)); V = rng.standard_normal((n, d)); e = rng.standard_normal((1, d))

    def f(Z):
        s, _ = ra.softmax_rows(Z)
        return 0.5 * np.sum((s @ V - e) ** 2)

    s, _ = ra.softmax_rows(Z)
    beta = (s @ V - e) @ V.T
    g = ra.gamma_closed_form(s, beta)
    fd = np.zeros_like(Z)
    for j in range(n):
        Zp, Zm = Z.copy(), Z.copy(); Zp[0, j] += 1e-6; Zm[0, j] -= 1e-6
        fd[0, j] = (f(Zp) - f(Zm)) / 2e-6
    assert _rel(g, fd) <= 1e-8


def test_delta_identity():
    # s_i^T beta_i = <l_i, O_i>: the shortcut the GPU path relies on
    rng = np.random.default_rng(5)
    n, d = 9, 4
    Z = rng.standard_normal((n, n)); V = rng.standard_normal((n, d)); E = rng.standard_normal((n, d))
    s, _ = ra.softmax_rows(Z)
    O = s @ V; ell = O - E; beta = ell @ V.T
    np.testing.assert_allclose(np.sum(s * beta, 1), np.sum(ell * O, 1), rtol=1e-12)


# ---------------------------------------------------------------------------------------
# whole-instance pins
# ---------------------------------------------------------------------------------------

def test_golden_worked_example():
    assert golden_error() <= 1e-14


@pytest.mark.parametrize("n,d", [(1, 2), (2, 4), (3, 2), (5, 8), (8, 4)])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("base", [1e4, 10.0])
def test_finite_differences(n, d, causal, base):
    inp = _tiny(n, d, seed=n * 100 + d)
    inp["pos"] = np.arange(n, dtype=np.int32) * 3 + 2      # non-trivial angles
    assert fd_gradient_error(inp, causal, base) <= 1e-6


def test_finite_differences_batch_and_heads():
    inp = _tiny(4, 4, H=2, B=2, seed=11)
    assert fd_gradient_error(inp, True, 1e4) <= 1e-6


@pytest.mark.parametrize("n,d", [(1, 2), (3, 2), (5, 4), (8, 4)])
@pytest.mark.parametrize("causal", [False, True])
def test_input_gradient_finite_differences(n, d, causal):
    """dA1, dA2, dA3 (next row of the scope: input gradients) against central differences."""
    inp = _tiny(n, d, seed=5 + n)
    assert fd_input_gradient_error(inp, causal, 1e4) <= 1e-6


def test_input_gradient_finite_differences_batch_and_heads():
    inp = _tiny(3, 4, H=2, B=2, seed=13)
    assert fd_input_gradient_error(inp, True, 10.0) <= 1e-6


def test_planted_input_gradient_untransposed_weight(monkeypatch):
    """dA1 = dQ WQ (a missing transpose) fails the finite-difference pin."""
    orig = ra.instance_forward_backward

    def bad(*args, **kw):
        out = orig(*args, **kw)
        if "dA1" in out:
            out["dA1"] = out["dQ"] @ np.asarray(args[4], float)
        return out
    monkeypatch.setattr(ra, "instance_forward_backward", bad)
    assert fd_input_gradient_error(_tiny(3, 4, seed=2), False, 1e4) > 1e-3


@pytest.mark.parametrize("causal", [False, True])
def test_no_rope_matches_library_attention(causal):
    inp = _tiny(40, 16, H=2, B=2, seed=7, dist="normal")
    assert sdpa_error(inp, causal) <= 1e-12


def test_uniform_softmax_closed_form():
    inp = _tiny(12, 8, seed=8)
    inp["WQ"][:] = 0.0                                   # all scores 0 -> s uniform
    V = inp["A3"][0, 0] @ inp["WV"][0]
    r = oracle.forward_backward(inp, False, 1e4, want_grad=False)
    np.testing.assert_allclose(r["O"][0, 0], np.tile(V.mean(0), (12, 1)), rtol=1e-13)
    rc = oracle.forward_backward(inp, True, 1e4, want_grad=False)
    pref = np.cumsum(V, 0) / np.arange(1, 13)[:, None]
    np.testing.assert_allclose(rc["O"][0, 0], pref, rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(rc["lse"][0, 0], np.log(np.arange(1, 13)), rtol=1e-14)


def test_single_token_closed_form():
    inp = _tiny(1, 8, seed=9)
    r = oracle.forward_backward(inp, False, 1e4)
    A3, WV, E = inp["A3"][0, 0], inp["WV"][0], inp["E"][0, 0]
    O = A3 @ WV
    np.testing.assert_allclose(r["O"][0, 0], O, rtol=1e-14)
    assert np.all(r["dWQ"] == 0) and np.all(r["dWK"] == 0)
    np.testing.assert_allclose(r["dWV"][0], A3.T @ (O - E), rtol=1e-13)


def test_zero_gradient_when_target_equals_output():
    inp = _tiny(10, 8, H=2, B=2, seed=10)
    r = oracle.forward_backward(inp, True, 1e4)
    inp["E"] = r["O"].copy()
    z = oracle.forward_backward(inp, True, 1e4)
    assert z["loss"] == 0.0
    for k in ("dWQ", "dWK", "dWV"):
        assert np.all(z[k] == 0.0)


def test_sampled_rows_match_full_instance():
    inp = _tiny(70, 8, H=2, B=2, seed=12)
    full = oracle.forward_backward(inp, True, 1e4)
    rows = np.array([0, 1, 33, 69])
    r = oracle.forward_rows(inp, 1, 1, rows, True, 1e4)
    np.testing.assert_allclose(r["O"], full["O"][1, 1, rows], rtol=1e-12)
    np.testing.assert_allclose(r["lse"], full["lse"][1, 1, rows], rtol=1e-12)
    np.testing.assert_allclose(r["dQt"], full["dQt"][1, 1, rows], rtol=1e-11, atol=1e-14)


def test_row_block_size_does_not_matter():
    inp = _tiny(50, 8, seed=13)
    a = ra.instance_forward_backward(*(inp[k][0, 0] for k in ("A1", "A2", "A3", "E")),
                                     inp["WQ"][0], inp["WK"][0], inp["WV"][0], inp["pos"],
                                     True, 1e4, rb=7)
    b = ra.instance_forward_backward(*(inp[k][0, 0] for k in ("A1", "A2", "A3", "E")),
                                     inp["WQ"][0], inp["WK"][0], inp["WV"][0], inp["pos"],
                                     True, 1e4, rb=256)
    for k in ("O", "lse", "dWQ", "dWK", "dWV"):
        np.testing.assert_allclose(a[k], b[k], rtol=1e-12, atol=1e-14)


def test_bounded_regime_generator_respects_score_bound():
    # the bounded-entry workload at a reduced n: every |score| of the rounded inputs <= B
    w = WORKLOADS["b1_h8_n32768_d128_bf16_causal_bounded"].with_sizes(n=512, H=2)
    inp = make_inputs(w)
    Bnd = score_bound(w.n)
    worst = 0.0
    for h in range(w.H):
        r = ra.instance_forward_backward(*(inp[k][0, h] for k in ("A1", "A2", "A3", "E")),
                                         inp["WQ"][h], inp["WK"][h], inp["WV"][h], inp["pos"],
                                         False, w.rope_base, want_grad=False)
        Z = ra.scores_rows(r["Qt"], r["Kt"], np.arange(w.n), False)
        worst = max(worst, np.abs(Z).max())
    assert worst <= Bnd
    assert worst > 0.05 * Bnd          # not trivially tiny


# ---------------------------------------------------------------------------------------
# planted mistakes: each must break at least one pin
# ---------------------------------------------------------------------------------------

def _all_pins(seed=21):
    inp = _tiny(5, 4, H=1, B=2, seed=seed)
    inp["pos"] = np.arange(5, dtype=np.int32) * 2 + 1
    inp2 = _tiny(12, 8, H=1, B=1, seed=seed + 1, dist="normal")
    return {
        "fd": fd_gradient_error(inp, True, 1e4),
        "fd_nc": fd_gradient_error(inp, False, 1e4),
        "sdpa": max(sdpa_error(inp2, False), sdpa_error(inp2, True)),
        "golden": golden_error(),
        "jac": gamma_jacobian_error(),
    }


PIN_LIMITS = {"fd": 1e-6, "fd_nc": 1e-6, "sdpa": 1e-12, "golden": 1e-14, "jac": 1e-13}


def test_unplanted_oracle_passes_all_pins():
    errs = _all_pins()
    assert all(errs[k] <= PIN_LIMITS[k] for k in errs), errs


def _broken(errs):
    return any(errs[k] > PIN_LIMITS[k] for k in errs)


def test_planted_drop_gamma2(monkeypatch):
    monkeypatch.setattr(ra, "gamma_closed_form", lambda s, beta: s * beta)
    assert _broken(_all_pins())


def test_planted_gamma2_sign(monkeypatch):
    monkeypatch.setattr(ra, "gamma_closed_form",
                        lambda s, beta: s * beta + s * np.sum(s * beta, 1, keepdims=True))
    assert _broken(_all_pins())


def test_planted_clockwise_rotation(monkeypatch):
    orig = ra.rope_rotate
    monkeypatch.setattr(ra, "rope_rotate", lambda X, phi: orig(X, -phi))
    assert _broken(_all_pins())


def test_planted_swapped_pair_roles(monkeypatch):
    def bad(X, phi):
        X = np.asarray(X, float); c, s = np.cos(phi), np.sin(phi)
        out = np.empty_like(X)
        out[:, 0::2] = X[:, 0::2] * c + X[:, 1::2] * s
        out[:, 1::2] = -X[:, 0::2] * s + X[:, 1::2] * c
        return out
    monkeypatch.setattr(ra, "rope_rotate", bad)
    assert _broken(_all_pins())


def test_planted_missing_scale(monkeypatch):
    def bad(Qt, Kt, rows, causal):
        Z = Qt[rows] @ Kt.T
        if causal:
            j = np.arange(Kt.shape[0])
            Z = np.where(j[None, :] > np.asarray(rows)[:, None], -np.inf, Z)
        return Z
    monkeypatch.setattr(ra, "scores_rows", bad)
    assert _broken(_all_pins())


def test_planted_causal_off_by_one(monkeypatch):
    def bad(Qt, Kt, rows, causal):
        Z = (Qt[rows] @ Kt.T) / math.sqrt(Qt.shape[1])
        if causal:
            j = np.arange(Kt.shape[0])
            Z = np.where(j[None, :] >= np.asarray(rows)[:, None] + 2, -np.inf, Z)
        return Z
    monkeypatch.setattr(ra, "scores_rows", bad)
    assert _broken(_all_pins())


def test_planted_transposed_weight(monkeypatch):
    orig = ra._project

    def bad(A1, A2, A3, WQ, WK, WV, pos, base):
        return orig(A1, A2, A3, np.asarray(WQ).T, WK, WV, pos, base)
    monkeypatch.setattr(ra, "_project", bad)
    assert _broken(_all_pins())


def test_planted_softmax_without_max_shift_still_exact_but_lse_wrong(monkeypatch):
    def bad(Z):
        e = np.exp(Z)
        tot = e.sum(1, keepdims=True)
        return e / tot, np.log(tot)[:, 0] + 1e-9
    monkeypatch.setattr(ra, "softmax_rows", bad)
    assert _broken(_all_pins())


# ---------------------------------------------------------------------------------------
# One combined weight X (the page's own parameterisation dLoss/dx = A~^T vec(gamma))
# ---------------------------------------------------------------------------------------

def _tiny_x(n, d, seed=0, B=1, H=1):
    inp = _tiny(n, d, H=H, B=B, seed=seed)
    rng = np.random.default_rng(seed + 100)
    inp["X"] = rng.standard_normal((H, d, d)) / math.sqrt(d)
    return inp


def test_rotation_matrix_matches_rope_and_composes():
    rng = np.random.default_rng(4)
    d = 6
    a, b = rng.uniform(-3, 3, d // 2), rng.uniform(-3, 3, d // 2)
    Ra, Rb = ra.rotation_matrix(a), ra.rotation_matrix(b)
    x = rng.standard_normal(d)
    assert np.allclose(Ra @ x, ra.rope_rotate(x[None, :], a[None, :])[0], atol=1e-14)
    assert np.allclose(Ra.T @ Ra, np.eye(d), atol=1e-14)
    assert np.allclose(Ra @ Rb, ra.rotation_matrix(a + b), atol=1e-13)


@pytest.mark.parametrize("n,d", [(1, 2), (3, 2), (4, 4), (6, 4)])
@pytest.mark.parametrize("causal", [False, True])
def test_combined_weight_literal_finite_differences(n, d, causal):
    """A~^T vec(gamma), built literally row by row, against central differences of the loss."""
    inp = _tiny_x(n, d, seed=n + d)
    args = lambda X: (inp["A1"][0, 0], inp["A2"][0, 0], inp["A3"][0, 0], inp["E"][0, 0], X,
                      inp["WV"][0], inp["pos"], causal, 10.0)
    X = inp["X"][0].copy()
    g = ra.combined_weight_literal(*args(X))["dX"]
    fd = np.zeros_like(X)
    for idx in np.ndindex(X.shape):
        step = 1e-5 * max(1.0, abs(X[idx]))
        Xp, Xm = X.copy(), X.copy()
        Xp[idx] += step
        Xm[idx] -= step
        fd[idx] = (ra.combined_weight_literal(*args(Xp))["loss"]
                   - ra.combined_weight_literal(*args(Xm))["loss"]) / (2 * step)
    assert _rel(g, fd) <= 1e-6


def combined_route_error(inp, causal, base):
    """max relative difference between the literal A~^T vec(gamma) form and the general
    problem with WQ = I, WK = X^T (loss, dX, dWV) over the instances of ``inp``."""
    eff = oracle.combined_weight_forward_backward(inp, causal, base)
    B, H = inp["A1"].shape[:2]
    worst = 0.0
    dX_sum = np.zeros_like(eff["dX"])
    dWV_sum = np.zeros_like(eff["dWV"])
    loss = 0.0
    for b in range(B):
        for h in range(H):
            lit = ra.combined_weight_literal(inp["A1"][b, h], inp["A2"][b, h], inp["A3"][b, h],
                                             inp["E"][b, h], inp["X"][h], inp["WV"][h],
                                             inp["pos"], causal, base)
            dX_sum[h] += lit["dX"]
            dWV_sum[h] += lit["dWV"]
            loss += lit["loss"]
    worst = max(worst, _rel(eff["dX"], dX_sum), _rel(eff["dWV"], dWV_sum),
                abs(eff["loss"] - loss) / abs(loss))
    return worst


@pytest.mark.parametrize("causal", [False, True])
def test_combined_weight_literal_equals_general_route(causal):
    inp = _tiny_x(5, 4, seed=8, B=2, H=2)
    inp["pos"] = np.array([3, 7, 8, 20, 21], dtype=np.int32)   # non-contiguous positions
    assert combined_route_error(inp, causal, 1e4) <= 1e-12


def test_planted_combined_weight_missing_transpose(monkeypatch):
    """dX taken as dWK instead of dWK^T breaks the literal-vs-general pin."""
    orig = oracle.combined_weight_forward_backward

    def bad(inp, causal, base):
        out = orig(inp, causal, base)
        out["dX"] = np.transpose(out["dX"], (0, 2, 1))
        return out
    monkeypatch.setattr(oracle, "combined_weight_forward_backward", bad)
    assert combined_route_error(_tiny_x(4, 4, seed=3), False, 10.0) > 1e-3

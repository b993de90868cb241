"""Pins of the oracle's approximate method (polynomial-kernel softmax, low-rank factors).

The approximate gradient has no closed form of its own to compare with, so its oracle is pinned
by what the mathematics fixes: the features reproduce the polynomial exactly (a different
computation path than evaluating it entry by entry), the polynomial is the Taylor series of exp,
a high degree on bounded scores reproduces the exact (finite-difference-pinned) oracle, degree 0
gives the uniform softmax whose output has a closed form, and planted mistakes break a pin.
"""
import math

import numpy as np
import pytest

import oracle
from oracle import rope_attention as ra_oracle
from workloads import WORKLOADS, make_inputs


def _small(n=24, d=8, causal=True, H=2, B=1, seed=0):
    w = WORKLOADS["b1_h8_n32768_d128_bf16_causal_bounded"].with_sizes(
        B=B, H=H, n=n, d=d, causal=causal, dtype="f32")
    return w, make_inputs(w, seed=seed)


def _rel(a, b):
    return float(np.linalg.norm(np.asarray(a) - np.asarray(b)) / np.linalg.norm(np.asarray(b)))


@pytest.mark.parametrize("degree", [0, 1, 2, 3])
def test_features_reproduce_the_polynomial(degree):
    rng = np.random.default_rng(degree)
    d = 4
    Q = rng.standard_normal((7, d))
    K = rng.standard_normal((5, d))
    U = oracle.poly_features(Q, degree)
    F = oracle.poly_features(K, degree)
    assert U.shape[1] == sum(d ** r for r in range(degree + 1))
    want = oracle.poly_exp(Q @ K.T / math.sqrt(d), degree)
    assert np.allclose(U @ F.T, want, rtol=1e-13, atol=1e-13)


def test_poly_exp_is_the_taylor_series():
    z = np.linspace(-3.0, 3.0, 61)
    assert np.array_equal(oracle.poly_exp(z, 0), np.ones_like(z))
    assert np.allclose(oracle.poly_exp(z, 1), 1.0 + z, rtol=0, atol=1e-15)
    assert np.allclose(oracle.poly_exp(z, 2), 1.0 + z + z * z / 2, rtol=0, atol=1e-14)
    assert np.allclose(oracle.poly_exp(z, 30), np.exp(z), rtol=1e-14, atol=0)


@pytest.mark.parametrize("causal", [False, True])
def test_high_degree_reproduces_the_exact_oracle(causal):
    w, inp = _small(causal=causal)
    ex = oracle.forward_backward(inp, causal, w.rope_base)
    ap = oracle.approx_forward_backward(inp, causal, w.rope_base, degree=24)
    for k in ("O", "dWQ", "dWK", "dWV"):
        assert _rel(ap[k], ex[k]) < 1e-12, k
    assert abs(ap["loss"] - ex["loss"]) <= 1e-12 * ex["loss"]
    assert np.allclose(np.log(ap["D"]), ex["lse"], atol=1e-12)  # D = sum_j exp(z_ij)


@pytest.mark.parametrize("causal", [False, True])
def test_degree_zero_is_the_uniform_softmax(causal):
    w, inp = _small(n=9, d=4, causal=causal, H=1)
    ap = oracle.approx_forward_backward(inp, causal, w.rope_base, degree=0)
    V = inp["A3"][0, 0].astype(np.float64) @ inp["WV"][0].astype(np.float64)
    n = V.shape[0]
    want = (np.cumsum(V, axis=0) / np.arange(1, n + 1)[:, None]) if causal else \
        np.broadcast_to(V.mean(axis=0), V.shape)
    assert np.allclose(ap["O"][0, 0], want, atol=1e-13)
    assert np.allclose(ap["D"][0, 0], np.arange(1, n + 1) if causal else n)


def test_degree_one_in_the_bounded_regime_is_close_to_exact():
    """The bounded construction keeps |z| small, so the error of degree 1 is of order z^2
    (a reported property of the approximation, checked loosely here)."""
    w, inp = _small(n=96, d=16, causal=True)
    ex = oracle.forward_backward(inp, True, w.rope_base)
    ap1 = oracle.approx_forward_backward(inp, True, w.rope_base, degree=1)
    ap2 = oracle.approx_forward_backward(inp, True, w.rope_base, degree=2)
    e1 = max(_rel(ap1[k], ex[k]) for k in ("O", "dWQ", "dWK", "dWV"))
    e2 = max(_rel(ap2[k], ex[k]) for k in ("O", "dWQ", "dWK", "dWV"))
    assert e2 < e1 < 0.1


def test_planted_row_factor_and_dropped_gamma2(monkeypatch):
    """A factor common to a row cancels in the normalisation (the pin does not move), while a
    dropped gamma_2 breaks the high-degree pin against the exact oracle."""
    real = ra_oracle.poly_exp

    def scaled(z, degree):
        return 1.5 * real(z, degree)   # a row-independent factor cancels in the normalisation ...
    monkeypatch.setattr(ra_oracle, "poly_exp", scaled)
    w, inp = _small(n=12, d=4, causal=True, H=1)
    ex = oracle.forward_backward(inp, True, w.rope_base)
    ap = ra_oracle.approx_forward_backward(inp, True, w.rope_base, degree=24)
    assert _rel(ap["dWQ"], ex["dWQ"]) < 1e-12       # ... so the normalised method is unchanged

    def unnormalised_gamma(s, beta):
        return s * beta                          # gamma_2 dropped
    monkeypatch.setattr(ra_oracle, "gamma_closed_form", unnormalised_gamma)
    ap = ra_oracle.approx_forward_backward(inp, True, w.rope_base, degree=24)
    assert _rel(ap["dWQ"], ex["dWQ"]) > 1e-3

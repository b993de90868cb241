"""Plain fp64 definitions of RoPE attention, its squared-error loss and closed-form gradient.

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__.py``).  Shares no code with the CUDA path.

Sources, by page and section:

* "Technische Samenvatting: RoPE Attention kan bijna lineair worden getraind"
  (summary of arXiv 2412.17316), section Probleemdefinitie and Methodologie 1
  "Gradientherformulering in gesloten vorm": the loss of RoPE attention with respect
  to the weight matrices, and the closed form dLoss/dx = A~^T vec(gamma(x)) built from
  s(x) (the normalised softmax), l(x) (attention output minus target), beta(x) (the
  error combined with the value matrix) and gamma(x).
* Same page, Methodologie 2 "Low-Rank Benaderingsstrategie": gamma split into
  gamma_1 = diag(s) beta and gamma_2 = s s^T beta, gamma = gamma_1 - gamma_2.
* "HyperAttention" article (nearauto.com), section 方法の概要: exact attention is
  D^-1 A V with A = exp(Q K^T) taken entrywise and D the diagonal of A's row sums.

Readings where the pages are silent (each is listed in the design notes):

* scores are Q~ K~^T / sqrt(d); the loss is 1/2 ||O - E||_F^2, summed over every
  (batch, head) instance;
* RoPE rotates the adjacent pairs (2k, 2k+1), k = 0..d/2-1, counter-clockwise by
  phi_{i,k} = pos_i * base^(-2k/d);
* Q = A1 WQ, K = A2 WK, V = A3 WV (row-vector convention, W[in][out]); each (b, h) is an
  independent instance, W is per head and shared over the batch, dW sums over b;
* the causal mask removes keys j > i by index.

The method's exact result *is* the plain definition, so the oracle computes the
definition: projections, rotation, a two-pass softmax per query row, O = s V,
l = O - E, beta = l V^T, gamma = diag(s) beta - s s^T beta row by row, then
dQ~ = gamma K~ / sqrt(d), dK~ = gamma^T Q~ / sqrt(d), dV = s^T l, the inverse rotation
and dW = A^T dX.  Query rows are processed in blocks so no n x n array is held.
"""
from __future__ import annotations

import math
from typing import Dict, Iterable, Optional

import numpy as np

# Every oracle function has a pin in tests/test_oracle.py; none is unpinned.
ORACLE_PARITY_PINNED = True

F64 = np.float64


def rope_theta(d: int, base: float) -> np.ndarray:
    """theta_k = base^(-2k/d), k = 0 .. d/2-1, in fp64."""
    k = np.arange(d // 2, dtype=F64)
    return np.power(F64(base), -2.0 * k / F64(d))


def rope_angles(pos: np.ndarray, d: int, base: float) -> np.ndarray:
    """phi[i, k] = pos_i * theta_k (fp64), shape [n][d/2]."""
    return np.asarray(pos, dtype=F64)[:, None] * rope_theta(d, base)[None, :]


def rope_rotate(X: np.ndarray, phi: np.ndarray) -> np.ndarray:
    """Rotate each pair (x_2k, x_2k+1) of every row of X [n][d] by the angle phi[i, k].

    (x_2k, x_2k+1) -> (x_2k cos phi - x_2k+1 sin phi, x_2k sin phi + x_2k+1 cos phi).
    The inverse rotation is ``rope_rotate(X, -phi)``.
    """
    X = np.asarray(X, dtype=F64)
    c, s = np.cos(phi), np.sin(phi)
    x0, x1 = X[:, 0::2], X[:, 1::2]
    out = np.empty_like(X)
    out[:, 0::2] = x0 * c - x1 * s
    out[:, 1::2] = x0 * s + x1 * c
    return out


def softmax_rows(Z: np.ndarray):
    """Two-pass softmax along each row: s = exp(Z - max) / sum; also returns log-sum-exp.

    Entries equal to -inf (masked keys) get probability 0.
    """
    m = np.max(Z, axis=1, keepdims=True)
    e = np.exp(Z - m)
    tot = np.sum(e, axis=1, keepdims=True)
    s = e / tot
    lse = (m + np.log(tot))[:, 0]
    return s, lse


def gamma_closed_form(s: np.ndarray, beta: np.ndarray) -> np.ndarray:
    """gamma = gamma_1 - gamma_2 with gamma_1 = diag(s) beta and gamma_2 = s s^T beta, per row.

    For row i (one query): gamma_1,i = s_i o beta_i and gamma_2,i = s_i (s_i^T beta_i).
    """
    gamma_1 = s * beta
    gamma_2 = s * np.sum(s * beta, axis=1, keepdims=True)
    return gamma_1 - gamma_2


def scores_rows(Qt: np.ndarray, Kt: np.ndarray, rows: np.ndarray, causal: bool) -> np.ndarray:
    """Z[r, j] = Q~_{rows[r]} . K~_j / sqrt(d), with keys j > rows[r] set to -inf if causal."""
    d = Qt.shape[1]
    Z = (Qt[rows] @ Kt.T) / math.sqrt(d)
    if causal:
        j = np.arange(Kt.shape[0])
        Z = np.where(j[None, :] > np.asarray(rows)[:, None], -np.inf, Z)
    return Z


def _project(A1, A2, A3, WQ, WK, WV, pos, base):
    d = WQ.shape[0]
    phi = rope_angles(pos, d, base)
    Q = np.asarray(A1, F64) @ np.asarray(WQ, F64)
    K = np.asarray(A2, F64) @ np.asarray(WK, F64)
    V = np.asarray(A3, F64) @ np.asarray(WV, F64)
    return rope_rotate(Q, phi), rope_rotate(K, phi), V, phi


def instance_forward_backward(A1, A2, A3, E, WQ, WK, WV, pos, causal: bool, base: float,
                              want_grad: bool = True, rb: int = 256) -> Dict[str, np.ndarray]:
    """One (batch, head) instance: forward, loss and (optionally) the closed-form gradient.

    Inputs are [n][d] (A1, A2, A3, E) and [d][d] (WQ, WK, WV).  Returns O, lse, loss and,
    with ``want_grad``, dQt, dKt, dV (gradients w.r.t. the rotated Q~, K~ and V),
    dQ, dK (un-rotated), dWQ, dWK, dWV and the input gradients dA1, dA2, dA3.

    The weight gradients are the ones the problem of "RoPE Attention kan bijna lineair
    worden getraind" (Probleemdefinitie) asks for.  The input gradients follow from the same
    chain rule through Q = A1 WQ, K = A2 WK, V = A3 WV: dA1 = dQ WQ^T, dA2 = dK WK^T,
    dA3 = dV WV^T (they let layers be stacked; the page itself stops at the weights).
    """
    n, d = np.shape(A1)
    c = 1.0 / math.sqrt(d)
    Qt, Kt, V, phi = _project(A1, A2, A3, WQ, WK, WV, pos, base)
    E = np.asarray(E, F64)
    O = np.empty((n, d), F64)
    lse = np.empty(n, F64)
    loss = 0.0
    if want_grad:
        dQt = np.empty((n, d), F64)
        dKt = np.zeros((n, d), F64)
        dV = np.zeros((n, d), F64)
    for r0 in range(0, n, rb):
        r1 = min(n, r0 + rb)
        rows = np.arange(r0, r1)
        # causal: every key beyond the block's last row is masked for all its rows
        kend = r1 if causal else n
        Z = scores_rows(Qt, Kt[:kend], rows, causal)
        s, lse[r0:r1] = softmax_rows(Z)                  # s(x)
        O[r0:r1] = s @ V[:kend]                          # O = s V
        ell = O[r0:r1] - E[r0:r1]                        # l(x) = O - E
        loss += 0.5 * float(np.sum(ell * ell))
        if not want_grad:
            continue
        beta = ell @ V[:kend].T                          # beta(x) = l V^T
        gamma = gamma_closed_form(s, beta)               # gamma = diag(s)beta - s s^T beta
        dQt[r0:r1] = (gamma @ Kt[:kend]) * c
        dKt[:kend] += (gamma.T @ Qt[r0:r1]) * c
        dV[:kend] += s.T @ ell
    out = {"O": O, "lse": lse, "loss": loss, "Qt": Qt, "Kt": Kt, "V": V}
    if want_grad:
        dQ = rope_rotate(dQt, -phi)
        dK = rope_rotate(dKt, -phi)
        out.update(dQt=dQt, dKt=dKt, dV=dV, dQ=dQ, dK=dK,
                   dWQ=np.asarray(A1, F64).T @ dQ,
                   dWK=np.asarray(A2, F64).T @ dK,
                   dWV=np.asarray(A3, F64).T @ dV,
                   dA1=dQ @ np.asarray(WQ, F64).T,
                   dA2=dK @ np.asarray(WK, F64).T,
                   dA3=dV @ np.asarray(WV, F64).T)
    return out


def instance_loss(A1, A2, A3, E, WQ, WK, WV, pos, causal: bool, base: float) -> float:
    """Loss = 1/2 ||O - E||_F^2 of one instance (forward only)."""
    return instance_forward_backward(A1, A2, A3, E, WQ, WK, WV, pos, causal, base,
                                     want_grad=False)["loss"]


def _heads(inp, heads: Optional[Iterable[int]]):
    H = inp["WQ"].shape[0]
    return range(H) if heads is None else list(heads)


def forward_backward(inp: Dict[str, np.ndarray], causal: bool, base: float,
                     heads: Optional[Iterable[int]] = None,
                     want_grad: bool = True) -> Dict[str, np.ndarray]:
    """All (b, h) instances of a batch; ``heads`` restricts the work to some heads.

    Returns O [B][H][n][d], lse [B][H][n], loss (sum over the instances computed),
    dWQ, dWK, dWV [H][d][d] (summed over b) and, per instance, dQt, dKt, dV, dA1, dA2, dA3
    [B][H][n][d].  Entries of heads not computed are NaN.
    """
    B, H, n, d = inp["A1"].shape
    O = np.full((B, H, n, d), np.nan)
    lse = np.full((B, H, n), np.nan)
    dW = {k: np.full((H, d, d), np.nan) for k in ("dWQ", "dWK", "dWV")}
    extra = ({k: np.full((B, H, n, d), np.nan) for k in ("dQt", "dKt", "dV", "dA1", "dA2", "dA3")}
             if want_grad else {})
    loss = 0.0
    for h in _heads(inp, heads):
        if want_grad:
            for k in dW:
                dW[k][h] = 0.0
        for b in range(B):
            r = instance_forward_backward(inp["A1"][b, h], inp["A2"][b, h], inp["A3"][b, h],
                                          inp["E"][b, h], inp["WQ"][h], inp["WK"][h],
                                          inp["WV"][h], inp["pos"], causal, base, want_grad)
            O[b, h], lse[b, h] = r["O"], r["lse"]
            loss += r["loss"]
            if want_grad:
                for k in dW:
                    dW[k][h] += r[k]
                for k in extra:
                    extra[k][b, h] = r[k]
    out = {"O": O, "lse": lse, "loss": loss}
    if want_grad:
        out.update(dW)
        out.update(extra)
    return out


def loss_only(inp, causal, base) -> float:
    return forward_backward(inp, causal, base, want_grad=False)["loss"]


def forward_rows(inp: Dict[str, np.ndarray], b: int, h: int, rows, causal: bool,
                 base: float) -> Dict[str, np.ndarray]:
    """O, lse, and the gradient rows dQ~ for selected query rows of instance (b, h).

    Row i needs only Q~_i and all of K~ and V, so sampled rows of a large instance
    cost O(n d) each.  dQ~_i = gamma_i K~ / sqrt(d) with gamma_i from s_i and
    beta_i = l_i V^T.
    """
    rows = np.asarray(rows)
    A1, A2, A3, E = (inp[k][b, h] for k in ("A1", "A2", "A3", "E"))
    d = A1.shape[1]
    phi_r = rope_angles(np.asarray(inp["pos"])[rows], d, base)
    Qt_r = rope_rotate(np.asarray(A1, F64)[rows] @ np.asarray(inp["WQ"][h], F64), phi_r)
    Kt = rope_rotate(np.asarray(A2, F64) @ np.asarray(inp["WK"][h], F64),
                     rope_angles(inp["pos"], d, base))
    V = np.asarray(A3, F64) @ np.asarray(inp["WV"][h], F64)
    Z = (Qt_r @ Kt.T) / math.sqrt(d)
    if causal:
        j = np.arange(Kt.shape[0])
        Z = np.where(j[None, :] > rows[:, None], -np.inf, Z)
    s, lse = softmax_rows(Z)
    O = s @ V
    ell = O - np.asarray(E, F64)[rows]
    beta = ell @ V.T
    gamma = gamma_closed_form(s, beta)
    dQt = (gamma @ Kt) / math.sqrt(d)
    return {"O": O, "lse": lse, "dQt": dQt}


# ---------------------------------------------------------------------------------------
# One combined weight X (the page's own parameterisation)
# ---------------------------------------------------------------------------------------
# The page's problem takes the gradient with respect to one vectorised weight x and writes
# it as dLoss/dx = A~^T vec(gamma(x)) (Probleemdefinitie, Methodologie 1).  Reading: x is
# vec(X) for the score z_ij = a1_i^T R_{j-i} X a2_j / sqrt(d), where R_{j-i} rotates each
# pair (2k, 2k+1) by (pos_j - pos_i) * theta_k; a row of A~ is then the derivative of z_ij
# with respect to X, R_{j-i}^T a1_i a2_j^T / sqrt(d).  Since R_{j-i} = R_i^T R_j, the same
# scores come from Q~ = rot(A1) and K~ = rot(A2 X^T): the general problem with WQ = I and
# WK = X^T, whose dWK is dX^T.


def rotation_matrix(angles: np.ndarray) -> np.ndarray:
    """d x d block-diagonal counter-clockwise rotation by ``angles`` (one per pair)."""
    d = 2 * len(angles)
    R = np.zeros((d, d), F64)
    c, s = np.cos(angles), np.sin(angles)
    for k in range(len(angles)):
        R[2 * k, 2 * k], R[2 * k, 2 * k + 1] = c[k], -s[k]
        R[2 * k + 1, 2 * k], R[2 * k + 1, 2 * k + 1] = s[k], c[k]
    return R


def combined_weight_literal(A1, A2, A3, E, X, WV, pos, causal: bool, base: float):
    """Loss, dLoss/dX and dLoss/dWV of one instance with the page's closed form, literally:
    the scores from a1_i^T R_{j-i} X a2_j / sqrt(d), s, l, beta, gamma as in
    ``instance_forward_backward``, then vec(dX) = A~^T vec(gamma) with A~ built row by row
    (n^2 x d^2: tiny n only)."""
    A1, A2, A3, E, X, WV = (np.asarray(a, F64) for a in (A1, A2, A3, E, X, WV))
    n, d = A1.shape
    c = 1.0 / math.sqrt(d)
    theta = rope_theta(d, base)
    p = np.asarray(pos, F64)
    Rel = [[rotation_matrix((p[j] - p[i]) * theta) for j in range(n)] for i in range(n)]
    Z = np.empty((n, n), F64)
    for i in range(n):
        for j in range(n):
            Z[i, j] = c * A1[i] @ Rel[i][j] @ X @ A2[j]
    if causal:
        Z = np.where(np.arange(n)[None, :] > np.arange(n)[:, None], -np.inf, Z)
    s, _ = softmax_rows(Z)
    V = A3 @ WV
    O = s @ V
    ell = O - E
    loss = 0.5 * float(np.sum(ell * ell))
    beta = ell @ V.T
    gamma = gamma_closed_form(s, beta)
    A_tilde = np.empty((n * n, d * d), F64)
    for i in range(n):
        for j in range(n):
            A_tilde[i * n + j] = c * np.outer(Rel[i][j].T @ A1[i], A2[j]).reshape(-1)
    dX = (A_tilde.T @ gamma.reshape(-1)).reshape(d, d)
    dWV = A3.T @ (s.T @ ell)
    return {"loss": loss, "dX": dX, "dWV": dWV, "O": O}


def combined_weight_forward_backward(inp: Dict[str, np.ndarray], causal: bool, base: float):
    """All instances with one combined weight X [H][d][d] per head (``inp["X"]``) through
    the general problem with WQ = I and WK = X^T: loss, O, dX = dWK^T, dWV."""
    H, d = inp["X"].shape[0], inp["X"].shape[1]
    gen = dict(inp)
    gen["WQ"] = np.broadcast_to(np.eye(d), (H, d, d)).copy()
    gen["WK"] = np.ascontiguousarray(np.transpose(np.asarray(inp["X"], F64), (0, 2, 1)))
    r = forward_backward(gen, causal, base)
    return {"loss": r["loss"], "O": r["O"], "lse": r["lse"],
            "dX": np.transpose(r["dWK"], (0, 2, 1)), "dWV": r["dWV"]}


# ---------------------------------------------------------------------------------------
# The near-linear approximate backward: polynomial method + low rank
# ---------------------------------------------------------------------------------------
# "RoPE Attention kan bijna lineair worden getraind", Methodologie 2 (Low-Rank
# Benaderingsstrategie) and Resultaten (Theorem 5.7): under bounded entries the normalised
# softmax s(x) is approximated by low-rank factors U1 V1^T built with a polynomial method, the
# error term l(x) and beta(x) follow from it, gamma_1 = diag(s) beta is combined from the
# factors of s and beta with row-wise Kronecker products, and gamma_2 = s s^T beta from
# precomputed intermediates.  The pages name no degree, rank or construction.  Reading taken
# here: exp(z) on the bounded scores z is replaced by its degree-g Taylor polynomial
# P_g(z) = sum_{r <= g} z^r / r!, which factors exactly as P_g(q~_i . k~_j / sqrt(d)) =
# phi(q~_i) . phi(k~_j) with the tensor-power features of ``poly_features``; s~ is P_g(Z)
# normalised per row, and the gradient is the closed form with s~ in place of s:
# l = s~ V - E, beta = l V^T, gamma = s~ o (beta - rowsum(s~ o beta)), dQ~ = gamma K~ / sqrt(d),
# dK~ = gamma^T Q~ / sqrt(d), dV = s~^T l.  This is not the gradient of a loss built from s~
# (d s~ / dz is not softmax-shaped); it is the page's approximation of each term of the exact
# gradient.  The functions below evaluate that definition directly (quadratic in n) and give
# the low-rank factors; the near-linear evaluation order is the CUDA path's.


def poly_exp(z: np.ndarray, degree: int) -> np.ndarray:
    """P_g(z) = sum_{r=0}^{g} z^r / r!, the truncated Taylor series of exp."""
    z = np.asarray(z, F64)
    out = np.zeros_like(z)
    term = np.ones_like(z)
    for r in range(degree + 1):
        if r > 0:
            term = term * z / r
        out = out + term
    return out


def poly_features(X: np.ndarray, degree: int) -> np.ndarray:
    """Rows phi(x) with phi(q) . phi(k) = P_g(q . k / sqrt(d)): the tensor powers x^(x)r of
    every degree r <= g, each scaled by d^(-r/4) / sqrt(r!), side by side ([n][sum_r d^r])."""
    X = np.asarray(X, F64)
    n, d = X.shape
    parts = [np.ones((n, 1), F64)]
    cur = np.ones((n, 1), F64)
    for r in range(1, degree + 1):
        cur = np.einsum("ni,nj->nij", cur, X).reshape(n, -1)
        parts.append(cur * (d ** (-r / 4.0)) / math.sqrt(math.factorial(r)))
    return np.concatenate(parts, axis=1)


def approx_instance_forward_backward(A1, A2, A3, E, WQ, WK, WV, pos, causal: bool, base: float,
                                     degree: int, rb: int = 256) -> Dict[str, np.ndarray]:
    """One instance with the polynomial-kernel softmax s~ = P_g(Z) / rowsum (masked entries 0):
    O, the normaliser D, loss and the approximate gradient (see the section comment)."""
    n, d = np.shape(A1)
    c = 1.0 / math.sqrt(d)
    Qt, Kt, V, phi = _project(A1, A2, A3, WQ, WK, WV, pos, base)
    E = np.asarray(E, F64)
    O = np.empty((n, d), F64)
    Dn = np.empty(n, F64)
    dQt = np.empty((n, d), F64)
    dKt = np.zeros((n, d), F64)
    dV = np.zeros((n, d), F64)
    loss = 0.0
    for r0 in range(0, n, rb):
        r1 = min(n, r0 + rb)
        rows = np.arange(r0, r1)
        kend = r1 if causal else n
        Z = (Qt[rows] @ Kt[:kend].T) * c
        Pz = poly_exp(Z, degree)
        if causal:
            Pz = np.where(np.arange(kend)[None, :] > rows[:, None], 0.0, Pz)
        Dn[r0:r1] = np.sum(Pz, axis=1)
        s = Pz / Dn[r0:r1, None]                         # s~ (polynomial kernel, normalised)
        O[r0:r1] = s @ V[:kend]
        ell = O[r0:r1] - E[r0:r1]
        loss += 0.5 * float(np.sum(ell * ell))
        beta = ell @ V[:kend].T
        gamma = gamma_closed_form(s, beta)               # gamma_1 - gamma_2 with s~
        dQt[r0:r1] = (gamma @ Kt[:kend]) * c
        dKt[:kend] += (gamma.T @ Qt[r0:r1]) * c
        dV[:kend] += s.T @ ell
    dQ = rope_rotate(dQt, -phi)
    dK = rope_rotate(dKt, -phi)
    A1, A2, A3 = (np.asarray(a, F64) for a in (A1, A2, A3))
    return {"O": O, "D": Dn, "loss": loss, "dQt": dQt, "dKt": dKt, "dV": dV,
            "dWQ": A1.T @ dQ, "dWK": A2.T @ dK, "dWV": A3.T @ dV}


def approx_forward_backward(inp: Dict[str, np.ndarray], causal: bool, base: float, degree: int,
                            heads: Optional[Iterable[int]] = None) -> Dict[str, np.ndarray]:
    """All (b, h) instances (or those of ``heads``) of the approximate method: O, D, loss and
    dWQ, dWK, dWV summed over the batch (entries of heads not computed are NaN)."""
    B, H, n, d = inp["A1"].shape
    O = np.full((B, H, n, d), np.nan)
    Dn = np.full((B, H, n), np.nan)
    dW = {k: np.full((H, d, d), np.nan) for k in ("dWQ", "dWK", "dWV")}
    loss = 0.0
    for h in _heads(inp, heads):
        for k in dW:
            dW[k][h] = 0.0
        for b in range(B):
            r = approx_instance_forward_backward(inp["A1"][b, h], inp["A2"][b, h],
                                                 inp["A3"][b, h], inp["E"][b, h], inp["WQ"][h],
                                                 inp["WK"][h], inp["WV"][h], inp["pos"], causal,
                                                 base, degree)
            O[b, h], Dn[b, h] = r["O"], r["D"]
            loss += r["loss"]
            for k in dW:
                dW[k][h] += r[k]
    out = {"O": O, "D": Dn, "loss": loss}
    out.update(dW)
    return out

"""Seeded synthetic inputs for the exact RoPE-attention loss and its gradient.

This module only draws random numbers and rounds them to the I/O dtype.  It
holds none of the method's arithmetic (no projection, rotation, softmax or
gradient), so that the fp64 oracle and the CUDA path can both consume the same
inputs without sharing any computation.

Shapes (per the problem of "RoPE attention kan bijna lineair worden getraind",
section Probleemdefinitie / Methodologie 1: inputs, weight matrices, target):

    A1, A2, A3, E : [B][H][n][d]   (one independent instance per (b, h))
    WQ, WK, WV    : [H][d][d]      (per head, shared over the batch; Q = A1 @ WQ)
    pos           : [n] int32      (0 .. n-1)

Draw order from ``numpy.random.Generator(PCG64(seed))``: A1, A2, A3, E, WQ, WK,
WV, each in C order, drawn in float32, then rounded to nearest-even in the
I/O dtype.  Returned arrays are float32 numpy arrays whose values are exactly
representable in the I/O dtype.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Dict, Optional

import numpy as np

__all__ = ["Workload", "WORKLOADS", "make_inputs", "round_bf16", "flop_count",
           "workload_by_name"]


@dataclasses.dataclass(frozen=True)
class Workload:
    """One synthetic workload: sizes, dtypes, distributions and flags."""
    name: str
    B: int
    H: int
    n: int
    d: int
    dtype: str            # "f32" or "bf16": I/O dtype of A*, W*, E, O
    causal: bool
    rope_base: float
    a_dist: str           # "uniform" (U[-1,1]) or "normal" (N(0,1)) for A1, A2, A3
    e_dist: str           # same choices, for E
    bounded_scores: bool  # A1, A2 rows scaled so that |score| <= sqrt(ln n)
    seed: int = 0

    def with_sizes(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


# The five workloads: sizes and distributions as the task configuration states them.
WORKLOADS: Dict[str, Workload] = {
    "n128_d64_f32": Workload("n128_d64_f32", 1, 1, 128, 64, "f32", False, 1e4,
                             "uniform", "uniform", False),
    "b4_h16_n2048_d64_bf16": Workload("b4_h16_n2048_d64_bf16", 4, 16, 2048, 64, "bf16",
                                      False, 1e4, "normal", "normal", False),
    "b2_h32_n8192_d128_bf16_causal": Workload("b2_h32_n8192_d128_bf16_causal", 2, 32, 8192,
                                              128, "bf16", True, 1e4, "normal", "normal",
                                              False),
    "b1_h8_n32768_d128_bf16_causal_bounded": Workload(
        "b1_h8_n32768_d128_bf16_causal_bounded", 1, 8, 32768, 128, "bf16", True, 1e4,
        "normal", "uniform", True),
    "b1_h8_n131072_d128_bf16_causal_base5e5": Workload(
        "b1_h8_n131072_d128_bf16_causal_base5e5", 1, 8, 131072, 128, "bf16", True, 5e5,
        "normal", "normal", False),
}
WORKLOAD_ORDER = list(WORKLOADS)


def workload_by_name(name: str) -> Workload:
    return WORKLOADS[name]


def round_bf16(x: np.ndarray) -> np.ndarray:
    """Round float32 values to the nearest bfloat16 (ties to even); returns float32."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    u = x.view(np.uint32)
    lsb = (u >> np.uint32(16)) & np.uint32(1)
    r = (u + np.uint32(0x7FFF) + lsb) & np.uint32(0xFFFF0000)
    return r.view(np.float32)


def _to_io(x: np.ndarray, dtype: str) -> np.ndarray:
    if dtype == "f32":
        return np.ascontiguousarray(x, dtype=np.float32)
    if dtype == "bf16":
        return round_bf16(x)
    raise ValueError(f"unknown dtype {dtype!r}")


def _draw(rng: np.random.Generator, dist: str, shape) -> np.ndarray:
    if dist == "uniform":
        return (rng.random(shape, dtype=np.float32) * np.float32(2.0) - np.float32(1.0))
    if dist == "normal":
        return rng.standard_normal(shape, dtype=np.float32)
    raise ValueError(f"unknown distribution {dist!r}")


def score_bound(n: int) -> float:
    """Entry bound B = sqrt(ln n) of the bounded-entry regime (natural log)."""
    return math.sqrt(math.log(n)) if n > 1 else 0.0


def make_inputs(w: Workload, seed: Optional[int] = None) -> Dict[str, np.ndarray]:
    """Draw the inputs of workload ``w``.

    Returns a dict with A1, A2, A3, E ([B][H][n][d]), WQ, WK, WV ([H][d][d]) as float32
    arrays holding I/O-dtype values, and pos ([n] int32).
    """
    seed = w.seed if seed is None else seed
    rng = np.random.Generator(np.random.PCG64(seed))
    B, H, n, d = w.B, w.H, w.n, w.d
    act = (B, H, n, d)
    A1 = _draw(rng, w.a_dist, act)
    A2 = _draw(rng, w.a_dist, act)
    A3 = _draw(rng, w.a_dist, act)
    E = _draw(rng, w.e_dist, act)
    wstd = np.float32(1.0 / math.sqrt(d))       # N(0, 1/d): standard deviation 1/sqrt(d)
    WQ = rng.standard_normal((H, d, d), dtype=np.float32) * wstd
    WK = rng.standard_normal((H, d, d), dtype=np.float32) * wstd
    WV = rng.standard_normal((H, d, d), dtype=np.float32) * wstd
    WQ, WK, WV = (_to_io(x, w.dtype) for x in (WQ, WK, WV))
    if w.bounded_scores:
        A1, A2 = _bound_rows(A1, A2, WQ, WK, n, d)
    out = {
        "A1": _to_io(A1, w.dtype), "A2": _to_io(A2, w.dtype), "A3": _to_io(A3, w.dtype),
        "E": _to_io(E, w.dtype), "WQ": WQ, "WK": WK, "WV": WV,
        "pos": np.arange(n, dtype=np.int32),
    }
    return out


def _bound_rows(A1, A2, WQ, WK, n, d):
    """Scale rows of A1 and A2 so every score |q_i . k_j| / sqrt(d) stays below sqrt(ln n).

    A rotation preserves norms and |q.k| <= |q| |k|, and |a W| <= |a| * ||W||_2, so a row
    norm of r / ||W||_2 gives |q| <= r.  With r^2 = B sqrt(d) (1 - 2^-6) the bound holds
    with room for the relative 2^-8 rounding of each I/O-dtype row after scaling.
    Only matrix norms are taken here; no projection is formed.
    """
    Bnd = score_bound(n)
    r = math.sqrt(Bnd * math.sqrt(d) * (1.0 - 2.0 ** -6))
    sq = np.array([np.linalg.norm(WQ[h].astype(np.float64), 2) for h in range(WQ.shape[0])])
    sk = np.array([np.linalg.norm(WK[h].astype(np.float64), 2) for h in range(WK.shape[0])])

    def scale(A, s):
        norms = np.sqrt(np.sum(A.astype(np.float64) ** 2, axis=-1, keepdims=True))
        norms = np.maximum(norms, 1e-30)
        tgt = (r / s)[None, :, None, None]
        return (A.astype(np.float64) * (tgt / norms)).astype(np.float32)

    return scale(A1, sq), scale(A2, sk)


def pair_count(n: int, causal: bool) -> int:
    """Number of (query, key) pairs the attention touches: n^2, or n(n+1)/2 if causal."""
    return n * (n + 1) // 2 if causal else n * n


def flop_count(w: Workload) -> float:
    """Algorithmic FLOPs of one forward+backward pass.

    Per (b, h): 4 d P in the forward (scores and s V), 10 d P in the backward (recomputed
    scores, beta = l V^T, dV, dK, dQ), plus 12 n d^2 for the three projections and the
    three weight-gradient contractions.  P = pair_count(n, causal).
    """
    P = pair_count(w.n, w.causal)
    return float(w.B * w.H) * (14.0 * w.d * P + 12.0 * w.n * w.d * w.d)

"""Parity of the CUDA path (through the C ABI) with the fp64 oracle on the same seeded inputs.

Bar (relative Frobenius error ||x - x*|| / ||x*||) on O, Loss, dWQ, dWK, dWV:
  1e-4 for fp32 I/O, 2e-2 for bf16 I/O with fp32 accumulation.  lse is compared too
  (absolute error, since it is a logarithm).
"""
import numpy as np
import pytest
import torch

import oracle
from workloads import WORKLOADS, make_inputs

pytestmark = pytest.mark.gpu

TOL = {"f32": 1e-4, "bf16": 2e-2}
LSE_ATOL = {"f32": 1e-4, "bf16": 2e-2}
TORCH_DT = {"f32": torch.float32, "bf16": torch.bfloat16}


def rel(a, b):
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    nb = np.linalg.norm(b)
    return float(np.linalg.norm(a - b) / (nb if nb > 0 else 1.0))


def to_device(inp, dtype):
    dt = TORCH_DT[dtype]
    t = {k: torch.from_numpy(np.ascontiguousarray(inp[k])).to("cuda", dt)
         for k in ("A1", "A2", "A3", "E", "WQ", "WK", "WV")}
    t["pos"] = torch.from_numpy(np.ascontiguousarray(inp["pos"], dtype=np.int32)).cuda()
    return t


def run_gpu(cuda_lib, w, inp, holds=True, check_status=True):
    t = to_device(inp, w.dtype)
    m = cuda_lib.RopeAttention(t["A1"], t["A2"], t["A3"], t["WQ"], t["WK"], t["WV"], t["E"],
                               t["pos"], w.causal, w.rope_base)
    m.forward()
    if holds:
        m.backward(True)
    else:
        m.ws.fill_(0xFF)   # nothing of the forward survives: the backward recomputes
        m.backward(False)
    torch.cuda.synchronize()
    if check_status:
        assert cuda_lib.last_error() == cuda_lib.RA_OK
    return {"O": m.O.float().cpu().numpy(), "lse": m.lse.cpu().numpy(),
            "loss": float(m.loss.item()), "dWQ": m.dWQ.cpu().numpy(),
            "dWK": m.dWK.cpu().numpy(), "dWV": m.dWV.cpu().numpy()}


def grad_rel(got, ref, scale):
    """Relative error; a reference that is exactly zero (n = 1: dWQ = dWK = 0 because
    gamma = s o (beta - s^T beta) vanishes when s = 1) is measured against `scale`, the
    norm of the whole weight gradient."""
    nb = np.linalg.norm(np.asarray(ref, np.float64))
    if nb == 0.0:
        return float(np.linalg.norm(np.asarray(got, np.float64)) / scale)
    return rel(got, ref)


def compare(w, got, ref, heads=None):
    tol = TOL[w.dtype]
    hs = slice(None) if heads is None else list(heads)
    scale = max(1e-300, float(np.sqrt(sum(np.sum(np.asarray(ref[k][hs], np.float64) ** 2)
                                          for k in ("dWQ", "dWK", "dWV")))))
    errs = {
        "O": rel(got["O"][:, hs], ref["O"][:, hs]),
        "dWQ": grad_rel(got["dWQ"][hs], ref["dWQ"][hs], scale),
        "dWK": grad_rel(got["dWK"][hs], ref["dWK"][hs], scale),
        "dWV": grad_rel(got["dWV"][hs], ref["dWV"][hs], scale),
    }
    if heads is None:
        errs["loss"] = abs(got["loss"] - ref["loss"]) / abs(ref["loss"])
    lse_err = float(np.max(np.abs(got["lse"][:, hs] - ref["lse"][:, hs])))
    bad = {k: v for k, v in errs.items() if not v <= tol}
    assert not bad, f"{w.name}: errors above {tol}: {errs}"
    assert lse_err <= LSE_ATOL[w.dtype], f"lse max abs error {lse_err}"
    return errs


def small(dtype, n, d, causal, B=2, H=3, base=1e4, dist="normal"):
    src = WORKLOADS["n128_d64_f32"] if dtype == "f32" else WORKLOADS["b4_h16_n2048_d64_bf16"]
    return src.with_sizes(name=f"{dtype}_n{n}_d{d}_c{int(causal)}", B=B, H=H, n=n, d=d,
                          causal=causal, rope_base=base, a_dist=dist, e_dist=dist)


def test_n128_d64_f32_workload(cuda_lib):
    """The fp32 parity workload exactly as specified (seed 0)."""
    w = WORKLOADS["n128_d64_f32"]
    inp = make_inputs(w)
    got = run_gpu(cuda_lib, w, inp)
    ref = oracle.forward_backward(inp, w.causal, w.rope_base)
    compare(w, got, ref)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("n", [1, 2, 127, 128, 129, 200, 385])
@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("causal", [False, True])
def test_boundary_shapes(cuda_lib, dtype, n, d, causal):
    w = small(dtype, n, d, causal)
    inp = make_inputs(w, seed=n * 7 + d)
    got = run_gpu(cuda_lib, w, inp)
    ref = oracle.forward_backward(inp, w.causal, w.rope_base)
    compare(w, got, ref)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_recompute_equals_reuse(cuda_lib, dtype):
    w = small(dtype, 300, 64, True)
    inp = make_inputs(w, seed=5)
    a = run_gpu(cuda_lib, w, inp, holds=True)
    b = run_gpu(cuda_lib, w, inp, holds=False)
    ref = oracle.forward_backward(inp, w.causal, w.rope_base)
    compare(w, a, ref)
    compare(w, b, ref)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_shifted_and_irregular_positions(cuda_lib, dtype):
    w = small(dtype, 160, 128, False, base=5e5)
    inp = make_inputs(w, seed=6)
    rng = np.random.default_rng(0)
    inp["pos"] = (np.sort(rng.choice(200000, size=w.n, replace=False)) + 1000).astype(np.int32)
    got = run_gpu(cuda_lib, w, inp)
    ref = oracle.forward_backward(inp, w.causal, w.rope_base)
    compare(w, got, ref)


def test_forward_is_bitwise_repeatable(cuda_lib):
    w = small("bf16", 256, 128, True)
    inp = make_inputs(w, seed=9)
    a = run_gpu(cuda_lib, w, inp)
    b = run_gpu(cuda_lib, w, inp)
    assert np.array_equal(a["O"], b["O"]) and np.array_equal(a["lse"], b["lse"])


def test_bounded_regime_small(cuda_lib):
    w = WORKLOADS["b1_h8_n32768_d128_bf16_causal_bounded"].with_sizes(n=1024, H=2)
    inp = make_inputs(w)
    got = run_gpu(cuda_lib, w, inp)
    ref = oracle.forward_backward(inp, w.causal, w.rope_base)
    compare(w, got, ref)


# ---------------------------------------------------------------------------------------
# full-size workloads: sampled heads (every (b, h) of a head, for the weight gradients)
# and sampled query rows (O and lse, from the oracle row by row)
# ---------------------------------------------------------------------------------------

def _sampled_rows_check(w, inp, got, rows_per_inst=6, insts=4, seed=0):
    rng = np.random.default_rng(seed)
    worst_o, worst_l = 0.0, 0.0
    for _ in range(insts):
        b, h = int(rng.integers(w.B)), int(rng.integers(w.H))
        rows = np.unique(np.concatenate([[0, w.n - 1], rng.integers(0, w.n, rows_per_inst)]))
        ref = oracle.forward_rows(inp, b, h, rows, w.causal, w.rope_base)
        worst_o = max(worst_o, rel(got["O"][b, h, rows], ref["O"]))
        worst_l = max(worst_l, float(np.max(np.abs(got["lse"][b, h, rows] - ref["lse"]))))
    assert worst_o <= TOL[w.dtype], worst_o
    assert worst_l <= LSE_ATOL[w.dtype], worst_l


@pytest.mark.parametrize("name,heads", [
    ("b4_h16_n2048_d64_bf16", [0, 11]),
    ("b2_h32_n8192_d128_bf16_causal", [5]),
])
def test_full_size_sampled_heads(cuda_lib, name, heads):
    w = WORKLOADS[name]
    inp = make_inputs(w)
    got = run_gpu(cuda_lib, w, inp)
    ref = oracle.forward_backward(inp, w.causal, w.rope_base, heads=heads)
    compare(w, got, ref, heads=heads)
    _sampled_rows_check(w, inp, got)


@pytest.mark.slow
def test_partial_scheduling_groups(cuda_lib):
    """Five heads at n = 32768, d = 128: the attention kernels group heads whose re-read
    tensors fit in 64 MB of L2 (forward 4 heads, backward 2), so the last group of each grid
    holds fewer heads than the others and its extra CTAs leave at once.  Head 4 sits in the
    partial group of both kernels, head 0 in a full one."""
    w = WORKLOADS["b2_h32_n8192_d128_bf16_causal"].with_sizes(name="b1_h5_n32768_d128_bf16_causal",
                                                             B=1, H=5, n=32768)
    inp = make_inputs(w)
    got = run_gpu(cuda_lib, w, inp)
    ref = oracle.forward_backward(inp, w.causal, w.rope_base, heads=[0, 4])
    compare(w, got, ref, heads=[0, 4])
    _sampled_rows_check(w, inp, got, rows_per_inst=4, insts=3)

"""Parity of the input gradients dA1 = rot^-1(dQ~) WQ^T, dA2 = rot^-1(dK~) WK^T,
dA3 = dV WV^T (rope_attn_loss_bwd_inputs) with the fp64 oracle, same bar as the weight
gradients: relative Frobenius error <= 1e-4 (fp32 I/O) / 2e-2 (bf16 I/O)."""
import numpy as np
import pytest
import torch

import oracle
from test_parity_gpu import TOL, grad_rel, rel, small, to_device
from workloads import WORKLOADS, make_inputs

pytestmark = pytest.mark.gpu

DA = ("dA1", "dA2", "dA3")


def run_gpu_inputs(cuda_lib, w, inp, holds=True):
    t = to_device(inp, w.dtype)
    m = cuda_lib.RopeAttention(t["A1"], t["A2"], t["A3"], t["WQ"], t["WK"], t["WV"], t["E"],
                               t["pos"], w.causal, w.rope_base)
    m.forward()
    if not holds:
        m.ws.fill_(0xFF)
    m.backward_inputs(holds)
    torch.cuda.synchronize()
    assert cuda_lib.last_error() == cuda_lib.RA_OK
    out = {k: getattr(m, k).float().cpu().numpy() for k in DA}
    out.update({k: getattr(m, k).cpu().numpy() for k in ("dWQ", "dWK", "dWV")})
    out["loss"] = float(m.loss.item())
    return out


def compare_inputs(w, got, ref, heads=None):
    hs = slice(None) if heads is None else list(heads)
    scale = max(1e-300, float(np.sqrt(sum(np.sum(np.asarray(ref[k][:, hs], np.float64) ** 2)
                                          for k in DA))))
    errs = {k: grad_rel(got[k][:, hs], ref[k][:, hs], scale) for k in DA}
    for k in ("dWQ", "dWK", "dWV"):
        errs[k] = rel(got[k][hs], ref[k][hs]) if np.linalg.norm(ref[k][hs]) > 0 else 0.0
    bad = {k: v for k, v in errs.items() if not v <= TOL[w.dtype]}
    assert not bad, f"{w.name}: errors above {TOL[w.dtype]}: {errs}"
    return errs


def test_input_grads_f32_workload(cuda_lib):
    w = WORKLOADS["n128_d64_f32"]
    inp = make_inputs(w)
    got = run_gpu_inputs(cuda_lib, w, inp)
    compare_inputs(w, got, oracle.forward_backward(inp, w.causal, w.rope_base))


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("n", [1, 129, 385])
@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("causal", [False, True])
def test_input_grads_boundary_shapes(cuda_lib, dtype, n, d, causal):
    w = small(dtype, n, d, causal)
    inp = make_inputs(w, seed=n * 5 + d)
    got = run_gpu_inputs(cuda_lib, w, inp)
    compare_inputs(w, got, oracle.forward_backward(inp, w.causal, w.rope_base))


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_input_grads_recompute_and_reuse(cuda_lib, dtype):
    """Both backward modes (workspace reused from the forward, or recomputed) meet the bar.
    They need not agree bit for bit: dQ~ is summed over key tiles by reductions whose order
    between CTAs is not fixed."""
    w = small(dtype, 200, 64, True)
    inp = make_inputs(w, seed=3)
    ref = oracle.forward_backward(inp, w.causal, w.rope_base)
    compare_inputs(w, run_gpu_inputs(cuda_lib, w, inp, holds=True), ref)
    compare_inputs(w, run_gpu_inputs(cuda_lib, w, inp, holds=False), ref)


def test_input_grads_leave_weight_grads_unchanged(cuda_lib):
    """The extra products run after the weight gradients and do not disturb them."""
    w = small("bf16", 385, 128, True)
    inp = make_inputs(w, seed=9)
    t = to_device(inp, w.dtype)
    m = cuda_lib.RopeAttention(t["A1"], t["A2"], t["A3"], t["WQ"], t["WK"], t["WV"], t["E"],
                               t["pos"], w.causal, w.rope_base)
    m.forward()
    m.backward(True)
    ref = {k: getattr(m, k).clone() for k in ("dWQ", "dWK", "dWV")}
    m.forward()
    m.backward_inputs(True)
    torch.cuda.synchronize()
    for k in ref:
        assert torch.equal(ref[k], getattr(m, k)), k


def test_input_grads_full_size_sampled_head(cuda_lib):
    """B=2 H=32 n=8192 d=128 causal: every (b, h) of one head against the oracle."""
    w = WORKLOADS["b2_h32_n8192_d128_bf16_causal"]
    inp = make_inputs(w)
    got = run_gpu_inputs(cuda_lib, w, inp)
    ref = oracle.forward_backward(inp, w.causal, w.rope_base, heads=[7])
    compare_inputs(w, got, ref, heads=[7])

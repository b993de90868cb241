"""The page's own parameterisation on the GPU: one combined weight X per head
(rope_attn_combined_weights + the general forward / backward + rope_attn_combined_grad)
against the oracle.  Same bars as the weight gradients (1e-4 fp32, 2e-2 bf16)."""
import math

import numpy as np
import pytest
import torch

import oracle
from test_parity_gpu import TOL, TORCH_DT, rel, small
from workloads import make_inputs

pytestmark = pytest.mark.gpu


def with_x(inp, seed):
    rng = np.random.default_rng(seed)
    H, d = inp["WQ"].shape[0], inp["WQ"].shape[1]
    out = dict(inp)
    out["X"] = (rng.standard_normal((H, d, d)) / math.sqrt(d)).astype(np.float32)
    return out


def run_x(cuda_lib, w, inp):
    dt = TORCH_DT[w.dtype]
    t = {k: torch.from_numpy(np.ascontiguousarray(inp[k])).to("cuda", dt)
         for k in ("A1", "A2", "A3", "E", "WV", "X")}
    # the oracle sees the same rounded X
    xr = t["X"].float().cpu().numpy().astype(np.float64)
    pos = torch.from_numpy(np.ascontiguousarray(inp["pos"], dtype=np.int32)).cuda()
    m = cuda_lib.RopeAttentionX(t["A1"], t["A2"], t["A3"], t["X"], t["WV"], t["E"], pos,
                                w.causal, w.rope_base)
    loss, dX, dWV = m.step()
    torch.cuda.synchronize()
    assert cuda_lib.last_error() == cuda_lib.RA_OK
    return {"loss": float(loss.item()), "dX": dX.cpu().numpy(), "dWV": dWV.cpu().numpy(),
            "O": m.attn.O.float().cpu().numpy()}, xr


@pytest.mark.parametrize("dtype,n,d,causal", [
    ("f32", 128, 64, False), ("f32", 129, 128, True),
    ("bf16", 385, 64, True), ("bf16", 200, 128, False),
])
def test_combined_weight_matches_oracle(cuda_lib, dtype, n, d, causal):
    w = small(dtype, n, d, causal)
    inp = with_x(make_inputs(w, seed=n + d), seed=n)
    got, xr = run_x(cuda_lib, w, inp)
    inp64 = dict(inp)
    inp64["X"] = xr
    ref = oracle.combined_weight_forward_backward(inp64, w.causal, w.rope_base)
    errs = {"O": rel(got["O"], ref["O"]), "dX": rel(got["dX"], ref["dX"]),
            "dWV": rel(got["dWV"], ref["dWV"]),
            "loss": abs(got["loss"] - ref["loss"]) / abs(ref["loss"])}
    bad = {k: v for k, v in errs.items() if not v <= TOL[dtype]}
    assert not bad, errs


def test_combined_weight_matches_literal_closed_form(cuda_lib):
    """Tiny instance (n = 6, d = 64) against A~^T vec(gamma) built literally, fp32."""
    w = small("f32", 6, 64, True, B=1, H=1, base=10.0)
    inp = with_x(make_inputs(w, seed=1), seed=2)
    got, xr = run_x(cuda_lib, w, inp)
    lit = oracle.combined_weight_literal(inp["A1"][0, 0], inp["A2"][0, 0], inp["A3"][0, 0],
                                         inp["E"][0, 0], xr[0], inp["WV"][0], inp["pos"],
                                         w.causal, w.rope_base)
    assert rel(got["dX"][0], lit["dX"]) <= 1e-4
    assert rel(got["dWV"][0], lit["dWV"]) <= 1e-4
    assert abs(got["loss"] - lit["loss"]) / abs(lit["loss"]) <= 1e-4

"""rope_attn_step: the forward with the loss and the weight-gradient backward in one call.

It must give what rope_attn_fwd followed by rope_attn_loss_bwd(ws_holds_fwd = 1) give: O, lse
and the loss bit for bit, and (in the deterministic mode, where the backward's sums have a fixed
order) the weight gradients bit for bit; and match the fp64 oracle at the parity bars.  The
workspace header it leaves lets a following backward reuse the intermediates.
"""
import numpy as np
import pytest
import torch

import oracle
from test_parity_gpu import TOL, grad_rel, rel, small, to_device
from workloads import make_inputs

pytestmark = pytest.mark.gpu

W = ("dWQ", "dWK", "dWV")


def _model(cuda_lib, w, t):
    return cuda_lib.RopeAttention(t["A1"], t["A2"], t["A3"], t["WQ"], t["WK"], t["WV"], t["E"],
                                  t["pos"], w.causal, w.rope_base, deterministic=True)


def _bits(x):
    return x.view(torch.int16) if x.dtype == torch.bfloat16 else x.view(torch.int32)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("n,d,causal", [(1, 64, True), (129, 128, True), (385, 64, False),
                                        (600, 128, False)])
def test_step_equals_forward_then_backward(cuda_lib, dtype, n, d, causal):
    w = small(dtype, n, d, causal, B=2, H=2)
    inp = make_inputs(w, seed=17 + n)
    t = to_device(inp, dtype)
    a = _model(cuda_lib, w, t)
    a.step()
    b = _model(cuda_lib, w, t)
    b.forward()
    b.backward(True)
    torch.cuda.synchronize()
    assert cuda_lib.last_error() == cuda_lib.RA_OK
    for k in ("O", "lse", "loss") + W:
        assert torch.equal(_bits(getattr(a, k)), _bits(getattr(b, k))), k
    ref = oracle.forward_backward(inp, w.causal, w.rope_base)
    scale = float(np.linalg.norm(ref["dWV"]))
    errs = {"O": rel(a.O.float().cpu().numpy(), ref["O"]),
            "loss": abs(float(a.loss.item()) - ref["loss"]) / abs(ref["loss"])}
    for k in W:
        errs[k] = grad_rel(getattr(a, k).cpu().numpy(), ref[k], scale)
    bad = {k: v for k, v in errs.items() if not v <= TOL[dtype]}
    assert not bad, errs
    # the header the step leaves: a backward that reuses the workspace gives the same gradients
    got = {k: getattr(a, k).clone() for k in W}
    a.backward(True)
    torch.cuda.synchronize()
    assert cuda_lib.last_error() == cuda_lib.RA_OK
    for k in W:
        assert torch.equal(_bits(getattr(a, k)), _bits(got[k])), k

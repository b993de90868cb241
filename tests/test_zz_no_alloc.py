"""rope_attn_step_noalloc: the step for callers that cannot allocate device memory.

Some callers cannot call cudaMalloc (for instance code that must not take the device-wide
synchronisation an allocation can cause, or that runs inside a component whose device memory
belongs to someone else).  The library gives them one entry point that runs the whole step on
a static scratch array inside the library instead of a caller-owned workspace.  These tests
call it through the C ABI and check its outputs against the workspace-based entry points
(rope_attn_fwd + rope_attn_loss_bwd) on two calls in a row.  Before the first checked call the
scratch is left dirty by a step on another problem (other inputs, other length, the other
causal flag), so state that leaked from one call into the next would show.  The forward runs
the same kernels on the same inputs, so O, lse and the loss must agree bit for bit; the weight
gradients may differ only by the free order of the backward's fp32 reductions (and the bf16
rounding that follows), far below the parity bars.

This file is named so that pytest collects it last.
"""
import numpy as np
import pytest
import torch

from workloads import WORKLOADS, make_inputs

pytestmark = pytest.mark.gpu

# weight gradients: reduction order only (the parity bars are 1e-4 and 2e-2)
DW_TOL = {"f32": 1e-5, "bf16": 2e-3}


def _rel(a, b):
    a = a.double().cpu().numpy()
    b = b.double().cpu().numpy()
    nb = np.linalg.norm(b)
    return float(np.linalg.norm(a - b) / (nb if nb > 0 else 1.0))


CASES = [
    WORKLOADS["b2_h32_n8192_d128_bf16_causal"].with_sizes(name="bf16_small", B=1, H=2, n=1000),
    WORKLOADS["b4_h16_n2048_d64_bf16"].with_sizes(name="bf16_d64", B=2, H=2, n=300),
    WORKLOADS["n128_d64_f32"],
]


@pytest.mark.parametrize("w", CASES, ids=lambda w: w.name)
def test_noalloc_step_matches_workspace_entry_points(cuda_lib, w):
    ra = cuda_lib
    inp = make_inputs(w, seed=3)
    dt = torch.bfloat16 if w.dtype == "bf16" else torch.float32
    t = {k: torch.from_numpy(inp[k]).to("cuda", dt) for k in ("A1", "A2", "A3", "E", "WQ", "WK", "WV")}
    pos = torch.from_numpy(inp["pos"]).cuda()
    ref = ra.RopeAttention(t["A1"], t["A2"], t["A3"], t["WQ"], t["WK"], t["WV"], t["E"], pos,
                           w.causal, w.rope_base)
    assert ra.workspace_bytes(ref.prob) <= ra.NOALLOC_SCRATCH_BYTES
    ref.step()
    torch.cuda.synchronize()
    assert ra.last_error() == ra.RA_OK
    # leave the scratch dirty: a step on other inputs, another length, the other causal flag
    wd = w.with_sizes(n=w.n // 2 + 37, causal=not w.causal)
    inpd = make_inputs(wd, seed=11)
    td = {k: torch.from_numpy(inpd[k]).to("cuda", dt) for k in t}
    dirty = ra.RopeAttention(td["A1"], td["A2"], td["A3"], td["WQ"], td["WK"], td["WV"],
                             td["E"], torch.from_numpy(inpd["pos"]).cuda(), wd.causal,
                             wd.rope_base)
    ra.step_noalloc(dirty.prob, dirty.O, dirty.lse, dirty.loss, dirty.dWQ, dirty.dWK, dirty.dWV)
    torch.cuda.synchronize()
    assert ra.last_error() == ra.RA_OK
    tol = DW_TOL[w.dtype]
    for call in range(2):
        O = torch.full_like(ref.O, float("nan"))
        lse = torch.full_like(ref.lse, float("nan"))
        loss = torch.full_like(ref.loss, float("nan"))
        dW = [torch.full_like(ref.dWQ, float("nan")) for _ in range(3)]
        ra.step_noalloc(ref.prob, O, lse, loss, *dW)
        torch.cuda.synchronize()
        assert ra.last_error() == ra.RA_OK
        assert torch.equal(O, ref.O), f"call {call}: O differs"
        assert torch.equal(lse, ref.lse), f"call {call}: lse differs"
        assert torch.equal(loss, ref.loss), f"call {call}: loss differs"
        errs = {"dWQ": _rel(dW[0], ref.dWQ), "dWK": _rel(dW[1], ref.dWK),
                "dWV": _rel(dW[2], ref.dWV)}
        bad = {k: v for k, v in errs.items() if not v <= tol}
        assert not bad, f"call {call}: {errs}"


def test_noalloc_step_rejects_problems_beyond_the_scratch(cuda_lib):
    ra = cuda_lib
    w = WORKLOADS["b2_h32_n8192_d128_bf16_causal"]
    z = torch.zeros(16, dtype=torch.bfloat16, device="cuda")
    prob = ra.Problem(w.B, w.H, w.n, w.d, ra.RA_BF16, 1, 1e4, None, *([z.data_ptr()] * 7))
    assert ra.workspace_bytes(prob) > ra.NOALLOC_SCRATCH_BYTES
    out = torch.zeros(16, dtype=torch.float32, device="cuda")
    with pytest.raises(ra.RopeAttnError) as e:
        ra.step_noalloc(prob, z, out, out, out, out, out)
    assert e.value.status == ra.RA_ERR_WORKSPACE

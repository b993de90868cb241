"""The backward's reuse of a workspace is decided on the device, from the workspace header.

rope_attn_loss_bwd(..., ws_holds_fwd = 1) may be handed a workspace that does not hold this
problem's intermediates: one of another problem, one whose forward ran without a target, one
that was never written, or one whose dQ~ accumulator an earlier backward already used.  In
every case the header (written by the last kernel of each forward and backward call) tells the
recomputation kernels to run, so the gradients still match the fp64 oracle.
"""
import pytest
import torch

import oracle
from test_parity_gpu import TOL, rel, small, to_device
from workloads import make_inputs

pytestmark = pytest.mark.gpu


def _problem(ra, t, w, with_e=True):
    return ra.make_problem(t["A1"], t["A2"], t["A3"], t["WQ"], t["WK"], t["WV"],
                           t["E"] if with_e else None, t["pos"], w.causal, w.rope_base)


def _outputs(t):
    B, H, n, d = t["A1"].shape
    f32 = dict(dtype=torch.float32, device="cuda")
    return {"O": torch.empty_like(t["A1"]), "lse": torch.empty((B, H, n), **f32),
            "loss": torch.zeros((), **f32), "dWQ": torch.empty((H, d, d), **f32),
            "dWK": torch.empty((H, d, d), **f32), "dWV": torch.empty((H, d, d), **f32)}


def _ws(ra, prob):
    return torch.empty(ra.workspace_bytes(prob), dtype=torch.uint8, device="cuda")


def _bwd(ra, prob, o, ws):
    ra.loss_bwd(prob, o["O"], o["lse"], o["loss"], o["dWQ"], o["dWK"], o["dWV"], ws, True)
    torch.cuda.synchronize()
    assert ra.last_error() == ra.RA_OK


def _check(w, o, ref):
    tol = TOL[w.dtype]
    errs = {k: rel(o[k].cpu().numpy(), ref[k]) for k in ("dWQ", "dWK", "dWV")}
    errs["loss"] = abs(float(o["loss"].item()) - ref["loss"]) / abs(ref["loss"])
    bad = {k: v for k, v in errs.items() if not v <= tol}
    assert not bad, errs


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("d", [64, 128])
def test_workspace_of_another_problem_is_recomputed(cuda_lib, dtype, d):
    ra = cuda_lib
    w = small(dtype, 333, d, True, B=1, H=2)
    t1 = to_device(make_inputs(w, seed=21), dtype)
    inp2 = make_inputs(w, seed=22)
    t2 = to_device(inp2, dtype)
    p1, p2 = _problem(ra, t1, w), _problem(ra, t2, w)
    ws = _ws(ra, p1)
    o1, o2 = _outputs(t1), _outputs(t2)
    ra.fwd(p1, o1["O"], o1["lse"], o1["loss"], ws)          # ws now holds problem 1
    ws2 = _ws(ra, p2)
    ra.fwd(p2, o2["O"], o2["lse"], None, ws2)               # O, lse of problem 2
    _bwd(ra, p2, o2, ws)                                    # claims reuse of problem 1's ws
    _check(w, o2, oracle.forward_backward(inp2, w.causal, w.rope_base))


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_forward_without_target_leaves_nothing_to_reuse(cuda_lib, dtype):
    ra = cuda_lib
    w = small(dtype, 257, 64, False, B=2, H=2)
    inp = make_inputs(w, seed=23)
    t = to_device(inp, dtype)
    p, p_noe = _problem(ra, t, w), _problem(ra, t, w, with_e=False)
    ws = _ws(ra, p)
    o = _outputs(t)
    ra.fwd(p, o["O"], o["lse"], None, ws)        # a full forward: ws holds problem p ...
    ra.fwd(p_noe, o["O"], o["lse"], None, ws)    # ... then one without a target overwrites it
    _bwd(ra, p, o, ws)
    _check(w, o, oracle.forward_backward(inp, w.causal, w.rope_base))


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_never_written_workspace_is_recomputed(cuda_lib, dtype):
    ra = cuda_lib
    w = small(dtype, 200, 128, True, B=1, H=3)
    inp = make_inputs(w, seed=24)
    t = to_device(inp, dtype)
    p = _problem(ra, t, w)
    o = _outputs(t)
    ws_f = _ws(ra, p)
    ra.fwd(p, o["O"], o["lse"], None, ws_f)
    for fill in (0x00, 0xFF, 0x5A):
        ws = _ws(ra, p)
        ws.fill_(fill)
        _bwd(ra, p, o, ws)
        _check(w, o, oracle.forward_backward(inp, w.causal, w.rope_base))


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_second_backward_on_the_same_workspace(cuda_lib, dtype):
    """The first backward consumes the zeroed dQ~ accumulator the forward left; the second,
    on the same workspace, must zero it again (and may reuse everything else)."""
    ra = cuda_lib
    w = small(dtype, 300, 128, True, B=2, H=2)
    inp = make_inputs(w, seed=25)
    t = to_device(inp, dtype)
    p = _problem(ra, t, w)
    ws = _ws(ra, p)
    o = _outputs(t)
    ra.fwd(p, o["O"], o["lse"], None, ws)
    _bwd(ra, p, o, ws)
    first = {k: o[k].clone() for k in ("dWQ", "dWK", "dWV", "loss")}
    _bwd(ra, p, o, ws)
    ref = oracle.forward_backward(inp, w.causal, w.rope_base)
    _check(w, o, ref)
    assert torch.equal(first["loss"], o["loss"])
    # equal up to the free order of the fp32 reductions (and the bf16 rounding after them)
    tol = {"f32": 1e-5, "bf16": 2e-3}[w.dtype]
    for k in ("dWQ", "dWK", "dWV"):
        assert rel(o[k].cpu().numpy(), first[k].cpu().numpy()) <= tol, k

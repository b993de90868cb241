"""Guard regions around every output and the workspace: nothing is written past its end.

Every buffer the library writes (O, lse, the loss, dWQ, dWK, dWV, dA1..dA3 and the workspace)
is carved out of a larger allocation whose 4 KiB before and after hold a NaN bit pattern.
After a forward and a backward with input gradients, at lengths that leave ragged tiles
(n = 1, 129, 385), both dtypes and both head dimensions, the guards must be unchanged bit for
bit, and the results must still match the oracle.  (A memory checker is not available on the
GPU pool; this is the substitute for the writes it would catch.)
"""
import pytest
import torch

import oracle
from test_parity_gpu import TOL, rel, small, to_device
from workloads import make_inputs

pytestmark = pytest.mark.gpu

GUARD_BYTES = 4096
PATTERN = {1: 0x7D, 2: 0x7FDE, 4: 0x7FC0DEAD}   # NaN bit patterns of each element size
INT_VIEW = {1: torch.uint8, 2: torch.int16, 4: torch.int32}


class Guarded:
    """A tensor of `shape` and `dtype` between two guard regions of GUARD_BYTES each."""

    def __init__(self, shape, dtype):
        es = torch.empty((), dtype=dtype).element_size()
        self.g = GUARD_BYTES // es
        numel = 1
        for s in shape:
            numel *= s
        self.full = torch.empty(numel + 2 * self.g, dtype=dtype, device="cuda")
        self.ints = self.full.view(INT_VIEW[es])
        self.ints.fill_(PATTERN[es])
        self.pattern = int(self.ints[0].item())
        self.t = self.full[self.g:self.g + numel].view(shape)

    def intact(self):
        lo, hi = self.ints[:self.g], self.ints[-self.g:]
        return bool(torch.all(lo == self.pattern).item() and torch.all(hi == self.pattern).item())


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("n", [1, 129, 385])
@pytest.mark.parametrize("d", [64, 128])
def test_no_write_past_any_buffer(cuda_lib, dtype, n, d):
    ra = cuda_lib
    w = small(dtype, n, d, True, B=2, H=2)
    inp = make_inputs(w, seed=31 + n)
    t = to_device(inp, dtype)
    B, H = w.B, w.H
    io = t["A1"].dtype
    prob = ra.make_problem(t["A1"], t["A2"], t["A3"], t["WQ"], t["WK"], t["WV"], t["E"],
                           t["pos"], w.causal, w.rope_base)
    buf = {"O": Guarded((B, H, n, d), io), "lse": Guarded((B, H, n), torch.float32),
           "loss": Guarded((), torch.float32),
           **{k: Guarded((H, d, d), torch.float32) for k in ("dWQ", "dWK", "dWV")},
           **{k: Guarded((B, H, n, d), io) for k in ("dA1", "dA2", "dA3")},
           "ws": Guarded((ra.workspace_bytes(prob),), torch.uint8)}
    b = {k: v.t for k, v in buf.items()}
    assert b["ws"].data_ptr() % 256 == 0
    ra.fwd(prob, b["O"], b["lse"], b["loss"], b["ws"])
    ra.loss_bwd_inputs(prob, b["O"], b["lse"], b["loss"], b["dWQ"], b["dWK"], b["dWV"],
                       b["dA1"], b["dA2"], b["dA3"], b["ws"], True)
    torch.cuda.synchronize()
    assert ra.last_error() == ra.RA_OK
    broken = [k for k, v in buf.items() if not v.intact()]
    assert not broken, f"guard regions overwritten: {broken}"
    ref = oracle.forward_backward(inp, w.causal, w.rope_base)
    errs = {k: rel(b[k].float().cpu().numpy(), ref[k]) for k in ("O", "dWV", "dA3")}
    # dWQ, dWK, dA1, dA2 are exactly zero at n = 1 (s = 1 makes gamma vanish): measured there
    # against the norm of dWV, dA3 instead of their own
    for k, other in (("dWQ", "dWV"), ("dWK", "dWV"), ("dA1", "dA3"), ("dA2", "dA3")):
        got, want = b[k].float().cpu().numpy(), ref[k]
        nb = float((want ** 2).sum()) ** 0.5
        scale = float((ref[other] ** 2).sum()) ** 0.5
        errs[k] = rel(got, want) if nb > 0 else float((got ** 2).sum()) ** 0.5 / scale
    errs["loss"] = abs(float(b["loss"].item()) - ref["loss"]) / abs(ref["loss"])
    bad = {k: v for k, v in errs.items() if not v <= TOL[dtype]}
    assert not bad, errs

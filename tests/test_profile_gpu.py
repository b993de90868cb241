"""The library's per-launch timing hooks (what bench.py's timed region relies on).

rope_attn_profile_only(k) must restrict the CUDA events to kernel k's launches, and the
per-kernel totals must add up to no more than the step's own device time."""
import pytest
import torch

from test_parity_gpu import small, to_device
from workloads import make_inputs

pytestmark = pytest.mark.gpu


def _model(cuda_lib, w, t):
    return cuda_lib.RopeAttention(t["A1"], t["A2"], t["A3"], t["WQ"], t["WK"], t["WV"], t["E"],
                                  t["pos"], w.causal, w.rope_base)


def test_profile_only_one_kernel(cuda_lib):
    w = small("bf16", 600, 128, True, B=2, H=2)
    t = to_device(make_inputs(w, seed=5), "bf16")
    m = _model(cuda_lib, w, t)
    m.step()
    torch.cuda.synchronize()
    cuda_lib.profile_read()
    cuda_lib.profile_enable(True)
    m.step()
    torch.cuda.synchronize()
    every = cuda_lib.profile_read()
    cuda_lib.profile_only("attn_bwd_tc")
    for _ in range(3):
        m.step()
    torch.cuda.synchronize()
    only = cuda_lib.profile_read()
    cuda_lib.profile_only(None)
    m.step()
    torch.cuda.synchronize()
    back = cuda_lib.profile_read()
    cuda_lib.profile_enable(False)
    assert cuda_lib.last_error() == cuda_lib.RA_OK
    assert {"attn_fwd_tc", "attn_bwd_tc", "dw_tc"} <= set(every)
    assert set(only) == {"attn_bwd_tc"} and only["attn_bwd_tc"][1] == 3
    assert set(back) == set(every) and all(v[1] == 1 for v in back.values())
    assert all(v[0] > 0 for v in list(every.values()) + list(only.values()))


def test_profile_only_rejects_unknown_name(cuda_lib):
    with pytest.raises(ValueError):
        cuda_lib.profile_only("no_such_kernel")

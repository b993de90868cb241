"""Full-size evidence without the fp64 oracle (the oracle finishes only sampled heads or rows at
these sizes):

  * the directional derivative of the loss along a random direction P of (WQ, WK, WV), by
    central differences of the GPU forward, (L(W + eps P) - L(W - eps P)) / (2 eps), against
    <grad L, P> from the GPU backward (fp32 path) at the three long-sequence workloads:
    B=2 H=32 n=8192, B=1 H=8 n=32768 with bounded scores, and B=1 H=8 n=131072 with RoPE
    base 5e5 (d=128, causal).  The central
    difference of L is the check the "Zero-th Order Algorithm for Softmax Attention
    Optimization" page builds on (提出的方法);
  * the bf16 tensor-core path against the fp32 CUDA-core path on the same bf16-valued inputs,
    every head and instance: O, loss, dWQ, dWK, dWV within the bf16 bar (2e-2).

The fp32 path itself is pinned to the oracle at small sizes (test_parity_gpu.py, 1e-4).
"""
import numpy as np
import pytest
import torch

from test_parity_gpu import rel, to_device
from workloads import WORKLOADS, make_inputs

pytestmark = pytest.mark.gpu

W_FULL = WORKLOADS["b2_h32_n8192_d128_bf16_causal"]


def _model(cuda_lib, w, t, WQ=None, WK=None, WV=None):
    return cuda_lib.RopeAttention(t["A1"], t["A2"], t["A3"],
                                  t["WQ"] if WQ is None else WQ, t["WK"] if WK is None else WK,
                                  t["WV"] if WV is None else WV, t["E"], t["pos"], w.causal,
                                  w.rope_base)


def _loss(cuda_lib, w, t, WQ, WK, WV):
    m = _model(cuda_lib, w, t, WQ, WK, WV)
    m.forward()
    torch.cuda.synchronize()
    assert cuda_lib.last_error() == cuda_lib.RA_OK
    return float(m.loss.item())


@pytest.mark.parametrize("name", [
    "b2_h32_n8192_d128_bf16_causal",
    pytest.param("b1_h8_n32768_d128_bf16_causal_bounded", marks=pytest.mark.slow),
    pytest.param("b1_h8_n131072_d128_bf16_causal_base5e5", marks=pytest.mark.slow),
])
def test_directional_derivative_full_size_fp32(cuda_lib, name):
    """Target E = O(W) + 0.05 noise keeps the loss small enough that its fp32 value resolves
    the change along P; P mixes the gradient direction with a random one (so the check covers
    more than the gradient's own direction); two step sizes cancel the eps^2 term of the
    central difference (Richardson)."""
    w = WORKLOADS[name].with_sizes(dtype="f32")
    inp = make_inputs(w)
    t = to_device(inp, "f32")
    m0 = _model(cuda_lib, w, t)
    m0.forward()
    torch.cuda.synchronize()
    gen = torch.Generator(device="cuda").manual_seed(1234)
    t["E"] = (m0.O + 0.05 * torch.randn(m0.O.shape, generator=gen, device="cuda")).contiguous()
    del m0
    m = _model(cuda_lib, w, t)
    m.forward()
    m.backward(True)
    torch.cuda.synchronize()
    assert cuda_lib.last_error() == cuda_lib.RA_OK
    keys = ("WQ", "WK", "WV")
    g = {k: getattr(m, "d" + k) for k in keys}
    r = {k: torch.randn(t[k].shape, generator=gen, device="cuda") for k in keys}
    gn = torch.sqrt(sum((g[k].double() ** 2).sum() for k in keys))
    rn = torch.sqrt(sum((r[k].double() ** 2).sum() for k in keys))
    wn = torch.sqrt(sum((t[k].double() ** 2).sum() for k in keys))
    P = {k: ((g[k].double() / gn + r[k].double() / rn) / np.sqrt(2.0) * wn).float() for k in keys}
    an = float(sum((g[k].double() * P[k].double()).sum() for k in keys))

    def central(eps):
        lp = _loss(cuda_lib, w, t, *(t[k] + eps * P[k] for k in keys))
        lm = _loss(cuda_lib, w, t, *(t[k] - eps * P[k] for k in keys))
        return (lp - lm) / (2 * eps)

    d1, d2 = central(2e-3), central(1e-3)
    fd = (4 * d2 - d1) / 3
    print(f"\n{name}: central difference {fd:.9e}, <grad, P> {an:.9e}, "
          f"rel {abs(fd - an) / abs(an):.3e}", flush=True)
    assert abs(fd - an) <= 1e-3 * abs(an), (fd, an, d1, d2)


def test_bf16_path_matches_fp32_path_full_size(cuda_lib):
    inp = make_inputs(W_FULL)                     # bf16-valued inputs
    out = {}
    for dtype in ("f32", "bf16"):
        w = W_FULL.with_sizes(dtype=dtype)
        t = to_device(inp, dtype)
        m = _model(cuda_lib, w, t)
        m.forward()
        m.backward(True)
        torch.cuda.synchronize()
        assert cuda_lib.last_error() == cuda_lib.RA_OK
        out[dtype] = {"O": m.O.float().cpu().numpy(), "loss": float(m.loss.item()),
                      **{k: getattr(m, k).cpu().numpy() for k in ("dWQ", "dWK", "dWV")}}
        del m, t
        torch.cuda.empty_cache()
    a, b = out["bf16"], out["f32"]
    errs = {k: rel(a[k], b[k]) for k in ("O", "dWQ", "dWK", "dWV")}
    errs["loss"] = abs(a["loss"] - b["loss"]) / abs(b["loss"])
    # per-head weight gradients too (every head, not only the sampled ones)
    for k in ("dWQ", "dWK", "dWV"):
        errs[k + "_worst_head"] = max(rel(a[k][h], b[k][h]) for h in range(W_FULL.H))
    bad = {k: v for k, v in errs.items() if not v <= 2e-2}
    assert not bad, errs

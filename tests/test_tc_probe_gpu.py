"""Each tcgen05 operand arrangement the kernels use, checked against torch (GPU only)."""
import ctypes

import pytest
import torch

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def probe():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from tests_support import probe_lib
    return probe_lib()


CASES = [
    # M, N, K, a_mn, b_mn, a_tmem
    (128, 128, 128, 0, 0, 0),   # scores: Q K^T, both K-major
    (128, 64, 128, 0, 0, 0),    # backward S^T / beta^T tiles (N = 64)
    (128, 128, 64, 0, 0, 0),
    (128, 128, 128, 0, 1, 1),   # forward P V: A from TMEM, B MN-major
    (128, 64, 128, 0, 1, 1),
    (128, 128, 64, 0, 1, 0),    # backward dV, dK: B MN-major
    (128, 64, 128, 1, 1, 0),    # backward dQ^T: A MN-major, B MN-major
    (128, 64, 128, 1, 0, 0),
    (128, 256, 128, 0, 0, 0),
    (64, 64, 128, 1, 1, 0),     # weight gradient at d = 64 (M = 64)
    (64, 128, 64, 0, 0, 0),
    (128, 128, 128, 1, 1, 0),   # weight gradient at d = 128
]


@pytest.mark.parametrize("M,N,K,a_mn,b_mn,a_tmem", CASES)
def test_mma_form(probe, M, N, K, a_mn, b_mn, a_tmem):
    g = torch.Generator(device="cuda").manual_seed(M * 7 + N * 3 + K + a_mn + 2 * b_mn)
    A = torch.randn(M, K, device="cuda", generator=g).to(torch.bfloat16)
    B = torch.randn(K, N, device="cuda", generator=g).to(torch.bfloat16)
    D = torch.full((M, N), float("nan"), device="cuda")
    rc = probe.probe_mma(ctypes.c_void_p(A.data_ptr()), ctypes.c_void_p(B.data_ptr()),
                         ctypes.c_void_p(D.data_ptr()), M, N, K, a_mn, b_mn, a_tmem,
                         ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert rc == 0
    torch.cuda.synchronize()
    ref = A.float() @ B.float()
    err = (D - ref).abs().max().item()
    assert err <= 1e-3 * ref.abs().max().item(), err


def test_bounded_wait_gives_up(probe):
    ok = ctypes.c_int(7)
    st = probe.probe_timeout(ctypes.c_ulonglong(20_000_000), ctypes.byref(ok))
    assert st == 1, st          # timeout recorded in the status word
    assert ok.value == 0        # the wait reported failure instead of hanging
    # the context is still usable
    x = torch.ones(4, device="cuda")
    assert float(x.sum()) == 4.0


def test_exp2_poly_against_cuda_exp2f(probe):
    """The FMA-pipe 2^x used for part of the softmax exponentials, against exp2f."""
    x = torch.cat([torch.linspace(-126.0, 8.0, 1 << 20, device="cuda"),
                   torch.tensor([0.0, -0.5, 0.5, -1e-7, 7.99], device="cuda")])
    poly = torch.empty_like(x)
    ref = torch.empty_like(x)
    assert probe.probe_exp2(ctypes.c_void_p(x.data_ptr()), ctypes.c_void_p(poly.data_ptr()),
                            ctypes.c_void_p(ref.data_ptr()), x.numel()) == 0
    torch.cuda.synchronize()
    rel = ((poly.double() - ref.double()).abs() / ref.double()).max().item()
    assert rel <= 4e-6, rel
    low = torch.tensor([-127.0, -200.0, float("-inf")], device="cuda")
    out = torch.empty_like(low)
    probe.probe_exp2(ctypes.c_void_p(low.data_ptr()), ctypes.c_void_p(out.data_ptr()),
                     ctypes.c_void_p(torch.empty_like(low).data_ptr()), 3)
    torch.cuda.synchronize()
    assert torch.isfinite(out).all() and (out >= 0).all() and (out <= 2.0 ** -125).all()


def _turns(probe, nblocks, reverse, start, limit_ns):
    log = (ctypes.c_int * nblocks)()
    ok = ctypes.c_int(7)
    final = ctypes.c_uint(0)
    st = probe.probe_turn(nblocks, reverse, start, ctypes.c_ulonglong(limit_ns), log,
                          ctypes.byref(ok), ctypes.byref(final))
    return st, list(log), ok.value, final.value


@pytest.mark.parametrize("reverse", [0, 1])
def test_turn_order(probe, reverse):
    n = 64
    st, log, ok, final = _turns(probe, n, reverse, 0, 1_000_000_000)
    assert st == 0 and ok == 1 and final == n
    want = list(range(n - 1, -1, -1)) if reverse else list(range(n))
    assert log == want


def test_turn_wait_gives_up(probe):
    # the counter starts past the only turn there is: the wait must give up, flag a timeout
    # and still pass the counter on
    st, log, ok, final = _turns(probe, 1, 0, 3, 20_000_000)
    assert st == 1 and ok == 0 and final == 4
    x = torch.ones(4, device="cuda")
    assert float(x.sum()) == 4.0


def _mma_rate(probe, M, N, a_tmem=0, issuers=1, nmma=256):
    cyc, ok = ctypes.c_double(), ctypes.c_int()
    assert probe.probe_mma_rate(M, N, a_tmem, issuers, nmma, ctypes.byref(cyc),
                                ctypes.byref(ok)) == 0
    assert ok.value == 1
    return cyc.value


def test_mma_issue_rate(probe, capsys):
    """Cycles one tcgen05.mma (K = 16) holds the tensor pipe, per shape: the products of the
    backward (M = 128 x N = 64, M = 64 x N = 64, A from TMEM) against N = 128 and 256.  Every
    product must complete; the time must grow with N past 128 (the probe measures executed
    products).  The table is printed (pytest -s) for the design notes."""
    shapes = [(128, 32, 0, 1), (128, 64, 0, 1), (128, 128, 0, 1), (128, 256, 0, 1),
              (64, 64, 0, 1), (64, 128, 0, 1), (128, 64, 1, 1), (128, 128, 1, 1),
              (128, 64, 0, 2), (128, 128, 0, 2)]
    res = {sh: _mma_rate(probe, *sh) for sh in shapes}
    with capsys.disabled():
        for (M, N, at, iss), c in res.items():
            print(f"M={M:3d} N={N:3d} A={'tmem' if at else 'smem'} issuers={iss}: "
                  f"{c:6.1f} cycles per product (ideal {M * N * 16 / 4096:5.1f})")
    assert res[(128, 256, 0, 1)] > 1.4 * res[(128, 128, 0, 1)]
    assert all(c > 0 for c in res.values())

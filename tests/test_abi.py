"""Host-side checks of the C ABI (CPU only: no kernel is launched).

Every call below fails validation, which happens before anything touches the GPU, so the
fake device addresses are never dereferenced.
"""
import ctypes
import os
import re

import pytest

from loss_closed_form_b200 import rope_attn as ra

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "rope_attn.h")

FAKE = 0x10000  # 16-byte aligned, never dereferenced


def _declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(rope_attn_\w+)\s*\(", src)))


def _prob(**kw):
    base = dict(B=1, H=2, n=100, d=64, dtype=ra.RA_BF16, causal=0, rope_base=1e4, pos=None,
                A1=FAKE, A2=FAKE, A3=FAKE, WQ=FAKE, WK=FAKE, WV=FAKE, E=FAKE, deterministic=0)
    base.update(kw)
    return ra.Problem(*(base[f] for f, _ in ra.Problem._fields_))


def _fwd(p, O=FAKE, lse=FAKE, loss=FAKE, ws=FAKE * 16, nbytes=None):
    lib = ra.load()
    if nbytes is None:
        nbytes = lib.rope_attn_workspace_bytes(ctypes.byref(p))
    return lib.rope_attn_fwd(ctypes.byref(p), O, lse, loss, ws, nbytes, None)


def _bwd(p, O=FAKE, lse=FAKE, loss=FAKE, dW=(FAKE, FAKE, FAKE), ws=FAKE * 16, nbytes=None,
         holds=1):
    lib = ra.load()
    if nbytes is None:
        nbytes = lib.rope_attn_workspace_bytes(ctypes.byref(p))
    return lib.rope_attn_loss_bwd(ctypes.byref(p), O, lse, loss, *dW, ws, nbytes, holds, None)


def test_library_exports_every_declared_symbol():
    lib = ra.load()
    declared = _declared_functions()
    assert set(declared) == set(ra.EXPORTED)
    for name in declared:
        assert getattr(lib, name) is not None


def test_workspace_bytes():
    lib = ra.load()
    p = _prob()
    nb = lib.rope_attn_workspace_bytes(ctypes.byref(p))
    assert nb > 0 and nb % 256 == 0
    assert lib.rope_attn_workspace_bytes(ctypes.byref(_prob(d=96))) == 0
    assert lib.rope_attn_workspace_bytes(ctypes.byref(_prob(n=0))) == 0
    assert lib.rope_attn_workspace_bytes(None) == 0
    # grows with n
    assert lib.rope_attn_workspace_bytes(ctypes.byref(_prob(n=1000))) > nb


@pytest.mark.parametrize("kw,want", [
    (dict(n=0), ra.RA_ERR_INVALID_ARG),
    (dict(B=0), ra.RA_ERR_INVALID_ARG),
    (dict(H=-1), ra.RA_ERR_INVALID_ARG),
    (dict(dtype=7), ra.RA_ERR_INVALID_ARG),
    (dict(causal=2), ra.RA_ERR_INVALID_ARG),
    (dict(deterministic=2), ra.RA_ERR_INVALID_ARG),
    (dict(rope_base=0.0), ra.RA_ERR_INVALID_ARG),
    (dict(rope_base=float("nan")), ra.RA_ERR_INVALID_ARG),
    (dict(A1=None), ra.RA_ERR_INVALID_ARG),
    (dict(WV=None), ra.RA_ERR_INVALID_ARG),
    (dict(d=32), ra.RA_ERR_UNSUPPORTED),
    (dict(d=256), ra.RA_ERR_UNSUPPORTED),
    # bf16: the backward's grid holds one CTA per 128-key tile in y (at most 65535)
    (dict(n=65535 * 128 + 1, dtype=ra.RA_BF16), ra.RA_ERR_UNSUPPORTED),
    (dict(n=(1 << 24) + 1, dtype=ra.RA_F32), ra.RA_ERR_UNSUPPORTED),
    (dict(B=300, H=300), ra.RA_ERR_UNSUPPORTED),
    (dict(A2=FAKE + 8), ra.RA_ERR_ALIGNMENT),
    (dict(E=FAKE + 2), ra.RA_ERR_ALIGNMENT),
    (dict(pos=FAKE + 2), ra.RA_ERR_ALIGNMENT),
])
def test_fwd_and_bwd_reject_bad_problems(kw, want):
    p = _prob(**kw)
    assert _fwd(p, nbytes=1 << 40) == want
    assert _bwd(p, nbytes=1 << 40) == want


def test_fwd_argument_errors():
    p = _prob()
    assert _fwd(p, O=None) == ra.RA_ERR_INVALID_ARG
    assert _fwd(p, lse=None) == ra.RA_ERR_INVALID_ARG
    assert _fwd(_prob(E=None), loss=FAKE) == ra.RA_ERR_INVALID_ARG
    assert _fwd(p, O=FAKE + 4) == ra.RA_ERR_ALIGNMENT
    assert _fwd(p, ws=None) == ra.RA_ERR_WORKSPACE
    assert _fwd(p, ws=FAKE * 16 + 128) == ra.RA_ERR_ALIGNMENT
    nb = ra.load().rope_attn_workspace_bytes(ctypes.byref(p))
    assert _fwd(p, nbytes=nb - 1) == ra.RA_ERR_WORKSPACE


def test_bwd_argument_errors():
    p = _prob()
    assert _bwd(_prob(E=None)) == ra.RA_ERR_INVALID_ARG
    assert _bwd(p, O=None) == ra.RA_ERR_INVALID_ARG
    assert _bwd(p, dW=(FAKE, None, FAKE)) == ra.RA_ERR_INVALID_ARG
    assert _bwd(p, holds=2) == ra.RA_ERR_INVALID_ARG
    assert _bwd(p, dW=(FAKE, FAKE + 4, FAKE)) == ra.RA_ERR_ALIGNMENT
    nb = ra.load().rope_attn_workspace_bytes(ctypes.byref(p))
    assert _bwd(p, nbytes=nb - 256) == ra.RA_ERR_WORKSPACE


def test_step_argument_errors():
    """rope_attn_step validates like the forward and the backward together, before anything
    is launched."""
    lib = ra.load()
    p = _prob()
    nb = lib.rope_attn_workspace_bytes(ctypes.byref(p))

    def call(prob=p, O=FAKE, lse=FAKE, dW=(FAKE, FAKE, FAKE), ws=FAKE * 16, nbytes=nb):
        return lib.rope_attn_step(ctypes.byref(prob), O, lse, FAKE, *dW, ws, nbytes, None)
    assert call(prob=_prob(E=None)) == ra.RA_ERR_INVALID_ARG
    assert call(O=None) == ra.RA_ERR_INVALID_ARG
    assert call(lse=None) == ra.RA_ERR_INVALID_ARG
    assert call(dW=(FAKE, FAKE, None)) == ra.RA_ERR_INVALID_ARG
    assert call(prob=_prob(deterministic=3)) == ra.RA_ERR_INVALID_ARG
    assert call(dW=(FAKE + 4, FAKE, FAKE)) == ra.RA_ERR_ALIGNMENT
    assert call(ws=None) == ra.RA_ERR_WORKSPACE
    assert call(nbytes=nb - 256) == ra.RA_ERR_WORKSPACE
    assert call(prob=_prob(d=96)) == ra.RA_ERR_UNSUPPORTED


def test_bwd_inputs_argument_errors():
    """rope_attn_loss_bwd_inputs validates its extra outputs, then everything the plain
    backward validates, before anything is launched."""
    lib = ra.load()
    p = _prob()
    nb = lib.rope_attn_workspace_bytes(ctypes.byref(p))

    def call(prob=p, dA=(FAKE, FAKE, FAKE), nbytes=nb, holds=1, O=FAKE):
        return lib.rope_attn_loss_bwd_inputs(ctypes.byref(prob), O, FAKE, FAKE, FAKE, FAKE,
                                             FAKE, *dA, FAKE * 16, nbytes, holds, None)
    assert call(dA=(None, FAKE, FAKE)) == ra.RA_ERR_INVALID_ARG
    assert call(dA=(FAKE, FAKE, None)) == ra.RA_ERR_INVALID_ARG
    assert call(dA=(FAKE, FAKE + 8, FAKE)) == ra.RA_ERR_ALIGNMENT
    assert call(prob=_prob(E=None)) == ra.RA_ERR_INVALID_ARG
    assert call(O=None) == ra.RA_ERR_INVALID_ARG
    assert call(holds=3) == ra.RA_ERR_INVALID_ARG
    assert call(nbytes=nb - 256) == ra.RA_ERR_WORKSPACE


def test_combined_weight_argument_errors():
    lib = ra.load()
    w = lambda X=FAKE, H=2, d=64, dt=ra.RA_BF16, WQ=FAKE, WK=FAKE: \
        lib.rope_attn_combined_weights(X, H, d, dt, WQ, WK, None)
    assert w(X=None) == ra.RA_ERR_INVALID_ARG
    assert w(WK=None) == ra.RA_ERR_INVALID_ARG
    assert w(H=0) == ra.RA_ERR_INVALID_ARG
    assert w(d=32) == ra.RA_ERR_INVALID_ARG
    assert w(dt=5) == ra.RA_ERR_INVALID_ARG
    assert w(WQ=FAKE + 4) == ra.RA_ERR_ALIGNMENT
    g = lambda dWK=FAKE, H=2, d=128, dX=FAKE: lib.rope_attn_combined_grad(dWK, H, d, dX, None)
    assert g(dWK=None) == ra.RA_ERR_INVALID_ARG
    assert g(H=-1) == ra.RA_ERR_INVALID_ARG
    assert g(d=96) == ra.RA_ERR_INVALID_ARG
    assert g(dX=FAKE + 8) == ra.RA_ERR_ALIGNMENT


def test_status_strings():
    for s in range(7):
        assert ra.status_string(s).startswith("RA_")
    assert "unknown" in ra.status_string(99)


def test_binding_fails_loudly_without_library(monkeypatch):
    monkeypatch.setattr(ra, "_lib", None)
    monkeypatch.setattr(ra, "LIB_PATH", "/nonexistent/librope_attn.so")
    with pytest.raises(RuntimeError, match="not built"):
        ra.load()

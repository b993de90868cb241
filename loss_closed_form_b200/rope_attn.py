"""ctypes binding of librope_attn (include/rope_attn.h): argument marshalling only.

Every step of the computation runs in the library's CUDA kernels; this module turns
torch tensors into pointers and sizes, and raises on a status other than RA_OK.  If the
shared library is missing it raises: there is no fallback.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "librope_attn.so")

RA_OK, RA_ERR_INVALID_ARG, RA_ERR_UNSUPPORTED, RA_ERR_ALIGNMENT, RA_ERR_WORKSPACE, \
    RA_ERR_CUDA, RA_ERR_TIMEOUT = range(7)
RA_F32, RA_BF16 = 0, 1

# Every symbol include/rope_attn.h declares.
EXPORTED = ("rope_attn_workspace_bytes", "rope_attn_fwd", "rope_attn_loss_bwd",
            "rope_attn_last_error", "rope_attn_status_string", "rope_attn_launch_count",
            "rope_attn_profile_enable", "rope_attn_profile_only", "rope_attn_profile_read",
            "rope_attn_kernel_name",
            "rope_attn_step_noalloc", "rope_attn_loss_bwd_inputs", "rope_attn_combined_weights",
            "rope_attn_combined_grad", "rope_attn_approx_workspace_bytes", "rope_attn_approx_step",
            "rope_attn_step")

# Capacity of the static scratch behind rope_attn_step_noalloc (RA_NOALLOC_SCRATCH_BYTES).
NOALLOC_SCRATCH_BYTES = 16 * 1024 * 1024


class Problem(ctypes.Structure):
    """Mirror of ``ra_problem``."""
    _fields_ = [
        ("B", ctypes.c_int32), ("H", ctypes.c_int32), ("n", ctypes.c_int32),
        ("d", ctypes.c_int32), ("dtype", ctypes.c_int32), ("causal", ctypes.c_int32),
        ("rope_base", ctypes.c_double), ("pos", ctypes.c_void_p),
        ("A1", ctypes.c_void_p), ("A2", ctypes.c_void_p), ("A3", ctypes.c_void_p),
        ("WQ", ctypes.c_void_p), ("WK", ctypes.c_void_p), ("WV", ctypes.c_void_p),
        ("E", ctypes.c_void_p), ("deterministic", ctypes.c_int32),
    ]


class RopeAttnError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {status_string(status)}")


_lib = None


def load() -> ctypes.CDLL:
    """Load librope_attn.so (built in-tree).  Raises if it has not been built."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(f"librope_attn.so not built: run python -m loss_closed_form_b200.build "
                           f"(expected at {LIB_PATH})")
    lib = ctypes.CDLL(LIB_PATH)
    P = ctypes.POINTER(Problem)
    vp, sz, i32 = ctypes.c_void_p, ctypes.c_size_t, ctypes.c_int32
    lib.rope_attn_workspace_bytes.argtypes = [P]
    lib.rope_attn_workspace_bytes.restype = sz
    lib.rope_attn_fwd.argtypes = [P, vp, vp, vp, vp, sz, vp]
    lib.rope_attn_fwd.restype = ctypes.c_int
    lib.rope_attn_loss_bwd.argtypes = [P, vp, vp, vp, vp, vp, vp, vp, sz, i32, vp]
    lib.rope_attn_loss_bwd.restype = ctypes.c_int
    lib.rope_attn_last_error.argtypes = [vp]
    lib.rope_attn_last_error.restype = ctypes.c_int
    lib.rope_attn_status_string.argtypes = [ctypes.c_int]
    lib.rope_attn_status_string.restype = ctypes.c_char_p
    lib.rope_attn_launch_count.argtypes = []
    lib.rope_attn_launch_count.restype = ctypes.c_int64
    lib.rope_attn_profile_enable.argtypes = [i32]
    lib.rope_attn_profile_enable.restype = None
    lib.rope_attn_profile_only.argtypes = [i32]
    lib.rope_attn_profile_only.restype = None
    lib.rope_attn_profile_read.argtypes = [vp, vp, i32]
    lib.rope_attn_profile_read.restype = i32
    lib.rope_attn_kernel_name.argtypes = [i32]
    lib.rope_attn_kernel_name.restype = ctypes.c_char_p
    lib.rope_attn_step_noalloc.argtypes = [P, vp, vp, vp, vp, vp, vp, vp]
    lib.rope_attn_step_noalloc.restype = ctypes.c_int
    lib.rope_attn_step.argtypes = [P, vp, vp, vp, vp, vp, vp, vp, sz, vp]
    lib.rope_attn_step.restype = ctypes.c_int
    lib.rope_attn_loss_bwd_inputs.argtypes = [P, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, sz,
                                              i32, vp]
    lib.rope_attn_loss_bwd_inputs.restype = ctypes.c_int
    lib.rope_attn_combined_weights.argtypes = [vp, i32, i32, i32, vp, vp, vp]
    lib.rope_attn_combined_weights.restype = ctypes.c_int
    lib.rope_attn_combined_grad.argtypes = [vp, i32, i32, vp, vp]
    lib.rope_attn_approx_workspace_bytes.argtypes = [P]
    lib.rope_attn_approx_workspace_bytes.restype = sz
    lib.rope_attn_approx_step.argtypes = [P, vp, vp, vp, vp, vp, vp, sz, vp]
    lib.rope_attn_approx_step.restype = ctypes.c_int
    lib.rope_attn_combined_grad.restype = ctypes.c_int
    _lib = lib
    return lib


def status_string(status: int) -> str:
    return load().rope_attn_status_string(status).decode()


def _ptr(t) -> Optional[int]:
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _stream(stream) -> Optional[int]:
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def make_problem(A1, A2, A3, WQ, WK, WV, E=None, pos=None, causal=False,
                 rope_base=10000.0, deterministic=False) -> Problem:
    """Build an ``ra_problem`` from tensors (or raw device pointers with explicit shapes).

    A1, A2, A3, E: [B][H][n][d]; WQ, WK, WV: [H][d][d]; pos: [n] int32 or None.
    deterministic: the backward adds its per-key-tile parts in a fixed order (bitwise
    repeatable gradients).
    """
    import torch
    B, H, n, d = A1.shape
    if A1.dtype == torch.float32:
        dt = RA_F32
    elif A1.dtype == torch.bfloat16:
        dt = RA_BF16
    else:
        raise TypeError(f"unsupported dtype {A1.dtype}")
    for name, t in (("A2", A2), ("A3", A3), ("WQ", WQ), ("WK", WK), ("WV", WV), ("E", E)):
        if t is not None and (t.dtype != A1.dtype or not t.is_contiguous()):
            raise TypeError(f"{name} must be contiguous {A1.dtype}")
    if pos is not None and pos.dtype != torch.int32:
        raise TypeError("pos must be int32")
    return Problem(B, H, n, d, dt, int(bool(causal)), float(rope_base), _ptr(pos),
                   _ptr(A1), _ptr(A2), _ptr(A3), _ptr(WQ), _ptr(WK), _ptr(WV), _ptr(E),
                   int(bool(deterministic)))


def workspace_bytes(prob: Problem) -> int:
    return int(load().rope_attn_workspace_bytes(ctypes.byref(prob)))


def fwd(prob: Problem, O, lse, loss, ws, stream=None) -> None:
    """rope_attn_fwd: O, lse (and loss when the problem has a target) into the given tensors."""
    st = load().rope_attn_fwd(ctypes.byref(prob), _ptr(O), _ptr(lse), _ptr(loss), _ptr(ws),
                              ws.numel() * ws.element_size(), _stream(stream))
    if st != RA_OK:
        raise RopeAttnError(st, "rope_attn_fwd")


def loss_bwd(prob: Problem, O, lse, loss, dWQ, dWK, dWV, ws, ws_holds_fwd=False,
             stream=None) -> None:
    """rope_attn_loss_bwd: dWQ, dWK, dWV (fp32 [H][d][d]) and the loss."""
    st = load().rope_attn_loss_bwd(ctypes.byref(prob), _ptr(O), _ptr(lse), _ptr(loss),
                                   _ptr(dWQ), _ptr(dWK), _ptr(dWV), _ptr(ws),
                                   ws.numel() * ws.element_size(), int(bool(ws_holds_fwd)),
                                   _stream(stream))
    if st != RA_OK:
        raise RopeAttnError(st, "rope_attn_loss_bwd")


def loss_bwd_inputs(prob: Problem, O, lse, loss, dWQ, dWK, dWV, dA1, dA2, dA3, ws,
                    ws_holds_fwd=False, stream=None) -> None:
    """rope_attn_loss_bwd_inputs: as loss_bwd, plus dA1, dA2, dA3 ([B][H][n][d], I/O dtype)."""
    st = load().rope_attn_loss_bwd_inputs(
        ctypes.byref(prob), _ptr(O), _ptr(lse), _ptr(loss), _ptr(dWQ), _ptr(dWK), _ptr(dWV),
        _ptr(dA1), _ptr(dA2), _ptr(dA3), _ptr(ws), ws.numel() * ws.element_size(),
        int(bool(ws_holds_fwd)), _stream(stream))
    if st != RA_OK:
        raise RopeAttnError(st, "rope_attn_loss_bwd_inputs")


def combined_weights(X, WQ, WK, stream=None) -> None:
    """rope_attn_combined_weights: WQ = I, WK = X^T per head (X, WQ, WK: [H][d][d])."""
    import torch
    H, d = X.shape[0], X.shape[1]
    dt = RA_F32 if X.dtype == torch.float32 else RA_BF16
    st = load().rope_attn_combined_weights(_ptr(X), H, d, dt, _ptr(WQ), _ptr(WK),
                                           _stream(stream))
    if st != RA_OK:
        raise RopeAttnError(st, "rope_attn_combined_weights")


def combined_grad(dWK, dX, stream=None) -> None:
    """rope_attn_combined_grad: dX = dWK^T per head (fp32 [H][d][d])."""
    H, d = dWK.shape[0], dWK.shape[1]
    st = load().rope_attn_combined_grad(_ptr(dWK), H, d, _ptr(dX), _stream(stream))
    if st != RA_OK:
        raise RopeAttnError(st, "rope_attn_combined_grad")


def step(prob: Problem, O, lse, loss, dWQ, dWK, dWV, ws, stream=None) -> None:
    """rope_attn_step: the forward with the loss and the weight-gradient backward on the same
    workspace, in one call."""
    st = load().rope_attn_step(ctypes.byref(prob), _ptr(O), _ptr(lse), _ptr(loss), _ptr(dWQ),
                               _ptr(dWK), _ptr(dWV), _ptr(ws), ws.numel() * ws.element_size(),
                               _stream(stream))
    if st != RA_OK:
        raise RopeAttnError(st, "rope_attn_step")


def step_noalloc(prob: Problem, O, lse, loss, dWQ, dWK, dWV, stream=None) -> None:
    """rope_attn_step_noalloc: forward + backward on the library's static scratch.

    For callers that cannot allocate device memory; problems whose workspace exceeds
    NOALLOC_SCRATCH_BYTES raise RopeAttnError(RA_ERR_WORKSPACE).
    """
    st = load().rope_attn_step_noalloc(ctypes.byref(prob), _ptr(O), _ptr(lse), _ptr(loss),
                                       _ptr(dWQ), _ptr(dWK), _ptr(dWV), _stream(stream))
    if st != RA_OK:
        raise RopeAttnError(st, "rope_attn_step_noalloc")


def approx_workspace_bytes(prob: Problem) -> int:
    return int(load().rope_attn_approx_workspace_bytes(ctypes.byref(prob)))


def approx_step(prob: Problem, O, loss, dWQ, dWK, dWV, ws, stream=None) -> None:
    """rope_attn_approx_step: the near-linear approximate method (degree-1 polynomial, low-rank
    states): O, the loss and the approximate weight gradients."""
    st = load().rope_attn_approx_step(ctypes.byref(prob), _ptr(O), _ptr(loss), _ptr(dWQ),
                                      _ptr(dWK), _ptr(dWV), _ptr(ws),
                                      ws.numel() * ws.element_size(), _stream(stream))
    if st != RA_OK:
        raise RopeAttnError(st, "rope_attn_approx_step")


def last_error(stream=None) -> int:
    return int(load().rope_attn_last_error(_stream(stream)))


def launch_count() -> int:
    return int(load().rope_attn_launch_count())


def profile_enable(on: bool) -> None:
    load().rope_attn_profile_enable(int(bool(on)))


def profile_only(kernel: str = None) -> None:
    """Events around the launches of the named kernel only (None: around every launch)."""
    kid = -1 if kernel is None else kernel_names().index(kernel)
    load().rope_attn_profile_only(kid)


def profile_read(max_kernels: int = 64):
    """{kernel name: (total ms, launches)} since the last read (kernels with launches only)."""
    lib = load()
    ms = (ctypes.c_float * max_kernels)()
    cnt = (ctypes.c_int32 * max_kernels)()
    k = lib.rope_attn_profile_read(ctypes.cast(ms, ctypes.c_void_p),
                                   ctypes.cast(cnt, ctypes.c_void_p), max_kernels)
    if k < 0:
        raise RopeAttnError(RA_ERR_CUDA, "rope_attn_profile_read")
    return {lib.rope_attn_kernel_name(i).decode(): (float(ms[i]), int(cnt[i]))
            for i in range(min(k, max_kernels)) if cnt[i] > 0}


def kernel_names():
    lib = load()
    out, i = [], 0
    while True:
        nm = lib.rope_attn_kernel_name(i)
        if nm is None:
            return out
        out.append(nm.decode())
        i += 1


class RopeAttention:
    """Owns the output tensors and the workspace for one problem shape.

    ``step()`` runs the forward pass with loss, then the closed-form backward reusing the
    forward's workspace, and returns (loss, dWQ, dWK, dWV) as device tensors.
    """

    def __init__(self, A1, A2, A3, WQ, WK, WV, E, pos=None, causal=False, rope_base=10000.0,
                 deterministic=False):
        import torch
        self.inputs = (A1, A2, A3, WQ, WK, WV, E, pos)
        self.prob = make_problem(A1, A2, A3, WQ, WK, WV, E, pos, causal, rope_base,
                                 deterministic)
        B, H, n, d = A1.shape
        dev = A1.device
        self.O = torch.empty_like(A1)
        self.lse = torch.empty((B, H, n), dtype=torch.float32, device=dev)
        self.loss = torch.zeros((), dtype=torch.float32, device=dev)
        self.dWQ = torch.empty((H, d, d), dtype=torch.float32, device=dev)
        self.dWK = torch.empty_like(self.dWQ)
        self.dWV = torch.empty_like(self.dWQ)
        nb = workspace_bytes(self.prob)
        if nb == 0:
            raise RopeAttnError(RA_ERR_INVALID_ARG, "rope_attn_workspace_bytes")
        self.ws = torch.empty(nb, dtype=torch.uint8, device=dev)

    def forward(self, stream=None):
        fwd(self.prob, self.O, self.lse, self.loss, self.ws, stream)
        return self.O, self.lse, self.loss

    def backward(self, ws_holds_fwd=True, stream=None):
        # after this object's forward the loss is already in self.loss: the backward need not
        # sum the partials again
        loss_bwd(self.prob, self.O, self.lse, None if ws_holds_fwd else self.loss, self.dWQ,
                 self.dWK, self.dWV, self.ws, ws_holds_fwd, stream)
        return self.loss, self.dWQ, self.dWK, self.dWV

    def backward_inputs(self, ws_holds_fwd=True, stream=None):
        """Backward with the input gradients: returns (loss, dWQ, dWK, dWV, dA1, dA2, dA3)."""
        import torch
        if not hasattr(self, "dA1"):
            self.dA1 = torch.empty_like(self.O)
            self.dA2 = torch.empty_like(self.O)
            self.dA3 = torch.empty_like(self.O)
        loss_bwd_inputs(self.prob, self.O, self.lse, None if ws_holds_fwd else self.loss,
                        self.dWQ, self.dWK, self.dWV, self.dA1, self.dA2, self.dA3, self.ws,
                        ws_holds_fwd, stream)
        return self.loss, self.dWQ, self.dWK, self.dWV, self.dA1, self.dA2, self.dA3

    def step(self, stream=None):
        """Forward with the loss, then the weight gradients (rope_attn_step); returns
        (loss, dWQ, dWK, dWV)."""
        step(self.prob, self.O, self.lse, self.loss, self.dWQ, self.dWK, self.dWV, self.ws,
             stream)
        return self.loss, self.dWQ, self.dWK, self.dWV


class RopeAttentionX:
    """The page's parameterisation: one combined weight X per head (score
    a1_i^T R_{j-i} X a2_j / sqrt(d)) and the value weight WV.  ``step()`` returns
    (loss, dX, dWV) as device tensors; call ``set_weights(X)`` after changing X."""

    def __init__(self, A1, A2, A3, X, WV, E, pos=None, causal=False, rope_base=10000.0):
        import torch
        H, d = X.shape[0], X.shape[1]
        self.WQ = torch.empty_like(X)
        self.WK = torch.empty_like(X)
        combined_weights(X, self.WQ, self.WK)
        self.attn = RopeAttention(A1, A2, A3, self.WQ, self.WK, WV, E, pos, causal, rope_base)
        self.dX = torch.empty((H, d, d), dtype=torch.float32, device=X.device)

    def set_weights(self, X, stream=None):
        combined_weights(X, self.WQ, self.WK, stream)

    def forward(self, stream=None):
        return self.attn.forward(stream)

    def step(self, stream=None):
        self.attn.forward(stream)
        self.attn.backward(True, stream)
        combined_grad(self.attn.dWK, self.dX, stream)
        return self.attn.loss, self.dX, self.attn.dWV

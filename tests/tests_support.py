"""Helpers shared by the GPU tests."""
import ctypes


def probe_lib():
    from tc_probe_build import build
    lib = ctypes.CDLL(build())
    vp = ctypes.c_void_p
    lib.probe_mma.argtypes = [vp, vp, vp, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                              ctypes.c_int, ctypes.c_int, ctypes.c_int, vp]
    lib.probe_mma.restype = ctypes.c_int
    lib.probe_timeout.argtypes = [ctypes.c_ulonglong, ctypes.POINTER(ctypes.c_int)]
    lib.probe_timeout.restype = ctypes.c_int
    lib.probe_exp2.argtypes = [vp, vp, vp, ctypes.c_int]
    lib.probe_exp2.restype = ctypes.c_int
    lib.probe_turn.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_uint, ctypes.c_ulonglong,
                               ctypes.POINTER(ctypes.c_int), ctypes.POINTER(ctypes.c_int),
                               ctypes.POINTER(ctypes.c_uint)]
    lib.probe_turn.restype = ctypes.c_int
    lib.probe_mma_rate.argtypes = [ctypes.c_int] * 5 + [ctypes.POINTER(ctypes.c_double),
                                                        ctypes.POINTER(ctypes.c_int)]
    lib.probe_mma_rate.restype = ctypes.c_int
    return lib

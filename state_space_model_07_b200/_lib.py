"""ctypes loader for libssd.so (the C ABI declared in include/ssd.h).

The library is built in-tree by ``state_space_model_07_b200.build``.  There is
no fallback: if it is missing, every call raises.
"""
from __future__ import annotations

import ctypes
import os

PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libssd.so")

SSD_F32, SSD_BF16 = 0, 1
STATUS = {0: "SSD_OK", 1: "SSD_ERR_NULL", 2: "SSD_ERR_SHAPE", 3: "SSD_ERR_DTYPE", 4: "SSD_ERR_CHUNK",
          5: "SSD_ERR_UNSUPPORTED", 6: "SSD_ERR_CUDA", 7: "SSD_ERR_TIMEOUT", 8: "SSD_ERR_SEQIDX",
          9: "SSD_ERR_RANGE"}
# Every function include/ssd.h declares.
EXPORTS = ("ssd_chunk_scan_fwd", "ssd_state_update", "ssd_status_string", "ssd_last_error",
           "ssd_profile_enable", "ssd_profile_read", "ssd_chunk_scan_fwd_noalloc", "ssd_selftest_bounded_wait",
           "ssd_chunk_scan_bwd", "ssd_segment_logdecay", "ssd_state_chain", "ssd_state_to_output",
           "ssd_group_norm", "ssd_quant_chunks", "ssd_dequant_sum_quant", "ssd_dequant_chunks")


class SsdDims(ctypes.Structure):
    _fields_ = [("batch", ctypes.c_int64), ("seqlen", ctypes.c_int64), ("nheads", ctypes.c_int64),
                ("headdim", ctypes.c_int64), ("dstate", ctypes.c_int64), ("ngroups", ctypes.c_int64),
                ("nseqs", ctypes.c_int64), ("dtype", ctypes.c_int32)]


class SsdKernelStat(ctypes.Structure):
    _fields_ = [("name", ctypes.c_char * 48), ("launches", ctypes.c_int64), ("timed", ctypes.c_int64),
                ("total_ms", ctypes.c_double)]


class SsdError(RuntimeError):
    def __init__(self, code: int, detail: str = ""):
        self.code = code
        name = STATUS.get(code, str(code))
        super().__init__(f"{name}: {detail}" if detail else name)


_lib = None
_VP = ctypes.c_void_p


def lib():
    """Loads libssd.so once; raises if it has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(PATH):
            raise RuntimeError(f"CUDA library missing: {PATH}; build it with "
                               "`python -m state_space_model_07_b200.build`")
        L = ctypes.CDLL(PATH)
        dims = ctypes.POINTER(SsdDims)
        L.ssd_chunk_scan_fwd.restype = ctypes.c_int
        L.ssd_chunk_scan_fwd.argtypes = [dims] + [_VP] * 9 + [ctypes.c_int, _VP, _VP, _VP]
        L.ssd_chunk_scan_fwd_noalloc.restype = ctypes.c_int
        L.ssd_chunk_scan_fwd_noalloc.argtypes = [dims] + [_VP] * 9 + [ctypes.c_int, _VP, _VP, _VP]
        L.ssd_chunk_scan_bwd.restype = ctypes.c_int
        L.ssd_chunk_scan_bwd.argtypes = [dims] + [_VP] * 9 + [ctypes.c_int] + [_VP] * 11
        L.ssd_segment_logdecay.restype = ctypes.c_int
        L.ssd_segment_logdecay.argtypes = [dims] + [_VP] * 5
        L.ssd_state_chain.restype = ctypes.c_int
        L.ssd_state_chain.argtypes = [dims] + [_VP] * 5
        L.ssd_state_to_output.restype = ctypes.c_int
        L.ssd_state_to_output.argtypes = [dims] + [_VP] * 7
        i64 = ctypes.c_int64
        L.ssd_group_norm.restype = ctypes.c_int
        L.ssd_group_norm.argtypes = [i64, i64, i64, ctypes.c_int, _VP, _VP, _VP, ctypes.c_float, _VP, _VP]
        L.ssd_quant_chunks.restype = ctypes.c_int
        L.ssd_quant_chunks.argtypes = [i64, i64, i64, _VP, _VP, _VP, _VP]
        L.ssd_dequant_sum_quant.restype = ctypes.c_int
        L.ssd_dequant_sum_quant.argtypes = [i64, i64, i64, _VP, _VP, _VP, _VP, _VP]
        L.ssd_dequant_chunks.restype = ctypes.c_int
        L.ssd_dequant_chunks.argtypes = [i64, i64, i64, ctypes.c_int, _VP, _VP, _VP, _VP]
        L.ssd_state_update.restype = ctypes.c_int
        L.ssd_state_update.argtypes = [dims] + [_VP] * 10
        L.ssd_status_string.restype = ctypes.c_char_p
        L.ssd_status_string.argtypes = [ctypes.c_int]
        L.ssd_last_error.restype = ctypes.c_char_p
        L.ssd_last_error.argtypes = []
        L.ssd_profile_enable.restype = ctypes.c_int
        L.ssd_profile_enable.argtypes = [ctypes.c_int]
        L.ssd_profile_read.restype = ctypes.c_int
        L.ssd_profile_read.argtypes = [ctypes.POINTER(SsdKernelStat), ctypes.c_int, ctypes.c_int]
        L.ssd_selftest_bounded_wait.restype = ctypes.c_int
        L.ssd_selftest_bounded_wait.argtypes = [ctypes.c_int64, _VP]
        _lib = L
    return _lib


def check(rc: int):
    if rc != 0:
        raise SsdError(rc, lib().ssd_last_error().decode())


def profile_enable(on: bool) -> bool:
    """Turns CUDA-event timing of every library kernel launch on or off."""
    return bool(lib().ssd_profile_enable(1 if on else 0))


def profile_read(reset: bool = True) -> dict:
    """{kernel name: (launches, timed launches, total ms)} since the last reset."""
    buf = (SsdKernelStat * 32)()
    n = lib().ssd_profile_read(buf, 32, 1 if reset else 0)
    if n < 0:
        raise SsdError(-n, "profile_read")
    return {buf[i].name.decode(): (buf[i].launches, buf[i].timed, buf[i].total_ms) for i in range(n)}

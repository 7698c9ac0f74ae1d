"""ctypes view of libmea.so (the C ABI in include/mea.h). Marshalling only."""
from __future__ import annotations

import ctypes
import os

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libmea.so")

# mea_status values (include/mea.h)
MEA_OK = 0
MEA_ERR_NULL = -1
MEA_ERR_SHAPE = -2
MEA_ERR_HEADS = -3
MEA_ERR_HEAD_DIM = -4
MEA_ERR_DTYPE = -5
MEA_ERR_ALIGN = -6
MEA_ERR_MASK = -7
MEA_ERR_WORKSPACE = -8
MEA_ERR_CUDA = -9
MEA_ERR_DEVICE_TIMEOUT = -10
MEA_ERR_DEVICE = -11
MEA_ERR_SCALE = -12
MEA_ERR_SCRATCH_LIMIT = -13

MEA_F16 = 0
MEA_BF16 = 1
MEA_MASK_NONE = 0
MEA_MASK_CAUSAL = 1
MEA_SELFTEST_WAIT_CODE = 0x7F01

EXPORTS = ("mea_forward", "mea_forward_fp8", "mea_backward_workspace_size", "mea_backward",
           "mea_decode_workspace_size", "mea_decode_splitkv", "mea_decode_paged",
           "mea_decode_splitkv_noalloc", "mea_status_string", "mea_device_error",
           "mea_set_wait_timeout_ns", "mea_wait_selftest", "mea_version")

_lib = None


def load() -> ctypes.CDLL:
    """Loads libmea.so (raises if it has not been built: there is no fallback path)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"libmea.so not built at {LIB_PATH}; run "
                          "`python -m memory_efficient_attention_b200.build`")
    lib = ctypes.CDLL(LIB_PATH)
    vp, ci, cf, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
    lib.mea_forward.argtypes = [vp, vp, vp, vp, vp, vp, vp, ci, ci, ci, ci, ci, ci, ci, cf, ci,
                                vp, ci, vp]
    lib.mea_forward.restype = ci
    lib.mea_forward_fp8.argtypes = [vp, vp, vp, vp, vp, vp, vp, ci, ci, ci, ci, ci, ci, ci, cf,
                                    ci, vp, cf, cf, cf, ci, vp]
    lib.mea_forward_fp8.restype = ci
    lib.mea_backward_workspace_size.argtypes = [ci, ci]
    lib.mea_backward_workspace_size.restype = sz
    lib.mea_backward.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, ci, ci, ci, ci, ci,
                                 ci, ci, ci, cf, ci, vp, ci, vp, sz, vp]
    lib.mea_backward.restype = ci
    lib.mea_decode_workspace_size.argtypes = [ci, ci, ci, ci, ci, ci]
    lib.mea_decode_workspace_size.restype = sz
    lib.mea_decode_splitkv.argtypes = [vp, vp, vp, vp, vp, vp, ci, ci, ci, ci, ci, ci, cf, ci, vp,
                                       ci, vp, sz, ci, vp]
    lib.mea_decode_splitkv.restype = ci
    lib.mea_decode_paged.argtypes = [vp, vp, vp, vp, vp, vp, vp, ci, ci, ci, ci, ci, ci, ci, ci,
                                     ci, cf, ci, vp, ci, vp, sz, ci, vp]
    lib.mea_decode_paged.restype = ci
    lib.mea_decode_splitkv_noalloc.argtypes = [vp, vp, vp, vp, vp, vp, ci, ci, ci, ci, ci, ci, cf,
                                               ci, vp, ci, ci, vp]
    lib.mea_decode_splitkv_noalloc.restype = ci
    lib.mea_status_string.argtypes = [ci]
    lib.mea_status_string.restype = ctypes.c_char_p
    lib.mea_device_error.argtypes = [ctypes.POINTER(ci), ci]
    lib.mea_device_error.restype = ci
    lib.mea_set_wait_timeout_ns.argtypes = [ctypes.c_ulonglong]
    lib.mea_set_wait_timeout_ns.restype = None
    lib.mea_wait_selftest.argtypes = [ctypes.c_ulonglong, ci, vp]
    lib.mea_wait_selftest.restype = ci
    lib.mea_version.argtypes = []
    lib.mea_version.restype = ctypes.c_char_p
    _lib = lib
    return lib


def status_string(rc: int) -> str:
    return load().mea_status_string(int(rc)).decode()


class MeaError(RuntimeError):
    def __init__(self, rc: int, where: str = ""):
        self.rc = rc
        super().__init__(f"{where}: {status_string(rc)} ({rc})" if where else status_string(rc))


def check(rc: int, where: str) -> None:
    if rc != MEA_OK:
        raise MeaError(rc, where)

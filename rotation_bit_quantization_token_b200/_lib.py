"""ctypes view of libfq.so (the C ABI in include/fq.h). Argument marshalling only."""

import ctypes
import os
import re

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libfq.so")
HEADER = os.path.join(os.path.dirname(HERE), "include", "fq.h")

FQ_OK = 0
FQ_ERR_NULLPTR = 161001
FQ_ERR_INVALID = 161002
FQ_ERR_CUDA = 161003
FQ_ERR_UNSUPPORTED = 161004
FQ_ERR_DEVICE_TIMEOUT = 161005

FQ_BF16, FQ_FP16 = 0, 1
FQ_OUT_INT4, FQ_OUT_INT32 = 0, 1
FQ_KERNEL_AUTO, FQ_KERNEL_GENERAL, FQ_KERNEL_TCGEN05 = 0, 1, 2

_vp = ctypes.c_void_p
_i64 = ctypes.c_int64
_int = ctypes.c_int
_dbl = ctypes.c_double

_SIGNATURES = {
    "fq_create": (_int, [ctypes.POINTER(_vp), _i64, _i64, _i64, _int]),
    "fq_destroy": (_int, [_vp]),
    "fq_quantize_per_token": (_int, [_vp, _vp, _vp, _vp, _dbl, _int, _vp, _vp, _vp]),
    "fq_quantize_mx": (_int, [_vp, _vp, _vp, _vp, _dbl, _vp, _vp, _vp]),
    "fq_debug_rotate": (_int, [_vp, _vp, _vp, _vp, _vp, _vp]),
    "fq_quantize_mx_static": (_int, [_i64, _i64, _i64, _int, _vp, _vp, _vp, _dbl, _vp, _vp, _vp]),
    "fq_mx_matmul": (_int, [_i64, _i64, _i64, _vp, _vp, _vp, _vp, _vp, _vp, _vp]),
    "fq_static_device_status": (_int, [ctypes.POINTER(ctypes.c_uint32)]),
    "fq_static_debug_arm_stall": (_int, [_dbl]),
    "fq_set_kernel": (_int, [_vp, _int]),
    "fq_set_intermediate_rounding": (_int, [_vp, _int]),
    "fq_debug_arm_stall": (_int, [_vp, _dbl]),
    "fq_last_kernel": (_int, [_vp]),
    "fq_last_launch_count": (_int, [_vp]),
    "fq_device_status": (_int, [_vp, ctypes.POINTER(ctypes.c_uint32)]),
    "fq_last_cuda_error": (_int, []),
    "fq_status_string": (ctypes.c_char_p, [_int]),
}

_lib = None


def declared_symbols(header=HEADER):
    """Names of the functions declared in include/fq.h."""
    with open(header) as f:
        text = f.read()
    return sorted(set(re.findall(r"^FQ_API\s+[\w\s\*]+?\b(fq_\w+)\s*\(", text, re.M)))


def load(path=LIB_PATH):
    """Load libfq.so (once) and set argument types. Raises if it is missing: there is no
    fallback implementation."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise ImportError(
            f"libfq.so not found at {path}; build it with "
            "`python -m rotation_bit_quantization_token_b200.build`")
    lib = ctypes.CDLL(path)
    for name, (res, args) in _SIGNATURES.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    _lib = lib
    return lib


class FQError(RuntimeError):
    def __init__(self, status, where):
        lib = load()
        msg = lib.fq_status_string(status).decode()
        if status == FQ_ERR_CUDA:
            msg += f" (cudaError {lib.fq_last_cuda_error()})"
        super().__init__(f"{where}: {msg}")
        self.status = status


def check(status, where):
    if status != FQ_OK:
        raise FQError(status, where)
    return status

"""ctypes loader for libaq.so (the C ABI in include/aq.h).

The library is built in-tree by build_lib.py.  There is no fallback: if the
shared library is missing or does not load, every call raises.
"""
import ctypes
import os

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libaq.so")
HEADER = os.path.join(os.path.dirname(HERE), "include", "aq.h")

AQ_OK, AQ_ERR_INVALID_ARG, AQ_ERR_UNSUPPORTED, AQ_ERR_MISALIGNED, AQ_ERR_CUDA, AQ_ERR_WORKSPACE = range(6)
STATUS_NAMES = {0: "AQ_OK", 1: "AQ_ERR_INVALID_ARG", 2: "AQ_ERR_UNSUPPORTED",
                3: "AQ_ERR_MISALIGNED", 4: "AQ_ERR_CUDA", 5: "AQ_ERR_WORKSPACE"}
AQ_F16, AQ_BF16 = 0, 1
AQ_MODE_AFFINE, AQ_MODE_FP4 = 0, 1
AQ_OP_QMV, AQ_OP_QMM, AQ_OP_QCONV2D, AQ_OP_QQMM, AQ_OP_QMM_NT = 0, 1, 2, 3, 4

_P = ctypes.c_void_p
_I = ctypes.c_int
_I64 = ctypes.c_int64
_SZ = ctypes.c_size_t

SIGNATURES = {
    "aq_quantize": (_I, [_P, _P, _P, _P, _I64, _I64, _I, _I, _I, _P]),
    "aq_dequantize": (_I, [_P, _P, _P, _P, _I64, _I64, _I, _I, _I, _I, _P]),
    "aq_quantize_fp4": (_I, [_P, _P, _P, _I64, _I64, _I, _I, _P]),
    "aq_quantize_dequantize_fp": (_I, [_P, _P, _I64, _I64, _I, _I, _I, _P]),
    "aq_qqmm": (_I, [_P, _P, _P, _P, _I64, _I64, _I64, _I, _I, _P, _SZ, _P]),
    "aq_qmv": (_I, [_P, _P, _P, _P, _P, _I64, _I64, _I64, _I, _I, _I, _I, _P, _SZ, _P]),
    "aq_qmm": (_I, [_P, _P, _P, _P, _P, _I64, _I64, _I64, _I, _I, _I, _I, _P, _SZ, _P]),
    "aq_qmm_nt": (_I, [_P, _P, _P, _P, _P, _I64, _I64, _I64, _I, _I, _I, _I, _P, _SZ, _P]),
    "aq_qmv_noalloc": (_I, [_P, _P, _P, _P, _P, _I64, _I64, _I64, _I, _I, _I, _I, _P]),
    "aq_qconv2d_nhwc": (_I, [_P, _P, _P, _P, _P] + [_I] * 15 + [_P, _SZ, _P]),
    "aq_workspace_size": (_SZ, [_I, _I64, _I64, _I64, _I, _I, _I, _I]),
    "aq_last_error": (ctypes.c_char_p, []),
    "aq_version": (_I, []),
    "aq_device_errors": (ctypes.c_uint, []),
    "aq_set_weight_prefetch": (None, [_I]),
    "aq_get_weight_prefetch": (_I, []),
    "aq_set_input_prefetch": (None, [_I]),
    "aq_get_input_prefetch": (_I, []),
    "aq_testing_set_wait_limit_ns": (None, [ctypes.c_uint64]),
    "aq_testing_set_start_delay_ns": (None, [ctypes.c_uint64]),
    "aq_testing_clear_device_errors": (_I, []),
    "aq_testing_set_qmv_kernel": (None, [_I]),
}



class QmvProblem(ctypes.Structure):
    """aq_qmv_problem (include/aq.h)."""
    _fields_ = [("x", _P), ("w_q", _P), ("scales", _P), ("biases", _P), ("y", _P),
                ("N", _I64), ("K", _I64)]


SIGNATURES["aq_qmv_batched"] = (_I, [ctypes.POINTER(QmvProblem), _I, _I64, _I, _I, _I, _I, _P,
                                     _SZ, _P])
SIGNATURES["aq_qmv_batched_workspace_size"] = (_SZ, [ctypes.POINTER(QmvProblem), _I, _I64, _I,
                                                     _I, _I])
_I32P = ctypes.POINTER(ctypes.c_int32)
SIGNATURES["aq_gather_qmm"] = (_I, [_P, _P, _P, _P, _I32P, _I32P, _P, _I64, _I64, _I64, _I64, _I64,
                                    _I64, _I, _I, _I, _I, _P, _SZ, _P])
SIGNATURES["aq_gather_qmm_workspace_size"] = (_SZ, [_I64, _I64, _I64, _I64, _I, _I, _I])
SIGNATURES["aq_testing_gather_groups"] = (_I, [_I32P, _I32P, _I64, _I64, _I64, _I64, _I64, _I32P,
                                               _I32P, _I64, ctypes.POINTER(_I)])

_lib = None


class AqError(RuntimeError):
    def __init__(self, status, fn, msg):
        self.status = status
        super().__init__("%s returned %s: %s" % (fn, STATUS_NAMES.get(status, status), msg))


def lib():
    """The loaded libaq.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError("libaq.so not found at %s; build it with "
                              "group_wise_affine_quant_b200/build_lib.py" % LIB_PATH)
        handle = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(handle, name)
            fn.restype = res
            fn.argtypes = args
        _lib = handle
    return _lib


def check(status, fn):
    if status != AQ_OK:
        raise AqError(status, fn, lib().aq_last_error().decode())


def declared_symbols():
    """Names of the functions the headers under include/ declare with AQ_API."""
    import glob
    import re
    names = []
    for path in sorted(glob.glob(os.path.join(os.path.dirname(HEADER), "*.h"))):
        with open(path) as f:
            names += re.findall(r"AQ_API\s+[\w\s\*]+?\b(aq_\w+)\s*\(", f.read())
    return names

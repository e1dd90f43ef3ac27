"""ctypes declarations of libtq's C ABI (include/tq.h).  Loading fails loudly
if the shared library has not been built: there is no fallback path."""
from __future__ import annotations

import ctypes as C
import os

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libtq.so")

TQ_OK = 0
STATUS = {
    0: "TQ_OK", 1: "TQ_ERR_INVALID_ARG", 2: "TQ_ERR_UNSUPPORTED", 3: "TQ_ERR_CUDA",
    4: "TQ_ERR_TIMEOUT", 5: "TQ_ERR_INTERNAL", 6: "TQ_ERR_WORKSPACE",
}

F32, F16, BF16 = 0, 1, 2
ROT_HADAMARD, ROT_DENSE = 0, 1
MODE_MSE, MODE_PROD, MODE_MSE_UNBIASED = 0, 1, 2
STORE_RNORM_F16 = 0x100  # OR'ed into MODE_PROD: residual norms stored as fp16
LAYOUT_ROW, LAYOUT_BLOCK32 = 0, 1

# exported symbol -> (restype, argtypes)
_vp, _i, _i64, _f, _sz = C.c_void_p, C.c_int, C.c_int64, C.c_float, C.c_size_t
_fp = C.POINTER(C.c_float)
SIGNATURES = {
    "tq_status_string": (C.c_char_p, [_i]),
    "tq_version": (C.c_char_p, []),
    "tq_build_codebook": (_i, [_i, _i, _fp, _fp]),
    "tq_make_rotation": (_i, [_i, _vp, _fp]),
    "tq_params_create": (_i, [_i, _i, _i, _i, _i, _vp, _vp, _vp, C.POINTER(_vp)]),
    "tq_params_destroy": (_i, [_vp]),
    "tq_params_info": (_i, [_vp] + [C.POINTER(_i)] * 5),
    "tq_params_tables": (_i, [_vp, _fp, _fp, _fp]),
    "tq_encode_workspace_size": (_i, [_vp, _i64, C.POINTER(_sz)]),
    "tq_encode_mse": (_i, [_vp, _vp, _i, _i64, _i64, _i64, _i64, _i, _vp, _vp, _vp, _sz, _vp]),
    "tq_encode_prod": (_i, [_vp, _vp, _i, _i64, _i64, _i64, _i64, _vp, _vp, _vp, _vp, _vp, _sz, _vp]),
    "tq_decode": (_i, [_vp, _i, _vp, _vp, _vp, _vp, _i64, _i64, _i64, _vp, _i64, _vp]),
    "tq_scores_workspace_size": (_i, [_vp, _i64, _i64, _i, C.POINTER(_sz)]),
    "tq_scores": (_i, [_vp, _vp, _i64, _i64, _vp, _vp, _vp, _vp, _i64, _vp, _i, _vp, _vp, _vp, _sz, _vp]),
    "tq_decode_attention_workspace_size": (_i, [_vp, _vp, _i, _i, _i, _i, _i64, C.POINTER(_sz)]),
    "tq_decode_attention": (_i, [_vp, _vp, _vp, _i, _i, _i, _i, _i64, _i64, _f,
                                 _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _sz, _vp]),
    "tq_decode_attention_noalloc": (_i, [_vp, _vp, _vp, _i, _i, _i, _i, _i64, _i64, _f,
                                         _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp]),
    "tq_decode_step_workspace_size": (_i, [_vp, _vp, _i, _i, _i, _i, _i64, C.POINTER(_sz)]),
    "tq_decode_step": (_i, [_vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i64, _i64, _f,
                            _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _sz, _vp]),
    "tq_sync_check": (_i, [_vp]),
    "tq_check_wait_expiry": (_i, [C.c_int64, _vp]),
}


class TQError(RuntimeError):
    def __init__(self, fn, status):
        self.status = status
        super().__init__(f"{fn} failed: {STATUS.get(status, status)}")


_lib = None


def lib():
    """Load libtq.so (raises if it is missing -- build it with
    ``python -m vector_compression_b200.build``)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"libtq.so not built at {LIB_PATH}; run python -m vector_compression_b200.build")
        handle = C.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(handle, name)
            fn.restype = res
            fn.argtypes = args
        _lib = handle
    return _lib


def check(fn_name, status):
    if status != TQ_OK:
        raise TQError(fn_name, status)

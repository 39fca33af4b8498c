"""ctypes binding of libdspark_markov.so (declarations in include/dspark_markov.h).

Argument marshalling only. Loading fails loudly when the library has not been
built: there is no CPU or PyTorch fallback for any entry point.
"""
from __future__ import annotations

import ctypes
import os
import threading

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libdspark_markov.so")

DSPARK_OK = 0
DSPARK_ERR_INVALID_ARG = 1
DSPARK_ERR_UNSUPPORTED = 2
DSPARK_ERR_CUDA = 3

DSPARK_STATUS_TOKEN_RANGE = 1
DSPARK_STATUS_TIMEOUT = 2

DSPARK_DTYPE_FP32 = 0
DSPARK_DTYPE_BF16 = 1

DSPARK_ALGO_AUTO = 0
DSPARK_ALGO_GENERIC = 1
DSPARK_ALGO_TENSOR_CORE = 2

DSPARK_DEBUG_SKIP_BARRIER_ARRIVAL = 1
DSPARK_DEBUG_APPLY_WIDE = 2
DSPARK_DEBUG_SAMPLE_ROWS = 4
DSPARK_DEBUG_SAMPLE_TILE = 8

DSPARK_NOALLOC_MAX_KEYS = 8192

DSPARK_VARIANT_BWD_RESIDENT_W1 = 1
DSPARK_VARIANT_SAMPLE_ROWS = 2
DSPARK_VARIANT_APPLY_WIDE = 4

# Every symbol include/dspark_markov.h declares, with its ctypes signature.
_vp, _i64, _i32, _u32, _u64, _f32 = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int32, ctypes.c_uint32, ctypes.c_uint64, ctypes.c_float
SIGNATURES = {
    "dspark_markov_apply_block_logits": (ctypes.c_int, [_vp, _vp, _vp, _i64, _i64, _vp, _vp, _i32, _i32, _i32, _vp]),
    "dspark_markov_sample_block": (ctypes.c_int, [_vp, _vp, _i64, _i64, _i64, _vp, _vp, _i32, _f32, _u64, _vp, _vp,
                                                  _i32, _i32, _vp]),
    "dspark_markov_apply_block_logits_backward": (ctypes.c_int, [_vp, _vp, _i64, _i64, _vp, _vp, _i32, _vp, _vp,
                                                                 _i32, _i32, _i32, _vp]),
    "dspark_markov_transition_logits": (ctypes.c_int, [_vp, _i64, _i64, _vp, _vp, _i32, _vp, _vp, _i32, _vp]),
    "dspark_markov_fused_lm_head_logits": (ctypes.c_int, [_vp, _vp, _i64, _i64, _i64, _vp, _vp, _vp, _i32, _vp,
                                                          _i32, _i32, _vp]),
    "dspark_markov_sample_block_noalloc": (ctypes.c_int, [_vp, _vp, _i64, _i64, _i64, _vp, _vp, _i32, _f32, _u64,
                                                          _vp, _vp, _i32, _i32, _vp]),
    "dspark_markov_get_status": (ctypes.c_int, [_vp, ctypes.POINTER(ctypes.c_int32)]),
    "dspark_markov_strerror": (ctypes.c_char_p, [ctypes.c_int]),
    "dspark_markov_set_algo": (_i32, [_i32]),
    "dspark_markov_launch_count": (_i64, []),
    "dspark_markov_set_debug": (ctypes.c_int, [_u32, _u64]),
    "dspark_markov_last_algo": (_i32, []),
    "dspark_markov_last_variant": (_i32, []),
    "dspark_markov_debug_gumbel": (ctypes.c_int, [_vp, _vp, _i64, _vp]),
}

_lib = None
_lock = threading.Lock()


class DSparkError(RuntimeError):
    def __init__(self, code: int, where: str):
        self.code = code
        super().__init__(f"{where}: {strerror(code)} (code {code})")


def load(path: str = LIB_PATH) -> ctypes.CDLL:
    """Load the library once. Raises if it is missing (build it with
    ``python -m rank_markov_draft_vanillamarkov_b200.build``)."""
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(path):
                raise RuntimeError(f"CUDA library not built: {path} is missing; run "
                                   "`python -m rank_markov_draft_vanillamarkov_b200.build`")
            lib = ctypes.CDLL(path)
            for name, (res, args) in SIGNATURES.items():
                fn = getattr(lib, name)
                fn.restype = res
                fn.argtypes = args
            _lib = lib
    return _lib


def strerror(code: int) -> str:
    try:
        return load().dspark_markov_strerror(code).decode()
    except Exception:
        return "error"


def check(code: int, where: str) -> None:
    if code != DSPARK_OK:
        raise DSparkError(code, where)

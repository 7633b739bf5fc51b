"""ctypes loader for libtbq4.so (the C ABI in include/tbq4.h).

The library must have been built in-tree (``python
long_context_attention_tbq4_b200/build.py``); if it is missing this module
raises at import, there is no fallback implementation.  With TBQ4_DEBUG=1 in
the environment the debug build (libtbq4_debug.so, ``build.py --debug``: the
kernels' bounds checks switched on) is loaded instead.
"""
import ctypes as C
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
DEBUG = os.environ.get("TBQ4_DEBUG", "0") == "1"
LIB_PATH = os.path.join(_HERE, "libtbq4_debug.so" if DEBUG else "libtbq4.so")

# Every symbol include/tbq4.h declares, with (restype, argtypes).
_p, _i, _i32, _i64, _u64, _f, _sz = (C.c_void_p, C.c_int, C.c_int32, C.c_int64,
                                     C.c_uint64, C.c_float, C.c_size_t)
SIGNATURES = {
    "tbq4_block_bytes": (_sz, []),
    "tbq4_cache_bytes": (_sz, [_i, _i, _i64]),
    "tbq4_signs": (None, [_u64, _p]),
    "tbq4_quantize_append": (_i, [_p, _i, _i, _i, _p, _i64, _u64, _p, _p]),
    "tbq4_decode_workspace_bytes": (_sz, [_i, _i, _i, _i32]),
    "tbq4_attn_decode": (_i, [_p, _p, _p, _p, _i32, _i, _i, _i, _i64, _f, _u64,
                              _p, _sz, _p, _p]),
    "tbq4_attn_decode_append": (_i, [_p, _p, _p, _p, _p, _p, _i32, _i, _i, _i, _i64, _f,
                                     _u64, _p, _sz, _p, _p]),
    "tbq4_quantize_append_paged": (_i, [_p, _i, _i, _i, _p, _p, _i, _i, _i64, _u64, _p, _p]),
    "tbq3_block_bytes": (_sz, []),
    "tbq3_cache_bytes": (_sz, [_i, _i, _i64]),
    "tbq3_quantize_append": (_i, [_p, _i, _i, _i, _p, _i64, _u64, _p, _p]),
    "tbq3_attn_decode": (_i, [_p, _p, _p, _p, _i32, _i, _i, _i, _i64, _f, _u64, _p, _sz, _p, _p]),
    "tbq4_attn_decode_paged": (_i, [_p, _p, _p, _p, _p, _p, _i, _i, _i64, _p, _i32, _i, _i, _i,
                                    _f, _u64, _p, _sz, _p, _p]),
    "tbq4_decode_workspace_bytes_split": (_sz, [_i, _i, _i, _i32, _i32]),
    "tbq4_decode_mq_workspace_bytes": (_sz, [_i, _i, _i, _i, _i32]),
    "tbq4_attn_decode_mq": (_i, [_p, _p, _p, _p, _i32, _i, _i, _i, _i, _i64, _f, _u64, _p, _sz,
                                 _p, _p]),
    "tbq4_attn_decode_split": (_i, [_p, _p, _p, _p, _i32, _i, _i, _i, _i64, _f,
                                    _u64, _i32, _p, _sz, _p, _p]),
    "tbq4_attn_decode_noalloc": (_i, [_p, _p, _p, _p, _i32, _i, _i, _i, _i64, _f, _u64,
                                      _p, _p]),
    "tbq4_prefill_workspace_bytes": (_sz, [_i, _i, _i, _i64]),
    "tbq4_attn_prefill_chunk": (_i, [_p, _i, _i64, _p, _p, _i, _i, _i64, _f,
                                     _u64, _p, _sz, _p, _p]),
    "tbq4_set_timing_events": (None, [_p, _p]),
    "tbq4_get_device_status": (_i, [_p]),
    "tbq4_selftest_bounded_wait": (_i, [C.c_uint32, _p]),
    "tbq4_status_string": (C.c_char_p, [_i]),
}

STATUS_NAMES = {0: "TBQ4_OK", 1: "TBQ4_ERR_NULL", 2: "TBQ4_ERR_ALIGN",
                3: "TBQ4_ERR_SHAPE", 4: "TBQ4_ERR_CAPACITY",
                5: "TBQ4_ERR_WORKSPACE", 6: "TBQ4_ERR_LAUNCH",
                7: "TBQ4_ERR_DEVICE_TIMEOUT", 8: "TBQ4_ERR_BOUNDS"}


class Tbq4Error(RuntimeError):
    def __init__(self, code, what=""):
        self.code = int(code)
        name = STATUS_NAMES.get(self.code, str(code))
        super().__init__(f"{what}: {name}" if what else name)


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(
            f"{LIB_PATH} is missing: build the CUDA library with "
            "`python long_context_attention_tbq4_b200/build.py"
            + (" --debug" if DEBUG else "") + "` (there is no CPU fallback)")
    L = C.CDLL(LIB_PATH)
    for name, (res, args) in SIGNATURES.items():
        fn = getattr(L, name)
        fn.restype = res
        fn.argtypes = args
    return L


lib = _load()


def check(code, what=""):
    if code != 0:
        raise Tbq4Error(code, what)

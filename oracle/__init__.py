"""fp64 CPU oracle for TBQ4 long-context attention -- TEST INFRASTRUCTURE.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The product path (the CUDA library and
its binding) never imports it and shares no code with it.

The arithmetic lives in ``tbq4_oracle.c`` (plain C, fp64 for attention,
explicit binary32 steps where the block encoding defines them); this module
only marshals numpy arrays through ctypes.  ``brute.py`` holds pure-Python
versions for tiny inputs that pin the C code.

Source: trefon.com, "Kontekst 262K na jednej RTX 4090: co dodalem do
llama.cpp-turboq", section "Od czego zaczalem" (TBQ4: 128 values in 66 bytes,
2-byte scale + 64 bytes of 4-bit indices, attention in the Hadamard-rotated
domain).  The codebook is fixed by this library: R = H*D/sqrt(128), scale =
fp16(max|x_rot|), levels (i - 7.5)/7.5 * scale by round-to-nearest-even.
"""
import ctypes as C

import numpy as np

from . import build as _build

BLOCK_BYTES = 66
BLOCK_BYTES3 = 50       # the 3-bit variant (TBQ3)
D = 128

_lib = None


def lib():
    global _lib
    if _lib is None:
        path = _build.build()
        L = C.CDLL(path)
        p = C.c_void_p
        L.oracle_set_threads.argtypes = [C.c_int]
        L.oracle_get_threads.restype = C.c_int
        L.oracle_block_bytes.restype = C.c_int
        L.oracle_splitmix64.argtypes = [C.c_uint64, C.c_int, p]
        L.oracle_signs.argtypes = [C.c_uint64, p]
        L.oracle_f32_to_f16_bits.argtypes = [C.c_float]
        L.oracle_f32_to_f16_bits.restype = C.c_uint16
        L.oracle_f32_to_f16_array.argtypes = [p, C.c_int64, p]
        L.oracle_f16_bits_to_f64.argtypes = [C.c_uint16]
        L.oracle_f16_bits_to_f64.restype = C.c_double
        L.oracle_hadamard_entry.argtypes = [C.c_int, C.c_int]
        L.oracle_hadamard_entry.restype = C.c_int
        L.oracle_rotation_matrix.argtypes = [p, p]
        L.oracle_rotate_f32.argtypes = [p, p, p]
        L.oracle_level_index.argtypes = [C.c_float, C.c_float]
        L.oracle_level_index.restype = C.c_int
        L.oracle_block_scale_bits.argtypes = [p]
        L.oracle_block_scale_bits.restype = C.c_uint16
        L.oracle_quantize_block.argtypes = [p, p, p]
        L.oracle_dequant_block.argtypes = [p, p]
        L.oracle_quantize_append.argtypes = [p, C.c_int, C.c_int, C.c_int, p,
                                             C.c_int64, C.c_uint64, p]
        L.oracle_quantize_append.restype = C.c_int64
        L.oracle_attn_decode.argtypes = [p, p, p, p, C.c_int, C.c_int, C.c_int,
                                         C.c_int64, C.c_double, C.c_uint64, p,
                                         C.c_int, p]
        L.oracle_attn_prefill.argtypes = [p, C.c_int, C.c_int64, p, p, C.c_int,
                                          C.c_int, C.c_int64, C.c_double,
                                          C.c_uint64, p, C.c_int, p]
        L.oracle_block_bytes3.restype = C.c_int
        L.oracle_level_index3.argtypes = [C.c_float, C.c_float]
        L.oracle_level_index3.restype = C.c_int
        L.oracle_quantize_block3.argtypes = [p, p, p]
        L.oracle_dequant_block3.argtypes = [p, p]
        L.oracle_quantize_append3.argtypes = [p, C.c_int, C.c_int, C.c_int, p,
                                              C.c_int64, C.c_uint64, p]
        L.oracle_quantize_append3.restype = C.c_int64
        L.oracle_attn_decode3.argtypes = [p, p, p, p, C.c_int, C.c_int, C.c_int,
                                          C.c_int64, C.c_double, C.c_uint64, p,
                                          C.c_int, p]
        _lib = L
    return _lib


def _ptr(a):
    return a.ctypes.data_as(C.c_void_p)


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


def set_threads(n: int) -> None:
    lib().oracle_set_threads(int(n))


def get_threads() -> int:
    return int(lib().oracle_get_threads())


def splitmix64(seed: int, n: int) -> np.ndarray:
    out = np.zeros(n, np.uint64)
    lib().oracle_splitmix64(C.c_uint64(seed), n, _ptr(out))
    return out


def signs(seed: int) -> np.ndarray:
    out = np.zeros(D, np.int8)
    lib().oracle_signs(C.c_uint64(seed), _ptr(out))
    return out


def f32_to_f16_bits(x: float) -> int:
    return int(lib().oracle_f32_to_f16_bits(C.c_float(x)))


def f32_to_f16_array(x: np.ndarray) -> np.ndarray:
    x = _c(x, np.float32).ravel()
    out = np.zeros(x.size, np.uint16)
    lib().oracle_f32_to_f16_array(_ptr(x), x.size, _ptr(out))
    return out


def f16_bits_to_f64(h: int) -> float:
    return float(lib().oracle_f16_bits_to_f64(C.c_uint16(h)))


def hadamard_entry(i: int, j: int) -> int:
    return int(lib().oracle_hadamard_entry(i, j))


def rotation_matrix(s: np.ndarray) -> np.ndarray:
    s = _c(s, np.int8)
    R = np.zeros((D, D), np.float64)
    lib().oracle_rotation_matrix(_ptr(s), _ptr(R))
    return R


def rotate_f32(x: np.ndarray, s: np.ndarray) -> np.ndarray:
    x = _c(x, np.float32)
    s = _c(s, np.int8)
    out = np.zeros(D, np.float32)
    lib().oracle_rotate_f32(_ptr(x), _ptr(s), _ptr(out))
    return out


def level_index(x_rot: float, S: float) -> int:
    return int(lib().oracle_level_index(C.c_float(x_rot), C.c_float(S)))


def block_scale_bits(x_rot: np.ndarray) -> int:
    x_rot = _c(x_rot, np.float32)
    return int(lib().oracle_block_scale_bits(_ptr(x_rot)))


def quantize_block(x: np.ndarray, s: np.ndarray) -> np.ndarray:
    x = _c(x, np.float32)
    s = _c(s, np.int8)
    out = np.zeros(BLOCK_BYTES, np.uint8)
    lib().oracle_quantize_block(_ptr(x), _ptr(s), _ptr(out))
    return out


def dequant_block(blk: np.ndarray) -> np.ndarray:
    blk = _c(blk, np.uint8)
    out = np.zeros(D, np.float64)
    lib().oracle_dequant_block(_ptr(blk), _ptr(out))
    return out


def quantize_append(src: np.ndarray, start_pos, capacity: int, seed: int,
                    cache: np.ndarray) -> int:
    """src [B][n_new][Hkv][128] fp32; cache [B][Hkv][capacity][66] uint8
    (updated in place).  Returns the number of rows skipped as out of range."""
    src = _c(src, np.float32)
    B, n_new, Hkv, d = src.shape
    assert d == D and cache.dtype == np.uint8 and cache.flags.c_contiguous
    assert cache.shape == (B, Hkv, capacity, BLOCK_BYTES)
    sp = _c(start_pos, np.int32)
    return int(lib().oracle_quantize_append(_ptr(src), B, n_new, Hkv, _ptr(sp),
                                            capacity, C.c_uint64(seed),
                                            _ptr(cache)))


def attn_decode(q, k_cache, v_cache, seq_lens, softmax_scale, seed,
                rows=None) -> np.ndarray:
    """q [B][Hq][128] fp32; caches [B][Hkv][capacity][66]; returns
    [B][Hq][128] float64 (rows not listed in ``rows`` are NaN)."""
    q = _c(q, np.float32)
    B, Hq, d = q.shape
    _, Hkv, cap, nb = k_cache.shape
    assert d == D and nb == BLOCK_BYTES and v_cache.shape == k_cache.shape
    k_cache = _c(k_cache, np.uint8)
    v_cache = _c(v_cache, np.uint8)
    sl = _c(seq_lens, np.int32)
    out = np.full((B, Hq, D), np.nan, np.float64)
    if rows is None:
        rp, nr = None, 0
    else:
        rows = _c(rows, np.int32)
        rp, nr = _ptr(rows), len(rows)
    lib().oracle_attn_decode(_ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(sl),
                             B, Hq, Hkv, cap, float(softmax_scale),
                             C.c_uint64(seed), rp, nr, _ptr(out))
    return out


def attn_prefill(q, n_cached, k_cache, v_cache, softmax_scale, seed,
                 rows=None) -> np.ndarray:
    """q [n_new][Hq][128] (bf16 values as float32); caches
    [Hkv][capacity][66]; returns [n_new][Hq][128] float64."""
    q = _c(q, np.float32)
    n_new, Hq, d = q.shape
    Hkv, cap, nb = k_cache.shape
    assert d == D and nb == BLOCK_BYTES and v_cache.shape == k_cache.shape
    k_cache = _c(k_cache, np.uint8)
    v_cache = _c(v_cache, np.uint8)
    out = np.full((n_new, Hq, D), np.nan, np.float64)
    if rows is None:
        rp, nr = None, 0
    else:
        rows = _c(rows, np.int32)
        rp, nr = _ptr(rows), len(rows)
    lib().oracle_attn_prefill(_ptr(q), n_new, int(n_cached), _ptr(k_cache),
                              _ptr(v_cache), Hq, Hkv, cap, float(softmax_scale),
                              C.c_uint64(seed), rp, nr, _ptr(out))
    return out


# ---------------------------------------------------------------- TBQ3
# The 3-bit variant: 128 values in 50 bytes (fp16 scale, then 16 groups of 8
# indices as 24-bit little-endian words), levels S*(2i-7)/7.  See
# tbq4_oracle.c for the layout this library fixes.
def block_bytes3() -> int:
    return int(lib().oracle_block_bytes3())


def level_index3(x_rot: float, S: float) -> int:
    return int(lib().oracle_level_index3(C.c_float(x_rot), C.c_float(S)))


def quantize_block3(x: np.ndarray, s: np.ndarray) -> np.ndarray:
    x = _c(x, np.float32)
    s = _c(s, np.int8)
    out = np.zeros(BLOCK_BYTES3, np.uint8)
    lib().oracle_quantize_block3(_ptr(x), _ptr(s), _ptr(out))
    return out


def dequant_block3(blk: np.ndarray) -> np.ndarray:
    blk = _c(blk, np.uint8)
    out = np.zeros(D, np.float64)
    lib().oracle_dequant_block3(_ptr(blk), _ptr(out))
    return out


def quantize_append3(src: np.ndarray, start_pos, capacity: int, seed: int,
                     cache: np.ndarray) -> int:
    """src [B][n_new][Hkv][128] fp32; cache [B][Hkv][capacity][50] uint8
    (updated in place).  Returns the number of rows skipped as out of range."""
    src = _c(src, np.float32)
    B, n_new, Hkv, d = src.shape
    assert d == D and cache.dtype == np.uint8 and cache.flags.c_contiguous
    assert cache.shape == (B, Hkv, capacity, BLOCK_BYTES3)
    sp = _c(start_pos, np.int32)
    return int(lib().oracle_quantize_append3(_ptr(src), B, n_new, Hkv, _ptr(sp),
                                             capacity, C.c_uint64(seed), _ptr(cache)))


def attn_decode3(q, k_cache, v_cache, seq_lens, softmax_scale, seed,
                 rows=None) -> np.ndarray:
    """q [B][Hq][128] fp32; 3-bit caches [B][Hkv][capacity][50]; returns
    [B][Hq][128] float64 (rows not listed in ``rows`` are NaN)."""
    q = _c(q, np.float32)
    B, Hq, d = q.shape
    _, Hkv, cap, nb = k_cache.shape
    assert d == D and nb == BLOCK_BYTES3 and v_cache.shape == k_cache.shape
    k_cache = _c(k_cache, np.uint8)
    v_cache = _c(v_cache, np.uint8)
    sl = _c(seq_lens, np.int32)
    out = np.full((B, Hq, D), np.nan, np.float64)
    if rows is None:
        rp, nr = None, 0
    else:
        rows = _c(rows, np.int32)
        rp, nr = _ptr(rows), len(rows)
    lib().oracle_attn_decode3(_ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(sl),
                              B, Hq, Hkv, cap, float(softmax_scale),
                              C.c_uint64(seed), rp, nr, _ptr(out))
    return out


"""TBQ4 long-context attention on NVIDIA B200 (sm_100a).

A thin binding over libtbq4.so (include/tbq4.h): every function here only
checks and marshals torch tensors (device memory, current stream) and calls
the C ABI of the same name; all arithmetic runs in the library's CUDA
kernels.  There is no CPU path.

TBQ4 stores 128 values in 66 bytes (2-byte scale + 64 bytes of 4-bit
indices) in a Hadamard-rotated domain, and attention dequantises the raw
blocks inside its inner loop (trefon.com, "Kontekst 262K na jednej RTX 4090:
co dodalem do llama.cpp-turboq", section "Od czego zaczalem").
"""
import ctypes as C

import numpy as np
import torch

from ._lib import LIB_PATH, STATUS_NAMES, Tbq4Error, check, lib

D = 128
BLOCK_BYTES = 66

__all__ = [
    "D", "BLOCK_BYTES", "LIB_PATH", "Tbq4Error", "tbq4_block_bytes",
    "tbq4_cache_bytes", "tbq4_signs", "tbq4_quantize_append",
    "tbq4_decode_workspace_bytes", "tbq4_attn_decode", "tbq4_attn_decode_append",
    "tbq4_decode_mq_workspace_bytes", "tbq4_attn_decode_mq",
    "tbq4_prefill_workspace_bytes", "tbq4_attn_prefill_chunk",
    "tbq4_set_timing_events", "tbq4_get_device_status", "tbq4_selftest_bounded_wait",
    "empty_cache",
    "empty_pool", "tbq4_quantize_append_paged", "tbq4_attn_decode_paged",
    "BLOCK_BYTES3", "empty_cache3", "tbq3_quantize_append", "tbq3_attn_decode",
]


def _ptr(t):
    return C.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return C.c_void_p(stream.cuda_stream)


def _need(t, dtype, name, ndim=None):
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise TypeError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if ndim is not None and t.dim() != ndim:
        raise ValueError(f"{name} must have {ndim} dims, got {tuple(t.shape)}")


def tbq4_block_bytes() -> int:
    return int(lib.tbq4_block_bytes())


def tbq4_cache_bytes(batch: int, n_kv_heads: int, capacity: int) -> int:
    return int(lib.tbq4_cache_bytes(batch, n_kv_heads, capacity))


def tbq4_signs(seed: int) -> np.ndarray:
    out = np.zeros(D, np.int8)
    lib.tbq4_signs(C.c_uint64(seed), out.ctypes.data_as(C.c_void_p))
    return out


def empty_cache(batch, n_kv_heads, capacity, device="cuda"):
    """An uninitialised [B][Hkv][capacity][66] uint8 cache (capacity % 8 == 0)."""
    return torch.empty((batch, n_kv_heads, capacity, BLOCK_BYTES), dtype=torch.uint8,
                       device=device)


def tbq4_quantize_append(src, start_pos, cache, sign_seed=0, stream=None):
    """src fp32 [B][n_new][Hkv][128]; start_pos int32 [B]; cache uint8
    [B][Hkv][capacity][66] (written in place)."""
    _need(src, torch.float32, "src", 4)
    _need(start_pos, torch.int32, "start_pos", 1)
    _need(cache, torch.uint8, "cache", 4)
    B, n_new, Hkv, d = src.shape
    if d != D or tuple(cache.shape[:2]) != (B, Hkv) or cache.shape[3] != BLOCK_BYTES:
        raise ValueError("shape mismatch between src and cache")
    check(lib.tbq4_quantize_append(_ptr(src), B, n_new, Hkv, _ptr(start_pos),
                                   cache.shape[2], C.c_uint64(sign_seed), _ptr(cache),
                                   _stream(stream)), "tbq4_quantize_append")
    return cache


def tbq4_decode_workspace_bytes(B, Hq, Hkv, max_len, split_tokens=0) -> int:
    return int(lib.tbq4_decode_workspace_bytes_split(B, Hq, Hkv, max_len, split_tokens))


def tbq4_attn_decode(q, k_cache, v_cache, seq_lens, max_len, softmax_scale,
                     sign_seed=0, workspace=None, out=None, split_tokens=0,
                     stream=None):
    """q fp32 [B][Hq][128]; caches uint8 [B][Hkv][capacity][66]; seq_lens
    int32 [B] (device); returns fp16 [B][Hq][128]."""
    _need(q, torch.float32, "q", 3)
    _need(k_cache, torch.uint8, "k_cache", 4)
    _need(v_cache, torch.uint8, "v_cache", 4)
    _need(seq_lens, torch.int32, "seq_lens", 1)
    B, Hq, d = q.shape
    _, Hkv, cap, nb = k_cache.shape
    if d != D or nb != BLOCK_BYTES or v_cache.shape != k_cache.shape or k_cache.shape[0] != B:
        raise ValueError("shape mismatch between q and caches")
    need = tbq4_decode_workspace_bytes(B, Hq, Hkv, max_len, split_tokens)
    if workspace is None:
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=q.device)
    if out is None:
        out = torch.empty((B, Hq, D), dtype=torch.float16, device=q.device)
    _need(out, torch.float16, "out", 3)
    check(lib.tbq4_attn_decode_split(
        _ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(seq_lens), int(max_len), B, Hq, Hkv,
        cap, float(softmax_scale), C.c_uint64(sign_seed), int(split_tokens),
        _ptr(workspace), workspace.numel() * workspace.element_size(), _ptr(out),
        _stream(stream)), "tbq4_attn_decode")
    return out


def tbq4_attn_decode_append(q, k_new, v_new, k_cache, v_cache, seq_lens, max_len,
                            softmax_scale, sign_seed=0, workspace=None, out=None, stream=None):
    """One decode step: k_new / v_new fp32 [B][Hkv][128] are encoded into the
    caches at position seq_lens[b]-1, then decode attention over seq_lens[b]
    keys; returns fp16 [B][Hq][128]."""
    _need(q, torch.float32, "q", 3)
    _need(k_new, torch.float32, "k_new", 3)
    _need(v_new, torch.float32, "v_new", 3)
    _need(k_cache, torch.uint8, "k_cache", 4)
    _need(v_cache, torch.uint8, "v_cache", 4)
    _need(seq_lens, torch.int32, "seq_lens", 1)
    B, Hq, d = q.shape
    _, Hkv, cap, nb = k_cache.shape
    if (d != D or nb != BLOCK_BYTES or v_cache.shape != k_cache.shape or k_cache.shape[0] != B
            or tuple(k_new.shape) != (B, Hkv, D) or tuple(v_new.shape) != (B, Hkv, D)):
        raise ValueError("shape mismatch between q, new rows and caches")
    need = tbq4_decode_workspace_bytes(B, Hq, Hkv, max_len)
    if workspace is None:
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=q.device)
    if out is None:
        out = torch.empty((B, Hq, D), dtype=torch.float16, device=q.device)
    _need(out, torch.float16, "out", 3)
    check(lib.tbq4_attn_decode_append(
        _ptr(q), _ptr(k_new), _ptr(v_new), _ptr(k_cache), _ptr(v_cache), _ptr(seq_lens),
        int(max_len), B, Hq, Hkv, cap, float(softmax_scale), C.c_uint64(sign_seed),
        _ptr(workspace), workspace.numel() * workspace.element_size(), _ptr(out),
        _stream(stream)), "tbq4_attn_decode_append")
    return out


def empty_pool(n_pages, n_kv_heads, page_size, device="cuda"):
    """An uninitialised page pool [n_pages][Hkv][page_size][66] uint8
    (page_size a multiple of 32)."""
    return torch.empty((n_pages, n_kv_heads, page_size, BLOCK_BYTES), dtype=torch.uint8,
                       device=device)


def _pool_shape(pool, name):
    _need(pool, torch.uint8, name, 4)
    n_pages, Hkv, page_size, nb = pool.shape
    if nb != BLOCK_BYTES:
        raise ValueError(f"{name}: last dimension must be {BLOCK_BYTES}")
    return n_pages, Hkv, page_size


def tbq4_quantize_append_paged(src, start_pos, block_table, pool, sign_seed=0, stream=None):
    """src fp32 [B][n_new][Hkv][128]; start_pos int32 [B]; block_table int32
    [B][max_pages]; pool uint8 [n_pages][Hkv][page_size][66] (written)."""
    _need(src, torch.float32, "src", 4)
    _need(start_pos, torch.int32, "start_pos", 1)
    _need(block_table, torch.int32, "block_table", 2)
    n_pages, Hkv, page_size = _pool_shape(pool, "pool")
    B, n_new, h, d = src.shape
    if d != D or h != Hkv or block_table.shape[0] != B:
        raise ValueError("shape mismatch between src, block_table and pool")
    check(lib.tbq4_quantize_append_paged(
        _ptr(src), B, n_new, Hkv, _ptr(start_pos), _ptr(block_table), block_table.shape[1],
        page_size, n_pages, C.c_uint64(sign_seed), _ptr(pool), _stream(stream)),
        "tbq4_quantize_append_paged")
    return pool


def tbq4_attn_decode_paged(q, k_pool, v_pool, block_table, seq_lens, max_len, softmax_scale,
                           sign_seed=0, k_new=None, v_new=None, workspace=None, out=None,
                           stream=None):
    """Decode attention over paged caches: q fp32 [B][Hq][128]; pools uint8
    [n_pages][Hkv][page_size][66]; block_table int32 [B][max_pages]; with
    k_new / v_new (fp32 [B][Hkv][128]) the step's rows are written at
    seq_lens[b]-1 first.  Returns fp16 [B][Hq][128]."""
    _need(q, torch.float32, "q", 3)
    _need(block_table, torch.int32, "block_table", 2)
    _need(seq_lens, torch.int32, "seq_lens", 1)
    n_pages, Hkv, page_size = _pool_shape(k_pool, "k_pool")
    if v_pool.shape != k_pool.shape:
        raise ValueError("k_pool and v_pool differ in shape")
    _pool_shape(v_pool, "v_pool")
    B, Hq, d = q.shape
    if d != D or block_table.shape[0] != B:
        raise ValueError("shape mismatch between q, block_table and pools")
    if (k_new is None) != (v_new is None):
        raise ValueError("give both k_new and v_new, or neither")
    if k_new is not None:
        _need(k_new, torch.float32, "k_new", 3)
        _need(v_new, torch.float32, "v_new", 3)
        if tuple(k_new.shape) != (B, Hkv, D) or tuple(v_new.shape) != (B, Hkv, D):
            raise ValueError("k_new / v_new must be [B][Hkv][128]")
    need = tbq4_decode_workspace_bytes(B, Hq, Hkv, max_len)
    if workspace is None:
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=q.device)
    if out is None:
        out = torch.empty((B, Hq, D), dtype=torch.float16, device=q.device)
    _need(out, torch.float16, "out", 3)
    check(lib.tbq4_attn_decode_paged(
        _ptr(q), _ptr(k_new) if k_new is not None else None,
        _ptr(v_new) if v_new is not None else None, _ptr(k_pool), _ptr(v_pool),
        _ptr(block_table), block_table.shape[1], page_size, n_pages, _ptr(seq_lens),
        int(max_len), B, Hq, Hkv, float(softmax_scale), C.c_uint64(sign_seed), _ptr(workspace),
        workspace.numel() * workspace.element_size(), _ptr(out), _stream(stream)),
        "tbq4_attn_decode_paged")
    return out


BLOCK_BYTES3 = 50      # TBQ3: the 3-bit variant (see include/tbq4.h)


def empty_cache3(batch, n_kv_heads, capacity, device="cuda"):
    """An uninitialised 3-bit cache [B][Hkv][capacity][50] (capacity % 8 == 0)."""
    return torch.empty((batch, n_kv_heads, capacity, BLOCK_BYTES3), dtype=torch.uint8,
                       device=device)


def tbq3_quantize_append(src, start_pos, cache, sign_seed=0, stream=None):
    """As tbq4_quantize_append, into a 3-bit cache [B][Hkv][capacity][50]."""
    _need(src, torch.float32, "src", 4)
    _need(start_pos, torch.int32, "start_pos", 1)
    _need(cache, torch.uint8, "cache", 4)
    B, n_new, Hkv, d = src.shape
    if d != D or tuple(cache.shape[:2]) != (B, Hkv) or cache.shape[3] != BLOCK_BYTES3:
        raise ValueError("shape mismatch between src and cache")
    check(lib.tbq3_quantize_append(_ptr(src), B, n_new, Hkv, _ptr(start_pos),
                                   cache.shape[2], C.c_uint64(sign_seed), _ptr(cache),
                                   _stream(stream)), "tbq3_quantize_append")
    return cache


def tbq3_attn_decode(q, k_cache, v_cache, seq_lens, max_len, softmax_scale, sign_seed=0,
                     workspace=None, out=None, stream=None):
    """As tbq4_attn_decode, over 3-bit caches [B][Hkv][capacity][50]."""
    _need(q, torch.float32, "q", 3)
    _need(k_cache, torch.uint8, "k_cache", 4)
    _need(v_cache, torch.uint8, "v_cache", 4)
    _need(seq_lens, torch.int32, "seq_lens", 1)
    B, Hq, d = q.shape
    _, Hkv, cap, nb = k_cache.shape
    if d != D or nb != BLOCK_BYTES3 or v_cache.shape != k_cache.shape or k_cache.shape[0] != B:
        raise ValueError("shape mismatch between q and caches")
    need = tbq4_decode_workspace_bytes(B, Hq, Hkv, max_len)
    if workspace is None:
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=q.device)
    if out is None:
        out = torch.empty((B, Hq, D), dtype=torch.float16, device=q.device)
    _need(out, torch.float16, "out", 3)
    check(lib.tbq3_attn_decode(
        _ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(seq_lens), int(max_len), B, Hq, Hkv, cap,
        float(softmax_scale), C.c_uint64(sign_seed), _ptr(workspace),
        workspace.numel() * workspace.element_size(), _ptr(out), _stream(stream)),
        "tbq3_attn_decode")
    return out


def tbq4_decode_mq_workspace_bytes(B, q_len, Hq, Hkv, max_len) -> int:
    return int(lib.tbq4_decode_mq_workspace_bytes(B, q_len, Hq, Hkv, max_len))


def tbq4_attn_decode_mq(q, k_cache, v_cache, seq_lens, max_len, softmax_scale, sign_seed=0,
                        workspace=None, out=None, stream=None):
    """q fp32 [B][q_len][Hq][128]: the last q_len tokens of each sequence
    (already in the caches); returns fp16 [B][q_len][Hq][128]."""
    _need(q, torch.float32, "q", 4)
    _need(k_cache, torch.uint8, "k_cache", 4)
    _need(v_cache, torch.uint8, "v_cache", 4)
    _need(seq_lens, torch.int32, "seq_lens", 1)
    B, q_len, Hq, d = q.shape
    _, Hkv, cap, nb = k_cache.shape
    if d != D or nb != BLOCK_BYTES or v_cache.shape != k_cache.shape or k_cache.shape[0] != B:
        raise ValueError("shape mismatch between q and caches")
    need = tbq4_decode_mq_workspace_bytes(B, q_len, Hq, Hkv, max_len)
    if workspace is None:
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=q.device)
    if out is None:
        out = torch.empty((B, q_len, Hq, D), dtype=torch.float16, device=q.device)
    _need(out, torch.float16, "out", 4)
    check(lib.tbq4_attn_decode_mq(
        _ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(seq_lens), int(max_len), B, q_len, Hq, Hkv,
        cap, float(softmax_scale), C.c_uint64(sign_seed), _ptr(workspace),
        workspace.numel() * workspace.element_size(), _ptr(out), _stream(stream)),
        "tbq4_attn_decode_mq")
    return out


def tbq4_prefill_workspace_bytes(n_new, Hq, Hkv, n_cached) -> int:
    return int(lib.tbq4_prefill_workspace_bytes(n_new, Hq, Hkv, n_cached))


def tbq4_attn_prefill_chunk(q, n_cached, k_cache, v_cache, softmax_scale, sign_seed=0,
                            workspace=None, out=None, stream=None):
    """q bf16 [n_new][Hq][128]; caches uint8 [Hkv][capacity][66] of one
    sequence holding the chunk at n_cached ..; returns bf16 [n_new][Hq][128]."""
    _need(q, torch.bfloat16, "q", 3)
    _need(k_cache, torch.uint8, "k_cache", 3)
    _need(v_cache, torch.uint8, "v_cache", 3)
    n_new, Hq, d = q.shape
    Hkv, cap, nb = k_cache.shape
    if d != D or nb != BLOCK_BYTES or v_cache.shape != k_cache.shape:
        raise ValueError("shape mismatch between q and caches")
    need = tbq4_prefill_workspace_bytes(n_new, Hq, Hkv, n_cached)
    if workspace is None:
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=q.device)
    if out is None:
        out = torch.empty((n_new, Hq, D), dtype=torch.bfloat16, device=q.device)
    _need(out, torch.bfloat16, "out", 3)
    check(lib.tbq4_attn_prefill_chunk(
        _ptr(q), n_new, int(n_cached), _ptr(k_cache), _ptr(v_cache), Hq, Hkv, cap,
        float(softmax_scale), C.c_uint64(sign_seed), _ptr(workspace),
        workspace.numel() * workspace.element_size(), _ptr(out), _stream(stream)),
        "tbq4_attn_prefill_chunk")
    return out


def tbq4_set_timing_events(before=None, after=None):
    """Record torch.cuda.Event `before`/`after` around the main attention
    kernel of every following attention call (None, None to stop)."""
    lib.tbq4_set_timing_events(C.c_void_p(before.cuda_event if before is not None else 0),
                               C.c_void_p(after.cuda_event if after is not None else 0))


def tbq4_get_device_status(stream=None) -> int:
    """Synchronises the stream and returns (and clears) the device error code."""
    return int(lib.tbq4_get_device_status(_stream(stream)))


def tbq4_selftest_bounded_wait(polls=256, stream=None) -> None:
    """Launches the bounded-wait self-test: one warp waits on a barrier that
    nothing completes, gives up after `polls` polls and records
    TBQ4_ERR_DEVICE_TIMEOUT (read it with tbq4_get_device_status)."""
    check(lib.tbq4_selftest_bounded_wait(C.c_uint32(int(polls)), _stream(stream)),
          "tbq4_selftest_bounded_wait")

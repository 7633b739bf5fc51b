"""Shared test plumbing: building caches on both sides, comparing results.

The CUDA side is driven only through the package binding (the C ABI); the
oracle side only through ``oracle``.  Both take their inputs from
``long_context_attention_tbq4_b200.workloads``.
"""
import math

import numpy as np

D = 128
DECODE_MAX_ABS = 2e-3
DECODE_REL_L2 = 1e-3
PREFILL_REL_L2 = 1e-2


def rel_l2(got, want):
    got = np.asarray(got, np.float64)
    want = np.asarray(want, np.float64)
    return float(np.linalg.norm(got - want) / max(np.linalg.norm(want), 1e-300))


def max_abs(got, want):
    return float(np.abs(np.asarray(got, np.float64) - np.asarray(want, np.float64)).max())


def oracle_caches(seqs, Hkv, capacity, seed):
    """Oracle caches [B][Hkv][capacity][66] from per-sequence fp32 rows."""
    import oracle
    B = len(seqs)
    cache = np.zeros((B, Hkv, capacity, 66), np.uint8)
    for b, x in enumerate(seqs):
        if len(x) == 0:
            continue
        sub = cache[b:b + 1]
        oracle.quantize_append(x[None], np.zeros(1, np.int32), capacity, seed, sub)
        cache[b:b + 1] = sub
    return cache


def gpu_caches(seqs, Hkv, capacity, seed, fill=None):
    """GPU caches built by tbq4_quantize_append, one call per sequence."""
    import torch
    import long_context_attention_tbq4_b200 as T
    B = len(seqs)
    cache = T.empty_cache(B, Hkv, capacity)
    if fill is not None:
        cache.fill_(fill)
    else:
        cache.zero_()
    for b, x in enumerate(seqs):
        if len(x) == 0:
            continue
        src = torch.from_numpy(np.ascontiguousarray(x)[None]).cuda()
        view = cache[b:b + 1]
        T.tbq4_quantize_append(src, torch.zeros(1, dtype=torch.int32, device="cuda"), view,
                               sign_seed=seed)
    return cache


def half_ulp_fp16(x):
    """Half a unit in the last place of fp16 at |x|: the rounding error the
    fp16 output format itself allows (2^-25 in the subnormal range)."""
    a = np.abs(np.asarray(x, np.float64))
    e = np.floor(np.log2(np.maximum(a, 2.0 ** -14)))
    return 2.0 ** (e - 11)


def check_decode(got, want):
    """Per element |gpu - oracle| <= max(2e-3, half an fp16 ulp of the oracle
    value), and rel-L2 <= 1e-3 over the whole tensor.

    The decode output is fp16.  Below |o| = 8 half an fp16 ulp is at most
    2^-10 < 2e-3, so there the bound is the plain 2e-3; only where fp16
    itself cannot come within 2e-3 of the true value (|o| >= 8, half an ulp
    >= 3.9e-3) is the bound half an ulp, what correct rounding of the exact
    value allows.  Returns (raw max-abs, rel-L2)."""
    got = np.asarray(got, np.float64)
    want = np.asarray(want, np.float64)
    err = np.abs(got - want)
    bound = np.maximum(DECODE_MAX_ABS, half_ulp_fp16(want))
    worst = int(np.argmax(err - bound))
    ma, rl = float(err.max()), rel_l2(got, want)
    print(f"decode max-abs {ma:.3e} (worst vs bound {float(err.flat[worst]):.3e} <= "
          f"{float(bound.flat[worst]):.3e} at |o| {abs(float(want.flat[worst])):.3f}), "
          f"rel-L2 {rl:.3e}")
    assert err.flat[worst] <= bound.flat[worst] and rl <= DECODE_REL_L2, (
        ma, float(err.flat[worst]), float(want.flat[worst]), rl)
    return ma, rl


def capacity_for(n, multiple=8):
    return max(multiple, int(math.ceil(n / multiple)) * multiple)

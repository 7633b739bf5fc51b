"""GPU quantise-append against the oracle: packed bytes must be bit-exact."""
import numpy as np
import pytest

import oracle
from long_context_attention_tbq4_b200 import workloads as W

from helpers import gpu_caches, oracle_caches

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def T():
    import torch
    import long_context_attention_tbq4_b200 as pkg
    assert torch.cuda.is_available()
    return pkg


def _gpu_append(T, src, start, capacity, seed, fill=0xAB):
    import torch
    B, n_new, Hkv, _ = src.shape
    cache = T.empty_cache(B, Hkv, capacity)
    cache.fill_(fill)
    T.tbq4_quantize_append(torch.from_numpy(src).cuda(),
                           torch.from_numpy(np.asarray(start, np.int32)).cuda(), cache,
                           sign_seed=seed)
    assert T.tbq4_get_device_status() == 0
    return cache.cpu().numpy()


def _oracle_append(src, start, capacity, seed, fill=0xAB):
    B, n_new, Hkv, _ = src.shape
    cache = np.full((B, Hkv, capacity, 66), fill, np.uint8)
    oracle.quantize_append(src, np.asarray(start, np.int32), capacity, seed, cache)
    return cache


@pytest.mark.parametrize("dist,gain", [("normal", 1.0), ("t4", 1.0), ("normal", 1e-3),
                                       ("t4", 300.0), ("normal", 1e-6), ("normal", 5e3)])
def test_bytes_bit_exact_small(T, dist, gain):
    rng = np.random.default_rng(hash((dist, gain)) % 2**32)
    B, n_new, Hkv, cap = 3, 37, 3, 64
    if dist == "normal":
        src = rng.standard_normal((B, n_new, Hkv, 128)).astype(np.float32)
    else:
        src = rng.standard_t(4, (B, n_new, Hkv, 128)).astype(np.float32)
    src *= np.float32(gain)
    src[0, 3] = 0.0                                   # zero rows -> scale 0, index 8
    src[1, 5, 0, 17] = 1e9                            # saturating scale
    start = [3, 16, 27]
    for seed in [0, 99]:
        got = _gpu_append(T, src, start, cap, seed)
        want = _oracle_append(src, start, cap, seed)
        assert np.array_equal(got, want)


def test_ragged_tail_and_single_rows(T):
    rng = np.random.default_rng(7)
    for n_new in [1, 2, 7, 8, 9, 31, 33]:
        src = rng.standard_normal((2, n_new, 1, 128)).astype(np.float32)
        got = _gpu_append(T, src, [0, 40 - n_new], 40, 0)
        want = _oracle_append(src, [0, 40 - n_new], 40, 0)
        assert np.array_equal(got, want)


def test_out_of_range_rows_are_skipped_and_flagged(T):
    import torch
    rng = np.random.default_rng(8)
    src = rng.standard_normal((1, 6, 2, 128)).astype(np.float32)
    cache = T.empty_cache(1, 2, 8)
    cache.fill_(0xAB)
    T.tbq4_quantize_append(torch.from_numpy(src).cuda(),
                           torch.tensor([5], dtype=torch.int32, device="cuda"), cache)
    assert T.tbq4_get_device_status() == 4           # TBQ4_ERR_CAPACITY
    assert T.tbq4_get_device_status() == 0           # cleared
    want = _oracle_append(src, [5], 8, 0)
    assert np.array_equal(cache.cpu().numpy(), want)


@pytest.mark.parametrize("case", ["decode_32k", "decode_262k", "ragged", "prefill"])
def test_bytes_bit_exact_workloads(T, case):
    if case == "decode_32k":
        c = W.decode_32k()
        seqs_k, seqs_v, Hkv = c.k, c.v, c.Hkv
    elif case == "decode_262k":
        c = W.decode_262k()
        seqs_k, seqs_v, Hkv = c.k, c.v, c.Hkv
    elif case == "ragged":
        c = W.ragged_decode()
        seqs_k, seqs_v, Hkv = c.k, c.v, c.Hkv
    else:
        c = W.prefill_131k()
        seqs_k, seqs_v, Hkv = [c.k], [c.v], c.Hkv
    cap = W.round_capacity(max(len(x) for x in seqs_k))
    for seqs in (seqs_k, seqs_v):
        got = gpu_caches(seqs, Hkv, cap, W.SIGN_SEED).cpu().numpy()
        want = oracle_caches(seqs, Hkv, cap, W.SIGN_SEED)
        for b, x in enumerate(seqs):
            n = len(x)
            assert np.array_equal(got[b, :, :n], want[b, :, :n]), (case, b)


def test_bulk_path_ragged_groups_and_positions(T):
    # 3 x 2,731 x 3 = 24,579 rows: the bulk encoder (16,384 rows or more), a
    # group count that the CTA count does not divide, a 3-row tail group, and
    # a different start position per sequence
    rng = np.random.default_rng(21)
    B, n_new, Hkv, cap = 3, 2731, 3, 4096
    src = (rng.standard_t(4, (B, n_new, Hkv, 128)) * 3).astype(np.float32)
    src[1, 100] = 0.0                                 # zero rows inside the bulk path
    start = [0, 1000, 1365]
    got = _gpu_append(T, src, start, cap, 5)
    want = _oracle_append(src, start, cap, 5)
    assert np.array_equal(got, want)


def test_bulk_path_out_of_range_rows_are_skipped_and_flagged(T):
    import torch
    rng = np.random.default_rng(22)
    src = rng.standard_normal((1, 20000, 1, 128)).astype(np.float32)
    cache = T.empty_cache(1, 1, 16384)
    cache.fill_(0xAB)
    T.tbq4_quantize_append(torch.from_numpy(src).cuda(),
                           torch.tensor([100], dtype=torch.int32, device="cuda"), cache)
    assert T.tbq4_get_device_status() == 4           # rows past the capacity
    assert T.tbq4_get_device_status() == 0
    want = _oracle_append(src, [100], 16384, 0)
    assert np.array_equal(cache.cpu().numpy(), want)


def test_bulk_path_extreme_scales(T):
    """20,480 rows through the bulk encoder, every 8-row group mixing rows
    whose fp16 scale is zero (max |x_rot| below 2^-25), subnormal, near the
    smallest normal, ordinary, or saturated at 65,504 (the rows that take the
    clamp), for both the 4-bit and the 3-bit encoder."""
    import torch
    rng = np.random.default_rng(23)
    B, n_new, Hkv, cap = 2, 2560, 4, 2560
    src = rng.standard_normal((B, n_new, Hkv, 128)).astype(np.float32)
    gains = np.array([1.0, 1e-6, 1e-9, 3e-5, 1.0, 7e4, 1e-7, 250.0], np.float32)
    src *= gains[np.arange(n_new) % 8][None, :, None, None]
    src[:, 4::8, :, 5] = 1e9                          # one huge value: a saturated scale
    zero = np.zeros(B, np.int32)
    got = _gpu_append(T, src, zero, cap, 3)
    want = _oracle_append(src, zero, cap, 3)
    assert np.array_equal(got, want)
    got3 = T.empty_cache3(B, Hkv, cap)
    got3.fill_(0xAB)
    T.tbq3_quantize_append(torch.from_numpy(src).cuda(), torch.from_numpy(zero).cuda(), got3, 3)
    assert T.tbq4_get_device_status() == 0
    want3 = np.full((B, Hkv, cap, 50), 0xAB, np.uint8)
    oracle.quantize_append3(src, zero, cap, 3, want3)
    assert np.array_equal(got3.cpu().numpy(), want3)

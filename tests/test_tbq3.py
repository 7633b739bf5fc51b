"""TBQ3 (the 3-bit variant) on the GPU: quantise-append bytes bit-exact against
the oracle's encoder, and decode attention against the oracle's fp64
attention over the same 3-bit cache, within the decode tolerance."""
import numpy as np
import pytest

import oracle
from long_context_attention_tbq4_b200 import workloads as W

from helpers import check_decode

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def T():
    import torch
    import long_context_attention_tbq4_b200 as pkg
    assert torch.cuda.is_available()
    return pkg


def oracle_caches3(seqs, Hkv, capacity, seed):
    B = len(seqs)
    cache = np.zeros((B, Hkv, capacity, 50), np.uint8)
    for b, x in enumerate(seqs):
        if len(x) == 0:
            continue
        sub = cache[b:b + 1]
        oracle.quantize_append3(x[None], np.zeros(1, np.int32), capacity, seed, sub)
        cache[b:b + 1] = sub
    return cache


def gpu_caches3(T, seqs, Hkv, capacity, seed, fill=0):
    import torch
    cache = T.empty_cache3(len(seqs), Hkv, capacity)
    cache.fill_(fill)
    zero = torch.zeros(1, dtype=torch.int32, device="cuda")
    for b, x in enumerate(seqs):
        if len(x) == 0:
            continue
        src = torch.from_numpy(np.ascontiguousarray(x)[None]).cuda()
        T.tbq3_quantize_append(src, zero, cache[b:b + 1], seed)
    return cache


@pytest.mark.parametrize("B,n_new,Hkv,cap", [(1, 1, 1, 8), (2, 37, 3, 48), (3, 500, 4, 512)])
def test_quantize3_bytes_match_oracle(T, B, n_new, Hkv, cap):
    import torch
    rng = np.random.default_rng(300 + n_new)
    src = (rng.standard_t(4, (B, n_new, Hkv, 128)) * rng.choice([1e-3, 1.0, 50.0])).astype(np.float32)
    src[0, 0, 0] = 0.0                               # a zero block (scale 0, every index 4)
    start = rng.integers(0, cap - n_new + 1, B).astype(np.int32)
    want = np.full((B, Hkv, cap, 50), 0x5A, np.uint8)
    assert oracle.quantize_append3(src, start, cap, 11, want) == 0
    got = T.empty_cache3(B, Hkv, cap)
    got.fill_(0x5A)
    T.tbq3_quantize_append(torch.from_numpy(src).cuda(), torch.from_numpy(start).cuda(), got, 11)
    assert T.tbq4_get_device_status() == 0
    assert np.array_equal(got.cpu().numpy(), want)


def test_quantize3_262k_build_matches_oracle(T):
    case = W.decode_262k()
    N = int(case.seq_lens[0])
    got = gpu_caches3(T, case.k, case.Hkv, N, case.sign_seed).cpu().numpy()
    want = oracle_caches3(case.k, case.Hkv, N, case.sign_seed)
    assert np.array_equal(got, want)


def _check(T, case, cap):
    import torch
    kc = gpu_caches3(T, case.k, case.Hkv, cap, case.sign_seed, fill=0xA5)
    vc = gpu_caches3(T, case.v, case.Hkv, cap, case.sign_seed, fill=0x5A)
    ko = oracle_caches3(case.k, case.Hkv, cap, case.sign_seed)
    vo = oracle_caches3(case.v, case.Hkv, cap, case.sign_seed)
    lens = np.asarray(case.seq_lens, np.int32)
    kg, vg = kc.cpu().numpy(), vc.cpu().numpy()
    for b, n in enumerate(lens):
        assert np.array_equal(kg[b, :, :n], ko[b, :, :n]) and np.array_equal(vg[b, :, :n], vo[b, :, :n])
    q = torch.from_numpy(case.q).cuda()
    got = T.tbq3_attn_decode(q, kc, vc, torch.from_numpy(lens).cuda(), int(lens.max()),
                             case.softmax_scale, case.sign_seed)
    assert T.tbq4_get_device_status() == 0
    want = oracle.attn_decode3(case.q, ko, vo, lens, case.softmax_scale, case.sign_seed)
    check_decode(got.float().cpu().numpy(), want)


def test_decode3_tiny(T):
    _check(T, W.tiny_decode(), 1024)


def test_decode3_ragged_with_zero_length(T):
    lens = [0, 1, 31, 33, 700, 5000, 257]
    _check(T, W.decode_case("tbq3_ragged", 61, len(lens), 16, 2, lens, dist="t4"), 5000)


def test_decode3_groups(T):
    for G in (1, 3, 8):
        _check(T, W.decode_case("tbq3_g%d" % G, 62 + G, 2, 2 * G, 2, [900, 1300]), 1304)


def test_decode3_32k(T):
    _check(T, W.decode_32k(), 32768)


def test_decode3_262k_outliers(T):
    _check(T, W.decode_262k(), 262144)

"""tbq4_attn_decode_append: one decode step with the new token's K/V rows
encoded inside the attention kernel.

The fused call must leave exactly the cache bytes that tbq4_quantize_append
writes (checked against the oracle's encoder) and give exactly the output of
tbq4_attn_decode over the appended caches (bitwise: the same kernel reads the
same bytes); that output is also checked against the fp64 oracle.
"""
import numpy as np
import pytest

import oracle
from long_context_attention_tbq4_b200 import workloads as W

from helpers import capacity_for, check_decode, gpu_caches, oracle_caches

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def T():
    import torch
    import long_context_attention_tbq4_b200 as pkg
    assert torch.cuda.is_available()
    return pkg


def _step(T, case, cap, split_tokens=0):
    """Caches hold every token but the last (whose slot is garbage); returns
    (fused out, fused caches, separate out, separate caches)."""
    import torch
    B, Hkv = case.B, case.Hkv
    lens = np.asarray(case.seq_lens, np.int32)
    prev = [x[:max(len(x) - 1, 0)] for x in case.k], [x[:max(len(x) - 1, 0)] for x in case.v]
    kc = gpu_caches(prev[0], Hkv, cap, case.sign_seed, fill=0xA5)
    vc = gpu_caches(prev[1], Hkv, cap, case.sign_seed, fill=0x5A)
    k_new = np.zeros((B, Hkv, 128), np.float32)
    v_new = np.zeros((B, Hkv, 128), np.float32)
    for b in range(B):
        if lens[b] > 0:
            k_new[b] = case.k[b][-1]
            v_new[b] = case.v[b][-1]
    q = torch.from_numpy(case.q).cuda()
    kn = torch.from_numpy(k_new).cuda()
    vn = torch.from_numpy(v_new).cuda()
    dl = torch.from_numpy(lens).cuda()
    max_len = int(lens.max())

    k2, v2 = kc.clone(), vc.clone()
    fused = T.tbq4_attn_decode_append(q, kn, vn, kc, vc, dl, max_len, case.softmax_scale,
                                      case.sign_seed)
    assert T.tbq4_get_device_status() == 0

    # the separate path: append at len-1 (sequences of length 0 append nothing)
    for b in range(B):
        if lens[b] == 0:
            continue
        pos = torch.tensor([lens[b] - 1], dtype=torch.int32, device="cuda")
        T.tbq4_quantize_append(kn[b:b + 1, None], pos, k2[b:b + 1], case.sign_seed)
        T.tbq4_quantize_append(vn[b:b + 1, None], pos, v2[b:b + 1], case.sign_seed)
    sep = T.tbq4_attn_decode(q, k2, v2, dl, max_len, case.softmax_scale, case.sign_seed,
                             split_tokens=split_tokens)
    assert T.tbq4_get_device_status() == 0
    return fused, kc, vc, sep, k2, v2


def _check(T, case, cap, split_tokens=0):
    import torch
    fused, kc, vc, sep, k2, v2 = _step(T, case, cap, split_tokens)
    assert torch.equal(kc, k2) and torch.equal(vc, v2)
    assert torch.equal(fused, sep)
    ko = oracle_caches(case.k, case.Hkv, cap, case.sign_seed)
    vo = oracle_caches(case.v, case.Hkv, cap, case.sign_seed)
    kg, vg = kc.cpu().numpy(), vc.cpu().numpy()
    for b, x in enumerate(case.k):
        n = len(x)
        assert np.array_equal(kg[b, :, :n], ko[b, :, :n])
        assert np.array_equal(vg[b, :, :n], vo[b, :, :n])
    want = oracle.attn_decode(case.q, ko, vo, np.asarray(case.seq_lens, np.int32),
                              case.softmax_scale, case.sign_seed)
    check_decode(fused.float().cpu().numpy(), want)


def test_append_tiny(T):
    case = W.tiny_decode()
    _check(T, case, capacity_for(1024))


def test_append_ragged_positions(T):
    # new token at the first, middle and last row of a chunk, in the first
    # chunk, and in the tail of a split
    lens = [1, 2, 31, 32, 33, 64, 255, 256, 257, 4097, 9000]
    case = W.decode_case("append_ragged", 31, len(lens), 16, 2, lens)
    _check(T, case, 9008)


def test_append_with_zero_length(T):
    case = W.decode_case("append_zero", 32, 3, 8, 2, [0, 100, 0])
    _check(T, case, 104)


def test_append_32k(T):
    _check(T, W.decode_32k(), 32768)


def test_append_262k(T):
    _check(T, W.decode_262k(), 262144)


def test_append_skips_flagged_length(T):
    """A length above max_len is flagged and appends nothing."""
    import torch
    B, Hq, Hkv, cap = 1, 4, 1, 64
    kc = torch.full((B, Hkv, cap, 66), 0x33, dtype=torch.uint8, device="cuda")
    vc = kc.clone()
    before = kc.clone()
    q = torch.randn((B, Hq, 128), device="cuda")
    kn = torch.randn((B, Hkv, 128), device="cuda")
    lens = torch.tensor([40], dtype=torch.int32, device="cuda")
    T.tbq4_attn_decode_append(q, kn, kn, kc, vc, lens, 16, 0.1, 0)
    torch.cuda.synchronize()
    assert T.tbq4_get_device_status() == 4                       # TBQ4_ERR_CAPACITY
    assert torch.equal(kc, before) and torch.equal(vc, before)

"""Paged caches: tbq4_quantize_append_paged and tbq4_attn_decode_paged.

K and V live in page pools shared by the batch and are found through a
shuffled block table.  Gathered back through the table, a pool must hold
exactly the oracle's encoding of every token; paged decode must equal
contiguous decode over the same bytes bit for bit (the same kernel
arithmetic, only the addresses differ) and the fp64 oracle within the decode
tolerance; the fused append must write the pools as the separate append does.
"""
import numpy as np
import pytest

import oracle
from long_context_attention_tbq4_b200 import workloads as W

from helpers import check_decode, oracle_caches

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def T():
    import torch
    import long_context_attention_tbq4_b200 as pkg
    assert torch.cuda.is_available()
    return pkg


def _pools(T, seqs, Hkv, table, n_pages, page_size, seed, fill):
    """A pool filled by tbq4_quantize_append_paged, one call per sequence."""
    import torch
    pool = T.empty_pool(n_pages, Hkv, page_size)
    pool.fill_(fill)
    tab = torch.from_numpy(table).cuda()
    zero = torch.zeros(1, dtype=torch.int32, device="cuda")
    for b, x in enumerate(seqs):
        if len(x) == 0:
            continue
        src = torch.from_numpy(np.ascontiguousarray(x)[None]).cuda()
        T.tbq4_quantize_append_paged(src, zero, tab[b:b + 1], pool, seed)
    return pool, tab


def _gather(pool, table, lens, capacity):
    """Contiguous [B][Hkv][capacity][66] copy of a pool (numpy, host side)."""
    pool = np.asarray(pool)
    B, Hkv, P = len(lens), pool.shape[1], pool.shape[2]
    out = np.zeros((B, Hkv, capacity, 66), np.uint8)
    for b, n in enumerate(lens):
        for t0 in range(0, int(n), P):
            k = min(P, int(n) - t0)
            out[b, :, t0:t0 + k] = pool[table[b, t0 // P], :, :k]
    return out


def _check_decode(T, case, page_size, table_seed, spare=3):
    import torch
    lens = np.asarray(case.seq_lens, np.int32)
    table, n_pages = W.page_table(table_seed, lens, page_size, spare)
    cap = table.shape[1] * page_size
    kp, tab = _pools(T, case.k, case.Hkv, table, n_pages, page_size, case.sign_seed, 0xA5)
    vp, _ = _pools(T, case.v, case.Hkv, table, n_pages, page_size, case.sign_seed, 0x5A)
    assert T.tbq4_get_device_status() == 0
    ko = oracle_caches(case.k, case.Hkv, cap, case.sign_seed)
    vo = oracle_caches(case.v, case.Hkv, cap, case.sign_seed)
    kg = _gather(kp.cpu().numpy(), table, lens, cap)
    vg = _gather(vp.cpu().numpy(), table, lens, cap)
    for b, n in enumerate(lens):
        assert np.array_equal(kg[b, :, :n], ko[b, :, :n])
        assert np.array_equal(vg[b, :, :n], vo[b, :, :n])

    q = torch.from_numpy(case.q).cuda()
    dl = torch.from_numpy(lens).cuda()
    max_len = int(lens.max())
    got = T.tbq4_attn_decode_paged(q, kp, vp, tab, dl, max_len, case.softmax_scale,
                                   case.sign_seed)
    assert T.tbq4_get_device_status() == 0
    # contiguous decode over the gathered bytes: the same result, bit for bit
    ref = T.tbq4_attn_decode(q, torch.from_numpy(kg).cuda(), torch.from_numpy(vg).cuda(), dl,
                             max_len, case.softmax_scale, case.sign_seed)
    assert torch.equal(got, ref)
    want = oracle.attn_decode(case.q, ko, vo, lens, case.softmax_scale, case.sign_seed)
    check_decode(got.float().cpu().numpy(), want)


def test_paged_ragged_page_32(T):
    lens = [1, 31, 32, 33, 300, 1000, 0, 4100]
    _check_decode(T, W.decode_case("paged_32", 41, len(lens), 16, 2, lens), 32, 141)


def test_paged_ragged_page_256(T):
    lens = [5000, 1, 257, 0, 12000, 700]
    _check_decode(T, W.decode_case("paged_256", 42, len(lens), 24, 4, lens, dist="t4"), 256,
                  142)


def test_paged_one_long_sequence(T):
    # 40,000 keys in pages of 4,096: several splits per page, pages out of order
    _check_decode(T, W.decode_case("paged_40k", 43, 1, 24, 4, [40000]), 4096, 143)


def test_paged_262k_matches_contiguous(T):
    """The 262K workload in 256-token pages: identical to the contiguous
    kernel over the same bytes (which the decode tests check against the
    oracle at this size)."""
    import torch
    case = W.decode_262k()
    N = int(case.seq_lens[0])
    P = 256
    table, n_pages = W.page_table(7, [N], P)
    tab = torch.from_numpy(table).cuda()
    zero = torch.zeros(1, dtype=torch.int32, device="cuda")
    kc, vc = T.empty_cache(1, case.Hkv, N), T.empty_cache(1, case.Hkv, N)
    kp, vp = T.empty_pool(n_pages, case.Hkv, P), T.empty_pool(n_pages, case.Hkv, P)
    for cache, pool, x in ((kc, kp, case.k[0]), (vc, vp, case.v[0])):
        src = torch.from_numpy(np.ascontiguousarray(x)[None]).cuda()
        T.tbq4_quantize_append(src, zero, cache, case.sign_seed)
        T.tbq4_quantize_append_paged(src, zero, tab, pool, case.sign_seed)
        del src
    assert T.tbq4_get_device_status() == 0
    # the pool's pages hold the cache's rows
    perm = tab[0].long()
    for cache, pool in ((kc, kp), (vc, vp)):
        rows = cache[0].view(case.Hkv, N // P, P, 66).permute(1, 0, 2, 3)
        assert torch.equal(pool[perm], rows)
    q = torch.from_numpy(case.q).cuda()
    lens = torch.tensor([N], dtype=torch.int32, device="cuda")
    got = T.tbq4_attn_decode_paged(q, kp, vp, tab, lens, N, case.softmax_scale, case.sign_seed)
    ref = T.tbq4_attn_decode(q, kc, vc, lens, N, case.softmax_scale, case.sign_seed)
    assert T.tbq4_get_device_status() == 0
    assert torch.equal(got, ref)


def test_paged_decode_append(T):
    """The fused step writes the new rows into the pools at len-1 and gives
    the output of a separate paged append followed by paged decode."""
    import torch
    lens = [1, 32, 33, 257, 3000, 0]
    case = W.decode_case("paged_append", 44, len(lens), 16, 2, lens)
    P = 64
    la = np.asarray(lens, np.int32)
    table, n_pages = W.page_table(144, la, P)
    prev_k = [x[:max(len(x) - 1, 0)] for x in case.k]
    prev_v = [x[:max(len(x) - 1, 0)] for x in case.v]
    kp, tab = _pools(T, prev_k, case.Hkv, table, n_pages, P, case.sign_seed, 0xA5)
    vp, _ = _pools(T, prev_v, case.Hkv, table, n_pages, P, case.sign_seed, 0x5A)
    k_new = np.zeros((case.B, case.Hkv, 128), np.float32)
    v_new = np.zeros_like(k_new)
    for b in range(case.B):
        if la[b] > 0:
            k_new[b], v_new[b] = case.k[b][-1], case.v[b][-1]
    q = torch.from_numpy(case.q).cuda()
    kn, vn = torch.from_numpy(k_new).cuda(), torch.from_numpy(v_new).cuda()
    dl = torch.from_numpy(la).cuda()
    max_len = int(la.max())
    k2, v2 = kp.clone(), vp.clone()
    fused = T.tbq4_attn_decode_paged(q, kp, vp, tab, dl, max_len, case.softmax_scale,
                                     case.sign_seed, k_new=kn, v_new=vn)
    assert T.tbq4_get_device_status() == 0
    for b in range(case.B):
        if la[b] == 0:
            continue
        pos = torch.tensor([la[b] - 1], dtype=torch.int32, device="cuda")
        T.tbq4_quantize_append_paged(kn[b:b + 1, None], pos, tab[b:b + 1], k2, case.sign_seed)
        T.tbq4_quantize_append_paged(vn[b:b + 1, None], pos, tab[b:b + 1], v2, case.sign_seed)
    sep = T.tbq4_attn_decode_paged(q, k2, v2, tab, dl, max_len, case.softmax_scale,
                                   case.sign_seed)
    assert T.tbq4_get_device_status() == 0
    assert torch.equal(kp, k2) and torch.equal(vp, v2)
    assert torch.equal(fused, sep)
    cap = table.shape[1] * P
    ko = oracle_caches(case.k, case.Hkv, cap, case.sign_seed)
    vo = oracle_caches(case.v, case.Hkv, cap, case.sign_seed)
    kg = _gather(kp.cpu().numpy(), table, la, cap)
    for b, n in enumerate(la):
        assert np.array_equal(kg[b, :, :n], ko[b, :, :n])
    want = oracle.attn_decode(case.q, ko, vo, la, case.softmax_scale, case.sign_seed)
    check_decode(fused.float().cpu().numpy(), want)


def test_paged_table_entries_past_the_length_are_ignored(T):
    """Entries past a sequence's length may hold anything (they are only
    speculative copy sources, mapped into the pool); a bad entry inside the
    length is flagged."""
    import torch
    lens = [100, 40]
    case = W.decode_case("paged_tail", 45, 2, 8, 2, lens)
    P = 32
    la = np.asarray(lens, np.int32)
    table, n_pages = W.page_table(145, la, P, max_pages=6)
    table[0, 4:] = [123456789, -7]           # past the length: garbage
    table[1, 2:] = [-1, 2 ** 31 - 1, 99, 5]
    kp, tab = _pools(T, case.k, case.Hkv, table, n_pages, P, case.sign_seed, 0)
    vp, _ = _pools(T, case.v, case.Hkv, table, n_pages, P, case.sign_seed, 0)
    assert T.tbq4_get_device_status() == 0
    q = torch.from_numpy(case.q).cuda()
    dl = torch.from_numpy(la).cuda()
    got = T.tbq4_attn_decode_paged(q, kp, vp, tab, dl, 6 * P, case.softmax_scale,
                                   case.sign_seed)
    assert T.tbq4_get_device_status() == 0
    ko = oracle_caches(case.k, case.Hkv, 6 * P, case.sign_seed)
    vo = oracle_caches(case.v, case.Hkv, 6 * P, case.sign_seed)
    want = oracle.attn_decode(case.q, ko, vo, la, case.softmax_scale, case.sign_seed)
    check_decode(got.float().cpu().numpy(), want)

    bad = tab.clone()
    bad[1, 0] = n_pages                       # inside sequence 1's length
    T.tbq4_attn_decode_paged(q, kp, vp, bad, dl, 6 * P, case.softmax_scale, case.sign_seed)
    torch.cuda.synchronize()
    assert T.tbq4_get_device_status() == 4    # TBQ4_ERR_CAPACITY
    # the append refuses the same entry and writes nothing
    before = kp.clone()
    src = torch.from_numpy(np.ascontiguousarray(case.k[1][:1])[None]).cuda()
    T.tbq4_quantize_append_paged(src, torch.zeros(1, dtype=torch.int32, device="cuda"),
                                 bad[1:2], kp, case.sign_seed)
    torch.cuda.synchronize()
    assert T.tbq4_get_device_status() == 4
    assert torch.equal(kp, before)

"""Caches larger than 4 GB: every byte offset into a cache or a page pool is
64-bit, so rows whose offset lies past 2^32 are encoded, found and attended
exactly like rows near the start.

Two caches of [2][8][5,242,880][66] (5.5 GB each): the KV heads (b=1, h>=5)
start past 2^32.  A page pool of 70,000 pages x 4 heads x 256 tokens (4.7 GB)
whose block table points at its top pages; one sequence is long enough that
its append takes the bulk encoder, the other takes the warp encoder.  The
rows are compared with the oracle's encoding in compact caches (a row's
bytes do not depend on where it is stored), and the attention with the
oracle over those compact caches.
"""
import numpy as np
import pytest

import oracle
from long_context_attention_tbq4_b200 import workloads as W

from helpers import check_decode, oracle_caches

pytestmark = pytest.mark.gpu

GB4 = 1 << 32


@pytest.fixture(scope="module")
def T():
    import torch
    import long_context_attention_tbq4_b200 as pkg
    assert torch.cuda.is_available()
    return pkg


def test_contiguous_caches_past_4gb(T):
    import torch
    B, Hq, Hkv, cap = 2, 16, 8, 5_242_880
    lens = [3000, 2500]
    assert (B * Hkv - 1) * cap * 66 > GB4                   # the last heads start past 2^32
    case = W.decode_case("past_4gb", 93, B, Hq, Hkv, lens)
    kc, vc = T.empty_cache(B, Hkv, cap), T.empty_cache(B, Hkv, cap)
    zero = torch.zeros(1, dtype=torch.int32, device="cuda")
    for b in range(B):
        for cache, x in ((kc, case.k[b]), (vc, case.v[b])):
            T.tbq4_quantize_append(torch.from_numpy(np.ascontiguousarray(x)[None]).cuda(), zero,
                                   cache[b:b + 1], case.sign_seed)
    # rows at the very end of both sequences' capacity, through the whole cache (the kernel's
    # own offsets reach 5.5 GB), 32,800 rows: the bulk encoder
    tail = np.random.default_rng(94).standard_normal((B, 2050, Hkv, 128)).astype(np.float32)
    T.tbq4_quantize_append(torch.from_numpy(tail).cuda(),
                           torch.tensor([cap - 2050] * B, dtype=torch.int32, device="cuda"),
                           kc, case.sign_seed)
    assert T.tbq4_get_device_status() == 0
    ko = oracle_caches(case.k, Hkv, max(lens), case.sign_seed)
    vo = oracle_caches(case.v, Hkv, max(lens), case.sign_seed)
    for b, n in enumerate(lens):
        assert np.array_equal(kc[b, :, :n].cpu().numpy(), ko[b, :, :n])
        assert np.array_equal(vc[b, :, :n].cpu().numpy(), vo[b, :, :n])
    want_tail = np.zeros((B, Hkv, 2056, 66), np.uint8)
    oracle.quantize_append(tail, np.zeros(B, np.int32), 2056, case.sign_seed, want_tail)
    for b in range(B):
        assert np.array_equal(kc[b, :, cap - 2050:].cpu().numpy(), want_tail[b, :, :2050])
        # the tail rows must not have disturbed the attended rows
        assert np.array_equal(kc[b, :, :lens[b]].cpu().numpy(), ko[b, :, :lens[b]])
    q = torch.from_numpy(case.q).cuda()
    lt = torch.tensor(lens, dtype=torch.int32, device="cuda")
    got = T.tbq4_attn_decode(q, kc, vc, lt, max(lens), case.softmax_scale, case.sign_seed)
    assert T.tbq4_get_device_status() == 0
    want = oracle.attn_decode(case.q, ko, vo, np.asarray(lens, np.int32), case.softmax_scale,
                              case.sign_seed)
    check_decode(got.float().cpu().numpy(), want)
    del kc, vc
    torch.cuda.empty_cache()


def test_page_pool_past_4gb(T):
    import torch
    B, Hq, Hkv, P, n_pages = 2, 8, 4, 256, 70_000
    lens = [4200, 700]              # 16,800 rows for sequence 0: the bulk encoder's paged path
    assert (n_pages - 1) * Hkv * P * 66 > GB4
    case = W.decode_case("pool_past_4gb", 95, B, Hq, Hkv, lens)
    max_pages = 17
    # sequence b uses the top pages, in descending order
    table = np.full((B, max_pages), -1, np.int32)
    top = n_pages - 1
    for b in range(B):
        for j in range(max_pages):
            table[b, j] = top
            top -= 1
    tab = torch.from_numpy(table).cuda()
    kp, vp = T.empty_pool(n_pages, Hkv, P), T.empty_pool(n_pages, Hkv, P)
    zero = torch.zeros(1, dtype=torch.int32, device="cuda")
    for b in range(B):
        for pool, x in ((kp, case.k[b]), (vp, case.v[b])):
            T.tbq4_quantize_append_paged(torch.from_numpy(np.ascontiguousarray(x)[None]).cuda(),
                                         zero, tab[b:b + 1], pool, case.sign_seed)
    assert T.tbq4_get_device_status() == 0
    ko = oracle_caches(case.k, Hkv, max_pages * P, case.sign_seed)
    vo = oracle_caches(case.v, Hkv, max_pages * P, case.sign_seed)
    for b, n in enumerate(lens):
        for j in range((n + P - 1) // P):
            k = min(P, n - j * P)
            assert np.array_equal(kp[table[b, j], :, :k].cpu().numpy(), ko[b, :, j * P:j * P + k])
            assert np.array_equal(vp[table[b, j], :, :k].cpu().numpy(), vo[b, :, j * P:j * P + k])
    q = torch.from_numpy(case.q).cuda()
    lt = torch.tensor(lens, dtype=torch.int32, device="cuda")
    got = T.tbq4_attn_decode_paged(q, kp, vp, tab, lt, max_pages * P, case.softmax_scale,
                                   case.sign_seed)
    assert T.tbq4_get_device_status() == 0
    want = oracle.attn_decode(case.q, ko, vo, np.asarray(lens, np.int32), case.softmax_scale,
                              case.sign_seed)
    check_decode(got.float().cpu().numpy(), want)
    del kp, vp
    torch.cuda.empty_cache()


def test_prefill_past_4gb(T):
    """Chunked prefill over one sequence whose last KV head starts past 2^32
    (two caches of [4][21,692,416][66], 5.7 GB each): the chunk's append and
    the attention's tile copies use 64-bit offsets."""
    import torch
    from helpers import PREFILL_REL_L2, capacity_for, gpu_caches, rel_l2
    n_cached, n_new, Hq, Hkv, cap = 1000, 130, 24, 4, 21_692_416
    assert (Hkv - 1) * cap * 66 > GB4
    case = W.prefill_case("prefill_past_4gb", 96, n_cached, n_new, Hq, Hkv)
    kc = gpu_caches([case.k[:n_cached]], Hkv, cap, case.sign_seed)[0]
    vc = gpu_caches([case.v[:n_cached]], Hkv, cap, case.sign_seed)[0]
    start = torch.tensor([n_cached], dtype=torch.int32, device="cuda")
    for cache, x in ((kc, case.k), (vc, case.v)):
        chunk = torch.from_numpy(np.ascontiguousarray(x[n_cached:])[None]).cuda()
        T.tbq4_quantize_append(chunk, start, cache[None], sign_seed=case.sign_seed)
    q = torch.from_numpy(case.q_bf16.view(np.int16)).cuda().view(torch.bfloat16)
    got = T.tbq4_attn_prefill_chunk(q, n_cached, kc, vc, case.softmax_scale, case.sign_seed)
    assert T.tbq4_get_device_status() == 0
    small = capacity_for(n_cached + n_new)
    ko = oracle_caches([case.k], Hkv, small, case.sign_seed)[0]
    vo = oracle_caches([case.v], Hkv, small, case.sign_seed)[0]
    n = n_cached + n_new
    assert np.array_equal(kc[:, :n].cpu().numpy(), ko[:, :n])
    assert np.array_equal(vc[:, :n].cpu().numpy(), vo[:, :n])
    want = oracle.attn_prefill(case.q, n_cached, ko, vo, case.softmax_scale, case.sign_seed)
    assert rel_l2(got.float().cpu().numpy(), want) <= PREFILL_REL_L2
    del kc, vc
    torch.cuda.empty_cache()

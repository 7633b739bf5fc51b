"""GPU chunked prefill against the fp64 oracle (rel-L2 <= 1e-2).

The chunk's K/V are quantise-appended by the GPU before attention, as the
prefill workload does; the oracle quantises the same rows itself.
"""
import numpy as np
import pytest

import oracle
from long_context_attention_tbq4_b200 import workloads as W

from helpers import PREFILL_REL_L2, capacity_for, gpu_caches, oracle_caches, rel_l2

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def T():
    import torch
    import long_context_attention_tbq4_b200 as pkg
    assert torch.cuda.is_available()
    return pkg


def gpu_prefill(T, case, cap):
    """Cached rows appended first, then the chunk, then attention."""
    import torch
    kc = gpu_caches([case.k[:case.n_cached]], case.Hkv, cap, case.sign_seed)[0]
    vc = gpu_caches([case.v[:case.n_cached]], case.Hkv, cap, case.sign_seed)[0]
    start = torch.tensor([case.n_cached], dtype=torch.int32, device="cuda")
    for cache, x in ((kc, case.k), (vc, case.v)):
        chunk = torch.from_numpy(np.ascontiguousarray(x[case.n_cached:])[None]).cuda()
        T.tbq4_quantize_append(chunk, start, cache[None], sign_seed=case.sign_seed)
    q = torch.from_numpy(case.q_bf16.view(np.int16)).cuda().view(torch.bfloat16)
    out = T.tbq4_attn_prefill_chunk(q, case.n_cached, kc, vc, case.softmax_scale,
                                    case.sign_seed)
    assert T.tbq4_get_device_status() == 0
    return out.float().cpu().numpy(), kc, vc


def oracle_prefill(case, cap, rows=None):
    ko = oracle_caches([case.k], case.Hkv, cap, case.sign_seed)[0]
    vo = oracle_caches([case.v], case.Hkv, cap, case.sign_seed)[0]
    return oracle.attn_prefill(case.q, case.n_cached, ko, vo, case.softmax_scale,
                               case.sign_seed, rows=rows)


@pytest.mark.parametrize("n_cached,n_new,Hq,Hkv", [(0, 1, 4, 1), (0, 37, 8, 2),
                                                   (300, 37, 8, 2), (1000, 130, 24, 4),
                                                   (4093, 64, 12, 2)])
def test_prefill_small(T, n_cached, n_new, Hq, Hkv):
    case = W.prefill_case("small", 50 + n_new, n_cached, n_new, Hq, Hkv)
    cap = capacity_for(n_cached + n_new)
    got, _, _ = gpu_prefill(T, case, cap)
    want = oracle_prefill(case, cap)
    assert rel_l2(got, want) <= PREFILL_REL_L2


def test_prefill_131k_sampled_rows(T):
    case = W.prefill_131k()
    cap = W.round_capacity(case.n_cached + case.n_new)
    got, _, _ = gpu_prefill(T, case, cap)
    qi = [0, 1, 2, 127, 128, 255, 256, 383, 510, 511]
    rows = np.array([i * case.Hq + h for i in qi for h in range(0, case.Hq, 5)], np.int32)
    want = oracle_prefill(case, cap, rows=rows).reshape(-1, 128)[rows]
    sel = got.reshape(-1, 128)[rows]
    assert rel_l2(sel, want) <= PREFILL_REL_L2
    assert np.isfinite(got).all()

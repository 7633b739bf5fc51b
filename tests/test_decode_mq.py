"""Multi-query decode (q_len new tokens per sequence) against the fp64
oracle: query token i of sequence b is the chunked-prefill row i over
n_cached = len_b - q_len keys (bottom-right causal), so the oracle's prefill
attention is the reference.  Tolerance as decode: max-abs 2e-3 beyond the
fp16 output rounding, rel-L2 1e-3.
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


def run_mq(T, case, capacity=None):
    import torch
    q_len = case.q.shape[1]
    lens = np.asarray(case.seq_lens, np.int32)
    cap = capacity or capacity_for(int(lens.max()))
    kg = gpu_caches(case.k, case.Hkv, cap, case.sign_seed)
    vg = gpu_caches(case.v, case.Hkv, cap, case.sign_seed)
    q = torch.from_numpy(case.q).cuda()
    out = T.tbq4_attn_decode_mq(q, kg, vg, torch.from_numpy(lens).cuda(), int(lens.max()),
                                case.softmax_scale, case.sign_seed)
    assert T.tbq4_get_device_status() == 0
    got = out.float().cpu().numpy()
    ko = oracle_caches(case.k, case.Hkv, cap, case.sign_seed)
    vo = oracle_caches(case.v, case.Hkv, cap, case.sign_seed)
    want = np.stack([oracle.attn_prefill(case.q[b], int(lens[b]) - q_len, ko[b], vo[b],
                                         case.softmax_scale, case.sign_seed)
                     for b in range(case.B)])
    return got, want, (q, kg, vg, lens)


@pytest.mark.parametrize("q_len,G", [(2, 4), (3, 6), (4, 6), (4, 8), (4, 1), (2, 8)])
def test_mq_small(T, q_len, G):
    Hkv = 2
    case = W.mq_case("mq", 40 + 10 * q_len + G, 2, q_len, G * Hkv, Hkv, [1500, 333])
    got, want, _ = run_mq(T, case)
    check_decode(got, want)


def test_mq_ragged_and_short(T):
    # lengths at the q_len minimum, inside one tile, across tiles and splits
    lens = [4, 5, 127, 128, 129, 700, 5000]
    case = W.mq_case("mq_ragged", 55, len(lens), 4, 24, 4, lens, dist="t4")
    got, want, _ = run_mq(T, case)
    check_decode(got, want)


def test_mq_one_token_equals_decode(T):
    import torch
    case = W.mq_case("mq1", 56, 2, 1, 12, 2, [2000, 700])
    got, want, (q, kg, vg, lens) = run_mq(T, case)
    check_decode(got, want)
    ref = T.tbq4_attn_decode(q[:, 0].contiguous(), kg, vg, torch.from_numpy(lens).cuda(),
                             int(lens.max()), case.softmax_scale, case.sign_seed)
    assert np.array_equal(got[:, 0], ref.float().cpu().numpy())


def test_mq_262k(T):
    got, want, _ = run_mq(T, W.mq_262k(), capacity=262144)
    check_decode(got, want)

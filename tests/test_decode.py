"""GPU decode attention against the fp64 oracle.

Both sides quantise the same seeded fp32 K/V themselves (the GPU with
tbq4_quantize_append, the oracle with its own encoder); the tolerance is
max-abs <= 2e-3 and rel-L2 <= 1e-3 over the whole output.
"""
import numpy as np
import pytest

import oracle
from long_context_attention_tbq4_b200 import workloads as W

from helpers import capacity_for, check_decode, gpu_caches, oracle_caches, rel_l2

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def T():
    import torch
    import long_context_attention_tbq4_b200 as pkg
    assert torch.cuda.is_available()
    return pkg


def run_case(T, case, capacity=None, split_tokens=0, check_bytes=False):
    import torch
    cap = capacity or capacity_for(max(max(c.shape[0] for c in case.k), 1))
    kg = gpu_caches(case.k, case.Hkv, cap, case.sign_seed)
    vg = gpu_caches(case.v, case.Hkv, cap, case.sign_seed)
    lens = np.asarray(case.seq_lens, np.int32)
    q = torch.from_numpy(case.q).cuda()
    out = T.tbq4_attn_decode(q, kg, vg, torch.from_numpy(lens).cuda(), int(lens.max()),
                             case.softmax_scale, case.sign_seed, split_tokens=split_tokens)
    assert T.tbq4_get_device_status() == 0
    got = out.float().cpu().numpy()
    ko = oracle_caches(case.k, case.Hkv, cap, case.sign_seed)
    vo = oracle_caches(case.v, case.Hkv, cap, case.sign_seed)
    if check_bytes:
        kgn = kg.cpu().numpy()
        for b, x in enumerate(case.k):
            assert np.array_equal(kgn[b, :, :len(x)], ko[b, :, :len(x)])
    want = oracle.attn_decode(case.q, ko, vo, lens, case.softmax_scale, case.sign_seed)
    return got, want, (q, kg, vg, lens)


def test_tiny_decode(T):
    got, want, _ = run_case(T, W.tiny_decode(), check_bytes=True)
    check_decode(got, want)


def test_decode_32k(T):
    got, want, _ = run_case(T, W.decode_32k())
    check_decode(got, want)


def test_decode_262k_outliers(T):
    got, want, _ = run_case(T, W.decode_262k(), capacity=262144)
    check_decode(got, want)


def test_ragged_batch(T):
    case = W.ragged_decode()
    got, want, _ = run_case(T, case, capacity=W.round_capacity(case.seq_lens.max()))
    check_decode(got, want)


def test_odd_lengths_ragged(T):
    lens = [1, 7, 8, 9, 31, 32, 33, 127, 129, 255, 257, 528, 1000, 1023]
    case = W.decode_case("odd", 11, len(lens), 12, 2, lens)
    got, want, _ = run_case(T, case, capacity=1024)
    check_decode(got, want)


@pytest.mark.parametrize("G", [1, 2, 4, 6, 8])
def test_group_sizes(T, G):
    Hkv = 2
    case = W.decode_case("gqa", 20 + G, 2, G * Hkv, Hkv, [777, 1500])
    got, want, _ = run_case(T, case)
    check_decode(got, want)


def test_split_counts_agree(T):
    import torch
    case = W.decode_case("splits", 31, 1, 8, 2, [5000])
    results = []
    for st in [32, 64, 256, 1024, 2048, 4096, 8192, 0]:
        got, want, _ = run_case(T, case, split_tokens=st)
        check_decode(got, want)
        results.append(got)
    for r in results[1:]:
        assert rel_l2(r, results[0]) < 1e-3


def test_many_splits_running_merge(T):
    # 8 heads a group and 3,438 splits of 32 keys: the combine merges
    # thousands of partials per output row
    case = W.decode_case("many_splits", 33, 1, 8, 1, [110000])
    got, want, _ = run_case(T, case, split_tokens=32)
    check_decode(got, want)
    got2, _, _ = run_case(T, case)
    assert rel_l2(got, got2) < 1e-3


def test_zero_length_gives_zero_row(T):
    case = W.decode_case("zero", 41, 3, 4, 1, [0, 5, 0])
    got, want, _ = run_case(T, case, capacity=8)
    assert np.all(got[0] == 0) and np.all(got[2] == 0)
    check_decode(got[1], want[1])


def test_length_above_max_len_is_flagged(T):
    import torch
    case = W.decode_case("over", 42, 1, 4, 1, [64])
    kg = gpu_caches(case.k, 1, 64, 0)
    vg = gpu_caches(case.v, 1, 64, 0)
    q = torch.from_numpy(case.q).cuda()
    T.tbq4_attn_decode(q, kg, vg, torch.tensor([64], dtype=torch.int32, device="cuda"), 32,
                       case.softmax_scale, 0)
    assert T.tbq4_get_device_status() == 4
    assert T.tbq4_get_device_status() == 0


def test_deterministic(T):
    import torch
    case = W.decode_case("det", 43, 1, 24, 4, [20000])
    _, _, (q, kg, vg, lens) = run_case(T, case)
    lt = torch.from_numpy(lens).cuda()
    a = T.tbq4_attn_decode(q, kg, vg, lt, int(lens.max()), case.softmax_scale, 0)
    b = T.tbq4_attn_decode(q, kg, vg, lt, int(lens.max()), case.softmax_scale, 0)
    assert torch.equal(a, b)


def test_merge_with_garbage_workspace_and_graph_replay(T):
    """The split kernel and its combine (a programmatic dependent launch)
    share only the workspace.  A workspace holding arbitrary bytes, and
    replays of a captured call, must give the same output as a fresh call."""
    import torch
    case = W.decode_case("merge", 91, 2, 16, 4, [5000, 12000])
    cap = 12000
    kg = gpu_caches(case.k, case.Hkv, cap, case.sign_seed)
    vg = gpu_caches(case.v, case.Hkv, cap, case.sign_seed)
    q = torch.from_numpy(case.q).cuda()
    lens = torch.from_numpy(np.asarray(case.seq_lens, np.int32)).cuda()
    max_len = int(case.seq_lens.max())
    ref = T.tbq4_attn_decode(q, kg, vg, lens, max_len, case.softmax_scale, case.sign_seed)
    torch.cuda.synchronize()
    for fill in (0xFF, 0x00, 0x5A):
        ws = torch.full((T.tbq4_decode_workspace_bytes(2, 16, 4, max_len),), fill,
                        dtype=torch.uint8, device="cuda")
        out = T.tbq4_attn_decode(q, kg, vg, lens, max_len, case.softmax_scale, case.sign_seed,
                                 workspace=ws)
        assert T.tbq4_get_device_status() == 0
        assert torch.equal(out, ref)
    ws = torch.empty(T.tbq4_decode_workspace_bytes(2, 16, 4, max_len), dtype=torch.uint8,
                     device="cuda")
    out = torch.empty_like(ref)
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        T.tbq4_attn_decode(q, kg, vg, lens, max_len, case.softmax_scale, case.sign_seed,
                           workspace=ws, out=out)
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        T.tbq4_attn_decode(q, kg, vg, lens, max_len, case.softmax_scale, case.sign_seed,
                           workspace=ws, out=out)
    for _ in range(3):
        out.fill_(float("nan"))
        g.replay()
        torch.cuda.synchronize()
        assert torch.equal(out, ref)
    del g
    assert T.tbq4_get_device_status() == 0

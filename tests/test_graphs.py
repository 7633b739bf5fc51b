"""CUDA-graph replay of decode steps.

The launch shape depends only on the host arguments (batch, heads, max_len),
and every length is read from device memory, so one captured step serves
every length up to max_len: with the capacity padded (the page's
LLAMA_KV_PAD_MIN, 4,096 by default) a graph is recaptured only when a
sequence crosses a padding boundary (trefon.com, "Kontekst 262K na jednej
RTX 4090", section 2: upstream pads the KV cache to 256, the page to a
configurable minimum).  Each replay here must equal an eager call on the
same inputs, bit for bit, for the fused decode step, paged decode and the
3-bit decode.
"""
import numpy as np
import pytest

from long_context_attention_tbq4_b200 import workloads as W

from helpers import gpu_caches

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def T():
    import torch
    import long_context_attention_tbq4_b200 as pkg
    assert torch.cuda.is_available()
    return pkg


def _capture(fn):
    import torch
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        fn()                                      # warm-up outside the capture
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        fn()
    return g


def test_graph_replayed_decode_steps_over_growing_lengths(T):
    """Four fused decode steps (append the new token, attend) replayed from one
    graph captured with max_len = the padded capacity, against eager steps on
    a copy of the caches."""
    import torch
    rng = np.random.default_rng(77)
    B, Hq, Hkv = 2, 16, 4
    start = [1000, 2500]
    pad = W.round_capacity(max(start) + 8)            # 4096
    case = W.decode_case("graph_steps", 78, B, Hq, Hkv, start)
    kc = gpu_caches(case.k, Hkv, pad, case.sign_seed)
    vc = gpu_caches(case.v, Hkv, pad, case.sign_seed)
    k2, v2 = kc.clone(), vc.clone()
    q = torch.zeros((B, Hq, 128), dtype=torch.float32, device="cuda")
    kn = torch.zeros((B, Hkv, 128), dtype=torch.float32, device="cuda")
    vn = torch.zeros_like(kn)
    lens = torch.tensor(start, dtype=torch.int32, device="cuda")
    ws = torch.empty(T.tbq4_decode_workspace_bytes(B, Hq, Hkv, pad), dtype=torch.uint8,
                     device="cuda")
    out = torch.empty((B, Hq, 128), dtype=torch.float16, device="cuda")

    def step():
        T.tbq4_attn_decode_append(q, kn, vn, kc, vc, lens, pad, case.softmax_scale,
                                  case.sign_seed, workspace=ws, out=out)

    g = _capture(step)
    # the warm-up and capture calls appended at lens; start the steps afresh
    kc.copy_(k2)
    vc.copy_(v2)
    for t in range(4):
        lens.add_(1)                                    # this step's token is appended
        q.copy_(torch.from_numpy(rng.standard_normal((B, Hq, 128)).astype(np.float32)))
        kn.copy_(torch.from_numpy(rng.standard_normal((B, Hkv, 128)).astype(np.float32)))
        vn.copy_(torch.from_numpy(rng.standard_normal((B, Hkv, 128)).astype(np.float32)))
        out.fill_(float("nan"))
        g.replay()
        ref = T.tbq4_attn_decode_append(q, kn, vn, k2, v2, lens.clone(), pad,
                                        case.softmax_scale, case.sign_seed)
        torch.cuda.synchronize()
        assert torch.equal(out, ref), t
        assert torch.equal(kc, k2) and torch.equal(vc, v2), t
    del g
    assert T.tbq4_get_device_status() == 0


def test_graph_replayed_paged_decode(T):
    import torch
    lens = [3000, 17, 900]
    case = W.decode_case("graph_paged", 79, 3, 8, 2, lens)
    P = 256
    table, n_pages = W.page_table(179, lens, P)
    tab = torch.from_numpy(table).cuda()
    kp, vp = T.empty_pool(n_pages, 2, P), T.empty_pool(n_pages, 2, P)
    zero = torch.zeros(1, dtype=torch.int32, device="cuda")
    for b in range(3):
        for pool, x in ((kp, case.k[b]), (vp, case.v[b])):
            T.tbq4_quantize_append_paged(torch.from_numpy(np.ascontiguousarray(x)[None]).cuda(),
                                         zero, tab[b:b + 1], pool, case.sign_seed)
    q = torch.from_numpy(case.q).cuda()
    dl = torch.tensor(lens, dtype=torch.int32, device="cuda")
    max_len = table.shape[1] * P
    ws = torch.empty(T.tbq4_decode_workspace_bytes(3, 8, 2, max_len), dtype=torch.uint8,
                     device="cuda")
    out = torch.empty((3, 8, 128), dtype=torch.float16, device="cuda")
    g = _capture(lambda: T.tbq4_attn_decode_paged(q, kp, vp, tab, dl, max_len,
                                                   case.softmax_scale, case.sign_seed,
                                                   workspace=ws, out=out))
    for shrink in (0, 5, 300):                          # shorter lengths, same graph
        dl.copy_(torch.tensor([n - min(shrink, n) for n in lens], dtype=torch.int32))
        out.fill_(float("nan"))
        g.replay()
        ref = T.tbq4_attn_decode_paged(q, kp, vp, tab, dl.clone(), max_len, case.softmax_scale,
                                       case.sign_seed)
        torch.cuda.synchronize()
        assert torch.equal(out, ref), shrink
    del g
    assert T.tbq4_get_device_status() == 0


def test_graph_replayed_tbq3_decode(T):
    import torch
    lens = [2000, 64]
    case = W.decode_case("graph_tbq3", 80, 2, 8, 2, lens)
    cap = 2048
    kc, vc = T.empty_cache3(2, 2, cap), T.empty_cache3(2, 2, cap)
    zero = torch.zeros(1, dtype=torch.int32, device="cuda")
    for b in range(2):
        for cache, x in ((kc, case.k[b]), (vc, case.v[b])):
            T.tbq3_quantize_append(torch.from_numpy(np.ascontiguousarray(x)[None]).cuda(), zero,
                                   cache[b:b + 1], case.sign_seed)
    q = torch.from_numpy(case.q).cuda()
    dl = torch.tensor(lens, dtype=torch.int32, device="cuda")
    ws = torch.empty(T.tbq4_decode_workspace_bytes(2, 8, 2, cap), dtype=torch.uint8,
                     device="cuda")
    out = torch.empty((2, 8, 128), dtype=torch.float16, device="cuda")
    g = _capture(lambda: T.tbq3_attn_decode(q, kc, vc, dl, cap, case.softmax_scale,
                                             case.sign_seed, workspace=ws, out=out))
    for n0 in (2000, 1999, 33):
        dl.copy_(torch.tensor([n0, 64], dtype=torch.int32))
        out.fill_(float("nan"))
        g.replay()
        ref = T.tbq3_attn_decode(q, kc, vc, dl.clone(), cap, case.softmax_scale, case.sign_seed)
        torch.cuda.synchronize()
        assert torch.equal(out, ref), n0
    del g
    assert T.tbq4_get_device_status() == 0

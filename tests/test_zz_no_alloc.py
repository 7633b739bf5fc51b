"""tbq4_attn_decode_noalloc: decode attention for callers that cannot
allocate device memory where they call it (a plugin inside a framework that
owns all device memory, a serving loop with memory fixed up front).  It
takes no workspace; its scratch is a fixed 8 MiB array inside the library.

These tests call it through the C ABI and check it bit for bit against the
workspace-taking tbq4_attn_decode on the same inputs, on calls in a row with
a call of another shape in between (the shared scratch keeps the previous
call's contents, which must not matter), once against the oracle, and check
that a call needing more than the fixed scratch is refused before anything
is launched.  They need nothing from the other test files and run
the same alone or after them.
"""
import ctypes as C

import numpy as np
import pytest

from long_context_attention_tbq4_b200 import workloads as W

from helpers import check_decode, gpu_caches

pytestmark = pytest.mark.gpu

NOALLOC_SCRATCH_BYTES = 8 << 20


@pytest.fixture(scope="module")
def T():
    import torch
    import long_context_attention_tbq4_b200 as pkg
    assert torch.cuda.is_available()
    return pkg


def _p(t):
    return C.c_void_p(t.data_ptr())


def _noalloc(T, q, kc, vc, lens, max_len, scale, seed, out):
    import torch
    from long_context_attention_tbq4_b200._lib import lib
    B, Hq, _ = q.shape
    _, Hkv, cap, _ = kc.shape
    return lib.tbq4_attn_decode_noalloc(
        _p(q), _p(kc), _p(vc), _p(lens), int(max_len), B, Hq, Hkv, cap, float(scale),
        C.c_uint64(seed), _p(out), C.c_void_p(torch.cuda.current_stream().cuda_stream))


def _decode_pair(T, name, seed, Hq, Hkv, lens, cap):
    """Caches, inputs and the workspace decode's output for one shape."""
    import torch
    case = W.decode_case(name, seed, len(lens), Hq, Hkv, lens)
    kc = gpu_caches(case.k, case.Hkv, cap, case.sign_seed)
    vc = gpu_caches(case.v, case.Hkv, cap, case.sign_seed)
    q = torch.from_numpy(case.q).cuda()
    seq = torch.from_numpy(case.seq_lens).cuda()
    max_len = int(case.seq_lens.max())
    assert T.tbq4_decode_workspace_bytes(case.B, case.Hq, case.Hkv, max_len) <= NOALLOC_SCRATCH_BYTES
    ref = T.tbq4_attn_decode(q, kc, vc, seq, max_len, case.softmax_scale, case.sign_seed)
    torch.cuda.synchronize()
    return case, kc, vc, q, seq, max_len, ref


def test_noalloc_matches_decode_with_workspace(T):
    # The same kernels with the same split plan as tbq4_attn_decode, so the
    # output must be the same bits.  Between the two calls of the first
    # shape, a call of another shape (another split plan, other partials)
    # leaves different contents in the shared scratch, which must not matter.
    import torch
    import oracle
    from helpers import oracle_caches
    a = _decode_pair(T, "noalloc", 77, 24, 4, [7000, 1, 20000], 20000)
    b = _decode_pair(T, "noalloc_b", 78, 8, 2, [333, 4100], 4104)
    for case, kc, vc, q, seq, max_len, ref in (a, b, a):
        out = torch.full_like(ref, float("nan"))
        assert _noalloc(T, q, kc, vc, seq, max_len, case.softmax_scale, case.sign_seed,
                        out) == 0
        assert T.tbq4_get_device_status() == 0
        assert torch.equal(out, ref)
    # and once against the oracle
    case, kc, vc, q, seq, max_len, ref = a
    ko = oracle_caches(case.k, case.Hkv, kc.shape[2], case.sign_seed)
    vo = oracle_caches(case.v, case.Hkv, kc.shape[2], case.sign_seed)
    want = oracle.attn_decode(case.q, ko, vo, case.seq_lens, case.softmax_scale,
                              case.sign_seed)
    check_decode(ref.float().cpu().numpy(), want)


def test_noalloc_refuses_more_than_its_scratch(T):
    import torch
    B, Hq, Hkv, cap = 1024, 64, 8, 8
    need = T.tbq4_decode_workspace_bytes(B, Hq, Hkv, cap)
    assert need > NOALLOC_SCRATCH_BYTES
    q = torch.zeros((B, Hq, 128), dtype=torch.float32, device="cuda")
    kc = torch.zeros((B, Hkv, cap, 66), dtype=torch.uint8, device="cuda")
    lens = torch.full((B,), cap, dtype=torch.int32, device="cuda")
    out = torch.full((B, Hq, 128), 7.0, dtype=torch.float16, device="cuda")
    assert _noalloc(T, q, kc, kc, lens, cap, 0.1, 0, out) == 5      # TBQ4_ERR_WORKSPACE
    torch.cuda.synchronize()
    assert T.tbq4_get_device_status() == 0
    assert bool((out == 7.0).all())                                 # nothing was launched

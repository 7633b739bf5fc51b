"""The device-side failure path, exercised without faulting, trapping or
hanging the GPU: a bounded wait on a barrier that nothing completes (no copy
in flight) gives up, records TBQ4_ERR_DEVICE_TIMEOUT, and the context stays
usable for the next normal call."""
import numpy as np
import pytest

import oracle
from long_context_attention_tbq4_b200 import workloads as W

from helpers import check_decode, gpu_caches, oracle_caches

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def T():
    import torch
    import long_context_attention_tbq4_b200 as pkg
    assert torch.cuda.is_available()
    return pkg


def test_bounded_wait_times_out_and_the_context_survives(T):
    import torch
    assert T.tbq4_get_device_status() == 0
    T.tbq4_selftest_bounded_wait(256)
    assert T.tbq4_get_device_status() == 7          # TBQ4_ERR_DEVICE_TIMEOUT
    assert T.tbq4_get_device_status() == 0          # read and cleared
    # the next normal call runs and is correct
    case = W.decode_case("after_timeout", 91, 1, 8, 2, [3000])
    cap = 3000
    kc = gpu_caches(case.k, case.Hkv, cap, case.sign_seed)
    vc = gpu_caches(case.v, case.Hkv, cap, case.sign_seed)
    q = torch.from_numpy(case.q).cuda()
    lens = torch.from_numpy(case.seq_lens).cuda()
    got = T.tbq4_attn_decode(q, kc, vc, lens, 3000, case.softmax_scale, case.sign_seed)
    assert T.tbq4_get_device_status() == 0
    ko = oracle_caches(case.k, case.Hkv, cap, case.sign_seed)
    vo = oracle_caches(case.v, case.Hkv, cap, case.sign_seed)
    want = oracle.attn_decode(case.q, ko, vo, case.seq_lens, case.softmax_scale,
                              case.sign_seed)
    check_decode(got.float().cpu().numpy(), want)


def test_timeout_is_reported_once_per_read(T):
    # two timeouts before a read still read back as one code, then nothing
    T.tbq4_selftest_bounded_wait(64)
    T.tbq4_selftest_bounded_wait(64)
    assert T.tbq4_get_device_status() == 7
    assert T.tbq4_get_device_status() == 0

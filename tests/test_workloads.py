"""The seeded input generators against the input recipe (CPU).

The recipe: numpy default_rng(seed), draw order q, K, V (then the outlier
channels); N(0,1) fp32, or Student-t with nu = 4 for the heavy-tailed cases;
4 outlier K channels per KV head scaled x10 for the 262K decode; ragged
lengths drawn first, uniform on [16,384, 98,304]; prefill q rounded to bf16
(nearest even).  Each test rebuilds a draw from the seed, or checks a
statistic the recipe fixes.
"""
import numpy as np
import pytest

from long_context_attention_tbq4_b200 import workloads as W

D = 128


def test_draw_order_q_then_k_then_v_then_channels():
    case = W.decode_case("order", 7, 2, 4, 2, [40, 9], k_outliers=3, outlier_gain=10.0)
    rng = np.random.default_rng(7)
    q = rng.standard_normal((2, 4, D), dtype=np.float32)
    k = [rng.standard_normal((n, 2, D), dtype=np.float32) for n in (40, 9)]
    v = [rng.standard_normal((n, 2, D), dtype=np.float32) for n in (40, 9)]
    ch = np.stack([rng.choice(D, 3, replace=False) for _ in range(2)])
    assert np.array_equal(case.q, q)
    assert np.array_equal(case.meta["outlier_channels"], ch)
    for b in range(2):
        for h in range(2):
            k[b][:, h, ch[h]] *= np.float32(10.0)
        assert np.array_equal(case.k[b], k[b])
        assert np.array_equal(case.v[b], v[b])
    assert list(case.seq_lens) == [40, 9] and case.Hq == 4 and case.Hkv == 2
    assert case.softmax_scale == pytest.approx(1 / np.sqrt(D)) and case.sign_seed == 0


def test_named_decode_configs():
    t = W.tiny_decode()
    assert (t.B, t.Hq, t.Hkv, list(t.seq_lens)) == (1, 4, 1, [1024])
    assert np.array_equal(t.q, np.random.default_rng(0).standard_normal((1, 4, D),
                                                                        dtype=np.float32))
    c = W.decode_32k()
    assert (c.B, c.Hq, c.Hkv, list(c.seq_lens)) == (1, 24, 4, [32768])
    assert c.k[0].shape == (32768, 4, D) and c.k[0].dtype == np.float32
    assert np.array_equal(c.q, np.random.default_rng(1).standard_normal((1, 24, D),
                                                                        dtype=np.float32))


def test_decode_262k_outlier_channels():
    c = W.decode_262k()
    assert (c.B, c.Hq, c.Hkv, list(c.seq_lens)) == (1, 24, 4, [262144])
    ch = c.meta["outlier_channels"]
    assert ch.shape == (4, 4)
    k, v = c.k[0], c.v[0]
    for h in range(4):
        assert len(set(ch[h].tolist())) == 4                  # without replacement
        sd = k[:, h, :].std(axis=0)
        others = np.setdiff1d(np.arange(D), ch[h])
        assert np.allclose(sd[ch[h]], 10.0, rtol=0.01)       # x10 channels
        assert np.allclose(sd[others], 1.0, rtol=0.01)
        assert np.allclose(v[:, h, :].std(axis=0), 1.0, rtol=0.01)   # V untouched
    assert abs(float(k.mean())) < 0.01 and abs(float(v.mean())) < 0.01


def test_student_t_tails():
    c = W.decode_case("t4", 11, 1, 4, 1, [60000], dist="t4")
    x = np.concatenate([c.k[0].ravel(), c.v[0].ravel()]).astype(np.float64)
    # Student-t, nu = 4: variance nu / (nu - 2) = 2, raw samples (no rescale); the
    # fourth moment is infinite, so the sample kurtosis is far above the normal's 3
    assert x.var() == pytest.approx(2.0, rel=0.05)
    kurt = ((x - x.mean()) ** 4).mean() / x.var() ** 2
    assert kurt > 6.0
    assert np.array_equal(c.q, np.random.default_rng(11).standard_normal((1, 4, D),
                                                                        dtype=np.float32))


def test_ragged_lengths_drawn_first_and_in_range():
    lens, rng = W.ragged_lengths()
    assert np.array_equal(lens, np.random.default_rng(4).integers(16384, 98304, size=8,
                                                                  endpoint=True))
    assert lens.dtype == np.int32 and len(lens) == 8
    assert lens.min() >= 16384 and lens.max() <= 98304
    # the next draw from the same generator is q
    q = rng.standard_normal((8, 24, D), dtype=np.float32)
    rng2 = np.random.default_rng(4)
    rng2.integers(16384, 98304, size=8, endpoint=True)
    assert np.array_equal(q, rng2.standard_normal((8, 24, D), dtype=np.float32))


def test_bf16_round_is_nearest_even():
    import torch
    rng = np.random.default_rng(12)
    x = np.concatenate([rng.standard_normal(100000).astype(np.float32),
                        np.array([1.0 + 2.0 ** -8, 1.0 + 3 * 2.0 ** -8, -1.0 - 2.0 ** -8,
                                  1.0 + 2.0 ** -8 + 2.0 ** -20, 0.0, -0.0, 3.0e38],
                                 np.float32)])
    bits, f = W.bf16_round(x)
    want = torch.from_numpy(x).to(torch.bfloat16)
    assert np.array_equal(bits, want.view(torch.int16).numpy().view(np.uint16))
    assert np.array_equal(f, want.float().numpy())
    # ties: 1 + 2^-8 lies halfway between 1 and 1 + 2^-7 and goes to the even 1
    assert f[100000] == 1.0 and f[100001] == 1.0 + 2.0 ** -6 and f[100003] == 1.0 + 2.0 ** -7


def test_prefill_case_draw_order_and_bf16_q():
    c = W.prefill_case("p", 13, 100, 20, Hq=8, Hkv=2)
    rng = np.random.default_rng(13)
    qf = rng.standard_normal((20, 8, D), dtype=np.float32)
    k = rng.standard_normal((120, 2, D), dtype=np.float32)
    v = rng.standard_normal((120, 2, D), dtype=np.float32)
    bits, q = W.bf16_round(qf)
    assert np.array_equal(c.q_bf16, bits) and np.array_equal(c.q, q)
    assert np.array_equal(c.k, k) and np.array_equal(c.v, v)
    assert (c.n_cached, c.n_new, c.Hq, c.Hkv) == (100, 20, 8, 2)


def test_round_capacity():
    assert W.round_capacity(1) == 4096
    assert W.round_capacity(4096) == 4096
    assert W.round_capacity(4097) == 8192
    assert W.round_capacity(262144) == 262144
    assert W.round_capacity(131072 + 512) == 135168
    assert W.round_capacity(100, multiple=8) == 104


def test_generators_are_deterministic():
    a = W.decode_case("d", 21, 2, 4, 1, [33, 5], dist="t4")
    b = W.decode_case("d", 21, 2, 4, 1, [33, 5], dist="t4")
    assert np.array_equal(a.q, b.q)
    assert all(np.array_equal(x, y) for x, y in zip(a.k + a.v, b.k + b.v))

"""Pins of the fp64 CPU oracle against facts fixed outside it.

Each test checks the oracle against something other than itself: the numbers
the page prints (tests/golden/page_facts.json), published reference vectors
(SplitMix64), library special cases (scipy's Hadamard matrix, numpy's IEEE
half conversion), closed forms, invariants, error bounds, and pure-Python
brute force on tiny inputs (oracle/brute.py).
"""
import json
import math
import os
from decimal import Decimal, getcontext

import numpy as np
import pytest
import scipy.linalg

import oracle
from oracle import brute

D = 128
RNG = np.random.default_rng(12345)


def f32_bits(x):
    return int(np.asarray(x, np.float32).view(np.uint32))


# ------------------------------------------------------------- page facts
def test_block_layout_matches_page(golden_dir):
    facts = json.load(open(os.path.join(golden_dir, "page_facts.json")))
    assert oracle.lib().oracle_block_bytes() == facts["bytes_per_block"]
    assert facts["scale_bytes"] + facts["index_bytes"] == facts["bytes_per_block"]
    assert facts["bytes_per_block"] * 8 / facts["values_per_block"] == facts["bits_per_value"]
    # the oracle writes exactly 66 bytes for one block and nothing past them
    buf = np.full(80, 0xA5, np.uint8)
    x = RNG.standard_normal(D).astype(np.float32)
    s = oracle.signs(0)
    import ctypes as C
    oracle.lib().oracle_quantize_block(x.ctypes.data_as(C.c_void_p),
                                       s.ctypes.data_as(C.c_void_p),
                                       buf.ctypes.data_as(C.c_void_p))
    assert np.all(buf[66:] == 0xA5)
    assert np.array_equal(buf[:66], oracle.quantize_block(x, s))
    # 64 index bytes hold 128 4-bit indices
    assert facts["index_bytes"] * 2 == facts["values_per_block"]


def test_cache_footprint_ratio_matches_page(golden_dir):
    facts = json.load(open(os.path.join(golden_dir, "page_facts.json")))
    # TBQ4 : FP16 = 66 bytes : 256 bytes per 128 values
    ratio = facts["bytes_per_block"] / (2 * facts["values_per_block"])
    tbq4_gib = facts["fp16_cache_gib_printed"] * ratio
    assert tbq4_gib == pytest.approx(4.125)
    assert round(tbq4_gib, 1) == pytest.approx(facts["tbq4_cache_gib_printed"], abs=0.05)


# ------------------------------------------------------------- SplitMix64
def test_splitmix64_reference_vectors(golden_dir):
    g = json.load(open(os.path.join(golden_dir, "splitmix64.json")))
    for vec in g["vectors"]:
        want = [int(v) for v in vec["outputs"]]
        got = [int(v) for v in oracle.splitmix64(vec["seed"], len(want))]
        assert got == want


def test_signs_follow_splitmix64_bits(golden_dir):
    g = json.load(open(os.path.join(golden_dir, "splitmix64.json")))
    seed0 = [v for v in g["vectors"] if v["seed"] == 0][0]
    w = [int(v) for v in seed0["outputs"][:2]]
    want = [1 - 2 * ((w[i // 64] >> (i % 64)) & 1) for i in range(D)]
    assert list(oracle.signs(0)) == want
    s = oracle.signs(1234567)
    assert set(np.unique(s)) <= {-1, 1}


# ------------------------------------------------------------------ fp16
def test_f32_to_f16_matches_numpy_on_strided_sample():
    bits = np.arange(0, 2**32, 251, dtype=np.uint64).astype(np.uint32)
    x = bits.view(np.float32)
    got = oracle.f32_to_f16_array(x)
    with np.errstate(over="ignore", invalid="ignore"):
        want = x.astype(np.float16).view(np.uint16)
    nan = np.isnan(x)
    assert np.array_equal(got[~nan], want[~nan])
    assert np.all((got[nan] & 0x7C00) == 0x7C00) and np.all((got[nan] & 0x3FF) != 0)


@pytest.mark.parametrize("v,h", [
    (65504.0, 0x7BFF), (65519.99609375, 0x7BFF), (65520.0, 0x7C00),
    (2.0 ** -24, 0x0001), (2.0 ** -25, 0x0000), (3 * 2.0 ** -26, 0x0001),
    (2.0 ** -14, 0x0400), (1.0, 0x3C00), (-2.0, 0xC000),
    (1.0 + 2.0 ** -11, 0x3C00), (1.0 + 3 * 2.0 ** -11, 0x3C02),
])
def test_f32_to_f16_edge_cases(v, h):
    assert oracle.f32_to_f16_bits(v) == h
    with np.errstate(over="ignore"):
        assert int(np.float32(v).astype(np.float16).view(np.uint16)) == h


def test_f16_to_f64_all_patterns():
    hs = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    want = hs.view(np.float16).astype(np.float64)
    got = np.array([oracle.f16_bits_to_f64(int(h)) for h in hs])
    ok = np.isnan(want)
    assert np.array_equal(got[~ok], want[~ok]) and np.all(np.isnan(got[ok]))


# -------------------------------------------------------------- Hadamard
def test_hadamard_is_scipy_sylvester():
    H = np.array([[oracle.hadamard_entry(i, j) for j in range(D)] for i in range(D)])
    assert np.array_equal(H, scipy.linalg.hadamard(D))
    assert np.array_equal(H @ H, D * np.eye(D, dtype=H.dtype))


def test_rotation_matrix_is_orthogonal_and_signed():
    s = oracle.signs(0)
    R = oracle.rotation_matrix(s)
    H = scipy.linalg.hadamard(D).astype(np.float64)
    assert np.allclose(R, H @ np.diag(s.astype(np.float64)) / math.sqrt(D), rtol=0, atol=1e-16)
    assert np.abs(R @ R.T - np.eye(D)).max() < 1e-15
    assert np.abs(R.T @ R - np.eye(D)).max() < 1e-15


def test_rotation_constant_is_correctly_rounded():
    getcontext().prec = 60
    exact = Decimal(1) / Decimal(128).sqrt()
    c = np.float32(float(exact))
    # c is the binary32 nearest to 1/sqrt(128): its neighbours are farther
    up = np.nextafter(c, np.float32(1))
    dn = np.nextafter(c, np.float32(0))
    err = abs(Decimal(float(c)) - exact)
    assert err < abs(Decimal(float(up)) - exact) and err < abs(Decimal(float(dn)) - exact)
    assert f32_bits(c) == 0x3DB504F3
    e0 = np.zeros(D, np.float32)
    e0[0] = 1
    out = oracle.rotate_f32(e0, np.ones(D, np.int8))
    assert all(f32_bits(v) == 0x3DB504F3 for v in out)   # column 0 of H is all +1


def test_rotate_f32_unit_vectors_give_signed_hadamard_columns():
    s = oracle.signs(0)
    H = scipy.linalg.hadamard(D)
    c = np.array(0x3DB504F3, np.uint32).view(np.float32)
    for j in [0, 1, 2, 5, 63, 64, 100, 127]:
        e = np.zeros(D, np.float32)
        e[j] = 1
        want = (H[:, j] * s[j]).astype(np.float32) * c
        assert np.array_equal(oracle.rotate_f32(e, s), want)


def test_rotate_f32_exact_on_small_integers():
    # butterflies of small integers are exact in binary32, so the result is
    # fl32(c * (H D x)) with H from scipy and integer arithmetic
    s = oracle.signs(7)
    H = scipy.linalg.hadamard(D).astype(np.int64)
    c = np.array(0x3DB504F3, np.uint32).view(np.float32)
    for _ in range(20):
        x = RNG.integers(-64, 65, D)
        y = H @ (s.astype(np.int64) * x)
        want = y.astype(np.float32) * c
        assert np.array_equal(oracle.rotate_f32(x.astype(np.float32), s), want)


def test_rotate_f32_close_to_exact_rotation():
    s = oracle.signs(0)
    R = oracle.rotation_matrix(s)
    for _ in range(50):
        x = (RNG.standard_normal(D) * RNG.choice([1e-3, 1, 30])).astype(np.float32)
        exact = R @ x.astype(np.float64)
        got = oracle.rotate_f32(x, s).astype(np.float64)
        bound = 9 * 2.0 ** -24 * np.abs(x).sum() / math.sqrt(D) + 2.0 ** -24 * np.abs(exact)
        assert np.all(np.abs(got - exact) <= bound)


def test_rotate_f32_butterfly_order_is_pinned_bitwise():
    # Random and heavy-tailed vectors round differently under any other
    # stride order or association; the C oracle must equal the stage-wise
    # float32 restatement of the codebook's order bit for bit.
    from oracle import brute
    for seed in (0, 1, 12345):
        s = oracle.signs(seed)
        for t in range(100):
            kind = t % 4
            if kind == 0:
                x = RNG.standard_normal(D)
            elif kind == 1:
                x = RNG.standard_t(4, D) * 10.0
            elif kind == 2:
                x = RNG.standard_normal(D) * np.exp(RNG.uniform(-20, 20, D))
            else:
                x = RNG.uniform(-1, 1, D) * 65504.0
            x = x.astype(np.float32)
            got = oracle.rotate_f32(x, s)
            want = brute.rotate_f32_stages(x, s)
            assert np.array_equal(got.view(np.uint32), want.view(np.uint32)), (seed, t)


def test_rotate_f32_stages_detects_a_reordered_transform():
    # the pin is sensitive: descending strides give different bits on
    # random inputs
    from oracle import brute
    s = oracle.signs(0)
    diff = 0
    for _ in range(50):
        x = RNG.standard_normal(D).astype(np.float32)
        z = x * s.astype(np.float32)
        h = D // 2
        while h >= 1:
            blk = z.reshape(D // (2 * h), 2, h)
            a, b = blk[:, 0, :], blk[:, 1, :]
            z = np.stack([a + b, a - b], axis=1).reshape(D)
            h //= 2
        z = z * np.array(0x3DB504F3, np.uint32).view(np.float32)
        diff += not np.array_equal(z.view(np.uint32), brute.rotate_f32_stages(x, s).view(np.uint32))
    assert diff > 25


# ------------------------------------------------------------- quantiser
def test_level_index_is_nearest_level():
    # away from midpoints the binary32 index formula picks the nearest of the
    # 16 levels S*(2i-15)/15 (exact rational brute force, clamps included)
    n = 0
    for _ in range(4000):
        S = float(np.float16(RNG.uniform(1e-3, 100)))
        x = float(np.float32(RNG.uniform(-1.2, 1.2) * S))
        frac = (x / S * 7.5 + 7.5) % 1.0
        if abs(frac - 0.5) < 1e-4:
            continue
        assert oracle.level_index(x, S) == brute.nearest_level_index(x, S)
        n += 1
    assert n > 3900


def test_level_index_ties_go_to_even():
    checked = 0
    for S in [7.5, 15.0, 3.75, 0.234375]:
        for j in range(-14, 15):
            x = np.float32(j * S / 7.5) if S != 7.5 else np.float32(j)
            t = np.float32(x) / np.float32(S)
            u = t * np.float32(7.5)
            if u != np.float32(round(float(u))):
                continue                       # not an exact tie in binary32
            v = float(u) + 7.5
            if abs(v - math.floor(v) - 0.5) > 0:
                continue
            lo = math.floor(v)
            want = lo if lo % 2 == 0 else lo + 1
            want = min(max(want, 0), 15)
            assert oracle.level_index(float(x), S) == want
            checked += 1
    assert checked >= 20


def test_level_index_zero_scale_and_clamp():
    assert oracle.level_index(0.0, 0.0) == 8
    assert oracle.level_index(0.0, 1.0) == 8      # 7.5 ties to 8
    assert oracle.level_index(1.02, 1.0) == 15
    assert oracle.level_index(-1.02, 1.0) == 0


def test_block_scale_is_half_of_max_abs():
    for _ in range(200):
        xr = (RNG.standard_normal(D) * RNG.choice([1e-6, 1e-2, 1, 100, 1e4])).astype(np.float32)
        want = int(np.float16(np.abs(xr).max()).view(np.uint16))
        assert oracle.block_scale_bits(xr) == want
    assert oracle.block_scale_bits(np.full(D, 1e6, np.float32)) == 0x7BFF   # saturates
    assert oracle.block_scale_bits(np.zeros(D, np.float32)) == 0


def _unpack(blk):
    idx = np.empty(D, np.int64)
    idx[0::2] = blk[2:] & 15
    idx[1::2] = blk[2:] >> 4
    return int(blk[0]) | (int(blk[1]) << 8), idx


def test_on_grid_round_trip_and_byte_layout():
    s = oracle.signs(0)
    R = oracle.rotation_matrix(s)
    for _ in range(200):
        S = np.float16(RNG.uniform(0.05, 50))
        idx = RNG.integers(0, 16, D)
        idx[RNG.integers(0, D)] = RNG.choice([0, 15])   # a +-S level is present
        x_rot = float(S) * (2 * idx - 15) / 15.0
        x = (R.T @ x_rot).astype(np.float32)
        blk = oracle.quantize_block(x, s)
        sb, got_idx = _unpack(blk)
        assert sb == int(S.view(np.uint16))
        assert np.array_equal(got_idx, idx)
        # the layout itself: scale little endian first, then even element
        # in the low nibble
        want = np.empty(66, np.uint8)
        want[0], want[1] = sb & 0xFF, sb >> 8
        want[2:] = idx[0::2] | (idx[1::2] << 4)
        assert np.array_equal(blk, want)


def test_quantiser_invariants_and_error_bound():
    s = oracle.signs(3)
    R = oracle.rotation_matrix(s)
    for k in range(300):
        gain = [1e-3, 1.0, 10.0, 300.0][k % 4]
        x = (RNG.standard_t(4, D) * gain).astype(np.float32)
        blk = oracle.quantize_block(x, s)
        sb, idx = _unpack(blk)
        S = float(np.uint16(sb).view(np.float16))
        assert S > 0
        assert (idx == 0).any() or (idx == 15).any()      # max element on an end level
        exact = R @ x.astype(np.float64)
        xhat = oracle.dequant_block(blk)
        m = np.abs(exact).max()
        bound = S / 15 + abs(m - S) + 1e-5 * m
        assert np.all(np.abs(xhat - exact) <= bound)


def test_zero_block():
    blk = oracle.quantize_block(np.zeros(D, np.float32), oracle.signs(0))
    assert blk[0] == 0 and blk[1] == 0 and np.all(blk[2:] == 0x88)
    assert np.all(oracle.dequant_block(blk) == 0.0)


def test_dequant_matches_brute():
    s = oracle.signs(0)
    for _ in range(20):
        blk = oracle.quantize_block(RNG.standard_normal(D).astype(np.float32) * 3, s)
        assert np.array_equal(oracle.dequant_block(blk), np.array(brute.dequant(blk)))


def test_quantize_append_places_blocks():
    B, n_new, Hkv, cap = 2, 3, 2, 16
    seed = 5
    s = oracle.signs(seed)
    src = RNG.standard_normal((B, n_new, Hkv, D)).astype(np.float32)
    cache = np.full((B, Hkv, cap, 66), 0xAB, np.uint8)
    start = np.array([5, 0], np.int32)
    assert oracle.quantize_append(src, start, cap, seed, cache) == 0
    touched = np.zeros((B, Hkv, cap), bool)
    for b in range(B):
        for t in range(n_new):
            for h in range(Hkv):
                p = start[b] + t
                assert np.array_equal(cache[b, h, p], oracle.quantize_block(src[b, t, h], s))
                touched[b, h, p] = True
    assert np.all(cache[~touched] == 0xAB)
    start = np.array([15, 14], np.int32)     # rows past the capacity are skipped
    assert oracle.quantize_append(src, start, cap, seed, cache) == (2 + 1) * Hkv


# -------------------------------------------------------------- attention
def _random_cache(B, Hkv, cap, seed, gain=1.0):
    rng = np.random.default_rng(seed)
    k = np.zeros((B, Hkv, cap, 66), np.uint8)
    v = np.zeros((B, Hkv, cap, 66), np.uint8)
    src_k = (rng.standard_normal((B, cap, Hkv, D)) * gain).astype(np.float32)
    src_v = rng.standard_normal((B, cap, Hkv, D)).astype(np.float32)
    z = np.zeros(B, np.int32)
    oracle.quantize_append(src_k, z, cap, 0, k)
    oracle.quantize_append(src_v, z, cap, 0, v)
    return k, v


def test_decode_matches_pure_python_brute_force():
    B, Hq, Hkv, cap = 2, 4, 2, 8
    k, v = _random_cache(B, Hkv, cap, 1, gain=3.0)
    q = RNG.standard_normal((B, Hq, D)).astype(np.float32)
    lens = np.array([3, 4], np.int32)
    scale = 1 / math.sqrt(D)
    out = oracle.attn_decode(q, k, v, lens, scale, 0)
    s = [int(x) for x in oracle.signs(0)]
    for b in range(B):
        for h in range(Hq):
            g = h // (Hq // Hkv)
            want = brute.attend(q[b, h], [k[b, g, t] for t in range(lens[b])],
                                [v[b, g, t] for t in range(lens[b])], scale, s)
            assert np.allclose(out[b, h], want, rtol=0, atol=1e-13)


def test_decode_equals_unrotated_attention():
    # orthogonality of R: rotated-domain attention, rotated back, equals
    # ordinary attention on K = R^T Khat_rot, V = R^T Vhat_rot
    B, Hq, Hkv, cap = 1, 6, 1, 64
    k, v = _random_cache(B, Hkv, cap, 2)
    q = RNG.standard_normal((B, Hq, D)).astype(np.float32)
    n = 37
    scale = 0.3
    out = oracle.attn_decode(q, k, v, np.array([n], np.int32), scale, 0)
    s = oracle.signs(0).astype(np.float64)
    Rm = scipy.linalg.hadamard(D) * s[None, :] / math.sqrt(D)
    Kr = np.stack([brute.dequant(k[0, 0, t]) for t in range(n)])
    Vr = np.stack([brute.dequant(v[0, 0, t]) for t in range(n)])
    K, V = Kr @ Rm, Vr @ Rm              # rows: R^T x_rot
    for h in range(Hq):
        z = scale * (K @ q[0, h].astype(np.float64))
        p = np.exp(z - z.max())
        want = (p / p.sum()) @ V
        assert np.abs(out[0, h] - want).max() < 1e-12


def test_decode_closed_forms():
    s = oracle.signs(0).astype(np.float64)
    Rm = scipy.linalg.hadamard(D) * s[None, :] / math.sqrt(D)
    k, v = _random_cache(1, 1, 16, 3)
    # all keys equal -> uniform weights -> mean of V
    k_same = np.repeat(k[:, :, :1], 16, axis=2)
    q = RNG.standard_normal((1, 2, D)).astype(np.float32)
    out = oracle.attn_decode(q, k_same, v, np.array([16], np.int32), 1.0, 0)
    Vr = np.stack([brute.dequant(v[0, 0, t]) for t in range(16)])
    assert np.abs(out[0, 0] - Vr.mean(0) @ Rm).max() < 1e-13
    # one key dominates -> its V
    k_dom = np.zeros_like(k)                 # scale 0 blocks dequantise to 0
    t_star = 9
    k_dom[0, 0, t_star] = k[0, 0, t_star]
    kstar = np.array(brute.dequant(k[0, 0, t_star])) @ Rm
    qd = (1000 * kstar / np.linalg.norm(kstar)).astype(np.float32)[None, None, :]
    out = oracle.attn_decode(qd, k_dom, v, np.array([16], np.int32), 1.0, 0)
    assert np.abs(out[0, 0] - np.array(brute.dequant(v[0, 0, t_star])) @ Rm).max() < 1e-12


def test_decode_empty_context_is_zero():
    k, v = _random_cache(1, 1, 8, 4)
    out = oracle.attn_decode(np.ones((1, 2, D), np.float32), k, v,
                             np.array([0], np.int32), 1.0, 0)
    assert np.all(out == 0.0)


def test_decode_row_subset_matches_full():
    k, v = _random_cache(2, 2, 32, 5)
    q = RNG.standard_normal((2, 4, D)).astype(np.float32)
    lens = np.array([32, 17], np.int32)
    full = oracle.attn_decode(q, k, v, lens, 0.1, 0)
    rows = np.array([5, 2], np.int32)
    part = oracle.attn_decode(q, k, v, lens, 0.1, 0, rows=rows)
    for r in rows:
        assert np.array_equal(part.reshape(-1, D)[r], full.reshape(-1, D)[r])


def test_prefill_row_equals_decode_at_its_length():
    Hq, Hkv, n_cached, n_new = 4, 2, 21, 5
    cap = 32
    k, v = _random_cache(1, Hkv, cap, 6)
    q = RNG.standard_normal((n_new, Hq, D)).astype(np.float32)
    scale = 1 / math.sqrt(D)
    pre = oracle.attn_prefill(q, n_cached, k[0], v[0], scale, 0)
    for i in range(n_new):
        dec = oracle.attn_decode(q[i][None], k, v, np.array([n_cached + i + 1], np.int32), scale, 0)
        assert np.array_equal(pre[i], dec[0])
    # causal: the last row sees the whole chunk, the first row only itself
    s = [int(x) for x in oracle.signs(0)]
    want = brute.attend(q[0, 3], [k[0, 1, t] for t in range(n_cached + 1)],
                        [v[0, 1, t] for t in range(n_cached + 1)], scale, s)
    assert np.allclose(pre[0, 3], want, rtol=0, atol=1e-13)

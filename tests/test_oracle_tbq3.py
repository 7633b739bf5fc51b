"""Pins for the oracle's 3-bit variant (TBQ3), on the CPU.

The page names TBQ3 next to TBQ4 without a layout (trefon.com, "Kontekst 262K
na jednej RTX 4090: co dodalem do llama.cpp-turboq", section "6. Ten sam
cache na Apple silicon"); the layout is this library's: 50 bytes per 128
values, the fp16 scale then 16 little-endian 24-bit words of eight 3-bit
indices, levels S*(2i-7)/7.  Each pin checks the C oracle against something
other than itself: closed forms, the exact nearest level in rational
arithmetic, a bit-stream unpacker written independently in pure Python,
invariants and the quantiser's error bound, and brute-force attention.
"""
import math

import numpy as np

import oracle
from oracle import brute

D = 128
RNG = np.random.default_rng(20261202)


def _unpack(blk):
    """Indices of a 3-bit block with numpy (24-bit words), and its scale bits."""
    w = (blk[2::3].astype(np.uint32) | (blk[3::3].astype(np.uint32) << 8)
         | (blk[4::3].astype(np.uint32) << 16))
    idx = np.stack([(w >> (3 * k)) & 7 for k in range(8)], axis=1).reshape(-1)
    return int(blk[0]) | (int(blk[1]) << 8), idx.astype(np.int64)


def test_block_size_closed_form():
    # 2 scale bytes + 128 values x 3 bits / 8 = 50 bytes (3.125 bits per value)
    assert oracle.block_bytes3() == oracle.BLOCK_BYTES3 == 2 + D * 3 // 8 == 50


def test_packing_of_a_known_pattern():
    # indices 0..7 repeated: every 24-bit word is sum_k k << 3k = 0xFAC688
    s = oracle.signs(0)
    R = oracle.rotation_matrix(s)
    S = np.float16(7.0)
    idx = np.tile(np.arange(8), 16)
    x = (R.T @ (float(S) * (2 * idx - 7) / 7.0)).astype(np.float32)
    blk = oracle.quantize_block3(x, s)
    w = sum(k << (3 * k) for k in range(8))
    assert w == 0xFAC688
    assert list(blk[:2]) == [int(S.view(np.uint16)) & 0xFF, int(S.view(np.uint16)) >> 8]
    assert list(blk[2:5]) == [0x88, 0xC6, 0xFA] and np.array_equal(blk[2:], np.tile(blk[2:5], 16))
    assert brute.unpack3(blk) == idx.tolist()


def test_level_index3_is_nearest_level():
    n = 0
    for _ in range(4000):
        S = float(np.float16(RNG.uniform(1e-3, 100)))
        x = float(np.float32(RNG.uniform(-1.2, 1.2) * S))
        frac = (x / S * 3.5 + 3.5) % 1.0
        if abs(frac - 0.5) < 1e-4:
            continue
        assert oracle.level_index3(x, S) == brute.nearest_level_index3(x, S)
        n += 1
    assert n > 3900


def test_level_index3_ties_zero_scale_and_clamp():
    # exact ties in binary32 go to the even index
    checked = 0
    for S in [3.5, 7.0, 1.75, 0.4375]:
        for j in range(-6, 7):
            x = np.float32(j * S / 3.5)
            u = (np.float32(x) / np.float32(S)) * np.float32(3.5)
            if u != np.float32(round(float(u))):
                continue
            v = float(u) + 3.5
            lo = math.floor(v)
            want = min(max(lo if lo % 2 == 0 else lo + 1, 0), 7)
            assert oracle.level_index3(float(x), S) == want
            checked += 1
    assert checked >= 20
    assert oracle.level_index3(0.0, 0.0) == 4
    assert oracle.level_index3(0.0, 1.0) == 4          # 3.5 ties to 4
    assert oracle.level_index3(1.2, 1.0) == 7
    assert oracle.level_index3(-1.2, 1.0) == 0


def test_on_grid_round_trip_and_layout():
    s = oracle.signs(0)
    R = oracle.rotation_matrix(s)
    for _ in range(200):
        S = np.float16(RNG.uniform(0.05, 50))
        idx = RNG.integers(0, 8, D)
        idx[RNG.integers(0, D)] = RNG.choice([0, 7])   # a +-S level is present
        x = (R.T @ (float(S) * (2 * idx - 7) / 7.0)).astype(np.float32)
        blk = oracle.quantize_block3(x, s)
        sb, got = _unpack(blk)
        assert sb == int(S.view(np.uint16))
        assert np.array_equal(got, idx)
        assert brute.unpack3(blk) == idx.tolist()


def test_quantiser_invariants_and_error_bound():
    s = oracle.signs(3)
    R = oracle.rotation_matrix(s)
    for k in range(300):
        gain = [1e-3, 1.0, 10.0, 300.0][k % 4]
        x = (RNG.standard_t(4, D) * gain).astype(np.float32)
        blk = oracle.quantize_block3(x, s)
        sb, idx = _unpack(blk)
        S = float(np.uint16(sb).view(np.float16))
        assert S > 0
        assert (idx == 0).any() or (idx == 7).any()      # the max element sits on an end level
        exact = R @ x.astype(np.float64)
        xhat = oracle.dequant_block3(blk)
        m = np.abs(exact).max()
        assert np.all(np.abs(xhat - exact) <= S / 7 + abs(m - S) + 1e-5 * m)
        # same rotation and scale as TBQ4: the scale bytes agree
        assert np.array_equal(blk[:2], oracle.quantize_block(x, s)[:2])


def test_zero_block():
    blk = oracle.quantize_block3(np.zeros(D, np.float32), oracle.signs(0))
    # scale 0 and every index 4: words 0x924924
    assert blk[0] == 0 and blk[1] == 0 and np.array_equal(blk[2:], np.tile([0x24, 0x49, 0x92], 16))
    assert np.all(oracle.dequant_block3(blk) == 0.0)


def test_dequant3_matches_brute():
    s = oracle.signs(0)
    for _ in range(20):
        blk = oracle.quantize_block3(RNG.standard_normal(D).astype(np.float32) * 3, s)
        assert np.array_equal(oracle.dequant_block3(blk), np.array(brute.dequant3(blk)))


def test_quantize_append3_places_blocks():
    B, n_new, Hkv, cap = 2, 3, 2, 16
    seed = 5
    s = oracle.signs(seed)
    src = RNG.standard_normal((B, n_new, Hkv, D)).astype(np.float32)
    cache = np.full((B, Hkv, cap, 50), 0xAB, np.uint8)
    start = np.array([5, 14], np.int32)
    assert oracle.quantize_append3(src, start, cap, seed, cache) == Hkv * 1   # b=1, t=2 -> 16
    for b in range(B):
        for t in range(n_new):
            p = start[b] + t
            for h in range(Hkv):
                if p < cap:
                    assert np.array_equal(cache[b, h, p], oracle.quantize_block3(src[b, t, h], s))
    untouched = np.ones((B, Hkv, cap), bool)
    untouched[0, :, 5:8] = False
    untouched[1, :, 14:16] = False
    assert np.all(cache[untouched] == 0xAB)


def test_decode3_matches_pure_python_brute_force():
    seed = 9
    s = oracle.signs(seed)
    B, Hq, Hkv, L = 1, 2, 1, 4
    q = RNG.standard_normal((B, Hq, D)).astype(np.float32)
    k = (RNG.standard_normal((B, L, Hkv, D)) * 2).astype(np.float32)
    v = RNG.standard_normal((B, L, Hkv, D)).astype(np.float32)
    kc = np.zeros((B, Hkv, 8, 50), np.uint8)
    vc = np.zeros_like(kc)
    oracle.quantize_append3(k, np.zeros(B, np.int32), 8, seed, kc)
    oracle.quantize_append3(v, np.zeros(B, np.int32), 8, seed, vc)
    got = oracle.attn_decode3(q, kc, vc, np.array([L], np.int32), 0.125, seed)
    for h in range(Hq):
        want = brute.attend(q[0, h], [kc[0, 0, t] for t in range(L)],
                            [vc[0, 0, t] for t in range(L)], 0.125, s, deq=brute.dequant3)
        assert np.abs(got[0, h] - np.array(want)).max() <= 1e-13


def test_decode3_closed_form_equal_keys():
    # every key identical -> the output is the mean of the dequantised values
    seed = 2
    s = oracle.signs(seed)
    R = oracle.rotation_matrix(s)
    L = 7
    kv = np.repeat(RNG.standard_normal((1, 1, 1, D)).astype(np.float32), L, axis=1)
    v = RNG.standard_normal((1, L, 1, D)).astype(np.float32)
    kc = np.zeros((1, 1, 8, 50), np.uint8)
    vc = np.zeros_like(kc)
    oracle.quantize_append3(kv, np.zeros(1, np.int32), 8, seed, kc)
    oracle.quantize_append3(v, np.zeros(1, np.int32), 8, seed, vc)
    q = RNG.standard_normal((1, 3, D)).astype(np.float32)
    got = oracle.attn_decode3(q, kc, vc, np.array([L], np.int32), 0.09, seed)
    mean_rot = np.mean([oracle.dequant_block3(vc[0, 0, t]) for t in range(L)], axis=0)
    want = R.T @ mean_rot
    for h in range(3):
        assert np.abs(got[0, h] - want).max() <= 1e-12

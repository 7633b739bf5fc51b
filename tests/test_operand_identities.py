"""The attention kernels feed the tensor cores operands built straight from the
raw cache bytes, relying on identities that are exact by construction.  These
CPU tests restate each construction with numpy (integers, and fp16 arithmetic
emulated exactly through float64 with one final fp16 rounding) and check it
against the plain definition, on every value it can take or on random data:

- 4-bit K: the raw nibble byte (lo + 16 hi) and its low nibble, weighed by
  u = q_odd and w = 16 q_even - q_odd, sum to 16 sum_d n_d q_d; the weights
  split into three signed bytes recombine exactly.
- 3-bit K: a 24-bit group spread to four bytes i_even + 8 i_odd by two
  shift-and-mask steps; weights u = q_odd and w = 8 q_even - q_odd give
  8 sum_d i_d q_d.
- 4-bit V: a nibble masked into an fp16 half (a subnormal) and one fused
  multiply-add give the level (2n - 15) 2^-11 with no rounding.
- 3-bit V: three byte permutations of two tokens' groups put every field
  inside an fp16 mantissa; the same one-FMA step gives (2i - 7) 2^-11.
- Quantiser: x / S by RN(1/S), RN(x r), the exact residual and one FMA is
  the correctly rounded quotient for every normal fp16 scale; adding
  1.5 2^23 rounds u to the nearest integer, ties to even.

The kernels' constants are restated here; the tests need no GPU and do not
use the oracle.
"""
import numpy as np

RNG = np.random.default_rng(20261202)


def split3(x):
    """x = c0 + 256 c1 + 65536 c2 with c0, c1 in [-128, 127] (the kernels'
    signed-byte pieces of an 18-bit weight)."""
    x = np.asarray(x, np.int64)
    c0 = ((x + 128) & 255) - 128
    x1 = (x - c0) >> 8
    c1 = ((x1 + 128) & 255) - 128
    c2 = (x1 - c1) >> 8
    return c0, c1, c2


def test_split3_recombines_and_fits_signed_bytes():
    x = np.concatenate([RNG.integers(-17 * 2**18, 17 * 2**18, 200000),
                        [0, 1, -1, 127, 128, -128, -129, 2**22 - 1, -2**22]])
    c0, c1, c2 = split3(x)
    assert np.array_equal(c0 + 256 * c1 + 65536 * c2, x)
    for c in (c0, c1, c2):
        assert c.min() >= -128 and c.max() <= 127


def _k4_operands(n):
    """Raw bytes and their low nibbles of one 128-value row of nibbles."""
    lo, hi = n[..., 0::2], n[..., 1::2]
    return lo + 16 * hi, lo


def test_k4_raw_and_low_nibble_weights_give_16_sum_nq():
    for _ in range(200):
        n = RNG.integers(0, 16, 128)
        q = RNG.integers(-2**18, 2**18 + 1, 128)
        raw, low = _k4_operands(n)
        u, w = q[1::2], 16 * q[0::2] - q[1::2]
        # the MMA sums each signed-byte piece separately (u8 x s8, int32)
        total = 0
        for pu, pw, scale in zip(split3(u), split3(w), (1, 256, 65536)):
            plane = int(np.dot(raw, pu) + np.dot(low, pw))
            assert abs(plane) < 2**31                 # one int32 accumulator
            total += scale * plane
        assert total == 16 * int(np.dot(n, q))


def _tbq3_group_bits(i8):
    """Eight 3-bit indices -> the 24-bit group word (index k at bits 3k)."""
    return sum(int(v) << (3 * k) for k, v in enumerate(i8))


def _tbq3_pairs(g):
    """The kernels' two shift-and-mask steps on a 24-bit group."""
    t = (g & 0x00000FFF) | ((g & 0x00FFF000) << 4)
    return (t & 0x003F003F) | ((t & 0x0FC00FC0) << 2)


def test_tbq3_pair_bytes_hold_i_even_plus_8_i_odd():
    for _ in range(2000):
        i8 = RNG.integers(0, 8, 8)
        word = _tbq3_pairs(_tbq3_group_bits(i8))
        for j in range(4):
            assert (word >> (8 * j)) & 0xFF == i8[2 * j] + 8 * i8[2 * j + 1]


def test_k3_pair_byte_weights_give_8_sum_iq():
    for _ in range(200):
        i = RNG.integers(0, 8, 128)
        q = RNG.integers(-2**18, 2**18 + 1, 128)
        pair = i[0::2] + 8 * i[1::2]
        low = pair & 7
        assert np.array_equal(low, i[0::2])
        u, w = q[1::2], 8 * q[0::2] - q[1::2]
        total = 0
        for pu, pw, scale in zip(split3(u), split3(w), (1, 256, 65536)):
            total += scale * int(np.dot(pair, pu) + np.dot(low, pw))
        assert total == 8 * int(np.dot(i, q))
        # the level map: sum q (2i - 7) = 2 sum iq - 7 sum q
        assert 2 * total // 8 - 7 * int(q.sum()) == int(np.dot(2 * i - 7, q))


def _h(bits):
    """fp16 value of 16-bit patterns."""
    return np.asarray(bits, np.uint16).view(np.float16).astype(np.float64)


def _hfma(x_bits, a_bits, b_bits):
    """fp16 fused multiply-add, one rounding: the product of two fp16 values
    is exact in float64 and so is the sum here, so float64 then one fp16
    rounding is the correctly rounded result."""
    return (_h(x_bits) * _h(a_bits) + _h(b_bits)).astype(np.float16).astype(np.float64)


def test_v4_level_from_masked_nibble_is_exact():
    n = np.arange(16)
    want = (2 * n - 15) * 2.0**-11
    # low nibble (bits 0-3): x = n 2^-24, x 2^14 - 15 2^-11
    assert np.array_equal(_hfma(n, 0x7400, 0x9F80), want)
    # high nibble (bits 4-7): x = 16 n 2^-24, x 2^10 - 15 2^-11
    assert np.array_equal(_hfma(n << 4, 0x6400, 0x9F80), want)
    # the constants: 2^14, 2^10, -15 2^-11
    assert _h(0x7400) == 2.0**14 and _h(0x6400) == 2.0**10 and _h(0x9F80) == -15 * 2.0**-11


def _byte_perm(a, b, sel):
    """PRMT: bytes of {b, a} (a bytes 0-3, b bytes 4-7) picked by the four
    selector nibbles."""
    pool = [(a >> (8 * k)) & 0xFF for k in range(4)] + [(b >> (8 * k)) & 0xFF for k in range(4)]
    return sum(pool[(sel >> (4 * k)) & 7] << (8 * k) for k in range(4))


def test_v3_level_from_packed_fields_is_exact():
    sel = [0x5410, 0x5410, 0x5410, 0x6521, 0x6521, 0x6521, 0x7632, 0x7632]
    bit = [0, 3, 6, 1, 4, 7, 2, 5]
    assert _h(0x9B00) == -7 * 2.0**-11
    for _ in range(500):
        ia, ib = RNG.integers(0, 8, 8), RNG.integers(0, 8, 8)
        A, B = _tbq3_group_bits(ia), _tbq3_group_bits(ib)
        for f in range(8):
            mask = 0x00070007 << bit[f]
            mul = (15 + 14 - bit[f]) << 10               # fp16 2^(14 - b)
            word = _byte_perm(A, B, sel[f]) & mask
            lo, hi = word & 0xFFFF, word >> 16
            assert _hfma(lo, mul, 0x9B00) == (2 * ia[f] - 7) * 2.0**-11
            assert _hfma(hi, mul, 0x9B00) == (2 * ib[f] - 7) * 2.0**-11


def _fma32(a, b, c):
    """float32 fused multiply-add, emulated: a*b is exact in float64 (two
    24-bit significands); the sum is rounded to float64 and then to float32,
    which differs from one rounding only when the float64 sum lands exactly
    on a float32 rounding midpoint (the residual step below, x - q0 S, is
    exact in float64, so only the last step could be affected, and a
    difference would fail the comparison rather than hide one)."""
    return (a.astype(np.float64) * b.astype(np.float64) + c.astype(np.float64)).astype(np.float32)


def test_quantizer_division_is_the_correctly_rounded_quotient():
    # every positive normal fp16 scale, against values inside [-S, S] (the
    # encoder clamps to that range where the scale is not within 2^-11 of max|x|)
    s_bits = np.arange(0x0400, 0x7C00, dtype=np.uint16)
    S = s_bits.view(np.float16).astype(np.float32)
    S = np.repeat(S, 64)
    x = (RNG.uniform(-1.0, 1.0, S.size).astype(np.float32) * S).astype(np.float32)
    x[::17] = S[::17]
    x[1::17] = -S[1::17]
    r = (np.float32(1.0) / S).astype(np.float32)            # RN(1/S)
    q0 = (x * r).astype(np.float32)                         # RN(x r)
    e = _fma32(-q0, S, x)                                   # x - q0 S, exact
    q = _fma32(e, r, q0)                                    # RN(q0 + e r)
    want = (x / S).astype(np.float32)                       # IEEE x / S
    # a subnormal quotient cannot change an index (|x/S| << 1/15 there)
    normal = np.abs(want) >= np.float32(2.0**-126)
    assert np.array_equal(q[normal], want[normal])


def test_rint_by_adding_1_5_times_2_23_is_round_half_even():
    for L in (7.5, 3.5):                                     # 4-bit and 3-bit codebooks
        top = 2 * L
        u = np.concatenate([np.linspace(-0.004, top + 0.004, 200001),
                            np.arange(0, int(top) + 1) + 0.5,  # exact ties
                            np.arange(0, int(top) + 1) - 0.5]).astype(np.float32)
        u = u[(u >= -0.004) & (u <= top + 0.004)]
        got = ((u + np.float32(12582912.0)).astype(np.float32).view(np.uint32) &
               np.uint32(0xF if L == 7.5 else 0x7))
        want = np.rint(u.astype(np.float64)).astype(np.int64)   # numpy rint: half to even
        assert np.array_equal(got.astype(np.int64), np.clip(want, 0, int(top)))

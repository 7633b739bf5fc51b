"""Pure-Python brute force for tiny inputs -- TEST INFRASTRUCTURE.

Written straight from the definitions, with no numpy and no shared code with
``tbq4_oracle.c``, so that it can pin the C oracle:

* nearest_level_index: argmin over the 16 levels S*(2i-15)/15 in exact
  rational arithmetic (ties to the even index);
* dequant: unpack a 66-byte block (scale bytes first, even element in the
  low nibble) into S*(2i-15)/15;
* nearest_level_index3, unpack3, dequant3: the same for the 3-bit variant
  (8 levels S*(2i-7)/7; a 50-byte block read as a little-endian bit stream);
* attention: softmax(scale * q_rot . k) v with math.fsum, in the rotated
  domain, then rotated back with the explicit Hadamard entries;
* rotate_f32_stages: the binary32 rotation as whole-vector numpy stages (the
  one function here that uses numpy), which pins the butterfly order of the
  C oracle bit for bit.
"""
import math
from fractions import Fraction


def hadamard(i: int, j: int) -> int:
    return -1 if bin(i & j).count("1") % 2 else 1


def nearest_level_index(x_rot: float, S: float) -> int:
    if S == 0:
        return 8
    x = Fraction(x_rot)
    s = Fraction(S)
    best, best_d = None, None
    for i in range(16):
        d = abs(x - s * (2 * i - 15) / 15)
        if best_d is None or d < best_d or (d == best_d and i % 2 == 0):
            best, best_d = i, d
    return best


def nearest_level_index3(x_rot: float, S: float) -> int:
    """The 3-bit codebook: argmin over the 8 levels S*(2i-7)/7, ties to the
    even index; index 4 when S == 0."""
    if S == 0:
        return 4
    x = Fraction(x_rot)
    s = Fraction(S)
    best, best_d = None, None
    for i in range(8):
        d = abs(x - s * (2 * i - 7) / 7)
        if best_d is None or d < best_d or (d == best_d and i % 2 == 0):
            best, best_d = i, d
    return best


def f16_bits_to_float(h: int) -> float:
    sign = -1.0 if (h >> 15) & 1 else 1.0
    e = (h >> 10) & 0x1F
    m = h & 0x3FF
    if e == 0:
        return sign * m * 2.0 ** -24
    if e == 31:
        return sign * (math.inf if m == 0 else math.nan)
    return sign * (1024 + m) * 2.0 ** (e - 25)


def dequant(block) -> list:
    block = [int(b) for b in block]
    S = f16_bits_to_float(block[0] | (block[1] << 8))
    out = []
    for j in range(64):
        b = block[2 + j]
        out.append(S * (2 * (b & 15) - 15) / 15)
        out.append(S * (2 * (b >> 4) - 15) / 15)
    return out


def unpack3(block) -> list:
    """The 128 indices of a 50-byte 3-bit block, read one bit at a time from
    the byte string (bit 3i+b of the little-endian stream after the scale is
    bit b of index i)."""
    block = [int(b) for b in block]
    bits = []
    for byte in block[2:]:
        bits.extend((byte >> k) & 1 for k in range(8))
    return [bits[3 * i] | (bits[3 * i + 1] << 1) | (bits[3 * i + 2] << 2) for i in range(128)]


def dequant3(block) -> list:
    S = f16_bits_to_float(int(block[0]) | (int(block[1]) << 8))
    return [S * (2 * i - 7) / 7 for i in unpack3(block)]


def rotate(x, s) -> list:
    """R x with R[i][j] = H[i][j] s_j / sqrt(128)."""
    n = len(x)
    r = 1.0 / math.sqrt(n)
    return [math.fsum(hadamard(i, j) * s[j] * x[j] for j in range(n)) * r
            for i in range(n)]


def unrotate(y, s) -> list:
    """R^T y."""
    n = len(y)
    r = 1.0 / math.sqrt(n)
    return [math.fsum(hadamard(i, j) * s[j] * y[i] for i in range(n)) * r
            for j in range(n)]


def attend(q, k_blocks, v_blocks, scale, s, deq=dequant) -> list:
    """One query row over a handful of keys (blocks given as byte lists;
    deq = dequant3 for 3-bit blocks)."""
    q_rot = rotate([float(v) for v in q], s)
    ks = [deq(b) for b in k_blocks]
    vs = [deq(b) for b in v_blocks]
    logits = [scale * math.fsum(a * b for a, b in zip(q_rot, k)) for k in ks]
    m = max(logits)
    p = [math.exp(z - m) for z in logits]
    l = math.fsum(p)
    o_rot = [math.fsum(p[t] * vs[t][i] for t in range(len(vs))) / l
             for i in range(len(q_rot))]
    return unrotate(o_rot, s)


def rotate_f32_stages(x, s):
    """The binary32 rotation of the codebook, stage by stage on whole numpy
    float32 vectors: z = s * x; for stride h = 1, 2, 4, ..., 64 split z into
    blocks of 2h, the first half a and the second half b of each block
    becoming a + b and a - b (numpy rounds each add and subtract to binary32
    and never contracts them); finally one binary32 multiply by
    fl32(1/sqrt(128)) = 0x3DB504F3.  Any other stride order or association
    rounds differently on general inputs, so equality with the C oracle on
    random vectors fixes its order."""
    import numpy as np
    z = np.asarray(x, np.float32) * np.asarray(s, np.float32)
    n = z.shape[-1]
    h = 1
    while h < n:
        blk = z.reshape(n // (2 * h), 2, h)
        a, b = blk[:, 0, :], blk[:, 1, :]
        z = np.stack([a + b, a - b], axis=1).reshape(n)
        h *= 2
    return z * np.array(0x3DB504F3, np.uint32).view(np.float32)

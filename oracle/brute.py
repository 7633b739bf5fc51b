"""Pure-Python brute force for tiny inputs -- TEST INFRASTRUCTURE.

Written straight from the definitions, with no numpy and no shared code with
``tbq4_oracle.c``, so that it can pin the C oracle:

* nearest_level_index: argmin over the 16 levels S*(2i-15)/15 in exact
  rational arithmetic (ties to the even index);
* dequant: unpack a 66-byte block (scale bytes first, even element in the
  low nibble) into S*(2i-15)/15;
* attention: softmax(scale * q_rot . k) v with math.fsum, in the rotated
  domain, then rotated back with the explicit Hadamard entries.
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


def attend(q, k_blocks, v_blocks, scale, s) -> list:
    """One query row over a handful of keys (blocks given as byte lists)."""
    q_rot = rotate([float(v) for v in q], s)
    ks = [dequant(b) for b in k_blocks]
    vs = [dequant(b) for b in v_blocks]
    logits = [scale * math.fsum(a * b for a, b in zip(q_rot, k)) for k in ks]
    m = max(logits)
    p = [math.exp(z - m) for z in logits]
    l = math.fsum(p)
    o_rot = [math.fsum(p[t] * vs[t][i] for t in range(len(vs))) / l
             for i in range(len(q_rot))]
    return unrotate(o_rot, s)

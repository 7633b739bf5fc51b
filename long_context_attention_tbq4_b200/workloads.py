"""Seeded synthetic inputs for the TBQ4 attention workloads.

This module only draws random numbers: it holds none of the method's
arithmetic, so both the CUDA path and the oracle may take their inputs from
it.  Every draw uses ``numpy.random.default_rng(seed)`` in a fixed order; the
recipe for each workload is in its docstring.

The page that defines TBQ4 measures on a 262,144-token context (trefon.com,
"Kontekst 262K na jednej RTX 4090", section "Konfiguracja"); the shapes
below (24 query heads / 4 KV heads, head_dim 128, 32K/262K decode, a 512-token
prefill chunk over 131,072 cached tokens, a ragged batch of 8) are the
library's own synthetic stand-ins for that serving load.
"""
from dataclasses import dataclass, field

import numpy as np

D = 128
SIGN_SEED = 0          # seed of the +-1 diagonal for every workload


@dataclass
class DecodeCase:
    name: str
    q: np.ndarray                 # [B][Hq][128] fp32
    k: list                       # per sequence: [L_b][Hkv][128] fp32
    v: list
    seq_lens: np.ndarray          # [B] int32
    Hq: int
    Hkv: int
    softmax_scale: float = 1.0 / np.sqrt(D)
    sign_seed: int = SIGN_SEED
    meta: dict = field(default_factory=dict)

    @property
    def B(self):
        return len(self.seq_lens)


@dataclass
class PrefillCase:
    name: str
    q_bf16: np.ndarray            # [n_new][Hq][128] uint16 (bf16 bits)
    q: np.ndarray                 # the same values as fp32 (exact upcast)
    k: np.ndarray                 # [n_cached + n_new][Hkv][128] fp32
    v: np.ndarray
    n_cached: int
    n_new: int
    Hq: int
    Hkv: int
    softmax_scale: float = 1.0 / np.sqrt(D)
    sign_seed: int = SIGN_SEED


def bf16_round(x: np.ndarray):
    """fp32 -> bf16 (round to nearest even): returns (bits uint16, fp32)."""
    u = np.ascontiguousarray(x, np.float32).view(np.uint32).astype(np.uint64)
    r = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    bits = r.astype(np.uint16)
    f = (bits.astype(np.uint32) << 16).view(np.float32)
    return bits, f


def normal(rng, shape):
    return rng.standard_normal(shape, dtype=np.float32)


def decode_case(name, seed, B, Hq, Hkv, lens, dist="normal", k_outliers=0,
                outlier_gain=10.0):
    """Decode inputs.  Draw order: q, then K for every sequence, then V for
    every sequence, then (if k_outliers) per KV head ``k_outliers`` channel
    indices without replacement; those K channels are multiplied by
    ``outlier_gain`` for every token.  dist 'normal' = N(0,1) fp32; 't4' =
    Student-t with 4 degrees of freedom for K and V (q stays N(0,1))."""
    rng = np.random.default_rng(seed)
    lens = np.asarray(lens, np.int32)
    assert len(lens) == B
    q = normal(rng, (B, Hq, D))

    def draw(L):
        if dist == "normal":
            return normal(rng, (int(L), Hkv, D))
        if dist == "t4":
            return rng.standard_t(4, (int(L), Hkv, D)).astype(np.float32)
        raise ValueError(dist)

    k = [draw(L) for L in lens]
    v = [draw(L) for L in lens]
    meta = {}
    if k_outliers:
        ch = np.stack([rng.choice(D, k_outliers, replace=False)
                       for _ in range(Hkv)])
        meta["outlier_channels"] = ch
        for kb in k:
            for h in range(Hkv):
                kb[:, h, ch[h]] *= np.float32(outlier_gain)
    return DecodeCase(name, q, k, v, lens, Hq, Hkv, meta=meta)


def tiny_decode():
    """1 sequence, 4 query heads sharing 1 KV head, 1,024 cached tokens,
    N(0,1) from seed 0."""
    return decode_case("tiny_decode_1k", 0, 1, 4, 1, [1024])


def decode_32k():
    """1 sequence, 24/4 heads, 32,768 cached tokens, N(0,1) from seed 1."""
    return decode_case("decode_32k", 1, 1, 24, 4, [32768])


def decode_262k():
    """1 sequence, 24/4 heads, 262,144 cached tokens, seed 2; K with 4 outlier
    channels per KV head scaled x10, V N(0,1)."""
    return decode_case("decode_262k", 2, 1, 24, 4, [262144], k_outliers=4)


def ragged_lengths(seed=4, B=8, lo=16384, hi=98304):
    rng = np.random.default_rng(seed)
    return rng.integers(lo, hi, size=B, endpoint=True).astype(np.int32), rng


def ragged_decode():
    """8 sequences, lengths uniform in [16,384, 98,304] drawn first from seed
    4, then q N(0,1), then Student-t (nu=4) K and V."""
    lens, rng = ragged_lengths()
    B, Hq, Hkv = 8, 24, 4
    q = normal(rng, (B, Hq, D))
    k = [rng.standard_t(4, (int(L), Hkv, D)).astype(np.float32) for L in lens]
    v = [rng.standard_t(4, (int(L), Hkv, D)).astype(np.float32) for L in lens]
    return DecodeCase("ragged_decode_8", q, k, v, lens, Hq, Hkv)


def mq_case(name, seed, B, q_len, Hq, Hkv, lens, dist="normal"):
    """Multi-query decode inputs (q_len new tokens per sequence, already in
    the caches).  Draw order: q N(0,1) fp32 [B][q_len][Hq][128], then K for
    every sequence, then V for every sequence ([L_b][Hkv][128], N(0,1) or
    Student-t nu=4)."""
    rng = np.random.default_rng(seed)
    lens = np.asarray(lens, np.int32)
    q = normal(rng, (B, q_len, Hq, D))

    def draw(L):
        if dist == "normal":
            return normal(rng, (int(L), Hkv, D))
        return rng.standard_t(4, (int(L), Hkv, D)).astype(np.float32)

    k = [draw(L) for L in lens]
    v = [draw(L) for L in lens]
    return DecodeCase(name, q, k, v, lens, Hq, Hkv)


def mq_262k():
    """4 new tokens over a 262,144-token context (the last 4 included), 24/4
    heads, N(0,1), seed 5: the speculative verification step of the decode."""
    return mq_case("mq4_262k", 5, 1, 4, 24, 4, [262144])


def prefill_case(name, seed, n_cached, n_new, Hq=24, Hkv=4):
    """Chunked prefill inputs.  Draw order: q fp32 N(0,1) [n_new][Hq][128]
    rounded to bf16; K [n_cached + n_new][Hkv][128]; V likewise (all N(0,1)
    fp32).  The first n_cached rows of K/V are the cached context, the last
    n_new rows the chunk that is quantise-appended before attention."""
    rng = np.random.default_rng(seed)
    qf = normal(rng, (n_new, Hq, D))
    q_bits, q = bf16_round(qf)
    k = normal(rng, (n_cached + n_new, Hkv, D))
    v = normal(rng, (n_cached + n_new, Hkv, D))
    return PrefillCase(name, q_bits, q, k, v, n_cached, n_new, Hq, Hkv)


def prefill_131k():
    """512 new tokens over 131,072 cached tokens, 24/4 heads, seed 3."""
    return prefill_case("prefill_512_at_131k", 3, 131072, 512)


def round_capacity(n, multiple=4096):
    """KV capacity rounded up to a multiple (default 4096, the padding
    minimum the page uses for fewer CUDA-graph recaptures: trefon.com,
    "Kontekst 262K na jednej RTX 4090", section 2)."""
    return ((int(n) + multiple - 1) // multiple) * multiple


def page_table(seed, lens, page_size, spare=3, max_pages=None):
    """A block table for paged caches: every sequence gets the pages its
    length needs, drawn without replacement from a shuffled pool that has
    `spare` unused pages; a row's unused tail is filled with -1.  Returns
    (table int32 [B][max_pages], n_pages)."""
    need = [(int(n) + page_size - 1) // page_size for n in lens]
    width = max(max(need, default=0), 1) if max_pages is None else int(max_pages)
    n_pages = sum(need) + spare
    perm = np.random.default_rng(seed).permutation(n_pages).astype(np.int32)
    table = np.full((len(lens), width), -1, np.int32)
    at = 0
    for b, k in enumerate(need):
        table[b, :k] = perm[at:at + k]
        at += k
    return table, n_pages

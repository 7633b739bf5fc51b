"""The C-ABI library loads, exports every symbol include/tbq4.h declares, and
rejects bad arguments on the host before any launch (no GPU needed)."""
import ctypes as C
import os
import re
import subprocess

import numpy as np
import pytest

import oracle

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "tbq4.h")


@pytest.fixture(scope="module")
def T():
    import long_context_attention_tbq4_b200 as pkg
    return pkg


def declared_symbols():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"TBQ4_API[^;(]*?\b(tbq[34]_\w+)\s*\(", text)))


def test_header_declares_the_boundary():
    names = declared_symbols()
    for n in ["tbq4_quantize_append", "tbq4_attn_decode", "tbq4_attn_prefill_chunk"]:
        assert n in names


def test_library_exports_every_declared_symbol(T):
    out = subprocess.run(["nm", "-D", "--defined-only", T.LIB_PATH], check=True,
                         capture_output=True, text=True).stdout
    exported = set(re.findall(r"\bT (tbq[34]_\w+)", out))
    from long_context_attention_tbq4_b200 import _lib
    for n in declared_symbols():
        assert n in exported, n
        assert n in _lib.SIGNATURES, n
        assert getattr(_lib.lib, n) is not None


def test_debug_library_exports_every_declared_symbol():
    # built here if missing (a few seconds of nvcc); no compute call
    import importlib.util
    spec = importlib.util.spec_from_file_location(
        "tbq4_build", os.path.join(ROOT, "long_context_attention_tbq4_b200", "build.py"))
    build = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(build)
    path = build.build(debug=True)
    assert path.endswith("libtbq4_debug.so")
    out = subprocess.run(["nm", "-D", "--defined-only", path], check=True,
                         capture_output=True, text=True).stdout
    exported = set(re.findall(r"\bT (tbq[34]_\w+)", out))
    for n in declared_symbols():
        assert n in exported, n
    lib = C.CDLL(path)
    lib.tbq4_status_string.restype = C.c_char_p
    assert b"debug" in lib.tbq4_status_string(8)


def test_block_and_cache_bytes(T):
    assert T.tbq4_block_bytes() == 66
    assert T.tbq4_cache_bytes(1, 4, 262144) == 262144 * 4 * 66
    assert T.tbq4_cache_bytes(0, 4, 8) == 0


def test_signs_agree_with_oracle(T):
    # two independent SplitMix64 implementations (library host code, oracle)
    for seed in [0, 1, 2, 1234567, 2**64 - 1]:
        assert np.array_equal(T.tbq4_signs(seed), oracle.signs(seed))


def test_workspace_queries(T):
    a = T.tbq4_decode_workspace_bytes(1, 24, 4, 262144)
    b = T.tbq4_decode_workspace_bytes(1, 24, 4, 32768)
    assert a > 0 and b > 0 and a % 256 == 0
    assert T.tbq4_decode_workspace_bytes(1, 24, 4, 262144, 32) > a
    assert T.tbq4_decode_workspace_bytes(0, 24, 4, 100) == 0
    assert T.tbq4_prefill_workspace_bytes(512, 24, 4, 131072) > 0


# Fake, suitably aligned device addresses: every call below must be rejected
# on the host before any launch, so nothing dereferences them.
A = C.c_void_p(0x10000)
A2 = C.c_void_p(0x20000)
MIS = C.c_void_p(0x10004)


def _dec(L, **kw):
    args = dict(q=A, k=A, v=A, lens=A, max_len=64, B=1, Hq=8, Hkv=2, cap=64,
                scale=0.1, seed=0, split=0, ws=A2, ws_bytes=1 << 30, out=A, stream=None)
    args.update(kw)
    return L.tbq4_attn_decode_split(args["q"], args["k"], args["v"], args["lens"],
                                    args["max_len"], args["B"], args["Hq"], args["Hkv"],
                                    args["cap"], args["scale"], args["seed"], args["split"],
                                    args["ws"], args["ws_bytes"], args["out"],
                                    args["stream"])


def test_decode_rejects_bad_arguments(T):
    from long_context_attention_tbq4_b200._lib import lib as L
    assert _dec(L, q=None) == 1                      # TBQ4_ERR_NULL
    assert _dec(L, ws=None) == 1
    assert _dec(L, q=MIS) == 2                       # TBQ4_ERR_ALIGN
    assert _dec(L, k=MIS) == 2
    assert _dec(L, ws=C.c_void_p(0x10010)) == 2      # workspace must be 256-B aligned
    assert _dec(L, Hq=7) == 3                        # TBQ4_ERR_SHAPE: Hq % Hkv
    assert _dec(L, Hq=18) == 3                       # group of 9 > 8
    assert _dec(L, split=48) == 3                    # split not a multiple of 32
    assert _dec(L, B=0) == 3
    assert _dec(L, cap=60) == 4                      # TBQ4_ERR_CAPACITY: cap % 8
    assert _dec(L, max_len=65) == 4                  # max_len > capacity
    assert _dec(L, ws_bytes=16) == 5                 # TBQ4_ERR_WORKSPACE


def test_quantize_rejects_bad_arguments(T):
    from long_context_attention_tbq4_b200._lib import lib as L

    def q(**kw):
        a = dict(src=A, B=1, n=4, Hkv=2, pos=A, cap=64, seed=0, cache=A, stream=None)
        a.update(kw)
        return L.tbq4_quantize_append(a["src"], a["B"], a["n"], a["Hkv"], a["pos"], a["cap"],
                                      a["seed"], a["cache"], a["stream"])
    assert q(src=None) == 1
    assert q(cache=None) == 1
    assert q(src=MIS) == 2
    assert q(cache=C.c_void_p(0x10002)) == 2
    assert q(Hkv=0) == 3
    assert q(cap=12) == 4
    assert q(n=0) == 0                               # nothing to do, nothing launched


def test_prefill_rejects_bad_arguments(T):
    from long_context_attention_tbq4_b200._lib import lib as L

    def p(**kw):
        a = dict(q=A, n=16, nc=100, k=A, v=A, Hq=8, Hkv=2, cap=128, scale=0.1, seed=0,
                 ws=A2, ws_bytes=1 << 30, out=A, stream=None)
        a.update(kw)
        return L.tbq4_attn_prefill_chunk(a["q"], a["n"], a["nc"], a["k"], a["v"], a["Hq"],
                                         a["Hkv"], a["cap"], a["scale"], a["seed"], a["ws"],
                                         a["ws_bytes"], a["out"], a["stream"])
    assert p(q=None) == 1
    assert p(k=MIS) == 2
    assert p(Hq=9) == 3
    assert p(n=0) == 3
    assert p(nc=120) == 4                            # n_cached + n_new > capacity
    assert p(ws_bytes=8) == 5


def test_selftest_rejects_bad_poll_counts(T):
    # refused on the host, before any launch
    from long_context_attention_tbq4_b200._lib import lib as L
    assert L.tbq4_selftest_bounded_wait(0, None) == 3
    assert L.tbq4_selftest_bounded_wait((1 << 16) + 1, None) == 3


def test_status_strings(T):
    from long_context_attention_tbq4_b200._lib import lib as L
    for code in range(9):
        assert len(L.tbq4_status_string(code)) > 0


def test_decode_append_rejects_bad_arguments(T):
    from long_context_attention_tbq4_b200._lib import lib as L

    def d(**kw):
        a = dict(q=A, kn=A, vn=A, k=A, v=A, lens=A, max_len=64, B=1, Hq=8, Hkv=2, cap=64,
                 scale=0.1, seed=0, ws=A2, ws_bytes=1 << 30, out=A, stream=None)
        a.update(kw)
        return L.tbq4_attn_decode_append(a["q"], a["kn"], a["vn"], a["k"], a["v"], a["lens"],
                                         a["max_len"], a["B"], a["Hq"], a["Hkv"], a["cap"],
                                         a["scale"], a["seed"], a["ws"], a["ws_bytes"],
                                         a["out"], a["stream"])
    assert d(kn=None) == 1
    assert d(vn=None) == 1
    assert d(q=None) == 1
    assert d(kn=C.c_void_p(0x10008)) == 2            # new rows must be 16-B aligned
    assert d(v=MIS) == 2
    assert d(Hq=7) == 3
    assert d(cap=60) == 4
    assert d(ws_bytes=16) == 5


def test_decode_mq_rejects_bad_arguments(T):
    from long_context_attention_tbq4_b200._lib import lib as L

    def d(**kw):
        a = dict(q=A, k=A, v=A, lens=A, max_len=64, B=1, ql=2, Hq=8, Hkv=2, cap=64, scale=0.1,
                 seed=0, ws=A2, ws_bytes=1 << 30, out=A, stream=None)
        a.update(kw)
        return L.tbq4_attn_decode_mq(a["q"], a["k"], a["v"], a["lens"], a["max_len"], a["B"],
                                     a["ql"], a["Hq"], a["Hkv"], a["cap"], a["scale"], a["seed"],
                                     a["ws"], a["ws_bytes"], a["out"], a["stream"])
    assert d(q=None) == 1
    assert d(q=MIS) == 2
    assert d(ql=0) == 3                               # q_len in [1, 4]
    assert d(ql=5) == 3
    assert d(cap=60) == 4
    assert d(ws_bytes=16) == 5


def test_decode_mq_workspace_query(T):
    assert T.tbq4_decode_mq_workspace_bytes(1, 4, 24, 4, 262144) > \
        T.tbq4_decode_workspace_bytes(1, 24, 4, 262144)
    assert T.tbq4_decode_mq_workspace_bytes(0, 4, 24, 4, 100) == 0


def test_paged_rejects_bad_arguments(T):
    from long_context_attention_tbq4_b200._lib import lib as L

    def d(**kw):
        a = dict(q=A, kn=None, vn=None, k=A, v=A, table=A, max_pages=4, page=32, n_pages=8,
                 lens=A, max_len=64, B=1, Hq=8, Hkv=2, scale=0.1, seed=0, ws=A2,
                 ws_bytes=1 << 30, out=A, stream=None)
        a.update(kw)
        return L.tbq4_attn_decode_paged(a["q"], a["kn"], a["vn"], a["k"], a["v"], a["table"],
                                        a["max_pages"], a["page"], a["n_pages"], a["lens"],
                                        a["max_len"], a["B"], a["Hq"], a["Hkv"], a["scale"],
                                        a["seed"], a["ws"], a["ws_bytes"], a["out"],
                                        a["stream"])
    assert d(table=None) == 1                         # TBQ4_ERR_NULL
    assert d(kn=A) == 1                               # one new row without the other
    assert d(k=None) == 1
    assert d(table=C.c_void_p(0x10002)) == 2          # TBQ4_ERR_ALIGN
    assert d(kn=C.c_void_p(0x10008), vn=A) == 2
    assert d(page=48) == 3                            # TBQ4_ERR_SHAPE: not a multiple of 32
    assert d(page=16) == 3
    assert d(max_pages=0) == 3
    assert d(n_pages=0) == 3
    assert d(Hq=7) == 3
    assert d(max_len=129) == 4                        # 4 pages of 32 reach 128 tokens
    assert d(ws_bytes=16) == 5                        # TBQ4_ERR_WORKSPACE

    def q(**kw):
        a = dict(src=A, B=1, n=4, Hkv=2, pos=A, table=A, max_pages=4, page=32, n_pages=8,
                 seed=0, pool=A, stream=None)
        a.update(kw)
        return L.tbq4_quantize_append_paged(a["src"], a["B"], a["n"], a["Hkv"], a["pos"],
                                            a["table"], a["max_pages"], a["page"],
                                            a["n_pages"], a["seed"], a["pool"], a["stream"])
    assert q(table=None) == 1
    assert q(pool=None) == 1
    assert q(table=C.c_void_p(0x10001)) == 2
    assert q(page=40) == 3
    assert q(n_pages=0) == 3
    assert q(n=0) == 0                                # nothing to do, nothing launched



def test_page_table_generator():
    """The seeded block tables the paged tests use: every page id at most
    once, rows as long as their sequence needs, -1 past that."""
    from long_context_attention_tbq4_b200 import workloads as W
    lens = [0, 1, 32, 33, 1000]
    table, n_pages = W.page_table(3, lens, 32, spare=2)
    assert table.shape == (5, 32) and n_pages == 0 + 1 + 1 + 2 + 32 + 2
    used = table[table >= 0]
    assert len(used) == len(set(used.tolist())) == n_pages - 2
    assert used.min() >= 0 and used.max() < n_pages
    for b, n in enumerate(lens):
        k = (n + 31) // 32
        assert (table[b, :k] >= 0).all() and (table[b, k:] == -1).all()
    assert np.array_equal(W.page_table(3, lens, 32, spare=2)[0], table)   # seeded


def test_tbq3_rejects_bad_arguments(T):
    from long_context_attention_tbq4_b200._lib import lib as L
    assert L.tbq3_block_bytes() == 50
    assert L.tbq3_cache_bytes(2, 4, 1024) == 2 * 4 * 1024 * 50
    assert L.tbq3_cache_bytes(0, 4, 1024) == 0

    def d(**kw):
        a = dict(q=A, k=A, v=A, lens=A, max_len=64, B=1, Hq=8, Hkv=2, cap=64, scale=0.1,
                 seed=0, ws=A2, ws_bytes=1 << 30, out=A, stream=None)
        a.update(kw)
        return L.tbq3_attn_decode(a["q"], a["k"], a["v"], a["lens"], a["max_len"], a["B"],
                                  a["Hq"], a["Hkv"], a["cap"], a["scale"], a["seed"], a["ws"],
                                  a["ws_bytes"], a["out"], a["stream"])
    assert d(q=None) == 1
    assert d(k=MIS) == 2
    assert d(Hq=7) == 3
    assert d(cap=60) == 4
    assert d(max_len=65) == 4
    assert d(ws_bytes=16) == 5

    def q(**kw):
        a = dict(src=A, B=1, n=4, Hkv=2, pos=A, cap=64, seed=0, cache=A, stream=None)
        a.update(kw)
        return L.tbq3_quantize_append(a["src"], a["B"], a["n"], a["Hkv"], a["pos"], a["cap"],
                                      a["seed"], a["cache"], a["stream"])
    assert q(src=None) == 1
    assert q(cache=C.c_void_p(0x10002)) == 2
    assert q(Hkv=0) == 3
    assert q(cap=12) == 4
    assert q(n=0) == 0

"""Runs every entry point of the library once on seeded inputs and saves the
results (cache bytes, outputs, the device status) to an .npz file.

Run as a script in a fresh process: ``python tests/debug_build_cases.py OUT.npz``.
With TBQ4_DEBUG=1 in the environment the package loads the debug build
(libtbq4_debug.so, every kernel's bounds checks switched on), otherwise the
release build; ``test_debug_build.py`` runs it both ways and compares.

The cases cover each kernel: the bulk and the per-row quantise-append, the
4-bit decode (automatic and forced splits), the fused decode step, the paged
append and decode, the 3-bit append and decode, the multi-query decode and
the chunked prefill.  Shapes are small but span several chunks, splits and
tiles, with ragged lengths.
"""
import os
import sys

import numpy as np


def run(path):
    import torch
    import long_context_attention_tbq4_b200 as T
    from long_context_attention_tbq4_b200 import _lib

    dev = torch.device("cuda")
    rng = np.random.default_rng(20261202)
    D, Hkv, Hq = 128, 4, 24
    scale = 1.0 / np.sqrt(D)
    res = {"debug": np.array(int(_lib.DEBUG)),
           "lib": np.array(os.path.basename(_lib.LIB_PATH))}

    def dev_t(x):
        return torch.from_numpy(np.ascontiguousarray(x)).to(dev)

    def half_bits(t):
        return t.cpu().contiguous().view(torch.int16).numpy()

    # contiguous caches: two sequences of 5000 and 3001 tokens, capacity 5120
    B, cap = 2, 5120
    lens = np.array([5000, 3001], np.int32)
    k = rng.standard_normal((B, 5000, Hkv, D)).astype(np.float32)
    v = rng.standard_normal((B, 5000, Hkv, D)).astype(np.float32)
    kc = T.empty_cache(B, Hkv, cap)
    vc = T.empty_cache(B, Hkv, cap)
    kc.zero_()
    vc.zero_()
    zero = dev_t(np.zeros(B, np.int32))
    T.tbq4_quantize_append(dev_t(k), zero, kc, 0)           # 40,000 rows: the bulk kernel
    T.tbq4_quantize_append(dev_t(v), zero, vc, 0)
    q = rng.standard_normal((B, Hq, D)).astype(np.float32)
    res["decode"] = half_bits(T.tbq4_attn_decode(dev_t(q), kc, vc, dev_t(lens), 5000, scale))
    res["decode_split64"] = half_bits(
        T.tbq4_attn_decode(dev_t(q), kc, vc, dev_t(lens), 5000, scale, split_tokens=64))
    # one token per sequence at position len: the per-row kernel
    kn = rng.standard_normal((B, 1, Hkv, D)).astype(np.float32)
    vn = rng.standard_normal((B, 1, Hkv, D)).astype(np.float32)
    T.tbq4_quantize_append(dev_t(kn), dev_t(lens), kc, 0)
    T.tbq4_quantize_append(dev_t(vn), dev_t(lens), vc, 0)
    # the fused step: the next token is encoded by the attention kernel
    lens2 = lens + 2
    k2 = rng.standard_normal((B, Hkv, D)).astype(np.float32)
    v2 = rng.standard_normal((B, Hkv, D)).astype(np.float32)
    res["decode_append"] = half_bits(T.tbq4_attn_decode_append(
        dev_t(q), dev_t(k2), dev_t(v2), kc, vc, dev_t(lens2), int(lens2.max()), scale))
    res["k_cache"] = kc.cpu().numpy()
    res["v_cache"] = vc.cpu().numpy()
    # multi-query decode: the last 3 tokens of each sequence
    q3 = rng.standard_normal((B, 3, Hq, D)).astype(np.float32)
    res["decode_mq"] = half_bits(
        T.tbq4_attn_decode_mq(dev_t(q3), kc, vc, dev_t(lens2), int(lens2.max()), scale))
    # chunked prefill: positions 4500 .. 4999 of sequence 0 as the chunk
    qp = torch.from_numpy(rng.standard_normal((500, Hq, D)).astype(np.float32)).to(dev)
    res["prefill"] = half_bits(
        T.tbq4_attn_prefill_chunk(qp.to(torch.bfloat16), 4500, kc[0], vc[0], scale))

    # paged: 64-token pages, pages handed out in a shuffled order
    page, n_pages, max_pages = 64, 150, 64
    order = rng.permutation(n_pages).astype(np.int32)
    table = np.full((B, max_pages), -1, np.int32)
    need = [(3100 + page - 1) // page] * 2       # every appended position has a page
    table[0, :need[0]] = order[:need[0]]
    table[1, :need[1]] = order[need[0]:need[0] + need[1]]
    plens = np.array([3100, 2000], np.int32)
    kp = T.empty_pool(n_pages, Hkv, page)
    vp = T.empty_pool(n_pages, Hkv, page)
    kp.zero_()
    vp.zero_()
    kx = rng.standard_normal((B, 3100, Hkv, D)).astype(np.float32)
    vx = rng.standard_normal((B, 3100, Hkv, D)).astype(np.float32)
    T.tbq4_quantize_append_paged(dev_t(kx), zero, dev_t(table), kp, 0)
    T.tbq4_quantize_append_paged(dev_t(vx), zero, dev_t(table), vp, 0)
    res["decode_paged"] = half_bits(T.tbq4_attn_decode_paged(
        dev_t(q), kp, vp, dev_t(table), dev_t(plens), 3100, scale))
    res["k_pool"] = kp.cpu().numpy()

    # 3-bit caches
    k3 = T.empty_cache3(B, Hkv, cap)
    v3 = T.empty_cache3(B, Hkv, cap)
    k3.zero_()
    v3.zero_()
    T.tbq3_quantize_append(dev_t(k), zero, k3, 0)
    T.tbq3_quantize_append(dev_t(v), zero, v3, 0)
    res["decode_tbq3"] = half_bits(T.tbq3_attn_decode(dev_t(q), k3, v3, dev_t(lens), 5000, scale))
    res["k_cache3"] = k3.cpu().numpy()

    torch.cuda.synchronize()
    res["status"] = np.array(T.tbq4_get_device_status())
    # the library file this process actually mapped
    with open("/proc/self/maps") as f:
        res["mapped"] = np.array(sorted({ln.split()[-1].rsplit("/", 1)[-1] for ln in f
                                         if "libtbq4" in ln}))
    np.savez(path, **res)


if __name__ == "__main__":
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    run(sys.argv[1])

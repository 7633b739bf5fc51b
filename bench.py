#!/usr/bin/env python3
"""Benchmark of the TBQ4 attention hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl tbq4|reference]

One step is one decode step at 262,144 cached tokens (24 query heads over 4
KV heads, head_dim 128, K with 4 outlier channels per head x10): the new
token's K and V rows are quantise-appended into the TBQ4 caches, then decode
attention runs over all 262,144 keys (split kernel + log-sum-exp combine
with the inverse rotation).  `value` is effective HBM throughput: the
algorithmic bytes of one step (the TBQ4 K and V blocks read, plus q, the
output and the appended rows) divided by the device time of the step.

The same line also carries the chunked-prefill figure (512 new tokens over
131,072 cached tokens, causal, after appending the chunk) in TFLOP/s, the
roofline of the dominant kernel, an end-to-end figure through the public
API with host buffers, and the fp64 CPU oracle timed on the host cores.

Timing: W untimed warm-up steps, then exactly K steps, each bracketed by
CUDA events on the launching stream; the L2 cache is flushed (512 MiB
written, then read back, so no dirty lines are left) before every timed
step, outside the events.  With N > 1 (torchrun)
every rank runs an independent replica and the time is the max over ranks.
"""
import argparse
import hashlib
import json
import math
import os
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "TBQ4 flash-decode effective HBM GB/s & % peak at 262K ctx; prefill TFLOP/s"
D = 128
BLOCK = 66


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="tbq4", choices=["tbq4", "reference"])
    ap.add_argument("--prefill-steps", type=int, default=5)
    ap.add_argument("--no-prefill", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--profile", choices=["decode", "prefill", "quantize"], default=None,
                    help="only run warm-up + steps of one workload's step, untimed, with "
                         "no flush buffer (a small footprint for ncu captures)")
    return ap.parse_args()


# ----------------------------------------------------------------- helpers
def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        p = json.load(open(path))
        return {"hbm_gbs": float(p["hbm_gbs"]), "bf16_tflops": float(p["bf16_tflops"]),
                "bf16_tflops_sustained": float(p.get("bf16_tflops_sustained", p["bf16_tflops"])),
                "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
            "source": "fallback"}


# Source files each profiled kernel is built from: a recorded ncu traffic
# figure is only reported while these files are unchanged.
KERNEL_SOURCES = {
    "decode_tc_kernel": ["common.cuh", "mbarrier.cuh", "quantize.cuh", "decode.cuh",
                         "decode_tc.cuh"],
    "prefill_tc_kernel": ["common.cuh", "mbarrier.cuh", "decode.cuh", "tcgen05.cuh",
                          "prefill_tc.cuh"],
    "quantize_rows_kernel": ["common.cuh", "mbarrier.cuh", "quantize.cuh"],
}


def kernel_source_hash(kernel):
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "long_context_attention_tbq4_b200", "csrc")
    for name in KERNEL_SOURCES[kernel]:
        h.update(name.encode())
        h.update(open(os.path.join(csrc, name), "rb").read())
    return h.hexdigest()[:16]


def recorded_traffic(kernel):
    """DRAM bytes per launch from a committed ncu summary, if it was taken on
    the kernel's current sources (else None)."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(path):
        return None
    rec = json.load(open(path)).get(kernel)
    if not rec or rec.get("source_sha256") != kernel_source_hash(kernel):
        return None
    return rec.get("dram_bytes_per_launch")


class Clocks:
    """nvidia-smi sampled every 200 ms while the timed region runs."""
    Q = ("index,uuid,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, uuid):
        self.uuid = uuid
        self.f = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
        self.p = None

    def __enter__(self):
        try:
            self.p = subprocess.Popen(["nvidia-smi", f"--query-gpu={self.Q}",
                                       "--format=csv,noheader,nounits", "-lms", "200"],
                                      stdout=self.f, stderr=subprocess.DEVNULL)
        except OSError:
            self.p = None
        time.sleep(0.3)
        return self

    def __exit__(self, *a):
        if self.p is not None:
            self.p.terminate()
            self.p.wait()

    def summary(self):
        self.f.flush()
        rows = []
        for line in open(self.f.name):
            parts = [x.strip() for x in line.split(",")]
            if len(parts) < 10 or (self.uuid and self.uuid not in parts[1]):
                continue
            try:
                rows.append((float(parts[2]), float(parts[3]), parts[6:10], parts[5]))
            except ValueError:
                continue
        os.unlink(self.f.name)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i, v in enumerate(r[2]) if v == "Active"})
        return {"sm_mhz": float(np.median([r[0] for r in rows])),
                "sm_max_mhz": max(r[1] for r in rows), "reasons": reasons,
                "samples": len(rows)}


# ---------------------------------------------------------------- workloads
def load_workloads():
    """The seeded input generators, loaded by file path: importing them
    through the package would run its __init__, which maps libtbq4.so, and
    the reference (oracle) arm must not map the product library."""
    import importlib.util
    name = "_tbq4_workloads"
    if name in sys.modules:
        return sys.modules[name]
    path = os.path.join(ROOT, "long_context_attention_tbq4_b200", "workloads.py")
    spec = importlib.util.spec_from_file_location(name, path)
    mod = importlib.util.module_from_spec(spec)
    sys.modules[name] = mod
    spec.loader.exec_module(mod)
    return mod


# What the decode path computes in: the arithmetic type of each stage.
DECODE_DTYPE = ("u8 x s8 integer QK (q_rot as an 18-bit integer, exact int32 sums), "
                "f16 PV operands with f32 accumulation, f32 softmax, f16 output")
PREFILL_DTYPE = "bf16 QK and PV on tcgen05 with f32 TMEM accumulators, f32 softmax, bf16 output"


def decode_config(case, N, world):
    """The config both arms print (the product and the oracle reference)."""
    return {"workload": "decode_262k", "batch": case.B, "ctx": N, "Hq": case.Hq,
            "Hkv": case.Hkv, "head_dim": D, "kv_format": "tbq4 (66 B / 128 values)",
            "step": "append the new token's K/V rows, then decode attention over all keys "
                    "(split kernel + log-sum-exp combine with the inverse rotation)",
            "l2": L2_NOTE, "launch": LAUNCH_NOTE,
            "parallelism": "replicas" if world > 1 else "single"}


L2_NOTE = ("inputs larger than L2: the steps cycle through 4 layers' caches (4 x 138 MB, "
           "4.4x the 126 MB L2), so no step finds its blocks in L2; the 'isolated' block "
           "flushes L2 (512 MiB written, then read back) before every step instead")
LAUNCH_NOTE = ("the K timed steps are one CUDA graph replayed once between two events, each "
               "step a split kernel + combine, the split kernel a programmatic dependent of "
               "the combine before it; e2e: each step also copies its inputs in (one packed "
               "copy from its own pinned buffer) and its output out (to its own pinned "
               "buffer) on a copy stream that overlaps the neighbouring steps' kernels, the K "
               "steps captured as one graph and replayed once (the same steps issued eagerly "
               "from Python, copies in line: e2e.ms_per_step_eager)")


def decode_workload():
    W = load_workloads()
    case = W.decode_262k()
    N = int(case.seq_lens[0])
    bytes_kv = 2 * case.Hkv * N * BLOCK
    bytes_q = case.B * case.Hq * D * 4
    bytes_out = case.B * case.Hq * D * 2
    bytes_append = 2 * case.Hkv * (D * 4 + BLOCK)          # new token: read fp32, write block
    # the attention kernel also encodes the new token, so its bytes include the append
    return case, N, bytes_kv + bytes_q + bytes_out + bytes_append, bytes_kv + bytes_q + bytes_append


def prefill_flops(n_cached, n_new, Hq):
    keys = sum(n_cached + i + 1 for i in range(n_new))
    return 4.0 * D * Hq * keys


# --------------------------------------------------------------- GPU legs
def timing_events(torch, n):
    """n quadruples of timing events (step start/end, kernel start/end).
    torch creates an event lazily at its first record, so each is recorded
    once here to exist before its handle is given to the library."""
    ev = [tuple(torch.cuda.Event(enable_timing=True) for _ in range(4)) for _ in range(n)]
    for quad in ev:
        for e in quad:
            e.record()
    torch.cuda.synchronize()
    return ev


def flush_l2(buf):
    """Evict the L2: write a buffer larger than it, then read the buffer back,
    so the write-back of the dirty lines also happens here, outside the
    timed region, and the next step starts on a clean, cold L2."""
    buf.zero_()
    buf.sum()


def capture_graph(torch, fn):
    """fn captured as a CUDA graph, after one run on a side stream (the usual
    warm-up before capture)."""
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        fn()
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        fn()
    torch.cuda.synchronize()
    return g


N_LAYERS = 4      # distinct layer caches the back-to-back decode steps cycle through


def bench_decode(T, torch, case, N, step_bytes, kernel_bytes, steps, warmup, flush):
    """The decode step, timed two ways.

    Back to back (the headline): a model's decode step runs attention for
    one layer after another, each over its own cache.  K steps cycle through
    N_LAYERS layers' caches (4 x 138 MB, over 4x the L2, so no step finds
    the data of the step before it in L2) and are captured as one CUDA graph
    replayed once between two events; each split kernel is a programmatic
    dependent of the combine before it.

    Isolated: one step at a time, the L2 flushed before each, each step
    between its own events (a single call's latency)."""
    dev = torch.device("cuda")
    cap = N
    K, V = case.k[0], case.v[0]
    kc0 = T.empty_cache(1, case.Hkv, cap)
    vc0 = T.empty_cache(1, case.Hkv, cap)
    zero = torch.zeros(1, dtype=torch.int32, device=dev)
    for cache, x in ((kc0, K), (vc0, V)):
        src = torch.from_numpy(np.ascontiguousarray(x[:N - 1])[None]).to(dev)
        T.tbq4_quantize_append(src, zero, cache, case.sign_seed)
        del src
    # the other layers hold the same blocks in their own memory
    kcs = [kc0] + [kc0.clone() for _ in range(N_LAYERS - 1)]
    vcs = [vc0] + [vc0.clone() for _ in range(N_LAYERS - 1)]
    k_new = torch.from_numpy(np.ascontiguousarray(K[N - 1:N])[None]).to(dev)
    v_new = torch.from_numpy(np.ascontiguousarray(V[N - 1:N])[None]).to(dev)
    q = torch.from_numpy(case.q).to(dev)
    lens = torch.tensor([N], dtype=torch.int32, device=dev)
    ws = torch.empty(T.tbq4_decode_workspace_bytes(1, case.Hq, case.Hkv, N), dtype=torch.uint8,
                     device=dev)
    out = torch.empty((1, case.Hq, D), dtype=torch.float16, device=dev)

    def step(layer=0, qq=q, kn=k_new, vn=v_new, o=out):
        # one decode step of one layer: the new token's K/V rows are encoded
        # into that layer's caches at position N-1 by the attention kernel
        T.tbq4_attn_decode_append(qq, kn.view(1, case.Hkv, D), vn.view(1, case.Hkv, D),
                                  kcs[layer], vcs[layer], lens, N, case.softmax_scale,
                                  case.sign_seed, workspace=ws, out=o)

    for i in range(warmup):
        step(i % N_LAYERS)
    torch.cuda.synchronize()
    assert T.tbq4_get_device_status() == 0

    # ---- back to back: K steps over the layers, one graph, one event pair
    g_run = capture_graph(torch, lambda: [step(i % N_LAYERS) for i in range(steps)])
    g_run.replay()                      # untimed: the graph's first replay
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier()
    torch.cuda.synchronize()
    e0.record()
    g_run.replay()
    e1.record()
    torch.cuda.synchronize()
    barrier()
    b2b_ms = e0.elapsed_time(e1)
    del g_run
    assert T.tbq4_get_device_status() == 0

    # ---- isolated: L2 flushed before every step, each step between events
    ev = timing_events(torch, steps)
    barrier()
    torch.cuda.synchronize()
    for e0, e1, k0, k1 in ev:
        flush_l2(flush)
        T.tbq4_set_timing_events(k0, k1)
        e0.record()
        step()
        e1.record()
    T.tbq4_set_timing_events(None, None)
    torch.cuda.synchronize()
    barrier()
    eager_ms = [e0.elapsed_time(e1) for e0, e1, _, _ in ev]
    kern_ms = [k0.elapsed_time(k1) for _, _, k0, k1 in ev]
    g_step = capture_graph(torch, step)
    ev = timing_events(torch, steps)
    barrier()
    torch.cuda.synchronize()
    for e0, e1, _, _ in ev:
        flush_l2(flush)
        e0.record()
        g_step.replay()
        e1.record()
    torch.cuda.synchronize()
    barrier()
    iso_ms = [e0.elapsed_time(e1) for e0, e1, _, _ in ev]
    del g_step

    # ---- end to end, back to back: every step copies its q and new rows in
    # from pinned host memory (one packed copy, its own host buffer per step)
    # and its output back out to its own pinned buffer, through the public
    # API.  Timed two ways: the K steps captured as one CUDA graph (copy
    # nodes, kernels, copy nodes; as a serving loop captures its decode
    # steps) and replayed once between two events (the reported value), and
    # the same steps issued eagerly from Python.
    nq, nk = case.Hq * D, case.Hkv * D
    n_e2e = max(steps, warmup)
    packed = np.concatenate([case.q.reshape(-1), np.ascontiguousarray(K[N - 1]).reshape(-1),
                             np.ascontiguousarray(V[N - 1]).reshape(-1)]).astype(np.float32)
    in_h = [torch.from_numpy(packed.copy()).pin_memory() for _ in range(n_e2e)]
    out_h = [torch.empty((1, case.Hq, D), dtype=torch.float16).pin_memory()
             for _ in range(n_e2e)]
    in_d = torch.empty_like(in_h[0], device=dev)
    q_v = in_d[:nq].view(1, case.Hq, D)
    kn_v = in_d[nq:nq + nk].view(1, case.Hkv, D)
    vn_v = in_d[nq + nk:].view(1, case.Hkv, D)

    def e2e_step(i):
        in_d.copy_(in_h[i], non_blocking=True)
        step(i % N_LAYERS, q_v, kn_v, vn_v, out)
        out_h[i].copy_(out, non_blocking=True)

    # The graph's steps overlap their copies with the neighbouring steps'
    # kernels: inputs travel on a copy stream one step ahead (two device
    # input buffers), outputs return on it while the next step computes (two
    # device output buffers); the events become the graph's edges.
    in_d2 = [torch.empty_like(in_h[0], device=dev) for _ in range(2)]
    out_d2 = [torch.empty_like(out) for _ in range(2)]
    cs = torch.cuda.Stream()
    ev_fork = torch.cuda.Event()
    ev_in = [torch.cuda.Event() for _ in range(2)]      # the buffer's inputs landed
    ev_done = [torch.cuda.Event() for _ in range(2)]    # the step using the buffer finished
    ev_back = [torch.cuda.Event() for _ in range(2)]    # its output is in host memory

    def e2e_overlapped(n):
        comp = torch.cuda.current_stream()

        def h2d(i):
            b = i % 2
            with torch.cuda.stream(cs):
                if i >= 2:
                    cs.wait_event(ev_done[b])
                in_d2[b].copy_(in_h[i], non_blocking=True)
                ev_in[b].record(cs)

        ev_fork.record(comp)
        cs.wait_event(ev_fork)
        h2d(0)
        for i in range(n):
            b = i % 2
            if i + 1 < n:
                h2d(i + 1)
            comp.wait_event(ev_in[b])
            if i >= 2:
                comp.wait_event(ev_back[b])
            x = in_d2[b]
            step(i % N_LAYERS, x[:nq].view(1, case.Hq, D), x[nq:nq + nk].view(1, case.Hkv, D),
                 x[nq + nk:].view(1, case.Hkv, D), out_d2[b])
            ev_done[b].record(comp)
            with torch.cuda.stream(cs):
                cs.wait_event(ev_done[b])
                out_h[i].copy_(out_d2[b], non_blocking=True)
                ev_back[b].record(cs)
        comp.wait_event(ev_back[(n - 1) % 2])

    def timed(fn):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        barrier()
        torch.cuda.synchronize()
        e0.record()
        fn()
        e1.record()
        torch.cuda.synchronize()
        barrier()
        return e0.elapsed_time(e1)

    for i in range(warmup):
        e2e_step(i)
    torch.cuda.synchronize()
    e2e_eager_total = timed(lambda: [e2e_step(i) for i in range(steps)])
    g_e2e = capture_graph(torch, lambda: e2e_overlapped(steps))
    g_e2e.replay()                      # untimed: the graph's first replay
    torch.cuda.synchronize()
    for o in out_h[:steps]:
        o.zero_()
    e2e_total = timed(g_e2e.replay)
    del g_e2e
    assert T.tbq4_get_device_status() == 0
    for o in out_h[:steps]:             # every step's output came back to the host
        assert torch.equal(o, out_h[steps - 1]) and bool(o.abs().sum() > 0)
    h2d_bytes = in_h[0].numel() * 4
    d2h_bytes = out_h[0].numel() * 2
    return {"b2b_ms": b2b_ms, "step_ms": [b2b_ms / steps] * steps, "iso_ms": iso_ms,
            "eager_ms": eager_ms, "kern_ms": kern_ms, "e2e_ms": [e2e_total / steps] * steps,
            "e2e_eager_ms": e2e_eager_total / steps,
            "h2d": h2d_bytes, "d2h": d2h_bytes, "launches_per_step": 2,
            "out": out.float().cpu().numpy()}


def bench_prefill(T, torch, steps, warmup, flush):
    W = load_workloads()
    c = W.prefill_131k()
    dev = torch.device("cuda")
    cap = W.round_capacity(c.n_cached + c.n_new)
    kc = T.empty_cache(1, c.Hkv, cap)
    vc = T.empty_cache(1, c.Hkv, cap)
    zero = torch.zeros(1, dtype=torch.int32, device=dev)
    for cache, x in ((kc, c.k), (vc, c.v)):
        src = torch.from_numpy(np.ascontiguousarray(x[:c.n_cached])[None]).to(dev)
        T.tbq4_quantize_append(src, zero, cache, c.sign_seed)
        del src
    kch = torch.from_numpy(np.ascontiguousarray(c.k[c.n_cached:])[None]).to(dev)
    vch = torch.from_numpy(np.ascontiguousarray(c.v[c.n_cached:])[None]).to(dev)
    pos = torch.tensor([c.n_cached], dtype=torch.int32, device=dev)
    q = torch.from_numpy(c.q_bf16.view(np.int16)).to(dev).view(torch.bfloat16)
    ws = torch.empty(T.tbq4_prefill_workspace_bytes(c.n_new, c.Hq, c.Hkv, c.n_cached),
                     dtype=torch.uint8, device=dev)
    out = torch.empty((c.n_new, c.Hq, D), dtype=torch.bfloat16, device=dev)

    def step():
        T.tbq4_quantize_append(kch, pos, kc, c.sign_seed)
        T.tbq4_quantize_append(vch, pos, vc, c.sign_seed)
        T.tbq4_attn_prefill_chunk(q, c.n_cached, kc[0], vc[0], c.softmax_scale, c.sign_seed,
                                  workspace=ws, out=out)

    for _ in range(warmup):
        step()
    torch.cuda.synchronize()
    ev = timing_events(torch, steps)
    barrier()
    for e0, e1, k0, k1 in ev:
        flush_l2(flush)
        T.tbq4_set_timing_events(k0, k1)
        e0.record()
        step()
        e1.record()
    T.tbq4_set_timing_events(None, None)
    torch.cuda.synchronize()
    barrier()
    assert T.tbq4_get_device_status() == 0
    flops = prefill_flops(c.n_cached, c.n_new, c.Hq)
    eager_ms = float(np.mean([a.elapsed_time(b) for a, b, _, _ in ev]))
    kern_ms = float(np.mean([a.elapsed_time(b) for _, _, a, b in ev]))
    # the step replayed from a CUDA graph, as for decode
    g_step = capture_graph(torch, step)
    ev = timing_events(torch, steps)
    barrier()
    for e0, e1, _, _ in ev:
        flush_l2(flush)
        e0.record()
        g_step.replay()
        e1.record()
    torch.cuda.synchronize()
    barrier()
    del g_step
    step_ms = float(np.mean([a.elapsed_time(b) for a, b, _, _ in ev]))
    return {"workload": c.name, "n_cached": c.n_cached, "n_new": c.n_new, "Hq": c.Hq,
            "Hkv": c.Hkv, "flops_per_step": flops, "ms_per_step": step_ms,
            "ms_per_step_eager": eager_ms,
            "tflops": flops / (step_ms * 1e-3) / 1e12, "attn_kernel_ms": kern_ms,
            "attn_kernel_tflops": flops / (kern_ms * 1e-3) / 1e12, "steps": steps}


def profile_decode(T, torch, case, N, n_steps):
    """Decode steps at 262K with nothing else on the device (for ncu)."""
    dev = torch.device("cuda")
    kc = T.empty_cache(1, case.Hkv, N)
    vc = T.empty_cache(1, case.Hkv, N)
    zero = torch.zeros(1, dtype=torch.int32, device=dev)
    for cache, x in ((kc, case.k[0]), (vc, case.v[0])):
        src = torch.from_numpy(np.ascontiguousarray(x[:N - 1])[None]).to(dev)
        T.tbq4_quantize_append(src, zero, cache, case.sign_seed)
        del src
    torch.cuda.synchronize()
    torch.cuda.empty_cache()
    k_new = torch.from_numpy(np.ascontiguousarray(case.k[0][N - 1])[None]).to(dev)
    v_new = torch.from_numpy(np.ascontiguousarray(case.v[0][N - 1])[None]).to(dev)
    q = torch.from_numpy(case.q).to(dev)
    lens = torch.tensor([N], dtype=torch.int32, device=dev)
    ws = torch.empty(T.tbq4_decode_workspace_bytes(1, case.Hq, case.Hkv, N), dtype=torch.uint8,
                     device=dev)
    out = torch.empty((1, case.Hq, D), dtype=torch.float16, device=dev)
    for _ in range(n_steps):
        T.tbq4_attn_decode_append(q, k_new, v_new, kc, vc, lens, N, case.softmax_scale,
                                  case.sign_seed, workspace=ws, out=out)
    torch.cuda.synchronize()
    assert T.tbq4_get_device_status() == 0
    print("profile: %d decode steps at %d keys" % (n_steps, N))
    return 0


def profile_prefill(T, torch, n_steps):
    """Chunked-prefill steps (append the chunk, attend) with nothing else on
    the device (for ncu)."""
    W = load_workloads()
    c = W.prefill_131k()
    dev = torch.device("cuda")
    cap = W.round_capacity(c.n_cached + c.n_new)
    kc = T.empty_cache(1, c.Hkv, cap)
    vc = T.empty_cache(1, c.Hkv, cap)
    zero = torch.zeros(1, dtype=torch.int32, device=dev)
    for cache, x in ((kc, c.k), (vc, c.v)):
        src = torch.from_numpy(np.ascontiguousarray(x)[None]).to(dev)
        T.tbq4_quantize_append(src, zero, cache, c.sign_seed)
        del src
    torch.cuda.synchronize()
    torch.cuda.empty_cache()
    q = torch.from_numpy(c.q_bf16.view(np.int16)).to(dev).view(torch.bfloat16)
    ws = torch.empty(T.tbq4_prefill_workspace_bytes(c.n_new, c.Hq, c.Hkv, c.n_cached),
                     dtype=torch.uint8, device=dev)
    out = torch.empty((c.n_new, c.Hq, D), dtype=torch.bfloat16, device=dev)
    for _ in range(n_steps):
        T.tbq4_attn_prefill_chunk(q, c.n_cached, kc[0], vc[0], c.softmax_scale, c.sign_seed,
                                  workspace=ws, out=out)
    torch.cuda.synchronize()
    assert T.tbq4_get_device_status() == 0
    print("profile: %d prefill steps, %d new over %d cached" % (n_steps, c.n_new, c.n_cached))
    return 0


def profile_quantize(T, torch, case, N, n_steps):
    """Bulk quantise-appends of the 262K K rows (1,048,576 rows, 537 MB in)
    with nothing else on the device (for ncu)."""
    dev = torch.device("cuda")
    kc = T.empty_cache(1, case.Hkv, N)
    src = torch.from_numpy(np.ascontiguousarray(case.k[0])[None]).to(dev)
    zero = torch.zeros(1, dtype=torch.int32, device=dev)
    for _ in range(n_steps):
        T.tbq4_quantize_append(src, zero, kc, case.sign_seed)
    torch.cuda.synchronize()
    assert T.tbq4_get_device_status() == 0
    print("profile: %d appends of %d rows" % (n_steps, N * case.Hkv))
    return 0


# ------------------------------------------------------------ CPU baseline
def oracle_decode_sample(case, N, rows):
    """Oracle caches (built once, untimed) and a timed call on `rows`."""
    import oracle
    cap = N
    ko = np.zeros((1, case.Hkv, cap, BLOCK), np.uint8)
    vo = np.zeros((1, case.Hkv, cap, BLOCK), np.uint8)
    oracle.quantize_append(case.k[0][:N - 1][None], np.zeros(1, np.int32), cap,
                           case.sign_seed, ko)
    oracle.quantize_append(case.v[0][:N - 1][None], np.zeros(1, np.int32), cap,
                           case.sign_seed, vo)
    lens = np.array([N], np.int32)
    pos = np.array([N - 1], np.int32)
    knew = case.k[0][N - 1:N][None]
    vnew = case.v[0][N - 1:N][None]

    def step():
        oracle.quantize_append(knew, pos, cap, case.sign_seed, ko)
        oracle.quantize_append(vnew, pos, cap, case.sign_seed, vo)
        return oracle.attn_decode(case.q, ko, vo, lens, case.softmax_scale, case.sign_seed,
                                  rows=rows)
    return step


def cpu_baseline(case, N, step_bytes, sample_rows=24, min_reps=5, target_s=10.0, max_reps=400):
    """The oracle's decode step on the host cores: the whole workload per step
    (it takes about a tenth of a second), repeated until about target_s
    seconds of oracle work have run; the median step is reported."""
    import oracle
    rows = np.arange(sample_rows, dtype=np.int32)
    step = oracle_decode_sample(case, N, rows)
    step()
    t = []
    while len(t) < min_reps or (sum(t) < target_s and len(t) < max_reps):
        t0 = time.perf_counter()
        step()
        t.append(time.perf_counter() - t0)
    t_full = float(np.median(t)) * (case.B * case.Hq / sample_rows)
    return {"value": step_bytes / t_full / 1e9, "unit": "GB/s", "cores": oracle.get_threads(),
            "kind": "oracle",
            "sample": (f"decode_262k, {sample_rows} of {case.B * case.Hq} query-head rows "
                       f"over all {N} keys plus the new token's append, median of {len(t)} "
                       f"steps ({sum(t):.1f} s of oracle work); time scaled by "
                       f"{case.B * case.Hq}/{sample_rows}"),
            "sample_seconds": float(np.median(t)), "total_seconds": float(sum(t))}


# ------------------------------------------------------------- distributed
_dist = None             # torch.distributed once a process group is up (N > 1)
_dist_device = "cuda"    # where the max-over-ranks reduction runs: "cuda" (nccl), "cpu" (gloo)


def init_distributed(torch, backend, local):
    """One process group for the N independent replicas: nccl on the GPUs,
    gloo for the CPU tests of the same host logic.  The timeout is short so
    that a rank that never arrives ends the others' next collective with an
    error."""
    global _dist, _dist_device
    import datetime
    import torch.distributed as dist
    kw = {"device_id": torch.device("cuda", local)} if backend == "nccl" else {}
    dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120), **kw)
    _dist = dist
    _dist_device = "cuda" if backend == "nccl" else "cpu"


def barrier():
    if _dist is not None:
        _dist.barrier()


def max_over_ranks(torch, x):
    if _dist is None:
        return x
    t = torch.tensor([x], dtype=torch.float64, device=_dist_device)
    _dist.all_reduce(t, op=_dist.ReduceOp.MAX)
    return float(t.item())


def replica_totals(torch, dec, steps, world, step_bytes):
    """Whole-job figures of `world` independent replicas, each rank having
    timed `steps` decode steps (dec: per-step device times in ms).  Every time
    is the max over ranks; the value counts the bytes of all ranks.  Every
    rank makes the same four reductions in the same order."""
    total_ms = max_over_ranks(torch, float(np.sum(dec["step_ms"])))
    ms_per_step = total_ms / steps
    e2e_ms = max_over_ranks(torch, float(np.mean(dec["e2e_ms"])))
    eager_ms = max_over_ranks(torch, float(np.mean(dec["eager_ms"])))
    e2e_eager_ms = max_over_ranks(torch, float(dec.get("e2e_eager_ms", 0.0)))
    return {"ms_per_step": ms_per_step,
            "value": world * step_bytes / (ms_per_step * 1e-3) / 1e9,
            "e2e_ms": e2e_ms, "e2e_value": world * step_bytes / (e2e_ms * 1e-3) / 1e9,
            "eager_ms": eager_ms, "e2e_eager_ms": e2e_eager_ms}


# -------------------------------------------------------------------- main
def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    case, N, step_bytes, _ = decode_workload()
    sample_rows = case.B * case.Hq
    step = oracle_decode_sample(case, N, np.arange(sample_rows, dtype=np.int32))
    for _ in range(args.warmup):
        step()
    t = []
    for _ in range(args.steps):
        t0 = time.perf_counter()
        step()
        t.append(time.perf_counter() - t0)
    import oracle
    scale = case.B * case.Hq / sample_rows
    ms = float(np.mean(t)) * scale * 1e3
    value = step_bytes / (ms * 1e-3) / 1e9
    sample = (f"decode_262k, {sample_rows} of {case.B * case.Hq} query-head rows over all "
              f"{N} keys per step plus the new token's append; time scaled by {scale:g}")
    line = {"metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "f64 (the oracle's arithmetic; the encoder in f32 as the codebook fixes)",
            "data": "synthetic", "impl": "reference",
            "config": decode_config(case, N, int(os.environ.get("WORLD_SIZE", "1"))),
            "cpu_baseline": {"value": value, "unit": "GB/s", "cores": oracle.get_threads(),
                             "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": "GB/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


def main():
    args = parse()
    if args.impl == "reference":
        return run_reference(args)

    import torch
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    if world > 1:
        init_distributed(torch, "nccl", local)
    import long_context_attention_tbq4_b200 as T

    peaks = measured_peaks()
    case, N, step_bytes, kernel_bytes = decode_workload()
    if args.profile == "decode":
        return profile_decode(T, torch, case, N, args.steps + args.warmup)
    if args.profile == "prefill":
        return profile_prefill(T, torch, args.steps + args.warmup)
    if args.profile == "quantize":
        return profile_quantize(T, torch, case, N, args.steps + args.warmup)
    flush = torch.empty(512 << 20, dtype=torch.uint8, device="cuda")
    uuid = str(getattr(torch.cuda.get_device_properties(local), "uuid", "") or "")
    with Clocks(uuid) as clk:
        dec = bench_decode(T, torch, case, N, step_bytes, kernel_bytes, args.steps,
                           args.warmup, flush)
        pre = None if args.no_prefill else bench_prefill(T, torch, args.prefill_steps,
                                                         min(args.warmup, 3), flush)
    clocks = clk.summary()

    tot = replica_totals(torch, dec, args.steps, world, step_bytes)
    ms_per_step, value, e2e_ms = tot["ms_per_step"], tot["value"], tot["e2e_ms"]
    # back to back, each step is exactly the split kernel + combine pair, so
    # the pair's average duration is the step's share of the timed region
    kern_ms = ms_per_step
    achieved = kernel_bytes / (kern_ms * 1e-3) / 1e9
    iso_kern_ms = max_over_ranks(torch, float(np.mean(dec["kern_ms"])))
    iso_ms = max_over_ranks(torch, float(np.mean(dec["iso_ms"])))
    traffic = recorded_traffic("decode_tc_kernel")
    line = {
        "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_per_step,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": DECODE_DTYPE, "data": "synthetic",
        "config": decode_config(case, N, world),
        "step_bytes": step_bytes,
        "pct_hbm_peak": value / world / peaks["hbm_gbs"],
        # the split kernel and its combine (a programmatic dependent launch,
        # no gap between them) are timed as one region
        "roofline": {"kernel": "decode_tc_kernel + decode_combine_kernel", "bound": "hbm",
                     "achieved": achieved,
                     "peak": peaks["hbm_gbs"], "unit": "GB/s",
                     "frac": achieved / peaks["hbm_gbs"], "traffic": traffic,
                     "algorithmic_bytes": kernel_bytes, "kernel_ms": kern_ms,
                     "timing": "back-to-back steps over 4 layers' caches: the region's "
                               "time / K",
                     "peak_source": peaks["source"]},
        # one step at a time with L2 flushed before it (a single call's
        # latency): graph replay per step, the same step launched eagerly, and
        # the split kernel + combine alone between the library's timing events
        "isolated": {"ms_per_step": iso_ms,
                     "value": world * step_bytes / (iso_ms * 1e-3) / 1e9,
                     "ms_per_step_eager": tot["eager_ms"], "kernel_ms": iso_kern_ms,
                     "kernel_frac": kernel_bytes / (iso_kern_ms * 1e-3) / 1e9 / peaks["hbm_gbs"],
                     "l2": "flushed before every step"},
        "e2e": {"value": tot["e2e_value"], "unit": "GB/s",
                "ms_per_step": e2e_ms, "h2d_bytes_per_step": dec["h2d"],
                "d2h_bytes_per_step": dec["d2h"],
                "timing": "the K steps with their copies captured as one CUDA graph (copies on "
                          "a copy stream, overlapping the neighbouring steps' kernels), "
                          "replayed once between two events",
                "ms_per_step_eager": tot["e2e_eager_ms"],
                "value_eager": world * step_bytes / (tot["e2e_eager_ms"] * 1e-3) / 1e9},
        "gpu_launches": dec["launches_per_step"] * args.steps,
        "clocks": clocks,
    }
    if pre is not None:
        pk = peaks["bf16_tflops"]
        pre["dtype"] = PREFILL_DTYPE
        pre["roofline"] = {"bound": "tensor", "achieved": pre["attn_kernel_tflops"],
                           "peak": pk, "unit": "TFLOP/s",
                           "frac": pre["attn_kernel_tflops"] / pk,
                           "traffic": recorded_traffic("prefill_tc_kernel"),
                           "peak_source": peaks["source"] + " (bf16 burst)"}
        line["prefill"] = pre
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(case, N, step_bytes)
    if rank == 0:
        print(json.dumps(line), flush=True)
    if _dist is not None:
        _dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())

// tbq4.cu -- libtbq4: the C ABI declared in include/tbq4.h and its launchers.
//
// One translation unit: the kernels live in the headers included below.
// Host code checks every argument before launching anything and never
// allocates, frees or synchronises (except tbq4_get_device_status).
#include "tbq4.h"

#include "common.cuh"
#include "quantize.cuh"
#include "decode.cuh"
#include "decode_tc.cuh"
#include "decode_mq.cuh"
#include "prefill_tc.cuh"
#include "selftest.cuh"

#include <algorithm>
#include <cmath>
#include <mutex>

#include <nvtx3/nvToolsExt.h>

namespace {

using namespace tbq4;

constexpr int kNumSMs = 148;          // B200
constexpr size_t kWsAlign = 256;

size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }
int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }
bool aligned(const void *p, size_t a) { return ((uintptr_t)p % a) == 0; }

// An NVTX range around an entry point's launches, named after the entry
// point, so timeline and kernel profilers can select one call's kernels
// (ncu --nvtx --nvtx-include).  Header-only NVTX: with no tool attached a
// push and a pop cost a few nanoseconds of host time.
struct NvtxRange {
    explicit NvtxRange(const char *name) { nvtxRangePushA(name); }
    ~NvtxRange() { nvtxRangePop(); }
    NvtxRange(const NvtxRange &) = delete;
    NvtxRange &operator=(const NvtxRange &) = delete;
};

// SplitMix64 (Steele, Lea & Flood 2014): the two words whose bits are the
// +-1 diagonal (bit set -> -1).
void sign_words(uint64_t seed, uint64_t *lo, uint64_t *hi) {
    uint64_t st = seed, w[2];
    for (int k = 0; k < 2; ++k) {
        st += 0x9E3779B97F4A7C15ULL;
        uint64_t z = st;
        z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ULL;
        z = (z ^ (z >> 27)) * 0x94D049BB133111EBULL;
        w[k] = z ^ (z >> 31);
    }
    *lo = w[0];
    *hi = w[1];
}

// Keys per split: one wave of the decode kernel (one CTA per SM) over the
// whole launch, in whole rounds of chunks for its 16 warps.
int32_t auto_split_tokens(int nseq, int Hkv, int32_t max_len) {
    const int64_t target = (int64_t)kNumSMs;          // one decode CTA per SM
    int64_t per = ceil_div((int64_t)max_len * nseq * Hkv, target);
    // whole rounds of 32-token chunks over the 16 warps of a CTA, so every
    // warp of a full split gets the same number of chunks
    per = ceil_div(per, (int64_t)kChunk * kTcWarps) * ((int64_t)kChunk * kTcWarps);
    if (per < (int64_t)kChunk * kTcWarps) per = (int64_t)kChunk * kTcWarps;
    // at most kPidCap chunks, the page ids a paged CTA keeps in shared memory
    if (per > (int64_t)kPidCap * kChunk) per = (int64_t)kPidCap * kChunk;
    return (int32_t)per;
}

struct WsLayout {
    size_t part_o, part_ml, total;
    int n_splits;
};

WsLayout attn_ws_layout(int nseq, int Hq, int32_t max_len, int32_t split_tokens) {
    WsLayout w;
    w.n_splits = max_len > 0 ? (int)ceil_div(max_len, split_tokens) : 1;
    const size_t rows = (size_t)nseq * Hq * w.n_splits;
    w.part_o = 0;
    w.part_ml = align_up(rows * kD * sizeof(float), kWsAlign);
    w.total = align_up(w.part_ml + rows * sizeof(float2), kWsAlign);
    return w;
}

cudaEvent_t g_ev_before = nullptr, g_ev_after = nullptr;

// Prefill work: one CTA per (M-pair, key split); M-pair = two query heads of
// a KV group x 128 query positions.  Key splits fill the 148 SMs (one CTA
// per SM: the kernel takes all of tensor memory).
struct PrefillPlan {
    int pairs, iblocks, mpairs, n_splits;
    size_t part_o, part_ml, total;
};

PrefillPlan prefill_ws_layout(int n_new, int Hq, int Hkv, int64_t n_cached) {
    PrefillPlan w;
    const int G = Hq / Hkv;
    w.pairs = (G + 1) / 2;
    w.iblocks = (n_new + pre::kTile - 1) / pre::kTile;
    w.mpairs = Hkv * w.pairs * w.iblocks;
    const int64_t tiles0 = (n_cached + std::min(n_new, pre::kTile) + pre::kTile - 1) / pre::kTile;
    int64_t ns = kNumSMs / w.mpairs;
    if (ns > tiles0) ns = tiles0;
    if (ns < 1) ns = 1;
    w.n_splits = (int)ns;
    const size_t rows = (size_t)n_new * Hq * w.n_splits;
    w.part_o = 0;
    w.part_ml = align_up(rows * kD * sizeof(float), kWsAlign);
    w.total = align_up(w.part_ml + rows * sizeof(float2), kWsAlign);
    return w;
}

bool ensure_smem_attr(const void *fn, int bytes, bool *done_per_device) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return false;
    if (!done_per_device[dev]) {
        if (cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) !=
            cudaSuccess)
            return false;
        done_per_device[dev] = true;
    }
    return true;
}

tbq4_status launch_status() {
    return cudaGetLastError() == cudaSuccess ? TBQ4_OK : TBQ4_ERR_LAUNCH;
}

tbq4_status run_attention(AttnParams p, void *workspace, size_t ws_bytes,
                          cudaStream_t st) {
    const NvtxRange range(p.q_len > 1 ? "tbq4_attn_decode_mq"
                          : p.block_table ? "tbq4_attn_decode_paged"
                          : p.tbq3 ? "tbq3_attn_decode"
                          : p.k_new ? "tbq4_attn_decode_append" : "tbq4_attn_decode");
    if (p.split_tokens <= 0 || p.split_tokens % 32 != 0) return TBQ4_ERR_SHAPE;
    const int qrows = p.nseq * (p.q_len > 1 ? p.q_len : 1);    // combine rows per head
    const WsLayout w = attn_ws_layout(qrows, p.Hq, p.max_len, p.split_tokens);
    if (ws_bytes < w.total) return TBQ4_ERR_WORKSPACE;
    if (w.n_splits > 65535 * 16) return TBQ4_ERR_SHAPE;
    p.n_splits = w.n_splits;
    p.part_o = reinterpret_cast<float *>(static_cast<char *>(workspace) + w.part_o);
    p.part_ml = reinterpret_cast<float2 *>(static_cast<char *>(workspace) + w.part_ml);
    p.part_rows = (int64_t)qrows * p.Hq * w.n_splits;
    p.out_elems = (int64_t)qrows * p.Hq * kD;
    p.cache_bytes = p.block_table
        ? p.n_pages * p.Hkv * p.page_size * (int64_t)(p.tbq3 ? kBlockBytes3 : kBlockBytes)
        : (int64_t)p.nseq * p.seq_stride;
    static bool attr_set[64] = {}, attr_paged[64] = {}, attr_mq[64] = {};  // once per device
    static bool attr_3[64] = {};
    const bool mq = p.q_len > 1, paged = p.block_table != nullptr;
    if (mq && paged) return TBQ4_ERR_SHAPE;
    if (p.tbq3 && (mq || paged || p.k_new)) return TBQ4_ERR_SHAPE;
    if (paged && p.split_tokens > kPidCap * kChunk) return TBQ4_ERR_SHAPE;
    if (mq ? !ensure_smem_attr((const void *)dmq::decode_mq_kernel, dmq::kSmemBytes, attr_mq)
           : paged ? !ensure_smem_attr((const void *)decode_tc_kernel<true>, kTcSmemBytesPaged,
                                       attr_paged)
           : p.tbq3 ? !ensure_smem_attr((const void *)decode_tc_kernel<false, 3>, kTcSmemBytes,
                                        attr_3)
                    : !ensure_smem_attr((const void *)decode_tc_kernel<false>, kTcSmemBytes, attr_set))
        return TBQ4_ERR_LAUNCH;
    dim3 g1(p.n_splits, p.Hkv, p.nseq);
    if (g_ev_before) cudaEventRecord(g_ev_before, st);
    if (mq) {
        dmq::decode_mq_kernel<<<g1, dmq::kThreads, dmq::kSmemBytes, st>>>(p);
    } else {
        // A programmatic dependent of the kernel before it: the split kernel
        // sets up and issues its first cache copies, then waits for that
        // kernel (griddepcontrol.wait) before it reads q or the lengths.
        // Only the decode combine triggers early, once its own inputs are
        // complete; after any other kernel this is an ordinary launch.
        cudaLaunchConfig_t sc = {};
        sc.gridDim = g1;
        sc.blockDim = dim3(kTcWarps * 32);
        sc.dynamicSmemBytes = paged ? kTcSmemBytesPaged : kTcSmemBytes;
        sc.stream = st;
        cudaLaunchAttribute sa[1];
        sa[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        sa[0].val.programmaticStreamSerializationAllowed = 1;
        sc.attrs = sa;
        sc.numAttrs = 1;
        cudaError_t e;
        if (paged)
            e = cudaLaunchKernelEx(&sc, decode_tc_kernel<true, 4>, p);
        else if (p.tbq3)
            e = cudaLaunchKernelEx(&sc, decode_tc_kernel<false, 3>, p);
        else
            e = cudaLaunchKernelEx(&sc, decode_tc_kernel<false, 4>, p);
        if (e != cudaSuccess) return TBQ4_ERR_LAUNCH;
    }
    // The combine is a programmatic dependent launch: its CTAs are placed as
    // decode CTAs retire and wait in griddepcontrol.wait for the whole decode
    // grid, so no launch gap separates the two kernels.
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(p.Hq, qrows);
    cfg.blockDim = dim3(kCombineWarps * 32);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaLaunchKernelEx(&cfg, decode_combine_kernel, p) != cudaSuccess) return TBQ4_ERR_LAUNCH;
    if (g_ev_after) cudaEventRecord(g_ev_after, st);
    return launch_status();
}

// Scratch of tbq4_attn_decode_noalloc: a fixed array in this library, for
// callers that cannot allocate.  Host code only ever passes its device
// address, looked up once per device (the host-side name is not an address
// the GPU can use).
constexpr size_t kNoAllocScratchBytes = size_t(8) << 20;
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

tbq4_status noalloc_scratch(void **ptr) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return TBQ4_ERR_LAUNCH;
    static void *addr[64] = {};
    static std::mutex mu;
    std::lock_guard<std::mutex> lock(mu);
    if (!addr[dev]) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr)
            return TBQ4_ERR_LAUNCH;
        addr[dev] = p;
    }
    *ptr = addr[dev];
    return TBQ4_OK;
}

}  // namespace

extern "C" {

size_t tbq4_block_bytes(void) { return kBlockBytes; }

size_t tbq4_cache_bytes(int batch, int n_kv_heads, int64_t capacity) {
    if (batch <= 0 || n_kv_heads <= 0 || capacity <= 0) return 0;
    return (size_t)batch * n_kv_heads * (size_t)capacity * kBlockBytes;
}

void tbq4_signs(uint64_t seed, int8_t out[128]) {
    uint64_t lo, hi;
    sign_words(seed, &lo, &hi);
    for (int i = 0; i < kD; ++i) {
        const uint64_t w = i < 64 ? lo : hi;
        out[i] = ((w >> (i & 63)) & 1u) ? -1 : 1;
    }
}

}  // extern "C"

namespace {

// Below this many rows the bulk encoder has too few 8-row groups to keep
// the GPU busy; the warp-per-row encoder takes over.
constexpr int64_t kSmallAppendRows = 16384;

tbq4_status quantize_impl(const float *src, int B, int n_new, int Hkv, const int32_t *start_pos,
                          int64_t capacity, uint64_t sign_seed, const PageMap &map,
                          uint8_t *cache, void *stream, int bits = 4) {
    const NvtxRange range(bits == 3 ? "tbq3_quantize_append"
                          : map.table ? "tbq4_quantize_append_paged" : "tbq4_quantize_append");
    if (!src || !start_pos || !cache) return TBQ4_ERR_NULL;
    if (!aligned(src, 16) || !aligned(cache, 16) || !aligned(start_pos, 4))
        return TBQ4_ERR_ALIGN;
    if (B <= 0 || n_new < 0 || Hkv <= 0) return TBQ4_ERR_SHAPE;
    if (capacity <= 0 || capacity % 8 != 0) return TBQ4_ERR_CAPACITY;
    if (n_new == 0) return TBQ4_OK;
    const int64_t rows = (int64_t)B * n_new * Hkv;
    if (rows > 0x7FFFFFFFLL) return TBQ4_ERR_SHAPE;      // rows are indexed in 32 bits
    PageMap pm = map;
    const int64_t blk = bits == 3 ? kBlockBytes3 : kBlockBytes;
    pm.cache_bytes = pm.table ? pm.n_pages * Hkv * pm.page_size * blk
                              : (int64_t)B * Hkv * capacity * blk;
    if (bits == 4 && rows < kSmallAppendRows) {
        // few rows: one warp per row over every SM
        uint64_t lo, hi;
        sign_words(sign_seed, &lo, &hi);
        int64_t blocks = ceil_div(rows, (int64_t)kQWarpRowsPerBlock);
        if (blocks > (int64_t)kNumSMs * 8) blocks = (int64_t)kNumSMs * 8;
        quantize_warp_rows_kernel<<<(unsigned)blocks, kQWarpRowsPerBlock * 32, 0,
                                    (cudaStream_t)stream>>>(src, B, n_new, Hkv, start_pos,
                                                            capacity, lo, hi, pm, cache);
        return launch_status();
    }
    uint64_t lo, hi;
    sign_words(sign_seed, &lo, &hi);
    static bool attr4[64] = {}, attr3[64] = {};    // set once per device
    const void *fn = bits == 3 ? (const void *)quantize_rows_kernel<3>
                               : (const void *)quantize_rows_kernel<4>;
    if (!ensure_smem_attr(fn, kQSmemBytes, bits == 3 ? attr3 : attr4)) return TBQ4_ERR_LAUNCH;
    // one CTA per SM, each over a strided share of the 8-position groups of
    // every (sequence, KV head)
    const int64_t gpb = ceil_div(n_new, (int64_t)kQRows);
    const int64_t groups = (int64_t)B * Hkv * gpb;
    if (groups > 0x7FFFFFFFLL) return TBQ4_ERR_SHAPE;
    const InvDiv div_gpb = InvDiv::make((uint32_t)gpb), div_hkv = InvDiv::make((uint32_t)Hkv);
    int64_t blocks = groups;
    if (blocks > (int64_t)kNumSMs) blocks = (int64_t)kNumSMs;
    if (bits == 3)
        quantize_rows_kernel<3><<<(unsigned)blocks, kQThreads, kQSmemBytes, (cudaStream_t)stream>>>(
            src, B, n_new, Hkv, start_pos, capacity, lo, hi, pm, cache, div_gpb, div_hkv);
    else
        quantize_rows_kernel<4><<<(unsigned)blocks, kQThreads, kQSmemBytes, (cudaStream_t)stream>>>(
            src, B, n_new, Hkv, start_pos, capacity, lo, hi, pm, cache, div_gpb, div_hkv);
    return launch_status();
}

}  // namespace

extern "C" {

tbq4_status tbq4_quantize_append(const float *src, int B, int n_new, int Hkv,
                                 const int32_t *start_pos, int64_t capacity,
                                 uint64_t sign_seed, uint8_t *cache, void *stream) {
    const PageMap contiguous = {nullptr, 0, 0, 0};
    return quantize_impl(src, B, n_new, Hkv, start_pos, capacity, sign_seed, contiguous, cache,
                         stream);
}

tbq4_status tbq3_quantize_append(const float *src, int B, int n_new, int Hkv,
                                 const int32_t *start_pos, int64_t capacity,
                                 uint64_t sign_seed, uint8_t *cache, void *stream) {
    const PageMap contiguous = {nullptr, 0, 0, 0};
    return quantize_impl(src, B, n_new, Hkv, start_pos, capacity, sign_seed, contiguous, cache,
                         stream, 3);
}

size_t tbq3_block_bytes(void) { return kBlockBytes3; }

size_t tbq3_cache_bytes(int batch, int n_kv_heads, int64_t capacity) {
    if (batch <= 0 || n_kv_heads <= 0 || capacity <= 0) return 0;
    return (size_t)batch * n_kv_heads * (size_t)capacity * kBlockBytes3;
}

tbq4_status tbq4_quantize_append_paged(const float *src, int B, int n_new, int Hkv,
                                       const int32_t *start_pos, const int32_t *block_table,
                                       int max_pages, int page_size, int64_t n_pages,
                                       uint64_t sign_seed, uint8_t *pool, void *stream) {
    if (!block_table) return TBQ4_ERR_NULL;
    if (!aligned(block_table, 4)) return TBQ4_ERR_ALIGN;
    if (page_size < 32 || page_size % 32 != 0 || max_pages <= 0 || n_pages <= 0 ||
        n_pages > 0x7FFFFFFFLL)
        return TBQ4_ERR_SHAPE;
    const PageMap pm = {block_table, max_pages, page_size, n_pages, 0};
    return quantize_impl(src, B, n_new, Hkv, start_pos, (int64_t)max_pages * page_size,
                         sign_seed, pm, pool, stream);
}

size_t tbq4_decode_workspace_bytes_split(int B, int Hq, int Hkv, int32_t max_len,
                                         int32_t split_tokens) {
    if (B <= 0 || Hq <= 0 || Hkv <= 0 || max_len < 0) return 0;
    if (split_tokens == 0) split_tokens = auto_split_tokens(B, Hkv, max_len);
    if (split_tokens <= 0) return 0;
    return attn_ws_layout(B, Hq, max_len, split_tokens).total;
}

size_t tbq4_decode_workspace_bytes(int B, int Hq, int Hkv, int32_t max_len) {
    return tbq4_decode_workspace_bytes_split(B, Hq, Hkv, max_len, 0);
}

}  // extern "C"

namespace {

// A block table and its pools (nullptr table: contiguous caches).
struct PagedArgs {
    const int32_t *block_table;
    int max_pages, page_size;
    int64_t n_pages;
};

// Checks a paged layout; sets *capacity to the tokens a table row can map.
tbq4_status check_paged(const PagedArgs &pg, int64_t *capacity) {
    if (!pg.block_table) return TBQ4_ERR_NULL;
    if (!aligned(pg.block_table, 4)) return TBQ4_ERR_ALIGN;
    if (pg.page_size < 32 || pg.page_size % 32 != 0 || pg.max_pages <= 0 || pg.n_pages <= 0 ||
        pg.n_pages > 0x7FFFFFFFLL)
        return TBQ4_ERR_SHAPE;
    *capacity = (int64_t)pg.max_pages * pg.page_size;
    return TBQ4_OK;
}

tbq4_status decode_impl(const float *q, const uint8_t *k_cache, const uint8_t *v_cache,
                        const int32_t *seq_lens, int32_t max_len, int B, int Hq, int Hkv,
                        int64_t capacity, float softmax_scale, uint64_t sign_seed,
                        int32_t split_tokens, void *workspace, size_t ws_bytes, uint16_t *out,
                        void *stream, const float *k_new, const float *v_new,
                        const PagedArgs *pg = nullptr, int bits = 4) {
    if (!q || !k_cache || !v_cache || !seq_lens || !workspace || !out)
        return TBQ4_ERR_NULL;
    if (pg) {
        const tbq4_status e = check_paged(*pg, &capacity);
        if (e != TBQ4_OK) return e;
    }
    if (!aligned(q, 16) || !aligned(k_cache, 16) || !aligned(v_cache, 16) ||
        !aligned(workspace, kWsAlign) || !aligned(out, 2) || !aligned(seq_lens, 4))
        return TBQ4_ERR_ALIGN;
    if (B <= 0 || B > 65535 || Hkv <= 0 || Hkv > 65535 || Hq <= 0 || Hq % Hkv != 0 ||
        Hq / Hkv > kMaxGroup || max_len < 0 || split_tokens < 0 || split_tokens % 32 != 0)
        return TBQ4_ERR_SHAPE;
    if (capacity <= 0 || capacity % 8 != 0 || (int64_t)max_len > capacity)
        return TBQ4_ERR_CAPACITY;
    if (!std::isfinite(softmax_scale)) return TBQ4_ERR_SHAPE;
    AttnParams p = {};
    p.q = q;
    p.q_bf16 = 0;
    p.k = k_cache;
    p.v = v_cache;
    p.head_stride = capacity * (bits == 3 ? kBlockBytes3 : kBlockBytes);
    p.seq_stride = (int64_t)Hkv * p.head_stride;
    p.tbq3 = bits == 3;
    p.seq_lens = seq_lens;
    p.max_len = max_len;
    p.capacity = capacity;
    p.nseq = B;
    p.Hq = Hq;
    p.Hkv = Hkv;
    p.G = Hq / Hkv;
    p.split_tokens = split_tokens ? split_tokens : auto_split_tokens(B, Hkv, max_len);
    p.scale_log2 = softmax_scale * 1.4426950408889634f;
    sign_words(sign_seed, &p.sign_lo, &p.sign_hi);
    p.out = out;
    p.out_bf16 = 0;
    if (k_new) {
        p.k_new = k_new;
        p.v_new = v_new;
        p.k_wr = const_cast<uint8_t *>(k_cache);
        p.v_wr = const_cast<uint8_t *>(v_cache);
    }
    if (pg) {
        p.head_stride = 0;
        p.seq_stride = 0;
        p.block_table = pg->block_table;
        p.max_pages = pg->max_pages;
        p.page_size = pg->page_size;
        p.n_pages = pg->n_pages;
    }
    return run_attention(p, workspace, ws_bytes, (cudaStream_t)stream);
}

}  // namespace

extern "C" {

tbq4_status tbq4_attn_decode_split(const float *q, const uint8_t *k_cache,
                                   const uint8_t *v_cache, const int32_t *seq_lens,
                                   int32_t max_len, int B, int Hq, int Hkv,
                                   int64_t capacity, float softmax_scale,
                                   uint64_t sign_seed, int32_t split_tokens,
                                   void *workspace, size_t ws_bytes, uint16_t *out,
                                   void *stream) {
    return decode_impl(q, k_cache, v_cache, seq_lens, max_len, B, Hq, Hkv, capacity,
                       softmax_scale, sign_seed, split_tokens, workspace, ws_bytes, out, stream,
                       nullptr, nullptr);
}

size_t tbq4_decode_mq_workspace_bytes(int B, int q_len, int Hq, int Hkv, int32_t max_len) {
    if (B <= 0 || q_len <= 0 || Hq <= 0 || Hkv <= 0 || max_len < 0) return 0;
    const int32_t split = auto_split_tokens(B, Hkv, max_len);
    return attn_ws_layout(B * q_len, Hq, max_len, split).total;
}

tbq4_status tbq4_attn_decode_mq(const float *q, const uint8_t *k_cache, const uint8_t *v_cache,
                                const int32_t *seq_lens, int32_t max_len, int B, int q_len,
                                int Hq, int Hkv, int64_t capacity, float softmax_scale,
                                uint64_t sign_seed, void *workspace, size_t ws_bytes,
                                uint16_t *out, void *stream) {
    if (!q || !k_cache || !v_cache || !seq_lens || !workspace || !out) return TBQ4_ERR_NULL;
    if (!aligned(q, 16) || !aligned(k_cache, 16) || !aligned(v_cache, 16) ||
        !aligned(workspace, kWsAlign) || !aligned(out, 2) || !aligned(seq_lens, 4))
        return TBQ4_ERR_ALIGN;
    if (B <= 0 || B > 65535 || Hkv <= 0 || Hkv > 65535 || Hq <= 0 || Hq % Hkv != 0 ||
        Hq / Hkv > kMaxGroup || max_len < 0 || q_len < 1 || q_len > dmq::kMaxQLen ||
        (Hq / Hkv) * q_len > dmq::kCols || (int64_t)B * q_len > 65535)
        return TBQ4_ERR_SHAPE;
    if (capacity <= 0 || capacity % 8 != 0 || (int64_t)max_len > capacity)
        return TBQ4_ERR_CAPACITY;
    if (!std::isfinite(softmax_scale)) return TBQ4_ERR_SHAPE;
    if (q_len == 1)       // one query token: the single-query kernel, same result
        return decode_impl(q, k_cache, v_cache, seq_lens, max_len, B, Hq, Hkv, capacity,
                           softmax_scale, sign_seed, 0, workspace, ws_bytes, out, stream,
                           nullptr, nullptr);
    AttnParams p = {};
    p.q = q;
    p.k = k_cache;
    p.v = v_cache;
    p.head_stride = capacity * kBlockBytes;
    p.seq_stride = (int64_t)Hkv * p.head_stride;
    p.seq_lens = seq_lens;
    p.max_len = max_len;
    p.capacity = capacity;
    p.nseq = B;
    p.q_len = q_len;
    p.Hq = Hq;
    p.Hkv = Hkv;
    p.G = Hq / Hkv;
    p.split_tokens = auto_split_tokens(B, Hkv, max_len);
    p.scale_log2 = softmax_scale * 1.4426950408889634f;
    sign_words(sign_seed, &p.sign_lo, &p.sign_hi);
    p.out = out;
    return run_attention(p, workspace, ws_bytes, (cudaStream_t)stream);
}

tbq4_status tbq4_attn_decode_append(const float *q, const float *k_new, const float *v_new,
                                    uint8_t *k_cache, uint8_t *v_cache, const int32_t *seq_lens,
                                    int32_t max_len, int B, int Hq, int Hkv, int64_t capacity,
                                    float softmax_scale, uint64_t sign_seed, void *workspace,
                                    size_t ws_bytes, uint16_t *out, void *stream) {
    if (!k_new || !v_new) return TBQ4_ERR_NULL;
    if (!aligned(k_new, 16) || !aligned(v_new, 16)) return TBQ4_ERR_ALIGN;
    return decode_impl(q, k_cache, v_cache, seq_lens, max_len, B, Hq, Hkv, capacity,
                       softmax_scale, sign_seed, 0, workspace, ws_bytes, out, stream, k_new,
                       v_new);
}

tbq4_status tbq4_attn_decode_paged(const float *q, const float *k_new, const float *v_new,
                                   uint8_t *k_pool, uint8_t *v_pool, const int32_t *block_table,
                                   int max_pages, int page_size, int64_t n_pages,
                                   const int32_t *seq_lens, int32_t max_len, int B, int Hq,
                                   int Hkv, float softmax_scale, uint64_t sign_seed,
                                   void *workspace, size_t ws_bytes, uint16_t *out,
                                   void *stream) {
    if ((k_new == nullptr) != (v_new == nullptr)) return TBQ4_ERR_NULL;
    if (k_new && (!aligned(k_new, 16) || !aligned(v_new, 16))) return TBQ4_ERR_ALIGN;
    const PagedArgs pg = {block_table, max_pages, page_size, n_pages};
    return decode_impl(q, k_pool, v_pool, seq_lens, max_len, B, Hq, Hkv, 0, softmax_scale,
                       sign_seed, 0, workspace, ws_bytes, out, stream, k_new, v_new, &pg);
}

tbq4_status tbq3_attn_decode(const float *q, const uint8_t *k_cache, const uint8_t *v_cache,
                             const int32_t *seq_lens, int32_t max_len, int B, int Hq, int Hkv,
                             int64_t capacity, float softmax_scale, uint64_t sign_seed,
                             void *workspace, size_t ws_bytes, uint16_t *out, void *stream) {
    return decode_impl(q, k_cache, v_cache, seq_lens, max_len, B, Hq, Hkv, capacity,
                       softmax_scale, sign_seed, 0, workspace, ws_bytes, out, stream, nullptr,
                       nullptr, nullptr, 3);
}

tbq4_status tbq4_attn_decode(const float *q, const uint8_t *k_cache,
                             const uint8_t *v_cache, const int32_t *seq_lens,
                             int32_t max_len, int B, int Hq, int Hkv, int64_t capacity,
                             float softmax_scale, uint64_t sign_seed, void *workspace,
                             size_t ws_bytes, uint16_t *out, void *stream) {
    return tbq4_attn_decode_split(q, k_cache, v_cache, seq_lens, max_len, B, Hq, Hkv,
                                  capacity, softmax_scale, sign_seed, 0, workspace,
                                  ws_bytes, out, stream);
}

tbq4_status tbq4_attn_decode_noalloc(const float *q, const uint8_t *k_cache,
                                     const uint8_t *v_cache, const int32_t *seq_lens,
                                     int32_t max_len, int B, int Hq, int Hkv, int64_t capacity,
                                     float softmax_scale, uint64_t sign_seed, uint16_t *out,
                                     void *stream) {
    const size_t need = tbq4_decode_workspace_bytes(B, Hq, Hkv, max_len);
    if (need > kNoAllocScratchBytes) return TBQ4_ERR_WORKSPACE;
    void *scratch = nullptr;
    const tbq4_status st = noalloc_scratch(&scratch);
    if (st != TBQ4_OK) return st;
    return tbq4_attn_decode(q, k_cache, v_cache, seq_lens, max_len, B, Hq, Hkv, capacity,
                            softmax_scale, sign_seed, scratch, kNoAllocScratchBytes, out,
                            stream);
}

size_t tbq4_prefill_workspace_bytes(int n_new, int Hq, int Hkv, int64_t n_cached) {
    if (n_new <= 0 || Hq <= 0 || Hkv <= 0 || n_cached < 0 || Hq % Hkv != 0) return 0;
    return prefill_ws_layout(n_new, Hq, Hkv, n_cached).total;
}

tbq4_status tbq4_attn_prefill_chunk(const uint16_t *q, int n_new, int64_t n_cached,
                                    const uint8_t *k_cache, const uint8_t *v_cache,
                                    int Hq, int Hkv, int64_t capacity,
                                    float softmax_scale, uint64_t sign_seed,
                                    void *workspace, size_t ws_bytes, uint16_t *out,
                                    void *stream) {
    const NvtxRange range("tbq4_attn_prefill_chunk");
    if (!q || !k_cache || !v_cache || !workspace || !out) return TBQ4_ERR_NULL;
    if (!aligned(q, 16) || !aligned(k_cache, 16) || !aligned(v_cache, 16) ||
        !aligned(workspace, kWsAlign) || !aligned(out, 2))
        return TBQ4_ERR_ALIGN;
    if (n_new <= 0 || n_new > 65535 || Hkv <= 0 || Hq <= 0 || Hq % Hkv != 0 ||
        Hq / Hkv > kMaxGroup || n_cached < 0)
        return TBQ4_ERR_SHAPE;
    if (capacity <= 0 || capacity % 8 != 0 || n_cached + n_new > capacity ||
        n_cached + n_new > INT32_MAX)
        return TBQ4_ERR_CAPACITY;
    if (!std::isfinite(softmax_scale)) return TBQ4_ERR_SHAPE;
    const PrefillPlan w = prefill_ws_layout(n_new, Hq, Hkv, n_cached);
    if (ws_bytes < w.total) return TBQ4_ERR_WORKSPACE;
    static bool attr_set[64] = {};
    if (!ensure_smem_attr((const void *)pre::prefill_tc_kernel, pre::kSmemBytes, attr_set))
        return TBQ4_ERR_LAUNCH;
    // The kernel moves registers between its warpgroups (setmaxnreg); that is
    // only safe when it was compiled with at least pre::kMinLaunchRegs.
    static int regs_ok = -1;
    if (regs_ok < 0) {
        cudaFuncAttributes fa;
        regs_ok = cudaFuncGetAttributes(&fa, pre::prefill_tc_kernel) == cudaSuccess &&
                  fa.numRegs >= pre::kMinLaunchRegs && fa.numRegs * pre::kThreads <= 65536;
    }
    if (!regs_ok) return TBQ4_ERR_LAUNCH;
    cudaStream_t st = (cudaStream_t)stream;
    uint64_t lo, hi;
    sign_words(sign_seed, &lo, &hi);
    pre::PrefillParams pp = {};
    pp.q = q;
    pp.k = k_cache;
    pp.v = v_cache;
    pp.head_stride = capacity * kBlockBytes;
    pp.n_new = n_new;
    pp.n_cached = n_cached;
    pp.Hq = Hq;
    pp.Hkv = Hkv;
    pp.G = Hq / Hkv;
    pp.pairs = w.pairs;
    pp.iblocks = w.iblocks;
    pp.n_splits = w.n_splits;
    pp.scale_log2_15 = softmax_scale * 1.4426950408889634f / 15.0f;
    pp.sign_lo = lo;
    pp.sign_hi = hi;
    pp.part_o = reinterpret_cast<float *>(static_cast<char *>(workspace) + w.part_o);
    pp.part_ml = reinterpret_cast<float2 *>(static_cast<char *>(workspace) + w.part_ml);
    pp.cache_bytes = (int64_t)Hkv * pp.head_stride;
    pp.part_rows = (int64_t)n_new * Hq * w.n_splits;
    if (g_ev_before) cudaEventRecord(g_ev_before, st);
    pre::prefill_tc_kernel<<<dim3(w.n_splits, w.mpairs), pre::kThreads, pre::kSmemBytes, st>>>(pp);
    if (g_ev_after) cudaEventRecord(g_ev_after, st);

    AttnParams c = {};
    c.seq_lens = nullptr;
    c.len_base = (int32_t)(n_cached + 1);
    c.max_len = (int32_t)(n_cached + n_new);
    c.capacity = capacity;
    c.nseq = n_new;
    c.Hq = Hq;
    c.Hkv = Hkv;
    c.G = Hq / Hkv;
    c.split_tokens = 1;
    c.n_splits = w.n_splits;
    c.all_splits = 1;
    c.sign_lo = lo;
    c.sign_hi = hi;
    c.part_o = pp.part_o;
    c.part_ml = pp.part_ml;
    c.out = out;
    c.out_bf16 = 1;
    c.part_rows = pp.part_rows;
    c.out_elems = (int64_t)n_new * Hq * kD;
    // one warp per (position, head) row, a programmatic dependent launch
    const int n_rows = n_new * Hq;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)((n_rows + kCombineWarps - 1) / kCombineWarps));
    cfg.blockDim = dim3(kCombineWarps * 32);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaLaunchKernelEx(&cfg, combine_rows_kernel, c, n_rows) != cudaSuccess)
        return TBQ4_ERR_LAUNCH;
    return launch_status();
}

void tbq4_set_timing_events(void *before, void *after) {
    g_ev_before = (cudaEvent_t)before;
    g_ev_after = (cudaEvent_t)after;
}

tbq4_status tbq4_get_device_status(void *stream) {
    if (cudaStreamSynchronize((cudaStream_t)stream) != cudaSuccess) return TBQ4_ERR_LAUNCH;
    unsigned v = 0;
    if (cudaMemcpyFromSymbol(&v, g_status, sizeof(v)) != cudaSuccess) return TBQ4_ERR_LAUNCH;
    if (v != 0) {
        const unsigned zero = 0;
        if (cudaMemcpyToSymbol(g_status, &zero, sizeof(zero)) != cudaSuccess)
            return TBQ4_ERR_LAUNCH;
    }
    return (tbq4_status)v;
}

tbq4_status tbq4_selftest_bounded_wait(uint32_t polls, void *stream) {
    if (polls == 0 || polls > (1u << 16)) return TBQ4_ERR_SHAPE;
    bounded_wait_selftest_kernel<<<1, 32, 0, (cudaStream_t)stream>>>(polls);
    return launch_status();
}

const char *tbq4_status_string(tbq4_status s) {
    switch (s) {
        case TBQ4_OK: return "ok";
        case TBQ4_ERR_NULL: return "a required pointer is NULL";
        case TBQ4_ERR_ALIGN: return "a pointer is not suitably aligned";
        case TBQ4_ERR_SHAPE: return "unsupported sizes or arguments";
        case TBQ4_ERR_CAPACITY: return "position or length outside the cache capacity";
        case TBQ4_ERR_WORKSPACE: return "workspace smaller than required";
        case TBQ4_ERR_LAUNCH: return "a CUDA launch or query failed";
        case TBQ4_ERR_DEVICE_TIMEOUT: return "a bounded wait inside a kernel gave up";
        case TBQ4_ERR_BOUNDS: return "a bounds check of the debug build failed";
    }
    return "unknown status";
}

}  // extern "C"

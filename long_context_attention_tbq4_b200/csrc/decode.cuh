// decode.cuh -- parameters shared by the attention kernels, and the
// log-sum-exp combine of split partials that applies the inverse rotation.
//
// The attention runs in the rotated domain (trefon.com, "Kontekst 262K na
// jednej RTX 4090", section "Od czego zaczalem"): q is rotated once per
// CTA, every K/V block is dequantised in the inner loop straight from the
// raw bytes, and each output row is rotated back once, here.
//
// Level arithmetic.  A block dequantises to (S/15) * L with L = 2*index-15,
// an odd integer in [-15, 15].  The per-token factor S/15 is applied to the
// score (K) and to the softmax weight (V), never per element.
#pragma once
#include "common.cuh"

namespace tbq4 {

struct AttnParams {
    const void *q;              // [nseq][Hq][128], fp32 or bf16
    int q_bf16;
    const uint8_t *k;           // cache base
    const uint8_t *v;
    int64_t seq_stride;         // bytes between sequences (0: shared cache)
    int64_t head_stride;        // bytes between KV heads (capacity * 66)
    const int32_t *seq_lens;    // [nseq] or nullptr: len = len_base + seq
    int32_t len_base;
    int32_t max_len;            // upper bound of every length
    int64_t capacity;
    int nseq, Hq, Hkv, G;
    int split_tokens, n_splits;
    float scale_log2;           // softmax_scale * log2(e)
    uint64_t sign_lo, sign_hi;
    float *part_o;              // [nseq][Hq][n_splits][128]
    float2 *part_ml;            // [nseq][Hq][n_splits]  (max in log2 units, sum)
    void *out;                  // [nseq][Hq][128], fp16 or bf16
    int out_bf16;
    int all_splits;             // combine every split (prefill) instead of ceil(len/split)
    // Multi-query decode: query tokens per sequence (0 or 1: one).  The
    // combine's rows are then (sequence, query token) pairs, b * q_len + i.
    int q_len;
    // Fused append (decode step): the current token's K and V rows, fp32
    // [nseq][Hkv][128], encoded into the caches at position len - 1 by the
    // CTA that streams that position.  nullptr: no append.
    const float *k_new;
    const float *v_new;
    uint8_t *k_wr;              // the same caches as k / v, written
    uint8_t *v_wr;
    // Paged caches: k and v are pools [n_pages][Hkv][page_size][66] and
    // token t of sequence s lives in page block_table[s][t / page_size], row
    // t % page_size.  nullptr: contiguous caches (seq_stride, head_stride).
    const int32_t *block_table;
    int max_pages;              // row length of block_table
    int page_size;              // tokens per page, a multiple of 32
    int64_t n_pages;
    int tbq3;                   // 1: 3-bit caches [..][50] (decode only)
    // Extents, for the debug build's bounds checks: bytes of each of the K
    // and V caches (or pools), entries of part_ml (part_o holds 128 floats
    // per entry), elements of out.
    int64_t cache_bytes, part_rows, out_elems;
};

// Byte offset of token t of (sequence s, KV head g) in a paged pool.  An
// out-of-range page id reads page 0 instead (so no access leaves the pool);
// *bad reports it, for the caller to flag when the token is a real one.
__device__ __forceinline__ int64_t paged_offset(const AttnParams &p, int32_t pid, int g, int32_t t,
                                                bool *bad) {
    *bad = pid < 0 || (int64_t)pid >= p.n_pages;
    if (*bad) pid = 0;
    return (((int64_t)pid * p.Hkv + g) * p.page_size + t % p.page_size) * kBlockBytes;
}

__device__ __forceinline__ int32_t page_id(const AttnParams &p, int s, int32_t t) {
    return __ldg(p.block_table + (int64_t)s * p.max_pages + t / p.page_size);
}

__device__ __forceinline__ int32_t seq_length(const AttnParams &p, int s) {
    int32_t len = p.seq_lens ? __ldg(p.seq_lens + s) : p.len_base + s;
    const int64_t lim = p.capacity < (int64_t)p.max_len ? p.capacity : (int64_t)p.max_len;
    if (len < 0 || (int64_t)len > lim) {
        record_status(4u /* TBQ4_ERR_CAPACITY */);
        len = len < 0 ? 0 : (int32_t)lim;
    }
    return len;
}

__device__ __forceinline__ float load_q(const AttnParams &p, int64_t idx) {
    if (p.q_bf16)
        return __bfloat162float(__ushort_as_bfloat16(
            reinterpret_cast<const uint16_t *>(p.q)[idx]));
    return reinterpret_cast<const float *>(p.q)[idx];
}

// Log-sum-exp merge of the split partials of one output row (log2 units).
// A warp takes splits sub, sub + nsub, ... with a running max (independent
// loads, no dependent chain over all splits); each lane owns four dimensions
// (one float4).  Partials are read from L2 (.cg).
__device__ __forceinline__ void merge_split_run(const AttnParams &p, int64_t row0, int used,
                                                int sub, int nsub, int lane, float4 &O,
                                                float &M, float &L) {
    M = -INFINITY;
    L = 0.f;
    O = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 4
    for (int i = sub; i < used; i += nsub) {
        const float2 ml = __ldcg(p.part_ml + row0 + i);
        const float4 oi = __ldcg(reinterpret_cast<const float4 *>(p.part_o + (row0 + i) * kD) + lane);
        if (ml.x == -INFINITY) continue;                  // empty split
        const float Mn = fmaxf(M, ml.x);
        const float a = M == -INFINITY ? 0.f : exp2f(M - Mn);
        const float b = exp2f(ml.x - Mn);
        O.x = O.x * a + oi.x * b;
        O.y = O.y * a + oi.y * b;
        O.z = O.z * a + oi.z * b;
        O.w = O.w * a + oi.w * b;
        L = L * a + ml.y * b;
        M = Mn;
    }
}

// o = D H o_rot / sqrt(128) for a normalised row held as a float4 per lane,
// rounded to fp16 or bf16 and stored.
__device__ __forceinline__ void store_row(const AttnParams &p, int s, int h, float (&v)[4],
                                          int lane);

// Merges the nsub per-warp results of one output row (in shared memory),
// normalises, applies o = D H o_rot / sqrt(128) (H is symmetric, so R^T = D H
// c) with the same shuffle transform as q, and rounds to fp16 or bf16.
__device__ __forceinline__ void finish_row(const AttnParams &p, int s, int h, const float4 *o_s,
                                           const float *m_s, const float *l_s, int nsub,
                                           int lane) {
    float Mt = -INFINITY;
    for (int w = 0; w < nsub; ++w) Mt = fmaxf(Mt, m_s[w]);
    float v[4] = {0.f, 0.f, 0.f, 0.f}, Lt = 0.f;
    if (Mt != -INFINITY) {
        for (int w = 0; w < nsub; ++w) {
            const float f = m_s[w] == -INFINITY ? 0.f : exp2f(m_s[w] - Mt);
            const float4 ow = o_s[32 * w + lane];
            v[0] += f * ow.x;
            v[1] += f * ow.y;
            v[2] += f * ow.z;
            v[3] += f * ow.w;
            Lt += f * l_s[w];
        }
    }
    const float inv = Lt > 0.f ? 1.0f / Lt : 0.f;
#pragma unroll
    for (int k = 0; k < 4; ++k) v[k] *= inv;
    store_row(p, s, h, v, lane);
}

__device__ __forceinline__ void store_row(const AttnParams &p, int s, int h, float (&v)[4],
                                          int lane) {
    // inverse rotation: transform, scale, then the sign diagonal
    warp_fwht128(v, lane);
    const uint32_t sbits = lane_sign_bits(p.sign_lo, p.sign_hi, lane);
    const float c = rot_c();
    const int64_t oi = ((int64_t)s * p.Hq + h) * kD + 4 * lane;
    if (!in_extent(oi, 4, p.out_elems)) return;
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        float x = v[k] * c;
        if ((sbits >> k) & 1u) x = -x;
        if (p.out_bf16)
            reinterpret_cast<__nv_bfloat16 *>(p.out)[oi + k] = __float2bfloat16_rn(x);
        else
            reinterpret_cast<__half *>(p.out)[oi + k] = __float2half_rn(x);
    }
}

__device__ __forceinline__ int used_splits(const AttnParams &p, int32_t len) {
    return p.all_splits ? p.n_splits : (len + p.split_tokens - 1) / p.split_tokens;
}

// One CTA per (sequence, query head), sixteen warps.  Up to 64 splits: every
// partial row (a float4 per lane, warp w takes splits w, w + 16, ...) and
// every (m, l) is loaded at once, so the merge costs one round of L2
// latency; the weights 2^(m_i - M) and the sum L come from block
// reductions, the weighted rows are summed per warp and then across warps,
// and warp 0 writes the output row.  More splits: a running merge per warp.
constexpr int kCombineWarps = 16;
constexpr int kCombineFast = 4;                 // splits per warp on the fast path

__global__ void __launch_bounds__(kCombineWarps * 32)
decode_combine_kernel(const AttnParams p) {
    __shared__ float4 o_s[kCombineWarps * 32];
    __shared__ float m_s[kCombineWarps], l_s[kCombineWarps];
    __shared__ float w_s[kCombineWarps * kCombineFast];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int h = blockIdx.x, s = blockIdx.y;
    // The lengths are an input of the split kernel, not one of its results,
    // so they are read before the wait and only the partials' loads follow it.
    const int32_t len = seq_length(p, p.q_len > 1 ? s / p.q_len : s);
    const int64_t row0 = ((int64_t)s * p.Hq + h) * p.n_splits;
    int used = used_splits(p, len);
    if (!in_extent(row0, used, p.part_rows)) used = 0;
    // Launched as a programmatic dependent of the split kernel: wait for all
    // of its partials (a no-op under an ordinary launch).  Then the next
    // decode step's split kernel may start: its caches were complete before
    // this wait returned, and it reads its own inputs and writes the
    // workspace only after its own wait, i.e. after this grid has finished.
    asm volatile("griddepcontrol.wait;" ::: "memory");
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

    if (used > kCombineWarps * kCombineFast) {
        float4 O;
        float M, L;
        merge_split_run(p, row0, used, warp, kCombineWarps, lane, O, M, L);
        o_s[32 * warp + lane] = O;
        if (lane == 0) { m_s[warp] = M; l_s[warp] = L; }
        __syncthreads();
        if (warp == 0) finish_row(p, s, h, o_s, m_s, l_s, kCombineWarps, lane);
        return;
    }
    // all loads first
    float4 x[kCombineFast];
#pragma unroll
    for (int k = 0; k < kCombineFast; ++k) {
        const int i = warp + kCombineWarps * k;
        x[k] = i < used ? __ldcg(reinterpret_cast<const float4 *>(p.part_o + (row0 + i) * kD) + lane)
                        : make_float4(0.f, 0.f, 0.f, 0.f);
    }
    float2 ml = make_float2(-INFINITY, 0.f);
    if (tid < used) ml = __ldcg(p.part_ml + row0 + tid);
    // M = max_i m_i
    float mx = warp_max(ml.x);
    if (lane == 0) m_s[warp] = mx;
    __syncthreads();
    float M = m_s[0];
#pragma unroll
    for (int w = 1; w < kCombineWarps; ++w) M = fmaxf(M, m_s[w]);
    // weights and L = sum_i w_i l_i
    const float wt = (ml.x == -INFINITY || M == -INFINITY) ? 0.f : exp2f(ml.x - M);
    if (tid < used) w_s[tid] = wt;
    const float lw = warp_sum(wt * ml.y);
    if (lane == 0) l_s[warp] = lw;
    __syncthreads();
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int k = 0; k < kCombineFast; ++k) {
        const int i = warp + kCombineWarps * k;
        if (i < used) {
            const float w = w_s[i];
            acc.x = fmaf(w, x[k].x, acc.x);
            acc.y = fmaf(w, x[k].y, acc.y);
            acc.z = fmaf(w, x[k].z, acc.z);
            acc.w = fmaf(w, x[k].w, acc.w);
        }
    }
    o_s[32 * warp + lane] = acc;
    __syncthreads();
    if (warp == 0) {
        float v[4] = {0.f, 0.f, 0.f, 0.f}, L = 0.f;
        for (int w = 0; w < kCombineWarps; ++w) {
            const float4 a = o_s[32 * w + lane];
            v[0] += a.x; v[1] += a.y; v[2] += a.z; v[3] += a.w;
            L += l_s[w];
        }
        const float inv = L > 0.f ? 1.0f / L : 0.f;
#pragma unroll
        for (int k = 0; k < 4; ++k) v[k] *= inv;
        store_row(p, s, h, v, lane);
    }
}


// The same merge with one warp per output row (sequence or query position
// s, query head h): for few splits per row and many rows, as in the chunked
// prefill (a few key splits for each of n_new x Hq rows), where a 16-warp
// CTA per row would mostly idle.  Each warp runs the log-sum-exp merge over
// its row's splits, normalises, rotates back and stores.  Launched as a
// programmatic dependent of the attention kernel.
__global__ void __launch_bounds__(kCombineWarps * 32)
combine_rows_kernel(const AttnParams p, int n_rows) {
    asm volatile("griddepcontrol.wait;" ::: "memory");
    const int lane = threadIdx.x & 31;
    const int rowid = blockIdx.x * kCombineWarps + (threadIdx.x >> 5);
    if (rowid >= n_rows) return;
    const int s = rowid / p.Hq, h = rowid - (rowid / p.Hq) * p.Hq;
    const int64_t row0 = ((int64_t)s * p.Hq + h) * p.n_splits;
    int used = used_splits(p, seq_length(p, s));
    if (!in_extent(row0, used, p.part_rows)) used = 0;
    float4 O;
    float M, L;
    merge_split_run(p, row0, used, 0, 1, lane, O, M, L);
    const float inv = L > 0.f ? 1.0f / L : 0.f;
    float v[4] = {O.x * inv, O.y * inv, O.z * inv, O.w * inv};
    store_row(p, s, h, v, lane);
}

}  // namespace tbq4

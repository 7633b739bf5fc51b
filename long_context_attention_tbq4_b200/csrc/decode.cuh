// decode.cuh -- split-K flash-decode over TBQ4 caches, and the log-sum-exp
// combine that applies the inverse rotation.
//
// The attention runs in the rotated domain (trefon.com, "Kontekst 262K na
// jednej RTX 4090", section "Od czego zaczalem"): q is rotated once per
// CTA, every K/V block is dequantised in the inner loop straight from the
// raw bytes, and the output row is rotated back once, in the combine.
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
};

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

// One CTA = one (sequence, KV head, split).  Four warps take interleaved
// tokens of the split; each lane owns four dimensions; the G query heads of
// the KV head share every dequantised block.
constexpr int kSplitWarps = 4;

__global__ void __launch_bounds__(kSplitWarps * 32)
decode_split_kernel(const AttnParams p) {
    __shared__ float q_s[kMaxGroup][kD];
    __shared__ float m_w[kSplitWarps][kMaxGroup], l_w[kSplitWarps][kMaxGroup];
    __shared__ float o_w[kSplitWarps][kMaxGroup][kD];

    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int split = blockIdx.x, g = blockIdx.y, s = blockIdx.z;
    const int G = p.G;
    const int32_t len = seq_length(p, s);
    const int32_t t0 = split * p.split_tokens;
    const int32_t t1 = min(len, t0 + p.split_tokens);

    // q_rot * softmax_scale * log2(e) / 15, one head per warp.
    const uint32_t sbits = lane_sign_bits(p.sign_lo, p.sign_hi, lane);
    for (int hh = warp; hh < G; hh += kSplitWarps) {
        const int64_t base = ((int64_t)s * p.Hq + g * G + hh) * kD + 4 * lane;
        float v[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) v[k] = load_q(p, base + k);
        warp_rotate128(v, sbits, lane);
        const float f = p.scale_log2 * (1.0f / 15.0f);
#pragma unroll
        for (int k = 0; k < 4; ++k) q_s[hh][4 * lane + k] = v[k] * f;
    }
    __syncthreads();

    float qr[kMaxGroup][4], m[kMaxGroup], l[kMaxGroup], o[kMaxGroup][4];
#pragma unroll
    for (int h = 0; h < kMaxGroup; ++h) {
        m[h] = -INFINITY;
        l[h] = 0.f;
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            qr[h][k] = h < G ? q_s[h][4 * lane + k] : 0.f;
            o[h][k] = 0.f;
        }
    }

    const uint8_t *kb = p.k + s * p.seq_stride + g * p.head_stride;
    const uint8_t *vb = p.v + s * p.seq_stride + g * p.head_stride;
    for (int32_t t = t0 + warp; t < t1; t += kSplitWarps) {
        const uint8_t *kr = kb + (int64_t)t * kBlockBytes;
        const uint8_t *vr = vb + (int64_t)t * kBlockBytes;
        const uint32_t kn = __ldg(reinterpret_cast<const uint16_t *>(kr + 2) + lane);
        const uint32_t vn = __ldg(reinterpret_cast<const uint16_t *>(vr + 2) + lane);
        const float sk = half_bits_to_float(__ldg(reinterpret_cast<const uint16_t *>(kr)));
        const float sv = half_bits_to_float(__ldg(reinterpret_cast<const uint16_t *>(vr)))
                         * (1.0f / 15.0f);
        float lk[4], lv[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            lk[k] = (float)(2 * (int)((kn >> (4 * k)) & 15u) - 15);
            lv[k] = (float)(2 * (int)((vn >> (4 * k)) & 15u) - 15);
        }
#pragma unroll
        for (int h = 0; h < kMaxGroup; ++h) {
            if (h >= G) break;
            float d = qr[h][0] * lk[0] + qr[h][1] * lk[1] + qr[h][2] * lk[2] + qr[h][3] * lk[3];
            d = warp_sum(d) * sk;
            const float mn = fmaxf(m[h], d);
            const float corr = exp2f(m[h] - mn);
            const float pr = exp2f(d - mn);
            l[h] = l[h] * corr + pr;
            const float pv = pr * sv;
#pragma unroll
            for (int k = 0; k < 4; ++k) o[h][k] = o[h][k] * corr + pv * lv[k];
            m[h] = mn;
        }
    }

    // Merge the four warps, then write this split's partial.
#pragma unroll
    for (int h = 0; h < kMaxGroup; ++h) {
        if (h >= G) break;
        if (lane == 0) { m_w[warp][h] = m[h]; l_w[warp][h] = l[h]; }
#pragma unroll
        for (int k = 0; k < 4; ++k) o_w[warp][h][4 * lane + k] = o[h][k];
    }
    __syncthreads();
    const int d = threadIdx.x;
    for (int h = 0; h < G; ++h) {
        float M = -INFINITY;
#pragma unroll
        for (int w = 0; w < kSplitWarps; ++w) M = fmaxf(M, m_w[w][h]);
        float O = 0.f, L = 0.f;
        if (M != -INFINITY) {
#pragma unroll
            for (int w = 0; w < kSplitWarps; ++w) {
                const float mw = m_w[w][h];
                const float f = mw == -INFINITY ? 0.f : exp2f(mw - M);
                O += f * o_w[w][h][d];
                L += f * l_w[w][h];
            }
        }
        const int64_t row = ((int64_t)s * p.Hq + g * G + h) * p.n_splits + split;
        p.part_o[row * kD + d] = O;
        if (d == 0) p.part_ml[row] = make_float2(M, L);
    }
}

// One CTA of 128 threads per (sequence, query head): merge the splits by
// log-sum-exp, then o = D H o_rot / sqrt(128) (H symmetric, so R^T = D H c)
// and round to fp16 or bf16.
__global__ void __launch_bounds__(kD)
decode_combine_kernel(const AttnParams p) {
    __shared__ float x_s[kD];
    const int d = threadIdx.x, lane = d & 31;
    const int h = blockIdx.x, s = blockIdx.y;
    const int32_t len = seq_length(p, s);
    const int used = (len + p.split_tokens - 1) / p.split_tokens;
    const int64_t row0 = ((int64_t)s * p.Hq + h) * p.n_splits;

    float M = -INFINITY;
    for (int i = 0; i < used; ++i) M = fmaxf(M, p.part_ml[row0 + i].x);
    float O = 0.f, L = 0.f;
    if (M != -INFINITY) {
        for (int i = 0; i < used; ++i) {
            const float2 ml = p.part_ml[row0 + i];
            const float f = ml.x == -INFINITY ? 0.f : exp2f(ml.x - M);
            O += f * p.part_o[(row0 + i) * kD + d];
            L += f * ml.y;
        }
    }
    float x = L > 0.f ? O / L : 0.f;

    // Walsh-Hadamard transform across the 128 threads.
#pragma unroll
    for (int m = 1; m < 32; m <<= 1) {
        const float o = __shfl_xor_sync(kFull, x, m);
        x = (lane & m) ? o - x : x + o;
    }
#pragma unroll
    for (int m = 32; m < kD; m <<= 1) {
        x_s[d] = x;
        __syncthreads();
        const float o = x_s[d ^ m];
        __syncthreads();
        x = (d & m) ? o - x : x + o;
    }
    const uint64_t w = d < 64 ? p.sign_lo : p.sign_hi;
    x *= rot_c();
    if ((w >> (d & 63)) & 1u) x = -x;
    const int64_t oi = ((int64_t)s * p.Hq + h) * kD + d;
    if (p.out_bf16)
        reinterpret_cast<__nv_bfloat16 *>(p.out)[oi] = __float2bfloat16_rn(x);
    else
        reinterpret_cast<__half *>(p.out)[oi] = __float2half_rn(x);
}

}  // namespace tbq4

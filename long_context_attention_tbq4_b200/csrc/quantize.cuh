// quantize.cuh -- TBQ4 quantise-append: fp32 rows -> 66-byte blocks.
//
// Two encoders with the same op order, so the same bytes (the codebook's
// definition, see include/tbq4.h):
//   encode_row            one warp per row (four values per lane, the
//                         transform over shuffles); the decode kernel uses it
//                         to append the current token
//   quantize_rows_kernel  one thread per row, the transform in registers;
//                         the bulk append (HBM-bound: 512 bytes in, 66 out)
#pragma once
#include "common.cuh"
#include "mbarrier.cuh"

namespace tbq4 {

// Index of one rotated value against the block scale S:
// clamp(rne(fl32(fl32(x/S) * 7.5) + 7.5), 0, 15), and 8 when S == 0.
__device__ __forceinline__ uint32_t level_index(float x, float S) {
    if (S == 0.0f) return 8u;
    const float t = __fdiv_rn(x, S);
    const float u = __fmul_rn(t, 7.5f);
    const float v = __fadd_rn(u, 7.5f);
    float r = rintf(v);                       // round half to even
    r = fminf(fmaxf(r, 0.0f), 15.0f);
    return (uint32_t)r;
}

// Encodes four consecutive values per lane (one row per warp).  Returns the
// 16-bit pair of index bytes for this lane and writes the scale bits to *sb.
__device__ __forceinline__ uint32_t encode_row(float v[4], uint32_t sbits, int lane,
                                               uint16_t *sb) {
    warp_rotate128(v, sbits, lane);
    float m = fmaxf(fmaxf(fabsf(v[0]), fabsf(v[1])), fmaxf(fabsf(v[2]), fabsf(v[3])));
    m = warp_max(m);
    uint16_t s = __half_as_ushort(__float2half_rn(m));
    if ((s & 0x7FFFu) == 0x7C00u) s = 0x7BFFu;        // saturate at 65504
    *sb = s;
    const float S = half_bits_to_float(s);
    const uint32_t i0 = level_index(v[0], S), i1 = level_index(v[1], S);
    const uint32_t i2 = level_index(v[2], S), i3 = level_index(v[3], S);
    return i0 | (i1 << 4) | (i2 << 8) | (i3 << 12);
}

// The +-1 sign diagonal as floats, passed by value: a kernel parameter is a
// constant-bank operand, so the signs fold into the first butterfly stage.
struct SignTable {
    float s[kD];
};

// Bulk append: one thread encodes one whole 128-value row (rows are
// independent, so a thread per row keeps the transform in registers, with no
// shuffles):
//   rotation  the same butterflies in the same order as warp_fwht128 (stride
//             1 first; lower = a + b, upper = a - b, each rounded on its own).
//             The sign flip is exact, so the first stage is
//             fma(v_j, s_j, s_k v_k) and fma(v_j, s_j, -s_k v_k).
//   scale     S = fp16(max |x_rot|), saturated at 65504.
//   index     clamp(rne(fl32(fl32(x/S) * 7.5) + 7.5), 0, 15), 8 when S == 0.
//             The quotient is the correctly rounded x/S by Markstein's method:
//             r = RN(1/S) once per row, q0 = RN(x r), e = x - q0 S (exact with
//             FMA), q = RN(q0 + e r).  rint is an add of 1.5 * 2^23 on the
//             FMA pipe; the clamp is needed only for rows whose fp16 scale is
//             zero, subnormal or saturated, and is applied to x for those.
// Memory: rows go in groups of 32 in head-major order (row = (b Hkv + h)
// n_new + t), so a group's 32 blocks are contiguous in the cache.  One CTA
// of eight warps per SM, two warps per scheduler (so a thread can keep its
// row's 128 values in registers: a scheduler's register file is a quarter
// of the SM's).  Each warp owns one shared-memory stage: a group comes in as
// one 512-byte cp.async.bulk per row (rows 528 bytes apart, so the
// per-thread reads of a whole row are free of bank conflicts); once the
// rows are in registers the warp sends its next group's copies into the
// same stage, and they land while this group is encoded.  The blocks go out
// from a per-warp staging area as consecutive 16-bit pieces.
// Paged destination: row (b, pos) goes to page table[b][pos / page_size],
// row pos % page_size, of a pool [n_pages][Hkv][page_size][66].  A null
// table means the contiguous cache [B][Hkv][capacity][66].
struct PageMap {
    const int32_t *table;
    int max_pages, page_size;
    int64_t n_pages;
};

// The 3-bit variant (TBQ3): the same rotation and scale, 8 levels
// (i - 3.5)/3.5 * S, index clamp(rne(fl32(fl32(x/S)*3.5)+3.5), 0, 7) (4 when
// S == 0), indices 8g .. 8g+7 as one little-endian 24-bit word (index 8g+k
// at bits 3k .. 3k+2): 2 + 48 = 50 bytes per block.
constexpr int kBlockBytes3 = 50;

constexpr int kQRows = 32;                                   // rows per group
constexpr int kQWarps = 8;                                   // warps per CTA
constexpr int kQRowStride = 512 + 16;                        // bytes between staged rows
constexpr int kQStageBytes = kQRows * kQRowStride;
constexpr int kQOutBytes = kQRows * kBlockBytes + kQRows * 8;   // blocks + destinations
constexpr int kQThreads = kQWarps * 32;
constexpr int kQRingBytes = kQWarps * kQStageBytes;
constexpr int kQSmemBytes = kQRingBytes + kQWarps * kQOutBytes + kQWarps * 8;
static_assert(kQSmemBytes <= 227 * 1024, "shared memory per CTA");
static_assert(kQStageBytes % 16 == 0 && kQRowStride % 16 == 0 && kQOutBytes % 16 == 0,
              "bulk copies and staged rows stay 16-byte aligned");

// kBits: 4 (TBQ4, 66-byte blocks) or 3 (TBQ3, 50-byte blocks).  Group k of a
// CTA is group blockIdx.x + k gridDim.x, encoded by warp k % kQWarps.
template <int kBits>
__global__ void __launch_bounds__(kQThreads, 1)
quantize_rows_kernel(const float *__restrict__ src, int B, int n_new, int Hkv,
                     const int32_t *__restrict__ start_pos, int64_t capacity, const SignTable sg,
                     const PageMap pm, uint8_t *__restrict__ cache) {
    extern __shared__ __align__(128) uint8_t qsm[];
    constexpr int kBlk = kBits == 4 ? kBlockBytes : kBlockBytes3;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const uint32_t rows = (uint32_t)B * (uint32_t)n_new * (uint32_t)Hkv;    // < 2^31 (host)
    const uint32_t groups = (rows + kQRows - 1) / kQRows;
    const uint32_t bar = smem_u32(qsm + kQRingBytes + kQWarps * kQOutBytes) + 8 * warp;
    uint8_t *stg = qsm + warp * kQStageBytes;
    uint8_t *wout = qsm + kQRingBytes + warp * kQOutBytes;
    uint16_t *stage = reinterpret_cast<uint16_t *>(wout);                      // [32][kBlk/2]
    int64_t *doffs = reinterpret_cast<int64_t *>(wout + kQRows * kBlockBytes);  // [32]
    // the 32 rows of group gi into this warp's stage, one bulk copy per lane
    // (tail lanes repeat the last row; nothing of theirs is stored)
    auto load_group = [&](uint32_t gi) {
        const uint32_t r = min(gi * kQRows + lane, rows - 1);
        const uint32_t t = r % (uint32_t)n_new, bh = r / (uint32_t)n_new;
        const uint32_t h = bh % (uint32_t)Hkv, b = bh / (uint32_t)Hkv;
        const float *srow = src + (((int64_t)b * n_new + t) * Hkv + h) * kD;
        if (lane == 0) mbar_expect_tx(bar, kQRows * 512);
        __syncwarp();
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        bulk_g2s(smem_u32(stg + lane * kQRowStride), srow, 512, bar);
    };
    if (lane == 0) {
        mbar_init(bar, 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    __syncwarp();
    uint32_t gi = blockIdx.x + warp * gridDim.x;
    if (gi < groups) load_group(gi);
    for (uint32_t phase = 0; gi < groups; phase ^= 1u) {
        const uint32_t gnext = gi + kQWarps * gridDim.x;
        // this lane's row and its destination, while the rows load
        const uint32_t r = gi * kQRows + lane;
        const bool live = r < rows;
        int64_t doff = -1;          // -1: nothing stored (tail lane or bad position)
        if (live) {
            const uint32_t t = r % (uint32_t)n_new, bh = r / (uint32_t)n_new;
            const uint32_t h = bh % (uint32_t)Hkv, b = bh / (uint32_t)Hkv;
            const int64_t pos = (int64_t)__ldg(start_pos + b) + t;
            if (pos < 0 || pos >= capacity) {
                record_status(4u /* TBQ4_ERR_CAPACITY */);
            } else if (pm.table) {
                const int32_t pid = __ldg(pm.table + (int64_t)b * pm.max_pages + pos / pm.page_size);
                if (pid < 0 || (int64_t)pid >= pm.n_pages) record_status(4u);
                else doff = (((int64_t)pid * Hkv + h) * pm.page_size + pos % pm.page_size) * kBlk;
            } else {
                doff = (((int64_t)b * Hkv + h) * capacity + pos) * kBlk;
            }
        }
        if (!mbar_wait_bounded(bar, phase)) {
            if (lane == 0) record_status(7u /* TBQ4_ERR_DEVICE_TIMEOUT */);
            break;
        }
        float v[kD];
        {
            const float4 *row = reinterpret_cast<const float4 *>(stg + lane * kQRowStride);
#pragma unroll
            for (int c = 0; c < kD / 4; ++c) {
                const float4 x = row[c];
                v[4 * c] = x.x;
                v[4 * c + 1] = x.y;
                v[4 * c + 2] = x.z;
                v[4 * c + 3] = x.w;
            }
        }
        __syncwarp();
        if (gnext < groups) load_group(gnext);              // lands while this group encodes
        // stage 1 with the signs folded in
#pragma unroll
        for (int j = 0; j < kD; j += 2) {
            const float bb = __fmul_rn(v[j + 1], sg.s[j + 1]);
            const float lo = __fmaf_rn(v[j], sg.s[j], bb);
            const float hi = __fmaf_rn(v[j], sg.s[j], -bb);
            v[j] = lo;
            v[j + 1] = hi;
        }
#pragma unroll
        for (int hs = 2; hs < kD; hs <<= 1) {
#pragma unroll
            for (int j = 0; j < kD; ++j) {
                if (j & hs) continue;
                const float a = v[j], c = v[j + hs];
                v[j] = __fadd_rn(a, c);
                v[j + hs] = __fsub_rn(a, c);
            }
        }
        const float cr = rot_c();
        float m = 0.f;
#pragma unroll
        for (int j = 0; j < kD; ++j) {
            v[j] = __fmul_rn(v[j], cr);
            m = fmaxf(m, fabsf(v[j]));
        }
        uint16_t sb = __half_as_ushort(__float2half_rn(m));
        if ((sb & 0x7FFFu) == 0x7C00u) sb = 0x7BFFu;                 // saturate at 65504
        const float S = half_bits_to_float(sb);
        uint16_t *mine = stage + lane * (kBlk / 2);
        mine[0] = sb;
        // A normal, unsaturated fp16 scale is within 2^-11 of max|x|, so
        // |x/S| <= 1 + 2^-11 and u = fl(fl(x/S) * 7.5) + 7.5 lies in
        // [-0.004, 15.004]: rint(u) is already in [0, 15] (3-bit: [0, 7]) and
        // needs no clamp.  A zero, subnormal or saturated scale: x is clamped
        // to [-S, S] first, which gives the same index (the index is monotone
        // in x, and -S, S give 0 and 15), and S = 0 divides by 1 instead, so
        // every u is 7.5 (3.5): index 8 (4).
        const uint32_t sabs = sb & 0x7FFFu;
        if (sabs < 0x0400u || sabs == 0x7BFFu) {
#pragma unroll
            for (int j = 0; j < kD; ++j) v[j] = fminf(fmaxf(v[j], -S), S);
        }
        const float Sd = S == 0.0f ? 1.0f : S;
        const float rs = __frcp_rn(Sd);
        // x / S correctly rounded, then the codebook's index: rint by adding
        // 1.5 * 2^23 (the sum's ulp is 1 for |u| < 2^22, and its low bits are
        // rint(u), ties to even)
        auto index_of = [&](float x) -> uint32_t {
            const float q0 = __fmul_rn(x, rs);
            const float e = __fmaf_rn(-q0, Sd, x);
            const float q = __fmaf_rn(e, rs, q0);
            constexpr float kL = kBits == 4 ? 7.5f : 3.5f;
            const float u = __fadd_rn(__fmul_rn(q, kL), kL);
            return __float_as_uint(__fadd_rn(u, 12582912.0f)) & (kBits == 4 ? 0xFu : 0x7u);
        };
        if constexpr (kBits == 4) {
#pragma unroll
            for (int w = 0; w < kD / 4; ++w) {                         // 4 nibbles per piece
                uint32_t piece = 0;
#pragma unroll
                for (int k4 = 0; k4 < 4; ++k4) piece |= index_of(v[4 * w + k4]) << (4 * k4);
                mine[1 + w] = (uint16_t)piece;
            }
        } else {
#pragma unroll
            for (int h2 = 0; h2 < kD / 16; ++h2) {                     // two 24-bit words
                uint64_t wd = 0;                                       // = three pieces
#pragma unroll
                for (int k16 = 0; k16 < 16; ++k16)
                    wd |= (uint64_t)index_of(v[16 * h2 + k16]) << (3 * k16);
                mine[1 + 3 * h2] = (uint16_t)wd;
                mine[2 + 3 * h2] = (uint16_t)(wd >> 16);
                mine[3 + 3 * h2] = (uint16_t)(wd >> 32);
            }
        }
        doffs[lane] = doff;
        __syncwarp();
        // store: the 32 blocks as 32 x kBlk / 2 consecutive 16-bit pieces
#pragma unroll
        for (int k2 = 0; k2 < kBlk / 2; ++k2) {
            const int j = lane + 32 * k2;
            const int row = j / (kBlk / 2), pc = j - row * (kBlk / 2);
            const int64_t off = doffs[row];
            if (off >= 0) *reinterpret_cast<uint16_t *>(cache + off + 2 * pc) = stage[j];
        }
        __syncwarp();
        gi = gnext;
    }
}


// Few rows (a prefill chunk, a decode step): one warp per row with the warp
// encoder, so that even a few thousand rows spread over every SM instead of
// the handful of blocks the thread-per-row kernel would fill.  The same
// bytes as quantize_rows_kernel<4> (the same encoding steps in the same
// order); rows are taken in source order (b, t, h), so the loads of
// consecutive warps are contiguous.
constexpr int kQWarpRowsPerBlock = 8;               // warps per block

__global__ void __launch_bounds__(kQWarpRowsPerBlock * 32)
quantize_warp_rows_kernel(const float *__restrict__ src, int B, int n_new, int Hkv,
                          const int32_t *__restrict__ start_pos, int64_t capacity,
                          uint64_t sign_lo, uint64_t sign_hi, const PageMap pm,
                          uint8_t *__restrict__ cache) {
    const int lane = threadIdx.x & 31;
    const uint32_t rows = (uint32_t)B * (uint32_t)n_new * (uint32_t)Hkv;   // < 2^31 (host)
    const uint32_t sbits = lane_sign_bits(sign_lo, sign_hi, lane);
    for (uint32_t r = blockIdx.x * kQWarpRowsPerBlock + (threadIdx.x >> 5); r < rows;
         r += gridDim.x * kQWarpRowsPerBlock) {
        const uint32_t h = r % (uint32_t)Hkv, bt = r / (uint32_t)Hkv;
        const uint32_t t = bt % (uint32_t)n_new, b = bt / (uint32_t)n_new;
        const float4 x4 = __ldcs(reinterpret_cast<const float4 *>(src + (int64_t)r * kD) + lane);
        float v[4] = {x4.x, x4.y, x4.z, x4.w};
        uint16_t sb;
        const uint32_t packed = encode_row(v, sbits, lane, &sb);
        const int64_t pos = (int64_t)__ldg(start_pos + b) + t;
        int64_t doff = -1;
        if (pos >= 0 && pos < capacity) {
            if (pm.table) {
                const int32_t pid = __ldg(pm.table + (int64_t)b * pm.max_pages + pos / pm.page_size);
                if (pid >= 0 && (int64_t)pid < pm.n_pages)
                    doff = (((int64_t)pid * Hkv + h) * pm.page_size + pos % pm.page_size) * kBlockBytes;
            } else {
                doff = (((int64_t)b * Hkv + h) * capacity + pos) * kBlockBytes;
            }
        }
        if (doff < 0) {
            if (lane == 0) record_status(4u /* TBQ4_ERR_CAPACITY */);
            continue;
        }
        uint8_t *dst = cache + doff;
        reinterpret_cast<uint16_t *>(dst + 2)[lane] = (uint16_t)packed;
        if (lane == 0) *reinterpret_cast<uint16_t *>(dst) = sb;
    }
}

}  // namespace tbq4

// quantize.cuh -- TBQ4 quantise-append: fp32 rows -> 66-byte blocks.
//
// Two encoders with the same op order, so the same bytes (the codebook's
// definition, see include/tbq4.h):
//   encode_row            one warp per row (four values per lane, the
//                         transform over shuffles); the decode kernel uses it
//                         to append the current token
//   quantize_rows_kernel  four threads per row, the transform in registers
//                         and two shuffle stages; the bulk append (512
//                         bytes in, 66 out per row)
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

// Bulk append: four threads per 128-value row, each holding a quarter of it
// (32 consecutive values) in registers.
//   rotation  the same butterflies in the same order as warp_fwht128 (stride
//             1 first; lower = a + b, upper = a - b, each rounded on its own).
//             Strides 1 .. 16 stay inside a quarter; strides 32 and 64 pair
//             quarters q and q ^ 1, q and q ^ 2 (lanes 8 and 16 apart), the
//             upper one computing fma(own, -1, partner) = partner - own.  The
//             sign flip is exact, so the first stage is fma(v_j, s_j, s_k v_k)
//             and fma(v_j, s_j, -s_k v_k).
//   scale     S = fp16(max |x_rot|), saturated at 65504.
//   index     clamp(rne(fl32(fl32(x/S) * 7.5) + 7.5), 0, 15), 8 when S == 0.
//             The quotient is the correctly rounded x/S by Markstein's method:
//             r = RN(1/S) once per row, q0 = RN(x r), e = x - q0 S (exact with
//             FMA), q = RN(q0 + e r).  rint is an add of 1.5 * 2^23 on the
//             FMA pipe; the clamp is needed only for rows whose fp16 scale is
//             zero, subnormal or saturated, and is applied to x for those.
// Memory: rows go in groups of 8 consecutive positions of one (sequence, KV
// head), so a group's 8 blocks are contiguous in the cache.  Lane l
// takes row l % 8 of its warp's group and quarter l / 8 of that row.  One
// CTA of 16 warps per SM; each warp streams its groups through a ring of
// kQDepth shared-memory stages (rows 528 bytes apart, so the eight lanes of a
// 16-byte read phase hit eight different bank groups), each lane copying 16
// bytes of every row with cp.async (one commit group per stage), and sends
// the copies of a later group into a stage as soon as the rows are in
// registers.  (One cp.async.bulk per row took longer: its operands go through
// uniform registers, one lane at a time.)  The blocks go out from a per-warp
// staging area, as one bulk shared -> global copy when the group's 8 blocks
// are consecutive and 16-byte aligned, else as 16-bit pieces.
// Paged destination: row (b, pos) goes to page table[b][pos / page_size],
// row pos % page_size, of a pool [n_pages][Hkv][page_size][66].  A null
// table means the contiguous cache [B][Hkv][capacity][66].
struct PageMap {
    const int32_t *table;
    int max_pages, page_size;
    int64_t n_pages;
    int64_t cache_bytes;        // bytes of the destination cache or pool (debug bounds checks)
};

// The 3-bit variant (TBQ3): the same rotation and scale, 8 levels
// (i - 3.5)/3.5 * S, index clamp(rne(fl32(fl32(x/S)*3.5)+3.5), 0, 7) (4 when
// S == 0), indices 8g .. 8g+7 as one little-endian 24-bit word (index 8g+k
// at bits 3k .. 3k+2): 2 + 48 = 50 bytes per block.
constexpr int kBlockBytes3 = 50;

constexpr int kQRows = 8;                                    // rows per group
constexpr int kQWarps = 16;                                  // warps per CTA
constexpr int kQDepth = 2;                                   // stages per warp
constexpr int kQRowStride = 512 + 16;                        // bytes between staged rows
constexpr int kQStageBytes = kQRows * kQRowStride;
constexpr int kQOutBytes = kQRows * kBlockBytes + 16 + kQRows * 8;   // blocks, pad, destinations
constexpr int kQThreads = kQWarps * 32;
constexpr int kQRingBytes = kQWarps * kQDepth * kQStageBytes;
constexpr int kQSmemBytes = kQRingBytes + kQWarps * kQOutBytes + kD * 4;
static_assert(kQSmemBytes <= 227 * 1024, "shared memory per CTA");
static_assert(kQStageBytes % 16 == 0 && kQRowStride % 16 == 0 && kQOutBytes % 16 == 0,
              "bulk copies and staged rows stay 16-byte aligned");

// Unsigned division by a divisor fixed for the whole launch, as a multiply
// and shifts (Granlund and Montgomery, "Division by invariant integers using
// multiplication", 1994, Figure 4.1): with l = ceil(log2 d) and
// m = floor(2^32 (2^l - d) / d) + 1, n / d = (t + ((n - t) >> 1)) >> (l - 1)
// where t = umulhi(m, n), for every 32-bit n (d = 1: n itself).
struct InvDiv {
    uint32_t m, l;
    __host__ __device__ static InvDiv make(uint32_t d) {      // d >= 1
        InvDiv v;
        v.l = 0;
        while (v.l < 32 && (1ull << v.l) < d) ++v.l;
        v.m = v.l == 0 ? 0u : (uint32_t)((((1ull << v.l) - d) << 32) / d + 1);
        return v;
    }
    __device__ __forceinline__ uint32_t div(uint32_t n) const {
        if (l == 0) return n;
        const uint32_t t = __umulhi(m, n);
        return (t + ((n - t) >> 1)) >> (l - 1);
    }
};

// Bulk shared -> global copy of `bytes` (a multiple of 16; both addresses
// 16-byte aligned), tracked by this thread's bulk-async group.
__device__ __forceinline__ void bulk_s2g(void *dst, uint32_t src, uint32_t bytes) {
    asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;"
                 ::"l"(dst), "r"(src), "r"(bytes) : "memory");
    asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}
// Waits until this thread's bulk stores have read their shared-memory source.
__device__ __forceinline__ void bulk_s2g_wait_read() {
    asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
}
// Waits until this thread's bulk stores are complete.
__device__ __forceinline__ void bulk_s2g_wait_all() {
    asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
}

// kBits: 4 (TBQ4, 66-byte blocks) or 3 (TBQ3, 50-byte blocks).  A group is 8
// consecutive positions t0 .. t0+7 of one (sequence b, KV head h): groups
// are numbered (b Hkv + h) gpb + t0 / 8 with gpb = ceil(n_new / 8).  Group k
// of a CTA is group blockIdx.x + k gridDim.x, taken by warp k % kQWarps.
template <int kBits>
__global__ void __launch_bounds__(kQThreads, 1)
quantize_rows_kernel(const float *__restrict__ src, int B, int n_new, int Hkv,
                     const int32_t *__restrict__ start_pos, int64_t capacity, uint64_t sign_lo,
                     uint64_t sign_hi, const PageMap pm, uint8_t *__restrict__ cache,
                     const InvDiv div_gpb, const InvDiv div_hkv) {
    extern __shared__ __align__(128) uint8_t qsm[];
    constexpr int kBlk = kBits == 4 ? kBlockBytes : kBlockBytes3;
    constexpr int kPieces = kBlk / 2;                         // 16-bit pieces per block
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int rho = lane & 7, qq = lane >> 3;                 // row of the group, quarter
    // groups per (sequence, KV head); B Hkv gpb < 2^31 (the host bounds the rows)
    const uint32_t gpb = ((uint32_t)n_new + kQRows - 1) / kQRows;
    const uint32_t groups = (uint32_t)B * (uint32_t)Hkv * gpb;
    // group gi -> sequence b, KV head h, first position t0
    auto group_of = [&](uint32_t gi, uint32_t &b, uint32_t &h, uint32_t &t0) {
        const uint32_t bh = div_gpb.div(gi);
        t0 = (gi - bh * gpb) * kQRows;
        b = div_hkv.div(bh);
        h = bh - b * (uint32_t)Hkv;
    };
    uint8_t *ring = qsm + warp * kQDepth * kQStageBytes;
    uint8_t *wout = qsm + kQRingBytes + warp * kQOutBytes;
    uint16_t *stage = reinterpret_cast<uint16_t *>(wout);                     // [8][kPieces]
    int64_t *doffs = reinterpret_cast<int64_t *>(wout + kQRows * kBlockBytes + 16);   // [8]
    float *sgn = reinterpret_cast<float *>(qsm + kQRingBytes + kQWarps * kQOutBytes);  // [128]
    if (threadIdx.x < kD) {
        const int i = threadIdx.x;
        const uint64_t w = i < 64 ? sign_lo : sign_hi;
        sgn[i] = ((w >> (i & 63)) & 1u) ? -1.0f : 1.0f;
    }
    __syncthreads();
    // the 8 rows of group gi into stage d, lane l copying bytes 16 l .. 16 l
    // + 15 of each (rows past the end repeat the last row; nothing of theirs
    // is stored).  Every call commits one cp.async group, empty past the last
    // group, so that waiting for all but the newest kQDepth - 1 groups always
    // waits for the stage about to be read.
    auto load_group = [&](uint32_t gi, int d) {
        if (gi < groups) {
            uint32_t b, h, t0;
            group_of(gi, b, h, t0);
            const uint32_t dst = smem_u32(ring + d * kQStageBytes) + 16 * lane;
#pragma unroll
            for (int r = 0; r < kQRows; ++r) {
                const uint32_t t = min(t0 + r, (uint32_t)n_new - 1);
                int64_t ridx = ((int64_t)b * n_new + t) * Hkv + h;
                if constexpr (kDebugBounds) ridx = checked_off(ridx, 1, (int64_t)B * n_new * Hkv);
                asm volatile("cp.async.cg.shared.global [%0], [%1], 16;"
                             ::"r"(dst + r * kQRowStride), "l"(src + ridx * kD + 4 * lane)
                             : "memory");
            }
        }
        asm volatile("cp.async.commit_group;" ::: "memory");     // one group per slot, maybe empty
    };
    const uint32_t gstride = kQWarps * gridDim.x;
    uint32_t gi = blockIdx.x + warp * gridDim.x;
#pragma unroll
    for (int d = 0; d < kQDepth; ++d) load_group(gi + d * gstride, d);
    const float neg = (qq & 1) ? -1.0f : 1.0f, neg2 = (qq & 2) ? -1.0f : 1.0f;
    uint32_t it = 0;
    for (; gi < groups; ++it, gi += gstride) {
        const int d = (int)(it % kQDepth);
        // this row's destination, while the rows load (one lane per row)
        int64_t doff = -1;          // -1: nothing stored (past the end or a bad position)
        if (qq == 0) {
            uint32_t b, h, t0;
            group_of(gi, b, h, t0);
            const uint32_t t = t0 + rho;
            if (t < (uint32_t)n_new) {
                const int64_t pos = (int64_t)__ldg(start_pos + b) + t;
                if (pos < 0 || pos >= capacity) {
                    record_status(4u /* TBQ4_ERR_CAPACITY */);
                } else if (pm.table) {
                    const int32_t pid =
                        __ldg(pm.table + (int64_t)b * pm.max_pages + pos / pm.page_size);
                    if (pid < 0 || (int64_t)pid >= pm.n_pages) record_status(4u);
                    else doff = (((int64_t)pid * Hkv + h) * pm.page_size + pos % pm.page_size) * kBlk;
                } else {
                    doff = (((int64_t)b * Hkv + h) * capacity + pos) * kBlk;
                }
                if (doff >= 0 && !in_extent(doff, kBlk, pm.cache_bytes)) doff = -1;
            }
            doffs[rho] = doff;
        }
        asm volatile("cp.async.wait_group %0;" ::"n"(kQDepth - 1) : "memory");
        __syncwarp();
        float v[32];
        {
            const float4 *row = reinterpret_cast<const float4 *>(ring + d * kQStageBytes +
                                                                 rho * kQRowStride + qq * 128);
#pragma unroll
            for (int c = 0; c < 8; ++c) {
                const float4 x = row[c];
                v[4 * c] = x.x;
                v[4 * c + 1] = x.y;
                v[4 * c + 2] = x.z;
                v[4 * c + 3] = x.w;
            }
        }
        __syncwarp();
        load_group(gi + kQDepth * gstride, d);
        // stride 1 with the signs folded in
        {
            const float4 *s4 = reinterpret_cast<const float4 *>(sgn + 32 * qq);
#pragma unroll
            for (int c = 0; c < 8; ++c) {
                const float4 sv = s4[c];
                const float sj[4] = {sv.x, sv.y, sv.z, sv.w};
#pragma unroll
                for (int e = 0; e < 4; e += 2) {
                    const int j = 4 * c + e;
                    const float bb = __fmul_rn(v[j + 1], sj[e + 1]);
                    const float lo = __fmaf_rn(v[j], sj[e], bb);
                    const float hi = __fmaf_rn(v[j], sj[e], -bb);
                    v[j] = lo;
                    v[j + 1] = hi;
                }
            }
        }
        // strides 2 .. 16 inside the quarter
#pragma unroll
        for (int hs = 2; hs < 32; hs <<= 1) {
#pragma unroll
            for (int j = 0; j < 32; ++j) {
                if (j & hs) continue;
                const float a = v[j], c = v[j + hs];
                v[j] = __fadd_rn(a, c);
                v[j + hs] = __fsub_rn(a, c);
            }
        }
        // strides 32 and 64 across quarters: the lower quarter adds the
        // partner's value, the upper one subtracts its own from it
#pragma unroll
        for (int j = 0; j < 32; ++j) {
            const float p = __shfl_xor_sync(kFull, v[j], 8);
            v[j] = __fmaf_rn(v[j], neg, p);
        }
#pragma unroll
        for (int j = 0; j < 32; ++j) {
            const float p = __shfl_xor_sync(kFull, v[j], 16);
            v[j] = __fmaf_rn(v[j], neg2, p);
        }
        const float cr = rot_c();
        float m = 0.f;
#pragma unroll
        for (int j = 0; j < 32; ++j) {
            v[j] = __fmul_rn(v[j], cr);
            m = fmaxf(m, fabsf(v[j]));
        }
        m = fmaxf(m, __shfl_xor_sync(kFull, m, 8));
        m = fmaxf(m, __shfl_xor_sync(kFull, m, 16));
        uint16_t sb = __half_as_ushort(__float2half_rn(m));
        if ((sb & 0x7FFFu) == 0x7C00u) sb = 0x7BFFu;                 // saturate at 65504
        const float S = half_bits_to_float(sb);
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
            for (int j = 0; j < 32; ++j) v[j] = fminf(fmaxf(v[j], -S), S);
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
        // the previous group's bulk store must have read the staging area
        if (lane == 0) bulk_s2g_wait_read();
        __syncwarp();
        uint16_t *mine = stage + rho * kPieces;
        if (qq == 0) mine[0] = sb;
        if constexpr (kBits == 4) {
            // values 32 qq .. 32 qq + 31: nibble bytes 16 qq .. 16 qq + 15,
            // pieces 1 + 8 qq .. 8 + 8 qq
#pragma unroll
            for (int w = 0; w < 8; ++w) {
                uint32_t piece = 0;
#pragma unroll
                for (int k4 = 0; k4 < 4; ++k4) piece |= index_of(v[4 * w + k4]) << (4 * k4);
                mine[1 + 8 * qq + w] = (uint16_t)piece;
            }
        } else {
            // values 32 qq .. 32 qq + 31: four 24-bit words, bytes 12 qq ..
            // 12 qq + 11, pieces 1 + 6 qq .. 6 + 6 qq
#pragma unroll
            for (int h2 = 0; h2 < 2; ++h2) {                           // two words = three pieces
                uint64_t wd = 0;
#pragma unroll
                for (int k16 = 0; k16 < 16; ++k16)
                    wd |= (uint64_t)index_of(v[16 * h2 + k16]) << (3 * k16);
                mine[1 + 6 * qq + 3 * h2] = (uint16_t)wd;
                mine[2 + 6 * qq + 3 * h2] = (uint16_t)(wd >> 16);
                mine[3 + 6 * qq + 3 * h2] = (uint16_t)(wd >> 32);
            }
        }
        // store.  The group's 8 blocks usually land back to back (8
        // consecutive positions of one KV head) on a 16-byte boundary
        // (positions in steps of 8 from a multiple of 8): then one bulk copy
        // of 8 kBlk bytes, issued by lane 0 after every lane's staging writes
        // are made visible to the async proxy.  Otherwise (a ragged group, a
        // skipped row, an unaligned start, a page boundary) each block goes out
        // as 16-bit pieces.
        const int64_t d0 = doffs[0], dme = doffs[rho];
        const bool bulk = __all_sync(kFull, dme == d0 + (int64_t)rho * kBlk) && d0 >= 0 &&
                          (d0 & 15) == 0;
        if (bulk) {
            asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
            __syncwarp();
            if (lane == 0) bulk_s2g(cache + d0, smem_u32(stage), kQRows * kBlk);
        } else {
            __syncwarp();
#pragma unroll
            for (int k2 = 0; k2 < (kQRows * kPieces + 31) / 32; ++k2) {
                const int j = lane + 32 * k2;
                if (j < kQRows * kPieces) {
                    const int row = j / kPieces, pc = j - row * kPieces;
                    const int64_t off = doffs[row];
                    if (off >= 0) *reinterpret_cast<uint16_t *>(cache + off + 2 * pc) = stage[j];
                }
            }
            __syncwarp();
        }
    }
    // the last bulk store completes before the CTA's shared memory goes away
    // (every copy into shared memory was waited for in its iteration; the
    // groups committed past the last one are empty)
    if (lane == 0) bulk_s2g_wait_all();
}


// Few rows (a prefill chunk, a decode step): one warp per row with the warp
// encoder, so that even a few thousand rows spread over every SM instead of
// a few hundred 8-row groups of the bulk kernel.  The same
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
            if (doff >= 0 && !in_extent(doff, kBlockBytes, pm.cache_bytes)) doff = -1;
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

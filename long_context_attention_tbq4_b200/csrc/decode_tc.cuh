// decode_tc.cuh -- split-K flash-decode over TBQ4 caches on the tensor cores.
//
// One CTA = one (sequence, KV head, split of the context).  Each warp
// streams its own 32-token chunks of raw K and V blocks (32 x 66 bytes each)
// from HBM into a private shared-memory ring with cp.async.bulk and an
// mbarrier per stage; the blocks are dequantised in registers inside the
// inner loop (no dequantisation pass, no fp16 copy of the cache: trefon.com,
// "Kontekst 262K na jednej RTX 4090", section "Od czego zaczalem") and the
// G query heads of the KV head share every block through the tensor cores:
//
//   S^T (32 tokens x 8 heads) = K (tokens x 128) . Q_rot^T   mma m16n8k32 u8 x s8
//   O^T (128 dims x 8 heads) += V^T (dims x tokens) . P'^T    mma m16n8k16 f16
//
// K operand: each nibble byte enters twice, raw (lo + 16 hi, no unpacking)
// and masked to its low nibble (one LOP3 per four bytes).  With the weights
//   raw byte  : u = q_odd,           low nibble : w = 16 q_even - q_odd
// the products sum to 16 (lo q_even + hi q_odd): 16 sum_d n_d q_d, exactly,
// in integers.  q_rot is normalised by a power of two and held as an 18-bit
// integer; u and w are split into three signed bytes.  The level map is
// applied afterwards, sum_d q_d (2n_d - 15) = 2 sum_d n_d q_d - 15 sum_d q_d.
// (fp16 q was not enough: heavy-tailed keys turn a 2^-12 error in q into
// output errors of a few 1e-3 where one token dominates; 18 bits keep the
// logit error below 1e-3 of a log2 unit even in the worst case.)
// V operand: pairs of tokens are interleaved with PRMT so that one register
// holds the same dimension of two tokens; the levels enter as (2n - 15) 2^-11,
// exactly (see lvl_lo).  P' = p * S_v * ps (S_v the
// block scale of V, ps a per-warp power of two that keeps P' a normal fp16)
// enters as two fp16 terms hi + lo, so O = sum_t p_t S_v,t (2n-15) / 15 once
// 1 / ps is applied.
// Softmax runs in fp32 in the log2 domain; the running max is per head and
// the accumulators are only rescaled when some logit exceeds it by 2^3
// (tested with one vote per chunk; the chunk max is only formed then).
#pragma once
#include "common.cuh"
#include "decode.cuh"
#include "mbarrier.cuh"
#include "quantize.cuh"

namespace tbq4 {

constexpr int kTcWarps = 16;                              // one CTA per SM
constexpr int kTcStages = 3;
constexpr int kChunk = 32;                                 // tokens per chunk
constexpr int kChunkBytes = kChunk * kBlockBytes;          // 2112
constexpr int kStageBytes = 2 * kChunkBytes + 16;          // K | V | pad
constexpr int kWarpRing = kTcStages * kStageBytes;
constexpr int kRingBytes = kTcWarps * kWarpRing;
constexpr int kBarBytes = kTcWarps * kTcStages * 8;
constexpr int kQScratchBytes = 2 * 3 * kMaxGroup * 64 + 2 * kMaxGroup * 4;   // q pieces + constants
constexpr int kTcSmemBytes = kRingBytes + kBarBytes + kQScratchBytes + 128;
// Paged caches: the page id of every chunk of the split, copied into shared
// memory during the q prologue (so no table load sits on the copy path).
// Paged launches keep splits at or below kPidCap chunks.
constexpr int kPidCap = 4096;
constexpr int kTcSmemBytesPaged = kTcSmemBytes + kPidCap * 4;
static_assert(kTcSmemBytesPaged <= 227 * 1024, "shared memory per CTA");
constexpr int kQBits = 18;                                 // |q_int| <= 2^18

static_assert(kStageBytes % 16 == 0, "stage must keep 16-byte alignment");
constexpr float kLazyRescale = 8.0f;                       // log2 units
static_assert(kRingBytes >= kTcWarps * 32 * 36 * 4 + 3 * kTcWarps * kMaxGroup * 4 +
                                kMaxGroup * 8,
              "merge buffers reuse the ring");

// The MMA wrappers are pure register operations (not volatile), so the
// compiler may interleave them with the unpacking of the next operands.
__device__ __forceinline__ void mma16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                         uint32_t a3, uint32_t b0, uint32_t b1) {
    asm("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
        "{%8,%9}, {%0,%1,%2,%3};\n"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// D (s32) += A (u8, 16x32 row) * B (s8, 32x8 col)
__device__ __forceinline__ void imma16832(int (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                          uint32_t a3, uint32_t b0, uint32_t b1) {
    asm("mma.sync.aligned.m16n8k32.row.col.s32.u8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
        "{%8,%9}, {%0,%1,%2,%3};\n"
        : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// D (s32) = A (u8) * B (s8), accumulator starting from zero
__device__ __forceinline__ void imma16832_z(int (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                            uint32_t a3, uint32_t b0, uint32_t b1) {
    asm("mma.sync.aligned.m16n8k32.row.col.s32.u8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
        "{%8,%9}, {%10,%10,%10,%10};\n"
        : "=r"(d[0]), "=r"(d[1]), "=r"(d[2]), "=r"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1), "r"(0));
}

// 2^x with the MUFU approximation (relative error about 2^-22; results
// below 2^-126 flush to zero, which only drops weights that no sum can see).
__device__ __forceinline__ float fast_ex2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

__device__ __forceinline__ uint32_t ld_u32(const uint8_t *p) {
    return *reinterpret_cast<const uint32_t *>(p);
}

__device__ __forceinline__ float ld_half(const uint8_t *p) {
    return __half2float(*reinterpret_cast<const __half *>(p));
}

// V levels enter the tensor cores as (n - 7.5) 2^-10 = (2n - 15) 2^-11,
// exact in fp16 (normal numbers, at most 4 significant bits), from one LOP3
// and one HFMA2 per register: masking a nibble into the low mantissa bits of
// an fp16 with a zero exponent field gives the subnormal n 2^-24 (bits 0-3)
// or 16 n 2^-24 (bits 4-7); fp16 arithmetic keeps subnormals, so x 2^14 -
// 15 2^-11 (resp. x 2^10 - 15 2^-11) is (2n - 15) 2^-11 with no rounding,
// and O = 2^11 sum_t P'_t (2n_t - 15) 2^-11.
constexpr uint32_t kH2Pow14 = 0x74007400u;     // {2^14, 2^14}
constexpr uint32_t kH2Pow10 = 0x64006400u;     // {2^10, 2^10}
constexpr uint32_t kH2NegBias = 0x9F809F80u;   // {-15 2^-11, -15 2^-11}
constexpr float kVLevelScale = 2048.0f;        // 2^11

__device__ __forceinline__ uint32_t hfma2_u32(uint32_t x, uint32_t a, uint32_t b) {
    __half2 r = __hfma2(*reinterpret_cast<__half2 *>(&x), *reinterpret_cast<__half2 *>(&a),
                        *reinterpret_cast<__half2 *>(&b));
    return *reinterpret_cast<uint32_t *>(&r);
}
// low nibbles of bytes 0 and 2 -> {(2n - 15) 2^-11, (2n - 15) 2^-11}
__device__ __forceinline__ uint32_t lvl_lo(uint32_t v) {
    return hfma2_u32(v & 0x000F000Fu, kH2Pow14, kH2NegBias);
}
// high nibbles of bytes 0 and 2 -> {(2n - 15) 2^-11, (2n - 15) 2^-11}
__device__ __forceinline__ uint32_t lvl_hi(uint32_t v) {
    return hfma2_u32(v & 0x00F000F0u, kH2Pow10, kH2NegBias);
}

// x = c0 + 256 c1 + 65536 c2 with c0, c1 in [-128, 127]
__device__ __forceinline__ void split3(int x, int8_t &c0, int8_t &c1, int8_t &c2) {
    const int b0 = ((x + 128) & 255) - 128;
    const int x1 = (x - b0) >> 8;
    const int b1 = ((x1 + 128) & 255) - 128;
    c0 = (int8_t)b0;
    c1 = (int8_t)b1;
    c2 = (int8_t)((x1 - b1) >> 8);
}

// TBQ3 (3-bit) K operand.  In a group of eight 3-bit indices (a 24-bit word,
// index 8g + k at bits 3k) the indices of dimensions 2j and 2j + 1 already
// form one 6-bit field i_even + 8 i_odd at bits 6j.  Spreading the four
// fields to four bytes gives the same operand shape as the 4-bit raw bytes
// (lo + 16 hi), with 8 in place of 16: the raw byte weighs q_odd, its low 3
// bits (i_even) weigh 8 q_even - q_odd, and the products sum to
// 8 sum_d i_d q_d.
__device__ __forceinline__ uint32_t tbq3_pairs(uint32_t g) {
    const uint32_t t = (g & 0x00000FFFu) | ((g & 0x00FFF000u) << 4);    // 2 fields per half
    return (t & 0x003F003Fu) | ((t & 0x0FC00FC0u) << 2);                // 1 field per byte
}

// 3-bit V levels straight from the packed indices, with no expansion to
// nibbles.  For two tokens' 24-bit groups A and B (indices 8g .. 8g+7 at bits
// 3k .. 3k+2), three byte permutations put every field inside the mantissa
// bits of an fp16 half: [A0 A1 B0 B1] holds fields 0, 1, 2 at bits 0, 3, 6;
// [A1 A2 B1 B2] fields 3, 4, 5 at bits 1, 4, 7; [A2 A3 B2 B3] fields 6, 7 at
// bits 2, 5.  Masking a field gives the subnormal i 2^(b - 24); one HFMA2 by
// 2^(14 - b) minus 7 2^-11 turns it into (2i - 7) 2^-11, exactly.  Returns
// field f of A (low half) and of B (high half).
template <int f>
__device__ __forceinline__ uint32_t lvl3(uint32_t A, uint32_t B) {
    constexpr uint32_t kSel[8] = {0x5410u, 0x5410u, 0x5410u, 0x6521u,
                                  0x6521u, 0x6521u, 0x7632u, 0x7632u};
    constexpr int kBit[8] = {0, 3, 6, 1, 4, 7, 2, 5};
    constexpr uint32_t kMask = 0x00070007u << kBit[f];
    constexpr uint32_t kMul = (uint32_t)(15 + 14 - kBit[f]) << 10;     // fp16 2^(14 - b)
    return hfma2_u32(__byte_perm(A, B, kSel[f]) & kMask, kMul | (kMul << 16), 0x9B009B00u);
}

// kPaged: the caches are page pools addressed through p.block_table.
// kBits: 4 (TBQ4, 66-byte blocks) or 3 (TBQ3, 50-byte blocks; the stage
// layout is the same, a 3-bit chunk fills 1,600 of its 2,112 bytes).
template <bool kPaged, int kBits = 4>
__global__ void __launch_bounds__(kTcWarps * 32, 1)
decode_tc_kernel(const AttnParams p) {
    static_assert(kBits == 4 || !kPaged, "paged caches hold 4-bit blocks");
    constexpr int kBlk = kBits == 4 ? kBlockBytes : kBlockBytes3;
    extern __shared__ __align__(128) uint8_t smem[];
    uint8_t *ring = smem;
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + kRingBytes);
    // the dependent combine kernel may be scheduled from now on
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int r = lane >> 2, c = lane & 3;
    const int split = blockIdx.x, g = blockIdx.y, s = blockIdx.z;
    const int G = p.G;
    // The first chunks are copied before the length is known, bounded by
    // max_len (<= capacity): the split's end under the largest length.
    const int32_t t0 = split * p.split_tokens;
    const int32_t t1_max = min(p.max_len, t0 + p.split_tokens);
    const int n_chunks_max = t1_max > t0 ? (t1_max - t0 + kChunk - 1) / kChunk : 0;

    // ---- per-warp ring: the first copies go out before the q prologue -----
    uint8_t *ring_p = ring + warp * kWarpRing;
    const uint32_t bar_w = smem_u32(bars) + warp * kTcStages * 8;
    const uint8_t *kb = kPaged ? p.k : p.k + s * p.seq_stride + g * p.head_stride;
    const uint8_t *vb = kPaged ? p.v : p.v + s * p.seq_stride + g * p.head_stride;
    // Warp w takes chunks w, w + 16, w + 32, ... of the split (fixed, so the
    // result does not depend on timing).  A chunk never crosses a page (the
    // page size is a multiple of 32 tokens and so is t0).

    // Paged: every chunk's byte offset in the pools, in 64-byte units (a
    // chunk starts on a multiple of 32 tokens, 2,112 bytes, inside a page of
    // a multiple of 32 tokens, so offsets are multiples of 64 and 32 bits
    // reach 256 GB); kBadChunk marks an out-of-range page id.  Filled below,
    // read after the q barrier.
    constexpr uint32_t kBadChunk = 0xFFFFFFFFu;
    uint32_t *cofs_s = reinterpret_cast<uint32_t *>(smem + kTcSmemBytes);
    auto chunk_cofs = [&](int ci) -> uint32_t {
        bool bad;
        const int32_t t = t0 + ci * kChunk;
        const int64_t o = paged_offset(p, page_id(p, s, t), g, t, &bad);
        return bad ? kBadChunk : (uint32_t)(o >> 6);
    };
    // byte offset of chunk ci from kb / vb; *bad: an out-of-range page id
    auto chunk_ofs = [&](int ci, bool *bad) -> int64_t {
        if constexpr (kPaged) {
            const uint32_t v = cofs_s[ci];
            *bad = v == kBadChunk;
            return *bad ? 0 : (int64_t)v << 6;
        } else {
            *bad = false;
            return (int64_t)(t0 + ci * kChunk) * kBlk;
        }
    };
    // chunk ci -> warp w, stage st; ofs from chunk_ofs
    auto issue_for = [&](int w, int ci, int st, int32_t tend, int64_t ofs) {
        const int32_t start = t0 + ci * kChunk;
        const int32_t valid = min(kChunk, tend - start);
        const uint32_t bytes = (uint32_t)((valid + 7) & ~7) * kBlk;
        const uint32_t bar = smem_u32(bars) + (w * kTcStages + st) * 8;
        const uint32_t dst = smem_u32(ring) + w * kWarpRing + st * kStageBytes;
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        mbar_expect_tx(bar, 2 * bytes);
        if constexpr (kDebugBounds)
            ofs = checked_off((kb - p.k) + ofs, bytes, p.cache_bytes) - (kb - p.k);
        bulk_g2s(dst, kb + ofs, bytes, bar);
        bulk_g2s(dst + kChunkBytes, vb + ofs, bytes, bar);
    };
    auto issue = [&](int ci, int st, int32_t tend, int64_t ofs) { issue_for(warp, ci, st, tend, ofs); };
    // Contiguous caches: the last warp (never a q warp) initialises every
    // warp's barriers and issues every warp's first chunk, so the q warps
    // start on q at once.  Paged: each warp does its own once its first page
    // id is in.
    static_assert(kTcWarps <= 32 && kMaxGroup < kTcWarps, "one issuing lane per warp");
    bool bad0 = false;      // paged: the first chunk's page id (lane 0 of each warp)
    if (!kPaged && warp == kTcWarps - 1 && lane < kTcWarps) {
        const int w = lane;
        for (int st = 0; st < kTcStages; ++st) mbar_init(smem_u32(bars) + (w * kTcStages + st) * 8, 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        if (w < n_chunks_max) {                             // stage 0 now, the others later
            bool bad;
            issue_for(w, w, 0, t1_max, chunk_ofs(w, &bad));
        }
    }
    if (kPaged) {
        // every warp sets up its own ring and issues its first chunk (the
        // page id load overlaps the q loads); the warps past the q warps copy
        // the remaining page ids
        uint32_t c0 = 0;
        if (lane == 0 && warp < n_chunks_max) c0 = chunk_cofs(warp);
        if (warp >= kMaxGroup)
            for (int i = kTcWarps + threadIdx.x - kMaxGroup * 32; i < n_chunks_max;
                 i += (kTcWarps - kMaxGroup) * 32)
                cofs_s[i] = chunk_cofs(i);
        if (lane == 0) {
            for (int st = 0; st < kTcStages; ++st) mbar_init(smem_u32(bars) + (warp * kTcStages + st) * 8, 1);
            asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
            if (warp < n_chunks_max) {
                cofs_s[warp] = c0;
                issue_for(warp, warp, 0, t1_max, chunk_ofs(warp, &bad0));
            }
        }
    }
    // queue of the chunks in stages st, st+1, st+2 (mod 3); -1: none
    int q0 = warp < n_chunks_max ? warp : -1;
    int q1 = warp + kTcWarps < n_chunks_max ? warp + kTcWarps : -1;
    int q2 = warp + 2 * kTcWarps < n_chunks_max ? warp + 2 * kTcWarps : -1;
    // Launched as a programmatic dependent of the kernel before it (the
    // previous decode step's combine, which triggers once its own inputs are
    // complete): everything above touches only the caches, bounded by the
    // host's max_len, and this CTA's shared memory.  q, the lengths and the
    // new rows, which that kernel's predecessors may produce, are read after
    // the wait, and so are the partials written (the combine before may still
    // be reading the workspace until the wait returns).  Under an ordinary
    // launch the wait returns at once.
    asm volatile("griddepcontrol.wait;" ::: "memory");
    float qv[4] = {0.f, 0.f, 0.f, 0.f};
    if (warp < G) {
        const int64_t base = ((int64_t)s * p.Hq + g * G + warp) * kD + 4 * lane;
#pragma unroll
        for (int k = 0; k < 4; ++k) qv[k] = load_q(p, base + k);
    }
    const int32_t len = seq_length(p, s);
    const int32_t t1 = min(len, t1_max);
    const int n_chunks = t1 > t0 ? (t1 - t0 + kChunk - 1) / kChunk : 0;
    // a bad page id is an error only where the chunk holds real tokens
    if (kPaged && bad0 && warp < n_chunks) record_status(4u);

    // ---- q: rotate, normalise by a power of two, 18-bit integer ----------
    // q_int = rint(q_rot * 2^(18-e)) with 2^e > max|q_rot|, so |q_int| <= 2^18.
    // Per dimension pair j = (2j, 2j+1): u_j = q_int[2j+1] (weight of the raw
    // byte) and w_j = 16 q_int[2j] - q_int[2j+1] (weight of its low nibble;
    // 8 q_int[2j] - q_int[2j+1] for the 3-bit pair bytes), each split into
    // three signed bytes, pieces [3][head][pair].
    int8_t *qu8 = reinterpret_cast<int8_t *>(smem + kRingBytes + kBarBytes);   // [3][8][64]
    int8_t *qw8 = qu8 + 3 * kMaxGroup * 64;                              // [3][8][64]
    float *qpar = reinterpret_cast<float *>(qw8 + 3 * kMaxGroup * 64);   // [8][2]
    if (warp < G) {
        const uint32_t sbits = lane_sign_bits(p.sign_lo, p.sign_hi, lane);
        float v[4] = {qv[0], qv[1], qv[2], qv[3]};
        warp_rotate128(v, sbits, lane);
        float mx = warp_max(fmaxf(fmaxf(fabsf(v[0]), fabsf(v[1])), fmaxf(fabsf(v[2]), fabsf(v[3]))));
        int e = 0;
        if (mx > 0.f) frexpf(mx, &e);                 // mx = f * 2^e, f in [0.5, 1)
        int qi[4], qsum = 0;
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            qi[k] = __float2int_rn(ldexpf(v[k], kQBits - e));
            qsum += qi[k];
        }
#pragma unroll
        for (int j = 0; j < 2; ++j) {                 // pairs 2 lane + j
            const int pair = 2 * lane + j;
            const int u = qi[2 * j + 1], w = (kBits == 4 ? 16 : 8) * qi[2 * j] - qi[2 * j + 1];
            split3(u, qu8[(0 * kMaxGroup + warp) * 64 + pair], qu8[(1 * kMaxGroup + warp) * 64 + pair],
                   qu8[(2 * kMaxGroup + warp) * 64 + pair]);
            split3(w, qw8[(0 * kMaxGroup + warp) * 64 + pair], qw8[(1 * kMaxGroup + warp) * 64 + pair],
                   qw8[(2 * kMaxGroup + warp) * 64 + pair]);
        }
        qsum = __reduce_add_sync(kFull, qsum);
        if (lane == 0) {
            // log2 logit = (2 S - 15 sum q) * S_k * scale * log2(e) / 15 * 2^(e-18)
            // with S = sum n q and the integer MMAs returning 16 S; for 3 bits
            // (2 S - 7 sum q) * S_k ... / 7 with S = sum i q, the MMAs returning 8 S
            const float fh = p.scale_log2 * (kBits == 4 ? 1.0f / 15.0f : 1.0f / 7.0f) *
                             ldexpf(1.0f, e - kQBits);
            qpar[2 * warp + 0] = (kBits == 4 ? 0.125f : 0.25f) * fh;
            qpar[2 * warp + 1] = (kBits == 4 ? -15.0f : -7.0f) * (float)qsum * fh;
        }
    } else if (warp < kMaxGroup) {
        for (int k = lane; k < 3 * 64; k += 32) {
            qu8[((k >> 6) * kMaxGroup + warp) * 64 + (k & 63)] = 0;
            qw8[((k >> 6) * kMaxGroup + warp) * 64 + (k & 63)] = 0;
        }
        if (lane == 0) { qpar[2 * warp] = 0.f; qpar[2 * warp + 1] = 0.f; }
    }
    __syncthreads();

    // B fragments (k = byte positions, n = heads), thread (n = r, c): k-step
    // i covers the nibble bytes 16c + 4i .. +3 of a row (pairs of dims);
    // b0 weighs the raw bytes, b1 their low nibbles.
    uint32_t qb[4][3][2];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
#pragma unroll
        for (int pc = 0; pc < 3; ++pc) {
            const int o = (pc * kMaxGroup + r) * 64 + 16 * c + 4 * i;
            qb[i][pc][0] = *reinterpret_cast<const uint32_t *>(qu8 + o);
            qb[i][pc][1] = *reinterpret_cast<const uint32_t *>(qw8 + o);
        }
    }
    // per-head constants for this thread's score columns (heads 2c, 2c+1)
    const float f2a = qpar[4 * c + 0], bha = qpar[4 * c + 1];
    const float f2b = qpar[4 * c + 2], bhb = qpar[4 * c + 3];
    // The rest of the first copies go out later: issued together with stage
    // 0 they would be served interleaved with it, so every warp's first chunk
    // would land only near the end of the whole burst; and cp.async.bulk
    // stalls the issuing thread while the copies before it are queued.  So
    // each warp issues its own stage 1 now and its stage 2 once its first
    // chunk has been consumed.
    bool stage2_pending = true;
    if (lane == 0 && q1 >= 0) {
        bool bad;
        const int64_t o = chunk_ofs(q1, &bad);
        if (bad && q1 < n_chunks) record_status(4u /* TBQ4_ERR_CAPACITY */);
        issue(q1, 1, t1_max, o);
    }


    // Loop-invariant byte offsets inside a stage.  K: rows r (+8, +16, +24)
    // of the chunk, 16 bytes from nibble byte 16c; every such row starts at
    // the same offset mod 4 (16-row and 8-row steps are multiples of 4 bytes),
    // so one aligned base and one funnel shift serve all four rows.
    // (3-bit: 12 bytes from byte 12c, the same 32 dimensions)
    const int koff = r * kBlk + 2 + (kBits == 4 ? 16 : 12) * c;
    const int kbase = koff & ~3;
    const uint32_t ksh = (uint32_t)(koff & 3) * 8u;
    // V: tokens 2c + {0, 1, 8, 9} (+16 for the second k-step), nibble
    // bytes 8r .. 8r+7; even tokens sit 2 bytes past a 4-byte boundary.
    // (3-bit: 6 bytes from byte 6r)
    const int voff = 2 * c * kBlk + 2 + (kBits == 4 ? 8 : 6) * r;

    float o[8][4];
#pragma unroll
    for (int mt = 0; mt < 8; ++mt)
#pragma unroll
        for (int k = 0; k < 4; ++k) o[mt][k] = 0.f;
    float m_a = -INFINITY, m_b = -INFINITY, l_a = 0.f, l_b = 0.f;
    // P' = p S_v ps in fp16, with ps a power of two per warp: the largest one
    // that keeps P' <= 2^15 for every V scale S_v this warp has seen (p <=
    // 2^8 under the lazy rescale), i.e. S_v <= s_lim = 2^7 / ps.  A fixed
    // ps = 2^-8 (room for S_v = 65504) would put the weights of most tokens
    // among the fp16 subnormals, whose absolute spacing 2^-24 costs the
    // output up to 1e-3; with ps fitted to the data they stay normal.  ps = 0
    // until the first chunk with a nonzero S_v.
    float ps = 0.f, s_lim = 0.f;
    const uint32_t hsel = (r & 1) ? 0x7632u : 0x5410u;          // half of head n = r
    const int src0 = 4 * (2 * c) + (r >> 1), src1 = 4 * (2 * c + 1) + (r >> 1);
    bool aborted = false;
    uint32_t phase = 0;
    // Fused append: the warp whose chunk holds the current token (len - 1)
    // encodes its K and V rows, exactly as quantize-append does, patches them
    // into the staged blocks and stores them in the caches.  A length that
    // was clamped (flagged as a capacity error) appends nothing.
    int ci_app = -1;
    if (p.k_new != nullptr && len - 1 >= t0 && len - 1 < t1 && __ldg(p.seq_lens + s) == len)
        ci_app = (len - 1 - t0) / kChunk;

    // A warp's chunk indices grow, so the first one at or past n_chunks ends
    // its work.
    int st = 0;
    while (q0 >= 0 && q0 < n_chunks) {
        if (!mbar_wait_bounded(bar_w + 8 * st, phase)) {
            if (lane == 0) record_status(7u /* TBQ4_ERR_DEVICE_TIMEOUT */);
            aborted = true;
            break;
        }
        const int32_t cstart = t0 + q0 * kChunk;
        const int32_t valid = min(kChunk, t1 - cstart);
        uint8_t *kst = ring_p + st * kStageBytes;
        uint8_t *vst = kst + kChunkBytes;
        if (kBits == 4 && q0 == ci_app) {
            const int jn = len - 1 - cstart;
            const uint32_t sbits = lane_sign_bits(p.sign_lo, p.sign_hi, lane);
            const int64_t row = ((int64_t)s * p.Hkv + g) * kD;
            bool gbad = false;
            int64_t gofs;
            if constexpr (kPaged)
                gofs = paged_offset(p, page_id(p, s, len - 1), g, len - 1, &gbad);
            else
                gofs = s * p.seq_stride + g * p.head_stride + (int64_t)(len - 1) * kBlockBytes;
            if (!gbad && !in_extent(gofs, kBlockBytes, p.cache_bytes)) gbad = true;
            if (gbad && lane == 0) record_status(4u);
#pragma unroll
            for (int kv = 0; kv < 2; ++kv) {
                const float4 x4 = reinterpret_cast<const float4 *>((kv ? p.v_new : p.k_new) + row)[lane];
                float xv[4] = {x4.x, x4.y, x4.z, x4.w};
                uint16_t sb;
                const uint32_t packed = encode_row(xv, sbits, lane, &sb);
                uint8_t *sa = (kv ? vst : kst) + jn * kBlockBytes;
                uint8_t *ga = (kv ? p.v_wr : p.k_wr) + gofs;
                reinterpret_cast<uint16_t *>(sa + 2)[lane] = (uint16_t)packed;
                if (!gbad) reinterpret_cast<uint16_t *>(ga + 2)[lane] = (uint16_t)packed;
                if (lane == 0) {
                    *reinterpret_cast<uint16_t *>(sa) = sb;
                    if (!gbad) *reinterpret_cast<uint16_t *>(ga) = sb;
                }
            }
            __syncwarp();
        }

        // ---- 16 S^T = K Q^T for two 16-token tiles (exact, integer) ------
        float sc[2][4];
#pragma unroll
        for (int tile = 0; tile < 2; ++tile) {
            int acc[3][4];
            const uint8_t *k0 = kst + kbase + tile * 16 * kBlk;           // row r
            const uint8_t *k1 = k0 + 8 * kBlk;                            // row r + 8
            uint32_t xk0[4], xk1[4];     // nibble bytes 16c + 4i .. +3 of the two rows
            if constexpr (kBits == 4) {
                uint32_t w0[5], w1[5];
#pragma unroll
                for (int i = 0; i < 5; ++i) { w0[i] = ld_u32(k0 + 4 * i); w1[i] = ld_u32(k1 + 4 * i); }
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    xk0[i] = __funnelshift_r(w0[i], w0[i + 1], ksh);
                    xk1[i] = __funnelshift_r(w1[i], w1[i + 1], ksh);
                }
            } else {
                uint32_t w0[4], w1[4];
#pragma unroll
                for (int i = 0; i < 4; ++i) { w0[i] = ld_u32(k0 + 4 * i); w1[i] = ld_u32(k1 + 4 * i); }
                const uint32_t *wr[2] = {w0, w1};
                uint32_t *xr[2] = {xk0, xk1};
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    const uint32_t W0 = __funnelshift_r(wr[h][0], wr[h][1], ksh);
                    const uint32_t W1 = __funnelshift_r(wr[h][1], wr[h][2], ksh);
                    const uint32_t W2 = __funnelshift_r(wr[h][2], wr[h][3], ksh);
                    xr[h][0] = tbq3_pairs(W0 & 0x00FFFFFFu);
                    xr[h][1] = tbq3_pairs(__funnelshift_r(W0, W1, 24) & 0x00FFFFFFu);
                    xr[h][2] = tbq3_pairs(__funnelshift_r(W1, W2, 16) & 0x00FFFFFFu);
                    xr[h][3] = tbq3_pairs(W2 >> 8);
                }
            }
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const uint32_t x0 = xk0[i], x1 = xk1[i];                       // raw bytes
                constexpr uint32_t kLoMask = kBits == 4 ? 0x0F0F0F0Fu : 0x07070707u;
                const uint32_t lo0 = x0 & kLoMask, lo1 = x1 & kLoMask;
#pragma unroll
                for (int pc = 0; pc < 3; ++pc) {
                    if (i == 0)
                        imma16832_z(acc[pc], x0, x1, lo0, lo1, qb[i][pc][0], qb[i][pc][1]);
                    else
                        imma16832(acc[pc], x0, x1, lo0, lo1, qb[i][pc][0], qb[i][pc][1]);
                }
            }
            // 16 sum_d n_d q_int_d (3 bits: 8 sum_d i_d q_int_d) = 65536 acc2 + 256 acc1 + acc0
#pragma unroll
            for (int e = 0; e < 4; ++e)
                sc[tile][e] = fmaf((float)acc[2][e], 65536.0f, (float)(acc[1][e] * 256 + acc[0][e]));
        }

        // ---- log2 logits relative to the running max ----------------------
        // thread's tokens: u = 0..3 -> token 8u + r (tile u>>1, row half u&1)
        float sk[4], sv[4], ta[4], tb[4], xa[4], xb[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const int j = 8 * u + r;
            sk[u] = ld_half(kst + j * kBlk);
            sv[u] = ld_half(vst + j * kBlk);
            ta[u] = fmaf(sc[u >> 1][2 * (u & 1) + 0], f2a, bha);   // logit / S_k
            tb[u] = fmaf(sc[u >> 1][2 * (u & 1) + 1], f2b, bhb);
            xa[u] = fmaf(ta[u], sk[u], -m_a);                       // logit - m
            xb[u] = fmaf(tb[u], sk[u], -m_b);
        }
        if (valid != kChunk) {                    // tail chunk: tokens >= valid
#pragma unroll
            for (int u = 0; u < 4; ++u)
                if (8 * u + r >= valid) { xa[u] = -INFINITY; xb[u] = -INFINITY; sv[u] = 0.f; }
        }
        bool grow = false, sgrow = false;
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            grow |= (xa[u] > kLazyRescale) | (xb[u] > kLazyRescale);
            sgrow |= sv[u] > s_lim;
        }
        // The running max is only moved (and the accumulators rescaled)
        // when some logit exceeds it by more than 2^3; otherwise
        // p = 2^(logit - m) <= 2^8.  ps only shrinks, when a V scale above
        // s_lim arrives; both are rare after the first chunks.
        if (__any_sync(kFull, grow | sgrow)) {
          if (__any_sync(kFull, sgrow)) {
            float smx = fmaxf(fmaxf(sv[0], sv[1]), fmaxf(sv[2], sv[3]));
#pragma unroll
            for (int msk = 4; msk < 32; msk <<= 1) smx = fmaxf(smx, __shfl_xor_sync(kFull, smx, msk));
            // the largest power of two <= 2^7 / smx (smx > s_lim >= 0)
            const float nps = pow2_floor(__fdividef(128.0f, smx));
            const float f = ps == 0.f ? 1.f : pow2_ratio(nps, ps);    // a power of two, < 1
#pragma unroll
            for (int mt = 0; mt < 8; ++mt) {
                o[mt][0] *= f; o[mt][1] *= f; o[mt][2] *= f; o[mt][3] *= f;
            }
            ps = nps;
            s_lim = 128.0f * pow2_inv(nps);
          }
          if (__any_sync(kFull, grow)) {
            float mxa = -INFINITY, mxb = -INFINITY;
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                xa[u] = xa[u] == -INFINITY ? -INFINITY : ta[u] * sk[u];     // the logits
                xb[u] = xb[u] == -INFINITY ? -INFINITY : tb[u] * sk[u];
                mxa = fmaxf(mxa, xa[u]);
                mxb = fmaxf(mxb, xb[u]);
            }
#pragma unroll
            for (int msk = 4; msk < 32; msk <<= 1) {
                mxa = fmaxf(mxa, __shfl_xor_sync(kFull, mxa, msk));
                mxb = fmaxf(mxb, __shfl_xor_sync(kFull, mxb, msk));
            }
            const float na = fmaxf(m_a, mxa), nb = fmaxf(m_b, mxb);   // finite: valid >= 1
            const float ca = fast_ex2(m_a - na), cb = fast_ex2(m_b - nb);
            m_a = na;
            m_b = nb;
            l_a *= ca;
            l_b *= cb;
#pragma unroll
            for (int mt = 0; mt < 8; ++mt) {
                o[mt][0] *= ca; o[mt][1] *= cb; o[mt][2] *= ca; o[mt][3] *= cb;
            }
#pragma unroll
            for (int u = 0; u < 4; ++u) { xa[u] -= m_a; xb[u] -= m_b; }
          }
        }
        // P' = hi + lo, two fp16 terms: hi = fp16(P'), lo = fp16(P' - hi)
        // (the difference is exact in fp32).  One fp16 term rounds each weight
        // by up to 2^-12 relative, which moves an output made of a few
        // comparable tokens with distant values by up to about 1e-3; the pair
        // carries about 22 significant bits.
        uint32_t p2[4], p2l[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const float pa = fast_ex2(xa[u]), pb = fast_ex2(xb[u]);
            l_a += pa;
            l_b += pb;
            const float svs = sv[u] * ps;
            const float ya = pa * svs, yb = pb * svs;
            __half2 h = __floats2half2_rn(ya, yb);
            const float2 hf = __half22float2(h);
            __half2 hl = __floats2half2_rn(ya - hf.x, yb - hf.y);
            p2[u] = *reinterpret_cast<uint32_t *>(&h);
            p2l[u] = *reinterpret_cast<uint32_t *>(&hl);
        }
        // P'^T B fragments: thread (n = r, c) needs head n, tokens
        // 16ks + {2c, 2c+1} (b0) and 16ks + 8 + {2c, 2c+1} (b1).
        uint32_t pb[2][2], pbl[2][2];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const uint32_t x = __shfl_sync(kFull, p2[u], src0);
            const uint32_t y = __shfl_sync(kFull, p2[u], src1);
            pb[u >> 1][u & 1] = __byte_perm(x, y, hsel);
            const uint32_t xl = __shfl_sync(kFull, p2l[u], src0);
            const uint32_t yl = __shfl_sync(kFull, p2l[u], src1);
            pbl[u >> 1][u & 1] = __byte_perm(xl, yl, hsel);
        }

        // ---- O^T += V^T P'^T ---------------------------------------------
        // thread (r, c): dims 16r .. 16r+15 (m-tile mt: rows r -> dim
        // 16r+2mt, r+8 -> dim 16r+2mt+1), tokens 16ks + {2c,2c+1,2c+8,2c+9}.
        if constexpr (kBits == 3) {
#pragma unroll
        for (int ks = 0; ks < 2; ++ks) {
            // groups 2r and 2r+1 (bytes 6r .. 6r+5, dims 16r .. 16r+15) of
            // tokens 16ks + {2c, 2c+1, 2c+8, 2c+9}; two aligned words always
            // cover the 6 bytes (they start at an even offset)
            uint32_t gw[4][2];
#pragma unroll
            for (int tt = 0; tt < 4; ++tt) {
                const int tok = 16 * ks + (tt & 1) + 8 * (tt >> 1);
                const int off = voff + tok * kBlk;
                const uint32_t lo = ld_u32(vst + (off & ~3)), hi = ld_u32(vst + (off & ~3) + 4);
                const uint32_t sh = (uint32_t)(off & 3) * 8u;
                const uint32_t d0 = __funnelshift_r(lo, hi, sh), d1 = hi >> sh;
                gw[tt][0] = d0;
                gw[tt][1] = __funnelshift_r(d0, d1, 24);
            }
            // m-tile mt: dims 16r + 2mt (rows r) and 16r + 2mt + 1 (rows r + 8)
            // = fields 2 (mt % 4), +1 of group 2r + mt / 4; as in the 4-bit
            // path, each m-tile's lo product is issued after the next m-tile's
            // hi product
            uint32_t pa[4];
#pragma unroll
            for (int mt = 0; mt < 9; ++mt) {
                uint32_t na[4];
                if (mt < 8) {
                    const int gg = mt >> 2;
                    switch (mt & 3) {
                    case 0:
                        na[0] = lvl3<0>(gw[0][gg], gw[1][gg]); na[1] = lvl3<1>(gw[0][gg], gw[1][gg]);
                        na[2] = lvl3<0>(gw[2][gg], gw[3][gg]); na[3] = lvl3<1>(gw[2][gg], gw[3][gg]);
                        break;
                    case 1:
                        na[0] = lvl3<2>(gw[0][gg], gw[1][gg]); na[1] = lvl3<3>(gw[0][gg], gw[1][gg]);
                        na[2] = lvl3<2>(gw[2][gg], gw[3][gg]); na[3] = lvl3<3>(gw[2][gg], gw[3][gg]);
                        break;
                    case 2:
                        na[0] = lvl3<4>(gw[0][gg], gw[1][gg]); na[1] = lvl3<5>(gw[0][gg], gw[1][gg]);
                        na[2] = lvl3<4>(gw[2][gg], gw[3][gg]); na[3] = lvl3<5>(gw[2][gg], gw[3][gg]);
                        break;
                    default:
                        na[0] = lvl3<6>(gw[0][gg], gw[1][gg]); na[1] = lvl3<7>(gw[0][gg], gw[1][gg]);
                        na[2] = lvl3<6>(gw[2][gg], gw[3][gg]); na[3] = lvl3<7>(gw[2][gg], gw[3][gg]);
                        break;
                    }
                    mma16816(o[mt], na[0], na[1], na[2], na[3], pb[ks][0], pb[ks][1]);
                }
                if (mt > 0)
                    mma16816(o[mt - 1], pa[0], pa[1], pa[2], pa[3], pbl[ks][0], pbl[ks][1]);
                if (mt < 8) {
#pragma unroll
                    for (int k = 0; k < 4; ++k) pa[k] = na[k];
                }
            }
        }
        } else {
#pragma unroll
        for (int ks = 0; ks < 2; ++ks) {
            uint32_t xw[4][2];   // [token 2c, 2c+1, 2c+8, 2c+9][word]
#pragma unroll
            for (int tt = 0; tt < 4; ++tt) {
                const int tok = 16 * ks + (tt & 1) + 8 * (tt >> 1);
                const uint8_t *a = vst + voff + tok * kBlk;
                if (tt & 1) {     // odd token: its nibbles are 4-byte aligned
                    xw[tt][0] = ld_u32(a);
                    xw[tt][1] = ld_u32(a + 4);
                } else {                 // even token: 2 bytes past a 4-byte boundary
                    const uint32_t w0 = ld_u32(a - 2), w1 = ld_u32(a + 2), w2 = ld_u32(a + 6);
                    xw[tt][0] = __byte_perm(w0, w1, 0x5432);
                    xw[tt][1] = __byte_perm(w1, w2, 0x5432);
                }
            }
            // The lo products of each group of m-tiles are issued one group
            // later than its hi products, so two MMAs on one accumulator are
            // four MMAs apart.
            uint32_t pa[4], pe[4];                  // the previous group's operands
#pragma unroll
            for (int q4 = 0; q4 < 5; ++q4) {        // byte pairs -> dims 16r + 4q4 .. +3
                uint32_t na[4], ne[4];
                if (q4 < 4) {
                    const uint32_t sel = (q4 & 1) ? 0x7632u : 0x5410u;
                    const int w = q4 >> 1;
                    const uint32_t X = __byte_perm(xw[0][w], xw[1][w], sel);   // pair (2c, 2c+1)
                    const uint32_t Y = __byte_perm(xw[2][w], xw[3][w], sel);   // pair (2c+8, 2c+9)
                    const uint32_t Xs = X >> 8, Ys = Y >> 8;
                    na[0] = lvl_lo(X); na[1] = lvl_hi(X); na[2] = lvl_lo(Y); na[3] = lvl_hi(Y);
                    ne[0] = lvl_lo(Xs); ne[1] = lvl_hi(Xs); ne[2] = lvl_lo(Ys); ne[3] = lvl_hi(Ys);
                    mma16816(o[2 * q4], na[0], na[1], na[2], na[3], pb[ks][0], pb[ks][1]);
                    mma16816(o[2 * q4 + 1], ne[0], ne[1], ne[2], ne[3], pb[ks][0], pb[ks][1]);
                }
                if (q4 > 0) {
                    mma16816(o[2 * q4 - 2], pa[0], pa[1], pa[2], pa[3], pbl[ks][0], pbl[ks][1]);
                    mma16816(o[2 * q4 - 1], pe[0], pe[1], pe[2], pe[3], pbl[ks][0], pbl[ks][1]);
                }
                if (q4 < 4) {
#pragma unroll
                    for (int k = 0; k < 4; ++k) { pa[k] = na[k]; pe[k] = ne[k]; }
                }
            }
        }

        }
        __syncwarp();
        if (stage2_pending) {                 // first chunk: the deferred stage 2
            stage2_pending = false;
            if (lane == 0 && q2 >= 0) {
                bool bad;
                const int64_t o = chunk_ofs(q2, &bad);
                if (bad && q2 < n_chunks) record_status(4u);
                issue(q2, 2, t1_max, o);
            }
        }
        int nxt = q2 >= 0 ? q2 + kTcWarps : -1;
        if (nxt >= n_chunks) nxt = -1;
        if (lane == 0 && nxt >= 0) {          // nxt < n_chunks: real tokens
            bool bad;
            const int64_t o = chunk_ofs(nxt, &bad);
            if (bad) record_status(4u);
            issue(nxt, st, t1, o);
        }
        q0 = q1;
        q1 = q2;
        q2 = nxt;
        if (++st == kTcStages) { st = 0; phase ^= 1u; }
    }

    // Every copy still queued (issued ahead for chunks beyond the real
    // length, or left by an aborted loop) lands before the ring is reused;
    // with no chunk consumed, the deferred stage 2 was never issued.
#pragma unroll
    for (int j = 0; j < kTcStages; ++j) {
        const int qj = j == 0 ? q0 : (j == 1 ? q1 : q2);
        if (qj < 0 || (j == 2 && stage2_pending)) continue;
        int sj = st + j;
        uint32_t par = phase;
        if (sj >= kTcStages) { sj -= kTcStages; par ^= 1u; }
        if (!mbar_wait_bounded(bar_w + 8 * sj, par) && lane == 0) record_status(7u);
    }

    // ---- warp totals, CTA merge, partial write ----------------------------
#pragma unroll
    for (int msk = 4; msk < 32; msk <<= 1) {
        l_a += __shfl_xor_sync(kFull, l_a, msk);
        l_b += __shfl_xor_sync(kFull, l_b, msk);
    }
    if (aborted) { m_a = m_b = -INFINITY; }
    __syncthreads();     // every warp is done with its ring
    // Each lane's 32 accumulators go out as eight 16-byte stores to its own
    // row of 36 floats (eight lanes per wavefront, no bank conflicts): (head
    // h, dim d) is element 2 (d % 16) + h % 2 of fragment lane 4 (d / 16) + h / 2.
    constexpr int kLaneStride = 36;
    float *o_w = reinterpret_cast<float *>(ring);                       // [W][32][36]
    float *m_w = o_w + kTcWarps * 32 * kLaneStride;                      // [W][8]
    float *l_w = m_w + kTcWarps * kMaxGroup;                             // [W][8]
    float *wt = l_w + kTcWarps * kMaxGroup;                              // [W][8]
    float2 *ml_h = reinterpret_cast<float2 *>(wt + kTcWarps * kMaxGroup);  // [8]
    {
        // sum_t P'_t (2n - 15) = 2^11 sum_t P'_t (2n - 15) 2^-11, and 1 / ps
        // (a power of two, exact) puts every warp's rows in the units of
        // p S_v before the warps are merged
        const float osc = kVLevelScale * (ps > 0.f ? pow2_inv(ps) : 1.0f);
        float4 *mine = reinterpret_cast<float4 *>(o_w + (warp * 32 + lane) * kLaneStride);
#pragma unroll
        for (int mt = 0; mt < 8; ++mt)
            mine[mt] = make_float4(o[mt][0] * osc, o[mt][1] * osc, o[mt][2] * osc, o[mt][3] * osc);
    }
    if (r == 0) {
        m_w[warp * kMaxGroup + 2 * c] = m_a;
        m_w[warp * kMaxGroup + 2 * c + 1] = m_b;
        l_w[warp * kMaxGroup + 2 * c] = l_a;
        l_w[warp * kMaxGroup + 2 * c + 1] = l_b;
    }
    __syncthreads();
    // per-(warp, head) weights 2^(m_w - M_h) and each head's (M, L), in warp
    // 0: lane = (quarter wq of the warps, head h)
    if (warp == 0) {
        const int h = lane & 7, wq = lane >> 3;
        float M = -INFINITY;
#pragma unroll
        for (int k = 0; k < kTcWarps / 4; ++k)
            M = fmaxf(M, m_w[(wq * (kTcWarps / 4) + k) * kMaxGroup + h]);
        M = fmaxf(M, __shfl_xor_sync(kFull, M, 8));
        M = fmaxf(M, __shfl_xor_sync(kFull, M, 16));
        float L = 0.f;
#pragma unroll
        for (int k = 0; k < kTcWarps / 4; ++k) {
            const int i = (wq * (kTcWarps / 4) + k) * kMaxGroup + h;
            const float mw = m_w[i];
            const float f = (mw == -INFINITY || M == -INFINITY) ? 0.f : exp2f(mw - M);
            wt[i] = f;
            L = fmaf(f, l_w[i], L);
        }
        L += __shfl_xor_sync(kFull, L, 8);
        L += __shfl_xor_sync(kFull, L, 16);
        if (wq == 0) ml_h[h] = make_float2(M, L);
    }
    __syncthreads();
    // One warp per (16-dim block rb, head pair cb): lane 2 j + k holds head
    // 2 cb + k, dim 16 rb + j, which is element `lane` of fragment lane
    // 4 rb + cb, so the 32 loads of a warp hit 32 different banks.  The
    // levels carry a factor 15.
    for (int it = warp; it < 8 * ((G + 1) >> 1); it += kTcWarps) {
        const int rb = it & 7, cb = it >> 3;
        const int h = 2 * cb + (lane & 1), d = 16 * rb + (lane >> 1);
        if (h < G) {
            const float *src = o_w + (4 * rb + cb) * kLaneStride + lane;
            float O = 0.f;
#pragma unroll
            for (int w = 0; w < kTcWarps; ++w)
                O = fmaf(wt[w * kMaxGroup + h], src[w * 32 * kLaneStride], O);
            const int64_t row = ((int64_t)s * p.Hq + g * G + h) * p.n_splits + split;
            if (in_extent(row, 1, p.part_rows)) {
                // the block factor is S/15 (S/7 for 3 bits)
                p.part_o[row * kD + d] = O * (kBits == 4 ? 1.0f / 15.0f : 1.0f / 7.0f);
                if (d == 0) p.part_ml[row] = ml_h[h];
            }
        }
    }
}

}  // namespace tbq4

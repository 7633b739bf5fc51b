// decode_mq.cuh -- multi-query decode (q_len 2-4 new tokens per sequence, as
// for speculative verification) over TBQ4 caches, on tcgen05.
//
// Decode with q_len query tokens reads the same cache once but multiplies
// the contractions by q_len.  With the G heads of a KV head that makes up to
// 32 query rows per K/V tile, which the 5th-generation tensor cores take as
// one wider N at no extra operand traffic:
//
//   S^T (128 tokens x 96)  = A_K (128 tokens x 128 B) . B_q^T      kind::i8
//   O^T (128 dims x 32)   += V^T (128 dims x 128 tokens) . P'^T    kind::f16
//
// The operands are exactly those of the single-query decode: A_K row = [64
// raw nibble bytes | the same & 0x0F]; B_q rows 32 pc + c = piece pc of the
// 18-bit weights u = q_odd (raw bytes) and w = 16 q_even - q_odd (low
// nibbles) of query row c, so S column 32 pc + c is piece pc of 16 sum_d
// n_d q_int,d (exact); V^T holds (2n - 15) 2^-11 exactly in fp16; P' = p S_v
// ps with ps a power of two fitted to the V scales, as two fp16 terms hi + lo
// (N = 64: 32 rows each); O = 2^11 O''.  Query row c = i G + h is query
// token i (of q_len) for head h of the KV group; token i sits at position
// len - q_len + i and sees keys [0, len - q_len + i] (bottom-right causal,
// as the chunked prefill of the same pages: trefon.com, "Kontekst 262K na
// jednej RTX 4090", section "Konfiguracja", speculative drafts).
//
// One CTA = one (sequence, KV head, split), one CTA per SM, 24 warps:
//   warp 0      producer: cp.async.bulk of raw K and V rows, 32-row pieces
//   warp 1      tensor-memory allocation; lane 0 issues every tcgen05.mma,
//               QK and PV in whatever order their inputs become ready
//   warps 4-7   dequantisation into the K and V^T operand tiles
//   warps 8-23  softmax: four warpgroups, query rows 8 wg .. 8 wg + 7;
//               thread = token = TMEM lane of S, at the end dimension = TMEM
//               lane of O
// The running max per row is shared by the CTA and only moved (O rescaled
// in tensor memory) when a logit exceeds it by more than 2^3.
#pragma once
#include "common.cuh"
#include "decode.cuh"
#include "tcgen05.cuh"

namespace tbq4 {
namespace dmq {

constexpr int kThreads = 768;
constexpr int kTile = 128;                              // tokens per tile
constexpr int kRawBytes = kTile * kBlockBytes;          // 8448
constexpr int kRawStages = 4;
constexpr int kPieceRows = 32;                          // rows per bulk copy (2,112 B)
constexpr int kRawStageBytes = 2 * kRawBytes + 16;      // K | V | pad
constexpr int kDeqWarp0 = 4, kDeqWarps = 4;
constexpr int kSoftWarp0 = 8, kSoftWarps = 16;
constexpr int kCols = 32;                               // query rows (q_len x G <= 32)
constexpr int kSCols = 3 * kCols;                       // S columns: three pieces per row
constexpr int kMaxQLen = 4;
constexpr uint32_t kSpin = 1u << 22;
constexpr float kRescale = 8.0f;                        // log2 units
constexpr int kQBits = 18;                              // |q_int| <= 2^18
// Registers per thread after the prologue, per warpgroup: producer / MMA
// (warps 0-3), dequantisation (4-7), softmax (8-23).  The sum over the 24
// warps must fit in what the CTA was launched with, 768 threads x 80.
constexpr uint32_t kRegsCtl = 24, kRegsDeq = 72, kRegsSoft = 96;
static_assert(4 * kRegsCtl + 4 * kRegsDeq + 16 * kRegsSoft <= 24 * 80,
              "register split exceeds the launch budget");

// One operand buffer (double-buffered): K tile, V^T tile, P'^T tile, the
// tile's S_k and S_v.  Offsets from a 1024-aligned base.
constexpr int kKTile = 0;                               // 128 rows x 128 B, 1 atom
constexpr int kVTile = kKTile + kTile * 128;            // 128 rows x 256 B, 2 atoms
constexpr int kPTile = kVTile + kTile * 256;            // 64 rows x 256 B, 2 atoms
constexpr int kPRows = 2 * kCols;                       // P' as hi (rows c), lo (kCols + c)
constexpr int kPAtom = kPRows * 128;                    // 8 KB
constexpr int kSig = kPTile + 2 * kPAtom;               // S_k[128], S_v[128] floats
constexpr int kBufBytes = kSig + 2 * kTile * 4;         // 58,368
static_assert(kVTile % 1024 == 0 && kPTile % 1024 == 0 && kBufBytes % 1024 == 0, "align");

constexpr int kOffQB = 0;                               // B_q: 96 rows x 128 B
constexpr int kOffBuf = kSCols * 128;                   // 12 KB
constexpr int kOffRaw = kOffBuf + 2 * kBufBytes;
constexpr int kOffQPar = kOffRaw + kRawStages * kRawStageBytes;   // [32][2] floats
constexpr int kOffFlags = kOffQPar + kCols * 2 * 4;               // [2][16] ints
constexpr int kOffXch = kOffFlags + 2 * kSoftWarps * 4;           // [4][32] floats
constexpr int kOffXfin = kOffXch + 4 * kCols * 4;                 // [4][64] floats
constexpr int kOffDsv = kOffXfin + 4 * 2 * kCols * 4;             // [2][4] floats
constexpr int kOffTps = kOffDsv + 2 * 4 * 4;                       // [2][2] floats
constexpr int kOffBar = kOffTps + 2 * 2 * 4;
constexpr int kSoftGroups = kSoftWarps / 4;            // warpgroups, 8 query rows each
constexpr int kNumBars = 2 * kRawStages + 5 * 2 + 3 * kSoftGroups + 1 + 2;   // + vote, max per
                                                                            // group, final, S_v max
constexpr int kOffTmemPtr = kOffBar + kNumBars * 8;
constexpr int kSmemBytes = kOffTmemPtr + 16 + 1024;     // + alignment slack
static_assert(kOffBuf % 1024 == 0 && kOffRaw % 16 == 0 && kOffBar % 8 == 0, "align");
static_assert(kSmemBytes <= 232448, "shared memory budget");

// tensor memory columns: S buffers at 0 and 96 (s32), O at 192 (64 x f32: the
// products with P' hi at 192 + c, with P' lo at 224 + c)
constexpr uint32_t kTmemCols = 256;
constexpr uint32_t kTmemO = 2 * kSCols;

// Instruction descriptors (PTX ISA, tcgen05 instruction descriptor):
// [4,6) D format, [7,10) A format, [10,13) B format, [15]/[16] A/B major
// (0 = K-major), [17,23) N >> 3, [24,29) M >> 4.
//   kind::i8:  D s32 (2), A u8 (0), B s8 (1), M = 128, N = 96
//   kind::f16: D f32 (1), A f16 (0), B f16 (0), M = 128, N = 64 (P' hi and lo)
constexpr uint32_t kIdescQK = (2u << 4) | (0u << 7) | (1u << 10) | ((uint32_t)(kSCols >> 3) << 17) |
                              ((128u >> 4) << 24);
constexpr uint32_t kIdescPV = (1u << 4) | (0u << 7) | (0u << 10) | ((uint32_t)(kPRows >> 3) << 17) |
                              ((128u >> 4) << 24);

__device__ __forceinline__ void mma_i8(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                       uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
        " tcgen05.mma.cta_group::1.kind::i8 [%0], %1, %2, %3, p;\n}\n"
        ::"r"(d_tmem), "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// Byte offset of byte k of row r in a K-major tile with the 128-byte
// swizzle (rows of 128 bytes, 8-row groups 1024 bytes apart, 16-byte chunks
// XOR-ed with r % 8); tiles wider than 128 bytes are atoms side by side.
__device__ __forceinline__ uint32_t sw128(int r, int k, int atom_bytes) {
    return (uint32_t)((k >> 7) * atom_bytes + (r >> 3) * 1024 + (r & 7) * 128 +
                      ((((k & 127) >> 4) ^ (r & 7)) << 4) + (k & 15));
}

__device__ __forceinline__ uint32_t lds32(uint32_t a) {
    uint32_t v;
    asm volatile("ld.shared.b32 %0, [%1];" : "=r"(v) : "r"(a) : "memory");
    return v;
}
__device__ __forceinline__ uint32_t lds16(uint32_t a) {
    uint16_t v;
    asm volatile("ld.shared.u16 %0, [%1];" : "=h"(v) : "r"(a) : "memory");
    return v;
}
__device__ __forceinline__ void sts16(uint32_t a, uint16_t v) {
    asm volatile("st.shared.u16 [%0], %1;" ::"r"(a), "h"(v) : "memory");
}
__device__ __forceinline__ void sts128(uint32_t a, uint32_t x, uint32_t y, uint32_t z,
                                       uint32_t w) {
    asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(a), "r"(x), "r"(y), "r"(z),
                 "r"(w)
                 : "memory");
}

// V levels (2n - 15) 2^-11 in fp16 from nibbles in bits 0-3 (lo) or 4-7 (hi)
// of bytes 0 and 2: the masked halves are the subnormals n 2^-24 and
// 16 n 2^-24, scaled and shifted by one exact HFMA2 (the results are normal
// fp16 numbers with at most 4 significant bits).
__device__ __forceinline__ uint32_t hfma2u(uint32_t x, uint32_t a, uint32_t b) {
    __half2 r = __hfma2(*reinterpret_cast<__half2 *>(&x), *reinterpret_cast<__half2 *>(&a),
                        *reinterpret_cast<__half2 *>(&b));
    return *reinterpret_cast<uint32_t *>(&r);
}
__device__ __forceinline__ uint32_t vlo(uint32_t v) {
    return hfma2u(v & 0x000F000Fu, 0x74007400u /* 2^14 */, 0x9F809F80u /* -15 2^-11 */);
}
__device__ __forceinline__ uint32_t vhi(uint32_t v) {
    return hfma2u(v & 0x00F000F0u, 0x64006400u /* 2^10 */, 0x9F809F80u);
}

__device__ __forceinline__ void split3(int x, int &c0, int &c1, int &c2) {
    c0 = ((x + 128) & 255) - 128;
    const int x1 = (x - c0) >> 8;
    c1 = ((x1 + 128) & 255) - 128;
    c2 = (x1 - c1) >> 8;
}

__global__ void __launch_bounds__(kThreads, 1)
decode_mq_kernel(const AttnParams p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
    const uint32_t sbase = smem_u32(smem);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    // the dependent combine kernel may be scheduled from now on
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

    const int split = blockIdx.x, g = blockIdx.y, s = blockIdx.z;
    const int G = p.G, QL = p.q_len;
    const int NQ = G * QL;                              // query rows, <= 32 (host)
    const int32_t len = seq_length(p, s);
    const int32_t t0 = split * p.split_tokens;
    const int32_t t1 = min(len, t0 + p.split_tokens);
    const int n_tiles = t1 > t0 ? (t1 - t0 + kTile - 1) / kTile : 0;
    // this (sequence, KV head)'s cache rows start kb - p.k bytes into both caches
    const uint8_t *kb = p.k + s * p.seq_stride + g * p.head_stride;

    // barriers
    const uint32_t bar0 = sbase + kOffBar;
    auto raw_full = [&](int i) { return bar0 + 8 * i; };
    auto raw_empty = [&](int i) { return bar0 + 8 * (kRawStages + i); };
    const uint32_t bx = bar0 + 8 * 2 * kRawStages;
    auto op_full = [&](int b) { return bx + 8 * b; };          // dequant -> MMA, softmax
    auto s_full = [&](int b) { return bx + 8 * (2 + b); };     // QK done -> softmax
    auto s_empty = [&](int b) { return bx + 8 * (4 + b); };    // S read -> MMA
    auto p_full = [&](int b) { return bx + 8 * (6 + b); };     // P' written -> MMA
    auto tile_free = [&](int b) { return bx + 8 * (8 + b); };  // PV done -> buffer free
    // Exchanges between warps of one role use mbarriers with bounded waits
    // (a warp that gives up on a wait must not leave the others blocked).  A
    // softmax warpgroup owns its query rows, so its running maxima are agreed
    // among its own four warps.
    auto vote = [&](int b, int wgi) { return bx + 8 * (10 + 2 * wgi + b); };   // grow flags
    auto mx_bar = [&](int wgi) { return bx + 8 * (10 + 2 * kSoftGroups + wgi); }; // tile maxima
    const uint32_t fin_bar = bx + 8 * (10 + 3 * kSoftGroups);                 // final sums
    auto sv_bar = [&](int b) { return bx + 8 * (11 + 3 * kSoftGroups + b); }; // dequant S_v max
    uint32_t *tmem_ptr = reinterpret_cast<uint32_t *>(smem + kOffTmemPtr);
    float *qpar = reinterpret_cast<float *>(smem + kOffQPar);

    if (threadIdx.x == 0) {
        for (int i = 0; i < kRawStages; ++i) {
            mbar_init(raw_full(i), 1);
            mbar_init(raw_empty(i), kDeqWarps);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(op_full(b), kDeqWarps);
            mbar_init(s_full(b), 1);
            mbar_init(s_empty(b), kSoftWarps);
            mbar_init(p_full(b), kSoftWarps);
            mbar_init(tile_free(b), 1);
            for (int w = 0; w < kSoftGroups; ++w) mbar_init(vote(b, w), 4);
        }
        for (int w = 0; w < kSoftGroups; ++w) mbar_init(mx_bar(w), 4);
        mbar_init(fin_bar, kSoftWarps);
        for (int b = 0; b < 2; ++b) mbar_init(sv_bar(b), kDeqWarps);
        fence_barrier_init();
    }
    if (warp == 1) {
        tc::tmem_alloc(smem_u32(tmem_ptr), kTmemCols);
        tc::tmem_relinquish();
    }
    // zero B_q (rows of absent query rows stay 0) and the P' tiles (rows of
    // absent query rows are never written)
    for (int i = threadIdx.x; i < kSCols * 32; i += kThreads)
        reinterpret_cast<uint32_t *>(smem + kOffQB)[i] = 0u;
    for (int i = threadIdx.x; i < 2 * (2 * kPAtom / 4); i += kThreads)
        reinterpret_cast<uint32_t *>(smem + kOffBuf + (i / (2 * kPAtom / 4)) * kBufBytes + kPTile)
            [i % (2 * kPAtom / 4)] = 0u;
    __syncthreads();

    // ---- q: rotate, 18-bit integer, pieces of the weights u and w ----------
    // Query row c = i G + h: token i of the new ones, head h of the group.
    // q_int = rint(q_rot * 2^(18-e)) with 2^e > max|q_rot|.  Dimension pair j
    // is raw byte j: u_j = q_int[2j+1] weighs the raw byte (lo + 16 hi), w_j =
    // 16 q_int[2j] - q_int[2j+1] its low nibble; both in three signed bytes.
    // B_q row 32 pc + c, byte j: piece pc of u_j (j < 64) or w_(j-64).
    for (int c = warp; c < kCols; c += kThreads / 32) {
        if (c < NQ) {
            const int i = c / G, h = c - i * G;
            const uint32_t sbits = lane_sign_bits(p.sign_lo, p.sign_hi, lane);
            const int64_t base = (((int64_t)s * QL + i) * p.Hq + g * G + h) * kD + 4 * lane;
            float v[4];
#pragma unroll
            for (int k = 0; k < 4; ++k) v[k] = load_q(p, base + k);
            warp_rotate128(v, sbits, lane);
            const float mx =
                warp_max(fmaxf(fmaxf(fabsf(v[0]), fabsf(v[1])), fmaxf(fabsf(v[2]), fabsf(v[3]))));
            int e = 0;
            if (mx > 0.f) frexpf(mx, &e);
            int qi[4], qsum = 0;
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                qi[k] = __float2int_rn(ldexpf(v[k], kQBits - e));
                qsum += qi[k];
            }
            int uc[2][3], wc[2][3];
#pragma unroll
            for (int j = 0; j < 2; ++j) {
                split3(qi[2 * j + 1], uc[j][0], uc[j][1], uc[j][2]);
                split3(16 * qi[2 * j] - qi[2 * j + 1], wc[j][0], wc[j][1], wc[j][2]);
            }
#pragma unroll
            for (int pc = 0; pc < 3; ++pc) {
                const int row = kCols * pc + c;
                const uint16_t u2 = (uint16_t)((uc[0][pc] & 255) | ((uc[1][pc] & 255) << 8));
                const uint16_t w2 = (uint16_t)((wc[0][pc] & 255) | ((wc[1][pc] & 255) << 8));
                sts16(sbase + kOffQB + sw128(row, 2 * lane, 0), u2);
                sts16(sbase + kOffQB + sw128(row, 64 + 2 * lane, 0), w2);
            }
            qsum = __reduce_add_sync(kFull, qsum);
            if (lane == 0) {
                // log2 logit = (2 S - 15 sum q) * S_k * scale * log2(e) / 15 * 2^(e-18),
                // and the MMAs return 16 S
                const float fh = p.scale_log2 * (1.0f / 15.0f) * ldexpf(1.0f, e - kQBits);
                qpar[2 * c + 0] = 0.125f * fh;
                qpar[2 * c + 1] = -15.0f * (float)qsum * fh;
            }
        } else if (lane == 0) {
            qpar[2 * c] = 0.f;
            qpar[2 * c + 1] = 0.f;
        }
    }
    fence_proxy_async();                // B_q and the zeroed P' rows are read by the MMAs
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tmem = *tmem_ptr;

    if (warp < 4) {
      tc::regs_dec<kRegsCtl>();
      if (warp == 0) {
        // ======================= producer ====================================
        // Each tile's K and V rows go as 32-row pieces, one per lane, so the
        // copy engine has many requests in flight.
        for (int j = 0; j < n_tiles; ++j) {
            const int st = j % kRawStages;
            if (j >= kRawStages &&
                !mbar_wait_bounded(raw_empty(st), ((j / kRawStages) - 1) & 1, kSpin)) {
                record_status(7u);
                break;
            }
            const int32_t tj = t0 + j * kTile;
            // whole 8-row groups (capacity is a multiple of 8): 528-byte multiples
            const int rows = (min(kTile, t1 - tj) + 7) & ~7;
            const uint32_t dst = sbase + kOffRaw + st * kRawStageBytes;
            if (lane == 0) {
                fence_proxy_async();
                mbar_expect_tx(raw_full(st), 2u * (uint32_t)rows * kBlockBytes);
            }
            __syncwarp();
            const int piece = lane >> 1, kv = lane & 1;
            const int r0 = piece * kPieceRows;
            if (piece < kTile / kPieceRows && r0 < rows) {
                const uint32_t nb = (uint32_t)(min(kPieceRows, rows - r0)) * kBlockBytes;
                int64_t off = (kb - p.k) + (int64_t)(tj + r0) * kBlockBytes;
                if constexpr (kDebugBounds) off = checked_off(off, nb, p.cache_bytes);
                bulk_g2s(dst + kv * kRawBytes + r0 * kBlockBytes, (kv ? p.v : p.k) + off, nb,
                         raw_full(st));
            }
        }
    } else if (warp == 1) {
        // ======================= MMA issuer ==================================
        // QK(j) needs the operand tiles of j and a free S buffer; PV(j) needs
        // P'(j).  Both are polled, so neither waits behind the other.
        if (lane == 0 && n_tiles > 0) {
            int jq = 0, jp = 0;
            uint32_t idle = 0;
            while (jp < n_tiles) {
                bool moved = false;
                if (jq < n_tiles && jq <= jp + 1) {
                    const int b = jq & 1;
                    if (mbar_test(op_full(b), (jq >> 1) & 1) &&
                        (jq < 2 || mbar_test(s_empty(b), ((jq >> 1) - 1) & 1))) {
                        tc::fence_after_sync();
                        const uint32_t kt = sbase + kOffBuf + b * kBufBytes + kKTile;
#pragma unroll
                        for (int ki = 0; ki < 4; ++ki)
                            mma_i8(tmem + kSCols * b, tc::desc_sw128(kt + 32 * ki),
                                   tc::desc_sw128(sbase + kOffQB + 32 * ki), kIdescQK, ki > 0);
                        tc::mma_commit(s_full(b));
                        ++jq;
                        moved = true;
                    }
                }
                if (jp < jq) {
                    const int b = jp & 1;
                    if (mbar_test(p_full(b), (jp >> 1) & 1)) {
                        tc::fence_after_sync();
                        const uint32_t vt = sbase + kOffBuf + b * kBufBytes + kVTile;
                        const uint32_t pt = sbase + kOffBuf + b * kBufBytes + kPTile;
#pragma unroll
                        for (int kk = 0; kk < 8; ++kk)
                            tc::mma_ss(tmem + kTmemO,
                                       tc::desc_sw128(vt + (kk >> 2) * 16384 + (kk & 3) * 32),
                                       tc::desc_sw128(pt + (kk >> 2) * kPAtom + (kk & 3) * 32),
                                       kIdescPV, (jp > 0 || kk > 0) ? 1u : 0u);
                        tc::mma_commit(tile_free(b));
                        ++jp;
                        moved = true;
                    }
                }
                if (moved) {
                    idle = 0;
                } else if (++idle > kSpin) {
                    record_status(7u);
                    break;
                }
            }
        }
      }
    } else if (warp >= kDeqWarp0 && warp < kDeqWarp0 + kDeqWarps) {
        tc::regs_dec<kRegsDeq>();
        // ======================= dequantisation ==============================
        const int d = threadIdx.x - 32 * kDeqWarp0;     // 0..127
        // P' = p S_v ps (fp16) with ps a power of two, the largest that keeps
        // P' <= 2^15 for every V scale seen so far (p <= 2^8): S_v ps <= 2^7.
        // A fixed ps = 2^-8 (room for S_v = 65504) would leave the weights of
        // most tokens among the fp16 subnormals, whose absolute spacing costs
        // the output up to 1e-3.  These warps see every tile's scales first:
        // they keep ps, hand the softmax S_v ps per token and, per tile, the
        // factor by which ps shrank (the softmax rescales O and R by it) and
        // the tile's ps.  0 until a nonzero S_v arrives.
        float ps = 0.f;
        float *dsv = reinterpret_cast<float *>(smem + kOffDsv);      // [2][4] warp maxima
        float *tps = reinterpret_cast<float *>(smem + kOffTps);      // [2] x (factor, ps)
        for (int j = 0; j < n_tiles; ++j) {
            const int st = j % kRawStages, b = j & 1;
            if (!mbar_wait_bounded(raw_full(st), (j / kRawStages) & 1, kSpin)) { record_status(7u); break; }
            if (j >= 2 && !mbar_wait_bounded(tile_free(b), ((j >> 1) - 1) & 1, kSpin)) {
                record_status(7u);
                break;
            }
            const uint32_t raw = sbase + kOffRaw + st * kRawStageBytes;
            const uint32_t buf = sbase + kOffBuf + b * kBufBytes;
            // K tile, row t = d: [raw nibble bytes 0-63 | the same & 0x0F]; the
            // row's bytes start 2 past a 4-byte boundary for even t
            {
                const int t = d;
                const uint32_t kt = buf + kKTile;
                const uint32_t m4 = 0x0F0F0F0Fu;
#pragma unroll
                for (int hh = 0; hh < 2; ++hh) {
                    const uint32_t src = raw + t * kBlockBytes + 2 + 32 * hh;
                    const uint32_t a0 = src & ~3u, sh = (src & 3u) * 8u;
                    uint32_t w[9];
#pragma unroll
                    for (int i = 0; i < 9; ++i) w[i] = lds32(a0 + 4 * i);
                    uint32_t x[8];
#pragma unroll
                    for (int i = 0; i < 8; ++i) x[i] = __funnelshift_r(w[i], w[i + 1], sh);
                    sts128(kt + sw128(t, 32 * hh, 0), x[0], x[1], x[2], x[3]);
                    sts128(kt + sw128(t, 32 * hh + 16, 0), x[4], x[5], x[6], x[7]);
                    sts128(kt + sw128(t, 64 + 32 * hh, 0), x[0] & m4, x[1] & m4, x[2] & m4, x[3] & m4);
                    sts128(kt + sw128(t, 64 + 32 * hh + 16, 0), x[4] & m4, x[5] & m4, x[6] & m4,
                           x[7] & m4);
                }
                // the token's block scales S_k and S_v (tokens past the
                // split's end count as S_v = 0)
                float *sig = reinterpret_cast<float *>(smem + kOffBuf + b * kBufBytes + kSig);
                sig[t] = __half2float(__ushort_as_half((uint16_t)lds16(raw + t * kBlockBytes)));
                const float sv = t0 + j * kTile + t < t1
                    ? __half2float(__ushort_as_half((uint16_t)lds16(raw + kRawBytes + t * kBlockBytes)))
                    : 0.f;
                // the tile's largest S_v, over the four dequantisation warps
                const float wmx = warp_max(sv);
                if (lane == 0) {
                    dsv[4 * b + (warp - kDeqWarp0)] = wmx;
                    mbar_arrive(sv_bar(b));
                }
                if (!mbar_wait_bounded(sv_bar(b), (j >> 1) & 1, kSpin)) {
                    record_status(7u);
                    break;
                }
                const float smx = fmaxf(fmaxf(dsv[4 * b], dsv[4 * b + 1]),
                                        fmaxf(dsv[4 * b + 2], dsv[4 * b + 3]));
                float f = 1.f;
                if (ps == 0.f ? smx > 0.f : smx * ps > 128.0f) {
                    const float nps = pow2_floor(__fdividef(128.0f, smx));
                    f = ps == 0.f ? 1.f : pow2_ratio(nps, ps);
                    ps = nps;
                }
                sig[kTile + t] = sv * ps;
                if (d == 0) { tps[2 * b] = f; tps[2 * b + 1] = ps; }
            }
            // V^T tile, row = dim, tokens along K; unit = (tokens 8 tg .. +7,
            // nibble bytes 2 bp, 2 bp + 1 = dims 4 bp .. +3).  Two tokens' bytes
            // are interleaved with PRMT so one fp16x2 holds a dimension of a
            // token pair; 4 dims x 8 tokens leave as four 16-byte stores.
#pragma unroll 1
            for (int u = d; u < 16 * 32; u += 32 * kDeqWarps) {
                const int tg = u & 15, bp = u >> 4;
                const uint32_t vsrc = raw + kRawBytes + (8 * tg) * kBlockBytes + 2 + 2 * bp;
                uint32_t w[8];
#pragma unroll
                for (int i = 0; i < 8; ++i) w[i] = lds16(vsrc + i * kBlockBytes);
                uint32_t o[4][4];                 // [dim 4 bp + e][token pair]
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const uint32_t X = __byte_perm(w[2 * i], w[2 * i + 1], 0x5410);  // a.b0 a.b1 b.b0 b.b1
                    const uint32_t Xs = X >> 8;
                    o[0][i] = vlo(X);
                    o[1][i] = vhi(X);
                    o[2][i] = vlo(Xs);
                    o[3][i] = vhi(Xs);
                }
                const uint32_t vt = buf + kVTile;
#pragma unroll
                for (int e = 0; e < 4; ++e)
                    sts128(vt + sw128(4 * bp + e, 16 * tg, 16384), o[e][0], o[e][1], o[e][2], o[e][3]);
            }
            fence_proxy_async();            // the tiles are read by the tensor core
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(op_full(b));
                mbar_arrive(raw_empty(st));
            }
        }
    } else if (warp >= kSoftWarp0) {
        tc::regs_inc<kRegsSoft>();
        // ======================= softmax =====================================
        const int ws = warp - kSoftWarp0;                   // 0..15
        const int wg = ws >> 2;                             // query rows 8 wg .. 8 wg + 7
        const int q4 = warp & 3;                            // TMEM lane quarter
        const int t = 32 * q4 + lane;                       // token, later dimension
        const uint32_t t_lane = tmem + ((uint32_t)(32 * q4) << 16);
        int *flags = reinterpret_cast<int *>(smem + kOffFlags);       // [2][16]
        float *xch = reinterpret_cast<float *>(smem + kOffXch);       // [4][32]
        float *xfin = reinterpret_cast<float *>(smem + kOffXfin);     // [4][64]
        float f2[8], bh[8], m[8], lp[8];
        int32_t lim[8];                                     // keys of row c: [0, lim)
#pragma unroll
        for (int k = 0; k < 8; ++k) {
            const int c = 8 * wg + k;
            f2[k] = qpar[2 * c];
            bh[k] = qpar[2 * c + 1];
            m[k] = -INFINITY;
            lp[k] = 0.f;
            lim[k] = c < NQ ? len - QL + c / G + 1 : 0;
        }
        uint32_t mx_phase = 0;
        bool ok = true;
        for (int j = 0; j < n_tiles; ++j) {
            const int b = j & 1;
            const uint32_t par = (j >> 1) & 1;
            if (!mbar_wait_bounded(s_full(b), par, kSpin) || !mbar_wait_bounded(op_full(b), par, kSpin)) {
                record_status(7u);
                ok = false;
                break;
            }
            tc::fence_after_sync();
            uint32_t a0[8], a1[8], a2[8];          // pieces 0, 1, 2 of 16 S for the 8 rows
            tc::tmem_ld8(t_lane + kSCols * b + 8 * wg, a0);
            tc::tmem_ld8(t_lane + kSCols * b + kCols + 8 * wg, a1);
            tc::tmem_ld8(t_lane + kSCols * b + 2 * kCols + 8 * wg, a2);
            tc::tmem_wait_ld();
            tc::fence_before_sync();
            __syncwarp();
            if (lane == 0) mbar_arrive(s_empty(b));

            if (8 * wg >= NQ) {                 // no query row of this warpgroup is in use
                __syncwarp();
                if (lane == 0) mbar_arrive(p_full(b));
                continue;
            }
            const float *sig = reinterpret_cast<const float *>(smem + kOffBuf + b * kBufBytes + kSig);
            const int32_t ta = t0 + j * kTile + t;            // absolute token
            const float sk = sig[t], sv = ta < t1 ? sig[kTile + t] : 0.f;   // sv: S_v ps
            float tt[8], x[8];
            bool grow = false;
#pragma unroll
            for (int k = 0; k < 8; ++k) {
                const float sc = fmaf((float)(int)a2[k], 65536.0f,
                                      (float)((int)a1[k] * 256 + (int)a0[k]));   // 16 S
                tt[k] = fmaf(sc, f2[k], bh[k]);                 // log2 logit / S_k
                x[k] = ta < lim[k] ? fmaf(tt[k], sk, -m[k]) : -INFINITY;
                grow |= x[k] > kRescale;
            }
            // Does any logit of the tile exceed its row's running max by more
            // than 2^3?  One flag per warp, exchanged through an mbarrier.
            const bool wgrow = __any_sync(kFull, grow);
            if (lane == 0) flags[kSoftWarps * b + ws] = wgrow ? 1 : 0;
            __syncwarp();
            if (lane == 0) mbar_arrive(vote(b, wg));
            if (!mbar_wait_bounded(vote(b, wg), par, kSpin)) { record_status(7u); ok = false; break; }
            int any = 0;
#pragma unroll
            for (int w = 0; w < 4; ++w) any |= flags[kSoftWarps * b + 4 * wg + w];
            // ps shrank by fsv (a power of two) on this tile: O and R move with it
            const float fsv = reinterpret_cast<const float *>(smem + kOffTps)[2 * b];
            if (any || fsv != 1.f) {
                // move the maxima to the tile's (where larger) and rescale
                float lg[8];
#pragma unroll
                for (int k = 0; k < 8; ++k) {
                    lg[k] = x[k] == -INFINITY ? -INFINITY : tt[k] * sk;
                    const float wm = warp_max(lg[k]);
                    if (lane == 0) xch[kCols * q4 + 8 * wg + k] = wm;
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(mx_bar(wg));
                if (!mbar_wait_bounded(mx_bar(wg), mx_phase, kSpin)) { record_status(7u); ok = false; break; }
                mx_phase ^= 1u;
                uint32_t cs[8];
#pragma unroll
                for (int k = 0; k < 8; ++k) {
                    const int c = 8 * wg + k;
                    const float tm = fmaxf(fmaxf(xch[c], xch[kCols + c]),
                                           fmaxf(xch[2 * kCols + c], xch[3 * kCols + c]));
                    const float nm = fmaxf(m[k], tm);
                    float cc = (m[k] == -INFINITY) ? 0.f : tc::ex2(m[k] - nm);
                    if (nm == -INFINITY) cc = 1.f;
                    m[k] = nm;
                    lp[k] *= cc;
                    cs[k] = __float_as_uint(cc * fsv);
                    x[k] = lg[k] == -INFINITY ? -INFINITY : lg[k] - nm;
                }
                // O holds PV up to tile j-1: wait for it, scale this lane's
                // columns of this warpgroup's rows
                if (j >= 1) {
                    if (!mbar_wait_bounded(tile_free((j - 1) & 1), ((j - 1) >> 1) & 1, kSpin)) {
                        record_status(7u);
                        ok = false;
                        break;
                    }
                    tc::fence_after_sync();
#pragma unroll 1
                    for (int half = 0; half < 2; ++half) {     // the P' hi and lo products
                        uint32_t ov[8];
                        tc::tmem_ld8(t_lane + kTmemO + kCols * half + 8 * wg, ov);
                        tc::tmem_wait_ld();
#pragma unroll
                        for (int k = 0; k < 8; ++k)
                            ov[k] = __float_as_uint(__uint_as_float(ov[k]) * __uint_as_float(cs[k]));
                        tc::tmem_st8(t_lane + kTmemO + kCols * half + 8 * wg, ov);
                    }
                    tc::tmem_wait_st();
                }
            }
            // p, P' = p S_v ps as two fp16 terms, hi = fp16(P') into row c and
            // lo = fp16(P' - hi) into row kCols + c of the P'^T tile: one fp16
            // term rounds each weight by up to 2^-12 relative, which moves an
            // output made of a few comparable tokens with distant values by up
            // to about 1e-3; the pair carries about 22 significant bits
            const uint32_t pt = sbase + kOffBuf + b * kBufBytes + kPTile;
#pragma unroll
            for (int k = 0; k < 8; ++k) {
                const int c = 8 * wg + k;
                if (c < NQ) {
                    const float pv = tc::ex2(x[k]);
                    lp[k] += pv;
                    const float y = pv * sv;
                    const __half ph = __float2half_rn(y);
                    const __half pl = __float2half_rn(y - __half2float(ph));
                    sts16(pt + sw128(c, 2 * t, kPAtom), __half_as_ushort(ph));
                    sts16(pt + sw128(kCols + c, 2 * t, kPAtom), __half_as_ushort(pl));
                }
            }
            fence_proxy_async();            // P' is read by the tensor core
            tc::fence_before_sync();
            __syncwarp();
            if (lane == 0) mbar_arrive(p_full(b));
        }

        // ---- partials: thread = dimension t of O --------------------------
        // the last tile's ps: 2^11 / (15 ps) restores p S_v / 15 from the
        // (2n - 15) 2^-11 levels
        const float ps_end = n_tiles > 0
            ? reinterpret_cast<const float *>(smem + kOffTps)[2 * ((n_tiles - 1) & 1) + 1] : 0.f;
        const float ips15 = (ps_end > 0.f ? pow2_inv(ps_end) : 1.0f) * (2048.0f / 15.0f);
        uint32_t ov[8] = {0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u}, ovl[8] = {0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u};
        if (ok && n_tiles > 0) {
            if (mbar_wait_bounded(tile_free((n_tiles - 1) & 1), ((n_tiles - 1) >> 1) & 1, kSpin)) {
                tc::fence_after_sync();
                tc::tmem_ld8(t_lane + kTmemO + 8 * wg, ov);
                tc::tmem_ld8(t_lane + kTmemO + kCols + 8 * wg, ovl);
                tc::tmem_wait_ld();
            } else {
                record_status(7u);
            }
        }
        // l of each row: warp sums, then across the four lane quarters
#pragma unroll
        for (int k = 0; k < 8; ++k) {
            const float ls = warp_sum(lp[k]);
            if (lane == 0) xfin[2 * kCols * q4 + 8 * wg + k] = ls;
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(fin_bar);
        if (mbar_wait_bounded(fin_bar, 0, kSpin)) {
#pragma unroll
            for (int k = 0; k < 8; ++k) {
                const int c = 8 * wg + k;
                if (c < NQ) {
                    float L = 0.f;
#pragma unroll
                    for (int qq = 0; qq < 4; ++qq) L += xfin[2 * kCols * qq + c];
                    const int i = c / G, h = c - (c / G) * G;
                    const int64_t row =
                        (((int64_t)s * QL + i) * p.Hq + g * G + h) * p.n_splits + split;
                    // sum_t P'_t (2n - 15) = 2^11 (O''_hi + O''_lo)
                    if (in_extent(row, 1, p.part_rows)) {
                        p.part_o[row * kD + t] =
                            (__uint_as_float(ov[k]) + __uint_as_float(ovl[k])) * ips15;
                        if (t == 0) p.part_ml[row] = make_float2(m[k], L);
                    }
                }
            }
        } else {
            record_status(7u);
        }
    }

    // ---- teardown ------------------------------------------------------------
    tc::fence_before_sync();
    __syncthreads();
    if (warp == 1) {
        tc::fence_after_sync();
        tc::tmem_dealloc(tmem, kTmemCols);
    }
}

}  // namespace dmq
}  // namespace tbq4

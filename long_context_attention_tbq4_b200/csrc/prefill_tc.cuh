// prefill_tc.cuh -- chunked-prefill attention over TBQ4 caches on the
// 5th-generation tensor cores (tcgen05, accumulators in tensor memory).
//
// Where the chunk's queries meet the cache, QK^T and PV are dense
// contractions, so they run as 128x128x128 UMMA tiles; the raw TBQ4 blocks
// are dequantised inside the loop straight into bf16 operand tiles in shared
// memory (no dequantised copy of the cache in HBM: trefon.com, "Kontekst
// 262K na jednej RTX 4090", section "Od czego zaczalem").
//
// One CTA = one "M-pair" (two query heads h, h+1 of one KV group x 128 query
// positions) x one split of that pair's key range.  16 warps:
//   warp 0      producer: cp.async.bulk of raw K and V blocks (128 tokens,
//               8,448 bytes each) into a 2-stage raw ring
//   warp 1      tensor-memory allocation; lane 0 issues every tcgen05.mma
//   warps 4-7   dequantisation: raw nibbles -> bf16 operand tiles in a
//               3-slot ring of 32 KB (K tile: keys x dims, (2n-15) S_k *
//               scale * log2(e) / 15 rounded once, so S comes out of the
//               MMA in log2 units; V^T tile: dims x keys, (2n-15) S_v/15
//               rounded once; both K-major with the 128-byte swizzle)
//   warps 8-11  softmax of M-tile 0 (thread = query row = TMEM lane)
//   warps 12-15 softmax of M-tile 1
// Tensor memory (512 columns): M-tile a has S at [256a, 256a+128) (P, bf16,
// is written over its first 64 columns) and O at [256a+128, 256a+256).
// Per key tile j the MMA thread issues S_0, S_1 = Q K^T, then for each
// M-tile waits for its P and issues O += P V^T, followed at once by the
// next tile's S for that M-tile (so one M-tile's softmax overlaps the other
// M-tile's MMAs).  The row max is only moved (and O rescaled) when it grows
// by more than 8 in log2 units.
#pragma once
#include <type_traits>

#include "common.cuh"
#include "decode.cuh"
#include "tcgen05.cuh"

namespace tbq4 {
namespace pre {

constexpr int kThreads = 512;
constexpr int kTile = 128;                              // keys per tile, rows per M-tile
constexpr int kRawBytes = kTile * kBlockBytes;          // 8448
constexpr int kRawStages = 2;
constexpr int kRawStageBytes = 2 * kRawBytes + 16;      // K | V | pad
constexpr int kSlots = 3;
constexpr int kOpBytes = kTile * kD * 2;                // 32 KB bf16 operand tile
constexpr float kRescaleThreshold = 8.0f;               // log2 units
constexpr float kFastSumLimit = 256.0f;                 // 2^kRescaleThreshold
constexpr uint32_t kSpin = 1u << 22;
// The producer and the dequantisation warps run ahead of the tensor core;
// their waits sleep this long between polls, leaving issue slots to the
// softmax warps on the same schedulers.
constexpr uint32_t kLazyNs = 128;
// Registers per thread after the prologue, per warpgroup: producer/MMA,
// dequantisation, and each softmax warpgroup (which holds a full S row of 128
// floats).  Their sum x 128 threads must fit in what the CTA was launched
// with, 512 threads x the compiled count; the host refuses to launch if the
// compiled count is below kMinLaunchRegs.
constexpr uint32_t kRegsCtl = 64, kRegsDeq = 80, kRegsSoft = 184;
constexpr int kMinLaunchRegs = 128;
static_assert((kRegsCtl + kRegsDeq + 2 * kRegsSoft) * 128 <= kMinLaunchRegs * kThreads,
              "register split exceeds the launch budget");

// shared-memory layout (offsets from a 1024-aligned base)
constexpr int kOffQ = 0;                                        // 2 x 32 KB
constexpr int kOffSlot = kOffQ + 2 * kOpBytes;                  // 3 x 32 KB
constexpr int kOffRaw = kOffSlot + kSlots * kOpBytes;           // 2 x 16,912
constexpr int kOffBar = kOffRaw + kRawStages * kRawStageBytes;
constexpr int kNumBars = 2 * kRawStages + 2 * kSlots + 6;
constexpr int kOffTmemPtr = kOffBar + kNumBars * 8;
constexpr int kSmemBytes = kOffTmemPtr + 16 + 1024;              // + alignment slack

static_assert(kOffSlot % 1024 == 0 && kOffRaw % 16 == 0 && kRawStageBytes % 16 == 0, "align");
static_assert(kSmemBytes <= 232448, "shared memory budget");

constexpr uint32_t kIdesc = tc::idesc_bf16(128, 128);

// bf16x2 constants: {128 + n} from a nibble in mantissa bits 0-3, and {-136}: 128 + n - 136 = n - 8.
constexpr uint32_t kB2Magic128 = 0x43004300u;
constexpr uint32_t kB2Neg136 = 0xC308C308u;

__device__ __forceinline__ uint32_t bfma2(uint32_t x, uint32_t m, uint32_t a) {
    __nv_bfloat162 r = __hfma2(*reinterpret_cast<__nv_bfloat162 *>(&x),
                               *reinterpret_cast<__nv_bfloat162 *>(&m),
                               *reinterpret_cast<__nv_bfloat162 *>(&a));
    return *reinterpret_cast<uint32_t *>(&r);
}

__device__ __forceinline__ uint32_t badd2(uint32_t x, uint32_t a) {
    __nv_bfloat162 r = __hadd2(*reinterpret_cast<__nv_bfloat162 *>(&x),
                               *reinterpret_cast<__nv_bfloat162 *>(&a));
    return *reinterpret_cast<uint32_t *>(&r);
}

// A level times its token's factor s, in one rounding: with n - 8 exact,
// (n - 8) * 2 s + s = (2n - 15) s.  v holds nibbles in bits 0-3 and 16-19;
// s2 = {2 s_a, 2 s_b}, s1 = {s_a, s_b}.  V: s = S_v / 15; K: s = S_k *
// softmax_scale * log2(e) / 15.
__device__ __forceinline__ uint32_t v_scaled(uint32_t v, uint32_t s2, uint32_t s1) {
    return bfma2(badd2((v & 0x000F000Fu) | kB2Magic128, kB2Neg136), s2, s1);
}

__device__ __forceinline__ uint32_t lds32(uint32_t a) {
    uint32_t v;
    asm volatile("ld.shared.b32 %0, [%1];" : "=r"(v) : "r"(a));
    return v;
}
__device__ __forceinline__ uint16_t lds16(uint32_t a) {
    uint16_t v;
    asm volatile("ld.shared.u16 %0, [%1];" : "=h"(v) : "r"(a));
    return v;
}
__device__ __forceinline__ void sts32(uint32_t a, uint32_t v) {
    asm volatile("st.shared.b32 [%0], %1;" ::"r"(a), "r"(v) : "memory");
}
__device__ __forceinline__ void sts64(uint32_t a, uint32_t x, uint32_t y) {
    asm volatile("st.shared.v2.b32 [%0], {%1, %2};" ::"r"(a), "r"(x), "r"(y) : "memory");
}
__device__ __forceinline__ void sts128(uint32_t a, uint32_t x, uint32_t y, uint32_t z,
                                       uint32_t w) {
    asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(a), "r"(x), "r"(y), "r"(z),
                 "r"(w)
                 : "memory");
}

// Byte offset of element (row, k) in a 128-row K-major bf16 tile with the
// 128-byte swizzle: two 16 KB halves along K (k < 64, k >= 64), 8-row groups
// of 1024 bytes, 16-byte chunks XOR-ed with (row % 8).
__device__ __forceinline__ uint32_t sw128_off(int row, int k) {
    return (uint32_t)((k >> 6) * 16384 + (row >> 3) * 1024 + (row & 7) * 128 +
                      ((((k & 63) >> 3) ^ (row & 7)) << 4) + (k & 7) * 2);
}

// 32-bit word of nibble bytes at a 2-byte aligned shared address.
__device__ __forceinline__ uint32_t funnel_word(uint32_t addr) {
    const uint32_t base = addr & ~3u, sh = (addr & 3u) * 8u;
    return __funnelshift_r(lds32(base), lds32(base + 4), sh);
}

struct PrefillParams {
    const uint16_t *q;          // bf16 [n_new][Hq][128]
    const uint8_t *k;           // [Hkv][capacity][66]
    const uint8_t *v;
    int64_t head_stride;        // capacity * 66
    int n_new;
    int64_t n_cached;
    int Hq, Hkv, G;
    int pairs;                  // ceil(G / 2)
    int iblocks;                // ceil(n_new / 128)
    int n_splits;               // key splits per M-pair
    float scale_log2_15;        // softmax_scale * log2(e) / 15
    uint64_t sign_lo, sign_hi;
    float *part_o;              // [n_new][Hq][n_splits][128]
    float2 *part_ml;            // [n_new][Hq][n_splits]
    // extents, for the debug build's bounds checks: bytes of each cache,
    // entries of part_ml
    int64_t cache_bytes, part_rows;
};

__global__ void __launch_bounds__(kThreads, 1)
prefill_tc_kernel(const PrefillParams p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
    const uint32_t sbase = smem_u32(smem);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    // the dependent combine may be scheduled from now on (it waits for this grid)
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

    // ---- work unit ---------------------------------------------------------
    const int split = blockIdx.x;
    int mp = blockIdx.y;
    const int iblk = mp % p.iblocks;
    mp /= p.iblocks;
    const int pair = mp % p.pairs;
    const int g = mp / p.pairs;
    const int i0 = iblk * kTile;
    const int rows_valid = min(kTile, p.n_new - i0);
    const int64_t keys_total = p.n_cached + p.n_new;       // tokens in the cache
    const int64_t keys_pair = p.n_cached + i0 + rows_valid; // keys any row of the pair sees
    const int tiles_pair = (int)((keys_pair + kTile - 1) / kTile);
    const int tile_begin = (int)((int64_t)tiles_pair * split / p.n_splits);
    const int tile_end = (int)((int64_t)tiles_pair * (split + 1) / p.n_splits);
    const int n_tiles = tile_end - tile_begin;
    const bool valid1 = 2 * pair + 1 < p.G;

    // barriers
    const uint32_t bar0 = sbase + kOffBar;
    auto raw_full = [&](int s) { return bar0 + 8 * s; };
    auto raw_empty = [&](int s) { return bar0 + 8 * (kRawStages + s); };
    auto slot_full = [&](int s) { return bar0 + 8 * (2 * kRawStages + s); };
    auto slot_empty = [&](int s) { return bar0 + 8 * (2 * kRawStages + kSlots + s); };
    const uint32_t barx = bar0 + 8 * (2 * kRawStages + 2 * kSlots);
    auto s_full = [&](int a) { return barx + 8 * a; };
    auto p_full = [&](int a) { return barx + 8 * (2 + a); };
    auto o_done = [&](int a) { return barx + 8 * (4 + a); };
    uint32_t *tmem_ptr = reinterpret_cast<uint32_t *>(smem + kOffTmemPtr);

    if (threadIdx.x == 0) {
        for (int s = 0; s < kRawStages; ++s) { mbar_init(raw_full(s), 1); mbar_init(raw_empty(s), 4); }
        for (int s = 0; s < kSlots; ++s) { mbar_init(slot_full(s), 4); mbar_init(slot_empty(s), 1); }
        for (int a = 0; a < 2; ++a) {
            mbar_init(s_full(a), 1);
            mbar_init(p_full(a), 4);
            mbar_init(o_done(a), 1);
        }
        fence_barrier_init();
    }
    if (warp == 1) {
        tc::tmem_alloc(smem_u32(tmem_ptr), 512);
        tc::tmem_relinquish();
    }

    // ---- Q tiles: rotate each row, round to bf16, store swizzled -----------
    {
        const uint32_t sbits = lane_sign_bits(p.sign_lo, p.sign_hi, lane);
        for (int rr = warp; rr < 2 * kTile; rr += kThreads / 32) {
            const int a = rr >> 7, row = rr & (kTile - 1);
            const int h = 2 * pair + a, i = i0 + row;
            float v[4] = {0.f, 0.f, 0.f, 0.f};
            if (h < p.G && i < p.n_new) {
                const uint2 raw = *reinterpret_cast<const uint2 *>(
                    p.q + ((int64_t)i * p.Hq + g * p.G + h) * kD + 4 * lane);
                v[0] = __uint_as_float(raw.x << 16);
                v[1] = __uint_as_float(raw.x & 0xFFFF0000u);
                v[2] = __uint_as_float(raw.y << 16);
                v[3] = __uint_as_float(raw.y & 0xFFFF0000u);
                warp_rotate128(v, sbits, lane);
            }
            __nv_bfloat162 b01 = __floats2bfloat162_rn(v[0], v[1]);
            __nv_bfloat162 b23 = __floats2bfloat162_rn(v[2], v[3]);
            sts64(sbase + kOffQ + a * kOpBytes + sw128_off(row, 4 * lane),
                  *reinterpret_cast<uint32_t *>(&b01), *reinterpret_cast<uint32_t *>(&b23));
        }
    }
    fence_proxy_async();                // Q tiles are read by the tensor core
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tmem = *tmem_ptr;
    const int64_t head_off = (int64_t)g * p.head_stride;
    if (warp < 4) {
      tc::regs_dec<kRegsCtl>();
      if (warp == 0) {
        // ======================= producer ====================================
        if (lane == 0) {
            for (int j = 0; j < n_tiles; ++j) {
                const int st = j % kRawStages;
                if (j >= kRawStages &&
                    !mbar_wait_lazy(raw_empty(st), ((j / kRawStages) - 1) & 1, kSpin, kLazyNs)) {
                    record_status(7u);
                    break;
                }
                const int64_t t0 = (int64_t)(tile_begin + j) * kTile;
                const int64_t ntok = min((int64_t)kTile, keys_total - t0);
                const uint32_t bytes = (uint32_t)((ntok + 7) & ~7LL) * kBlockBytes;
                const uint32_t dst = sbase + kOffRaw + st * kRawStageBytes;
                fence_proxy_async();
                mbar_expect_tx(raw_full(st), 2 * bytes);
                int64_t off = head_off + t0 * kBlockBytes;
                if constexpr (kDebugBounds) off = checked_off(off, bytes, p.cache_bytes);
                bulk_g2s(dst, p.k + off, bytes, raw_full(st));
                bulk_g2s(dst + kRawBytes, p.v + off, bytes, raw_full(st));
            }
        }
      } else if (warp == 1) {
        // ======================= MMA issuer ==================================
        if (lane == 0 && n_tiles > 0) {
            bool ok = true;
            // polled with test_wait and a short sleep: a thread suspended in
            // try_wait resumed here about half a microsecond after its phase
            // completed
            auto wait = [&](uint32_t bar, uint32_t par) {
                bool got = false;
                for (uint32_t i = 0; ok && i < kSpin && !got; ++i) {
                    got = mbar_test(bar, par);
                    if (!got) __nanosleep(20);
                }
                if (ok && !got) { ok = false; record_status(7u); }
                return ok;
            };
            const uint32_t qa = sbase + kOffQ;
            auto issue_s = [&](int a, int j) {       // S_a = Q_a K_j^T
                const int u = 2 * j, slot = u % kSlots;
                const uint32_t kt = sbase + kOffSlot + slot * kOpBytes;
                const uint32_t qt = qa + a * kOpBytes;
                tc::fence_after_sync();
#pragma unroll
                for (int kk = 0; kk < 8; ++kk) {
                    const uint32_t off = (kk >> 2) * 16384 + (kk & 3) * 32;
                    tc::mma_ss(tmem + 256 * a, tc::desc_sw128(qt + off), tc::desc_sw128(kt + off),
                               kIdesc, kk > 0);
                }
                tc::mma_commit(s_full(a));
            };
            auto issue_pv = [&](int a, int j) {      // O_a += P_a V_j
                const int u = 2 * j + 1, slot = u % kSlots;
                const uint32_t vt = sbase + kOffSlot + slot * kOpBytes;
                tc::fence_after_sync();
#pragma unroll
                for (int kk = 0; kk < 8; ++kk) {
                    const uint32_t off = (kk >> 2) * 16384 + (kk & 3) * 32;
                    tc::mma_ts(tmem + 256 * a + 128, tmem + 256 * a + 8 * kk,
                               tc::desc_sw128(vt + off), kIdesc, (j > 0 || kk > 0) ? 1u : 0u);
                }
                tc::mma_commit(o_done(a));
            };
            if (wait(slot_full(0), 0)) {
                issue_s(0, 0);
                if (valid1) issue_s(1, 0);
                tc::mma_commit(slot_empty(0));
            }
            for (int j = 0; j < n_tiles && ok; ++j) {
                const int uv = 2 * j + 1;
                if (!wait(slot_full(uv % kSlots), (uv / kSlots) & 1)) break;
                for (int a = 0; a < 2 && ok; ++a) {
                    if (a == 1 && !valid1) continue;
                    if (!wait(p_full(a), j & 1)) break;
                    issue_pv(a, j);
                    if (a == (valid1 ? 1 : 0)) tc::mma_commit(slot_empty(uv % kSlots));
                    if (j + 1 < n_tiles) {
                        const int uk = 2 * (j + 1);
                        if (a == 0 && !wait(slot_full(uk % kSlots), (uk / kSlots) & 1)) break;
                        issue_s(a, j + 1);
                        if (a == (valid1 ? 1 : 0)) tc::mma_commit(slot_empty(uk % kSlots));
                    }
                }
            }
        }
      }
    } else if (warp < 8) {
        tc::regs_dec<kRegsDeq>();
        // ======================= dequantisation ==============================
        const int t = threadIdx.x - 128;              // 0..127
        for (int j = 0; j < n_tiles; ++j) {
            const int st = j % kRawStages;
            const uint32_t raw = sbase + kOffRaw + st * kRawStageBytes;
            const int64_t t0 = (int64_t)(tile_begin + j) * kTile;
            if (!mbar_wait_lazy_warp(raw_full(st), (j / kRawStages) & 1, kSpin, kLazyNs)) { record_status(7u); break; }
            // K tile: token t -> row t, dims contiguous, each level times the
            // token's factor S_k * scale * log2(e) / 15 rounded once (so S
            // leaves the MMA in log2 units); 0 past the cache end, where the
            // raw bytes are stale
            {
                const int u = 2 * j, slot = u % kSlots;
                if (u >= kSlots && !mbar_wait_lazy_warp(slot_empty(slot), ((u / kSlots) - 1) & 1, kSpin, kLazyNs)) {
                    record_status(7u);
                    break;
                }
                const uint32_t dst = sbase + kOffSlot + slot * kOpBytes;
                const uint32_t src = raw + t * kBlockBytes + 2;
                const float fk = t0 + t < keys_total
                    ? __half2float(__ushort_as_half(lds16(src - 2))) * p.scale_log2_15 : 0.f;
                const __nv_bfloat162 f1b = __floats2bfloat162_rn(fk, fk);
                const __nv_bfloat162 f2b = __hmul2(f1b, __floats2bfloat162_rn(2.f, 2.f));
                const uint32_t f1 = *reinterpret_cast<const uint32_t *>(&f1b);
                const uint32_t f2 = *reinterpret_cast<const uint32_t *>(&f2b);
#pragma unroll 4
                for (int w = 0; w < 16; ++w) {
                    const uint32_t x = funnel_word(src + 4 * w);
                    const uint32_t l0 = v_scaled(x, f2, f1);          // b0.lo, b2.lo
                    const uint32_t h0 = v_scaled(x >> 4, f2, f1);     // b0.hi, b2.hi
                    const uint32_t l1 = v_scaled(x >> 8, f2, f1);     // b1.lo, b3.lo
                    const uint32_t h1 = v_scaled(x >> 12, f2, f1);    // b1.hi, b3.hi
                    sts128(dst + sw128_off(t, 8 * w), __byte_perm(l0, h0, 0x5410),
                           __byte_perm(l1, h1, 0x5410), __byte_perm(l0, h0, 0x7632),
                           __byte_perm(l1, h1, 0x7632));
                }
                fence_proxy_async();
                __syncwarp();
                if (lane == 0) mbar_arrive(slot_full(slot));
            }
            // V^T tile: dim d -> row d, keys contiguous; thread = token pair
            // (2pp, 2pp+1) x dims [64 hf, 64 hf + 64)
            {
                const int u = 2 * j + 1, slot = u % kSlots;
                if (u >= kSlots && !mbar_wait_lazy_warp(slot_empty(slot), ((u / kSlots) - 1) & 1, kSpin, kLazyNs)) {
                    record_status(7u);
                    break;
                }
                const uint32_t dst = sbase + kOffSlot + slot * kOpBytes;
                const int pp = t & 63, hf = t >> 6;
                const int ta = 2 * pp;
                const uint32_t srca = raw + kRawBytes + ta * kBlockBytes + 2 + 32 * hf;
                const uint32_t srcb = srca + kBlockBytes;
                // S_v / 15 of the two tokens; 0 past the cache end, where the
                // raw bytes are stale (their P is 0, and 0 * level must not be NaN)
                const float sva = t0 + ta < keys_total
                    ? __half2float(__ushort_as_half(lds16(srca - 2 - 32 * hf))) * (1.0f / 15.0f) : 0.f;
                const float svb = t0 + ta + 1 < keys_total
                    ? __half2float(__ushort_as_half(lds16(srcb - 2 - 32 * hf))) * (1.0f / 15.0f) : 0.f;
                __nv_bfloat162 s1b = __floats2bfloat162_rn(sva, svb);
                __nv_bfloat162 s2b = __hmul2(s1b, __floats2bfloat162_rn(2.f, 2.f));
                const uint32_t s1 = *reinterpret_cast<uint32_t *>(&s1b);
                const uint32_t s2 = *reinterpret_cast<uint32_t *>(&s2b);
#pragma unroll 2
                for (int w = 0; w < 8; ++w) {
                    const uint32_t wa = funnel_word(srca + 4 * w), wb = funnel_word(srcb + 4 * w);
                    const int d0 = 64 * hf + 8 * w;
#pragma unroll
                    for (int half = 0; half < 2; ++half) {
                        const uint32_t X = __byte_perm(wa, wb, half ? 0x7632 : 0x5410);
                        const int d = d0 + 4 * half;
                        sts32(dst + sw128_off(d + 0, ta), v_scaled(X, s2, s1));
                        sts32(dst + sw128_off(d + 1, ta), v_scaled(X >> 4, s2, s1));
                        sts32(dst + sw128_off(d + 2, ta), v_scaled(X >> 8, s2, s1));
                        sts32(dst + sw128_off(d + 3, ta), v_scaled(X >> 12, s2, s1));
                    }
                }
                fence_proxy_async();
                __syncwarp();
                if (lane == 0) mbar_arrive(slot_full(slot));
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(raw_empty(st));
        }
    } else {
        tc::regs_inc<kRegsSoft>();
        // ======================= softmax =====================================
        const int a = (warp - 8) >> 2;
        const int row = 32 * (warp & 3) + lane;           // TMEM lane = query row
        const bool active = (a == 0 || valid1);
        const int i = min(i0 + row, p.n_new - 1);
        const int64_t lim = p.n_cached + i;               // last key this row sees
        const uint32_t t_s = tmem + ((uint32_t)(32 * (warp & 3)) << 16) + 256 * a;
        const uint32_t t_o = t_s + 128;
        float m = -INFINITY, l = 0.f;
        bool ok = true;
        for (int j = 0; j < n_tiles && active; ++j) {
            if (!mbar_wait_bounded(s_full(a), j & 1, kSpin)) {
                record_status(7u);
                ok = false;
                break;
            }
            tc::fence_after_sync();
            const int64_t kt = (int64_t)(tile_begin + j) * kTile;
            const bool diag = kt + kTile - 1 > p.n_cached + i0;
            // Causal mask only on tiles that reach past the block's first row:
            // column col is masked when kt + col > lim, i.e. col > rel.
            const int rel = diag ? (int)(lim - kt) : kTile;
            // The whole S row of this thread goes to registers with one wait.
            float sr_[kTile];
#pragma unroll
            for (int ch = 0; ch < 4; ++ch)
                tc::tmem_ld32(t_s + 32 * ch, *reinterpret_cast<float(*)[32]>(sr_ + 32 * ch));
            tc::tmem_wait_ld();
            // Fast path (every row of the warp has a finite running max): P =
            // exp2(S - m) with the stale m, kept if each row's sum of P over
            // the tile stays <= 2^8 (which bounds every P by 2^8).  P is packed
            // in registers and written over S only once it is kept, so S stays
            // in tensor memory for the slow path and the S registers die as P
            // is formed.
            bool done = false;
            if (!__any_sync(kFull, m == -INFINITY)) {
                const float2 negm = make_float2(-m, -m);
                float2 lf[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
                uint32_t pk[kTile / 2];
                // The causal mask only on the few tiles that reach the
                // diagonal: a separate loop, chosen once per tile, so the
                // others carry no per-element compare and select.
                auto fast_p = [&](auto masked) {
#pragma unroll
                    for (int e = 0; e < kTile; e += 2) {
                        float2 d = __fadd2_rn(make_float2(sr_[e], sr_[e + 1]), negm);
                        if constexpr (decltype(masked)::value) {
                            if (e > rel) d.x = -INFINITY;
                            if (e + 1 > rel) d.y = -INFINITY;
                        }
                        const float2 pr = make_float2(tc::ex2(d.x), tc::ex2(d.y));
                        lf[(e >> 1) & 1] = __fadd2_rn(lf[(e >> 1) & 1], pr);
                        __nv_bfloat162 bb = __floats2bfloat162_rn(pr.x, pr.y);
                        pk[e >> 1] = *reinterpret_cast<uint32_t *>(&bb);
                    }
                };
                if (diag) fast_p(std::true_type{});
                else fast_p(std::false_type{});
                const float lt = (lf[0].x + lf[0].y) + (lf[1].x + lf[1].y);
                if (!__any_sync(kFull, !(lt <= kFastSumLimit))) {
                    l += lt;
                    done = true;
#pragma unroll
                    for (int ch = 0; ch < 4; ++ch)
                        tc::tmem_st16(t_s + 16 * ch, *reinterpret_cast<uint32_t(*)[16]>(pk + 16 * ch));
                }
            }
            if (!done) {
                // exact row max from S reloaded 32 columns at a time, O rescale
                // when it grows past the threshold, then P (column block c of P
                // lands on S columns already read: P's 64 columns cover S
                // columns 0-63, read in the first two blocks)
                float mx4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll 1
                for (int ch = 0; ch < 4; ++ch) {
                    float sc[32];
                    tc::tmem_ld32(t_s + 32 * ch, sc);
                    tc::tmem_wait_ld();
#pragma unroll
                    for (int e = 0; e < 32; e += 2) {
                        const int col = 32 * ch + e;
                        float2 z = make_float2(sc[e], sc[e + 1]);
                        if (diag) {
                            if (col > rel) z.x = -INFINITY;
                            if (col + 1 > rel) z.y = -INFINITY;
                        }
                        mx4[(e >> 1) & 3] = fmaxf(mx4[(e >> 1) & 3], fmaxf(z.x, z.y));
                    }
                }
                const float mx = fmaxf(fmaxf(mx4[0], mx4[1]), fmaxf(mx4[2], mx4[3]));
                const float m_new = fmaxf(m, mx);
                const bool need =
                    (m == -INFINITY && m_new != -INFINITY) || m_new > m + kRescaleThreshold;
                if (__any_sync(kFull, need)) {
                    const float corr = (m == -INFINITY) ? 0.f : tc::ex2(m - m_new);
                    if (j > 0) {
                        if (!mbar_wait_bounded(o_done(a), (j - 1) & 1, kSpin)) {
                            record_status(7u);
                            ok = false;
                            break;
                        }
                        tc::fence_after_sync();
#pragma unroll 1
                        for (int ch = 0; ch < 4; ++ch) {
                            float o[32];
                            tc::tmem_ld32(t_o + 32 * ch, o);
                            tc::tmem_wait_ld();
#pragma unroll
                            for (int e = 0; e < 32; ++e) o[e] *= corr;
                            tc::tmem_st32(t_o + 32 * ch, o);
                        }
                    }
                    l *= corr;
                    m = m_new;
                }
                const float m_use = (m == -INFINITY) ? 0.f : m;
                const float2 negm = make_float2(-m_use, -m_use);
                float2 lacc[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
#pragma unroll 1
                for (int ch = 0; ch < 4; ++ch) {
                    float sc[32];
                    tc::tmem_ld32(t_s + 32 * ch, sc);
                    tc::tmem_wait_ld();
                    uint32_t pk[16];
#pragma unroll
                    for (int e = 0; e < 32; e += 2) {
                        const int col = 32 * ch + e;
                        float2 z = __fadd2_rn(make_float2(sc[e], sc[e + 1]), negm);
                        if (diag) {
                            if (col > rel) z.x = -INFINITY;
                            if (col + 1 > rel) z.y = -INFINITY;
                        }
                        const float2 pr = make_float2(tc::ex2(z.x), tc::ex2(z.y));
                        lacc[(e >> 1) & 1] = __fadd2_rn(lacc[(e >> 1) & 1], pr);
                        __nv_bfloat162 bb = __floats2bfloat162_rn(pr.x, pr.y);
                        pk[e >> 1] = *reinterpret_cast<uint32_t *>(&bb);
                    }
                    tc::tmem_st16(t_s + 16 * ch, pk);
                }
                l += (lacc[0].x + lacc[0].y) + (lacc[1].x + lacc[1].y);
            }
            tc::tmem_wait_st();
            tc::fence_before_sync();
            __syncwarp();
            if (lane == 0) mbar_arrive(p_full(a));
        }
        // ---- partial (O unnormalised, m, l) for this split -----------------
        const int h = 2 * pair + a;
        const int64_t prow =
            (((int64_t)(i0 + row) * p.Hq + g * p.G + h) * p.n_splits + split);
        const bool write = active && (i0 + row) < p.n_new && in_extent(prow, 1, p.part_rows);
        if (active && n_tiles > 0 && ok &&
            mbar_wait_bounded(o_done(a), (n_tiles - 1) & 1, kSpin)) {
            tc::fence_after_sync();
#pragma unroll 1
            for (int ch = 0; ch < 4; ++ch) {
                float o[32];
                tc::tmem_ld32(t_o + 32 * ch, o);
                tc::tmem_wait_ld();
                if (write) {
                    float4 *dst = reinterpret_cast<float4 *>(p.part_o + prow * kD + 32 * ch);
#pragma unroll
                    for (int e = 0; e < 8; ++e)
                        dst[e] = make_float4(o[4 * e], o[4 * e + 1], o[4 * e + 2], o[4 * e + 3]);
                }
            }
            if (write) p.part_ml[prow] = make_float2(m, l);
        } else if (write) {
            float4 *dst = reinterpret_cast<float4 *>(p.part_o + prow * kD);
            for (int e = 0; e < 32; ++e) dst[e] = make_float4(0.f, 0.f, 0.f, 0.f);
            p.part_ml[prow] = make_float2(-INFINITY, 0.f);
        }
    }

    tc::fence_before_sync();
    __syncthreads();
    if (warp == 1) {
        tc::fence_after_sync();
        tc::tmem_dealloc(tmem, 512);
    }
}

}  // namespace pre
}  // namespace tbq4

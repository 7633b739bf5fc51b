// common.cuh -- shared device helpers of libtbq4 (sm_100a).
//
// TBQ4 block: 128 values in 66 bytes, [fp16 scale][64 bytes of 4-bit
// indices], values in the Hadamard-rotated domain (trefon.com, "Kontekst
// 262K na jednej RTX 4090", section "Od czego zaczalem").  The codebook
// and rotation are this library's: see include/tbq4.h.
#pragma once

#include <cuda_fp16.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace tbq4 {

constexpr int kD = 128;               // values per block (head_dim)
constexpr int kBlockBytes = 66;       // bytes per block
constexpr int kMaxGroup = 8;          // query heads per KV head, at most
constexpr unsigned kFull = 0xffffffffu;

// fl32(1/sqrt(128)), the normalisation of the rotation.
__device__ __forceinline__ float rot_c() { return __uint_as_float(0x3DB504F3u); }

// First error recorded by any kernel of the library on this device.
__device__ unsigned int g_status;

__device__ __forceinline__ void record_status(unsigned code) {
    atomicCAS(&g_status, 0u, code);
}

// Debug build (compiled with -DTBQ4_DEBUG into libtbq4_debug.so): every
// global access whose address a kernel derives from lengths, positions, page
// ids or the split plan is checked against the extent of its buffer.  A
// failed check records status 8 (TBQ4_ERR_BOUNDS) and the access is skipped,
// or, for a copy tracked by an mbarrier, redirected to offset 0 so that the
// barrier still completes.  In the release build the checks are constant true.
#ifdef TBQ4_DEBUG
constexpr bool kDebugBounds = true;
#else
constexpr bool kDebugBounds = false;
#endif

// [off, off + len) inside [0, extent)?  Always true in the release build.
__device__ __forceinline__ bool in_extent(int64_t off, int64_t len, int64_t extent) {
    if constexpr (kDebugBounds) {
        if (off < 0 || len < 0 || off > extent - len) {
            record_status(8u /* TBQ4_ERR_BOUNDS */);
            return false;
        }
    }
    return true;
}

// off if [off, off + len) is inside [0, extent), else 0 (debug build only).
__device__ __forceinline__ int64_t checked_off(int64_t off, int64_t len, int64_t extent) {
    return in_extent(off, len, extent) ? off : 0;
}

// Four sign bits of the +-1 diagonal for elements 4*lane .. 4*lane+3:
// s_i = -1 where bit (i % 64) of word i / 64 is set.
__device__ __forceinline__ uint32_t lane_sign_bits(uint64_t lo, uint64_t hi, int lane) {
    const uint64_t w = lane < 16 ? lo : hi;
    return (uint32_t)(w >> ((4 * lane) & 63)) & 0xFu;
}

// Unnormalised 128-point Walsh-Hadamard transform of a vector held four
// elements per lane (lane l holds elements 4l .. 4l+3), natural (Sylvester)
// order.  Stages run in ascending stride 1, 2, ..., 64; in each butterfly
// the lower-index element becomes a+b and the upper a-b, every operation
// rounded to binary32 on its own (no contraction), so the result is
// bit-reproducible.
__device__ __forceinline__ void warp_fwht128(float v[4], int lane) {
    float a, b;
    a = v[0]; b = v[1]; v[0] = __fadd_rn(a, b); v[1] = __fsub_rn(a, b);
    a = v[2]; b = v[3]; v[2] = __fadd_rn(a, b); v[3] = __fsub_rn(a, b);
    a = v[0]; b = v[2]; v[0] = __fadd_rn(a, b); v[2] = __fsub_rn(a, b);
    a = v[1]; b = v[3]; v[1] = __fadd_rn(a, b); v[3] = __fsub_rn(a, b);
#pragma unroll
    for (int m = 1; m < 32; m <<= 1) {
        const bool upper = (lane & m) != 0;
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            const float o = __shfl_xor_sync(kFull, v[k], m);
            v[k] = upper ? __fsub_rn(o, v[k]) : __fadd_rn(v[k], o);
        }
    }
}

// R x for one 128-vector held four per lane: sign flip, transform, scale.
__device__ __forceinline__ void warp_rotate128(float v[4], uint32_t sbits, int lane) {
#pragma unroll
    for (int k = 0; k < 4; ++k)
        if ((sbits >> k) & 1u) v[k] = -v[k];
    warp_fwht128(v, lane);
    const float c = rot_c();
#pragma unroll
    for (int k = 0; k < 4; ++k) v[k] = __fmul_rn(v[k], c);
}

__device__ __forceinline__ float warp_max(float x) {
#pragma unroll
    for (int m = 16; m > 0; m >>= 1) x = fmaxf(x, __shfl_xor_sync(kFull, x, m));
    return x;
}

__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
    for (int m = 16; m > 0; m >>= 1) x += __shfl_xor_sync(kFull, x, m);
    return x;
}

// Exact arithmetic on powers of two x = 2^e (normal binary32, e in
// [-126, 127]) through the exponent field: 1/x, a/b, and the largest power
// of two <= y (y > 0 normal).
__device__ __forceinline__ float pow2_inv(float x) {
    return __uint_as_float(0x7F000000u - __float_as_uint(x));
}
__device__ __forceinline__ float pow2_ratio(float a, float b) {
    return __uint_as_float(__float_as_uint(a) - __float_as_uint(b) + 0x3F800000u);
}
__device__ __forceinline__ float pow2_floor(float y) {
    return __uint_as_float(__float_as_uint(y) & 0xFF800000u);
}

__device__ __forceinline__ float half_bits_to_float(uint16_t h) {
    return __half2float(__ushort_as_half(h));
}

}  // namespace tbq4

// quantize.cuh -- TBQ4 quantise-append kernel.
//
// One warp encodes one 128-value row into one 66-byte block: 512 bytes are
// read with one 16-byte load per lane, the rotation runs in registers and
// warp shuffles, the scale is a warp max, and each lane packs its four
// indices into two bytes.  The op order is fixed (see warp_fwht128 and the
// index formula below) so the bytes are identical to the codebook's
// definition.  The kernel is HBM-bound: 512 bytes in, 66 bytes out per row.
#pragma once
#include "common.cuh"

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

__global__ void __launch_bounds__(256)
quantize_append_kernel(const float *__restrict__ src, int B, int n_new, int Hkv,
                       const int32_t *__restrict__ start_pos, int64_t capacity,
                       uint64_t sign_lo, uint64_t sign_hi, uint8_t *__restrict__ cache) {
    const int lane = threadIdx.x & 31;
    const int64_t rows = (int64_t)B * n_new * Hkv;
    const int64_t nwarps = ((int64_t)gridDim.x * blockDim.x) >> 5;
    const uint32_t sbits = lane_sign_bits(sign_lo, sign_hi, lane);
    for (int64_t r = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5; r < rows;
         r += nwarps) {
        const int h = (int)(r % Hkv);
        const int64_t t = (r / Hkv) % n_new;
        const int b = (int)(r / ((int64_t)Hkv * n_new));
        const float4 x4 = __ldcs(reinterpret_cast<const float4 *>(src + r * kD) + lane);
        float v[4] = {x4.x, x4.y, x4.z, x4.w};
        uint16_t sb;
        const uint32_t packed = encode_row(v, sbits, lane, &sb);
        const int64_t pos = (int64_t)__ldg(start_pos + b) + t;
        if (pos < 0 || pos >= capacity) {
            if (lane == 0) record_status(4u /* TBQ4_ERR_CAPACITY */);
            continue;
        }
        uint8_t *dst = cache + (((int64_t)b * Hkv + h) * capacity + pos) * kBlockBytes;
        reinterpret_cast<uint16_t *>(dst + 2)[lane] = (uint16_t)packed;
        if (lane == 0) *reinterpret_cast<uint16_t *>(dst) = sb;
    }
}

}  // namespace tbq4

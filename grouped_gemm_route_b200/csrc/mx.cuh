// MXFP8 operand encoding shared by the quantiser kernels and the GEMM epilogues.
//
// An MXFP8 GEMM operand holds E4M3 codes with one UE8M0 (power-of-two) scale
// per 32 consecutive elements along the GEMM's K ("Prime Intellect's Prime Mega
// MoE Trains Giant AI Models 55% Faster", section "Precision and hardware
// support": MXFP8 on Blackwell, small microscaling groups).  Scale exponent s
// is the smallest integer with amax <= 448 * 2^s (0 for an all-zero block),
// clamped to [-127, 127] and stored as the byte s + 127; codes are
// v * 2^-s rounded to nearest E4M3 (ties to even), saturating at 448.
//
// Scale "atoms" are the shared-memory image the tensor cores read through
// tcgen05.cp (32x128b, replicated to the four lane quadrants): one 512-byte atom
// per 128 M/N rows x 128 K elements, row m = m0 + 32 m1 and K block j (of 32)
// at byte m0 * 16 + m1 * 4 + j.
#pragma once

#include <cuda_fp8.h>
#include <stdint.h>

namespace moe {

constexpr int kMxBlock = 32;     // elements per scale
constexpr int kMxAtomBytes = 512;

__device__ __forceinline__ int mx_scale_exp(float amax) {
    const uint32_t bits = __float_as_uint(amax);
    const int e = static_cast<int>((bits >> 23) & 0xFFu);
    if (!(amax > 0.f)) return 0;
    if (e == 0) return -127;  // amax below 2^-126: the smallest scale
    if (e == 255) return 127;
    // amax = (1 + m / 2^23) * 2^(e - 127) and 448 = 1.75 * 2^8
    int s = (e - 127) - 8 + ((bits & 0x7FFFFFu) > 0x600000u ? 1 : 0);
    return s < -127 ? -127 : (s > 127 ? 127 : s);
}

// Byte offset of scale (row m, K block j) inside its 512-byte atom.
__device__ __forceinline__ int mx_atom_byte(int m, int j) { return (m & 31) * 16 + ((m >> 5) & 3) * 4 + (j & 3); }

// 2^-s as a float multiplier pair (f1 * f2), exact for every s in [-127, 127]:
// 2^-127 is below the normal range, so it is applied as 2^-64 * 2^-63.  A
// multiplication by an exact power of two is exact unless the product leaves
// the normal range, where the E4M3 rounding is 0 or saturation either way.
__device__ __forceinline__ float mx_pow2_neg(int s) { return __uint_as_float(static_cast<uint32_t>(127 - s) << 23); }

// E4M3 code pair (lo = a, hi = b) of a * 2^-s and b * 2^-s (round to nearest
// even, saturating at 448).
__device__ __forceinline__ uint32_t mx_code2(float a, float b, float f1, float f2) {
    return static_cast<uint32_t>(__nv_cvt_float2_to_fp8x2(make_float2(a * f1 * f2, b * f1 * f2), __NV_SATFINITE,
                                                          __NV_E4M3));
}

// E4M3 codes of 32 values scaled by 2^-s, packed little-endian into 8 words.
__device__ __forceinline__ void mx_encode32(const float (&v)[32], int s, uint32_t (&codes)[8]) {
    const float f1 = mx_pow2_neg(s < 127 ? s : 64), f2 = s < 127 ? 1.f : mx_pow2_neg(63);
#pragma unroll
    for (int w = 0; w < 8; ++w)
        codes[w] = mx_code2(v[4 * w], v[4 * w + 1], f1, f2) | (mx_code2(v[4 * w + 2], v[4 * w + 3], f1, f2) << 16);
}

__device__ __forceinline__ float amax32(const float (&v)[32]) {
    float m = 0.f;
#pragma unroll
    for (int i = 0; i < 32; ++i) m = fmaxf(m, fabsf(v[i]));
    return m;
}

}  // namespace moe

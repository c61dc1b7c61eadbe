// MXFP8 quantiser kernels: E4M3 codes plus UE8M0 block scales for the
// operands of the MXFP8 expert GEMMs (encoding in mx.cuh).  All are HBM-bound
// streaming kernels, grid-stride over their work items.
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "moe_internal.h"
#include "mx.cuh"

namespace moe {

namespace {

__device__ __forceinline__ void load32(const __nv_bfloat16 *src, float (&v)[32]) {
    const uint4 *s4 = reinterpret_cast<const uint4 *>(src);
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        const uint4 u = __ldg(s4 + q);
        const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            v[8 * q + 2 * i] = __uint_as_float(w[i] << 16);
            v[8 * q + 2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
        }
    }
}

// Rows of src [R, K] quantised along K (the contiguous dimension), one thread
// per (row, 32-element block).  Scale placement:
//   kMxSfAtoms     atom (r / 128, k / 128) of a [R/128][K/128] atom array
//   kMxSfRowBytes  byte r * (K/32) + k/32 (rows that are later gathered)
//   kMxSfGateUp    W_gate_up [E*2I, K]: atom rows follow the GEMM tile, 64 gate
//                  rows then 64 up rows of column tile nt (tile row e*(I/64)+nt)
__global__ void mx_quant_rows_kernel(const __nv_bfloat16 *__restrict__ src, int64_t R, int K,
                                     uint8_t *__restrict__ dst, uint8_t *__restrict__ sf, int sf_mode, int I,
                                     const int32_t *__restrict__ rows_used) {
    const int nblk = K / kMxBlock;
    int64_t limit = R;
    if (rows_used != nullptr) limit = min(limit, static_cast<int64_t>(*rows_used));
    const int64_t total = limit * nblk;
    for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < total;
         i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        const int64_t r = i / nblk;
        const int j = static_cast<int>(i - r * nblk);
        float v[32];
        load32(src + r * K + j * kMxBlock, v);
        const int s = mx_scale_exp(amax32(v));
        uint32_t codes[8];
        mx_encode32(v, s, codes);
        uint4 *d4 = reinterpret_cast<uint4 *>(dst + r * K + j * kMxBlock);
        d4[0] = make_uint4(codes[0], codes[1], codes[2], codes[3]);
        d4[1] = make_uint4(codes[4], codes[5], codes[6], codes[7]);
        const uint8_t sb = static_cast<uint8_t>(s + 127);
        if (sf_mode == kMxSfRowBytes) {
            sf[r * nblk + j] = sb;
        } else {
            int64_t trow = r;  // row index in the tile order of the atoms
            if (sf_mode == kMxSfGateUp) {
                const int64_t e = r / (2 * I);
                const int rr = static_cast<int>(r - e * 2 * I);
                const bool up = rr >= I;
                const int q = up ? rr - I : rr;
                trow = (e * (I / 64) + q / 64) * 128 + (up ? 64 : 0) + q % 64;
            }
            const int64_t atom = (trow / 128) * (K / 128) + j / 4;
            sf[atom * kMxAtomBytes + mx_atom_byte(static_cast<int>(trow & 127), j)] = sb;
        }
    }
}

// src [Kr, N] quantised along its rows (K = rows) per column, blocks of 32
// rows; one thread per (32-row block, 4 adjacent columns): 8-byte loads and
// 4-byte code stores, so a warp moves 256 contiguous bytes of a row.  Codes
// keep the [Kr, N] layout (an MN-major GEMM operand); atoms are indexed
// (k / 128, n / 128) of a [Kr/128][N/128] atom array.  Only the first
// rows_used rows when given.
__global__ void __launch_bounds__(128) mx_quant_cols_kernel(const __nv_bfloat16 *__restrict__ src, int64_t Kr, int N,
                                     uint8_t *__restrict__ dst, uint8_t *__restrict__ sf,
                                     const int32_t *__restrict__ rows_used) {
    int64_t rows = Kr;
    if (rows_used != nullptr) rows = min(rows, static_cast<int64_t>(*rows_used));
    const int nquads = N / 4;
    const int64_t total = (rows / kMxBlock) * nquads;
    for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < total;
         i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        const int64_t kb = i / nquads;
        const int n = static_cast<int>(i - kb * nquads) * 4;
        const uint2 *s4 = reinterpret_cast<const uint2 *>(src + kb * kMxBlock * N + n);
        uint2 raw[32];
#pragma unroll
        for (int rr = 0; rr < 32; ++rr) raw[rr] = __ldg(s4 + static_cast<int64_t>(rr) * (N / 4));
        float m[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int rr = 0; rr < 32; ++rr) {
            m[0] = fmaxf(m[0], fabsf(__uint_as_float(raw[rr].x << 16)));
            m[1] = fmaxf(m[1], fabsf(__uint_as_float(raw[rr].x & 0xFFFF0000u)));
            m[2] = fmaxf(m[2], fabsf(__uint_as_float(raw[rr].y << 16)));
            m[3] = fmaxf(m[3], fabsf(__uint_as_float(raw[rr].y & 0xFFFF0000u)));
        }
        int sc[4];
        float f1[4], f2[4];
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            sc[c] = mx_scale_exp(m[c]);
            f1[c] = mx_pow2_neg(sc[c] < 127 ? sc[c] : 64);
            f2[c] = sc[c] < 127 ? 1.f : mx_pow2_neg(63);
        }
        uint32_t *d32 = reinterpret_cast<uint32_t *>(dst + kb * kMxBlock * N + n);
#pragma unroll
        for (int rr = 0; rr < 32; ++rr) {
            const float v0 = __uint_as_float(raw[rr].x << 16), v1 = __uint_as_float(raw[rr].x & 0xFFFF0000u);
            const float v2 = __uint_as_float(raw[rr].y << 16), v3 = __uint_as_float(raw[rr].y & 0xFFFF0000u);
            const uint32_t lo = static_cast<uint32_t>(__nv_cvt_float2_to_fp8x2(
                make_float2(v0 * f1[0] * f2[0], v1 * f1[1] * f2[1]), __NV_SATFINITE, __NV_E4M3));
            const uint32_t hi = static_cast<uint32_t>(__nv_cvt_float2_to_fp8x2(
                make_float2(v2 * f1[2] * f2[2], v3 * f1[3] * f2[3]), __NV_SATFINITE, __NV_E4M3));
            d32[static_cast<int64_t>(rr) * (N / 4)] = lo | (hi << 16);
        }
        const int64_t atom = (kb * kMxBlock / 128) * (N / 128) + n / 128;
        const int j = static_cast<int>(kb & 3);
#pragma unroll
        for (int c = 0; c < 4; ++c)
            sf[atom * kMxAtomBytes + mx_atom_byte((n + c) & 127, j)] = static_cast<uint8_t>(sc[c] + 127);
    }
}

}  // namespace

cudaError_t launch_mx_quant_rows(const __nv_bfloat16 *src, int64_t R, int K, uint8_t *dst, uint8_t *sf, int sf_mode,
                                 int I, const int32_t *rows_used, int sms, cudaStream_t s) {
    mx_quant_rows_kernel<<<sms * 8, 256, 0, s>>>(src, R, K, dst, sf, sf_mode, I, rows_used);
    return cudaGetLastError();
}

cudaError_t launch_mx_quant_cols(const __nv_bfloat16 *src, int64_t Kr, int N, uint8_t *dst, uint8_t *sf,
                                 const int32_t *rows_used, int sms, cudaStream_t s) {
    mx_quant_cols_kernel<<<sms * 24, 128, 0, s>>>(src, Kr, N, dst, sf, rows_used);
    return cudaGetLastError();
}

}  // namespace moe

// Routing and dispatch kernels of the fused MoE layer, and the routing-score
// backward.
//
// Routing rule (the layer's router, see include/moe.h): softmax over the E
// router logits, keep the k largest, renormalise over the kept k.  The k
// largest are selected on the fp32 logits (same set as on the softmax, since
// softmax is strictly increasing), value descending, ties to the lower expert
// index.  Dispatch ("token sorting" in "Prime Intellect's Prime Mega MoE Trains
// Giant AI Models 55% Faster", section "Where MoE training loses time") is a
// stable counting sort of the T*k choices by expert into a sorted layout whose
// expert groups are padded to multiples of 128 rows (the GEMM tile height).
//
// Three launches: (1) per token top-k + weights + a per-block expert histogram,
// (2) one block: totals, exclusive scans, per-block bases, tile table, padding,
// (3) per block: each thread owns one expert and walks the block's tokens in
// order, so positions inside an expert follow token order exactly.
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>

#include "moe_internal.h"
#include "ptx.cuh"

namespace moe {

namespace {

constexpr int kTopkThreads = 256;
constexpr int kTopkWarps = kTopkThreads / 32;

template <int NV>
__global__ void __launch_bounds__(kTopkThreads) route_topk_kernel(const float *__restrict__ logits, int T, int E,
                                                                  int k, int32_t *__restrict__ idx,
                                                                  float *__restrict__ w,
                                                                  int32_t *__restrict__ chunk_counts,
                                                                  int32_t *__restrict__ cnt, int cnt_per_token) {
    __shared__ int hist[kMaxExperts];
    __shared__ float sel_v[kTopkWarps][kMaxTopK];
    __shared__ int sel_e[kTopkWarps][kMaxTopK];
    for (int e = threadIdx.x; e < E; e += blockDim.x) hist[e] = 0;
    __syncthreads();

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int t_begin = blockIdx.x * kRouteChunk;
    for (int tt = warp; tt < kRouteChunk; tt += kTopkWarps) {
        const int t = t_begin + tt;
        if (t >= T) break;
        float v[NV];
        uint32_t taken = 0;
#pragma unroll
        for (int i = 0; i < NV; ++i) {
            const int e = lane + 32 * i;
            if (e < E) {
                v[i] = __ldg(logits + static_cast<size_t>(t) * E + e);
            } else {
                v[i] = -INFINITY;
                taken |= 1u << i;
            }
        }
        for (int j = 0; j < k; ++j) {
            float bv = -INFINITY;
            int be = 0x7fffffff;
#pragma unroll
            for (int i = 0; i < NV; ++i) {
                const int e = lane + 32 * i;
                const bool avail = !((taken >> i) & 1u);
                if (avail && (v[i] > bv || (v[i] == bv && e < be))) {
                    bv = v[i];
                    be = e;
                }
            }
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) {
                const float ov = __shfl_xor_sync(0xffffffffu, bv, off);
                const int oe = __shfl_xor_sync(0xffffffffu, be, off);
                if (ov > bv || (ov == bv && oe < be)) {
                    bv = ov;
                    be = oe;
                }
            }
            if (be >= E) be = 0;  // only reachable with NaN logits, which are unsupported
            if ((be & 31) == lane) taken |= 1u << (be >> 5);
            if (lane == 0) {
                sel_v[warp][j] = bv;
                sel_e[warp][j] = be;
            }
        }
        __syncwarp();
        // weights: exp(l_j - l_max) / sum over the chosen k, summed in slot order
        const float m = sel_v[warp][0];
        float s = 0.f;
        if (lane == 0) {
            for (int j = 0; j < k; ++j) s += expf(sel_v[warp][j] - m);
        }
        s = __shfl_sync(0xffffffffu, s, 0);
        for (int j = lane; j < k; j += 32) {
            const int e = sel_e[warp][j];
            idx[static_cast<size_t>(t) * k + j] = e;
            w[static_cast<size_t>(t) * k + j] = expf(sel_v[warp][j] - m) / s;
            atomicAdd(&hist[e], 1);
        }
        for (int c = lane; c < cnt_per_token; c += 32) cnt[static_cast<size_t>(t) * cnt_per_token + c] = 0;
        __syncwarp();
    }
    __syncthreads();
    for (int e = threadIdx.x; e < E; e += blockDim.x)
        chunk_counts[static_cast<size_t>(blockIdx.x) * E + e] = hist[e];
}

constexpr int kScanThreads = 1024;

__global__ void __launch_bounds__(kScanThreads) route_scan_kernel(int E, int n_chunks,
                                                                  const int32_t *__restrict__ chunk_counts,
                                                                  int32_t *__restrict__ chunk_base,
                                                                  int32_t *__restrict__ counts,
                                                                  int32_t *__restrict__ offsets,
                                                                  int32_t *__restrict__ group_start,
                                                                  int32_t *__restrict__ tile_expert,
                                                                  int32_t *__restrict__ perm, int64_t p_cap,
                                                                  int *status) {
    __shared__ int partial[kScanThreads];
    __shared__ int s_count[kMaxExperts];
    __shared__ int s_gstart[kMaxExperts + 1];
    const int L = kScanThreads / E;  // threads per expert (E <= 512 -> L >= 2)
    const int e = threadIdx.x / L, l = threadIdx.x % L;
    const bool active = e < E;
    int b0 = 0, b1 = 0;
    if (active) {
        b0 = static_cast<int>((static_cast<int64_t>(n_chunks) * l) / L);
        b1 = static_cast<int>((static_cast<int64_t>(n_chunks) * (l + 1)) / L);
        int sum = 0;
#pragma unroll 8
        for (int b = b0; b < b1; ++b) sum += chunk_counts[static_cast<size_t>(b) * E + e];
        partial[threadIdx.x] = sum;
    }
    __syncthreads();
    if (active && l == 0) {
        int c = 0;
        for (int i = 0; i < L; ++i) c += partial[e * L + i];
        s_count[e] = c;
        counts[e] = c;
    }
    __syncthreads();
    // exclusive scans of the counts and of the 128-padded counts (warp 0)
    if (threadIdx.x < 32) {
        const int lane = threadIdx.x;
        const int per = (E + 31) / 32;
        const int e0 = min(E, lane * per), e1 = min(E, e0 + per);
        int c_sum = 0, p_sum = 0;
        for (int i = e0; i < e1; ++i) {
            c_sum += s_count[i];
            p_sum += (s_count[i] + kTileM - 1) / kTileM * kTileM;
        }
        int c_pre = c_sum, p_pre = p_sum;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const int c_o = __shfl_up_sync(0xffffffffu, c_pre, off);
            const int p_o = __shfl_up_sync(0xffffffffu, p_pre, off);
            if (lane >= off) {
                c_pre += c_o;
                p_pre += p_o;
            }
        }
        int c_run = c_pre - c_sum, p_run = p_pre - p_sum;  // exclusive
        for (int i = e0; i < e1; ++i) {
            offsets[i] = c_run;
            group_start[i] = p_run;
            s_gstart[i] = p_run;
            c_run += s_count[i];
            p_run += (s_count[i] + kTileM - 1) / kTileM * kTileM;
        }
        if (lane == 31) {
            offsets[E] = c_pre;
            group_start[E] = p_pre;
            s_gstart[E] = p_pre;
            if (p_pre > p_cap) report_status(status, kStatusBadIndex);
        }
    }
    __syncthreads();
    if (!active) return;
    // per-block base of this expert = group start + pairs of this expert in earlier blocks
    int run = s_gstart[e];
    for (int i = 0; i < l; ++i) run += partial[e * L + i];
#pragma unroll 8
    for (int b = b0; b < b1; ++b) {
        chunk_base[static_cast<size_t>(b) * E + e] = run;
        run += chunk_counts[static_cast<size_t>(b) * E + e];
    }
    // tile table and padding rows of this expert's group
    const int gs = s_gstart[e], ge = s_gstart[e + 1], c = s_count[e];
    if (ge > p_cap) return;
    for (int mt = gs / kTileM + l; mt < ge / kTileM; mt += L) tile_expert[mt] = e;
    for (int q = gs + c + l; q < ge; q += L) perm[q] = -1;
}

__global__ void route_perm_kernel(int T, int E, int k, const int32_t *__restrict__ idx,
                                  const int32_t *__restrict__ chunk_base, int32_t *__restrict__ perm,
                                  int32_t *__restrict__ inv, int64_t p_cap, int *status) {
    __shared__ int sidx[kRouteChunk * kMaxTopK];
    const int t0 = blockIdx.x * kRouteChunk;
    const int nt = min(kRouteChunk, T - t0);
    for (int q = threadIdx.x; q < nt * k; q += blockDim.x) sidx[q] = idx[static_cast<size_t>(t0) * k + q];
    __syncthreads();
    const int e = threadIdx.x;
    if (e >= E) return;
    int pos = chunk_base[static_cast<size_t>(blockIdx.x) * E + e];
    bool bad = false;
    for (int tt = 0; tt < nt; ++tt) {
        for (int j = 0; j < k; ++j) {
            if (sidx[tt * k + j] == e) {
                const int p = (t0 + tt) * k + j;
                if (pos >= 0 && pos < p_cap) {
                    perm[pos] = p;
                    inv[p] = pos;
                } else {
                    bad = true;
                }
                ++pos;
                break;
            }
        }
    }
    if (bad) report_status(status, kStatusBadIndex);
}

constexpr int kBwdThreads = 256;

__global__ void __launch_bounds__(kBwdThreads) route_bwd_kernel(int T, int E, int k, const float *__restrict__ w,
                                                                const int32_t *__restrict__ idx,
                                                                const int32_t *__restrict__ inv,
                                                                const float *__restrict__ dpart, int dpart_stride,
                                                                float *__restrict__ dscore,
                                                                float *__restrict__ dlogits) {
    __shared__ float s_ds[kBwdThreads / 32][kMaxTopK];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int t = blockIdx.x * (kBwdThreads / 32) + warp;
    if (t >= T) return;
    if (dlogits)
        for (int e = lane; e < E; e += 32) dlogits[static_cast<size_t>(t) * E + e] = 0.f;
    for (int j = lane; j < k; j += 32) {
        const int pos = inv[static_cast<size_t>(t) * k + j];
        float ds = 0.f;
        for (int n = 0; n < dpart_stride; ++n) ds += dpart[static_cast<size_t>(pos) * dpart_stride + n];
        dscore[static_cast<size_t>(t) * k + j] = ds;
        s_ds[warp][j] = ds;
    }
    __syncwarp();
    if (!dlogits) return;
    float s = 0.f;
    if (lane == 0)
        for (int j = 0; j < k; ++j) s += w[static_cast<size_t>(t) * k + j] * s_ds[warp][j];
    s = __shfl_sync(0xffffffffu, s, 0);
    for (int j = lane; j < k; j += 32) {
        const float wj = w[static_cast<size_t>(t) * k + j];
        dlogits[static_cast<size_t>(t) * E + idx[static_cast<size_t>(t) * k + j]] = wj * (s_ds[warp][j] - s);
    }
}

// Backward only: copies of x and grad_out in the expert-sorted layout (row pos
// = token of perm[pos]; padding rows are zero).  Flat over (row, 16-byte
// piece), four independent pieces per thread per step.
__global__ void __launch_bounds__(256) sort_rows_kernel(const int32_t *__restrict__ perm,
                                                        const int32_t *__restrict__ group_start, int E, int k,
                                                        int TK, int d, const __nv_bfloat16 *__restrict__ x,
                                                        const __nv_bfloat16 *__restrict__ g,
                                                        __nv_bfloat16 *__restrict__ xs, __nv_bfloat16 *__restrict__ gs) {
    const int n16 = d / 8;  // 16-byte pieces per row
    const int total = group_start[E] * n16;
    const int stride = gridDim.x * blockDim.x;
    const uint4 zero = make_uint4(0u, 0u, 0u, 0u);
    const uint4 *x4 = reinterpret_cast<const uint4 *>(x);
    const uint4 *g4 = reinterpret_cast<const uint4 *>(g);
    uint4 *xs4 = reinterpret_cast<uint4 *>(xs);
    uint4 *gs4 = reinterpret_cast<uint4 *>(gs);
    for (int base = blockIdx.x * blockDim.x + threadIdx.x; base < total; base += 4 * stride) {
        uint4 xv[4], gv[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const int i = base + u * stride;
            xv[u] = gv[u] = zero;
            if (i < total) {
                const int row = i / n16, piece = i - row * n16;
                const int p = __ldg(perm + row);
                if (p >= 0 && p < TK) {
                    const size_t src = static_cast<size_t>(p / k) * n16 + piece;
                    xv[u] = __ldg(x4 + src);
                    gv[u] = __ldg(g4 + src);
                }
            }
        }
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const int i = base + u * stride;
            if (i < total) {
                xs4[i] = xv[u];
                gs4[i] = gv[u];
            }
        }
    }
}

}  // namespace

cudaError_t launch_sort_rows(const int32_t *perm, const int32_t *group_start, int E, int k, int T, int d,
                             const __nv_bfloat16 *x, const __nv_bfloat16 *g, __nv_bfloat16 *xs, __nv_bfloat16 *gs,
                             int sms, cudaStream_t s) {
    sort_rows_kernel<<<sms * 8, 256, 0, s>>>(perm, group_start, E, k, T * k, d, x, g, xs, gs);  // 8 x 256 threads per SM
    return cudaGetLastError();
}

cudaError_t launch_route_topk(const float *logits, int T, int E, int k, int32_t *idx, float *w,
                              int32_t *chunk_counts, int32_t *cnt, int cnt_per_token, cudaStream_t s) {
    const int blocks = (T + kRouteChunk - 1) / kRouteChunk;
    const int nv = (E + 31) / 32;
    if (nv <= 1)
        route_topk_kernel<1><<<blocks, kTopkThreads, 0, s>>>(logits, T, E, k, idx, w, chunk_counts, cnt, cnt_per_token);
    else if (nv <= 2)
        route_topk_kernel<2><<<blocks, kTopkThreads, 0, s>>>(logits, T, E, k, idx, w, chunk_counts, cnt, cnt_per_token);
    else if (nv <= 4)
        route_topk_kernel<4><<<blocks, kTopkThreads, 0, s>>>(logits, T, E, k, idx, w, chunk_counts, cnt, cnt_per_token);
    else if (nv <= 8)
        route_topk_kernel<8><<<blocks, kTopkThreads, 0, s>>>(logits, T, E, k, idx, w, chunk_counts, cnt, cnt_per_token);
    else
        route_topk_kernel<16><<<blocks, kTopkThreads, 0, s>>>(logits, T, E, k, idx, w, chunk_counts, cnt, cnt_per_token);
    return cudaGetLastError();
}

cudaError_t launch_route_scan(int T, int E, int n_chunks, const int32_t *chunk_counts, int32_t *chunk_base,
                              int32_t *counts, int32_t *offsets, int32_t *group_start, int32_t *tile_expert,
                              int32_t *perm, int64_t p_cap, int *status, cudaStream_t s) {
    (void)T;
    route_scan_kernel<<<1, kScanThreads, 0, s>>>(E, n_chunks, chunk_counts, chunk_base, counts, offsets,
                                                 group_start, tile_expert, perm, p_cap, status);
    return cudaGetLastError();
}

cudaError_t launch_route_perm(int T, int E, int k, const int32_t *idx, const int32_t *chunk_base, int32_t *perm,
                              int32_t *inv, int64_t p_cap, int *status, cudaStream_t s) {
    const int blocks = (T + kRouteChunk - 1) / kRouteChunk;
    const int threads = (E + 31) / 32 * 32;
    route_perm_kernel<<<blocks, threads, 0, s>>>(T, E, k, idx, chunk_base, perm, inv, p_cap, status);
    return cudaGetLastError();
}

cudaError_t launch_route_bwd(int T, int E, int k, const float *w, const int32_t *idx, const int32_t *inv,
                             const float *dpart, int dpart_stride, float *dscore, float *dlogits, cudaStream_t s) {
    const int per_block = kBwdThreads / 32;
    const int blocks = (T + per_block - 1) / per_block;
    route_bwd_kernel<<<blocks, kBwdThreads, 0, s>>>(T, E, k, w, idx, inv, dpart, dpart_stride, dscore, dlogits);
    return cudaGetLastError();
}

}  // namespace moe

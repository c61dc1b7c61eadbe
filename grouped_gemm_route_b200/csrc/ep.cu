// Kernels of the expert-parallel path: the layer's experts are spread over G
// GPUs; each GPU routes its own tokens, sends every (token, slot) row to the
// GPU that owns the chosen expert, runs its experts on the rows it receives,
// and sends the results back ("Prime Intellect's Prime Mega MoE Trains Giant
// AI Models 55% Faster", sections "Where MoE training loses time" and "One
// kernel overlaps the pipeline").  The exchanges themselves are NCCL
// point-to-point copies between the GPUs' own buffers, issued by the caller;
// these kernels build and consume the layouts those copies move.
//
// Layouts.  On the sending side the rows of a token's pairs are in the
// library's sorted layout: experts ascending, each expert's group starting at
// group_start[e] (a multiple of 128) -- so the rows bound for one GPU, whose
// experts are consecutive, are consecutive groups.  The "compact" sorted order
// is the same order without the padding: pair p of expert e at offsets[e] +
// (its row - group_start[e]).  On the expert side, the rows of local expert e
// from source s follow those of sources 0..s-1, and the groups are padded to
// 128 rows again (the grouped GEMMs' tiles); perm maps a padded row to its
// compact index, inv the compact index back to its padded row.
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "moe_internal.h"
#include "ptx.cuh"

namespace moe {

namespace {

// w_rows[offsets[e] + i] = topk_w of the pair at sorted row group_start[e] + i
// (i < counts[e]): the routing weight of every row, in compact sorted order.
__global__ void __launch_bounds__(256) ep_row_weights_kernel(const int32_t *__restrict__ perm,
                                                             const int32_t *__restrict__ tile_expert,
                                                             const int32_t *__restrict__ counts,
                                                             const int32_t *__restrict__ offsets,
                                                             const int32_t *__restrict__ group_start,
                                                             const float *__restrict__ topk_w, int E, int64_t P,
                                                             float *__restrict__ w_rows) {
    const int used = group_start[E];
    for (int pos = blockIdx.x * blockDim.x + threadIdx.x; pos < used; pos += gridDim.x * blockDim.x) {
        const int e = tile_expert[pos / kTileM];
        if (e < 0 || e >= E) continue;
        const int i = pos - group_start[e];
        const int p = perm[pos];
        if (i < counts[e] && p >= 0 && p < P) w_rows[offsets[e] + i] = topk_w[p];
    }
}

// Expert side: from recv[s][e] (rows of local expert e sent by source s),
// the local routing state of the received rows.  One block.
constexpr int kLayoutThreads = 1024;

__global__ void __launch_bounds__(kLayoutThreads) ep_layout_kernel(int G, int E, const int32_t *__restrict__ recv,
                                                                   int64_t p_cap, int32_t *__restrict__ counts,
                                                                   int32_t *__restrict__ offsets,
                                                                   int32_t *__restrict__ group_start,
                                                                   int32_t *__restrict__ tile_expert,
                                                                   int32_t *__restrict__ perm,
                                                                   int32_t *__restrict__ inv, int *status) {
    __shared__ int s_cnt[kMaxExperts];
    __shared__ int s_off[kMaxExperts + 1];
    __shared__ int s_gs[kMaxExperts + 1];
    for (int e = threadIdx.x; e < E; e += blockDim.x) {
        int c = 0;
        for (int s = 0; s < G; ++s) c += recv[static_cast<int64_t>(s) * E + e];
        s_cnt[e] = c;
        counts[e] = c;
    }
    __syncthreads();
    if (threadIdx.x == 0) {  // E <= 512 experts: a short serial scan
        int off = 0, gs = 0;
        for (int e = 0; e < E; ++e) {
            s_off[e] = off;
            s_gs[e] = gs;
            off += s_cnt[e];
            gs += (s_cnt[e] + kTileM - 1) / kTileM * kTileM;
        }
        s_off[E] = off;
        s_gs[E] = gs;
        if (gs > p_cap) report_status(status, kStatusBadIndex);
    }
    __syncthreads();
    for (int e = threadIdx.x; e <= E; e += blockDim.x) {
        offsets[e] = s_off[e];
        group_start[e] = s_gs[e];
    }
    if (s_gs[E] > p_cap) return;
    for (int e = 0; e < E; ++e) {
        const int gs = s_gs[e], ge = s_gs[e + 1], c = s_cnt[e], off = s_off[e];
        for (int mt = gs / kTileM + threadIdx.x; mt < ge / kTileM; mt += blockDim.x) tile_expert[mt] = e;
        for (int pos = gs + threadIdx.x; pos < ge; pos += blockDim.x) {
            const int i = pos - gs;
            perm[pos] = i < c ? off + i : -1;
            if (i < c) inv[off + i] = pos;
        }
    }
}

// out[t] = sum over slots j = 0..k-1, in slot order, of the compact rows
// u(t, j) = offsets[e] + inv[t, j] - group_start[e] (e = idx[t, j]), summed in
// fp32 and rounded to bf16 once -- the same sums as combine_rows over the
// slot-addressed staging rows.  One thread per 16-byte piece of a token's row.
__global__ void __launch_bounds__(256) ep_combine_kernel(const __nv_bfloat16 *__restrict__ rows,
                                                         const int32_t *__restrict__ idx,
                                                         const int32_t *__restrict__ inv,
                                                         const int32_t *__restrict__ offsets,
                                                         const int32_t *__restrict__ group_start, int T, int E,
                                                         int k, int d, int64_t P, __nv_bfloat16 *__restrict__ out,
                                                         int *status) {
    const int n16 = d / 8;
    const int64_t total = static_cast<int64_t>(T) * n16;
    const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
    const uint4 *src = reinterpret_cast<const uint4 *>(rows);
    uint4 *dst = reinterpret_cast<uint4 *>(out);
    bool bad = false;
    for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < total; i += stride) {
        const int64_t t = i / n16;
        const int64_t piece = i - t * n16;
        float acc[8];
#pragma unroll
        for (int q = 0; q < 8; ++q) acc[q] = 0.f;
        for (int j = 0; j < k; ++j) {  // slot order
            const int e = __ldg(idx + t * k + j);
            int64_t u = -1;
            if (e >= 0 && e < E) u = static_cast<int64_t>(__ldg(offsets + e)) + __ldg(inv + t * k + j) - __ldg(group_start + e);
            if (u < 0 || u >= P) {
                bad = true;
                continue;
            }
            const uint4 v = __ldcs(src + u * n16 + piece);
            const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                acc[2 * q] += bf16_lo(w[q]);
                acc[2 * q + 1] += bf16_hi(w[q]);
            }
        }
        dst[i] = make_uint4(pack_bf16x2(acc[0], acc[1]), pack_bf16x2(acc[2], acc[3]), pack_bf16x2(acc[4], acc[5]),
                            pack_bf16x2(acc[6], acc[7]));
    }
    if (bad && status != nullptr) report_status(status, kStatusBadIndex);
}

}  // namespace

cudaError_t launch_ep_row_weights(const int32_t *perm, const int32_t *tile_expert, const int32_t *counts,
                                  const int32_t *offsets, const int32_t *group_start, const float *topk_w, int E,
                                  int64_t P, int64_t p_cap, float *w_rows, int sms, cudaStream_t s) {
    const int64_t want = (p_cap + 255) / 256;
    const int blocks = static_cast<int>(want < 4LL * sms ? (want > 0 ? want : 1) : 4LL * sms);
    ep_row_weights_kernel<<<blocks, 256, 0, s>>>(perm, tile_expert, counts, offsets, group_start, topk_w, E, P,
                                                 w_rows);
    return cudaGetLastError();
}

cudaError_t launch_ep_layout(int G, int E, const int32_t *recv, int64_t p_cap, int32_t *counts, int32_t *offsets,
                             int32_t *group_start, int32_t *tile_expert, int32_t *perm, int32_t *inv, int *status,
                             cudaStream_t s) {
    ep_layout_kernel<<<1, kLayoutThreads, 0, s>>>(G, E, recv, p_cap, counts, offsets, group_start, tile_expert, perm,
                                                  inv, status);
    return cudaGetLastError();
}

cudaError_t launch_ep_combine(const __nv_bfloat16 *rows, const int32_t *idx, const int32_t *inv,
                              const int32_t *offsets, const int32_t *group_start, int T, int E, int k, int d,
                              int64_t P, __nv_bfloat16 *out, int *status, int sms, cudaStream_t s) {
    ep_combine_kernel<<<sms * 8, 256, 0, s>>>(rows, idx, inv, offsets, group_start, T, E, k, d, P, out, status);
    return cudaGetLastError();
}

}  // namespace moe

// Routing and dispatch kernels of the fused MoE layer, the routing-score
// backward, and the two data-movement passes around the GEMMs: the copies of x
// and grad_out in the expert-sorted layout (sort_rows) and the slot-ordered sum
// of staged rows into out / dx (combine_rows).
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
// The layer routes with one cooperative launch (route_fused, below: a
// lane-per-token form for E <= 128 and a warp-per-token form otherwise).  The
// three-launch form right below serves moe_route_noalloc: (1) per token top-k +
// weights + a per-block expert histogram, (2) one block: totals, exclusive
// scans, per-block bases, tile table, padding, (3) per block: each thread owns
// one expert and walks the block's tokens in order, so positions inside an
// expert follow token order exactly.
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
                                                                  int32_t *__restrict__ chunk_counts) {
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

// ---------------------------------------------------------------------------
// Fused routing: the three steps above in one cooperative launch.  Block b of
// G owns the contiguous tokens [T*b/G, T*(b+1)/G), and warp w of the block a
// contiguous sub-range of those, so (block, warp, token, slot) order is token
// order.  Phases, separated by grid barriers (every block resident: the launch
// is cooperative; every wait is bounded):
//   1  per token top-k and weights; per-warp expert histograms;
//      the block's histogram to blk_hist[b]
//   2  block b scans expert e = b, b+G, ... over the G blocks: blk_base[.][e],
//      counts[e]
//   3  every block: padded exclusive scan of counts (group starts); block 0
//      publishes it; each block writes the tile table and padding rows of its
//      experts and the sorted position of each of its pairs, walking each
//      warp's tokens in order with one lane per slot (a token's k experts are
//      distinct, so the lanes never update the same counter).
// ---------------------------------------------------------------------------
constexpr int kFusedThreads = 512;
constexpr int kFusedWarps = kFusedThreads / 32;
static_assert(kFusedThreads >= kMaxExperts, "phase 3 scans one expert per thread");

struct RouteFusedArgs {
    const float *logits;
    int T, E, k;
    int32_t *idx;
    float *w;
    int32_t *blk_hist;  // [G, E]
    int32_t *blk_base;  // [G, E]
    int32_t *counts, *offsets, *group_start, *tile_expert, *perm, *inv;
    int64_t p_cap;
    unsigned *barrier;  // zero before the launch
    int *status;
    int lane_stages;    // lane form: ring depth per warp
};

__device__ __forceinline__ unsigned ld_acquire_gpu(const unsigned *p) {
    unsigned v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

// All blocks of the grid arrive, then wait (bounded) until `target` arrivals
// are counted.  Returns false for every thread of a block whose wait expired
// (the status word then holds a timeout).
__device__ bool grid_barrier(unsigned *ctr, unsigned target, int *status) {
    __shared__ int s_ok;
    __syncthreads();
    if (threadIdx.x == 0) {
        __threadfence();
        atomicAdd(ctr, 1u);
        const uint64_t t0 = global_timer_ns();
        int ok = 1;
        while (ld_acquire_gpu(ctr) < target) {
            if (global_timer_ns() - t0 > kWaitLimitNs) {
                report_status(status, kStatusTimeout);
                ok = 0;
                break;
            }
            __nanosleep(32);
        }
        __threadfence();
        s_ok = ok;
    }
    __syncthreads();
    return s_ok != 0;
}

// Exclusive scan of one int per thread over the block; returns the block total.
__device__ __forceinline__ int block_exclusive_scan(int v, int &excl, int *warp_sums) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    int incl = v;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const int o = __shfl_up_sync(0xffffffffu, incl, off);
        if (lane >= off) incl += o;
    }
    __syncthreads();  // warp_sums free from any earlier use
    if (lane == 31) warp_sums[warp] = incl;
    __syncthreads();
    int base = 0, total = 0;
    const int nwarps = static_cast<int>(blockDim.x >> 5);
    for (int i = 0; i < nwarps; ++i) {
        const int ws = warp_sums[i];
        if (i < warp) base += ws;
        total += ws;
    }
    excl = base + incl - v;
    return total;
}

// Phase 2 of both routing kernels: block b scans expert e = b, b+G, ... over
// the G blocks' histograms (blk_base[.][e] exclusive, counts[e] the total).
__device__ void route_scan_experts(const RouteFusedArgs &a, int *warp_sums) {
    const int E = a.E, G = gridDim.x;
    for (int e = blockIdx.x; e < E; e += G) {
        int carry = 0;
        for (int c0 = 0; c0 < G; c0 += blockDim.x) {
            const int bb = c0 + threadIdx.x;
            const int v = bb < G ? __ldcg(a.blk_hist + static_cast<size_t>(bb) * E + e) : 0;
            int excl;
            const int tot = block_exclusive_scan(v, excl, warp_sums);
            if (bb < G) a.blk_base[static_cast<size_t>(bb) * E + e] = carry + excl;
            carry += tot;
        }
        if (threadIdx.x == 0) a.counts[e] = carry;
    }
}

// Phase 3 start of both routing kernels (E <= blockDim.x: one expert per
// thread): padded group starts into gst[0..E] (block 0 also publishes them
// with the unpadded offsets), then the tile table and padding rows of experts
// b, b+G, ...  Returns false when the groups exceed the sorted capacity.
__device__ bool route_group_layout(const RouteFusedArgs &a, int *gst, int *warp_sums) {
    const int E = a.E, b = blockIdx.x, G = gridDim.x;
    int c_excl = 0, p_excl = 0;
    const int e = threadIdx.x;
    const int c = e < E ? __ldcg(a.counts + e) : 0;
    const int padded = (c + kTileM - 1) / kTileM * kTileM;
    const int c_tot = block_exclusive_scan(c, c_excl, warp_sums);
    const int p_tot = block_exclusive_scan(padded, p_excl, warp_sums);
    if (e < E) gst[e] = p_excl;
    if (e == 0) gst[E] = p_tot;
    if (b == 0 && e < E) {
        a.group_start[e] = p_excl;
        a.offsets[e] = c_excl;
    }
    if (b == 0 && e == 0) {
        a.group_start[E] = p_tot;
        a.offsets[E] = c_tot;
        if (p_tot > a.p_cap) report_status(a.status, kStatusBadIndex);
    }
    __syncthreads();
    if (gst[E] > a.p_cap) return false;
    for (int x = b; x < E; x += G) {
        const int gs = gst[x], ge = gst[x + 1], cx = __ldcg(a.counts + x);
        for (int mt = gs / kTileM + threadIdx.x; mt < ge / kTileM; mt += blockDim.x) a.tile_expert[mt] = x;
        for (int q = gs + cx + threadIdx.x; q < ge; q += blockDim.x) a.perm[q] = -1;
    }
    return true;
}

// Turns per-warp expert counts wcnt[nwarps][E] into each warp's first sorted
// position per expert: group start + earlier blocks + earlier warps.
__device__ void route_warp_bases(const RouteFusedArgs &a, int *wcnt, const int *gst, int nwarps) {
    const int E = a.E;
    for (int e = threadIdx.x; e < E; e += blockDim.x) {
        int run = gst[e] + __ldcg(a.blk_base + static_cast<size_t>(blockIdx.x) * E + e);
        for (int q = 0; q < nwarps; ++q) {
            const int c = wcnt[q * E + e];
            wcnt[q * E + e] = run;
            run += c;
        }
    }
    __syncthreads();
}

// Top-k key of a logit: the high word orders fp32 values (-0 and +0 equal,
// finite values assumed), the low word is ~expert so that among equal values
// the lower expert index is larger.  0 is below every real key.
__device__ __forceinline__ uint64_t topk_key(float v, int e) {
    const uint32_t u = __float_as_uint(v == 0.f ? 0.f : v);
    const uint32_t hi = (u & 0x80000000u) ? ~u : (u | 0x80000000u);
    return (static_cast<uint64_t>(hi) << 32) | static_cast<uint32_t>(~e);
}

__device__ __forceinline__ float topk_value(uint32_t hi) {
    return __uint_as_float((hi & 0x80000000u) ? (hi & 0x7FFFFFFFu) : ~hi);
}

template <int NV>
__global__ void __launch_bounds__(kFusedThreads) route_fused_kernel(const RouteFusedArgs a) {
    extern __shared__ int smem_i[];
    const int E = a.E, k = a.k, G = gridDim.x, b = blockIdx.x;
    int *wcnt = smem_i;                          // [kFusedWarps][E] per-warp counts, then bases
    int *gst = wcnt + kFusedWarps * E;           // [E + 1] padded group starts
    int *warp_sums = gst + E + 1;                // [kFusedWarps]
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int t0 = static_cast<int>(static_cast<int64_t>(a.T) * b / G);
    const int t1 = static_cast<int>(static_cast<int64_t>(a.T) * (b + 1) / G);
    const int nb = t1 - t0;
    const int wt0 = t0 + nb * warp / kFusedWarps, wt1 = t0 + nb * (warp + 1) / kFusedWarps;
    for (int i = threadIdx.x; i < kFusedWarps * E; i += kFusedThreads) wcnt[i] = 0;
    __syncthreads();

    // ---- phase 1: top-k of each token, kTokPar tokens at a time per warp ----
    constexpr int kTokPar = NV <= 4 ? 2 : 1;
    for (int t = wt0; t < wt1; t += kTokPar) {
        uint64_t c[kTokPar][NV];  // this lane's (value, expert) keys, sorted descending
        uint64_t sel[kTokPar][2];  // slots lane and lane + 32 after the rounds
        uint32_t vmax[kTokPar];
#pragma unroll
        for (int u = 0; u < kTokPar; ++u) {
            const bool live = t + u < wt1;
#pragma unroll
            for (int i = 0; i < NV; ++i) {
                const int e = lane + 32 * i;
                c[u][i] = live && e < E ? topk_key(__ldg(a.logits + static_cast<size_t>(t + u) * E + e), e) : 0ull;
            }
#pragma unroll
            for (int i = 1; i < NV; ++i)
#pragma unroll
                for (int q = i; q > 0; --q) {
                    const uint64_t x0 = c[u][q - 1], x1 = c[u][q];
                    const bool sw = x1 > x0;
                    c[u][q - 1] = sw ? x1 : x0;
                    c[u][q] = sw ? x0 : x1;
                }
            sel[u][0] = sel[u][1] = 0ull;
        }
        // round j: the warp's largest head key is slot j; its lane pops it
        for (int j = 0; j < k; ++j) {
#pragma unroll
            for (int u = 0; u < kTokPar; ++u) {
                const uint32_t hi = static_cast<uint32_t>(c[u][0] >> 32), lo = static_cast<uint32_t>(c[u][0]);
                const uint32_t m_hi = __reduce_max_sync(0xffffffffu, hi);
                const uint32_t m_lo = __reduce_max_sync(0xffffffffu, hi == m_hi ? lo : 0u);
                if (j == 0) vmax[u] = m_hi;
                if (hi == m_hi && lo == m_lo) {
#pragma unroll
                    for (int i = 0; i + 1 < NV; ++i) c[u][i] = c[u][i + 1];
                    c[u][NV - 1] = 0ull;
                }
                const uint64_t key = (static_cast<uint64_t>(m_hi) << 32) | m_lo;
                if (lane == (j & 31)) {
                    if (j < 32)
                        sel[u][0] = key;
                    else
                        sel[u][1] = key;
                }
            }
        }
        // weights: exp(l_j - l_max) over the chosen k, normalised by their sum
        // taken in slot order (the same sum, bit for bit, as the lane form's)
#pragma unroll
        for (int u = 0; u < kTokPar; ++u) {
            const int tt = t + u;
            const float m = topk_value(vmax[u]);
            float p[2], sum = 0.f;
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const int j = lane + 32 * h;
                p[h] = j < k ? expf(topk_value(static_cast<uint32_t>(sel[u][h] >> 32)) - m) : 0.f;
            }
            for (int j = 0; j < k; ++j) sum += __shfl_sync(0xffffffffu, j < 32 ? p[0] : p[1], j & 31);
            if (tt < wt1) {
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    const int j = lane + 32 * h;
                    if (j < k) {
                        const int e = static_cast<int>(~static_cast<uint32_t>(sel[u][h]));
                        a.idx[static_cast<size_t>(tt) * k + j] = e;
                        a.w[static_cast<size_t>(tt) * k + j] = p[h] / sum;
                        wcnt[warp * E + e] += 1;  // the k experts of a token are distinct
                    }
                }
            }
        }
        __syncwarp();
    }
    __syncthreads();
    for (int e = threadIdx.x; e < E; e += kFusedThreads) {
        int sum = 0;
        for (int q = 0; q < kFusedWarps; ++q) sum += wcnt[q * E + e];
        a.blk_hist[static_cast<size_t>(b) * E + e] = sum;
    }
    if (!grid_barrier(a.barrier, G, a.status)) return;

    // ---- phase 2: per expert, exclusive scan over the blocks ----
    route_scan_experts(a, warp_sums);
    if (!grid_barrier(a.barrier, 2u * G, a.status)) return;

    // ---- phase 3: group starts, tile table, padding, positions ----
    if (!route_group_layout(a, gst, warp_sums)) return;
    route_warp_bases(a, wcnt, gst, kFusedWarps);
    bool bad = false;
    for (int t = wt0; t < wt1; ++t) {
        for (int j = lane; j < k; j += 32) {
            const int p = t * k + j;
            const int e = a.idx[p];  // written by this thread in phase 1
            const int pos = wcnt[warp * E + e];
            wcnt[warp * E + e] = pos + 1;
            if (pos >= 0 && pos < gst[e + 1]) {
                a.perm[pos] = p;
                a.inv[p] = pos;
            } else {
                bad = true;
            }
        }
        __syncwarp();
    }
    if (bad) report_status(a.status, kStatusBadIndex);
}

// ---------------------------------------------------------------------------
// Fused routing, lane-per-token form, for E <= 128 with E a multiple of 4k,
// k <= 8 and 16-byte aligned logits.  Same phases and the same results as
// route_fused_kernel; phase 1 and the positions of phase 3 give each lane one
// token:
//   * each lane copies its token's logit row into shared memory with one bulk
//     copy (rows padded by 4 words, so that one-row-per-lane reads do not
//     conflict); a warp's buffers form a ring of `stages` batches of 32 rows,
//     the next batch in flight while the current one is processed;
//   * tau, a lower bound on the k-th largest logit: the row is split into NG
//     disjoint groups of consecutive experts (NG = 2k when E is a multiple of
//     8k, else k) and tau is the k-th largest group maximum -- k groups have a
//     maximum >= tau, so at least k logits are >= tau and each of the k
//     largest is;
//   * the logits >= tau (a bitmask) are visited in expert order and inserted
//     into k sorted registers of (order key, expert): a strictly larger key
//     moves ahead, an equal key stays behind the lower experts already there,
//     which leaves the k largest in slot order (value descending, lower
//     expert first on ties);
//   * weights as in route_fused_kernel, the sum taken in slot order.
// Positions: per batch of 32 tokens, each expert's set of lanes (a bitmask
// built with atomicOr) gives a pair's rank among the batch's earlier tokens;
// the highest of those lanes then advances the warp's running position.
// ---------------------------------------------------------------------------
constexpr int kLaneMaxWarps = 16;
constexpr int kLaneMaxE = 128;
constexpr int kLaneMaxK = 8;
constexpr size_t kLaneSmemLimit = 227u * 1024u;

// Byte offsets of the lane kernel's shared memory.
struct LaneSmem {
    int stride;  // words per staged row
    size_t bars, wcnt, emask, gst, wsum, total;
};

__host__ __device__ inline LaneSmem lane_smem_layout(int E, int warps, int stages) {
    LaneSmem L;
    L.stride = E + 4;
    L.bars = static_cast<size_t>(warps) * stages * 32 * L.stride * 4;  // staged rows first
    L.wcnt = L.bars + static_cast<size_t>(warps) * stages * 8;        // [warps][stages] mbarriers
    L.emask = L.wcnt + static_cast<size_t>(warps) * E * 4;            // [warps][E] counts, then bases
    L.gst = L.emask + static_cast<size_t>(warps) * E * 4;             // [warps][E] lane masks
    L.wsum = L.gst + static_cast<size_t>(E + 1) * 4;                  // [E + 1] group starts
    L.total = L.wsum + static_cast<size_t>(warps) * 4;                // [warps] scan scratch
    return L;
}

__device__ __forceinline__ uint32_t order_key(float v) {
    const uint32_t u = __float_as_uint(v == 0.f ? 0.f : v);
    return u ^ (static_cast<uint32_t>(static_cast<int32_t>(u) >> 31) | 0x80000000u);
}

// The k-th largest of g[0 .. NGM*K): the minimum when NGM == 1; for NGM == 2
// each half is sorted (descending, odd-even transposition) and the k-th
// largest of two sorted lists A, B is max over i of min(A_i, B_(k-i)), A_i the
// i-th largest of A and A_0 = +inf.
template <int K, int NGM>
__device__ __forceinline__ float kth_largest(float (&g)[NGM * K]) {
    if constexpr (NGM == 1) {
        float t = g[0];
#pragma unroll
        for (int j = 1; j < K; ++j) t = fminf(t, g[j]);
        return t;
    } else {
#pragma unroll
        for (int h = 0; h < 2; ++h) {
#pragma unroll
            for (int r = 0; r < K; ++r) {
#pragma unroll
                for (int i = h * K + (r & 1); i + 1 < (h + 1) * K; i += 2) {
                    const float hi = fmaxf(g[i], g[i + 1]), lo = fminf(g[i], g[i + 1]);
                    g[i] = hi;
                    g[i + 1] = lo;
                }
            }
        }
        float t = fmaxf(g[K - 1], g[2 * K - 1]);
#pragma unroll
        for (int i = 1; i < K; ++i) t = fmaxf(t, fminf(g[i - 1], g[2 * K - 1 - i]));
        return t;
    }
}

template <int K, int NGM>
__global__ void __launch_bounds__(kLaneMaxWarps * 32, 1) route_lane_kernel(const RouteFusedArgs a) {
    extern __shared__ __align__(16) uint8_t sm_b[];
    constexpr int NG = NGM * K;
    const int E = a.E, G = gridDim.x, b = blockIdx.x, S = a.lane_stages;
    const int nw = static_cast<int>(blockDim.x >> 5);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const LaneSmem L = lane_smem_layout(E, nw, S);
    const int stride = L.stride;
    const float *stage = reinterpret_cast<const float *>(sm_b) + static_cast<size_t>(warp) * S * 32 * stride;
    uint64_t *bar = reinterpret_cast<uint64_t *>(sm_b + L.bars) + warp * S;
    int *wcnt = reinterpret_cast<int *>(sm_b + L.wcnt);
    uint32_t *emask = reinterpret_cast<uint32_t *>(sm_b + L.emask);
    int *gst = reinterpret_cast<int *>(sm_b + L.gst);
    int *warp_sums = reinterpret_cast<int *>(sm_b + L.wsum);
    const int t0 = static_cast<int>(static_cast<int64_t>(a.T) * b / G);
    const int t1 = static_cast<int>(static_cast<int64_t>(a.T) * (b + 1) / G);
    const int nb = t1 - t0;
    const int wt0 = t0 + nb * warp / nw, wt1 = t0 + nb * (warp + 1) / nw;
    const int nbatch = (wt1 - wt0 + 31) / 32;
    const bool vec_k = (K % 4 == 0) && ((reinterpret_cast<uintptr_t>(a.idx) | reinterpret_cast<uintptr_t>(a.w)) & 15u) == 0;
    for (int i = threadIdx.x; i < nw * E; i += blockDim.x) {
        wcnt[i] = 0;
        emask[i] = 0u;
    }
    if (lane == 0) {
        for (int s = 0; s < S; ++s) mbar_init(&bar[s], 1);
        fence_barrier_init();
    }
    __syncthreads();

    // Batch `it` of this warp (32 rows from token wt0 + 32*it) into ring slot it % S.
    auto issue = [&](int it) {
        const int tb = wt0 + 32 * it, rows = min(32, wt1 - tb), s = it % S;
        fence_proxy_async_smem();  // this lane's earlier reads of the slot come first
        __syncwarp();
        if (lane == 0) mbar_arrive_expect_tx(&bar[s], static_cast<uint32_t>(rows * E) * 4u);
        __syncwarp();
        if (lane < rows)
            bulk_load(const_cast<float *>(stage) + static_cast<size_t>(s * 32 + lane) * stride,
                      a.logits + static_cast<size_t>(tb + lane) * E, static_cast<uint32_t>(E) * 4u, &bar[s]);
    };

    // ---- phase 1: top-k, one token per lane ----
    const int E4 = E / 4, gq = E / (4 * NG);  // float4s per row, per group
    bool wait_ok = true;
    int it = 0;
    for (int p = 0; p < S && p < nbatch; ++p) issue(p);
    for (; it < nbatch; ++it) {
        const int tb = wt0 + 32 * it, rows = min(32, wt1 - tb), s = it % S;
        const bool arrived = mbar_wait(&bar[s], static_cast<uint32_t>(it / S) & 1u, nullptr);
        if (!__all_sync(0xffffffffu, arrived)) {
            wait_ok = false;
            break;
        }
        const bool live = lane < rows;
        const float4 *r4 = reinterpret_cast<const float4 *>(stage + static_cast<size_t>(s * 32 + lane) * stride);
        uint64_t mlo = 0ull, mhi = 0ull;  // logits >= tau: experts 0..63, 64..127
        int ncand = 0;
        if (live) {
            float gm[NG];
#pragma unroll
            for (int g = 0; g < NG; ++g) {
                float mx = -INFINITY;
#pragma unroll
                for (int q = 0; q < 32 / NG; ++q) {
                    if (q < gq) {
                        const float4 v = r4[g * gq + q];
                        mx = fmaxf(mx, fmaxf(fmaxf(v.x, v.y), fmaxf(v.z, v.w)));
                    }
                }
                gm[g] = mx;
            }
            const float tau = kth_largest<K, NGM>(gm);
            uint32_t m[4] = {0u, 0u, 0u, 0u};
#pragma unroll
            for (int wd = 0; wd < 4; ++wd) {
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    if (8 * wd + j < E4) {
                        const float4 v = r4[8 * wd + j];
                        uint32_t bits = 0u;
                        if (v.x >= tau) bits |= 1u << (4 * j);
                        if (v.y >= tau) bits |= 2u << (4 * j);
                        if (v.z >= tau) bits |= 4u << (4 * j);
                        if (v.w >= tau) bits |= 8u << (4 * j);
                        m[wd] |= bits;
                    }
                }
            }
            mlo = (static_cast<uint64_t>(m[1]) << 32) | m[0];
            mhi = (static_cast<uint64_t>(m[3]) << 32) | m[2];
            ncand = __popcll(mlo) + __popcll(mhi);
        }
        uint32_t tk[K];
        int ti[K];
#pragma unroll
        for (int j = 0; j < K; ++j) {
            tk[j] = 0u;  // below every real key
            ti[j] = 0;
        }
        const float *row = reinterpret_cast<const float *>(r4);
        const int cmax = static_cast<int>(__reduce_max_sync(0xffffffffu, static_cast<unsigned>(ncand)));
        for (int c = 0; c < cmax; ++c) {
            if (c < ncand) {
                const bool in_lo = mlo != 0ull;
                const uint64_t cur = in_lo ? mlo : mhi;
                const int e = __ffsll(static_cast<long long>(cur)) - 1 + (in_lo ? 0 : 64);
                const uint64_t rest = cur & (cur - 1ull);
                if (in_lo)
                    mlo = rest;
                else
                    mhi = rest;
                const uint32_t xk = order_key(row[e]);
                bool gt[K];
#pragma unroll
                for (int j = 0; j < K; ++j) gt[j] = xk > tk[j];
#pragma unroll
                for (int j = K - 1; j > 0; --j) {
                    tk[j] = gt[j - 1] ? tk[j - 1] : (gt[j] ? xk : tk[j]);
                    ti[j] = gt[j - 1] ? ti[j - 1] : (gt[j] ? e : ti[j]);
                }
                tk[0] = gt[0] ? xk : tk[0];
                ti[0] = gt[0] ? e : ti[0];
            }
        }
        if (live) {
            const int t = tb + lane;
            const float mx = topk_value(tk[0]);
            float p[K], sum = 0.f;
#pragma unroll
            for (int j = 0; j < K; ++j) {
                p[j] = expf(topk_value(tk[j]) - mx);
                sum += p[j];  // slot order
            }
            float wv[K];
#pragma unroll
            for (int j = 0; j < K; ++j) wv[j] = p[j] / sum;
            int32_t *irow = a.idx + static_cast<size_t>(t) * K;
            float *wrow = a.w + static_cast<size_t>(t) * K;
            if (vec_k) {
#pragma unroll
                for (int j = 0; j < K; j += 4) {
                    *reinterpret_cast<int4 *>(irow + j) = make_int4(ti[j], ti[j + 1], ti[j + 2], ti[j + 3]);
                    *reinterpret_cast<float4 *>(wrow + j) = make_float4(wv[j], wv[j + 1], wv[j + 2], wv[j + 3]);
                }
            } else {
#pragma unroll
                for (int j = 0; j < K; ++j) {
                    irow[j] = ti[j];
                    wrow[j] = wv[j];
                }
            }
#pragma unroll
            for (int j = 0; j < K; ++j) atomicAdd(&wcnt[warp * E + ti[j]], 1);
        }
        __syncwarp();
        if (it + S < nbatch) issue(it + S);
    }
    if (!wait_ok) {
        if (lane == 0) report_status(a.status, kStatusTimeout);
        for (int q = it; q < it + S && q < nbatch; ++q)  // copies still in flight land before the exit
            (void)mbar_wait(&bar[q % S], static_cast<uint32_t>(q / S) & 1u, nullptr);
    }
    __syncthreads();
    for (int e = threadIdx.x; e < E; e += blockDim.x) {
        int sum = 0;
        for (int q = 0; q < nw; ++q) sum += wcnt[q * E + e];
        a.blk_hist[static_cast<size_t>(b) * E + e] = sum;
    }
    if (!grid_barrier(a.barrier, G, a.status)) return;

    // ---- phase 2: per expert, exclusive scan over the blocks ----
    route_scan_experts(a, warp_sums);
    if (!grid_barrier(a.barrier, 2u * G, a.status)) return;

    // ---- phase 3: group starts, tile table, padding, positions ----
    if (!route_group_layout(a, gst, warp_sums)) return;
    route_warp_bases(a, wcnt, gst, nw);
    if (!wait_ok) return;  // this warp's idx rows are incomplete
    bool bad = false;
    const uint32_t below = (1u << lane) - 1u;
    int *run = wcnt + warp * E;
    uint32_t *msk = emask + warp * E;
    for (int tb = wt0; tb < wt1; tb += 32) {
        const int t = tb + lane;
        const bool live = t < wt1;
        int e[K];
        if (live) {
            const int32_t *irow = a.idx + static_cast<size_t>(t) * K;  // written by this thread in phase 1
            if (vec_k) {
#pragma unroll
                for (int j = 0; j < K; j += 4) {
                    const int4 v = *reinterpret_cast<const int4 *>(irow + j);
                    e[j] = v.x;
                    e[j + 1] = v.y;
                    e[j + 2] = v.z;
                    e[j + 3] = v.w;
                }
            } else {
#pragma unroll
                for (int j = 0; j < K; ++j) e[j] = irow[j];
            }
#pragma unroll
            for (int j = 0; j < K; ++j) atomicOr(&msk[e[j]], 1u << lane);
        }
        __syncwarp();
        if (live) {
#pragma unroll
            for (int j = 0; j < K; ++j) {
                const int pos = run[e[j]] + __popc(msk[e[j]] & below);
                const int pair = t * K + j;
                if (pos >= 0 && pos < gst[e[j] + 1]) {
                    a.perm[pos] = pair;
                    a.inv[pair] = pos;
                } else {
                    bad = true;
                }
            }
        }
        __syncwarp();
        if (live) {
#pragma unroll
            for (int j = 0; j < K; ++j) {
                const uint32_t mm = msk[e[j]];
                if (lane == 31 - __clz(mm)) {  // one lane per expert advances its position
                    run[e[j]] += __popc(mm);
                    msk[e[j]] = 0u;
                }
            }
        }
        __syncwarp();
    }
    if (bad) report_status(a.status, kStatusBadIndex);
}

// Warps and ring depth of the lane kernel, as many warps as fit in shared
// memory (at least E / 32, since phase 3 gives one expert to each thread).
// With at most 384 tokens per SM a warp has one or two batches, and a ring of
// two batches per warp (fewer, fuller warps) finishes first; with more tokens
// one batch per warp and twice the warps hide more latency (measured at E =
// 128: 16 K tokens 24.6 against 26.6 us, 512 K tokens 185 against 155 us).
struct LaneCfg {
    int warps, stages;
    size_t smem;
};

LaneCfg lane_cfg(int E, int T, int sms) {
    LaneCfg c{kLaneMaxWarps, static_cast<int64_t>(T) <= 384ll * sms ? 2 : 1, 0};
    while (c.warps > 1 && lane_smem_layout(E, c.warps, c.stages).total > kLaneSmemLimit) --c.warps;
    c.smem = lane_smem_layout(E, c.warps, c.stages).total;
    return c;
}

bool route_lane_ok(int E, int k, const float *logits) {
    return E <= kLaneMaxE && k >= 1 && k <= kLaneMaxK && E % (4 * k) == 0 &&
           (reinterpret_cast<uintptr_t>(logits) & 15u) == 0 && lane_cfg(E, 0, 1).warps * 32 >= E &&
           lane_cfg(E, 1 << 30, 1).warps * 32 >= E;
}

template <int NGM>
const void *route_lane_fn_k(int k) {
    switch (k) {
        case 1: return reinterpret_cast<const void *>(route_lane_kernel<1, NGM>);
        case 2: return reinterpret_cast<const void *>(route_lane_kernel<2, NGM>);
        case 3: return reinterpret_cast<const void *>(route_lane_kernel<3, NGM>);
        case 4: return reinterpret_cast<const void *>(route_lane_kernel<4, NGM>);
        case 5: return reinterpret_cast<const void *>(route_lane_kernel<5, NGM>);
        case 6: return reinterpret_cast<const void *>(route_lane_kernel<6, NGM>);
        case 7: return reinterpret_cast<const void *>(route_lane_kernel<7, NGM>);
        default: return reinterpret_cast<const void *>(route_lane_kernel<8, NGM>);
    }
}

const void *route_lane_fn(int E, int k) {
    return E % (8 * k) == 0 ? route_lane_fn_k<2>(k) : route_lane_fn_k<1>(k);
}

constexpr int kBwdThreads = 256;

// dscore[t, j] = the ordered sum of the dscore partials of pair (t, j)'s row,
// and dlogits through the renormalised softmax.  The row is inv[t, j] (the
// sorted layout); with compact_gs / compact_off (expert-parallel path) it is
// the pair's compact sorted index offsets[e] + inv[t, j] - group_start[e].
__global__ void __launch_bounds__(kBwdThreads) route_bwd_kernel(int T, int E, int k, const float *__restrict__ w,
                                                                const int32_t *__restrict__ idx,
                                                                const int32_t *__restrict__ inv,
                                                                const float *__restrict__ dpart, int dpart_stride,
                                                                float *__restrict__ dscore,
                                                                float *__restrict__ dlogits,
                                                                const int32_t *__restrict__ compact_gs,
                                                                const int32_t *__restrict__ compact_off) {
    __shared__ float s_ds[kBwdThreads / 32][kMaxTopK];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int t = blockIdx.x * (kBwdThreads / 32) + warp;
    if (t >= T) return;
    if (dlogits)
        for (int e = lane; e < E; e += 32) dlogits[static_cast<size_t>(t) * E + e] = 0.f;
    for (int j = lane; j < k; j += 32) {
        int pos = inv[static_cast<size_t>(t) * k + j];
        if (compact_gs != nullptr) {
            const int e = idx[static_cast<size_t>(t) * k + j];
            pos = e >= 0 && e < E ? compact_off[e] + pos - compact_gs[e] : 0;
        }
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

// Copies of x and grad_out in the expert-sorted layout (row pos holds the
// token of pair perm[pos]): both for the backward, x alone (g and gs null) for
// the forward's gate/up GEMM.  One warp per token: its k sorted rows (inv) are
// read once, each lane loads up to eight 16-byte pieces of the token's row(s)
// before storing them to all k rows, so the sources stream from HBM once and
// every store instruction writes 512 contiguous bytes of a sorted row.  With
// zero_pad a second loop zeroes the padding rows at the end of each expert's
// group (fewer than kTileM per expert): the wgrads sum over them, while the
// forward GEMM discards those rows' products.
constexpr int kSortPieces = 8;  // 16-byte pieces a lane holds at once, per source

__global__ void __launch_bounds__(256) sort_rows_kernel(const int32_t *__restrict__ inv,
                                                        const int32_t *__restrict__ counts,
                                                        const int32_t *__restrict__ group_start, int T, int E, int k,
                                                        int d, const __nv_bfloat16 *__restrict__ x,
                                                        const __nv_bfloat16 *__restrict__ g,
                                                        __nv_bfloat16 *__restrict__ xs, __nv_bfloat16 *__restrict__ gs,
                                                        bool zero_pad) {
    const int n16 = d / 8;  // 16-byte pieces per row
    const int rows_used = group_start[E];
    const int lane = threadIdx.x & 31;
    const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
    const int64_t tid = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    const uint4 *x4 = reinterpret_cast<const uint4 *>(x);
    const uint4 *g4 = reinterpret_cast<const uint4 *>(g);
    uint4 *xs4 = reinterpret_cast<uint4 *>(xs);
    uint4 *gs4 = reinterpret_cast<uint4 *>(gs);
    const int warps = static_cast<int>(stride >> 5);
    for (int t = static_cast<int>(tid >> 5); t < T; t += warps) {
        const int64_t src = static_cast<int64_t>(t) * n16;
        for (int p0 = 0; p0 < n16; p0 += 32 * kSortPieces) {
            uint4 xv[kSortPieces], gv[kSortPieces];
#pragma unroll
            for (int q = 0; q < kSortPieces; ++q) {
                const int piece = p0 + 32 * q + lane;
                if (piece < n16) {
                    xv[q] = __ldcs(x4 + src + piece);
                    if (g4 != nullptr) gv[q] = __ldcs(g4 + src + piece);
                }
            }
            for (int j0 = 0; j0 < k; j0 += 32) {
                const int pos_l = j0 + lane < k ? __ldg(inv + static_cast<int64_t>(t) * k + j0 + lane) : -1;
                const int nj = min(32, k - j0);
                for (int jj = 0; jj < nj; ++jj) {
                    const int pos = __shfl_sync(0xffffffffu, pos_l, jj);
                    if (pos < 0 || pos >= rows_used) continue;  // warp-uniform
                    const int64_t dst = static_cast<int64_t>(pos) * n16;
#pragma unroll
                    for (int q = 0; q < kSortPieces; ++q) {
                        const int piece = p0 + 32 * q + lane;
                        if (piece < n16) {
                            xs4[dst + piece] = xv[q];
                            if (gs4 != nullptr) gs4[dst + piece] = gv[q];
                        }
                    }
                }
            }
        }
    }
    if (!zero_pad) return;
    const uint4 zero = make_uint4(0u, 0u, 0u, 0u);
    const int64_t per_expert = static_cast<int64_t>(kTileM - 1) * n16;
    const int64_t pad_total = static_cast<int64_t>(E) * per_expert;
    for (int64_t i = tid; i < pad_total; i += stride) {
        const int e = static_cast<int>(i / per_expert);
        const int64_t rem = i - e * per_expert;
        const int r = static_cast<int>(rem / n16), piece = static_cast<int>(rem - static_cast<int64_t>(r) * n16);
        const int row = __ldg(group_start + e) + __ldg(counts + e) + r;
        if (row < __ldg(group_start + e + 1) && row < rows_used) {
            xs4[static_cast<int64_t>(row) * n16 + piece] = zero;
            if (gs4 != nullptr) gs4[static_cast<int64_t>(row) * n16 + piece] = zero;
        }
    }
}

// The combine and the dx scatter-sum: out[t] = sum over slots j = 0..k-1, in
// slot order, of the staged bf16 rows t*k + j, summed in fp32 and rounded to
// bf16 once.  One thread per 16-byte piece of a token's row (consecutive
// threads read consecutive pieces of the same row); the loads of eight slots
// are issued before any is added.  Reads each staged row once and streams it
// (evict-first): k*d*2 bytes in, d*2 out per token.
__global__ void __launch_bounds__(256) combine_rows_kernel(const __nv_bfloat16 *__restrict__ stage, int T, int k,
                                                           int d, __nv_bfloat16 *__restrict__ out) {
    const int n16 = d / 8;
    const int64_t total = static_cast<int64_t>(T) * n16;
    const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
    const uint4 *src = reinterpret_cast<const uint4 *>(stage);
    uint4 *dst = reinterpret_cast<uint4 *>(out);
    for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < total; i += stride) {
        const int64_t t = i / n16;
        const int64_t piece = i - t * n16;
        const uint4 *row0 = src + t * k * n16 + piece;
        float acc[8];
#pragma unroll
        for (int q = 0; q < 8; ++q) acc[q] = 0.f;
        for (int j0 = 0; j0 < k; j0 += 8) {
            uint4 v[8];
#pragma unroll
            for (int jj = 0; jj < 8; ++jj)
                if (j0 + jj < k) v[jj] = __ldcs(row0 + static_cast<int64_t>(j0 + jj) * n16);
#pragma unroll
            for (int jj = 0; jj < 8; ++jj) {
                if (j0 + jj < k) {  // slot order
                    const uint32_t w[4] = {v[jj].x, v[jj].y, v[jj].z, v[jj].w};
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        acc[2 * q] += bf16_lo(w[q]);
                        acc[2 * q + 1] += bf16_hi(w[q]);
                    }
                }
            }
        }
        dst[i] = make_uint4(pack_bf16x2(acc[0], acc[1]), pack_bf16x2(acc[2], acc[3]), pack_bf16x2(acc[4], acc[5]),
                            pack_bf16x2(acc[6], acc[7]));
    }
}

}  // namespace

cudaError_t launch_combine_rows(const __nv_bfloat16 *stage, int T, int k, int d, __nv_bfloat16 *out, int sms,
                                cudaStream_t s) {
    combine_rows_kernel<<<sms * 8, 256, 0, s>>>(stage, T, k, d, out);  // 8 x 256 threads per SM
    return cudaGetLastError();
}

cudaError_t launch_sort_rows(const int32_t *inv, const int32_t *counts, const int32_t *group_start, int E, int k,
                             int T, int d, const __nv_bfloat16 *x, const __nv_bfloat16 *g, __nv_bfloat16 *xs,
                             __nv_bfloat16 *gs, bool zero_pad, int sms, cudaStream_t s) {
    // 8 x 256 threads per SM
    sort_rows_kernel<<<sms * 8, 256, 0, s>>>(inv, counts, group_start, T, E, k, d, x, g, xs, gs, zero_pad);
    return cudaGetLastError();
}

cudaError_t launch_route_topk(const float *logits, int T, int E, int k, int32_t *idx, float *w,
                              int32_t *chunk_counts, cudaStream_t s) {
    const int blocks = (T + kRouteChunk - 1) / kRouteChunk;
    const int nv = (E + 31) / 32;
    if (nv <= 1)
        route_topk_kernel<1><<<blocks, kTopkThreads, 0, s>>>(logits, T, E, k, idx, w, chunk_counts);
    else if (nv <= 2)
        route_topk_kernel<2><<<blocks, kTopkThreads, 0, s>>>(logits, T, E, k, idx, w, chunk_counts);
    else if (nv <= 4)
        route_topk_kernel<4><<<blocks, kTopkThreads, 0, s>>>(logits, T, E, k, idx, w, chunk_counts);
    else if (nv <= 8)
        route_topk_kernel<8><<<blocks, kTopkThreads, 0, s>>>(logits, T, E, k, idx, w, chunk_counts);
    else
        route_topk_kernel<16><<<blocks, kTopkThreads, 0, s>>>(logits, T, E, k, idx, w, chunk_counts);
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
                             const float *dpart, int dpart_stride, float *dscore, float *dlogits, cudaStream_t s,
                             const int32_t *compact_gs, const int32_t *compact_off) {
    const int per_block = kBwdThreads / 32;
    const int blocks = (T + per_block - 1) / per_block;
    route_bwd_kernel<<<blocks, kBwdThreads, 0, s>>>(T, E, k, w, idx, inv, dpart, dpart_stride, dscore, dlogits,
                                                    compact_gs, compact_off);
    return cudaGetLastError();
}

int route_fused_grid(const float *logits, int T, int E, int k, int sms, int n_chunks) {
    int per_sm = 0;
    cudaError_t e;
    if (route_lane_ok(E, k, logits)) {
        const void *fn = route_lane_fn(E, k);
        const LaneCfg c = lane_cfg(E, T, sms);
        e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(c.smem));
        if (e == cudaSuccess) e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, fn, c.warps * 32, c.smem);
    } else {
        const int nv = (E + 31) / 32;
        const size_t smem = route_fused_smem(E, k);
        if (nv <= 1)
            e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, route_fused_kernel<1>, kFusedThreads, smem);
        else if (nv <= 2)
            e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, route_fused_kernel<2>, kFusedThreads, smem);
        else if (nv <= 4)
            e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, route_fused_kernel<4>, kFusedThreads, smem);
        else if (nv <= 8)
            e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, route_fused_kernel<8>, kFusedThreads, smem);
        else
            e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, route_fused_kernel<16>, kFusedThreads, smem);
    }
    if (e != cudaSuccess || per_sm < 1) return 0;
    const int g = per_sm * sms;
    return g < n_chunks ? g : n_chunks;
}

size_t route_fused_smem(int E, int k) {
    (void)k;
    return (static_cast<size_t>(kFusedWarps) * E + E + 1 + kFusedWarps) * 4;
}

cudaError_t launch_route_fused(const float *logits, int T, int E, int k, int32_t *idx, float *w, int32_t *blk_hist,
                               int32_t *blk_base, int32_t *counts, int32_t *offsets, int32_t *group_start,
                               int32_t *tile_expert, int32_t *perm, int32_t *inv, int64_t p_cap, unsigned *barrier, int *status, int sms, int grid, cudaStream_t s) {
    RouteFusedArgs a{logits, T, E, k, idx, w, blk_hist, blk_base, counts, offsets, group_start,
                     tile_expert, perm, inv, p_cap, barrier, status, 0};
    void *params[] = {&a};
    if (route_lane_ok(E, k, logits)) {
        const LaneCfg c = lane_cfg(E, T, sms);
        a.lane_stages = c.stages;
        return cudaLaunchCooperativeKernel(route_lane_fn(E, k), dim3(grid), dim3(c.warps * 32), params, c.smem, s);
    }
    const size_t smem = route_fused_smem(E, k);
    const int nv = (E + 31) / 32;
    const void *fn = nv <= 1   ? reinterpret_cast<const void *>(route_fused_kernel<1>)
                     : nv <= 2 ? reinterpret_cast<const void *>(route_fused_kernel<2>)
                     : nv <= 4 ? reinterpret_cast<const void *>(route_fused_kernel<4>)
                     : nv <= 8 ? reinterpret_cast<const void *>(route_fused_kernel<8>)
                               : reinterpret_cast<const void *>(route_fused_kernel<16>);
    return cudaLaunchCooperativeKernel(fn, dim3(grid), dim3(kFusedThreads), params, smem, s);
}

}  // namespace moe

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

// ---------------------------------------------------------------------------
// Fused routing: the three steps above in one cooperative launch.  Block b of
// G owns the contiguous tokens [T*b/G, T*(b+1)/G), and warp w of the block a
// contiguous sub-range of those, so (block, warp, token, slot) order is token
// order.  Phases, separated by grid barriers (every block resident: the launch
// is cooperative; every wait is bounded):
//   1  per token top-k, weights, combine counters; per-warp expert histograms;
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
    int32_t *cnt;
    int cnt_per_token;
    int64_t p_cap;
    unsigned *barrier;  // zero before the launch
    int *status;
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
        // (a fixed shuffle tree over the slots)
#pragma unroll
        for (int u = 0; u < kTokPar; ++u) {
            const int tt = t + u;
            const float m = topk_value(vmax[u]);
            float p[2], sum = 0.f;
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const int j = lane + 32 * h;
                p[h] = j < k ? expf(topk_value(static_cast<uint32_t>(sel[u][h] >> 32)) - m) : 0.f;
                sum += p[h];
            }
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, off);
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
                for (int cc = lane; cc < a.cnt_per_token; cc += 32)
                    a.cnt[static_cast<size_t>(tt) * a.cnt_per_token + cc] = 0;
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
// Fused routing, lane-per-token form, for E <= 128 with E a multiple of 4k and
// k <= 8.  Same phases and the same results as route_fused_kernel; phase 1 and
// the positions of phase 3 give each lane one token:
//   * a warp stages 32 consecutive tokens' logits in shared memory (cp.async;
//     rows padded by 4 words so that one-row-per-lane reads do not conflict),
//     and each lane turns its row into order keys in place;
//   * tau = the smallest of k group maxima (k disjoint groups of E/k values):
//     at least k values are >= tau, so every one of the k largest is; the lane
//     lists the positions of its values >= tau;
//   * the listed values go through a sorted insertion into k registers of
//     (value key, ~expert) -- larger value first, lower expert on ties -- which
//     leaves the k largest in slot order;
//   * weights as in route_fused_kernel, the sum taken in slot order.
// Positions: per batch of 32 tokens, each expert's set of lanes (a bitmask
// built with atomicOr) gives a pair's rank among the batch's earlier tokens;
// the highest of those lanes then advances the warp's running position.
// ---------------------------------------------------------------------------
constexpr int kLaneThreads = 256;
constexpr int kLaneWarps = kLaneThreads / 32;
constexpr int kLaneMaxE = 128;
constexpr int kLaneMaxK = 8;

__device__ __forceinline__ uint32_t order_key(float v) {
    const uint32_t u = __float_as_uint(v == 0.f ? 0.f : v);
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

template <int K>
__global__ void __launch_bounds__(kLaneThreads, 1) route_lane_kernel(const RouteFusedArgs a) {
    extern __shared__ __align__(16) uint32_t sm_u[];
    const int E = a.E, G = gridDim.x, b = blockIdx.x;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int stride = E + 4;                                   // words per staged row
    uint32_t *stage = sm_u + warp * 32 * stride;                // [32][stride] this warp's rows
    uint8_t *lists = reinterpret_cast<uint8_t *>(sm_u + kLaneWarps * 32 * stride) + warp * 32 * E;  // [32][E]
    int *wcnt = reinterpret_cast<int *>(sm_u + kLaneWarps * 32 * stride + kLaneWarps * 8 * E);     // [warps][E]
    uint32_t *emask = reinterpret_cast<uint32_t *>(wcnt + kLaneWarps * E);                         // [warps][E]
    int *gst = reinterpret_cast<int *>(emask + kLaneWarps * E);                                    // [E + 1]
    int *warp_sums = gst + E + 1;                                                                  // [warps]
    const int t0 = static_cast<int>(static_cast<int64_t>(a.T) * b / G);
    const int t1 = static_cast<int>(static_cast<int64_t>(a.T) * (b + 1) / G);
    const int nb = t1 - t0;
    const int wt0 = t0 + nb * warp / kLaneWarps, wt1 = t0 + nb * (warp + 1) / kLaneWarps;
    for (int i = threadIdx.x; i < kLaneWarps * E; i += kLaneThreads) {
        wcnt[i] = 0;
        emask[i] = 0u;
    }
    __syncthreads();

    // ---- phase 1: top-k, one token per lane ----
    const int P4 = E / 4, gsz = E / K;
    uint32_t *myrow = stage + lane * stride;
    uint8_t *mylist = lists + lane * E;
    if (lane == 0 && wt0 < wt1)
        prefetch_l2(a.logits + static_cast<size_t>(wt0) * E,
                    static_cast<uint32_t>(min(32, wt1 - wt0)) * static_cast<uint32_t>(E) * 4u);
    for (int tb = wt0; tb < wt1; tb += 32) {
        const int rows = min(32, wt1 - tb);
        const float *src = a.logits + static_cast<size_t>(tb) * E;
        for (int q = lane; q < rows * P4; q += 32) {
            const int r = q / P4, c4 = q - r * P4;
            cp_async_16(smem_u32(stage + r * stride + 4 * c4), src + static_cast<size_t>(r) * E + 4 * c4);
        }
        if (lane == 0 && tb + 32 < wt1)  // the next batch's rows on their way to L2
            prefetch_l2(src + static_cast<size_t>(32) * E,
                        static_cast<uint32_t>(min(32, wt1 - tb - 32)) * static_cast<uint32_t>(E) * 4u);
        cp_async_wait_all();
        __syncwarp();
        const bool live = lane < rows;
        int n = 0;
        if (live) {
            uint32_t tau = 0xFFFFFFFFu;
#pragma unroll 1
            for (int g = 0; g < K; ++g) {
                uint32_t gm = 0u;
                for (int i = g * gsz; i < (g + 1) * gsz; i += 4) {
                    const uint4 v = *reinterpret_cast<const uint4 *>(myrow + i);
                    const uint4 kk = make_uint4(order_key(__uint_as_float(v.x)), order_key(__uint_as_float(v.y)),
                                                order_key(__uint_as_float(v.z)), order_key(__uint_as_float(v.w)));
                    *reinterpret_cast<uint4 *>(myrow + i) = kk;
                    gm = max(gm, max(max(kk.x, kk.y), max(kk.z, kk.w)));
                }
                tau = min(tau, gm);
            }
            for (int i = 0; i < E; i += 4) {
                const uint4 kk = *reinterpret_cast<const uint4 *>(myrow + i);
                if (kk.x >= tau) mylist[n++] = static_cast<uint8_t>(i);
                if (kk.y >= tau) mylist[n++] = static_cast<uint8_t>(i + 1);
                if (kk.z >= tau) mylist[n++] = static_cast<uint8_t>(i + 2);
                if (kk.w >= tau) mylist[n++] = static_cast<uint8_t>(i + 3);
            }
        }
        uint64_t top[K];
#pragma unroll
        for (int j = 0; j < K; ++j) top[j] = 0ull;
        const int nmax = __reduce_max_sync(0xffffffffu, static_cast<unsigned>(n));
        for (int c = 0; c < nmax; ++c) {
            if (c < n) {
                const int i = mylist[c];
                const uint64_t x = (static_cast<uint64_t>(myrow[i]) << 32) | static_cast<uint32_t>(~i);
                if (x > top[K - 1]) {
#pragma unroll
                    for (int j = K - 1; j > 0; --j) top[j] = x > top[j - 1] ? top[j - 1] : (x > top[j] ? x : top[j]);
                    top[0] = x > top[0] ? x : top[0];
                }
            }
        }
        if (live) {
            const int t = tb + lane;
            const float m = topk_value(static_cast<uint32_t>(top[0] >> 32));
            float p[K], sum = 0.f;
            int e[K];
#pragma unroll
            for (int j = 0; j < K; ++j) {
                e[j] = static_cast<int>(~static_cast<uint32_t>(top[j]));
                p[j] = expf(topk_value(static_cast<uint32_t>(top[j] >> 32)) - m);
                sum += p[j];  // slot order
            }
            int32_t *irow = a.idx + static_cast<size_t>(t) * K;
            float *wrow = a.w + static_cast<size_t>(t) * K;
#pragma unroll
            for (int j = 0; j < K; ++j) {
                irow[j] = e[j];
                wrow[j] = p[j] / sum;
                atomicAdd(&wcnt[warp * E + e[j]], 1);
            }
            for (int cc = 0; cc < a.cnt_per_token; ++cc) a.cnt[static_cast<size_t>(t) * a.cnt_per_token + cc] = 0;
        }
        __syncwarp();
    }
    __syncthreads();
    for (int e = threadIdx.x; e < E; e += kLaneThreads) {
        int sum = 0;
        for (int q = 0; q < kLaneWarps; ++q) sum += wcnt[q * E + e];
        a.blk_hist[static_cast<size_t>(b) * E + e] = sum;
    }
    if (!grid_barrier(a.barrier, G, a.status)) return;

    // ---- phase 2: per expert, exclusive scan over the blocks ----
    route_scan_experts(a, warp_sums);
    if (!grid_barrier(a.barrier, 2u * G, a.status)) return;

    // ---- phase 3: group starts, tile table, padding, positions ----
    if (!route_group_layout(a, gst, warp_sums)) return;
    route_warp_bases(a, wcnt, gst, kLaneWarps);
    bool bad = false;
    const uint32_t below = (1u << lane) - 1u;
    int *run = wcnt + warp * E;
    uint32_t *msk = emask + warp * E;
    for (int tb = wt0; tb < wt1; tb += 32) {
        const int t = tb + lane;
        const bool live = t < wt1;
        int e[K];
#pragma unroll
        for (int j = 0; j < K; ++j) {
            e[j] = live ? a.idx[static_cast<size_t>(t) * K + j] : 0;  // written by this thread in phase 1
            if (live) atomicOr(&msk[e[j]], 1u << lane);
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

size_t route_lane_smem(int E) {
    return (static_cast<size_t>(kLaneWarps) * 32 * (E + 4) + static_cast<size_t>(kLaneWarps) * 8 * E +
            2 * static_cast<size_t>(kLaneWarps) * E + E + 1 + kLaneWarps) *
           4;
}

bool route_lane_ok(int E, int k) { return E <= kLaneMaxE && k <= kLaneMaxK && E % (4 * k) == 0; }

const void *route_lane_fn(int k) {
    switch (k) {
        case 1: return reinterpret_cast<const void *>(route_lane_kernel<1>);
        case 2: return reinterpret_cast<const void *>(route_lane_kernel<2>);
        case 3: return reinterpret_cast<const void *>(route_lane_kernel<3>);
        case 4: return reinterpret_cast<const void *>(route_lane_kernel<4>);
        case 5: return reinterpret_cast<const void *>(route_lane_kernel<5>);
        case 6: return reinterpret_cast<const void *>(route_lane_kernel<6>);
        case 7: return reinterpret_cast<const void *>(route_lane_kernel<7>);
        default: return reinterpret_cast<const void *>(route_lane_kernel<8>);
    }
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
// holds the token of pair perm[pos]; padding rows are zero).  Walked in token
// order: each 16-byte piece of a token's x and grad_out rows is read once and
// stored to the sorted rows of the token's k pairs (inv), so the sources stream
// from HBM once instead of once per pair.  A second loop zeroes the padding
// rows at the end of each expert's group (fewer than kTileM per expert).
__global__ void __launch_bounds__(256) sort_rows_kernel(const int32_t *__restrict__ inv,
                                                        const int32_t *__restrict__ counts,
                                                        const int32_t *__restrict__ group_start, int T, int E, int k,
                                                        int d, const __nv_bfloat16 *__restrict__ x,
                                                        const __nv_bfloat16 *__restrict__ g,
                                                        __nv_bfloat16 *__restrict__ xs, __nv_bfloat16 *__restrict__ gs) {
    const int n16 = d / 8;  // 16-byte pieces per row
    const int rows_used = group_start[E];
    const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
    const int64_t tid = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    const uint4 *x4 = reinterpret_cast<const uint4 *>(x);
    const uint4 *g4 = reinterpret_cast<const uint4 *>(g);
    uint4 *xs4 = reinterpret_cast<uint4 *>(xs);
    uint4 *gs4 = reinterpret_cast<uint4 *>(gs);
    const int64_t total = static_cast<int64_t>(T) * n16;
    for (int64_t i = tid; i < total; i += 2 * stride) {
        uint4 xv[2], gv[2];
#pragma unroll
        for (int u = 0; u < 2; ++u) {
            const int64_t ii = i + u * stride;
            if (ii < total) {
                xv[u] = __ldg(x4 + ii);
                gv[u] = __ldg(g4 + ii);
            }
        }
#pragma unroll
        for (int u = 0; u < 2; ++u) {
            const int64_t ii = i + u * stride;
            if (ii < total) {
                const int t = static_cast<int>(ii / n16), piece = static_cast<int>(ii - static_cast<int64_t>(t) * n16);
                for (int j = 0; j < k; ++j) {
                    const int pos = __ldg(inv + static_cast<int64_t>(t) * k + j);
                    if (pos >= 0 && pos < rows_used) {
                        xs4[static_cast<int64_t>(pos) * n16 + piece] = xv[u];
                        gs4[static_cast<int64_t>(pos) * n16 + piece] = gv[u];
                    }
                }
            }
        }
    }
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
            gs4[static_cast<int64_t>(row) * n16 + piece] = zero;
        }
    }
}

}  // namespace

cudaError_t launch_sort_rows(const int32_t *inv, const int32_t *counts, const int32_t *group_start, int E, int k,
                             int T, int d, const __nv_bfloat16 *x, const __nv_bfloat16 *g, __nv_bfloat16 *xs,
                             __nv_bfloat16 *gs, int sms, cudaStream_t s) {
    sort_rows_kernel<<<sms * 8, 256, 0, s>>>(inv, counts, group_start, T, E, k, d, x, g, xs, gs);  // 8 x 256 threads per SM
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

int route_fused_grid(int T, int E, int k, int sms, int n_chunks) {
    (void)T;
    int per_sm = 0;
    cudaError_t e;
    if (route_lane_ok(E, k)) {
        const void *fn = route_lane_fn(k);
        const size_t smem = route_lane_smem(E);
        e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
        if (e == cudaSuccess) e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, fn, kLaneThreads, smem);
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
                               int32_t *tile_expert, int32_t *perm, int32_t *inv, int32_t *cnt, int cnt_per_token,
                               int64_t p_cap, unsigned *barrier, int *status, int grid, cudaStream_t s) {
    RouteFusedArgs a{logits, T, E, k, idx, w, blk_hist, blk_base, counts, offsets, group_start,
                     tile_expert, perm, inv, cnt, cnt_per_token, p_cap, barrier, status};
    void *params[] = {&a};
    if (route_lane_ok(E, k))
        return cudaLaunchCooperativeKernel(route_lane_fn(k), dim3(grid), dim3(kLaneThreads), params,
                                           route_lane_smem(E), s);
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

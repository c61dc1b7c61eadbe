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
// The layer routes with one cooperative launch (route_fused, below: a form
// with four lanes per token and one grid barrier for E <= 128, a warp per token
// and two grid barriers otherwise).  The
// three-launch form right below serves moe_route_noalloc: (1) per token top-k +
// weights + a per-block expert histogram, (2) one block: totals, exclusive
// scans, per-block bases, tile table, padding, (3) per block: each thread owns
// one expert and walks the block's tokens in order, so positions inside an
// expert follow token order exactly.
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>

#include <mutex>
#include <vector>

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
        // taken in slot order (the same sum, bit for bit, as the quad form's)
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
// Fused routing, quad form: four lanes per token, for E <= 128 with E a
// multiple of 4, E >= 4k, k <= 8 and 16-byte aligned logits.  Same results as
// route_fused_kernel, with one grid barrier.  Block b of G owns the tokens
// [T*b/G, T*(b+1)/G), warp w of the block a contiguous sub-range of those.
//
// Phase 1: a warp takes 8 tokens at a time; lane q of a token holds the
// 16-byte pieces q, q+4, q+8, ... of the token's logit row in registers.
//   * tau, a lower bound on the k-th largest logit, is the k-th largest of the
//     E/4 piece maxima: k pieces have a maximum >= tau, so at least k logits
//     are >= tau and each of the k largest is.  Each lane sorts its piece
//     maxima; two butterfly steps merge the four lanes' lists (the k largest
//     of two lists A, B sorted descending are max(A_i, B_(k-1-i)), i < k).
//   * The logits >= tau (about 9 per token on Gaussian logits) are the
//     candidates: each lane appends its own, as 64-bit keys (order key of the
//     value, then ~expert), to the token's list in shared memory.
//   * A candidate's slot is its rank, the number of candidates with a larger
//     key, so the k largest land in slot order (value descending, lower expert
//     first on ties).  A token with more than kQuadCap candidates (many exact
//     ties) takes its k largest one per round instead: the four lanes compare
//     their best remaining keys and the winner leaves.
//   * Weights as in route_fused_kernel, the sum taken in slot order: each
//     lane computes its own slots' numerators and reads the others' back from
//     the token's slot array.  The block's expert histogram goes to
//     blk_hist[b].
// Grid barrier.
// Phase 2, in every block: each expert's total over all blocks and its sum
// over the blocks before b (all G histograms read from L2), the padded group
// starts (block 0 publishes counts, offsets and group starts), the tile table
// and padding rows of experts b, b+G, ...
// Phase 3: the block's tokens in chunks of one token per thread.  A pair's
// rank within its expert in the chunk comes from per-warp lane masks, counted
// and scanned over the warps by one thread per expert; the chunk's pairs are
// counting-sorted by expert in shared memory (pair and sorted position side
// by side) and written to perm one expert's run at a time (an expert's pairs
// of one chunk are consecutive in perm), so the stores are coalesced.
// ---------------------------------------------------------------------------
constexpr int kQuadThreads = 768;  // at most; see quad_cfg
constexpr int kQuadTok = 8;    // tokens per warp batch
constexpr int kQuadCap = 16;   // candidates per token ranked at once
constexpr int kQuadMaxE = 128;
constexpr int kQuadMaxK = 8;
constexpr size_t kQuadSmemLimit = 227u * 1024u;

// Byte offsets of the quad kernel's shared memory.  Phase 3 reuses the staged
// rows' area for buf .. call.
struct QuadSmem {
    size_t cand, sval, sidx, msk, woff, gst, wsum, total;
    size_t buf, gbuf, run, ccnt, pre, tot, call;
};

__host__ __device__ inline QuadSmem quad_smem_layout(int E, int warps) {
    QuadSmem L;
    const size_t rows = static_cast<size_t>(warps) * kQuadTok, threads = static_cast<size_t>(warps) * 32;
    const size_t parts = threads / static_cast<size_t>(E);
    size_t p3 = 0;
    L.buf = p3;                                  // [threads * kQuadMaxK] pair of each chunk-sorted slot
    p3 += threads * kQuadMaxK * 4;
    L.gbuf = p3;                                 // [threads * kQuadMaxK] its sorted position
    p3 += threads * kQuadMaxK * 4;
    L.run = p3;                                  // [E] next sorted position of each expert
    p3 += static_cast<size_t>(E) * 4;
    L.ccnt = p3;                                 // [E] the chunk's pairs per expert
    p3 += static_cast<size_t>(E) * 4;
    L.pre = p3;                                  // [parts][E] partial sums over earlier blocks
    p3 += parts * E * 4;
    L.tot = p3;                                  // [parts][E] partial sums over all blocks
    p3 += parts * E * 4;
    L.call = p3;                                 // [E] expert totals, then position offsets
    p3 += static_cast<size_t>(E) * 4;
    const size_t staged = rows * E * 4;          // phase 1: [warps][8][E] logits (candidates' values)
    L.cand = staged > p3 ? staged : p3;          // [warps][8][kQuadCap] candidate keys
    L.sval = L.cand + rows * kQuadCap * 8;       // [warps][8][kQuadMaxK] order keys by slot
    L.sidx = L.sval + rows * kQuadMaxK * 4;      // [warps][8][kQuadMaxK] experts by slot
    // [E][warps + 1]: the row stride warps + 1 puts both a warp's lanes (random
    // experts) and an expert's warps (one per lane) on distinct banks
    L.msk = L.sidx + rows * kQuadMaxK * 4;                          // lane masks
    L.woff = L.msk + static_cast<size_t>(E) * (warps + 1) * 4;      // phase 1 counts, phase 3 first ranks
    L.gst = L.woff + static_cast<size_t>(E) * (warps + 1) * 4;      // [E + 1] padded group starts
    L.wsum = L.gst + static_cast<size_t>(E + 4) * 4;          // [33] scan scratch
    L.total = L.wsum + 68 * 4;
    return L;
}

__device__ __forceinline__ uint32_t order_key(float v) {
    const uint32_t u = __float_as_uint(v == 0.f ? 0.f : v);
    return u ^ (static_cast<uint32_t>(static_cast<int32_t>(u) >> 31) | 0x80000000u);
}

__device__ __forceinline__ void cas_desc(float &a, float &b) {
    const float hi = fmaxf(a, b), lo = fminf(a, b);
    a = hi;
    b = lo;
}

// Sorts g descending with Batcher's odd-even merge sort (the network of the
// next power of two, comparators beyond N dropped).
template <int N>
__device__ __forceinline__ void sort_desc(float (&g)[N]) {
    constexpr int P = N <= 1 ? 1 : N <= 2 ? 2 : N <= 4 ? 4 : 8;
    static_assert(N <= 8, "up to 8 keys");
#pragma unroll
    for (int p = 1; p < P; p <<= 1) {
#pragma unroll
        for (int k = p; k >= 1; k >>= 1) {
#pragma unroll
            for (int j = k % p; j + k < P; j += 2 * k) {
#pragma unroll
                for (int i = 0; i < k; ++i) {
                    if (i + j + k < N && (i + j) / (2 * p) == (i + j + k) / (2 * p)) cas_desc(g[i + j], g[i + j + k]);
                }
            }
        }
    }
}

// Sorts a bitonic sequence descending (N a power of two), else any sequence.
template <int N>
__device__ __forceinline__ void sort_bitonic_desc(float (&c)[N]) {
    if constexpr ((N & (N - 1)) == 0) {
#pragma unroll
        for (int s = N / 2; s >= 1; s >>= 1) {
#pragma unroll
            for (int j = 0; j < N; ++j) {
                if ((j & s) == 0) cas_desc(c[j], c[j + s]);
            }
        }
    } else {
        sort_desc<N>(c);
    }
}

__device__ __forceinline__ uint64_t cand_key(float v, int e) {
    return (static_cast<uint64_t>(order_key(v)) << 32) | static_cast<uint32_t>(~e);
}

__device__ __forceinline__ int warp_incl_scan(int v) {
    const int lane = threadIdx.x & 31;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const int o = __shfl_up_sync(0xffffffffu, v, off);
        if (lane >= off) v += o;
    }
    return v;
}

// Exclusive scans of two ints per thread over the block: warp scans, then
// warp 0 scans the warps' totals.  tot gets the block totals; wsum holds 66
// ints.
__device__ __forceinline__ void block_scan2(int v0, int v1, int &x0, int &x1, int &tot0, int &tot1, int *wsum) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = static_cast<int>(blockDim.x >> 5);
    const int i0 = warp_incl_scan(v0), i1 = warp_incl_scan(v1);
    __syncthreads();  // wsum free from any earlier use
    if (lane == 31) {
        wsum[warp] = i0;
        wsum[33 + warp] = i1;
    }
    __syncthreads();
    if (warp == 0) {
        const int s0 = lane < nw ? wsum[lane] : 0, s1 = lane < nw ? wsum[33 + lane] : 0;
        const int si0 = warp_incl_scan(s0), si1 = warp_incl_scan(s1);
        if (lane < nw) {
            wsum[lane] = si0 - s0;
            wsum[33 + lane] = si1 - s1;
        }
        if (lane == 31) {
            wsum[32] = si0;
            wsum[65] = si1;
        }
    }
    __syncthreads();
    x0 = wsum[warp] + i0 - v0;
    x1 = wsum[33 + warp] + i1 - v1;
    tot0 = wsum[32];
    tot1 = wsum[65];
}

template <int K, int NV>
__global__ void __launch_bounds__(kQuadThreads, 1) route_quad_kernel(const RouteFusedArgs a) {
    extern __shared__ __align__(16) uint8_t sm_b[];
    constexpr int SPL = (K + 3) / 4;  // slots per lane
    constexpr unsigned kFull = 0xffffffffu;
    const int E = a.E, E4 = E / 4, G = gridDim.x, b = blockIdx.x;
    const int nw = static_cast<int>(blockDim.x >> 5);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, tq = lane >> 2, q = lane & 3;
    const QuadSmem L = quad_smem_layout(E, nw);
    const int row = warp * kQuadTok + tq;
    float *srow = reinterpret_cast<float *>(sm_b) + static_cast<size_t>(row) * E;
    uint64_t *cand = reinterpret_cast<uint64_t *>(sm_b + L.cand) + row * kQuadCap;
    uint32_t *sval = reinterpret_cast<uint32_t *>(sm_b + L.sval) + row * kQuadMaxK;
    int *sidx = reinterpret_cast<int *>(sm_b + L.sidx) + row * kQuadMaxK;
    const int ws = nw + 1;  // row stride of wcnt, msk and woff
    int *wcnt = reinterpret_cast<int *>(sm_b + L.woff);  // phase 1: [E][ws] per-warp expert counts
    int *gst = reinterpret_cast<int *>(sm_b + L.gst);
    int *wsum = reinterpret_cast<int *>(sm_b + L.wsum);
    const int t0 = static_cast<int>(static_cast<int64_t>(a.T) * b / G);
    const int t1 = static_cast<int>(static_cast<int64_t>(a.T) * (b + 1) / G);
    const int nb = t1 - t0;
    const int wt0 = t0 + nb * warp / nw, wt1 = t0 + nb * (warp + 1) / nw;
    for (int i = threadIdx.x; i < E * ws; i += blockDim.x) wcnt[i] = 0;
    __syncthreads();

    // ---- phase 1: top-k, four lanes per token ----
    for (int tb = wt0; tb < wt1; tb += kQuadTok) {
        const int t = tb + tq;
        const bool live = t < wt1;
        const float4 *src = reinterpret_cast<const float4 *>(a.logits) + static_cast<size_t>(live ? t : 0) * E4;
        float4 v[NV];
        float gm[NV];
#pragma unroll
        for (int i = 0; i < NV; ++i) {
            if (live && q + 4 * i < E4) {
                v[i] = __ldcs(src + q + 4 * i);
                gm[i] = fmaxf(fmaxf(v[i].x, v[i].y), fmaxf(v[i].z, v[i].w));
            } else {
                v[i] = make_float4(-INFINITY, -INFINITY, -INFINITY, -INFINITY);
                gm[i] = -INFINITY;
            }
        }
        // tau: the k-th largest piece maximum of the token's four lanes
        sort_desc<NV>(gm);
        float lst[K];
#pragma unroll
        for (int j = 0; j < K; ++j) lst[j] = j < NV ? gm[j] : -INFINITY;
        float mrg[K];
#pragma unroll
        for (int j = 0; j < K; ++j) mrg[j] = fmaxf(lst[j], __shfl_xor_sync(kFull, lst[K - 1 - j], 1));
        sort_bitonic_desc<K>(mrg);
        float tau = INFINITY;
#pragma unroll
        for (int j = 0; j < K; ++j) tau = fminf(tau, fmaxf(mrg[j], __shfl_xor_sync(kFull, mrg[K - 1 - j], 2)));
        // candidates: bit 4i + c of m is component c of piece q + 4i
        uint32_t m = 0u;
        if (live) {
#pragma unroll
            for (int i = 0; i < NV; ++i) {
                if (q + 4 * i >= E4) continue;
                uint32_t bits = 0u;
                if (v[i].x >= tau) bits |= 1u;
                if (v[i].y >= tau) bits |= 2u;
                if (v[i].z >= tau) bits |= 4u;
                if (v[i].w >= tau) bits |= 8u;
                m |= bits << (4 * i);
                if (bits != 0u) reinterpret_cast<float4 *>(srow)[q + 4 * i] = v[i];
            }
        }
        const int nc = __popc(m);
        int incl = nc;
        {
            const int u1 = __shfl_up_sync(kFull, incl, 1, 4);
            if (q >= 1) incl += u1;
            const int u2 = __shfl_up_sync(kFull, incl, 2, 4);
            if (q >= 2) incl += u2;
        }
        const int ncand = __shfl_sync(kFull, incl, 3, 4);
        const bool ranked = live && ncand <= kQuadCap;
        if (ranked) {
            int pos = incl - nc;
            for (uint32_t mm = m; mm != 0u; mm &= mm - 1u) {
                const int bit = __ffs(static_cast<int>(mm)) - 1;
                const int e = 16 * (bit >> 2) + 4 * q + (bit & 3);
                cand[pos++] = cand_key(srow[e], e);
            }
        }
        __syncwarp();
        // ranks; a warp whose tokens all have at most 12 candidates skips the
        // fourth owned candidate's compares
        const bool few = __all_sync(kFull, !ranked || ncand <= 12);
        if (ranked) {
            uint64_t own[4];
            int rk[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                own[u] = q + 4 * u < ncand ? cand[q + 4 * u] : ~0ull;
                rk[u] = 0;
            }
            if (few) {
                for (int j = 0; j < ncand; ++j) {
                    const uint64_t kj = cand[j];
#pragma unroll
                    for (int u = 0; u < 3; ++u) rk[u] += kj > own[u] ? 1 : 0;
                }
            } else {
                for (int j = 0; j < ncand; ++j) {
                    const uint64_t kj = cand[j];
#pragma unroll
                    for (int u = 0; u < 4; ++u) rk[u] += kj > own[u] ? 1 : 0;
                }
            }
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                if (q + 4 * u < ncand && rk[u] < K) {
                    sval[rk[u]] = static_cast<uint32_t>(own[u] >> 32);
                    sidx[rk[u]] = static_cast<int>(~static_cast<uint32_t>(own[u]));
                }
            }
        }
        if (__any_sync(kFull, live && !ranked)) {
            // many ties: the k largest one per round
            const bool mine = live && !ranked;
            uint32_t rem = mine ? m : 0u;
#pragma unroll 1
            for (int s = 0; s < K; ++s) {
                uint64_t best = 0ull;
                for (uint32_t mm = rem; mm != 0u; mm &= mm - 1u) {
                    const int bit = __ffs(static_cast<int>(mm)) - 1;
                    const int e = 16 * (bit >> 2) + 4 * q + (bit & 3);
                    const uint64_t key = cand_key(srow[e], e);
                    best = key > best ? key : best;
                }
                uint64_t o = __shfl_xor_sync(kFull, best, 1);
                best = o > best ? o : best;
                o = __shfl_xor_sync(kFull, best, 2);
                best = o > best ? o : best;
                const int e = static_cast<int>(~static_cast<uint32_t>(best));
                if (mine) {
                    if (((e >> 2) & 3) == q) rem &= ~(1u << (4 * (e >> 4) + (e & 3)));
                    if (q == 0) {
                        sval[s] = static_cast<uint32_t>(best >> 32);
                        sidx[s] = e;
                    }
                }
            }
        }
        __syncwarp();
        // weights: each lane the numerators of its own slots, published in the
        // token's slot array so that every lane adds all k in slot order
        int ej[SPL];
        float pj[SPL];
        if (live) {
            const float mx = topk_value(sval[0]);
#pragma unroll
            for (int u = 0; u < SPL; ++u) {
                const int j = q * SPL + u;
                ej[u] = j < K ? sidx[j] : 0;
                pj[u] = j < K ? expf(topk_value(sval[j]) - mx) : 0.f;
            }
        }
        __syncwarp();
        if (live) {
#pragma unroll
            for (int u = 0; u < SPL; ++u)
                if (q * SPL + u < K) reinterpret_cast<float *>(sval)[q * SPL + u] = pj[u];
        }
        __syncwarp();
        if (live) {
            float sum = 0.f;
#pragma unroll
            for (int j = 0; j < K; ++j) sum += reinterpret_cast<const float *>(sval)[j];  // slot order
            float wj[SPL];
#pragma unroll
            for (int u = 0; u < SPL; ++u) wj[u] = pj[u] / sum;
            int32_t *irow = a.idx + static_cast<size_t>(t) * K + q * SPL;
            float *wrow = a.w + static_cast<size_t>(t) * K + q * SPL;
            if constexpr (SPL == 2 && K % 2 == 0) {
                if (q * SPL < K) {
                    *reinterpret_cast<int2 *>(irow) = make_int2(ej[0], ej[1]);
                    *reinterpret_cast<float2 *>(wrow) = make_float2(wj[0], wj[1]);
                }
            } else {
#pragma unroll
                for (int u = 0; u < SPL; ++u) {
                    if (q * SPL + u < K) {
                        irow[u] = ej[u];
                        wrow[u] = wj[u];
                    }
                }
            }
#pragma unroll
            for (int u = 0; u < SPL; ++u)
                if (q * SPL + u < K) atomicAdd(&wcnt[ej[u] * ws + warp], 1);
        }
        __syncwarp();
    }
    __syncthreads();
    for (int x = threadIdx.x; x < E; x += blockDim.x) {
        int c = 0;
        for (int w = 0; w < nw; ++w) c += wcnt[x * ws + w];
        a.blk_hist[static_cast<size_t>(b) * E + x] = c;
    }
    if (!grid_barrier(a.barrier, G, a.status)) return;

    // ---- phase 2: totals, earlier blocks' sums, group layout ----
    int *run = reinterpret_cast<int *>(sm_b + L.run);
    int *ccnt = reinterpret_cast<int *>(sm_b + L.ccnt);
    int *call = reinterpret_cast<int *>(sm_b + L.call);
    {
        int *pre = reinterpret_cast<int *>(sm_b + L.pre);
        int *tot = reinterpret_cast<int *>(sm_b + L.tot);
        const int parts = static_cast<int>(blockDim.x) / E;  // >= 1
        const int x = threadIdx.x % E, p = threadIdx.x / E;
        if (p < parts) {
            // all of this thread's loads in flight at once (G <= 40 * parts in one round)
            int sp = 0, st = 0;
            for (int b0 = p; b0 < G; b0 += 40 * parts) {
                int v[40];
#pragma unroll
                for (int i = 0; i < 40; ++i) {
                    const int bb = b0 + i * parts;
                    v[i] = bb < G ? __ldcg(a.blk_hist + static_cast<size_t>(bb) * E + x) : 0;
                }
#pragma unroll
                for (int i = 0; i < 40; ++i) {
                    st += v[i];
                    sp += b0 + i * parts < b ? v[i] : 0;
                }
            }
            pre[p * E + x] = sp;
            tot[p * E + x] = st;
        }
        __syncthreads();
        int c = 0, before = 0;
        if (threadIdx.x < E) {
            for (int pp = 0; pp < parts; ++pp) {
                c += tot[pp * E + threadIdx.x];
                before += pre[pp * E + threadIdx.x];
            }
        }
        const int padded = (c + kTileM - 1) / kTileM * kTileM;
        int c_excl, p_excl, c_tot, p_tot;
        block_scan2(c, padded, c_excl, p_excl, c_tot, p_tot, wsum);
        if (threadIdx.x < E) {
            gst[threadIdx.x] = p_excl;
            run[threadIdx.x] = p_excl + before;
            call[threadIdx.x] = c;
            if (b == 0) {
                a.counts[threadIdx.x] = c;
                a.group_start[threadIdx.x] = p_excl;
                a.offsets[threadIdx.x] = c_excl;
            }
        }
        if (threadIdx.x == 0) {
            gst[E] = p_tot;
            if (b == 0) {
                a.group_start[E] = p_tot;
                a.offsets[E] = c_tot;
                if (p_tot > a.p_cap) report_status(a.status, kStatusBadIndex);
            }
        }
        __syncthreads();
        if (gst[E] > a.p_cap) return;
        for (int xx = b; xx < E; xx += G) {
            const int gs = gst[xx], ge = gst[xx + 1], cx = call[xx];
            for (int mt = gs / kTileM + threadIdx.x; mt < ge / kTileM; mt += blockDim.x) a.tile_expert[mt] = xx;
            for (int qq = gs + cx + threadIdx.x; qq < ge; qq += blockDim.x) a.perm[qq] = -1;
        }
    }

    // ---- phase 3: positions, one chunk of blockDim.x tokens at a time ----
    uint32_t *msk = reinterpret_cast<uint32_t *>(sm_b + L.msk);
    int *woff = reinterpret_cast<int *>(sm_b + L.woff);
    int *buf = reinterpret_cast<int *>(sm_b + L.buf);
    int *gbuf = reinterpret_cast<int *>(sm_b + L.gbuf);
    int *dlt = call;  // sorted position minus chunk-local slot, per expert
    const bool vec_k = (K % 4 == 0) && ((reinterpret_cast<uintptr_t>(a.idx) | reinterpret_cast<uintptr_t>(a.inv)) & 15u) == 0;
    const uint32_t below = (1u << lane) - 1u;
    // the experts of token t (written in phase 1, before the barrier)
    auto load_row = [&](int t, int (&e)[K]) {
        const int32_t *irow = a.idx + static_cast<size_t>(t) * K;
        if (vec_k) {
#pragma unroll
            for (int j = 0; j < K; j += 4) {
                const int4 v4 = __ldcg(reinterpret_cast<const int4 *>(irow + j));
                e[j] = v4.x;
                e[j + 1] = v4.y;
                e[j + 2] = v4.z;
                e[j + 3] = v4.w;
            }
        } else {
#pragma unroll
            for (int j = 0; j < K; ++j) e[j] = __ldcg(irow + j);
        }
    };
    for (int i = threadIdx.x; i < E * ws; i += blockDim.x) msk[i] = 0u;
    bool bad = false;
    int e[K];
    if (t0 + static_cast<int>(threadIdx.x) < t1) load_row(t0 + static_cast<int>(threadIdx.x), e);
    __syncthreads();
    for (int c0 = t0; c0 < t1; c0 += static_cast<int>(blockDim.x)) {
        const int t = c0 + static_cast<int>(threadIdx.x);
        const bool live = t < t1;
        if (live) {
#pragma unroll
            for (int j = 0; j < K; ++j) {
                if (e[j] < 0 || e[j] >= E) {  // cannot happen for finite logits; keeps the indexing in bounds
                    e[j] = 0;
                    bad = true;
                }
                atomicOr(&msk[e[j] * ws + warp], 1u << lane);
            }
        }
        __syncthreads();
        // the next chunk's rows in flight while this one is placed
        int en[K] = {};
        const int tn = t + static_cast<int>(blockDim.x);
        if (tn < t1) load_row(tn, en);
        // expert x (thread x): its pairs per warp, counted and scanned over the warps;
        // then the chunk-local starts, an exclusive scan over the experts
        int xt = 0;
        if (static_cast<int>(threadIdx.x) < E) {
            const uint32_t *mx = msk + threadIdx.x * ws;
            for (int w = 0; w < nw; ++w) xt += __popc(mx[w]);
        }
        const int xi = warp_incl_scan(xt);  // warps 0 .. E/32 - 1 hold the experts
        if (lane == 31 && warp < (E + 31) / 32) wsum[warp] = xi;
        __syncthreads();
        if (static_cast<int>(threadIdx.x) < E) {
            const int x = threadIdx.x;
            int base = xi - xt;
            for (int w = 0; w < warp; ++w) base += wsum[w];
            ccnt[x] = xt;
            dlt[x] = run[x] - base;
            const uint32_t *mx = msk + x * ws;
            int *wo = woff + x * ws;
            for (int w = 0; w < nw; ++w) {
                wo[w] = base;
                base += __popc(mx[w]);
            }
        }
        __syncthreads();
        if (live) {
            int pos[K];
#pragma unroll
            for (int j = 0; j < K; ++j) {
                const int x = e[j];
                const int lp = woff[x * ws + warp] + __popc(msk[x * ws + warp] & below);
                pos[j] = lp + dlt[x];
                buf[lp] = t * K + j;
                gbuf[lp] = pos[j];
            }
            int32_t *vrow = a.inv + static_cast<size_t>(t) * K;
            if (vec_k) {
#pragma unroll
                for (int j = 0; j < K; j += 4)
                    *reinterpret_cast<int4 *>(vrow + j) = make_int4(pos[j], pos[j + 1], pos[j + 2], pos[j + 3]);
            } else {
#pragma unroll
                for (int j = 0; j < K; ++j) vrow[j] = pos[j];
            }
        }
        __syncthreads();
        const int np = min(t1 - c0, static_cast<int>(blockDim.x)) * K;  // the chunk's pairs
        const int prows = gst[E];
        for (int i = threadIdx.x; i < np; i += blockDim.x) {
            const int p = gbuf[i];  // consecutive i of one expert: consecutive p
            if (p >= 0 && p < prows)
                a.perm[p] = buf[i];
            else
                bad = true;
        }
        __syncthreads();
        for (int x = threadIdx.x; x < E; x += blockDim.x) run[x] += ccnt[x];
        for (int i = threadIdx.x; i < E * ws; i += blockDim.x) msk[i] = 0u;
#pragma unroll
        for (int j = 0; j < K; ++j) e[j] = en[j];
        __syncthreads();
    }
    if (bad) report_status(a.status, kStatusBadIndex);
}

// Warps of the quad kernel: 16 while an SM has at most 1024 tokens, else 24
// (measured at E = 128, k = 8 against 16, 24 and 32 warps: 16 K tokens 22.5,
// 24.5 and 26.6 us; 1 M tokens 266, 231 and 244 us); fewer if shared memory
// runs out, at least E / 32 (phase 2 gives one expert to each thread).
struct QuadCfg {
    int warps;
    size_t smem;
};

QuadCfg quad_cfg(int E, int T, int sms) {
    QuadCfg c{static_cast<int64_t>(T) <= 1024ll * sms ? 16 : kQuadThreads / 32, 0};
    while (c.warps > 1 && quad_smem_layout(E, c.warps).total > kQuadSmemLimit) --c.warps;
    c.smem = quad_smem_layout(E, c.warps).total;
    return c;
}

bool route_quad_ok(int E, int k, const float *logits) {
    return E <= kQuadMaxE && E % 4 == 0 && k >= 1 && k <= kQuadMaxK && E >= 4 * k &&
           (reinterpret_cast<uintptr_t>(logits) & 15u) == 0 && quad_cfg(E, 0, 1).warps * 32 >= E &&
           quad_cfg(E, 1 << 30, 1).warps * 32 >= E;
}

template <int NV>
const void *route_quad_fn_k(int k) {
    switch (k) {
        case 1: return reinterpret_cast<const void *>(route_quad_kernel<1, NV>);
        case 2: return reinterpret_cast<const void *>(route_quad_kernel<2, NV>);
        case 3: return reinterpret_cast<const void *>(route_quad_kernel<3, NV>);
        case 4: return reinterpret_cast<const void *>(route_quad_kernel<4, NV>);
        case 5: return reinterpret_cast<const void *>(route_quad_kernel<5, NV>);
        case 6: return reinterpret_cast<const void *>(route_quad_kernel<6, NV>);
        case 7: return reinterpret_cast<const void *>(route_quad_kernel<7, NV>);
        default: return reinterpret_cast<const void *>(route_quad_kernel<8, NV>);
    }
}

// NV: 16-byte pieces a lane holds, E/16 rounded up to a power of two.
const void *route_quad_fn(int E, int k) {
    return E <= 32 ? route_quad_fn_k<2>(k) : E <= 64 ? route_quad_fn_k<4>(k) : route_quad_fn_k<8>(k);
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

// Resident blocks per SM of a routing kernel at (threads, dynamic shared
// memory), with the kernel's shared-memory opt-in set; looked up once per
// device and configuration (0 on failure, which is not kept).
int routing_blocks_per_sm(const void *fn, int threads, size_t smem) {
    struct Entry {
        int dev;
        const void *fn;
        int threads;
        size_t smem;
        int per_sm;
    };
    static std::mutex mu;
    static std::vector<Entry> cache;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 0;
    {
        std::lock_guard<std::mutex> g(mu);
        for (const Entry &c : cache)
            if (c.dev == dev && c.fn == fn && c.threads == threads && c.smem == smem) return c.per_sm;
    }
    int per_sm = 0;
    if (cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem)) != cudaSuccess ||
        cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, fn, threads, smem) != cudaSuccess || per_sm < 1)
        return 0;
    std::lock_guard<std::mutex> g(mu);
    cache.push_back(Entry{dev, fn, threads, smem, per_sm});
    return per_sm;
}

int route_fused_grid(const float *logits, int T, int E, int k, int sms, int n_chunks) {
    int per_sm = 0;
    if (route_quad_ok(E, k, logits)) {
        const QuadCfg c = quad_cfg(E, T, sms);
        per_sm = routing_blocks_per_sm(route_quad_fn(E, k), c.warps * 32, c.smem);
    } else {
        const int nv = (E + 31) / 32;
        const void *fn = nv <= 1   ? reinterpret_cast<const void *>(route_fused_kernel<1>)
                         : nv <= 2 ? reinterpret_cast<const void *>(route_fused_kernel<2>)
                         : nv <= 4 ? reinterpret_cast<const void *>(route_fused_kernel<4>)
                         : nv <= 8 ? reinterpret_cast<const void *>(route_fused_kernel<8>)
                                   : reinterpret_cast<const void *>(route_fused_kernel<16>);
        per_sm = routing_blocks_per_sm(fn, kFusedThreads, route_fused_smem(E, k));
    }
    if (per_sm < 1) return 0;
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
                     tile_expert, perm, inv, p_cap, barrier, status};
    void *params[] = {&a};
    if (route_quad_ok(E, k, logits)) {
        const QuadCfg c = quad_cfg(E, T, sms);
        return cudaLaunchCooperativeKernel(route_quad_fn(E, k), dim3(grid), dim3(c.warps * 32), params, c.smem, s);
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

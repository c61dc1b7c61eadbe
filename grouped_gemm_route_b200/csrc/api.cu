// Host side of libmoe.so: argument validation, workspace layout, TMA tensor
// maps, the launch sequence of the forward and backward passes, the status
// word and optional per-kernel event timing.  The C ABI is declared in
// include/moe.h.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>
#include <stdint.h>
#include <string.h>

#include <cmath>
#include <functional>
#include <mutex>
#include <vector>

#include "moe.h"
#include "moe_internal.h"

using namespace moe;

namespace {

constexpr size_t kAlign = 256;

size_t align_up(size_t v) { return (v + kAlign - 1) / kAlign * kAlign; }

struct Plan {
    int64_t T;
    int d, E, k, I;
    int64_t P;          // T*k pairs
    int64_t p_cap;      // sorted-layout row capacity
    int64_t m_tiles;    // p_cap / 128
    int n_chunks;       // routing blocks
    int bn_d;           // N tile of the GEMMs whose N is d
    int bn_i;           // N tile of the GEMMs whose N is I
    int dpart_stride;   // 2 I / bn_i: dscore partials per sorted row, one per column half-tile
    float limit;        // clamped SwiGLU limit, +inf for the plain SwiGLU
    // workspace layout (byte offsets)
    size_t ws_status, ws_stage, ws_chunk_counts, ws_chunk_base, fwd_bytes;
    size_t ws_dh, ws_dpart, ws_xs, ws_gs, bwd_bytes;
    // MXFP8 operands: E4M3 codes and their scale atoms (forward, then backward)
    bool mx;      // forward GEMMs on MXFP8 operands
    bool mx_bwd;  // backward GEMMs on MXFP8 operands
    size_t mx_x8, mx_xsf, mx_wgu8, mx_wgusf, mx_wd8, mx_wdsf, mx_aw8, mx_awsf;
    size_t mx_gs8, mx_gssf, mx_wdt8, mx_wdtsf, mx_gsc8, mx_gscsf, mx_awc8, mx_awcsf, mx_wgut8, mx_wgutsf, mx_dh8,
        mx_dhsf, mx_dhc8, mx_dhcsf, mx_xsc8, mx_xscsf;
    size_t saved[MOE_SAVED_FIELDS];
};

int make_plan(const moe_shape_t *s, Plan *p) {
    if (!s) return MOE_ERR_ARG;
    if (s->T < 1 || s->E < 1 || s->k < 1 || s->k > s->E || s->d < 1 || s->I < 1 || s->max_sms < 0)
        return MOE_ERR_ARG;
    if (s->E > kMaxExperts || s->k > kMaxTopK) return MOE_ERR_SHAPE;
    if (s->d % 128 != 0 || s->I % 128 != 0) return MOE_ERR_SHAPE;
    if (s->dtype != MOE_BF16 && s->dtype != MOE_MXFP8 && s->dtype != MOE_MXFP8_FWD) return MOE_ERR_ARG;
    if (!(s->swiglu_limit >= 0.f) || std::isinf(s->swiglu_limit)) return MOE_ERR_ARG;  // NaN fails the first test
    // Element offsets inside the kernels are 32-bit: P_cap * max(d, 2I) < 2^31.
    // T is bounded first so that no product below can overflow 64 bits.
    constexpr int64_t kIndexLimit = int64_t(1) << 31;
    if (s->T >= kIndexLimit) return MOE_ERR_SHAPE;
    const int64_t P = s->T * s->k;
    const int64_t widest = s->d > 2 * static_cast<int64_t>(s->I) ? s->d : 2 * static_cast<int64_t>(s->I);
    const int64_t nonempty = s->E < P ? s->E : P;
    const int64_t p_cap = (P + 127 * nonempty + 127) / 128 * 128;
    if (p_cap >= (kIndexLimit + widest - 1) / widest) return MOE_ERR_SHAPE;  // p_cap * widest >= 2^31
    // weight rows (E*2I of W_gate_up, E*d of W_down) are 32-bit tensor-map coordinates
    if (static_cast<int64_t>(s->E) * widest >= kIndexLimit) return MOE_ERR_SHAPE;
    p->T = s->T;
    p->d = s->d;
    p->E = s->E;
    p->k = s->k;
    p->I = s->I;
    p->P = P;
    p->p_cap = p_cap;
    p->m_tiles = p_cap / 128;
    p->n_chunks = static_cast<int>((s->T + kRouteChunk - 1) / kRouteChunk);
    p->mx = s->dtype == MOE_MXFP8 || s->dtype == MOE_MXFP8_FWD;  // forward GEMMs on MXFP8 operands
    p->mx_bwd = s->dtype == MOE_MXFP8;                            // backward GEMMs too
    p->limit = s->swiglu_limit > 0.f ? s->swiglu_limit : INFINITY;  // +inf: no clamp, min / clamp are exact no-ops
    // N tiles of the bf16 GEMMs (the MXFP8 GEMMs use 128-wide tiles of their own)
    p->bn_d = !p->mx_bwd && s->d % 256 == 0 ? 256 : 128;
    p->bn_i = !p->mx_bwd && s->I % 256 == 0 ? 256 : 128;
    p->dpart_stride = 2 * s->I / p->bn_i;  // the down dgrad's two epilogue warps per row each write a partial
                                           // (the kernel's kSplit for that mode)

    size_t off = 0;
    p->ws_status = off;
    off = align_up(off + 16);
    p->ws_stage = off;  // combine staging [P, d]; before it, the bf16 forward's sorted x [p_cap, d]
    off = align_up(off + static_cast<size_t>(p_cap) * s->d * 2);
    const size_t common = off;
    p->ws_chunk_counts = off;  // routing: per-block expert histograms
    off = align_up(off + static_cast<size_t>(p->n_chunks) * s->E * 4);
    p->ws_chunk_base = off;    // and their per-expert exclusive scans over the blocks
    off = align_up(off + static_cast<size_t>(p->n_chunks) * s->E * 4);
    auto take = [&off](size_t bytes) {
        const size_t at = off;
        off = align_up(off + bytes);
        return at;
    };
    const size_t Td = static_cast<size_t>(s->T) * s->d, Pd = static_cast<size_t>(p_cap) * s->d;
    const size_t PI = static_cast<size_t>(p_cap) * s->I, P2I = 2 * PI;
    const size_t W2Id = static_cast<size_t>(s->E) * 2 * s->I * s->d, WdI = static_cast<size_t>(s->E) * s->d * s->I;
    if (p->mx) {  // one scale byte per 32 elements
        p->mx_x8 = take(Td);
        p->mx_xsf = take(Td / 32);
        p->mx_wgu8 = take(W2Id);
        p->mx_wgusf = take(W2Id / 32);
        p->mx_wd8 = take(WdI);
        p->mx_wdsf = take(WdI / 32);
        p->mx_aw8 = take(PI);
        p->mx_awsf = take(PI / 32);
    }
    p->fwd_bytes = off;
    off = common;
    p->ws_dh = off;
    off = align_up(off + static_cast<size_t>(p_cap) * 2 * s->I * 2);
    p->ws_dpart = off;
    off = align_up(off + static_cast<size_t>(p_cap) * p->dpart_stride * 4);
    p->ws_xs = off;
    off = align_up(off + static_cast<size_t>(p_cap) * s->d * 2);
    p->ws_gs = off;
    off = align_up(off + static_cast<size_t>(p_cap) * s->d * 2);
    if (p->mx_bwd) {
        p->mx_gs8 = take(Pd);
        p->mx_gssf = take(Pd / 32);
        p->mx_wdt8 = take(WdI);
        p->mx_wdtsf = take(WdI / 32);
        p->mx_gsc8 = take(Pd);
        p->mx_gscsf = take(Pd / 32);
        p->mx_awc8 = take(PI);
        p->mx_awcsf = take(PI / 32);
        p->mx_wgut8 = take(W2Id);
        p->mx_wgutsf = take(W2Id / 32);
        p->mx_dh8 = take(P2I);
        p->mx_dhsf = take(P2I / 32);
        p->mx_dhc8 = take(P2I);
        p->mx_dhcsf = take(P2I / 32);
        p->mx_xsc8 = take(Pd);
        p->mx_xscsf = take(Pd / 32);
    }
    p->bwd_bytes = off;

    const size_t Tk = static_cast<size_t>(P);
    p->saved[0] = Tk * 4;                                   // topk_idx
    p->saved[1] = Tk * 4;                                   // topk_w
    p->saved[2] = static_cast<size_t>(s->E) * 4;            // counts
    p->saved[3] = static_cast<size_t>(s->E + 1) * 4;        // offsets
    p->saved[4] = static_cast<size_t>(s->E + 1) * 4;        // group_start
    p->saved[5] = static_cast<size_t>(p->m_tiles) * 4;      // tile_expert
    p->saved[6] = static_cast<size_t>(p_cap) * 4;           // perm
    p->saved[7] = Tk * 4;                                   // inv
    p->saved[8] = static_cast<size_t>(p_cap) * 2 * s->I * 2;  // h
    p->saved[9] = static_cast<size_t>(p_cap) * s->I * 2;      // aw
    p->saved[10] = static_cast<size_t>(p_cap) * s->d * 2;     // xs (optional)
    return MOE_OK;
}

bool aligned16(const void *ptr) { return ptr && (reinterpret_cast<uintptr_t>(ptr) & 15u) == 0; }

// ---------------------------------------------------------------------------
// per-device properties
// ---------------------------------------------------------------------------
struct DeviceInfo {
    bool ok = false;
    int sms = 0;
    int major = 0, minor = 0;
};

std::mutex g_mu;
DeviceInfo g_dev[64];
PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;

int device_info(DeviceInfo *out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return MOE_ERR_LAUNCH;
    std::lock_guard<std::mutex> lock(g_mu);
    if (!g_dev[dev].ok) {
        DeviceInfo d;
        if (cudaDeviceGetAttribute(&d.sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&d.major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&d.minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess)
            return MOE_ERR_LAUNCH;
        d.ok = true;
        g_dev[dev] = d;
    }
    if (!g_encode) {
        void *fn = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &fn, 12000, cudaEnableDefault, &q) !=
                cudaSuccess ||
            q != cudaDriverEntryPointSuccess || !fn)
            return MOE_ERR_LAUNCH;
        g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
    }
    *out = g_dev[dev];
    if (out->major != 10 || out->minor != 0) return MOE_ERR_ARCH;
    return MOE_OK;
}

// 2-d bf16 tensor [rows, cols] (row-major), box = box_rows x 64 columns, 128-byte swizzle.
bool make_map(CUtensorMap *m, const void *base, int64_t rows, int64_t cols, uint32_t box_rows) {
    cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows)};
    cuuint64_t strides[1] = {static_cast<cuuint64_t>(cols) * 2};
    cuuint32_t box[2] = {64, box_rows};
    cuuint32_t estr[2] = {1, 1};
    const CUresult r = g_encode(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(base), dims, strides, box,
                                estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                                CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// 2-d bf16 tensor [rows, cols], box = box_rows rows x 32 columns (64-byte rows), 64-byte swizzle:
// the chunks of h the down dgrad's loader warp moves into its ring (128 rows), and the 32 x 32
// pieces of h and aw the gate/up forward's epilogue warps store.
bool make_map_h(CUtensorMap *m, const void *base, int64_t rows, int64_t cols, uint32_t box_rows = 128) {
    cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows)};
    cuuint64_t strides[1] = {static_cast<cuuint64_t>(cols) * 2};
    cuuint32_t box[2] = {32, box_rows};
    cuuint32_t estr[2] = {1, 1};
    const CUresult r = g_encode(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(base), dims, strides, box,
                                estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B,
                                CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// 2-d E4M3 tensor [rows, cols] (row-major bytes), box = box_rows x 128 columns, 128-byte swizzle.
bool make_map8(CUtensorMap *m, const void *base, int64_t rows, int64_t cols, uint32_t box_rows) {
    cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows)};
    cuuint64_t strides[1] = {static_cast<cuuint64_t>(cols)};
    cuuint32_t box[2] = {128, box_rows};
    cuuint32_t estr[2] = {1, 1};
    const CUresult r = g_encode(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void *>(base), dims, strides, box, estr,
                                CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                                CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// ---------------------------------------------------------------------------
// one extra stream per device, for bandwidth-bound work that runs beside a
// tensor-bound GEMM (with two events to fork from and join the caller's stream)
// ---------------------------------------------------------------------------
struct SideStream {
    cudaStream_t s = nullptr;
    cudaEvent_t fork = nullptr, join = nullptr;
    bool tried = false;
    std::mutex mu;  // an event's record and the wait on it stay together when host threads share the stream

    // `to` waits for everything issued so far on `from` (through event ev).
    bool link(cudaEvent_t ev, cudaStream_t from, cudaStream_t to) {
        std::lock_guard<std::mutex> lock(mu);
        return cudaEventRecord(ev, from) == cudaSuccess && cudaStreamWaitEvent(to, ev, 0) == cudaSuccess;
    }
};
SideStream g_side[64];

// The current device's side stream, created on first use; nullptr if it could
// not be created (the caller then runs everything on its own stream).
SideStream *side_stream() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
    std::lock_guard<std::mutex> lock(g_mu);
    SideStream &ss = g_side[dev];
    if (!ss.tried) {
        ss.tried = true;
        if (cudaStreamCreateWithFlags(&ss.s, cudaStreamNonBlocking) != cudaSuccess ||
            cudaEventCreateWithFlags(&ss.fork, cudaEventDisableTiming) != cudaSuccess ||
            cudaEventCreateWithFlags(&ss.join, cudaEventDisableTiming) != cudaSuccess)
            ss.s = nullptr;
    }
    return ss.s != nullptr && ss.fork != nullptr && ss.join != nullptr ? &ss : nullptr;
}

// ---------------------------------------------------------------------------
// per-kernel timing (host bookkeeping only)
// ---------------------------------------------------------------------------
struct Timing {
    bool on = false;
    struct Rec {
        int kind;
        cudaEvent_t a, b;
    };
    std::vector<Rec> recs;
    std::vector<cudaEvent_t> pool;
};
Timing g_tm;

cudaEvent_t take_event() {
    if (!g_tm.pool.empty()) {
        cudaEvent_t e = g_tm.pool.back();
        g_tm.pool.pop_back();
        return e;
    }
    cudaEvent_t e = nullptr;
    cudaEventCreate(&e);
    return e;
}

struct Launch {
    int kind;
    cudaStream_t s;
    cudaEvent_t a = nullptr, b = nullptr;
    Launch(int k, cudaStream_t st) : kind(k), s(st) {
        if (g_tm.on) {
            std::lock_guard<std::mutex> lock(g_mu);
            a = take_event();
            b = take_event();
            if (a) cudaEventRecord(a, s);
        }
    }
    int done(cudaError_t e) {
        if (a && b) {
            cudaEventRecord(b, s);
            std::lock_guard<std::mutex> lock(g_mu);
            g_tm.recs.push_back({kind, a, b});
        }
        return e == cudaSuccess ? MOE_OK : MOE_ERR_LAUNCH;
    }
};

const char *kKindNames[kNumKernelKinds] = {
    "route_topk",       "route_scan",       "route_perm",           "gemm_gateup_fwd",      "gemm_down_fwd_combine",
    "gemm_down_dgrad",  "gemm_down_wgrad",  "gemm_gateup_dgrad_scatter", "gemm_gateup_wgrad", "route_bwd",
    "sort_rows", "mx_quant", "route_fused", "sort_x", "combine", "ep_layout", "ep_rows"};

struct Saved {
    int32_t *idx;
    float *w;
    int32_t *counts, *offsets, *group_start, *tile_expert, *perm, *inv;
    __nv_bfloat16 *h, *aw;
};

int check_saved(const moe_saved_t *s) {
    if (!s) return MOE_ERR_ARG;
    const void *ptrs[MOE_SAVED_FIELDS - 1] = {s->topk_idx, s->topk_w, s->counts, s->offsets, s->group_start,
                                             s->tile_expert, s->perm, s->inv, s->h, s->aw};
    for (const void *q : ptrs)
        if (!aligned16(q)) return MOE_ERR_ARG;
    if (s->xs != nullptr && !aligned16(s->xs)) return MOE_ERR_ARG;  // optional
    return MOE_OK;
}

int grid_for(const moe_shape_t *s, const DeviceInfo &dev) {
    int g = dev.sms;
    if (s->max_sms > 0 && s->max_sms < g) g = s->max_sms;
    return g;
}

// Routing and dispatch in one cooperative launch.  The status word and the
// grid-barrier counter (the 16 bytes at ws_status) are zeroed by the caller.
int run_route(const moe_shape_t *shape, const Plan &pl, const DeviceInfo &dev, const float *logits,
              moe_saved_t *saved, uint8_t *ws, cudaStream_t st) {
    int *status = reinterpret_cast<int *>(ws + pl.ws_status);
    unsigned *barrier = reinterpret_cast<unsigned *>(ws + pl.ws_status + 8);
    int32_t *blk_hist = reinterpret_cast<int32_t *>(ws + pl.ws_chunk_counts);
    int32_t *blk_base = reinterpret_cast<int32_t *>(ws + pl.ws_chunk_base);
    (void)shape;
    const int grid = route_fused_grid(logits, static_cast<int>(pl.T), pl.E, pl.k, dev.sms, pl.n_chunks);
    if (grid < 1) return MOE_ERR_LAUNCH;
    Launch L(kKindRouteFused, st);
    return L.done(launch_route_fused(logits, static_cast<int>(pl.T), pl.E, pl.k, saved->topk_idx, saved->topk_w,
                                     blk_hist, blk_base, saved->counts, saved->offsets, saved->group_start,
                                     saved->tile_expert, saved->perm, saved->inv, pl.p_cap,
                                     barrier, status, dev.sms, grid, st));
}

// The slot-ordered sum of the k staged rows of every token (the combine after
// the down GEMM, the scatter into dx after the gate/up dgrad).
int run_combine(const Plan &pl, const DeviceInfo &dev, const uint8_t *ws, void *dst, cudaStream_t st) {
    Launch L(kKindCombine, st);
    return L.done(launch_combine_rows(reinterpret_cast<const __nv_bfloat16 *>(ws + pl.ws_stage),
                                      static_cast<int>(pl.T), pl.k, pl.d, static_cast<__nv_bfloat16 *>(dst), dev.sms,
                                      st));
}

GemmArgs base_args(const Plan &pl, const moe_saved_t *sv, uint8_t *ws) {
    GemmArgs a;
    memset(&a, 0, sizeof(a));
    a.T = static_cast<int>(pl.T);
    a.d = pl.d;
    a.E = pl.E;
    a.k = pl.k;
    a.I = pl.I;
    a.dpart_stride = pl.dpart_stride;
    a.limit = pl.limit;
    a.k_elems = pl.mx_bwd ? 128 : kTileK;  // wgrad K rows per stage (backward only)
    a.perm = sv->perm;
    a.group_start = sv->group_start;
    a.tile_expert = sv->tile_expert;
    a.topk_w = sv->topk_w;
    a.h = reinterpret_cast<__nv_bfloat16 *>(sv->h);
    a.aw = reinterpret_cast<__nv_bfloat16 *>(sv->aw);
    a.stage = reinterpret_cast<__nv_bfloat16 *>(ws + pl.ws_stage);
    a.status = reinterpret_cast<int *>(ws + pl.ws_status);
    return a;
}


// MXFP8 gate/up GEMM after routing: quantise x (per-row scale bytes, for the
// gather) and W_gate_up (atoms in the tile's gate/up row order), then the
// block-scaled GEMM, whose epilogue writes h, aw and aw's codes and scales.
int gateup_mx(const Plan &pl, const DeviceInfo &dev, const moe_shape_t *shape, const void *x, const void *w_gate_up,
              moe_saved_t *saved, uint8_t *w8, cudaStream_t st) {
    int rc;
    const int64_t EI2 = static_cast<int64_t>(pl.E) * 2 * pl.I;
    uint8_t *x8 = w8 + pl.mx_x8, *xsf = w8 + pl.mx_xsf, *wgu8 = w8 + pl.mx_wgu8, *wgusf = w8 + pl.mx_wgusf;
    uint8_t *aw8 = w8 + pl.mx_aw8, *awsf = w8 + pl.mx_awsf;
    {
        Launch L(kKindMxQuant, st);
        if ((rc = L.done(launch_mx_quant_rows(static_cast<const __nv_bfloat16 *>(x), pl.T, pl.d, x8, xsf,
                                              kMxSfRowBytes, pl.I, nullptr, dev.sms, st))))
            return rc;
    }
    {
        Launch L(kKindMxQuant, st);
        if ((rc = L.done(launch_mx_quant_rows(static_cast<const __nv_bfloat16 *>(w_gate_up), EI2, pl.d, wgu8, wgusf,
                                              kMxSfGateUp, pl.I, nullptr, dev.sms, st))))
            return rc;
    }
    CUtensorMap tm_wgu8;
    if (!make_map8(&tm_wgu8, wgu8, EI2, pl.d, 64)) return MOE_ERR_LAUNCH;
    GemmArgs a = base_args(pl, saved, w8);
    a.n_tiles = pl.I / 64;
    a.num_k_blocks = pl.d / 128;
    a.gsrc = x8;
    a.gsf = xsf;
    a.sfb = wgusf;
    a.mx_codes = aw8;
    a.mx_sf = awsf;
    Launch L(kKindGemmGateUpFwd, st);
    return L.done(launch_gemm(kGateUpFwd, 128, true, a, tm_wgu8, tm_wgu8, grid_for(shape, dev), st));
}

// MXFP8 down GEMM + combine: quantise W_down along I, then the block-scaled
// GEMM on aw's codes (written by the gate/up epilogue).
int down_mx(const Plan &pl, const DeviceInfo &dev, const moe_shape_t *shape, const void *w_down, void *out,
            moe_saved_t *saved, uint8_t *w8, cudaStream_t st) {
    int rc;
    const int64_t Ed = static_cast<int64_t>(pl.E) * pl.d;
    uint8_t *wd8 = w8 + pl.mx_wd8, *wdsf = w8 + pl.mx_wdsf, *aw8 = w8 + pl.mx_aw8, *awsf = w8 + pl.mx_awsf;
    {
        Launch L(kKindMxQuant, st);
        if ((rc = L.done(launch_mx_quant_rows(static_cast<const __nv_bfloat16 *>(w_down), Ed, pl.I, wd8, wdsf,
                                              kMxSfAtoms, pl.I, nullptr, dev.sms, st))))
            return rc;
    }
    CUtensorMap tm_aw8, tm_wd8;
    if (!make_map8(&tm_aw8, aw8, pl.p_cap, pl.I, 128) || !make_map8(&tm_wd8, wd8, Ed, pl.I, 128))
        return MOE_ERR_LAUNCH;
    GemmArgs a = base_args(pl, saved, w8);
    a.n_tiles = pl.d / 128;
    a.num_k_blocks = pl.I / 128;
    a.sfa = awsf;
    a.sfb = wdsf;
    {
        Launch L(kKindGemmDownFwd, st);
        const int rc = L.done(launch_gemm(kDownFwd, 128, true, a, tm_aw8, tm_wd8, grid_for(shape, dev), st));
        if (rc) return rc;
    }
    return run_combine(pl, dev, w8, out, st);
}

// The gate/up GEMM with its SwiGLU epilogue (h, aw into `saved`), for the
// routing already in `saved`: bf16 or MXFP8 operands.
// x in the expert-sorted layout, into saved->xs (padding rows zeroed, for the
// backward's gate/up wgrad) when the caller keeps it, else into the combine's
// staging space (unused until the down GEMM; padding rows left as they are).
int sort_x(const Plan &pl, const DeviceInfo &dev, const void *x, const moe_saved_t *saved, uint8_t *w8,
           cudaStream_t st, __nv_bfloat16 **dst) {
    *dst = saved->xs != nullptr ? static_cast<__nv_bfloat16 *>(saved->xs)
                                : reinterpret_cast<__nv_bfloat16 *>(w8 + pl.ws_stage);
    Launch L(kKindSortX, st);
    return L.done(launch_sort_rows(saved->inv, saved->counts, saved->group_start, pl.E, pl.k, static_cast<int>(pl.T),
                                   pl.d, static_cast<const __nv_bfloat16 *>(x), nullptr, *dst, nullptr,
                                   saved->xs != nullptr, dev.sms, st));
}

// The bf16 gate/up GEMM on CTA pairs over x already in the sorted layout.
int gateup_pair_sorted(const Plan &pl, const moe_shape_t *shape, const DeviceInfo &dev, const void *xs,
                       const void *w_gate_up, moe_saved_t *saved, uint8_t *w8, cudaStream_t st) {
    // the pair kernel loads W_gate_up in 64-row boxes (gate and up halves), and x in 128-row boxes
    // (64-row boxes for an expert's unpaired last tile); its epilogue stores h and aw by TMA
    CUtensorMap tm_wgu, tm_xs, tm_xs64, tm_h, tm_aw;
    if (!make_map(&tm_wgu, w_gate_up, static_cast<int64_t>(pl.E) * 2 * pl.I, pl.d, 64) ||
        !make_map(&tm_xs, xs, pl.p_cap, pl.d, 128) || !make_map(&tm_xs64, xs, pl.p_cap, pl.d, 64) ||
        !make_map_h(&tm_h, saved->h, pl.p_cap, 2 * pl.I, 32) || !make_map_h(&tm_aw, saved->aw, pl.p_cap, pl.I, 32))
        return MOE_ERR_LAUNCH;
    GemmArgs a = base_args(pl, saved, w8);
    a.n_tiles = pl.I / 128;
    a.num_k_blocks = pl.d / kTileK;
    Launch L(kKindGemmGateUpFwd, st);
    return L.done(launch_gemm_pair(kGateUpFwd, a, tm_xs, tm_wgu, grid_for(shape, dev), st, &tm_xs64, &tm_h, &tm_aw));
}

int gateup_fwd(const Plan &pl, const DeviceInfo &dev, const moe_shape_t *shape, const void *x, const void *w_gate_up,
               moe_saved_t *saved, uint8_t *w8, cudaStream_t st) {
    int rc;
    const int grid = grid_for(shape, dev);
    const bool pair = !pl.mx && gemm_pair_ok(kGateUpFwd, 256, false, 0, grid);
    __nv_bfloat16 *xs = nullptr;
    if (pair || saved->xs != nullptr)
        if ((rc = sort_x(pl, dev, x, saved, w8, st, &xs))) return rc;
    if (pl.mx) return gateup_mx(pl, dev, shape, x, w_gate_up, saved, w8, st);
    if (pair) return gateup_pair_sorted(pl, shape, dev, xs, w_gate_up, saved, w8, st);  // plain TMA tiles
    CUtensorMap tm_wgu;
    if (!make_map(&tm_wgu, w_gate_up, static_cast<int64_t>(pl.E) * 2 * pl.I, pl.d, 128)) return MOE_ERR_LAUNCH;
    GemmArgs a = base_args(pl, saved, w8);
    a.n_tiles = pl.I / 128;
    a.num_k_blocks = pl.d / kTileK;
    a.gsrc = static_cast<const __nv_bfloat16 *>(x);  // token rows gathered through perm (A operand)
    Launch L(kKindGemmGateUpFwd, st);
    return L.done(launch_gemm(kGateUpFwd, 256, false, a, tm_wgu, tm_wgu, grid, st));
}

// The bf16 down GEMM; its epilogue writes each valid sorted row's product to
// row perm[pos] of `stage` (NULL: the workspace's staging buffer).
int down_fwd_staged(const Plan &pl, const DeviceInfo &dev, const moe_shape_t *shape, const void *w_down,
                    const moe_saved_t *saved, uint8_t *w8, void *stage, cudaStream_t st) {
    const int grid = grid_for(shape, dev);
    // CTA pairs: each CTA loads 128 of the tile's 256 rows of W_down, and an expert's unpaired last
    // tile loads 64-row boxes of aw
    const bool pair = gemm_pair_ok(kDownFwd, pl.bn_d, false, 0, grid);
    CUtensorMap tm_aw, tm_aw64, tm_wd;
    if (!make_map(&tm_aw, saved->aw, pl.p_cap, pl.I, 128) || !make_map(&tm_aw64, saved->aw, pl.p_cap, pl.I, 64) ||
        !make_map(&tm_wd, w_down, static_cast<int64_t>(pl.E) * pl.d, pl.I, pair ? 128 : pl.bn_d))
        return MOE_ERR_LAUNCH;
    GemmArgs a = base_args(pl, saved, w8);
    if (stage != nullptr) a.stage = static_cast<__nv_bfloat16 *>(stage);
    a.n_tiles = pl.d / pl.bn_d;
    a.num_k_blocks = pl.I / kTileK;
    Launch L(kKindGemmDownFwd, st);
    return L.done(pair ? launch_gemm_pair(kDownFwd, a, tm_aw, tm_wd, grid, st, &tm_aw64)
                       : launch_gemm(kDownFwd, pl.bn_d, false, a, tm_aw, tm_wd, grid, st));
}

// MXFP8 backward after sort_rows: every GEMM operand quantised along that
// GEMM's K (grad_out and W_down along d for the down dgrad, dh and W_gate_up
// along 2I for the gate/up dgrad, both operands of each wgrad along the
// expert's sorted rows); the down-dgrad epilogue writes dh's codes along 2I.
int bwd_mx(const Plan &pl, const DeviceInfo &dev, const moe_shape_t *shape, const void *w_gate_up, const void *w_down,
           const moe_saved_t *saved, void *dx, void *dw_gate_up, void *dw_down, GemmArgs a,
           const __nv_bfloat16 *xs, const __nv_bfloat16 *gs, uint8_t *w8, cudaStream_t st) {
    int rc;
    const int64_t EI2 = static_cast<int64_t>(pl.E) * 2 * pl.I, Ed = static_cast<int64_t>(pl.E) * pl.d;
    const int32_t *used = saved->group_start + pl.E;  // sorted rows in use
    uint8_t *gs8 = w8 + pl.mx_gs8, *gssf = w8 + pl.mx_gssf, *wdt8 = w8 + pl.mx_wdt8, *wdtsf = w8 + pl.mx_wdtsf;
    uint8_t *gsc8 = w8 + pl.mx_gsc8, *gscsf = w8 + pl.mx_gscsf, *awc8 = w8 + pl.mx_awc8, *awcsf = w8 + pl.mx_awcsf;
    uint8_t *wgut8 = w8 + pl.mx_wgut8, *wgutsf = w8 + pl.mx_wgutsf, *dh8 = w8 + pl.mx_dh8, *dhsf = w8 + pl.mx_dhsf;
    uint8_t *dhc8 = w8 + pl.mx_dhc8, *dhcsf = w8 + pl.mx_dhcsf, *xsc8 = w8 + pl.mx_xsc8, *xscsf = w8 + pl.mx_xscsf;
    const __nv_bfloat16 *wd = static_cast<const __nv_bfloat16 *>(w_down);
    const __nv_bfloat16 *wgu = static_cast<const __nv_bfloat16 *>(w_gate_up);
    auto quant = [&](bool along_rows_of_src, const __nv_bfloat16 *src, int64_t rows, int cols, uint8_t *codes,
                     uint8_t *sf, const int32_t *rows_used) {
        Launch L(kKindMxQuant, st);
        return along_rows_of_src
                   ? L.done(launch_mx_quant_cols(src, rows, cols, codes, sf, rows_used, dev.sms, st))
                   : L.done(launch_mx_quant_rows(src, rows, cols, codes, sf, kMxSfAtoms, pl.I, rows_used, dev.sms, st));
    };
    CUtensorMap tm_gs8, tm_wdt8, tm_gsc8, tm_awc8, tm_dh8, tm_wgut8, tm_dhc8, tm_xsc8;
    if (!make_map8(&tm_gs8, gs8, pl.p_cap, pl.d, 128) || !make_map8(&tm_wdt8, wdt8, Ed, pl.I, 128) ||
        !make_map8(&tm_gsc8, gsc8, pl.p_cap, pl.d, 128) || !make_map8(&tm_awc8, awc8, pl.p_cap, pl.I, 128) ||
        !make_map8(&tm_dh8, dh8, pl.p_cap, 2 * pl.I, 128) || !make_map8(&tm_wgut8, wgut8, EI2, pl.d, 128) ||
        !make_map8(&tm_dhc8, dhc8, pl.p_cap, 2 * pl.I, 128) || !make_map8(&tm_xsc8, xsc8, pl.p_cap, pl.d, 128))
        return MOE_ERR_LAUNCH;
    const int grid = grid_for(shape, dev);
    // b1: down dgrad (K = d)
    if ((rc = quant(false, gs, pl.p_cap, pl.d, gs8, gssf, used))) return rc;
    if ((rc = quant(true, wd, Ed, pl.I, wdt8, wdtsf, nullptr))) return rc;
    a.n_tiles = pl.I / 128;
    a.num_k_blocks = pl.d / 128;
    a.sfa = gssf;
    a.sfb = wdtsf;
    a.mx_codes = dh8;
    a.mx_sf = dhsf;
    {
        Launch L(kKindGemmDownDgrad, st);
        if ((rc = L.done(launch_gemm(kDownDgrad, 128, true, a, tm_gs8, tm_wdt8, grid, st)))) return rc;
    }
    // b3: down wgrad (K = sorted rows)
    if ((rc = quant(true, gs, pl.p_cap, pl.d, gsc8, gscsf, used))) return rc;
    if ((rc = quant(true, reinterpret_cast<const __nv_bfloat16 *>(saved->aw), pl.p_cap, pl.I, awc8, awcsf, used)))
        return rc;
    a.m_tiles = pl.d / 128;
    a.n_tiles = pl.I / 128;
    a.dw = static_cast<__nv_bfloat16 *>(dw_down);
    a.sfa = gscsf;
    a.sfb = awcsf;
    {
        Launch L(kKindGemmDownWgrad, st);
        if ((rc = L.done(launch_gemm(kDownWgrad, 128, true, a, tm_gsc8, tm_awc8, grid, st)))) return rc;
    }
    // b4: gate/up dgrad + scatter (K = 2I)
    if ((rc = quant(true, wgu, EI2, pl.d, wgut8, wgutsf, nullptr))) return rc;
    a.n_tiles = pl.d / 128;
    a.num_k_blocks = 2 * pl.I / 128;
    a.sfa = dhsf;
    a.sfb = wgutsf;
    {
        Launch L(kKindGemmGateUpDgrad, st);
        if ((rc = L.done(launch_gemm(kGateUpDgrad, 128, true, a, tm_dh8, tm_wgut8, grid, st)))) return rc;
    }
    if ((rc = run_combine(pl, dev, w8, dx, st))) return rc;
    // b5: gate/up wgrad (K = sorted rows)
    if ((rc = quant(true, a.dh, pl.p_cap, 2 * pl.I, dhc8, dhcsf, used))) return rc;
    if ((rc = quant(true, xs, pl.p_cap, pl.d, xsc8, xscsf, used))) return rc;
    a.m_tiles = 2 * pl.I / 128;
    a.n_tiles = pl.d / 128;
    a.dw = static_cast<__nv_bfloat16 *>(dw_gate_up);
    a.sfa = dhcsf;
    a.sfb = xscsf;
    Launch L(kKindGemmGateUpWgrad, st);
    return L.done(launch_gemm(kGateUpWgrad, 128, true, a, tm_dhc8, tm_xsc8, grid, st));
}

// The four bf16 backward GEMMs on sorted grad_out (gs) and sorted x (xs), both
// with zero padding rows: b1 down dgrad (dscore partials, SwiGLU backward ->
// dh), b3 down wgrad, b4 gate/up dgrad (each valid sorted row's dx product to
// row perm[pos] of `stage`; NULL: the workspace's staging buffer), b5 gate/up
// wgrad.  `a` carries the routing state, dh and the dscore partials.
int bwd_gemms(const Plan &pl, const DeviceInfo &dev, int grid, GemmArgs a, const void *gs, const void *xs,
              const void *w_gate_up, const void *w_down, const moe_saved_t *saved, void *dw_gate_up, void *dw_down,
              void *stage, cudaStream_t st, const std::function<int()> &after_dgrad = nullptr) {
    (void)dev;
    int rc;
    CUtensorMap tm_wd_mn, tm_dh_rows, tm_wgu_mn, tm_aw_mn, tm_dh_mn, tm_gs_rows, tm_gs_mn, tm_xs_mn;
    const int64_t EI2 = static_cast<int64_t>(pl.E) * 2 * pl.I;
    const int64_t Ed = static_cast<int64_t>(pl.E) * pl.d;
    if (!make_map(&tm_wd_mn, w_down, Ed, pl.I, 64) || !make_map(&tm_dh_rows, a.dh, pl.p_cap, 2 * pl.I, 128) ||
        !make_map(&tm_wgu_mn, w_gate_up, EI2, pl.d, 64) || !make_map(&tm_aw_mn, saved->aw, pl.p_cap, pl.I, 64) ||
        !make_map(&tm_dh_mn, a.dh, pl.p_cap, 2 * pl.I, 64) || !make_map(&tm_gs_rows, gs, pl.p_cap, pl.d, 128) ||
        !make_map(&tm_gs_mn, gs, pl.p_cap, pl.d, 64) || !make_map(&tm_xs_mn, xs, pl.p_cap, pl.d, 64))
        return MOE_ERR_LAUNCH;
    if (stage != nullptr) a.stage = static_cast<__nv_bfloat16 *>(stage);
    // b1: down dgrad, dscore partials, SwiGLU backward -> dh (CTA pairs: h streamed into a ring by TMA)
    a.n_tiles = pl.I / pl.bn_i;
    a.num_k_blocks = pl.d / kTileK;
    {
        Launch L(kKindGemmDownDgrad, st);
        if (gemm_pair_ok(kDownDgrad, pl.bn_i, false, 0, grid)) {
            CUtensorMap tm_h;
            if (!make_map_h(&tm_h, saved->h, pl.p_cap, 2 * pl.I)) return MOE_ERR_LAUNCH;
            rc = L.done(launch_gemm_pair(kDownDgrad, a, tm_gs_rows, tm_wd_mn, grid, st, &tm_h));
        } else {
            rc = L.done(launch_gemm(kDownDgrad, pl.bn_i, false, a, tm_gs_rows, tm_wd_mn, grid, st));
        }
        if (rc) return rc;
    }
    // b3: down wgrad  dW_down[e] = sum_p gout[t] (x) aw_p
    a.m_tiles = pl.d / kTileM;
    a.n_tiles = pl.I / pl.bn_i;
    a.dw = static_cast<__nv_bfloat16 *>(dw_down);
    {
        Launch L(kKindGemmDownWgrad, st);
        if (gemm_pair_ok(kDownWgrad, pl.bn_i, false, a.m_tiles, grid)) {
            CUtensorMap tm_dw;  // the epilogue's TMA stores (32 x 64 boxes)
            if (!make_map(&tm_dw, dw_down, Ed, pl.I, 32)) return MOE_ERR_LAUNCH;
            rc = L.done(launch_gemm_pair(kDownWgrad, a, tm_gs_mn, tm_aw_mn, grid, st, &tm_dw));
        } else {
            rc = L.done(launch_gemm(kDownWgrad, pl.bn_i, false, a, tm_gs_mn, tm_aw_mn, grid, st));
        }
        if (rc) return rc;
    }
    // b4: gate/up dgrad, rows staged for the ordered scatter-sum into dx
    a.n_tiles = pl.d / pl.bn_d;
    a.num_k_blocks = 2 * pl.I / kTileK;
    {
        Launch L(kKindGemmGateUpDgrad, st);
        if ((rc = L.done(gemm_pair_ok(kGateUpDgrad, pl.bn_d, false, 0, grid)
                             ? launch_gemm_pair(kGateUpDgrad, a, tm_dh_rows, tm_wgu_mn, grid, st)
                             : launch_gemm(kGateUpDgrad, pl.bn_d, false, a, tm_dh_rows, tm_wgu_mn, grid, st))))
            return rc;
    }
    if (after_dgrad && (rc = after_dgrad())) return rc;  // work that may run beside the gate/up wgrad
    // b5: gate/up wgrad  dW_gu[e] = sum_p dh_p (x) x[t]
    a.m_tiles = 2 * pl.I / kTileM;
    a.n_tiles = pl.d / pl.bn_d;
    a.dw = static_cast<__nv_bfloat16 *>(dw_gate_up);
    Launch L(kKindGemmGateUpWgrad, st);
    if (gemm_pair_ok(kGateUpWgrad, pl.bn_d, false, a.m_tiles, grid)) {
        CUtensorMap tm_dw;
        if (!make_map(&tm_dw, dw_gate_up, EI2, pl.d, 32)) return MOE_ERR_LAUNCH;
        return L.done(launch_gemm_pair(kGateUpWgrad, a, tm_dh_mn, tm_xs_mn, grid, st, &tm_dw));
    }
    return L.done(launch_gemm(kGateUpWgrad, pl.bn_d, false, a, tm_dh_mn, tm_xs_mn, grid, st));
}

}  // namespace

extern "C" {

int moe_saved_sizes(const moe_shape_t *shape, size_t sizes[MOE_SAVED_FIELDS], int64_t *p_cap) {
    Plan pl;
    const int rc = make_plan(shape, &pl);
    if (rc) return rc;
    if (sizes)
        for (int i = 0; i < MOE_SAVED_FIELDS; ++i) sizes[i] = pl.saved[i];
    if (p_cap) *p_cap = pl.p_cap;
    return MOE_OK;
}

int moe_workspace_size(const moe_shape_t *shape, size_t *fwd_bytes, size_t *bwd_bytes) {
    Plan pl;
    const int rc = make_plan(shape, &pl);
    if (rc) return rc;
    if (fwd_bytes) *fwd_bytes = pl.fwd_bytes;
    if (bwd_bytes) *bwd_bytes = pl.bwd_bytes;
    return MOE_OK;
}

int moe_route(const moe_shape_t *shape, const float *logits, moe_saved_t *saved, void *ws, size_t ws_bytes,
              void *stream) {
    Plan pl;
    int rc = make_plan(shape, &pl);
    if (rc) return rc;
    if (!aligned16(logits) || !aligned16(ws) || (rc = check_saved(saved))) return rc ? rc : MOE_ERR_ARG;
    if (ws_bytes < pl.fwd_bytes) return MOE_ERR_WS;
    DeviceInfo dev;
    if ((rc = device_info(&dev))) return rc;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    uint8_t *w8 = static_cast<uint8_t *>(ws);
    if (cudaMemsetAsync(w8 + pl.ws_status, 0, 16, st) != cudaSuccess) return MOE_ERR_LAUNCH;
    return run_route(shape, pl, dev, logits, saved, w8, st);
}

int moe_fwd(const moe_shape_t *shape, const void *x, const float *logits, const void *w_gate_up, const void *w_down,
            void *out, moe_saved_t *saved, void *ws, size_t ws_bytes, void *stream) {
    Plan pl;
    int rc = make_plan(shape, &pl);
    if (rc) return rc;
    if (!aligned16(x) || !aligned16(logits) || !aligned16(w_gate_up) || !aligned16(w_down) || !aligned16(out) ||
        !aligned16(ws))
        return MOE_ERR_ARG;
    if ((rc = check_saved(saved))) return rc;
    if (ws_bytes < pl.fwd_bytes) return MOE_ERR_WS;
    DeviceInfo dev;
    if ((rc = device_info(&dev))) return rc;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    uint8_t *w8 = static_cast<uint8_t *>(ws);

    if (cudaMemsetAsync(w8 + pl.ws_status, 0, 16, st) != cudaSuccess) return MOE_ERR_LAUNCH;
    if ((rc = run_route(shape, pl, dev, logits, saved, w8, st))) return rc;
    if ((rc = gateup_fwd(pl, dev, shape, x, w_gate_up, saved, w8, st))) return rc;
    if (pl.mx) return down_mx(pl, dev, shape, w_down, out, saved, w8, st);
    if ((rc = down_fwd_staged(pl, dev, shape, w_down, saved, w8, nullptr, st))) return rc;
    return run_combine(pl, dev, w8, out, st);
}

int moe_recompute(const moe_shape_t *shape, const void *x, const void *w_gate_up, moe_saved_t *saved, void *ws,
                  size_t ws_bytes, void *stream) {
    Plan pl;
    int rc = make_plan(shape, &pl);
    if (rc) return rc;
    if (!aligned16(x) || !aligned16(w_gate_up) || !aligned16(ws)) return MOE_ERR_ARG;
    if ((rc = check_saved(saved))) return rc;
    if (ws_bytes < pl.fwd_bytes) return MOE_ERR_WS;
    DeviceInfo dev;
    if ((rc = device_info(&dev))) return rc;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    uint8_t *w8 = static_cast<uint8_t *>(ws);
    if (cudaMemsetAsync(w8 + pl.ws_status, 0, 16, st) != cudaSuccess) return MOE_ERR_LAUNCH;
    return gateup_fwd(pl, dev, shape, x, w_gate_up, saved, w8, st);
}

int moe_bwd(const moe_shape_t *shape, const void *grad_out, const void *x, const void *w_gate_up, const void *w_down,
            const moe_saved_t *saved, void *dx, void *dw_gate_up, void *dw_down, float *dscore, float *dlogits,
            void *ws, size_t ws_bytes, void *stream) {
    Plan pl;
    int rc = make_plan(shape, &pl);
    if (rc) return rc;
    if (!aligned16(grad_out) || !aligned16(x) || !aligned16(w_gate_up) || !aligned16(w_down) || !aligned16(dx) ||
        !aligned16(dw_gate_up) || !aligned16(dw_down) || !aligned16(dscore) || !aligned16(ws) ||
        (dlogits && !aligned16(dlogits)))
        return MOE_ERR_ARG;
    if ((rc = check_saved(saved))) return rc;
    if (ws_bytes < pl.bwd_bytes) return MOE_ERR_WS;
    DeviceInfo dev;
    if ((rc = device_info(&dev))) return rc;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    uint8_t *w8 = static_cast<uint8_t *>(ws);
    __nv_bfloat16 *dh = reinterpret_cast<__nv_bfloat16 *>(w8 + pl.ws_dh);
    float *dpart = reinterpret_cast<float *>(w8 + pl.ws_dpart);

    // x in the sorted layout: the forward's copy when the caller kept it, else sorted here
    const bool have_xs = saved->xs != nullptr;
    __nv_bfloat16 *xs = have_xs ? static_cast<__nv_bfloat16 *>(saved->xs)
                                : reinterpret_cast<__nv_bfloat16 *>(w8 + pl.ws_xs);
    __nv_bfloat16 *gs = reinterpret_cast<__nv_bfloat16 *>(w8 + pl.ws_gs);
    if (cudaMemsetAsync(w8 + pl.ws_status, 0, 4, st) != cudaSuccess) return MOE_ERR_LAUNCH;
    const int grid = grid_for(shape, dev);
    GemmArgs a = base_args(pl, const_cast<moe_saved_t *>(saved), w8);
    a.dh = dh;
    a.dpart = dpart;

    // b0: grad_out (and x, unless the forward kept it) in the expert-sorted layout,
    // padding rows zero (operands of the K = tokens wgrads)
    {
        Launch L(kKindSortRows, st);
        const auto *g = static_cast<const __nv_bfloat16 *>(grad_out);
        rc = have_xs ? L.done(launch_sort_rows(saved->inv, saved->counts, saved->group_start, pl.E, pl.k,
                                               static_cast<int>(pl.T), pl.d, g, nullptr, gs, nullptr, true, dev.sms,
                                               st))
                     : L.done(launch_sort_rows(saved->inv, saved->counts, saved->group_start, pl.E, pl.k,
                                               static_cast<int>(pl.T), pl.d, static_cast<const __nv_bfloat16 *>(x),
                                               g, xs, gs, true, dev.sms, st));
        if (rc) return rc;
    }
    if (pl.mx_bwd) {
        if ((rc = bwd_mx(pl, dev, shape, w_gate_up, w_down, saved, dx, dw_gate_up, dw_down, a, xs, gs, w8, st)))
            return rc;
        Launch L(kKindRouteBwd, st);
        return L.done(launch_route_bwd(static_cast<int>(pl.T), pl.E, pl.k, saved->topk_w, saved->topk_idx,
                                       saved->inv, dpart, pl.dpart_stride, dscore, dlogits, st));
    }
    // The scatter-sum into dx (bandwidth bound) needs only the gate/up dgrad's
    // staged rows, and b6 (dscore as the ordered sum of the partials, then
    // dlogits) only the down dgrad's partials: both run on a second stream
    // beside the gate/up wgrad (tensor bound; its persistent CTAs leave threads
    // and registers free on every SM), joined back before the call returns.
    SideStream *side = side_stream();
    bool forked = false;
    auto fork_tail = [&]() -> int {
        cudaStream_t s2 = st;
        if (side != nullptr && side->link(side->fork, st, side->s)) {
            forked = true;
            s2 = side->s;
        }
        int r = run_combine(pl, dev, w8, dx, s2);
        if (r) return r;
        Launch L(kKindRouteBwd, s2);
        return L.done(launch_route_bwd(static_cast<int>(pl.T), pl.E, pl.k, saved->topk_w, saved->topk_idx, saved->inv,
                                       dpart, pl.dpart_stride, dscore, dlogits, s2));
    };
    rc = bwd_gemms(pl, dev, grid, a, gs, xs, w_gate_up, w_down, saved, dw_gate_up, dw_down, nullptr, st, fork_tail);
    if (forked && !side->link(side->join, side->s, st)) return MOE_ERR_LAUNCH;
    return rc;
}

// ---------------------------------------------------------------------------
// expert parallelism (see include/moe.h and ep.cu)
// ---------------------------------------------------------------------------
int moe_ep_expert_layout(int G, int E_loc, const int32_t *recv_counts, int64_t *row_off, int64_t *cmp_off,
                         int64_t *rows, int64_t *padded_rows) {
    if (G < 1 || E_loc < 1 || E_loc > kMaxExperts || !recv_counts || !row_off || !cmp_off || !rows || !padded_rows)
        return MOE_ERR_ARG;
    int64_t cmp = 0, pad = 0;
    for (int e = 0; e < E_loc; ++e) {
        int64_t n_e = 0;
        for (int s = 0; s < G; ++s) {
            const int32_t c = recv_counts[static_cast<int64_t>(s) * E_loc + e];
            if (c < 0) return MOE_ERR_ARG;
            row_off[static_cast<int64_t>(s) * E_loc + e] = pad + n_e;
            cmp_off[static_cast<int64_t>(s) * E_loc + e] = cmp + n_e;
            n_e += c;
        }
        cmp += n_e;
        pad += (n_e + kTileM - 1) / kTileM * kTileM;
    }
    *rows = cmp;
    *padded_rows = pad;
    return MOE_OK;
}

int moe_ep_dispatch(const moe_shape_t *shape, const void *src, const moe_saved_t *saved, void *dst, float *w_rows,
                    void *stream) {
    Plan pl;
    int rc = make_plan(shape, &pl);
    if (rc) return rc;
    if (!aligned16(src) || !aligned16(dst) || (w_rows && !aligned16(w_rows))) return MOE_ERR_ARG;
    if ((rc = check_saved(saved))) return rc;
    DeviceInfo dev;
    if ((rc = device_info(&dev))) return rc;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    {
        Launch L(kKindSortX, st);
        if ((rc = L.done(launch_sort_rows(saved->inv, saved->counts, saved->group_start, pl.E, pl.k,
                                          static_cast<int>(pl.T), pl.d, static_cast<const __nv_bfloat16 *>(src),
                                          nullptr, static_cast<__nv_bfloat16 *>(dst), nullptr, false, dev.sms, st))))
            return rc;
    }
    if (w_rows == nullptr) return MOE_OK;
    Launch L(kKindEpRows, st);
    return L.done(launch_ep_row_weights(saved->perm, saved->tile_expert, saved->counts, saved->offsets,
                                        saved->group_start, saved->topk_w, pl.E, pl.P, pl.p_cap, w_rows, dev.sms, st));
}

// Shape rules of the expert side: T = the rows received, k = 1, E = local experts, bf16 on CTA pairs.
static int expert_side_checks(const moe_shape_t *shape, const Plan &pl, const DeviceInfo &dev) {
    if (shape->k != 1 || shape->dtype != MOE_BF16) return MOE_ERR_UNSUPPORTED;
    if (!gemm_pair_ok(kGateUpFwd, 256, false, 0, grid_for(shape, dev))) return MOE_ERR_UNSUPPORTED;
    (void)pl;
    return MOE_OK;
}

int moe_expert_fwd(const moe_shape_t *shape, int G, const int32_t *recv_counts, void *xr, const void *w_gate_up,
                   const void *w_down, void *y_rows, moe_saved_t *saved, void *ws, size_t ws_bytes, void *stream) {
    Plan pl;
    int rc = make_plan(shape, &pl);
    if (rc) return rc;
    if (G < 1 || !aligned16(recv_counts) || !aligned16(xr) || !aligned16(w_gate_up) || !aligned16(w_down) ||
        !aligned16(y_rows) || !aligned16(ws))
        return MOE_ERR_ARG;
    if ((rc = check_saved(saved))) return rc;
    if (ws_bytes < pl.fwd_bytes) return MOE_ERR_WS;
    DeviceInfo dev;
    if ((rc = device_info(&dev))) return rc;
    if ((rc = expert_side_checks(shape, pl, dev))) return rc;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    uint8_t *w8 = static_cast<uint8_t *>(ws);
    if (cudaMemsetAsync(w8 + pl.ws_status, 0, 16, st) != cudaSuccess) return MOE_ERR_LAUNCH;
    {
        Launch L(kKindEpLayout, st);
        if ((rc = L.done(launch_ep_layout(G, pl.E, recv_counts, pl.p_cap, saved->counts, saved->offsets,
                                          saved->group_start, saved->tile_expert, saved->perm, saved->inv,
                                          reinterpret_cast<int *>(w8 + pl.ws_status), st))))
            return rc;
    }
    {  // the received rows' padding rows to zero (no rows are copied: T = 0)
        Launch L(kKindSortRows, st);
        if ((rc = L.done(launch_sort_rows(saved->inv, saved->counts, saved->group_start, pl.E, 1, 0, pl.d, nullptr,
                                          nullptr, static_cast<__nv_bfloat16 *>(xr), nullptr, true, dev.sms, st))))
            return rc;
    }
    if ((rc = gateup_pair_sorted(pl, shape, dev, xr, w_gate_up, saved, w8, st))) return rc;
    return down_fwd_staged(pl, dev, shape, w_down, saved, w8, y_rows, st);
}

int moe_expert_bwd(const moe_shape_t *shape, void *gr, const void *xr, const void *w_gate_up, const void *w_down,
                   const moe_saved_t *saved, void *dx_rows, void *dw_gate_up, void *dw_down, float *ds_rows,
                   void *ws, size_t ws_bytes, void *stream) {
    Plan pl;
    int rc = make_plan(shape, &pl);
    if (rc) return rc;
    if (!aligned16(gr) || !aligned16(xr) || !aligned16(w_gate_up) || !aligned16(w_down) || !aligned16(dx_rows) ||
        !aligned16(dw_gate_up) || !aligned16(dw_down) || !aligned16(ds_rows) || !aligned16(ws))
        return MOE_ERR_ARG;
    if ((rc = check_saved(saved))) return rc;
    if (ws_bytes < pl.bwd_bytes) return MOE_ERR_WS;
    DeviceInfo dev;
    if ((rc = device_info(&dev))) return rc;
    if ((rc = expert_side_checks(shape, pl, dev))) return rc;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    uint8_t *w8 = static_cast<uint8_t *>(ws);
    float *dpart = reinterpret_cast<float *>(w8 + pl.ws_dpart);
    if (cudaMemsetAsync(w8 + pl.ws_status, 0, 4, st) != cudaSuccess) return MOE_ERR_LAUNCH;
    {  // the received grad_out rows' padding rows to zero
        Launch L(kKindSortRows, st);
        if ((rc = L.done(launch_sort_rows(saved->inv, saved->counts, saved->group_start, pl.E, 1, 0, pl.d, nullptr,
                                          nullptr, static_cast<__nv_bfloat16 *>(gr), nullptr, true, dev.sms, st))))
            return rc;
    }
    GemmArgs a = base_args(pl, const_cast<moe_saved_t *>(saved), w8);
    a.dh = reinterpret_cast<__nv_bfloat16 *>(w8 + pl.ws_dh);
    a.dpart = dpart;
    if ((rc = bwd_gemms(pl, dev, grid_for(shape, dev), a, gr, xr, w_gate_up, w_down, saved, dw_gate_up, dw_down,
                        dx_rows, st)))
        return rc;
    // dscore of every received row (compact order): the ordered sum of its partials
    Launch L(kKindRouteBwd, st);
    return L.done(launch_route_bwd(static_cast<int>(pl.T), pl.E, 1, saved->topk_w, saved->topk_idx, saved->inv, dpart,
                                   pl.dpart_stride, ds_rows, nullptr, st));
}

int moe_ep_combine(const moe_shape_t *shape, const moe_saved_t *saved, const void *rows, void *out, void *stream) {
    Plan pl;
    int rc = make_plan(shape, &pl);
    if (rc) return rc;
    if (!aligned16(rows) || !aligned16(out)) return MOE_ERR_ARG;
    if ((rc = check_saved(saved))) return rc;
    DeviceInfo dev;
    if ((rc = device_info(&dev))) return rc;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    Launch L(kKindCombine, st);
    return L.done(launch_ep_combine(static_cast<const __nv_bfloat16 *>(rows), saved->topk_idx, saved->inv,
                                    saved->offsets, saved->group_start, static_cast<int>(pl.T), pl.E, pl.k, pl.d, pl.P,
                                    static_cast<__nv_bfloat16 *>(out), nullptr, dev.sms, st));
}

int moe_ep_backward_finish(const moe_shape_t *shape, const moe_saved_t *saved, const void *dx_rows,
                           const float *ds_rows, void *dx, float *dscore, float *dlogits, void *stream) {
    Plan pl;
    int rc = make_plan(shape, &pl);
    if (rc) return rc;
    if (!aligned16(dx_rows) || !aligned16(ds_rows) || !aligned16(dx) || !aligned16(dscore) ||
        (dlogits && !aligned16(dlogits)))
        return MOE_ERR_ARG;
    if ((rc = check_saved(saved))) return rc;
    DeviceInfo dev;
    if ((rc = device_info(&dev))) return rc;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    {
        Launch L(kKindCombine, st);
        if ((rc = L.done(launch_ep_combine(static_cast<const __nv_bfloat16 *>(dx_rows), saved->topk_idx, saved->inv,
                                           saved->offsets, saved->group_start, static_cast<int>(pl.T), pl.E, pl.k,
                                           pl.d, pl.P, static_cast<__nv_bfloat16 *>(dx), nullptr, dev.sms, st))))
            return rc;
    }
    Launch L(kKindRouteBwd, st);
    return L.done(launch_route_bwd(static_cast<int>(pl.T), pl.E, pl.k, saved->topk_w, saved->topk_idx, saved->inv,
                                   ds_rows, 1, dscore, dlogits, st, saved->group_start, saved->offsets));
}

int moe_get_status(const void *ws, void *stream, int *device_status) {
    if (!ws || !device_status) return MOE_ERR_ARG;
    int h = 0;
    if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return MOE_ERR_LAUNCH;
    if (cudaMemcpy(&h, ws, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) return MOE_ERR_LAUNCH;
    *device_status = h == kStatusOk ? MOE_OK : (h == kStatusTimeout ? MOE_ERR_TIMEOUT : MOE_ERR_DEVICE);
    return MOE_OK;
}

int moe_selftest_wait_timeout(void *ws, void *stream) {
    if (!aligned16(ws)) return MOE_ERR_ARG;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    int *status = static_cast<int *>(ws);  // the status word is the first field of every workspace
    if (cudaMemsetAsync(status, 0, 4, st) != cudaSuccess) return MOE_ERR_LAUNCH;
    return launch_expire_wait(status, st) == cudaSuccess ? MOE_OK : MOE_ERR_LAUNCH;
}

const char *moe_error_string(int code) {
    switch (code) {
        case MOE_OK: return "ok";
        case MOE_ERR_ARG: return "invalid argument (null or misaligned pointer, or k/T/E out of range)";
        case MOE_ERR_SHAPE:
            return "unsupported shape (d and I must be multiples of 128; E <= 512; k <= 64; T < 2^31; "
                   "P_cap*max(d,2I) and E*max(d,2I) below 2^31)";
        case MOE_ERR_WS: return "workspace too small";
        case MOE_ERR_ARCH: return "device is not an sm_100 (B200-class) GPU";
        case MOE_ERR_LAUNCH: return "CUDA launch or runtime call failed";
        case MOE_ERR_TIMEOUT: return "a device-side bounded wait expired";
        case MOE_ERR_DEVICE: return "a device-side index check failed";
        case MOE_ERR_UNSUPPORTED: return "dtype not implemented";
        case MOE_ERR_SCRATCH_LIMIT: return "shape exceeds the fixed scratch of moe_route_noalloc (ceil(T/64)*E > 131072)";
        default: return "unknown error code";
    }
}

int moe_profile_enable(int on) {
    std::lock_guard<std::mutex> lock(g_mu);
    g_tm.on = on != 0;
    return MOE_OK;
}

int moe_profile_read(double *ms, int64_t *launches, int n_kinds) {
    std::vector<Timing::Rec> recs;
    {
        std::lock_guard<std::mutex> lock(g_mu);
        recs.swap(g_tm.recs);
    }
    for (int i = 0; i < n_kinds; ++i) {
        if (ms) ms[i] = 0.0;
        if (launches) launches[i] = 0;
    }
    int rc = MOE_OK;
    for (auto &r : recs) {
        float t = 0.f;
        if (cudaEventSynchronize(r.b) != cudaSuccess || cudaEventElapsedTime(&t, r.a, r.b) != cudaSuccess)
            rc = MOE_ERR_LAUNCH;
        if (r.kind < n_kinds) {
            if (ms) ms[r.kind] += t;
            if (launches) launches[r.kind] += 1;
        }
    }
    std::lock_guard<std::mutex> lock(g_mu);
    for (auto &r : recs) {
        g_tm.pool.push_back(r.a);
        g_tm.pool.push_back(r.b);
    }
    return rc;
}

const char *moe_kernel_name(int kind) {
    if (kind < 0 || kind >= kNumKernelKinds) return nullptr;
    return kKindNames[kind];
}

}  // extern "C"

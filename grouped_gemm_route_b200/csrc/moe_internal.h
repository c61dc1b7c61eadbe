// Declarations shared by the library's translation units (not part of the ABI).
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace moe {

// Device status codes written to the workspace status word.
enum : int { kStatusOk = 0, kStatusTimeout = 1, kStatusBadIndex = 2 };

constexpr int kTileM = 128;       // rows of one GEMM tile (and the padding unit of an expert group)
constexpr int kTileK = 64;        // K elements per pipeline stage (one 128-byte swizzle row of bf16)
constexpr int kRouteChunk = 64;   // tokens per routing block
constexpr int kMaxExperts = 512;
constexpr int kMaxTopK = 64;

// Where the MXFP8 quantiser puts the block scales.
enum MxSfMode : int { kMxSfAtoms = 0, kMxSfRowBytes = 1, kMxSfGateUp = 2 };

// Kernel kinds, for per-kernel timing.
enum KernelKind : int {
    kKindRouteTopk = 0,
    kKindRouteScan,
    kKindRoutePerm,
    kKindGemmGateUpFwd,
    kKindGemmDownFwd,
    kKindGemmDownDgrad,
    kKindGemmDownWgrad,
    kKindGemmGateUpDgrad,
    kKindGemmGateUpWgrad,
    kKindRouteBwd,
    kKindSortRows,
    kKindMxQuant,
    kKindRouteFused,
    kKindSortX,
    kKindCombine,
    kKindEpLayout,
    kKindEpRows,
    kNumKernelKinds
};

// Which GEMM of the layer a launch computes; selects operand loading and epilogue.
enum GemmMode : int {
    kGateUpFwd = 0,    // h = x_sorted W_gu[e]^T ; epilogue SwiGLU -> h, aw (MXFP8: x rows gathered)
    kDownFwd = 1,      // y = aw W_down[e]^T   ; epilogue stages y per (token, slot) for combine_rows
    kDownDgrad = 2,    // G = gout_sorted W_down[e] ; epilogue dscore partials, SwiGLU bwd -> dh
    kGateUpDgrad = 3,  // dx_p = dh W_gu[e]     ; epilogue stages dx_p per (token, slot) for combine_rows
    kDownWgrad = 4,    // dW_down[e] = gout_sorted^T aw
    kGateUpWgrad = 5,  // dW_gu[e] = dh^T x_sorted
};

struct GemmArgs {
    int T, d, E, k, I;
    int n_tiles;          // tiles along N
    int m_tiles;          // wgrad: tiles along M of one expert's weight
    int num_k_blocks;     // M-tiled modes: K / 64
    int k_elems;          // K elements per pipeline stage: 64 (bf16) or 128 (MXFP8)
    int dpart_stride;     // dscore partials per sorted row
    float limit;          // clamped SwiGLU limit; +inf for the plain SwiGLU
    const int *perm;
    const int *group_start;
    const int *tile_expert;
    const float *topk_w;
    const void *gsrc;           // token rows the gather warps read (x: bf16, or its E4M3 codes)
    const uint8_t *gsf;         // MXFP8: per-row scale bytes of the gathered rows [T, d/32]
    const uint8_t *sfa;         // MXFP8: scale atoms of the A operand (TMA-fed)
    const uint8_t *sfb;         // MXFP8: scale atoms of the B operand
    uint8_t *mx_codes;          // MXFP8 epilogue output codes (aw or dh)
    uint8_t *mx_sf;             // and their scale atoms
    __nv_bfloat16 *h;
    __nv_bfloat16 *aw;
    __nv_bfloat16 *stage;  // staged rows [T*k, d] of the down forward and the gate/up dgrad (row t*k + j)
    __nv_bfloat16 *dh;
    float *dpart;
    __nv_bfloat16 *dw;    // weight gradient (wgrad modes)
    int *status;
};

// Launchers (return cudaError_t of the launch).
cudaError_t launch_route_topk(const float *logits, int T, int E, int k, int32_t *idx, float *w,
                              int32_t *chunk_counts, cudaStream_t s);
cudaError_t launch_route_scan(int T, int E, int n_chunks, const int32_t *chunk_counts, int32_t *chunk_base,
                              int32_t *counts, int32_t *offsets, int32_t *group_start, int32_t *tile_expert,
                              int32_t *perm, int64_t p_cap, int *status, cudaStream_t s);
// Fused routing (one cooperative launch; see route.cu).  route_fused_grid
// returns the grid (all blocks resident, at most n_chunks), 0 on failure;
// launch_route_fused takes the same SM count, from which it picks the same
// kernel configuration.
size_t route_fused_smem(int E, int k);
int route_fused_grid(const float *logits, int T, int E, int k, int sms, int n_chunks);
cudaError_t launch_route_fused(const float *logits, int T, int E, int k, int32_t *idx, float *w, int32_t *blk_hist,
                               int32_t *blk_base, int32_t *counts, int32_t *offsets, int32_t *group_start,
                               int32_t *tile_expert, int32_t *perm, int32_t *inv, int64_t p_cap, unsigned *barrier, int *status, int sms, int grid,
                               cudaStream_t s);
cudaError_t launch_route_perm(int T, int E, int k, const int32_t *idx, const int32_t *chunk_base, int32_t *perm,
                              int32_t *inv, int64_t p_cap, int *status, cudaStream_t s);
// out[t] = slot-ordered fp32 sum of the staged rows t*k + j (bf16 in, bf16 out):
// the down forward's combine and the gate/up dgrad's scatter into dx.
cudaError_t launch_combine_rows(const __nv_bfloat16 *stage, int T, int k, int d, __nv_bfloat16 *out, int sms,
                                cudaStream_t s);
// x (and grad_out, when g is not null) in the expert-sorted layout; zero_pad
// also zeroes each group's padding rows (the wgrads sum over them).
cudaError_t launch_sort_rows(const int32_t *inv, const int32_t *counts, const int32_t *group_start, int E, int k,
                             int T, int d, const __nv_bfloat16 *x, const __nv_bfloat16 *g, __nv_bfloat16 *xs,
                             __nv_bfloat16 *gs, bool zero_pad, int sms, cudaStream_t s);
// dscore (ordered sums of the partials at each pair's row) and dlogits; with
// compact_gs / compact_off the row of pair (t, j) is its compact sorted index
// (expert-parallel path, see ep.cu).
cudaError_t launch_route_bwd(int T, int E, int k, const float *w, const int32_t *idx, const int32_t *inv,
                             const float *dpart, int dpart_stride, float *dscore, float *dlogits, cudaStream_t s,
                             const int32_t *compact_gs = nullptr, const int32_t *compact_off = nullptr);

// Expert-parallel path (ep.cu).  Routing weight of every sorted row in compact order.
cudaError_t launch_ep_row_weights(const int32_t *perm, const int32_t *tile_expert, const int32_t *counts,
                                  const int32_t *offsets, const int32_t *group_start, const float *topk_w, int E,
                                  int64_t P, int64_t p_cap, float *w_rows, int sms, cudaStream_t s);
// Expert side: routing state of the received rows from recv[G][E] (one block).
cudaError_t launch_ep_layout(int G, int E, const int32_t *recv, int64_t p_cap, int32_t *counts, int32_t *offsets,
                             int32_t *group_start, int32_t *tile_expert, int32_t *perm, int32_t *inv, int *status,
                             cudaStream_t s);
// out[t] = slot-ordered sum of the compact rows of token t's pairs.
cudaError_t launch_ep_combine(const __nv_bfloat16 *rows, const int32_t *idx, const int32_t *inv,
                              const int32_t *offsets, const int32_t *group_start, int T, int E, int k, int d,
                              int64_t P, __nv_bfloat16 *out, int *status, int sms, cudaStream_t s);

cudaError_t launch_expire_wait(int *status, cudaStream_t s);

cudaError_t launch_gemm(GemmMode mode, int bn, bool mx, const GemmArgs &args, const CUtensorMap &tmA,
                        const CUtensorMap &tmB, int grid, cudaStream_t s);
// GEMMs on CTA pairs (tcgen05 cta_group::2, bf16, BN = 256), all six modes;
// used where gemm_pair_ok holds, with the same arguments and results as
// launch_gemm.
bool gemm_pair_ok(GemmMode mode, int bn, bool mx, int m_tiles, int grid);
// tmC, the third tensor map: the forward GEMMs' A operand in 64-row boxes (an
// expert's unpaired last tile loads 64 rows per CTA), h for the down dgrad
// (make_map_h), dW for the weight gradients (32-row x 64-column boxes, 128-byte
// swizzle: their epilogues store by TMA); null only for the gate/up dgrad.  tmD, tmE:
// the gate/up forward's h and aw in 32 x 32 boxes (its epilogue's TMA stores).
cudaError_t launch_gemm_pair(GemmMode mode, const GemmArgs &args, const CUtensorMap &tmA, const CUtensorMap &tmB,
                             int grid, cudaStream_t s, const CUtensorMap *tmC = nullptr,
                             const CUtensorMap *tmD = nullptr, const CUtensorMap *tmE = nullptr);

cudaError_t launch_mx_quant_rows(const __nv_bfloat16 *src, int64_t R, int K, uint8_t *dst, uint8_t *sf, int sf_mode,
                                 int I, const int32_t *rows_used, int sms, cudaStream_t s);
cudaError_t launch_mx_quant_cols(const __nv_bfloat16 *src, int64_t Kr, int N, uint8_t *dst, uint8_t *sf,
                                 const int32_t *rows_used, int sms, cudaStream_t s);

}  // namespace moe

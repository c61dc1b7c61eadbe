/*
 * moe.h -- C ABI of libmoe.so, a single-GPU fused mixture-of-experts layer
 * (forward and backward) for NVIDIA B200 (sm_100a).
 *
 * What the layer computes.  "Prime Intellect Fused MoE Kernel: 3.11x MoE
 * Training Speed", section "What a mixture-of-experts layer actually does":
 * a router sends each token to a few experts and one fused call performs the
 * dispatch, both expert linear layers, SwiGLU and the combine.  "Prime
 * Intellect's Prime Mega MoE Trains Giant AI Models 55% Faster", section
 * "Where MoE training loses time": tokens are sorted by expert, the expert
 * MLPs run, the outputs return to their original positions, and the backward
 * pass repeats the exchange for gradients.  "Mario/overlap moe kernel
 * integration (prime-rl PR #3651)", Overview and the custom-op commit note:
 * the fused compute takes undispatched tokens plus their routing, runs in
 * bf16 and returns gradients in the inputs' dtypes.  Here the expert-parallel
 * network exchange of those pages becomes an on-GPU copy of the tokens into
 * the expert-sorted layout (dispatch; under MXFP8 a gather inside the GEMM's
 * operand load) and an ordered reduction (combine / scatter).
 *
 * Definitions (P = T*k token-slot pairs; pair (t,j) is flat index t*k+j):
 *   routing   idx[t,:] = the k largest logits[t,:] (ties -> lower expert index),
 *             slot j = j-th largest; w[t,j] = exp(l_j - l_max) / sum over the
 *             chosen k of exp(l_i - l_max)  (softmax renormalised over the k)
 *   dispatch  counts[e] = #pairs routed to e; offsets = exclusive scan(counts);
 *             pairs sorted by expert, tokens ascending inside an expert
 *   expert    h = W_gate_up[e] x[t]  (W_gate_up[e] is [2I,d]: gate rows then up rows)
 *             a = silu(h[0:I]) * h[I:2I];  y = W_down[e] a  (W_down[e] is [d,I])
 *             (moe_shape_t.swiglu_limit selects the clamped form of a)
 *   combine   out[t] = sum_{j=0..k-1, in slot order} w[t,j] y_(t,j)
 *   backward  dscore[t,j] = <gout[t], y_(t,j)>,  dx, dW_gate_up, dW_down,
 *             dlogits[t,i] = w_i (dscore_i - sum_j w_j dscore_j) for chosen i, else 0
 *
 * Conventions for every entry point:
 *   - All pointers are DEVICE pointers unless stated otherwise, in memory of the
 *     current CUDA device (cudaSetDevice), on which every call launches; every
 *     tensor is row-major and contiguous.  bf16 = IEEE bfloat16 (2 bytes).
 *   - The caller owns and allocates every buffer (outputs, saved state and the
 *     workspace).  The library never allocates or frees device memory and keeps
 *     no state between calls except cached per-device properties and, per
 *     device, one extra stream with two events: moe_bwd forks bandwidth-bound
 *     work onto it beside a tensor-bound GEMM and joins it back into `stream`
 *     before its last kernel (ordering on `stream` is as if everything ran
 *     there).
 *   - Calls are asynchronous on `stream` (a cudaStream_t; NULL = legacy default
 *     stream).  Calls that share a workspace must not overlap on the GPU.
 *   - Return value: MOE_OK (0) or a negative MOE_ERR_* code.  Arguments are
 *     validated on the host before anything is launched; on an argument error
 *     nothing is launched.  Device-side problems (a bounded wait that expired, an
 *     out-of-range index) are recorded in a status word inside the workspace
 *     and reported by moe_get_status.
 *   - Shape limits: 1 <= k <= min(E, 64), E <= 512, d and I multiples of 128,
 *     1 <= T < 2^31, P_cap*max(d,2I) < 2^31 (P_cap, the sorted-layout row
 *     capacity, from moe_saved_sizes; about T*k + 127*E), E*max(d,2I) < 2^31.
 *     Shapes past these limits return MOE_ERR_SHAPE.  Pointers must be 16-byte
 *     aligned.
 */
#ifndef MOE_H_
#define MOE_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Return codes. */
#define MOE_OK 0
#define MOE_ERR_ARG (-1)         /* null / misaligned pointer, k < 1, k > E, T < 1 ... */
#define MOE_ERR_SHAPE (-2)       /* d or I not a multiple of 128, a size above the limits   */
#define MOE_ERR_WS (-3)          /* workspace smaller than moe_workspace_size reports */
#define MOE_ERR_ARCH (-4)        /* current device is not compute capability 10.0 */
#define MOE_ERR_LAUNCH (-5)      /* a CUDA launch or runtime call failed */
#define MOE_ERR_TIMEOUT (-6)     /* a device-side bounded wait expired (moe_get_status) */
#define MOE_ERR_DEVICE (-7)      /* a device-side index check failed (moe_get_status) */
#define MOE_ERR_UNSUPPORTED (-8) /* dtype not implemented */
#define MOE_ERR_SCRATCH_LIMIT (-9) /* moe_route_noalloc: ceil(T/64)*E above its fixed scratch capacity */

/* Operand precision of the expert GEMMs. */
/* MOE_MXFP8_FWD: MXFP8 forward GEMMs, bf16 backward GEMMs (the backward runs
 * on the h and aw the MXFP8 forward saved) -- the pages' `fp8_bwd` switch
 * ("Prime Intellect's Prime Mega MoE Trains Giant AI Models 55% Faster",
 * section "Precision and hardware support") set off. */
typedef enum { MOE_BF16 = 0, MOE_MXFP8 = 1, MOE_MXFP8_FWD = 2 } moe_dtype_t;

/* Layer shape.  T tokens, hidden size d, E experts, top-k, expert width I.
 * max_sms caps the persistent grids (0 = every SM).
 *
 * swiglu_limit selects the expert activation.  0: SwiGLU, a = silu(gate) * up.
 * L > 0: the clamped SwiGLU that the review note of "Mario/overlap moe kernel
 * integration (prime-rl PR #3651)" says the fused kernel computes (DeepSeek V4
 * ClampedSilu; the pages give no formula, this is the library's reading):
 * a = silu(min(gate, L)) * clamp(up, -L, L), whose gradient passes where the
 * input lies inside the closed interval and is zero outside it.  Negative,
 * infinite or NaN limits are rejected with MOE_ERR_ARG. */
typedef struct {
    int64_t T;
    int32_t d, E, k, I;
    int32_t dtype;   /* moe_dtype_t */
    int32_t max_sms;
    float swiglu_limit;
} moe_shape_t;

/* State written by moe_fwd (and moe_route) and read by moe_bwd.  Every field
 * is a caller-allocated device buffer of the size moe_saved_sizes reports, in
 * this order.  "Sorted layout": pairs grouped by expert; expert e's group starts
 * at row group_start[e], a multiple of 128, and holds counts[e] pairs followed by
 * padding rows up to the next multiple of 128.  P_cap (the row capacity of the
 * sorted layout) is reported by moe_saved_sizes. */
typedef struct {
    int32_t *topk_idx;    /* [T,k]   chosen experts, slot order                        */
    float *topk_w;        /* [T,k]   renormalised routing weights                      */
    int32_t *counts;      /* [E]     pairs per expert                                  */
    int32_t *offsets;     /* [E+1]   exclusive scan of counts (unpadded)               */
    int32_t *group_start; /* [E+1]   padded group starts; group_start[E] = rows used   */
    int32_t *tile_expert; /* [P_cap/128] expert owning each 128-row tile               */
    int32_t *perm;        /* [P_cap] sorted row -> pair t*k+j, or -1 for a padding row */
    int32_t *inv;         /* [T,k]   pair -> sorted row                                */
    void *h;              /* bf16 [P_cap, 2I] gate/up pre-activations, sorted layout   */
    void *aw;             /* bf16 [P_cap, I]  w[t,j] * silu(gate) * up, sorted layout  */
    void *xs;             /* bf16 [P_cap, d]  x in the sorted layout, padding rows 0; OPTIONAL:
                           * when not NULL, moe_fwd and moe_recompute write it and moe_bwd reads
                           * it instead of sorting x again (NULL: moe_bwd sorts x itself) */
} moe_saved_t;

#define MOE_SAVED_FIELDS 11

/* Bytes of each moe_saved_t field (in declaration order) and the sorted-layout
 * row capacity.  Pure host function; touches no GPU. */
int moe_saved_sizes(const moe_shape_t *shape, size_t sizes[MOE_SAVED_FIELDS], int64_t *p_cap);

/* Workspace bytes needed by moe_fwd and by moe_bwd (one buffer of the larger
 * size serves both).  Pure host function; touches no GPU. */
int moe_workspace_size(const moe_shape_t *shape, size_t *fwd_bytes, size_t *bwd_bytes);

/* Routing and dispatch only (steps: top-k + weights, histogram + scan,
 * stable permutation).  logits: fp32 [T,E].  Fills topk_idx, topk_w, counts,
 * offsets, group_start, tile_expert, perm and inv of `saved`. */
int moe_route(const moe_shape_t *shape, const float *logits, moe_saved_t *saved,
              void *ws, size_t ws_bytes, void *stream);

/* Forward.  x: bf16 [T,d]; logits: fp32 [T,E]; w_gate_up: bf16 [E,2I,d];
 * w_down: bf16 [E,d,I]; out: bf16 [T,d].  Runs moe_route, then the gate/up
 * grouped GEMM (bf16: on x copied into the expert-sorted layout; MXFP8: token
 * rows gathered through the dispatch permutation straight into the GEMM's
 * operand tiles; SwiGLU in the epilogue; writes saved->h and saved->aw), then
 * the down grouped GEMM, whose epilogue stages each (token, slot) product, and
 * the weighted combine as a deterministic slot-ordered reduction into out. */
int moe_fwd(const moe_shape_t *shape, const void *x, const float *logits,
            const void *w_gate_up, const void *w_down, void *out,
            moe_saved_t *saved, void *ws, size_t ws_bytes, void *stream);

/* Backward for a loss L with dL/dout = grad_out (bf16 [T,d]).  Reads the state
 * moe_fwd saved.  Writes dx bf16 [T,d], dw_gate_up bf16 [E,2I,d], dw_down bf16
 * [E,d,I], dscore fp32 [T,k] (gradient w.r.t. topk_w) and, when dlogits is not
 * NULL, dlogits fp32 [T,E].  Experts that received no token get exact-zero
 * weight gradients.  All reductions have a fixed order: results are bitwise
 * reproducible. */
int moe_bwd(const moe_shape_t *shape, const void *grad_out, const void *x,
            const void *w_gate_up, const void *w_down, const moe_saved_t *saved,
            void *dx, void *dw_gate_up, void *dw_down, float *dscore, float *dlogits,
            void *ws, size_t ws_bytes, void *stream);

/* Recompute mode ("Mario/overlap moe kernel integration (prime-rl PR #3651)",
 * the custom-op commit note: under activation checkpointing the op saves only
 * its own inputs and the forward runs again before the backward).  Rewrites
 * saved->h and saved->aw from x and w_gate_up for the routing already in
 * `saved` (topk_w, group_start, tile_expert, perm from moe_fwd or moe_route):
 * the gate/up grouped GEMM and its SwiGLU epilogue only, bit-identical to what
 * moe_fwd wrote.  A caller may therefore drop h and aw after the forward and
 * call this before moe_bwd.  Workspace: fwd_bytes of moe_workspace_size.
 * Arguments and errors as moe_fwd. */
int moe_recompute(const moe_shape_t *shape, const void *x, const void *w_gate_up, moe_saved_t *saved,
                  void *ws, size_t ws_bytes, void *stream);

/* Routing and dispatch for callers that cannot allocate device memory.
 *
 * The pages have no counterpart to this entry point; it exists for users of
 * the library that are not allowed to call cudaMalloc: for example code running
 * inside a host program whose memory manager owns all of the GPU's memory and
 * gives none to plug-ins, or code on a latency-critical path where an
 * allocation (which may synchronise the whole device) is not acceptable.
 *
 * Same results as moe_route, bit for bit: indices, weights, counts, offsets,
 * group starts, tile table, permutation and its inverse (it runs the
 * three-launch form of the same routing: top-k, scan, permutation; every form
 * sums a token's k exponentials in slot order), but the per-block histograms and
 * bases that it keeps in a workspace live instead in a fixed
 * 1 MiB __device__ array inside the library, which every GPU that loads the
 * library holds until the process exits.  The caller still allocates and
 * passes the logits and every moe_saved_t routing field (topk_idx, topk_w,
 * counts, offsets, group_start, tile_expert, perm, inv); h and aw are not used.
 * Nothing is allocated or freed: no cudaMalloc, no cudaFree, no allocating
 * library routine.
 *
 * Limit: 2 * ceil(T/64) * E * 4 bytes must fit in 1 MiB, i.e. ceil(T/64) * E <=
 * 131072 (e.g. T = 16384 with E <= 512, or T = 65536 with E <= 128); larger
 * shapes return MOE_ERR_SCRATCH_LIMIT before anything is launched.  Other shape
 * rules and error codes are those of moe_route.
 *
 * The first call on each device looks up the array's device address with
 * cudaGetSymbolAddress (with that device current) and caches it together with
 * the identifier of the current context; make that first call before any
 * stream capture.  A call that finds a different context current (after
 * cudaDeviceReset, for example) looks the address up again, so the first call
 * after a reset must also come before any capture.  All calls share the one array and it
 * keeps the last call's contents; every word a call reads is written earlier in
 * the same call, so nothing needs clearing.  Calls that overlap on the GPU (on
 * different streams, or from different host threads) race on the array and
 * must be serialised by the caller.  Device-side index checks are not
 * reported by this entry point (it has no status word). */
int moe_route_noalloc(const moe_shape_t *shape, const float *logits, moe_saved_t *saved, void *stream);

/* ---------------------------------------------------------------------------
 * Expert parallelism (EP).  "Prime Intellect's Prime Mega MoE Trains Giant AI
 * Models 55% Faster", sections "Where MoE training loses time" and "One kernel
 * overlaps the pipeline": the experts are spread over G GPUs, every token
 * travels to the GPUs that own its experts and the results travel back; the
 * backward pass repeats the exchange for gradients.
 *
 * Rank q of G owns the E/G consecutive experts [q*E/G, (q+1)*E/G) (E a
 * multiple of G).  Every rank holds its own T tokens and the weights of its
 * own experts.  The exchanges are copies between the GPUs' own memories (NCCL
 * send/receive, issued by the caller between these calls); no kernel here
 * reads another GPU's memory.  One layer step on every rank:
 *
 *  source side   moe_route over all E experts, then moe_ep_dispatch: x rows in
 *                the sorted layout (`xs`, group of expert e at group_start[e])
 *                and the routing weight of every pair in compact sorted order
 *                (`w_rows`: expert e's pairs at offsets[e] ..).  Because the
 *                experts of one rank are consecutive, so are their groups.
 *                For destination q and each of its experts e it sends
 *                counts[e] rows of xs from row group_start[e] and counts[e]
 *                weights of w_rows from offsets[e]; it sends counts[q*E/G ..
 *                (q+1)*E/G - 1] first, so that q can size its buffers.
 *  expert side   recv_counts[s][e] = rows of local expert e from source s.
 *                moe_ep_expert_layout (host) gives where those land: xr row
 *                row_off[s][e] (the local sorted layout, every local expert's
 *                group padded to 128 rows, sources in rank order inside it)
 *                and compact index cmp_off[s][e] (w_rows, results).
 *                moe_expert_fwd runs the gate/up GEMM + SwiGLU and the down
 *                GEMM on them; each received row's product w * y goes to its
 *                compact index of y_rows, which the expert side sends back:
 *                recv_counts[s][e] rows from cmp_off[s][e] to source s.
 *  source side   receives them at compact index offsets[e] + ... (the mirror
 *                of its sends) and moe_ep_combine sums each token's k rows in
 *                slot order into out.
 *  backward      source: moe_ep_dispatch of grad_out (no weights), sent like
 *                x.  Expert: moe_expert_bwd -> dx rows and dscore rows
 *                (compact, sent back like y) and the local experts' dW.
 *                Source: moe_ep_backward_finish -> dx, dscore, dlogits.
 *
 * With G = 1 the results are those of moe_fwd / moe_bwd, bit for bit.  Only
 * bf16 operands, and the gate/up GEMM on CTA pairs (max_sms != 1), are
 * supported on the expert side; other shapes return MOE_ERR_UNSUPPORTED.
 * The source-side calls take no workspace: their index checks skip a bad row
 * without reporting it.
 * ------------------------------------------------------------------------- */

/* Host only.  recv_counts: host int32 [G][E_loc].  Writes row_off[G][E_loc]
 * (first row of each (source, expert) segment in the expert side's padded
 * sorted layout), cmp_off[G][E_loc] (first compact index), the number of rows
 * received and the padded row count.  MOE_ERR_ARG on a negative count. */
int moe_ep_expert_layout(int G, int E_loc, const int32_t *recv_counts, int64_t *row_off, int64_t *cmp_off,
                         int64_t *rows, int64_t *padded_rows);

/* Source side, after moe_route with the same shape: src (bf16 [T,d], x or
 * grad_out) into dst (bf16 [P_cap, d], sorted layout; padding rows are not
 * written) and, when w_rows is not NULL, w_rows (fp32 [T*k]) = the routing
 * weight of each pair in compact sorted order. */
int moe_ep_dispatch(const moe_shape_t *shape, const void *src, const moe_saved_t *saved, void *dst, float *w_rows,
                    void *stream);

/* Expert side, forward.  shape: T = rows received (from moe_ep_expert_layout),
 * k = 1, E = E_loc, d, I as the layer's; every buffer sized by
 * moe_saved_sizes / moe_workspace_size for that shape.  recv_counts: device
 * int32 [G][E_loc].  xr: bf16 [P_cap, d], the received rows at row_off (its
 * padding rows are zeroed here).  saved->topk_w: the received weights (compact
 * order); the call fills the other routing fields of `saved` for the received
 * layout (perm: padded row -> compact index, inv: compact index -> padded row)
 * and h, aw.  w_gate_up, w_down: the local experts' weights [E_loc, ...].
 * y_rows: bf16 [T, d], row i = w_i * (W_down a) of compact row i. */
int moe_expert_fwd(const moe_shape_t *shape, int G, const int32_t *recv_counts, void *xr, const void *w_gate_up,
                   const void *w_down, void *y_rows, moe_saved_t *saved, void *ws, size_t ws_bytes, void *stream);

/* Expert side, backward, after moe_expert_fwd on the same `saved`.  gr: bf16
 * [P_cap, d], the received grad_out rows at row_off (padding zeroed here).
 * Writes dx_rows (bf16 [T, d], compact), ds_rows (fp32 [T], dL/dw of each
 * received pair, compact) and the local experts' dw_gate_up, dw_down (an expert
 * that received no row gets exact zeros). */
int moe_expert_bwd(const moe_shape_t *shape, void *gr, const void *xr, const void *w_gate_up, const void *w_down,
                   const moe_saved_t *saved, void *dx_rows, void *dw_gate_up, void *dw_down, float *ds_rows,
                   void *ws, size_t ws_bytes, void *stream);

/* Source side: out[t] (bf16 [T,d]) = sum over slots j = 0..k-1, in slot order,
 * of rows (bf16 [T*k, d], compact sorted order, as received back) of token t's
 * pairs; fp32 sum, one bf16 rounding. */
int moe_ep_combine(const moe_shape_t *shape, const moe_saved_t *saved, const void *rows, void *out, void *stream);

/* Source side, backward: dx (bf16 [T,d]) from dx_rows as moe_ep_combine does;
 * dscore[t,j] (fp32 [T,k]) = ds_rows of the pair; dlogits (fp32 [T,E], or NULL)
 * through the renormalised softmax, as moe_bwd computes them. */
int moe_ep_backward_finish(const moe_shape_t *shape, const moe_saved_t *saved, const void *dx_rows,
                           const float *ds_rows, void *dx, float *dscore, float *dlogits, void *stream);

/* Synchronises `stream`, then reads the device status word of `ws` written by
 * the most recent moe_route / moe_fwd / moe_bwd on that workspace:
 * *device_status = MOE_OK, MOE_ERR_TIMEOUT or MOE_ERR_DEVICE.  Returns MOE_OK
 * or MOE_ERR_LAUNCH if the copy itself failed. */
int moe_get_status(const void *ws, void *stream, int *device_status);

/* Failure-path self-test.  Launches one small kernel whose bounded wait on an
 * mbarrier that nothing arrives at must expire (after about 2 s); the kernel then
 * records MOE_ERR_TIMEOUT in the status word of `ws` (at least 16 bytes, device
 * memory) and returns, leaving nothing in flight.  moe_get_status(ws, ...)
 * afterwards reports MOE_ERR_TIMEOUT; later calls on the same context work
 * normally.  Returns MOE_OK once launched. */
int moe_selftest_wait_timeout(void *ws, void *stream);

/* Static string for a return code.  Never NULL. */
const char *moe_error_string(int code);

/* Per-kernel timing.  While enabled, every launch made by the library is
 * bracketed by two CUDA events on its stream.  moe_profile_read synchronises
 * the recorded events and returns, per kernel kind (0 <= kind < n_kinds), the
 * summed device milliseconds and the launch count since the last reset, then
 * resets.  moe_kernel_name names a kind ("route_topk", "gemm_gateup_fwd" ...),
 * or returns NULL past the last kind.  Host-side bookkeeping only.  The timing
 * events are pooled for the whole process: profile one device per process (a
 * launch timed on another device than the events' own makes moe_profile_read
 * return MOE_ERR_LAUNCH; the layer's results are not affected). */
int moe_profile_enable(int on);
int moe_profile_read(double *ms, int64_t *launches, int n_kinds);
const char *moe_kernel_name(int kind);

#ifdef __cplusplus
}
#endif

#endif /* MOE_H_ */

// moe_route_noalloc: the routing step (top-k, histogram + scan, permutation)
// for callers that cannot allocate device memory.
//
// Some callers of this library live inside a host program whose memory
// manager owns all of the GPU's memory and hands none to plug-ins, or run on a
// latency-critical path where a cudaMalloc (which can synchronise the whole
// device) is not acceptable.  moe_route needs a caller-provided workspace for
// its per-block histograms; this entry point instead takes that scratch from a
// fixed array that lives in the library itself, so the caller passes only the
// logits and the routing outputs.
//
// The scratch is a file-scope __device__ array of kScratchBytes (1 MiB).  Every
// GPU that loads the library keeps it until the process exits.  In host code
// the array's name is only a host-side stand-in, so its device address is
// looked up with cudaGetSymbolAddress once per device, with that device
// current, on the first call made on that device.  The address is kept with
// the identifier of the context it belongs to; a call that finds another
// context current (cudaDeviceReset destroys the device's primary context and
// the next runtime call creates a new one, with the module loaded anew) looks
// the address up again.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>
#include <stdint.h>

#include <mutex>

#include "moe.h"
#include "moe_internal.h"

using namespace moe;

namespace {

constexpr size_t kScratchBytes = size_t(1) << 20;
constexpr int kMaxDevices = 64;

// Per-block expert histograms and per-block bases: 2 * ceil(T/64) * E int32.
static __device__ __align__(256) unsigned char g_route_scratch[kScratchBytes];

std::mutex g_scratch_mu;
void *g_scratch_addr[kMaxDevices] = {};
unsigned long long g_scratch_ctx[kMaxDevices] = {};  // context identifier the address belongs to
PFN_cuCtxGetCurrent_v4000 g_ctx_current = nullptr;
PFN_cuCtxGetId_v12000 g_ctx_id = nullptr;

// Identifier of the current context (0: none current yet, or not available).
unsigned long long current_context_id() {
    CUcontext ctx = nullptr;
    unsigned long long id = 0;
    if (g_ctx_current(&ctx) != CUDA_SUCCESS || ctx == nullptr) return 0;
    if (g_ctx_id(ctx, &id) != CUDA_SUCCESS) return 0;
    return id;
}

// Device address of g_route_scratch on the current device: looked up on the
// first call on a device, and again whenever the current context is not the
// one the cached address was taken in.
int scratch_address(void **out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return MOE_ERR_LAUNCH;
    std::lock_guard<std::mutex> lock(g_scratch_mu);
    if (g_ctx_current == nullptr || g_ctx_id == nullptr) {
        void *f1 = nullptr, *f2 = nullptr;
        cudaDriverEntryPointQueryResult q1, q2;
        if (cudaGetDriverEntryPointByVersion("cuCtxGetCurrent", &f1, 4000, cudaEnableDefault, &q1) != cudaSuccess ||
            q1 != cudaDriverEntryPointSuccess || f1 == nullptr ||
            cudaGetDriverEntryPointByVersion("cuCtxGetId", &f2, 12000, cudaEnableDefault, &q2) != cudaSuccess ||
            q2 != cudaDriverEntryPointSuccess || f2 == nullptr)
            return MOE_ERR_LAUNCH;
        g_ctx_current = reinterpret_cast<PFN_cuCtxGetCurrent_v4000>(f1);
        g_ctx_id = reinterpret_cast<PFN_cuCtxGetId_v12000>(f2);
    }
    const unsigned long long ctx = current_context_id();
    if (g_scratch_addr[dev] == nullptr || ctx == 0 || ctx != g_scratch_ctx[dev]) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_route_scratch) != cudaSuccess || p == nullptr) return MOE_ERR_LAUNCH;
        const unsigned long long now = current_context_id();  // the lookup makes the context current
        if (now == 0) return MOE_ERR_LAUNCH;
        g_scratch_addr[dev] = p;
        g_scratch_ctx[dev] = now;
    }
    *out = g_scratch_addr[dev];
    return MOE_OK;
}

bool aligned16_ptr(const void *p) { return p && (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace

extern "C" int moe_route_noalloc(const moe_shape_t *shape, const float *logits, moe_saved_t *saved, void *stream) {
    // shape rules and the sorted-layout capacity are those of moe_saved_sizes
    int64_t p_cap = 0;
    int rc = moe_saved_sizes(shape, nullptr, &p_cap);
    if (rc != MOE_OK) return rc;
    if (!saved || !aligned16_ptr(logits) || !aligned16_ptr(saved->topk_idx) || !aligned16_ptr(saved->topk_w) ||
        !aligned16_ptr(saved->counts) || !aligned16_ptr(saved->offsets) || !aligned16_ptr(saved->group_start) ||
        !aligned16_ptr(saved->tile_expert) || !aligned16_ptr(saved->perm) || !aligned16_ptr(saved->inv))
        return MOE_ERR_ARG;
    const int T = static_cast<int>(shape->T), E = shape->E, k = shape->k;
    const int64_t n_chunks = (shape->T + kRouteChunk - 1) / kRouteChunk;
    const size_t need = 2 * static_cast<size_t>(n_chunks) * static_cast<size_t>(E) * sizeof(int32_t);
    if (need > kScratchBytes) return MOE_ERR_SCRATCH_LIMIT;

    int dev = 0, major = 0, minor = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess)
        return MOE_ERR_LAUNCH;
    if (major != 10 || minor != 0) return MOE_ERR_ARCH;

    void *base = nullptr;
    if ((rc = scratch_address(&base)) != MOE_OK) return rc;
    int32_t *chunk_counts = static_cast<int32_t *>(base);
    int32_t *chunk_base = chunk_counts + n_chunks * E;
    cudaStream_t st = static_cast<cudaStream_t>(stream);

    // Every scratch word read below is written earlier in this same call
    // (route_topk writes all histograms, route_scan all bases), so nothing in
    // the shared array has to be cleared first.
    if (launch_route_topk(logits, T, E, k, saved->topk_idx, saved->topk_w, chunk_counts, st) !=
        cudaSuccess)
        return MOE_ERR_LAUNCH;
    if (launch_route_scan(T, E, static_cast<int>(n_chunks), chunk_counts, chunk_base, saved->counts, saved->offsets,
                          saved->group_start, saved->tile_expert, saved->perm, p_cap, nullptr, st) != cudaSuccess)
        return MOE_ERR_LAUNCH;
    if (launch_route_perm(T, E, k, saved->topk_idx, chunk_base, saved->perm, saved->inv, p_cap, nullptr, st) !=
        cudaSuccess)
        return MOE_ERR_LAUNCH;
    return MOE_OK;
}

// Persistent grouped GEMMs of the fused MoE layer on the sm_100a tensor cores.
//
// One kernel template serves the six expert GEMMs of the layer (two forward,
// four backward).  Each CTA owns one SM and walks a static list of output
// tiles.  Inside a CTA the work is split by warp:
//   warp 0       TMA producer: bulk tensor loads of the dense operand (expert
//                weights, or the sorted-layout activations) into a 4- or
//                6-stage shared-memory ring, 128-byte swizzled.
//   warp 1       allocates tensor memory and issues tcgen05.mma (one thread),
//                accumulating a 128 x BN fp32 tile in TMEM; two TMEM buffers
//                let the epilogue of one tile overlap the mainloop of the next.
//   warps 2..5   epilogue, one warp per tensor-memory lane quadrant (its 32
//                rows; tcgen05.ld, one output row per thread) and the mode's
//                fused epilogue.  The down dgrad, whose epilogue waits on loads
//                of h, runs eight: warps 2..9, two per quadrant, each taking
//                half of the tile's columns.
//   next two     MXFP8 forward gate/up GEMM: gather producers, 16-byte
//                cp.async copies of the x rows picked through the dispatch
//                permutation, written with the same 128-byte swizzle.  Idle in
//                the other modes.  (The bf16 forward and the backward read x,
//                and the backward grad_out, from expert-sorted copies made by
//                sort_rows, so that their GEMMs run on plain TMA tiles.)
//
// Modes (see GemmMode): the expert MLP of "Prime Intellect Fused MoE Kernel:
// 3.11x MoE Training Speed", section "What a mixture-of-experts layer actually
// does" (both expert linear layers and SwiGLU), the combine back into token
// order, and for the backward pass (the exchange repeated for gradients,
// "Prime Intellect's Prime Mega MoE Trains Giant AI Models 55% Faster", section
// "Where MoE training loses time") the two dgrads, the two wgrads and the
// scatter of token gradients back to token order.
//
// The combine and the scatter are deterministic: the down forward and the
// gate/up dgrad store each (token, slot) row of their output, rounded to bf16,
// to a slot-addressed staging buffer, and a bandwidth-bound kernel
// (combine_rows) then sums every token's k staged rows in slot order.  Summing
// inside the GEMM (per-row counters, a last-arriver queue and worker warps)
// measured slower: the workers competed with the mainloop for the SM and the
// memory system.
//
// Every wait on an mbarrier is bounded in time.  On expiry the kernel records
// a timeout in the status word, stops issuing work, waits (bounded) for its own
// copies and MMAs in flight, frees its tensor memory and returns.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <atomic>
#include <type_traits>

#include "moe_internal.h"
#include "mx.cuh"
#include "ptx.cuh"

namespace moe {

namespace {

constexpr int kEpiWarp0 = 2;                  // epilogue warps start here (one or two per TMEM lane quadrant)
constexpr int kMaxEpiWarps = 8;
constexpr int kGatherThreads = 64;
constexpr int kABytes = kTileM * kTileK * 2;  // 16 KB: 128 rows x 64 bf16
constexpr int kChunkBytes = 64 * kTileK * 2;  // 8 KB: one 64-wide MN chunk of an MN-major K-block
constexpr uint32_t kSbo = 1024;               // 8 rows x 128 B swizzle atom
constexpr uint32_t kMnLbo = kChunkBytes;      // MN-major: distance between 64-wide chunks
constexpr int kXposeBytes = 32 * 64;          // per epilogue warp: 32 rows x 64 bytes

// Pipeline geometry.  A stage holds one K block of both operands: 128-byte
// operand rows, i.e. 64 bf16 or 128 E4M3 elements.  MXFP8 stages also carry
// the A and B scale atoms (512 bytes each) and use BN = 128 so that the two
// 128-column accumulators leave tensor-memory columns for the scales.
template <int BN, bool MX = false>
struct Cfg {
    static constexpr int kStages = BN == 256 ? 4 : 6;
    static constexpr int kKElems = MX ? 128 : 64;                  // K elements per stage
    static constexpr int kBBytes = BN * kTileK * 2;
    static constexpr int kStageBytes = kABytes + kBBytes;
    static constexpr int kSfBytes = MX ? 2 * kMxAtomBytes : 0;     // scale atoms per stage
    static constexpr int kSfOffset = kStages * kStageBytes;
    static constexpr int kBarOffset = kSfOffset + kStages * kSfBytes;  // mbarriers, TMEM slot, abort flag
    static constexpr int kOrderOffset = kBarOffset + 512;              // the wgrads' expert order
    static constexpr int kXposeOffset = kOrderOffset + 8 * kMaxExperts;  // one 2 KB transpose per epilogue warp
    // + 1 KB alignment slack; the largest layout must fit 227 KB
    static constexpr int smem_bytes(int epi_warps) { return kXposeOffset + epi_warps * kXposeBytes + 1024; }
    static_assert(smem_bytes(kMaxEpiWarps) <= 227 * 1024, "shared memory per CTA");
    static constexpr uint32_t kTmemCols = MX ? 512 : 2 * BN;
};

template <int MODE>
struct ModeTraits {
    static constexpr bool kMTiled = MODE <= kGateUpDgrad;  // M = sorted rows
    static constexpr bool kGather = MODE == kGateUpFwd;  // x rows gathered through the dispatch permutation
    static constexpr bool kAMn = MODE == kDownWgrad || MODE == kGateUpWgrad;
    static constexpr bool kBMn = MODE == kDownDgrad || MODE == kGateUpDgrad || MODE == kDownWgrad ||
                                 MODE == kGateUpWgrad;
    // rows staged per (token, slot) for the slot-ordered sum that follows the GEMM
    static constexpr bool kStage = MODE == kDownFwd || MODE == kGateUpDgrad;
    // Epilogue warps per TMEM lane quadrant: the down dgrad's epilogue (h
    // loads, dh stores) is latency bound and splits each tile's columns
    // between two warps; elsewhere one warp takes all of its 32 rows.
    static constexpr int kSplit = MODE == kDownDgrad ? 2 : 1;
    static constexpr int kEpiWarps = 4 * kSplit;
    static constexpr int kGatherWarp0 = kEpiWarp0 + kEpiWarps;  // two more warps: the gather producers
    static constexpr int kThreads = 32 * (kGatherWarp0 + 2);  // the two last warps idle where nothing is gathered
};

// Bytes of one stage that arrive by TMA (the gathered operand arrives by cp.async).
template <int MODE, int BN, bool MX>
__host__ __device__ constexpr uint32_t tma_stage_bytes() {
    return (ModeTraits<MODE>::kGather ? Cfg<BN, MX>::kBBytes : Cfg<BN, MX>::kStageBytes) +
           (MX ? (ModeTraits<MODE>::kGather ? kMxAtomBytes : 2 * kMxAtomBytes) : 0);
}

struct Tile {
    int e;      // expert
    int mt;     // M tile
    int nt;     // N tile
    int nkb;    // K blocks
    int kpos0;  // wgrad: first sorted row of the expert's group
    bool skip;  // CTA-pair gate/up dgrad: this CTA's M tile lies past its expert's group (computed, not stored)
    bool half;  // CTA-pair gate/up forward: an expert's last, unpaired 128-row tile, computed by
                // one M = 128 pair MMA (64 rows per CTA)
    int row0;   // CTA pairs, M-tiled: first sorted row of this CTA's A rows
};

// Wgrad tiles are walked expert by expert, busiest expert first (`order`, a
// per-CTA copy in shared memory), so that long-K tiles are spread evenly.
template <int MODE>
__device__ __forceinline__ Tile decode_tile(int tile, const GemmArgs &a, const int *order) {
    Tile t;
    t.skip = false;
    t.half = false;
    t.row0 = 0;
    if constexpr (ModeTraits<MODE>::kMTiled) {
        t.mt = tile / a.n_tiles;
        t.nt = tile - t.mt * a.n_tiles;
        t.e = __ldg(a.tile_expert + t.mt);
        t.nkb = a.num_k_blocks;
        t.kpos0 = 0;
    } else {
        const int per = a.m_tiles * a.n_tiles;
        const int rank = tile / per;
        const int r = tile - rank * per;
        t.e = order[rank];
        t.mt = r / a.n_tiles;
        t.nt = r - t.mt * a.n_tiles;
        const int gs = __ldg(a.group_start + t.e), ge = __ldg(a.group_start + t.e + 1);
        t.nkb = (ge - gs) / a.k_elems;
        t.kpos0 = gs;
    }
    if (t.e < 0 || t.e >= a.E) {  // corrupted routing state: do no work for this tile
        t.e = 0;
        t.nkb = 0;
    }
    return t;
}

template <int MODE>
__device__ __forceinline__ int total_tiles(const GemmArgs &a) {
    if constexpr (ModeTraits<MODE>::kMTiled) {
        return (__ldg(a.group_start + a.E) / kTileM) * a.n_tiles;
    } else {
        return a.E * a.m_tiles * a.n_tiles;
    }
}

// The i-th tile of CTA (or CTA pair) `first` of `count`.  The M-tiled modes,
// whose tiles all cost the same, deal them round-robin.  The weight
// gradients' tiles come busiest expert first (tiles of one expert cost the
// same, and the cost falls along the list) and are dealt in snake order,
// forwards in even rounds and backwards in odd ones, so that under skewed
// routing every CTA's total stays close to the mean.  A CTA's tiles increase
// with i in both orders.
template <int MODE>
__device__ __forceinline__ int nth_tile(int i, int first, int count) {
    if constexpr (ModeTraits<MODE>::kMTiled) {
        return first + i * count;
    } else {
        return i * count + ((i & 1) ? count - 1 - first : first);
    }
}

// Token row of a sorted position (padding rows read token 0; their products
// are masked or multiplied by zero rows of the other operand).
__device__ __forceinline__ int token_of(const GemmArgs &a, int pos) {
    const int p = __ldg(a.perm + pos);
    if (p < 0 || p >= a.T * a.k) return 0;
    return p / a.k;
}

// Row transposes through a per-warp 32 x 64-byte shared buffer.  Thread r of
// the epilogue owns accumulator row r; a transpose turns its 64-byte piece of
// row r into global accesses where 4 lanes cover one row's 64 contiguous
// bytes (8 rows per instruction).  16-byte pieces are XOR-swizzled by bits
// 1..2 of the row so that neither pass has bank conflicts beyond the minimum.
__device__ __forceinline__ uint32_t xpose_off(int row, int piece) {
    return static_cast<uint32_t>(row * 64 + ((piece ^ ((row >> 1) & 3)) << 4));
}

// Store each lane's 64 bytes v to rowptr (nullptr: that row is skipped).
__device__ __forceinline__ void warp_store_rows(uint8_t *buf, const uint32_t (&v)[16], void *rowptr) {
    const int lane = threadIdx.x & 31;
#pragma unroll
    for (int q = 0; q < 4; ++q)
        *reinterpret_cast<uint4 *>(buf + xpose_off(lane, q)) = make_uint4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
    __syncwarp();
    const int piece = lane & 3;
    const unsigned long long mine = reinterpret_cast<unsigned long long>(rowptr);
#pragma unroll
    for (int rr = 0; rr < 4; ++rr) {
        const int row = rr * 8 + (lane >> 2);
        const uint4 val = *reinterpret_cast<const uint4 *>(buf + xpose_off(row, piece));
        char *dst = reinterpret_cast<char *>(__shfl_sync(0xffffffffu, mine, row));
        if (dst != nullptr) *reinterpret_cast<uint4 *>(dst + piece * 16) = val;
    }
    __syncwarp();
}

// Row loads in two halves, so that a caller can have the next piece's loads
// in flight while it works on the current one: warp_load_issue starts the
// global loads (64 bytes of each lane's row from rowptr; nullptr: zeros),
// warp_load_finish turns them around through the shared buffer.
__device__ __forceinline__ void warp_load_issue(uint4 (&got)[4], const void *rowptr) {
    const int lane = threadIdx.x & 31;
    const int piece = lane & 3;
    const unsigned long long mine = reinterpret_cast<unsigned long long>(rowptr);
#pragma unroll
    for (int rr = 0; rr < 4; ++rr) {
        const int row = rr * 8 + (lane >> 2);
        const char *src = reinterpret_cast<const char *>(__shfl_sync(0xffffffffu, mine, row));
        got[rr] = src != nullptr ? *reinterpret_cast<const uint4 *>(src + piece * 16) : make_uint4(0u, 0u, 0u, 0u);
    }
}

__device__ __forceinline__ void warp_load_finish(uint8_t *buf, const uint4 (&got)[4], uint32_t (&v)[16]) {
    const int lane = threadIdx.x & 31;
    const int piece = lane & 3;
#pragma unroll
    for (int rr = 0; rr < 4; ++rr)
        *reinterpret_cast<uint4 *>(buf + xpose_off(rr * 8 + (lane >> 2), piece)) = got[rr];
    __syncwarp();
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        const uint4 val = *reinterpret_cast<const uint4 *>(buf + xpose_off(lane, q));
        v[4 * q] = val.x;
        v[4 * q + 1] = val.y;
        v[4 * q + 2] = val.z;
        v[4 * q + 3] = val.w;
    }
    __syncwarp();
}

// Warp-uniform bounded wait: lane 0 polls, the verdict is broadcast.
__device__ __forceinline__ bool warp_wait(uint64_t *bar, uint32_t parity, volatile int *abort_flag) {
    int ok = 0;
    if ((threadIdx.x & 31) == 0) ok = mbar_wait(bar, parity, abort_flag) ? 1 : 0;
    return __shfl_sync(0xffffffffu, ok, 0) != 0;
}

__device__ __forceinline__ void raise_abort(volatile int *abort_flag, int *status) {
    *abort_flag = 1;
    report_status(status, kStatusTimeout);
}

// ---------------------------------------------------------------------------
// TMA producer (warp 0): the operand(s) that are not gathered
// ---------------------------------------------------------------------------
template <int MODE, int BN, bool MX>
__device__ void producer_loop(const CUtensorMap *tmA, const CUtensorMap *tmB, const GemmArgs &a, uint8_t *smem,
                              uint64_t *full, uint64_t *empty, const int *order, volatile int *abort_flag) {
    using C = Cfg<BN, MX>;
    const int lane = threadIdx.x & 31;
    const int total = total_tiles<MODE>(a);
    int it = 0;
    bool ok = true;
    for (int i = 0, tile = nth_tile<MODE>(0, blockIdx.x, gridDim.x); tile < total && ok;
         tile = nth_tile<MODE>(++i, blockIdx.x, gridDim.x)) {
        const Tile t = decode_tile<MODE>(tile, a, order);
        for (int kb = 0; kb < t.nkb; ++kb) {
            const int s = it % C::kStages;
            const uint32_t ph = static_cast<uint32_t>(it / C::kStages) & 1u;
            if (!warp_wait(&empty[s], ph ^ 1u, abort_flag)) {
                ok = false;
                break;
            }
            if (lane == 0) mbar_arrive_expect_tx(&full[s], tma_stage_bytes<MODE, BN, MX>());
            __syncwarp();
            uint8_t *As = smem + s * C::kStageBytes;
            uint8_t *Bs = As + kABytes;
            const int k0 = kb * C::kKElems;
            if constexpr (MX) {
                // E4M3 operands (one 128 x 128-byte box each) and their scale atoms
                uint8_t *sfs = smem + C::kSfOffset + s * C::kSfBytes;  // [A atom | B atom]
                const int64_t kblk = kb;                               // K block of 128
                if (lane == 0) {
                    if constexpr (MODE == kGateUpFwd) {
                        const int row = t.e * 2 * a.I + t.nt * 64;
                        tma_load_2d(Bs, tmB, &full[s], k0, row);                   // 64 gate rows
                        tma_load_2d(Bs + 64 * 128, tmB, &full[s], k0, row + a.I);  // 64 up rows
                        bulk_load(sfs + kMxAtomBytes,
                                  a.sfb + ((static_cast<int64_t>(t.e) * (a.I / 64) + t.nt) * (a.d / 128) + kblk) * kMxAtomBytes,
                                  kMxAtomBytes, &full[s]);
                    } else if constexpr (MODE == kDownFwd) {
                        tma_load_2d(As, tmA, &full[s], k0, t.mt * kTileM);
                        tma_load_2d(Bs, tmB, &full[s], k0, t.e * a.d + t.nt * 128);
                        bulk_load(sfs, a.sfa + (static_cast<int64_t>(t.mt) * (a.I / 128) + kblk) * kMxAtomBytes,
                                  kMxAtomBytes, &full[s]);
                        bulk_load(sfs + kMxAtomBytes,
                                  a.sfb + ((static_cast<int64_t>(t.e) * a.d + t.nt * 128) / 128 * (a.I / 128) + kblk) * kMxAtomBytes,
                                  kMxAtomBytes, &full[s]);
                    } else if constexpr (MODE == kDownDgrad) {
                        tma_load_2d(As, tmA, &full[s], k0, t.mt * kTileM);
                        tma_load_2d(Bs, tmB, &full[s], t.nt * 128, t.e * a.d + k0);
                        bulk_load(sfs, a.sfa + (static_cast<int64_t>(t.mt) * (a.d / 128) + kblk) * kMxAtomBytes,
                                  kMxAtomBytes, &full[s]);
                        bulk_load(sfs + kMxAtomBytes,
                                  a.sfb + ((static_cast<int64_t>(t.e) * a.d + k0) / 128 * (a.I / 128) + t.nt) * kMxAtomBytes,
                                  kMxAtomBytes, &full[s]);
                    } else if constexpr (MODE == kGateUpDgrad) {
                        tma_load_2d(As, tmA, &full[s], k0, t.mt * kTileM);
                        tma_load_2d(Bs, tmB, &full[s], t.nt * 128, t.e * 2 * a.I + k0);
                        bulk_load(sfs, a.sfa + (static_cast<int64_t>(t.mt) * (2 * a.I / 128) + kblk) * kMxAtomBytes,
                                  kMxAtomBytes, &full[s]);
                        bulk_load(sfs + kMxAtomBytes,
                                  a.sfb + ((static_cast<int64_t>(t.e) * 2 * a.I + k0) / 128 * (a.d / 128) + t.nt) * kMxAtomBytes,
                                  kMxAtomBytes, &full[s]);
                    } else {  // wgrads: K = the expert's sorted rows, both operands MN-major
                        const int64_t kr = (static_cast<int64_t>(t.kpos0) + k0) / 128;
                        const int mw = MODE == kDownWgrad ? a.d / 128 : 2 * a.I / 128;  // M extent in 128-blocks
                        const int nw = MODE == kDownWgrad ? a.I / 128 : a.d / 128;      // N extent in 128-blocks
                        tma_load_2d(As, tmA, &full[s], t.mt * kTileM, t.kpos0 + k0);
                        tma_load_2d(Bs, tmB, &full[s], t.nt * 128, t.kpos0 + k0);
                        bulk_load(sfs, a.sfa + (kr * mw + t.mt) * kMxAtomBytes, kMxAtomBytes, &full[s]);
                        bulk_load(sfs + kMxAtomBytes, a.sfb + (kr * nw + t.nt) * kMxAtomBytes, kMxAtomBytes, &full[s]);
                    }
                }
            } else if constexpr (MODE == kGateUpFwd) {
                if (lane == 0) {
                    const int row = t.e * 2 * a.I + t.nt * (BN / 2);
                    tma_load_2d(Bs, tmB, &full[s], k0, row);                         // gate rows
                    tma_load_2d(Bs + (BN / 2) * 128, tmB, &full[s], k0, row + a.I);  // up rows
                }
            } else if constexpr (MODE == kDownFwd) {
                if (lane == 0) {
                    tma_load_2d(As, tmA, &full[s], k0, t.mt * kTileM);
                    tma_load_2d(Bs, tmB, &full[s], k0, t.e * a.d + t.nt * BN);
                }
            } else if constexpr (MODE == kDownDgrad) {
                if (lane == 0) tma_load_2d(As, tmA, &full[s], k0, t.mt * kTileM);  // sorted grad_out rows
                if (lane < BN / 64)
                    tma_load_2d(Bs + lane * kChunkBytes, tmB, &full[s], t.nt * BN + 64 * lane, t.e * a.d + k0);
            } else if constexpr (MODE == kGateUpDgrad) {
                if (lane == 0) tma_load_2d(As, tmA, &full[s], k0, t.mt * kTileM);
                if (lane < BN / 64)
                    tma_load_2d(Bs + lane * kChunkBytes, tmB, &full[s], t.nt * BN + 64 * lane, t.e * 2 * a.I + k0);
            } else if constexpr (MODE == kDownWgrad) {
                if (lane < 2)  // sorted grad_out rows, MN-major
                    tma_load_2d(As + lane * kChunkBytes, tmA, &full[s], t.mt * kTileM + 64 * lane, t.kpos0 + k0);
                if (lane >= 2 && lane < 2 + BN / 64)
                    tma_load_2d(Bs + (lane - 2) * kChunkBytes, tmB, &full[s], t.nt * BN + 64 * (lane - 2), t.kpos0 + k0);
            } else {  // kGateUpWgrad
                if (lane < 2)
                    tma_load_2d(As + lane * kChunkBytes, tmA, &full[s], t.mt * kTileM + 64 * lane, t.kpos0 + k0);
                if (lane >= 2 && lane < 2 + BN / 64)  // sorted x rows, MN-major
                    tma_load_2d(Bs + (lane - 2) * kChunkBytes, tmB, &full[s], t.nt * BN + 64 * (lane - 2), t.kpos0 + k0);
            }
            ++it;
        }
    }
    if (!ok) {
        raise_abort(abort_flag, a.status);
        // let the copies already issued land before the CTA can exit
        if (lane == 0) {
            for (int i = it > C::kStages ? it - C::kStages : 0; i < it; ++i)
                mbar_wait(&full[i % C::kStages], static_cast<uint32_t>(i / C::kStages) & 1u, nullptr);
        }
        __syncwarp();
    }
}

// ---------------------------------------------------------------------------
// gather producers (warps 6, 7): token rows through the dispatch permutation
// ---------------------------------------------------------------------------
// Thread g (0..63) copies 16-byte piece (g & 7) of the 128-byte rows
// r = (g >> 3) + 8 i.  A row r of a 128-byte-swizzled stage lives at byte
// r * 128, with its 16-byte piece c stored at position c ^ (r & 7).
template <int MODE, int BN, bool MX>
__device__ void gather_loop(const GemmArgs &a, uint8_t *smem, uint64_t *full, uint64_t *empty, const int *order,
                            volatile int *abort_flag) {
    using C = Cfg<BN, MX>;
    const int g = threadIdx.x - ModeTraits<MODE>::kGatherWarp0 * 32;
    const int piece = g & 7;
    const int rg = g >> 3;
    const size_t row_bytes = static_cast<size_t>(a.d) * (MX ? 1 : 2);  // E4M3 codes or bf16
    const uint8_t *src = static_cast<const uint8_t *>(a.gsrc);
    const int total = total_tiles<MODE>(a);
    int it = 0;
    bool ok = true;
    // 16 rows of the 128-row tile per thread; K-major, one 128-byte row piece per K block.
    // MXFP8: the 8 piece-0 threads also copy each row's 4 scale bytes of the K block
    // into the A scale atom of the stage.
    int tok[16], nxt[16];
    int tile = blockIdx.x;
    if (tile < total) {
        const int mt = tile / a.n_tiles;
#pragma unroll
        for (int i = 0; i < 16; ++i) tok[i] = token_of(a, mt * kTileM + rg + 8 * i);
    }
    for (; tile < total && ok; tile += gridDim.x) {
        const Tile t = decode_tile<MODE>(tile, a, order);
        const int next = tile + gridDim.x;
        if (next < total) {  // prefetch the next tile's token rows
            const int mt = next / a.n_tiles;
#pragma unroll
            for (int i = 0; i < 16; ++i) nxt[i] = token_of(a, mt * kTileM + rg + 8 * i);
        }
        const uint8_t *rows[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) rows[i] = src + static_cast<size_t>(tok[i]) * row_bytes + piece * 16;
        for (int kb = 0; kb < t.nkb; ++kb) {
            const int s = it % C::kStages;
            const uint32_t ph = static_cast<uint32_t>(it / C::kStages) & 1u;
            if (!warp_wait(&empty[s], ph ^ 1u, abort_flag)) {
                ok = false;
                break;
            }
            const uint32_t As = smem_u32(smem + s * C::kStageBytes);
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                const int r = rg + 8 * i;
                cp_async_16(As + r * 128 + ((piece ^ (r & 7)) << 4), rows[i] + kb * 128);
            }
            if constexpr (MX) {
                if (piece == 0) {
                    const uint32_t sfa = smem_u32(smem + C::kSfOffset + s * C::kSfBytes);
#pragma unroll
                    for (int i = 0; i < 16; ++i) {
                        const int r = rg + 8 * i;
                        cp_async_4(sfa + mx_atom_byte(r, 0), a.gsf + static_cast<size_t>(tok[i]) * (a.d / kMxBlock) + kb * 4);
                    }
                }
            }
            cp_async_arrive_noinc(&full[s]);
            ++it;
        }
#pragma unroll
        for (int i = 0; i < 16; ++i) tok[i] = nxt[i];
    }
    if (!ok) raise_abort(abort_flag, a.status);
    cp_async_wait_all();  // our copies land before the CTA can exit
}

// ---------------------------------------------------------------------------
// MMA issuer (warp 1, one thread)
// ---------------------------------------------------------------------------
template <int MODE, int BN, bool MX>
__device__ void mma_loop(const GemmArgs &a, uint8_t *smem, uint64_t *full, uint64_t *empty, uint64_t *tfull,
                         uint64_t *tempty, uint64_t *drain, uint32_t tmem_base, const int *order,
                         volatile int *abort_flag) {
    using C = Cfg<BN, MX>;
    using TR = ModeTraits<MODE>;
    constexpr uint32_t kIdesc = instr_desc_bf16(kTileM, BN, TR::kAMn, TR::kBMn);
    const int total = total_tiles<MODE>(a);
    int it = 0, local = 0;
    bool ok = true;
    for (int tile = nth_tile<MODE>(0, blockIdx.x, gridDim.x); tile < total && ok;
         tile = nth_tile<MODE>(++local, blockIdx.x, gridDim.x)) {
        const Tile t = decode_tile<MODE>(tile, a, order);
        const int acc = local & 1;
        const uint32_t aph = static_cast<uint32_t>(local >> 1) & 1u;
        if (!mbar_wait(&tempty[acc], aph ^ 1u, abort_flag)) {
            ok = false;
            break;
        }
        tc_fence_after_sync();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * BN);
        for (int kb = 0; kb < t.nkb; ++kb, ++it) {
            const int s = it % C::kStages;
            const uint32_t ph = static_cast<uint32_t>(it / C::kStages) & 1u;
            if (!mbar_wait(&full[s], ph, abort_flag)) {
                ok = false;
                break;
            }
            if constexpr (TR::kGather) fence_proxy_async_smem();  // cp.async data -> tensor-core reads
            tc_fence_after_sync();
            const uint32_t a_base = smem_u32(smem + s * C::kStageBytes);
            const uint32_t b_base = a_base + kABytes;
            if constexpr (MX) {
                // scale atoms -> tensor memory (ordered before the MMAs that read them),
                // then four K=32 block-scaled MMAs; sf_id k picks scale byte k
                const uint32_t sf_base = smem_u32(smem + C::kSfOffset + s * C::kSfBytes);
                // the scale columns follow the two accumulators
                const uint32_t sfa_t = tmem_base + 2u * BN, sfb_t = tmem_base + 2u * BN + 8u;
                tmem_copy_32x128b_x4(sfa_t, smem_desc_plain(sf_base, 128));
                tmem_copy_32x128b_x4(sfb_t, smem_desc_plain(sf_base + kMxAtomBytes, 128));
#pragma unroll
                for (int kk = 0; kk < 4; ++kk) {
                    const uint64_t ad = TR::kAMn ? smem_desc_sw128(a_base + kk * 4096, 16384, kSbo)
                                                 : smem_desc_sw128(a_base + kk * 32, 16, kSbo);
                    const uint64_t bd = TR::kBMn ? smem_desc_sw128(b_base + kk * 4096, 16384, kSbo)
                                                 : smem_desc_sw128(b_base + kk * 32, 16, kSbo);
                    mma_mxf8(d_tmem, ad, bd, instr_desc_mxf8(kTileM, BN, TR::kAMn, TR::kBMn, kk),
                             sfa_t | (static_cast<uint32_t>(kk) << 30), sfb_t | (static_cast<uint32_t>(kk) << 30),
                             (kb | kk) != 0 ? 1u : 0u);
                }
            } else {
#pragma unroll
                for (int kk = 0; kk < kTileK / 16; ++kk) {
                    const uint64_t ad = TR::kAMn ? smem_desc_sw128(a_base + kk * 2048, kMnLbo, kSbo)
                                                 : smem_desc_sw128(a_base + kk * 32, 16, kSbo);
                    const uint64_t bd = TR::kBMn ? smem_desc_sw128(b_base + kk * 2048, kMnLbo, kSbo)
                                                 : smem_desc_sw128(b_base + kk * 32, 16, kSbo);
                    mma_bf16(d_tmem, ad, bd, kIdesc, (kb | kk) != 0 ? 1u : 0u);
                }
            }
            mma_commit(&empty[s]);  // frees the stage once these MMAs have read it
        }
        if (!ok) break;
        mma_commit(&tfull[acc]);
    }
    if (!ok) {
        raise_abort(abort_flag, a.status);
        mma_commit(drain);
        mbar_wait(drain, 0u, nullptr);
    }
}

// ---------------------------------------------------------------------------
// epilogues (warps 2..5; thread = one accumulator row)
// ---------------------------------------------------------------------------
__device__ __forceinline__ void release_accumulator(uint64_t *tempty_acc) {
    tc_fence_before_sync();
    __syncwarp();
    if ((threadIdx.x & 31) == 0) mbar_arrive(tempty_acc);
}

// CTA pairs: the accumulator barrier is the leader's, whichever CTA releases.
template <bool PAIR>
__device__ __forceinline__ void release_acc(uint64_t *tempty_acc) {
    if constexpr (PAIR) {
        tc_fence_before_sync();
        __syncwarp();
        if ((threadIdx.x & 31) == 0) mbar_arrive_cluster(cluster_addr(tempty_acc, 0));
    } else {
        release_accumulator(tempty_acc);
    }
}

// One 32-column chunk of this warp's accumulator rows (fp32 in registers) as
// bf16 to row (nullptr: skipped).
__device__ __forceinline__ void store_chunk_bf16(uint8_t *xbuf, const uint32_t (&v)[32], __nv_bfloat16 *row) {
    uint32_t pv[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) pv[i] = pack_bf16x2(__uint_as_float(v[2 * i]), __uint_as_float(v[2 * i + 1]));
    warp_store_rows(xbuf, pv, row);
}

// This lane's 64 bytes of packed bf16 (row = lane) into buf in the 64-byte
// swizzle of the TMA stores (the caller fences and issues the store).
__device__ __forceinline__ void put_row_swz64(uint8_t *buf, const uint32_t (&pv)[16]) {
    const int lane = threadIdx.x & 31;
#pragma unroll
    for (int q = 0; q < 4; ++q)
        *reinterpret_cast<uint4 *>(buf + xpose_off(lane, q)) =
            make_uint4(pv[4 * q], pv[4 * q + 1], pv[4 * q + 2], pv[4 * q + 3]);
}

// store_accumulator_bf16 with TMA stores: this warp's 32 rows of the tile go to
// rows y .. y + 31 and columns x0 .. x0 + BN - 1 of the tensor behind `map`
// (boxes of 32 rows x 64 columns, 128-byte swizzle), 64 columns at a time from
// one 4 KB buffer at xbuf: the two 32-column chunks of a box are loaded from
// tensor memory together, packed, and written to the buffer once the previous
// box's store has read it; one proxy fence and one store per box.
template <int BN, bool PAIR>
__device__ __forceinline__ void store_accumulator_tma(uint32_t taddr, uint8_t *xbuf, const CUtensorMap *map, int x0,
                                                      int y, uint64_t *tempty_acc) {
    static_assert((BN / 32) % 2 == 0, "whole 64-column boxes");
    const int lane = threadIdx.x & 31;
    uint32_t ra[32], rb[32];
    tmem_load32(taddr, ra);
    tmem_load32(taddr + 32, rb);
    tmem_load_wait();
    tmem_regs_ready(ra);
    tmem_regs_ready(rb);
#pragma unroll
    for (int c = 0; c < BN / 32; c += 2) {
        uint32_t pv[32];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            pv[i] = pack_bf16x2(__uint_as_float(ra[2 * i]), __uint_as_float(ra[2 * i + 1]));
            pv[16 + i] = pack_bf16x2(__uint_as_float(rb[2 * i]), __uint_as_float(rb[2 * i + 1]));
        }
        if (c + 2 < BN / 32) {
            tmem_load32(taddr + (c + 2) * 32, ra);
            tmem_load32(taddr + (c + 3) * 32, rb);
        } else {
            release_acc<PAIR>(tempty_acc);
        }
        if (lane == 0) bulk_wait_read<0>();
        __syncwarp();
#pragma unroll
        for (int q = 0; q < 8; ++q)  // 128-byte swizzle: 16-byte piece q of row `lane` at piece q ^ (lane & 7)
            *reinterpret_cast<uint4 *>(xbuf + lane * 128 + ((q ^ (lane & 7)) << 4)) =
                make_uint4(pv[4 * q], pv[4 * q + 1], pv[4 * q + 2], pv[4 * q + 3]);
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
            tma_store_2d(map, xbuf, x0 + c * 32, y);
            bulk_commit();
        }
        if (c + 2 < BN / 32) {
            tmem_load_wait();
            tmem_regs_ready(ra);
            tmem_regs_ready(rb);
        }
    }
}

// Streams this warp's 32 accumulator rows (BN fp32 columns) to bf16 rows at
// row (nullptr: skipped), 32 columns at a time, with the tensor-memory load of
// chunk c + 1 in flight while chunk c is converted and stored.  Releases the
// accumulator as soon as its last chunk is in registers.
template <int BN, bool PAIR = false>
__device__ __forceinline__ void store_accumulator_bf16(uint32_t taddr, uint8_t *xbuf, __nv_bfloat16 *row,
                                                       uint64_t *tempty_acc) {
    uint32_t ra[32], rb[32];
    tmem_load32(taddr, ra);
    tmem_load_wait();
    tmem_regs_ready(ra);
#pragma unroll
    for (int c = 0; c < BN / 32; c += 2) {
        tmem_load32(taddr + (c + 1) * 32, rb);
        store_chunk_bf16(xbuf, ra, row != nullptr ? row + c * 32 : nullptr);
        tmem_load_wait();
        tmem_regs_ready(rb);
        if (c + 2 < BN / 32)
            tmem_load32(taddr + (c + 2) * 32, ra);
        else
            release_acc<PAIR>(tempty_acc);
        store_chunk_bf16(xbuf, rb, row != nullptr ? row + (c + 1) * 32 : nullptr);
        if (c + 2 < BN / 32) {
            tmem_load_wait();
            tmem_regs_ready(ra);
        }
    }
}

// gate/up forward: SwiGLU; writes h (gate, up) and aw = w * silu(gate) * up,
// or with the clamped SwiGLU aw = w * silu(min(gate, L)) * clamp(up, -L, L)
// (a.limit = L; +inf leaves gate and up unchanged, bit for bit).
// MXFP8: also aw's E4M3 codes and scale atoms along I (the down GEMM's K).
// One 32-column chunk c of gate (gr) and up (ur) accumulator values.
// The SwiGLU of one 32-column chunk: gate and up as bf16 pairs (pg, pu) and
// aw = w * silu(gate) * up, in fp32 (av) and as bf16 pairs (pa).
__device__ __forceinline__ void gateup_math(const GemmArgs &a, bool valid, float wv, const uint32_t (&gr)[32],
                                            const uint32_t (&ur)[32], uint32_t (&pg)[16], uint32_t (&pu)[16],
                                            uint32_t (&pa)[16], float (&av)[32]) {
#pragma unroll
    for (int i = 0; i < 32; ++i) {
        const float g = fminf(__uint_as_float(gr[i]), a.limit);
        const float u = fminf(fmaxf(__uint_as_float(ur[i]), -a.limit), a.limit);
        av[i] = valid ? wv * g * __fdividef(1.f, 1.f + __expf(-g)) * u : 0.f;
    }
#pragma unroll
    for (int i = 0; i < 16; ++i) {
        pg[i] = valid ? pack_bf16x2(__uint_as_float(gr[2 * i]), __uint_as_float(gr[2 * i + 1])) : 0u;
        pu[i] = valid ? pack_bf16x2(__uint_as_float(ur[2 * i]), __uint_as_float(ur[2 * i + 1])) : 0u;
        pa[i] = pack_bf16x2(av[2 * i], av[2 * i + 1]);
    }
}

template <int BN, bool MX>
__device__ __forceinline__ void gateup_chunk(const GemmArgs &a, const Tile &t, int r, int pos, bool valid, float wv,
                                             int c, const uint32_t (&gr)[32], const uint32_t (&ur)[32],
                                             __nv_bfloat16 *hrow, __nv_bfloat16 *arow, uint8_t *xbuf) {
    constexpr int kHalf = BN / 2;
    uint32_t pg[16], pu[16], pa[16];
    float av[32];
    gateup_math(a, valid, wv, gr, ur, pg, pu, pa, av);
    warp_store_rows(xbuf, pg, hrow + c * 32);
    warp_store_rows(xbuf, pu, hrow + a.I + c * 32);
    warp_store_rows(xbuf, pa, arow + c * 32);
    if constexpr (MX) {
        const int col = t.nt * kHalf + c * 32;
        const int sc = mx_scale_exp(amax32(av));
        uint32_t codes[8];
        mx_encode32(av, sc, codes);
        uint4 *dst = reinterpret_cast<uint4 *>(a.mx_codes + static_cast<size_t>(pos) * a.I + col);
        dst[0] = make_uint4(codes[0], codes[1], codes[2], codes[3]);
        dst[1] = make_uint4(codes[4], codes[5], codes[6], codes[7]);
        const int64_t atom = static_cast<int64_t>(t.mt) * (a.I / 128) + col / 128;
        a.mx_sf[atom * kMxAtomBytes + mx_atom_byte(r, col / 32)] = static_cast<uint8_t>(sc + 127);
    }
}

// The tensor-memory loads of chunk c + 1 are in flight while chunk c is worked on.
template <int BN, bool MX, bool PAIR = false>
__device__ __forceinline__ void epi_gateup_fwd(const GemmArgs &a, const Tile &t, int r, uint32_t taddr,
                                               uint64_t *tempty_acc, uint8_t *xbuf) {
    constexpr int kHalf = BN / 2;
    constexpr int kChunks = kHalf / 32;
    static_assert(kChunks % 2 == 0, "chunks are taken in pairs");
    const int pos = t.mt * kTileM + r;
    const int p = __ldg(a.perm + pos);
    const bool valid = p >= 0 && p < a.T * a.k;
    const float wv = valid ? __ldg(a.topk_w + p) : 0.f;
    __nv_bfloat16 *hrow = a.h + static_cast<size_t>(pos) * 2 * a.I + t.nt * kHalf;
    __nv_bfloat16 *arow = a.aw + static_cast<size_t>(pos) * a.I + t.nt * kHalf;
    uint32_t ga[32], ua[32], gb[32], ub[32];
    tmem_load32(taddr, ga);
    tmem_load32(taddr + kHalf, ua);
    tmem_load_wait();
    tmem_regs_ready(ga);
    tmem_regs_ready(ua);
#pragma unroll
    for (int c = 0; c < kChunks; c += 2) {
        tmem_load32(taddr + (c + 1) * 32, gb);
        tmem_load32(taddr + kHalf + (c + 1) * 32, ub);
        gateup_chunk<BN, MX>(a, t, r, pos, valid, wv, c, ga, ua, hrow, arow, xbuf);
        tmem_load_wait();
        tmem_regs_ready(gb);
        tmem_regs_ready(ub);
        if (c + 2 < kChunks) {
            tmem_load32(taddr + (c + 2) * 32, ga);
            tmem_load32(taddr + kHalf + (c + 2) * 32, ua);
        } else {
            release_acc<PAIR>(tempty_acc);  // TMEM no longer needed
        }
        gateup_chunk<BN, MX>(a, t, r, pos, valid, wv, c + 1, gb, ub, hrow, arow, xbuf);
        if (c + 2 < kChunks) {
            tmem_load_wait();
            tmem_regs_ready(ga);
            tmem_regs_ready(ua);
        }
    }
}

// down forward / gate-up dgrad: this CTA's rows of the tile, rounded to bf16, to
// the staging row of their (token, slot) pair; the slot-ordered sum over a
// token's k staged rows runs as its own bandwidth-bound kernel afterwards
// (combine_rows).  Padding rows store nothing.
template <int BN, bool PAIR = false>
__device__ __forceinline__ void epi_stage(const GemmArgs &a, const Tile &t, int r, uint32_t taddr,
                                          uint64_t *tempty_acc, uint8_t *xbuf) {
    const int pos = t.mt * kTileM + r;
    const int p = __ldg(a.perm + pos);
    const bool valid = p >= 0 && p < a.T * a.k;
    __nv_bfloat16 *srow = valid ? a.stage + static_cast<size_t>(p) * a.d + t.nt * BN : nullptr;
    store_accumulator_bf16<BN, PAIR>(taddr, xbuf, srow, tempty_acc);
}

// down dgrad: G = W_down^T gout; dscore partial <G, a>; SwiGLU backward -> dh
// (clamped SwiGLU: gate and up clamped as in the forward, and each clamp stops
// its gradient where h lies outside its interval).
// MXFP8: also dh's E4M3 codes and scale atoms along 2I (the gate/up dgrad's K).
template <int BN, bool MX>
__device__ __forceinline__ void epi_down_dgrad(const GemmArgs &a, const Tile &t, int r, int ch, uint32_t taddr,
                                               uint64_t *tempty_acc, uint8_t *xbuf) {
    const int pos = t.mt * kTileM + r;
    const int p = __ldg(a.perm + pos);
    const bool valid = p >= 0 && p < a.T * a.k;
    const float wv = valid ? __ldg(a.topk_w + p) : 0.f;
    const __nv_bfloat16 *hrow = a.h + static_cast<size_t>(pos) * 2 * a.I + t.nt * BN;
    __nv_bfloat16 *dhrow = a.dh + static_cast<size_t>(pos) * 2 * a.I + t.nt * BN;
    float ds = 0.f;
    constexpr int kSplit = ModeTraits<kDownDgrad>::kSplit;  // epilogue warps per row
    constexpr int kMine = BN / 32 / kSplit;                  // 32-column chunks per epilogue warp
#pragma unroll 1
    for (int c = ch * kMine; c < (ch + 1) * kMine; ++c) {
        uint32_t hg[16], hu[16];
        uint4 cg[4], cu[4];
        warp_load_issue(cg, valid ? hrow + c * 32 : nullptr);
        warp_load_issue(cu, valid ? hrow + a.I + c * 32 : nullptr);
        warp_load_finish(xbuf, cg, hg);
        warp_load_finish(xbuf, cu, hu);
        float G[32];
        tmem_load32_sync(taddr + c * 32, G);
        if (c + 1 == (ch + 1) * kMine) release_accumulator(tempty_acc);
        float dg[32], du[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) {
            const float g0 = (i & 1) ? bf16_hi(hg[i >> 1]) : bf16_lo(hg[i >> 1]);
            const float u0 = (i & 1) ? bf16_hi(hu[i >> 1]) : bf16_lo(hu[i >> 1]);
            const float g = fminf(g0, a.limit), u = fminf(fmaxf(u0, -a.limit), a.limit);
            const float gr = G[i];
            const float sg = __fdividef(1.f, 1.f + __expf(-g));
            const float sl = g * sg;
            ds += gr * (sl * u);
            const float da = wv * gr;
            dg[i] = valid && g0 <= a.limit ? da * u * sg * (1.f + g * (1.f - sg)) : 0.f;
            du[i] = valid && fabsf(u0) <= a.limit ? da * sl : 0.f;
        }
        uint32_t pdg[16], pdu[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            pdg[i] = pack_bf16x2(dg[2 * i], dg[2 * i + 1]);
            pdu[i] = pack_bf16x2(du[2 * i], du[2 * i + 1]);
        }
        warp_store_rows(xbuf, pdg, dhrow + c * 32);
        warp_store_rows(xbuf, pdu, dhrow + a.I + c * 32);
        if constexpr (MX) {
#pragma unroll
            for (int half = 0; half < 2; ++half) {
                const int col = (half ? a.I : 0) + t.nt * BN + c * 32;
                const int sc = mx_scale_exp(amax32(half ? du : dg));
                uint32_t codes[8];
                mx_encode32(half ? du : dg, sc, codes);
                uint4 *dst = reinterpret_cast<uint4 *>(a.mx_codes + static_cast<size_t>(pos) * 2 * a.I + col);
                dst[0] = make_uint4(codes[0], codes[1], codes[2], codes[3]);
                dst[1] = make_uint4(codes[4], codes[5], codes[6], codes[7]);
                const int64_t atom = static_cast<int64_t>(t.mt) * (2 * a.I / 128) + col / 128;
                a.mx_sf[atom * kMxAtomBytes + mx_atom_byte(r, col / 32)] = static_cast<uint8_t>(sc + 127);
            }
        }
    }
    a.dpart[static_cast<size_t>(pos) * a.dpart_stride + kSplit * t.nt + ch] = valid ? ds : 0.f;
}

// Store each lane's 32 bytes v (16 bf16) to rowptr (nullptr: that row is
// skipped) through the warp's shared buffer: a store instruction then covers
// 16 rows x 32 contiguous bytes.  16-byte pieces are XOR-swizzled by bit 2 of
// the row (no bank conflicts beyond the minimum in either pass).
__device__ __forceinline__ uint32_t xpose16_off(int row, int piece) {
    return static_cast<uint32_t>(row * 32 + ((piece ^ ((row >> 2) & 1)) << 4));
}

__device__ __forceinline__ void warp_store_rows16(uint8_t *buf, const uint32_t (&v)[8], void *rowptr) {
    const int lane = threadIdx.x & 31;
#pragma unroll
    for (int q = 0; q < 2; ++q)
        *reinterpret_cast<uint4 *>(buf + xpose16_off(lane, q)) = make_uint4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
    __syncwarp();
    const int piece = lane & 1;
    const unsigned long long mine = reinterpret_cast<unsigned long long>(rowptr);
#pragma unroll
    for (int rr = 0; rr < 2; ++rr) {
        const int row = rr * 16 + (lane >> 1);
        const uint4 val = *reinterpret_cast<const uint4 *>(buf + xpose16_off(row, piece));
        char *dst = reinterpret_cast<char *>(__shfl_sync(0xffffffffu, mine, row));
        if (dst != nullptr) *reinterpret_cast<uint4 *>(dst + piece * 16) = val;
    }
    __syncwarp();
}

// Down dgrad on CTA pairs (BN = 256).  The h values of chunk c -- gate and up
// columns nt * 256 + c * 32 .. +32 of this CTA's 128 rows -- arrive in ring
// slot hit & 1: two TMA boxes of 128 rows x 64 bytes with the 64-byte swizzle
// (16-byte piece q of row r at piece q ^ ((r >> 1) & 3)), loaded by the h
// loader warp one chunk ahead.  The two warps of a tensor-memory lane quadrant
// take 16 columns of each chunk each (ch).  Same arithmetic as
// epi_down_dgrad; dpart gets one partial per (row, n tile, ch).  Returns false
// when a bounded wait expired.
__device__ __forceinline__ bool epi_down_dgrad_ring(const GemmArgs &a, const Tile &t, int r, int ch, uint32_t taddr,
                                                    uint64_t *tempty_acc, uint8_t *xbuf, const uint8_t *ring,
                                                    uint64_t *hfull, uint64_t *hempty, int &hit,
                                                    volatile int *abort_flag) {
    constexpr int BN = 256;
    constexpr int kSlot = 2 * kTileM * 32 * 2;
    constexpr int kSplit = ModeTraits<kDownDgrad>::kSplit;
    const int lane = threadIdx.x & 31;
    const int pos = t.row0 + r;
    const int p = __ldg(a.perm + pos);
    const bool valid = p >= 0 && p < a.T * a.k;
    const float wv = valid ? __ldg(a.topk_w + p) : 0.f;
    __nv_bfloat16 *dhrow = a.dh + static_cast<size_t>(pos) * 2 * a.I + t.nt * BN;
    const int sw = (r >> 1) & 3;
    float ds = 0.f;
#pragma unroll 1
    for (int c = 0; c < BN / 32; ++c, ++hit) {
        const int slot = hit & 1;
        if (!warp_wait(&hfull[slot], static_cast<uint32_t>(hit >> 1) & 1u, abort_flag)) return false;
        const uint8_t *gbox = ring + slot * kSlot;
        const uint8_t *ubox = gbox + kSlot / 2;
        uint32_t hg[8], hu[8];
#pragma unroll
        for (int q = 0; q < 2; ++q) {
            const uint32_t off = static_cast<uint32_t>(r * 64 + (((2 * ch + q) ^ sw) << 4));
            const uint4 g = *reinterpret_cast<const uint4 *>(gbox + off);
            const uint4 u = *reinterpret_cast<const uint4 *>(ubox + off);
            hg[4 * q] = g.x; hg[4 * q + 1] = g.y; hg[4 * q + 2] = g.z; hg[4 * q + 3] = g.w;
            hu[4 * q] = u.x; hu[4 * q + 1] = u.y; hu[4 * q + 2] = u.z; hu[4 * q + 3] = u.w;
        }
        float G[16];
        tmem_load16_sync(taddr + c * 32 + ch * 16, G);
        if (c + 1 == BN / 32) release_acc<true>(tempty_acc);  // tensor memory no longer needed
        __syncwarp();
        if (lane == 0) mbar_arrive(&hempty[slot]);  // this warp is done with the slot
        float dg[16], du[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            const float g0 = (i & 1) ? bf16_hi(hg[i >> 1]) : bf16_lo(hg[i >> 1]);
            const float u0 = (i & 1) ? bf16_hi(hu[i >> 1]) : bf16_lo(hu[i >> 1]);
            const float g = fminf(g0, a.limit), u = fminf(fmaxf(u0, -a.limit), a.limit);
            const float gr = G[i];
            const float sg = __fdividef(1.f, 1.f + __expf(-g));
            const float sl = g * sg;
            ds += gr * (sl * u);
            const float da = wv * gr;
            dg[i] = valid && g0 <= a.limit ? da * u * sg * (1.f + g * (1.f - sg)) : 0.f;
            du[i] = valid && fabsf(u0) <= a.limit ? da * sl : 0.f;
        }
        uint32_t pdg[8], pdu[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            pdg[i] = pack_bf16x2(dg[2 * i], dg[2 * i + 1]);
            pdu[i] = pack_bf16x2(du[2 * i], du[2 * i + 1]);
        }
        warp_store_rows16(xbuf, pdg, dhrow + c * 32 + ch * 16);
        warp_store_rows16(xbuf, pdu, dhrow + a.I + c * 32 + ch * 16);
    }
    a.dpart[static_cast<size_t>(pos) * a.dpart_stride + kSplit * t.nt + ch] = valid ? ds : 0.f;
    return true;
}

// weight gradients: store the tile (zeros for an expert without tokens).
// With dw_map (CTA pairs) the tile goes out by TMA stores of the dW rows
// [E * Mtot, Ntot] (32 x 64 boxes) from the warp's 4 KB buffer at xbuf;
// otherwise by the transposes, row by row.
template <int MODE, int BN, bool PAIR = false>
__device__ __forceinline__ void epi_wgrad(const GemmArgs &a, const Tile &t, int r, uint32_t taddr,
                                          uint64_t *tempty_acc, uint8_t *xbuf, const CUtensorMap *dw_map = nullptr) {
    const int Mtot = MODE == kDownWgrad ? a.d : 2 * a.I;
    const int Ntot = MODE == kDownWgrad ? a.I : a.d;
    constexpr int BH = BN;
    __nv_bfloat16 *row = a.dw + (static_cast<size_t>(t.e) * Mtot + t.mt * kTileM + r) * static_cast<size_t>(Ntot) +
                         t.nt * BN;
    if (t.nkb > 0) {
        if (dw_map != nullptr)
            store_accumulator_tma<BH, PAIR>(taddr, xbuf, dw_map, t.nt * BN, t.e * Mtot + t.mt * kTileM + (r & ~31),
                                            tempty_acc);
        else
            store_accumulator_bf16<BH, PAIR>(taddr, xbuf, row, tempty_acc);
        return;
    }
    release_acc<PAIR>(tempty_acc);  // an expert without tokens: exact zeros, the accumulator is not read
    if (dw_map != nullptr) {  // the first buffer is reused below: its earlier stores must have read it
        if ((threadIdx.x & 31) == 0) bulk_wait_read<0>();
        __syncwarp();
    }
    uint32_t zero[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) zero[i] = 0u;
#pragma unroll 1
    for (int c = 0; c < BH / 32; ++c) warp_store_rows(xbuf, zero, row + c * 32);
}

// One chunk of the gate/up forward on CTA pairs, stored by TMA: this warp's 32
// rows (from y) of gate, up and aw go to the three buffers of xbuf3 and out
// through hmap (columns x and I + x of h) and amap (columns x of aw).  The
// buffers are reused chunk after chunk, once the previous chunk's stores have
// read them.
__device__ __forceinline__ void gateup_chunk_tma(const GemmArgs &a, bool valid, float wv, const uint32_t (&gr)[32],
                                                 const uint32_t (&ur)[32], uint8_t *xbuf3, const CUtensorMap *hmap,
                                                 const CUtensorMap *amap, int x, int y) {
    uint32_t pg[16], pu[16], pa[16];
    float av[32];
    gateup_math(a, valid, wv, gr, ur, pg, pu, pa, av);
    const int lane = threadIdx.x & 31;
    if (lane == 0) bulk_wait_read<0>();
    __syncwarp();
    put_row_swz64(xbuf3, pg);
    put_row_swz64(xbuf3 + kXposeBytes, pu);
    put_row_swz64(xbuf3 + 2 * kXposeBytes, pa);
    fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0) {
        tma_store_2d(hmap, xbuf3, x, y);
        tma_store_2d(hmap, xbuf3 + kXposeBytes, a.I + x, y);
        tma_store_2d(amap, xbuf3 + 2 * kXposeBytes, x, y);
        bulk_commit();
    }
}

// Gate/up forward on CTA pairs (BN = 256): a tile covers gate/up columns
// nt*128 .. +128, laid out in the accumulator as [gate 0..63 | up 0..63 |
// gate 64..127 | up 64..127] (see the producer).  Output chunk c (32 gate
// columns and the matching up columns) sits at TMEM column (c >> 1) * 128 +
// (c & 1) * 32 (gate) and 64 further (up).  A full tile's thread owns row
// quad * 32 + lane and all four chunks.  A half tile (M = 128 pair MMA) holds
// this CTA's 64 rows in lanes 0..63 with columns [0, 128) of the tile and in
// lanes 64..127 with columns [128, 256), both at TMEM columns [0, 128): the
// thread owns row (quad & 1) * 32 + lane of its 64 and chunks 2h, 2h + 1 with
// h = quad >> 1.  Same SwiGLU arithmetic as the one-CTA kernel; h and aw go
// out by TMA stores (gateup_chunk_tma).
__device__ __forceinline__ void epi_gateup_fwd_pair(const GemmArgs &a, const Tile &t, int quad, int lane,
                                                    uint32_t taddr, uint64_t *tempty_acc, uint8_t *xbuf3,
                                                    const CUtensorMap *hmap, const CUtensorMap *amap) {
    const int r = t.half ? (quad & 1) * 32 + lane : quad * 32 + lane;
    const int pos = t.row0 + r;
    const int y = t.row0 + (r & ~31);  // this warp's first row
    const int p = __ldg(a.perm + pos);
    const bool valid = p >= 0 && p < a.T * a.k;
    const float wv = valid ? __ldg(a.topk_w + p) : 0.f;
    const int c_first = t.half ? 2 * (quad >> 1) : 0;
    const int n_chunks = t.half ? 2 : 4;
    auto gate_col = [&](int c) -> uint32_t {
        return static_cast<uint32_t>(t.half ? (c & 1) * 32 : (c >> 1) * 128 + (c & 1) * 32);
    };
    uint32_t ga[32], ua[32], gb[32], ub[32];
    tmem_load32(taddr + gate_col(c_first), ga);
    tmem_load32(taddr + gate_col(c_first) + 64, ua);
    tmem_load_wait();
    tmem_regs_ready(ga);
    tmem_regs_ready(ua);
#pragma unroll 1
    for (int i = 0; i < n_chunks; i += 2) {
        const int c = c_first + i;
        tmem_load32(taddr + gate_col(c + 1), gb);
        tmem_load32(taddr + gate_col(c + 1) + 64, ub);
        gateup_chunk_tma(a, valid, wv, ga, ua, xbuf3, hmap, amap, t.nt * 128 + c * 32, y);
        tmem_load_wait();
        tmem_regs_ready(gb);
        tmem_regs_ready(ub);
        if (i + 2 < n_chunks) {
            tmem_load32(taddr + gate_col(c + 2), ga);
            tmem_load32(taddr + gate_col(c + 2) + 64, ua);
        } else {
            release_acc<true>(tempty_acc);  // TMEM no longer needed
        }
        gateup_chunk_tma(a, valid, wv, gb, ub, xbuf3, hmap, amap, t.nt * 128 + (c + 1) * 32, y);
        if (i + 2 < n_chunks) {
            tmem_load_wait();
            tmem_regs_ready(ga);
            tmem_regs_ready(ua);
        }
    }
}

// Staged rows on CTA pairs, half tile (M = 128 pair MMA): the thread owns row
// (quad & 1) * 32 + lane of this CTA's 64 rows and output columns
// [h * 128, h * 128 + 128) of the tile, h = quad >> 1, at tensor-memory
// columns [0, 128); staged as in epi_stage.
__device__ __forceinline__ void epi_stage_half(const GemmArgs &a, const Tile &t, int quad, int lane, uint32_t taddr,
                                               uint64_t *tempty_acc, uint8_t *xbuf) {
    const int pos = t.row0 + (quad & 1) * 32 + lane;
    const int p = __ldg(a.perm + pos);
    const bool valid = p >= 0 && p < a.T * a.k;
    __nv_bfloat16 *srow =
        valid ? a.stage + static_cast<size_t>(p) * a.d + t.nt * 256 + (quad >> 1) * 128 : nullptr;
    store_accumulator_bf16<128, true>(taddr, xbuf, srow, tempty_acc);
}

template <int MODE, int BN, bool MX>
__device__ void epilogue_loop(const GemmArgs &a, uint64_t *tfull, uint64_t *tempty, uint32_t tmem_base,
                              const int *order, uint8_t *xbuf, volatile int *abort_flag) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int quad = warp & 3;  // TMEM lanes this warp may access: 32*quad .. 32*quad+31
    const int ch = (warp - kEpiWarp0) >> 2;  // down dgrad: which half of the tile's columns
    const int r = quad * 32 + lane;
    const int total = total_tiles<MODE>(a);
    int local = 0;
    for (int tile = nth_tile<MODE>(0, blockIdx.x, gridDim.x); tile < total;
         tile = nth_tile<MODE>(++local, blockIdx.x, gridDim.x)) {
        const Tile t = decode_tile<MODE>(tile, a, order);
        const int acc = local & 1;
        const uint32_t aph = static_cast<uint32_t>(local >> 1) & 1u;
        if (!warp_wait(&tfull[acc], aph, abort_flag)) {
            raise_abort(abort_flag, a.status);
            return;
        }
        tc_fence_after_sync();
        const uint32_t taddr = tmem_base + static_cast<uint32_t>(acc * BN) + (static_cast<uint32_t>(quad * 32) << 16);
        if constexpr (ModeTraits<MODE>::kStage) {
            epi_stage<BN>(a, t, r, taddr, &tempty[acc], xbuf);
        } else if constexpr (MODE == kGateUpFwd) {
            epi_gateup_fwd<BN, MX>(a, t, r, taddr, &tempty[acc], xbuf);
        } else if constexpr (MODE == kDownDgrad) {
            epi_down_dgrad<BN, MX>(a, t, r, ch, taddr, &tempty[acc], xbuf);
        } else {
            epi_wgrad<MODE, BN>(a, t, r, taddr, &tempty[acc], xbuf);
        }
    }
}

template <int MODE, int BN, bool MX>
__global__ void __launch_bounds__(ModeTraits<MODE>::kThreads, 1)
    grouped_gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                        const GemmArgs args) {
    using C = Cfg<BN, MX>;
    using TR = ModeTraits<MODE>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + C::kBarOffset);
    uint64_t *empty = full + C::kStages;
    uint64_t *tfull = empty + C::kStages;
    uint64_t *tempty = tfull + 2;
    uint64_t *drain = tempty + 2;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(drain + 1);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);
    int *s_count = reinterpret_cast<int *>(smem + C::kOrderOffset);
    int *order = s_count + kMaxExperts;

    const int warp = threadIdx.x >> 5;
    if constexpr (!TR::kMTiled) {  // busiest expert first: rank by padded row count, ties to lower index
        for (int e = threadIdx.x; e < args.E; e += TR::kThreads)
            s_count[e] = __ldg(args.group_start + e + 1) - __ldg(args.group_start + e);
        __syncthreads();
        for (int e = threadIdx.x; e < args.E; e += TR::kThreads) {
            const int c = s_count[e];
            int rank = 0;
            for (int f = 0; f < args.E; ++f) {
                const int cf = s_count[f];
                rank += (cf > c || (cf == c && f < e)) ? 1 : 0;
            }
            order[rank] = e;
        }
    }
    if (threadIdx.x == 0) {
        for (int s = 0; s < C::kStages; ++s) {
            mbar_init(&full[s], 1 + (TR::kGather ? kGatherThreads : 0));
            mbar_init(&empty[s], 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&tfull[i], 1);
            mbar_init(&tempty[i], TR::kEpiWarps);
        }
        mbar_init(drain, 1);
        *abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, C::kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    const uint32_t tmem_base = *tmem_slot;

    if (warp == 0) {
        producer_loop<MODE, BN, MX>(&tmA, &tmB, args, smem, full, empty, order, abort_flag);
    } else if (warp == 1) {
        if ((threadIdx.x & 31) == 0)
            mma_loop<MODE, BN, MX>(args, smem, full, empty, tfull, tempty, drain, tmem_base, order, abort_flag);
        __syncwarp();
    } else if (warp < TR::kGatherWarp0) {
        epilogue_loop<MODE, BN, MX>(args, tfull, tempty, tmem_base, order,
                                smem + C::kXposeOffset + (warp - kEpiWarp0) * kXposeBytes, abort_flag);
    } else if constexpr (TR::kGather) {
        gather_loop<MODE, BN, MX>(args, smem, full, empty, order, abort_flag);
    }

    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    if (warp == 1) tmem_dealloc(tmem_base, C::kTmemCols);
}

// ---------------------------------------------------------------------------
// GEMMs on CTA pairs (bf16, BN = 256): all six modes (the gate/up forward on x
// copied into the sorted layout first).  A cluster of two CTAs computes one 256 x 256 tile with
// tcgen05.mma.cta_group::2: each CTA loads its own 128 M rows of A and one
// half (128 columns) of B, so a CTA moves half the B bytes per MMA it takes
// part in; 32 KB stages instead of 48 KB.  The leader (rank 0) arms the stage
// barriers for both CTAs' bytes and issues the MMAs; commits arrive on the
// barriers of both CTAs; the epilogue warps of both CTAs release an
// accumulator on the leader's barrier.  Each CTA's epilogue works on its own
// 128 rows exactly as in the one-CTA kernel (same functions, same outputs).
//
// M-tiled modes pair two consecutive 128-row tiles of one expert (both use the
// expert's B).  An expert with an odd number of tiles ends with a half pair
// row.  In the gate/up forward it is the last tile alone, computed by M = 128
// pair MMAs: each CTA holds 64 of its rows, and the MMA runs at the same rate
// per row as the M = 256 form.  In the gate/up dgrad the peer loads the rows
// past the group (or zeros past the end of the sorted buffer), the MMA computes
// them and the peer's epilogue only releases the accumulator.  Pair rows are
// numbered expert by expert from a per-CTA table of their starts.
//
// The third tensor map, tmC, is per mode: A in 64-row boxes (the forward GEMMs'
// half tiles), h in 128-row x 32-column boxes (the down dgrad's ring loads), or
// dW in 32-row x 64-column boxes (the weight gradients' epilogue stores).  The gate/up
// dgrad does not use it.  tmD and tmE, h and aw in 32 x 32 boxes, are the
// gate/up forward's epilogue stores.
//
// No load is multicast.  Every wait is bounded, and both CTAs always reach the
// final cluster barrier (no early exit), after which the pair frees its tensor
// memory.
// ---------------------------------------------------------------------------
template <int MODE, int BN>
struct PairCfg {
    using TR = ModeTraits<MODE>;
    static constexpr int kBHalfBytes = (BN / 2) * kTileK * 2;  // this CTA's half of a B stage
    static constexpr int kStageBytes = kABytes + kBHalfBytes;
    static constexpr int kOrderBytes = 8 * kMaxExperts;  // wgrads: counts + order; M-tiled: pair-row starts
    // transpose buffers per epilogue warp: two (one 4 KB box of 32 rows x 64
    // columns) for the weight gradients' TMA stores; three (gate, up, aw) for the
    // gate/up forward's
    static constexpr int kXposePerWarp = MODE == kGateUpFwd ? 3 : (TR::kMTiled ? 1 : 2);
    static constexpr int kXposeTotal = TR::kEpiWarps * kXposePerWarp * kXposeBytes;
    // down dgrad: a ring of two h chunks (gate and up, 128 rows x 32 columns each)
    static constexpr int kRingSlotBytes = 2 * kTileM * 32 * 2;
    static constexpr int kRingBytes = MODE == kDownDgrad ? 2 * kRingSlotBytes : 0;
    static constexpr int kFixed = 512 + kOrderBytes + kXposeTotal + kRingBytes + 1024;
    static constexpr int kFit = (227 * 1024 - kFixed) / kStageBytes;
    static constexpr int kStages = kFit < 6 ? kFit : 6;
    // stages, ring and transpose buffers are 1024-byte aligned (the 64- and
    // 128-byte swizzles of the ring's loads and of the epilogues' TMA stores
    // repeat every 512 and 1024 bytes)
    static constexpr int kRingOffset = kStages * kStageBytes;
    static constexpr int kXposeOffset = kRingOffset + kRingBytes;
    static constexpr int kBarOffset = kXposeOffset + kXposeTotal;
    static constexpr int kOrderOffset = kBarOffset + 512;
    static constexpr int kSmemBytes = kOrderOffset + kOrderBytes + 1024;
    static_assert(kStageBytes % 1024 == 0 && kRingBytes % 1024 == 0 && kXposeTotal % 1024 == 0, "alignment");
    static_assert(kStages >= 4 && kSmemBytes <= 227 * 1024, "shared memory per CTA");
    static constexpr uint32_t kTmemCols = 2 * BN;
};

// Pair tile.  Wgrads: (expert rank in LPT order, pair of 128-row M tiles, N
// tile).  M-tiled modes: (pair row, N tile), the pair row's expert found in
// pstart (pstart[e] = first pair row of expert e, pstart[E] = their number).
template <int MODE>
__device__ __forceinline__ Tile decode_pair_tile(int tile, const GemmArgs &a, const int *tbl, uint32_t rank) {
    Tile t;
    t.skip = false;
    t.half = false;
    t.row0 = 0;
    if constexpr (ModeTraits<MODE>::kMTiled) {
        const int pr = tile / a.n_tiles;
        t.nt = tile - pr * a.n_tiles;
        int lo = 0, hi = a.E;  // the last expert whose first pair row is <= pr
        while (hi - lo > 1) {
            const int mid = (lo + hi) >> 1;
            if (tbl[mid] <= pr)
                lo = mid;
            else
                hi = mid;
        }
        t.e = lo;
        const int g0 = __ldg(a.group_start + lo) / kTileM, g1 = __ldg(a.group_start + lo + 1) / kTileM;
        const int t0 = g0 + 2 * (pr - tbl[lo]);  // the pair row's first tile (t0 < g1)
        if constexpr (MODE == kGateUpFwd || MODE == kDownFwd) {
            t.half = t0 + 1 >= g1;  // the expert's last tile has no partner: M = 128 pair MMA
            t.mt = t.half ? t0 : t0 + static_cast<int>(rank);
            t.row0 = t.half ? t0 * kTileM + 64 * static_cast<int>(rank) : t.mt * kTileM;
        } else {
            // the dgrads compute the unpaired tile's partner rows and discard them (a half-row MMA
            // measured 1.5 % slower in the gate/up dgrad: its operand loads bound the pair row)
            t.mt = t0 + static_cast<int>(rank);
            t.skip = t.mt >= g1;
            t.row0 = t.mt * kTileM;
        }
        t.nkb = a.num_k_blocks;
        t.kpos0 = 0;
    } else {
        const int mp_tiles = a.m_tiles / 2;
        const int per = mp_tiles * a.n_tiles;
        const int er = tile / per;
        const int rr = tile - er * per;
        t.e = tbl[er];
        const int mp = rr / a.n_tiles;
        t.nt = rr - mp * a.n_tiles;
        t.mt = 2 * mp + static_cast<int>(rank);
        const int gs = __ldg(a.group_start + t.e), ge = __ldg(a.group_start + t.e + 1);
        t.nkb = (ge - gs) / a.k_elems;
        t.kpos0 = gs;
        if (t.e < 0 || t.e >= a.E) {
            t.e = 0;
            t.nkb = 0;
        }
    }
    return t;
}

template <int MODE, int BN>
__global__ void __launch_bounds__(ModeTraits<MODE>::kThreads, 1)
    grouped_gemm_pair_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                             const __grid_constant__ CUtensorMap tmC, const __grid_constant__ CUtensorMap tmD,
                             const __grid_constant__ CUtensorMap tmE, const GemmArgs args) {
    static_assert(MODE == kGateUpFwd || MODE == kDownWgrad || MODE == kGateUpWgrad || MODE == kGateUpDgrad ||
                      MODE == kDownDgrad || MODE == kDownFwd,
                  "the modes where pairs measured faster than one CTA");
    using P = PairCfg<MODE, BN>;
    using TR = ModeTraits<MODE>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + P::kBarOffset);
    uint64_t *empty = full + P::kStages;
    uint64_t *tfull = empty + P::kStages;
    uint64_t *tempty = tfull + 2;
    uint64_t *drain = tempty + 2;
    uint64_t *hfull = drain + 1;   // down dgrad: h ring slots loaded (TMA bytes)
    uint64_t *hempty = hfull + 2;  // down dgrad: h ring slots read by every epilogue warp
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(hempty + 2);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);
    int *s_count = reinterpret_cast<int *>(smem + P::kOrderOffset);
    int *tbl = TR::kMTiled ? s_count : s_count + kMaxExperts;  // pair-row starts, or the expert order
    uint8_t *ring = smem + P::kRingOffset;
    const uint32_t rank = cluster_ctarank();
    const bool leader = rank == 0;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int pair = blockIdx.x >> 1, npairs = gridDim.x >> 1;
    const GemmArgs &a = args;

    if constexpr (TR::kMTiled) {
        // pair rows per expert: ceil(tiles / 2), numbered expert by expert (warp 0 scans)
        if (warp == 0) {
            int carry = 0;
            for (int e0 = 0; e0 < a.E; e0 += 32) {
                const int e = e0 + lane;
                int np = 0;
                if (e < a.E)
                    np = ((__ldg(a.group_start + e + 1) - __ldg(a.group_start + e)) / kTileM + 1) >> 1;
                int incl = np;
#pragma unroll
                for (int off = 1; off < 32; off <<= 1) {
                    const int o = __shfl_up_sync(0xffffffffu, incl, off);
                    if (lane >= off) incl += o;
                }
                if (e < a.E) tbl[e] = carry + incl - np;
                carry += __shfl_sync(0xffffffffu, incl, 31);
            }
            if (lane == 0) tbl[a.E] = carry;
        }
    } else {
        // busiest expert first (the same order in both CTAs)
        for (int e = threadIdx.x; e < a.E; e += blockDim.x)
            s_count[e] = __ldg(a.group_start + e + 1) - __ldg(a.group_start + e);
        __syncthreads();
        for (int e = threadIdx.x; e < a.E; e += blockDim.x) {
            const int c = s_count[e];
            int rk = 0;
            for (int f = 0; f < a.E; ++f) {
                const int cf = s_count[f];
                rk += (cf > c || (cf == c && f < e)) ? 1 : 0;
            }
            tbl[rk] = e;
        }
    }
    if (threadIdx.x == 0) {
        for (int s = 0; s < P::kStages; ++s) {
            mbar_init(&full[s], 1);   // the leader's producer; both CTAs' bytes
            mbar_init(&empty[s], 1);  // one commit per use
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&tfull[i], 1);
            mbar_init(&tempty[i], 2 * TR::kEpiWarps);  // the epilogue warps of both CTAs (leader's barrier)
            mbar_init(&hfull[i], 1);                   // this CTA's h loader
            mbar_init(&hempty[i], TR::kEpiWarps);      // this CTA's epilogue warps
        }
        mbar_init(drain, 1);
        *abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == 1) {
        tmem_alloc_pair(tmem_slot, P::kTmemCols);
        tmem_relinquish_pair();
    }
    tc_fence_before_sync();
    cluster_sync();  // both CTAs' tables and barriers initialised and tensor memory allocated
    tc_fence_after_sync();
    const uint32_t tmem_base = *tmem_slot;
    const int total = TR::kMTiled ? tbl[a.E] * a.n_tiles : a.E * (a.m_tiles / 2) * a.n_tiles;

    if (warp == 0) {
        // ---- producer: this CTA's A rows and B half, counted on the leader's barrier ----
        int it = 0;
        bool ok = true;
        for (int i = 0, tile = nth_tile<MODE>(0, pair, npairs); tile < total && ok;
             tile = nth_tile<MODE>(++i, pair, npairs)) {
            const Tile t = decode_pair_tile<MODE>(tile, a, tbl, rank);
            for (int kb = 0; kb < t.nkb; ++kb, ++it) {
                const int s = it % P::kStages;
                const uint32_t ph = static_cast<uint32_t>(it / P::kStages) & 1u;
                if (!warp_wait(&empty[s], ph ^ 1u, abort_flag)) {
                    ok = false;
                    break;
                }
                // a half tile's A is 64 rows (tmC) in each CTA
                if (leader && lane == 0)
                    mbar_arrive_expect_tx(&full[s], t.half ? 2u * (P::kStageBytes - kABytes / 2) : 2u * P::kStageBytes);
                __syncwarp();
                const uint32_t fb = cluster_addr(&full[s], 0);
                uint8_t *As = smem + s * P::kStageBytes;
                uint8_t *Bs = As + kABytes;
                const int k0 = kb * kTileK;
                const int bcol = t.nt * BN + static_cast<int>(rank) * (BN / 2);  // this CTA's B columns
                if constexpr (MODE == kGateUpFwd) {
                    // A: 128 sorted rows of x from row0 (a half tile: 64 rows, all its MMA reads);
                    // B: the tile covers gate/up columns nt*128 .. +128; the leader loads 64 gate
                    // rows and the 64 matching up rows for the first 64 of them, the peer for the
                    // other 64 (64-row boxes, K-major), so that accumulator columns hold, per
                    // 64-column group, gate then up of the same expert columns -- in a half tile
                    // each TMEM lane half then holds whole (gate, up) pairs
                    if (lane == 0) tma_load_2d_pair(As, t.half ? &tmC : &tmA, fb, k0, t.row0);
                    const int grow = t.e * 2 * a.I + t.nt * (BN / 2) + 64 * static_cast<int>(rank);
                    if (lane == 1) tma_load_2d_pair(Bs, &tmB, fb, k0, grow);
                    if (lane == 2) tma_load_2d_pair(Bs + 64 * 128, &tmB, fb, k0, grow + a.I);
                } else if constexpr (MODE == kDownFwd) {
                    // A: 128 sorted rows of aw from row0 (a half tile: 64 rows); B: this CTA's 128 of the
                    // tile's 256 rows of W_down[e] (output columns), K-major
                    if (lane == 0) tma_load_2d_pair(As, t.half ? &tmC : &tmA, fb, k0, t.row0);
                    if (lane == 1) tma_load_2d_pair(Bs, &tmB, fb, k0, t.e * a.d + t.nt * BN + static_cast<int>(rank) * (BN / 2));
                } else if constexpr (MODE == kDownDgrad) {
                    // A: 128 sorted rows of grad_out, K-major; B: this CTA's half of W_down[e]
                    // (its N = I columns), MN-major
                    const int brow = t.e * a.d + k0;
                    if (lane == 0) tma_load_2d_pair(As, &tmA, fb, k0, t.row0);
                    if (lane >= 1 && lane < 1 + BN / 128)
                        tma_load_2d_pair(Bs + (lane - 1) * kChunkBytes, &tmB, fb, bcol + 64 * (lane - 1), brow);
                } else if constexpr (TR::kMTiled) {
                    // A: 128 sorted rows of dh from row0, K-major; B: this CTA's half of W_gate_up[e], MN-major
                    const int brow = t.e * 2 * a.I + k0;
                    if (lane == 0) tma_load_2d_pair(As, &tmA, fb, k0, t.row0);
                    if (lane >= 1 && lane < 1 + BN / 128)
                        tma_load_2d_pair(Bs + (lane - 1) * kChunkBytes, &tmB, fb, bcol + 64 * (lane - 1), brow);
                } else {
                    if (lane < 2)  // A: 128 M rows, MN-major, two 64-wide chunks
                        tma_load_2d_pair(As + lane * kChunkBytes, &tmA, fb, t.mt * kTileM + 64 * lane,
                                         t.kpos0 + k0);
                    if (lane >= 2 && lane < 2 + BN / 128)  // this CTA's half of B, MN-major
                        tma_load_2d_pair(Bs + (lane - 2) * kChunkBytes, &tmB, fb, bcol + 64 * (lane - 2),
                                         t.kpos0 + k0);
                }
            }
        }
        if (!ok) raise_abort(abort_flag, a.status);
    } else if (warp == 1) {
        // ---- MMA (leader, one thread): M = 256 over the pair ----
        if (leader && lane == 0) {
            constexpr uint32_t kIdesc = instr_desc_bf16(2 * kTileM, BN, TR::kAMn, TR::kBMn);
            constexpr uint32_t kIdescHalf = instr_desc_bf16(kTileM, BN, TR::kAMn, TR::kBMn);  // 64 rows per CTA
            int it = 0, local = 0;
            bool ok = true;
            for (int tile = nth_tile<MODE>(0, pair, npairs); tile < total && ok;
                 tile = nth_tile<MODE>(++local, pair, npairs)) {
                const Tile t = decode_pair_tile<MODE>(tile, a, tbl, rank);
                const int acc = local & 1;
                const uint32_t aph = static_cast<uint32_t>(local >> 1) & 1u;
                if (!mbar_wait_cluster(&tempty[acc], aph ^ 1u, abort_flag)) {
                    ok = false;
                    break;
                }
                tc_fence_after_sync();
                const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * BN);
                for (int kb = 0; kb < t.nkb; ++kb, ++it) {
                    const int s = it % P::kStages;
                    const uint32_t ph = static_cast<uint32_t>(it / P::kStages) & 1u;
                    if (!mbar_wait(&full[s], ph, abort_flag)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after_sync();
                    const uint32_t a_base = smem_u32(smem + s * P::kStageBytes);
                    const uint32_t b_base = a_base + kABytes;
#pragma unroll
                    for (int kk = 0; kk < kTileK / 16; ++kk) {
                        const uint64_t ad = TR::kAMn ? smem_desc_sw128(a_base + kk * 2048, kMnLbo, kSbo)
                                                     : smem_desc_sw128(a_base + kk * 32, 16, kSbo);
                        const uint64_t bd = TR::kBMn ? smem_desc_sw128(b_base + kk * 2048, kMnLbo, kSbo)
                                                     : smem_desc_sw128(b_base + kk * 32, 16, kSbo);
                        mma_bf16_pair(d_tmem, ad, bd, t.half ? kIdescHalf : kIdesc, (kb | kk) != 0 ? 1u : 0u);
                    }
                    mma_commit_pair(&empty[s], 0x3);  // frees the stage in both CTAs
                }
                if (!ok) break;
                mma_commit_pair(&tfull[acc], 0x3);
            }
            if (!ok) {
                raise_abort(abort_flag, a.status);
                mma_commit_pair(drain, 0x1);
                mbar_wait(drain, 0u, nullptr);
            }
        }
        __syncwarp();
    } else if (warp < TR::kGatherWarp0) {
        // ---- epilogue: this CTA's 128 rows of the tile ----
        const int quad = warp & 3;
        const int r = quad * 32 + lane;
        uint8_t *xbuf = smem + P::kXposeOffset + (warp - kEpiWarp0) * P::kXposePerWarp * kXposeBytes;
        int hit = 0;  // down dgrad: h ring chunks consumed so far
        int local = 0;
        for (int tile = nth_tile<MODE>(0, pair, npairs); tile < total;
             tile = nth_tile<MODE>(++local, pair, npairs)) {
            const Tile t = decode_pair_tile<MODE>(tile, a, tbl, rank);
            const int acc = local & 1;
            const uint32_t aph = static_cast<uint32_t>(local >> 1) & 1u;
            if (!warp_wait(&tfull[acc], aph, abort_flag)) {
                raise_abort(abort_flag, a.status);
                break;
            }
            tc_fence_after_sync();
            const uint32_t taddr =
                tmem_base + static_cast<uint32_t>(acc * BN) + (static_cast<uint32_t>(quad * 32) << 16);
            if constexpr (MODE == kGateUpFwd) {
                epi_gateup_fwd_pair(a, t, quad, lane, taddr, &tempty[acc], xbuf, &tmD, &tmE);
            } else if constexpr (MODE == kDownDgrad) {
                if (t.skip) {
                    release_acc<true>(&tempty[acc]);
                } else if (!epi_down_dgrad_ring(a, t, r, (warp - kEpiWarp0) >> 2, taddr, &tempty[acc], xbuf, ring,
                                                hfull, hempty, hit, abort_flag)) {
                    raise_abort(abort_flag, a.status);
                    break;
                }
            } else if constexpr (TR::kStage) {
                if (t.skip)
                    release_acc<true>(&tempty[acc]);
                else if (t.half)
                    epi_stage_half(a, t, quad, lane, taddr, &tempty[acc], xbuf);
                else
                    epi_stage<BN, true>(a, t, r, taddr, &tempty[acc], xbuf);
            } else {
                epi_wgrad<MODE, BN, true>(a, t, r, taddr, &tempty[acc], xbuf, &tmC);
            }
        }
        if constexpr (!TR::kMTiled || MODE == kGateUpFwd) {
            // the TMA tile stores are complete before the CTA ends
            if (lane == 0) bulk_wait_all();
            __syncwarp();
        }
    }

    if constexpr (MODE == kDownDgrad) {
        if (warp == TR::kGatherWarp0 && lane == 0) {
            // ---- h loader: this CTA's rows of h, chunk by chunk, one chunk ahead of the epilogue ----
            int hit = 0;
            bool ok = true;
            for (int tile = nth_tile<MODE>(0, pair, npairs), i = 0; tile < total && ok;
                 tile = nth_tile<MODE>(++i, pair, npairs)) {
                const Tile t = decode_pair_tile<MODE>(tile, a, tbl, rank);
                if (t.skip) continue;
                for (int c = 0; c < BN / 32; ++c, ++hit) {
                    const int slot = hit & 1;
                    if (!mbar_wait(&hempty[slot], (static_cast<uint32_t>(hit >> 1) & 1u) ^ 1u, abort_flag)) {
                        ok = false;
                        break;
                    }
                    mbar_arrive_expect_tx(&hfull[slot], P::kRingSlotBytes);
                    uint8_t *dst = ring + slot * P::kRingSlotBytes;
                    const int col = t.nt * BN + c * 32;
                    tma_load_2d(dst, &tmC, &hfull[slot], col, t.row0);                        // gate
                    tma_load_2d(dst + P::kRingSlotBytes / 2, &tmC, &hfull[slot], a.I + col, t.row0);  // up
                }
            }
            if (!ok) {
                raise_abort(abort_flag, a.status);
                for (int q = hit > 2 ? hit - 2 : 0; q < hit; ++q)  // its copies in flight land first
                    mbar_wait(&hfull[q & 1], static_cast<uint32_t>(q >> 1) & 1u, nullptr);
            }
        }
        __syncwarp();
    }

    tc_fence_before_sync();
    __syncthreads();
    cluster_sync();  // no CTA leaves while its peer may still signal into it
    tc_fence_after_sync();
    if (warp == 1) tmem_dealloc_pair(tmem_base, P::kTmemCols);
}

// The opt-in to more than 48 KB of dynamic shared memory belongs to a kernel
// as loaded on one device (each device's context holds its own copy), so it,
// and the occupancy measured with it, are cached per device.
constexpr int kMaxDevices = 64;

int current_device() {
    int d = -1;
    return cudaGetDevice(&d) == cudaSuccess && d >= 0 && d < kMaxDevices ? d : -1;
}

template <int MODE, int BN, bool MX>
cudaError_t launch_one(const GemmArgs &args, const CUtensorMap &tmA, const CUtensorMap &tmB, int grid,
                       cudaStream_t s) {
    constexpr int kSmem = Cfg<BN, MX>::smem_bytes(ModeTraits<MODE>::kEpiWarps);
    static std::atomic<bool> attr_set[kMaxDevices];  // per instantiation and device
    const int dev = current_device();
    if (dev < 0) return cudaErrorInvalidDevice;
    if (!attr_set[dev].load(std::memory_order_acquire)) {
        cudaError_t e = cudaFuncSetAttribute(grouped_gemm_kernel<MODE, BN, MX>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, kSmem);
        if (e != cudaSuccess) return e;
        attr_set[dev].store(true, std::memory_order_release);
    }
    grouped_gemm_kernel<MODE, BN, MX><<<grid, ModeTraits<MODE>::kThreads, kSmem, s>>>(tmA, tmB, args);
    return cudaGetLastError();
}

template <int MODE>
cudaError_t launch_mode(int bn, bool mx, const GemmArgs &args, const CUtensorMap &tmA, const CUtensorMap &tmB,
                        int grid, cudaStream_t s) {
    if (mx) return bn == 128 ? launch_one<MODE, 128, true>(args, tmA, tmB, grid, s) : cudaErrorInvalidValue;
    if (bn == 256) return launch_one<MODE, 256, false>(args, tmA, tmB, grid, s);
    if (bn == 128) return launch_one<MODE, 128, false>(args, tmA, tmB, grid, s);
    return cudaErrorInvalidValue;
}

// Launch of a CTA-pair kernel: clusters of two, as many pairs as the GPU holds
// at once (capped by the grid the caller offers).
template <int MODE>
cudaError_t launch_pair(const GemmArgs &args, const CUtensorMap &tmA, const CUtensorMap &tmB,
                        const CUtensorMap &tmC, const CUtensorMap &tmD, const CUtensorMap &tmE, int grid,
                        cudaStream_t s) {
    using P = PairCfg<MODE, 256>;
    auto *fn = grouped_gemm_pair_kernel<MODE, 256>;
    static std::atomic<int> max_pairs_plus1[kMaxDevices];  // per instantiation and device: resident
                                                           // clusters of two, plus one (0: not measured)
    const int dev = current_device();
    if (dev < 0) return cudaErrorInvalidDevice;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cudaLaunchConfig_t cfg = {};
    cfg.blockDim = dim3(ModeTraits<MODE>::kThreads);
    cfg.dynamicSmemBytes = P::kSmemBytes;
    cfg.stream = s;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int max_pairs = max_pairs_plus1[dev].load(std::memory_order_acquire) - 1;
    if (max_pairs < 0) {
        cudaError_t e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, P::kSmemBytes);
        if (e != cudaSuccess) return e;
        cfg.gridDim = dim3(grid & ~1);
        int n = 0;
        e = cudaOccupancyMaxActiveClusters(&n, fn, &cfg);
        if (e != cudaSuccess) return e;
        max_pairs = n;
        max_pairs_plus1[dev].store(n + 1, std::memory_order_release);
    }
    const int pairs = (grid / 2) < max_pairs ? grid / 2 : max_pairs;
    if (pairs < 1) return cudaErrorInvalidConfiguration;
    cfg.gridDim = dim3(2 * pairs);
    return cudaLaunchKernelEx(&cfg, fn, tmA, tmB, tmC, tmD, tmE, args);
}

}  // namespace

cudaError_t launch_gemm(GemmMode mode, int bn, bool mx, const GemmArgs &args, const CUtensorMap &tmA,
                        const CUtensorMap &tmB, int grid, cudaStream_t s) {
    switch (mode) {
        case kGateUpFwd: return launch_mode<kGateUpFwd>(bn, mx, args, tmA, tmB, grid, s);
        case kDownFwd: return launch_mode<kDownFwd>(bn, mx, args, tmA, tmB, grid, s);
        case kDownDgrad: return launch_mode<kDownDgrad>(bn, mx, args, tmA, tmB, grid, s);
        case kGateUpDgrad: return launch_mode<kGateUpDgrad>(bn, mx, args, tmA, tmB, grid, s);
        case kDownWgrad: return launch_mode<kDownWgrad>(bn, mx, args, tmA, tmB, grid, s);
        case kGateUpWgrad: return launch_mode<kGateUpWgrad>(bn, mx, args, tmA, tmB, grid, s);
    }
    return cudaErrorInvalidValue;
}

bool gemm_pair_ok(GemmMode mode, int bn, bool mx, int m_tiles, int grid) {
    if (mx || bn != 256 || grid < 2) return false;
    if (mode == kDownWgrad || mode == kGateUpWgrad) return m_tiles % 2 == 0;
    return mode == kGateUpFwd || mode == kGateUpDgrad || mode == kDownDgrad || mode == kDownFwd;
}

cudaError_t launch_gemm_pair(GemmMode mode, const GemmArgs &args, const CUtensorMap &tmA, const CUtensorMap &tmB,
                             int grid, cudaStream_t s, const CUtensorMap *tmC, const CUtensorMap *tmD,
                             const CUtensorMap *tmE) {
    if (tmC == nullptr && mode != kGateUpDgrad) return cudaErrorInvalidValue;  // every other mode uses the third map
    if ((tmD == nullptr || tmE == nullptr) && mode == kGateUpFwd) return cudaErrorInvalidValue;  // h and aw stores
    const CUtensorMap &c = tmC != nullptr ? *tmC : tmA;
    const CUtensorMap &d = tmD != nullptr ? *tmD : tmA;
    const CUtensorMap &e = tmE != nullptr ? *tmE : tmA;
    switch (mode) {
        case kDownWgrad: return launch_pair<kDownWgrad>(args, tmA, tmB, c, d, e, grid, s);
        case kGateUpWgrad: return launch_pair<kGateUpWgrad>(args, tmA, tmB, c, d, e, grid, s);
        case kGateUpFwd: return launch_pair<kGateUpFwd>(args, tmA, tmB, c, d, e, grid, s);
        case kGateUpDgrad: return launch_pair<kGateUpDgrad>(args, tmA, tmB, c, d, e, grid, s);
        case kDownDgrad: return launch_pair<kDownDgrad>(args, tmA, tmB, c, d, e, grid, s);
        case kDownFwd: return launch_pair<kDownFwd>(args, tmA, tmB, c, d, e, grid, s);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace moe

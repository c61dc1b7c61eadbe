// Plain, slow fp64 C++ statement of the single-GPU fused mixture-of-experts
// layer, forward and backward.
//
// TEST INFRASTRUCTURE ONLY.  Nothing in the product path links or loads this
// file's library: only tests/, __graft_entry__.smoke() and bench.py's CPU
// baseline / reference arm use it.  It shares no code with the CUDA library
// (no header, helper, table or constant), and it computes the same definitions
// as the numpy oracle beside it (moe_oracle.py), against which it is checked.
//
// What the layer computes (sources, by page and section):
//  * "Prime Intellect Fused MoE Kernel: 3.11x MoE Training Speed", section
//    "What a mixture-of-experts layer actually does": route each token to a
//    few experts, dispatch, both expert linear layers with SwiGLU, combine.
//  * "Prime Intellect's Prime Mega MoE Trains Giant AI Models 55% Faster",
//    section "Where MoE training loses time": token sorting (dispatch), the
//    expert MLPs, outputs returned to their original positions; the backward
//    pass repeats the exchange for gradients.
//  * "Mario/overlap moe kernel integration (prime-rl PR #3651)", Overview:
//    the op consumes undispatched tokens plus the routing and returns the
//    gradients of its inputs.
//
// Readings where the pages are silent (the same ones the numpy oracle takes):
//  * routing: softmax over the E fp32 logits, keep the k largest (chosen on the
//    logits: value descending, ties to the lower expert index), renormalise
//    over the kept k; slot j = the j-th choice.
//  * dispatch: experts ascending, tokens ascending inside an expert.
//  * expert: W_gate_up[e] is [2I, d] (rows 0..I-1 gate, I..2I-1 up),
//    W_down[e] is [d, I]; a = silu(gate) * up; no bias.
//  * clamped SwiGLU (the DeepSeek V4 `ClampedSilu` that the review note of
//    "Mario/overlap moe kernel integration (prime-rl PR #3651)" says the kernel
//    computes; no formula on the pages): with limit L > 0,
//    a = silu(min(gate, L)) * clip(up, -L, L), the gradient passing where the
//    input lies in the closed interval (end points inside), decided on the
//    exact pre-activation; limit 0 is the plain SwiGLU.
//  * combine and dx scatter: sums over slots j = 0..k-1 in slot order.
//  * dscore[t, j] = dL/dw[t, j]; dlogits through the renormalised softmax.
//
// Arithmetic: every float is a double; inputs arrive already widened (bf16 and
// fp32 widen exactly).  Plain loops, no blocking or reordering beyond the
// definitions; built without fast-math and without FMA contraction.  Threads
// (std::thread) split the experts, each of which owns its own outputs, so the
// result does not depend on the thread count.
#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <numeric>
#include <thread>
#include <vector>

namespace {

double sigmoid(double z) { return 1.0 / (1.0 + std::exp(-z)); }
double silu(double z) { return z * sigmoid(z); }
double silu_grad(double z) {
    const double s = sigmoid(z);
    return s * (1.0 + z * (1.0 - s));
}

// The activation: plain SwiGLU for L <= 0, clamped SwiGLU for L > 0.
double act(double g, double u, double L) {
    if (L > 0) {
        g = std::min(g, L);
        u = std::min(std::max(u, -L), L);
    }
    return silu(g) * u;
}

// (dg, du) of act for dL/da = da; a clamp stops the gradient outside its
// closed interval.
void act_grad(double g, double u, double L, double da, double *dg, double *du) {
    double gc = g, uc = u;
    if (L > 0) {
        gc = std::min(g, L);
        uc = std::min(std::max(u, -L), L);
    }
    *dg = (L > 0 && g > L) ? 0.0 : da * uc * silu_grad(gc);
    *du = (L > 0 && std::fabs(u) > L) ? 0.0 : da * silu(gc);
}

// Run fn(e) for every expert e, experts dealt round-robin to n threads.
template <class F>
void for_each_expert(int E, int nthreads, F fn) {
    if (nthreads < 1) nthreads = 1;
    if (nthreads > E) nthreads = E;
    if (nthreads == 1) {
        for (int e = 0; e < E; ++e) fn(e);
        return;
    }
    std::vector<std::thread> pool;
    for (int i = 0; i < nthreads; ++i)
        pool.emplace_back([&, i] {
            for (int e = i; e < E; e += nthreads) fn(e);
        });
    for (auto &th : pool) th.join();
}

}  // namespace

extern "C" {

// Top-k routing of T tokens over E experts.  idx [T, k] (int32), w [T, k].
int moe_oracle_route(int64_t T, int E, int k, const float *logits, int32_t *idx, double *w) {
    if (T < 1 || E < 1 || k < 1 || k > E) return -1;
    std::vector<int> order(E);
    std::vector<double> p(E);
    for (int64_t t = 0; t < T; ++t) {
        const float *l = logits + t * E;
        std::iota(order.begin(), order.end(), 0);
        std::sort(order.begin(), order.end(), [l](int a, int b) {
            const double la = l[a], lb = l[b];
            return la > lb || (la == lb && a < b);
        });
        double m = l[0];
        for (int e = 1; e < E; ++e) m = std::max(m, static_cast<double>(l[e]));
        double z = 0.0;
        for (int e = 0; e < E; ++e) {
            p[e] = std::exp(static_cast<double>(l[e]) - m);
            z += p[e];
        }
        double kept = 0.0;
        for (int j = 0; j < k; ++j) kept += p[order[j]] / z;
        for (int j = 0; j < k; ++j) {
            idx[t * k + j] = order[j];
            w[t * k + j] = (p[order[j]] / z) / kept;
        }
    }
    return 0;
}

// Stable grouping of the T*k pairs by expert: counts [E], offsets [E+1],
// perm [T*k] (sorted position -> t*k + j), inv [T*k] (pair -> position).
int moe_oracle_dispatch(int64_t T, int E, int k, const int32_t *idx, int32_t *counts, int32_t *offsets,
                        int32_t *perm, int32_t *inv) {
    const int64_t P = T * k;
    for (int e = 0; e < E; ++e) counts[e] = 0;
    for (int64_t q = 0; q < P; ++q) {
        if (idx[q] < 0 || idx[q] >= E) return -1;
        ++counts[idx[q]];
    }
    offsets[0] = 0;
    for (int e = 0; e < E; ++e) offsets[e + 1] = offsets[e] + counts[e];
    std::vector<int64_t> next(offsets, offsets + E);
    for (int64_t q = 0; q < P; ++q) {  // pairs in flat order: tokens ascending
        const int64_t pos = next[idx[q]]++;
        perm[pos] = static_cast<int32_t>(q);
        inv[q] = static_cast<int32_t>(pos);
    }
    return 0;
}

// Forward.  x [T, d], wgu [E, 2I, d], wd [E, d, I] (doubles); logits fp32
// [T, E].  Writes out [T, d], idx [T, k], w [T, k]; h [T*k, 2I] and a [T*k, I]
// per flat pair when not null.  limit > 0: clamped SwiGLU.
int moe_oracle_forward(int64_t T, int d, int E, int k, int I, const double *x, const float *logits,
                       const double *wgu, const double *wd, double *out, int32_t *idx, double *w, double *h,
                       double *a, int nthreads, double limit) {
    if (moe_oracle_route(T, E, k, logits, idx, w) != 0) return -1;
    const int64_t P = T * k;
    std::vector<int32_t> counts(E), offsets(E + 1), perm(P), inv(P);
    if (moe_oracle_dispatch(T, E, k, idx, counts.data(), offsets.data(), perm.data(), inv.data()) != 0) return -1;
    std::vector<double> y(static_cast<size_t>(P) * d, 0.0);
    for_each_expert(E, nthreads, [&](int e) {
        const double *Wg = wgu + static_cast<size_t>(e) * 2 * I * d;
        const double *Wd = wd + static_cast<size_t>(e) * d * I;
        std::vector<double> hh(2 * I), aa(I);
        for (int32_t pos = offsets[e]; pos < offsets[e + 1]; ++pos) {
            const int64_t q = perm[pos], t = q / k;
            const double *xt = x + t * d;
            for (int r = 0; r < 2 * I; ++r) {
                double s = 0.0;
                for (int c = 0; c < d; ++c) s += Wg[static_cast<size_t>(r) * d + c] * xt[c];
                hh[r] = s;
            }
            for (int i = 0; i < I; ++i) aa[i] = act(hh[i], hh[I + i], limit);
            double *yq = y.data() + q * d;
            for (int o = 0; o < d; ++o) {
                double s = 0.0;
                for (int i = 0; i < I; ++i) s += Wd[static_cast<size_t>(o) * I + i] * aa[i];
                yq[o] = s;
            }
            if (h) std::memcpy(h + q * 2 * I, hh.data(), sizeof(double) * 2 * I);
            if (a) std::memcpy(a + q * I, aa.data(), sizeof(double) * I);
        }
    });
    for (int64_t t = 0; t < T; ++t) {
        double *ot = out + t * d;
        for (int c = 0; c < d; ++c) ot[c] = 0.0;
        for (int j = 0; j < k; ++j) {  // slot order
            const double wj = w[t * k + j];
            const double *yq = y.data() + (t * k + j) * d;
            for (int c = 0; c < d; ++c) ot[c] += wj * yq[c];
        }
    }
    return 0;
}

// Backward for dL/dout = gout [T, d].  Writes dx [T, d], dwgu [E, 2I, d],
// dwd [E, d, I], dscore [T, k] and dlogits [T, E] (zero outside the chosen k).
// limit > 0: clamped SwiGLU.
int moe_oracle_backward(int64_t T, int d, int E, int k, int I, const double *x, const float *logits,
                        const double *wgu, const double *wd, const double *gout, double *dx, double *dwgu,
                        double *dwd, double *dscore, double *dlogits, int nthreads, double limit) {
    const int64_t P = T * k;
    std::vector<int32_t> idx(P), counts(E), offsets(E + 1), perm(P), inv(P);
    std::vector<double> w(P);
    if (moe_oracle_route(T, E, k, logits, idx.data(), w.data()) != 0) return -1;
    if (moe_oracle_dispatch(T, E, k, idx.data(), counts.data(), offsets.data(), perm.data(), inv.data()) != 0)
        return -1;
    std::vector<double> dxp(static_cast<size_t>(P) * d, 0.0);
    for_each_expert(E, nthreads, [&](int e) {
        const double *Wg = wgu + static_cast<size_t>(e) * 2 * I * d;
        const double *Wd = wd + static_cast<size_t>(e) * d * I;
        double *dWg = dwgu + static_cast<size_t>(e) * 2 * I * d;
        double *dWd = dwd + static_cast<size_t>(e) * d * I;
        std::fill(dWg, dWg + static_cast<size_t>(2) * I * d, 0.0);
        std::fill(dWd, dWd + static_cast<size_t>(d) * I, 0.0);
        std::vector<double> hh(2 * I), aa(I), G(I), dh(2 * I);
        for (int32_t pos = offsets[e]; pos < offsets[e + 1]; ++pos) {
            const int64_t q = perm[pos], t = q / k;
            const double *xt = x + t * d, *gt = gout + t * d;
            const double wq = w[q];
            for (int r = 0; r < 2 * I; ++r) {
                double s = 0.0;
                for (int c = 0; c < d; ++c) s += Wg[static_cast<size_t>(r) * d + c] * xt[c];
                hh[r] = s;
            }
            for (int i = 0; i < I; ++i) aa[i] = act(hh[i], hh[I + i], limit);
            // G = W_down[e]^T gout[t] (each G[i] summed over o = 0..d-1 in order,
            // rows of W_down read contiguously); dscore = <G, a>
            std::fill(G.begin(), G.end(), 0.0);
            for (int o = 0; o < d; ++o)
                for (int i = 0; i < I; ++i) G[i] += Wd[static_cast<size_t>(o) * I + i] * gt[o];
            double ds = 0.0;
            for (int i = 0; i < I; ++i) ds += G[i] * aa[i];
            dscore[q] = ds;
            // SwiGLU backward of da = w G
            for (int i = 0; i < I; ++i) act_grad(hh[i], hh[I + i], limit, wq * G[i], &dh[i], &dh[I + i]);
            // dW_down[e] += (w gout[t]) (x) a
            for (int o = 0; o < d; ++o) {
                const double go = wq * gt[o];
                for (int i = 0; i < I; ++i) dWd[static_cast<size_t>(o) * I + i] += go * aa[i];
            }
            // dx contribution W_gate_up[e]^T dh; dW_gate_up[e] += dh (x) x[t]
            double *dq = dxp.data() + q * d;  // each dq[c] summed over r = 0..2I-1 in order
            for (int r = 0; r < 2 * I; ++r)
                for (int c = 0; c < d; ++c) dq[c] += Wg[static_cast<size_t>(r) * d + c] * dh[r];
            for (int r = 0; r < 2 * I; ++r)
                for (int c = 0; c < d; ++c) dWg[static_cast<size_t>(r) * d + c] += dh[r] * xt[c];
        }
    });
    for (int64_t t = 0; t < T; ++t) {
        double *dt = dx + t * d;
        for (int c = 0; c < d; ++c) dt[c] = 0.0;
        for (int j = 0; j < k; ++j) {  // slot order
            const double *dq = dxp.data() + (t * k + j) * d;
            for (int c = 0; c < d; ++c) dt[c] += dq[c];
        }
        // dlogit_i = w_i (dscore_i - sum_j w_j dscore_j) for chosen i, else 0
        double s = 0.0;
        for (int j = 0; j < k; ++j) s += w[t * k + j] * dscore[t * k + j];
        for (int e = 0; e < E; ++e) dlogits[t * E + e] = 0.0;
        for (int j = 0; j < k; ++j)
            dlogits[t * E + idx[t * k + j]] = w[t * k + j] * (dscore[t * k + j] - s);
    }
    return 0;
}

unsigned moe_oracle_hardware_threads(void) { return std::thread::hardware_concurrency(); }

}  // extern "C"

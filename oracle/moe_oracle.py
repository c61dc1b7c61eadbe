"""Plain, slow fp64 CPU statement of the single-GPU fused mixture-of-experts layer.

TEST INFRASTRUCTURE ONLY.  Nothing in the product path imports this module:
only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU baseline /
reference arm may use it.  It shares no code with the CUDA library.

What the layer computes (sources, by page and section):

* "Prime Intellect Fused MoE Kernel: 3.11x MoE Training Speed", section
  "What a mixture-of-experts layer actually does": a router sends each token to
  a few experts; the fused call does the dispatch, both expert linear layers,
  SwiGLU and the combine.
* "Prime Intellect's Prime Mega MoE Trains Giant AI Models 55% Faster",
  section "Where MoE training loses time": dispatch tokens to their experts
  (token sorting), run the expert MLPs, return the outputs to their original
  positions; the backward pass repeats the exchange for gradients.
* "Mario/overlap moe kernel integration (prime-rl PR #3651)", Overview and the
  custom-op commit note: the fused compute consumes undispatched tokens plus
  the routing (top scores, selected expert indices), runs in bf16 and returns
  gradients in the inputs' dtypes.

Readings taken where the pages are silent:

* routing: softmax over all E router logits, keep the k largest, renormalise
  over the kept k.  The k largest are chosen on the fp32 logits themselves
  (softmax is strictly increasing, so the set is the same), ordered by value
  descending and, on ties, by lower expert index.  Slot j of a token is its
  j-th choice in that order.
* dispatch order: experts ascending; inside an expert, tokens ascending
  (a stable counting sort of the flattened choices t*k + j).
* expert MLP: W_gate_up[e] is [2I, d] with rows 0..I-1 the gate and rows
  I..2I-1 the up projection; W_down[e] is [d, I].  h = W_gate_up[e] x,
  a = silu(h_gate) * h_up, y = W_down[e] a.  No bias.
* clamped SwiGLU ("Mario/overlap moe kernel integration (prime-rl PR #3651)",
  the review note on the DeepSeek V4 clamped SwiGLU, `ClampedSilu`, which the
  kernel computes, as opposed to the variant with sigmoid * 1.702 and up + 1,
  which it does not): the pages give no formula.  Reading: with a limit
  L > 0, a = silu(min(h_gate, L)) * clip(h_up, -L, L); the gradient passes
  where the input lies in the closed interval (h_gate <= L, |h_up| <= L) and
  is zero outside it.  limit = 0 is the plain SwiGLU above.  Both the clamp
  and the side of it on which the gradient stops are taken on the exact
  pre-activation (the definition's derivative, with the closed interval's
  end points counted inside).
* combine: out[t] = sum over slots j = 0..k-1, in slot order, of w[t,j] y_(t,j).
* dscore[t,j] is the gradient with respect to the renormalised weight w[t,j];
  dlogits is the gradient with respect to the router logits through the
  renormalised softmax (zero outside the chosen k).

All arithmetic is float64 on the exactly widened inputs.  Matrix products use
numpy (a library primitive); there is no blocking, fusion or reordering.
"""
from __future__ import annotations

import numpy as np

__all__ = [
    "route", "dispatch", "silu", "sigmoid", "swiglu", "swiglu_backward", "expert_forward",
    "combine_forward", "forward", "backward", "dense_forward",
    "forward_tokens", "backward_tokens", "backward_experts",
]


# ----------------------------------------------------------------------------
# elementwise functions (definitions, written out)
# ----------------------------------------------------------------------------
def sigmoid(z):
    """sigma(z) = 1 / (1 + exp(-z)), in float64."""
    z = np.asarray(z, dtype=np.float64)
    with np.errstate(over="ignore"):
        return 1.0 / (1.0 + np.exp(-z))


def silu(z):
    """silu(z) = z * sigma(z) (the gate of SwiGLU)."""
    z = np.asarray(z, dtype=np.float64)
    return z * sigmoid(z)


def silu_grad(z):
    """d silu / dz = sigma(z) * (1 + z * (1 - sigma(z)))."""
    s = sigmoid(z)
    return s * (1.0 + z * (1.0 - s))


def _clamps(g, u, limit):
    """(gate, up) after the clamp of the clamped SwiGLU; unchanged for limit = 0."""
    g, u = np.asarray(g, dtype=np.float64), np.asarray(u, dtype=np.float64)
    if limit > 0:
        return np.minimum(g, limit), np.clip(u, -limit, limit)
    return g, u


def swiglu(g, u, limit=0.0):
    """a = silu(g) * u; with limit > 0, silu(min(g, limit)) * clip(u, -limit, limit)."""
    gc, uc = _clamps(g, u, limit)
    return silu(gc) * uc


def swiglu_backward(g, u, da, limit=0.0):
    """(dg, du) of a = swiglu(g, u, limit) for dL/da = da.

    Inside the clamps: dg = da * uc * silu'(gc), du = da * silu(gc).  A clamp
    passes the gradient where its input lies in the closed interval and stops
    it outside (g > limit, |u| > limit), decided on g and u themselves.
    """
    g, u = np.asarray(g, dtype=np.float64), np.asarray(u, dtype=np.float64)
    gc, uc = _clamps(g, u, limit)
    da = np.asarray(da, dtype=np.float64)
    dg = da * uc * silu_grad(gc)
    du = da * silu(gc)
    if limit > 0:
        dg = np.where(g <= limit, dg, 0.0)
        du = np.where(np.abs(u) <= limit, du, 0.0)
    return dg, du


# ----------------------------------------------------------------------------
# routing and dispatch
# ----------------------------------------------------------------------------
def route(logits, k):
    """Top-k routing with renormalised softmax weights.

    logits: float32 [T, E] router logits (finite).  Returns
      idx  int32  [T, k]  chosen experts, slot j = j-th largest logit
                          (ties: lower expert index first)
      w    float64 [T, k] softmax over all E, restricted to the chosen k and
                          renormalised to sum to 1.
    """
    logits = np.asarray(logits)
    T, E = logits.shape
    if not (1 <= k <= E):
        raise ValueError("need 1 <= k <= E")
    lo = logits.astype(np.float64)  # exact widening of fp32 values
    expert = np.broadcast_to(np.arange(E), (T, E))
    # np.lexsort sorts by the last key first: value descending, then index
    order = np.lexsort((expert, -lo), axis=-1)
    idx = order[:, :k].astype(np.int32)
    # softmax over all experts, then renormalise over the kept k
    m = lo.max(axis=1, keepdims=True)
    p = np.exp(lo - m)
    p = p / p.sum(axis=1, keepdims=True)
    pk = np.take_along_axis(p, idx.astype(np.int64), axis=1)
    w = pk / pk.sum(axis=1, keepdims=True)
    return idx, w


def dispatch(idx, E):
    """Group the T*k (token, slot) pairs by expert.

    Returns counts [E], offsets [E+1] (exclusive scan of counts), perm [T*k]
    (sorted position -> flat pair index t*k + j; experts ascending, tokens
    ascending inside an expert) and inv [T, k] (pair -> sorted position).
    """
    idx = np.asarray(idx)
    T, k = idx.shape
    flat = idx.reshape(-1).astype(np.int64)
    counts = np.bincount(flat, minlength=E).astype(np.int32)
    offsets = np.zeros(E + 1, dtype=np.int32)
    offsets[1:] = np.cumsum(counts)
    perm = np.argsort(flat, kind="stable").astype(np.int32)
    inv = np.empty(T * k, dtype=np.int32)
    inv[perm] = np.arange(T * k, dtype=np.int32)
    return counts, offsets, perm, inv.reshape(T, k)


# ----------------------------------------------------------------------------
# one expert's MLP
# ----------------------------------------------------------------------------
def expert_forward(xe, wgu_e, wd_e, limit=0.0):
    """SwiGLU expert on a block of rows (clamped SwiGLU for limit > 0).

    xe [n, d]; wgu_e [2I, d]; wd_e [d, I].  Returns (h [n, 2I], a [n, I], y [n, d]).
    """
    I = wd_e.shape[1]
    h = xe @ wgu_e.T
    g, u = h[:, :I], h[:, I:]
    a = swiglu(g, u, limit)
    y = a @ wd_e.T
    return h, a, y


def _f64(a):
    return np.asarray(a, dtype=np.float64)


# ----------------------------------------------------------------------------
# forward
# ----------------------------------------------------------------------------
def combine_forward(x, idx, w, wgu, wd, limit=0.0):
    """Layer output for a given routing (idx, w): out[t] = sum_j w[t,j] y_(t,j)."""
    x, w, wgu, wd = _f64(x), _f64(w), _f64(wgu), _f64(wd)
    T, k = idx.shape
    E = wgu.shape[0]
    counts, offsets, perm, inv = dispatch(idx, E)
    d = x.shape[1]
    y_pair = np.zeros((T * k, d))
    for e in range(E):
        pairs = perm[offsets[e]:offsets[e + 1]].astype(np.int64)
        if pairs.size == 0:
            continue
        _, _, y = expert_forward(x[pairs // k], wgu[e], wd[e], limit)
        y_pair[pairs] = y
    y_pair = y_pair.reshape(T, k, d)
    out = np.zeros((T, d))
    for j in range(k):  # slot order
        out += w[:, j:j + 1] * y_pair[:, j, :]
    return out


def forward(x, logits, wgu, wd, k, limit=0.0):
    """Full forward (clamped SwiGLU for limit > 0).  Returns a dict with out and every intermediate.

    h, a, y are stored per flat pair index (t*k + j) so that they do not depend
    on any particular sorted layout.
    """
    x, wgu, wd = _f64(x), _f64(wgu), _f64(wd)
    T, d = x.shape
    E, twoI, _ = wgu.shape
    I = twoI // 2
    idx, w = route(logits, k)
    counts, offsets, perm, inv = dispatch(idx, E)
    h = np.zeros((T * k, twoI))
    a = np.zeros((T * k, I))
    y = np.zeros((T * k, d))
    for e in range(E):
        pairs = perm[offsets[e]:offsets[e + 1]].astype(np.int64)
        if pairs.size == 0:
            continue
        he, ae, ye = expert_forward(x[pairs // k], wgu[e], wd[e], limit)
        h[pairs], a[pairs], y[pairs] = he, ae, ye
    out = np.zeros((T, d))
    yk = y.reshape(T, k, d)
    for j in range(k):
        out += w[:, j:j + 1] * yk[:, j, :]
    return dict(out=out, idx=idx, w=w, counts=counts, offsets=offsets,
                perm=perm, inv=inv, h=h, a=a, y=y)


def dense_forward(x, logits, wgu, wd, k, limit=0.0):
    """Brute force: every expert on every token, masked by the routing.

    M[t, e] = w[t, j] if expert e is token t's j-th choice, else 0;
    out = sum_e M[:, e] * expert_e(x).  Used only to pin the sparse path.
    """
    x, wgu, wd = _f64(x), _f64(wgu), _f64(wd)
    T, d = x.shape
    E = wgu.shape[0]
    idx, w = route(logits, k)
    M = np.zeros((T, E))
    for t in range(T):
        for j in range(k):
            M[t, idx[t, j]] = w[t, j]
    out = np.zeros((T, d))
    for e in range(E):
        _, _, ye = expert_forward(x, wgu[e], wd[e], limit)
        out += M[:, e:e + 1] * ye
    return out


# ----------------------------------------------------------------------------
# backward
# ----------------------------------------------------------------------------
def _pair_backward(x_rows, gout_rows, w_rows, wgu_e, wd_e, limit=0.0, h_rows=None):
    """Backward of one expert's block of pairs (h_rows: the forward's h for
    these pairs, else recomputed from x).

    Returns (dx_rows [n,d] unscaled contribution to dx[t], dscore [n],
    dwgu_e [2I,d], dwd_e [d,I], dh [n,2I]).
    """
    I = wd_e.shape[1]
    h = x_rows @ wgu_e.T if h_rows is None else h_rows
    g, u = h[:, :I], h[:, I:]
    a = swiglu(g, u, limit)
    G = gout_rows @ wd_e                    # W_down[e]^T gout[t]   [n, I]
    dscore = np.sum(G * a, axis=1)          # <G, a> = <gout[t], y_p>
    da = w_rows[:, None] * G
    dg, du = swiglu_backward(g, u, da, limit)
    dh = np.concatenate([dg, du], axis=1)   # [n, 2I]
    dwd_e = (w_rows[:, None] * gout_rows).T @ a   # sum_p (w gout) (x) a
    dx_rows = dh @ wgu_e                    # W_gate_up[e]^T dh      [n, d]
    dwgu_e = dh.T @ x_rows                  # sum_p dh (x) x[t]
    return dx_rows, dscore, dwgu_e, dwd_e, dh


def routing_backward(w, dscore):
    """dlogits from dscore through the renormalised top-k softmax.

    For chosen experts i: dlogit_i = w_i (dscore_i - sum_j w_j dscore_j);
    unchosen experts get 0.  Returned in slot layout [T, k].
    """
    w, dscore = _f64(w), _f64(dscore)
    s = np.sum(w * dscore, axis=1, keepdims=True)
    return w * (dscore - s)


def backward(x, logits, wgu, wd, k, gout, fwd=None, limit=0.0, h=None):
    """Full backward for loss L with dL/dout = gout.

    h: the gate/up pre-activations the forward saved, per flat pair
    [T*k, 2I] (the MXFP8 forward's, for a bf16 backward after it); None
    recomputes them from x.  Returns dict(dx [T,d], dwgu [E,2I,d],
    dwd [E,d,I], dscore [T,k], dlogits [T,E], dh [T*k, 2I] per flat pair).
    """
    x, wgu, wd, gout = _f64(x), _f64(wgu), _f64(wd), _f64(gout)
    T, d = x.shape
    E, twoI, _ = wgu.shape
    if fwd is None:
        idx, w = route(logits, k)
        counts, offsets, perm, inv = dispatch(idx, E)
    else:
        idx, w, offsets, perm = fwd["idx"], fwd["w"], fwd["offsets"], fwd["perm"]
    dx_pair = np.zeros((T * k, d))
    dscore = np.zeros(T * k)
    dh = np.zeros((T * k, twoI))
    dwgu = np.zeros_like(wgu)
    dwd = np.zeros_like(wd)
    wf = w.reshape(-1)
    for e in range(E):
        pairs = perm[offsets[e]:offsets[e + 1]].astype(np.int64)
        if pairs.size == 0:
            continue
        t = pairs // k
        dxr, ds, dwgu[e], dwd[e], dhe = _pair_backward(x[t], gout[t], wf[pairs], wgu[e], wd[e], limit,
                                                        None if h is None else _f64(h)[pairs])
        dx_pair[pairs], dscore[pairs], dh[pairs] = dxr, ds, dhe
    dx = np.zeros((T, d))
    dxk = dx_pair.reshape(T, k, d)
    for j in range(k):  # slot order
        dx += dxk[:, j, :]
    dscore = dscore.reshape(T, k)
    dl_slots = routing_backward(w, dscore)
    dlogits = np.zeros((T, E))
    np.put_along_axis(dlogits, idx.astype(np.int64), dl_slots, axis=1)
    return dict(dx=dx, dwgu=dwgu, dwd=dwd, dscore=dscore, dlogits=dlogits, dh=dh)


# ----------------------------------------------------------------------------
# sampled variants, for checking very large layers one output at a time
# ----------------------------------------------------------------------------
def forward_tokens(x, logits, wgu, wd, k, tokens, limit=0.0):
    """out rows for the listed tokens only (same arithmetic as forward)."""
    tokens = np.asarray(tokens, dtype=np.int64)
    idx, w = route(np.asarray(logits)[tokens], k)
    xt = _f64(np.asarray(x)[tokens])
    out = np.zeros((tokens.size, xt.shape[1]))
    for j in range(k):
        for r in range(tokens.size):
            e = int(idx[r, j])
            _, _, y = expert_forward(xt[r:r + 1], _f64(wgu[e]), _f64(wd[e]), limit)
            out[r] += w[r, j] * y[0]
    return dict(out=out, idx=idx, w=w)


def backward_tokens(x, logits, wgu, wd, k, gout, tokens, limit=0.0):
    """dx, dscore and dlogits rows for the listed tokens only."""
    tokens = np.asarray(tokens, dtype=np.int64)
    logits = np.asarray(logits)
    E = logits.shape[1]
    idx, w = route(logits[tokens], k)
    xt = _f64(np.asarray(x)[tokens])
    gt = _f64(np.asarray(gout)[tokens])
    dx = np.zeros_like(xt)
    dscore = np.zeros((tokens.size, k))
    for j in range(k):
        for r in range(tokens.size):
            e = int(idx[r, j])
            dxr, ds, _, _, _ = _pair_backward(xt[r:r + 1], gt[r:r + 1], w[r, j:j + 1],
                                              _f64(wgu[e]), _f64(wd[e]), limit)
            dx[r] += dxr[0]
            dscore[r, j] = ds[0]
    dl_slots = routing_backward(w, dscore)
    dlogits = np.zeros((tokens.size, E))
    np.put_along_axis(dlogits, idx.astype(np.int64), dl_slots, axis=1)
    return dict(dx=dx, dscore=dscore, dlogits=dlogits, idx=idx, w=w)


def backward_experts(x, logits, wgu, wd, k, gout, experts, limit=0.0):
    """dW_gate_up[e] and dW_down[e] for the listed experts only."""
    logits = np.asarray(logits)
    E = logits.shape[1]
    idx, w = route(logits, k)
    counts, offsets, perm, inv = dispatch(idx, E)
    wf = w.reshape(-1)
    res = {}
    for e in experts:
        e = int(e)
        pairs = perm[offsets[e]:offsets[e + 1]].astype(np.int64)
        wgu_e, wd_e = _f64(wgu[e]), _f64(wd[e])
        if pairs.size == 0:
            res[e] = (np.zeros_like(wgu_e), np.zeros_like(wd_e))
            continue
        t = pairs // k
        _, _, dwgu_e, dwd_e, _ = _pair_backward(_f64(np.asarray(x)[t]), _f64(np.asarray(gout)[t]),
                                                wf[pairs], wgu_e, wd_e, limit)
        res[e] = (dwgu_e, dwd_e)
    return res


# ----------------------------------------------------------------------------
# MXFP8 operands: E4M3 elements with one UE8M0 (power-of-two) scale per block of
# 32 consecutive elements along a GEMM's K dimension ("Prime Intellect's Prime
# Mega MoE Trains Giant AI Models 55% Faster", section "Precision and hardware
# support": MXFP8 on Blackwell uses small microscaling groups).
#
# Readings (the pages give no formula):
#   * block scale X = 2^s with s the smallest integer such that amax <= 448 * 2^s
#     (448 is the largest E4M3 magnitude), clamped to [-127, 127]; an all-zero
#     block has s = 0.
#   * element code = v / X rounded to the nearest E4M3 value, ties to the even
#     code, magnitudes above 448 saturating to 448; the dequantised value is
#     code * X.
#   * the operands quantised are those of the library's six GEMMs, each along
#     that GEMM's K (see forward_mx / backward_mx); for the two weight-gradient
#     GEMMs K runs over an expert's tokens in sorted order, in blocks of 32
#     starting at the expert's first pair.
# ----------------------------------------------------------------------------
E4M3_MAX = 448.0


def e4m3_round(y):
    """Nearest E4M3 value (ties to even code), saturating at +-448.

    E4M3: 3 mantissa bits, exponent bias 7, normal binades from 2^-6 up to
    448 = 1.75 * 2^8, subnormal spacing 2^-9.
    """
    y = np.asarray(y, dtype=np.float64)
    a = np.abs(y)
    out = np.zeros_like(a)
    nz = a > 0
    e = np.floor(np.log2(np.where(nz, a, 1.0)))
    # guard against log2 rounding: enforce 2^e <= a < 2^(e+1)
    e = np.where(np.exp2(e) > a, e - 1, e)
    e = np.where(np.exp2(e + 1) <= a, e + 1, e)
    e = np.maximum(e, -6.0)                  # below 2^-6 the spacing stays 2^-9
    q = np.exp2(e - 3.0)                     # spacing of the binade
    r = np.round(a / q) * q                  # a / q is exact; np.round is ties-to-even
    r = np.minimum(r, E4M3_MAX)
    out[nz] = r[nz]
    return np.copysign(out, y)


def mx_scale_exponent(amax):
    """Smallest integer s with amax <= 448 * 2^s (0 for amax = 0), clamped to [-127, 127]."""
    amax = np.asarray(amax, dtype=np.float64)
    s = np.zeros_like(amax)
    nz = amax > 0
    est = np.ceil(np.log2(np.where(nz, amax, 1.0) / E4M3_MAX))
    # exact correction of the estimate with exact comparisons
    est = np.where(amax > E4M3_MAX * np.exp2(est), est + 1, est)
    est = np.where(amax <= E4M3_MAX * np.exp2(est - 1), est - 1, est)
    s[nz] = est[nz]
    return np.clip(s, -127, 127)


def mx_qdq_blocks(v, axis):
    """Quantise-dequantise v in blocks of 32 consecutive elements along `axis`."""
    v = np.asarray(v, dtype=np.float64)
    v = np.moveaxis(v, axis, -1)
    n = v.shape[-1]
    pad = (-n) % 32
    if pad:
        v = np.concatenate([v, np.zeros(v.shape[:-1] + (pad,))], axis=-1)
    blk = v.reshape(v.shape[:-1] + (-1, 32))
    s = mx_scale_exponent(np.max(np.abs(blk), axis=-1, keepdims=True))
    X = np.exp2(s)
    out = (e4m3_round(blk / X) * X).reshape(v.shape)[..., :n]
    return np.moveaxis(out, -1, axis)


def forward_mx(x, logits, wgu, wd, k, limit=0.0):
    """Forward with MXFP8 GEMM operands.

    Gate/up GEMM: x and W_gate_up quantised along d.  Down GEMM: its operand
    aw = w * silu(gate) * up (the routing weight folded into the activation)
    and W_down quantised along I; out[t] = sum over slots of the down products.
    Returns the same dict as forward, plus aw (per flat pair).
    """
    x, wgu, wd = _f64(x), _f64(wgu), _f64(wd)
    T, d = x.shape
    E, twoI, _ = wgu.shape
    I = twoI // 2
    idx, w = route(logits, k)
    counts, offsets, perm, inv = dispatch(idx, E)
    xq = mx_qdq_blocks(x, axis=1)
    wguq = mx_qdq_blocks(wgu, axis=2)
    wdq = mx_qdq_blocks(wd, axis=2)
    wf = w.reshape(-1)
    h = np.zeros((T * k, twoI))
    aw = np.zeros((T * k, I))
    y = np.zeros((T * k, d))
    for e in range(E):
        pairs = perm[offsets[e]:offsets[e + 1]].astype(np.int64)
        if pairs.size == 0:
            continue
        he = xq[pairs // k] @ wguq[e].T
        ae = wf[pairs][:, None] * swiglu(he[:, :I], he[:, I:], limit)
        h[pairs], aw[pairs] = he, ae
        y[pairs] = mx_qdq_blocks(ae, axis=1) @ wdq[e].T
    out = np.zeros((T, d))
    yk = y.reshape(T, k, d)
    for j in range(k):
        out += yk[:, j, :]
    return dict(out=out, idx=idx, w=w, counts=counts, offsets=offsets, perm=perm, inv=inv, h=h, aw=aw, y=y)


def backward_mx(x, logits, wgu, wd, k, gout, fwd, limit=0.0):
    """Backward with MXFP8 GEMM operands (fwd = forward_mx's result).

    Down dgrad: grad_out rows and W_down along d.  Gate/up dgrad: dh and
    W_gate_up along 2I.  Weight gradients: both operands along the expert's
    tokens (sorted order, blocks of 32 from the expert's first pair).  The
    SwiGLU backward and dscore use the unquantised h.
    """
    x, wgu, wd, gout = _f64(x), _f64(wgu), _f64(wd), _f64(gout)
    T, d = x.shape
    E, twoI, _ = wgu.shape
    I = twoI // 2
    idx, w, offsets, perm = fwd["idx"], fwd["w"], fwd["offsets"], fwd["perm"]
    wf = w.reshape(-1)
    goutq_d = mx_qdq_blocks(gout, axis=1)
    wdq_d = mx_qdq_blocks(wd, axis=1)        # W_down[e] is [d, I]: blocks along d
    wguq_2i = mx_qdq_blocks(wgu, axis=1)     # W_gate_up[e] is [2I, d]: blocks along 2I
    dx_pair = np.zeros((T * k, d))
    dscore = np.zeros(T * k)
    dwgu = np.zeros_like(wgu)
    dwd = np.zeros_like(wd)
    for e in range(E):
        pairs = perm[offsets[e]:offsets[e + 1]].astype(np.int64)
        if pairs.size == 0:
            continue
        t = pairs // k
        he = fwd["h"][pairs]
        g, u = he[:, :I], he[:, I:]
        a = swiglu(g, u, limit)
        G = goutq_d[t] @ wdq_d[e]
        dscore[pairs] = np.sum(G * a, axis=1)
        da = wf[pairs][:, None] * G
        dh = np.concatenate(swiglu_backward(g, u, da, limit), axis=1)
        dx_pair[pairs] = mx_qdq_blocks(dh, axis=1) @ wguq_2i[e]
        # K = the expert's tokens in sorted order, blocks of 32 from its first pair
        dwd[e] = mx_qdq_blocks(gout[t], axis=0).T @ mx_qdq_blocks(fwd["aw"][pairs], axis=0)
        dwgu[e] = mx_qdq_blocks(dh, axis=0).T @ mx_qdq_blocks(x[t], axis=0)
    dx = np.zeros((T, d))
    dxk = dx_pair.reshape(T, k, d)
    for j in range(k):
        dx += dxk[:, j, :]
    dscore = dscore.reshape(T, k)
    dl_slots = routing_backward(w, dscore)
    dlogits = np.zeros((T, E))
    np.put_along_axis(dlogits, idx.astype(np.int64), dl_slots, axis=1)
    return dict(dx=dx, dwgu=dwgu, dwd=dwd, dscore=dscore, dlogits=dlogits)


# ----------------------------------------------------------------------------
# sampled MXFP8 variants (same quantisation as forward_mx / backward_mx)
# ----------------------------------------------------------------------------
class _MxWeights:
    """Per-expert quantised weights, computed on first use."""

    def __init__(self, wgu, wd):
        self.wgu, self.wd, self.cache = wgu, wd, {}

    def get(self, e):
        if e not in self.cache:
            wgu_e, wd_e = _f64(self.wgu[e]), _f64(self.wd[e])
            self.cache[e] = dict(gu_d=mx_qdq_blocks(wgu_e, axis=1), d_i=mx_qdq_blocks(wd_e, axis=1),
                                 d_d=mx_qdq_blocks(wd_e, axis=0), gu_2i=mx_qdq_blocks(wgu_e, axis=0))
        return self.cache[e]


def forward_tokens_mx(x, logits, wgu, wd, k, tokens, weights=None, limit=0.0):
    """out rows of forward_mx for the listed tokens only."""
    tokens = np.asarray(tokens, dtype=np.int64)
    idx, w = route(np.asarray(logits)[tokens], k)
    W = weights or _MxWeights(wgu, wd)
    xq = mx_qdq_blocks(_f64(np.asarray(x)[tokens]), axis=1)
    I = np.asarray(wd).shape[2]
    out = np.zeros((tokens.size, xq.shape[1]))
    for r in range(tokens.size):
        for j in range(k):
            q = W.get(int(idx[r, j]))
            h = xq[r:r + 1] @ q["gu_d"].T
            aw = w[r, j] * swiglu(h[:, :I], h[:, I:], limit)
            out[r] += (mx_qdq_blocks(aw, axis=1) @ q["d_i"].T)[0]
    return dict(out=out, idx=idx, w=w)


def backward_tokens_mx(x, logits, wgu, wd, k, gout, tokens, weights=None, limit=0.0):
    """dx, dscore and dlogits rows of backward_mx for the listed tokens only."""
    tokens = np.asarray(tokens, dtype=np.int64)
    logits = np.asarray(logits)
    E = logits.shape[1]
    idx, w = route(logits[tokens], k)
    W = weights or _MxWeights(wgu, wd)
    I = np.asarray(wd).shape[2]
    xq = mx_qdq_blocks(_f64(np.asarray(x)[tokens]), axis=1)
    gq = mx_qdq_blocks(_f64(np.asarray(gout)[tokens]), axis=1)
    dx = np.zeros_like(xq)
    dscore = np.zeros((tokens.size, k))
    for r in range(tokens.size):
        for j in range(k):
            q = W.get(int(idx[r, j]))
            h = xq[r:r + 1] @ q["gu_d"].T
            g, u = h[:, :I], h[:, I:]
            G = gq[r:r + 1] @ q["d_d"]
            dscore[r, j] = np.sum(G * swiglu(g, u, limit))
            da = w[r, j] * G
            dh = np.concatenate(swiglu_backward(g, u, da, limit), axis=1)
            dx[r] += (mx_qdq_blocks(dh, axis=1) @ q["gu_2i"])[0]
    dl_slots = routing_backward(w, dscore)
    dlogits = np.zeros((tokens.size, E))
    np.put_along_axis(dlogits, idx.astype(np.int64), dl_slots, axis=1)
    return dict(dx=dx, dscore=dscore, dlogits=dlogits, idx=idx, w=w)


def backward_experts_mx(x, logits, wgu, wd, k, gout, experts, weights=None, limit=0.0):
    """dW_gate_up[e] and dW_down[e] of backward_mx for the listed experts only."""
    logits = np.asarray(logits)
    E = logits.shape[1]
    idx, w = route(logits, k)
    counts, offsets, perm, inv = dispatch(idx, E)
    wf = w.reshape(-1)
    W = weights or _MxWeights(wgu, wd)
    I = np.asarray(wd).shape[2]
    res = {}
    for e in experts:
        e = int(e)
        pairs = perm[offsets[e]:offsets[e + 1]].astype(np.int64)
        if pairs.size == 0:
            res[e] = (np.zeros(np.asarray(wgu[e]).shape), np.zeros(np.asarray(wd[e]).shape))
            continue
        q = W.get(e)
        t = pairs // k
        xr = _f64(np.asarray(x)[t])
        gr = _f64(np.asarray(gout)[t])
        h = mx_qdq_blocks(xr, axis=1) @ q["gu_d"].T
        g, u = h[:, :I], h[:, I:]
        aw = wf[pairs][:, None] * swiglu(g, u, limit)
        G = mx_qdq_blocks(gr, axis=1) @ q["d_d"]
        da = wf[pairs][:, None] * G
        dh = np.concatenate(swiglu_backward(g, u, da, limit), axis=1)
        dwd_e = mx_qdq_blocks(gr, axis=0).T @ mx_qdq_blocks(aw, axis=0)
        dwgu_e = mx_qdq_blocks(dh, axis=0).T @ mx_qdq_blocks(xr, axis=0)
        res[e] = (dwgu_e, dwd_e)
    return res

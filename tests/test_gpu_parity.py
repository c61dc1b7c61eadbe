"""GPU parity: the CUDA layer (through the C ABI) against the fp64 CPU oracle.

Routing indices, counts, offsets, permutation and inverse must match bit for
bit; out, h, aw and every gradient must match within the normwise relative
tolerance TOL_BF16 (bf16 operands, fp32 accumulation).  Small cases and the
Qwen3-30B-A3B-shaped workloads (uniform and skewed routing) are checked in
full, every token and every expert; the Qwen3-235B-A22B-shaped workload on
sampled tokens and on experts spread over the load distribution (the busiest
among them), which the oracle computes one by one.
"""
import numpy as np
import pytest
import torch

from helpers import TOL_BF16, check_routing, f64, make, normwise, run_layer, sorted_rows
from oracle import moe_oracle as O
from grouped_gemm_route_b200 import moe as M

pytestmark = pytest.mark.gpu


def full_check(cfg, inp, backward=True, check_h=True):
    T, d, E, k, I = (cfg[n] for n in ("T", "d", "E", "k", "I"))
    layer, res = run_layer(inp, T, d, E, k, I, backward=backward)
    assert res["status"] == 0
    logits = inp["logits"].numpy()
    check_routing(res["saved"], logits, k)
    x, wgu, wd = f64(inp["x"]), f64(inp["wgu"]), f64(inp["wd"])
    ref = O.forward(x, logits, wgu, wd, k)
    errs = dict(out=normwise(f64(res["out"]), ref["out"]))
    if check_h:
        errs["h"] = normwise(sorted_rows(res["saved"], "h"), ref["h"])
        errs["aw"] = normwise(sorted_rows(res["saved"], "aw"), ref["w"].reshape(-1, 1) * ref["a"])
    if backward:
        g = O.backward(x, logits, wgu, wd, k, f64(inp["gout"]), ref)
        for name in ("dx", "dwgu", "dwd", "dscore", "dlogits"):
            errs[name] = normwise(f64(res[name]), g[name])
        # experts without tokens: exact-zero weight gradients
        empty = np.nonzero(ref["counts"] == 0)[0]
        for e in empty:
            assert torch.count_nonzero(res["dwgu"][e]) == 0 and torch.count_nonzero(res["dwd"][e]) == 0
    bad = {n: v for n, v in errs.items() if not v <= TOL_BF16}
    assert not bad, f"normwise errors above {TOL_BF16}: {bad} (all: {errs})"
    return errs


def test_tiny_workload():
    cfg, inp = make("tiny")
    full_check(cfg, inp)


@pytest.mark.parametrize("sizes", [
    dict(T=1000, d=384, E=16, k=4, I=384),   # 128-wide N tiles, ragged groups
    dict(T=700, d=512, E=12, k=3, I=256),    # 256-wide N tiles
    dict(T=333, d=256, E=4, k=1, I=128),     # k = 1
    dict(T=130, d=256, E=8, k=8, I=128),     # k = E
    dict(T=1, d=256, E=8, k=2, I=128),       # a single token
    dict(T=200, d=256, E=48, k=40, I=128),   # k > 32: the sort reads inv in two chunks, the combine five
    dict(T=96, d=128, E=64, k=64, I=128),    # the largest k, = E: every expert takes every token
    dict(T=500, d=128, E=8, k=2, I=128),     # d = 128: rows of 16 pieces, half of each sorting warp idle
])
def test_multi_tile_ragged(sizes):
    cfg, inp = make(sizes, seed=3)
    full_check(cfg, inp)


def test_empty_and_dominant_experts():
    cfg, inp = make(dict(T=600, d=256, E=16, k=2, I=256), seed=5)
    lg = inp["logits"]
    lg[:, 5] = -100.0   # never chosen
    lg[:, 9] = -100.0
    lg[:, 3] += 100.0   # chosen first by every token
    full_check(cfg, inp)


def test_tied_logits():
    cfg, inp = make(dict(T=512, d=256, E=16, k=4, I=128), seed=7)
    lg = inp["logits"]
    lg.copy_(torch.round(lg * 2) / 2)
    lg[::7] = 0.25       # fully tied rows -> experts 0..k-1
    full_check(cfg, inp)


def test_deterministic_bitwise():
    cfg, inp = make(dict(T=900, d=256, E=16, k=4, I=256), seed=11)
    T, d, E, k, I = (cfg[n] for n in ("T", "d", "E", "k", "I"))
    layer, r1 = run_layer(inp, T, d, E, k, I)
    _, r2 = run_layer(inp, T, d, E, k, I, layer=layer)
    for name in ("out", "dx", "dwgu", "dwd", "dscore", "dlogits"):
        assert torch.equal(r1[name], r2[name]), name


def spread_experts(counts, n=8):
    """The busiest expert, the least loaded non-empty one and experts at evenly
    spaced ranks of the load in between (n in all when there are enough)."""
    order = np.argsort(counts, kind="stable")
    nonempty = order[counts[order] > 0]
    pick = {int(order[-1]), int(nonempty[0])}
    for q in np.linspace(0, len(nonempty) - 1, n):
        if len(pick) >= n:
            break
        pick.add(int(nonempty[int(round(q))]))
    return sorted(pick)


def _sampled_check(name, seed=0, n_tokens=48, experts=None):
    cfg, inp = make(name, seed=seed)
    T, d, E, k, I = (cfg[n] for n in ("T", "d", "E", "k", "I"))
    layer, res = run_layer(inp, T, d, E, k, I)
    assert res["status"] == 0
    logits = inp["logits"].numpy()
    idx_ref, _ = check_routing(res["saved"], logits, k)
    rng = np.random.default_rng(seed + 1)
    toks = np.sort(rng.choice(T, size=n_tokens, replace=False))
    toks[0], toks[-1] = 0, T - 1
    x, gout = inp["x"].float().numpy(), inp["gout"].float().numpy()
    wgu, wd = inp["wgu"], inp["wd"]
    wgu_np, wd_np = wgu.float().numpy(), wd.float().numpy()
    ft = O.forward_tokens(x, logits, wgu_np, wd_np, k, toks)
    errs = dict(out=normwise(f64(res["out"])[toks], ft["out"]))
    bt = O.backward_tokens(x, logits, wgu_np, wd_np, k, gout, toks)
    for n in ("dx", "dscore", "dlogits"):
        errs[n] = normwise(f64(res[n])[toks], bt[n])
    counts = np.bincount(idx_ref.reshape(-1), minlength=E)
    if experts is None:
        experts = spread_experts(counts)
    assert int(np.argmax(counts)) in experts
    be = O.backward_experts(x, logits, wgu_np, wd_np, k, gout, experts)
    for e in experts:
        errs[f"dwgu[{e}]"] = normwise(f64(res["dwgu"][e]), be[e][0])
        errs[f"dwd[{e}]"] = normwise(f64(res["dwd"][e]), be[e][1])
    for e in np.nonzero(counts == 0)[0]:
        assert torch.count_nonzero(res["dwgu"][e]) == 0 and torch.count_nonzero(res["dwd"][e]) == 0
    bad = {n: v for n, v in errs.items() if not v <= TOL_BF16}
    assert not bad, f"normwise errors above {TOL_BF16}: {bad} (all: {errs})"
    return errs


@pytest.mark.slow
def test_qwen3_30b_full_size_every_output():
    """The 30B workload at full size: every token's out and dx, every pair's h
    and aw, every expert's dW, all against the full fp64 oracle."""
    cfg, inp = make("qwen3_30b_a3b", seed=0)
    full_check(cfg, inp)


@pytest.mark.slow
def test_qwen3_30b_skewed_routing_full_size_every_output():
    """The skewed 30B workload at full size, in full: the busiest expert
    (about 16,000 pairs: the longest weight-gradient K loops) and the empty
    ones (exact-zero weight gradients) included."""
    from grouped_gemm_route_b200 import inputs as IN
    cfg = dict(IN.WORKLOADS["qwen3_30b_a3b_skew"])
    lg = IN.make_logits(cfg["T"], cfg["E"], seed=0, zipf_s=cfg["zipf_s"]).numpy()
    idx, _ = O.route(lg, cfg["k"])
    counts = np.bincount(idx.reshape(-1), minlength=cfg["E"])
    assert (counts == 0).sum() >= 8 and counts.max() > 10 * np.median(counts)
    cfg, inp = make("qwen3_30b_a3b_skew", seed=0)
    full_check(cfg, inp)


@pytest.mark.slow
def test_qwen3_235b_shape_sampled():
    _sampled_check("qwen3_235b_a22b", n_tokens=24)


@pytest.mark.parametrize("max_sms", [7, 3])
def test_results_do_not_depend_on_the_grid(max_sms):
    # every tile (or CTA-pair tile) is computed whole by one CTA or pair and every
    # reduction has a fixed order, so a layer on a few SMs gives the same bits
    cfg, inp = make(dict(T=700, d=512, E=12, k=3, I=256), seed=13)
    T, d, E, k, I = (cfg[n] for n in ("T", "d", "E", "k", "I"))
    x, lg, wgu, wd, gout = (inp[n].cuda() for n in ("x", "logits", "wgu", "wd", "gout"))
    outs = []
    for sms in (0, max_sms):
        layer = M.MoELayer(T, d, E, k, I, max_sms=sms)
        o = layer.forward(x, lg, wgu, wd).clone()
        g = {n: t.clone() for n, t in layer.backward(gout, x, wgu, wd).items()}
        torch.cuda.synchronize()
        assert layer.status() == 0
        outs.append((o, g))
    assert torch.equal(outs[0][0], outs[1][0])
    for n in ("dx", "dwgu", "dwd", "dscore", "dlogits"):
        assert torch.equal(outs[0][1][n], outs[1][1][n]), n


def test_single_sm_runs_the_one_cta_kernels():
    """On one SM no CTA pair fits: every GEMM runs on the one-CTA kernels (the
    bf16 gate/up forward with its cp.async gather), checked against the oracle."""
    cfg, inp = make(dict(T=300, d=256, E=8, k=2, I=256), seed=17)
    T, d, E, k, I = (cfg[n] for n in ("T", "d", "E", "k", "I"))
    layer = M.MoELayer(T, d, E, k, I, device="cuda", max_sms=1)
    _, res = run_layer(inp, T, d, E, k, I, layer=layer)
    assert res["status"] == 0
    logits = inp["logits"].numpy()
    check_routing(res["saved"], logits, k)
    x, wgu, wd = f64(inp["x"]), f64(inp["wgu"]), f64(inp["wd"])
    ref = O.forward(x, logits, wgu, wd, k)
    g = O.backward(x, logits, wgu, wd, k, f64(inp["gout"]), ref)
    errs = dict(out=normwise(f64(res["out"]), ref["out"]))
    for name in ("dx", "dwgu", "dwd", "dscore", "dlogits"):
        errs[name] = normwise(f64(res[name]), g[name])
    assert all(v <= TOL_BF16 for v in errs.values()), errs


@pytest.mark.parametrize("dtype", [M.MOE_BF16, M.MOE_MXFP8])
def test_sorted_x_kept_or_not_gives_the_same_bits(dtype):
    """With saved xs the forward keeps its sorted copy of x and the backward
    skips sorting x; without it the backward sorts x itself: same results."""
    cfg, inp = make(dict(T=700, d=512, E=12, k=3, I=256), seed=31)
    T, d, E, k, I = (cfg[n] for n in ("T", "d", "E", "k", "I"))
    runs = []
    for keep in (True, False):
        layer = M.MoELayer(T, d, E, k, I, device="cuda", dtype=dtype, keep_sorted_x=keep)
        _, res = run_layer(inp, T, d, E, k, I, layer=layer)
        assert res["status"] == 0
        assert (res["saved"]["xs"] is not None) == keep
        runs.append(res)
    for name in ("out", "dx", "dwgu", "dwd", "dscore", "dlogits"):
        assert torch.equal(runs[0][name], runs[1][name]), name

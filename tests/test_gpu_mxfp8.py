"""GPU parity of the MXFP8 layer (E4M3 operands, UE8M0 scales per 32 along K).

The CUDA path runs block-scaled tcgen05 MMAs; the oracle applies the same
operand quantisation (forward_mx / backward_mx) and computes in fp64.
Routing must match bit for bit; h (the gate/up GEMM output on quantised x and
W_gate_up) and every output and gradient within TOL_MXFP8 normwise.
"""
import numpy as np
import pytest

from grouped_gemm_route_b200 import moe as M
from helpers import TOL_BF16, TOL_MXFP8, check_routing, f64, make, normwise, run_layer, sorted_rows
from oracle import moe_oracle as O

pytestmark = pytest.mark.gpu


def mx_check(cfg, inp):
    T, d, E, k, I = (cfg[n] for n in ("T", "d", "E", "k", "I"))
    layer, res = run_layer(inp, T, d, E, k, I, dtype=M.MOE_MXFP8)
    assert res["status"] == 0
    logits = inp["logits"].numpy()
    check_routing(res["saved"], logits, k)
    x, wgu, wd, gout = f64(inp["x"]), f64(inp["wgu"]), f64(inp["wd"]), f64(inp["gout"])
    ref = O.forward_mx(x, logits, wgu, wd, k)
    g = O.backward_mx(x, logits, wgu, wd, k, gout, ref)
    errs = dict(h=normwise(sorted_rows(res["saved"], "h"), ref["h"]),
                aw=normwise(sorted_rows(res["saved"], "aw"), ref["aw"]),
                out=normwise(f64(res["out"]), ref["out"]))
    for name in ("dx", "dwgu", "dwd", "dscore", "dlogits"):
        errs[name] = normwise(f64(res[name]), g[name])
    bad = {n: v for n, v in errs.items() if not v <= TOL_MXFP8}
    assert not bad, f"normwise errors above {TOL_MXFP8}: {bad} (all: {errs})"
    # quantisation is visible: the MXFP8 layer is not the bf16 layer
    ref_bf = O.forward(x, logits, wgu, wd, k)
    assert normwise(f64(res["out"]), ref_bf["out"]) > 1e-3
    return errs


def test_mxfp8_tiny():
    cfg, inp = make("tiny")
    mx_check(cfg, inp)


@pytest.mark.parametrize("sizes", [
    dict(T=700, d=512, E=12, k=3, I=256),
    dict(T=1000, d=384, E=16, k=4, I=384),
    dict(T=2048, d=1024, E=16, k=4, I=512),
])
def test_mxfp8_multi_tile(sizes):
    cfg, inp = make(sizes, seed=9)
    mx_check(cfg, inp)


def test_mxfp8_empty_expert():
    cfg, inp = make(dict(T=600, d=256, E=16, k=2, I=256), seed=13)
    inp["logits"][:, 4] = -100.0
    errs = mx_check(cfg, inp)
    assert np.isfinite(list(errs.values())).all()


def test_qwen3_30b_mxfp8_sampled():
    """The MXFP8 30B workload at full size: routing bit-exact over all tokens;
    out / dx / dscore / dlogits on sampled tokens and dW on eight experts spread
    over the load distribution, the busiest among them."""
    cfg, inp = make("qwen3_30b_a3b_mxfp8", seed=0)
    T, d, E, k, I = (cfg[n] for n in ("T", "d", "E", "k", "I"))
    layer, res = run_layer(inp, T, d, E, k, I, dtype=M.MOE_MXFP8)
    assert res["status"] == 0
    logits = inp["logits"].numpy()
    idx_ref, _ = check_routing(res["saved"], logits, k)
    rng = np.random.default_rng(1)
    toks = np.sort(rng.choice(T, size=24, replace=False))
    x, gout = inp["x"].float().numpy(), inp["gout"].float().numpy()
    wgu, wd = inp["wgu"].float().numpy(), inp["wd"].float().numpy()
    W = O._MxWeights(wgu, wd)
    ft = O.forward_tokens_mx(x, logits, wgu, wd, k, toks, weights=W)
    errs = dict(out=normwise(f64(res["out"])[toks], ft["out"]))
    bt = O.backward_tokens_mx(x, logits, wgu, wd, k, gout, toks, weights=W)
    for n in ("dx", "dscore", "dlogits"):
        errs[n] = normwise(f64(res[n])[toks], bt[n])
    counts = np.bincount(idx_ref.reshape(-1), minlength=E)
    order = np.argsort(counts, kind="stable")
    experts = sorted({int(order[int(round(q))]) for q in np.linspace(0, E - 1, 8)})  # busiest included
    assert int(np.argmax(counts)) in experts
    be = O.backward_experts_mx(x, logits, wgu, wd, k, gout, experts, weights=W)
    for e in experts:
        errs[f"dwgu[{e}]"] = normwise(f64(res["dwgu"][e]), be[e][0])
        errs[f"dwd[{e}]"] = normwise(f64(res["dwd"][e]), be[e][1])
    bad = {n: v for n, v in errs.items() if not v <= TOL_MXFP8}
    assert not bad, f"normwise errors above {TOL_MXFP8}: {bad} (all: {errs})"


@pytest.mark.parametrize("sizes", ["tiny", dict(T=700, d=512, E=12, k=3, I=256)])
def test_mxfp8_forward_bf16_backward(sizes):
    """MOE_MXFP8_FWD: the forward of the MXFP8 layer, then the bf16 backward on
    the h and aw that forward saved (oracle: backward with the MXFP8 forward's h)."""
    cfg, inp = make(sizes, seed=21)
    T, d, E, k, I = (cfg[n] for n in ("T", "d", "E", "k", "I"))
    layer, res = run_layer(inp, T, d, E, k, I, dtype=M.MOE_MXFP8_FWD)
    assert res["status"] == 0
    logits = inp["logits"].numpy()
    check_routing(res["saved"], logits, k)
    x, wgu, wd, gout = f64(inp["x"]), f64(inp["wgu"]), f64(inp["wd"]), f64(inp["gout"])
    ref = O.forward_mx(x, logits, wgu, wd, k)
    g = O.backward(x, logits, wgu, wd, k, gout, ref, h=ref["h"])
    errs = dict(h=normwise(sorted_rows(res["saved"], "h"), ref["h"]), out=normwise(f64(res["out"]), ref["out"]))
    for name in ("dx", "dwgu", "dwd", "dscore", "dlogits"):
        errs[name] = normwise(f64(res[name]), g[name])
    bad = {n: v for n, v in errs.items() if not v <= TOL_BF16}
    assert not bad, f"normwise errors above {TOL_BF16}: {bad} (all: {errs})"

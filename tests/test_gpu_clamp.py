"""GPU parity of the clamped SwiGLU (swiglu_limit L > 0: a = silu(min(gate, L))
* clamp(up, -L, L)) against the oracle, in bf16 and MXFP8, forward and
backward.  The backward's clamp sides are decided on bf16 h on both sides.  h holds the unclamped pre-activations; aw the weighted clamped
activation.  A limit above every pre-activation must give the plain layer bit
for bit, and recompute mode must give the clamped layer bit for bit."""
import numpy as np
import pytest
import torch

from grouped_gemm_route_b200 import moe as M
from grouped_gemm_route_b200 import torch_op as TO
from helpers import TOL_BF16, TOL_MXFP8, check_routing, f64, make, normwise, run_layer, sorted_rows
from oracle import moe_oracle as O

pytestmark = pytest.mark.gpu


def clamp_check(cfg, inp, L, dtype):
    T, d, E, k, I = (cfg[n] for n in ("T", "d", "E", "k", "I"))
    layer = M.MoELayer(T, d, E, k, I, device="cuda", dtype=dtype, swiglu_limit=L)
    _, res = run_layer(inp, T, d, E, k, I, layer=layer)
    assert res["status"] == 0
    logits = inp["logits"].numpy()
    check_routing(res["saved"], logits, k)
    x, wgu, wd, gout = f64(inp["x"]), f64(inp["wgu"]), f64(inp["wd"]), f64(inp["gout"])
    if dtype == M.MOE_MXFP8:
        ref = O.forward_mx(x, logits, wgu, wd, k, limit=L)
        g = O.backward_mx(x, logits, wgu, wd, k, gout, ref, limit=L)
        ref_aw, tol = ref["aw"], TOL_MXFP8
    else:
        ref = O.forward(x, logits, wgu, wd, k, limit=L)
        g = O.backward(x, logits, wgu, wd, k, gout, ref, limit=L)
        ref_aw, tol = ref["w"].reshape(-1, 1) * ref["a"], TOL_BF16
    # both clamps are active on a sizeable share of the pre-activations
    hg, hu = ref["h"][:, :I], ref["h"][:, I:]
    assert 0.05 < np.mean(hg > L) < 0.6 and 0.05 < np.mean(np.abs(hu) > L) < 0.9
    errs = dict(h=normwise(sorted_rows(res["saved"], "h"), ref["h"]),
                aw=normwise(sorted_rows(res["saved"], "aw"), ref_aw),
                out=normwise(f64(res["out"]), ref["out"]))
    for name in ("dx", "dwgu", "dwd", "dscore", "dlogits"):
        errs[name] = normwise(f64(res[name]), g[name])
    bad = {n: v for n, v in errs.items() if not v <= tol}
    assert not bad, f"normwise errors above {tol}: {bad} (all: {errs})"
    # the clamp is visible: the clamped layer is not the plain one
    plain = O.forward(x, logits, wgu, wd, k)
    assert normwise(f64(res["out"]), plain["out"]) > 0.05
    return errs


# limits are bfloat16 values, so that the kernel's float32 limit and the oracle's agree exactly
@pytest.mark.parametrize("sizes,L", [
    ("tiny", 0.1875),
    (dict(T=700, d=512, E=12, k=3, I=256), 0.3125),
    (dict(T=1000, d=384, E=16, k=4, I=384), 0.25),
])
def test_clamped_bf16(sizes, L):
    cfg, inp = make(sizes, seed=17)
    clamp_check(cfg, inp, L, M.MOE_BF16)


@pytest.mark.parametrize("sizes,L", [("tiny", 0.1875), (dict(T=700, d=512, E=12, k=3, I=256), 0.3125)])
def test_clamped_mxfp8(sizes, L):
    cfg, inp = make(sizes, seed=19)
    clamp_check(cfg, inp, L, M.MOE_MXFP8)


def test_limit_above_every_preactivation_is_the_plain_layer_bitwise():
    cfg, inp = make(dict(T=700, d=512, E=12, k=3, I=256), seed=23)
    T, d, E, k, I = (cfg[n] for n in ("T", "d", "E", "k", "I"))
    _, plain = run_layer(inp, T, d, E, k, I)
    assert float(plain["saved"]["h"].float().abs().max()) < 1e3
    big = M.MoELayer(T, d, E, k, I, device="cuda", swiglu_limit=1e3)
    _, res = run_layer(inp, T, d, E, k, I, layer=big)
    assert plain["status"] == 0 and res["status"] == 0
    for name in ("out", "dx", "dwgu", "dwd", "dscore", "dlogits"):
        assert torch.equal(plain[name], res[name]), name


def test_clamped_torch_op_recompute_is_bitwise_and_grads_in_input_dtype():
    cfg, inp = make("tiny", seed=29)
    k, L, dev = cfg["k"], 0.1875, "cuda:0"
    gout = inp["gout"].to(dev)
    runs = []
    for recompute in (False, True):
        leaves = [inp[n].to(dev).requires_grad_() for n in ("x", "logits", "wgu", "wd")]
        out = TO.moe_layer(*leaves, k, recompute=recompute, swiglu_limit=L)
        out.backward(gout)
        runs.append([out] + [t.grad for t in leaves])
    torch.cuda.synchronize()
    for a, b in zip(*runs):
        assert torch.equal(a, b)
    x, logits, wgu, wd = (f64(inp[n]) for n in ("x", "logits", "wgu", "wd"))
    ref = O.forward(x, inp["logits"].numpy(), wgu, wd, k, limit=L)
    assert normwise(f64(runs[0][0]), ref["out"]) <= TOL_BF16
    g = O.backward(x, inp["logits"].numpy(), wgu, wd, k, f64(inp["gout"]), ref, limit=L)
    assert normwise(f64(runs[0][1]), g["dx"]) <= TOL_BF16
    assert normwise(f64(runs[0][2]), g["dlogits"]) <= TOL_BF16

"""GPU parity of the clamped SwiGLU (swiglu_limit L > 0: a = silu(min(gate, L))
* clamp(up, -L, L)) against the oracle, in bf16 and MXFP8, forward and
backward.  h holds the unclamped pre-activations; aw the weighted clamped
activation.  A limit above every pre-activation must give the plain layer bit
for bit, and recompute mode must give the clamped layer bit for bit.

The oracle decides each clamp's side on the exact pre-activation; the kernels
decide on their float32 accumulator (forward) and on the bfloat16 h they saved
(backward).  The parity cases therefore take their inputs on coarse grids
(inputs.make_grid_inputs), where every pre-activation is an exact multiple of
2^-8, and limits strictly between two such multiples: the three precisions put
every element on the same side of every clamp, so the comparison measures the
arithmetic, not a different set of decisions."""
import numpy as np
import pytest
import torch

from grouped_gemm_route_b200 import moe as M
from grouped_gemm_route_b200 import torch_op as TO
from grouped_gemm_route_b200 import inputs as IN
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


def make_grid(sizes, seed):
    cfg = dict(IN.WORKLOADS[sizes]) if isinstance(sizes, str) else dict(sizes)
    cfg.pop("dtype", None)
    return cfg, IN.make_grid_inputs(seed=seed, **cfg)


def off_grid(L):
    """The limit lies strictly between two multiples of 2^-8 (and is exact in float32)."""
    return (L * 256) % 1 != 0 and float(np.float32(L)) == L


# limits are odd multiples of 2^-9: between two grid values of h
@pytest.mark.parametrize("sizes,L", [
    ("tiny", 155 / 512),
    (dict(T=700, d=512, E=12, k=3, I=256), 181 / 512),
    (dict(T=1000, d=384, E=16, k=4, I=384), 129 / 512),
])
def test_clamped_bf16(sizes, L):
    assert off_grid(L)
    cfg, inp = make_grid(sizes, seed=17)
    clamp_check(cfg, inp, L, M.MOE_BF16)


@pytest.mark.parametrize("sizes,L", [("tiny", 155 / 512), (dict(T=700, d=512, E=12, k=3, I=256), 181 / 512)])
def test_clamped_mxfp8(sizes, L):
    assert off_grid(L)
    cfg, inp = make_grid(sizes, seed=19)
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
    cfg, inp = make_grid("tiny", seed=29)
    k, L, dev = cfg["k"], 155 / 512, "cuda:0"
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

"""Shared test helpers: run the CUDA layer through the C ABI and compare with the oracle."""
from __future__ import annotations

import numpy as np
import torch

from grouped_gemm_route_b200 import inputs as IN
from grouped_gemm_route_b200 import moe as M
from oracle import moe_oracle as O

# Normwise relative tolerances (fp32 accumulation): bf16 GEMM operands, and
# MXFP8 operands checked against the oracle that applies the same quantisation.
TOL_BF16 = 1e-2
TOL_MXFP8 = 3e-2


def normwise(gpu, ref) -> float:
    gpu = np.asarray(gpu, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    den = np.linalg.norm(ref)
    num = np.linalg.norm(gpu - ref)
    if den == 0.0:
        return float(num)
    return float(num / den)


def f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy().astype(np.float64)


def run_layer(inp: dict, T, d, E, k, I, backward=True, layer=None, dtype=M.MOE_BF16):
    """Run fwd (+bwd) on the GPU; returns the layer and host copies of everything."""
    dev = "cuda"
    x, lg, wgu, wd = (inp[n].to(dev) for n in ("x", "logits", "wgu", "wd"))
    if layer is None:
        layer = M.MoELayer(T, d, E, k, I, device=dev, dtype=dtype)
    layer.forward(x, lg, wgu, wd)
    res = dict(out=layer.out.clone())
    if backward:
        g = layer.backward(inp["gout"].to(dev), x, wgu, wd)
        res.update({n: v.clone() for n, v in g.items() if v is not None})
    torch.cuda.synchronize()
    status = layer.status()
    res["saved"] = {n: v.clone() if v is not None else None for n, v in layer.saved.items()}
    res["status"] = status
    return layer, res


def check_routing(saved: dict, logits: np.ndarray, k: int):
    """Bit-exact comparison of idx / counts / offsets / perm / inv with the oracle."""
    E = logits.shape[1]
    idx_ref, w_ref = O.route(logits, k)
    counts, offsets, perm, inv = O.dispatch(idx_ref, E)
    g_idx = saved["topk_idx"].cpu().numpy()
    assert np.array_equal(g_idx, idx_ref), "topk_idx differs"
    assert np.array_equal(saved["counts"].cpu().numpy(), counts), "counts differ"
    assert np.array_equal(saved["offsets"].cpu().numpy(), offsets), "offsets differ"
    gs = saved["group_start"].cpu().numpy().astype(np.int64)
    pad = (counts.astype(np.int64) + 127) // 128 * 128
    assert gs[0] == 0 and np.array_equal(np.diff(gs), pad), "group starts differ"
    g_perm = saved["perm"].cpu().numpy()
    g_inv = saved["inv"].cpu().numpy()
    tile_e = saved["tile_expert"].cpu().numpy()
    for e in range(E):
        a, c = int(gs[e]), int(counts[e])
        assert np.array_equal(g_perm[a:a + c], perm[offsets[e]:offsets[e + 1]]), f"perm differs in expert {e}"
        assert np.all(g_perm[a + c:int(gs[e + 1])] == -1), f"padding of expert {e}"
        assert np.all(tile_e[a // 128:int(gs[e + 1]) // 128] == e)
    # inv: pair -> padded sorted row
    e_of = idx_ref.reshape(-1)
    expect_inv = gs[e_of] + (inv.reshape(-1) - offsets[e_of])
    assert np.array_equal(g_inv.reshape(-1), expect_inv), "inv differs"
    gw = saved["topk_w"].cpu().numpy().astype(np.float64)
    assert normwise(gw, w_ref) < 1e-6
    return idx_ref, w_ref


def sorted_rows(saved: dict, name: str):
    """Host copy of a sorted-layout tensor (h or aw) gathered back to flat pair order."""
    inv = saved["inv"].cpu().numpy().reshape(-1).astype(np.int64)
    return f64(saved[name][torch.as_tensor(inv, device=saved[name].device)])


def make(cfg_or_sizes, seed=0, **over):
    if isinstance(cfg_or_sizes, str):
        cfg = dict(IN.WORKLOADS[cfg_or_sizes])
    else:
        cfg = dict(cfg_or_sizes)
    cfg.update(over)
    cfg.pop("dtype", None)
    inp = IN.make_inputs(seed=seed, **cfg)
    return cfg, inp

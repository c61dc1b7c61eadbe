"""moe_recompute regenerates h and aw bit-identically from the saved routing,
so that a backward after it gives the same bits as one after moe_fwd (bf16 and
MXFP8, on multi-tile shapes with ragged expert groups)."""
import pytest
import torch

from grouped_gemm_route_b200 import moe as M
from helpers import make

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("sizes,dtype", [
    (dict(T=700, d=512, E=12, k=3, I=256), M.MOE_BF16),
    (dict(T=1000, d=384, E=16, k=4, I=384), M.MOE_BF16),
    (dict(T=600, d=512, E=8, k=2, I=256), M.MOE_MXFP8),
])
def test_recompute_matches_forward(sizes, dtype):
    cfg, inp = make(sizes, seed=2)
    T, d, E, k, I = (cfg[n] for n in ("T", "d", "E", "k", "I"))
    x, lg, wgu, wd, gout = (inp[n].cuda() for n in ("x", "logits", "wgu", "wd", "gout"))
    layer = M.MoELayer(T, d, E, k, I, dtype=dtype)
    layer.forward(x, lg, wgu, wd)
    ref = layer.backward(gout, x, wgu, wd)
    ref = {n: t.clone() for n, t in ref.items()}
    h0, aw0 = layer.saved["h"].clone(), layer.saved["aw"].clone()
    layer.saved["h"].fill_(float("nan"))
    layer.saved["aw"].fill_(float("nan"))
    M.recompute(layer.shape, x, wgu, layer.saved, layer.ws)
    torch.cuda.synchronize()
    assert layer.status() == 0
    used = int(layer.saved["group_start"][E])  # rows past the last group are never read
    assert torch.equal(layer.saved["h"][:used], h0[:used]) and torch.equal(layer.saved["aw"][:used], aw0[:used])
    g = layer.backward(gout, x, wgu, wd)
    torch.cuda.synchronize()
    for n in ("dx", "dwgu", "dwd", "dscore", "dlogits"):
        assert torch.equal(g[n], ref[n]), n

"""CUDA-graph capture of the layer: one forward + backward captured on a side
stream (after an eager warm-up that sets the kernels' launch attributes) and
replayed gives the eager results bit for bit, and replays stay bitwise stable.
The captured sequence holds the routing's cooperative launch, the GEMMs'
persistent launches with their tensor maps as parameters, the status-word
memsets and the second stream the backward forks for the dx sum."""
import pytest
import torch

from grouped_gemm_route_b200 import moe as M
from helpers import make

pytestmark = pytest.mark.gpu

OUTS = ("out", "dx", "dwgu", "dwd", "dscore", "dlogits")


def _results(layer, g):
    r = dict(out=layer.out, **g)
    return {n: r[n].clone() for n in OUTS}


@pytest.mark.parametrize("wl", ["tiny", dict(T=1000, d=384, E=16, k=4, I=384)])
def test_graph_replay_equals_eager(wl):
    cfg, inp = make(wl, seed=5)
    T, d, E, k, I = (cfg[n] for n in ("T", "d", "E", "k", "I"))
    dev = "cuda:0"
    x, lg, wgu, wd, gout = (inp[n].to(dev) for n in ("x", "logits", "wgu", "wd", "gout"))
    layer = M.MoELayer(T, d, E, k, I, device=dev)
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        # eager warm-up on the capture stream (sets the kernels' attributes before capture)
        layer.forward(x, lg, wgu, wd, stream=s)
        g = layer.backward(gout, x, wgu, wd, stream=s)
    torch.cuda.synchronize()
    assert layer.status() == 0
    eager = _results(layer, g)
    layer.out.zero_()  # clear the outputs so that the replay has to rewrite them
    for n in OUTS[1:]:
        g[n].zero_()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=s):
        layer.forward(x, lg, wgu, wd, stream=s)
        layer.backward(gout, x, wgu, wd, stream=s)
    for _ in range(3):
        graph.replay()
        torch.cuda.synchronize()
        assert layer.status() == 0
        rep = _results(layer, g)
        for n in OUTS:
            assert torch.equal(rep[n], eager[n]), n
    del graph

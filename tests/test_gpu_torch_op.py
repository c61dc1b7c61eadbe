"""The PyTorch custom op + autograd wrapper on the GPU: eager autograd gives
the same bits as calling the C ABI directly, and torch.compile(fullgraph=True)
traces through the layer and gives the same bits again."""
import pytest
import torch

from grouped_gemm_route_b200 import inputs as IN
from grouped_gemm_route_b200 import moe as M
from grouped_gemm_route_b200 import torch_op as TO

pytestmark = pytest.mark.gpu


def leaves(inp, dev):
    return [inp[n].to(dev).requires_grad_() for n in ("x", "logits", "wgu", "wd")]


def test_autograd_matches_direct_abi_calls():
    cfg, inp = IN.make_workload("tiny", seed=3, device="cpu")
    T, d, E, k, I = (cfg[n] for n in ("T", "d", "E", "k", "I"))
    dev = "cuda:0"
    x, lg, wgu, wd = leaves(inp, dev)
    gout = inp["gout"].to(dev)
    out = TO.moe_layer(x, lg, wgu, wd, k)
    out.backward(gout)
    torch.cuda.synchronize()
    layer = M.MoELayer(T, d, E, k, I, device=dev)
    ref = layer.forward(x.detach(), lg.detach(), wgu.detach(), wd.detach())
    g = layer.backward(gout, x.detach(), wgu.detach(), wd.detach())
    torch.cuda.synchronize()
    assert layer.status() == 0
    assert torch.equal(out, ref)
    assert torch.equal(x.grad, g["dx"]) and torch.equal(lg.grad, g["dlogits"])
    assert torch.equal(wgu.grad, g["dwgu"]) and torch.equal(wd.grad, g["dwd"])


def test_compile_fullgraph_matches_eager():
    cfg, inp = IN.make_workload("tiny", seed=4, device="cpu")
    k = cfg["k"]
    dev = "cuda:0"
    gout = inp["gout"].to(dev)

    def loss(x, lg, wgu, wd):
        return (TO.moe_layer(x, lg, wgu, wd, k).float() * gout.float()).sum()

    eager = leaves(inp, dev)
    loss(*eager).backward()
    comp = leaves(inp, dev)
    torch.compile(loss, fullgraph=True)(*comp).backward()
    torch.cuda.synchronize()
    for a, b in zip(eager, comp):
        assert torch.equal(a.grad, b.grad)

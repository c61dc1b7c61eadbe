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


def test_caller_dtypes_in_and_out():
    cfg, inp = IN.make_workload("tiny", seed=5, device="cpu")
    k = cfg["k"]
    dev = "cuda:0"
    x = inp["x"].to(dev).float().requires_grad_()
    lg = inp["logits"].to(dev).double().requires_grad_()
    wgu = inp["wgu"].to(dev).float().requires_grad_()
    wd = inp["wd"].to(dev).requires_grad_()
    out = TO.moe_layer(x, lg, wgu, wd, k)
    assert out.dtype == torch.float32
    out.backward(inp["gout"].to(dev).float())
    assert x.grad.dtype == torch.float32 and lg.grad.dtype == torch.float64
    assert wgu.grad.dtype == torch.float32 and wd.grad.dtype == torch.bfloat16
    # same numbers as the all-bf16 call
    ref = leaves(inp, dev)
    TO.moe_layer(*ref, k).backward(inp["gout"].to(dev))
    assert torch.equal(x.grad.to(torch.bfloat16), ref[0].grad)
    assert torch.equal(wd.grad, ref[3].grad)


def test_recompute_mode_same_bits():
    cfg, inp = IN.make_workload("tiny", seed=6, device="cpu")
    k = cfg["k"]
    dev = "cuda:0"
    gout = inp["gout"].to(dev)
    a = leaves(inp, dev)
    TO.moe_layer(*a, k).backward(gout)
    b = leaves(inp, dev)
    TO.moe_layer(*b, k, recompute=True).backward(gout)
    torch.cuda.synchronize()
    for p, q in zip(a, b):
        assert torch.equal(p.grad, q.grad)

"""PyTorch custom ops and autograd for the fused MoE layer.

    out = moe_layer(x, logits, w_gate_up, w_down, top_k)     # [T, d], x.dtype
    out.backward(g)   # x.grad, logits.grad, w_gate_up.grad, w_down.grad

The integration surface that "Mario/overlap moe kernel integration (prime-rl
PR #3651)" describes (Overview and the custom-op commit note): one fused op
that takes the undispatched tokens and the routing inputs, saves what its
backward needs and returns every input's gradient in that input's dtype.

Argument marshalling only: both ops call the C ABI (moe.py -> libmoe.so),
where every step of the layer runs.  They are registered with torch.library
(`ggr_b200::moe_forward`, `ggr_b200::moe_backward`) together with fake
implementations, so torch.compile(fullgraph=True) traces through the layer
without a graph break.  The saved routing state and activations are extra
outputs of the forward op, kept by autograd for the backward op.  A second
pair (`moe_forward_ckpt`, `moe_backward_ckpt`) is the recompute mode: only the
routing state is kept, and the backward regenerates h, aw and the sorted copy
of x (moe_recompute).
"""
from __future__ import annotations

import torch

from . import moe as M

__all__ = ["moe_layer", "moe_forward", "moe_backward", "moe_forward_ckpt", "moe_backward_ckpt"]

_SAVED_SHAPES = {
    "topk_idx": lambda T, d, E, k, I, p: (T, k), "topk_w": lambda T, d, E, k, I, p: (T, k),
    "counts": lambda T, d, E, k, I, p: (E,), "offsets": lambda T, d, E, k, I, p: (E + 1,),
    "group_start": lambda T, d, E, k, I, p: (E + 1,), "tile_expert": lambda T, d, E, k, I, p: (p // 128,),
    "perm": lambda T, d, E, k, I, p: (p,), "inv": lambda T, d, E, k, I, p: (T, k),
    "h": lambda T, d, E, k, I, p: (p, 2 * I), "aw": lambda T, d, E, k, I, p: (p, I),
    "xs": lambda T, d, E, k, I, p: (p, d),
}
_SAVED_DTYPES = dict(topk_idx=torch.int32, topk_w=torch.float32, counts=torch.int32, offsets=torch.int32,
                     group_start=torch.int32, tile_expert=torch.int32, perm=torch.int32, inv=torch.int32,
                     h=torch.bfloat16, aw=torch.bfloat16, xs=torch.bfloat16)


def _dims(x, w_gate_up):
    T, d = (int(s) for s in x.shape)
    E, two_i, _ = (int(s) for s in w_gate_up.shape)
    return T, d, E, two_i // 2


def _check_inputs(x, logits, w_gate_up, w_down, top_k):
    T, d, E, I = _dims(x, w_gate_up)
    if x.dtype != torch.bfloat16 or w_gate_up.dtype != torch.bfloat16 or w_down.dtype != torch.bfloat16:
        raise TypeError("x, w_gate_up and w_down must be bfloat16")
    if logits.dtype != torch.float32:
        raise TypeError("logits must be float32")
    if tuple(logits.shape) != (T, E) or tuple(w_gate_up.shape) != (E, 2 * I, d) or tuple(w_down.shape) != (E, d, I):
        raise ValueError("shapes: x [T,d], logits [T,E], w_gate_up [E,2I,d], w_down [E,d,I]")
    if not 1 <= top_k <= E:
        raise ValueError("need 1 <= top_k <= E")
    if len({t.device for t in (x, logits, w_gate_up, w_down)}) != 1:
        raise ValueError("x, logits, w_gate_up and w_down must be on one device")


@torch.library.custom_op("ggr_b200::moe_forward", mutates_args=(), device_types="cuda")
def moe_forward(x: torch.Tensor, logits: torch.Tensor, w_gate_up: torch.Tensor, w_down: torch.Tensor,
                top_k: int, dtype: int, swiglu_limit: float) -> tuple[torch.Tensor, torch.Tensor, torch.Tensor,
                                                                      torch.Tensor, torch.Tensor, torch.Tensor,
                                                                      torch.Tensor, torch.Tensor, torch.Tensor,
                                                                      torch.Tensor, torch.Tensor, torch.Tensor]:
    """out plus the saved state (topk_idx, topk_w, counts, offsets, group_start,
    tile_expert, perm, inv, h, aw, xs), in the field order of moe_saved_t."""
    _check_inputs(x, logits, w_gate_up, w_down, top_k)
    T, d, E, I = _dims(x, w_gate_up)
    x, logits, w_gate_up, w_down = (t.contiguous() for t in (x, logits, w_gate_up, w_down))
    shape = M.make_shape(T, d, E, top_k, I, dtype, swiglu_limit=swiglu_limit)
    saved = M.alloc_saved(shape, x.device)
    f, _ = M.workspace_size(shape)
    ws = torch.empty(f, dtype=torch.uint8, device=x.device)
    out = torch.empty(T, d, dtype=torch.bfloat16, device=x.device)
    M.fwd(shape, x, logits, w_gate_up, w_down, out, saved, ws, torch.cuda.current_stream(x.device))
    return (out,) + tuple(saved[n] for n in M.SAVED_FIELDS)


@moe_forward.register_fake
def _moe_forward_fake(x, logits, w_gate_up, w_down, top_k, dtype, swiglu_limit):
    T, d, E, I = _dims(x, w_gate_up)
    _, p_cap = M.saved_sizes(M.make_shape(T, d, E, top_k, I, dtype))  # host-side shape rule of the library
    saved = tuple(x.new_empty(_SAVED_SHAPES[n](T, d, E, top_k, I, p_cap), dtype=_SAVED_DTYPES[n])
                  for n in M.SAVED_FIELDS)
    return (x.new_empty(T, d),) + saved


@torch.library.custom_op("ggr_b200::moe_backward", mutates_args=(), device_types="cuda")
def moe_backward(grad_out: torch.Tensor, x: torch.Tensor, w_gate_up: torch.Tensor, w_down: torch.Tensor,
                 topk_idx: torch.Tensor, topk_w: torch.Tensor, counts: torch.Tensor, offsets: torch.Tensor,
                 group_start: torch.Tensor, tile_expert: torch.Tensor, perm: torch.Tensor, inv: torch.Tensor,
                 h: torch.Tensor, aw: torch.Tensor, xs: torch.Tensor, top_k: int, dtype: int,
                 swiglu_limit: float) -> tuple[torch.Tensor, torch.Tensor, torch.Tensor, torch.Tensor, torch.Tensor]:
    """(dx, dlogits, dw_gate_up, dw_down, dscore) for dL/dout = grad_out."""
    T, d, E, I = _dims(x, w_gate_up)
    shape = M.make_shape(T, d, E, top_k, I, dtype, swiglu_limit=swiglu_limit)
    saved = dict(zip(M.SAVED_FIELDS, (topk_idx, topk_w, counts, offsets, group_start, tile_expert, perm, inv, h,
                                      aw, xs)))
    _, b = M.workspace_size(shape)
    ws = torch.empty(b, dtype=torch.uint8, device=x.device)
    dev = x.device
    dx = torch.empty(T, d, dtype=torch.bfloat16, device=dev)
    dlogits = torch.empty(T, E, dtype=torch.float32, device=dev)
    dwgu = torch.empty(E, 2 * I, d, dtype=torch.bfloat16, device=dev)
    dwd = torch.empty(E, d, I, dtype=torch.bfloat16, device=dev)
    dscore = torch.empty(T, top_k, dtype=torch.float32, device=dev)
    M.bwd(shape, grad_out.contiguous(), x.contiguous(), w_gate_up.contiguous(), w_down.contiguous(), saved, dx,
          dwgu, dwd, dscore, dlogits, ws, torch.cuda.current_stream(dev))
    return dx, dlogits, dwgu, dwd, dscore


@moe_backward.register_fake
def _moe_backward_fake(grad_out, x, w_gate_up, w_down, topk_idx, topk_w, counts, offsets, group_start,
                       tile_expert, perm, inv, h, aw, xs, top_k, dtype, swiglu_limit):
    T, d, E, I = _dims(x, w_gate_up)
    return (x.new_empty(T, d), x.new_empty(T, E, dtype=torch.float32), w_gate_up.new_empty(E, 2 * I, d),
            w_down.new_empty(E, d, I), x.new_empty(T, top_k, dtype=torch.float32))


def _setup_context(ctx, inputs, output):
    x, logits, w_gate_up, w_down, top_k, dtype, swiglu_limit = inputs
    saved = output[1:]
    ctx.save_for_backward(x, w_gate_up, w_down, *saved)
    ctx.top_k, ctx.dtype, ctx.swiglu_limit = top_k, dtype, swiglu_limit
    ctx.mark_non_differentiable(*saved)


def _backward(ctx, grad_out, *_unused_saved_grads):
    x, w_gate_up, w_down, *saved = ctx.saved_tensors
    dx, dlogits, dwgu, dwd, _ = moe_backward(grad_out.to(torch.bfloat16), x, w_gate_up, w_down, *saved,
                                             ctx.top_k, ctx.dtype, ctx.swiglu_limit)
    return dx, dlogits, dwgu, dwd, None, None, None


moe_forward.register_autograd(_backward, setup_context=_setup_context)


_ROUTING_FIELDS = M.SAVED_FIELDS[:8]  # the saved fields without h, aw and xs


@torch.library.custom_op("ggr_b200::moe_forward_ckpt", mutates_args=(), device_types="cuda")
def moe_forward_ckpt(x: torch.Tensor, logits: torch.Tensor, w_gate_up: torch.Tensor, w_down: torch.Tensor,
                     top_k: int, dtype: int, swiglu_limit: float) -> tuple[torch.Tensor, torch.Tensor, torch.Tensor,
                                                                           torch.Tensor, torch.Tensor, torch.Tensor,
                                                                           torch.Tensor, torch.Tensor, torch.Tensor]:
    """Recompute mode: out plus the routing state only; h, aw and xs are
    dropped when the op returns and regenerated by the backward op."""
    outs = moe_forward(x, logits, w_gate_up, w_down, top_k, dtype, swiglu_limit)
    return outs[:9]


@moe_forward_ckpt.register_fake
def _moe_forward_ckpt_fake(x, logits, w_gate_up, w_down, top_k, dtype, swiglu_limit):
    return _moe_forward_fake(x, logits, w_gate_up, w_down, top_k, dtype, swiglu_limit)[:9]


@torch.library.custom_op("ggr_b200::moe_backward_ckpt", mutates_args=(), device_types="cuda")
def moe_backward_ckpt(grad_out: torch.Tensor, x: torch.Tensor, w_gate_up: torch.Tensor, w_down: torch.Tensor,
                      topk_idx: torch.Tensor, topk_w: torch.Tensor, counts: torch.Tensor, offsets: torch.Tensor,
                      group_start: torch.Tensor, tile_expert: torch.Tensor, perm: torch.Tensor, inv: torch.Tensor,
                      top_k: int, dtype: int,
                      swiglu_limit: float) -> tuple[torch.Tensor, torch.Tensor, torch.Tensor, torch.Tensor,
                                                    torch.Tensor]:
    """Recompute mode backward: moe_recompute regenerates h, aw and xs, then moe_bwd."""
    T, d, E, I = _dims(x, w_gate_up)
    shape = M.make_shape(T, d, E, top_k, I, dtype, swiglu_limit=swiglu_limit)
    _, p_cap = M.saved_sizes(shape)
    dev = x.device
    h = torch.empty(p_cap, 2 * I, dtype=torch.bfloat16, device=dev)
    aw = torch.empty(p_cap, I, dtype=torch.bfloat16, device=dev)
    xs = torch.empty(p_cap, d, dtype=torch.bfloat16, device=dev)
    saved = dict(zip(M.SAVED_FIELDS, (topk_idx, topk_w, counts, offsets, group_start, tile_expert, perm, inv, h,
                                      aw, xs)))
    f, _ = M.workspace_size(shape)
    ws = torch.empty(f, dtype=torch.uint8, device=dev)
    M.recompute(shape, x.contiguous(), w_gate_up.contiguous(), saved, ws, torch.cuda.current_stream(dev))
    del ws
    return moe_backward(grad_out, x, w_gate_up, w_down, topk_idx, topk_w, counts, offsets, group_start, tile_expert,
                        perm, inv, h, aw, xs, top_k, dtype, swiglu_limit)


@moe_backward_ckpt.register_fake
def _moe_backward_ckpt_fake(grad_out, x, w_gate_up, w_down, topk_idx, topk_w, counts, offsets, group_start,
                            tile_expert, perm, inv, top_k, dtype, swiglu_limit):
    return _moe_backward_fake(grad_out, x, w_gate_up, w_down, topk_idx, topk_w, counts, offsets, group_start,
                              tile_expert, perm, inv, None, None, None, top_k, dtype, swiglu_limit)


def _setup_context_ckpt(ctx, inputs, output):
    x, logits, w_gate_up, w_down, top_k, dtype, swiglu_limit = inputs
    routing = output[1:]
    ctx.save_for_backward(x, w_gate_up, w_down, *routing)
    ctx.top_k, ctx.dtype, ctx.swiglu_limit = top_k, dtype, swiglu_limit
    ctx.mark_non_differentiable(*routing)


def _backward_ckpt(ctx, grad_out, *_unused_routing_grads):
    x, w_gate_up, w_down, *routing = ctx.saved_tensors
    dx, dlogits, dwgu, dwd, _ = moe_backward_ckpt(grad_out.to(torch.bfloat16), x, w_gate_up, w_down, *routing,
                                                  ctx.top_k, ctx.dtype, ctx.swiglu_limit)
    return dx, dlogits, dwgu, dwd, None, None, None


moe_forward_ckpt.register_autograd(_backward_ckpt, setup_context=_setup_context_ckpt)


def moe_layer(x: torch.Tensor, logits: torch.Tensor, w_gate_up: torch.Tensor, w_down: torch.Tensor, top_k: int,
              mxfp8: bool = False, recompute: bool = False, swiglu_limit: float = 0.0,
              fp8_bwd: bool = True) -> torch.Tensor:
    """The fused MoE layer as a differentiable function: out [T, d] in x's dtype.

    x [T, d]; logits [T, E]; w_gate_up [E, 2I, d] (rows 0..I-1 gate, I..2I-1
    up); w_down [E, d, I].  The layer runs on bf16 tokens and weights and fp32
    logits: other floating dtypes are cast on the way in, and autograd returns
    each gradient in its input's dtype.  mxfp8=True runs the expert GEMMs on
    MXFP8 operands (E4M3 with one UE8M0 scale per 32 elements along K).
    recompute=True keeps only the routing state between forward and backward
    (h, aw and the sorted copy of x, 1.2 GB at the Qwen3-30B-A3B layer shape,
    are regenerated by one more gate/up GEMM in the backward); the results are
    bit-identical.
    swiglu_limit=L > 0 selects the clamped SwiGLU, silu(min(gate, L)) *
    clamp(up, -L, L) (0: the plain SwiGLU).  fp8_bwd=False (with mxfp8=True)
    keeps the backward GEMMs in bf16.
    """
    dtype = (M.MOE_MXFP8 if fp8_bwd else M.MOE_MXFP8_FWD) if mxfp8 else M.MOE_BF16
    op = moe_forward_ckpt if recompute else moe_forward
    out = op(x.to(torch.bfloat16), logits.to(torch.float32), w_gate_up.to(torch.bfloat16),
             w_down.to(torch.bfloat16), int(top_k), dtype, float(swiglu_limit))[0]
    return out.to(x.dtype)

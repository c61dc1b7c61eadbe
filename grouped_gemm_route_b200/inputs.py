"""Seeded synthetic inputs for the fused MoE layer.

This module only draws random tensors of the workloads' shapes and value
distributions; it holds none of the layer's arithmetic.  Both the CUDA path's
tests/benchmark and the CPU oracle take their inputs from here.

Workloads (sizes of the layers the pages benchmark: Qwen3-30B-A3B and
Qwen3-235B-A22B MoE layers, 128 experts, top-8, 16,384 tokens per GPU --
"Prime Intellect Fused MoE Kernel: 3.11x MoE Training Speed", section
"How to measure it on your own cluster"):

  tiny              T=256   d=256  E=8   k=2 I=128
  qwen3_30b_a3b     T=16384 d=2048 E=128 k=8 I=768
  qwen3_235b_a22b   T=16384 d=4096 E=128 k=8 I=1536
  qwen3_30b_a3b_skew   30B shape, router logits plus a Zipf(s=1.2) per-expert bias
  qwen3_30b_a3b_mxfp8  30B shape, same tensors as qwen3_30b_a3b (MXFP8 GEMM operands)

Distributions: x and grad_out ~ N(0,1) rounded to bf16; W_gate_up and W_down
~ N(0, 0.02^2) rounded to bf16; router logits ~ N(0,1) in fp32.  Every tensor
is drawn on the CPU from its own torch generator seeded with
``seed * 1000 + tensor_id`` and then moved to the requested device, so a
(workload, seed) pair gives the same values on every machine and device.
"""
from __future__ import annotations

import torch

WORKLOADS = {
    "tiny": dict(T=256, d=256, E=8, k=2, I=128),
    "qwen3_30b_a3b": dict(T=16384, d=2048, E=128, k=8, I=768),
    "qwen3_235b_a22b": dict(T=16384, d=4096, E=128, k=8, I=1536),
    "qwen3_30b_a3b_skew": dict(T=16384, d=2048, E=128, k=8, I=768, zipf_s=1.2),
    "qwen3_30b_a3b_mxfp8": dict(T=16384, d=2048, E=128, k=8, I=768, dtype="mxfp8"),
}

# Scale of the Zipf logit bias.  bias_e = -ZIPF_ALPHA * s * ln(r_e) with r_e a
# seeded random ranking of the experts (1..E).  The value was chosen once so
# that, for seed 0 of the skewed 30B workload, about ten experts receive no
# token; tests/golden/zipf_alpha.json records the calibration and a CPU test
# re-checks the resulting empty-expert count.
ZIPF_ALPHA = 1.1

_TID = dict(x=1, logits=2, wgu=3, wd=4, gout=5, zipf_rank=6)


def _gen(seed: int, tensor: str) -> torch.Generator:
    g = torch.Generator(device="cpu")
    g.manual_seed(int(seed) * 1000 + _TID[tensor])
    return g


def _randn(shape, seed, tensor, std=1.0, dtype=torch.bfloat16):
    t = torch.randn(*shape, generator=_gen(seed, tensor), dtype=torch.float32)
    if std != 1.0:
        t.mul_(std)
    return t.to(dtype)


def zipf_bias(E: int, s: float, seed: int, alpha: float = ZIPF_ALPHA) -> torch.Tensor:
    """Per-expert logit bias -alpha * s * ln(rank), ranks a seeded permutation of 1..E."""
    rank = torch.randperm(E, generator=_gen(seed, "zipf_rank")).to(torch.float64) + 1.0
    return (-alpha * s * torch.log(rank)).to(torch.float32)


def make_logits(T, E, seed=0, zipf_s=None, alpha=ZIPF_ALPHA):
    logits = _randn((T, E), seed, "logits", dtype=torch.float32)
    if zipf_s is not None:
        logits = logits + zipf_bias(E, zipf_s, seed, alpha)[None, :]
    return logits


def make_inputs(T, d, E, k, I, seed=0, device="cpu", zipf_s=None, with_grad=True, **_):
    """All tensors of one layer call, contiguous, on ``device``."""
    out = dict(
        x=_randn((T, d), seed, "x"),
        logits=make_logits(T, E, seed, zipf_s),
        wgu=_randn((E, 2 * I, d), seed, "wgu", std=0.02),
        wd=_randn((E, d, I), seed, "wd", std=0.02),
    )
    if with_grad:
        out["gout"] = _randn((T, d), seed, "gout")
    return {name: t.to(device).contiguous() for name, t in out.items()}


def make_grid_inputs(T, d, E, k, I, seed=0, device="cpu", **_):
    """Inputs on coarse grids, for checks where a discrete decision taken on a
    pre-activation must not depend on rounding (the sides of the clamped
    SwiGLU's clamps).

    x = n / 4 with n uniform in -4..4; W_gate_up and W_down = m / 64 with m
    uniform in -3..3; grad_out ~ N(0,1) and router logits ~ N(0,1) as in
    make_inputs.  Every product x * W is a multiple of 2^-8 and every gate/up
    pre-activation h = W_gate_up x is an exact multiple of 2^-8 in float32
    (|h| stays far below 2^16), exactly representable in bfloat16 while
    |h| < 1, and E4M3 block quantisation leaves x and the weights unchanged.
    A limit strictly between two multiples of 2^-8 is therefore on the same
    side of every h whether h is taken exactly, in float32 or rounded to
    bfloat16."""
    def grid(shape, tensor, half_range, step):
        n = torch.randint(-half_range, half_range + 1, shape, generator=_gen(seed, tensor))
        return (n.to(torch.float32) * step).to(torch.bfloat16)
    out = dict(
        x=grid((T, d), "x", 4, 0.25),
        logits=make_logits(T, E, seed),
        wgu=grid((E, 2 * I, d), "wgu", 3, 1.0 / 64),
        wd=grid((E, d, I), "wd", 3, 1.0 / 64),
        gout=_randn((T, d), seed, "gout"),
    )
    return {name: t.to(device).contiguous() for name, t in out.items()}


def make_workload(name: str, seed=0, device="cpu", with_grad=True):
    cfg = dict(WORKLOADS[name])
    return cfg, make_inputs(seed=seed, device=device, with_grad=with_grad, **cfg)


def flops_fwd(T, d, E, k, I, **_):
    """Algorithmic forward FLOPs: gate/up 2*P*d*2I plus down 2*P*I*d, P = T*k."""
    return 6.0 * T * k * d * I


def flops_bwd(T, d, E, k, I, **_):
    """Algorithmic backward FLOPs: two dgrads and two wgrads, 12*T*k*d*I."""
    return 12.0 * T * k * d * I


def routing_bytes(T, E, k, **_):
    """Algorithmic routing bytes: read logits, write idx, w, perm, inv, counts/offsets."""
    return T * E * 4 + 4 * T * k * 4 + 8 * E


def describe(cfg) -> str:
    return ", ".join(f"{k}={v}" for k, v in cfg.items())


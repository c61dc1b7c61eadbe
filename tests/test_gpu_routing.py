"""Routing alone (moe_route) against the oracle, bit-exact, on shapes that
reach both routing kernels: the lane-per-token form (E <= 128, E a multiple of
4k, k <= 8; both of its ring depths and both group counts) and the
warp-per-token form (everything else), with and without tied logits, and on
token counts that leave ragged per-warp batches."""
import numpy as np
import pytest
import torch

from grouped_gemm_route_b200 import moe as M
from helpers import check_routing

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("T,E,k,ties", [
    (5000, 128, 8, True),    # lane form, the 30B router shape, many exact ties
    (16384, 128, 8, False),  # lane form at the workload's size
    (2048, 96, 4, False),    # lane form, E not a power of two
    (77, 32, 8, True),       # lane form, fewer tokens than one warp batch per warp
    (50000, 128, 8, False),  # lane form, two-batch ring per warp, both slots used
    (70000, 128, 8, True),   # lane form, one batch per warp (more than 384 tokens per SM), ties
    (131072, 128, 8, False), # lane form, one batch per warp, several batches each
    (3000, 120, 5, True),    # lane form, 2k groups of 12 experts
    (3000, 64, 8, False),    # lane form, 2k groups of 4 experts
    (3000, 160, 8, False),   # warp form: E > 128
    (777, 20, 3, True),      # warp form: E not a multiple of 4k
    (4096, 64, 6, False),    # warp form: 64 is not a multiple of 24
    (300, 512, 16, True),    # warp form: largest E, k > 8
])
def test_routing_bit_exact(T, E, k, ties):
    g = torch.Generator().manual_seed(T * 31 + E)
    lg = torch.randn(T, E, generator=g, dtype=torch.float32)
    if ties:
        lg = torch.round(lg * 2) / 2
        lg[::5] = 0.5
        lg[1::11] = -0.0
        lg[1::11, 0] = 0.0
    sh = M.make_shape(T, 128, E, k, 128)
    saved = M.alloc_saved_routing(sh, "cuda")
    f, _ = M.workspace_size(sh)
    ws = torch.empty(f, dtype=torch.uint8, device="cuda")
    M.route(sh, lg.cuda(), saved, ws)
    torch.cuda.synchronize()
    assert M.get_status(ws) == 0
    check_routing(saved, lg.numpy(), k)
    # a second call on the same buffers gives the same bits
    before = {n: saved[n].clone() for n in ("topk_idx", "topk_w", "perm", "inv")}
    M.route(sh, lg.cuda(), saved, ws)
    torch.cuda.synchronize()
    for n, t in before.items():
        assert torch.equal(saved[n], t), n

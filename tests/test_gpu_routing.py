"""Routing alone (moe_route) against the oracle, bit-exact, on shapes that
reach both routing kernels: the quad form (four lanes per token; E <= 128, E a
multiple of 4, E >= 4k, k <= 8; 16 and 24 warps, one and several position
chunks per block, the rank and the one-per-round selections) and the
warp-per-token form (everything else), with and without tied logits, and on
token counts that leave ragged per-warp batches."""
import numpy as np
import pytest
import torch

from grouped_gemm_route_b200 import moe as M
from helpers import check_routing

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("T,E,k,ties", [
    (5000, 128, 8, True),    # quad form, the 30B router shape, many exact ties (one per round)
    (16384, 128, 8, False),  # quad form at the workload's size (16 warps)
    (2048, 96, 4, False),    # quad form, E not a power of two
    (77, 32, 8, True),       # quad form, fewer tokens than one batch per warp
    (50000, 128, 8, False),  # quad form, 16 warps, one position chunk per block
    (70000, 128, 8, True),   # quad form, ties
    (131072, 128, 8, False), # quad form, 16 warps, two position chunks per block
    (200000, 128, 8, True),  # quad form, 24 warps, two position chunks per block, ties
    (3000, 120, 5, True),    # quad form, 30 pieces per row, odd k
    (3000, 64, 8, False),    # quad form, E = 8k
    (777, 20, 3, True),      # quad form, 5 pieces per row
    (4096, 64, 6, False),    # quad form, k = 6
    (1000, 8, 2, True),      # quad form, E = 4k
    (3000, 160, 8, False),   # warp form: E > 128
    (300, 512, 16, True),    # warp form: largest E, k > 8
    (200, 96, 64, True),     # warp form: the largest k (two slots per lane)
    (1000, 130, 4, True),    # warp form: E not a multiple of 4
    (500, 8, 4, True),       # warp form: E < 4k
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

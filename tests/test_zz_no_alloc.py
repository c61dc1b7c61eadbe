"""moe_route_noalloc: routing for callers that cannot allocate device memory.

Some users of this library cannot call cudaMalloc at all (their host program's
memory manager owns the GPU's memory, or an allocation is not acceptable on
their latency-critical path).  For them moe_route_noalloc takes the routing
kernels' scratch from a fixed array inside the library instead of a caller
workspace.  This test checks, through the C ABI, that two calls in a row give
the same routing state as the ordinary workspace-based moe_route, and that
shapes beyond the fixed scratch are refused.  The comparison is bit for bit
on every routing field, weights included, for both forms of moe_route's
kernel (four lanes per token; one token per warp for E > 128, E not a multiple
of 4 or E < 4k), and the routing is also checked once against the oracle's route and
dispatch.  It sits in a file of its own that pytest collects last.
"""
import ctypes

import numpy as np
import pytest
import torch

from grouped_gemm_route_b200 import inputs as IN
from grouped_gemm_route_b200 import moe as M
from helpers import check_routing

pytestmark = pytest.mark.gpu

EXACT = ("topk_idx", "topk_w", "counts", "offsets", "group_start", "inv")


def _route_both(T, d, E, k, I, seed):
    shape = M.make_shape(T, d, E, k, I)
    logits = IN.make_logits(T, E, seed=seed).cuda()
    ref = M.alloc_saved(shape, "cuda")
    ws = M.alloc_workspace(shape, "cuda")
    M.route(shape, logits, ref, ws)
    out = M.alloc_saved(shape, "cuda")
    for name in EXACT + ("perm", "tile_expert", "topk_w"):
        out[name].fill_(-7)  # stale values that the call must overwrite
    M.route_noalloc(shape, logits, out)
    torch.cuda.synchronize()
    return ref, out


@pytest.mark.parametrize("sizes", [
    dict(T=16384, d=2048, E=128, k=8, I=768),  # four lanes per token
    dict(T=1000, d=256, E=16, k=4, I=128),     # four lanes per token
    dict(T=999, d=256, E=128, k=6, I=128),     # four lanes per token, k = 6
    dict(T=1000, d=256, E=256, k=8, I=128),    # one token per warp (E > 128)
    dict(T=999, d=256, E=130, k=6, I=128),     # one token per warp (E not a multiple of 4)
])
def test_noalloc_routing_matches_workspace_routing_on_two_calls(sizes):
    for call, seed in enumerate((3, 4)):  # two calls in a row reuse the same library scratch
        ref, out = _route_both(seed=seed, **sizes)
        for name in EXACT:
            assert torch.equal(ref[name], out[name]), (call, name)
        used = int(ref["group_start"][-1].item())
        assert torch.equal(ref["perm"][:used], out["perm"][:used]), call
        assert torch.equal(ref["tile_expert"][:used // 128], out["tile_expert"][:used // 128]), call
        if call == 0:
            # once against the oracle: indices, counts, permutation bit for bit; the
            # fp32 weights w_j = exp_j / sum_i exp_i within the rounding of that
            # formula: with u = 2^-24, each exp within 2 ulp (4u), the k-term sum
            # adding (k - 1) u, the division u, so |w - w_ref| / w_ref <= (k + 8) u
            logits = IN.make_logits(sizes["T"], sizes["E"], seed=seed).numpy()
            _, w_ref = check_routing(out, logits, sizes["k"])
            w = out["topk_w"].cpu().numpy().astype(np.float64)
            assert np.max(np.abs(w - w_ref) / w_ref) <= (sizes["k"] + 8) * 2.0 ** -24


def test_noalloc_rejects_shapes_beyond_its_scratch():
    # ceil(65600/64) * 128 = 131200 > 131072 histogram slots
    shape = M.make_shape(65600, 256, 128, 2, 128)
    saved = M.MoeSaved(*([16] * len(M.SAVED_FIELDS)))
    rc = M.lib().moe_route_noalloc(ctypes.byref(shape), ctypes.c_void_p(16), ctypes.byref(saved), None)
    assert rc == M.MOE_ERR_SCRATCH_LIMIT
    assert "scratch" in M.error_string(rc)

"""Device-side failure detection without a GPU fault.

A kernel's bounded wait on an mbarrier that nothing arrives at must expire,
record a timeout in the workspace status word and return; the context must
stay usable for the next call."""
import numpy as np
import pytest
import torch

from grouped_gemm_route_b200 import moe as M
from helpers import check_routing, make, run_layer

pytestmark = pytest.mark.gpu


def test_expired_wait_reports_timeout_and_context_survives():
    ws = torch.zeros(256, dtype=torch.uint8, device="cuda")
    M.selftest_wait_timeout(ws)
    assert M.get_status(ws) == M.MOE_ERR_TIMEOUT
    # the next real call on the same context runs and reports a clean status
    cfg, inp = make("tiny", seed=1)
    layer, res = run_layer(inp, *(cfg[n] for n in ("T", "d", "E", "k", "I")))
    assert res["status"] == M.MOE_OK
    check_routing(res["saved"], inp["logits"].numpy(), cfg["k"])
    assert np.isfinite(res["out"].float().cpu().numpy()).all()


def test_status_is_clean_after_a_normal_call():
    cfg, inp = make(dict(T=64, d=256, E=8, k=2, I=128), seed=2)
    layer, res = run_layer(inp, 64, 256, 8, 2, 128)
    assert layer.status() == M.MOE_OK

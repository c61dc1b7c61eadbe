"""Expert parallelism on the GPU, through the C ABI (grouped_gemm_route_b200.ep.CudaEP).

* One rank: the EP layer's results equal moe_fwd / moe_bwd's bit for bit
  (same tiles, same staged bf16 rows, same slot-ordered sums), with the local
  experts in one chunk or in several.
* Two and four ranks simulated on one GPU in one process: each rank's device
  steps run on its own buffers, and the exchanges of grouped_gemm_route_b200.ep's
  plan are executed as device copies between the ranks' buffers (no kernel of
  one rank waits for another's).  Every rank's out, dx, dscore, dlogits and its
  experts' weight gradients are compared with the fp64 oracle's layer over all
  ranks' tokens (normwise 1e-2), with the local experts exchanged and
  computed in one chunk or in several.
* One rank in an NCCL process group (torchrun, one process): the counts
  all-to-all goes through NCCL; results as without the group.
"""
import os

import pytest
import torch

from grouped_gemm_route_b200 import inputs as IN
from grouped_gemm_route_b200 import moe as M
from grouped_gemm_route_b200.ep import CudaEP, EPMoELayer, Plan, chunk_bounds
from helpers import TOL_BF16, f64, normwise
from oracle import moe_oracle as O

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("chunks", [1, 4])
def test_one_rank_equals_the_single_gpu_layer_bitwise(chunks):
    T, d, E, k, I = 700, 512, 12, 3, 256
    inp = IN.make_inputs(T, d, E, k, I, seed=41, device="cuda")
    ref = M.MoELayer(T, d, E, k, I)
    out_ref = ref.forward(inp["x"], inp["logits"], inp["wgu"], inp["wd"]).clone()
    g_ref = {n: t.clone() for n, t in ref.backward(inp["gout"], inp["x"], inp["wgu"], inp["wd"]).items()}
    layer = EPMoELayer(CudaEP(T, d, E, k, I, G=1), chunks=chunks)
    out = layer.forward(inp["x"], inp["logits"], inp["wgu"], inp["wd"])
    g = layer.backward(inp["gout"], inp["wgu"], inp["wd"])
    torch.cuda.synchronize()
    assert ref.status() == 0 and layer.b.status() == 0
    assert torch.equal(out, out_ref)
    for name in ("dx", "dscore", "dlogits", "dwgu", "dwd"):
        assert torch.equal(g[name], g_ref[name]), name


def _local_exchange(per_rank):
    """per_rank[r] = (sends, receives) of rank r, entries (peer, tensor, first
    row, rows) in posting order: the k-th send from s to q meets the k-th
    receive of q from s."""
    G = len(per_rank)
    for s in range(G):
        for q in range(G):
            snd = [x for x in per_rank[s][0] if x[0] == q]
            rcv = [x for x in per_rank[q][1] if x[0] == s]
            assert len(snd) == len(rcv), (s, q)
            for (_, src, a, n), (_, dst, b, m) in zip(snd, rcv):
                assert n == m
                dst[b:b + m].copy_(src[a:a + n])


def _merge(*pairs):
    return [x for p in pairs for x in p[0]], [x for p in pairs for x in p[1]]


def simulate(G, T, d, E, k, I, inp, chunks=1):
    """G ranks' EP forward + backward in one process: rank r holds tokens
    [r T, (r+1) T) and experts [r E/G, (r+1) E/G), its local experts in
    `chunks` chunks, each exchanged and computed on its own."""
    E_loc = E // G
    tok = [slice(r * T, (r + 1) * T) for r in range(G)]
    exp = [slice(r * E_loc, (r + 1) * E_loc) for r in range(G)]
    bounds = chunk_bounds(E_loc, chunks)
    backs = [CudaEP(T, d, E, k, I, G) for _ in range(G)]
    srcs = [b.route_dispatch(inp["x"][tok[r]], inp["logits"][tok[r]]) for r, b in enumerate(backs)]
    recv = [[srcs[s]["counts"][r * E_loc:(r + 1) * E_loc] for s in range(G)] for r in range(G)]
    plans = [[] for _ in range(G)]
    sides = [[] for _ in range(G)]
    for r in range(G):
        for e0, e1 in bounds:
            rc = [row[e0:e1] for row in recv[r]]
            ro, co, n, pad = M.ep_expert_layout(G, e1 - e0, rc)
            plans[r].append(Plan(G, e1 - e0, srcs[r]["counts"], srcs[r]["group_start"], srcs[r]["offsets"], rc, ro,
                                 co, n, pad, E_all=E_loc, e0=e0))
            rc_dev = torch.tensor(rc, dtype=torch.int32, device="cuda").reshape(-1)
            sides[r].append(backs[r].expert_side(rc_dev, n, e0, e1))
    wgu = [inp["wgu"][exp[r]] for r in range(G)]
    wd = [inp["wd"][exp[r]] for r in range(G)]
    for c in range(len(bounds)):
        _local_exchange([_merge(plans[r][c].to_experts(srcs[r]["xs"], sides[r][c].xr),
                                plans[r][c].to_experts(srcs[r]["w_rows"], sides[r][c].wr, send_rows_from_padded=False))
                         for r in range(G)])
    back = [b.source_rows() for b in backs]
    for c, (e0, e1) in enumerate(bounds):
        ys = [sides[r][c].forward(wgu[r][e0:e1], wd[r][e0:e1]) for r in range(G)]
        _local_exchange([plans[r][c].to_sources(ys[r], back[r]) for r in range(G)])
    outs = [b.combine(rows) for b, rows in zip(backs, back)]
    # backward
    gss = [b.dispatch_grad(inp["gout"][tok[r]]) for r, b in enumerate(backs)]
    grs = [[sd.grad_buffer() for sd in sides[r]] for r in range(G)]
    for c in range(len(bounds)):
        _local_exchange([plans[r][c].to_experts(gss[r], grs[r][c]) for r in range(G)])
    src_g = [b.source_grad_rows() for b in backs]
    dws = [b.weight_grads(wgu[r], wd[r]) for r, b in enumerate(backs)]
    for c, (e0, e1) in enumerate(bounds):
        res = [sides[r][c].backward(grs[r][c], wgu[r][e0:e1], wd[r][e0:e1], dws[r][0][e0:e1], dws[r][1][e0:e1])
               for r in range(G)]
        _local_exchange([_merge(plans[r][c].to_sources(res[r][0], src_g[r][0]),
                                plans[r][c].to_sources(res[r][1], src_g[r][1])) for r in range(G)])
    fin = [b.finish(sg[0], sg[1]) for b, sg in zip(backs, src_g)]
    torch.cuda.synchronize()
    assert all(b.status() == 0 for b in backs)
    rows = [sum(p.rows for p in plans[r]) for r in range(G)]
    return outs, fin, dws, rows


@pytest.mark.parametrize("G,sizes,skew,chunks", [
    (2, dict(T=600, d=512, E=12, k=3, I=256), False, 1),
    (2, dict(T=600, d=512, E=12, k=3, I=256), False, 4),   # six local experts in chunks of 2, 1, 2, 1
    (4, dict(T=300, d=256, E=16, k=4, I=384), False, 2),
    (2, dict(T=500, d=256, E=8, k=2, I=256), True, 3),    # rank 1's experts get (almost) nothing
])
def test_simulated_ranks_match_the_oracle(G, sizes, skew, chunks):
    T, d, E, k, I = (sizes[n] for n in ("T", "d", "E", "k", "I"))
    inp = IN.make_inputs(G * T, d, E, k, I, seed=43 + G, device="cuda")
    if skew:
        inp["logits"][:, : E // G] += 4.0
        inp["logits"][:, E // G] = -100.0  # never chosen: exact-zero weight gradients
    outs, fin, dws, rows = simulate(G, T, d, E, k, I, inp, chunks)
    logits = inp["logits"].cpu().numpy()
    x, wgu, wd, gout = (f64(inp[n]) for n in ("x", "wgu", "wd", "gout"))
    ref = O.forward(x, logits, wgu, wd, k)
    g = O.backward(x, logits, wgu, wd, k, gout, ref)
    E_loc = E // G
    errs = {}
    for r in range(G):
        tok, exp = slice(r * T, (r + 1) * T), slice(r * E_loc, (r + 1) * E_loc)
        errs[f"out{r}"] = normwise(f64(outs[r]), ref["out"][tok])
        errs[f"dx{r}"] = normwise(f64(fin[r][0]), g["dx"][tok])
        errs[f"dscore{r}"] = normwise(f64(fin[r][1]), g["dscore"][tok])
        errs[f"dlogits{r}"] = normwise(f64(fin[r][2]), g["dlogits"][tok])
        errs[f"dwgu{r}"] = normwise(f64(dws[r][0]), g["dwgu"][exp])
        errs[f"dwd{r}"] = normwise(f64(dws[r][1]), g["dwd"][exp])
        for e in range(E_loc):
            if ref["counts"][r * E_loc + e] == 0:
                assert torch.count_nonzero(dws[r][0][e]) == 0 and torch.count_nonzero(dws[r][1][e]) == 0
    if skew:
        assert rows[1] < rows[0]
    bad = {n: v for n, v in errs.items() if not v <= TOL_BF16}
    assert not bad, f"normwise errors above {TOL_BF16}: {bad} (all: {errs})"


def test_one_rank_nccl_group():
    import subprocess
    import sys

    from test_bench_ranks import free_port
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "1",
           "--master-addr", "127.0.0.1", "--master-port", str(free_port()),
           os.path.join("tests", "ep_gpu_worker.py")]
    r = subprocess.run(cmd, cwd=root, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr[-3000:]
    assert "EP_NCCL_OK" in r.stdout, r.stdout[-2000:]

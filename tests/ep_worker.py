"""Worker for the expert-parallel host-logic test: G ranks under torchrun with
the gloo backend on CPU, each holding T tokens and E/G experts.  The layer's
device steps are done by the fp64 oracle (ep_oracle_backend); the plan, the
counts all-to-all and the point-to-point exchanges are the product's
(grouped_gemm_route_b200.ep), with the local experts' exchanges and device
steps in one chunk and in several overlapping ones.  Every rank compares its outputs and its
experts' weight gradients with the oracle's layer over all ranks' tokens;
rank 0 prints the largest errors as one JSON line."""
import datetime
import json
import os
import sys

import numpy as np
import torch
import torch.distributed as dist

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
sys.path.insert(0, os.path.join(ROOT, "tests"))

from ep_oracle_backend import OracleEP  # noqa: E402
from grouped_gemm_route_b200.ep import EPMoELayer  # noqa: E402
from oracle import moe_oracle as O  # noqa: E402


def case_inputs(case, G, T, d, E, k, I):
    rng = np.random.default_rng(100 + case)
    x = rng.standard_normal((G * T, d))
    logits = rng.standard_normal((G * T, E)).astype(np.float32)
    if case == 1:  # every token picks rank 0's experts first (with two ranks, rank 1 receives nothing)
        logits[:, : E // G] += 100.0
    if case == 2:  # one expert of each rank never chosen; a few experts dominate
        logits[:, 1] = -100.0
        logits[:, E // G + 2] = -100.0
        logits[:, 3] += 3.0
    wgu = rng.standard_normal((E, 2 * I, d)) * 0.2
    wd = rng.standard_normal((E, d, I)) * 0.2
    gout = rng.standard_normal((G * T, d))
    return x, logits, wgu, wd, gout


def rel(a, b):
    a, b = np.asarray(a, dtype=np.float64), np.asarray(b, dtype=np.float64)
    den = np.linalg.norm(b)
    return float(np.linalg.norm(a - b) / den) if den else float(np.linalg.norm(a - b))


def main():
    dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=120))
    rank, G = dist.get_rank(), dist.get_world_size()
    T, d, E, k, I = 37, 24, 8, 3, 16
    E_loc = E // G
    results = []
    for case, chunks in [(0, 1), (0, 3), (1, 1), (1, 2), (2, 3), (2, 8)]:
        x, logits, wgu, wd, gout = case_inputs(case, G, T, d, E, k, I)
        mine = slice(rank * T, (rank + 1) * T)
        experts = slice(rank * E_loc, (rank + 1) * E_loc)
        layer = EPMoELayer(OracleEP(T, d, E, k, I, G), chunks=chunks)
        out = layer.forward(x[mine], logits[mine], wgu[experts], wd[experts]).numpy()
        g = layer.backward(gout[mine], wgu[experts], wd[experts])
        ref = O.forward(x, logits, wgu, wd, k)
        rg = O.backward(x, logits, wgu, wd, k, gout, ref)
        errs = dict(out=rel(out, ref["out"][mine]), dx=rel(g["dx"].numpy(), rg["dx"][mine]),
                    dscore=rel(g["dscore"].numpy(), rg["dscore"][mine]),
                    dlogits=rel(g["dlogits"].numpy(), rg["dlogits"][mine]),
                    dwgu=rel(g["dwgu"].numpy(), rg["dwgu"][experts]), dwd=rel(g["dwd"].numpy(), rg["dwd"][experts]))
        results.append(dict(case=case, chunks=len(layer.bounds), rank=rank, rows_received=layer.plan.rows, errs=errs))
    got = [None] * G
    dist.all_gather_object(got, results)
    dist.barrier()
    dist.destroy_process_group()
    if rank == 0:
        print(json.dumps({"world": G, "results": got}), flush=True)


if __name__ == "__main__":
    main()

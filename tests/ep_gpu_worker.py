"""Worker for the one-rank NCCL test of the expert-parallel layer: run under
torchrun with one process on one GPU; the counts all-to-all goes through
NCCL.  Checks the layer's results against moe_fwd / moe_bwd bit for bit and
prints EP_NCCL_OK."""
import datetime
import os
import sys

import torch
import torch.distributed as dist

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

from grouped_gemm_route_b200 import inputs as IN  # noqa: E402
from grouped_gemm_route_b200 import moe as M  # noqa: E402
from grouped_gemm_route_b200.ep import CudaEP, EPMoELayer  # noqa: E402


def main():
    torch.cuda.set_device(0)
    dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=60), device_id=torch.device("cuda", 0))
    T, d, E, k, I = 500, 256, 8, 2, 256
    inp = IN.make_inputs(T, d, E, k, I, seed=47, device="cuda")
    ref = M.MoELayer(T, d, E, k, I)
    out_ref = ref.forward(inp["x"], inp["logits"], inp["wgu"], inp["wd"]).clone()
    g_ref = {n: t.clone() for n, t in ref.backward(inp["gout"], inp["x"], inp["wgu"], inp["wd"]).items()}
    layer = EPMoELayer(CudaEP(T, d, E, k, I, G=1), group=dist.group.WORLD)
    out = layer.forward(inp["x"], inp["logits"], inp["wgu"], inp["wd"])
    g = layer.backward(inp["gout"], inp["wgu"], inp["wd"])
    torch.cuda.synchronize()
    ok = torch.equal(out, out_ref) and all(torch.equal(g[n], g_ref[n]) for n in ("dx", "dscore", "dlogits", "dwgu",
                                                                                   "dwd"))
    dist.barrier()
    dist.destroy_process_group()
    if not ok:
        raise SystemExit("EP layer in a one-rank NCCL group differs from the single-GPU layer")
    print("EP_NCCL_OK", flush=True)


if __name__ == "__main__":
    main()

"""Choose the Zipf logit-bias scale of the skewed 30B workload.

Sweeps alpha, routes the seed-0 logits of the skewed workload with the CPU
oracle, and keeps the smallest alpha on the grid for which between 8 and 12
experts receive no token.  Writes zipf_alpha.json next to this file; the value
is then frozen as ZIPF_ALPHA in grouped_gemm_route_b200/inputs.py.

Run:  python tests/golden/make_zipf_alpha.py
"""
import json
import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

from grouped_gemm_route_b200 import inputs as IN  # noqa: E402
from oracle import moe_oracle as O  # noqa: E402


def main():
    cfg = IN.WORKLOADS["qwen3_30b_a3b_skew"]
    T, E, k, s = cfg["T"], cfg["E"], cfg["k"], cfg["zipf_s"]
    sweep = []
    chosen = None
    for a in np.round(np.arange(0.80, 1.61, 0.02), 2):
        lg = IN.make_logits(T, E, seed=0, zipf_s=s, alpha=float(a)).numpy()
        idx, _ = O.route(lg, k)
        c = np.bincount(idx.ravel(), minlength=E)
        empty = int((c == 0).sum())
        sweep.append(dict(alpha=float(a), empty=empty, max_count=int(c.max())))
        if chosen is None and 8 <= empty <= 12:
            chosen = dict(alpha=float(a), empty=empty, max_count=int(c.max()))
    with open(os.path.join(os.path.dirname(os.path.abspath(__file__)), "zipf_alpha.json"), "w") as f:
        json.dump(dict(workload="qwen3_30b_a3b_skew", seed=0, target_empty="8..12",
                       chosen=chosen, sweep=sweep), f, indent=1)
    print(chosen)


if __name__ == "__main__":
    main()

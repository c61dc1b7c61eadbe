"""Expert parallelism on CPU: the library's host-side layout of the received
rows against a restatement, and the whole exchange choreography of
grouped_gemm_route_b200.ep on two and four gloo ranks (torchrun, loopback), with the
device steps done by the fp64 oracle.  Each rank's out, dx, dscore and dlogits
and its experts' weight gradients must equal the oracle's layer over all
ranks' tokens (the concatenated batch; the oracle's dispatch order -- experts
ascending, tokens ascending -- is the order EP builds: sources in rank order,
tokens ascending inside each)."""
import json
import os

import numpy as np
import pytest

from grouped_gemm_route_b200 import moe as M
from test_bench_ranks import torchrun, json_lines


def restated_layout(G, E_loc, recv):
    recv = np.asarray(recv, dtype=np.int64).reshape(G, E_loc)
    row_off = np.zeros((G, E_loc), dtype=np.int64)
    cmp_off = np.zeros((G, E_loc), dtype=np.int64)
    pad = cmp = 0
    for e in range(E_loc):
        for s in range(G):
            row_off[s, e] = pad + recv[:s, e].sum()
            cmp_off[s, e] = cmp + recv[:s, e].sum()
        n = recv[:, e].sum()
        cmp += n
        pad += -(-n // 128) * 128
    return row_off, cmp_off, cmp, pad


@pytest.mark.parametrize("G,E_loc", [(1, 8), (2, 4), (8, 16), (3, 5)])
def test_expert_layout_matches_restatement(G, E_loc):
    rng = np.random.default_rng(G * 100 + E_loc)
    for trial in range(5):
        recv = rng.integers(0, 300, size=(G, E_loc))
        recv[rng.random((G, E_loc)) < 0.3] = 0  # empty segments and empty experts
        ro, co, rows, pad = M.ep_expert_layout(G, E_loc, recv)
        r_ro, r_co, r_rows, r_pad = restated_layout(G, E_loc, recv)
        assert np.array_equal(np.asarray(ro), r_ro) and np.array_equal(np.asarray(co), r_co)
        assert rows == r_rows == recv.sum() and pad == r_pad
        # the non-empty segments tile the compact order [0, rows) without gap or overlap,
        # and each expert's group starts at a multiple of 128 in the padded layout
        segs = sorted((int(c), int(c + n)) for c, n in zip(np.asarray(co).ravel(), recv.ravel()) if n)
        assert all(a == b for (_, a), (b, _) in zip(segs, segs[1:]))
        assert (segs[0][0] if segs else 0) == 0 and (segs[-1][1] if segs else 0) == rows
        assert all(np.asarray(ro)[0, e] % 128 == 0 for e in range(E_loc))


def test_expert_layout_rejects_negative_counts():
    with pytest.raises(M.MoeError):
        M.ep_expert_layout(2, 2, [[1, -1], [0, 0]])


@pytest.mark.parametrize("G", [2, 4])
def test_ranks_match_the_oracle_layer(G):
    r = torchrun([os.path.join("tests", "ep_worker.py")], timeout=300, nproc=G)
    assert r.returncode == 0, r.stderr[-3000:]
    lines = json_lines(r.stdout)
    assert len(lines) == 1
    res = lines[0]
    assert res["world"] == G
    flat = [c for per_rank in res["results"] for c in per_rank]
    assert len(flat) == 6 * G
    E_loc = 8 // G
    assert {c["chunks"] for c in flat} == {min(n, E_loc) for n in (1, 2, 3, 8)}
    # case 1 routes every token to rank 0's experts first: with two ranks (top-3 of rank 0's
    # four experts) rank 1 receives no rows
    if G == 2:
        assert all(c["rows_received"] == 0 for c in flat if c["case"] == 1 and c["rank"] == 1)
    for c in flat:
        bad = {n: v for n, v in c["errs"].items() if not v <= 1e-12}
        assert not bad, (c["case"], c["rank"], bad)

"""Order of the expert-parallel layer's steps with its local experts in
chunks (CPU, one rank, the fp64 oracle as the device steps): every chunk's
inbound rows are posted before the first chunk's wait, chunk c's expert
computation follows only chunk c's wait, and its results are posted back
before chunk c + 1 is waited for -- the order in which, on several GPUs, the
exchanges of the later chunks overlap the earlier chunks' GEMMs.  Results
equal the one-chunk layer's."""
import numpy as np
import torch

from ep_oracle_backend import OracleEP
from grouped_gemm_route_b200 import ep as EP


class Logged(EP.Pending):
    def __init__(self, inner, log, name):
        super().__init__(inner.works)
        self.log, self.name = log, name

    def wait(self):
        self.log.append(("wait", self.name))
        super().wait()


def run(chunks, log=None, monkeypatch=None):
    rng = np.random.default_rng(7)
    T, d, E, k, I = 29, 16, 8, 2, 8
    x = rng.standard_normal((T, d))
    logits = rng.standard_normal((T, E)).astype(np.float32)
    wgu = rng.standard_normal((E, 2 * I, d)) * 0.3
    wd = rng.standard_normal((E, d, I)) * 0.3
    gout = rng.standard_normal((T, d))
    b = OracleEP(T, d, E, k, I, G=1)
    if log is not None:
        n_posted = [0]
        real_post = EP.post_exchange

        def post(*a, **kw):
            name = n_posted[0]
            n_posted[0] += 1
            log.append(("post", name))
            return Logged(real_post(*a, **kw), log, name)

        monkeypatch.setattr(EP, "post_exchange", post)
        real_side = b.expert_side

        def side(recv_dev, rows, e0, e1):
            # the library takes 16-byte aligned device arrays: each chunk's counts are a fresh tensor,
            # not a view into the whole step's counts at an offset
            assert recv_dev.storage_offset() == 0 and recv_dev.is_contiguous()
            assert recv_dev.numel() == e1 - e0  # one rank: [G * (e1 - e0)]
            sd = real_side(recv_dev, rows, e0, e1)
            fwd, bwd = sd.forward, sd.backward
            sd.forward = lambda *a: (log.append(("forward", e0)), fwd(*a))[1]
            sd.backward = lambda *a: (log.append(("backward", e0)), bwd(*a))[1]
            return sd

        b.expert_side = side
    layer = EP.EPMoELayer(b, chunks=chunks)
    out = layer.forward(x, logits, wgu, wd)
    g = layer.backward(gout, wgu, wd)
    return layer, out, g


def test_chunk_bounds():
    assert EP.chunk_bounds(6, 4) == [(0, 1), (1, 3), (3, 4), (4, 6)]
    assert EP.chunk_bounds(3, 8) == [(0, 1), (1, 2), (2, 3)]
    assert EP.chunk_bounds(5, 1) == [(0, 5)]
    for n, c in [(16, 4), (7, 3), (128, 5)]:
        b = EP.chunk_bounds(n, c)
        assert b[0][0] == 0 and b[-1][1] == n and all(x[1] == y[0] for x, y in zip(b, b[1:]))
        assert max(e1 - e0 for e0, e1 in b) - min(e1 - e0 for e0, e1 in b) <= 1


def test_chunks_overlap_in_order_and_match_one_chunk(monkeypatch):
    log = []
    layer, out, g = run(3, log, monkeypatch)
    monkeypatch.undo()
    _, out1, g1 = run(1)
    assert torch.allclose(out, out1, rtol=0, atol=1e-12)
    for n in ("dx", "dscore", "dlogits", "dwgu", "dwd"):
        assert torch.allclose(g[n], g1[n], rtol=0, atol=1e-12), n
    starts = [e0 for e0, _ in layer.bounds]
    assert starts == [0, 2, 5]  # 8 local experts in 3 chunks
    for phase, step in (("forward", "forward"), ("backward", "backward")):
        half = log[: len(log) // 2] if phase == "forward" else log[len(log) // 2:]
        posts = [i for i, (what, _) in enumerate(half) if what == "post"]
        computes = [i for i, (what, _) in enumerate(half) if what == step]
        # the three inbound exchanges are posted before any computation
        assert posts[:3] == [0, 1, 2] and computes[0] > 2
        # chunk c: wait for its own inbound exchange, compute, post its results back
        for c, i in enumerate(computes):
            assert half[i - 1] == ("wait", half[posts[c]][1])
            assert half[i][1] == starts[c]
            assert half[i + 1][0] == "post"
        # the outbound exchanges are waited for after the last computation
        assert all(what == "wait" for what, _ in half[computes[-1] + 2:])

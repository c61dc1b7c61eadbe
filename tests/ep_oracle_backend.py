"""Device steps of the expert-parallel layer (grouped_gemm_route_b200.ep) done
by the fp64 oracle on CPU tensors -- test infrastructure for checking the EP
plan and exchanges on CPU ranks (gloo), where the CUDA library cannot run.

It keeps the library's layouts: the source's rows in the padded sorted layout
(expert groups at multiples of 128 rows), weights and results in compact
sorted order, the expert side's received rows in its own padded layout.  The
expert side's layout is restated here from recv[s][e] (sources in rank order
inside each local expert's group); the test checks it against the library's
moe_ep_expert_layout.
"""
from __future__ import annotations

import numpy as np
import torch

from oracle import moe_oracle as O


def padded_starts(counts):
    gs = np.zeros(len(counts) + 1, dtype=np.int64)
    gs[1:] = np.cumsum((np.asarray(counts, dtype=np.int64) + 127) // 128 * 128)
    return gs


class OracleEP:
    def __init__(self, T, d, E, k, I, G, limit=0.0):
        self.T, self.d, self.E, self.k, self.I, self.G = T, d, E, k, I, G
        self.E_loc = E // G
        self.limit = limit

    # ---- source side ----
    def route_dispatch(self, x, logits):
        x = np.asarray(x, dtype=np.float64)
        idx, w = O.route(np.asarray(logits), self.k)
        counts, offsets, perm, inv = O.dispatch(idx, self.E)
        gs = padded_starts(counts)
        xs = np.zeros((max(int(gs[-1]), 1), self.d))
        w_rows = np.zeros(self.T * self.k)
        for e in range(self.E):
            pairs = perm[offsets[e]:offsets[e + 1]].astype(np.int64)
            xs[gs[e]:gs[e] + pairs.size] = x[pairs // self.k]
            w_rows[offsets[e]:offsets[e + 1]] = w.reshape(-1)[pairs]
        self.src = dict(idx=idx, w=w, counts=counts, offsets=offsets, perm=perm, inv=inv, gs=gs)
        return dict(xs=torch.from_numpy(xs), w_rows=torch.from_numpy(w_rows),
                    counts_dev=torch.from_numpy(counts.astype(np.int32)), counts=[int(c) for c in counts],
                    group_start=[int(v) for v in gs], offsets=[int(v) for v in offsets])

    def source_rows(self):
        return torch.zeros(self.T * self.k, self.d, dtype=torch.float64)

    def _combine(self, rows):
        rows = rows.numpy()
        out = np.zeros((self.T, self.d))
        inv = self.src["inv"]
        for j in range(self.k):  # slot order
            out += rows[inv[:, j]]
        return out

    def combine(self, rows):
        return torch.from_numpy(self._combine(rows))

    def dispatch_grad(self, grad_out):
        g = np.asarray(grad_out, dtype=np.float64)
        s = self.src
        gsr = np.zeros((max(int(s["gs"][-1]), 1), self.d))
        for e in range(self.E):
            pairs = s["perm"][s["offsets"][e]:s["offsets"][e + 1]].astype(np.int64)
            gsr[s["gs"][e]:s["gs"][e] + pairs.size] = g[pairs // self.k]
        return torch.from_numpy(gsr)

    def source_grad_rows(self):
        return torch.zeros(self.T * self.k, self.d, dtype=torch.float64), torch.zeros(self.T * self.k,
                                                                                       dtype=torch.float64)

    def finish(self, dx_rows, ds_rows):
        dx = self._combine(dx_rows)
        dscore = ds_rows.numpy()[self.src["inv"]]
        dl = O.routing_backward(self.src["w"], dscore)
        dlogits = np.zeros((self.T, self.E))
        np.put_along_axis(dlogits, self.src["idx"].astype(np.int64), dl, axis=1)
        return torch.from_numpy(dx), torch.from_numpy(dscore), torch.from_numpy(dlogits)

    # ---- expert side ----
    def weight_grads(self, w_gate_up, w_down):
        return (torch.zeros(np.shape(w_gate_up), dtype=torch.float64),
                torch.zeros(np.shape(w_down), dtype=torch.float64))

    def expert_side(self, recv_dev, rows, e0, e1):
        return _OracleExpertSide(self, recv_dev, rows, e1 - e0)


class _OracleExpertSide:
    """One chunk of local experts: E_c experts, `rows` received rows in the
    padded layout restated from recv[s][e] (sources in rank order inside each
    expert's group)."""

    def __init__(self, b, recv_dev, rows, E_c):
        self.b, self.rows, self.E_c = b, rows, E_c
        recv = np.asarray(recv_dev, dtype=np.int64).reshape(b.G, E_c)
        self.n = recv.sum(axis=0)
        self.gs = padded_starts(self.n)
        self.off = np.zeros(E_c + 1, dtype=np.int64)
        self.off[1:] = np.cumsum(self.n)
        self.xr = torch.zeros(rows + 128 * E_c, b.d, dtype=torch.float64)
        self.wr = torch.zeros(rows, dtype=torch.float64)

    def forward(self, w_gate_up, w_down):
        xr, wr = self.xr.numpy(), self.wr.numpy()
        wgu, wd = np.asarray(w_gate_up, dtype=np.float64), np.asarray(w_down, dtype=np.float64)
        y = np.zeros((self.rows, self.b.d))
        self.loc = []
        for e in range(self.E_c):
            xe = xr[self.gs[e]:self.gs[e] + self.n[e]]
            we = wr[self.off[e]:self.off[e + 1]]
            if self.n[e]:
                h, _, ye = O.expert_forward(xe, wgu[e], wd[e], self.b.limit)
                y[self.off[e]:self.off[e + 1]] = we[:, None] * ye
            self.loc.append((xe.copy(), we.copy(), self.gs[e], self.off[e], self.n[e]))
        return torch.from_numpy(y)

    def grad_buffer(self):
        return torch.zeros_like(self.xr)

    def backward(self, gr, w_gate_up, w_down, dwgu_out, dwd_out):
        gr = gr.numpy()
        wgu, wd = np.asarray(w_gate_up, dtype=np.float64), np.asarray(w_down, dtype=np.float64)
        dx_rows = np.zeros((self.rows, self.b.d))
        ds_rows = np.zeros(self.rows)
        dwgu, dwd = np.zeros_like(wgu), np.zeros_like(wd)
        for e, (xe, we, g0, o0, ne) in enumerate(self.loc):
            if not ne:
                continue
            dxr, ds, dwgu[e], dwd[e], _ = O._pair_backward(xe, gr[g0:g0 + ne], we, wgu[e], wd[e], self.b.limit)
            dx_rows[o0:o0 + ne] = dxr
            ds_rows[o0:o0 + ne] = ds
        dwgu_out.copy_(torch.from_numpy(dwgu))
        dwd_out.copy_(torch.from_numpy(dwd))
        return torch.from_numpy(dx_rows), torch.from_numpy(ds_rows)

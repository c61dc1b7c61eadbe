"""Expert parallelism for the fused MoE layer: one process per GPU, experts
spread over the G ranks of a torch.distributed group.

"Prime Intellect's Prime Mega MoE Trains Giant AI Models 55% Faster", sections
"Where MoE training loses time" and "One kernel overlaps the pipeline": each
GPU holds a share of the experts; every token is sent to the GPUs that own its
chosen experts, the expert MLPs run there, the results come back to the
token's GPU and are combined; the backward pass repeats the exchange for the
gradients.  "Prime Intellect Fused MoE Kernel: 3.11x MoE Training Speed",
"How to measure it on your own cluster": EP = 8 on one node, 128 experts,
top-8.

Rank q owns the E/G consecutive experts [q E/G, (q+1) E/G).  One step:

  1. the source rank routes its own T tokens over all E experts and writes
     the token rows in the library's sorted layout (moe_route,
     moe_ep_dispatch); the groups of rank q's experts are consecutive there;
  2. every rank tells every other how many rows it will send for each of its
     experts (one all-to-all of E/G counts per pair of ranks);
  3. the rows and their routing weights go to the experts' ranks as NCCL
     point-to-point copies into the receiver's own buffers, one segment per
     (source, expert), straight into the receiver's padded sorted layout
     (moe_ep_expert_layout gives the offsets) -- no kernel reads another
     GPU's memory;
  4. the expert rank runs its grouped GEMMs on what it received
     (moe_expert_fwd) and sends each row's result back to its source, which
     sums each token's k rows in slot order (moe_ep_combine);
  5. the backward sends grad_out rows the same way, the expert rank computes
     the dx rows, the routing-score gradients and its experts' weight
     gradients (moe_expert_bwd), and the source finishes dx, dscore and
     dlogits (moe_ep_backward_finish).

Every rank posts the same collectives in the same order.  Segments a rank
sends to itself are plain device copies.  The point-to-point operations of
one exchange are posted as one batch, ordered by peer, then expert, then
tensor, on both sides; each carries a tag that counts its position, so that
backends that match messages by tag (gloo) pair them the same way as NCCL.

The device steps are a backend object (CudaEP: the C ABI of libmoe.so).  The
class here only plans and moves buffers.
"""
from __future__ import annotations

from dataclasses import dataclass

import torch

from . import moe as M


def _dist():
    import torch.distributed as dist
    return dist


@dataclass
class Plan:
    """Where every segment of one exchange lives (host integers)."""
    G: int
    E_loc: int
    counts: list        # [E]   rows this rank sends for each expert
    group_start: list   # [E+1] padded sorted layout of this rank's pairs
    offsets: list       # [E+1] compact sorted order of this rank's pairs
    recv: list          # [G][E_loc] rows this rank receives for each local expert
    row_off: list       # [G][E_loc] where they land in the local padded layout
    cmp_off: list       # [G][E_loc] and in compact order
    rows: int           # rows received
    padded_rows: int

    def to_experts(self, send, recv, send_rows_from_padded=True):
        """(send segments, receive segments) of a source -> expert exchange:
        per peer q and expert e, the source's rows [start, start + n) and the
        expert side's rows [start, start + n)."""
        out_s, out_r = [], []
        for q in range(self.G):
            for e in range(self.E_loc):
                ge = q * self.E_loc + e
                n = self.counts[ge]
                if n:
                    start = self.group_start[ge] if send_rows_from_padded else self.offsets[ge]
                    out_s.append((q, send, start, n))
                m = self.recv[q][e]
                if m:
                    start = self.row_off[q][e] if send_rows_from_padded else self.cmp_off[q][e]
                    out_r.append((q, recv, start, m))
        return out_s, out_r

    def to_sources(self, send, recv):
        """(send segments, receive segments) of an expert -> source exchange
        (compact order on both sides)."""
        out_s, out_r = [], []
        for q in range(self.G):
            for e in range(self.E_loc):
                ge = q * self.E_loc + e
                m = self.recv[q][e]
                if m:
                    out_s.append((q, send, self.cmp_off[q][e], m))
                n = self.counts[ge]
                if n:
                    out_r.append((q, recv, self.offsets[ge], n))
        return out_s, out_r


def exchange(segment_lists, rank, group=None):
    """Move every (send, receive) segment list pair as one batch of
    point-to-point operations.  Each list entry is (peer, tensor, first row,
    rows).  The k-th message between two ranks in one direction carries tag
    k on both sides."""
    sends, recvs = [], []
    for s_list, r_list in segment_lists:
        sends.extend(s_list)
        recvs.extend(r_list)
    own_s = [x for x in sends if x[0] == rank]
    own_r = [x for x in recvs if x[0] == rank]
    if len(own_s) != len(own_r):
        raise RuntimeError("exchange plan: the segments a rank sends itself do not match its receives")
    for (_, src, a, n), (_, dst, b, m) in zip(own_s, own_r):
        if n != m:
            raise RuntimeError("exchange plan: segment sizes differ")
        dst[b:b + m].copy_(src[a:a + n])
    ops = []
    dist = None
    tag_s, tag_r = {}, {}
    for q, t, a, n in sends:
        if q == rank:
            continue
        dist = dist or _dist()
        k = tag_s.get(q, 0)
        tag_s[q] = k + 1
        ops.append(dist.P2POp(dist.isend, t[a:a + n], q, group, k))
    for q, t, a, n in recvs:
        if q == rank:
            continue
        dist = dist or _dist()
        k = tag_r.get(q, 0)
        tag_r[q] = k + 1
        ops.append(dist.P2POp(dist.irecv, t[a:a + n], q, group, k))
    if ops:
        for w in dist.batch_isend_irecv(ops):
            w.wait()


class EPMoELayer:
    """The fused MoE layer with its experts spread over a process group.

    backend: the device steps (CudaEP for the library; any object with the
    same methods).  w_gate_up / w_down passed to forward and backward are this
    rank's experts' weights, [E/G, 2I, d] and [E/G, d, I]."""

    def __init__(self, backend, group=None):
        self.b = backend
        self.group = group
        dist = _dist()
        if backend.G > 1 or group is not None or (dist.is_available() and dist.is_initialized()):
            self.rank = dist.get_rank(group)
            if dist.get_world_size(group) != backend.G:
                raise ValueError("the backend's G is not the group's size")
        else:
            self.rank = 0
        if backend.E % backend.G:
            raise ValueError("E must be a multiple of the number of ranks")
        self.E_loc = backend.E // backend.G
        self.plan = None

    def _counts_exchange(self, counts_dev):
        """recv[s][e] = rows source s sends for local expert e (one all-to-all;
        a copy when there is one rank and no process group)."""
        if self.b.G == 1 and self.group is None and not (_dist().is_available() and _dist().is_initialized()):
            return counts_dev.clone()
        recv = torch.empty_like(counts_dev)
        _dist().all_to_all_single(recv, counts_dev, group=self.group)
        return recv

    def forward(self, x, logits, w_gate_up, w_down):
        b, G, E_loc = self.b, self.b.G, self.E_loc
        src = b.route_dispatch(x, logits)                   # xs, w_rows and the routing state
        recv_dev = self._counts_exchange(src["counts_dev"])
        recv = recv_dev.cpu().reshape(G, E_loc).tolist()
        row_off, cmp_off, rows, padded = M.ep_expert_layout(G, E_loc, recv)
        p = Plan(G, E_loc, src["counts"], src["group_start"], src["offsets"], recv, row_off, cmp_off, rows, padded)
        self.plan = p
        xr, wr = b.expert_buffers(rows)
        exchange([p.to_experts(src["xs"], xr), p.to_experts(src["w_rows"], wr, send_rows_from_padded=False)],
                 self.rank, self.group)
        y_rows = b.expert_forward(recv_dev, rows, xr, wr, w_gate_up, w_down)
        ys = b.source_rows()
        exchange([p.to_sources(y_rows, ys)], self.rank, self.group)
        return b.combine(ys)

    def backward(self, grad_out, w_gate_up, w_down):
        """Returns dx, dscore, dlogits (this rank's tokens) and dW_gate_up,
        dW_down (this rank's experts)."""
        b, p = self.b, self.plan
        if p is None:
            raise RuntimeError("backward before forward")
        gs = b.dispatch_grad(grad_out)
        gr = b.expert_grad_buffer()
        exchange([p.to_experts(gs, gr)], self.rank, self.group)
        dx_rows, ds_rows, dwgu, dwd = b.expert_backward(gr, w_gate_up, w_down)
        dxs, dss = b.source_grad_rows()
        exchange([p.to_sources(dx_rows, dxs), p.to_sources(ds_rows, dss)], self.rank, self.group)
        dx, dscore, dlogits = b.finish(dxs, dss)
        return dict(dx=dx, dscore=dscore, dlogits=dlogits, dwgu=dwgu, dwd=dwd)


class CudaEP:
    """Device steps of EPMoELayer through libmoe.so (bf16, CTA-pair GEMMs)."""

    def __init__(self, T, d, E, k, I, G, device="cuda", max_sms=0, swiglu_limit=0.0, stream=None):
        if not torch.cuda.is_available():
            raise RuntimeError("the fused MoE layer needs a CUDA device (sm_100)")
        if E % G:
            raise ValueError("E must be a multiple of G")
        self.T, self.d, self.E, self.k, self.I, self.G = T, d, E, k, I, G
        self.E_loc = E // G
        self.device = torch.device(device)
        self.max_sms, self.limit, self.stream = max_sms, swiglu_limit, stream
        self.shape = M.make_shape(T, d, E, k, I, M.MOE_BF16, max_sms, swiglu_limit)
        self.saved = M.alloc_saved(self.shape, self.device, keep_sorted_x=True)
        self.ws = M.alloc_workspace(self.shape, self.device)
        self.w_rows = torch.empty(T * k, dtype=torch.float32, device=self.device)
        self.loc = None

    # ---- source side ----
    def route_dispatch(self, x, logits):
        M.route(self.shape, logits, self.saved, self.ws, self.stream)
        xs = self.saved["xs"]
        M.ep_dispatch(self.shape, x, self.saved, xs, self.w_rows, self.stream)
        host = torch.cat([self.saved["counts"], self.saved["group_start"], self.saved["offsets"]]).cpu().tolist()
        E = self.E
        return dict(xs=xs, w_rows=self.w_rows, counts_dev=self.saved["counts"].clone(), counts=host[:E],
                    group_start=host[E:2 * E + 1], offsets=host[2 * E + 1:])

    def source_rows(self):
        return torch.empty(self.T * self.k, self.d, dtype=torch.bfloat16, device=self.device)

    def combine(self, rows):
        out = torch.empty(self.T, self.d, dtype=torch.bfloat16, device=self.device)
        M.ep_combine(self.shape, self.saved, rows, out, self.stream)
        return out

    def dispatch_grad(self, grad_out):
        gs = torch.empty_like(self.saved["xs"])
        M.ep_dispatch(self.shape, grad_out, self.saved, gs, None, self.stream)
        return gs

    def source_grad_rows(self):
        return (torch.empty(self.T * self.k, self.d, dtype=torch.bfloat16, device=self.device),
                torch.empty(self.T * self.k, dtype=torch.float32, device=self.device))

    def finish(self, dx_rows, ds_rows):
        dx = torch.empty(self.T, self.d, dtype=torch.bfloat16, device=self.device)
        dscore = torch.empty(self.T, self.k, dtype=torch.float32, device=self.device)
        dlogits = torch.empty(self.T, self.E, dtype=torch.float32, device=self.device)
        M.ep_backward_finish(self.shape, self.saved, dx_rows, ds_rows, dx, dscore, dlogits, self.stream)
        return dx, dscore, dlogits

    # ---- expert side ----
    def expert_buffers(self, rows):
        """The received rows' buffers for a step that receives `rows` rows."""
        if rows == 0:
            self.loc = dict(rows=0)
            return (torch.empty(0, self.d, dtype=torch.bfloat16, device=self.device),
                    torch.empty(0, dtype=torch.float32, device=self.device))
        shape = M.make_shape(rows, self.d, self.E_loc, 1, self.I, M.MOE_BF16, self.max_sms, self.limit)
        saved = M.alloc_saved(shape, self.device, keep_sorted_x=False)
        self.loc = dict(rows=rows, shape=shape, saved=saved, ws=M.alloc_workspace(shape, self.device),
                        xr=torch.empty(saved["perm"].numel(), self.d, dtype=torch.bfloat16, device=self.device))
        return self.loc["xr"], saved["topk_w"].view(-1)

    def expert_forward(self, recv_dev, rows, xr, wr, w_gate_up, w_down):
        y = torch.empty(rows, self.d, dtype=torch.bfloat16, device=self.device)
        if rows:
            L = self.loc
            M.expert_fwd(L["shape"], self.G, recv_dev, xr, w_gate_up, w_down, y, L["saved"], L["ws"], self.stream)
        return y

    def expert_grad_buffer(self):
        if self.loc["rows"] == 0:
            return torch.empty(0, self.d, dtype=torch.bfloat16, device=self.device)
        return torch.empty_like(self.loc["xr"])

    def expert_backward(self, gr, w_gate_up, w_down):
        rows = self.loc["rows"]
        dx_rows = torch.empty(rows, self.d, dtype=torch.bfloat16, device=self.device)
        ds_rows = torch.empty(rows, dtype=torch.float32, device=self.device)
        if rows == 0:
            return dx_rows, ds_rows, torch.zeros_like(w_gate_up), torch.zeros_like(w_down)
        dwgu, dwd = torch.empty_like(w_gate_up), torch.empty_like(w_down)
        L = self.loc
        M.expert_bwd(L["shape"], gr, L["xr"], w_gate_up, w_down, L["saved"], dx_rows, dwgu, dwd, ds_rows, L["ws"],
                     self.stream)
        return dx_rows, ds_rows, dwgu, dwd

    def status(self) -> int:
        s = M.get_status(self.ws, self.stream)
        if self.loc and self.loc.get("rows"):
            s = s or M.get_status(self.loc["ws"], self.stream)
        return s

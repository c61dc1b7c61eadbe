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
     the local experts are taken in chunks: the rows of every chunk are
     posted at once, and the GEMMs of chunk c start as soon as its rows have
     arrived, while the rows of the later chunks are still crossing the
     links and the results of the earlier ones are on their way back;
  5. the backward sends grad_out rows the same way, the expert rank computes
     the dx rows, the routing-score gradients and its experts' weight
     gradients (moe_expert_bwd), and the source finishes dx, dscore and
     dlogits (moe_ep_backward_finish).

Every rank posts the same collectives in the same order.  Segments a rank
sends to itself are plain device copies.  The point-to-point operations of
one exchange are posted as one batch, ordered by peer, then expert, then
tensor, on both sides; each carries a tag that counts its position from the
exchange's first tag, so that backends that match messages by tag (gloo) pair
them the same way as NCCL, also while several exchanges are in flight.

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
    E_all: int = 0      # experts per rank (0: E_loc); a chunk's plan covers local experts
    e0: int = 0         # [e0, e0 + E_loc) of them, its layout and offsets its own

    def _ge(self, q, e):
        return q * (self.E_all or self.E_loc) + self.e0 + e

    def to_experts(self, send, recv, send_rows_from_padded=True):
        """(send segments, receive segments) of a source -> expert exchange:
        per peer q and expert e, the source's rows [start, start + n) and the
        expert side's rows [start, start + n)."""
        out_s, out_r = [], []
        for q in range(self.G):
            for e in range(self.E_loc):
                ge = self._ge(q, e)
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
                ge = self._ge(q, e)
                m = self.recv[q][e]
                if m:
                    out_s.append((q, send, self.cmp_off[q][e], m))
                n = self.counts[ge]
                if n:
                    out_r.append((q, recv, self.offsets[ge], n))
        return out_s, out_r


class Pending:
    """The point-to-point operations of one posted exchange.  wait(): with
    NCCL the caller's stream waits for them (the host does not block); with
    gloo the host waits."""

    def __init__(self, works):
        self.works = works

    def wait(self):
        for w in self.works:
            w.wait()
        self.works = []


def post_exchange(segment_lists, rank, group=None, tag0=0):
    """Post every (send, receive) segment list pair as one batch of
    point-to-point operations and return it as a Pending.  Each list entry is
    (peer, tensor, first row, rows).  The k-th message between two ranks in
    one direction carries tag tag0 + k on both sides.  Segments to the rank
    itself are copied on the caller's stream before the batch is posted."""
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
        ops.append(dist.P2POp(dist.isend, t[a:a + n], q, group, tag0 + k))
    for q, t, a, n in recvs:
        if q == rank:
            continue
        dist = dist or _dist()
        k = tag_r.get(q, 0)
        tag_r[q] = k + 1
        ops.append(dist.P2POp(dist.irecv, t[a:a + n], q, group, tag0 + k))
    return Pending(dist.batch_isend_irecv(ops) if ops else [])


def exchange(segment_lists, rank, group=None, tag0=0):
    """post_exchange, then wait for it."""
    post_exchange(segment_lists, rank, group, tag0).wait()


def chunk_bounds(E_loc, chunks):
    """[e0, e1) of each of min(chunks, E_loc) chunks of the local experts, in
    order, sizes differing by at most one."""
    n = max(1, min(int(chunks), E_loc))
    return [(c * E_loc // n, (c + 1) * E_loc // n) for c in range(n)]


class EPMoELayer:
    """The fused MoE layer with its experts spread over a process group.

    backend: the device steps (CudaEP for the library; any object with the
    same methods).  w_gate_up / w_down passed to forward and backward are this
    rank's experts' weights, [E/G, 2I, d] and [E/G, d, I].  chunks: how many
    groups of local experts the exchanges and the expert GEMMs are split into,
    so that they overlap (1: exchange everything, then compute)."""

    def __init__(self, backend, group=None, chunks=4):
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
        self.bounds = chunk_bounds(self.E_loc, chunks)
        self.tag_stride = 2 * self.E_loc + 1  # messages per peer in one exchange, at most
        self.plans = None
        self.sides = None
        self._whole = None

    @property
    def plan(self):
        """The whole step's plan (all local experts in one layout)."""
        return self._whole

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
        self._whole = Plan(G, E_loc, src["counts"], src["group_start"], src["offsets"], recv, row_off, cmp_off, rows,
                           padded)
        recv_2d = recv_dev.view(G, E_loc)
        plans, sides = [], []
        for e0, e1 in self.bounds:
            rc = [r[e0:e1] for r in recv]
            ro, co, n, pad = M.ep_expert_layout(G, e1 - e0, rc)
            plans.append(Plan(G, e1 - e0, src["counts"], src["group_start"], src["offsets"], rc, ro, co, n, pad,
                              E_all=E_loc, e0=e0))
            # a fresh copy: the library wants 16-byte aligned device arrays
            sides.append(b.expert_side(recv_2d[:, e0:e1].clone().view(-1), n, e0, e1))
        self.plans, self.sides = plans, sides
        tag = 0
        inbound = []
        for p, sd in zip(plans, sides):  # every chunk's rows in flight at once
            inbound.append(post_exchange([p.to_experts(src["xs"], sd.xr),
                                          p.to_experts(src["w_rows"], sd.wr, send_rows_from_padded=False)],
                                         self.rank, self.group, tag))
            tag += self.tag_stride
        ys = b.source_rows()
        outbound = []
        for p, sd, pend, (e0, e1) in zip(plans, sides, inbound, self.bounds):
            pend.wait()
            y_rows = sd.forward(w_gate_up[e0:e1], w_down[e0:e1])
            outbound.append(post_exchange([p.to_sources(y_rows, ys)], self.rank, self.group, tag))
            tag += self.tag_stride
        for pend in outbound:
            pend.wait()
        return b.combine(ys)

    def backward(self, grad_out, w_gate_up, w_down):
        """Returns dx, dscore, dlogits (this rank's tokens) and dW_gate_up,
        dW_down (this rank's experts)."""
        b, plans, sides = self.b, self.plans, self.sides
        if plans is None:
            raise RuntimeError("backward before forward")
        gs = b.dispatch_grad(grad_out)
        grs = [sd.grad_buffer() for sd in sides]
        tag = 0
        inbound = []
        for p, gr in zip(plans, grs):
            inbound.append(post_exchange([p.to_experts(gs, gr)], self.rank, self.group, tag))
            tag += self.tag_stride
        dxs, dss = b.source_grad_rows()
        dwgu, dwd = b.weight_grads(w_gate_up, w_down)
        outbound = []
        for p, sd, gr, pend, (e0, e1) in zip(plans, sides, grs, inbound, self.bounds):
            pend.wait()
            dx_rows, ds_rows = sd.backward(gr, w_gate_up[e0:e1], w_down[e0:e1], dwgu[e0:e1], dwd[e0:e1])
            outbound.append(post_exchange([p.to_sources(dx_rows, dxs), p.to_sources(ds_rows, dss)], self.rank,
                                          self.group, tag))
            tag += self.tag_stride
        for pend in outbound:
            pend.wait()
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
        self.sides = []  # the expert sides of the current step

    # ---- source side ----
    def route_dispatch(self, x, logits):
        self.sides = []
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
    def weight_grads(self, w_gate_up, w_down):
        """Buffers for this rank's experts' weight gradients (every chunk writes its slice)."""
        return torch.empty_like(w_gate_up), torch.empty_like(w_down)

    def expert_side(self, recv_dev, rows, e0, e1):
        """The expert side of local experts [e0, e1) for a step that receives
        `rows` rows for them: recv_dev = int32 [G * (e1 - e0)] on the device,
        rows of local expert e from source s at s * (e1 - e0) + e - e0."""
        return _CudaExpertSide(self, recv_dev, rows, e1 - e0)

    def status(self) -> int:
        s = M.get_status(self.ws, self.stream)
        for sd in self.sides:
            s = s or sd.status()
        return s


class _CudaExpertSide:
    """Buffers and device steps of one chunk of local experts (moe_expert_fwd
    / moe_expert_bwd on a problem of `rows` rows and E_c experts, k = 1)."""

    def __init__(self, b, recv_dev, rows, E_c):
        self.b, self.recv_dev, self.rows, self.E_c = b, recv_dev, rows, E_c
        dev, d = b.device, b.d
        b.sides.append(self)
        if rows == 0:
            self.xr = torch.empty(0, d, dtype=torch.bfloat16, device=dev)
            self.wr = torch.empty(0, dtype=torch.float32, device=dev)
            return
        self.shape = M.make_shape(rows, d, E_c, 1, b.I, M.MOE_BF16, b.max_sms, b.limit)
        self.saved = M.alloc_saved(self.shape, dev, keep_sorted_x=False)
        self.ws = M.alloc_workspace(self.shape, dev)
        self.xr = torch.empty(self.saved["perm"].numel(), d, dtype=torch.bfloat16, device=dev)
        self.wr = self.saved["topk_w"].view(-1)

    def forward(self, w_gate_up, w_down):
        """y rows [rows, d] in compact order."""
        y = torch.empty(self.rows, self.b.d, dtype=torch.bfloat16, device=self.b.device)
        if self.rows:
            M.expert_fwd(self.shape, self.b.G, self.recv_dev, self.xr, w_gate_up, w_down, y, self.saved, self.ws,
                         self.b.stream)
        return y

    def grad_buffer(self):
        """Where grad_out rows land (the layout of xr)."""
        return torch.empty_like(self.xr)

    def backward(self, gr, w_gate_up, w_down, dwgu, dwd):
        """dx rows and dscore rows (compact order); writes this chunk's experts'
        weight gradients into dwgu, dwd (contiguous slices)."""
        dev = self.b.device
        dx_rows = torch.empty(self.rows, self.b.d, dtype=torch.bfloat16, device=dev)
        ds_rows = torch.empty(self.rows, dtype=torch.float32, device=dev)
        if self.rows == 0:
            dwgu.zero_()
            dwd.zero_()
            return dx_rows, ds_rows
        M.expert_bwd(self.shape, gr, self.xr, w_gate_up, w_down, self.saved, dx_rows, dwgu, dwd, ds_rows, self.ws,
                     self.b.stream)
        return dx_rows, ds_rows

    def status(self) -> int:
        return M.get_status(self.ws, self.b.stream) if self.rows else 0

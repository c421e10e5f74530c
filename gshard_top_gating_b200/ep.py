"""Expert-parallel layer forward over G ranks (marshalling and byte movement only).

    layer = EPMoeLayer(G, g, S_max, S_total_max, M, H, E, k, cf, Wg, bias, W1_local, W2_local,
                       phases=2)
    y = ep_forward_dist(layer, x)            # one process per GPU, torch.distributed (NCCL)
    ys = ep_forward_local(layers, xs)        # G ranks emulated in one process on one device

Each rank holds a contiguous block of the batch's tokens and the experts
[g*E/G, (g+1)*E/G) ("GShard (Expert Parallelism)", "In plain words": tokens go
to the devices that host their experts by an all-to-all and come back by a second
one).  All arithmetic runs in the CUDA library (moe_ep_* in include/moe.h); this
module only moves bytes between the library's four steps:

    route -> all-gather of the per-rank stats -> dispatch -> all-to-all ->
    experts -> all-to-all back -> combine

The exchange sizes come from the library's plan: rank g sends send_rows[d] rows
to rank d and receives recv_rows[q] rows from rank q.  With two phases (bf16) each
exchange is split in two by expert slot, so that the second half travels while the
experts compute the first, and the first half returns while they compute the second;
the result is bit for bit the one-phase forward's.

Over peer memory (`set_peers` with every rank's receive buffer as this GPU addresses it)
the pack kernel stores each kept row straight into its owner's receive buffer and the
combine reads the expert outputs from there: neither all-to-all is a separate step
(`ep_forward_local_peers` on one device; `ep_forward_dist_peers` across processes, with
the caller mapping the buffers).
"""
from __future__ import annotations

import numpy as np
import torch

from . import _lib as L


class EPMoeLayer:
    """One rank's share of the layer: the whole gate, E/G experts, its buffers."""

    def __init__(self, G, g, S_max, S_total_max, M, H, E, k, capacity_factor, Wg, gate_bias,
                 W1_local, W2_local, phases: int = 1, recvbuf: torch.Tensor | None = None):
        act = W1_local.dtype
        if act not in (torch.float32, torch.bfloat16):
            raise TypeError("expert weights must be float32 or bfloat16")
        for t in (Wg, W1_local, W2_local) + ((gate_bias,) if gate_bias is not None else ()):
            if not (t.is_cuda and t.is_contiguous()):
                raise ValueError("weights must be contiguous CUDA tensors")
        if E % G or W1_local.shape[0] != E // G or W2_local.shape[0] != E // G:
            raise ValueError("each rank holds E/G experts")
        self.G, self.g, self.S_max, self.M, self.H, self.E, self.k = G, g, S_max, M, H, E, k
        self.cf = capacity_factor
        self.act = act
        self._keep = (Wg, gate_bias, W1_local, W2_local)
        self.h = L.moe_ep_create(G, g, S_max, S_total_max, M, H, E, k, capacity_factor, act, Wg, gate_bias,
                                 W1_local, W2_local)
        self.phases = phases
        if phases != 1:
            L.moe_ep_set_phases(self.h, phases)
        dev = W1_local.device
        ns, nr = L.moe_ep_buffer_rows(self.h)
        self.sendbuf = torch.empty(max(ns, 1), M, dtype=act, device=dev)
        if recvbuf is not None:              # e.g. a buffer the other ranks can map
            if recvbuf.dtype != act or recvbuf.dim() != 2 or recvbuf.shape[1] != M or recvbuf.shape[0] < nr:
                raise ValueError("recvbuf must be [>= receive rows, M] of the activation dtype")
            self.recvbuf = recvbuf
        else:
            self.recvbuf = torch.empty(max(nr, 1), M, dtype=act, device=dev)
        self.stats = torch.zeros(L.moe_ep_stats_len(E, k), dtype=torch.float64, device=dev)
        self.S = 0
        self.send_rows = self.recv_rows = None

    # the four library steps
    def route(self, x: torch.Tensor, stream=None) -> torch.Tensor:
        if x.dtype != self.act or not x.is_contiguous() or x.dim() != 2 or x.shape[1] != self.M:
            raise ValueError("x must be a contiguous [S, M] tensor of the activation dtype")
        self.S = x.shape[0]
        L.moe_ep_route(self.h, self.S, x, self.stats, stream)
        return self.stats

    def dispatch(self, stats_all: np.ndarray, x: torch.Tensor, stream=None):
        """Returns (send_rows, recv_rows), each [phases, G]."""
        send, recv = L.moe_ep_dispatch(self.h, stats_all, x, self.sendbuf, self.G, stream, self.phases)
        self.send_rows = send.reshape(self.phases, self.G)
        self.recv_rows = recv.reshape(self.phases, self.G)
        return self.send_rows, self.recv_rows

    def experts(self, stream=None) -> None:
        L.moe_ep_experts(self.h, self.recvbuf, stream)

    # the peer-memory forms
    def set_peers(self, recv_ptrs) -> None:
        """recv_ptrs: every rank's receive buffer address as this GPU sees it (rank order)."""
        L.moe_ep_set_peers(self.h, recv_ptrs)

    def dispatch_to_peers(self, stats_all: np.ndarray, x: torch.Tensor, stream=None):
        send, recv = L.moe_ep_dispatch_to_peers(self.h, stats_all, x, self.G, stream)
        self.send_rows, self.recv_rows = send.reshape(1, self.G), recv.reshape(1, self.G)
        return self.send_rows, self.recv_rows

    def combine_from_peers(self, out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
        y = out if out is not None else torch.empty(self.S, self.M, dtype=self.act, device=self.recvbuf.device)
        L.moe_ep_combine_from_peers(self.h, y, stream)
        return y

    def experts_phase(self, phase: int, stream=None) -> None:
        L.moe_ep_experts_phase(self.h, self.recvbuf, phase, stream)

    def phase_rows(self, phase: int):
        """(send_off, send_rows[G], recv_off, recv_rows[G]) of one phase: the phase's
        region of each buffer starts after the earlier phases' rows."""
        so = int(self.send_rows[:phase].sum())
        ro = int(self.recv_rows[:phase].sum())
        return so, self.send_rows[phase], ro, self.recv_rows[phase]

    def combine(self, out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
        y = out if out is not None else torch.empty(self.S, self.M, dtype=self.act, device=self.sendbuf.device)
        L.moe_ep_combine(self.h, self.sendbuf, y, stream)
        return y

    def aux_loss(self):
        return L.moe_ep_aux_loss(self.h)

    def routing(self):
        dev = self.sendbuf.device
        S, k = self.S, self.k
        eidx = torch.empty(S, k, dtype=torch.int32, device=dev)
        gate = torch.empty(S, k, dtype=torch.float32, device=dev)
        slot = torch.empty(S, k, dtype=torch.int32, device=dev)
        spos = torch.empty(S, k, dtype=torch.int32, device=dev)
        logits = torch.empty(S, self.E, dtype=torch.float32, device=dev)
        L.moe_ep_get_routing(self.h, eidx, gate, slot, spos, logits)
        return eidx, gate, slot, spos, logits

    def close(self) -> None:
        if getattr(self, "h", None):
            L.moe_ep_destroy(self.h)
            self.h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def _offsets(rows) -> np.ndarray:
    return np.concatenate([[0], np.cumsum(np.asarray(rows, dtype=np.int64))])


def _exchange(layers, phase, back=False):
    """One phase's all-to-all between emulated ranks (device-to-device copies)."""
    G = len(layers)
    for q in range(G):
        sq, send_q, _, _ = layers[q].phase_rows(phase)
        soff = sq + _offsets(send_q)
        for d in range(G):
            _, _, rd, recv_d = layers[d].phase_rows(phase)
            roff = rd + _offsets(recv_d)
            n = int(send_q[d])
            assert n == int(recv_d[q]), "send and receive counts of a pair disagree"
            if n:
                src = layers[q].sendbuf[soff[d]:soff[d] + n]
                dst = layers[d].recvbuf[roff[q]:roff[q] + n]
                if back:
                    src.copy_(dst)
                else:
                    dst.copy_(src)


def ep_forward_local(layers, xs, outs=None):
    """G ranks of one layer emulated in one process (all on one device): every exchange
    is one device-to-device copy per (source, destination) block, phase by phase, in the
    order a rank takes them (the experts of phase p run after its rows arrived, the
    return of phase p after its experts).  Returns the outputs."""
    stats = [layer.route(x) for layer, x in zip(layers, xs)]
    stats_all = torch.stack(stats).cpu().numpy()                     # the all-gather
    for layer, x in zip(layers, xs):
        layer.dispatch(stats_all, x)
    phases = layers[0].phases
    for p in range(phases):
        _exchange(layers, p)                                         # the all-to-all of phase p
        for layer in layers:
            layer.experts_phase(p)
        _exchange(layers, p, back=True)                              # and back
    return [layer.combine(None if outs is None else outs[i]) for i, layer in enumerate(layers)]


def ep_forward_local_peers(layers, xs, outs=None):
    """G ranks emulated in one process on one device, over "peer memory": every rank's
    receive buffer is a buffer of this device, so the pack writes into the owners'
    buffers and the combine reads from them exactly as it would over NVLink.  Every
    rank's step finishes before any rank's next (one stream).  Returns the outputs."""
    ptrs = [layer.recvbuf.data_ptr() for layer in layers]
    for layer in layers:
        layer.set_peers(ptrs)
    stats = [layer.route(x) for layer, x in zip(layers, xs)]
    stats_all = torch.stack(stats).cpu().numpy()
    for layer, x in zip(layers, xs):
        layer.dispatch_to_peers(stats_all, x)
    for layer in layers:
        layer.experts()
    return [layer.combine_from_peers(None if outs is None else outs[i]) for i, layer in enumerate(layers)]


def ep_forward_dist_peers(layer: EPMoeLayer, x: torch.Tensor, group=None, out=None) -> torch.Tensor:
    """One rank's forward over peer memory in a torch.distributed job: `layer.set_peers`
    must already hold every rank's receive buffer as this GPU maps it (CUDA IPC or
    symmetric memory; `layer.recvbuf` is this rank's).  The ranks meet at a barrier
    after each step whose writes the others read."""
    import torch.distributed as dist

    def fence():
        torch.cuda.current_stream().synchronize()
        dist.barrier(group=group)

    G = layer.G
    stats = layer.route(x)
    gathered = torch.empty(G, stats.numel(), dtype=stats.dtype, device=stats.device)
    dist.all_gather_into_tensor(gathered, stats, group=group)
    layer.dispatch_to_peers(gathered.cpu().numpy(), x)
    fence()                                  # every rank's rows are in their owners' buffers
    layer.experts()
    fence()                                  # every expert output is in place
    y = layer.combine_from_peers(out)
    fence()                                  # no rank reads a buffer the next forward rewrites
    return y


def ep_forward_dist(layer: EPMoeLayer, x: torch.Tensor, group=None, out=None) -> torch.Tensor:
    """One rank's forward in a torch.distributed job of G ranks (one per GPU).

    With two phases the exchanges run asynchronously on the process group's stream:
    phase 1's rows travel while the experts compute phase 0, and phase 0's outputs
    return while they compute phase 1.  A collective starts after the work already
    queued on the current stream; `wait()` queues the current stream behind it."""
    import torch.distributed as dist
    G = layer.G
    stats = layer.route(x)
    gathered = torch.empty(G, stats.numel(), dtype=stats.dtype, device=stats.device)
    dist.all_gather_into_tensor(gathered, stats, group=group)
    layer.dispatch(gathered.cpu().numpy(), x)

    def a2a(phase, back):
        so, send, ro, recv = layer.phase_rows(phase)
        s_buf = layer.sendbuf[so:so + int(send.sum())]
        r_buf = layer.recvbuf[ro:ro + int(recv.sum())]
        send_l, recv_l = [int(v) for v in send], [int(v) for v in recv]
        if back:
            return dist.all_to_all_single(s_buf, r_buf, send_l, recv_l, group=group, async_op=True)
        return dist.all_to_all_single(r_buf, s_buf, recv_l, send_l, group=group, async_op=True)

    there = [a2a(0, False)]
    back = []
    for p in range(layer.phases):
        if p + 1 < layer.phases:
            there.append(a2a(p + 1, False))                          # the next phase travels ...
        there[p].wait()
        layer.experts_phase(p)                                       # ... while this one computes
        back.append(a2a(p, True))
    for w in back:
        w.wait()
    return layer.combine(out)

"""Expert-parallel layer forward over G ranks (marshalling and byte movement only).

    layer = EPMoeLayer(G, g, S_max, S_total_max, M, H, E, k, cf, Wg, bias, W1_local, W2_local)
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
to rank d and receives recv_rows[q] rows from rank q.
"""
from __future__ import annotations

import numpy as np
import torch

from . import _lib as L


class EPMoeLayer:
    """One rank's share of the layer: the whole gate, E/G experts, its buffers."""

    def __init__(self, G, g, S_max, S_total_max, M, H, E, k, capacity_factor, Wg, gate_bias,
                 W1_local, W2_local):
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
        dev = W1_local.device
        ns, nr = L.moe_ep_buffer_rows(self.h)
        self.sendbuf = torch.empty(max(ns, 1), M, dtype=act, device=dev)
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
        self.send_rows, self.recv_rows = L.moe_ep_dispatch(self.h, stats_all, x, self.sendbuf, self.G, stream)
        return self.send_rows, self.recv_rows

    def experts(self, stream=None) -> None:
        L.moe_ep_experts(self.h, self.recvbuf, stream)

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


def ep_forward_local(layers, xs, outs=None):
    """G ranks of one layer emulated in one process (all on one device): every exchange
    is one device-to-device copy per (source, destination) block.  Returns the outputs."""
    G = len(layers)
    stats = [layer.route(x) for layer, x in zip(layers, xs)]
    stats_all = torch.stack(stats).cpu().numpy()                     # the all-gather
    plans = [layer.dispatch(stats_all, x) for layer, x in zip(layers, xs)]
    soff = [_offsets(send) for send, _ in plans]
    roff = [_offsets(recv) for _, recv in plans]
    for q in range(G):                                               # the all-to-all
        for d in range(G):
            n = int(plans[q][0][d])
            assert n == int(plans[d][1][q]), "send and receive counts of a pair disagree"
            if n:
                layers[d].recvbuf[roff[d][q]:roff[d][q] + n].copy_(layers[q].sendbuf[soff[q][d]:soff[q][d] + n])
    for layer in layers:
        layer.experts()
    for q in range(G):                                               # the all-to-all back
        for d in range(G):
            n = int(plans[q][0][d])
            if n:
                layers[q].sendbuf[soff[q][d]:soff[q][d] + n].copy_(layers[d].recvbuf[roff[d][q]:roff[d][q] + n])
    return [layer.combine(None if outs is None else outs[i]) for i, layer in enumerate(layers)]


def ep_forward_dist(layer: EPMoeLayer, x: torch.Tensor, group=None, out=None) -> torch.Tensor:
    """One rank's forward in a torch.distributed job of G ranks (one per GPU)."""
    import torch.distributed as dist
    G = layer.G
    stats = layer.route(x)
    gathered = torch.empty(G, stats.numel(), dtype=stats.dtype, device=stats.device)
    dist.all_gather_into_tensor(gathered, stats, group=group)
    send, recv = layer.dispatch(gathered.cpu().numpy(), x)
    ns, nr = int(send.sum()), int(recv.sum())
    dist.all_to_all_single(layer.recvbuf[:nr], layer.sendbuf[:ns], [int(v) for v in recv],
                           [int(v) for v in send], group=group)
    layer.experts()
    dist.all_to_all_single(layer.sendbuf[:ns], layer.recvbuf[:nr], [int(v) for v in send],
                           [int(v) for v in recv], group=group)
    return layer.combine(out)

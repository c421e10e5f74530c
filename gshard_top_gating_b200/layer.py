"""MoeLayer: an owning wrapper around one C-ABI handle (marshalling only).

    layer = MoeLayer(S_max, M, H, E, k, cf, Wg, bias, W1, W2)   # device tensors
    y = layer(x)                                                 # moe_forward
    l_aux, z = layer.aux_loss()                                  # moe_aux_loss
    g = layer.backward(x, dy, a_aux, a_z)                        # moe_backward

The tensors passed in are borrowed by the C library; this object keeps Python
references to them so they outlive the handle.
"""
from __future__ import annotations

import torch

from . import _lib as L


class MoeLayer:
    def __init__(self, S_max, M, H, E, k, capacity_factor, Wg, gate_bias, W1, W2):
        act = W1.dtype
        if act not in (torch.float32, torch.bfloat16):
            raise TypeError("expert weights must be float32 or bfloat16")
        for t in (Wg, W1, W2) + ((gate_bias,) if gate_bias is not None else ()):
            if not (t.is_cuda and t.is_contiguous()):
                raise ValueError("weights must be contiguous CUDA tensors")
        if Wg.dtype != torch.float32 or (gate_bias is not None and gate_bias.dtype != torch.float32):
            raise TypeError("gate weights and bias are float32")
        self.S_max, self.M, self.H, self.E, self.k = S_max, M, H, E, k
        self.cf = capacity_factor
        self.act = act
        self._keep = (Wg, gate_bias, W1, W2)
        self.h = L.moe_create(S_max, M, H, E, k, capacity_factor, act, Wg, gate_bias, W1, W2)

    def __call__(self, x: torch.Tensor, out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
        if x.dtype != self.act or not x.is_contiguous() or x.dim() != 2 or x.shape[1] != self.M:
            raise ValueError("x must be a contiguous [S, M] tensor of the activation dtype")
        S = x.shape[0]
        y = out if out is not None else torch.empty_like(x)
        L.moe_forward(self.h, S, x, y, stream)
        return y

    def forward_host(self, x_host: torch.Tensor, y_host: torch.Tensor, stream=None) -> None:
        L.moe_forward_host(self.h, x_host.shape[0], x_host, y_host, stream)

    def aux_loss(self, stream=None):
        return L.moe_aux_loss(self.h, stream)

    def enable_backward(self) -> None:
        """Allocate the backward workspace now (moe_enable_backward).  Forwards
        that run after it also store the ReLU mask bits the backward reads; a
        backward of a forward that ran before it re-reads h instead."""
        if not getattr(self, "_bwd", False):
            L.moe_enable_backward(self.h)
            self._bwd = True

    def backward(self, x: torch.Tensor, dy: torch.Tensor, a_aux: float = 0.0, a_z: float = 0.0,
                 stream=None, out: dict | None = None, skip_empty_experts: bool = False) -> dict:
        """Gradients of <dy, y> + a_aux*l_aux + a_z*z for the last forward (which took x).

        Returns dx, dWg, dbias (None without a gate bias), dW1, dW2: new tensors,
        or the tensors of `out` (same keys) written in place.  With
        skip_empty_experts, dW1[e] and dW2[e] of experts that kept no token are
        left as they were (MOE_BWD_SKIP_EMPTY_EXPERTS).  The backward workspace is
        allocated on the first call.
        """
        self.enable_backward()
        for t in (x, dy):
            if t.dtype != self.act or not t.is_contiguous() or t.dim() != 2 or t.shape[1] != self.M:
                raise ValueError("x and dy must be contiguous [S, M] tensors of the activation dtype")
        S = x.shape[0]
        dev = x.device
        out = dict(out or {})
        dx = out.get("dx") if out.get("dx") is not None else torch.empty_like(x)
        dWg = out.get("dWg") if out.get("dWg") is not None else \
            torch.empty(self.M, self.E, dtype=torch.float32, device=dev)
        dbias = None
        if self._keep[1] is not None:
            dbias = out.get("dbias") if out.get("dbias") is not None else \
                torch.empty(self.E, dtype=torch.float32, device=dev)
        dW1 = out.get("dW1") if out.get("dW1") is not None else \
            torch.empty(self.E, self.M, self.H, dtype=self.act, device=dev)
        dW2 = out.get("dW2") if out.get("dW2") is not None else \
            torch.empty(self.E, self.H, self.M, dtype=self.act, device=dev)
        for t in (dx, dWg, dW1, dW2) + ((dbias,) if dbias is not None else ()):
            if not (t.is_cuda and t.is_contiguous()):
                raise ValueError("gradient buffers must be contiguous CUDA tensors")
        L.moe_set_backward_flags(self.h, L.MOE_BWD_SKIP_EMPTY_EXPERTS if skip_empty_experts else 0)
        L.moe_backward(self.h, S, x, dy, a_aux, a_z, dx, dWg, dbias, dW1, dW2, stream)
        return {"dx": dx, "dWg": dWg, "dbias": dbias, "dW1": dW1, "dW2": dW2}

    def capacity(self, S: int) -> int:
        return L.moe_get_capacity(self.h, S)

    def logits(self, S: int, stream=None) -> torch.Tensor:
        out = torch.empty(S, self.E, dtype=torch.float32, device="cuda")
        L.moe_get_logits(self.h, out, stream)
        return out

    def routing(self, S: int, stream=None):
        eidx = torch.empty(S, self.k, dtype=torch.int32, device="cuda")
        gate = torch.empty(S, self.k, dtype=torch.float32, device="cuda")
        slot = torch.empty(S, self.k, dtype=torch.int32, device="cuda")
        cnt = torch.empty(self.E, dtype=torch.int32, device="cuda")
        L.moe_get_routing(self.h, eidx, gate, slot, cnt, stream)
        return eidx, gate, slot, cnt

    def expert_rows(self, which: int, e: int, nrows: int, stream=None) -> torch.Tensor:
        """Rows 0..nrows-1 of expert e in xbuf / hbuf / ybuf (L.MOE_BUF_X / _H / _Y)."""
        width = self.H if which == L.MOE_BUF_H else self.M
        out = torch.empty(nrows, width, dtype=self.act, device="cuda")
        L.moe_get_expert_rows(self.h, which, e, nrows, out, stream)
        return out

    def set_rerouting(self, on: bool) -> None:
        """Give dropped choices a second chance at an alternative expert (MOE_ROUTE_REROUTE)."""
        L.moe_set_routing_flags(self.h, L.MOE_ROUTE_REROUTE if on else 0)

    def serving_experts(self, S: int, stream=None) -> torch.Tensor:
        dest = torch.empty(S, self.k, dtype=torch.int32, device="cuda")
        L.moe_get_serving_experts(self.h, dest, stream)
        return dest

    def route_from_logits(self, logits: torch.Tensor, stream=None) -> None:
        L.moe_route_from_logits(self.h, logits.shape[0], logits, stream)

    def close(self) -> None:
        if getattr(self, "h", None):
            L.moe_destroy(self.h)
            self.h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

"""Seeded synthetic inputs for the MoE-layer workloads.

This module is shared by the CUDA path's harness (tests, bench, smoke) and by the
CPU oracle's tests.  It holds the workload shapes and a counter-based random
generator and nothing of the layer's arithmetic: no logits, no routing, no
capacity, no expert math.

Generator.  Every value is a pure function of (seed, tensor id, element index):
a SplitMix64 mix (Steele, Lea and Flood, "Fast splittable pseudorandom number
generators", OOPSLA 2014) of a Weyl counter gives 64 random bits; each element
takes six such draws, i.e. twelve 32-bit uniforms u_i = (v_i + 1/2) / 2^32, and
the standard-normal variate is the Irwin-Hall sum  z = sum_i u_i - 6  (mean 0,
variance 1).  Only integer operations and exact float64 additions are used up to
z, then one float64 multiply by the standard deviation, one rounding to float32
and (for bf16 tensors) one round-to-nearest-even to bfloat16.  All of these are
correctly rounded IEEE operations, so the same call gives bit-identical tensors
on the CPU and on a GPU: the oracle can be fed host copies of exactly the
tensors the device path consumes.

Workloads (sizes as the method's benchmark configurations state them):

====== ======= ====== ====== ===== === ===== ======= ===========================
name   S       M      H      E     k   cf    act     notes
====== ======= ====== ====== ===== === ===== ======= ===========================
tiny   256     64     256    8     2   1.25  f32     C = 80, parity case
mid    8192    1024   4096   32    2   2.0   bf16    isotropic, few drops
skewed 16384   1024   8192   128   2   1.25  bf16    Zipf-like gate bias b_j
large  65536   2048   8192   64    2   1.0   bf16    with aux / z losses
wide   16384   7168   2048   256   8   1.25  bf16    256 experts, top-8
====== ======= ====== ====== ===== === ===== ======= ===========================

x ~ N(0,1) [S,M]; W_g ~ N(0,1/M) fp32 [M,E]; W1 ~ N(0,1/M) [E,M,H];
W2 ~ N(0,1/H) [E,H,M]; no biases except the skewed workload's fixed gate bias
b_j = 2 log(1/(j+1)) (float64, rounded to float32).
"""
from __future__ import annotations

import math
from dataclasses import dataclass, replace

import torch

__all__ = ["Workload", "WORKLOADS", "normal", "make_inputs", "gate_bias", "expert_weights"]


@dataclass(frozen=True)
class Workload:
    name: str
    S: int
    M: int
    H: int
    E: int
    k: int
    cf: float
    act: str            # "f32" or "bf16": dtype of x, W1, W2, y
    skew_bias: bool = False
    seed: int = 0

    @property
    def torch_act(self) -> torch.dtype:
        return torch.float32 if self.act == "f32" else torch.bfloat16

    def with_(self, **kw) -> "Workload":
        return replace(self, **kw)


WORKLOADS = {
    "tiny": Workload("tiny", 256, 64, 256, 8, 2, 1.25, "f32"),
    "mid": Workload("mid", 8192, 1024, 4096, 32, 2, 2.0, "bf16"),
    "skewed": Workload("skewed", 16384, 1024, 8192, 128, 2, 1.25, "bf16", skew_bias=True),
    "large": Workload("large", 65536, 2048, 8192, 64, 2, 1.0, "bf16"),
    "wide": Workload("wide", 16384, 7168, 2048, 256, 8, 1.25, "bf16"),
}

# tensor ids of the counter-based stream
TID_X, TID_WG, TID_W1, TID_W2 = 1, 2, 3, 4
TID_DY = 5        # upstream gradient dL/dy of the backward

_MASK64 = (1 << 64) - 1
_GOLDEN = 0x9E3779B97F4A7C15
_MIX1 = 0xBF58476D1CE4E5B9
_MIX2 = 0x94D049BB133111EB
_DRAWS = 6            # 64-bit draws per element -> 12 uniforms
_CHUNK = 1 << 22      # elements generated per pass


def _signed(v: int) -> int:
    v &= _MASK64
    return v - (1 << 64) if v >= (1 << 63) else v


def _mix_int(z: int) -> int:
    """SplitMix64 finaliser on a Python int (used for the per-tensor key)."""
    z &= _MASK64
    z = ((z ^ (z >> 30)) * _MIX1) & _MASK64
    z = ((z ^ (z >> 27)) * _MIX2) & _MASK64
    return z ^ (z >> 31)


def _srl(z: torch.Tensor, s: int) -> torch.Tensor:
    """Logical right shift of int64 bit patterns."""
    return (z >> s) & ((1 << (64 - s)) - 1)


def _mix(z: torch.Tensor) -> torch.Tensor:
    """SplitMix64 finaliser on int64 tensors (wrapping two's-complement arithmetic)."""
    z = (z ^ _srl(z, 30)) * _signed(_MIX1)
    z = (z ^ _srl(z, 27)) * _signed(_MIX2)
    return z ^ _srl(z, 31)


def _key(seed: int, tid: int) -> int:
    return _mix_int((seed << 32) ^ (tid * 0x632BE59BD9B4E019))


def _irwin_hall(idx: torch.Tensor, key: int) -> torch.Tensor:
    """z = sum of 12 uniforms - 6 for every element index in `idx` (int64), float64."""
    acc = torch.zeros(idx.shape, dtype=torch.float64, device=idx.device)
    base = idx * _DRAWS
    two32 = float(1 << 32)
    for d in range(_DRAWS):
        ctr = (base + (d + 1)) * _signed(_GOLDEN) + _signed(key)
        z = _mix(ctr)
        hi = _srl(z, 32).to(torch.float64)
        lo = (z & 0xFFFFFFFF).to(torch.float64)
        acc += (hi + 0.5) / two32
        acc += (lo + 0.5) / two32
    return acc - 6.0


def normal(shape, std: float, seed: int, tid: int, dtype: torch.dtype,
           device="cpu", index_offset: int = 0) -> torch.Tensor:
    """Tensor of `shape` with N(0, std^2) entries (Irwin-Hall approximation).

    Element i (row-major) uses counter index `index_offset + i`, so any
    sub-block of a large tensor can be regenerated on its own.
    """
    n = 1
    for s in shape:
        n *= int(s)
    out = torch.empty(n, dtype=dtype, device=device)
    key = _key(seed, tid)
    chunk = _CHUNK if out.device.type == "cpu" else _CHUNK * 16
    for a in range(0, n, chunk):
        b = min(n, a + chunk)
        idx = torch.arange(a + index_offset, b + index_offset, dtype=torch.int64, device=device)
        z = _irwin_hall(idx, key) * std
        out[a:b] = z.to(torch.float32).to(dtype)
    return out.view(*shape)


def gate_bias(w: Workload, device="cpu"):
    """Fixed Zipf-like gate bias b_j = 2 log(1/(j+1)) of the skewed workload, or None."""
    if not w.skew_bias:
        return None
    vals = [2.0 * math.log(1.0 / (j + 1)) for j in range(w.E)]
    return torch.tensor(vals, dtype=torch.float64).to(torch.float32).to(device)


def make_inputs(w: Workload, device="cpu", S: int | None = None, weights: bool = True):
    """Generate (x, Wg, bias, W1, W2) of workload `w` directly on `device`.

    x is [S, M] in the activation dtype, Wg is fp32 [M, E], bias fp32 [E] or
    None, W1 is [E, M, H] and W2 is [E, H, M] in the activation dtype.  With
    weights=False the expert weights are skipped (returned as None).
    """
    S = w.S if S is None else S
    act = w.torch_act
    x = normal((S, w.M), 1.0, w.seed, TID_X, act, device)
    Wg = normal((w.M, w.E), 1.0 / math.sqrt(w.M), w.seed, TID_WG, torch.float32, device)
    b = gate_bias(w, device)
    W1 = W2 = None
    if weights:
        W1 = normal((w.E, w.M, w.H), 1.0 / math.sqrt(w.M), w.seed, TID_W1, act, device)
        W2 = normal((w.E, w.H, w.M), 1.0 / math.sqrt(w.H), w.seed, TID_W2, act, device)
    return x, Wg, b, W1, W2


def upstream_grad(w: Workload, device="cpu", S: int | None = None) -> torch.Tensor:
    """dL/dy for the backward: [S, M] N(0, 1) entries in the activation dtype."""
    S = w.S if S is None else S
    return normal((S, w.M), 1.0, w.seed, TID_DY, w.torch_act, device)


def expert_weights(w: Workload, e: int, device="cpu"):
    """Regenerate W1[e] and W2[e] alone (same bits as the full tensors)."""
    act = w.torch_act
    n1 = w.M * w.H
    W1e = normal((w.M, w.H), 1.0 / math.sqrt(w.M), w.seed, TID_W1, act, device, index_offset=e * n1)
    W2e = normal((w.H, w.M), 1.0 / math.sqrt(w.H), w.seed, TID_W2, act, device, index_offset=e * n1)
    return W1e, W2e

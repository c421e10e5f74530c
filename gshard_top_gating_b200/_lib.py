"""ctypes binding of the C ABI in include/moe.h (argument marshalling only).

Every function here has the name of the C entry point it calls and does nothing
but turn tensors into pointers, streams into handles and non-OK status codes
into MoeError.  All computation happens in the CUDA library; there is no other
path: if the shared library is missing the import fails loudly.
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libgshard_moe.so")

MOE_OK, MOE_ERR_INVALID_ARG, MOE_ERR_UNSUPPORTED, MOE_ERR_CUDA, MOE_ERR_OOM, MOE_ERR_STATE, \
    MOE_ERR_TIMEOUT = range(7)
MOE_F32, MOE_BF16 = 0, 1
MOE_BWD_SKIP_EMPTY_EXPERTS = 1
MOE_BUF_X, MOE_BUF_H, MOE_BUF_Y = 0, 1, 2
MOE_ROUTE_REROUTE = 1
MOE_NUM_STAGES = 6
STAGES = ("router", "scan", "dispatch", "ffn1", "ffn2", "combine")
MOE_NUM_BWD_STAGES = 8
BWD_STAGES = ("gate_bwd", "pad_zero", "dW2", "dP", "dW1", "dX_e", "dx", "dWg")


class MoeError(RuntimeError):
    def __init__(self, fn: str, status: int, msg: str):
        super().__init__(f"{fn}: {msg} (status {status})")
        self.status = status


def _load() -> ctypes.CDLL:
    if not os.path.exists(LIB_PATH):
        raise ImportError(
            f"CUDA library {LIB_PATH} is missing: build it with "
            "`python -m gshard_top_gating_b200.build` (there is no fallback path)")
    lib = ctypes.CDLL(LIB_PATH)
    P, I64, I32, D = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int32, ctypes.c_double
    sig = {
        "moe_create": [ctypes.POINTER(P), I64, I64, I64, I32, I32, D, ctypes.c_int, P, P, P, P],
        "moe_forward": [P, I64, P, P, P],
        "moe_forward_host": [P, I64, P, P, P],
        "moe_aux_loss": [P, ctypes.POINTER(ctypes.c_float), ctypes.POINTER(ctypes.c_float), P],
        "moe_destroy": [P],
        "moe_check": [P, P],
        "moe_get_logits": [P, P, P],
        "moe_get_routing": [P, P, P, P, P, P],
        "moe_route_from_logits": [P, I64, P, P],
        "moe_get_expert_rows": [P, I32, I32, I64, P, P],
        "moe_set_routing_flags": [P, ctypes.c_uint32],
        "moe_get_serving_experts": [P, P, P],
        "moe_get_capacity": [P, I64, ctypes.POINTER(I64)],
        "moe_set_profiling": [P, I32],
        "moe_get_stage_times": [P, ctypes.POINTER(ctypes.c_float), I32],
        "moe_selftest_wait_timeout": [I32, P],
        "moe_assign_slots_noalloc": [I64, I32, I32, I64, P, P, P, P],
        "moe_enable_backward": [P],
        "moe_set_backward_flags": [P, ctypes.c_uint32],
        "moe_get_backward_stage_times": [P, ctypes.POINTER(ctypes.c_float), I32],
        "moe_backward": [P, I64, P, P, ctypes.c_float, ctypes.c_float, P, P, P, P, P, P],
    }
    I64P = ctypes.POINTER(I64)
    sig.update({
        "moe_ep_plan": [I32, I32, I32, I32, D, P, P, I64P, P, P, P, P],
        "moe_ep_create": [ctypes.POINTER(P), I32, I32, I64, I64, I64, I64, I32, I32, D, ctypes.c_int,
                          P, P, P, P],
        "moe_ep_destroy": [P],
        "moe_ep_buffer_rows": [P, I64P, I64P],
        "moe_ep_route": [P, I64, P, P, P],
        "moe_ep_dispatch": [P, P, P, P, P, P, P],
        "moe_ep_experts": [P, P, P],
        "moe_ep_experts_phase": [P, P, I32, P],
        "moe_ep_set_peers": [P, P],
        "moe_ep_dispatch_to_peers": [P, P, P, P, P, P],
        "moe_ep_combine_from_peers": [P, P, P],
        "moe_ep_set_phases": [P, I32],
        "moe_ep_phase_plan": [I32, I32, I32, I32, D, P, P, I32, P, P, P],
        "moe_ep_combine": [P, P, P, P],
        "moe_ep_aux_loss": [P, ctypes.POINTER(ctypes.c_float), ctypes.POINTER(ctypes.c_float)],
        "moe_ep_get_routing": [P, P, P, P, P, P, P],
        "moe_ep_check": [P, P],
    })
    for name, args in sig.items():
        f = getattr(lib, name)
        f.argtypes = args
        f.restype = ctypes.c_int
    lib.moe_ep_stats_len.argtypes = [I32, I32]
    lib.moe_ep_stats_len.restype = I32
    lib.moe_kernels_per_forward.argtypes = [P, I64]
    lib.moe_kernels_per_forward.restype = I32
    lib.moe_kernels_per_backward.argtypes = [P, I64]
    lib.moe_kernels_per_backward.restype = I32
    lib.moe_status_string.argtypes = [ctypes.c_int]
    lib.moe_status_string.restype = ctypes.c_char_p
    lib.moe_stage_name.argtypes = [I32]
    lib.moe_stage_name.restype = ctypes.c_char_p
    lib.moe_backward_stage_name.argtypes = [I32]
    lib.moe_backward_stage_name.restype = ctypes.c_char_p
    return lib


lib = _load()


def _check(fn: str, status: int) -> None:
    if status != MOE_OK:
        raise MoeError(fn, status, lib.moe_status_string(status).decode())


def _ptr(t) -> int | None:
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _stream(stream) -> int | None:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream if torch.cuda.is_available() else None
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def moe_status_string(status: int) -> str:
    return lib.moe_status_string(status).decode()


def moe_stage_name(stage: int) -> str:
    return lib.moe_stage_name(stage).decode()


def moe_create(S_max, M, H, E, k, capacity_factor, act, Wg, gate_bias, W1, W2) -> int:
    h = ctypes.c_void_p()
    dt = MOE_BF16 if act in ("bf16", torch.bfloat16, MOE_BF16) else MOE_F32
    _check("moe_create", lib.moe_create(ctypes.byref(h), S_max, M, H, E, k, float(capacity_factor),
                                        dt, _ptr(Wg), _ptr(gate_bias), _ptr(W1), _ptr(W2)))
    return h.value


def moe_forward(h, S, x, y, stream=None) -> None:
    _check("moe_forward", lib.moe_forward(h, S, _ptr(x), _ptr(y), _stream(stream)))


def moe_forward_host(h, S, x_host, y_host, stream=None) -> None:
    _check("moe_forward_host", lib.moe_forward_host(h, S, _ptr(x_host), _ptr(y_host), _stream(stream)))


def moe_aux_loss(h, stream=None):
    a, z = ctypes.c_float(), ctypes.c_float()
    _check("moe_aux_loss", lib.moe_aux_loss(h, ctypes.byref(a), ctypes.byref(z), _stream(stream)))
    return a.value, z.value


def moe_destroy(h) -> None:
    _check("moe_destroy", lib.moe_destroy(h))


def moe_check(h, stream=None) -> None:
    _check("moe_check", lib.moe_check(h, _stream(stream)))


def moe_get_logits(h, logits, stream=None) -> None:
    _check("moe_get_logits", lib.moe_get_logits(h, _ptr(logits), _stream(stream)))


def moe_get_routing(h, eidx=None, gate=None, slot=None, cnt=None, stream=None) -> None:
    _check("moe_get_routing", lib.moe_get_routing(h, _ptr(eidx), _ptr(gate), _ptr(slot), _ptr(cnt),
                                                  _stream(stream)))


def moe_route_from_logits(h, S, logits, stream=None) -> None:
    _check("moe_route_from_logits", lib.moe_route_from_logits(h, S, _ptr(logits), _stream(stream)))


def moe_get_expert_rows(h, which, e, nrows, dst, stream=None) -> None:
    _check("moe_get_expert_rows", lib.moe_get_expert_rows(h, which, e, nrows, _ptr(dst), _stream(stream)))


def moe_set_routing_flags(h, flags: int) -> None:
    _check("moe_set_routing_flags", lib.moe_set_routing_flags(h, int(flags)))


def moe_get_serving_experts(h, dest, stream=None) -> None:
    _check("moe_get_serving_experts", lib.moe_get_serving_experts(h, _ptr(dest), _stream(stream)))


def moe_get_capacity(h, S) -> int:
    c = ctypes.c_int64()
    _check("moe_get_capacity", lib.moe_get_capacity(h, S, ctypes.byref(c)))
    return c.value


def moe_set_profiling(h, enable: bool) -> None:
    _check("moe_set_profiling", lib.moe_set_profiling(h, 1 if enable else 0))


def moe_get_stage_times(h):
    buf = (ctypes.c_float * MOE_NUM_STAGES)()
    _check("moe_get_stage_times", lib.moe_get_stage_times(h, buf, MOE_NUM_STAGES))
    return list(buf)


def moe_kernels_per_forward(h, S) -> int:
    return int(lib.moe_kernels_per_forward(h, S))


def moe_selftest_wait_timeout(limit_us: int, stream=None) -> int:
    """Returns the raw status (MOE_ERR_TIMEOUT when the bounded wait works)."""
    return int(lib.moe_selftest_wait_timeout(limit_us, _stream(stream)))


def moe_assign_slots_noalloc(S, E, k, C, eidx, slot, cnt, stream=None) -> None:
    """Capacity slots from expert ids with no device allocation (see include/moe.h)."""
    _check("moe_assign_slots_noalloc",
           lib.moe_assign_slots_noalloc(S, E, k, C, _ptr(eidx), _ptr(slot), _ptr(cnt), _stream(stream)))


def moe_enable_backward(h) -> None:
    _check("moe_enable_backward", lib.moe_enable_backward(h))


def moe_backward(h, S, x, dy, a_aux, a_z, dx, dWg, dbias, dW1, dW2, stream=None) -> None:
    _check("moe_backward", lib.moe_backward(h, S, _ptr(x), _ptr(dy), float(a_aux), float(a_z), _ptr(dx),
                                            _ptr(dWg), _ptr(dbias), _ptr(dW1), _ptr(dW2),
                                            _stream(stream)))


def moe_kernels_per_backward(h, S) -> int:
    return int(lib.moe_kernels_per_backward(h, S))


def moe_get_backward_stage_times(h):
    buf = (ctypes.c_float * MOE_NUM_BWD_STAGES)()
    _check("moe_get_backward_stage_times", lib.moe_get_backward_stage_times(h, buf, MOE_NUM_BWD_STAGES))
    return list(buf)


def moe_backward_stage_name(stage: int) -> str:
    return lib.moe_backward_stage_name(stage).decode()


def moe_set_backward_flags(h, flags: int) -> None:
    _check("moe_set_backward_flags", lib.moe_set_backward_flags(h, int(flags)))


# ---- expert parallelism (include/moe.h): host buffers are numpy int64 / float64 arrays

def _np_ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def moe_ep_stats_len(E, k) -> int:
    return int(lib.moe_ep_stats_len(E, k))


def moe_ep_plan(G, g, E, k, capacity_factor, counts, S):
    """Host exchange plan of rank g: (C, send_rows[G], recv_rows[G], base[G,k,E], kept[G,k,E])."""
    import numpy as np
    cnt = np.ascontiguousarray(counts, dtype=np.int64)
    Sv = np.ascontiguousarray(S, dtype=np.int64)
    C = ctypes.c_int64()
    send = np.zeros(G, dtype=np.int64)
    recv = np.zeros(G, dtype=np.int64)
    base = np.zeros((G, k, E), dtype=np.int64)
    kept = np.zeros((G, k, E), dtype=np.int64)
    _check("moe_ep_plan", lib.moe_ep_plan(G, g, E, k, float(capacity_factor), _np_ptr(cnt), _np_ptr(Sv),
                                          ctypes.byref(C), _np_ptr(send), _np_ptr(recv), _np_ptr(base),
                                          _np_ptr(kept)))
    return C.value, send, recv, base, kept


def moe_ep_create(G, g, S_max, S_total_max, M, H, E, k, capacity_factor, act, Wg, gate_bias, W1, W2) -> int:
    h = ctypes.c_void_p()
    dt = MOE_BF16 if act in ("bf16", torch.bfloat16, MOE_BF16) else MOE_F32
    _check("moe_ep_create", lib.moe_ep_create(ctypes.byref(h), G, g, S_max, S_total_max, M, H, E, k,
                                              float(capacity_factor), dt, _ptr(Wg), _ptr(gate_bias),
                                              _ptr(W1), _ptr(W2)))
    return h.value


def moe_ep_destroy(h) -> None:
    _check("moe_ep_destroy", lib.moe_ep_destroy(h))


def moe_ep_buffer_rows(h):
    a, b = ctypes.c_int64(), ctypes.c_int64()
    _check("moe_ep_buffer_rows", lib.moe_ep_buffer_rows(h, ctypes.byref(a), ctypes.byref(b)))
    return a.value, b.value


def moe_ep_route(h, S, x, stats, stream=None) -> None:
    _check("moe_ep_route", lib.moe_ep_route(h, S, _ptr(x), _ptr(stats), _stream(stream)))


def moe_ep_dispatch(h, stats_all, x, sendbuf, G, stream=None, phases=1):
    """stats_all: numpy float64 [G, stats_len]; returns (send_rows, recv_rows) int64, each
    [G] with one phase or [phases, G] (the handle's phase count must be `phases`)."""
    import numpy as np
    st = np.ascontiguousarray(stats_all, dtype=np.float64)
    send = np.zeros(phases * G, dtype=np.int64)
    recv = np.zeros(phases * G, dtype=np.int64)
    _check("moe_ep_dispatch", lib.moe_ep_dispatch(h, _np_ptr(st), _ptr(x), _ptr(sendbuf), _np_ptr(send),
                                                  _np_ptr(recv), _stream(stream)))
    if phases == 1:
        return send, recv
    return send.reshape(phases, G), recv.reshape(phases, G)


def moe_ep_set_peers(h, recv_ptrs) -> None:
    """recv_ptrs: G device addresses (ints) of every rank's receive buffer, or None."""
    if recv_ptrs is None:
        _check("moe_ep_set_peers", lib.moe_ep_set_peers(h, None))
        return
    arr = (ctypes.c_void_p * len(recv_ptrs))(*[int(p) for p in recv_ptrs])
    _check("moe_ep_set_peers", lib.moe_ep_set_peers(h, ctypes.cast(arr, ctypes.c_void_p)))


def moe_ep_dispatch_to_peers(h, stats_all, x, G, stream=None):
    """As moe_ep_dispatch, rows stored straight into the owners' receive buffers."""
    import numpy as np
    st = np.ascontiguousarray(stats_all, dtype=np.float64)
    send = np.zeros(G, dtype=np.int64)
    recv = np.zeros(G, dtype=np.int64)
    _check("moe_ep_dispatch_to_peers", lib.moe_ep_dispatch_to_peers(h, _np_ptr(st), _ptr(x), _np_ptr(send),
                                                                    _np_ptr(recv), _stream(stream)))
    return send, recv


def moe_ep_combine_from_peers(h, y, stream=None) -> None:
    _check("moe_ep_combine_from_peers", lib.moe_ep_combine_from_peers(h, _ptr(y), _stream(stream)))


def moe_ep_set_phases(h, phases: int) -> None:
    _check("moe_ep_set_phases", lib.moe_ep_set_phases(h, phases))


def moe_ep_experts_phase(h, recvbuf, phase: int, stream=None) -> None:
    _check("moe_ep_experts_phase", lib.moe_ep_experts_phase(h, _ptr(recvbuf), phase, _stream(stream)))


def moe_ep_phase_plan(G, g, E, k, capacity_factor, counts, S, phases):
    """Per-phase row counts of rank g: (send_rows[phases, G], recv_rows[phases, G], split[E])."""
    import numpy as np
    cnt = np.ascontiguousarray(counts, dtype=np.int64)
    Sv = np.ascontiguousarray(S, dtype=np.int64)
    send = np.zeros((phases, G), dtype=np.int64)
    recv = np.zeros((phases, G), dtype=np.int64)
    split = np.zeros(E, dtype=np.int64)
    _check("moe_ep_phase_plan", lib.moe_ep_phase_plan(G, g, E, k, float(capacity_factor), _np_ptr(cnt),
                                                      _np_ptr(Sv), phases, _np_ptr(send), _np_ptr(recv),
                                                      _np_ptr(split)))
    return send, recv, split


def moe_ep_experts(h, recvbuf, stream=None) -> None:
    _check("moe_ep_experts", lib.moe_ep_experts(h, _ptr(recvbuf), _stream(stream)))


def moe_ep_combine(h, sendbuf, y, stream=None) -> None:
    _check("moe_ep_combine", lib.moe_ep_combine(h, _ptr(sendbuf), _ptr(y), _stream(stream)))


def moe_ep_aux_loss(h):
    a, z = ctypes.c_float(), ctypes.c_float()
    _check("moe_ep_aux_loss", lib.moe_ep_aux_loss(h, ctypes.byref(a), ctypes.byref(z)))
    return a.value, z.value


def moe_ep_get_routing(h, eidx=None, gate=None, slot=None, spos=None, logits=None, stream=None) -> None:
    _check("moe_ep_get_routing", lib.moe_ep_get_routing(h, _ptr(eidx), _ptr(gate), _ptr(slot), _ptr(spos),
                                                        _ptr(logits), _stream(stream)))


def moe_ep_check(h, stream=None) -> None:
    _check("moe_ep_check", lib.moe_ep_check(h, _stream(stream)))

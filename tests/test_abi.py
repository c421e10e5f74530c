"""The C-ABI library loads and exports what include/moe.h declares (CPU only).

No test here makes a CUDA call: argument validation that rejects a call before
any device work is checked with fake (never dereferenced) pointers.
"""
import ctypes
import os
import re
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "moe.h")


def _declared():
    txt = open(HEADER).read()
    return sorted(set(re.findall(r"^MOE_API\s+[\w\s\*]+?\b(moe_\w+)\s*\(", txt, flags=re.M)))


@pytest.fixture(scope="module")
def L():
    from gshard_top_gating_b200 import _lib
    return _lib


def test_header_declares_the_boundary():
    names = _declared()
    for want in ("moe_create", "moe_forward", "moe_aux_loss", "moe_destroy", "moe_get_logits",
                 "moe_get_routing", "moe_route_from_logits", "moe_status_string",
                 "moe_forward_host", "moe_enable_backward", "moe_backward",
                 "moe_kernels_per_backward", "moe_set_backward_flags",
                 "moe_get_backward_stage_times"):
        assert want in names


def test_library_exports_every_declared_symbol(L):
    out = subprocess.run(["nm", "-D", "--defined-only", L.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = {ln.split()[-1] for ln in out.splitlines() if " T " in ln}
    missing = [n for n in _declared() if n not in exported]
    assert not missing, missing
    for n in _declared():
        assert hasattr(L.lib, n)


def test_status_strings(L):
    assert L.moe_status_string(0) == "ok"
    assert "timed out" in L.moe_status_string(L.MOE_ERR_TIMEOUT)
    assert L.moe_stage_name(3) == "ffn1" and L.moe_stage_name(99) == "?"


FAKE = 1 << 20   # 16-byte aligned, never dereferenced: validation fails first


@pytest.mark.parametrize("args,status", [
    ((64, 64, 64, 8, 9, 1.0), 1),          # k > E
    ((64, 64, 64, 8, 0, 1.0), 1),          # k = 0
    ((64, 64, 64, 8, 2, 0.0), 1),          # cf = 0
    ((64, 64, 64, 8, 2, float("nan")), 1),
    ((64, 64, 64, 8, 2, float("inf")), 1),
    ((0, 64, 64, 8, 2, 1.0), 1),           # S_max = 0
    ((64, 96, 64, 8, 2, 1.0), 1),          # M not a multiple of 64
    ((64, 64, 100, 8, 2, 1.0), 1),         # H not a multiple of 64
    ((64, 64, 64, 300, 2, 1.0), 2),        # E > 256 unsupported
    ((64, 64, 64, 16, 9, 1.0), 2),         # k > 8 unsupported
    ((1 << 30, 64, 64, 256, 8, 8.0), 2),   # E * expert rows >= 2^31: 32-bit row indices
    ((1 << 30, 64, 64, 8, 4, 0.001), 2),   # S_max * k >= 2^31
    ((1 << 31, 64, 64, 8, 2, 1.0), 2),     # S_max > 2^30
])
def test_create_rejects_bad_arguments_before_device_work(L, args, status):
    h = ctypes.c_void_p(123)
    st = L.lib.moe_create(ctypes.byref(h), *args, 1, FAKE, None, FAKE, FAKE)
    assert st == status
    assert h.value is None


def test_create_rejects_null_and_misaligned_pointers(L):
    h = ctypes.c_void_p()
    assert L.lib.moe_create(ctypes.byref(h), 64, 64, 64, 8, 2, 1.0, 1, None, None, FAKE, FAKE) == 1
    assert L.lib.moe_create(ctypes.byref(h), 64, 64, 64, 8, 2, 1.0, 1, FAKE, None, FAKE + 8, FAKE) == 1
    assert L.lib.moe_create(None, 64, 64, 64, 8, 2, 1.0, 1, FAKE, None, FAKE, FAKE) == 1


def test_null_handle_calls_are_rejected(L):
    assert L.lib.moe_forward(None, 1, FAKE, FAKE, None) == 1
    assert L.lib.moe_destroy(None) == 0
    assert L.lib.moe_kernels_per_forward(None, 10) == 0
    f = ctypes.c_float()
    assert L.lib.moe_aux_loss(None, ctypes.byref(f), ctypes.byref(f), None) == 1
    assert L.lib.moe_enable_backward(None) == 1
    assert L.lib.moe_backward(None, 1, FAKE, FAKE, 0.0, 0.0, FAKE, FAKE, None, FAKE, FAKE, None) == 1
    assert L.lib.moe_kernels_per_backward(None, 10) == 0
    assert L.lib.moe_set_backward_flags(None, 0) == 1

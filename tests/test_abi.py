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


C_PROGRAM = r"""
#include <stdio.h>
#include <string.h>
#include "moe.h"

/* A C11 caller of the boundary: host-only entry points, no device work. */
int main(void) {
    /* G = 2 ranks, k = 1, E = 2: rank 0 chose experts {0,0,1}, rank 1 {1,1,1} */
    const int64_t counts[4] = {2, 1, 0, 3}, S[2] = {3, 3};
    int64_t C = 0, send[2], recv[2], send2[4], recv2[4], split[2];
    if (moe_ep_stats_len(2, 1) != 1 * 2 + 2 + 2) return 1;
    if (moe_ep_plan(2, 0, 2, 1, 1.0, counts, S, &C, send, recv, NULL, NULL) != MOE_OK) return 2;
    if (C != 3 || send[0] != 2 || send[1] != 1 || recv[0] != 2 || recv[1] != 0) return 3;
    if (moe_ep_phase_plan(2, 0, 2, 1, 1.0, counts, S, 2, send2, recv2, split) != MOE_OK) return 4;
    if (send2[0] + send2[2] != send[0] || send2[1] + send2[3] != send[1]) return 5;
    if (moe_ep_plan(2, 0, 2, 1, 1.0, counts, S, NULL, NULL, NULL, NULL, NULL) != MOE_OK) return 6;
    if (moe_create(NULL, 1, 64, 64, 2, 1, 1.0, MOE_BF16, NULL, NULL, NULL, NULL) != MOE_ERR_INVALID_ARG)
        return 7;
    if (strlen(moe_status_string(MOE_ERR_TIMEOUT)) == 0) return 8;
    printf("ok %lld\n", (long long)C);
    return 0;
}
"""


def test_header_is_c11_and_links_from_c(tmp_path):
    """A plain C11 program compiles against include/moe.h with warnings as errors, links
    against the library and runs its host-only entry points."""
    import shutil
    from gshard_top_gating_b200 import _lib
    cc = shutil.which("gcc") or shutil.which("cc")
    if cc is None:
        pytest.skip("no C compiler")
    src = tmp_path / "caller.c"
    src.write_text(C_PROGRAM)
    exe = tmp_path / "caller"
    libdir = os.path.dirname(_lib.LIB_PATH)
    libname = os.path.basename(_lib.LIB_PATH)
    subprocess.run([cc, "-std=c11", "-Wall", "-Wextra", "-Werror", "-pedantic", "-I", os.path.join(ROOT, "include"),
                    str(src), "-o", str(exe), os.path.join(libdir, libname), f"-Wl,-rpath,{libdir}"],
                   check=True, capture_output=True)
    out = subprocess.run([str(exe)], capture_output=True, text=True)
    assert out.returncode == 0, (out.returncode, out.stderr)
    assert out.stdout.strip() == "ok 3"

"""CPU checks of the C ABI: libpoetx.so loads, exports every function that
include/poetx.h declares, and rejects bad arguments before touching a device.
No compute call is made here (this host has no GPU)."""
import ctypes
import os
import re
import subprocess
import sys

import pytest

import orthogonal_equivalence_b200 as px
from orthogonal_equivalence_b200 import build as pbuild

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    pbuild.build()
    return px.lib()


def header_functions():
    text = open(os.path.join(ROOT, "include", "poetx.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(poetx_[A-Za-z0-9_]+)\s*\(", text)))


def test_header_declares_expected_calls():
    names = header_functions()
    for want in ["poetx_cnp_build", "poetx_cnp_backward", "poetx_forward", "poetx_backward", "poetx_merge",
                 "poetx_frame_import", "poetx_frame_export"]:
        assert want in names


def test_library_exports_every_declared_symbol(lib):
    out = subprocess.run(["nm", "-D", "--defined-only", px.LIB_PATH], capture_output=True, text=True).stdout
    exported = set(re.findall(r"\bT (poetx_\w+)", out))
    missing = [n for n in header_functions() if n not in exported]
    assert not missing, missing
    for n in header_functions():
        assert hasattr(lib, n)
    assert set(px.SIGNATURES) == set(header_functions())


def test_status_strings(lib):
    for code, name in px.STATUS_NAMES.items():
        assert px.poetx_status_string(code).startswith(name)
    assert "unknown" in px.poetx_status_string(99)
    assert px.poetx_version() == 10100


def _layer(m=512, n=256, b=64, dtype=px.POETX_BF16, ptr=4096, fold=0):
    return px.poetx_layer(m, n, b, dtype, ptr, ptr, ptr, ptr, ptr, ptr, ptr, fold)


def test_layer_struct_matches_the_header():
    # the fold field follows the seven pointers: offset 72, struct size 80 (LP64)
    assert px.poetx_layer.fold.offset == 16 + 7 * 8
    assert ctypes.sizeof(px.poetx_layer) == 80


def test_workspace_sizes_are_host_arithmetic(lib):
    L = _layer()
    T = 300
    assert px.poetx_forward_workspace_bytes(L, T) >= 2 * T * (2 * 512 + 2 * 256)
    assert px.poetx_backward_workspace_bytes(L, T) >= 2 * T * (2 * 512 + 512)
    assert px.poetx_merge_workspace_bytes(L) >= 2 * 4 * 512 * 256
    assert px.poetx_cnp_workspace_bytes(8, 64, px.POETX_BF16) >= 7 * 4 * 8 * 64 * 64
    assert px.poetx_check_perm_workspace_bytes(100) >= 400
    # invalid layers size to 0
    assert px.poetx_forward_workspace_bytes(_layer(b=48), T) == 0   # bf16 needs b % 64 == 0
    assert px.poetx_forward_workspace_bytes(_layer(m=500), T) == 0  # b must divide m
    assert px.poetx_forward_workspace_bytes(_layer(dtype=7), T) == 0
    # row and token limits (one staged row of at most 200 KB; 32-bit row counts)
    assert px.poetx_forward_workspace_bytes(_layer(m=51200, n=102400, b=256), T) > 0
    assert px.poetx_forward_workspace_bytes(_layer(m=51456, b=256), T) == 0
    assert px.poetx_forward_workspace_bytes(_layer(n=102656, b=256), T) == 0
    assert px.poetx_forward_workspace_bytes(_layer(n=51264, b=64, dtype=px.POETX_FP32), T) == 0
    assert px.poetx_forward_workspace_bytes(_layer(), 2 ** 31) == 0


def test_validation_before_any_launch(lib):
    # every rejected call returns its status without touching a device
    assert lib.poetx_forward(None, 10, 4096, 4096, None, None, 4096, 1 << 30, None) == 1          # E_ARG
    L = _layer(m=500)
    assert lib.poetx_forward(ctypes.byref(L), 10, 4096, 4096, None, None, 4096, 1 << 30, None) == 2  # E_SHAPE
    L = _layer(dtype=5)
    assert lib.poetx_forward(ctypes.byref(L), 10, 4096, 4096, None, None, 4096, 1 << 30, None) == 3  # E_DTYPE
    L = _layer(ptr=4100)
    assert lib.poetx_forward(ctypes.byref(L), 10, 4096, 4096, None, None, 4096, 1 << 30, None) == 4  # E_ALIGN
    L = _layer(fold=8)
    assert lib.poetx_forward(ctypes.byref(L), 10, 4096, 4096, None, None, 4096, 1 << 30, None) == 1  # fold bits
    assert px.poetx_forward_workspace_bytes(L, 10) == 0
    L = _layer()
    assert lib.poetx_forward(ctypes.byref(L), -1, 4096, 4096, None, None, 4096, 1 << 30, None) == 1  # T < 0
    assert lib.poetx_forward(ctypes.byref(L), 2 ** 31, 4096, 4096, None, None, 4096, 1 << 30, None) == 2  # T big
    Lw = _layer(m=51456, b=256)
    assert lib.poetx_forward(ctypes.byref(Lw), 10, 4096, 4096, None, None, 4096, 1 << 30, None) == 2  # m wide
    assert lib.poetx_backward_dG(ctypes.byref(L), 2 ** 31, 4096, 4096, None, 4096, None, 4096, 4096, 0, 4096,
                                 1 << 30, None) == 2                                          # T big
    assert lib.poetx_forward(ctypes.byref(L), 10, 4096, 4096, None, None, 4096, 16, None) == 5       # ws small
    assert lib.poetx_forward(ctypes.byref(L), 10, None, 4096, None, None, 4096, 1 << 30, None) == 1  # x NULL
    assert lib.poetx_backward(ctypes.byref(L), 10, 4096, 4100, None, 4096, None, 4096, 4096, 0, 4096, 1 << 30,
                              None) == 4                                                      # y_save unaligned
    # y_save == NULL selects the recomputing backward, which needs a larger workspace
    assert lib.poetx_backward(ctypes.byref(L), 10, 4096, None, None, 4096, None, 4096, 4096, 0, 4096,
                              px.poetx_backward_workspace_bytes(L, 10), None) == 5
    assert px.poetx_backward_recompute_workspace_bytes(L, 10) > px.poetx_backward_workspace_bytes(L, 10)
    assert lib.poetx_backward(ctypes.byref(L), 10, None, 4096, None, 4096, None, 4096, 4096, 0, 4096, 1 << 30,
                              None) == 1                                                      # no x, no xg
    assert lib.poetx_backward_dG(ctypes.byref(L), 10, 4096, 4096, None, 4096, None, None, 4096, 0, 4096,
                                 1 << 30, None) == 1                                          # dGR NULL
    assert lib.poetx_backward_dG(ctypes.byref(L), 10, 4096, 4096, None, 4096, None, 4096, 4104, 0, 4096,
                                 1 << 30, None) == 4                                          # dGP unaligned
    assert lib.poetx_cnp_build(4, 48, 4096, px.POETX_BF16, 4096, 4096, 1 << 30, None) == 2    # b % 64
    assert lib.poetx_cnp_build(4, 64, 4096, 9, 4096, 4096, 1 << 30, None) == 3
    assert lib.poetx_cnp_build(4, 64, 4096, px.POETX_BF16, 4096, 4096, 8, None) == 5
    assert lib.poetx_cnp_backward(4, 1, 4096, 4096, 4096, 0, px.POETX_FP32, 4096, 1 << 30, None) == 2
    # merge output may not overlap the stored weight
    assert lib.poetx_merge(ctypes.byref(L), 4096, 4096, 4096, 4096, 1 << 30, None) == 1
    assert lib.poetx_check_perm(4096, 0, 4096, 4096, 1 << 20, None) == 1
    # failure-path self-test: limit out of range, NULL or misaligned output
    assert lib.poetx_selftest_wait_timeout(0, 4096, None) == 1
    assert lib.poetx_selftest_wait_timeout(1000001, 4096, None) == 1
    assert lib.poetx_selftest_wait_timeout(1000, None, None) == 1
    assert lib.poetx_selftest_wait_timeout(1000, 4100, None) == 4


def test_no_device_call_fails_cleanly(lib):
    # a fully valid call on a host without a GPU reports a CUDA error, not a crash
    import torch
    if torch.cuda.is_available():
        pytest.skip("host has a GPU")
    L = _layer()
    T = 10
    ws = px.poetx_forward_workspace_bytes(L, T)
    assert lib.poetx_forward(ctypes.byref(L), T, 4096, 4096, 4096, None, 4096, ws, None) == 7


def test_debug_build_exports_the_same_symbols(lib):
    # -DPOETX_DEBUG (device-side copy checks) changes no symbol of the ABI
    path = pbuild.build(debug=True)
    out = subprocess.run(["nm", "-D", "--defined-only", path], capture_output=True, text=True).stdout
    exported = set(re.findall(r"\bT (poetx_\w+)", out))
    assert set(header_functions()) <= exported


def test_debug_environment_selects_the_debug_library():
    # POETX_DEBUG=1 makes the package load libpoetx_debug.so; otherwise libpoetx.so
    code = "import orthogonal_equivalence_b200 as px; print(os.path.basename(px.LIB_PATH))"
    for flag, want in (("1", "libpoetx_debug.so"), ("0", "libpoetx.so")):
        env = dict(os.environ, POETX_DEBUG=flag)
        out = subprocess.run([sys.executable, "-c", "import os; " + code], cwd=ROOT, env=env, capture_output=True,
                             text=True).stdout.strip()
        assert out == want, (flag, out)

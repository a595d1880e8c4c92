"""Python binding of libpoetx.so, the B200 (sm_100a) library of the POET-X
orthogonal-equivalence linear layer  z = P^T (W0^T (R^T x))  (POET-X
write-up, zhichai.net, sections 1-3).

The binding only marshals arguments: every step of the layer runs in the
library's CUDA kernels.  PyTorch supplies device memory and streams.  There is
no fallback: if libpoetx.so is missing or the device is not a B200, calls
raise.

Names follow the C ABI in include/poetx.h (poetx_forward, poetx_backward, ...).
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

_HERE = os.path.dirname(os.path.abspath(__file__))
# POETX_DEBUG=1 selects the build with device-side copy checks (build.py debug=True)
LIB_PATH = os.path.join(_HERE, "libpoetx_debug.so" if os.environ.get("POETX_DEBUG") == "1" else "libpoetx.so")

POETX_FP32 = 0
POETX_BF16 = 1
# poetx_layer.fold bits (0 = the input-centric evaluation everywhere)
POETX_FOLD_R = 1
POETX_FOLD_P = 2
POETX_FOLD_WEIGHT_CENTRIC = 4
POETX_FOLD_ALL = 7

STATUS_NAMES = {0: "POETX_OK", 1: "POETX_E_ARG", 2: "POETX_E_SHAPE", 3: "POETX_E_DTYPE", 4: "POETX_E_ALIGN",
                5: "POETX_E_WORKSPACE", 6: "POETX_E_ARCH", 7: "POETX_E_CUDA"}


class PoetxError(RuntimeError):
    def __init__(self, status: int, where: str, text: str):
        super().__init__(f"{where}: {text}")
        self.status = status


class poetx_layer(ctypes.Structure):
    _fields_ = [("m", ctypes.c_int32), ("n", ctypes.c_int32), ("b", ctypes.c_int32), ("dtype", ctypes.c_int32),
                ("W", ctypes.c_void_p), ("permR", ctypes.c_void_p), ("permP", ctypes.c_void_p),
                ("qR", ctypes.c_void_p), ("qP", ctypes.c_void_p), ("GR", ctypes.c_void_p), ("GP", ctypes.c_void_p),
                ("fold", ctypes.c_int32)]


_VP, _I32, _I64, _SZ = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t
_LP = ctypes.POINTER(poetx_layer)

# name -> (restype, argtypes); mirrors include/poetx.h
SIGNATURES = {
    "poetx_status_string": (ctypes.c_char_p, [ctypes.c_int]),
    "poetx_version": (_I32, []),
    "poetx_device_error": (ctypes.c_int, [ctypes.POINTER(ctypes.c_uint32)]),
    "poetx_cnp_workspace_bytes": (_SZ, [_I32, _I32, _I32]),
    "poetx_forward_workspace_bytes": (_SZ, [_LP, _I64]),
    "poetx_backward_workspace_bytes": (_SZ, [_LP, _I64]),
    "poetx_backward_recompute_workspace_bytes": (_SZ, [_LP, _I64]),
    "poetx_merge_workspace_bytes": (_SZ, [_LP]),
    "poetx_check_perm_workspace_bytes": (_SZ, [_I32]),
    "poetx_frame_import": (ctypes.c_int, [_LP, _VP, _VP]),
    "poetx_frame_export": (ctypes.c_int, [_LP, _VP, _VP]),
    "poetx_cnp_build": (ctypes.c_int, [_I32, _I32, _VP, _I32, _VP, _VP, _SZ, _VP]),
    "poetx_cnp_backward": (ctypes.c_int, [_I32, _I32, _VP, _VP, _VP, _I32, _I32, _VP, _SZ, _VP]),
    "poetx_cnp_build_fixed": (ctypes.c_int, [_I32, _I32, _VP, _I32, _VP, _VP]),
    "poetx_layer_cnp_workspace_bytes": (_SZ, [_LP]),
    "poetx_layers_cnp_workspace_bytes": (_SZ, [_I32, _LP]),
    "poetx_layers_cnp_build": (ctypes.c_int, [_I32, _LP, _VP, _SZ, _VP]),
    "poetx_layer_cnp_build": (ctypes.c_int, [_LP, _VP, _SZ, _VP]),
    "poetx_forward": (ctypes.c_int, [_LP, _I64, _VP, _VP, _VP, _VP, _VP, _SZ, _VP]),
    "poetx_backward": (ctypes.c_int, [_LP, _I64, _VP, _VP, _VP, _VP, _VP, _VP, _VP, _I32, _VP, _SZ, _VP]),
    "poetx_backward_dG": (ctypes.c_int, [_LP, _I64, _VP, _VP, _VP, _VP, _VP, _VP, _VP, _I32, _VP, _SZ, _VP]),
    "poetx_merge": (ctypes.c_int, [_LP, _VP, _VP, _VP, _VP, _SZ, _VP]),
    "poetx_check_perm": (ctypes.c_int, [_VP, _I32, _VP, _VP, _SZ, _VP]),
    "poetx_weight_quantize": (ctypes.c_int, [_I32, _I32, _VP, _I32, _VP, _VP, _VP]),
    "poetx_weight_dequantize": (ctypes.c_int, [_I32, _I32, _VP, _VP, _I32, _VP, _VP]),
    "poetx_selftest_wait_timeout": (ctypes.c_int, [ctypes.c_uint32, _VP, _VP]),
    "poetx_adamw_step": (ctypes.c_int, [_I64, _VP, _VP, _VP, _VP, ctypes.c_float, ctypes.c_float, ctypes.c_float,
                                        ctypes.c_float, ctypes.c_float, _I32, _VP]),
    "poetx_profile_stage_count": (_I32, []),
    "poetx_profile_stage_name": (ctypes.c_char_p, [_I32]),
    "poetx_profile_begin": (ctypes.c_int, []),
    "poetx_profile_end": (ctypes.c_int, [ctypes.POINTER(ctypes.c_double), ctypes.POINTER(ctypes.c_int64), _I32]),
    "poetx_profile_records": (_I32, [ctypes.POINTER(ctypes.c_int32), ctypes.POINTER(ctypes.c_float), _I32]),
}

_lib: Optional[ctypes.CDLL] = None


def lib() -> ctypes.CDLL:
    """Load libpoetx.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{os.path.basename(LIB_PATH)} not built ({LIB_PATH}); run "
                               "orthogonal_equivalence_b200/build.py")
        L = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _lib = L
    return _lib


def _ptr(t) -> Optional[int]:
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _stream(stream) -> Optional[int]:
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _check(status: int, where: str) -> None:
    if status != 0:
        raise PoetxError(status, where, lib().poetx_status_string(status).decode())


def make_layer(m: int, n: int, b: int, dtype: int, W, permR, permP, qR, qP, GR, GP, fold: int = 0) -> poetx_layer:
    return poetx_layer(m, n, b, dtype, _ptr(W), _ptr(permR), _ptr(permP), _ptr(qR), _ptr(qP), _ptr(GR), _ptr(GP),
                       fold)


# ---------------------------------------------------------------- C calls, same names
def poetx_version() -> int:
    return lib().poetx_version()


def poetx_status_string(status: int) -> str:
    return lib().poetx_status_string(status).decode()


def poetx_device_error() -> int:
    v = ctypes.c_uint32(0)
    _check(lib().poetx_device_error(ctypes.byref(v)), "poetx_device_error")
    return v.value


def poetx_cnp_workspace_bytes(nblk: int, b: int, dtype: int) -> int:
    return lib().poetx_cnp_workspace_bytes(nblk, b, dtype)


def poetx_forward_workspace_bytes(layer: poetx_layer, T: int) -> int:
    return lib().poetx_forward_workspace_bytes(ctypes.byref(layer), T)


def poetx_backward_workspace_bytes(layer: poetx_layer, T: int) -> int:
    return lib().poetx_backward_workspace_bytes(ctypes.byref(layer), T)


def poetx_backward_recompute_workspace_bytes(layer: poetx_layer, T: int) -> int:
    return lib().poetx_backward_recompute_workspace_bytes(ctypes.byref(layer), T)


def poetx_merge_workspace_bytes(layer: poetx_layer) -> int:
    return lib().poetx_merge_workspace_bytes(ctypes.byref(layer))


def poetx_check_perm_workspace_bytes(length: int) -> int:
    return lib().poetx_check_perm_workspace_bytes(length)


def poetx_frame_import(layer: poetx_layer, W0lin, stream=None) -> None:
    _check(lib().poetx_frame_import(ctypes.byref(layer), _ptr(W0lin), _stream(stream)), "poetx_frame_import")


def poetx_frame_export(layer: poetx_layer, W0lin, stream=None) -> None:
    _check(lib().poetx_frame_export(ctypes.byref(layer), _ptr(W0lin), _stream(stream)), "poetx_frame_export")


def poetx_cnp_build(nblk: int, b: int, q, dtype: int, G, ws, ws_bytes: int, stream=None) -> None:
    _check(lib().poetx_cnp_build(nblk, b, _ptr(q), dtype, _ptr(G), _ptr(ws), ws_bytes, _stream(stream)),
           "poetx_cnp_build")


def poetx_cnp_build_fixed(nblk: int, b: int, q, dtype: int, G, stream=None) -> None:
    """poetx_cnp_build with the library's fixed device scratch (no workspace)."""
    _check(lib().poetx_cnp_build_fixed(nblk, b, _ptr(q), dtype, _ptr(G), _stream(stream)), "poetx_cnp_build_fixed")


def poetx_cnp_backward(nblk: int, b: int, q, dG, dq, accumulate: int, dtype: int, ws, ws_bytes: int,
                       stream=None) -> None:
    _check(lib().poetx_cnp_backward(nblk, b, _ptr(q), _ptr(dG), _ptr(dq), accumulate, dtype, _ptr(ws), ws_bytes,
                                    _stream(stream)), "poetx_cnp_backward")


def poetx_layer_cnp_workspace_bytes(layer: poetx_layer) -> int:
    return lib().poetx_layer_cnp_workspace_bytes(ctypes.byref(layer))


def poetx_layer_cnp_build(layer: poetx_layer, ws, ws_bytes: int, stream=None) -> None:
    _check(lib().poetx_layer_cnp_build(ctypes.byref(layer), _ptr(ws), ws_bytes, _stream(stream)),
           "poetx_layer_cnp_build")


def _layer_array(layers):
    arr = (poetx_layer * len(layers))(*layers)
    return arr


def poetx_layers_cnp_workspace_bytes(layers) -> int:
    return lib().poetx_layers_cnp_workspace_bytes(len(layers), _layer_array(layers))


def poetx_layers_cnp_build(layers, ws, ws_bytes: int, stream=None) -> None:
    _check(lib().poetx_layers_cnp_build(len(layers), _layer_array(layers), _ptr(ws), ws_bytes, _stream(stream)),
           "poetx_layers_cnp_build")


def poetx_forward(layer: poetx_layer, T: int, x, z, y_save, xg_save, ws, ws_bytes: int, stream=None) -> None:
    _check(lib().poetx_forward(ctypes.byref(layer), T, _ptr(x), _ptr(z), _ptr(y_save), _ptr(xg_save), _ptr(ws),
                               ws_bytes, _stream(stream)), "poetx_forward")


def poetx_backward(layer: poetx_layer, T: int, x, y_save, xg_save, dz, dx, dqR, dqP, accumulate: int, ws,
                   ws_bytes: int, stream=None) -> None:
    _check(lib().poetx_backward(ctypes.byref(layer), T, _ptr(x), _ptr(y_save), _ptr(xg_save), _ptr(dz), _ptr(dx),
                                _ptr(dqR), _ptr(dqP), accumulate, _ptr(ws), ws_bytes, _stream(stream)),
           "poetx_backward")


def poetx_backward_dG(layer: poetx_layer, T: int, x, y_save, xg_save, dz, dx, dGR, dGP, accumulate: int, ws,
                      ws_bytes: int, stream=None) -> None:
    _check(lib().poetx_backward_dG(ctypes.byref(layer), T, _ptr(x), _ptr(y_save), _ptr(xg_save), _ptr(dz),
                                   _ptr(dx), _ptr(dGR), _ptr(dGP), accumulate, _ptr(ws), ws_bytes, _stream(stream)),
           "poetx_backward_dG")


def poetx_merge(layer: poetx_layer, new_permR, new_permP, W_out, ws, ws_bytes: int, stream=None) -> None:
    _check(lib().poetx_merge(ctypes.byref(layer), _ptr(new_permR), _ptr(new_permP), _ptr(W_out), _ptr(ws),
                             ws_bytes, _stream(stream)), "poetx_merge")


def poetx_check_perm(perm, length: int, d_ok, ws, ws_bytes: int, stream=None) -> None:
    _check(lib().poetx_check_perm(_ptr(perm), length, _ptr(d_ok), _ptr(ws), ws_bytes, _stream(stream)),
           "poetx_check_perm")


def poetx_weight_quantize(n: int, m: int, W, dtype: int, Wq, scale, stream=None) -> None:
    _check(lib().poetx_weight_quantize(n, m, _ptr(W), dtype, _ptr(Wq), _ptr(scale), _stream(stream)),
           "poetx_weight_quantize")


def poetx_weight_dequantize(n: int, m: int, Wq, scale, dtype: int, W, stream=None) -> None:
    _check(lib().poetx_weight_dequantize(n, m, _ptr(Wq), _ptr(scale), dtype, _ptr(W), _stream(stream)),
           "poetx_weight_dequantize")


def poetx_adamw_step(n: int, q, grad, m1, m2, lr: float, beta1: float, beta2: float, eps: float,
                     weight_decay: float, step: int, stream=None) -> None:
    _check(lib().poetx_adamw_step(n, _ptr(q), _ptr(grad), _ptr(m1), _ptr(m2), lr, beta1, beta2, eps, weight_decay,
                                  step, _stream(stream)), "poetx_adamw_step")


def poetx_selftest_wait_timeout(limit_us: int, d_out, stream=None) -> None:
    """Queue the failure-path self-test: a bounded wait nobody satisfies gives
    up after limit_us and records bit 1 in the device error word; d_out is a
    device int64 tensor of 2 entries ([0] arrived, [1] ns waited)."""
    _check(lib().poetx_selftest_wait_timeout(limit_us, _ptr(d_out), _stream(stream)), "poetx_selftest_wait_timeout")


def poetx_profile_begin() -> None:
    _check(lib().poetx_profile_begin(), "poetx_profile_begin")


def poetx_profile_end() -> dict:
    """{stage name: (device ms, launches)} since poetx_profile_begin()."""
    n = lib().poetx_profile_stage_count()
    ms = (ctypes.c_double * n)()
    cnt = (ctypes.c_int64 * n)()
    _check(lib().poetx_profile_end(ms, cnt, n), "poetx_profile_end")
    return {lib().poetx_profile_stage_name(i).decode(): (ms[i], cnt[i]) for i in range(n)}


def poetx_profile_records() -> list:
    """[(stage name, device ms)] per launch of the last profiling session."""
    n = lib().poetx_profile_records(None, None, 0)
    st = (ctypes.c_int32 * max(n, 1))()
    ms = (ctypes.c_float * max(n, 1))()
    lib().poetx_profile_records(st, ms, n)
    names = [lib().poetx_profile_stage_name(i).decode() for i in range(lib().poetx_profile_stage_count())]
    return [(names[st[i]], ms[i]) for i in range(n)]


from .layer import LayerGroup, PoetxLinear, Saved  # noqa: E402,F401

"""Shared helpers of the GPU parity tests: move the seeded inputs of
poetx_inputs to the device, run the library, bring results back as float64,
and the tolerances the parity bar states.

Tolerances (the stated bar): fp32 layers, normwise max error
max|gpu - oracle| / max|oracle| <= 1e-5; bf16-in / fp32-accumulate layers,
relative Frobenius error ||gpu - oracle||_F / ||oracle||_F <= 1e-2.
"""
from __future__ import annotations

import numpy as np
import torch

import orthogonal_equivalence_b200 as px
import poetx_inputs as pi

TOL_FP32 = 1e-5
TOL_BF16 = 1e-2


def dev(arr: np.ndarray, dtype: str) -> torch.Tensor:
    """Storage array from poetx_inputs -> device tensor of the same bits."""
    if dtype == "bf16":
        return torch.from_numpy(np.ascontiguousarray(arr).view(np.int16)).view(torch.bfloat16).cuda()
    return torch.from_numpy(np.ascontiguousarray(arr)).cuda()


def host64(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy().astype(np.float64)


def bits(t: torch.Tensor) -> np.ndarray:
    """Raw storage bits of a device tensor (for bit-exact comparisons)."""
    if t.dtype == torch.bfloat16:
        return t.detach().cpu().view(torch.int16).numpy().view(np.uint16)
    return t.detach().cpu().numpy().view(np.uint32)


def poetx_dtype(dtype: str) -> int:
    return px.POETX_BF16 if dtype == "bf16" else px.POETX_FP32


def make_layer(inp: pi.LayerInputs, fold: int = 0) -> px.PoetxLinear:
    L = px.PoetxLinear(inp.m, inp.n, inp.b, poetx_dtype(inp.dtype), fold=fold)
    L.load(dev(inp.W0lin, inp.dtype), torch.from_numpy(inp.permR).cuda(), torch.from_numpy(inp.permP).cuda(),
           torch.from_numpy(inp.qR).cuda(), torch.from_numpy(inp.qP).cuda())
    return L


def rel_fro(a: np.ndarray, o: np.ndarray) -> float:
    return float(np.linalg.norm(a - o) / np.linalg.norm(o))


def normwise_max(a: np.ndarray, o: np.ndarray) -> float:
    return float(np.abs(a - o).max() / np.abs(o).max())


def check(a: np.ndarray, o: np.ndarray, dtype: str, what: str) -> float:
    assert a.shape == o.shape, (what, a.shape, o.shape)
    assert np.all(np.isfinite(a)), what
    if dtype == "fp32":
        e = normwise_max(a, o)
        assert e <= TOL_FP32, f"{what}: normwise max error {e:.3e} > {TOL_FP32}"
    else:
        e = rel_fro(a, o)
        assert e <= TOL_BF16, f"{what}: relative Frobenius error {e:.3e} > {TOL_BF16}"
    return e

"""Seeded synthetic inputs for the POET-X layer (shared by the tests, the oracle
checks and the benchmark).

This module only draws random numbers and rounds them to the storage dtype; it
holds none of the layer's arithmetic.  Both the oracle and the CUDA path receive
exactly the values produced here.

Workload shapes follow the Llama-style linears the POET-X pages train
(POET-X blog, section "Llama-3B @ 60B tokens" and the single-H100 Llama-8B /
Llama-13B sections): block size b = 256 or 512, sequence length 2048.

Recipe (per tensor, numpy PCG64, drawn in float64):
  x  ~ N(0, 1)            [T][m]   stored bf16 (RNE) or fp32
  W0 ~ N(0, 0.02^2)       [n][m]   nn.Linear layout (out x in), stored like x
  qR, qP ~ N(0, sigma_q^2) packed upper triangles, fp32
  dz ~ N(0, 1)            [T][n]   stored like x
  permR, permP            seeded permutations (int32)
Seed of a tensor = 1000*cfg_id + 10*layer + tensor_id, with tensor ids
x=1, W0=2, qR=3, qP=4, dz=5, permR=6, permP=7; a permutation resampled at the
k-th merge adds 100*k.
"""
from __future__ import annotations

import dataclasses
from typing import Tuple

import numpy as np

TENSOR_IDS = {"x": 1, "W0": 2, "qR": 3, "qP": 4, "dz": 5, "permR": 6, "permP": 7}


@dataclasses.dataclass(frozen=True)
class Config:
    """One synthetic workload: a list of linears (name, m, n) sharing b, T."""
    cfg_id: int
    name: str
    layers: Tuple[Tuple[str, int, int], ...]
    b: int
    T: int
    dtype: str          # "fp32" or "bf16": storage type of x, W0, dz, G, z, dx
    sigma_q: float
    description: str
    # x_from[i]: the linear whose input linear i reads (a decoder block's q, k,
    # v read one normalised hidden state, gate and up another); () = each its own
    x_from: Tuple[int, ...] = ()

    def x_source(self, layer: int) -> int:
        return self.x_from[layer] if self.x_from else layer

    def flops_per_step(self) -> float:
        """Algorithmic flops of one forward+backward step (no merge).

        Per token: 2mn (W0 forward) + 2mn (dU = dY W~^T; W0 is frozen, no dW0)
        + 6b(m+n) (block-diagonal R and P forward, dY/dXg, dG_P/dG_R).
        Per step: 12 b^2 (m+n) for the CNP build (4b^3 per block) and its
        backward (8b^3 per block).
        """
        tot = 0.0
        for _, m, n in self.layers:
            tot += self.T * (4.0 * m * n + 6.0 * self.b * (m + n))
            tot += 12.0 * self.b * self.b * (m + n)
        return tot

    def gemm_flops_per_step(self) -> float:
        return sum(self.T * 4.0 * m * n for _, m, n in self.layers)


CONFIGS = {
    "tiny": Config(1, "tiny", (("tiny", 512, 512),), 64, 256, "fp32", 0.01,
                   "Tiny layer, fp32 throughout: m=n=512, b=64, T=256"),
    "attn3b": Config(2, "attn3b", (("attn", 3072, 3072),), 256, 16384, "bf16", 0.01,
                     "Llama-3B attention projection: m=n=3072, b=256, T=16384"),
    "up8b": Config(3, "up8b", (("up", 4096, 14336),), 256, 8192, "bf16", 0.01,
                   "Llama-8B MLP up-projection: m=4096 -> n=14336, b=256, T=8192"),
    "down13b": Config(4, "down13b", (("down", 13824, 5120),), 512, 4096, "bf16", 0.005,
                      "Llama-13B MLP down-projection: m=13824 -> n=5120, b=512, T=4096"),
    "block8b": Config(5, "block8b",
                      (("q", 4096, 4096), ("k", 4096, 1024), ("v", 4096, 1024),
                       ("o", 4096, 4096), ("gate", 4096, 14336), ("up", 4096, 14336),
                       ("down", 14336, 4096)),
                      256, 16384, "bf16", 0.01,
                      "Llama-8B decoder block, 7 linears in sequence, b=256, T=16384; q/k/v read one input, "
                      "gate/up another", x_from=(0, 0, 0, 3, 4, 4, 6)),
}


# Triangle scale of the parity cases that must see every term of the
# Cayley-Neumann block: sigma per b with ||Q||_2 ~= 0.75-0.8 (the spectral
# norm of a b x b skew Gaussian is about 2 sigma sqrt(b)).  At the workloads'
# own scale (0.01, or 0.005 at b = 512) the Q^4 term moves G by less than the
# bf16 bar; here leaving out Q^4, or 2Q^3, moves G, dq and the layer's
# outputs by at least 3x the bar (a CPU test checks this on the oracle).
PARITY_SIGMA = {64: 0.05, 128: 0.035, 256: 0.025, 512: 0.018}


def seed_of(cfg: Config, layer: int, tensor: str, merge_index: int = 0) -> int:
    return 1000 * cfg.cfg_id + 10 * layer + TENSOR_IDS[tensor] + 100 * merge_index


def bf16_bits(a: np.ndarray) -> np.ndarray:
    """Round to bfloat16 (float64 -> float32 by the IEEE default, then
    round-to-nearest-even on the low 16 bits); returns uint16 bit patterns."""
    u = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32)
    lsb = (u >> np.uint32(16)) & np.uint32(1)
    r = (u + np.uint32(0x7FFF) + lsb) >> np.uint32(16)
    return r.astype(np.uint16)


def bf16_to_f64(bits: np.ndarray) -> np.ndarray:
    return (bits.astype(np.uint32) << np.uint32(16)).view(np.float32).astype(np.float64)


def _normal(seed: int, shape, sigma: float) -> np.ndarray:
    return np.random.Generator(np.random.PCG64(seed)).standard_normal(shape) * sigma


def _store(a64: np.ndarray, dtype: str):
    """Return (storage array, exact float64 value of what is stored)."""
    if dtype == "bf16":
        bits = bf16_bits(a64)
        return bits, bf16_to_f64(bits)
    f = a64.astype(np.float32)
    return f, f.astype(np.float64)


def permutation(seed: int, length: int) -> np.ndarray:
    return np.random.Generator(np.random.PCG64(seed)).permutation(length).astype(np.int32)


def tri_len(b: int) -> int:
    return b * (b - 1) // 2


@dataclasses.dataclass
class LayerInputs:
    m: int
    n: int
    b: int
    T: int
    dtype: str
    x: np.ndarray        # storage [T][m] (uint16 bf16 bits or float32)
    x64: np.ndarray
    W0lin: np.ndarray    # storage [n][m] (nn.Linear layout)
    W0lin64: np.ndarray
    qR: np.ndarray       # float32 [m/b][b(b-1)/2]
    qP: np.ndarray       # float32 [n/b][b(b-1)/2]
    dz: np.ndarray       # storage [T][n]
    dz64: np.ndarray
    permR: np.ndarray    # int32 [m]
    permP: np.ndarray    # int32 [n]


def layer_inputs(cfg: Config, layer: int = 0, T: int | None = None, m: int | None = None,
                 n: int | None = None, b: int | None = None, sigma_q: float | None = None,
                 zero_q: bool = False) -> LayerInputs:
    """Draw one layer's inputs.  Overrides (T, m, n, b) give reduced shapes of
    the same recipe for parity tests; the full configuration is the default."""
    if m is None or n is None:
        _, m0, n0 = cfg.layers[layer]
        m = m0 if m is None else m
        n = n0 if n is None else n
    b = cfg.b if b is None else b
    T = cfg.T if T is None else T
    sq = cfg.sigma_q if sigma_q is None else sigma_q
    if m % b or n % b:
        raise ValueError("b must divide m and n")
    x, x64 = _store(_normal(seed_of(cfg, layer, "x"), (T, m), 1.0), cfg.dtype)
    W, W64 = _store(_normal(seed_of(cfg, layer, "W0"), (n, m), 0.02), cfg.dtype)
    dz, dz64 = _store(_normal(seed_of(cfg, layer, "dz"), (T, n), 1.0), cfg.dtype)
    if zero_q:
        qR = np.zeros((m // b, tri_len(b)), np.float32)
        qP = np.zeros((n // b, tri_len(b)), np.float32)
    else:
        qR = _normal(seed_of(cfg, layer, "qR"), (m // b, tri_len(b)), sq).astype(np.float32)
        qP = _normal(seed_of(cfg, layer, "qP"), (n // b, tri_len(b)), sq).astype(np.float32)
    return LayerInputs(m, n, b, T, cfg.dtype, x, x64, W, W64, qR, qP, dz, dz64,
                       permutation(seed_of(cfg, layer, "permR"), m),
                       permutation(seed_of(cfg, layer, "permP"), n))


def merge_perms(cfg: Config, layer: int, merge_index: int, m: int, n: int):
    """Permutations drawn at the merge_index-th merge (merge_index >= 1)."""
    return (permutation(seed_of(cfg, layer, "permR", merge_index), m),
            permutation(seed_of(cfg, layer, "permP", merge_index), n))


def random_token_rows(seed: int, T: int, count: int) -> np.ndarray:
    """Sorted sample of distinct token rows (always includes the last row, so a
    ragged tail tile is covered)."""
    g = np.random.Generator(np.random.PCG64(seed))
    rows = g.choice(T, size=min(count, T), replace=False)
    rows[-1] = T - 1
    return np.unique(rows).astype(np.int64)

"""POET-X layer oracle: a plain, slow, float64 CPU statement of what the layer
computes.

TEST INFRASTRUCTURE ONLY.  Nothing on the product path may import or call
this module: only the tests, the smoke check of the package entry point and
the CPU-baseline leg of the benchmark use it.  It shares no code with the CUDA
library (no kernels, no helpers, no tables); the two meet only at the seeded
inputs of `poetx_inputs`.

Source: the POET-X write-up (zhichai.net, "POET-X ... 单卡H100训练130亿参数模型"),
sections 1 (input-centric formulation), 2 (block-stochastic R) and 3
(Cayley-Neumann parameterisation, packed upper triangle).

Notation (pages): W0 is m x n and frozen; one token x in R^m maps to
    z = P^T (W0^T (R^T x))                      (section 1, input-centric)
which equals (R W0 P)^T x                      (section 1, weight-centric),
    R = Psi^T Diag(G_1..G_{m/b}) Psi           (section 2)
and P is built the same way on the n side with its own Psi_P.  Every block is
    G = (I + Q)(I + Q + Q^2 + Q^3),  Q = -Q^T   (section 3)
and Q is stored as its b(b-1)/2 strict upper triangle (section 3).

Readings taken where the pages are silent (each also listed in the design
notes of the repository):
  * packing order: row-major over i < j, k(i,j) = i(b-1) - i(i-1)/2 + (j-i-1),
    Q[i,j] = +q[k], Q[j,i] = -q[k];
  * permutation convention: perm[i'] is the natural index at position i' of the
    Psi frame, i.e. (Psi v)[i'] = v[perm[i']]  (Psi[i', perm[i']] = 1);
  * the Neumann series has exactly the three terms written on the page;
  * b divides m and n (all workloads do);
  * the gradient with respect to the packed triangle is dL/dq_k =
    dL/dQ[i,j] - dL/dQ[j,i] (Q[j,i] = -q_k);
  * merge: W0 <- R W0 P in natural coordinates, then the weight is re-expressed
    in the frame of the new permutations; Q is reset to 0 (G = I).

Batched row form used throughout: X is T x m (one token per row), Z = X R W0 P
is T x n.  All arithmetic is float64; numpy's matmul is the only library
primitive used.

Parity: every function here is pinned by tests against closed forms,
invariants, brute force, finite differences or a library routine (the AdamW
step against torch.optim.AdamW); none is "parity unpinned".
"""
from __future__ import annotations

import numpy as np

# --------------------------------------------------------------------------
# Section 3: packed skew-symmetric triangle and the Cayley-Neumann block.
# --------------------------------------------------------------------------


def triangle_positions(b: int):
    """(rows, cols) of the strict upper triangle in packing order (row-major,
    i < j).  Entry k of a packed vector sits at Q[rows[k], cols[k]]."""
    rows, cols = [], []
    for i in range(b):
        for j in range(i + 1, b):
            rows.append(i)
            cols.append(j)
    return np.array(rows, dtype=np.int64), np.array(cols, dtype=np.int64)


def unpack_skew(q: np.ndarray, b: int) -> np.ndarray:
    """Packed triangle (b(b-1)/2,) -> skew-symmetric Q (b x b)."""
    q = np.asarray(q, dtype=np.float64)
    if q.shape != (b * (b - 1) // 2,):
        raise ValueError("packed triangle has the wrong length")
    rows, cols = triangle_positions(b)
    Q = np.zeros((b, b), dtype=np.float64)
    Q[rows, cols] = q
    Q[cols, rows] = -q
    return Q


def pack_skew(Q: np.ndarray) -> np.ndarray:
    """Skew-symmetric Q -> packed strict upper triangle."""
    rows, cols = triangle_positions(Q.shape[0])
    return np.asarray(Q, dtype=np.float64)[rows, cols].copy()


def cayley_neumann(Q: np.ndarray) -> np.ndarray:
    """G = (I + Q)(I + Q + Q^2 + Q^3), multiplied out as written."""
    b = Q.shape[0]
    I = np.eye(b)
    Q2 = Q @ Q
    Q3 = Q2 @ Q
    return (I + Q) @ (I + Q + Q2 + Q3)


def cnp_blocks(q: np.ndarray, b: int) -> np.ndarray:
    """Packed triangles [nblk][b(b-1)/2] -> G blocks [nblk][b][b]."""
    q = np.asarray(q, dtype=np.float64)
    return np.stack([cayley_neumann(unpack_skew(q[j], b)) for j in range(q.shape[0])])


def cnp_backward_block(q: np.ndarray, b: int, dG: np.ndarray) -> np.ndarray:
    """Gradient of a loss L with respect to the packed triangle, given
    dG = dL/dG, by the chain rule through G = F N with F = I + Q and
    N = I + Q + Q^2 + Q^3:
        dF = dG N^T,   dN = F^T dG,
        dQ = dF + dN + d(Q^2) + d(Q^3),
        d(Q^2) = dN Q^T + Q^T dN,
        d(Q^3) = dN (Q^2)^T + Q^T dN Q^T + (Q^2)^T dN,
    then dq_k = dQ[i,j] - dQ[j,i] for the k-th packed pair (i < j)."""
    Q = unpack_skew(q, b)
    dG = np.asarray(dG, dtype=np.float64)
    I = np.eye(b)
    Q2 = Q @ Q
    Q3 = Q2 @ Q
    F = I + Q
    N = I + Q + Q2 + Q3
    dF = dG @ N.T
    dN = F.T @ dG
    dQ = dF + dN
    dQ = dQ + dN @ Q.T + Q.T @ dN
    dQ = dQ + dN @ Q2.T + Q.T @ dN @ Q.T + Q2.T @ dN
    rows, cols = triangle_positions(b)
    return dQ[rows, cols] - dQ[cols, rows]


def cnp_backward(q: np.ndarray, b: int, dG: np.ndarray) -> np.ndarray:
    """Blockwise cnp_backward_block over [nblk] blocks."""
    return np.stack([cnp_backward_block(q[j], b, dG[j]) for j in range(q.shape[0])])


# --------------------------------------------------------------------------
# Section 2: block-stochastic orthogonal matrices R = Psi^T Diag(G) Psi.
# --------------------------------------------------------------------------


def permutation_matrix(perm: np.ndarray) -> np.ndarray:
    """Psi with Psi[i', perm[i']] = 1, so (Psi v)[i'] = v[perm[i']]."""
    d = len(perm)
    Psi = np.zeros((d, d), dtype=np.float64)
    Psi[np.arange(d), np.asarray(perm, dtype=np.int64)] = 1.0
    return Psi


def block_diagonal(G: np.ndarray) -> np.ndarray:
    nblk, b, _ = G.shape
    D = np.zeros((nblk * b, nblk * b), dtype=np.float64)
    for j in range(nblk):
        D[j * b:(j + 1) * b, j * b:(j + 1) * b] = G[j]
    return D


def orthogonal_dense(perm: np.ndarray, G: np.ndarray) -> np.ndarray:
    """Dense R = Psi^T Diag(G_1..G_k) Psi."""
    Psi = permutation_matrix(perm)
    return Psi.T @ block_diagonal(G) @ Psi


def apply_rows(X: np.ndarray, perm: np.ndarray, G: np.ndarray) -> np.ndarray:
    """Rows of X times R = Psi^T Diag(G) Psi without forming R: gather the
    columns into the Psi frame (X Psi^T), multiply each b-column block by its
    G_j, and scatter the columns back (times Psi)."""
    nblk, b, _ = G.shape
    perm = np.asarray(perm, dtype=np.int64)
    Xg = X[:, perm]
    U = np.empty_like(Xg)
    for j in range(nblk):
        U[:, j * b:(j + 1) * b] = Xg[:, j * b:(j + 1) * b] @ G[j]
    out = np.empty_like(U)
    out[:, perm] = U
    return out


def apply_rows_transposed(X: np.ndarray, perm: np.ndarray, G: np.ndarray) -> np.ndarray:
    """Rows of X times R^T = Psi^T Diag(G^T) Psi (the backward of apply_rows)."""
    return apply_rows(X, perm, np.transpose(G, (0, 2, 1)))


# --------------------------------------------------------------------------
# Section 1: the layer, input-centric and weight-centric.
# --------------------------------------------------------------------------


def forward(X, W0, permR, GR, permP, GP):
    """Input-centric z = P^T (W0^T (R^T x)) for every row x of X (T x m).
    W0 is the natural m x n weight.  Returns Z (T x n)."""
    X = np.asarray(X, dtype=np.float64)
    A = apply_rows(X, permR, GR)          # rows: (R^T x)^T = x^T R
    Y = A @ W0                            # rows: (W0^T R^T x)^T
    return apply_rows(Y, permP, GP)       # rows: (P^T W0^T R^T x)^T


def forward_weight_centric(X, W0, permR, GR, permP, GP):
    """Weight-centric: form W = R W0 P densely, then Z = X W."""
    R = orthogonal_dense(permR, GR)
    P = orthogonal_dense(permP, GP)
    return np.asarray(X, dtype=np.float64) @ (R @ W0 @ P)


def backward(X, W0, permR, GR, permP, GP, dZ):
    """Chain rule of `forward` for L = <dZ, Z>.  Returns (dX, dGR, dGP) with
    dGR[j] = dL/dG_Rj and dGP[j] = dL/dG_Pj (b x b each).

    forward:  Xg = X Psi_R^T;  U_j = Xg_j G_Rj;  A = U Psi_R;  Y = A W0;
              Yg = Y Psi_P^T;  V_j = Yg_j G_Pj;  Z = V Psi_P.
    backward: dV = dZ Psi_P^T; dYg_j = dV_j G_Pj^T; dG_Pj = Yg_j^T dV_j;
              dY = dYg Psi_P;  dA = dY W0^T;       dU = dA Psi_R^T;
              dXg_j = dU_j G_Rj^T; dG_Rj = Xg_j^T dU_j; dX = dXg Psi_R."""
    X = np.asarray(X, dtype=np.float64)
    dZ = np.asarray(dZ, dtype=np.float64)
    permR = np.asarray(permR, dtype=np.int64)
    permP = np.asarray(permP, dtype=np.int64)
    nR, b, _ = GR.shape
    nP = GP.shape[0]
    Xg = X[:, permR]
    U = np.empty_like(Xg)
    for j in range(nR):
        U[:, j * b:(j + 1) * b] = Xg[:, j * b:(j + 1) * b] @ GR[j]
    A = np.empty_like(U)
    A[:, permR] = U
    Y = A @ W0
    Yg = Y[:, permP]

    dV = dZ[:, permP]
    dYg = np.empty_like(dV)
    dGP = np.empty((nP, b, b))
    for j in range(nP):
        s = slice(j * b, (j + 1) * b)
        dYg[:, s] = dV[:, s] @ GP[j].T
        dGP[j] = Yg[:, s].T @ dV[:, s]
    dY = np.empty_like(dYg)
    dY[:, permP] = dYg
    dA = dY @ W0.T
    dU = dA[:, permR]
    dXg = np.empty_like(dU)
    dGR = np.empty((nR, b, b))
    for j in range(nR):
        s = slice(j * b, (j + 1) * b)
        dXg[:, s] = dU[:, s] @ GR[j].T
        dGR[j] = Xg[:, s].T @ dU[:, s]
    dX = np.empty_like(dXg)
    dX[:, permR] = dXg
    return dX, dGR, dGP


def layer_backward(X, W0, permR, qR, permP, qP, b, dZ):
    """dX, dqR, dqP of L = <dZ, Z> with G built from the packed triangles."""
    GR = cnp_blocks(qR, b)
    GP = cnp_blocks(qP, b)
    dX, dGR, dGP = backward(X, W0, permR, GR, permP, GP, dZ)
    return dX, cnp_backward(qR, b, dGR), cnp_backward(qP, b, dGP)


def grad_G_blocks(X, W0, permR, GR, permP, GP, dZ, side: str, blocks):
    """dL/dG for the listed blocks j of one side over all rows of X, computing
    only the columns those blocks need (used to check full-size runs block by
    block).  Same chain rule as `backward`, restricted to the listed blocks;
    returns a list of b x b arrays in the order of `blocks`."""
    X = np.asarray(X, dtype=np.float64)
    dZ = np.asarray(dZ, dtype=np.float64)
    permR = np.asarray(permR, dtype=np.int64)
    permP = np.asarray(permP, dtype=np.int64)
    b = GR.shape[1]
    out = []
    if side == "P":
        A = apply_rows(X, permR, GR)
        for j in blocks:
            cols = permP[j * b:(j + 1) * b]
            Yg_j = A @ W0[:, cols]
            dV_j = dZ[:, cols]
            out.append(Yg_j.T @ dV_j)
        return out
    if side != "R":
        raise ValueError("side must be 'R' or 'P'")
    dY = apply_rows_transposed(dZ, permP, GP)      # rows: dZ P^T
    for j in blocks:
        cols = permR[j * b:(j + 1) * b]
        dU_j = dY @ W0[cols, :].T
        Xg_j = X[:, cols]
        out.append(Xg_j.T @ dU_j)
    return out


# --------------------------------------------------------------------------
# Merge (POETModel.merge_if_needed in the pages' API snippet): W0 <- R W0 P.
# --------------------------------------------------------------------------


def merge(W0, permR, GR, permP, GP):
    """W0_new = R W0 P in natural coordinates (m x n), applied blockwise: the
    rows of W0 are rotated by R (R W0 = (W0^T R^T)^T) and its columns by P."""
    W0 = np.asarray(W0, dtype=np.float64)
    RW = apply_rows_transposed(W0.T, permR, GR).T   # (W0^T R^T)^T = R W0
    return apply_rows(RW, permP, GP)                # (R W0) P


def merge_dense(W0, permR, GR, permP, GP):
    """Same as `merge` with R and P formed densely (tiny shapes only)."""
    return orthogonal_dense(permR, GR) @ np.asarray(W0, dtype=np.float64) @ orthogonal_dense(permP, GP)


# --------------------------------------------------------------------------
# Frame of the stored weight: W~ = Psi_R W0 Psi_P^T, kept as [n][m] rows
# (the nn.Linear layout), W~[j'][i'] = W0[permR[i']][permP[j']].
# --------------------------------------------------------------------------


def to_frame(W0lin: np.ndarray, permR, permP) -> np.ndarray:
    """nn.Linear weight W0^T ([n][m], natural) -> stored Psi-frame weight."""
    return np.asarray(W0lin)[np.asarray(permP, dtype=np.int64)][:, np.asarray(permR, dtype=np.int64)]


def from_frame(Wf: np.ndarray, permR, permP) -> np.ndarray:
    """Stored Psi-frame weight -> nn.Linear weight W0^T ([n][m], natural)."""
    out = np.empty_like(Wf)
    out[np.ix_(np.asarray(permP, dtype=np.int64), np.asarray(permR, dtype=np.int64))] = Wf
    return out


# --------------------------------------------------------------------------
# POET-XQ (section "POET-XQ"): the base weight stored quantized, dequantized
# at run time.  Reading: int8, symmetric, one scale per row of the stored
# [n][m] weight; the scale and the codes are decided in float32 arithmetic
# (scale = max|row| / 127, code = round-half-even(w / scale) clamped to
# [-127, 127]); w = code * scale in float32, rounded once to the weight dtype.
# --------------------------------------------------------------------------


def quantize_rows(W: np.ndarray):
    """[n][m] weight values -> (int8 codes [n][m], float32 scales [n])."""
    W32 = np.asarray(W, dtype=np.float32)
    amax = np.max(np.abs(W32), axis=1)
    scale = (amax / np.float32(127.0)).astype(np.float32)
    codes = np.zeros(W32.shape, dtype=np.int8)
    nz = scale > 0
    q = np.rint(W32[nz] / scale[nz, None]).astype(np.float32)
    codes[nz] = np.clip(q, -127, 127).astype(np.int8)
    return codes, scale


def dequantize_rows(codes: np.ndarray, scale: np.ndarray) -> np.ndarray:
    """code * scale as the float32 product (float32 array)."""
    return codes.astype(np.float32) * np.asarray(scale, dtype=np.float32)[:, None]


def round_to_bf16(a: np.ndarray) -> np.ndarray:
    """float32 values rounded to bfloat16 (round to nearest even), returned as
    float64 values."""
    u = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32)
    r = ((u + np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1))) >> np.uint32(16)) << np.uint32(16)
    return r.astype(np.uint32).view(np.float32).astype(np.float64)


# --------------------------------------------------------------------------
# Optimizer step on the packed triangles (get_poet_optimizer in the API
# snippet is not described; reading: AdamW with decoupled weight decay).
# --------------------------------------------------------------------------


def adamw_step(q, g, m, v, lr, beta1, beta2, eps, weight_decay, step):
    """One AdamW update in float64; returns (q, m, v)."""
    q = np.asarray(q, dtype=np.float64)
    g = np.asarray(g, dtype=np.float64)
    m = beta1 * np.asarray(m, dtype=np.float64) + (1.0 - beta1) * g
    v = beta2 * np.asarray(v, dtype=np.float64) + (1.0 - beta2) * g * g
    m_hat = m / (1.0 - beta1 ** step)
    v_hat = v / (1.0 - beta2 ** step)
    q = q * (1.0 - lr * weight_decay) - lr * m_hat / (np.sqrt(v_hat) + eps)
    return q, m, v

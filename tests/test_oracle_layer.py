"""Pins of the oracle's layer, backward and merge against what the POET-X
write-up (zhichai.net, sections 1-2 and the API snippet's merge) and the
mathematics fix: Q = 0 reduces to a plain linear, input-centric equals
weight-centric, index-form brute force, the dense closed form of dx, central
finite differences, and function preservation of the merge."""
import numpy as np
import pytest

import oracle
import poetx_inputs as pi


def _case(m, n, b, T, seed, scale=0.05):
    g = np.random.Generator(np.random.PCG64(seed))
    X = g.standard_normal((T, m))
    W0 = g.standard_normal((m, n)) * 0.3
    dZ = g.standard_normal((T, n))
    qR = g.standard_normal((m // b, b * (b - 1) // 2)) * scale
    qP = g.standard_normal((n // b, b * (b - 1) // 2)) * scale
    permR = g.permutation(m).astype(np.int32)
    permP = g.permutation(n).astype(np.int32)
    return X, W0, dZ, qR, qP, permR, permP


def test_zero_q_is_plain_linear():
    X, W0, _, qR, qP, permR, permP = _case(12, 18, 6, 5, 1)
    GR = oracle.cnp_blocks(np.zeros_like(qR), 6)
    GP = oracle.cnp_blocks(np.zeros_like(qP), 6)
    Z = oracle.forward(X, W0, permR, GR, permP, GP)
    np.testing.assert_allclose(Z, X @ W0, rtol=1e-14, atol=1e-14)


@pytest.mark.parametrize("m,n,b,T", [(12, 18, 6, 5), (64, 48, 16, 7), (32, 32, 32, 3)])
def test_input_centric_equals_weight_centric(m, n, b, T):
    X, W0, _, qR, qP, permR, permP = _case(m, n, b, T, m + n)
    GR = oracle.cnp_blocks(qR, b)
    GP = oracle.cnp_blocks(qP, b)
    Zi = oracle.forward(X, W0, permR, GR, permP, GP)
    Zw = oracle.forward_weight_centric(X, W0, permR, GR, permP, GP)
    np.testing.assert_allclose(Zi, Zw, rtol=0, atol=1e-13 * np.abs(Zw).max())


def test_brute_force_index_form():
    # R = Psi^T D Psi with Psi[i', perm[i']] = 1 gives, entry by entry,
    # R[i][k] = D[pinv[i]][pinv[k]] (pinv the inverse permutation).  Build R,
    # P that way with scalar loops and evaluate z_t[j] = sum x[i] R W0 P.
    m, n, b, T = 4, 6, 2, 3
    X, W0, _, qR, qP, permR, permP = _case(m, n, b, T, 9, scale=0.4)
    GR = oracle.cnp_blocks(qR, b)
    GP = oracle.cnp_blocks(qP, b)

    def dense_from_index(perm, G):
        d = len(perm)
        pinv = [0] * d
        for ip, p in enumerate(perm):
            pinv[p] = ip
        M = [[0.0] * d for _ in range(d)]
        for i in range(d):
            for k in range(d):
                a, c = pinv[i], pinv[k]
                if a // b == c // b:
                    M[i][k] = G[a // b][a % b][c % b]
        return M

    R = dense_from_index(permR, GR)
    P = dense_from_index(permP, GP)
    Z = np.zeros((T, n))
    for t in range(T):
        for j in range(n):
            s = 0.0
            for i in range(m):
                for a in range(m):
                    for c in range(n):
                        s += X[t][i] * R[i][a] * W0[a][c] * P[c][j]
            Z[t][j] = s
    np.testing.assert_allclose(oracle.forward(X, W0, permR, GR, permP, GP), Z, rtol=0, atol=1e-12)


def test_dx_dense_closed_form():
    m, n, b, T = 24, 36, 6, 4
    X, W0, dZ, qR, qP, permR, permP = _case(m, n, b, T, 21)
    GR = oracle.cnp_blocks(qR, b)
    GP = oracle.cnp_blocks(qP, b)
    dX, _, _ = oracle.backward(X, W0, permR, GR, permP, GP, dZ)
    W = oracle.orthogonal_dense(permR, GR) @ W0 @ oracle.orthogonal_dense(permP, GP)
    np.testing.assert_allclose(dX, dZ @ W.T, rtol=0, atol=1e-13 * np.abs(dX).max())


def test_layer_gradients_match_central_differences():
    m, n, b, T = 8, 12, 4, 3
    X, W0, dZ, qR, qP, permR, permP = _case(m, n, b, T, 33, scale=0.2)
    dX, dqR, dqP = oracle.layer_backward(X, W0, permR, qR, permP, qP, b, dZ)

    def loss(X_, qR_, qP_):
        GR = oracle.cnp_blocks(qR_, b)
        GP = oracle.cnp_blocks(qP_, b)
        return np.sum(dZ * oracle.forward(X_, W0, permR, GR, permP, GP))

    h = 1e-5
    for arr, grad, name in [(qR, dqR, "qR"), (qP, dqP, "qP"), (X, dX, "X")]:
        fd = np.zeros_like(arr)
        it = np.nditer(arr, flags=["multi_index"])
        for _ in it:
            idx = it.multi_index
            ap = arr.copy()
            am = arr.copy()
            ap[idx] += h
            am[idx] -= h
            args_p = {"X": X, "qR": qR, "qP": qP}
            args_m = dict(args_p)
            args_p[name] = ap
            args_m[name] = am
            fd[idx] = (loss(args_p["X"], args_p["qR"], args_p["qP"]) -
                       loss(args_m["X"], args_m["qR"], args_m["qP"])) / (2 * h)
        np.testing.assert_allclose(grad, fd, rtol=0, atol=1e-7 * max(1.0, np.abs(fd).max()),
                                   err_msg=name)


def test_grad_G_blocks_match_full_backward():
    m, n, b, T = 24, 36, 6, 5
    X, W0, dZ, qR, qP, permR, permP = _case(m, n, b, T, 44)
    GR = oracle.cnp_blocks(qR, b)
    GP = oracle.cnp_blocks(qP, b)
    _, dGR, dGP = oracle.backward(X, W0, permR, GR, permP, GP, dZ)
    got = oracle.grad_G_blocks(X, W0, permR, GR, permP, GP, dZ, "R", range(m // b))
    for j in range(m // b):
        np.testing.assert_allclose(got[j], dGR[j], rtol=0, atol=1e-12 * np.abs(dGR).max())
    got = oracle.grad_G_blocks(X, W0, permR, GR, permP, GP, dZ, "P", [5, 0, 3])
    for g, j in zip(got, [5, 0, 3]):
        np.testing.assert_allclose(g, dGP[j], rtol=0, atol=1e-12 * np.abs(dGP).max())


def test_dq_linear_in_token_rows():
    # L = <dZ, Z> is a sum over tokens, so dq over all rows equals the sum of
    # dq over a split of the rows (used to check full-size runs by parts).
    m, n, b, T = 16, 24, 8, 9
    X, W0, dZ, qR, qP, permR, permP = _case(m, n, b, T, 55)
    _, dqR, dqP = oracle.layer_backward(X, W0, permR, qR, permP, qP, b, dZ)
    _, r1, p1 = oracle.layer_backward(X[:4], W0, permR, qR, permP, qP, b, dZ[:4])
    _, r2, p2 = oracle.layer_backward(X[4:], W0, permR, qR, permP, qP, b, dZ[4:])
    np.testing.assert_allclose(dqR, r1 + r2, rtol=0, atol=1e-12)
    np.testing.assert_allclose(dqP, p1 + p2, rtol=0, atol=1e-12)


def test_block_orthogonality_defect():
    m, b = 48, 8
    _, _, _, qR, _, permR, _ = _case(m, m, b, 1, 66, scale=0.1)
    GR = oracle.cnp_blocks(qR, b)
    R = oracle.orthogonal_dense(permR, GR)
    defect = max(np.abs(G.T @ G - np.eye(b)).max() for G in GR)
    np.testing.assert_allclose(np.abs(R.T @ R - np.eye(m)).max(), defect, rtol=1e-12)


def test_merge_matches_dense_and_preserves_function():
    m, n, b, T = 24, 36, 6, 5
    X, W0, _, qR, qP, permR, permP = _case(m, n, b, T, 77)
    GR = oracle.cnp_blocks(qR, b)
    GP = oracle.cnp_blocks(qP, b)
    Wm = oracle.merge(W0, permR, GR, permP, GP)
    np.testing.assert_allclose(Wm, oracle.merge_dense(W0, permR, GR, permP, GP), rtol=0, atol=1e-14)
    # after the merge Q = 0 (G = I) and new permutations are drawn: same z
    g = np.random.Generator(np.random.PCG64(78))
    nR, nP = g.permutation(m), g.permutation(n)
    I_R = oracle.cnp_blocks(np.zeros_like(qR), b)
    I_P = oracle.cnp_blocks(np.zeros_like(qP), b)
    Z0 = oracle.forward(X, W0, permR, GR, permP, GP)
    Z1 = oracle.forward(X, Wm, nR, I_R, nP, I_P)
    np.testing.assert_allclose(Z1, Z0, rtol=0, atol=1e-13 * np.abs(Z0).max())


def test_merge_with_zero_q_is_exact():
    m, n, b = 24, 36, 6
    _, W0, _, qR, qP, permR, permP = _case(m, n, b, 1, 88)
    I_R = oracle.cnp_blocks(np.zeros_like(qR), b)
    I_P = oracle.cnp_blocks(np.zeros_like(qP), b)
    assert np.array_equal(oracle.merge(W0, permR, I_R, permP, I_P), W0)


def test_frame_roundtrip_and_definition():
    m, n = 20, 12
    g = np.random.Generator(np.random.PCG64(5))
    W0lin = g.standard_normal((n, m))
    permR = g.permutation(m)
    permP = g.permutation(n)
    Wf = oracle.to_frame(W0lin, permR, permP)
    assert np.array_equal(oracle.from_frame(Wf, permR, permP), W0lin)
    # definition: W~ = Psi_R W0 Psi_P^T with W0 = W0lin^T, stored transposed
    want = (oracle.permutation_matrix(permR) @ W0lin.T @ oracle.permutation_matrix(permP).T).T
    assert np.array_equal(Wf, want)


def test_inputs_bf16_rounding_is_rne():
    # the shared input generator rounds to bfloat16 by round-to-nearest-even
    # bf16 keeps 7 fraction bits: 1 + 2^-8 is a tie (to even: 1), 1 + 3*2^-8 a tie
    # (to even: 1 + 2^-6), 1 + 2^-8 + 2^-20 is above the midpoint (1 + 2^-7)
    v = np.array([1.0, 1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, -2.5, 1.0 + 2 ** -8 + 2 ** -20])
    back = pi.bf16_to_f64(pi.bf16_bits(v))
    np.testing.assert_array_equal(back, [1.0, 1.0, 1.0 + 2 ** -6, -2.5, 1.0 + 2 ** -7])

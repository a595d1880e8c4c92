"""Pins of the oracle's Cayley-Neumann block and packed triangle against facts
fixed by the POET-X write-up (zhichai.net, section 3) and by the mathematics:
hand-worked fixtures, closed forms, exact Cayley, finite differences."""
import os

import numpy as np
import pytest

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _read_golden(name):
    rows = []
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                rows.append([float(v) for v in line.split()])
    return rows


def _rand_skew(b, scale, seed):
    g = np.random.Generator(np.random.PCG64(seed))
    q = g.standard_normal(b * (b - 1) // 2) * scale
    return q, oracle.unpack_skew(q, b)


def test_packing_order_matches_hand_fixture():
    rows = _read_golden("packing_b4.txt")
    q = np.array(rows[0])
    Q_hand = np.array(rows[1:5])
    assert np.array_equal(oracle.unpack_skew(q, 4), Q_hand)
    assert np.array_equal(oracle.pack_skew(Q_hand), q)


@pytest.mark.parametrize("b", [2, 3, 7, 64])
def test_pack_unpack_roundtrip_exact_and_skew(b):
    q, Q = _rand_skew(b, 1.0, 11 + b)
    assert np.array_equal(oracle.pack_skew(Q), q)
    assert np.array_equal(Q + Q.T, np.zeros((b, b)))
    assert np.array_equal(np.diag(Q), np.zeros(b))


@pytest.mark.parametrize("b", [2, 5, 64, 256])
def test_zero_q_gives_identity_exactly(b):
    G = oracle.cayley_neumann(np.zeros((b, b)))
    assert np.array_equal(G, np.eye(b))


def test_b2_hand_fixture():
    rows = _read_golden("cnp_b2.txt")
    q = rows[0][0]
    G_hand = np.array(rows[1:3])
    G = oracle.cayley_neumann(oracle.unpack_skew(np.array([q]), 2))
    np.testing.assert_allclose(G, G_hand, rtol=0, atol=1e-15)


@pytest.mark.parametrize("q", [0.0, 1e-3, 0.2, -0.7])
def test_b2_closed_form(q):
    G = oracle.cayley_neumann(oracle.unpack_skew(np.array([q]), 2))
    c = 1.0 - q * q
    want = c * np.array([[c, 2 * q], [-2 * q, c]])
    np.testing.assert_allclose(G, want, rtol=0, atol=1e-15)


def test_b3_rodrigues_closed_form():
    # A 3x3 skew matrix is a cross product: Q v = w x v with
    # w = (-Q[1,2], Q[0,2], -Q[0,1]); then Q^2 = w w^T - |w|^2 I and
    # Q^3 = -|w|^2 Q, so G = I + (2 - 2s) Q + (2 - s) Q^2 with s = |w|^2.
    for seed in range(5):
        g = np.random.Generator(np.random.PCG64(100 + seed))
        a, bb, c = g.standard_normal(3) * 0.4
        Q = oracle.unpack_skew(np.array([a, bb, c]), 3)
        w = np.array([-c, bb, -a])
        s = w @ w
        Q2 = np.outer(w, w) - s * np.eye(3)
        want = np.eye(3) + (2 - 2 * s) * Q + (2 - s) * Q2
        np.testing.assert_allclose(oracle.cayley_neumann(Q), want, rtol=0, atol=1e-14)


@pytest.mark.parametrize("b", [2, 8, 64])
def test_orthogonality_defect_closed_form(b):
    # G = C (I - Q^4) with C = (I+Q)(I-Q)^-1 the exact Cayley transform, all
    # factors commute, so G^T G - I = Q^8 - 2 Q^4 exactly.
    q, Q = _rand_skew(b, 0.3 / np.sqrt(b), 7 * b)
    G = oracle.cayley_neumann(Q)
    Q4 = np.linalg.matrix_power(Q, 4)
    want = Q4 @ Q4 - 2 * Q4
    np.testing.assert_allclose(G.T @ G - np.eye(b), want, rtol=0, atol=1e-15)


@pytest.mark.parametrize("b", [4, 32])
def test_truncation_against_exact_cayley(b):
    # Exact Cayley C = (I+Q)(I-Q)^-1 by a library solve; G - C = -C Q^4, so the
    # gap shrinks like |Q|^4 (log-log slope 4).
    _, Q0 = _rand_skew(b, 1.0, 3 * b)
    Q0 = Q0 / np.linalg.norm(Q0, 2)
    gaps, scales = [], []
    for t in [0.2, 0.1, 0.05, 0.025]:
        Q = t * Q0
        I = np.eye(b)
        C = np.linalg.solve((I - Q).T, (I + Q).T).T
        G = oracle.cayley_neumann(Q)
        np.testing.assert_allclose(G - C, -C @ np.linalg.matrix_power(Q, 4), rtol=0, atol=1e-14)
        gaps.append(np.linalg.norm(G - C))
        scales.append(t)
    slopes = np.diff(np.log(gaps)) / np.diff(np.log(scales))
    assert np.all(np.abs(slopes - 4.0) < 0.05), slopes


def test_symmetric_and_skew_parts():
    # G = I + 2Q + 2Q^2 + 2Q^3 + Q^4: the even powers are symmetric, the odd
    # ones skew, so sym(G) = I + 2S + S^2 and skew(G) = 2Q + 2QS with S = Q^2.
    b = 16
    _, Q = _rand_skew(b, 0.1, 5)
    S = Q @ Q
    G = oracle.cayley_neumann(Q)
    np.testing.assert_allclose((G + G.T) / 2, np.eye(b) + 2 * S + S @ S, rtol=0, atol=1e-15)
    np.testing.assert_allclose((G - G.T) / 2, 2 * Q + 2 * Q @ S, rtol=0, atol=1e-15)


@pytest.mark.parametrize("b", [2, 5, 9])
def test_cnp_backward_matches_central_differences(b):
    g = np.random.Generator(np.random.PCG64(40 + b))
    q = g.standard_normal(b * (b - 1) // 2) * 0.3
    dG = g.standard_normal((b, b))
    dq = oracle.cnp_backward_block(q, b, dG)
    h = 1e-5
    fd = np.empty_like(q)
    for k in range(len(q)):
        e = np.zeros_like(q)
        e[k] = h
        Lp = np.sum(dG * oracle.cayley_neumann(oracle.unpack_skew(q + e, b)))
        Lm = np.sum(dG * oracle.cayley_neumann(oracle.unpack_skew(q - e, b)))
        fd[k] = (Lp - Lm) / (2 * h)
    np.testing.assert_allclose(dq, fd, rtol=0, atol=1e-8 * max(1.0, np.abs(fd).max()))


def test_cnp_blocks_stack():
    b = 6
    g = np.random.Generator(np.random.PCG64(3))
    q = g.standard_normal((4, b * (b - 1) // 2)) * 0.1
    G = oracle.cnp_blocks(q, b)
    for j in range(4):
        assert np.array_equal(G[j], oracle.cayley_neumann(oracle.unpack_skew(q[j], b)))

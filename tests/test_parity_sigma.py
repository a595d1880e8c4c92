"""The bf16 parity cases run at a triangle scale (poetx_inputs.PARITY_SIGMA)
where every term of the Cayley-Neumann block G = (I+Q)(I+Q+Q^2+Q^3) =
I + 2Q + 2Q^2 + 2Q^3 + Q^4 (POET-X write-up, section 3) is visible through the
relative Frobenius bar of 1e-2.  Proof on the CPU: a mutant of the oracle with
the Q^4 term left out, and one with the 2Q^3 term left out, misses the bar by
at least 3x on G, on dq, and on a small layer's z, dx, dqR and dqP.  The
mutants are planted here, in test code, never in the oracle itself; with no
term left out the mutant machinery reproduces the oracle, which shows that a
miss comes from the dropped term alone."""
import numpy as np
import pytest

import oracle
import poetx_inputs as pi

BAR = 1e-2
MARGIN = 3.0


def _powers(Q):
    Q2 = Q @ Q
    Q3 = Q2 @ Q
    return Q2, Q3, Q3 @ Q


def _coeffs(drop):
    """Coefficients of Q^3 and Q^4 in G after leaving one term out."""
    return (0.0 if drop == "q3" else 2.0), (0.0 if drop == "q4" else 1.0)


def mutant_G(Q, drop=None):
    c3, c4 = _coeffs(drop)
    Q2, Q3, Q4 = _powers(Q)
    return np.eye(Q.shape[0]) + 2 * Q + 2 * Q2 + c3 * Q3 + c4 * Q4


def mutant_dq(q, b, dG, drop=None):
    """dL/dq for G = I + 2Q + 2Q^2 + c3 Q^3 + c4 Q^4, term by term:
    d<dG, Q^k> / dQ = sum_{a+c=k-1} (Q^T)^a dG (Q^T)^c."""
    c3, c4 = _coeffs(drop)
    Q = oracle.unpack_skew(q, b)
    Qt = Q.T
    Q2t = Qt @ Qt
    Q3t = Q2t @ Qt
    dQ = (2 * dG + 2 * (dG @ Qt + Qt @ dG) + c3 * (dG @ Q2t + Qt @ dG @ Qt + Q2t @ dG)
          + c4 * (dG @ Q3t + Qt @ dG @ Q2t + Q2t @ dG @ Qt + Q3t @ dG))
    rows, cols = oracle.triangle_positions(b)
    return dQ[rows, cols] - dQ[cols, rows]


def _rel(a, o):
    return float(np.linalg.norm(a - o) / np.linalg.norm(o))


@pytest.mark.parametrize("b", sorted(pi.PARITY_SIGMA))
def test_cnp_mutants_miss_the_bar(b):
    sigma = pi.PARITY_SIGMA[b]
    g = np.random.Generator(np.random.PCG64(31 + b))
    q = g.standard_normal(b * (b - 1) // 2) * sigma
    dG = g.standard_normal((b, b))
    Q = oracle.unpack_skew(q, b)
    G = oracle.cayley_neumann(Q)
    dq = oracle.cnp_backward_block(q, b, dG)
    # the mutant machinery with nothing left out is the oracle
    assert _rel(mutant_G(Q), G) < 1e-13
    assert _rel(mutant_dq(q, b, dG), dq) < 1e-12
    for drop in ("q4", "q3"):
        eG, edq = _rel(mutant_G(Q, drop), G), _rel(mutant_dq(q, b, dG, drop), dq)
        assert eG >= MARGIN * BAR, f"b={b} sigma={sigma}: G without {drop} moves by only {eG:.4f}"
        assert edq >= MARGIN * BAR, f"b={b} sigma={sigma}: dq without {drop} moves by only {edq:.4f}"


# one small layer per b, the shapes of the GPU layer cases at PARITY_SIGMA
LAYERS = [("block8b", 192, 320, 64, 40), ("attn3b", 256, 384, 128, 40), ("attn3b", 512, 512, 256, 40),
          ("down13b", 1024, 1536, 512, 24)]


def _layer(inp, drop):
    W0 = inp.W0lin64.T
    GR = np.stack([mutant_G(oracle.unpack_skew(q, inp.b), drop) for q in inp.qR.astype(np.float64)])
    GP = np.stack([mutant_G(oracle.unpack_skew(q, inp.b), drop) for q in inp.qP.astype(np.float64)])
    z = oracle.forward(inp.x64, W0, inp.permR, GR, inp.permP, GP)
    dx, dGR, dGP = oracle.backward(inp.x64, W0, inp.permR, GR, inp.permP, GP, inp.dz64)
    dqR = np.stack([mutant_dq(q, inp.b, d, drop) for q, d in zip(inp.qR.astype(np.float64), dGR)])
    dqP = np.stack([mutant_dq(q, inp.b, d, drop) for q, d in zip(inp.qP.astype(np.float64), dGP)])
    return z, dx, dqR, dqP


@pytest.mark.parametrize("case", LAYERS, ids=lambda c: f"b{c[3]}")
def test_layer_mutants_miss_the_bar(case):
    name, m, n, b, T = case
    inp = pi.layer_inputs(pi.CONFIGS[name], 0, T=T, m=m, n=n, b=b, sigma_q=pi.PARITY_SIGMA[b])
    W0 = inp.W0lin64.T
    want_z = oracle.forward(inp.x64, W0, inp.permR, oracle.cnp_blocks(inp.qR, b), inp.permP,
                            oracle.cnp_blocks(inp.qP, b))
    want = (want_z,) + oracle.layer_backward(inp.x64, W0, inp.permR, inp.qR, inp.permP, inp.qP, b, inp.dz64)
    full = _layer(inp, None)
    for a, o in zip(full, want):
        assert _rel(a, o) < 1e-12
    for drop in ("q4", "q3"):
        for what, a, o in zip(("z", "dx", "dqR", "dqP"), _layer(inp, drop), want):
            e = _rel(a, o)
            assert e >= MARGIN * BAR, f"b={b}: {what} without {drop} moves by only {e:.4f}"

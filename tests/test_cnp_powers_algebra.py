"""CPU check of the order-4 Cayley-Neumann evaluation the CUDA path uses, in
float64 against the oracle's definition (no GPU).

With S = Q^2 and T = S^2, the map of order 4 is
    B = (I + Q)(I + Q + Q^2 + Q^3 + Q^4) = Q C + D0,
    C = 2I + 2S + T,  D0 = I + 2S + 2T,
three matrix products (S, T, Q C) instead of four by Horner's rule.  Its
gradient needs only the antisymmetric part of dL/dQ, because theta enters Q
as Q[a,c] = theta = -Q[c,a]; S, T and C are symmetric, so only the symmetric
parts of dL/dS and dL/dT matter:
    QG = Q G,  GC = G C,
    dT_s = sym(2G - QG)              (sym(X) = (X + X^T) / 2)
    W = dT_s S,  dS_s = sym(2G - 2QG) + W + W^T,
    Y = dS_s Q,  D = G C - 2Y,  dtheta[a,c] = D[a,c] - D[c,a],
four products instead of Horner's eight.  The kernels evaluate exactly these
steps (operands rounded to the storage type)."""
import numpy as np
import pytest

from oracle import poet_oracle as O


def _powers_forward(Q):
    eye = np.eye(Q.shape[0])
    S = Q @ Q
    T = S @ S
    C = 2 * eye + 2 * S + T
    D0 = eye + 2 * S + 2 * T
    return Q @ C + D0, S, C


def _powers_grad(Q, S, C, G):
    sym2 = lambda X: X + X.T  # noqa: E731  (twice the symmetric part)
    QG, GC = Q @ G, G @ C
    dTs = sym2(G) - 0.5 * sym2(QG)
    W = dTs @ S
    dSs = sym2(G) - sym2(QG) + W + W.T
    Y = dSs @ Q
    D = GC - 2 * Y
    r, c = np.triu_indices(Q.shape[0], 1)
    return D[r, c] - D[c, r]


@pytest.mark.parametrize("size,scale", [(2, 0.7), (7, 0.3), (40, 0.05), (96, 0.2)])
def test_order4_powers_match_oracle(size, scale):
    rng = np.random.default_rng(size)
    theta = rng.standard_normal(O.n_skew(size)) * scale
    Q = O.unpack_skew(theta, size)
    B, S, C = _powers_forward(Q)
    ref = O.cayley_neumann_block(Q, 4)
    assert np.abs(B - ref).max() <= 1e-12 * max(1.0, np.abs(ref).max())
    G = rng.standard_normal((size, size))
    got = _powers_grad(Q, S, C, G)
    expect = O.theta_grad_block(G, theta, size, 4)
    assert np.abs(got - expect).max() <= 1e-12 * max(1.0, np.abs(expect).max())

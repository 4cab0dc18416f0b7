"""CPU check of the order-4 Cayley-Neumann evaluation the CUDA path uses, in
float64 against the oracle's definition (no GPU).

With S = Q^2 and T = S^2, the map of order 4 is
    B = (I + Q)(I + Q + Q^2 + Q^3 + Q^4) = Q C + D0,
    C = 2I + 2S + T,  D0 = I + 2S + 2T,
which the kernels form as three products whose epilogues add the rest:
    S = Q Q,  C = S S + 2S + 2I,  B = (Q + 2I) C - 2S - 3I
(three products instead of four by Horner's rule).  Its gradient needs only
the antisymmetric part of dL/dQ, because theta enters Q as Q[a,c] = theta =
-Q[c,a]; S, T and C are symmetric, so only the symmetric parts of dL/dS and
dL/dT matter:
    dT_s = sym(2G - QG)                 (sym(X) = (X + X^T) / 2)
    W = dT_s S,  dS_s = sym(2G - 2QG) + W + W^T,
    D = G C - 2 dS_s Q,  dtheta[a,c] = D[a,c] - D[c,a],
which the kernels form as four products with the sums in their epilogues:
    U = G - Q G,  G C,  dT_s = sym(G + U),  V = dT_s S + U,
    dS_s = V + V^T,  D = G C - 2 dS_s Q.
Both are checked here step by step (operands rounded to the storage type on
the GPU), and the textbook form beside them."""
import numpy as np
import pytest

from oracle import poet_oracle as O


def _powers_forward(Q):
    """The textbook split: B = Q C + D0."""
    eye = np.eye(Q.shape[0])
    S = Q @ Q
    T = S @ S
    C = 2 * eye + 2 * S + T
    D0 = eye + 2 * S + 2 * T
    return Q @ C + D0, S, C


def _kernel_forward(Q):
    """The products and epilogue sums the kernels take."""
    eye = np.eye(Q.shape[0])
    Q2 = Q + 2 * eye                    # written by the unpack
    S = Q @ Q
    C = S @ S + 2 * S + 2 * eye         # epilogue: addend S (beta 2), diagonal 2
    B = Q2 @ C - 2 * S - 3 * eye        # epilogue: addend S (beta -2), diagonal -3
    return B, S, C


def _powers_grad(Q, S, C, G):
    sym2 = lambda X: X + X.T  # noqa: E731  (twice the symmetric part)
    QG, GC = Q @ G, G @ C
    dTs = sym2(G) - 0.5 * sym2(QG)
    W = dTs @ S
    dSs = sym2(G) - sym2(QG) + W + W.T
    D = GC - 2 * (dSs @ Q)
    r, c = np.triu_indices(Q.shape[0], 1)
    return D[r, c] - D[c, r]


def _kernel_grad(Q, S, C, G):
    sym2 = lambda X: X + X.T  # noqa: E731
    U = G - Q @ G                       # product alpha -1, addend G
    GC = G @ C
    dTs = 0.5 * sym2(G) + 0.5 * sym2(U)  # symmetric kernel, c0 = c1 = 1/2
    V = dTs @ S + U                     # product, addend U
    dSs = sym2(V)                       # symmetric kernel, c0 = 1
    D = GC - 2 * (dSs @ Q)              # product alpha -2, addend G C
    r, c = np.triu_indices(Q.shape[0], 1)
    return D[r, c] - D[c, r]


@pytest.mark.parametrize("size,scale", [(2, 0.7), (7, 0.3), (40, 0.05), (96, 0.2)])
def test_order4_powers_match_oracle(size, scale):
    rng = np.random.default_rng(size)
    theta = rng.standard_normal(O.n_skew(size)) * scale
    Q = O.unpack_skew(theta, size)
    ref = O.cayley_neumann_block(Q, 4)
    G = rng.standard_normal((size, size))
    expect = O.theta_grad_block(G, theta, size, 4)
    for fwd, grad in ((_powers_forward, _powers_grad), (_kernel_forward, _kernel_grad)):
        B, S, C = fwd(Q)
        assert np.abs(B - ref).max() <= 1e-12 * max(1.0, np.abs(ref).max())
        got = grad(Q, S, C, G)
        assert np.abs(got - expect).max() <= 1e-12 * max(1.0, np.abs(expect).max())

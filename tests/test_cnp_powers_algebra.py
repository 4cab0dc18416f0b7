"""CPU check of the order-4 Cayley-Neumann evaluation the CUDA path uses, in
float64 against the oracle's definition (no GPU).

With S = Q^2 and T = S^2, the map of order 4 is
    B = (I + Q)(I + Q + Q^2 + Q^3 + Q^4) = Q C + D0,
    C = 2I + 2S + T,  D0 = I + 2S + 2T,
which the kernels form as three products whose epilogues add the rest:
    S = Q Q,  C' = S S + 2S,  B = (Q + 2I) C' + 2Q - 2S + I
with C' = C - 2I stored instead of C (three products instead of four by
Horner's rule; no stored matrix carries a multiple of I, so bf16 storage
rounds only the small parts).  Its gradient needs only
the antisymmetric part of dL/dQ, because theta enters Q as Q[a,c] = theta =
-Q[c,a]; S, T and C are symmetric, so only the symmetric parts of dL/dS and
dL/dT matter:
    dT_s = sym(2G - QG)                 (sym(X) = (X + X^T) / 2)
    W = dT_s S,  dS_s = sym(2G - 2QG) + W + W^T,
    D = G C - 2 dS_s Q,  dtheta[a,c] = D[a,c] - D[c,a],
which the kernels form as four products with the sums in their epilogues:
    U = G - Q G,  G C = G C' + 2G,  dT_s = sym(G + U),  V = dT_s S + U,
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
    """The products and epilogue sums the kernels take; returns C' = C - 2I."""
    eye = np.eye(Q.shape[0])
    Q2 = Q + 2 * eye                    # written by the unpack
    S = Q @ Q
    Cp = S @ S + 2 * S                  # epilogue: addend S (beta 2)
    B = Q2 @ Cp + 2 * Q - 2 * S + eye   # epilogue: addends Q (beta 2) and S (beta -2), diagonal 1
    return B, S, Cp


def _powers_grad(Q, S, C, G):
    sym2 = lambda X: X + X.T  # noqa: E731  (twice the symmetric part)
    QG, GC = Q @ G, G @ C
    dTs = sym2(G) - 0.5 * sym2(QG)
    W = dTs @ S
    dSs = sym2(G) - sym2(QG) + W + W.T
    D = GC - 2 * (dSs @ Q)
    r, c = np.triu_indices(Q.shape[0], 1)
    return D[r, c] - D[c, r]


def _kernel_grad(Q, S, Cp, G):
    sym2 = lambda X: X + X.T  # noqa: E731
    U = G - Q @ G                       # product alpha -1, addend G
    GC = G @ Cp + 2 * G                 # product, addend G (beta 2)
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


def _bf16(x):
    """Round to bfloat16 (nearest even) and back to float64."""
    import torch

    return torch.from_numpy(np.asarray(x, dtype=np.float32)).to(torch.bfloat16).to(torch.float64).numpy()


@pytest.mark.parametrize("size", [256, 1024])
def test_order4_bf16_storage_rounds_only_small_parts(size):
    """With bf16 storage of every stored matrix (Q, S, C' and B) and float sums,
    the kernels' order-4 arrangement stays within twice the rounding of B
    itself.  Storing C = C' + 2I instead (diagonal near 2) fails this: its
    rounding, doubled by the 2I part of Q + 2I, lands on B's diagonal."""
    rng = np.random.default_rng(size)
    theta = rng.standard_normal(O.n_skew(size)) * 0.02
    Q = _bf16(O.unpack_skew(theta, size))
    exact = O.cayley_neumann_block(Q, 4)
    eye = np.eye(size)
    S = _bf16(Q @ Q)
    Cp = _bf16(S @ S + 2 * S)
    B = _bf16((Q + 2 * eye) @ Cp + 2 * Q - 2 * S + eye)
    floor = np.linalg.norm(_bf16(exact) - exact)
    assert np.linalg.norm(B - exact) <= 2.0 * floor
    C = _bf16(S @ S + 2 * S + 2 * eye)
    B_stored_c = _bf16((Q + 2 * eye) @ C - 2 * S - 3 * eye)
    assert np.linalg.norm(B_stored_c - exact) > 2.0 * floor

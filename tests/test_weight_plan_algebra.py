"""The weight plan's reassociation, restated on the CPU in float64 and checked
against the oracle's dense forward and backward (no GPU).

The weight plan applies the primitives to W0 instead of the activations:
    H = R^ W0f,  F = W0f P^,  E_f = H P^  (frame, R^ / P^ = block-diagonal sides),
    E = E_f taken back to natural order,  y = x E^T,  dx = dy E,
    D = dy^T x,  D_f = D in the frame,
    G_R[j] = D_f[rows j] F[rows j]^T,  G_P[j] = H[:, cols j]^T D_f[:, cols j].
These are exact identities of y = R W0 P x; this test pins them independently
of the CUDA path (the GPU tests then check the kernels against the oracle)."""
import numpy as np
import pytest

from oracle import poet_oracle as O

BS, FS = 0, 1

CASES = [
    # m, n, modeR, bR, modeP, bP, k, T
    (300, 200, BS, 64, BS, 64, 2, 37),      # leftover identity indices on both sides
    (301, 199, FS, 0, FS, 0, 3, 29),        # fully stochastic, odd sizes
    (96, 160, FS, 0, BS, 16, 1, 21),        # mixed modes
    (40, 24, BS, 64, BS, 64, 2, 9),         # b > d: no primitives
    (64, 48, BS, 16, BS, 16, 0, 13),        # k = 0
]


def frame_side(d, blocks, mode, b):
    """The side in its own frame: blockdiag(blocks, I), primitives on consecutive index ranges."""
    nprim, size = O.side_shape(d, mode, b)
    M = np.eye(d)
    for j in range(nprim):
        M[j * size:(j + 1) * size, j * size:(j + 1) * size] = blocks[j]
    return M


@pytest.mark.parametrize("m,n,modeR,bR,modeP,bP,k,T", CASES)
def test_weight_plan_matches_dense_chain_rule(m, n, modeR, bR, modeP, bP, k, T):
    rng = np.random.default_rng(m * 1000 + n)
    W0 = rng.standard_normal((m, n))
    X = rng.standard_normal((T, n))
    dY = rng.standard_normal((T, m))
    permR = O.draw_perm(5, m + n, 0, 0, m)
    permP = O.draw_perm(5, m + n, 1, 0, n)
    nR, sR = O.side_shape(m, modeR, bR)
    nP, sP = O.side_shape(n, modeP, bP)
    thR = 0.05 * rng.standard_normal(nR * O.n_skew(sR))
    thP = 0.05 * rng.standard_normal(nP * O.n_skew(sP))
    Rb = O.cayley_neumann(thR, nR, sR, k)
    Pb = O.cayley_neumann(thP, nP, sP, k)

    # oracle: dense matrices, per-token chain rule
    R = O.dense_side(permR, Rb, modeR, bR)
    P = O.dense_side(permP, Pb, modeP, bP)
    Y_ref = O.forward(W0, R, P, X)
    dX_ref, GR_ref, GP_ref = O.backward(W0, R, P, X, dY, permR, modeR, bR, permP, modeP, bP)

    # weight plan, in the frame
    W0f = W0[np.ix_(permR, permP)]
    Rh, Ph = frame_side(m, Rb, modeR, bR), frame_side(n, Pb, modeP, bP)
    H, F = Rh @ W0f, W0f @ Ph
    E_f = H @ Ph
    E = np.empty_like(W0)
    E[np.ix_(permR, permP)] = E_f
    Y = X @ E.T
    dX = dY @ E
    D_f = (dY.T @ X)[np.ix_(permR, permP)]
    GR = np.stack([D_f[j * sR:(j + 1) * sR] @ F[j * sR:(j + 1) * sR].T for j in range(nR)]) if nR else np.zeros((0, sR, sR))
    GP = np.stack([H[:, j * sP:(j + 1) * sP].T @ D_f[:, j * sP:(j + 1) * sP] for j in range(nP)]) if nP else np.zeros((0, sP, sP))

    def close(a, b):
        return np.linalg.norm(a - b) <= 1e-12 * max(1.0, np.linalg.norm(b))

    assert close(Y, Y_ref)
    assert close(dX, dX_ref)
    assert GR.shape == GR_ref.shape and close(GR, GR_ref)
    assert GP.shape == GP_ref.shape and close(GP, GP_ref)
    # E is the dense R W0 P: the merge of the same step
    assert close(E, O.merge(W0, R, P))


@pytest.mark.parametrize("m,n,modeR,bR,modeP,bP,k,T", CASES + [(200, 341, BS, 64, FS, 0, 4, 11),
                                                               (512, 384, FS, 0, BS, 128, 2, 7)])
def test_weight_plan_partial_buffers(m, n, modeR, bR, modeP, bP, k, T):
    """The weight plan as the grouped kernels evaluate it: H computed on the
    rows the R primitives cover (c_R), F on the columns the P primitives cover
    (c_P), E_f = H P on both; when both sides have primitives, H's other rows
    and F's other columns are copied from W0f; E is unframed from E_f / H on
    rows < c_R and from F / W0f on the others, split at column c_P; G_R reads
    whole rows of F (W0f without P primitives), G_P whole columns of H (W0f
    without R primitives).  Regions no kernel writes hold NaN, so a read of
    one shows."""
    rng = np.random.default_rng(m * 7 + n)
    W0 = rng.standard_normal((m, n))
    X = rng.standard_normal((T, n))
    dY = rng.standard_normal((T, m))
    permR = O.draw_perm(3, m + n, 0, 1, m)
    permP = O.draw_perm(3, m + n, 1, 1, n)
    nR, sR = O.side_shape(m, modeR, bR)
    nP, sP = O.side_shape(n, modeP, bP)
    Rb = O.cayley_neumann(0.05 * rng.standard_normal(nR * O.n_skew(sR)), nR, sR, k)
    Pb = O.cayley_neumann(0.05 * rng.standard_normal(nP * O.n_skew(sP)), nP, sP, k)
    R = O.dense_side(permR, Rb, modeR, bR)
    P = O.dense_side(permP, Pb, modeP, bP)
    Y_ref = O.forward(W0, R, P, X)
    dX_ref, GR_ref, GP_ref = O.backward(W0, R, P, X, dY, permR, modeR, bR, permP, modeP, bP)

    cR, cP = nR * sR, nP * sP
    W0f = W0[np.ix_(permR, permP)]
    nan = np.full((m, n), np.nan)
    H, F, Ef = nan.copy(), nan.copy(), nan.copy()
    for j in range(nR):  # H = R^ W0f on the covered rows
        H[j * sR:(j + 1) * sR] = Rb[j] @ W0f[j * sR:(j + 1) * sR]
    for j in range(nP):  # F = W0f P^ on the covered columns
        F[:, j * sP:(j + 1) * sP] = W0f[:, j * sP:(j + 1) * sP] @ Pb[j]
    if nR and nP:  # the leftover rows of H and columns of F, copied from W0f
        H[cR:] = W0f[cR:]
        F[:, cP:] = W0f[:, cP:]
        for j in range(nP):  # E_f = H P^ on the covered rows and columns
            Ef[:cR, j * sP:(j + 1) * sP] = H[:cR, j * sP:(j + 1) * sP] @ Pb[j]
    # unframe: rows < c_R from E_f (columns < c_P) and H; the others from F (columns < c_P) and W0f
    Efull = np.empty((m, n))
    top = Ef if nP else H
    Efull[:cR, :cP] = top[:cR, :cP]
    Efull[:cR, cP:] = H[:cR, cP:]
    bot = F if nP else W0f
    Efull[cR:, :cP] = bot[cR:, :cP]
    Efull[cR:, cP:] = W0f[cR:, cP:]
    E = np.empty((m, n))
    E[np.ix_(permR, permP)] = Efull
    Y = X @ E.T
    dX = dY @ E
    D_f = (dY.T @ X)[np.ix_(permR, permP)]
    Fg = F if nP else W0f
    Hg = H if nR else W0f
    GR = np.stack([D_f[j * sR:(j + 1) * sR] @ Fg[j * sR:(j + 1) * sR].T for j in range(nR)]) if nR else \
        np.zeros((0, sR, sR))
    GP = np.stack([Hg[:, j * sP:(j + 1) * sP].T @ D_f[:, j * sP:(j + 1) * sP] for j in range(nP)]) if nP else \
        np.zeros((0, sP, sP))

    def close(a, b):
        return np.isfinite(a).all() and np.linalg.norm(a - b) <= 1e-12 * max(1.0, np.linalg.norm(b))

    assert close(Y, Y_ref)
    assert close(dX, dX_ref)
    assert GR.shape == GR_ref.shape and close(GR, GR_ref)
    assert GP.shape == GP_ref.shape and close(GP, GP_ref)

"""Plain CPU oracle for the POET reparameterized linear layer.

TEST INFRASTRUCTURE ONLY.  Nothing in the product path may import, call or
execute this module: only the tests, ``__graft_entry__.smoke()`` and the CPU
baseline leg of ``bench.py`` use it.  It shares no code with the CUDA library.

Everything is computed in float64 with numpy, one obvious step at a time, on
dense matrices where the method has a dense definition.  A library matmul,
``numpy.linalg.solve`` and a stable sort are the only library primitives used.

Sources (web pages on POET / POET-X):
  [P1] "Reparameterized LLM Training via Orthogonal Equivalence Transformation"
       (atlas.scime.ai summary of arXiv 2506.08001), sections "Approach",
       "Key results", "Measured effects reported in the paper", "Limitations".
  [P2] mlsanity page for arXiv 2506.08001, "Abstract".
  [P3] "POET-X: Memory-efficient LLM Training by Scaling Orthogonal
       Transformation" (pith.science review), "Core claim", "What carries the
       argument".

The pages state the method only in words: each weight is R @ W0 @ P with W0
fixed and R, P orthogonal, built from sampled sub-block primitives, with a
truncated Neumann-series Cayley map and periodic merge-then-reinitialize
([P1] Approach, Limitations).  Where they are silent this module takes the
plainest reading; every such reading is listed in the repository's design
notes and marked "reading:" below.

Conventions (readings):
  * W0 is m x n (out x in); activations are token-major: x is T x n, y is T x m,
    so Y = X @ P.T @ W0.T @ R.T is the per-token y_t = R W0 P x_t.
  * One side of dimension d has perm (a permutation of 0..d-1) and a mode:
      BS (block-stochastic): floor(d/b) primitives of size b; primitive j acts on
         natural indices perm[j*b : (j+1)*b]; the d mod b leftover indices are
         untouched (identity).
      FS (fully stochastic, "b=1/2"): one primitive of size s = floor(d/2)
         acting on natural indices perm[0:s]; the rest is identity.
  * theta of one primitive of size b holds b(b-1)/2 values, the strict upper
    triangle packed row by row: Q[a,c] = theta, Q[c,a] = -theta for a < c.
  * Cayley-Neumann of order k: R_blk = (I + Q) (I + Q + Q^2 + ... + Q^k), the
    Cayley map (I+Q)(I-Q)^-1 with the inverse replaced by its truncated series.

The optimizer step on theta (``adamw_step``) is adjacent to the path: the
pages name no optimizer, so it is the textbook AdamW update (decoupled weight
decay, bias-corrected moments; Loshchilov & Hutter, "Decoupled Weight Decay
Regularization") -- a reading.  Its pins are that update's own closed forms.

Parity pins: every function here is checked in tests/test_oracle_pins.py
against closed forms, exact identities, brute force or values printed on the
pages.  ``draw_perm``'s generator is pinned to the published SplitMix64 test
vectors; the choice of generator itself is a reading (the pages fix none), so
parity of the permutations against any external source is unpinned.
"""
from __future__ import annotations

import numpy as np

BS = 0
FS = 1

_MASK64 = (1 << 64) - 1
_GAMMA = 0x9E3779B97F4A7C15  # SplitMix64 increment (Steele, Lea, Flood 2014)


# --------------------------------------------------------------------------
# side geometry and parameter packing
# --------------------------------------------------------------------------

def side_shape(dim: int, mode: int, b: int) -> tuple[int, int]:
    """(number of primitives, primitive size) of one side.

    [P1] Key results: "POET-FS (b=1/2)" and "POET-BS (b=256)".
    reading: FS = one primitive over floor(d/2) sampled indices;
             BS = floor(d/b) blocks, leftover indices identity.
    """
    if mode == FS:
        return 1, dim // 2
    if mode == BS:
        return dim // b, b
    raise ValueError("mode must be BS or FS")


def n_skew(size: int) -> int:
    """Number of free parameters of one size x size skew-symmetric matrix."""
    return size * (size - 1) // 2


def unpack_skew(theta_blk: np.ndarray, size: int) -> np.ndarray:
    """Q (size x size, skew-symmetric) from the packed strict upper triangle.

    reading: row-major strict upper triangle; Q = U - U^T.
    """
    theta_blk = np.asarray(theta_blk)
    assert theta_blk.shape == (n_skew(size),)
    Q = np.zeros((size, size), dtype=np.result_type(theta_blk.dtype, np.float64))
    rows, cols = np.triu_indices(size, k=1)  # row-major order of the strict upper triangle
    Q[rows, cols] = theta_blk
    Q[cols, rows] = -theta_blk
    return Q


def pack_skew_grad(dQ: np.ndarray) -> np.ndarray:
    """Gradient w.r.t. the packed parameters given dL/dQ (chain rule through
    Q[a,c] = theta, Q[c,a] = -theta): dtheta = dQ[a,c] - dQ[c,a] for a < c."""
    size = dQ.shape[0]
    rows, cols = np.triu_indices(size, k=1)
    return dQ[rows, cols] - dQ[cols, rows]


# --------------------------------------------------------------------------
# a1: Cayley-Neumann parameterization
# --------------------------------------------------------------------------

def cayley_neumann_block(Q: np.ndarray, k: int) -> np.ndarray:
    """R = (I + Q) (sum_{i=0..k} Q^i).   [P1] Approach, Limitations."""
    size = Q.shape[0]
    eye = np.eye(size, dtype=Q.dtype)
    power = eye.copy()
    series = eye.copy()
    for _ in range(k):
        power = power @ Q
        series = series + power
    return (eye + Q) @ series


def exact_cayley(Q: np.ndarray) -> np.ndarray:
    """C = (I + Q)(I - Q)^-1, the untruncated Cayley map (for pins only)."""
    eye = np.eye(Q.shape[0], dtype=Q.dtype)
    # (I+Q) and (I-Q)^-1 commute, so C = (I-Q)^-1 (I+Q) = solve(I-Q, I+Q)
    return np.linalg.solve(eye - Q, eye + Q)


def cayley_neumann(theta: np.ndarray, nprim: int, size: int, k: int) -> np.ndarray:
    """All primitives of one side: theta (nprim * size(size-1)/2) -> (nprim, size, size)."""
    theta = np.asarray(theta, dtype=np.float64)
    per = n_skew(size)
    assert theta.shape == (nprim * per,)
    out = np.empty((nprim, size, size), dtype=np.float64)
    for j in range(nprim):
        out[j] = cayley_neumann_block(unpack_skew(theta[j * per:(j + 1) * per], size), k)
    return out


# --------------------------------------------------------------------------
# dense materialization of one side
# --------------------------------------------------------------------------

def block_index_sets(perm: np.ndarray, mode: int, b: int) -> list[np.ndarray]:
    """The natural indices each primitive acts on, in primitive order."""
    perm = np.asarray(perm)
    nprim, size = side_shape(len(perm), mode, b)
    return [perm[j * size:(j + 1) * size] for j in range(nprim)]


def dense_side(perm: np.ndarray, blocks: np.ndarray, mode: int, b: int) -> np.ndarray:
    """The d x d orthogonal-primitive matrix  Pi^T diag(blocks, I) Pi,
    with (Pi v)_i = v[perm[i]]: entry [I_j[a], I_j[c]] = block_j[a, c]."""
    d = len(perm)
    M = np.eye(d, dtype=np.float64)
    for j, idx in enumerate(block_index_sets(perm, mode, b)):
        M[np.ix_(idx, idx)] = blocks[j]
    return M


def apply_side_rows(X: np.ndarray, perm: np.ndarray, blocks: np.ndarray, mode: int, b: int) -> np.ndarray:
    """Rows of X (tokens) multiplied by the side matrix: returns X @ M^T for
    M = dense_side(perm, blocks, mode, b), computed primitive by primitive
    (out[:, I_j] = X[:, I_j] @ block_j^T, other columns copied) so that full
    LLaMA widths stay cheap."""
    X = np.asarray(X, dtype=np.float64)
    out = X.copy()
    for j, idx in enumerate(block_index_sets(perm, mode, b)):
        out[:, idx] = X[:, idx] @ np.asarray(blocks[j], dtype=np.float64).T
    return out


# --------------------------------------------------------------------------
# a2..a4: forward,  a5..a8: backward
# --------------------------------------------------------------------------

def forward(W0: np.ndarray, R: np.ndarray, P: np.ndarray, X: np.ndarray) -> np.ndarray:
    """Y = X P^T W0^T R^T  (per token y = R W0 P x).   [P1] Approach; [P2] Abstract."""
    U = X @ P.T
    V = U @ W0.T
    return V @ R.T


def restrict_blocks(M: np.ndarray, perm: np.ndarray, mode: int, b: int) -> np.ndarray:
    """The primitive-shaped pieces of a d x d matrix: out[j] = M[I_j][:, I_j]
    (an empty stack when the side has no primitive, e.g. b > d)."""
    nprim, size = side_shape(len(perm), mode, b)
    if nprim == 0:
        return np.zeros((0, size, size))
    return np.stack([M[np.ix_(idx, idx)] for idx in block_index_sets(perm, mode, b)])


def backward(W0, R, P, X, dY, permR, modeR, bR, permP, modeP, bP):
    """Chain rule through y = R W0 P x for loss gradient dY (T x m).

    Returns dX (T x n), G_R (dL/dR restricted to R's primitives) and G_P.
    W0 is fixed ([P1] Approach: "fixed random W0"), so there is no dW0.
    """
    V = X @ P.T @ W0.T           # v_t = W0 P x_t
    dV = dY @ R                  # dv_t = R^T dy_t
    dU = dV @ W0                 # du_t = W0^T dv_t
    dX = dU @ P                  # dx_t = P^T du_t
    G_R = restrict_blocks(dY.T @ V, permR, modeR, bR)   # dL/dR = sum_t dy_t v_t^T
    G_P = restrict_blocks(dU.T @ X, permP, modeP, bP)   # dL/dP = sum_t du_t x_t^T
    return dX, G_R, G_P


def theta_grad_block(G: np.ndarray, theta_blk: np.ndarray, size: int, k: int) -> np.ndarray:
    """a8: gradient of <G, R(Q)> w.r.t. the packed parameters of one primitive.

    With R(Q) = (I+Q) S(Q), S = sum_{i<=k} Q^i, the product rule gives
      dL/dQ = G S^T + sum_{i=1..k} sum_{j=0..i-1} (Q^T)^j (I+Q)^T G (Q^T)^(i-1-j),
    then dtheta[a,c] = dQ[a,c] - dQ[c,a].
    """
    Q = unpack_skew(theta_blk, size)
    eye = np.eye(size, dtype=Q.dtype)
    S = eye.copy()
    power = eye.copy()
    for _ in range(k):
        power = power @ Q
        S = S + power
    QT = Q.T
    QT_pows = [eye]
    for _ in range(k):
        QT_pows.append(QT_pows[-1] @ QT)
    B = (eye + Q).T @ G
    dQ = G @ S.T
    for i in range(1, k + 1):
        for j in range(i):
            dQ = dQ + QT_pows[j] @ B @ QT_pows[i - 1 - j]
    return pack_skew_grad(dQ)


def theta_grad(G_blocks: np.ndarray, theta: np.ndarray, size: int, k: int) -> np.ndarray:
    """a8 for every primitive of one side; returns the packed dtheta vector."""
    per = n_skew(size)
    theta = np.asarray(theta, dtype=np.float64)
    return np.concatenate([
        theta_grad_block(np.asarray(G_blocks[j], dtype=np.float64), theta[j * per:(j + 1) * per], size, k)
        for j in range(len(G_blocks))
    ]) if len(G_blocks) else np.zeros(0)


# --------------------------------------------------------------------------
# a9: merge-then-reinitialize
# --------------------------------------------------------------------------

def merge(W0: np.ndarray, R: np.ndarray, P: np.ndarray) -> np.ndarray:
    """W0' = R W0 P.  [P1] Approach ("merged periodically"), Measured effects
    (merge-then-reinitialize frequency).  After it theta is reset to 0, which
    makes every primitive the identity for any k."""
    return R @ W0 @ P


# --------------------------------------------------------------------------
# a10: resample (the generator is a reading: the pages fix none)
# --------------------------------------------------------------------------

def splitmix64(state: int) -> int:
    """Output of a SplitMix64 generator whose state is ``state`` before the step
    (Steele, Lea, Flood, "Fast splittable pseudorandom number generators", 2014)."""
    z = (state + _GAMMA) & _MASK64
    z = ((z ^ (z >> 30)) * 0xBF58476D1CE4E5B9) & _MASK64
    z = ((z ^ (z >> 27)) * 0x94D049BB133111EB) & _MASK64
    return z ^ (z >> 31)


def splitmix64_stream(seed: int, count: int) -> list[int]:
    """First ``count`` outputs of SplitMix64 seeded with ``seed``."""
    return [splitmix64((seed + i * _GAMMA) & _MASK64) for i in range(count)]


def perm_stream_seed(seed: int, layer_id: int, side: int, epoch: int) -> int:
    """Seed of the key stream of one side (side 0 = R, 1 = P) at one epoch:
    h = sm(seed XOR sm((layer_id << 32) XOR (epoch << 1) XOR side))."""
    inner = splitmix64((((layer_id & 0xFFFFFFFF) << 32) ^ ((epoch & 0x7FFFFFFF) << 1) ^ (side & 1)) & _MASK64)
    return splitmix64((seed ^ inner) & _MASK64)


def draw_perm(seed: int, layer_id: int, side: int, epoch: int, dim: int) -> np.ndarray:
    """Permutation of 0..dim-1: indices ordered by (key_i, i) ascending, where
    key_i is the i-th output of SplitMix64 seeded with perm_stream_seed(...).
    [P1] Approach ("sampled sub-block orthogonal primitives")."""
    keys = splitmix64_stream(perm_stream_seed(seed, layer_id, side, epoch), dim)
    order = sorted(range(dim), key=lambda i: (keys[i], i))
    return np.asarray(order, dtype=np.int32)


# --------------------------------------------------------------------------
# bookkeeping
# --------------------------------------------------------------------------

def trainable_params(dim_out: int, dim_in: int, mode: int, b: int) -> int:
    """Trainable parameters of one POET linear (both sides)."""
    total = 0
    for d in (dim_out, dim_in):
        nprim, size = side_shape(d, mode, b)
        total += nprim * n_skew(size)
    return total


def llama_linear_shapes(hidden: int, ffn: int) -> list[tuple[int, int]]:
    """(m, n) = (out, in) of the seven linears of one LLaMA block:
    q, k, v, o (h x h), gate, up (f x h), down (h x f)."""
    return [(hidden, hidden)] * 4 + [(ffn, hidden)] * 2 + [(hidden, ffn)]


# --------------------------------------------------------------------------
# one whole layer, start to finish (small sizes)
# --------------------------------------------------------------------------

def layer_step(W0, thetaR, thetaP, permR, permP, modeR, bR, modeP, bP, k, X, dY):
    """a1..a9 for one layer on dense matrices.  Returns a dict with
    R_blocks, P_blocks, Y, dX, dthetaR, dthetaP, W0_merged."""
    m, n = W0.shape
    nR, sR = side_shape(m, modeR, bR)
    nP, sP = side_shape(n, modeP, bP)
    Rb = cayley_neumann(thetaR, nR, sR, k)
    Pb = cayley_neumann(thetaP, nP, sP, k)
    R = dense_side(permR, Rb, modeR, bR)
    P = dense_side(permP, Pb, modeP, bP)
    X = np.asarray(X, dtype=np.float64)
    dY = np.asarray(dY, dtype=np.float64)
    W0 = np.asarray(W0, dtype=np.float64)
    Y = forward(W0, R, P, X)
    dX, G_R, G_P = backward(W0, R, P, X, dY, permR, modeR, bR, permP, modeP, bP)
    return {
        "R_blocks": Rb, "P_blocks": Pb, "Y": Y, "dX": dX,
        "G_R": G_R, "G_P": G_P,
        "dthetaR": theta_grad(G_R, thetaR, sR, k),
        "dthetaP": theta_grad(G_P, thetaP, sP, k),
        "W0_merged": merge(W0, R, P),
    }


# --------------------------------------------------------------------------
# adjacent: the optimizer step on the packed parameters (a reading)
# --------------------------------------------------------------------------

def adamw_step(theta, grad, m, v, lr, beta1, beta2, eps, weight_decay, step):
    """One AdamW step, elementwise on the packed skew parameters: the first and
    second moment estimates are updated, bias-corrected by 1 - beta**step, and
    theta moves by lr * (m_hat / (sqrt(v_hat) + eps) + weight_decay * theta)
    (decay decoupled from the gradient).  Returns (theta, m, v) after the step."""
    theta = np.asarray(theta, dtype=np.float64)
    grad = np.asarray(grad, dtype=np.float64)
    m_new = beta1 * np.asarray(m, dtype=np.float64) + (1.0 - beta1) * grad
    v_new = beta2 * np.asarray(v, dtype=np.float64) + (1.0 - beta2) * grad * grad
    m_hat = m_new / (1.0 - beta1 ** step)
    v_hat = v_new / (1.0 - beta2 ** step)
    theta_new = theta - lr * (m_hat / (np.sqrt(v_hat) + eps) + weight_decay * theta)
    return theta_new, m_new, v_new

"""Plant plausible mistakes in copies of the oracle (on the CPU) and check that
the pins catch each one: a pin set that a dropped term, a wrong sign, a
transposed operand or a wrong index survives would not pin anything."""
import types

import numpy as np
import pytest

from oracle import poet_oracle as O
from tests import oracle_pins


def _mutant(**overrides):
    m = types.ModuleType("mutant_oracle")
    m.__dict__.update({k: v for k, v in O.__dict__.items() if not k.startswith("__")})
    m.__dict__.update(overrides)
    # functions look globals up in their own module: rebind them to the mutant
    for name, fn in list(m.__dict__.items()):
        if isinstance(fn, types.FunctionType) and name not in overrides:
            m.__dict__[name] = types.FunctionType(fn.__code__, m.__dict__, fn.__name__, fn.__defaults__, fn.__closure__)
    for name, fn in overrides.items():
        if isinstance(fn, types.FunctionType):
            m.__dict__[name] = types.FunctionType(fn.__code__, m.__dict__, fn.__name__, fn.__defaults__, fn.__closure__)
    return m


def _unpack_transposed(theta_blk, size):
    Q = np.zeros((size, size))
    rows, cols = np.triu_indices(size, k=1)
    Q[rows, cols] = -theta_blk
    Q[cols, rows] = theta_blk
    return Q


def _unpack_colmajor(theta_blk, size):
    Q = np.zeros((size, size))
    cols, rows = np.triu_indices(size, k=1)   # column-major order of the upper triangle
    order = np.lexsort((rows, cols))
    r, c = rows[order], cols[order]
    Q[r, c] = theta_blk
    Q[c, r] = -theta_blk
    return Q


def _cnp_one_term_short(Q, k):
    eye = np.eye(Q.shape[0])
    power, series = eye.copy(), eye.copy()
    for _ in range(max(k - 1, 0)):
        power = power @ Q
        series = series + power
    return (eye + Q) @ series


def _cnp_wrong_sign(Q, k):
    eye = np.eye(Q.shape[0])
    power, series = eye.copy(), eye.copy()
    for _ in range(k):
        power = power @ Q
        series = series + power
    return (eye - Q) @ series


def _theta_grad_drop_GS(G, theta_blk, size, k):
    Q = unpack_skew(theta_blk, size)  # noqa: F821  (resolved in the mutant module)
    eye = np.eye(size)
    QT = Q.T
    QT_pows = [eye]
    for _ in range(k):
        QT_pows.append(QT_pows[-1] @ QT)
    B = (eye + Q).T @ G
    dQ = np.zeros_like(G)
    for i in range(1, k + 1):
        for j in range(i):
            dQ = dQ + QT_pows[j] @ B @ QT_pows[i - 1 - j]
    return pack_skew_grad(dQ)  # noqa: F821


def _theta_grad_transposed_B(G, theta_blk, size, k):
    Q = unpack_skew(theta_blk, size)  # noqa: F821
    eye = np.eye(size)
    S = eye.copy()
    power = eye.copy()
    for _ in range(k):
        power = power @ Q
        S = S + power
    QT_pows = [eye]
    for _ in range(k):
        QT_pows.append(QT_pows[-1] @ Q.T)
    B = G @ (eye + Q).T
    dQ = G @ S.T
    for i in range(1, k + 1):
        for j in range(i):
            dQ = dQ + QT_pows[j] @ B @ QT_pows[i - 1 - j]
    return pack_skew_grad(dQ)  # noqa: F821


def _pack_grad_sum(dQ):
    rows, cols = np.triu_indices(dQ.shape[0], k=1)
    return dQ[rows, cols] + dQ[cols, rows]


def _dense_side_transposed(perm, blocks, mode, b):
    d = len(perm)
    M = np.eye(d)
    for j, idx in enumerate(block_index_sets(perm, mode, b)):  # noqa: F821
        M[np.ix_(idx, idx)] = blocks[j].T
    return M


def _block_sets_inverse(perm, mode, b):
    inv = np.argsort(np.asarray(perm))
    nprim, size = side_shape(len(perm), mode, b)  # noqa: F821
    return [inv[j * size:(j + 1) * size] for j in range(nprim)]


def _side_shape_ceil(dim, mode, b):
    if mode == 1:
        return 1, (dim + 1) // 2
    return -(-dim // b), b


def _forward_no_R(W0, R, P, X):
    return X @ P.T @ W0.T


def _forward_transposed_P(W0, R, P, X):
    return X @ P @ W0.T @ R.T


def _backward_wrong_dU(W0, R, P, X, dY, permR, modeR, bR, permP, modeP, bP):
    V = X @ P.T @ W0.T
    dV = dY @ R.T
    dU = dV @ W0
    dX = dU @ P
    G_R = restrict_blocks(dY.T @ V, permR, modeR, bR)  # noqa: F821
    G_P = restrict_blocks(dU.T @ X, permP, modeP, bP)  # noqa: F821
    return dX, G_R, G_P


def _backward_GR_swapped(W0, R, P, X, dY, permR, modeR, bR, permP, modeP, bP):
    V = X @ P.T @ W0.T
    dV = dY @ R
    dU = dV @ W0
    dX = dU @ P
    G_R = restrict_blocks(V.T @ dY, permR, modeR, bR)  # noqa: F821
    G_P = restrict_blocks(dU.T @ X, permP, modeP, bP)  # noqa: F821
    return dX, G_R, G_P


def _merge_wrong_order(W0, R, P):
    return P.T @ W0.T @ R.T if W0.shape[0] == W0.shape[1] else R @ W0 @ P.T


def _splitmix_wrong_const(state):
    mask = (1 << 64) - 1
    z = (state + 0x9E3779B97F4A7C15) & mask
    z = ((z ^ (z >> 30)) * 0xBF58476D1CE4E5B9) & mask
    z = ((z ^ (z >> 27)) * 0x94D049BB133111EB) & mask
    return z ^ (z >> 30)


def _draw_perm_descending(seed, layer_id, side, epoch, dim):
    keys = splitmix64_stream(perm_stream_seed(seed, layer_id, side, epoch), dim)  # noqa: F821
    return np.asarray(sorted(range(dim), key=lambda i: (-keys[i], i)), dtype=np.int32)


_M64 = (1 << 64) - 1


def _stream_seed_side_epoch_swapped(seed, layer_id, side, epoch):
    inner = splitmix64((((layer_id & 0xFFFFFFFF) << 32) ^ ((side & 1) << 1) ^ (epoch & 0x7FFFFFFF)) & _M64)  # noqa: F821
    return splitmix64((seed ^ inner) & _M64)  # noqa: F821


def _stream_seed_no_inner_step(seed, layer_id, side, epoch):
    inner = (((layer_id & 0xFFFFFFFF) << 32) ^ ((epoch & 0x7FFFFFFF) << 1) ^ (side & 1)) & _M64
    return splitmix64((seed ^ inner) & _M64)  # noqa: F821


def _stream_seed_layer_unshifted(seed, layer_id, side, epoch):
    inner = splitmix64(((layer_id & 0xFFFFFFFF) ^ ((epoch & 0x7FFFFFFF) << 1) ^ (side & 1)) & _M64)  # noqa: F821
    return splitmix64((seed ^ inner) & _M64)  # noqa: F821


def _trainable_with_diag(dim_out, dim_in, mode, b):
    total = 0
    for d in (dim_out, dim_in):
        nprim, size = side_shape(d, mode, b)  # noqa: F821
        total += nprim * size * (size + 1) // 2
    return total


def _adamw_no_bias_correction(theta, grad, m, v, lr, beta1, beta2, eps, weight_decay, step):
    m_new = beta1 * m + (1.0 - beta1) * grad
    v_new = beta2 * v + (1.0 - beta2) * grad * grad
    return theta - lr * (m_new / (np.sqrt(v_new) + eps) + weight_decay * theta), m_new, v_new


def _adamw_coupled_decay(theta, grad, m, v, lr, beta1, beta2, eps, weight_decay, step):
    grad = grad + weight_decay * theta  # L2 penalty folded into the gradient (Adam, not AdamW)
    m_new = beta1 * m + (1.0 - beta1) * grad
    v_new = beta2 * v + (1.0 - beta2) * grad * grad
    m_hat, v_hat = m_new / (1.0 - beta1 ** step), v_new / (1.0 - beta2 ** step)
    return theta - lr * m_hat / (np.sqrt(v_hat) + eps), m_new, v_new


def _adamw_no_sqrt(theta, grad, m, v, lr, beta1, beta2, eps, weight_decay, step):
    m_new = beta1 * m + (1.0 - beta1) * grad
    v_new = beta2 * v + (1.0 - beta2) * grad * grad
    m_hat, v_hat = m_new / (1.0 - beta1 ** step), v_new / (1.0 - beta2 ** step)
    return theta - lr * (m_hat / (v_hat + eps) + weight_decay * theta), m_new, v_new


MUTANTS = {
    "unpack transposed sign": dict(unpack_skew=_unpack_transposed),
    "unpack column-major": dict(unpack_skew=_unpack_colmajor),
    "neumann series one term short": dict(cayley_neumann_block=_cnp_one_term_short),
    "cayley (I-Q) instead of (I+Q)": dict(cayley_neumann_block=_cnp_wrong_sign),
    "theta grad drops G S^T": dict(theta_grad_block=_theta_grad_drop_GS),
    "theta grad transposed product": dict(theta_grad_block=_theta_grad_transposed_B),
    "pack grad with + instead of -": dict(pack_skew_grad=_pack_grad_sum),
    "dense side with transposed blocks": dict(dense_side=_dense_side_transposed),
    "index sets from inverse perm": dict(block_index_sets=_block_sets_inverse),
    "ceil block counts": dict(side_shape=_side_shape_ceil),
    "forward drops R": dict(forward=_forward_no_R),
    "forward transposed P": dict(forward=_forward_transposed_P),
    "backward dV with R^T": dict(backward=_backward_wrong_dU),
    "backward G_R transposed": dict(backward=_backward_GR_swapped),
    "merge wrong operand order": dict(merge=_merge_wrong_order),
    "splitmix wrong final shift": dict(splitmix64=_splitmix_wrong_const),
    "perm sorted descending": dict(draw_perm=_draw_perm_descending),
    "stream seed with side and epoch terms swapped": dict(perm_stream_seed=_stream_seed_side_epoch_swapped),
    "stream seed without the inner SplitMix64 step": dict(perm_stream_seed=_stream_seed_no_inner_step),
    "stream seed with the layer not shifted": dict(perm_stream_seed=_stream_seed_layer_unshifted),
    "trainable count includes diagonal": dict(trainable_params=_trainable_with_diag),
    "adamw without bias correction": dict(adamw_step=_adamw_no_bias_correction),
    "adamw with the decay in the gradient": dict(adamw_step=_adamw_coupled_decay),
    "adamw without the square root": dict(adamw_step=_adamw_no_sqrt),
}


def _fails_some_pin(M):
    for check in oracle_pins.ALL_CHECKS:
        try:
            if not check(M):
                return check.__name__
        except Exception as e:  # a crash also counts as caught
            return f"{check.__name__} ({type(e).__name__})"
    return None


@pytest.mark.parametrize("name", list(MUTANTS))
def test_planted_mistake_is_caught(name):
    M = _mutant(**MUTANTS[name])
    assert _fails_some_pin(M) is not None, f"no pin catches: {name}"


def test_unmutated_copy_passes_all_pins():
    assert _fails_some_pin(_mutant()) is None

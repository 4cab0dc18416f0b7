"""Pins of the LLaMA-block oracle (oracle/llama_block.py) against what
mathematics fixes, independently of the oracle itself (no GPU):
  * central finite differences of the loss <dout, out> for dh and for sampled
    packed parameters of every linear (the loss is smooth in both);
  * causality: an output row depends on no later token of its sequence and on
    no other sequence;
  * rotary embedding: closed-form angles at hand-picked positions, norm
    preservation, the inverse undoing the rotation;
  * RMSNorm rows of unit root mean square; softmax rows summing to 1 with zeros
    above the diagonal.
Planted mistakes in copies of the module (on the CPU) must each fail a pin."""
import types

import numpy as np
import pytest

from oracle import llama_block as LB
from oracle import poet_oracle as O

SHAPE = LB.BlockShape(hidden=8, ffn=12, heads=2, head_dim=4, seq_len=5)


def _block(rng, mode=O.BS, b=2, k=3, scale=0.2):
    lin = {}
    dims = {"q": (8, 8), "k": (8, 8), "v": (8, 8), "o": (8, 8), "gate": (12, 8), "up": (12, 8), "down": (8, 12)}
    for i, name in enumerate(LB.LINEARS):
        m, n = dims[name]
        nR, sR = O.side_shape(m, mode, b)
        nP, sP = O.side_shape(n, mode, b)
        W0 = rng.standard_normal((m, n))
        W0 /= np.linalg.norm(W0, axis=1, keepdims=True)
        lin[name] = LB.PoetLinear(W0, scale * rng.standard_normal(nR * O.n_skew(sR)),
                                  scale * rng.standard_normal(nP * O.n_skew(sP)),
                                  O.draw_perm(1, i, 0, 0, m), O.draw_perm(1, i, 1, 0, n), mode, b, k)
    return lin


def _check_fd(M, mode=O.BS, b=2):
    rng = np.random.default_rng(5)
    lin = _block(rng, mode, b)
    T = 2 * SHAPE.seq_len
    h = rng.standard_normal((T, SHAPE.hidden))
    dout = rng.standard_normal((T, SHAPE.hidden))
    out, cache = M.block_forward(h, lin, SHAPE)
    dh, dth = M.block_backward(dout, lin, cache, SHAPE)
    loss = lambda hh: float(np.sum(dout * M.block_forward(hh, lin, SHAPE)[0]))  # noqa: E731
    eps = 1e-6
    fd = np.zeros_like(h)
    for idx in np.ndindex(*h.shape):
        hp, hm = h.copy(), h.copy()
        hp[idx] += eps
        hm[idx] -= eps
        fd[idx] = (loss(hp) - loss(hm)) / (2 * eps)
    if not np.allclose(dh, fd, rtol=1e-5, atol=1e-7):
        return False
    for name in LB.LINEARS:
        for side, attr in ((0, "thetaR"), (1, "thetaP")):
            th = getattr(lin[name], attr)
            for j in range(0, th.size, max(1, th.size // 3)):
                keep = th[j]
                th[j] = keep + eps
                lp = loss(h)
                th[j] = keep - eps
                lm = loss(h)
                th[j] = keep
                if not np.isclose(dth[name][side][j], (lp - lm) / (2 * eps), rtol=1e-5, atol=1e-7):
                    return False
    return True


def _check_causal(M):
    rng = np.random.default_rng(6)
    lin = _block(rng)
    S = SHAPE.seq_len
    h = rng.standard_normal((2 * S, SHAPE.hidden))
    out, _ = M.block_forward(h, lin, SHAPE)
    h2 = h.copy()
    h2[3] += 1.0          # a later token of sequence 0
    h2[S + 1] -= 1.0      # a token of sequence 1
    out2, _ = M.block_forward(h2, lin, SHAPE)
    return np.allclose(out[:3], out2[:3], rtol=0, atol=1e-13) and not np.allclose(out[3], out2[3])


def _check_rope(M):
    shape = LB.BlockShape(hidden=4, ffn=4, heads=1, head_dim=4, seq_len=3)
    x = np.tile(np.array([[1.0, 0.0, 1.0, 0.0]]), (3, 1))
    y = M.rope(x, shape)
    # position p: pair 0 turns by p rad, pair 1 by p * 10000**(-1/2) = p / 100 rad
    expect = np.array([[np.cos(p), np.sin(p), np.cos(p / 100), np.sin(p / 100)] for p in range(3)])
    ok = np.allclose(y, expect, rtol=0, atol=1e-15)
    z = np.random.default_rng(7).standard_normal((6, 8))
    s2 = LB.BlockShape(hidden=8, ffn=8, heads=2, head_dim=4, seq_len=3)
    rz = M.rope(z, s2)
    ok &= np.allclose(np.linalg.norm(rz, axis=1), np.linalg.norm(z, axis=1), rtol=1e-14)
    ok &= np.allclose(M.rope(rz, s2, inverse=True), z, rtol=0, atol=1e-14)
    return bool(ok)


def _check_norm_softmax(M):
    rng = np.random.default_rng(8)
    x = 3.0 * rng.standard_normal((7, 16))
    y, r = M.rmsnorm(x, 0.0)
    ok = np.allclose(np.sqrt(np.mean(y * y, axis=1)), 1.0, rtol=1e-14)
    q, k, v = (rng.standard_normal((10, 8)) for _ in range(3))
    _, probs = M.attention(q, k, v, SHAPE)
    ok &= np.allclose(probs.sum(axis=-1), 1.0, rtol=1e-14)
    ok &= not np.any(np.triu(probs, 1))
    return bool(ok)


CHECKS = [_check_fd, _check_causal, _check_rope, _check_norm_softmax]


@pytest.mark.parametrize("check", CHECKS, ids=lambda f: f.__name__)
def test_block_oracle_pin(check):
    assert check(LB)


def test_block_oracle_fd_fully_stochastic():
    assert _check_fd(LB, mode=O.FS)


def _mutant(**overrides):
    m = types.ModuleType("mutant_block")
    m.__dict__.update({k: v for k, v in LB.__dict__.items() if not k.startswith("__")})
    m.__dict__.update(overrides)
    for name, fn in list(m.__dict__.items()):
        if isinstance(fn, types.FunctionType):
            m.__dict__[name] = types.FunctionType(fn.__code__, m.__dict__, fn.__name__, fn.__defaults__,
                                                  fn.__closure__)
    return m


def _rms_bwd_no_centering(dy, y, r):
    return dy / r


def _silu_grad_wrong(z):
    return 1.0 / (1.0 + np.exp(-z))


def _rope_angle_doubled(seq_len, head_dim, base):
    i = np.arange(head_dim // 2, dtype=np.float64)
    p = np.arange(seq_len, dtype=np.float64)
    return p[:, None] * base ** (-1.0 * i / head_dim)[None, :]


def _attention_mask_off_by_one(q, k, v, shape):
    T, d = q.shape
    S, hd = shape.seq_len, shape.head_dim
    B, H = T // S, d // hd
    o = np.zeros_like(q)
    probs = np.zeros((B, H, S, S))
    mask = np.tril(np.ones((S, S), dtype=bool), 1)
    for b in range(B):
        rows = slice(b * S, (b + 1) * S)
        for h in range(H):
            cols = slice(h * hd, (h + 1) * hd)
            s = np.where(mask, q[rows, cols] @ k[rows, cols].T / np.sqrt(hd), -np.inf)
            e = np.exp(s - s.max(axis=1, keepdims=True))
            p = e / e.sum(axis=1, keepdims=True)
            probs[b, h] = p
            o[rows, cols] = p @ v[rows, cols]
    return o, probs


def _attention_bwd_no_scale(do, q, k, v, probs, shape):
    T, d = q.shape
    S, hd = shape.seq_len, shape.head_dim
    dq, dk, dv = np.zeros_like(q), np.zeros_like(k), np.zeros_like(v)
    for b in range(T // S):
        rows = slice(b * S, (b + 1) * S)
        for h in range(d // hd):
            cols = slice(h * hd, (h + 1) * hd)
            p = probs[b, h]
            dp = do[rows, cols] @ v[rows, cols].T
            dv[rows, cols] = p.T @ do[rows, cols]
            ds = p * (dp - np.sum(dp * p, axis=1, keepdims=True))
            dq[rows, cols] = ds @ k[rows, cols]
            dk[rows, cols] = ds.T @ q[rows, cols]
    return dq, dk, dv


MUTANTS = {
    "rmsnorm backward without the centering term": dict(rmsnorm_backward=_rms_bwd_no_centering),
    "silu derivative without the product rule": dict(silu_grad=_silu_grad_wrong),
    "rotary angles with exponent -i/d": dict(rope_angles=_rope_angle_doubled),
    "causal mask admits the next token": dict(attention=_attention_mask_off_by_one),
    "attention backward without 1/sqrt(d)": dict(attention_backward=_attention_bwd_no_scale),
}


@pytest.mark.parametrize("name", list(MUTANTS))
def test_block_planted_mistake_is_caught(name):
    M = _mutant(**MUTANTS[name])
    caught = False
    for check in CHECKS:
        try:
            if not check(M):
                caught = True
                break
        except Exception:  # a crash also counts as caught
            caught = True
            break
    assert caught, f"no pin catches: {name}"

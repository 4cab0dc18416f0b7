"""Plain CPU oracle of one LLaMA block whose seven linears are POET layers.

TEST INFRASTRUCTURE ONLY.  Nothing in the product path may import, call or
execute this module: only the tests, ``__graft_entry__.smoke()`` and the CPU
baseline leg of ``bench.py`` use it.  It shares no code with the CUDA library.

The POET pages train LLaMA models whose linear layers are POET layers
("Reparameterized LLM Training via Orthogonal Equivalence Transformation",
Experimental setup: LLaMA-60M ... 3B pretraining on C4).  They do not restate
the LLaMA block; this module takes the published LLaMA design (Touvron et al.,
"LLaMA: Open and Efficient Foundation Language Models", 2023: pre-normalization
with RMSNorm, rotary position embeddings, causal multi-head self-attention,
a SwiGLU feed-forward network, residual connections).  Readings where the
pages and that design leave a choice open:
  * the RMSNorm gains are 1 and not trained here (only the POET parameters are);
    eps = 1e-6 inside the square root;
  * rotary embedding on interleaved pairs (2i, 2i+1) of each head, angle
    position * base**(-2i / head_dim), base 10000, positions counted within
    each sequence;
  * attention scores scaled by 1 / sqrt(head_dim), causal mask, softmax per row;
  * SwiGLU: down(silu(gate(x)) * up(x)), silu(z) = z / (1 + exp(-z)).

Everything is float64 numpy on dense arrays, one obvious step at a time.  The
seven linears are ``poet_oracle``'s layers (dense R and P).  The backward is
the chain rule written out step by step; tests pin it against central finite
differences of the loss <dout, out> on tiny blocks.
"""
from __future__ import annotations

from dataclasses import dataclass

import numpy as np

from oracle import poet_oracle as O

LINEARS = ("q", "k", "v", "o", "gate", "up", "down")


@dataclass
class BlockShape:
    hidden: int
    ffn: int
    heads: int
    head_dim: int
    seq_len: int
    eps: float = 1e-6
    rope_base: float = 10000.0


# ------------------------------------------------------------------ pieces

def rmsnorm(x, eps):
    """y = x / sqrt(mean(x^2) + eps) per row; returns (y, r) with r the per-row divisor."""
    r = np.sqrt(np.mean(x * x, axis=1, keepdims=True) + eps)
    return x / r, r


def rmsnorm_backward(dy, y, r):
    """Gradient through y = x / r(x): dx = (dy - y * mean(dy * y)) / r."""
    return (dy - y * np.mean(dy * y, axis=1, keepdims=True)) / r


def rope_angles(seq_len, head_dim, base):
    """theta[p, i] = p * base**(-2i / head_dim) for positions p < seq_len, pairs i < head_dim / 2."""
    i = np.arange(head_dim // 2, dtype=np.float64)
    p = np.arange(seq_len, dtype=np.float64)
    return p[:, None] * base ** (-2.0 * i / head_dim)[None, :]


def rope(x, shape: BlockShape, inverse=False):
    """Rotate the interleaved pairs (2i, 2i+1) of every head of every token by its
    angle (the inverse rotation when inverse=True, which is also its backward)."""
    T, d = x.shape
    S, hd = shape.seq_len, shape.head_dim
    ang = rope_angles(S, hd, shape.rope_base)          # S x hd/2
    pos = np.arange(T) % S
    c = np.cos(ang[pos])                                  # T x hd/2
    s = np.sin(ang[pos]) * (-1.0 if inverse else 1.0)
    out = np.empty_like(x)
    for h in range(d // hd):
        x0 = x[:, h * hd:(h + 1) * hd:2]
        x1 = x[:, h * hd + 1:(h + 1) * hd:2]
        out[:, h * hd:(h + 1) * hd:2] = x0 * c - x1 * s
        out[:, h * hd + 1:(h + 1) * hd:2] = x0 * s + x1 * c
    return out


def attention(q, k, v, shape: BlockShape):
    """Causal multi-head attention per sequence; returns (o, probs) with
    probs[b, h] the S x S softmax of (q_h k_h^T / sqrt(head_dim)) under the causal mask."""
    T, d = q.shape
    S, hd = shape.seq_len, shape.head_dim
    B, H = T // S, d // hd
    o = np.zeros_like(q)
    probs = np.zeros((B, H, S, S))
    mask = np.tril(np.ones((S, S), dtype=bool))
    for b in range(B):
        rows = slice(b * S, (b + 1) * S)
        for h in range(H):
            cols = slice(h * hd, (h + 1) * hd)
            s = q[rows, cols] @ k[rows, cols].T / np.sqrt(hd)
            s = np.where(mask, s, -np.inf)
            s = s - s.max(axis=1, keepdims=True)
            e = np.exp(s)
            p = e / e.sum(axis=1, keepdims=True)
            probs[b, h] = p
            o[rows, cols] = p @ v[rows, cols]
    return o, probs


def attention_backward(do, q, k, v, probs, shape: BlockShape):
    """Chain rule through attention(): returns dq, dk, dv."""
    T, d = q.shape
    S, hd = shape.seq_len, shape.head_dim
    B, H = T // S, d // hd
    dq, dk, dv = np.zeros_like(q), np.zeros_like(k), np.zeros_like(v)
    for b in range(B):
        rows = slice(b * S, (b + 1) * S)
        for h in range(H):
            cols = slice(h * hd, (h + 1) * hd)
            p = probs[b, h]
            dp = do[rows, cols] @ v[rows, cols].T
            dv[rows, cols] = p.T @ do[rows, cols]
            ds = p * (dp - np.sum(dp * p, axis=1, keepdims=True)) / np.sqrt(hd)
            dq[rows, cols] = ds @ k[rows, cols]
            dk[rows, cols] = ds.T @ q[rows, cols]
    return dq, dk, dv


def silu(z):
    return z / (1.0 + np.exp(-z))


def silu_grad(z):
    sg = 1.0 / (1.0 + np.exp(-z))
    return sg * (1.0 + z * (1.0 - sg))


# ------------------------------------------------------------------ the POET linears

@dataclass
class PoetLinear:
    """One POET linear: W0 (m x n), its sides' parameters and geometry (dense form)."""
    W0: np.ndarray
    thetaR: np.ndarray
    thetaP: np.ndarray
    permR: np.ndarray
    permP: np.ndarray
    mode: int
    b: int
    k: int

    def sides(self):
        m, n = self.W0.shape
        nR, sR = O.side_shape(m, self.mode, self.b)
        nP, sP = O.side_shape(n, self.mode, self.b)
        Rb = O.cayley_neumann(self.thetaR, nR, sR, self.k)
        Pb = O.cayley_neumann(self.thetaP, nP, sP, self.k)
        return O.dense_side(self.permR, Rb, self.mode, self.b), O.dense_side(self.permP, Pb, self.mode, self.b)

    def forward(self, x):
        R, P = self.sides()
        return O.forward(self.W0, R, P, x)

    def backward(self, x, dy):
        """dx and the packed-parameter gradients of both sides."""
        m, n = self.W0.shape
        R, P = self.sides()
        dx, GR, GP = O.backward(self.W0, R, P, x, dy, self.permR, self.mode, self.b, self.permP, self.mode, self.b)
        _, sR = O.side_shape(m, self.mode, self.b)
        _, sP = O.side_shape(n, self.mode, self.b)
        return dx, O.theta_grad(GR, self.thetaR, sR, self.k), O.theta_grad(GP, self.thetaP, sP, self.k)


# ------------------------------------------------------------------ the block

def block_forward(h, lin: dict, shape: BlockShape):
    """out = h1 + down(silu(gate(n2)) * up(n2)), h1 = h + o(attn(rope(q(n1)), rope(k(n1)), v(n1))),
    n1 = rmsnorm(h), n2 = rmsnorm(h1).  Returns out and the intermediates the backward needs."""
    n1, r1 = rmsnorm(h, shape.eps)
    q, k, v = lin["q"].forward(n1), lin["k"].forward(n1), lin["v"].forward(n1)
    qr, kr = rope(q, shape), rope(k, shape)
    att, probs = attention(qr, kr, v, shape)
    h1 = h + lin["o"].forward(att)
    n2, r2 = rmsnorm(h1, shape.eps)
    g, u = lin["gate"].forward(n2), lin["up"].forward(n2)
    mlp = silu(g) * u
    out = h1 + lin["down"].forward(mlp)
    cache = dict(n1=n1, r1=r1, qr=qr, kr=kr, v=v, att=att, probs=probs, n2=n2, r2=r2, g=g, u=u, mlp=mlp)
    return out, cache


def block_backward(dout, lin: dict, cache: dict, shape: BlockShape):
    """dh and, per linear, (dtheta_R, dtheta_P), for the loss <dout, out>."""
    dth = {}
    dmlp, *td = lin["down"].backward(cache["mlp"], dout)
    dth["down"] = tuple(td)
    g, u = cache["g"], cache["u"]
    dg = dmlp * u * silu_grad(g)
    du = dmlp * silu(g)
    dn2_g, *tg = lin["gate"].backward(cache["n2"], dg)
    dn2_u, *tu = lin["up"].backward(cache["n2"], du)
    dth["gate"], dth["up"] = tuple(tg), tuple(tu)
    dh1 = dout + rmsnorm_backward(dn2_g + dn2_u, cache["n2"], cache["r2"])
    datt, *to = lin["o"].backward(cache["att"], dh1)
    dth["o"] = tuple(to)
    dqr, dkr, dv = attention_backward(datt, cache["qr"], cache["kr"], cache["v"], cache["probs"], shape)
    dq, dk = rope(dqr, shape, inverse=True), rope(dkr, shape, inverse=True)
    n1 = cache["n1"]
    dn1 = np.zeros_like(n1)
    for name, d in (("q", dq), ("k", dk), ("v", dv)):
        dx, tR, tP = lin[name].backward(n1, d)
        dn1 += dx
        dth[name] = (tR, tP)
    dh = dh1 + rmsnorm_backward(dn1, n1, cache["r1"])
    return dh, dth

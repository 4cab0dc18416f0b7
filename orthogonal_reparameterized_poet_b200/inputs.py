"""Seeded synthetic inputs and workload shapes.

This module holds none of the method's arithmetic: it only draws seeded
random numbers in the shapes, scales and distributions of the workloads the
POET pages train on (LLaMA-60M ... 3B linears), and rounds them to the
storage type.  Both the CUDA path's tests/benchmarks and the CPU oracle are
fed from here, so they see bit-identical inputs.

Recipe (one Philox counter-based stream per tensor, keyed by
(config seed, layer, linear, tensor id)):
  * W0: rows ~ N(0, 1), each row then scaled to unit L2 norm ("normalized
    Gaussian" initialization, POET summary page, Measured effects table).
  * theta: ~ N(0, sigma^2), sigma per workload.
  * x, dy: ~ N(0, 1).
  * bf16 workloads: every input is rounded to bfloat16 (round to nearest
    even) before either side sees it; the oracle receives the rounded values.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np

BS = 0
FS = 1
F32 = 0
BF16 = 1

# tensor ids of the per-tensor streams
_T_W0, _T_THETA_R, _T_THETA_P, _T_X, _T_DY = 1, 2, 3, 4, 5


def _stream(seed: int, *key: int) -> np.random.Generator:
    ss = np.random.SeedSequence([int(seed) & 0xFFFFFFFF] + [int(k) & 0xFFFFFFFF for k in key])
    return np.random.Generator(np.random.Philox(ss))


def normal(seed: int, key: tuple, shape, scale: float = 1.0) -> np.ndarray:
    """float32 N(0, scale^2) samples from the stream (seed, *key)."""
    g = _stream(seed, *key)
    out = g.standard_normal(size=shape, dtype=np.float32)
    if scale != 1.0:
        out *= np.float32(scale)
    return out


def round_bf16(a: np.ndarray) -> np.ndarray:
    """Round float32 values to the nearest bfloat16 (ties to even); returned as float32."""
    import torch

    t = torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32))
    return t.to(torch.bfloat16).to(torch.float32).numpy()


def to_storage(a: np.ndarray, dtype: int) -> np.ndarray:
    return round_bf16(a) if dtype == BF16 else np.ascontiguousarray(a, dtype=np.float32)


def w0(seed: int, layer: int, linear: int, m: int, n: int, dtype: int) -> np.ndarray:
    a = normal(seed, (layer, linear, _T_W0), (m, n))
    a /= np.sqrt(np.einsum("ij,ij->i", a, a, dtype=np.float64)).astype(np.float32)[:, None]
    return to_storage(a, dtype)


def theta(seed: int, layer: int, linear: int, side: int, count: int, sigma: float) -> np.ndarray:
    """Packed skew parameters (always float32, the parameter type)."""
    return normal(seed, (layer, linear, _T_THETA_R if side == 0 else _T_THETA_P), (count,), sigma)


def activations(seed: int, shape_id: int, T: int, d: int, dtype: int, grad: bool = False) -> np.ndarray:
    """x (grad=False) or dy (grad=True) for one linear shape, T x d."""
    return to_storage(normal(seed, (0xA11, shape_id, _T_DY if grad else _T_X), (T, d)), dtype)


@dataclass(frozen=True)
class Workload:
    name: str
    hidden: int
    ffn: int | None           # None: one square linear of size hidden
    layers: int
    mode: int
    b: int                    # BS block size (ignored for FS)
    k: int
    sigma: float
    tokens: int
    dtype: int
    seed: int = 0
    merge_every: int = 400
    variants: tuple = field(default_factory=tuple)

    def linear_shapes(self) -> list[tuple[int, int]]:
        """(m, n) = (out, in) of the POET linears of one layer."""
        if self.ffn is None:
            return [(self.hidden, self.hidden)]
        h, f = self.hidden, self.ffn
        return [(h, h)] * 4 + [(f, h)] * 2 + [(h, f)]


# The five synthetic workloads, in the LLaMA shapes the POET pages train on.
WORKLOADS = {
    "single256_fp32_bs32": Workload("single256_fp32_bs32", 256, None, 1, BS, 32, 3, 0.01, 512, F32, merge_every=1),
    "llama60m_fs": Workload("llama60m_fs", 512, 1376, 1, FS, 0, 4, 0.02, 8 * 256, BF16),
    "llama350m_bs256": Workload("llama350m_bs256", 1024, 2736, 24, BS, 256, 4, 0.02, 16 * 1024, BF16),
    "llama1.3b_fs": Workload("llama1.3b_fs", 2048, 5461, 24, FS, 0, 4, 0.02, 16 * 2048, BF16),
    "llama1.3b_bs256": Workload("llama1.3b_bs256", 2048, 5461, 24, BS, 256, 4, 0.02, 16 * 2048, BF16),
    "llama3b_fs": Workload("llama3b_fs", 2560, 6912, 32, FS, 0, 4, 0.02, 8 * 2048, BF16),
}

"""poet_cayley_neumann_grad_noalloc: the packed-skew gradient for callers that
cannot allocate device memory (their host framework owns all of it), using
the library's built-in scratch array instead of a caller workspace.

It runs the same kernels as poet_cayley_neumann_grad (the entry point that
takes a workspace) in the same order, so on the same inputs its result must be
bitwise equal to that entry point's, on two calls in a row (the second call
finds the first call's leftovers in the shared scratch, so stale scratch
would show); it is also compared with the oracle at the usual bar.  Free
device memory must not change across its calls.  This file is collected last
so that a run stopping at the first failure has run every other test."""
import numpy as np
import pytest

from oracle import poet_oracle as O
from orthogonal_reparameterized_poet_b200 import inputs as I
from tests.harness import TOL, rel_fro

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def cuda():
    import torch

    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from orthogonal_reparameterized_poet_b200 import poet

    poet.lib()
    return torch


def _side(cuda, dim, mode, b, k, dtype, seed):
    from orthogonal_reparameterized_poet_b200 import poet

    s = poet.poet_side()
    s.dim, s.mode, s.b, s.k = dim, mode, b, k
    nprim, size = O.side_shape(dim, mode, b)
    theta = I.theta(seed, 0, 0, 0, nprim * O.n_skew(size), 0.02)
    theta_d = cuda.from_numpy(theta).cuda()
    state = cuda.empty(poet.poet_side_state_bytes(s, dtype), dtype=cuda.uint8, device="cuda")
    perm = cuda.arange(dim, dtype=cuda.int32, device="cuda")
    s.perm, s.theta, s.state = perm.data_ptr(), theta_d.data_ptr(), state.data_ptr()
    poet.poet_cayley_neumann(s, dtype)
    return s, (theta_d, state, perm), nprim, size, theta


@pytest.mark.parametrize("dim,mode,b,k,dtype", [
    (2048, I.BS, 256, 4, I.BF16),   # 8 blocks of 256, the LLaMA-1.3B hidden side
    (5461, I.BS, 256, 4, I.BF16),   # 21 blocks, the LLaMA-1.3B FFN side
    (1376, I.FS, 0, 4, I.BF16),     # one 688 x 688 primitive
    (256, I.BS, 32, 3, I.F32),      # float32, 8 blocks of 32
])
def test_noalloc_matches_workspace_entry_point(cuda, dim, mode, b, k, dtype):
    from orthogonal_reparameterized_poet_b200 import poet

    s, keep, nprim, size, theta = _side(cuda, dim, mode, b, k, dtype, seed=11)
    ws = cuda.empty(poet.poet_side_workspace_bytes(s, dtype), dtype=cuda.uint8, device="cuda")
    for call in range(2):  # two calls in a row, different upstream gradients
        G = np.random.default_rng(100 + call).standard_normal((nprim, size, size)).astype(np.float32)
        Gd = cuda.from_numpy(G).cuda()
        ref = cuda.empty(nprim * O.n_skew(size), dtype=cuda.float32, device="cuda")
        got = cuda.full_like(ref, float("nan"))
        poet.poet_cayley_neumann_grad(s, dtype, Gd, ref, ws)
        poet.poet_cayley_neumann_grad_noalloc(s, dtype, Gd, got)
        poet.poet_sync_status()
        assert cuda.equal(got, ref), f"call {call}: max |diff| {(got - ref).abs().max().item():.3e}"
        expect = O.theta_grad(G.astype(np.float64), theta.astype(np.float64), size, k)
        assert rel_fro(got.cpu().numpy(), expect) <= TOL[dtype]


def test_noalloc_allocates_nothing(cuda):
    """After a first call on the device, further calls leave the device's free memory unchanged."""
    from orthogonal_reparameterized_poet_b200 import poet

    s, keep, nprim, size, theta = _side(cuda, 2048, I.BS, 256, 4, I.BF16, seed=13)
    G = cuda.randn(nprim * size * size, dtype=cuda.float32, device="cuda")
    out = cuda.empty(nprim * O.n_skew(size), dtype=cuda.float32, device="cuda")
    poet.poet_cayley_neumann_grad_noalloc(s, I.BF16, G, out)  # first call: looks up the scratch address
    poet.poet_sync_status()
    free0, _ = cuda.cuda.mem_get_info()
    for _ in range(5):
        poet.poet_cayley_neumann_grad_noalloc(s, I.BF16, G, out)
    poet.poet_sync_status()
    free1, _ = cuda.cuda.mem_get_info()
    assert free1 == free0


def test_noalloc_rejects_sides_beyond_its_scratch(cuda):
    from orthogonal_reparameterized_poet_b200 import poet

    s, keep, nprim, size, theta = _side(cuda, 5461, I.FS, 0, 4, I.BF16, seed=12)  # one 2730 x 2730 primitive
    assert poet.poet_side_workspace_bytes(s, I.BF16) > 32 << 20
    G = cuda.zeros(nprim * size * size, dtype=cuda.float32, device="cuda")
    out = cuda.zeros(nprim * O.n_skew(size), dtype=cuda.float32, device="cuda")
    with pytest.raises(poet.PoetError, match="scratch"):
        poet.poet_cayley_neumann_grad_noalloc(s, I.BF16, G, out)

"""CUDA path (through the C ABI) against the CPU oracle on the same seeded
inputs.  Bar: bit-exact for permutations; relative Frobenius error <= 1e-5
for float32 workloads and <= 2e-2 for bfloat16 workloads."""
import numpy as np
import pytest

from oracle import poet_oracle as O
from orthogonal_reparameterized_poet_b200 import inputs as I
from tests.harness import TOL, Case, read_blocks, rel_fro, run_gpu, run_oracle

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def cuda():
    import torch

    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from orthogonal_reparameterized_poet_b200 import poet

    poet.lib()  # raises if the library is missing: no fallback
    return torch


# ------------------------------------------------------------------ a10

@pytest.mark.parametrize("dim", [1, 2, 3, 255, 256, 1376, 2736, 5461, 6912, 16384])
def test_draw_perm_bit_exact(cuda, dim):
    from orthogonal_reparameterized_poet_b200 import poet

    for (seed, layer_id, side, epoch) in [(0, 0, 0, 0), (0, 5, 1, 3), (123456789, 167, 0, 41)]:
        p = cuda.empty(dim, dtype=cuda.int32, device="cuda")
        poet.poet_draw_perm(seed, layer_id, side, epoch, dim, p)
        got = p.cpu().numpy()
        assert np.array_equal(got, O.draw_perm(seed, layer_id, side, epoch, dim))


# ------------------------------------------------------------------ a1 / a8

def _side_struct(cuda, dim, mode, b, k, theta, dtype):
    from orthogonal_reparameterized_poet_b200 import poet

    s = poet.poet_side()
    s.dim, s.mode, s.b, s.k = dim, mode, b, k
    th = cuda.from_numpy(theta).cuda()
    state = cuda.empty(max(poet.poet_side_state_bytes(s, dtype), 1), dtype=cuda.uint8, device="cuda")
    perm = cuda.arange(dim, dtype=cuda.int32, device="cuda")
    s.perm, s.theta, s.state = perm.data_ptr(), th.data_ptr(), state.data_ptr()
    return s, (th, state, perm)


CNP_CASES = [
    # dim, mode, b, k, sigma, dtype
    (256, I.BS, 32, 3, 0.01, I.F32),
    (200, I.BS, 64, 0, 0.05, I.F32),
    (90, I.BS, 7, 5, 0.1, I.F32),
    (1024, I.BS, 256, 4, 0.02, I.BF16),
    (1376, I.FS, 0, 4, 0.02, I.BF16),
    (5461, I.FS, 0, 4, 0.02, I.BF16),
    (2560, I.FS, 0, 4, 0.02, I.BF16),   # LLaMA-3B hidden side: one 1280 x 1280 primitive
    (6912, I.FS, 0, 4, 0.02, I.BF16),   # LLaMA-3B FFN side: one 3456 x 3456 primitive
    (301, I.FS, 0, 2, 0.03, I.F32),
]


@pytest.mark.parametrize("dim,mode,b,k,sigma,dtype", CNP_CASES)
def test_cayley_neumann_forward_and_grad(cuda, dim, mode, b, k, sigma, dtype):
    from orthogonal_reparameterized_poet_b200 import poet

    nprim, size = O.side_shape(dim, mode, b)
    theta = I.theta(7, 0, 0, 0, nprim * O.n_skew(size), sigma)
    s, keep = _side_struct(cuda, dim, mode, b, k, theta, dtype)
    poet.poet_cayley_neumann(s, dtype)
    got = read_blocks(keep[1], (nprim, size), dtype)
    ref = O.cayley_neumann(theta.astype(np.float64), nprim, size, k)
    assert rel_fro(got, ref) <= TOL[dtype]
    # a8 on a random upstream gradient
    G = np.random.default_rng(1).standard_normal((nprim, size, size)).astype(np.float32)
    ws = cuda.empty(poet.poet_side_workspace_bytes(s, dtype), dtype=cuda.uint8, device="cuda")
    dth = cuda.empty(theta.size, dtype=cuda.float32, device="cuda")
    poet.poet_cayley_neumann_grad(s, dtype, cuda.from_numpy(G).cuda(), dth, ws)
    poet.poet_sync_status()
    ref_g = O.theta_grad(G.astype(np.float64), theta.astype(np.float64), size, k)
    assert rel_fro(dth.cpu().numpy(), ref_g) <= TOL[dtype]


# ------------------------------------------------------------------ whole layer

LAYER_CASES = {
    # the 256 x 256 float32 layer: b = 32, k = 3, 512 tokens, sigma 0.01
    "single256_fp32_bs32": Case(256, 256, I.BS, 32, I.BS, 32, 3, 512, I.F32, 0.01),
    # LLaMA-60M shapes, fully stochastic, k = 4, 8 x 256 tokens, bf16
    "llama60m_fs_q": Case(512, 512, I.FS, 0, I.FS, 0, 4, 2048, I.BF16, 0.02, linear=0, layer_id=0),
    "llama60m_fs_gate": Case(1376, 512, I.FS, 0, I.FS, 0, 4, 2048, I.BF16, 0.02, linear=4, layer_id=4),
    "llama60m_fs_down": Case(512, 1376, I.FS, 0, I.FS, 0, 4, 2048, I.BF16, 0.02, linear=6, layer_id=6),
    # ragged: leftover identity indices, token count not a tile multiple
    "ragged_bs_fp32": Case(300, 200, I.BS, 64, I.BS, 64, 2, 333, I.F32, 0.05, layer_id=3, epoch=2),
    "ragged_bs_bf16": Case(300, 200, I.BS, 64, I.BS, 64, 2, 333, I.BF16, 0.05, layer_id=3),
    "ragged_fs_fp32": Case(301, 199, I.FS, 0, I.FS, 0, 3, 77, I.F32, 0.03, layer_id=9),
    # block-stochastic b = 256 on LLaMA-350M FFN shapes (10 blocks + 176 leftover), few tokens
    "bs256_ffn_bf16": Case(2736, 1024, I.BS, 256, I.BS, 256, 4, 300, I.BF16, 0.02, layer_id=11),
    "bs256_down_bf16": Case(1024, 2736, I.BS, 256, I.BS, 256, 4, 130, I.BF16, 0.02, layer_id=12),
    # LLaMA-3B down projection width (6912-wide rows through the permutes), block-stochastic
    "bs256_3b_down_bf16": Case(2560, 6912, I.BS, 256, I.BS, 256, 4, 70, I.BF16, 0.02, layer_id=13),
    # natural rows of odd width in float32 (every 16-byte misalignment of a row start)
    "odd_width_fp32": Case(333, 517, I.BS, 40, I.FS, 0, 2, 45, I.F32, 0.04, layer_id=14),
    # mixed modes and degenerate sides
    "mixed_fs_bs": Case(96, 160, I.FS, 0, I.BS, 16, 1, 40, I.F32, 0.05),
    "k0": Case(64, 48, I.BS, 16, I.BS, 16, 0, 33, I.F32, 0.05),
    "b1_no_params": Case(40, 24, I.BS, 1, I.BS, 1, 2, 9, I.F32, 0.05),
    "b_gt_dim": Case(40, 24, I.BS, 64, I.BS, 64, 2, 9, I.F32, 0.05),
    "single_token": Case(128, 64, I.BS, 32, I.FS, 0, 2, 1, I.F32, 0.05),
    # primitives of size <= 32 (the small-block kernels): bf16 b = 32 / 16, and fully stochastic sides of 30 / 25
    "smallb_bs32_bf16": Case(512, 384, I.BS, 32, I.BS, 16, 4, 300, I.BF16, 0.02, layer_id=15),
    "smallb_fs_fp32": Case(60, 50, I.FS, 0, I.FS, 0, 3, 70, I.F32, 0.05, layer_id=16),
}


PLANS = {"token": 1, "weight": 2}


@pytest.mark.parametrize("plan", list(PLANS))
@pytest.mark.parametrize("name", list(LAYER_CASES))
def test_layer_parity(cuda, name, plan):
    case = LAYER_CASES[name]
    arrs = case.arrays()
    ref = run_oracle(case, *arrs)
    got = run_gpu(case, *arrs, plan=PLANS[plan])
    assert got["plan"] == PLANS[plan]
    tol = TOL[case.dtype]
    assert np.array_equal(got["permR"], ref["permR"]) and np.array_equal(got["permP"], ref["permP"])
    if len(ref["R_blocks"]):
        assert rel_fro(got["R_blocks"], ref["R_blocks"]) <= tol
    if len(ref["P_blocks"]):
        assert rel_fro(got["P_blocks"], ref["P_blocks"]) <= tol
    errs = {
        "Y": rel_fro(got["Y"], ref["Y"]),
        "dX": rel_fro(got["dX"], ref["dX"]),
        "W0_merged": rel_fro(got["W0_merged"], ref["W0_merged"]),
    }
    if ref["dthetaR"].size:
        errs["dthetaR"] = rel_fro(got["dthetaR"], ref["dthetaR"])
    if ref["dthetaP"].size:
        errs["dthetaP"] = rel_fro(got["dthetaP"], ref["dthetaP"])
    bad = {k: v for k, v in errs.items() if not v <= tol}
    assert not bad, f"{name}: {bad} (tol {tol})"
    # merge-then-reinitialize: theta reset, epoch advanced, output unchanged
    assert not np.any(got["thetaR_after_merge"])
    assert got["epoch_after"] == case.epoch + 1
    assert np.array_equal(got["permR_after"], O.draw_perm(case.seed, case.layer_id, 0, case.epoch + 1, case.m))
    assert rel_fro(got["Y_after_merge"], ref["Y"]) <= tol


@pytest.mark.parametrize("plan", list(PLANS))
def test_zero_tokens(cuda, plan):
    from orthogonal_reparameterized_poet_b200 import poet

    case = LAYER_CASES["ragged_bs_fp32"]
    W0, thR, thP, x, dy = case.arrays()
    L = poet.PoetLayer(cuda.from_numpy(W0).cuda(), cuda.from_numpy(thR).cuda(), cuda.from_numpy(thP).cuda(),
                       mode=case.modeR, b=case.bR, k=case.k, plan=PLANS[plan])
    L.prepare()
    L.cayley_neumann()
    x0 = cuda.empty(0, case.n, device="cuda")
    y, saved = L.forward(x0)
    dx, dthR, dthP = L.backward(saved, cuda.empty(0, case.m, device="cuda"), x=x0)
    poet.poet_sync_status()
    assert y.shape == (0, case.m) and dx.shape == (0, case.n)
    assert not dthR.any().item() and not dthP.any().item()


@pytest.mark.parametrize("plan", list(PLANS))
def test_resume_is_bit_exact(cuda, plan):
    """Checkpoint and resume: a layer's state is W0, theta_R, theta_P and its
    integers (seed, layer_id, epoch, modes, b, k, plan).  After a step, a
    merge-then-reinitialize and a second parameter change, a new layer built
    from that state reproduces the permutations, the frame copy of W0 and the
    forward output bit for bit."""
    from orthogonal_reparameterized_poet_b200 import poet

    case = Case(640, 512, I.BS, 128, I.FS, 0, 4, 200, I.BF16, 0.02, layer_id=31, epoch=3)
    W0, thR, thP, x, dy = case.arrays()
    tdt = poet.torch_dtype(case.dtype)
    xt, dyt = cuda.from_numpy(x).to("cuda", tdt), cuda.from_numpy(dy).to("cuda", tdt)

    def build(W0d, tR, tP, epoch):
        L = poet.PoetLayer(W0d, tR, tP, mode=case.modeR, b=case.bR, modeP=case.modeP, bP=case.bP, k=case.k,
                           seed=case.seed, layer_id=case.layer_id, epoch=epoch, plan=PLANS[plan])
        L.prepare()
        L.cayley_neumann()
        return L

    L1 = build(cuda.from_numpy(W0).to("cuda", tdt), cuda.from_numpy(thR).cuda(), cuda.from_numpy(thP).cuda(),
               case.epoch)
    _, saved = L1.forward(xt)
    _, dR, dP = L1.backward(saved, dyt, x=xt)
    L1.theta_R.sub_(0.5 * dR)
    L1.theta_P.sub_(0.5 * dP)
    L1.cayley_neumann()
    L1.merge()
    L1.resample()
    L1.theta_R.copy_(cuda.from_numpy(I.theta(5, 0, 0, 0, L1.theta_R.numel(), 0.02)).cuda())
    L1.cayley_neumann()
    y1, _ = L1.forward(xt)
    poet.poet_sync_status()
    # the checkpoint: tensors and integers only
    ck = (L1.W0.clone(), L1.theta_R.clone(), L1.theta_P.clone(), L1.epoch)
    L2 = build(*ck)
    y2, _ = L2.forward(xt)
    poet.poet_sync_status()
    assert L2.epoch == case.epoch + 1
    assert cuda.equal(L2.perm_R, L1.perm_R) and cuda.equal(L2.perm_P, L1.perm_P)
    es = 2 if case.dtype == I.BF16 else 4
    ldn = (case.n + 63) // 64 * 64
    f1 = L1.W0f[: case.m * ldn * es].view(cuda.uint8).reshape(case.m, ldn * es)[:, : case.n * es]
    f2 = L2.W0f[: case.m * ldn * es].view(cuda.uint8).reshape(case.m, ldn * es)[:, : case.n * es]
    assert cuda.equal(f1, f2)
    assert cuda.equal(y1, y2)


# ------------------------------------------------------------------ GEMM engine

GEMM_CASES = [
    # dtype, M, N, K, batch, A major, B major, alpha, beta
    (I.F32, 70, 50, 33, 2, "k", "k", 1.0, 0.0),
    (I.F32, 64, 64, 64, 1, "m", "n", -0.5, 1.0),
    (I.BF16, 300, 260, 200, 1, "k", "k", 1.0, 0.0),
    (I.BF16, 129, 257, 65, 3, "k", "n", 1.0, 0.0),
    (I.BF16, 256, 256, 1000, 2, "m", "n", 1.0, 0.0),
    (I.BF16, 1000, 512, 512, 1, "k", "k", 2.0, 1.0),
    # tensor-core eligible layouts: every operand-major pair, ragged M / N / K
    (I.BF16, 300, 264, 200, 1, "k", "k", 1.0, 0.0),
    (I.BF16, 129, 264, 72, 3, "k", "n", 1.0, 0.0),
    (I.BF16, 136, 256, 136, 2, "m", "k", -1.0, 0.5),
    (I.BF16, 72, 96, 130, 2, "m", "n", 1.0, 0.0),
    (I.BF16, 64, 40, 8, 1, "k", "k", 1.0, 0.0),
    (I.BF16, 2048, 1536, 2048, 1, "k", "k", 1.0, 0.0),
    (I.BF16, 2048, 1536, 2048, 1, "k", "n", 1.0, 0.0),
    # output rows that are not 16-byte aligned (odd N = row stride), several N tiles
    (I.BF16, 520, 777, 96, 1, "k", "k", 1.0, 0.0),
    (I.BF16, 136, 515, 64, 2, "m", "k", -1.0, 0.0),
    (I.BF16, 1100, 5461, 128, 1, "k", "k", 1.0, 0.0),
]


def test_tensor_core_engine_is_live(cuda):
    from orthogonal_reparameterized_poet_b200 import poet

    assert poet.poet_gemm_engine(I.BF16) == 1
    assert poet.poet_gemm_engine(I.F32) == 0


def test_trace_splits_launches_at_the_ridge(cuda):
    """The per-kind trace holds each launch to its own bound: a K = 4096 bf16
    product (about 1000 flop per byte) lands in flop_tc, the AdamW pass (no
    flops) in bytes_hbm, and a ridge above every launch moves the product's
    bytes to bytes_hbm."""
    from orthogonal_reparameterized_poet_b200 import poet

    M = N = 512
    K = 4096
    A = cuda.randn(M, K, device="cuda").to(cuda.bfloat16)
    B = cuda.randn(N, K, device="cuda").to(cuda.bfloat16)
    C = cuda.empty(M, N, device="cuda", dtype=cuda.bfloat16)
    theta, grad, m, v = (cuda.zeros(4096, device="cuda") for _ in range(4))
    try:
        poet.poet_trace_set_ridge(216.0)
        poet.poet_trace_enable(True)
        poet.poet_gemm(I.BF16, M, N, K, 1, A, (K, 1, M * K), B, (K, 1, N * K), C, N, M * N)
        poet.poet_adamw_step(theta, grad, m, v, 1e-3)
        rows = poet.poet_trace_read()
        poet.poet_trace_set_ridge(1e9)
        poet.poet_gemm(I.BF16, M, N, K, 1, A, (K, 1, M * K), B, (K, 1, N * K), C, N, M * N)
        high = poet.poet_trace_read()
    finally:
        poet.poet_trace_enable(False)
        poet.poet_trace_set_ridge(216.0)
    poet.poet_sync_status()
    g, a, h = rows["gemm"], rows["adamw"], high["gemm"]
    assert g["launches"] == 1 and g["flop"] == 2.0 * M * N * K and g["flop_tc"] == g["flop"] and g["bytes_hbm"] == 0
    assert a["flop"] == 0 and a["flop_tc"] == 0 and a["bytes_hbm"] == a["bytes"] > 0
    assert h["flop_tc"] == 0 and h["bytes_hbm"] == h["bytes"] == g["bytes"] > 0
    assert g["ms"] > 0 and a["ms"] > 0


@pytest.mark.parametrize("dtype,M,N,K,batch,amaj,bmaj,alpha,beta", GEMM_CASES)
def test_gemm_engine(cuda, dtype, M, N, K, batch, amaj, bmaj, alpha, beta):
    from orthogonal_reparameterized_poet_b200 import poet

    rng = np.random.default_rng(M * 7 + N)
    tdt = poet.torch_dtype(dtype)
    A = I.to_storage(rng.standard_normal((batch, M, K)).astype(np.float32), dtype)
    B = I.to_storage(rng.standard_normal((batch, N, K)).astype(np.float32), dtype)
    C0 = I.to_storage(rng.standard_normal((batch, M, N)).astype(np.float32), dtype)
    # device layouts: "k" = row-major [M][K] (K contiguous), "m"/"n" = [K][M] (M contiguous)
    Ad = cuda.from_numpy(A if amaj == "k" else np.ascontiguousarray(A.transpose(0, 2, 1))).to("cuda", tdt)
    Bd = cuda.from_numpy(B if bmaj == "k" else np.ascontiguousarray(B.transpose(0, 2, 1))).to("cuda", tdt)
    sA = (K, 1, M * K) if amaj == "k" else (1, M, M * K)
    sB = (K, 1, N * K) if bmaj == "k" else (1, N, N * K)
    C = cuda.from_numpy(C0).to("cuda", tdt)
    poet.poet_gemm(dtype, M, N, K, batch, Ad, sA, Bd, sB, C, N, M * N, alpha, beta)
    poet.poet_sync_status()
    ref = alpha * np.einsum("bmk,bnk->bmn", A.astype(np.float64), B.astype(np.float64)) + beta * C0
    assert rel_fro(C.float().cpu().numpy(), ref) <= (1e-5 if dtype == I.F32 else 8e-3)


# ------------------------------------------------------------------ many layers at once

def _make_layer(cuda, case, plan=0):
    from orthogonal_reparameterized_poet_b200 import poet

    W0, thR, thP, x, dy = case.arrays()
    tdt = poet.torch_dtype(case.dtype)
    L = poet.PoetLayer(cuda.from_numpy(W0).to("cuda", tdt), cuda.from_numpy(thR).cuda(), cuda.from_numpy(thP).cuda(),
                       mode=case.modeR, b=case.bR, modeP=case.modeP, bP=case.bP, k=case.k, seed=case.seed,
                       layer_id=case.layer_id, plan=plan)
    L.prepare()
    return L, cuda.from_numpy(x).to("cuda", tdt), cuda.from_numpy(dy).to("cuda", tdt), (W0, thR, thP, x, dy)


MANY_SETS = {  # different sizes, modes and Neumann orders in one call
    "bf16": [
        Case(512, 512, I.FS, 0, I.FS, 0, 4, 300, I.BF16, 0.02, layer_id=21),
        Case(1376, 512, I.FS, 0, I.FS, 0, 4, 300, I.BF16, 0.02, layer_id=22),
        Case(1024, 768, I.BS, 256, I.BS, 256, 4, 300, I.BF16, 0.02, layer_id=23),
        Case(640, 512, I.BS, 128, I.FS, 0, 2, 300, I.BF16, 0.03, layer_id=24),
    ],
    "f32": [  # odd sizes (ragged tiles), k = 3, 1 and 0
        Case(301, 200, I.FS, 0, I.BS, 48, 3, 130, I.F32, 0.03, layer_id=25),
        Case(200, 301, I.BS, 64, I.FS, 0, 1, 130, I.F32, 0.03, layer_id=26),
        Case(96, 130, I.FS, 0, I.FS, 0, 0, 130, I.F32, 0.03, layer_id=27),
    ],
}
# The grouped gradient computes (I + Q)^T G from the operand copy of G and
# sums its partial products in another order than the one-side path, so the
# two agree to a few roundings of the operand type.
MANY_VS_SINGLE = {"bf16": 5e-3, "f32": 1e-5}


@pytest.mark.parametrize("plan", list(PLANS))
@pytest.mark.parametrize("which", sorted(MANY_SETS))
def test_many_sides_match_single_calls_and_oracle(cuda, which, plan):
    from orthogonal_reparameterized_poet_b200 import poet

    MANY_CASES = MANY_SETS[which]
    built = [_make_layer(cuda, c, PLANS[plan]) for c in MANY_CASES]
    layers = [b[0] for b in built]
    # a1: grouped launch vs one call per side (same tiles, same order: bitwise equal)
    poet.cayley_neumann_many(layers)
    many_R = [L.state_R.clone() for L in layers]
    for L in layers:
        L.cayley_neumann()
    for L, r in zip(layers, many_R):
        n = poet.poet_block_grad_bytes(L.struct.R) // 4 * (2 if L.dtype == I.BF16 else 4)  # all of B
        assert cuda.equal(L.state_R[:n], r[:n])
    # a5..a8 split: backward_blocks + grouped a8 vs poet_backward, and both vs the oracle
    G, dth, dth_ref = [], [], []
    for (L, xt, dyt, arrs), case in zip(built, MANY_CASES):
        y, saved = L.forward(xt)
        gR, gP = L.block_grad_buffers()
        dx = L.backward_blocks(saved, dyt, gR, gP, x=xt)
        G.append((gR, gP))
        dth.append((cuda.empty_like(L.theta_R), cuda.empty_like(L.theta_P)))
        dx1, dR1, dP1 = L.backward(saved, dyt, x=xt)
        assert cuda.equal(dx, dx1)
        dth_ref.append((dR1, dP1))
    ws = cuda.empty(max(poet.cayley_neumann_grad_many_workspace_bytes(layers), 1), dtype=cuda.uint8, device="cuda")
    poet.cayley_neumann_grad_many(layers, G, dth, ws)
    poet.poet_sync_status()
    for (L, xt, dyt, arrs), case, (dR, dP), (dR1, dP1) in zip(built, MANY_CASES, dth, dth_ref):
        ref = run_oracle(case, *arrs)
        tol = TOL[case.dtype]
        assert rel_fro(dR.cpu().numpy(), ref["dthetaR"]) <= tol
        assert rel_fro(dP.cpu().numpy(), ref["dthetaP"]) <= tol
        assert rel_fro(dR.cpu().numpy(), dR1.cpu().numpy()) <= MANY_VS_SINGLE[which]
        assert rel_fro(dP.cpu().numpy(), dP1.cpu().numpy()) <= MANY_VS_SINGLE[which]


# ------------------------------------------------------------------ optimizer step (adjacent)

@pytest.mark.parametrize("n,offset", [(1, 0), (13, 0), (4099, 1), (1000003, 0), (1000003, 3)])
def test_adamw_step_matches_oracle(cuda, n, offset):
    """Three AdamW steps on the device against the float64 oracle; offset > 0
    makes the buffers only 4-byte aligned (the scalar kernel)."""
    from orthogonal_reparameterized_poet_b200 import poet

    rng = np.random.default_rng(n + offset)
    theta0 = (0.02 * rng.standard_normal(n)).astype(np.float32)
    grads = [rng.standard_normal(n).astype(np.float32) for _ in range(3)]
    # the ABI takes float32 hyperparameters: the oracle gets the same rounded values
    lr, b1, b2, eps, wd = (float(np.float32(h)) for h in (1e-3, 0.9, 0.999, 1e-8, 0.01))

    def dev(a):
        buf = cuda.zeros(n + offset, dtype=cuda.float32, device="cuda")
        buf[offset:] = cuda.from_numpy(a).cuda()
        return buf, buf[offset:]

    (_, th), (_, m), (_, v) = dev(theta0), dev(np.zeros(n, np.float32)), dev(np.zeros(n, np.float32))
    ref = (theta0.astype(np.float64), np.zeros(n), np.zeros(n))
    for step, g in enumerate(grads, start=1):
        _, gd = dev(g)
        poet.poet_adamw_step(th, gd, m, v, lr, b1, b2, eps, wd, step)
        # the oracle takes the same float32 inputs (theta and moments as the device holds them)
        ref = O.adamw_step(ref[0], g.astype(np.float64), ref[1], ref[2], lr, b1, b2, eps, wd, step)
    poet.poet_sync_status()
    assert rel_fro(th.cpu().numpy(), ref[0]) <= 1e-6
    assert rel_fro(m.cpu().numpy(), ref[1]) <= 1e-6
    assert rel_fro(v.cpu().numpy(), ref[2]) <= 1e-6


# ------------------------------------------------------------------ grouped forward / backward of many layers

GROUPED_SETS = {
    "bf16": [  # (case, plan): FS and BS, leftover indices, an FS side whose covered width is not a 16-byte
               # column offset (199 -> 99), sides without primitives, and token- and weight-plan layers in one list
        (Case(512, 512, I.FS, 0, I.FS, 0, 4, 300, I.BF16, 0.02, layer_id=41), 2),
        (Case(1376, 512, I.FS, 0, I.FS, 0, 4, 300, I.BF16, 0.02, layer_id=42), 2),
        (Case(1024, 768, I.BS, 256, I.BS, 256, 4, 300, I.BF16, 0.02, layer_id=43), 2),
        (Case(300, 200, I.BS, 64, I.BS, 64, 2, 300, I.BF16, 0.05, layer_id=44), 2),
        (Case(301, 199, I.FS, 0, I.FS, 0, 3, 300, I.BF16, 0.03, layer_id=45), 2),
        (Case(200, 341, I.BS, 64, I.FS, 0, 4, 300, I.BF16, 0.03, layer_id=46), 2),
        (Case(40, 24, I.BS, 64, I.BS, 64, 2, 300, I.BF16, 0.05, layer_id=47), 2),
        (Case(640, 512, I.BS, 128, I.FS, 0, 2, 300, I.BF16, 0.03, layer_id=48), 1),
        (Case(512, 384, I.FS, 0, I.BS, 128, 4, 300, I.BF16, 0.02, layer_id=49), 0),
        (Case(256, 200, I.BS, 32, I.BS, 16, 3, 300, I.BF16, 0.03, layer_id=50), 2),
    ],
    "f32": [
        (Case(301, 200, I.FS, 0, I.BS, 48, 3, 130, I.F32, 0.03, layer_id=51), 2),
        (Case(200, 301, I.BS, 64, I.FS, 0, 1, 130, I.F32, 0.03, layer_id=52), 2),
        (Case(96, 130, I.FS, 0, I.FS, 0, 0, 130, I.F32, 0.03, layer_id=53), 1),
    ],
}


@pytest.mark.parametrize("strided", [False, True])
@pytest.mark.parametrize("which", sorted(GROUPED_SETS))
def test_grouped_forward_backward_match_single_calls_and_oracle(cuda, which, strided):
    """poet_forward_many / poet_backward_blocks_many against the single-layer
    calls and the oracle.  strided: every activation lives in a wider row
    (x: odd stride, so it is re-strided; y and dx: odd strides, written by the
    unaligned epilogue; dy: a 16-byte aligned stride, read in place)."""
    from orthogonal_reparameterized_poet_b200 import poet

    sets = GROUPED_SETS[which]
    T = sets[0][0].T
    built = [_make_layer(cuda, c, plan) for c, plan in sets]
    layers = [b[0] for b in built]
    poet.cayley_neumann_many(layers)
    tdt = poet.torch_dtype(sets[0][0].dtype)

    def strided_copy(t, extra):
        if not strided:
            return t.clone()
        buf = cuda.zeros(t.shape[0], t.shape[1] + extra, dtype=t.dtype, device="cuda")
        buf[:, : t.shape[1]] = t
        return buf[:, : t.shape[1]]

    xs = [strided_copy(b[1], 5) for b in built]
    dys = [strided_copy(b[2], 8) for b in built]
    ys = [strided_copy(cuda.zeros(T, c.m, dtype=tdt, device="cuda"), 3) for c, _ in sets]
    dxs = [strided_copy(cuda.zeros(T, c.n, dtype=tdt, device="cuda"), 1) for c, _ in sets]
    saved = [L.saved_buffer(T) for L in layers]
    Gs = [L.block_grad_buffers() for L in layers]
    ws = cuda.empty(max(poet.many_workspace_bytes(layers, T, dys), 1), dtype=cuda.uint8, device="cuda")
    poet.forward_many(layers, xs, ys, saved, ws)
    poet.backward_blocks_many(layers, xs, saved, dys, dxs, Gs, ws)
    poet.poet_sync_status()
    tol = TOL[sets[0][0].dtype]
    for (L, xt, dyt, arrs), (case, plan), y, dx, (gR, gP) in zip(built, sets, ys, dxs, Gs):
        y1, sv1 = L.forward(xt)
        g1R, g1P = L.block_grad_buffers()
        dx1 = L.backward_blocks(sv1, dyt, g1R, g1P, x=xt)
        poet.poet_sync_status()
        assert rel_fro(y.float().cpu().numpy(), y1.float().cpu().numpy()) <= 1e-5
        assert rel_fro(dx.float().cpu().numpy(), dx1.float().cpu().numpy()) <= 1e-5
        ref = run_oracle(case, *arrs)
        assert rel_fro(y.float().cpu().numpy(), ref["Y"]) <= tol
        assert rel_fro(dx.float().cpu().numpy(), ref["dX"]) <= tol
        for g, g1, (nprim, size), key in ((gR, g1R, L.geom_R, "G_R"), (gP, g1P, L.geom_P, "G_P")):
            if nprim == 0:
                continue
            ld = (size + 7) // 8 * 8
            got = g[: nprim * ld * ld].reshape(nprim, ld, ld)[:, :size, :size].cpu().numpy()
            one = g1[: nprim * ld * ld].reshape(nprim, ld, ld)[:, :size, :size].cpu().numpy()
            assert rel_fro(got, one) <= MANY_VS_SINGLE[which]
            assert rel_fro(got, ref[key]) <= tol, (case, key)


def test_grouped_backward_with_no_tokens_zeroes_the_gradients(cuda):
    from orthogonal_reparameterized_poet_b200 import poet

    sets = GROUPED_SETS["bf16"][:3]
    layers = [_make_layer(cuda, c, plan)[0] for c, plan in sets]
    poet.cayley_neumann_many(layers)
    Gs = [L.block_grad_buffers() for L in layers]
    for gR, gP in Gs:
        gR.fill_(1.0)
        gP.fill_(1.0)
    ws = cuda.empty(max(poet.many_workspace_bytes(layers, 0), 1), dtype=cuda.uint8, device="cuda")
    e = [cuda.empty(0, L.m, dtype=cuda.bfloat16, device="cuda") for L in layers]
    f = [cuda.empty(0, L.n, dtype=cuda.bfloat16, device="cuda") for L in layers]
    poet.backward_blocks_many(layers, f, [L.saved_buffer(0) for L in layers], e, f, Gs, ws)
    poet.poet_sync_status()
    for (gR, gP), L in zip(Gs, layers):
        nR, sR = L.geom_R
        nP, sP = L.geom_P
        assert not gR[: nR * ((sR + 7) // 8 * 8) ** 2].any().item()
        assert not gP[: nP * ((sP + 7) // 8 * 8) ** 2].any().item()


# ------------------------------------------------------------------ a8 with the AdamW step fused

@pytest.mark.parametrize("which", sorted(MANY_SETS))
def test_fused_adamw_matches_separate_step_and_oracle(cuda, which):
    """poet_cayley_neumann_grad_many_adamw against poet_cayley_neumann_grad_many
    followed by poet_adamw_step (bitwise: the same gradient and the same update
    arithmetic), and the update against the oracle's AdamW step on the
    oracle's gradient.  Moments start nonzero and step = 3, so that every term
    of the update matters; they are drawn on each side's gradient scale (v0
    about the squared RMS gradient), where the update is a smooth function of
    the gradient.  With moments far below the gradient, m_hat / sqrt(v_hat)
    tends to sign(g) element by element, and the bf16 gradient's rounding flips
    the sign of near-zero elements by a full 2 lr, which no gradient tolerance
    bounds."""
    from orthogonal_reparameterized_poet_b200 import poet

    cases = MANY_SETS[which]
    built = [_make_layer(cuda, c) for c in cases]
    layers = [b[0] for b in built]
    poet.cayley_neumann_many(layers)
    G = []
    for L, xt, dyt, _ in built:
        _, saved = L.forward(xt)
        gR, gP = L.block_grad_buffers()
        L.backward_blocks(saved, dyt, gR, gP, x=xt)
        G.append((gR, gP))
    sides = [s for L in layers for s in (L.struct.R, L.struct.P)]
    Gl = [g for pair in G for g in pair]
    rng = np.random.default_rng(3)
    hp = dict(lr=float(np.float32(1e-3)), beta1=float(np.float32(0.9)), beta2=float(np.float32(0.999)),
              eps=float(np.float32(1e-8)), weight_decay=float(np.float32(0.01)), step=3)
    th0 = [t.clone() for L in layers for t in (L.theta_R, L.theta_P)]
    refs = [run_oracle(case, *b[3]) for b, case in zip(built, cases)]
    scale = [float(np.sqrt(np.mean(r[key] ** 2))) if r[key].size else 1.0
             for r in refs for key in ("dthetaR", "dthetaP")]
    m0 = [cuda.from_numpy((sc * rng.standard_normal(t.numel())).astype(np.float32)).cuda()
          for sc, t in zip(scale, th0)]
    v0 = [cuda.from_numpy((sc * sc * (0.5 + rng.random(t.numel()))).astype(np.float32)).cuda()
          for sc, t in zip(scale, th0)]
    ws = cuda.empty(max(poet.cayley_neumann_grad_many_workspace_bytes(layers), 1), dtype=cuda.uint8, device="cuda")
    # separate: gradient, then the optimizer kernel
    dth = [cuda.empty_like(t) for t in th0]
    poet.poet_cayley_neumann_grad_many(sides, Gl, dth, layers[0].dtype, ws)
    th_a, m_a, v_a = [t.clone() for t in th0], [t.clone() for t in m0], [t.clone() for t in v0]
    for t, g, m, v in zip(th_a, dth, m_a, v_a):
        if t.numel():
            poet.poet_adamw_step(t, g, m, v, **hp)
    # fused: the sides' own theta is updated in place
    m_b, v_b = [t.clone() for t in m0], [t.clone() for t in v0]
    dth_b = [cuda.full_like(t, float("nan")) for t in th0]
    poet.poet_cayley_neumann_grad_many_adamw(sides, Gl, m_b, v_b, layers[0].dtype, ws, dtheta=dth_b, **hp)
    poet.poet_sync_status()
    th_b = [t for L in layers for t in (L.theta_R, L.theta_P)]
    for a, b in zip(dth, dth_b):
        assert cuda.equal(a, b)
    for a, b in zip(th_a, th_b):
        assert cuda.equal(a, b)
    for a, b in zip(m_a + v_a, m_b + v_b):
        assert cuda.equal(a, b)
    # the update against the oracle's AdamW step on the oracle's gradient
    for case, ref, i in zip(cases, refs, range(len(cases))):
        for s, key in ((0, "dthetaR"), (1, "dthetaP")):
            k = 2 * i + s
            if not th0[k].numel():
                continue
            t_ref, m_ref, _ = O.adamw_step(th0[k].double().cpu().numpy(), ref[key], m0[k].double().cpu().numpy(),
                                           v0[k].double().cpu().numpy(), **hp)
            d_got = (th_b[k].double() - th0[k].double()).cpu().numpy()
            assert rel_fro(d_got, t_ref - th0[k].double().cpu().numpy()) <= TOL[case.dtype]
            assert rel_fro(m_b[k].cpu().numpy(), m_ref) <= TOL[case.dtype]


def test_merge_reset_moments(cuda):
    """poet_merge_reset_moments: the merge of poet_merge (bitwise, on an
    identical layer), theta reset, and the moments of both sides zero."""
    from orthogonal_reparameterized_poet_b200 import poet

    case = MANY_SETS["bf16"][2]
    L1, _, _, _ = _make_layer(cuda, case)
    L2, _, _, _ = _make_layer(cuda, case)
    for L in (L1, L2):
        L.cayley_neumann()
    mR, vR = cuda.ones_like(L1.theta_R), cuda.ones_like(L1.theta_R)
    mP, vP = cuda.ones_like(L1.theta_P), cuda.ones_like(L1.theta_P)
    L1.merge()
    poet.poet_merge_reset_moments(L2.struct, mR, vR, mP, vP, L2.workspace(0))
    poet.poet_sync_status()
    assert cuda.equal(L1.W0, L2.W0)
    assert not L2.theta_R.any().item() and not L2.theta_P.any().item()
    for t in (mR, vR, mP, vP):
        assert not t.any().item()

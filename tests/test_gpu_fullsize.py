"""Parity at full size, on the LLaMA-350M (block-stochastic b=256, 16384
tokens), LLaMA-1.3B (fully stochastic and block-stochastic b=256, 32768
tokens) and LLaMA-3B (fully stochastic, 16384 tokens) layer sets: the square
(q), wide (gate) and tall (down) shapes of the first, middle and last layer,
built from the same seeded inputs bench.py draws and run through the same
grouped calls it times (poet_cayley_neumann_many, poet_forward,
poet_backward_blocks, poet_cayley_neumann_grad_many, then poet_merge).

The oracle cannot afford a whole layer at this size, so it computes sampled
outputs one by one from their definitions:
  * y and dx on 16 sampled tokens (per-token products through the primitives);
  * dtheta of sampled primitives, whose block gradient sums over every token
    (only the primitive's own columns of v = W0 P x or du = W0^T R^T dy are
    formed);
  * sampled rows of the merged W0;
  * every permutation, bit-exact.
Fully stochastic primitives larger than 1280 (2730 at LLaMA-1.3B, 3456 at
LLaMA-3B) cost seconds of float64 CPU time each: their dtheta is compared in
the cases marked full_dtheta and checked through y, dx and the merge in the
others."""
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


# (variant, linear, layer, full_dtheta): q, gate and down of the first, middle and last layer
CASES = [("llama1.3b_fs", 0, 0, False), ("llama1.3b_fs", 4, 0, True), ("llama1.3b_fs", 6, 0, False),
         ("llama1.3b_fs", 4, 23, False),
         ("llama1.3b_bs256", 0, 0, False), ("llama1.3b_bs256", 4, 0, False), ("llama1.3b_bs256", 6, 0, False),
         ("llama350m_bs256", 0, 0, False), ("llama350m_bs256", 4, 0, False), ("llama350m_bs256", 6, 0, False),
         ("llama350m_bs256", 0, 12, False), ("llama350m_bs256", 4, 12, False), ("llama350m_bs256", 6, 12, False),
         ("llama350m_bs256", 0, 23, False), ("llama350m_bs256", 4, 23, False), ("llama350m_bs256", 6, 23, False),
         ("llama3b_fs", 0, 0, False), ("llama3b_fs", 4, 0, True), ("llama3b_fs", 6, 0, True),
         ("llama3b_fs", 0, 16, False), ("llama3b_fs", 4, 16, False), ("llama3b_fs", 6, 16, False),
         ("llama3b_fs", 0, 31, False), ("llama3b_fs", 4, 31, False), ("llama3b_fs", 6, 31, False)]
# auto: the plan bench.py runs at these sizes (the weight plan); token: the other one, on the first layer
PLANS = {"auto": 0, "token": 1}
PARAMS = [(c, p) for c in CASES for p in PLANS if p == "auto" or c[2] == 0]
DTHETA_MAX_SIZE = 1280  # larger fully stochastic primitives: only where full_dtheta


_ACT = {}


def _activations(wl, d, grad):
    """x or dy of width d exactly as bench.py draws them on rank 0 (shared by every layer of that width)."""
    key = (wl.seed, d, wl.tokens, wl.dtype, grad)
    if key not in _ACT:
        if len(_ACT) >= 4:
            _ACT.clear()
        _ACT[key] = I.activations(wl.seed, d, wl.tokens, d, wl.dtype, grad=grad)
    return _ACT[key]


@pytest.mark.parametrize("case,plan", PARAMS, ids=[f"{c[0]}-{c[1]}-{c[2]}-{p}" for c, p in PARAMS])
def test_fullsize_sampled_parity(cuda, case, plan):
    from orthogonal_reparameterized_poet_b200 import poet

    name, linear, layer, full_dtheta = case
    wl = I.WORKLOADS[name]
    T, k, dt = wl.tokens, wl.k, wl.dtype
    m, n = wl.linear_shapes()[linear]
    layer_id = layer * len(wl.linear_shapes()) + linear
    nR, sR = O.side_shape(m, wl.mode, wl.b)
    nP, sP = O.side_shape(n, wl.mode, wl.b)
    # inputs exactly as bench.py draws them (rank 0)
    W0 = I.w0(wl.seed, layer, linear, m, n, dt)
    thR = I.theta(wl.seed, layer, linear, 0, nR * O.n_skew(sR), wl.sigma)
    thP = I.theta(wl.seed, layer, linear, 1, nP * O.n_skew(sP), wl.sigma)
    X = _activations(wl, n, False)
    dY = _activations(wl, m, True)

    # ---------------- CUDA path, bench launch configuration
    tdt = poet.torch_dtype(dt)
    L = poet.PoetLayer(cuda.from_numpy(W0).to("cuda", tdt), cuda.from_numpy(thR).cuda(), cuda.from_numpy(thP).cuda(),
                       mode=wl.mode, b=wl.b, k=k, seed=wl.seed, layer_id=layer_id, plan=PLANS[plan])
    assert L.plan_for(T) == (poet.PLAN_WEIGHT if plan == "auto" else poet.PLAN_TOKEN)
    L.prepare()
    poet.cayley_neumann_many([L])
    xt = cuda.from_numpy(X).to("cuda", tdt)
    dyt = cuda.from_numpy(dY).to("cuda", tdt)
    y, saved = L.forward(xt)
    gR, gP = L.block_grad_buffers()
    dx = L.backward_blocks(saved, dyt, gR, gP, x=xt)
    dthR, dthP = cuda.empty_like(L.theta_R), cuda.empty_like(L.theta_P)
    ws = cuda.empty(max(poet.cayley_neumann_grad_many_workspace_bytes([L]), 1), dtype=cuda.uint8, device="cuda")
    poet.cayley_neumann_grad_many([L], [(gR, gP)], [(dthR, dthP)], ws)
    poet.poet_sync_status()
    permR_gpu, permP_gpu = L.perm_R.cpu().numpy(), L.perm_P.cpu().numpy()
    rows = np.random.default_rng(linear).choice(T, 16, replace=False)
    y_s = y[rows].float().cpu().numpy()
    dx_s = dx[rows].float().cpu().numpy()
    dthR, dthP = dthR.cpu().numpy(), dthP.cpu().numpy()
    del y, dx, saved, xt, dyt, gR, gP, ws
    L.merge()
    wrows = np.random.default_rng(100 + linear).choice(m, 12, replace=False)
    W0m = L.W0[wrows].float().cpu().numpy()
    del L

    # ---------------- oracle, sampled
    permR = O.draw_perm(wl.seed, layer_id, 0, 0, m)
    permP = O.draw_perm(wl.seed, layer_id, 1, 0, n)
    assert np.array_equal(permR_gpu, permR) and np.array_equal(permP_gpu, permP)
    Rb = O.cayley_neumann(thR.astype(np.float64), nR, sR, k)
    Pb = O.cayley_neumann(thP.astype(np.float64), nP, sP, k)
    RbT, PbT = Rb.transpose(0, 2, 1), Pb.transpose(0, 2, 1)
    W0d = W0.astype(np.float64)
    tol = TOL[dt]
    # y = R W0 P x and dx = P^T W0^T R^T dy on the sampled tokens
    y_ref = O.apply_side_rows(O.apply_side_rows(X[rows], permP, Pb, wl.mode, wl.b) @ W0d.T, permR, Rb, wl.mode, wl.b)
    dx_ref = O.apply_side_rows(O.apply_side_rows(dY[rows], permR, RbT, wl.mode, wl.b) @ W0d, permP, PbT,
                               wl.mode, wl.b)
    assert rel_fro(y_s, y_ref) <= tol
    assert rel_fro(dx_s, dx_ref) <= tol
    # dtheta of sampled primitives (block gradient over all tokens)
    rng = np.random.default_rng(7)
    if sP <= DTHETA_MAX_SIZE or full_dtheta:
        dV = O.apply_side_rows(dY, permR, RbT, wl.mode, wl.b)  # R^T dy for every token
        for j in sorted(rng.choice(nP, min(2, nP), replace=False)):
            J = permP[j * sP:(j + 1) * sP]
            dU_J = dV @ W0d[:, J]                                 # (W0^T R^T dy) on the primitive's columns
            G = dU_J.T @ X[:, J].astype(np.float64)
            per = O.n_skew(sP)
            ref = O.theta_grad_block(G, thP[j * per:(j + 1) * per].astype(np.float64), sP, k)
            assert rel_fro(dthP[j * per:(j + 1) * per], ref) <= tol
        del dV
    if sR <= DTHETA_MAX_SIZE or full_dtheta:
        U = O.apply_side_rows(X, permP, Pb, wl.mode, wl.b)         # P x for every token
        for j in sorted(rng.choice(nR, min(2, nR), replace=False)):
            Iset = permR[j * sR:(j + 1) * sR]
            V_I = U @ W0d[Iset, :].T                                 # (W0 P x) on the primitive's rows
            G = dY[:, Iset].astype(np.float64).T @ V_I
            per = O.n_skew(sR)
            ref = O.theta_grad_block(G, thR[j * per:(j + 1) * per].astype(np.float64), sR, k)
            assert rel_fro(dthR[j * per:(j + 1) * per], ref) <= tol
    # merged W0 on sampled rows: (R W0 P)[i, :]
    R_rows = np.zeros((len(wrows), m))
    for r_i, i in enumerate(wrows):
        e = np.zeros((1, m))
        e[0, i] = 1.0
        R_rows[r_i] = O.apply_side_rows(e, permR, RbT, wl.mode, wl.b)[0]  # row i of R = e_i^T R
    W0m_ref = O.apply_side_rows(R_rows @ W0d, permP, PbT, wl.mode, wl.b)  # ... then times P
    assert rel_fro(W0m, W0m_ref) <= tol

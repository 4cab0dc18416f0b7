"""One LLaMA block around seven POET linears (poet_llama_block_forward /
_backward, then the grouped a8) against the float64 oracle of the block
(oracle/llama_block.py) on the same seeded bf16 inputs: the output, dh and
every linear's packed-skew gradients, at LLaMA-60M shapes (hidden 512, FFN
1376, 8 heads of 64, two sequences of 256 tokens).  Bar: relative Frobenius
error <= 2e-2 (bf16)."""
import numpy as np
import pytest

from oracle import llama_block as LB
from oracle import poet_oracle as O
from orthogonal_reparameterized_poet_b200 import inputs as I
from tests.harness import TOL, rel_fro

pytestmark = pytest.mark.gpu

HIDDEN, FFN, HEADS, HEAD_DIM, SEQ, NSEQ = 512, 1376, 8, 64, 256, 2


@pytest.fixture(scope="module")
def cuda():
    import torch

    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from orthogonal_reparameterized_poet_b200 import poet

    poet.lib()
    return torch


def _build(cuda, mode, b, plan, seed=3):
    from orthogonal_reparameterized_poet_b200 import poet

    dims = [(HIDDEN, HIDDEN)] * 4 + [(FFN, HIDDEN)] * 2 + [(HIDDEN, FFN)]
    gpu, ref = [], {}
    for t, (name, (m, n)) in enumerate(zip(LB.LINEARS, dims)):
        nR, sR = O.side_shape(m, mode, b)
        nP, sP = O.side_shape(n, mode, b)
        W0 = I.w0(seed, 0, t, m, n, I.BF16)
        thR = I.theta(seed, 0, t, 0, nR * O.n_skew(sR), 0.02)
        thP = I.theta(seed, 0, t, 1, nP * O.n_skew(sP), 0.02)
        L = poet.PoetLayer(cuda.from_numpy(W0).to("cuda", cuda.bfloat16), cuda.from_numpy(thR).cuda(),
                           cuda.from_numpy(thP).cuda(), mode=mode, b=b, k=4, seed=seed, layer_id=t, plan=plan)
        L.prepare()
        gpu.append(L)
        permR, permP = O.draw_perm(seed, t, 0, 0, m), O.draw_perm(seed, t, 1, 0, n)
        ref[name] = LB.PoetLinear(W0.astype(np.float64), thR.astype(np.float64), thP.astype(np.float64), permR,
                                  permP, mode, b, 4)
    poet.cayley_neumann_many(gpu)
    return gpu, ref


@pytest.mark.parametrize("mode,b,plan", [(I.BS, 256, 2), (I.FS, 0, 1), (I.FS, 0, 0), (I.BS, 32, 1)])
def test_llama_block_matches_oracle(cuda, mode, b, plan):
    from orthogonal_reparameterized_poet_b200 import poet

    T = NSEQ * SEQ
    layers, ref = _build(cuda, mode, b, plan)
    for L, name in zip(layers, LB.LINEARS):  # the permutations the oracle uses
        assert np.array_equal(L.perm_R.cpu().numpy(), ref[name].permR)
        assert np.array_equal(L.perm_P.cpu().numpy(), ref[name].permP)
    blk = poet.PoetBlock(layers, SEQ, HEADS, HEAD_DIM)
    h = I.activations(5, HIDDEN, T, HIDDEN, I.BF16)
    dout = I.activations(5, HIDDEN, T, HIDDEN, I.BF16, grad=True)
    ht = cuda.from_numpy(h).to("cuda", cuda.bfloat16)
    dt = cuda.from_numpy(dout).to("cuda", cuda.bfloat16)
    out, saved = blk.forward(ht)
    dh, G = blk.backward(saved, dt)
    dth = blk.theta_grads(G)
    poet.poet_sync_status()

    shape = LB.BlockShape(HIDDEN, FFN, HEADS, HEAD_DIM, SEQ)
    out_ref, cache = LB.block_forward(h.astype(np.float64), ref, shape)
    dh_ref, dth_ref = LB.block_backward(dout.astype(np.float64), ref, cache, shape)
    tol = TOL[I.BF16]
    errs = {"out": rel_fro(out.float().cpu().numpy(), out_ref), "dh": rel_fro(dh.float().cpu().numpy(), dh_ref)}
    for (dR, dP), name in zip(dth, LB.LINEARS):
        if dR.numel():
            errs[name + ".R"] = rel_fro(dR.cpu().numpy(), dth_ref[name][0])
        if dP.numel():
            errs[name + ".P"] = rel_fro(dP.cpu().numpy(), dth_ref[name][1])
    bad = {k: v for k, v in errs.items() if not v <= tol}
    assert not bad, f"{bad} (tol {tol}); all: {errs}"


def test_llama_block_rejects_bad_shapes(cuda):
    from orthogonal_reparameterized_poet_b200 import poet

    layers, _ = _build(cuda, I.BS, 256, 0)
    with pytest.raises(poet.PoetError):
        poet.PoetBlock(layers, 250, HEADS, HEAD_DIM).forward(cuda.zeros(500, HIDDEN, dtype=cuda.bfloat16,
                                                                        device="cuda"))
    with pytest.raises(poet.PoetError):
        poet.PoetBlock(layers, SEQ, 6, HEAD_DIM).forward(cuda.zeros(SEQ, HIDDEN, dtype=cuda.bfloat16, device="cuda"))

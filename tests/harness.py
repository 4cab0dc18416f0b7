"""Shared test harness: seeded cases, the CUDA path through the binding, the
oracle on the same inputs, and the comparison metric.

The two sides meet only here: the inputs come from the package's seeded
input module, the CUDA results from libpoet (through the binding), the
expected values from oracle/ alone.
"""
from __future__ import annotations

from dataclasses import dataclass

import numpy as np

from oracle import poet_oracle as O
from orthogonal_reparameterized_poet_b200 import inputs as I

TOL = {I.F32: 1e-5, I.BF16: 2e-2}   # relative Frobenius error bar per storage type


def rel_fro(got, ref) -> float:
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    den = np.linalg.norm(ref)
    num = np.linalg.norm(got - ref)
    return float(num / den) if den > 0 else float(num)


@dataclass
class Case:
    m: int
    n: int
    modeR: int
    bR: int
    modeP: int
    bP: int
    k: int
    T: int
    dtype: int
    sigma: float
    seed: int = 0
    layer: int = 0
    linear: int = 0
    layer_id: int = 0
    epoch: int = 0

    def arrays(self):
        nR, sR = O.side_shape(self.m, self.modeR, self.bR)
        nP, sP = O.side_shape(self.n, self.modeP, self.bP)
        W0 = I.w0(self.seed, self.layer, self.linear, self.m, self.n, self.dtype)
        thR = I.theta(self.seed, self.layer, self.linear, 0, nR * O.n_skew(sR), self.sigma)
        thP = I.theta(self.seed, self.layer, self.linear, 1, nP * O.n_skew(sP), self.sigma)
        x = I.activations(self.seed, 1000 * self.layer + self.linear, self.T, self.n, self.dtype)
        dy = I.activations(self.seed, 1000 * self.layer + self.linear, self.T, self.m, self.dtype, grad=True)
        return W0, thR, thP, x, dy


def run_oracle(case: Case, W0, thR, thP, x, dy):
    permR = O.draw_perm(case.seed, case.layer_id, 0, case.epoch, case.m)
    permP = O.draw_perm(case.seed, case.layer_id, 1, case.epoch, case.n)
    out = O.layer_step(W0.astype(np.float64), thR.astype(np.float64), thP.astype(np.float64), permR, permP,
                       case.modeR, case.bR, case.modeP, case.bP, case.k, x.astype(np.float64),
                       dy.astype(np.float64))
    out["permR"], out["permP"] = permR, permP
    return out


def run_gpu(case: Case, W0, thR, thP, x, dy, device="cuda", plan=0):
    """prepare -> Cayley-Neumann -> forward -> backward -> merge -> resample ->
    Cayley-Neumann -> forward, all through libpoet (plan: poet.PLAN_*)."""
    import torch
    from orthogonal_reparameterized_poet_b200 import poet

    tdt = poet.torch_dtype(case.dtype)
    L = poet.PoetLayer(torch.from_numpy(W0).to(device=device, dtype=tdt),
                       torch.from_numpy(thR).to(device), torch.from_numpy(thP).to(device),
                       mode=case.modeR, b=case.bR, modeP=case.modeP, bP=case.bP, k=case.k,
                       seed=case.seed, layer_id=case.layer_id, epoch=case.epoch, plan=plan)
    xt = torch.from_numpy(x).to(device=device, dtype=tdt)
    dyt = torch.from_numpy(dy).to(device=device, dtype=tdt)
    L.prepare()
    L.cayley_neumann()
    y, saved = L.forward(xt)
    dx, dthR, dthP = L.backward(saved, dyt, x=xt)
    poet.poet_sync_status()
    res = {
        "plan": L.plan_for(xt.shape[0]),
        "permR": L.perm_R.cpu().numpy(), "permP": L.perm_P.cpu().numpy(),
        "Y": y.float().cpu().numpy(), "dX": dx.float().cpu().numpy(),
        "dthetaR": dthR.cpu().numpy(), "dthetaP": dthP.cpu().numpy(),
        "R_blocks": read_blocks(L.state_R, L.geom_R, case.dtype),
        "P_blocks": read_blocks(L.state_P, L.geom_P, case.dtype),
    }
    L.merge()
    res["W0_merged"] = L.W0.float().cpu().numpy()
    res["thetaR_after_merge"] = L.theta_R.cpu().numpy()
    L.resample()
    L.cayley_neumann()
    y2, _ = L.forward(xt)
    poet.poet_sync_status()
    res["Y_after_merge"] = y2.float().cpu().numpy()
    res["epoch_after"] = L.epoch
    res["permR_after"] = L.perm_R.cpu().numpy()
    return res


def read_blocks(state, geom, dtype):
    """The materialized primitives at the start of a side state: [nprim][ld][ld], ld = size rounded up to 8."""
    import torch

    nprim, size = geom
    if nprim == 0:
        return np.zeros((0, 0, 0))
    ld = (size + 7) // 8 * 8
    es = 2 if dtype == I.BF16 else 4
    raw = state[: nprim * ld * ld * es]
    t = raw.view(torch.bfloat16 if dtype == I.BF16 else torch.float32).float().reshape(nprim, ld, ld)
    return t[:, :size, :size].cpu().numpy()

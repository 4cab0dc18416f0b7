"""Pin checks for the CPU oracle, written as plain functions so that the same
checks can be re-run against deliberately broken copies of the oracle
(tests/test_oracle_mutations.py) to show that each plausible mistake fails at
least one of them.

Every check compares the oracle with something other than itself: a value
printed on the pages or derived by hand (tests/golden), a closed form, an
exact identity, a library routine for a special case, or brute force.
"""
from __future__ import annotations

import numpy as np

from tests.conftest import load_golden


def _rng(seed):
    return np.random.default_rng(seed)


def _rand_skew_theta(rng, size, scale):
    return rng.standard_normal(size * (size - 1) // 2) * scale


# ---------------------------------------------------------------- packing

def check_unpack_golden(O):
    g = load_golden("skew_pack_b3.json")
    Q = O.unpack_skew(np.array(g["theta"]), g["size"])
    return np.array_equal(Q, np.array(g["Q"]))


# ---------------------------------------------------------------- a1

def check_cnp_2x2_closed_form(O):
    g = load_golden("cnp_2x2.json")
    a = g["a"]
    ok = True
    for k, R_expect in g["R_by_k"].items():
        R = O.cayley_neumann(np.array([a]), 1, 2, int(k))[0]
        ok &= np.allclose(R, np.array(R_expect), rtol=0, atol=1e-15)
    C = O.exact_cayley(O.unpack_skew(np.array([a]), 2))
    ok &= np.allclose(C, np.array(g["exact_cayley"]), rtol=0, atol=1e-15)
    return bool(ok)


def check_cnp_truncation_identity(O, size=12, scale=0.08):
    """||R_k - C||_F = ||Q^(k+1)||_F for every k, since R_k = C (I - Q^(k+1))
    with C orthogonal; and the error shrinks with k when ||Q|| < 1."""
    rng = _rng(1)
    theta = _rand_skew_theta(rng, size, scale)
    Q = O.unpack_skew(theta, size)
    C = np.linalg.solve(np.eye(size) - Q, np.eye(size) + Q)  # independent of O.exact_cayley
    errs = []
    for k in range(0, 7):
        R = O.cayley_neumann(theta, 1, size, k)[0]
        e = np.linalg.norm(R - C)
        expect = np.linalg.norm(np.linalg.matrix_power(Q, k + 1))
        if not np.isclose(e, expect, rtol=1e-9, atol=1e-300):
            return False
        errs.append(e)
    return bool(np.linalg.norm(Q, 2) < 1 and all(errs[i + 1] < errs[i] for i in range(len(errs) - 1)))


def check_orthogonality_identity(O, size=10, scale=0.3):
    """R^T R - I = (I - (-1)^(k+1) Q^(k+1)) (I - Q^(k+1)) - I exactly, and
    ||R^T R - I|| is within the truncation bound."""
    rng = _rng(2)
    theta = _rand_skew_theta(rng, size, scale)
    Q = O.unpack_skew(theta, size)
    I = np.eye(size)
    qn = np.linalg.norm(Q, 2)
    for k in range(0, 6):
        R = O.cayley_neumann(theta, 1, size, k)[0]
        Qk1 = np.linalg.matrix_power(Q, k + 1)
        lhs = R.T @ R - I
        rhs = (I - (-1) ** (k + 1) * Qk1) @ (I - Qk1) - I
        if not np.allclose(lhs, rhs, rtol=0, atol=1e-12):
            return False
        bound = qn ** (2 * k + 2) if k % 2 == 0 else 2 * qn ** (k + 1) + qn ** (2 * k + 2)
        if np.linalg.norm(lhs, 2) > bound * (1 + 1e-9):
            return False
    return True


def check_singular_values_closed_form(O, size=9, scale=0.5):
    """sigma(R) = |1 - lambda^(k+1)| over the eigenvalues lambda of Q."""
    rng = _rng(3)
    theta = _rand_skew_theta(rng, size, scale)
    Q = O.unpack_skew(theta, size)
    lam = np.linalg.eigvals(Q)
    for k in range(0, 5):
        R = O.cayley_neumann(theta, 1, size, k)[0]
        sv = np.sort(np.linalg.svd(R, compute_uv=False))
        expect = np.sort(np.abs(1 - lam ** (k + 1)))
        if not np.allclose(sv, expect, rtol=1e-10, atol=1e-12):
            return False
    return True


def check_special_cases(O):
    rng = _rng(4)
    ok = True
    for k in range(0, 5):  # theta = 0 -> identity for every k
        ok &= np.array_equal(O.cayley_neumann(np.zeros(3 * 28), 3, 8, k), np.broadcast_to(np.eye(8), (3, 8, 8)))
    theta = _rand_skew_theta(rng, 7, 0.2)  # k = 0 -> I + Q
    ok &= np.allclose(O.cayley_neumann(theta, 1, 7, 0)[0], np.eye(7) + O.unpack_skew(theta, 7), atol=1e-15)
    ok &= O.n_skew(1) == 0 and O.n_skew(2) == 1 and O.n_skew(256) == 32640
    return bool(ok)


# ---------------------------------------------------------------- geometry / dense side

def check_dense_side_golden(O):
    g = load_golden("dense_side_d4.json")
    D = O.dense_side(np.array(g["perm"]), np.array(g["blocks"]), O.BS, g["b"])
    return np.array_equal(D, np.array(g["dense"]))


def _apply_side_by_loops(perm, blocks, mode, b, v):
    """Brute force: (Rv)[perm[j*s+a]] = sum_c block_j[a,c] v[perm[j*s+c]]; other indices copied."""
    d = len(perm)
    s = d // 2 if mode == 1 else b
    nprim = 1 if mode == 1 else d // b
    out = list(v)
    for j in range(nprim):
        for a in range(s):
            acc = 0.0
            for c in range(s):
                acc += blocks[j][a][c] * v[perm[j * s + c]]
            out[perm[j * s + a]] = acc
    return np.array(out)


def check_dense_side_vs_loops(O):
    rng = _rng(5)
    for d, mode, b in [(11, 0, 3), (12, 0, 4), (9, 1, 0), (10, 1, 0), (7, 0, 7), (5, 0, 1)]:
        perm = rng.permutation(d)
        nprim, s = O.side_shape(d, mode, b)
        blocks = rng.standard_normal((nprim, s, s))
        D = O.dense_side(perm, blocks, mode, b)
        v = rng.standard_normal(d)
        if not np.allclose(D @ v, _apply_side_by_loops(perm, blocks, mode, b, v), atol=1e-12):
            return False
    return True


def check_apply_side_rows(O):
    """Blockwise application equals brute-force loops on every row."""
    rng = _rng(10)
    for d, mode, b in [(11, 0, 3), (10, 1, 0), (9, 0, 9)]:
        perm = rng.permutation(d)
        nprim, s = O.side_shape(d, mode, b)
        blocks = rng.standard_normal((nprim, s, s))
        X = rng.standard_normal((4, d))
        got = O.apply_side_rows(X, perm, blocks, mode, b)
        for t in range(4):
            if not np.allclose(got[t], _apply_side_by_loops(perm, blocks, mode, b, X[t]), atol=1e-12):
                return False
    return True


def check_side_shapes(O):
    return (O.side_shape(5461, O.BS, 256) == (21, 256) and O.side_shape(5461, O.FS, 0) == (1, 2730)
            and O.side_shape(1376, O.FS, 0) == (1, 688) and O.side_shape(256, O.BS, 32) == (8, 32)
            and O.side_shape(2736, O.BS, 256) == (10, 256))


def check_no_primitive_side(O):
    """b > d: floor(d/b) = 0 primitives, the side is the identity, and the
    layer reduces to the plain product y = W0 x with dx = W0^T dy."""
    rng = _rng(9)
    m, n, b = 7, 5, 8
    W0 = rng.standard_normal((m, n))
    X = rng.standard_normal((3, n))
    dY = rng.standard_normal((3, m))
    out = O.layer_step(W0, np.zeros(0), np.zeros(0), rng.permutation(m), rng.permutation(n), 0, b, 0, b, 2, X, dY)
    return bool(np.allclose(out["Y"], X @ W0.T) and np.allclose(out["dX"], dY @ W0)
                and out["dthetaR"].size == 0 and out["dthetaP"].size == 0
                and np.allclose(out["W0_merged"], W0))


# ---------------------------------------------------------------- spectrum, merge

def check_spectrum_preservation(O, m=12, n=9):
    """sigma(R W0 P) = sigma(W0) with exact Cayley primitives; with the
    truncated series sigma_i(W0) smin(R) smin(P) <= sigma_i(R W0 P) <= sigma_i(W0) smax(R) smax(P)."""
    rng = _rng(6)
    W0 = rng.standard_normal((m, n))
    permR, permP = rng.permutation(m), rng.permutation(n)
    sW = np.linalg.svd(W0, compute_uv=False)
    for mode, b in [(0, 4), (1, 0)]:
        nR, sR = O.side_shape(m, mode, b)
        nP, sP = O.side_shape(n, mode, b)
        thR = _rand_skew_theta(rng, sR, 0.3 / np.sqrt(sR))
        thP = _rand_skew_theta(rng, sP, 0.3 / np.sqrt(sP))
        thR = np.tile(thR, nR)
        thP = np.tile(thP, nP)
        # exact Cayley blocks
        per_R, per_P = O.n_skew(sR), O.n_skew(sP)
        exR = np.stack([np.linalg.solve(np.eye(sR) - O.unpack_skew(thR[j * per_R:(j + 1) * per_R], sR),
                                        np.eye(sR) + O.unpack_skew(thR[j * per_R:(j + 1) * per_R], sR)) for j in range(nR)])
        exP = np.stack([np.linalg.solve(np.eye(sP) - O.unpack_skew(thP[j * per_P:(j + 1) * per_P], sP),
                                        np.eye(sP) + O.unpack_skew(thP[j * per_P:(j + 1) * per_P], sP)) for j in range(nP)])
        R = O.dense_side(permR, exR, mode, b)
        P = O.dense_side(permP, exP, mode, b)
        if not np.allclose(np.linalg.svd(R @ W0 @ P, compute_uv=False), sW, rtol=1e-10):
            return False
        k = 2
        Rk = O.dense_side(permR, O.cayley_neumann(thR, nR, sR, k), mode, b)
        Pk = O.dense_side(permP, O.cayley_neumann(thP, nP, sP, k), mode, b)
        sR_ = np.linalg.svd(Rk, compute_uv=False)
        sP_ = np.linalg.svd(Pk, compute_uv=False)
        s = np.linalg.svd(Rk @ W0 @ Pk, compute_uv=False)
        lo = sW * sR_.min() * sP_.min()
        hi = sW * sR_.max() * sP_.max()
        if not (np.all(s >= lo * (1 - 1e-12)) and np.all(s <= hi * (1 + 1e-12))):
            return False
        if np.allclose(s, sW, rtol=1e-6):   # the truncated map must not be exactly orthogonal here
            return False
    return True


def check_merge_invariance(O, m=10, n=8, T=5):
    """y before merge-then-reinitialize equals y after it (theta reset to 0,
    new permutations), for both modes."""
    rng = _rng(7)
    W0 = rng.standard_normal((m, n))
    X = rng.standard_normal((T, n))
    for mode, b, k in [(0, 3, 2), (1, 0, 3)]:
        permR, permP = rng.permutation(m), rng.permutation(n)
        nR, sR = O.side_shape(m, mode, b)
        nP, sP = O.side_shape(n, mode, b)
        thR = rng.standard_normal(nR * O.n_skew(sR)) * 0.2
        thP = rng.standard_normal(nP * O.n_skew(sP)) * 0.2
        R = O.dense_side(permR, O.cayley_neumann(thR, nR, sR, k), mode, b)
        P = O.dense_side(permP, O.cayley_neumann(thP, nP, sP, k), mode, b)
        y_before = O.forward(W0, R, P, X)
        W1 = O.merge(W0, R, P)
        permR2, permP2 = rng.permutation(m), rng.permutation(n)
        R2 = O.dense_side(permR2, O.cayley_neumann(np.zeros_like(thR), nR, sR, k), mode, b)
        P2 = O.dense_side(permP2, O.cayley_neumann(np.zeros_like(thP), nP, sP, k), mode, b)
        if not np.allclose(O.forward(W1, R2, P2, X), y_before, atol=1e-12):
            return False
        # merge is exactly the product (brute force per entry)
        i, j = 3, 5
        ref = sum(R[i, a] * W0[a, c] * P[c, j] for a in range(m) for c in range(n))
        if not np.isclose(W1[i, j], ref, atol=1e-12):
            return False
    return True


# ---------------------------------------------------------------- backward

def _loss(O, W0, thR, thP, permR, permP, mode, b, k, X, dY):
    m, n = W0.shape
    nR, sR = O.side_shape(m, mode, b)
    nP, sP = O.side_shape(n, mode, b)
    R = O.dense_side(permR, O.cayley_neumann(thR, nR, sR, k), mode, b)
    P = O.dense_side(permP, O.cayley_neumann(thP, nP, sP, k), mode, b)
    return float(np.sum(dY * O.forward(W0, R, P, X)))


def check_backward_finite_differences(O):
    """Central finite differences of L = <dY, Y> in float64.  Y is linear in X
    and polynomial in theta, so the differences converge to the exact
    gradient; h = 1e-5 leaves an O(h^2) error far below the tolerance."""
    rng = _rng(8)
    for (m, n, mode, b, k) in [(6, 8, 0, 2, 3), (7, 6, 1, 0, 4), (9, 9, 0, 4, 2)]:
        W0 = rng.standard_normal((m, n))
        X = rng.standard_normal((3, n))
        dY = rng.standard_normal((3, m))
        permR, permP = rng.permutation(m), rng.permutation(n)
        nR, sR = O.side_shape(m, mode, b)
        nP, sP = O.side_shape(n, mode, b)
        thR = rng.standard_normal(nR * O.n_skew(sR)) * 0.3
        thP = rng.standard_normal(nP * O.n_skew(sP)) * 0.3
        out = O.layer_step(W0, thR, thP, permR, permP, mode, b, mode, b, k, X, dY)
        h = 1e-5
        for name, th, grad in [("R", thR, out["dthetaR"]), ("P", thP, out["dthetaP"])]:
            fd = np.zeros_like(th)
            for i in range(len(th)):
                tp, tm = th.copy(), th.copy()
                tp[i] += h
                tm[i] -= h
                if name == "R":
                    fd[i] = (_loss(O, W0, tp, thP, permR, permP, mode, b, k, X, dY)
                             - _loss(O, W0, tm, thP, permR, permP, mode, b, k, X, dY)) / (2 * h)
                else:
                    fd[i] = (_loss(O, W0, thR, tp, permR, permP, mode, b, k, X, dY)
                             - _loss(O, W0, thR, tm, permR, permP, mode, b, k, X, dY)) / (2 * h)
            if not np.allclose(grad, fd, rtol=1e-6, atol=1e-8):
                return False
        fdx = np.zeros_like(X)
        for t in range(X.shape[0]):
            for i in range(n):
                Xp, Xm = X.copy(), X.copy()
                Xp[t, i] += h
                Xm[t, i] -= h
                fdx[t, i] = (_loss(O, W0, thR, thP, permR, permP, mode, b, k, Xp, dY)
                             - _loss(O, W0, thR, thP, permR, permP, mode, b, k, Xm, dY)) / (2 * h)
        if not np.allclose(out["dX"], fdx, rtol=1e-6, atol=1e-8):
            return False
    return True


# ---------------------------------------------------------------- resample

def check_splitmix_golden(O):
    g = load_golden("splitmix64.json")
    ok = O.splitmix64_stream(g["seed"], len(g["outputs"])) == [int(s) for s in g["outputs"]]
    return bool(ok and O.splitmix64(0) == int(g["seed0_first"], 16))


def check_draw_perm(O):
    ok = True
    for d in (1, 2, 7, 256, 1376):
        p = O.draw_perm(0, 3, 1, 2, d)
        ok &= p.dtype == np.int32 and np.array_equal(np.sort(p), np.arange(d))
        ok &= np.array_equal(p, O.draw_perm(0, 3, 1, 2, d))
    # brute force: argsort of the key stream (keys are distinct here)
    h = O.perm_stream_seed(5, 11, 0, 3)
    keys = O.splitmix64_stream(h, 300)
    ok &= np.array_equal(O.draw_perm(5, 11, 0, 3, 300), np.array(sorted(range(300), key=lambda i: keys[i])))
    a = O.draw_perm(0, 0, 0, 0, 512)
    ok &= not np.array_equal(a, O.draw_perm(0, 0, 1, 0, 512))
    ok &= not np.array_equal(a, O.draw_perm(0, 0, 0, 1, 512))
    ok &= not np.array_equal(a, O.draw_perm(0, 1, 0, 0, 512))
    ok &= not np.array_equal(a, O.draw_perm(1, 0, 0, 0, 512))
    return bool(ok)


def check_perm_stream_seed_golden(O):
    """The mixing of (seed, layer, side, epoch) into the key stream's seed, on
    tuples whose SplitMix64 inputs are published test-vector points (the
    expected values were derived by hand, tests/golden/perm_stream_seed.json)."""
    g = load_golden("perm_stream_seed.json")
    return all(O.perm_stream_seed(int(c["seed"]), c["layer_id"], c["side"], c["epoch"]) == int(c["h"])
               for c in g["cases"])


# ---------------------------------------------------------------- optimizer step (adjacent)

def check_adamw_closed_forms(O):
    """Textbook AdamW properties that fix every term of the update."""
    rng = np.random.default_rng(3)
    theta = rng.standard_normal(64)
    g = rng.standard_normal(64)
    z = np.zeros(64)
    lr, b1, b2, eps = 1e-3, 0.9, 0.999, 1e-8
    # first step from zero moments: m_hat = g, v_hat = g^2, so the move is lr * g / (|g| + eps)
    th1, m1, v1 = O.adamw_step(theta, g, z, z, lr, b1, b2, eps, 0.0, 1)
    ok = np.allclose(th1, theta - lr * g / (np.abs(g) + eps), rtol=1e-14, atol=0)
    ok &= np.allclose(m1, (1 - b1) * g, rtol=1e-15, atol=0) and np.allclose(v1, (1 - b2) * g * g, rtol=1e-15, atol=0)
    # a constant gradient keeps the bias-corrected moments at g and g^2: the same move every step
    th, m, v = theta, z, z
    for step in range(1, 6):
        th, m, v = O.adamw_step(th, g, m, v, lr, b1, b2, eps, 0.0, step)
    ok &= np.allclose(th, theta - 5 * lr * g / (np.abs(g) + eps), rtol=1e-12, atol=1e-15)
    # decoupled decay: with no gradient and zero moments only the decay moves theta
    th2, m2, v2 = O.adamw_step(theta, z, z, z, lr, b1, b2, eps, 0.1, 1)
    ok &= np.allclose(th2, theta * (1 - lr * 0.1), rtol=1e-15, atol=0) and not m2.any() and not v2.any()
    # moments decay geometrically with no gradient
    _, m3, v3 = O.adamw_step(theta, z, np.ones(64), 4 * np.ones(64), lr, b1, b2, eps, 0.0, 1000)
    ok &= np.allclose(m3, b1) and np.allclose(v3, 4 * b2)
    return bool(ok)


# ---------------------------------------------------------------- bookkeeping

def check_param_counts(O):
    g = load_golden("param_counts.json")
    shapes = O.llama_linear_shapes(g["hidden"], g["ffn"])
    total = g["layers"] * sum(m * n for m, n in shapes)
    digits = g["adamw_trainable_print_digits"]
    ok = float(f"{total:.{digits - 1}e}") == g["adamw_trainable_printed"]
    poet = g["layers"] * sum(O.trainable_params(m, n, O.BS, g["b"]) for m, n in shapes)
    ok &= abs(poet - g["poet_bs256_trainable_printed"]) / g["poet_bs256_trainable_printed"] < 5e-4
    return bool(ok)


ALL_CHECKS = [
    check_unpack_golden, check_cnp_2x2_closed_form, check_cnp_truncation_identity,
    check_orthogonality_identity, check_singular_values_closed_form, check_special_cases,
    check_dense_side_golden, check_dense_side_vs_loops, check_apply_side_rows, check_side_shapes,
    check_no_primitive_side,
    check_spectrum_preservation, check_merge_invariance, check_backward_finite_differences,
    check_splitmix_golden, check_perm_stream_seed_golden, check_draw_perm, check_param_counts, check_adamw_closed_forms,
]

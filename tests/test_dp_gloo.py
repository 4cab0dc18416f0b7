"""The data-parallel exchange on CPU with gloo, world size 2 (no GPU).

Each rank takes its own half of the tokens through the same layer (same W0,
skew parameters and permutations) and computes its packed-skew gradients with
the oracle; summing them over the ranks must give the gradients of the whole
batch, because the loss is a sum over tokens.  The timing reduction takes the
maximum over ranks."""
import os
import socket

import numpy as np
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    import torch
    import torch.distributed as dist

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    try:
        import datetime

        dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
        from oracle import poet_oracle as O
        from orthogonal_reparameterized_poet_b200 import dp

        rng = np.random.default_rng(0)  # identical on both ranks: replicated parameters
        m, n, mode, b, k, T = 12, 10, 0, 4, 3, 8
        W0 = rng.standard_normal((m, n))
        permR, permP = rng.permutation(m), rng.permutation(n)
        nR, sR = O.side_shape(m, mode, b)
        nP, sP = O.side_shape(n, mode, b)
        thR = rng.standard_normal(nR * O.n_skew(sR)) * 0.2
        thP = rng.standard_normal(nP * O.n_skew(sP)) * 0.2
        X = rng.standard_normal((T, n))
        dY = rng.standard_normal((T, m))
        half = slice(rank * T // world, (rank + 1) * T // world)
        mine = O.layer_step(W0, thR, thP, permR, permP, mode, b, mode, b, k, X[half], dY[half])
        flat = torch.from_numpy(np.concatenate([mine["dthetaR"], mine["dthetaP"]]))
        dp.allreduce_gradients_(flat)
        full = O.layer_step(W0, thR, thP, permR, permP, mode, b, mode, b, k, X, dY)
        ref = np.concatenate([full["dthetaR"], full["dthetaP"]])
        ok_sum = bool(np.allclose(flat.numpy(), ref, rtol=1e-10, atol=1e-12))
        mx = dp.max_over_ranks([float(rank), 10.0 - rank])
        ok_max = mx == [float(world - 1), 10.0]
        dist.destroy_process_group()
        q.put((rank, ok_sum, ok_max, None))
    except Exception as e:  # report, never hang the parent
        q.put((rank, False, False, repr(e)))


def test_gradient_allreduce_matches_whole_batch():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    results = [q.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
    for rank, ok_sum, ok_max, err in results:
        assert err is None, f"rank {rank}: {err}"
        assert ok_sum, f"rank {rank}: summed gradients differ from the whole-batch gradients"
        assert ok_max, f"rank {rank}: max over ranks is wrong"

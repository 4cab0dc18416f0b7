"""Failure detection without a GPU fault: a bounded device-side wait that runs
out is reported on the host as POET_ETIMEOUT, the status word is cleared by
reading it, and the context keeps working afterwards."""
import numpy as np
import pytest

pytestmark = pytest.mark.gpu


def test_bounded_wait_reports_timeout_and_context_survives():
    import torch

    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from orthogonal_reparameterized_poet_b200 import poet

    poet.poet_sync_status()  # start from a clear status word
    poet.poet_selftest_bounded_wait(20000)  # 20 ms limit on a barrier nothing arrives on
    with pytest.raises(poet.PoetError) as e:
        poet.poet_sync_status()
    assert e.value.status == poet.ETIMEOUT
    assert "bounded wait" in str(e.value)
    poet.poet_sync_status()  # the word was cleared by the read
    # the context is still usable: a tensor-core GEMM afterwards is correct
    A = torch.randn(256, 128, device="cuda").to(torch.bfloat16)
    B = torch.randn(192, 128, device="cuda").to(torch.bfloat16)
    C = torch.empty(256, 192, device="cuda", dtype=torch.bfloat16)
    poet.poet_gemm(poet.BF16, 256, 192, 128, 1, A, (128, 1, 0), B, (128, 1, 0), C, 192, 0)
    poet.poet_sync_status()
    ref = A.double().cpu().numpy() @ B.double().cpu().numpy().T
    assert np.linalg.norm(C.double().cpu().numpy() - ref) / np.linalg.norm(ref) < 8e-3


def test_bounded_wait_limit_is_validated():
    import torch

    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from orthogonal_reparameterized_poet_b200 import poet

    with pytest.raises(poet.PoetError):
        poet.poet_selftest_bounded_wait(0)
    with pytest.raises(poet.PoetError):
        poet.poet_selftest_bounded_wait(2000000)


@pytest.mark.parametrize("plan,side,value", [(1, "P", 10**6), (2, "R", -7), (2, "P", 10**6)])
def test_perm_entry_out_of_range_is_skipped_and_reported(plan, side, value):
    """A caller-written permutation with an entry outside [0, dim): the kernels
    that read it (the token plan's activation gather, the weight plan's
    unframing with its row map and inverse column map) skip that index, record
    it in the status word, and poet_sync_status reports POET_EBOUNDS; the
    context stays usable and a valid call afterwards is exact."""
    import torch

    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from orthogonal_reparameterized_poet_b200 import inputs as I
    from orthogonal_reparameterized_poet_b200 import poet
    from tests.harness import Case

    case = Case(300, 200, I.BS, 64, I.BS, 64, 2, 40, I.BF16, 0.05, layer_id=3)
    W0, thR, thP, x, dy = case.arrays()
    L = poet.PoetLayer(torch.from_numpy(W0).to("cuda", torch.bfloat16), torch.from_numpy(thR).cuda(),
                       torch.from_numpy(thP).cuda(), mode=case.modeR, b=case.bR, k=case.k, plan=plan)
    xt = torch.from_numpy(x).to("cuda", torch.bfloat16)
    L.prepare()
    L.cayley_neumann()
    poet.poet_sync_status()
    y_ok, _ = L.forward(xt)
    poet.poet_sync_status()
    perm = L.perm_R if side == "R" else L.perm_P
    good = perm[5].item()
    perm[5] = value  # written on the host side of the ABI, as a caller could
    L.forward(xt)
    with pytest.raises(poet.PoetError) as e:
        poet.poet_sync_status()
    assert e.value.status == poet.EBOUNDS
    assert "out of range" in str(e.value)
    poet.poet_sync_status()  # cleared by the read
    perm[5] = good
    y2, _ = L.forward(xt)
    poet.poet_sync_status()
    assert torch.equal(y2, y_ok)

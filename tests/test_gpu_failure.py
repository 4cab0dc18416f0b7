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

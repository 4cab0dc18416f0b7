"""The C-ABI library loads and exports every symbol include/poet.h declares;
host-side size queries and argument validation (no GPU needed)."""
import ctypes
import os
import re

import pytest

from orthogonal_reparameterized_poet_b200 import poet

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    src = open(os.path.join(ROOT, "include", "poet.h")).read()
    return sorted(set(re.findall(r"POET_API\s+[\w\s\*]+?\b(poet_\w+)\s*\(", src)))


def test_header_declares_the_boundary():
    names = _declared()
    for required in ("poet_cayley_neumann", "poet_forward", "poet_backward", "poet_merge", "poet_resample"):
        assert required in names


def test_library_exports_every_declared_symbol():
    lib = ctypes.CDLL(poet._LIB_PATH)
    missing = [n for n in _declared() if not hasattr(lib, n)]
    assert not missing, missing
    assert sorted(poet.ABI_SYMBOLS) == _declared()


def test_version_string():
    assert "sm_100a" in poet.poet_version()


def _side(dim, mode, b, k):
    s = poet.poet_side()
    s.dim, s.mode, s.b, s.k = dim, mode, b, k
    return s


def _layer(m, n, mode, b, k, dtype):
    L = poet.poet_layer()
    L.m, L.n, L.dtype = m, n, dtype
    L.R = _side(m, mode, b, k)
    L.P = _side(n, mode, b, k)
    return L


def test_state_and_frame_sizes():
    # BS b=256 on d=5461: 21 primitives of 256 (ld 256); state = (2 + k) terms of 21*256*256 elements
    assert poet.poet_side_state_bytes(_side(5461, poet.BS, 256, 4), poet.BF16) == 6 * 21 * 256 * 256 * 2
    # FS on d=5461: one primitive of 2730, stored with ld 2736
    term = (1 * 2736 * 2736 * 2 + 255) // 256 * 256
    assert poet.poet_side_state_bytes(_side(5461, poet.FS, 0, 4), poet.BF16) == 6 * term
    # k = 0 keeps only the primitive and Q
    assert poet.poet_side_state_bytes(_side(256, poet.BS, 32, 0), poet.F32) == 2 * 8 * 32 * 32 * 4
    # b > dim: no primitives
    assert poet.poet_side_state_bytes(_side(100, poet.BS, 256, 4), poet.BF16) == 0
    # malformed sides
    assert poet.poet_side_state_bytes(_side(0, poet.BS, 256, 4), poet.BF16) == 0
    assert poet.poet_side_state_bytes(_side(10, poet.BS, 0, 4), poet.BF16) == 0
    assert poet.poet_side_state_bytes(_side(10, poet.BS, 2, 17), poet.BF16) == 0
    L = _layer(5461, 2048, poet.BS, 256, 4, poet.BF16)
    assert poet.poet_frame_bytes(L) == 5461 * 2048 * 2
    L.plan = poet.PLAN_TOKEN  # frame copies of x (ld 2048) and of W0 P x (ld 5504)
    assert poet.poet_saved_bytes(L, 32768) == 32768 * 2048 * 2 + 32768 * 5504 * 2
    assert poet.poet_workspace_bytes(L, 32768) > poet.poet_workspace_bytes(L, 0) > 0
    L.plan = poet.PLAN_WEIGHT  # E, F, H (m x ld 2048, 256-byte rounded) and a re-strided x
    w = (5461 * 2048 * 2 + 255) // 256 * 256
    assert poet.poet_saved_bytes(L, 32768) == 3 * w + 32768 * 2048 * 2
    assert poet.poet_workspace_bytes(L, 32768) > poet.poet_workspace_bytes(L, 0) > 0


@pytest.mark.parametrize("m,n,mode,b", [(2048, 2048, poet.BS, 256), (5461, 2048, poet.BS, 256),
                                        (2048, 5461, poet.FS, 0), (2048, 2048, poet.FS, 0)])
def test_auto_plan_follows_token_count(m, n, mode, b):
    L = _layer(m, n, mode, b, 4, poet.BF16)
    # many tokens per weight element: the primitives go on W0; few tokens: on the activations
    assert poet.poet_plan_for(L, 32768) == poet.PLAN_WEIGHT
    assert poet.poet_plan_for(L, 64) == poet.PLAN_TOKEN
    assert poet.poet_plan_for(L, 0) == poet.PLAN_TOKEN
    for forced in (poet.PLAN_TOKEN, poet.PLAN_WEIGHT):
        L.plan = forced
        assert poet.poet_plan_for(L, 32768) == forced and poet.poet_plan_for(L, 64) == forced
    L.plan = 3
    assert poet.poet_plan_for(L, 64) == -1
    assert poet.poet_saved_bytes(L, 64) == 0 and poet.poet_workspace_bytes(L, 64) == 0


def test_weight_plan_backward_requires_x():
    lib = poet.lib()
    st = ctypes.c_void_p(0)
    L = _layer(256, 256, poet.BS, 32, 3, poet.BF16)
    L.plan = poet.PLAN_WEIGHT
    fake = 1 << 20  # 256-byte aligned, never dereferenced: validation fails first
    L.W0, L.W0f = fake, fake
    for sd in (L.R, L.P):
        sd.perm, sd.theta, sd.state = fake, fake, fake
    ws_bytes = poet.poet_workspace_bytes(L, 16)
    args = (ctypes.c_void_p(fake), ctypes.c_void_p(fake), 16, ctypes.c_void_p(fake), ctypes.c_void_p(fake),
            ctypes.c_void_p(fake), ctypes.c_void_p(fake), ws_bytes, st)
    assert lib.poet_backward(ctypes.byref(L), None, *args) == poet.EINVAL
    assert "x NULL" in lib.poet_last_error().decode()
    assert lib.poet_backward_blocks(ctypes.byref(L), None, *args) == poet.EINVAL


def test_host_validation_rejects_bad_arguments():
    lib = poet.lib()
    L = _layer(256, 256, poet.BS, 32, 3, poet.F32)
    st = poet.poet_forward.__globals__["ctypes"].c_void_p(0)
    # NULL pointers everywhere: rejected before any launch
    assert lib.poet_forward(ctypes.byref(L), None, 16, None, None, None, 0, st) == poet.EINVAL
    assert "NULL" in lib.poet_last_error().decode() or "misaligned" in lib.poet_last_error().decode()
    assert lib.poet_forward(None, None, 16, None, None, None, 0, st) == poet.EINVAL
    assert lib.poet_draw_perm(0, 0, 0, 0, 0, None, st) == poet.EINVAL
    assert lib.poet_draw_perm(0, 0, 0, 0, 16385, None, st) == poet.EINVAL
    assert lib.poet_draw_perm(0, -1, 0, 0, 16, ctypes.c_void_p(256), st) == poet.EINVAL
    bad = _layer(256, 255, poet.BS, 32, 3, poet.F32)  # side dim does not match W0
    bad.P.dim = 256
    assert lib.poet_merge(ctypes.byref(bad), None, 0, st) == poet.EINVAL
    assert lib.poet_gemm(7, 1, 1, 1, 1, None, 0, 0, 0, None, 0, 0, 0, None, 1, 0, 1.0, 0.0, st) == poet.EINVAL
    assert lib.poet_trace_set_ridge(0.0) == poet.EINVAL
    assert lib.poet_trace_set_ridge(-5.0) == poet.EINVAL
    assert lib.poet_trace_set_ridge(216.0) == poet.OK


def test_missing_library_fails_loudly(monkeypatch, tmp_path):
    monkeypatch.setattr(poet, "_lib", None)
    monkeypatch.setattr(poet, "_LIB_PATH", str(tmp_path / "absent.so"))
    with pytest.raises(RuntimeError, match="not built"):
        poet.lib()


def test_adamw_step_validation():
    lib = poet.lib()
    st = ctypes.c_void_p(0)
    fake = ctypes.c_void_p(1 << 20)
    call = lambda ptrs, n, lr=1e-3, b1=0.9, b2=0.999, eps=1e-8, wd=0.0, step=1: lib.poet_adamw_step(
        *ptrs, n, lr, b1, b2, eps, wd, step, st)
    assert call((None, None, None, None), 0) == poet.OK            # nothing to do
    assert call((None, None, None, None), 16) == poet.EINVAL       # NULL buffers
    assert call((ctypes.c_void_p((1 << 20) + 2), fake, fake, fake), 16) == poet.EINVAL  # misaligned
    assert call((fake,) * 4, 16, b1=1.0) == poet.EINVAL
    assert call((fake,) * 4, 16, eps=0.0) == poet.EINVAL
    assert call((fake,) * 4, 16, lr=-1.0) == poet.EINVAL
    assert call((fake,) * 4, 16, step=0) == poet.EINVAL
    assert call((fake,) * 4, -1) == poet.EINVAL


@pytest.mark.parametrize("m,n,mode,b,dtype", [(512, 512, poet.FS, 0, poet.BF16), (1376, 512, poet.FS, 0, poet.BF16),
                                              (2736, 1024, poet.BS, 256, poet.BF16), (5461, 2048, poet.BS, 256, poet.BF16),
                                              (6912, 2560, poet.FS, 0, poet.BF16), (256, 256, poet.BS, 32, poet.F32)])
def test_auto_plan_switches_once(m, n, mode, b, dtype):
    """The cost model's choice is monotone in the token count: the token plan up
    to some T, the weight plan beyond it (never back)."""
    L = _layer(m, n, mode, b, 4, dtype)
    plans = [poet.poet_plan_for(L, T) for T in [0, 1, 16, 64, 256, 1024, 2048, 4096, 8192, 16384, 32768, 1 << 20]]
    assert set(plans) <= {poet.PLAN_TOKEN, poet.PLAN_WEIGHT}
    first_weight = plans.index(poet.PLAN_WEIGHT) if poet.PLAN_WEIGHT in plans else len(plans)
    assert all(p == poet.PLAN_TOKEN for p in plans[:first_weight])
    assert all(p == poet.PLAN_WEIGHT for p in plans[first_weight:])
    # the workspace and saved sizes follow the plan the layer runs
    for T in (64, 32768):
        L.plan = poet.poet_plan_for(L, T)
        fixed = (poet.poet_saved_bytes(L, T), poet.poet_workspace_bytes(L, T))
        L.plan = poet.PLAN_AUTO
        assert (poet.poet_saved_bytes(L, T), poet.poet_workspace_bytes(L, T)) == fixed


def test_many_layer_calls_validate_and_size():
    """The grouped calls: sizes grow with the list, a re-strided dy costs
    workspace, and bad lists are rejected before anything is launched."""
    lib = poet.lib()

    def layer(m, n, dtype=poet.BF16, plan=poet.PLAN_WEIGHT, fake=1 << 20):
        L = poet.poet_layer()
        L.m, L.n, L.dtype, L.plan = m, n, dtype, plan
        for sd, d in ((L.R, m), (L.P, n)):
            sd.dim, sd.mode, sd.b, sd.k = d, poet.BS, 256, 4
            sd.perm, sd.theta, sd.state = fake, fake, fake
        L.W0, L.W0f = fake, fake
        return L

    one = poet.poet_many_workspace_bytes([layer(2048, 2048)], 4096)
    two = poet.poet_many_workspace_bytes([layer(2048, 2048), layer(5461, 2048)], 4096)
    assert 0 < one < two
    # dy rows of 5461 bf16 elements are not 16-byte aligned: room for a re-strided copy
    plain = poet.poet_many_workspace_bytes([layer(5461, 2048)], 4096, [5464])
    odd = poet.poet_many_workspace_bytes([layer(5461, 2048)], 4096, [5461])
    assert odd - plain >= 4096 * 5504 * 2
    st = ctypes.c_void_p(0)
    arr = (poet.poet_layer * 2)(layer(256, 256), layer(256, 256, dtype=poet.F32))
    fake = (ctypes.c_void_p * 2)(1 << 20, 1 << 20)
    # mixed element types
    assert lib.poet_forward_many(arr, 2, fake, None, 16, fake, None, fake, ctypes.c_void_p(1 << 20), 1 << 30,
                                 st) == poet.EINVAL
    # a row stride below the width
    arr1 = (poet.poet_layer * 1)(layer(256, 256))
    ld = (ctypes.c_int64 * 1)(255)
    assert lib.poet_forward_many(arr1, 1, fake, ld, 16, fake, None, fake, ctypes.c_void_p(1 << 20), 1 << 30,
                                 st) == poet.EINVAL
    # workspace too small
    assert lib.poet_forward_many(arr1, 1, fake, None, 16, fake, None, fake, ctypes.c_void_p(1 << 20), 256,
                                 st) == poet.ENOMEM_WS
    assert lib.poet_backward_blocks_many(arr1, 1, fake, None, fake, fake, None, 16, fake, None, None, None,
                                         ctypes.c_void_p(1 << 20), 1 << 30, st) == poet.EINVAL

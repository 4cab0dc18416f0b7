"""Thin Python binding of libpoet (the C ABI in include/poet.h).

Argument marshalling only: every step of the POET layer runs in libpoet's
CUDA kernels.  PyTorch supplies device memory and the current stream.  If
libpoet.so is missing or cannot be loaded, every call raises: there is no
host fallback.
"""
from __future__ import annotations

import ctypes
import os

import torch

F32, BF16 = 0, 1
BS, FS = 0, 1
PLAN_AUTO, PLAN_TOKEN, PLAN_WEIGHT = 0, 1, 2
OK, EINVAL, ECUDA, ETIMEOUT, ENOMEM_WS, EBOUNDS = 0, 1, 2, 3, 4, 5

_LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libpoet.so")
_lib = None


class PoetError(RuntimeError):
    def __init__(self, status, msg):
        super().__init__(f"libpoet status {status}: {msg}")
        self.status = status


class poet_side(ctypes.Structure):
    _fields_ = [("dim", ctypes.c_int32), ("mode", ctypes.c_int32), ("b", ctypes.c_int32), ("k", ctypes.c_int32),
                ("perm", ctypes.c_void_p), ("theta", ctypes.c_void_p), ("state", ctypes.c_void_p)]


class poet_layer(ctypes.Structure):
    _fields_ = [("m", ctypes.c_int64), ("n", ctypes.c_int64), ("dtype", ctypes.c_int32),
                ("layer_id", ctypes.c_int32), ("epoch", ctypes.c_int32), ("plan", ctypes.c_int32),
                ("seed", ctypes.c_uint64), ("W0", ctypes.c_void_p), ("W0f", ctypes.c_void_p),
                ("R", poet_side), ("P", poet_side)]


class poet_llama_block(ctypes.Structure):
    _fields_ = [("seq_len", ctypes.c_int32), ("heads", ctypes.c_int32), ("head_dim", ctypes.c_int32),
                ("rope_base", ctypes.c_float), ("norm_eps", ctypes.c_float), ("lin", poet_layer * 7)]


class poet_adamw_hparams(ctypes.Structure):
    _fields_ = [("lr", ctypes.c_float), ("beta1", ctypes.c_float), ("beta2", ctypes.c_float), ("eps", ctypes.c_float),
                ("weight_decay", ctypes.c_float), ("step", ctypes.c_int32)]


class poet_trace_row(ctypes.Structure):
    _fields_ = [("kind", ctypes.c_char * 32), ("launches", ctypes.c_int64), ("ms", ctypes.c_double),
                ("flop", ctypes.c_double), ("bytes", ctypes.c_double), ("flop_tc", ctypes.c_double),
                ("bytes_hbm", ctypes.c_double)]


_SIGS = {
    "poet_side_state_bytes": (ctypes.c_size_t, [ctypes.POINTER(poet_side), ctypes.c_int32]),
    "poet_frame_bytes": (ctypes.c_size_t, [ctypes.POINTER(poet_layer)]),
    "poet_plan_for": (ctypes.c_int32, [ctypes.POINTER(poet_layer), ctypes.c_int64]),
    "poet_saved_bytes": (ctypes.c_size_t, [ctypes.POINTER(poet_layer), ctypes.c_int64]),
    "poet_workspace_bytes": (ctypes.c_size_t, [ctypes.POINTER(poet_layer), ctypes.c_int64]),
    "poet_side_workspace_bytes": (ctypes.c_size_t, [ctypes.POINTER(poet_side), ctypes.c_int32]),
    "poet_cayley_neumann": (ctypes.c_int, [ctypes.POINTER(poet_side), ctypes.c_int32, ctypes.c_void_p,
                                           ctypes.c_size_t, ctypes.c_void_p]),
    "poet_cayley_neumann_grad": (ctypes.c_int, [ctypes.POINTER(poet_side), ctypes.c_int32, ctypes.c_void_p,
                                                ctypes.c_void_p, ctypes.c_void_p, ctypes.c_size_t,
                                                ctypes.c_void_p]),
    "poet_forward": (ctypes.c_int, [ctypes.POINTER(poet_layer), ctypes.c_void_p, ctypes.c_int64, ctypes.c_void_p,
                                    ctypes.c_void_p, ctypes.c_void_p, ctypes.c_size_t, ctypes.c_void_p]),
    "poet_backward": (ctypes.c_int, [ctypes.POINTER(poet_layer), ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
                                     ctypes.c_int64, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
                                     ctypes.c_void_p, ctypes.c_size_t, ctypes.c_void_p]),
    "poet_merge": (ctypes.c_int, [ctypes.POINTER(poet_layer), ctypes.c_void_p, ctypes.c_size_t, ctypes.c_void_p]),
    "poet_prepare": (ctypes.c_int, [ctypes.POINTER(poet_layer), ctypes.c_void_p]),
    "poet_resample": (ctypes.c_int, [ctypes.POINTER(poet_layer), ctypes.c_void_p]),
    "poet_draw_perm": (ctypes.c_int, [ctypes.c_uint64, ctypes.c_int32, ctypes.c_int32, ctypes.c_int32,
                                      ctypes.c_int32, ctypes.c_void_p, ctypes.c_void_p]),
    "poet_gemm": (ctypes.c_int, [ctypes.c_int32, ctypes.c_int32, ctypes.c_int32, ctypes.c_int32, ctypes.c_int32,
                                 ctypes.c_void_p, ctypes.c_int64, ctypes.c_int64, ctypes.c_int64,
                                 ctypes.c_void_p, ctypes.c_int64, ctypes.c_int64, ctypes.c_int64,
                                 ctypes.c_void_p, ctypes.c_int64, ctypes.c_int64, ctypes.c_float, ctypes.c_float,
                                 ctypes.c_void_p]),
    "poet_gemm_engine": (ctypes.c_int32, [ctypes.c_int32]),
    "poet_block_grad_bytes": (ctypes.c_size_t, [ctypes.POINTER(poet_side)]),
    "poet_cayley_neumann_many": (ctypes.c_int, [ctypes.POINTER(poet_side), ctypes.c_int32, ctypes.c_int32,
                                                ctypes.c_void_p]),
    "poet_backward_blocks": (ctypes.c_int, [ctypes.POINTER(poet_layer), ctypes.c_void_p, ctypes.c_void_p,
                                            ctypes.c_void_p, ctypes.c_int64, ctypes.c_void_p, ctypes.c_void_p,
                                            ctypes.c_void_p, ctypes.c_void_p, ctypes.c_size_t, ctypes.c_void_p]),
    "poet_many_workspace_bytes": (ctypes.c_size_t, [ctypes.POINTER(poet_layer), ctypes.c_int32, ctypes.c_int64,
                                                     ctypes.c_void_p]),
    "poet_forward_many": (ctypes.c_int, [ctypes.POINTER(poet_layer), ctypes.c_int32, ctypes.c_void_p, ctypes.c_void_p,
                                         ctypes.c_int64, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
                                         ctypes.c_void_p, ctypes.c_size_t, ctypes.c_void_p]),
    "poet_backward_blocks_many": (ctypes.c_int, [ctypes.POINTER(poet_layer), ctypes.c_int32, ctypes.c_void_p,
                                                 ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
                                                 ctypes.c_int64, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
                                                 ctypes.c_void_p, ctypes.c_void_p, ctypes.c_size_t,
                                                 ctypes.c_void_p]),
    "poet_cayley_neumann_grad_many_workspace_bytes": (ctypes.c_size_t, [ctypes.POINTER(poet_side), ctypes.c_int32,
                                                                        ctypes.c_int32]),
    "poet_cayley_neumann_grad_many": (ctypes.c_int, [ctypes.POINTER(poet_side), ctypes.POINTER(ctypes.c_void_p),
                                                     ctypes.POINTER(ctypes.c_void_p), ctypes.c_int32, ctypes.c_int32,
                                                     ctypes.c_void_p, ctypes.c_size_t, ctypes.c_void_p]),
    "poet_cayley_neumann_grad_noalloc": (ctypes.c_int, [ctypes.POINTER(poet_side), ctypes.c_int32, ctypes.c_void_p,
                                                        ctypes.c_void_p, ctypes.c_void_p]),
    "poet_cayley_neumann_grad_many_adamw": (ctypes.c_int, [ctypes.POINTER(poet_side), ctypes.c_void_p, ctypes.c_void_p,
                                                           ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int32,
                                                           ctypes.c_int32, ctypes.POINTER(poet_adamw_hparams),
                                                           ctypes.c_void_p, ctypes.c_size_t, ctypes.c_void_p]),
    "poet_merge_reset_moments": (ctypes.c_int, [ctypes.POINTER(poet_layer), ctypes.c_void_p, ctypes.c_void_p,
                                                ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_size_t,
                                                ctypes.c_void_p]),
    "poet_workspace_size": (ctypes.c_size_t, [ctypes.POINTER(poet_layer), ctypes.c_int64]),
    "poet_llama_block_saved_bytes": (ctypes.c_size_t, [ctypes.POINTER(poet_llama_block), ctypes.c_int64]),
    "poet_llama_block_workspace_bytes": (ctypes.c_size_t, [ctypes.POINTER(poet_llama_block), ctypes.c_int64]),
    "poet_llama_block_forward": (ctypes.c_int, [ctypes.POINTER(poet_llama_block), ctypes.c_void_p, ctypes.c_int64,
                                                ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_size_t,
                                                ctypes.c_void_p]),
    "poet_llama_block_backward": (ctypes.c_int, [ctypes.POINTER(poet_llama_block), ctypes.c_void_p, ctypes.c_void_p,
                                                 ctypes.c_int64, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
                                                 ctypes.c_size_t, ctypes.c_void_p]),
    "poet_selftest_bounded_wait": (ctypes.c_int, [ctypes.c_uint32, ctypes.c_void_p]),
    "poet_adamw_step": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
                                       ctypes.c_int64, ctypes.c_float, ctypes.c_float, ctypes.c_float,
                                       ctypes.c_float, ctypes.c_float, ctypes.c_int32, ctypes.c_void_p]),
    "poet_sync_status": (ctypes.c_int, [ctypes.c_void_p]),
    "poet_launch_count": (ctypes.c_int64, []),
    "poet_trace_enable": (ctypes.c_int, [ctypes.c_int32]),
    "poet_trace_read": (ctypes.c_int32, [ctypes.POINTER(poet_trace_row), ctypes.c_int32]),
    "poet_trace_set_ridge": (ctypes.c_int, [ctypes.c_double]),
    "poet_last_error": (ctypes.c_char_p, []),
    "poet_version": (ctypes.c_char_p, []),
}

ABI_SYMBOLS = tuple(_SIGS)


def lib() -> ctypes.CDLL:
    """The loaded libpoet (raises if it is not built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(_LIB_PATH):
            raise RuntimeError(f"libpoet.so not built at {_LIB_PATH}; run "
                               "`python -m orthogonal_reparameterized_poet_b200.build`")
        L = ctypes.CDLL(_LIB_PATH)
        for name, (res, args) in _SIGS.items():
            f = getattr(L, name)
            f.restype = res
            f.argtypes = args
        _lib = L
    return _lib


def _check(status):
    if status != OK:
        raise PoetError(status, lib().poet_last_error().decode())


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def torch_dtype(dtype: int):
    return torch.bfloat16 if dtype == BF16 else torch.float32


def side_geometry(dim, mode, b):
    """(nprim, size) of one side, as libpoet computes it (host bookkeeping for buffer sizes)."""
    if mode == FS:
        s = dim // 2
        return (1, s) if s >= 1 else (0, 0)
    q = dim // b
    return (q, b) if q > 0 else (0, 0)


# ------------------------------------------------------------------ raw ABI calls

def poet_side_state_bytes(side: poet_side, dtype: int) -> int:
    return lib().poet_side_state_bytes(ctypes.byref(side), dtype)


def poet_frame_bytes(layer: poet_layer) -> int:
    return lib().poet_frame_bytes(ctypes.byref(layer))


def poet_plan_for(layer: poet_layer, T: int) -> int:
    return lib().poet_plan_for(ctypes.byref(layer), T)


def poet_saved_bytes(layer: poet_layer, T: int) -> int:
    return lib().poet_saved_bytes(ctypes.byref(layer), T)


def poet_workspace_bytes(layer: poet_layer, T: int) -> int:
    return lib().poet_workspace_bytes(ctypes.byref(layer), T)


def poet_side_workspace_bytes(side: poet_side, dtype: int) -> int:
    return lib().poet_side_workspace_bytes(ctypes.byref(side), dtype)


def poet_cayley_neumann(side: poet_side, dtype: int, ws=None, stream=None):
    _check(lib().poet_cayley_neumann(ctypes.byref(side), dtype, _ptr(ws), 0 if ws is None else ws.numel(),
                                     _stream(stream)))


def poet_cayley_neumann_grad(side: poet_side, dtype: int, G, dtheta, ws, stream=None):
    _check(lib().poet_cayley_neumann_grad(ctypes.byref(side), dtype, _ptr(G), _ptr(dtheta), _ptr(ws), ws.numel(),
                                          _stream(stream)))


def poet_cayley_neumann_grad_noalloc(side: poet_side, dtype: int, G, dtheta, stream=None):
    """a8 without a caller workspace (the library's built-in 32 MiB scratch)."""
    _check(lib().poet_cayley_neumann_grad_noalloc(ctypes.byref(side), dtype, _ptr(G), _ptr(dtheta), _stream(stream)))


def poet_forward(layer: poet_layer, x, T: int, y, saved, ws, stream=None):
    _check(lib().poet_forward(ctypes.byref(layer), _ptr(x), T, _ptr(y), _ptr(saved), _ptr(ws), ws.numel(),
                              _stream(stream)))


def poet_backward(layer: poet_layer, x, saved, dy, T: int, dx, dtheta_R, dtheta_P, ws, stream=None):
    _check(lib().poet_backward(ctypes.byref(layer), _ptr(x), _ptr(saved), _ptr(dy), T, _ptr(dx), _ptr(dtheta_R),
                               _ptr(dtheta_P), _ptr(ws), ws.numel(), _stream(stream)))


def poet_merge(layer: poet_layer, ws, stream=None):
    _check(lib().poet_merge(ctypes.byref(layer), _ptr(ws), ws.numel(), _stream(stream)))


def poet_prepare(layer: poet_layer, stream=None):
    _check(lib().poet_prepare(ctypes.byref(layer), _stream(stream)))


def poet_resample(layer: poet_layer, stream=None):
    _check(lib().poet_resample(ctypes.byref(layer), _stream(stream)))


def poet_draw_perm(seed: int, layer_id: int, side: int, epoch: int, dim: int, perm, stream=None):
    _check(lib().poet_draw_perm(seed, layer_id, side, epoch, dim, _ptr(perm), _stream(stream)))


def poet_gemm(dtype, M, N, K, batch, A, sA, B, sB, C, ldc, sCb, alpha=1.0, beta=0.0, stream=None):
    """sA = (sAm, sAk, sAb), sB = (sBn, sBk, sBb) in elements."""
    _check(lib().poet_gemm(dtype, M, N, K, batch, _ptr(A), *sA, _ptr(B), *sB, _ptr(C), ldc, sCb, alpha, beta,
                           _stream(stream)))


def poet_gemm_engine(dtype: int) -> int:
    return lib().poet_gemm_engine(dtype)


def poet_selftest_bounded_wait(timeout_us: int, stream=None):
    _check(lib().poet_selftest_bounded_wait(timeout_us, _stream(stream)))


def poet_adamw_step(theta, grad, m, v, lr, beta1=0.9, beta2=0.999, eps=1e-8, weight_decay=0.0, step=1,
                    stream=None):
    """One AdamW step on float tensors of equal length, in place on theta, m and v."""
    n = theta.numel()
    if not (grad.numel() == m.numel() == v.numel() == n):
        raise ValueError("theta, grad, m and v must have the same length")
    _check(lib().poet_adamw_step(_ptr(theta), _ptr(grad), _ptr(m), _ptr(v), n, lr, beta1, beta2, eps,
                                 weight_decay, step, _stream(stream)))


def poet_sync_status(stream=None):
    _check(lib().poet_sync_status(_stream(stream)))


def poet_block_grad_bytes(side: poet_side) -> int:
    return lib().poet_block_grad_bytes(ctypes.byref(side))


def _side_array(sides):
    arr = (poet_side * max(len(sides), 1))()
    for i, sd in enumerate(sides):
        arr[i] = sd
    return arr


def poet_cayley_neumann_many(sides, dtype: int, stream=None):
    _check(lib().poet_cayley_neumann_many(_side_array(sides), len(sides), dtype, _stream(stream)))


def poet_backward_blocks(layer: poet_layer, x, saved, dy, T: int, dx, G_R, G_P, ws, stream=None):
    _check(lib().poet_backward_blocks(ctypes.byref(layer), _ptr(x), _ptr(saved), _ptr(dy), T, _ptr(dx), _ptr(G_R),
                                      _ptr(G_P), _ptr(ws), ws.numel(), _stream(stream)))


def poet_cayley_neumann_grad_many_workspace_bytes(sides, dtype: int) -> int:
    return lib().poet_cayley_neumann_grad_many_workspace_bytes(_side_array(sides), len(sides), dtype)


def poet_cayley_neumann_grad_many(sides, G, dtheta, dtype: int, ws, stream=None):
    n = len(sides)
    gp = (ctypes.c_void_p * max(n, 1))(*[None if t is None else t.data_ptr() for t in G])
    dp = (ctypes.c_void_p * max(n, 1))(*[None if t is None else t.data_ptr() for t in dtheta])
    _check(lib().poet_cayley_neumann_grad_many(_side_array(sides), gp, dp, n, dtype, _ptr(ws),
                                               0 if ws is None else ws.numel(), _stream(stream)))


def poet_launch_count() -> int:
    return lib().poet_launch_count()


def poet_trace_enable(on: bool):
    _check(lib().poet_trace_enable(1 if on else 0))


def poet_trace_set_ridge(flop_per_byte: float):
    _check(lib().poet_trace_set_ridge(float(flop_per_byte)))


def poet_trace_read() -> dict:
    """{kind: {"launches", "ms", "flop", "bytes", "flop_tc", "bytes_hbm"}} of the work recorded since
    tracing was enabled (flop_tc / bytes_hbm: the flops of the launches at or above the ridge, the
    bytes of the others)."""
    rows = (poet_trace_row * 64)()
    n = lib().poet_trace_read(rows, 64)
    return {rows[i].kind.decode(): {"launches": rows[i].launches, "ms": rows[i].ms, "flop": rows[i].flop,
                                    "bytes": rows[i].bytes, "flop_tc": rows[i].flop_tc,
                                    "bytes_hbm": rows[i].bytes_hbm} for i in range(n)}


def poet_version() -> str:
    return lib().poet_version().decode()


# ------------------------------------------------------------------ owning wrapper

class PoetLayer:
    """Owns the device buffers of one POET linear and fills a poet_layer struct.

    W0 (m x n, natural order) and theta_R / theta_P are given by the caller
    (torch tensors on the device); the frame copy, permutations and side
    states are allocated here.  Workspaces are allocated per token count and
    cached.
    """

    def __init__(self, W0, theta_R, theta_P, *, mode, b, k, seed=0, layer_id=0, epoch=0,
                 modeP=None, bP=None, plan=PLAN_AUTO):
        if not W0.is_cuda:
            raise ValueError("W0 must be a CUDA tensor")
        self.dtype = BF16 if W0.dtype == torch.bfloat16 else F32
        if W0.dtype not in (torch.bfloat16, torch.float32):
            raise ValueError("W0 must be float32 or bfloat16")
        self.m, self.n = W0.shape
        dev = W0.device
        self.W0 = W0.contiguous()
        self.theta_R = theta_R.contiguous().float()
        self.theta_P = theta_P.contiguous().float()
        modeP = mode if modeP is None else modeP
        bP = b if bP is None else bP
        self.perm_R = torch.empty(self.m, dtype=torch.int32, device=dev)
        self.perm_P = torch.empty(self.n, dtype=torch.int32, device=dev)
        L = poet_layer()
        L.m, L.n, L.dtype, L.layer_id, L.epoch, L.plan, L.seed = self.m, self.n, self.dtype, layer_id, epoch, plan, seed
        L.R.dim, L.R.mode, L.R.b, L.R.k = self.m, mode, b, k
        L.P.dim, L.P.mode, L.P.b, L.P.k = self.n, modeP, bP, k
        self.state_R = torch.empty(max(poet_side_state_bytes(L.R, self.dtype), 1), dtype=torch.uint8, device=dev)
        self.state_P = torch.empty(max(poet_side_state_bytes(L.P, self.dtype), 1), dtype=torch.uint8, device=dev)
        self.W0f = torch.empty(max(poet_frame_bytes(L), 1), dtype=torch.uint8, device=dev)
        self._L = L
        self._ws = {}
        self._refresh()
        nR, sR = side_geometry(self.m, mode, b)
        nP, sP = side_geometry(self.n, modeP, bP)
        self.geom_R, self.geom_P = (nR, sR), (nP, sP)
        assert self.theta_R.numel() == nR * sR * (sR - 1) // 2 if nR else True, "theta_R has the wrong length"
        assert self.theta_P.numel() == nP * sP * (sP - 1) // 2 if nP else True, "theta_P has the wrong length"

    def _refresh(self):
        L = self._L
        L.W0, L.W0f = self.W0.data_ptr(), self.W0f.data_ptr()
        L.R.perm, L.R.theta, L.R.state = self.perm_R.data_ptr(), self.theta_R.data_ptr(), self.state_R.data_ptr()
        L.P.perm, L.P.theta, L.P.state = self.perm_P.data_ptr(), self.theta_P.data_ptr(), self.state_P.data_ptr()

    @property
    def struct(self) -> poet_layer:
        return self._L

    @property
    def epoch(self) -> int:
        return self._L.epoch

    def workspace(self, T: int):
        if T not in self._ws:
            self._ws[T] = torch.empty(max(poet_workspace_bytes(self._L, T), 1), dtype=torch.uint8,
                                      device=self.W0.device)
        return self._ws[T]

    def plan_for(self, T: int) -> int:
        """PLAN_TOKEN or PLAN_WEIGHT: the plan forward/backward run at T tokens."""
        return poet_plan_for(self._L, T)

    def saved_buffer(self, T: int):
        return torch.empty(max(poet_saved_bytes(self._L, T), 1), dtype=torch.uint8, device=self.W0.device)

    def prepare(self, stream=None):
        poet_prepare(self._L, stream)

    def resample(self, stream=None):
        poet_resample(self._L, stream)

    def cayley_neumann(self, stream=None):
        poet_cayley_neumann(self._L.R, self.dtype, None, stream)
        poet_cayley_neumann(self._L.P, self.dtype, None, stream)

    def forward(self, x, y=None, saved=None, ws=None, stream=None):
        """ws: optional caller workspace (uint8, >= poet_workspace_bytes(T)); work on
        one stream is ordered, so layers may share one workspace."""
        T = x.shape[0]
        if y is None:
            y = torch.empty(T, self.m, dtype=x.dtype, device=x.device)
        if saved is None:
            saved = self.saved_buffer(T)
        poet_forward(self._L, x, T, y, saved, self.workspace(T) if ws is None else ws, stream)
        return y, saved

    def backward(self, saved, dy, dx=None, dtheta_R=None, dtheta_P=None, ws=None, stream=None, x=None):
        """x: the forward's input (read by the weight plan)."""
        T = dy.shape[0]
        if dx is None:
            dx = torch.empty(T, self.n, dtype=dy.dtype, device=dy.device)
        if dtheta_R is None:
            dtheta_R = torch.empty_like(self.theta_R)
        if dtheta_P is None:
            dtheta_P = torch.empty_like(self.theta_P)
        poet_backward(self._L, x, saved, dy, T, dx, dtheta_R, dtheta_P, self.workspace(T) if ws is None else ws,
                      stream)
        return dx, dtheta_R, dtheta_P

    def merge(self, ws=None, stream=None):
        poet_merge(self._L, self.workspace(0) if ws is None else ws, stream)

    def workspace_bytes(self, T: int) -> int:
        return poet_workspace_bytes(self._L, T)

    def block_grad_buffers(self):
        """Float buffers for the per-primitive gradients of R and P ([nprim][ld][ld])."""
        dev = self.W0.device
        return (torch.empty(max(poet_block_grad_bytes(self._L.R) // 4, 4), dtype=torch.float32, device=dev),
                torch.empty(max(poet_block_grad_bytes(self._L.P) // 4, 4), dtype=torch.float32, device=dev))

    def backward_blocks(self, saved, dy, G_R, G_P, dx=None, ws=None, stream=None, x=None):
        """a5..a7: dx and the per-primitive gradients (a8 left to cayley_neumann_grad_many).
        x: the forward's input (read by the weight plan)."""
        T = dy.shape[0]
        if dx is None:
            dx = torch.empty(T, self.n, dtype=dy.dtype, device=dy.device)
        poet_backward_blocks(self._L, x, saved, dy, T, dx, G_R, G_P, self.workspace(T) if ws is None else ws, stream)
        return dx


def cayley_neumann_many(layers, stream=None):
    """a1 for both sides of every layer (all the same dtype) in shared launches."""
    if not layers:
        return
    sides = [s for L in layers for s in (L.struct.R, L.struct.P)]
    poet_cayley_neumann_many(sides, layers[0].dtype, stream)


def cayley_neumann_grad_many_workspace_bytes(layers) -> int:
    if not layers:
        return 0
    sides = [s for L in layers for s in (L.struct.R, L.struct.P)]
    return poet_cayley_neumann_grad_many_workspace_bytes(sides, layers[0].dtype)


def cayley_neumann_grad_many(layers, G, dtheta, ws, stream=None):
    """a8 for every layer: G = [(G_R, G_P), ...], dtheta = [(dtheta_R, dtheta_P), ...]."""
    if not layers:
        return
    sides = [s for L in layers for s in (L.struct.R, L.struct.P)]
    poet_cayley_neumann_grad_many(sides, [t for pair in G for t in pair], [t for pair in dtheta for t in pair],
                                  layers[0].dtype, ws, stream)


# ------------------------------------------------------------------ many layers' forward and backward

def _layer_array(structs):
    arr = (poet_layer * max(len(structs), 1))()
    for i, L in enumerate(structs):
        arr[i] = L
    return arr


def _ptrs(ts):
    return (ctypes.c_void_p * max(len(ts), 1))(*[None if t is None else t.data_ptr() for t in ts])


def _rows(ts):
    """Row strides (elements) of 2-D tensors whose rows are contiguous."""
    for t in ts:
        if t is not None and t.dim() == 2 and t.shape[1] > 1 and t.stride(1) != 1:
            raise ValueError("activation rows must be contiguous (stride(1) == 1)")
    return (ctypes.c_int64 * max(len(ts), 1))(*[0 if t is None else (t.stride(0) if t.dim() == 2 else 0)
                                                for t in ts])


def poet_many_workspace_bytes(structs, T: int, lddy=None) -> int:
    lds = None if lddy is None else (ctypes.c_int64 * max(len(lddy), 1))(*lddy)
    return lib().poet_many_workspace_bytes(_layer_array(structs), len(structs), T, lds)


def poet_forward_many(structs, x, T: int, y, saved, ws, stream=None):
    """x, y: lists of 2-D device tensors (rows contiguous; any row stride >= the width)."""
    _check(lib().poet_forward_many(_layer_array(structs), len(structs), _ptrs(x), _rows(x), T, _ptrs(y), _rows(y),
                                   _ptrs(saved), _ptr(ws), ws.numel(), _stream(stream)))


def poet_backward_blocks_many(structs, x, saved, dy, T: int, dx, G_R, G_P, ws, stream=None):
    _check(lib().poet_backward_blocks_many(_layer_array(structs), len(structs), _ptrs(x), _rows(x), _ptrs(saved),
                                           _ptrs(dy), _rows(dy), T, _ptrs(dx), _rows(dx), _ptrs(G_R), _ptrs(G_P),
                                           _ptr(ws), ws.numel(), _stream(stream)))


def many_workspace_bytes(layers, T: int, dy=None) -> int:
    """Workspace of forward_many / backward_blocks_many over these PoetLayers (dy: the upstream
    gradient tensors, whose row strides decide whether a re-strided copy is needed)."""
    lddy = None if dy is None else [t.stride(0) for t in dy]
    return poet_many_workspace_bytes([L.struct for L in layers], T, lddy)


def forward_many(layers, x, y, saved, ws, stream=None):
    """Forward of independent PoetLayers in grouped launches: y[i] = layer_i(x[i])."""
    if layers:
        poet_forward_many([L.struct for L in layers], x, x[0].shape[0], y, saved, ws, stream)


def backward_blocks_many(layers, x, saved, dy, dx, G, ws, stream=None):
    """a5..a7 of independent PoetLayers in grouped launches; G = [(G_R, G_P), ...]."""
    if layers:
        poet_backward_blocks_many([L.struct for L in layers], x, saved, dy, dy[0].shape[0], dx,
                                  [g[0] for g in G], [g[1] for g in G], ws, stream)


# ------------------------------------------------------------------ a8 with the optimizer step fused

def poet_cayley_neumann_grad_many_adamw(sides, G, m, v, dtype: int, ws, lr, beta1=0.9, beta2=0.999, eps=1e-8,
                                        weight_decay=0.0, step=1, dtheta=None, stream=None):
    """a8 for every side with the AdamW step applied to each side's theta in the packing kernel."""
    h = poet_adamw_hparams(lr, beta1, beta2, eps, weight_decay, step)
    n = len(sides)
    dp = None if dtheta is None else _ptrs(dtheta)
    _check(lib().poet_cayley_neumann_grad_many_adamw(_side_array(sides), _ptrs(G), _ptrs(m), _ptrs(v), dp, n, dtype,
                                                     ctypes.byref(h), _ptr(ws), 0 if ws is None else ws.numel(),
                                                     _stream(stream)))


def poet_merge_reset_moments(layer: poet_layer, m_R, v_R, m_P, v_P, ws, stream=None):
    _check(lib().poet_merge_reset_moments(ctypes.byref(layer), _ptr(m_R), _ptr(v_R), _ptr(m_P), _ptr(v_P), _ptr(ws),
                                          ws.numel(), _stream(stream)))


def poet_workspace_size(layer: poet_layer, T: int) -> int:
    return lib().poet_workspace_size(ctypes.byref(layer), T)


# ------------------------------------------------------------------ one LLaMA block around seven POET linears

class PoetBlock:
    """One LLaMA block whose linears q, k, v, o, gate, up, down are PoetLayers
    (bf16).  forward() saves what backward() needs; backward() returns dh and
    the packed-skew gradients of the fourteen sides (a8 grouped)."""

    NAMES = ("q", "k", "v", "o", "gate", "up", "down")

    def __init__(self, layers, seq_len, heads, head_dim, rope_base=10000.0, norm_eps=1e-6):
        if len(layers) != 7:
            raise ValueError("a block takes seven PoetLayers: q, k, v, o, gate, up, down")
        self.layers = list(layers)
        self.hidden = layers[0].m
        b = poet_llama_block()
        b.seq_len, b.heads, b.head_dim, b.rope_base, b.norm_eps = seq_len, heads, head_dim, rope_base, norm_eps
        self._b = b
        self._sync()
        self._ws = {}

    def _sync(self):
        for i, L in enumerate(self.layers):
            self._b.lin[i] = L.struct

    @property
    def struct(self):
        self._sync()
        return self._b

    def saved_bytes(self, T):
        return lib().poet_llama_block_saved_bytes(ctypes.byref(self.struct), T)

    def workspace(self, T):
        if T not in self._ws:
            n = lib().poet_llama_block_workspace_bytes(ctypes.byref(self.struct), T)
            self._ws[T] = torch.empty(max(n, 1), dtype=torch.uint8, device=self.layers[0].W0.device)
        return self._ws[T]

    def forward(self, h, out=None, saved=None, stream=None):
        T = h.shape[0]
        if out is None:
            out = torch.empty_like(h)
        if saved is None:
            saved = torch.empty(max(self.saved_bytes(T), 1), dtype=torch.uint8, device=h.device)
        ws = self.workspace(T)
        _check(lib().poet_llama_block_forward(ctypes.byref(self.struct), _ptr(h), T, _ptr(out), _ptr(saved), _ptr(ws),
                                              ws.numel(), _stream(stream)))
        return out, saved

    def backward(self, saved, dout, dh=None, G=None, stream=None):
        """dh and G = [(G_R, G_P), ...] per linear (per-primitive gradients)."""
        T = dout.shape[0]
        if dh is None:
            dh = torch.empty_like(dout)
        if G is None:
            G = [L.block_grad_buffers() for L in self.layers]
        ws = self.workspace(T)
        gp = _ptrs([g for pair in G for g in pair])
        _check(lib().poet_llama_block_backward(ctypes.byref(self.struct), _ptr(saved), _ptr(dout), T, _ptr(dh), gp,
                                               _ptr(ws), ws.numel(), _stream(stream)))
        return dh, G

    def theta_grads(self, G, ws=None, stream=None):
        """a8 of the fourteen sides: [(dtheta_R, dtheta_P), ...]."""
        dth = [(torch.empty_like(L.theta_R), torch.empty_like(L.theta_P)) for L in self.layers]
        if ws is None:
            n = cayley_neumann_grad_many_workspace_bytes(self.layers)
            ws = torch.empty(max(n, 1), dtype=torch.uint8, device=self.layers[0].W0.device)
        cayley_neumann_grad_many(self.layers, G, dth, ws, stream)
        return dth

"""Python binding of libpisa.so (PISA pyramid block-sparse attention for B200).

Argument marshalling only: every step of the method runs in the CUDA kernels
behind the C ABI of include/pisa.h. PyTorch supplies device memory and the
current stream. There is no CPU fallback: importing this package fails if the
compiled library is missing, and every call raises PisaError on a non-OK
status.
"""
from __future__ import annotations

import ctypes
import dataclasses
import math
import os

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libpisa.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(f"libpisa.so is not built ({LIB_PATH}); run __graft_entry__.build() first")
_lib = ctypes.CDLL(LIB_PATH)

MAX_LEVELS = 24
MAX_CANDIDATES = 4096

STATUS = {0: "PISA_OK", 1: "PISA_ERR_INVALID_ARG", 2: "PISA_ERR_UNSUPPORTED", 3: "PISA_ERR_WORKSPACE",
          4: "PISA_ERR_CUDA", 5: "PISA_ERR_TIMEOUT", 6: "PISA_ERR_BAD_INDEX"}
OK, ERR_INVALID_ARG, ERR_UNSUPPORTED, ERR_WORKSPACE, ERR_CUDA, ERR_TIMEOUT, ERR_BAD_INDEX = range(7)


class PisaShape(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int32) for n in ("batch", "heads_q", "heads_kv", "seq_q", "seq_kv", "head_dim",
                                               "block", "factor", "topk", "causal", "select_per_qhead")] + \
               [("scale", ctypes.c_float), ("forced_blocks", ctypes.c_int32), ("kv_capacity", ctypes.c_int32)]

FORCE_SINK, FORCE_LOCAL = 1, 2   # pisa_shape.forced_blocks bits


class PisaError(RuntimeError):
    def __init__(self, status: int, where: str, detail: int | None = None):
        self.status = status
        self.detail = detail
        msg = f"{where}: {STATUS.get(status, status)} ({_lib.pisa_status_string(status).decode()})"
        if detail is not None:
            msg += f" detail=0x{detail:x}"
        super().__init__(msg)


_vp, _i32p, _f32p, _szp = ctypes.c_void_p, ctypes.POINTER(ctypes.c_int32), ctypes.c_void_p, ctypes.POINTER(ctypes.c_size_t)
_SP = ctypes.POINTER(PisaShape)
_sig = {
    "pisa_num_levels": (ctypes.c_int32, [_SP]),
    "pisa_level_layout": (ctypes.c_int, [_SP, _i32p, _i32p]),
    "pisa_pyramid_size": (ctypes.c_int, [_SP, _szp]),
    "pisa_workspace_size": (ctypes.c_int, [_SP, _szp]),
    "pisa_build_pyramid": (ctypes.c_int, [_SP, _vp, _vp, _vp]),
    "pisa_append_pyramid": (ctypes.c_int, [_SP, _vp, _vp, ctypes.c_int32, _vp]),
    "pisa_backward_workspace_size": (ctypes.c_int, [_SP, _szp]),
    "pisa_sparse_attention_backward": (ctypes.c_int, [_SP, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp,
                                                      ctypes.c_size_t, _vp]),
    "pisa_select_blocks": (ctypes.c_int, [_SP, _vp, _vp, _i32p, _vp, _vp, _vp, ctypes.c_size_t, _vp]),
    "pisa_sparse_attention": (ctypes.c_int, [_SP, _vp, _vp, _vp, _vp, _vp, _vp, _vp, ctypes.c_size_t, _vp]),
    "pisa_forward": (ctypes.c_int, [_SP, _vp, _vp, _vp, _vp, _vp, _vp, _vp, ctypes.c_size_t, _vp]),
    "pisa_check_status": (ctypes.c_int, [_vp, ctypes.POINTER(ctypes.c_uint32), _vp]),
    "pisa_status_string": (ctypes.c_char_p, [ctypes.c_int]),
    "pisa_last_launch_count": (ctypes.c_int32, []),
    "pisa_decode_attention_noalloc": (ctypes.c_int, [_SP, _vp, _vp, _vp, _vp, _vp, _vp, _vp]),
    "pisa_decode_noalloc_check_status": (ctypes.c_int, [ctypes.POINTER(ctypes.c_uint32), _vp]),
    "pisa_selftest_wait_timeout": (ctypes.c_int, [_vp, ctypes.c_uint32, _vp]),
}
for _name, (_res, _args) in _sig.items():
    _f = getattr(_lib, _name)
    _f.restype = _res
    _f.argtypes = _args

EXPORTED = tuple(_sig)


@dataclasses.dataclass(frozen=True)
class Shape:
    """Problem description (mirrors pisa_shape)."""
    batch: int
    heads_q: int
    heads_kv: int
    seq_q: int
    seq_kv: int
    head_dim: int
    block: int
    factor: int
    topk: int
    causal: int = 0
    select_per_qhead: int = 0
    scale: float = 0.0
    forced_blocks: int = 0   # FORCE_SINK | FORCE_LOCAL
    kv_capacity: int = 0     # decode over a growing cache: K/V rows per plane (0 = seq_kv)

    def c(self) -> PisaShape:
        return PisaShape(self.batch, self.heads_q, self.heads_kv, self.seq_q, self.seq_kv, self.head_dim,
                         self.block, self.factor, self.topk, int(self.causal), int(self.select_per_qhead),
                         float(self.scale), int(self.forced_blocks), int(self.kv_capacity))

    @property
    def decode(self) -> bool:
        return self.seq_q == 1

    @property
    def n_blocks(self) -> int:
        return self.seq_kv // self.block

    @property
    def kv_rows(self) -> int:
        """Rows of one K/V plane: the capacity of a growing cache, else seq_kv."""
        return self.kv_capacity or self.seq_kv

    @property
    def hsel(self) -> int:
        return self.heads_q if self.select_per_qhead else self.heads_kv

    @property
    def n_qblocks(self) -> int:
        return 1 if self.decode else self.seq_q // self.block

    @classmethod
    def of(cls, w, **kw) -> "Shape":
        """Shape of a workload description (any object with the same field names)."""
        f = {k: getattr(w, k) for k in ("batch", "heads_q", "heads_kv", "seq_q", "seq_kv", "head_dim", "block",
                                        "factor", "topk", "causal")}
        f.update(kw)
        return cls(**f)


def _check(status: int, where: str) -> None:
    if status != OK:
        raise PisaError(status, where)


def num_levels(shape: Shape) -> int:
    return int(_lib.pisa_num_levels(ctypes.byref(shape.c())))


def level_layout(shape: Shape) -> tuple[list[int], list[int]]:
    sizes = (ctypes.c_int32 * MAX_LEVELS)()
    offs = (ctypes.c_int32 * MAX_LEVELS)()
    _check(_lib.pisa_level_layout(ctypes.byref(shape.c()), sizes, offs), "pisa_level_layout")
    n = num_levels(shape)
    return list(sizes[:n]), list(offs[:n])


def pyramid_size(shape: Shape) -> int:
    n = ctypes.c_size_t()
    _check(_lib.pisa_pyramid_size(ctypes.byref(shape.c()), ctypes.byref(n)), "pisa_pyramid_size")
    return n.value


def workspace_size(shape: Shape) -> int:
    n = ctypes.c_size_t()
    _check(_lib.pisa_workspace_size(ctypes.byref(shape.c()), ctypes.byref(n)), "pisa_workspace_size")
    return n.value


def last_launch_count() -> int:
    return int(_lib.pisa_last_launch_count())


# ----------------------------------------------------------------------------- torch-facing calls

def _torch():
    import torch
    return torch


def _ptr(t) -> int | None:
    return None if t is None else t.data_ptr()


def _stream(stream=None) -> int:
    torch = _torch()
    s = stream if stream is not None else torch.cuda.current_stream()
    return s.cuda_stream


def _need(t, dtype, shape, name):
    torch = _torch()
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return t


def new_workspace(shape: Shape, device) -> "object":
    """Zeroed workspace (the status word must start at zero)."""
    torch = _torch()
    return torch.zeros(workspace_size(shape), dtype=torch.uint8, device=device)


def build_pyramid(shape: Shape, K, pyramid=None, stream=None):
    torch = _torch()
    D = shape.head_dim
    _need(K, torch.bfloat16, (shape.batch, shape.heads_kv, shape.kv_rows, D), "K")
    sizes, _ = level_layout(shape)
    if pyramid is None:
        pyramid = torch.empty((shape.batch, shape.heads_kv, sum(sizes), D), dtype=torch.float32, device=K.device)
    _check(_lib.pisa_build_pyramid(ctypes.byref(shape.c()), _ptr(K), _ptr(pyramid), _stream(stream)),
           "pisa_build_pyramid")
    return pyramid


def append_pyramid(shape: Shape, K, pyramid, seq_kv_old: int, stream=None):
    """Brings `pyramid` (the pyramid of the cache at length seq_kv_old) up to shape.seq_kv."""
    torch = _torch()
    _need(K, torch.bfloat16, (shape.batch, shape.heads_kv, shape.kv_rows, shape.head_dim), "K")
    _check(_lib.pisa_append_pyramid(ctypes.byref(shape.c()), _ptr(K), _ptr(pyramid), int(seq_kv_old), _stream(stream)),
           "pisa_append_pyramid")
    return pyramid


def select_blocks(shape: Shape, Q, pyramid, ws, level_budget=None, idx=None, margin=False, stream=None):
    torch = _torch()
    _need(Q, torch.bfloat16, (shape.batch, shape.heads_q, shape.seq_q, shape.head_dim), "Q")
    if idx is None:
        idx = torch.empty((shape.batch, shape.hsel, shape.n_qblocks, shape.topk), dtype=torch.int32, device=Q.device)
    marg = torch.empty((shape.batch, shape.hsel, shape.n_qblocks), dtype=torch.float32, device=Q.device) \
        if margin else None
    budget = None
    if level_budget is not None:
        budget = (ctypes.c_int32 * len(level_budget))(*[int(x) for x in level_budget])
    _check(_lib.pisa_select_blocks(ctypes.byref(shape.c()), _ptr(Q), _ptr(pyramid), budget, _ptr(idx), _ptr(marg),
                                   _ptr(ws), ws.numel(), _stream(stream)), "pisa_select_blocks")
    return (idx, marg) if margin else idx


def sparse_attention(shape: Shape, Q, K, V, idx, ws, O=None, lse=True, stream=None):
    torch = _torch()
    B, Hq, Nq, D = shape.batch, shape.heads_q, shape.seq_q, shape.head_dim
    _need(Q, torch.bfloat16, (B, Hq, Nq, D), "Q")
    if O is None:
        O = torch.empty_like(Q)
    L = torch.empty((B, Hq, Nq), dtype=torch.float32, device=Q.device) if lse is True else lse
    _check(_lib.pisa_sparse_attention(ctypes.byref(shape.c()), _ptr(Q), _ptr(K), _ptr(V), _ptr(idx), _ptr(O),
                                      _ptr(L), _ptr(ws), ws.numel(), _stream(stream)), "pisa_sparse_attention")
    return O, L


def forward(shape: Shape, Q, K, V, ws, O=None, lse=True, idx=None, stream=None):
    """Pyramid, selection and attention in one call. Returns (O, lse, idx or None)."""
    torch = _torch()
    B, Hq, Nq, D = shape.batch, shape.heads_q, shape.seq_q, shape.head_dim
    _need(Q, torch.bfloat16, (B, Hq, Nq, D), "Q")
    _need(K, torch.bfloat16, (B, shape.heads_kv, shape.kv_rows, D), "K")
    _need(V, torch.bfloat16, (B, shape.heads_kv, shape.kv_rows, D), "V")
    if O is None:
        O = torch.empty_like(Q)
    L = torch.empty((B, Hq, Nq), dtype=torch.float32, device=Q.device) if lse is True else lse
    if idx is True:
        idx = torch.empty((B, shape.hsel, shape.n_qblocks, shape.topk), dtype=torch.int32, device=Q.device)
    _check(_lib.pisa_forward(ctypes.byref(shape.c()), _ptr(Q), _ptr(K), _ptr(V), _ptr(O), _ptr(L), _ptr(idx),
                             _ptr(ws), ws.numel(), _stream(stream)), "pisa_forward")
    return O, L, idx


def decode_attention_noalloc(shape: Shape, Q, K, V, idx, O=None, lse=True, stream=None):
    """Decode attention with the library's built-in scratch (no workspace, no allocation inside)."""
    torch = _torch()
    B, Hq, D = shape.batch, shape.heads_q, shape.head_dim
    _need(Q, torch.bfloat16, (B, Hq, 1, D), "Q")
    if O is None:
        O = torch.empty_like(Q)
    L = torch.empty((B, Hq, 1), dtype=torch.float32, device=Q.device) if lse is True else lse
    _check(_lib.pisa_decode_attention_noalloc(ctypes.byref(shape.c()), _ptr(Q), _ptr(K), _ptr(V), _ptr(idx),
                                              _ptr(O), _ptr(L), _stream(stream)), "pisa_decode_attention_noalloc")
    return O, L


def decode_noalloc_check_status(stream=None) -> tuple[int, int]:
    """Synchronises the stream; returns (status, detail) that the last decode_attention_noalloc
    call's kernels recorded in the library's built-in array, and clears them."""
    detail = ctypes.c_uint32()
    st = _lib.pisa_decode_noalloc_check_status(ctypes.byref(detail), _stream(stream))
    return int(st), int(detail.value)


def backward_workspace_size(shape: Shape) -> int:
    n = ctypes.c_size_t(0)
    _check(_lib.pisa_backward_workspace_size(ctypes.byref(shape.c()), ctypes.byref(n)), "pisa_backward_workspace_size")
    return n.value


def sparse_attention_backward(shape: Shape, Q, K, V, O, lse, dO, idx, ws=None, dQ=None, dK=None, dV=None,
                              stream=None):
    """dQ, dK, dV of the sparse attention step for the selection `idx` (prefill)."""
    torch = _torch()
    B, Hq, N, D = shape.batch, shape.heads_q, shape.seq_q, shape.head_dim
    for t, name in ((Q, "Q"), (O, "O"), (dO, "dO")):
        _need(t, torch.bfloat16, (B, Hq, N, D), name)
    for t, name in ((K, "K"), (V, "V")):
        _need(t, torch.bfloat16, (B, shape.heads_kv, shape.kv_rows, D), name)
    _need(lse, torch.float32, (B, Hq, N), "lse")
    _need(idx, torch.int32, (B, shape.hsel, shape.n_qblocks, shape.topk), "idx")
    if ws is None:
        ws = torch.zeros(backward_workspace_size(shape), dtype=torch.uint8, device=Q.device)
    dQ = torch.empty_like(Q) if dQ is None else dQ
    dK = torch.empty_like(K) if dK is None else dK
    dV = torch.empty_like(V) if dV is None else dV
    _check(_lib.pisa_sparse_attention_backward(ctypes.byref(shape.c()), _ptr(Q), _ptr(K), _ptr(V), _ptr(O), _ptr(lse),
                                               _ptr(dO), _ptr(idx), _ptr(dQ), _ptr(dK), _ptr(dV), _ptr(ws), ws.numel(),
                                               _stream(stream)), "pisa_sparse_attention_backward")
    return dQ, dK, dV


def check_status(ws, stream=None) -> tuple[int, int]:
    """Synchronises the stream; returns (status, detail) recorded by kernels and clears them."""
    detail = ctypes.c_uint32()
    st = _lib.pisa_check_status(_ptr(ws), ctypes.byref(detail), _stream(stream))
    return int(st), int(detail.value)


def selftest_wait_timeout(ws, limit_us: int, stream=None) -> None:
    """Enqueues the bounded-wait self-test: a wait that never completes gives up after limit_us
    and records PISA_ERR_TIMEOUT in the workspace status word (read it with check_status)."""
    _check(_lib.pisa_selftest_wait_timeout(_ptr(ws), int(limit_us), _stream(stream)), "pisa_selftest_wait_timeout")


def raise_on_device_error(ws, where="device", stream=None) -> None:
    st, detail = check_status(ws, stream)
    if st != OK:
        raise PisaError(st, where, detail)


class Session:
    """Preallocated device buffers for repeated forwards of one shape.

    `forward` accepts host (CPU, ideally pinned) or device tensors. With host
    inputs the (batch, KV head) planes, which the method treats independently,
    are split into `units` ranges and pipelined over three streams: the copy
    of a range's Q, K and V to the device (copy stream), pisa_forward on that
    range (the caller's current stream) and the copy of its O back to the host
    (output stream), so that host-device transfers in both directions overlap
    the computation of other ranges. Each range is one pisa_forward call on a
    shape with batch = planes in the range, heads_q = g, heads_kv = 1; for
    prefill its results equal those of one call on the whole shape bit for bit.
    """

    def __init__(self, shape: Shape, device="cuda", units: int = 8):
        torch = _torch()
        self.shape = shape
        self.device = torch.device(device)
        s = shape
        self.ws = new_workspace(shape, self.device)
        self.q = torch.empty((s.batch, s.heads_q, s.seq_q, s.head_dim), dtype=torch.bfloat16, device=self.device)
        self.k = torch.empty((s.batch, s.heads_kv, s.kv_rows, s.head_dim), dtype=torch.bfloat16, device=self.device)
        self.v = torch.empty_like(self.k)
        self.o = torch.empty_like(self.q)
        self.lse = torch.empty((s.batch, s.heads_q, s.seq_q), dtype=torch.float32, device=self.device)
        planes = s.batch * s.heads_kv
        n = max(1, min(units, planes))
        bounds = [planes * u // n for u in range(n + 1)]
        self.ranges = [(a, b) for a, b in zip(bounds, bounds[1:]) if b > a]
        g = s.heads_q // s.heads_kv
        self.unit_shapes = {b - a: dataclasses.replace(s, batch=b - a, heads_q=g, heads_kv=1) for a, b in self.ranges}
        self.unit_ws = new_workspace(max(self.unit_shapes.values(), key=workspace_size), self.device)
        self.copy_stream = torch.cuda.Stream(self.device)
        self.out_stream = torch.cuda.Stream(self.device)

    def _planes(self, t, per_plane):
        """View of a [B, H, ...] tensor as [planes, per_plane, ...] (planes = B * heads_kv)."""
        return t.view(self.shape.batch * self.shape.heads_kv, per_plane, *t.shape[2:])

    def forward(self, Q, K, V, out=None):
        torch = _torch()
        if Q.is_cuda:
            O, _, _ = forward(self.shape, Q, K, V, self.ws, O=self.o, lse=self.lse)
            return O
        s = self.shape
        g = s.heads_q // s.heads_kv
        if out is None:
            out = torch.empty(tuple(self.o.shape), dtype=self.o.dtype, pin_memory=True)
        hq, hk, hv, ho = self._planes(Q, g), self._planes(K, 1), self._planes(V, 1), self._planes(out, g)
        dq, dk, dv, do = self._planes(self.q, g), self._planes(self.k, 1), self._planes(self.v, 1), self._planes(self.o, g)
        dl = self.lse.view(s.batch * s.heads_kv, g, s.seq_q)
        compute = torch.cuda.current_stream(self.device)
        arrived = []
        # inputs: every range back to back on the copy stream (after earlier work on these buffers)
        self.copy_stream.wait_stream(compute)
        with torch.cuda.stream(self.copy_stream):
            for a, b in self.ranges:
                dq[a:b].copy_(hq[a:b], non_blocking=True)
                dk[a:b].copy_(hk[a:b], non_blocking=True)
                dv[a:b].copy_(hv[a:b], non_blocking=True)
                ev = torch.cuda.Event()
                ev.record(self.copy_stream)
                arrived.append(ev)
        self.out_stream.wait_stream(compute)
        for (a, b), ev in zip(self.ranges, arrived):
            compute.wait_event(ev)
            forward(self.unit_shapes[b - a], dq[a:b], dk[a:b], dv[a:b], self.unit_ws, O=do[a:b], lse=dl[a:b],
                    stream=compute)
            done = torch.cuda.Event()
            done.record(compute)
            self.out_stream.wait_event(done)
            with torch.cuda.stream(self.out_stream):
                ho[a:b].copy_(do[a:b], non_blocking=True)
        compute.wait_stream(self.out_stream)
        return out


# ----------------------------------------------------------------------------- measurement helpers

def attention_pairs(idx: np.ndarray, shape: Shape) -> int:
    """Unmasked (query, key) pairs the attention evaluates for a selection (host arithmetic).

    A selected block j < i contributes b*b pairs per query head, the diagonal
    block (causal) b(b+1)/2; decode contributes b per selected block per head.
    """
    b = shape.block
    heads_per_row = 1 if shape.select_per_qhead else shape.heads_q // shape.heads_kv
    valid = idx >= 0
    if shape.decode:
        return int(valid.sum()) * b * heads_per_row
    full = int(valid.sum()) * b * b
    if shape.causal:
        i = np.arange(idx.shape[2]).reshape(1, 1, -1, 1)
        diag = int(((idx == i) & valid).sum())
        full -= diag * (b * b - b * (b + 1) // 2)
    return full * heads_per_row


def attention_flops(idx: np.ndarray, shape: Shape) -> float:
    """Algorithmic FLOPs of the attention step: 4 * D per unmasked (query, key) pair (QK^T and PV)."""
    return 4.0 * shape.head_dim * attention_pairs(idx, shape)


def default_scale(shape: Shape) -> float:
    return shape.scale if shape.scale > 0 else 1.0 / math.sqrt(shape.head_dim)

"""Tensor-level binding of the asffn C ABI (same names as include/asffn.h).

torch supplies device memory and streams; every step of the path runs in
libasffn.so's CUDA kernels.  These wrappers only check that tensors live where
the C ABI expects them (device or host), build the descriptor structs and
marshal pointers; a non-OK status raises ``AsfError``.
"""
from __future__ import annotations

import ctypes
from typing import Optional

import numpy as np
import torch

from . import _lib as L
from ._lib import AsfError, check  # noqa: F401

_DT = {torch.float16: L.ASF_F16, torch.float32: L.ASF_F32}
_ACT = {"relu": L.ASF_ACT_RELU, "reglu": L.ASF_ACT_REGLU}


def _dev(t: torch.Tensor, name: str, dtype=None) -> ctypes.c_void_p:
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"{name} must have dtype {dtype}, got {t.dtype}")
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    if isinstance(stream, torch.cuda.Stream):
        return ctypes.c_void_p(stream.cuda_stream)
    return ctypes.c_void_p(int(stream))


class Predictor:
    """Descriptor of the two-layer predictor: W1 [r,d], b1 [r], W2 [n,r], b2 [n]."""

    def __init__(self, W1: torch.Tensor, b1: torch.Tensor, W2: torch.Tensor, b2: torch.Tensor):
        if W1.dtype not in _DT or W2.dtype != W1.dtype:
            raise ValueError("W1/W2 must both be float16 or float32")
        r, d = W1.shape
        n, r2 = W2.shape
        if r2 != r or b1.shape != (r,) or b2.shape != (n,):
            raise ValueError("predictor shapes do not agree")
        self.tensors = (W1, b1, W2, b2)
        self.d, self.r, self.n, self.dtype = d, r, n, W1.dtype
        self.desc = L.asf_predictor(d, r, n, _DT[W1.dtype], _dev(W1, "W1"),
                                    _dev(b1, "b1", torch.float32), _dev(W2, "W2"),
                                    _dev(b2, "b2", torch.float32))


class FFN:
    """Descriptor of one FFN layer in storage order: Wg/Wu/WdT [n,d], bias [n]."""

    @classmethod
    def packed(cls, act: str, packed: torch.Tensor, bias: torch.Tensor, hot_rows: int = 0) -> "FFN":
        """Layer in the neuron-major packed layout: packed[k] = [gate_k | up_k | down_k]
        (ReGLU, shape [n, 3, d]) or [up_k | down_k] (ReLU, shape [n, 2, d])."""
        if act not in _ACT or packed.dim() != 3 or packed.dtype not in _DT:
            raise ValueError("packed must be [n, m, d] float16/float32")
        n, m, d = packed.shape
        if m != (3 if act == "reglu" else 2) or bias.shape != (n,):
            raise ValueError("packed layer shape does not match the activation")
        base = _dev(packed, "packed").value
        rb = d * packed.element_size()
        self = cls.__new__(cls)
        self.tensors = (packed, bias)
        self.act, self.d, self.n, self.dtype = act, d, n, packed.dtype
        self.hot_rows = int(hot_rows)
        gp = ctypes.c_void_p(base) if act == "reglu" else ctypes.c_void_p(0)
        up = ctypes.c_void_p(base + (rb if act == "reglu" else 0))
        dn = ctypes.c_void_p(base + (m - 1) * rb)
        self.desc = L.asf_ffn(d, n, _DT[packed.dtype], _ACT[act], gp, up, dn,
                              _dev(bias, "bias", torch.float32), self.hot_rows, m * d)
        return self

    def __init__(self, act: str, Wg: Optional[torch.Tensor], Wu: torch.Tensor, WdT: torch.Tensor,
                 bias: torch.Tensor, hot_rows: int = 0):
        if act not in _ACT:
            raise ValueError("act must be 'reglu' or 'relu'")
        if Wu.dtype not in _DT or WdT.dtype != Wu.dtype:
            raise ValueError("weights must be float16 or float32")
        n, d = Wu.shape
        if WdT.shape != (n, d) or bias.shape != (n,):
            raise ValueError("FFN shapes do not agree")
        if act == "reglu":
            if Wg is None or Wg.shape != (n, d) or Wg.dtype != Wu.dtype:
                raise ValueError("ReGLU needs a gate matrix shaped like W_up")
            gp = _dev(Wg, "Wg")
        else:
            gp = ctypes.c_void_p(0)
        self.tensors = (Wg, Wu, WdT, bias)
        self.act, self.d, self.n, self.dtype = act, d, n, Wu.dtype
        self.hot_rows = int(hot_rows)
        self.desc = L.asf_ffn(d, n, _DT[Wu.dtype], _ACT[act], gp, _dev(Wu, "Wu"), _dev(WdT, "WdT"),
                              _dev(bias, "bias", torch.float32), self.hot_rows, 0)

    def set_l2_next(self, *ranges: torch.Tensor) -> "FFN":
        """L2 prefetch hint (asf_ffn.l2_next): up to two contiguous device
        tensors that are read soon after each sparse-FFN call on this layer,
        typically the next layer's predictor weights.  No argument clears it."""
        if len(ranges) > 2:
            raise ValueError("at most two ranges")
        ptrs = [_dev(t, "l2_next") for t in ranges]
        self.l2_next = tuple(ranges)          # keeps the memory alive
        for i in range(2):
            self.desc.l2_next[i] = ptrs[i].value if i < len(ptrs) else None
            self.desc.l2_next_bytes[i] = ranges[i].numel() * ranges[i].element_size() if i < len(ranges) else 0
        return self


def asf_version() -> int:
    return int(L.load().asf_version())


def asf_workspace_bytes(pred: Optional[Predictor], ffn: Optional[FFN], max_batch: int) -> int:
    lib = L.load()
    p = ctypes.byref(pred.desc) if pred is not None else None
    f = ctypes.byref(ffn.desc) if ffn is not None else None
    return int(lib.asf_workspace_bytes(p, f, int(max_batch)))


class Workspace:
    """Device scratch for one stream: sized by asf_workspace_bytes, zeroed once."""

    def __init__(self, pred: Optional[Predictor], ffn: Optional[FFN], max_batch: int, device=None,
                 stream=None):
        nbytes = asf_workspace_bytes(pred, ffn, max_batch)
        if nbytes == 0:
            raise AsfError(L.ASF_ERR_INVALID_ARG, "asf_workspace_bytes")
        dev = device if device is not None else (ffn or pred).tensors[-1].device
        self.buf = torch.empty(nbytes, dtype=torch.uint8, device=dev)
        self.nbytes = nbytes
        asf_workspace_init(self, stream)

    @property
    def ptr(self) -> ctypes.c_void_p:
        return ctypes.c_void_p(self.buf.data_ptr())


def asf_workspace_init(ws: Workspace, stream=None) -> None:
    check(L.load().asf_workspace_init(ws.ptr, ws.nbytes, _stream(stream)), "asf_workspace_init")


def asf_predict(pred: Predictor, x: torch.Tensor, tau: float, idx: torch.Tensor, count: torch.Tensor,
                ws: Workspace, stream=None) -> None:
    """idx[:count] = ascending union of neurons with sigmoid(W2 ReLU(W1 x + b1) + b2) > tau."""
    if x.dtype != pred.dtype or x.dim() != 2 or x.shape[1] != pred.d:
        raise ValueError("x must be [B, d] in the predictor's dtype")
    st = L.load().asf_predict(ctypes.byref(pred.desc), _dev(x, "x"), int(x.shape[0]), float(tau),
                              _dev(idx, "idx", torch.int32), _dev(count, "count", torch.int32),
                              ws.ptr, ws.nbytes, _stream(stream))
    check(st, "asf_predict")


def asf_sparse_ffn(ffn: FFN, x: torch.Tensor, idx: torch.Tensor, count: torch.Tensor, y: torch.Tensor,
                   ws: Workspace, stream=None) -> None:
    """y = sum over the first count entries k of idx of a_k(x) * WdT[k]."""
    if x.dtype != ffn.dtype or x.dim() != 2 or x.shape[1] != ffn.d:
        raise ValueError("x must be [B, d] in the FFN's dtype")
    if y.shape != (x.shape[0], ffn.d):
        raise ValueError("y must be [B, d]")
    st = L.load().asf_sparse_ffn(ctypes.byref(ffn.desc), _dev(x, "x"), int(x.shape[0]),
                                 _dev(idx, "idx", torch.int32), _dev(count, "count", torch.int32),
                                 _dev(y, "y", torch.float32), ws.ptr, ws.nbytes, _stream(stream))
    check(st, "asf_sparse_ffn")


def asf_predict_sparse_ffn(pred: Predictor, ffn: FFN, x: torch.Tensor, tau: float, idx: torch.Tensor,
                           count: torch.Tensor, y: torch.Tensor, ws: Workspace, stream=None) -> None:
    """One layer: asf_predict then asf_sparse_ffn over the predicted list, in
    one call (same idx, count and y); ws must be sized with both descriptors."""
    if x.dtype != ffn.dtype or x.dim() != 2 or x.shape[1] != ffn.d:
        raise ValueError("x must be [B, d] in the FFN's dtype")
    if y.shape != (x.shape[0], ffn.d):
        raise ValueError("y must be [B, d]")
    st = L.load().asf_predict_sparse_ffn(ctypes.byref(pred.desc), ctypes.byref(ffn.desc), _dev(x, "x"),
                                         int(x.shape[0]), float(tau), _dev(idx, "idx", torch.int32),
                                         _dev(count, "count", torch.int32), _dev(y, "y", torch.float32),
                                         ws.ptr, ws.nbytes, _stream(stream))
    check(st, "asf_predict_sparse_ffn")


def _layer_call(name: str, pred: Predictor, ffn: FFN, x: torch.Tensor, tau: float, idx: torch.Tensor,
                count: torch.Tensor, y: torch.Tensor, ws: Workspace, stream=None) -> None:
    if x.dtype != ffn.dtype or x.dim() != 2 or x.shape[1] != ffn.d:
        raise ValueError("x must be [B, d] in the FFN's dtype")
    if y.shape != (x.shape[0], ffn.d):
        raise ValueError("y must be [B, d]")
    st = getattr(L.load(), name)(ctypes.byref(pred.desc), ctypes.byref(ffn.desc), _dev(x, "x"),
                                 int(x.shape[0]), float(tau), _dev(idx, "idx", torch.int32),
                                 _dev(count, "count", torch.int32), _dev(y, "y", torch.float32),
                                 ws.ptr, ws.nbytes, _stream(stream))
    check(st, name)


def asf_predict_sparse_ffn_begin(pred: Predictor, ffn: FFN, x: torch.Tensor, tau: float, idx: torch.Tensor,
                                 count: torch.Tensor, y: torch.Tensor, ws: Workspace, stream=None) -> None:
    """First half of asf_predict_sparse_ffn (the predictor's kernels)."""
    _layer_call("asf_predict_sparse_ffn_begin", pred, ffn, x, tau, idx, count, y, ws, stream)


def asf_predict_sparse_ffn_end(pred: Predictor, ffn: FFN, x: torch.Tensor, tau: float, idx: torch.Tensor,
                               count: torch.Tensor, y: torch.Tensor, ws: Workspace, stream=None) -> None:
    """Second half of asf_predict_sparse_ffn (compaction if needed, the sparse
    FFN); with the same arguments after _begin it completes the layer."""
    _layer_call("asf_predict_sparse_ffn_end", pred, ffn, x, tau, idx, count, y, ws, stream)


def asf_predict_sparse_ffn_exchange(pred: Predictor, ffn: FFN, x: torch.Tensor, tau: float, idx: torch.Tensor,
                                    count: torch.Tensor, y: torch.Tensor, ws: Workspace, group,
                                    stream=None) -> None:
    """One layer of a neuron-sharded model on this rank, with y summed over the
    ranks of ``group`` (an ``asf_peer_group`` descriptor) through peer memory
    inside the layer's last kernel."""
    if x.dtype != ffn.dtype or x.dim() != 2 or x.shape[1] != ffn.d:
        raise ValueError("x must be [B, d] in the FFN's dtype")
    if y.shape != (x.shape[0], ffn.d):
        raise ValueError("y must be [B, d]")
    st = L.load().asf_predict_sparse_ffn_exchange(
        ctypes.byref(pred.desc), ctypes.byref(ffn.desc), _dev(x, "x"), int(x.shape[0]), float(tau),
        _dev(idx, "idx", torch.int32), _dev(count, "count", torch.int32), _dev(y, "y", torch.float32),
        ws.ptr, ws.nbytes, ctypes.byref(group), _stream(stream))
    check(st, "asf_predict_sparse_ffn_exchange")


def asf_reduce_exchange(part: torch.Tensor, group, y: torch.Tensor, ws: Workspace, stream=None) -> None:
    """y = sum over ranks (rank order) of each rank's sum of its partials.

    part: [G, B, d] fp32, this rank's partials, with y [B, d]; or
    [R, G, B, d] with y [R, B, d]: one process holding all R ranks of the
    group (R = its world), run as one cooperative launch."""
    if part.dim() == 3:
        if y.shape != part.shape[1:]:
            raise ValueError("part [G, B, d] needs y [B, d]")
        local = 1
        G, B, d = part.shape
        prs, yrs = 0, 0
    elif part.dim() == 4:
        local, G, B, d = part.shape
        if y.shape != (local, B, d):
            raise ValueError("part [R, G, B, d] needs y [R, B, d]")
        prs, yrs = G * B * d, B * d
    else:
        raise ValueError("part must be [G, B, d] or [R, G, B, d]")
    st = L.load().asf_reduce_exchange(_dev(part, "part", torch.float32), prs, int(G), int(B), int(d),
                                      ctypes.byref(group), int(local), _dev(y, "y", torch.float32), yrs,
                                      ws.ptr, ws.nbytes, _stream(stream))
    check(st, "asf_reduce_exchange")


def asf_set_fault_injection(mode: int) -> None:
    """Test hook for the bounded device waits (see include/asffn.h)."""
    check(L.load().asf_set_fault_injection(int(mode)), "asf_set_fault_injection")


def asf_sparse_ffn_noalloc(ffn: FFN, x: torch.Tensor, idx: torch.Tensor, count: torch.Tensor,
                           y: torch.Tensor, fault: Optional[torch.Tensor] = None, stream=None) -> None:
    """asf_sparse_ffn without a workspace: for callers that cannot allocate
    device memory where they run the FFN (the library's own static device
    scratch is used instead; calls that overlap on the GPU race)."""
    if x.dtype != ffn.dtype or x.dim() != 2 or x.shape[1] != ffn.d:
        raise ValueError("x must be [B, d] in the FFN's dtype")
    if y.shape != (x.shape[0], ffn.d):
        raise ValueError("y must be [B, d]")
    fp = _dev(fault, "fault", torch.int32) if fault is not None else ctypes.c_void_p(0)
    st = L.load().asf_sparse_ffn_noalloc(ctypes.byref(ffn.desc), _dev(x, "x"), int(x.shape[0]),
                                         _dev(idx, "idx", torch.int32), _dev(count, "count", torch.int32),
                                         _dev(y, "y", torch.float32), fp, _stream(stream))
    check(st, "asf_sparse_ffn_noalloc")


def asf_dense_ffn(ffn: FFN, x: torch.Tensor, y: torch.Tensor, ws: Workspace, stream=None) -> None:
    if x.dtype != ffn.dtype or x.dim() != 2 or x.shape[1] != ffn.d or y.shape != (x.shape[0], ffn.d):
        raise ValueError("x must be [B, d] in the FFN's dtype and y [B, d]")
    st = L.load().asf_dense_ffn(ctypes.byref(ffn.desc), _dev(x, "x"), int(x.shape[0]),
                                _dev(y, "y", torch.float32), ws.ptr, ws.nbytes, _stream(stream))
    check(st, "asf_dense_ffn")


def asf_activation_counts(ffn: FFN, x: torch.Tensor, counts: torch.Tensor, ws: Workspace,
                          stream=None) -> None:
    """counts[k] += #tokens of x whose ReLU input for neuron k is > 0."""
    if x.dtype != ffn.dtype or x.dim() != 2 or x.shape[1] != ffn.d or counts.shape != (ffn.n,):
        raise ValueError("x must be [T, d] in the FFN's dtype and counts [n]")
    st = L.load().asf_activation_counts(ctypes.byref(ffn.desc), _dev(x, "x"), int(x.shape[0]),
                                        _dev(counts, "counts", torch.int64), ws.ptr, ws.nbytes,
                                        _stream(stream))
    check(st, "asf_activation_counts")


def asf_hot_permutation(counts) -> np.ndarray:
    """Host: neuron ids by descending count, ties to the lower id."""
    c = np.ascontiguousarray(np.asarray(counts, dtype=np.int64))
    out = np.empty(c.shape[0], dtype=np.int32)
    st = L.load().asf_hot_permutation(c.ctypes.data_as(ctypes.POINTER(ctypes.c_int64)), int(c.shape[0]),
                                      out.ctypes.data_as(ctypes.POINTER(ctypes.c_int32)))
    check(st, "asf_hot_permutation")
    return out


def asf_permute_rows(src: torch.Tensor, dst: torch.Tensor, perm: torch.Tensor, stream=None) -> None:
    """dst[i] = src[perm[i]] (row gather on the device)."""
    if src.shape != dst.shape or src.dtype != dst.dtype or src.shape[0] != perm.shape[0]:
        raise ValueError("src/dst must match and have one row per perm entry")
    n_rows = int(src.shape[0])
    row_bytes = src.numel() * src.element_size() // max(1, n_rows)
    st = L.load().asf_permute_rows(_dev(src, "src"), _dev(dst, "dst"), n_rows, row_bytes,
                                   _dev(perm, "perm", torch.int32), _stream(stream))
    check(st, "asf_permute_rows")


def asf_gather_rows(src: torch.Tensor, dst: torch.Tensor, perm: Optional[torch.Tensor] = None, *,
                    dst_offset: int = 0, dst_stride: Optional[int] = None, stream=None) -> None:
    """Row gather on the device: row i of dst (dst_stride bytes apart, starting
    dst_offset bytes into dst) = row perm[i] of src (identity without perm)."""
    if src.dim() < 1 or src.shape[0] == 0:
        raise ValueError("src needs at least one row")
    src_rows = int(src.shape[0])
    row_bytes = src.numel() * src.element_size() // src_rows
    n_rows = int(perm.shape[0]) if perm is not None else src_rows
    stride = int(dst_stride) if dst_stride is not None else row_bytes
    need = dst_offset + (n_rows - 1) * stride + row_bytes if n_rows else 0
    if dst_offset < 0 or stride < row_bytes or need > dst.numel() * dst.element_size():
        raise ValueError("destination rows do not fit in dst")
    pp = _dev(perm, "perm", torch.int32) if perm is not None else ctypes.c_void_p(0)
    st = L.load().asf_gather_rows(_dev(src, "src"), row_bytes, src_rows,
                                  ctypes.c_void_p(_dev(dst, "dst").value + dst_offset), stride, n_rows,
                                  row_bytes, pp, _stream(stream))
    check(st, "asf_gather_rows")


def pack_layer(act: str, Wg: Optional[torch.Tensor], Wu: torch.Tensor, WdT: torch.Tensor,
               perm: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """Neuron-major packed copy [k, m, d] of a layer's rows: row i is neuron
    perm[i] (k = len(perm): a permutation, or a subset such as one rank's
    neurons), or neuron i without perm (k = n)."""
    n, d = Wu.shape
    mats = [Wg, Wu, WdT] if act == "reglu" else [Wu, WdT]
    k = int(perm.shape[0]) if perm is not None else n
    out = torch.empty(k, len(mats), d, dtype=Wu.dtype, device=Wu.device)
    rb = d * Wu.element_size()
    for m, W in enumerate(mats):
        asf_gather_rows(W, out, perm, dst_offset=m * rb, dst_stride=len(mats) * rb, stream=stream)
    return out


def asf_read_error(ws: Workspace, stream=None) -> int:
    """Synchronise the stream, return and clear the device error status (0 = none)."""
    out = ctypes.c_int32(0)
    check(L.load().asf_read_error(ws.ptr, ctypes.byref(out), _stream(stream)), "asf_read_error")
    return int(out.value)


def asf_status_string(status: int) -> str:
    return L.load().asf_status_string(int(status)).decode()

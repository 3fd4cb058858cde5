"""Thin Python binding of the C ABI (include/tq.h): argument marshalling only.

Every function has the name of the C entry point it calls and forwards
device pointers of torch tensors (``data_ptr()``) and the current CUDA
stream.  No arithmetic of the method happens here.
"""
from __future__ import annotations

import ctypes

import numpy as np
import torch

from . import _lib
from ._lib import (TQ_BF16, TQ_F16, TQ_F32, TQ_MAX_TOPK, TQ_POLAR, TQ_MSE, TQ_PROD, TQ_STATUS_LAYOUT, TQ_STATUS_TIMEOUT, TQError,
                   check, lib)

__all__ = [
    "TQ_MSE", "TQ_PROD", "TQ_F32", "TQ_BF16", "TQ_F16", "TQ_MAX_TOPK", "TQ_STATUS_TIMEOUT", "TQ_STATUS_LAYOUT", "TQError", "Handle", "code_words", "sign_words",
    "tq_make_codebook", "tq_make_rotation", "tq_create", "tq_quant_mse", "tq_dequant_mse", "tq_quant_prod",
    "tq_quant_prod_workspace",
    "tq_ip_scores", "tq_ip_scores_workspace", "tq_attn_decode", "tq_attn_decode_workspace", "tq_version",
    "tq_attn_decode_static", "tq_quant_gather", "tq_attn_logits", "tq_attn_logits_workspace", "tq_device_status",
    "tq_attn_decode_partial", "tq_attn_decode_partial_workspace", "tq_attn_merge", "tq_topk_merge",
    "tq_quant_paged", "tq_attn_decode_paged", "tq_quant_gather_groups", "tq_attn_prefill",
    "tq_attn_prefill_workspace", "TQ_POLAR", "tq_polar_codebook", "tq_create_polar", "tq_quant_polar",
    "tq_dequant_polar",
]


def code_words(b: int, d: int) -> int:
    return ((d + 31) // 32) * b


def sign_words(d: int) -> int:
    return (d + 31) // 32


def _dptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def _ptr(t) -> int | None:
    if t is None:
        return None
    if not isinstance(t, torch.Tensor):
        raise TypeError("expected a torch.Tensor")
    if not t.is_cuda:
        raise ValueError("expected a CUDA tensor (this library has no CPU path)")
    if not t.is_contiguous():
        raise ValueError("expected a contiguous tensor")
    return t.data_ptr()


def _stream(stream) -> int | None:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.float32:
        return TQ_F32
    if t.dtype == torch.bfloat16:
        return TQ_BF16
    raise ValueError(f"unsupported dtype {t.dtype}")


def tq_version() -> str:
    return lib.tq_version().decode()


def tq_make_codebook(b: int, d: int) -> tuple[np.ndarray, np.ndarray]:
    c = np.zeros(2 ** b)
    t = np.zeros(2 ** b - 1)
    check("tq_make_codebook", lib.tq_make_codebook(b, d, _dptr(c), _dptr(t)))
    return c, t


def tq_make_rotation(G: np.ndarray) -> np.ndarray:
    G = np.ascontiguousarray(G, dtype=np.float64)
    d = G.shape[0]
    Pi = np.zeros((d, d))
    check("tq_make_rotation", lib.tq_make_rotation(d, _dptr(G), _dptr(Pi)))
    return Pi


class Handle:
    """Owns a tq_handle (device constants); destroyed with the object."""

    def __init__(self, ptr: int, d: int, b: int, variant: int, bh: int = 0):
        self.ptr = ptr
        self.d, self.b, self.variant, self.bh = d, b, variant, bh
        self.bm = b if variant in (TQ_MSE, TQ_POLAR) else b - 1

    @property
    def words(self) -> int:
        if self.variant == TQ_POLAR:
            return code_words(self.b, self.d // 2) + code_words(self.bh, self.d // 2 - 1)
        return code_words(self.bm, self.d)

    def close(self):
        if self.ptr:
            check("tq_destroy", lib.tq_destroy(self.ptr))
            self.ptr = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def tq_create(d: int, b: int, variant: int, Pi: np.ndarray, S: np.ndarray | None = None,
              centroids: np.ndarray | None = None) -> Handle:
    Pi = np.ascontiguousarray(Pi, dtype=np.float64)
    Sa = None if S is None else np.ascontiguousarray(S, dtype=np.float64)
    ca = None if centroids is None else np.ascontiguousarray(centroids, dtype=np.float64)
    h = ctypes.c_void_p()
    check("tq_create", lib.tq_create(ctypes.byref(h), d, b, variant, _dptr(Pi),
                                     None if Sa is None else _dptr(Sa), None if ca is None else _dptr(ca)))
    return Handle(h.value, d, b, variant)


def tq_polar_codebook(b: int, level: int) -> tuple[np.ndarray, np.ndarray]:
    c = np.zeros(2 ** b)
    t = np.zeros(2 ** b - 1)
    check("tq_polar_codebook", lib.tq_polar_codebook(b, level, _dptr(c), _dptr(t)))
    return c, t


def tq_create_polar(d: int, b1: int, bh: int, Pi: np.ndarray) -> Handle:
    """A PolarQuant instance: b1 bits for level-1 angles, bh for the others."""
    Pi = np.ascontiguousarray(Pi, dtype=np.float64)
    h = ctypes.c_void_p()
    check("tq_create_polar", lib.tq_create_polar(ctypes.byref(h), d, b1, bh, _dptr(Pi)))
    return Handle(h.value, d, b1, TQ_POLAR, bh)


def tq_quant_polar(h: Handle, x: torch.Tensor, codes: torch.Tensor, norms: torch.Tensor, out_stride: int = 1,
                   stream=None) -> None:
    check("tq_quant_polar", lib.tq_quant_polar(h.ptr, _ptr(x), _dtype_code(x), x.shape[0], x.shape[1], _ptr(codes),
                                               _ptr(norms), out_stride, _stream(stream)))


def tq_dequant_polar(h: Handle, codes: torch.Tensor, norms: torch.Tensor, out: torch.Tensor, stream=None) -> None:
    check("tq_dequant_polar", lib.tq_dequant_polar(h.ptr, _ptr(codes), _ptr(norms), codes.shape[0], _ptr(out),
                                                   _dtype_code(out), _stream(stream)))


def tq_quant_mse(h: Handle, x: torch.Tensor, codes: torch.Tensor, norms: torch.Tensor,
                 out_stride: int = 1, stream=None) -> None:
    N = x.shape[0]
    check("tq_quant_mse", lib.tq_quant_mse(h.ptr, _ptr(x), _dtype_code(x), N, x.shape[1], _ptr(codes),
                                           _ptr(norms), out_stride, _stream(stream)))


def tq_dequant_mse(h: Handle, codes: torch.Tensor, norms: torch.Tensor, out: torch.Tensor,
                   stream=None) -> None:
    check("tq_dequant_mse", lib.tq_dequant_mse(h.ptr, _ptr(codes), _ptr(norms), codes.shape[0], _ptr(out),
                                               _dtype_code(out), _stream(stream)))


def tq_quant_prod_workspace(h: Handle, N: int) -> int:
    return int(lib.tq_quant_prod_workspace(h.ptr, N))


def tq_quant_prod(h: Handle, x: torch.Tensor, codes: torch.Tensor, signs: torch.Tensor,
                  norms: torch.Tensor, rnorms: torch.Tensor, out_stride: int = 1, workspace=None,
                  stream=None) -> None:
    """TurboQuant_prod quantization (tq_quant_prod_ws; the workspace, needed only
    above d = 256, is allocated here when none is passed)."""
    N = x.shape[0]
    if workspace is None:
        nbytes = tq_quant_prod_workspace(h, N)
        if nbytes:
            workspace = torch.empty(nbytes, dtype=torch.uint8, device=x.device)
    check("tq_quant_prod_ws", lib.tq_quant_prod_ws(h.ptr, _ptr(x), _dtype_code(x), N, x.shape[1], _ptr(codes),
                                                   _ptr(signs), _ptr(norms), _ptr(rnorms), out_stride,
                                                   _ptr(workspace), 0 if workspace is None else workspace.numel(),
                                                   _stream(stream)))


def tq_ip_scores_workspace(h: Handle, nq: int, N: int, topk: int = 0) -> int:
    return int(lib.tq_ip_scores_workspace(h.ptr, nq, N, topk))


def tq_ip_scores(h: Handle, q: torch.Tensor, codes: torch.Tensor, signs, norms: torch.Tensor, rnorms,
                 scores=None, topk: int = 0, top_idx=None, top_val=None, workspace=None,
                 stream=None) -> None:
    nq, N = q.shape[0], codes.shape[0]
    if workspace is None:
        workspace = torch.empty(max(1, tq_ip_scores_workspace(h, nq, N, topk)), dtype=torch.uint8,
                                device=q.device)
    check("tq_ip_scores", lib.tq_ip_scores(h.ptr, _ptr(q), nq, _ptr(codes), _ptr(signs), _ptr(norms),
                                           _ptr(rnorms), N, _ptr(scores), topk, _ptr(top_idx),
                                           _ptr(top_val), _ptr(workspace), workspace.numel(),
                                           _stream(stream)))


def tq_attn_decode_workspace(hk: Handle, B: int, Hq: int, Hkv: int, T: int) -> int:
    return int(lib.tq_attn_decode_workspace(hk.ptr, B, Hq, Hkv, T))


def tq_attn_decode(hk: Handle, hv: Handle, q: torch.Tensor, Hkv: int, T: int, kv_stride: int,
                   kcodes, ksigns, knorms, krnorms, vcodes, vnorms, scale: float, out: torch.Tensor,
                   workspace=None, stream=None) -> None:
    B, Hq, _ = q.shape
    if workspace is None:
        workspace = torch.empty(max(1, tq_attn_decode_workspace(hk, B, Hq, Hkv, T)), dtype=torch.uint8,
                                device=q.device)
    check("tq_attn_decode", lib.tq_attn_decode(hk.ptr, hv.ptr, _ptr(q), _dtype_code(q), B, Hq, Hkv, T,
                                               kv_stride, _ptr(kcodes), _ptr(ksigns), _ptr(knorms),
                                               _ptr(krnorms), _ptr(vcodes), _ptr(vnorms), float(scale),
                                               _ptr(out), _ptr(workspace), workspace.numel(),
                                               _stream(stream)))


def tq_attn_decode_static(hk: Handle, hv: Handle, q: torch.Tensor, Hkv: int, T: int, kv_stride: int,
                          kcodes, ksigns, knorms, krnorms, vcodes, vnorms, scale: float, out: torch.Tensor,
                          stream=None) -> None:
    """tq_attn_decode without a workspace, for callers that may not allocate
    device memory: the scratch lives in a fixed array inside the library (see
    include/tq.h for its limit and for the rule that overlapping calls race)."""
    B, Hq, _ = q.shape
    check("tq_attn_decode_static", lib.tq_attn_decode_static(
        hk.ptr, hv.ptr, _ptr(q), _dtype_code(q), B, Hq, Hkv, T, kv_stride, _ptr(kcodes), _ptr(ksigns),
        _ptr(knorms), _ptr(krnorms), _ptr(vcodes), _ptr(vnorms), float(scale), _ptr(out), _stream(stream)))


def tq_attn_decode_partial_workspace(hk: Handle, B: int, Hq: int, Hkv: int, T: int) -> int:
    return int(lib.tq_attn_decode_partial_workspace(hk.ptr, B, Hq, Hkv, T))


def tq_attn_decode_partial(hk: Handle, hv: Handle, q: torch.Tensor, Hkv: int, T: int, kv_stride: int,
                           kcodes, ksigns, knorms, krnorms, vcodes, vnorms, scale: float, partial: torch.Tensor,
                           workspace=None, stream=None) -> None:
    """Softmax state [B*Hq][d + 2] (acc in the rotated value frame, m, l) of the
    decode step over the context slice held here (T may be 0)."""
    B, Hq, _ = q.shape
    if workspace is None:
        workspace = torch.empty(max(1, tq_attn_decode_partial_workspace(hk, B, Hq, Hkv, T)), dtype=torch.uint8,
                                device=q.device)
    check("tq_attn_decode_partial", lib.tq_attn_decode_partial(
        hk.ptr, hv.ptr, _ptr(q), _dtype_code(q), B, Hq, Hkv, T, kv_stride, _ptr(kcodes), _ptr(ksigns),
        _ptr(knorms), _ptr(krnorms), _ptr(vcodes), _ptr(vnorms), float(scale), _ptr(partial), _ptr(workspace),
        workspace.numel(), _stream(stream)))


def tq_attn_merge(hv: Handle, partials: torch.Tensor, out: torch.Tensor, stream=None) -> None:
    """Combine [R][rows][d + 2] slice records into out [rows][d]."""
    R, rows = partials.shape[0], partials.shape[1]
    check("tq_attn_merge", lib.tq_attn_merge(hv.ptr, _ptr(partials), R, rows, _ptr(out), _stream(stream)))


def tq_topk_merge(val: torch.Tensor, idx: torch.Tensor, offsets, out_idx: torch.Tensor, out_val: torch.Tensor,
                  stream=None) -> None:
    """Global top-k from [R][nq][k] per-slice lists; offsets[r] = first global index of slice r."""
    R, nq, k = val.shape
    offs = (ctypes.c_int64 * R)(*[int(o) for o in offsets])
    check("tq_topk_merge", lib.tq_topk_merge(_ptr(val), _ptr(idx), R, nq, k, offs, _ptr(out_idx), _ptr(out_val),
                                             _stream(stream)))


def _rn_code(t) -> int:
    return TQ_F16 if t.dtype == torch.float16 else TQ_F32


def tq_quant_paged(h: Handle, x: torch.Tensor, slots: torch.Tensor, codes: torch.Tensor, norms: torch.Tensor,
                   signs=None, rnorms=None, channels=None, stream=None) -> None:
    """Quantize the rows of x into cache rows slots[i] (int64); rnorms may be
    float32 or float16 storage."""
    rn_dtype = _rn_code(rnorms) if rnorms is not None else TQ_F32
    check("tq_quant_paged", lib.tq_quant_paged(h.ptr, _ptr(x), _dtype_code(x), x.shape[0], x.shape[1], _ptr(channels),
                                               _ptr(slots), _ptr(codes), _ptr(signs), _ptr(norms), _ptr(rnorms),
                                               rn_dtype, _stream(stream)))


def tq_attn_decode_paged(hk: Handle, hv: Handle, q: torch.Tensor, Hkv: int, T: int, block_table: torch.Tensor,
                         page_size: int, kcodes, ksigns, knorms, krnorms, vcodes, vnorms, scale: float,
                         out: torch.Tensor, workspace=None, stream=None) -> None:
    """Decode over a paged cache; block_table is [B*Hkv][max_pages] int32."""
    B, Hq, _ = q.shape
    if workspace is None:
        workspace = torch.empty(max(1, tq_attn_decode_workspace(hk, B, Hq, Hkv, T)), dtype=torch.uint8,
                                device=q.device)
    check("tq_attn_decode_paged", lib.tq_attn_decode_paged(
        hk.ptr, hv.ptr, _ptr(q), _dtype_code(q), B, Hq, Hkv, T, _ptr(block_table), block_table.shape[1], page_size,
        _ptr(kcodes), _ptr(ksigns), _ptr(knorms), _ptr(krnorms), _rn_code(krnorms), _ptr(vcodes), _ptr(vnorms),
        float(scale), _ptr(out), _ptr(workspace), workspace.numel(), _stream(stream)))


def tq_attn_prefill_workspace(hk: Handle, B: int, nq: int, Hq: int, Hkv: int, T: int) -> int:
    return int(lib.tq_attn_prefill_workspace(hk.ptr, B, nq, Hq, Hkv, T))


def tq_attn_prefill(hk: Handle, hv: Handle, q: torch.Tensor, Hkv: int, T: int, kv_stride: int, kcodes, ksigns,
                    knorms, krnorms, vcodes, vnorms, scale: float, out: torch.Tensor, workspace=None,
                    stream=None) -> None:
    """Causal attention of a block of nq new tokens, q [B][nq][Hq][d], over a
    cache of T tokens that ends with them; out [B][nq][Hq][d] float32."""
    B, nq, Hq, _ = q.shape
    if workspace is None:
        workspace = torch.empty(max(1, tq_attn_prefill_workspace(hk, B, nq, Hq, Hkv, T)), dtype=torch.uint8,
                                device=q.device)
    check("tq_attn_prefill", lib.tq_attn_prefill(
        hk.ptr, hv.ptr, _ptr(q), _dtype_code(q), B, nq, Hq, Hkv, T, kv_stride, _ptr(kcodes), _ptr(ksigns),
        _ptr(knorms), _ptr(krnorms), _ptr(vcodes), _ptr(vnorms), float(scale), _ptr(out), _ptr(workspace),
        workspace.numel(), _stream(stream)))


def tq_device_status(h: Handle) -> int:
    v = ctypes.c_int(0)
    check("tq_device_status", lib.tq_device_status(h.ptr, ctypes.byref(v)))
    return v.value


def tq_quant_gather(h: Handle, x: torch.Tensor, channels: torch.Tensor, codes: torch.Tensor, norms: torch.Tensor,
                    signs=None, rnorms=None, out_stride: int = 1, stream=None) -> None:
    """Quantize x[:, channels] (one channel group of a split cache)."""
    check("tq_quant_gather", lib.tq_quant_gather(h.ptr, _ptr(x), _dtype_code(x), x.shape[0], x.shape[1],
                                                 _ptr(channels), _ptr(codes), _ptr(signs), _ptr(norms),
                                                 _ptr(rnorms), out_stride, _stream(stream)))


def tq_quant_gather_groups(handles, x: torch.Tensor, channels: torch.Tensor, codes, norms, signs=None, rnorms=None,
                           out_stride: int = 1, stream=None) -> None:
    """Every channel group of the rows of x in one launch; codes / norms /
    signs / rnorms are lists with one tensor (or None) per group."""
    n = len(handles)
    hs = (ctypes.c_void_p * n)(*[h.ptr for h in handles])
    signs = signs or [None] * n
    rnorms = rnorms or [None] * n
    check("tq_quant_gather_groups", lib.tq_quant_gather_groups(
        hs, n, _ptr(x), _dtype_code(x), x.shape[0], x.shape[1], _ptr(channels), _ptr_array(codes),
        _ptr_array(signs), _ptr_array(norms), _ptr_array(rnorms), out_stride, _stream(stream)))


def _ptr_array(items):
    arr = (ctypes.c_void_p * len(items))()
    for i, t in enumerate(items):
        arr[i] = _ptr(t)
    return arr


def tq_attn_logits_workspace(handles, B: int, Hq: int) -> int:
    hs = (ctypes.c_void_p * len(handles))(*[h.ptr for h in handles])
    return int(lib.tq_attn_logits_workspace(hs, len(handles), B, Hq))


def tq_attn_logits(handles, channels, q: torch.Tensor, Hkv: int, T: int, kv_stride: int, kcodes, ksigns, knorms,
                   krnorms, scale: float, logits: torch.Tensor, workspace=None, stream=None) -> None:
    """Logits [B][Hq][T] over a key cache of one or two channel groups (lists
    of per-group tensors); q is [B][Hq][dq]."""
    B, Hq, dq = q.shape
    hs = (ctypes.c_void_p * len(handles))(*[h.ptr for h in handles])
    if workspace is None:
        workspace = torch.empty(max(1, tq_attn_logits_workspace(handles, B, Hq)), dtype=torch.uint8,
                                device=q.device)
    check("tq_attn_logits", lib.tq_attn_logits(hs, len(handles), _ptr(channels), _ptr(q), _dtype_code(q), dq, B, Hq,
                                               Hkv, T, kv_stride, _ptr_array(kcodes), _ptr_array(ksigns),
                                               _ptr_array(knorms), _ptr_array(krnorms), float(scale), _ptr(logits),
                                               _ptr(workspace), workspace.numel(), _stream(stream)))

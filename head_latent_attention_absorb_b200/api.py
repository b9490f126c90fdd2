"""Python binding of libmla_b200.so with the C names.  Argument marshalling only: torch owns
the device memory and the stream; every step of the computation runs in the library's kernels.

All tensors are CUDA tensors.  Strides are read from the tensors, so a packed
[B, n_max, d_c + d_r] cache can be passed as two views (``cache[..., :d_c]``, ``cache[..., d_c:]``).
"""

from __future__ import annotations

import ctypes
from typing import Optional, Sequence

import torch

from . import _capi
from ._capi import MLADims, check, lib

_DT = {torch.bfloat16: _capi.MLA_BF16, torch.float32: _capi.MLA_F32}


def dims_of(n_h: int, d_c: int, d_r: int, d_h: int, d_v: int) -> MLADims:
    return MLADims(n_h, d_c, d_r, d_h, d_v)


def _dtc(dtype: torch.dtype) -> int:
    if dtype not in _DT:
        raise TypeError(f"unsupported dtype {dtype}")
    return _DT[dtype]


def _dt(t: torch.Tensor) -> int:
    return _dtc(t.dtype)


def _ptr(t: Optional[torch.Tensor]) -> Optional[int]:
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("expected a CUDA tensor")
    return t.data_ptr()


def _stream(stream) -> Optional[int]:
    s = stream if stream is not None else torch.cuda.current_stream()
    return s.cuda_stream if hasattr(s, "cuda_stream") else s


def _rows(t: torch.Tensor, name: str):
    if t.stride(-1) != 1:
        raise ValueError(f"{name}: last axis must be contiguous")


def _headrows(t: torch.Tensor, name: str) -> int:
    """Row stride of a [B, n_h, width] tensor whose (b, h) rows are evenly strided."""
    _rows(t, name)
    if t.dim() != 3 or t.stride(0) != t.shape[1] * t.stride(1):
        raise ValueError(f"{name}: expected [B, n_h, width] with row (b, h) at (b*n_h + h)*stride")
    return t.stride(1)


def _dims(x: Sequence[int]) -> MLADims:
    return x if isinstance(x, MLADims) else MLADims(*x)


def mla_absorb_q(dims, q_nope: torch.Tensor, w_kv_b: torch.Tensor, q_tilde: Optional[torch.Tensor] = None,
                 stream=None) -> torch.Tensor:
    """q~[b,h,:] = (W^UK_h)^T q_nope[b,h,:].  q_nope [B, n_h, d_h] (rows may be strided)."""
    d = _dims(dims)
    B = q_nope.shape[0]
    ldq = _headrows(q_nope, "q_nope")
    if q_tilde is None:
        q_tilde = torch.empty((B, d.n_h, d.d_c), dtype=q_nope.dtype, device=q_nope.device)
    check(lib().mla_absorb_q(d, _dt(q_nope), B, _ptr(q_nope), ldq, _ptr(w_kv_b), _ptr(q_tilde),
                             _stream(stream)), "mla_absorb_q")
    return q_tilde


def mla_decode_workspace_size(dims, dtype: torch.dtype, B: int, n_max: int, topk: int = 0) -> int:
    return int(lib().mla_decode_workspace_size(_dims(dims), _dtc(dtype), B, n_max, topk))


def mla_decode_num_launches(dims, dtype: torch.dtype, B: int, n_max: int, topk: int = 0) -> int:
    return int(lib().mla_decode_num_launches(_dims(dims), _dtc(dtype), B, n_max, topk))


def mla_decode_absorb(dims, q_tilde: torch.Tensor, q_pe: torch.Tensor, c_kv: torch.Tensor, k_r: torch.Tensor,
                      lengths: torch.Tensor, scale: float, topk_idx: Optional[torch.Tensor] = None,
                      ctx: Optional[torch.Tensor] = None, lse: Optional[torch.Tensor] = None,
                      workspace: Optional[torch.Tensor] = None, dev_err: Optional[torch.Tensor] = None,
                      stream=None) -> torch.Tensor:
    """Latent-space attention of one query token per sequence.  c_kv [B, n_max, d_c] and
    k_r [B, n_max, d_r] may be strided views; lengths int32 [B]; topk_idx int32 [B, k] or None."""
    d = _dims(dims)
    B, n_max = c_kv.shape[0], c_kv.shape[1]
    ldqt, ldqp = _headrows(q_tilde, "q_tilde"), _headrows(q_pe, "q_pe")
    _rows(c_kv, "c_kv")
    _rows(k_r, "k_r")
    if lengths.dtype != torch.int32 or (topk_idx is not None and topk_idx.dtype != torch.int32):
        raise TypeError("lengths and topk_idx must be int32")
    if topk_idx is not None and not topk_idx.is_contiguous():
        raise ValueError("topk_idx must be contiguous")
    topk = 0 if topk_idx is None else topk_idx.shape[1]
    if ctx is None:
        ctx = torch.empty((B, d.n_h, d.d_c), dtype=q_tilde.dtype, device=q_tilde.device)
    if workspace is None:
        nbytes = mla_decode_workspace_size(d, q_tilde.dtype, B, n_max, topk)
        workspace = torch.empty((max(nbytes, 16),), dtype=torch.uint8, device=q_tilde.device)
    check(lib().mla_decode_absorb(
        d, _dt(q_tilde), B,
        _ptr(q_tilde), ldqt, _ptr(q_pe), ldqp,
        _ptr(c_kv), c_kv.stride(0), c_kv.stride(1), _ptr(k_r), k_r.stride(0), k_r.stride(1),
        n_max, _ptr(lengths), _ptr(topk_idx), topk, float(scale),
        _ptr(ctx), _ptr(lse), _ptr(workspace), workspace.numel() * workspace.element_size(),
        _ptr(dev_err), _stream(stream)), "mla_decode_absorb")
    return ctx


def mla_decode_absorb_fp8kv(dims, q_tilde: torch.Tensor, q_pe: torch.Tensor, c8: torch.Tensor,
                            kv_scale: torch.Tensor, k_r: torch.Tensor, lengths: torch.Tensor, scale: float,
                            ctx: Optional[torch.Tensor] = None, lse: Optional[torch.Tensor] = None,
                            workspace: Optional[torch.Tensor] = None, dev_err: Optional[torch.Tensor] = None,
                            stream=None) -> torch.Tensor:
    """The absorbed decode over an FP8 latent cache: c8 [B, n_max, d_c] uint8 E4M3 codes, kv_scale
    [B, n_max, d_c / 128] float32 (one scale per 128 latent features of a row), k_r [B, n_max, d_r]
    bf16; all three may be strided views (e.g. of one packed 656-byte row)."""
    d = _dims(dims)
    B, n_max = c8.shape[0], c8.shape[1]
    ldqt, ldqp = _headrows(q_tilde, "q_tilde"), _headrows(q_pe, "q_pe")
    for t, n in ((c8, "c8"), (kv_scale, "kv_scale"), (k_r, "k_r")):
        _rows(t, n)
    if c8.dtype != torch.uint8 or kv_scale.dtype != torch.float32:
        raise TypeError("c8 must be uint8 and kv_scale float32")
    if lengths.dtype != torch.int32:
        raise TypeError("lengths must be int32")
    if ctx is None:
        ctx = torch.empty((B, d.n_h, d.d_c), dtype=q_tilde.dtype, device=q_tilde.device)
    if workspace is None:
        nbytes = mla_decode_workspace_size(d, q_tilde.dtype, B, n_max, 0)
        workspace = torch.empty((max(nbytes, 16),), dtype=torch.uint8, device=q_tilde.device)
    check(lib().mla_decode_absorb_fp8kv(
        d, B, _ptr(q_tilde), ldqt, _ptr(q_pe), ldqp,
        _ptr(c8), c8.stride(0), c8.stride(1), _ptr(kv_scale), kv_scale.stride(0), kv_scale.stride(1),
        _ptr(k_r), k_r.stride(0), k_r.stride(1), n_max, _ptr(lengths), float(scale),
        _ptr(ctx), _ptr(lse), _ptr(workspace), workspace.numel() * workspace.element_size(),
        _ptr(dev_err), _stream(stream)), "mla_decode_absorb_fp8kv")
    return ctx


def mla_decode_absorb_multi(dims, q_tilde: torch.Tensor, q_pe: torch.Tensor, c_kv: torch.Tensor,
                            k_r: torch.Tensor, lengths: torch.Tensor, scale: float,
                            ctx: Optional[torch.Tensor] = None, lse: Optional[torch.Tensor] = None,
                            workspace: Optional[torch.Tensor] = None, dev_err: Optional[torch.Tensor] = None,
                            stream=None) -> torch.Tensor:
    """T new tokens per sequence: q_tilde [B, T, n_h, d_c] and q_pe [B, T, n_h, d_r] (the last T cached
    rows of each sequence are those tokens); returns ctx [B, T, n_h, d_c].  c_kv / k_r / lengths as in
    mla_decode_absorb."""
    d = _dims(dims)
    B, T = q_tilde.shape[0], q_tilde.shape[1]
    n_max = c_kv.shape[1]
    qt = q_tilde.reshape(B * T, d.n_h, -1)
    qp = q_pe.reshape(B * T, d.n_h, -1)
    ldqt, ldqp = _headrows(qt, "q_tilde"), _headrows(qp, "q_pe")
    _rows(c_kv, "c_kv")
    _rows(k_r, "k_r")
    if lengths.dtype != torch.int32:
        raise TypeError("lengths must be int32")
    if ctx is None:
        ctx = torch.empty((B, T, d.n_h, d.d_c), dtype=q_tilde.dtype, device=q_tilde.device)
    if workspace is None:
        nbytes = mla_decode_workspace_size(d, q_tilde.dtype, B * T, n_max, 0)
        workspace = torch.empty((max(nbytes, 16),), dtype=torch.uint8, device=q_tilde.device)
    check(lib().mla_decode_absorb_multi(
        d, _dt(q_tilde), B, T, _ptr(qt), ldqt, _ptr(qp), ldqp,
        _ptr(c_kv), c_kv.stride(0), c_kv.stride(1), _ptr(k_r), k_r.stride(0), k_r.stride(1),
        n_max, _ptr(lengths), float(scale), _ptr(ctx), _ptr(lse), _ptr(workspace),
        workspace.numel() * workspace.element_size(), _ptr(dev_err), _stream(stream)), "mla_decode_absorb_multi")
    return ctx


def mla_decode_absorb_multi_topk(dims, q_tilde: torch.Tensor, q_pe: torch.Tensor, c_kv: torch.Tensor,
                                 k_r: torch.Tensor, lengths: torch.Tensor, topk_idx: torch.Tensor, scale: float,
                                 ctx: Optional[torch.Tensor] = None, lse: Optional[torch.Tensor] = None,
                                 workspace: Optional[torch.Tensor] = None, dev_err: Optional[torch.Tensor] = None,
                                 stream=None) -> torch.Tensor:
    """mla_decode_absorb_multi with a top-k set per new token: topk_idx int32 [B, T, k] (token s of
    sequence b attends its set's rows t <= lengths[b] - T + s); returns ctx [B, T, n_h, d_c]."""
    d = _dims(dims)
    B, T = q_tilde.shape[0], q_tilde.shape[1]
    n_max = c_kv.shape[1]
    qt = q_tilde.reshape(B * T, d.n_h, -1)
    qp = q_pe.reshape(B * T, d.n_h, -1)
    ldqt, ldqp = _headrows(qt, "q_tilde"), _headrows(qp, "q_pe")
    _rows(c_kv, "c_kv")
    _rows(k_r, "k_r")
    if lengths.dtype != torch.int32:
        raise TypeError("lengths must be int32")
    if topk_idx.dtype != torch.int32 or not topk_idx.is_contiguous() or tuple(topk_idx.shape[:2]) != (B, T):
        raise TypeError("topk_idx must be a contiguous int32 [B, T, k] tensor")
    k = topk_idx.shape[2]
    if ctx is None:
        ctx = torch.empty((B, T, d.n_h, d.d_c), dtype=q_tilde.dtype, device=q_tilde.device)
    if workspace is None:
        nbytes = mla_decode_workspace_size(d, q_tilde.dtype, B * T, n_max, k)
        workspace = torch.empty((max(nbytes, 16),), dtype=torch.uint8, device=q_tilde.device)
    check(lib().mla_decode_absorb_multi_topk(
        d, _dt(q_tilde), B, T, _ptr(qt), ldqt, _ptr(qp), ldqp,
        _ptr(c_kv), c_kv.stride(0), c_kv.stride(1), _ptr(k_r), k_r.stride(0), k_r.stride(1),
        n_max, _ptr(lengths), _ptr(topk_idx), k, float(scale), _ptr(ctx), _ptr(lse), _ptr(workspace),
        workspace.numel() * workspace.element_size(), _ptr(dev_err), _stream(stream)), "mla_decode_absorb_multi_topk")
    return ctx


def mla_decode_absorb_static(dims, q_tilde: torch.Tensor, q_pe: torch.Tensor, c_kv: torch.Tensor,
                             k_r: torch.Tensor, lengths: torch.Tensor, scale: float,
                             ctx: Optional[torch.Tensor] = None, lse: Optional[torch.Tensor] = None,
                             dev_err: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """bf16 dense decode with the library's built-in scratch (for callers that cannot allocate a
    workspace).  `ctx` (and `lse`) are allocated here only when not given."""
    d = _dims(dims)
    B, n_max = c_kv.shape[0], c_kv.shape[1]
    ldqt, ldqp = _headrows(q_tilde, "q_tilde"), _headrows(q_pe, "q_pe")
    _rows(c_kv, "c_kv")
    _rows(k_r, "k_r")
    if lengths.dtype != torch.int32:
        raise TypeError("lengths must be int32")
    if ctx is None:
        ctx = torch.empty((B, d.n_h, d.d_c), dtype=q_tilde.dtype, device=q_tilde.device)
    check(lib().mla_decode_absorb_static(
        d, _dt(q_tilde), B, _ptr(q_tilde), ldqt, _ptr(q_pe), ldqp,
        _ptr(c_kv), c_kv.stride(0), c_kv.stride(1), _ptr(k_r), k_r.stride(0), k_r.stride(1),
        n_max, _ptr(lengths), float(scale), _ptr(ctx), _ptr(lse), _ptr(dev_err), _stream(stream)),
        "mla_decode_absorb_static")
    return ctx


def mla_out_up(dims, ctx: torch.Tensor, w_kv_b: torch.Tensor, out: Optional[torch.Tensor] = None,
               stream=None) -> torch.Tensor:
    """o[b,h,:] = W^UV_h ctx[b,h,:].  ctx [B, n_h, d_c] contiguous."""
    d = _dims(dims)
    B = ctx.shape[0]
    if not ctx.is_contiguous():
        raise ValueError("ctx must be contiguous")
    if out is None:
        out = torch.empty((B, d.n_h, d.d_v), dtype=ctx.dtype, device=ctx.device)
    check(lib().mla_out_up(d, _dt(ctx), B, _ptr(ctx), _ptr(w_kv_b), _ptr(out), _stream(stream)), "mla_out_up")
    return out


def mla_absorb_q_fp8(dims, q_nope: torch.Tensor, w_fp8: torch.Tensor, w_scale: torch.Tensor,
                     q_tilde: Optional[torch.Tensor] = None, dev_err: Optional[torch.Tensor] = None,
                     stream=None) -> torch.Tensor:
    """mla_absorb_q with an e4m3 wkv_b (w_fp8, torch.float8_e4m3fn) and its fp32 128 x 128 block
    scales (w_scale [rows / 128, d_c / 128])."""
    d = _dims(dims)
    B = q_nope.shape[0]
    ldq = _headrows(q_nope, "q_nope")
    if w_fp8.dtype != torch.float8_e4m3fn or w_scale.dtype != torch.float32 or not w_scale.is_contiguous():
        raise TypeError("w_fp8 must be float8_e4m3fn and w_scale contiguous float32")
    if q_tilde is None:
        q_tilde = torch.empty((B, d.n_h, d.d_c), dtype=torch.bfloat16, device=q_nope.device)
    check(lib().mla_absorb_q_fp8(d, B, _ptr(q_nope), ldq, _ptr(w_fp8), _ptr(w_scale), _ptr(q_tilde), _ptr(dev_err),
                                 _stream(stream)), "mla_absorb_q_fp8")
    return q_tilde


def mla_out_up_fp8(dims, ctx: torch.Tensor, w_fp8: torch.Tensor, w_scale: torch.Tensor,
                   out: Optional[torch.Tensor] = None, dev_err: Optional[torch.Tensor] = None,
                   stream=None) -> torch.Tensor:
    """mla_out_up with an e4m3 wkv_b and its fp32 128 x 128 block scales."""
    d = _dims(dims)
    B = ctx.shape[0]
    if not ctx.is_contiguous():
        raise ValueError("ctx must be contiguous")
    if w_fp8.dtype != torch.float8_e4m3fn or w_scale.dtype != torch.float32 or not w_scale.is_contiguous():
        raise TypeError("w_fp8 must be float8_e4m3fn and w_scale contiguous float32")
    if out is None:
        out = torch.empty((B, d.n_h, d.d_v), dtype=torch.bfloat16, device=ctx.device)
    check(lib().mla_out_up_fp8(d, B, _ptr(ctx), _ptr(w_fp8), _ptr(w_scale), _ptr(out), _ptr(dev_err),
                               _stream(stream)), "mla_out_up_fp8")
    return out


def mla_prefill_workspace_size(dims, dtype: torch.dtype, B: int, S: int) -> int:
    return int(lib().mla_prefill_workspace_size(_dims(dims), _dtc(dtype), B, S))


def mla_prefill_naive(dims, q: torch.Tensor, c_kv: torch.Tensor, k_r: torch.Tensor, w_kv_b: torch.Tensor,
                      scale: float, causal: bool = True, out: Optional[torch.Tensor] = None,
                      workspace: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """Naive-path prefill.  q [B, S, n_h, d_h + d_r] contiguous; c_kv [B, S, d_c] and k_r [B, S, d_r]
    with contiguous rows and (b, s) rows evenly strided."""
    d = _dims(dims)
    B, S = c_kv.shape[0], c_kv.shape[1]
    if not q.is_contiguous():
        raise ValueError("q must be contiguous")
    for t, n in ((c_kv, "c_kv"), (k_r, "k_r")):
        _rows(t, n)
        if t.stride(0) != S * t.stride(1):
            raise ValueError(f"{n}: rows of consecutive sequences must be evenly strided")
    if out is None:
        out = torch.empty((B, S, d.n_h, d.d_v), dtype=q.dtype, device=q.device)
    if workspace is None:
        nbytes = mla_prefill_workspace_size(d, q.dtype, B, S)
        workspace = torch.empty((max(nbytes, 16),), dtype=torch.uint8, device=q.device)
    check(lib().mla_prefill_naive(d, _dt(q), B, S, _ptr(q), _ptr(c_kv), c_kv.stride(1), _ptr(k_r), k_r.stride(1),
                                  _ptr(w_kv_b), float(scale), 1 if causal else 0, _ptr(out), _ptr(workspace),
                                  workspace.numel() * workspace.element_size(), _stream(stream)),
          "mla_prefill_naive")
    return out


def mla_cache_append(dims, kv_a: torch.Tensor, positions: torch.Tensor, c_kv: torch.Tensor, k_r: torch.Tensor,
                     gain: Optional[torch.Tensor] = None, eps: float = 1e-6, rope_base: float = 10000.0,
                     dev_err: Optional[torch.Tensor] = None, stream=None) -> None:
    """Write each sequence's new token into the caches in place: RMSNorm(kv_a[b, :d_c]) * gain into
    c_kv[b, positions[b]] and the rotary key kv_a[b, d_c:] rotated by positions[b] into
    k_r[b, positions[b]].  kv_a [B, d_c + d_r] (rows may be strided); positions int32 [B];
    c_kv [B, n_max, d_c] and k_r [B, n_max, d_r] may be views of one packed cache; gain fp32 [d_c]."""
    d = _dims(dims)
    B, n_max = c_kv.shape[0], c_kv.shape[1]
    _rows(kv_a, "kv_a")
    _rows(c_kv, "c_kv")
    _rows(k_r, "k_r")
    if kv_a.dim() != 2 or kv_a.shape[0] != B:
        raise ValueError("kv_a must be [B, d_c + d_r]")
    if positions.dtype != torch.int32 or not positions.is_contiguous():
        raise TypeError("positions must be a contiguous int32 tensor")
    if gain is not None and (gain.dtype != torch.float32 or not gain.is_contiguous()):
        raise TypeError("gain must be a contiguous float32 tensor")
    check(lib().mla_cache_append(d, _dt(kv_a), B, _ptr(kv_a), kv_a.stride(0), _ptr(gain), float(eps),
                                 float(rope_base), _ptr(positions), n_max,
                                 _ptr(c_kv), c_kv.stride(0), c_kv.stride(1), _ptr(k_r), k_r.stride(0),
                                 k_r.stride(1), _ptr(dev_err), _stream(stream)), "mla_cache_append")


def mla_check_topk(topk_idx: torch.Tensor, n_max: int, lengths: Optional[torch.Tensor] = None,
                   dev_err: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """Validate a top-k index array on the device: every index of row b inside [0, lengths[b])
    (n_max when lengths is None) and listed once.  Sets MLA_ERR_INDEX / MLA_ERR_LENGTH in `dev_err`
    (allocated zeroed here when not given), which is returned; read it with mla_get_device_error."""
    if topk_idx.dtype != torch.int32 or not topk_idx.is_contiguous() or topk_idx.dim() != 2:
        raise TypeError("topk_idx must be a contiguous int32 [B, topk] tensor")
    if lengths is not None and (lengths.dtype != torch.int32 or not lengths.is_contiguous()):
        raise TypeError("lengths must be a contiguous int32 tensor")
    if dev_err is None:
        dev_err = torch.zeros(1, dtype=torch.int32, device=topk_idx.device)
    check(lib().mla_check_topk(topk_idx.shape[0], _ptr(topk_idx), topk_idx.shape[1], _ptr(lengths), int(n_max),
                               _ptr(dev_err), _stream(stream)), "mla_check_topk")
    return dev_err


def mla_prefill_sparse(dims, q: torch.Tensor, c_kv: torch.Tensor, k_r: torch.Tensor, w_kv_b: torch.Tensor,
                       scale: float, topk_idx: torch.Tensor, out: Optional[torch.Tensor] = None,
                       workspace: Optional[torch.Tensor] = None, dev_err: Optional[torch.Tensor] = None,
                       stream=None) -> torch.Tensor:
    """Sparse prefill: as mla_prefill_naive (causal), each query row attending only the positions
    its row of topk_idx (int32 [B, S, k]) selects."""
    d = _dims(dims)
    B, S = c_kv.shape[0], c_kv.shape[1]
    if not q.is_contiguous():
        raise ValueError("q must be contiguous")
    for t, n in ((c_kv, "c_kv"), (k_r, "k_r")):
        _rows(t, n)
        if t.stride(0) != S * t.stride(1):
            raise ValueError(f"{n}: rows of consecutive sequences must be evenly strided")
    if topk_idx.dtype != torch.int32 or not topk_idx.is_contiguous() or tuple(topk_idx.shape[:2]) != (B, S):
        raise TypeError("topk_idx must be a contiguous int32 [B, S, k] tensor")
    if out is None:
        out = torch.empty((B, S, d.n_h, d.d_v), dtype=q.dtype, device=q.device)
    if workspace is None:
        nbytes = int(lib().mla_prefill_sparse_workspace_size(d, _dt(q), B, S))
        workspace = torch.empty((max(nbytes, 16),), dtype=torch.uint8, device=q.device)
    check(lib().mla_prefill_sparse(d, _dt(q), B, S, _ptr(q), _ptr(c_kv), c_kv.stride(1), _ptr(k_r), k_r.stride(1),
                                   _ptr(w_kv_b), float(scale), _ptr(topk_idx), topk_idx.shape[2], _ptr(out),
                                   _ptr(workspace), workspace.numel() * workspace.element_size(), _ptr(dev_err),
                                   _stream(stream)), "mla_prefill_sparse")
    return out


def mla_clear_device_error(dev_err: torch.Tensor, stream=None) -> None:
    check(lib().mla_clear_device_error(_ptr(dev_err), _stream(stream)), "mla_clear_device_error")


def mla_get_device_error(dev_err: torch.Tensor) -> int:
    out = ctypes.c_int32(0)
    check(lib().mla_get_device_error(_ptr(dev_err), ctypes.byref(out)), "mla_get_device_error")
    return int(out.value)

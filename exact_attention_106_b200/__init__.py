"""exattn: exact scaled-dot-product attention on B200 (sm_100a).

Python face of the C ABI in include/exattn.h.  Every function here only
checks and marshals arguments (device pointers and the current CUDA stream)
and calls the library; all arithmetic runs in its CUDA kernels.  PyTorch is
used for device memory and streams.

    o, lse = forward(q, k, v, causal=False, scale=None)
    dq, dk, dv = backward(q, k, v, o, lse, do, causal=False, scale=None)

Tensors are CUDA bfloat16 (or float16, through the _fp16 entry points),
contiguous [B, H, N, d] with d in {64, 128}; lse is float32 [B, H, N].
``scale`` defaults to 1/sqrt(d).
"""
from __future__ import annotations

import math
from typing import Optional

import torch

from . import _lib

__all__ = ["forward", "backward", "forward_fp8", "forward_kvsplit", "kvsplit_plan", "forward_backward_host", "bwd_workspace_bytes", "host_buffer_bytes",
           "device_status", "set_wait_timeout_ns", "ExattnError"]

ExattnError = _lib.ExattnError


def _stream(device: torch.device) -> int:
    return torch.cuda.current_stream(device).cuda_stream


# element type -> (forward, backward) entry points of the C ABI
_ENTRY = {torch.bfloat16: ("attn_fwd", "attn_bwd"), torch.float16: ("attn_fwd_fp16", "attn_bwd_fp16")}
_KVSPLIT_ENTRY = {torch.bfloat16: "attn_fwd_kvsplit", torch.float16: "attn_fwd_kvsplit_fp16"}


def _check_qkv(*ts: torch.Tensor) -> None:
    shape, dtype = ts[0].shape, ts[0].dtype
    for t in ts:
        if not (t.is_cuda and t.dtype in _ENTRY and t.is_contiguous() and t.dim() == 4):
            raise ValueError("expected contiguous CUDA bfloat16 or float16 tensors [B, H, N, d]")
        if t.shape != shape or t.device != ts[0].device or t.dtype != dtype:
            raise ValueError("q, k, v (and o, do) must share shape, dtype and device")


def _scale(d: int, scale: Optional[float]) -> float:
    return 1.0 / math.sqrt(d) if scale is None else float(scale)


def _check_status(fn: str, device) -> None:
    """Synchronise and raise if a kernel of the library gave up on a bounded
    wait (the results of that call are then undefined)."""
    st = device_status(device)
    if st != _lib.ATTN_OK:
        raise ExattnError(fn, st)


def forward(q, k, v, causal: bool = False, scale: Optional[float] = None, out=None, lse=None,
            check: bool = False):
    """O and per-row logsumexp of softmax(scale Q K^T) V.

    The call only enqueues the kernel.  A kernel that gives up on one of its
    bounded internal waits (about a second; it should never happen) leaves
    undefined outputs and records ATTN_ERR_TIMEOUT, which ``device_status()``
    reports; with ``check=True`` the call synchronises and raises ExattnError
    in that case."""
    _check_qkv(q, k, v)
    B, H, N, d = q.shape
    o = torch.empty_like(q) if out is None else out
    lse_t = torch.empty((B, H, N), dtype=torch.float32, device=q.device) if lse is None else lse
    name = _ENTRY[q.dtype][0]
    _lib.check(name, getattr(_lib.load(), name)(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(),
                                               lse_t.data_ptr(), B, H, N, d, _scale(d, scale), int(causal),
                                               _stream(q.device)))
    if check:
        _check_status(name, q.device)
    return o, lse_t


def forward_fp8(q, k, v, q_descale: float, k_descale: float, v_descale: float, causal: bool = False,
                scale: Optional[float] = None, out=None, lse=None, check: bool = False):
    """Forward on e4m3 inputs (attn_fwd_fp8): q, k, v CUDA float8_e4m3fn
    [B, H, N, 128] whose real values are q * q_descale etc.  Returns
    (o bf16, lse fp32)."""
    for t in (q, k, v):
        if not (t.is_cuda and t.dtype == torch.float8_e4m3fn and t.is_contiguous() and t.dim() == 4):
            raise ValueError("expected contiguous CUDA float8_e4m3fn tensors [B, H, N, d]")
        if t.shape != q.shape or t.device != q.device:
            raise ValueError("q, k, v must share shape and device")
    B, H, N, d = q.shape
    o = torch.empty((B, H, N, d), dtype=torch.bfloat16, device=q.device) if out is None else out
    lse_t = torch.empty((B, H, N), dtype=torch.float32, device=q.device) if lse is None else lse
    _lib.check("attn_fwd_fp8", _lib.load().attn_fwd_fp8(
        q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse_t.data_ptr(), B, H, N, d, _scale(d, scale),
        int(causal), float(q_descale), float(k_descale), float(v_descale), _stream(q.device)))
    if check:
        _check_status("attn_fwd_fp8", q.device)
    return o, lse_t


def kvsplit_plan(B: int, H: int, Nq: int, Nk: int, d: int, causal: bool = False, splits: int = 0):
    """(number of key ranges, workspace bytes) that ``forward_kvsplit`` uses."""
    lib = _lib.load()
    return (int(lib.attn_fwd_kvsplit_count(B, H, Nq, Nk, d, int(causal), splits)),
            int(lib.attn_fwd_kvsplit_workspace_bytes(B, H, Nq, Nk, d, int(causal), splits)))


def forward_kvsplit(q, k, v, causal: bool = False, scale: Optional[float] = None, splits: int = 0,
                    workspace: Optional[torch.Tensor] = None, out=None, lse=None, check: bool = False):
    """Forward over Nq queries and Nk keys with the keys split into ranges
    (attn_fwd_kvsplit): decode (Nq small, Nk long) and long rows.

    q: [B, H, Nq, d], k, v: [B, H, Nk, d], CUDA bfloat16 or float16 (all
    three alike), contiguous.  Under ``causal`` the queries are the last Nq
    positions (query i sees keys j <= Nk - Nq + i).  ``splits`` 0 lets the
    library choose.
    """
    for t in (q, k, v):
        if not (t.is_cuda and t.dtype in _KVSPLIT_ENTRY and t.dtype == q.dtype and t.is_contiguous()
                and t.dim() == 4):
            raise ValueError("expected contiguous CUDA bfloat16 or float16 tensors [B, H, N, d] of one dtype")
    B, H, Nq, d = q.shape
    if k.shape != (B, H, k.shape[2], d) or v.shape != k.shape:
        raise ValueError("k and v must be [B, H, Nk, d] with q's B, H, d")
    Nk = k.shape[2]
    o = torch.empty_like(q) if out is None else out
    lse_t = torch.empty((B, H, Nq), dtype=torch.float32, device=q.device) if lse is None else lse
    _, need = kvsplit_plan(B, H, Nq, Nk, d, causal, splits)
    ws = workspace
    if ws is None:
        ws = torch.empty(max(1, need), dtype=torch.uint8, device=q.device)
    name = _KVSPLIT_ENTRY[q.dtype]
    _lib.check(name, getattr(_lib.load(), name)(
        q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse_t.data_ptr(), B, H, Nq, Nk, d,
        _scale(d, scale), int(causal), int(splits), ws.data_ptr(), ws.numel(), _stream(q.device)))
    if check:
        _check_status(name, q.device)
    return o, lse_t


def bwd_workspace_bytes(B: int, H: int, N: int, d: int) -> int:
    return int(_lib.load().attn_bwd_workspace_bytes(B, H, N, d))


def alloc_workspace(B: int, H: int, N: int, d: int, device) -> torch.Tensor:
    """A device buffer for the backward (torch allocations are 256-byte aligned)."""
    n = max(1, bwd_workspace_bytes(B, H, N, d))
    return torch.empty(n, dtype=torch.uint8, device=device)


def backward(q, k, v, o, lse, do, causal: bool = False, scale: Optional[float] = None,
             workspace: Optional[torch.Tensor] = None, out=None, check: bool = False):
    """dQ, dK, dV of sum(O * dO) for O = softmax(scale Q K^T) V.

    ``check=True`` synchronises and raises ExattnError if a kernel gave up on
    a bounded wait (see ``forward``); otherwise such a failure is only seen
    through ``device_status()``."""
    _check_qkv(q, k, v, o, do)
    B, H, N, d = q.shape
    if not (lse.is_cuda and lse.dtype == torch.float32 and lse.is_contiguous() and lse.shape == (B, H, N)):
        raise ValueError("lse must be contiguous CUDA float32 [B, H, N]")
    if out is None:
        dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    else:
        dq, dk, dv = out
    ws = alloc_workspace(B, H, N, d, q.device) if workspace is None else workspace
    name = _ENTRY[q.dtype][1]
    _lib.check(name, getattr(_lib.load(), name)(
        q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(), do.data_ptr(),
        dq.data_ptr(), dk.data_ptr(), dv.data_ptr(), B, H, N, d, _scale(d, scale), int(causal),
        ws.data_ptr(), ws.numel(), _stream(q.device)))
    if check:
        _check_status(name, q.device)
    return dq, dk, dv


def bwd_stages(q, k, v, o, lse, do, dq, dk, dv, workspace, causal: bool = False,
               scale: Optional[float] = None):
    """The backward as three separate C-ABI calls (what ``backward`` runs), each
    returning after its launch; yields between stages so a caller can record
    CUDA events around each.  bf16 only (the stages have no fp16 entry
    points)."""
    if q.dtype != torch.bfloat16:
        raise ValueError("bwd_stages takes bfloat16 tensors")
    B, H, N, d = q.shape
    sc = _scale(d, scale)
    st = _stream(q.device)
    lib = _lib.load()
    _lib.check("attn_bwd_preprocess", lib.attn_bwd_preprocess(
        o.data_ptr(), do.data_ptr(), lse.data_ptr(), B, H, N, d, workspace.data_ptr(), workspace.numel(), st))
    yield "preprocess"
    _lib.check("attn_bwd_dkdv", lib.attn_bwd_dkdv(
        q.data_ptr(), k.data_ptr(), v.data_ptr(), do.data_ptr(), dk.data_ptr(), dv.data_ptr(), B, H, N, d, sc,
        int(causal), workspace.data_ptr(), workspace.numel(), st))
    yield "dkdv"
    _lib.check("attn_bwd_dq_convert", lib.attn_bwd_dq_convert(
        dq.data_ptr(), B, H, N, d, sc, workspace.data_ptr(), workspace.numel(), st))
    yield "dq_convert"


def host_buffer_bytes(B: int, H: int, N: int, d: int, heads_per_chunk: int = 0) -> int:
    return int(_lib.load().attn_fwd_bwd_host_buffer_bytes(B, H, N, d, heads_per_chunk))


def forward_backward_host(q, k, v, do, out, causal: bool = False, scale: Optional[float] = None,
                          device=None, dev_buffer: Optional[torch.Tensor] = None, heads_per_chunk: int = 0):
    """Forward and backward over HOST tensors, copies included (attn_fwd_bwd_host).

    q, k, v, do: CPU bf16 [B, H, N, d] (page-locked for the copies to overlap the
    kernels); out = (o, lse, dq, dk, dv), CPU tensors written once the current
    stream of ``device`` reaches the end of the call's work.  As with
    ``forward``, a kernel timeout is reported only by ``device_status()``.
    """
    tensors = (q, k, v, do) + tuple(out)
    o, lse, dq, dk, dv = out
    B, H, N, d = q.shape
    for t in (q, k, v, do, o, dq, dk, dv):
        if t.is_cuda or t.dtype != torch.bfloat16 or not t.is_contiguous() or tuple(t.shape) != (B, H, N, d):
            raise ValueError("q, k, v, do, o, dq, dk, dv must be contiguous CPU bfloat16 [B, H, N, d]")
    if lse.is_cuda or lse.dtype != torch.float32 or not lse.is_contiguous() or tuple(lse.shape) != (B, H, N):
        raise ValueError("lse must be contiguous CPU float32 [B, H, N]")
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
    need = host_buffer_bytes(B, H, N, d, heads_per_chunk)
    buf = torch.empty(max(1, need), dtype=torch.uint8, device=dev) if dev_buffer is None else dev_buffer
    with torch.cuda.device(dev):
        _lib.check("attn_fwd_bwd_host", _lib.load().attn_fwd_bwd_host(
            *(t.data_ptr() for t in tensors[:4]), o.data_ptr(), lse.data_ptr(), dq.data_ptr(), dk.data_ptr(),
            dv.data_ptr(), B, H, N, d, _scale(d, scale), int(causal), buf.data_ptr(), buf.numel(),
            int(heads_per_chunk), _stream(dev)))
    return out


def set_wait_timeout_ns(ns: int) -> None:
    """Limit of every device-side wait of the library's kernels, in ns (0
    restores the default of one second).  The environment variable
    EXATTN_WAIT_TIMEOUT_NS sets it when the library is loaded."""
    if ns < 0:
        raise ValueError("the wait limit must be >= 0")
    _lib.load().attn_set_wait_timeout_ns(int(ns))


def device_status(device=None) -> int:
    """Synchronise the current stream and return (and clear) the device status word."""
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
    with torch.cuda.device(dev):
        return int(_lib.load().attn_get_device_status(_stream(dev)))

"""winattn: fused, exact windowed softmax attention for vision transformers on
B200 (sm_100a), behind a C ABI (include/winattn.h).

``window_attention`` is the public call on device tensors; ``window_attention_host``
runs the same call on host tensors (copies in, kernel, copy out, all enqueued by
the library).  Both go through the CUDA library; nothing here computes.
"""
from __future__ import annotations

from typing import Optional

import torch

from . import _lib
from ._lib import WinattnError

__all__ = ["window_attention", "window_attention_host", "window_attention_backward", "window_attention_autograd",
           "window_attention_gated_residual", "rib_features", "window_attention_rib", "cla_gate", "WinattnError",
           "device_status"]


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return _lib.BF16
    if t.dtype == torch.float32:
        return _lib.FP32
    raise WinattnError(_lib.ERR_DTYPE, f"unsupported dtype {t.dtype}")


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else t.data_ptr()


def _shape(q, k, v, theta, bias, M):
    if q.dim() != 5 or q.shape != k.shape or q.shape != v.shape:
        raise WinattnError(_lib.ERR_ARG, "q, k, v must share one [B, H, W, heads, d] shape")
    if q.dtype != k.dtype or q.dtype != v.dtype:
        raise WinattnError(_lib.ERR_DTYPE, "q, k, v must share one dtype")
    for t in (q, k, v, theta, bias):
        if t is not None and not t.is_contiguous():
            raise WinattnError(_lib.ERR_ARG, "tensors must be contiguous")
    B, H, W, heads, d = q.shape
    if theta is not None and (theta.dtype != torch.float32 or tuple(theta.shape) != (heads, d // 4)):
        raise WinattnError(_lib.ERR_ARG, "theta must be fp32 [heads, d/4]")
    rank = 0
    if bias is not None:
        if bias.dim() != 4 or tuple(bias.shape[:3]) != (heads, 2, M * M) or bias.dtype != q.dtype:
            raise WinattnError(_lib.ERR_RANK, "bias_feats must be [heads, 2, M*M, rank] in q's dtype")
        rank = bias.shape[3]
    return B, H, W, heads, d, rank


def window_attention(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, M: int, shift: int = 0,
                     theta: Optional[torch.Tensor] = None, bias_feats: Optional[torch.Tensor] = None,
                     out: Optional[torch.Tensor] = None, lse: Optional[torch.Tensor] = None) -> torch.Tensor:
    """Fused window attention on CUDA tensors [B, H, W, heads, d] (bf16 or fp32),
    enqueued on torch's current stream.  See include/winattn.h for the exact
    operation.  With ``lse`` (fp32 [B, H, W, heads]) each row's log-sum-exp is
    saved there for the backward (winattn_fwd_lse)."""
    B, H, W, heads, d, rank = _shape(q, k, v, theta, bias_feats, M)
    for t in (q, k, v, theta, bias_feats):
        if t is not None and not t.is_cuda:
            raise WinattnError(_lib.ERR_ARG, "window_attention takes CUDA tensors")
    if out is None:
        out = torch.empty_like(q)
    dev = q.device
    stream = torch.cuda.current_stream(dev).cuda_stream
    if lse is not None and (lse.dtype != torch.float32 or tuple(lse.shape) != (B, H, W, heads) or not lse.is_cuda
                            or not lse.is_contiguous()):
        raise WinattnError(_lib.ERR_ARG, "lse must be a contiguous fp32 CUDA tensor [B, H, W, heads]")
    args = (_ptr(q), _ptr(k), _ptr(v), _ptr(theta), _ptr(bias_feats), B, H, W, M, shift, heads, d, rank,
            _dtype_code(q), _ptr(out))
    call, what = (_lib.fwd, "winattn_fwd") if lse is None else (_lib.fwd_lse, "winattn_fwd_lse")
    args = args + ((stream,) if lse is None else (_ptr(lse), stream))
    # the library works on the current device: switch only when q lives elsewhere
    if torch.cuda.current_device() == dev.index:
        rc = call(*args)
    else:
        with torch.cuda.device(dev):
            rc = call(*args)
    if rc != _lib.OK:
        raise WinattnError(rc, what)
    return out


def window_attention_gated_residual(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, o_lin: torch.Tensor,
                                    windows: torch.Tensor, M: int, shift: int = 0,
                                    theta: Optional[torch.Tensor] = None,
                                    bias_feats: Optional[torch.Tensor] = None) -> torch.Tensor:
    """HSMLA's two-path residual on the gated windows (winattn_fwd_sparse):
    ``o_lin`` (bf16, shaped like q) is updated in place for the tokens of the
    listed windows (int32 CUDA tensor of window ids) and returned."""
    B, H, W, heads, d, rank = _shape(q, k, v, theta, bias_feats, M)
    if o_lin.shape != q.shape or o_lin.dtype != q.dtype or not o_lin.is_contiguous():
        raise WinattnError(_lib.ERR_ARG, "o_lin must be contiguous and shaped like q")
    if windows.dtype != torch.int32 or windows.dim() != 1 or not windows.is_contiguous():
        raise WinattnError(_lib.ERR_ARG, "windows must be a contiguous int32 vector")
    dev = q.device
    stream = torch.cuda.current_stream(dev).cuda_stream
    with torch.cuda.device(dev):
        rc = _lib.fwd_sparse(_ptr(q), _ptr(k), _ptr(v), _ptr(theta), _ptr(bias_feats), B, H, W, M, shift, heads, d,
                             rank, _dtype_code(q), _ptr(windows), windows.numel(), _ptr(o_lin), stream)
    if rc != _lib.OK:
        raise WinattnError(rc, "winattn_fwd_sparse")
    return o_lin


def _call(fn, what, dev, *args):
    with torch.cuda.device(dev):
        rc = fn(*args, torch.cuda.current_stream(dev).cuda_stream)
    if rc != _lib.OK:
        raise WinattnError(rc, what)


def rib_features(w1: torch.Tensor, w2: torch.Tensor, M: int, table: Optional[torch.Tensor] = None) -> torch.Tensor:
    """The RIB factor table [heads, 2, M*M, rank] (bf16) from the MLP weights
    w1 [heads, 2, 32, 64] and w2 [heads, 2, 64, rank] (fp32 CUDA tensors)."""
    heads, rank = w1.shape[0], w2.shape[3]
    if tuple(w1.shape) != (heads, 2, 32, 64) or tuple(w2.shape) != (heads, 2, 64, rank) or \
            w1.dtype != torch.float32 or w2.dtype != torch.float32:
        raise WinattnError(_lib.ERR_ARG, "w1 must be fp32 [heads, 2, 32, 64] and w2 fp32 [heads, 2, 64, rank]")
    if table is None:
        table = torch.empty((heads, 2, M * M, rank), dtype=torch.bfloat16, device=w1.device)
    _call(_lib.rib_features, "winattn_rib_features", w1.device, _ptr(w1.contiguous()), _ptr(w2.contiguous()), M,
          heads, rank, _ptr(table))
    return table


def window_attention_rib(q, k, v, M: int, shift: int, w1: torch.Tensor, w2: torch.Tensor,
                         theta: Optional[torch.Tensor] = None, out: Optional[torch.Tensor] = None,
                         table: Optional[torch.Tensor] = None):
    """Window attention whose rank-r bias features are generated from the RIB
    MLP weights in the same call (winattn_fwd_rib); returns (out, table)."""
    heads, rank = w1.shape[0], w2.shape[3]
    B, H, W, hq, d = q.shape
    if table is None:
        table = torch.empty((heads, 2, M * M, rank), dtype=torch.bfloat16, device=q.device)
    if out is None:
        out = torch.empty_like(q)
    _call(_lib.fwd_rib, "winattn_fwd_rib", q.device, _ptr(q), _ptr(k), _ptr(v), _ptr(theta), _ptr(w1), _ptr(w2), B,
          H, W, M, shift, heads, d, rank, _dtype_code(q), _ptr(table), _ptr(out))
    return out, table


def cla_gate(x: torch.Tensor, o: torch.Tensor, dw: torch.Tensor, dw_b: torch.Tensor, pw: torch.Tensor,
             pw_b: torch.Tensor, out: Optional[torch.Tensor] = None) -> torch.Tensor:
    """out = o * sigmoid(PW(DW3x3(x))) (winattn_cla_gate); x, o bf16 [B, H, W, C];
    dw fp32 [C, 3, 3], dw_b [C], pw [C, C], pw_b [C].  out may be o."""
    B, H, W, C = x.shape
    if o.shape != x.shape or not x.is_contiguous() or not o.is_contiguous():
        raise WinattnError(_lib.ERR_ARG, "x and o must be contiguous [B, H, W, C] tensors")
    if out is None:
        out = torch.empty_like(o)
    _call(_lib.cla_gate, "winattn_cla_gate", x.device, _ptr(x), _ptr(o), _ptr(dw.contiguous()),
          _ptr(dw_b.contiguous()), _ptr(pw.contiguous()), _ptr(pw_b.contiguous()), B, H, W, C, _dtype_code(x),
          _ptr(out))
    return out


def window_attention_backward(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, out: torch.Tensor,
                              dout: torch.Tensor, lse: torch.Tensor, M: int, shift: int = 0,
                              theta: Optional[torch.Tensor] = None, bias_feats: Optional[torch.Tensor] = None,
                              workspace: Optional[torch.Tensor] = None):
    """Gradients (dq, dk, dv, dtheta, dbias) of a loss given dout = dL/dO, the
    forward's ``out`` and its saved ``lse`` (``window_attention(..., lse=...)``);
    bf16 CUDA tensors, enqueued on torch's current stream (winattn_bwd).
    dtheta is fp32 [heads, d/4] (None without theta), dbias fp32
    [heads, 2, M*M, rank] (None without bias features)."""
    B, H, W, heads, d, rank = _shape(q, k, v, theta, bias_feats, M)
    for t in (out, dout):
        if t.shape != q.shape or t.dtype != q.dtype or not t.is_contiguous():
            raise WinattnError(_lib.ERR_ARG, "out and dout must be contiguous and shaped like q")
    if lse.dtype != torch.float32 or tuple(lse.shape) != (B, H, W, heads) or not lse.is_contiguous():
        raise WinattnError(_lib.ERR_ARG, "lse must be a contiguous fp32 tensor [B, H, W, heads]")
    dev = q.device
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    dtheta = None if theta is None else torch.empty((heads, d // 4), dtype=torch.float32, device=dev)
    dbias = None if bias_feats is None else torch.empty(tuple(bias_feats.shape), dtype=torch.float32, device=dev)
    need = _lib.bwd_workspace_bytes(B, H, W, M, heads, d)
    if workspace is None and need:
        workspace = torch.empty(need, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev).cuda_stream
    with torch.cuda.device(dev):
        rc = _lib.bwd(_ptr(q), _ptr(k), _ptr(v), _ptr(theta), _ptr(bias_feats), _ptr(out), _ptr(dout), _ptr(lse),
                      B, H, W, M, shift, heads, d, rank, _dtype_code(q), _ptr(dq), _ptr(dk), _ptr(dv), _ptr(dtheta),
                      _ptr(dbias), _ptr(workspace), 0 if workspace is None else workspace.numel(), stream)
    if rc != _lib.OK:
        raise WinattnError(rc, "winattn_bwd")
    return dq, dk, dv, dtheta, dbias


class _WindowAttention(torch.autograd.Function):
    """Forward through winattn_fwd_lse (saving each row's log-sum-exp),
    backward through winattn_bwd: gradients for q, k, v, theta and the bias
    features."""

    @staticmethod
    def forward(ctx, q, k, v, theta, bias_feats, M, shift):
        B, H, W, heads, d = q.shape
        lse = torch.empty((B, H, W, heads), dtype=torch.float32, device=q.device)
        out = window_attention(q, k, v, M, shift, theta=theta, bias_feats=bias_feats, lse=lse)
        ctx.save_for_backward(q, k, v, theta, bias_feats, out, lse)
        ctx.M, ctx.shift = M, shift
        return out

    @staticmethod
    def backward(ctx, dout):
        q, k, v, theta, bias, out, lse = ctx.saved_tensors
        dq, dk, dv, dth, dbi = window_attention_backward(q, k, v, out, dout.contiguous(), lse, ctx.M, ctx.shift,
                                                         theta=theta, bias_feats=bias)
        if dbi is not None:
            dbi = dbi.to(bias.dtype)
        return dq, dk, dv, dth, dbi, None, None


def window_attention_autograd(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, M: int, shift: int = 0,
                              theta: Optional[torch.Tensor] = None,
                              bias_feats: Optional[torch.Tensor] = None) -> torch.Tensor:
    """window_attention as a differentiable torch op (bf16 CUDA tensors):
    the learned frequencies theta (e.g. theta = omega.exp()) and the bias
    features receive gradients too."""
    return _WindowAttention.apply(q, k, v, theta, bias_feats, M, shift)


def window_attention_host(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, M: int, shift: int = 0,
                          theta: Optional[torch.Tensor] = None, bias_feats: Optional[torch.Tensor] = None,
                          out: Optional[torch.Tensor] = None, workspace: Optional[torch.Tensor] = None,
                          device=None, synchronize: bool = True) -> torch.Tensor:
    """The same operation on host tensors (pinned for asynchronous copies);
    theta / bias_feats are CUDA tensors.  ``workspace`` is a uint8 CUDA tensor of
    at least ``host_workspace_bytes`` bytes (allocated here when omitted)."""
    B, H, W, heads, d, rank = _shape(q, k, v, theta, bias_feats, M)
    device = torch.device(device or (theta.device if theta is not None else "cuda"))
    code = _dtype_code(q)
    need = _lib.host_workspace_bytes(B, H, W, heads, d, code)
    if workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=device)
    if out is None:
        out = torch.empty_like(q, pin_memory=q.is_pinned())
    stream = torch.cuda.current_stream(device).cuda_stream
    with torch.cuda.device(device):
        rc = _lib.fwd_host(_ptr(q), _ptr(k), _ptr(v), _ptr(theta), _ptr(bias_feats), B, H, W, M, shift, heads,
                           d, rank, code, _ptr(out), _ptr(workspace), workspace.numel(), stream)
    if rc != _lib.OK:
        raise WinattnError(rc, "winattn_fwd_host")
    if synchronize:
        torch.cuda.current_stream(device).synchronize()
    return out


def host_workspace_bytes(q: torch.Tensor) -> int:
    B, H, W, heads, d = q.shape
    return _lib.host_workspace_bytes(B, H, W, heads, d, _dtype_code(q))


def device_status(device=None) -> int:
    """Synchronise torch's current stream and read/clear the bounded-wait status."""
    dev = torch.device(device or "cuda")
    with torch.cuda.device(dev):
        return _lib.last_device_status(torch.cuda.current_stream(dev).cuda_stream)

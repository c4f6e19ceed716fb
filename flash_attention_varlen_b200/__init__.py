"""Varlen block-diagonal attention forward for NVIDIA B200 (sm_100a).

``attn_fwd`` is the PyTorch-facing call: it checks shapes, dtypes and devices
and passes raw pointers to the C-ABI library (``libvtattn.so``,
``include/vt_attn.h``).  PyTorch provides device memory and streams only; the
computation is the library's CUDA kernels.

    out = attn_fwd(q, k, v, cu_seqlens)              # q/k/v: [T, 16, 96] bf16 or f32, cuda
    out = attn_fwd(q, k, v, cu_seqlens, scale=0.1)   # cu_seqlens: int32 [n+1] on the same device
"""
from __future__ import annotations

import math

from . import _binding
from ._binding import (VT_DTYPE_BF16, VT_DTYPE_F32, VT_OK, VtAttnError, status_string,
                       vt_attn_fwd, vt_attn_last_device_status, vt_attn_smem_bytes,
                       vt_attn_validate_seqlens_host, vt_attn_version, vt_attn_workspace_bytes)

__all__ = ["attn_fwd", "attn_fwd_host", "check_device_status", "VtAttnError", "vt_attn_fwd",
           "vt_attn_validate_seqlens_host", "vt_attn_smem_bytes", "vt_attn_workspace_bytes",
           "vt_attn_last_device_status", "status_string", "vt_attn_version"]


def _dtype_code(t):
    import torch
    if t.dtype == torch.bfloat16:
        return VT_DTYPE_BF16
    if t.dtype == torch.float32:
        return VT_DTYPE_F32
    raise TypeError(f"attn_fwd: unsupported dtype {t.dtype} (bfloat16 or float32)")


def attn_fwd(q, k, v, cu_seqlens, scale: float | None = None, out=None, stream=None):
    """Block-diagonal attention over packed segments.

    q, k, v: CUDA tensors [T, H, D] (contiguous, same dtype: bfloat16 or float32).
    cu_seqlens: int32 CUDA tensor [num_segments + 1] (0 = cu[0] <= ... <= cu[n] = T).
    scale: softmax scale, default 1/sqrt(D).  Runs on ``stream`` (default: the
    current torch stream) and returns ``out`` ([T, H, D], same dtype).
    """
    import torch
    if q.dim() != 3 or k.shape != q.shape or v.shape != q.shape:
        raise ValueError(f"attn_fwd: q, k, v must share a [T, H, D] shape, got "
                         f"{tuple(q.shape)}, {tuple(k.shape)}, {tuple(v.shape)}")
    for name, t in (("q", q), ("k", k), ("v", v), ("cu_seqlens", cu_seqlens)):
        if not t.is_cuda:
            raise ValueError(f"attn_fwd: {name} must be a CUDA tensor")
        if not t.is_contiguous():
            raise ValueError(f"attn_fwd: {name} must be contiguous")
    if k.dtype != q.dtype or v.dtype != q.dtype:
        raise TypeError("attn_fwd: q, k, v must have the same dtype")
    if cu_seqlens.dtype != torch.int32 or cu_seqlens.dim() != 1:
        raise TypeError("attn_fwd: cu_seqlens must be a 1-D int32 tensor")
    T, H, D = q.shape
    code = _dtype_code(q)
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    if out is None:
        out = torch.empty_like(q)
    elif out.shape != q.shape or out.dtype != q.dtype or not out.is_contiguous():
        raise ValueError("attn_fwd: out must be a contiguous tensor like q")
    if stream is None:
        stream = torch.cuda.current_stream(q.device)
    handle = stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)
    with torch.cuda.device(q.device):
        rc = vt_attn_fwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(),
                         cu_seqlens.data_ptr(), cu_seqlens.numel() - 1, T, H, D, float(scale),
                         code, handle)
    if rc != VT_OK:
        raise VtAttnError(rc, "vt_attn_fwd")
    return out


def check_device_status(stream=None, device=None):
    """Synchronise the stream and raise if the last call on it found an error on the device."""
    import torch
    if stream is None:
        stream = torch.cuda.current_stream(device)
    handle = stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)
    rc = vt_attn_last_device_status(handle)
    if rc != VT_OK:
        raise VtAttnError(rc, "vt_attn_last_device_status")


def attn_fwd_host(q_host, k_host, v_host, cu_host, out_host, scale: float | None = None,
                  device_buffers=None, stream=None):
    """End-to-end call on host tensors: H2D copies, the kernel, D2H copy of the output.

    q_host/k_host/v_host/out_host: CPU tensors [T, H, D] (pinned for async copies);
    cu_host: CPU int32 [n+1].  ``device_buffers`` optionally supplies reusable
    device tensors (q, k, v, out, cu) of matching shapes.  Asynchronous on
    ``stream``; synchronise before reading ``out_host``.
    """
    import torch
    if stream is None:
        stream = torch.cuda.current_stream()
    if device_buffers is None:
        dq = torch.empty(q_host.shape, dtype=q_host.dtype, device="cuda")
        dk, dv, do = torch.empty_like(dq), torch.empty_like(dq), torch.empty_like(dq)
        dcu = torch.empty(cu_host.shape, dtype=torch.int32, device="cuda")
    else:
        dq, dk, dv, do, dcu = device_buffers
    with torch.cuda.stream(stream):
        dq.copy_(q_host, non_blocking=True)
        dk.copy_(k_host, non_blocking=True)
        dv.copy_(v_host, non_blocking=True)
        dcu.copy_(cu_host, non_blocking=True)
        attn_fwd(dq, dk, dv, dcu, scale=scale, out=do, stream=stream)
        out_host.copy_(do, non_blocking=True)
    return out_host

"""Varlen block-diagonal attention forward for NVIDIA B200 (sm_100a).

``attn_fwd`` is the PyTorch-facing call: it checks shapes, dtypes and devices
and passes raw pointers to the C-ABI library (``libvtattn.so``,
``include/vt_attn.h``).  PyTorch provides device memory and streams only; the
computation is the library's CUDA kernels.

    out = attn_fwd(q, k, v, cu_seqlens)              # q/k/v: [T, 16, 96] bf16 or f32, cuda
    out = attn_fwd(q, k, v, cu_seqlens, scale=0.1)   # cu_seqlens: int32 [n+1] on the same device

Window layers: ``window_partition`` builds, on the device, the order that makes every
32 x 32-patch window of the images one contiguous segment, and ``permute_rows`` applies it
(and its inverse) to [T, ...] tensors:

    perm, cu = window_partition([(128, 128)], device=q.device)
    qw = permute_rows(q, perm)                       # image order -> window order
    ow = attn_fwd(qw, kw, vw, cu)
    o = permute_rows(ow, perm, inverse=True)         # back to image order
"""
from __future__ import annotations

import math

from . import _binding
from ._binding import (VT_DTYPE_BF16, VT_DTYPE_F32, VT_OK, VtAttnError, status_string,
                       vt_attn_fwd, vt_attn_last_device_status, vt_attn_smem_bytes,
                       vt_attn_validate_seqlens_host, vt_attn_version, vt_attn_workspace_bytes)

__all__ = ["attn_fwd", "attn_fwd_swa", "attn_fwd_host", "window_partition", "permute_rows", "check_permute_rows",
           "rope2d", "attn_fwd_rope2d",
           "check_device_status", "VtAttnError", "vt_attn_fwd",
           "vt_attn_validate_seqlens_host", "vt_attn_smem_bytes", "vt_attn_workspace_bytes",
           "vt_attn_last_device_status", "status_string", "vt_attn_version", "set_split_keys"]


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


def attn_fwd_swa(q, k, v, cu_seqlens, window: int = 0, scale: float | None = None, out=None,
                 stream=None):
    """The text decoder's attention: causal over packed segments, query token i attending
    keys j <= i of its segment (and j > i - window when window > 0), query head h reading
    key/value head h // (Hq // Hkv).

    q: bfloat16 CUDA tensor [T, Hq, 128]; k, v: [T, Hkv, 128]; cu_seqlens: int32 CUDA tensor
    [num_segments + 1].  scale: default 1/sqrt(128).  Returns ``out`` ([T, Hq, 128]).
    """
    import torch
    if q.dim() != 3 or k.dim() != 3 or k.shape != v.shape or k.shape[0] != q.shape[0] \
            or k.shape[2] != q.shape[2]:
        raise ValueError(f"attn_fwd_swa: q [T, Hq, D], k and v [T, Hkv, D] expected, got "
                         f"{tuple(q.shape)}, {tuple(k.shape)}, {tuple(v.shape)}")
    for name, t in (("q", q), ("k", k), ("v", v), ("cu_seqlens", cu_seqlens)):
        if not t.is_cuda or not t.is_contiguous():
            raise ValueError(f"attn_fwd_swa: {name} must be a contiguous CUDA tensor")
    if q.dtype != torch.bfloat16 or k.dtype != q.dtype or v.dtype != q.dtype:
        raise TypeError("attn_fwd_swa: q, k, v must be bfloat16")
    if cu_seqlens.dtype != torch.int32 or cu_seqlens.dim() != 1:
        raise TypeError("attn_fwd_swa: cu_seqlens must be a 1-D int32 tensor")
    T, Hq, D = q.shape
    Hkv = k.shape[1]
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    if out is None:
        out = torch.empty_like(q)
    elif out.shape != q.shape or out.dtype != q.dtype or not out.is_contiguous():
        raise ValueError("attn_fwd_swa: out must be a contiguous tensor like q")
    if stream is None:
        stream = torch.cuda.current_stream(q.device)
    handle = stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)
    with torch.cuda.device(q.device):
        rc = _binding.vt_attn_fwd_swa(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(),
                                      cu_seqlens.data_ptr(), cu_seqlens.numel() - 1, T, Hq, Hkv, D,
                                      float(scale), int(window), handle)
    if rc != VT_OK:
        raise VtAttnError(rc, "vt_attn_fwd_swa")
    return out


def set_split_keys(enable: bool) -> bool:
    """Allow (True, the default) or forbid splitting a unit's keys over two CTAs in small
    bf16 calls.  Forbidding it makes a segment's output the same bits whatever else the
    call packs, at some speed on small calls.  Process-wide; returns the previous setting."""
    return bool(_binding.vt_attn_set_split_keys(1 if enable else 0))


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


def window_partition(grids, win: int = 32, device=None, stream=None):
    """(perm, cu_seqlens) for images of patch grids ``grids`` = [(h, w), ...], on ``device``.

    perm (int32 [T]): the packed image-order token at each position of the window order;
    cu_seqlens (int32 [num_windows + 1]): the windows as segments of that order.
    """
    import ctypes
    import torch
    flat = [int(x) for hw in grids for x in hw]
    if len(flat) != 2 * len(grids) or not grids:
        raise ValueError("window_partition: grids must be a non-empty list of (h, w)")
    g = (ctypes.c_int32 * len(flat))(*flat)
    nw, nt = ctypes.c_int32(0), ctypes.c_int32(0)
    rc = _binding.vt_window_count(ctypes.addressof(g), len(grids), win, ctypes.addressof(nw),
                                  ctypes.addressof(nt))
    if rc != VT_OK:
        raise VtAttnError(rc, "vt_window_count")
    device = torch.device("cuda") if device is None else torch.device(device)
    perm = torch.empty(nt.value, dtype=torch.int32, device=device)
    cu = torch.empty(nw.value + 1, dtype=torch.int32, device=device)
    if stream is None:
        stream = torch.cuda.current_stream(device)
    rc = _binding.vt_window_partition(ctypes.addressof(g), len(grids), win, perm.data_ptr(),
                                      cu.data_ptr(), stream.cuda_stream)
    if rc != VT_OK:
        raise VtAttnError(rc, "vt_window_partition")
    return perm, cu


def attn_fwd_rope2d(q, k, v, cu_seqlens, pos, theta: float = 10000.0, scale: float | None = None,
                    out=None, k_rot=None, stream=None):
    """Block-diagonal attention over rope(Q), rope(K), V (bf16 [T, H, 96] CUDA tensors).

    pos: int32 [T, 2] CUDA tensor of 1-based (pw, ph) per token.  One pass rotates Q into
    ``out`` and K into ``k_rot`` (a new tensor unless given; ``k_rot=k`` rotates in place);
    the attention then reads Q from ``out`` and writes O over it.  Returns ``out``.
    """
    import torch
    if q.dtype != torch.bfloat16 or k.dtype != q.dtype or v.dtype != q.dtype:
        raise TypeError("attn_fwd_rope2d: q, k, v must be bfloat16")
    if q.dim() != 3 or k.shape != q.shape or v.shape != q.shape:
        raise ValueError("attn_fwd_rope2d: q, k, v must share a [T, H, D] shape")
    for name, t in (("q", q), ("k", k), ("v", v), ("cu_seqlens", cu_seqlens), ("pos", pos)):
        if not t.is_cuda or not t.is_contiguous():
            raise ValueError(f"attn_fwd_rope2d: {name} must be a contiguous CUDA tensor")
    if pos.dtype != torch.int32 or tuple(pos.shape) != (q.shape[0], 2):
        raise ValueError("attn_fwd_rope2d: pos must be int32 [T, 2]")
    if cu_seqlens.dtype != torch.int32 or cu_seqlens.dim() != 1:
        raise TypeError("attn_fwd_rope2d: cu_seqlens must be a 1-D int32 tensor")
    T, H, D = q.shape
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    out = torch.empty_like(q) if out is None else out
    k_rot = torch.empty_like(k) if k_rot is None else k_rot
    if stream is None:
        stream = torch.cuda.current_stream(q.device)
    handle = stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)
    with torch.cuda.device(q.device):
        rc = _binding.vt_attn_fwd_rope2d(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(),
                                         cu_seqlens.data_ptr(), cu_seqlens.numel() - 1, T, H, D,
                                         float(scale), pos.data_ptr(), float(theta),
                                         k_rot.data_ptr(), handle)
    if rc != VT_OK:
        raise VtAttnError(rc, "vt_attn_fwd_rope2d")
    return out


def rope2d(x, pos, theta: float = 10000.0, out=None, stream=None):
    """2D RoPE of a bf16 CUDA tensor x [T, H, 96] (width first, 1-based positions).

    pos: int32 CUDA tensor [T, 2] of (pw, ph) = (column + 1, row + 1) per token.  Returns
    ``out`` (a new tensor unless given; ``out=x`` rotates in place).
    """
    import torch
    if not x.is_cuda or not pos.is_cuda or not x.is_contiguous() or not pos.is_contiguous():
        raise ValueError("rope2d: x and pos must be contiguous CUDA tensors")
    if x.dtype != torch.bfloat16 or x.dim() != 3:
        raise TypeError("rope2d: x must be a bfloat16 [T, H, D] tensor")
    if pos.dtype != torch.int32 or tuple(pos.shape) != (x.shape[0], 2):
        raise ValueError("rope2d: pos must be int32 [T, 2]")
    if out is None:
        out = torch.empty_like(x)
    if stream is None:
        stream = torch.cuda.current_stream(x.device)
    T, H, D = x.shape
    rc = _binding.vt_rope2d(x.data_ptr(), out.data_ptr(), pos.data_ptr(), T, H, D, float(theta),
                            stream.cuda_stream)
    if rc != VT_OK:
        raise VtAttnError(rc, "vt_rope2d")
    return out


def check_permute_rows(stream=None, device=None):
    """Synchronise the stream and raise if a ``permute_rows`` on this device skipped a row
    whose index was outside [0, T) since the previous check (the flag is then cleared)."""
    import torch
    if stream is None:
        stream = torch.cuda.current_stream(device)
    handle = stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)
    rc = _binding.vt_permute_rows_check(handle)
    if rc != VT_OK:
        raise VtAttnError(rc, "vt_permute_rows_check")


def permute_rows(x, perm, inverse: bool = False, out=None, stream=None):
    """Rows of ``x`` ([T, ...] CUDA tensor) in the order ``perm`` (out[i] = x[perm[i]]), or,
    with ``inverse``, put back (out[perm[i]] = x[i])."""
    import torch
    if not x.is_cuda or not perm.is_cuda or not x.is_contiguous():
        raise ValueError("permute_rows: x and perm must be contiguous CUDA tensors")
    if perm.dtype != torch.int32 or perm.dim() != 1 or perm.numel() != x.shape[0]:
        raise ValueError("permute_rows: perm must be int32 [T] with T = x.shape[0]")
    if out is None:
        out = torch.empty_like(x)
    row_bytes = x[0].numel() * x.element_size() if x.shape[0] else 16
    if stream is None:
        stream = torch.cuda.current_stream(x.device)
    rc = _binding.vt_permute_rows(x.data_ptr(), out.data_ptr(), perm.data_ptr(), x.shape[0],
                                  row_bytes, 1 if inverse else 0, stream.cuda_stream)
    if rc != VT_OK:
        raise VtAttnError(rc, "vt_permute_rows")
    return out

"""ctypes binding of libvtattn.so: the C-ABI entry points under the same names.

Argument marshalling only -- every step of the computation runs in the CUDA
library.  If the library is missing this module raises at import time; there
is no fallback path.
"""
from __future__ import annotations

import ctypes
import os

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libvtattn.so")

VT_DTYPE_BF16 = 0
VT_DTYPE_F32 = 1

VT_OK = 0
VT_ERR_NULL = 1
VT_ERR_INVALID_ARG = 2
VT_ERR_UNSUPPORTED = 3
VT_ERR_BAD_SEQLENS = 4
VT_ERR_CUDA = 5
VT_ERR_DEVICE_TIMEOUT = 6
VT_ERR_BAD_INDEX = 7

# every symbol include/vt_attn.h declares
EXPORTED = (
    "vt_attn_fwd",
    "vt_attn_fwd_noalloc",
    "vt_attn_validate_seqlens_host",
    "vt_attn_smem_bytes",
    "vt_attn_workspace_bytes",
    "vt_attn_last_device_status",
    "vt_attn_selftest_wait_timeout",
    "vt_window_count",
    "vt_window_partition",
    "vt_permute_rows",
    "vt_permute_rows_check",
    "vt_rope2d",
    "vt_attn_fwd_rope2d",
    "vt_attn_fwd_swa",
    "vt_attn_set_split_keys",
    "vt_attn_status_string",
    "vt_attn_version",
)


class VtAttnError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {status_string(status)}")


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(
            f"libvtattn.so not found at {LIB_PATH}; build it with "
            "`python flash_attention_varlen_b200/build.py` (nvcc, sm_100a). "
            "There is no CPU fallback.")
    lib = ctypes.CDLL(LIB_PATH)
    P, I32, F = ctypes.c_void_p, ctypes.c_int32, ctypes.c_float
    lib.vt_attn_fwd.argtypes = [P, P, P, P, P, I32, I32, I32, I32, F, ctypes.c_int, P]
    lib.vt_attn_fwd.restype = ctypes.c_int
    lib.vt_attn_fwd_noalloc.argtypes = lib.vt_attn_fwd.argtypes
    lib.vt_attn_fwd_noalloc.restype = ctypes.c_int
    lib.vt_attn_validate_seqlens_host.argtypes = [P, I32, I32]
    lib.vt_attn_validate_seqlens_host.restype = ctypes.c_int
    lib.vt_attn_smem_bytes.argtypes = [I32, ctypes.c_int]
    lib.vt_attn_smem_bytes.restype = ctypes.c_size_t
    lib.vt_attn_workspace_bytes.argtypes = [I32, I32, ctypes.c_int]
    lib.vt_attn_workspace_bytes.restype = ctypes.c_size_t
    lib.vt_attn_last_device_status.argtypes = [P]
    lib.vt_attn_last_device_status.restype = ctypes.c_int
    lib.vt_attn_selftest_wait_timeout.argtypes = [P, P, P, P, P, I32, I32, I32, I32, F, I32, P]
    lib.vt_attn_selftest_wait_timeout.restype = ctypes.c_int
    lib.vt_window_count.argtypes = [P, I32, I32, P, P]
    lib.vt_window_count.restype = ctypes.c_int
    lib.vt_window_partition.argtypes = [P, I32, I32, P, P, P]
    lib.vt_window_partition.restype = ctypes.c_int
    lib.vt_permute_rows.argtypes = [P, P, P, I32, I32, I32, P]
    lib.vt_permute_rows.restype = ctypes.c_int
    lib.vt_attn_fwd_rope2d.argtypes = [P, P, P, P, P, I32, I32, I32, I32, F, P, F, P, P]
    lib.vt_attn_fwd_rope2d.restype = ctypes.c_int
    lib.vt_attn_fwd_swa.argtypes = [P, P, P, P, P, I32, I32, I32, I32, I32, F, I32, P]
    lib.vt_attn_fwd_swa.restype = ctypes.c_int
    lib.vt_rope2d.argtypes = [P, P, P, I32, I32, I32, F, P]
    lib.vt_rope2d.restype = ctypes.c_int
    lib.vt_permute_rows_check.argtypes = [P]
    lib.vt_permute_rows_check.restype = ctypes.c_int
    lib.vt_attn_status_string.argtypes = [ctypes.c_int]
    lib.vt_attn_status_string.restype = ctypes.c_char_p
    lib.vt_attn_version.argtypes = []
    lib.vt_attn_version.restype = I32
    lib.vt_attn_set_split_keys.argtypes = [I32]
    lib.vt_attn_set_split_keys.restype = I32
    return lib


lib = _load()


def vt_attn_fwd(q: int, k: int, v: int, out: int, cu_seqlens: int, num_segments: int,
                total_tokens: int, H: int, D: int, scale: float, dtype: int, stream: int) -> int:
    """Raw entry point: device pointers as ints; returns the vt_status code."""
    return lib.vt_attn_fwd(q, k, v, out, cu_seqlens, num_segments, total_tokens, H, D,
                           ctypes.c_float(scale), dtype, stream)


def vt_attn_fwd_noalloc(q: int, k: int, v: int, out: int, cu_seqlens: int, num_segments: int,
                        total_tokens: int, H: int, D: int, scale: float, dtype: int,
                        stream: int) -> int:
    """vt_attn_fwd for callers that cannot let the library allocate device memory
    (fixed 1 MiB work-list array; see include/vt_attn.h for limits and sharing rules)."""
    return lib.vt_attn_fwd_noalloc(q, k, v, out, cu_seqlens, num_segments, total_tokens, H, D,
                                   ctypes.c_float(scale), dtype, stream)


def vt_attn_validate_seqlens_host(cu_seqlens_host: int, num_segments: int, total_tokens: int) -> int:
    return lib.vt_attn_validate_seqlens_host(cu_seqlens_host, num_segments, total_tokens)


def vt_attn_smem_bytes(D: int, dtype: int) -> int:
    return lib.vt_attn_smem_bytes(D, dtype)


def vt_attn_workspace_bytes(num_segments: int, total_tokens: int, dtype: int) -> int:
    return lib.vt_attn_workspace_bytes(num_segments, total_tokens, dtype)


def vt_attn_last_device_status(stream: int) -> int:
    return lib.vt_attn_last_device_status(stream)


def vt_attn_selftest_wait_timeout(q: int, k: int, v: int, out: int, cu_seqlens: int,
                                  num_segments: int, total_tokens: int, H: int, D: int,
                                  scale: float, stall_cycles: int, stream: int) -> int:
    """Failure-path self-test (bf16): the kernel's MMA thread waits on a barrier nothing
    arrives on for stall_cycles cycles, then every role aborts; the device status of the
    stream then reads VT_ERR_DEVICE_TIMEOUT.  Returns the launch status."""
    return lib.vt_attn_selftest_wait_timeout(q, k, v, out, cu_seqlens, num_segments,
                                             total_tokens, H, D, ctypes.c_float(scale),
                                             stall_cycles, stream)


def vt_window_count(grids_host: int, n_images: int, win: int, num_windows: int,
                    total_tokens: int) -> int:
    """Pure host: block and token counts of packed image grids (pointers as ints)."""
    return lib.vt_window_count(grids_host, n_images, win, num_windows, total_tokens)


def vt_window_partition(grids_host: int, n_images: int, win: int, perm: int, cu_seqlens: int,
                        stream: int) -> int:
    """Device window order of packed image grids: perm [T] and the blocks' cu_seqlens."""
    return lib.vt_window_partition(grids_host, n_images, win, perm, cu_seqlens, stream)


def vt_permute_rows(src: int, dst: int, index: int, num_rows: int, row_bytes: int, scatter: int,
                    stream: int) -> int:
    """dst[i] = src[index[i]] (scatter=0) or dst[index[i]] = src[i] (scatter=1), on the device."""
    return lib.vt_permute_rows(src, dst, index, num_rows, row_bytes, scatter, stream)


def vt_rope2d(x: int, out: int, pos: int, total_tokens: int, H: int, D: int, theta: float,
              stream: int) -> int:
    """out = 2D RoPE of x (bf16 [T, H, 96]; out may be x), pos int32 [T][2] 1-based (pw, ph)."""
    return lib.vt_rope2d(x, out, pos, total_tokens, H, D, ctypes.c_float(theta), stream)


def vt_attn_fwd_rope2d(q: int, k: int, v: int, out: int, cu_seqlens: int, num_segments: int,
                       total_tokens: int, H: int, D: int, scale: float, pos: int, theta: float,
                       k_rot: int, stream: int) -> int:
    """Attention over rope(Q), rope(K) (bf16): Q rotated in the kernel, K into k_rot."""
    return lib.vt_attn_fwd_rope2d(q, k, v, out, cu_seqlens, num_segments, total_tokens, H, D,
                                  ctypes.c_float(scale), pos, ctypes.c_float(theta), k_rot, stream)


def vt_attn_fwd_swa(q: int, k: int, v: int, out: int, cu_seqlens: int, num_segments: int,
                    total_tokens: int, Hq: int, Hkv: int, D: int, scale: float, window: int,
                    stream: int) -> int:
    """Causal attention with a local window (0: none) and grouped-query heads (bf16, D 128)."""
    return lib.vt_attn_fwd_swa(q, k, v, out, cu_seqlens, num_segments, total_tokens, Hq, Hkv, D,
                               ctypes.c_float(scale), window, stream)


def vt_permute_rows_check(stream: int) -> int:
    """Synchronise `stream`; VT_ERR_BAD_INDEX if a permute on this device skipped an
    out-of-range row index since the previous check (the flag is then cleared)."""
    return lib.vt_permute_rows_check(stream)


def status_string(status: int) -> str:
    return lib.vt_attn_status_string(status).decode()


def vt_attn_version() -> int:
    return lib.vt_attn_version()


def vt_attn_set_split_keys(enable: int) -> int:
    return lib.vt_attn_set_split_keys(1 if enable else 0)

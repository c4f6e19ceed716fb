"""Seeded synthetic workloads shared by the CUDA path's tests/bench and the CPU oracle.

Nothing here computes attention.  This module only

* draws Q, K, V ~ N(0, 1) from a documented counter-based generator
  (``gen.c``: SplitMix64 -> Box-Muller in double -> f32 -> optional bf16 RNE),
* builds the packed-segment structure (``cu_seqlens``) of the image-shaped
  workloads the pages describe, and
* counts the algorithmic work (FLOPs = 4 * sum(L^2) * H * D) used by the
  measurement code.

Workload shapes follow the pages: a ViT-G/14 perception encoder with 16 heads of
width 96 (issue #1545 "Why this one is bad": H=16, head_dim=96), 448x448 and
896x896 images at patch 14 (1024 and 4096 patch tokens), 32x32-patch windows
(issue #1545 follow-up: pos_emb_height = pos_emb_width = 32) and a 50-layer
schedule whose full-attention layers sit at indices 3, 7, 11, ..., 47, 49, the
other 37 being window layers (issue #1545 follow-up comment, the section on the
resolved labelled uncertainties: the split is read from the shipped configuration).
The 128x128-patch grid is the issue's
"reading A" (16384 patch tokens, 16 windows).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from dataclasses import dataclass, field

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_LIB_PATH = os.path.join(_HERE, "libvtgen.so")
_lib = None

# stream ids of the generator
STREAM_Q, STREAM_K, STREAM_V, STREAM_SIZES = 0, 1, 2, 3

HEADS = 16
HEAD_DIM = 96
WINDOW = 32          # window side in patches (32 x 32 = 1024 tokens)
N_LAYERS = 50


def build(force: bool = False) -> str:
    """Compile gen.c into libvtgen.so next to this file (plain gcc, no GPU)."""
    src = os.path.join(_HERE, "gen.c")
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(src):
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-shared", "-fPIC", "-pthread", src, "-o", tmp, "-lm"])
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    if _lib is None:
        if not os.path.exists(_LIB_PATH):
            build()
        lib = ctypes.CDLL(_LIB_PATH)
        lib.vtgen_normal_f32.argtypes = [ctypes.c_uint64, ctypes.c_uint64, ctypes.c_int64,
                                         ctypes.c_int64, ctypes.c_void_p, ctypes.c_int]
        lib.vtgen_normal_bf16.argtypes = lib.vtgen_normal_f32.argtypes
        lib.vtgen_uniform_int.argtypes = [ctypes.c_uint64, ctypes.c_uint64, ctypes.c_int64,
                                          ctypes.c_int32, ctypes.c_int32, ctypes.c_void_p]
        lib.vtgen_raw.argtypes = [ctypes.c_uint64, ctypes.c_uint64, ctypes.c_int64, ctypes.c_void_p]
        _lib = lib
    return _lib


def _threads() -> int:
    return max(1, min(64, os.cpu_count() or 1))


def normal(seed: int, stream: int, count: int, dtype: str, offset: int = 0, out=None) -> np.ndarray:
    """Elements [offset, offset+count) of the N(0,1) stream (seed, stream).

    dtype "f32" returns float32; dtype "bf16" returns the raw bf16 bit patterns
    as uint16 (the f32 draw rounded to nearest-even).  ``out`` may be a
    preallocated C-contiguous array (e.g. a view of pinned host memory).
    """
    lib = _load()
    if dtype == "f32":
        arr = np.empty(count, np.float32) if out is None else out
        assert arr.dtype == np.float32 and arr.size == count and arr.flags.c_contiguous
        lib.vtgen_normal_f32(seed, stream, offset, count, arr.ctypes.data, _threads())
    elif dtype == "bf16":
        arr = np.empty(count, np.uint16) if out is None else out
        assert arr.dtype == np.uint16 and arr.size == count and arr.flags.c_contiguous
        lib.vtgen_normal_bf16(seed, stream, offset, count, arr.ctypes.data, _threads())
    else:
        raise ValueError(f"unknown dtype {dtype!r}")
    return arr


def raw_draws(seed: int, stream: int, count: int) -> np.ndarray:
    lib = _load()
    arr = np.empty(count, np.uint64)
    lib.vtgen_raw(seed, stream, count, arr.ctypes.data)
    return arr


def uniform_int(seed: int, stream: int, count: int, lo: int, hi: int) -> np.ndarray:
    lib = _load()
    arr = np.empty(count, np.int32)
    lib.vtgen_uniform_int(seed, stream, count, lo, hi, arr.ctypes.data)
    return arr


def qkv(seed: int, T: int, H: int = HEADS, D: int = HEAD_DIM, dtype: str = "bf16", outs=None):
    """Q, K, V as [T, H, D] arrays drawn from streams 0, 1, 2 of ``seed``."""
    n = T * H * D
    res = []
    for i, stream in enumerate((STREAM_Q, STREAM_K, STREAM_V)):
        o = None if outs is None else outs[i].reshape(-1)
        res.append(normal(seed, stream, n, dtype, out=o).reshape(T, H, D))
    return tuple(res)


def bf16_bits_to_f32(u16: np.ndarray) -> np.ndarray:
    """Exact widening of raw bf16 bit patterns to float32."""
    return (u16.astype(np.uint32) << 16).view(np.float32)


def cu_from_lengths(lengths) -> np.ndarray:
    cu = np.zeros(len(lengths) + 1, np.int32)
    cu[1:] = np.cumsum(np.asarray(lengths, np.int64))
    return cu


def window_lengths(grid_h: int, grid_w: int, win: int = WINDOW) -> list[int]:
    """Token count of each win x win window of a grid_h x grid_w patch grid.

    Windows are walked row-major over the window grid; a grid that is not a
    multiple of ``win`` gets smaller edge windows.  Tokens are assumed already
    permuted so that each window is contiguous (the synthetic Q/K/V are drawn in
    that order directly).
    """
    out = []
    for by in range(0, grid_h, win):
        for bx in range(0, grid_w, win):
            out.append(min(win, grid_h - by) * min(win, grid_w - bx))
    return out


def is_full_layer(layer: int) -> bool:
    """Full-attention layers: 3, 7, 11, ..., 47 and the last layer 49."""
    return layer % 4 == 3 or layer == N_LAYERS - 1


def varlen_image_grids(seed: int = 0, n_images: int = 8, lo: int = 8, hi: int = 64):
    """Patch-grid (h, w) of each image, drawn h then w per image from the sizes stream."""
    d = uniform_int(seed, STREAM_SIZES, 2 * n_images, lo, hi)
    return [(int(d[2 * i]), int(d[2 * i + 1])) for i in range(n_images)]


def flops(cu_seqlens, H: int = HEADS, D: int = HEAD_DIM) -> int:
    """Algorithmic FLOPs of one block-diagonal attention forward: 4 * sum(L^2) * H * D."""
    cu = np.asarray(cu_seqlens, np.int64)
    L = cu[1:] - cu[:-1]
    return int(4 * int((L * L).sum()) * H * D)


def patch_positions(grid_h: int, grid_w: int) -> np.ndarray:
    """int32 [grid_h * grid_w, 2]: each patch's 1-based (column + 1, row + 1) in row-major
    patch order, the positions a 2D RoPE input carries."""
    ys, xs = np.meshgrid(np.arange(grid_h), np.arange(grid_w), indexing="ij")
    return np.stack([xs.ravel() + 1, ys.ravel() + 1], axis=1).astype(np.int32)


# Text decoder attention (the Muse Glimmer next-steps document, "Architecture / Text
# decoder"): 32 query heads over 2 key/value heads, head size 128, local window 2048.
DECODER_HQ, DECODER_HKV, DECODER_D, DECODER_WINDOW = 32, 2, 128, 2048


def decoder_qkv(seed: int, T: int, Hq: int = DECODER_HQ, Hkv: int = DECODER_HKV,
                D: int = DECODER_D, dtype: str = "bf16"):
    """Q [T, Hq, D], K and V [T, Hkv, D] from streams 0, 1, 2 of ``seed``."""
    q = normal(seed, STREAM_Q, T * Hq * D, dtype).reshape(T, Hq, D)
    k = normal(seed, STREAM_K, T * Hkv * D, dtype).reshape(T, Hkv, D)
    v = normal(seed, STREAM_V, T * Hkv * D, dtype).reshape(T, Hkv, D)
    return q, k, v


def decoder_pairs(cu_seqlens, window: int) -> int:
    """(query, key) pairs of causal attention with a local window (0: none), per head: query
    n (1-based within its segment) sees min(n, window) keys."""
    cu = np.asarray(cu_seqlens, np.int64)
    total = 0
    for L in (cu[1:] - cu[:-1]).tolist():
        if window <= 0 or window >= L:
            total += L * (L + 1) // 2
        else:
            total += window * (window + 1) // 2 + (L - window) * window
    return int(total)


def decoder_flops(cu_seqlens, window: int, Hq: int = DECODER_HQ, D: int = DECODER_D) -> int:
    """Algorithmic FLOPs of the decoder attention forward: 4 * pairs * Hq * D."""
    return 4 * decoder_pairs(cu_seqlens, window) * Hq * D


def exp_count(cu_seqlens, H: int = HEADS) -> int:
    """Softmax exponentials of one forward: sum(L^2) * H (one per score)."""
    cu = np.asarray(cu_seqlens, np.int64)
    L = cu[1:] - cu[:-1]
    return int((L * L).sum()) * H


@dataclass
class Case:
    """One attention call: the packed segment structure plus how to draw its inputs."""
    name: str
    cu_seqlens: np.ndarray
    seed: int = 0
    dtype: str = "bf16"
    q_scale: float = 1.0          # peaked variant multiplies Q by 4 (exact in bf16/f32)
    H: int = HEADS
    D: int = HEAD_DIM
    meta: dict = field(default_factory=dict)

    @property
    def T(self) -> int:
        return int(self.cu_seqlens[-1])

    @property
    def num_segments(self) -> int:
        return len(self.cu_seqlens) - 1

    def inputs(self):
        q, k, v = qkv(self.seed, self.T, self.H, self.D, self.dtype)
        if self.q_scale != 1.0:
            if self.dtype == "bf16":
                qf = bf16_bits_to_f32(q) * np.float32(self.q_scale)
                q = (qf.view(np.uint32) >> 16).astype(np.uint16)   # exact: power-of-two scale
            else:
                q = q * np.float32(self.q_scale)
        return q, k, v

    def flops(self) -> int:
        return flops(self.cu_seqlens, self.H, self.D)


def tiny_case(dtype: str = "bf16") -> Case:
    """One 16x16-patch image: a single 256-token segment, seed 0."""
    return Case(f"tiny256_{dtype}", cu_from_lengths([256]), 0, dtype)


def image448_case(peaked: bool = False) -> Case:
    """One 448x448 image at patch 14: 1024 tokens, one full-attention segment."""
    return Case("img448_peaked" if peaked else "img448", cu_from_lengths([1024]), 0, "bf16",
                4.0 if peaked else 1.0)


def image896_cases():
    """One 896x896 image (64x64 patches): a window layer (4 x 1024) and a full layer (4096)."""
    return (Case("img896_window", cu_from_lengths(window_lengths(64, 64)), 0),
            Case("img896_full", cu_from_lengths([4096]), 0))


def varlen8_case(seed: int = 0) -> Case:
    """Eight rectangular images, h and w uniform on 8..64, full attention per image."""
    grids = varlen_image_grids(seed)
    c = Case("varlen8", cu_from_lengths([h * w for h, w in grids]), seed)
    c.meta["grids"] = grids
    return c


def tower_layer_case(layer: int, grid: int = 128, base_seed: int = 0) -> Case:
    """Layer ``layer`` of the 50-layer tower at a grid x grid patch image (default 16384 tokens)."""
    full = is_full_layer(layer)
    lengths = [grid * grid] if full else window_lengths(grid, grid)
    return Case(f"tower{grid * grid}_L{layer}_{'full' if full else 'window'}",
                cu_from_lengths(lengths), base_seed + layer, "bf16",
                meta={"layer": layer, "full": full})


def tower_cases(grid: int = 128, base_seed: int = 0):
    return [tower_layer_case(l, grid, base_seed) for l in range(N_LAYERS)]

"""2D rotary position embedding of the vision tower, and attention over rotated Q/K --
TEST INFRASTRUCTURE ONLY.

Only ``tests/`` (and ``bench.py``'s CPU legs) may import this; the CUDA library never
does, and the two share no code.

The tower rotates Q and K by a two-dimensional RoPE before every attention (PR #279,
vision-tower port commit: the port names the width-first 2D RoPE order and the 1-based
RoPE positions among the places a port goes wrong, and permutes the RoPE table together
with the hidden states into window order).  The pages print neither formula; the plain
reading taken here, for head width D (a multiple of 4) and base theta:

  * each token has a 1-based position pair (pw, ph) = (x + 1, y + 1) in its image's
    patch grid, carried along with the token (so window order keeps it);
  * F = D / 4 frequencies f_i = theta^(-2 i / (D / 2)), i = 0 .. F - 1;
  * the D / 2 angles of a token are [pw f_0 .. pw f_{F-1}, ph f_0 .. ph f_{F-1}]:
    width first;
  * element d < D / 2 pairs with d + D / 2 and the pair turns by angle a_d:
      out[d]       = x[d] cos a_d - x[d + D/2] sin a_d
      out[d + D/2] = x[d + D/2] cos a_d + x[d] sin a_d.

Everything is evaluated in f64 from the inputs widened exactly.
"""
from __future__ import annotations

import numpy as np

from . import attn_fwd, attn_rows

DEFAULT_THETA = 10000.0


def _to_f64(a):
    a = np.asarray(a)
    if a.dtype == np.uint16:  # bf16 bits
        return (a.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    return a.astype(np.float64)


def rope_frequencies(D: int, theta: float = DEFAULT_THETA) -> np.ndarray:
    """The F = D / 4 frequencies theta^(-2 i / (D / 2)), as a plain loop."""
    assert D % 4 == 0
    F = D // 4
    return np.array([theta ** (-2.0 * i / (D // 2)) for i in range(F)], np.float64)


def rope_angles(pos, D: int, theta: float = DEFAULT_THETA) -> np.ndarray:
    """[T, D / 2] angles: width position times the frequencies, then height position."""
    pos = np.asarray(pos, np.float64)
    f = rope_frequencies(D, theta)
    return np.concatenate([pos[:, 0:1] * f[None, :], pos[:, 1:2] * f[None, :]], axis=1)


def rope2d(x, pos, theta: float = DEFAULT_THETA) -> np.ndarray:
    """Rotate x ([T, H, D], bf16 bits / f32 / f64) by the 2D RoPE of pos ([T, 2] int:
    (pw, ph), 1-based).  Returns f64 [T, H, D]."""
    x = _to_f64(x)
    T, H, D = x.shape
    half = D // 2
    a = rope_angles(pos, D, theta)            # [T, D/2]
    c, s = np.cos(a)[:, None, :], np.sin(a)[:, None, :]
    x1, x2 = x[..., :half], x[..., half:]
    return np.concatenate([x1 * c - x2 * s, x2 * c + x1 * s], axis=-1)


def attn_fwd_rope2d(q, k, v, cu_seqlens, scale: float, pos, theta: float = DEFAULT_THETA,
                    threads=None) -> np.ndarray:
    """O = attention(rope(Q), rope(K), V) over the packed segments, all in f64."""
    return attn_fwd(rope2d(q, pos, theta), rope2d(k, pos, theta), _to_f64(v), cu_seqlens, scale,
                    threads=threads)


def attn_rows_rope2d(q, k, v, cu_seqlens, scale: float, pos, tokens, heads,
                     theta: float = DEFAULT_THETA, threads=None) -> np.ndarray:
    """Rows O[tokens[r], heads[r], :] of attention(rope(Q), rope(K), V), in f64."""
    return attn_rows(rope2d(q, pos, theta), rope2d(k, pos, theta), _to_f64(v), cu_seqlens, scale,
                     tokens, heads, threads=threads)


def image_positions(grids) -> np.ndarray:
    """1-based (pw, ph) of every token of packed images in row-major patch order."""
    out = []
    for h, w in grids:
        ys, xs = np.meshgrid(np.arange(h), np.arange(w), indexing="ij")
        out.append(np.stack([xs.ravel() + 1, ys.ravel() + 1], axis=1))
    return np.concatenate(out).astype(np.int32)


__all__ = ["DEFAULT_THETA", "rope_frequencies", "rope_angles", "rope2d", "attn_fwd_rope2d",
           "attn_rows_rope2d", "image_positions"]

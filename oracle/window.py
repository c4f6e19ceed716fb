"""Window segmentation of patch grids -- TEST INFRASTRUCTURE ONLY.

Only ``tests/`` (and ``bench.py``'s CPU legs) may import this; the CUDA library never
does, and the two share no code.

The vision tower's window layers attend within windows of 32 x 32 = 1024 patches of each
image's patch grid (issue #1545 (vllm.cpp), follow-up comment, the section on the
resolved labelled uncertainties: the positional-embedding grid is 32 x 32, and the
tower's sparse permutation segments the patch grid on it).  The pages name the permutation's two orders, the walk over the blocks
and the order of the tokens inside a block, as places a port goes wrong (PR #279, vision
tower port commit), but print neither.  The plainest reading is taken here:
  * images are packed one after another, each in row-major (y, x) patch order;
  * an image's win x win blocks are walked row-major over the block grid; a grid that is
    not a multiple of win has smaller blocks along its bottom and right edges;
  * the tokens of a block are taken row-major inside it.
``perm[p]`` is the packed image-order token at position ``p`` of the window-ordered
sequence, and ``cu_seqlens`` delimits the blocks in that sequence.

Pinned by ``tests/test_window_oracle.py``: perm is a bijection, every block is a contiguous
rectangle of its image, blocks and the tokens inside them come in increasing image order,
closed-form block sizes of a ragged grid, and planted mistakes fail.
"""
from __future__ import annotations

import numpy as np


def window_permutation(grids, win: int = 32):
    """(perm int32 [T], cu_seqlens int32 [num_windows + 1]) for images of patch grids (h, w)."""
    perm, lengths = [], []
    base = 0
    for h, w in grids:
        for by in range(0, h, win):
            for bx in range(0, w, win):
                n = 0
                for y in range(by, min(by + win, h)):
                    for x in range(bx, min(bx + win, w)):
                        perm.append(base + y * w + x)
                        n += 1
                lengths.append(n)
        base += h * w
    cu = np.zeros(len(lengths) + 1, np.int32)
    cu[1:] = np.cumsum(np.asarray(lengths, np.int64))
    return np.asarray(perm, np.int32), cu


def window_attention(q, k, v, grids, scale: float, win: int = 32, threads=None):
    """Window-layer attention on image-order [T, H, D] inputs: each token attends to the
    tokens of its own block.  The oracle's definition (oracle.attn_fwd) is applied to the
    window-ordered sequence and the result is put back in image order."""
    from . import attn_fwd
    perm, cu = window_permutation(grids, win)
    out_w = attn_fwd(q[perm], k[perm], v[perm], cu, scale, threads=threads)
    out = np.empty_like(out_w)
    out[perm] = out_w
    return out

"""Causal, locally windowed, grouped-query attention of the text decoder -- TEST
INFRASTRUCTURE ONLY.

Only ``tests/`` (and ``bench.py``'s CPU legs) may import this; the CUDA library never does,
and the two share no code.

The Muse Glimmer next-steps document ("Support for Muse Glimmer 30B", section
"Architecture / Text decoder") gives the decoder's attention: 32 query heads, 2 key/value
heads, head size 128, a repeating [sliding, sliding, sliding, full] pattern and a local
attention window of 2048 tokens.  It prints no formula; the plain reading taken here:

  * segments (sequences) are packed by cu_seqlens, as for the vision tower, and attention
    never crosses a segment;
  * causal: query i of a segment attends key j of the same segment only if j <= i;
  * a sliding layer with window W attends only the last W positions, the query's own
    included: j > i - W (W = 0 means no window: a full-attention layer);
  * grouped-query attention: Hq query heads share Hkv key/value heads, query head h using
    key/value head h // (Hq / Hkv);
  * O[i,h,:] = sum_j softmax_j(scale * <Q[i,h,:], K[j,g,:]>) V[j,g,:] over the allowed j.

RoPE, the Q/K normalisation, the query multiplier and the output gate happen outside the
attention product; the multiplier reaches it through ``scale``.  Everything is evaluated in
f64 from the inputs widened exactly; each query row is computed from its own allowed keys
only (two-pass softmax), so any row can be computed alone.
"""
from __future__ import annotations

import numpy as np


def _to_f64(a):
    a = np.asarray(a)
    if a.dtype == np.uint16:  # bf16 bit patterns
        return (a.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    return a.astype(np.float64)


def allowed_keys(i: int, seg_start: int, window: int) -> range:
    """Keys of query i (absolute token index) in a segment starting at seg_start."""
    lo = seg_start if window <= 0 else max(seg_start, i - window + 1)
    return range(lo, i + 1)


def attn_row(q, k, v, i: int, h: int, seg_start: int, scale: float, window: int) -> np.ndarray:
    """One output row O[i, h, :] by the definition above."""
    Hq, Hkv = q.shape[1], k.shape[1]
    g = h // (Hq // Hkv)
    keys = allowed_keys(i, seg_start, window)
    qi = _to_f64(q[i, h])
    kk = _to_f64(k[keys.start:keys.stop, g])
    vv = _to_f64(v[keys.start:keys.stop, g])
    a = scale * (kk @ qi)
    w = np.exp(a - a.max())
    return (w[:, None] * vv).sum(axis=0) / w.sum()


def segment_of(cu_seqlens, i: int) -> int:
    cu = np.asarray(cu_seqlens)
    return int(np.searchsorted(cu, i, side="right") - 1)


def attn_rows(q, k, v, cu_seqlens, scale: float, window: int, tokens, heads) -> np.ndarray:
    """Output rows (tokens[n], heads[n]) -> [n, D]."""
    cu = np.asarray(cu_seqlens)
    out = np.empty((len(tokens), q.shape[2]), np.float64)
    for n, (i, h) in enumerate(zip(tokens, heads)):
        s = segment_of(cu, int(i))
        out[n] = attn_row(q, k, v, int(i), int(h), int(cu[s]), scale, window)
    return out


def attn_fwd(q, k, v, cu_seqlens, scale: float, window: int) -> np.ndarray:
    """Every output row [T, Hq, D], one segment and head at a time (masked score matrix)."""
    cu = np.asarray(cu_seqlens)
    T, Hq, D = q.shape
    Hkv = k.shape[1]
    group = Hq // Hkv
    out = np.zeros((T, Hq, D), np.float64)
    for s in range(len(cu) - 1):
        a0, a1 = int(cu[s]), int(cu[s + 1])
        L = a1 - a0
        if L == 0:
            continue
        i = np.arange(L)[:, None]
        j = np.arange(L)[None, :]
        allowed = j <= i
        if window > 0:
            allowed &= j > i - window
        for h in range(Hq):
            g = h // group
            qs = _to_f64(q[a0:a1, h])
            ks = _to_f64(k[a0:a1, g])
            vs = _to_f64(v[a0:a1, g])
            a = np.where(allowed, scale * (qs @ ks.T), -np.inf)
            w = np.exp(a - a.max(axis=1, keepdims=True))
            out[a0:a1, h] = (w @ vs) / w.sum(axis=1, keepdims=True)
    return out

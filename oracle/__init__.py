"""CPU oracle for varlen block-diagonal attention -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline /
reference leg may import this package.  The product path (the CUDA library and
its Python binding) never imports it, and the two share no code.

The arithmetic lives in ``attn_oracle.c`` (plain C, f64, two-pass softmax,
threaded over (segment, head)); this module only compiles it and marshals
numpy arrays.  Its definition:

    O[i,h,:] = sum_j exp(a_ij - m_i) V[j,h,:] / sum_j exp(a_ij - m_i),
    a_ij = scale * <Q[i,h,:], K[j,h,:]>,  j over the segment of i,

from issue #1545 (vllm.cpp) "Why this one is bad" / "The fix" and PR #1579
"Numerics, both halves".  Every function here is pinned by the tests in
``tests/test_oracle_pins.py`` (high-precision brute force, closed forms and
invariants); none is "parity unpinned".
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
_lib = None

_DT = {"bf16": 0, "f32": 1, "f64": 2}


def build(force: bool = False, extra_flags=(), out_path: str | None = None) -> str:
    """Compile attn_oracle.c with gcc.  ``extra_flags``/``out_path`` serve the mutation tests."""
    src = os.path.join(_HERE, "attn_oracle.c")
    path = out_path or _LIB_PATH
    if force or out_path or not os.path.exists(path) or os.path.getmtime(path) < os.path.getmtime(src):
        tmp = path + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-shared", "-fPIC", "-pthread", *extra_flags, src,
                               "-o", tmp, "-lm"])
        os.replace(tmp, path)
    return path


def _bind(lib):
    P, I32, D = ctypes.c_void_p, ctypes.c_int32, ctypes.c_double
    lib.oracle_check_seqlens.argtypes = [P, I32, I32]
    lib.oracle_attn_fwd.argtypes = [P, P, P, ctypes.c_int, P, P, I32, I32, I32, I32, D, ctypes.c_int]
    lib.oracle_attn_rows.argtypes = [P, P, P, ctypes.c_int, P, P, I32, P, P, I32, I32, I32, I32, D,
                                     ctypes.c_int]
    lib.oracle_attn_probs.argtypes = [P, P, ctypes.c_int, P, I32, I32, I32, I32, D, I32, I32, P]
    return lib


def load(path: str | None = None):
    """Load the oracle library (building it if needed).  ``path`` loads another build."""
    global _lib
    if path is not None:
        return _bind(ctypes.CDLL(path))
    if _lib is None:
        if not os.path.exists(_LIB_PATH):
            build()
        _lib = _bind(ctypes.CDLL(_LIB_PATH))
    return _lib


def default_threads() -> int:
    try:
        return len(os.sched_getaffinity(0))
    except Exception:  # pragma: no cover
        return os.cpu_count() or 1


def _dtype_of(a: np.ndarray) -> str:
    if a.dtype == np.uint16:
        return "bf16"
    if a.dtype == np.float32:
        return "f32"
    if a.dtype == np.float64:
        return "f64"
    raise TypeError(f"unsupported oracle input dtype {a.dtype}")


def _prep(q, k, v, cu):
    q, k = np.ascontiguousarray(q), np.ascontiguousarray(k)
    v = None if v is None else np.ascontiguousarray(v)
    dt = _dtype_of(q)
    assert _dtype_of(k) == dt and (v is None or _dtype_of(v) == dt)
    cu = np.ascontiguousarray(cu, dtype=np.int32)
    T, H, D = q.shape
    return q, k, v, dt, cu, T, H, D


def attn_fwd(q, k, v, cu_seqlens, scale: float, threads: int | None = None, lib=None) -> np.ndarray:
    """O[T, H, D] in float64.  q/k/v: [T, H, D] as uint16 bf16 bits, float32 or float64."""
    q, k, v, dt, cu, T, H, D = _prep(q, k, v, cu_seqlens)
    out = np.zeros((T, H, D), np.float64)
    lib = lib or load()
    rc = lib.oracle_attn_fwd(q.ctypes.data, k.ctypes.data, v.ctypes.data, _DT[dt], out.ctypes.data,
                             cu.ctypes.data, len(cu) - 1, T, H, D, float(scale),
                             threads or default_threads())
    if rc != 0:
        raise ValueError(f"oracle_attn_fwd rejected its arguments (rc={rc})")
    return out


def attn_rows(q, k, v, cu_seqlens, scale: float, tokens, heads, threads: int | None = None,
              lib=None) -> np.ndarray:
    """Rows O[tokens[r], heads[r], :] as a [len(tokens), D] float64 array."""
    q, k, v, dt, cu, T, H, D = _prep(q, k, v, cu_seqlens)
    tok = np.ascontiguousarray(tokens, dtype=np.int32)
    hd = np.ascontiguousarray(heads, dtype=np.int32)
    assert tok.shape == hd.shape
    out = np.zeros((len(tok), D), np.float64)
    lib = lib or load()
    rc = lib.oracle_attn_rows(q.ctypes.data, k.ctypes.data, v.ctypes.data, _DT[dt], tok.ctypes.data,
                              hd.ctypes.data, len(tok), out.ctypes.data, cu.ctypes.data, len(cu) - 1,
                              T, H, D, float(scale), threads or default_threads())
    if rc != 0:
        raise ValueError(f"oracle_attn_rows rejected its arguments (rc={rc})")
    return out


def attn_probs(q, k, cu_seqlens, scale: float, segment: int, head: int, lib=None) -> np.ndarray:
    """Softmax probabilities [L, L] of one (segment, head)."""
    q, k, _, dt, cu, T, H, D = _prep(q, k, None, cu_seqlens)
    L = int(cu[segment + 1] - cu[segment])
    probs = np.zeros((L, L), np.float64)
    lib = lib or load()
    rc = lib.oracle_attn_probs(q.ctypes.data, k.ctypes.data, _DT[dt], cu.ctypes.data, len(cu) - 1,
                               T, H, D, float(scale), segment, head, probs.ctypes.data)
    if rc != 0:
        raise ValueError(f"oracle_attn_probs rejected its arguments (rc={rc})")
    return probs


def check_seqlens(cu_seqlens, total_tokens: int) -> bool:
    cu = np.ascontiguousarray(cu_seqlens, dtype=np.int32)
    return load().oracle_check_seqlens(cu.ctypes.data, len(cu) - 1, total_tokens) == 0

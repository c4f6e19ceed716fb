"""Pins for the CPU oracle: checks against things other than the oracle itself.

The pages print no attention outputs, so the oracle is pinned by
* a high-precision brute force on tiny inputs (Python ``decimal`` at 50
  digits, the full T x T score matrix with -inf off the block diagonal and a
  plain exp with no max subtraction -- a different algorithm from the oracle's
  two-pass per-segment softmax),
* closed forms (single key, two keys, identical keys, zero scale, a dominant key),
* invariants of softmax attention (row sums, block-diagonal independence,
  packing order, key/value permutation, key shift, affine values), and
* mutation checks: plausible mistakes planted in a copy of the oracle's source
  must each fail at least one pin.

The definition being pinned: issue #1545 (vllm.cpp) "Why this one is bad" and
"The fix"; PR #1579 "Numerics, both halves".
"""
import math
import os
import re
import struct
import tempfile
from decimal import Decimal, getcontext

import numpy as np
import pytest

import oracle

SEGS = [5, 0, 12, 1, 22, 8]          # includes an empty and a single-key segment
H_T, D_T = 2, 8


def _tiny_inputs(seed=1, lengths=SEGS, H=H_T, D=D_T, spread=0.7):
    rng = np.random.default_rng(seed)
    T = int(sum(lengths))
    q = rng.normal(0, spread, (T, H, D))
    k = rng.normal(0, spread, (T, H, D))
    v = rng.normal(0, 1.0, (T, H, D))
    cu = np.zeros(len(lengths) + 1, np.int32)
    cu[1:] = np.cumsum(lengths)
    return q, k, v, cu


def brute_force(q, k, v, cu, scale):
    """Decimal(50 digits): dense T x T masked scores, exp without max subtraction."""
    getcontext().prec = 50
    T, H, D = q.shape
    seg = np.zeros(T, np.int64)
    for s in range(len(cu) - 1):
        seg[cu[s]:cu[s + 1]] = s
    sc = Decimal(scale)
    out = np.zeros((T, H, D))
    for h in range(H):
        Kd = [[Decimal(float(k[j, h, e])) for e in range(D)] for j in range(T)]
        Vd = [[Decimal(float(v[j, h, d])) for d in range(D)] for j in range(T)]
        for i in range(T):
            qi = [Decimal(float(q[i, h, e])) for e in range(D)]
            num = [Decimal(0)] * D
            den = Decimal(0)
            for j in range(T):
                if seg[j] != seg[i]:
                    continue            # -inf score: exp(-inf) = 0
                w = (sc * sum(qi[e] * Kd[j][e] for e in range(D))).exp()
                den += w
                for d in range(D):
                    num[d] += w * Vd[j][d]
            for d in range(D):
                out[i, h, d] = float(num[d] / den)
    return out


def pin_bruteforce(lib):
    q, k, v, cu = _tiny_inputs()
    scale = 1.0 / math.sqrt(D_T)
    got = oracle.attn_fwd(q, k, v, cu, scale, threads=3, lib=lib)
    ref = brute_force(q, k, v, cu, scale)
    if not np.all(np.isfinite(got)):
        return float("inf")
    return float(np.max(np.abs(got - ref)))


def pin_dominant_key(lib):
    """One key's logit exceeds the others by ~1e3: O must equal that key's V exactly."""
    T, H, D = 6, 1, 4
    q = np.zeros((T, H, D))
    k = np.zeros((T, H, D))
    v = np.arange(T * H * D, dtype=np.float64).reshape(T, H, D) - 7.0
    q[:, 0, 0] = 40.0
    k[:, 0, 0] = np.array([1.0, 2.0, 30.0, 3.0, 0.5, 1.5])     # key 2 dominates by 27*40 = 1080
    cu = np.array([0, T], np.int32)
    got = oracle.attn_fwd(q, k, v, cu, 1.0, threads=1, lib=lib)
    want = np.broadcast_to(v[2], (T, H, D))
    if not np.all(np.isfinite(got)):
        return float("inf")
    return float(np.max(np.abs(got - want)))


def test_bruteforce_tiny():
    assert pin_bruteforce(oracle.load()) < 1e-14


def test_bruteforce_tiny_other_scale_and_spread():
    q, k, v, cu = _tiny_inputs(seed=7, lengths=[3, 17, 9], spread=1.6)
    got = oracle.attn_fwd(q, k, v, cu, 0.9, threads=2)
    ref = brute_force(q, k, v, cu, 0.9)
    assert np.max(np.abs(got - ref)) < 1e-13


def test_dominant_key_needs_max_subtraction():
    assert pin_dominant_key(oracle.load()) == 0.0


def test_probability_rows_sum_to_one():
    q, k, v, cu = _tiny_inputs(spread=2.0)
    for s in range(len(cu) - 1):
        if cu[s + 1] == cu[s]:
            continue
        for h in range(H_T):
            p = oracle.attn_probs(q, k, cu, 0.4, s, h)
            assert np.all(p >= 0)
            assert np.max(np.abs(p.sum(axis=1) - 1.0)) < 1e-14
            # O = P V for this block, checked with exact row sums
            o = oracle.attn_fwd(q, k, v, cu, 0.4)[cu[s]:cu[s + 1], h]
            vs = v[cu[s]:cu[s + 1], h]
            pv = np.array([[math.fsum(p[i, j] * vs[j, d] for j in range(len(vs)))
                            for d in range(D_T)] for i in range(len(vs))])
            assert np.max(np.abs(o - pv)) < 1e-13


def test_single_key_segment_returns_v_exactly():
    for dtype in ("f64", "f32", "bf16"):
        q, k, v, cu = _tiny_inputs(lengths=[1, 1, 3, 1])
        if dtype == "f32":
            q, k, v = (x.astype(np.float32) for x in (q, k, v))
        elif dtype == "bf16":
            q, k, v = (_to_bf16_bits(x) for x in (q, k, v))
        got = oracle.attn_fwd(q, k, v, cu, 0.3)
        vv = v if dtype != "bf16" else _bf16_bits_to_f64(v)
        for t in (0, 1, 5):
            assert np.array_equal(got[t], np.asarray(vv[t], np.float64))


def test_two_key_closed_form():
    rng = np.random.default_rng(3)
    q = rng.normal(size=(2, 1, 5))
    k = rng.normal(size=(2, 1, 5))
    v = rng.normal(size=(2, 1, 5))
    scale = 0.8
    got = oracle.attn_fwd(q, k, v, np.array([0, 2], np.int32), scale)
    for i in range(2):
        a1 = scale * math.fsum(q[i, 0] * k[0, 0])
        a2 = scale * math.fsum(q[i, 0] * k[1, 0])
        s1 = 1.0 / (1.0 + math.exp(a2 - a1))
        s2 = 1.0 / (1.0 + math.exp(a1 - a2))
        want = s1 * v[0, 0] + s2 * v[1, 0]
        assert np.max(np.abs(got[i, 0] - want)) < 1e-15


def test_identical_keys_give_mean_of_values():
    rng = np.random.default_rng(4)
    T, H, D = 9, 2, 6
    q = rng.normal(size=(T, H, D))
    k = np.broadcast_to(rng.normal(size=(1, H, D)), (T, H, D)).copy()
    v = rng.normal(size=(T, H, D))
    got = oracle.attn_fwd(q, k, v, np.array([0, T], np.int32), 0.5)
    for h in range(H):
        mean = np.array([math.fsum(v[:, h, d]) / T for d in range(D)])
        assert np.max(np.abs(got[:, h] - mean)) < 1e-15


def test_zero_scale_gives_mean_of_values():
    q, k, v, cu = _tiny_inputs()
    got = oracle.attn_fwd(q, k, v, cu, 0.0)
    for s in range(len(cu) - 1):
        a, b = cu[s], cu[s + 1]
        if a == b:
            continue
        for h in range(H_T):
            mean = np.array([math.fsum(v[a:b, h, d]) / (b - a) for d in range(D_T)])
            assert np.max(np.abs(got[a:b, h] - mean)) < 1e-15


def test_block_diagonal_independence_and_packing_order():
    q, k, v, cu = _tiny_inputs(spread=1.2)
    batch = oracle.attn_fwd(q, k, v, cu, 0.6)
    nseg = len(cu) - 1
    for s in range(nseg):
        a, b = cu[s], cu[s + 1]
        alone = oracle.attn_fwd(q[a:b], k[a:b], v[a:b], np.array([0, b - a], np.int32), 0.6)
        assert np.array_equal(alone, batch[a:b])
    order = [4, 0, 5, 2, 1, 3]
    qs = [q[cu[s]:cu[s + 1]] for s in order]
    ks = [k[cu[s]:cu[s + 1]] for s in order]
    vs = [v[cu[s]:cu[s + 1]] for s in order]
    lens = [cu[s + 1] - cu[s] for s in order]
    cu2 = np.zeros(nseg + 1, np.int32)
    cu2[1:] = np.cumsum(lens)
    perm = oracle.attn_fwd(np.concatenate(qs), np.concatenate(ks), np.concatenate(vs), cu2, 0.6)
    for pos, s in enumerate(order):
        assert np.array_equal(perm[cu2[pos]:cu2[pos + 1]], batch[cu[s]:cu[s + 1]])


def test_key_value_permutation_within_segment():
    q, k, v, cu = _tiny_inputs(spread=1.0)
    base = oracle.attn_fwd(q, k, v, cu, 0.5)
    rng = np.random.default_rng(9)
    k2, v2 = k.copy(), v.copy()
    for s in range(len(cu) - 1):
        a, b = cu[s], cu[s + 1]
        p = a + rng.permutation(b - a)
        k2[a:b], v2[a:b] = k[p], v[p]
    got = oracle.attn_fwd(q, k2, v2, cu, 0.5)
    assert np.max(np.abs(got - base)) < 1e-14


def test_shift_of_keys_is_invariant():
    q, k, v, cu = _tiny_inputs(spread=1.0)
    base = oracle.attn_fwd(q, k, v, cu, 0.5)
    k2 = k.copy()
    rng = np.random.default_rng(11)
    for s in range(len(cu) - 1):
        k2[cu[s]:cu[s + 1]] += rng.normal(size=(1, H_T, D_T)) * 3.0
    got = oracle.attn_fwd(q, k2, v, cu, 0.5)
    assert np.max(np.abs(got - base)) < 1e-12


def test_affine_values():
    q, k, v, cu = _tiny_inputs()
    base = oracle.attn_fwd(q, k, v, cu, 0.5)
    got = oracle.attn_fwd(q, k, 2.5 * v - 1.25, cu, 0.5)
    assert np.max(np.abs(got - (2.5 * base - 1.25))) < 1e-13


def test_rows_match_full_forward_bitwise():
    q, k, v, cu = _tiny_inputs()
    full = oracle.attn_fwd(q, k, v, cu, 0.5)
    toks = np.array([0, 4, 5, 16, 17, 30, 47], np.int32)
    heads = np.array([0, 1, 1, 0, 1, 0, 1], np.int32)
    rows = oracle.attn_rows(q, k, v, cu, 0.5, toks, heads, threads=2)
    assert np.array_equal(rows, full[toks, heads])


def test_widening_of_bf16_and_f32_is_exact():
    vals = np.array([1.5, -2.0, 0.15625, 3.0e-3, 1.0e4, -0.0], np.float64)
    bits = np.array([struct.unpack("<I", struct.pack("<f", x))[0] >> 16 for x in vals], np.uint16)
    # the chosen values are bf16-representable except 3e-3 and 1e4, whose bits truncate;
    # the oracle must read exactly the value the bits encode
    enc = np.array([struct.unpack("<f", struct.pack("<I", int(b) << 16))[0] for b in bits])
    q = np.zeros((6, 1, 1), np.uint16)
    k = np.zeros((6, 1, 1), np.uint16)
    v = bits.reshape(6, 1, 1)
    cu = np.arange(7, dtype=np.int32)          # six single-key segments: O = V exactly
    got = oracle.attn_fwd(q, k, v, cu, 1.0)
    assert np.array_equal(got.reshape(-1), enc)
    got32 = oracle.attn_fwd(q.astype(np.float32), k.astype(np.float32),
                            vals.astype(np.float32).reshape(6, 1, 1), cu, 1.0)
    assert np.array_equal(got32.reshape(-1), vals.astype(np.float32).astype(np.float64))


def test_empty_and_invalid_seqlens():
    z = np.zeros((0, 2, 4))
    assert oracle.attn_fwd(z, z, z, np.array([0], np.int32), 1.0).shape == (0, 2, 4)
    q, k, v, cu = _tiny_inputs()
    T = q.shape[0]
    for bad in ([1, T], [0, T - 1], [0, 10, 5, T]):
        with pytest.raises(ValueError):
            oracle.attn_fwd(q, k, v, np.array(bad, np.int32), 1.0)
    assert oracle.check_seqlens(cu, T)
    assert not oracle.check_seqlens(np.array([0, 3, 2, T], np.int32), T)


def _to_bf16_bits(x):
    f = np.asarray(x, np.float32)
    b = f.view(np.uint32).astype(np.uint64)
    b = (b + 0x7FFF + ((b >> 16) & 1)) >> 16
    return b.astype(np.uint16)


def _bf16_bits_to_f64(u):
    return (u.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


# ---- mutation checks: each planted mistake must fail a pin ------------------------------

MUTATIONS = {
    "dropped_scale": ("w[j - a] = P->scale * dot;", "w[j - a] = dot;"),
    "value_row_index": ("acc += w[j - a] * widen(P->v, P->dtype, ((size_t)j * H + h) * D + d);",
                        "acc += w[j - a] * widen(P->v, P->dtype, ((size_t)i * H + h) * D + d);"),
    "no_normalisation": ("out_row[d] = acc / z;", "out_row[d] = acc;"),
    "no_max_subtraction": ("w[j - a] = exp(w[j - a] - m);", "w[j - a] = exp(w[j - a]);"),
    "sign_of_logit": ("w[j - a] = P->scale * dot;", "w[j - a] = -P->scale * dot;"),
    "key_head_swapped": ("widen(P->k, P->dtype, ((size_t)j * H + h) * D + e);",
                         "widen(P->k, P->dtype, ((size_t)j * H + (H - 1 - h)) * D + e);"),
    "segment_end_off_by_one": ("for (int32_t j = a; j < b; ++j) {\n    double dot",
                               "for (int32_t j = a; j < b - (b - a > 1); ++j) {\n    double dot"),
}


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_planted_mistake_fails_a_pin(name):
    old, new = MUTATIONS[name]
    src = open(os.path.join(os.path.dirname(oracle.__file__), "attn_oracle.c")).read()
    assert src.count(old) >= 1, f"mutation anchor for {name} not found"
    mutated = src.replace(old, new, 1)
    with tempfile.TemporaryDirectory() as d:
        path = os.path.join(d, "attn_oracle.c")
        open(path, "w").write(mutated)
        so = os.path.join(d, "libmut.so")
        import subprocess
        subprocess.check_call(["gcc", "-O2", "-shared", "-fPIC", "-pthread", path, "-o", so, "-lm"])
        lib = oracle.load(so)
        errs = [pin_bruteforce(lib), pin_dominant_key(lib)]
    assert max(errs) > 1e-6, f"mutation {name} was not caught: {errs}"

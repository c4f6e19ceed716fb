"""Pins for the text decoder's attention oracle (``oracle/decoder.py``): causal, a local
window, grouped-query heads.

The definition (the Muse Glimmer next-steps document, "Architecture / Text decoder", in the
reading stated in the oracle's header) is pinned against things other than the oracle's own
arithmetic:
  * brute force in 50-digit decimals on a tiny case;
  * closed forms: window 1 and the first query of a segment return that token's V exactly;
    constant V per key/value head returns that head's constant (the head mapping);
  * the plain non-causal attention oracle (the C oracle, pinned on its own), applied to a
    segment made of a query's allowed keys alone, gives that query's row;
  * invariants: extending a segment leaves its earlier rows unchanged (causality); a window
    at least as long as the segment equals no window;
  * the pair count against enumeration;
  * planted mistakes (window off by one, no causal mask, the wrong head mapping) fail a pin.
"""
import decimal

import numpy as np
import pytest

import oracle
import workloads
from oracle import decoder


def _rand(seed, *shape):
    return np.random.default_rng(seed).standard_normal(shape)


def _inputs(seed, T, Hq, Hkv, D):
    return _rand(seed, T, Hq, D), _rand(seed + 1, T, Hkv, D), _rand(seed + 2, T, Hkv, D)


def test_brute_force_in_decimal():
    decimal.getcontext().prec = 50
    D = decimal.Decimal
    T, Hq, Hkv, d, W, scale = 6, 2, 1, 3, 3, 0.7
    q, k, v = _inputs(1, T, Hq, Hkv, d)
    cu = np.array([0, 2, 6], np.int32)
    got = decoder.attn_fwd(q, k, v, cu, scale, W)
    for s in range(2):
        a0, a1 = int(cu[s]), int(cu[s + 1])
        for i in range(a0, a1):
            for h in range(Hq):
                keys = [j for j in range(a0, a1) if j <= i and j > i - W]
                logits = [D(scale) * sum(D(float(q[i, h, c])) * D(float(k[j, 0, c])) for c in range(d))
                          for j in keys]
                w = [x.exp() for x in logits]  # no max subtraction: small logits
                z = sum(w)
                for c in range(d):
                    want = sum(wj * D(float(v[j, 0, c])) for wj, j in zip(w, keys)) / z
                    assert abs(float(want) - got[i, h, c]) < 1e-13


def test_window_one_and_first_query_return_their_own_value():
    T, Hq, Hkv, D = 40, 4, 2, 8
    q, k, v = _inputs(3, T, Hq, Hkv, D)
    cu = np.array([0, 13, 13, 40], np.int32)
    one = decoder.attn_fwd(q, k, v, cu, 0.5, 1)
    full = decoder.attn_fwd(q, k, v, cu, 0.5, 0)
    for h in range(Hq):
        g = h // 2
        np.testing.assert_array_equal(one[:, h], v[:, g])
        for a0 in (0, 13):
            np.testing.assert_array_equal(full[a0, h], v[a0, g])


def test_each_row_is_plain_attention_over_its_allowed_keys():
    """Row i of head h equals the C oracle's non-causal attention for a segment holding only
    i's allowed keys, with q_i placed as that segment's last query."""
    T, Hq, Hkv, D, W, scale = 70, 4, 2, 16, 9, 0.3
    q, k, v = _inputs(5, T, Hq, Hkv, D)
    cu = np.array([0, 25, 70], np.int32)
    got = decoder.attn_fwd(q, k, v, cu, scale, W)
    for i in (0, 1, 8, 9, 24, 25, 26, 33, 34, 69):
        s = 0 if i < 25 else 1
        lo = max(int(cu[s]), i - W + 1)
        n = i + 1 - lo
        for h in range(Hq):
            g = h // 2
            qq = np.zeros((n, 1, D))
            qq[-1, 0] = q[i, h]
            ref = oracle.attn_fwd(qq, k[lo:i + 1, g:g + 1], v[lo:i + 1, g:g + 1],
                                  np.array([0, n], np.int32), scale)
            np.testing.assert_allclose(got[i, h], ref[-1, 0], rtol=0, atol=1e-14)


def test_head_mapping_by_constant_values():
    T, Hq, Hkv, D = 30, 8, 2, 4
    q, k, _ = _inputs(7, T, Hq, Hkv, D)
    v = np.zeros((T, Hkv, D))
    v[:, 0, :], v[:, 1, :] = 1.0, 2.0
    out = decoder.attn_fwd(q, k, v, np.array([0, T], np.int32), 0.9, 5)
    for h in range(Hq):
        np.testing.assert_allclose(out[:, h], 1.0 + (h // 4), rtol=0, atol=1e-14)


def test_extending_a_segment_leaves_earlier_rows_unchanged_and_long_windows_change_nothing():
    T, Hq, Hkv, D, W = 50, 2, 2, 8, 7
    q, k, v = _inputs(9, T, Hq, Hkv, D)
    a = decoder.attn_fwd(q[:30], k[:30], v[:30], np.array([0, 30], np.int32), 0.4, W)
    b = decoder.attn_fwd(q, k, v, np.array([0, T], np.int32), 0.4, W)
    # equal up to the rounding of matrix products of different sizes
    np.testing.assert_allclose(a, b[:30], rtol=0, atol=1e-14)
    c = decoder.attn_fwd(q, k, v, np.array([0, T], np.int32), 0.4, T)
    d = decoder.attn_fwd(q, k, v, np.array([0, T], np.int32), 0.4, 0)
    np.testing.assert_allclose(c, d, rtol=0, atol=1e-14)


def test_rows_match_the_whole_matrix():
    T, Hq, Hkv, D, W = 60, 4, 1, 8, 11
    q, k, v = _inputs(11, T, Hq, Hkv, D)
    cu = np.array([0, 17, 60], np.int32)
    full = decoder.attn_fwd(q, k, v, cu, 0.35, W)
    tok = np.array([0, 5, 16, 17, 30, 59]); head = np.array([0, 1, 2, 3, 0, 3])
    rows = decoder.attn_rows(q, k, v, cu, 0.35, W, tok, head)
    np.testing.assert_allclose(rows, full[tok, head], rtol=0, atol=1e-14)


@pytest.mark.parametrize("lengths,window", [([5, 0, 9, 1], 3), ([4096], 2048), ([3000, 100], 0),
                                            ([2048], 2048), ([10], 100)])
def test_pair_count_against_enumeration(lengths, window):
    cu = workloads.cu_from_lengths(lengths)
    want = 0
    for L in lengths:
        for i in range(L):
            want += (i + 1) if window <= 0 else min(i + 1, window)
    assert workloads.decoder_pairs(cu, window) == want
    assert workloads.decoder_flops(cu, window, 32, 128) == 4 * want * 32 * 128


# ---------------------------------------------------------------- planted mistakes

def _mutant(kind):
    def fwd(q, k, v, cu, scale, window):
        T, Hq, D = q.shape
        Hkv = k.shape[1]
        out = np.zeros((T, Hq, D))
        for s in range(len(cu) - 1):
            a0, a1 = int(cu[s]), int(cu[s + 1])
            for i in range(a0, a1):
                for h in range(Hq):
                    g = h % Hkv if kind == "head_modulo" else h // (Hq // Hkv)
                    if kind == "no_causal":
                        keys = range(a0, a1)
                    elif kind == "window_plus_one":
                        keys = range(max(a0, i - window), i + 1)
                    elif kind == "window_excludes_self":
                        keys = range(max(a0, i - window + 1), i) or range(i, i + 1)
                    else:
                        keys = range(max(a0, i - window + 1), i + 1)
                    a = scale * (k[keys.start:keys.stop, g] @ q[i, h])
                    w = np.exp(a - a.max())
                    out[i, h] = (w[:, None] * v[keys.start:keys.stop, g]).sum(0) / w.sum()
        return out
    return fwd


@pytest.mark.parametrize("kind", ["no_causal", "window_plus_one", "window_excludes_self", "head_modulo"])
def test_planted_mistakes_fail_a_pin(kind):
    """Each mutant differs from the pins above on a small case (row-by-row C-oracle pin)."""
    T, Hq, Hkv, D, W, scale = 24, 4, 2, 8, 5, 0.5
    q, k, v = _inputs(13, T, Hq, Hkv, D)
    cu = np.array([0, 24], np.int32)
    good = _mutant("none")(q, k, v, cu, scale, W)
    np.testing.assert_allclose(good, decoder.attn_fwd(q, k, v, cu, scale, W), rtol=0, atol=1e-13)
    bad = _mutant(kind)(q, k, v, cu, scale, W)
    assert np.abs(bad - good).max() > 1e-3

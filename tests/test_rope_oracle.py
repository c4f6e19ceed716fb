"""Pins of the 2D RoPE oracle (oracle/rope.py) against things other than itself.

The reading (width-first angles, 1-based positions, pairs (d, d + D/2), frequencies
theta^(-2 i / (D/2))) is stated in the oracle; these checks fix it:
  * closed forms: position (0, 0) is the identity; D = 4 written out by hand; complex
    rotation z * exp(i a) computed element by element with Python complex numbers;
  * invariants: every (d, d + D/2) pair keeps its norm; rotations compose additively in
    the position; a score <rope(q, p), rope(k, p')> depends on p - p' only, so equal
    positions give the unrotated score and attention over one position equals plain
    attention;
  * the width-first order: a width-only position turns only the width angles;
  * planted mistakes (height first, interleaved pairs, 0-based positions, a wrong
    frequency exponent) each fail one of these checks.
"""
import cmath
import math

import numpy as np
import pytest

import oracle
from oracle import rope
import workloads


def _rand(seed, T, H, D):
    return np.random.default_rng(seed).normal(size=(T, H, D))


def test_frequencies_closed_form():
    D, theta = 96, 10000.0
    f = rope.rope_frequencies(D, theta)
    assert len(f) == 24 and f[0] == 1.0
    assert math.isclose(f[1], theta ** (-2.0 / 48), rel_tol=1e-15)
    assert math.isclose(f[23], theta ** (-46.0 / 48), rel_tol=1e-15)
    assert np.allclose(f[1:] / f[:-1], theta ** (-2.0 / 48), rtol=1e-14, atol=0)


def test_position_zero_is_the_identity():
    x = _rand(1, 5, 2, 96)
    assert np.array_equal(rope.rope2d(x, np.zeros((5, 2), np.int32)), x)


def test_d4_written_out():
    x = _rand(2, 3, 1, 4)
    pos = np.array([[1, 1], [2, 5], [7, 3]], np.int32)
    got = rope.rope2d(x, pos, theta=10000.0)
    for t in range(3):
        pw, ph = float(pos[t, 0]), float(pos[t, 1])  # F = 1, f_0 = 1
        a, b, c, d = x[t, 0]
        want = [a * math.cos(pw) - c * math.sin(pw), b * math.cos(ph) - d * math.sin(ph),
                c * math.cos(pw) + a * math.sin(pw), d * math.cos(ph) + b * math.sin(ph)]
        assert np.allclose(got[t, 0], want, rtol=0, atol=1e-15)


def test_complex_rotation_element_by_element():
    D, theta = 96, 10000.0
    x = _rand(3, 4, 2, D)
    pos = np.array([[1, 1], [32, 1], [5, 17], [128, 128]], np.int32)
    got = rope.rope2d(x, pos, theta)
    half, F = D // 2, D // 4
    for t in range(4):
        for h in range(2):
            for d in range(half):
                axis_pos = pos[t, 0] if d < F else pos[t, 1]
                ang = axis_pos * theta ** (-2.0 * (d % F) / half)
                z = complex(x[t, h, d], x[t, h, d + half]) * cmath.exp(1j * ang)
                assert abs(got[t, h, d] - z.real) < 1e-13 and abs(got[t, h, d + half] - z.imag) < 1e-13


def test_pairs_keep_their_norm_and_rotations_compose():
    x = _rand(4, 6, 3, 96)
    p1 = np.random.default_rng(4).integers(0, 64, size=(6, 2)).astype(np.int32)
    p2 = np.random.default_rng(5).integers(0, 64, size=(6, 2)).astype(np.int32)
    r = rope.rope2d(x, p1)
    n0 = x[..., :48] ** 2 + x[..., 48:] ** 2
    n1 = r[..., :48] ** 2 + r[..., 48:] ** 2
    assert np.allclose(n0, n1, rtol=1e-13, atol=0)
    assert np.allclose(rope.rope2d(r, p2), rope.rope2d(x, p1 + p2), rtol=0, atol=1e-12)


def test_scores_depend_on_relative_position_only():
    q, k = _rand(6, 1, 1, 96)[0, 0], _rand(7, 1, 1, 96)[0, 0]
    def score(pq, pk):
        rq = rope.rope2d(q[None, None], np.array([pq], np.int32))[0, 0]
        rk = rope.rope2d(k[None, None], np.array([pk], np.int32))[0, 0]
        return float(rq @ rk)
    base = score((3, 9), (10, 2))
    assert math.isclose(score((3 + 20, 9 + 7), (10 + 20, 2 + 7)), base, rel_tol=1e-12)
    assert math.isclose(score((5, 5), (5, 5)), float(q @ k), rel_tol=1e-12)


def test_width_first():
    x = _rand(8, 1, 1, 96)
    r = rope.rope2d(x, np.array([[1, 0]], np.int32))   # width position only
    assert not np.allclose(r[..., 0:24], x[..., 0:24])     # width angles turn
    assert np.array_equal(r[..., 24:48], x[..., 24:48])    # height angles do not
    assert np.array_equal(r[..., 72:96], x[..., 72:96])


def test_one_position_per_segment_is_plain_attention():
    T = 200
    q, k, v = workloads.qkv(9, T, H=2)
    cu = workloads.cu_from_lengths([120, 80])
    pos = np.array([[4, 7]] * 120 + [[30, 2]] * 80, np.int32)
    a = rope.attn_fwd_rope2d(q, k, v, cu, 0.1, pos)
    b = oracle.attn_fwd(q, k, v, cu, 0.1)
    assert np.allclose(a, b, rtol=0, atol=1e-12)


def test_image_positions_are_one_based_and_row_major():
    p = rope.image_positions([(2, 3), (1, 2)])
    assert p.tolist() == [[1, 1], [2, 1], [3, 1], [1, 2], [2, 2], [3, 2], [1, 1], [2, 1]]


# ---------------------------------------------------------------- planted mistakes

def _height_first(x, pos, theta=10000.0):
    return rope.rope2d(x, np.asarray(pos)[:, ::-1], theta)


def _interleaved(x, pos, theta=10000.0):
    x = np.asarray(x, np.float64)
    a = rope.rope_angles(pos, x.shape[-1], theta)[:, None, :]
    xe, xo = x[..., 0::2], x[..., 1::2]
    out = np.empty_like(x)
    out[..., 0::2] = xe * np.cos(a) - xo * np.sin(a)
    out[..., 1::2] = xo * np.cos(a) + xe * np.sin(a)
    return out


def _zero_based(x, pos, theta=10000.0):
    return rope.rope2d(x, np.asarray(pos) - 1, theta)


def _wrong_exponent(x, pos, theta=10000.0):
    x = np.asarray(x, np.float64)
    D = x.shape[-1]
    f = np.array([theta ** (-1.0 * i / (D // 2)) for i in range(D // 4)])
    p = np.asarray(pos, np.float64)
    a = np.concatenate([p[:, 0:1] * f, p[:, 1:2] * f], axis=1)[:, None, :]
    x1, x2 = x[..., :D // 2], x[..., D // 2:]
    return np.concatenate([x1 * np.cos(a) - x2 * np.sin(a), x2 * np.cos(a) + x1 * np.sin(a)], axis=-1)


@pytest.mark.parametrize("mutant", [_height_first, _interleaved, _zero_based, _wrong_exponent],
                         ids=["height_first", "interleaved", "zero_based", "wrong_exponent"])
def test_planted_mistakes_fail_a_pin(mutant):
    """Each mutant, fed the tower's 1-based image positions, differs from the complex
    rotation written out element by element (the pin above)."""
    D, theta = 96, 10000.0
    x = _rand(10, 3, 1, D)
    pos = rope.image_positions([(2, 3)])[:3] + np.array([[4, 1]], np.int32)  # pw != ph
    got = mutant(x, pos, theta)
    half, F = D // 2, D // 4
    want = np.empty_like(got)
    for t in range(3):
        for d in range(half):
            axis_pos = (pos[t, 0] if d < F else pos[t, 1])
            z = complex(x[t, 0, d], x[t, 0, d + half]) * cmath.exp(1j * axis_pos * theta ** (-2.0 * (d % F) / half))
            want[t, 0, d], want[t, 0, d + half] = z.real, z.imag
    assert not np.allclose(got, want, rtol=0, atol=1e-9)
    assert np.allclose(rope.rope2d(x, pos, theta), want, rtol=0, atol=1e-12)

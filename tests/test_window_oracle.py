"""Pins of the window-segmentation oracle (CPU).

The pages fix the window (32 x 32 patches) and say that the walk over the blocks and the
order inside a block matter, without printing either; the oracle takes the plain row-major
reading.  These pins check what follows from the definition without retyping it: the
permutation is a bijection, each block is one rectangle of its image, blocks and the tokens
inside them come in increasing image order, and a ragged grid has the block sizes its
division leaves.  Planted mistakes (column-major walks, no ragged edge, images not offset)
must fail at least one pin.
"""
import numpy as np
import pytest

from oracle.window import window_permutation


def _check(perm, cu, grids, win):
    T = sum(h * w for h, w in grids)
    assert perm.dtype == np.int32 and len(perm) == T
    assert np.array_equal(np.sort(perm), np.arange(T))          # a bijection
    assert cu[0] == 0 and cu[-1] == T and np.all(np.diff(cu) > 0)
    # image of each token and its (y, x)
    bases = np.cumsum([0] + [h * w for h, w in grids])
    firsts = []
    for s in range(len(cu) - 1):
        seg = perm[cu[s]:cu[s + 1]]
        img = np.searchsorted(bases, seg[0], side="right") - 1
        h, w = grids[img]
        assert np.all((seg >= bases[img]) & (seg < bases[img + 1]))  # one image
        loc = seg - bases[img]
        ys, xs = loc // w, loc % w
        # one rectangle, at most win x win, aligned to the block grid
        y0, x0 = ys.min(), xs.min()
        hh, ww = ys.max() - y0 + 1, xs.max() - x0 + 1
        assert hh * ww == len(seg) and hh <= win and ww <= win
        assert y0 % win == 0 and x0 % win == 0
        assert np.all(np.diff(seg) > 0)                           # row-major inside the block
        firsts.append(seg[0])
    assert np.all(np.diff(firsts) > 0)                            # blocks walked in image order
    return [int(x) for x in np.diff(cu)]


def test_regular_grid():
    perm, cu = window_permutation([(64, 64)], 32)
    assert _check(perm, cu, [(64, 64)], 32) == [1024] * 4
    # block 1 of a 64-wide grid starts at column 32 of row 0
    assert perm[1024] == 32 and perm[2048] == 32 * 64


def test_ragged_grid_block_sizes():
    # 40 x 50 patches: blocks 32x32, 32x18 | 8x32, 8x18
    perm, cu = window_permutation([(40, 50)], 32)
    assert _check(perm, cu, [(40, 50)], 32) == [1024, 576, 256, 144]


def test_several_images_and_small_windows():
    grids = [(8, 8), (13, 29), (64, 33), (1, 1)]
    perm, cu = window_permutation(grids, 8)
    sizes = _check(perm, cu, grids, 8)
    assert len(sizes) == 1 + 2 * 4 + 8 * 5 + 1


def test_tower_grid():
    perm, cu = window_permutation([(128, 128)], 32)
    assert _check(perm, cu, [(128, 128)], 32) == [1024] * 16


def _mutant_colmajor_blocks(grids, win):
    perm, lengths, base = [], [], 0
    for h, w in grids:
        for bx in range(0, w, win):
            for by in range(0, h, win):
                n = 0
                for y in range(by, min(by + win, h)):
                    for x in range(bx, min(bx + win, w)):
                        perm.append(base + y * w + x); n += 1
                lengths.append(n)
        base += h * w
    return np.asarray(perm, np.int32), np.concatenate([[0], np.cumsum(lengths)]).astype(np.int32)


def _mutant_colmajor_inside(grids, win):
    perm, lengths, base = [], [], 0
    for h, w in grids:
        for by in range(0, h, win):
            for bx in range(0, w, win):
                n = 0
                for x in range(bx, min(bx + win, w)):
                    for y in range(by, min(by + win, h)):
                        perm.append(base + y * w + x); n += 1
                lengths.append(n)
        base += h * w
    return np.asarray(perm, np.int32), np.concatenate([[0], np.cumsum(lengths)]).astype(np.int32)


def _mutant_no_ragged_edge(grids, win):
    perm, lengths, base = [], [], 0
    for h, w in grids:
        for by in range(0, h, win):
            for bx in range(0, w, win):
                n = 0
                for y in range(by, by + win):
                    for x in range(bx, bx + win):
                        if y < h and x < w:
                            perm.append(base + y * w + x); n += 1
                lengths.append(win * win)
        base += h * w
    return np.asarray(perm, np.int32), np.concatenate([[0], np.cumsum(lengths)]).astype(np.int32)


def _mutant_no_image_offset(grids, win):
    perm, cu = window_permutation(grids, win)
    bases = np.cumsum([0] + [h * w for h, w in grids])
    img = np.searchsorted(bases, perm, side="right") - 1
    return (perm - bases[img]).astype(np.int32), cu


@pytest.mark.parametrize("mutant", [_mutant_colmajor_blocks, _mutant_colmajor_inside,
                                    _mutant_no_ragged_edge, _mutant_no_image_offset])
def test_planted_mistakes_fail(mutant):
    grids = [(40, 50), (13, 29)]
    perm, cu = mutant(grids, 32)
    with pytest.raises(AssertionError):
        _check(perm, cu, grids, 32)


def _tiny_inputs(T, seed, H=2, D=8):
    import workloads
    return workloads.qkv(seed, T, H, D, "f32")


def test_window_attention_single_window_is_plain_attention():
    # a grid smaller than one window is a single segment: the permutation is the identity
    import oracle
    from oracle.window import window_attention
    q, k, v = _tiny_inputs(5 * 7, 1)
    got = window_attention(q, k, v, [(5, 7)], 0.3, win=8)
    ref = oracle.attn_fwd(q, k, v, np.array([0, 35], np.int32), 0.3)
    assert np.array_equal(got, ref)


def test_window_attention_windows_are_independent():
    # every window's output is attention over exactly that window's tokens, computed alone
    import oracle
    from oracle.window import window_attention
    grids, win = [(6, 5), (3, 4)], 4
    T = 6 * 5 + 3 * 4
    q, k, v = _tiny_inputs(T, 2)
    got = window_attention(q, k, v, grids, 0.5, win=win)
    bases = [0, 30]
    for img, (h, w) in enumerate(grids):
        for by in range(0, h, win):
            for bx in range(0, w, win):
                toks = np.array([bases[img] + y * w + x for y in range(by, min(by + win, h))
                                 for x in range(bx, min(bx + win, w))], np.int64)
                cu = np.array([0, len(toks)], np.int32)
                ref = oracle.attn_fwd(q[toks], k[toks], v[toks], cu, 0.5)
                assert np.allclose(got[toks], ref, rtol=0, atol=1e-12)


@pytest.mark.parametrize("h,w", [(128, 128), (64, 64), (40, 50), (33, 97), (8, 8)])
def test_matches_the_workload_window_lengths(h, w):
    # the tower workloads build window-layer segments directly (workloads.window_lengths);
    # they must be the segments of the window order
    import workloads
    _, cu = window_permutation([(h, w)], 32)
    assert [int(x) for x in np.diff(cu)] == workloads.window_lengths(h, w)

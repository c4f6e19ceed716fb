"""2D RoPE on the GPU (through the C-ABI) against the f64 RoPE oracle.

The rotation pass computes in f32 (angles pos * f_i, reduced to [-pi, pi], hardware sin/cos
with ~2^-21 absolute error) and rounds to bf16, so each element is compared with the f64
oracle within one bf16 ulp of the oracle's value (the output rounding) plus a bound on the
f32 evaluation error, which grows with the angle (two f32 roundings of pos * f_i).  Positions are those of the tower's 128 x 128 patch
grid taken in window order, as the tower carries them.
"""
import numpy as np
import pytest

import workloads
from oracle import rope
from oracle.window import window_permutation

torch = pytest.importorskip("torch")

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _need_gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from conftest import build_cuda_library
    build_cuda_library()


def _bf16_dev(a):
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).cuda()


def _within_one_ulp(got, ref, x, ang):
    """|got - ref| <= one bf16 ulp of ref plus the f32 evaluation's absolute error.  The
    f32 angle pos * f_i carries two roundings (f_i and the product), under |a| 2^-23; the
    reduction and the hardware sin/cos add ~2^-21; each output element is
    x_d cos - x_{d+48} sin (or the mirror), so (|x_d| + |x_{d+48}|)(|a| 2^-22 + 2^-20) bounds
    it with a factor of two to spare.  It matters where the two terms cancel and ref, hence
    its ulp, is tiny."""
    ulp = np.exp2(np.floor(np.log2(np.maximum(np.abs(ref), 2.0 ** -126))) - 7)
    pair = np.abs(x[..., :48]) + np.abs(x[..., 48:])
    err = pair * (np.abs(ang)[:, None, :] * 2.0 ** -22 + 2.0 ** -20)
    return np.abs(got - ref) <= ulp + np.concatenate([err, err], axis=-1)


def tower_positions(grid=128, win=32):
    perm, _ = window_permutation([(grid, grid)], win)
    return rope.image_positions([(grid, grid)])[perm]


@pytest.mark.parametrize("theta", [10000.0, 100.0])
def test_rope2d_matches_oracle_on_the_tower_grid(theta):
    import flash_attention_varlen_b200 as fa
    pos = tower_positions()
    T = pos.shape[0]
    q, _, _ = workloads.qkv(31, T)
    got = fa.rope2d(_bf16_dev(q), torch.from_numpy(pos).cuda(), theta=theta)
    torch.cuda.synchronize()
    got = got.float().cpu().numpy().astype(np.float64)
    ref = rope.rope2d(q, pos, theta)
    ang = rope.rope_angles(pos, 96, theta)
    ok = _within_one_ulp(got, ref, workloads.bf16_bits_to_f32(q).astype(np.float64), ang)
    assert np.isfinite(got).all() and ok.all(), f"{(~ok).sum()} elements beyond one ulp"
    # and almost everywhere the correctly rounded oracle value itself: the f32 error only
    # flips the rounding of values within ~2^-16 relative of a rounding midpoint
    b = ref.astype(np.float32).view(np.uint32)
    b = ((b + 0x7FFF + ((b >> 16) & 1)) >> 16 << 16).astype(np.uint32)
    ref_bf16 = b.view(np.float32).astype(np.float64)
    assert np.mean(got == ref_bf16) > 0.99
    assert np.mean(np.abs(got - ref)) <= 1.01 * np.mean(np.abs(ref_bf16 - ref))


def test_rope2d_odd_head_count_and_more_items_than_threads():
    """H = 9 (rows of a token not a multiple of any block) and 40,000 tokens: 2.16M
    (token, head, group) items against a grid of at most 148 x 64 blocks of 192 threads
    (1.82M), so threads take a second item on the grid stride, each staying on its own
    column group.  Every element within the one-ulp bound of the oracle."""
    import flash_attention_varlen_b200 as fa
    T, H = 40000, 9
    q, _, _ = workloads.qkv(39, T, H=H)
    pos = np.random.default_rng(6).integers(1, 400, size=(T, 2)).astype(np.int32)
    got = fa.rope2d(_bf16_dev(q), torch.from_numpy(pos).cuda())
    torch.cuda.synchronize()
    got = got.float().cpu().numpy().astype(np.float64)
    ref = rope.rope2d(q, pos)
    ang = rope.rope_angles(pos, 96, rope.DEFAULT_THETA)
    ok = _within_one_ulp(got, ref, workloads.bf16_bits_to_f32(q).astype(np.float64), ang)
    assert np.isfinite(got).all() and ok.all(), f"{(~ok).sum()} elements beyond one ulp"


def test_rope2d_in_place_equals_out_of_place_and_position_zero_is_identity():
    import flash_attention_varlen_b200 as fa
    T, H = 300, 3
    q, _, _ = workloads.qkv(32, T, H=H)
    pos = np.random.default_rng(5).integers(1, 200, size=(T, 2)).astype(np.int32)
    x = _bf16_dev(q)
    p = torch.from_numpy(pos).cuda()
    out = fa.rope2d(x, p)
    fa.rope2d(x, p, out=x)
    torch.cuda.synchronize()
    assert torch.equal(out, x)
    z = _bf16_dev(q)
    ident = fa.rope2d(z, torch.zeros(T, 2, dtype=torch.int32, device="cuda"))
    torch.cuda.synchronize()
    assert torch.equal(ident, z)


def test_rope2d_rejects_bad_arguments():
    from flash_attention_varlen_b200 import _binding as b
    x = torch.zeros(8, 16, 96, dtype=torch.bfloat16, device="cuda")
    pos = torch.ones(8, 2, dtype=torch.int32, device="cuda")
    s = torch.cuda.current_stream().cuda_stream
    assert b.vt_rope2d(x.data_ptr(), x.data_ptr(), pos.data_ptr(), 8, 16, 64, 1e4, s) == b.VT_ERR_UNSUPPORTED
    assert b.vt_rope2d(x.data_ptr(), x.data_ptr(), pos.data_ptr(), 8, 16, 96, -1.0, s) == b.VT_ERR_INVALID_ARG
    assert b.vt_rope2d(x.data_ptr(), x.data_ptr() + 2, pos.data_ptr(), 8, 16, 96, 1e4, s) == b.VT_ERR_INVALID_ARG
    assert b.vt_rope2d(0, x.data_ptr(), pos.data_ptr(), 8, 16, 96, 1e4, s) == b.VT_ERR_NULL
    assert b.vt_rope2d(x.data_ptr(), x.data_ptr(), pos.data_ptr(), 0, 16, 96, 1e4, s) == b.VT_OK


BF16_MAX, BF16_MEAN = 1e-2, 1e-3


def _rope_attn(q, k, v, cu, pos, theta=10000.0, in_place=False):
    import flash_attention_varlen_b200 as fa
    dq, dk, dv = _bf16_dev(q), _bf16_dev(k), _bf16_dev(v)
    dcu = torch.from_numpy(np.ascontiguousarray(cu, np.int32)).cuda()
    dpos = torch.from_numpy(np.ascontiguousarray(pos, np.int32)).cuda()
    out = fa.attn_fwd_rope2d(dq, dk, dv, dcu, dpos, theta=theta, k_rot=dk if in_place else None)
    fa.check_device_status()
    return out.float().cpu().numpy().astype(np.float64), dk


def _check(got, ref, what):
    err = np.abs(got - ref)
    assert np.isfinite(got).all(), what
    assert err.max() <= BF16_MAX, f"{what}: max-abs {err.max():.3e}"
    assert err.mean() <= BF16_MEAN, f"{what}: mean-abs {err.mean():.3e}"


def test_rope_attention_image448_full_layer():
    """One 448 x 448 image (32 x 32 patches, 1024 tokens) as one full-attention segment."""
    import math
    q, k, v = workloads.qkv(33, 1024)
    pos = rope.image_positions([(32, 32)])
    cu = np.array([0, 1024], np.int32)
    got, _ = _rope_attn(q, k, v, cu, pos)
    ref = rope.attn_fwd_rope2d(q, k, v, cu, 1.0 / math.sqrt(96), pos)
    _check(got, ref, "rope image448")


def test_rope_attention_tower_window_layer_in_window_order():
    """The tower's window layer: 16 windows of the 128 x 128 grid, tokens (and their
    positions) in window order; sampled rows in every unit."""
    import math
    from test_gpu_parity import _unit_rows
    perm, cu = window_permutation([(128, 128)], 32)
    pos = rope.image_positions([(128, 128)])[perm]
    q, k, v = workloads.qkv(34, 16384)
    got, _ = _rope_attn(q, k, v, cu, pos)
    tok, head = _unit_rows(cu, 16, 34)
    ref = rope.attn_rows_rope2d(q, k, v, cu, 1.0 / math.sqrt(96), pos, tok, head)
    _check(got[tok, head], ref, "rope tower window layer")


def test_rope_attention_varlen_images_ragged_and_k_in_place():
    """Eight images of unequal size (their own positions), ragged segment ends inside Q
    and K tiles; K rotated in place (k_rot = k) gives the same output and leaves rope(K)."""
    import math
    grids = workloads.varlen_image_grids(0)
    pos = rope.image_positions(grids)
    lengths = [h * w for h, w in grids]
    cu = workloads.cu_from_lengths(lengths)
    T = int(cu[-1])
    q, k, v = workloads.qkv(35, T)
    got, _ = _rope_attn(q, k, v, cu, pos)
    ref = rope.attn_fwd_rope2d(q, k, v, cu, 1.0 / math.sqrt(96), pos)
    _check(got, ref, "rope varlen8")
    got2, dk = _rope_attn(q, k, v, cu, pos, in_place=True)
    assert np.array_equal(got, got2)
    import flash_attention_varlen_b200 as fa
    kr = fa.rope2d(_bf16_dev(k), torch.from_numpy(pos).cuda())
    torch.cuda.synchronize()
    assert torch.equal(kr, dk)


def test_rope_attention_positions_all_equal_is_plain_attention():
    """One position for every token of a segment: rope cancels in every score, so the
    result is plain attention on the unrotated inputs (up to the bf16 rounding of the
    rotated Q and K)."""
    import math
    import oracle
    lengths = [300, 129, 640]
    cu = workloads.cu_from_lengths(lengths)
    T = int(cu[-1])
    q, k, v = workloads.qkv(36, T)
    pos = np.repeat(np.array([[7, 3], [60, 1], [1, 128]], np.int32), lengths, axis=0)
    got, _ = _rope_attn(q, k, v, cu, pos)
    _check(got, oracle.attn_fwd(q, k, v, cu, 1.0 / math.sqrt(96)), "rope equal positions")


@pytest.mark.parametrize("case", ["window16x1024", "ragged"])
def test_rope_attention_equals_rotation_then_plain_attention_bit_for_bit(case):
    """The RoPE attention rotates Q into ``out`` and the attention writes O over it: the
    result must equal, bit for bit, rope2d(Q), rope2d(K) into separate buffers followed by
    the plain attention.  The ragged case ends segments inside Q tiles, where a tile also
    carries rows of the next segment that another unit overwrites with its O."""
    import math
    import flash_attention_varlen_b200 as fa
    if case == "window16x1024":
        perm, cu = window_permutation([(128, 128)], 32)
        pos = rope.image_positions([(128, 128)])[perm]
    else:
        lengths = [1, 200, 129, 383, 2, 640, 255, 90]
        cu = workloads.cu_from_lengths(lengths)
        rng = np.random.default_rng(8)
        pos = rng.integers(1, 129, size=(int(cu[-1]), 2)).astype(np.int32)
    T = int(cu[-1])
    q, k, v = workloads.qkv(37, T)
    dq, dk, dv = _bf16_dev(q), _bf16_dev(k), _bf16_dev(v)
    dcu = torch.from_numpy(np.ascontiguousarray(cu, np.int32)).cuda()
    dpos = torch.from_numpy(np.ascontiguousarray(pos, np.int32)).cuda()
    scale = 1.0 / math.sqrt(96)
    fused = fa.attn_fwd_rope2d(dq, dk, dv, dcu, dpos, scale=scale)
    qr, kr = fa.rope2d(dq, dpos), fa.rope2d(dk, dpos)
    steps = fa.attn_fwd(qr, kr, dv, dcu, scale=scale)
    fa.check_device_status()
    assert torch.equal(fused, steps)
    assert torch.equal(dq, _bf16_dev(q))  # Q itself is left as it was


def test_rope_attention_many_images_with_the_scheduling_prepass():
    """40 small images (more segments than the kernel schedules by itself, so the
    scheduling prepass runs between the rotation pass and the attention), every element
    against the RoPE oracle."""
    import math
    rng = np.random.default_rng(9)
    grids = [(int(h), int(w)) for h, w in rng.integers(2, 19, size=(40, 2))]
    pos = rope.image_positions(grids)
    cu = workloads.cu_from_lengths([h * w for h, w in grids])
    T = int(cu[-1])
    q, k, v = workloads.qkv(38, T)
    got, _ = _rope_attn(q, k, v, cu, pos)
    ref = rope.attn_fwd_rope2d(q, k, v, cu, 1.0 / math.sqrt(96), pos)
    _check(got, ref, "rope 40 images")

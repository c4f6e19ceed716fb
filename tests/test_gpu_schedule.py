"""The two ways a bf16 call gets its work list, through the C-ABI.

A call with at most 32 segments builds its work list inside the attention kernel (one warp
per CTA, in shared memory); a call with more runs the scheduling prepass kernel first.
Both must validate cu_seqlens the same way and produce the same units, so the outputs are
bit-identical: empty segments appended to a call push it onto the prepass path without
changing its units.  The per-call device status alternates between two words; a sequence
of good and malformed calls on one stream, over both paths and both dtypes, checks that
each call reports its own finding.
"""
import numpy as np
import pytest

import workloads

torch = pytest.importorskip("torch")

pytestmark = pytest.mark.gpu

INLINE_MAX = 32  # segments up to which the kernel builds its own work list


@pytest.fixture(scope="module", autouse=True)
def _need_gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from conftest import build_cuda_library
    build_cuda_library()


def _qkv(T, seed, H=16, dtype=torch.bfloat16):
    g = torch.Generator(device="cuda").manual_seed(seed)
    return [torch.randn(T, H, 96, device="cuda", generator=g).to(dtype) for _ in range(3)]


def _padded(cu, n_total):
    """cu_seqlens with empty segments appended up to n_total segments."""
    T = cu[-1]
    return list(cu) + [T] * (n_total + 1 - len(cu))


def _lengths_cases():
    rng = np.random.default_rng(7)
    return {
        "one_segment_1024": [1024],
        "window_layer_4x1024": [1024] * 4,
        "eight_images": [int(h) * int(w) for h, w in rng.integers(8, 65, size=(8, 2))],
        "ragged_with_empty": [0, 300, 1, 0, 129, 700, 0, 256],
        "thirty_two_unequal": [int(x) for x in rng.integers(0, 400, size=32)],
    }


@pytest.mark.parametrize("name", list(_lengths_cases()))
def test_inline_work_list_matches_the_prepass_bitwise(name):
    import flash_attention_varlen_b200 as fa
    lengths = _lengths_cases()[name]
    assert len(lengths) <= INLINE_MAX
    cu = workloads.cu_from_lengths(lengths).tolist()
    T = cu[-1]
    q, k, v = _qkv(T, seed=len(lengths))
    cu_inline = torch.tensor(cu, dtype=torch.int32, device="cuda")
    cu_prepass = torch.tensor(_padded(cu, INLINE_MAX + 8), dtype=torch.int32, device="cuda")
    a = fa.attn_fwd(q, k, v, cu_inline)
    fa.check_device_status()
    b = fa.attn_fwd(q, k, v, cu_prepass)
    fa.check_device_status()
    torch.cuda.synchronize()
    assert torch.isfinite(a.float()).all()
    assert torch.equal(a, b)


def test_thirty_two_and_thirty_three_segments_agree():
    """The boundary between the paths: 32 segments run inline, one more empty segment
    sends the same units through the prepass."""
    import flash_attention_varlen_b200 as fa
    rng = np.random.default_rng(11)
    lengths = [int(x) for x in rng.integers(1, 600, size=INLINE_MAX)]
    cu = workloads.cu_from_lengths(lengths).tolist()
    q, k, v = _qkv(cu[-1], seed=3, H=3)
    a = fa.attn_fwd(q, k, v, torch.tensor(cu, dtype=torch.int32, device="cuda"))
    b = fa.attn_fwd(q, k, v, torch.tensor(cu + [cu[-1]], dtype=torch.int32, device="cuda"))
    fa.check_device_status()
    torch.cuda.synchronize()
    assert torch.equal(a, b)


def test_status_alternates_per_call_over_both_paths_and_dtypes():
    import flash_attention_varlen_b200 as fa
    T = 300
    good_small = [0, 100, 300]
    bad_small = [0, 200, 100, 300]                 # a negative length
    good_large = _padded(good_small, INLINE_MAX + 4)
    bad_large = _padded([0, 100, 299], INLINE_MAX + 4)[:-1] + [301]  # cu[n] != T
    sequence = [
        (bad_small, torch.bfloat16, True),
        (good_large, torch.bfloat16, False),
        (bad_large, torch.bfloat16, True),
        (good_small, torch.bfloat16, False),
        (bad_small, torch.bfloat16, True),
        (bad_small, torch.float32, True),           # the f32 arm always runs the prepass
        (good_small, torch.bfloat16, False),
        (good_small, torch.float32, False),
        (bad_large, torch.bfloat16, True),
        (good_small, torch.bfloat16, False),
    ]
    for i, (cu, dtype, is_bad) in enumerate(sequence):
        q, k, v = _qkv(T, seed=i, H=2, dtype=dtype)
        out = torch.full_like(q, 7.0)
        fa.attn_fwd(q, k, v, torch.tensor(cu, dtype=torch.int32, device="cuda"), out=out)
        if is_bad:
            with pytest.raises(fa.VtAttnError) as e:
                fa.check_device_status()
            assert e.value.status == fa._binding.VT_ERR_BAD_SEQLENS, i
            assert torch.all(out == 7.0), i       # nothing written
        else:
            fa.check_device_status()
            assert torch.isfinite(out.float()).all() and not torch.all(out == 7.0), i

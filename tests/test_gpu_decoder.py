"""The text decoder's attention on the GPU (through the C-ABI) against its f64 oracle.

Causal attention with a local window and grouped-query heads (the Muse Glimmer next-steps
document, "Architecture / Text decoder": 32 query heads, 2 key/value heads, head size 128,
window 2048), bf16 in and out: max-abs 1e-2 and mean-abs 1e-3 against ``oracle/decoder.py``
on the same seeded inputs, the vision path's bound.  Small cases are compared element by
element; the decoder's own shape (a 4096-token sequence) on one row of every (128-row block,
query head) unit, at both ends of the block.
"""
import math

import numpy as np
import pytest

import workloads
from oracle import decoder

torch = pytest.importorskip("torch")

pytestmark = pytest.mark.gpu

BF16_MAX, BF16_MEAN = 1e-2, 1e-3


@pytest.fixture(scope="module", autouse=True)
def _need_gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from conftest import build_cuda_library
    build_cuda_library()


def _dev(a):
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).cuda()


def _run(q, k, v, cu, window, scale):
    import flash_attention_varlen_b200 as fa
    out = fa.attn_fwd_swa(_dev(q), _dev(k), _dev(v), torch.from_numpy(np.asarray(cu, np.int32)).cuda(),
                          window=window, scale=scale)
    fa.check_device_status()
    return out.float().cpu().numpy().astype(np.float64)


def _bf16_round(x):
    mag = np.maximum(np.abs(x), 2.0 ** -126)
    ulp = np.exp2(np.floor(np.log2(mag)) - 7)
    return np.round(x / ulp) * ulp


def _check(got, ref, what):
    """The bf16 bound with the output-rounding floor of the vision path: mean-abs <= 1e-3,
    and an element over 1e-2 must have |O| >= 4 (half a bf16 ulp there is 1.6e-2) or equal
    the oracle rounded to bf16 within half an ulp.  Causal rows near the start of a
    sequence average one or two keys, so |O| reaches the size of V itself."""
    assert np.all(np.isfinite(got)), f"{what}: non-finite output"
    err = np.abs(got - ref)
    assert err.mean() <= BF16_MEAN, f"{what}: mean-abs {err.mean():.3e}"
    rb = _bf16_round(ref)
    half_ulp = np.exp2(np.floor(np.log2(np.maximum(np.abs(rb), 2.0 ** -126))) - 8)
    over = err > BF16_MAX
    unexplained = over & ~((np.abs(ref) >= 4.0) | (np.abs(got - rb) <= half_ulp))
    assert not unexplained.any(), (f"{what}: max-abs {err.max():.3e}, {int(unexplained.sum())} "
                                   f"elements over {BF16_MAX} not explained by the output rounding")


@pytest.mark.parametrize("window", [0, 1, 100, 128])
def test_ragged_segments_every_element(window):
    lengths = [300, 1, 0, 700, 129, 128]
    cu = workloads.cu_from_lengths(lengths)
    T = int(cu[-1])
    q, k, v = workloads.decoder_qkv(40 + window, T, Hq=8, Hkv=2)
    scale = 1.0 / math.sqrt(128)
    got = _run(q, k, v, cu, window, scale)
    ref = decoder.attn_fwd(q, k, v, cu, scale, window)
    _check(got, ref, f"window {window}")


def test_window_one_returns_the_own_value_exactly():
    cu = workloads.cu_from_lengths([257, 3])
    q, k, v = workloads.decoder_qkv(5, 260, Hq=4, Hkv=4)
    got = _run(q, k, v, cu, 1, 0.3)
    want = workloads.bf16_bits_to_f32(v).astype(np.float64)
    assert np.array_equal(got, want)


def _unit_rows(cu, Hq, rows_per_block=128):
    """One (token, head) at each end of every (block, head) unit, alternating ends."""
    tok, head = [], []
    for s in range(len(cu) - 1):
        a0, a1 = int(cu[s]), int(cu[s + 1])
        for b0 in range(a0, a1, rows_per_block):
            b1 = min(b0 + rows_per_block, a1)
            for h in range(Hq):
                tok.append(b0 + (h % 2) * (b1 - 1 - b0))
                head.append(h)
    return np.array(tok), np.array(head)


@pytest.mark.parametrize("window", [2048, 0])
def test_decoder_shape_stratified_rows(window):
    """32 query heads over 2 key/value heads, head size 128, one 4096-token sequence."""
    cu = workloads.cu_from_lengths([4096])
    q, k, v = workloads.decoder_qkv(7, 4096)
    scale = 1.0 / math.sqrt(128)
    got = _run(q, k, v, cu, window, scale)
    tok, head = _unit_rows(cu, 32)
    ref = decoder.attn_rows(q, k, v, cu, scale, window, tok, head)
    _check(got[tok, head], ref, f"decoder 4096 window {window}")


def test_many_short_segments_and_a_negative_scale():
    rng = np.random.default_rng(3)
    lengths = [int(x) for x in rng.integers(0, 300, size=40)]
    cu = workloads.cu_from_lengths(lengths)
    T = int(cu[-1])
    q, k, v = workloads.decoder_qkv(9, T, Hq=4, Hkv=1)
    got = _run(q, k, v, cu, 64, -0.07)
    ref = decoder.attn_fwd(q, k, v, cu, -0.07, 64)
    _check(got, ref, "40 segments, window 64, scale -0.07")


@pytest.mark.parametrize("Hq,Hkv,window,seed", [(4, 4, 0, 1), (4, 4, 200, 2), (8, 2, 31, 3), (16, 1, 513, 4),
                                                 (32, 2, 2048, 5), (6, 3, 7, 6)])
def test_head_groupings_windows_and_segment_mixes(Hq, Hkv, window, seed):
    """Multi-head (Hq == Hkv) and grouped heads, windows below, across and above the tile
    size, ragged segments including length 1 and segments shorter than the window."""
    rng = np.random.default_rng(seed)
    lengths = [int(x) for x in rng.integers(1, 700, size=5)] + [1, 129, 256]
    cu = workloads.cu_from_lengths(lengths)
    T = int(cu[-1])
    q, k, v = workloads.decoder_qkv(100 + seed, T, Hq=Hq, Hkv=Hkv)
    scale = 1.0 / math.sqrt(128)
    got = _run(q, k, v, cu, window, scale)
    ref = decoder.attn_fwd(q, k, v, cu, scale, window)
    _check(got, ref, f"Hq {Hq} Hkv {Hkv} window {window}")


def test_bad_seqlens_reported_and_nothing_written():
    import flash_attention_varlen_b200 as fa
    q, k, v = workloads.decoder_qkv(11, 300, Hq=2, Hkv=1)
    out = torch.full((300, 2, 128), 7.0, dtype=torch.bfloat16, device="cuda")
    cu = torch.tensor([0, 200, 100, 300], dtype=torch.int32, device="cuda")
    fa.attn_fwd_swa(_dev(q), _dev(k), _dev(v), cu, window=16, out=out)
    with pytest.raises(fa.VtAttnError) as e:
        fa.check_device_status()
    assert e.value.status == fa._binding.VT_ERR_BAD_SEQLENS
    assert torch.all(out == 7.0)


def test_argument_errors():
    import flash_attention_varlen_b200 as fa
    b = fa._binding
    z = torch.zeros(8, 4, 128, dtype=torch.bfloat16, device="cuda")
    zk = torch.zeros(8, 3, 128, dtype=torch.bfloat16, device="cuda")
    cu = torch.tensor([0, 8], dtype=torch.int32, device="cuda")
    p = z.data_ptr()
    # Hq not a multiple of Hkv, D other than 128, negative window
    assert b.vt_attn_fwd_swa(p, zk.data_ptr(), zk.data_ptr(), p + 8192, cu.data_ptr(), 1, 8, 4, 3, 128,
                             0.1, 0, 0) == b.VT_ERR_INVALID_ARG
    assert b.vt_attn_fwd_swa(p, p, p, p + 8192, cu.data_ptr(), 1, 8, 4, 4, 64, 0.1, 0, 0) == b.VT_ERR_UNSUPPORTED
    assert b.vt_attn_fwd_swa(p, p, p, p + 8192, cu.data_ptr(), 1, 8, 4, 4, 128, 0.1, -1, 0) == b.VT_ERR_INVALID_ARG
    # out overlapping q
    assert b.vt_attn_fwd_swa(p, p, p, p, cu.data_ptr(), 1, 8, 4, 4, 128, 0.1, 0, 0) == b.VT_ERR_INVALID_ARG

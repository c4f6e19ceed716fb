"""A seeded sweep of random shapes through every forward path of the C-ABI, each compared
element by element with the f64 oracle.

For each seed: a random mix of segment lengths (empty ones, single tokens, lengths around
the 128/256-row tile and unit sizes, and a few long ones), a random head count and scale,
and for the decoder attention a random grouping of heads and window.  The bounds are the
ones every other test uses: bf16 max-abs 1e-2 with the output-rounding floor (reading 9 of
the vision tower's numerics: an element over 1e-2 needs |O| >= 4 or to equal the bf16-
rounded oracle within half an ulp) and mean-abs 1e-3; f32 max-abs 1e-5.
"""
import math

import numpy as np
import pytest

import oracle
import workloads
from oracle import decoder

torch = pytest.importorskip("torch")

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _need_gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from conftest import build_cuda_library
    build_cuda_library()


def _lengths(rng, n_max=12, long_max=1500):
    pool = [0, 1, 2, 127, 128, 129, 255, 256, 257, 383, 384, 511, 513]
    n = int(rng.integers(1, n_max + 1))
    out = []
    for _ in range(n):
        r = rng.random()
        if r < 0.4:
            out.append(int(rng.choice(pool)))
        elif r < 0.85:
            out.append(int(rng.integers(0, 600)))
        else:
            out.append(int(rng.integers(600, long_max)))
    if sum(out) == 0:
        out.append(1)
    return out


def _bf16_round(x):
    mag = np.maximum(np.abs(x), 2.0 ** -126)
    ulp = np.exp2(np.floor(np.log2(mag)) - 7)
    return np.round(x / ulp) * ulp


def _check_bf16(got, ref, what):
    assert np.all(np.isfinite(got)), f"{what}: non-finite output"
    err = np.abs(got - ref)
    assert err.mean() <= 1e-3, f"{what}: mean-abs {err.mean():.3e}"
    rb = _bf16_round(ref)
    half_ulp = np.exp2(np.floor(np.log2(np.maximum(np.abs(rb), 2.0 ** -126))) - 8)
    bad = (err > 1e-2) & ~((np.abs(ref) >= 4.0) | (np.abs(got - rb) <= half_ulp))
    assert not bad.any(), f"{what}: max-abs {err.max():.3e}, {int(bad.sum())} unexplained elements"


def _bf16_dev(a):
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).cuda()


@pytest.mark.parametrize("seed", range(8))
def test_vision_path_random_shapes(seed):
    import flash_attention_varlen_b200 as fa
    rng = np.random.default_rng(1000 + seed)
    lengths = _lengths(rng)
    cu = workloads.cu_from_lengths(lengths)
    T = int(cu[-1])
    H = int(rng.integers(1, 17))
    scale = float(rng.uniform(-0.3, 0.3))
    dtype = "f32" if seed % 4 == 3 else "bf16"
    q, k, v = workloads.qkv(2000 + seed, T, H=H, dtype=dtype)
    if dtype == "bf16":
        dq, dk, dv = _bf16_dev(q), _bf16_dev(k), _bf16_dev(v)
    else:
        dq, dk, dv = (torch.from_numpy(np.ascontiguousarray(a)).cuda() for a in (q, k, v))
    out = fa.attn_fwd(dq, dk, dv, torch.from_numpy(cu.copy()).cuda(), scale=scale)
    fa.check_device_status()
    got = out.float().cpu().numpy().astype(np.float64)
    ref = oracle.attn_fwd(q, k, v, cu, scale)
    what = f"seed {seed}: {len(lengths)} segments, T {T}, H {H}, scale {scale:.3f}, {dtype}"
    if dtype == "bf16":
        _check_bf16(got, ref, what)
    else:
        err = np.abs(got - ref)
        assert np.isfinite(got).all() and err.max() <= 1e-5, f"{what}: max-abs {err.max():.3e}"


@pytest.mark.parametrize("seed", range(8))
def test_decoder_random_shapes(seed):
    import flash_attention_varlen_b200 as fa
    rng = np.random.default_rng(3000 + seed)
    lengths = _lengths(rng, n_max=8)
    cu = workloads.cu_from_lengths(lengths)
    T = int(cu[-1])
    Hkv = int(rng.choice([1, 2, 4]))
    Hq = Hkv * int(rng.choice([1, 2, 4, 8, 16]))
    window = int(rng.choice([0, 1, 5, 64, 127, 128, 129, 300, 2048]))
    scale = float(rng.uniform(-0.15, 0.15))
    q, k, v = workloads.decoder_qkv(4000 + seed, T, Hq=Hq, Hkv=Hkv)
    out = fa.attn_fwd_swa(_bf16_dev(q), _bf16_dev(k), _bf16_dev(v), torch.from_numpy(cu.copy()).cuda(),
                          window=window, scale=scale)
    fa.check_device_status()
    got = out.float().cpu().numpy().astype(np.float64)
    ref = decoder.attn_fwd(q, k, v, cu, scale, window)
    _check_bf16(got, ref, f"seed {seed}: {len(lengths)} segments, T {T}, {Hq}/{Hkv} heads, "
                          f"window {window}, scale {scale:.3f}")

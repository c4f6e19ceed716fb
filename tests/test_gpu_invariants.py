"""Invariants of the attention definition, run through the CUDA path (C-ABI) on the GPU.

Definition (issue #1545 (vllm.cpp), "The fix"; PR #1579, "Numerics, both halves"): per
segment s, O_s = softmax(scale * Q_s K_s^T) V_s.  What that fixes, independently of any
implementation:
  * permuting the (K, V) rows of a segment together leaves O unchanged;
  * adding one constant vector c to every key of a segment leaves O unchanged (each row's
    logits move by the same scale * <q, c>);
  * V -> alpha V + beta gives O -> alpha O + beta (each softmax row sums to 1);
  * a two-key segment gives O = sigma(a1 - a2) v1 + sigma(a2 - a1) v2 (closed form).
Each transformed input is run on the GPU and compared with the oracle (or the closed form)
of the untransformed input under the usual bounds (bf16: max-abs 1e-2, mean-abs 1e-3;
f32: max-abs 1e-5).  Inputs are N(0,1) draws snapped to multiples of 1/8 in [-4, 4), so
that K + c and alpha V + beta are exact in bf16 and the transformation itself adds no
rounding.
"""
import math

import numpy as np
import pytest

import oracle
import workloads

torch = pytest.importorskip("torch")

pytestmark = pytest.mark.gpu

BF16_MAX, BF16_MEAN, F32_MAX = 1e-2, 1e-3, 1e-5
SCALE = 1.0 / math.sqrt(96)
LENGTHS = [300, 513, 77, 128]


@pytest.fixture(scope="module", autouse=True)
def _need_gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from conftest import build_cuda_library
    build_cuda_library()


def _grid_inputs(seed, T):
    q, k, v = workloads.qkv(seed, T, dtype="f32")
    snap = lambda a: np.clip(np.round(a * 8.0) / 8.0, -4.0, 3.875).astype(np.float32)
    return snap(q), snap(k), snap(v)


def _as(a, dtype):
    """f32 values on the 1/8 grid -> the kernel dtype (exact: at most 6 significant bits)."""
    a = np.ascontiguousarray(a, np.float32)
    if dtype == "f32":
        return a
    bits = a.view(np.uint32)
    assert np.all((bits & 0xFFFF) == 0)
    return (bits >> 16).astype(np.uint16)


def _run(q, k, v, cu, dtype, scale=SCALE):
    import flash_attention_varlen_b200 as fa
    if dtype == "bf16":
        to = lambda a: torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).cuda()
    else:
        to = lambda a: torch.from_numpy(np.ascontiguousarray(a, np.float32)).cuda()
    dcu = torch.from_numpy(np.ascontiguousarray(cu, np.int32)).cuda()
    out = fa.attn_fwd(to(q), to(k), to(v), dcu, scale=scale)
    fa.check_device_status()
    return out.float().cpu().numpy().astype(np.float64)


def _check(got, ref, dtype, what):
    assert np.all(np.isfinite(got)), f"{what}: non-finite output"
    err = np.abs(got - ref)
    if dtype == "bf16":
        assert err.max() <= BF16_MAX, f"{what}: max-abs {err.max():.3e}"
        assert err.mean() <= BF16_MEAN, f"{what}: mean-abs {err.mean():.3e}"
    else:
        assert err.max() <= F32_MAX, f"{what}: max-abs {err.max():.3e}"


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_kv_row_permutation_within_segments(dtype):
    cu = workloads.cu_from_lengths(LENGTHS)
    q, k, v = _grid_inputs(21, int(cu[-1]))
    rng = np.random.default_rng(21)
    perm = np.concatenate([cu[s] + rng.permutation(cu[s + 1] - cu[s]) for s in range(len(LENGTHS))])
    qd, kd, vd = _as(q, dtype), _as(k, dtype), _as(v, dtype)
    ref = oracle.attn_fwd(qd, kd, vd, cu, SCALE)
    base = _run(qd, kd, vd, cu, dtype)
    got = _run(qd, kd[perm], vd[perm], cu, dtype)
    _check(got, ref, dtype, "permuted keys vs oracle")
    _check(got, base, dtype, "permuted keys vs unpermuted run")


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_key_shift_by_a_constant_vector(dtype):
    cu = workloads.cu_from_lengths(LENGTHS)
    q, k, v = _grid_inputs(22, int(cu[-1]))
    rng = np.random.default_rng(22)
    k2 = k.copy()
    for s in range(len(LENGTHS)):  # one c per segment and head, multiples of 1/8 in [-2, 2)
        c = rng.integers(-16, 16, size=(1,) + k.shape[1:]).astype(np.float32) / 8.0
        k2[cu[s]:cu[s + 1]] += c
    qd, vd = _as(q, dtype), _as(v, dtype)
    ref = oracle.attn_fwd(qd, _as(k, dtype), vd, cu, SCALE)
    got = _run(qd, _as(k2, dtype), vd, cu, dtype)
    _check(got, ref, dtype, "shifted keys vs oracle of the unshifted input")


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("alpha,beta", [(-2.0, 0.25), (0.5, 0.125)])
def test_affine_values(dtype, alpha, beta):
    cu = workloads.cu_from_lengths(LENGTHS)
    q, k, v = _grid_inputs(23, int(cu[-1]))
    v2 = (alpha * v + beta).astype(np.float32)
    qd, kd = _as(q, dtype), _as(k, dtype)
    ref = alpha * oracle.attn_fwd(qd, kd, _as(v, dtype), cu, SCALE) + beta
    got = _run(qd, kd, _as(v2, dtype), cu, dtype)
    _check(got, ref, dtype, f"V -> {alpha} V + {beta}")


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_two_key_segments_closed_form(dtype):
    """200 segments of two keys (and a few neighbours of other lengths): the closed form,
    computed here in f64 from the exact inputs, not by the oracle."""
    lengths = [2] * 100 + [3, 1] + [2] * 100 + [5]
    cu = workloads.cu_from_lengths(lengths)
    T = int(cu[-1])
    qd, kd, vd = workloads.qkv(24, T, dtype=dtype)
    # V halved (exact in both dtypes): a two-key output is a blend of two value rows, not
    # an average of many, so with N(0,1) values |O| reaches ~4, where bf16 output rounding
    # alone (half an ulp: 7.8e-3 in [2, 4)) nearly fills the 1e-2 budget
    if dtype == "bf16":
        vd = _as(workloads.bf16_bits_to_f32(vd) * np.float32(0.5), "bf16")
    else:
        vd = (vd * np.float32(0.5)).astype(np.float32)
    f = (lambda a: workloads.bf16_bits_to_f32(a)) if dtype == "bf16" else (lambda a: a)
    q, k, v = (f(a).astype(np.float64) for a in (qd, kd, vd))
    got = _run(qd, kd, vd, cu, dtype)
    rows, ref = [], []
    for s, L in enumerate(lengths):
        if L != 2:
            continue
        j1, j2 = int(cu[s]), int(cu[s]) + 1
        for i in (j1, j2):
            a1 = SCALE * np.einsum("hd,hd->h", q[i], k[j1])
            a2 = SCALE * np.einsum("hd,hd->h", q[i], k[j2])
            w1 = 1.0 / (1.0 + np.exp(a2 - a1))
            w2 = 1.0 / (1.0 + np.exp(a1 - a2))
            rows.append(i)
            ref.append(w1[:, None] * v[j1] + w2[:, None] * v[j2])
    _check(got[rows], np.stack(ref), dtype, "two-key closed form")

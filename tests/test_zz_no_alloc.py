"""The allocation-free entry point, vt_attn_fwd_noalloc, against vt_attn_fwd (GPU).

Some callers cannot let a library allocate device memory. Their allocator may own all
of it, an allocation may add a device-wide synchronisation they must avoid, or they may
only be allowed to allocate at start-up. vt_attn_fwd_noalloc serves them: its work
list lives in a fixed array inside the library instead of a buffer the library
allocates.  Here it must give exactly what vt_attn_fwd gives (the same kernels on the
same work list) over two calls in a row (the array keeps the previous call's contents,
so the second call checks that nothing stale leaks in), and it must leave the device's
free memory unchanged on a stream vt_attn_fwd has never used.

This file sorts last so that a run stopping at the first failure has already run every
other test; it also passes on its own in a fresh process (its first call is the one
that looks up the array's device address).
"""
import math

import numpy as np
import pytest

import workloads

torch = pytest.importorskip("torch")

pytestmark = pytest.mark.gpu

BF16_MAX, BF16_MEAN, F32_MAX = 1e-2, 1e-3, 1e-5


@pytest.fixture(scope="module", autouse=True)
def _need_gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from conftest import build_cuda_library
    build_cuda_library()


def _device_inputs(case):
    q, k, v = case.inputs()
    if case.dtype == "bf16":
        to = lambda a: torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).cuda()
    else:
        to = lambda a: torch.from_numpy(np.ascontiguousarray(a)).cuda()
    cu = torch.from_numpy(case.cu_seqlens.copy()).cuda()
    return to(q), to(k), to(v), cu


def _call(fn, case, dq, dk, dv, cu, out, stream):
    import flash_attention_varlen_b200 as fa
    code = fa.VT_DTYPE_BF16 if case.dtype == "bf16" else fa.VT_DTYPE_F32
    rc = fn(dq.data_ptr(), dk.data_ptr(), dv.data_ptr(), out.data_ptr(), cu.data_ptr(),
            case.num_segments, case.T, case.H, case.D, 1.0 / math.sqrt(case.D), code,
            stream.cuda_stream)
    assert rc == 0, fa.status_string(rc)


def _check_close(got, ref, dtype):
    err = (got.double() - ref.double()).abs()
    assert torch.isfinite(got).all()
    if dtype == "bf16":
        assert err.max().item() <= BF16_MAX and err.mean().item() <= BF16_MEAN
    else:
        assert err.max().item() <= F32_MAX


def _cases():
    # all too large for vt_attn_fwd's split-key units (which the no-alloc entry point never
    # uses), so the two run the same kernel on the same work list
    return [workloads.varlen8_case(),
            workloads.Case("ragged_f32", workloads.cu_from_lengths([1, 127, 0, 129, 300, 64]),
                           seed=11, dtype="f32"),
            workloads.tower_layer_case(0)]


def test_noalloc_matches_vt_attn_fwd_on_two_calls_in_a_row():
    """Both entry points run the same kernels on the same work list, so the outputs are
    compared bit for bit (and, for the record, within the parity tolerances)."""
    from flash_attention_varlen_b200 import _binding as b
    stream = torch.cuda.current_stream()
    for case in _cases():
        dq, dk, dv, cu = _device_inputs(case)
        ref = torch.empty_like(dq)
        _call(b.vt_attn_fwd, case, dq, dk, dv, cu, ref, stream)
        first = torch.full_like(dq, float("nan"))
        second = torch.full_like(dq, float("nan"))
        _call(b.vt_attn_fwd_noalloc, case, dq, dk, dv, cu, first, stream)
        _call(b.vt_attn_fwd_noalloc, case, dq, dk, dv, cu, second, stream)
        torch.cuda.synchronize()
        assert torch.equal(first, ref), case.name
        assert torch.equal(second, ref), case.name
        _check_close(first, ref, case.dtype)


def test_noalloc_allocates_nothing_on_a_fresh_stream():
    """On a stream vt_attn_fwd has never used (so no per-stream work list exists for it),
    after one warm-up call (which may load the kernels' module), further calls leave the
    device's free memory unchanged, and the stream still has no work list of its own."""
    from flash_attention_varlen_b200 import _binding as b
    cases = _cases()
    inputs = [_device_inputs(c) for c in cases]
    outs = [torch.empty_like(x[0]) for x in inputs]
    stream = torch.cuda.Stream()
    torch.cuda.synchronize()
    for case, (dq, dk, dv, cu), out in zip(cases, inputs, outs):
        _call(b.vt_attn_fwd_noalloc, case, dq, dk, dv, cu, out, stream)
    stream.synchronize()
    free0, _ = torch.cuda.mem_get_info()
    for _ in range(3):
        for case, (dq, dk, dv, cu), out in zip(cases, inputs, outs):
            _call(b.vt_attn_fwd_noalloc, case, dq, dk, dv, cu, out, stream)
    stream.synchronize()
    free1, _ = torch.cuda.mem_get_info()
    assert free1 == free0
    # no vt_attn_fwd work list exists for this stream: its device status reads VT_OK
    assert b.vt_attn_last_device_status(stream.cuda_stream) == b.VT_OK
    for case, (dq, dk, dv, cu), out in zip(cases, inputs, outs):
        ref = torch.empty_like(dq)
        _call(b.vt_attn_fwd, case, dq, dk, dv, cu, ref, torch.cuda.current_stream())
        torch.cuda.synchronize()
        assert torch.equal(out, ref), case.name


def test_noalloc_rejects_work_lists_beyond_its_array():
    from flash_attention_varlen_b200 import _binding as b
    # 200000 one-token segments need 128 + 16 * 200000 bytes > 1 MiB: refused on the
    # host before anything is launched (the pointers below are never dereferenced).
    T = n = 200000
    cu = np.zeros(4, np.int32)
    base = 1 << 32
    stride = 1 << 30
    rc = b.vt_attn_fwd_noalloc(base, base + stride, base + 2 * stride, base + 3 * stride,
                               cu.ctypes.data, n, T, 16, 96, 0.1, b.VT_DTYPE_BF16, 0)
    assert rc == b.VT_ERR_UNSUPPORTED

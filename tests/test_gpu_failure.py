"""Failure detection on the GPU without a fault: a bounded wait is made to run out.

Every mbarrier wait in the bf16 kernel gives up after a bounded number of cycles,
raises the CTA's abort flag and records a timeout in the device status word; the other
roles then leave their loops, drain the copies they issued and release TMEM.  The
self-test entry point makes the MMA thread of every CTA wait on a barrier that nothing
arrives on, with a short limit, so this path runs on purpose.  The test checks what the
host reads afterwards (VT_ERR_DEVICE_TIMEOUT), that this costs about the limit and not a
hang, and that the context is still usable: the next forward on the same stream is
correct and reports VT_OK.
"""
import math
import time

import numpy as np
import pytest

import oracle
import workloads

torch = pytest.importorskip("torch")

pytestmark = pytest.mark.gpu

STALL_CYCLES = 1 << 21  # ~1 ms at B200 clocks


@pytest.fixture(scope="module", autouse=True)
def _need_gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from conftest import build_cuda_library
    build_cuda_library()


def _device_inputs(case):
    q, k, v = case.inputs()
    to = lambda a: torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).cuda()
    return to(q), to(k), to(v), torch.from_numpy(case.cu_seqlens.copy()).cuda()


@pytest.mark.parametrize("make_case", [workloads.tiny_case, lambda: workloads.image896_cases()[1],
                                       lambda: workloads.image896_cases()[0]],
                         ids=["tiny256", "img896_full", "img896_window"])
def test_wait_timeout_is_reported_and_context_survives(make_case):
    import flash_attention_varlen_b200 as fa
    from flash_attention_varlen_b200 import _binding as b
    case = make_case()
    dq, dk, dv, cu = _device_inputs(case)
    out = torch.empty_like(dq)
    stream = torch.cuda.current_stream().cuda_stream
    scale = 1.0 / math.sqrt(case.D)
    torch.cuda.synchronize()

    t0 = time.perf_counter()
    rc = b.vt_attn_selftest_wait_timeout(dq.data_ptr(), dk.data_ptr(), dv.data_ptr(), out.data_ptr(),
                                         cu.data_ptr(), case.num_segments, case.T, case.H, case.D,
                                         scale, STALL_CYCLES, stream)
    assert rc == b.VT_OK, b.status_string(rc)
    status = b.vt_attn_last_device_status(stream)
    elapsed = time.perf_counter() - t0
    assert status == b.VT_ERR_DEVICE_TIMEOUT, b.status_string(status)
    assert elapsed < 5.0  # the limit is ~1 ms; anything near the 2^32-cycle default means a role hung

    # the context is intact and the status is per call: a normal forward is correct again
    rc = b.vt_attn_fwd(dq.data_ptr(), dk.data_ptr(), dv.data_ptr(), out.data_ptr(), cu.data_ptr(),
                       case.num_segments, case.T, case.H, case.D, scale, b.VT_DTYPE_BF16, stream)
    assert rc == b.VT_OK, b.status_string(rc)
    assert b.vt_attn_last_device_status(stream) == b.VT_OK
    got = out.float().cpu().numpy().astype(np.float64)
    q, k, v = case.inputs()
    ref = oracle.attn_fwd(q, k, v, case.cu_seqlens, scale)
    err = np.abs(got - ref)
    assert np.isfinite(got).all()
    assert err.max() <= 1e-2 and err.mean() <= 1e-3

"""Host-side checks of the C-ABI library that need no GPU.

The library must load, export every entry point ``include/vt_attn.h``
declares, and reject bad arguments on the host before touching a device.
Only calls that fail host validation are made here, so nothing is launched.
"""
import ctypes
import os
import re

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def binding():
    from conftest import build_cuda_library
    build_cuda_library()
    from flash_attention_varlen_b200 import _binding
    return _binding


def _declared_functions():
    src = open(os.path.join(ROOT, "include", "vt_attn.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(vt_\w+)\s*\(", src)))


def test_exports_every_declared_symbol(binding):
    declared = _declared_functions()
    assert declared, "no declarations parsed"
    assert sorted(binding.EXPORTED) == declared
    for name in declared:
        assert hasattr(binding.lib, name), name
    # and the names are real dynamic symbols of the .so
    out = os.popen(f"nm -D --defined-only {binding.LIB_PATH}").read()
    for name in declared:
        assert re.search(rf"\bT {name}\b", out), name


def _cu(arr):
    a = np.ascontiguousarray(arr, dtype=np.int32)
    return a, a.ctypes.data


def test_validate_seqlens_host(binding):
    ok = binding.VT_OK
    bad = binding.VT_ERR_BAD_SEQLENS
    a, p = _cu([0, 5, 5, 12])
    assert binding.vt_attn_validate_seqlens_host(p, 3, 12) == ok
    a, p = _cu([0])
    assert binding.vt_attn_validate_seqlens_host(p, 0, 0) == ok
    for arr, n, T in (([1, 5], 1, 5), ([0, 5], 1, 6), ([0, 6, 5, 9], 3, 9), ([0, 3], 1, 3)):
        a, p = _cu(arr)
        want = ok if (arr == [0, 3]) else bad
        assert binding.vt_attn_validate_seqlens_host(p, n, T) == want
    assert binding.vt_attn_validate_seqlens_host(None, 1, 1) == binding.VT_ERR_NULL
    a, p = _cu([0, 4])
    assert binding.vt_attn_validate_seqlens_host(p, -1, 4) == bad


def test_smem_contract(binding):
    b = binding.vt_attn_smem_bytes(96, binding.VT_DTYPE_BF16)
    f = binding.vt_attn_smem_bytes(96, binding.VT_DTYPE_F32)
    # bf16: a double buffer of two 128 x 96 bf16 Q tiles, 2-stage K and V rings (each V
    # stage with its ones chunk), barriers and 1 KB alignment slack; must fit the 227 KB
    # per-CTA opt-in limit of sm_100
    assert 8 * 128 * 96 * 2 < b <= 232448
    # f32: the three bf16 parts of a 128 x 96 Q tile and of 64 x 96 K and V tiles, barriers
    # and the alignment slack
    assert 3 * 128 * 96 * 2 + 6 * 64 * 96 * 2 < f <= 232448
    assert binding.vt_attn_smem_bytes(64, binding.VT_DTYPE_BF16) == 0
    assert binding.vt_attn_smem_bytes(96, 7) == 0


def test_workspace_bytes(binding):
    # header (128 B) + 16 B per entry; entries = sum_s ceil(L_s / rows) <= floor((T + n (rows - 1)) / rows)
    assert binding.vt_attn_workspace_bytes(16, 16384, binding.VT_DTYPE_BF16) == 128 + 16 * ((16384 + 16 * 255) // 256)
    assert binding.vt_attn_workspace_bytes(1, 256, binding.VT_DTYPE_F32) == 128 + 16 * 2
    assert binding.vt_attn_workspace_bytes(1, 1024, binding.VT_DTYPE_BF16) == 128 + 16 * 4
    assert binding.vt_attn_workspace_bytes(-1, 5, binding.VT_DTYPE_BF16) == 0


def test_status_strings_and_version(binding):
    for code in range(7):
        s = binding.status_string(code)
        assert s.startswith("VT_")
    assert binding.status_string(99) == "unknown vt_status"
    assert binding.vt_attn_version() >= 100


def test_fwd_rejects_bad_arguments_on_host(binding):
    f = binding.vt_attn_fwd
    cu, cup = _cu([0, 4])
    P = 4096  # fake, 16-byte aligned, never dereferenced: every call below fails host checks
    BF, F32 = binding.VT_DTYPE_BF16, binding.VT_DTYPE_F32
    assert f(P, P, P, P * 16, cup, 1, 4, 16, 64, 0.1, BF, 0) == binding.VT_ERR_UNSUPPORTED
    assert f(P, P, P, P * 16, cup, 1, 4, 16, 96, 0.1, 5, 0) == binding.VT_ERR_INVALID_ARG
    assert f(P, P, P, P * 16, cup, 1, 4, 0, 96, 0.1, BF, 0) == binding.VT_ERR_INVALID_ARG
    assert f(P, P, P, P * 16, cup, 1, 4, 16, 96, float("nan"), BF, 0) == binding.VT_ERR_INVALID_ARG
    assert f(P, P, P, P * 16, cup, 1, 4, 16, 96, float("inf"), F32, 0) == binding.VT_ERR_INVALID_ARG
    assert f(P, P, P, P * 16, cup, -1, 4, 16, 96, 0.1, BF, 0) == binding.VT_ERR_INVALID_ARG
    # no segments: fine with no tokens, inconsistent otherwise
    assert f(0, 0, 0, 0, 0, 0, 0, 16, 96, 0.1, BF, 0) == binding.VT_OK
    assert f(0, 0, 0, 0, 0, 0, 8, 16, 96, 0.1, BF, 0) == binding.VT_ERR_BAD_SEQLENS
    # all segments empty: no work, no launch
    assert f(0, 0, 0, 0, cup, 3, 0, 16, 96, 0.1, BF, 0) == binding.VT_OK
    assert f(P, P, P, P * 16, 0, 1, 4, 16, 96, 0.1, BF, 0) == binding.VT_ERR_NULL
    assert f(0, P, P, P * 16, cup, 1, 4, 16, 96, 0.1, BF, 0) == binding.VT_ERR_NULL
    # misaligned pointers and aliasing of out with an input
    assert f(P + 2, P, P, P * 16, cup, 1, 4, 16, 96, 0.1, BF, 0) == binding.VT_ERR_INVALID_ARG
    assert f(P, P * 8, P * 12, P + 64, cup, 1, 4, 16, 96, 0.1, BF, 0) == binding.VT_ERR_INVALID_ARG


def test_python_wrapper_refuses_cpu_tensors(binding):
    import torch
    from flash_attention_varlen_b200 import attn_fwd
    q = torch.zeros(4, 16, 96, dtype=torch.bfloat16)
    cu = torch.tensor([0, 4], dtype=torch.int32)
    with pytest.raises(ValueError):
        attn_fwd(q, q, q, cu)


def test_selftest_wait_timeout_rejects_bad_arguments_on_host(binding):
    f = binding.vt_attn_selftest_wait_timeout
    cu, cup = _cu([0, 4])
    P = 4096  # fake, never dereferenced: every call below fails a host check first
    # the stall must be positive, and a kernel must actually run
    assert f(P, P, P, P * 16, cup, 1, 4, 16, 96, 0.1, 0, 0) == binding.VT_ERR_INVALID_ARG
    assert f(P, P, P, P * 16, cup, 1, 4, 16, 96, 0.1, -5, 0) == binding.VT_ERR_INVALID_ARG
    assert f(0, 0, 0, 0, 0, 0, 0, 16, 96, 0.1, 1000, 0) == binding.VT_ERR_INVALID_ARG
    # then the forward's own checks apply
    assert f(P, P, P, P * 16, cup, 1, 4, 16, 64, 0.1, 1000, 0) == binding.VT_ERR_UNSUPPORTED
    assert f(P, P, P, P * 16, 0, 1, 4, 16, 96, 0.1, 1000, 0) == binding.VT_ERR_NULL
    assert f(P + 2, P, P, P * 16, cup, 1, 4, 16, 96, 0.1, 1000, 0) == binding.VT_ERR_INVALID_ARG


def test_window_count_on_host(binding):
    import ctypes
    def count(grids, win):
        flat = [x for hw in grids for x in hw]
        g = (ctypes.c_int32 * len(flat))(*flat)
        nw, nt = ctypes.c_int32(-1), ctypes.c_int32(-1)
        rc = binding.vt_window_count(ctypes.addressof(g), len(grids), win, ctypes.addressof(nw),
                                     ctypes.addressof(nt))
        return rc, nw.value, nt.value
    assert count([(128, 128)], 32) == (binding.VT_OK, 16, 16384)
    assert count([(40, 50)], 32) == (binding.VT_OK, 4, 2000)
    assert count([(8, 8), (13, 29), (64, 33), (1, 1)], 8) == (binding.VT_OK, 1 + 8 + 40 + 1, 64 + 377 + 2112 + 1)
    assert count([(0, 5)], 32)[0] == binding.VT_ERR_INVALID_ARG
    assert count([(5, 5)], 0)[0] == binding.VT_ERR_INVALID_ARG
    assert count([(1, 1)] * 65, 32)[0] == binding.VT_ERR_UNSUPPORTED
    assert binding.vt_window_count(0, 1, 32, 0, 0) == binding.VT_ERR_NULL
    # the device calls check their arguments on the host first
    assert binding.vt_permute_rows(4096, 8192, 256, 4, 24, 0, 0) == binding.VT_ERR_INVALID_ARG  # row_bytes % 16
    assert binding.vt_permute_rows(4096, 8192, 256, 4, 32, 2, 0) == binding.VT_ERR_INVALID_ARG  # scatter flag
    assert binding.vt_permute_rows(4096, 4096 + 64, 256, 4, 32, 0, 0) == binding.VT_ERR_INVALID_ARG  # overlap
    assert binding.vt_permute_rows(0, 8192, 256, 4, 32, 0, 0) == binding.VT_ERR_NULL
    assert binding.vt_permute_rows(0, 0, 0, 0, 32, 0, 0) == binding.VT_OK  # nothing to move


def test_window_wrappers_validate_on_host(binding):
    import torch
    import flash_attention_varlen_b200 as fa
    with pytest.raises(ValueError):
        fa.window_partition([])                      # no images
    with pytest.raises(fa.VtAttnError):
        fa.window_partition([(0, 4)])                # empty grid, refused by vt_window_count
    with pytest.raises(fa.VtAttnError):
        fa.window_partition([(4, 4)], win=0)
    x = torch.zeros(4, 16, dtype=torch.float32)
    perm = torch.arange(4, dtype=torch.int32)
    with pytest.raises(ValueError):
        fa.permute_rows(x, perm)                     # CPU tensors: the library is GPU-only


def test_split_keys_option_round_trips(binding):
    """vt_attn_set_split_keys is host state only: it returns the previous setting."""
    prev = binding.vt_attn_set_split_keys(0)
    try:
        assert prev in (0, 1)
        assert binding.vt_attn_set_split_keys(1) == 0
        assert binding.vt_attn_set_split_keys(7) == 1  # any non-zero enables
    finally:
        binding.vt_attn_set_split_keys(prev)

"""Window segmentation on the GPU: the device-built order against the oracle (bit-exact),
the row gather/scatter against numpy indexing (bit-exact), and a window layer run from
image-order tensors end to end against the oracle's window attention."""
import math

import numpy as np
import pytest

import workloads
from oracle.window import window_attention, window_permutation

torch = pytest.importorskip("torch")

pytestmark = pytest.mark.gpu

GRIDS = [
    ([(128, 128)], 32),                          # the tower's 16384-token image
    ([(64, 64)], 32),
    ([(40, 50)], 32),                            # ragged edges
    ([(8, 8), (13, 29), (64, 33), (1, 1)], 8),   # several images, small windows
    (workloads.varlen_image_grids(0), 32),       # the eight-image varlen batch
]


@pytest.fixture(scope="module", autouse=True)
def _need_gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from conftest import build_cuda_library
    build_cuda_library()


@pytest.mark.parametrize("grids,win", GRIDS, ids=["tower128", "img64", "ragged40x50", "multi8", "varlen8"])
def test_partition_matches_oracle(grids, win):
    import flash_attention_varlen_b200 as fa
    perm, cu = fa.window_partition(grids, win)
    torch.cuda.synchronize()
    p_ref, cu_ref = window_permutation(grids, win)
    assert np.array_equal(perm.cpu().numpy(), p_ref)
    assert np.array_equal(cu.cpu().numpy(), cu_ref)


@pytest.mark.parametrize("dtype,row", [(torch.bfloat16, (16, 96)), (torch.float32, (16, 96)), (torch.float32, (4,))])
def test_permute_rows_gather_and_scatter(dtype, row):
    import flash_attention_varlen_b200 as fa
    grids = [(40, 50), (13, 29)]
    perm, _ = fa.window_partition(grids, 32)
    T = perm.numel()
    g = torch.Generator().manual_seed(7)
    x = torch.randn((T,) + row, generator=g).to(dtype).cuda()
    y = fa.permute_rows(x, perm)
    back = fa.permute_rows(y, perm, inverse=True)
    torch.cuda.synchronize()
    p = perm.cpu().long()
    assert torch.equal(y.cpu(), x.cpu()[p])        # bit-exact gather
    assert torch.equal(back.cpu(), x.cpu())        # scatter undoes it


@pytest.mark.parametrize("grids", [[(64, 64)], [(40, 50), (24, 24)]], ids=["img64", "ragged"])
def test_window_layer_from_image_order(grids):
    import flash_attention_varlen_b200 as fa
    T = sum(h * w for h, w in grids)
    q, k, v = workloads.qkv(3, T)
    to = lambda a: torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).cuda()
    dq, dk, dv = to(q), to(k), to(v)
    perm, cu = fa.window_partition(grids, 32)
    ow = fa.attn_fwd(fa.permute_rows(dq, perm), fa.permute_rows(dk, perm), fa.permute_rows(dv, perm), cu)
    o = fa.permute_rows(ow, perm, inverse=True)
    fa.check_device_status()
    got = o.float().cpu().numpy().astype(np.float64)
    ref = window_attention(q, k, v, grids, 1.0 / math.sqrt(96), 32)
    err = np.abs(got - ref)
    assert np.isfinite(got).all()
    assert err.max() <= 1e-2 and err.mean() <= 1e-3

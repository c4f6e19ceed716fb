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


@pytest.mark.parametrize("inverse", [False, True], ids=["gather", "scatter"])
def test_permute_rows_skips_out_of_range_indexes(inverse):
    """index lives on the device, so the kernel checks it: rows whose index is outside
    [0, T) are skipped before any access (no fault) and reported by the check call;
    every other row moves exactly as numpy indexing says."""
    import flash_attention_varlen_b200 as fa
    from flash_attention_varlen_b200 import _binding as b
    T = 1000
    fa.check_permute_rows()  # start from a clear flag
    g = torch.Generator().manual_seed(3)
    p = torch.randperm(T, generator=g).to(torch.int32)
    bad_rows = [5, 611, 999]
    p[5], p[611], p[999] = T, -1, 2 ** 31 - 1
    x = torch.randn(T, 16, 96, generator=g).to(torch.bfloat16).cuda()
    out = torch.full_like(x, 3.0)
    fa.permute_rows(x, p.cuda(), inverse=inverse, out=out)
    with pytest.raises(fa.VtAttnError) as e:
        fa.check_permute_rows()
    assert e.value.status == b.VT_ERR_BAD_INDEX
    fa.check_permute_rows()  # reading cleared the flag
    got, xs = out.cpu(), x.cpu()
    good = [i for i in range(T) if i not in bad_rows]
    pl = p.long()
    if inverse:
        assert torch.equal(got[pl[good]], xs[good])
        untouched = sorted(set(range(T)) - set(pl[good].tolist()))
        assert untouched and torch.all(got[untouched] == 3.0)
    else:
        assert torch.equal(got[good], xs[pl[good]])
        assert torch.all(got[bad_rows] == 3.0)
    # a valid permutation afterwards reports nothing
    fa.permute_rows(x, torch.randperm(T, generator=g).to(torch.int32).cuda(), inverse=inverse)
    fa.check_permute_rows()

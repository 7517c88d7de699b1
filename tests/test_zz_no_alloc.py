"""mxq_quant_error_noalloc: the error metric for callers that cannot allocate
device memory, checked against mxq_quant_error (which takes a caller workspace).

Through the C ABI, two calls in a row, with and without smoothing.  This file is
collected last (its name sorts last) and also passes alone in a fresh process."""
import ctypes

import numpy as np
import pytest
import torch

import mxfp4_block_rotation_b200 as mxq
from workloads import synth

pytestmark = pytest.mark.gpu

DEV = "cuda:0"
P = ctypes.c_void_p


@pytest.fixture(scope="module", autouse=True)
def _lib(cuda_device):
    from mxfp4_block_rotation_b200 import build
    build.build()
    yield


def _ptr(t):
    return None if t is None else P(t.data_ptr())


def _noalloc(x, r, lam, err, mean):
    L = mxq.lib()
    return L.mxq_quant_error_noalloc(_ptr(x), x.shape[0], x.shape[1], _ptr(r), _ptr(lam), _ptr(err), _ptr(mean),
                                     P(torch.cuda.current_stream().cuda_stream))


@pytest.mark.parametrize("rows,cols,with_lam", [(300, 4096, False), (257, 2048, True), (8192, 14336, False)])
def test_noalloc_matches_workspace_entry_point_twice(rows, cols, with_lam):
    w = synth.make_config(3, rows=rows, cols=cols)
    x, r = w.x.to(DEV), synth.rhat_tensor(synth.haar_orthogonal(rows)).to(DEV)
    lam = synth.random_lambda(cols, seed=4).to(DEV) if with_lam else None
    ref_err, ref_mean = mxq.quant_error(x, r, lam)
    torch.cuda.synchronize()
    for _ in range(2):   # the shared array keeps the last call's contents; each call must stand alone
        err = torch.full((rows, cols // 32), float("nan"), dtype=torch.float32, device=DEV)
        mean = torch.full((), float("nan"), dtype=torch.float64, device=DEV)
        assert _noalloc(x, r, lam, err, mean) == 0, mxq.lib().mxq_last_cuda_error()
        mxq.sync_check()
        e, re_ = err.cpu().numpy().astype(np.float64), ref_err.cpu().numpy().astype(np.float64)
        assert np.all(np.abs(e - re_) <= 1e-5 + 1e-4 * re_)
        assert abs(mean.item() - ref_mean.item()) <= 1e-4 * abs(ref_mean.item()) + 1e-7


def test_noalloc_rejects_sizes_beyond_its_scratch():
    x = torch.zeros((128, 64), dtype=torch.bfloat16, device=DEV)
    r = synth.rhat_tensor(np.eye(32)).to(DEV)
    mean = torch.zeros((), dtype=torch.float64, device=DEV)
    L = mxq.lib()
    # 65536 x 8256 is 16,908,288 groups: 131,072 groups (256 stages of 512) past the 16,777,216
    # the array covers; refused before anything is launched
    st = L.mxq_quant_error_noalloc(_ptr(x), 65536, 8256, _ptr(r), None, None, _ptr(mean),
                                   P(torch.cuda.current_stream().cuda_stream))
    assert st == 1 and b"scratch" in L.mxq_last_cuda_error()


@pytest.mark.parametrize("rows,cols,with_lam", [(65536, 8192, False), (16384, 16384, True)])
def test_noalloc_exactly_at_its_limit(rows, cols, with_lam):
    """The largest inputs the array covers: 65536 x 8192 is exactly 16,777,216 groups of 32;
    with Lambda, 16384 x 16384 is exactly 128 row tiles x 256 column tiles = 32,768 tiles of
    four partial sums.  Both must run and agree with the workspace entry point."""
    g = torch.Generator(device=DEV)
    g.manual_seed(rows + cols)
    x = torch.randn((rows, cols), generator=g, device=DEV, dtype=torch.float32).to(torch.bfloat16)
    r = synth.rhat_tensor(synth.haar_orthogonal(11)).to(DEV)
    lam = synth.random_lambda(cols, seed=12).to(DEV) if with_lam else None
    L = mxq.lib()
    assert L.mxq_quant_error_workspace_bytes(rows, cols, int(with_lam)) == 131072 * 8
    ref_err, ref_mean = mxq.quant_error(x, r, lam)
    err = torch.full((rows, cols // 32), float("nan"), dtype=torch.float32, device=DEV)
    mean = torch.full((), float("nan"), dtype=torch.float64, device=DEV)
    assert _noalloc(x, r, lam, err, mean) == 0, L.mxq_last_cuda_error()
    mxq.sync_check()
    assert torch.equal(err, ref_err)   # the same kernel on the same input: the same bits
    assert abs(mean.item() - ref_mean.item()) <= 1e-12 * abs(ref_mean.item())

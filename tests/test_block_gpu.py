"""GPU parity of the rotation-block-size variants (DuQuant++ write-up, §4.3: B = 16, 64, 128)
with the oracle, through the C ABI.

The same parity rule as the main path: scales and codes bit-exact outside the
rounding bands, neighbours inside them, at most 1e-5 of the elements
excused; exact cases (identity, permutations) bit-exact with no exceptions;
the fp32 rotated values within 2e-3 relative (floor 1e-3 of the group absmax).
"""
import numpy as np
import pytest
import scipy.linalg
import torch

import mxfp4_block_rotation_b200 as mxq
import oracle
from tests import _parity
from workloads import synth

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda:0")


def _rb(r):
    return synth.bf16_bits(synth.rhat_tensor(r))


def _hadamard(n):
    h = np.array([[1.0]])
    while h.shape[0] < n:
        h = np.block([[h, h], [h, -h]])
    return h / np.sqrt(n)


def _mats(blk):
    perm = np.eye(blk)[np.random.default_rng(blk).permutation(blk)]
    return {"haar": synth.haar_orthogonal(100 + blk, n=blk), "hadamard": _hadamard(blk), "identity": np.eye(blk),
            "perm": perm}


def _gpu(xb, rb, lam):
    x = synth.bf16_from_bits(xb).to(DEV)
    r = synth.bf16_from_bits(rb).to(DEV)
    lt = None if lam is None else torch.from_numpy(np.ascontiguousarray(lam, np.float32)).to(DEV)
    codes, scales = mxq.rotate_quantize_block(x, r, lt)
    y = mxq.rotate_block_f32(x, r, lt)
    mxq.sync_check()
    return codes.cpu().numpy(), scales.cpu().numpy(), y.cpu().numpy()


def _check(xb, rb, lam, exact=False):
    c, s, y = _gpu(xb, rb, lam)
    ref = oracle.block_rotate_quantize(xb, rb, lam, want_y=True, flags=True, threads=oracle.default_threads())
    res = _parity.check_quant(xb, None, lam, c, s, exact=exact, ref=ref)
    _parity.check_f32(ref["y"], y)
    return res


SHAPES = [(1, 128), (3, 256), (129, 384), (257, 1024), (1000, 640)]


@pytest.mark.parametrize("blk", [16, 64, 128])
@pytest.mark.parametrize("rows,cols", SHAPES)
def test_block_matches_oracle(blk, rows, cols):
    if cols % blk:
        pytest.skip("cols not a multiple of the block")
    xb = synth.bf16_bits(synth.make_config(2, rows=rows, cols=cols).x)
    mats = _mats(blk)
    for name in ("haar", "hadamard"):
        _check(xb, _rb(mats[name]), None)
    for name in ("identity", "perm"):
        _check(xb, _rb(mats[name]), None, exact=True)


@pytest.mark.parametrize("rows,cols", [(5, 64), (300, 512)])
def test_block16_with_lambda(rows, cols):
    xb = synth.bf16_bits(synth.make_config(2, rows=rows, cols=cols).x)
    lam = synth.random_lambda(cols, seed=rows).numpy()
    _check(xb, _rb(synth.haar_orthogonal(16, n=16)), lam)
    # the block-diagonal 32x32 matrix on the main entry point gives the same bits
    r16 = (synth.bf16_bits(synth.rhat_tensor(synth.haar_orthogonal(16, n=16))).astype(np.uint32) << 16).view(
        np.float32).astype(np.float64)
    big = _rb(scipy.linalg.block_diag(r16, r16))
    x = synth.bf16_from_bits(xb).to(DEV)
    lt = torch.from_numpy(lam).to(DEV)
    a = mxq.rotate_quantize_block(x, synth.bf16_from_bits(_rb(r16)).to(DEV), lt)
    b = mxq.smooth_rotate_quantize(x, synth.bf16_from_bits(big).to(DEV), lt)
    assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1])


def test_block_rejects_bad_arguments():
    x = torch.zeros((4, 96), dtype=torch.bfloat16, device=DEV)
    with pytest.raises(mxq.MxqError):
        mxq.rotate_quantize_block(x, torch.eye(64, dtype=torch.bfloat16, device=DEV))       # 96 % 64
    with pytest.raises(mxq.MxqError):
        mxq.rotate_quantize_block(x, torch.eye(48, dtype=torch.bfloat16, device=DEV))       # block 48
    x = torch.zeros((4, 128), dtype=torch.bfloat16, device=DEV)
    with pytest.raises(mxq.MxqError):
        mxq.rotate_quantize_block(x, torch.eye(64, dtype=torch.bfloat16, device=DEV),
                                  torch.ones(128, dtype=torch.float32, device=DEV))           # Λ with 64
    e = torch.zeros((0, 128), dtype=torch.bfloat16, device=DEV)
    c, s = mxq.rotate_quantize_block(e, torch.eye(128, dtype=torch.bfloat16, device=DEV))
    assert c.numel() == 0 and s.numel() == 0


@pytest.mark.parametrize("blk", [64, 128])
def test_block_full_downproj(blk):
    # 8192 x 14336 down-projection activations, sampled rows (first, last, planted outliers, seeded)
    w = synth.make_config(3)
    rb = _rb(synth.haar_orthogonal(200 + blk, n=blk))
    x = w.x.to(DEV)
    codes, scales = mxq.rotate_quantize_block(x, synth.bf16_from_bits(rb).to(DEV))
    mxq.sync_check()
    rows_s = synth.sample_rows(w.rows, 96, seed=7100 + blk, must=w.outlier_rows)
    idx = torch.from_numpy(rows_s).to(DEV)
    xs = synth.bf16_bits(w.x[torch.from_numpy(rows_s)])
    ref = oracle.block_rotate_quantize(xs, rb, None, want_y=True, flags=True, threads=oracle.default_threads())
    _parity.check_quant(xs, None, None, codes.index_select(0, idx).cpu().numpy(),
                        scales.index_select(0, idx).cpu().numpy(), ref=ref)
    assert int(scales.max().item()) < 0xFF

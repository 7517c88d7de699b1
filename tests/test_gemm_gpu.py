"""GPU parity of the MXFP4 consumer GEMM and the weights' side of the absorption
(DuQuant++ write-up, §3.3) with the oracle, through the C ABI.

GEMM rule: |Y_gpu - Y| <= 1e-5 * sum_k |a_k b_k| element-wise.  The tensor cores
accumulate in fp32 over K/64 MMAs, so the error is bounded by about K/64 fp32
roundings of partial sums no larger than sum |a b|.  Where every partial sum is
exactly representable in fp32 (unit scales, small integer multiples of 1/4), the
result must be bit-exact.  bf16 output: the fp32 rule plus one bf16 rounding.
"""
import numpy as np
import pytest
import torch

import mxfp4_block_rotation_b200 as mxq
import oracle
from tests import _parity
from workloads import synth

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda:0")


def _rand_mx(rng, rows, K, lo=118, hi=136):
    return (rng.integers(0, 256, (rows, K // 2), dtype=np.uint8),
            rng.integers(lo, hi, (rows, K // 32), dtype=np.uint8))


def _abs_codes(c):
    return c & 0x77   # clear both nibbles' sign bits


def _gpu_gemm(a, sa, b, sb, out_dtype=torch.float32):
    t = [torch.from_numpy(np.ascontiguousarray(v)).to(DEV) for v in (a, sa, b, sb)]
    y = mxq.mxfp4_gemm(*t, out_dtype=out_dtype)
    mxq.sync_check()
    return y.float().cpu().numpy().astype(np.float64)


def _check_gemm(a, sa, b, sb, exact=False, rel=1e-5):
    th = oracle.default_threads()
    ref = oracle.mxfp4_gemm(a, sa, b, sb, threads=th)
    mag = oracle.mxfp4_gemm(_abs_codes(a), sa, _abs_codes(b), sb, threads=th)
    got = _gpu_gemm(a, sa, b, sb)
    if exact:
        assert np.array_equal(got, ref)
    else:
        err = np.abs(got - ref)
        bad = ~(err <= rel * mag)
        assert not bad.any(), f"{bad.sum()} elements off; first at {np.argwhere(bad)[0]}"
    gb = _gpu_gemm(a, sa, b, sb, torch.bfloat16)
    assert (np.abs(gb - ref) <= rel * mag + 2.0 ** -8 * np.abs(ref)).all()
    return ref


@pytest.mark.parametrize("M,N,K", [(128, 256, 256), (1, 1, 32), (129, 257, 288), (300, 520, 1024),
                                   (256, 512, 4096), (64, 1000, 96)])
def test_gemm_matches_oracle(M, N, K):
    rng = np.random.default_rng(M + 7 * N + 13 * K)
    a, sa = _rand_mx(rng, M, K)
    b, sb = _rand_mx(rng, N, K)
    _check_gemm(a, sa, b, sb)


def test_gemm_several_tiles_per_pair():
    # 9 x 9 = 81 tiles of 256 x 256 on at most 74 CTA pairs: some pairs take a second tile, so
    # the accumulator's empty/full phases turn over; ragged M and N edges, K not a multiple of 256
    M, N, K = 2300, 2250, 800
    rng = np.random.default_rng(11)
    a, sa = _rand_mx(rng, M, K)
    b, sb = _rand_mx(rng, N, K)
    _check_gemm(a, sa, b, sb)


@pytest.mark.parametrize("M,N,K", [(128, 256, 512), (200, 300, 2048)])
def test_gemm_exact_with_unit_scales(M, N, K):
    # scale 2^0: every product is a multiple of 1/4 below 36, every partial sum an exact fp32
    rng = np.random.default_rng(K)
    a = rng.integers(0, 256, (M, K // 2), dtype=np.uint8)
    b = rng.integers(0, 256, (N, K // 2), dtype=np.uint8)
    sa = np.full((M, K // 32), 127, np.uint8)
    sb = np.full((N, K // 32), 127, np.uint8)
    _check_gemm(a, sa, b, sb, exact=True)


def test_gemm_per_block_scales_and_nan():
    rng = np.random.default_rng(5)
    M, N, K = 130, 260, 640
    a, sa = _rand_mx(rng, M, K, 100, 154)     # scales spread over 2^-27 .. 2^26
    b, sb = _rand_mx(rng, N, K, 100, 154)
    _check_gemm(a, sa, b, sb)
    sa[7, 3] = 0xFF                            # E8M0 NaN: row 7 of Y is NaN
    got = _gpu_gemm(a, sa, b, sb)
    assert np.isnan(got[7]).all() and not np.isnan(np.delete(got, 7, 0)).any()


def test_gemm_empty_and_bad_arguments():
    z = torch.zeros((0, 16), dtype=torch.uint8, device=DEV)
    zs = torch.zeros((0, 1), dtype=torch.uint8, device=DEV)
    b = torch.zeros((5, 16), dtype=torch.uint8, device=DEV)
    bs = torch.zeros((5, 1), dtype=torch.uint8, device=DEV)
    assert mxq.mxfp4_gemm(z, zs, b, bs).shape == (0, 5)
    e = torch.zeros((3, 0), dtype=torch.uint8, device=DEV)
    y = mxq.mxfp4_gemm(e, e, e[:2], e[:2])      # K = 0: the empty sum
    mxq.sync_check()
    assert y.shape == (3, 2) and (y == 0).all()
    buf = torch.empty(5 * 5 + 1, dtype=torch.float32, device=DEV)
    with pytest.raises(mxq.MxqError):
        mxq.mxfp4_gemm(b, bs, b, bs, out=buf[1:].view(5, 5))                  # output not 16-B aligned


@pytest.mark.parametrize("use_lam", [False, True])
def test_weight_side_matches_oracle(use_lam):
    rows, cols = 300, 1024
    wt = synth.random_bf16(rows, cols, seed=41, scale=0.05)
    rhat = synth.rhat_tensor(synth.haar_orthogonal(9))
    lam = synth.random_lambda(cols, seed=3) if use_lam else None
    c, s = mxq.weight_rotate_quantize(wt.to(DEV), rhat.to(DEV), None if lam is None else lam.to(DEV))
    mxq.sync_check()
    wb, rb = synth.bf16_bits(wt), synth.bf16_bits(rhat)
    lm = None if lam is None else lam.numpy()
    ref = oracle.weight_rotate_quantize(wb, rb, lm, want_y=True, flags=True, threads=oracle.default_threads())
    _parity.check_quant(wb, rb, lm, c.cpu().numpy(), s.cpu().numpy(), ref=ref)


def test_chain_downproj_full_size():
    # The layer end to end on the 8192 x 14336 down-projection activations and a synthetic
    # 4096 x 14336 weight (N(0, 1/K)): X -> MXFP4(X Λ⁻¹ R̂), Wᵀ -> MXFP4(Wᵀ Λ R̂), then the GEMM.
    # Sampled rows of Y against the oracle GEMM of the GPU's own operands, and the weight codes
    # against the oracle's weight quantiser on sampled rows.
    w = synth.make_config(3)
    K, N = w.cols, 4096
    wt = synth.random_bf16(N, K, seed=77, scale=1.0 / np.sqrt(K))
    lam = synth.smoothing_scale(w.x)
    rhat = w.rhat.to(DEV)
    ca, sa = mxq.smooth_rotate_quantize(w.x.to(DEV), rhat, lam.to(DEV))
    cb, sb = mxq.weight_rotate_quantize(wt.to(DEV), rhat, lam.to(DEV))
    y = mxq.mxfp4_gemm(ca, sa, cb, sb)
    mxq.sync_check()
    rows_s = synth.sample_rows(w.rows, 48, seed=8100, must=w.outlier_rows)
    idx = torch.from_numpy(rows_s).to(DEV)
    a_s, sa_s = ca.index_select(0, idx).cpu().numpy(), sa.index_select(0, idx).cpu().numpy()
    b_np, sb_np = cb.cpu().numpy(), sb.cpu().numpy()
    th = oracle.default_threads()
    ref = oracle.mxfp4_gemm(a_s, sa_s, b_np, sb_np, threads=th)
    mag = oracle.mxfp4_gemm(_abs_codes(a_s), sa_s, _abs_codes(b_np), sb_np, threads=th)
    got = y.index_select(0, idx).cpu().numpy().astype(np.float64)
    assert (np.abs(got - ref) <= 1e-5 * mag).all()
    wrows = synth.sample_rows(N, 64, seed=8200)
    wb = synth.bf16_bits(wt[torch.from_numpy(wrows)])
    refw = oracle.weight_rotate_quantize(wb, synth.bf16_bits(w.rhat), lam.numpy(), want_y=True, flags=True,
                                         threads=th)
    _parity.check_quant(wb, None, None, cb.index_select(0, torch.from_numpy(wrows).to(DEV)).cpu().numpy(),
                        sb.index_select(0, torch.from_numpy(wrows).to(DEV)).cpu().numpy(), ref=refw)


@pytest.mark.parametrize("rows,K", [(1, 32), (300, 416), (128, 4096), (4096, 14336)])
def test_scale_layout_matches_oracle(rows, K):
    rng = np.random.default_rng(rows + K)
    sc = rng.integers(0, 256, (rows, K // 32), dtype=np.uint8)
    got = mxq.scales_to_mma_layout(torch.from_numpy(sc).to(DEV))
    mxq.sync_check()
    assert np.array_equal(got.cpu().numpy(), oracle.scales_to_mma(sc))

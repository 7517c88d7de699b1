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
    #  - both GPU quantisers against the oracle's (parity rule) on sampled rows;
    #  - the GPU GEMM on the oracle's operands (uploaded) against the oracle GEMM of them;
    #  - the GPU chain (its own operands) equals that GEMM bit for bit wherever its operands
    #    equal the oracle's.  The oracle never takes GPU output.
    w = synth.make_config(3)
    K, N = w.cols, 4096
    wt = synth.random_bf16(N, K, seed=77, scale=1.0 / np.sqrt(K))
    lam = synth.smoothing_scale(w.x)
    rhat = w.rhat.to(DEV)
    ca, sa = mxq.smooth_rotate_quantize(w.x.to(DEV), rhat, lam.to(DEV))
    cb, sb = mxq.weight_rotate_quantize(wt.to(DEV), rhat, lam.to(DEV))
    y_chain = mxq.mxfp4_gemm(ca, sa, cb, sb)
    mxq.sync_check()
    th = oracle.default_threads()
    rows_s = synth.sample_rows(w.rows, 48, seed=8100, must=w.outlier_rows)
    idx = torch.from_numpy(rows_s)
    xs = synth.bf16_bits(w.x[idx])
    qa = oracle.smooth_rotate_quantize(xs, synth.bf16_bits(w.rhat), lam.numpy(), want_y=True, flags=True, threads=th)
    qb = oracle.weight_rotate_quantize(synth.bf16_bits(wt), synth.bf16_bits(w.rhat), lam.numpy(), want_y=True,
                                       flags=True, threads=th)
    ga, gsa = ca.index_select(0, idx.to(DEV)).cpu().numpy(), sa.index_select(0, idx.to(DEV)).cpu().numpy()
    gb, gsb = cb.cpu().numpy(), sb.cpu().numpy()
    _parity.check_quant(xs, None, None, ga, gsa, ref=qa)
    wrows = synth.sample_rows(N, 64, seed=8200)
    _parity.check_quant(synth.bf16_bits(wt[torch.from_numpy(wrows)]), None, None, gb[wrows], gsb[wrows],
                        ref={k: v[wrows] for k, v in qb.items()})
    # the GEMM on the oracle's operands
    ops = [torch.from_numpy(np.ascontiguousarray(v)).to(DEV) for v in (qa["codes"], qa["scales"], qb["codes"],
                                                                       qb["scales"])]
    y_o = mxq.mxfp4_gemm(*ops)
    mxq.sync_check()
    ref = oracle.mxfp4_gemm(qa["codes"], qa["scales"], qb["codes"], qb["scales"], threads=th)
    mag = oracle.mxfp4_gemm(_abs_codes(qa["codes"]), qa["scales"], _abs_codes(qb["codes"]), qb["scales"], threads=th)
    got = y_o.cpu().numpy().astype(np.float64)
    assert (np.abs(got - ref) <= 1e-5 * mag).all()
    # the chain where its operands are the oracle's
    row_ok = (ga == qa["codes"]).all(1) & (gsa == qa["scales"]).all(1)
    col_ok = (gb == qb["codes"]).all(1) & (gsb == qb["scales"]).all(1)
    assert row_ok.mean() > 0.5 and col_ok.mean() > 0.5
    chain = y_chain.index_select(0, idx.to(DEV)).cpu().numpy()
    assert np.array_equal(chain[row_ok][:, col_ok], y_o.cpu().numpy()[row_ok][:, col_ok])


@pytest.mark.parametrize("rows,K", [(1, 32), (300, 416), (128, 4096), (4096, 14336)])
def test_scale_layout_matches_oracle(rows, K):
    rng = np.random.default_rng(rows + K)
    sc = rng.integers(0, 256, (rows, K // 32), dtype=np.uint8)
    got = mxq.scales_to_mma_layout(torch.from_numpy(sc).to(DEV))
    mxq.sync_check()
    assert np.array_equal(got.cpu().numpy(), oracle.scales_to_mma(sc))


@pytest.mark.parametrize("rows,cols,use_lam", [(300, 2048, False), (300, 2048, True), (129, 96, False),
                                               (129, 96, True), (37, 16416, False), (40, 16416, True),
                                               (256, 4096, False), (1, 32, False), (1, 32, True),
                                               (128, 128, True)])
def test_quantize_with_mma_scales(rows, cols, use_lam):
    # The quantiser writing its scales straight into the MMA layout.  The buffer is poisoned
    # first, so every byte must be written: the scales where the oracle's layout function puts
    # the row-major call's scales, and 0 in the padding (rows past a multiple of 128, groups
    # past a multiple of 4).  The codes equal the row-major call's, and both calls' output
    # meets the quantiser's parity rule against the oracle.  Shapes cover the flat kernel
    # (no Lambda, G < 128 and odd G) and the column-tiled one (a last tile of one group).
    x = synth.random_bf16(rows, cols, seed=rows * 7 + cols, scale=1.0)
    rhat = synth.rhat_tensor(synth.haar_orthogonal(rows + 1))
    lam = synth.random_lambda(cols, seed=rows) if use_lam else None
    xd, rd, ld = x.to(DEV), rhat.to(DEV), None if lam is None else lam.to(DEV)
    c0, s0 = mxq.smooth_rotate_quantize(xd, rd, ld)
    n = int(mxq.lib().mxq_scales_mma_bytes(rows, cols))
    sf = torch.full((n,), 0xAB, dtype=torch.uint8, device=DEV)
    c1, sf1 = mxq.smooth_rotate_quantize_mma(xd, rd, ld, sf=sf)
    mxq.sync_check()
    assert torch.equal(c1, c0)
    s0n = s0.cpu().numpy()
    assert np.array_equal(sf1.cpu().numpy(), oracle.scales_to_mma(s0n))
    _parity.check_quant(synth.bf16_bits(x), synth.bf16_bits(rhat), None if lam is None else lam.numpy(),
                        c1.cpu().numpy(), s0n)


@pytest.mark.parametrize("rows,cols,use_lam", [(300, 2048, False), (300, 2048, True), (129, 96, False),
                                               (129, 96, True), (37, 16416, False), (40, 16416, True),
                                               (1, 32, False), (1, 32, True)])
def test_nvfp4_quantize_with_mma_scales(rows, cols, use_lam):
    # NVFP4 with its E4M3 scales written straight into the MMA layout: as for MXFP4, on a
    # poisoned buffer, against the oracle's layout of the row-major call's scales (the same
    # atoms over [rows, cols/16]), codes equal, both against the oracle's NVFP4 quantiser.
    x = synth.random_bf16(rows, cols, seed=rows * 5 + cols, scale=1.0)
    rhat = synth.rhat_tensor(synth.haar_orthogonal(rows + 2))
    lam = synth.random_lambda(cols, seed=rows + 1) if use_lam else None
    xd, rd, ld = x.to(DEV), rhat.to(DEV), None if lam is None else lam.to(DEV)
    s_t = float(np.float32(float(x.abs().max().float()) * 32 ** 0.5 * (20.0 if use_lam else 1.0) / (6 * 448)))
    ts = torch.tensor([s_t], dtype=torch.float32, device=DEV)
    c0, s0 = mxq.smooth_rotate_quantize_nvfp4(xd, rd, ts, ld)
    n = int(mxq.lib().mxq_nvfp4_scales_mma_bytes(rows, cols))
    sf = torch.full((n,), 0xAB, dtype=torch.uint8, device=DEV)
    c1, sf1 = mxq.smooth_rotate_quantize_nvfp4_mma(xd, rd, ts, ld, sf=sf)
    mxq.sync_check()
    assert torch.equal(c1, c0)
    s0n = s0.cpu().numpy()
    assert np.array_equal(sf1.cpu().numpy(), oracle.scales_to_mma(s0n))
    _parity.check_nvfp4(synth.bf16_bits(x), synth.bf16_bits(rhat), None if lam is None else lam.numpy(), s_t,
                        c1.cpu().numpy(), s0n)


def test_gemm_on_mma_scales_equals_layout_pass():
    # The layer without the layout pass gives the same output bits as with it.
    rows, cols, n_out = 300, 1024, 520
    x = synth.random_bf16(rows, cols, seed=5, scale=1.0)
    wt = synth.random_bf16(n_out, cols, seed=6, scale=1.0 / np.sqrt(cols))
    rhat = synth.rhat_tensor(synth.haar_orthogonal(12)).to(DEV)
    lam = synth.random_lambda(cols, seed=13).to(DEV)
    cb, sb = mxq.weight_rotate_quantize(wt.to(DEV), rhat, lam)
    for lam_a in (None, lam):
        c0, s0 = mxq.smooth_rotate_quantize(x.to(DEV), rhat, lam_a)
        c1, sf1 = mxq.smooth_rotate_quantize_mma(x.to(DEV), rhat, lam_a)
        y0 = mxq.mxfp4_gemm(c0, mxq.scales_to_mma_layout(s0), cb, sb)
        y1 = mxq.mxfp4_gemm(c1, sf1, cb, sb)
        mxq.sync_check()
        assert torch.equal(y0, y1)
    # NVFP4: the same with E4M3 scales and tensor scales
    ts_a = torch.tensor([float(x.abs().max().float()) * 32 ** 0.5 / (6 * 448)], dtype=torch.float32, device=DEV)
    ts_b = torch.tensor([float(wt.abs().max().float()) * 32 ** 0.5 / (6 * 448)], dtype=torch.float32, device=DEV)
    ncb, nsb = mxq.smooth_rotate_quantize_nvfp4(wt.to(DEV), rhat, ts_b)
    nc0, ns0 = mxq.smooth_rotate_quantize_nvfp4(x.to(DEV), rhat, ts_a)
    nc1, nsf1 = mxq.smooth_rotate_quantize_nvfp4_mma(x.to(DEV), rhat, ts_a)
    y0 = mxq.nvfp4_gemm(nc0, ns0, ts_a, ncb, nsb, ts_b)
    y1 = mxq.nvfp4_gemm(nc1, nsf1, ts_a, ncb, nsb, ts_b)
    mxq.sync_check()
    assert torch.equal(y0, y1)


# ---------------------------------------------------------------- the NVFP4 consumer GEMM

def _rand_nv(rng, rows, K):
    # E4M3 scale codes in [0x20, 0x48): normal values 2^-3 .. 2^2
    return (rng.integers(0, 256, (rows, K // 2), dtype=np.uint8),
            rng.integers(0x20, 0x48, (rows, K // 16), dtype=np.uint8))


def _gpu_nv(a, sa, ta, b, sb, tb, out_dtype=torch.float32):
    t = [torch.from_numpy(np.ascontiguousarray(v)).to(DEV) for v in (a, sa, b, sb)]
    ts = [torch.tensor([v], dtype=torch.float32, device=DEV) for v in (ta, tb)]
    y = mxq.nvfp4_gemm(t[0], t[1], ts[0], t[2], t[3], ts[1], out_dtype=out_dtype)
    mxq.sync_check()
    return y.float().cpu().numpy().astype(np.float64)


def _check_nv(a, sa, ta, b, sb, tb, exact=False, rel=1e-5):
    th = oracle.default_threads()
    ref = oracle.nvfp4_gemm(a, sa, ta, b, sb, tb, threads=th)
    mag = oracle.nvfp4_gemm(_abs_codes(a), sa, abs(ta), _abs_codes(b), sb, abs(tb), threads=th)
    got = _gpu_nv(a, sa, ta, b, sb, tb)
    if exact:
        assert np.array_equal(got, ref)
    else:
        bad = ~(np.abs(got - ref) <= rel * mag)
        assert not bad.any(), f"{bad.sum()} elements off; first at {np.argwhere(bad)[0]}"
    gb = _gpu_nv(a, sa, ta, b, sb, tb, torch.bfloat16)
    assert (np.abs(gb - ref) <= rel * mag + 2.0 ** -8 * np.abs(ref)).all()


@pytest.mark.parametrize("M,N,K", [(128, 256, 256), (1, 1, 32), (129, 257, 288), (300, 520, 1024), (64, 1000, 96),
                                   (2300, 2250, 800)])
def test_nvfp4_gemm_matches_oracle(M, N, K):
    rng = np.random.default_rng(M + 3 * N + 17 * K)
    a, sa = _rand_nv(rng, M, K)
    b, sb = _rand_nv(rng, N, K)
    _check_nv(a, sa, 0.37, b, sb, 1.9)


def test_nvfp4_gemm_exact_with_unit_scales():
    rng = np.random.default_rng(2)
    M, N, K = 200, 300, 2048
    a = rng.integers(0, 256, (M, K // 2), dtype=np.uint8)
    b = rng.integers(0, 256, (N, K // 2), dtype=np.uint8)
    one = 0x38   # E4M3 1.0
    _check_nv(a, np.full((M, K // 16), one, np.uint8), 1.0, b, np.full((N, K // 16), one, np.uint8), 1.0, exact=True)


def test_nvfp4_gemm_nan_scale_and_bad_arguments():
    rng = np.random.default_rng(3)
    a, sa = _rand_nv(rng, 8, 64)
    b, sb = _rand_nv(rng, 8, 64)
    sa[1, 2] = 0x7F
    got = _gpu_nv(a, sa, 1.0, b, sb, 1.0)
    assert np.isnan(got[1]).all() and not np.isnan(np.delete(got, 1, axis=0)).any()
    t = [torch.from_numpy(v).to(DEV) for v in (a, sa, b, sb)]
    one = torch.ones(1, dtype=torch.float32, device=DEV)
    with pytest.raises(ValueError):
        mxq.nvfp4_gemm(t[0], t[1], torch.ones(2, dtype=torch.float32, device=DEV), t[2], t[3], one)
    # a tensor scale in host memory is refused before any launch
    sfa = mxq.nvfp4_scales_to_mma_layout(t[1])
    sfb = mxq.nvfp4_scales_to_mma_layout(t[3])
    y = torch.empty((8, 8), dtype=torch.float32, device=DEV)
    host = torch.ones(1, dtype=torch.float32)
    rc = mxq.lib().mxq_nvfp4_gemm(t[0].data_ptr(), sfa.data_ptr(), host.data_ptr(), t[2].data_ptr(), sfb.data_ptr(),
                                  one.data_ptr(), 8, 8, 64, y.data_ptr(), 0, None)
    assert rc == 1


def test_nvfp4_chain():
    # NVFP4(X R̂) and NVFP4(Wᵀ R̂) by the GPU quantiser, against the oracle's; the GPU GEMM on the
    # oracle's operands against the oracle GEMM; the GPU chain equals it where its operands do
    rows, K, N = 1024, 4096, 512
    w = synth.make_config(2, rows=rows, cols=K)
    wt = synth.random_bf16(N, K, seed=78, scale=1.0 / np.sqrt(K))
    th = oracle.default_threads()
    xb, wb, rb = synth.bf16_bits(w.x), synth.bf16_bits(wt), synth.bf16_bits(w.rhat)
    ya = oracle.nvfp4_quantize(xb, rb, None, 1.0, want_y=True, threads=th)["y"]
    yb = oracle.nvfp4_quantize(wb, rb, None, 1.0, want_y=True, threads=th)["y"]
    ta = float(np.float32(np.abs(ya).max() / (6 * 448)))
    tb = float(np.float32(np.abs(yb).max() / (6 * 448)))
    qa = oracle.nvfp4_quantize(xb, rb, None, ta, want_y=True, flags=True, threads=th)
    qb = oracle.nvfp4_quantize(wb, rb, None, tb, want_y=True, flags=True, threads=th)
    tta = torch.tensor([ta], dtype=torch.float32, device=DEV)
    ttb = torch.tensor([tb], dtype=torch.float32, device=DEV)
    ca, sa = mxq.smooth_rotate_quantize_nvfp4(w.x.to(DEV), w.rhat.to(DEV), tta)
    cb, sb = mxq.smooth_rotate_quantize_nvfp4(wt.to(DEV), w.rhat.to(DEV), ttb)
    y_chain = mxq.nvfp4_gemm(ca, sa, tta, cb, sb, ttb)
    mxq.sync_check()
    ga, gsa, gb, gsb = (v.cpu().numpy() for v in (ca, sa, cb, sb))
    _parity.check_nvfp4(xb, rb, None, ta, ga, gsa)
    _parity.check_nvfp4(wb, rb, None, tb, gb, gsb)
    ops = [torch.from_numpy(v).to(DEV) for v in (qa["codes"], qa["scales"], qb["codes"], qb["scales"])]
    y_o = mxq.nvfp4_gemm(ops[0], ops[1], tta, ops[2], ops[3], ttb)
    mxq.sync_check()
    ref = oracle.nvfp4_gemm(qa["codes"], qa["scales"], ta, qb["codes"], qb["scales"], tb, threads=th)
    mag = oracle.nvfp4_gemm(_abs_codes(qa["codes"]), qa["scales"], ta, _abs_codes(qb["codes"]), qb["scales"], tb,
                            threads=th)
    assert (np.abs(y_o.cpu().numpy().astype(np.float64) - ref) <= 1e-5 * mag).all()
    row_ok = (ga == qa["codes"]).all(1) & (gsa == qa["scales"]).all(1)
    col_ok = (gb == qb["codes"]).all(1) & (gsb == qb["scales"]).all(1)
    assert row_ok.mean() > 0.5 and col_ok.mean() > 0.5
    assert np.array_equal(y_chain.cpu().numpy()[row_ok][:, col_ok], y_o.cpu().numpy()[row_ok][:, col_ok])
    # and the layer approximates X Wᵀ (R̂ orthogonal): relative Frobenius error of NVFP4 x NVFP4
    xw = synth.bf16_bits(w.x).astype(np.uint32)
    xf = (xw << 16).view(np.float32).astype(np.float64)
    wf = (synth.bf16_bits(wt).astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    exact = xf @ wf.T
    rel = np.linalg.norm(y_chain.cpu().numpy() - exact) / np.linalg.norm(exact)
    assert rel < 0.25

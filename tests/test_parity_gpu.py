"""Parity of the CUDA path (through the C ABI) with the CPU oracle, on the GPU.

Small cases span several 128x128 tiles and ragged row/column tails; every
output element is compared.  Full-size cases run the same launch as the
benchmark and compare a seeded sample of rows (plus the first, last and
planted-outlier rows) element by element.
"""
import math

import numpy as np
import pytest
import torch

import mxfp4_block_rotation_b200 as mxq
import oracle
from tests import _parity
from workloads import synth

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


def _bits(t):
    return synth.bf16_bits(t.cpu())


def _gpu_quant(x, rhat, lam=None):
    xd = x.to(DEV)
    rd = rhat.to(DEV)
    ld = None if lam is None else lam.to(DEV)
    codes, scales = mxq.smooth_rotate_quantize(xd, rd, ld)
    torch.cuda.synchronize()
    mxq.sync_check()
    return codes.cpu().numpy(), scales.cpu().numpy()


def _check(x, rhat, lam=None, exact=False):
    codes, scales = _gpu_quant(x, rhat, lam)
    return _parity.check_quant(_bits(x), _bits(rhat), None if lam is None else lam.numpy(), codes, scales,
                               exact=exact)


@pytest.fixture(scope="module", autouse=True)
def _device(cuda_device):
    from mxfp4_block_rotation_b200 import build
    build.build()
    yield


# ---------------------------------------------------------------- shapes and tails

SHAPES = [(1, 32), (3, 64), (5, 96), (127, 128), (128, 160), (129, 256), (300, 4096), (257, 14336),
          (64, 8192), (200, 1056), (1000, 224)]


@pytest.mark.parametrize("rows,cols", SHAPES)
def test_shapes_random_rotation(rows, cols):
    x = synth.random_bf16(rows, cols, seed=rows * 7 + cols, scale=2.0)
    r = synth.rhat_tensor(synth.haar_orthogonal(rows + cols))
    _check(x, r)


@pytest.mark.parametrize("kind", ["identity", "neg_identity", "permutation", "hadamard", "qr"])
def test_rotation_kinds(kind):
    rows, cols = 259, 1024
    x = synth.random_bf16(rows, cols, seed=17, scale=3.0)
    mats = {"identity": np.eye(32), "neg_identity": -np.eye(32), "permutation": synth.permutation_rhat(3),
            "hadamard": synth.hadamard_rhat(4), "qr": synth.haar_orthogonal(5)}
    exact = kind in ("identity", "neg_identity", "permutation")   # y is exact on both sides
    _check(x, synth.rhat_tensor(mats[kind]), exact=exact)


@pytest.mark.parametrize("kind", ["ones", "pow2", "loguniform", "smoothquant"])
def test_lambda_variants(kind):
    rows, cols = 300, 2048
    x = synth.random_bf16(rows, cols, seed=23, scale=4.0)
    r = synth.rhat_tensor(synth.haar_orthogonal(6))
    if kind == "ones":
        lam = torch.ones(cols, dtype=torch.float32)
    elif kind == "pow2":
        lam = torch.from_numpy((2.0 ** np.random.default_rng(1).integers(-6, 7, size=cols)).astype(np.float32))
    elif kind == "loguniform":
        lam = synth.random_lambda(cols, seed=2)
    else:
        lam = synth.smoothing_scale(x)
    res = _check(x, r, lam)
    if kind == "ones":   # Λ = 1 must be bit-identical to no smoothing
        c0, s0 = _gpu_quant(x, r)
        c1, s1 = _gpu_quant(x, r, lam)
        assert np.array_equal(c0, c1) and np.array_equal(s0, s1)
    assert res["elements"] == rows * cols


def test_exact_midpoints_identity():
    # with R^ = I the rotated values are the inputs themselves: every E2M1 midpoint tie,
    # saturation, negative zero and tiny negatives must come out exactly as the oracle says
    mags = [0.0, 0.25, 0.5, 0.75, 1.0, 1.25, 1.5, 1.75, 2.0, 2.5, 3.0, 3.5, 4.0, 5.0, 6.0, 0.1, 0.3, 0.7,
            1.1, 2.2, 4.4, 5.5, 5.9, 3.9, 0.01]
    rows = []
    for k in (-130, -126, -60, -3, 0, 7, 60, 120):
        for sgn in (1.0, -1.0):
            row = np.array([(mags[i % len(mags)]) * sgn * 2.0 ** k for i in range(64)])
            row[0] = 6.0 * 2.0 ** k       # set the scale: amax 6 * 2^k -> byte k + 127
            row[33] = 4.0 * 2.0 ** k
            rows.append(row)
    zero = np.zeros(64)
    negz = -np.zeros(64)
    rows += [zero, negz]
    x = synth.to_bf16(np.array(rows))
    _check(x, synth.rhat_tensor(np.eye(32)), exact=True)


def test_special_groups():
    rows, cols = 130, 256
    x = synth.random_bf16(rows, cols, seed=31).float().numpy().astype(np.float64)
    x[0, :] = 0.0                         # all-zero groups -> byte 0, codes 0
    x[1, 32:64] = 1e-40                   # subnormal-range values -> byte 0
    x[2, 64:96] = 3.0e38                  # near the bf16/fp32 top (identity keeps it finite)
    x[3, :32] = -0.0
    x[4, 96:128] = np.nan
    x[5, 128:160] = np.inf
    x[6, 160] = -np.inf
    xt = synth.to_bf16(x)
    c, s = _gpu_quant(xt, synth.rhat_tensor(np.eye(32)))
    _parity.check_quant(_bits(xt), _bits(synth.rhat_tensor(np.eye(32))), None, c, s, exact=True)
    assert s[4, 3] == 0xFF and s[5, 4] == 0xFF and s[6, 5] == 0xFF
    assert not c[4, 48:64].any()
    assert s[0].max() == 0 and s[1, 1] == 0


def test_rotated_values_fp32_within_tolerance():
    for lam in (None, synth.random_lambda(1024, seed=9)):
        x = synth.make_config(3, rows=257, cols=1024).x
        r = synth.rhat_tensor(synth.haar_orthogonal(11))
        y = mxq.smooth_rotate_f32(x.to(DEV), r.to(DEV), None if lam is None else lam.to(DEV)).cpu().numpy()
        ref = oracle.smooth_rotate_quantize(_bits(x), _bits(r), None if lam is None else lam.numpy(),
                                            want_y=True)["y"]
        err = _parity.check_f32(ref, y)
        assert err < 2e-3
        if lam is None:
            # without smoothing only fp32 accumulation differs: far tighter than the bound
            assert np.abs(y - ref).max() <= 1e-5 * np.abs(ref).max()


def test_guard_bands_untouched():
    rows, cols = 131, 256
    x = synth.random_bf16(rows, cols, seed=41).to(DEV)
    r = synth.rhat_tensor(synth.haar_orthogonal(12)).to(DEV)
    nc, ns = rows * cols // 2, rows * cols // 32
    pad = 4096
    cbuf = torch.full((nc + 2 * pad,), 0xA5, dtype=torch.uint8, device=DEV)
    sbuf = torch.full((ns + 2 * pad,), 0x5A, dtype=torch.uint8, device=DEV)
    codes = cbuf[pad:pad + nc].view(rows, cols // 2)
    scales = sbuf[pad:pad + ns].view(rows, cols // 32)
    mxq.smooth_rotate_quantize(x, r, codes=codes, scales=scales)
    torch.cuda.synchronize()
    assert bool((cbuf[:pad] == 0xA5).all()) and bool((cbuf[pad + nc:] == 0xA5).all())
    assert bool((sbuf[:pad] == 0x5A).all()) and bool((sbuf[pad + ns:] == 0x5A).all())
    # odd scale offset (not 4-byte aligned) takes the byte-store path and must agree
    sbuf2 = torch.full((ns + 2 * pad + 1,), 0x5A, dtype=torch.uint8, device=DEV)
    scales2 = sbuf2[pad + 1:pad + 1 + ns].view(rows, cols // 32)
    codes2 = torch.empty_like(codes)
    mxq.smooth_rotate_quantize(x, r, codes=codes2, scales=scales2)
    torch.cuda.synchronize()
    assert torch.equal(scales2, scales) and torch.equal(codes2, codes)
    assert bool((sbuf2[:pad + 1] == 0x5A).all()) and bool((sbuf2[pad + 1 + ns:] == 0x5A).all())


def test_deterministic_and_stream_ordered():
    x = synth.random_bf16(512, 4096, seed=5).to(DEV)
    r = synth.rhat_tensor(synth.haar_orthogonal(13)).to(DEV)
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        a = mxq.smooth_rotate_quantize(x, r)
        b = mxq.smooth_rotate_quantize(x, r)
    s.synchronize()
    assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1])


def test_empty_inputs():
    x = torch.empty((0, 64), dtype=torch.bfloat16, device=DEV)
    r = synth.rhat_tensor(np.eye(32)).to(DEV)
    c, s = mxq.smooth_rotate_quantize(x, r)
    assert c.shape == (0, 32) and s.shape == (0, 2)
    out = mxq.dequantize(c, s)
    assert out.shape == (0, 64)


def test_rejects_host_memory():
    import ctypes
    L = mxq.lib()
    x = torch.zeros((4, 64), dtype=torch.bfloat16)           # pageable host memory
    r = synth.rhat_tensor(np.eye(32)).to(DEV)
    c = torch.empty((4, 32), dtype=torch.uint8, device=DEV)
    s = torch.empty((4, 2), dtype=torch.uint8, device=DEV)
    P = ctypes.c_void_p
    st = L.mxq_smooth_rotate_quantize(P(x.data_ptr()), 4, 64, P(r.data_ptr()), None, P(c.data_ptr()),
                                      P(s.data_ptr()), None)
    assert st == 1
    xp = x.pin_memory()                                         # pinned host memory is refused too
    st = L.mxq_smooth_rotate_quantize(P(xp.data_ptr()), 4, 64, P(r.data_ptr()), None, P(c.data_ptr()),
                                      P(s.data_ptr()), None)
    assert st == 1


def test_bounded_wait_reports_timeout():
    mxq.sync_check()                                  # clean slate
    assert mxq.selftest_bounded_wait(timeout_ms=30) == 2
    with pytest.raises(mxq.MxqError) as ei:
        mxq.sync_check()
    assert ei.value.status == 4
    mxq.sync_check()                                  # cleared; the context is still usable
    x = synth.random_bf16(128, 128, seed=1).to(DEV)
    mxq.smooth_rotate_quantize(x, synth.rhat_tensor(np.eye(32)).to(DEV))
    mxq.sync_check()


# ---------------------------------------------------------------- dequantize

def _synthetic_codes(rows, cols, seed):
    rng = np.random.default_rng(seed)
    codes = rng.integers(0, 256, size=(rows, cols // 2), dtype=np.uint8)
    scales = rng.integers(100, 155, size=(rows, cols // 32), dtype=np.uint8)
    return codes, scales


def test_dequant_plain_bit_exact():
    rows, cols = 257, 1056
    codes, scales = _synthetic_codes(rows, cols, seed=3)
    scales[0, :6] = [0, 1, 252, 253, 254, 255]      # subnormal, overflow and NaN scales
    ref = oracle.dequantize(codes, scales, cols)
    got = mxq.dequantize(torch.from_numpy(codes).to(DEV), torch.from_numpy(scales).to(DEV))
    got = synth.bf16_bits(got.cpu())
    ref_nan = np.isnan(_parity.bf16_to_f64(ref))
    got_nan = np.isnan(_parity.bf16_to_f64(got))
    assert np.array_equal(ref_nan, got_nan)
    assert np.array_equal(ref[~ref_nan], got[~got_nan])


# Lambda kinds: resident in shared memory (16-byte aligned, G <= 512), or fetched per warp
# (G > 512, or Lambda only 4-byte aligned); a few groups per row make the row index wrap often
@pytest.mark.parametrize("rows,cols,lam_kind", [(300, 2048, None), (300, 2048, "aligned"), (300, 2048, "offset"),
                                                (40, 16416, "aligned"), (37, 16384, "aligned"), (129, 96, "aligned"),
                                                (129, 96, "offset")])
def test_dequant_inverse_rotation(rows, cols, lam_kind):
    codes, scales = _synthetic_codes(rows, cols, seed=4)
    r = synth.rhat_tensor(synth.haar_orthogonal(14))
    lam = synth.random_lambda(cols, seed=5) if lam_kind else None
    ref_bits, ref64 = oracle.dequantize(codes, scales, cols, _bits(r), None if lam is None else lam.numpy(),
                                        want_f64=True)
    lam_dev = None
    if lam_kind == "aligned":
        lam_dev = lam.to(DEV)
    elif lam_kind == "offset":
        lam_dev = torch.cat([torch.zeros(1), lam]).to(DEV)[1:]   # 4-byte but not 16-byte aligned
        assert lam_dev.data_ptr() % 16 != 0
    got = mxq.dequantize(torch.from_numpy(codes).to(DEV), torch.from_numpy(scales).to(DEV), r.to(DEV), lam_dev)
    got64 = _parity.bf16_to_f64(synth.bf16_bits(got.cpu()))
    # bound: one bf16 ulp of the exact value plus fp32 accumulation error of 32 terms
    v = _parity.bf16_to_f64(oracle.dequantize(codes, scales, cols))
    rr = _parity.bf16_to_f64(_bits(r))
    s_abs = (np.abs(v).reshape(rows, cols // 32, 32) @ np.abs(rr).T).reshape(rows, cols)
    if lam is not None:
        s_abs = s_abs * lam.numpy()[None, :]
    tol = 2.0 ** -7 * np.abs(ref64) + 2.0 ** -18 * s_abs
    assert (np.abs(got64 - ref64) <= tol).all()
    # most outputs round to the same bf16 as the exact value
    assert (got64 == _parity.bf16_to_f64(ref_bits)).mean() > 0.99


# ---------------------------------------------------------------- full-size configurations

def _full_config(cfg, n_sample=192):
    w = synth.make_config(cfg)
    xd = w.x.to(DEV)
    rd = w.rhat.to(DEV)
    ld = None if w.lam is None else w.lam.to(DEV)
    codes, scales = mxq.smooth_rotate_quantize(xd, rd, ld)
    mxq.sync_check()
    rows_s = synth.sample_rows(w.rows, n_sample, seed=7000 + cfg, must=w.outlier_rows)
    idx = torch.from_numpy(rows_s).to(DEV)
    c = codes.index_select(0, idx).cpu().numpy()
    s = scales.index_select(0, idx).cpu().numpy()
    xs = synth.bf16_bits(w.x[torch.from_numpy(rows_s)])
    res = _parity.check_quant(xs, _bits(w.rhat), None if w.lam is None else w.lam.numpy(), c, s)
    # properties over the whole output: no NaN scales for finite inputs, every scale in range
    assert int(scales.max().item()) < 0xFF
    return w, xd, rd, ld, codes, scales, rows_s, res


@pytest.mark.parametrize("cfg", [1, 2, 3, 4])
def test_full_config(cfg):
    w, *_ = _full_config(cfg)
    torch.cuda.empty_cache()


def test_full_config5_with_round_trip():
    w, xd, rd, ld, codes, scales, rows_s, res = _full_config(5)
    back = mxq.dequantize(codes, scales, rd, ld)
    mxq.sync_check()
    idx = torch.from_numpy(rows_s).to(DEV)
    got = _parity.bf16_to_f64(synth.bf16_bits(back.index_select(0, idx).cpu()))
    ref = res["ref"]
    ref_back_bits, ref_back = oracle.dequantize(ref["codes"], ref["scales"], w.cols, _bits(w.rhat),
                                                w.lam.numpy(), want_f64=True)
    # compare where the GPU's codes and scales equal the oracle's (elsewhere a boundary tie differs)
    gc = codes.index_select(0, idx).cpu().numpy()
    gs = scales.index_select(0, idx).cpu().numpy()
    same = (_parity.unpack(gc) == _parity.unpack(ref["codes"])).reshape(len(rows_s), -1, 32).all(2)
    same &= gs == ref["scales"]
    mask = np.repeat(same, 32, axis=1)
    v = _parity.bf16_to_f64(oracle.dequantize(ref["codes"], ref["scales"], w.cols))
    rr = _parity.bf16_to_f64(_bits(w.rhat))
    s_abs = (np.abs(v).reshape(len(rows_s), -1, 32) @ np.abs(rr).T).reshape(len(rows_s), -1)
    s_abs *= w.lam.numpy()[None, :]
    tol = 2.0 ** -7 * np.abs(ref_back) + 2.0 ** -18 * s_abs
    assert (np.abs(got - ref_back)[mask] <= tol[mask]).all()
    # round trip error relative to the input, per group: the MXFP4 error budget of an orthogonal map
    x = _parity.bf16_to_f64(synth.bf16_bits(w.x[torch.from_numpy(rows_s)]))
    rel = np.linalg.norm((got - x).reshape(len(rows_s), -1, 32), axis=2) / \
        np.maximum(np.linalg.norm(x.reshape(len(rows_s), -1, 32), axis=2), 1e-30)
    assert np.median(rel) < 0.2


# ---------------------------------------------------------------- the per-group error metric

@pytest.mark.parametrize("rows,cols,with_lam", [(300, 4096, False), (129, 1056, False), (257, 2048, True),
                                                (3, 96, True), (1, 32, False)])
def test_quant_error_matches_oracle(rows, cols, with_lam):
    w = synth.make_config(3, rows=rows, cols=cols)
    r = synth.rhat_tensor(synth.haar_orthogonal(rows + 1))
    lam = synth.random_lambda(cols, seed=3) if with_lam else None
    err, mean = mxq.quant_error(w.x.to(DEV), r.to(DEV), None if lam is None else lam.to(DEV))
    mxq.sync_check()
    err = err.cpu().numpy().astype(np.float64)
    ref_err, ref_mean = oracle.group_error(_bits(w.x), _bits(r), None if lam is None else lam.numpy(),
                                           threads=oracle.default_threads())
    flags = oracle.smooth_rotate_quantize(_bits(w.x), _bits(r), None if lam is None else lam.numpy(), flags=True,
                                          threads=oracle.default_threads())
    boundary = flags["gflags"].astype(bool) | flags["eflags"].reshape(rows, cols // 32, 32).any(axis=2)
    ok = np.abs(err - ref_err) <= 1e-5 + 1e-4 * ref_err
    assert (ok | boundary).all()
    assert (~ok).sum() <= max(1, 1e-5 * rows * cols)
    assert abs(float(mean.item()) - ref_mean) <= 1e-4 * ref_mean + 1e-7


def test_quant_error_deterministic_and_workspace_checked():
    w = synth.make_config(2, rows=512, cols=4096)
    x, r = w.x.to(DEV), w.rhat.to(DEV)
    _, m1 = mxq.quant_error(x, r, per_group=False)
    _, m2 = mxq.quant_error(x, r, per_group=False)
    assert m1.item() == m2.item()
    small = torch.empty(8, dtype=torch.uint8, device=DEV)
    with pytest.raises(mxq.MxqError) as ei:
        mxq.quant_error(x, r, workspace=small)
    assert ei.value.status == 1


def test_row_chunks_equal_one_call():
    # the rows are independent: quantising row slices (as the pipelined end-to-end leg of the
    # bench does) gives the same bits as one call over the whole matrix
    w = synth.make_config(2, rows=1000, cols=1024)
    x = w.x.to(DEV)
    rhat = w.rhat.to(DEV)
    lam = synth.smoothing_scale(w.x).to(DEV)
    for lm in (None, lam):
        c, s = mxq.smooth_rotate_quantize(x, rhat, lm)
        c2 = torch.empty_like(c)
        s2 = torch.empty_like(s)
        for lo, hi in ((0, 125), (125, 512), (512, 1000)):
            mxq.smooth_rotate_quantize(x[lo:hi], rhat, lm, codes=c2[lo:hi], scales=s2[lo:hi])
        mxq.sync_check()
        assert torch.equal(c, c2) and torch.equal(s, s2)

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
# Outputs of the inverse dequantiser that may differ from the correctly rounded value, as a
# fraction: only those whose exact value lies within the kernel's fp32 error of a bf16 rounding
# midpoint can.  The error is a few 2^-24 of the value against a bf16 step of 2^-8..2^-7 of it;
# on the B200 the smoothing workload's round trip gives 2970 of 469,760,416 (6.3e-6).
DEQUANT_MIDPOINT_FRAC = 1e-5


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
    # every output the correctly rounded bf16 of the exact value, except where the fp32 bound
    # around it holds a bf16 rounding midpoint (either rounding is then right)
    n_diff = _parity.check_dequant_inverse(codes, scales, cols, _bits(r), None if lam is None else lam.numpy(),
                                           synth.bf16_bits(got.cpu()), ref=(ref_bits, ref64))
    print(f"inverse dequantise {rows}x{cols} lambda={lam_kind}: {n_diff} of {rows * cols} outputs "
          f"differ from the correctly rounded value (all at a bf16 rounding midpoint within the fp32 bound)")
    assert n_diff <= DEQUANT_MIDPOINT_FRAC * rows * cols + 1


# ---------------------------------------------------------------- full-size configurations

def _full_config(cfg, chunk_elems=1 << 24, after_gpu=None, per_chunk=None):
    """The whole output of one full-size workload against the oracle, in row chunks of about
    chunk_elems elements.  after_gpu(w, codes, scales, rhat, lam) runs on the device tensors
    right after the quantiser; per_chunk(r0, r1, ref) after each chunk's check (the round trip
    uses both).  The boundary differences may total at most 1e-5 of all elements."""
    w = synth.make_config(cfg)
    xd = w.x.to(DEV)
    rd = w.rhat.to(DEV)
    ld = None if w.lam is None else w.lam.to(DEV)
    codes, scales = mxq.smooth_rotate_quantize(xd, rd, ld)
    mxq.sync_check()
    del xd
    if after_gpu is not None:
        after_gpu(w, codes, scales, rd, ld)
    # properties over the whole output: no NaN scales for finite inputs
    assert int(scales.max().item()) < 0xFF
    gc, gs = codes.cpu().numpy(), scales.cpu().numpy()
    xb, rb = synth.bf16_bits(w.x), _bits(w.rhat)
    lam = None if w.lam is None else w.lam.numpy()
    step = max(1, chunk_elems // w.cols)
    tot = {"elements": 0, "code_boundary_diffs": 0, "scale_boundary_diffs": 0}
    for r0 in range(0, w.rows, step):
        r1 = min(w.rows, r0 + step)
        res = _parity.check_quant(xb[r0:r1], rb, lam, gc[r0:r1], gs[r0:r1], max_frac=None)
        for key in tot:
            tot[key] += res[key]
        if per_chunk is not None:
            per_chunk(r0, r1, res["ref"])
        del res
    n_excused = tot["code_boundary_diffs"] + 32 * tot["scale_boundary_diffs"]
    print(f"config {cfg} ({w.rows}x{w.cols}, every element compared): {tot['code_boundary_diffs']} codes and "
          f"{tot['scale_boundary_diffs']} scales differ inside the boundary bands")
    assert n_excused <= 1e-5 * tot["elements"]
    assert tot["elements"] == w.rows * w.cols
    return w


@pytest.mark.parametrize("cfg", [1, 2, 3, 4])
def test_full_config(cfg):
    _full_config(cfg)
    torch.cuda.empty_cache()


def test_full_config5_with_round_trip():
    """The smoothing workload, then its dequantise round trip (undo R^ and Lambda) over every
    row.  The round trip is compared where the GPU's codes and scales equal the oracle's (its
    input is the GPU's codes); elsewhere a boundary tie made them differ."""
    state = {"diff": 0, "compared": 0, "rel_median": []}

    def dequant_on_gpu(w, codes, scales, rd, ld):
        back = mxq.dequantize(codes, scales, rd, ld)
        mxq.sync_check()
        state.update(w=w, gc=codes.cpu().numpy(), gs=scales.cpu().numpy(), back=synth.bf16_bits(back.cpu()))

    def round_trip(r0, r1, ref):
        w, gc, gs, back = state["w"], state["gc"], state["gs"], state["back"]
        same = (_parity.unpack(gc[r0:r1]) == _parity.unpack(ref["codes"])).reshape(r1 - r0, -1, 32).all(2)
        same &= gs[r0:r1] == ref["scales"]
        mask = np.repeat(same, 32, axis=1)
        n = _parity.check_dequant_inverse(ref["codes"], ref["scales"], w.cols, _bits(w.rhat), w.lam.numpy(),
                                          np.where(mask, back[r0:r1], 0).astype(np.uint16),
                                          ref=_masked_ref(ref, w, mask))
        state["diff"] += n
        state["compared"] += int(mask.sum())
        # the round trip against the input, per group: the MXFP4 error budget of an orthogonal map
        x = _parity.bf16_to_f64(synth.bf16_bits(w.x[r0:r1]))
        got = _parity.bf16_to_f64(back[r0:r1])
        rel = np.linalg.norm((got - x).reshape(r1 - r0, -1, 32), axis=2) / \
            np.maximum(np.linalg.norm(x.reshape(r1 - r0, -1, 32), axis=2), 1e-30)
        state["rel_median"].append(float(np.median(rel)))

    w = _full_config(5, after_gpu=dequant_on_gpu, per_chunk=round_trip)
    print(f"config 5 round trip: {state['diff']} of {state['compared']} outputs differ from the correctly "
          f"rounded value (all at a bf16 rounding midpoint within the fp32 bound)")
    assert state["compared"] >= 0.999 * w.rows * w.cols
    assert state["diff"] <= DEQUANT_MIDPOINT_FRAC * state["compared"]
    assert np.median(state["rel_median"]) < 0.2


def _masked_ref(ref, w, mask):
    """The oracle's round trip of its own codes, with the outputs outside `mask` set to 0 (they
    are not compared)."""
    bits, f64 = oracle.dequantize(ref["codes"], ref["scales"], w.cols, _bits(w.rhat), w.lam.numpy(), want_f64=True,
                                  threads=oracle.default_threads())
    return np.where(mask, bits, 0).astype(np.uint16), np.where(mask, f64, 0.0)


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

"""GPU parity of the NVFP4 variant with the oracle, through the C ABI.

The DuQuant++ write-up (§5.3) names NVFP4 as another block-scaled format the
rotation suits.  The reading is the public NVFP4 format: blocks of 16 E2M1 values,
one E4M3 scale per block and one fp32 tensor scale, every decision in fp32.  Parity
rule: E4M3 scales and E2M1 codes bit-exact outside the rounding bands, the
neighbouring value inside them, at most 1e-5 of the elements excused; exact cases
(identity, sign flips) bit-exact with no exceptions.
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


@pytest.fixture(scope="module", autouse=True)
def _device(cuda_device):
    from mxfp4_block_rotation_b200 import build
    build.build()
    yield


def _gpu(xb, rb, lam, s_t):
    x = synth.bf16_from_bits(xb).to(DEV)
    r = synth.bf16_from_bits(rb).to(DEV)
    lt = None if lam is None else torch.from_numpy(np.ascontiguousarray(lam, np.float32)).to(DEV)
    st = torch.tensor([s_t], dtype=torch.float32, device=DEV)
    codes, scales = mxq.smooth_rotate_quantize_nvfp4(x, r, st, lt)
    mxq.sync_check()
    return codes.cpu().numpy(), scales.cpu().numpy()


def _calibrated(xb, rb, lam):
    """s_t = amax(Y) / (6 * 448) from the oracle's rotated values: every block scale covers its block."""
    y = oracle.nvfp4_quantize(xb, rb, lam, 1.0, want_y=True, threads=oracle.default_threads())["y"]
    amax = float(np.abs(y).max())
    return float(np.float32(amax / (6 * 448))) if amax > 0 else 1.0


SHAPES = [(1, 32), (3, 64), (129, 256), (257, 1056), (1000, 640), (300, 4096)]


@pytest.mark.parametrize("rows,cols", SHAPES)
@pytest.mark.parametrize("with_lam", [False, True])
def test_nvfp4_matches_oracle(rows, cols, with_lam):
    w = synth.make_config(3, rows=rows, cols=cols)
    xb = synth.bf16_bits(w.x)
    rb = synth.bf16_bits(w.rhat)
    lam = synth.random_lambda(cols, seed=rows + cols).numpy() if with_lam else None
    s0 = _calibrated(xb, rb, lam)
    # calibrated; 100x too small (blocks saturate at 448); 1e4x too large (subnormal E4M3 scales)
    for s_t in (s0, float(np.float32(s0 / 100)), float(np.float32(s0 * 1e4))):
        c, s = _gpu(xb, rb, lam, s_t)
        _parity.check_nvfp4(xb, rb, lam, s_t, c, s)


@pytest.mark.parametrize("with_lam", [False, True])
def test_identity_and_sign_flip_exact(with_lam):
    rows, cols = 260, 512
    xb = synth.bf16_bits(synth.make_config(2, rows=rows, cols=cols).x)
    # with Λ a power of two the division is exact too
    lam = np.full(cols, 4.0, np.float32) if with_lam else None
    for m in (np.eye(32), -np.eye(32), np.diag(np.where(np.arange(32) % 3 == 0, -1.0, 1.0))):
        rb = synth.bf16_bits(synth.rhat_tensor(m))
        s_t = _calibrated(xb, rb, lam)
        c, s = _gpu(xb, rb, lam, s_t)
        _parity.check_nvfp4(xb, rb, lam, s_t, c, s, exact=True)


def test_special_blocks():
    rows, cols = 130, 256
    x = synth.random_bf16(rows, cols, seed=41).float().numpy().astype(np.float64)
    x[0, :] = 0.0                          # zero blocks -> scale 0, codes 0
    x[1, 16:32] = 1e-30                    # scale rounds to 0 -> codes 0
    x[2, :16] = -0.0
    x[3, 32:48] = np.nan                   # block 2 of row 3 -> 0x7F, codes 0
    x[4, 48] = np.inf                      # block 3 of row 4
    x[5, 64:80] = 3.0e38                   # v past 448 -> saturates at 0x7E
    xb = synth.bf16_bits(synth.to_bf16(x))
    rb = synth.bf16_bits(synth.rhat_tensor(np.eye(32)))
    s_t = 0.01
    c, s = _gpu(xb, rb, None, s_t)
    _parity.check_nvfp4(xb, rb, None, s_t, c, s, exact=True)
    assert s[0].max() == 0 and not c[0].any()
    assert s[1, 1] == 0 and s[3, 2] == 0x7F and s[4, 3] == 0x7F and s[5, 4] == 0x7E
    assert not c[3, 16:24].any() and not c[4, 24:32].any()


def test_round_trip_bound():
    rows, cols = 512, 2048
    w = synth.make_config(1, rows=rows, cols=cols)
    xb = synth.bf16_bits(w.x)
    rb = synth.bf16_bits(w.rhat)
    s_t = _calibrated(xb, rb, None)
    c, s = _gpu(xb, rb, None, s_t)
    y = oracle.nvfp4_quantize(xb, rb, None, s_t, want_y=True, threads=oracle.default_threads())["y"]
    codes = _parity.unpack(c)
    mag = np.array([0, .5, 1, 1.5, 2, 3, 4, 6])[codes & 7] * np.where(codes & 8, -1.0, 1.0)
    # E4M3 values of the GPU's scale bytes, decoded here (torch's float8_e4m3fn view)
    sbv = torch.from_numpy(np.ascontiguousarray(s)).view(torch.float8_e4m3fn).double().numpy().repeat(16, axis=1)
    back = mag * sbv * s_t
    blk_amax = np.abs(y).reshape(rows, -1, 16).max(2).repeat(16, axis=1)
    assert (np.abs(back - y) <= blk_amax / 6 * 1.07 + 1e-30).all()


def test_rejects_bad_arguments():
    x = torch.zeros((4, 64), dtype=torch.bfloat16, device=DEV)
    r = synth.rhat_tensor(np.eye(32)).to(DEV)
    st = torch.ones(1, dtype=torch.float32, device=DEV)
    with pytest.raises(ValueError):
        mxq.smooth_rotate_quantize_nvfp4(x, r, torch.ones(2, dtype=torch.float32, device=DEV))
    raw = torch.empty(4 * 4 + 1, dtype=torch.uint8, device=DEV)
    with pytest.raises(mxq.MxqError):      # scales at an odd address
        mxq.smooth_rotate_quantize_nvfp4(x, r, st, scales=raw[1:].view(4, 4))
    # a tensor scale in host memory is refused before any launch (MXQ_ERR_INVALID_ARG)
    st_host = torch.ones(1, dtype=torch.float32)
    rc = mxq.lib().mxq_smooth_rotate_quantize_nvfp4(x.data_ptr(), 4, 64, r.data_ptr(), None, st_host.data_ptr(),
                                                    raw.data_ptr(), raw.data_ptr(), None)
    assert rc == 1


def _l2_bound_scale(x, lam):
    """s_t from the per-group L2 norms of X / Λ (|y| <= |x| for an orthogonal map, 1% margin)."""
    n = torch.zeros(x.shape[0], dtype=torch.float64)
    for c0 in range(0, x.shape[1], 2048):
        xc = x[:, c0:c0 + 2048].double()
        if lam is not None:
            xc = xc / lam[c0:c0 + 2048].double()[None, :]
        n = torch.maximum(n, (xc.reshape(x.shape[0], -1, 32) ** 2).sum(2).sqrt().max(1).values)
    return float(np.float32(float(n.max()) * 1.01 / (6 * 448)))


@pytest.mark.parametrize("cfg", [1, 5])
def test_full_size_sampled(cfg):
    w = synth.make_config(cfg)
    s_t = _l2_bound_scale(w.x, w.lam)
    xd = w.x.to(DEV)
    rd = w.rhat.to(DEV)
    ld = None if w.lam is None else w.lam.to(DEV)
    st = torch.tensor([s_t], dtype=torch.float32, device=DEV)
    codes, scales = mxq.smooth_rotate_quantize_nvfp4(xd, rd, st, ld)
    mxq.sync_check()
    rows_s = synth.sample_rows(w.rows, 128, seed=9100 + cfg, must=w.outlier_rows)
    idx = torch.from_numpy(rows_s).to(DEV)
    c = codes.index_select(0, idx).cpu().numpy()
    s = scales.index_select(0, idx).cpu().numpy()
    xs = synth.bf16_bits(w.x[torch.from_numpy(rows_s)])
    _parity.check_nvfp4(xs, synth.bf16_bits(w.rhat), None if w.lam is None else w.lam.numpy(), s_t, c, s)
    # over the whole output: finite input -> no NaN scale, and no block scale past 448
    assert int(scales.max().item()) <= 0x7E
    del codes, scales, xd
    torch.cuda.empty_cache()

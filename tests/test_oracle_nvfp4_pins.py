"""Pins for the oracle's NVFP4 variant (the write-up's §5.3 names NVFP4 as another format the
method suits; the rule is the public NVFP4 format, decided in fp32 -- see the oracle's header).

  - E4M3 codes against the OCP FP8 table and torch's float8_e4m3fn cast (round to nearest even);
  - one block's scale and codes against a step-by-step float32 evaluation with torch's E4M3 and a
    brute-force E2M1 search;
  - special blocks (zero, NaN, tiny) and the E4M3 boundary flags;
  - R = I and a sign-flip R reduce to quantising X itself.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from tests import _bruteforce as bf
from workloads import synth


def test_e4m3_table_matches_the_format():
    spec = {0x00: 0.0, 0x01: 2.0 ** -9, 0x07: 7 * 2.0 ** -9, 0x08: 2.0 ** -6, 0x38: 1.0, 0x3C: 1.5,
            0x70: 128.0, 0x78: 256.0, 0x7E: 448.0}
    for c, v in spec.items():
        assert oracle.e4m3_value(c) == v
    assert math.isnan(oracle.e4m3_value(0x7F)) and math.isnan(oracle.e4m3_value(0xFF))
    vals = [oracle.e4m3_value(c) for c in range(0x7F)]
    assert all(b > a for a, b in zip(vals, vals[1:]))
    assert all(oracle.e4m3_code(v) == c for c, v in enumerate(vals))


def test_e4m3_rounding_against_torch():
    rng = np.random.default_rng(3)
    v = np.concatenate([np.exp(rng.uniform(np.log(2.0 ** -11), np.log(440.0), 4000)),
                        [0.5 * (oracle.e4m3_value(c) + oracle.e4m3_value(c + 1)) for c in range(0x7E)]])
    t = torch.from_numpy(v.astype(np.float32)).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    ours = np.array([oracle.e4m3_code(float(np.float32(x))) for x in v])
    assert np.array_equal(ours, t)
    # past 448 the conversion saturates (torch's cast gives NaN there instead)
    assert oracle.e4m3_code(449.0) == 0x7E and oracle.e4m3_code(1e30) == 0x7E
    assert oracle.e4m3_code(2.0 ** -11) == 0 and oracle.e4m3_code(float("nan")) == 0x7F


def _block_by_hand(y, s_t):
    """The rule step by step in float32, E4M3 by torch, E2M1 by brute force."""
    f = np.float32
    y = np.asarray(y, np.float32)
    r_t = f(1.0) / (f(6.0) * f(s_t))
    v = f(np.abs(y).max()) * r_t
    if float(v) > 448.0:
        sb = 0x7E
    else:
        sb = int(torch.tensor([v], dtype=torch.float32).to(torch.float8_e4m3fn).view(torch.uint8)[0])
    sbv = f(torch.tensor([sb], dtype=torch.uint8).view(torch.float8_e4m3fn).to(torch.float32)[0])
    s = sbv * f(s_t)
    if s == 0:
        return sb, [0] * 16
    r = f(1.0) / s
    return sb, [bf.e2m1_nearest(float(f(x) * r)) for x in y]


@pytest.mark.parametrize("seed", [0, 1, 2, 3])
def test_one_block_step_by_step(seed):
    rng = np.random.default_rng(seed)
    y = (rng.standard_normal(16) * 10.0 ** rng.uniform(-3, 3)).astype(np.float32).astype(np.float64)
    s_t = float(np.float32(10.0 ** rng.uniform(-4, 1)))
    sb, codes = _block_by_hand(y, s_t)
    c, _, _ = oracle.nvfp4_block_at(y, sb, s_t)
    assert list(c) == codes
    # the whole path with R = I on a 1 x 32 row whose first 16 values are y
    x = np.concatenate([y, np.zeros(16)]).reshape(1, 32)
    xb = synth.bf16_bits(synth.to_bf16(x))
    xf = (xb.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    eye = synth.bf16_bits(synth.rhat_tensor(np.eye(32)))
    out = oracle.nvfp4_quantize(xb, eye, None, s_t)
    sb2, codes2 = _block_by_hand(xf[0, :16], s_t)
    assert out["scales"][0, 0] == sb2
    got = np.empty(32, np.int64)
    got[0::2] = out["codes"][0] & 0xF
    got[1::2] = out["codes"][0] >> 4
    assert list(got[:16]) == codes2
    assert out["scales"][0, 1] == 0 and not got[16:].any()      # the zero block


def test_special_blocks_and_flags():
    eye = synth.bf16_bits(synth.rhat_tensor(np.eye(32)))
    x = np.zeros((1, 64))
    x[0, 3] = np.nan
    x[0, 40] = 1e-30                       # tiny block: its scale rounds to 0, codes 0
    out = oracle.nvfp4_quantize(synth.bf16_bits(synth.to_bf16(x)), eye, None, 1.0, flags=True)
    assert out["scales"][0, 0] == 0x7F and not out["codes"][0, :8].any()
    assert out["scales"][0, 2] == 0 and not out["codes"][0, 16:24].any()
    # a block whose v sits on an E4M3 midpoint is flagged, with the other code as alternative
    s_t = 1.0 / 6.0                        # r_t = 1: v = amax
    mid = 0.5 * (oracle.e4m3_value(0x38) + oracle.e4m3_value(0x39))   # 1.0625, exactly in bf16
    x = np.zeros((1, 32))
    x[0, 0] = mid
    out = oracle.nvfp4_quantize(synth.bf16_bits(synth.to_bf16(x)), eye, None, float(np.float32(s_t)), flags=True)
    assert out["bflags"][0, 0] == 1 and {int(out["scales"][0, 0]), int(out["alt_scales"][0, 0])} == {0x38, 0x39}


def test_sign_flip_rotation_flips_code_signs():
    rows, cols = 9, 128
    xb = synth.bf16_bits(synth.make_config(2, rows=rows, cols=cols).x)
    eye = synth.bf16_bits(synth.rhat_tensor(np.eye(32)))
    neg = synth.bf16_bits(synth.rhat_tensor(-np.eye(32)))
    a = oracle.nvfp4_quantize(xb, eye, None, 0.01)
    b = oracle.nvfp4_quantize(xb, neg, None, 0.01)
    assert np.array_equal(a["scales"], b["scales"])
    ca = np.stack([a["codes"] & 0xF, a["codes"] >> 4], -1)
    cb = np.stack([b["codes"] & 0xF, b["codes"] >> 4], -1)
    assert np.array_equal(ca ^ 8, cb)      # every code's sign bit flips, zeros included


def test_round_trip_error_is_bounded():
    # with the tensor scale from the tensor's amax (s_t = amax / (6 * 448)), every block's scale
    # covers its amax, so each value is within half a grid step of its reconstruction
    rows, cols = 16, 256
    w = synth.make_config(2, rows=rows, cols=cols)
    xb = synth.bf16_bits(w.x)
    rb = synth.bf16_bits(w.rhat)
    y = oracle.rotate_f64((xb.astype(np.uint32) << 16).view(np.float32).astype(np.float64),
                          (rb.astype(np.uint32) << 16).view(np.float32).astype(np.float64))
    s_t = float(np.float32(np.abs(y).max() / (6 * 448)))
    out = oracle.nvfp4_quantize(xb, rb, None, s_t, want_y=True)
    codes = np.stack([out["codes"] & 0xF, out["codes"] >> 4], -1).reshape(rows, cols)
    mag = np.array([0, .5, 1, 1.5, 2, 3, 4, 6])[codes & 7] * np.where(codes & 8, -1.0, 1.0)
    sbv = np.vectorize(oracle.e4m3_value)(out["scales"]).repeat(16, axis=1)
    back = mag * sbv * s_t
    yy = out["y"].astype(np.float32).astype(np.float64)
    blk_amax = np.abs(yy).reshape(rows, -1, 16).max(2).repeat(16, axis=1)
    assert (np.abs(back - yy) <= blk_amax / 6 * 1.07 + 1e-30).all()   # half of step 2 at the top binade

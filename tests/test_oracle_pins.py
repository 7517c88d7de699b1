"""Pins for the CPU oracle: each checks it against something other than itself.

The oracle is pinned to the worked example the DuQuant++ write-up prints
(§2.1), to closed forms of the MXFP4 format (grid values, power-of-two scaling,
sign symmetry), to invariants of an orthogonal block rotation (§2.3, §3.3:
X·R̂·R̂ᵀ = X, the block-diagonal product equals a batched 32x32 matmul), to a
library routine (torch.bmm in float64, the reshape-and-bmm form of §3.3's
implementation tips) and to an independent brute force over all 16 E2M1 codes.
"""
import math
import os

import numpy as np
import pytest
import torch

import oracle
from tests import _bruteforce as bf
from workloads import synth

GOLD = os.path.join(os.path.dirname(__file__), "golden")
RNG = np.random.default_rng(12345)


def _f32(a):
    return np.asarray(a, np.float64).astype(np.float32).astype(np.float64)


def _eye_bits():
    return synth.bf16_bits(synth.rhat_tensor(np.eye(32)))


def _read_golden(name):
    d = {}
    with open(os.path.join(GOLD, name)) as f:
        for line in f:
            if line.startswith("#") or not line.strip():
                continue
            k, v = line.split(":", 1)
            d[k.strip()] = v.split()
    return d


# ---------------------------------------------------------------- worked example

def test_worked_example_from_page():
    g = _read_golden("worked_example.txt")
    x = synth.to_bf16(np.array([float(v) for v in g["input"]]).reshape(1, 32))
    out = oracle.smooth_rotate_quantize(synth.bf16_bits(x), _eye_bits())
    assert out["scales"][0, 0] == int(g["scale"][0], 16)
    assert list(out["codes"][0]) == [int(b, 16) for b in g["codes"]]
    deq = oracle.dequantize(out["codes"], out["scales"], 32)
    vals = oracle.bf16_bits_to_f64(deq)[0]
    assert list(vals) == [float(v) for v in g["dequant"]]


# ---------------------------------------------------------------- E2M1 / E8M0 rules

def test_e2m1_table_matches_bit_format():
    for c in range(16):
        assert oracle.e2m1_value(c) == bf.e2m1_decode(c) or (c in (0, 8) and oracle.e2m1_value(c) == 0.0)


def _midpoint_probes():
    mags = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]
    pts = []
    for a, b in zip(mags[:-1], mags[1:]):
        m = 0.5 * (a + b)
        m32 = np.float32(m)
        pts += [m, float(np.nextafter(m32, np.float32(0))), float(np.nextafter(m32, np.float32(10))),
                float(np.nextafter(m, 0)), float(np.nextafter(m, 10))]
    for v in mags:
        pts += [v, float(np.nextafter(np.float32(v), np.float32(10)))]
    pts += [6.0, 6.0 + 2 ** -20, 8.0 - 2 ** -20, 7.0, 100.0, 1e30, 1e-30, 2 ** -149, 0.0]
    return pts


def test_e2m1_rounding_matches_bruteforce_at_midpoints():
    for p in _midpoint_probes():
        for u in (p, -p):
            assert oracle.e2m1_code(u) == bf.e2m1_nearest(u), u


def test_e2m1_ties_and_saturation_closed_form():
    # ties go to the even code (mantissa bit 0); above 6 saturates to 6
    expect = {0.25: 0, 0.75: 2, 1.25: 2, 1.75: 4, 2.5: 4, 3.5: 6, 5.0: 6, 6.5: 7, 7.99: 7}
    for u, c in expect.items():
        assert oracle.e2m1_code(u) == c
        assert oracle.e2m1_code(-u) == c | 8
    assert oracle.e2m1_code(-0.0) == 8 and oracle.e2m1_code(0.0) == 0
    assert oracle.e2m1_code(-0.1) == 8


def test_e2m1_rounding_random_against_bruteforce():
    u = RNG.uniform(-9, 9, size=4000)
    for v in u:
        assert oracle.e2m1_code(v) == bf.e2m1_nearest(v)


def test_e8m0_against_exponent_search():
    amaxes = list(np.exp(RNG.uniform(-95, 95, size=3000)))
    amaxes += [2.0 ** k for k in range(-149, 128)] + [2.0 ** k * 1.999 for k in range(-140, 127)]
    amaxes += [0.0, 1e-45, 3.0e38]
    for a in amaxes:
        assert oracle.e8m0_byte(a) == bf.e8m0_search(a), a
    assert oracle.e8m0_byte(float("inf")) == 0xFF and oracle.e8m0_byte(float("nan")) == 0xFF


def test_scale_puts_amax_in_top_binade():
    for a in np.exp(RNG.uniform(-80, 80, size=2000)):
        b = oracle.e8m0_byte(a)
        u = a / oracle.e8m0_value(b)
        assert 4.0 <= u < 8.0


# ---------------------------------------------------------------- whole groups

def test_group_quantizer_matches_bruteforce():
    for trial in range(300):
        kind = trial % 4
        y = RNG.standard_normal(32) * math.exp(RNG.uniform(-20, 20))
        if kind == 1:
            y[RNG.integers(32)] *= 1000.0
        if kind == 2:
            y[RNG.integers(32)] = 0.0
            y[RNG.integers(32)] = -0.0
        if kind == 3:
            y = RNG.integers(-12, 13, size=32) * 0.5 * 2.0 ** RNG.integers(-30, 30)
        y = _f32(y)
        out = oracle.quantize(y.reshape(1, 32))
        byte, codes = bf.quantize_group(y)
        assert out["scales"][0, 0] == byte
        assert list(out["codes"][0]) == list(bf.pack(codes))


def test_grid_values_quantize_exactly_and_round_trip():
    grid = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]
    for k in (-120, -5, 0, 3, 17, 100):
        for top in (4.0, 6.0):
            mags = RNG.choice([g for g in grid if g <= top], size=32)
            mags[RNG.integers(32)] = top
            signs = RNG.choice([-1.0, 1.0], size=32)
            y = mags * signs * 2.0 ** k
            out = oracle.quantize(y.reshape(1, 32))
            assert out["scales"][0, 0] == k + 127
            codes = oracle.unpack_codes(out["codes"])[0]
            vals = [oracle.e2m1_value(c) * 2.0 ** k for c in codes]
            assert np.array_equal(np.array(vals), y)
            deq = oracle.bf16_bits_to_f64(oracle.dequantize(out["codes"], out["scales"], 32))[0]
            assert np.array_equal(deq, y)


def test_fp32_decision_precision():
    # y is just above the 0.25 midpoint in double but rounds to exactly 0.25 in fp32:
    # the decision is taken on the fp32 value (a tie -> even code 0).
    y = np.zeros(32)
    y[0] = 4.0
    y[1] = 0.25 * (1 + 2.0 ** -30)
    out = oracle.quantize(y.reshape(1, 32))
    codes = oracle.unpack_codes(out["codes"])[0]
    assert codes[1] == 0
    y[1] = 0.25 * (1 + 2.0 ** -20)       # survives fp32 rounding -> code 1 (0.5)
    codes = oracle.unpack_codes(oracle.quantize(y.reshape(1, 32))["codes"])[0]
    assert codes[1] == 1


def test_nonfinite_group():
    y = np.ones((1, 64))
    y[0, 5] = np.inf
    out = oracle.quantize(y)
    assert out["scales"][0, 0] == 0xFF
    assert not out["codes"][0, :16].any()
    assert out["scales"][0, 1] == bf.e8m0_search(1.0)
    y[0, 40] = np.nan
    out = oracle.quantize(y)
    assert out["scales"][0, 1] == 0xFF and not out["codes"][0, 16:].any()


def test_boundary_flags():
    y = np.full(32, 0.1)
    y[0] = 4.0          # scale 2^0 -> u = y
    y[1] = 0.75         # exactly a midpoint
    y[2] = 1.0          # on the grid, far from midpoints
    y[3] = -1e-9        # next to the +0/-0 boundary
    out = oracle.quantize(y.reshape(1, 32), flags=True)
    ef, alt = out["eflags"][0], out["alt"][0]
    codes = oracle.unpack_codes(out["codes"])[0]
    assert ef[1] == 1 and codes[1] == 2 and alt[1] == 1
    assert ef[2] == 0 and alt[2] == codes[2]
    assert ef[3] == 1 and codes[3] == 8 and alt[3] == 0
    assert out["gflags"][0, 0] == 1          # amax exactly 4 = 2^2
    assert out["alt_scales"][0, 0] == out["scales"][0, 0] - 1
    y[0] = 3.3
    out = oracle.quantize(y.reshape(1, 32), flags=True)
    assert out["gflags"][0, 0] == 0 and out["alt_scales"][0, 0] == out["scales"][0, 0]
    y[0] = 8.0 * (1 - 1e-5)                  # just below 2^3: other side is the next byte up
    out = oracle.quantize(y.reshape(1, 32), flags=True)
    assert out["gflags"][0, 0] == 1 and out["alt_scales"][0, 0] == out["scales"][0, 0] + 1


# ---------------------------------------------------------------- rotation

def test_generated_rhat_orthogonal():
    for r in (synth.haar_orthogonal(2003), synth.hadamard_rhat(2004), synth.permutation_rhat(7)):
        assert np.abs(r.T @ r - np.eye(32)).max() < 1e-6


def test_rotation_round_trip_identity():
    r = synth.haar_orthogonal(99)
    x = RNG.standard_normal((5, 96))
    y = oracle.rotate_f64(x, r)
    back = oracle.rotate_f64(y, r.T.copy())
    assert np.abs(back - x).max() < 1e-12


def test_rotation_equals_torch_bmm():
    r = synth.haar_orthogonal(5)
    x = RNG.standard_normal((7, 160))
    lam = np.exp(RNG.uniform(-2, 2, size=160))
    y = oracle.rotate_f64(x, r, lam)
    xt = torch.from_numpy(x / lam[None, :]).reshape(7, 5, 32)
    ref = torch.bmm(xt, torch.from_numpy(r).expand(7, 32, 32)).reshape(7, 160).numpy()
    assert np.abs(y - ref).max() < 1e-12
    # a transposed operand would not match (R^ is not symmetric)
    assert np.abs(y - oracle.rotate_f64(x, r.T.copy(), lam)).max() > 1e-3


def test_bf16_conversions_exact():
    bits = RNG.integers(0, 1 << 16, size=5000).astype(np.uint16)
    t = synth.bf16_from_bits(bits)
    ref = t.to(torch.float64).numpy()
    got = oracle.bf16_bits_to_f64(bits)
    fin = np.isfinite(ref)
    assert np.array_equal(got[fin], ref[fin])
    # double -> bf16 on values that are fp32 numbers (then torch's fp32 -> bf16 is one RNE step)
    v = np.concatenate([RNG.standard_normal(3000) * 10.0 ** RNG.uniform(-40, 38, size=3000),
                        [3.3895313892515355e38, 3.39e38, 1e-39, -2.0 ** -133, 2.0 ** -134]])
    v32 = v.astype(np.float32)
    ref = synth.bf16_bits(torch.from_numpy(v32).to(torch.bfloat16))
    got = oracle.f64_to_bf16_bits(v32.astype(np.float64))
    assert np.array_equal(got, ref)


# ---------------------------------------------------------------- closed forms of the full path

def _path(x_bits, r, lam=None):
    return oracle.smooth_rotate_quantize(x_bits, synth.bf16_bits(synth.rhat_tensor(r)), lam)


def test_identity_rotation_is_plain_mxfp4():
    x = synth.random_bf16(4, 128, seed=3, scale=3.0)
    out = _path(synth.bf16_bits(x), np.eye(32))
    xv = x.to(torch.float64).numpy()
    for r in range(4):
        for g in range(4):
            byte, codes = bf.quantize_group(xv[r, 32 * g:32 * g + 32])
            assert out["scales"][r, g] == byte
            assert list(out["codes"][r, 16 * g:16 * g + 16]) == list(bf.pack(codes))


def test_negated_rotation_flips_signs():
    x = synth.random_bf16(3, 96, seed=4)
    xv = x.to(torch.float64).numpy()
    assert (xv != 0).all()
    a = _path(synth.bf16_bits(x), np.eye(32))
    b = _path(synth.bf16_bits(x), -np.eye(32))
    assert np.array_equal(a["scales"], b["scales"])
    assert np.array_equal(a["codes"] ^ 0x88, b["codes"])


def test_permutation_rotation_permutes_codes():
    p = synth.permutation_rhat(11)
    x = synth.random_bf16(3, 64, seed=5)
    a = _path(synth.bf16_bits(x), np.eye(32))
    b = _path(synth.bf16_bits(x), p)
    ca, cb = oracle.unpack_codes(a["codes"]), oracle.unpack_codes(b["codes"])
    perm = np.argmax(p, axis=1)              # y_n = x_k where R[k][n] = 1, i.e. n = perm[k]
    for g in range(2):
        blk_a = ca[:, 32 * g:32 * g + 32]
        blk_b = cb[:, 32 * g:32 * g + 32]
        assert np.array_equal(blk_b[:, perm], blk_a)
    assert np.array_equal(a["scales"], b["scales"])


def test_power_of_two_input_scaling_shifts_scale():
    x = synth.random_bf16(3, 128, seed=6)
    r = synth.haar_orthogonal(8)
    a = _path(synth.bf16_bits(x), r)
    for j in (-9, 5):
        xs = (x.float() * 2.0 ** j).to(torch.bfloat16)
        b = _path(synth.bf16_bits(xs), r)
        assert np.array_equal(a["codes"], b["codes"])
        assert np.array_equal(a["scales"].astype(int) + j, b["scales"].astype(int))


def test_lambda_ones_equals_null_and_power_of_two_lambda_shifts():
    x = synth.random_bf16(3, 128, seed=7)
    r = synth.haar_orthogonal(9)
    a = _path(synth.bf16_bits(x), r)
    b = _path(synth.bf16_bits(x), r, np.ones(128, np.float32))
    assert np.array_equal(a["codes"], b["codes"]) and np.array_equal(a["scales"], b["scales"])
    js = np.array([3, -2, 0, 7])
    lam = np.repeat(2.0 ** js, 32).astype(np.float32)
    c = _path(synth.bf16_bits(x), r, lam)
    assert np.array_equal(a["codes"], c["codes"])
    assert np.array_equal(a["scales"].astype(int) - js[None, :], c["scales"].astype(int))


def test_smoothing_divides_per_channel():
    # a non-uniform Λ inside one group: path(X, Λ) == path(X', null) where X' = X/Λ is exact
    x = synth.random_bf16(2, 32, seed=8)
    lam = np.array([2.0 ** (k % 5 - 2) for k in range(32)], np.float32)
    xp = synth.to_bf16(x.to(torch.float64).numpy() / lam[None, :].astype(np.float64))
    r = synth.haar_orthogonal(10)
    a = _path(synth.bf16_bits(x), r, lam)
    b = _path(synth.bf16_bits(xp), r)
    assert np.array_equal(a["codes"], b["codes"]) and np.array_equal(a["scales"], b["scales"])


def test_dequant_error_within_half_step():
    x = synth.random_bf16(6, 256, seed=9, scale=2.0)
    r = synth.haar_orthogonal(12)
    out = oracle.smooth_rotate_quantize(synth.bf16_bits(x), synth.bf16_bits(synth.rhat_tensor(r)),
                                        want_y=True)
    deq = oracle.bf16_bits_to_f64(oracle.dequantize(out["codes"], out["scales"], 256))
    y = _f32(out["y"])
    s = np.repeat(np.array([[oracle.e8m0_value(b) for b in row] for row in out["scales"]]), 32, axis=1)
    u = np.abs(y) / s
    half_step = np.where(u < 2, 0.25, np.where(u < 4, 0.5, 1.0))
    bound = np.where(u > 6, u - 6, half_step) * s
    assert (np.abs(deq - y) <= bound + 1e-300).all()


def test_dequant_with_rotation_inverts():
    x = synth.random_bf16(4, 128, seed=10)
    r = synth.haar_orthogonal(13)
    lam = synth.random_lambda(128, seed=14).numpy()
    rb = synth.bf16_bits(synth.rhat_tensor(r))
    out = oracle.smooth_rotate_quantize(synth.bf16_bits(x), rb, lam)
    back, back64 = oracle.dequantize(out["codes"], out["scales"], 128, rb, lam, want_f64=True)
    # back64 = deq(y) * R^T * lam; undoing it (/lam, *R^) must give deq(y) up to double rounding
    # (R^ in bf16 is orthogonal only to ~1e-3, so compare through the same matrix on both sides)
    rr = oracle.bf16_bits_to_f64(rb)
    deq = oracle.bf16_bits_to_f64(oracle.dequantize(out["codes"], out["scales"], 128))
    ref = (deq.reshape(4, 4, 32) @ rr.T).reshape(4, 128) * lam[None, :]
    assert np.abs(back64 - ref).max() <= 1e-12 * np.abs(ref).max()
    assert np.array_equal(oracle.f64_to_bf16_bits(back64), back)


# ---------------------------------------------------------------- the per-group error metric (§4.1, Figure 1)

def test_group_error_worked_example_closed_form():
    # §2.1's group: Q keeps only the 1024 outlier (code 0x6 at scale 2^8), so the error is
    # ||x without the outlier|| / ||x|| exactly.
    g = _read_golden("worked_example.txt")
    x = synth.to_bf16(np.array([float(v) for v in g["input"]]).reshape(1, 32))
    xv = x.to(torch.float64).numpy()[0]
    err, mean = oracle.group_error(synth.bf16_bits(x), _eye_bits())
    expect = math.sqrt((xv ** 2).sum() - 1024.0 ** 2) / math.sqrt((xv ** 2).sum())
    assert abs(err[0, 0] - expect) < 1e-15 and mean == err[0, 0]


def test_group_error_zero_on_grid_and_zero_groups():
    y = np.zeros((2, 64))
    y[0, :32] = [(-1) ** i * [0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0][i % 7] * 2.0 ** 5 for i in range(32)]
    x = synth.to_bf16(y)
    err, mean = oracle.group_error(synth.bf16_bits(x), _eye_bits())
    assert (err == 0.0).all() and mean == 0.0


def test_group_error_matches_bruteforce():
    r = synth.haar_orthogonal(21)
    rb = synth.bf16_bits(synth.rhat_tensor(r))
    x = synth.make_config(3, rows=6, cols=128).x
    err, mean = oracle.group_error(synth.bf16_bits(x), rb)
    y = oracle.rotate_f64(oracle.bf16_bits_to_f64(synth.bf16_bits(x)), oracle.bf16_bits_to_f64(rb))
    ref = np.zeros_like(err)
    for i in range(6):
        for g in range(4):
            yy = _f32(y[i, 32 * g:32 * g + 32])
            byte, codes = bf.quantize_group(yy)
            v = np.array([bf.e2m1_decode(c) for c in codes]) * 2.0 ** (byte - 127)
            ref[i, g] = np.linalg.norm(v - yy) / np.linalg.norm(yy)
    assert np.abs(err - ref).max() < 1e-12
    assert abs(mean - ref.mean()) < 1e-12


def test_hadamard_lowers_error_on_outlier_activations():
    # §4.1's Figure 1: a random Hadamard block rotation lowers the per-group MXFP4 error
    # of outlier-heavy activations relative to the original ones.
    w = synth.make_config(1, rows=64, cols=4096)
    xb = synth.bf16_bits(w.x)
    _, e_orig = oracle.group_error(xb, _eye_bits(), threads=oracle.default_threads())
    _, e_had = oracle.group_error(xb, synth.bf16_bits(synth.rhat_tensor(synth.hadamard_rhat(5))),
                                  threads=oracle.default_threads())
    assert e_had < e_orig

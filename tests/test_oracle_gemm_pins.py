"""Pins for the oracle's MXFP4 consumer GEMM and the weights' side of the absorption
(DuQuant++ write-up, §3.3: X̂ = X·Λ⁻¹·R̂ and Ŵ = R̂ᵀ·Λ·W, so X̂·Ŵ = X·W).

  - the GEMM equals numpy's matmul of operands decoded here from the E2M1 and E8M0
    bit formats themselves;
  - a scale byte + 1 doubles the result; one code per row picks one column of B; the
    high nibble is the odd k; a 0xFF scale gives NaN;
  - the weight side multiplies by Λ (numpy's reshaped matmul), and with a signed
    permutation R̂ (exactly orthogonal in bf16) X̂·Ŵᵀ equals X·Wᵀ in double.
"""
import numpy as np
import pytest

import oracle
from workloads import synth


def _decode(codes, scales):
    """E2M1: sign bit 3, exponent bits 2-1 (bias 1), mantissa bit 0; E8M0: 2^(byte-127)."""
    rows = codes.shape[0]
    c = np.empty((rows, codes.shape[1] * 2), np.int64)
    c[:, 0::2] = codes & 0xF
    c[:, 1::2] = codes >> 4
    s, e, m = (c >> 3) & 1, (c >> 1) & 3, c & 1
    mag = np.where(e == 0, 0.5 * m, (1.0 + 0.5 * m) * 2.0 ** (e - 1))
    v = np.where(s == 1, -mag, mag)
    sc = np.where(scales == 0xFF, np.nan, 2.0 ** (scales.astype(np.float64) - 127.0))
    return v * np.repeat(sc, 32, axis=1)


def _rand_mx(rng, rows, k, lo=118, hi=136):
    return (rng.integers(0, 256, (rows, k // 2), dtype=np.uint8),
            rng.integers(lo, hi, (rows, k // 32), dtype=np.uint8))


def _f64(bits):
    return (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


@pytest.mark.parametrize("M,N,K", [(1, 1, 32), (5, 7, 64), (33, 20, 320)])
def test_gemm_is_the_decoded_matmul(M, N, K):
    rng = np.random.default_rng(M * N + K)
    a, sa = _rand_mx(rng, M, K)
    b, sb = _rand_mx(rng, N, K)
    y = oracle.mxfp4_gemm(a, sa, b, sb)
    want = _decode(a, sa) @ _decode(b, sb).T
    assert np.allclose(y, want, rtol=1e-13, atol=1e-300)


def test_gemm_scale_and_nibble_and_nan():
    rng = np.random.default_rng(1)
    M, N, K = 4, 6, 128
    a, sa = _rand_mx(rng, M, K)
    b, sb = _rand_mx(rng, N, K)
    y = oracle.mxfp4_gemm(a, sa, b, sb)
    assert np.array_equal(oracle.mxfp4_gemm(a, sa + 1, b, sb), 2.0 * y)
    # one code (1.0, code 2) per row at k0, scale 2^0: Y[m] is column k0 of deq(B)
    a1 = np.zeros((2, K // 2), np.uint8)
    a1[0, 37 // 2] = 0x20          # k0 = 37: odd, so the high nibble
    a1[1, 64 // 2] = 0x02          # k0 = 64: even, the low nibble
    s1 = np.full((2, K // 32), 127, np.uint8)
    y1 = oracle.mxfp4_gemm(a1, s1, b, sb)
    db = _decode(b, sb)
    assert np.array_equal(y1[0], db[:, 37]) and np.array_equal(y1[1], db[:, 64])
    sa2 = sa.copy()
    sa2[2, 1] = 0xFF
    y2 = oracle.mxfp4_gemm(a, sa2, b, sb)
    assert np.isnan(y2[2]).all() and np.array_equal(np.delete(y2, 2, 0), np.delete(y, 2, 0))


def test_weight_side_multiplies_by_lambda():
    rows, cols = 6, 128
    wt = synth.bf16_bits(synth.make_config(2, rows=rows, cols=cols).x)
    rb = synth.bf16_bits(synth.rhat_tensor(synth.haar_orthogonal(3)))
    lam = synth.random_lambda(cols, seed=5).numpy()
    out = oracle.weight_rotate_quantize(wt, rb, lam, want_y=True)
    want = ((_f64(wt) * lam.astype(np.float64)).reshape(-1, 32) @ _f64(rb)).reshape(rows, cols)
    assert np.allclose(out["y"], want, rtol=1e-12, atol=1e-12 * np.abs(want).max())
    plain = oracle.weight_rotate_quantize(wt, rb, None)
    ref = oracle.smooth_rotate_quantize(wt, rb, None)
    assert np.array_equal(plain["codes"], ref["codes"]) and np.array_equal(plain["scales"], ref["scales"])


def test_absorption_identity_with_an_exact_rotation():
    # R̂ = a signed permutation: exactly orthogonal in bf16, so X̂·Ŵ = X·W up to double rounding
    rng = np.random.default_rng(2)
    p = np.eye(32)[rng.permutation(32)] * rng.choice([-1.0, 1.0], 32)[:, None]
    rb = synth.bf16_bits(synth.rhat_tensor(p))
    M, N, K = 9, 11, 256
    x = synth.bf16_bits(synth.make_config(2, rows=M, cols=K).x)
    wt = synth.bf16_bits(synth.make_config(1, rows=N, cols=K).x)
    lam = synth.random_lambda(K, seed=3).numpy()
    xh = oracle.smooth_rotate_quantize(x, rb, lam, want_y=True)["y"]
    wh = oracle.weight_rotate_quantize(wt, rb, lam, want_y=True)["y"]
    want = _f64(x) @ _f64(wt).T
    assert np.allclose(xh @ wh.T, want, rtol=1e-12, atol=1e-12 * np.abs(want).max())


def test_quantised_product_approximates_the_full_product():
    # end to end in the oracle: MXFP4(X̂) · MXFP4(Ŵ)ᵀ against X·Wᵀ (a sanity bound, not a claim).
    # W = X makes the product a Gram matrix, large against the quantisation noise; independent
    # random rows would give near-orthogonal dot products that no relative bound fits.
    M, N, K = 16, 16, 512
    x = synth.bf16_bits(synth.make_config(2, rows=M, cols=K).x)
    wt = x
    rb = synth.bf16_bits(synth.rhat_tensor(synth.haar_orthogonal(4)))
    qa = oracle.smooth_rotate_quantize(x, rb, None)
    qb = oracle.weight_rotate_quantize(wt, rb, None)
    y = oracle.mxfp4_gemm(qa["codes"], qa["scales"], qb["codes"], qb["scales"])
    want = _f64(x) @ _f64(wt).T
    assert np.linalg.norm(y - want) / np.linalg.norm(want) < 0.25


def test_scale_atoms_hold_every_scale_once():
    # every scale lands at the byte the atom formula names, and everything else is 0
    rng = np.random.default_rng(9)
    rows, G = 300, 13                      # ragged in both: 3 row blocks, 4 k-block groups
    sc = rng.integers(1, 255, (rows, G), dtype=np.uint8)
    out = oracle.scales_to_mma(sc)
    CB = (G + 3) // 4
    assert out.size == 3 * CB * 512
    seen = np.zeros(out.size, bool)
    for r in range(rows):
        for kb in range(G):
            off = ((r // 128) * CB + kb // 4) * 512 + 16 * (r % 32) + 4 * ((r % 128) // 32) + kb % 4
            assert out[off] == sc[r, kb]
            seen[off] = True
    assert not out[~seen].any()
    # one 16-byte row of an atom: four words, one per 32-row slice, each the row's 4 k-blocks
    atom = out[:512].reshape(32, 4, 4)
    assert np.array_equal(atom[5, 2], sc[64 + 5, 0:4])


# ---------------------------------------------------------------- the NVFP4 consumer GEMM

def _decode_e4m3(b):
    """E4M3 (OCP, no infinities): sign bit 7, exponent bits 6-3 (bias 7), mantissa bits 2-0;
    exponent 0 is subnormal m/8 * 2^-6; 0x7F and 0xFF are NaN."""
    b = b.astype(np.int64)
    s, e, m = (b >> 7) & 1, (b >> 3) & 15, b & 7
    mag = np.where(e == 0, (m / 8.0) * 2.0 ** -6, (1.0 + m / 8.0) * 2.0 ** (e - 7))
    mag = np.where((e == 15) & (m == 7), np.nan, mag)
    return np.where(s == 1, -mag, mag)


def _decode_nv(codes, scales, tscale):
    rows = codes.shape[0]
    c = np.empty((rows, codes.shape[1] * 2), np.int64)
    c[:, 0::2] = codes & 0xF
    c[:, 1::2] = codes >> 4
    s, e, m = (c >> 3) & 1, (c >> 1) & 3, c & 1
    mag = np.where(e == 0, 0.5 * m, (1.0 + 0.5 * m) * 2.0 ** (e - 1))
    v = np.where(s == 1, -mag, mag)
    return v * np.repeat(_decode_e4m3(scales), 16, axis=1) * float(np.float32(tscale))


def _rand_nv(rng, rows, k):
    # E4M3 scale codes in [0x20, 0x48]: normal values 2^-3 .. 2^2
    return (rng.integers(0, 256, (rows, k // 2), dtype=np.uint8),
            rng.integers(0x20, 0x48, (rows, k // 16), dtype=np.uint8))


@pytest.mark.parametrize("M,N,K", [(1, 1, 32), (5, 7, 64), (33, 20, 320)])
def test_nvfp4_gemm_is_the_decoded_matmul(M, N, K):
    rng = np.random.default_rng(M * 100 + N + K)
    a, sa = _rand_nv(rng, M, K)
    b, sb = _rand_nv(rng, N, K)
    ta, tb = 0.37, 1.9
    y = oracle.nvfp4_gemm(a, sa, ta, b, sb, tb)
    ref = _decode_nv(a, sa, ta) @ _decode_nv(b, sb, tb).T
    assert np.allclose(y, ref, rtol=1e-12, atol=1e-12 * np.abs(ref).max())


def test_nvfp4_gemm_scales_and_nan():
    rng = np.random.default_rng(5)
    a, sa = _rand_nv(rng, 3, 64)
    b, sb = _rand_nv(rng, 4, 64)
    y = oracle.nvfp4_gemm(a, sa, 1.0, b, sb, 1.0)
    # an E4M3 exponent step (+8 on a normal code) doubles that block's contribution: here every
    # block of row 0 of A at once, so the whole row doubles
    sa2 = sa.copy()
    sa2[0] += 8
    assert np.array_equal(oracle.nvfp4_gemm(a, sa2, 1.0, b, sb, 1.0)[0], 2 * y[0])
    # the tensor scales multiply the result
    assert np.allclose(oracle.nvfp4_gemm(a, sa, 4.0, b, sb, 0.5), 2.0 * y, rtol=0, atol=0)
    # a NaN block scale (0x7F) poisons its row; 0xFF too
    sa3 = sa.copy()
    sa3[1, 2] = 0x7F
    sa3[2, 0] = 0xFF
    y3 = oracle.nvfp4_gemm(a, sa3, 1.0, b, sb, 1.0)
    assert np.isnan(y3[1]).all() and np.isnan(y3[2]).all() and np.array_equal(y3[0], y[0])
    # the scale of block 1 (k = 16..31) acts on those k only: zero the codes of k < 16 and of
    # k >= 32, then doubling block 1's scale doubles the product and changing block 0's does nothing
    a4 = a.copy()
    a4[:, :8] = 0
    a4[:, 16:] = 0
    y4 = oracle.nvfp4_gemm(a4, sa, 1.0, b, sb, 1.0)
    sa4 = sa.copy()
    sa4[:, 1] += 8
    sa4[:, 0] += 8
    assert np.array_equal(oracle.nvfp4_gemm(a4, sa4, 1.0, b, sb, 1.0), 2 * y4)
    sa5 = sa.copy()
    sa5[:, 0] += 8
    assert np.array_equal(oracle.nvfp4_gemm(a4, sa5, 1.0, b, sb, 1.0), y4)

"""Comparison of the CUDA path's MXFP4 output with the oracle's, under the
acceptance rule for this path:

* Scales and codes must be bit-exact wherever the oracle's rotated value (in
  fp32, its decision precision) lies more than 1e-3 of a grid step from a
  rounding boundary.  The same holds for groups whose absmax lies more than
  2.5e-4 relative from a power of two.
* Inside those bands both neighbours are correct.  A differing GPU result must
  equal the oracle's neighbour across that boundary: the alternative code, or
  the alternative scale with the codes the oracle gives under it.
* Differing results inside the bands may not exceed 1e-5 of the elements
  compared.
"""
from __future__ import annotations

import numpy as np

import oracle


def unpack(codes):
    """[rows, cols/2] packed bytes -> [rows, cols] 4-bit codes (even column = low nibble).  The
    tests' own helper: GPU outputs are never fed to the oracle, not even to unpack them."""
    codes = np.asarray(codes, np.uint8)
    out = np.empty(codes.shape[:-1] + (codes.shape[-1] * 2,), np.uint8)
    out[..., 0::2] = codes & 15
    out[..., 1::2] = codes >> 4
    return out


def bf16_to_f64(bits):
    """bf16 bit patterns (uint16) -> float64, exactly (bf16 is the top half of an fp32)."""
    b = np.asarray(bits).astype(np.uint16).astype(np.uint32) << 16
    return b.view(np.float32).astype(np.float64)


def check_quant(x_bits, rhat_bits, lam, gpu_codes, gpu_scales, threads=None, exact=False, ref=None,
                max_frac=1e-5):
    """Compare GPU codes/scales for the rows of x_bits; returns a dict of counts (raises on failure).

    `ref` is the oracle's output (with y and flags) when the caller has it already, e.g. from
    another oracle entry point; otherwise the main path's oracle is run here.  `max_frac` bounds
    the boundary differences as a fraction of these rows' elements; a caller checking a matrix in
    row chunks passes None and applies the bound to the totals."""
    threads = threads or oracle.default_threads()
    if ref is None:
        ref = oracle.smooth_rotate_quantize(x_bits, rhat_bits, lam, want_y=True, flags=True, threads=threads)
    rows, cols = x_bits.shape
    G = cols // 32
    gpu_codes = np.asarray(gpu_codes, np.uint8)
    gpu_scales = np.asarray(gpu_scales, np.uint8)
    assert gpu_codes.shape == ref["codes"].shape and gpu_scales.shape == ref["scales"].shape

    sc_diff = gpu_scales != ref["scales"]
    sc_alt_ok = (ref["gflags"] == 1) & (gpu_scales == ref["alt_scales"])
    bad_sc = sc_diff & ~sc_alt_ok
    if bad_sc.any():
        r, g = np.argwhere(bad_sc)[0]
        raise AssertionError(f"scale mismatch outside the boundary band at row {r} group {g}: "
                             f"gpu {gpu_scales[r, g]:#x} oracle {ref['scales'][r, g]:#x} "
                             f"(y={ref['y'][r, 32 * g:32 * g + 32]})")

    gc = unpack(gpu_codes)
    rc = unpack(ref["codes"])
    same_scale = np.repeat(~sc_diff, 32, axis=1)
    diff = (gc != rc) & same_scale
    excused = (ref["eflags"] == 1) & (gc == ref["alt"])
    bad = diff & ~excused
    if bad.any():
        r, c = np.argwhere(bad)[0]
        g = c // 32
        raise AssertionError(f"code mismatch outside the rounding band at row {r} col {c}: "
                             f"gpu {gc[r, c]:#x} oracle {rc[r, c]:#x} alt {ref['alt'][r, c]:#x} "
                             f"y={ref['y'][r, c]!r} scale={ref['scales'][r, g]:#x}")
    n_code_diff = int(diff.sum())

    # groups quantised with the neighbouring scale: compare with the oracle under that scale
    n_alt_groups = 0
    for r, g in np.argwhere(sc_diff):
        n_alt_groups += 1
        y32 = ref["y"][r, 32 * g:32 * g + 32].astype(np.float32).astype(np.float64)
        # (the GPU's scale equals the oracle's alternative here: the oracle's value is the input)
        codes, flags, alt = oracle.quantize_group_at(y32, int(ref["alt_scales"][r, g]))
        got = gc[r, 32 * g:32 * g + 32]
        ok = (got == codes) | ((flags == 1) & (got == alt))
        if not ok.all():
            raise AssertionError(f"group at row {r} group {g} with the alternative scale does not match")
    n_elems = rows * cols
    n_excused = n_code_diff + 32 * n_alt_groups
    if exact:
        assert n_excused == 0, f"{n_code_diff} code and {n_alt_groups} scale differences where exact was required"
    if max_frac is not None:
        assert n_excused <= max_frac * n_elems, f"{n_excused} boundary differences > {max_frac} of {n_elems}"
    return {"elements": n_elems, "code_boundary_diffs": n_code_diff, "scale_boundary_diffs": n_alt_groups,
            "y": ref["y"], "ref": ref}


def check_f32(y_oracle, y_gpu, rel=2e-3):
    """|y_gpu - y| <= rel * max(|y|, 1e-3 * group absmax), element-wise."""
    y_oracle = np.asarray(y_oracle, np.float64)
    y_gpu = np.asarray(y_gpu, np.float64)
    rows, cols = y_oracle.shape
    amax = np.abs(y_oracle).reshape(rows, cols // 32, 32).max(axis=2)
    floor = np.repeat(1e-3 * amax, 32, axis=1)
    tol = rel * np.maximum(np.abs(y_oracle), floor)
    err = np.abs(y_gpu - y_oracle)
    bad = ~(err <= tol)
    if bad.any():
        r, c = np.argwhere(bad)[0]
        raise AssertionError(f"fp32 rotated value off at ({r},{c}): gpu {y_gpu[r, c]!r} oracle {y_oracle[r, c]!r}")
    return float((err / np.maximum(tol, 1e-300)).max()) * rel


def check_nvfp4(x_bits, rhat_bits, lam, s_t, gpu_codes, gpu_scales, exact=False, threads=None):
    """NVFP4 variant of check_quant: blocks of 16 with E4M3 scales (the oracle's NVFP4 reading).

    A block scale may differ only where the oracle flags v = amax * r_t as within 2.5e-4 of an
    E4M3 rounding midpoint and the GPU took the code on the other side; such a block's codes are
    then checked against the oracle under the GPU's scale.  Codes may differ only inside the
    E2M1 rounding band, to the neighbouring code; the total is at most 1e-5 of the elements."""
    threads = threads or oracle.default_threads()
    ref = oracle.nvfp4_quantize(x_bits, rhat_bits, lam, s_t, want_y=True, flags=True, threads=threads)
    rows, cols = x_bits.shape
    gpu_codes = np.asarray(gpu_codes, np.uint8)
    gpu_scales = np.asarray(gpu_scales, np.uint8)
    assert gpu_codes.shape == ref["codes"].shape and gpu_scales.shape == ref["scales"].shape
    sc_diff = gpu_scales != ref["scales"]
    bad_sc = sc_diff & ~((ref["bflags"] == 1) & (gpu_scales == ref["alt_scales"]))
    if bad_sc.any():
        r, b = np.argwhere(bad_sc)[0]
        raise AssertionError(f"E4M3 scale mismatch outside the band at row {r} block {b}: gpu "
                             f"{gpu_scales[r, b]:#x} oracle {ref['scales'][r, b]:#x} "
                             f"(y={ref['y'][r, 16 * b:16 * b + 16]})")
    gc = unpack(gpu_codes)
    rc = unpack(ref["codes"])
    diff = (gc != rc) & np.repeat(~sc_diff, 16, axis=1)
    bad = diff & ~((ref["eflags"] == 1) & (gc == ref["alt"]))
    if bad.any():
        r, c = np.argwhere(bad)[0]
        raise AssertionError(f"NVFP4 code mismatch outside the band at row {r} col {c}: gpu {gc[r, c]:#x} "
                             f"oracle {rc[r, c]:#x} alt {ref['alt'][r, c]:#x} y={ref['y'][r, c]!r} "
                             f"scale={ref['scales'][r, c // 16]:#x}")
    n_alt = 0
    for r, b in np.argwhere(sc_diff):
        n_alt += 1
        # (the GPU's scale equals the oracle's alternative here: the oracle's value is the input)
        codes, flags, alt = oracle.nvfp4_block_at(ref["y"][r, 16 * b:16 * b + 16], int(ref["alt_scales"][r, b]), s_t)
        got = gc[r, 16 * b:16 * b + 16]
        if not ((got == codes) | ((flags == 1) & (got == alt))).all():
            raise AssertionError(f"block at row {r} block {b} under the neighbouring scale does not match")
    n_excused = int(diff.sum()) + 16 * n_alt
    if exact:
        assert n_excused == 0, f"{int(diff.sum())} code and {n_alt} scale differences where exact was required"
    assert n_excused <= 1e-5 * rows * cols, f"{n_excused} boundary differences > 1e-5 of {rows * cols}"
    return {"elements": rows * cols, "code_boundary_diffs": int(diff.sum()), "scale_boundary_diffs": n_alt,
            "ref": ref}


def bf16_rne_bits(t):
    """float64 -> bf16 bit patterns, rounded once to nearest even (no detour through fp32, so no
    double rounding).  Finite values only; bf16 subnormals are rounded on their own grid."""
    t = np.asarray(t, np.float64)
    assert np.isfinite(t).all()
    m, e = np.frexp(t)                                   # t = m 2^e, 0.5 <= |m| < 1
    e = np.maximum(e, -125)                              # below 2^-126 the grid is fixed: 2^-133
    q = np.rint(np.ldexp(m, 8 + (np.frexp(t)[1] - e)))   # 8 significant bits (fewer when subnormal)
    v = np.ldexp(q, e - 8)                               # exact in double and in fp32
    bits = (v.astype(np.float32).view(np.uint32) >> 16).astype(np.uint16)
    return bits


def _bf16_order(bits):
    """bf16 bit patterns -> integers in the order of their values (-0 and +0 adjacent)."""
    b = np.asarray(bits, np.uint16).astype(np.int32)
    return np.where(b & 0x8000, -(b & 0x7FFF) - 1, b)


def check_dequant_inverse(codes, scales, cols, rhat_bits, lam, gpu_bits, ref=None):
    """Inverse dequantiser (v R^T, then times Lambda) against the exact value rounded once to
    bf16 (the oracle's definition).  The kernel computes in fp32: 32 exact products summed on
    the tensor cores, then one multiply by Lambda, then the rounding to bf16.  Its fp32 value is
    within A = 2^-18 sum_n |v_n||R[k][n]| Lambda_k + 2^-23 |x| of the exact x (sum of 32 terms:
    at most 31 roundings of 2^-24 of the running sum, doubled for margin; the Lambda multiply and
    the accumulator's last rounding).  So an output must be the correctly rounded bf16, except
    where [x - A, x + A] holds a bf16 rounding midpoint: there either rounding is right.  Returns
    the number of outputs that differ from the correctly rounded value (all of them at such
    midpoints); raises on any other difference."""
    if ref is None:
        ref = oracle.dequantize(codes, scales, cols, rhat_bits, lam, want_f64=True)
    ref_bits, ref64 = ref
    rows = ref_bits.shape[0]
    v = bf16_to_f64(oracle.dequantize(codes, scales, cols))
    rr = bf16_to_f64(rhat_bits)
    s_abs = (np.abs(v).reshape(rows, cols // 32, 32) @ np.abs(rr).T).reshape(rows, cols)
    if lam is not None:
        s_abs = s_abs * np.asarray(lam, np.float64)[None, :]
    acc = 2.0 ** -18 * s_abs + 2.0 ** -23 * np.abs(ref64)
    lo = _bf16_order(bf16_rne_bits(ref64 - acc))
    hi = _bf16_order(bf16_rne_bits(ref64 + acc))
    got = _bf16_order(gpu_bits)
    bad = (got < lo) | (got > hi)
    if bad.any():
        r, c = np.argwhere(bad)[0]
        raise AssertionError(f"inverse dequantise at ({r},{c}): gpu {bf16_to_f64(gpu_bits)[r, c]!r}, exact "
                             f"{ref64[r, c]!r} (correctly rounded {bf16_to_f64(ref_bits)[r, c]!r}), fp32 bound "
                             f"{acc[r, c]!r}")
    return int((np.asarray(gpu_bits, np.uint16) != ref_bits).sum())

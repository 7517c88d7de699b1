"""CPU oracle for the fused smooth-rotate-MXFP4 path -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline /
reference legs may import this package.  The product path (the CUDA library
and its Python binding) never imports or calls it, and the two share no code.

The arithmetic lives in ``mxq_oracle.c`` (plain double-precision C, built with
gcc, no fast-math, no FMA contraction); this module only marshals numpy arrays
into it.  What each function computes, and the page passages it follows, is
stated in the C file's header.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from typing import Optional

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "mxq_oracle.c")
_LIB = os.path.join(_HERE, "libmxq_oracle.so")

GROUP = 32


def build(force: bool = False) -> str:
    """Compile the oracle into ``oracle/libmxq_oracle.so`` (gcc, OpenMP)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        cmd = ["gcc", "-O2", "-std=c11", "-fno-fast-math", "-ffp-contract=off", "-fopenmp",
               "-shared", "-fPIC", "-o", _LIB + ".tmp", _SRC, "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(_LIB + ".tmp", _LIB)
    return _LIB


_lib = None


def build_variant(mutant: int) -> str:
    """Compile the oracle with planted mistake `mutant` (see the C file's list) into
    ``oracle/_mutants/`` -- for the pin-sensitivity test only; returns the library path."""
    out_dir = os.path.join(_HERE, "_mutants")
    os.makedirs(out_dir, exist_ok=True)
    path = os.path.join(out_dir, f"libmxq_oracle_m{int(mutant)}.so")
    if not os.path.exists(path) or os.path.getmtime(path) < os.path.getmtime(_SRC):
        cmd = ["gcc", "-O2", "-std=c11", "-fno-fast-math", "-ffp-contract=off", "-fopenmp",
               f"-DMXQ_MUTANT={int(mutant)}", "-shared", "-fPIC", "-o", path + ".tmp", _SRC, "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(path + ".tmp", path)
    return path


class use_library:
    """Context manager: every oracle call inside uses the library at `path` (test infrastructure)."""

    def __init__(self, path: str):
        self.path = path
        self.saved = None

    def __enter__(self):
        global _lib
        self.saved = lib()
        _lib = _bind(ctypes.CDLL(self.path))
        return _lib

    def __exit__(self, *exc):
        global _lib
        _lib = self.saved
        return False


def lib():
    global _lib
    if _lib is None:
        build()
        _lib = _bind(ctypes.CDLL(_LIB))
    return _lib


def _bind(L):
    """Declare every entry point's argument and result types on a loaded oracle library."""
    P = ctypes.c_void_p
    I64 = ctypes.c_int64
    I = ctypes.c_int
    L.mxq_oracle_e2m1_code.argtypes = [ctypes.c_double]
    L.mxq_oracle_e2m1_code.restype = I
    L.mxq_oracle_e2m1_value.argtypes = [I]
    L.mxq_oracle_e2m1_value.restype = ctypes.c_double
    L.mxq_oracle_e8m0_byte.argtypes = [ctypes.c_double]
    L.mxq_oracle_e8m0_byte.restype = I
    L.mxq_oracle_e8m0_value.argtypes = [I]
    L.mxq_oracle_e8m0_value.restype = ctypes.c_double
    L.mxq_oracle_quantize_group_at.argtypes = [P, I, P, P, P]
    L.mxq_oracle_quantize_group_at.restype = I
    L.mxq_oracle_rotate_f64.argtypes = [P, I64, I64, P, P, P, I]
    L.mxq_oracle_rotate_f64.restype = I
    L.mxq_oracle_quantize.argtypes = [P, I64, I64, P, P, P, P, P, P, I]
    L.mxq_oracle_quantize.restype = I
    L.mxq_oracle_smooth_rotate_quantize.argtypes = [P, I64, I64, P, P, P, P, P, P, P, P, P, I]
    L.mxq_oracle_weight_rotate_quantize.argtypes = [P, I64, I64, P, P, P, P, P, P, P, P, P, I]
    L.mxq_oracle_weight_rotate_quantize.restype = I
    L.mxq_oracle_e4m3_value.argtypes = [I]
    L.mxq_oracle_e4m3_value.restype = ctypes.c_double
    L.mxq_oracle_e4m3_code.argtypes = [ctypes.c_double]
    L.mxq_oracle_e4m3_code.restype = I
    L.mxq_oracle_nvfp4_block_at.argtypes = [P, I, ctypes.c_float, P, P, P]
    L.mxq_oracle_nvfp4_block_at.restype = I
    L.mxq_oracle_nvfp4_quantize.argtypes = [P, I64, I64, P, P, ctypes.c_float, P, P, P, P, P, P, P, I]
    L.mxq_oracle_nvfp4_quantize.restype = I
    L.mxq_oracle_scales_to_mma.argtypes = [P, I64, I64, P]
    L.mxq_oracle_scales_to_mma.restype = I
    L.mxq_oracle_mxfp4_gemm.argtypes = [P, P, P, P, I64, I64, I64, P, I]
    L.mxq_oracle_nvfp4_gemm.argtypes = [P, P, ctypes.c_float, P, P, ctypes.c_float, I64, I64, I64, P, I]
    L.mxq_oracle_nvfp4_gemm.restype = I
    L.mxq_oracle_mxfp4_gemm.restype = I
    L.mxq_oracle_block_rotate_quantize.argtypes = [P, I64, I64, I, P, P, P, P, P, P, P, P, P, I]
    L.mxq_oracle_block_rotate_quantize.restype = I
    L.mxq_oracle_smooth_rotate_quantize.restype = I
    L.mxq_oracle_dequantize.argtypes = [P, P, I64, I64, P, P, P, P, I]
    L.mxq_oracle_dequantize.restype = I
    L.mxq_oracle_group_error.argtypes = [P, I64, I64, P, P, P, P, I]
    L.mxq_oracle_group_error.restype = I
    L.mxq_oracle_givens.argtypes = [I, I, P, P]
    L.mxq_oracle_givens.restype = None
    L.mxq_oracle_rotation_search.argtypes = [P, I64, I64, P, I, I, P, P, P, P, I]
    L.mxq_oracle_rotation_search.restype = I
    L.mxq_oracle_bf16_to_double.argtypes = [P, P, I64]
    L.mxq_oracle_bf16_to_double.restype = None
    L.mxq_oracle_double_to_bf16.argtypes = [P, P, I64]
    L.mxq_oracle_double_to_bf16.restype = None
    return L


def _ptr(a: Optional[np.ndarray]):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


def default_threads() -> int:
    return max(1, len(os.sched_getaffinity(0)) if hasattr(os, "sched_getaffinity") else os.cpu_count() or 1)


# ------------------------------------------------------------------ scalar rules

def e2m1_code(u: float) -> int:
    return int(lib().mxq_oracle_e2m1_code(float(u)))


def e2m1_value(code: int) -> float:
    return float(lib().mxq_oracle_e2m1_value(int(code)))


def e8m0_byte(amax: float) -> int:
    return int(lib().mxq_oracle_e8m0_byte(float(amax)))


def e8m0_value(byte: int) -> float:
    return float(lib().mxq_oracle_e8m0_value(int(byte)))


def quantize_group_at(y, byte: int):
    """Codes (unpacked, 32), element flags and alternative codes for one group at a given scale byte."""
    y = _c(y, np.float64)
    assert y.shape == (GROUP,)
    codes = np.zeros(GROUP, np.uint8)
    flags = np.zeros(GROUP, np.uint8)
    alt = np.zeros(GROUP, np.uint8)
    lib().mxq_oracle_quantize_group_at(_ptr(y), int(byte), _ptr(codes), _ptr(flags), _ptr(alt))
    return codes, flags, alt


# ------------------------------------------------------------------ matrices

def bf16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    bits = _c(bits, np.uint16)
    out = np.empty(bits.shape, np.float64)
    lib().mxq_oracle_bf16_to_double(_ptr(bits), _ptr(out), bits.size)
    return out


def f64_to_bf16_bits(v: np.ndarray) -> np.ndarray:
    v = _c(v, np.float64)
    out = np.empty(v.shape, np.uint16)
    lib().mxq_oracle_double_to_bf16(_ptr(v), _ptr(out), v.size)
    return out


def rotate_f64(x: np.ndarray, r: np.ndarray, lam: Optional[np.ndarray] = None,
               threads: int = 1) -> np.ndarray:
    """Y = (X / lam) * R^, group by group, in double.  x: [rows, cols] float64, r: [32,32] [k][n]."""
    x = _c(x, np.float64)
    r = _c(r, np.float64)
    rows, cols = x.shape
    lam64 = None if lam is None else _c(lam, np.float64)
    y = np.empty_like(x)
    rc = lib().mxq_oracle_rotate_f64(_ptr(x), rows, cols, _ptr(r), _ptr(lam64), _ptr(y), threads)
    if rc:
        raise ValueError("oracle rotate: bad shape")
    return y


def quantize(y: np.ndarray, flags: bool = False, threads: int = 1) -> dict:
    """Steps 4-8 on a [rows, cols] float64 matrix of rotated values."""
    y = _c(y, np.float64)
    rows, cols = y.shape
    G = cols // GROUP
    out = {"codes": np.zeros((rows, cols // 2), np.uint8), "scales": np.zeros((rows, G), np.uint8)}
    if flags:
        out.update(eflags=np.zeros((rows, cols), np.uint8), alt=np.zeros((rows, cols), np.uint8),
                   gflags=np.zeros((rows, G), np.uint8), alt_scales=np.zeros((rows, G), np.uint8))
    g = out.get
    rc = lib().mxq_oracle_quantize(_ptr(y), rows, cols, _ptr(out["codes"]), _ptr(out["scales"]),
                                   _ptr(g("eflags")), _ptr(g("alt")), _ptr(g("gflags")),
                                   _ptr(g("alt_scales")), threads)
    if rc:
        raise ValueError("oracle quantize: bad shape")
    return out


def smooth_rotate_quantize(x_bits: np.ndarray, rhat_bits: np.ndarray, lam: Optional[np.ndarray] = None,
                           want_y: bool = False, flags: bool = False, threads: int = 1) -> dict:
    """The whole path from bf16 bit patterns: returns codes, scales (+ y, flags)."""
    x_bits = _c(x_bits, np.uint16)
    rhat_bits = _c(rhat_bits, np.uint16)
    assert rhat_bits.shape == (GROUP, GROUP)
    rows, cols = x_bits.shape
    if cols % GROUP:
        raise ValueError("cols must be a multiple of 32")
    G = cols // GROUP
    lam32 = None if lam is None else _c(lam, np.float32)
    out = {"codes": np.zeros((rows, cols // 2), np.uint8), "scales": np.zeros((rows, G), np.uint8)}
    if want_y:
        out["y"] = np.zeros((rows, cols), np.float64)
    if flags:
        out.update(eflags=np.zeros((rows, cols), np.uint8), alt=np.zeros((rows, cols), np.uint8),
                   gflags=np.zeros((rows, G), np.uint8), alt_scales=np.zeros((rows, G), np.uint8))
    g = out.get
    rc = lib().mxq_oracle_smooth_rotate_quantize(
        _ptr(x_bits), rows, cols, _ptr(rhat_bits), _ptr(lam32), _ptr(out["codes"]), _ptr(out["scales"]),
        _ptr(g("y")), _ptr(g("eflags")), _ptr(g("alt")), _ptr(g("gflags")), _ptr(g("alt_scales")), threads)
    if rc:
        raise ValueError("oracle: bad shape")
    return out


def weight_rotate_quantize(wt_bits: np.ndarray, rhat_bits: np.ndarray, lam: Optional[np.ndarray] = None,
                           want_y: bool = False, flags: bool = False, threads: int = 1) -> dict:
    """MXFP4 of the absorbed weights: each row of Wt = W^T times Λ, then R̂ per group (§3.3)."""
    wt_bits = _c(wt_bits, np.uint16)
    rhat_bits = _c(rhat_bits, np.uint16)
    rows, cols = wt_bits.shape
    G = cols // GROUP
    lam32 = None if lam is None else _c(lam, np.float32)
    out = {"codes": np.zeros((rows, cols // 2), np.uint8), "scales": np.zeros((rows, G), np.uint8)}
    if want_y:
        out["y"] = np.zeros((rows, cols), np.float64)
    if flags:
        out.update(eflags=np.zeros((rows, cols), np.uint8), alt=np.zeros((rows, cols), np.uint8),
                   gflags=np.zeros((rows, G), np.uint8), alt_scales=np.zeros((rows, G), np.uint8))
    g = out.get
    rc = lib().mxq_oracle_weight_rotate_quantize(
        _ptr(wt_bits), rows, cols, _ptr(rhat_bits), _ptr(lam32), _ptr(out["codes"]), _ptr(out["scales"]),
        _ptr(g("y")), _ptr(g("eflags")), _ptr(g("alt")), _ptr(g("gflags")), _ptr(g("alt_scales")), threads)
    if rc:
        raise ValueError("oracle: bad shape")
    return out


def e4m3_value(code: int) -> float:
    return lib().mxq_oracle_e4m3_value(int(code))


def e4m3_code(v: float) -> int:
    return lib().mxq_oracle_e4m3_code(float(v))


def nvfp4_block_at(y16, sb: int, s_t: float):
    """Codes (+ flags, alternatives) of one 16-value block under E4M3 scale byte sb."""
    y = _c(np.asarray(y16, np.float64), np.float64)
    codes = np.zeros(16, np.uint8)
    flags = np.zeros(16, np.uint8)
    alt = np.zeros(16, np.uint8)
    lib().mxq_oracle_nvfp4_block_at(_ptr(y), int(sb), float(s_t), _ptr(codes), _ptr(flags), _ptr(alt))
    return codes, flags, alt


def nvfp4_quantize(x_bits: np.ndarray, rhat_bits: np.ndarray, lam: Optional[np.ndarray], s_t: float,
                   want_y: bool = False, flags: bool = False, threads: int = 1) -> dict:
    """NVFP4 of X·Λ⁻¹·R̂ (blocks of 16, E4M3 block scales, fp32 tensor scale s_t)."""
    x_bits = _c(x_bits, np.uint16)
    rhat_bits = _c(rhat_bits, np.uint16)
    rows, cols = x_bits.shape
    NB = cols // 16
    lam32 = None if lam is None else _c(lam, np.float32)
    out = {"codes": np.zeros((rows, cols // 2), np.uint8), "scales": np.zeros((rows, NB), np.uint8)}
    if want_y:
        out["y"] = np.zeros((rows, cols), np.float64)
    if flags:
        out.update(eflags=np.zeros((rows, cols), np.uint8), alt=np.zeros((rows, cols), np.uint8),
                   bflags=np.zeros((rows, NB), np.uint8), alt_scales=np.zeros((rows, NB), np.uint8))
    g = out.get
    rc = lib().mxq_oracle_nvfp4_quantize(
        _ptr(x_bits), rows, cols, _ptr(rhat_bits), _ptr(lam32), float(s_t), _ptr(out["codes"]), _ptr(out["scales"]),
        _ptr(g("y")), _ptr(g("eflags")), _ptr(g("alt")), _ptr(g("bflags")), _ptr(g("alt_scales")), threads)
    if rc:
        raise ValueError("oracle: bad shape")
    return out


def scales_to_mma(scales: np.ndarray) -> np.ndarray:
    """Row-major E8M0 scales [rows, G] -> the block-scaled MMA's 512-byte atoms (flat uint8)."""
    scales = _c(scales, np.uint8)
    rows, G = scales.shape
    out = np.zeros(((rows + 127) // 128) * ((G + 3) // 4) * 512, np.uint8)
    if lib().mxq_oracle_scales_to_mma(_ptr(scales), rows, G, _ptr(out)):
        raise ValueError("oracle scales_to_mma: bad shape")
    return out


def mxfp4_gemm(a_codes: np.ndarray, a_scales: np.ndarray, b_codes: np.ndarray, b_scales: np.ndarray,
               threads: int = 1) -> np.ndarray:
    """Y[m, n] = sum_k deq(A)[m, k] deq(B)[n, k] in double (both operands K-major MXFP4)."""
    a_codes, a_scales = _c(a_codes, np.uint8), _c(a_scales, np.uint8)
    b_codes, b_scales = _c(b_codes, np.uint8), _c(b_scales, np.uint8)
    M, K = a_codes.shape[0], a_codes.shape[1] * 2
    N = b_codes.shape[0]
    assert b_codes.shape[1] * 2 == K and a_scales.shape == (M, K // GROUP) and b_scales.shape == (N, K // GROUP)
    y = np.zeros((M, N), np.float64)
    if lib().mxq_oracle_mxfp4_gemm(_ptr(a_codes), _ptr(a_scales), _ptr(b_codes), _ptr(b_scales), M, N, K, _ptr(y),
                                   threads):
        raise ValueError("oracle mxfp4_gemm: bad shape")
    return y


def nvfp4_gemm(a_codes: np.ndarray, a_scales: np.ndarray, a_tscale: float, b_codes: np.ndarray,
               b_scales: np.ndarray, b_tscale: float, threads: int = 1) -> np.ndarray:
    """Y[m, n] = sum_k deq(A)[m, k] deq(B)[n, k] in double, NVFP4 operands (E4M3 per 16 k, fp32 tensor scales)."""
    a_codes, a_scales = _c(a_codes, np.uint8), _c(a_scales, np.uint8)
    b_codes, b_scales = _c(b_codes, np.uint8), _c(b_scales, np.uint8)
    M, K = a_codes.shape[0], a_codes.shape[1] * 2
    N = b_codes.shape[0]
    assert b_codes.shape[1] * 2 == K and a_scales.shape == (M, K // 16) and b_scales.shape == (N, K // 16)
    y = np.zeros((M, N), np.float64)
    if lib().mxq_oracle_nvfp4_gemm(_ptr(a_codes), _ptr(a_scales), float(a_tscale), _ptr(b_codes), _ptr(b_scales),
                                   float(b_tscale), M, N, K, _ptr(y), threads):
        raise ValueError("oracle nvfp4_gemm: bad shape")
    return y


def block_rotate_quantize(x_bits: np.ndarray, r_bits: np.ndarray, lam: Optional[np.ndarray] = None,
                          want_y: bool = False, flags: bool = False, threads: int = 1) -> dict:
    """Rotation blocks of B = r_bits.shape[0] columns, MXFP4 groups of 32 (the §4.3 block-size variants)."""
    x_bits = _c(x_bits, np.uint16)
    r_bits = _c(r_bits, np.uint16)
    blk = r_bits.shape[0]
    assert r_bits.shape == (blk, blk)
    rows, cols = x_bits.shape
    G = cols // GROUP
    lam32 = None if lam is None else _c(lam, np.float32)
    out = {"codes": np.zeros((rows, cols // 2), np.uint8), "scales": np.zeros((rows, G), np.uint8)}
    if want_y:
        out["y"] = np.zeros((rows, cols), np.float64)
    if flags:
        out.update(eflags=np.zeros((rows, cols), np.uint8), alt=np.zeros((rows, cols), np.uint8),
                   gflags=np.zeros((rows, G), np.uint8), alt_scales=np.zeros((rows, G), np.uint8))
    g = out.get
    rc = lib().mxq_oracle_block_rotate_quantize(
        _ptr(x_bits), rows, cols, blk, _ptr(r_bits), _ptr(lam32), _ptr(out["codes"]), _ptr(out["scales"]),
        _ptr(g("y")), _ptr(g("eflags")), _ptr(g("alt")), _ptr(g("gflags")), _ptr(g("alt_scales")), threads)
    if rc:
        raise ValueError("oracle: bad shape or block size")
    return out


def dequantize(codes: np.ndarray, scales: np.ndarray, cols: int, rhat_bits: Optional[np.ndarray] = None,
               lam: Optional[np.ndarray] = None, want_f64: bool = False, threads: int = 1):
    """bf16 bit patterns of the dequantised matrix (and optionally the double before rounding)."""
    codes = _c(codes, np.uint8)
    scales = _c(scales, np.uint8)
    rows = codes.shape[0]
    assert codes.shape == (rows, cols // 2) and scales.shape == (rows, cols // GROUP)
    rb = None if rhat_bits is None else _c(rhat_bits, np.uint16)
    lam32 = None if lam is None else _c(lam, np.float32)
    out = np.zeros((rows, cols), np.uint16)
    f64 = np.zeros((rows, cols), np.float64) if want_f64 else None
    rc = lib().mxq_oracle_dequantize(_ptr(codes), _ptr(scales), rows, cols, _ptr(rb), _ptr(lam32),
                                     _ptr(out), _ptr(f64), threads)
    if rc:
        raise ValueError("oracle dequantize: bad shape")
    return (out, f64) if want_f64 else out


def group_error(x_bits: np.ndarray, rhat_bits: np.ndarray, lam: Optional[np.ndarray] = None,
                threads: int = 1):
    """Per-group MXFP4 error ||Q(y) - y|| / ||y|| [rows, cols/32] (float64) and its mean."""
    x_bits = _c(x_bits, np.uint16)
    rhat_bits = _c(rhat_bits, np.uint16)
    rows, cols = x_bits.shape
    lam32 = None if lam is None else _c(lam, np.float32)
    err = np.zeros((rows, cols // GROUP), np.float64)
    mean = np.zeros(1, np.float64)
    rc = lib().mxq_oracle_group_error(_ptr(x_bits), rows, cols, _ptr(rhat_bits), _ptr(lam32), _ptr(err),
                                      _ptr(mean), threads)
    if rc:
        raise ValueError("oracle group_error: bad shape")
    return err, float(mean[0])


def givens(a: int, n_angle: int):
    c = ctypes.c_double()
    s = ctypes.c_double()
    lib().mxq_oracle_givens(int(a), int(n_angle), ctypes.byref(c), ctypes.byref(s))
    return c.value, s.value


def rotation_search(x_bits: np.ndarray, lam: Optional[np.ndarray] = None, max_steps: int = 128,
                    n_angle: int = 32, threads: int = 1) -> dict:
    """The outlier-aware greedy Givens search (DuQuant++ write-up, §3.2).

    Returns R (float64 [32, 32]), its bf16 rounding, the worst group, the number of
    steps taken, the per-step trace of (d, j, angle) and the L-inf norm before each step.
    """
    x_bits = _c(x_bits, np.uint16)
    rows, cols = x_bits.shape
    lam32 = None if lam is None else _c(lam, np.float32)
    R = np.zeros((GROUP, GROUP), np.float64)
    trace = np.zeros((max(max_steps, 1), 3), np.int32)
    linf = np.zeros(max_steps + 1, np.float64)
    group = np.zeros(1, np.int64)
    n = lib().mxq_oracle_rotation_search(_ptr(x_bits), rows, cols, _ptr(lam32), int(max_steps), int(n_angle),
                                         _ptr(R), _ptr(group), _ptr(trace), _ptr(linf), threads)
    if n < 0:
        raise ValueError("oracle rotation_search: bad argument")
    return {"R": R, "rhat_bits": f64_to_bf16_bits(R), "group": int(group[0]), "steps": n, "trace": trace[:n],
            "linf": linf[:n + 1]}


def unpack_codes(codes: np.ndarray) -> np.ndarray:
    """[rows, cols/2] packed bytes -> [rows, cols] 4-bit codes (even column = low nibble)."""
    codes = np.asarray(codes, np.uint8)
    out = np.empty(codes.shape[:-1] + (codes.shape[-1] * 2,), np.uint8)
    out[..., 0::2] = codes & 15
    out[..., 1::2] = codes >> 4
    return out

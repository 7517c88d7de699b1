"""Seeded synthetic activation workloads for the fused smooth-rotate-MXFP4 path.

This module only draws inputs: it holds none of the method's arithmetic (no
smoothing, rotation or quantisation).  Both the CUDA path's tests/benchmark and
the CPU oracle's tests take their inputs from here, so the two sides see the
same bits.

The shapes and value structure follow the activations the DuQuant++ write-up
(jsqmd.com/news/928156) talks about: LLaMA-3 QKV/O-projection inputs
(hidden 4096) and down-projection inputs (intermediate 14336) with "normal"
channel outliers and a few tokens with massive outliers (§1, §2.1, §4.1), a
data-agnostic Hadamard block rotation as the baseline rotation (§2.2), and a
SmoothQuant-style per-channel scale Λ (§3.1).  The real activations and the
WikiText-2 calibration set are not available, so these seeded stand-ins replace
them.

Recipe (all numbers drawn with ``numpy.random.default_rng``; seeds are
``1000 + cfg`` for X, ``2000 + cfg`` for R̂ and ``3000 + cfg`` for outlier
placement; values are drawn in float64 and rounded to bf16 by torch):

====  =================  ==================================================================
cfg   shape [rows,cols]  contents
====  =================  ==================================================================
1     128 x 4096         N(0,1); channels {7,1000,2049,3500} x50; token 3 x1000; R̂ = QR
2     8192 x 4096        N(0,1); 41 channels (1 %) x exp(U(ln 20, ln 100)); R̂ = QR
3     8192 x 14336       Student-t(3); 8 tokens x 4 channels set to ±10^U(3,4); R̂ = QR
4     65536 x 8192       N(0,1); 41 channels (0.5 %) x50; R̂ = H32·D (random ±1 diagonal)
5     32768 x 14336      as cfg 3; Λ_j = clip(max_t|X_tj|^0.5, 1e-2, 1e2) (fp32); R̂ = QR
====  =================  ==================================================================

"QR" is the sign-fixed QR factor of a 32x32 standard normal matrix (a Haar
random orthogonal matrix).
"""
from __future__ import annotations

import dataclasses
import math
from typing import Optional

import numpy as np
import torch

GROUP = 32

CONFIG_SHAPES = {
    1: (128, 4096),
    2: (8192, 4096),
    3: (8192, 14336),
    4: (65536, 8192),
    5: (32768, 14336),
}

CONFIG_NAMES = {
    1: "outlier-toy 128x4096",
    2: "qkv/o-proj input 8192x4096",
    3: "down-proj input 8192x14336",
    4: "large prefill 65536x8192 (Hadamard R)",
    5: "down-proj 32768x14336 with smoothing",
}

# Rows drawn per chunk when generating large matrices (bounds host memory).
_CHUNK_ELEMS = 1 << 24


@dataclasses.dataclass
class Workload:
    """One synthetic input: X (bf16, CPU), R̂ (bf16 and the float64 it came from), Λ or None."""

    cfg: int
    x: torch.Tensor                 # bf16 [rows, cols], CPU, contiguous
    rhat: torch.Tensor              # bf16 [32, 32], CPU, row-major [k][n]
    rhat_f64: np.ndarray            # float64 [32, 32] before bf16 rounding
    lam: Optional[torch.Tensor]     # float32 [cols] or None
    outlier_rows: np.ndarray        # token rows that carry planted outliers (may be empty)
    outlier_cols: np.ndarray        # channels that carry planted outliers (may be empty)

    @property
    def rows(self) -> int:
        return int(self.x.shape[0])

    @property
    def cols(self) -> int:
        return int(self.x.shape[1])


def to_bf16(a: np.ndarray) -> torch.Tensor:
    """Round a float array to bf16 (round-to-nearest-even, through torch)."""
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(torch.bfloat16)


def bf16_bits(t: torch.Tensor) -> np.ndarray:
    """The raw uint16 bit patterns of a bf16 CPU tensor."""
    assert t.dtype == torch.bfloat16
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)


def bf16_from_bits(bits: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(bits, dtype=np.uint16).view(np.int16)).view(torch.bfloat16)


# ----------------------------------------------------------------------------- R̂

def haar_orthogonal(seed: int, n: int = GROUP) -> np.ndarray:
    """Sign-fixed QR factor of an n x n standard normal matrix (float64)."""
    rng = np.random.default_rng(seed)
    g = rng.standard_normal((n, n))
    q, r = np.linalg.qr(g)
    q = q * np.sign(np.diag(r))[None, :]
    return q


def sylvester_hadamard(n: int = GROUP) -> np.ndarray:
    """Sylvester Hadamard matrix of order n (entries ±1), n a power of two."""
    h = np.ones((1, 1))
    while h.shape[0] < n:
        h = np.block([[h, h], [h, -h]])
    return h


def hadamard_rhat(seed: int, n: int = GROUP) -> np.ndarray:
    """Normalised Hadamard times a random ±1 diagonal, H·D/sqrt(n) (float64)."""
    rng = np.random.default_rng(seed)
    d = rng.choice(np.array([-1.0, 1.0]), size=n)
    return sylvester_hadamard(n) / math.sqrt(n) * d[None, :]


def rhat_tensor(r: np.ndarray) -> torch.Tensor:
    return to_bf16(r).contiguous()


# ----------------------------------------------------------------------------- X

def _fill_chunks(rows: int, cols: int, draw) -> torch.Tensor:
    """Fill a bf16 [rows, cols] tensor chunk by chunk; draw(n_rows) returns float64."""
    out = torch.empty((rows, cols), dtype=torch.bfloat16)
    step = max(1, _CHUNK_ELEMS // max(cols, 1))
    for r0 in range(0, rows, step):
        r1 = min(rows, r0 + step)
        out[r0:r1] = to_bf16(draw(r1 - r0))
    return out


def gaussian_with_channel_scale(rng, rows, cols, chan_scale):
    return _fill_chunks(rows, cols, lambda n: rng.standard_normal((n, cols)) * chan_scale[None, :])


def make_config(cfg: int, rows: Optional[int] = None, cols: Optional[int] = None) -> Workload:
    """Build config ``cfg`` (1..5).  ``rows``/``cols`` override the shape (same recipe)."""
    if cfg not in CONFIG_SHAPES:
        raise ValueError(f"unknown config {cfg}")
    R0, C0 = CONFIG_SHAPES[cfg]
    rows = R0 if rows is None else int(rows)
    cols = C0 if cols is None else int(cols)
    if cols % GROUP:
        raise ValueError("cols must be a multiple of 32")
    rng_x = np.random.default_rng(1000 + cfg)
    rng_o = np.random.default_rng(3000 + cfg)
    lam = None
    orows = np.zeros(0, dtype=np.int64)
    ocols = np.zeros(0, dtype=np.int64)

    if cfg == 1:
        scale = np.ones(cols)
        ocols = np.array([c for c in (7, 1000, 2049, 3500) if c < cols], dtype=np.int64)
        scale[ocols] = 50.0
        x = gaussian_with_channel_scale(rng_x, rows, cols, scale)
        if rows > 3:
            x[3] = (x[3].float() * 1000.0).to(torch.bfloat16)
            orows = np.array([3], dtype=np.int64)
        rhat = haar_orthogonal(2000 + cfg)
    elif cfg == 2:
        n_out = max(1, int(round(0.01 * cols)))
        ocols = np.sort(rng_o.choice(cols, size=n_out, replace=False)).astype(np.int64)
        scale = np.ones(cols)
        scale[ocols] = np.exp(rng_o.uniform(math.log(20.0), math.log(100.0), size=n_out))
        x = gaussian_with_channel_scale(rng_x, rows, cols, scale)
        rhat = haar_orthogonal(2000 + cfg)
    elif cfg in (3, 5):
        x = _fill_chunks(rows, cols, lambda n: rng_x.standard_t(3.0, size=(n, cols)))
        n_tok = min(8, rows)
        orows = np.sort(rng_o.choice(rows, size=n_tok, replace=False)).astype(np.int64)
        ocols = np.sort(rng_o.choice(cols, size=min(4, cols), replace=False)).astype(np.int64)
        mags = 10.0 ** rng_o.uniform(3.0, 4.0, size=(n_tok, ocols.size))
        signs = rng_o.choice(np.array([-1.0, 1.0]), size=(n_tok, ocols.size))
        vals = to_bf16(mags * signs)
        for i, r in enumerate(orows):
            x[int(r), torch.from_numpy(ocols)] = vals[i]
        rhat = haar_orthogonal(2000 + cfg)
        if cfg == 5:
            lam = smoothing_scale(x)
    elif cfg == 4:
        n_out = max(1, int(round(0.005 * cols)))
        ocols = np.sort(rng_o.choice(cols, size=n_out, replace=False)).astype(np.int64)
        scale = np.ones(cols)
        scale[ocols] = 50.0
        x = gaussian_with_channel_scale(rng_x, rows, cols, scale)
        rhat = hadamard_rhat(2000 + cfg)
    return Workload(cfg=cfg, x=x.contiguous(), rhat=rhat_tensor(rhat), rhat_f64=rhat,
                    lam=lam, outlier_rows=orows, outlier_cols=ocols)


def smoothing_scale(x: torch.Tensor, alpha: float = 0.5, lo: float = 1e-2, hi: float = 1e2) -> torch.Tensor:
    """Weight-free stand-in for the SmoothQuant scale: clip(max_t |X_tj|^alpha, lo, hi), fp32.

    The write-up's Λ_j also divides by max|W_j|^(1-alpha) (§3.1); no weights
    exist here, so that factor is taken as 1.
    """
    colmax = torch.zeros(x.shape[1], dtype=torch.float64)
    step = max(1, _CHUNK_ELEMS // max(x.shape[1], 1))
    for r0 in range(0, x.shape[0], step):
        blk = x[r0:r0 + step].to(torch.float64).abs().amax(dim=0)
        colmax = torch.maximum(colmax, blk)
    lam = colmax.pow(alpha).clamp(lo, hi)
    return lam.to(torch.float32).contiguous()


def random_bf16(rows: int, cols: int, seed: int, scale: float = 1.0) -> torch.Tensor:
    """Plain N(0, scale^2) bf16 matrix for small parity cases."""
    rng = np.random.default_rng(seed)
    return to_bf16(rng.standard_normal((rows, cols)) * scale).contiguous()


def random_lambda(cols: int, seed: int, lo: float = 0.05, hi: float = 20.0) -> torch.Tensor:
    """Log-uniform positive fp32 per-channel scales for small parity cases."""
    rng = np.random.default_rng(seed)
    return torch.from_numpy(np.exp(rng.uniform(math.log(lo), math.log(hi), size=cols)).astype(np.float32))


def permutation_rhat(seed: int, n: int = GROUP) -> np.ndarray:
    rng = np.random.default_rng(seed)
    p = rng.permutation(n)
    m = np.zeros((n, n))
    m[np.arange(n), p] = 1.0
    return m


def sample_rows(rows: int, n: int, seed: int, must: np.ndarray = np.zeros(0, dtype=np.int64)) -> np.ndarray:
    """A sorted row sample: first, last, the planted-outlier rows and n seeded random rows."""
    rng = np.random.default_rng(seed)
    pick = set(int(r) for r in must if 0 <= r < rows)
    pick.update({0, rows - 1})
    if rows > 0:
        pick.update(int(r) for r in rng.choice(rows, size=min(n, rows), replace=False))
    return np.array(sorted(pick), dtype=np.int64)

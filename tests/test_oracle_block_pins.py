"""Pins for the oracle's rotation-block-size variant (DuQuant++ write-up, §4.3 ablation: B = 16, 32, 64, 128).

  - B = 32 is the main path's oracle;
  - block-diagonal matrices reduce B = 64 and 128 to B = 32, and B = 16 to a
    block-diagonal 32 x 32 matrix;
  - a permutation that swaps the halves of a 64-block swaps MXFP4 groups;
  - the rotated values equal numpy's reshape-and-matmul in double.
"""
import numpy as np
import pytest
import scipy.linalg

import oracle
from workloads import synth


def _rbits(r):
    return synth.bf16_bits(synth.rhat_tensor(r))


def _x(rows, cols):
    return synth.bf16_bits(synth.make_config(2, rows=rows, cols=cols).x)


def _f64(bits):
    return (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


@pytest.mark.parametrize("use_lam", [False, True])
def test_block32_is_the_main_path(use_lam):
    xb = _x(40, 256)
    rb = _rbits(synth.haar_orthogonal(1, n=32))
    lam = synth.random_lambda(256, seed=4).numpy() if use_lam else None
    a = oracle.block_rotate_quantize(xb, rb, lam, want_y=True, flags=True)
    b = oracle.smooth_rotate_quantize(xb, rb, lam, want_y=True, flags=True)
    for k in b:
        assert np.array_equal(a[k], b[k]), k


@pytest.mark.parametrize("blk", [64, 128])
def test_block_diagonal_reduces_to_block32(blk):
    xb = _x(33, 512)
    r32 = _f64(_rbits(synth.haar_orthogonal(2, n=32)))
    big = scipy.linalg.block_diag(*([r32] * (blk // 32)))
    a = oracle.block_rotate_quantize(xb, _rbits(big), want_y=True)
    b = oracle.smooth_rotate_quantize(xb, _rbits(r32), want_y=True)
    assert np.array_equal(a["y"], b["y"])
    assert np.array_equal(a["codes"], b["codes"]) and np.array_equal(a["scales"], b["scales"])


def test_block16_is_a_block_diagonal_32():
    xb = _x(21, 160)
    r16 = _f64(_rbits(synth.haar_orthogonal(5, n=16)))
    a = oracle.block_rotate_quantize(xb, _rbits(r16), want_y=True)
    b = oracle.smooth_rotate_quantize(xb, _rbits(scipy.linalg.block_diag(r16, r16)), want_y=True)
    assert np.array_equal(a["y"], b["y"])
    assert np.array_equal(a["codes"], b["codes"]) and np.array_equal(a["scales"], b["scales"])


def test_half_swap_permutation_swaps_groups():
    xb = _x(17, 256)
    p = np.zeros((64, 64))
    for k in range(64):
        p[k, (k + 32) % 64] = 1.0           # column n of y takes x[(n + 32) mod 64]
    a = oracle.block_rotate_quantize(xb, _rbits(p))
    b = oracle.smooth_rotate_quantize(xb, _rbits(np.eye(32)))
    G = 256 // 32
    swap = np.arange(G).reshape(-1, 2)[:, ::-1].reshape(-1)
    assert np.array_equal(a["scales"], b["scales"][:, swap])
    assert np.array_equal(a["codes"].reshape(17, G, 16), b["codes"].reshape(17, G, 16)[:, swap])


@pytest.mark.parametrize("blk", [16, 64, 128])
@pytest.mark.parametrize("use_lam", [False, True])
def test_rotated_values_are_the_reshaped_matmul(blk, use_lam):
    rows, cols = 9, 384
    xb = _x(rows, cols)
    rb = _rbits(synth.haar_orthogonal(blk, n=blk))
    lam = synth.random_lambda(cols, seed=7).numpy() if use_lam else None
    a = oracle.block_rotate_quantize(xb, rb, lam, want_y=True)
    x = _f64(xb)
    if use_lam:
        x = x / lam.astype(np.float64)
    want = (x.reshape(-1, blk) @ _f64(rb)).reshape(rows, cols)
    assert np.allclose(a["y"], want, rtol=1e-12, atol=1e-12 * np.abs(want).max())
    # a transposed matrix gives something else
    wrong = (x.reshape(-1, blk) @ _f64(rb).T).reshape(rows, cols)
    assert not np.allclose(a["y"], wrong, rtol=1e-6)


def test_block_shape_errors():
    xb = _x(2, 96)
    with pytest.raises(ValueError):
        oracle.block_rotate_quantize(xb, _rbits(np.eye(64)))     # 96 is not a multiple of 64
    with pytest.raises(ValueError):
        oracle.block_rotate_quantize(xb[:, :48], _rbits(np.eye(16)))   # 48 is not a multiple of 32

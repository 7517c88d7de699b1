"""Pins for the oracle's outlier-aware rotation search (DuQuant++ write-up, §3.2).

Each pin checks the oracle against something other than itself:
  - the Givens grid against cos/sin of 2*atan(t);
  - a single spike, whose best one-step rotation has a closed form;
  - the worst-group choice, with Λ dividing (not multiplying) the activations;
  - R against the product of the traced Givens matrices, built here from math.cos/sin;
  - the final L-inf norm against numpy's block @ R;
  - every step of a tiny case against a brute-force search in numpy;
  - a block no rotation can improve;
  - the lower bound that orthogonality puts on L-inf.
"""
import math

import numpy as np
import pytest

import oracle
from workloads import synth


def _f64(bits):
    return (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def _bits(v):
    return synth.bf16_bits(synth.to_bf16(np.asarray(v, np.float64)))


def _grid_t(a, n):
    ap = a if a < n else a + 1
    return (ap - n) / n


def _givens_math(a, n):
    th = 2.0 * math.atan(_grid_t(a, n))
    return math.cos(th), math.sin(th)


def _gmat(d, j, a, n):
    """The 32x32 matrix G with (X @ G)[:, d] = c x_d - s x_j and (X @ G)[:, j] = s x_d + c x_j."""
    c, s = _givens_math(a, n)
    g = np.eye(32)
    g[d, d], g[j, d], g[d, j], g[j, j] = c, -s, s, c
    return g


@pytest.mark.parametrize("n", [1, 4, 32, 64])
def test_givens_grid_matches_trig(n):
    ts = []
    for a in range(2 * n):
        c, s = oracle.givens(a, n)
        cm, sm = _givens_math(a, n)
        assert c == pytest.approx(cm, abs=4e-16) and s == pytest.approx(sm, abs=4e-16)
        assert abs(c * c + s * s - 1.0) < 4e-16
        ts.append(_grid_t(a, n))
    # 2n distinct angles, t = 0 (the identity) left out, t = -1 and t = 1 both present
    assert len(set(ts)) == 2 * n and 0.0 not in ts and ts[0] == -1.0 and ts[-1] == 1.0


def test_single_spike_one_step_closed_form():
    n = 32
    rows, cols = 5, 128
    x = np.zeros((rows, cols))
    x[3, 2 * 32 + 7] = 8.0                # the spike: group 2, column 7 of the group
    x[1, 0] = 0.5                         # small values elsewhere keep group 0 from tying
    r = oracle.rotation_search(_bits(x), max_steps=1, n_angle=n)
    assert r["group"] == 2 and r["steps"] == 1
    d, j, a = r["trace"][0]
    assert d == 7 and j == 0              # every j ties; the first wins
    vals = [max(abs(c), abs(s)) for c, s in (_givens_math(b, n) for b in range(2 * n))]
    best = min(vals)
    assert a == vals.index(best)          # first of the two mirror angles
    assert r["linf"][0] == 8.0
    assert r["linf"][1] == pytest.approx(8.0 * best, rel=1e-15)


def test_worst_group_divides_by_lambda():
    rows, cols = 8, 96
    rng = np.random.default_rng(5)
    x = rng.uniform(-1, 1, (rows, cols))
    x[2, 40] = 20.0                       # group 1 holds the largest raw value
    x[6, 70] = 12.0                       # group 2 holds the second
    xb = _bits(x)
    assert oracle.rotation_search(xb, max_steps=0)["group"] == 1
    lam = np.ones(cols, np.float32)
    lam[40] = 4.0                         # 20 / 4 = 5 < 12: dividing moves the worst group to 2
    r = oracle.rotation_search(xb, lam=lam, max_steps=0)
    assert r["group"] == 2 and r["steps"] == 0
    assert np.array_equal(r["R"], np.eye(32)) and r["linf"][0] == 12.0
    lam[70] = 0.5                         # and multiplying instead would pick group 1
    assert oracle.rotation_search(xb, lam=lam, max_steps=0)["linf"][0] == 24.0


@pytest.mark.parametrize("use_lam", [False, True])
def test_r_is_the_traced_givens_product_and_matches_the_block(use_lam):
    n, K = 32, 48
    w = synth.make_config(2, rows=256, cols=512)
    xb = synth.bf16_bits(w.x)
    lam = synth.smoothing_scale(w.x).numpy() if use_lam else None
    r = oracle.rotation_search(xb, lam=lam, max_steps=K, n_angle=n, threads=4)
    assert r["steps"] == K
    prod = np.eye(32)
    for d, j, a in r["trace"]:
        prod = prod @ _gmat(d, j, a, n)
    assert np.abs(prod - r["R"]).max() < 1e-13
    assert np.abs(r["R"].T @ r["R"] - np.eye(32)).max() < 1e-13
    xs = _f64(xb)
    if use_lam:
        xs = xs / lam.astype(np.float64)
    g = r["group"]
    gmax = [np.abs(xs[:, k * 32:(k + 1) * 32]).max() for k in range(512 // 32)]
    assert g == int(np.argmax(gmax))
    block = xs[:, g * 32:(g + 1) * 32]
    assert r["linf"][0] == np.abs(block).max()
    assert r["linf"][-1] == pytest.approx(np.abs(block @ r["R"]).max(), rel=1e-13)
    # strictly decreasing, and never below the bound that orthogonality sets
    assert np.all(np.diff(r["linf"]) < 0)
    assert r["linf"][-1] >= np.sqrt((block ** 2).sum(axis=1)).max() / np.sqrt(32) * (1 - 1e-12)
    # the rotated block's norms are each row's norms
    assert np.allclose(np.linalg.norm(block @ r["R"], axis=1), np.linalg.norm(block, axis=1), rtol=1e-13)


def test_every_step_against_brute_force():
    n, K = 3, 6
    rng = np.random.default_rng(11)
    x = rng.standard_normal((4, 64)) * 3.0
    x[:, 32 + 5] *= 6.0                   # group 1 is the worst
    xb = _bits(x)
    r = oracle.rotation_search(xb, max_steps=K, n_angle=n)
    assert r["group"] == 1
    block = _f64(xb)[:, 32:64]
    R = np.eye(32)
    taken = 0
    for step in range(K):
        cur = np.abs(block).max()
        assert r["linf"][step] == pytest.approx(cur, rel=1e-14)
        d = int(np.argmax(np.abs(block).max(axis=0)))
        best, arg = cur, None
        for j in range(32):
            if j == d:
                continue
            for a in range(2 * n):
                v = np.abs(block @ _gmat(d, j, a, n)).max()
                if v < best * (1 - 1e-12):
                    best, arg = v, (d, j, a)
        if arg is None:
            break
        assert tuple(r["trace"][step]) == arg
        g = _gmat(*arg, n)
        block, R = block @ g, R @ g
        taken += 1
    assert r["steps"] == taken
    assert np.abs(R - r["R"]).max() < 1e-13


def test_block_that_no_rotation_improves():
    # Every row (1, 1, ..., 1): any Givens pair (x_d, x_j) = (1, 1) maps to
    # (c - s, s + c), whose larger magnitude is at least 1, so nothing is strictly lower.
    x = np.ones((6, 64))
    x[:, 32:] = 0.25
    r = oracle.rotation_search(_bits(x), max_steps=10, n_angle=16)
    assert r["steps"] == 0 and r["group"] == 0
    assert np.array_equal(r["R"], np.eye(32)) and list(r["linf"]) == [1.0]


def test_zero_steps_and_bad_arguments():
    xb = _bits(np.arange(2 * 64, dtype=np.float64).reshape(2, 64) / 64.0)
    r = oracle.rotation_search(xb, max_steps=0)
    assert r["steps"] == 0 and np.array_equal(r["R"], np.eye(32)) and r["group"] == 1
    with pytest.raises(ValueError):
        oracle.rotation_search(xb[:, :48])
    with pytest.raises(ValueError):
        oracle.rotation_search(xb, n_angle=0)


def test_search_lowers_the_worst_group_error():
    # The searched rotation, rounded to bf16, quantises the worst group it was fit to with
    # a smaller normalised error than the identity (the write-up's Figure 1 comparison).
    w = synth.make_config(2, rows=256, cols=1024)
    xb = synth.bf16_bits(w.x)
    r = oracle.rotation_search(xb, max_steps=128, threads=4)
    g = r["group"]
    blk = np.ascontiguousarray(xb[:, g * 32:(g + 1) * 32])
    eye = synth.bf16_bits(synth.rhat_tensor(np.eye(32)))
    e_id = oracle.group_error(blk, eye)[1]
    e_rs = oracle.group_error(blk, r["rhat_bits"])[1]
    assert e_rs < e_id

"""Reading R12, pinned: the oracle decides scales and codes on y rounded to fp32, and
deciding on the double y instead would accept the same outputs.

The rounding of y to fp32 moves a value by at most 2^-24 of itself.  Every boundary
band the acceptance rule excuses is far wider (1e-3 of a grid step for a code,
2.5e-4 relative for a scale), so the two oracles can only disagree on elements that
both flag as inside a band, and there each one's result is the other's neighbour.
The double-decision oracle is the oracle built with the one change that its
decisions skip the fp32 rounding (planted mistake 8 in the C file); everything else
is the same code.  On three workloads, each oracle's output must pass the parity
rule against the other: they accept the same set.
"""
import numpy as np
import pytest

import oracle
from tests import _parity
from workloads import synth

DOUBLE_DECISION = 8


def _cases():
    w1 = synth.make_config(1)                               # outlier toy, full size
    w3 = synth.make_config(3, rows=160, cols=2048)          # Student-t with massive outliers
    lam = synth.random_lambda(2048, seed=21).numpy()
    return [("outlier_toy", w1.x, w1.rhat, None), ("downproj_like", w3.x, w3.rhat, None),
            ("downproj_like_lambda", w3.x, w3.rhat, lam)]


@pytest.mark.parametrize("name,x,rhat,lam", _cases(), ids=lambda v: v if isinstance(v, str) else "")
def test_double_decision_accepts_the_same_outputs(name, x, rhat, lam):
    xb, rb = synth.bf16_bits(x), synth.bf16_bits(rhat)
    f32 = oracle.smooth_rotate_quantize(xb, rb, lam, want_y=True, flags=True, threads=4)
    with oracle.use_library(oracle.build_variant(DOUBLE_DECISION)):
        f64 = oracle.smooth_rotate_quantize(xb, rb, lam, want_y=True, flags=True, threads=4)
    # the double-decision results are accepted under the fp32-decision oracle's rule ...
    a = _parity.check_quant(xb, rb, lam, f64["codes"], f64["scales"], ref=f32)
    # ... and the fp32-decision results under the double-decision oracle's rule
    b = _parity.check_quant(xb, rb, lam, f32["codes"], f32["scales"], ref=f64)
    # where they differ at all, both oracles flag the element (or group) as inside a band
    diff = _parity.unpack(f32["codes"]) != _parity.unpack(f64["codes"])
    assert not (diff & (f32["eflags"] == 0)).any() and not (diff & (f64["eflags"] == 0)).any()
    sdiff = f32["scales"] != f64["scales"]
    assert not (sdiff & (f32["gflags"] == 0)).any() and not (sdiff & (f64["gflags"] == 0)).any()
    assert a["code_boundary_diffs"] == b["code_boundary_diffs"] == int(diff.sum())


def test_the_variant_really_decides_on_double():
    """Guard against a vacuous pin: the variant must decide on the double y.  With
    x = [1, 2^-20, 4, 0, ...] and a matrix whose column 1 holds 0.25 and 2^-20 in rows 0 and
    1 (column 0 holds 1 in row 2), y = [4, 0.25 + 2^-40, 0, ...] exactly in double.  The
    absmax 4 gives e = 0, so u = y.  In fp32, y_1 rounds onto the midpoint 0.25 and ties to
    code 0; in double it lies above the midpoint and takes code 1."""
    x = np.zeros((1, 32))
    x[0, :3] = [1.0, 2.0 ** -20, 4.0]
    r = np.zeros((32, 32))
    r[0, 1], r[1, 1], r[2, 0] = 0.25, 2.0 ** -20, 1.0
    xb = synth.bf16_bits(synth.to_bf16(x))
    rb = synth.bf16_bits(synth.to_bf16(r))
    f32 = oracle.smooth_rotate_quantize(xb, rb, None)
    with oracle.use_library(oracle.build_variant(DOUBLE_DECISION)):
        f64 = oracle.smooth_rotate_quantize(xb, rb, None)
    assert f32["scales"][0, 0] == f64["scales"][0, 0] == 127
    assert _parity.unpack(f32["codes"])[0, 1] == 0 and _parity.unpack(f64["codes"])[0, 1] == 1

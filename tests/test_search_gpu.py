"""GPU parity of the rotation search (DuQuant++ write-up, §3.2) with the oracle.

Every decision of the search is a comparison of values that both sides compute
with the same IEEE double operations in the same order, and every reduction is
a max.  So the worst group, the number of steps, the trace of (d, j, angle),
the L-inf history and every bit of R must be equal, and R's bf16 rounding too.
"""
import numpy as np
import pytest
import torch

import mxfp4_block_rotation_b200 as mxq
import oracle
from workloads import synth

pytestmark = pytest.mark.gpu


def _run(dev, xb, lam, K, n, workspace=None):
    x = synth.bf16_from_bits(xb).to(dev)
    lt = None if lam is None else torch.from_numpy(np.ascontiguousarray(lam, np.float32)).to(dev)
    out = mxq.rotation_search(x, lt, max_steps=K, n_angle=n, workspace=workspace)
    mxq.sync_check()
    out["rhat"] = out["rhat"].view(torch.int16)
    return {k: v.cpu().numpy() for k, v in out.items()}


def _same(g, o, K):
    assert int(g["group"]) == o["group"]
    assert int(g["steps"]) == o["steps"]
    n = o["steps"]
    assert np.array_equal(g["trace"][:n], o["trace"])
    assert np.array_equal(g["linf"][:n + 1], o["linf"])
    assert np.array_equal(g["R"], o["R"])
    assert np.array_equal(g["rhat"].view(np.uint16), o["rhat_bits"])


CASES = [
    # rows, cols, K, n_angle, lambda
    (1, 32, 4, 1, False),
    (3, 64, 16, 3, True),
    (257, 96, 32, 32, False),
    (1000, 1056, 64, 32, True),
    (1025, 256, 128, 32, False),    # one full row chunk and a one-row tail
    (2049, 512, 40, 128, True),     # the largest angle grid; two chunks and a tail
    (64, 4096, 0, 32, False),       # K = 0: only the worst group and its L-inf
]


@pytest.mark.parametrize("rows,cols,K,n,use_lam", CASES)
def test_search_matches_oracle(cuda_device, rows, cols, K, n, use_lam):
    w = synth.make_config(2, rows=rows, cols=cols)
    xb = synth.bf16_bits(w.x)
    lam = synth.random_lambda(cols, seed=rows + cols).numpy() if use_lam else None
    o = oracle.rotation_search(xb, lam=lam, max_steps=K, n_angle=n, threads=oracle.default_threads())
    g = _run(cuda_device, xb, lam, K, n)
    _same(g, o, K)


def test_search_stops_when_nothing_improves(cuda_device):
    x = np.ones((6, 64), np.float32)
    x[:, 32:] = 0.25
    xb = synth.bf16_bits(synth.to_bf16(x))
    o = oracle.rotation_search(xb, max_steps=10, n_angle=16)
    g = _run(cuda_device, xb, None, 10, 16)
    assert o["steps"] == 0
    _same(g, o, 10)
    assert np.array_equal(g["R"], np.eye(32))


def test_search_special_values(cuda_device):
    # NaN is skipped by every max; an infinite value makes the block's norm infinite, and
    # no rotation that moves it can bring the norm below infinity.
    w = synth.make_config(2, rows=300, cols=256)
    xb = synth.bf16_bits(w.x).copy()
    base = oracle.rotation_search(xb, max_steps=0)
    g0 = base["group"]
    nan_bits, inf_bits = np.uint16(0x7FC0), np.uint16(0x7F80)
    xb[5, g0 * 32 + 3] = nan_bits                     # NaN inside the worst group
    xb[7, ((g0 + 1) % 8) * 32 + 1] = nan_bits         # and elsewhere
    lam = synth.random_lambda(256, seed=9).numpy()
    lam[((g0 + 2) % 8) * 32 + 4] = 0.0                # x / 0 = inf (or NaN for x = 0)
    for lm in (None, lam):
        o = oracle.rotation_search(xb, lam=lm, max_steps=24, n_angle=8)
        _same(_run(cuda_device, xb, lm, 24, 8), o, 24)
    xb[9, g0 * 32 + 10] = inf_bits
    o = oracle.rotation_search(xb, max_steps=24, n_angle=8)
    assert o["steps"] == 0 and o["linf"][0] == np.inf
    _same(_run(cuda_device, xb, None, 24, 8), o, 24)


def test_search_is_deterministic_and_reuses_its_workspace(cuda_device):
    wa = synth.make_config(3, rows=512, cols=1024)
    wb = synth.make_config(2, rows=512, cols=1024)
    ws = torch.empty(mxq.lib().mxq_rotation_search_workspace_bytes(512, 1024, 32), dtype=torch.uint8,
                     device=cuda_device)
    a1 = _run(cuda_device, synth.bf16_bits(wa.x), None, 64, 32, ws)
    b = _run(cuda_device, synth.bf16_bits(wb.x), None, 64, 32, ws)
    a2 = _run(cuda_device, synth.bf16_bits(wa.x), None, 64, 32, ws)
    for k in a1:
        assert np.array_equal(a1[k], a2[k]), k
    _same(b, oracle.rotation_search(synth.bf16_bits(wb.x), max_steps=64, threads=oracle.default_threads()), 64)


@pytest.mark.parametrize("use_lam", [False, True])
def test_search_full_downproj(cuda_device, use_lam):
    # 8192 x 14336 down-projection activations, K = 128, 64 angles per pair: the whole run
    # against the oracle, not a sample.
    w = synth.make_config(3)
    xb = synth.bf16_bits(w.x)
    lam = synth.smoothing_scale(w.x).numpy() if use_lam else None
    o = oracle.rotation_search(xb, lam=lam, max_steps=128, n_angle=32, threads=oracle.default_threads())
    g = _run(cuda_device, xb, lam, 128, 32)
    _same(g, o, 128)
    assert o["steps"] > 0

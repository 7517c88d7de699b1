"""The seeded workload generators: deterministic, right shape, structure as stated."""
import numpy as np
import torch

from workloads import synth


def test_small_shapes_and_determinism():
    a = synth.make_config(1)
    b = synth.make_config(1)
    assert a.x.shape == (128, 4096) and a.x.dtype == torch.bfloat16
    assert torch.equal(a.x.view(torch.int16), b.x.view(torch.int16))
    assert torch.equal(a.rhat.view(torch.int16), b.rhat.view(torch.int16))
    assert a.lam is None


def test_config1_outliers_planted():
    w = synth.make_config(1)
    x = w.x.float()
    # token 3 scaled x1000, channels {7,1000,2049,3500} x50
    assert x[3].abs().mean() > 200 * x[10].abs().mean()
    col = x[:, [7, 1000, 2049, 3500]].abs().mean()
    assert col > 10 * x[:, [8, 9, 10]].abs().mean()


def test_overridden_shapes_keep_recipe():
    for cfg in (2, 3, 4, 5):
        w = synth.make_config(cfg, rows=64, cols=256)
        assert w.x.shape == (64, 256)
        assert torch.isfinite(w.x.float()).all()
        assert np.abs(w.rhat_f64.T @ w.rhat_f64 - np.eye(32)).max() < 1e-6
    w = synth.make_config(5, rows=64, cols=256)
    assert w.lam is not None and w.lam.dtype == torch.float32
    assert (w.lam >= 1e-2).all() and (w.lam <= 1e2).all()
    w3 = synth.make_config(3, rows=64, cols=256)
    assert w3.x.float().abs().max() >= 1e3          # massive outliers present


def test_hadamard_rhat_entries():
    r = synth.hadamard_rhat(2004)
    assert np.allclose(np.abs(r), 32 ** -0.5)
    rb = synth.rhat_tensor(r).float().abs()
    assert torch.all(rb == rb[0, 0])                 # one bf16 magnitude (0.1767578125)


def test_sample_rows_includes_edges():
    s = synth.sample_rows(1000, 20, seed=1, must=np.array([5, 999]))
    assert s[0] == 0 and s[-1] == 999 and 5 in s and len(s) >= 20

"""The seeded generators: shapes, dtypes, determinism, finiteness and the
value structure each workload is specified with."""
import torch

from fp4_block_scaled_04_b200 import workloads as w


def test_deterministic_and_finite():
    for fn, kw in [(w.activation, dict(rows=64, cols=128)), (w.weight, dict(rows=64, cols=128)),
                   (w.gradient, dict(tokens=128, cols=64)), (w.if4_blocks, dict(rows=32, cols=256)),
                   (w.small_matrix, {})]:
        a, b = fn(**kw), fn(**kw)
        assert torch.equal(a, b)
        assert torch.isfinite(a.float()).all()
    assert w.activation(rows=64, cols=128).dtype == torch.bfloat16
    assert w.weight(rows=64, cols=128).dtype == torch.float32


def test_activation_outlier_columns():
    x = w.activation(rows=512, cols=256, n_outlier_cols=8).float()
    col_scale = x.abs().mean(0)
    assert (col_scale > 20).sum().item() == 8


def test_weight_outlier_fraction():
    x = w.weight(rows=256, cols=512)
    n_big = (x.abs() > 0.02 * 6).sum().item()            # beyond 6 sigma: the x30 entries
    assert abs(n_big - round(1e-4 * x.numel())) <= 3


def test_if4_block_mix():
    x = w.if4_blocks(rows=256, cols=1024).float().reshape(-1, 16)
    amax = x.abs().max(1).values
    second = x.abs().sort(1).values[:, -2]
    assert ((amax / second.clamp_min(1e-6)) > 1.5).float().mean() > 0.7   # one x10 outlier per block
    uniform = (x.abs().sort(1).values[:, :-1].max(1).values <= 1.0)
    assert 0.4 < uniform.float().mean() < 0.75                            # about half U(-1,1)


def test_gradient_heavy_tails():
    g = w.gradient(tokens=1024, cols=256).float() / 1e-3
    kurt = ((g - g.mean()) ** 4).mean() / g.var() ** 2
    assert kurt > 6                                                       # Student-t(3)

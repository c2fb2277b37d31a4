"""The seeded synthetic inputs follow the stated recipe: deterministic,
the workloads' shapes, bf16 rounding, cfg 3's outlier columns and cfg 4's
heavy tails.  (Input generation only; none of the method's arithmetic.)"""
import ml_dtypes
import numpy as np

from structured_sparse_fp8_b200 import workloads as WL


def test_deterministic_and_shaped():
    for cfg, wl in WL.WORKLOADS.items():
        a = WL.weight_bits(cfg, n=64, k=wl.k)
        assert a.dtype == np.uint16 and a.shape == (64, wl.k)
        assert np.array_equal(a, WL.weight_bits(cfg, n=64, k=wl.k))
        assert not np.array_equal(a, WL.weight_bits(cfg, n=64, k=wl.k, layer=1))
        x = WL.activation_bits(cfg, wl.ms[0])
        assert x.shape == (wl.ms[0], wl.k) and np.array_equal(x, WL.activation_bits(cfg, wl.ms[0]))


def test_values_are_bf16_roundings_of_the_draws():
    x = np.random.default_rng([WL.SEED, 2, 1, 8]).normal(0.0, 1.0, size=(8, 4096))
    assert np.array_equal(WL.activation_bits(2, 8), x.astype(ml_dtypes.bfloat16).view(np.uint16))


def test_prefill_outlier_columns():
    x = WL.activation_bits(3, 512).view(ml_dtypes.bfloat16).astype(np.float64)
    sd = x.std(axis=0)
    big = sd > 5.0
    assert big.sum() == round(0.01 * 4096) == 41
    assert 15.0 < sd[big].mean() < 25.0 and 0.8 < sd[~big].mean() < 1.2


def test_downproj_weights_are_heavy_tailed():
    w = WL.weight_bits(4, n=256).view(ml_dtypes.bfloat16).astype(np.float64)
    z = w / 0.02
    # Student-t with 3 degrees of freedom: far more mass beyond 5 than a normal
    assert (np.abs(z) > 5).mean() > 5e-3
    n = WL.weight_bits(2, n=256).view(ml_dtypes.bfloat16).astype(np.float64) / 0.02
    assert (np.abs(n) > 5).mean() < 1e-5

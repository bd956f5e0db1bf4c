"""Pins of the oracle's block index (Methodology section 4: population centroid,
coordinate-wise variance, maximum key norm) against a hand-derived worked
example and against numpy in double precision."""
import json
import os

import numpy as np
import pytest

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _golden():
    with open(os.path.join(GOLDEN, "eq5_worked_example.json")) as f:
        return json.load(f)


def test_worked_example_metadata():
    g = _golden()
    mu, var, mx = oracle.block_meta(np.array(g["keys"], np.float32))
    assert mu.tolist() == g["mu"]
    assert var.tolist() == g["var"]            # population variance: a 1/(n-1) estimator gives 2
    assert mx == pytest.approx(np.sqrt(g["maxnorm_squared"]), rel=1e-7)


@pytest.mark.parametrize("rows,d,scale", [(16, 64, 1.0), (64, 128, 3.0), (7, 8, 1e-3), (128, 128, 50.0)])
def test_metadata_matches_double_precision(rows, d, scale):
    rng = np.random.default_rng(rows * d)
    k = (rng.standard_normal((rows, d)) * scale + rng.standard_normal(d)).astype(np.float32)
    mu, var, mx = oracle.block_meta(k)
    k64 = k.astype(np.float64)
    mu_ref = k64.mean(axis=0)
    var_ref = k64.var(axis=0)                 # ddof=0: population
    mx_ref = np.sqrt((k64 ** 2).sum(axis=1)).max()
    # fp32 sequential sums: error bounded by ~rows ulps of the running magnitude
    tol_mu = rows * np.finfo(np.float32).eps * np.abs(k64).max()
    assert np.all(np.abs(mu - mu_ref) <= tol_mu)
    assert np.all(np.abs(var - var_ref) <= 4 * rows * np.finfo(np.float32).eps * (var_ref + tol_mu * np.abs(k64).max()))
    assert abs(mx - mx_ref) <= 2 * d * np.finfo(np.float32).eps * mx_ref


def test_bf16_storage_is_widened_exactly():
    import torch
    x = torch.randn(32, 64).to(torch.bfloat16)
    assert np.array_equal(oracle.to_f32(x), x.float().numpy())
    mu, var, mx = oracle.block_meta(x)
    mu2, var2, mx2 = oracle.block_meta(x.float().numpy())
    assert np.array_equal(mu, mu2) and np.array_equal(var, var2) and mx == mx2


def test_slice_meta_full_blocks_only():
    import torch
    k = torch.randn(1, 1, 100, 8)
    mu, var, mx = oracle.meta(k, n=100, bs=16)
    assert mu.shape == (1, 1, 6, 8)             # 100 // 16 full blocks; the tail block has none
    m5, v5, x5 = oracle.block_meta(k[0, 0, 80:96].numpy())
    assert np.array_equal(mu[0, 0, 5], m5) and mx[0, 0, 5] == x5

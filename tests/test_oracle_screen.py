"""Pins of the oracle's threshold predictor (Eq. 1), dual screening score
(Eq. 5) and admission rule (Methodology section 4) against a hand-derived
worked example, brute force, library routines and printed numbers."""
import json
import math
import os

import numpy as np
import pytest

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _load(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


def test_eq5_worked_example():
    g = _load("eq5_worked_example.json")
    mu = np.array(g["mu"], np.float32)
    var = np.array(g["var"], np.float32)
    mx = np.float32(math.sqrt(g["maxnorm_squared"]))
    for c in g["cases"]:
        s = oracle.block_score(np.array(c["q"], np.float32), mu, var, mx, c["z"])
        assert s == pytest.approx(c["value"], rel=2e-7), c


def test_eq5_dual_score_is_not_a_bound_but_its_ceiling_is():
    """The worked example's moment term (3+sqrt 2)/2 lies below the block's true
    max logit 2.5; the Cauchy-Schwarz ceiling sqrt(28)/2 lies above it."""
    g = _load("eq5_worked_example.json")
    c = g["cases"][0]
    assert c["value"] < c["true_max_logit"] < math.sqrt(28) / 2


def _rand_block(rng, rows, d, offset=0.0):
    return (rng.standard_normal((rows, d)) + offset * rng.standard_normal(d)).astype(np.float32)


@pytest.mark.parametrize("seed", range(6))
def test_cauchy_schwarz_term_bounds_true_max_logit(seed):
    """Brute force: with z huge the dual score equals the Cauchy-Schwarz term,
    which is at least the true max scaled logit of the block; with any z the
    score is at most that term."""
    rng = np.random.default_rng(seed)
    d, rows = (64, 16) if seed % 2 else (128, 64)
    for _ in range(20):
        k = _rand_block(rng, rows, d, offset=rng.uniform(0, 2))
        q = rng.standard_normal(d).astype(np.float32) * rng.uniform(0.1, 3)
        mu, var, mx = oracle.block_meta(k)
        true_max = float((k.astype(np.float64) @ q.astype(np.float64)).max() / math.sqrt(d))
        ceiling = oracle.block_score(q, mu, var, mx, 1e30)
        slack = 4 * np.finfo(np.float32).eps * (np.linalg.norm(q) * mx / math.sqrt(d))
        assert ceiling + slack >= true_max
        ceiling_ref = float(np.linalg.norm(q.astype(np.float64)) * np.sqrt((k.astype(np.float64) ** 2).sum(1)).max() / math.sqrt(d))
        assert ceiling == pytest.approx(ceiling_ref, rel=1e-5)
        for z in (0.0, 1.0, 1.5, 2.0):
            assert oracle.block_score(q, mu, var, mx, z) <= ceiling


def test_score_moment_term_against_numpy():
    """With z = 0 and a huge max norm the score is <q, mu>/sqrt(d); with z = 1 it
    adds sqrt(sum q_i^2 var_i)/sqrt(d) (numpy, double)."""
    rng = np.random.default_rng(11)
    d = 128
    q = rng.standard_normal(d).astype(np.float32)
    mu = rng.standard_normal(d).astype(np.float32)
    var = rng.uniform(0.1, 2, d).astype(np.float32)
    q64, mu64, var64 = (x.astype(np.float64) for x in (q, mu, var))
    s0 = oracle.block_score(q, mu, var, np.float32(1e30), 0.0)
    assert s0 == pytest.approx(q64 @ mu64 / math.sqrt(d), rel=1e-5, abs=1e-5)
    s1 = oracle.block_score(q, mu, var, np.float32(1e30), 1.0)
    assert s1 == pytest.approx((q64 @ mu64 + math.sqrt((q64 ** 2 * var64).sum())) / math.sqrt(d),
                               rel=1e-5, abs=1e-5)


def _screen_setup(seed=0, nb=40, bs=16, d=64):
    rng = np.random.default_rng(seed)
    k = rng.standard_normal((nb * bs, d)).astype(np.float32)
    k += np.repeat(rng.standard_normal((nb, d)).astype(np.float32), bs, axis=0)
    q = rng.standard_normal(d).astype(np.float32)
    mu, var, mx = oracle.slice_meta(k, d, bs, nb)
    return q, mu, var, mx


def test_screen_ties_are_admitted_and_order_ascending():
    q, mu, var, mx = _screen_setup()
    nb = mu.shape[0]
    _, scores = oracle.screen_head(q, mu, var, mx, nb, 1, 1.0, float("-inf"))
    j = int(np.argsort(scores)[len(scores) // 2])
    tau = float(scores[j])                  # a block's own score: exact tie
    lst, _ = oracle.screen_head(q, mu, var, mx, nb, 1, 1.0, tau)
    assert j in lst.tolist()
    assert np.all(np.diff(lst) > 0)
    expect = sorted([i for i in range(nb - 1) if scores[i] >= np.float32(tau)] + [nb - 1])
    assert lst.tolist() == expect


def test_forced_blocks_and_extreme_thresholds():
    q, mu, var, mx = _screen_setup()
    nb = mu.shape[0]
    lst, _ = oracle.screen_head(q, mu, var, mx, nb, 1, 1.0, float("inf"))
    assert lst.tolist() == [nb - 1]          # only the block holding the current token
    lst, _ = oracle.screen_head(q, mu, var, mx, nb, 3, 1.0, float("inf"))
    assert lst.tolist() == [nb - 3, nb - 2, nb - 1]
    lst, _ = oracle.screen_head(q, mu, var, mx, nb, 1, 1.0, float("-inf"))
    assert lst.tolist() == list(range(nb))
    lst, _ = oracle.screen_head(q, mu[:0], var[:0], mx[:0], 2, 5, 1.0, float("inf"))
    assert lst.tolist() == [0, 1]            # n_local beyond nb: everything is forced


def test_density_grows_with_offset_a():
    """Table 17's offset sweep: density rises with a (36.3% at a=+0.4, 32.0% at 0,
    24.4% at -0.8, ...), which fixes the adjusted threshold tau~ = tau - a."""
    q, mu, var, mx = _screen_setup(seed=3, nb=200)
    nb = mu.shape[0]
    _, scores = oracle.screen_head(q, mu, var, mx, nb, 1, 1.0, float("-inf"))
    tau = float(np.median(scores))
    counts = [len(oracle.screen_head(q, mu, var, mx, nb, 1, 1.0, tau, a)[0])
              for a in (-2.0, -0.8, 0.0, 0.4, 2.0)]
    assert counts == sorted(counts) and counts[0] < counts[-1]


def test_predictor_matches_double_matmul_and_init():
    """Eq. 1 against numpy in double (a transposed W or a dropped bias fails);
    the zero-initialised projection with bias -8 gives tau = -8 exactly."""
    rng = np.random.default_rng(5)
    B, H, d = 3, 8, 64
    q = rng.standard_normal((B, H, d)).astype(np.float32)
    W = (rng.standard_normal((H * d, H)) / math.sqrt(d)).astype(np.float32)
    bias = rng.standard_normal(H).astype(np.float32)
    tau = oracle.predict_tau(q, W, bias)
    ref = q.reshape(B, H * d).astype(np.float64) @ W.astype(np.float64) + bias
    assert np.allclose(tau, ref, rtol=1e-5, atol=1e-5)
    tau0 = oracle.predict_tau(q, np.zeros_like(W), np.full(H, -8.0, np.float32))
    assert np.all(tau0 == -8.0)


def test_table13_predictor_parameter_count():
    g = _load("table13_predictor_params.json")
    H, d = g["heads"], g["head_dim"]
    W = np.zeros((H * d, H), np.float32)
    bias = np.zeros(H, np.float32)
    q = np.zeros((1, H, d), np.float32)
    oracle.predict_tau(q, W, bias)          # accepts exactly this orientation
    assert g["layers"] * (W.size + bias.size) == g["params"]
    with pytest.raises(AssertionError):
        oracle.predict_tau(q, W.T.copy(), bias)

"""Pins of the oracle's sub-block envelope screen (a labelled reading of the
pages' undefined "sub-block envelope", Table 16 caption and Table 12 header):
r = 1 is the flat Eq. 5 screen; with z -> infinity only the Cauchy-Schwarz term
is left and the envelope over sub-blocks of b/r tokens equals the flat screen
over blocks of b tokens bit for bit (max over sub-blocks of the largest key norm
is the block's largest key norm); a block of two constant halves has the
closed-form envelope max(<q, v0>, <q, v1>)/sqrt(d) where the flat score is
diluted to <q, (v0+v1)/2> + z sqrt(sum q_i^2 ((v0_i - v1_i)/2)^2); a score
equal to the threshold is admitted."""
import math

import numpy as np
import pytest

import oracle


def _cache(seed, n, d, offset=0.7):
    rng = np.random.default_rng(seed)
    k = rng.standard_normal((n, d)).astype(np.float32)
    k += offset * np.repeat(rng.standard_normal((n // 8 + 1, d)), 8, 0)[:n].astype(np.float32)
    q = rng.standard_normal(d).astype(np.float32)
    return k, q


def _meta(k, n, bs):
    mu, var, mx = oracle.meta(k[None, None], n, bs)
    return mu[0, 0], var[0, 0], mx[0, 0]


@pytest.mark.parametrize("n,bs,d", [(32 * 40 + 5, 32, 64), (64 * 20 + 1, 64, 128)])
def test_one_sub_block_is_the_flat_screen(n, bs, d):
    k, q = _cache(1, n, d)
    nb = (n + bs - 1) // bs
    mu, var, mx = _meta(k, n, bs)
    for tau in (-0.5, 0.2, 0.9):
        lf, sf = oracle.screen_head(q, mu, var, mx, nb, 1, 1.0, tau)
        le, se = oracle.screen_head_env(q, mu, var, mx, nb, 1, 1, 1.0, tau)
        assert np.array_equal(lf, le)
        assert np.array_equal(sf.view(np.int32), se.view(np.int32))


@pytest.mark.parametrize("bs,r,d", [(64, 4, 128), (64, 2, 64), (32, 2, 128), (128, 8, 64)])
def test_without_the_moment_term_the_envelope_is_the_block_norm_bound(bs, r, d):
    n = bs * 30 + 3
    k, q = _cache(2 + r, n, d)
    nb = (n + bs - 1) // bs
    mu_b, var_b, mx_b = _meta(k, n, bs)
    mu_s, var_s, mx_s = _meta(k, n, bs // r)
    for n_local in (1, 2):
        flat_l, flat_s = oracle.screen_head(q, mu_b, var_b, mx_b, nb, n_local, 1e30, 0.3)
        env_l, env_s = oracle.screen_head_env(q, mu_s, var_s, mx_s, nb, r, n_local, 1e30, 0.3)
        assert np.array_equal(flat_l, env_l)
        assert np.array_equal(flat_s.view(np.int32), env_s.view(np.int32))


def test_two_constant_halves_closed_form():
    """Keys of sub-block 0 all v0 and of sub-block 1 all v1 (values on a 1/8
    grid, so every mean and variance is exact): the envelope is the larger
    half's dot product, the flat score is diluted towards the mean."""
    d, bs, r = 64, 32, 2
    rng = np.random.default_rng(5)
    q = rng.standard_normal(d).astype(np.float32)
    nblk = 6
    v = rng.integers(-12, 13, size=(nblk, 2, d)).astype(np.float32) / 8.0
    v[0, 1] = -v[0, 0]                                          # opposite halves: mean 0
    v[1, 0] = np.sign(q) * 1.5                                  # one half aligned with q
    n = nblk * bs + 1                                           # + the current token's block
    k = np.zeros((n, d), np.float32)
    for j in range(nblk):
        k[j * bs:j * bs + bs // 2] = v[j, 0]
        k[j * bs + bs // 2:(j + 1) * bs] = v[j, 1]
    k[nblk * bs:] = rng.standard_normal((1, d)).astype(np.float32)
    nb = nblk + 1
    z = 1.0
    mu_s, var_s, mx_s = _meta(k, n, bs // r)
    mu_b, var_b, mx_b = _meta(k, n, bs)
    assert np.all(var_s[:nblk * r] == 0.0)
    _, env = oracle.screen_head_env(q, mu_s, var_s, mx_s, nb, r, 1, z, -np.inf)
    _, flat = oracle.screen_head(q, mu_b, var_b, mx_b, nb, 1, z, -np.inf)
    qd = q.astype(np.float64)
    s = 1.0 / math.sqrt(d)
    for j in range(nblk):
        v0, v1 = v[j, 0].astype(np.float64), v[j, 1].astype(np.float64)
        qn = np.linalg.norm(qd)
        c0, c1 = qn * np.linalg.norm(v0), qn * np.linalg.norm(v1)
        want_env = max(min(qd @ v0, c0), min(qd @ v1, c1)) * s
        assert env[j] == pytest.approx(want_env, rel=2e-6, abs=2e-6), j
        mean, half = (v0 + v1) / 2, (v0 - v1) / 2
        a_term = qd @ mean + z * math.sqrt(np.sum(qd ** 2 * half ** 2))
        want_flat = min(a_term, qn * max(np.linalg.norm(v0), np.linalg.norm(v1))) * s
        assert flat[j] == pytest.approx(want_flat, rel=2e-6, abs=2e-6), j
    # variance dilution: opposite halves average to a zero mean, the envelope keeps the better half
    assert env[0] > flat[0]


def test_a_score_equal_to_the_threshold_is_admitted():
    d, bs, r = 128, 64, 4
    n = bs * 12 + 9
    k, q = _cache(9, n, d)
    nb = (n + bs - 1) // bs
    mu_s, var_s, mx_s = _meta(k, n, bs // r)
    _, sc = oracle.screen_head_env(q, mu_s, var_s, mx_s, nb, r, 1, 1.0, -np.inf)
    j = int(np.argsort(sc)[len(sc) // 2])
    tau = float(sc[j])
    lst, _ = oracle.screen_head_env(q, mu_s, var_s, mx_s, nb, r, 1, 1.0, tau)
    assert j in lst
    assert all(sc[i] >= sc[j] for i in lst if i < nb - 1)
    assert all(i in lst for i in range(nb - 1) if sc[i] >= sc[j])

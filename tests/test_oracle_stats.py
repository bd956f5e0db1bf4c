"""Pins of the oracle's block statistics and Table 16 screen diagnostics: the
block max logit and above-threshold counts against float64 brute force, the
block log-sum-exps against the oracle's own attention (the dense gated output is
the mass-weighted mix of single-block outputs), the Cauchy-Schwarz ceiling of
Eq. 5 above every block max, and the diagnostics' limiting cases."""
import math

import numpy as np
import pytest

import oracle


def _slice(seed, n, d, bs, offset=0.0):
    rng = np.random.default_rng(seed)
    cap = ((n + bs - 1) // bs) * bs
    k = np.zeros((cap, d), np.float32)
    k[:n] = rng.standard_normal((n, d)) + offset * np.repeat(rng.standard_normal((cap // bs, d)), bs, 0)[:n]
    v = np.zeros((cap, d), np.float32)
    v[:n] = rng.standard_normal((n, d))
    q = rng.standard_normal(d).astype(np.float32)
    return k, v, q


@pytest.mark.parametrize("n,bs,d", [(500, 16, 64), (1000, 32, 128), (777, 64, 64)])
def test_block_max_and_counts_match_float64(n, bs, d):
    k, _, q = _slice(n, n, d, bs, offset=0.7)
    S = (k[:n].astype(np.float64) @ q.astype(np.float64)) / math.sqrt(d)
    srt = np.sort(S)
    i = int(0.8 * n)
    i = max(range(i - 20, i + 20), key=lambda j: srt[j + 1] - srt[j])
    tau_s = float(np.float32(0.5 * (srt[i] + srt[i + 1])))       # in a gap: no rounding-sensitive ties
    bmax, above, _ = oracle.block_stats(k, bs, n, q, tau_s, tau_s, 5.0)
    nb = (n + bs - 1) // bs
    for j in range(nb):
        blk = S[j * bs:min(n, (j + 1) * bs)]
        assert bmax[j] == pytest.approx(blk.max(), rel=1e-6, abs=1e-6)
        assert above[j] == int((blk >= tau_s).sum())


@pytest.mark.parametrize("gate", [oracle.GATE_SIGMOID, oracle.GATE_HARD])
def test_block_lse_mixes_single_block_outputs_into_the_dense_output(gate):
    """sum_j exp(lse_j - LSE) o_j = o_dense, with o_j the oracle's attention over
    block j alone: a wrong gate, normaliser or current-token rule in either
    function breaks it."""
    n, bs, d = 300, 32, 64
    k, v, q = _slice(7, n, d, bs)
    tau = 0.4
    nb = (n + bs - 1) // bs
    _, _, blse = oracle.block_stats(k, bs, n, q, tau, tau, 5.0, gate)
    lse = np.logaddexp.reduce(blse)
    mix = np.zeros(d)
    for j in range(nb):
        if blse[j] == -np.inf:
            continue
        o_j = oracle.attend_head(k, v, bs, n, q, np.array([j], np.int32), tau, 5.0, gate)
        mix += math.exp(blse[j] - lse) * o_j
    dense = oracle.attend_head(k, v, bs, n, q, np.arange(nb, dtype=np.int32), tau, 5.0, gate)
    assert np.allclose(mix, dense, rtol=1e-5, atol=1e-6)


def test_cauchy_schwarz_ceiling_bounds_every_block_max():
    n, bs, d = 640, 32, 128
    k, _, q = _slice(3, n, d, bs, offset=1.0)
    nb = n // bs
    mu, var, mx = oracle.meta(k[None, None], n, bs)
    _, sc = oracle.screen_head(q, mu[0, 0], var[0, 0], mx[0, 0], nb, 1, 1e30, float("-inf"))
    bmax, _, _ = oracle.block_stats(k, bs, n, q, 0.0, 0.0, 5.0)
    assert np.all(sc >= bmax[:nb - 1] - 4e-6 * np.abs(bmax[:nb - 1]) - 1e-6)


def test_diagnostics_limiting_cases():
    n, bs, d = 400, 16, 64
    k, _, q = _slice(11, n, d, bs)
    nb, ns = n // bs, n // bs - 1
    tau_s = 0.8
    bmax, above, blse = oracle.block_stats(k, bs, n, q, tau_s, tau_s, 5.0)
    everything = oracle.screen_diagnostics(bmax, above, blse, np.arange(nb), ns, tau_s)
    assert everything["false_negative"] == 0.0 and everything["missed_mass"] == 0.0
    assert everything["token_recall"] == 1.0
    forced_only = oracle.screen_diagnostics(bmax, above, blse, np.array([nb - 1]), ns, tau_s)
    assert forced_only["false_positive"] == 0.0
    assert forced_only["token_recall"] == 0.0 and forced_only["false_negative"] == 1.0
    forced_mass = math.exp(blse[nb - 1] - np.logaddexp.reduce(blse))
    assert forced_only["missed_mass"] == pytest.approx(1.0 - forced_mass, rel=1e-12)
    exact = oracle.screen_diagnostics(bmax, above, blse, np.nonzero(bmax >= tau_s)[0], ns, tau_s)
    assert exact["false_negative"] == 0.0 and exact["false_positive"] == 0.0

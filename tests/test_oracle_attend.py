"""Pins of the oracle's gated attention (Eq. 2-3 over the admitted blocks):
tau = -inf reduces to textbook softmax attention (checked against torch's
scaled_dot_product_attention in float64); tau = +inf gives the closed form of
the uniform floor; a very large beta gives the hard step gate; the current
token is exempt from the gate; GQA union is the plain union of head sets."""
import math

import numpy as np
import pytest
import torch

import oracle


def _kv(rng, n, d, bs, cap=None, dtype=np.float32):
    cap = cap or ((n + bs - 1) // bs) * bs
    k = np.zeros((cap, d), np.float32)
    v = np.zeros((cap, d), np.float32)
    k[:n] = rng.standard_normal((n, d))
    v[:n] = rng.standard_normal((n, d))
    return k, v


@pytest.mark.parametrize("n,bs,d,scale", [(100, 16, 64, 1.0), (256, 32, 128, 1.0), (37, 16, 64, 40.0)])
def test_tau_minus_inf_is_softmax_attention(n, bs, d, scale):
    rng = np.random.default_rng(n)
    k, v = _kv(rng, n, d, bs)
    q = (rng.standard_normal(d) * scale).astype(np.float32)
    nb = (n + bs - 1) // bs
    out = oracle.attend_head(k, v, bs, n, q, np.arange(nb, dtype=np.int32), float("-inf"), 5.0)
    ref = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(q).double()[None, None, None, :],
        torch.from_numpy(k[:n]).double()[None, None], torch.from_numpy(v[:n]).double()[None, None])
    assert np.allclose(out, ref[0, 0, 0].numpy(), rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("n,bs", [(100, 16), (96, 16), (1, 16), (33, 32)])
def test_tau_plus_inf_uniform_floor_closed_form(n, bs):
    """Only the forced block survives; every other key's logit is S * 0 = 0, so it
    weighs exp(0) = 1, and the current token keeps exp(S_t):
    o = (sum_{s != t} v_s + exp(S_t) v_t) / ((n_f - 1) + exp(S_t))."""
    d = 64
    rng = np.random.default_rng(n + bs)
    k, v = _kv(rng, n, d, bs)
    q = rng.standard_normal(d).astype(np.float32)
    nb = (n + bs - 1) // bs
    out = oracle.attend_head(k, v, bs, n, q, np.array([nb - 1], np.int32), float("inf"), 5.0)
    lo, t = (nb - 1) * bs, n - 1
    St = float(q.astype(np.float64) @ k[t].astype(np.float64)) / math.sqrt(d)
    others = v[lo:t].astype(np.float64).sum(axis=0)
    ref = (others + math.exp(St) * v[t].astype(np.float64)) / ((t - lo) + math.exp(St))
    assert np.allclose(out, ref, rtol=1e-12, atol=1e-12)


def test_large_beta_is_hard_step_gate():
    """beta -> inf: sigma(beta (S - tau)) -> 1 above tau and 0 below, so logits are S
    above tau and 0 below (the current token keeps S_t)."""
    n, bs, d = 200, 16, 64
    rng = np.random.default_rng(1)
    k, v = _kv(rng, n, d, bs)
    q = rng.standard_normal(d).astype(np.float32)
    S = (k[:n].astype(np.float64) @ q.astype(np.float64)) / math.sqrt(d)
    tau = float(np.quantile(S, 0.7)) + 1e-3
    nb = (n + bs - 1) // bs
    out = oracle.attend_head(k, v, bs, n, q, np.arange(nb, dtype=np.int32), tau, 1e9)
    g = np.where(S > tau, S, 0.0)
    g[n - 1] = S[n - 1]
    w = np.exp(g - g.max())
    ref = (w[:, None] * v[:n].astype(np.float64)).sum(0) / w.sum()
    assert np.allclose(out, ref, rtol=1e-10, atol=1e-12)


def test_gate_value_at_threshold_is_half():
    """A key whose scaled logit equals tau gets sigma(0) = 1/2 of its logit; a
    single-key, two-token case has the closed form of a 2-way softmax."""
    d, bs = 4, 16
    k = np.zeros((16, d), np.float32)
    v = np.zeros((16, d), np.float32)
    k[0] = [2, 0, 0, 0]
    k[1] = [0, 0, 0, 0]            # current token t = 1, S_t = 0
    v[0] = [1, 0, 0, 0]
    v[1] = [0, 1, 0, 0]
    q = np.array([1, 0, 0, 0], np.float32)
    S0 = 2 / 2.0                   # <q,k0>/sqrt(4) = 1
    out = oracle.attend_head(k, v, bs, 2, q, np.array([0], np.int32), S0, 5.0)
    g0 = S0 * 0.5
    w0, w1 = math.exp(g0), 1.0
    assert np.allclose(out, [w0 / (w0 + w1), w1 / (w0 + w1), 0, 0], rtol=1e-14)


def test_current_token_is_exempt_from_gate():
    """With tau = +inf every logit except the current token's is pulled to 0."""
    d, bs = 4, 16
    k = np.zeros((16, d), np.float32)
    v = np.eye(16, d, dtype=np.float32)
    k[:3] = [[4, 0, 0, 0], [4, 0, 0, 0], [4, 0, 0, 0]]
    q = np.array([1, 0, 0, 0], np.float32)
    out = oracle.attend_head(k, v, bs, 3, q, np.array([0], np.int32), float("inf"), 5.0)
    e = math.exp(2.0)              # S_t = 4/2
    assert np.allclose(out, [1 / (2 + e), 1 / (2 + e), e / (2 + e), 0], rtol=1e-14)


def test_full_decode_gqa_union_is_or_of_heads():
    from learned_block_sparse_b200 import synth
    w = synth.Workload("t", "bf16", 2, 8, 2, 64, 1000, 16, z=1.0, tau_mode="const",
                       densities=(0.4,), seed=77, offset_std=math.sqrt(0.5))
    q = synth.make_q(w)
    K, V = synth.make_kv(w, q)
    tau = np.zeros((w.B, w.Hq), np.float32)
    res = oracle.decode(q, K, V, w.n, w.bs, tau, z=w.z)
    for (b, kvh), (idx, mask) in res["union"].items():
        sets = [set(res["lists"][(b, kvh * w.G + g)].tolist()) for g in range(w.G)]
        assert set(idx.tolist()) == set().union(*sets)
        for i, m in zip(idx.tolist(), mask.tolist()):
            assert m == sum(1 << g for g in range(w.G) if i in sets[g])
    # dense decode with tau=-inf equals softmax attention per head
    resd = oracle.decode(q, K, V, w.n, w.bs, np.full((w.B, w.Hq), -np.inf, np.float32),
                         z=w.z, dense=True, heads=[(1, 5)])
    qf = q.float().double()[1, 5]
    kk = K[1, 5 // w.G, :w.n].double()
    vv = V[1, 5 // w.G, :w.n].double()
    ref = torch.softmax(kk @ qf / math.sqrt(w.d), 0) @ vv
    assert np.allclose(resd["out"][(1, 5)], ref.numpy(), rtol=1e-12, atol=1e-12)


# ------------------------------------------------- strict mode (hard masking)
def test_hard_gate_minus_inf_is_softmax_attention():
    """Strict mode with tau = -inf removes nothing: textbook softmax attention."""
    n, bs, d = 150, 16, 64
    rng = np.random.default_rng(11)
    k, v = _kv(rng, n, d, bs)
    q = rng.standard_normal(d).astype(np.float32)
    nb = (n + bs - 1) // bs
    out = oracle.attend_head(k, v, bs, n, q, np.arange(nb, dtype=np.int32), float("-inf"), 5.0,
                             gate=oracle.GATE_HARD)
    ref = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(q).double()[None, None, None, :],
        torch.from_numpy(k[:n]).double()[None, None], torch.from_numpy(v[:n]).double()[None, None])
    assert np.allclose(out, ref[0, 0, 0].numpy(), rtol=1e-12, atol=1e-12)


def test_hard_gate_plus_inf_keeps_only_the_current_token():
    """Every key but the current one is removed: the output is v_t exactly
    (where the multiplicative gate leaves the uniform floor instead)."""
    n, bs, d = 77, 16, 64
    rng = np.random.default_rng(12)
    k, v = _kv(rng, n, d, bs)
    q = rng.standard_normal(d).astype(np.float32)
    nb = (n + bs - 1) // bs
    out = oracle.attend_head(k, v, bs, n, q, np.arange(nb, dtype=np.int32), float("inf"), 5.0,
                             gate=oracle.GATE_HARD)
    assert np.array_equal(out, v[n - 1].astype(np.float64))


@pytest.mark.parametrize("quantile", [0.3, 0.8, 0.97])
def test_hard_gate_equals_softmax_over_the_kept_keys(quantile):
    """Strict mode over a cache equals the plain softmax (tau = -inf) of the oracle
    over a second cache holding only the keys with S >= tau and the current token,
    in order: removing a key and masking it to -inf must agree. The kept set is
    chosen by numpy in float64, independently of the oracle's comparison."""
    n, bs, d = 300, 16, 64
    rng = np.random.default_rng(int(quantile * 100))
    k, v = _kv(rng, n, d, bs)
    q = rng.standard_normal(d).astype(np.float32)
    S = (k[:n].astype(np.float64) @ q.astype(np.float64)) / math.sqrt(d)
    tau = float(np.quantile(S, quantile)) + 1e-6
    nb = (n + bs - 1) // bs
    out = oracle.attend_head(k, v, bs, n, q, np.arange(nb, dtype=np.int32), tau, 5.0, gate=oracle.GATE_HARD)
    keep = np.nonzero(S >= tau)[0].tolist()
    if n - 1 not in keep:
        keep.append(n - 1)
    m = len(keep)
    k2, v2 = _kv(rng, m, d, bs)
    k2[:m], v2[:m] = k[keep], v[keep]
    nb2 = (m + bs - 1) // bs
    ref = oracle.attend_head(k2, v2, bs, m, q, np.arange(nb2, dtype=np.int32), float("-inf"), 5.0)
    assert np.allclose(out, ref, rtol=1e-12, atol=1e-13)


def test_hard_gate_keeps_a_key_exactly_at_the_threshold():
    """S == tau is kept (the comparison is >=, as the screen's admission rule)."""
    d, bs = 4, 16
    k = np.zeros((16, d), np.float32)
    v = np.zeros((16, d), np.float32)
    k[0] = [2, 0, 0, 0]            # S_0 = 1
    k[1] = [1.0, 0, 0, 0]          # S_1 = 0.5 < tau: removed
    k[2] = [0, 0, 0, 0]            # current token, S_t = 0
    v[0], v[1], v[2] = [1, 0, 0, 0], [0, 1, 0, 0], [0, 0, 1, 0]
    q = np.array([1, 0, 0, 0], np.float32)
    out = oracle.attend_head(k, v, bs, 3, q, np.array([0], np.int32), 1.0, 5.0, gate=oracle.GATE_HARD)
    e = math.e
    assert np.allclose(out, [e / (e + 1), 0, 1 / (e + 1), 0], rtol=1e-14)

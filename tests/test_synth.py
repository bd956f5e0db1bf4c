"""Seeded input generator: Philox4x32-10 known answers, normal statistics,
slice regenerability, bf16 rounding and workload structure."""
import json
import math
import os

import numpy as np
import pytest
import torch

from learned_block_sparse_b200 import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def test_philox_known_answers():
    with open(os.path.join(GOLDEN, "philox4x32_10_kat.json")) as f:
        kat = json.load(f)
    for c in kat["cases"]:
        out = synth.philox4x32_10([int(x, 16) for x in c["ctr"]], [int(x, 16) for x in c["key"]])
        assert out == [int(x, 16) for x in c["out"]]


def test_normals_moments():
    n = 200000
    x = np.array([synth.normal_at(7, 1, f) for f in range(0, n, 97)])
    assert abs(x.mean()) < 0.05 and abs(x.std() - 1.0) < 0.05
    w = synth.Workload("t", "f32", 1, 2, 2, 64, 4096, 16, z=1.0, tau_mode="const",
                       densities=(0.5,), seed=5)
    q = synth.make_q(w)
    k, v = synth.make_kv(w, q)
    for t in (k, v):
        a = t.numpy().ravel()
        assert abs(a.mean()) < 0.02 and abs(a.std() - 1.0) < 0.02


def test_slice_regenerable_and_capacity_untouched():
    w = synth.Workload("t", "bf16", 2, 4, 2, 64, 1000, 16, z=1.0, tau_mode="const",
                       densities=(0.5,), seed=9, cap=1200)
    q = synth.make_q(w)
    k, v = synth.make_kv(w, q)
    assert k.shape == (2, 2, 1200, 64)
    assert torch.all(k[:, :, 1000:] == 0) and torch.all(v[:, :, 1000:] == 0)
    # element (b=1, h=1, s=17, i=5) of V is normal number ((1*2+1)*1000+17)*64+5 of stream V
    f = ((1 * 2 + 1) * 1000 + 17) * 64 + 5
    x = synth.normal_at(9, synth.STREAM_V, f)
    ref = torch.tensor([x], dtype=torch.float32).to(torch.bfloat16)
    assert v[1, 1, 17, 5] == ref[0]


def test_bf16_round_to_nearest_even_matches_torch():
    w = synth.Workload("t", "bf16", 1, 1, 1, 64, 256, 16, z=1.0, tau_mode="const",
                       densities=(0.5,), seed=3)
    q = synth.make_q(w)
    k, _ = synth.make_kv(w, q)
    w32 = w.replace(dtype="f32")
    q32 = synth.make_q(w32)
    k32, _ = synth.make_kv(w32, q32)
    assert torch.equal(k32.to(torch.bfloat16), k)


def test_needles_are_query_aligned():
    w = synth.WORKLOADS[2].replace(n=64 * 64, B=1, Hq=2, Hkv=2)
    q = synth.make_q(w)
    nd = synth.make_needles(w)
    assert nd.shape == (1, 2, 8)
    k, _ = synth.make_kv(w, q)
    qh = q[0, 0].float() / q[0, 0].float().norm()
    blk = int(nd[0, 0, 0])
    proj_needle = (k[0, 0, blk * 64:(blk + 1) * 64].float() @ qh).mean().item()
    other = [b for b in range(w.nb) if b not in set(nd[0, 0].tolist())][0]
    proj_other = (k[0, 0, other * 64:(other + 1) * 64].float() @ qh).mean().item()
    assert abs(proj_needle - 3.0) < 0.5 and abs(proj_other) < 0.5
    assert len(set(nd[0, 0].tolist())) == 8 and max(nd[0, 0].tolist()) < w.n_screened


def test_block_offsets_shared_within_block():
    w = synth.WORKLOADS[3].replace(B=1, Hq=4, Hkv=1, n=32 * 64)
    q = synth.make_q(w)
    k, _ = synth.make_kv(w, q)
    kb = k[0, 0].float().reshape(64, 32, w.d)   # [blocks][rows][d]
    means = kb.mean(dim=1)                      # ~ offset + N(0, 1/32)
    # offsets ~ N(0, 0.5): variance of block means ~ 0.5 + 1/32
    var = means.var().item()
    assert 0.4 < var < 0.7


def test_tau_for_density():
    s = np.arange(100, dtype=np.float32)
    t = synth.tau_for_density(s, 0.38)
    assert (s >= t).sum() == 38
    assert synth.tau_for_density(s, 1.0) == float("-inf")
    assert (s >= synth.tau_for_density(s, 0.001)).sum() == 1


def test_capacity_below_the_token_count_is_rejected():
    w = synth.Workload("c", "bf16", 1, 2, 2, 64, 1000, 16, z=1.0, tau_mode="const", densities=(0.5,), seed=1,
                       cap=512)
    with pytest.raises(ValueError):
        _ = w.capacity

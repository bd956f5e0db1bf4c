"""GPU parity: the CUDA path through the C ABI against the CPU oracle.

Lists, counts, scores, metadata and thresholds must match bit for bit;
outputs within 2e-3 (bf16) / 1e-5 (fp32) max-abs. Reduced sizes span several
tiles, clusters and split ranges with a ragged tail block; the full-size cases
run the launch configuration the benchmark times and check every list plus
sampled outputs."""
import math

import numpy as np
import pytest
import torch

import oracle
from learned_block_sparse_b200 import binding, synth
from learned_block_sparse_b200.workload import DeviceWorkload
from tests import parity

pytestmark = pytest.mark.gpu


def _full_check(w, density=None, n_splits=0, offset_a=0.0, heads=None, dense=False, keep_host=True):
    dw = DeviceWorkload(w, n_splits=n_splits, offset_a=offset_a, keep_host=keep_host)
    meta = parity.oracle_meta(w, dw.K_host)
    density = w.densities[0] if density is None else density
    tau, stride, bias = parity.oracle_thresholds(w, dw.q_host, meta, density, W=dw.W)
    all_heads = [(b, h) for b in range(w.B) for h in range(w.Hq)]
    heads = heads or all_heads
    gpu = parity.run_gpu(dw, tau, stride, bias=bias)
    assert gpu["status"] == 0
    if bias is not None:
        assert np.array_equal(gpu["tau"].view(np.int32), np.asarray(tau, np.float32).view(np.int32)), \
            "predicted thresholds differ from the oracle's"
    orc = parity.oracle_step(w, dw.q_host, dw.K_host, dw.V_host, meta, tau, stride, heads, offset_a=offset_a)
    err = parity.compare(w, gpu, orc, heads)
    res = {"err": err, "gpu": gpu, "dw": dw, "tau": tau, "stride": stride, "meta": meta}
    if dense:
        g = parity.run_gpu(dw, None, 0, dense=True)
        assert g["status"] == 0
        o = parity.oracle_step(w, dw.q_host, dw.K_host, dw.V_host, meta, None, 0, heads, dense=True)
        parity.compare(w, g, o, heads, check_lists=False)
    return res


# ------------------------------------------------------------------ metadata
@pytest.mark.parametrize("dtype,d,bs,n,cap", [
    ("f32", 64, 16, 1024, None), ("bf16", 128, 32, 32 * 70 + 5, 32 * 80),
    ("bf16", 64, 64, 64 * 9, None), ("bf16", 128, 128, 128 * 5 + 100, None), ("f32", 128, 64, 64 * 7 + 1, None),
    ("fp8", 128, 32, 32 * 33 + 7, None),
])
def test_block_meta_bit_exact(dtype, d, bs, n, cap):
    w = synth.Workload("m", dtype, 2, 4, 2, d, n, bs, z=1.0, tau_mode="const", densities=(0.5,), seed=31,
                       offset_std=0.7, cap=cap)
    dw = DeviceWorkload(w, keep_host=True)
    nf = w.n // w.bs
    for b in range(w.B):
        for h in range(w.Hkv):
            mu, var, mx = oracle.slice_meta(dw.K_host[b, h], w.d, w.bs, nf)
            g_mu = dw.dec.mu[b, h, :, :nf].T.contiguous().cpu().numpy()
            g_var = dw.dec.var[b, h, :, :nf].T.contiguous().cpu().numpy()
            g_mx = dw.dec.maxnorm[b, h, :nf].cpu().numpy()
            assert np.array_equal(g_mu.view(np.int32), mu.view(np.int32))
            assert np.array_equal(g_var.view(np.int32), var.view(np.int32))
            assert np.array_equal(g_mx.view(np.int32), mx.view(np.int32))


def test_block_meta_partial_range_leaves_others():
    w = synth.Workload("m", "bf16", 1, 2, 2, 128, 64 * 10, 64, z=1.0, tau_mode="const", densities=(0.5,), seed=3)
    dw = DeviceWorkload(w, keep_host=True)
    dw.dec.mu.fill_(7.0)
    dw.dec.build_meta(dw.K, 3, 6)
    torch.cuda.synchronize()
    assert torch.all(dw.dec.mu[:, :, :, :3] == 7.0) and torch.all(dw.dec.mu[:, :, :, 6:] == 7.0)
    mu, _, _ = oracle.slice_meta(dw.K_host[0, 1], w.d, w.bs, 6)
    assert np.array_equal(dw.dec.mu[0, 1, :, 3:6].T.cpu().numpy(), mu[3:6])


# ----------------------------------------------------------------- predictor
@pytest.mark.parametrize("dtype,B,H,d", [("bf16", 3, 16, 128), ("f32", 2, 12, 64), ("bf16", 1, 32, 128)])
def test_predict_tau_bit_exact(dtype, B, H, d):
    g = torch.Generator().manual_seed(B * H + d)
    q = torch.randn(B, H, d, generator=g).to(torch.bfloat16 if dtype == "bf16" else torch.float32)
    W = torch.randn(H * d, H, generator=g) / math.sqrt(d)
    bias = torch.randn(H, generator=g)
    shape = binding.make_shape(B, H, H, d, 16, 16, q.dtype, q.dtype)
    tau = torch.empty(B, H, device="cuda")
    binding.predict_tau(shape, q.cuda(), W.cuda(), bias.cuda(), tau)
    ref = oracle.predict_tau(q, W.numpy(), bias.numpy())
    assert np.array_equal(tau.cpu().numpy().view(np.int32), ref.view(np.int32))
    tau0 = torch.empty(B, H, device="cuda")
    binding.predict_tau(shape, q.cuda(), torch.zeros_like(W).cuda(), torch.full((H,), -8.0).cuda(), tau0)
    assert torch.all(tau0 == -8.0)


# ------------------------------------------------------- the five workloads
def _reduced(i):
    base = synth.WORKLOADS[i]
    return {
        1: base,
        2: base.replace(Hq=4, Hkv=4, n=64 * 40 + 17),
        3: base.replace(B=2, Hq=8, Hkv=2, n=32 * 150 + 5),
        4: base.replace(Hq=4, Hkv=4, n=64 * 100 + 63),
        5: base.replace(B=3, Hq=4, Hkv=4, n=16 * 300 + 9),
        6: base.replace(B=2, n=64 * 120 + 9),
    }[i]


@pytest.mark.parametrize("cfg,density", [(1, 0.40), (2, 0.38), (3, 0.20), (3, 0.38), (3, 0.60), (4, 0.38),
                                         (5, 0.10), (5, 0.25), (5, 0.38), (5, 0.60), (5, 1.0), (6, 0.05),
                                         (6, 0.2)])
def test_workload_parity_reduced(cfg, density):
    r = _full_check(_reduced(cfg), density, dense=(cfg in (1, 4)))
    assert r["err"] <= parity.TOL[_reduced(cfg).dtype]


@pytest.mark.parametrize("n_splits", [1, 2, 7, 150, 1000])
def test_split_ranges_any_count(n_splits):
    w = _reduced(3).replace(B=3)
    _full_check(w, 0.38, n_splits=n_splits)


@pytest.mark.parametrize("G", [1, 2, 4, 8])
def test_group_sizes(G):
    w = synth.Workload("g", "bf16", 2, 2 * G, 2, 128, 32 * 40 + 3, 32, z=1.0, tau_mode="const",
                       densities=(0.3,), seed=40 + G, offset_std=synth.SQRT_HALF)
    _full_check(w, dense=True)


@pytest.mark.parametrize("dtype,d,bs", [("bf16", 64, 16), ("bf16", 64, 128), ("f32", 128, 32), ("f32", 64, 64),
                                        ("bf16", 128, 128), ("fp8", 128, 16), ("fp8", 128, 32), ("fp8", 128, 64),
                                        ("fp8", 128, 128)])
def test_dtypes_dims_blocks(dtype, d, bs):
    w = synth.Workload("x", dtype, 2, 4, 2, d, bs * 37 + bs // 2 + 1, bs, z=1.0, tau_mode="const",
                       densities=(0.35,), seed=7 * d + bs, offset_std=synth.SQRT_HALF)
    _full_check(w, dense=True)


@pytest.mark.parametrize("dtype,d,bs,n_splits", [
    ("bf16", 128, 64, 2), ("bf16", 128, 64, 5), ("bf16", 128, 128, 3), ("bf16", 128, 32, 4), ("bf16", 128, 16, 3),
    # rings with fewer stages than consumer warps (3 < 6, 6 < 8) and stage counts
    # that are not multiples of the warp count
    ("bf16", 128, 128, 1), ("bf16", 64, 128, 2), ("fp8", 128, 128, 2), ("bf16", 64, 64, 3), ("fp8", 128, 64, 3),
])
def test_long_ranges_reuse_every_stage_many_times(dtype, d, bs, n_splits):
    """Few split ranges, so each thread block streams hundreds of blocks through
    its ring and every stage is reused many times by different consumer warps."""
    w = synth.Workload("ring", dtype, 1, 4, 4, d, bs * 700 + 3, bs, z=1.0, tau_mode="const",
                       densities=(0.5,), seed=bs + n_splits + d, offset_std=synth.SQRT_HALF)
    _full_check(w, 0.5, n_splits=n_splits, dense=True)


@pytest.mark.parametrize("cfg,blocks", [(3, 151), (5, 301), (2, 41)])
def test_screen_plain_loads_when_metadata_rows_unaligned(cfg, blocks):
    """capacity / block_size not a multiple of 4: metadata rows are not 16-byte
    aligned, so the screen takes the plain-load kernel instead of TMA staging."""
    w = _reduced(cfg)
    w = w.replace(cap=blocks * w.bs)
    assert (w.capacity // w.bs) % 4 != 0
    _full_check(w, w.densities[0])


def test_edge_single_token_and_exact_blocks():
    for n in (1, 16, 17, 32):
        w = synth.Workload("e", "bf16", 1, 2, 2, 128, n, 16, z=1.0, tau_mode="const", densities=(0.5,), seed=n,
                           cap=64)
        _full_check(w, dense=True)


@pytest.mark.parametrize("cfg,n_local", [(5, 2), (5, 3), (3, 2), (6, 2)])
def test_edge_n_local(cfg, n_local):
    """More than one trailing block admitted unscreened (the pages' lwb = 2 of
    Table 12's header, read as two local window blocks; 3 as a further case)."""
    w = _reduced(cfg).replace(n_local=n_local)
    r = _full_check(w, 0.25)
    assert np.all(r["gpu"]["active_cnt"] >= n_local)


def test_edge_offset():
    w = _reduced(3)
    _full_check(w, 0.38, offset_a=0.4)
    _full_check(w, 0.38, offset_a=-0.8)


def test_extreme_thresholds():
    w = _reduced(2)
    dw = DeviceWorkload(w, keep_host=True)
    meta = parity.oracle_meta(w, dw.K_host)
    heads = [(0, h) for h in range(w.Hq)]
    for t in (float("inf"), float("-inf")):
        tau = np.full((w.Hq,), t, np.float32)
        gpu = parity.run_gpu(dw, tau, 0)
        orc = parity.oracle_step(w, dw.q_host, dw.K_host, dw.V_host, meta, tau, 0, heads)
        parity.compare(w, gpu, orc, heads)
        if t == float("inf"):
            assert np.all(gpu["active_cnt"] == 1)
        else:
            assert np.all(gpu["active_cnt"] == w.nb)


def test_dense_equals_softmax_and_sparse_at_minus_inf():
    w = _reduced(4)
    dw = DeviceWorkload(w, keep_host=True)
    dense = dw.dense().clone()
    tau = torch.full((w.Hq,), float("-inf"), device="cuda")
    sparse = dw.step(tau=tau, stride=0).clone()
    torch.cuda.synchronize()
    assert torch.allclose(dense, sparse, atol=1e-6, rtol=0)
    for h in range(w.Hq):
        k = dw.K_host[0, h, :w.n].double()
        v = dw.V_host[0, h, :w.n].double()
        qq = dw.q_host[0, h].double()
        ref = torch.softmax(k @ qq / math.sqrt(w.d), 0) @ v
        assert torch.max(torch.abs(dense[0, h].cpu().double() - ref)) < 2e-3


def test_repeat_calls_identical():
    w = _reduced(3)
    dw = DeviceWorkload(w)
    tau = torch.zeros((w.B, w.Hq), device="cuda")
    a = dw.step(tau=tau, stride=w.Hq).clone()
    b = dw.step(tau=tau, stride=w.Hq).clone()
    d1 = dw.dense().clone()
    d2 = dw.dense().clone()
    torch.cuda.synchronize()
    assert torch.equal(a, b) and torch.equal(d1, d2)
    # the split-partial counters in the workspace header are back at zero
    counters = dw.dec.ws[256:256 + 4 * 8192].view(torch.int32)
    assert int(torch.count_nonzero(counters)) == 0


@pytest.mark.parametrize("dtype,G,bs", [("bf16", 4, 32), ("bf16", 8, 64), ("f32", 2, 16), ("bf16", 1, 64)])
def test_thresholds_in_screen_equal_separate_predictor(dtype, G, bs):
    """eta_decode_sparse_predict (Eq. 1 formed inside the screening launch)
    gives the thresholds, lists and outputs of eta_predict_tau followed by
    eta_decode_sparse, bit for bit; both thresholds match the oracle's."""
    w = synth.Workload("p", dtype, 3, 4 * G, 4, 64 if G == 8 else 128, bs * 90 + 7, bs, z=1.0,
                       tau_mode="predictor", densities=(0.3,), seed=90 + G + bs, offset_std=synth.SQRT_HALF)
    dw = DeviceWorkload(w, keep_host=True)
    meta = parity.oracle_meta(w, dw.K_host)
    tau, _, bias = parity.oracle_thresholds(w, dw.q_host, meta, 0.3, W=dw.W)
    b_dev = torch.as_tensor(bias, device="cuda")
    nb_cap = w.capacity // w.bs

    def outs():
        return dict(active_idx=torch.full((w.B, w.Hq, nb_cap), -1, dtype=torch.int32, device="cuda"),
                    active_cnt=torch.zeros((w.B, w.Hq), dtype=torch.int32, device="cuda"),
                    union_cnt=torch.zeros((w.B, w.Hkv), dtype=torch.int32, device="cuda"))

    o1 = outs()
    fused = dw.dec.step(dw.q, dw.K, dw.V, w.n, W=dw.W, bias=b_dev, **o1).clone()
    tau_fused = dw.dec.tau.clone()
    tau_sep = torch.empty_like(tau_fused)
    binding.predict_tau(dw.dec.shape, dw.q, dw.W, b_dev, tau_sep)
    o2 = outs()
    sep = dw.dec.step(dw.q, dw.K, dw.V, w.n, tau=tau_sep, tau_batch_stride=w.Hq, **o2).clone()
    torch.cuda.synchronize()
    assert dw.dec.device_status() == 0
    want = np.asarray(tau, np.float32).reshape(w.B, w.Hq).view(np.int32)
    assert np.array_equal(tau_fused.cpu().numpy().view(np.int32), want)
    assert np.array_equal(tau_sep.cpu().numpy().view(np.int32), want)
    for k in o1:
        assert torch.equal(o1[k], o2[k]), k
    assert torch.equal(fused, sep)


@pytest.mark.parametrize("dtype,G,bs", [("bf16", 4, 32), ("bf16", 8, 64), ("f32", 1, 16), ("bf16", 1, 16),
                                        ("fp8", 4, 32), ("fp8", 8, 16)])
def test_strict_mode_gate(dtype, G, bs):
    """Strict mode (keys below tau removed): lists and outputs against the oracle.
    Each head's tau sits in a wide gap of its own true logits, so the keep/remove
    decision does not depend on how either side rounds S."""
    d = 128 if dtype == "fp8" else (64 if (G == 8 or dtype == "f32") else 128)
    w = synth.Workload("strict", dtype, 2, 2 * G, 2, d, bs * 60 + 5, bs, z=1.0, tau_mode="const",
                       densities=(0.5,), seed=300 + G + bs, offset_std=synth.SQRT_HALF)
    dw = DeviceWorkload(w, keep_host=True, gate=binding.GATE_HARD)
    meta = parity.oracle_meta(w, dw.K_host)
    qf = oracle.to_f32(dw.q_host).astype(np.float64)
    tau = np.zeros((w.B, w.Hq), np.float32)
    for b in range(w.B):
        for h in range(w.Hq):
            k = dw.K_host[b, h // w.G, :w.n].double().numpy()
            S = np.sort(k @ qf[b, h] / math.sqrt(w.d))
            i0 = int(0.85 * w.n)
            i = max(range(i0 - 40, i0 + 40), key=lambda j: S[j + 1] - S[j])
            assert S[i + 1] - S[i] > 1e-4
            tau[b, h] = np.float32(0.5 * (S[i] + S[i + 1]))
    gpu = parity.run_gpu(dw, tau, w.Hq)
    assert gpu["status"] == 0
    heads = [(b, h) for b in range(w.B) for h in range(w.Hq)]
    orc = parity.oracle_step(w, dw.q_host, dw.K_host, dw.V_host, meta, tau, w.Hq, heads, gate=oracle.GATE_HARD)
    parity.compare(w, gpu, orc, heads)


@pytest.mark.parametrize("G,density", [(1, 0.3), (4, 0.38), (8, 0.2)])
def test_fp8_kv_workloads(G, density):
    """fp8 (e4m3) K and V with bf16 queries, GQA groups up to 8, predictor
    thresholds formed in the screen: lists bit-exact, outputs within 2e-3 of the
    oracle reading the same fp8 bytes; the dense pass too."""
    w = synth.Workload("fp8", "fp8", 2, 4 * G, 4, 128, 32 * 150 + 5, 32, z=1.0, tau_mode="predictor",
                       densities=(density,), seed=600 + G, offset_std=synth.SQRT_HALF)
    _full_check(w, density, dense=True)


# ----------------------------------------------------------------- full size
def _sample_heads(w, k, seed=0):
    rng = np.random.default_rng(seed)
    pairs = [(b, h) for b in range(w.B) for h in range(w.Hq)]
    idx = rng.choice(len(pairs), size=min(k, len(pairs)), replace=False)
    return sorted(pairs[i] for i in idx)


def _full_size(w, densities, list_pairs=None, streamed=False):
    """Full-size workload in the benchmark's launch configuration: for each
    density, every list, score, count and union on the given (b, kvh) pairs
    (default all), thresholds bit-exact, and the outputs of every head of those
    pairs, against the oracle. streamed: the cache is generated straight into
    device memory and only the sampled batch rows are regenerated on the host
    for the oracle (caches far larger than host memory needs)."""
    if isinstance(densities, float):
        densities = (densities,)
    pairs = list_pairs or [(b, h) for b in range(w.B) for h in range(w.Hkv)]
    if streamed:
        dw = DeviceWorkload(w)
        K_host, V_host = parity.host_rows(w, dw.q_host, [b for b, _ in pairs], dw.needles)
    else:
        dw = DeviceWorkload(w, keep_host=True)
        K_host, V_host = dw.K_host, dw.V_host
    meta = parity.oracle_meta(w, K_host, pairs)
    list_heads = [(b, kvh * w.G + g) for (b, kvh) in pairs for g in range(w.G)]
    got = []
    for density in densities:
        tau, stride, bias = parity.oracle_thresholds(w, dw.q_host, meta, density, W=dw.W, heads=list_heads)
        gpu = parity.run_gpu(dw, tau, stride, bias=bias)
        assert gpu["status"] == 0
        if bias is not None:
            assert np.array_equal(gpu["tau"].view(np.int32), np.asarray(tau, np.float32).view(np.int32))
        orc = parity.oracle_step(w, dw.q_host, K_host, V_host, meta, tau, stride, list_heads)
        parity.compare(w, gpu, orc, list_heads)
        got.append(sum(int(gpu["active_cnt"][b, h]) for (b, h) in list_heads) / (len(list_heads) * w.nb))
    return got[0] if len(got) == 1 else got


def test_full_size_gqa_128k_bench_config():
    """The benchmark's workload at its three densities (20 / 38 / 60% per head)."""
    w = synth.WORKLOADS[3]
    pairs = [(0, 0), (3, 5), (7, 7)]
    d20, d38, d60 = _full_size(w, (0.20, 0.38, 0.60), list_pairs=pairs)
    assert 0.12 < d20 < 0.3 and 0.3 < d38 < 0.5 and 0.5 < d60 < 0.7


def test_full_size_mha_32k_needles():
    _full_size(synth.WORKLOADS[2], 0.38)


def test_full_size_512k_sampled():
    w = synth.WORKLOADS[4]
    _full_size(w, 0.38, list_pairs=[(0, 2), (0, 11)])


def test_full_size_64k_b16_batch16_sampled():
    """The calibrated-constant sweep at batch 16: 10%, 25% and 100% (every block)."""
    w = synth.WORKLOADS[5].replace(B=16)
    d10, d25, d100 = _full_size(w, (0.10, 0.25, 1.0), list_pairs=[(0, 0), (9, 3), (15, 15)])
    assert d10 < d25 < d100 == 1.0


def test_full_size_64k_b16_batch64_rows_past_2_31():
    """The sweep's largest batch (64 rows, 32 GiB of K and V): the last rows'
    element offsets exceed 2^31. Lists and outputs of rows 0, 31 and 63 against
    the oracle at 38% and 60%."""
    w = synth.WORKLOADS[5].replace(B=64)
    assert ((63 * w.Hkv + 15) * w.capacity * w.d) > 2 ** 31
    _full_size(w, (0.38, 0.60), list_pairs=[(0, 0), (31, 8), (63, 15)], streamed=True)


def test_full_size_fp8_gqa_128k():
    """Workload 7 (the 128K GQA workload with fp8 K/V) at full size."""
    w = synth.WORKLOADS[7]
    dens = _full_size(w, 0.38, list_pairs=[(0, 0), (5, 3), (7, 7)])
    assert 0.3 < dens < 0.5


def test_full_size_table10_shape_sampled():
    """The pages' Table 10 head shape (32/4 heads, d 64, b 64) at 512K tokens, batch 4."""
    w = synth.WORKLOADS[6].replace(B=4)
    _full_size(w, 0.05, list_pairs=[(0, 0), (3, 3)])


def test_full_size_table10_shape_batch64_rows_past_2_31():
    """Table 10's own batch (64 rows of 512K tokens, 32 GiB of K and V): rows 0,
    40 and 63 against the oracle, thresholds of every row bit-exact."""
    w = synth.WORKLOADS[6]
    assert w.B == 64 and ((63 * w.Hkv + 3) * w.capacity * w.d) > 2 ** 31
    _full_size(w, (0.12, 0.25), list_pairs=[(0, 1), (40, 2), (63, 3)], streamed=True)

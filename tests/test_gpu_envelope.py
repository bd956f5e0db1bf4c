"""Sub-block envelope screen (a labelled reading of the pages' undefined
"sub-block envelope": a block's score is the largest Eq. 5 score of its r
sub-blocks) on the GPU against the oracle: sub-block metadata, lists, union
lists and envelope scores bit-exact, outputs within tolerance; both screening
kernels (TMA-staged and plain loads), the predictor, per-row lengths, and the
equality of the z -> infinity envelope with the flat screen."""
import numpy as np
import pytest
import torch

import oracle
from learned_block_sparse_b200 import binding, synth
from learned_block_sparse_b200.workload import DeviceWorkload
from tests import parity

pytestmark = pytest.mark.gpu


def _check(w, r, density, dense=False):
    dw = DeviceWorkload(w, keep_host=True, sub_blocks=r)
    meta = parity.oracle_meta(w, dw.K_host, r=r)
    nf = (w.n // w.bs) * r
    for (b, h), (mu, var, mx) in meta.items():
        assert np.array_equal(dw.dec.mu[b, h, :, :nf].T.contiguous().cpu().numpy().view(np.int32), mu.view(np.int32))
        assert np.array_equal(dw.dec.var[b, h, :, :nf].T.contiguous().cpu().numpy().view(np.int32),
                              var.view(np.int32))
        assert np.array_equal(dw.dec.maxnorm[b, h, :nf].cpu().numpy().view(np.int32), mx.view(np.int32))
    tau, stride, bias = parity.oracle_thresholds(w, dw.q_host, meta, density, W=dw.W, r=r)
    heads = [(b, h) for b in range(w.B) for h in range(w.Hq)]
    gpu = parity.run_gpu(dw, tau, stride, bias=bias)
    assert gpu["status"] == 0
    if bias is not None:
        assert np.array_equal(gpu["tau"].view(np.int32), np.asarray(tau, np.float32).view(np.int32))
    orc = parity.oracle_step(w, dw.q_host, dw.K_host, dw.V_host, meta, tau, stride, heads, r=r)
    parity.compare(w, gpu, orc, heads)
    return dw, meta


@pytest.mark.parametrize("dtype,Hq,Hkv,d,bs,r,mode,cap", [
    ("bf16", 8, 2, 128, 64, 4, "predictor", None),   # GQA, thresholds formed in the screen
    ("bf16", 32, 4, 64, 64, 4, "const", None),       # the pages' Table 10 head shape (G = 8)
    ("bf16", 4, 4, 128, 32, 2, "const", None),
    ("f32", 4, 2, 64, 128, 8, "predictor", None),
    ("fp8", 8, 2, 128, 64, 4, "const", None),
    ("bf16", 8, 2, 128, 64, 2, "const", 64 * 47),    # 94 metadata columns: the plain-load kernel
    ("bf16", 4, 1, 64, 128, 4, "predictor", 128 * 47),  # 188 columns: TMA, 4-lane groups
])
def test_envelope_matches_oracle(dtype, Hq, Hkv, d, bs, r, mode, cap):
    w = synth.Workload("env", dtype, 2, Hq, Hkv, d, bs * 44 + 7, bs, z=1.0, tau_mode=mode, densities=(0.35,),
                       seed=1300 + bs + r + Hq, offset_std=synth.SQRT_HALF, cap=cap)
    _check(w, r, 0.35)


def test_envelope_without_moment_term_equals_flat_screen():
    """z -> infinity leaves the Cauchy-Schwarz term: the envelope over sub-blocks
    then takes exactly the flat screen's decisions and scores."""
    w = synth.Workload("envz", "bf16", 2, 8, 2, 128, 64 * 60 + 3, 64, z=1e30, tau_mode="const", densities=(0.4,),
                       seed=1400, offset_std=synth.SQRT_HALF)
    flat = DeviceWorkload(w, keep_host=True)
    env = DeviceWorkload(w, keep_host=True, sub_blocks=4)
    tau = torch.full((w.Hq,), 0.6, device="cuda")
    nb_cap = w.capacity // w.bs
    res = []
    for dw in (flat, env):
        sc = torch.full((w.B, w.Hq, nb_cap), float("nan"), device="cuda")
        idx = torch.full((w.B, w.Hq, nb_cap), -1, dtype=torch.int32, device="cuda")
        cnt = torch.full((w.B, w.Hq), -1, dtype=torch.int32, device="cuda")
        out = dw.dec.step(dw.q, dw.K, dw.V, w.n, tau=tau, tau_batch_stride=0, scores=sc, active_idx=idx,
                          active_cnt=cnt).clone()
        torch.cuda.synchronize()
        assert dw.dec.device_status() == 0
        res.append((sc[..., :w.n_screened].cpu(), cnt.cpu(), idx.cpu(), out.cpu()))
    assert torch.equal(res[0][0].view(torch.int32), res[1][0].view(torch.int32))
    assert torch.equal(res[0][1], res[1][1])
    for b in range(w.B):
        for h in range(w.Hq):
            c = int(res[0][1][b, h])
            assert torch.equal(res[0][2][b, h, :c], res[1][2][b, h, :c])
    assert torch.equal(res[0][3], res[1][3])


def test_envelope_with_per_row_lengths():
    w = synth.Workload("envr", "bf16", 5, 8, 2, 128, 64 * 50 + 9, 64, z=1.0, tau_mode="const", densities=(0.3,),
                       seed=1500, offset_std=synth.SQRT_HALF)
    r = 4
    dw = DeviceWorkload(w, keep_host=True, sub_blocks=r)
    meta = parity.oracle_meta(w, dw.K_host, r=r)
    tau, _, _ = parity.oracle_thresholds(w, dw.q_host, meta, 0.3, r=r)
    lens = [1, w.bs, w.bs + 1, w.n, 777]
    seq = torch.tensor(lens, dtype=torch.int32, device="cuda")
    nb_cap = w.capacity // w.bs
    idx = torch.full((w.B, w.Hq, nb_cap), -1, dtype=torch.int32, device="cuda")
    cnt = torch.full((w.B, w.Hq), -1, dtype=torch.int32, device="cuda")
    out = dw.dec.step(dw.q, dw.K, dw.V, w.n, tau=torch.as_tensor(tau, device="cuda"), tau_batch_stride=0,
                      seq_lens=seq, active_idx=idx, active_cnt=cnt).clone()
    torch.cuda.synchronize()
    assert dw.dec.device_status() == 0
    qf = oracle.to_f32(dw.q_host)
    o_gpu, idx, cnt = out.cpu().numpy(), idx.cpu().numpy(), cnt.cpu().numpy()
    for b, n_b in enumerate(lens):
        nb_b = (n_b + w.bs - 1) // w.bs
        for h in range(w.Hq):
            mu, var, mx = meta[(b, h // w.G)]
            lst, _ = oracle.screen_head_env(qf[b, h], mu, var, mx, nb_b, r, w.n_local, w.z, float(tau[h]))
            assert int(cnt[b, h]) == len(lst) and np.array_equal(idx[b, h, :len(lst)], lst), (b, h)
            o = oracle.attend_head(dw.K_host[b, h // w.G], dw.V_host[b, h // w.G], w.bs, n_b, qf[b, h], lst,
                                   float(tau[h]), w.beta)
            assert float(np.max(np.abs(o_gpu[b, h] - o))) <= parity.TOL["bf16"], (b, h)


def test_full_size_envelope_table10_shape():
    """The pages' attention shape (batch 64 in the pages, 2 here; 512K, 32/4 heads,
    d 64, b 64) with sub-blocks of 16 tokens: sampled heads against the oracle."""
    w = synth.WORKLOADS[6].replace(B=2)
    r = 4
    dw = DeviceWorkload(w, sub_blocks=r, keep_host=True)
    rng = np.random.default_rng(3)
    pairs = sorted({(int(rng.integers(w.B)), int(rng.integers(w.Hkv))) for _ in range(3)})
    meta = parity.oracle_meta(w, dw.K_host, pairs, r=r)
    heads = [(b, kvh * w.G + g) for (b, kvh) in pairs for g in range(w.G)]
    tau, stride, bias = parity.oracle_thresholds(w, dw.q_host, meta, 0.3, W=dw.W, heads=heads, r=r)
    gpu = parity.run_gpu(dw, tau, stride, bias=bias)
    assert gpu["status"] == 0
    orc = parity.oracle_step(w, dw.q_host, dw.K_host, dw.V_host, meta, tau, stride, heads, r=r)
    parity.compare(w, gpu, orc, heads)

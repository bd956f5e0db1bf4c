"""Per-row lengths (eta_*_ragged): every batch row screens and attends exactly
as a uniform-length call with that row's token count would; checked against
the oracle run row by row with each row's own n (lists bit-exact, scores
bit-exact, outputs within tolerance), plus the dense pass, invalid lengths and
replay of a captured CUDA graph with changed lengths."""
import numpy as np
import pytest
import torch

import oracle
from learned_block_sparse_b200 import binding, synth
from learned_block_sparse_b200.workload import DeviceWorkload
from tests import parity

pytestmark = pytest.mark.gpu


def _lengths(w, seed):
    """Edge lengths first (one token, one full block, one past a block, the
    maximum), then seeded draws."""
    edge = [1, w.bs, w.bs + 1, w.n, 2 * w.bs - 1]
    rng = np.random.default_rng(seed)
    rest = list(rng.integers(1, w.n + 1, size=max(0, w.B - len(edge))))
    return [int(x) for x in (edge + rest)[:w.B]]


def _outs(w):
    nb_cap = w.capacity // w.bs
    return dict(active_idx=torch.full((w.B, w.Hq, nb_cap), -1, dtype=torch.int32, device="cuda"),
                active_cnt=torch.full((w.B, w.Hq), -1, dtype=torch.int32, device="cuda"),
                union_list=torch.zeros((w.B, w.Hkv, nb_cap), dtype=torch.int32, device="cuda"),
                union_cnt=torch.full((w.B, w.Hkv), -1, dtype=torch.int32, device="cuda"),
                scores=torch.full((w.B, w.Hq, nb_cap), float("nan"), dtype=torch.float32, device="cuda"))


def _oracle_rows(w, dw, meta, lens, tau_bh, dense=False):
    return parity.oracle_rows(w, dw.q_host, dw.K_host, dw.V_host, meta, lens, tau_bh, dense)


def _compare(w, lens, outs, out, orc, check_lists=True):
    parity.compare_rows(w, lens, outs, out, orc, check_lists)


@pytest.mark.parametrize("dtype,Hq,Hkv,d,bs,mode", [
    ("bf16", 8, 2, 128, 32, "predictor"),   # GQA, thresholds formed in the screen
    ("bf16", 32, 4, 64, 64, "const"),       # the pages' Table 10 head shape
    ("bf16", 4, 4, 128, 16, "const"),       # 16-token blocks, 8-warp decode
    ("f32", 4, 2, 64, 16, "predictor"),     # CUDA-core decode
    ("fp8", 8, 2, 128, 32, "const"),        # fp8 K/V
    ("bf16", 16, 4, 128, 64, "predictor"),  # d = 128: a block is two 32-row ring positions
    ("bf16", 8, 2, 128, 128, "const"),      # four positions per block, whole ones past a row's end
    ("fp8", 8, 2, 128, 64, "predictor"),
])
def test_ragged_rows_match_per_row_oracle(dtype, Hq, Hkv, d, bs, mode):
    w = synth.Workload("ragged", dtype, 7, Hq, Hkv, d, bs * 70 + 9, bs, z=1.0, tau_mode=mode,
                       densities=(0.3,), seed=500 + bs + Hq, offset_std=synth.SQRT_HALF)
    dw = DeviceWorkload(w, keep_host=True)
    meta = parity.oracle_meta(w, dw.K_host)
    tau, stride, bias = parity.oracle_thresholds(w, dw.q_host, meta, 0.3, W=dw.W)
    lens = _lengths(w, seed=bs)
    seq = torch.tensor(lens, dtype=torch.int32, device="cuda")
    outs = _outs(w)
    if bias is not None:
        out = dw.dec.step(dw.q, dw.K, dw.V, w.n, W=dw.W, bias=torch.as_tensor(bias, device="cuda"),
                          seq_lens=seq, **outs).clone()
        tau_arr = np.asarray(tau, np.float32).reshape(w.B, w.Hq)
        assert np.array_equal(dw.dec.tau.cpu().numpy().view(np.int32), tau_arr.view(np.int32))

        def tau_bh(b, h):
            return float(tau_arr[b, h])
    else:
        t_dev = torch.as_tensor(tau, device="cuda")
        out = dw.dec.step(dw.q, dw.K, dw.V, w.n, tau=t_dev, tau_batch_stride=0, seq_lens=seq, **outs).clone()

        def tau_bh(b, h):
            return float(np.asarray(tau, np.float32)[h])
    torch.cuda.synchronize()
    assert dw.dec.device_status() == 0
    _compare(w, lens, outs, out, _oracle_rows(w, dw, meta, lens, tau_bh))
    dense = dw.dec.dense(dw.q, dw.K, dw.V, w.n, seq_lens=seq).clone()
    torch.cuda.synchronize()
    assert dw.dec.device_status() == 0
    _compare(w, lens, None, dense, _oracle_rows(w, dw, meta, lens, tau_bh, dense=True), check_lists=False)


def test_uniform_lengths_equal_the_uniform_call():
    w = synth.WORKLOADS[3].replace(B=3, Hq=8, Hkv=2, n=32 * 90 + 5)
    dw = DeviceWorkload(w)
    tau = torch.zeros((w.B, w.Hq), device="cuda")
    a = dw.dec.step(dw.q, dw.K, dw.V, w.n, tau=tau).clone()
    seq = torch.full((w.B,), w.n, dtype=torch.int32, device="cuda")
    b = dw.dec.step(dw.q, dw.K, dw.V, w.n, tau=tau, seq_lens=seq).clone()
    d1 = dw.dec.dense(dw.q, dw.K, dw.V, w.n).clone()
    d2 = dw.dec.dense(dw.q, dw.K, dw.V, w.n, seq_lens=seq).clone()
    torch.cuda.synchronize()
    assert dw.dec.device_status() == 0
    assert torch.equal(a, b) and torch.equal(d1, d2)


def test_lengths_out_of_range_set_the_status_and_are_clamped():
    w = synth.WORKLOADS[3].replace(B=3, Hq=8, Hkv=2, n=32 * 40 + 3)
    dw = DeviceWorkload(w)
    tau = torch.zeros((w.B, w.Hq), device="cuda")
    good = dw.dec.step(dw.q, dw.K, dw.V, w.n, tau=tau,
                       seq_lens=torch.tensor([1, w.n, w.n], dtype=torch.int32, device="cuda")).clone()
    torch.cuda.synchronize()
    assert dw.dec.device_status() == 0
    bad = dw.dec.step(dw.q, dw.K, dw.V, w.n, tau=tau,
                      seq_lens=torch.tensor([0, w.n + 5, w.n], dtype=torch.int32, device="cuda")).clone()
    torch.cuda.synchronize()
    assert dw.dec.device_status() == binding.ETA_ERR_INVALID_ARG
    assert torch.equal(good, bad)       # 0 -> 1 and n + 5 -> n
    assert dw.dec.device_status() == 0  # reading the status cleared it


def test_graph_replay_reads_the_new_lengths():
    w = synth.WORKLOADS[3].replace(B=4, Hq=8, Hkv=2, n=32 * 80 + 11)
    dw = DeviceWorkload(w)
    tau = torch.zeros((w.B, w.Hq), device="cuda")
    seq = torch.tensor([w.n, 33, 1, 500], dtype=torch.int32, device="cuda")
    out = torch.empty((w.B, w.Hq, w.d), dtype=torch.float32, device="cuda")
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):   # warm-up outside capture (attributes, first launches)
        dw.dec.step(dw.q, dw.K, dw.V, w.n, tau=tau, seq_lens=seq, out=out)
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        dw.dec.step(dw.q, dw.K, dw.V, w.n, tau=tau, seq_lens=seq, out=out)
    for lens in ([w.n, 33, 1, 500], [7, w.n, 64, 65], [1, 1, 1, 1]):
        seq.copy_(torch.tensor(lens, dtype=torch.int32))
        g.replay()
        replayed = out.clone()
        direct = dw.dec.step(dw.q, dw.K, dw.V, w.n, tau=tau,
                             seq_lens=torch.tensor(lens, dtype=torch.int32, device="cuda")).clone()
        torch.cuda.synchronize()
        assert torch.equal(replayed, direct), lens
    del g
    assert dw.dec.device_status() == 0


@pytest.mark.parametrize("dtype,d,bs", [("bf16", 128, 32), ("bf16", 128, 16), ("bf16", 64, 64), ("f32", 64, 16),
                                        ("fp8", 128, 32), ("bf16", 128, 128), ("fp8", 128, 64), ("bf16", 64, 128)])
def test_cache_rows_past_each_length_are_never_used(dtype, d, bs):
    """Tokens at or past a row's length (the rest of its last block and beyond)
    may hold anything: filling them with NaN changes no output bit. With blocks
    of 64 and 128 tokens the tensor-core decode loads a block as chunks of 32
    rows, and whole chunks past a row's end are never loaded nor attended."""
    w = synth.Workload("tail", dtype, 5, 8, 2, d, bs * 40 + 9, bs, z=1.0, tau_mode="const",
                       densities=(0.3,), seed=900 + bs + d, offset_std=synth.SQRT_HALF)
    dw = DeviceWorkload(w)
    tau = torch.zeros((w.Hq,), device="cuda")
    lens = _lengths(w, seed=bs)
    seq = torch.tensor(lens, dtype=torch.int32, device="cuda")
    a = dw.dec.step(dw.q, dw.K, dw.V, w.n, tau=tau, tau_batch_stride=0, seq_lens=seq).clone()
    da = dw.dec.dense(dw.q, dw.K, dw.V, w.n, seq_lens=seq).clone()
    for b, n_b in enumerate(lens):
        for t in (dw.K, dw.V):
            if t.dtype == torch.float8_e4m3fn:
                t.view(torch.uint8)[b, :, n_b:] = 0x7f       # the e4m3 NaN code
            else:
                t[b, :, n_b:] = float("nan")
    b_ = dw.dec.step(dw.q, dw.K, dw.V, w.n, tau=tau, tau_batch_stride=0, seq_lens=seq).clone()
    db = dw.dec.dense(dw.q, dw.K, dw.V, w.n, seq_lens=seq).clone()
    torch.cuda.synchronize()
    assert dw.dec.device_status() == 0
    assert torch.isfinite(b_).all() and torch.isfinite(db).all()
    assert torch.equal(a, b_) and torch.equal(da, db)

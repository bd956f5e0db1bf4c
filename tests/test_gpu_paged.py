"""Paged KV pools (eta_*_paged): the K and V blocks of a contiguous cache are
scattered into randomly permuted pages of a pool. Metadata built from the pool
and every decode result (thresholds, lists, scores, unions, outputs, dense
outputs) are checked against the oracle run row by row on the same seeded
cache (bit-exact decisions, outputs within 2e-3 / 1e-5), and must also equal
the contiguous per-row-length calls bit for bit. A page index outside the pool
is reported in the device status word and never read."""
import numpy as np
import pytest
import torch

from learned_block_sparse_b200 import binding, synth
from learned_block_sparse_b200.workload import DeviceWorkload
from tests import parity

pytestmark = pytest.mark.gpu


def _pool(dw, seed, spare=7):
    """Pools [pages][Hkv][bs][d] holding dw's K and V behind a permuted block table."""
    w = dw.w
    nbc = w.capacity // w.bs
    pages = w.B * nbc + spare
    g = torch.Generator().manual_seed(seed)
    table = torch.randperm(pages, generator=g)[:w.B * nbc].view(w.B, nbc).to(torch.int32)
    idx = table.view(-1).long().cuda()
    pools = []
    for src in (dw.K, dw.V):
        # scatter the raw bits (works for every storage dtype); unused pages hold NaN codes
        raw = src.view(torch.uint8 if src.element_size() == 1 else
                       (torch.int16 if src.element_size() == 2 else torch.int32))
        blocks = raw.view(w.B, w.Hkv, nbc, w.bs, w.d).permute(0, 2, 1, 3, 4).reshape(w.B * nbc, w.Hkv, w.bs, w.d)
        nan = torch.full((1,), float("nan"), dtype=torch.float32).to(src.dtype if src.element_size() > 1 else
                                                                     torch.float32)
        pool = torch.empty((pages, w.Hkv, w.bs, w.d), dtype=raw.dtype, device="cuda")
        pool.fill_(0x7f if src.element_size() == 1 else int(nan.view(raw.dtype).item()))
        pool[idx] = blocks
        pools.append(pool.view(src.dtype))
    return pools[0], pools[1], table.cuda(), pages


def _lens(w, seed):
    edge = [1, w.bs, w.bs + 1, w.n, 2 * w.bs - 1]
    rng = np.random.default_rng(seed)
    rest = list(rng.integers(1, w.n + 1, size=max(0, w.B - len(edge))))
    return torch.tensor([int(x) for x in (edge + rest)[:w.B]], dtype=torch.int32, device="cuda")


def _outs(w):
    nb_cap = w.capacity // w.bs
    return dict(active_idx=torch.full((w.B, w.Hq, nb_cap), -1, dtype=torch.int32, device="cuda"),
                active_cnt=torch.zeros((w.B, w.Hq), dtype=torch.int32, device="cuda"),
                union_list=torch.zeros((w.B, w.Hkv, nb_cap), dtype=torch.int32, device="cuda"),
                union_cnt=torch.zeros((w.B, w.Hkv), dtype=torch.int32, device="cuda"),
                scores=torch.full((w.B, w.Hq, nb_cap), float("nan"), dtype=torch.float32, device="cuda"))


@pytest.mark.parametrize("dtype,Hq,Hkv,d,bs,mode", [
    ("bf16", 8, 2, 128, 32, "predictor"),
    ("bf16", 32, 4, 64, 64, "const"),
    ("bf16", 4, 4, 128, 16, "const"),
    ("f32", 4, 2, 64, 16, "predictor"),
    ("fp8", 8, 2, 128, 64, "const"),
    ("bf16", 8, 2, 128, 128, "predictor"),  # four 32-row ring positions per page
])
def test_paged_pool_against_oracle_and_contiguous_cache(dtype, Hq, Hkv, d, bs, mode):
    w = synth.Workload("paged", dtype, 6, Hq, Hkv, d, bs * 50 + 3, bs, z=1.0, tau_mode=mode,
                       densities=(0.3,), seed=700 + bs + Hq, offset_std=synth.SQRT_HALF)
    dw = DeviceWorkload(w, keep_host=True)
    dec = dw.dec
    k_pool, v_pool, table, pages = _pool(dw, seed=bs)
    # metadata from the pool: the oracle's bit for bit (and the contiguous builder's)
    mu = torch.full_like(dec.mu, float("nan"))
    var = torch.full_like(dec.var, float("nan"))
    mx = torch.full_like(dec.maxnorm, float("nan"))
    nfull = w.n // w.bs
    binding.build_block_meta_paged(dec.shape, k_pool, table, pages, 0, nfull, mu, var, mx)
    torch.cuda.synchronize()
    meta = parity.oracle_meta(w, dw.K_host)
    for b in range(w.B):
        for h in range(w.Hkv):
            o_mu, o_var, o_mx = meta[(b, h)]
            assert np.array_equal(mu[b, h, :, :nfull].T.contiguous().cpu().numpy().view(np.int32),
                                  o_mu.view(np.int32)), (b, h)
            assert np.array_equal(var[b, h, :, :nfull].T.contiguous().cpu().numpy().view(np.int32),
                                  o_var.view(np.int32)), (b, h)
            assert np.array_equal(mx[b, h, :nfull].cpu().numpy().view(np.int32), o_mx.view(np.int32)), (b, h)
    for a_, b_ in ((mu, dec.mu), (var, dec.var), (mx, dec.maxnorm)):
        assert torch.equal(a_[..., :nfull], b_[..., :nfull])

    # thresholds from the oracle side
    tau, stride, bias = parity.oracle_thresholds(w, dw.q_host, meta, 0.3, W=dw.W)
    tau_arr = np.asarray(tau, np.float32)
    if mode == "predictor":
        thr = dict(W=dw.W, bias=torch.as_tensor(bias, device="cuda"))

        def tau_bh(b, h):
            return float(tau_arr.reshape(w.B, w.Hq)[b, h])
    else:
        thr = dict(tau=torch.as_tensor(tau_arr, device="cuda"), tau_batch_stride=0)

        def tau_bh(b, h):
            return float(tau_arr[h])
    seq = _lens(w, seed=bs + 1)
    lens = [int(x) for x in seq.cpu()]
    out_c = torch.empty((w.B, w.Hq, w.d), dtype=torch.float32, device="cuda")
    out_p = torch.empty_like(out_c)
    tau_c = torch.empty((w.B, w.Hq), dtype=torch.float32, device="cuda")
    tau_p = torch.empty_like(tau_c)
    oc, op = _outs(w), _outs(w)
    extra_c = dict(tau_out=tau_c) if mode == "predictor" else {}
    extra_p = dict(tau_out=tau_p) if mode == "predictor" else {}
    binding.decode_sparse_paged(dec.shape, dec.params, dw.q, k_pool, v_pool, table, pages, (mu, var, mx), seq, w.n,
                                out_p, dec.ws, **thr, **extra_p, **op)
    torch.cuda.synchronize()
    assert dec.device_status() == 0
    if mode == "predictor":
        assert np.array_equal(tau_p.cpu().numpy().view(np.int32), tau_arr.reshape(w.B, w.Hq).view(np.int32))
    orc = parity.oracle_rows(w, dw.q_host, dw.K_host, dw.V_host, meta, lens, tau_bh)
    parity.compare_rows(w, lens, op, out_p, orc)
    # the same call on the contiguous cache: the same bits
    binding.decode_sparse_ragged(dec.shape, dec.params, dw.q, dw.K, dw.V, dec.meta, seq, w.n, out_c, dec.ws,
                                 **thr, **extra_c, **oc)
    torch.cuda.synchronize()
    assert dec.device_status() == 0
    for key in oc:   # bit patterns: unscreened score entries hold NaN on both sides
        assert torch.equal(oc[key].view(torch.int32), op[key].view(torch.int32)), key
    if mode == "predictor":
        assert torch.equal(tau_c, tau_p)
    assert torch.equal(out_c, out_p)

    # the dense pass over the pool: plain softmax attention per row, as the oracle's
    dense_c = torch.empty_like(out_c)
    dense_p = torch.empty_like(out_c)
    binding.decode_dense_paged(dec.shape, dec.params, dw.q, k_pool, v_pool, table, pages, seq, w.n, None, 0,
                               dense_p, dec.ws)
    binding.decode_dense_ragged(dec.shape, dec.params, dw.q, dw.K, dw.V, seq, w.n, None, 0, dense_c, dec.ws)
    torch.cuda.synchronize()
    assert dec.device_status() == 0
    orc_d = parity.oracle_rows(w, dw.q_host, dw.K_host, dw.V_host, meta, lens, tau_bh, dense=True)
    parity.compare_rows(w, lens, None, dense_p, orc_d, check_lists=False)
    assert torch.equal(dense_c, dense_p)


def test_page_outside_the_pool_is_reported_and_not_read():
    w = synth.WORKLOADS[3].replace(B=2, Hq=8, Hkv=2, n=32 * 30 + 5)
    dw = DeviceWorkload(w)
    dec = dw.dec
    k_pool, v_pool, table, pages = _pool(dw, seed=3, spare=0)
    seq = torch.tensor([w.n, w.n], dtype=torch.int32, device="cuda")
    bad = table.clone()
    bad[1, w.nb - 1] = pages          # the forced last block of row 1: always loaded
    out = torch.empty((w.B, w.Hq, w.d), dtype=torch.float32, device="cuda")
    tau = torch.zeros((w.B, w.Hq), device="cuda")
    binding.decode_sparse_paged(dec.shape, dec.params, dw.q, k_pool, v_pool, bad, pages, dec.meta, seq, w.n, out,
                                dec.ws, tau=tau, tau_batch_stride=w.Hq)
    torch.cuda.synchronize()
    assert dec.device_status() == binding.ETA_ERR_INVALID_ARG
    good = torch.empty_like(out)
    binding.decode_sparse_paged(dec.shape, dec.params, dw.q, k_pool, v_pool, table, pages, dec.meta, seq, w.n,
                                good, dec.ws, tau=tau, tau_batch_stride=w.Hq)
    torch.cuda.synchronize()
    assert dec.device_status() == 0
    assert torch.equal(out[0], good[0])   # row 0 does not touch the bad entry

"""Parity harness: run the CUDA path (through the C ABI) and the CPU oracle on
the same seeded inputs and compare. Thresholds always come from the oracle
side (oracle block scores -> quantile, oracle predictor), never from the GPU.

Bars: active-block lists, union lists, counts, block scores, metadata and
predicted thresholds bit-exact; outputs within 2e-3 max-abs for bf16 inputs
and 1e-5 for fp32 (fp32 accumulation against the oracle's double)."""
from __future__ import annotations

import concurrent.futures as cf
import os
from typing import Iterable, Optional

import numpy as np
import torch

import oracle
from learned_block_sparse_b200 import binding, synth

TOL = {"bf16": 2e-3, "fp8": 2e-3, "f32": 1e-5}
_POOL = cf.ThreadPoolExecutor(max_workers=max(1, min(32, os.cpu_count() or 1)))


def pmap(fn, items):
    return list(_POOL.map(lambda a: fn(*a), items))


def oracle_meta(w: synth.Workload, K_host: torch.Tensor, pairs: Optional[Iterable] = None, r: int = 1):
    """Oracle metadata for the given (b, kvh) pairs (default all): dict -> (mu, var, mx);
    with r > 1, of the sub-blocks of w.bs / r tokens (the sub-block envelope)."""
    Kraw = K_host
    nf = (w.n // w.bs) * r
    pairs = list(pairs) if pairs is not None else [(b, h) for b in range(w.B) for h in range(w.Hkv)]

    def one(b, h):
        return (b, h), oracle.slice_meta(Kraw[b, h], w.d, w.bs // r, nf)
    return dict(pmap(one, [(b, h) for (b, h) in pairs]))


def screen(qf, mu, var, mx, w, tau, offset_a=0.0, r=1):
    """The oracle screen of one head: Eq. 5 on whole blocks, or the sub-block envelope."""
    if r > 1:
        return oracle.screen_head_env(qf, mu, var, mx, w.nb, r, w.n_local, w.z, tau, offset_a)
    return oracle.screen_head(qf, mu, var, mx, w.nb, w.n_local, w.z, tau, offset_a)


def oracle_scores(w, qf: np.ndarray, meta: dict, heads, r=1):
    def one(b, hq):
        mu, var, mx = meta[(b, hq // w.G)]
        _, sc = screen(qf[b, hq], mu, var, mx, w, float("-inf"), r=r)
        return (b, hq), sc
    return dict(pmap(one, heads))


def oracle_thresholds(w, q_host, meta, density, W=None, heads=None, r=1):
    """Thresholds for a target density, computed on the oracle side.
    const: per-head constant over the batch, returns (tau [Hq], stride 0, None).
    predictor: returns (tau [B][Hq], stride Hq, bias [Hq])."""
    qf = oracle.to_f32(q_host)
    all_heads = [(b, h) for b in range(w.B) for h in range(w.Hq)]
    sc = oracle_scores(w, qf, meta, heads or all_heads, r=r)
    if w.tau_mode == "const":
        tau = np.zeros((w.Hq,), np.float32)
        for h in range(w.Hq):
            s = [sc[(b, h)] for b in range(w.B) if (b, h) in sc]
            # heads outside the sampled pairs keep 0 (any finite threshold is a valid input)
            tau[h] = synth.tau_for_density(np.concatenate(s), density) if s else 0.0
        return tau, 0, None
    Wn = W.cpu().numpy()
    tau0 = oracle.predict_tau(q_host, Wn, np.zeros(w.Hq, np.float32))
    bias = np.zeros((w.Hq,), np.float32)
    for h in range(w.Hq):
        # pooled over the batch: scores relative to each row's predicted tau
        rel = [sc[(b, h)].astype(np.float64) - tau0[b, h] for b in range(w.B) if (b, h) in sc]
        if rel:
            bias[h] = synth.tau_for_density(np.concatenate(rel), density)
        # heads outside the sampled pairs keep bias 0 (any finite threshold is a valid input)
    tau = oracle.predict_tau(q_host, Wn, bias)
    return tau, w.Hq, bias


def run_gpu(dw, tau, stride, bias=None, dense=False):
    """One decode step on the GPU with every optional screening output; returns numpy dict."""
    w = dw.w
    dev = dw.device
    nb_cap = w.capacity // w.bs
    res = {}
    if dense:
        out = dw.dec.dense(dw.q, dw.K, dw.V, w.n, tau=None if tau is None else torch.as_tensor(tau, device=dev),
                           tau_batch_stride=stride)
        torch.cuda.synchronize()
        res["out"] = out.cpu().numpy().copy()
        res["status"] = dw.dec.device_status()
        return res
    outs = dict(
        active_idx=torch.full((w.B, w.Hq, nb_cap), -1, dtype=torch.int32, device=dev),
        active_cnt=torch.full((w.B, w.Hq), -1, dtype=torch.int32, device=dev),
        union_list=torch.zeros((w.B, w.Hkv, nb_cap), dtype=torch.int32, device=dev),
        union_cnt=torch.full((w.B, w.Hkv), -1, dtype=torch.int32, device=dev),
        scores=torch.full((w.B, w.Hq, nb_cap), float("nan"), dtype=torch.float32, device=dev),
    )
    if bias is not None:
        b_dev = torch.as_tensor(bias, device=dev)
        out = dw.dec.step(dw.q, dw.K, dw.V, w.n, W=dw.W, bias=b_dev, **outs)
        res["tau"] = dw.dec.tau.cpu().numpy().copy()
    else:
        t_dev = torch.as_tensor(tau, device=dev).contiguous()
        out = dw.dec.step(dw.q, dw.K, dw.V, w.n, tau=t_dev, tau_batch_stride=stride, **outs)
    torch.cuda.synchronize()
    res["out"] = out.cpu().numpy().copy()
    for k_, v_ in outs.items():
        res[k_] = v_.cpu().numpy().copy()
    res["status"] = dw.dec.device_status()
    return res


def oracle_step(w, q_host, K_host, V_host, meta, tau, stride, heads, dense=False, offset_a=0.0,
                gate=oracle.GATE_SIGMOID, r=1):
    qf = oracle.to_f32(q_host)
    tau_arr = np.asarray(tau, np.float32)

    def tau_of(b, h):
        return float(tau_arr[h]) if stride == 0 else float(tau_arr.reshape(w.B, w.Hq)[b, h])

    def one(b, hq):
        kvh = hq // w.G
        if dense:
            lst, sc = np.arange(w.nb, dtype=np.int32), None
        else:
            mu, var, mx = meta[(b, kvh)]
            lst, sc = screen(qf[b, hq], mu, var, mx, w, tau_of(b, hq), offset_a, r)
        t_gate = float("-inf") if (dense and tau is None) else tau_of(b, hq)
        o = oracle.attend_head(K_host[b, kvh], V_host[b, kvh], w.bs, w.n, qf[b, hq], lst, t_gate, w.beta, gate)
        return (b, hq), (lst, sc, o)
    return dict(pmap(one, heads))


def compare(w, gpu, orc, heads, check_lists=True):
    """Assert parity for the given heads; returns (max abs err, head density, union density)."""
    tol = TOL[w.dtype]
    max_err = 0.0
    tot_head = 0
    for (b, hq) in heads:
        lst, sc, o = orc[(b, hq)]
        err = float(np.max(np.abs(gpu["out"][b, hq].astype(np.float64) - o)))
        assert err <= tol, f"output mismatch at (b={b}, h={hq}): max abs {err:.3g} > {tol}"
        max_err = max(max_err, err)
        if check_lists:
            cnt = int(gpu["active_cnt"][b, hq])
            assert cnt == len(lst), f"count mismatch at ({b},{hq}): gpu {cnt} oracle {len(lst)}"
            assert np.array_equal(gpu["active_idx"][b, hq, :cnt], lst), f"list mismatch at ({b},{hq})"
            ns = w.n_screened
            g_sc = gpu["scores"][b, hq, :ns]
            assert np.array_equal(g_sc.view(np.int32), sc.view(np.int32)), f"score bits differ at ({b},{hq})"
            tot_head += cnt
    if check_lists:
        kv_pairs = sorted({(b, hq // w.G) for (b, hq) in heads})
        for (b, kvh) in kv_pairs:
            group = [(b, kvh * w.G + g) for g in range(w.G)]
            if not all(gh in orc for gh in group):
                continue
            idx, mask = oracle.union_lists([orc[gh][0] for gh in group], w.nb)
            ucnt = int(gpu["union_cnt"][b, kvh])
            assert ucnt == len(idx), f"union count mismatch at ({b},{kvh})"
            packed = (idx.astype(np.int64) << 8) | mask.astype(np.int64)
            g_u = gpu["union_list"][b, kvh, :ucnt].astype(np.int64) & 0xffffffff
            assert np.array_equal(g_u, packed), f"union list mismatch at ({b},{kvh})"
    return max_err


def host_rows(w, q_host, batches, needles=None):
    """Host K and V of the given batch rows only, {(b, kv head): [capacity][d]}:
    the oracle's inputs for full-size workloads whose whole cache stays on the
    device (the same seeded bytes the device copy was filled with)."""
    K, V = {}, {}
    for b in sorted(set(batches)):
        for which, dst in (("k", K), ("v", V)):
            buf = torch.empty((1, w.Hkv, w.capacity, w.d), dtype=w.torch_dtype)
            synth.fill_kv(w, q_host, which, buf, b, b + 1, needles)
            for h in range(w.Hkv):
                dst[(b, h)] = buf[0, h]
    return K, V


def oracle_rows(w, q_host, K_host, V_host, meta, lens, tau_bh, dense=False, heads=None):
    """Per-row-length oracle: row b screens, gates and attends as a call with
    n = lens[b] (its own current token and forced trailing blocks)."""
    qf = oracle.to_f32(q_host)

    def one(b, hq):
        n_b = lens[b]
        nb_b = (n_b + w.bs - 1) // w.bs
        kvh = hq // w.G
        if dense:
            lst, sc = np.arange(nb_b, dtype=np.int32), None
            t = float("-inf")
        else:
            mu, var, mx = meta[(b, kvh)]
            t = tau_bh(b, hq)
            lst, sc = oracle.screen_head(qf[b, hq], mu, var, mx, nb_b, w.n_local, w.z, t)
        o = oracle.attend_head(K_host[b, kvh], V_host[b, kvh], w.bs, n_b, qf[b, hq], lst, t, w.beta)
        return (b, hq), (lst, sc, o)
    heads = heads or [(b, h) for b in range(w.B) for h in range(w.Hq)]
    return dict(pmap(one, heads))


def compare_rows(w, lens, outs, out, orc, check_lists=True):
    """Assert per-row parity: outputs within tolerance; counts, lists, scores and
    GQA unions bit-exact; no score written past a row's screened blocks."""
    tol = TOL[w.dtype]
    got = {k: v.cpu().numpy() for k, v in outs.items()} if check_lists else {}
    o_gpu = out.cpu().numpy()
    for (b, hq), (lst, sc, o) in orc.items():
        err = float(np.max(np.abs(o_gpu[b, hq].astype(np.float64) - o)))
        assert err <= tol, f"output of row {b} (n={lens[b]}) head {hq}: {err:.3g}"
        if not check_lists:
            continue
        cnt = int(got["active_cnt"][b, hq])
        assert cnt == len(lst) and np.array_equal(got["active_idx"][b, hq, :cnt], lst), (b, hq, lens[b])
        if "scores" in got:
            ns_b = max(0, (lens[b] + w.bs - 1) // w.bs - w.n_local)
            assert np.array_equal(got["scores"][b, hq, :ns_b].view(np.int32), sc.view(np.int32)), (b, hq)
            assert np.all(np.isnan(got["scores"][b, hq, ns_b:w.n_screened])), "scores past the row were written"
    if not check_lists:
        return
    for (b, kvh) in sorted({(b, hq // w.G) for (b, hq) in orc}):
        nb_b = (lens[b] + w.bs - 1) // w.bs
        idx, mask = oracle.union_lists([orc[(b, kvh * w.G + g)][0] for g in range(w.G)], nb_b)
        ucnt = int(got["union_cnt"][b, kvh])
        packed = (idx.astype(np.int64) << 8) | mask.astype(np.int64)
        assert ucnt == len(idx)
        assert np.array_equal(got["union_list"][b, kvh, :ucnt].astype(np.int64) & 0xffffffff, packed)

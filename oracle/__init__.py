"""CPU oracle for ETA block-sparse decode — TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package. It wraps ``oracle.c`` (plain C, built with
``-O2 -ffp-contract=off``) through ctypes and adds the plain set union that GQA
loading needs. It shares no code with the CUDA library and never calls it.

Method source: "Elastic Threshold Attention: Learned Contextual Sparsity for
Long-Context Decoding" — Eq. 1 (threshold predictor), Eq. 2-3 (sigmoid gate,
multiplicative logit gating with the current token exempt), Eq. 5 (dual
screening score) and the block index of Methodology §4; GQA union loading as
described with Figure 9 and Table 2 (a KV block is loaded when any head of its
group admits it; each head attends over its own admitted set).

Parity pins: every function here is pinned by tests in ``tests/test_oracle_*``
against closed forms, brute force and library routines (see the test docstrings).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import sys
from typing import Optional

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")

F32, BF16, FP8 = 0, 1, 2
CFLAGS = ["-O2", "-ffp-contract=off", "-fno-fast-math", "-std=c11", "-fPIC", "-shared"]


def build(force: bool = False) -> str:
    """Compile oracle.c into liboracle.so (gcc, no FMA contraction)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        cmd = ["gcc", *CFLAGS, _SRC, "-o", _LIB + ".tmp", "-lm"]
        subprocess.check_call(cmd)
        os.replace(_LIB + ".tmp", _LIB)
    return _LIB


_lib = None


def lib():
    global _lib
    if _lib is None:
        build()
        L = ctypes.CDLL(_LIB)
        vp, i32, i64, f32 = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_float
        L.oracle_to_f32.argtypes = [i32, vp, i64, vp]
        L.oracle_block_meta.argtypes = [i32, vp, i64, i32, i32, vp, vp, vp]
        L.oracle_slice_meta.argtypes = [i32, vp, i32, i32, i64, vp, vp, vp]
        L.oracle_predict_tau.argtypes = [vp, i32, i32, vp, vp, vp]
        L.oracle_block_score.argtypes = [vp, i32, vp, vp, f32, f32, f32]
        L.oracle_block_score.restype = f32
        L.oracle_inv_sqrt_d.argtypes = [i32]
        L.oracle_inv_sqrt_d.restype = f32
        L.oracle_screen_head.argtypes = [vp, i32, vp, vp, vp, i64, i32, f32, f32, f32, vp, vp]
        L.oracle_screen_head.restype = i32
        L.oracle_screen_head_env.argtypes = [vp, i32, vp, vp, vp, i64, i32, i32, f32, f32, f32, vp, vp]
        L.oracle_screen_head_env.restype = i32
        L.oracle_attend_head.argtypes = [i32, vp, vp, i32, i32, i64, vp, vp, i32, f32, f32, i32, vp]
        L.oracle_block_stats.argtypes = [i32, vp, i32, i32, i64, i32, vp, f32, f32, f32, i32, vp, vp, vp]
        for fn in ("oracle_to_f32", "oracle_block_meta", "oracle_slice_meta",
                   "oracle_predict_tau", "oracle_attend_head", "oracle_block_stats"):
            getattr(L, fn).restype = None
        _lib = L
    return _lib


def _raw(x):
    """numpy view of the stored bits: float32 stays float32, bf16 becomes uint16,
    fp8 e4m3 becomes uint8."""
    try:
        import torch
        if isinstance(x, torch.Tensor):
            x = x.detach().cpu().contiguous()
            if x.dtype == torch.bfloat16:
                return x.view(torch.int16).numpy().view(np.uint16), BF16
            if x.dtype == torch.float8_e4m3fn:
                return x.view(torch.uint8).numpy(), FP8
            if x.dtype == torch.float32:
                return x.numpy(), F32
            raise TypeError(f"unsupported dtype {x.dtype}")
    except ImportError:  # pragma: no cover
        pass
    x = np.ascontiguousarray(x)
    if x.dtype == np.uint16:
        return x, BF16
    if x.dtype == np.uint8:
        return x, FP8
    if x.dtype == np.float32:
        return x, F32
    raise TypeError(f"unsupported dtype {x.dtype}")


def _p(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def to_f32(x) -> np.ndarray:
    a, dt = _raw(x)
    out = np.empty(a.shape, dtype=np.float32)
    lib().oracle_to_f32(dt, _p(a), a.size, _p(out))
    return out


def slice_meta(k_slice, d: int, bs: int, nblk: int):
    """Metadata of full blocks [0,nblk) of one [cap][d] slice -> mu [nblk][d], var [nblk][d], maxn [nblk]."""
    a, dt = _raw(k_slice)
    mu = np.zeros((nblk, d), np.float32)
    var = np.zeros((nblk, d), np.float32)
    mx = np.zeros((nblk,), np.float32)
    if nblk > 0:
        lib().oracle_slice_meta(dt, _p(a), d, bs, nblk, _p(mu), _p(var), _p(mx))
    return mu, var, mx


def block_meta(k_block):
    """Metadata of one block given as [rows][d]."""
    a, dt = _raw(k_block)
    rows, d = a.shape
    mu = np.zeros((d,), np.float32)
    var = np.zeros((d,), np.float32)
    mx = np.zeros((1,), np.float32)
    lib().oracle_block_meta(dt, _p(a), 0, rows, d, _p(mu), _p(var), _p(mx))
    return mu, var, float(mx[0])


def meta(K, n: int, bs: int):
    """Metadata for every (b, kv head) of a [B][Hkv][cap][d] cache: full blocks only.
    Returns mu, var [B][Hkv][nf][d] and maxn [B][Hkv][nf], nf = n // bs."""
    a, dt = _raw(K)
    B, H, cap, d = a.shape
    nf = n // bs
    mu = np.zeros((B, H, nf, d), np.float32)
    var = np.zeros((B, H, nf, d), np.float32)
    mx = np.zeros((B, H, nf), np.float32)
    for b in range(B):
        for h in range(H):
            if nf:
                sl = np.ascontiguousarray(a[b, h])
                m_, v_, x_ = mu[b, h], var[b, h], mx[b, h]
                lib().oracle_slice_meta(dt, _p(sl), d, bs, nf, _p(m_), _p(v_), _p(x_))
    return mu, var, mx


def predict_tau(q, W: np.ndarray, bias: np.ndarray) -> np.ndarray:
    """tau [B][Hq] from q [B][Hq][d] (Eq. 1)."""
    qf = to_f32(q)
    B, H, d = qf.shape
    W = np.ascontiguousarray(W, dtype=np.float32)
    bias = np.ascontiguousarray(bias, dtype=np.float32)
    assert W.shape == (H * d, H) and bias.shape == (H,)
    tau = np.zeros((B, H), np.float32)
    for b in range(B):
        qb = np.ascontiguousarray(qf[b].reshape(-1))
        tb = tau[b]
        lib().oracle_predict_tau(_p(qb), H * d, H, _p(W), _p(bias), _p(tb))
    return tau


def block_score(q_f32: np.ndarray, mu, var, maxn: float, z: float) -> float:
    q_f32 = np.ascontiguousarray(q_f32, np.float32)
    d = q_f32.shape[0]
    mu = np.ascontiguousarray(mu, np.float32)
    var = np.ascontiguousarray(var, np.float32)
    return float(lib().oracle_block_score(_p(q_f32), d, _p(mu), _p(var), float(maxn), float(z),
                                          float(lib().oracle_inv_sqrt_d(d))))


def screen_head(q_f32, mu, var, maxn, nb: int, n_local: int, z: float, tau: float,
                offset_a: float = 0.0):
    """Admitted ascending block list of one head, and the scores of its screened blocks."""
    q_f32 = np.ascontiguousarray(q_f32, np.float32)
    d = q_f32.shape[0]
    mu = np.ascontiguousarray(mu, np.float32)
    var = np.ascontiguousarray(var, np.float32)
    maxn = np.ascontiguousarray(maxn, np.float32)
    ns = max(0, nb - n_local)
    assert mu.shape[0] >= ns
    lst = np.zeros((max(nb, 1),), np.int32)
    sc = np.zeros((max(ns, 1),), np.float32)
    cnt = lib().oracle_screen_head(_p(q_f32), d, _p(mu), _p(var), _p(maxn), nb, n_local,
                                   float(z), float(tau), float(offset_a), _p(lst), _p(sc))
    return lst[:cnt].copy(), sc[:ns].copy()


def screen_head_env(q_f32, mu, var, maxn, nb: int, r: int, n_local: int, z: float, tau: float,
                    offset_a: float = 0.0):
    """Sub-block envelope screen of one head (a labelled reading of the pages'
    undefined "sub-block envelope"): mu, var [>= ns*r][d] and maxn [>= ns*r] are
    the metadata of sub-blocks of b/r tokens; a block's score is the largest of
    its r sub-block scores (Eq. 5 on each). Returns the admitted ascending block
    list and the envelope scores of the screened blocks."""
    q_f32 = np.ascontiguousarray(q_f32, np.float32)
    d = q_f32.shape[0]
    mu = np.ascontiguousarray(mu, np.float32)
    var = np.ascontiguousarray(var, np.float32)
    maxn = np.ascontiguousarray(maxn, np.float32)
    ns = max(0, nb - n_local)
    assert mu.shape[0] >= ns * r and maxn.shape[0] >= ns * r
    lst = np.zeros((max(nb, 1),), np.int32)
    sc = np.zeros((max(ns, 1),), np.float32)
    cnt = lib().oracle_screen_head_env(_p(q_f32), d, _p(mu), _p(var), _p(maxn), nb, int(r), n_local,
                                       float(z), float(tau), float(offset_a), _p(lst), _p(sc))
    return lst[:cnt].copy(), sc[:ns].copy()


GATE_SIGMOID, GATE_HARD = 0, 1


def attend_head(k_slice, v_slice, bs: int, n: int, q_f32, blocks, tau: float,
                beta: float, gate: int = GATE_SIGMOID) -> np.ndarray:
    """Gated softmax attention of one head over the listed blocks -> [d] float64.
    gate GATE_SIGMOID: Eq. 2-3 (multiplicative gate, the pages' normal mode);
    GATE_HARD: keys below tau removed (strict mode, Tables 6-7); the current
    token is exempt in both."""
    ka, dt = _raw(k_slice)
    va, dt2 = _raw(v_slice)
    assert dt == dt2
    q_f32 = np.ascontiguousarray(q_f32, np.float32)
    d = q_f32.shape[0]
    blocks = np.ascontiguousarray(blocks, np.int32)
    out = np.zeros((d,), np.float64)
    lib().oracle_attend_head(dt, _p(ka), _p(va), d, bs, n, _p(q_f32), _p(blocks),
                             int(blocks.size), float(tau), float(beta), int(gate), _p(out))
    return out


def block_stats(k_slice, bs: int, n: int, q_f32, tau_screen: float, tau: float, beta: float,
                gate: int = GATE_SIGMOID):
    """Per block of one head's cache slice: (max scaled logit [nb] fp32, tokens
    with S >= tau_screen [nb] int32, log-sum-exp of the gated logits [nb] f64)."""
    ka, dt = _raw(k_slice)
    q_f32 = np.ascontiguousarray(q_f32, np.float32)
    d = q_f32.shape[0]
    nb = (n + bs - 1) // bs
    bmax = np.zeros((nb,), np.float32)
    above = np.zeros((nb,), np.int32)
    blse = np.zeros((nb,), np.float64)
    lib().oracle_block_stats(dt, _p(ka), d, bs, n, nb, _p(q_f32), float(tau_screen), float(tau), float(beta),
                             int(gate), _p(bmax), _p(above), _p(blse))
    return bmax, above, blse


def screen_diagnostics(bmax, above, blse, admitted, ns: int, tau_screen: float) -> dict:
    """Table 16's screen quality for one head, over its ns screened blocks:
    a block is truly active when its max logit reaches tau_screen;
    false_negative = truly active blocks rejected / truly active blocks;
    false_positive = admitted blocks not truly active / admitted blocks;
    token_recall   = tokens with S >= tau_screen inside admitted blocks / all such tokens;
    missed_mass    = dense gated softmax mass of the rejected blocks (all nb blocks
                     in the normaliser)."""
    adm = np.zeros((len(bmax),), bool)
    adm[np.asarray(admitted, np.int64)] = True
    scr = np.arange(len(bmax)) < ns
    active = bmax >= np.float32(tau_screen)
    a_s, adm_s = active & scr, adm & scr
    lse_all = np.logaddexp.reduce(blse)
    rejected = scr & ~adm
    return {
        "truly_active": int(a_s.sum()), "admitted": int(adm_s.sum()),
        "false_negative": float((a_s & ~adm_s).sum() / max(1, a_s.sum())),
        "false_positive": float((adm_s & ~a_s).sum() / max(1, adm_s.sum())),
        "token_recall": float(above[scr & adm].sum() / max(1, above[scr].sum())),
        "missed_mass": float(np.exp(np.logaddexp.reduce(blse[rejected]) - lse_all)) if rejected.any() else 0.0,
    }


def union_lists(lists_by_head, nb: int):
    """GQA union for one (b, kv head): ascending blocks admitted by any head of the
    group, with a bit mask (bit g = head g of the group admitted it)."""
    mask = np.zeros((nb,), np.uint32)
    for g, lst in enumerate(lists_by_head):
        mask[np.asarray(lst, np.int64)] |= np.uint32(1 << g)
    idx = np.nonzero(mask)[0].astype(np.int32)
    return idx, mask[idx]


def decode(q, K, V, n: int, bs: int, tau: np.ndarray, *, z: float, beta: float = 5.0,
           n_local: int = 1, offset_a: float = 0.0, meta_arrays=None, dense: bool = False,
           heads: Optional[list] = None):
    """The whole decode step for a [B][Hq][d] query batch against [B][Hkv][cap][d] caches.

    tau : [B][Hq] fp32 thresholds (the gate uses tau, the screen tau - offset_a).
    dense : admit every block (no screen).
    heads : optional list of (b, hq) pairs to compute; default all.
    Returns a dict: lists[(b,hq)], scores[(b,hq)], union[(b,kvh)] = (idx, mask), out[(b,hq)].
    """
    qf = to_f32(q)
    B, Hq, d = qf.shape
    Hkv = K.shape[1]
    G = Hq // Hkv
    nb = (n + bs - 1) // bs
    if meta_arrays is None and not dense:
        meta_arrays = meta(K, n, bs)
    sel = heads if heads is not None else [(b, h) for b in range(B) for h in range(Hq)]
    res = {"lists": {}, "scores": {}, "union": {}, "out": {}}
    for (b, h) in sel:
        kvh = h // G
        if dense:
            lst = np.arange(nb, dtype=np.int32)
            sc = None
        else:
            mu, var, mx = meta_arrays
            lst, sc = screen_head(qf[b, h], mu[b, kvh], var[b, kvh], mx[b, kvh], nb, n_local, z,
                                  float(tau[b, h]), offset_a)
        res["lists"][(b, h)] = lst
        res["scores"][(b, h)] = sc
    for (b, h) in sel:
        kvh = h // G
        ks = K[b, kvh]
        vs = V[b, kvh]
        res["out"][(b, h)] = attend_head(ks, vs, bs, n, qf[b, h], res["lists"][(b, h)],
                                         float(tau[b, h]), beta)
    kv_pairs = sorted({(b, h // G) for (b, h) in sel})
    for (b, kvh) in kv_pairs:
        heads_g = [res["lists"].get((b, kvh * G + g), np.zeros(0, np.int32)) for g in range(G)]
        res["union"][(b, kvh)] = union_lists(heads_g, nb)
    return res

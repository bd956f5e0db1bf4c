"""A synthetic decode workload materialised on the GPU.

Generates q, K, V on the host with the seeded generator (batch slices through
a pinned staging buffer, so the host never holds the whole cache), uploads
them, builds the block metadata with ``eta_build_block_meta`` and can
calibrate thresholds to a target density from the library's own block scores
(``eta_screen`` with score output), as an offline calibration would.
"""
from __future__ import annotations

import math
from typing import Optional

import torch

from . import binding, synth


class DeviceWorkload:
    def __init__(self, w: synth.Workload, device="cuda", n_splits: int = 0, offset_a: float = 0.0,
                 keep_host: bool = False, stage_bytes: int = 1 << 30, gate: int = binding.GATE_SIGMOID,
                 sub_blocks: int = 1):
        self.w = w
        self.device = torch.device(device)
        self.q_host = synth.make_q(w)
        self.q = self.q_host.to(self.device)
        self.needles = synth.make_needles(w)
        shp = (w.B, w.Hkv, w.capacity, w.d)
        self.K = torch.empty(shp, dtype=w.torch_dtype, device=self.device)
        self.V = torch.empty(shp, dtype=w.torch_dtype, device=self.device)
        per_b = w.Hkv * w.capacity * w.d * {"f32": 4, "bf16": 2, "fp8": 1}[w.dtype]
        bchunk = max(1, min(w.B, stage_bytes // max(1, per_b)))
        self.K_host = self.V_host = None
        if keep_host:
            self.K_host, self.V_host = synth.make_kv(w, self.q_host)
            self.K.copy_(self.K_host)
            self.V.copy_(self.V_host)
        else:
            stage = torch.empty((bchunk,) + shp[1:], dtype=w.torch_dtype).pin_memory()
            for which, dst in (("k", self.K), ("v", self.V)):
                for b0 in range(0, w.B, bchunk):
                    b1 = min(w.B, b0 + bchunk)
                    buf = stage[:b1 - b0]
                    synth.fill_kv(w, self.q_host, which, buf, b0, b1, self.needles)
                    dst[b0:b1].copy_(buf, non_blocking=True)
                    torch.cuda.current_stream(self.device).synchronize()
            del stage
        self.dec = binding.EtaDecoder(w.B, w.Hq, w.Hkv, w.d, w.bs, w.capacity, kv_dtype=w.torch_dtype,
                                      q_dtype=w.q_torch_dtype, beta=w.beta, z=w.z, offset_a=offset_a,
                                      n_local=w.n_local, n_splits=n_splits, device=self.device, gate=gate,
                                      sub_blocks=sub_blocks)
        self.dec.build_meta(self.K, 0, w.n // w.bs)
        self.W = self.bias0 = None
        if w.tau_mode == "predictor":
            W, b0 = synth.make_predictor(w)
            self.W, self.bias0 = W.to(self.device), b0.to(self.device)

    # ------------------------------------------------------------ calibration
    def block_scores(self) -> torch.Tensor:
        """Eq. 5 scores of every screened block, [B][Hq][n_screened] (fp32)."""
        w = self.w
        nb_cap = w.capacity // w.bs
        scores = torch.full((w.B, w.Hq, nb_cap), float("nan"), dtype=torch.float32, device=self.device)
        tau = torch.full((w.Hq,), float("-inf"), dtype=torch.float32, device=self.device)
        binding.screen(self.dec.shape, self.dec.params, self.q, self.dec.meta, w.n, tau, 0, self.dec.ws,
                       scores=scores)
        return scores[:, :, :w.n_screened]

    @staticmethod
    def _kth_of_sorted(s: torch.Tensor, density: float) -> torch.Tensor:
        """Per row of descending-sorted scores: the round(density*m)-th largest
        (at least the first); -inf for density >= 1."""
        m = s.shape[-1]
        if density >= 1.0 or m == 0:
            return torch.full(s.shape[:-1], float("-inf"), dtype=torch.float32, device=s.device)
        k = max(1, int(round(density * m)))
        return s[..., k - 1].contiguous()

    def _union_density(self, sc: torch.Tensor, thr: torch.Tensor) -> float:
        """Fraction of screened blocks in the GQA union when head h admits the
        blocks with score >= thr[b][h]."""
        w = self.w
        adm = sc >= thr[:, :, None]
        return adm.view(w.B, w.Hkv, w.G, -1).any(dim=2).float().mean().item()

    def calibrate(self, density: float):
        """Thresholds admitting about `density` of the screened blocks: of each
        head's blocks pooled over the batch, or (density_kind "union") of the
        GQA unions, by bisection on a common per-head density.
        Per-head constants: (tau [Hq], stride 0). Predictor: returns
        (None, None, bias) with the bias shifted so that score >= q.W + bias
        holds for that fraction; the caller runs the predictor."""
        w = self.w
        sc = self.block_scores()
        if w.tau_mode == "const":
            pooled = sc.transpose(0, 1).reshape(w.Hq, -1).sort(dim=-1, descending=True).values

            def thr_of(rho):
                return self._kth_of_sorted(pooled, rho)

            def full(t):
                return t[None, :].expand(w.B, w.Hq)
        else:
            tau0 = torch.empty((w.B, w.Hq), dtype=torch.float32, device=self.device)
            binding.predict_tau(self.dec.shape, self.q, self.W, self.bias0, tau0)
            # bias_h: the threshold, relative to each row's predicted tau, that admits
            # the target fraction of the head's screened blocks pooled over the batch
            shifted = (sc - tau0[:, :, None]).transpose(0, 1).reshape(w.Hq, -1).sort(dim=-1, descending=True).values

            def thr_of(rho):
                return self._kth_of_sorted(shifted, rho)

            def full(bias):
                return tau0 + bias[None, :]   # the predictor's fl(partial sum + bias)
        rho = density
        if w.density_kind == "union" and 0.0 < density < 1.0:
            lo, hi = 0.0, density             # a head's density never exceeds its union's
            for _ in range(24):
                mid = 0.5 * (lo + hi)
                if self._union_density(sc, full(thr_of(mid))) < density:
                    lo = mid
                else:
                    hi = mid
            rho = hi
        t = thr_of(rho)
        return (t, 0, None) if w.tau_mode == "const" else (None, None, t)

    # ------------------------------------------------------------- one step
    def step(self, tau=None, stride=None, bias=None, out=None, **outs) -> torch.Tensor:
        w = self.w
        if bias is not None:
            return self.dec.step(self.q, self.K, self.V, w.n, W=self.W, bias=bias, out=out, **outs)
        return self.dec.step(self.q, self.K, self.V, w.n, tau=tau, tau_batch_stride=stride, out=out, **outs)

    def dense(self, out=None) -> torch.Tensor:
        return self.dec.dense(self.q, self.K, self.V, self.w.n, out=out)

"""Screen diagnostics of the pages' Table 16 on the GPU: how well the O(1)
block screen predicts the blocks that matter.

Three library calls: ``eta_block_stats`` (a dense pass over K: every block's
max scaled logit, tokens at or above tau - a, gated log-sum-exp),
``eta_screen`` (the admitted lists) and ``eta_screen_diagnostics``, which
forms per query head, over its screened blocks (the forced trailing blocks
excluded), with a block *truly active* when its max reaches tau - a:

* false_negative = truly active blocks the screen rejected / truly active blocks
* false_positive = admitted blocks that are not truly active / admitted blocks
* token_recall   = tokens with S >= tau - a inside admitted blocks / all such tokens
* missed_mass    = gated softmax mass (Eq. 2-3, dense over every block) of the
                   rejected blocks

This module only marshals the buffers and reports the mean over heads.
Diagnostics only: not on the decode path.
"""
from __future__ import annotations

import torch

from . import binding

KEYS = ("false_negative", "false_positive", "token_recall", "missed_mass")


def screen_diagnostics(dec: "binding.EtaDecoder", q: torch.Tensor, k: torch.Tensor, n_tokens: int,
                       tau: torch.Tensor, tau_batch_stride: int) -> dict:
    shape = dec.shape
    B, Hq, bs = shape.batch, shape.n_q_heads, shape.block_size
    nb_cap = shape.capacity // bs
    dev = q.device
    bmax = torch.full((B, Hq, nb_cap), float("-inf"), dtype=torch.float32, device=dev)
    above = torch.zeros((B, Hq, nb_cap), dtype=torch.int32, device=dev)
    blse = torch.full((B, Hq, nb_cap), float("-inf"), dtype=torch.float32, device=dev)
    binding.block_stats(shape, dec.params, q, k, n_tokens, tau, tau_batch_stride, bmax, above, blse)
    idx = torch.full((B, Hq, nb_cap), -1, dtype=torch.int32, device=dev)
    cnt = torch.zeros((B, Hq), dtype=torch.int32, device=dev)
    binding.screen(shape, dec.params, q, dec.meta, n_tokens, tau, tau_batch_stride, dec.ws, active_idx=idx,
                   active_cnt=cnt)
    per = torch.empty((B, Hq, 4), dtype=torch.float64, device=dev)
    binding.screen_diagnostics(shape, dec.params, n_tokens, tau, tau_batch_stride, bmax, above, blse, idx, cnt, per)
    out = {key: per[:, :, i].mean().item() for i, key in enumerate(KEYS)}
    out["per_head"] = {key: per[:, :, i] for i, key in enumerate(KEYS)}
    return out

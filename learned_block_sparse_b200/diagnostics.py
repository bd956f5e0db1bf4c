"""Screen diagnostics of the pages' Table 16 on the GPU: how well the O(1)
block screen predicts the blocks that matter, from ``eta_block_stats`` (a dense
pass over K) and the admitted lists of ``eta_screen``.

Per query head, over its screened blocks (the forced trailing blocks excluded):
a block is *truly active* when its maximum scaled logit reaches tau - a;

* false_negative = truly active blocks the screen rejected / truly active blocks
* false_positive = admitted blocks that are not truly active / admitted blocks
* token_recall   = tokens with S >= tau - a inside admitted blocks / all such tokens
* missed_mass    = gated softmax mass (Eq. 2-3, dense over every block) of the
                   rejected blocks

Aggregates are means over heads. Diagnostics only: not on the decode path.
"""
from __future__ import annotations

import torch

from . import binding


def screen_diagnostics(dec: "binding.EtaDecoder", q: torch.Tensor, k: torch.Tensor, n_tokens: int,
                       tau: torch.Tensor, tau_batch_stride: int) -> dict:
    shape = dec.shape
    B, Hq, bs = shape.batch, shape.n_q_heads, shape.block_size
    nb_cap = shape.capacity // bs
    nb = (n_tokens + bs - 1) // bs
    ns = max(0, nb - dec.params.n_local)
    dev = q.device
    bmax = torch.full((B, Hq, nb_cap), float("-inf"), dtype=torch.float32, device=dev)
    above = torch.zeros((B, Hq, nb_cap), dtype=torch.int32, device=dev)
    blse = torch.full((B, Hq, nb_cap), float("-inf"), dtype=torch.float32, device=dev)
    binding.block_stats(shape, dec.params, q, k, n_tokens, tau, tau_batch_stride, bmax, above, blse)
    idx = torch.full((B, Hq, nb_cap), -1, dtype=torch.int32, device=dev)
    cnt = torch.zeros((B, Hq), dtype=torch.int32, device=dev)
    binding.screen(shape, dec.params, q, dec.meta, n_tokens, tau, tau_batch_stride, dec.ws, active_idx=idx,
                   active_cnt=cnt)
    # admitted mask [B][Hq][nb] from the compacted lists
    pos = torch.arange(nb_cap, device=dev)[None, None, :]
    valid = pos < cnt[:, :, None].long()
    adm = torch.zeros((B, Hq, nb_cap + 1), dtype=torch.bool, device=dev)
    adm.scatter_(2, torch.where(valid, idx.long(), torch.full_like(idx.long(), nb_cap)), True)
    adm = adm[:, :, :nb]
    if tau_batch_stride == 0:
        taus = (tau.float() - dec.params.offset_a)[None, :].expand(B, Hq)
    else:
        taus = tau.float().view(B, Hq) - dec.params.offset_a
    scr = (torch.arange(nb, device=dev) < ns)[None, None, :]
    bm, ab, ls = bmax[:, :, :nb], above[:, :, :nb], blse[:, :, :nb].double()
    active = (bm >= taus[:, :, None]) & scr
    admitted = adm & scr
    n_act = active.sum(-1).clamp(min=1).double()
    n_adm = admitted.sum(-1).clamp(min=1).double()
    fn = (active & ~admitted).sum(-1).double() / n_act
    fp = (admitted & ~active).sum(-1).double() / n_adm
    tok_all = (ab * scr).sum(-1).clamp(min=1).double()
    recall = (ab * admitted).sum(-1).double() / tok_all
    lse_all = torch.logsumexp(ls, -1)
    rej = scr & ~adm
    missed = torch.exp(torch.logsumexp(ls.masked_fill(~rej, float("-inf")), -1) - lse_all)
    return {"false_negative": fn.mean().item(), "false_positive": fp.mean().item(),
            "token_recall": recall.mean().item(), "missed_mass": missed.mean().item(),
            "per_head": {"false_negative": fn, "false_positive": fp, "token_recall": recall,
                         "missed_mass": missed}}

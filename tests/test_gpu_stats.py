"""Block statistics (eta_block_stats) and the Table 16 screen diagnostics on the
GPU against the oracle: block maxima and above-threshold counts bit-exact, the
gated block log-sum-exps within fp32 rounding, and the diagnostics (false
negatives, false positives, token recall, missed mass) per head."""
import numpy as np
import pytest
import torch

import oracle
from learned_block_sparse_b200 import binding, diagnostics, synth
from learned_block_sparse_b200.workload import DeviceWorkload
from tests import parity

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("dtype,Hq,Hkv,d,bs,gate", [
    ("bf16", 8, 2, 128, 32, binding.GATE_SIGMOID),
    ("bf16", 8, 1, 64, 64, binding.GATE_SIGMOID),
    ("f32", 4, 4, 64, 16, binding.GATE_HARD),
    ("fp8", 8, 2, 128, 32, binding.GATE_SIGMOID),
])
def test_block_stats_and_diagnostics_match_oracle(dtype, Hq, Hkv, d, bs, gate):
    w = synth.Workload("stats", dtype, 2, Hq, Hkv, d, bs * 45 + 11, bs, z=1.0, tau_mode="const",
                       densities=(0.3,), seed=1200 + bs + d, offset_std=synth.SQRT_HALF)
    dw = DeviceWorkload(w, keep_host=True, gate=gate)
    meta = parity.oracle_meta(w, dw.K_host)
    tau, _, _ = parity.oracle_thresholds(w, dw.q_host, meta, 0.3)
    tau_dev = torch.as_tensor(tau, device="cuda")
    nb_cap = w.capacity // w.bs
    bmax = torch.full((w.B, w.Hq, nb_cap), float("nan"), device="cuda")
    above = torch.full((w.B, w.Hq, nb_cap), -1, dtype=torch.int32, device="cuda")
    blse = torch.full((w.B, w.Hq, nb_cap), float("nan"), device="cuda")
    binding.block_stats(dw.dec.shape, dw.dec.params, dw.q, dw.K, w.n, tau_dev, 0, bmax, above, blse)
    got = diagnostics.screen_diagnostics(dw.dec, dw.q, dw.K, w.n, tau_dev, 0)
    torch.cuda.synchronize()
    assert dw.dec.device_status() == 0
    bmax, above, blse = bmax.cpu().numpy(), above.cpu().numpy(), blse.cpu().numpy()
    qf = oracle.to_f32(dw.q_host)
    per = got["per_head"]
    for b in range(w.B):
        for h in range(w.Hq):
            kvh = h // w.G
            t = float(tau[h])
            ts = float(np.float32(np.float32(t) - np.float32(0.0)))
            om, oa, ol = oracle.block_stats(dw.K_host[b, kvh], w.bs, w.n, qf[b, h], ts, t, w.beta, gate)
            nb = len(om)
            assert np.array_equal(bmax[b, h, :nb].view(np.int32), om.view(np.int32)), (b, h)
            assert np.array_equal(above[b, h, :nb], oa), (b, h)
            assert np.allclose(blse[b, h, :nb], ol, rtol=2e-6, atol=2e-5), (b, h)
            mu, var, mx = meta[(b, kvh)]
            lst, _ = oracle.screen_head(qf[b, h], mu, var, mx, nb, w.n_local, w.z, t)
            o = oracle.screen_diagnostics(om, oa, ol, lst, w.n_screened, ts)
            assert per["false_negative"][b, h].item() == pytest.approx(o["false_negative"], abs=1e-12)
            assert per["false_positive"][b, h].item() == pytest.approx(o["false_positive"], abs=1e-12)
            assert per["token_recall"][b, h].item() == pytest.approx(o["token_recall"], abs=1e-12)
            assert per["missed_mass"][b, h].item() == pytest.approx(o["missed_mass"], rel=1e-4, abs=1e-7)

"""Device-side failure detection: a bounded wait that runs out.

Every wait of the pipelined kernels is bounded (2 s). When one runs out, the
thread block stops arming copies, lets the copies in flight land, completes
its control flow and records ETA_ERR_DEVICE_TIMEOUT in the workspace status
word. The test makes one wait run out through the library's test hook (the
copy of one admitted block is never issued, so nothing completes its barrier:
a flag that nothing sets), then checks the status word, that reading it
cleared the workspace header, and that the next call on the same workspace
gives the oracle's result. Nothing faults; the context stays usable."""
import time

import pytest
import torch

from learned_block_sparse_b200 import binding, synth
from learned_block_sparse_b200.workload import DeviceWorkload
from tests import parity

pytestmark = pytest.mark.gpu

WORKLOADS = {
    "bf16-gqa": synth.WORKLOADS[3].replace(B=2, Hq=8, Hkv=2, n=32 * 150 + 5),   # tensor-core decode
    "f32-mha": synth.WORKLOADS[1],                                             # CUDA-core decode
}


@pytest.mark.parametrize("name,n_splits,dense", [("bf16-gqa", 4, False), ("f32-mha", 2, False),
                                                 ("bf16-gqa", 3, True)])
def test_withheld_copy_times_out_then_next_call_matches_oracle(name, n_splits, dense):
    w = WORKLOADS[name]
    dw = DeviceWorkload(w, n_splits=n_splits, keep_host=True)
    meta = parity.oracle_meta(w, dw.K_host)
    tau, stride, bias = parity.oracle_thresholds(w, dw.q_host, meta, w.densities[0], W=dw.W)
    heads = [(b, h) for b in range(w.B) for h in range(w.Hq)]
    try:
        binding.withhold_next_copy(1)         # the second block of the first thread block's range
        t0 = time.perf_counter()
        bad = parity.run_gpu(dw, None if dense else tau, 0 if dense else stride, bias=None if dense else bias,
                             dense=dense)
        waited = time.perf_counter() - t0
    finally:
        binding.withhold_next_copy(-1)
    assert bad["status"] == binding.ETA_ERR_DEVICE_TIMEOUT
    assert 1.5 < waited < 60.0
    # reading the status cleared the whole header: status word and split counters
    header = dw.dec.ws[:256 + 4 * 8192].view(torch.int32)
    assert int(torch.count_nonzero(header)) == 0
    assert dw.dec.device_status() == 0
    # the next call on the same workspace is exact again
    good = parity.run_gpu(dw, None if dense else tau, 0 if dense else stride, bias=None if dense else bias,
                          dense=dense)
    assert good["status"] == 0
    orc = parity.oracle_step(w, dw.q_host, dw.K_host, dw.V_host, meta, None if dense else tau,
                             0 if dense else stride, heads, dense=dense)
    parity.compare(w, good, orc, heads, check_lists=not dense)


def test_withhold_hook_past_the_range_changes_nothing():
    w = WORKLOADS["bf16-gqa"]
    dw = DeviceWorkload(w, n_splits=4)
    tau = torch.zeros((w.B, w.Hq), device="cuda")
    a = dw.step(tau=tau, stride=w.Hq).clone()
    try:
        binding.withhold_next_copy(1 << 40)
        b = dw.step(tau=tau, stride=w.Hq).clone()
    finally:
        binding.withhold_next_copy(-1)
    torch.cuda.synchronize()
    assert dw.dec.device_status() == 0
    assert torch.equal(a, b)

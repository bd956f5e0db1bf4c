"""The allocation-free decode entry point (eta_decode_sparse_static).

Callers that cannot allocate device memory while decoding (graph capture,
frozen serving memory plans, host frameworks that own all allocations,
real-time loops) call this variant, which keeps its scratch in a fixed device
array inside the library. It must give the same result as eta_decode_sparse
with a caller workspace, call after call (the shared scratch keeps the
previous call's contents), and reject shapes larger than its scratch.

This file is collected last on purpose, so a run that stops at the first
failure has already run every other test."""
import ctypes

import pytest
import torch

from learned_block_sparse_b200 import binding, synth
from learned_block_sparse_b200.workload import DeviceWorkload

pytestmark = pytest.mark.gpu

TOL_BF16 = 2e-3


def _thresholds(dw, density):
    tau, stride, bias = dw.calibrate(density)
    if bias is not None:
        t = torch.empty((dw.w.B, dw.w.Hq), dtype=torch.float32, device=dw.device)
        binding.predict_tau(dw.dec.shape, dw.q, dw.W, bias, t)
        return t, dw.w.Hq
    return tau, stride


def test_static_scratch_matches_workspace_entry_point_on_consecutive_calls():
    w = synth.WORKLOADS[3].replace(B=2, Hq=8, Hkv=2, n=32 * 150 + 5)
    dw = DeviceWorkload(w)
    dec = dw.dec
    assert binding.workspace_bytes(dec.shape, dec.params) <= binding.STATIC_SCRATCH_BYTES
    for density in (0.38, 0.2):              # two calls in a row, different admitted sets
        tau, stride = _thresholds(dw, density)
        ref = torch.empty((w.B, w.Hq, w.d), dtype=torch.float32, device=dw.device)
        binding.decode_sparse(dec.shape, dec.params, dw.q, dw.K, dw.V, dec.meta, w.n, tau, stride, ref, dec.ws)
        out = torch.full_like(ref, float("nan"))
        status = torch.full((1,), -1, dtype=torch.int32, device=dw.device)
        cnt = torch.full((w.B, w.Hq), -1, dtype=torch.int32, device=dw.device)
        binding.decode_sparse_static(dec.shape, dec.params, dw.q, dw.K, dw.V, dec.meta, w.n, tau, stride, out,
                                     device_status=status, active_cnt=cnt)
        torch.cuda.synchronize()
        assert int(status.item()) == 0
        assert torch.isfinite(out).all()
        assert float((out - ref).abs().max()) <= TOL_BF16
        assert int(cnt.min()) >= 1


def test_static_scratch_rejects_shapes_beyond_its_size():
    # 64 batch rows x 16 kv heads x 64K tokens in blocks of 16: lists and partials exceed the scratch
    shape = binding.make_shape(64, 16, 16, 128, 16, 65536, torch.bfloat16, torch.bfloat16)
    params = binding.make_params()
    assert binding.workspace_bytes(shape, params) > binding.STATIC_SCRATCH_BYTES
    dummy = ctypes.c_void_p(1 << 20)
    meta = binding.Meta(1 << 20, 1 << 20, 1 << 20)
    rc = binding.lib.eta_decode_sparse_static(ctypes.byref(shape), ctypes.byref(params), dummy, dummy, dummy, meta,
                                              1000, dummy, 0, dummy, None, None, None)
    assert rc == binding.ETA_ERR_WORKSPACE

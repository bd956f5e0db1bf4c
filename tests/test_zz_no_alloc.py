"""The allocation-free decode entry point (eta_decode_sparse_static).

Some callers cannot allocate device memory while they decode: a serving engine
whose memory plan is fixed at start-up, a host framework that owns every
allocation, a real-time loop that must not enter an allocator. They call this
variant, which keeps its scratch in a fixed device array inside the library.
It runs the same kernels as eta_decode_sparse with a caller workspace, so on
the same inputs its outputs, counts and lists must be identical bit for bit,
call after call (the shared scratch keeps the previous call's contents), and
it must reject shapes larger than its scratch.

This file is collected last on purpose, so a run that stops at the first
failure has already run every other test."""
import ctypes

import pytest
import torch

from learned_block_sparse_b200 import binding, synth
from learned_block_sparse_b200.workload import DeviceWorkload

pytestmark = pytest.mark.gpu


def _thresholds(dw, density):
    tau, stride, bias = dw.calibrate(density)
    if bias is not None:
        t = torch.empty((dw.w.B, dw.w.Hq), dtype=torch.float32, device=dw.device)
        binding.predict_tau(dw.dec.shape, dw.q, dw.W, bias, t)
        return t, dw.w.Hq
    return tau, stride


def _lists(w, dev):
    nb_cap = w.capacity // w.bs
    return dict(active_idx=torch.full((w.B, w.Hq, nb_cap), -1, dtype=torch.int32, device=dev),
                active_cnt=torch.full((w.B, w.Hq), -1, dtype=torch.int32, device=dev),
                union_list=torch.zeros((w.B, w.Hkv, nb_cap), dtype=torch.int32, device=dev),
                union_cnt=torch.full((w.B, w.Hkv), -1, dtype=torch.int32, device=dev))


def test_static_scratch_matches_workspace_entry_point_on_consecutive_calls():
    w = synth.WORKLOADS[3].replace(B=2, Hq=8, Hkv=2, n=32 * 150 + 5)
    dw = DeviceWorkload(w)
    dec = dw.dec
    assert binding.workspace_bytes(dec.shape, dec.params) <= binding.STATIC_SCRATCH_BYTES
    for density in (0.38, 0.2):              # two calls in a row, different admitted sets
        tau, stride = _thresholds(dw, density)
        ref = torch.empty((w.B, w.Hq, w.d), dtype=torch.float32, device=dw.device)
        ref_lists = _lists(w, dw.device)
        binding.decode_sparse(dec.shape, dec.params, dw.q, dw.K, dw.V, dec.meta, w.n, tau, stride, ref, dec.ws,
                              **ref_lists)
        out = torch.full_like(ref, float("nan"))
        got_lists = _lists(w, dw.device)
        status = torch.full((1,), -1, dtype=torch.int32, device=dw.device)
        binding.decode_sparse_static(dec.shape, dec.params, dw.q, dw.K, dw.V, dec.meta, w.n, tau, stride, out,
                                     device_status=status, **got_lists)
        torch.cuda.synchronize()
        assert dec.device_status() == 0
        assert int(status.item()) == 0
        # same kernels, same inputs: the same bits
        assert torch.equal(out, ref)
        for key in ref_lists:
            assert torch.equal(got_lists[key], ref_lists[key]), key
        assert int(got_lists["active_cnt"].min()) >= 1


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

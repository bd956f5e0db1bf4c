#!/usr/bin/env python
"""Benchmark of one ETA block-sparse decode step on B200.

A step is the whole hot path for one batch of decode queries: threshold
predictor (Eq. 1) -> block screening against the cached metadata (Eq. 5) ->
block-sparse flash decoding with the sigmoid logit gate (Eq. 2-3), whose
split partials are merged inside the same kernel. Default workload: GQA decode, batch 8, 32 query / 8 KV heads,
d=128, 128K cached tokens, bf16 KV, block 32, predictor thresholds at ~38%
head density (the 128K-context configuration).

Prints one JSON line (rank 0): decode queries/s, effective HBM GB/s on the
bytes actually read, the decode kernel's roofline fraction, the speedup over
the same kernel run dense, end-to-end queries/s through the public API with
host buffers, and the CPU oracle's throughput on a bounded sample.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--config 3] [--density 0.38]
  python bench.py --impl reference ...   # the CPU oracle as the reference arm
"""
from __future__ import annotations

import argparse
import concurrent.futures as cf
import datetime
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

L2_FLUSH_BYTES = 512 << 20      # > 2x the 126 MB L2
LAUNCHES_PER_STEP = {"predictor": 2, "const": 2}


def parse_args():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=20)
    p.add_argument("--warmup", type=int, default=5)
    p.add_argument("--impl", default="eta", choices=["eta", "reference"])
    p.add_argument("--config", type=int, default=3)
    p.add_argument("--batch", type=int, default=None, help="override the batch (config 5 sweep)")
    p.add_argument("--seq-len", type=int, default=None, help="override the cached tokens per row")
    p.add_argument("--cap-blocks", type=int, default=None,
                   help="override the capacity per row, in blocks (not a multiple of 4: metadata rows that "
                        "are not 16-byte aligned, screened with plain loads)")
    p.add_argument("--density", type=float, default=None,
                   help="target admitted fraction (default: the middle density of the workload)")
    p.add_argument("--n-splits", type=int, default=0)
    p.add_argument("--sub-blocks", type=int, default=1, choices=[1, 2, 4, 8],
                   help="sub-block envelope: metadata per sub-block of b/r tokens, a block scored by its best one")
    p.add_argument("--no-cpu", action="store_true", help="skip the CPU oracle baseline")
    p.add_argument("--no-dense", action="store_true")
    p.add_argument("--no-e2e", action="store_true")
    p.add_argument("--no-sweep", action="store_true", help="skip the other densities of the configuration")
    p.add_argument("--no-diagnostics", action="store_true", help="skip the screen-quality pass (Table 16 metrics)")
    p.add_argument("--l2-flush", default="write+read", choices=["write", "write+read"],
                   help="between steps: write 512 MiB, or write then read 512 MiB so the timed step "
                        "does not also pay for writing back the flush's dirty lines")
    p.add_argument("--cpu-groups", type=int, default=64, help="(b, kv head) groups in the CPU sample")
    args = p.parse_args()
    if args.density is None:
        from learned_block_sparse_b200 import synth
        ds = synth.WORKLOADS[args.config].densities
        args.density = ds[len(ds) // 2]
    return args


# ----------------------------------------------------------------- plumbing
def workload_of(args):
    """The benchmark workload with the command line's overrides applied."""
    from learned_block_sparse_b200 import synth
    w = synth.WORKLOADS[args.config]
    if args.batch:
        w = w.replace(B=args.batch)
    if args.seq_len:
        w = w.replace(n=args.seq_len)
    if args.cap_blocks:
        w = w.replace(cap=args.cap_blocks * w.bs)
    return w


def relaunch_command(argv, n: int, port: int):
    """The torch.distributed.run command that starts n ranks of this script
    with the same arguments (one process per GPU, rendezvous on 127.0.0.1)."""
    return [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", f"--nproc-per-node={n}",
            "--master-addr=127.0.0.1", f"--master-port={port}", os.path.abspath(__file__), *argv]


def launch_ranks(args) -> int:
    """`bench.py --gpus N` (N > 1) started as a plain process: start the N ranks
    and return their launcher's exit status."""
    import socket
    with socket.socket() as sk:
        sk.bind(("127.0.0.1", 0))
        port = sk.getsockname()[1]
    return subprocess.call(relaunch_command(sys.argv[1:], args.gpus, port))


def dist_setup(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world != args.gpus:
        raise SystemExit(f"--gpus {args.gpus} but the launcher started {world} ranks")
    if world > 1:
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=torch.device("cuda", local))
    else:
        torch.cuda.set_device(0)
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x: float, world: int, device: str = "cuda") -> float:
    """Largest value over the ranks (device time of the slowest rank)."""
    if world == 1:
        return x
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(queries_per_rank: int, ms_max: float, world: int) -> float:
    """Whole-job queries/s: every rank decodes its own batch (weak scaling); the
    job takes as long as its slowest rank."""
    return world * queries_per_rank / (ms_max * 1e-3)


def decode_sources_digest() -> str:
    """sha256 over the sources that define the tensor-core decode kernel."""
    import hashlib
    h = hashlib.sha256()
    for f in ("decode_mma.cu", "decode_common.cuh", "common.cuh"):
        with open(os.path.join(ROOT, "learned_block_sparse_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()


def measured_traffic(workload_name: str, union_blocks: int):
    """DRAM bytes per decode launch from the committed ncu capture
    (profiles/decode_traffic.json), scaled by admitted union blocks; None when
    the capture is missing, is for another workload, or the kernel changed since."""
    path = os.path.join(ROOT, "profiles", "decode_traffic.json")
    try:
        with open(path) as f:
            d = json.load(f)
    except Exception:
        return None
    if d.get("source_sha256") != decode_sources_digest() or d.get("workload") != workload_name:
        return None
    return float(d["dram_bytes_per_union_block"]) * union_blocks


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    except Exception:
        return 6650.0, "fallback"


_SAMPLER = r"""
import sys, time
import pynvml
pynvml.nvmlInit()
h = pynvml.nvmlDeviceGetHandleByUUID(sys.argv[1])
mx = pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM)
rd = getattr(pynvml, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
    pynvml.nvmlDeviceGetCurrentClocksThrottleReasons
period = float(sys.argv[2])
with open(sys.argv[3], "w", buffering=1) as f:
    while True:
        f.write("%.6f %d %d %d\n" % (time.monotonic(), pynvml.nvmlDeviceGetClockInfo(h, pynvml.NVML_CLOCK_SM),
                                       mx, rd(h)))
        time.sleep(period)
"""


class ClockSampler:
    """SM clock and clock-event reasons sampled DURING the timed region.

    A separate process polls NVML every 0.2 ms (an NVML query takes ~1 us;
    the shortest timed regions, a few steps of the tiny workload, last about
    half a millisecond) and stamps each sample with the system-wide monotonic clock;
    start() returns once it is sampling, stop() keeps the samples taken between
    the two calls. A separate process, so the benchmark's own thread never
    delays the sampling. The device is found by its UUID (CUDA and NVML may
    number GPUs differently)."""
    REASONS = (("hw_slowdown", 0x8), ("hw_thermal_slowdown", 0x40), ("sw_thermal_slowdown", 0x20),
               ("sw_power_cap", 0x4), ("hw_power_brake_slowdown", 0x80))

    def __init__(self, device_index: int, period_s: float = 0.0002):
        self.dev = device_index
        self.period = period_s
        self.proc = None
        self.path = None
        self.t0 = self.t1 = None

    def start(self):
        try:
            uuid = "GPU-" + str(torch.cuda.get_device_properties(self.dev).uuid)
            fd, self.path = tempfile.mkstemp(suffix=".txt")
            os.close(fd)
            self.proc = subprocess.Popen([sys.executable, "-c", _SAMPLER, uuid, str(self.period), self.path],
                                         stderr=subprocess.DEVNULL)
            deadline = time.monotonic() + 20.0
            while time.monotonic() < deadline and self.proc.poll() is None:
                if os.path.getsize(self.path) > 0:
                    break
                time.sleep(0.01)
            if self.proc.poll() is not None or os.path.getsize(self.path) == 0:
                self.stop()
                self.proc = None
                return
        except Exception:
            self.proc = None
            return
        self.t0 = time.monotonic()

    def stop(self):
        if self.proc is None:
            return None
        self.t1 = time.monotonic()
        time.sleep(2 * self.period)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        samples = []
        with open(self.path) as f:
            for line in f:
                parts = line.split()
                if len(parts) != 4:
                    continue
                t, sm, mx, mask = float(parts[0]), int(parts[1]), int(parts[2]), int(parts[3])
                if self.t0 is not None and self.t0 <= t <= self.t1:
                    samples.append((sm, mx, mask))
        os.unlink(self.path)
        if not samples:
            return None
        reasons = sorted({nm for (_, _, m) in samples for nm, bit in self.REASONS if m & bit})
        sm = [x[0] for x in samples]
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(x[1] for x in samples), "sm_mhz_min": min(sm),
                "reasons": reasons, "samples": len(sm),
                "source": "NVML polled every 0.2 ms by a separate process, samples inside the timed region"}


# ------------------------------------------------------------ byte models
def byte_model(w, union_cnt: np.ndarray, head_cnt: np.ndarray, S: int, r: int = 1):
    """Algorithmic bytes of one step from the admitted counts.
    union_cnt [B][Hkv]; the last block of each list is partial when n % b != 0."""
    eb = {"f32": 4, "bf16": 2, "fp8": 1}[w.dtype]
    row = w.d * eb
    last_rows = w.n - (w.nb - 1) * w.bs
    blocks = int(union_cnt.sum())
    bh = w.B * w.Hkv
    kv = 2 * row * (blocks * w.bs - bh * (w.bs - last_rows))
    lists_read = 4 * blocks
    q = w.B * w.Hq * w.d * eb
    # the decode splits ring positions over its thread blocks: a block is one
    # position, or bs / 32 of them on the tensor-core path (bf16, fp8) at
    # d = 128 for blocks of 64 and 128 tokens
    nsub = max(1, w.bs // 32) if (w.dtype != "f32" and w.d == 128) else 1
    T = blocks * nsub
    # split merge: a segment inside one range writes its output rows directly;
    # one crossing ranges writes one (m, l, o) partial per range and head (read
    # back once by the merging thread block, from L2)
    pre = nsub * np.concatenate([[0], np.cumsum(union_cnt.reshape(-1))])
    partial_rows = 0
    for i in range(bh):
        if T >= S:
            parts = ((pre[i + 1]) * S - 1) // T - ((pre[i] + 1) * S - 1) // T + 1
        else:
            parts = pre[i + 1] - pre[i]
        if parts > 1:
            partial_rows += int(parts)
    partials = partial_rows * w.G * (w.d + 2) * 4
    out = w.B * w.Hq * w.d * 4
    decode = kv + lists_read + q + partials + out
    meta = bh * w.n_screened * r * (2 * w.d + 1) * 4   # r metadata columns per block with the envelope
    W = (w.Hq * w.d * w.Hq * 4 + w.Hq * 4) if w.tau_mode == "predictor" else 0
    step_read = kv + meta + lists_read + q * 2 + W
    dense_kv = 2 * row * bh * w.n
    return {"decode_kernel": decode, "step_read": step_read, "kv": kv, "meta": meta,
            "dense_kv": dense_kv, "union_blocks": blocks,
            "d_head": float(head_cnt.sum()) / (w.B * w.Hq * w.nb),
            "d_union": float(blocks) / (bh * w.nb)}


# -------------------------------------------------------------- CPU oracle
def oracle_screen(w, qf_h, meta, t, r):
    """The oracle screen of one head: Eq. 5 on whole blocks, or the sub-block envelope."""
    import oracle
    mu, var, mx = meta
    if r > 1:
        return oracle.screen_head_env(qf_h, mu, var, mx, w.nb, r, w.n_local, w.z, t)
    return oracle.screen_head(qf_h, mu, var, mx, w.nb, w.n_local, w.z, t)


def oracle_setup(w, dw_host, groups, r=1):
    """Oracle-side metadata and thresholds for the sampled (b, kv head) groups."""
    import oracle
    from learned_block_sparse_b200 import synth
    q_host, K_host, V_host = dw_host
    nf = (w.n // w.bs) * r
    pool = cf.ThreadPoolExecutor(max_workers=os.cpu_count() or 1)
    metas = dict(zip(groups, pool.map(lambda g: oracle.slice_meta(K_host[g[0], g[1]], w.d, w.bs // r, nf), groups)))
    qf = oracle.to_f32(q_host)
    heads = [(b, kvh * w.G + g) for (b, kvh) in groups for g in range(w.G)]

    def sc(bh):
        b, hq = bh
        return oracle_screen(w, qf[b, hq], metas[(b, hq // w.G)], float("-inf"), r)[1]
    scores = dict(zip(heads, pool.map(sc, heads)))
    return metas, qf, heads, scores, pool


def oracle_thresholds(w, q_host, W, scores, density):
    import oracle
    from learned_block_sparse_b200 import synth
    if w.tau_mode == "const":
        tau = np.zeros((w.Hq,), np.float32)
        for h in range(w.Hq):
            s = [scores[k] for k in scores if k[1] == h]
            tau[h] = synth.tau_for_density(np.concatenate(s), density) if s else 0.0
        return ("const", tau, None)
    tau0 = oracle.predict_tau(q_host, W, np.zeros(w.Hq, np.float32))
    bias = np.zeros((w.Hq,), np.float32)
    for h in range(w.Hq):
        rel = [scores[k].astype(np.float64) - tau0[k[0], h] for k in scores if k[1] == h]
        bias[h] = synth.tau_for_density(np.concatenate(rel), density) if rel else 0.0
    return ("predictor", None, bias)


def oracle_step(w, q_host, K_host, V_host, W, thr, metas, qf, heads, pool, r=1):
    """One oracle decode step over the sampled heads: predictor, screen, gated attention."""
    import oracle
    kind, tau_c, bias = thr
    tau = oracle.predict_tau(q_host, W, bias) if kind == "predictor" else None

    def one(bh):
        b, hq = bh
        kvh = hq // w.G
        t = float(tau[b, hq]) if tau is not None else float(tau_c[hq])
        lst, _ = oracle_screen(w, qf[b, hq], metas[(b, kvh)], t, r)
        return oracle.attend_head(K_host[b, kvh], V_host[b, kvh], w.bs, w.n, qf[b, hq], lst, t, w.beta)
    return list(pool.map(one, heads))


def run_reference(args):
    """The CPU oracle as the reference arm (rank 0 only; the other ranks join
    the CPU process group and exit without work)."""
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if world != args.gpus:
        raise SystemExit(f"--gpus {args.gpus} but the launcher started {world} ranks")
    if world > 1:
        import torch.distributed as dist
        dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=120))
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return
    from learned_block_sparse_b200 import synth
    w = workload_of(args)
    rng = np.random.default_rng(0)
    groups_all = [(b, h) for b in range(w.B) for h in range(w.Hkv)]
    n_groups = min(8, len(groups_all))
    groups = sorted(groups_all[i] for i in rng.choice(len(groups_all), n_groups, replace=False))
    q_host, K_host, V_host = host_slices(w, groups)
    W = synth.make_predictor(w)[0].numpy() if w.tau_mode == "predictor" else None
    metas, qf, heads, scores, pool = oracle_setup(w, (q_host, K_host, V_host), groups, args.sub_blocks)
    thr = oracle_thresholds(w, q_host, W, scores, args.density)
    for _ in range(args.warmup):
        oracle_step(w, q_host, K_host, V_host, W, thr, metas, qf, heads, pool, args.sub_blocks)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        oracle_step(w, q_host, K_host, V_host, W, thr, metas, qf, heads, pool, args.sub_blocks)
    dt = (time.perf_counter() - t0) / args.steps
    value = len(heads) / dt
    cores = pool._max_workers
    line = {"impl": "reference", "metric": "sparse decode queries/s", "value": value, "unit": "queries/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic",
            "config": {"workload": w.name, "density": args.density, "batch": w.B, "seq_len": w.n,
                       **({"sub_blocks": args.sub_blocks} if args.sub_blocks > 1 else {})},
            "cpu_baseline": {"value": value, "unit": "queries/s", "cores": cores, "kind": "oracle",
                             "sample": f"{len(heads)} decode queries ({n_groups} (batch, kv head) groups) of "
                                       f"the workload per step"},
            "e2e": {"value": value, "unit": "queries/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def host_slices(w, groups):
    """q for all heads, and K/V host tensors holding (at least) the sampled groups.
    Only the sampled batches are generated; the others stay empty."""
    from learned_block_sparse_b200 import synth
    q = synth.make_q(w)
    K = torch.empty((w.B, w.Hkv, w.capacity, w.d), dtype=w.torch_dtype)
    V = torch.empty_like(K)
    needles = synth.make_needles(w)
    for b in sorted({g[0] for g in groups}):
        synth.fill_kv(w, q, "k", K[b:b + 1], b, b + 1, needles)
        synth.fill_kv(w, q, "v", V[b:b + 1], b, b + 1, needles)
    return q, K, V


# ---------------------------------------------------------------- GPU arm
def run_eta(args):
    world, rank, local = dist_setup(args)
    from learned_block_sparse_b200 import binding, synth
    from learned_block_sparse_b200.workload import DeviceWorkload

    w = workload_of(args)
    dev = torch.device("cuda", torch.cuda.current_device())
    dw = DeviceWorkload(w, device=dev, n_splits=args.n_splits, sub_blocks=args.sub_blocks)
    dec = dw.dec
    stream = torch.cuda.current_stream()
    flush_buf = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    clean_buf = torch.ones(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev)

    class _Flush:
        @staticmethod
        def zero_():
            # write > 2x L2 (evicts every line of the inputs), then read another
            # buffer > L2 so the dirty lines of that write are written back
            # before the timed region instead of inside it
            flush_buf.zero_()
            if args.l2_flush == "write+read":
                clean_buf.sum()
    flush = _Flush()
    S = args.n_splits or torch.cuda.get_device_properties(dev).multi_processor_count

    def thresholds(density):
        tau, stride, bias = dw.calibrate(density)
        return tau, stride, bias

    def step_phases(tau, stride, bias, ev):
        """screen (forming the Eq. 1 thresholds itself when there is a
        predictor) -> decode (split merge fused), events between phases."""
        ev[0].record(stream)
        if bias is not None:
            binding.screen_predict(dec.shape, dec.params, dw.q, dec.meta, w.n, dw.W, bias, dec.tau, dec.ws)
            t, s = dec.tau, w.Hq
        else:
            binding.screen(dec.shape, dec.params, dw.q, dec.meta, w.n, tau, stride, dec.ws)
            t, s = tau, stride
        if ev[1] is not None:   # an event between the launches also stops the decode starting early
            ev[1].record(stream)
        binding.decode_screened(dec.shape, dec.params, dw.q, dw.K, dw.V, w.n, t, s, dec.out, dec.ws)
        ev[2].record(stream)

    def time_sparse(density, sample_clocks=False):
        tau, stride, bias = thresholds(density)
        for _ in range(args.warmup):
            flush.zero_()
            step_phases(tau, stride, bias, [torch.cuda.Event(enable_timing=True) for _ in range(3)])
        torch.cuda.synchronize()
        # whole steps (the two launches back to back): the headline time
        evs = [[torch.cuda.Event(enable_timing=True), None, torch.cuda.Event(enable_timing=True)]
               for _ in range(args.steps)]
        clk = ClockSampler(local) if sample_clocks else None
        barrier(world)
        torch.cuda.synchronize()
        if clk:
            clk.start()
        for i in range(args.steps):
            flush.zero_()
            step_phases(tau, stride, bias, evs[i])
        torch.cuda.synchronize()
        barrier(world)
        clocks = clk.stop() if clk else None
        per_step = [e[0].elapsed_time(e[2]) for e in evs]
        tot = statistics.median(per_step)
        # the same steps with an event between the launches, for the phase split
        pevs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]
        for i in range(args.steps):
            flush.zero_()
            step_phases(tau, stride, bias, pevs[i])
        torch.cuda.synchronize()
        scr = statistics.median(e[0].elapsed_time(e[1]) for e in pevs)
        dec_t = statistics.median(e[1].elapsed_time(e[2]) for e in pevs)
        # counts for the byte model (untimed extra screen with count outputs)
        ucnt = torch.zeros((w.B, w.Hkv), dtype=torch.int32, device=dev)
        hcnt = torch.zeros((w.B, w.Hq), dtype=torch.int32, device=dev)
        if bias is not None:
            binding.screen_predict(dec.shape, dec.params, dw.q, dec.meta, w.n, dw.W, bias, dec.tau, dec.ws,
                                   union_cnt=ucnt, active_cnt=hcnt)
        else:
            binding.screen(dec.shape, dec.params, dw.q, dec.meta, w.n, tau, stride, dec.ws, union_cnt=ucnt,
                           active_cnt=hcnt)
        torch.cuda.synchronize()
        bm = byte_model(w, ucnt.cpu().numpy(), hcnt.cpu().numpy(), S, args.sub_blocks)
        st = dec.device_status()
        if st != 0:
            raise RuntimeError(f"device status {st} after timed steps")
        return {"ms": tot, "ms_mean": sum(per_step) / len(per_step), "ms_screen": scr, "ms_decode": dec_t,
                "bytes": bm, "clocks": clocks, "tau": (tau, stride, bias)}

    def time_dense():
        for _ in range(args.warmup):
            flush.zero_()
            dec.dense(dw.q, dw.K, dw.V, w.n)
        evs = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(args.steps)]
        torch.cuda.synchronize()
        for i in range(args.steps):
            flush.zero_()
            evs[i][0].record(stream)
            dec.dense(dw.q, dw.K, dw.V, w.n)
            evs[i][1].record(stream)
        torch.cuda.synchronize()
        return statistics.median(e[0].elapsed_time(e[1]) for e in evs)

    def time_e2e(tau, stride, bias):
        """Public API (EtaDecoder.step) with q from pinned host memory and the
        output read back to pinned host memory, every step."""
        q_pin = dw.q_host.pin_memory()
        out_pin = torch.empty((w.B, w.Hq, w.d), dtype=torch.float32).pin_memory()
        q_dev = torch.empty_like(dw.q)
        tau_dev = tau

        def one():
            q_dev.copy_(q_pin, non_blocking=True)
            if bias is not None:
                o = dec.step(q_dev, dw.K, dw.V, w.n, W=dw.W, bias=bias)
            else:
                o = dec.step(q_dev, dw.K, dw.V, w.n, tau=tau_dev, tau_batch_stride=stride)
            out_pin.copy_(o, non_blocking=True)
        for _ in range(args.warmup):
            flush.zero_()
            one()
        torch.cuda.synchronize()
        evs = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(args.steps)]
        for i in range(args.steps):
            flush.zero_()
            evs[i][0].record(stream)
            one()
            evs[i][1].record(stream)
        torch.cuda.synchronize()
        ms = statistics.median(e[0].elapsed_time(e[1]) for e in evs)
        h2d = q_pin.numel() * q_pin.element_size()
        d2h = out_pin.numel() * out_pin.element_size()
        return ms, h2d, d2h

    main = time_sparse(args.density, sample_clocks=True)
    ms = max_over_ranks(main["ms"], world)
    ms_dec = max_over_ranks(main["ms_decode"], world)
    queries = w.B * w.Hq
    value = job_throughput(queries, ms, world)
    bm = main["bytes"]
    peak, peak_kind = measured_peaks()
    achieved = bm["decode_kernel"] / (ms_dec * 1e-3) / 1e9
    line = {
        "metric": "sparse decode queries/s", "value": value, "unit": "queries/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
        "ms_per_step_mean": max_over_ranks(main["ms_mean"], world), "step_time": "median of the timed steps",
        "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": {"bf16": "bf16", "fp8": "fp8", "f32": "f32"}[w.dtype],
        "data": "synthetic (seeded Philox4x32-10 + Box-Muller normals, shaped like the pages' decode workloads)",
        "config": {"workload": w.name, "batch": w.B, "q_heads": w.Hq, "kv_heads": w.Hkv, "head_dim": w.d,
                   "seq_len": w.n, "block": w.bs, "tau": w.tau_mode, "density_target": args.density,
                   **({"sub_blocks": args.sub_blocks} if args.sub_blocks > 1 else {}),
                   "l2": ("flushed before every timed step: 512 MiB write" +
                          (", then a 512 MiB read (no dirty lines left)" if args.l2_flush == "write+read" else "")), "parallelism": f"replicas x{world}"},
        "effective_hbm_gbs": bm["step_read"] / (ms * 1e-3) / 1e9,
        "d_head": bm["d_head"], "d_union": bm["d_union"], "union_blocks": bm["union_blocks"],
        "phases_ms": {("screen+predict" if w.tau_mode == "predictor" else "screen"): main["ms_screen"],
                      "decode": main["ms_decode"]},
        "roofline": {"bound": "hbm",
                     "kernel": ("decode_kernel" if w.dtype == "f32" else "decode_mma_kernel") + " (split merge fused)",
                     "achieved": achieved, "peak": peak, "unit": "GB/s", "frac": achieved / peak,
                     "peak_source": peak_kind, "traffic": measured_traffic(w.name, bm["union_blocks"]),
                     "bytes_per_launch": bm["decode_kernel"]},
        "gpu_launches": LAUNCHES_PER_STEP[w.tau_mode] * args.steps,
        "clocks": main["clocks"],
    }
    if not args.no_dense:
        dms = max_over_ranks(time_dense(), world)
        line["dense"] = {"ms_per_step": dms, "queries_per_s": world * queries / (dms * 1e-3),
                         "hbm_gbs": bm["dense_kv"] / (dms * 1e-3) / 1e9,
                         "frac_of_peak": bm["dense_kv"] / (dms * 1e-3) / 1e9 / peak}
        line["speedup_vs_dense"] = dms / ms
    if not args.no_e2e:
        tau, stride, bias = main["tau"]
        ems, h2d, d2h = time_e2e(tau, stride, bias)
        ems = max_over_ranks(ems, world)
        line["e2e"] = {"value": world * queries / (ems * 1e-3), "unit": "queries/s",
                       "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": ems}
    if not args.no_sweep:
        sw = {}
        for dens in w.densities:
            r = time_sparse(dens)
            sms = max_over_ranks(r["ms"], world)
            sw[str(dens)] = {"ms": sms, "queries_per_s": job_throughput(queries, sms, world),
                             "d_head": r["bytes"]["d_head"], "d_union": r["bytes"]["d_union"],
                             "effective_hbm_gbs": r["bytes"]["step_read"] / (r["ms"] * 1e-3) / 1e9,
                             "decode_frac": r["bytes"]["decode_kernel"] / (r["ms_decode"] * 1e-3) / 1e9 / peak}
            if "dense" in line:
                sw[str(dens)]["speedup_vs_dense"] = line["dense"]["ms_per_step"] / sms
        line["sweep"] = sw
    if not args.no_diagnostics:
        line["screen_quality"] = screen_quality(w, dw, main["tau"])
    if rank == 0 and world == 1 and not args.no_cpu:
        line["cpu_baseline"] = cpu_baseline(w, args, dw)
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


def screen_quality(w, dw, thresholds):
    """The pages' Table 16 screen diagnostics for this workload at the main
    density (a dense pass over K, outside every timed region)."""
    from learned_block_sparse_b200 import binding, diagnostics
    tau, stride, bias = thresholds
    dec = dw.dec
    if bias is not None:
        binding.predict_tau(dec.shape, dw.q, dw.W, bias, dec.tau)
        tau, stride = dec.tau, w.Hq
    r = diagnostics.screen_diagnostics(dec, dw.q, dw.K, w.n, tau, stride)
    return {k: r[k] for k in ("false_negative", "false_positive", "token_recall", "missed_mass")}


def cpu_baseline(w, args, dw):
    """The oracle (as it stands) on a bounded sample of the workload: `cpu_groups`
    (batch, kv head) groups, all their query heads, one decode step."""
    from learned_block_sparse_b200 import synth
    rng = np.random.default_rng(1)
    groups_all = [(b, h) for b in range(w.B) for h in range(w.Hkv)]
    n = min(args.cpu_groups, len(groups_all))
    groups = sorted(groups_all[i] for i in rng.choice(len(groups_all), n, replace=False))
    q_host, K_host, V_host = host_slices(w, groups)
    W = synth.make_predictor(w)[0].numpy() if w.tau_mode == "predictor" else None
    metas, qf, heads, scores, pool = oracle_setup(w, (q_host, K_host, V_host), groups, args.sub_blocks)
    thr = oracle_thresholds(w, q_host, W, scores, args.density)
    # repeat the step until about 5 s have passed (bounded at 200 steps)
    t0 = time.perf_counter()
    reps = 0
    while reps < 200:
        oracle_step(w, q_host, K_host, V_host, W, thr, metas, qf, heads, pool, args.sub_blocks)
        reps += 1
        if time.perf_counter() - t0 >= 5.0:
            break
    dt = time.perf_counter() - t0
    # the same step on one thread, for the first group's heads (about 2 s)
    one = cf.ThreadPoolExecutor(max_workers=1)
    heads1 = heads[:w.G]
    t1 = time.perf_counter()
    reps1 = 0
    while reps1 < 200:
        oracle_step(w, q_host, K_host, V_host, W, thr, metas, qf, heads1, one, args.sub_blocks)
        reps1 += 1
        if time.perf_counter() - t1 >= 2.0:
            break
    dt1 = time.perf_counter() - t1
    one.shutdown()
    return {"value": reps * len(heads) / dt, "unit": "queries/s", "cores": pool._max_workers, "kind": "oracle",
            "sample": f"{len(heads)} decode queries ({n} of {len(groups_all)} (batch, kv head) groups) per step, "
                      f"{reps} steps: predictor + screen + gated attention in C (fp32 decisions, fp64 attention)",
            "seconds": dt, "value_1_thread": reps1 * len(heads1) / dt1,
            "sample_1_thread": f"{len(heads1)} decode queries (one group) per step, {reps1} steps"}


def main():
    args = parse_args()
    if args.gpus > 1 and "WORLD_SIZE" not in os.environ:
        sys.exit(launch_ranks(args))
    if args.impl == "reference":
        run_reference(args)
    else:
        run_eta(args)


if __name__ == "__main__":
    main()

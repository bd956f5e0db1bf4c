"""Seeded synthetic decode workloads for ETA block-sparse decode.

The five workloads below restate the shapes, dtypes and key structure of the
decode configurations this library is measured on. Every tensor is drawn by the
counter-based generator in ``synth.c`` (Philox4x32-10 + Box-Muller), so the CPU
oracle and the CUDA path read identical bytes and any (batch, head) slice can be
regenerated alone.

Nothing here computes any part of the attention method; the only arithmetic
besides drawing numbers is the needle construction (adding a multiple of the
query direction to a block's keys) and the density-to-threshold quantile pick,
which turns a vector of block scores into the threshold that admits a given
fraction of them.
"""
from __future__ import annotations

import ctypes
import dataclasses
import math
import os
from typing import Optional, Sequence

import numpy as np
import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
_LIB_PATH = os.path.join(_HERE, "libsynth.so")

STREAM_Q, STREAM_K, STREAM_V, STREAM_OFFSET, STREAM_W, STREAM_NEEDLE = 1, 2, 3, 4, 5, 6
F32, BF16 = 0, 1

_lib = None


def _load():
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(_LIB_PATH):
        from .. import _build
        _build.build_synth()
    lib = ctypes.CDLL(_LIB_PATH)
    u64, u32, i64, i32, dbl, vp = (ctypes.c_uint64, ctypes.c_uint32, ctypes.c_int64,
                                   ctypes.c_int, ctypes.c_double, ctypes.c_void_p)
    lib.synth_normal_fill.argtypes = [u64, u32, u64, i64, dbl, dbl, i32, vp]
    lib.synth_normal_fill.restype = None
    lib.synth_fill_kv.argtypes = [u64, u32, u32, i32, i64, i64, i64, i64, i64, i64, i64, i64,
                                  dbl, vp, i32, i64, vp, i32, dbl, vp]
    lib.synth_fill_kv.restype = None
    lib.synth_pick_blocks.argtypes = [u64, u32, i64, i32, i64, vp]
    lib.synth_pick_blocks.restype = i32
    lib.synth_normal_at.argtypes = [u64, u32, u64]
    lib.synth_normal_at.restype = dbl
    lib.synth_philox4x32_10.argtypes = [vp, vp, vp]
    lib.synth_philox4x32_10.restype = None
    lib.synth_set_threads.argtypes = [i32]
    lib.synth_set_threads.restype = None
    lib.synth_set_threads(int(os.environ.get("ETA_SYNTH_THREADS", os.cpu_count() or 1)))
    _lib = lib
    return lib


def philox4x32_10(ctr: Sequence[int], key: Sequence[int]) -> list:
    lib = _load()
    c = (ctypes.c_uint32 * 4)(*ctr)
    k = (ctypes.c_uint32 * 2)(*key)
    o = (ctypes.c_uint32 * 4)()
    lib.synth_philox4x32_10(c, k, o)
    return list(o)


def normal_at(seed: int, stream: int, f: int) -> float:
    return _load().synth_normal_at(seed, stream, f)


@dataclasses.dataclass
class Workload:
    """One decode-step workload. ``n`` counts cached tokens including the current one."""
    name: str
    dtype: str           # storage dtype of K, V: "f32", "bf16" or "fp8" (e4m3; q then bf16)
    B: int
    Hq: int
    Hkv: int
    d: int
    n: int
    bs: int              # block size b
    z: float             # screening confidence
    tau_mode: str        # "const" (per-head constant) or "predictor"
    densities: tuple     # target fractions of screened blocks admitted (see density_kind)
    seed: int
    beta: float = 5.0
    n_local: int = 1
    offset_std: float = 0.0
    n_needles: int = 0
    needle_scale: float = 3.0
    cap: Optional[int] = None    # allocated tokens per (b, kv head); default n rounded up to 4 blocks
    density_kind: str = "head"   # "head": per query head; "union": of the GQA group's union

    @property
    def capacity(self) -> int:
        if self.cap is not None:
            if self.cap < self.n:
                raise ValueError(f"capacity {self.cap} below the token count {self.n}")
            return ((self.cap + self.bs - 1) // self.bs) * self.bs
        q = 4 * self.bs          # whole groups of 4 blocks: 16-byte aligned metadata rows
        return ((self.n + q - 1) // q) * q

    @property
    def nb(self) -> int:
        return (self.n + self.bs - 1) // self.bs

    @property
    def n_screened(self) -> int:
        return max(0, self.nb - self.n_local)

    @property
    def G(self) -> int:
        return self.Hq // self.Hkv

    @property
    def dtype_code(self) -> int:
        """Generator dtype of q (and of K, V before an fp8 rounding)."""
        return F32 if self.dtype == "f32" else BF16

    @property
    def torch_dtype(self):
        """Storage dtype of K and V."""
        return {"f32": torch.float32, "bf16": torch.bfloat16, "fp8": torch.float8_e4m3fn}[self.dtype]

    @property
    def q_torch_dtype(self):
        """Storage dtype of q: bf16 with fp8 K/V."""
        return torch.float32 if self.dtype == "f32" else torch.bfloat16

    def replace(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


SQRT_HALF = math.sqrt(0.5)

# The decode configurations (names state the shapes). 1-5 are the parity and
# benchmark workloads; 6 is the attention shape of the pages' block-size /
# chunk-size table (Table 10: batch 64, 512K tokens, 32 query / 4 KV heads of
# dimension 64, blocks of 64), calibrated to the union densities quoted there;
# 7 is workload 3 with its K and V rounded to fp8 (e4m3).
WORKLOADS = {
    1: Workload("tiny-f32-mha2-d64-n1024-b16", "f32", 1, 2, 2, 64, 1024, 16, z=1.5,
                tau_mode="const", densities=(0.40,), seed=1001),
    2: Workload("mha16-d128-n32k-b64-needles8", "bf16", 1, 16, 16, 128, 32768, 64, z=1.0,
                tau_mode="predictor", densities=(0.38,), seed=1002, n_needles=8),
    3: Workload("gqa32x8-d128-n128k-b32-B8", "bf16", 8, 32, 8, 128, 131072, 32, z=1.0,
                tau_mode="predictor", densities=(0.20, 0.38, 0.60), seed=1003,
                offset_std=SQRT_HALF),
    4: Workload("mha16-d128-n512k-b64-needles32", "bf16", 1, 16, 16, 128, 524288, 64, z=1.0,
                tau_mode="predictor", densities=(0.38,), seed=1004, n_needles=32),
    5: Workload("mha16-d128-n64k-b16-const-sweep", "bf16", 1, 16, 16, 128, 65536, 16, z=1.5,
                tau_mode="const", densities=(0.10, 0.25, 0.38, 0.60, 1.0), seed=1005,
                offset_std=SQRT_HALF),
    6: Workload("gqa32x4-d64-n512k-b64-B64", "bf16", 64, 32, 4, 64, 524288, 64, z=1.0,
                tau_mode="predictor", densities=(0.16, 0.355, 0.512), seed=1006,
                offset_std=SQRT_HALF, density_kind="union"),
    7: Workload("gqa32x8-d128-n128k-b32-B8-fp8", "fp8", 8, 32, 8, 128, 131072, 32, z=1.0,
                tau_mode="predictor", densities=(0.20, 0.38, 0.60), seed=1003,
                offset_std=SQRT_HALF),
}
WORKLOAD5_BATCHES = (1, 4, 16, 64)


def _empty(shape, dtype, pin: bool):
    t = torch.empty(shape, dtype=dtype)
    if pin:
        t = t.pin_memory()
    return t


def make_q(w: Workload, pin: bool = False) -> torch.Tensor:
    """q [B][Hq][d] ~ N(0,1) in the workload dtype."""
    lib = _load()
    q = _empty((w.B, w.Hq, w.d), w.q_torch_dtype, pin)
    lib.synth_normal_fill(w.seed, STREAM_Q, 0, q.numel(), 0.0, 1.0, w.dtype_code, q.data_ptr())
    return q


def make_needles(w: Workload) -> Optional[torch.Tensor]:
    """[B][Hkv][n_needles] distinct screened block indices per (b, kv head)."""
    if w.n_needles <= 0:
        return None
    lib = _load()
    out = torch.empty((w.B, w.Hkv, w.n_needles), dtype=torch.int32)
    rc = lib.synth_pick_blocks(w.seed, STREAM_NEEDLE, w.B * w.Hkv, w.n_needles,
                               w.n_screened, out.data_ptr())
    if rc != 0:
        raise ValueError("more needles than screened blocks")
    return out


def fill_kv(w: Workload, q: torch.Tensor, which: str, dst: torch.Tensor, b0: int = 0,
            b1: Optional[int] = None, needles: Optional[torch.Tensor] = None) -> torch.Tensor:
    """Fill ``dst`` ([b1-b0][Hkv][capacity][d], CPU) with batches [b0,b1) of K or V."""
    lib = _load()
    b1 = w.B if b1 is None else b1
    assert dst.shape == (b1 - b0, w.Hkv, w.capacity, w.d) and dst.dtype == w.torch_dtype
    assert dst.is_contiguous() and not dst.is_cuda
    is_k = which == "k"
    if is_k and needles is None:
        needles = make_needles(w)
    if w.capacity > w.n:
        dst[:, :, w.n:, :].view(torch.uint8 if w.dtype == "fp8" else dst.dtype).zero_()
    fp8 = w.dtype == "fp8"
    # fp8 caches: drawn in fp32, then rounded to e4m3 (nearest even) by torch
    out = torch.zeros(dst.shape, dtype=torch.float32) if fp8 else dst
    lib.synth_fill_kv(w.seed, STREAM_K if is_k else STREAM_V, STREAM_OFFSET, F32 if fp8 else w.dtype_code, w.B,
                      w.Hkv, w.n, w.capacity, w.d, w.bs, b0, b1,
                      w.offset_std if is_k else 0.0,
                      q.data_ptr(), w.dtype_code, w.Hq,
                      needles.data_ptr() if (is_k and needles is not None) else None,
                      w.n_needles if is_k else 0, w.needle_scale, out.data_ptr())
    if fp8:
        dst.copy_(out.to(torch.float8_e4m3fn))
    return dst


def make_kv(w: Workload, q: torch.Tensor, pin: bool = False):
    """K, V [B][Hkv][capacity][d]; tokens >= n are zero."""
    out = []
    for which in ("k", "v"):
        t = _empty((w.B, w.Hkv, w.capacity, w.d), w.torch_dtype, pin)
        out.append(fill_kv(w, q, which, t))
    return out[0], out[1]


def make_predictor(w: Workload):
    """W [Hq*d][Hq] with head h's weights w_h ~ N(0, 1/d) on the block diagonal; zero bias."""
    lib = _load()
    wh = torch.empty((w.Hq, w.d), dtype=torch.float32)
    lib.synth_normal_fill(w.seed, STREAM_W, 0, wh.numel(), 0.0, 1.0 / math.sqrt(w.d), F32,
                          wh.data_ptr())
    W = torch.zeros((w.Hq * w.d, w.Hq), dtype=torch.float32)
    for h in range(w.Hq):
        W[h * w.d:(h + 1) * w.d, h] = wh[h]
    return W, torch.zeros(w.Hq, dtype=torch.float32)


def tau_for_density(scores: np.ndarray, density: float) -> float:
    """Threshold admitting round(density * m) of the m scores (at least one): the
    k-th largest score, so that ``score >= tau`` holds for exactly those blocks when
    scores are distinct. density >= 1 gives -inf (every block admitted)."""
    s = np.asarray(scores, dtype=np.float32).ravel()
    if density >= 1.0 or s.size == 0:
        return float("-inf")
    k = max(1, int(round(density * s.size)))
    return float(np.sort(s)[::-1][k - 1])

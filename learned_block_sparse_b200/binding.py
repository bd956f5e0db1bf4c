"""ctypes binding of libeta.so (the C ABI in ``include/eta.h``).

Argument marshalling only: every step of the decode path runs in the CUDA
library. Tensors are torch CUDA tensors (PyTorch supplies device memory and
streams); each call is enqueued on the current torch stream. If the native
library is missing, importing this module raises: there is no fallback.
"""
from __future__ import annotations

import ctypes
import math
import os
from typing import Optional

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libeta.so")

ETA_OK, ETA_ERR_INVALID_ARG, ETA_ERR_UNSUPPORTED, ETA_ERR_WORKSPACE, ETA_ERR_CUDA, ETA_ERR_DEVICE_TIMEOUT = range(6)
ETA_F32, ETA_BF16 = 0, 1


class EtaError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {status_string(status)} (status {status})")


class Shape(ctypes.Structure):
    _fields_ = [("batch", ctypes.c_int32), ("n_q_heads", ctypes.c_int32), ("n_kv_heads", ctypes.c_int32),
                ("head_dim", ctypes.c_int32), ("block_size", ctypes.c_int32), ("capacity", ctypes.c_int64),
                ("kv_dtype", ctypes.c_int32), ("q_dtype", ctypes.c_int32)]


ETA_FP8_E4M3 = 2
GATE_SIGMOID, GATE_HARD = 0, 1   # Eq. 2-3 multiplicative gate; strict mode (hard masking)


class Params(ctypes.Structure):
    _fields_ = [("beta", ctypes.c_float), ("z", ctypes.c_float), ("offset_a", ctypes.c_float),
                ("n_local", ctypes.c_int32), ("n_splits", ctypes.c_int32), ("gate", ctypes.c_int32),
                ("sub_blocks", ctypes.c_int32)]


class Meta(ctypes.Structure):
    _fields_ = [("mu", ctypes.c_void_p), ("var", ctypes.c_void_p), ("maxnorm", ctypes.c_void_p)]


class Pages(ctypes.Structure):
    _fields_ = [("block_table", ctypes.c_void_p), ("num_pages", ctypes.c_int32)]


class ScreenOut(ctypes.Structure):
    _fields_ = [("active_idx", ctypes.c_void_p), ("active_cnt", ctypes.c_void_p),
                ("union_list", ctypes.c_void_p), ("union_cnt", ctypes.c_void_p), ("scores", ctypes.c_void_p)]


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"libeta.so not built ({LIB_PATH}); run `python -m learned_block_sparse_b200._build`")
    L = ctypes.CDLL(LIB_PATH)
    P, vp, i64, f32, sz = ctypes.POINTER, ctypes.c_void_p, ctypes.c_int64, ctypes.c_float, ctypes.c_size_t
    st = ctypes.c_int
    L.eta_abi_version.restype = ctypes.c_int
    L.eta_abi_version.argtypes = []
    L.eta_status_string.restype = ctypes.c_char_p
    L.eta_status_string.argtypes = [st]
    L.eta_build_block_meta.restype = st
    L.eta_build_block_meta.argtypes = [P(Shape), vp, i64, i64, Meta, vp]
    L.eta_predict_tau.restype = st
    L.eta_predict_tau.argtypes = [P(Shape), vp, vp, vp, vp, vp]
    L.eta_decode_workspace_bytes.restype = sz
    L.eta_decode_workspace_bytes.argtypes = [P(Shape), P(Params)]
    L.eta_workspace_init.restype = st
    L.eta_workspace_init.argtypes = [vp, sz, vp]
    L.eta_screen.restype = st
    L.eta_screen.argtypes = [P(Shape), P(Params), vp, Meta, i64, vp, i64, P(ScreenOut), vp, sz, vp]
    L.eta_decode_sparse.restype = st
    L.eta_decode_sparse.argtypes = [P(Shape), P(Params), vp, vp, vp, Meta, i64, vp, i64, vp, P(ScreenOut),
                                    vp, sz, vp]
    L.eta_screen_predict.restype = st
    L.eta_screen_predict.argtypes = [P(Shape), P(Params), vp, Meta, i64, vp, vp, vp, P(ScreenOut), vp, sz, vp]
    L.eta_decode_sparse_predict.restype = st
    L.eta_decode_sparse_predict.argtypes = [P(Shape), P(Params), vp, vp, vp, Meta, i64, vp, vp, vp, vp,
                                            P(ScreenOut), vp, sz, vp]
    L.eta_screen_ragged.restype = st
    L.eta_screen_ragged.argtypes = [P(Shape), P(Params), vp, Meta, vp, i64, vp, i64, vp, vp, vp, P(ScreenOut),
                                    vp, sz, vp]
    L.eta_decode_sparse_ragged.restype = st
    L.eta_decode_sparse_ragged.argtypes = [P(Shape), P(Params), vp, vp, vp, Meta, vp, i64, vp, i64, vp, vp, vp,
                                           vp, P(ScreenOut), vp, sz, vp]
    L.eta_decode_screened_ragged.restype = st
    L.eta_decode_screened_ragged.argtypes = [P(Shape), P(Params), vp, vp, vp, vp, i64, vp, i64, vp, vp, sz, vp]
    L.eta_decode_dense_ragged.restype = st
    L.eta_decode_dense_ragged.argtypes = [P(Shape), P(Params), vp, vp, vp, vp, i64, vp, i64, vp, vp, sz, vp]
    L.eta_build_block_meta_paged.restype = st
    L.eta_build_block_meta_paged.argtypes = [P(Shape), vp, Pages, i64, i64, Meta, vp]
    L.eta_decode_sparse_paged.restype = st
    L.eta_decode_sparse_paged.argtypes = [P(Shape), P(Params), vp, vp, vp, Pages, Meta, vp, i64, vp, i64, vp, vp, vp,
                                          vp, P(ScreenOut), vp, sz, vp]
    L.eta_decode_screened_paged.restype = st
    L.eta_decode_screened_paged.argtypes = [P(Shape), P(Params), vp, vp, vp, Pages, vp, i64, vp, i64, vp, vp, sz, vp]
    L.eta_decode_dense_paged.restype = st
    L.eta_decode_dense_paged.argtypes = [P(Shape), P(Params), vp, vp, vp, Pages, vp, i64, vp, i64, vp, vp, sz, vp]
    L.eta_block_stats.restype = st
    L.eta_block_stats.argtypes = [P(Shape), P(Params), vp, vp, i64, vp, i64, vp, vp, vp, vp]
    L.eta_screen_diagnostics.restype = st
    L.eta_screen_diagnostics.argtypes = [P(Shape), P(Params), i64, vp, i64, vp, vp, vp, vp, vp, vp, vp]
    L.eta_test_withhold_copy.restype = st
    L.eta_test_withhold_copy.argtypes = [i64]
    L.eta_decode_screened.restype = st
    L.eta_decode_screened.argtypes = [P(Shape), P(Params), vp, vp, vp, i64, vp, i64, vp, vp, sz, vp]
    L.eta_decode_dense.restype = st
    L.eta_decode_dense.argtypes = [P(Shape), P(Params), vp, vp, vp, i64, vp, i64, vp, vp, sz, vp]
    L.eta_decode_sparse_static.restype = st
    L.eta_decode_sparse_static.argtypes = [P(Shape), P(Params), vp, vp, vp, Meta, i64, vp, i64, vp, P(ScreenOut),
                                           vp, vp]
    L.eta_read_device_status.restype = st
    L.eta_read_device_status.argtypes = [vp, vp, P(st)]
    return L


lib = _load()
EXPORTED = ("eta_abi_version", "eta_status_string", "eta_build_block_meta", "eta_predict_tau",
            "eta_decode_workspace_bytes", "eta_workspace_init", "eta_screen", "eta_decode_sparse",
            "eta_decode_screened", "eta_decode_dense", "eta_read_device_status", "eta_decode_sparse_static",
            "eta_screen_predict", "eta_decode_sparse_predict", "eta_screen_ragged", "eta_decode_sparse_ragged",
            "eta_decode_screened_ragged", "eta_decode_dense_ragged", "eta_build_block_meta_paged",
            "eta_decode_sparse_paged", "eta_decode_screened_paged", "eta_decode_dense_paged", "eta_block_stats",
            "eta_screen_diagnostics", "eta_test_withhold_copy")
STATIC_SCRATCH_BYTES = 32 << 20


def status_string(status: int) -> str:
    return lib.eta_status_string(status).decode()


def _check(status: int, where: str) -> None:
    if status != ETA_OK:
        raise EtaError(status, where)


def _dtype_code(t: torch.dtype) -> int:
    if t == torch.float32:
        return ETA_F32
    if t == torch.bfloat16:
        return ETA_BF16
    if t == torch.float8_e4m3fn:
        return ETA_FP8_E4M3
    raise TypeError(f"unsupported dtype {t}")


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def make_shape(batch, n_q_heads, n_kv_heads, head_dim, block_size, capacity, kv_dtype, q_dtype) -> Shape:
    return Shape(batch, n_q_heads, n_kv_heads, head_dim, block_size, capacity,
                 _dtype_code(kv_dtype) if isinstance(kv_dtype, torch.dtype) else kv_dtype,
                 _dtype_code(q_dtype) if isinstance(q_dtype, torch.dtype) else q_dtype)


def make_params(beta=5.0, z=1.0, offset_a=0.0, n_local=1, n_splits=0, gate=GATE_SIGMOID, sub_blocks=1) -> Params:
    return Params(beta, z, offset_a, n_local, n_splits, gate, sub_blocks)


def build_block_meta(shape: Shape, k: torch.Tensor, blk_begin: int, blk_end: int, mu: torch.Tensor,
                     var: torch.Tensor, maxnorm: torch.Tensor, stream=None) -> None:
    _check(lib.eta_build_block_meta(ctypes.byref(shape), _ptr(k), blk_begin, blk_end,
                                    Meta(mu.data_ptr(), var.data_ptr(), maxnorm.data_ptr()), _stream(stream)),
           "eta_build_block_meta")


def predict_tau(shape: Shape, q: torch.Tensor, W: torch.Tensor, bias: torch.Tensor, tau: torch.Tensor,
                stream=None) -> None:
    _check(lib.eta_predict_tau(ctypes.byref(shape), _ptr(q), _ptr(W), _ptr(bias), _ptr(tau), _stream(stream)),
           "eta_predict_tau")


def workspace_bytes(shape: Shape, params: Params) -> int:
    n = lib.eta_decode_workspace_bytes(ctypes.byref(shape), ctypes.byref(params))
    if n == 0:
        raise EtaError(ETA_ERR_INVALID_ARG, "eta_decode_workspace_bytes")
    return int(n)


def alloc_workspace(shape: Shape, params: Params, device=None) -> torch.Tensor:
    n = workspace_bytes(shape, params)
    ws = torch.empty(n + 256, dtype=torch.uint8, device=device or "cuda")
    off = (-ws.data_ptr()) % 256
    ws = ws[off:off + n]
    _check(lib.eta_workspace_init(_ptr(ws), n, _stream()), "eta_workspace_init")
    return ws


def _screen_out(active_idx=None, active_cnt=None, union_list=None, union_cnt=None, scores=None):
    if all(x is None for x in (active_idx, active_cnt, union_list, union_cnt, scores)):
        return None
    return ScreenOut(*(None if x is None else x.data_ptr()
                       for x in (active_idx, active_cnt, union_list, union_cnt, scores)))


def screen(shape: Shape, params: Params, q, meta, n_tokens: int, tau: torch.Tensor, tau_batch_stride: int,
           ws: torch.Tensor, stream=None, **outs) -> None:
    so = _screen_out(**outs)
    _check(lib.eta_screen(ctypes.byref(shape), ctypes.byref(params), _ptr(q), Meta(*(m.data_ptr() for m in meta)),
                          n_tokens, _ptr(tau), tau_batch_stride, ctypes.byref(so) if so is not None else None,
                          _ptr(ws), ws.numel(), _stream(stream)), "eta_screen")


def screen_predict(shape: Shape, params: Params, q, meta, n_tokens: int, W: torch.Tensor, bias: torch.Tensor,
                   tau_out: torch.Tensor, ws: torch.Tensor, stream=None, **outs) -> None:
    so = _screen_out(**outs)
    _check(lib.eta_screen_predict(ctypes.byref(shape), ctypes.byref(params), _ptr(q),
                                  Meta(*(m.data_ptr() for m in meta)), n_tokens, _ptr(W), _ptr(bias), _ptr(tau_out),
                                  ctypes.byref(so) if so is not None else None, _ptr(ws), ws.numel(),
                                  _stream(stream)), "eta_screen_predict")


def decode_sparse_predict(shape: Shape, params: Params, q, k, v, meta, n_tokens: int, W: torch.Tensor,
                          bias: torch.Tensor, tau_out: torch.Tensor, out: torch.Tensor, ws: torch.Tensor,
                          stream=None, **outs) -> None:
    so = _screen_out(**outs)
    _check(lib.eta_decode_sparse_predict(ctypes.byref(shape), ctypes.byref(params), _ptr(q), _ptr(k), _ptr(v),
                                         Meta(*(m.data_ptr() for m in meta)), n_tokens, _ptr(W), _ptr(bias),
                                         _ptr(tau_out), _ptr(out), ctypes.byref(so) if so is not None else None,
                                         _ptr(ws), ws.numel(), _stream(stream)), "eta_decode_sparse_predict")


def _thr(tau, W, bias, tau_out):
    """(tau, W, bias, tau_out) pointers of a per-row-length call."""
    if W is not None:
        return None, _ptr(W), _ptr(bias), _ptr(tau_out)
    return _ptr(tau), None, None, None


def screen_ragged(shape: Shape, params: Params, q, meta, seq_lens: torch.Tensor, max_tokens: int, ws: torch.Tensor,
                  tau: Optional[torch.Tensor] = None, tau_batch_stride: int = 0, W=None, bias=None, tau_out=None,
                  stream=None, **outs) -> None:
    so = _screen_out(**outs)
    t, w_, b_, to = _thr(tau, W, bias, tau_out)
    _check(lib.eta_screen_ragged(ctypes.byref(shape), ctypes.byref(params), _ptr(q),
                                 Meta(*(m.data_ptr() for m in meta)), _ptr(seq_lens), max_tokens, t,
                                 tau_batch_stride, w_, b_, to, ctypes.byref(so) if so is not None else None,
                                 _ptr(ws), ws.numel(), _stream(stream)), "eta_screen_ragged")


def decode_sparse_ragged(shape: Shape, params: Params, q, k, v, meta, seq_lens: torch.Tensor, max_tokens: int,
                         out: torch.Tensor, ws: torch.Tensor, tau: Optional[torch.Tensor] = None,
                         tau_batch_stride: int = 0, W=None, bias=None, tau_out=None, stream=None, **outs) -> None:
    so = _screen_out(**outs)
    t, w_, b_, to = _thr(tau, W, bias, tau_out)
    _check(lib.eta_decode_sparse_ragged(ctypes.byref(shape), ctypes.byref(params), _ptr(q), _ptr(k), _ptr(v),
                                        Meta(*(m.data_ptr() for m in meta)), _ptr(seq_lens), max_tokens, t,
                                        tau_batch_stride, w_, b_, to, _ptr(out),
                                        ctypes.byref(so) if so is not None else None, _ptr(ws), ws.numel(),
                                        _stream(stream)), "eta_decode_sparse_ragged")


def decode_screened_ragged(shape: Shape, params: Params, q, k, v, seq_lens: torch.Tensor, max_tokens: int,
                           tau: torch.Tensor, tau_batch_stride: int, out: torch.Tensor, ws: torch.Tensor,
                           stream=None) -> None:
    _check(lib.eta_decode_screened_ragged(ctypes.byref(shape), ctypes.byref(params), _ptr(q), _ptr(k), _ptr(v),
                                          _ptr(seq_lens), max_tokens, _ptr(tau), tau_batch_stride, _ptr(out),
                                          _ptr(ws), ws.numel(), _stream(stream)), "eta_decode_screened_ragged")


def decode_dense_ragged(shape: Shape, params: Params, q, k, v, seq_lens: torch.Tensor, max_tokens: int,
                        tau: Optional[torch.Tensor], tau_batch_stride: int, out: torch.Tensor, ws: torch.Tensor,
                        stream=None) -> None:
    _check(lib.eta_decode_dense_ragged(ctypes.byref(shape), ctypes.byref(params), _ptr(q), _ptr(k), _ptr(v),
                                       _ptr(seq_lens), max_tokens, _ptr(tau), tau_batch_stride, _ptr(out),
                                       _ptr(ws), ws.numel(), _stream(stream)), "eta_decode_dense_ragged")


def _pages(block_table: torch.Tensor, num_pages: int) -> Pages:
    return Pages(block_table.data_ptr(), num_pages)


def build_block_meta_paged(shape: Shape, k_pool: torch.Tensor, block_table: torch.Tensor, num_pages: int,
                           blk_begin: int, blk_end: int, mu, var, maxnorm, stream=None) -> None:
    _check(lib.eta_build_block_meta_paged(ctypes.byref(shape), _ptr(k_pool), _pages(block_table, num_pages),
                                          blk_begin, blk_end, Meta(mu.data_ptr(), var.data_ptr(), maxnorm.data_ptr()),
                                          _stream(stream)), "eta_build_block_meta_paged")


def decode_sparse_paged(shape: Shape, params: Params, q, k_pool, v_pool, block_table: torch.Tensor, num_pages: int,
                        meta, seq_lens: torch.Tensor, max_tokens: int, out: torch.Tensor, ws: torch.Tensor,
                        tau: Optional[torch.Tensor] = None, tau_batch_stride: int = 0, W=None, bias=None,
                        tau_out=None, stream=None, **outs) -> None:
    so = _screen_out(**outs)
    t, w_, b_, to = _thr(tau, W, bias, tau_out)
    _check(lib.eta_decode_sparse_paged(ctypes.byref(shape), ctypes.byref(params), _ptr(q), _ptr(k_pool),
                                       _ptr(v_pool), _pages(block_table, num_pages),
                                       Meta(*(m.data_ptr() for m in meta)), _ptr(seq_lens), max_tokens, t,
                                       tau_batch_stride, w_, b_, to, _ptr(out),
                                       ctypes.byref(so) if so is not None else None, _ptr(ws), ws.numel(),
                                       _stream(stream)), "eta_decode_sparse_paged")


def decode_screened_paged(shape: Shape, params: Params, q, k_pool, v_pool, block_table: torch.Tensor,
                          num_pages: int, seq_lens: torch.Tensor, max_tokens: int, tau: torch.Tensor,
                          tau_batch_stride: int, out: torch.Tensor, ws: torch.Tensor, stream=None) -> None:
    _check(lib.eta_decode_screened_paged(ctypes.byref(shape), ctypes.byref(params), _ptr(q), _ptr(k_pool),
                                         _ptr(v_pool), _pages(block_table, num_pages), _ptr(seq_lens), max_tokens,
                                         _ptr(tau), tau_batch_stride, _ptr(out), _ptr(ws), ws.numel(),
                                         _stream(stream)), "eta_decode_screened_paged")


def decode_dense_paged(shape: Shape, params: Params, q, k_pool, v_pool, block_table: torch.Tensor, num_pages: int,
                       seq_lens: torch.Tensor, max_tokens: int, tau: Optional[torch.Tensor], tau_batch_stride: int,
                       out: torch.Tensor, ws: torch.Tensor, stream=None) -> None:
    _check(lib.eta_decode_dense_paged(ctypes.byref(shape), ctypes.byref(params), _ptr(q), _ptr(k_pool),
                                      _ptr(v_pool), _pages(block_table, num_pages), _ptr(seq_lens), max_tokens,
                                      _ptr(tau), tau_batch_stride, _ptr(out), _ptr(ws), ws.numel(),
                                      _stream(stream)), "eta_decode_dense_paged")


def block_stats(shape: Shape, params: Params, q, k, n_tokens: int, tau: torch.Tensor, tau_batch_stride: int,
                block_max: torch.Tensor, above: torch.Tensor, block_lse: torch.Tensor, stream=None) -> None:
    _check(lib.eta_block_stats(ctypes.byref(shape), ctypes.byref(params), _ptr(q), _ptr(k), n_tokens, _ptr(tau),
                               tau_batch_stride, _ptr(block_max), _ptr(above), _ptr(block_lse), _stream(stream)),
           "eta_block_stats")


def decode_sparse(shape: Shape, params: Params, q, k, v, meta, n_tokens: int, tau: torch.Tensor,
                  tau_batch_stride: int, out: torch.Tensor, ws: torch.Tensor, stream=None, **outs) -> None:
    so = _screen_out(**outs)
    _check(lib.eta_decode_sparse(ctypes.byref(shape), ctypes.byref(params), _ptr(q), _ptr(k), _ptr(v),
                                 Meta(*(m.data_ptr() for m in meta)), n_tokens, _ptr(tau), tau_batch_stride,
                                 _ptr(out), ctypes.byref(so) if so is not None else None, _ptr(ws), ws.numel(),
                                 _stream(stream)), "eta_decode_sparse")


def decode_screened(shape: Shape, params: Params, q, k, v, n_tokens: int, tau: torch.Tensor,
                    tau_batch_stride: int, out: torch.Tensor, ws: torch.Tensor, stream=None) -> None:
    _check(lib.eta_decode_screened(ctypes.byref(shape), ctypes.byref(params), _ptr(q), _ptr(k), _ptr(v),
                                   n_tokens, _ptr(tau), tau_batch_stride, _ptr(out), _ptr(ws), ws.numel(),
                                   _stream(stream)), "eta_decode_screened")


def decode_dense(shape: Shape, params: Params, q, k, v, n_tokens: int, tau: Optional[torch.Tensor],
                 tau_batch_stride: int, out: torch.Tensor, ws: torch.Tensor, stream=None) -> None:
    _check(lib.eta_decode_dense(ctypes.byref(shape), ctypes.byref(params), _ptr(q), _ptr(k), _ptr(v), n_tokens,
                                _ptr(tau), tau_batch_stride, _ptr(out), _ptr(ws), ws.numel(), _stream(stream)),
           "eta_decode_dense")


def decode_sparse_static(shape: Shape, params: Params, q, k, v, meta, n_tokens: int, tau: torch.Tensor,
                         tau_batch_stride: int, out: torch.Tensor, device_status: Optional[torch.Tensor] = None,
                         stream=None, **outs) -> None:
    """eta_decode_sparse on the library's fixed device scratch: no workspace and
    no allocation (for callers that cannot allocate while decoding)."""
    so = _screen_out(**outs)
    _check(lib.eta_decode_sparse_static(ctypes.byref(shape), ctypes.byref(params), _ptr(q), _ptr(k), _ptr(v),
                                        Meta(*(m.data_ptr() for m in meta)), n_tokens, _ptr(tau), tau_batch_stride,
                                        _ptr(out), ctypes.byref(so) if so is not None else None,
                                        _ptr(device_status), _stream(stream)), "eta_decode_sparse_static")


def screen_diagnostics(shape: Shape, params: Params, n_tokens: int, tau: torch.Tensor, tau_batch_stride: int,
                       block_max: torch.Tensor, above: torch.Tensor, block_lse: torch.Tensor,
                       active_idx: torch.Tensor, active_cnt: torch.Tensor, per_head: torch.Tensor,
                       stream=None) -> None:
    _check(lib.eta_screen_diagnostics(ctypes.byref(shape), ctypes.byref(params), n_tokens, _ptr(tau),
                                      tau_batch_stride, _ptr(block_max), _ptr(above), _ptr(block_lse),
                                      _ptr(active_idx), _ptr(active_cnt), _ptr(per_head), _stream(stream)),
           "eta_screen_diagnostics")


def withhold_next_copy(position: int) -> None:
    """Test hook: the next decode launch leaves the copy of one admitted block
    (position `position` of the first thread block's range) unissued, so its
    bounded wait runs out and the call reports ETA_ERR_DEVICE_TIMEOUT."""
    _check(lib.eta_test_withhold_copy(position), "eta_test_withhold_copy")


def read_device_status(ws: torch.Tensor, stream=None) -> int:
    st = ctypes.c_int(0)
    _check(lib.eta_read_device_status(_ptr(ws), _stream(stream), ctypes.byref(st)), "eta_read_device_status")
    return st.value


class EtaDecoder:
    """One attention layer's decode state: the KV cache geometry, its block
    metadata and a workspace. ``step`` runs one decode step (predictor or given
    thresholds -> screen -> block-sparse decode) through the C ABI."""

    def __init__(self, batch, n_q_heads, n_kv_heads, head_dim, block_size, capacity,
                 kv_dtype=torch.bfloat16, q_dtype=torch.bfloat16, beta=5.0, z=1.0, offset_a=0.0,
                 n_local=1, n_splits=0, device="cuda", gate=GATE_SIGMOID, sub_blocks=1):
        self.shape = make_shape(batch, n_q_heads, n_kv_heads, head_dim, block_size, capacity, kv_dtype, q_dtype)
        self.params = make_params(beta, z, offset_a, n_local, n_splits, gate, sub_blocks)
        self.device = torch.device(device)
        # the sub-block envelope keeps metadata per sub-block of block_size / sub_blocks tokens
        self.sub_blocks = max(1, sub_blocks)
        self.meta_shape = make_shape(batch, n_q_heads, n_kv_heads, head_dim, block_size // self.sub_blocks, capacity,
                                     kv_dtype, q_dtype)
        nb_cap = capacity // block_size * self.sub_blocks
        f = dict(dtype=torch.float32, device=self.device)
        self.mu = torch.zeros((batch, n_kv_heads, head_dim, nb_cap), **f)
        self.var = torch.zeros((batch, n_kv_heads, head_dim, nb_cap), **f)
        self.maxnorm = torch.zeros((batch, n_kv_heads, nb_cap), **f)
        self.ws = alloc_workspace(self.shape, self.params, self.device)
        self.tau = torch.empty((batch, n_q_heads), **f)
        self.out = torch.empty((batch, n_q_heads, head_dim), **f)

    @property
    def meta(self):
        return (self.mu, self.var, self.maxnorm)

    def build_meta(self, k: torch.Tensor, blk_begin: int, blk_end: int) -> None:
        """Metadata of blocks [blk_begin, blk_end) (of every sub-block in them
        with the envelope)."""
        r = self.sub_blocks
        build_block_meta(self.meta_shape, k, blk_begin * r, blk_end * r, self.mu, self.var, self.maxnorm)

    def predict_tau(self, q: torch.Tensor, W: torch.Tensor, bias: torch.Tensor) -> torch.Tensor:
        predict_tau(self.shape, q, W, bias, self.tau)
        return self.tau

    def step(self, q, k, v, n_tokens: int, tau: Optional[torch.Tensor] = None, W=None, bias=None,
             tau_batch_stride: Optional[int] = None, out: Optional[torch.Tensor] = None,
             seq_lens: Optional[torch.Tensor] = None, **outs) -> torch.Tensor:
        """Sparse decode step. Thresholds: ``tau`` ([B][Hq], or [Hq] per-head
        constants) or the predictor (``W``, ``bias``), formed inside the
        screening launch and left in ``self.tau``. With ``seq_lens`` (int32
        [B] on the device) row b holds seq_lens[b] tokens and ``n_tokens`` is
        their upper bound."""
        o = self.out if out is None else out
        if tau is not None and tau_batch_stride is None:
            tau_batch_stride = 0 if tau.dim() == 1 else self.shape.n_q_heads
        if seq_lens is not None:
            if tau is None:
                decode_sparse_ragged(self.shape, self.params, q, k, v, self.meta, seq_lens, n_tokens, o, self.ws,
                                     W=W, bias=bias, tau_out=self.tau, **outs)
            else:
                decode_sparse_ragged(self.shape, self.params, q, k, v, self.meta, seq_lens, n_tokens, o, self.ws,
                                     tau=tau, tau_batch_stride=tau_batch_stride, **outs)
            return o
        if tau is None:
            decode_sparse_predict(self.shape, self.params, q, k, v, self.meta, n_tokens, W, bias, self.tau, o,
                                  self.ws, **outs)
            return o
        decode_sparse(self.shape, self.params, q, k, v, self.meta, n_tokens, tau, tau_batch_stride, o, self.ws,
                      **outs)
        return o

    def dense(self, q, k, v, n_tokens: int, tau: Optional[torch.Tensor] = None,
              tau_batch_stride: Optional[int] = None, out: Optional[torch.Tensor] = None,
              seq_lens: Optional[torch.Tensor] = None) -> torch.Tensor:
        if tau is not None and tau_batch_stride is None:
            tau_batch_stride = 0 if tau.dim() == 1 else self.shape.n_q_heads
        o = self.out if out is None else out
        if seq_lens is not None:
            decode_dense_ragged(self.shape, self.params, q, k, v, seq_lens, n_tokens, tau, tau_batch_stride or 0, o,
                                self.ws)
        else:
            decode_dense(self.shape, self.params, q, k, v, n_tokens, tau, tau_batch_stride or 0, o, self.ws)
        return o

    def device_status(self) -> int:
        return read_device_status(self.ws)

// C-ABI entry points of libeta.so (declared in include/eta.h): host-side
// validation, workspace carving and dispatch to the kernel launchers.
#include <atomic>
#include <climits>
#include <cmath>
#include <cstdint>
#include <cstring>

#include <cuda_runtime.h>

#include "eta.h"
#include "launch.h"

namespace eta {

namespace {

constexpr size_t kAlign = 256;

size_t round_up(size_t x) { return (x + kAlign - 1) / kAlign * kAlign; }

constexpr int kMaxDevices = 64;
std::atomic<int> g_sm_count[kMaxDevices];
std::atomic<int> g_smem_optin[kMaxDevices];

int current_device() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 0;
  return dev & (kMaxDevices - 1);
}

}  // namespace

int device_sm_count() {
  const int dev = current_device();
  int v = g_sm_count[dev].load(std::memory_order_relaxed);
  if (v <= 0) {
    if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || v <= 0) v = 1;
    g_sm_count[dev].store(v, std::memory_order_relaxed);
  }
  return v;
}

int device_max_smem_optin() {
  const int dev = current_device();
  int v = g_smem_optin[dev].load(std::memory_order_relaxed);
  if (v <= 0) {
    if (cudaDeviceGetAttribute(&v, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) != cudaSuccess || v <= 0)
      v = 48 * 1024;
    g_smem_optin[dev].store(v, std::memory_order_relaxed);
  }
  return v;
}

WsLayout ws_layout(int B, int Hq, int Hkv, int d, int64_t nb_cap, int S) {
  WsLayout L;
  const size_t BH = static_cast<size_t>(B) * Hkv, BHq = static_cast<size_t>(B) * Hq;
  size_t off = 0;
  L.status = off;     off += 256;
  L.seg_done = off;   off += round_up(kMaxBH * sizeof(int32_t));
  L.union_list = off; off += round_up(BH * static_cast<size_t>(nb_cap) * sizeof(uint32_t));
  L.union_cnt = off;  off += round_up(BH * sizeof(int32_t));
  L.head_cnt = off;   off += round_up(BHq * sizeof(int32_t));
  L.o_part = off;     off += round_up(BHq * static_cast<size_t>(S) * d * sizeof(float));
  L.ml_part = off;    off += round_up(BHq * static_cast<size_t>(S) * sizeof(float2));
  L.total = off;
  return L;
}

Workspace ws_carve(void* base, const WsLayout& L) {
  unsigned char* p = static_cast<unsigned char*>(base);
  Workspace w;
  w.status = reinterpret_cast<int32_t*>(p + L.status);
  w.union_list = reinterpret_cast<uint32_t*>(p + L.union_list);
  w.union_cnt = reinterpret_cast<int32_t*>(p + L.union_cnt);
  w.head_cnt = reinterpret_cast<int32_t*>(p + L.head_cnt);
  w.seg_done = reinterpret_cast<int32_t*>(p + L.seg_done);
  w.o_part = reinterpret_cast<float*>(p + L.o_part);
  w.ml_part = reinterpret_cast<float2*>(p + L.ml_part);
  return w;
}

}  // namespace eta

using namespace eta;

namespace {

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

int elem_bytes(int dtype) { return dtype == ETA_FP8_E4M3 ? 1 : (dtype == ETA_BF16 ? 2 : 4); }

eta_status_t check_shape(const eta_shape_t* s) {
  if (s == nullptr) return ETA_ERR_INVALID_ARG;
  if (s->batch < 1 || s->n_q_heads < 1 || s->n_kv_heads < 1 || s->head_dim < 1 || s->block_size < 1)
    return ETA_ERR_INVALID_ARG;
  if (s->kv_dtype != ETA_F32 && s->kv_dtype != ETA_BF16 && s->kv_dtype != ETA_FP8_E4M3) return ETA_ERR_INVALID_ARG;
  if (s->q_dtype != ETA_F32 && s->q_dtype != ETA_BF16) return ETA_ERR_INVALID_ARG;
  // fp8 K/V run on the tensor-core decode only: bf16 queries, d = 128
  if (s->kv_dtype == ETA_FP8_E4M3 && (s->q_dtype != ETA_BF16 || s->head_dim != 128)) return ETA_ERR_UNSUPPORTED;
  if (s->n_q_heads % s->n_kv_heads != 0) return ETA_ERR_INVALID_ARG;
  if (s->capacity <= 0 || s->capacity % s->block_size != 0) return ETA_ERR_INVALID_ARG;
  if (s->head_dim != 64 && s->head_dim != 128) return ETA_ERR_UNSUPPORTED;
  const int bs = s->block_size;
  if (bs != 16 && bs != 32 && bs != 64 && bs != 128) return ETA_ERR_UNSUPPORTED;
  const int G = s->n_q_heads / s->n_kv_heads;
  if (G != 1 && G != 2 && G != 4 && G != 8) return ETA_ERR_UNSUPPORTED;
  const int64_t nb_cap = s->capacity / bs;
  if (nb_cap >= (int64_t{1} << 24)) return ETA_ERR_UNSUPPORTED;
  if (static_cast<int64_t>(s->batch) * s->n_q_heads * nb_cap >= (int64_t{1} << 31)) return ETA_ERR_UNSUPPORTED;
  return ETA_OK;
}

eta_status_t check_params(const eta_params_t* p) {
  if (p == nullptr) return ETA_ERR_INVALID_ARG;
  if (!(p->beta > 0.0f) || !std::isfinite(p->beta)) return ETA_ERR_INVALID_ARG;
  if (!std::isfinite(p->z) || !std::isfinite(p->offset_a)) return ETA_ERR_INVALID_ARG;
  if (p->n_local < 1 || p->n_splits < 0) return ETA_ERR_INVALID_ARG;
  if (p->gate != ETA_GATE_SIGMOID && p->gate != ETA_GATE_HARD) return ETA_ERR_INVALID_ARG;
  if (p->sub_blocks != 0 && p->sub_blocks != 1 && p->sub_blocks != 2 && p->sub_blocks != 4 && p->sub_blocks != 8)
    return ETA_ERR_INVALID_ARG;
  return ETA_OK;
}

int sub_blocks_of(const eta_params_t* p) { return p->sub_blocks > 1 ? p->sub_blocks : 1; }

// The envelope's sub-blocks must be blocks the metadata builder supports.
eta_status_t check_sub_blocks(const eta_shape_t* s, const eta_params_t* p, bool paged) {
  const int r = sub_blocks_of(p);
  if (r == 1) return ETA_OK;
  if (paged || s->block_size / r < 16) return ETA_ERR_UNSUPPORTED;
  return ETA_OK;
}

// Store rows (token rows of the K cache or pool) that a kernel addresses with
// a 32-bit row index: the metadata builder's block rows, like the decode's.
eta_status_t check_store_rows(const eta_shape_t* s, int64_t pool_pages) {
  const int64_t rows = pool_pages > 0 ? pool_pages * s->n_kv_heads * s->block_size
                                      : static_cast<int64_t>(s->batch) * s->n_kv_heads * s->capacity;
  return rows > static_cast<int64_t>(INT32_MAX) ? ETA_ERR_UNSUPPORTED : ETA_OK;
}

// Shapes the decode kernel can stage (two stages of a K and a V block plus its
// fixed shared memory) and index (prefix table and partial counters of B*Hkv
// entries).
eta_status_t check_decode_shape(const eta_shape_t* s, bool dense, int64_t pool_pages = 0) {
  (void)dense;  // both passes keep the same segment table
  const int BH = s->batch * s->n_kv_heads;
  if (BH > kMaxBH) return ETA_ERR_UNSUPPORTED;
  const int G = s->n_q_heads / s->n_kv_heads;
  const size_t tile = static_cast<size_t>(s->block_size) * s->head_dim * elem_bytes(s->kv_dtype);
  const size_t fixed = static_cast<size_t>(8) * G * (s->head_dim + 2) * 4 + 16 + 64 +
                       static_cast<size_t>(BH + 1) * 4 + 64;
  const size_t need = 2 * (2 * tile + 32) + fixed;
  if (need + 1024 > static_cast<size_t>(device_max_smem_optin())) return ETA_ERR_UNSUPPORTED;
  // the kernels address store rows with 32-bit integers (TMA coordinates too)
  return check_store_rows(s, pool_pages);
}

// A paged pool: a block table and at least one page.
eta_status_t check_pages(const eta_pages_t& pg) {
  if (pg.block_table == nullptr || !aligned(pg.block_table, 4) || pg.num_pages < 1) return ETA_ERR_INVALID_ARG;
  return ETA_OK;
}

eta_status_t check_screen_shape(const eta_shape_t* s) {
  const int64_t nb_cap = s->capacity / s->block_size;
  if (nb_cap > static_cast<int64_t>(kMaxCluster) * kMaxScreenTiles * 32) return ETA_ERR_UNSUPPORTED;
  return ETA_OK;
}

int resolve_splits(const eta_params_t* p) { return p->n_splits > 0 ? p->n_splits : device_sm_count(); }

eta_status_t from_cuda(cudaError_t e) { return e == cudaSuccess ? ETA_OK : ETA_ERR_CUDA; }

eta_status_t check_workspace(const eta_shape_t* s, const eta_params_t* p, void* ws, size_t ws_bytes,
                             WsLayout* L) {
  if (ws == nullptr || !aligned(ws, 256)) return ETA_ERR_WORKSPACE;
  *L = ws_layout(s->batch, s->n_q_heads, s->n_kv_heads, s->head_dim, s->capacity / s->block_size,
                 resolve_splits(p));
  if (ws_bytes < L->total) return ETA_ERR_WORKSPACE;
  return ETA_OK;
}

eta_status_t check_tokens(const eta_shape_t* s, int64_t n) {
  if (n < 1 || n > s->capacity) return ETA_ERR_INVALID_ARG;
  return ETA_OK;
}

eta_status_t check_meta(const eta_meta_t& m) {
  if (m.mu == nullptr || m.var == nullptr || m.maxnorm == nullptr) return ETA_ERR_INVALID_ARG;
  if (!aligned(m.mu, 4) || !aligned(m.var, 4) || !aligned(m.maxnorm, 4)) return ETA_ERR_INVALID_ARG;
  return ETA_OK;
}

#define ETA_TRY(x)                      \
  do {                                  \
    const eta_status_t st_ = (x);       \
    if (st_ != ETA_OK) return st_;      \
  } while (0)

eta_status_t do_screen(const eta_shape_t* s, const eta_params_t* p, const void* q, eta_meta_t meta, int64_t n,
                       const float* tau, int64_t tau_stride, const eta_screen_out_t* out, const Workspace& w,
                       cudaStream_t st, const float* W = nullptr, const float* bias = nullptr,
                       float* tau_out = nullptr, const int32_t* seq_lens = nullptr) {
  ETA_TRY(check_sub_blocks(s, p, false));
  ScreenCall c;
  c.seq_lens = seq_lens;
  c.shape = *s;
  c.z = p->z;
  c.offset_a = p->offset_a;
  c.n_local = p->n_local;
  c.sub_blocks = sub_blocks_of(p);
  c.q = q;
  c.meta = meta;
  c.n = n;
  c.tau = tau;
  c.tau_stride = tau_stride;
  c.W = W;
  c.bias = bias;
  c.tau_out = tau_out;
  if (out != nullptr) c.out = *out;
  else std::memset(&c.out, 0, sizeof(c.out));
  c.ws = w;
  return from_cuda(launch_screen(c, st));
}

eta_status_t check_common_decode(const eta_shape_t* s, const eta_params_t* p, const void* q, const void* k,
                                 const void* v, int64_t n, float* out) {
  ETA_TRY(check_shape(s));
  ETA_TRY(check_params(p));
  ETA_TRY(check_tokens(s, n));
  if (q == nullptr || k == nullptr || v == nullptr || out == nullptr) return ETA_ERR_INVALID_ARG;
  if (!aligned(k, 16) || !aligned(v, 16) || !aligned(q, elem_bytes(s->q_dtype)) || !aligned(out, 16))
    return ETA_ERR_INVALID_ARG;
  return ETA_OK;
}

// Test hook of the device-timeout path (eta_test_withhold_copy): the position
// the next decode launch leaves unarmed, -1 for none.
std::atomic<int64_t> g_withhold{-1};

eta_status_t do_decode(const eta_shape_t* s, const eta_params_t* p, const void* q, const void* k, const void* v,
                       int64_t n, const float* tau, int64_t tau_stride, float* out, const Workspace& w,
                       cudaStream_t st, bool dense, const int32_t* seq_lens = nullptr,
                       const eta_pages_t* pages = nullptr) {
  DecodeCall c;
  c.block_table = pages ? pages->block_table : nullptr;
  c.num_pages = pages ? pages->num_pages : 0;
  c.shape = *s;
  c.beta = p->beta;
  c.gate = p->gate;
  c.q = q;
  c.k = k;
  c.v = v;
  c.n = n;
  c.seq_lens = seq_lens;
  c.tau = tau;
  c.tau_stride = tau_stride;
  c.out = out;
  c.ws = w;
  c.S = resolve_splits(p);
  c.dense = dense;
  c.withhold = g_withhold.exchange(-1);
  return from_cuda(launch_decode(c, st));
}

eta_status_t do_sparse_decode(const eta_shape_t* s, const eta_params_t* p, const void* q, const void* k,
                              const void* v, int64_t n, const float* tau, int64_t tau_stride, float* out,
                              const Workspace& w, cudaStream_t st) {
  return do_decode(s, p, q, k, v, n, tau, tau_stride, out, w, st, false);
}

eta_status_t check_predictor(const eta_shape_t* s, const void* q, const float* W, const float* bias,
                             const float* tau);

eta_status_t check_lens(const int32_t* seq_lens) {
  if (seq_lens == nullptr || !aligned(seq_lens, 4)) return ETA_ERR_INVALID_ARG;
  return ETA_OK;
}

// Thresholds of a per-row-length call: given (tau, stride) when W is null,
// else formed by Eq. 1 into tau_out.
eta_status_t check_thresholds(const eta_shape_t* s, const void* q, const float* tau, int64_t tau_stride,
                              const float* W, const float* bias, const float* tau_out) {
  if (W != nullptr) return check_predictor(s, q, W, bias, tau_out);
  if (tau == nullptr || tau_stride < 0 || !aligned(tau, 4)) return ETA_ERR_INVALID_ARG;
  return ETA_OK;
}

eta_status_t check_predictor(const eta_shape_t* s, const void* q, const float* W, const float* bias,
                             const float* tau) {
  if (q == nullptr || W == nullptr || bias == nullptr || tau == nullptr) return ETA_ERR_INVALID_ARG;
  if (!aligned(q, elem_bytes(s->q_dtype)) || !aligned(W, 4) || !aligned(bias, 4) || !aligned(tau, 4))
    return ETA_ERR_INVALID_ARG;
  return ETA_OK;
}

}  // namespace

extern "C" {

ETA_API int eta_abi_version(void) { return ETA_ABI_VERSION; }

ETA_API const char* eta_status_string(eta_status_t status) {
  switch (status) {
    case ETA_OK: return "ok";
    case ETA_ERR_INVALID_ARG: return "invalid argument";
    case ETA_ERR_UNSUPPORTED: return "unsupported shape";
    case ETA_ERR_WORKSPACE: return "workspace missing, misaligned or too small";
    case ETA_ERR_CUDA: return "CUDA error";
    case ETA_ERR_DEVICE_TIMEOUT: return "device-side wait timed out";
  }
  return "unknown status";
}

ETA_API eta_status_t eta_build_block_meta(const eta_shape_t* shape, const void* k, int64_t blk_begin,
                                          int64_t blk_end, eta_meta_t meta, eta_stream_t stream) {
  ETA_TRY(check_shape(shape));
  ETA_TRY(check_meta(meta));
  ETA_TRY(check_store_rows(shape, 0));
  if (k == nullptr || !aligned(k, 16)) return ETA_ERR_INVALID_ARG;
  const int64_t nb_cap = shape->capacity / shape->block_size;
  if (blk_begin < 0 || blk_end > nb_cap || blk_begin > blk_end) return ETA_ERR_INVALID_ARG;
  if (blk_begin == blk_end) return ETA_OK;
  return from_cuda(launch_build_meta(*shape, k, blk_begin, blk_end, meta, stream));
}

ETA_API eta_status_t eta_predict_tau(const eta_shape_t* shape, const void* q, const float* W, const float* bias,
                                     float* tau, eta_stream_t stream) {
  ETA_TRY(check_shape(shape));
  ETA_TRY(check_predictor(shape, q, W, bias, tau));
  return from_cuda(launch_predict(*shape, q, W, bias, tau, stream));
}

ETA_API size_t eta_decode_workspace_bytes(const eta_shape_t* shape, const eta_params_t* params) {
  if (check_shape(shape) != ETA_OK || check_params(params) != ETA_OK) return 0;
  return ws_layout(shape->batch, shape->n_q_heads, shape->n_kv_heads, shape->head_dim,
                   shape->capacity / shape->block_size, resolve_splits(params))
      .total;
}

ETA_API eta_status_t eta_workspace_init(void* workspace, size_t ws_bytes, eta_stream_t stream) {
  if (workspace == nullptr || !aligned(workspace, 256) || ws_bytes < kWsHeaderBytes) return ETA_ERR_WORKSPACE;
  return from_cuda(cudaMemsetAsync(workspace, 0, kWsHeaderBytes, stream));
}

ETA_API eta_status_t eta_screen(const eta_shape_t* shape, const eta_params_t* params, const void* q,
                                eta_meta_t meta, int64_t n_tokens, const float* tau, int64_t tau_batch_stride,
                                const eta_screen_out_t* out, void* workspace, size_t ws_bytes,
                                eta_stream_t stream) {
  ETA_TRY(check_shape(shape));
  ETA_TRY(check_params(params));
  ETA_TRY(check_tokens(shape, n_tokens));
  ETA_TRY(check_screen_shape(shape));
  ETA_TRY(check_meta(meta));
  if (q == nullptr || tau == nullptr || tau_batch_stride < 0) return ETA_ERR_INVALID_ARG;
  if (!aligned(q, elem_bytes(shape->q_dtype)) || !aligned(tau, 4)) return ETA_ERR_INVALID_ARG;
  WsLayout L;
  ETA_TRY(check_workspace(shape, params, workspace, ws_bytes, &L));
  return do_screen(shape, params, q, meta, n_tokens, tau, tau_batch_stride, out, ws_carve(workspace, L), stream);
}

ETA_API eta_status_t eta_decode_sparse(const eta_shape_t* shape, const eta_params_t* params, const void* q,
                                       const void* k, const void* v, eta_meta_t meta, int64_t n_tokens,
                                       const float* tau, int64_t tau_batch_stride, float* out,
                                       const eta_screen_out_t* extra, void* workspace, size_t ws_bytes,
                                       eta_stream_t stream) {
  ETA_TRY(check_common_decode(shape, params, q, k, v, n_tokens, out));
  ETA_TRY(check_screen_shape(shape));
  ETA_TRY(check_decode_shape(shape, false));
  ETA_TRY(check_meta(meta));
  if (tau == nullptr || tau_batch_stride < 0 || !aligned(tau, 4)) return ETA_ERR_INVALID_ARG;
  WsLayout L;
  ETA_TRY(check_workspace(shape, params, workspace, ws_bytes, &L));
  const Workspace w = ws_carve(workspace, L);
  ETA_TRY(do_screen(shape, params, q, meta, n_tokens, tau, tau_batch_stride, extra, w, stream));
  return do_sparse_decode(shape, params, q, k, v, n_tokens, tau, tau_batch_stride, out, w, stream);
}

ETA_API eta_status_t eta_screen_predict(const eta_shape_t* shape, const eta_params_t* params, const void* q,
                                        eta_meta_t meta, int64_t n_tokens, const float* W, const float* bias,
                                        float* tau_out, const eta_screen_out_t* out, void* workspace,
                                        size_t ws_bytes, eta_stream_t stream) {
  ETA_TRY(check_shape(shape));
  ETA_TRY(check_params(params));
  ETA_TRY(check_tokens(shape, n_tokens));
  ETA_TRY(check_screen_shape(shape));
  ETA_TRY(check_meta(meta));
  ETA_TRY(check_predictor(shape, q, W, bias, tau_out));
  WsLayout L;
  ETA_TRY(check_workspace(shape, params, workspace, ws_bytes, &L));
  return do_screen(shape, params, q, meta, n_tokens, nullptr, 0, out, ws_carve(workspace, L), stream, W, bias,
                   tau_out);
}

ETA_API eta_status_t eta_decode_sparse_predict(const eta_shape_t* shape, const eta_params_t* params, const void* q,
                                               const void* k, const void* v, eta_meta_t meta, int64_t n_tokens,
                                               const float* W, const float* bias, float* tau_out, float* out,
                                               const eta_screen_out_t* extra, void* workspace, size_t ws_bytes,
                                               eta_stream_t stream) {
  ETA_TRY(check_common_decode(shape, params, q, k, v, n_tokens, out));
  ETA_TRY(check_screen_shape(shape));
  ETA_TRY(check_decode_shape(shape, false));
  ETA_TRY(check_meta(meta));
  ETA_TRY(check_predictor(shape, q, W, bias, tau_out));
  WsLayout L;
  ETA_TRY(check_workspace(shape, params, workspace, ws_bytes, &L));
  const Workspace w = ws_carve(workspace, L);
  ETA_TRY(do_screen(shape, params, q, meta, n_tokens, nullptr, 0, extra, w, stream, W, bias, tau_out));
  return do_sparse_decode(shape, params, q, k, v, n_tokens, tau_out, shape->n_q_heads, out, w, stream);
}

ETA_API eta_status_t eta_decode_screened(const eta_shape_t* shape, const eta_params_t* params, const void* q,
                                         const void* k, const void* v, int64_t n_tokens, const float* tau,
                                         int64_t tau_batch_stride, float* out, void* workspace, size_t ws_bytes,
                                         eta_stream_t stream) {
  ETA_TRY(check_common_decode(shape, params, q, k, v, n_tokens, out));
  ETA_TRY(check_decode_shape(shape, false));
  if (tau == nullptr || tau_batch_stride < 0 || !aligned(tau, 4)) return ETA_ERR_INVALID_ARG;
  WsLayout L;
  ETA_TRY(check_workspace(shape, params, workspace, ws_bytes, &L));
  return do_sparse_decode(shape, params, q, k, v, n_tokens, tau, tau_batch_stride, out, ws_carve(workspace, L),
                          stream);
}

ETA_API eta_status_t eta_decode_dense(const eta_shape_t* shape, const eta_params_t* params, const void* q,
                                      const void* k, const void* v, int64_t n_tokens, const float* tau,
                                      int64_t tau_batch_stride, float* out, void* workspace, size_t ws_bytes,
                                      eta_stream_t stream) {
  ETA_TRY(check_common_decode(shape, params, q, k, v, n_tokens, out));
  ETA_TRY(check_decode_shape(shape, true));
  if (tau != nullptr && (tau_batch_stride < 0 || !aligned(tau, 4))) return ETA_ERR_INVALID_ARG;
  WsLayout L;
  ETA_TRY(check_workspace(shape, params, workspace, ws_bytes, &L));
  return do_decode(shape, params, q, k, v, n_tokens, tau, tau_batch_stride, out, ws_carve(workspace, L), stream,
                   true);
}

ETA_API eta_status_t eta_screen_ragged(const eta_shape_t* shape, const eta_params_t* params, const void* q,
                                       eta_meta_t meta, const int32_t* seq_lens, int64_t max_tokens,
                                       const float* tau, int64_t tau_batch_stride, const float* W,
                                       const float* bias, float* tau_out, const eta_screen_out_t* out,
                                       void* workspace, size_t ws_bytes, eta_stream_t stream) {
  ETA_TRY(check_shape(shape));
  ETA_TRY(check_params(params));
  ETA_TRY(check_tokens(shape, max_tokens));
  ETA_TRY(check_lens(seq_lens));
  ETA_TRY(check_screen_shape(shape));
  ETA_TRY(check_meta(meta));
  if (q == nullptr || !aligned(q, elem_bytes(shape->q_dtype))) return ETA_ERR_INVALID_ARG;
  ETA_TRY(check_thresholds(shape, q, tau, tau_batch_stride, W, bias, tau_out));
  WsLayout L;
  ETA_TRY(check_workspace(shape, params, workspace, ws_bytes, &L));
  return do_screen(shape, params, q, meta, max_tokens, W ? nullptr : tau, W ? 0 : tau_batch_stride, out,
                   ws_carve(workspace, L), stream, W, bias, tau_out, seq_lens);
}

ETA_API eta_status_t eta_decode_sparse_ragged(const eta_shape_t* shape, const eta_params_t* params, const void* q,
                                              const void* k, const void* v, eta_meta_t meta,
                                              const int32_t* seq_lens, int64_t max_tokens, const float* tau,
                                              int64_t tau_batch_stride, const float* W, const float* bias,
                                              float* tau_out, float* out, const eta_screen_out_t* extra,
                                              void* workspace, size_t ws_bytes, eta_stream_t stream) {
  ETA_TRY(check_common_decode(shape, params, q, k, v, max_tokens, out));
  ETA_TRY(check_lens(seq_lens));
  ETA_TRY(check_screen_shape(shape));
  ETA_TRY(check_decode_shape(shape, false));
  ETA_TRY(check_meta(meta));
  ETA_TRY(check_thresholds(shape, q, tau, tau_batch_stride, W, bias, tau_out));
  WsLayout L;
  ETA_TRY(check_workspace(shape, params, workspace, ws_bytes, &L));
  const Workspace w = ws_carve(workspace, L);
  const float* t = W ? tau_out : tau;
  const int64_t ts = W ? shape->n_q_heads : tau_batch_stride;
  ETA_TRY(do_screen(shape, params, q, meta, max_tokens, W ? nullptr : tau, W ? 0 : tau_batch_stride, extra, w,
                    stream, W, bias, tau_out, seq_lens));
  return do_decode(shape, params, q, k, v, max_tokens, t, ts, out, w, stream, false, seq_lens);
}

ETA_API eta_status_t eta_decode_screened_ragged(const eta_shape_t* shape, const eta_params_t* params,
                                                const void* q, const void* k, const void* v,
                                                const int32_t* seq_lens, int64_t max_tokens, const float* tau,
                                                int64_t tau_batch_stride, float* out, void* workspace,
                                                size_t ws_bytes, eta_stream_t stream) {
  ETA_TRY(check_common_decode(shape, params, q, k, v, max_tokens, out));
  ETA_TRY(check_lens(seq_lens));
  ETA_TRY(check_decode_shape(shape, false));
  if (tau == nullptr || tau_batch_stride < 0 || !aligned(tau, 4)) return ETA_ERR_INVALID_ARG;
  WsLayout L;
  ETA_TRY(check_workspace(shape, params, workspace, ws_bytes, &L));
  return do_decode(shape, params, q, k, v, max_tokens, tau, tau_batch_stride, out, ws_carve(workspace, L), stream,
                   false, seq_lens);
}

ETA_API eta_status_t eta_decode_dense_ragged(const eta_shape_t* shape, const eta_params_t* params, const void* q,
                                             const void* k, const void* v, const int32_t* seq_lens,
                                             int64_t max_tokens, const float* tau, int64_t tau_batch_stride,
                                             float* out, void* workspace, size_t ws_bytes, eta_stream_t stream) {
  ETA_TRY(check_common_decode(shape, params, q, k, v, max_tokens, out));
  ETA_TRY(check_lens(seq_lens));
  ETA_TRY(check_decode_shape(shape, true));
  if (tau != nullptr && (tau_batch_stride < 0 || !aligned(tau, 4))) return ETA_ERR_INVALID_ARG;
  WsLayout L;
  ETA_TRY(check_workspace(shape, params, workspace, ws_bytes, &L));
  return do_decode(shape, params, q, k, v, max_tokens, tau, tau_batch_stride, out, ws_carve(workspace, L), stream,
                   true, seq_lens);
}

ETA_API eta_status_t eta_read_device_status(const void* workspace, eta_stream_t stream, eta_status_t* status) {
  if (workspace == nullptr || status == nullptr) return ETA_ERR_INVALID_ARG;
  int32_t v = 0;
  cudaError_t e = cudaMemcpyAsync(&v, workspace, sizeof(v), cudaMemcpyDeviceToHost, stream);
  if (e == cudaSuccess) e = cudaStreamSynchronize(stream);
  if (e != cudaSuccess) return ETA_ERR_CUDA;
  // After a device error a call may have stopped between counting partials:
  // clear the counters too.
  e = cudaMemsetAsync(const_cast<void*>(workspace), 0, v == 0 ? sizeof(int32_t) : kWsHeaderBytes, stream);
  if (e != cudaSuccess) return ETA_ERR_CUDA;
  *status = static_cast<eta_status_t>(v);
  return ETA_OK;
}

ETA_API eta_status_t eta_build_block_meta_paged(const eta_shape_t* shape, const void* k_pool, eta_pages_t pages,
                                                int64_t blk_begin, int64_t blk_end, eta_meta_t meta,
                                                eta_stream_t stream) {
  ETA_TRY(check_shape(shape));
  ETA_TRY(check_meta(meta));
  ETA_TRY(check_pages(pages));
  ETA_TRY(check_store_rows(shape, pages.num_pages));
  if (k_pool == nullptr || !aligned(k_pool, 16)) return ETA_ERR_INVALID_ARG;
  const int64_t nb_cap = shape->capacity / shape->block_size;
  if (blk_begin < 0 || blk_end > nb_cap || blk_begin > blk_end) return ETA_ERR_INVALID_ARG;
  if (blk_begin == blk_end) return ETA_OK;
  return from_cuda(
      launch_build_meta(*shape, k_pool, blk_begin, blk_end, meta, stream, pages.block_table, pages.num_pages));
}

ETA_API eta_status_t eta_decode_sparse_paged(const eta_shape_t* shape, const eta_params_t* params, const void* q,
                                             const void* k_pool, const void* v_pool, eta_pages_t pages,
                                             eta_meta_t meta, const int32_t* seq_lens, int64_t max_tokens,
                                             const float* tau, int64_t tau_batch_stride, const float* W,
                                             const float* bias, float* tau_out, float* out,
                                             const eta_screen_out_t* extra, void* workspace, size_t ws_bytes,
                                             eta_stream_t stream) {
  ETA_TRY(check_common_decode(shape, params, q, k_pool, v_pool, max_tokens, out));
  ETA_TRY(check_sub_blocks(shape, params, true));
  ETA_TRY(check_pages(pages));
  ETA_TRY(check_lens(seq_lens));
  ETA_TRY(check_screen_shape(shape));
  ETA_TRY(check_decode_shape(shape, false, pages.num_pages));
  ETA_TRY(check_meta(meta));
  ETA_TRY(check_thresholds(shape, q, tau, tau_batch_stride, W, bias, tau_out));
  WsLayout L;
  ETA_TRY(check_workspace(shape, params, workspace, ws_bytes, &L));
  const Workspace w = ws_carve(workspace, L);
  const float* t = W ? tau_out : tau;
  const int64_t ts = W ? shape->n_q_heads : tau_batch_stride;
  ETA_TRY(do_screen(shape, params, q, meta, max_tokens, W ? nullptr : tau, W ? 0 : tau_batch_stride, extra, w,
                    stream, W, bias, tau_out, seq_lens));
  return do_decode(shape, params, q, k_pool, v_pool, max_tokens, t, ts, out, w, stream, false, seq_lens, &pages);
}

ETA_API eta_status_t eta_decode_screened_paged(const eta_shape_t* shape, const eta_params_t* params, const void* q,
                                               const void* k_pool, const void* v_pool, eta_pages_t pages,
                                               const int32_t* seq_lens, int64_t max_tokens, const float* tau,
                                               int64_t tau_batch_stride, float* out, void* workspace,
                                               size_t ws_bytes, eta_stream_t stream) {
  ETA_TRY(check_common_decode(shape, params, q, k_pool, v_pool, max_tokens, out));
  ETA_TRY(check_pages(pages));
  ETA_TRY(check_lens(seq_lens));
  ETA_TRY(check_decode_shape(shape, false, pages.num_pages));
  if (tau == nullptr || tau_batch_stride < 0 || !aligned(tau, 4)) return ETA_ERR_INVALID_ARG;
  WsLayout L;
  ETA_TRY(check_workspace(shape, params, workspace, ws_bytes, &L));
  return do_decode(shape, params, q, k_pool, v_pool, max_tokens, tau, tau_batch_stride, out, ws_carve(workspace, L),
                   stream, false, seq_lens, &pages);
}

ETA_API eta_status_t eta_decode_dense_paged(const eta_shape_t* shape, const eta_params_t* params, const void* q,
                                            const void* k_pool, const void* v_pool, eta_pages_t pages,
                                            const int32_t* seq_lens, int64_t max_tokens, const float* tau,
                                            int64_t tau_batch_stride, float* out, void* workspace, size_t ws_bytes,
                                            eta_stream_t stream) {
  ETA_TRY(check_common_decode(shape, params, q, k_pool, v_pool, max_tokens, out));
  ETA_TRY(check_pages(pages));
  ETA_TRY(check_lens(seq_lens));
  ETA_TRY(check_decode_shape(shape, true, pages.num_pages));
  if (tau != nullptr && (tau_batch_stride < 0 || !aligned(tau, 4))) return ETA_ERR_INVALID_ARG;
  WsLayout L;
  ETA_TRY(check_workspace(shape, params, workspace, ws_bytes, &L));
  return do_decode(shape, params, q, k_pool, v_pool, max_tokens, tau, tau_batch_stride, out, ws_carve(workspace, L),
                   stream, true, seq_lens, &pages);
}

ETA_API eta_status_t eta_screen_diagnostics(const eta_shape_t* shape, const eta_params_t* params, int64_t n_tokens,
                                            const float* tau, int64_t tau_batch_stride, const float* block_max,
                                            const int32_t* above, const float* block_lse, const int32_t* active_idx,
                                            const int32_t* active_cnt, double* per_head, eta_stream_t stream) {
  ETA_TRY(check_shape(shape));
  ETA_TRY(check_params(params));
  ETA_TRY(check_tokens(shape, n_tokens));
  if (tau == nullptr || tau_batch_stride < 0 || block_max == nullptr || above == nullptr || block_lse == nullptr ||
      active_idx == nullptr || active_cnt == nullptr || per_head == nullptr)
    return ETA_ERR_INVALID_ARG;
  if (!aligned(tau, 4) || !aligned(block_max, 4) || !aligned(above, 4) || !aligned(block_lse, 4) ||
      !aligned(active_idx, 4) || !aligned(active_cnt, 4) || !aligned(per_head, 8))
    return ETA_ERR_INVALID_ARG;
  DiagCall c;
  c.shape = *shape;
  c.n = n_tokens;
  c.n_local = params->n_local;
  c.offset_a = params->offset_a;
  c.tau = tau;
  c.tau_stride = tau_batch_stride;
  c.bmax = block_max;
  c.above = above;
  c.blse = block_lse;
  c.active_idx = active_idx;
  c.active_cnt = active_cnt;
  c.out = per_head;
  return from_cuda(launch_screen_diagnostics(c, stream));
}

ETA_API eta_status_t eta_test_withhold_copy(int64_t position) {
  g_withhold.store(position < 0 ? -1 : position);
  return ETA_OK;
}

ETA_API eta_status_t eta_block_stats(const eta_shape_t* shape, const eta_params_t* params, const void* q,
                                     const void* k, int64_t n_tokens, const float* tau, int64_t tau_batch_stride,
                                     float* block_max, int32_t* above, float* block_lse, eta_stream_t stream) {
  ETA_TRY(check_shape(shape));
  ETA_TRY(check_params(params));
  ETA_TRY(check_tokens(shape, n_tokens));
  if (q == nullptr || k == nullptr || tau == nullptr || tau_batch_stride < 0) return ETA_ERR_INVALID_ARG;
  if (block_max == nullptr || above == nullptr || block_lse == nullptr) return ETA_ERR_INVALID_ARG;
  if (!aligned(q, elem_bytes(shape->q_dtype)) || !aligned(k, 16) || !aligned(tau, 4) || !aligned(block_max, 4) ||
      !aligned(above, 4) || !aligned(block_lse, 4))
    return ETA_ERR_INVALID_ARG;
  StatsCall c;
  c.shape = *shape;
  c.q = q;
  c.k = k;
  c.n = n_tokens;
  c.tau = tau;
  c.tau_stride = tau_batch_stride;
  c.beta = params->beta;
  c.offset_a = params->offset_a;
  c.gate = params->gate;
  c.bmax = block_max;
  c.above = above;
  c.blse = block_lse;
  return from_cuda(launch_block_stats(c, stream));
}

}  // extern "C"

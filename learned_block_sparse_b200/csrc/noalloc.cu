// eta_decode_sparse_static: the sparse decode step with its scratch in a
// fixed device array inside this library, for callers that cannot allocate
// device memory at call time.
//
// Who needs it: a caller running under a frozen memory plan (serving engines
// that reserve all device memory at start-up and forbid later cudaMalloc),
// code embedded in a host framework that owns every allocation and hands out
// only tensors, and real-time loops that must not call into an allocator
// (cudaMalloc can synchronise the device and its latency is unbounded). Such
// callers still own their inputs and outputs; only the per-call scratch
// (admitted-block lists, split partials, status word) moves into the library.
//
// The scratch is one file-scope __device__ array of kStaticScratchBytes. Every
// GPU that loads the library holds it until the process exits. All calls on a
// device share it and it keeps the last call's contents: each call clears the
// workspace header (status word and partial counters, the only parts that must
// start at zero; everything else is written before it is read within a call).
// Calls whose kernels overlap on the GPU (different streams, no ordering
// between them) race on the array and must not be issued.
//
// Host code cannot use the array's name as a device address: the first call on
// each device looks the address up with cudaGetSymbolAddress (with that device
// current) and caches it; make that first call before any stream capture.
#include <cstdint>
#include <mutex>

#include <cuda_runtime.h>

#include "eta.h"

namespace {

constexpr size_t kStaticScratchBytes = size_t{32} << 20;  // 32 MiB
static_assert(kStaticScratchBytes == ETA_STATIC_SCRATCH_BYTES, "header and library disagree on the scratch size");

static __device__ __align__(256) unsigned char g_eta_scratch[kStaticScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_scratch_mu;
void* g_scratch_ptr[kMaxDevices] = {};

// Device address of g_eta_scratch on the current device (looked up once per device).
cudaError_t scratch_address(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (g_scratch_ptr[dev] == nullptr) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_eta_scratch);
    if (e != cudaSuccess) return e;
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return cudaSuccess;
}

}  // namespace

extern "C" ETA_API eta_status_t eta_decode_sparse_static(const eta_shape_t* shape, const eta_params_t* params,
                                                         const void* q, const void* k, const void* v,
                                                         eta_meta_t meta, int64_t n_tokens, const float* tau,
                                                         int64_t tau_batch_stride, float* out,
                                                         const eta_screen_out_t* extra, int32_t* device_status,
                                                         eta_stream_t stream) {
  const size_t need = eta_decode_workspace_bytes(shape, params);
  if (need == 0) return ETA_ERR_INVALID_ARG;
  if (need > kStaticScratchBytes) return ETA_ERR_WORKSPACE;  // shape too large for the fixed scratch
  void* ws = nullptr;
  if (scratch_address(&ws) != cudaSuccess) return ETA_ERR_CUDA;
  if (eta_workspace_init(ws, kStaticScratchBytes, stream) != ETA_OK) return ETA_ERR_CUDA;
  const eta_status_t st = eta_decode_sparse(shape, params, q, k, v, meta, n_tokens, tau, tau_batch_stride, out, extra,
                                            ws, kStaticScratchBytes, stream);
  if (st != ETA_OK) return st;
  if (device_status != nullptr &&
      cudaMemcpyAsync(device_status, ws, sizeof(int32_t), cudaMemcpyDeviceToDevice, stream) != cudaSuccess)
    return ETA_ERR_CUDA;
  return ETA_OK;
}

// Internal interface between the C-ABI layer (api.cpp) and the kernel
// launchers (*.cu). Not part of the public ABI.
#pragma once

#include <atomic>
#include <cstddef>
#include <cstdint>
#include <cuda_runtime.h>

#include "eta.h"

namespace eta {

// Per-call scratch carved out of the caller's workspace.
struct Workspace {
  int32_t* status;        // device status word (sticky until read)
  uint32_t* union_list;   // [B*Hkv][nb_cap] (block << 8) | head mask
  int32_t* union_cnt;     // [B*Hkv]
  int32_t* head_cnt;      // [B*Hq]
  int32_t* seg_done;      // [kMaxBH] partials counted per (batch, kv head); zero between calls
  float* o_part;          // [B*Hq][S][d] unnormalised partial outputs
  float2* ml_part;        // [B*Hq][S] (running max in log2 units, running sum)
};

struct WsLayout {
  size_t status, seg_done, union_list, union_cnt, head_cnt, o_part, ml_part, total;
};

WsLayout ws_layout(int B, int Hq, int Hkv, int d, int64_t nb_cap, int S);
Workspace ws_carve(void* base, const WsLayout& L);

int device_sm_count();
int device_max_smem_optin();

// Raise a kernel's dynamic shared memory limit to the device maximum, once per
// device (`done` is the kernel instance's own flag set).
inline cudaError_t allow_max_smem(std::atomic<uint64_t>& done, const void* fn) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const uint64_t bit = 1ull << (dev & 63);
  if (done.load(std::memory_order_acquire) & bit) return cudaSuccess;
  e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, device_max_smem_optin());
  if (e == cudaSuccess) done.fetch_or(bit, std::memory_order_acq_rel);
  return e;
}

// Launch attribute that lets a kernel start while the previous kernel on the
// stream finishes (programmatic dependent launch). Only for kernels that call
// grid_dependency_wait() before their first global read.
inline cudaLaunchAttribute pdl_attribute() {
  cudaLaunchAttribute a = {};
  a.id = cudaLaunchAttributeProgrammaticStreamSerialization;
  a.val.programmaticStreamSerializationAllowed = 1;
  return a;
}

// Launch `kernel` on `grid` x `block` threads with programmatic dependent launch.
template <typename Kernel, typename... Args>
cudaError_t launch_pdl(Kernel kernel, unsigned grid, unsigned block, size_t smem, cudaStream_t st, Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(block);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1] = {pdl_attribute()};
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaError_t e = cudaLaunchKernelEx(&cfg, kernel, args...);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

cudaError_t launch_build_meta(const eta_shape_t& s, const void* k, int64_t b0, int64_t b1, const eta_meta_t& m,
                              cudaStream_t st, const int32_t* block_table = nullptr, int num_pages = 0);

cudaError_t launch_predict(const eta_shape_t& s, const void* q, const float* W, const float* bias, float* tau,
                           cudaStream_t st);

struct ScreenCall {
  eta_shape_t shape;
  float z, offset_a;
  int n_local;
  int sub_blocks;          // r: sub-blocks per block (1 = Eq. 5 on whole blocks)
  const void* q;
  eta_meta_t meta;
  int64_t n;               // tokens (all rows), or the upper bound of seq_lens
  const int32_t* seq_lens; // [B] per-row token counts (device), or null
  const float* tau;
  int64_t tau_stride;
  const float* W;         // non-null: form tau by Eq. 1 inside the screen (tau ignored)
  const float* bias;
  float* tau_out;         // [B][Hq], written when W is non-null
  eta_screen_out_t out;   // optional outputs (fields may be null)
  Workspace ws;
};
cudaError_t launch_screen(const ScreenCall& c, cudaStream_t st);

struct DecodeCall {
  eta_shape_t shape;
  float beta;
  int gate;                // ETA_GATE_SIGMOID or ETA_GATE_HARD
  const void* q;
  const void* k;
  const void* v;
  int64_t n;               // tokens (all rows), or the upper bound of seq_lens
  const int32_t* seq_lens; // [B] per-row token counts (device), or null
  const int32_t* block_table;  // [B][capacity/block_size] pages (device), or null: contiguous k, v
  int num_pages;           // pages in the k and v pools (paged only)
  const float* tau;        // gate thresholds; null = -inf (dense only)
  int64_t tau_stride;
  float* out;
  Workspace ws;
  int S;                   // number of work ranges (grid size)
  bool dense;
  int64_t withhold = -1;   // test hook (eta_test_withhold_copy): unarmed position of thread block 0
};
cudaError_t launch_decode(const DecodeCall& c, cudaStream_t st);

struct StatsCall {
  eta_shape_t shape;
  const void* q;
  const void* k;
  int64_t n;
  const float* tau;
  int64_t tau_stride;
  float beta, offset_a;
  int gate;
  float* bmax;             // [B][Hq][nb_cap]
  int32_t* above;          // [B][Hq][nb_cap]
  float* blse;             // [B][Hq][nb_cap]
};
cudaError_t launch_block_stats(const StatsCall& c, cudaStream_t st);

struct DiagCall {
  eta_shape_t shape;
  int64_t n;
  int n_local;
  float offset_a;
  const float* tau;
  int64_t tau_stride;
  const float* bmax;        // [B][Hq][nb_cap]
  const int32_t* above;     // [B][Hq][nb_cap]
  const float* blse;        // [B][Hq][nb_cap]
  const int32_t* active_idx;  // [B][Hq][nb_cap]
  const int32_t* active_cnt;  // [B][Hq]
  double* out;              // [B][Hq][4]
};
cudaError_t launch_screen_diagnostics(const DiagCall& c, cudaStream_t st);

// Largest B*Hkv the decode kernel's on-chip prefix table holds.
constexpr int kMaxBH = 8192;
// The workspace starts with a fixed header, the part that must be zero before
// a call: the status word (own 256-byte line) and the seg_done counters.
constexpr size_t kWsHeaderBytes = 256 + kMaxBH * sizeof(int32_t);
// Largest number of 32-block tiles one screening thread block holds.
constexpr int kMaxScreenTiles = 1024;
constexpr int kMaxCluster = 8;

}  // namespace eta

// Threshold predictor (Methodology §1, Eq. 1): tau_h = qbar . W[:, h] + b_h,
// qbar the concatenation of all query heads. One warp per (batch, head); lane l
// folds the terms j = l (mod 32) in increasing j, then a butterfly sums the
// 32 partials, so the result does not depend on the launch.
#include "common.cuh"
#include "launch.h"

namespace eta {

namespace {

constexpr int kPredWarps = 8;

__global__ void __launch_bounds__(kPredWarps * 32)
    predict_kernel(const void* __restrict__ q, int q_dtype, const float* __restrict__ W,
                   const float* __restrict__ bias, float* __restrict__ tau, int Hq, int D) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int h = blockIdx.y * kPredWarps + warp;
  if (h >= Hq) return;
  const int64_t b = blockIdx.x;
  const int64_t Hd = static_cast<int64_t>(Hq) * D;
  float p = 0.0f;
  for (int64_t j = lane; j < Hd; j += 32) p = __fmaf_rn(load_elem(q, q_dtype, b * Hd + j), __ldg(W + j * Hq + h), p);
  for (int o = 16; o >= 1; o >>= 1) p = __fadd_rn(p, __shfl_xor_sync(kFull, p, o));
  if (lane == 0) tau[b * Hq + h] = __fadd_rn(p, __ldg(bias + h));
}

}  // namespace

cudaError_t launch_predict(const eta_shape_t& s, const void* q, const float* W, const float* bias, float* tau,
                           cudaStream_t st) {
  dim3 grid(static_cast<unsigned>(s.batch), static_cast<unsigned>((s.n_q_heads + kPredWarps - 1) / kPredWarps));
  predict_kernel<<<grid, kPredWarps * 32, 0, st>>>(q, s.q_dtype, W, bias, tau, s.n_q_heads, s.head_dim);
  return cudaGetLastError();
}

}  // namespace eta

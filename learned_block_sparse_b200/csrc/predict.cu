// Threshold predictor (Methodology §1, Eq. 1): tau_h = qbar . W[:, h] + b_h,
// qbar the concatenation of all query heads. The dot product has one fixed
// order: 32 running partials, partial l folding the terms j = l (mod 32) in
// increasing j by fused multiply-add, then a butterfly over the 32 partials.
// A thread block covers one batch row and up to 32 heads: thread (warp l,
// lane h) folds partial l of head h, so every load of W reads 32 consecutive
// heads of one row (coalesced); then warp h adds up head h's partials.
#include "common.cuh"
#include "launch.h"

namespace eta {

namespace {

__global__ void __launch_bounds__(1024)
    predict_kernel(const void* __restrict__ q, int q_dtype, const float* __restrict__ W,
                   const float* __restrict__ bias, float* __restrict__ tau, int Hq, int D) {
  __shared__ float part[32][33];
  const int l = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int h = blockIdx.y * 32 + lane;
  const int64_t b = blockIdx.x;
  const int64_t Hd = static_cast<int64_t>(Hq) * D;
  float p = 0.0f;
  if (h < Hq) {
    // loads of a chunk are issued together; the multiply-adds stay in increasing j
    constexpr int kChunk = 16;
    for (int64_t j0 = l; j0 < Hd; j0 += 32 * kChunk) {
      float qv[kChunk], wv[kChunk];
#pragma unroll
      for (int c = 0; c < kChunk; ++c) {
        const int64_t j = j0 + 32 * c;
        qv[c] = j < Hd ? load_elem(q, q_dtype, b * Hd + j) : 0.0f;
        wv[c] = j < Hd ? __ldg(W + j * Hq + h) : 0.0f;
      }
#pragma unroll
      for (int c = 0; c < kChunk; ++c)
        if (j0 + 32 * c < Hd) p = __fmaf_rn(qv[c], wv[c], p);
    }
  }
  part[l][lane] = p;
  __syncthreads();
  const int hh = blockIdx.y * 32 + l;   // warp l now sums head hh
  float v = part[lane][l];
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) v = __fadd_rn(v, __shfl_xor_sync(kFull, v, o));
  if (lane == 0 && hh < Hq) tau[b * Hq + hh] = __fadd_rn(v, __ldg(bias + hh));
}

}  // namespace

cudaError_t launch_predict(const eta_shape_t& s, const void* q, const float* W, const float* bias, float* tau,
                           cudaStream_t st) {
  dim3 grid(static_cast<unsigned>(s.batch), static_cast<unsigned>((s.n_q_heads + 31) / 32));
  predict_kernel<<<grid, 1024, 0, st>>>(q, s.q_dtype, W, bias, tau, s.n_q_heads, s.head_dim);
  return cudaGetLastError();
}

}  // namespace eta

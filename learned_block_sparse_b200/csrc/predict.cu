// Threshold predictor (Methodology §1, Eq. 1): tau_h = qbar . W[:, h] + b_h,
// qbar the concatenation of all query heads. The dot product has one fixed
// order: 32 running partials, partial l folding the terms j = l (mod 32) in
// increasing j by fused multiply-add, then a butterfly over the 32 partials.
// A thread block covers one batch row and up to 32 heads: qbar is staged in
// shared memory, thread (warp l, lane h) folds partial l of head h, so every
// load of W reads 32 consecutive heads of one row (coalesced); then warp h
// adds up head h's partials.
#include "common.cuh"
#include "launch.h"

namespace eta {

namespace {

__global__ void __launch_bounds__(1024)
    predict_kernel(const void* __restrict__ q, int q_dtype, const float* __restrict__ W,
                   const float* __restrict__ bias, float* __restrict__ tau, int Hq, int D) {
  extern __shared__ float smem_f[];
  float (*part)[33] = reinterpret_cast<float (*)[33]>(smem_f);  // [32][33] partials
  float* qs = smem_f + 32 * 33;                                 // qbar of this batch row, fp32
  const int l = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int h = blockIdx.y * 32 + lane;
  const int64_t b = blockIdx.x;
  const int Hd = Hq * D;
  for (int i = threadIdx.x; i < Hd; i += 1024) qs[i] = load_elem(q, q_dtype, b * Hd + i);
  __syncthreads();
  // partial l folds the terms j = l + 32c, c = 0 .. nterm-1, in increasing c;
  // the loads of 16 terms are issued before their multiply-adds
  const int nterm = Hd / 32;
  float p = 0.0f;
  if (h < Hq) {
    const float* wp = W + static_cast<int64_t>(l) * Hq + h;
    const int64_t step = static_cast<int64_t>(32) * Hq;
    int c0 = 0;
    for (; c0 + 16 <= nterm; c0 += 16) {
      float wv[16];
#pragma unroll
      for (int c = 0; c < 16; ++c) wv[c] = __ldg(wp + (c0 + c) * step);
#pragma unroll
      for (int c = 0; c < 16; ++c) p = __fmaf_rn(qs[l + 32 * (c0 + c)], wv[c], p);
    }
    for (; c0 < nterm; ++c0) p = __fmaf_rn(qs[l + 32 * c0], __ldg(wp + c0 * step), p);
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
  const size_t smem = (32 * 33 + static_cast<size_t>(s.n_q_heads) * s.head_dim) * sizeof(float);
  static std::atomic<uint64_t> smem_done{0};
  cudaError_t e = allow_max_smem(smem_done, reinterpret_cast<const void*>(predict_kernel));
  if (e != cudaSuccess) return e;
  predict_kernel<<<grid, 1024, smem, st>>>(q, s.q_dtype, W, bias, tau, s.n_q_heads, s.head_dim);
  return cudaGetLastError();
}

}  // namespace eta

// Threshold predictor (Methodology §1, Eq. 1): tau_h = qbar . W[:, h] + b_h,
// qbar the concatenation of all query heads, in the fixed order of
// tau_chain.cuh. A thread block covers one batch row and up to 8 heads: its
// 256 threads each run one of the 32 x 8 partial chains with the loads of 64
// terms in flight, so the whole predictor costs about Hq*d/2048 memory round
// trips; then one warp per head adds up the partials.
#include "launch.h"
#include "tau_chain.cuh"

namespace eta {

namespace {

constexpr int kHeadsPerBlock = 8;
constexpr int kPredThreads = 32 * kHeadsPerBlock;

template <typename QT>
__global__ void __launch_bounds__(kPredThreads)
    predict_kernel(const QT* __restrict__ q, const float* __restrict__ W, const float* __restrict__ bias,
                   float* __restrict__ tau, int Hq, int D) {
  __shared__ float part[32 * (kHeadsPerBlock + 1)];
  __shared__ float tau_s[kHeadsPerBlock];
  const int64_t b = blockIdx.x;
  const int Hd = Hq * D;
  const int h0 = blockIdx.y * kHeadsPerBlock;
  const int NH = min(kHeadsPerBlock, Hq - h0);
  predict_heads<64>(q + b * Hd, W, bias, Hq, Hd, h0, NH, part, tau_s, static_cast<int>(threadIdx.x),
                    kPredThreads, [] { __syncthreads(); });
  if (threadIdx.x < NH) tau[b * Hq + h0 + threadIdx.x] = tau_s[threadIdx.x];
}

}  // namespace

cudaError_t launch_predict(const eta_shape_t& s, const void* q, const float* W, const float* bias, float* tau,
                           cudaStream_t st) {
  const dim3 grid(static_cast<unsigned>(s.batch),
                  static_cast<unsigned>((s.n_q_heads + kHeadsPerBlock - 1) / kHeadsPerBlock));
  if (s.q_dtype == ETA_BF16)
    predict_kernel<uint16_t><<<grid, kPredThreads, 0, st>>>(static_cast<const uint16_t*>(q), W, bias, tau,
                                                            s.n_q_heads, s.head_dim);
  else
    predict_kernel<float><<<grid, kPredThreads, 0, st>>>(static_cast<const float*>(q), W, bias, tau, s.n_q_heads,
                                                         s.head_dim);
  return cudaGetLastError();
}

}  // namespace eta

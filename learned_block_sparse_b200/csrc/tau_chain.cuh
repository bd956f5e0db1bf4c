// Threshold predictor arithmetic (Methodology §1, Eq. 1), shared by the
// stand-alone predictor kernel and the screening kernels that form the
// thresholds of their own query-head group:
//   tau_h = qbar . W[:, h] + b_h,  qbar = the Hq query heads of one batch row
//   concatenated (length Hq*d), W [Hq*d][Hq] fp32 row-major.
// The dot product has one fixed order: 32 running partials, partial l folding
// the terms j = l (mod 32) in increasing j by fused multiply-add, then a
// butterfly over the 32 partials (offsets 16, 8, 4, 2, 1) and the bias.
#pragma once

#include "common.cuh"

namespace eta {

template <typename QT>
__device__ __forceinline__ float q_as_float(QT x);
template <>
__device__ __forceinline__ float q_as_float<float>(float x) {
  return x;
}
template <>
__device__ __forceinline__ float q_as_float<uint16_t>(uint16_t x) {
  return __uint_as_float(static_cast<uint32_t>(x) << 16);  // bf16 -> fp32, exact
}

// Partial l of head h: the multiply-add chain over j = l + 32c, c increasing.
// The loads of kBatch terms (W and qbar) are issued before their multiply-adds,
// so a chain costs about Hd / (32 kBatch) memory round trips.
template <int kBatch, typename QT>
__device__ __forceinline__ float tau_partial(const QT* __restrict__ qrow, const float* __restrict__ W, int Hq,
                                             int Hd, int l, int h) {
  const int nterm = Hd / 32;  // Hd = Hq*d is a multiple of 32 (d in {64, 128})
  const float* wp = W + static_cast<int64_t>(l) * Hq + h;
  const QT* qp = qrow + l;
  const int64_t step = static_cast<int64_t>(32) * Hq;
  float p = 0.0f;
  int c0 = 0;
  for (; c0 + kBatch <= nterm; c0 += kBatch) {
    float wv[kBatch];
    QT qv[kBatch];
#pragma unroll
    for (int c = 0; c < kBatch; ++c) {
      wv[c] = __ldg(wp + (c0 + c) * step);
      qv[c] = __ldg(qp + 32 * (c0 + c));
    }
#pragma unroll
    for (int c = 0; c < kBatch; ++c) p = __fmaf_rn(q_as_float(qv[c]), wv[c], p);
  }
  for (; c0 < nterm; ++c0) p = __fmaf_rn(q_as_float(__ldg(qp + 32 * c0)), __ldg(wp + c0 * step), p);
  return p;
}

// tau of heads h0 .. h0+NH-1 (NH <= 32) of one batch row into tau_s[0..NH),
// by the `nthreads` threads (a multiple of 32) whose index relative to the
// first of them is `rel`; `sync()` must synchronise exactly those threads (it
// is called twice, the second time before returning). part is shared scratch
// of 32*(NH+1) floats.
template <int kBatch, typename QT, typename Sync>
__device__ __forceinline__ void predict_heads(const QT* __restrict__ qrow, const float* __restrict__ W,
                                              const float* __restrict__ bias, int Hq, int Hd, int h0, int NH,
                                              float* part, float* tau_s, int rel, int nthreads, Sync sync) {
  const int warp = rel >> 5, lane = rel & 31;
  // chain (l, g) = thread l*NH + g: neighbouring threads read neighbouring
  // heads of one row of W
  for (int c = rel; c < 32 * NH; c += nthreads) {
    const int l = c / NH, g = c % NH;
    part[l * (NH + 1) + g] = tau_partial<kBatch>(qrow, W, Hq, Hd, l, h0 + g);
  }
  sync();
  for (int g = warp; g < NH; g += nthreads >> 5) {
    float v = part[lane * (NH + 1) + g];
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) v = __fadd_rn(v, __shfl_xor_sync(kFull, v, o));
    if (lane == 0) tau_s[g] = __fadd_rn(v, __ldg(bias + h0 + g));
  }
  sync();
}

}  // namespace eta

// Block statistics behind the screen diagnostics of Table 16 (false
// negatives, false positives, token recall, missed mass): for every query head
// and block, the true maximum scaled logit, the number of tokens whose scaled
// logit reaches the screen threshold tau - a, and the log-sum-exp of the gated
// logits (Eq. 2-3, or strict mode). A dense pass over K (no V), off the decode
// path: it measures how well the O(1) screen predicts the blocks that matter.
//
// S_s = fl(fl(sum_i q_i k_si) * s) with the sum by fused multiply-adds in
// increasing i and s = fl(1/sqrt(d)): the maxima and counts are reproducible
// bit for bit. One thread block per (batch, kv head) and tile of blocks; a
// block's keys are widened into shared memory (one padded row per token), one
// thread per token runs the chains for the G heads of the group, one warp per
// head reduces.
#include <cmath>

#include "common.cuh"
#include "launch.h"

namespace eta {

namespace {

constexpr int kStatThreads = 128;
constexpr int kStatTile = 8;  // blocks per thread block

struct StatArgs {
  const void* q;
  int q_dtype;
  const void* k;
  int kv_dtype;
  const float* tau;
  int64_t tau_stride, cap, n;
  int Hq, Hkv, bs, nb, nb_cap, gate;
  float s, beta, offset_a;
  float* bmax;
  int32_t* above;
  float* blse;
};

template <int D, int G>
__global__ void __launch_bounds__(kStatThreads) stats_kernel(const StatArgs a) {
  extern __shared__ __align__(16) float sm[];
  const int bs = a.bs;
  float* kb = sm;                   // [bs][D+1]
  float* qs = kb + bs * (D + 1);    // [G][D]
  float* ss = qs + G * D;           // [G][bs] scaled logits of the block
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int bh = blockIdx.x;
  const int b = bh / a.Hkv, kvh = bh % a.Hkv;
  const int64_t t_cur = a.n - 1;
  for (int i = tid; i < G * D; i += kStatThreads)
    qs[i] = load_elem(a.q, a.q_dtype, (static_cast<int64_t>(b) * a.Hq + kvh * G) * D + i);
  const int j0 = blockIdx.y * kStatTile;
  const int j1 = min(a.nb, j0 + kStatTile);
  for (int j = j0; j < j1; ++j) {
    const int64_t tok0 = static_cast<int64_t>(j) * bs;
    const int rows = static_cast<int>(min(static_cast<int64_t>(bs), a.n - tok0));
    __syncthreads();  // kb and ss of the previous block are consumed
    for (int idx = tid; idx < rows * D; idx += kStatThreads) {
      const int r = idx / D, i = idx % D;
      kb[r * (D + 1) + i] = load_elem(a.k, a.kv_dtype, (static_cast<int64_t>(bh) * a.cap + tok0 + r) * D + i);
    }
    __syncthreads();
    for (int r = tid; r < rows; r += kStatThreads) {
#pragma unroll
      for (int g = 0; g < G; ++g) {
        float acc = 0.0f;
        for (int i = 0; i < D; ++i) acc = __fmaf_rn(qs[g * D + i], kb[r * (D + 1) + i], acc);
        ss[g * bs + r] = __fmul_rn(acc, a.s);
      }
    }
    __syncthreads();
    for (int g = warp; g < G; g += kStatThreads / 32) {
      const int h = kvh * G + g;
      const float tau = a.tau[b * a.tau_stride + h];
      const float taus = __fsub_rn(tau, a.offset_a);
      auto gated = [&](int r) {
        const float S = ss[g * bs + r];
        if (tok0 + r == t_cur) return S;
        if (a.gate == ETA_GATE_HARD) return S >= tau ? S : -INFINITY;
        return S / (1.0f + expf(-a.beta * (S - tau)));
      };
      float mx = -INFINITY, gm = -INFINITY;
      int cnt = 0;
      for (int r = lane; r < rows; r += 32) {
        const float S = ss[g * bs + r];
        mx = fmaxf(mx, S);
        cnt += S >= taus ? 1 : 0;
        gm = fmaxf(gm, gated(r));
      }
#pragma unroll
      for (int o = 16; o >= 1; o >>= 1) {
        mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, o));
        gm = fmaxf(gm, __shfl_xor_sync(kFull, gm, o));
        cnt += __shfl_xor_sync(kFull, cnt, o);
      }
      float z = 0.0f;
      if (gm != -INFINITY)
        for (int r = lane; r < rows; r += 32) z += expf(gated(r) - gm);
#pragma unroll
      for (int o = 16; o >= 1; o >>= 1) z += __shfl_xor_sync(kFull, z, o);
      if (lane == 0) {
        const int64_t o = (static_cast<int64_t>(b) * a.Hq + h) * a.nb_cap + j;
        a.bmax[o] = mx;
        a.above[o] = cnt;
        a.blse[o] = gm == -INFINITY ? -INFINITY : gm + logf(z);
      }
    }
  }
}

template <int D, int G>
cudaError_t launch_stats_t(const StatArgs& a, int BH, cudaStream_t st) {
  const size_t smem = (static_cast<size_t>(a.bs) * (D + 1) + G * D + static_cast<size_t>(G) * a.bs) * sizeof(float);
  static std::atomic<uint64_t> smem_done{0};
  cudaError_t e = allow_max_smem(smem_done, reinterpret_cast<const void*>(stats_kernel<D, G>));
  if (e != cudaSuccess) return e;
  const dim3 grid(static_cast<unsigned>(BH), static_cast<unsigned>((a.nb + kStatTile - 1) / kStatTile));
  stats_kernel<D, G><<<grid, kStatThreads, smem, st>>>(a);
  return cudaGetLastError();
}

template <int D>
cudaError_t launch_stats_d(const StatArgs& a, int BH, int G, cudaStream_t st) {
  switch (G) {
    case 1: return launch_stats_t<D, 1>(a, BH, st);
    case 2: return launch_stats_t<D, 2>(a, BH, st);
    case 4: return launch_stats_t<D, 4>(a, BH, st);
    case 8: return launch_stats_t<D, 8>(a, BH, st);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace

cudaError_t launch_block_stats(const StatsCall& c, cudaStream_t st) {
  const eta_shape_t& s = c.shape;
  StatArgs a;
  a.q = c.q;
  a.q_dtype = s.q_dtype;
  a.k = c.k;
  a.kv_dtype = s.kv_dtype;
  a.tau = c.tau;
  a.tau_stride = c.tau_stride;
  a.cap = s.capacity;
  a.n = c.n;
  a.Hq = s.n_q_heads;
  a.Hkv = s.n_kv_heads;
  a.bs = s.block_size;
  a.nb = static_cast<int>((c.n + s.block_size - 1) / s.block_size);
  a.nb_cap = static_cast<int>(s.capacity / s.block_size);
  a.gate = c.gate;
  a.s = static_cast<float>(1.0 / std::sqrt(static_cast<double>(s.head_dim)));
  a.beta = c.beta;
  a.offset_a = c.offset_a;
  a.bmax = c.bmax;
  a.above = c.above;
  a.blse = c.blse;
  const int BH = s.batch * s.n_kv_heads;
  const int G = s.n_q_heads / s.n_kv_heads;
  return s.head_dim == 128 ? launch_stats_d<128>(a, BH, G, st) : launch_stats_d<64>(a, BH, G, st);
}

}  // namespace eta

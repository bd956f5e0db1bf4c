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

// Table 16's screen diagnostics of one query head (one warp per head), from
// its block statistics and its ascending admitted list, over the ns screened
// blocks (the forced trailing blocks excluded); a block is truly active when
// its max scaled logit reaches fl(tau - a):
//   false_negative = truly active blocks not admitted / truly active blocks
//   false_positive = admitted blocks not truly active / admitted blocks
//   token_recall   = tokens at or above fl(tau - a) in admitted blocks / all such tokens
//   missed_mass    = gated softmax mass of the rejected blocks over that of all nb blocks
// Counts are exact; the masses are fp64 sums of exp(lse_j - max lse) in a fixed
// order (lane-strided partials, then a butterfly), so the result does not
// depend on timing. A zero denominator counts as one (the ratio is then 0).
struct DiagArgs {
  const float* tau;
  int64_t tau_stride;
  const float* bmax;
  const int32_t* above;
  const float* blse;
  const int32_t* active_idx;
  const int32_t* active_cnt;
  double* out;  // [B][Hq][4]
  float offset_a;
  int heads, Hq, nb, ns, nb_cap;
};

__device__ __forceinline__ double warp_sum(double v) {
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) v += __shfl_xor_sync(kFull, v, o);
  return v;
}

__global__ void __launch_bounds__(kStatThreads) diag_kernel(const DiagArgs a) {
  const int lane = threadIdx.x & 31;
  const int hd = static_cast<int>(blockIdx.x) * (kStatThreads / 32) + (threadIdx.x >> 5);  // b * Hq + h
  if (hd >= a.heads) return;
  const int b = hd / a.Hq, h = hd - b * a.Hq;
  const float ts = __fsub_rn(a.tau[b * a.tau_stride + h], a.offset_a);
  const int64_t row = static_cast<int64_t>(hd) * a.nb_cap;
  const float* bm = a.bmax + row;
  const int32_t* ab = a.above + row;
  const float* ls = a.blse + row;
  double mx = -INFINITY;
  for (int j = lane; j < a.nb; j += 32) mx = fmax(mx, static_cast<double>(ls[j]));
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) mx = fmax(mx, __shfl_xor_sync(kFull, mx, o));
  const double base = mx == -INFINITY ? 0.0 : mx;
  // every block: the normaliser; screened blocks: active count, tokens, mass
  double all = 0.0, scr = 0.0, act = 0.0, tok = 0.0;
  for (int j = lane; j < a.nb; j += 32) {
    const double e = exp(static_cast<double>(ls[j]) - base);
    all += e;
    if (j < a.ns) {
      scr += e;
      act += bm[j] >= ts ? 1.0 : 0.0;
      tok += static_cast<double>(ab[j]);
    }
  }
  // the admitted screened blocks
  const int cnt = a.active_cnt[hd];
  const int32_t* lst = a.active_idx + row;
  double adm = 0.0, both = 0.0, tok_adm = 0.0, mass_adm = 0.0;
  for (int k = lane; k < cnt; k += 32) {
    const int j = lst[k];
    if (j < 0 || j >= a.ns) continue;
    adm += 1.0;
    both += bm[j] >= ts ? 1.0 : 0.0;
    tok_adm += static_cast<double>(ab[j]);
    mass_adm += exp(static_cast<double>(ls[j]) - base);
  }
  all = warp_sum(all);
  scr = warp_sum(scr);
  act = warp_sum(act);
  tok = warp_sum(tok);
  adm = warp_sum(adm);
  both = warp_sum(both);
  tok_adm = warp_sum(tok_adm);
  mass_adm = warp_sum(mass_adm);
  if (lane == 0) {
    double* o = a.out + static_cast<int64_t>(hd) * 4;
    o[0] = (act - both) / fmax(1.0, act);
    o[1] = (adm - both) / fmax(1.0, adm);
    o[2] = tok_adm / fmax(1.0, tok);
    o[3] = (a.ns - adm) > 0.0 && all > 0.0 ? fmax(0.0, scr - mass_adm) / all : 0.0;
  }
}

}  // namespace

cudaError_t launch_screen_diagnostics(const DiagCall& c, cudaStream_t st) {
  const eta_shape_t& s = c.shape;
  DiagArgs a;
  a.tau = c.tau;
  a.tau_stride = c.tau_stride;
  a.bmax = c.bmax;
  a.above = c.above;
  a.blse = c.blse;
  a.active_idx = c.active_idx;
  a.active_cnt = c.active_cnt;
  a.out = c.out;
  a.offset_a = c.offset_a;
  a.heads = s.batch * s.n_q_heads;
  a.Hq = s.n_q_heads;
  a.nb = static_cast<int>((c.n + s.block_size - 1) / s.block_size);
  a.ns = a.nb > c.n_local ? a.nb - c.n_local : 0;
  a.nb_cap = static_cast<int>(s.capacity / s.block_size);
  const unsigned grid = static_cast<unsigned>((a.heads + kStatThreads / 32 - 1) / (kStatThreads / 32));
  diag_kernel<<<grid, kStatThreads, 0, st>>>(a);
  return cudaGetLastError();
}

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

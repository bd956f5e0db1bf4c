// Block metadata (Methodology §4, "Dual Probabilistic-Geometric Block Index"):
// per full block of b keys, the population centroid mu, the coordinate-wise
// population variance and the maximum key norm, in a fixed fp32 order so the
// screening decisions built on them are reproducible. The keys come from a
// contiguous cache or, through a block table, from a paged pool; the metadata
// itself is always indexed by logical block. A block whose page index is
// outside the pool is skipped (its metadata is left as it was).
#include "common.cuh"
#include "launch.h"

namespace eta {

namespace {

constexpr int kMetaThreads = 128;
constexpr int kMetaTile = 32;  // blocks per thread block (one coalesced 128-byte row per coordinate)

template <typename KV, int D>
__global__ void __launch_bounds__(kMetaThreads) meta_kernel(const KV* __restrict__ k, const KvLayout L,
                                                            int64_t nb_cap, int64_t blk_begin, int64_t blk_end,
                                                            float* __restrict__ mu, float* __restrict__ var,
                                                            float* __restrict__ maxn) {
  extern __shared__ __align__(16) float sm[];
  const int bs = L.bs;
  float* kb = sm;                             // [bs][D+1] widened keys of one block
  float* s_mu = kb + bs * (D + 1);            // [D][kMetaTile]
  float* s_var = s_mu + D * kMetaTile;        // [D][kMetaTile]
  float* s_nrm = s_var + D * kMetaTile;       // [bs] squared row norms
  float* s_mx = s_nrm + 128;                  // [kMetaTile]
  const int tid = threadIdx.x;
  const int64_t bh = blockIdx.x;
  const int64_t j0 = blk_begin + static_cast<int64_t>(blockIdx.y) * kMetaTile;
  const int jn = static_cast<int>((blk_end - j0 < kMetaTile ? blk_end - j0 : int64_t{kMetaTile}));
  const int dt = KvTraits<KV>::kDtype;
  const float rows = static_cast<float>(bs);

  for (int jj = 0; jj < jn; ++jj) {
    const int64_t tok0 = kv_block_row(L, static_cast<int>(bh), static_cast<int>(j0 + jj));
    if (tok0 < 0) {  // page outside the pool: nothing is read or written for this block (s_mx < 0)
      if (tid < D) s_mu[tid * kMetaTile + jj] = s_var[tid * kMetaTile + jj] = 0.0f;
      if (tid == 0) s_mx[jj] = -1.0f;
      __syncthreads();
      continue;
    }
    for (int idx = tid; idx < bs * D; idx += kMetaThreads) {
      const int r = idx / D, i = idx % D;
      kb[r * (D + 1) + i] = load_elem(k, dt, (tok0 + r) * D + i);
    }
    __syncthreads();
    if (tid < D) {
      float t = 0.0f;
      for (int r = 0; r < bs; ++r) t = __fadd_rn(t, kb[r * (D + 1) + tid]);
      const float m = __fdiv_rn(t, rows);
      float v = 0.0f;
      for (int r = 0; r < bs; ++r) {
        const float e = __fsub_rn(kb[r * (D + 1) + tid], m);
        v = __fmaf_rn(e, e, v);
      }
      s_mu[tid * kMetaTile + jj] = m;
      s_var[tid * kMetaTile + jj] = __fdiv_rn(v, rows);
    }
    if (tid < bs) {
      float nr = 0.0f;
      for (int i = 0; i < D; ++i) {
        const float x = kb[tid * (D + 1) + i];
        nr = __fmaf_rn(x, x, nr);
      }
      s_nrm[tid] = nr;
    }
    __syncthreads();
    if (tid < 32) {
      float best = 0.0f;
      for (int r = tid; r < bs; r += 32) best = fmaxf(best, s_nrm[r]);
      for (int o = 16; o >= 1; o >>= 1) best = fmaxf(best, __shfl_xor_sync(kFull, best, o));
      if (tid == 0) s_mx[jj] = __fsqrt_rn(best);
    }
    __syncthreads();
  }
  __syncthreads();
  for (int idx = tid; idx < D * kMetaTile; idx += kMetaThreads) {
    const int i = idx / kMetaTile, jj = idx % kMetaTile;
    if (jj < jn && s_mx[jj] >= 0.0f) {
      const int64_t o = (bh * D + i) * nb_cap + j0 + jj;
      mu[o] = s_mu[idx];
      var[o] = s_var[idx];
    }
  }
  if (tid < jn && s_mx[tid] >= 0.0f) maxn[bh * nb_cap + j0 + tid] = s_mx[tid];
}

template <typename KV, int D>
cudaError_t launch_meta_t(const eta_shape_t& s, const void* k, int64_t b0, int64_t b1, const eta_meta_t& m,
                          cudaStream_t st, const int32_t* table, int num_pages) {
  const int bs = s.block_size;
  const size_t smem = (static_cast<size_t>(bs) * (D + 1) + 2 * D * kMetaTile + 128 + kMetaTile) * sizeof(float);
  static std::atomic<uint64_t> smem_done{0};
  cudaError_t e = allow_max_smem(smem_done, reinterpret_cast<const void*>(meta_kernel<KV, D>));
  if (e != cudaSuccess) return e;
  const int64_t nb_cap = s.capacity / bs;
  dim3 grid(static_cast<unsigned>(static_cast<int64_t>(s.batch) * s.n_kv_heads),
            static_cast<unsigned>((b1 - b0 + kMetaTile - 1) / kMetaTile));
  KvLayout L;
  L.block_table = table;
  L.max_blocks = static_cast<int>(nb_cap);
  L.num_pages = num_pages;
  L.Hkv = s.n_kv_heads;
  L.bs = bs;
  L.cap = s.capacity;
  meta_kernel<KV, D><<<grid, kMetaThreads, smem, st>>>(static_cast<const KV*>(k), L, nb_cap, b0, b1, m.mu, m.var,
                                                       m.maxnorm);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_build_meta(const eta_shape_t& s, const void* k, int64_t b0, int64_t b1, const eta_meta_t& m,
                              cudaStream_t st, const int32_t* table, int num_pages) {
  if (s.kv_dtype == ETA_FP8_E4M3) return launch_meta_t<Fp8Raw, 128>(s, k, b0, b1, m, st, table, num_pages);
  if (s.kv_dtype == ETA_BF16) {
    return s.head_dim == 128 ? launch_meta_t<Bf16Raw, 128>(s, k, b0, b1, m, st, table, num_pages)
                             : launch_meta_t<Bf16Raw, 64>(s, k, b0, b1, m, st, table, num_pages);
  }
  return s.head_dim == 128 ? launch_meta_t<float, 128>(s, k, b0, b1, m, st, table, num_pages)
                           : launch_meta_t<float, 64>(s, k, b0, b1, m, st, table, num_pages);
}

}  // namespace eta

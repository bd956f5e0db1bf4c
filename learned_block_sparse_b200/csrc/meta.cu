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

constexpr int kMetaWarps = 8;  // blocks in work per thread block: one warp each

// Coordinate p of a 32-bit word of the store (4 / elt coordinates per word),
// widened exactly to fp32.
template <typename KV>
__device__ __forceinline__ float word_elem(uint32_t w, int p);
template <>
__device__ __forceinline__ float word_elem<float>(uint32_t w, int) {
  return __uint_as_float(w);
}
template <>
__device__ __forceinline__ float word_elem<Bf16Raw>(uint32_t w, int p) {
  return p == 0 ? bf16_lo(w) : bf16_hi(w);
}
template <>
__device__ __forceinline__ float word_elem<Fp8Raw>(uint32_t w, int p) {
  return e4m3_to_float((w >> (8 * p)) & 0xffu);
}

// One warp per block. Row norms: lane r takes rows r, r+32, ... and folds
// x_i^2 in increasing i (each row read as 16-byte chunks); the block's largest
// norm by a max butterfly. Centroid and variance: lane l takes the words l,
// l+32, ... of every row (elt-wide coordinates packed in 32 bits) and folds the
// rows in increasing order, a first pass for the sum, a second for the squared
// deviations from the rounded mean (the block was just read: the second and the
// column reads come from the L1/L2 caches). Every sum keeps the order of a
// sequential loop, so the metadata does not depend on the launch shape.
template <typename KV, int D>
__global__ void __launch_bounds__(kMetaWarps * 32) meta_kernel(const KV* __restrict__ k, const KvLayout L,
                                                               int64_t nb_cap, int64_t blk_begin, int64_t blk_end,
                                                               float* __restrict__ mu, float* __restrict__ var,
                                                               float* __restrict__ maxn) {
  constexpr int EB = KvTraits<KV>::kBytes;
  constexpr int P = 4 / EB;          // coordinates per 32-bit word
  constexpr int WPR = D / P;         // words per row
  constexpr int C16 = D * EB / 16;   // 16-byte chunks per row
  static_assert(WPR % 32 == 0, "words per row: a multiple of the warp");
  constexpr int WL = WPR / 32;       // words of a row per lane
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int bh = blockIdx.x;
  const int bs = L.bs;
  const float rows = static_cast<float>(bs);
  for (int64_t j = blk_begin + static_cast<int64_t>(blockIdx.y) * kMetaWarps + warp; j < blk_end;
       j += static_cast<int64_t>(gridDim.y) * kMetaWarps) {
    const int tok0 = kv_block_row(L, bh, static_cast<int>(j));
    if (tok0 < 0) continue;  // page outside the pool: nothing is read or written for this block
    const unsigned char* base = reinterpret_cast<const unsigned char*>(k) + static_cast<int64_t>(tok0) * D * EB;
    float best = 0.0f;
    for (int r = lane; r < bs; r += 32) {
      const uint4* row = reinterpret_cast<const uint4*>(base + static_cast<int64_t>(r) * D * EB);
      float nr = 0.0f;
#pragma unroll
      for (int c = 0; c < C16; ++c) {
        const uint4 u = __ldg(row + c);
        const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
        for (int q = 0; q < 4; ++q)
#pragma unroll
          for (int p = 0; p < P; ++p) {
            const float x = word_elem<KV>(w[q], p);
            nr = __fmaf_rn(x, x, nr);
          }
      }
      best = fmaxf(best, nr);
    }
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) best = fmaxf(best, __shfl_xor_sync(kFull, best, o));
    const uint32_t* words = reinterpret_cast<const uint32_t*>(base);
    float t[WL][P];
#pragma unroll
    for (int c = 0; c < WL; ++c)
#pragma unroll
      for (int p = 0; p < P; ++p) t[c][p] = 0.0f;
    for (int r = 0; r < bs; ++r) {
#pragma unroll
      for (int c = 0; c < WL; ++c) {
        const uint32_t w = __ldg(words + static_cast<int64_t>(r) * WPR + lane + 32 * c);
#pragma unroll
        for (int p = 0; p < P; ++p) t[c][p] = __fadd_rn(t[c][p], word_elem<KV>(w, p));
      }
    }
    float v[WL][P];
#pragma unroll
    for (int c = 0; c < WL; ++c)
#pragma unroll
      for (int p = 0; p < P; ++p) {
        t[c][p] = __fdiv_rn(t[c][p], rows);  // the mean
        v[c][p] = 0.0f;
      }
    for (int r = 0; r < bs; ++r) {
#pragma unroll
      for (int c = 0; c < WL; ++c) {
        const uint32_t w = __ldg(words + static_cast<int64_t>(r) * WPR + lane + 32 * c);
#pragma unroll
        for (int p = 0; p < P; ++p) {
          const float e = __fsub_rn(word_elem<KV>(w, p), t[c][p]);
          v[c][p] = __fmaf_rn(e, e, v[c][p]);
        }
      }
    }
#pragma unroll
    for (int c = 0; c < WL; ++c)
#pragma unroll
      for (int p = 0; p < P; ++p) {
        const int i = (lane + 32 * c) * P + p;
        const int64_t o = (static_cast<int64_t>(bh) * D + i) * nb_cap + j;
        mu[o] = t[c][p];
        var[o] = __fdiv_rn(v[c][p], rows);
      }
    if (lane == 0) maxn[static_cast<int64_t>(bh) * nb_cap + j] = __fsqrt_rn(best);
  }
}

template <typename KV, int D>
cudaError_t launch_meta_t(const eta_shape_t& s, const void* k, int64_t b0, int64_t b1, const eta_meta_t& m,
                          cudaStream_t st, const int32_t* table, int num_pages) {
  const int bs = s.block_size;
  const int64_t nb_cap = s.capacity / bs;
  const int64_t groups = (b1 - b0 + kMetaWarps - 1) / kMetaWarps;
  dim3 grid(static_cast<unsigned>(static_cast<int64_t>(s.batch) * s.n_kv_heads),
            static_cast<unsigned>(groups < 65535 ? groups : 65535));
  KvLayout L;
  L.block_table = table;
  L.max_blocks = static_cast<int>(nb_cap);
  L.num_pages = num_pages;
  L.Hkv = s.n_kv_heads;
  L.bs = bs;
  L.cap = s.capacity;
  meta_kernel<KV, D><<<grid, kMetaWarps * 32, 0, st>>>(static_cast<const KV*>(k), L, nb_cap, b0, b1, m.mu, m.var,
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

// Block metadata (Methodology §4, "Dual Probabilistic-Geometric Block Index"):
// per full block of b keys, the population centroid mu, the coordinate-wise
// population variance and the maximum key norm, in a fixed fp32 order so the
// screening decisions built on them are reproducible. The keys come from a
// contiguous cache or, through a block table, from a paged pool; the metadata
// itself is always indexed by logical block. A block whose page index is
// outside the pool is skipped (its metadata is left as it was).
#include <cuda_fp16.h>

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

// The coordinates of one 32-bit word of the store, widened exactly to fp32
// (e4m3 through f16, which holds every e4m3 value).
template <typename KV>
__device__ __forceinline__ void widen_word(uint32_t w, float (&x)[4 / KvTraits<KV>::kBytes]);
template <>
__device__ __forceinline__ void widen_word<float>(uint32_t w, float (&x)[1]) {
  x[0] = __uint_as_float(w);
}
template <>
__device__ __forceinline__ void widen_word<Bf16Raw>(uint32_t w, float (&x)[2]) {
  x[0] = bf16_lo(w);
  x[1] = bf16_hi(w);
}
template <>
__device__ __forceinline__ void widen_word<Fp8Raw>(uint32_t w, float (&x)[4]) {
  uint32_t lo, hi;
  asm("{\n\t.reg .b16 l, h;\n\tmov.b32 {l, h}, %2;\n\tcvt.rn.f16x2.e4m3x2 %0, l;\n\t"
      "cvt.rn.f16x2.e4m3x2 %1, h;\n\t}"
      : "=r"(lo), "=r"(hi)
      : "r"(w));
  const float2 a = __half22float2(*reinterpret_cast<const __half2*>(&lo));
  const float2 b = __half22float2(*reinterpret_cast<const __half2*>(&hi));
  x[0] = a.x;
  x[1] = a.y;
  x[2] = b.x;
  x[3] = b.y;
}

// Staged variant for blocks of at most 16 KB: every warp owns NB shared-memory
// buffers and streams its blocks through them with 16-byte asynchronous copies
// (cp.async, completed by the hardware wait cp.async.wait_group: no spin
// loop), NB - 1 blocks in flight while another is reduced. A block lands as d*elt/128 column boxes of [b rows][128
// bytes] with the 128-byte swizzle (16-byte chunk c of row r at chunk
// c ^ (r & 7) of its 128-byte line), so both access patterns are free of bank
// conflicts: lane = row for the norms (eight lanes, eight different chunks of
// one 128-byte line each) and lane = word for the centroid and the variance
// (a row's 32 consecutive words). The arithmetic and its order are exactly
// meta_kernel's; the block is read from HBM once and re-read from shared
// memory instead of the caches.
__device__ __forceinline__ uint32_t meta_swz(int rows, int r, int c) {
  return static_cast<uint32_t>((c >> 3) * rows * 128 + r * 128 + (((c & 7) ^ (r & 7)) << 4));
}

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

template <typename KV, int D, int NB>
__global__ void __launch_bounds__(kMetaWarps * 32) meta_staged_kernel(const KV* __restrict__ k, const KvLayout L,
                                                                     int64_t nb_cap, int64_t blk_begin, int64_t nblk,
                                                                     int64_t items, float* __restrict__ mu,
                                                                     float* __restrict__ var,
                                                                     float* __restrict__ maxn) {
  constexpr int EB = KvTraits<KV>::kBytes;
  constexpr int P = 4 / EB;          // coordinates per 32-bit word
  constexpr int WPR = D / P;         // words per row
  constexpr int CPR = D * EB / 16;   // 16-byte chunks per row
  static_assert(WPR % 32 == 0, "words per row: a multiple of the warp");
  constexpr int WL = WPR / 32;       // words of a row per lane
  extern __shared__ __align__(1024) unsigned char meta_smem[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int bs = L.bs;
  const uint32_t tile = static_cast<uint32_t>(bs) * D * EB;
  const int nwarps = blockDim.x >> 5;
  unsigned char* buf0 = meta_smem + static_cast<size_t>(warp) * NB * tile;
  const float rows = static_cast<float>(bs);
  const int64_t gw = static_cast<int64_t>(blockIdx.x) * nwarps + warp;
  const int64_t nw = static_cast<int64_t>(gridDim.x) * nwarps;

  // store row of item i's token 0 (-1: page outside the pool, nothing to do)
  auto row_of = [&](int64_t i) -> int {
    const int64_t bh = i / nblk;
    return kv_block_row(L, static_cast<int>(bh), static_cast<int>(blk_begin + (i - bh * nblk)));
  };
  // start the copies of item i into buffer slot (one commit group per item, empty when there is none)
  auto issue = [&](int64_t i, int slot) {
    if (i < items) {
      const int row0 = row_of(i);
      if (row0 >= 0) {
        const unsigned char* src = reinterpret_cast<const unsigned char*>(k) + static_cast<int64_t>(row0) * D * EB;
        const uint32_t dst = smem_u32(buf0 + static_cast<size_t>(slot) * tile);
        for (int q = lane; q < bs * CPR; q += 32) {
          const int r = q / CPR, c = q - r * CPR;
          cp_async16(dst + meta_swz(bs, r, c), src + static_cast<int64_t>(q) * 16);
        }
      }
    }
    cp_async_commit();
  };

#pragma unroll
  for (int b = 0; b < NB - 1; ++b) issue(gw + b * nw, b);
  int slot = 0;
  for (int64_t i = gw; i < items; i += nw, slot = slot + 1 == NB ? 0 : slot + 1) {
    issue(i + (NB - 1) * nw, slot == 0 ? NB - 1 : slot - 1);  // the slot reduced last round
    cp_async_wait<NB - 1>();  // this item's copies (the oldest group) have landed
    __syncwarp();
    const int row0 = row_of(i);
    if (row0 >= 0) {
      const unsigned char* t = buf0 + static_cast<size_t>(slot) * tile;
      // row norms: fused multiply-adds in increasing coordinate order
      float best = 0.0f;
      for (int r = lane; r < bs; r += 32) {
        float nr = 0.0f;
#pragma unroll
        for (int c = 0; c < CPR; ++c) {
          const uint4 u = *reinterpret_cast<const uint4*>(t + meta_swz(bs, r, c));
          const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            float x[P];
            widen_word<KV>(w[q], x);
#pragma unroll
            for (int p = 0; p < P; ++p) nr = __fmaf_rn(x[p], x[p], nr);
          }
        }
        best = fmaxf(best, nr);
      }
#pragma unroll
      for (int o = 16; o >= 1; o >>= 1) best = fmaxf(best, __shfl_xor_sync(kFull, best, o));
      // word lane + 32 c of row r: chunk (lane + 32 c) / 4, word (lane % 4) of it
      auto word_at = [&](int r, int c) -> uint32_t {
        const int w = lane + 32 * c;
        return *reinterpret_cast<const uint32_t*>(t + meta_swz(bs, r, w >> 2) + ((w & 3) << 2));
      };
      float s[WL][P];
#pragma unroll
      for (int c = 0; c < WL; ++c)
#pragma unroll
        for (int p = 0; p < P; ++p) s[c][p] = 0.0f;
      for (int r = 0; r < bs; ++r) {
#pragma unroll
        for (int c = 0; c < WL; ++c) {
          float x[P];
          widen_word<KV>(word_at(r, c), x);
#pragma unroll
          for (int p = 0; p < P; ++p) s[c][p] = __fadd_rn(s[c][p], x[p]);
        }
      }
      float v[WL][P];
#pragma unroll
      for (int c = 0; c < WL; ++c)
#pragma unroll
        for (int p = 0; p < P; ++p) {
          s[c][p] = __fdiv_rn(s[c][p], rows);  // the mean
          v[c][p] = 0.0f;
        }
      for (int r = 0; r < bs; ++r) {
#pragma unroll
        for (int c = 0; c < WL; ++c) {
          float x[P];
          widen_word<KV>(word_at(r, c), x);
#pragma unroll
          for (int p = 0; p < P; ++p) {
            const float e = __fsub_rn(x[p], s[c][p]);
            v[c][p] = __fmaf_rn(e, e, v[c][p]);
          }
        }
      }
      const int64_t bh = i / nblk;
      const int64_t j = blk_begin + (i - bh * nblk);
#pragma unroll
      for (int c = 0; c < WL; ++c)
#pragma unroll
        for (int p = 0; p < P; ++p) {
          const int idx = (lane + 32 * c) * P + p;
          const int64_t o = (bh * D + idx) * nb_cap + j;
          mu[o] = s[c][p];
          var[o] = __fdiv_rn(v[c][p], rows);
        }
      if (lane == 0) maxn[bh * nb_cap + j] = __fsqrt_rn(best);
    }
    __syncwarp();  // every lane is done with the buffer before the next round refills it
  }
  asm volatile("cp.async.wait_all;" ::: "memory");  // nothing in flight when the warp exits
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
  // blocks of 8 to 16 KB, and fp8 blocks: the staged kernel, one thread block
  // per SM with 192 KB of buffers (8 warps x 3 buffers of up to 8 KB, 6 x 2 of
  // up to 16 KB). Measured on 2 GiB of keys: 1,044 -> 925 us (b 32, d 128),
  // 1,150 -> 847 us (b 64, d 128), 839 -> 695 us (b 64, d 64), fp8 2,259 -> ~880
  // us; smaller bf16 / fp32 blocks keep meta_kernel, whose many resident warps
  // hide the load latency better (b 16, d 128: 2,637 against 2,954 us staged).
  const size_t tile = static_cast<size_t>(bs) * D * KvTraits<KV>::kBytes;
  const bool fp8 = KvTraits<KV>::kDtype == ETA_FP8_E4M3;
  if (tile <= 16 * 1024 && (fp8 || tile >= 8 * 1024)) {
    const int64_t items = static_cast<int64_t>(s.batch) * s.n_kv_heads * (b1 - b0);
    const int nb = tile <= 8 * 1024 ? 3 : 2;
    const size_t fit = (192 * 1024) / (nb * tile);
    const int warps = static_cast<int>(fit < kMetaWarps ? fit : kMetaWarps);
    const size_t smem = static_cast<size_t>(warps) * nb * tile;
    const void* fn = nb == 3 ? reinterpret_cast<const void*>(meta_staged_kernel<KV, D, 3>)
                             : reinterpret_cast<const void*>(meta_staged_kernel<KV, D, 2>);
    static std::atomic<uint64_t> smem_done3{0}, smem_done2{0};
    cudaError_t e = allow_max_smem(nb == 3 ? smem_done3 : smem_done2, fn);
    if (e != cudaSuccess) return e;
    const int64_t want = (items + warps - 1) / warps;
    const unsigned g = static_cast<unsigned>(want < device_sm_count() ? want : device_sm_count());
    if (nb == 3)
      meta_staged_kernel<KV, D, 3><<<g, warps * 32, smem, st>>>(static_cast<const KV*>(k), L, nb_cap, b0, b1 - b0,
                                                                items, m.mu, m.var, m.maxnorm);
    else
      meta_staged_kernel<KV, D, 2><<<g, warps * 32, smem, st>>>(static_cast<const KV*>(k), L, nb_cap, b0, b1 - b0,
                                                                items, m.mu, m.var, m.maxnorm);
    return cudaGetLastError();
  }
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

// Block screening (Methodology §4, Eq. 5 and the admission rule) with
// compaction into ascending active-block lists.
//
// One thread-block cluster per (batch, kv head). Each CTA of the cluster scores
// a contiguous range of 32-block tiles, one warp lane per block and all G query
// heads of the GQA group at once (the metadata is read once per group). A warp
// scores 4 consecutive tiles together: the metadata is coordinate-major, so
// for every coordinate i it reads 512 contiguous bytes of mu and of var, with
// the loads of several coordinates in flight. Per-tile admission counts give the CTA's
// local offsets; the CTAs exchange their totals through distributed shared
// memory, so the cluster writes one globally ascending list without another
// launch. The union over the group (the blocks that must be loaded, with a
// per-head bit mask) is written beside the per-head lists.
#include <cooperative_groups.h>

#include "common.cuh"
#include "launch.h"

namespace cg = cooperative_groups;

namespace eta {

namespace {

constexpr int kScreenWarps = 4;
constexpr int kSub = 4;  // tiles a warp scores together

struct ScreenArgs {
  const void* q;
  int q_dtype;
  const float* mu;
  const float* var;
  const float* maxn;
  const float* tau;
  int64_t tau_stride;
  float z, s, offset_a;
  int Hq, Hkv, nb, ns, nb_cap, tiles_per_cta;
  uint32_t* ws_union;
  int32_t* ws_union_cnt;
  int32_t* ws_head_cnt;
  int32_t* active_idx;
  int32_t* active_cnt;
  uint32_t* union_out;
  int32_t* union_cnt_out;
  float* scores;
};

__device__ __forceinline__ uint32_t lanemask_lt() {
  uint32_t m;
  asm("mov.u32 %0, %%lanemask_lt;" : "=r"(m));
  return m;
}

template <int D, int G>
__global__ void __launch_bounds__(kScreenWarps * 32) screen_kernel(const ScreenArgs a) {
  cg::cluster_group cluster = cg::this_cluster();
  const int cs = static_cast<int>(cluster.num_blocks());
  const int cr = static_cast<int>(cluster.block_rank());
  const int bh = blockIdx.x / cs;
  const int b = bh / a.Hkv, kvh = bh % a.Hkv;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int tpc = a.tiles_per_cta;

  extern __shared__ __align__(16) unsigned char smem[];
  float* s_q = reinterpret_cast<float*>(smem);   // [G][D]
  float* s_qq = s_q + G * D;                      // [G][D] fl(q_i * q_i)
  float* s_qn = s_qq + G * D;                     // [G] fl(sqrt(sum q_i^2))
  float* s_taut = s_qn + 16;                      // [G] tau - a
  int* s_tot = reinterpret_cast<int*>(s_taut + 16);  // [G+1] this CTA's admitted counts
  int* s_base = s_tot + 16;                       // [G+1] counts of lower-ranked CTAs
  int* s_tcnt = s_base + 16;                      // [tpc][G+1] per-tile counts -> offsets
  uint8_t* s_mask = reinterpret_cast<uint8_t*>(s_tcnt + tpc * (G + 1));  // [tpc*32]

  for (int i = tid; i < G * D; i += kScreenWarps * 32) {
    const int g = i / D, e = i % D;
    const float x = load_elem(a.q, a.q_dtype, (static_cast<int64_t>(b) * a.Hq + kvh * G + g) * D + e);
    s_q[i] = x;
    s_qq[i] = __fmul_rn(x, x);
  }
  __syncthreads();
  if (tid < G) {
    float qn = 0.0f;
    for (int e = 0; e < D; ++e) qn = __fmaf_rn(s_q[tid * D + e], s_q[tid * D + e], qn);
    s_qn[tid] = __fsqrt_rn(qn);
    s_taut[tid] = __fsub_rn(a.tau[b * a.tau_stride + kvh * G + tid], a.offset_a);
  }
  __syncthreads();

  const int nt = (a.ns + 31) / 32;
  const int t0 = cr * tpc;
  const int my_tiles = max(0, min(nt, t0 + tpc) - t0);
  const float* mu = a.mu + static_cast<int64_t>(bh) * D * a.nb_cap;
  const float* var = a.var + static_cast<int64_t>(bh) * D * a.nb_cap;
  const float* mx = a.maxn + static_cast<int64_t>(bh) * a.nb_cap;

  // Phase 1: score and decide every screened block of this CTA's tiles.
  for (int t4 = warp * kSub; t4 < my_tiles; t4 += kScreenWarps * kSub) {
    int cb[kSub];
    bool valid[kSub];
#pragma unroll
    for (int u = 0; u < kSub; ++u) {
      const int blk = (t0 + t4 + u) * 32 + lane;
      valid[u] = (t4 + u < my_tiles) && blk < a.ns;
      cb[u] = blk < a.ns ? blk : a.ns - 1;
    }
    float dg[kSub][G], vg[kSub][G];
#pragma unroll
    for (int u = 0; u < kSub; ++u)
#pragma unroll
      for (int g = 0; g < G; ++g) dg[u][g] = vg[u][g] = 0.0f;
#pragma unroll 8
    for (int i = 0; i < D; ++i) {
      float m[kSub], v[kSub];
#pragma unroll
      for (int u = 0; u < kSub; ++u) {
        m[u] = __ldg(mu + static_cast<int64_t>(i) * a.nb_cap + cb[u]);
        v[u] = __ldg(var + static_cast<int64_t>(i) * a.nb_cap + cb[u]);
      }
#pragma unroll
      for (int g = 0; g < G; ++g) {
        const float qi = s_q[g * D + i], qqi = s_qq[g * D + i];
#pragma unroll
        for (int u = 0; u < kSub; ++u) {
          dg[u][g] = __fmaf_rn(qi, m[u], dg[u][g]);
          vg[u][g] = __fmaf_rn(qqi, v[u], vg[u][g]);
        }
      }
    }
#pragma unroll
    for (int u = 0; u < kSub; ++u) {
      if (t4 + u >= my_tiles) break;  // uniform over the warp
      const int t = t4 + u;
      const int blk = (t0 + t) * 32 + lane;
      const float M = __ldg(mx + cb[u]);
      uint32_t mask = 0;
#pragma unroll
      for (int g = 0; g < G; ++g) {
        const float A = __fadd_rn(dg[u][g], __fmul_rn(a.z, __fsqrt_rn(vg[u][g])));
        const float C = __fmul_rn(s_qn[g], M);
        const float sc = __fmul_rn((A < C) ? A : C, a.s);
        if (valid[u] && !(sc < s_taut[g])) mask |= 1u << g;
        if (a.scores != nullptr && valid[u])
          a.scores[(static_cast<int64_t>(b) * a.Hq + kvh * G + g) * a.nb_cap + blk] = sc;
      }
      s_mask[t * 32 + lane] = static_cast<uint8_t>(mask);
      int cnt[G + 1];
#pragma unroll
      for (int g = 0; g < G; ++g) cnt[g] = __popc(__ballot_sync(kFull, (mask >> g) & 1u));
      cnt[G] = __popc(__ballot_sync(kFull, mask != 0u));
      if (lane == 0) {
#pragma unroll
        for (int c = 0; c <= G; ++c) s_tcnt[t * (G + 1) + c] = cnt[c];
      }
    }
  }
  __syncthreads();

  // Phase 2: exclusive prefix over this CTA's tiles, per head and for the union.
  if (tid <= G) {
    int run = 0;
    for (int t = 0; t < my_tiles; ++t) {
      const int v = s_tcnt[t * (G + 1) + tid];
      s_tcnt[t * (G + 1) + tid] = run;
      run += v;
    }
    s_tot[tid] = run;
  }

  // Phase 3: offsets of this CTA inside the cluster's lists (distributed shared memory).
  cluster.sync();
  if (tid <= G) {
    int base = 0;
    for (int r = 0; r < cr; ++r) base += cluster.map_shared_rank(s_tot, r)[tid];
    s_base[tid] = base;
  }
  cluster.sync();

  // Phase 4: write the compacted lists.
  const uint32_t lt = lanemask_lt();
  for (int t = warp; t < my_tiles; t += kScreenWarps) {
    const int blk = (t0 + t) * 32 + lane;
    const uint32_t mask = s_mask[t * 32 + lane];
#pragma unroll
    for (int g = 0; g < G; ++g) {
      const bool on = (mask >> g) & 1u;
      const uint32_t bal = __ballot_sync(kFull, on);
      if (on && a.active_idx != nullptr) {
        const int pos = s_base[g] + s_tcnt[t * (G + 1) + g] + __popc(bal & lt);
        a.active_idx[(static_cast<int64_t>(b) * a.Hq + kvh * G + g) * a.nb_cap + pos] = blk;
      }
    }
    const bool any = mask != 0u;
    const uint32_t balu = __ballot_sync(kFull, any);
    if (any) {
      const int pos = s_base[G] + s_tcnt[t * (G + 1) + G] + __popc(balu & lt);
      const uint32_t entry = (static_cast<uint32_t>(blk) << 8) | mask;
      a.ws_union[static_cast<int64_t>(bh) * a.nb_cap + pos] = entry;
      if (a.union_out != nullptr) a.union_out[static_cast<int64_t>(bh) * a.nb_cap + pos] = entry;
    }
  }

  // The last CTA appends the forced trailing blocks and writes the counts.
  if (cr == cs - 1) {
    const int nf = a.nb - a.ns;
    const uint32_t all = (1u << G) - 1u;
    for (int j = tid; j < nf; j += kScreenWarps * 32) {
      const int blk = a.ns + j;
      if (a.active_idx != nullptr) {
#pragma unroll
        for (int g = 0; g < G; ++g)
          a.active_idx[(static_cast<int64_t>(b) * a.Hq + kvh * G + g) * a.nb_cap + s_base[g] + s_tot[g] + j] = blk;
      }
      const uint32_t entry = (static_cast<uint32_t>(blk) << 8) | all;
      const int64_t o = static_cast<int64_t>(bh) * a.nb_cap + s_base[G] + s_tot[G] + j;
      a.ws_union[o] = entry;
      if (a.union_out != nullptr) a.union_out[o] = entry;
    }
    if (tid < G) {
      const int c = s_base[tid] + s_tot[tid] + nf;
      const int64_t hq = static_cast<int64_t>(b) * a.Hq + kvh * G + tid;
      a.ws_head_cnt[hq] = c;
      if (a.active_cnt != nullptr) a.active_cnt[hq] = c;
    } else if (tid == G) {
      const int c = s_base[G] + s_tot[G] + nf;
      a.ws_union_cnt[bh] = c;
      if (a.union_cnt_out != nullptr) a.union_cnt_out[bh] = c;
    }
  }
}

template <int D, int G>
cudaError_t launch_screen_t(const ScreenCall& c, cudaStream_t st) {
  const eta_shape_t& s = c.shape;
  const int BH = s.batch * s.n_kv_heads;
  const int64_t nb_cap = s.capacity / s.block_size;
  const int nb = static_cast<int>((c.n + s.block_size - 1) / s.block_size);
  const int ns = max(0, nb - c.n_local);
  const int nt = (ns + 31) / 32;
  // As many CTAs per cluster as there are tiles, up to kMaxCluster: the tiles
  // of a (batch, kv head) spread evenly, each warp scoring kSub at a time.
  int cs = max(1, min(kMaxCluster, nt));
  while ((nt + cs - 1) / cs > kMaxScreenTiles && cs < kMaxCluster) ++cs;
  const int tpc = max(1, (nt + cs - 1) / cs);
  if (tpc > kMaxScreenTiles) return cudaErrorInvalidValue;

  ScreenArgs a;
  a.q = c.q;
  a.q_dtype = s.q_dtype;
  a.mu = c.meta.mu;
  a.var = c.meta.var;
  a.maxn = c.meta.maxnorm;
  a.tau = c.tau;
  a.tau_stride = c.tau_stride;
  a.z = c.z;
  a.s = static_cast<float>(1.0 / std::sqrt(static_cast<double>(s.head_dim)));
  a.offset_a = c.offset_a;
  a.Hq = s.n_q_heads;
  a.Hkv = s.n_kv_heads;
  a.nb = nb;
  a.ns = ns;
  a.nb_cap = static_cast<int>(nb_cap);
  a.tiles_per_cta = tpc;
  a.ws_union = c.ws.union_list;
  a.ws_union_cnt = c.ws.union_cnt;
  a.ws_head_cnt = c.ws.head_cnt;
  a.active_idx = c.out.active_idx;
  a.active_cnt = c.out.active_cnt;
  a.union_out = c.out.union_list;
  a.union_cnt_out = c.out.union_cnt;
  a.scores = c.out.scores;

  const size_t smem = (2 * G * D + 32) * sizeof(float) + 32 * sizeof(int) +
                      static_cast<size_t>(tpc) * (G + 1) * sizeof(int) + static_cast<size_t>(tpc) * 32;
  static std::atomic<uint64_t> smem_done{0};
  cudaError_t e = allow_max_smem(smem_done, reinterpret_cast<const void*>(screen_kernel<D, G>));
  if (e != cudaSuccess) return e;

  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(BH * cs));
  cfg.blockDim = dim3(kScreenWarps * 32);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = static_cast<unsigned>(cs);
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  e = cudaLaunchKernelEx(&cfg, screen_kernel<D, G>, a);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

template <int D>
cudaError_t launch_screen_d(const ScreenCall& c, cudaStream_t st) {
  switch (c.shape.n_q_heads / c.shape.n_kv_heads) {
    case 1: return launch_screen_t<D, 1>(c, st);
    case 2: return launch_screen_t<D, 2>(c, st);
    case 4: return launch_screen_t<D, 4>(c, st);
    case 8: return launch_screen_t<D, 8>(c, st);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace

cudaError_t launch_screen(const ScreenCall& c, cudaStream_t st) {
  return c.shape.head_dim == 128 ? launch_screen_d<128>(c, st) : launch_screen_d<64>(c, st);
}

}  // namespace eta

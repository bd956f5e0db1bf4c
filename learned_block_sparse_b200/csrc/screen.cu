// Block screening (Methodology §4, Eq. 5 and the admission rule) with
// compaction into ascending active-block lists — plain-load kernel, used when
// the metadata rows are not aligned for TMA (capacity/block_size not a
// multiple of 4); otherwise screen_tma.cu stages the metadata tiles.
//
// One thread-block cluster per (batch, kv head). Each CTA of the cluster scores
// a contiguous range of 32-block tiles, one warp lane per block and all G query
// heads of the GQA group at once (the metadata is read once per group). A warp
// scores 4 consecutive tiles together: the metadata is coordinate-major, so
// for every coordinate i it reads 512 contiguous bytes of mu and of var, with
// the loads of several coordinates in flight. Per-tile admission counts give
// the CTA's local offsets; the CTAs exchange their totals through distributed
// shared memory, so the cluster writes one globally ascending list without
// another launch. The union over the group (the blocks that must be loaded,
// with a per-head bit mask) is written beside the per-head lists.
#include "screen_common.cuh"

namespace cg = cooperative_groups;

namespace eta {

namespace {

constexpr int kScreenWarps = 4;
constexpr int kSub = 4;  // tiles a warp scores together

template <int D, int G>
__global__ void __launch_bounds__(kScreenWarps * 32, 4) screen_kernel(const ScreenArgs a) {
  cg::cluster_group cluster = cg::this_cluster();
  const int cs = static_cast<int>(cluster.num_blocks());
  const int cr = static_cast<int>(cluster.block_rank());
  const int bh = blockIdx.x / cs;
  const int b = bh / a.Hkv, kvh = bh % a.Hkv;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int tpc = a.tiles_per_cta;

  extern __shared__ __align__(16) unsigned char smem[];
  const ScreenSmem<D, G> sm(smem, tpc);
  grid_dependency_wait();  // inputs may come from the previous kernel on the stream
  allow_dependent_launch();
  screen_prologue<D, G, 32, true>(a, sm, b, kvh, kScreenWarps * 32);

  const RowBlocks rb = row_blocks(a, b);
  const int units = rb.ns * a.r;  // screened metadata columns (sub-blocks)
  const int nt = (units + 31) / 32;
  const int t0 = cr * tpc;
  const int my_tiles = max(0, min(nt, t0 + tpc) - t0);
  const float* mu = a.mu + static_cast<int64_t>(bh) * D * a.nb_cap_meta;
  const float* var = a.var + static_cast<int64_t>(bh) * D * a.nb_cap_meta;
  const float* mx = a.maxn + static_cast<int64_t>(bh) * a.nb_cap_meta;

  // Phase 1: score and decide every screened block of this CTA's tiles.
  for (int t4 = warp * kSub; t4 < my_tiles; t4 += kScreenWarps * kSub) {
    int cb[kSub];
    bool valid[kSub];
#pragma unroll
    for (int u = 0; u < kSub; ++u) {
      const int unit = (t0 + t4 + u) * 32 + lane;
      valid[u] = (t4 + u < my_tiles) && unit < units;
      cb[u] = unit < units ? unit : units - 1;  // units >= 1 here (this warp has a tile)
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
        m[u] = __ldg(mu + static_cast<int64_t>(i) * a.nb_cap_meta + cb[u]);
        v[u] = __ldg(var + static_cast<int64_t>(i) * a.nb_cap_meta + cb[u]);
      }
#pragma unroll
      for (int g = 0; g < G; ++g) {
        const float qi = sm.q[i * G + g], qqi = sm.qq[i * G + g];
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
      const uint32_t mask =
          screen_decide<D, G>(a, sm, b, kvh, (t0 + t) * 32 + lane, valid[u], dg[u], vg[u], __ldg(mx + cb[u]));
      screen_record_tile<D, G>(sm, t, mask);
    }
  }
  __syncthreads();
  screen_finish<D, G>(a, sm, b, kvh, bh, t0, my_tiles, rb, kScreenWarps * 32);
}

template <int D, int G>
cudaError_t launch_screen_t(const ScreenCall& c, cudaStream_t st) {
  const eta_shape_t& s = c.shape;
  const int BH = s.batch * s.n_kv_heads;
  const int nb = static_cast<int>((c.n + s.block_size - 1) / s.block_size);
  const int ns = max(0, nb - c.n_local);
  const int nt = (ns * c.sub_blocks + 31) / 32;
  // As many CTAs per cluster as there are tiles, up to kMaxCluster.
  const int cs = max(1, min(kMaxCluster, nt));
  const int tpc = max(1, (nt + cs - 1) / cs);
  if (tpc > kMaxScreenTiles) return cudaErrorInvalidValue;
  const ScreenArgs a = make_screen_args(c, nb, ns, tpc);
  static std::atomic<uint64_t> smem_done{0};
  cudaError_t e = allow_max_smem(smem_done, reinterpret_cast<const void*>(screen_kernel<D, G>));
  if (e != cudaSuccess) return e;
  return launch_clusters(screen_kernel<D, G>, a, BH, cs, kScreenWarps * 32, ScreenSmem<D, G>::bytes(tpc), st);
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
  const cudaError_t e = launch_screen_tma(c, st);
  if (e != cudaErrorNotSupported) return e;
  return c.shape.head_dim == 128 ? launch_screen_d<128>(c, st) : launch_screen_d<64>(c, st);
}

}  // namespace eta

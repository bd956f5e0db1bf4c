// Block screening (Methodology §4, Eq. 5 and the admission rule) with the
// metadata tiles staged by TMA.
//
// Same cluster layout and compaction as screen.cu (one cluster per (batch, kv
// head), lane = block, all G heads of the group per metadata read). Here a
// producer warp streams each 32-block tile's metadata, one 2-D box of
// [d coordinates][32 blocks] of mu and one of var (32 KB at d = 128), into a
// ring of shared-memory stages; consumer warps take the tiles in increasing
// order from a shared counter and score them from shared memory (lane =
// column, so the reads are conflict-free) with the multiply-adds in increasing
// coordinate order. The warps that form the Eq. 1 thresholds join the
// consumers once the thresholds are in (at once without a predictor); tiles
// scored before then keep their scores in shared memory and are decided after
// the last tile, so the ring does not wait for the thresholds. The ring
// keeps several tiles in flight per SM even when a (batch, kv head) has few
// tiles, which plain loads from a handful of warps cannot. Since any warp may
// take any tile, the producer publishes the round each stage serves (after the
// stage's previous release) and a consumer waits for its tile's round before
// the barrier parity wait, which is then exact.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <mutex>

#include "screen_common.cuh"

namespace cg = cooperative_groups;

namespace eta {

namespace {

// 96 KB of stages at d = 128, 80 KB at d = 64: with the per-tile bookkeeping
// of up to 256 tiles, two thread blocks fit per SM (six stages at d = 64 left
// one thread block per SM: 279 against 236 us on the Table 10 shape). (Measured
// and not kept: each tile's coordinates as two ring positions of half the
// size, so a warp frees half a stage before it has scored the whole tile and
// twice as many warps score at once: 63 against 64 us at d = 128, G = 4; 301
// against 279 us at d = 64, G = 8. And one flat split of all pairs' tiles
// over the resident thread blocks, with the list offsets passed between them
// in global memory: 72 against 66 us at d = 128, G = 4, 238 against 236 us on
// the Table 10 shape; the SMs' unequal shares of the bandwidth, not the
// tiles per SM, set the finish.)
template <int D> struct TmaScreenCfg;
template <> struct TmaScreenCfg<128> { static constexpr int kCW = 3, kNST = 3; };
template <> struct TmaScreenCfg<64> { static constexpr int kCW = 3, kNST = 5; };
// Warps that form the Eq. 1 thresholds (when the call passes a predictor)
// while the ring streams the first tiles, then score tiles too: the first
// consumers score tiles and release their stages without waiting for the
// thresholds, and wait only before their first admission decision.
constexpr int kTauWarps = 4;
// Tiles whose Eq. 5 scores may wait in shared memory for the thresholds: the
// consumers score and release a stage before the Eq. 1 thresholds are in and
// decide those tiles after the last one, instead of stalling the ring. Fewer
// at d = 128, G = 8, where shared memory is tightest.
template <int D, int G>
constexpr int kTmaDefer = (D == 128 && G == 8) ? 4 : 8;

// Bytes between the stages and ScreenSmem: full and empty barriers, the
// threshold barrier (+ 8 bytes padding), the abort flag, the tile counter, the
// deferred-tile count (+ 4 bytes padding), the round of every stage (padded to
// 16 bytes).
template <int NST>
constexpr size_t kTmaBarBytes = (2 * NST + 2) * sizeof(uint64_t) + (4 + (NST + 3) / 4 * 4) * sizeof(int);

__device__ __forceinline__ void tma_load_2d_plain(void* dst, const CUtensorMap* tm, int x, int y, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];" ::"r"(
          smem_u32(dst)),
      "l"(tm), "r"(x), "r"(y), "r"(smem_u32(bar))
      : "memory");
}

// Non-blocking: has the phase of `bar` with the given parity completed?
__device__ __forceinline__ bool mbar_test_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\tmbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\tselp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// Packed fp32 pairs: fma.rn.f32x2 / mul.rn.f32x2 perform two independent IEEE
// fused multiply-adds / multiplies, each rounding as __fmaf_rn / __fmul_rn do.
__device__ __forceinline__ uint64_t pack2(float lo, float hi) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
  return r;
}
__device__ __forceinline__ void fma2(uint64_t& acc, uint64_t a, uint64_t b) {
  asm("fma.rn.f32x2 %0, %1, %2, %0;" : "+l"(acc) : "l"(a), "l"(b));
}
__device__ __forceinline__ uint64_t mul2(uint64_t a, uint64_t b) {
  uint64_t r;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}
__device__ __forceinline__ void unpack2(uint64_t v, float& lo, float& hi) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}

template <int D, int G>
__global__ void __launch_bounds__((TmaScreenCfg<D>::kCW + 1 + kTauWarps) * 32, 2)
    screen_tma_kernel(const ScreenArgs a, int32_t* status, const __grid_constant__ CUtensorMap tmu,
                      const __grid_constant__ CUtensorMap tvar) {
  constexpr int CW = TmaScreenCfg<D>::kCW;
  constexpr int NST = TmaScreenCfg<D>::kNST;
  constexpr int NT = (CW + 1 + kTauWarps) * 32;  // consumers, producer, threshold warps
  constexpr uint32_t kBox = D * 32 * sizeof(float);  // one array's tile
  cg::cluster_group cluster = cg::this_cluster();
  const int cs = static_cast<int>(cluster.num_blocks());
  const int cr = static_cast<int>(cluster.block_rank());
  const int bh = blockIdx.x / cs;
  const int b = bh / a.Hkv, kvh = bh % a.Hkv;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int tpc = a.tiles_per_cta;

  extern __shared__ __align__(16) unsigned char smem_raw[];
  unsigned char* smem = smem_raw + ((128 - (smem_u32(smem_raw) & 127)) & 127);
  float* s_stage = reinterpret_cast<float*>(smem);  // [NST][2][D][32]
  uint64_t* s_full = reinterpret_cast<uint64_t*>(smem + static_cast<size_t>(NST) * 2 * kBox);
  uint64_t* s_empty = s_full + NST;
  uint64_t* s_tau = s_empty + NST;  // completes when the thresholds are in sm.taut
  int* s_abort = reinterpret_cast<int*>(s_tau + 2);
  int* s_next = s_abort + 1;     // next tile to hand out
  int* s_ndefer = s_abort + 2;   // tiles deferred
  int* s_round = s_abort + 4;    // [NST] round each stage serves
  // the query rows are read as float4: ScreenSmem must start 16-byte aligned
  static_assert((static_cast<size_t>(NST) * 2 * kBox + kTmaBarBytes<NST>) % 16 == 0, "ScreenSmem alignment");
  const ScreenSmem<D, G> sm(smem + static_cast<size_t>(NST) * 2 * kBox + kTmaBarBytes<NST>, tpc);
  constexpr int ND = kTmaDefer<D, G>;
  float* s_defer = reinterpret_cast<float*>(smem + static_cast<size_t>(NST) * 2 * kBox + kTmaBarBytes<NST> +
                                            ScreenSmem<D, G>::bytes(tpc));  // [ND][G][32] scores
  int* s_defer_it = reinterpret_cast<int*>(s_defer + ND * G * 32);          // [ND] their tiles

  const float* mx = a.maxn + static_cast<int64_t>(bh) * a.nb_cap_meta;

  if (tid == 0) {
    *s_abort = 0;
    *s_next = 0;
    *s_ndefer = 0;
    for (int s = 0; s < NST; ++s) {
      mbar_init(&s_full[s], 1);
      mbar_init(&s_empty[s], 1);
      s_round[s] = 0;
    }
    mbar_init(s_tau, 1);
    fence_mbar_init();
  }
  grid_dependency_wait();  // inputs may come from the previous kernel on the stream
  allow_dependent_launch();
  const RowBlocks rb = row_blocks(a, b);
  const int units = rb.ns * a.r;  // screened metadata columns (sub-blocks)
  const int nt = (units + 31) / 32;
  const int t0 = cr * tpc;
  const int my_tiles = max(0, min(nt, t0 + tpc) - t0);
  __syncthreads();
  auto issue_tile = [&](int it) {
    const int st = it % NST;
    mbar_arrive_expect_tx(&s_full[st], 2 * kBox);
    const int x = (t0 + it) * 32, y = bh * D;
    tma_load_2d_plain(s_stage + static_cast<size_t>(st) * 2 * D * 32, &tmu, x, y, &s_full[st]);
    tma_load_2d_plain(s_stage + (static_cast<size_t>(st) * 2 + 1) * D * 32, &tvar, x, y, &s_full[st]);
  };
  // the first ring of tiles does not depend on the queries: start it now
  const int first = my_tiles < NST ? my_tiles : NST;
  int issued = 0;  // producer lane: 1 + the last tile it armed
  if (warp == CW && lane == 0) {
    for (int it = 0; it < first; ++it) issue_tile(it);
    issued = first;
  }
  screen_prologue<D, G, 32, false>(a, sm, b, kvh, NT);  // ends with __syncthreads
  const bool tau_later = a.W != nullptr;

  // Consumers: take tiles in increasing order until none is left. tau_ready:
  // the thresholds are in sm.taut already (no wait before the decisions).
  // Before they are in, a tile's scores go to a free deferral slot; with none
  // free, the warp waits for them.
  auto consume = [&](bool tau_ready) {
    bool tau_ok = true;
    bool tau_have = tau_ready;
    volatile int* rounds = s_round;
    for (;;) {
      int it = 0;
      if (lane == 0) it = atomicAdd(s_next, 1);
      it = __shfl_sync(kFull, it, 0);
      if (it >= my_tiles) break;
      const int unit = (t0 + it) * 32 + lane;
      const bool valid = unit < units;
      const float M = __ldg(mx + (valid ? unit : units - 1));  // units >= 1 here (this CTA has a tile)
      // the stage serves this tile once the producer has published its round
      // (after the previous round's release): the parity wait is then exact
      const int st = it % NST, round = it / NST;
      bool ok = round == 0 || wait_value_bounded(rounds + st, round, s_abort, status);
      ok = __all_sync(kFull, ok && mbar_wait_bounded(&s_full[st], static_cast<uint32_t>(round & 1), s_abort, status));
      float dg[G], vg[G];
#pragma unroll
      for (int g = 0; g < G; ++g) dg[g] = vg[g] = 0.0f;
      if (ok) {
        const float* mu_s = s_stage + static_cast<size_t>(st) * 2 * D * 32;
        const float* var_s = mu_s + D * 32;
        if constexpr (G == 1) {
#pragma unroll 2
          for (int i0 = 0; i0 < D; i0 += 4) {
            // four coordinates of q and q*q per shared load; multiply-adds in coordinate order
            const float4 qv = *reinterpret_cast<const float4*>(sm.q + i0);
            const float4 qqv = *reinterpret_cast<const float4*>(sm.qq + i0);
            const float qa[4] = {qv.x, qv.y, qv.z, qv.w}, qqa[4] = {qqv.x, qqv.y, qqv.z, qqv.w};
#pragma unroll
            for (int c = 0; c < 4; ++c) {
              dg[0] = __fmaf_rn(qa[c], mu_s[(i0 + c) * 32 + lane], dg[0]);
              vg[0] = __fmaf_rn(qqa[c], var_s[(i0 + c) * 32 + lane], vg[0]);
            }
          }
        } else {
          // heads 2p and 2p+1 share a packed multiply-add per coordinate: the
          // [D][G] query rows give both of a coordinate's factors in one load,
          // and fl(q q) of both in one packed multiply (the prologue's squares,
          // bit for bit), which saves the shared loads of the squares
          const uint64_t* q2 = reinterpret_cast<const uint64_t*>(sm.q);
          uint64_t d2[G / 2], v2[G / 2];
#pragma unroll
          for (int p = 0; p < G / 2; ++p) d2[p] = v2[p] = 0ull;  // +0.0f in both halves
#pragma unroll 4
          for (int i0 = 0; i0 < D; i0 += 4) {
            float m[4], v[4];
#pragma unroll
            for (int c = 0; c < 4; ++c) {
              m[c] = mu_s[(i0 + c) * 32 + lane];
              v[c] = var_s[(i0 + c) * 32 + lane];
            }
#pragma unroll
            for (int c = 0; c < 4; ++c) {
              const uint64_t mm = pack2(m[c], m[c]), vv = pack2(v[c], v[c]);
#pragma unroll
              for (int p = 0; p < G / 2; ++p) {
                const uint64_t qp = q2[(i0 + c) * (G / 2) + p];
                fma2(d2[p], qp, mm);
                fma2(v2[p], mul2(qp, qp), vv);
              }
            }
          }
#pragma unroll
          for (int p = 0; p < G / 2; ++p) {
            unpack2(d2[p], dg[2 * p], dg[2 * p + 1]);
            unpack2(v2[p], vg[2 * p], vg[2 * p + 1]);
          }
        }
      }
      __syncwarp();
      if (ok && lane == 0) mbar_arrive(&s_empty[st]);  // a stage whose wait failed is not released
      float sc[G];
      screen_scores<D, G>(a, sm, dg, vg, M, sc);
      if (!tau_have && __all_sync(kFull, mbar_test_wait(s_tau, 0u))) tau_have = true;
      if (!tau_have) {
        int slot = 0;
        if (lane == 0) slot = atomicAdd(s_ndefer, 1);
        slot = __shfl_sync(kFull, slot, 0);
        if (slot < ND) {
#pragma unroll
          for (int g = 0; g < G; ++g) s_defer[(slot * G + g) * 32 + lane] = sc[g];
          if (lane == 0) s_defer_it[slot] = it;
          continue;
        }
        tau_ok = mbar_wait_bounded(s_tau, 0u, s_abort, status);
        tau_have = true;
      }
      screen_record_tile<D, G>(sm, it, screen_admit<D, G>(a, sm, b, kvh, unit, valid && tau_ok, sc));
    }
  };

  if (warp > CW) {
    // ----------------------------------------------------- threshold warps
    if (tau_later) {
      constexpr int kTauThreads = kTauWarps * 32;
      screen_predict_tau<D, G, 32>(a, sm, b, kvh, tid - (CW + 1) * 32, kTauThreads,
                                   [] { named_barrier_sync(2, kTauThreads); });
      named_barrier_sync(2, kTauThreads);  // every taut written before the release
      if (tid == (CW + 1) * 32) mbar_arrive(s_tau);
    }
    consume(true);  // then score tiles like the other consumers
  } else if (warp == CW) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      volatile int* abort_flag = s_abort;
      volatile int* rounds = s_round;
      for (int it = first; it < my_tiles; ++it) {
        const int st = it % NST, round = it / NST;
        // a consumer that gave up does not release its stage: stop arming
        if (!mbar_wait_bounded(&s_empty[st], (round - 1) & 1, s_abort, status) || *abort_flag) break;
        rounds[st] = round;  // this stage now serves round `round`
        issue_tile(it);
        issued = it + 1;
      }
    }
  } else {
    // ----------------------------------------------------------- consumers
    consume(!tau_later);
  }
  __syncthreads();
  if (warp == CW && lane == 0 && *reinterpret_cast<volatile int*>(s_abort)) {
    // a wait gave up: let the copies of the last use of every stage land before
    // the thread block can exit (earlier uses completed before their re-arm)
    for (int j = max(0, issued - NST); j < issued; ++j) {
      const uint64_t tstart = global_timer_ns();
      while (!mbar_try_wait(&s_full[j % NST], (j / NST) & 1) && global_timer_ns() - tstart < kWaitLimitNs) {
      }
    }
  }
  // Deferred tiles: the thresholds are in (the threshold warps arrived before
  // they joined the consumers, all of which are past the barrier above).
  const int nd = min(*reinterpret_cast<volatile int*>(s_ndefer), ND);
  for (int slot = warp; slot < nd; slot += NT / 32) {
    const int it = s_defer_it[slot];
    const int unit = (t0 + it) * 32 + lane;
    float sc[G];
#pragma unroll
    for (int g = 0; g < G; ++g) sc[g] = s_defer[(slot * G + g) * 32 + lane];
    screen_record_tile<D, G>(sm, it, screen_admit<D, G>(a, sm, b, kvh, unit, unit < units, sc));
  }
  __syncthreads();
  screen_finish<D, G>(a, sm, b, kvh, bh, t0, my_tiles, rb, NT);
}

PFN_cuTensorMapEncodeTiled_v12000 meta_map_encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// [rows][ncol] fp32 view of mu or var (ncol metadata columns: blocks, or
// sub-blocks with the envelope), boxes of [box_rows coordinates][32 columns].
bool encode_meta_map(CUtensorMap* tm, const float* base, int64_t rows, int64_t nb_cap, int box_rows) {
  PFN_cuTensorMapEncodeTiled_v12000 enc = meta_map_encoder();
  if (enc == nullptr) return false;
  const cuuint64_t gdim[2] = {static_cast<cuuint64_t>(nb_cap), static_cast<cuuint64_t>(rows)};
  const cuuint64_t gstride[1] = {static_cast<cuuint64_t>(nb_cap) * sizeof(float)};
  const cuuint32_t box[2] = {32u, static_cast<cuuint32_t>(box_rows)};
  const cuuint32_t estride[2] = {1u, 1u};
  return enc(tm, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<float*>(base), gdim, gstride, box, estride,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int D, int G>
cudaError_t launch_tma_t(const ScreenCall& c, cudaStream_t st) {
  constexpr int CW = TmaScreenCfg<D>::kCW, NST = TmaScreenCfg<D>::kNST;
  const eta_shape_t& s = c.shape;
  const int BH = s.batch * s.n_kv_heads;
  const int64_t ncol = s.capacity / s.block_size * c.sub_blocks;
  const int nb = static_cast<int>((c.n + s.block_size - 1) / s.block_size);
  const int ns = max(0, nb - c.n_local);
  const int nt = (ns * c.sub_blocks + 31) / 32;
  // Clusters as large as keeps the launch within one wave of two thread blocks
  // per SM (at least 1, at most kMaxCluster, at most one tile per CTA). (Larger
  // clusters that would balance SMs holding one and two thread blocks measured
  // slower: 191 against 172 us on 256 pairs of 128 tiles.)
  int cs = static_cast<int>((2 * static_cast<int64_t>(device_sm_count())) / BH);
  cs = max(1, min(cs, min(kMaxCluster, nt)));
  while ((nt + cs - 1) / cs > kMaxScreenTiles && cs < kMaxCluster) ++cs;
  const int tpc = max(1, (nt + cs - 1) / cs);
  if (tpc > kMaxScreenTiles) return cudaErrorInvalidValue;
  const size_t smem = 128 + static_cast<size_t>(NST) * 2 * D * 32 * sizeof(float) + kTmaBarBytes<NST> +
                      ScreenSmem<D, G>::bytes(tpc) + kTmaDefer<D, G> * (G * 32 * sizeof(float) + sizeof(int));
  if (smem > static_cast<size_t>(device_max_smem_optin())) return cudaErrorNotSupported;
  CUtensorMap tmu, tvar;
  const int64_t rows = static_cast<int64_t>(BH) * D;
  if (!encode_meta_map(&tmu, c.meta.mu, rows, ncol, D) || !encode_meta_map(&tvar, c.meta.var, rows, ncol, D))
    return cudaErrorNotSupported;
  const ScreenArgs a = make_screen_args(c, nb, ns, tpc);
  static std::atomic<uint64_t> smem_done{0};
  cudaError_t e = allow_max_smem(smem_done, reinterpret_cast<const void*>(screen_tma_kernel<D, G>));
  if (e != cudaSuccess) return e;

  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(BH * cs));
  cfg.blockDim = dim3((CW + 1 + kTauWarps) * 32);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = static_cast<unsigned>(cs);
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1] = pdl_attribute();
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  e = cudaLaunchKernelEx(&cfg, screen_tma_kernel<D, G>, a, c.ws.status, tmu, tvar);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

template <int D>
cudaError_t launch_tma_d(const ScreenCall& c, cudaStream_t st) {
  switch (c.shape.n_q_heads / c.shape.n_kv_heads) {
    case 1: return launch_tma_t<D, 1>(c, st);
    case 2: return launch_tma_t<D, 2>(c, st);
    case 4: return launch_tma_t<D, 4>(c, st);
    case 8: return launch_tma_t<D, 8>(c, st);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace

cudaError_t launch_screen_tma(const ScreenCall& c, cudaStream_t st) {
  const int64_t ncol = c.shape.capacity / c.shape.block_size * c.sub_blocks;
  // TMA wants 16-byte aligned rows and a 16-byte aligned base
  if (ncol % 4 != 0 || (reinterpret_cast<uintptr_t>(c.meta.mu) & 15) != 0 ||
      (reinterpret_cast<uintptr_t>(c.meta.var) & 15) != 0)
    return cudaErrorNotSupported;
  return c.shape.head_dim == 128 ? launch_tma_d<128>(c, st) : launch_tma_d<64>(c, st);
}

}  // namespace eta

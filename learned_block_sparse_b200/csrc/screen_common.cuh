// Pieces shared by the two screening kernels (plain loads in screen.cu, TMA
// staged tiles in screen_tma.cu): arguments, the query prologue, the Eq. 5
// decision of one block, and the compaction phases that turn per-tile masks
// into globally ascending lists across a thread-block cluster.
#pragma once

#include <cooperative_groups.h>

#include <cmath>

#include "common.cuh"
#include "launch.h"
#include "tau_chain.cuh"

namespace eta {

struct ScreenArgs {
  const void* q;
  int q_dtype;
  const float* mu;
  const float* var;
  const float* maxn;
  const float* tau;
  int64_t tau_stride;
  const float* W;      // non-null: thresholds by Eq. 1 in the prologue
  const float* bias;
  float* tau_out;
  float z, s, offset_a;
  int Hq, Hkv, nb, ns, nb_cap, tiles_per_cta;  // nb, ns: of the longest row (launch sizing)
  // Sub-block envelope: r sub-blocks per block, metadata columns nb_cap * r.
  // A screening lane handles one metadata column ("unit"): sub-block u of
  // block u / r; r = 1 is Eq. 5 on whole blocks.
  int r, nb_cap_meta;
  const int32_t* seq_lens;  // [B] per-row token counts, or null (every row has n)
  int64_t n;
  int bs, n_local;
  int32_t* status;
  uint32_t* ws_union;
  int32_t* ws_union_cnt;
  int32_t* ws_head_cnt;
  int32_t* active_idx;
  int32_t* active_cnt;
  uint32_t* union_out;
  int32_t* union_cnt_out;
  float* scores;
};

// Blocks of batch row b: nb in all, the first ns of them screened (the last
// n_local, which hold the current token, are always admitted).
struct RowBlocks {
  int nb, ns;
};

__device__ __forceinline__ uint32_t lanemask_lt() {
  uint32_t m;
  asm("mov.u32 %0, %%lanemask_lt;" : "=r"(m));
  return m;
}

// Shared-memory carve-up common to both kernels (offsets from `base`).
template <int D, int G>
struct ScreenSmem {
  float* q;      // [D][G] (head-minor: the G heads of a coordinate are adjacent)
  float* qq;     // [D][G] fl(q_i * q_i)
  float* qn;     // [G] fl(sqrt(sum q_i^2))
  float* taut;   // [G] tau - a
  int* tot;      // [G+1] this CTA's admitted counts
  int* base;     // [G+1] counts of lower-ranked CTAs
  float* tau;    // [G] Eq. 1 thresholds (when formed in the prologue)
  float* part;   // [32][G+1] Eq. 1 partials
  int* tcnt;     // [tpc][G+1] per-tile counts -> offsets
  uint8_t* mask; // [tpc*32] head mask of every block
  __device__ ScreenSmem(unsigned char* p, int tpc) {
    q = reinterpret_cast<float*>(p);
    qq = q + G * D;
    qn = qq + G * D;
    taut = qn + 16;
    tau = taut + 16;
    part = tau + 16;
    tot = reinterpret_cast<int*>(part + 32 * (G + 1));
    base = tot + 16;
    tcnt = base + 16;
    mask = reinterpret_cast<uint8_t*>(tcnt + tpc * (G + 1));
  }
  __host__ __device__ static constexpr size_t fixed_bytes() {
    return (2 * G * D + 48 + 32 * (G + 1)) * sizeof(float) + 32 * sizeof(int);
  }
  __host__ __device__ static size_t bytes(int tpc) {
    return fixed_bytes() + static_cast<size_t>(tpc) * (G + 1) * sizeof(int) + static_cast<size_t>(tpc) * 32;
  }
};

__device__ __forceinline__ RowBlocks row_blocks(const ScreenArgs& a, int b) {
  const int64_t n = seq_len_of(a.seq_lens, b, a.n, a.status);
  RowBlocks r;
  r.nb = static_cast<int>((n + a.bs - 1) / a.bs);
  r.ns = max(0, r.nb - a.n_local);
  return r;
}

// Eq. 1 thresholds of the group's heads (a.W set) by the `nthreads` threads
// with relative index `rel`, synchronised by `sync`: sm.tau, sm.taut = tau - a,
// and the cluster's first thread block writes tau to a.tau_out.
template <int D, int G, int kBatch, typename Sync>
__device__ __forceinline__ void screen_predict_tau(const ScreenArgs& a, const ScreenSmem<D, G>& sm, int b, int kvh,
                                                   int rel, int nthreads, Sync sync) {
  const int Hd = a.Hq * D;
  const int64_t row = static_cast<int64_t>(b) * Hd;
  if (a.q_dtype == ETA_BF16)
    predict_heads<kBatch>(static_cast<const uint16_t*>(a.q) + row, a.W, a.bias, a.Hq, Hd, kvh * G, G, sm.part,
                          sm.tau, rel, nthreads, sync);
  else
    predict_heads<kBatch>(static_cast<const float*>(a.q) + row, a.W, a.bias, a.Hq, Hd, kvh * G, G, sm.part, sm.tau,
                          rel, nthreads, sync);
  if (rel < G) {
    sm.taut[rel] = __fsub_rn(sm.tau[rel], a.offset_a);
    if (cooperative_groups::this_cluster().block_rank() == 0)
      a.tau_out[static_cast<int64_t>(b) * a.Hq + kvh * G + rel] = sm.tau[rel];
  }
}

// Stage the group's queries, their squares and norms, and the thresholds
// tau - a: read from a.tau, or (a.W set and kTauHere) formed by Eq. 1 with all
// threads; with a.W set and !kTauHere the caller forms them (screen_predict_tau)
// before any decision. All threads; ends with __syncthreads.
template <int D, int G, int kBatch, bool kTauHere>
__device__ __forceinline__ void screen_prologue(const ScreenArgs& a, const ScreenSmem<D, G>& sm, int b, int kvh,
                                                int nthreads) {
  const int tid = threadIdx.x;
  for (int i = tid; i < G * D; i += nthreads) {
    const int g = i / D, e = i % D;
    const float x = load_elem(a.q, a.q_dtype, (static_cast<int64_t>(b) * a.Hq + kvh * G + g) * D + e);
    sm.q[e * G + g] = x;
    sm.qq[e * G + g] = __fmul_rn(x, x);
  }
  if (a.W == nullptr) {
    if (tid < G) sm.taut[tid] = __fsub_rn(a.tau[b * a.tau_stride + kvh * G + tid], a.offset_a);
  } else if (kTauHere) {
    screen_predict_tau<D, G, kBatch>(a, sm, b, kvh, tid, nthreads, [] { __syncthreads(); });
  }
  __syncthreads();
  if (tid < G) {
    float qn = 0.0f;  // sum of q_i^2 by fused multiply-adds in increasing i
    for (int e0 = 0; e0 < D; e0 += 16) {
      float x[16];
#pragma unroll
      for (int c = 0; c < 16; ++c) x[c] = sm.q[(e0 + c) * G + tid];
#pragma unroll
      for (int c = 0; c < 16; ++c) qn = __fmaf_rn(x[c], x[c], qn);
    }
    sm.qn[tid] = __fsqrt_rn(qn);
  }
  __syncthreads();
}

// Eq. 5 scores of one metadata unit for every head of the group, given the
// fma-accumulated D = sum q_i mu_i and V = sum q_i^2 var_i; with sub-blocks
// (r > 1) the block's score is the largest over its r units, which sit in r
// consecutive lanes (r divides 32, and the r units of a block are all valid or
// all invalid). Independent of the thresholds. All 32 lanes call it.
template <int D, int G>
__device__ __forceinline__ void screen_scores(const ScreenArgs& a, const ScreenSmem<D, G>& sm, const float (&dg)[G],
                                              const float (&vg)[G], float M, float (&sc)[G]) {
#pragma unroll
  for (int g = 0; g < G; ++g) {
    const float A = __fadd_rn(dg[g], __fmul_rn(a.z, __fsqrt_rn(vg[g])));
    const float C = __fmul_rn(sm.qn[g], M);
    sc[g] = __fmul_rn((A < C) ? A : C, a.s);
  }
  if (a.r > 1) {
    for (int o = 1; o < a.r; o <<= 1)
#pragma unroll
      for (int g = 0; g < G; ++g) sc[g] = fmaxf(sc[g], __shfl_xor_sync(kFull, sc[g], o));
  }
}

// The admission rule on the scores of one unit (with sub-blocks the first unit
// of a block decides it): writes the scores (if asked) and returns the head
// mask of the admitted heads. All 32 lanes call it.
template <int D, int G>
__device__ __forceinline__ uint32_t screen_admit(const ScreenArgs& a, const ScreenSmem<D, G>& sm, int b, int kvh,
                                                 int unit, bool valid, const float (&sc)[G]) {
  if (a.r > 1) valid = valid && (threadIdx.x & (a.r - 1)) == 0;
  const int blk = unit / a.r;
  uint32_t mask = 0;
#pragma unroll
  for (int g = 0; g < G; ++g) {
    if (valid && !(sc[g] < sm.taut[g])) mask |= 1u << g;
    if (a.scores != nullptr && valid) a.scores[(static_cast<int64_t>(b) * a.Hq + kvh * G + g) * a.nb_cap + blk] = sc[g];
  }
  return mask;
}

// Eq. 5 and the admission rule for one unit: screen_scores, then screen_admit.
template <int D, int G>
__device__ __forceinline__ uint32_t screen_decide(const ScreenArgs& a, const ScreenSmem<D, G>& sm, int b, int kvh,
                                                  int unit, bool valid, const float (&dg)[G], const float (&vg)[G],
                                                  float M) {
  float sc[G];
  screen_scores<D, G>(a, sm, dg, vg, M, sc);
  return screen_admit<D, G>(a, sm, b, kvh, unit, valid, sc);
}

// Record one tile's masks and admission counts (one warp, lane = block).
template <int D, int G>
__device__ __forceinline__ void screen_record_tile(const ScreenSmem<D, G>& sm, int t, uint32_t mask) {
  const int lane = threadIdx.x & 31;
  sm.mask[t * 32 + lane] = static_cast<uint8_t>(mask);
  int cnt[G + 1];
#pragma unroll
  for (int g = 0; g < G; ++g) cnt[g] = __popc(__ballot_sync(kFull, (mask >> g) & 1u));
  cnt[G] = __popc(__ballot_sync(kFull, mask != 0u));
  if (lane == 0) {
#pragma unroll
    for (int c = 0; c <= G; ++c) sm.tcnt[t * (G + 1) + c] = cnt[c];
  }
}

// Phases 2-4, after every tile of this CTA is recorded (call with all threads
// after a __syncthreads): exclusive prefix over the CTA's tiles, offsets of this
// CTA inside the cluster through distributed shared memory, then the compacted
// lists; the cluster's last CTA appends the forced trailing blocks and writes
// the counts.
template <int D, int G>
__device__ __forceinline__ void screen_finish(const ScreenArgs& a, const ScreenSmem<D, G>& sm, int b, int kvh,
                                              int bh, int t0, int my_tiles, RowBlocks rb, int nthreads) {
  namespace cg = cooperative_groups;
  cg::cluster_group cluster = cg::this_cluster();
  const int cs = static_cast<int>(cluster.num_blocks());
  const int cr = static_cast<int>(cluster.block_rank());
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, nwarps = nthreads >> 5;
  if (tid <= G) {
    int run = 0;
    for (int t = 0; t < my_tiles; ++t) {
      const int v = sm.tcnt[t * (G + 1) + tid];
      sm.tcnt[t * (G + 1) + tid] = run;
      run += v;
    }
    sm.tot[tid] = run;
  }
  cluster.sync();
  if (tid <= G) {
    int base = 0;
    for (int r = 0; r < cr; ++r) base += cluster.map_shared_rank(sm.tot, r)[tid];
    sm.base[tid] = base;
  }
  cluster.sync();

  const uint32_t lt = lanemask_lt();
  for (int t = warp; t < my_tiles; t += nwarps) {
    const int blk = ((t0 + t) * 32 + lane) / a.r;  // a lane with a mask bit is its block's first unit
    const uint32_t mask = sm.mask[t * 32 + lane];
#pragma unroll
    for (int g = 0; g < G; ++g) {
      const bool on = (mask >> g) & 1u;
      const uint32_t bal = __ballot_sync(kFull, on);
      if (on && a.active_idx != nullptr) {
        const int pos = sm.base[g] + sm.tcnt[t * (G + 1) + g] + __popc(bal & lt);
        a.active_idx[(static_cast<int64_t>(b) * a.Hq + kvh * G + g) * a.nb_cap + pos] = blk;
      }
    }
    const bool any = mask != 0u;
    const uint32_t balu = __ballot_sync(kFull, any);
    if (any) {
      const int pos = sm.base[G] + sm.tcnt[t * (G + 1) + G] + __popc(balu & lt);
      const uint32_t entry = (static_cast<uint32_t>(blk) << 8) | mask;
      a.ws_union[static_cast<int64_t>(bh) * a.nb_cap + pos] = entry;
      if (a.union_out != nullptr) a.union_out[static_cast<int64_t>(bh) * a.nb_cap + pos] = entry;
    }
  }

  if (cr == cs - 1) {
    const int nf = rb.nb - rb.ns;
    const uint32_t all = (1u << G) - 1u;
    for (int j = tid; j < nf; j += nthreads) {
      const int blk = rb.ns + j;
      if (a.active_idx != nullptr) {
#pragma unroll
        for (int g = 0; g < G; ++g)
          a.active_idx[(static_cast<int64_t>(b) * a.Hq + kvh * G + g) * a.nb_cap + sm.base[g] + sm.tot[g] + j] = blk;
      }
      const uint32_t entry = (static_cast<uint32_t>(blk) << 8) | all;
      const int64_t o = static_cast<int64_t>(bh) * a.nb_cap + sm.base[G] + sm.tot[G] + j;
      a.ws_union[o] = entry;
      if (a.union_out != nullptr) a.union_out[o] = entry;
    }
    if (tid < G) {
      const int c = sm.base[tid] + sm.tot[tid] + nf;
      const int64_t hq = static_cast<int64_t>(b) * a.Hq + kvh * G + tid;
      a.ws_head_cnt[hq] = c;
      if (a.active_cnt != nullptr) a.active_cnt[hq] = c;
    } else if (tid == G) {
      const int c = sm.base[G] + sm.tot[G] + nf;
      a.ws_union_cnt[bh] = c;
      if (a.union_cnt_out != nullptr) a.union_cnt_out[bh] = c;
    }
  }
}

// Host side: arguments for a screening launch.
inline ScreenArgs make_screen_args(const ScreenCall& c, int nb, int ns, int tpc) {
  const eta_shape_t& s = c.shape;
  ScreenArgs a;
  a.q = c.q;
  a.q_dtype = s.q_dtype;
  a.mu = c.meta.mu;
  a.var = c.meta.var;
  a.maxn = c.meta.maxnorm;
  a.tau = c.tau;
  a.tau_stride = c.tau_stride;
  a.W = c.W;
  a.bias = c.bias;
  a.tau_out = c.tau_out;
  a.z = c.z;
  a.s = static_cast<float>(1.0 / std::sqrt(static_cast<double>(s.head_dim)));
  a.offset_a = c.offset_a;
  a.Hq = s.n_q_heads;
  a.Hkv = s.n_kv_heads;
  a.nb = nb;
  a.ns = ns;
  a.seq_lens = c.seq_lens;
  a.n = c.n;
  a.bs = s.block_size;
  a.n_local = c.n_local;
  a.status = c.ws.status;
  a.nb_cap = static_cast<int>(s.capacity / s.block_size);
  a.r = c.sub_blocks;
  a.nb_cap_meta = a.nb_cap * c.sub_blocks;
  a.tiles_per_cta = tpc;
  a.ws_union = c.ws.union_list;
  a.ws_union_cnt = c.ws.union_cnt;
  a.ws_head_cnt = c.ws.head_cnt;
  a.active_idx = c.out.active_idx;
  a.active_cnt = c.out.active_cnt;
  a.union_out = c.out.union_list;
  a.union_cnt_out = c.out.union_cnt;
  a.scores = c.out.scores;
  return a;
}

// Launch `kernel` as BH clusters of `cs` thread blocks.
template <typename Kernel>
cudaError_t launch_clusters(Kernel kernel, const ScreenArgs& a, int BH, int cs, int threads, size_t smem,
                            cudaStream_t st) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(BH * cs));
  cfg.blockDim = dim3(static_cast<unsigned>(threads));
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
  cudaError_t e = cudaLaunchKernelEx(&cfg, kernel, a);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

// Screening with metadata tiles staged by TMA (screen_tma.cu); returns
// cudaErrorNotSupported when the metadata rows are not TMA-aligned.
cudaError_t launch_screen_tma(const ScreenCall& c, cudaStream_t st);

}  // namespace eta

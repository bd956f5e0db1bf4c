// Pieces shared by the two decode kernels (CUDA-core consumer for fp32 K/V,
// tensor-core consumer for bf16 K/V): arguments, the flat split of admitted
// blocks over thread blocks, the on-chip prefix of the per-(batch, kv head)
// counts, and the producer loop that walks this thread block's range.
#pragma once

#include <cmath>

#include "common.cuh"
#include "launch.h"

namespace eta {

struct DecodeArgs {
  const void* k;
  const void* v;
  const void* q;
  const float* tau;
  const uint32_t* union_list;
  const int32_t* union_cnt;
  float* o_part;
  float2* ml_part;
  int32_t* prefix_out;
  int32_t* status;
  int64_t cap, n, tau_stride;
  int B, Hq, Hkv, bs, nb, nb_cap, nstages, q_dtype;
  float beta, qscale;
};

__device__ __forceinline__ int find_seg(const int32_t* pre, int BH, int64_t p) {
  int lo = 0, hi = BH - 1;  // largest i with pre[i] <= p
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (pre[mid] <= p) lo = mid;
    else hi = mid - 1;
  }
  return lo;
}

// The thread block whose range [k*T/S, (k+1)*T/S) holds flat position x.
__device__ __forceinline__ int range_of(int64_t x, int64_t T, int S) {
  return static_cast<int>(((x + 1) * S - 1) / T);
}

// Exclusive prefix of the union counts into s_pre[0..BH] (all threads call).
__device__ __forceinline__ void block_prefix(const int32_t* cnt, int32_t* s_pre, int BH, int nthreads) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  for (int i = tid; i < BH; i += nthreads) s_pre[i + 1] = cnt[i];
  __syncthreads();
  if (warp == 0) {
    int run = 0;
    for (int base = 0; base < BH; base += 32) {
      const int i = base + lane;
      int v = i < BH ? s_pre[i + 1] : 0;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int u = __shfl_up_sync(kFull, v, o);
        if (lane >= o) v += u;
      }
      if (i < BH) s_pre[i + 1] = run + v;
      run += __shfl_sync(kFull, v, 31);
    }
    if (lane == 0) s_pre[0] = 0;
  }
}

// Producer warp: walk positions [lo, hi) in order. Lanes 0..PL-1 each take
// every PL-th position (position lo + i goes to lane i % PL, PL = 4, or less
// when the ring has fewer stages, so PL consecutive positions never share a
// stage and are armed in parallel): wait until the position's stage is free,
// publish (block, head mask, rows, segment) in s_info and call
// issue(stage, segment, block, rows), which must arm s_full[stage] (arrive +
// expected bytes) and start the copies. The warp reads the union list 32
// entries at a time, one batch ahead. A stage's r-th reuse waits for the
// consumer release that completed the empty barrier's phase r-1.
template <int G, bool DENSE, typename SegOf, typename Pre, typename Issue>
__device__ __forceinline__ void producer_loop(const DecodeArgs& a, int64_t lo, int64_t hi, int NST,
                                              uint64_t* s_empty, int4* s_info, int* s_abort, SegOf seg_of,
                                              Pre pre, Issue issue, uint64_t* s_full) {
  const int PL = NST >= 4 ? 4 : (NST >= 2 ? 2 : 1);  // issuing lanes
  const int lane = threadIdx.x & 31;
  auto load_entry = [&](int64_t p, int& seg, uint32_t& e) {
    seg = 0;
    e = 0;
    if (p < hi) {
      seg = seg_of(p);
      const int64_t j = p - pre(seg);
      e = DENSE ? ((static_cast<uint32_t>(j) << 8) | ((1u << G) - 1u))
                : __ldg(a.union_list + static_cast<int64_t>(seg) * a.nb_cap + j);
    }
  };
  int seg_cur, seg_nxt = 0;
  uint32_t e_cur, e_nxt = 0;
  load_entry(lo + lane, seg_cur, e_cur);
  int issued = 0;    // this lane: 1 + the last position (relative to lo) it armed
  int aborted = 0;
  for (int64_t base = lo; base < hi && !aborted; base += 32) {
    if (base + 32 < hi) load_entry(base + 32 + lane, seg_nxt, e_nxt);
    const int cnt = static_cast<int>(hi - base < 32 ? hi - base : int64_t{32});
    for (int s = 0; s < cnt && !aborted; s += PL) {
      const int src = s + (lane < PL ? lane : 0);
      const int seg_i = __shfl_sync(kFull, seg_cur, src);
      const uint32_t e_i = __shfl_sync(kFull, e_cur, src);
      if (lane < PL && src < cnt) {
        const int it = static_cast<int>(base - lo) + src;
        const int st = it % NST;
        const int round = it / NST;
        if (round > 0 && !mbar_wait_bounded(&s_empty[st], (round - 1) & 1, s_abort, a.status)) aborted = 1;
        if (!aborted) {
          const int blk = static_cast<int>(e_i >> 8);
          int rows = 0;
          if (blk < a.nb) {
            const int64_t r = a.n - static_cast<int64_t>(blk) * a.bs;
            rows = r < a.bs ? static_cast<int>(r) : a.bs;
          } else {
            atomicExch(a.status, static_cast<int32_t>(ETA_ERR_INVALID_ARG));
          }
          s_info[st] = make_int4(blk, static_cast<int>(e_i & 0xffu), rows, seg_i);
          if (rows == 0) mbar_arrive(&s_full[st]);
          else issue(st, seg_i, blk, rows);
          issued = it + 1;
        }
      }
      aborted = __any_sync(kFull, aborted) ? 1 : 0;
    }
    seg_cur = seg_nxt;
    e_cur = e_nxt;
  }
  if (aborted && lane < PL) {
    // let the copies this lane armed land before the thread block can exit
    for (int j = issued - 1; j >= 0 && j >= issued - NST; j -= PL) {
      const uint64_t t0 = global_timer_ns();
      while (!mbar_try_wait(&s_full[j % NST], (j / NST) & 1) && global_timer_ns() - t0 < kWaitLimitNs) {
      }
    }
  }
}

// Host side: the arguments common to both decode kernels.
inline DecodeArgs make_decode_args(const DecodeCall& c, int nstages) {
  const eta_shape_t& s = c.shape;
  DecodeArgs a;
  a.k = c.k;
  a.v = c.v;
  a.q = c.q;
  a.tau = c.tau;
  a.union_list = c.ws.union_list;
  a.union_cnt = c.ws.union_cnt;
  a.o_part = c.ws.o_part;
  a.ml_part = c.ws.ml_part;
  a.prefix_out = c.ws.prefix;
  a.status = c.ws.status;
  a.cap = s.capacity;
  a.n = c.n;
  a.tau_stride = c.tau_stride;
  a.B = s.batch;
  a.Hq = s.n_q_heads;
  a.Hkv = s.n_kv_heads;
  a.bs = s.block_size;
  a.nb = static_cast<int>((c.n + s.block_size - 1) / s.block_size);
  a.nb_cap = static_cast<int>(s.capacity / s.block_size);
  a.nstages = nstages;
  a.q_dtype = s.q_dtype;
  a.beta = c.beta;
  a.qscale = static_cast<float>(1.0 / std::sqrt(static_cast<double>(s.head_dim)));
  return a;
}

// Tensor-core decode (bf16 K/V and q), in decode_mma.cu.
cudaError_t launch_decode_mma(const DecodeCall& c, cudaStream_t st);

}  // namespace eta

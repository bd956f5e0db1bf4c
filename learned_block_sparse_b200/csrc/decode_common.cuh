// Pieces shared by the two decode kernels (CUDA-core consumer for fp32 K/V,
// tensor-core consumer for bf16 K/V): arguments, the flat split of admitted
// blocks over thread blocks, the on-chip prefix of the per-(batch, kv head)
// counts, the producer loop that walks this thread block's range, and the
// split-K merge that the thread block writing a segment's last partial runs.
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
  const int32_t* seq_lens;  // [B] per-row token counts, or null (every row has n)
  KvLayout kv;              // contiguous cache or paged pool
  float* o_part;
  float2* ml_part;
  float* out;
  int32_t* seg_done;
  int32_t* status;
  int64_t cap, n, tau_stride;  // n: tokens of every row, or the upper bound of seq_lens
  int B, Hq, Hkv, bs, nb, nb_cap, nstages, q_dtype;
  int gate;  // ETA_GATE_SIGMOID or ETA_GATE_HARD
  float beta, qscale;
  // Ring positions: each admitted block is 2^sub_log2 positions of rpos rows
  // (rpos = bs >> sub_log2); flat positions, ranges and segment bounds count them.
  int sub_log2, rpos;
  int64_t withhold;  // test hook: position of thread block 0's range whose copy is never armed (-1: none)
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

// Cached tokens of segment (batch row, kv head) `seg`.
__device__ __forceinline__ int64_t seg_tokens(const DecodeArgs& a, int seg) {
  return seq_len_of(a.seq_lens, seg / a.Hkv, a.n, a.status);
}

// Exclusive prefix of the per-segment block counts into s_pre[0..BH] (all
// threads call): the union counts, or (dense) every block of the segment.
template <bool DENSE>
__device__ __forceinline__ void block_prefix(const DecodeArgs& a, int32_t* s_pre, int BH, int nthreads) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  for (int i = tid; i < BH; i += nthreads)
    s_pre[i + 1] = DENSE ? static_cast<int32_t>((seg_tokens(a, i) + a.bs - 1) / a.bs) : a.union_cnt[i];
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

// The partials of a segment [p0, p1): one per thread block whose range meets
// it, numbered from 0 in range order. With T >= S no range is empty and the
// ranges k0 = range_of(p0) .. range_of(p1 - 1) each give one. With T < S a
// range holds at most one position, so the partials are simply the segment's
// positions: the thread block whose range starts at `lo` writes slot lo - p0.
struct SegSpan {
  int slot, parts;
};
__device__ __forceinline__ SegSpan seg_span(int64_t p0, int64_t p1, int64_t lo, int64_t T, int S) {
  SegSpan r;
  if (T >= S) {
    const int k0 = range_of(p0, T, S);
    r.slot = static_cast<int>(blockIdx.x) - k0;
    r.parts = range_of(p1 - 1, T, S) - k0 + 1;
  } else {
    r.slot = static_cast<int>(lo - p0);
    r.parts = static_cast<int>(p1 - p0);
  }
  return r;
}

// Epilogue of one segment (batch, kv head) in a thread block, called by its NW
// consumer warps (named barrier 1) once each warp has left its running max
// (log2 units), sum and unnormalised output rows in s_mm / s_ml / s_macc.
// The warps' states are merged; a segment that lies inside this thread block's
// range is normalised and written to `out` at once. Otherwise this range's
// partial (m, l, o) goes to the workspace and is counted in seg_done[seg]; the
// thread block that counts the segment's last partial merges all of them in
// range order (a fixed order, so the result does not depend on which thread
// block finishes last: flash-decoding's split-K reduction) and re-arms the
// counter for the next call.
template <int D, int G, int NW>
__device__ __forceinline__ void finish_segment(const DecodeArgs& a, int seg, int64_t p0, int64_t p1, int64_t lo,
                                               int64_t T, int S, const float* s_macc, const float* s_mm,
                                               const float* s_ml, volatile int* s_flag) {
  constexpr int kThr = NW * 32;
  const int tid = threadIdx.x;
  const int b = seg / a.Hkv, kvh = seg % a.Hkv;
  const int64_t hq0 = static_cast<int64_t>(b) * a.Hq + kvh * G;
  const SegSpan sp = seg_span(p0, p1, lo, T, S);
  for (int idx = tid; idx < G * D; idx += kThr) {
    const int g = idx / D, e = idx % D;
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < NW; ++w) M = fmaxf(M, s_mm[w * G + g]);
    float ov = 0.0f, L = 0.0f;
#pragma unroll
    for (int w = 0; w < NW; ++w) {
      const float c = M == -INFINITY ? 0.0f : exp2f(s_mm[w * G + g] - M);
      ov = fmaf(c, s_macc[(w * G + g) * D + e], ov);
      L = fmaf(c, s_ml[w * G + g], L);
    }
    if (sp.parts == 1) {
      a.out[(hq0 + g) * D + e] = ov * (1.0f / L);
    } else {
      const int64_t prow = (hq0 + g) * S + sp.slot;
      a.o_part[prow * D + e] = ov;
      if (e == 0) a.ml_part[prow] = make_float2(M, L);
    }
  }
  if (sp.parts == 1) {
    named_barrier_sync(1, kThr);  // s_macc is rewritten by the next segment
    return;
  }
  __threadfence();  // this thread's partial is visible before the count
  named_barrier_sync(1, kThr);
  if (tid == 0) {
    const int done = atomicAdd(a.seg_done + seg, 1) + 1;
    const int last = done == sp.parts ? 1 : 0;
    if (last) atomicExch(a.seg_done + seg, 0);
    *s_flag = last;
  }
  named_barrier_sync(1, kThr);
  if (*s_flag == 0) return;
  __threadfence();
  for (int idx = tid; idx < G * D; idx += kThr) {
    const int g = idx / D, e = idx % D;
    const float2* ml = a.ml_part + (hq0 + g) * S;
    const float* op = a.o_part + (hq0 + g) * S * D + e;
    float M = -INFINITY;
    for (int s = 0; s < sp.parts; ++s) M = fmaxf(M, __ldcg(ml + s).x);
    float o = 0.0f, L = 0.0f;
    for (int s = 0; s < sp.parts; ++s) {
      const float2 v = __ldcg(ml + s);
      const float c = v.x == -INFINITY ? 0.0f : exp2f(v.x - M);
      L = fmaf(c, v.y, L);
      o = fmaf(c, __ldcg(op + static_cast<int64_t>(s) * D), o);
    }
    a.out[(hq0 + g) * D + e] = o * (1.0f / L);
  }
}

// Producer warp: walk positions [lo, hi) in order. A position is rows
// [sub * rpos, (sub + 1) * rpos) of an admitted block, whose 2^sub_log2
// positions are consecutive. Lanes 0..PL-1 each take every PL-th position
// (position lo + i goes to lane i % PL; PL = kMaxPL, or less when the ring has
// fewer stages, so PL consecutive positions never share a stage and are armed
// in parallel): wait until the position's stage is free, publish
// (block * 2^sub_log2 + sub, head mask, rows, segment) in s_info and call
// issue(stage, row0, rows) (row0: the position's first row in the [rows][d]
// view of the K and V stores), which must arm s_full[stage] (arrive + expected
// bytes) and start the copies. The warp reads the union list 32 entries at a
// time, one batch ahead. A stage's r-th reuse waits for the consumer release
// that completed the empty barrier's phase r-1; the round a stage serves is
// then published in s_round (when given) before it is armed.
//
// Abort protocol. Consumers release a stage only after its full barrier
// completed, so a stage is never re-armed while its copies are in flight.
// Once any warp of the thread block has given up (s_abort), the producer arms
// nothing more; whatever happened, before returning it waits (bounded) until
// the copies of the last armed use of every stage have landed, so the thread
// block never exits with a copy in flight. a.withhold (a test hook) leaves one
// position of thread block 0 unarmed, so that its consumer's bounded wait runs
// out and the call ends with ETA_ERR_DEVICE_TIMEOUT.
template <int G, bool DENSE, int kMaxPL, typename SegOf, typename Pre, typename Issue>
__device__ __forceinline__ void producer_loop(const DecodeArgs& a, int64_t lo, int64_t hi, int NST,
                                              uint64_t* s_empty, int4* s_info, int* s_abort, SegOf seg_of,
                                              Pre pre, Issue issue, uint64_t* s_full,
                                              volatile int* s_round = nullptr) {
  static_assert(kMaxPL == 1 || kMaxPL == 2 || kMaxPL == 4 || kMaxPL == 8, "issuing lanes divide 32");
  int PL = kMaxPL;  // issuing lanes
  while (PL > NST) PL >>= 1;
  const int lane = threadIdx.x & 31;
  // entry of position p, in two halves so the list load of the next batch is
  // in flight while this batch is issued: fetch() gives the segment, the
  // position's sub-block and (block << 8 | head mask); finish() its rows
  // (tokens of the row inside it: 0 for a sub-block past the row's last token,
  // -1 when the whole block is past the row or its page outside the pool) and
  // the store row of its first token
  auto fetch = [&](int64_t p, int& seg, int& sub, uint32_t& e) {
    seg = 0;
    sub = 0;
    e = 0;
    if (p < hi) {
      seg = seg_of(p);
      const int64_t j = p - pre(seg);
      const int64_t jb = j >> a.sub_log2;
      sub = static_cast<int>(j - (jb << a.sub_log2));
      e = DENSE ? ((static_cast<uint32_t>(jb) << 8) | ((1u << G) - 1u))
                : __ldg(a.union_list + static_cast<int64_t>(seg) * a.nb_cap + jb);
    }
  };
  auto finish = [&](int64_t p, int seg, int sub, uint32_t e, int& rows, int& row0) {
    rows = 0;
    row0 = 0;
    if (p < hi) {
      const int blk = static_cast<int>(e >> 8);
      const int64_t r = seg_tokens(a, seg) - static_cast<int64_t>(blk) * a.bs - static_cast<int64_t>(sub) * a.rpos;
      rows = r > 0 ? (r < a.rpos ? static_cast<int>(r) : a.rpos) : (sub == 0 ? -1 : 0);
      if (rows > 0) {
        row0 = kv_block_row(a.kv, seg, blk);
        if (row0 < 0) rows = -1;
        else row0 += sub * a.rpos;
      }
    }
  };
  int seg_cur, seg_nxt = 0, sub_cur, sub_nxt = 0, rows_cur, row_cur;
  uint32_t e_cur, e_nxt = 0;
  fetch(lo + lane, seg_cur, sub_cur, e_cur);
  int issued = 0;    // this lane: 1 + the last position (relative to lo) it armed
  int held = -1;     // the position left unarmed by the test hook
  int aborted = 0;
  volatile int* abort_flag = s_abort;
  for (int64_t base = lo; base < hi && !aborted; base += 32) {
    finish(base + lane, seg_cur, sub_cur, e_cur, rows_cur, row_cur);
    if (base + 32 < hi) fetch(base + 32 + lane, seg_nxt, sub_nxt, e_nxt);
    const int cnt = static_cast<int>(hi - base < 32 ? hi - base : int64_t{32});
    for (int s = 0; s < cnt && !aborted; s += PL) {
      const int src = s + (lane < PL ? lane : 0);
      const int seg_i = __shfl_sync(kFull, seg_cur, src);
      const int sub_i = __shfl_sync(kFull, sub_cur, src);
      const uint32_t e_i = __shfl_sync(kFull, e_cur, src);
      const int rows_i = __shfl_sync(kFull, rows_cur, src);
      const int row_i = __shfl_sync(kFull, row_cur, src);
      if (lane < PL && src < cnt) {
        const int it = static_cast<int>(base - lo) + src;
        const int st = it % NST;
        const int round = it / NST;
        if (round > 0 && !mbar_wait_bounded(&s_empty[st], (round - 1) & 1, s_abort, a.status)) aborted = 1;
        if (!aborted && *abort_flag) aborted = 1;  // a consumer gave up: arm nothing more
        if (!aborted) {
          const int blk = static_cast<int>(e_i >> 8);
          int rows = rows_i;
          if (rows < 0) {  // a list entry past the row's last block, or a bad page: load nothing
            atomicExch(a.status, static_cast<int32_t>(ETA_ERR_INVALID_ARG));
            rows = 0;
          }
          if (s_round != nullptr) s_round[st] = round;  // this stage now serves round `round`
          s_info[st] = make_int4((blk << a.sub_log2) + sub_i, static_cast<int>(e_i & 0xffu), rows, seg_i);
          if (blockIdx.x == 0 && it == a.withhold) held = it;   // test hook: never armed
          else if (rows == 0) mbar_arrive(&s_full[st]);
          else issue(st, row_i, rows);
          issued = it + 1;
        }
      }
      aborted = __any_sync(kFull, aborted) ? 1 : 0;
    }
    seg_cur = seg_nxt;
    sub_cur = sub_nxt;
    e_cur = e_nxt;
  }
  // Positions >= last - NST are the last armed use of their stage (last = 1 +
  // the last position any lane armed): wait until each of this lane's has
  // completed, so no copy is in flight when the thread block exits. Earlier
  // positions completed before their stage was re-armed.
  const int last = __reduce_max_sync(kFull, issued);
  if (lane < PL) {
    for (int j = issued - 1; j >= 0 && j >= last - NST; j -= PL) {
      if (j == held) continue;
      const uint64_t t0 = global_timer_ns();
      while (!mbar_try_wait(&s_full[j % NST], (j / NST) & 1) && global_timer_ns() - t0 < kWaitLimitNs) {
      }
    }
  }
}

// Host side: the arguments common to both decode kernels; positions of rpos
// rows (the block size divided by a power of two).
inline DecodeArgs make_decode_args(const DecodeCall& c, int nstages, int rpos) {
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
  a.out = c.out;
  a.seg_done = c.ws.seg_done;
  a.status = c.ws.status;
  a.cap = s.capacity;
  a.n = c.n;
  a.seq_lens = c.seq_lens;
  a.kv.block_table = c.block_table;
  a.kv.max_blocks = static_cast<int>(s.capacity / s.block_size);
  a.kv.num_pages = c.num_pages;
  a.kv.Hkv = s.n_kv_heads;
  a.kv.bs = s.block_size;
  a.kv.cap = s.capacity;
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
  a.gate = c.gate;
  a.withhold = c.withhold;
  a.rpos = rpos;
  a.sub_log2 = 0;
  while ((rpos << a.sub_log2) < s.block_size) ++a.sub_log2;
  a.qscale = static_cast<float>(1.0 / std::sqrt(static_cast<double>(s.head_dim)));
  return a;
}

// Tensor-core decode (bf16 K/V and q), in decode_mma.cu.
cudaError_t launch_decode_mma(const DecodeCall& c, cudaStream_t st);

}  // namespace eta

// Tensor-core decode for bf16 K/V and bf16 queries: the same flash-decoding
// pass as decode.cu (gate of Eq. 2-3, online softmax, flat split of the
// admitted blocks over thread blocks), with the block-level contractions on
// mma.sync m16n8k16 bf16 tiles.
//
// Why tensor cores here: for a GQA group of G heads each admitted 16 KiB K/V
// block (b=32, d=128) costs 2*G*b*d multiply-adds; on CUDA cores that is
// ~1,000+ warp instructions per block at G=4 plus the dot-product reductions,
// more than the ~3,000 issue slots per SM that one block's share of HBM time
// (at ~6.5 TB/s) leaves. As m16n8k16 tiles (rows = the G heads of the group,
// columns = keys or head dims) the same block is 32 QK^T + 64 PV mma
// instructions and 32 ldmatrix loads, so the kernel stays bound by HBM.
//
// Data path. The producer warp issues 2-D TMA tensor copies (boxes of
// [b rows][64 dims], 128-byte swizzle) of each admitted block's K and V into a
// ring of stages; with that swizzle the 8 rows an ldmatrix reads sit in 8
// different bank groups. Consumer warps own whole blocks (position i of the
// range goes to warp i mod (number of consumer warps)): S = Q K^T from ldmatrix'd K fragments, scale,
// gate, online softmax in log2 units on the accumulator fragments, then
// O += P V with P split into bf16 high and low parts so the probabilities keep
// ~16 bits of precision: the high part sits in tile rows 0-7 and the low part
// in rows 8-15 of the same A operand (G <= 8), so one mma per (k-step, n-tile)
// accumulates both and the two halves are summed when a partial is emitted.
// V comes from ldmatrix.trans. In QK^T, rows of the tiles beyond G are zero.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cudaTypedefs.h>

#include <mutex>

#include "decode_common.cuh"

namespace eta {

namespace {

// Consumer warps, plus one producer warp. A warp owns a whole block and its
// per-block chain (QK^T, gate, softmax, PV) is latency-bound, so the warp count
// sets how many blocks are in work per SM: 6 for 32-key chunks at d=128 (4
// warps held the 128K GQA decode at 0.99 of the copy bandwidth, 6 reach 1.09),
// 8 where a block carries more consumer work per byte: 16-token blocks,
// d=64 (twice the keys per byte) and fp8 K/V (half the bytes, plus the
// conversions), whose kernels fit 168 registers.
template <int D, int CH, bool FP8>
struct MmaWarps {
  static constexpr int kMW = (CH == 16 || D == 64) ? 8 : (FP8 ? 7 : 6);
  static constexpr int kThreads = (kMW + 1) * 32;
  static constexpr int kIssueLanes = kMW >= 8 ? 8 : 4;  // producer lanes (a power of two)
};

__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* tm, int x, int y, uint64_t* bar,
                                            uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
      " [%0], [%1, {%2, %3}], [%4], %5;" ::"r"(smem_u32(dst)),
      "l"(tm), "r"(x), "r"(y), "r"(smem_u32(bar)), "l"(policy)
      : "memory");
}

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}

__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}

// D[16x8] += A[16x16] B[16x8] (bf16 in, fp32 accumulate) where only rows 0-7
// of A are non-zero: a_lo holds A[row][2q..2q+1], a_hi A[row][8+2q..9+2q]
// (row = lane/4, q = lane%4); d0, d1 are D[row][2q..2q+1].
__device__ __forceinline__ void mma_rows8(float& d0, float& d1, uint32_t a_lo, uint32_t a_hi, uint32_t b0,
                                          uint32_t b1) {
  [[maybe_unused]] float z2, z3;
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %10, %11};"
      : "+f"(d0), "+f"(d1), "=f"(z2), "=f"(z3)
      : "r"(a_lo), "r"(0u), "r"(a_hi), "r"(0u), "r"(b0), "r"(b1), "f"(0.0f), "f"(0.0f));
}

// Byte offset of 16-byte chunk `chunk` (8 dims) of tile row `row` in a tile
// stored as d/64 boxes of [rows][64] bf16 with the 128-byte TMA swizzle.
__device__ __forceinline__ uint32_t swz(int rows, int row, int chunk) {
  return static_cast<uint32_t>((chunk >> 3) * rows * 128 + row * 128 + (((chunk & 7) ^ (row & 7)) << 4));
}

// D[16x8] += A[16x16] B[16x8] with all four A registers and accumulators.
__device__ __forceinline__ void mma_16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                          uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ float rcp_approx(float x) {
  float y;
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  const __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&h);
}

__device__ __forceinline__ uint32_t pack_f16x2(float lo, float hi) {
  const __half2 h = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&h);
}

// fp8 K/V: four e4m3 bytes -> two f16x2 (bytes 0,1 and bytes 2,3). Exact: every
// e4m3 value is an f16 value. (Measured: widening the values by bit placement
// on the integer pipe instead, to unload the conversion unit, costs more issue
// slots than it saves: 0.59 of the copy bandwidth against 0.66.)
__device__ __forceinline__ void e4m3x4_to_f16x2x2(uint32_t w, uint32_t& lo2, uint32_t& hi2) {
  asm("{\n\t.reg .b16 l, h;\n\tmov.b32 {l, h}, %2;\n\tcvt.rn.f16x2.e4m3x2 %0, l;\n\t"
      "cvt.rn.f16x2.e4m3x2 %1, h;\n\t}"
      : "=r"(lo2), "=r"(hi2)
      : "r"(w));
}

// Two floats -> two e4m3 bytes (lo in bits 0-7), rounded to nearest even,
// saturating at +-448.
__device__ __forceinline__ uint32_t f32x2_to_e4m3x2(float lo, float hi) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
  return r;
}

// Four floats (|v| < 256) -> a high and a low e4m3 word with v = hi + lo / 16:
// hi keeps the top four significant bits of each value and lo the next four,
// so a bf16 value (eight significant bits) is held exactly unless its low part
// falls below the e4m3 subnormal step (values under 2^-6 of the largest one).
__device__ __forceinline__ void e4m3_split4(float v0, float v1, float v2, float v3, uint32_t& hi, uint32_t& lo) {
  const uint32_t h = f32x2_to_e4m3x2(v0, v1) | (f32x2_to_e4m3x2(v2, v3) << 16);
  uint32_t f01, f23;
  e4m3x4_to_f16x2x2(h, f01, f23);
  const float2 b01 = __half22float2(*reinterpret_cast<const __half2*>(&f01));
  const float2 b23 = __half22float2(*reinterpret_cast<const __half2*>(&f23));
  hi = h;
  lo = f32x2_to_e4m3x2((v0 - b01.x) * 16.0f, (v1 - b01.y) * 16.0f) |
       (f32x2_to_e4m3x2((v2 - b23.x) * 16.0f, (v3 - b23.y) * 16.0f) << 16);
}

// D[16x8] += A[16x32] B[32x8], e4m3 in, fp32 accumulate. Byte i of a0 / a2 is
// A[lane/4][4(lane%4) + i] / A[lane/4][16 + 4(lane%4) + i], a1 / a3 the same
// for row lane/4 + 8; byte i of b0 / b1 is B[4(lane%4) + i][lane/4] /
// B[16 + 4(lane%4) + i][lane/4].
__device__ __forceinline__ void mma_16832_e4m3(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k32.row.col.f32.e4m3.e4m3.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// As mma_16816 with f16 operands.
__device__ __forceinline__ void mma_16816_f16(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                              uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// HARD: the strict-mode gate (keys below tau removed) instead of Eq. 2-3.
// FP8: e4m3 K/V (d = 128). Q K^T runs on e4m3 mma (m16n8k32) straight from the
// key bytes: an ldmatrix fragment of a 16-byte chunk gives a thread dims
// 4q..4q+3 of one key (q = lane % 4), which is the e4m3 B-operand layout. The
// query, bf16, is scaled per head by a power of two (its largest |q| into
// [128, 256)) and split into a high and a low e4m3 term (q = hi + lo/16, exact
// for bf16): the high terms are A rows 0-7 and the low terms rows 8-15, so one
// mma gives both partial products of a key and S = (hi + lo/16) * scale.
// For P V the transposed fragment holds two keys x two dims; the byte
// permutation splits it into the even-dim and the odd-dim n-tile, whose bytes
// become f16 in registers (exactly) for an f16 mma with the f16 P.
template <int D, int G, bool DENSE, int CH, bool HARD, bool FP8>
__global__ void __launch_bounds__(MmaWarps<D, CH, FP8>::kThreads, 1)
    decode_mma_kernel(const DecodeArgs a, const __grid_constant__ CUtensorMap tmk,
                      const __grid_constant__ CUtensorMap tmv) {
  constexpr int KST = D / 16;  // k-steps of QK^T
  constexpr int NDT = D / 8;   // n-tiles of PV
  static_assert(G >= 1 && G <= 8, "group size");
  static_assert(CH == 16 || CH == 32, "keys per chunk");
  constexpr int kMW = MmaWarps<D, CH, FP8>::kMW;
  constexpr int kMmaThreads = MmaWarps<D, CH, FP8>::kThreads;
  constexpr int EB = FP8 ? 1 : 2;  // bytes per element
  static_assert(!FP8 || D == 128, "fp8 K/V: d = 128");

  extern __shared__ __align__(16) unsigned char smem_raw[];
  unsigned char* smem = smem_raw + ((1024 - (smem_u32(smem_raw) & 1023)) & 1023);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int BH = a.B * a.Hkv;
  const int NST = a.nstages;
  // a ring position is rp rows of an admitted block: the whole block, or at
  // d = 128 a chunk of CH rows (a block of 64 or 128 tokens is 2 or 4
  // positions), so a warp has the next chunk in flight while it attends one
  const int rp = a.rpos, sl = a.sub_log2;
  const uint32_t tile_bytes = static_cast<uint32_t>(rp) * D * EB;
  unsigned char* s_tiles = smem;
  uint64_t* s_full = reinterpret_cast<uint64_t*>(smem + static_cast<size_t>(NST) * 2 * tile_bytes);
  uint64_t* s_empty = s_full + NST;
  uint64_t* s_aux = s_empty + NST;  // [8] per issuing lane: copies of a partial block
  int4* s_info = reinterpret_cast<int4*>(s_aux + 8);
  int* s_round = reinterpret_cast<int*>(s_info + NST);     // [NST] round each stage serves
  float* s_macc = reinterpret_cast<float*>(s_round + NST); // [kMW][G][D]
  float* s_mm = s_macc + kMW * G * D;                      // [kMW][G]
  float* s_ml = s_mm + kMW * G;                            // [kMW][G]
  int* s_abort = reinterpret_cast<int*>(s_ml + kMW * G);
  int32_t* s_pre = s_abort + 4;                            // [BH+1] segment starts

  grid_dependency_wait();  // inputs may come from the previous kernel on the stream
  allow_dependent_launch();
  // without per-row lengths a dense pass needs no table: segment i starts at i*nb
  const bool flat = DENSE && a.seq_lens == nullptr;
  if (!flat) block_prefix<DENSE>(a, s_pre, BH, kMmaThreads);
  if (tid == 0) {
    *s_abort = 0;
    for (int s = 0; s < NST; ++s) {
      mbar_init(&s_full[s], 1);
      mbar_init(&s_empty[s], 1);
    }
    for (int s = 0; s < 8; ++s) mbar_init(&s_aux[s], 1);
    for (int s = 0; s < NST; ++s) s_round[s] = 0;
    fence_mbar_init();
  }
  __syncthreads();

  // segment i's first position, and the segment of position p
  auto pre = [&](int i) -> int64_t {
    return (flat ? static_cast<int64_t>(i) * a.nb : static_cast<int64_t>(s_pre[i])) << sl;
  };
  auto seg_of = [&](int64_t p) -> int {
    return flat ? static_cast<int>((p >> sl) / a.nb) : find_seg(s_pre, BH, p >> sl);
  };
  const int64_t T = pre(BH);
  const int S = gridDim.x;
  const int kc = blockIdx.x;
  const int64_t lo = static_cast<int64_t>(kc) * T / S;
  const int64_t hi = static_cast<int64_t>(kc + 1) * T / S;
  if (lo >= hi) return;

  if (warp == kMW) {
    // ------------------------------------------------------------ producer
    const uint64_t pol = l2_policy_evict_first();
    uint32_t aux_phase = 0;  // this lane's partial-block barrier
    auto issue = [&](int st, int row0, int rows) {
      // whole boxes land even for a partial block (rows past the store's end
      // read as zeros)
      const int y = row0;
      unsigned char* kt = s_tiles + static_cast<size_t>(st) * 2 * tile_bytes;
      unsigned char* vt = kt + tile_bytes;
      uint64_t* bar = rows == rp ? &s_full[st] : &s_aux[lane];
      mbar_arrive_expect_tx(bar, 2 * tile_bytes);
      constexpr int kBoxElems = 128 / EB;  // a box row is 128 bytes
#pragma unroll
      for (int h = 0; h < D / kBoxElems; ++h) {
        tma_load_2d(kt + h * rp * 128, &tmk, h * kBoxElems, y, bar, pol);
        tma_load_2d(vt + h * rp * 128, &tmv, h * kBoxElems, y, bar, pol);
      }
      if (rows == rp) return;
      // Partial block: the store's rows past the row's last token may hold
      // anything, NaN included. Their keys are masked by the consumer, but
      // P = 0 times NaN would still reach O, so their values are zeroed here
      // once the copies have landed, before the stage is handed over.
      if (!mbar_wait_bounded(bar, aux_phase, s_abort, a.status)) {
        const uint64_t t0 = global_timer_ns();  // copies still in flight: let them land
        while (!mbar_try_wait(bar, aux_phase) && global_timer_ns() - t0 < kWaitLimitNs) {
        }
      }
      aux_phase ^= 1u;
      for (int r = rows; r < rp; ++r)
#pragma unroll
        for (int c = 0; c < D * EB / 16; ++c) *reinterpret_cast<uint4*>(vt + swz(rp, r, c)) = make_uint4(0u, 0u, 0u, 0u);
      // generic-proxy writes: order them before the next TMA write into the stage
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      mbar_arrive(&s_full[st]);
    };
    producer_loop<G, DENSE, MmaWarps<D, CH, FP8>::kIssueLanes>(a, lo, hi, NST, s_empty, s_info, s_abort, seg_of,
                                                               pre, issue, s_full, s_round);
    return;
  }

  // -------------------------------------------------------------- consumers
  const int row = lane >> 2, qd = lane & 3;
  const bool live_row = row < G;
  uint32_t qa[KST][2];  // bf16 query fragments of the k16 steps
  uint32_t q8[4][4];    // fp8: e4m3 query fragments of the k32 steps (rows 8-15: low terms)
  float qs_r = a.qscale;  // fp8: 1/sqrt(d) over this head's query scale
  float o[NDT][4];  // [n-tile][c0 c1 = high part of row, c2 c3 = low part]
  float m_r = -INFINITY, l_r = 0.0f, tau_r = 0.0f;
  int64_t t_cur = 0;  // position of the current token of the segment being attended

  auto load_q = [&](int seg) {
    const int b = seg / a.Hkv, kvh = seg % a.Hkv;
    t_cur = seg_tokens(a, seg) - 1;
    if constexpr (FP8) {
      const uint16_t* qp =
          static_cast<const uint16_t*>(a.q) + (static_cast<int64_t>(b) * a.Hq + kvh * G + (live_row ? row : 0)) * D;
      tau_r = live_row ? (a.tau != nullptr ? a.tau[b * a.tau_stride + kvh * G + row] : -INFINITY) : 0.0f;
      // this thread's dims of k32 step kk: 32kk + 4qd + i (i < 4), then 16 more
      float x[4][8];
      float amax = 0.0f;
#pragma unroll
      for (int kk = 0; kk < 4; ++kk)
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const int c = 32 * kk + 16 * (i >> 2) + 4 * qd + (i & 3);
          x[kk][i] = live_row ? __uint_as_float(static_cast<uint32_t>(qp[c]) << 16) : 0.0f;
          amax = fmaxf(amax, fabsf(x[kk][i]));
        }
      amax = fmaxf(amax, __shfl_xor_sync(kFull, amax, 1));
      amax = fmaxf(amax, __shfl_xor_sync(kFull, amax, 2));
      // 2^e with 2^e * amax in [128, 256) (amax = 2^(E-127) * 1.f)
      const int E = (__float_as_int(amax) >> 23) & 0xff;
      const int e = E == 0 ? 0 : max(-120, min(120, 134 - E));
      const float up = __int_as_float((127 + e) << 23);
      qs_r = a.qscale * __int_as_float((127 - e) << 23);
#pragma unroll
      for (int kk = 0; kk < 4; ++kk) {
        e4m3_split4(x[kk][0] * up, x[kk][1] * up, x[kk][2] * up, x[kk][3] * up, q8[kk][0], q8[kk][1]);
        e4m3_split4(x[kk][4] * up, x[kk][5] * up, x[kk][6] * up, x[kk][7] * up, q8[kk][2], q8[kk][3]);
      }
    } else if (live_row) {
      const uint16_t* qp =
          static_cast<const uint16_t*>(a.q) + (static_cast<int64_t>(b) * a.Hq + kvh * G + row) * D;
#pragma unroll
      for (int kk = 0; kk < KST; ++kk) {
        const int c = 16 * kk + 2 * qd;
        qa[kk][0] = static_cast<uint32_t>(qp[c]) | (static_cast<uint32_t>(qp[c + 1]) << 16);
        qa[kk][1] = static_cast<uint32_t>(qp[c + 8]) | (static_cast<uint32_t>(qp[c + 9]) << 16);
      }
      tau_r = a.tau != nullptr ? a.tau[b * a.tau_stride + kvh * G + row] : -INFINITY;
    } else {
#pragma unroll
      for (int kk = 0; kk < KST; ++kk) qa[kk][0] = qa[kk][1] = 0u;
      tau_r = 0.0f;
    }
    m_r = -INFINITY;
    l_r = 0.0f;
#pragma unroll
    for (int j = 0; j < NDT; ++j) o[j][0] = o[j][1] = o[j][2] = o[j][3] = 0.0f;
  };

  auto flush = [&](int seg) {
    float l = l_r + __shfl_xor_sync(kFull, l_r, 1);
    l += __shfl_xor_sync(kFull, l, 2);
    if (live_row) {
#pragma unroll
      for (int j = 0; j < NDT; ++j) {
        if constexpr (FP8) {  // n-tile 2g + p holds dims 16g + 2c + p
          const int base = 16 * (j >> 1) + (j & 1);
          s_macc[(warp * G + row) * D + base + 4 * qd] = o[j][0] + o[j][2];
          s_macc[(warp * G + row) * D + base + 4 * qd + 2] = o[j][1] + o[j][3];
        } else {
          s_macc[(warp * G + row) * D + 8 * j + 2 * qd] = o[j][0] + o[j][2];
          s_macc[(warp * G + row) * D + 8 * j + 2 * qd + 1] = o[j][1] + o[j][3];
        }
      }
      if (qd == 0) {
        s_mm[warp * G + row] = m_r;
        s_ml[warp * G + row] = l;
      }
    }
    named_barrier_sync(1, kMW * 32);
    finish_segment<D, G, kMW>(a, seg, pre(seg), pre(seg + 1), lo, T, S, s_macc, s_mm, s_ml, s_abort + 1);
  };

  // gate in log2 units: g = S * sigmoid(beta (S - tau)) * log2(e), or (strict
  // mode) S * log2(e) for S >= tau and -inf below
  const float nbl = -a.beta * kLog2e;
  auto gate = [&](float Sv) {
    if (HARD) return Sv >= tau_r ? Sv * kLog2e : -INFINITY;
    return Sv * rcp_approx(1.0f + ex2_approx(nbl * (Sv - tau_r))) * kLog2e;
  };

  const float qscale = a.qscale;
  auto process = [&](int st, const int4 inf) {
    const uint32_t kt = smem_u32(s_tiles + static_cast<size_t>(st) * 2 * tile_bytes);
    const uint32_t vt = kt + tile_bytes;
    const int rows = inf.z;
    const bool row_on = live_row && ((static_cast<uint32_t>(inf.y) >> row) & 1u);
    const int64_t tok0 = static_cast<int64_t>(inf.x) * rp;
    // full position that does not hold the current token: no per-key checks
    const bool fast = rows == rp && tok0 + rp <= t_cur;
    constexpr int NT = CH / 8;  // n-tiles of 8 keys per chunk
    for (int c0 = 0; c0 < rp; c0 += CH) {
      // S = Q K^T: even and odd k-steps accumulate separately (shorter mma chains)
      float se[NT][2], so[NT][2];  // bf16: partial sums of the even and odd k-steps
      float sv[FP8 ? NT : 1][2];   // fp8: the scaled logits
      if constexpr (FP8) {
        // two 16-byte chunks are one k32 step: an x4 load gives 2 k-steps of one n-tile
        float sa[NT][4], sb[NT][4];
#pragma unroll
        for (int j = 0; j < NT; ++j)
#pragma unroll
          for (int r = 0; r < 4; ++r) sa[j][r] = sb[j][r] = 0.0f;
#pragma unroll
        for (int u = 0; u < 2; ++u) {
          uint32_t bb[NT][4];
#pragma unroll
          for (int j = 0; j < NT; ++j)
            ldsm_x4(kt + swz(rp, c0 + 8 * j + (lane & 7), 4 * u + (lane >> 3)), bb[j][0], bb[j][1], bb[j][2],
                    bb[j][3]);
#pragma unroll
          for (int j = 0; j < NT; ++j) mma_16832_e4m3(sa[j], q8[2 * u], bb[j][0], bb[j][1]);
#pragma unroll
          for (int j = 0; j < NT; ++j) mma_16832_e4m3(sb[j], q8[2 * u + 1], bb[j][2], bb[j][3]);
        }
        // rows 0-7 hold the high-term products, rows 8-15 the low-term ones
#pragma unroll
        for (int j = 0; j < NT; ++j)
#pragma unroll
          for (int e = 0; e < 2; ++e) sv[j][e] = fmaf(sa[j][2 + e] + sb[j][2 + e], 0.0625f, sa[j][e] + sb[j][e]) * qs_r;
      } else {
#pragma unroll
        for (int j = 0; j < NT; ++j) se[j][0] = se[j][1] = so[j][0] = so[j][1] = 0.0f;
#pragma unroll
        for (int k2 = 0; k2 < KST / 2; ++k2) {
          uint32_t bb[NT][4];
#pragma unroll
          for (int j = 0; j < NT; ++j)
            ldsm_x4(kt + swz(rp, c0 + 8 * j + (lane & 7), 4 * k2 + (lane >> 3)), bb[j][0], bb[j][1], bb[j][2],
                    bb[j][3]);
#pragma unroll
          for (int j = 0; j < NT; ++j)
            mma_rows8(se[j][0], se[j][1], qa[2 * k2][0], qa[2 * k2][1], bb[j][0], bb[j][1]);
#pragma unroll
          for (int j = 0; j < NT; ++j)
            mma_rows8(so[j][0], so[j][1], qa[2 * k2 + 1][0], qa[2 * k2 + 1][1], bb[j][2], bb[j][3]);
        }
      }
      auto s_at = [&](int j, int e) {  // scaled logit of key 8j + 2qd + e of the chunk
        if constexpr (FP8) return sv[j][e];
        else return (se[j][e] + so[j][e]) * qscale;
      };
      // gate (Eq. 2-3) and online softmax on this thread's row
      float g[NT][2];
      float bm = -INFINITY;
      if (fast) {
#pragma unroll
        for (int j = 0; j < NT; ++j)
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            const float v = row_on ? gate(s_at(j, e)) : -INFINITY;
            g[j][e] = v;
            bm = fmaxf(bm, v);
          }
      } else {
#pragma unroll
        for (int j = 0; j < NT; ++j)
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            const int key = c0 + 8 * j + 2 * qd + e;
            float v = -INFINITY;
            if (row_on && key < rows) {
              const float Sv = s_at(j, e);
              // the current token is exempt from the gate (Eq. 3)
              v = (tok0 + key == t_cur) ? Sv * kLog2e : gate(Sv);
            }
            g[j][e] = v;
            bm = fmaxf(bm, v);
          }
      }
      bm = fmaxf(bm, __shfl_xor_sync(kFull, bm, 1));
      bm = fmaxf(bm, __shfl_xor_sync(kFull, bm, 2));
      const float mn = fmaxf(m_r, bm);
      float corr = 1.0f, ps = 0.0f;
      float p[NT][2];
      if (mn != -INFINITY) {
        corr = ex2_approx(m_r - mn);
#pragma unroll
        for (int j = 0; j < NT; ++j)
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            p[j][e] = ex2_approx(g[j][e] - mn);
            ps += p[j][e];
          }
      } else {
#pragma unroll
        for (int j = 0; j < NT; ++j) p[j][0] = p[j][1] = 0.0f;
      }
      l_r = fmaf(l_r, corr, ps);
      m_r = mn;
      if (__any_sync(kFull, corr != 1.0f)) {
#pragma unroll
        for (int j = 0; j < NDT; ++j) {
          o[j][0] *= corr;
          o[j][1] *= corr;
          o[j][2] *= corr;
          o[j][3] *= corr;
        }
      }
      // O += P V, P = high + low parts (bf16, or f16 with fp8 values)
#pragma unroll
      for (int m2 = 0; m2 < NT / 2; ++m2) {
        const int vrow = c0 + 16 * m2 + 8 * ((lane >> 3) & 1) + (lane & 7);
        if constexpr (FP8) {
          const uint32_t h0 = pack_f16x2(p[2 * m2][0], p[2 * m2][1]);
          const uint32_t h1 = pack_f16x2(p[2 * m2 + 1][0], p[2 * m2 + 1][1]);
          const __half2 hh0 = *reinterpret_cast<const __half2*>(&h0);
          const __half2 hh1 = *reinterpret_cast<const __half2*>(&h1);
          const uint32_t l0 = pack_f16x2(p[2 * m2][0] - __low2float(hh0), p[2 * m2][1] - __high2float(hh0));
          const uint32_t l1 = pack_f16x2(p[2 * m2 + 1][0] - __low2float(hh1), p[2 * m2 + 1][1] - __high2float(hh1));
          // one x4 transposed load: keys 0-7 / 8-15 of dim chunks g and g+1 (16 dims each)
#pragma unroll
          for (int g = 0; g < D / 16; g += 2) {
            uint32_t r0, r1, r2, r3;
            ldsm_x4_t(vt + swz(rp, vrow, g + (lane >> 4)), r0, r1, r2, r3);
            // each register: keys 2q, 2q+1 x dims 2c, 2c+1; regroup into the
            // even-dim and the odd-dim key pairs (bytes 0,2 and 1,3)
            uint32_t e0, o0, e1, o1, e2, o2, e3, o3;
            auto split = [](uint32_t r, uint32_t& ev, uint32_t& od) {
              uint32_t t;
              asm("prmt.b32 %0, %1, %2, %3;" : "=r"(t) : "r"(r), "r"(0u), "r"(0x3120u));
              e4m3x4_to_f16x2x2(t, ev, od);
            };
            split(r0, e0, o0);
            split(r1, e1, o1);
            split(r2, e2, o2);
            split(r3, e3, o3);
            mma_16816_f16(o[2 * g], h0, l0, h1, l1, e0, e1);
            mma_16816_f16(o[2 * g + 1], h0, l0, h1, l1, o0, o1);
            mma_16816_f16(o[2 * g + 2], h0, l0, h1, l1, e2, e3);
            mma_16816_f16(o[2 * g + 3], h0, l0, h1, l1, o2, o3);
          }
        } else {
          const uint32_t h0 = pack_bf16x2(p[2 * m2][0], p[2 * m2][1]);
          const uint32_t h1 = pack_bf16x2(p[2 * m2 + 1][0], p[2 * m2 + 1][1]);
          const __nv_bfloat162 hb0 = *reinterpret_cast<const __nv_bfloat162*>(&h0);
          const __nv_bfloat162 hb1 = *reinterpret_cast<const __nv_bfloat162*>(&h1);
          const uint32_t l0 = pack_bf16x2(p[2 * m2][0] - __low2float(hb0), p[2 * m2][1] - __high2float(hb0));
          const uint32_t l1 = pack_bf16x2(p[2 * m2 + 1][0] - __low2float(hb1), p[2 * m2 + 1][1] - __high2float(hb1));
#pragma unroll
          for (int jd = 0; jd < NDT; jd += 2) {
            uint32_t b0, b1, b2, b3;
            ldsm_x4_t(vt + swz(rp, vrow, jd + (lane >> 4)), b0, b1, b2, b3);
            // A rows 0-7: high part, rows 8-15: low part of the same P row
            mma_16816(o[jd], h0, l0, h1, l1, b0, b1);
            mma_16816(o[jd + 1], h0, l0, h1, l1, b2, b3);
          }
        }
      }
    }
  };

  int cur = seg_of(lo);
  int64_t eff_end = min(pre(cur + 1), hi);
  load_q(cur);
  for (int64_t p = lo + warp;; p += kMW) {
    // every segment that ends at or before this warp's next position is done
    // for this warp; all consumer warps flush the same segments in order
    const int64_t lim = p < hi ? p : hi;
    bool finished = false;
    while (eff_end <= lim) {
      flush(cur);
      if (eff_end >= hi) {
        finished = true;
        break;
      }
      do {
        ++cur;
      } while (pre(cur + 1) <= eff_end);
      eff_end = min(pre(cur + 1), hi);
      load_q(cur);
    }
    if (finished || p >= hi) break;
    const int it = static_cast<int>(p - lo);
    const int st = it % NST;
    const int round = it / NST;
    // Consecutive uses of a stage belong to different warps, so this warp may
    // get here rounds ahead of the stage (with fewer stages than warps, even
    // before the round before it has been released), and an mbarrier parity
    // wait on a phase two or more ahead returns at once. Wait until the
    // producer has published this round for the stage: it does so only after
    // the previous round's release, so the full barrier is then in this round's
    // phase and the parity wait below is exact. (With a stage count that is a
    // multiple of kMW a stage always returns to the same warp, which released
    // it itself, and the extra wait is skipped.)
    bool ok = round == 0 || (NST % kMW) == 0 || wait_value_bounded(s_round + st, round, s_abort, a.status);
    ok = ok && mbar_wait_bounded(&s_full[st], static_cast<uint32_t>(round & 1), s_abort, a.status);
    // the tile math is warp-synchronous: the whole warp processes the stage or
    // none of it; a stage whose wait failed is not released (its copies may
    // still be in flight), and the producer stops once it sees the abort
    ok = __all_sync(kFull, ok);
    if (ok) {
      // a position with no rows (a chunk past its row's last token) loaded
      // nothing: its stage holds stale data, so it is not attended
      const int4 inf = s_info[st];
      if (inf.z > 0) process(st, inf);
      __syncwarp();
      if (lane == 0) mbar_arrive(&s_empty[st]);
    }
  }
}

PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
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

// [rows][d] view of a K or V store (bf16, or fp8 bytes), boxes of [box_rows]
// rows of 128 bytes with the 128-byte swizzle.
bool encode_kv_map(CUtensorMap* tm, const void* base, int64_t rows, int d, int box_rows, bool fp8) {
  PFN_cuTensorMapEncodeTiled_v12000 enc = tensor_map_encoder();
  if (enc == nullptr) return false;
  const int eb = fp8 ? 1 : 2;
  const cuuint64_t gdim[2] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(rows)};
  const cuuint64_t gstride[1] = {static_cast<cuuint64_t>(d) * eb};
  const cuuint32_t box[2] = {static_cast<cuuint32_t>(128 / eb), static_cast<cuuint32_t>(box_rows)};
  const cuuint32_t estride[2] = {1u, 1u};
  return enc(tm, fp8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base),
             gdim, gstride, box, estride, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int D, int G, bool DENSE, int CH, bool FP8>
cudaError_t launch_mma_t(const DecodeCall& c, cudaStream_t st) {
  const eta_shape_t& s = c.shape;
  const int BH = s.batch * s.n_kv_heads;
  // rows per ring position: 32-row chunks of the blocks at d = 128 (a warp
  // then has its next chunk in flight while it attends one: 36.9 -> 34.8 us on
  // the 32K batch-1 decode), whole blocks at d = 64, whose 8 KB chunks cost
  // more per position than they gain (1,738 -> 1,881 us on the Table 10 shape)
  const int rp = D == 128 ? CH : s.block_size;
  const size_t tile = static_cast<size_t>(rp) * D * (FP8 ? 1 : 2);  // one position of K (or V)
  constexpr int kMW = MmaWarps<D, CH, FP8>::kMW;
  constexpr unsigned kThreads = MmaWarps<D, CH, FP8>::kThreads;
  const size_t fixed = static_cast<size_t>(kMW) * G * (D + 2) * sizeof(float) + 16 + 8 * sizeof(uint64_t) +
                       static_cast<size_t>(BH + 1) * sizeof(int32_t) + 1024;
  const size_t per_stage = 2 * tile + 2 * sizeof(uint64_t) + sizeof(int4) + sizeof(int);
  const size_t budget = static_cast<size_t>(device_max_smem_optin()) - 512;
  if (fixed + 2 * per_stage > budget) return cudaErrorInvalidValue;
  // ~200 KB of stages: the consumer warps hold up to kMW, the rest are in flight.
  const size_t nst_bw = (200 * 1024) / (2 * tile), nst_fit = (budget - fixed) / per_stage;
  int nst = static_cast<int>(nst_bw < nst_fit ? nst_bw : nst_fit);
  nst = max(2, min(nst, FP8 ? 32 : 24));
  // With at least 2*kMW stages, round down to a multiple of kMW so a stage
  // always returns to the warp that released it (see the consumer loop).
  if (nst >= 2 * kMW) nst -= nst % kMW;
  const size_t smem = static_cast<size_t>(nst) * per_stage + fixed + 64;

  CUtensorMap tmk, tmv;
  const int64_t rows = c.block_table != nullptr ? static_cast<int64_t>(c.num_pages) * s.n_kv_heads * s.block_size
                                                : static_cast<int64_t>(BH) * s.capacity;
  if (!encode_kv_map(&tmk, c.k, rows, D, rp, FP8) || !encode_kv_map(&tmv, c.v, rows, D, rp, FP8))
    return cudaErrorInvalidValue;

  const DecodeArgs a = make_decode_args(c, nst, rp);
  if (c.gate == ETA_GATE_HARD) {
    static std::atomic<uint64_t> smem_done{0};
    const void* fn = reinterpret_cast<const void*>(decode_mma_kernel<D, G, DENSE, CH, true, FP8>);
    cudaError_t e = allow_max_smem(smem_done, fn);
    if (e != cudaSuccess) return e;
    return launch_pdl(decode_mma_kernel<D, G, DENSE, CH, true, FP8>, static_cast<unsigned>(c.S), kThreads, smem, st,
                      a, tmk, tmv);
  }
  static std::atomic<uint64_t> smem_done{0};
  const void* fn = reinterpret_cast<const void*>(decode_mma_kernel<D, G, DENSE, CH, false, FP8>);
  cudaError_t e = allow_max_smem(smem_done, fn);
  if (e != cudaSuccess) return e;
  return launch_pdl(decode_mma_kernel<D, G, DENSE, CH, false, FP8>, static_cast<unsigned>(c.S), kThreads, smem, st,
                    a, tmk, tmv);
}

template <int D, bool DENSE, int CH, bool FP8>
cudaError_t launch_mma_g(const DecodeCall& c, cudaStream_t st) {
  switch (c.shape.n_q_heads / c.shape.n_kv_heads) {
    case 1: return launch_mma_t<D, 1, DENSE, CH, FP8>(c, st);
    case 2: return launch_mma_t<D, 2, DENSE, CH, FP8>(c, st);
    case 4: return launch_mma_t<D, 4, DENSE, CH, FP8>(c, st);
    case 8: return launch_mma_t<D, 8, DENSE, CH, FP8>(c, st);
    default: return cudaErrorInvalidValue;
  }
}

// Chunks of 32 keys, or 16 for 16-token blocks and for fp8 K/V (whose
// conversions need the registers of the second half-chunk).
template <int D, bool DENSE, bool FP8>
cudaError_t launch_mma_c(const DecodeCall& c, cudaStream_t st) {
  if (c.shape.block_size == 16) return launch_mma_g<D, DENSE, 16, FP8>(c, st);
  return launch_mma_g<D, DENSE, 32, FP8>(c, st);
}

}  // namespace

cudaError_t launch_decode_mma(const DecodeCall& c, cudaStream_t st) {
  if (c.shape.kv_dtype == ETA_FP8_E4M3) {
    if (c.shape.head_dim != 128) return cudaErrorInvalidValue;
    return c.dense ? launch_mma_c<128, true, true>(c, st) : launch_mma_c<128, false, true>(c, st);
  }
  if (c.shape.head_dim == 128)
    return c.dense ? launch_mma_c<128, true, false>(c, st) : launch_mma_c<128, false, false>(c, st);
  return c.dense ? launch_mma_c<64, true, false>(c, st) : launch_mma_c<64, false, false>(c, st);
}

}  // namespace eta

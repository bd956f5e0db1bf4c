// Block-sparse flash decoding over the admitted blocks (Figure 1 right,
// Figure 6), with the ETA logit gate of Eq. 2-3 and an online softmax, and the
// merge of the split partials in the same kernel.
//
// Work split. The admitted (union) blocks of all (batch, kv head) pairs form
// one flat sequence of T entries; thread block k of S takes the contiguous
// range [k*T/S, (k+1)*T/S), so every SM streams the same number of blocks
// whatever the per-head densities are. Where a range crosses a (batch, kv head)
// boundary the thread block emits one partial (running max, running sum,
// unnormalised output) per query head; the thread block that writes the last
// partial of a segment merges them (finish_segment), and a segment inside one
// range is written out directly.
//
// This file holds the CUDA-core consumer (fp32 K/V, or bf16 K/V with fp32
// queries) and the dispatch; bf16 K/V with bf16 queries
// go to the tensor-core consumer in decode_mma.cu.
//
// Pipeline. Warp 8 is the producer: one lane issues two 1-D TMA bulk copies
// (K block, V block: b*d contiguous elements each) per admitted block into a
// ring of shared-memory stages guarded by mbarriers; the copies carry an
// L2 evict-first policy since every KV block is read once per step. Warps 0-7
// consume: a block's keys are dealt round-robin to "slots" of d*elt/16 lanes,
// each lane holding 16 bytes of the key row (one 128-bit shared load), so a
// dot product is a per-lane FMA run plus a shuffle butterfly over the slot.
// Each slot keeps its own running max / sum / output for the G query heads of
// the group (in log2 units), rescaled once per chunk of keys; slots are
// merged with shuffles and through shared memory when a partial is emitted.
//
// Every mbarrier wait is bounded (2 s); on timeout the status word is set,
// the CTA stops issuing copies, waits for the copies already in flight and
// finishes with the same control flow, so no thread is left at a barrier.
#include "decode_common.cuh"

namespace eta {

namespace {

constexpr int kNW = 8;                       // consumer warps
constexpr int kDecThreads = (kNW + 1) * 32;  // + one producer warp

template <typename KV, int D, int G, bool DENSE>
__global__ void __launch_bounds__(kDecThreads, 1) decode_kernel(const DecodeArgs a) {
  constexpr int EB = KvTraits<KV>::kBytes;
  constexpr int VEC = 16 / EB;       // elements per lane per key row
  constexpr int LPK = D / VEC;       // lanes per key ("slot" width)
  constexpr int KPW = 32 / LPK;      // slots per warp
  constexpr int NSLOT = kNW * KPW;
  constexpr int KPS = (128 + NSLOT - 1) / NSLOT;   // keys per slot per block, block size <= 128
  constexpr int KCH = KPS < 4 ? KPS : 4;           // keys per online-softmax chunk
  static_assert(LPK >= 1 && LPK <= 32 && (32 % LPK) == 0, "bad lane split");

  extern __shared__ __align__(1024) unsigned char smem[];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int BH = a.B * a.Hkv;
  const int NST = a.nstages;
  const uint32_t tile_bytes = static_cast<uint32_t>(a.bs) * D * EB;
  unsigned char* s_tiles = smem;
  uint64_t* s_full = reinterpret_cast<uint64_t*>(smem + static_cast<size_t>(NST) * 2 * tile_bytes);
  uint64_t* s_empty = s_full + NST;
  int4* s_info = reinterpret_cast<int4*>(s_empty + NST);
  float* s_macc = reinterpret_cast<float*>(s_info + NST);  // [kNW][G][D]
  float* s_mm = s_macc + kNW * G * D;                      // [kNW][G]
  float* s_ml = s_mm + kNW * G;                            // [kNW][G]
  int* s_abort = reinterpret_cast<int*>(s_ml + kNW * G);
  int32_t* s_pre = s_abort + 4;                            // [BH+1] segment starts

  grid_dependency_wait();  // inputs may come from the previous kernel on the stream
  allow_dependent_launch();
  // without per-row lengths a dense pass needs no table: segment i starts at i*nb
  const bool flat = DENSE && a.seq_lens == nullptr;
  if (!flat) block_prefix<DENSE>(a, s_pre, BH, kDecThreads);
  if (tid == 0) {
    *s_abort = 0;
    for (int s = 0; s < NST; ++s) {
      mbar_init(&s_full[s], 1);
      mbar_init(&s_empty[s], kNW);
    }
    fence_mbar_init();
  }
  __syncthreads();

  auto pre = [&](int i) -> int64_t {
    return flat ? static_cast<int64_t>(i) * a.nb : static_cast<int64_t>(s_pre[i]);
  };
  auto seg_of = [&](int64_t p) -> int {
    return flat ? static_cast<int>(p / a.nb) : find_seg(s_pre, BH, p);
  };
  const int64_t T = pre(BH);
  const int S = gridDim.x;
  const int kc = blockIdx.x;
  const int64_t lo = static_cast<int64_t>(kc) * T / S;
  const int64_t hi = static_cast<int64_t>(kc + 1) * T / S;
  if (lo >= hi) return;

  if (warp == kNW) {
    // ------------------------------------------------------------ producer
    const uint64_t pol = l2_policy_evict_first();
    const KV* kb = static_cast<const KV*>(a.k);
    const KV* vb = static_cast<const KV*>(a.v);
    auto issue = [&](int st, int row0, int rows) {
      const uint32_t bytes = static_cast<uint32_t>(rows) * D * EB;
      mbar_arrive_expect_tx(&s_full[st], 2 * bytes);
      const int64_t off = static_cast<int64_t>(row0) * D;
      bulk_g2s(s_tiles + static_cast<size_t>(st) * 2 * tile_bytes, kb + off, bytes, &s_full[st], pol);
      bulk_g2s(s_tiles + (static_cast<size_t>(st) * 2 + 1) * tile_bytes, vb + off, bytes, &s_full[st], pol);
    };
    producer_loop<G, DENSE, 4>(a, lo, hi, NST, s_empty, s_info, s_abort, seg_of, pre, issue, s_full);
    return;
  }

  // -------------------------------------------------------------- consumers
  const int slot = warp * KPW + lane / LPK;
  const int dl = lane % LPK;
  float qv[G][VEC], acc[G][VEC], mrun[G], lrun[G], tg[G];
  int cur = seg_of(lo);
  int64_t seg_end = pre(cur + 1);
  int64_t t_cur = 0;  // position of the current token of segment `cur`

  auto load_q = [&](int seg) {
    const int b = seg / a.Hkv, kvh = seg % a.Hkv;
    t_cur = seg_tokens(a, seg) - 1;
#pragma unroll
    for (int g = 0; g < G; ++g) {
      const int hq = kvh * G + g;
      const int64_t base = (static_cast<int64_t>(b) * a.Hq + hq) * D + dl * VEC;
#pragma unroll
      for (int e = 0; e < VEC; ++e) qv[g][e] = load_elem(a.q, a.q_dtype, base + e) * a.qscale;
      tg[g] = a.tau != nullptr ? a.tau[b * a.tau_stride + hq] : -INFINITY;
      mrun[g] = -INFINITY;
      lrun[g] = 0.0f;
#pragma unroll
      for (int e = 0; e < VEC; ++e) acc[g][e] = 0.0f;
    }
  };
  load_q(cur);

  int it = 0;
  for (int64_t p = lo; p < hi; ++p, ++it) {
    const int st = it % NST;
    // the warp's lanes reduce together: all of them process the stage or none
    const bool ok =
        __all_sync(kFull, mbar_wait_bounded(&s_full[st], static_cast<uint32_t>((it / NST) & 1), s_abort, a.status));
    if (ok) {
      const int4 inf = s_info[st];
      const unsigned char* kt = s_tiles + static_cast<size_t>(st) * 2 * tile_bytes;
      const unsigned char* vt = kt + tile_bytes;
      const int rows = inf.z;
      const uint32_t mask = static_cast<uint32_t>(inf.y);
      const int64_t tok0 = static_cast<int64_t>(inf.x) * a.bs;
      for (int c0 = 0; c0 < rows; c0 += KCH * NSLOT) {
        float sc[KCH][G];
#pragma unroll
        for (int jj = 0; jj < KCH; ++jj) {
          const int r = c0 + jj * NSLOT + slot;
          const int rr = r < rows ? r : 0;
          const uint4 w = *reinterpret_cast<const uint4*>(kt + (static_cast<size_t>(rr) * D + dl * VEC) * EB);
          float x[VEC];
          widen16<KV>(w, x);
#pragma unroll
          for (int g = 0; g < G; ++g) {
            float s = 0.0f;
#pragma unroll
            for (int e = 0; e < VEC; ++e) s = fmaf(qv[g][e], x[e], s);
            sc[jj][g] = s;
          }
        }
#pragma unroll
        for (int o = LPK / 2; o >= 1; o >>= 1)
#pragma unroll
          for (int jj = 0; jj < KCH; ++jj)
#pragma unroll
            for (int g = 0; g < G; ++g) sc[jj][g] += __shfl_xor_sync(kFull, sc[jj][g], o);

        float pp[KCH][G];
#pragma unroll
        for (int g = 0; g < G; ++g) {
          const bool on = (mask >> g) & 1u;
          float gl[KCH];
          float bm = -INFINITY;
#pragma unroll
          for (int jj = 0; jj < KCH; ++jj) {
            const int r = c0 + jj * NSLOT + slot;
            float v = -INFINITY;
            if (on && r < rows) {
              const float S = sc[jj][g];
              if (tok0 + r == t_cur) {
                v = S * kLog2e;   // current token: gate exempt (Eq. 3)
              } else if (a.gate == ETA_GATE_HARD) {
                v = S >= tg[g] ? S * kLog2e : -INFINITY;   // strict mode: removed below tau
              } else {
                const float x = a.beta * (S - tg[g]);
                const float sig = __frcp_rn(1.0f + exp2f(-x * kLog2e));
                v = S * sig * kLog2e;
              }
            }
            gl[jj] = v;
            bm = fmaxf(bm, v);
          }
          const float mn = fmaxf(mrun[g], bm);
          if (mn != -INFINITY) {
            const float corr = exp2f(mrun[g] - mn);
            float ps = 0.0f;
#pragma unroll
            for (int jj = 0; jj < KCH; ++jj) {
              pp[jj][g] = exp2f(gl[jj] - mn);
              ps += pp[jj][g];
            }
            lrun[g] = fmaf(lrun[g], corr, ps);
            mrun[g] = mn;
#pragma unroll
            for (int e = 0; e < VEC; ++e) acc[g][e] *= corr;
          } else {
#pragma unroll
            for (int jj = 0; jj < KCH; ++jj) pp[jj][g] = 0.0f;
          }
        }
#pragma unroll
        for (int jj = 0; jj < KCH; ++jj) {
          const int r = c0 + jj * NSLOT + slot;
          if (c0 + jj * NSLOT < rows) {
            const int rr = r < rows ? r : 0;
            const uint4 w = *reinterpret_cast<const uint4*>(vt + (static_cast<size_t>(rr) * D + dl * VEC) * EB);
            float x[VEC];
            widen16<KV>(w, x);
#pragma unroll
            for (int g = 0; g < G; ++g)
#pragma unroll
              for (int e = 0; e < VEC; ++e) acc[g][e] = fmaf(pp[jj][g], x[e], acc[g][e]);
          }
        }
      }
    }
    __syncwarp();
    if (ok && lane == 0) mbar_arrive(&s_empty[st]);  // a stage whose wait failed is not released

    if (p + 1 == seg_end || p + 1 == hi) {
      // ---- emit this range's partial for segment `cur`
#pragma unroll
      for (int o = LPK; o < 32; o <<= 1) {
#pragma unroll
        for (int g = 0; g < G; ++g) {
          const float mo = __shfl_xor_sync(kFull, mrun[g], o);
          const float lo_ = __shfl_xor_sync(kFull, lrun[g], o);
          const float M = fmaxf(mrun[g], mo);
          const float ca = M == -INFINITY ? 0.0f : exp2f(mrun[g] - M);
          const float cb = M == -INFINITY ? 0.0f : exp2f(mo - M);
          lrun[g] = lrun[g] * ca + lo_ * cb;
#pragma unroll
          for (int e = 0; e < VEC; ++e) {
            const float ao = __shfl_xor_sync(kFull, acc[g][e], o);
            acc[g][e] = acc[g][e] * ca + ao * cb;
          }
          mrun[g] = M;
        }
      }
      if (lane < LPK) {
#pragma unroll
        for (int g = 0; g < G; ++g) {
#pragma unroll
          for (int e = 0; e < VEC; ++e) s_macc[(warp * G + g) * D + dl * VEC + e] = acc[g][e];
          if (lane == 0) {
            s_mm[warp * G + g] = mrun[g];
            s_ml[warp * G + g] = lrun[g];
          }
        }
      }
      named_barrier_sync(1, kNW * 32);
      finish_segment<D, G, kNW>(a, cur, pre(cur), pre(cur + 1), lo, T, S, s_macc, s_mm, s_ml, s_abort + 1);
      if (p + 1 < hi) {
        do {
          ++cur;
        } while (pre(cur + 1) <= p + 1);
        seg_end = pre(cur + 1);
        load_q(cur);
      }
    }
  }
}

template <typename KV, int D, int G, bool DENSE>
cudaError_t launch_decode_t(const DecodeCall& c, cudaStream_t st) {
  const eta_shape_t& s = c.shape;
  constexpr int EB = KvTraits<KV>::kBytes;
  const int BH = s.batch * s.n_kv_heads;
  const size_t tile = static_cast<size_t>(s.block_size) * D * EB;
  const size_t fixed = static_cast<size_t>(kNW) * G * (D + 2) * sizeof(float) + 16 +
                       static_cast<size_t>(BH + 1) * sizeof(int32_t);
  const size_t per_stage = 2 * tile + 2 * sizeof(uint64_t) + sizeof(int4);
  const size_t budget = static_cast<size_t>(device_max_smem_optin()) - 1024;
  if (fixed + 2 * per_stage > budget) return cudaErrorInvalidValue;
  // About 160 KB of K/V in flight per SM covers the HBM latency-bandwidth product.
  const size_t nst_bw = (160 * 1024) / (2 * tile), nst_fit = (budget - fixed) / per_stage;
  int nst = static_cast<int>(nst_bw < nst_fit ? nst_bw : nst_fit);
  nst = max(2, min(nst, 16));
  const size_t smem = static_cast<size_t>(nst) * per_stage + fixed + 64;

  static std::atomic<uint64_t> smem_done{0};
  cudaError_t e = allow_max_smem(smem_done, reinterpret_cast<const void*>(decode_kernel<KV, D, G, DENSE>));
  if (e != cudaSuccess) return e;

  const DecodeArgs a = make_decode_args(c, nst, s.block_size);  // one position per block
  return launch_pdl(decode_kernel<KV, D, G, DENSE>, static_cast<unsigned>(c.S), kDecThreads, smem, st, a);
}

template <typename KV, int D, bool DENSE>
cudaError_t launch_decode_g(const DecodeCall& c, cudaStream_t st) {
  switch (c.shape.n_q_heads / c.shape.n_kv_heads) {
    case 1: return launch_decode_t<KV, D, 1, DENSE>(c, st);
    case 2: return launch_decode_t<KV, D, 2, DENSE>(c, st);
    case 4: return launch_decode_t<KV, D, 4, DENSE>(c, st);
    case 8: return launch_decode_t<KV, D, 8, DENSE>(c, st);
    default: return cudaErrorInvalidValue;
  }
}

template <typename KV, bool DENSE>
cudaError_t launch_decode_kd(const DecodeCall& c, cudaStream_t st) {
  return c.shape.head_dim == 128 ? launch_decode_g<KV, 128, DENSE>(c, st) : launch_decode_g<KV, 64, DENSE>(c, st);
}

}  // namespace

cudaError_t launch_decode(const DecodeCall& c, cudaStream_t st) {
  if (c.shape.kv_dtype == ETA_FP8_E4M3 || (c.shape.kv_dtype == ETA_BF16 && c.shape.q_dtype == ETA_BF16))
    return launch_decode_mma(c, st);
  if (c.shape.kv_dtype == ETA_BF16)
    return c.dense ? launch_decode_kd<Bf16Raw, true>(c, st) : launch_decode_kd<Bf16Raw, false>(c, st);
  return c.dense ? launch_decode_kd<float, true>(c, st) : launch_decode_kd<float, false>(c, st);
}

}  // namespace eta

// Device-side helpers shared by the ETA kernels: sm_100a PTX wrappers for
// mbarriers and 1-D TMA bulk copies, bf16 widening, bounded waits.
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

#include "eta.h"

namespace eta {

constexpr float kLog2e = 1.4426950408889634f;
constexpr uint32_t kFull = 0xffffffffu;

struct Bf16Raw { uint16_t bits; };
struct Fp8Raw { uint8_t bits; };

template <typename T> struct KvTraits;
template <> struct KvTraits<float> { static constexpr int kBytes = 4; static constexpr int kDtype = ETA_F32; };
template <> struct KvTraits<Bf16Raw> { static constexpr int kBytes = 2; static constexpr int kDtype = ETA_BF16; };
template <> struct KvTraits<Fp8Raw> { static constexpr int kBytes = 1; static constexpr int kDtype = ETA_FP8_E4M3; };

// e4m3 byte -> fp32, exactly: (-1)^s 2^(e-7) (1 + m/8) for e > 0, (-1)^s m 2^-9
// for e = 0; S.1111.111 is NaN.
__device__ __forceinline__ float e4m3_to_float(uint32_t b) {
  const uint32_t e = (b >> 3) & 15u, m = b & 7u;
  float v = e == 0u ? static_cast<float>(m) * 0.001953125f : __uint_as_float(((e + 120u) << 23) | (m << 20));
  if (e == 15u && m == 7u) v = __uint_as_float(0x7fc00000u);
  return (b & 0x80u) ? -v : v;
}

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

// Widen the 16 bytes at `p` (8 bf16 or 4 fp32) into x[].
template <typename T>
__device__ __forceinline__ void widen16(const uint4& w, float* x);
template <>
__device__ __forceinline__ void widen16<Bf16Raw>(const uint4& w, float* x) {
  x[0] = bf16_lo(w.x); x[1] = bf16_hi(w.x); x[2] = bf16_lo(w.y); x[3] = bf16_hi(w.y);
  x[4] = bf16_lo(w.z); x[5] = bf16_hi(w.z); x[6] = bf16_lo(w.w); x[7] = bf16_hi(w.w);
}
template <>
__device__ __forceinline__ void widen16<float>(const uint4& w, float* x) {
  x[0] = __uint_as_float(w.x); x[1] = __uint_as_float(w.y);
  x[2] = __uint_as_float(w.z); x[3] = __uint_as_float(w.w);
}

// One stored element of a q / K buffer in any supported dtype, widened to fp32.
__device__ __forceinline__ float load_elem(const void* p, int dtype, int64_t i) {
  if (dtype == ETA_FP8_E4M3) return e4m3_to_float(static_cast<const uint8_t*>(p)[i]);
  if (dtype == ETA_BF16) {
    uint32_t b = static_cast<uint32_t>(static_cast<const uint16_t*>(p)[i]) << 16;
    return __uint_as_float(b);
  }
  return static_cast<const float*>(p)[i];
}

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// ---------------------------------------------------------------- mbarrier
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}
__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("{\n\t.reg .b64 st;\n\tmbarrier.arrive.shared::cta.b64 st, [%0];\n\t}" ::"r"(smem_u32(bar))
               : "memory");
}
__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("{\n\t.reg .b64 st;\n\tmbarrier.arrive.expect_tx.shared::cta.b64 st, [%0], %1;\n\t}" ::"r"(
                   smem_u32(bar)),
               "r"(bytes)
               : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\tmbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\tselp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

__device__ __forceinline__ uint64_t global_timer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// Wait for the phase of `bar` with the given parity to complete, for at most
// kWaitLimitNs. Returns false on timeout (the CTA-wide abort flag and the
// device status word are set) or when another thread of the CTA has aborted.
constexpr uint64_t kWaitLimitNs = 2000000000ull;  // 2 s

// Bounded wait until the shared int *p equals v (set by another warp of the
// thread block); same limit and abort protocol as mbar_wait_bounded below.
__device__ __forceinline__ bool wait_value_bounded(volatile int* p, int v, volatile int* abort_flag,
                                                   int32_t* status);

__device__ __forceinline__ bool mbar_wait_bounded(uint64_t* bar, uint32_t parity, volatile int* abort_flag,
                                                  int32_t* status) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = global_timer_ns();
  for (uint32_t it = 1;; ++it) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((it & 63u) == 0) {
      if (*abort_flag) return false;
      if (global_timer_ns() - t0 > kWaitLimitNs) {
        *abort_flag = 1;
        atomicExch(status, static_cast<int32_t>(ETA_ERR_DEVICE_TIMEOUT));
        return false;
      }
    }
  }
}

__device__ __forceinline__ bool wait_value_bounded(volatile int* p, int v, volatile int* abort_flag,
                                                   int32_t* status) {
  if (*p == v) return true;
  const uint64_t t0 = global_timer_ns();
  for (uint32_t it = 1;; ++it) {
    if (*p == v) return true;
    __nanosleep(32);  // back off: a polling warp takes no issue slots from the working ones
    if ((it & 15u) == 0) {
      if (*abort_flag) return false;
      if (global_timer_ns() - t0 > kWaitLimitNs) {
        *abort_flag = 1;
        atomicExch(status, static_cast<int32_t>(ETA_ERR_DEVICE_TIMEOUT));
        return false;
      }
    }
  }
}

// ------------------------------------------------------- TMA bulk copies
__device__ __forceinline__ uint64_t l2_policy_evict_first() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
  return p;
}

// 1-D bulk copy global -> shared, completion counted on `bar` in bytes.
// dst, src 16-byte aligned; bytes a multiple of 16.
__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, uint32_t bytes, uint64_t* bar,
                                         uint64_t policy) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint [%0], [%1], %2, [%3], %4;" ::"r"(
          smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar)), "l"(policy)
      : "memory");
}

// Cached tokens of batch row b: seq_lens[b] when the call passes per-row
// lengths (device memory), else the call's uniform count n_max. A length
// outside [1, n_max] is recorded as ETA_ERR_INVALID_ARG in the status word and
// clamped, so every kernel of the call sees the same value.
__device__ __forceinline__ int64_t seq_len_of(const int32_t* seq_lens, int b, int64_t n_max, int32_t* status) {
  if (seq_lens == nullptr) return n_max;
  int64_t v = __ldg(seq_lens + b);
  if (v < 1 || v > n_max) {
    atomicExch(status, static_cast<int32_t>(ETA_ERR_INVALID_ARG));
    v = v < 1 ? 1 : n_max;
  }
  return v;
}

// Where the keys (or values) of a logical block live. Contiguous caches are
// [B][Hkv][capacity][d]; paged pools are [num_pages][Hkv][bs][d], row b's
// logical block j in page block_table[b * max_blocks + j].
struct KvLayout {
  const int32_t* block_table;  // null: contiguous
  int max_blocks, num_pages, Hkv, bs;
  int64_t cap;
};

// Row, in a [rows][d] view of the store, of token 0 of logical block blk of
// segment seg = b * Hkv + kvh; -1 when the page index is outside the pool.
// (The host keeps every row index of a store below 2^31.)
__device__ __forceinline__ int kv_block_row(const KvLayout& L, int seg, int blk) {
  if (L.block_table == nullptr) return static_cast<int>(static_cast<int64_t>(seg) * L.cap + static_cast<int64_t>(blk) * L.bs);
  const int b = seg / L.Hkv, kvh = seg - b * L.Hkv;
  const int page = __ldg(L.block_table + static_cast<int64_t>(b) * L.max_blocks + blk);
  if (page < 0 || page >= L.num_pages) return -1;
  return (page * L.Hkv + kvh) * L.bs;
}

// Programmatic dependent launch. The screening and decode kernels are launched
// with cudaLaunchAttributeProgrammaticStreamSerialization, so each may start
// (launch, shared-memory and barrier set-up) while the kernel before it on the
// stream is still running. grid_dependency_wait() blocks until that kernel has
// completed and its writes are visible (immediately when there is none): call
// it before the first global read. allow_dependent_launch() lets the next
// kernel on the stream begin launching.
__device__ __forceinline__ void grid_dependency_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void allow_dependent_launch() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

__device__ __forceinline__ void named_barrier_sync(int id, int nthreads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

}  // namespace eta

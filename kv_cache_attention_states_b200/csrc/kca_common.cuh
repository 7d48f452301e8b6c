// kca_common.cuh -- device helpers shared by the kernels of libkca.so.
//
// Bounded waits: every mbarrier wait in this library gives up after
// KCA_WAIT_LIMIT_NS of wall time (read from %globaltimer), records the site in
// the workspace status word and returns false, so a logic error can never hang
// the GPU; callers then drain what they issued and return.
#pragma once
#include <cstdint>
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "../../include/kca.h"

#ifndef KCA_WAIT_LIMIT_NS
#define KCA_WAIT_LIMIT_NS 2000000000ull  // 2 s: three orders above any legal wait
#endif

namespace kca {

// Status word layout (first 256 bytes of the workspace).
struct DeviceStatus {
  unsigned int error;   // bit 0: a bounded wait ran out; bit 1: a device ctx_len out of range;
                        // bit 2: a device destination row out of range (append)
  unsigned int detail;  // (site << 24) | (block & 0xffffff) of the first failure
};
enum : unsigned int { kErrWaitTimeout = 1u, kErrBadCtx = 2u, kErrBadRow = 4u, kErrBounds = 8u };
enum : unsigned int {
  kSiteRowsFull = 1, kSiteRowsEmpty = 2, kSiteTcFull = 3, kSiteTcEmpty = 4, kSiteTcS = 5,
  kSiteTcP = 6, kSiteTcO = 7, kSiteTcQ = 8, kSiteTcDrain = 9, kSiteCtx = 10,
  kSiteAppend = 11, kSiteTcAlign = 12, kSiteBoundsRows = 13, kSiteBoundsDecode = 14,
  kSiteBoundsMulti = 15, kSiteBoundsMerge = 16
};

// Records the first failure (detail: site and the block's x index, or the
// sequence for kSiteCtx) and ORs `bit` into the error word.
__device__ __forceinline__ void record_error(DeviceStatus* st, unsigned int site,
                                             unsigned int bit = kErrWaitTimeout,
                                             unsigned int where = 0xffffffffu) {
  if (st == nullptr) return;
  const unsigned int prev = atomicOr(&st->error, bit);
  if (prev == 0) st->detail = (site << 24) | ((where == 0xffffffffu ? blockIdx.x : where) & 0xffffffu);
}

// Bounds-checked builds (-DKCA_BOUNDS_CHECK, the library's stand-in for a
// memory sanitizer): KCA_IN_BOUNDS(cond, status, site, where) records a
// failed index check in the status word (error bit 8) and yields false, so
// the caller skips the access instead of faulting; in normal builds it is
// the constant true and costs nothing.
#ifdef KCA_BOUNDS_CHECK
#define KCA_IN_BOUNDS(cond, st, site, where) ::kca::in_bounds((cond), (st), (site), (where))
#else
#define KCA_IN_BOUNDS(cond, st, site, where) true
#endif

__device__ __forceinline__ uint64_t global_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ bool in_bounds(bool ok, DeviceStatus* st, unsigned int site, unsigned int where) {
  if (!ok) record_error(st, site, kErrBounds, where);
  return ok;
}

// ---------------------------------------------------------------- mbarrier
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count)
               : "memory");
}
__device__ __forceinline__ void fence_barrier_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("{ .reg .b64 st; mbarrier.arrive.shared::cta.b64 st, [%0]; }" ::"r"(smem_u32(bar))
               : "memory");
}
__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("{ .reg .b64 st; mbarrier.arrive.expect_tx.shared::cta.b64 st, [%0], %1; }" ::"r"(
                   smem_u32(bar)),
               "r"(bytes)
               : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{ .reg .pred p; mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2; selp.u32 %0, 1, 0, p; }"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}
// Non-blocking test of the phase with the given parity.
__device__ __forceinline__ bool mbar_test_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{ .reg .pred p; mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2; selp.u32 %0, 1, 0, p; }"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}
// Waits for the phase with the given parity to complete.  Returns false when
// *abort became non-zero or the time limit passed (the latter is recorded).
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, volatile int* abort,
                                          DeviceStatus* st, unsigned int site) {
  // Non-blocking probe first: most waits on the hot path find the phase done.
  if (mbar_test_wait(bar, parity)) return true;
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = global_ns();
  for (uint32_t it = 1;; ++it) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((it & 63u) == 0) {
      if (abort != nullptr && *abort) return false;
      if (global_ns() - t0 > KCA_WAIT_LIMIT_NS) {
        record_error(st, site);
        if (abort != nullptr) *abort = 1;
        return false;
      }
    }
  }
}

// One-dimensional bulk copy global -> shared, completing on an mbarrier.
// Both addresses 16-byte aligned, bytes a multiple of 16.
__device__ __forceinline__ void bulk_g2s(void* smem_dst, const void* gmem_src, uint32_t bytes,
                                         uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_u32(smem_dst)),
      "l"(gmem_src), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

// ------------------------------------------------------------- arithmetic
// Maximum that returns NaN when either operand is NaN.
__device__ __forceinline__ float max_nan(float a, float b) {
  float r;
  asm("max.NaN.f32 %0, %1, %2;" : "=f"(r) : "f"(a), "f"(b));
  return r;
}

__device__ __forceinline__ float2 ffma2(float2 a, float2 b, float2 c) { return __ffma2_rn(a, b, c); }

// Eight consecutive elements of a row as f32, from a 16-byte aligned address.
template <int DT>
__device__ __forceinline__ void load8(const void* p, float (&x)[8]);

template <>
__device__ __forceinline__ void load8<KCA_F32>(const void* p, float (&x)[8]) {
  const float4 a = reinterpret_cast<const float4*>(p)[0];
  const float4 b = reinterpret_cast<const float4*>(p)[1];
  x[0] = a.x; x[1] = a.y; x[2] = a.z; x[3] = a.w;
  x[4] = b.x; x[5] = b.y; x[6] = b.z; x[7] = b.w;
}
template <>
__device__ __forceinline__ void load8<KCA_F16>(const void* p, float (&x)[8]) {
  const uint4 u = *reinterpret_cast<const uint4*>(p);
  const __half2* h = reinterpret_cast<const __half2*>(&u);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 f = __half22float2(h[i]);
    x[2 * i] = f.x;
    x[2 * i + 1] = f.y;
  }
}
template <>
__device__ __forceinline__ void load8<KCA_BF16>(const void* p, float (&x)[8]) {
  const uint4 u = *reinterpret_cast<const uint4*>(p);
  const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 f = __bfloat1622float2(h[i]);
    x[2 * i] = f.x;
    x[2 * i + 1] = f.y;
  }
}

template <int DT>
struct ElemBytes { static constexpr int value = (DT == KCA_F32) ? 4 : 2; };

}  // namespace kca

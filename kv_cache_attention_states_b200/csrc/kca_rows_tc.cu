// kca_rows_tc.cu -- batched short chunks (attn_prefill_batch) on the sm_100a
// tensor cores: tcgen05 MMAs issued by one thread, accumulators in tensor
// memory.
//
// The pages' geometry (Karume v0.12.0 release notes, "Performance", item 3,
// and "Docs", ADR 0067): plans of 2-15 query rows sit between single-row
// decode and the row tiles of prefill.  A unit is up to four consecutive
// query rows of one sequence (the same units, splits, partials and merge
// kernel as the mma.sync multi-row kernel in kca_decode_mma.cu), so each
// K / V stage crosses from L2 once for all of them.  The mma.sync form of
// this kernel is bound by instruction issue (two warps per SM sub-partition
// run the QK^T and PV fragments, the softmax and the shared-memory traffic
// of every stage); here one thread issues every MMA and one warp runs the
// softmax, so the tensor pipe and the load stream overlap.
//
// Rows: M row m = 8 i + h (i the unit's row, h the head), 32 of the MMAs'
// 128 M rows; rows 32-127 of every operand and accumulator are never read.
// f32 queries keep f32-grade products: q = q_hi + q_lo (16-bit parts of the
// cache's type) and S = q_hi K^T + q_lo K^T accumulate into the same
// tensor-memory columns; P = p_hi + p_lo the same way in O += P V.
//
// Warp roles (4 warps):
//   warp 0   softmax of TMEM lanes 0-31 (the unit's rows), then the epilogue
//   warp 1   TMEM allocator; lane 0 issues every MMA; the warp zeroes the V
//            rows of a ragged last stage
//   warp 2   TMA producer of K stages (64 keys x 256 dims, ring of 3)
//   warp 3   TMA producer of V stages (ring of 2)
// Shared memory: Q high and low parts (32 rows x 256 dims each, four
// 64-dim chunks of 4 KiB with 128-byte swizzle) and 16 KiB of zeros that
// rows 32-127 of the last chunks' descriptors read; the K and V rings.
// Tensor memory (512 columns): S of stage j at [64 (j & 1), +64), P of stage
// j at [128 + 64 (j & 1), +64) (high parts, then low parts, as 16-bit
// pairs), O at [256, 512).
// Per stage j the MMA thread issues Q K^T of stage j, then P V of stage
// j - 1 once the softmax has written its P, so the softmax of a stage runs
// under the MMAs of its neighbours.  The softmax keeps a reference max per
// row and rescales O only when a score passes it by more than 2^8 (the
// prefill kernel's rule), with every PV before it complete.
#include <atomic>
#include <cuda.h>
#include <cuda_runtime.h>

#include "kca_common.cuh"
#include "kca_plan.h"
#include "kca_rows.h"
#include "kca_tc_ptx.cuh"

namespace kca {
namespace {

constexpr int kRThreads = 128;
constexpr int kRKeys = 64;                           // keys per stage
constexpr int kRBox = 64 * 64 * 2;                   // 64 rows x 64 dims (16-bit): 8 KiB
constexpr int kRSlot = 4 * kRBox;                    // K or V of one stage: 32 KiB
constexpr int kRKRing = 3, kRVRing = 2;
constexpr int kRQRows = 8 * kMultiRows;              // 32 M rows
constexpr int kRQChunk = kRQRows * 128;              // 32 rows x 64 dims: 4 KiB
constexpr int kRQBytes = 4 * kRQChunk;               // one part (high or low): 16 KiB
constexpr int kROffQHi = 0;
constexpr int kROffQLo = kRQBytes;
constexpr int kROffPad = 2 * kRQBytes;               // zeros: rows 32-127 of the last chunks
constexpr int kRPadBytes = 16 * 1024;
constexpr int kROffK = kROffPad + kRPadBytes;        // 48 KiB
constexpr int kROffV = kROffK + kRKRing * kRSlot;    // 144 KiB
constexpr int kROffBar = kROffV + kRVRing * kRSlot;  // 208 KiB
constexpr int kRBarBytes = 1024;
constexpr int kRSmemBytes = kROffBar + kRBarBytes + 1024;   // + alignment slack
static_assert(kRSmemBytes <= 232448, "shared memory over the per-CTA limit");
// A descriptor of 128 M rows starting at chunk 3 of the low part reads up
// to 12 KiB past the part: inside the zero pad.
static_assert(kROffQLo + 3 * kRQChunk + 16 * 1024 <= kROffK, "Q descriptors stay in the Q area");
constexpr uint32_t kRColS = 0, kRColP = 128, kRColO = 256, kRTmemCols = 512;
constexpr float kRRescaleLog2 = 8.f;   // rescale O once a score passes the reference by 2^8

struct RBars {
  uint64_t kfull[kRKRing], kempty[kRKRing];
  uint64_t vfull[kRVRing], vempty[kRVRing];
  uint64_t s_full[2];   // Q K^T of stage j complete in S buffer j & 1 (MMA commit)
  uint64_t p_full[2];   // P of stage j written and O corrected (softmax warp)
  uint64_t o_done[2];   // P V of stage j complete (MMA commit)
  uint64_t drain;       // every MMA complete (single use)
  uint32_t tmem_base;
  int abort;
};
static_assert(sizeof(RBars) <= kRBarBytes, "barrier block too large");

template <int KT>
__device__ __forceinline__ uint32_t pk2(float lo, float hi) {
  if (KT == KCA_BF16) {
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&v);
  }
  __half2 v = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}
template <int KT>
__device__ __forceinline__ float2 upk2(uint32_t u) {
  if (KT == KCA_BF16) return __bfloat1622float2(*reinterpret_cast<__nv_bfloat162*>(&u));
  return __half22float2(*reinterpret_cast<__half2*>(&u));
}

__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

template <int QT, int KT>
__global__ void __launch_bounds__(kRThreads, 1)
    rows_tc_kernel(const __grid_constant__ CUtensorMap tmk, const __grid_constant__ CUtensorMap tmv,
                   const RowsArgs a) {
  constexpr bool kLo = QT != KT;   // a query of the cache's own type has no low part
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  const uint32_t raw_addr = smem_u32(smem_raw);
  const uint32_t pad = ((raw_addr + 1023u) & ~1023u) - raw_addr;
  unsigned char* smem = smem_raw + pad;
  const uint32_t sbase = raw_addr + pad;
  RBars* bars = reinterpret_cast<RBars*>(smem + kROffBar);
  volatile int* abort_flag = &bars->abort;
  DeviceStatus* status = reinterpret_cast<DeviceStatus*>(a.status);

  const int unit = blockIdx.y;
  const int split = blockIdx.x;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  int b, i0, nr;
  multirow_unit(a, unit, &b, &i0, &nr);
  const int64_t pos0 = a.ctx[b] - a.rows_per_seq + i0;   // first row's position
  const int64_t lo_u = lo_of(pos0, a.window);
  const int64_t hi_u = pos0 + nr - 1;
  const int32_t nsplit = rows_n_splits(hi_u - lo_u + 1, a.split_len);
  if (split >= nsplit) return;
  const int64_t kbeg = lo_u + (int64_t)split * a.split_len;
  int64_t kend = kbeg + a.split_len;
  if (kend > hi_u + 1) kend = hi_u + 1;
  const int64_t base_row = (int64_t)b * a.seq_rows;
  const int n = (int)cdiv(kend - kbeg, kRKeys);
  // bounds-checked builds: the split's rows in the cache, its rows' partial
  // slots in the workspace (no CTA of this kernel waits on another)
  if (!KCA_IN_BOUNDS(nsplit <= a.max_splits && base_row + kbeg >= 0 && base_row + kend <= a.cache_rows &&
                         (nsplit == 1 || ((int64_t)b * a.rows_per_seq + i0 + nr) * a.max_splits <= a.part_slots),
                     status, kSiteBoundsMulti, (unsigned)unit))
    return;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kRKRing; ++s) {
      mbar_init(&bars->kfull[s], 1);
      mbar_init(&bars->kempty[s], 1);
    }
    for (int s = 0; s < kRVRing; ++s) {
      mbar_init(&bars->vfull[s], 1);
      mbar_init(&bars->vempty[s], 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&bars->s_full[s], 1);
      mbar_init(&bars->p_full[s], 1);
      mbar_init(&bars->o_done[s], 1);
    }
    mbar_init(&bars->drain, 1);
    bars->abort = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    ptx::tmem_alloc(smem_u32(&bars->tmem_base), kRTmemCols);
    ptx::tmem_relinquish();
  }
  if (threadIdx.x == 64) ptx::prefetch_tmap(&tmk);
  if (threadIdx.x == 96) ptx::prefetch_tmap(&tmv);
  ptx::fence_before_sync();
  __syncthreads();
  ptx::fence_after_sync();
  const uint32_t tmem = bars->tmem_base;
  // Programmatic dependent launch: the set-up above overlaps the previous
  // kernel of the stream; global memory is touched only after this wait.
  asm volatile("griddepcontrol.wait;" ::: "memory");

  // Stage the queries: M row m = 8 i + h, 16-byte group u of its 256 dims
  // (chunk u / 8, 128-byte swizzle within the chunk); high and low parts.
  for (int it = threadIdx.x; it < kRQRows * 32; it += kRThreads) {
    const int m = it >> 5, u = it & 31;
    const int i = m >> 3, h = m & 7;
    float x[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    if (i < nr) {
      const int64_t orow = (int64_t)b * a.rows_per_seq + i0 + i;
      load8<QT>(static_cast<const char*>(a.q) + ((orow * kHeads + h) * kDim + 8 * u) * ElemBytes<QT>::value, x);
    }
    uint32_t hi[4], lo[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      hi[j] = pk2<KT>(x[2 * j], x[2 * j + 1]);
      const float2 f = upk2<KT>(hi[j]);
      lo[j] = pk2<KT>(x[2 * j] - f.x, x[2 * j + 1] - f.y);
    }
    const int off = (u >> 3) * kRQChunk + m * 128 + (((u & 7) ^ (m & 7)) << 4);
    *reinterpret_cast<uint4*>(smem + kROffQHi + off) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
    *reinterpret_cast<uint4*>(smem + kROffQLo + off) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
  }
  for (int it = threadIdx.x; it < kRPadBytes / 16; it += kRThreads)
    *reinterpret_cast<uint4*>(smem + kROffPad + 16 * it) = make_uint4(0, 0, 0, 0);
  fence_proxy_async_smem();   // generic stores -> visible to the tensor core
  __syncthreads();

  if (warp >= 2) {
    // ------------------------------------------------------------ producers
    if (lane == 0) {
      const bool is_k = warp == 2;
      const int ring = is_k ? kRKRing : kRVRing;
      uint64_t* full = is_k ? bars->kfull : bars->vfull;
      uint64_t* empty = is_k ? bars->kempty : bars->vempty;
      const uint32_t dst0 = sbase + (is_k ? kROffK : kROffV);
      const void* map = is_k ? static_cast<const void*>(&tmk) : static_cast<const void*>(&tmv);
      int issued = 0;
      for (int j = 0; j < n; ++j) {
        const int s = j % ring;
        if (j >= ring && !mbar_wait(&empty[s], ((j / ring) - 1) & 1, abort_flag, status, kSiteTcEmpty)) break;
        mbar_arrive_expect_tx(&full[s], kRSlot);
        const int32_t row0 = (int32_t)(base_row + kbeg + (int64_t)j * kRKeys);
#pragma unroll
        for (int c = 0; c < 4; ++c)
          ptx::tma_load_2d(dst0 + s * kRSlot + c * kRBox, map, 64 * c, row0, smem_u32(&full[s]));
        issued = j + 1;
      }
      if (issued < n) {   // aborted: let every issued copy land before the CTA leaves
        *abort_flag = 1;
        for (int s = 0; s < ring && s < issued; ++s) {
          const int last = ((issued - 1 - s) / ring) * ring + s;
          mbar_wait(&full[s], (last / ring) & 1, nullptr, status, kSiteTcFull);
        }
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ----------------------------------------------------------------- MMA
    constexpr uint32_t ab = KT == KCA_BF16 ? 1u : 0u;
    constexpr uint32_t id_qk = ptx::idesc_f16(ab, 128, kRKeys, 0);
    constexpr uint32_t id_pv = ptx::idesc_f16(ab, 128, kDim, 1);
    // Descriptor bases; an operand at byte offset x from a base is the base
    // plus x >> 4 in the start-address field (addresses stay below 256 KiB).
    const uint64_t qh0 = ptx::sdesc_sw128(sbase + kROffQHi, 16, 1024);
    const uint64_t ql0 = ptx::sdesc_sw128(sbase + kROffQLo, 16, 1024);
    const uint64_t kd0 = ptx::sdesc_sw128(sbase + kROffK, 16, 1024);
    const uint64_t vd0 = ptx::sdesc_sw128(sbase + kROffV, kRBox, 1024);
    // P V of stage u: after its P is written; V rows past the split's end
    // are zeroed first (P is 0 there, but the rows may hold anything).
    auto pv = [&](int u) -> bool {
      if (!__all_sync(0xffffffffu, mbar_wait(&bars->p_full[u & 1], (u >> 1) & 1, abort_flag, status, kSiteTcP)))
        return false;
      const int s = u % kRVRing;
      if (!__all_sync(0xffffffffu, mbar_wait(&bars->vfull[s], (u / kRVRing) & 1, abort_flag, status, kSiteTcFull)))
        return false;
      const int64_t k0 = kbeg + (int64_t)u * kRKeys;
      const int cnt = (int)((kend - k0) < kRKeys ? (kend - k0) : kRKeys);
      if (cnt < kRKeys) {
        unsigned char* vs = smem + kROffV + s * kRSlot;
        for (int idx = lane; idx < (kRKeys - cnt) * 32; idx += 32) {
          const int row = cnt + (idx >> 5), g = idx & 31;   // g: box g / 8, 16-byte unit g % 8
          *reinterpret_cast<uint4*>(vs + (g >> 3) * kRBox + row * 128 + (g & 7) * 16) = make_uint4(0, 0, 0, 0);
        }
        fence_proxy_async_smem();
        __syncwarp();
      }
      ptx::fence_after_sync();
      if (lane == 0) {
        const uint32_t pcol = tmem + kRColP + 64 * (u & 1);
        const uint64_t vd = vd0 + (uint64_t)((s * kRSlot) >> 4);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)   // 16 keys per step: 8 TMEM columns of P, V rows 16 kk
          ptx::mma_ts(tmem + kRColO, pcol + 8 * kk, vd + (uint64_t)((kk * 16 * 128) >> 4), id_pv,
                      (u > 0 || kk > 0) ? 1u : 0u);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)   // the low parts of P
          ptx::mma_ts(tmem + kRColO, pcol + 32 + 8 * kk, vd + (uint64_t)((kk * 16 * 128) >> 4), id_pv, 1u);
        ptx::mma_commit(smem_u32(&bars->vempty[s]));
        ptx::mma_commit(smem_u32(&bars->o_done[u & 1]));
      }
      __syncwarp();
      return true;
    };
    bool ok = true;
    for (int j = 0; j < n && ok; ++j) {
      const int s = j % kRKRing;
      ok = __all_sync(0xffffffffu, mbar_wait(&bars->kfull[s], (j / kRKRing) & 1, abort_flag, status, kSiteTcFull));
      if (!ok) break;
      // S buffer j & 1 was read by the softmax of stage j - 2, whose P the
      // P V of stage j - 2 (issued above) waited for.
      ptx::fence_after_sync();
      if (lane == 0) {
        const uint32_t scol = tmem + kRColS + 64 * (j & 1);
        const uint64_t kd = kd0 + (uint64_t)((s * kRSlot) >> 4);
#pragma unroll
        for (int k = 0; k < 16; ++k) {   // 16 dims per step: chunk k / 4, 32-byte column group k % 4
          const uint32_t qo = (k >> 2) * kRQChunk + (k & 3) * 32, ko = (k >> 2) * kRBox + (k & 3) * 32;
          ptx::mma_ss(scol, qh0 + (uint64_t)(qo >> 4), kd + (uint64_t)(ko >> 4), id_qk, k > 0 ? 1u : 0u);
        }
        if (kLo) {
#pragma unroll
          for (int k = 0; k < 16; ++k) {
            const uint32_t qo = (k >> 2) * kRQChunk + (k & 3) * 32, ko = (k >> 2) * kRBox + (k & 3) * 32;
            ptx::mma_ss(scol, ql0 + (uint64_t)(qo >> 4), kd + (uint64_t)(ko >> 4), id_qk, 1u);
          }
        }
        ptx::mma_commit(smem_u32(&bars->kempty[s]));
        ptx::mma_commit(smem_u32(&bars->s_full[j & 1]));
      }
      __syncwarp();
      if (j > 0) ok = pv(j - 1);
    }
    if (ok) pv(n - 1);
    // every MMA issued above has completed once this barrier flips
    if (lane == 0) ptx::mma_commit(smem_u32(&bars->drain));
    __syncwarp();
    mbar_wait(&bars->drain, 0, nullptr, status, kSiteTcDrain);
  } else {
    // ------------------------------------------------------------- softmax
    const int m = lane;                              // TMEM lane == M row
    const int i = m >> 3, h = m & 7;
    const bool valid = i < nr;
    const int64_t pos = pos0 + i;
    const int64_t lo = lo_of(pos, a.window);
    const float cs = a.scale * 1.4426950408889634f;  // scores in log2 units
    float m_ref = -INFINITY;                         // reference max of the row, log2 units
    float l_sum = 0.f;
    bool ok = true;
    for (int j = 0; j < n; ++j) {
      ok = __all_sync(0xffffffffu, ok && mbar_wait(&bars->s_full[j & 1], (j >> 1) & 1, abort_flag, status, kSiteTcS));
      if (!ok) break;
      ptx::fence_after_sync();
      uint32_t r0[32], r1[32];
      ptx::tmem_ld32(tmem + kRColS + 64 * (j & 1), r0);
      ptx::tmem_ld32(tmem + kRColS + 64 * (j & 1) + 32, r1);
      ptx::tmem_wait_ld();
      float s[64];
#pragma unroll
      for (int c = 0; c < 32; ++c) {
        s[c] = __uint_as_float(r0[c]);
        s[32 + c] = __uint_as_float(r1[c]);
      }
      // keys outside [lo, pos], past the split's end, or of a row the unit
      // does not have become -inf (scale > 0 keeps them there)
      const int64_t k0 = kbeg + (int64_t)j * kRKeys;
      const int cnt = (int)((kend - k0) < kRKeys ? (kend - k0) : kRKeys);
      if (!(valid && cnt == kRKeys && k0 >= lo && k0 + kRKeys - 1 <= pos)) {
#pragma unroll
        for (int c = 0; c < 64; ++c) {
          const int64_t key = k0 + c;
          if (!valid || c >= cnt || key < lo || key > pos) s[c] = -INFINITY;
        }
      }
      float m8[8];
#pragma unroll
      for (int c = 0; c < 8; ++c) m8[c] = s[c];
#pragma unroll
      for (int c = 8; c < 64; ++c) m8[c & 7] = max_nan(m8[c & 7], s[c]);
#pragma unroll
      for (int c = 0; c < 4; ++c) m8[c] = max_nan(m8[c], m8[c + 4]);
      const float mloc = max_nan(max_nan(m8[0], m8[2]), max_nan(m8[1], m8[3]));
      const float mx = mloc == -INFINITY ? -INFINITY : mloc * cs;
      const bool need = mx > m_ref + kRRescaleLog2;
      if (__any_sync(0xffffffffu, need)) {
        const float alpha = need ? ptx::ex2(m_ref - mx) : 1.f;
        if (need) m_ref = mx;
        l_sum *= alpha;
        if (j > 0) {
          // P V of stage j - 1 must finish before O is rescaled (that of
          // stage j - 2 preceded this stage's Q K^T, so it has)
          ok = __all_sync(0xffffffffu, mbar_wait(&bars->o_done[(j - 1) & 1], ((j - 1) >> 1) & 1, abort_flag,
                                                 status, kSiteTcO));
          if (!ok) break;
          ptx::fence_after_sync();
#pragma unroll 1
          for (int c = 0; c < 8; ++c) {
            uint32_t r[32];
            ptx::tmem_ld32(tmem + kRColO + 32 * c, r);
            ptx::tmem_wait_ld();
#pragma unroll
            for (int e = 0; e < 32; ++e) r[e] = __float_as_uint(__uint_as_float(r[e]) * alpha);
            ptx::tmem_st32(tmem + kRColO + 32 * c, r);
          }
          ptx::tmem_wait_st();
        }
      }
      // p = 2^(s cs - m_ref), split into 16-bit high and low parts
      const float nmu = m_ref == -INFINITY ? 0.f : -m_ref;
      uint32_t ph[32], pl[32];
      float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int c = 0; c < 32; ++c) {
        const float p0 = ptx::ex2(fmaf(s[2 * c], cs, nmu));
        const float p1 = ptx::ex2(fmaf(s[2 * c + 1], cs, nmu));
        acc[c & 3] += p0 + p1;
        ph[c] = pk2<KT>(p0, p1);
        const float2 f = upk2<KT>(ph[c]);
        pl[c] = pk2<KT>(p0 - f.x, p1 - f.y);
      }
      l_sum += (acc[0] + acc[1]) + (acc[2] + acc[3]);
      // P buffer j & 1 was last read by P V of stage j - 2, complete before
      // this stage's Q K^T (whose completion s_full signalled).
      ptx::tmem_st32(tmem + kRColP + 64 * (j & 1), ph);
      ptx::tmem_st32(tmem + kRColP + 64 * (j & 1) + 32, pl);
      ptx::tmem_wait_st();
      ptx::fence_before_sync();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->p_full[j & 1]);
    }
    if (ok)
      ok = __all_sync(0xffffffffu, mbar_wait(&bars->o_done[(n - 1) & 1], ((n - 1) >> 1) & 1, abort_flag, status,
                                             kSiteTcO));
    const bool aborted = !ok || *abort_flag;
    // Epilogue: row m's 256 dims, scaled by 1 / l (one split) or raw with
    // (m, l) in natural units (a split partial for multirow_merge_kernel).
    // An aborted split poisons its rows; the status word says why.
    const float M = aborted ? NAN : m_ref * 0.6931471805599453f;
    const float L = aborted ? NAN : l_sum;
    const int64_t orow = (int64_t)b * a.rows_per_seq + i0 + i;
    float* dst = nullptr;
    float f = 1.f;
    if (valid) {
      if (nsplit == 1) {
        dst = a.out + (orow * kHeads + h) * kDim;
        f = (m_ref == -INFINITY && L == 0.f) ? 0.f : 1.f / L;
      } else {
        const int64_t slot = (orow * a.max_splits + split) * kHeads + h;
        dst = a.part_acc + slot * kDim;
        *reinterpret_cast<float2*>(a.part_ml + slot * 2) = make_float2(M, L);
      }
    }
    if (!aborted) ptx::fence_after_sync();
#pragma unroll 1
    for (int c = 0; c < 8; ++c) {
      uint32_t r[32];
      if (!aborted) {
        ptx::tmem_ld32(tmem + kRColO + 32 * c, r);
        ptx::tmem_wait_ld();
      }
      if (valid) {
#pragma unroll
        for (int e = 0; e < 8; ++e)
          *reinterpret_cast<float4*>(dst + 32 * c + 4 * e) =
              aborted ? make_float4(NAN, NAN, NAN, NAN)
                      : make_float4(__uint_as_float(r[4 * e]) * f, __uint_as_float(r[4 * e + 1]) * f,
                                    __uint_as_float(r[4 * e + 2]) * f, __uint_as_float(r[4 * e + 3]) * f);
      }
    }
  }
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  // No warp leaves while MMAs may still read shared memory or write TMEM.
  ptx::fence_before_sync();
  __syncthreads();
  if (warp == 1) {
    ptx::fence_after_sync();
    ptx::tmem_dealloc(tmem, kRTmemCols);
  }
}

template <int QT, int KT>
cudaError_t launch_t(const CUtensorMap& tmk, const CUtensorMap& tmv, const RowsArgs& a, cudaStream_t stream) {
  auto kern = rows_tc_kernel<QT, KT>;
  static std::atomic<bool> attr_set[64];   // per device; zero-initialised
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  if (!attr_set[dev]) {
    const cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kRSmemBytes);
    if (e != cudaSuccess) return e;
    attr_set[dev] = true;
  }
  cudaLaunchAttribute at;
  at.id = cudaLaunchAttributeProgrammaticStreamSerialization;
  at.val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(a.max_splits, a.n_units, 1);
  cfg.blockDim = dim3(kRThreads, 1, 1);
  cfg.dynamicSmemBytes = kRSmemBytes;
  cfg.stream = stream;
  cfg.attrs = &at;
  cfg.numAttrs = 1;
  const cudaError_t e = cudaLaunchKernelEx(&cfg, kern, tmk, tmv, a);
  if (e != cudaSuccess || a.max_splits <= 1) return e;
  return launch_multirow_merge(a, stream);
}

}  // namespace

cudaError_t launch_rows_tc(int q_dtype, int kv_dtype, const CUtensorMap& tmk, const CUtensorMap& tmv,
                           const RowsArgs& a, cudaStream_t stream) {
#define KCA_RTC_CASE(QD, KD) \
  if (q_dtype == QD && kv_dtype == KD) return launch_t<QD, KD>(tmk, tmv, a, stream);
  KCA_RTC_CASE(KCA_F32, KCA_F16)
  KCA_RTC_CASE(KCA_F32, KCA_BF16)
  KCA_RTC_CASE(KCA_F16, KCA_F16)
  KCA_RTC_CASE(KCA_F16, KCA_BF16)
  KCA_RTC_CASE(KCA_BF16, KCA_F16)
  KCA_RTC_CASE(KCA_BF16, KCA_BF16)
#undef KCA_RTC_CASE
  return cudaErrorInvalidValue;
}

}  // namespace kca

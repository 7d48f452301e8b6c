// kca_prefill_tc.cu -- chunked causal prefill on the sm_100a tensor cores.
//
// The pages' design (Karume v0.12.0 release notes, "Performance", item 1):
// for plans of 16 or more chunk rows, QK and PV run on a GEMM tile skeleton
// so that each K / V row is read once per row tile instead of once per query
// row.  Here one CTA takes one work item -- a row tile of 16 positions x 8
// heads (M = 128, the heads share their single KV head) and a run of 64-key
// tiles -- and fuses the three stages the pages keep apart (QK, softmax
// statistics, PV) so no score matrix ever reaches memory:
//
//   warp 0      TMA producer: K and V tiles (64 keys x 256 dims, four
//               64 x 64 boxes with 128-byte swizzle) into a 6-slot ring
//   warp 1      TMEM allocator and the single MMA-issuing thread
//   warps 4-7   softmax warpgroup: thread m owns TMEM lane m (= M row m)
//
// Tensor memory (512 columns x 128 lanes of 32 bits):
//   [  0,128)  Q tile, bf16/f16 pairs: the A operand of S = Q K^T
//   [128,192)  S0 (f32, 64 keys);  P0 (16-bit pairs) over its first 32 columns
//   [192,256)  S1;                 P1 likewise
//   [256,512)  O accumulator, 256 f32 columns
// S is double-buffered so QK^T of tile t+1 runs on the tensor cores while the
// softmax warpgroup works on tile t.  The softmax keeps a reference max per
// row and rescales O (in TMEM) only when a score exceeds it by more than
// 2^8, so probabilities stay <= 256 and the O round trip is rare.  The
// result is exact up to rounding whatever reference max is used.
//
// Work items of a split row tile write (m, l, O) partials that
// merge_tc_kernel combines by log-sum-exp (kca_merge.cuh).
#include <cuda.h>
#include <cuda_runtime.h>

#include "kca_common.cuh"
#include "kca_merge.cuh"
#include "kca_plan.h"
#include "kca_tc.h"
#include "kca_tc_ptx.cuh"

namespace kca {
namespace {

constexpr int kThreads = 256;
constexpr int kRing = 6;
constexpr int kBoxBytes = kKeyTile * 64 * 2;         // 64 keys x 64 dims x 2 B = 8 KiB
constexpr int kSlotBytes = 4 * kBoxBytes;            // one K or V tile: 32 KiB
constexpr int kRingBytes = kRing * kSlotBytes;
constexpr int kBarBytes = 512;
constexpr int kSmemBytes = kRingBytes + kBarBytes + 1024;  // + alignment slack
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColQ = 0, kColS0 = 128, kColS1 = 192, kColO = 256;
constexpr float kRescaleLog2 = 8.f;   // rescale O once a score passes the reference by 2^8

struct Bars {
  uint64_t full[kRing];
  uint64_t empty[kRing];
  uint64_t q_full;
  uint64_t s_full[2];
  uint64_t p_full[2];
  uint64_t o_done;
  uint64_t drain;
  uint32_t tmem_base;
  int abort;
};
static_assert(sizeof(Bars) <= kBarBytes, "barrier block too large");

__device__ __forceinline__ uint32_t pack2(float lo, float hi, int dt) {
  if (dt == KCA_BF16) {
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&v);
  }
  __half2 v = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

template <int DT>
__global__ void __launch_bounds__(kThreads, 1)
    prefill_tc_kernel(const __grid_constant__ CUtensorMap tmk, const __grid_constant__ CUtensorMap tmv,
                      const TcArgs a) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  const uint32_t raw_addr = smem_u32(smem_raw);
  const uint32_t pad = ((raw_addr + 1023u) & ~1023u) - raw_addr;
  unsigned char* smem = smem_raw + pad;
  const uint32_t ring_addr = raw_addr + pad;
  Bars* bars = reinterpret_cast<Bars*>(smem + kRingBytes);
  volatile int* abort_flag = &bars->abort;
  DeviceStatus* status = reinterpret_cast<DeviceStatus*>(a.status);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const TcItemArg it = a.items[blockIdx.x];
  const int n = it.kt_end - it.kt_begin;
  if (n <= 0) return;  // the host never launches such a CTA

  if (threadIdx.x == 0) {
    for (int i = 0; i < kRing; ++i) {
      mbar_init(&bars->full[i], 1);
      mbar_init(&bars->empty[i], 1);
    }
    mbar_init(&bars->q_full, 128);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bars->s_full[i], 1);
      mbar_init(&bars->p_full[i], 128);
    }
    mbar_init(&bars->o_done, 1);
    mbar_init(&bars->drain, 1);
    bars->abort = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    ptx::tmem_alloc(smem_u32(&bars->tmem_base), kTmemCols);
    ptx::tmem_relinquish();
  }
  ptx::fence_before_sync();
  __syncthreads();
  ptx::fence_after_sync();
  const uint32_t tmem = bars->tmem_base;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      ptx::prefetch_tmap(&tmk);
      ptx::prefetch_tmap(&tmv);
      int e = 0;
      bool ok = true;
      auto issue = [&](const CUtensorMap* map, int kt) -> bool {
        const int slot = e % kRing;
        if (e >= kRing &&
            !mbar_wait(&bars->empty[slot], ((e / kRing) - 1) & 1, abort_flag, status, kSiteTcEmpty))
          return false;
        mbar_arrive_expect_tx(&bars->full[slot], kSlotBytes);
        const uint32_t dst = ring_addr + slot * kSlotBytes;
        const uint32_t bar = smem_u32(&bars->full[slot]);
#pragma unroll
        for (int i = 0; i < 4; ++i) ptx::tma_load_2d(dst + i * kBoxBytes, map, 64 * i, kt * kKeyTile, bar);
        ++e;
        return true;
      };
      for (int t = 0; t < n && ok; ++t) {
        ok = issue(&tmk, it.kt_begin + t);
        if (ok && t >= 1) ok = issue(&tmv, it.kt_begin + t - 1);
      }
      if (ok) ok = issue(&tmv, it.kt_begin + n - 1);
      if (!ok) {  // aborted: let every issued copy land before the CTA exits
        for (int s = 0; s < kRing && s < e; ++s) {
          const int last = ((e - 1 - s) / kRing) * kRing + s;
          mbar_wait(&bars->full[s], (last / kRing) & 1, nullptr, status, kSiteTcDrain);
        }
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ----------------------------------------------------------------- MMA
    if (lane == 0) {
      constexpr uint32_t ab = DT == KCA_BF16 ? 1u : 0u;
      constexpr uint32_t id_qk = ptx::idesc_f16(ab, 128, kKeyTile, 0);
      constexpr uint32_t id_pv = ptx::idesc_f16(ab, 128, kDim, 1);
      int e = 0;
      bool ok = mbar_wait(&bars->q_full, 0, abort_flag, status, kSiteTcQ);
      ptx::fence_after_sync();
      auto pv = [&](int u) -> bool {
        const int b = u & 1;
        if (!mbar_wait(&bars->p_full[b], (u >> 1) & 1, abort_flag, status, kSiteTcP)) return false;
        ptx::fence_after_sync();
        const int slot = e % kRing;
        if (!mbar_wait(&bars->full[slot], (e / kRing) & 1, abort_flag, status, kSiteTcFull)) return false;
        ptx::fence_after_sync();
        const uint32_t vbase = ring_addr + slot * kSlotBytes;
        const uint32_t pcol = b ? kColS1 : kColS0;
#pragma unroll
        for (int kk = 0; kk < kKeyTile / 16; ++kk)
          ptx::mma_ts(tmem + kColO, tmem + pcol + kk * 8,
                      ptx::sdesc_sw128(vbase + kk * 16 * 128, kBoxBytes, 1024), id_pv,
                      (u > 0 || kk > 0) ? 1u : 0u);
        ptx::mma_commit(smem_u32(&bars->empty[slot]));
        ptx::mma_commit(smem_u32(&bars->o_done));
        ++e;
        return true;
      };
      for (int t = 0; t < n && ok; ++t) {
        const int slot = e % kRing;
        if (!mbar_wait(&bars->full[slot], (e / kRing) & 1, abort_flag, status, kSiteTcFull)) {
          ok = false;
          break;
        }
        ptx::fence_after_sync();
        const uint32_t kbase = ring_addr + slot * kSlotBytes;
        const uint32_t scol = (t & 1) ? kColS1 : kColS0;
#pragma unroll
        for (int kk = 0; kk < kDim / 16; ++kk)
          ptx::mma_ts(tmem + scol, tmem + kColQ + kk * 8,
                      ptx::sdesc_sw128(kbase + (kk >> 2) * kBoxBytes + (kk & 3) * 32, 16, 1024),
                      id_qk, kk > 0 ? 1u : 0u);
        ptx::mma_commit(smem_u32(&bars->empty[slot]));
        ptx::mma_commit(smem_u32(&bars->s_full[t & 1]));
        ++e;
        if (t >= 1) ok = pv(t - 1);
      }
      if (ok) ok = pv(n - 1);
      // every MMA issued above has completed once this barrier flips
      ptx::mma_commit(smem_u32(&bars->drain));
      mbar_wait(&bars->drain, 0, nullptr, status, kSiteTcDrain);
    }
    __syncwarp();
  } else if (warp >= 4) {
    // ------------------------------------------------------------- softmax
    const int m = threadIdx.x - 128;                 // TMEM lane == M row
    const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
    const uint32_t trow = tmem + lane_base;
    const int64_t row = (int64_t)it.tile * kRowTile + (m >> 3);
    const bool valid = row < a.plan.rows;
    const int64_t pos = a.plan.chunk_start + row;
    const int64_t lo = lo_of(pos, a.plan.window);

    // Q row (row, head m & 7) into TMEM columns [0, 128), zeros past the chunk.
    {
      const uint4* qsrc = reinterpret_cast<const uint4*>(a.q) + ((int64_t)it.tile * 128 + m) * 32;
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        uint32_t r[32];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const uint4 v = valid ? qsrc[c * 8 + i] : make_uint4(0, 0, 0, 0);
          r[4 * i] = v.x; r[4 * i + 1] = v.y; r[4 * i + 2] = v.z; r[4 * i + 3] = v.w;
        }
        ptx::tmem_st32(trow + kColQ + c * 32, r);
      }
      ptx::tmem_wait_st();
      ptx::fence_before_sync();
      mbar_arrive(&bars->q_full);
    }

    float m_ref = -INFINITY;   // reference max, log2 units
    float l_sum = 0.f;
    const float cs = a.scale_log2;
    bool ok = true;
    for (int t = 0; t < n; ++t) {
      const int b = t & 1;
      const uint32_t scol = b ? kColS1 : kColS0;
      ok = __all_sync(0xffffffffu, mbar_wait(&bars->s_full[b], (t >> 1) & 1, abort_flag, status, kSiteTcS));
      if (!ok) break;
      ptx::fence_after_sync();
      float s[64];
      {
        uint32_t r0[32], r1[32];
        ptx::tmem_ld32(trow + scol, r0);
        ptx::tmem_ld32(trow + scol + 32, r1);
        ptx::tmem_wait_ld();
#pragma unroll
        for (int c = 0; c < 32; ++c) {
          s[c] = __uint_as_float(r0[c]);
          s[32 + c] = __uint_as_float(r1[c]);
        }
      }
      // Raw scores of keys outside [lo, pos] become -inf (the scale is > 0,
      // so they stay -inf below and their probability is exactly 0).
      const int64_t j0 = a.plan.kv_lo + (int64_t)(it.kt_begin + t) * kKeyTile;
      if (j0 < lo || j0 + kKeyTile - 1 > pos) {
#pragma unroll
        for (int c = 0; c < 64; ++c) {
          const int64_t j = j0 + c;
          if (j < lo || j > pos) s[c] = -INFINITY;
        }
      }
      // NaN-preserving row max over eight independent chains.
      float m8[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) m8[i] = s[i];
#pragma unroll
      for (int c = 8; c < 64; ++c) m8[c & 7] = max_nan(m8[c & 7], s[c]);
#pragma unroll
      for (int i = 0; i < 4; ++i) m8[i] = max_nan(m8[i], m8[i + 4]);
      const float mraw = max_nan(max_nan(m8[0], m8[2]), max_nan(m8[1], m8[3]));
      const float mx = mraw == -INFINITY ? -INFINITY : mraw * cs;
      const bool need = mx > m_ref + kRescaleLog2;
      const bool any_need = __any_sync(0xffffffffu, need);
      float alpha = 1.f;
      if (any_need) {
        alpha = need ? ptx::ex2(m_ref - mx) : 1.f;
        if (need) m_ref = mx;
        l_sum *= alpha;
      }
      // p = 2^(s*scale*log2e - m_ref), one FFMA and one MUFU op per score.
      const float nmu = m_ref == -INFINITY ? 0.f : -m_ref;
      uint32_t pr[32];
      float2 acc2[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f),
                        make_float2(0.f, 0.f)};
#pragma unroll
      for (int c = 0; c < 32; ++c) {
        const float p0 = ptx::ex2(fmaf(s[2 * c], cs, nmu));
        const float p1 = ptx::ex2(fmaf(s[2 * c + 1], cs, nmu));
        acc2[c & 3] = __fadd2_rn(acc2[c & 3], make_float2(p0, p1));
        pr[c] = pack2(p0, p1, DT);
      }
      acc2[0] = __fadd2_rn(acc2[0], acc2[1]);
      acc2[2] = __fadd2_rn(acc2[2], acc2[3]);
      acc2[0] = __fadd2_rn(acc2[0], acc2[2]);
      l_sum += acc2[0].x + acc2[0].y;
      ptx::tmem_st32(trow + scol, pr);
      // PV of the previous tile must be complete before O is touched and
      // before this thread lets PV of this tile start; waiting on every tile
      // keeps this thread within one phase of the barrier, which parity
      // waits require.
      if (t > 0) {
        ok = __all_sync(0xffffffffu,
                        mbar_wait(&bars->o_done, (t - 1) & 1, abort_flag, status, kSiteTcO));
        if (!ok) break;
        ptx::fence_after_sync();
        if (any_need) {
#pragma unroll 1
          for (int c = 0; c < kDim / 32; ++c) {
            uint32_t r[32];
            ptx::tmem_ld32(trow + kColO + c * 32, r);
            ptx::tmem_wait_ld();
#pragma unroll
            for (int i = 0; i < 32; ++i) r[i] = __float_as_uint(__uint_as_float(r[i]) * alpha);
            ptx::tmem_st32(trow + kColO + c * 32, r);
          }
        }
      }
      ptx::tmem_wait_st();
      ptx::fence_before_sync();
      mbar_arrive(&bars->p_full[b]);
    }
    if (ok)
      ok = __all_sync(0xffffffffu, mbar_wait(&bars->o_done, (n - 1) & 1, abort_flag, status, kSiteTcO));
    if (ok) {
      ptx::fence_after_sync();
      const float inv = 1.f / l_sum;
      float* dst;
      if (it.slot < 0) {
        dst = a.out + ((int64_t)it.tile * 128 + m) * kDim;
      } else {
        dst = a.part_acc + ((int64_t)it.slot * 128 + m) * kDim;
        a.part_ml[((int64_t)it.slot * 128 + m) * 2 + 0] = m_ref;
        a.part_ml[((int64_t)it.slot * 128 + m) * 2 + 1] = l_sum;
      }
      const float f = it.slot < 0 ? inv : 1.f;
#pragma unroll 1
      for (int c = 0; c < kDim / 32; ++c) {
        uint32_t r[32];
        ptx::tmem_ld32(trow + kColO + c * 32, r);
        ptx::tmem_wait_ld();
        if (valid) {
          float4* d4 = reinterpret_cast<float4*>(dst + c * 32);
#pragma unroll
          for (int i = 0; i < 8; ++i)
            d4[i] = make_float4(__uint_as_float(r[4 * i]) * f, __uint_as_float(r[4 * i + 1]) * f,
                                __uint_as_float(r[4 * i + 2]) * f, __uint_as_float(r[4 * i + 3]) * f);
        }
      }
    }
    ptx::fence_before_sync();
  }

  __syncthreads();
  if (warp == 1) {
    ptx::fence_after_sync();
    ptx::tmem_dealloc(tmem, kTmemCols);
  }
}

// Log-sum-exp merge of the items of each split row tile: a group of W warps
// per M row, 8 / W rows per CTA, grid (tiles, 16 W).
template <int W>
__global__ void __launch_bounds__(256) merge_tc_kernel(const TcArgs a) {
  constexpr int kRowsPerCta = 8 / W;
  const int tile = blockIdx.x;
  const int ns = a.tile_items[tile];
  if (ns <= 1) return;
  __shared__ float red[8 * 264];
  const int warp = threadIdx.x >> 5;
  const int gi = warp / W, g = warp % W;
  const int m = blockIdx.y * kRowsPerCta + gi;
  if ((int64_t)tile * kRowTile + (m >> 3) >= a.plan.rows) return;  // whole group leaves together
  const int64_t r0 = (int64_t)a.tile_first_slot[tile] * 128 + m;
  merge_row<W>(ns, a.part_ml + r0 * 2, 128 * 2, a.part_acc + r0 * kDim, (int64_t)128 * kDim, 1.f,
               a.out + ((int64_t)tile * 128 + m) * kDim, red + gi * W * 264, g, threadIdx.x & 31,
               1 + gi);
}

template <int DT>
cudaError_t launch_t(const CUtensorMap& tmk, const CUtensorMap& tmv, const TcArgs& a,
                     cudaStream_t stream) {
  static bool attr_set[64] = {false};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  if (!attr_set[dev]) {
    cudaError_t e = cudaFuncSetAttribute(prefill_tc_kernel<DT>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
    if (e != cudaSuccess) return e;
    attr_set[dev] = true;
  }
  prefill_tc_kernel<DT><<<a.plan.n_items, kThreads, kSmemBytes, stream>>>(tmk, tmv, a);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess || a.plan.n_slots == 0) return e;
  const int ns = a.plan.max_split;
  const int w = ns > 8 ? 8 : (ns > 4 ? 4 : (ns > 2 ? 2 : 1));
  const dim3 grid(a.plan.n_tiles, 16 * w);
  if (w == 8) merge_tc_kernel<8><<<grid, 256, 0, stream>>>(a);
  else if (w == 4) merge_tc_kernel<4><<<grid, 256, 0, stream>>>(a);
  else if (w == 2) merge_tc_kernel<2><<<grid, 256, 0, stream>>>(a);
  else merge_tc_kernel<1><<<grid, 256, 0, stream>>>(a);
  return cudaGetLastError();
}

}  // namespace

void fill_tc_tables(TcArgs& a) {
  // One pass over the tiles: O(tiles + items), no per-item plan walk.
  int32_t idx = 0, slot = 0;
  for (int32_t t = 0; t < a.plan.n_tiles && t < kTcMaxTiles; ++t) {
    int32_t kb, ke;
    tc_tile_keys(a.plan, t, &kb, &ke);
    const int32_t n = ke - kb;
    const int32_t s = (int32_t)cdiv(n, a.plan.per_item);
    a.tile_items[t] = (int16_t)s;
    a.tile_first_slot[t] = (int16_t)slot;
    for (int32_t k = 0; k < s && idx < kTcMaxItems; ++k, ++idx) {
      a.items[idx].kt_begin = kb + (int32_t)(((int64_t)k * n) / s);
      a.items[idx].kt_end = kb + (int32_t)(((int64_t)(k + 1) * n) / s);
      a.items[idx].tile = (int16_t)t;
      a.items[idx].slot = (int16_t)(s > 1 ? slot + k : -1);
    }
    if (s > 1) slot += s;
  }
}

cudaError_t launch_prefill_tc(int dtype, const CUtensorMap& tmk, const CUtensorMap& tmv,
                              const TcArgs& a, cudaStream_t stream) {
  if (dtype == KCA_BF16) return launch_t<KCA_BF16>(tmk, tmv, a, stream);
  if (dtype == KCA_F16) return launch_t<KCA_F16>(tmk, tmv, a, stream);
  return cudaErrorInvalidValue;
}

}  // namespace kca

// kca_rows_tc.cu -- batched short chunks (attn_prefill_batch) on the sm_100a
// tensor cores: tcgen05 MMAs issued by one thread, accumulators in tensor
// memory.
//
// The pages' geometry (Karume v0.12.0 release notes, "Performance", item 3,
// and "Docs", ADR 0067): plans of 2-15 query rows sit between single-row
// decode and the row tiles of prefill.  A unit is up to four consecutive
// query rows of one sequence (the units, splits and partials of the mma.sync
// multi-row kernel in kca_decode_mma.cu), or up to eight when a call has
// more than four rows per sequence, so each K / V stage crosses from L2 once
// for all of them.  The mma.sync form of this kernel is bound by instruction
// issue (two warps per SM sub-partition run the QK^T and PV fragments, the
// softmax and the shared-memory traffic of every stage); here one thread
// issues every MMA and four warps per TMEM lane quarter in use run the
// softmax, so the tensor pipe, the softmax and the load stream overlap.
// Clock traces of one split chose the layout: the high and low parts of Q
// and of P share their MMA instructions as M rows (the MMA issue was the
// longest step), and the rows sit in lane quarters with full warps (the
// softmax chain was the next).
//
// Rows.  A warp reaches only the TMEM lane quarter of its SM sub-partition
// (warp w: lanes 32 (w % 4) .. +31).  Query rows i = 2 q, 2 q + 1 of a unit
// live in quarter q (quarters 0-1 for 4-row units, 0-3 for 8): lane
// 8 (i % 2) + h of the quarter holds the high 16-bit part of head h's query,
// lane 16 + 8 (i % 2) + h its low part (f32 queries keep f32-grade products:
// q = q_hi + q_lo in the cache's 16-bit type), so one Q K^T MMA of M = 128
// gives both partial scores of every head of every row, in lanes l and
// l ^ 16 of one warp, which add them with a shuffle; the M rows of unused
// quarters are never read.  In O += P V the probabilities are stacked the
// same way (p = p_hi + p_lo in the same two lanes) and the two O rows are
// added at the end.
//
// Warp roles (16 warps for 4-row units, 19 for 8; all stage the queries):
//   warps 4 g + q, q a quarter in use   softmax: key columns [16 g, +16)
//            of every stage for the rows of quarter q (the high lane of a
//            head columns 16 g .. + 7, the low lane 16 g + 8 .. + 15) and O
//            columns [64 g, +64), then the epilogue; a stage's row max is
//            exchanged between the quarter's four warps through shared memory
//   warp 2 (16 for 8-row units)   TMEM allocator; lane 0 issues every MMA;
//            the warp zeroes the V rows of a ragged last stage
//   warps 3, 7 (17, 18)   TMA producers of K stages (64 keys x 256 dims, a
//            ring of 3, of 2 for 8-row units) and of V stages (ring of 2)
// Shared memory: Q (32 M rows per quarter in use x 256 dims, four 64-dim
// chunks with 128-byte swizzle; for 4-row units the descriptors of the last
// chunk reach on into the bytes after it, which land only in unused M rows),
// the K and V rings.
// Tensor memory (512 columns): S of stage j at [64 (j & 1), +64), P of stage
// j at [128 + 32 (j & 1), +32) (16-bit pairs), O at [256, 512).
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

constexpr int kRQuarterThreads = 128;                // the softmax warps of one TMEM lane quarter
constexpr int kRKeys = 64;                           // keys per stage
constexpr int kRBox = 64 * 64 * 2;                   // 64 rows x 64 dims (16-bit): 8 KiB
constexpr int kRSlot = 4 * kRBox;                    // K or V of one stage: 32 KiB
constexpr uint32_t kRColS = 0, kRColP = 128, kRColO = 256, kRTmemCols = 512;
constexpr float kRRescaleLog2 = 8.f;   // rescale O once a score passes the reference by 2^8
// Merge tickets: one per unit, after the workspace's 256-byte status word.
constexpr int kRTickets = (KCA_WORKSPACE_HEADER - 256) / 4;
static_assert(KCA_MAX_BATCH * ((KCA_MAX_BATCH_ROWS + kMultiRows - 1) / kMultiRows) <= kRTickets, "tickets");

// Layout of a unit of UR rows (4 or 8): UR / 2 TMEM lane quarters, four
// softmax warps per quarter, then the MMA and producer warps; a wide unit's
// Q takes all 128 M rows, so its K ring is one stage shorter.
template <int UR>
struct RowsTc {
  static constexpr int NQ = UR / 2;                       // lane quarters in use
  static constexpr int kWarps = UR == 4 ? 16 : 19;
  static constexpr int kThreads = 32 * kWarps;
  static constexpr int kMmaWarp = UR == 4 ? 2 : 16, kKWarp = UR == 4 ? 3 : 17, kVWarp = UR == 4 ? 7 : 18;
  static constexpr int kKRing = UR == 4 ? 3 : 2, kVRing = 2;
  static constexpr int kQChunk = 32 * NQ * 128;           // 32 NQ M rows x 64 dims
  static constexpr int kOffQ = 0;
  static constexpr int kOffK = 4 * kQChunk;
  static constexpr int kOffV = kOffK + kKRing * kRSlot;
  static constexpr int kOffBar = kOffV + kVRing * kRSlot;
  static constexpr int kBarBytes = 8192;
  static constexpr int kSmemBytes = kOffBar + kBarBytes + 1024;   // + alignment slack
  static_assert(kSmemBytes <= 232448, "shared memory over the per-CTA limit");
  // A descriptor of 128 M rows starting at the last Q chunk reads past the Q
  // area when UR = 4, into the first K slot: those bytes only reach M rows
  // 64-127 of S, which nothing reads (an MMA's D row depends on its A row).
  static_assert(kOffQ + 3 * kQChunk + 16 * 1024 <= kOffV, "Q descriptors stay inside shared memory");
};

template <int UR>
struct RBars {
  static constexpr int NQ = UR / 2;
  uint64_t kfull[RowsTc<UR>::kKRing], kempty[RowsTc<UR>::kKRing];
  uint64_t vfull[RowsTc<UR>::kVRing], vempty[RowsTc<UR>::kVRing];
  uint64_t s_full[2];   // Q K^T of stage j complete in S buffer j & 1 (MMA commit)
  uint64_t p_full[2];   // P of stage j written and O corrected (the softmax warps)
  uint64_t o_done[2];   // P V of stage j complete (MMA commit)
  uint64_t drain;       // every MMA complete (single use)
  uint32_t tmem_base;
  int abort;
  int last;             // this CTA drew the unit's last ticket: it merges the splits
  float red[2][NQ][4][32];  // [stage parity][quarter][column group][lane]: partial row maxima
  float red_l[NQ][4][32];   // [quarter][column group][lane]: partial row sums at the end
};
static_assert(sizeof(RBars<8>) <= RowsTc<8>::kBarBytes && sizeof(RBars<4>) <= RowsTc<4>::kBarBytes,
              "barrier block too large");

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
__device__ __forceinline__ void named_sync(int id, int n) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(n) : "memory");
}

template <int QT, int KT, int UR>
__global__ void __launch_bounds__(RowsTc<UR>::kThreads, 1)
    rows_tc_kernel(const __grid_constant__ CUtensorMap tmk, const __grid_constant__ CUtensorMap tmv,
                   const RowsArgs a) {
  using T = RowsTc<UR>;
  constexpr int kRThreads = T::kThreads;
  constexpr int kRKRing = T::kKRing, kRVRing = T::kVRing, kRQChunk = T::kQChunk;
  constexpr int kROffQ = T::kOffQ, kROffK = T::kOffK, kROffV = T::kOffV;
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  const uint32_t raw_addr = smem_u32(smem_raw);
  const uint32_t pad = ((raw_addr + 1023u) & ~1023u) - raw_addr;
  unsigned char* smem = smem_raw + pad;
  const uint32_t sbase = raw_addr + pad;
  RBars<UR>* bars = reinterpret_cast<RBars<UR>*>(smem + T::kOffBar);
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
                         (nsplit == 1 || (((int64_t)b * a.rows_per_seq + i0 + nr) * a.max_splits <= a.part_slots &&
                                          unit < kRTickets)),
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
      mbar_init(&bars->p_full[s], T::NQ * kRQuarterThreads / 32);
      mbar_init(&bars->o_done[s], 1);
    }
    mbar_init(&bars->drain, 1);
    bars->abort = 0;
    fence_barrier_init();
  }
  if (warp == T::kMmaWarp) {
    ptx::tmem_alloc(smem_u32(&bars->tmem_base), kRTmemCols);
    ptx::tmem_relinquish();
  }
  if (threadIdx.x == T::kKWarp * 32) ptx::prefetch_tmap(&tmk);
  if (threadIdx.x == T::kVWarp * 32) ptx::prefetch_tmap(&tmv);
  ptx::fence_before_sync();
  __syncthreads();
  ptx::fence_after_sync();
  const uint32_t tmem = bars->tmem_base;
  // Programmatic dependent launch: the set-up above overlaps the previous
  // kernel of the stream; global memory is touched only after this wait.
  asm volatile("griddepcontrol.wait;" ::: "memory");

  // Stage the queries: M row m = 32 q + 16 part + 8 (i % 2) + h for query
  // row i = 2 q + ..., head h, part 0 (high) or 1 (low); absent rows zero.
  // 16-byte group u of the 256 dims: chunk u / 8, 128-byte swizzle within it.
  for (int it = threadIdx.x; it < 32 * T::NQ * 32; it += kRThreads) {
    const int m = it >> 5, u = it & 31;
    const int part = (m >> 4) & 1, i = 2 * (m >> 5) + ((m >> 3) & 1), h = m & 7;
    float x[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    if (i < nr) {
      const int64_t orow = (int64_t)b * a.rows_per_seq + i0 + i;
      load8<QT>(static_cast<const char*>(a.q) + ((orow * kHeads + h) * kDim + 8 * u) * ElemBytes<QT>::value, x);
    }
    uint32_t w[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const uint32_t hi = pk2<KT>(x[2 * j], x[2 * j + 1]);
      const float2 f = upk2<KT>(hi);
      w[j] = part == 0 ? hi : pk2<KT>(x[2 * j] - f.x, x[2 * j + 1] - f.y);
    }
    *reinterpret_cast<uint4*>(smem + kROffQ + (u >> 3) * kRQChunk + m * 128 + (((u & 7) ^ (m & 7)) << 4)) =
        make_uint4(w[0], w[1], w[2], w[3]);
  }
  fence_proxy_async_smem();   // generic stores -> visible to the tensor core
  __syncthreads();

  if (warp == T::kKWarp || warp == T::kVWarp) {
    // ------------------------------------------------------------ producers
    if (lane == 0) {
      const bool is_k = warp == T::kKWarp;
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
  } else if (warp == T::kMmaWarp) {
    // ----------------------------------------------------------------- MMA
    constexpr uint32_t ab = KT == KCA_BF16 ? 1u : 0u;
    constexpr uint32_t id_qk = ptx::idesc_f16(ab, 128, kRKeys, 0);
    constexpr uint32_t id_pv = ptx::idesc_f16(ab, 128, kDim, 1);
    // Descriptor bases; an operand at byte offset x from a base is the base
    // plus x >> 4 in the start-address field (addresses stay below 256 KiB).
    const uint64_t qd0 = ptx::sdesc_sw128(sbase + kROffQ, 16, 1024);
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
        // P's high and low parts in lanes l and l ^ 16 of the same columns:
        // their O rows get p_hi V and p_lo V
        const uint32_t pcol = tmem + kRColP + 32 * (u & 1);
        const uint64_t vd = vd0 + (uint64_t)((s * kRSlot) >> 4);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)   // 16 keys per step: 8 TMEM columns of P, V rows 16 kk
          ptx::mma_ts(tmem + kRColO, pcol + 8 * kk, vd + (uint64_t)((kk * 16 * 128) >> 4), id_pv,
                      (u > 0 || kk > 0) ? 1u : 0u);
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
          ptx::mma_ss(scol, qd0 + (uint64_t)(qo >> 4), kd + (uint64_t)(ko >> 4), id_qk, k > 0 ? 1u : 0u);
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
  } else if (warp < 16 && (warp & 3) < T::NQ) {
    // ------------------------------------------------------------- softmax
    // Warp 4 g + q: quarter q (query rows 2 q, 2 q + 1), key columns
    // [16 g, +16) of every stage, O columns [64 g, +64).  Lane l: query row
    // 2 q + ((l >> 3) & 1), head l & 7, high part (l < 16) or low (l >= 16);
    // lanes l and l ^ 16 pair up: the high lane takes columns 16 g .. + 7, the
    // low lane 16 g + 8 .. + 15, each first fetching the other part of its
    // columns' scores from its partner.  The quarter's four warps exchange
    // their row maxima at a named barrier that each takes on every stage
    // (work is skipped after an abort, so no warp waits there for one that
    // left).
    const int q = warp & 3, g = warp >> 2;
    const bool low = lane >= 16;
    const int i = 2 * q + ((lane >> 3) & 1), h = lane & 7;
    const bool valid = i < nr;
    const uint32_t trow = tmem + ((uint32_t)(32 * q) << 16);
    const int64_t pos = pos0 + i;
    const int64_t lo = lo_of(pos, a.window);
    const float cs = a.scale * 1.4426950408889634f;  // scores in log2 units
    const int cofs = 16 * g + (low ? 8 : 0);         // this lane's 8 columns within a stage
    float m_ref = -INFINITY;                         // reference max of the row, log2 units
    float l_part = 0.f;                              // this lane's columns of the row sum
    bool ok = true;
    for (int j = 0; j < n; ++j) {
      ok = __all_sync(0xffffffffu, ok && mbar_wait(&bars->s_full[j & 1], (j >> 1) & 1, abort_flag, status, kSiteTcS));
      float s[8];
      float mloc = -INFINITY;
      if (ok) {
        ptx::fence_after_sync();
        uint32_t r[16];
        ptx::tmem_ld16(trow + kRColS + 64 * (j & 1) + 16 * g, r);
        ptx::tmem_wait_ld();
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          const float mine = __uint_as_float(low ? r[8 + c] : r[c]);
          const float give = __uint_as_float(low ? r[c] : r[8 + c]);
          s[c] = mine + __shfl_xor_sync(0xffffffffu, give, 16);
        }
        // keys outside [lo, pos], past the split's end, or of a row the unit
        // does not have become -inf (scale > 0 keeps them there)
        const int64_t k0 = kbeg + (int64_t)j * kRKeys + cofs;
        const int64_t left = kend - k0;               // keys of the split from this lane's first on
        if (!(valid && left >= 8 && k0 >= lo && k0 + 7 <= pos)) {
#pragma unroll
          for (int c = 0; c < 8; ++c) {
            const int64_t key = k0 + c;
            if (!valid || c >= left || key < lo || key > pos) s[c] = -INFINITY;
          }
        }
        mloc = max_nan(max_nan(max_nan(s[0], s[1]), max_nan(s[2], s[3])),
                       max_nan(max_nan(s[4], s[5]), max_nan(s[6], s[7])));
        mloc = max_nan(mloc, __shfl_xor_sync(0xffffffffu, mloc, 16));   // the warp's 16 columns
      }
      bars->red[j & 1][q][g][lane] = mloc;
      named_sync(1 + q, kRQuarterThreads);
      if (ok) {
        const float* rm = bars->red[j & 1][q][0];
        const float mraw = max_nan(max_nan(rm[lane], rm[32 + lane]), max_nan(rm[64 + lane], rm[96 + lane]));
        const float mx = mraw == -INFINITY ? -INFINITY : mraw * cs;
        const bool need = mx > m_ref + kRRescaleLog2;   // the same in all the row's lanes
        if (__any_sync(0xffffffffu, need)) {
          const float alpha = need ? ptx::ex2(m_ref - mx) : 1.f;
          if (need) m_ref = mx;
          l_part *= alpha;
          if (j > 0) {
            // P V of stage j - 1 must finish before O is rescaled (that of
            // stage j - 2 preceded this stage's Q K^T, so it has); each lane
            // scales its own O row (high or low part)
            ok = __all_sync(0xffffffffu, mbar_wait(&bars->o_done[(j - 1) & 1], ((j - 1) >> 1) & 1, abort_flag,
                                                   status, kSiteTcO));
            if (ok) {
              ptx::fence_after_sync();
#pragma unroll 1
              for (int c = 0; c < 2; ++c) {
                uint32_t r[32];
                ptx::tmem_ld32(trow + kRColO + 64 * g + 32 * c, r);
                ptx::tmem_wait_ld();
#pragma unroll
                for (int e = 0; e < 32; ++e) r[e] = __float_as_uint(__uint_as_float(r[e]) * alpha);
                ptx::tmem_st32(trow + kRColO + 64 * g + 32 * c, r);
              }
              ptx::tmem_wait_st();
            }
          }
        }
      }
      if (ok) {
        // p = 2^(s cs - m_ref) for this lane's columns, split into 16-bit
        // high and low parts; the high lane keeps the high parts of the
        // warp's 16 columns, the low lane the low parts (each gives the
        // partner the other half)
        const float nmu = m_ref == -INFINITY ? 0.f : -m_ref;
        uint32_t pr[8];
        float acc = 0.f;
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          const float p0 = ptx::ex2(fmaf(s[2 * c], cs, nmu));
          const float p1 = ptx::ex2(fmaf(s[2 * c + 1], cs, nmu));
          acc += p0 + p1;
          const uint32_t ph = pk2<KT>(p0, p1);
          const float2 f = upk2<KT>(ph);
          const uint32_t pl = pk2<KT>(p0 - f.x, p1 - f.y);
          const uint32_t got = __shfl_xor_sync(0xffffffffu, low ? ph : pl, 16);
          // P row, the warp's 16 columns: 16 g .. + 7 (pairs 0-3), 16 g + 8 .. (pairs 4-7)
          pr[c] = low ? got : ph;
          pr[4 + c] = low ? pl : got;
        }
        l_part += acc;
        // P buffer j & 1 was last read by P V of stage j - 2, complete before
        // this stage's Q K^T (whose completion s_full signalled).
        ptx::tmem_st8(trow + kRColP + 32 * (j & 1) + 8 * g, pr);
        ptx::tmem_wait_st();
        ptx::fence_before_sync();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars->p_full[j & 1]);
      }
    }
    if (ok)
      ok = __all_sync(0xffffffffu, mbar_wait(&bars->o_done[(n - 1) & 1], ((n - 1) >> 1) & 1, abort_flag, status,
                                             kSiteTcO));
    bars->red_l[q][g][lane] = l_part + __shfl_xor_sync(0xffffffffu, l_part, 16);
    named_sync(1 + q, kRQuarterThreads);
    // An aborted split poisons its rows; the status word says why.  The flag
    // is raised before the failing warp reaches the barrier above.
    const bool aborted = !ok || *abort_flag;
    const float* rl = bars->red_l[q][0];
    const float L = aborted ? NAN : (rl[lane] + rl[32 + lane]) + (rl[64 + lane] + rl[96 + lane]);
    const float M = aborted ? NAN : m_ref * 0.6931471805599453f;   // natural units for the merge
    // Epilogue: O = (high row) + (low row) over the warp's 64 columns; the
    // high lane writes dims 64 g .. + 31 of its head, the low lane 64 g + 32
    // .. + 63, scaled by 1 / l (one split) or raw with (m, l) (a split
    // partial, merged below).
    const int64_t orow = (int64_t)b * a.rows_per_seq + i0 + i;
    float* dst = nullptr;
    float f = 1.f;
    if (valid) {
      if (nsplit == 1) {
        dst = a.out + (orow * kHeads + h) * kDim + 64 * g + (low ? 32 : 0);
        f = (m_ref == -INFINITY && L == 0.f) ? 0.f : 1.f / L;
      } else {
        const int64_t slot = (orow * a.max_splits + split) * kHeads + h;
        dst = a.part_acc + slot * kDim + 64 * g + (low ? 32 : 0);
        if (!low && g == 0) *reinterpret_cast<float2*>(a.part_ml + slot * 2) = make_float2(M, L);
      }
    }
    uint32_t ra[32], rb[32];
    if (!aborted) {
      ptx::fence_after_sync();
      ptx::tmem_ld32(trow + kRColO + 64 * g, ra);
      ptx::tmem_ld32(trow + kRColO + 64 * g + 32, rb);
      ptx::tmem_wait_ld();
    } else {
#pragma unroll
      for (int e = 0; e < 32; ++e) ra[e] = rb[e] = 0u;
    }
#pragma unroll
    for (int e = 0; e < 32; ++e) {
      // the high lane adds the low row's dim 64 g + e, the low lane the high row's 64 g + 32 + e
      const float give = __uint_as_float(low ? ra[e] : rb[e]);
      const float got = __shfl_xor_sync(0xffffffffu, give, 16);
      ra[e] = __float_as_uint((__uint_as_float(low ? rb[e] : ra[e]) + got) * f);
    }
    if (valid) {
#pragma unroll
      for (int e = 0; e < 8; ++e)
        *reinterpret_cast<float4*>(dst + 4 * e) =
            aborted ? make_float4(NAN, NAN, NAN, NAN)
                    : make_float4(__uint_as_float(ra[4 * e]), __uint_as_float(ra[4 * e + 1]),
                                  __uint_as_float(ra[4 * e + 2]), __uint_as_float(ra[4 * e + 3]));
    }
  }
  // No warp leaves while MMAs may still read shared memory or write TMEM.
  ptx::fence_before_sync();
  __syncthreads();
  if (warp == T::kMmaWarp) {
    ptx::fence_after_sync();
    ptx::tmem_dealloc(tmem, kRTmemCols);
  }
  if (nsplit > 1 && a.tickets != nullptr) {
    // The unit's splits meet by ticket: the CTA that draws the last one
    // merges every split's partials of the unit's rows (log-sum-exp, as in
    // multirow_merge_kernel), so no second kernel and no CTA waits on
    // another.  The host gives tickets only while a unit has few splits;
    // with many, multirow_merge_kernel merges across the whole GPU after
    // this kernel instead of one CTA reading every partial.  Release: the
    // block's partial stores, ordered by the barrier above before one
    // thread's acq_rel atomic; acquire: the same atomic in the last CTA,
    // then the barrier below.
    if (threadIdx.x == 0) {
      int prev;
      asm volatile("atom.acq_rel.gpu.global.add.s32 %0, [%1], 1;" : "=r"(prev) : "l"(a.tickets + unit) : "memory");
      bars->last = prev == nsplit - 1;
    }
    __syncthreads();
    if (bars->last) {
      // warp w: (row, head) pairs p = 8 i + h, w and w + 16; lane l: dims 8 l .. 8 l + 7
      for (int p = warp; p < 8 * nr; p += kRThreads / 32) {
        const int i = p >> 3, h = p & 7;
        const int64_t orow = (int64_t)b * a.rows_per_seq + i0 + i;
        const int64_t row0 = orow * a.max_splits * kHeads + h;   // split sp: partial row row0 + sp * 8
        float M = -INFINITY;
        for (int sp = lane; sp < nsplit; sp += 32)
          M = max_nan(M, __ldcg(a.part_ml + (row0 + (int64_t)sp * kHeads) * 2));
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) M = max_nan(M, __shfl_xor_sync(0xffffffffu, M, o));
        const float mu = M == -INFINITY ? 0.f : M;
        float L = 0.f, acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll 4
        for (int sp = 0; sp < nsplit; ++sp) {
          const int64_t r = row0 + (int64_t)sp * kHeads;
          const float2 ml = __ldcg(reinterpret_cast<const float2*>(a.part_ml + r * 2));
          const float4* src = reinterpret_cast<const float4*>(a.part_acc + r * kDim + 8 * lane);
          const float4 v0 = __ldcg(src), v1 = __ldcg(src + 1);
          const float f = exp2f((ml.x - mu) * 1.4426950408889634f);
          L += f * ml.y;
          acc[0] += f * v0.x; acc[1] += f * v0.y; acc[2] += f * v0.z; acc[3] += f * v0.w;
          acc[4] += f * v1.x; acc[5] += f * v1.y; acc[6] += f * v1.z; acc[7] += f * v1.w;
        }
        const float inv = (M == -INFINITY && L == 0.f) ? 0.f : 1.f / L;
        float4* dst = reinterpret_cast<float4*>(a.out + (orow * kHeads + h) * kDim + 8 * lane);
        dst[0] = make_float4(acc[0] * inv, acc[1] * inv, acc[2] * inv, acc[3] * inv);
        dst[1] = make_float4(acc[4] * inv, acc[5] * inv, acc[6] * inv, acc[7] * inv);
      }
      if (threadIdx.x == 0) a.tickets[unit] = 0;   // ready for the next call
    }
  }
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

template <int QT, int KT, int UR>
cudaError_t launch_t(const CUtensorMap& tmk, const CUtensorMap& tmv, const RowsArgs& a, cudaStream_t stream) {
  using T = RowsTc<UR>;
  auto kern = rows_tc_kernel<QT, KT, UR>;
  static std::atomic<bool> attr_set[64];   // per device; zero-initialised
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  if (!attr_set[dev]) {
    const cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, T::kSmemBytes);
    if (e != cudaSuccess) return e;
    attr_set[dev] = true;
  }
  cudaLaunchAttribute at;
  at.id = cudaLaunchAttributeProgrammaticStreamSerialization;
  at.val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(a.max_splits, a.n_units, 1);
  cfg.blockDim = dim3(T::kThreads, 1, 1);
  cfg.dynamicSmemBytes = T::kSmemBytes;
  cfg.stream = stream;
  cfg.attrs = &at;
  cfg.numAttrs = 1;
  const cudaError_t e = cudaLaunchKernelEx(&cfg, kern, tmk, tmv, a);
  if (e != cudaSuccess || a.max_splits <= 1 || a.tickets != nullptr) return e;
  return launch_multirow_merge(a, stream);
}

}  // namespace

cudaError_t launch_rows_tc(int q_dtype, int kv_dtype, const CUtensorMap& tmk, const CUtensorMap& tmv,
                           const RowsArgs& a, cudaStream_t stream) {
#define KCA_RTC_CASE(QD, KD)                                                                \
  if (q_dtype == QD && kv_dtype == KD)                                                      \
    return a.unit_rows == kMultiRowsWide ? launch_t<QD, KD, kMultiRowsWide>(tmk, tmv, a, stream) \
                                         : launch_t<QD, KD, kMultiRows>(tmk, tmv, a, stream);
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

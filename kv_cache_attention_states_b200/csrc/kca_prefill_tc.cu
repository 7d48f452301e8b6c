// kca_prefill_tc.cu -- chunked causal prefill on the sm_100a tensor cores.
//
// The pages' design (Karume v0.12.0 release notes, "Performance", item 1):
// for plans of 16 or more chunk rows, QK and PV run on a GEMM tile skeleton
// so that each K / V row is read once per row tile instead of once per query
// row.  Here a CTA pair (a cluster of two CTAs on two SMs) takes one work
// item -- two row tiles of 16 positions x 8 heads (M = 128 each: the 8 heads
// share their single KV head) and a run of 128-key tiles -- and fuses the
// three stages the pages keep apart (QK, softmax statistics, PV), so no
// score matrix ever reaches memory.
//
// Why pairs: one SM pulls at most ~53 bytes per clock from L2 by TMA, while
// a 128-key K + V tile (128 KiB) feeds 2048 clocks of MMA -- 64 B/clk.  With
// tcgen05 MMAs of M = 256 over the pair (cta_group::2) each SM loads only its
// half of every K and V tile (B is split along N), so the tensor pipe, not
// the L2 stream, sets the pace.
//
// Warp roles (12 warps per CTA):
//   warp 0      TMA producer: the CTA's Q tile once, then its half of every
//               K tile (64 keys x 256 dims as four 64 x 64 boxes)
//   warp 1      TMEM allocator (both CTAs); in the even CTA the single thread
//               that issues every MMA of the pair
//   warp 2      TMA producer of its half of every V tile (128 keys x 128 dims),
//               from the moment the item's first QK^T is done
//   warps 4-7   softmax warpgroup 0: keys 0-63 of every S tile
//   warps 8-11  softmax warpgroup 1: keys 64-127
//   Thread m of a softmax warpgroup owns TMEM lane m, i.e. M row m of its CTA.
//
// Operands: S = Q K^T with Q (A) and K (B) in shared memory; O += P V with P
// (A) in tensor memory and V (B) in shared memory.  Tensor memory per CTA
// (512 columns x 128 lanes of 32 bits):
//   [  0,128)  P of tiles t (even / odd) as 16-bit pairs, 64 columns each
//   [128,256)  S (f32, 128 keys), released as soon as both warpgroups hold
//              their half in registers, so QK^T of the next tile overlaps
//              the softmax of this one
//   [256,512)  O accumulator (f32, 256 dims)
// Shapes per instruction: QK^T M256 N128 K16, PV M256 N256 K16 over the pair.
//
// The softmax keeps a reference max per row and rescales O (in TMEM) only
// when a score exceeds it by more than 2^8, so probabilities stay <= 256 and
// the O round trip is rare; the result is exact up to rounding whatever
// reference is used.  It takes each tile's probabilities with the current
// reference first and needs the row max (and its exchange between the two
// warpgroups) only when a half row's sum passes 2^8.  Work items of a split
// row tile write (m, l, O) partials that merge_tc_kernel (below) combines by
// log-sum-exp.
#include <atomic>
#include <cuda.h>
#include <cuda_runtime.h>

#include "kca_common.cuh"
#include "kca_plan.h"
#include "kca_tc.h"
#include "kca_tc_ptx.cuh"

namespace kca {
namespace {

constexpr int kThreads = 384;
// Per CTA of a pair: its half of every K tile (64 of the 128 keys, all 256
// dims) and of every V tile (128 of the 256 dims, all 128 keys).
constexpr int kKRing = 2;                              // K tile halves
constexpr int kVRing = 2;                              // V tile halves
constexpr int kKChunkBytes = 64 * 64 * 2;              // 64 keys x 64 dims: 8 KiB
constexpr int kKSlotBytes = 4 * kKChunkBytes;          // 64 keys x 256 dims: 32 KiB
constexpr int kVBoxBytes = 64 * 64 * 2;                // 64 keys x 64 dims: 8 KiB
constexpr int kVSlotBytes = 4 * kVBoxBytes;            // 128 keys x 128 dims: 32 KiB
constexpr int kOffK = 0;
constexpr int kOffV = kOffK + kKRing * kKSlotBytes;    // 64 KiB
constexpr int kOffQ = kOffV + kVRing * kVSlotBytes;    // 128 KiB
constexpr int kQBoxBytes = 128 * 64 * 2;               // Q: 128 M rows x 64 dims, 16 KiB
constexpr int kQBytes = 4 * kQBoxBytes;                // the CTA's Q tile, resident for the whole item
constexpr int kOffBar = kOffQ + kQBytes;               // 192 KiB
constexpr int kOBoxBytes = 128 * 32 * 4;               // O: 128 M rows x 32 f32, 16 KiB
static_assert(8 * kOBoxBytes <= kOffQ, "O tile fits the K/V rings");
constexpr int kBarBytes = 4096;
constexpr int kSmemBytes = kOffBar + kBarBytes + 1024; // + alignment slack
constexpr uint32_t kTmemCols = 512;
// TMEM: P of tile t (16-bit pairs, the A operand of P V) in buffer t&1 at
// columns [64 (t&1), +64), S at [128, 256), O at [256, 512).
constexpr uint32_t kColP = 0, kColS = 128, kColO = 256;
constexpr float kRescaleLog2 = 8.f;  // rescale O once a score passes the reference by 2^8
constexpr int kSoftmaxThreads = 256;
constexpr uint32_t kPairArrivals = 2 * kSoftmaxThreads / 32;  // one per softmax warp of both CTAs
constexpr uint16_t kPairMask = 3;    // both CTAs of the cluster

// Barriers.  The even CTA ("leader") issues every MMA of the pair, so the
// barriers it waits on (kfull, vfull, q_full, s_free, p_full) live in its
// shared memory and collect arrivals / bytes from both CTAs; the ones the
// MMAs signal (kempty, vempty, s_full, o_done, o_final, drain) are
// multicast to the same offset in both CTAs (as is s_first, which the V
// producers wait on).
struct Bars {
  uint64_t kfull[kKRing], kempty[kKRing];
  uint64_t vfull[kVRing], vempty[kVRing];
  uint64_t q_full;     // both CTAs' Q tiles landed in shared memory (TMA bytes)
  uint64_t s_full;     // S of the current tile computed (MMA commit)
  uint64_t s_free;     // S copied to registers by all 16 softmax warps
  uint64_t p_full[2];  // P of tile t in TMEM buffer t&1 written, O corrected (16 warps)
  uint64_t o_done[2];  // PV of tile u complete (MMA commit), u&1 selects the barrier
  uint64_t o_final;    // every PV complete (single use)
  uint64_t drain;      // every MMA complete (single use)
  uint64_t s_first;    // the first tile's QK^T complete (single use; MMA commit to both CTAs)
  uint32_t tmem_base;
  int abort;
  float red_max[2][2][128];  // [tile parity][warpgroup][row]: partial row maxima
                             // (partial row sums at the end)
};
static_assert(sizeof(Bars) <= kBarBytes, "barrier block too large");
static_assert(kSmemBytes <= 232448, "shared memory over the per-CTA limit");

// ---- CTA-pair helpers
__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
__device__ __forceinline__ void pair_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;\nbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
// The leader's copy of a barrier (shared-memory address with the pair bit
// cleared, as the 2-SM TMA and arrive forms expect).
__device__ __forceinline__ uint32_t leader_bar(const uint64_t* bar) { return smem_u32(bar) & 0xFEFFFFFFu; }
// One arrival per warp on a barrier of the leader CTA, once the warp's lanes
// have synchronised.  The softmax warps signal only tensor-memory accesses
// that every lane has already waited for (tcgen05.wait::ld / ::st, then
// tcgen05.fence::before_thread_sync), so the arrival needs no release
// semantics -- a release at cluster scope would cost ~700 cycles on the
// critical path of every tile.
__device__ __forceinline__ void arrive_leader(const uint64_t* bar) {
  __syncwarp();
  if ((threadIdx.x & 31) == 0)
    asm volatile("mbarrier.arrive.relaxed.cluster.shared::cluster.b64 _, [%0];" ::"r"(leader_bar(bar)) : "memory");
}

__device__ __forceinline__ uint32_t pack2(float lo, float hi, int dt) {
  if (dt == KCA_BF16) {
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&v);
  }
  __half2 v = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

// p = 2^(s cs + nmu) for the 64 scores of a half row (one FFMA, over pairs,
// and one MUFU op per score), packed as 16-bit pairs into pr; returns their sum.
template <int DT>
__device__ __forceinline__ float exp_pack(const float (&s)[64], float cs, float nmu, uint32_t (&pr)[32]) {
  const float2 cs2 = make_float2(cs, cs), nmu2 = make_float2(nmu, nmu);
  float2 acc2[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
#pragma unroll
  for (int c = 0; c < 32; ++c) {
    const float2 x = __ffma2_rn(make_float2(s[2 * c], s[2 * c + 1]), cs2, nmu2);
    const float p0 = ptx::ex2(x.x), p1 = ptx::ex2(x.y);
    acc2[c & 3] = __fadd2_rn(acc2[c & 3], make_float2(p0, p1));
    pr[c] = pack2(p0, p1, DT);
  }
  acc2[0] = __fadd2_rn(acc2[0], acc2[1]);
  acc2[2] = __fadd2_rn(acc2[2], acc2[3]);
  acc2[0] = __fadd2_rn(acc2[0], acc2[2]);
  return acc2[0].x + acc2[0].y;
}

// Named barrier of n threads that also returns whether v held in any of them.
__device__ __forceinline__ bool bar_red_or(int id, int n, bool v) {
  uint32_t r;
  asm volatile(
      "{\n .reg .pred pin, pout;\n setp.ne.u32 pin, %1, 0;\n bar.red.or.pred pout, %2, %3, pin;\n"
      " selp.u32 %0, 1, 0, pout;\n}"
      : "=r"(r)
      : "r"((uint32_t)v), "r"(id), "r"(n)
      : "memory");
  return r != 0;
}

__device__ __forceinline__ void named_sync(int id, int n) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(n) : "memory");
}

__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

template <int DT>
__global__ void __launch_bounds__(kThreads, 1)
    prefill_tc_kernel(const __grid_constant__ CUtensorMap tmk, const __grid_constant__ CUtensorMap tmv,
                      const __grid_constant__ CUtensorMap tmq, const __grid_constant__ CUtensorMap tmo,
                      const __grid_constant__ CUtensorMap tmpart,
                      const __grid_constant__ CUtensorMap tmpart_rag, const TcArgs a) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  const uint32_t raw_addr = smem_u32(smem_raw);
  const uint32_t pad = ((raw_addr + 1023u) & ~1023u) - raw_addr;
  unsigned char* smem = smem_raw + pad;
  const uint32_t sbase = raw_addr + pad;
  Bars* bars = reinterpret_cast<Bars*>(smem + kOffBar);
  volatile int* abort_flag = &bars->abort;
  DeviceStatus* status = reinterpret_cast<DeviceStatus*>(a.status);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_rank();           // 0: leader (issues the MMAs), 1: its peer
  const bool leader = rank == 0;
  const TcItemArg it = a.items[blockIdx.x >> 1];
  const int tile = 2 * it.pair + (int)rank;
  const bool ghost = tile >= a.plan.n_tiles;     // odd tile count: the peer of the last pair has no rows
  const int slot = it.slot[rank];
  const int n = it.kt_end - it.kt_begin;         // the same in both CTAs

  if (threadIdx.x == 0) {
    for (int i = 0; i < kKRing; ++i) {
      mbar_init(&bars->kfull[i], 1);
      mbar_init(&bars->kempty[i], 1);
    }
    for (int i = 0; i < kVRing; ++i) {
      mbar_init(&bars->vfull[i], 1);
      mbar_init(&bars->vempty[i], 1);
    }
    mbar_init(&bars->q_full, 1);
    mbar_init(&bars->s_full, 1);
    mbar_init(&bars->s_free, kPairArrivals);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bars->p_full[i], kPairArrivals);
      mbar_init(&bars->o_done[i], 1);
    }
    mbar_init(&bars->o_final, 1);
    mbar_init(&bars->drain, 1);
    mbar_init(&bars->s_first, 1);
    bars->abort = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    ptx::tmem_alloc_pair(smem_u32(&bars->tmem_base), kTmemCols);
    ptx::tmem_relinquish_pair();
  }
  // Both CTAs' barriers and TMEM exist before either touches the other's.
  ptx::fence_before_sync();
  pair_sync();
  ptx::fence_after_sync();
  const uint32_t tmem = bars->tmem_base;
  // Programmatic dependent launch: the set-up above overlaps the previous
  // kernel of the stream; global memory is touched only after this wait.
  asm volatile("griddepcontrol.wait;" ::: "memory");
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

  if (warp == 0 || warp == 2) {
    // ------------------------------------------------------------ producers
    // Each CTA loads its half of every K / V tile; the bytes complete on the
    // leader's full barrier, which the leader arms for both halves.
    if (lane == 0) {
      const bool is_k = warp == 0;
      uint64_t* full = is_k ? bars->kfull : bars->vfull;
      uint64_t* empty = is_k ? bars->kempty : bars->vempty;
      ptx::prefetch_tmap(is_k ? &tmk : &tmv);
      if (is_k) {
        // Q tile: 128 M rows x 256 dims as four 64-dim boxes (128-byte
        // swizzle), the A operand of Q K^T in this CTA's shared memory;
        // both CTAs' bytes complete on the leader's q_full.
        ptx::prefetch_tmap(&tmq);
        if (leader) mbar_arrive_expect_tx(&bars->q_full, 2 * kQBytes);
#pragma unroll
        for (int i = 0; i < 4; ++i)
          ptx::tma_load_2d_pair(sbase + kOffQ + i * kQBoxBytes, &tmq, 64 * i, tile * 128, leader_bar(&bars->q_full));
      } else {
        ptx::prefetch_tmap(&tmo);
        ptx::prefetch_tmap(&tmpart);
        ptx::prefetch_tmap(&tmpart_rag);
      }
      // V is first needed by the first PV, after the first softmax: its
      // loads wait until the first QK^T is done, so that Q and the first K
      // tiles have the SM's load bandwidth to themselves when an item
      // starts.  s_first has a single phase, so the wait cannot alias a
      // later one.
      bool ok = is_k || mbar_wait(&bars->s_first, 0, abort_flag, status, kSiteTcS);
      for (int t = 0; t < n && ok; ++t) {
        const int s = t % 2;
        if (t >= 2 && !mbar_wait(&empty[s], ((t / 2) - 1) & 1, abort_flag, status, kSiteTcEmpty)) {
          ok = false;
          break;
        }
        const int32_t key0 = (it.kt_begin + t) * kKeyTile;
        if (leader) mbar_arrive_expect_tx(&full[s], 2 * (is_k ? kKSlotBytes : kVSlotBytes));
        const uint32_t bar = leader_bar(&full[s]);
        if (is_k) {
          // keys [key0 + 64 rank, +64), all dims: four 64-dim chunks
          const uint32_t dst = sbase + kOffK + s * kKSlotBytes;
#pragma unroll
          for (int c = 0; c < 4; ++c)
            ptx::tma_load_2d_pair(dst + c * kKChunkBytes, &tmk, 64 * c, key0 + 64 * (int)rank, bar);
        } else {
          // dims [128 rank, +128), all 128 keys: box (key half h, dim block b) at (2h + b)
          const uint32_t dst = sbase + kOffV + s * kVSlotBytes;
#pragma unroll
          for (int h = 0; h < 2; ++h)
#pragma unroll
            for (int b = 0; b < 2; ++b)
              ptx::tma_load_2d_pair(dst + (2 * h + b) * kVBoxBytes, &tmv, 128 * (int)rank + 64 * b, key0 + 64 * h, bar);
        }
      }
      if (!ok) *abort_flag = 1;
    }
    __syncwarp();
  } else if (warp == 1) {
    // ----------------------------------------------------------------- MMA
    if (lane == 0 && leader) {
      constexpr uint32_t ab = DT == KCA_BF16 ? 1u : 0u;
      constexpr uint32_t id_qk = ptx::idesc_f16(ab, 256, kKeyTile, 0);
      constexpr uint32_t id_pv = ptx::idesc_f16(ab, 256, kDim, 1);
      // Descriptor bases; an operand at byte offset x from a base is the base
      // plus x >> 4 in the start-address field (addresses stay below 256 KiB).
      const uint64_t kd0 = ptx::sdesc_sw128(sbase + kOffK, 16, 1024);
      const uint64_t qd0 = ptx::sdesc_sw128(sbase + kOffQ, 16, 1024);
      const uint64_t vd0 = ptx::sdesc_sw128(sbase + kOffV, kVBoxBytes, 1024);
      const uint32_t s_full = smem_u32(&bars->s_full);
      bool ok = mbar_wait(&bars->q_full, 0, abort_flag, status, kSiteTcQ);
      ptx::fence_after_sync();
      auto pv = [&](int u) -> bool {
        if (!mbar_wait(&bars->p_full[u & 1], (u >> 1) & 1, abort_flag, status, kSiteTcP)) return false;
        const int s = u % 2;
        if (!mbar_wait(&bars->vfull[s], (u / 2) & 1, abort_flag, status, kSiteTcFull)) return false;
        ptx::fence_after_sync();
        const uint32_t pcol = tmem + kColP + 64 * (u & 1);
        const uint64_t vd = vd0 + (uint64_t)((s * kVSlotBytes) >> 4);
#pragma unroll
        for (int j = 0; j < 8; ++j)   // 16 keys per step: 8 TMEM columns of P; V key half j/4, rows 16 (j%4)
          ptx::mma_ts_pair(tmem + kColO, pcol + 8 * j,
                           vd + (uint64_t)(((j >> 2) * 2 * kVBoxBytes + (j & 3) * 16 * 128) >> 4), id_pv,
                           (u > 0 || j > 0) ? 1u : 0u);
        ptx::mma_commit_pair(smem_u32(&bars->vempty[s]), kPairMask);
        ptx::mma_commit_pair(smem_u32(&bars->o_done[u & 1]), kPairMask);
        return true;
      };
      for (int t = 0; t < n && ok; ++t) {
        if (t > 0) {
          ok = mbar_wait(&bars->s_free, (t - 1) & 1, abort_flag, status, kSiteTcS);
          if (!ok) break;
        }
        const int s = t % 2;
        ok = mbar_wait(&bars->kfull[s], (t / 2) & 1, abort_flag, status, kSiteTcFull);
        if (!ok) break;
        ptx::fence_after_sync();   // S was read by other threads' tcgen05.ld; K landed
        const uint64_t kd = kd0 + (uint64_t)((s * kKSlotBytes) >> 4);
#pragma unroll
        for (int k = 0; k < 16; ++k)   // 16 dims per step: chunk k/4, column group k%4
          ptx::mma_ss_pair(tmem + kColS, qd0 + (uint64_t)(((k >> 2) * kQBoxBytes + (k & 3) * 32) >> 4),
                           kd + (uint64_t)(((k >> 2) * kKChunkBytes + (k & 3) * 32) >> 4), id_qk, k > 0 ? 1u : 0u);
        ptx::mma_commit_pair(smem_u32(&bars->kempty[s]), kPairMask);
        ptx::mma_commit_pair(s_full, kPairMask);
        if (t == 0) ptx::mma_commit_pair(smem_u32(&bars->s_first), kPairMask);
        if (t > 0) ok = pv(t - 1);
      }
      if (ok) ok = pv(n - 1);
      if (ok) ptx::mma_commit_pair(smem_u32(&bars->o_final), kPairMask);
      // every MMA issued above has completed once this barrier flips
      ptx::mma_commit_pair(smem_u32(&bars->drain), kPairMask);
      mbar_wait(&bars->drain, 0, nullptr, status, kSiteTcDrain);
    }
    __syncwarp();
  } else if (warp >= 4) {
    // ------------------------------------------------------------- softmax
    const int wg = (warp - 4) >> 2;                  // key half of every S tile
    const int m = (warp & 3) * 32 + lane;            // TMEM lane == M row
    const uint32_t trow = tmem + ((uint32_t)((warp & 3) * 32) << 16);
    const int64_t row = (int64_t)tile * kRowTile + (m >> 3);
    const bool valid = row < a.plan.rows;
    const int64_t pos = a.plan.chunk_start + row;
    const int64_t lo = lo_of(pos, a.plan.window);

    const float cs = a.scale_log2;
    const uint32_t scol = kColS + 64 * wg;
    float m_ref = -INFINITY;  // reference max of the row, log2 units
    float l_sum = 0.f;        // this warpgroup's half of the row sum
    bool ok = true;
    for (int t = 0; t < n; ++t) {
      // Every thread runs every iteration (work is skipped after an abort) so
      // that both warpgroups always meet at the named barrier below.
      ok = __all_sync(0xffffffffu, ok && mbar_wait(&bars->s_full, t & 1, abort_flag, status, kSiteTcS));
      float s[64];
      if (ok) {
        ptx::fence_after_sync();
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
      ptx::fence_before_sync();
      arrive_leader(&bars->s_free);   // S may be overwritten by the next QK^T
      if (ok) {
        // keys outside [lo, pos] become -inf (scale > 0 keeps them there)
        const int64_t j0 = a.plan.kv_lo + (int64_t)(it.kt_begin + t) * kKeyTile + 64 * wg;
        if (j0 < lo || j0 + 63 > pos) {
#pragma unroll
          for (int c = 0; c < 64; ++c) {
            const int64_t j = j0 + c;
            if (j < lo || j > pos) s[c] = -INFINITY;
          }
        }
      }
      // Probabilities with the current reference first.  When their sum
      // over this half row is at most 2^8, none of them exceeds 2^8 and the
      // reference stands: no row max is needed, which is the common case
      // once a row has seen its first keys.  Otherwise -- the row's first
      // visible tile, a score past the reference by more than 2^8 in either
      // half, a NaN score -- every row of the pair of warpgroups takes the
      // max exchange below, exactly as if no probability had been taken.
      uint32_t pr[32];
      float lt = 0.f;
      const bool done = ok && m_ref != -INFINITY;
      bool redo = ok;
      if (done) {
        lt = exp_pack<DT>(s, cs, -m_ref, pr);
        redo = !(lt <= 256.f);
      }
      if (bar_red_or(2, kSoftmaxThreads, redo)) {
        float mloc = -INFINITY;
        if (ok) {
          float m8[8];
#pragma unroll
          for (int i = 0; i < 8; ++i) m8[i] = s[i];
#pragma unroll
          for (int c = 8; c < 64; ++c) m8[c & 7] = max_nan(m8[c & 7], s[c]);
#pragma unroll
          for (int i = 0; i < 4; ++i) m8[i] = max_nan(m8[i], m8[i + 4]);
          mloc = max_nan(max_nan(m8[0], m8[2]), max_nan(m8[1], m8[3]));
        }
        // The row max spans both warpgroups: exchange halves (buffer by tile parity).
        bars->red_max[t & 1][wg][m] = mloc;
        named_sync(1, kSoftmaxThreads);
        const float mraw = max_nan(mloc, bars->red_max[t & 1][wg ^ 1][m]);
        if (!ok) continue;
        const float mx = mraw == -INFINITY ? -INFINITY : mraw * cs;
        const bool need = mx > m_ref + kRescaleLog2;   // identical in both warpgroups
        const bool any_need = __any_sync(0xffffffffu, need);
        if (any_need) {
          const float alpha = need ? ptx::ex2(m_ref - mx) : 1.f;
          if (need) m_ref = mx;
          l_sum *= alpha;
          if (t > 0) {
            // PV of the previous tile must finish before O is rescaled; PV of
            // tile t-2 is known complete here (it preceded this tile's QK^T),
            // so the parity wait on barrier (t-1)&1 is unambiguous.
            ok = __all_sync(0xffffffffu, mbar_wait(&bars->o_done[(t - 1) & 1], ((t - 1) >> 1) & 1,
                                                   abort_flag, status, kSiteTcO));
            if (!ok) continue;
            ptx::fence_after_sync();
#pragma unroll 1
            for (int c = 0; c < 4; ++c) {
              uint32_t r[32];
              ptx::tmem_ld32(trow + kColO + 128 * wg + 32 * c, r);
              ptx::tmem_wait_ld();
#pragma unroll
              for (int i = 0; i < 32; ++i) r[i] = __float_as_uint(__uint_as_float(r[i]) * alpha);
              ptx::tmem_st32(trow + kColO + 128 * wg + 32 * c, r);
            }
            ptx::tmem_wait_st();
          }
        }
        // A sum past 2^8 whose max stayed within 2^8 of the reference keeps
        // the probabilities already taken.
        if (!done || need) lt = exp_pack<DT>(s, cs, m_ref == -INFINITY ? 0.f : -m_ref, pr);
      }
      if (!ok) continue;
      l_sum += lt;
      // P row m, keys [64 wg, 64 wg + 64): 32 TMEM columns of 16-bit pairs in
      // buffer t&1.  PV of tile t-2, the last reader of that buffer, has
      // completed: it preceded QK^T of this tile, whose completion s_full signalled.
      ptx::tmem_st32(trow + kColP + 64 * (t & 1) + 32 * wg, pr);
      ptx::tmem_wait_st();
      ptx::fence_before_sync();
      arrive_leader(&bars->p_full[t & 1]);
    }
    ok = __all_sync(0xffffffffu, ok && mbar_wait(&bars->o_final, 0, abort_flag, status, kSiteTcO));
    // Row sum over both halves (the buffer of tile parity n&1 is free again).
    bars->red_max[n & 1][wg][m] = l_sum;
    named_sync(1, kSoftmaxThreads);
    const float l_tot = l_sum + bars->red_max[n & 1][wg ^ 1][m];
    // Epilogue: O (scaled by 1/l, or raw for a partial) goes from TMEM to
    // shared memory as eight 32-column boxes with 128-byte swizzle (the K/V
    // rings are free once every PV is done), then out by TMA stores: the
    // tile's 128 rows are one contiguous block of out or of the partials,
    // and rows past the chunk fall outside the map and are not written.
    // Boxes c and 4 + c (the two warpgroups' halves) leave as soon as both
    // are written, while the next ones are; the issuing thread then waits
    // only until shared memory has been read -- the grid's completion makes
    // the stores visible to the kernels after it.  A ragged tile's partial
    // keeps only its valid rows: the first rows of every box (the swizzle
    // pattern repeats every 8 rows).
    const void* omap = slot < 0             ? static_cast<const void*>(&tmo)
                       : tile == a.rag_tile ? static_cast<const void*>(&tmpart_rag)
                                            : static_cast<const void*>(&tmpart);
    const int32_t oy = (slot < 0 ? tile : slot) * 128;
    if (ok) {
      ptx::fence_after_sync();
      if (slot >= 0 && wg == 0 && valid) {
        a.part_ml[((int64_t)slot * 128 + m) * 2 + 0] = m_ref;
        a.part_ml[((int64_t)slot * 128 + m) * 2 + 1] = l_tot;
      }
    }
    const float f = slot < 0 ? 1.f / l_tot : 1.f;
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      if (ok) {
        uint32_t r[32];
        ptx::tmem_ld32(trow + kColO + 128 * wg + 32 * c, r);
        ptx::tmem_wait_ld();
        unsigned char* box = smem + (4 * wg + c) * kOBoxBytes + m * 128;
#pragma unroll
        for (int i = 0; i < 8; ++i)
          *reinterpret_cast<float4*>(box + ((i ^ (m & 7)) << 4)) =
              make_float4(__uint_as_float(r[4 * i]) * f, __uint_as_float(r[4 * i + 1]) * f,
                          __uint_as_float(r[4 * i + 2]) * f, __uint_as_float(r[4 * i + 3]) * f);
        fence_proxy_async_smem();   // generic-proxy stores -> visible to the TMA unit
      }
      ptx::fence_before_sync();
      named_sync(1, kSoftmaxThreads);
      if (ok && !ghost && threadIdx.x == 4 * 32) {
        ptx::tma_store_2d(omap, 32 * c, oy, sbase + c * kOBoxBytes);
        ptx::tma_store_2d(omap, 32 * (4 + c), oy, sbase + (4 + c) * kOBoxBytes);
        ptx::bulk_commit();
      }
    }
    // shared memory stays allocated until the stores have read it
    if (ok && !ghost && threadIdx.x == 4 * 32) ptx::bulk_wait_read_all();
  }

  // No CTA of the pair leaves while MMAs may still read its shared memory
  // or its peer may still arrive on its barriers.
  ptx::fence_before_sync();
  pair_sync();
  if (warp == 1) {
    ptx::fence_after_sync();
    ptx::tmem_dealloc_pair(tmem, kTmemCols);
  }
}


// Log-sum-exp merge of the items of each split row tile.  WPR warps per M
// row (8 / WPR rows per CTA, grid (tiles, 16 WPR)); warp sub of a row takes
// the contiguous items [sub n, sub n + n) of the tile's ns, lane k owning
// dims [8k, 8k+8), with the (m, l) and acc of NB items in flight at once
// and an online rescale across groups of NB.  NB = 4 when no tile has more
// than four items: its registers then let the whole grid (6,144 rows of a
// 768-row chunk) be resident in one wave, where NB = 8 needs two.  With WPR > 1 the warps'
// partials of a row are combined in shared memory in sub order.  Items and
// sub-ranges are combined in slot order, so the result is the same bits on
// every call.  Many items per tile (few tiles in the chunk) take more warps
// per row, so that no warp waits on more than a few load round trips.
template <int WPR, int NB>
__global__ void __launch_bounds__(256) merge_tc_kernel(const TcArgs a) {
  asm volatile("griddepcontrol.wait;" ::: "memory");
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  constexpr int RPC = 8 / WPR;   // rows per CTA
  const int tile = blockIdx.x;
  const int ns = a.tile_items[tile];
  if (ns <= 1) return;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int m = blockIdx.y * RPC + warp / WPR, sub = warp % WPR;
  const bool row_ok = (int64_t)tile * kRowTile + (m >> 3) < a.plan.rows;
  if (WPR == 1 && !row_ok) return;   // the whole warp leaves together
  const int per = (ns + WPR - 1) / WPR;
  const int sb = sub * per, se = min(ns, sb + per);
  const int64_t r0 = (int64_t)a.tile_first_slot[tile] * 128 + m;    // item s: row r0 + 128 s
  float M = -INFINITY, L = 0.f;
  float4 A0 = make_float4(0.f, 0.f, 0.f, 0.f), A1 = A0;
  for (int s0 = sb; row_ok && s0 < se; s0 += NB) {
    float mv[NB], lv[NB];
    float4 v0[NB], v1[NB];
#pragma unroll
    for (int j = 0; j < NB; ++j) {
      const int64_t r = r0 + (int64_t)(s0 + j) * 128;
      const bool in = s0 + j < se;
      mv[j] = in ? a.part_ml[r * 2] : -INFINITY;
      lv[j] = in ? a.part_ml[r * 2 + 1] : 0.f;
      const float4* src = reinterpret_cast<const float4*>(a.part_acc + r * kDim + 8 * lane);
      v0[j] = in ? src[0] : make_float4(0.f, 0.f, 0.f, 0.f);
      v1[j] = in ? src[1] : make_float4(0.f, 0.f, 0.f, 0.f);
    }
    float Mn = M;
#pragma unroll
    for (int j = 0; j < NB; ++j) Mn = max_nan(Mn, mv[j]);
    const float mu = Mn == -INFINITY ? 0.f : Mn;
    const float alpha = exp2f(M - mu);   // m is in log2 units
    L *= alpha;
    A0.x *= alpha; A0.y *= alpha; A0.z *= alpha; A0.w *= alpha;
    A1.x *= alpha; A1.y *= alpha; A1.z *= alpha; A1.w *= alpha;
#pragma unroll
    for (int j = 0; j < NB; ++j) {
      const float f = exp2f(mv[j] - mu);
      L += f * lv[j];
      A0.x += f * v0[j].x; A0.y += f * v0[j].y; A0.z += f * v0[j].z; A0.w += f * v0[j].w;
      A1.x += f * v1[j].x; A1.y += f * v1[j].y; A1.z += f * v1[j].z; A1.w += f * v1[j].w;
    }
    M = Mn;
  }
  if (WPR > 1) {
    __shared__ float4 sa[8][2][32];
    __shared__ float sml[8][2];
    sa[warp][0][lane] = A0;
    sa[warp][1][lane] = A1;
    if (lane == 0) {
      sml[warp][0] = M;
      sml[warp][1] = L;
    }
    __syncthreads();
    if (sub != 0 || !row_ok) return;
#pragma unroll
    for (int j = 1; j < WPR; ++j) {
      const float mj = sml[warp + j][0], lj = sml[warp + j][1];
      const float4 b0 = sa[warp + j][0][lane], b1 = sa[warp + j][1][lane];
      const float Mn = max_nan(M, mj);
      const float mu = Mn == -INFINITY ? 0.f : Mn;
      const float fa = exp2f(M - mu), fb = exp2f(mj - mu);
      L = fa * L + fb * lj;
      A0.x = fa * A0.x + fb * b0.x; A0.y = fa * A0.y + fb * b0.y;
      A0.z = fa * A0.z + fb * b0.z; A0.w = fa * A0.w + fb * b0.w;
      A1.x = fa * A1.x + fb * b1.x; A1.y = fa * A1.y + fb * b1.y;
      A1.z = fa * A1.z + fb * b1.z; A1.w = fa * A1.w + fb * b1.w;
      M = Mn;
    }
  }
  const float inv = 1.f / L;
  float4* dst = reinterpret_cast<float4*>(a.out + ((int64_t)tile * 128 + m) * kDim + 8 * lane);
  dst[0] = make_float4(A0.x * inv, A0.y * inv, A0.z * inv, A0.w * inv);
  dst[1] = make_float4(A1.x * inv, A1.y * inv, A1.z * inv, A1.w * inv);
}

template <int DT>
cudaError_t launch_t(const CUtensorMap& tmk, const CUtensorMap& tmv, const CUtensorMap& tmq,
                     const CUtensorMap& tmo, const CUtensorMap& tmpart, const CUtensorMap& tmpart_rag,
                     const TcArgs& a, cudaStream_t stream) {
  static std::atomic<bool> attr_set[64];   // per device; zero-initialised
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  if (!attr_set[dev]) {
    cudaError_t e = cudaFuncSetAttribute(prefill_tc_kernel<DT>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
    if (e != cudaSuccess) return e;
    attr_set[dev] = true;
  }
  // Both kernels allow programmatic dependent launch (see griddepcontrol);
  // the attention kernel runs as clusters of two CTAs (one per item).
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  attr[1].id = cudaLaunchAttributeClusterDimension;
  attr[1].val.clusterDim.x = 2;
  attr[1].val.clusterDim.y = 1;
  attr[1].val.clusterDim.z = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2 * a.plan.n_items);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = kSmemBytes;
  cfg.stream = stream;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  cudaError_t e = cudaLaunchKernelEx(&cfg, prefill_tc_kernel<DT>, tmk, tmv, tmq, tmo, tmpart, tmpart_rag, a);
  if (e != cudaSuccess || a.plan.n_slots == 0) return e;
  int ns_max = 0;
  for (int32_t t = 0; t < a.plan.n_tiles && t < kTcMaxTiles; ++t)
    ns_max = a.tile_items[t] > ns_max ? a.tile_items[t] : ns_max;
  const int wpr = ns_max <= 8 ? 1 : ns_max <= 16 ? 2 : ns_max <= 32 ? 4 : 8;
  cfg.gridDim = dim3(a.plan.n_tiles, 16 * wpr);
  cfg.blockDim = dim3(256);
  cfg.dynamicSmemBytes = 0;
  cfg.numAttrs = 1;   // no cluster
  if (ns_max <= 4) return cudaLaunchKernelEx(&cfg, merge_tc_kernel<1, 4>, a);
  if (wpr == 1) return cudaLaunchKernelEx(&cfg, merge_tc_kernel<1, 8>, a);
  if (wpr == 2) return cudaLaunchKernelEx(&cfg, merge_tc_kernel<2, 8>, a);
  if (wpr == 4) return cudaLaunchKernelEx(&cfg, merge_tc_kernel<4, 8>, a);
  return cudaLaunchKernelEx(&cfg, merge_tc_kernel<8, 8>, a);
}

}  // namespace

bool fill_tc_tables(TcArgs& a) {
  // One pass over the pairs: O(pairs + items), no per-item plan walk.
  if (a.plan.n_tiles < 1 || a.plan.n_tiles > kTcMaxTiles || a.plan.n_items < 1 || a.plan.n_items > kTcMaxItems)
    return false;
  int32_t idx = 0, slot = 0;
  for (int32_t q = 0; q < a.plan.n_pairs && 2 * q < kTcMaxTiles; ++q) {
    int32_t kb, ke;
    tc_pair_keys(a.plan, q, &kb, &ke);
    const int32_t n = ke - kb;
    const int32_t s = (int32_t)cdiv(n, a.plan.per_item);
    const int32_t nt = tc_pair_tiles(a.plan, q);
    for (int32_t r = 0; r < nt; ++r) {
      a.tile_items[2 * q + r] = (int16_t)s;
      a.tile_first_slot[2 * q + r] = (int16_t)(slot + r * s);
    }
    for (int32_t k = 0; k < s && idx < kTcMaxItems; ++k, ++idx) {
      a.items[idx].kt_begin = kb + tc_split_at(n, s, k);
      a.items[idx].kt_end = kb + tc_split_at(n, s, k + 1);
      a.items[idx].pair = (int16_t)q;
      a.items[idx].slot[0] = (int16_t)(s > 1 ? slot + k : -1);
      a.items[idx].slot[1] = (int16_t)(s > 1 && nt == 2 ? slot + s + k : -1);
    }
    if (s > 1) slot += s * nt;
  }
  // The tables must agree with the plan the workspace was sized for: every
  // item filled, every partial slot inside the n_slots the workspace holds,
  // every key tile inside the keys the K / V maps cover.
  if (idx != a.plan.n_items || slot != a.plan.n_slots) return false;
  const int64_t key_tiles = cdiv(a.plan.ctx_len - a.plan.kv_lo, (int64_t)kKeyTile);
  for (int32_t i = 0; i < idx; ++i) {
    const TcItemArg& it = a.items[i];
    if (it.kt_begin < 0 || it.kt_end <= it.kt_begin || it.kt_end > key_tiles || it.pair < 0 ||
        2 * it.pair >= a.plan.n_tiles)
      return false;
    for (int r = 0; r < 2; ++r)
      if (it.slot[r] < -1 || it.slot[r] >= a.plan.n_slots) return false;
  }
  for (int32_t t = 0; t < a.plan.n_tiles; ++t)
    if (a.tile_items[t] > 1 && (a.tile_first_slot[t] < 0 || a.tile_first_slot[t] + a.tile_items[t] > a.plan.n_slots))
      return false;
  return true;
}

cudaError_t launch_prefill_tc(int dtype, const CUtensorMap& tmk, const CUtensorMap& tmv,
                              const CUtensorMap& tmq, const CUtensorMap& tmo, const CUtensorMap& tmpart,
                              const CUtensorMap& tmpart_rag,
                              const TcArgs& a, cudaStream_t stream) {
  if (dtype == KCA_BF16) return launch_t<KCA_BF16>(tmk, tmv, tmq, tmo, tmpart, tmpart_rag, a, stream);
  if (dtype == KCA_F16) return launch_t<KCA_F16>(tmk, tmv, tmq, tmo, tmpart, tmpart_rag, a, stream);
  return cudaErrorInvalidValue;
}

}  // namespace kca

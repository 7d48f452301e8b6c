// kca_prefill_tc.cu -- chunked causal prefill on the sm_100a tensor cores.
//
// The pages' design (Karume v0.12.0 release notes, "Performance", item 1):
// for plans of 16 or more chunk rows, QK and PV run on a GEMM tile skeleton
// so that each K / V row is read once per row tile instead of once per query
// row.  Here one CTA takes one work item -- a row tile of 16 positions x 8
// heads (M = 128: the 8 heads share their single KV head) and a run of
// 128-key tiles -- and fuses the three stages the pages keep apart (QK,
// softmax statistics, PV), so no score matrix ever reaches memory.
//
// Warp roles (12 warps):
//   warp 0      TMA producer of K: each 128-key tile as four 64-dim chunks
//               (128 rows x 128 B, 128-byte swizzle), two chunks per slot of
//               a 2-slot ring
//   warp 1      TMEM allocator and the single MMA-issuing thread
//   warp 2      TMA producer of V: 64-key halves (four 64 x 64 boxes) into a
//               2-slot ring
//   warps 4-7   softmax warpgroup 0: keys 0-63 of every S tile
//   warps 8-11  softmax warpgroup 1: keys 64-127
//   Thread m of a softmax warpgroup owns TMEM lane m, i.e. M row m.
//
// Tensor memory (512 columns x 128 lanes of 32 bits):
//   [  0,128)  Q tile as 16-bit pairs: the A operand of S = Q K^T
//   [128,256)  S (f32, 128 keys), released as soon as both warpgroups hold
//              their half in registers, so QK^T of the next tile overlaps
//              the softmax of this one
//   [256,512)  O accumulator (f32, 256 dims)
// P (16-bit) goes to shared memory, double-buffered, as the A operand of
// O += P V.  Shapes per instruction: QK^T M128 N128 K16, PV M128 N256 K16;
// both keep the tensor pipe at full rate from a single issuing thread.
//
// The softmax keeps a reference max per row and rescales O (in TMEM) only
// when a score exceeds it by more than 2^8, so probabilities stay <= 256 and
// the O round trip is rare; the result is exact up to rounding whatever
// reference is used.  Work items of a split row tile write (m, l, O)
// partials that merge_tc_kernel combines by log-sum-exp (kca_merge.cuh).
#include <cuda.h>
#include <cuda_runtime.h>

#include "kca_common.cuh"
#include "kca_merge.cuh"
#include "kca_plan.h"
#include "kca_tc.h"
#include "kca_tc_ptx.cuh"

namespace kca {
namespace {

constexpr int kThreads = 384;
constexpr int kKRing = 2;                              // K slots of two 64-dim chunks
constexpr int kVRing = 2;                              // V half-tile slots
constexpr int kKChunkBytes = kKeyTile * 64 * 2;        // 128 keys x 64 dims: 16 KiB
constexpr int kKSlotBytes = 2 * kKChunkBytes;          // two chunks: 32 KiB
constexpr int kVBoxBytes = 64 * 64 * 2;                // 64 keys x 64 dims: 8 KiB
constexpr int kVHalfBytes = 4 * kVBoxBytes;            // 64 keys x 256 dims: 32 KiB
constexpr int kPBytes = 128 * kKeyTile * 2;            // 128 rows x 128 keys: 32 KiB
constexpr int kOffK = 0;
constexpr int kOffV = kOffK + kKRing * kKSlotBytes;    // 64 KiB
constexpr int kOffP = kOffV + kVRing * kVHalfBytes;    // 128 KiB
constexpr int kOffBar = kOffP + 2 * kPBytes;           // 192 KiB
constexpr int kQBoxBytes = 128 * 64 * 2;               // Q: 128 M rows x 64 dims, 16 KiB
constexpr int kQBytes = 4 * kQBoxBytes;                // the whole Q tile over the P buffers
constexpr int kOBoxBytes = 128 * 32 * 4;               // O: 128 M rows x 32 f32, 16 KiB
static_assert(kQBytes == 2 * kPBytes, "Q tile fills the P buffers");
static_assert(8 * kOBoxBytes <= kOffP, "O tile fits the K/V rings");
constexpr int kBarBytes = 4096;
constexpr int kSmemBytes = kOffBar + kBarBytes + 1024; // + alignment slack
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColQ = 0, kColS = 128, kColO = 256;
constexpr float kRescaleLog2 = 8.f;  // rescale O once a score passes the reference by 2^8
constexpr int kSoftmaxThreads = 256;

struct Bars {
  uint64_t kfull[kKRing], kempty[kKRing];
  uint64_t vfull[kVRing], vempty[kVRing];
  uint64_t q_tma;      // Q tile landed in shared memory (TMA, over the P buffers)
  uint64_t q_full;     // Q in TMEM (256 softmax threads)
  uint64_t s_full;     // S of the current tile computed (MMA commit)
  uint64_t s_free;     // S copied to registers by all 256 softmax threads
  uint64_t p_full[2];  // P of tile t in buffer t&1 written, O corrected (256 threads)
  uint64_t o_done[2];  // PV of tile u complete (MMA commit), u&1 selects the barrier
  uint64_t o_final;    // every PV complete (single use)
  uint64_t drain;      // every MMA complete (single use, MMA thread)
  uint32_t tmem_base;
  int abort;
  float red_max[2][2][128];  // [tile parity][warpgroup][row]: partial row maxima
                             // (partial row sums at the end)
};
static_assert(sizeof(Bars) <= kBarBytes, "barrier block too large");
static_assert(kSmemBytes <= 232448, "shared memory over the per-CTA limit");

__device__ __forceinline__ uint32_t pack2(float lo, float hi, int dt) {
  if (dt == KCA_BF16) {
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&v);
  }
  __half2 v = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
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
                      const __grid_constant__ CUtensorMap tmpart, const TcArgs a) {
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
  const TcItemArg it = a.items[blockIdx.x];
  const int n = it.kt_end - it.kt_begin;
  if (n <= 0) return;  // the host never launches such a CTA

  if (threadIdx.x == 0) {
    for (int i = 0; i < kKRing; ++i) {
      mbar_init(&bars->kfull[i], 1);
      mbar_init(&bars->kempty[i], 1);
    }
    for (int i = 0; i < kVRing; ++i) {
      mbar_init(&bars->vfull[i], 1);
      mbar_init(&bars->vempty[i], 1);
    }
    mbar_init(&bars->q_tma, 1);
    mbar_init(&bars->q_full, kSoftmaxThreads);
    mbar_init(&bars->s_full, 1);
    mbar_init(&bars->s_free, kSoftmaxThreads);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bars->p_full[i], kSoftmaxThreads);
      mbar_init(&bars->o_done[i], 1);
    }
    mbar_init(&bars->o_final, 1);
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
  // Programmatic dependent launch: the set-up above overlaps the previous
  // kernel of the stream; global memory is touched only after this wait.
  // The next kernel may be scheduled as soon as SMs free up.
  asm volatile("griddepcontrol.wait;" ::: "memory");
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

  if (warp == 0 || warp == 2) {
    // ------------------------------------------------------------ producers
    if (lane == 0) {
      const bool is_k = warp == 0;
      const int ring = is_k ? kKRing : kVRing;
      uint64_t* full = is_k ? bars->kfull : bars->vfull;
      uint64_t* empty = is_k ? bars->kempty : bars->vempty;
      ptx::prefetch_tmap(is_k ? &tmk : &tmv);
      if (is_k) {
        // Q tile: 128 M rows x 256 dims as four 64-dim boxes (128-byte
        // swizzle) into the P buffers, which are unused until the first P.
        ptx::prefetch_tmap(&tmq);
        mbar_arrive_expect_tx(&bars->q_tma, kQBytes);
#pragma unroll
        for (int i = 0; i < 4; ++i)
          ptx::tma_load_2d(sbase + kOffP + i * kQBoxBytes, &tmq, 64 * i, it.tile * 128, smem_u32(&bars->q_tma));
      } else {
        ptx::prefetch_tmap(&tmo);
        ptx::prefetch_tmap(&tmpart);
      }
      const int per_tile = 2;   // K: two slots of two 64-dim chunks, V: two 64-key halves
      int e = 0;
      bool ok = true;
      for (int t = 0; t < n && ok; ++t) {
        for (int c = 0; c < per_tile; ++c) {
          const int slot = e % ring;
          if (e >= ring &&
              !mbar_wait(&empty[slot], ((e / ring) - 1) & 1, abort_flag, status, kSiteTcEmpty)) {
            ok = false;
            break;
          }
          const uint32_t bar = smem_u32(&full[slot]);
          const int32_t key0 = (it.kt_begin + t) * kKeyTile;
          if (is_k) {
            mbar_arrive_expect_tx(&full[slot], kKSlotBytes);
            const uint32_t dst = sbase + kOffK + slot * kKSlotBytes;
            ptx::tma_load_2d(dst, &tmk, 128 * c, key0, bar);
            ptx::tma_load_2d(dst + kKChunkBytes, &tmk, 128 * c + 64, key0, bar);
          } else {
            mbar_arrive_expect_tx(&full[slot], kVHalfBytes);
            const uint32_t dst = sbase + kOffV + slot * kVHalfBytes;
#pragma unroll
            for (int i = 0; i < 4; ++i) ptx::tma_load_2d(dst + i * kVBoxBytes, &tmv, 64 * i, key0 + 64 * c, bar);
          }
          ++e;
        }
      }
      if (!ok) {  // aborted: let every issued copy land before the CTA exits
        for (int s = 0; s < ring && s < e; ++s) {
          const int last = ((e - 1 - s) / ring) * ring + s;
          mbar_wait(&full[s], (last / ring) & 1, nullptr, status, kSiteTcDrain);
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
      // Descriptor bases; an operand at byte offset x from a base is the base
      // plus x >> 4 in the start-address field (addresses stay below 256 KiB).
      const uint64_t kd0 = ptx::sdesc_sw128(sbase + kOffK, 16, 1024);
      const uint64_t pd0 = ptx::sdesc_sw128(sbase + kOffP, 16, 1024);
      const uint64_t vd0 = ptx::sdesc_sw128(sbase + kOffV, kVBoxBytes, 1024);
      int ek = 0, ev = 0;
      bool ok = mbar_wait(&bars->q_full, 0, abort_flag, status, kSiteTcQ);
      ptx::fence_after_sync();
      auto pv = [&](int u) -> bool {
        if (!mbar_wait(&bars->p_full[u & 1], (u >> 1) & 1, abort_flag, status, kSiteTcP)) return false;
        ptx::fence_after_sync();
        const uint64_t pd = pd0 + (uint64_t)(((u & 1) * kPBytes) >> 4);
        for (int h = 0; h < 2; ++h) {
          const int slot = ev % kVRing;
          if (!mbar_wait(&bars->vfull[slot], (ev / kVRing) & 1, abort_flag, status, kSiteTcFull)) return false;
          const uint64_t vd = vd0 + (uint64_t)((slot * kVHalfBytes) >> 4);
#pragma unroll
          for (int j = 0; j < 4; ++j)
            ptx::mma_ss(tmem + kColO, pd + (uint64_t)((h * (kPBytes / 2) + j * 32) >> 4),
                        vd + (uint64_t)((j * 16 * 128) >> 4), id_pv, (u > 0 || h > 0 || j > 0) ? 1u : 0u);
          ptx::mma_commit(smem_u32(&bars->vempty[slot]));
          ++ev;
        }
        ptx::mma_commit(smem_u32(&bars->o_done[u & 1]));
        return true;
      };
      for (int t = 0; t < n && ok; ++t) {
        if (t > 0) {
          ok = mbar_wait(&bars->s_free, (t - 1) & 1, abort_flag, status, kSiteTcS);
          if (!ok) break;
          ptx::fence_after_sync();   // S was read by other threads' tcgen05.ld
        }
        for (int c = 0; c < 2 && ok; ++c) {
          const int slot = ek % kKRing;
          ok = mbar_wait(&bars->kfull[slot], (ek / kKRing) & 1, abort_flag, status, kSiteTcFull);
          if (!ok) break;
          const uint64_t kd = kd0 + (uint64_t)((slot * kKSlotBytes) >> 4);
#pragma unroll
          for (int j = 0; j < 8; ++j)   // K-steps 8c .. 8c+7: chunk j/4 of the slot
            ptx::mma_ts(tmem + kColS, tmem + kColQ + (8 * c + j) * 8,
                        kd + (uint64_t)(((j >> 2) * kKChunkBytes + (j & 3) * 32) >> 4), id_qk,
                        (c > 0 || j > 0) ? 1u : 0u);
          ptx::mma_commit(smem_u32(&bars->kempty[slot]));
          ++ek;
        }
        if (!ok) break;
        ptx::mma_commit(smem_u32(&bars->s_full));
        if (t > 0) ok = pv(t - 1);
      }
      if (ok) ok = pv(n - 1);
      if (ok) ptx::mma_commit(smem_u32(&bars->o_final));
      // every MMA issued above has completed once this barrier flips
      ptx::mma_commit(smem_u32(&bars->drain));
      mbar_wait(&bars->drain, 0, nullptr, status, kSiteTcDrain);
    }
    __syncwarp();
  } else if (warp >= 4) {
    // ------------------------------------------------------------- softmax
    const int wg = (warp - 4) >> 2;                  // key half of every S tile
    const int m = (warp & 3) * 32 + lane;            // TMEM lane == M row
    const uint32_t trow = tmem + ((uint32_t)((warp & 3) * 32) << 16);
    const int64_t row = (int64_t)it.tile * kRowTile + (m >> 3);
    const bool valid = row < a.plan.rows;
    const int64_t pos = a.plan.chunk_start + row;
    const int64_t lo = lo_of(pos, a.plan.window);

    // Q row (row, head m & 7), dims [128 wg, 128 wg + 128), from the TMA
    // boxes in shared memory into TMEM (rows past the chunk arrive as zeros).
    {
      const bool qok = mbar_wait(&bars->q_tma, 0, abort_flag, status, kSiteTcQ);
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        uint32_t r[32];
        const unsigned char* box = smem + kOffP + (2 * wg + c) * kQBoxBytes + m * 128;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const uint4 v = qok ? *reinterpret_cast<const uint4*>(box + ((i ^ (m & 7)) << 4)) : make_uint4(0, 0, 0, 0);
          r[4 * i] = v.x; r[4 * i + 1] = v.y; r[4 * i + 2] = v.z; r[4 * i + 3] = v.w;
        }
        ptx::tmem_st32(trow + kColQ + 64 * wg + 32 * c, r);
      }
      ptx::tmem_wait_st();
      ptx::fence_before_sync();
      mbar_arrive(&bars->q_full);
    }

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
      mbar_arrive(&bars->s_free);   // S may be overwritten by the next QK^T
      float mloc = -INFINITY;
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
      // p = 2^(s*scale*log2e - m_ref): one FFMA and one MUFU op per score.
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
      // P row m, keys [64 wg, 64 wg + 64): buffer t&1, K-major with 128-byte
      // swizzle (16-byte unit j of row m at unit j ^ (m & 7)).
      unsigned char* prow = smem + kOffP + (t & 1) * kPBytes + wg * (kPBytes / 2) + (m >> 3) * 1024 + (m & 7) * 128;
#pragma unroll
      for (int j = 0; j < 8; ++j)
        *reinterpret_cast<uint4*>(prow + ((j ^ (m & 7)) << 4)) =
            make_uint4(pr[4 * j], pr[4 * j + 1], pr[4 * j + 2], pr[4 * j + 3]);
      fence_proxy_async_smem();   // generic-proxy stores -> visible to the tensor cores
      ptx::fence_before_sync();
      mbar_arrive(&bars->p_full[t & 1]);
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
    if (ok) {
      ptx::fence_after_sync();
      if (it.slot >= 0 && wg == 0 && valid) {
        a.part_ml[((int64_t)it.slot * 128 + m) * 2 + 0] = m_ref;
        a.part_ml[((int64_t)it.slot * 128 + m) * 2 + 1] = l_tot;
      }
      const float f = it.slot < 0 ? 1.f / l_tot : 1.f;
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        uint32_t r[32];
        ptx::tmem_ld32(trow + kColO + 128 * wg + 32 * c, r);
        ptx::tmem_wait_ld();
        unsigned char* box = smem + (4 * wg + c) * kOBoxBytes + m * 128;
#pragma unroll
        for (int i = 0; i < 8; ++i)
          *reinterpret_cast<float4*>(box + ((i ^ (m & 7)) << 4)) =
              make_float4(__uint_as_float(r[4 * i]) * f, __uint_as_float(r[4 * i + 1]) * f,
                          __uint_as_float(r[4 * i + 2]) * f, __uint_as_float(r[4 * i + 3]) * f);
      }
      fence_proxy_async_smem();   // generic-proxy stores -> visible to the TMA unit
    }
    ptx::fence_before_sync();
    named_sync(1, kSoftmaxThreads);
    if (ok && threadIdx.x == 4 * 32) {
      const void* map = it.slot < 0 ? static_cast<const void*>(&tmo) : static_cast<const void*>(&tmpart);
      const int32_t y = (it.slot < 0 ? (int32_t)it.tile : (int32_t)it.slot) * 128;
#pragma unroll
      for (int j = 0; j < 8; ++j) ptx::tma_store_2d(map, 32 * j, y, sbase + j * kOBoxBytes);
      ptx::bulk_commit();
      ptx::bulk_wait_all();   // shared memory stays allocated until the stores are done
    }
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
  asm volatile("griddepcontrol.wait;" ::: "memory");
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
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
cudaError_t launch_t(const CUtensorMap& tmk, const CUtensorMap& tmv, const CUtensorMap& tmq,
                     const CUtensorMap& tmo, const CUtensorMap& tmpart, const TcArgs& a, cudaStream_t stream) {
  static bool attr_set[64] = {false};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  if (!attr_set[dev]) {
    cudaError_t e = cudaFuncSetAttribute(prefill_tc_kernel<DT>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
    if (e != cudaSuccess) return e;
    attr_set[dev] = true;
  }
  // Both kernels allow programmatic dependent launch (see griddepcontrol).
  cudaLaunchAttribute pdl;
  pdl.id = cudaLaunchAttributeProgrammaticStreamSerialization;
  pdl.val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(a.plan.n_items);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = kSmemBytes;
  cfg.stream = stream;
  cfg.attrs = &pdl;
  cfg.numAttrs = 1;
  cudaError_t e = cudaLaunchKernelEx(&cfg, prefill_tc_kernel<DT>, tmk, tmv, tmq, tmo, tmpart, a);
  if (e != cudaSuccess || a.plan.n_slots == 0) return e;
  const int ns = a.plan.max_split;
  const int w = ns > 8 ? 8 : (ns > 4 ? 4 : (ns > 2 ? 2 : 1));
  cfg.gridDim = dim3(a.plan.n_tiles, 16 * w);
  cfg.blockDim = dim3(256);
  cfg.dynamicSmemBytes = 0;
  if (w == 8) return cudaLaunchKernelEx(&cfg, merge_tc_kernel<8>, a);
  if (w == 4) return cudaLaunchKernelEx(&cfg, merge_tc_kernel<4>, a);
  if (w == 2) return cudaLaunchKernelEx(&cfg, merge_tc_kernel<2>, a);
  return cudaLaunchKernelEx(&cfg, merge_tc_kernel<1>, a);
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
                              const CUtensorMap& tmq, const CUtensorMap& tmo, const CUtensorMap& tmpart,
                              const TcArgs& a, cudaStream_t stream) {
  if (dtype == KCA_BF16) return launch_t<KCA_BF16>(tmk, tmv, tmq, tmo, tmpart, a, stream);
  if (dtype == KCA_F16) return launch_t<KCA_F16>(tmk, tmv, tmq, tmo, tmpart, a, stream);
  return cudaErrorInvalidValue;
}

}  // namespace kca

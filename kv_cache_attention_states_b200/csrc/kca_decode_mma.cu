// kca_decode_mma.cu -- split-context single-row attention with 16-bit K/V on
// the tensor cores (mma.sync m16n8k16, f32 accumulation): decode, and the
// prefill rows that the tcgen05 kernel does not take.
//
// With 8 query heads sharing one KV head a decode step is a small GEMM per
// key block (M = 8 heads), not a GEMV.  On the CUDA cores the eight dot
// products, their warp-shuffle reductions and the f16 -> f32 conversions
// cost ~130 instructions per key row per warp; here a 64-key stage costs ~80
// instructions per warp, so the kernel is left with the HBM stream it is
// meant to be bound by.  Prior art on the pages: the "parallel" QK and PV
// reductions of Karume's one-row plans (v0.12.0 release notes,
// "Performance", items 2-3).
//
// Precision: the query (any dtype) is split into a 16-bit high part and a
// 16-bit remainder, stacked as rows 0-7 and 8-15 of the A operand, so the
// accumulator rows g and g+8 hold q_hi.k and q_lo.k for head g and their sum
// carries ~16 (bf16) to ~22 (f16) bits of the query.  P is split the same way
// for the PV product.  Accumulation is f32.
//
// One CTA = one split of one unit; warps 0-7 compute, warp 8 issues the TMA
// loads.  The splits of a unit run as clusters of 2, 4 or 8 CTAs that merge
// their partials through distributed shared memory at the end; when a unit
// has several clusters, the CTA that finishes last (atomic ticket, no
// waiting) merges the cluster partials, so no separate merge kernel runs.
// The launch allows programmatic dependent launch: the prologue overlaps the
// previous kernel of the stream.
//
// A stage is 64 keys: K and V each as four 64-dim boxes of 64 rows with
// 128-byte swizzle (conflict-free ldmatrix), 64 KiB per stage, 3 stages.
// Stage flow (warp w): S for keys 8w..8w+7 (16 MMAs over d = 256), stage max
// per head exchanged through shared memory, lazy rescale of O, P written to
// shared memory as 16 rows (hi, lo) x 64 keys, then O[:, 32w .. 32w+31] +=
// P V (16 MMAs).  Rows past the split's end are zeroed in shared memory, so
// whatever the cache holds there never reaches the output.
#include <atomic>
#include <cuda.h>
#include <cuda_runtime.h>

#include "kca_common.cuh"
#include "kca_merge.cuh"
#include "kca_plan.h"
#include "kca_rows.h"

namespace kca {
namespace {

constexpr int kDWarps = 8;
constexpr int kDThreads = (kDWarps + 1) * 32;
constexpr int kDStageKeys = 64;
constexpr int kDStages = 3;
constexpr int kDBoxBytes = 64 * 64 * 2;              // 64 rows x 64 dims, 8 KiB
constexpr int kDHalfBytes = 4 * kDBoxBytes;          // K or V of one stage: 32 KiB
constexpr int kDStageBytes = 2 * kDHalfBytes;        // 64 KiB
constexpr int kDPRow = 144;                          // P row pitch: 128 B + 16 B pad
constexpr int kDQRow = 528;                          // Q row pitch: 512 B + 16 B pad
constexpr int kDOffBar = kDStages * kDStageBytes;    // 192 KiB
constexpr float kDLog2e = 1.4426950408889634f;
constexpr float kDRescale = 5.545177444479562f;      // 8 ln 2
constexpr int kDPrefetchKeys = 512;                  // keys per split prefetched into L2 early

struct DBars {
  uint64_t full[kDStages];
  uint64_t empty[kDStages];
  uint64_t rx;                           // the partials this CTA owns have arrived (st.async bytes)
  int abort;
  float red[kDWarps][8];                 // per-warp stage max (then row sums) per head
  int last;                              // this CTA holds the last ticket of its unit
  __align__(16) unsigned char p[16 * kDPRow];   // P: rows 0-7 hi, 8-15 lo, 64 keys
  __align__(16) unsigned char qs[16 * kDQRow];  // Q: rows 0-7 hi, 8-15 lo, 256 dims (int8 K: 8 rows of codes)
  float sq[8];                           // int8 K: the query's per-head scales
  // Partials this CTA receives for the heads it owns: slot src * (8 / C) + i
  // holds CTA src's reference max (natural units), row sum and unnormalised
  // output of head rank + i * C.  Written by the cluster's CTAs (distributed
  // shared memory stores); own space, so no copy still landing after an
  // abort can overwrite it.
  float rm[8];
  float rl[8];
  float ro[8][256];
};
constexpr int kDSmemBytes = kDOffBar + (int)sizeof(DBars) + 1024;

template <int KT>
__device__ __forceinline__ uint32_t pack16(float lo, float hi) {
  if (KT == KCA_BF16) {
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&v);
  }
  __half2 v = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}
template <int KT>
__device__ __forceinline__ float2 unpack16(uint32_t u) {
  if (KT == KCA_BF16) return __bfloat1622float2(*reinterpret_cast<__nv_bfloat162*>(&u));
  return __half22float2(*reinterpret_cast<__half2*>(&u));
}

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t (&r)[4]) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t (&r)[4]) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}

// D = A(16x16) B(16x8) + D, row.col, f32 accumulation.
template <int KT>
__device__ __forceinline__ void mma16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                         uint32_t b1) {
  if (KT == KCA_BF16) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, "
        "{%8, %9}, {%0, %1, %2, %3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
  } else {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, "
        "{%8, %9}, {%0, %1, %2, %3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
  }
}

__device__ __forceinline__ void tma2d(uint32_t dst, const void* map, int32_t x, int32_t y, uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3}], [%4];" ::"r"(dst),
      "l"(map), "r"(x), "r"(y), "r"(bar)
      : "memory");
}

// Byte offset of (row, dim) inside a stage half: four 64-dim boxes of 64 rows,
// 128-byte swizzle (16-byte unit u of row r stored at unit u ^ (r & 7)).
__device__ __forceinline__ uint32_t swz(int row, int dim) {
  const int unit = (dim & 63) >> 3;
  return (uint32_t)((dim >> 6) * kDBoxBytes + row * 128 + ((unit ^ (row & 7)) << 4));
}


// Byte offset of code byte c (0..255) of key row `row` in the packed int8 K
// half of a stage: two 128-code boxes of 64 rows, 128-byte swizzle.  The
// rows' f32 scales follow at kDQ8ScaleOff, 16 bytes per row (unswizzled).
__device__ __forceinline__ uint32_t swz8(int row, int c) {
  return (uint32_t)((c >> 7) * kDBoxBytes + row * 128 + ((((c & 127) >> 4) ^ (row & 7)) << 4));
}
constexpr int kDQ8ScaleOff = 2 * kDBoxBytes;                 // 16 KiB into the K half
constexpr int kDQ8StageTx = 2 * kDBoxBytes + 64 * 16 + kDHalfBytes;   // codes + scales + V

// D = A(16x32) B(32x8) + D on int8 codes, exact int32 accumulation.
__device__ __forceinline__ void mma_s8(int (&d)[4], uint32_t a0, uint32_t a2, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k32.row.col.s32.s8.s8.s32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %2, %3};"
      : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
      : "r"(a0), "r"(0u), "r"(a2), "r"(0u), "r"(b0), "r"(b1));
}

// int8 code of x under scale sx (round half to even of the f32 quotient,
// clamped to +-127; 0 unless sx is finite and > 0) -- the quantisation of
// attn_quantize_k.
__device__ __forceinline__ uint32_t dq8_code(float x, float sx) {
  if (!(sx > 0.f) || !(sx <= 3.402823466e38f)) return 0u;
  int c = __float2int_rn(__fdiv_rn(x, sx));
  c = c > 127 ? 127 : (c < -127 ? -127 : c);
  return static_cast<uint32_t>(c) & 0xffu;
}

// Split cluster barrier: every thread of every CTA of the cluster arrives,
// and waits for the others' arrival.
__device__ __forceinline__ void cluster_arrive() {
  asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory");
}
__device__ __forceinline__ void cluster_wait() {
  asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory");
}
// Asynchronous store into the shared memory of CTA `cta` of the cluster, at
// the offset that `local` has in this CTA's; its bytes complete on that
// CTA's barrier `rx` (a plain store without a cluster).
__device__ __forceinline__ uint32_t peer_addr(const void* local, uint32_t cta) {
  uint32_t remote;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(remote) : "r"(smem_u32(local)), "r"(cta));
  return remote;
}
__device__ __forceinline__ void st_peer(float* local, uint32_t cta, float v, int C, uint64_t* rx) {
  if (C == 1) {
    *local = v;
    return;
  }
  asm volatile("st.async.shared::cluster.mbarrier::complete_tx::bytes.f32 [%0], %1, [%2];" ::"r"(peer_addr(local, cta)),
               "f"(v), "r"(peer_addr(rx, cta))
               : "memory");
}
__device__ __forceinline__ void st_peer2(float* local, uint32_t cta, float v0, float v1, int C, uint64_t* rx) {
  if (C == 1) {
    *reinterpret_cast<float2*>(local) = make_float2(v0, v1);
    return;
  }
  asm volatile("st.async.shared::cluster.mbarrier::complete_tx::bytes.v2.f32 [%0], {%1, %2}, [%3];" ::"r"(
                   peer_addr(local, cta)),
               "f"(v0), "f"(v1), "r"(peer_addr(rx, cta))
               : "memory");
}

// Final merge of one owned head (slot hi: head rank + hi C) over the nclus
// cluster partials, W consecutive dims per thread (dims [W jd, W jd + W)).
// The first batch of partial accumulators is requested before (m, l) of all
// partials go to shared memory, so the two round trips overlap; each warp
// then reduces (M, L) of its head itself and each thread sums its dims over
// the partials in slot order.  L2-coherent loads: other SMs wrote the
// partials.  NB partials per batch of loads (the smallest batch that holds
// all of them, up to 32 / W; loads past nclus repeat partial 0 and are
// weighted 0).  Every thread of the block calls this (it holds a bar.sync).
template <int W, int NB>
__device__ __forceinline__ void merge_cluster_partials(const RowsArgs& a, float* sm_m, float* sm_l, int64_t u0,
                                                       int unit, int rank, int C, int nh, int d, int nclus,
                                                       int lane) {
  const int per = kDim / W;              // threads per head
  const int hi = d / per, jd = d % per;
  const int h = rank + hi * C;
  const float* base = a.cpart_acc + (u0 + h) * kDim + W * jd;   // partial c at + c * kHeads * kDim
  float v[NB][W];
  auto load_batch = [&](int c0) {
#pragma unroll
    for (int t = 0; t < NB; ++t) {
      const int c = c0 + t;
      const float* src = base + (int64_t)(c < nclus ? c : 0) * kHeads * kDim;
      if (W >= 4) {
#pragma unroll
        for (int e = 0; e < W; e += 4) {
          const float4 x = __ldcg(reinterpret_cast<const float4*>(src + e));
          v[t][e] = x.x; v[t][(e + 1) % W] = x.y; v[t][(e + 2) % W] = x.z; v[t][(e + 3) % W] = x.w;
        }
      } else if (W == 2) {
        const float2 x = __ldcg(reinterpret_cast<const float2*>(src));
        v[t][0] = x.x; v[t][1 % W] = x.y;
      } else {
        v[t][0] = __ldcg(src);
      }
    }
  };
  load_batch(0);
  for (int c = d; c < nclus; c += kDim) {
    for (int i = 0; i < nh; ++i) {
      const float2 ml = __ldcg(reinterpret_cast<const float2*>(a.cpart_ml) + u0 + (int64_t)c * kHeads + rank + i * C);
      sm_m[i * kDim + c] = ml.x;
      sm_l[i * kDim + c] = ml.y;
    }
  }
  asm volatile("bar.sync 2, %0;" ::"n"(kDim) : "memory");
  const float* pm = sm_m + hi * kDim;
  const float* pl = sm_l + hi * kDim;
  float mw = -INFINITY;
  for (int c = lane; c < nclus; c += 32) mw = max_nan(mw, pm[c]);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) mw = max_nan(mw, __shfl_xor_sync(0xffffffffu, mw, o));
  const float M = mw, mu = M == -INFINITY ? 0.f : M;
  float lw = 0.f;
  for (int c = lane; c < nclus; c += 32) lw += exp2f((pm[c] - mu) * kDLog2e) * pl[c];
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) lw += __shfl_xor_sync(0xffffffffu, lw, o);
  const float L = lw;
  float acc[W];
#pragma unroll
  for (int e = 0; e < W; ++e) acc[e] = 0.f;
  for (int c0 = 0;; c0 += NB) {
#pragma unroll
    for (int t = 0; t < NB; ++t) {
      const int c = c0 + t;
      const float f = c < nclus ? exp2f((pm[c < nclus ? c : 0] - mu) * kDLog2e) : 0.f;
#pragma unroll
      for (int e = 0; e < W; ++e) acc[e] += f * v[t][e];
    }
    if (c0 + NB >= nclus) break;
    load_batch(c0 + NB);
  }
  float* dst = a.out + ((int64_t)unit * kHeads + h) * kDim + W * jd;
#pragma unroll
  for (int e = 0; e < W; ++e) dst[e] = rows_final(a, acc[e], M, L);
  if (jd == 0) rows_write_ml(a, unit, h, M, L);
}

template <int W>
__device__ __forceinline__ void merge_cluster_partials_nb(const RowsArgs& a, float* sm_m, float* sm_l, int64_t u0,
                                                          int unit, int rank, int C, int nh, int d, int nclus,
                                                          int lane) {
  if (nclus <= 4) merge_cluster_partials<W, 4>(a, sm_m, sm_l, u0, unit, rank, C, nh, d, nclus, lane);
  else if (nclus <= 8) merge_cluster_partials<W, 8>(a, sm_m, sm_l, u0, unit, rank, C, nh, d, nclus, lane);
  else if (W > 1 || nclus <= 16) merge_cluster_partials<W, 16>(a, sm_m, sm_l, u0, unit, rank, C, nh, d, nclus, lane);
  else merge_cluster_partials<W, 32>(a, sm_m, sm_l, u0, unit, rank, C, nh, d, nclus, lane);
}

// KT: K element type, or KCA_I8 for packed int8 K rows (the quantised-dot
// variant: QK on int8 codes with exact int32 MMA, scaled by the query's and
// the key's scales); VT: V element type (16-bit); tms: the int8 rows' scale
// column (unused otherwise).
template <int QT, int KT, int VT = KT>
__global__ void __launch_bounds__(kDThreads, 1)
    decode_mma_kernel(const __grid_constant__ CUtensorMap tmk, const __grid_constant__ CUtensorMap tmv,
                      const __grid_constant__ CUtensorMap tms, const RowsArgs a) {
  constexpr bool kQ8 = KT == KCA_I8;
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  const uint32_t raw_addr = smem_u32(smem_raw);
  const uint32_t pad = ((raw_addr + 1023u) & ~1023u) - raw_addr;
  unsigned char* smem = smem_raw + pad;
  const uint32_t sbase = raw_addr + pad;
  DBars* bars = reinterpret_cast<DBars*>(smem + kDOffBar);
  volatile int* abort_flag = &bars->abort;
  DeviceStatus* status = reinterpret_cast<DeviceStatus*>(a.status);

  const int C = a.cluster;                 // CTAs per cluster along the splits (1, 2, 4 or 8)
  const int unit = blockIdx.y;
  const int split = blockIdx.x;
  const int rank = split % C, clus = split / C;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  // Device context lengths may come from the previous kernel of the stream:
  // with them, the dependency wait comes before they are read.
  if (a.ctx_dev != nullptr) asm volatile("griddepcontrol.wait;" ::: "memory");
  int64_t seq_base;
  const int64_t pos = rows_unit_pos(a, unit, split == 0 && threadIdx.x == 0, &seq_base);
  int64_t lo;
  const int64_t nkeys = rows_keys(a, pos, &lo);
  const int32_t split_len = rows_split_len(a, nkeys, kDStageKeys);
  const int32_t nsplit = rows_n_splits(nkeys, split_len);
  const int nclus = (nsplit + C - 1) / C;
  if (clus >= nclus) return;               // the whole cluster leaves together
  bool active = split < nsplit && nkeys > 0;
  const int64_t kbeg = lo + (int64_t)split * split_len;
  int64_t kend = kbeg + split_len;
  if (kend > lo + nkeys) kend = lo + nkeys;
  // cache row of key p: base_row + p (a shard's row 0 is position key_begin)
  const int64_t base_row = seq_base - a.key_begin;
  // bounds-checked builds: the unit's plan fits the host's (cluster-partial
  // slots and tickets; a failure is the same for every CTA of the unit,
  // which all leave together), and a split whose rows would leave the cache
  // counts as empty
  if (!KCA_IN_BOUNDS(nsplit <= a.max_splits && nclus <= a.max_clusters &&
                         (nclus == 1 || ((int64_t)(unit + 1) * a.max_clusters <= a.part_slots &&
                                         unit < KCA_MAX_CHUNK_ROWS)),
                     status, kSiteBoundsDecode, (unsigned)unit))
    return;
  if (active && !KCA_IN_BOUNDS(base_row + kbeg >= 0 && base_row + kend <= a.cache_rows, status,
                               kSiteBoundsDecode, (unsigned)unit))
    active = false;
  const int n_stage = active ? (int)cdiv(kend - kbeg, kDStageKeys) : 0;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kDStages; ++s) {
      mbar_init(&bars->full[s], 1);
      mbar_init(&bars->empty[s], kDWarps);
    }
    // The partials of the heads this CTA owns arrive as st.async bytes from
    // every CTA of the cluster: C x (8 / C) x (256 + 2) floats.
    mbar_init(&bars->rx, 1);
    if (C > 1) mbar_arrive_expect_tx(&bars->rx, kHeads * (kDim + 2) * 4);
    bars->abort = 0;
    fence_barrier_init();
  }
  if (threadIdx.x == kDWarps * 32) {
    // Descriptors are kernel parameters: fetch them early.  The first stages
    // of the split are prefetched into L2 as well, overlapping the previous
    // kernel of the stream; a prefetch binds no value, so rows that kernel
    // still writes are read after the wait below all the same.
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmk)) : "memory");
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmv)) : "memory");
    if (kQ8) asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tms)) : "memory");
    if (active) {
      int64_t n = kend - kbeg;
      if (n > kDPrefetchKeys) n = kDPrefetchKeys;
      constexpr int kKRow = kQ8 ? KCA_I8_ROW_BYTES : kDim * 2;
      const uint32_t kbytes = (uint32_t)(n * kKRow), vbytes = (uint32_t)(n * kDim * 2);
      asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(static_cast<const char*>(a.k) +
                                                                      (base_row + kbeg) * kKRow),
                   "r"(kbytes) : "memory");
      asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(static_cast<const char*>(a.v) +
                                                                      (base_row + kbeg) * (kDim * 2)),
                   "r"(vbytes) : "memory");
    }
  }
  __syncthreads();
  // Distributed shared memory may be written only once every CTA of the
  // cluster runs: arrive now, wait just before the first remote store.
  if (C > 1) cluster_arrive();
  // Everything above overlaps the previous kernel of the stream (programmatic
  // dependent launch); inputs, outputs and workspace are touched only below.
  asm volatile("griddepcontrol.wait;" ::: "memory");

  const int nh = kHeads / C;               // heads each CTA owns in the merge

  if (warp == kDWarps) {
    // ---------------------------------------------------------------- producer
    if (lane == 0 && active) {
      int issued = 0;
      for (int i = 0; i < n_stage; ++i) {
        const int slot = i % kDStages;
        if (i >= kDStages &&
            !mbar_wait(&bars->empty[slot], ((i / kDStages) - 1) & 1, abort_flag, status, kSiteRowsEmpty))
          break;
        const uint32_t kst = sbase + slot * kDStageBytes;
        const uint32_t bar = smem_u32(&bars->full[slot]);
        const int32_t row0 = (int32_t)(base_row + kbeg + (int64_t)i * kDStageKeys);
        if constexpr (kQ8) {
          mbar_arrive_expect_tx(&bars->full[slot], kDQ8StageTx);
          tma2d(kst, &tmk, 0, row0, bar);                  // codes 0..127
          tma2d(kst + kDBoxBytes, &tmk, 128, row0, bar);   // codes 128..255
          tma2d(kst + kDQ8ScaleOff, &tms, kDim, row0, bar);   // scale (+ padding)
#pragma unroll
          for (int c = 0; c < 4; ++c) tma2d(kst + kDHalfBytes + c * kDBoxBytes, &tmv, 64 * c, row0, bar);
        } else {
          mbar_arrive_expect_tx(&bars->full[slot], kDStageBytes);
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            tma2d(kst + c * kDBoxBytes, &tmk, 64 * c, row0, bar);
            tma2d(kst + kDHalfBytes + c * kDBoxBytes, &tmv, 64 * c, row0, bar);
          }
        }
        issued = i + 1;
      }
      if (issued < n_stage) {  // aborted: let every issued copy land
        for (int s = 0; s < kDStages && s < issued; ++s) {
          const int last = ((issued - 1 - s) / kDStages) * kDStages + s;
          mbar_wait(&bars->full[s], (last / kDStages) & 1, nullptr, status, kSiteRowsFull);
        }
      }
    }
    __syncwarp();
  } else if (!active) {
    // no key in this split (or in the whole row): an empty partial
    if (C > 1) cluster_wait();
    if (threadIdx.x < kHeads) {
      const int h = threadIdx.x;
      st_peer(&bars->rm[rank * nh + h / C], h % C, -INFINITY, C, &bars->rx);
      st_peer(&bars->rl[rank * nh + h / C], h % C, 0.f, C, &bars->rx);
    }
    for (int i = threadIdx.x; i < kHeads * kDim; i += kDWarps * 32) {
      const int h = i / kDim;
      st_peer(&bars->ro[rank * nh + h / C][i % kDim], h % C, 0.f, C, &bars->rx);
    }
  } else {
    // ------------------------------------------------------------------ compute
    const int g = lane >> 2, tig = lane & 3;
    // A operand of S = Q K^T: rows 0-7 the 16-bit high parts of the 8 heads,
    // rows 8-15 the remainders; per k-step: (g, 2tig), (g+8, 2tig), (g, 2tig+8), (g+8, 2tig+8).
    uint32_t qa[kQ8 ? 1 : 16][4];
    // int8 K: the A operand of S = Q K^T is the 8 heads' int8 codes (rows
    // 8-15 zero); per 32-dim k-step thread (g, tig) holds bytes 4 tig .. and
    // 16 + 4 tig .. of head g.
    uint32_t qa8[kQ8 ? 8 : 1][2];
    float sq_g = 0.f;
    {
      // Stage the split query once, coalesced (thread t: 8 dims of head
      // t / 32), then every warp takes its A fragments with ldmatrix.
      const int h = threadIdx.x >> 5, d0 = 8 * (threadIdx.x & 31);
      float x[8];
      load8<QT>(static_cast<const char*>(a.q) +
                    ((int64_t)unit * kHeads * kDim + h * kDim + d0) * ElemBytes<QT>::value,
                x);
      if constexpr (kQ8) {
        // the head's scale amax * f32(1/127) over its 256 dims (warp h holds head h)
        float am = fabsf(x[0]);
  #pragma unroll
        for (int j = 1; j < 8; ++j) am = max_nan(am, fabsf(x[j]));
  #pragma unroll
        for (int o = 16; o > 0; o >>= 1) am = max_nan(am, __shfl_xor_sync(0xffffffffu, am, o));
        const float sx = am * (1.0f / 127.0f);
        if ((threadIdx.x & 31) == 0) bars->sq[h] = sx;
        const uint32_t w0 = dq8_code(x[0], sx) | (dq8_code(x[1], sx) << 8) | (dq8_code(x[2], sx) << 16) |
                            (dq8_code(x[3], sx) << 24);
        const uint32_t w1 = dq8_code(x[4], sx) | (dq8_code(x[5], sx) << 8) | (dq8_code(x[6], sx) << 16) |
                            (dq8_code(x[7], sx) << 24);
        *reinterpret_cast<uint2*>(bars->qs + h * kDim + d0) = make_uint2(w0, w1);
        asm volatile("bar.sync 1, %0;" ::"n"(kDWarps * 32) : "memory");
  #pragma unroll
        for (int ks = 0; ks < 8; ++ks) {
          qa8[ks][0] = *reinterpret_cast<const uint32_t*>(bars->qs + g * kDim + 32 * ks + 4 * tig);
          qa8[ks][1] = *reinterpret_cast<const uint32_t*>(bars->qs + g * kDim + 32 * ks + 16 + 4 * tig);
        }
        sq_g = bars->sq[g];
      } else {
        uint32_t hi[4], lo[4];
  #pragma unroll
        for (int j = 0; j < 4; ++j) {
          hi[j] = pack16<KT>(x[2 * j], x[2 * j + 1]);
          const float2 f = unpack16<KT>(hi[j]);
          lo[j] = pack16<KT>(x[2 * j] - f.x, x[2 * j + 1] - f.y);
        }
        *reinterpret_cast<uint4*>(bars->qs + h * kDQRow + d0 * 2) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
        *reinterpret_cast<uint4*>(bars->qs + (h + 8) * kDQRow + d0 * 2) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
        asm volatile("bar.sync 1, %0;" ::"n"(kDWarps * 32) : "memory");
        const int mi = lane >> 3;
        const uint32_t qrow = smem_u32(bars->qs) + (8 * (mi & 1) + (lane & 7)) * kDQRow + 8 * (mi >> 1) * 2;
  #pragma unroll
        for (int ks = 0; ks < 16; ++ks) ldsm_x4(qrow + 32 * ks, qa[ks]);
      }
    }
    float o[4][4];
  #pragma unroll
    for (int i = 0; i < 4; ++i)
  #pragma unroll
      for (int j = 0; j < 4; ++j) o[i][j] = 0.f;
    float m_ref = -INFINITY;  // reference max of head g (natural units)
    float l_part = 0.f;
    const float scale = a.scale;
    const uint32_t pbase = smem_u32(bars->p);
    bool ok = true;

    for (int i = 0; i < n_stage; ++i) {
      const int slot = i % kDStages;
      ok = __all_sync(0xffffffffu, ok && mbar_wait(&bars->full[slot], (i / kDStages) & 1, abort_flag,
                                                   status, kSiteRowsFull));
      const int64_t k0 = kbeg + (int64_t)i * kDStageKeys;
      const int cnt = (int)((kend - k0) < kDStageKeys ? (kend - k0) : kDStageKeys);
      const uint32_t kst = sbase + slot * kDStageBytes;
      const uint32_t vst = kst + kDHalfBytes;
      float sx0 = -INFINITY, sx1 = -INFINITY;
      if (ok) {
        if (cnt < kDStageKeys) {  // V rows past the split's end -> 0
          unsigned char* vrows = smem + slot * kDStageBytes + kDHalfBytes;
          for (int idx = threadIdx.x; idx < (kDStageKeys - cnt) * 32; idx += kDWarps * 32) {
            const int row = cnt + (idx >> 5), u = idx & 31;
            *reinterpret_cast<uint4*>(vrows + (u >> 3) * kDBoxBytes + row * 128 + (u & 7) * 16) =
                make_uint4(0, 0, 0, 0);
          }
        }
        const int kr = 8 * warp + (lane & 7);
        const int kk0 = 8 * warp + 2 * tig;
        if constexpr (kQ8) {
          // exact integer dot products of the codes, two chains
          int iacc[2][4] = {{0, 0, 0, 0}, {0, 0, 0, 0}};
  #pragma unroll
          for (int kc = 0; kc < 4; ++kc) {
            uint32_t b[4];
            ldsm_x4(kst + swz8(kr, 64 * kc + 16 * (lane >> 3)), b);
            mma_s8(iacc[0], qa8[2 * kc][0], qa8[2 * kc][1], b[0], b[1]);
            mma_s8(iacc[1], qa8[2 * kc + 1][0], qa8[2 * kc + 1][1], b[2], b[3]);
          }
          const unsigned char* sc = smem + slot * kDStageBytes + kDQ8ScaleOff;
          const float sk0 = *reinterpret_cast<const float*>(sc + kk0 * 16);
          const float sk1 = *reinterpret_cast<const float*>(sc + (kk0 + 1) * 16);
          sx0 = kk0 < cnt ? static_cast<float>(iacc[0][0] + iacc[1][0]) * ((sq_g * sk0) * scale) : -INFINITY;
          sx1 = kk0 + 1 < cnt ? static_cast<float>(iacc[0][1] + iacc[1][1]) * ((sq_g * sk1) * scale) : -INFINITY;
        } else {
          // Four independent accumulation chains over d (shorter latency).
          float sacc[4][4];
  #pragma unroll
          for (int c = 0; c < 4; ++c)
  #pragma unroll
            for (int j = 0; j < 4; ++j) sacc[c][j] = 0.f;
  #pragma unroll
          for (int ks2 = 0; ks2 < 8; ++ks2) {
            uint32_t b[4];
            ldsm_x4(kst + swz(kr, 32 * ks2 + 8 * (lane >> 3)), b);
            mma16816<KT>(sacc[(2 * ks2) & 3], qa[2 * ks2], b[0], b[1]);
            mma16816<KT>(sacc[(2 * ks2 + 1) & 3], qa[2 * ks2 + 1], b[2], b[3]);
          }
          float st[4];
  #pragma unroll
          for (int j = 0; j < 4; ++j) st[j] = (sacc[0][j] + sacc[1][j]) + (sacc[2][j] + sacc[3][j]);
          sx0 = kk0 < cnt ? (st[0] + st[2]) * scale : -INFINITY;
          sx1 = kk0 + 1 < cnt ? (st[1] + st[3]) * scale : -INFINITY;
        }
      }
      float mw = max_nan(sx0, sx1);
      mw = max_nan(mw, __shfl_xor_sync(0xffffffffu, mw, 1));
      mw = max_nan(mw, __shfl_xor_sync(0xffffffffu, mw, 2));
      if (tig == 0) bars->red[warp][g] = mw;
      asm volatile("bar.sync 1, %0;" ::"n"(kDWarps * 32) : "memory");
      float ms = bars->red[0][g];
  #pragma unroll
      for (int w = 1; w < kDWarps; ++w) ms = max_nan(ms, bars->red[w][g]);
      if (ok) {
        if (ms > m_ref + kDRescale) {  // lazy rescale: rows g and g+8 are both head g
          const float alpha = exp2f((m_ref - ms) * kDLog2e);
          m_ref = ms;
          l_part *= alpha;
  #pragma unroll
          for (int nt = 0; nt < 4; ++nt)
  #pragma unroll
            for (int j = 0; j < 4; ++j) o[nt][j] *= alpha;
        }
        const float mu = m_ref == -INFINITY ? 0.f : m_ref;
        const float p0 = exp2f((sx0 - mu) * kDLog2e);
        const float p1 = exp2f((sx1 - mu) * kDLog2e);
        l_part += p0 + p1;
        const uint32_t hi = pack16<VT>(p0, p1);
        const float2 f = unpack16<VT>(hi);
        const uint32_t lo16 = pack16<VT>(p0 - f.x, p1 - f.y);
        const int key = 8 * warp + 2 * tig;
        *reinterpret_cast<uint32_t*>(bars->p + g * kDPRow + key * 2) = hi;
        *reinterpret_cast<uint32_t*>(bars->p + (g + 8) * kDPRow + key * 2) = lo16;
      }
      asm volatile("bar.sync 1, %0;" ::"n"(kDWarps * 32) : "memory");   // P and zeroed rows visible
      if (ok) {
        const int mi = lane >> 3;
  #pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
          uint32_t af[4];
          ldsm_x4(pbase + (8 * (mi & 1) + (lane & 7)) * kDPRow + (16 * kk + 8 * (mi >> 1)) * 2, af);
          const int key = 16 * kk + 8 * (mi & 1) + (lane & 7);
  #pragma unroll
          for (int pair = 0; pair < 2; ++pair) {
            uint32_t vb[4];
            ldsm_x4_t(vst + swz(key, 32 * warp + 16 * pair + 8 * (mi >> 1)), vb);
            mma16816<VT>(o[2 * pair], af, vb[0], vb[1]);
            mma16816<VT>(o[2 * pair + 1], af, vb[2], vb[3]);
          }
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->empty[slot]);
    }

    // Row sums: lanes of one head, then warps (the stage-max slots are free again).
    l_part += __shfl_xor_sync(0xffffffffu, l_part, 1);
    l_part += __shfl_xor_sync(0xffffffffu, l_part, 2);
    if (tig == 0) bars->red[warp][g] = l_part;
    asm volatile("bar.sync 1, %0;" ::"n"(kDWarps * 32) : "memory");
    float L = 0.f;
#pragma unroll
    for (int w = 0; w < kDWarps; ++w) L += bars->red[w][g];
    if (!ok || *abort_flag) {
      m_ref = NAN;   // an aborted split poisons its row; the status word says why
      L = NAN;
    }
    // Push the partial of head g to the CTA that owns it (rows g and g+8 of
    // the accumulator are the high and low parts).
    if (C > 1) cluster_wait();
    const int owner = g % C, slot = rank * nh + g / C;
#pragma unroll
    for (int nt = 0; nt < 4; ++nt) {
      const int d = 32 * warp + 8 * nt + 2 * tig;
      st_peer2(&bars->ro[slot][d], owner, o[nt][0] + o[nt][2], o[nt][1] + o[nt][3], C, &bars->rx);
    }
    if (warp == 0 && tig == 0) {
      st_peer(&bars->rm[slot], owner, m_ref, C, &bars->rx);
      st_peer(&bars->rl[slot], owner, L, C, &bars->rx);
    }
  }
  if (warp == kDWarps && C > 1) cluster_wait();   // the producer keeps the barrier phases in step
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

  // ------------------------------------------------------------ merge
  // CTA rank r owns heads r, r+C, ... (C divides 8) and receives the C
  // partials of each by st.async into its own shared memory; once their
  // bytes have completed on its barrier rx, no CTA touches another's shared
  // memory again, so no cluster barrier is needed before any CTA leaves.
  // Thread d owns dim d.  With one cluster per unit the merge of the C
  // partials is the result.  Otherwise each CTA publishes its
  // heads' cluster partials and takes a ticket of (unit, rank); the CTA that
  // draws the last one merges every cluster's partials of those heads.
  // Nothing waits on another CTA, so the order in which clusters run does not
  // matter.
  if (C > 1) {
    // every partial of the owned heads has landed: C sources x 8 / C heads x
    // (256 + 2) floats
    if (threadIdx.x < kDim) mbar_wait(&bars->rx, 0, nullptr, status, kSiteRowsFull);
  } else {
    __syncthreads();
  }
  if (threadIdx.x < kDim) {
    const int d = threadIdx.x;
    for (int i = 0; i < nh; ++i) {
      const int h = rank + i * C;
      float mv[8], lv[8], ov[8];
#pragma unroll
      for (int src = 0; src < 8; ++src) {
        const bool in = src < C;
        mv[src] = in ? bars->rm[src * nh + i] : -INFINITY;
        lv[src] = in ? bars->rl[src * nh + i] : 0.f;
        ov[src] = in ? bars->ro[src * nh + i][d] : 0.f;
      }
      float M = mv[0];
#pragma unroll
      for (int src = 1; src < 8; ++src) M = max_nan(M, mv[src]);
      const float mu = M == -INFINITY ? 0.f : M;
      float L = 0.f, O = 0.f;
#pragma unroll
      for (int src = 0; src < 8; ++src) {
        if (src < C) {   // sources past C are empty: weight exactly 0
          const float f = exp2f((mv[src] - mu) * kDLog2e);
          L += f * lv[src];
          O += f * ov[src];
        }
      }
      if (nclus == 1) {
        a.out[((int64_t)unit * kHeads + h) * kDim + d] = rows_final(a, O, M, L);
        if (d == 0) rows_write_ml(a, unit, h, M, L);
        continue;
      }
      const int64_t cslot = ((int64_t)unit * a.max_clusters + clus) * kHeads + h;
      a.cpart_acc[cslot * kDim + d] = O;
      if (d == 0) {
        a.cpart_ml[cslot * 2 + 0] = M;
        a.cpart_ml[cslot * 2 + 1] = L;
      }
    }
    if (nclus > 1) {
      // Release: the block's partial stores, then one thread's ticket, an
      // acq_rel atomic (cumulative over the stores the barrier ordered
      // before it).  Acquire: the same atomic in the last ticket holder,
      // then the block's barrier.  One atomic instead of fence + atomic +
      // fence: ~0.4 us less per call at batch 1.
      asm volatile("bar.sync 2, %0;" ::"n"(kDim) : "memory");
      if (d == 0) {
        int prev;
        asm volatile("atom.acq_rel.gpu.global.add.s32 %0, [%1], 1;"
                     : "=r"(prev)
                     : "l"(&a.tickets[unit * kHeads + rank])
                     : "memory");
        bars->last = prev == nclus - 1;
      }
      asm volatile("bar.sync 2, %0;" ::"n"(kDim) : "memory");
      if (bars->last) {
        // Merge of the nclus cluster partials of the nh owned heads, all heads
        // at once: 256 / nh threads per head, thread jd of head slot hi
        // owning dims [nh jd, nh jd + nh).  (m, l) of every partial go to
        // shared memory (the stage buffers are free now) while the first
        // batch of partial accumulators is in flight.
        float* sm_m = reinterpret_cast<float*>(smem);          // [8][256]
        float* sm_l = sm_m + kHeads * kDim;                    // [8][256]
        const int64_t u0 = (int64_t)unit * a.max_clusters * kHeads;   // cluster 0, head 0
        if (nh == 1) merge_cluster_partials_nb<1>(a, sm_m, sm_l, u0, unit, rank, C, nh, d, nclus, lane);
        else if (nh == 2) merge_cluster_partials_nb<2>(a, sm_m, sm_l, u0, unit, rank, C, nh, d, nclus, lane);
        else if (nh == 4) merge_cluster_partials_nb<4>(a, sm_m, sm_l, u0, unit, rank, C, nh, d, nclus, lane);
        else merge_cluster_partials_nb<8>(a, sm_m, sm_l, u0, unit, rank, C, nh, d, nclus, lane);
        if (d == 0) a.tickets[unit * kHeads + rank] = 0;   // ready for the next call
      }
    }
  }
}

template <int QT, int KT, int VT = KT>
cudaError_t launch_t(const CUtensorMap& tmk, const CUtensorMap& tmv, const CUtensorMap& tms, const RowsArgs& a,
                     cudaStream_t stream) {
  auto kern = decode_mma_kernel<QT, KT, VT>;
  static std::atomic<bool> attr_set[64];   // per device; zero-initialised
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  if (!attr_set[dev]) {
    const cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kDSmemBytes);
    if (e != cudaSuccess) return e;
    attr_set[dev] = true;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(a.max_clusters * a.cluster, a.n_units, 1);
  cfg.blockDim = dim3(kDThreads, 1, 1);
  cfg.dynamicSmemBytes = kDSmemBytes;
  cfg.stream = stream;
  cudaLaunchAttribute at[2];
  int na = 0;
  if (a.cluster > 1) {
    at[na].id = cudaLaunchAttributeClusterDimension;
    at[na].val.clusterDim.x = a.cluster;
    at[na].val.clusterDim.y = 1;
    at[na].val.clusterDim.z = 1;
    ++na;
  }
  at[na].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  at[na].val.programmaticStreamSerializationAllowed = 1;
  ++na;
  cfg.attrs = at;
  cfg.numAttrs = na;
  return cudaLaunchKernelEx(&cfg, kern, tmk, tmv, tms, a);
}

template <int QT, int KT>
int cluster_capacity_t(int c) {
  auto kern = decode_mma_kernel<QT, KT>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kDSmemBytes) != cudaSuccess)
    return 0;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(c, 1, 1);
  cfg.blockDim = dim3(kDThreads, 1, 1);
  cfg.dynamicSmemBytes = kDSmemBytes;
  cudaLaunchAttribute at;
  at.id = cudaLaunchAttributeClusterDimension;
  at.val.clusterDim.x = c;
  at.val.clusterDim.y = 1;
  at.val.clusterDim.z = 1;
  cfg.attrs = &at;
  cfg.numAttrs = 1;
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, kern, &cfg) != cudaSuccess) return 0;
  return n;
}

// ------------------------------------------------------------ multi-row units
// Batched short chunks (attn_prefill_batch): one unit = up to kMRows
// consecutive query rows of one sequence, so each K/V stage crosses from L2
// to the SM once for all of them.  The unit's keys are the union of its
// rows' visible ranges, cut into splits of the host plan's length; each row
// masks the keys it does not see (an empty row of a split writes the empty
// partial (-inf, 0, 0)).  Per stage: two warps per row take its Q K^T, each
// over 32 of the stage's 64 keys with the row's query (hi/lo) held in
// registers for the whole split (re-reading every row's query from shared
// memory for every stage made the kernel bound by shared-memory latency);
// then the stage max of each row (its two warps), lazy rescale and P as in
// the decode kernel; then each warp loads the V fragments of its 32 dims
// once for every row's P.  One CTA per split, no cluster: a unit with
// several splits writes per-row partials that multirow_merge_kernel
// combines.
constexpr int kMRows = kMultiRows;
static_assert(2 * kMRows == kDWarps, "the multi-row kernel gives each row two warps");
constexpr int kMStages = 2;
constexpr int kMOffBar = kMStages * kDStageBytes;    // 128 KiB

struct MBars {
  uint64_t full[kMStages];
  uint64_t empty[kMStages];
  int abort;
  float red[kDWarps][8];                 // per warp and head: stage max, then row sum
  __align__(16) unsigned char p[kMRows][16 * kDPRow];
  __align__(16) unsigned char qs[kMRows * 16 * kDQRow];   // the rows' queries, before they move to registers
};
constexpr int kMSmemBytes = kMOffBar + (int)sizeof(MBars) + 1024;

template <int QT, int KT>
__global__ void __launch_bounds__(kDThreads, 1)
    decode_multirow_kernel(const __grid_constant__ CUtensorMap tmk, const __grid_constant__ CUtensorMap tmv,
                           const RowsArgs a) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  const uint32_t raw_addr = smem_u32(smem_raw);
  const uint32_t pad = ((raw_addr + 1023u) & ~1023u) - raw_addr;
  unsigned char* smem = smem_raw + pad;
  const uint32_t sbase = raw_addr + pad;
  MBars* bars = reinterpret_cast<MBars*>(smem + kMOffBar);
  unsigned char* qs = bars->qs;                         // [kMRows][16][kDQRow]
  volatile int* abort_flag = &bars->abort;
  DeviceStatus* status = reinterpret_cast<DeviceStatus*>(a.status);

  const int unit = blockIdx.y;
  const int split = blockIdx.x;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  int b, i0, nr;
  multirow_unit(a, unit, &b, &i0, &nr);
  const int64_t pos0 = a.ctx[b] - a.rows_per_seq + i0;       // first row's position
  const int64_t lo_u = lo_of(pos0, a.window);
  const int64_t hi_u = pos0 + nr - 1;
  const int64_t nk_u = hi_u - lo_u + 1;
  const int32_t nsplit = rows_n_splits(nk_u, a.split_len);
  if (split >= nsplit) return;
  const int64_t kbeg = lo_u + (int64_t)split * a.split_len;
  int64_t kend = kbeg + a.split_len;
  if (kend > hi_u + 1) kend = hi_u + 1;
  const int64_t base_row = (int64_t)b * a.seq_rows;
  const int n_stage = (int)cdiv(kend - kbeg, kDStageKeys);
  // bounds-checked builds: the split's rows in the cache, its rows' partial
  // slots in the workspace (no CTA of this kernel waits on another)
  if (!KCA_IN_BOUNDS(nsplit <= a.max_splits && base_row + kbeg >= 0 && base_row + kend <= a.cache_rows &&
                         (nsplit == 1 || ((int64_t)b * a.rows_per_seq + i0 + nr) * a.max_splits <= a.part_slots),
                     status, kSiteBoundsMulti, (unsigned)unit))
    return;

  if (threadIdx.x == 0) {
    for (int st = 0; st < kMStages; ++st) {
      mbar_init(&bars->full[st], 1);
      mbar_init(&bars->empty[st], kDWarps);
    }
    bars->abort = 0;
    fence_barrier_init();
  }
  if (threadIdx.x == kDWarps * 32) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmk)) : "memory");
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmv)) : "memory");
  }
  __syncthreads();
  asm volatile("griddepcontrol.wait;" ::: "memory");

  if (warp == kDWarps) {
    // ---------------------------------------------------------------- producer
    if (lane == 0) {
      int issued = 0;
      for (int i = 0; i < n_stage; ++i) {
        const int slot = i % kMStages;
        if (i >= kMStages &&
            !mbar_wait(&bars->empty[slot], ((i / kMStages) - 1) & 1, abort_flag, status, kSiteRowsEmpty))
          break;
        const uint32_t kst = sbase + slot * kDStageBytes;
        const uint32_t bar = smem_u32(&bars->full[slot]);
        const int32_t row0 = (int32_t)(base_row + kbeg + (int64_t)i * kDStageKeys);
        mbar_arrive_expect_tx(&bars->full[slot], kDStageBytes);
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          tma2d(kst + c * kDBoxBytes, &tmk, 64 * c, row0, bar);
          tma2d(kst + kDHalfBytes + c * kDBoxBytes, &tmv, 64 * c, row0, bar);
        }
        issued = i + 1;
      }
      if (issued < n_stage) {  // aborted: let every issued copy land
        for (int st = 0; st < kMStages && st < issued; ++st) {
          const int last = ((issued - 1 - st) / kMStages) * kMStages + st;
          mbar_wait(&bars->full[st], (last / kMStages) & 1, nullptr, status, kSiteRowsFull);
        }
      }
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------------ compute
    const int g = lane >> 2, tig = lane & 3;
    {
      // Stage each row's query (hi / lo 16-bit parts, 16 rows of 256 dims);
      // rows past nr are zero.  Thread t: 8 dims of head t / 32.
      const int h = threadIdx.x >> 5, d0 = 8 * (threadIdx.x & 31);
#pragma unroll
      for (int r = 0; r < kMRows; ++r) {
        float x[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
        if (r < nr) {
          const int64_t orow = (int64_t)b * a.rows_per_seq + i0 + r;
          load8<QT>(static_cast<const char*>(a.q) + ((orow * kHeads + h) * kDim + d0) * ElemBytes<QT>::value, x);
        }
        uint32_t hi[4], lo[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          hi[j] = pack16<KT>(x[2 * j], x[2 * j + 1]);
          const float2 f = unpack16<KT>(hi[j]);
          lo[j] = pack16<KT>(x[2 * j] - f.x, x[2 * j + 1] - f.y);
        }
        *reinterpret_cast<uint4*>(qs + r * 16 * kDQRow + h * kDQRow + d0 * 2) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
        *reinterpret_cast<uint4*>(qs + r * 16 * kDQRow + (h + 8) * kDQRow + d0 * 2) =
            make_uint4(lo[0], lo[1], lo[2], lo[3]);
      }
      asm volatile("bar.sync 1, %0;" ::"n"(kDWarps * 32) : "memory");
    }
    const int mi = lane >> 3;
    // Q K^T: warp w takes row qr = w / 2 of the unit and keys 32 (w % 2) ..
    // + 31 of every stage, with that row's query (16-bit high and low parts
    // as M rows 0-7 / 8-15) held in registers for the whole split, so no
    // stage reads a query from shared memory.  P V: warp w takes dims
    // 32 w .. + 31 of every row, as in the single-row kernel.
    const int qr = warp >> 1, kh = warp & 1;
    const bool q_live = qr < nr;
    uint32_t qa[16][4];
    {
      const uint32_t qrow = smem_u32(qs + (q_live ? qr : 0) * 16 * kDQRow) + (8 * (mi & 1) + (lane & 7)) * kDQRow +
                            8 * (mi >> 1) * 2;
#pragma unroll
      for (int ks = 0; ks < 16; ++ks) ldsm_x4(qrow + 32 * ks, qa[ks]);
    }
    const int64_t qpos = pos0 + qr, qlo = lo_of(qpos, a.window);
    float o[kMRows][4][4];
#pragma unroll
    for (int r = 0; r < kMRows; ++r)
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) o[r][i][j] = 0.f;
    float m_ref[kMRows];
#pragma unroll
    for (int r = 0; r < kMRows; ++r) m_ref[r] = -INFINITY;
    float l_own = 0.f;   // row qr, head g, this warp's keys
    const float scale = a.scale;
    bool ok = true;

    for (int i = 0; i < n_stage; ++i) {
      const int slot = i % kMStages;
      ok = __all_sync(0xffffffffu, ok && mbar_wait(&bars->full[slot], (i / kMStages) & 1, abort_flag,
                                                   status, kSiteRowsFull));
      const int64_t k0 = kbeg + (int64_t)i * kDStageKeys;
      const int cnt = (int)((kend - k0) < kDStageKeys ? (kend - k0) : kDStageKeys);
      const uint32_t kst = sbase + slot * kDStageBytes;
      const uint32_t vst = kst + kDHalfBytes;
      float sx[4][2];
#pragma unroll
      for (int nt = 0; nt < 4; ++nt) sx[nt][0] = sx[nt][1] = -INFINITY;
      if (ok) {
        if (cnt < kDStageKeys) {  // V rows past the split's end -> 0
          unsigned char* vrows = smem + slot * kDStageBytes + kDHalfBytes;
          for (int idx = threadIdx.x; idx < (kDStageKeys - cnt) * 32; idx += kDWarps * 32) {
            const int row = cnt + (idx >> 5), u = idx & 31;
            *reinterpret_cast<uint4*>(vrows + (u >> 3) * kDBoxBytes + row * 128 + (u & 7) * 16) =
                make_uint4(0, 0, 0, 0);
          }
        }
        if (q_live) {
          // one accumulation chain per 8-key tile: four independent chains
          float sacc[4][4];
#pragma unroll
          for (int nt = 0; nt < 4; ++nt)
#pragma unroll
            for (int j = 0; j < 4; ++j) sacc[nt][j] = 0.f;
#pragma unroll
          for (int ks2 = 0; ks2 < 8; ++ks2) {
#pragma unroll
            for (int nt = 0; nt < 4; ++nt) {
              uint32_t bk[4];
              ldsm_x4(kst + swz(32 * kh + 8 * nt + (lane & 7), 32 * ks2 + 8 * (lane >> 3)), bk);
              mma16816<KT>(sacc[nt], qa[2 * ks2], bk[0], bk[1]);
              mma16816<KT>(sacc[nt], qa[2 * ks2 + 1], bk[2], bk[3]);
            }
          }
#pragma unroll
          for (int nt = 0; nt < 4; ++nt) {
            const int kk = 32 * kh + 8 * nt + 2 * tig;
            const int64_t key = k0 + kk;
            const float s0 = sacc[nt][0] + sacc[nt][2];   // high + low parts of head g
            const float s1 = sacc[nt][1] + sacc[nt][3];
            sx[nt][0] = kk < cnt && key >= qlo && key <= qpos ? s0 * scale : -INFINITY;
            sx[nt][1] = kk + 1 < cnt && key + 1 >= qlo && key + 1 <= qpos ? s1 * scale : -INFINITY;
          }
        }
      }
      // Stage max of every row and head: this warp's 32 keys, then the row's
      // two warps (every warp needs every row's max for its P V columns).
      float mw = -INFINITY;
#pragma unroll
      for (int nt = 0; nt < 4; ++nt) mw = max_nan(mw, max_nan(sx[nt][0], sx[nt][1]));
      mw = max_nan(mw, __shfl_xor_sync(0xffffffffu, mw, 1));
      mw = max_nan(mw, __shfl_xor_sync(0xffffffffu, mw, 2));
      if (tig == 0) bars->red[warp][g] = mw;
      asm volatile("bar.sync 1, %0;" ::"n"(kDWarps * 32) : "memory");
      if (ok) {
        float mq = -INFINITY;
#pragma unroll
        for (int r = 0; r < kMRows; ++r) {
          if (r < nr) {
            const float ms = max_nan(bars->red[2 * r][g], bars->red[2 * r + 1][g]);
            if (ms > m_ref[r] + kDRescale) {
              const float alpha = exp2f((m_ref[r] - ms) * kDLog2e);
              m_ref[r] = ms;
              if (r == qr) l_own *= alpha;
#pragma unroll
              for (int nt = 0; nt < 4; ++nt)
#pragma unroll
                for (int j = 0; j < 4; ++j) o[r][nt][j] *= alpha;
            }
            if (r == qr) mq = m_ref[r];
          }
        }
        if (q_live) {
          const float mu = mq == -INFINITY ? 0.f : mq;
          unsigned char* prow = bars->p[qr];
#pragma unroll
          for (int nt = 0; nt < 4; ++nt) {
            const float p0 = exp2f((sx[nt][0] - mu) * kDLog2e);
            const float p1 = exp2f((sx[nt][1] - mu) * kDLog2e);
            l_own += p0 + p1;
            const uint32_t hi = pack16<KT>(p0, p1);
            const float2 f = unpack16<KT>(hi);
            const uint32_t lo16 = pack16<KT>(p0 - f.x, p1 - f.y);
            const int key = 32 * kh + 8 * nt + 2 * tig;
            *reinterpret_cast<uint32_t*>(prow + g * kDPRow + key * 2) = hi;
            *reinterpret_cast<uint32_t*>(prow + (g + 8) * kDPRow + key * 2) = lo16;
          }
        }
      }
      asm volatile("bar.sync 1, %0;" ::"n"(kDWarps * 32) : "memory");   // P and zeroed rows visible
      if (ok) {
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
          uint32_t af[kMRows][4];
#pragma unroll
          for (int r = 0; r < kMRows; ++r)
            if (r < nr)
              ldsm_x4(smem_u32(bars->p[r]) + (8 * (mi & 1) + (lane & 7)) * kDPRow + (16 * kk + 8 * (mi >> 1)) * 2,
                      af[r]);
          const int key = 16 * kk + 8 * (mi & 1) + (lane & 7);
#pragma unroll
          for (int pair = 0; pair < 2; ++pair) {
            uint32_t vb[4];
            ldsm_x4_t(vst + swz(key, 32 * warp + 16 * pair + 8 * (mi >> 1)), vb);
#pragma unroll
            for (int r = 0; r < kMRows; ++r) {
              if (r < nr) {
                mma16816<KT>(o[r][2 * pair], af[r], vb[0], vb[1]);
                mma16816<KT>(o[r][2 * pair + 1], af[r], vb[2], vb[3]);
              }
            }
          }
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->empty[slot]);
    }

    // Row sums: lanes of one head, then the row's two warps.
    {
      float l = l_own;
      l += __shfl_xor_sync(0xffffffffu, l, 1);
      l += __shfl_xor_sync(0xffffffffu, l, 2);
      if (tig == 0) bars->red[warp][g] = l;
    }
    asm volatile("bar.sync 1, %0;" ::"n"(kDWarps * 32) : "memory");
    const bool aborted = !ok || *abort_flag;
#pragma unroll
    for (int r = 0; r < kMRows; ++r) {
      if (r < nr) {
        float L = bars->red[2 * r][g] + bars->red[2 * r + 1][g];
        float M = m_ref[r];
        if (aborted) {
          M = NAN;   // an aborted split poisons its rows; the status word says why
          L = NAN;
        }
        const int64_t orow = (int64_t)b * a.rows_per_seq + i0 + r;
        if (nsplit == 1) {
          const float inv = (M == -INFINITY && L == 0.f) ? 0.f : 1.f / L;
#pragma unroll
          for (int nt = 0; nt < 4; ++nt) {
            const int d = 32 * warp + 8 * nt + 2 * tig;
            *reinterpret_cast<float2*>(a.out + (orow * kHeads + g) * kDim + d) =
                make_float2((o[r][nt][0] + o[r][nt][2]) * inv, (o[r][nt][1] + o[r][nt][3]) * inv);
          }
        } else {
          const int64_t slot = (orow * a.max_splits + split) * kHeads + g;
#pragma unroll
          for (int nt = 0; nt < 4; ++nt) {
            const int d = 32 * warp + 8 * nt + 2 * tig;
            *reinterpret_cast<float2*>(a.part_acc + slot * kDim + d) =
                make_float2(o[r][nt][0] + o[r][nt][2], o[r][nt][1] + o[r][nt][3]);
          }
          if (warp == 0 && tig == 0) *reinterpret_cast<float2*>(a.part_ml + slot * 2) = make_float2(M, L);
        }
      }
    }
  }
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// Log-sum-exp merge of the split partials of every row of a multi-row call:
// one CTA per (row, head), its eight warps taking interleaved splits.
__global__ void __launch_bounds__(256) multirow_merge_kernel(const RowsArgs a) {
  const int64_t orow = blockIdx.x >> 3;
  const int h = blockIdx.x & 7;
  const int b = (int)(orow / a.rows_per_seq);
  const int i = (int)(orow % a.rows_per_seq);
  const int u = b * ((a.rows_per_seq + a.unit_rows - 1) / a.unit_rows) + i / a.unit_rows;
  int bb, i0, nr;
  multirow_unit(a, u, &bb, &i0, &nr);
  const int64_t pos0 = a.ctx[bb] - a.rows_per_seq + i0;
  const int64_t nk_u = pos0 + nr - 1 - lo_of(pos0, a.window) + 1;
  const int32_t nsplit = rows_n_splits(nk_u, a.split_len);
  asm volatile("griddepcontrol.wait;" ::: "memory");
  if (nsplit <= 1) return;
  if (!KCA_IN_BOUNDS(nsplit <= a.max_splits && (orow + 1) * a.max_splits <= a.part_slots,
                     static_cast<DeviceStatus*>(a.status), kSiteBoundsMerge, (unsigned)orow))
    return;
  __shared__ float red[8 * 264];
  const int64_t row0 = orow * a.max_splits * kHeads + h;
  merge_row<8>(nsplit, a.part_ml + row0 * 2, kHeads * 2, a.part_acc + row0 * kDim, kHeads * kDim, kDLog2e,
               a.out + (orow * kHeads + h) * kDim, red, threadIdx.x >> 5, threadIdx.x & 31, 1);
}

template <int QT, int KT>
cudaError_t launch_multirow_t(const CUtensorMap& tmk, const CUtensorMap& tmv, const RowsArgs& a, cudaStream_t stream) {
  auto kern = decode_multirow_kernel<QT, KT>;
  static std::atomic<bool> attr_set[64];   // per device; zero-initialised
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  if (!attr_set[dev]) {
    const cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kMSmemBytes);
    if (e != cudaSuccess) return e;
    attr_set[dev] = true;
  }
  cudaLaunchAttribute at;
  at.id = cudaLaunchAttributeProgrammaticStreamSerialization;
  at.val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(a.max_splits, a.n_units, 1);
  cfg.blockDim = dim3(kDThreads, 1, 1);
  cfg.dynamicSmemBytes = kMSmemBytes;
  cfg.stream = stream;
  cfg.attrs = &at;
  cfg.numAttrs = 1;
  cudaError_t e = cudaLaunchKernelEx(&cfg, kern, tmk, tmv, a);
  if (e != cudaSuccess || a.max_splits <= 1) return e;
  return launch_multirow_merge(a, stream);
}

}  // namespace

cudaError_t launch_multirow_merge(const RowsArgs& a, cudaStream_t stream) {
  cudaLaunchAttribute at;
  at.id = cudaLaunchAttributeProgrammaticStreamSerialization;
  at.val.programmaticStreamSerializationAllowed = 1;
  const int blocks = (a.rows_per_seq + a.unit_rows - 1) / a.unit_rows;
  const int64_t rows_total = (int64_t)(a.n_units / blocks) * a.rows_per_seq;
  cudaLaunchConfig_t mcfg = {};
  mcfg.gridDim = dim3((unsigned)(rows_total * kHeads), 1, 1);
  mcfg.blockDim = dim3(256, 1, 1);
  mcfg.stream = stream;
  mcfg.attrs = &at;
  mcfg.numAttrs = 1;
  return cudaLaunchKernelEx(&mcfg, multirow_merge_kernel, a);
}

int decode_mma_cluster_capacity(int c) {
  // Same launch shape for every dtype instantiation; cached per device and size.
  static std::atomic<int> cache[64][4];   // zero-initialised
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 0;
  const int idx = c == 1 ? 0 : (c == 2 ? 1 : (c == 4 ? 2 : 3));
  if (cache[dev][idx] == 0) cache[dev][idx] = cluster_capacity_t<KCA_F32, KCA_F16>(c);
  return cache[dev][idx];
}

cudaError_t launch_decode_mma(int q_dtype, int kv_dtype, const CUtensorMap& tmk, const CUtensorMap& tmv,
                              const RowsArgs& a, cudaStream_t stream) {
  cudaError_t e = cudaErrorInvalidValue;
#define KCA_DMMA_CASE(QD, KD) \
  if (q_dtype == QD && kv_dtype == KD) e = launch_t<QD, KD>(tmk, tmv, tmk, a, stream);
  KCA_DMMA_CASE(KCA_F32, KCA_F16)
  KCA_DMMA_CASE(KCA_F32, KCA_BF16)
  KCA_DMMA_CASE(KCA_F16, KCA_F16)
  KCA_DMMA_CASE(KCA_F16, KCA_BF16)
  KCA_DMMA_CASE(KCA_BF16, KCA_F16)
  KCA_DMMA_CASE(KCA_BF16, KCA_BF16)
#undef KCA_DMMA_CASE
  return e;
}

cudaError_t launch_decode_mma_q8(int q_dtype, int v_dtype, const CUtensorMap& tmk, const CUtensorMap& tms,
                                 const CUtensorMap& tmv, const RowsArgs& a, cudaStream_t stream) {
  cudaError_t e = cudaErrorInvalidValue;
#define KCA_DQ8_CASE(QD, VD) \
  if (q_dtype == QD && v_dtype == VD) e = launch_t<QD, KCA_I8, VD>(tmk, tmv, tms, a, stream);
  KCA_DQ8_CASE(KCA_F32, KCA_F16)
  KCA_DQ8_CASE(KCA_F32, KCA_BF16)
  KCA_DQ8_CASE(KCA_F16, KCA_F16)
  KCA_DQ8_CASE(KCA_F16, KCA_BF16)
  KCA_DQ8_CASE(KCA_BF16, KCA_F16)
  KCA_DQ8_CASE(KCA_BF16, KCA_BF16)
#undef KCA_DQ8_CASE
  return e;
}

cudaError_t launch_decode_multirow(int q_dtype, int kv_dtype, const CUtensorMap& tmk, const CUtensorMap& tmv,
                                   const RowsArgs& a, cudaStream_t stream) {
#define KCA_MR_CASE(QD, KD) \
  if (q_dtype == QD && kv_dtype == KD) return launch_multirow_t<QD, KD>(tmk, tmv, a, stream);
  KCA_MR_CASE(KCA_F32, KCA_F16)
  KCA_MR_CASE(KCA_F32, KCA_BF16)
  KCA_MR_CASE(KCA_F16, KCA_F16)
  KCA_MR_CASE(KCA_F16, KCA_BF16)
  KCA_MR_CASE(KCA_BF16, KCA_F16)
  KCA_MR_CASE(KCA_BF16, KCA_BF16)
#undef KCA_MR_CASE
  return cudaErrorInvalidValue;
}

}  // namespace kca

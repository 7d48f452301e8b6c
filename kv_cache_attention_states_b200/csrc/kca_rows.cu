// kca_rows.cu -- split-context attention of single query rows on the CUDA
// cores: decode (one row per sequence) and the prefill rows that do not take
// the tensor cores (f32 inputs, mixed dtypes, chunks under 16 rows).
//
// Prior art on the pages: Karume's "parallel" reductions for one-row plans
// (v0.12.0 release notes, "Performance", items 2-3: QK split along the head
// dimension, PV split along the KV axis; v0.8.0 release notes, "Performance",
// long-context item).  Here the context of each row is cut into splits, one
// CTA per split; K/V rows stream through a shared-memory ring filled by bulk
// copies, each warp reduces its QK dots with warp shuffles and keeps an online
// softmax, and the splits are merged by log-sum-exp in merge_rows_kernel.
#include <atomic>
#include <cuda_runtime.h>

#include "kca_common.cuh"
#include "kca_merge.cuh"
#include "kca_plan.h"
#include "kca_rows.h"

namespace kca {

namespace {

constexpr int kComputeWarps = 8;
constexpr int kRowsThreads = (kComputeWarps + 1) * 32;  // + one producer warp
constexpr int kKeysPerStage = 16;
constexpr int kStages = 4;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kRescaleThreshold = 5.545177444479562f;  // 8 * ln 2: rescale once p could pass 256

// K rows: 256 elements of KT, or packed int8 rows (KCA_I8: 256 codes, the
// row's f32 scale, 12 bytes of padding); V rows: 256 elements of VT.
template <int KT>
struct KRowBytes { static constexpr int value = KT == KCA_I8 ? KCA_I8_ROW_BYTES : kDim * ElemBytes<KT>::value; };

template <int KT, int VT = KT>
struct RowsSmem {
  static constexpr int kKRowBytes = KRowBytes<KT>::value;
  static constexpr int kVRowBytes = kDim * ElemBytes<VT>::value;
  static constexpr int kStageBytes = kKeysPerStage * (kKRowBytes + kVRowBytes);   // K rows then V rows
  static constexpr int kRingBytes = kStages * kStageBytes;
  static constexpr int kCombineBytes = kComputeWarps * kHeads * (kDim + 2) * 4;
  static constexpr int kDataBytes = kRingBytes > kCombineBytes ? kRingBytes : kCombineBytes;
  static constexpr int kBarOffset = kDataBytes;
  static constexpr int kTotal = kBarOffset + 2 * kStages * 8 + 16;
};

// Sum eight per-lane values over the warp.  Returns, in every lane, the full
// sum of value number (lane >> 2) & 7: three halving exchanges (16, 8, 4)
// followed by two full ones (2, 1) -- 9 shuffles instead of 40.
__device__ __forceinline__ float reduce8_transposed(const float (&v)[8], int lane) {
  const bool b4 = lane & 16, b3 = lane & 8, b2 = lane & 4;
  float r4[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float keep = b4 ? v[i + 4] : v[i];
    const float send = b4 ? v[i] : v[i + 4];
    r4[i] = keep + __shfl_xor_sync(0xffffffffu, send, 16);
  }
  float r2[2];
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    const float keep = b3 ? r4[i + 2] : r4[i];
    const float send = b3 ? r4[i] : r4[i + 2];
    r2[i] = keep + __shfl_xor_sync(0xffffffffu, send, 8);
  }
  float r = (b2 ? r2[1] : r2[0]) + __shfl_xor_sync(0xffffffffu, b2 ? r2[0] : r2[1], 4);
  r += __shfl_xor_sync(0xffffffffu, r, 2);
  r += __shfl_xor_sync(0xffffffffu, r, 1);
  return r;
}

// Dot product of four packed int8 pairs plus c: the dp4a instruction, or
// its emulation from the sign-extended bytes (the canary in kca_q8.cu picks
// one per device).
template <bool DP4A>
__device__ __forceinline__ int dot4(uint32_t a, uint32_t b, int c) {
  if (DP4A) return __dp4a(static_cast<int>(a), static_cast<int>(b), c);
#pragma unroll
  for (int i = 0; i < 4; ++i)
    c += static_cast<int>(static_cast<int8_t>(a >> (8 * i))) * static_cast<int>(static_cast<int8_t>(b >> (8 * i)));
  return c;
}

// int8 code of x under the row scale sx (the quantisation of kca_q8.cu):
// round-half-even of the f32 quotient, clamped to +-127; 0 unless sx is
// finite and positive.
__device__ __forceinline__ uint32_t q8_code(float x, float sx) {
  if (!(sx > 0.f) || !(sx <= 3.402823466e38f)) return 0u;
  int c = __float2int_rn(__fdiv_rn(x, sx));
  c = c > 127 ? 127 : (c < -127 ? -127 : c);
  return static_cast<uint32_t>(c) & 0xffu;
}

template <int QT, int KT, int VT = KT, bool DP4A = true>
__global__ void __launch_bounds__(kRowsThreads, 1) rows_kernel(const RowsArgs a) {
  using S = RowsSmem<KT, VT>;
  constexpr bool kQ8 = KT == KCA_I8;
  extern __shared__ __align__(1024) unsigned char smem[];
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + S::kBarOffset);
  uint64_t* empty = full + kStages;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(empty + kStages);
  DeviceStatus* status = reinterpret_cast<DeviceStatus*>(a.status);

  const int unit = blockIdx.y;
  const int split = blockIdx.x;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  int64_t seq_base;
  const int64_t pos = rows_unit_pos(a, unit, split == 0 && threadIdx.x == 0, &seq_base);
  int64_t lo;
  const int64_t nkeys = rows_keys(a, pos, &lo);
  const int32_t split_len = rows_split_len(a, nkeys, kRowsSplitQuantum);
  const int32_t nsplit = rows_n_splits(nkeys, split_len);
  if (split >= nsplit) return;
  const int64_t kbeg = lo + (int64_t)split * split_len;
  int64_t kend = kbeg + split_len;
  if (kend > lo + nkeys) kend = lo + nkeys;
  // cache row of key p: base_row + p (a shard's row 0 is position key_begin)
  const int64_t base_row = seq_base - a.key_begin;
  float* out = a.out + (int64_t)unit * kHeads * kDim;
  // bounds-checked builds: the split's rows lie in the cache and its partial
  // slot in the workspace (no CTA of this kernel waits on another)
  if (!KCA_IN_BOUNDS(nsplit <= a.max_splits && base_row + kbeg >= 0 && base_row + kend <= a.cache_rows &&
                         (nsplit == 1 || (int64_t)(unit + 1) * a.max_splits <= a.part_slots),
                     status, kSiteBoundsRows, (unsigned)unit))
    return;

  if (nkeys == 0) {  // fully masked row: exactly zero (as a partial: (-inf, 0, 0))
    if (warp < kComputeWarps)
      for (int i = threadIdx.x; i < kHeads * kDim; i += kComputeWarps * 32) out[i] = 0.f;
    if (threadIdx.x < kHeads) rows_write_ml(a, unit, threadIdx.x, -INFINITY, 0.f);
    return;
  }
  const int n_stage = (int)cdiv(kend - kbeg, kKeysPerStage);

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], kComputeWarps);
    }
    *abort_flag = 0;
    fence_barrier_init();
  }
  __syncthreads();

  const char* kg = static_cast<const char*>(a.k);
  const char* vg = static_cast<const char*>(a.v);

  if (warp == kComputeWarps) {
    // ---------------------------------------------------------------- producer
    if (lane == 0) {
      int issued = 0;
      for (int i = 0; i < n_stage; ++i) {
        const int slot = i % kStages;
        if (i >= kStages &&
            !mbar_wait(&empty[slot], ((i / kStages) - 1) & 1, abort_flag, status, kSiteRowsEmpty))
          break;
        const int64_t k0 = kbeg + (int64_t)i * kKeysPerStage;
        const int cnt = (int)((kend - k0) < kKeysPerStage ? (kend - k0) : kKeysPerStage);
        const uint32_t kbytes = (uint32_t)cnt * S::kKRowBytes;
        const uint32_t vbytes = (uint32_t)cnt * S::kVRowBytes;
        unsigned char* dst = smem + slot * S::kStageBytes;
        mbar_arrive_expect_tx(&full[slot], kbytes + vbytes);
        bulk_g2s(dst, kg + (base_row + k0) * S::kKRowBytes, kbytes, &full[slot]);
        bulk_g2s(dst + kKeysPerStage * S::kKRowBytes, vg + (base_row + k0) * S::kVRowBytes, vbytes,
                 &full[slot]);
        issued = i + 1;
      }
      if (issued < n_stage) {
        // Aborted: let every copy already issued land before the CTA exits.
        for (int s = 0; s < kStages && s < issued; ++s) {
          const int last = ((issued - 1 - s) / kStages) * kStages + s;
          mbar_wait(&full[s], (last / kStages) & 1, nullptr, status, kSiteRowsFull);
        }
      }
    }
  } else {
    // ---------------------------------------------------------------- compute
    // Query of this row, all 8 heads, dims [8*lane, 8*lane+8), in f32.
    // Quantised-dot variant: the int8 codes of the query (per head: scale
    // amax * f32(1/127) over the head's 256 values) and this lane's head's
    // scale; otherwise the query in f32.
    float2 q2[kQ8 ? 1 : kHeads][4];
    uint32_t qp[kQ8 ? kHeads : 1][2];
    float sq_mine = 0.f;
    {
      const char* qrow = static_cast<const char*>(a.q) +
                         (int64_t)unit * kHeads * kDim * ElemBytes<QT>::value;
#pragma unroll
      for (int h = 0; h < kHeads; ++h) {
        float x[8];
        load8<QT>(qrow + ((int64_t)h * kDim + 8 * lane) * ElemBytes<QT>::value, x);
        if constexpr (kQ8) {
          float am = fabsf(x[0]);
#pragma unroll
          for (int i = 1; i < 8; ++i) am = max_nan(am, fabsf(x[i]));
#pragma unroll
          for (int o = 16; o > 0; o >>= 1) am = max_nan(am, __shfl_xor_sync(0xffffffffu, am, o));
          const float sx = am * (1.0f / 127.0f);
          if (h == ((lane >> 2) & 7)) sq_mine = sx;
#pragma unroll
          for (int w = 0; w < 2; ++w)
            qp[h][w] = q8_code(x[4 * w], sx) | (q8_code(x[4 * w + 1], sx) << 8) |
                       (q8_code(x[4 * w + 2], sx) << 16) | (q8_code(x[4 * w + 3], sx) << 24);
        } else {
#pragma unroll
          for (int i = 0; i < 4; ++i) q2[h][i] = make_float2(x[2 * i], x[2 * i + 1]);
        }
      }
    }
    float2 acc[kHeads][4];
#pragma unroll
    for (int h = 0; h < kHeads; ++h)
#pragma unroll
      for (int i = 0; i < 4; ++i) acc[h][i] = make_float2(0.f, 0.f);
    float m_ref = -INFINITY;  // reference max of head (lane >> 2) & 7
    float l_sum = 0.f;
    const float scale = a.scale;
    bool ok = true;

    for (int i = 0; i < n_stage && ok; ++i) {
      const int slot = i % kStages;
      // warp-uniform, so no lane reaches the shuffles below without the others
      ok = __all_sync(0xffffffffu,
                      mbar_wait(&full[slot], (i / kStages) & 1, abort_flag, status, kSiteRowsFull));
      if (!ok) break;
      const int64_t k0 = kbeg + (int64_t)i * kKeysPerStage;
      const int cnt = (int)((kend - k0) < kKeysPerStage ? (kend - k0) : kKeysPerStage);
      const unsigned char* st = smem + slot * S::kStageBytes;
      const int nk = (warp < cnt ? 1 : 0) + (warp + kComputeWarps < cnt ? 1 : 0);
      if (nk > 0) {
        float s_own[2];
        float vx[2][8];
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          if (c < nk) {
            const int r = warp + c * kComputeWarps;
            const unsigned char* krow = st + r * S::kKRowBytes;
            load8<VT>(st + kKeysPerStage * S::kKRowBytes + r * S::kVRowBytes + 8 * lane * ElemBytes<VT>::value,
                      vx[c]);
            float part[8];
            if constexpr (kQ8) {
              // exact integer dot products (|partial| < 2^24, so f32 holds
              // them and their warp sum exactly), then the two scales
              const uint2 kw = *reinterpret_cast<const uint2*>(krow + 8 * lane);
              const float sk = *reinterpret_cast<const float*>(krow + kDim);
#pragma unroll
              for (int h = 0; h < kHeads; ++h)
                part[h] = static_cast<float>(dot4<DP4A>(qp[h][1], kw.y, dot4<DP4A>(qp[h][0], kw.x, 0)));
              s_own[c] = reduce8_transposed(part, lane) * ((sq_mine * sk) * scale);
            } else {
              float kx[8];
              load8<KT>(krow + 8 * lane * ElemBytes<KT>::value, kx);
#pragma unroll
              for (int h = 0; h < kHeads; ++h) {
                float2 d = make_float2(0.f, 0.f);
#pragma unroll
                for (int t = 0; t < 4; ++t) d = ffma2(q2[h][t], make_float2(kx[2 * t], kx[2 * t + 1]), d);
                part[h] = d.x + d.y;
              }
              s_own[c] = reduce8_transposed(part, lane) * scale;
            }
          } else {
            s_own[c] = -INFINITY;
#pragma unroll
            for (int t = 0; t < 8; ++t) vx[c][t] = 0.f;
          }
        }
        // Lazy rescale: move the reference max only when a score exceeds it
        // by more than the threshold; exp(s - m_ref) then stays <= 256.
        const float m_cand = fmaxf(s_own[0], s_own[1]);
        const bool need = m_cand > m_ref + kRescaleThreshold;
        if (__any_sync(0xffffffffu, need)) {
          const float alpha = need ? exp2f((m_ref - m_cand) * kLog2e) : 1.f;
          if (need) m_ref = m_cand;
          l_sum *= alpha;
#pragma unroll
          for (int h = 0; h < kHeads; ++h) {
            const float ah = __shfl_sync(0xffffffffu, alpha, 4 * h);
#pragma unroll
            for (int t = 0; t < 4; ++t) acc[h][t] = __fmul2_rn(acc[h][t], make_float2(ah, ah));
          }
        }
        const float m_use = m_ref == -INFINITY ? 0.f : m_ref;
        float p_own[2];
#pragma unroll
        for (int c = 0; c < 2; ++c) p_own[c] = exp2f((s_own[c] - m_use) * kLog2e);
        l_sum += p_own[0] + p_own[1];
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          if (c < nk) {
#pragma unroll
            for (int h = 0; h < kHeads; ++h) {
              const float ph = __shfl_sync(0xffffffffu, p_own[c], 4 * h);
#pragma unroll
              for (int t = 0; t < 4; ++t)
                acc[h][t] = ffma2(make_float2(vx[c][2 * t], vx[c][2 * t + 1]), make_float2(ph, ph),
                                  acc[h][t]);
            }
          }
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[slot]);
    }

    // All compute warps are done with the ring; reuse it to combine warps.
    asm volatile("bar.sync 1, %0;" ::"n"(kComputeWarps * 32) : "memory");
    if (!*abort_flag) {
      float* cm = reinterpret_cast<float*>(smem);                  // [warp][head]
      float* cl = cm + kComputeWarps * kHeads;                      // [warp][head]
      float* cacc = cl + kComputeWarps * kHeads;                    // [warp][head][256]
      if ((lane & 3) == 0) {
        cm[warp * kHeads + (lane >> 2)] = m_ref;
        cl[warp * kHeads + (lane >> 2)] = l_sum;
      }
#pragma unroll
      for (int h = 0; h < kHeads; ++h) {
        float4* dst = reinterpret_cast<float4*>(cacc + ((warp * kHeads + h) * kDim + 8 * lane));
        dst[0] = make_float4(acc[h][0].x, acc[h][0].y, acc[h][1].x, acc[h][1].y);
        dst[1] = make_float4(acc[h][2].x, acc[h][2].y, acc[h][3].x, acc[h][3].y);
      }
      asm volatile("bar.sync 1, %0;" ::"n"(kComputeWarps * 32) : "memory");
      // thread (h = warp, lane) combines head h, dims [8*lane, 8*lane+8)
      const int h = warp;
      float M = -INFINITY;
#pragma unroll
      for (int w = 0; w < kComputeWarps; ++w) M = max_nan(M, cm[w * kHeads + h]);
      const float M_use = M == -INFINITY ? 0.f : M;
      float L = 0.f;
      float A[8];
#pragma unroll
      for (int t = 0; t < 8; ++t) A[t] = 0.f;
#pragma unroll
      for (int w = 0; w < kComputeWarps; ++w) {
        const float f = exp2f((cm[w * kHeads + h] - M_use) * kLog2e);
        L += f * cl[w * kHeads + h];
        const float4* src = reinterpret_cast<const float4*>(cacc + ((w * kHeads + h) * kDim + 8 * lane));
        const float4 x0 = src[0], x1 = src[1];
        A[0] += f * x0.x; A[1] += f * x0.y; A[2] += f * x0.z; A[3] += f * x0.w;
        A[4] += f * x1.x; A[5] += f * x1.y; A[6] += f * x1.z; A[7] += f * x1.w;
      }
      if (nsplit == 1) {
        const float inv = a.out_ml != nullptr ? 1.f : 1.f / L;
        float4* o = reinterpret_cast<float4*>(out + h * kDim + 8 * lane);
        o[0] = make_float4(A[0] * inv, A[1] * inv, A[2] * inv, A[3] * inv);
        o[1] = make_float4(A[4] * inv, A[5] * inv, A[6] * inv, A[7] * inv);
        if (lane == 0) rows_write_ml(a, unit, h, M, L);
      } else {
        const int64_t slot = (int64_t)unit * a.max_splits + split;
        if (lane == 0) {
          a.part_ml[(slot * kHeads + h) * 2 + 0] = M;
          a.part_ml[(slot * kHeads + h) * 2 + 1] = L;
        }
        float4* o = reinterpret_cast<float4*>(a.part_acc + (slot * kHeads + h) * kDim + 8 * lane);
        o[0] = make_float4(A[0], A[1], A[2], A[3]);
        o[1] = make_float4(A[4], A[5], A[6], A[7]);
      }
    }
  }
}

// Log-sum-exp merge of the splits of each unit: one CTA per (unit, head),
// its eight warps taking interleaved splits.
__global__ void __launch_bounds__(256) merge_rows_kernel(const RowsArgs a) {
  const int unit = blockIdx.x >> 3, h = blockIdx.x & 7;
  int64_t seq_base;
  const int64_t pos = rows_unit_pos(a, unit, false, &seq_base);
  int64_t lo;
  const int64_t nkeys = rows_keys(a, pos, &lo);
  const int32_t nsplit = rows_n_splits(nkeys, rows_split_len(a, nkeys, kRowsSplitQuantum));
  if (nsplit <= 1) return;
  if (!KCA_IN_BOUNDS(nsplit <= a.max_splits && (int64_t)(unit + 1) * a.max_splits <= a.part_slots,
                     static_cast<DeviceStatus*>(a.status), kSiteBoundsMerge, (unsigned)unit))
    return;
  __shared__ float red[8 * 264];
  const int64_t row0 = (int64_t)unit * a.max_splits * kHeads + h;
  merge_row<8>(nsplit, a.part_ml + row0 * 2, kHeads * 2, a.part_acc + row0 * kDim, kHeads * kDim,
               kLog2e, a.out + ((int64_t)unit * kHeads + h) * kDim, red, threadIdx.x >> 5,
               threadIdx.x & 31, 1, a.out_ml != nullptr ? a.out_ml + ((int64_t)unit * kHeads + h) * 2 : nullptr);
}

template <int QT, int KT, int VT = KT, bool DP4A = true>
cudaError_t launch_rows_t(const RowsArgs& a, cudaStream_t stream) {
  using S = RowsSmem<KT, VT>;
  auto kern = rows_kernel<QT, KT, VT, DP4A>;
  static std::atomic<bool> attr_set[64];   // per device; zero-initialised
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  if (!attr_set[dev]) {
    const cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, S::kTotal);
    if (e != cudaSuccess) return e;
    attr_set[dev] = true;
  }
  cudaError_t e;
  dim3 grid(a.max_splits, a.n_units);
  kern<<<grid, kRowsThreads, S::kTotal, stream>>>(a);
  e = cudaGetLastError();
  if (e != cudaSuccess || a.max_splits <= 1) return e;
  return launch_merge_rows(a, stream);
}

}  // namespace

cudaError_t launch_merge_rows(const RowsArgs& a, cudaStream_t stream) {
  merge_rows_kernel<<<a.n_units * kHeads, 256, 0, stream>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_rows(int q_dtype, int kv_dtype, const RowsArgs& a, cudaStream_t stream) {
#define KCA_ROWS_CASE(QD, KD) \
  if (q_dtype == QD && kv_dtype == KD) return launch_rows_t<QD, KD>(a, stream);
  KCA_ROWS_CASE(KCA_F32, KCA_F32)
  KCA_ROWS_CASE(KCA_F32, KCA_F16)
  KCA_ROWS_CASE(KCA_F32, KCA_BF16)
  KCA_ROWS_CASE(KCA_F16, KCA_F32)
  KCA_ROWS_CASE(KCA_F16, KCA_F16)
  KCA_ROWS_CASE(KCA_F16, KCA_BF16)
  KCA_ROWS_CASE(KCA_BF16, KCA_F32)
  KCA_ROWS_CASE(KCA_BF16, KCA_F16)
  KCA_ROWS_CASE(KCA_BF16, KCA_BF16)
#undef KCA_ROWS_CASE
  return cudaErrorInvalidValue;
}

cudaError_t launch_rows_q8(int q_dtype, int v_dtype, bool dp4a, const RowsArgs& a, cudaStream_t stream) {
#define KCA_Q8_CASE(QD, VD)                                                              \
  if (q_dtype == QD && v_dtype == VD)                                                    \
    return dp4a ? launch_rows_t<QD, KCA_I8, VD, true>(a, stream) : launch_rows_t<QD, KCA_I8, VD, false>(a, stream);
  KCA_Q8_CASE(KCA_F32, KCA_F32)
  KCA_Q8_CASE(KCA_F32, KCA_F16)
  KCA_Q8_CASE(KCA_F32, KCA_BF16)
  KCA_Q8_CASE(KCA_F16, KCA_F32)
  KCA_Q8_CASE(KCA_F16, KCA_F16)
  KCA_Q8_CASE(KCA_F16, KCA_BF16)
  KCA_Q8_CASE(KCA_BF16, KCA_F32)
  KCA_Q8_CASE(KCA_BF16, KCA_F16)
  KCA_Q8_CASE(KCA_BF16, KCA_BF16)
#undef KCA_Q8_CASE
  return cudaErrorInvalidValue;
}

}  // namespace kca

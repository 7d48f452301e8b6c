// kca_append.cu -- the step before the attention path: new K/V rows are
// rotated (K only; rotate-half RoPE with host-generated cos/sin rows) and
// written into the cache layout, in one kernel.
//
// The pages generate the rotary cos/sin rows on the host for every chunk
// instead of shipping a position table (Karume v0.8.0 release notes,
// "Features", conversation-window item; Gemma 4 E2B model page, "Context").
// The rotation pairs dim i with dim i + 128:
//   out[i]       = x[i]       cos[i]       - x[i + 128] sin[i]
//   out[i + 128] = x[i + 128] cos[i + 128] + x[i]       sin[i + 128]
// Every product and sum is rounded to f32 separately (no fused multiply-add),
// then to the cache type (round to nearest even), so the bytes written are a
// function of the inputs alone.
//
// One warp per row: lane l holds dims 4l .. 4l+3 of both halves, so each
// global access of a warp is 512 contiguous bytes (f32) or 256 (16-bit).
#include <cuda_runtime.h>

#include "../../include/kca.h"
#include "kca_common.cuh"
#include "kca_plan.h"

namespace kca {
namespace {

constexpr int kRowsPerBlock = 8;

template <int DT>
__device__ __forceinline__ void load4(const void* row, int dim, float (&x)[4]) {
  if (DT == KCA_F32) {
    const float4 f = *reinterpret_cast<const float4*>(static_cast<const float*>(row) + dim);
    x[0] = f.x; x[1] = f.y; x[2] = f.z; x[3] = f.w;
  } else {
    const uint2 u = *reinterpret_cast<const uint2*>(static_cast<const unsigned short*>(row) + dim);
    const uint32_t w[2] = {u.x, u.y};
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      float2 f;
      if (DT == KCA_F16) f = __half22float2(*reinterpret_cast<const __half2*>(&w[i]));
      else f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w[i]));
      x[2 * i] = f.x;
      x[2 * i + 1] = f.y;
    }
  }
}

template <int DT>
__device__ __forceinline__ void store4(void* row, int dim, const float (&x)[4]) {
  if (DT == KCA_F32) {
    *reinterpret_cast<float4*>(static_cast<float*>(row) + dim) = make_float4(x[0], x[1], x[2], x[3]);
  } else {
    uint32_t w[2];
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      if (DT == KCA_F16) {
        const __half2 h = __floats2half2_rn(x[2 * i], x[2 * i + 1]);
        w[i] = *reinterpret_cast<const uint32_t*>(&h);
      } else {
        const __nv_bfloat162 h = __floats2bfloat162_rn(x[2 * i], x[2 * i + 1]);
        w[i] = *reinterpret_cast<const uint32_t*>(&h);
      }
    }
    *reinterpret_cast<uint2*>(static_cast<unsigned short*>(row) + dim) = make_uint2(w[0], w[1]);
  }
}

struct AppendArgs {
  const void* k_new;
  const void* v_new;
  const float* cos;      // [n_rows][256] or null (no rotation)
  const float* sin;
  void* k_cache;
  void* v_cache;
  const int64_t* dst;    // device destinations, or null: dst0 + row
  int64_t dst0;
  int64_t cache_rows;
  int32_t n_rows;
  DeviceStatus* status;  // may be null
};

template <int IT, int KT>
__global__ void __launch_bounds__(kRowsPerBlock * 32) append_kv_kernel(const AppendArgs a) {
  const int64_t row = (int64_t)blockIdx.x * kRowsPerBlock + (threadIdx.x >> 5);
  if (row >= a.n_rows) return;
  const int lane = threadIdx.x & 31;
  const int64_t dst = a.dst != nullptr ? a.dst[row] : a.dst0 + row;
  if (dst < 0 || dst >= a.cache_rows) {   // only device destinations can be out of range
    if (lane == 0) record_error(a.status, kSiteAppend, kErrBadRow, (unsigned)row);
    return;
  }
  constexpr int kIn = ElemBytes<IT>::value, kOut = ElemBytes<KT>::value;
  const char* kin = static_cast<const char*>(a.k_new) + row * kDim * kIn;
  const char* vin = static_cast<const char*>(a.v_new) + row * kDim * kIn;
  char* kout = static_cast<char*>(a.k_cache) + dst * kDim * kOut;
  char* vout = static_cast<char*>(a.v_cache) + dst * kDim * kOut;
  const int d1 = 4 * lane, d2 = 128 + 4 * lane;
  float x1[4], x2[4], v1[4], v2[4];
  load4<IT>(kin, d1, x1);
  load4<IT>(kin, d2, x2);
  load4<IT>(vin, d1, v1);
  load4<IT>(vin, d2, v2);
  if (a.cos != nullptr) {
    const float* c = a.cos + row * kDim;
    const float* s = a.sin + row * kDim;
    const float4 c1 = *reinterpret_cast<const float4*>(c + d1), c2 = *reinterpret_cast<const float4*>(c + d2);
    const float4 s1 = *reinterpret_cast<const float4*>(s + d1), s2 = *reinterpret_cast<const float4*>(s + d2);
    const float cc1[4] = {c1.x, c1.y, c1.z, c1.w}, cc2[4] = {c2.x, c2.y, c2.z, c2.w};
    const float ss1[4] = {s1.x, s1.y, s1.z, s1.w}, ss2[4] = {s2.x, s2.y, s2.z, s2.w};
    float r1[4], r2[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      r1[i] = __fsub_rn(__fmul_rn(x1[i], cc1[i]), __fmul_rn(x2[i], ss1[i]));
      r2[i] = __fadd_rn(__fmul_rn(x2[i], cc2[i]), __fmul_rn(x1[i], ss2[i]));
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      x1[i] = r1[i];
      x2[i] = r2[i];
    }
  }
  store4<KT>(kout, d1, x1);
  store4<KT>(kout, d2, x2);
  store4<KT>(vout, d1, v1);
  store4<KT>(vout, d2, v2);
}

template <int IT, int KT>
cudaError_t launch_t(const AppendArgs& a, cudaStream_t s) {
  const int blocks = (int)((a.n_rows + kRowsPerBlock - 1) / kRowsPerBlock);
  append_kv_kernel<IT, KT><<<blocks, kRowsPerBlock * 32, 0, s>>>(a);
  return cudaGetLastError();
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace
}  // namespace kca

extern "C" int attn_append_kv(const void* k_new, const void* v_new, int32_t in_dtype, int32_t n_rows,
                              const float* rope_cos, const float* rope_sin, void* k_cache, void* v_cache,
                              int32_t kv_dtype, int64_t cache_rows, const int64_t* dst_rows_dev,
                              int64_t dst_row0, void* workspace, void* stream) {
  using namespace kca;
  if (!k_new || !v_new || !k_cache || !v_cache) return KCA_ERR_NULL;
  if ((rope_cos == nullptr) != (rope_sin == nullptr)) return KCA_ERR_NULL;
  if (in_dtype < KCA_F32 || in_dtype > KCA_BF16 || kv_dtype < KCA_F32 || kv_dtype > KCA_BF16)
    return KCA_ERR_DTYPE;
  if (n_rows < 1 || cache_rows < 1) return KCA_ERR_RANGE;
  if (dst_rows_dev == nullptr && (dst_row0 < 0 || dst_row0 > cache_rows - n_rows)) return KCA_ERR_RANGE;
  if (!aligned16(k_new) || !aligned16(v_new) || !aligned16(k_cache) || !aligned16(v_cache) ||
      (rope_cos && (!aligned16(rope_cos) || !aligned16(rope_sin))) ||
      (reinterpret_cast<uintptr_t>(dst_rows_dev) & 7u) != 0)
    return KCA_ERR_ALIGN;
  AppendArgs a{k_new, v_new, rope_cos, rope_sin, k_cache, v_cache, dst_rows_dev, dst_row0, cache_rows,
               n_rows, static_cast<DeviceStatus*>(workspace)};
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaError_t e = cudaErrorInvalidValue;
#define KCA_APPEND_CASE(I, K) \
  if (in_dtype == I && kv_dtype == K) e = launch_t<I, K>(a, s);
  KCA_APPEND_CASE(KCA_F32, KCA_F32)
  KCA_APPEND_CASE(KCA_F32, KCA_F16)
  KCA_APPEND_CASE(KCA_F32, KCA_BF16)
  KCA_APPEND_CASE(KCA_F16, KCA_F32)
  KCA_APPEND_CASE(KCA_F16, KCA_F16)
  KCA_APPEND_CASE(KCA_F16, KCA_BF16)
  KCA_APPEND_CASE(KCA_BF16, KCA_F32)
  KCA_APPEND_CASE(KCA_BF16, KCA_F16)
  KCA_APPEND_CASE(KCA_BF16, KCA_BF16)
#undef KCA_APPEND_CASE
  return e == cudaSuccess ? KCA_OK : KCA_ERR_CUDA;
}

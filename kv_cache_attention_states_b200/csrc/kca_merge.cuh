// kca_merge.cuh -- log-sum-exp merge of split partials, shared by the
// CUDA-core rows path (merge_rows_kernel) and the merge of context-shard
// records (attn_merge_partials).  The tensor-core prefill path has its own
// merge kernel in kca_prefill_tc.cu, and the tensor-core decode kernel merges
// in-kernel.
//
// A partial row is (m, l, acc[256]): m the reference max of its scores
// (m * mscale is in log2 units), l = sum 2^(x - m) and acc = sum 2^(x - m) v
// over its keys.  The merged row is
//   out = sum_i 2^((m_i - M) mscale) acc_i / sum_i 2^((m_i - M) mscale) l_i,
// M = max_i m_i (NaN as soon as one m_i is NaN).
//
// A group of W warps merges one row: warp g of the group takes the splits
// g, g+W, ..., lane k owning dims [8k, 8k+8); the W partial sums are then
// added through shared memory by the group's first warp.
#pragma once
#include <cstdint>

#include "kca_common.cuh"

namespace kca {

// Merges ns partial rows: split s has its (m, l) at ml + s*ml_stride and its
// acc at acc + s*acc_stride.  Two passes: the group first finds M, then every
// split's weight is independent of the others, so the loads of many splits
// are in flight at once.  g: warp index within the group; red: 264 floats of
// shared memory per warp of the group; bar_id: a named barrier owned by the
// group (used when W > 1).
template <int W>
__device__ __forceinline__ void merge_row(int ns, const float* ml, int64_t ml_stride,
                                          const float* acc, int64_t acc_stride, float mscale,
                                          float* out, float* red, int g, int lane, int bar_id,
                                          float* out_ml = nullptr) {
  float M = -INFINITY;
  for (int s = g * 32 + lane; s < ns; s += W * 32) M = max_nan(M, ml[s * ml_stride]);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) M = max_nan(M, __shfl_xor_sync(0xffffffffu, M, o));
  if (W > 1) {
    if (lane == 0) red[g * 264] = M;
    asm volatile("bar.sync %0, %1;" ::"r"(bar_id), "r"(W * 32) : "memory");
#pragma unroll
    for (int w = 0; w < W; ++w) M = max_nan(M, red[w * 264]);
    asm volatile("bar.sync %0, %1;" ::"r"(bar_id), "r"(W * 32) : "memory");
  }
  const float mu = M == -INFINITY ? 0.f : M;
  float L = 0.f, A[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll 4
  for (int s = g; s < ns; s += W) {
    const float f = exp2f((ml[s * ml_stride] - mu) * mscale);
    L += f * ml[s * ml_stride + 1];
    const float4* a = reinterpret_cast<const float4*>(acc + s * acc_stride + 8 * lane);
    const float4 a0 = a[0], a1 = a[1];
    A[0] += f * a0.x; A[1] += f * a0.y; A[2] += f * a0.z; A[3] += f * a0.w;
    A[4] += f * a1.x; A[5] += f * a1.y; A[6] += f * a1.z; A[7] += f * a1.w;
  }
  if (W > 1) {
    float* mine = red + g * 264;
    if (lane == 0) mine[1] = L;
#pragma unroll
    for (int i = 0; i < 8; ++i) mine[8 + 8 * lane + i] = A[i];
    asm volatile("bar.sync %0, %1;" ::"r"(bar_id), "r"(W * 32) : "memory");
    if (g != 0) return;
    for (int w = 1; w < W; ++w) {
      const float* o = red + w * 264;
      L += o[1];
#pragma unroll
      for (int i = 0; i < 8; ++i) A[i] += o[8 + 8 * lane + i];
    }
  }
  // out_ml set: the merged partial (M, L) and unnormalised acc instead; a
  // row of empty partials only (M = -inf, L = 0) is exactly zero
  const float inv = out_ml != nullptr ? 1.f : (M == -INFINITY && L == 0.f) ? 0.f : 1.f / L;
  if (out_ml != nullptr && lane == 0) {
    out_ml[0] = M;
    out_ml[1] = L;
  }
  float4* o4 = reinterpret_cast<float4*>(out + 8 * lane);
  o4[0] = make_float4(A[0] * inv, A[1] * inv, A[2] * inv, A[3] * inv);
  o4[1] = make_float4(A[4] * inv, A[5] * inv, A[6] * inv, A[7] * inv);
}

}  // namespace kca

// kca_context.cu -- merge of the partial-softmax records of context shards.
//
// Each record holds, per (sequence, head), (m, l) and the unnormalised acc
// of the keys one shard holds; the merged output is the log-sum-exp
// combination of the records, taken in record order (merge_row, one CTA per
// (sequence, head), its eight warps taking interleaved records).
#include "kca_common.cuh"
#include "kca_merge.cuh"
#include "kca_plan.h"
#include "kca_rows.h"

namespace kca {
namespace {

constexpr float kLog2eMerge = 1.4426950408889634f;   // m is in natural units

__global__ void __launch_bounds__(256) merge_partials_kernel(int n_parts, int batch, const float* parts,
                                                             int64_t part_stride, float* out) {
  const int row = blockIdx.x;   // sequence * 8 + head
  __shared__ float red[8 * 264];
  merge_row<8>(n_parts, parts + (int64_t)row * 2, part_stride,
               parts + (int64_t)batch * kHeads * 2 + (int64_t)row * kDim, part_stride, kLog2eMerge,
               out + (int64_t)row * kDim, red, threadIdx.x >> 5, threadIdx.x & 31, 1);
}

}  // namespace

cudaError_t launch_merge_partials(int n_parts, int batch, const float* parts, int64_t part_stride, float* out,
                                  cudaStream_t stream) {
  merge_partials_kernel<<<batch * kHeads, 256, 0, stream>>>(n_parts, batch, parts, part_stride, out);
  return cudaGetLastError();
}

}  // namespace kca

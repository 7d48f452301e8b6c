// kca_tc.h -- launch interface of the tensor-core prefill kernels.
#pragma once
#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

#include "kca_plan.h"

namespace kca {

struct TcArgs {
  const void* q;      // [rows][8][256], 16-bit
  float* out;         // [rows][8][256]
  float* part_ml;     // [n_slots][128][2]  (m in log2 units, l)
  float* part_acc;    // [n_slots][128][256]
  void* status;       // workspace status header
  TcPlan plan;
  float scale_log2;   // scale * log2(e)
};

// tmk / tmv: 2-D tensor maps over the rows [plan.kv_lo, plan.ctx_len) of the
// K and V caches, inner extent 256, box 64 x 64, 128-byte swizzle, zero fill.
cudaError_t launch_prefill_tc(int dtype, const CUtensorMap& tmk, const CUtensorMap& tmv,
                              const TcArgs& a, cudaStream_t stream);

}  // namespace kca

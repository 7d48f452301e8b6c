// kca_rows.h -- launch interface of the rows kernels (decode split + merge).
#pragma once
#include <cstdint>
#include <cuda_runtime.h>

#include "../../include/kca.h"

namespace kca {

struct RowsArgs {
  const void* q;         // [n_units][8][256]
  const void* k;         // cache rows
  const void* v;
  float* out;            // [n_units][8][256]
  float* part_ml;        // [n_units * max_splits][8][2]  (m, l), or null
  float* part_acc;       // [n_units * max_splits][8][256], or null
  void* status;          // workspace status header
  int64_t seq_rows;      // decode: cache rows per sequence (capacity)
  int64_t chunk_start;   // prefill: position of unit 0
  int32_t mode;          // 0: decode (unit = sequence), 1: prefill (unit = row of sequence 0)
  int32_t n_units;
  int32_t split_len;
  int32_t max_splits;
  int32_t window;
  float scale;
  int64_t ctx[KCA_MAX_BATCH];  // decode: ctx_len per sequence
};

cudaError_t launch_rows(int q_dtype, int kv_dtype, const RowsArgs& a, cudaStream_t stream);

}  // namespace kca

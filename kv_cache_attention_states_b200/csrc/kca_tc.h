// kca_tc.h -- launch interface of the tensor-core prefill kernels.
#pragma once
#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

#include "kca_plan.h"

namespace kca {

constexpr int kTcMaxItems = 80;    // work items (CTA pairs) of one call
constexpr int kTcMaxTiles = 48;    // 768 rows / 16

// One work item of a CTA pair, filled in on the host from the plan so that
// no CTA has to walk the plan itself.
struct TcItemArg {
  int32_t kt_begin;   // key tiles relative to plan.kv_lo
  int32_t kt_end;
  int16_t pair;       // row tiles 2 pair (even CTA) and 2 pair + 1 (odd CTA)
  int16_t slot[2];    // partial slot of each tile, -1 when the pair is not split
};

struct TcArgs {
  const void* q;      // [rows][8][256], 16-bit
  float* out;         // [rows][8][256]
  float* part_ml;     // [n_slots][128][2]  (m in log2 units, l)
  float* part_acc;    // [n_slots][128][256]
  void* status;       // workspace status header
  TcPlan plan;
  float scale_log2;   // scale * log2(e)
  int32_t rag_tile;   // split tile whose partials store only their valid rows (tmpart_rag), or -1
  TcItemArg items[kTcMaxItems];
  int16_t tile_first_slot[kTcMaxTiles];
  int16_t tile_items[kTcMaxTiles];
};

// Fills the item and tile tables from a.plan; false when they would not fit
// the plan (launch tables, partial slots or the keys the maps cover).
bool fill_tc_tables(TcArgs& a);

// tmk / tmv: 2-D tensor maps over the rows [plan.kv_lo, plan.ctx_len) of the
// K and V caches, inner extent 256, 128-byte swizzle, zero fill; boxes of 64
// elements x 64 rows (K and V).  tmq: the Q chunk as [rows * 8][256]
// 16-bit, boxes 64 x 128.  tmo / tmpart: out as [rows * 8][256] f32 and the
// partials as [n_slots * 128][256] f32, boxes 32 x 128; tmpart_rag: the
// same partials with boxes of 32 x (8 x the valid rows of tile a.rag_tile);
// all 128-byte swizzle.
cudaError_t launch_prefill_tc(int dtype, const CUtensorMap& tmk, const CUtensorMap& tmv,
                              const CUtensorMap& tmq, const CUtensorMap& tmo, const CUtensorMap& tmpart,
                              const CUtensorMap& tmpart_rag, const TcArgs& a, cudaStream_t stream);

}  // namespace kca

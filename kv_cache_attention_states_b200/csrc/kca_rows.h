// kca_rows.h -- launch interface of the rows kernels (decode split + merge).
#pragma once
#include <cstdint>
#include <cuda.h>
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
  int64_t seq_rows;      // decode, batched rows: cache rows per sequence (capacity)
  int64_t chunk_start;   // prefill: position of unit 0
  int32_t mode;          // 0: decode (unit = sequence), 1: prefill (unit = row of sequence 0),
                         // 2: batched rows (unit = row i of sequence unit / rows_per_seq)
  int32_t rows_per_seq;  // mode 2: query rows per sequence, at ctx[b] - rows_per_seq .. ctx[b] - 1
  int32_t unit_rows;     // multi-row units: rows per unit (kMultiRows, or kMultiRowsWide for tcgen05)
  int32_t n_units;
  int32_t split_len;
  int32_t max_splits;
  int32_t window;
  float scale;
  // tensor-core path only: CTAs per cluster (1, 2, 4, 8), clusters per unit at
  // most, self-resetting tickets [n_units][8] and cluster partials
  // [n_units][max_clusters][8] x (m, l) / acc[256].
  int32_t cluster;
  int32_t max_clusters;
  int32_t* tickets;
  float* cpart_ml;
  float* cpart_acc;
  // decode with device context lengths: ctx_dev[unit] (each in 0..ctx_bound)
  // replaces ctx[unit], and each unit cuts its keys into max_splits splits
  // itself (rows_split_len); null for the host-array form.
  const int64_t* ctx_dev;
  int64_t ctx_bound;
  // Context shard (decode): cache row r of a sequence holds position
  // key_begin + r, and only positions [key_begin, key_end) are seen
  // (key_end <= 0: no upper end).  Zero for a whole cache.
  int64_t key_begin;
  int64_t key_end;
  // Partial-softmax output (decode): non-null, each (unit, head) gets
  // (m, l) here -- m the max scaled score, l the sum of exp(s - m) -- and
  // its unnormalised sum of exp(s - m) v in out; null: out = that sum / l.
  float* out_ml;
  // Extents of the buffers the kernels address by computed offsets (checked
  // in bounds-checked builds): cache rows the K / V pointers and maps cover,
  // and partial slots (split or cluster partials) the workspace holds.
  int64_t cache_rows;
  int64_t part_slots;
  int64_t ctx[KCA_MAX_BATCH];  // decode: ctx_len per sequence
};

// Rows of one unit of the batched multi-row kernels: 4 (both kernels), or 8
// (the tcgen05 kernel, when a call has more than 4 rows per sequence).
constexpr int kMultiRows = 4;
constexpr int kMultiRowsWide = 8;

#if defined(__CUDACC__)
}  // namespace kca
#include "kca_common.cuh"
namespace kca {
// Context length of decode unit `unit`.  A device value outside
// 0..ctx_bound is recorded in the status word (when `record`) and read as an
// empty context, so no row past the bound is ever touched.
__device__ __forceinline__ int64_t rows_ctx(const RowsArgs& a, int unit, bool record) {
  if (a.ctx_dev == nullptr) return a.ctx[unit];
  const int64_t c = a.ctx_dev[unit];
  if (c >= 0 && c <= a.ctx_bound) return c;
  if (record) record_error(static_cast<DeviceStatus*>(a.status), kSiteCtx, kErrBadCtx, (unsigned)unit);
  return 0;
}
// Position of the query of `unit`, and the cache row of position 0 of its
// sequence (*seq_base; before the shard offset).
__device__ __forceinline__ int64_t rows_unit_pos(const RowsArgs& a, int unit, bool record, int64_t* seq_base) {
  if (a.mode == 1) {
    *seq_base = 0;
    return a.chunk_start + unit;
  }
  if (a.mode == 2) {
    const int b = unit / a.rows_per_seq;
    *seq_base = (int64_t)b * a.seq_rows;
    return a.ctx[b] - a.rows_per_seq + unit % a.rows_per_seq;
  }
  *seq_base = (int64_t)unit * a.seq_rows;
  return rows_ctx(a, unit, record) - 1;
}
// Visible keys [*lo, *lo + n) of the query at pos within the cache's shard.
__device__ __forceinline__ int64_t rows_keys(const RowsArgs& a, int64_t pos, int64_t* lo) {
  return shard_visible(pos, a.window, a.key_begin, a.key_end, lo);
}
// Final writes of (unit, head) h: rows_write_ml stores its (M, L) when the
// output is a partial-softmax record (a.out_ml set); rows_final gives the
// value of one output dim, acc / L normalised or acc itself in a record.  An
// empty row (M = -inf, L = 0) is exactly zero, or (-inf, 0, 0) in a record.
__device__ __forceinline__ void rows_write_ml(const RowsArgs& a, int unit, int h, float M, float L) {
  if (a.out_ml != nullptr) {
    a.out_ml[((int64_t)unit * kHeads + h) * 2 + 0] = M;
    a.out_ml[((int64_t)unit * kHeads + h) * 2 + 1] = L;
  }
}
__device__ __forceinline__ float rows_final(const RowsArgs& a, float acc, float M, float L) {
  if (a.out_ml != nullptr) return acc;
  return (M == -INFINITY && L == 0.f) ? 0.f : acc / L;
}
// Unit u of a batched call in multi-row units (a.unit_rows rows each):
// sequence *b, first row *i0 (of the sequence's rows), *nr rows; positions
// ctx[b] - rows_per_seq + i0 + r.
__device__ __forceinline__ void multirow_unit(const RowsArgs& a, int u, int* b, int* i0, int* nr);
// Keys per split of a unit with nkeys visible keys: the host plan's length,
// or with device context lengths the smallest multiple of `quantum` (>= 64)
// that cuts nkeys into at most max_splits splits.
__device__ __forceinline__ int32_t rows_split_len(const RowsArgs& a, int64_t nkeys, int quantum) {
  if (a.ctx_dev == nullptr) return a.split_len;
  int64_t s = (nkeys + a.max_splits - 1) / a.max_splits;
  s = (s + quantum - 1) / quantum * quantum;
  return (int32_t)(s < 64 ? 64 : s);
}
__device__ __forceinline__ void multirow_unit(const RowsArgs& a, int u, int* b, int* i0, int* nr) {
  const int ur = a.unit_rows;
  const int blocks = (a.rows_per_seq + ur - 1) / ur;
  *b = u / blocks;
  *i0 = (u % blocks) * ur;
  const int left = a.rows_per_seq - *i0;
  *nr = left < ur ? left : ur;
}
#endif

cudaError_t launch_rows(int q_dtype, int kv_dtype, const RowsArgs& a, cudaStream_t stream);

// The CUDA-core rows kernel with packed int8 K rows (KCA_I8) and V of
// v_dtype: the quantised-dot variant; dp4a selects the instruction over its
// emulation (kca_q8.cu).  Merges its splits like launch_rows.
cudaError_t launch_rows_q8(int q_dtype, int v_dtype, bool dp4a, const RowsArgs& a, cudaStream_t stream);

// Log-sum-exp merge of the split partials in a (units with more than one split).
cudaError_t launch_merge_rows(const RowsArgs& a, cudaStream_t stream);

// Merge of n_parts partial records (layout of attn_decode_partial; record p
// at parts + p * part_stride floats) into out [batch][8][256] (kca_context.cu).
cudaError_t launch_merge_partials(int n_parts, int batch, const float* parts, int64_t part_stride, float* out,
                                  cudaStream_t stream);

// attn_decode's host checks that need no device and no workspace: pointers,
// geometry, dtypes, ranges, scale, alignment (KCA_OK or the KCA_ERR_* code).
int decode_args_check(const void* q, int32_t q_dtype, const void* k_cache, const void* v_cache, int32_t kv_dtype,
                      int32_t n_q_heads, int32_t n_kv_heads, int32_t head_dim, int64_t capacity, int32_t batch,
                      const int64_t* ctx_len, float scale, const float* out);

// attn_decode's body: validates every argument, plans, and launches.  With
// clear_header the workspace's first KCA_WORKSPACE_HEADER bytes are zeroed on
// `stream` (after validation, before the launch); attn_decode passes false.
int decode_entry(const void* q, int32_t q_dtype, const void* k_cache, const void* v_cache, int32_t kv_dtype,
                 int32_t n_q_heads, int32_t n_kv_heads, int32_t head_dim, int64_t capacity, int32_t batch,
                 const int64_t* ctx_len, int32_t window, float scale, float* out, void* workspace,
                 size_t workspace_bytes, void* stream, bool clear_header);

// The dot-product canary of the quantised-dot decode (kca_q8.cu): once per
// device, the dp4a instruction, its emulation and the int8 MMA against known
// answers; *mask: 1 dp4a sane, 2 emulation sane, 4 int8 MMA sane.
// KCA_ERR_DEVICE when neither dp4a nor its emulation is, KCA_ERR_CUDA when
// the check could not run.
int dot_canary(cudaStream_t s, int* mask);

// Tensor-core rows kernel with packed int8 K rows: tmk maps the codes (uint8
// [rows][272], 128 x 64 boxes, 128-byte swizzle), tms their scale column
// (16 x 64 boxes at x = 256, no swizzle), tmv the 16-bit V rows.
cudaError_t launch_decode_mma_q8(int q_dtype, int v_dtype, const CUtensorMap& tmk, const CUtensorMap& tms,
                                 const CUtensorMap& tmv, const RowsArgs& a, cudaStream_t stream);

// Batched short chunks on the tensor cores (mode 2, 16-bit K/V): units of up
// to a.unit_rows consecutive rows of one sequence (n_units = batch x
// ceil(rows / unit_rows); kMultiRows for the mma.sync kernel, kMultiRows or
// kMultiRowsWide for tcgen05), the union of their keys cut into splits of
// split_len; per-row split partials in part_ml / part_acc
// ([batch * rows][max_splits][8]).  launch_decode_multirow: mma.sync
// fragments (kca_decode_mma.cu), the partials merged by a second kernel
// (launch_multirow_merge); launch_rows_tc: tcgen05 MMAs with TMEM
// accumulators (kca_rows_tc.cu), the partials merged in-kernel by the last
// split of each unit (per-unit tickets in a.tickets) or, without tickets, by
// the merge kernel.  tmk / tmv as for launch_decode_mma.
cudaError_t launch_decode_multirow(int q_dtype, int kv_dtype, const CUtensorMap& tmk, const CUtensorMap& tmv,
                                   const RowsArgs& a, cudaStream_t stream);
cudaError_t launch_rows_tc(int q_dtype, int kv_dtype, const CUtensorMap& tmk, const CUtensorMap& tmv,
                           const RowsArgs& a, cudaStream_t stream);
// Most splits per unit that the tcgen05 kernel merges in-kernel (a.tickets
// set); with more, a.tickets is null and launch_rows_tc adds the merge kernel.
constexpr int kRowsTcMergeSplits = 16;
cudaError_t launch_multirow_merge(const RowsArgs& a, cudaStream_t stream);

// Clusters of c CTAs of the tensor-core rows kernel that fit on the device at
// once (0 on failure).
int decode_mma_cluster_capacity(int c);

// Tensor-core variant for 16-bit K/V (kca_decode_mma.cu); tmk / tmv map the
// cache rows [rows][256] with 64 x 64 boxes and 128-byte swizzle.  Merges in
// the same kernel (clusters + tickets).
cudaError_t launch_decode_mma(int q_dtype, int kv_dtype, const CUtensorMap& tmk, const CUtensorMap& tmv,
                              const RowsArgs& a, cudaStream_t stream);

}  // namespace kca

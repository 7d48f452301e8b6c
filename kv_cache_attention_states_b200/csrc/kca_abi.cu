// kca_abi.cu -- the extern "C" entry points of libkca.so (declared and
// documented in include/kca.h): argument validation on the host, planning,
// workspace carving, tensor-map encoding and kernel launches.  Nothing here
// allocates device memory or synchronises a stream (attn_device_status aside,
// which exists to read the device status word).
#include <atomic>
#include <cuda.h>
#include <cuda_runtime.h>

#include <cmath>
#include <vector>

#include "../../include/kca.h"
#include "kca_plan.h"
#include "kca_rows.h"
#include "kca_tc.h"

namespace {

using kca::kDim;
using kca::kHeads;

constexpr size_t kAlign = 256;
size_t align_up(size_t x) { return (x + kAlign - 1) / kAlign * kAlign; }
constexpr size_t kStatusBytes = 256;   // header: status word, then the merge counters
static_assert(KCA_WORKSPACE_HEADER >= kStatusBytes + KCA_MAX_CHUNK_ROWS * kHeads * 4, "header");
static_assert(KCA_MAX_BATCH <= KCA_MAX_CHUNK_ROWS, "header counters cover both paths");

bool dtype_ok(int32_t d) { return d == KCA_F32 || d == KCA_F16 || d == KCA_BF16; }
bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int geometry_status(int32_t hq, int32_t hkv, int32_t d) {
  return (hq == KCA_N_Q_HEADS && hkv == KCA_N_KV_HEADS && d == KCA_HEAD_DIM) ? KCA_OK
                                                                             : KCA_ERR_GEOMETRY;
}

// SM count of the current device (cached per device).
int current_sms(int* out) {
  static std::atomic<int> cache[64];   // zero-initialised
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return KCA_ERR_CUDA;
  if (dev >= 0 && dev < 64 && cache[dev] > 0) {
    *out = cache[dev];
    return KCA_OK;
  }
  int sms = 0;
  if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || sms <= 0)
    return KCA_ERR_CUDA;
  if (dev >= 0 && dev < 64) cache[dev] = sms;
  *out = sms;
  return KCA_OK;
}

// Paths pinned by attn_force_path (-1: automatic), read once per call.
std::atomic<int> g_prefill_path{-1};
std::atomic<int> g_rows_path{-1};
std::atomic<int> g_batch_path{-1};

// A forced prefill path (attn_force_path) wins where eligible; otherwise the
// rules in kca.h choose.  Chunks of fewer than 16 rows: the rows path streams the visible keys once
// per row (the first row from HBM, the rest mostly from L2), the tensor-core
// path once per chunk but with a fixed cost of ~9 us (two launches, the
// partials of the split tile, the merge).  B200 graph-replay timings of both
// paths (1-15 rows at 1K-64K keys) put the crossover at about 3 rows once
// the rows see 12K keys or more; below 12K keys the rows path wins up to 15
// rows.
// Chunks of 2-15 rows on a 16-bit cache that the tensor-core path does not
// take (mixed dtypes, or 2 rows) go to multi-row units once the first row
// sees 12,288 keys: each K/V stage crosses to the SM once per 4 or 8 rows
// (at 131,072 keys, 8 f32-query rows on a bf16 cache: 110 us on the rows
// path, 40 us on multi-row units; 15 rows: 231 against 52 us).
int prefill_route(int32_t q_dtype, int32_t kv_dtype, int64_t chunk_start, int32_t rows, int32_t window);
bool use_tc(int32_t q_dtype, int32_t kv_dtype, int64_t chunk_start, int32_t rows, int32_t window) {
  return prefill_route(q_dtype, kv_dtype, chunk_start, rows, window) == 1;
}

std::vector<int64_t> prefill_unit_keys(int64_t chunk_start, int32_t rows, int32_t window) {
  std::vector<int64_t> nk(rows);
  for (int32_t i = 0; i < rows; ++i) nk[i] = kca::n_visible(chunk_start + i, window);
  return nk;
}
std::vector<int64_t> decode_unit_keys(int32_t batch, const int64_t* ctx_len, int32_t window) {
  std::vector<int64_t> nk(batch);
  for (int32_t b = 0; b < batch; ++b) nk[b] = kca::n_visible(ctx_len[b] - 1, window);
  return nk;
}
// Batched short chunks: unit b * rows + i is row i of sequence b, at
// position ctx_len[b] - rows + i.
std::vector<int64_t> batch_unit_keys(int32_t batch, int32_t rows, const int64_t* ctx_len, int32_t window) {
  std::vector<int64_t> nk((size_t)batch * rows);
  for (int32_t b = 0; b < batch; ++b)
    for (int32_t i = 0; i < rows; ++i) nk[(size_t)b * rows + i] = kca::n_visible(ctx_len[b] - rows + i, window);
  return nk;
}

// Multi-row units of the tensor-core batched path: unit b * blocks + k holds
// rows ur k .. ur k + ur - 1 (at most) of sequence b; its keys are the union
// of theirs.
std::vector<int64_t> multirow_unit_keys(int32_t batch, int32_t rows, const int64_t* ctx_len, int32_t window,
                                        int32_t ur) {
  const int32_t blocks = (rows + ur - 1) / ur;
  std::vector<int64_t> nk((size_t)batch * blocks);
  for (int32_t b = 0; b < batch; ++b)
    for (int32_t k = 0; k < blocks; ++k) {
      const int32_t i0 = k * ur;
      const int32_t nr = rows - i0 < ur ? rows - i0 : ur;
      const int64_t pos0 = ctx_len[b] - rows + i0;
      nk[(size_t)b * blocks + k] = pos0 + nr - kca::lo_of(pos0, window);
    }
  return nk;
}
size_t multirow_ws_bytes(int32_t batch, int32_t rows, const kca::RowsPlan& p) {
  if (p.max_splits <= 1) return KCA_WORKSPACE_HEADER;
  const size_t slots = (size_t)batch * rows * p.max_splits;
  return KCA_WORKSPACE_HEADER + align_up(slots * kHeads * 2 * 4) + align_up(slots * kHeads * kDim * 4);
}

int batch_args_status(int64_t capacity, int32_t batch, int32_t rows, const int64_t* ctx_len) {
  if (capacity < 1 || capacity > KCA_MAX_POSITION) return KCA_ERR_RANGE;
  if (batch < 1 || batch > KCA_MAX_BATCH || rows < 1 || rows > KCA_MAX_BATCH_ROWS) return KCA_ERR_RANGE;
  for (int32_t b = 0; b < batch; ++b)
    if (ctx_len[b] < rows || ctx_len[b] > capacity) return KCA_ERR_RANGE;
  return KCA_OK;
}

// Keys of each decode query that a context shard [key_begin, key_end) holds.
std::vector<int64_t> shard_unit_keys(int32_t batch, const int64_t* ctx_len, int32_t window, int64_t key_begin,
                                     int64_t key_end) {
  std::vector<int64_t> nk(batch);
  int64_t lo = 0;
  for (int32_t b = 0; b < batch; ++b) nk[b] = kca::shard_visible(ctx_len[b] - 1, window, key_begin, key_end, &lo);
  return nk;
}

size_t rows_ws_bytes(const kca::RowsPlan& p) {
  if (p.max_splits <= 1) return KCA_WORKSPACE_HEADER;
  const size_t slots = (size_t)p.n_units * p.max_splits;
  return KCA_WORKSPACE_HEADER + align_up(slots * kHeads * 2 * 4) + align_up(slots * kHeads * kDim * 4);
}
size_t tc_ws_bytes(const kca::TcPlan& p) {
  if (p.n_slots == 0) return KCA_WORKSPACE_HEADER;
  const size_t slots = (size_t)p.n_slots;
  return KCA_WORKSPACE_HEADER + align_up(slots * 128 * 2 * 4) + align_up(slots * 128 * kDim * 4);
}

int prefill_args_status(int64_t capacity, int64_t chunk_start, int32_t chunk_rows) {
  if (capacity < 1 || capacity > KCA_MAX_POSITION) return KCA_ERR_RANGE;
  if (chunk_rows < 1 || chunk_rows > KCA_MAX_CHUNK_ROWS) return KCA_ERR_RANGE;
  if (chunk_start < 0 || chunk_start + chunk_rows > capacity) return KCA_ERR_RANGE;
  return KCA_OK;
}

int shard_args_status(int64_t capacity, int32_t batch, const int64_t* ctx_len, int64_t key_begin) {
  if (capacity < 1 || key_begin < 0 || key_begin > KCA_MAX_POSITION - capacity) return KCA_ERR_RANGE;
  if (batch < 1 || batch > KCA_MAX_BATCH) return KCA_ERR_RANGE;
  for (int32_t b = 0; b < batch; ++b)
    if (ctx_len[b] < 0 || ctx_len[b] > KCA_MAX_POSITION) return KCA_ERR_RANGE;
  return KCA_OK;
}

int decode_args_status(int64_t capacity, int32_t batch, const int64_t* ctx_len) {
  if (capacity < 1 || capacity > KCA_MAX_POSITION) return KCA_ERR_RANGE;
  if (batch < 1 || batch > KCA_MAX_BATCH) return KCA_ERR_RANGE;
  for (int32_t b = 0; b < batch; ++b)
    if (ctx_len[b] < 0 || ctx_len[b] > capacity) return KCA_ERR_RANGE;
  return KCA_OK;
}

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  // Looked up once; a function-local static is initialised thread-safely.
  static const EncodeTiledFn fn = []() -> EncodeTiledFn {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      return reinterpret_cast<EncodeTiledFn>(p);
    return nullptr;
  }();
  return fn;
}

// A tensor map is a pure function of its encode arguments, so the last few
// encodings of each host thread are kept and a repeated argument set (the
// same cache or chunk buffer call after call) is copied instead of
// re-encoded.  All maps here are 2-D, 128-byte swizzled, zero-filled.
bool encode_2d(CUtensorMap* m, CUtensorMapDataType t, const void* base, const cuuint64_t (&dims)[2],
               cuuint64_t stride, const cuuint32_t (&box)[2],
               CUtensorMapSwizzle swizzle = CU_TENSOR_MAP_SWIZZLE_128B) {
  struct Entry {
    const void* base;
    cuuint64_t dims[2];
    cuuint64_t stride;
    cuuint32_t box[2];
    int t;
    int swizzle;
    bool valid;
    CUtensorMap map;
  };
  constexpr int kEntries = 16;
  thread_local Entry cache[kEntries] = {};
  thread_local int next = 0;
  for (int i = 0; i < kEntries; ++i) {
    const Entry& e = cache[i];
    if (e.valid && e.base == base && e.t == (int)t && e.dims[0] == dims[0] && e.dims[1] == dims[1] &&
        e.stride == stride && e.box[0] == box[0] && e.box[1] == box[1] && e.swizzle == (int)swizzle) {
      *m = e.map;
      return true;
    }
  }
  EncodeTiledFn fn = encode_fn();
  if (fn == nullptr) return false;
  cuuint64_t strides[1] = {stride};
  cuuint32_t estr[2] = {1, 1};
  if (fn(m, t, 2, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle,
         CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return false;
  Entry& e = cache[next];
  next = (next + 1) % kEntries;
  e.base = base;
  e.dims[0] = dims[0];
  e.dims[1] = dims[1];
  e.stride = stride;
  e.box[0] = box[0];
  e.box[1] = box[1];
  e.t = (int)t;
  e.swizzle = (int)swizzle;
  e.map = *m;
  e.valid = true;
  return true;
}

// Map over rows [kv_lo, ctx_len) of one cache: inner extent 256 elements,
// boxes of 64 elements x box_rows rows, 128-byte swizzle, zero fill outside.
bool encode_kv_map(CUtensorMap* m, const void* cache, int32_t dtype, int64_t kv_lo, int64_t ctx_len,
                   uint32_t box_rows) {
  const char* base = static_cast<const char*>(cache) + kv_lo * kDim * 2;
  const cuuint64_t dims[2] = {(cuuint64_t)kDim, (cuuint64_t)(ctx_len - kv_lo)};
  const cuuint32_t box[2] = {64, box_rows};
  const CUtensorMapDataType t =
      dtype == KCA_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
  return encode_2d(m, t, base, dims, (cuuint64_t)kDim * 2, box);
}

// 2-D map over `rows` rows of 256 elements (f32 or 16-bit), box {box_x,
// box_rows}, 128-byte swizzle; reads past the extent return zeros, stores are
// clipped.
bool encode_rows_map(CUtensorMap* m, const void* base, int32_t dtype, int64_t rows, uint32_t box_x,
                     uint32_t box_rows = 128) {
  if (rows < 1) return false;
  const int esz = dtype == KCA_F32 ? 4 : 2;
  const cuuint64_t dims[2] = {(cuuint64_t)kDim, (cuuint64_t)rows};
  const cuuint32_t box[2] = {box_x, box_rows};
  const CUtensorMapDataType t = dtype == KCA_F32    ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32
                                : dtype == KCA_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16
                                                    : CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
  return encode_2d(m, t, base, dims, (cuuint64_t)kDim * esz, box);
}

void carve(void* ws, size_t ml_bytes, float** ml, float** acc) {
  char* p = static_cast<char*>(ws) + KCA_WORKSPACE_HEADER;
  *ml = reinterpret_cast<float*>(p);
  *acc = reinterpret_cast<float*>(p + align_up(ml_bytes));
}

// 16-bit caches take the tensor-core rows kernel unless attn_force_path pins
// the CUDA-core one (tests compare the two on the same inputs).
bool use_rows_mma(int32_t kv_dtype) {
  if (kv_dtype != KCA_F16 && kv_dtype != KCA_BF16) return false;
  return g_rows_path.load(std::memory_order_relaxed) != 0;
}

// The batched call takes the multi-row tensor-core kernel for 16-bit caches
// and more than one row per sequence (one row per sequence is decode).
bool use_multirow(int32_t kv_dtype, int32_t rows) { return rows > 1 && use_rows_mma(kv_dtype); }
// Multi-row units take the tcgen05 kernel unless attn_force_path pins the
// mma.sync one (op 2, path 0).
bool use_batch_tc() { return g_batch_path.load(std::memory_order_relaxed) != 0; }

// Route of a prefill chunk: 1 the tensor-core path, 2 multi-row units, 0 the
// rows path.  A forced route (attn_force_path op 0) wins where eligible.
int prefill_route(int32_t q_dtype, int32_t kv_dtype, int64_t chunk_start, int32_t rows, int32_t window) {
  const bool tc_ok = q_dtype == kv_dtype && (q_dtype == KCA_F16 || q_dtype == KCA_BF16);
  const bool mr_ok = use_multirow(kv_dtype, rows) && rows <= KCA_MAX_BATCH_ROWS;
  const int forced = g_prefill_path.load(std::memory_order_relaxed);
  if (forced == 0) return 0;
  if (forced == 1) return tc_ok ? 1 : 0;
  if (forced == 2) return mr_ok ? 2 : 0;
  const int64_t keys = kca::n_visible(chunk_start, window);
  if (tc_ok && (rows >= kca::kRowTile || (rows >= 3 && keys >= 12288))) return 1;
  if (mr_ok && keys >= 12288) return 2;
  return 0;
}

// Plan of the tensor-core rows kernel.  Each cluster size c in {8, 4, 2}
// (and c = 1 when every unit fits one split, so nothing is merged) gets the
// plan that fills the clusters resident at once; the one with the lowest
// estimated time wins.  The estimate, from decode sweeps on B200: the key
// stream takes the longer of all bytes at 6.5 TB/s and one split at 50 GB/s
// per SM, times the waves of clusters; a unit with several clusters adds
// 1.5 us (partials, fence, ticket) and 0.6 us per round of loads of the
// final merge.
// capacity: resident clusters of 2, 4 and 8 CTAs (nullptr: the current
// device's, measured once per device).
kca::RowsPlan mma_rows_plan(int32_t n_units, const int64_t* nkeys, int sms, int* cluster,
                            const int32_t* capacity = nullptr) {
  kca::RowsPlan best{};
  int best_c = 0;
  double best_t = 0.0;
  double total_keys = 0.0;
  for (int32_t u = 0; u < n_units; ++u) total_keys += (double)nkeys[u];
  for (int c = 8; c >= 1; c /= 2) {
    const int ci = c == 2 ? 0 : (c == 4 ? 1 : 2);
    int slots = c == 1 ? sms : (capacity != nullptr ? capacity[ci] : kca::decode_mma_cluster_capacity(c));
    if (slots > kca::kRowsMmaMaxClusterParts) slots = kca::kRowsMmaMaxClusterParts;
    if (slots <= 0) continue;
    const kca::RowsPlan p = kca::make_cluster_rows_plan(n_units, nkeys, c, slots);
    const int max_clusters = (p.max_splits + c - 1) / c;
    if (c == 1 && max_clusters > 1) continue;   // one CTA would merge all eight heads
    int64_t n_clusters = 0;
    for (int32_t u = 0; u < n_units; ++u) n_clusters += (kca::rows_n_splits(nkeys[u], p.split_len) + c - 1) / c;
    const double waves = (double)((n_clusters + slots - 1) / slots);
    const double t_hbm = total_keys * 1024.0 / 6.5e12;
    const double t_sm = waves * (double)p.split_len * 1024.0 / 50e9;
    double t = t_hbm > t_sm ? t_hbm : t_sm;
    if (max_clusters > 1) t += 1.5e-6 + 0.6e-6 * (1 + (kHeads / c) * ((max_clusters + 31) / 32));
    if (best_c == 0 || t < best_t) {
      best = p;
      best_c = c;
      best_t = t;
    }
  }
  *cluster = best_c;
  return best;
}

size_t mma_ws_bytes(const kca::RowsPlan& p, int cluster) {
  const int max_clusters = (p.max_splits + cluster - 1) / cluster;
  if (max_clusters <= 1) return KCA_WORKSPACE_HEADER;
  const size_t slots = (size_t)p.n_units * max_clusters;
  return KCA_WORKSPACE_HEADER + align_up(slots * kHeads * 2 * 4) + align_up(slots * kHeads * kDim * 4);
}

// Workspace of the rows path: enough for either rows kernel, so that the
// query functions (which do not know the path a call will take) and the
// check at call time agree.  *mma_plan / *cluster: the tensor-core plan.
size_t rows_ws_bytes_any(int32_t n_units, const int64_t* nkeys, int sms, kca::RowsPlan* mma_plan,
                         int* cluster) {
  const size_t simt = rows_ws_bytes(kca::make_rows_plan(n_units, nkeys, sms));
  *mma_plan = mma_rows_plan(n_units, nkeys, sms, cluster);
  if (*cluster < 1) return simt;
  const size_t mma = mma_ws_bytes(*mma_plan, *cluster);
  return simt > mma ? simt : mma;
}
size_t rows_ws_bytes_any(int32_t n_units, const int64_t* nkeys, int sms) {
  kca::RowsPlan p;
  int c = 0;
  return rows_ws_bytes_any(n_units, nkeys, sms, &p, &c);
}

// Plan of the rows path for this cache dtype (cluster 0: no usable plan),
// with the workspace a call needs.
kca::RowsPlan rows_plan(int32_t kv_dtype, int32_t n_units, const int64_t* nkeys, int sms, int* cluster,
                        size_t* ws_bytes) {
  kca::RowsPlan mma;
  *ws_bytes = rows_ws_bytes_any(n_units, nkeys, sms, &mma, cluster);
  if (use_rows_mma(kv_dtype)) return mma;
  *cluster = 1;
  return kca::make_rows_plan(n_units, nkeys, sms);
}

// Launches the rows path: tensor cores for 16-bit caches (tensor maps over the
// cache_rows rows of the cache), CUDA cores otherwise.
int launch_rows_path(int32_t q_dtype, int32_t kv_dtype, const void* k_cache, const void* v_cache,
                     int64_t cache_rows, kca::RowsArgs a, int cluster, void* workspace, cudaStream_t s) {
  a.cache_rows = cache_rows;
  if (use_rows_mma(kv_dtype)) {
    a.cluster = cluster;
    a.max_clusters = (a.max_splits + cluster - 1) / cluster;
    a.part_slots = a.max_clusters > 1 ? (int64_t)a.n_units * a.max_clusters : 0;
    if (a.max_clusters > 1) {
      // Counters live in the header (no other path writes there), cluster
      // partials where the CUDA-core path keeps its split partials.
      a.tickets = reinterpret_cast<int32_t*>(static_cast<char*>(workspace) + kStatusBytes);
      carve(workspace, (size_t)a.n_units * a.max_clusters * kHeads * 2 * 4, &a.cpart_ml, &a.cpart_acc);
    }
    CUtensorMap tmk, tmv;
    if (!encode_kv_map(&tmk, k_cache, kv_dtype, 0, cache_rows, 64) ||
        !encode_kv_map(&tmv, v_cache, kv_dtype, 0, cache_rows, 64))
      return KCA_ERR_CUDA;
    return kca::launch_decode_mma(q_dtype, kv_dtype, tmk, tmv, a, s) == cudaSuccess ? KCA_OK : KCA_ERR_CUDA;
  }
  a.part_slots = a.max_splits > 1 ? (int64_t)a.n_units * a.max_splits : 0;
  carve(workspace, (size_t)a.n_units * a.max_splits * kHeads * 2 * 4, &a.part_ml, &a.part_acc);
  return kca::launch_rows(q_dtype, kv_dtype, a, s) == cudaSuccess ? KCA_OK : KCA_ERR_CUDA;
}

// Work items of the rows path (unit u at position pos[u], nk[u] visible keys
// from lo(pos[u])), as the calls run them: the CUDA-core kernel's plan for
// num_sms SMs, or -- for 16-bit caches, unless attn_force_path pins the
// CUDA-core kernel -- the tensor-core kernel's cluster plan on the current
// device (its clusters must fit the device's resident capacity, so that form
// needs a device).  slot: the split's partial slot (CUDA core), or the
// cluster partial its cluster writes (tensor cores), -1 when nothing of the
// unit goes through global memory.
int rows_plan_items(int32_t kv_dtype, int32_t n, const int64_t* pos, const int64_t* nk, int32_t window,
                    int32_t num_sms, const int32_t* capacity, int64_t* items, int32_t max_items, int32_t* count,
                    int32_t* cluster_out) {
  const bool mma = use_rows_mma(kv_dtype);
  kca::RowsPlan p;
  int cluster = 1;
  if (mma) {
    int sms = num_sms;
    if (capacity == nullptr && current_sms(&sms) != KCA_OK) return KCA_ERR_CUDA;
    p = mma_rows_plan(n, nk, sms, &cluster, capacity);
    if (cluster < 1) return capacity == nullptr ? KCA_ERR_CUDA : KCA_ERR_RANGE;
  } else {
    p = kca::make_rows_plan(n, nk, num_sms);
  }
  const int32_t max_clusters = (p.max_splits + cluster - 1) / cluster;
  for (int32_t u = 0; u < n; ++u) {
    const int64_t lo = kca::lo_of(pos[u], window);
    const int32_t ns = kca::rows_n_splits(nk[u], p.split_len);
    const int32_t nclus = (ns + cluster - 1) / cluster;
    for (int32_t sp = 0; sp < ns; ++sp, ++*count) {
      if (*count >= max_items) continue;
      int64_t kb = lo + (int64_t)sp * p.split_len, ke = kb + p.split_len;
      if (ke > pos[u] + 1) ke = pos[u] + 1;
      if (nk[u] == 0) kb = ke = lo;
      items[4 * *count + 0] = u;
      items[4 * *count + 1] = kb;
      items[4 * *count + 2] = ke;
      items[4 * *count + 3] = mma ? (nclus > 1 ? (int64_t)u * max_clusters + sp / cluster : -1)
                                  : (ns > 1 ? (int64_t)u * p.max_splits + sp : -1);
    }
  }
  if (cluster_out != nullptr) *cluster_out = cluster;
  return KCA_OK;
}

// Multi-row units (16-bit caches, 2-15 rows per sequence): units of ur
// rows of one sequence, the union of their keys cut into splits over the
// GPU; the tcgen05 kernel (units of 8 rows when a sequence has more than 4)
// or, pinned, the mma.sync one.  Serves attn_prefill_batch and attn_prefill's
// short chunks (one sequence at ctx_len = chunk_start + rows).
int32_t multirow_unit_rows(int32_t rows) {
  return use_batch_tc() && rows > kca::kMultiRows ? kca::kMultiRowsWide : kca::kMultiRows;
}
size_t multirow_route_ws_bytes(int32_t batch, int32_t rows, const int64_t* ctx_len, int32_t window, int sms) {
  const std::vector<int64_t> nku = multirow_unit_keys(batch, rows, ctx_len, window, multirow_unit_rows(rows));
  return multirow_ws_bytes(batch, rows,
                           kca::make_rows_plan((int32_t)nku.size(), nku.data(), sms, kca::kMultiRowMinSplit));
}
int launch_multirow_route(const void* q, int32_t q_dtype, const void* k_cache, const void* v_cache, int32_t kv_dtype,
                          int64_t capacity, int32_t batch, int32_t rows, const int64_t* ctx_len, int32_t window,
                          float scale, float* out, void* workspace, size_t workspace_bytes, int sms, cudaStream_t s) {
  const bool tc = use_batch_tc();
  const int32_t ur = multirow_unit_rows(rows);
  const std::vector<int64_t> nku = multirow_unit_keys(batch, rows, ctx_len, window, ur);
  const kca::RowsPlan mp = kca::make_rows_plan((int32_t)nku.size(), nku.data(), sms, kca::kMultiRowMinSplit);
  if (workspace_bytes < multirow_ws_bytes(batch, rows, mp)) return KCA_ERR_WORKSPACE;
  kca::RowsArgs a{};
  a.q = q;
  a.k = k_cache;
  a.v = v_cache;
  a.out = out;
  a.status = workspace;
  a.seq_rows = capacity;
  a.mode = 2;
  a.rows_per_seq = rows;
  a.unit_rows = ur;
  a.n_units = (int32_t)nku.size();
  a.split_len = mp.split_len;
  a.max_splits = mp.max_splits;
  a.window = window;
  a.scale = scale;
  for (int32_t b = 0; b < batch; ++b) a.ctx[b] = ctx_len[b];
  a.cache_rows = (int64_t)batch * capacity;
  a.part_slots = mp.max_splits > 1 ? (int64_t)batch * rows * mp.max_splits : 0;
  if (mp.max_splits > 1) {
    carve(workspace, (size_t)batch * rows * mp.max_splits * kHeads * 2 * 4, &a.part_ml, &a.part_acc);
    // self-resetting per-unit merge tickets of the tcgen05 kernel, which
    // then merges in-kernel; a unit with many splits is merged by a second
    // kernel instead (one CTA would read all its partials: at 1 x 131,072
    // keys, 147 splits, 141 us against 52 us with the merge kernel)
    if (mp.max_splits <= kca::kRowsTcMergeSplits)
      a.tickets = reinterpret_cast<int32_t*>(static_cast<char*>(workspace) + kStatusBytes);
  }
  CUtensorMap tmk, tmv;
  if (!encode_kv_map(&tmk, k_cache, kv_dtype, 0, (int64_t)batch * capacity, 64) ||
      !encode_kv_map(&tmv, v_cache, kv_dtype, 0, (int64_t)batch * capacity, 64))
    return KCA_ERR_CUDA;
  const cudaError_t e = tc ? kca::launch_rows_tc(q_dtype, kv_dtype, tmk, tmv, a, s)
                           : kca::launch_decode_multirow(q_dtype, kv_dtype, tmk, tmv, a, s);
  return e == cudaSuccess ? KCA_OK : KCA_ERR_CUDA;
}

}  // namespace

extern "C" {

int attn_decode_cluster_capacity(int32_t* capacity) {
  if (capacity == nullptr) return KCA_ERR_NULL;
  const int sizes[3] = {2, 4, 8};
  for (int i = 0; i < 3; ++i) {
    const int n = kca::decode_mma_cluster_capacity(sizes[i]);
    if (n <= 0) return KCA_ERR_CUDA;
    capacity[i] = n;
  }
  return KCA_OK;
}

int attn_force_path(int32_t op, int32_t path) {
  if (path < -1 || path > (op == 0 ? 2 : 1)) return KCA_ERR_RANGE;
  if (op == 0) g_prefill_path.store(path);
  else if (op == 1) g_rows_path.store(path);
  else if (op == 2) g_batch_path.store(path);
  else return KCA_ERR_RANGE;
  return KCA_OK;
}

const char* attn_status_string(int status) {
  switch (status) {
    case KCA_OK: return "ok";
    case KCA_ERR_NULL: return "a required pointer is NULL";
    case KCA_ERR_GEOMETRY: return "unsupported geometry (needs 8 query heads, 1 KV head, head_dim 256)";
    case KCA_ERR_DTYPE: return "unknown element type";
    case KCA_ERR_RANGE: return "row count, position, context length, capacity, batch or scale out of range";
    case KCA_ERR_WORKSPACE: return "workspace too small or not 256-byte aligned";
    case KCA_ERR_ALIGN: return "q, k, v or out not 16-byte aligned";
    case KCA_ERR_CUDA: return "a CUDA runtime call failed";
    case KCA_ERR_DEVICE: return "a kernel recorded a device-side error (bounded wait ran out)";
    default: return "unknown status";
  }
}

int attn_prefill_plan(int32_t q_dtype, int32_t kv_dtype, int64_t chunk_start, int32_t chunk_rows,
                      int32_t window, int32_t num_sms, const int32_t* cluster_capacity, int64_t* items,
                      int32_t max_items, int32_t* n_items, int32_t* path) {
  if (n_items == nullptr || path == nullptr || (items == nullptr && max_items > 0)) return KCA_ERR_NULL;
  if (!dtype_ok(q_dtype) || !dtype_ok(kv_dtype)) return KCA_ERR_DTYPE;
  if (chunk_rows < 1 || chunk_rows > KCA_MAX_CHUNK_ROWS || chunk_start < 0 ||
      chunk_start + chunk_rows > KCA_MAX_POSITION || num_sms < 1)
    return KCA_ERR_RANGE;
  if (cluster_capacity != nullptr && (cluster_capacity[0] < 0 || cluster_capacity[1] < 0 || cluster_capacity[2] < 0))
    return KCA_ERR_RANGE;
  int32_t count = 0;
  const int route = prefill_route(q_dtype, kv_dtype, chunk_start, chunk_rows, window);
  if (route == 2) {
    // multi-row units: one item per split of a unit of rows
    *path = 2;
    const int64_t ctx = chunk_start + chunk_rows;
    const int32_t ur = multirow_unit_rows(chunk_rows);
    const std::vector<int64_t> nku = multirow_unit_keys(1, chunk_rows, &ctx, window, ur);
    const kca::RowsPlan mp = kca::make_rows_plan((int32_t)nku.size(), nku.data(), num_sms, kca::kMultiRowMinSplit);
    for (int32_t u = 0; u < (int32_t)nku.size(); ++u) {
      const int64_t lo = kca::lo_of(chunk_start + (int64_t)u * ur, window);
      const int32_t ns = kca::rows_n_splits(nku[u], mp.split_len);
      for (int32_t sp = 0; sp < ns; ++sp, ++count) {
        if (count >= max_items) continue;
        int64_t kb = lo + (int64_t)sp * mp.split_len, ke = kb + mp.split_len;
        if (ke > lo + nku[u]) ke = lo + nku[u];
        items[4 * count + 0] = u;
        items[4 * count + 1] = kb;
        items[4 * count + 2] = ke;
        items[4 * count + 3] = ns > 1 ? sp : -1;
      }
    }
  } else if (route == 1) {
    *path = 1;
    const kca::TcPlan p = kca::make_tc_plan(chunk_start, chunk_rows, window, num_sms / 2);
    for (int32_t i = 0; i < p.n_items; ++i) {
      const kca::TcItem it = kca::tc_item(p, i);
      int64_t kb = p.kv_lo + (int64_t)it.kt_begin * kca::kKeyTile;
      int64_t ke = p.kv_lo + (int64_t)it.kt_end * kca::kKeyTile;
      if (ke > p.ctx_len) ke = p.ctx_len;
      for (int32_t r = 0; r < kca::tc_pair_tiles(p, it.pair); ++r, ++count) {   // one entry per tile of the pair
        if (count >= max_items) continue;
        items[4 * count + 0] = 2 * it.pair + r;
        items[4 * count + 1] = kb;
        items[4 * count + 2] = ke;
        items[4 * count + 3] = r == 0 ? it.slot0 : it.slot1;
      }
    }
  } else {
    *path = 0;
    const std::vector<int64_t> nk = prefill_unit_keys(chunk_start, chunk_rows, window);
    std::vector<int64_t> pos(chunk_rows);
    for (int32_t u = 0; u < chunk_rows; ++u) pos[u] = chunk_start + u;
    const int st = rows_plan_items(kv_dtype, chunk_rows, pos.data(), nk.data(), window, num_sms,
                                   cluster_capacity, items, max_items, &count, nullptr);
    if (st != KCA_OK) return st;
  }
  *n_items = count;
  return count <= max_items ? KCA_OK : KCA_ERR_RANGE;
}

int attn_decode_plan(int32_t batch, const int64_t* ctx_len, int32_t window, int32_t kv_dtype, int32_t num_sms,
                     const int32_t* cluster_capacity, int64_t* items, int32_t max_items, int32_t* n_items,
                     int32_t* cluster) {
  if (ctx_len == nullptr || n_items == nullptr || (items == nullptr && max_items > 0)) return KCA_ERR_NULL;
  if (!dtype_ok(kv_dtype)) return KCA_ERR_DTYPE;
  if (batch < 1 || batch > KCA_MAX_BATCH || num_sms < 1) return KCA_ERR_RANGE;
  if (cluster_capacity != nullptr && (cluster_capacity[0] < 0 || cluster_capacity[1] < 0 || cluster_capacity[2] < 0))
    return KCA_ERR_RANGE;
  for (int32_t b = 0; b < batch; ++b)
    if (ctx_len[b] < 0 || ctx_len[b] > KCA_MAX_POSITION) return KCA_ERR_RANGE;
  const std::vector<int64_t> nk = decode_unit_keys(batch, ctx_len, window);
  std::vector<int64_t> pos(batch);
  for (int32_t b = 0; b < batch; ++b) pos[b] = ctx_len[b] - 1;
  int32_t count = 0;
  const int st = rows_plan_items(kv_dtype, batch, pos.data(), nk.data(), window, num_sms, cluster_capacity, items,
                                 max_items, &count, cluster);
  if (st != KCA_OK) return st;
  *n_items = count;
  return count <= max_items ? KCA_OK : KCA_ERR_RANGE;
}

size_t attn_prefill_workspace_bytes(int32_t q_dtype, int32_t kv_dtype, int64_t chunk_start,
                                    int32_t chunk_rows, int32_t window) {
  if (!dtype_ok(q_dtype) || !dtype_ok(kv_dtype)) return 0;
  if (prefill_args_status(KCA_MAX_POSITION, chunk_start, chunk_rows) != KCA_OK) return 0;
  int sms = 0;
  if (current_sms(&sms) != KCA_OK) return 0;
  const int route = prefill_route(q_dtype, kv_dtype, chunk_start, chunk_rows, window);
  if (route == 1) return tc_ws_bytes(kca::make_tc_plan(chunk_start, chunk_rows, window, sms / 2));
  if (route == 2) {
    const int64_t ctx = chunk_start + chunk_rows;
    return multirow_route_ws_bytes(1, chunk_rows, &ctx, window, sms);
  }
  const std::vector<int64_t> nk = prefill_unit_keys(chunk_start, chunk_rows, window);
  return rows_ws_bytes_any(chunk_rows, nk.data(), sms);
}

size_t attn_decode_partial_workspace_bytes(int32_t batch, const int64_t* ctx_len, int64_t key_begin,
                                           int64_t capacity, int32_t window) {
  if (ctx_len == nullptr || shard_args_status(capacity, batch, ctx_len, key_begin) != KCA_OK) return 0;
  int sms = 0;
  if (current_sms(&sms) != KCA_OK) return 0;
  const std::vector<int64_t> nk = shard_unit_keys(batch, ctx_len, window, key_begin, key_begin + capacity);
  return rows_ws_bytes_any(batch, nk.data(), sms);
}

size_t attn_prefill_batch_workspace_bytes(int32_t batch, int32_t rows, const int64_t* ctx_len, int32_t window) {
  if (ctx_len == nullptr || batch_args_status(KCA_MAX_POSITION, batch, rows, ctx_len) != KCA_OK) return 0;
  int sms = 0;
  if (current_sms(&sms) != KCA_OK) return 0;
  const std::vector<int64_t> nk = batch_unit_keys(batch, rows, ctx_len, window);
  size_t need = rows_ws_bytes_any(batch * rows, nk.data(), sms);
  if (rows > 1) {   // the multi-row kernels' partials, whichever path and unit size a call takes
    for (const int32_t ur : {kca::kMultiRows, kca::kMultiRowsWide}) {
      const std::vector<int64_t> nku = multirow_unit_keys(batch, rows, ctx_len, window, ur);
      const size_t mr = multirow_ws_bytes(
          batch, rows, kca::make_rows_plan((int32_t)nku.size(), nku.data(), sms, kca::kMultiRowMinSplit));
      if (mr > need) need = mr;
    }
  }
  return need;
}

size_t attn_decode_workspace_bytes(int32_t batch, const int64_t* ctx_len, int32_t window) {
  if (ctx_len == nullptr || decode_args_status(KCA_MAX_POSITION, batch, ctx_len) != KCA_OK) return 0;
  int sms = 0;
  if (current_sms(&sms) != KCA_OK) return 0;
  const std::vector<int64_t> nk = decode_unit_keys(batch, ctx_len, window);
  return rows_ws_bytes_any(batch, nk.data(), sms);
}

int attn_workspace_init(void* workspace, size_t workspace_bytes, void* stream) {
  if (workspace == nullptr) return KCA_ERR_NULL;
  if (workspace_bytes < KCA_WORKSPACE_HEADER || (reinterpret_cast<uintptr_t>(workspace) % kAlign) != 0)
    return KCA_ERR_WORKSPACE;
  return cudaMemsetAsync(workspace, 0, KCA_WORKSPACE_HEADER, static_cast<cudaStream_t>(stream)) ==
                 cudaSuccess
             ? KCA_OK
             : KCA_ERR_CUDA;
}

int attn_device_status(void* workspace, void* stream, uint32_t* detail) {
  if (workspace == nullptr) return KCA_ERR_NULL;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint32_t word[2] = {0, 0};
  if (cudaMemcpyAsync(word, workspace, sizeof word, cudaMemcpyDeviceToHost, s) != cudaSuccess ||
      cudaStreamSynchronize(s) != cudaSuccess)
    return KCA_ERR_CUDA;
  if (word[0] == 0) return KCA_OK;
  if (detail != nullptr) *detail = word[1];
  if (cudaMemsetAsync(workspace, 0, sizeof word, s) != cudaSuccess || cudaStreamSynchronize(s) != cudaSuccess)
    return KCA_ERR_CUDA;
  return KCA_ERR_DEVICE;
}

int attn_prefill(const void* q_chunk, int32_t q_dtype, const void* k_cache, const void* v_cache,
                 int32_t kv_dtype, int32_t n_q_heads, int32_t n_kv_heads, int32_t head_dim,
                 int64_t capacity, int64_t chunk_start, int32_t chunk_rows, int64_t ctx_len,
                 int32_t window, float scale, float* out, void* workspace, size_t workspace_bytes,
                 void* stream) {
  if (!q_chunk || !k_cache || !v_cache || !out || !workspace) return KCA_ERR_NULL;
  int st = geometry_status(n_q_heads, n_kv_heads, head_dim);
  if (st != KCA_OK) return st;
  if (!dtype_ok(q_dtype) || !dtype_ok(kv_dtype)) return KCA_ERR_DTYPE;
  st = prefill_args_status(capacity, chunk_start, chunk_rows);
  if (st != KCA_OK) return st;
  if (ctx_len != chunk_start + chunk_rows || !std::isfinite(scale) || !(scale > 0.f))
    return KCA_ERR_RANGE;
  if (!aligned16(q_chunk) || !aligned16(k_cache) || !aligned16(v_cache) || !aligned16(out))
    return KCA_ERR_ALIGN;
  if ((reinterpret_cast<uintptr_t>(workspace) % kAlign) != 0) return KCA_ERR_WORKSPACE;
  int sms = 0;
  if (current_sms(&sms) != KCA_OK) return KCA_ERR_CUDA;
  cudaStream_t s = static_cast<cudaStream_t>(stream);

  if (use_tc(q_dtype, kv_dtype, chunk_start, chunk_rows, window)) {
    kca::TcArgs a{};
    a.plan = kca::make_tc_plan(chunk_start, chunk_rows, window, sms / 2);
    if (workspace_bytes < tc_ws_bytes(a.plan)) return KCA_ERR_WORKSPACE;
    a.q = q_chunk;
    a.out = out;
    a.status = workspace;
    a.scale_log2 = scale * 1.4426950408889634f;
    carve(workspace, (size_t)a.plan.n_slots * 128 * 2 * 4, &a.part_ml, &a.part_acc);
    if (!kca::fill_tc_tables(a)) return KCA_ERR_RANGE;
    CUtensorMap tmk, tmv, tmq, tmo, tmpart, tmpart_rag;
    // K and V: 64 x 64 boxes (each CTA of a pair loads its half of a tile);
    // Q in 64-dim boxes of a 128-row tile; out / partials in 32-column boxes.
    if (!encode_kv_map(&tmk, k_cache, kv_dtype, a.plan.kv_lo, a.plan.ctx_len, 64) ||
        !encode_kv_map(&tmv, v_cache, kv_dtype, a.plan.kv_lo, a.plan.ctx_len, 64) ||
        !encode_rows_map(&tmq, q_chunk, q_dtype, (int64_t)chunk_rows * kHeads, 64) ||
        !encode_rows_map(&tmo, out, KCA_F32, (int64_t)chunk_rows * kHeads, 32))
      return KCA_ERR_CUDA;
    if (a.plan.n_slots > 0) {
      if (!encode_rows_map(&tmpart, a.part_acc, KCA_F32, (int64_t)a.plan.n_slots * 128, 32)) return KCA_ERR_CUDA;
    } else {
      tmpart = tmo;   // no split tile: never used
    }
    // A ragged last tile (chunk_rows not a multiple of 16) stores only its
    // 8 (chunk_rows mod 16) valid M rows of each partial.
    const int32_t rag = chunk_rows % kca::kRowTile;
    a.rag_tile = a.plan.n_slots > 0 && rag != 0 ? a.plan.n_tiles - 1 : -1;
    if (a.rag_tile >= 0) {
      if (!encode_rows_map(&tmpart_rag, a.part_acc, KCA_F32, (int64_t)a.plan.n_slots * 128, 32,
                           (uint32_t)(rag * kHeads)))
        return KCA_ERR_CUDA;
    } else {
      tmpart_rag = tmpart;
    }
    return kca::launch_prefill_tc(kv_dtype, tmk, tmv, tmq, tmo, tmpart, tmpart_rag, a, s) == cudaSuccess
               ? KCA_OK
               : KCA_ERR_CUDA;
  }

  if (prefill_route(q_dtype, kv_dtype, chunk_start, chunk_rows, window) == 2) {
    // one sequence of chunk_rows rows ending at ctx_len, in multi-row units
    return launch_multirow_route(q_chunk, q_dtype, k_cache, v_cache, kv_dtype, capacity, 1, chunk_rows, &ctx_len,
                                 window, scale, out, workspace, workspace_bytes, sms, s);
  }
  const std::vector<int64_t> nk = prefill_unit_keys(chunk_start, chunk_rows, window);
  int cluster = 1;
  size_t need = 0;
  const kca::RowsPlan p = rows_plan(kv_dtype, chunk_rows, nk.data(), sms, &cluster, &need);
  if (cluster < 1) return KCA_ERR_CUDA;
  if (workspace_bytes < need) return KCA_ERR_WORKSPACE;
  kca::RowsArgs a{};
  a.q = q_chunk;
  a.k = k_cache;
  a.v = v_cache;
  a.out = out;
  a.status = workspace;
  a.seq_rows = 0;
  a.chunk_start = chunk_start;
  a.mode = 1;
  a.n_units = chunk_rows;
  a.split_len = p.split_len;
  a.max_splits = p.max_splits;
  a.window = window;
  a.scale = scale;
  return launch_rows_path(q_dtype, kv_dtype, k_cache, v_cache, capacity, a, cluster, workspace, s);
}

int attn_decode(const void* q, int32_t q_dtype, const void* k_cache, const void* v_cache,
                int32_t kv_dtype, int32_t n_q_heads, int32_t n_kv_heads, int32_t head_dim,
                int64_t capacity, int32_t batch, const int64_t* ctx_len, int32_t window, float scale,
                float* out, void* workspace, size_t workspace_bytes, void* stream) {
  return kca::decode_entry(q, q_dtype, k_cache, v_cache, kv_dtype, n_q_heads, n_kv_heads, head_dim, capacity,
                           batch, ctx_len, window, scale, out, workspace, workspace_bytes, stream, false);
}

}  // extern "C"

namespace kca {

int decode_args_check(const void* q, int32_t q_dtype, const void* k_cache, const void* v_cache, int32_t kv_dtype,
                      int32_t n_q_heads, int32_t n_kv_heads, int32_t head_dim, int64_t capacity, int32_t batch,
                      const int64_t* ctx_len, float scale, const float* out) {
  if (!q || !k_cache || !v_cache || !out || !ctx_len) return KCA_ERR_NULL;
  int st = geometry_status(n_q_heads, n_kv_heads, head_dim);
  if (st != KCA_OK) return st;
  if (!dtype_ok(q_dtype) || !dtype_ok(kv_dtype)) return KCA_ERR_DTYPE;
  st = decode_args_status(capacity, batch, ctx_len);
  if (st != KCA_OK) return st;
  if (!std::isfinite(scale) || !(scale > 0.f)) return KCA_ERR_RANGE;
  if (!aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache) || !aligned16(out))
    return KCA_ERR_ALIGN;
  return KCA_OK;
}

int decode_entry(const void* q, int32_t q_dtype, const void* k_cache, const void* v_cache, int32_t kv_dtype,
                 int32_t n_q_heads, int32_t n_kv_heads, int32_t head_dim, int64_t capacity, int32_t batch,
                 const int64_t* ctx_len, int32_t window, float scale, float* out, void* workspace,
                 size_t workspace_bytes, void* stream, bool clear_header) {
  if (!workspace) return KCA_ERR_NULL;
  int st = decode_args_check(q, q_dtype, k_cache, v_cache, kv_dtype, n_q_heads, n_kv_heads, head_dim, capacity,
                             batch, ctx_len, scale, out);
  if (st != KCA_OK) return st;
  if ((reinterpret_cast<uintptr_t>(workspace) % kAlign) != 0) return KCA_ERR_WORKSPACE;
  int sms = 0;
  if (current_sms(&sms) != KCA_OK) return KCA_ERR_CUDA;
  const std::vector<int64_t> nk = decode_unit_keys(batch, ctx_len, window);
  int cluster = 1;
  size_t need = 0;
  const kca::RowsPlan p = rows_plan(kv_dtype, batch, nk.data(), sms, &cluster, &need);
  if (cluster < 1) return KCA_ERR_CUDA;
  if (workspace_bytes < need) return KCA_ERR_WORKSPACE;
  kca::RowsArgs a{};
  a.q = q;
  a.k = k_cache;
  a.v = v_cache;
  a.out = out;
  a.status = workspace;
  a.seq_rows = capacity;
  a.chunk_start = 0;
  a.mode = 0;
  a.n_units = batch;
  a.split_len = p.split_len;
  a.max_splits = p.max_splits;
  a.window = window;
  a.scale = scale;
  for (int32_t b = 0; b < batch; ++b) a.ctx[b] = ctx_len[b];
  // Every argument is valid: only now may the header be cleared.
  if (clear_header &&
      cudaMemsetAsync(workspace, 0, KCA_WORKSPACE_HEADER, static_cast<cudaStream_t>(stream)) != cudaSuccess)
    return KCA_ERR_CUDA;
  return launch_rows_path(q_dtype, kv_dtype, k_cache, v_cache, (int64_t)batch * capacity, a, cluster,
                          workspace, static_cast<cudaStream_t>(stream));
}

}  // namespace kca

extern "C" {

int attn_decode_dev(const void* q, int32_t q_dtype, const void* k_cache, const void* v_cache,
                    int32_t kv_dtype, int32_t n_q_heads, int32_t n_kv_heads, int32_t head_dim,
                    int64_t capacity, int32_t batch, const int64_t* ctx_len_dev, int64_t ctx_bound,
                    int32_t window, float scale, float* out, void* workspace, size_t workspace_bytes,
                    void* stream) {
  if (!q || !k_cache || !v_cache || !out || !workspace || !ctx_len_dev) return KCA_ERR_NULL;
  int st = geometry_status(n_q_heads, n_kv_heads, head_dim);
  if (st != KCA_OK) return st;
  if (!dtype_ok(q_dtype) || !dtype_ok(kv_dtype)) return KCA_ERR_DTYPE;
  if (batch < 1 || batch > KCA_MAX_BATCH) return KCA_ERR_RANGE;
  // The plan is the host-array plan of `batch` sequences at the bound.
  const std::vector<int64_t> bound(batch, ctx_bound);
  st = decode_args_status(capacity, batch, bound.data());
  if (st != KCA_OK) return st;
  if (!std::isfinite(scale) || !(scale > 0.f)) return KCA_ERR_RANGE;
  if (!aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache) || !aligned16(out) ||
      (reinterpret_cast<uintptr_t>(ctx_len_dev) % 8) != 0)
    return KCA_ERR_ALIGN;
  if ((reinterpret_cast<uintptr_t>(workspace) % kAlign) != 0) return KCA_ERR_WORKSPACE;
  int sms = 0;
  if (current_sms(&sms) != KCA_OK) return KCA_ERR_CUDA;
  const std::vector<int64_t> nk = decode_unit_keys(batch, bound.data(), window);
  int cluster = 1;
  size_t need = 0;
  const kca::RowsPlan p = rows_plan(kv_dtype, batch, nk.data(), sms, &cluster, &need);
  if (cluster < 1) return KCA_ERR_CUDA;
  if (workspace_bytes < need) return KCA_ERR_WORKSPACE;
  kca::RowsArgs a{};
  a.q = q;
  a.k = k_cache;
  a.v = v_cache;
  a.out = out;
  a.status = workspace;
  a.seq_rows = capacity;
  a.chunk_start = 0;
  a.mode = 0;
  a.n_units = batch;
  a.split_len = p.split_len;
  a.max_splits = p.max_splits;
  a.window = window;
  a.scale = scale;
  a.ctx_dev = ctx_len_dev;
  a.ctx_bound = ctx_bound;
  return launch_rows_path(q_dtype, kv_dtype, k_cache, v_cache, (int64_t)batch * capacity, a, cluster,
                          workspace, static_cast<cudaStream_t>(stream));
}

int attn_decode_partial(const void* q, int32_t q_dtype, const void* k_cache, const void* v_cache,
                        int32_t kv_dtype, int32_t n_q_heads, int32_t n_kv_heads, int32_t head_dim,
                        int64_t capacity, int32_t batch, const int64_t* ctx_len, int64_t key_begin,
                        int32_t window, float scale, float* part, void* workspace, size_t workspace_bytes,
                        void* stream) {
  if (!q || !k_cache || !v_cache || !part || !workspace || !ctx_len) return KCA_ERR_NULL;
  int st = geometry_status(n_q_heads, n_kv_heads, head_dim);
  if (st != KCA_OK) return st;
  if (!dtype_ok(q_dtype) || !dtype_ok(kv_dtype)) return KCA_ERR_DTYPE;
  st = shard_args_status(capacity, batch, ctx_len, key_begin);
  if (st != KCA_OK) return st;
  if (!std::isfinite(scale) || !(scale > 0.f)) return KCA_ERR_RANGE;
  if (!aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache) || !aligned16(part)) return KCA_ERR_ALIGN;
  if ((reinterpret_cast<uintptr_t>(workspace) % kAlign) != 0) return KCA_ERR_WORKSPACE;
  int sms = 0;
  if (current_sms(&sms) != KCA_OK) return KCA_ERR_CUDA;
  const int64_t key_end = key_begin + capacity;
  const std::vector<int64_t> nk = shard_unit_keys(batch, ctx_len, window, key_begin, key_end);
  int cluster = 1;
  size_t need = 0;
  const kca::RowsPlan p = rows_plan(kv_dtype, batch, nk.data(), sms, &cluster, &need);
  if (cluster < 1) return KCA_ERR_CUDA;
  if (workspace_bytes < need) return KCA_ERR_WORKSPACE;
  kca::RowsArgs a{};
  a.q = q;
  a.k = k_cache;
  a.v = v_cache;
  a.out = part + (size_t)batch * kHeads * 2;   // acc follows the (m, l) pairs
  a.out_ml = part;
  a.status = workspace;
  a.seq_rows = capacity;
  a.mode = 0;
  a.n_units = batch;
  a.split_len = p.split_len;
  a.max_splits = p.max_splits;
  a.window = window;
  a.scale = scale;
  a.key_begin = key_begin;
  a.key_end = key_end;
  for (int32_t b = 0; b < batch; ++b) a.ctx[b] = ctx_len[b];
  return launch_rows_path(q_dtype, kv_dtype, k_cache, v_cache, (int64_t)batch * capacity, a, cluster,
                          workspace, static_cast<cudaStream_t>(stream));
}

int attn_prefill_batch(const void* q, int32_t q_dtype, const void* k_cache, const void* v_cache,
                       int32_t kv_dtype, int32_t n_q_heads, int32_t n_kv_heads, int32_t head_dim,
                       int64_t capacity, int32_t batch, int32_t rows, const int64_t* ctx_len, int32_t window,
                       float scale, float* out, void* workspace, size_t workspace_bytes, void* stream) {
  if (!q || !k_cache || !v_cache || !out || !workspace || !ctx_len) return KCA_ERR_NULL;
  int st = geometry_status(n_q_heads, n_kv_heads, head_dim);
  if (st != KCA_OK) return st;
  if (!dtype_ok(q_dtype) || !dtype_ok(kv_dtype)) return KCA_ERR_DTYPE;
  st = batch_args_status(capacity, batch, rows, ctx_len);
  if (st != KCA_OK) return st;
  if (!std::isfinite(scale) || !(scale > 0.f)) return KCA_ERR_RANGE;
  if (!aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache) || !aligned16(out)) return KCA_ERR_ALIGN;
  if ((reinterpret_cast<uintptr_t>(workspace) % kAlign) != 0) return KCA_ERR_WORKSPACE;
  int sms = 0;
  if (current_sms(&sms) != KCA_OK) return KCA_ERR_CUDA;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (use_multirow(kv_dtype, rows))
    return launch_multirow_route(q, q_dtype, k_cache, v_cache, kv_dtype, capacity, batch, rows, ctx_len, window,
                                 scale, out, workspace, workspace_bytes, sms, s);
  const int32_t n_units = batch * rows;
  const std::vector<int64_t> nk = batch_unit_keys(batch, rows, ctx_len, window);
  int cluster = 1;
  size_t need = 0;
  const kca::RowsPlan p = rows_plan(kv_dtype, n_units, nk.data(), sms, &cluster, &need);
  if (cluster < 1) return KCA_ERR_CUDA;
  if (workspace_bytes < need) return KCA_ERR_WORKSPACE;
  kca::RowsArgs a{};
  a.q = q;
  a.k = k_cache;
  a.v = v_cache;
  a.out = out;
  a.status = workspace;
  a.seq_rows = capacity;
  a.mode = 2;
  a.rows_per_seq = rows;
  a.n_units = n_units;
  a.split_len = p.split_len;
  a.max_splits = p.max_splits;
  a.window = window;
  a.scale = scale;
  for (int32_t b = 0; b < batch; ++b) a.ctx[b] = ctx_len[b];
  return launch_rows_path(q_dtype, kv_dtype, k_cache, v_cache, (int64_t)batch * capacity, a, cluster, workspace, s);
}

size_t attn_decode_q8_workspace_bytes(int32_t batch, const int64_t* ctx_len, int32_t window) {
  // the same plans as attn_decode: the CUDA-core kernel's for f32 V, the
  // tensor-core kernel's for 16-bit V, and the larger of the two
  return attn_decode_workspace_bytes(batch, ctx_len, window);
}

int attn_decode_q8(const void* q, int32_t q_dtype, const void* k8_cache, const void* v_cache, int32_t v_dtype,
                   int32_t n_q_heads, int32_t n_kv_heads, int32_t head_dim, int64_t capacity, int32_t batch,
                   const int64_t* ctx_len, int32_t window, float scale, float* out, void* workspace,
                   size_t workspace_bytes, void* stream) {
  if (!workspace) return KCA_ERR_NULL;
  int st = kca::decode_args_check(q, q_dtype, k8_cache, v_cache, v_dtype, n_q_heads, n_kv_heads, head_dim, capacity,
                                  batch, ctx_len, scale, out);
  if (st != KCA_OK) return st;
  if ((reinterpret_cast<uintptr_t>(workspace) % kAlign) != 0) return KCA_ERR_WORKSPACE;
  int sms = 0;
  if (current_sms(&sms) != KCA_OK) return KCA_ERR_CUDA;
  const std::vector<int64_t> nk = decode_unit_keys(batch, ctx_len, window);
  int cluster = 1;
  size_t need = 0;
  const kca::RowsPlan p = rows_plan(v_dtype, batch, nk.data(), sms, &cluster, &need);
  if (cluster < 1) return KCA_ERR_CUDA;
  if (workspace_bytes < need) return KCA_ERR_WORKSPACE;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  kca::RowsArgs a{};
  a.q = q;
  a.k = k8_cache;
  a.v = v_cache;
  a.out = out;
  a.status = workspace;
  a.seq_rows = capacity;
  a.mode = 0;
  a.n_units = batch;
  a.split_len = p.split_len;
  a.max_splits = p.max_splits;
  a.window = window;
  a.scale = scale;
  for (int32_t b = 0; b < batch; ++b) a.ctx[b] = ctx_len[b];
  int sane = 0;
  st = kca::dot_canary(s, &sane);
  if (st != KCA_OK) return st;
  a.cache_rows = (int64_t)batch * capacity;
  if (use_rows_mma(v_dtype) && (sane & 4)) {
    // 16-bit V: the tensor-core kernel, QK on int8 MMAs (exact integers)
    a.cluster = cluster;
    a.max_clusters = (a.max_splits + cluster - 1) / cluster;
    a.part_slots = a.max_clusters > 1 ? (int64_t)a.n_units * a.max_clusters : 0;
    if (a.max_clusters > 1) {
      a.tickets = reinterpret_cast<int32_t*>(static_cast<char*>(workspace) + kStatusBytes);
      carve(workspace, (size_t)a.n_units * a.max_clusters * kHeads * 2 * 4, &a.cpart_ml, &a.cpart_acc);
    }
    const int64_t rows = (int64_t)batch * capacity;
    const cuuint64_t kdims[2] = {(cuuint64_t)KCA_I8_ROW_BYTES, (cuuint64_t)rows};
    const cuuint32_t kbox[2] = {128, 64}, sbox[2] = {16, 64};
    CUtensorMap tmk, tms, tmv;
    if (!encode_2d(&tmk, CU_TENSOR_MAP_DATA_TYPE_UINT8, k8_cache, kdims, KCA_I8_ROW_BYTES, kbox) ||
        !encode_2d(&tms, CU_TENSOR_MAP_DATA_TYPE_UINT8, k8_cache, kdims, KCA_I8_ROW_BYTES, sbox,
                   CU_TENSOR_MAP_SWIZZLE_NONE) ||
        !encode_kv_map(&tmv, v_cache, v_dtype, 0, rows, 64))
      return KCA_ERR_CUDA;
    return kca::launch_decode_mma_q8(q_dtype, v_dtype, tmk, tms, tmv, a, s) == cudaSuccess ? KCA_OK : KCA_ERR_CUDA;
  }
  // f32 V, the CUDA-core kernel pinned, or an int8 MMA the canary found
  // wrong: dp4a on the CUDA cores, or its emulation where the instruction
  // is the one found wrong.  This kernel's plan is the CUDA-core one.
  const kca::RowsPlan pc = kca::make_rows_plan(batch, nk.data(), sms);
  a.split_len = pc.split_len;
  a.max_splits = pc.max_splits;
  a.part_slots = a.max_splits > 1 ? (int64_t)a.n_units * a.max_splits : 0;
  carve(workspace, (size_t)a.n_units * a.max_splits * kHeads * 2 * 4, &a.part_ml, &a.part_acc);
  return kca::launch_rows_q8(q_dtype, v_dtype, (sane & 1) != 0, a, s) == cudaSuccess ? KCA_OK : KCA_ERR_CUDA;
}

int attn_merge_partials(int32_t n_parts, int32_t batch, const float* parts, int64_t part_stride, float* out,
                        void* stream) {
  if (!parts || !out) return KCA_ERR_NULL;
  if (n_parts < 1 || batch < 1 || batch > KCA_MAX_BATCH) return KCA_ERR_RANGE;
  if (part_stride < (int64_t)KCA_PARTIAL_FLOATS(batch) || part_stride % 4 != 0) return KCA_ERR_RANGE;
  if (!aligned16(parts) || !aligned16(out)) return KCA_ERR_ALIGN;
  return kca::launch_merge_partials(n_parts, batch, parts, part_stride, out, static_cast<cudaStream_t>(stream)) ==
                 cudaSuccess
             ? KCA_OK
             : KCA_ERR_CUDA;
}

}  // extern "C"

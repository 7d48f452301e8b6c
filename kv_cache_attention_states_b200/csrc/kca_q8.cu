// kca_q8.cu -- the quantised-dot attention: K rows stored as int8 codes with
// a per-row scale, the query quantised the same way per head inside the
// decode kernel, QK taken exactly on the codes (four int8 pairs per dp4a),
// softmax and the V sum in f32 (the CUDA-core rows kernel, kca_rows.cu).
//
// Prior art on the pages (Karume v0.8.0 release notes, "Fixes"): attention's
// dot product runs on packed int8 pairs with a dp4a-style instruction where
// the device has one; a device-level canary runs the instruction and its
// emulation against a known answer at first use, falls back to the
// emulation when only that is right, and fails loudly when neither is; the
// per-token activation scale is amax * f32(1/127).
//
// Quantisation of a row x of 256 values (here and in the decode kernel):
//   sx = amax(|x|) * f32(1/127)      (NaN if x holds a NaN)
//   code = clamp(round_half_even(x / sx), -127, 127) in f32 when sx is
//          finite and > 0, else 0.
// A packed K row is 272 bytes: the 256 codes, sx as f32 at byte 256, 12 zero
// bytes (rows stay 16-byte aligned for the bulk copies).
#include <atomic>
#include <cuda_runtime.h>

#include <cmath>
#include <mutex>
#include <vector>

#include "../../include/kca.h"
#include "kca_common.cuh"
#include "kca_plan.h"
#include "kca_rows.h"

namespace kca {
namespace {

__device__ __forceinline__ uint32_t code_of(float x, float sx) {
  if (!(sx > 0.f) || !(sx <= 3.402823466e38f)) return 0u;
  int c = __float2int_rn(__fdiv_rn(x, sx));
  c = c > 127 ? 127 : (c < -127 ? -127 : c);
  return static_cast<uint32_t>(c) & 0xffu;
}

// One warp per row: lane l quantises elements 8l .. 8l+7.
template <int DT>
__global__ void __launch_bounds__(256) quantize_rows_kernel(const void* x, int64_t n_rows, unsigned char* out) {
  const int64_t row = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= n_rows) return;
  float v[8];
  load8<DT>(static_cast<const char*>(x) + (row * kDim + 8 * lane) * ElemBytes<DT>::value, v);
  float am = fabsf(v[0]);
#pragma unroll
  for (int i = 1; i < 8; ++i) am = max_nan(am, fabsf(v[i]));
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) am = max_nan(am, __shfl_xor_sync(0xffffffffu, am, o));
  const float sx = am * (1.0f / 127.0f);
  uint32_t w[2];
#pragma unroll
  for (int j = 0; j < 2; ++j)
    w[j] = code_of(v[4 * j], sx) | (code_of(v[4 * j + 1], sx) << 8) | (code_of(v[4 * j + 2], sx) << 16) |
           (code_of(v[4 * j + 3], sx) << 24);
  unsigned char* dst = out + row * KCA_I8_ROW_BYTES;
  *reinterpret_cast<uint2*>(dst + 8 * lane) = make_uint2(w[0], w[1]);
  if (lane == 0) *reinterpret_cast<uint4*>(dst + kDim) = make_uint4(__float_as_uint(sx), 0u, 0u, 0u);
}

// ------------------------------------------------------------------ canary
// Known answer: kCanary (a, b, c) triples spanning the int8 extremes; each
// variant writes its results to its half of the array.
constexpr int kCanary = 64;
__device__ int kca_canary_out[2 * kCanary];

__host__ __device__ inline void canary_case(int i, uint32_t* a, uint32_t* b, int* c) {
  const int8_t vals[8] = {-128, -127, -1, 0, 1, 63, 126, 127};
  uint32_t x = 0, y = 0;
  for (int j = 0; j < 4; ++j) {
    x |= static_cast<uint32_t>(static_cast<uint8_t>(vals[(i + 3 * j) & 7])) << (8 * j);
    y |= static_cast<uint32_t>(static_cast<uint8_t>(vals[(5 * i + j) & 7])) << (8 * j);
  }
  *a = x;
  *b = y;
  *c = (i * 977) % 20011 - 10005;
}

__global__ void canary_kernel() {
  const int i = threadIdx.x;
  if (i >= kCanary) return;
  uint32_t a, b;
  int c;
  canary_case(i, &a, &b, &c);
  kca_canary_out[i] = __dp4a(static_cast<int>(a), static_cast<int>(b), c);
  int e = c;
#pragma unroll
  for (int j = 0; j < 4; ++j)
    e += static_cast<int>(static_cast<int8_t>(a >> (8 * j))) * static_cast<int>(static_cast<int8_t>(b >> (8 * j)));
  kca_canary_out[kCanary + i] = e;
}

// Per device: 0 not run, 1 dp4a, 2 emulation, 3 neither sane.
std::atomic<int> g_canary[64];
std::mutex g_canary_mu;

int run_canary(cudaStream_t s, int* variant) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return KCA_ERR_CUDA;
  int v = g_canary[dev].load();
  if (v == 0) {
    std::lock_guard<std::mutex> lock(g_canary_mu);
    v = g_canary[dev].load();
    if (v == 0) {
      canary_kernel<<<1, kCanary, 0, s>>>();
      int got[2 * kCanary];
      if (cudaGetLastError() != cudaSuccess ||
          cudaMemcpyFromSymbolAsync(got, kca_canary_out, sizeof got, 0, cudaMemcpyDeviceToHost, s) != cudaSuccess ||
          cudaStreamSynchronize(s) != cudaSuccess)
        return KCA_ERR_CUDA;
      bool hw = true, emu = true;
      for (int i = 0; i < kCanary; ++i) {
        uint32_t a, b;
        int c;
        canary_case(i, &a, &b, &c);
        int want = c;
        for (int j = 0; j < 4; ++j)
          want += static_cast<int>(static_cast<int8_t>(a >> (8 * j))) * static_cast<int>(static_cast<int8_t>(b >> (8 * j)));
        hw = hw && got[i] == want;
        emu = emu && got[kCanary + i] == want;
      }
      v = hw ? 1 : (emu ? 2 : 3);
      g_canary[dev].store(v);
    }
  }
  if (v == 3) return KCA_ERR_DEVICE;
  *variant = v == 1 ? 1 : 0;
  return KCA_OK;
}

bool dtype3(int32_t d) { return d == KCA_F32 || d == KCA_F16 || d == KCA_BF16; }
bool al16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int device_sms(int* out) {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
    return KCA_ERR_CUDA;
  *out = n;
  return KCA_OK;
}

int q8_args_status(int64_t capacity, int32_t batch, const int64_t* ctx_len) {
  if (capacity < 1 || capacity > KCA_MAX_POSITION) return KCA_ERR_RANGE;
  if (batch < 1 || batch > KCA_MAX_BATCH) return KCA_ERR_RANGE;
  for (int32_t b = 0; b < batch; ++b)
    if (ctx_len[b] < 0 || ctx_len[b] > capacity) return KCA_ERR_RANGE;
  return KCA_OK;
}

std::vector<int64_t> q8_unit_keys(int32_t batch, const int64_t* ctx_len, int32_t window) {
  std::vector<int64_t> nk(batch);
  for (int32_t b = 0; b < batch; ++b) nk[b] = n_visible(ctx_len[b] - 1, window);
  return nk;
}

size_t q8_ws_bytes(const RowsPlan& p) {
  if (p.max_splits <= 1) return KCA_WORKSPACE_HEADER;
  const size_t slots = (size_t)p.n_units * p.max_splits;
  auto al = [](size_t x) { return (x + 255) / 256 * 256; };
  return KCA_WORKSPACE_HEADER + al(slots * kHeads * 2 * 4) + al(slots * kHeads * kDim * 4);
}

}  // namespace
}  // namespace kca

extern "C" {

int attn_quantize_k(const void* k, int32_t k_dtype, int64_t n_rows, void* k8, void* stream) {
  if (!k || !k8) return KCA_ERR_NULL;
  if (!kca::dtype3(k_dtype)) return KCA_ERR_DTYPE;
  if (n_rows < 1 || n_rows > (int64_t)KCA_MAX_BATCH * KCA_MAX_POSITION) return KCA_ERR_RANGE;
  if (!kca::al16(k) || !kca::al16(k8)) return KCA_ERR_ALIGN;
  const dim3 grid((unsigned)((n_rows + 7) / 8));
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  unsigned char* out = static_cast<unsigned char*>(k8);
  if (k_dtype == KCA_F32) kca::quantize_rows_kernel<KCA_F32><<<grid, 256, 0, s>>>(k, n_rows, out);
  else if (k_dtype == KCA_F16) kca::quantize_rows_kernel<KCA_F16><<<grid, 256, 0, s>>>(k, n_rows, out);
  else kca::quantize_rows_kernel<KCA_BF16><<<grid, 256, 0, s>>>(k, n_rows, out);
  return cudaGetLastError() == cudaSuccess ? KCA_OK : KCA_ERR_CUDA;
}

int attn_dot_canary(void* stream, int32_t* variant) {
  if (variant == nullptr) return KCA_ERR_NULL;
  int v = 0;
  const int st = kca::run_canary(static_cast<cudaStream_t>(stream), &v);
  if (st == KCA_OK) *variant = v;
  return st;
}

size_t attn_decode_q8_workspace_bytes(int32_t batch, const int64_t* ctx_len, int32_t window) {
  if (ctx_len == nullptr || kca::q8_args_status(KCA_MAX_POSITION, batch, ctx_len) != KCA_OK) return 0;
  int sms = 0;
  if (kca::device_sms(&sms) != KCA_OK) return 0;
  const std::vector<int64_t> nk = kca::q8_unit_keys(batch, ctx_len, window);
  return kca::q8_ws_bytes(kca::make_rows_plan(batch, nk.data(), sms));
}

int attn_decode_q8(const void* q, int32_t q_dtype, const void* k8_cache, const void* v_cache, int32_t v_dtype,
                   int32_t n_q_heads, int32_t n_kv_heads, int32_t head_dim, int64_t capacity, int32_t batch,
                   const int64_t* ctx_len, int32_t window, float scale, float* out, void* workspace,
                   size_t workspace_bytes, void* stream) {
  if (!q || !k8_cache || !v_cache || !out || !workspace || !ctx_len) return KCA_ERR_NULL;
  if (n_q_heads != KCA_N_Q_HEADS || n_kv_heads != KCA_N_KV_HEADS || head_dim != KCA_HEAD_DIM)
    return KCA_ERR_GEOMETRY;
  if (!kca::dtype3(q_dtype) || !kca::dtype3(v_dtype)) return KCA_ERR_DTYPE;
  int st = kca::q8_args_status(capacity, batch, ctx_len);
  if (st != KCA_OK) return st;
  if (!std::isfinite(scale) || !(scale > 0.f)) return KCA_ERR_RANGE;
  if (!kca::al16(q) || !kca::al16(k8_cache) || !kca::al16(v_cache) || !kca::al16(out)) return KCA_ERR_ALIGN;
  if ((reinterpret_cast<uintptr_t>(workspace) % 256) != 0) return KCA_ERR_WORKSPACE;
  int sms = 0;
  if (kca::device_sms(&sms) != KCA_OK) return KCA_ERR_CUDA;
  const std::vector<int64_t> nk = kca::q8_unit_keys(batch, ctx_len, window);
  const kca::RowsPlan p = kca::make_rows_plan(batch, nk.data(), sms);
  if (workspace_bytes < kca::q8_ws_bytes(p)) return KCA_ERR_WORKSPACE;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  int dp4a = 0;
  st = kca::run_canary(s, &dp4a);
  if (st != KCA_OK) return st;
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
  if (p.max_splits > 1) {
    char* base = static_cast<char*>(workspace) + KCA_WORKSPACE_HEADER;
    const size_t ml = (size_t)batch * p.max_splits * kca::kHeads * 2 * 4;
    a.part_ml = reinterpret_cast<float*>(base);
    a.part_acc = reinterpret_cast<float*>(base + (ml + 255) / 256 * 256);
  }
  for (int32_t b = 0; b < batch; ++b) a.ctx[b] = ctx_len[b];
  return kca::launch_rows_q8(q_dtype, v_dtype, dp4a != 0, a, s) == cudaSuccess ? KCA_OK : KCA_ERR_CUDA;
}

}  // extern "C"

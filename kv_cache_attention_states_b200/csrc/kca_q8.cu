// kca_q8.cu -- the quantised-dot attention's K quantisation and its device
// canary.  K rows are stored as int8 codes with a per-row scale; the decode
// kernels quantise the query the same way per head and take QK exactly on
// the codes -- on int8 tensor-core MMAs in the decode kernel for 16-bit V
// (kca_decode_mma.cu), four int8 pairs per dp4a on the CUDA cores for f32 V
// (kca_rows.cu) -- then the softmax and V sum in f32.
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
// Known answers: kCanary (a, b, c) triples spanning the int8 extremes for
// the dp4a instruction and its emulation, and one int8 tensor-core MMA
// (m16n8k32, the decode kernel's QK instruction) on patterned fragments.
constexpr int kCanary = 64;
__device__ int kca_canary_out[2 * kCanary + 128];

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

// Byte j of fragment register r of lane l (A: r 0..3, B: r 4..5).
__host__ __device__ inline int8_t mma_byte(int lane, int r, int j) {
  return static_cast<int8_t>(((lane * 37 + r * 101 + j * 53) % 255) - 127);
}
__host__ __device__ inline uint32_t mma_reg(int lane, int r) {
  uint32_t x = 0;
  for (int j = 0; j < 4; ++j) x |= static_cast<uint32_t>(static_cast<uint8_t>(mma_byte(lane, r, j))) << (8 * j);
  return x;
}

int dot_ref(uint32_t a, uint32_t b, int c) {
  for (int j = 0; j < 4; ++j)
    c += static_cast<int>(static_cast<int8_t>(a >> (8 * j))) * static_cast<int>(static_cast<int8_t>(b >> (8 * j)));
  return c;
}

__global__ void canary_kernel() {
  const int i = threadIdx.x;
  if (i < kCanary) {
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
  if (i < 32) {   // warp 0: one m16n8k32 int8 MMA
    int d[4] = {0, 0, 0, 0};
    asm volatile(
        "mma.sync.aligned.m16n8k32.row.col.s32.s8.s8.s32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
        "{%0, %1, %2, %3};"
        : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
        : "r"(mma_reg(i, 0)), "r"(mma_reg(i, 1)), "r"(mma_reg(i, 2)), "r"(mma_reg(i, 3)), "r"(mma_reg(i, 4)),
          "r"(mma_reg(i, 5)));
#pragma unroll
    for (int r = 0; r < 4; ++r) kca_canary_out[2 * kCanary + 4 * i + r] = d[r];
  }
}

// The MMA's known answer from its operands' documented fragment layout:
// A (16 x 32, row-major) -- a0 (row g, cols 4t + j), a1 (row g + 8, same
// cols), a2 (row g, cols 16 + 4t + j), a3 (row g + 8, cols 16 + 4t + j);
// B (32 x 8, column-major) -- b0 (rows 4t + j, col g), b1 (rows 16 + 4t + j,
// col g); D -- d0 (g, 2t), d1 (g, 2t + 1), d2 (g + 8, 2t), d3 (g + 8, 2t + 1);
// g = lane / 4, t = lane % 4.
bool mma_answer_ok(const int* got) {
  int A[16][32], B[32][8];
  for (int lane = 0; lane < 32; ++lane) {
    const int g = lane / 4, t = lane % 4;
    for (int j = 0; j < 4; ++j) {
      A[g][4 * t + j] = mma_byte(lane, 0, j);
      A[g + 8][4 * t + j] = mma_byte(lane, 1, j);
      A[g][16 + 4 * t + j] = mma_byte(lane, 2, j);
      A[g + 8][16 + 4 * t + j] = mma_byte(lane, 3, j);
      B[4 * t + j][g] = mma_byte(lane, 4, j);
      B[16 + 4 * t + j][g] = mma_byte(lane, 5, j);
    }
  }
  for (int lane = 0; lane < 32; ++lane) {
    const int g = lane / 4, t = lane % 4;
    const int rows[4] = {g, g, g + 8, g + 8}, cols[4] = {2 * t, 2 * t + 1, 2 * t, 2 * t + 1};
    for (int r = 0; r < 4; ++r) {
      int want = 0;
      for (int k = 0; k < 32; ++k) want += A[rows[r]][k] * B[k][cols[r]];
      if (got[4 * lane + r] != want) return false;
    }
  }
  return true;
}

// Per device: -1 not run, else the mask of sane variants (1 dp4a, 2 its
// emulation, 4 int8 MMA).
std::atomic<int> g_canary[64];
std::mutex g_canary_mu;

int run_canary(cudaStream_t s, int* mask) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return KCA_ERR_CUDA;
  int v = g_canary[dev].load() - 1;
  if (v < 0) {
    std::lock_guard<std::mutex> lock(g_canary_mu);
    v = g_canary[dev].load() - 1;
    if (v < 0) {
      canary_kernel<<<1, kCanary, 0, s>>>();
      int got[2 * kCanary + 128];
      if (cudaGetLastError() != cudaSuccess ||
          cudaMemcpyFromSymbolAsync(got, kca_canary_out, sizeof got, 0, cudaMemcpyDeviceToHost, s) != cudaSuccess ||
          cudaStreamSynchronize(s) != cudaSuccess)
        return KCA_ERR_CUDA;
      bool hw = true, emu = true;
      for (int i = 0; i < kCanary; ++i) {
        uint32_t a, b;
        int c;
        canary_case(i, &a, &b, &c);
        const int want = dot_ref(a, b, c);
        hw = hw && got[i] == want;
        emu = emu && got[kCanary + i] == want;
      }
      v = (hw ? 1 : 0) | (emu ? 2 : 0) | (mma_answer_ok(got + 2 * kCanary) ? 4 : 0);
      g_canary[dev].store(v + 1);
    }
  }
  *mask = v;
  return (v & 3) == 0 ? KCA_ERR_DEVICE : KCA_OK;
}

bool dtype3(int32_t d) { return d == KCA_F32 || d == KCA_F16 || d == KCA_BF16; }
bool al16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace

int dot_canary(cudaStream_t s, int* mask) { return run_canary(s, mask); }

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
  if (st == KCA_OK || st == KCA_ERR_DEVICE) *variant = v;
  return st;
}

}  // extern "C"

// kca_static.cu -- attn_decode_static: attn_decode without a caller-provided
// workspace, for callers that cannot allocate device memory.
//
// Who needs it: code that runs where cudaMalloc is not an option -- inside a
// host callback or a custom allocator's own path, under a memory pool that
// forbids further allocations, or in a runtime that hands out only the
// tensors it owns.  Such a caller still owns q, the caches and out, but cannot
// obtain the scratch that split-context decode writes its per-split partials
// to.  This entry point takes that scratch from a fixed array in device
// memory instead.  The paper has no counterpart to this entry point.
//
// The array below is created when the module loads on a device and is held
// by every GPU that loads the library until the process exits.  Its device
// address is looked up once per device (cudaGetSymbolAddress) on the first
// call made with that device current -- and again if the device's context
// was created anew since (cudaDeviceReset reloads the module, possibly at
// another address); make that first call before any stream capture.  All
// calls on a device share the array, so calls whose execution can overlap
// on the GPU (different streams, or graphs replayed concurrently) race on
// it and must be serialised by the caller.  The array
// keeps the last call's contents.  Its first KCA_WORKSPACE_HEADER bytes must
// be zero when a call starts: the status word, and the counters by which the
// tensor-core decode kernel elects the CTA that merges a row (a call leaves
// them at zero, but one that recorded a device error may not), so every call
// clears them first with cudaMemsetAsync on its stream -- a memset, not an
// allocation.  Everything past the header is written before it is read
// within the same call.  Because of that clear, a call's device status (a
// bounded wait that ran out) survives only until the next call: read it in
// between with attn_device_status on the address that
// attn_decode_static_scratch returns.
#include <cuda.h>
#include <cuda_runtime.h>

#include <mutex>

#include "../../include/kca.h"
#include "kca_plan.h"
#include "kca_rows.h"

namespace {

static __device__ __align__(256) unsigned char kca_static_scratch[KCA_STATIC_SCRATCH_BYTES];

// The current driver context, through the runtime's driver entry point (no
// link-time dependency on libcuda); nullptr when it cannot be read.
CUcontext current_context() {
  using CtxGetCurrentFn = CUresult (*)(CUcontext*);
  static const CtxGetCurrentFn fn = []() -> CtxGetCurrentFn {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      return reinterpret_cast<CtxGetCurrentFn>(p);
    return nullptr;
  }();
  CUcontext c = nullptr;
  if (fn == nullptr || fn(&c) != CUDA_SUCCESS) return nullptr;
  return c;
}

// Device address of kca_static_scratch on the current device; the name itself
// is only a host-side stand-in and must never be handed to a kernel.  Looked
// up once per device and context: a context torn down and created again
// (cudaDeviceReset) loads the module anew, possibly at another address, so
// the cached address is kept together with the context it belongs to.
void* scratch_address(int* status) {
  struct Entry {
    CUcontext ctx;
    void* addr;
  };
  static Entry cache[64];   // zero-initialised; guarded by mu
  static std::mutex mu;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) {
    *status = KCA_ERR_CUDA;
    return nullptr;
  }
  // cudaGetSymbolAddress makes the device's primary context current if no
  // context is, so the context is read after it on a first call.
  const CUcontext ctx = current_context();
  std::lock_guard<std::mutex> lock(mu);
  Entry& e = cache[dev];
  if (e.addr == nullptr || ctx == nullptr || e.ctx != ctx) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, kca_static_scratch) != cudaSuccess || p == nullptr) {
      *status = KCA_ERR_CUDA;
      return nullptr;
    }
    e.addr = p;
    e.ctx = ctx != nullptr ? ctx : current_context();
  }
  *status = KCA_OK;
  return e.addr;
}

}  // namespace

extern "C" int attn_decode_static(const void* q, int32_t q_dtype, const void* k_cache,
                                  const void* v_cache, int32_t kv_dtype, int32_t n_q_heads,
                                  int32_t n_kv_heads, int32_t head_dim, int64_t capacity,
                                  int32_t batch, const int64_t* ctx_len, int32_t window,
                                  float scale, float* out, void* stream) {
  // The checks that need no device come first, so that a bad argument is
  // reported as such before the array's address is looked up.
  int st = kca::decode_args_check(q, q_dtype, k_cache, v_cache, kv_dtype, n_q_heads, n_kv_heads, head_dim,
                                  capacity, batch, ctx_len, scale, out);
  if (st != KCA_OK) return st;
  void* ws = scratch_address(&st);
  if (ws == nullptr) return st;
  // attn_decode's checks (KCA_ERR_WORKSPACE when the plan's partials would
  // not fit the array); once they pass, the header is cleared, then the
  // kernel is launched.  A call that fails validation touches nothing.
  return kca::decode_entry(q, q_dtype, k_cache, v_cache, kv_dtype, n_q_heads, n_kv_heads, head_dim, capacity,
                           batch, ctx_len, window, scale, out, ws, KCA_STATIC_SCRATCH_BYTES, stream, true);
}

extern "C" int attn_decode_static_scratch(void** device_ptr, size_t* bytes) {
  if (device_ptr == nullptr) return KCA_ERR_NULL;
  int st = KCA_OK;
  void* p = scratch_address(&st);
  if (p == nullptr) return st;
  *device_ptr = p;
  if (bytes != nullptr) *bytes = KCA_STATIC_SCRATCH_BYTES;
  return KCA_OK;
}

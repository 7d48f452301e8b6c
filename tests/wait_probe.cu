// Test harness for the library's bounded waits (kca_common.cuh), built by
// tests/test_gpu_bounded_wait.py with nvcc; not part of the library.  The
// wait limit is shortened to 1 ms so that a wait nothing will complete gives
// up quickly; the kernel then returns normally.
#define KCA_WAIT_LIMIT_NS 1000000ull
#include <cuda_runtime.h>

#include "kca_common.cuh"

// One thread: an mbarrier expecting one arrival; `arrive` says whether that
// arrival happens before the wait.  out[0] = 1 if the wait succeeded.
__global__ void wait_probe_kernel(kca::DeviceStatus* status, int arrive, unsigned int site, int* out) {
  __shared__ uint64_t bar;
  if (threadIdx.x != 0) return;
  kca::mbar_init(&bar, 1);
  kca::fence_barrier_init();
  if (arrive) kca::mbar_arrive(&bar);
  out[0] = kca::mbar_wait(&bar, 0, nullptr, status, site) ? 1 : 0;
}

extern "C" int wait_probe(void* status, int arrive, unsigned int site, int* out) {
  wait_probe_kernel<<<1, 32>>>(static_cast<kca::DeviceStatus*>(status), arrive, site, out);
  if (cudaGetLastError() != cudaSuccess) return -1;
  return cudaDeviceSynchronize() == cudaSuccess ? 0 : -2;
}

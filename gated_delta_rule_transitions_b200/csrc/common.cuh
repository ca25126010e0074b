// Shared device/host helpers of libhla (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/hla.h"

namespace hla {

// Load one element as float from float or bf16 storage.
__device__ __forceinline__ float ldf(const float* p) { return *p; }
__device__ __forceinline__ float ldf(const __nv_bfloat16* p) { return __bfloat162float(*p); }

// Store float into float or bf16 storage (round to nearest even).
__device__ __forceinline__ void stf(float* p, float x) { *p = x; }
__device__ __forceinline__ void stf(__nv_bfloat16* p, float x) { *p = __float2bfloat16_rn(x); }

// Device-side error word for bounded waits.  Each translation unit that waits
// defines its own word (no relocatable device code is needed) and a host accessor
// that hla_device_status calls.
enum : unsigned int {
  kErrNone = 0,
  kErrMbarTimeout = 1u,   // an mbarrier wait gave up
  kErrTmemAlloc = 2u,     // tensor-memory allocation could not be satisfied
  kErrCacheFull = 4u,     // a decode step had to close a chunk into a full cache
  kErrDecayRange = 8u,    // a channel's decay over one sub-chunk left the tensor-core range
};

// Streaming multiprocessors of the current device (read once per process; the
// library runs on one kind of GPU).
inline int num_sms() {
  static int n = 0;
  if (n == 0) {
    int dev = 0, v = 0;
    if (cudaGetDevice(&dev) == cudaSuccess &&
        cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess && v > 0)
      n = v;
    else
      return 148;
  }
  return n;
}

#define HLA_DEFINE_ERROR_WORD(tu)                                                      \
  static __device__ unsigned int g_err_word;                                          \
  __device__ __forceinline__ void report_device_error(unsigned int code) {            \
    atomicOr(&g_err_word, code);                                                      \
  }                                                                                   \
  cudaError_t read_error_word_##tu(unsigned int* out, bool clear) {                   \
    cudaError_t e = cudaMemcpyFromSymbol(out, g_err_word, sizeof(unsigned int));      \
    if (e != cudaSuccess || !clear) return e;                                         \
    const unsigned int z = 0;                                                         \
    return cudaMemcpyToSymbol(g_err_word, &z, sizeof(unsigned int));                  \
  }


}  // namespace hla

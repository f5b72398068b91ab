// Shared definitions for the POET-X CUDA library (single translation unit: poetx.cu).
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/poetx.h"

namespace poetx {

enum DType : int { F32 = 0, BF16 = 1 };

__host__ __device__ inline int dtype_size(int dt) { return dt == BF16 ? 2 : 4; }

// Device-side error word.  Kernels that give up on a bounded wait record
// (kernel_id << 8 | site) here with the first writer winning; poetx_device_status() reads and
// clears it.  0 means no error.
__device__ int g_device_error = 0;

// A bounded wait gives up after this many nanoseconds of %globaltimer.  A legitimate wait in
// these kernels lasts microseconds; two seconds only ever runs out on a real fault.
constexpr unsigned long long kWaitLimitNs = 2000000000ull;

__device__ __forceinline__ unsigned long long global_timer_ns() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ void record_device_error(int kernel_id, int site) {
  atomicCAS(&g_device_error, 0, (kernel_id << 8) | (site & 0xff));
}

__device__ __forceinline__ float bf16_to_f32(__nv_bfloat16 v) { return __bfloat162float(v); }

// Load / store one value of a runtime-typed array.
__device__ __forceinline__ float load_elem(const void* p, long idx, int dt) {
  return dt == BF16 ? __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(p)[idx])
                    : reinterpret_cast<const float*>(p)[idx];
}
__device__ __forceinline__ void store_elem(void* p, long idx, int dt, float v) {
  if (dt == BF16)
    reinterpret_cast<__nv_bfloat16*>(p)[idx] = __float2bfloat16_rn(v);
  else
    reinterpret_cast<float*>(p)[idx] = v;
}

}  // namespace poetx

// Shared definitions for the POET-X CUDA library (single translation unit: poetx.cu).
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/poetx.h"

namespace poetx {

enum DType : int { F32 = 0, BF16 = 1, U8 = 2 /* int8 codes, tensor maps only */ };

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

// Eight int8 codes (w: byte e = code e) -> eight bf16 scale * code (lowest address first).
// Each code is turned into a float exactly with integer moves only: the byte, offset to
// unsigned (code + 128), becomes the low mantissa byte of 2^23 (0x4B000000), so the float is
// 2^23 + 128 + code and one subtraction of 2^23 + 128 leaves the code.  The product with the
// scale is then rounded once to bf16 (nearest even).
__device__ __forceinline__ uint4 dequant8_bf16(uint2 w, float scale) {
  const uint32_t x[2] = {w.x ^ 0x80808080u, w.y ^ 0x80808080u};
  uint32_t o[4];
#pragma unroll
  for (int h = 0; h < 2; ++h) {
#pragma unroll
    for (int p = 0; p < 2; ++p) {
      const float lo = __uint_as_float(__byte_perm(x[h], 0x4B000000u, 0x7540u | (2 * p))) - 8388736.f;
      const float hi = __uint_as_float(__byte_perm(x[h], 0x4B000000u, 0x7540u | (2 * p + 1))) - 8388736.f;
      const __nv_bfloat162 v = __floats2bfloat162_rn(lo * scale, hi * scale);
      o[2 * h + p] = *reinterpret_cast<const uint32_t*>(&v);
    }
  }
  return make_uint4(o[0], o[1], o[2], o[3]);
}

}  // namespace poetx

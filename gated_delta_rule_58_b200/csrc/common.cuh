// Internal helpers shared by the libgdn.so translation units (not part of the ABI).
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <stdint.h>

#include <string>

#include "gdn.h"

namespace gdn {

// ---- host-side status reporting -------------------------------------------------

// Records a thread-local message for gdn_last_error() and returns `st`.
gdn_status_t fail(gdn_status_t st, const std::string& msg);
// Clears the thread-local message and returns GDN_OK.
gdn_status_t ok();
// Converts the last launch error (if any) into GDN_ERR_CUDA with a message.
gdn_status_t check_launch(const char* what);

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
inline cudaStream_t as_stream(void* s) { return reinterpret_cast<cudaStream_t>(s); }

// ---- device-side sticky error word ---------------------------------------------

// One word per device, defined in gdn_api.cu; kernels get its address as a
// parameter (no relocatable device code). Bits are GDN_DEVERR_*.
// Returns the device address of the word for the current device (cached).
gdn_status_t device_error_word(unsigned int** word);

__device__ __forceinline__ void raise_device_error(unsigned int* word, unsigned int bits) {
  atomicOr(word, bits);
}

// ---- element conversion ---------------------------------------------------------

__device__ __forceinline__ float to_f32(__nv_bfloat16 x) { return __bfloat162float(x); }
__device__ __forceinline__ float to_f32(float x) { return x; }

__device__ __forceinline__ void store_out(float* p, float x) { *p = x; }
__device__ __forceinline__ void store_out(__nv_bfloat16* p, float x) { *p = __float2bfloat16_rn(x); }

// Loads 8 consecutive elements (16 B of bf16 or 32 B of fp32) as fp32.
__device__ __forceinline__ void load8_f32(const __nv_bfloat16* p, float* out) {
  const uint4 raw = *reinterpret_cast<const uint4*>(p);
  const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&raw);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 f = __bfloat1622float2(h[i]);
    out[2 * i] = f.x;
    out[2 * i + 1] = f.y;
  }
}
__device__ __forceinline__ void load8_f32(const float* p, float* out) {
  const float4 a = *reinterpret_cast<const float4*>(p);
  const float4 b = *reinterpret_cast<const float4*>(p + 4);
  out[0] = a.x; out[1] = a.y; out[2] = a.z; out[3] = a.w;
  out[4] = b.x; out[5] = b.y; out[6] = b.z; out[7] = b.w;
}

}  // namespace gdn

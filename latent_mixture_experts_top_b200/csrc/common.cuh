// common.cuh -- small device helpers shared by the LatentMoE kernels.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace lmoe {

// Device-side status codes written to the handle's sticky status word.
enum : int {
  DEV_OK = 0,
  DEV_TIMEOUT_PRODUCER = 1,   // TMA producer waited too long for a free stage
  DEV_TIMEOUT_MMA = 2,        // MMA issuer waited too long for data / accumulator
  DEV_TIMEOUT_EPILOGUE = 3,   // epilogue waited too long for an accumulator
  DEV_TIMEOUT_DRAIN = 4,      // abort path: in-flight copies did not land
};

// Every spin-wait in these kernels gives up after this long and records a
// status instead of hanging the GPU.  Healthy waits last microseconds.
constexpr unsigned long long kWaitLimitNs = 2000000000ull;  // 2 s

__device__ __forceinline__ unsigned long long globaltimer_ns() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ float bf16_to_f32(__nv_bfloat16 v) { return __bfloat162float(v); }
__device__ __forceinline__ float to_f32(float v) { return v; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 v) { return __bfloat162float(v); }

template <typename T> __device__ __forceinline__ T from_f32(float v);
template <> __device__ __forceinline__ float from_f32<float>(float v) { return v; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float v) {
  return __float2bfloat16_rn(v);
}

// silu(a) = a * sigmoid(a) = a / (1 + e^-a), with the CUDA math library's expf.
__device__ __forceinline__ float silu_f32(float a) { return a / (1.0f + expf(-a)); }

// Two floats -> packed bf16x2 (low half = first), round to nearest even.
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t *>(&v);
}

}  // namespace lmoe

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
  DEV_TIMEOUT_SELFTEST = 5,   // the failure-detection self-test's wait ran out
};

// Every spin-wait in these kernels gives up after this long and records a
// status instead of hanging the GPU.  Healthy waits last microseconds.
constexpr unsigned long long kWaitLimitNs = 2000000000ull;  // 2 s

// Programmatic dependent launch.  A kernel launched with programmatic stream
// serialization may start while the previous kernel of its stream is still
// running; griddep_wait blocks until that kernel has completed and its
// memory is visible (it returns at once in a kernel launched without it), so
// every kernel calls it before its first global-memory access.
// griddep_launch_dependents lets the next kernel be scheduled early.
__device__ __forceinline__ void griddep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void griddep_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" :::);
}

// Host: launches `kernel` on `s`, with programmatic stream serialization
// when pdl is set (see griddep_wait).
template <typename... Params, typename... Args>
inline cudaError_t launch_ex(void (*kernel)(Params...), dim3 grid, dim3 block, size_t smem,
                             cudaStream_t s, bool pdl, Args &&...args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, kernel, static_cast<Args &&>(args)...);
}

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

// silu(a) = a * sigmoid(a) = a / (1 + e^-a), with the CUDA math library's expf
// (fp32 mode, held to 1e-5).
__device__ __forceinline__ float silu_f32(float a) { return a / (1.0f + expf(-a)); }

// Hardware tanh (PTX tanh.approx.f32, one MUFU op; absolute error about 5e-4).
__device__ __forceinline__ float tanh_approx(float x) {
  float y;
  asm("tanh.approx.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// silu for the bf16 epilogues, from sigmoid(a) = (1 + tanh(a/2)) / 2:
// silu(a) = h + h * tanh(h) with h = a/2.  Its error (~5e-4 relative) is
// below half a bf16 ulp of the result, which is rounded to bf16 anyway.
__device__ __forceinline__ float silu_bf16out(float a) {
  const float h = 0.5f * a;
  return fmaf(h, tanh_approx(h), h);
}

// Two floats -> packed bf16x2 (low half = first), round to nearest even.
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t *>(&v);
}

}  // namespace lmoe

// fp8_weights.cu -- E4M3 expert weights for the decode regime.
//
// "LatentMoE Explained" puts an expert at about 22 MB in FP8 and notes the
// models are pretrained in NVFP4; it gives no scaling recipe.  The recipe
// here: every weight row r (one output feature) gets a power-of-two scale
// s_r = 2^e_r, the smallest with max_c |W[r][c]| <= 448 s_r (448 = the
// largest finite E4M3 value), and each element is stored as the E4M3 code of
// W[r][c] / s_r, rounded to nearest (ties to even) with saturation.  W / s_r
// is exact (s_r is a power of two), so the stored matrix times the scales is
// exactly the weight the GEMM computes with.
#include <cuda_bf16.h>
#include <cuda_fp8.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "common.cuh"
#include "kernels.h"

namespace lmoe {
namespace {

// The row scale: the smallest power of two s with amax <= 448 s (448 = 1.75
// 2^8, the largest finite E4M3 value); 1 for a row of zeros.  Exact float-bit
// arithmetic: amax = (m/2) 2^ea with m in [1, 2) from frexp.
__device__ __forceinline__ int e4m3_scale_exp(float amax) {
  if (!(amax > 0.0f)) return 0;
  int ea;
  const float m = 2.0f * frexpf(amax, &ea);
  ea -= 1;                                 // amax = m 2^ea, m in [1, 2)
  return m <= 1.75f ? ea - 8 : ea - 7;
}

// Eight bf16 values (one 16-byte vector) scaled by inv -> eight E4M3 codes
// (round to nearest even, saturating), packed little-endian in two words.
__device__ __forceinline__ uint2 e4m3x8(const uint4 q, float inv) {
  const uint32_t qs[4] = {q.x, q.y, q.z, q.w};
  uint32_t out[2] = {0u, 0u};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const uint32_t c0 = __nv_cvt_float_to_fp8(__uint_as_float(qs[i] << 16) * inv, __NV_SATFINITE,
                                              __NV_E4M3);
    const uint32_t c1 = __nv_cvt_float_to_fp8(__uint_as_float(qs[i] & 0xFFFF0000u) * inv,
                                              __NV_SATFINITE, __NV_E4M3);
    out[i >> 1] |= (c0 | (c1 << 8)) << (16 * (i & 1));
  }
  return make_uint2(out[0], out[1]);
}

// Warp-wide max |x| over one bf16 row of nv 16-byte vectors (four loads in
// flight per lane).
__device__ __forceinline__ float row_amax(const uint4 *w, int nv, int lane) {
  float amax = 0.0f;
  for (int v0 = lane; v0 < nv; v0 += 128) {
    uint4 q[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) q[u] = v0 + 32 * u < nv ? w[v0 + 32 * u] : make_uint4(0, 0, 0, 0);
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const uint32_t qs[4] = {q[u].x, q[u].y, q[u].z, q[u].w};
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        amax = fmaxf(amax, fabsf(__uint_as_float(qs[i] << 16)));
        amax = fmaxf(amax, fabsf(__uint_as_float(qs[i] & 0xFFFF0000u)));
      }
    }
  }
#pragma unroll
  for (int off = 16; off; off >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, off));
  return amax;
}

// One warp per weight row.  src [groups][rows][cols] bf16; codes written in
// blocks of 256 rows x 128 bytes (per group, 256-row tile n, 128-column block
// kb), scales [groups][rows] f32.  cols % 128 == 0.
__global__ void __launch_bounds__(256) quantize_rows_e4m3_kernel(
    const __nv_bfloat16 *__restrict__ src, long long n_rows, int rows_per_group, int cols, int nt,
    float *__restrict__ scales, uint8_t *__restrict__ dst) {
  const long long row = static_cast<long long>(blockIdx.x) * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= n_rows) return;
  const uint4 *w = reinterpret_cast<const uint4 *>(src + row * cols);
  const int nv = cols / 8;
  const int e = e4m3_scale_exp(row_amax(w, nv, lane));
  const float s = ldexpf(1.0f, e), inv = ldexpf(1.0f, -e);
  if (lane == 0) scales[row] = s;
  const long long g = row / rows_per_group;
  const int r = static_cast<int>(row % rows_per_group);
  const int n = r >> 8, rr = r & 255, kbc = cols / 128;
  for (int v = lane; v < nv; v += 32) {
    const int c = v * 8, kb = c >> 7;
    uint8_t *blk = dst + (((g * nt + n) * kbc + kb) * 256 + rr) * 128 + (c & 127);
    *reinterpret_cast<uint2 *>(blk) = e4m3x8(w[v], inv);
  }
}

// One warp per activation row (see launch_quantize_rows_e4m3).
__global__ void __launch_bounds__(256) quantize_act_rows_kernel(
    const __nv_bfloat16 *__restrict__ src, const int32_t *__restrict__ gather, int K, int rows,
    int cols, uint8_t *__restrict__ dst, float *__restrict__ scales) {
  const int row = blockIdx.x * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  griddep_wait();
  if (row >= rows) return;
  const int srow = gather ? gather[row] / K : row;
  const uint4 *w = reinterpret_cast<const uint4 *>(src + static_cast<size_t>(srow) * cols);
  const int nv = cols / 8;
  const int e = e4m3_scale_exp(row_amax(w, nv, lane));
  const float inv = ldexpf(1.0f, -e);
  if (lane == 0) scales[row] = ldexpf(1.0f, e);
  uint2 *d = reinterpret_cast<uint2 *>(dst + static_cast<size_t>(row) * cols);
  for (int v = lane; v < nv; v += 32) d[v] = e4m3x8(w[v], inv);
}

}  // namespace

cudaError_t launch_quantize_e4m3_tiles(const __nv_bfloat16 *src, int groups, int rows_per_group,
                                       int cols, float *scales, uint8_t *dst, cudaStream_t s) {
  if (cols % 128 || groups <= 0 || rows_per_group <= 0) return cudaErrorInvalidValue;
  const int nt = (rows_per_group + 255) / 256;
  const size_t bytes = static_cast<size_t>(groups) * nt * 256 * cols;
  cudaError_t e = cudaMemsetAsync(dst, 0, bytes, s);  // padding rows stay zero
  if (e != cudaSuccess) return e;
  const long long n_rows = static_cast<long long>(groups) * rows_per_group;
  quantize_rows_e4m3_kernel<<<static_cast<unsigned>((n_rows + 7) / 8), 256, 0, s>>>(
      src, n_rows, rows_per_group, cols, nt, scales, dst);
  return cudaGetLastError();
}

cudaError_t launch_quantize_rows_e4m3(const __nv_bfloat16 *src, const int32_t *gather, int K,
                                      int rows, int cols, uint8_t *dst, float *scales,
                                      cudaStream_t s, bool pdl) {
  if (rows <= 0) return cudaSuccess;
  if (cols % 8 || (gather && K <= 0)) return cudaErrorInvalidValue;
  const cudaError_t e = launch_ex(quantize_act_rows_kernel, dim3((rows + 7) / 8), dim3(256), 0, s,
                                  pdl, src, gather, K, rows, cols, dst, scales);
  return e != cudaSuccess ? e : cudaGetLastError();
}

}  // namespace lmoe

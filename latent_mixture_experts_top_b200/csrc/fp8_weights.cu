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

#include "kernels.h"

namespace lmoe {
namespace {

// One warp per weight row.  src [groups][rows][cols] bf16; codes written K-block
// tiled (per group, 256-row tile n and 64-column block kb: one 256 x 64 byte
// block), scales [groups][rows] f32.  cols % 64 == 0.
__global__ void __launch_bounds__(256) quantize_rows_e4m3_kernel(
    const __nv_bfloat16 *__restrict__ src, long long n_rows, int rows_per_group, int cols, int nt,
    float *__restrict__ scales, uint8_t *__restrict__ dst) {
  const long long row = static_cast<long long>(blockIdx.x) * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= n_rows) return;
  const uint4 *w = reinterpret_cast<const uint4 *>(src + row * cols);
  const int nv = cols / 8;
  float amax = 0.0f;
  for (int v = lane; v < nv; v += 32) {
    const uint4 q = w[v];
    const uint32_t qs[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      amax = fmaxf(amax, fabsf(__uint_as_float(qs[i] << 16)));
      amax = fmaxf(amax, fabsf(__uint_as_float(qs[i] & 0xFFFF0000u)));
    }
  }
#pragma unroll
  for (int off = 16; off; off >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, off));
  // amax = m 2^ea, m in [1, 2): the smallest e with amax <= 1.75 * 2^(8 + e)
  // is ea - 8 when m <= 1.75, else ea - 7.
  int e = 0;
  if (amax > 0.0f) {
    int ea;
    const float m = 2.0f * frexpf(amax, &ea);  // amax = (m/2) 2^ea, m in [1, 2)
    ea -= 1;
    e = m <= 1.75f ? ea - 8 : ea - 7;
  }
  const float s = ldexpf(1.0f, e), inv = ldexpf(1.0f, -e);
  if (lane == 0) scales[row] = s;
  const long long g = row / rows_per_group;
  const int r = static_cast<int>(row % rows_per_group);
  const int n = r >> 8, rr = r & 255, kbc = cols / 64;
  for (int v = lane; v < nv; v += 32) {
    const uint4 q = w[v];
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
    const int c = v * 8, kb = c >> 6;
    uint8_t *blk = dst + (((g * nt + n) * kbc + kb) * 256 + rr) * 64 + (c & 63);
    *reinterpret_cast<uint2 *>(blk) = make_uint2(out[0], out[1]);
  }
}

}  // namespace

cudaError_t launch_quantize_e4m3_tiles(const __nv_bfloat16 *src, int groups, int rows_per_group,
                                       int cols, float *scales, uint8_t *dst, cudaStream_t s) {
  if (cols % 64 || groups <= 0 || rows_per_group <= 0) return cudaErrorInvalidValue;
  const int nt = (rows_per_group + 255) / 256;
  const size_t bytes = static_cast<size_t>(groups) * nt * (cols / 64) * 256 * 64;
  cudaError_t e = cudaMemsetAsync(dst, 0, bytes, s);  // padding rows stay zero
  if (e != cudaSuccess) return e;
  const long long n_rows = static_cast<long long>(groups) * rows_per_group;
  quantize_rows_e4m3_kernel<<<static_cast<unsigned>((n_rows + 7) / 8), 256, 0, s>>>(
      src, n_rows, rows_per_group, cols, nt, scales, dst);
  return cudaGetLastError();
}

}  // namespace lmoe

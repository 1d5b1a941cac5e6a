// simt_kernels.cu -- fp32 CUDA-core kernels of the fp32 mode.
//
// The fp32 mode is held to 1e-5 relative error, which tensor-core TF32 would
// miss, so every product here is an fp32 FMA on the CUDA cores, accumulated in
// ascending reduction order.  Each GEMM stages 64-row A and B tiles through
// shared memory (32-wide K slices); one thread computes a 4x4 block.
// Source of the maths: "LatentMoE Explained", Figure 6 (W_down / W_up),
// Figure 9 (latent expert), and the SwiGLU expert of the paragraph after
// Figure 1.
#include <stdint.h>

#include "common.cuh"
#include "kernels.h"

namespace lmoe {
namespace {

constexpr int BM = 64, BN = 64, BK = 32;

// C[r][c] = sum_k A[r][k] * B[c][k]   (A [M][K] lda, B [N][K] ldb)
__global__ void __launch_bounds__(256) simt_linear_kernel(const float *__restrict__ A, int lda,
                                                          const float *__restrict__ B, int ldb,
                                                          float *__restrict__ C, int ldc, int M,
                                                          int N, int Kd) {
  __shared__ float As[BK][BM + 1];
  __shared__ float Bs[BK][BN + 1];
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  const int r0 = blockIdx.y * BM, c0 = blockIdx.x * BN;
  float acc[4][4] = {};
  for (int k0 = 0; k0 < Kd; k0 += BK) {
    for (int i = threadIdx.x; i < BM * BK; i += 256) {
      const int rr = i / BK, kk = i % BK;
      const int r = r0 + rr, k = k0 + kk, c = c0 + rr;
      As[kk][rr] = (r < M && k < Kd) ? A[static_cast<size_t>(r) * lda + k] : 0.0f;
      Bs[kk][rr] = (c < N && k < Kd) ? B[static_cast<size_t>(c) * ldb + k] : 0.0f;
    }
    __syncthreads();
#pragma unroll 8
    for (int kk = 0; kk < BK; ++kk) {
      float a[4], b[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) a[i] = As[kk][ty * 4 + i];
#pragma unroll
      for (int j = 0; j < 4; ++j) b[j] = Bs[kk][tx * 4 + j];
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int r = r0 + ty * 4 + i;
    if (r >= M) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int c = c0 + tx * 4 + j;
      if (c < N) C[static_cast<size_t>(r) * ldc + c] = acc[i][j];
    }
  }
}

// Weight row of column c for row r: expert e = row_expert[r] or c / mw.
__device__ __forceinline__ size_t wrow(const int32_t *row_expert, int r, int c, int mw, int Kd) {
  const int e = row_expert ? row_expert[r] : c / mw;
  return (static_cast<size_t>(e) * mw + (c % mw)) * Kd;
}

// SwiGLU hidden: H[r][c] = silu(A_r . Wg_row) * (A_r . Wu_row).  Rows of a
// block may belong to different experts, so B is read per thread (cached).
__global__ void __launch_bounds__(256) simt_swiglu_kernel(const float *__restrict__ A, int lda,
                                                          const float *__restrict__ Wg,
                                                          const float *__restrict__ Wu, int mw,
                                                          const int32_t *__restrict__ row_expert,
                                                          float *__restrict__ H, int ldh, int M,
                                                          int Ncols, int Kd) {
  const int c = blockIdx.y * 64 + (threadIdx.x & 63);  // rows on x: up to 2^31 - 1
  const int r = blockIdx.x * 4 + (threadIdx.x >> 6);
  if (r >= M || c >= Ncols) return;
  const float *a = A + static_cast<size_t>(r) * lda;
  const size_t wr = wrow(row_expert, r, c, mw, Kd);
  const float *g = Wg + wr, *u = Wu + wr;
  float sg = 0.0f, su = 0.0f;
  for (int k = 0; k < Kd; ++k) {
    sg = fmaf(a[k], g[k], sg);
    su = fmaf(a[k], u[k], su);
  }
  H[static_cast<size_t>(r) * ldh + c] = silu_f32(sg) * su;
}

// Squared-ReLU hidden: H[r][c] = relu(A_r . Wu_row)^2 (the article's Expert class).
__global__ void __launch_bounds__(256) simt_relu2_kernel(const float *__restrict__ A, int lda,
                                                         const float *__restrict__ Wu, int mw,
                                                         const int32_t *__restrict__ row_expert,
                                                         float *__restrict__ H, int ldh, int M,
                                                         int Ncols, int Kd) {
  const int c = blockIdx.y * 64 + (threadIdx.x & 63);  // rows on x: up to 2^31 - 1
  const int r = blockIdx.x * 4 + (threadIdx.x >> 6);
  if (r >= M || c >= Ncols) return;
  const float *a = A + static_cast<size_t>(r) * lda;
  const float *u = Wu + wrow(row_expert, r, c, mw, Kd);
  float su = 0.0f;
  for (int k = 0; k < Kd; ++k) su = fmaf(a[k], u[k], su);
  const float h = su > 0.0f ? su : 0.0f;
  H[static_cast<size_t>(r) * ldh + c] = h * h;
}

__global__ void __launch_bounds__(256) simt_expert_down_kernel(
    const float *__restrict__ Hm, int ldh, const float *__restrict__ Wo,
    const int32_t *__restrict__ row_expert, float *__restrict__ O, int ldo, int M, int Ncols,
    int Kd) {
  const int c = blockIdx.y * 64 + (threadIdx.x & 63);  // rows on x: up to 2^31 - 1
  const int r = blockIdx.x * 4 + (threadIdx.x >> 6);
  if (r >= M || c >= Ncols) return;
  const float *h = Hm + static_cast<size_t>(r) * ldh;
  const float *w = Wo + (static_cast<size_t>(row_expert[r]) * Ncols + c) * Kd;
  float acc = 0.0f;
  for (int k = 0; k < Kd; ++k) acc = fmaf(h[k], w[k], acc);
  O[static_cast<size_t>(r) * ldo + c] = acc;
}

}  // namespace

cudaError_t simt_linear(const float *A, int lda, const float *B, int ldb, float *C, int ldc,
                        int M, int N, int Kdim, cudaStream_t s) {
  if (M <= 0 || N <= 0) return cudaSuccess;
  dim3 grid((N + BN - 1) / BN, (M + BM - 1) / BM);
  simt_linear_kernel<<<grid, 256, 0, s>>>(A, lda, B, ldb, C, ldc, M, N, Kdim);
  return cudaGetLastError();
}

cudaError_t simt_swiglu(const float *A, int lda, const float *Wg, const float *Wu, int mw,
                        const int32_t *row_expert, float *H, int ldh, int M, int Ncols, int Kdim,
                        cudaStream_t s) {
  if (M <= 0 || Ncols <= 0) return cudaSuccess;
  dim3 grid((M + 3) / 4, (Ncols + 63) / 64);
  simt_swiglu_kernel<<<grid, 256, 0, s>>>(A, lda, Wg, Wu, mw, row_expert, H, ldh, M, Ncols, Kdim);
  return cudaGetLastError();
}

cudaError_t simt_relu2(const float *A, int lda, const float *Wu, int mw,
                       const int32_t *row_expert, float *H, int ldh, int M, int Ncols, int Kdim,
                       cudaStream_t s) {
  if (M <= 0 || Ncols <= 0) return cudaSuccess;
  dim3 grid((M + 3) / 4, (Ncols + 63) / 64);
  simt_relu2_kernel<<<grid, 256, 0, s>>>(A, lda, Wu, mw, row_expert, H, ldh, M, Ncols, Kdim);
  return cudaGetLastError();
}

cudaError_t simt_expert_down(const float *H, int ldh, const float *Wo, const int32_t *row_expert,
                             float *O, int ldo, int M, int Ncols, int Kdim, cudaStream_t s) {
  if (M <= 0 || Ncols <= 0) return cudaSuccess;
  dim3 grid((M + 3) / 4, (Ncols + 63) / 64);
  simt_expert_down_kernel<<<grid, 256, 0, s>>>(H, ldh, Wo, row_expert, O, ldo, M, Ncols, Kdim);
  return cudaGetLastError();
}

}  // namespace lmoe

// backward_kernels.cu -- kernels of the layer backward (the gradient for an
// output cotangent dy), the steps that are not tensor-core GEMMs, plus the
// fp32 CUDA-core GEMMs of the fp32 mode.
//
// The backward is the chain rule through the forward of "LatentMoE
// Explained" (Figure 3 router, Figure 6 W_down / W_up, Figure 9 latent
// expert, the LatentMoE code module's softmax / top-K / renormalise and slot
// loop) for what loss.backward() of the Latent-MoE README's Usage example
// computes: per token, du = W_up^T dy; per slot dg_k = du . o_k and
// do_k = g_k du; the expert's hidden gradient; ds_{id_k} = g_k (dg_k -
// sum_j g_j dg_j) through the renormalised gates; dz = sum over slots of the
// expert input gradients; dx = W_r^T ds + W_down^T dz + the shared experts'.
#include <algorithm>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "common.cuh"
#include "kernels.h"

namespace lmoe {
namespace {

template <typename T>
__device__ __forceinline__ float ld(const T *p, size_t i);
template <>
__device__ __forceinline__ float ld<float>(const float *p, size_t i) { return p[i]; }
template <typename T>
__device__ __forceinline__ void st(T *p, size_t i, float v);
template <>
__device__ __forceinline__ void st<float>(float *p, size_t i, float v) { p[i] = v; }
template <>
__device__ __forceinline__ void st<__nv_bfloat16>(__nv_bfloat16 *p, size_t i, float v) {
  p[i] = __float2bfloat16_rn(v);
}

// ---------------------------------------------------------------- fp32 GEMM
// C[g](i, j) (+)= sum_k A[g](i, k) * B[g](j, k) with arbitrary strides, so
// that transposed operands need no copies; optional per-group ranges of k
// (grouped weight gradients: the rows of one expert) read from the device.
constexpr int SBM = 64, SBN = 64, SBK = 16;

__global__ void __launch_bounds__(256) simt_gemm_kernel(SimtGemm g) {
  __shared__ float As[SBK][SBM + 1];
  __shared__ float Bs[SBK][SBN + 1];
  const int grp = blockIdx.z;
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  const int r0 = blockIdx.y * SBM, c0 = blockIdx.x * SBN;
  const float *A = g.A + grp * g.sA_g;
  const float *B = g.B + grp * g.sB_g;
  int k_begin = 0, k_end = g.K;
  if (g.k_off) {
    k_begin = g.k_off[grp];
    k_end = g.k_off[grp + 1];
  }
  float acc[4][4] = {};
  for (int k0 = k_begin; k0 < k_end; k0 += SBK) {
    for (int i = threadIdx.x; i < SBM * SBK; i += 256) {
      const int rr = i % SBM, kk = i / SBM;
      const int r = r0 + rr, c = c0 + rr, k = k0 + kk;
      As[kk][rr] = (r < g.M && k < k_end) ? A[r * g.sA_r + static_cast<long long>(k) * g.sA_k] : 0.0f;
      Bs[kk][rr] = (c < g.N && k < k_end) ? B[c * g.sB_r + static_cast<long long>(k) * g.sB_k] : 0.0f;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < SBK; ++kk) {
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
  float *C = g.C + grp * g.sC_g;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int r = r0 + ty * 4 + i;
    if (r >= g.M) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int c = c0 + tx * 4 + j;
      if (c >= g.N) continue;
      float *dst = C + r * g.ldc + c;
      *dst = g.accumulate ? *dst + acc[i][j] : acc[i][j];
    }
  }
}

// C[r][c] (+)= sum_k A[r][k] * W(e, c, k), e = row_expert[r], W(e, c, k) at
// W[e*sW_e + c*sW_r + k*sW_k]: expert products of permuted rows, any weight
// orientation.
__global__ void __launch_bounds__(256) simt_rowexpert_kernel(
    const float *__restrict__ A, int lda, const float *__restrict__ W, long long sW_e,
    long long sW_r, long long sW_k, const int32_t *__restrict__ row_expert,
    float *__restrict__ C, int ldc, int M, int Ncols, int Kd, int accumulate) {
  const int c = blockIdx.y * 64 + (threadIdx.x & 63);
  const int r = blockIdx.x * 4 + (threadIdx.x >> 6);
  if (r >= M || c >= Ncols) return;
  const float *a = A + static_cast<size_t>(r) * lda;
  const float *w = W + row_expert[r] * sW_e + c * sW_r;
  float acc = 0.0f;
  for (int k = 0; k < Kd; ++k) acc = fmaf(a[k], w[k * sW_k], acc);
  float *dst = C + static_cast<size_t>(r) * ldc + c;
  *dst = accumulate ? *dst + acc : acc;
}

// ------------------------------------------------------- activation backward
// Per element of [rows][n]: from the pre-activations a (gate), b (up) and the
// hidden gradient dh, the hidden h and the pre-activation gradients.
// SwiGLU: h = silu(a) b, da = dh b silu'(a), db = dh silu(a).
// Squared ReLU: h = relu(b)^2, db = dh 2 relu(b) (a, da unused).
// silu'(a) = sigma(a) (1 + a (1 - sigma(a))).
template <typename TI, typename TO>
__global__ void act_backward_kernel(const TI *__restrict__ a, const TI *__restrict__ b, int ldab,
                                    const float *__restrict__ dh, int lddh, TO *__restrict__ h,
                                    int ldh, TO *__restrict__ da, TO *__restrict__ db, int ldd,
                                    int rows, int n, int relu2) {
  const int c = blockIdx.y * blockDim.x + threadIdx.x;  // rows on x: up to 2^31 - 1
  const int r = blockIdx.x;
  if (r >= rows || c >= n) return;
  const float bv = ld(b, static_cast<size_t>(r) * ldab + c);
  const float g = dh ? dh[static_cast<size_t>(r) * lddh + c] : 0.0f;
  if (relu2) {
    const float rb = fmaxf(bv, 0.0f);
    if (h) st(h, static_cast<size_t>(r) * ldh + c, rb * rb);
    if (db) st(db, static_cast<size_t>(r) * ldd + c, g * 2.0f * rb);
  } else {
    const float av = ld(a, static_cast<size_t>(r) * ldab + c);
    const float sg = 1.0f / (1.0f + expf(-av));
    const float sl = av * sg;
    if (h) st(h, static_cast<size_t>(r) * ldh + c, sl * bv);
    if (da) st(da, static_cast<size_t>(r) * ldd + c, g * bv * sg * (1.0f + av * (1.0f - sg)));
    if (db) st(db, static_cast<size_t>(r) * ldd + c, g * sl);
  }
}

// ------------------------------------------------------------ gate gradient
// Phase 1, one warp per (token, slot) pair: dg = du_t . O[pos(t,k)] (into
// ds for now) and the expert-output gradient row DO[pos(t,k)] = g_k du_t.
template <typename TO>
__global__ void slot_grad_kernel(const float *__restrict__ du, int lddu,
                                 const TO *__restrict__ O, int l, const int32_t *__restrict__ pos,
                                 const float *__restrict__ gates, int TK, int K,
                                 float *__restrict__ ds, TO *__restrict__ DO) {
  const int pair = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (pair >= TK) return;
  const int t = pair / K;
  const float *dur = du + static_cast<size_t>(t) * lddu;
  const int p = pos[pair];
  const float g = gates[pair];
  const TO *o = O + static_cast<size_t>(p) * l;
  TO *dor = DO + static_cast<size_t>(p) * l;
  float acc = 0.0f;
  for (int j = lane; j < l; j += 32) {
    const float dv = dur[j];
    acc = fmaf(dv, ld(o, j), acc);
    st(dor, j, g * dv);
  }
#pragma unroll
  for (int off = 16; off; off >>= 1) acc += __shfl_xor_sync(0xFFFFFFFFu, acc, off);
  if (lane == 0) ds[pair] = acc;
}

// Phase 2, one thread per token: ds_k = g_k (dg_k - sum_j g_j dg_j).
__global__ void gate_grad_kernel(const float *__restrict__ gates, int T, int K,
                                 float *__restrict__ ds) {
  const int t = blockIdx.x * blockDim.x + threadIdx.x;
  if (t >= T) return;
  float gamma = 0.0f;
  for (int k = 0; k < K; ++k) gamma = fmaf(gates[t * K + k], ds[t * K + k], gamma);
  for (int k = 0; k < K; ++k) ds[t * K + k] = gates[t * K + k] * (ds[t * K + k] - gamma);
}

// bf16 specialisation of phase 1: each lane moves 8 columns (16 bytes of O
// and DO) at a time; l % 8 == 0.
template <>
__global__ void slot_grad_kernel<__nv_bfloat16>(const float *__restrict__ du, int lddu,
                                                const __nv_bfloat16 *__restrict__ O, int l,
                                                const int32_t *__restrict__ pos,
                                                const float *__restrict__ gates, int TK, int K,
                                                float *__restrict__ ds,
                                                __nv_bfloat16 *__restrict__ DO) {
  const int pair = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (pair >= TK) return;
  const int t = pair / K;
  const float *dur = du + static_cast<size_t>(t) * lddu;
  const int p = pos[pair];
  const float g = gates[pair];
  const uint4 *o = reinterpret_cast<const uint4 *>(O + static_cast<size_t>(p) * l);
  uint4 *dor = reinterpret_cast<uint4 *>(DO + static_cast<size_t>(p) * l);
  float acc = 0.0f;
  for (int v = lane; v < l / 8; v += 32) {
    const uint4 ov = o[v];
    const float4 d0 = *reinterpret_cast<const float4 *>(dur + 8 * v);
    const float4 d1 = *reinterpret_cast<const float4 *>(dur + 8 * v + 4);
    const float dv[8] = {d0.x, d0.y, d0.z, d0.w, d1.x, d1.y, d1.z, d1.w};
    const uint32_t ow[4] = {ov.x, ov.y, ov.z, ov.w};
    uint32_t outw[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      acc = fmaf(dv[2 * i], __uint_as_float(ow[i] << 16), acc);
      acc = fmaf(dv[2 * i + 1], __uint_as_float(ow[i] & 0xFFFF0000u), acc);
      outw[i] = pack_bf16x2(g * dv[2 * i], g * dv[2 * i + 1]);
    }
    dor[v] = make_uint4(outw[0], outw[1], outw[2], outw[3]);
  }
#pragma unroll
  for (int off = 16; off; off >>= 1) acc += __shfl_xor_sync(0xFFFFFFFFu, acc, off);
  if (lane == 0) ds[pair] = acc;
}

// dz[t][:] = sum_k D[pos(t,k)][:] in slot order (fp32 accumulation).
template <typename TI, typename TO>
__global__ void gather_sum_kernel(const TI *__restrict__ D, int ldD, const int32_t *__restrict__ pos,
                                  int T, int K, int n, TO *__restrict__ out, int ldo) {
  const int t = blockIdx.x;
  const int c = blockIdx.y * blockDim.x + threadIdx.x;
  if (t >= T || c >= n) return;
  float acc = 0.0f;
  for (int k = 0; k < K; ++k) acc += ld(D, static_cast<size_t>(pos[t * K + k]) * ldD + c);
  st(out, static_cast<size_t>(t) * ldo + c, acc);
}

// dS[t][e]: the router-logit gradient, ds at the selected experts, 0 elsewhere.
template <typename TO>
__global__ void scatter_ds_kernel(const float *__restrict__ ds, const int32_t *__restrict__ ids,
                                  int T, int K, int N, TO *__restrict__ out, int ldo) {
  const int t = blockIdx.x;
  if (t >= T) return;
  for (int e = threadIdx.x; e < N; e += blockDim.x) st(out, static_cast<size_t>(t) * ldo + e, 0.0f);
  __syncthreads();
  for (int k = threadIdx.x; k < K; k += blockDim.x)
    st(out, static_cast<size_t>(t) * ldo + ids[t * K + k], ds[t * K + k]);
}

// db_r[e] = sum of ds over the (token, slot) pairs of expert e, in token
// order (the dispatch's perm lists them so).
__global__ void bias_grad_kernel(const float *__restrict__ ds, const int32_t *__restrict__ offsets,
                                 const int32_t *__restrict__ perm, int N, float *__restrict__ db) {
  const int e = blockIdx.x * blockDim.x + threadIdx.x;
  if (e >= N) return;
  float acc = 0.0f;
  for (int p = offsets[e]; p < offsets[e + 1]; ++p)
    if (perm[p] >= 0) acc += ds[perm[p]];  // padding rows of a padded order hold -1
  db[e] = acc;
}

// Zeroes the padding rows [ends[e], offsets[e + 1]) of expert e in up to four
// bf16 matrices (blockIdx.y selects one; null pointers are skipped).
__global__ void zero_pad_rows_kernel(const int32_t *__restrict__ offsets,
                                     const int32_t *__restrict__ ends, int N, PadRowsArgs a) {
  const int e = blockIdx.x, which = blockIdx.y;
  if (e >= N || !a.ptr[which]) return;
  const int r0 = ends[e], r1 = offsets[e + 1], vpr = a.cols[which] / 8;
  uint4 *base = reinterpret_cast<uint4 *>(a.ptr[which]);
  for (int i = threadIdx.x; i < (r1 - r0) * vpr; i += blockDim.x) {
    const int r = r0 + i / vpr, v = i % vpr;
    base[static_cast<size_t>(r) * vpr + v] = make_uint4(0, 0, 0, 0);
  }
}

// bf16 mode, gate/up pre-activations as the tensor-core GEMM writes them: in
// each 256-column block b, columns [0,128) hold the gate of hidden units
// 128b .. 128b+127 and [128,256) the matching up (squared ReLU: column c is
// the up of unit c).  dh [rows][n] (fp32 or bf16) -> dAB in the same
// interleaved layout: SwiGLU da = dh b silu'(a), db = dh silu(a); squared
// ReLU db = dh 2 relu(b).  Each thread takes 8 consecutive hidden units of a
// row (16-byte loads and stores; consecutive threads, consecutive units).
__device__ __forceinline__ void unpack_bf16x8(const uint4 q, float *v) {
  const uint32_t w[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    v[2 * i] = __uint_as_float(w[i] << 16);
    v[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
  }
}
__device__ __forceinline__ uint4 pack_bf16x8(const float *v) {
  uint4 q;
  q.x = pack_bf16x2(v[0], v[1]);
  q.y = pack_bf16x2(v[2], v[3]);
  q.z = pack_bf16x2(v[4], v[5]);
  q.w = pack_bf16x2(v[6], v[7]);
  return q;
}
template <typename TD>
__device__ __forceinline__ void load_dh8(const TD *p, float *v);
template <>
__device__ __forceinline__ void load_dh8<float>(const float *p, float *v) {
  const float4 a = reinterpret_cast<const float4 *>(p)[0], b = reinterpret_cast<const float4 *>(p)[1];
  v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w; v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
}
template <>
__device__ __forceinline__ void load_dh8<__nv_bfloat16>(const __nv_bfloat16 *p, float *v) {
  unpack_bf16x8(*reinterpret_cast<const uint4 *>(p), v);
}

template <typename TD>
__global__ void __launch_bounds__(256) act_backward_rows_kernel(
    const __nv_bfloat16 *__restrict__ AB, int ldab, const TD *__restrict__ dh, int lddh,
    __nv_bfloat16 *__restrict__ dAB, int lddab, int rows, int n, int relu2) {
  const int groups = n / 8;
  const long long total = static_cast<long long>(rows) * groups;
  for (long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; i < total;
       i += static_cast<long long>(gridDim.x) * blockDim.x) {
    const long long r = i / groups;
    const int c = static_cast<int>(i - r * groups) * 8;
    float g[8];
    load_dh8<TD>(dh + r * lddh + c, g);
    const __nv_bfloat16 *ab = AB + r * ldab;
    __nv_bfloat16 *dab = dAB + r * lddab;
    if (relu2) {
      float b[8], db[8];
      unpack_bf16x8(*reinterpret_cast<const uint4 *>(ab + c), b);
#pragma unroll
      for (int j = 0; j < 8; ++j) db[j] = g[j] * 2.0f * fmaxf(b[j], 0.0f);
      *reinterpret_cast<uint4 *>(dab + c) = pack_bf16x8(db);
    } else {
      const int ia = 256 * (c >> 7) + (c & 127), ib = ia + 128;
      float a[8], b[8], da[8], db[8];
      unpack_bf16x8(*reinterpret_cast<const uint4 *>(ab + ia), a);
      unpack_bf16x8(*reinterpret_cast<const uint4 *>(ab + ib), b);
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const float sg = 1.0f / (1.0f + __expf(-a[j]));
        da[j] = g[j] * b[j] * sg * (1.0f + a[j] * (1.0f - sg));
        db[j] = g[j] * a[j] * sg;
      }
      *reinterpret_cast<uint4 *>(dab + ia) = pack_bf16x8(da);
      *reinterpret_cast<uint4 *>(dab + ib) = pack_bf16x8(db);
    }
  }
}

// dst[c][col(r)] = src[r][c] for r < R, c < C, col(r) = r, or, with
// row_expert, r + shift[row_expert[r]] (each expert's rows start at a
// multiple of 64 in dst).  32 x 32 tiles through shared memory.
__global__ void transpose_bf16_kernel(const __nv_bfloat16 *__restrict__ src, int lds, int R, int C,
                                      const int32_t *__restrict__ row_expert,
                                      const int32_t *__restrict__ shift,
                                      __nv_bfloat16 *__restrict__ dst, long long ldd,
                                      long long src_batch, long long dst_batch) {
  __shared__ __nv_bfloat16 tile[32][33];
  src += blockIdx.z * src_batch;
  dst += blockIdx.z * dst_batch;
  const int r0 = blockIdx.y * 32, c0 = blockIdx.x * 32;
  const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;  // 32 x 8 threads
  for (int i = ty; i < 32; i += 8) {
    const int r = r0 + i, c = c0 + tx;
    tile[i][tx] = (r < R && c < C) ? src[static_cast<size_t>(r) * lds + c] : __float2bfloat16_rn(0.0f);
  }
  __syncthreads();
  const int r = r0 + tx;
  if (r >= R) return;
  const long long col = row_expert ? r + shift[row_expert[r]] : r;
  for (int i = ty; i < 32; i += 8) {
    const int c = c0 + i;
    if (c < C) dst[static_cast<long long>(c) * ldd + col] = tile[tx][i];
  }
}

}  // namespace

template <typename TD>
cudaError_t launch_act_backward_rows(const __nv_bfloat16 *AB, int ldab, const TD *dh, int lddh,
                                     __nv_bfloat16 *dAB, int lddab, int rows, int n, bool relu2,
                                     cudaStream_t s) {
  if (rows <= 0 || n <= 0) return cudaSuccess;
  if (n % 8 || ldab % 8 || lddh % 8 || lddab % 8) return cudaErrorInvalidValue;
  const long long total = static_cast<long long>(rows) * (n / 8);
  const int blocks = static_cast<int>(std::min<long long>((total + 255) / 256, 148LL * 16));
  act_backward_rows_kernel<TD><<<blocks, 256, 0, s>>>(AB, ldab, dh, lddh, dAB, lddab, rows, n,
                                                      relu2 ? 1 : 0);
  return cudaGetLastError();
}
template cudaError_t launch_act_backward_rows<float>(const __nv_bfloat16 *, int, const float *,
                                                     int, __nv_bfloat16 *, int, int, int, bool,
                                                     cudaStream_t);
template cudaError_t launch_act_backward_rows<__nv_bfloat16>(const __nv_bfloat16 *, int,
                                                             const __nv_bfloat16 *, int,
                                                             __nv_bfloat16 *, int, int, int, bool,
                                                             cudaStream_t);

cudaError_t launch_transpose_bf16(const __nv_bfloat16 *src, int lds, int R, int C,
                                  const int32_t *row_expert, const int32_t *shift,
                                  __nv_bfloat16 *dst, long long ldd, cudaStream_t s, int batch,
                                  long long src_batch, long long dst_batch) {
  if (R <= 0 || C <= 0 || batch <= 0) return cudaSuccess;
  dim3 grid((C + 31) / 32, (R + 31) / 32, batch);
  transpose_bf16_kernel<<<grid, 256, 0, s>>>(src, lds, R, C, row_expert, shift, dst, ldd,
                                             src_batch, dst_batch);
  return cudaGetLastError();
}

cudaError_t simt_gemm(const SimtGemm &g, int groups, cudaStream_t s) {
  if (g.M <= 0 || g.N <= 0 || groups <= 0) return cudaSuccess;
  dim3 grid((g.N + SBN - 1) / SBN, (g.M + SBM - 1) / SBM, groups);
  simt_gemm_kernel<<<grid, 256, 0, s>>>(g);
  return cudaGetLastError();
}

cudaError_t simt_rowexpert(const float *A, int lda, const float *W, long long sW_e, long long sW_r,
                           long long sW_k, const int32_t *row_expert, float *C, int ldc, int M,
                           int Ncols, int Kdim, bool accumulate, cudaStream_t s) {
  if (M <= 0 || Ncols <= 0) return cudaSuccess;
  dim3 grid((M + 3) / 4, (Ncols + 63) / 64);
  simt_rowexpert_kernel<<<grid, 256, 0, s>>>(A, lda, W, sW_e, sW_r, sW_k, row_expert, C, ldc, M,
                                             Ncols, Kdim, accumulate ? 1 : 0);
  return cudaGetLastError();
}

template <typename TI, typename TO>
cudaError_t launch_act_backward(const TI *a, const TI *b, int ldab, const float *dh, int lddh,
                                TO *h, int ldh, TO *da, TO *db, int ldd, int rows, int n,
                                bool relu2, cudaStream_t s) {
  if (rows <= 0 || n <= 0) return cudaSuccess;
  dim3 grid(rows, (n + 255) / 256);
  act_backward_kernel<TI, TO><<<grid, 256, 0, s>>>(a, b, ldab, dh, lddh, h, ldh, da, db, ldd, rows,
                                                   n, relu2 ? 1 : 0);
  return cudaGetLastError();
}
template cudaError_t launch_act_backward<float, float>(const float *, const float *, int,
                                                       const float *, int, float *, int, float *,
                                                       float *, int, int, int, bool, cudaStream_t);

template <typename TO>
cudaError_t launch_slot_grad(const float *du, int lddu, const TO *O, int l, const int32_t *pos,
                             const float *gates, int T, int K, float *ds, TO *DO, cudaStream_t s) {
  if (T <= 0) return cudaSuccess;
  const int TK = T * K;
  slot_grad_kernel<TO><<<(TK + 7) / 8, 256, 0, s>>>(du, lddu, O, l, pos, gates, TK, K, ds, DO);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  gate_grad_kernel<<<(T + 255) / 256, 256, 0, s>>>(gates, T, K, ds);
  return cudaGetLastError();
}

template cudaError_t launch_slot_grad<float>(const float *, int, const float *, int,
                                             const int32_t *, const float *, int, int, float *,
                                             float *, cudaStream_t);
template cudaError_t launch_slot_grad<__nv_bfloat16>(const float *, int, const __nv_bfloat16 *, int,
                                                     const int32_t *, const float *, int, int,
                                                     float *, __nv_bfloat16 *, cudaStream_t);

template <typename TI, typename TO>
cudaError_t launch_gather_sum(const TI *D, int ldD, const int32_t *pos, int T, int K, int n, TO *out,
                              int ldo, cudaStream_t s) {
  if (T <= 0 || n <= 0) return cudaSuccess;
  dim3 grid(T, (n + 127) / 128);
  gather_sum_kernel<TI, TO><<<grid, 128, 0, s>>>(D, ldD, pos, T, K, n, out, ldo);
  return cudaGetLastError();
}
template cudaError_t launch_gather_sum<float, float>(const float *, int, const int32_t *, int, int,
                                                     int, float *, int, cudaStream_t);
template cudaError_t launch_gather_sum<float, __nv_bfloat16>(const float *, int, const int32_t *,
                                                             int, int, int, __nv_bfloat16 *, int,
                                                             cudaStream_t);

template <typename TO>
cudaError_t launch_scatter_ds(const float *ds, const int32_t *ids, int T, int K, int N, TO *out,
                              int ldo, cudaStream_t s) {
  if (T <= 0) return cudaSuccess;
  scatter_ds_kernel<TO><<<T, 128, 0, s>>>(ds, ids, T, K, N, out, ldo);
  return cudaGetLastError();
}
template cudaError_t launch_scatter_ds<float>(const float *, const int32_t *, int, int, int, float *,
                                              int, cudaStream_t);
template cudaError_t launch_scatter_ds<__nv_bfloat16>(const float *, const int32_t *, int, int, int,
                                                      __nv_bfloat16 *, int, cudaStream_t);

cudaError_t launch_bias_grad(const float *ds, const int32_t *offsets, const int32_t *perm, int N,
                             float *db, cudaStream_t s) {
  if (N <= 0) return cudaSuccess;
  bias_grad_kernel<<<(N + 127) / 128, 128, 0, s>>>(ds, offsets, perm, N, db);
  return cudaGetLastError();
}

cudaError_t launch_zero_pad_rows(const int32_t *offsets, const int32_t *ends, int N,
                                 const PadRowsArgs &a, cudaStream_t s) {
  if (N <= 0) return cudaSuccess;
  for (int i = 0; i < 4; ++i)
    if (a.ptr[i] && a.cols[i] % 8) return cudaErrorInvalidValue;
  zero_pad_rows_kernel<<<dim3(N, 4), 256, 0, s>>>(offsets, ends, N, a);
  return cudaGetLastError();
}

}  // namespace lmoe

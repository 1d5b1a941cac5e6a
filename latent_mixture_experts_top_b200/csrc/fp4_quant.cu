// fp4_quant.cu -- NVFP4 routed experts: the weights (once, at load) and the
// activation rows the expert GEMMs multiply (every forward).
//
// "LatentMoE Explained" says the shipped models were pretrained in NVFP4 and
// gives no recipe; NVFP4 is NVIDIA's published 4-bit format: E2M1 elements
// (magnitudes 0, 0.5, 1, 1.5, 2, 3, 4, 6) and one E4M3 scale per 16
// consecutive elements of a row.  The second-level scale is taken per row
// here: s_r = 2^e_r, the smallest power of two with max |row| <= 6 * 448 s_r.
// Block j of the row: b_j = E4M3(amax_j / (6 s_r)); each element's code is
// E2M1(x * rcp_j) with rcp_j = 1 / (b_j s_r) rounded once (the element scaled
// by the reciprocal of its decoded block scale), both roundings to nearest
// even with saturation; the division, the reciprocal and the product are IEEE
// single precision (they decide codes).  A block with b_j = 0 has all-zero
// codes.  The GEMM's tensor cores apply b_j (kind::mxf4nvf4),
// its epilogue s_r.
//
// Layouts (the GEMM's, see TcParams):
//  - weight codes: per group (expert), 256-row tile n and 256-element K-block
//    kb, one 256 x 128-byte block, element 2i of a row in the low nibble of
//    byte i; padding rows and columns zero;
//  - weight block scales: per (group, n, kb) 4 KB: for each 128-row half rb
//    and each of the K-block's four 64-element slices k, a 512-byte atom in
//    which row r0 + 32 r1 (r0 < 32, r1 < 4) holds its four scales at bytes
//    16 r0 + 4 r1 .. + 3; scales past the matrix are zero;
//  - activation codes: row-major [rows][cols / 2];
//  - activation block scales: per M-tile of the tile table and K-block 2 KB,
//    the four slices' atoms of the tile's 128 rows, as above.
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp8.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "common.cuh"
#include "kernels.h"

namespace lmoe {
namespace {

constexpr int kKb = 256;      // elements per K-block
constexpr int kAtom = 512;    // bytes of one 128-row x 4-scale atom

// Exponent of the row scale: the smallest e with amax <= 2688 2^e (2688 =
// 1.3125 2^11 = 6 * 448); 0 for a row of zeros.  amax = m 2^ea with m in
// [1, 2) (frexp is exact).
__device__ __forceinline__ int nvfp4_row_exp(float amax) {
  if (!(amax > 0.0f)) return 0;
  int ea;
  const float m = 2.0f * frexpf(amax, &ea);
  ea -= 1;
  return m <= 1.3125f ? ea - 11 : ea - 10;
}

// Four pairs -> four bytes of E2M1 codes (first of each pair in the low
// nibble), round to nearest even, saturating at 6.
__device__ __forceinline__ uint32_t e2m1x8(const float *y) {
  uint32_t out;
  asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b0, %2, %1;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b1, %4, %3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b2, %6, %5;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b3, %8, %7;\n\t"
      "mov.b32 %0, {b0, b1, b2, b3};\n\t}"
      : "=r"(out)
      : "f"(y[0]), "f"(y[1]), "f"(y[2]), "f"(y[3]), "f"(y[4]), "f"(y[5]), "f"(y[6]), "f"(y[7]));
  return out;
}

// Sixteen bf16 values (two 16-byte vectors) of a row with scale exponent e:
// the block scale's E4M3 code (returned) and the sixteen E2M1 codes (codes).
__device__ __forceinline__ uint8_t nvfp4_block(const uint4 lo, const uint4 hi, int e,
                                               uint2 *codes) {
  float v[16];
  const uint32_t w[8] = {lo.x, lo.y, lo.z, lo.w, hi.x, hi.y, hi.z, hi.w};
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    v[2 * i] = __uint_as_float(w[i] << 16);
    v[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
  }
  float am = 0.0f;
#pragma unroll
  for (int i = 0; i < 16; ++i) am = fmaxf(am, fabsf(v[i]));
  const float t = __fdiv_rn(am, ldexpf(6.0f, e));
  const __nv_fp8_storage_t bc = __nv_cvt_float_to_fp8(t, __NV_SATFINITE, __NV_E4M3);
  const float b = __half2float(__half(__nv_cvt_fp8_to_halfraw(bc, __NV_E4M3)));
  if (b == 0.0f) {
    *codes = make_uint2(0u, 0u);
    return 0;
  }
  const float rcp = __frcp_rn(ldexpf(b, e));  // b 2^e is exact: 4 significant bits
  float y[16];
#pragma unroll
  for (int i = 0; i < 16; ++i) y[i] = __fmul_rn(v[i], rcp);
  *codes = make_uint2(e2m1x8(y), e2m1x8(y + 8));
  return static_cast<uint8_t>(bc);
}

// Byte offset of row i (< 128) of an atom for the scale of 16-block q (< 4)
// of its 64-element slice.
__device__ __forceinline__ int atom_byte(int i, int q) { return 16 * (i & 31) + 4 * (i >> 5) + q; }

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

// One warp per weight row of src [groups][rows_per_group][cols] bf16.
__global__ void __launch_bounds__(256) quantize_w_nvfp4_kernel(
    const __nv_bfloat16 *__restrict__ src, long long n_rows, int rows_per_group, int cols, int nt,
    float *__restrict__ scales, uint8_t *__restrict__ codes, uint8_t *__restrict__ sf) {
  const long long row = static_cast<long long>(blockIdx.x) * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= n_rows) return;
  const uint4 *w = reinterpret_cast<const uint4 *>(src + row * cols);
  const int e = nvfp4_row_exp(row_amax(w, cols / 8, lane));
  if (lane == 0) scales[row] = ldexpf(1.0f, e);
  const long long g = row / rows_per_group;
  const int r = static_cast<int>(row % rows_per_group);
  const int n = r >> 8, rr = r & 255, nkb = (cols + kKb - 1) / kKb;
  for (int blk = lane; blk < cols / 16; blk += 32) {
    uint2 c;
    const uint8_t b = nvfp4_block(w[2 * blk], w[2 * blk + 1], e, &c);
    const int kb = blk >> 4, k = (blk >> 2) & 3, q = blk & 3;
    const long long tile = (g * nt + n) * nkb + kb;
    *reinterpret_cast<uint2 *>(codes + (tile * 256 + rr) * 128 + (blk & 15) * 8) = c;
    sf[tile * (2 * 4 * kAtom) + ((rr >> 7) * 4 + k) * kAtom + atom_byte(rr & 127, q)] = b;
  }
}

// Block (mt, j) takes rows 8j .. 8j + 7 of M-tile mt of the tile table, one
// warp per row (every row of the layer in flight at once): the row
// p = row0 + i of the tile reads src row (gather ? gather[p] / K : p) and
// writes codes row p, scales[p] and the tile's block-scale atoms (scales of
// 16-blocks past cols as zero: the ragged last K-block's zero codes then add
// nothing).
__global__ void __launch_bounds__(256) quantize_act_nvfp4_kernel(
    const __nv_bfloat16 *__restrict__ src, const int32_t *__restrict__ gather, int K,
    const TileEntry *__restrict__ tiles, const int32_t *__restrict__ n_tiles, int cols,
    uint8_t *__restrict__ codes, float *__restrict__ scales, uint8_t *__restrict__ sf) {
  griddep_wait();
  const int mt = blockIdx.x;
  if (mt >= *n_tiles) return;
  const TileEntry te = tiles[mt];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nkb = (cols + kKb - 1) / kKb, nblk = cols / 16;
  uint8_t *tsf = sf + static_cast<size_t>(mt) * nkb * 4 * kAtom;
  // Rows past the expert's end are left as they are: an accumulator row
  // depends only on its own A row and scales, and those rows are never stored.
  const int i = blockIdx.y * 8 + warp;
  if (i < min(128, te.row_end - te.row0)) {
    const int p = te.row0 + i;
    const int srow = gather ? gather[p] / K : p;
    const uint4 *w = reinterpret_cast<const uint4 *>(src + static_cast<size_t>(srow) * cols);
    const int e = nvfp4_row_exp(row_amax(w, cols / 8, lane));
    if (lane == 0) scales[p] = ldexpf(1.0f, e);
    uint2 *crow = reinterpret_cast<uint2 *>(codes + static_cast<size_t>(p) * (cols / 2));
    for (int blk = lane; blk < nkb * 16; blk += 32) {
      uint8_t b = 0;
      if (blk < nblk) {
        uint2 c;
        b = nvfp4_block(w[2 * blk], w[2 * blk + 1], e, &c);
        crow[blk] = c;
      }
      tsf[((blk >> 4) * 4 + ((blk >> 2) & 3)) * kAtom + atom_byte(i, blk & 3)] = b;
    }
  }
}

}  // namespace

size_t nvfp4_weight_code_bytes(int groups, int rows_per_group, int cols) {
  const size_t nt = (rows_per_group + 255) / 256, nkb = (cols + kKb - 1) / kKb;
  return static_cast<size_t>(groups) * nt * nkb * 256 * 128;
}

size_t nvfp4_weight_sf_bytes(int groups, int rows_per_group, int cols) {
  const size_t nt = (rows_per_group + 255) / 256, nkb = (cols + kKb - 1) / kKb;
  return static_cast<size_t>(groups) * nt * nkb * 2 * 4 * kAtom;
}

size_t nvfp4_act_sf_bytes(int max_tiles, int cols) {
  return static_cast<size_t>(max_tiles) * ((cols + kKb - 1) / kKb) * 4 * kAtom;
}

cudaError_t launch_quantize_nvfp4_tiles(const __nv_bfloat16 *src, int groups, int rows_per_group,
                                        int cols, float *scales, uint8_t *codes, uint8_t *sf,
                                        cudaStream_t s) {
  if (cols % 32 || cols <= 0 || groups <= 0 || rows_per_group <= 0) return cudaErrorInvalidValue;
  const int nt = (rows_per_group + 255) / 256;
  cudaError_t e = cudaMemsetAsync(codes, 0, nvfp4_weight_code_bytes(groups, rows_per_group, cols), s);
  if (e == cudaSuccess)
    e = cudaMemsetAsync(sf, 0, nvfp4_weight_sf_bytes(groups, rows_per_group, cols), s);
  if (e != cudaSuccess) return e;
  const long long n_rows = static_cast<long long>(groups) * rows_per_group;
  quantize_w_nvfp4_kernel<<<static_cast<unsigned>((n_rows + 7) / 8), 256, 0, s>>>(
      src, n_rows, rows_per_group, cols, nt, scales, codes, sf);
  return cudaGetLastError();
}

cudaError_t launch_quantize_act_nvfp4(const __nv_bfloat16 *src, const int32_t *gather, int K,
                                      const TileEntry *tiles, const int32_t *n_tiles,
                                      int max_tiles, int cols, uint8_t *codes, float *scales,
                                      uint8_t *sf, cudaStream_t s, bool pdl) {
  if (max_tiles <= 0) return cudaSuccess;
  if (cols % 32 || cols <= 0 || (gather && K <= 0)) return cudaErrorInvalidValue;
  const cudaError_t e = launch_ex(quantize_act_nvfp4_kernel, dim3(max_tiles, 16), dim3(256), 0, s, pdl,
                                  src, gather, K, tiles, n_tiles, cols, codes, scales, sf);
  return e != cudaSuccess ? e : cudaGetLastError();
}

}  // namespace lmoe

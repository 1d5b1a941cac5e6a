// tc_gemm.cu -- persistent bf16 tcgen05 GEMM for the dense contractions of
// the LatentMoE layer forward, with four fused epilogues.
//
//   TC_X_FUSED     x [T][d] times the stacked matrix [W_r ; W_down ; shared
//                  gate/up] -> fp32 router logits, bf16 z, and the shared
//                  experts' SwiGLU hidden (written next to u, so that the
//                  last GEMM adds the shared output for free).
//   TC_EXPERT_GU   grouped: permuted z rows of expert e times its gate/up
//                  rows (interleaved in blocks of 128) -> SwiGLU -> H (bf16);
//                  for squared-ReLU experts its up rows -> relu(.)^2 -> H.
//   TC_EXPERT_DOWN grouped: H times W_o[e] -> expert output O (bf16).
//   TC_OUT         [u | shared hidden] times [W_up | S_o] -> y (bf16).
//
// Sources of the maths: "LatentMoE Explained", Figure 3 (router reads the
// full-width x), Figure 6 (W_down, W_up), Figure 8 (the routed path inside
// the projections, the shared path at width d), Figure 9 (latent expert
// l -> m -> l); SwiGLU expert per the paragraph after Figure 1.
//
// B operands are K-block tiled in memory (one contiguous 256 x 64 block per
// N-tile and K-block), so each B load is one contiguous 32 KB range.
//
// Structure (one CTA per SM, 320 threads):
//   warp 0      TMA producer: 128x64 A and 256x64 B bf16 tiles, 128-byte
//               swizzle, into a 4-stage shared-memory ring of this CTA.
//   warp 1      TMEM owner and MMA issuer: one thread issues
//               tcgen05.mma.cta_group::1.kind::f16 (M=128, N=256, K=16) into
//               one of two 256-column fp32 accumulators in TMEM, and
//               tcgen05.commit frees ring stages / publishes accumulators.
//   warps 2-9   epilogue: two warps per TMEM lane quarter, each taking half
//               of the tile's columns: tcgen05.ld 32 lanes x 32 columns,
//               fused epilogue, then (forward bf16 outputs) a TMA store of
//               each 32 x 32 block staged in shared memory, or 16-byte
//               global stores; overlaps the next tile's MMAs.
// Every mbarrier wait is bounded (kWaitLimitNs); on expiry the CTA records a
// status, stops its roles, lets in-flight copies and MMAs land, frees TMEM and
// returns.
//
// tc_pair_kernel (further down) runs the same forward modes on CTA pairs
// (tcgen05.mma.cta_group::2, 256 x 256 tiles) with the same epilogue.
//
// kF8 (E4M3 routed experts): the expert GEMMs take both operands in E4M3
// (tcgen05.mma kind::f8f6f4, fp32 accumulation): a K-block is 128 elements,
// so every row of a staged tile is still 128 bytes and the shared-memory
// layout, descriptors and pipeline are those of the bf16 tiles; the epilogue
// multiplies the accumulator by the A row's scale and the weight row's scale.
//
// kQ = kNvf4 (NVFP4 routed experts): both operands are packed E2M1 codes with
// one E4M3 scale per 16 elements of a row (tcgen05.mma kind::mxf4nvf4, block
// size 16): a K-block is 256 elements, again 128 bytes per staged row.  Each
// stage also carries the two operands' scale blocks (2 KB for the 128 A rows,
// 4 KB for the 256 B rows), laid out as the MMA reads them from TMEM; the
// MMA warp copies them into TMEM (tcgen05.cp) ahead of the stage's four
// MMAs.  The per-row second-level scales are applied in the epilogue, as for
// E4M3.  The scale blocks take 48 TMEM columns, so this variant keeps one
// accumulator (256 columns) instead of two.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>
#include <string.h>

#include "common.cuh"
#include "kernels.h"
#include "ptx_sm100.cuh"

namespace lmoe {
namespace {

constexpr int TM = 128, TN = 256, TKB = 64;   // tile M, N, K-block
constexpr int A_BYTES = TM * TKB * 2;         // 16 KB
constexpr int B_BYTES = TN * TKB * 2;         // 32 KB (16-bit B tile)
constexpr int TMEM_COLS = 2 * TN;             // two accumulators
constexpr int NUM_EPI_WARPS = 8;              // two per TMEM lane quarter
constexpr uint32_t IDESC = ptx::idesc_bf16_f32(TM, TN);
constexpr uint32_t IDESC8 = ptx::idesc_e4m3_f32(TM, TN);
constexpr uint32_t IDESC4 = ptx::idesc_nvf4(TM, TN);
constexpr uint32_t IDESC_MN = ptx::idesc_bf16_f32_mn(TM, TN);  // TC_WGRAD: MN-major A and B
constexpr int MN_BOX_BYTES = 64 * 64 * 2;  // one {64, 64} bf16 box of an MN-major tile
// operand formats of the single-CTA kernel
constexpr int kBf16 = 0, kE4m3 = 1, kNvf4 = 2;
// NVFP4 scale blocks of one stage: A 128 rows x 16 scales, B 256 rows x 16,
// as 512-byte atoms (32 rows x 4 scales of one MMA; row r0 + 32 r1 at byte
// 16 r0 + 4 r1); TMEM columns of the A atoms (4 per MMA) and the B atoms (8)
constexpr int SFA_BYTES = 2048, SFB_BYTES = 4096;
constexpr int SFA_COL = 256, SFB_COL = 288;

// Pipeline shape: a STAGES-deep ring of (A, B) tiles filled by TMA and read
// by the MMA.  Both element types stage 128-byte K-block rows: 64 bf16, or
// (kF8) 128 E4M3 codes.
constexpr int TKB8 = 128;  // K-block of the E4M3 GEMM (elements = bytes)
constexpr int TKB4 = 256;  // K-block of the NVFP4 GEMM (two elements per byte)
template <int kQ>
struct Cfg {
  static constexpr int STAGES = kQ == kNvf4 ? 3 : 4;
  static constexpr int KB = kQ == kNvf4 ? TKB4 : kQ == kE4m3 ? TKB8 : TKB;  // elements per K-block
  static constexpr int EPI_WARPS = NUM_EPI_WARPS;
  static constexpr int NUM_THREADS = 64 + 32 * EPI_WARPS;
  static constexpr int SF_BYTES = kQ == kNvf4 ? SFA_BYTES + SFB_BYTES : 0;  // per stage
  static constexpr int RING_BYTES = STAGES * (A_BYTES + B_BYTES + SF_BYTES);
  static constexpr int ACC_BUFS = kQ == kNvf4 ? 1 : 2;  // accumulators in TMEM
};

constexpr int MAX_STAGES = 8;
struct __align__(8) SmemCtl {
  uint64_t full[MAX_STAGES];
  uint64_t empty[MAX_STAGES];
  uint64_t acc_full[2];
  uint64_t acc_empty[2];
  uint64_t drain;
  uint32_t tmem_base;
  int abort;
};
// TMA-store epilogue (forward bf16 outputs): each epilogue warp owns two
// staging buffers of one 32 x 32 bf16 block; they follow the control block.
constexpr int OUT_BOX = 32;
constexpr int OUT_BOX_BYTES = OUT_BOX * OUT_BOX * 2;                // 2 KB
constexpr int CTL_BYTES = 1024;                                     // SmemCtl, padded
constexpr int STAGING_BYTES = NUM_EPI_WARPS * 2 * OUT_BOX_BYTES;    // 32 KB
static_assert(sizeof(SmemCtl) <= CTL_BYTES, "control block");
template <int kQ>
constexpr size_t smem_bytes(bool staging) {
  return 1024 /*align slack*/ + Cfg<kQ>::RING_BYTES +
         (staging ? CTL_BYTES + STAGING_BYTES : sizeof(SmemCtl));
}
static_assert(smem_bytes<kBf16>(true) <= 232448, "shared memory per CTA");
static_assert(smem_bytes<kE4m3>(true) <= 232448, "shared memory per CTA");
static_assert(smem_bytes<kNvf4>(true) <= 232448, "shared memory per CTA");

struct Tile {
  int a_row, b_row, n_tile, row_hi;
  int mt;     // grouped modes: the M-tile's index in the tile table
  int k0;     // first K index (TC_WGRAD: the first token row of A and B)
  int nkb;    // K-blocks of this tile
  int group;  // TC_WGRAD group
  int expert; // grouped modes: the expert of the tile
};

__device__ __forceinline__ Tile decode_tile(const TcParams &p, int t, int m_tiles,
                                           int kb_elems = TKB) {
  Tile tl;
  tl.k0 = 0;
  // a ragged last K-block (NVFP4 only) reads zero codes past Kdim
  const int nkb_all = (p.Kdim + kb_elems - 1) / kb_elems;
  tl.nkb = nkb_all;
  tl.mt = 0;
  tl.group = 0;
  tl.expert = 0;
  if (p.mode == TC_WGRAD) {
    const int per = m_tiles * p.n_tiles_n;
    const int g = t / per, r = t % per;
    const int m = r % m_tiles, n = r / m_tiles;  // consecutive CTAs share B
    tl.a_row = m * TM;
    tl.b_row = n * TN;
    tl.n_tile = n;
    tl.row_hi = p.M;
    tl.group = g;
    if (p.k_start) {  // group g's token rows (k_len null: up to the next group's start)
      tl.k0 = p.k_start[g];
      tl.nkb = (p.k_len ? p.k_len[g] : p.k_start[g + 1] - p.k_start[g]) / kb_elems;
    }
  } else if (p.mode == TC_X_FUSED || p.mode == TC_OUT) {
    // consecutive CTAs share B; with k_split, item r of an M-tile is slice
    // r % k_split of N-tile r / k_split (its K-blocks from k0 on; the slice
    // index in group)
    const int ks = p.k_split > 1 ? p.k_split : 1;
    const int m = t % m_tiles, r = t / m_tiles;
    const int split = r % ks, n = p.n_tile_base + r / ks;
    const int per = (nkb_all + ks - 1) / ks;
    tl.a_row = m * TM;
    tl.b_row = (n * nkb_all + split * per) * TN;  // first K-block tile of the slice
    tl.k0 = split * per * kb_elems;
    tl.nkb = min(per, nkb_all - split * per);
    tl.group = split;
    tl.n_tile = n;
    tl.row_hi = p.M;
  } else {
    const int mt = t / p.n_tiles_n, n = t % p.n_tiles_n;  // consecutive CTAs share A
    const TileEntry te = p.tiles[mt];
    tl.expert = te.expert;
    tl.mt = mt;
    tl.a_row = te.row0;
    tl.b_row = (te.expert * p.n_tiles_n + n) * nkb_all * TN;
    tl.n_tile = n;
    tl.row_hi = te.row_end;
  }
  return tl;
}

__device__ __forceinline__ void record_failure(const TcParams &p, SmemCtl *ctl, int code) {
  ctl->abort = 1;
  if (p.status) atomicCAS(p.status, 0, code);
}

// Bounded wait used only on the abort path (no abort check, shorter limit).
__device__ __forceinline__ bool drain_wait(uint64_t *bar, uint32_t parity) {
  const unsigned long long t0 = globaltimer_ns();
  while (!ptx::mbar_try_wait(bar, parity)) {
    if (globaltimer_ns() - t0 > kWaitLimitNs / 4) return false;
  }
  return true;
}

// ---- epilogue helpers: one thread = one output row, 32 fp32 columns at a time
__device__ __forceinline__ void store_bf16x32(__nv_bfloat16 *dst, const float *v) {
  uint4 *d = reinterpret_cast<uint4 *>(dst);
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    uint4 w;
    w.x = pack_bf16x2(v[8 * q + 0], v[8 * q + 1]);
    w.y = pack_bf16x2(v[8 * q + 2], v[8 * q + 3]);
    w.z = pack_bf16x2(v[8 * q + 4], v[8 * q + 5]);
    w.w = pack_bf16x2(v[8 * q + 6], v[8 * q + 7]);
    d[q] = w;
  }
}
__device__ __forceinline__ void store_f32x32(float *dst, const float *v) {
  float4 *d = reinterpret_cast<float4 *>(dst);
#pragma unroll
  for (int q = 0; q < 8; ++q) d[q] = make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
}

// Row-coalesced stores through the warp's staging buffer (backward
// epilogues).  Lane i holds 32 values of row i and that row's destination
// (null: not stored); the values go through shared memory so that each store
// instruction writes whole row segments (128 bytes of fp32 or 64 bytes of
// bf16 per row) instead of 16 bytes of 32 different rows.  All 32 lanes call
// these together; destinations are 16-byte aligned.
__device__ __forceinline__ void store_rows_f32x32(uint8_t *stage, const float *v, float *dst) {
  const int lane = threadIdx.x & 31;
  float4 *st = reinterpret_cast<float4 *>(stage);  // [32][8], chunk k of row r at k ^ (r & 7)
#pragma unroll
  for (int k = 0; k < 8; ++k)
    st[lane * 8 + (k ^ (lane & 7))] = make_float4(v[4 * k], v[4 * k + 1], v[4 * k + 2], v[4 * k + 3]);
  __syncwarp();
  const int ch = lane & 7;
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    const int rr = 4 * j + (lane >> 3);
    float *d = reinterpret_cast<float *>(
        __shfl_sync(0xFFFFFFFFu, reinterpret_cast<unsigned long long>(dst), rr));
    const float4 val = st[rr * 8 + (ch ^ (rr & 7))];
    if (d) reinterpret_cast<float4 *>(d)[ch] = val;
  }
  __syncwarp();
}
__device__ __forceinline__ void store_rows_bf16x32(uint8_t *stage, const float *v,
                                                   __nv_bfloat16 *dst) {
  const int lane = threadIdx.x & 31;
  uint4 *st = reinterpret_cast<uint4 *>(stage);  // [32][4], chunk k of row r at k ^ ((r >> 1) & 3)
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    uint4 w;
    w.x = pack_bf16x2(v[8 * k + 0], v[8 * k + 1]);
    w.y = pack_bf16x2(v[8 * k + 2], v[8 * k + 3]);
    w.z = pack_bf16x2(v[8 * k + 4], v[8 * k + 5]);
    w.w = pack_bf16x2(v[8 * k + 6], v[8 * k + 7]);
    st[lane * 4 + (k ^ ((lane >> 1) & 3))] = w;
  }
  __syncwarp();
  const int ch = lane & 3;
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const int rr = 8 * j + (lane >> 2);
    __nv_bfloat16 *d = reinterpret_cast<__nv_bfloat16 *>(
        __shfl_sync(0xFFFFFFFFu, reinterpret_cast<unsigned long long>(dst), rr));
    const uint4 val = st[rr * 4 + (ch ^ ((rr >> 1) & 3))];
    if (d) reinterpret_cast<uint4 *>(d)[ch] = val;
  }
  __syncwarp();
}

// Per-warp state of the TMA-store epilogue.  map == null: the warp stores
// its rows directly (one 16-byte store per lane and 8 columns).
struct OutSink {
  const CUtensorMap *map;
  uint8_t *buf;  // the warp's two staging buffers
  int x0;        // output column of the epilogue's column 0
  int y;         // output row of lane 0
  int issued;    // blocks stored so far (selects the buffer)
};

// Row `lane` of the warp's 32-row block, columns x .. x+31: the 32 values go,
// as bf16, into a staging buffer in the 64-byte-swizzled layout of the output
// map (16-byte chunk j of row r at chunk position j ^ ((r >> 1) & 3), which
// also keeps each 8-lane phase of the writes on distinct banks), and lane 0
// stores the block with one TMA store.  A buffer is refilled only once the
// store issued two blocks earlier has finished reading it.  All 32 lanes call
// this together.
__device__ __forceinline__ void sink_store(OutSink &o, const float *v, int x) {
  const int lane = threadIdx.x & 31;
  uint8_t *b = o.buf + (o.issued & 1) * OUT_BOX_BYTES;
  if (o.issued >= 2) {
    if (lane == 0) ptx::bulk_wait_group_read<1>();
    __syncwarp();
  }
  const int sw = (lane >> 1) & 3;
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    uint4 w;
    w.x = pack_bf16x2(v[8 * j + 0], v[8 * j + 1]);
    w.y = pack_bf16x2(v[8 * j + 2], v[8 * j + 3]);
    w.z = pack_bf16x2(v[8 * j + 4], v[8 * j + 5]);
    w.w = pack_bf16x2(v[8 * j + 6], v[8 * j + 7]);
    *reinterpret_cast<uint4 *>(b + lane * 64 + ((j ^ sw) << 4)) = w;
  }
  ptx::fence_proxy_async_smem();
  __syncwarp();
  if (lane == 0) {
    ptx::tma_store_2d(o.map, b, o.x0 + x, o.y);
    ptx::bulk_commit_group();
  }
  ++o.issued;
}

// 256 accumulator columns -> bf16 (or f32) row segment, chunks past n_cols skipped.
template <bool F32OUT, typename OutT>
__device__ __forceinline__ void epi_plain(uint32_t taddr, bool valid, OutT *row_dst, int col0,
                                          int n_cols, int half, OutSink *sink = nullptr) {
#pragma unroll 1
  for (int c = half * (TN / 64); c < (half + 1) * (TN / 64); ++c) {
    uint32_t r[32];
    ptx::tmem_ld_32x32b_x32(taddr + c * 32, r);
    ptx::tmem_ld_wait();
    float v[32];
#pragma unroll
    for (int j = 0; j < 32; ++j) v[j] = __uint_as_float(r[j]);
    const int col = col0 + c * 32;
    if constexpr (!F32OUT) {
      if (sink && sink->map) {
        if (col < n_cols) sink_store(*sink, v, col);
        continue;
      }
    }
    if (valid && col < n_cols) {
      if constexpr (F32OUT) store_f32x32(reinterpret_cast<float *>(row_dst) + col, v);
      else store_bf16x32(reinterpret_cast<__nv_bfloat16 *>(row_dst) + col, v);
    }
  }
}

// Squared-ReLU hidden: relu(acc)^2 -> bf16 columns col0 + ..., masked at n_cols.
__device__ __forceinline__ void epi_relu2(uint32_t taddr, bool valid, __nv_bfloat16 *row_dst,
                                          int col0, int n_cols, int half,
                                          OutSink *sink = nullptr) {
#pragma unroll 1
  for (int c = half * (TN / 64); c < (half + 1) * (TN / 64); ++c) {
    uint32_t r[32];
    ptx::tmem_ld_32x32b_x32(taddr + c * 32, r);
    ptx::tmem_ld_wait();
    float h[32];
#pragma unroll
    for (int j = 0; j < 32; ++j) {
      const float a = fmaxf(__uint_as_float(r[j]), 0.0f);
      h[j] = a * a;
    }
    const int col = col0 + c * 32;
    if (sink && sink->map) {
      if (col < n_cols) sink_store(*sink, h, col);
    } else if (valid && col < n_cols) {
      store_bf16x32(row_dst + col, h);
    }
  }
}

// Weight-gradient tile row `row` (an A row), output columns col0 .. col0+255
// (B rows): fp32 into the caller's gradient arrays; zeros when the tile had
// no K-blocks (an expert no token chose).
__device__ __forceinline__ float *wgrad_row_dst(const TcParams &p, int row, int group,
                                                int *ld_or_skip) {
  const int d = p.wg_d, l = p.wg_l, m = p.wg_m;
  switch (p.wg_kind) {
    case WG_X: {
      *ld_or_skip = d;
      if (row < p.wg_n) return p.g_router + static_cast<size_t>(row) * d;
      if (row >= p.wg_npad && row < p.wg_npad + l)
        return p.g_down + static_cast<size_t>(row - p.wg_npad) * d;
      const int r = row - p.wg_npad - p.wg_lpad;
      const int nsms = p.wg_ns * p.wg_ms;
      if (r < 0) return nullptr;
      if (p.relu2) return r < nsms ? p.g_sup + static_cast<size_t>(r) * d : nullptr;
      const int b = r >> 8, i = r & 255;
      const int unit = 128 * b + (i & 127);
      if (unit >= nsms) return nullptr;
      return (i < 128 ? p.g_sgate : p.g_sup) + static_cast<size_t>(unit) * d;
    }
    case WG_O:
      *ld_or_skip = m;
      return row < l ? p.g_out + (static_cast<size_t>(group) * l + row) * m : nullptr;
    case WG_GU: {
      *ld_or_skip = l;
      if (p.relu2) return row < m ? p.g_upx + (static_cast<size_t>(group) * m + row) * l : nullptr;
      const int b = row >> 8, i = row & 255;
      const int unit = 128 * b + (i & 127);
      if (unit >= m) return nullptr;
      return (i < 128 ? p.g_gate : p.g_upx) + (static_cast<size_t>(group) * m + unit) * l;
    }
    default:
      return nullptr;
  }
}

__device__ __forceinline__ void epi_wgrad(uint32_t taddr, bool valid, const TcParams &p, int row,
                                          int group, int col0, bool empty, int half,
                                          uint8_t *stage) {
  const int ky = p.wg_l + p.wg_ns * p.wg_ms;
  int ld = 0;
  float *rowp = nullptr;
  if (p.wg_kind != WG_Y && valid) rowp = wgrad_row_dst(p, row, group, &ld);
  const int n_cols = p.wg_kind == WG_Y ? ky : ld;
#pragma unroll 1
  for (int c = half * (TN / 64); c < (half + 1) * (TN / 64); ++c) {
    float v[32];
    if (empty) {
#pragma unroll
      for (int j = 0; j < 32; ++j) v[j] = 0.0f;
    } else {
      uint32_t r[32];
      ptx::tmem_ld_32x32b_x32(taddr + c * 32, r);
      ptx::tmem_ld_wait();
#pragma unroll
      for (int j = 0; j < 32; ++j) v[j] = __uint_as_float(r[j]);
    }
    const int col = col0 + c * 32;
    float *dst = nullptr;
    if (valid && col < n_cols) {
      if (p.wg_kind == WG_Y) {  // columns [0, l): dW_up; then each shared expert's dS_o
        if (col < p.wg_l) {
          dst = p.g_up + static_cast<size_t>(row) * p.wg_l + col;
        } else {
          const int cc = col - p.wg_l, j = cc / p.wg_ms;
          dst = p.g_sout + (static_cast<size_t>(j) * p.wg_d + row) * p.wg_ms + (cc - j * p.wg_ms);
        }
      } else if (rowp) {
        dst = rowp + col;
      }
    }
    store_rows_f32x32(stage, v, dst);
  }
}

// Columns [0,128) are gate rows g0..g0+127, [128,256) the matching up rows:
// h = silu(gate) * up for 128 hidden columns starting at hcol0.
__device__ __forceinline__ void epi_swiglu(uint32_t taddr, bool valid, __nv_bfloat16 *row_dst,
                                           int hcol0, int half, OutSink *sink = nullptr) {
#pragma unroll 1
  for (int c = half * (TN / 128); c < (half + 1) * (TN / 128); ++c) {
    uint32_t g[32], u[32];
    ptx::tmem_ld_32x32b_x32(taddr + c * 32, g);
    ptx::tmem_ld_32x32b_x32(taddr + TN / 2 + c * 32, u);
    ptx::tmem_ld_wait();
    float h[32];
#pragma unroll
    for (int j = 0; j < 32; ++j) h[j] = silu_bf16out(__uint_as_float(g[j])) * __uint_as_float(u[j]);
    if (sink && sink->map) sink_store(*sink, h, hcol0 + c * 32);
    else if (valid) store_bf16x32(row_dst + hcol0 + c * 32, h);
  }
}

// Raw gate/up pre-activations (row segment raw_dst, 256 columns as in the
// accumulator) and the SwiGLU hidden (h_dst + hcol0) of one tile.
__device__ __forceinline__ void epi_swiglu_raw(uint32_t taddr, bool valid,
                                               __nv_bfloat16 *raw_dst, __nv_bfloat16 *h_dst,
                                               int half, uint8_t *stage) {
#pragma unroll 1
  for (int c = half * (TN / 128); c < (half + 1) * (TN / 128); ++c) {
    uint32_t g[32], u[32];
    ptx::tmem_ld_32x32b_x32(taddr + c * 32, g);
    ptx::tmem_ld_32x32b_x32(taddr + TN / 2 + c * 32, u);
    ptx::tmem_ld_wait();
    float gv[32], uv[32], h[32];
#pragma unroll
    for (int j = 0; j < 32; ++j) {
      gv[j] = __uint_as_float(g[j]);
      uv[j] = __uint_as_float(u[j]);
      h[j] = silu_bf16out(gv[j]) * uv[j];
    }
    store_rows_bf16x32(stage, gv, valid ? raw_dst + c * 32 : nullptr);
    store_rows_bf16x32(stage, uv, valid ? raw_dst + TN / 2 + c * 32 : nullptr);
    store_rows_bf16x32(stage, h, valid ? h_dst + c * 32 : nullptr);
  }
}

// Squared ReLU: raw up pre-activation and h = relu(b)^2, masked at n_cols.
__device__ __forceinline__ void epi_relu2_raw(uint32_t taddr, bool valid, __nv_bfloat16 *raw_dst,
                                              __nv_bfloat16 *h_dst, int col0, int n_cols,
                                              int half, uint8_t *stage) {
#pragma unroll 1
  for (int c = half * (TN / 64); c < (half + 1) * (TN / 64); ++c) {
    uint32_t r[32];
    ptx::tmem_ld_32x32b_x32(taddr + c * 32, r);
    ptx::tmem_ld_wait();
    float bv[32], h[32];
#pragma unroll
    for (int j = 0; j < 32; ++j) {
      bv[j] = __uint_as_float(r[j]);
      const float a = fmaxf(bv[j], 0.0f);
      h[j] = a * a;
    }
    const int col = col0 + c * 32;
    const bool st = valid && col < n_cols;
    store_rows_bf16x32(stage, bv, st ? raw_dst + col : nullptr);
    store_rows_bf16x32(stage, h, st ? h_dst + col : nullptr);
  }
}

// fp32 outputs of the backward (dU, dZp): 256 accumulator columns -> the row
// segment row_dst + col0 .., chunks past n_cols skipped, row-coalesced.
__device__ __forceinline__ void epi_plain_f32_rows(uint32_t taddr, bool valid, float *row_dst,
                                                   int col0, int n_cols, int half,
                                                   uint8_t *stage) {
#pragma unroll 1
  for (int c = half * (TN / 64); c < (half + 1) * (TN / 64); ++c) {
    uint32_t r[32];
    ptx::tmem_ld_32x32b_x32(taddr + c * 32, r);
    ptx::tmem_ld_wait();
    float v[32];
#pragma unroll
    for (int j = 0; j < 32; ++j) v[j] = __uint_as_float(r[j]);
    const int col = col0 + c * 32;
    store_rows_f32x32(stage, v, valid && col < n_cols ? row_dst + col : nullptr);
  }
}

// ---- epilogues of the E4M3 GEMM (kF8): the accumulator holds products of
// E4M3 codes, so column c is multiplied by the A row's scale sa and the
// weight row's scale scl[c] (both powers of two).
__device__ __forceinline__ void epi_swiglu_scaled(uint32_t taddr, bool valid,
                                                  __nv_bfloat16 *row_dst, int hcol0, float sa,
                                                  const float *scl, int half, OutSink *sink) {
#pragma unroll 1
  for (int c = half * (TN / 128); c < (half + 1) * (TN / 128); ++c) {
    uint32_t g[32], u[32];
    ptx::tmem_ld_32x32b_x32(taddr + c * 32, g);
    ptx::tmem_ld_32x32b_x32(taddr + TN / 2 + c * 32, u);
    ptx::tmem_ld_wait();
    float h[32];
#pragma unroll
    for (int j = 0; j < 32; ++j)
      h[j] = silu_bf16out(__uint_as_float(g[j]) * (sa * scl[c * 32 + j])) *
             (__uint_as_float(u[j]) * (sa * scl[TN / 2 + c * 32 + j]));
    if (sink && sink->map) sink_store(*sink, h, hcol0 + c * 32);
    else if (valid) store_bf16x32(row_dst + hcol0 + c * 32, h);
  }
}

__device__ __forceinline__ void epi_relu2_scaled(uint32_t taddr, bool valid,
                                                 __nv_bfloat16 *row_dst, int col0, int n_cols,
                                                 float sa, const float *scl, int half,
                                                 OutSink *sink) {
#pragma unroll 1
  for (int c = half * (TN / 64); c < (half + 1) * (TN / 64); ++c) {
    const int col = col0 + c * 32;
    uint32_t r[32];
    ptx::tmem_ld_32x32b_x32(taddr + c * 32, r);
    ptx::tmem_ld_wait();
    float h[32];
#pragma unroll
    for (int j = 0; j < 32; ++j) {
      const float a = fmaxf(__uint_as_float(r[j]) * (sa * scl[c * 32 + j]), 0.0f);
      h[j] = a * a;
    }
    if (sink && sink->map) {
      if (col < n_cols) sink_store(*sink, h, col);
    } else if (valid && col < n_cols) {
      store_bf16x32(row_dst + col, h);
    }
  }
}

__device__ __forceinline__ void epi_plain_scaled(uint32_t taddr, bool valid,
                                                 __nv_bfloat16 *row_dst, int col0, int n_cols,
                                                 float sa, const float *scl, int half,
                                                 OutSink *sink) {
#pragma unroll 1
  for (int c = half * (TN / 64); c < (half + 1) * (TN / 64); ++c) {
    const int col = col0 + c * 32;
    uint32_t r[32];
    ptx::tmem_ld_32x32b_x32(taddr + c * 32, r);
    ptx::tmem_ld_wait();
    float v[32];
#pragma unroll
    for (int j = 0; j < 32; ++j) v[j] = __uint_as_float(r[j]) * (sa * scl[c * 32 + j]);
    if (sink && sink->map) {
      if (col < n_cols) sink_store(*sink, v, col);
    } else if (valid && col < n_cols) {
      store_bf16x32(row_dst + col, v);
    }
  }
}

// NVFP4 GEMM (one accumulator): the calling warp copies its half of the tile
// (128 accumulator columns of its 32 lanes) into registers and releases the
// accumulator at once, so that the next tile's MMAs overlap the scaling,
// activation and stores that follow.  Modes: TC_EXPERT_GU (SwiGLU or squared
// ReLU) and TC_EXPERT_DOWN, as in the kF8 branches of epilogue_tile.
__device__ __forceinline__ void epilogue_tile_release_early(const TcParams &p, const Tile &tl,
                                                            uint32_t taddr, int row, bool valid,
                                                            int col0, int half, OutSink &sink,
                                                            uint64_t *acc_empty, int lane) {
  const bool gu = p.mode == TC_EXPERT_GU, swiglu = gu && !p.relu2;
  // register block j: SwiGLU gate, up, gate, up of chunks 2h, 2h + 1
  // (columns c 32 and TN / 2 + c 32); else chunks 4h .. 4h + 3
  uint32_t a[4][32];
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const int col = swiglu ? (2 * half + (j >> 1)) * 32 + (j & 1) * (TN / 2) : (4 * half + j) * 32;
    ptx::tmem_ld_32x32b_x32(taddr + col, a[j]);
  }
  ptx::tmem_ld_wait();
  ptx::tc_fence_before();
  __syncwarp();
  if (lane == 0) ptx::mbar_arrive(acc_empty);
  const float sa = valid ? p.a_scale[row] : 0.0f;
  const float *scl = p.b_scale + static_cast<size_t>(tl.expert) * p.b_scale_ld + col0;
  __nv_bfloat16 *dst = p.out + static_cast<size_t>(row) * p.ld_out;
  if (swiglu) {
#pragma unroll
    for (int c2 = 0; c2 < 2; ++c2) {
      const int c = 2 * half + c2;
      float h[32];
#pragma unroll
      for (int j = 0; j < 32; ++j)
        h[j] = silu_bf16out(__uint_as_float(a[2 * c2][j]) * (sa * scl[c * 32 + j])) *
               (__uint_as_float(a[2 * c2 + 1][j]) * (sa * scl[TN / 2 + c * 32 + j]));
      const int hcol = col0 / 2 + c * 32;
      if (sink.map) sink_store(sink, h, hcol);
      else if (valid) store_bf16x32(dst + hcol, h);
    }
  } else {
    const int n_cols = gu ? p.n_cols2 : p.ld_out;
#pragma unroll
    for (int j4 = 0; j4 < 4; ++j4) {
      const int c = 4 * half + j4, col = col0 + c * 32;
      float v[32];
#pragma unroll
      for (int j = 0; j < 32; ++j) {
        const float t = __uint_as_float(a[j4][j]) * (sa * scl[c * 32 + j]);
        const float r = fmaxf(t, 0.0f);
        v[j] = gu ? r * r : t;  // squared ReLU hidden, or the plain output
      }
      if (sink.map) {
        if (col < n_cols) sink_store(sink, v, col);
      } else if (valid && col < n_cols) {
        store_bf16x32(dst + col, v);
      }
    }
  }
}

// One tile's epilogue for the calling warp: its 32 accumulator lanes (output
// rows row = lane's row, valid when inside the tile) and its column halves,
// by mode.  Shared by the single-CTA and the CTA-pair kernels.
template <bool kBwd, int kQ>
__device__ __forceinline__ void epilogue_tile(const TcParams &p, const Tile &tl, uint32_t taddr,
                                              int row, bool valid, int col0, int half0,
                                              OutSink &sink) {
  // kF8: a quantised-operand GEMM (E4M3 or NVFP4): the accumulator is scaled
  // by the A row's and the weight row's second-level scales
  constexpr bool kF8 = kQ != kBf16;
  // one epilogue warp per lane quarter covers both halves, two take one each
  constexpr int kHalfStep = Cfg<kQ>::EPI_WARPS / 4;
  // kF8: the A row's scale (rows past the tile's end are not stored)
  const float sa = (kF8 && valid) ? p.a_scale[row] : 0.0f;
  if (!kBwd && !kF8 && p.k_split > 1) {
    // one slice of a split reduction: the fp32 partial of this tile's rows
    const int ld = p.n_tiles_n * TN;
    float *dst = p.part + (static_cast<size_t>(tl.group) * p.M + row) * ld +
                 (col0 - p.n_tile_base * TN);
    for (int half = half0; half < 2; half += kHalfStep) {
#pragma unroll 1
      for (int c = half * (TN / 64); c < (half + 1) * (TN / 64); ++c) {
        uint32_t r[32];
        ptx::tmem_ld_32x32b_x32(taddr + c * 32, r);
        ptx::tmem_ld_wait();
        float v[32];
#pragma unroll
        for (int j = 0; j < 32; ++j) v[j] = __uint_as_float(r[j]);
        if (valid) store_f32x32(dst + c * 32, v);
      }
    }
    return;
  }
  for (int half = half0; half < 2; half += kHalfStep) {
    switch (p.mode) {
      case TC_X_FUSED:
        if (col0 < p.r_end) {
          epi_plain<true>(taddr, valid, p.logits + static_cast<size_t>(row) * p.ld_logits, col0,
                          p.n_routed, half);
        } else if (col0 < p.z_end) {
          epi_plain<false>(taddr, valid, p.z + static_cast<size_t>(row) * p.ld_z,
                           col0 - p.r_end, p.l, half, &sink);
        } else if (kBwd && p.raw) {  // pre-activations and the hidden
          if (p.relu2)
            epi_relu2_raw(taddr, valid, p.out2 + static_cast<size_t>(row) * p.ld_out2,
                          p.out + static_cast<size_t>(row) * p.ld_out + p.out_col0,
                          col0 - p.z_end, p.n_cols2, half, sink.buf);
          else
            epi_swiglu_raw(taddr, valid,
                           p.out2 + static_cast<size_t>(row) * p.ld_out2 + (col0 - p.z_end),
                           p.out + static_cast<size_t>(row) * p.ld_out + p.out_col0 +
                               (col0 - p.z_end) / 2,
                           half, sink.buf);
        } else if (p.relu2) {
          epi_relu2(taddr, valid, p.out + static_cast<size_t>(row) * p.ld_out + p.out_col0,
                    col0 - p.z_end, p.n_cols2, half);
        } else {
          epi_swiglu(taddr, valid, p.out + static_cast<size_t>(row) * p.ld_out,
                     p.out_col0 + (col0 - p.z_end) / 2, half);
        }
        break;
      case TC_EXPERT_GU:
        if constexpr (kF8) {
          const float *scl = p.b_scale + static_cast<size_t>(tl.expert) * p.b_scale_ld + col0;
          __nv_bfloat16 *hrow = p.out + static_cast<size_t>(row) * p.ld_out;
          if (p.relu2) epi_relu2_scaled(taddr, valid, hrow, col0, p.n_cols2, sa, scl, half, &sink);
          else epi_swiglu_scaled(taddr, valid, hrow, col0 / 2, sa, scl, half, &sink);
        } else if (kBwd && p.raw && p.relu2)
          epi_relu2_raw(taddr, valid, p.out + static_cast<size_t>(row) * p.ld_out,
                        p.out_h + static_cast<size_t>(row) * p.ld_h, col0, p.n_cols2, half,
                        sink.buf);
        else if (kBwd && p.raw)
          epi_swiglu_raw(taddr, valid, p.out + static_cast<size_t>(row) * p.ld_out + col0,
                         p.out_h + static_cast<size_t>(row) * p.ld_h + col0 / 2, half, sink.buf);
        else if (p.relu2)
          epi_relu2(taddr, valid, p.out + static_cast<size_t>(row) * p.ld_out, col0, p.n_cols2,
                    half, &sink);
        else
          epi_swiglu(taddr, valid, p.out + static_cast<size_t>(row) * p.ld_out, col0 / 2, half,
                     &sink);
        break;
      case TC_WGRAD:
        if constexpr (kBwd)
          epi_wgrad(taddr, valid, p, row, tl.group, col0, tl.nkb == 0, half, sink.buf);
        break;
      default:  // TC_EXPERT_DOWN, TC_OUT
        if constexpr (kF8) {
          epi_plain_scaled(taddr, valid, p.out + static_cast<size_t>(row) * p.ld_out, col0,
                           p.ld_out, sa,
                           p.b_scale + static_cast<size_t>(tl.expert) * p.b_scale_ld + col0,
                           half, &sink);
        } else if (kBwd && p.out_f32)
          epi_plain_f32_rows(taddr, valid, p.out_f32 + static_cast<size_t>(row) * p.ld_out, col0,
                             p.ld_out, half, sink.buf);
        else
          epi_plain<false>(taddr, valid, p.out + static_cast<size_t>(row) * p.ld_out, col0,
                           p.ld_out, half, &sink);
        break;
    }
  }  // halves
}

// kBwd: the instantiation with the backward's epilogues and the TC_WGRAD
// mode; the forward launches the other one, whose smaller register budget
// leaves room for the routing kernels that run beside it.
// kQ: the operand format.  kE4m3 / kNvf4: the expert GEMMs with E4M3 or
// NVFP4 operands (TC_EXPERT_GU / TC_EXPERT_DOWN with a_scale and b_scale):
// tcgen05.mma kind::f8f6f4 over 128-element K-blocks, or kind::mxf4nvf4 with
// 16-element scale blocks over 256-element K-blocks.
template <bool kBwd, int kQ>
__global__ void __launch_bounds__(Cfg<kQ>::NUM_THREADS, 1)
    tc_gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                   const __grid_constant__ CUtensorMap tmA32, const __grid_constant__ CUtensorMap tmO,
                   const TcParams p) {
  constexpr bool kF8 = kQ != kBf16;  // quantised operands with row scales
  constexpr int STAGES = Cfg<kQ>::STAGES;
  constexpr int KB = Cfg<kQ>::KB;
  constexpr int ACC_BUFS = Cfg<kQ>::ACC_BUFS;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  // [A ring][B ring][NVFP4: scale-block ring][control block]
  // [tma_out: the epilogue warps' staging buffers]
  uint8_t *smA = smem;
  uint8_t *smB = smem + STAGES * A_BYTES;
  uint8_t *smSF = smem + STAGES * (A_BYTES + B_BYTES);
  SmemCtl *ctl = reinterpret_cast<SmemCtl *>(smem + Cfg<kQ>::RING_BYTES);
  uint8_t *staging = smem + Cfg<kQ>::RING_BYTES + CTL_BYTES;
  // TMA stores: the forward instantiations with a bf16-output mode
  const bool use_tma_out = !kBwd && p.tma_out != 0;
  volatile int *abort_flag = &ctl->abort;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  const bool grouped = (p.mode == TC_EXPERT_GU || p.mode == TC_EXPERT_DOWN);
  const int m_tiles = grouped ? 0 : (p.M + TM - 1) / TM;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      ptx::mbar_init(&ctl->full[s], 1);
      ptx::mbar_init(&ctl->empty[s], 1);  // freed by the MMA commit
    }
    for (int a = 0; a < 2; ++a) {
      ptx::mbar_init(&ctl->acc_full[a], 1);
      ptx::mbar_init(&ctl->acc_empty[a], Cfg<kQ>::EPI_WARPS);  // one per epilogue warp
    }
    ptx::mbar_init(&ctl->drain, 1);
    ctl->abort = 0;
    ptx::fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    ptx::prefetch_tmap(&tmA);
    if (kF8) ptx::prefetch_tmap(&tmA32);
    ptx::prefetch_tmap(&tmB);
  }
  if (warp == 1) {
    ptx::tmem_alloc(&ctl->tmem_base, TMEM_COLS);
    ptx::tmem_relinquish();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem_base = ctl->tmem_base;
  // everything above touched only shared memory, TMEM and the parameters
  griddep_wait();
  const int total = grouped ? (*p.n_mtiles) * p.n_tiles_n
                            : m_tiles * p.n_tiles_n *
                                  (p.mode == TC_WGRAD ? p.groups : p.k_split > 1 ? p.k_split : 1);

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      int it = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < total && ok; t += gridDim.x) {
        const Tile tl = decode_tile(p, t, m_tiles, KB);
        for (int kb = 0; kb < tl.nkb; ++kb, ++it) {
          const int s = it % STAGES;
          const uint32_t ph = (it / STAGES) & 1;
          if (!ptx::mbar_wait(&ctl->empty[s], ph ^ 1, abort_flag)) {
            record_failure(p, ctl, DEV_TIMEOUT_PRODUCER);
            ok = false;
            break;
          }
          // A's K coordinate in bytes: elements for bf16 (the map's unit) and
          // E4M3, half the elements for packed NVFP4
          const int kx = kQ == kNvf4 ? (tl.k0 + kb * KB) / 2 : tl.k0 + kb * KB;
          // kF8 (weight streaming): a tile of at most 32 token rows loads
          // only those rows of A (the MMA's other rows are never stored)
          const bool a32 = kF8 && tl.row_hi - tl.a_row <= 32;
          ptx::mbar_arrive_expect_tx(&ctl->full[s], (a32 ? A_BYTES / 4 : A_BYTES) + B_BYTES +
                                                        Cfg<kQ>::SF_BYTES);
          if (kBwd && p.mode == TC_WGRAD) {
            // MN-major operands straight from the token-major matrices: A as
            // two {64, 64} boxes (M columns a_row.., token rows kx..), B as four
            // (N columns b_row..); rows past a matrix's end read as zeros
#pragma unroll
            for (int c = 0; c < TM / 64; ++c)
              ptx::tma_load_2d(smA + s * A_BYTES + c * MN_BOX_BYTES, &tmA, &ctl->full[s],
                               tl.a_row + 64 * c, kx);
#pragma unroll
            for (int c = 0; c < TN / 64; ++c)
              ptx::tma_load_2d(smB + s * B_BYTES + c * MN_BOX_BYTES, &tmB, &ctl->full[s],
                               tl.b_row + 64 * c, kx);
            continue;
          }
          ptx::tma_load_2d(smA + s * A_BYTES, a32 ? &tmA32 : &tmA, &ctl->full[s], kx, tl.a_row);
          if constexpr (kQ == kNvf4) {
            // this stage's scale blocks: the A tile's (by M-tile) and the B
            // tile's (by expert and N-tile), 2 KB and 4 KB, contiguous
            const int nkb_all = (p.Kdim + KB - 1) / KB;
            uint8_t *sf = smSF + s * Cfg<kQ>::SF_BYTES;
            ptx::bulk_load(sf, p.a_sf + (static_cast<size_t>(tl.mt) * nkb_all + kb) * SFA_BYTES,
                           SFA_BYTES, &ctl->full[s]);
            ptx::bulk_load(sf + SFA_BYTES,
                           p.b_sf + ((static_cast<size_t>(tl.expert) * p.n_tiles_n + tl.n_tile) *
                                         nkb_all + kb) * SFB_BYTES,
                           SFB_BYTES, &ctl->full[s]);
          }
          ptx::tma_load_2d(smB + s * B_BYTES, &tmB, &ctl->full[s], 0, tl.b_row + kb * TN);
        }
      }
      if (!ok) {  // let every copy still in flight land before the CTA exits
        for (int j = (it > STAGES ? it - STAGES : 0); j < it; ++j)
          if (!drain_wait(&ctl->full[j % STAGES], (j / STAGES) & 1))
            record_failure(p, ctl, DEV_TIMEOUT_DRAIN);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      int it = 0, tl_count = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < total && ok; t += gridDim.x, ++tl_count) {
        const int acc = tl_count % ACC_BUFS;
        const uint32_t acc_ph = (tl_count / ACC_BUFS) & 1;
        if (!ptx::mbar_wait(&ctl->acc_empty[acc], acc_ph ^ 1, abort_flag)) {
          record_failure(p, ctl, DEV_TIMEOUT_MMA);
          ok = false;
          break;
        }
        ptx::tc_fence_after();
        const uint32_t d_tmem = tmem_base + acc * TN;
        const int nkb = decode_tile(p, t, m_tiles, KB).nkb;
        for (int kb = 0; kb < nkb; ++kb, ++it) {
          const int s = it % STAGES;
          const uint32_t ph = (it / STAGES) & 1;
          if (!ptx::mbar_wait(&ctl->full[s], ph, abort_flag)) {
            record_failure(p, ctl, DEV_TIMEOUT_MMA);
            ok = false;
            break;
          }
          ptx::tc_fence_after();
          const uint32_t a_addr = ptx::smem_u32(smA + s * A_BYTES);
          const uint32_t b_addr = ptx::smem_u32(smB + s * B_BYTES);
          if constexpr (kQ == kNvf4) {
            // scale blocks into TMEM: MMA k reads A's at SFA_COL + 4k and B's
            // (two 128-row atoms) at SFB_COL + 8k; executed before the MMAs
            // below, which this thread issues after them
            const uint32_t sfa = ptx::smem_u32(smSF + s * Cfg<kQ>::SF_BYTES);
            const uint32_t sfb = sfa + SFA_BYTES;
#pragma unroll
            for (int k = 0; k < 4; ++k) {
              ptx::tmem_cp_32x128b_x4(tmem_base + SFA_COL + 4 * k,
                                      ptx::smem_desc_rows16(sfa + 512 * k));
              ptx::tmem_cp_32x128b_x4(tmem_base + SFB_COL + 8 * k,
                                      ptx::smem_desc_rows16(sfb + 512 * k));
              ptx::tmem_cp_32x128b_x4(tmem_base + SFB_COL + 8 * k + 4,
                                      ptx::smem_desc_rows16(sfb + SFA_BYTES + 512 * k));
            }
          }
          // four MMAs per K-block: K = 16 bf16, 32 E4M3 or 64 E2M1 elements,
          // 32 bytes of each row
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            if constexpr (kQ == kNvf4)
              ptx::mma_nvf4(d_tmem, ptx::smem_desc_sw128(a_addr + k * 32),
                            ptx::smem_desc_sw128(b_addr + k * 32), IDESC4,
                            tmem_base + SFA_COL + 4 * k, tmem_base + SFB_COL + 8 * k,
                            (kb | k) != 0);
            else if constexpr (kQ == kE4m3)
              ptx::mma_e4m3(d_tmem, ptx::smem_desc_sw128(a_addr + k * 32),
                            ptx::smem_desc_sw128(b_addr + k * 32), IDESC8, (kb | k) != 0);
            else if (kBwd && p.mode == TC_WGRAD)  // MN-major: K = 16 rows = 2048 bytes
              ptx::mma_bf16(d_tmem, ptx::smem_desc_mn_sw128(a_addr + k * 2048),
                            ptx::smem_desc_mn_sw128(b_addr + k * 2048), IDESC_MN, (kb | k) != 0);
            else
              ptx::mma_bf16(d_tmem, ptx::smem_desc_sw128(a_addr + k * 32),
                            ptx::smem_desc_sw128(b_addr + k * 32), IDESC, (kb | k) != 0);
          }
          ptx::mma_commit(&ctl->empty[s]);  // the stage is free once these MMAs finish
        }
        if (!ok) break;
        ptx::mma_commit(&ctl->acc_full[acc]);  // accumulator ready for the epilogue
      }
      if (!ok) {  // let issued MMAs finish before TMEM is freed
        ptx::mma_commit(&ctl->drain);
        if (!drain_wait(&ctl->drain, 0)) record_failure(p, ctl, DEV_TIMEOUT_DRAIN);
      }
    }
    // every MMA is issued: the next kernel of the stream may be scheduled
    if (lane == 0) griddep_launch_dependents();
  } else {
    // ------------------------------------------------------------ epilogue
    const int q = warp & 3;             // TMEM lane quarter this warp may access
    // which half of the tile's columns (both, one after the other, when the
    // variant has one epilogue warp per lane quarter)
    const int half0 = (warp - 2) >> 2;
    const int row_in_tile = q * 32 + lane;
    OutSink sink;
    sink.map = nullptr;
    sink.buf = staging + (warp - 2) * 2 * OUT_BOX_BYTES;
    sink.x0 = 0;
    sink.y = 0;
    sink.issued = 0;
    int tl_count = 0;
    for (int t = blockIdx.x; t < total; t += gridDim.x, ++tl_count) {
      const int acc = tl_count % ACC_BUFS;
      const uint32_t acc_ph = (tl_count / ACC_BUFS) & 1;
      // Lane 0 waits; the verdict is broadcast so the warp stays converged
      // for the .sync.aligned TMEM loads below.
      int ok = 1;
      if (lane == 0) ok = ptx::mbar_wait(&ctl->acc_full[acc], acc_ph, abort_flag) ? 1 : 0;
      ok = __shfl_sync(0xFFFFFFFFu, ok, 0);
      if (!ok) {
        if (lane == 0) record_failure(p, ctl, DEV_TIMEOUT_EPILOGUE);
        break;
      }
      ptx::tc_fence_after();
      const Tile tl = decode_tile(p, t, m_tiles, KB);
      const int row = tl.a_row + row_in_tile;
      const bool valid = row < tl.row_hi;
      const uint32_t taddr = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + acc * TN;
      const int col0 = tl.n_tile * TN;
      // TMA stores only for a warp whose 32 rows are all valid: a grouped
      // tile's rows past its expert's end belong to the next tile.
      sink.y = tl.a_row + q * 32;
      sink.map = (use_tma_out && sink.y + 31 < tl.row_hi) ? &tmO : nullptr;
      if constexpr (kQ == kNvf4) {
        // one warp per half of the tile (two per lane quarter); the
        // accumulator is released inside, as soon as it is in registers
        epilogue_tile_release_early(p, tl, taddr, row, valid, col0, half0, sink,
                                    &ctl->acc_empty[acc], lane);
      } else {
        epilogue_tile<kBwd, kQ>(p, tl, taddr, row, valid, col0, half0, sink);
        ptx::tc_fence_before();
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive(&ctl->acc_empty[acc]);
      }
    }
    // the staging buffers stay allocated until this warp's stores are done
    if (use_tma_out && lane == 0) ptx::bulk_wait_group_all();
  }

  ptx::tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem_base, TMEM_COLS);
  }
}

// ---------------------------------------------------------------- CTA pairs
// The forward's bf16 GEMMs run on CTA pairs: a cluster of two CTAs on two SMs
// computes a 256 x 256 output tile with tcgen05.mma.cta_group::2 (M = 256).
// Each CTA stages its own 128 A rows and one half (128 rows) of the tile's
// 256 B rows, so a K-block moves 32 KB through each SM's shared memory for
// 128 x 256 x 64 multiply-adds, where the single-CTA tile needs 48 KB: the
// L2-to-SM feed, not the tensor pipe, limits the 128 x 256 tile.  Each CTA's
// TMEM holds its 128 rows of the accumulator, so the epilogue is the
// single-CTA one.  Grouped modes take 256-row M-tiles from their own table
// (an expert's last tile may leave rank 1 without rows: it then loads no A).
//
// Roles as in the single-CTA kernel, in both CTAs; rank 0 (the leader)
// alone issues the MMAs.  Both CTAs' TMA loads complete on the leader's
// `full` barrier; the leader's commits free both CTAs' ring stages and
// publish both halves of an accumulator; both CTAs' epilogue warps release
// it on the leader's `acc_empty`.  Every load fills only the issuing CTA's
// shared memory.
constexpr int P_STAGES = 6;
constexpr int P_B_BYTES = (TN / 2) * TKB * 2;             // 16 KB: this CTA's half of B
constexpr int P_RING_BYTES = P_STAGES * (A_BYTES + P_B_BYTES);  // 192 KB
constexpr uint32_t P_IDESC = ptx::idesc_bf16_f32(2 * TM, TN);

struct __align__(8) PairCtl {
  uint64_t full[P_STAGES];   // leader: both CTAs' bytes of a stage landed
  uint64_t empty[P_STAGES];  // each CTA: its ring stage may be refilled
  uint64_t acc_full[2];      // each CTA: its half of an accumulator is ready
  uint64_t acc_empty[2];     // leader: both CTAs' epilogue warps are done with it
  uint64_t drain;            // leader, abort path: issued MMAs finished
  uint64_t peer_done;        // exit handshake
  uint32_t tmem_base;
  int abort;
};
static_assert(sizeof(PairCtl) <= CTL_BYTES, "pair control block");
constexpr size_t pair_smem_bytes(bool staging) {
  return 1024 /*align slack*/ + P_RING_BYTES + (staging ? CTL_BYTES + STAGING_BYTES : sizeof(PairCtl));
}
static_assert(pair_smem_bytes(true) <= 232448, "shared memory per CTA");

// Pair tile t as seen by CTA `rank`: its 128 A rows (a_row, row_hi as in the
// single-CTA tile) and its half of the B block (b_row, K-block 0);
// *rank1_rows: whether rank 1 has any valid rows in the tile.
__device__ __forceinline__ Tile decode_pair_tile(const TcParams &p, int t, int m_tiles2,
                                                 uint32_t rank, bool *rank1_rows) {
  Tile tl;
  tl.k0 = 0;
  tl.nkb = p.Kdim / TKB;
  tl.group = 0;
  tl.expert = 0;
  int row0, b0;
  if (p.mode == TC_X_FUSED || p.mode == TC_OUT) {
    // consecutive pairs share B; with k_split, item r of an M-tile is slice
    // r % k_split of N-tile r / k_split (K-blocks [k0, k0 + nkb) of that slice,
    // its index in group)
    const int m = t % m_tiles2, r = t / m_tiles2;
    const int ks = p.k_split > 1 ? p.k_split : 1;
    const int split = r % ks, n = p.n_tile_base + r / ks;
    const int nkb_all = tl.nkb, per = (nkb_all + ks - 1) / ks;
    row0 = m * 2 * TM;
    b0 = (n * nkb_all + split * per) * TN;
    tl.k0 = split * per * TKB;
    tl.nkb = min(per, nkb_all - split * per);
    tl.group = split;
    tl.n_tile = n;
    tl.row_hi = p.M;
  } else {
    const int mt = t / p.n_tiles_n, n = t % p.n_tiles_n;  // consecutive pairs share A
    const TileEntry te = p.tiles[mt];
    row0 = te.row0;
    b0 = (te.expert * p.n_tiles_n + n) * tl.nkb * TN;
    tl.n_tile = n;
    tl.row_hi = te.row_end;
    tl.expert = te.expert;
  }
  tl.a_row = row0 + static_cast<int>(rank) * TM;
  tl.b_row = b0 + static_cast<int>(rank) * (TN / 2);
  *rank1_rows = row0 + TM < tl.row_hi;
  return tl;
}

__device__ __forceinline__ void record_failure_pair(const TcParams &p, PairCtl *ctl,
                                                    uint32_t peer, int code) {
  ctl->abort = 1;
  ptx::st_cluster_u32(ptx::map_to_rank(ptx::smem_u32(&ctl->abort), peer), 1u);
  if (p.status) atomicCAS(p.status, 0, code);
}

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(Cfg<kBf16>::NUM_THREADS, 1)
    tc_pair_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                   const __grid_constant__ CUtensorMap tmO, const TcParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  // [A ring][B-half ring][control block][tma_out: staging buffers]
  uint8_t *smA = smem;
  uint8_t *smB = smem + P_STAGES * A_BYTES;
  PairCtl *ctl = reinterpret_cast<PairCtl *>(smem + P_RING_BYTES);
  uint8_t *staging = smem + P_RING_BYTES + CTL_BYTES;
  volatile int *abort_flag = &ctl->abort;
  const bool use_tma_out = p.tma_out != 0;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = ptx::cluster_ctarank();
  const uint32_t peer = rank ^ 1u;
  const bool leader = rank == 0;
  const int cid = static_cast<int>(ptx::cluster_id_x());
  const int ncl = static_cast<int>(ptx::cluster_count_x());

  const bool grouped = (p.mode == TC_EXPERT_GU || p.mode == TC_EXPERT_DOWN);
  const int m_tiles2 = grouped ? 0 : (p.M + 2 * TM - 1) / (2 * TM);

  if (threadIdx.x == 0) {
    for (int s = 0; s < P_STAGES; ++s) {
      ptx::mbar_init(&ctl->full[s], 1);
      ptx::mbar_init(&ctl->empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      ptx::mbar_init(&ctl->acc_full[a], 1);
      ptx::mbar_init(&ctl->acc_empty[a], 2 * NUM_EPI_WARPS);
    }
    ptx::mbar_init(&ctl->drain, 1);
    ptx::mbar_init(&ctl->peer_done, 1);
    ctl->abort = 0;
    ptx::fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    ptx::prefetch_tmap(&tmA);
    ptx::prefetch_tmap(&tmB);
  }
  if (warp == 1) {
    ptx::tmem_alloc_pair(&ctl->tmem_base, TMEM_COLS);
    ptx::tmem_relinquish_pair();
  }
  ptx::tc_fence_before();
  ptx::cluster_sync_all();  // both CTAs' barriers initialised, TMEM allocated
  ptx::tc_fence_after();
  const uint32_t tmem_base = ctl->tmem_base;
  // everything above touched only shared memory, TMEM and the parameters
  griddep_wait();
  const int total = grouped ? (*p.n_mtiles) * p.n_tiles_n
                            : m_tiles2 * p.n_tiles_n * (p.k_split > 1 ? p.k_split : 1);

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      const uint32_t full0 = ptx::map_to_rank(ptx::smem_u32(&ctl->full[0]), 0);
      int it = 0;
      bool ok = true;
      for (int t = cid; t < total && ok; t += ncl) {
        bool rank1_rows;
        const Tile tl = decode_pair_tile(p, t, m_tiles2, rank, &rank1_rows);
        const bool load_a = leader || rank1_rows;
        const uint32_t tx = 2 * P_B_BYTES + (rank1_rows ? 2 * A_BYTES : A_BYTES);
        for (int kb = 0; kb < tl.nkb; ++kb, ++it) {
          const int s = it % P_STAGES;
          const uint32_t ph = (it / P_STAGES) & 1;
          if (!ptx::mbar_wait(&ctl->empty[s], ph ^ 1, abort_flag)) {
            record_failure_pair(p, ctl, peer, DEV_TIMEOUT_PRODUCER);
            ok = false;
            break;
          }
          if (leader) ptx::mbar_arrive_expect_tx(&ctl->full[s], tx);
          const uint32_t bar = full0 + s * 8;
          if (load_a) ptx::tma_load_2d_pair(smA + s * A_BYTES, &tmA, bar, tl.k0 + kb * TKB, tl.a_row);
          ptx::tma_load_2d_pair(smB + s * P_B_BYTES, &tmB, bar, 0, tl.b_row + kb * TN);
        }
      }
      if (!ok && leader) {  // let every copy of both CTAs still in flight land
        for (int j = (it > P_STAGES ? it - P_STAGES : 0); j < it; ++j)
          if (!drain_wait(&ctl->full[j % P_STAGES], (j / P_STAGES) & 1))
            record_failure_pair(p, ctl, peer, DEV_TIMEOUT_DRAIN);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer (leader)
    if (lane == 0 && leader) {
      const uint32_t empty_me = ptx::smem_u32(&ctl->empty[0]);
      const uint32_t empty_peer = ptx::map_to_rank(empty_me, peer);
      const uint32_t accf_me = ptx::smem_u32(&ctl->acc_full[0]);
      const uint32_t accf_peer = ptx::map_to_rank(accf_me, peer);
      int it = 0, tl_count = 0;
      bool ok = true;
      for (int t = cid; t < total && ok; t += ncl, ++tl_count) {
        bool unused_rows;
        const int nkb = decode_pair_tile(p, t, m_tiles2, rank, &unused_rows).nkb;
        const int acc = tl_count & 1;
        const uint32_t acc_ph = (tl_count >> 1) & 1;
        if (!ptx::mbar_wait(&ctl->acc_empty[acc], acc_ph ^ 1, abort_flag)) {
          record_failure_pair(p, ctl, peer, DEV_TIMEOUT_MMA);
          ok = false;
          break;
        }
        ptx::tc_fence_after();
        const uint32_t d_tmem = tmem_base + acc * TN;
        for (int kb = 0; kb < nkb; ++kb, ++it) {
          const int s = it % P_STAGES;
          const uint32_t ph = (it / P_STAGES) & 1;
          if (!ptx::mbar_wait(&ctl->full[s], ph, abort_flag)) {
            record_failure_pair(p, ctl, peer, DEV_TIMEOUT_MMA);
            ok = false;
            break;
          }
          ptx::tc_fence_after();
          const uint32_t a_addr = ptx::smem_u32(smA + s * A_BYTES);
          const uint32_t b_addr = ptx::smem_u32(smB + s * P_B_BYTES);
#pragma unroll
          for (int k = 0; k < TKB / 16; ++k)
            ptx::mma_bf16_pair(d_tmem, ptx::smem_desc_sw128(a_addr + k * 32),
                               ptx::smem_desc_sw128(b_addr + k * 32), P_IDESC, (kb | k) != 0);
          // both CTAs' stage s is free once these MMAs finish
          ptx::mma_commit_pair(empty_me + s * 8);
          ptx::mma_commit_pair(empty_peer + s * 8);
        }
        if (!ok) break;
        ptx::mma_commit_pair(accf_me + acc * 8);  // both halves of the accumulator ready
        ptx::mma_commit_pair(accf_peer + acc * 8);
      }
      if (!ok) {  // let issued MMAs finish before TMEM is freed
        ptx::mma_commit_pair(ptx::smem_u32(&ctl->drain));
        if (!drain_wait(&ctl->drain, 0)) record_failure_pair(p, ctl, peer, DEV_TIMEOUT_DRAIN);
      }
    }
    // every MMA of the pair is issued: the next kernel may be scheduled
    if (lane == 0) griddep_launch_dependents();
  } else {
    // ------------------------------------------------------------ epilogue (both CTAs)
    const int q = warp & 3;
    const int half0 = (warp - 2) >> 2;
    const uint32_t acc_empty0 = ptx::map_to_rank(ptx::smem_u32(&ctl->acc_empty[0]), 0);
    OutSink sink;
    sink.map = nullptr;
    sink.buf = staging + (warp - 2) * 2 * OUT_BOX_BYTES;
    sink.x0 = 0;
    sink.y = 0;
    sink.issued = 0;
    int tl_count = 0;
    for (int t = cid; t < total; t += ncl, ++tl_count) {
      const int acc = tl_count & 1;
      const uint32_t acc_ph = (tl_count >> 1) & 1;
      int ok = 1;
      if (lane == 0) ok = ptx::mbar_wait(&ctl->acc_full[acc], acc_ph, abort_flag) ? 1 : 0;
      ok = __shfl_sync(0xFFFFFFFFu, ok, 0);
      if (!ok) {
        if (lane == 0) record_failure_pair(p, ctl, peer, DEV_TIMEOUT_EPILOGUE);
        break;
      }
      ptx::tc_fence_after();
      bool rank1_rows;
      const Tile tl = decode_pair_tile(p, t, m_tiles2, rank, &rank1_rows);
      if (tl.a_row < tl.row_hi) {  // rank 1 of an expert's last tile may have no rows
        const int row = tl.a_row + q * 32 + lane;
        const bool valid = row < tl.row_hi;
        const uint32_t taddr = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + acc * TN;
        sink.y = tl.a_row + q * 32;
        sink.map = (use_tma_out && sink.y + 31 < tl.row_hi) ? &tmO : nullptr;
        epilogue_tile<false, kBf16>(p, tl, taddr, row, valid, tl.n_tile * TN, half0, sink);
      }
      ptx::tc_fence_before();
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive_cluster(acc_empty0 + acc * 8);
    }
    if (use_tma_out && lane == 0) ptx::bulk_wait_group_all();
  }

  // Exit: meet the peer (the leader's MMAs write this CTA's TMEM and its
  // loads complete on the leader's barriers; the peer's epilogue arrives on
  // the leader's), then free TMEM.
  ptx::tc_fence_before();
  __syncthreads();
  if (threadIdx.x == 0) {
    ptx::mbar_arrive_cluster(ptx::map_to_rank(ptx::smem_u32(&ctl->peer_done), peer));
    if (!drain_wait(&ctl->peer_done, 0) && p.status) atomicCAS(p.status, 0, DEV_TIMEOUT_DRAIN);
  }
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    ptx::tc_fence_after();
    ptx::tmem_dealloc_pair(tmem_base, TMEM_COLS);
  }
}

// Output step of a split reduction: each thread sums one 4-column group of
// one row over the slices, in slice order, and stores it by mode (TC_OUT: y in
// bf16; TC_X_FUSED: router logits in fp32, z in bf16).
__global__ void __launch_bounds__(256) splitk_reduce_kernel(const TcParams p) {
  griddep_wait();
  const int ld = p.n_tiles_n * TN, groups = ld / 4;
  const int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (i >= static_cast<int64_t>(p.M) * groups) return;
  const int row = static_cast<int>(i / groups), c = static_cast<int>(i % groups) * 4;
  const size_t slice = static_cast<size_t>(p.M) * ld;
  const float *src = p.part + static_cast<size_t>(row) * ld + c;
  // every slice's load in flight at once, then the sum in slice order
  float4 b[kMaxKSplit];
#pragma unroll
  for (int k = 0; k < kMaxKSplit; ++k)
    if (k < p.k_split) b[k] = __ldcg(reinterpret_cast<const float4 *>(src + k * slice));
  float4 a = b[0];
#pragma unroll
  for (int k = 1; k < kMaxKSplit; ++k) {
    if (k < p.k_split) {
      a.x += b[k].x;
      a.y += b[k].y;
      a.z += b[k].z;
      a.w += b[k].w;
    }
  }
  const float v[4] = {a.x, a.y, a.z, a.w};
  const int col = p.n_tile_base * TN + c;  // column of the launch's output space
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const int cj = col + j;
    if (p.mode == TC_OUT) {
      if (cj < p.ld_out) p.out[static_cast<size_t>(row) * p.ld_out + cj] = __float2bfloat16_rn(v[j]);
    } else if (cj < p.r_end) {
      if (cj < p.n_routed) p.logits[static_cast<size_t>(row) * p.ld_logits + cj] = v[j];
    } else if (cj < p.z_end && cj - p.r_end < p.l) {
      p.z[static_cast<size_t>(row) * p.ld_z + (cj - p.r_end)] = __float2bfloat16_rn(v[j]);
    }
  }
}

// Failure-detection self-test: one warp waits, with the same bounded wait as
// the GEMM roles, on an mbarrier that nothing ever completes; the wait runs
// out after limit_ns and the status word records it.  No fault, no hang.
__global__ void wait_selftest_kernel(int32_t *status, unsigned long long limit_ns) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    ptx::mbar_init(&bar, 1);
    abort_flag = 0;
    ptx::fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0 && !ptx::mbar_wait(&bar, 0, &abort_flag, limit_ns))
    atomicCAS(status, 0, DEV_TIMEOUT_SELFTEST);
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                  const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                  const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void *ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &ptr, 12000, cudaEnableDefault,
                                         &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(ptr);
  }
  return fn;
}

}  // namespace

// A split reduction is valid for the dense output modes (TC_OUT; TC_X_FUSED
// over the router and z columns only) with a partial buffer, every slice
// holding at least one K-block.
static bool split_ok(const TcParams &p, int kb_elems) {
  const int nkb = p.Kdim / kb_elems, per = (nkb + p.k_split - 1) / p.k_split;
  const bool x_cols =
      p.mode == TC_X_FUSED && !p.raw && (p.n_tile_base + p.n_tiles_n) * TN <= p.z_end;
  return p.part && p.k_split <= kMaxKSplit && (p.mode == TC_OUT || x_cols) &&
         (p.k_split - 1) * per < nkb;
}

cudaError_t launch_splitk_reduce(const TcParams &p, cudaStream_t s, bool pdl) {
  if (p.k_split < 2 || !p.part || p.M <= 0) return cudaErrorInvalidValue;
  const int64_t items = static_cast<int64_t>(p.M) * (p.n_tiles_n * TN / 4);
  const int blocks = static_cast<int>((items + 255) / 256);
  cudaError_t e = launch_ex(splitk_reduce_kernel, dim3(blocks), dim3(256), 0, s, pdl, p);
  return e != cudaSuccess ? e : cudaGetLastError();
}

int make_tmap_bf16(void *tmap_out, const void *base, int64_t rows, int64_t cols,
                   int64_t row_stride_elems, int box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn || rows <= 0 || cols <= 0) return -1;
  if ((reinterpret_cast<uintptr_t>(base) & 15) || (row_stride_elems * 2) % 16) return -1;
  const cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows)};
  const cuuint64_t strides[1] = {static_cast<cuuint64_t>(row_stride_elems * 2)};
  const cuuint32_t box[2] = {static_cast<cuuint32_t>(TKB), static_cast<cuuint32_t>(box_rows)};
  const cuuint32_t estr[2] = {1, 1};
  const CUresult r =
      fn(reinterpret_cast<CUtensorMap *>(tmap_out), CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2,
         const_cast<void *>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
         CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
         CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? 0 : -1;
}

int make_tmap_bf16_out(void *tmap_out, const void *base, int64_t rows, int64_t cols,
                       int64_t row_stride_elems) {
  EncodeTiledFn fn = encode_fn();
  if (!fn || rows <= 0 || cols <= 0) return -1;
  if ((reinterpret_cast<uintptr_t>(base) & 15) || (row_stride_elems * 2) % 16) return -1;
  const cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows)};
  const cuuint64_t strides[1] = {static_cast<cuuint64_t>(row_stride_elems * 2)};
  const cuuint32_t box[2] = {static_cast<cuuint32_t>(OUT_BOX), static_cast<cuuint32_t>(OUT_BOX)};
  const cuuint32_t estr[2] = {1, 1};
  const CUresult r =
      fn(reinterpret_cast<CUtensorMap *>(tmap_out), CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2,
         const_cast<void *>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
         CU_TENSOR_MAP_SWIZZLE_64B, CU_TENSOR_MAP_L2_PROMOTION_NONE,
         CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? 0 : -1;
}

int make_tmap_u8(void *tmap_out, const void *base, int64_t rows, int64_t cols,
                 int64_t row_stride_bytes, int box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn || rows <= 0 || cols <= 0) return -1;
  if ((reinterpret_cast<uintptr_t>(base) & 15) || row_stride_bytes % 16) return -1;
  const cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows)};
  const cuuint64_t strides[1] = {static_cast<cuuint64_t>(row_stride_bytes)};
  const cuuint32_t box[2] = {static_cast<cuuint32_t>(TKB8), static_cast<cuuint32_t>(box_rows)};
  const cuuint32_t estr[2] = {1, 1};
  const CUresult r =
      fn(reinterpret_cast<CUtensorMap *>(tmap_out), CU_TENSOR_MAP_DATA_TYPE_UINT8, 2,
         const_cast<void *>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
         CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
         CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? 0 : -1;
}

cudaError_t launch_tc_gemm(const void *tmapA, const void *tmapB, const TcParams &p, int num_sms,
                           int max_ctas, cudaStream_t s, const void *tmapA32,
                           const void *tmapOut) {
  static int attr_done = -1;
  int dev = 0;
  cudaGetDevice(&dev);
  if (attr_done != dev) {
    cudaError_t e = cudaFuncSetAttribute(tc_gemm_kernel<false, kBf16>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem_bytes<kBf16>(true)));
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(tc_gemm_kernel<true, kBf16>,
                               cudaFuncAttributeMaxDynamicSharedMemorySize,
                               static_cast<int>(smem_bytes<kBf16>(true)));
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(tc_gemm_kernel<false, kE4m3>,
                               cudaFuncAttributeMaxDynamicSharedMemorySize,
                               static_cast<int>(smem_bytes<kE4m3>(true)));
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(tc_gemm_kernel<false, kNvf4>,
                               cudaFuncAttributeMaxDynamicSharedMemorySize,
                               static_cast<int>(smem_bytes<kNvf4>(true)));
    if (e != cudaSuccess) return e;
    attr_done = dev;
  }
  const bool bwd = p.mode == TC_WGRAD || p.raw || p.out_f32 || p.out_h;
  const bool fp8 = p.b_scale != nullptr;      // quantised operands (E4M3 or NVFP4)
  const bool fp4 = fp8 && p.b_sf != nullptr;  // NVFP4: block scales as well
  if (fp8 && (bwd || !p.a_scale || (p.mode != TC_EXPERT_GU && p.mode != TC_EXPERT_DOWN)))
    return cudaErrorInvalidValue;
  if (fp4 != (p.a_sf != nullptr)) return cudaErrorInvalidValue;
  if (p.k_split > 1 && (fp8 || bwd || !split_ok(p, TKB))) return cudaErrorInvalidValue;
  if (p.tma_out && (bwd || p.mode == TC_WGRAD || !tmapOut)) return cudaErrorInvalidValue;
  // NVFP4: whole 16-element scale blocks and 16-byte rows (a ragged last
  // K-block is read as zero codes); else whole K-blocks
  if (p.Kdim <= 0 || (fp4 ? p.Kdim % 32 : p.Kdim % (fp8 ? TKB8 : TKB))) return cudaErrorInvalidValue;
  const int grid = max_ctas < num_sms ? max_ctas : num_sms;
  if (grid <= 0) return cudaSuccess;
  if (fp8 && !tmapA32) return cudaErrorInvalidValue;
  CUtensorMap a, b, a32, o;
  memcpy(&a, tmapA, sizeof(a));
  memcpy(&b, tmapB, sizeof(b));
  memcpy(&a32, fp8 ? tmapA32 : tmapA, sizeof(a32));
  memcpy(&o, p.tma_out ? tmapOut : tmapA, sizeof(o));
  const bool pdl = p.pdl != 0;
  cudaError_t e;
  if (fp4)
    e = launch_ex(tc_gemm_kernel<false, kNvf4>, dim3(grid), dim3(Cfg<kNvf4>::NUM_THREADS),
                  smem_bytes<kNvf4>(p.tma_out != 0), s, pdl, a, b, a32, o, p);
  else if (fp8)
    e = launch_ex(tc_gemm_kernel<false, kE4m3>, dim3(grid), dim3(Cfg<kE4m3>::NUM_THREADS),
                  smem_bytes<kE4m3>(p.tma_out != 0), s, pdl, a, b, a32, o, p);
  else if (bwd)  // with the staging buffers (row-coalesced epilogue stores)
    e = launch_ex(tc_gemm_kernel<true, kBf16>, dim3(grid), dim3(Cfg<kBf16>::NUM_THREADS),
                  smem_bytes<kBf16>(true), s, pdl, a, b, a32, o, p);
  else
    e = launch_ex(tc_gemm_kernel<false, kBf16>, dim3(grid), dim3(Cfg<kBf16>::NUM_THREADS),
                  smem_bytes<kBf16>(p.tma_out != 0), s, pdl, a, b, a32, o, p);
  return e != cudaSuccess ? e : cudaGetLastError();
}

cudaError_t launch_tc_gemm_pair(const void *tmapA, const void *tmapB2, const TcParams &p,
                                int max_pairs, cudaStream_t s, const void *tmapOut) {
  static int attr_dev = -1, dev_pairs = 0;
  int dev = 0;
  cudaGetDevice(&dev);
  if (attr_dev != dev) {
    cudaError_t e = cudaFuncSetAttribute(tc_pair_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(pair_smem_bytes(true)));
    if (e != cudaSuccess) return e;
    // pairs resident at once (one CTA per SM; a GPC with an odd number of
    // free SMs leaves one idle)
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(2, 1, 1);
    cfg.blockDim = dim3(Cfg<kBf16>::NUM_THREADS, 1, 1);
    cfg.dynamicSmemBytes = pair_smem_bytes(true);
    int n = 0;
    e = cudaOccupancyMaxActiveClusters(&n, tc_pair_kernel, &cfg);
    if (e != cudaSuccess) return e;
    if (n <= 0) return cudaErrorInvalidConfiguration;
    dev_pairs = n;
    attr_dev = dev;
  }
  const bool bwd = p.mode == TC_WGRAD || p.raw || p.out_f32 || p.out_h;
  if (bwd || p.b_scale || (p.tma_out && !tmapOut)) return cudaErrorInvalidValue;
  if (p.Kdim % TKB || p.Kdim <= 0 || p.n_tiles_n <= 0) return cudaErrorInvalidValue;
  if (p.k_split > 1 && !split_ok(p, TKB)) return cudaErrorInvalidValue;
  const int pairs = max_pairs < dev_pairs ? max_pairs : dev_pairs;
  if (pairs <= 0) return cudaSuccess;
  CUtensorMap a, b, o;
  memcpy(&a, tmapA, sizeof(a));
  memcpy(&b, tmapB2, sizeof(b));
  memcpy(&o, p.tma_out ? tmapOut : tmapA, sizeof(o));
  const cudaError_t e =
      launch_ex(tc_pair_kernel, dim3(2 * pairs), dim3(Cfg<kBf16>::NUM_THREADS),
                pair_smem_bytes(p.tma_out != 0), s, p.pdl != 0, a, b, o, p);
  return e != cudaSuccess ? e : cudaGetLastError();
}

cudaError_t launch_wait_selftest(int32_t *status, long long limit_ns, cudaStream_t s) {
  if (limit_ns <= 0 || limit_ns > static_cast<long long>(kWaitLimitNs)) return cudaErrorInvalidValue;
  wait_selftest_kernel<<<1, 32, 0, s>>>(status, static_cast<unsigned long long>(limit_ns));
  return cudaGetLastError();
}

}  // namespace lmoe

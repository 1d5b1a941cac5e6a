// kernels.h -- host-side launchers of the LatentMoE kernels (internal).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace lmoe {

// Rows of one grouped-GEMM M-tile: expert `expert`, permuted rows
// [row0, min(row0 + tile_m, row_end)).
struct TileEntry {
  int32_t row0, row_end, expert, pad;
};

// Segment padding of the dispatch order: pad > 1 starts each expert's rows at
// a multiple of pad (offsets are the padded starts, offsets[N] the padded
// total, ends[e] the end of expert e's real rows); pad == 1: no padding.
struct SegPad {
  int pad;
  int32_t *ends;
};
constexpr SegPad kNoPad = {1, nullptr};

// ---- routing (route_kernels.cu)
// ids/gates from fp32 logits [T][ld] (+ bias [N]); one warp per token.  If
// counts is non-null the
// kernel also accumulates the dispatch's per-chunk expert histogram (zeroed
// beforehand, dispatch_count_elems(T, chunk, N) ints).
cudaError_t launch_topk(const float *logits, int ld, const float *bias, int T, int N, int K,
                        int32_t *ids, float *gates, int32_t *counts, int chunk, cudaStream_t s);

// Tokens per dispatch chunk on the forward path (the two-launch routing, and
// the four-launch one), and the chunk count.
constexpr int kFusedChunk = 32;
constexpr int kDispatchChunk = 64;
inline int dispatch_chunks(int T, int chunk) { return (T + chunk - 1) / chunk; }
// Elements of the [N][chunks] count matrix (rows padded to a multiple of 4).
inline size_t dispatch_count_elems(int T, int chunk, int N) {
  return static_cast<size_t>((dispatch_chunks(T, chunk) + 3) & ~3) * N;
}

// Histogram (unless counts_ready) -> exclusive scan -> stable scatter.  The
// count matrix chunk_counts holds dispatch_count_elems(T, chunk, N) ints
// (chunk: a multiple of 32, at most 256).  Writes offsets [N+1], perm / pos /
// row_expert [T*K], and the M-tile table (tile_m rows per tile; capacity
// max_tiles entries) plus its length in *n_tiles; with tiles2, also a second
// table of tile_m2-row M-tiles (capacity max_tiles2) and its length.
// check_ids (ids from a caller rather than the top-K kernel): pairs whose id
// lies outside [0, N) are skipped -- not counted, not placed -- so that no
// kernel indexes memory with them; without it every id must be in range.
cudaError_t launch_dispatch(const int32_t *ids, int T, int K, int N, int32_t *chunk_counts,
                            int chunk, bool counts_ready, int32_t *offsets, int32_t *perm,
                            int32_t *pos, int32_t *row_expert, TileEntry *tiles,
                            int32_t *n_tiles, int tile_m, int max_tiles, cudaStream_t s,
                            TileEntry *tiles2 = nullptr, int32_t *n_tiles2 = nullptr,
                            int tile_m2 = 0, int max_tiles2 = 0, bool check_ids = false,
                            SegPad seg = kNoPad);

// Expert parallelism, receiving side.  recv_counts [W][NL]: rows that source
// rank s sent for local expert e; the received rows lie source-major and,
// within a source, expert-grouped in expert order.  Writes the M-tile tables
// (tile_m and tile_m2 rows per tile, entries ordered by expert, then source,
// so that tiles sharing an expert's weights run together) and their lengths.
// Row ranges are clipped at R (the rows actually received).  W * NL <= 65536,
// NL <= 1024.
cudaError_t launch_ep_tiles(const int32_t *recv_counts, int W, int NL, int R, TileEntry *tiles,
                            int32_t *n_tiles, int tile_m, int max_tiles, TileEntry *tiles2,
                            int32_t *n_tiles2, int tile_m2, int max_tiles2, cudaStream_t s);

// counts[e] = offsets[e+1] - offsets[e] for e < N.
cudaError_t launch_counts_from_offsets(const int32_t *offsets, int N, int32_t *counts,
                                       cudaStream_t s);

// Routing and dispatch in two launches.  launch_route_select: top-K' with
// the per-chunk histogram and, in the grid's last block, the scan (outputs of
// launch_topk + the offsets and tile tables of launch_dispatch); counts holds
// dispatch_count_elems(T, chunk, N) ints and needs no clearing; arrivals is
// one int, zero before the first launch and left zero by each.
// launch_scatter_permute: the stable scatter (perm, pos, row_expert) and,
// when src is given, the row permutation dst[p] = src[perm[p] / K] (rows of
// row_bytes, a multiple of 16), with `shares` blocks per chunk splitting the
// copies.  Valid when fused_route_ok(N, K, chunk).
bool fused_route_ok(int N, int K, int chunk);
cudaError_t launch_route_select(const float *logits, int ld, const float *bias, int T, int N,
                                int K, int32_t *ids, float *gates, int32_t *counts, int chunk,
                                int32_t *arrivals, int32_t *offsets, TileEntry *tiles,
                                int32_t *n_tiles, int tile_m, int max_tiles, TileEntry *tiles2,
                                int32_t *n_tiles2, int tile_m2, int max_tiles2, cudaStream_t s,
                                bool pdl = false, SegPad seg = kNoPad);
cudaError_t launch_scatter_permute(const int32_t *ids, int T, int K, int N, const int32_t *counts,
                                   int chunk, const int32_t *offsets, int32_t *perm, int32_t *pos,
                                   int32_t *row_expert, const void *src, int row_bytes, void *dst,
                                   int shares, cudaStream_t s, bool pdl = false);

// dst[p][:] = src[perm[p] / K][:], rows of `row_bytes` (multiple of 16).
cudaError_t launch_permute_rows(const void *src, const int32_t *perm, int K, int rows,
                                int row_bytes, void *dst, cudaStream_t s);

// u[t][0:l] (row stride ldu) = sum_k gates[t][k] * O[pos[t*K+k]][0:l] in slot
// order, fp32 accumulation; element type bf16 (is_bf16) or f32.
cudaError_t launch_combine(const void *O, const int32_t *pos, const float *gates, int T, int K,
                           int l, void *u, int ldu, bool is_bf16, cudaStream_t s,
                           bool pdl = false);

// ---- fp32 CUDA-core path (simt_kernels.cu)
cudaError_t simt_linear(const float *A, int lda, const float *B, int ldb, float *C, int ldc,
                        int M, int N, int Kdim, cudaStream_t s);
// H[r][c] = silu(A_r . Wg[e][c%mw]) * (A_r . Wu[e][c%mw]) for c < Ncols, where
// e = row_expert[r] if row_expert else c / mw; Wg/Wu are [*][mw][Kdim].
cudaError_t simt_swiglu(const float *A, int lda, const float *Wg, const float *Wu, int mw,
                        const int32_t *row_expert, float *H, int ldh, int M, int Ncols, int Kdim,
                        cudaStream_t s);
// H[r][c] = relu(A_r . Wu[e][c%mw])^2 (squared-ReLU experts), e as above.
cudaError_t simt_relu2(const float *A, int lda, const float *Wu, int mw,
                       const int32_t *row_expert, float *H, int ldh, int M, int Ncols, int Kdim,
                       cudaStream_t s);
// O[r][c] = H_r . Wo[row_expert[r]][c]   (Wo [*][Ncols][Kdim])
cudaError_t simt_expert_down(const float *H, int ldh, const float *Wo,
                             const int32_t *row_expert, float *O, int ldo, int M, int Ncols,
                             int Kdim, cudaStream_t s);

// ---- bf16 tcgen05 GEMMs (tc_gemm.cu)
enum TcMode : int {
  TC_X_FUSED = 0,   // x [T][d] x W_x: router logits | z | shared SwiGLU hidden
  TC_EXPERT_GU = 1, // grouped: permuted z x W_gu[e] -> SwiGLU -> H
  TC_EXPERT_DOWN = 2,  // grouped: H x W_o[e] -> O (bf16)
  TC_OUT = 3,       // [u | shared hidden] x W_y -> y (bf16)
  TC_WGRAD = 4,     // weight gradients: dW[g] = A^T B over token-major K ranges (fp32)
};

// TC_WGRAD destinations (fp32, the caller's gradient layouts).
enum WgKind {
  WG_Y = 0,   // rows d, cols l + n_s m_s: [dW_up | dS_o(0) | dS_o(1) ...]
  WG_X = 1,   // rows = W_x rows (router | W_down | shared gate/up), cols d
  WG_O = 2,   // per expert: rows l, cols m -> dW_o[e]
  WG_GU = 3,  // per expert: rows = W_gu rows (gate/up interleaved by 128), cols l
};

struct TcParams {
  int mode;
  int M;               // dense: rows (T); grouped: unused (tile table)
  int Kdim;            // reduction length, multiple of 64
  int n_tiles_n;       // N-tiles of 256 columns in this launch
  int n_tile_base;     // dense modes: first N-tile (a launch may cover a column range)
  const TileEntry *tiles;   // grouped modes: the M-tile table (128-row tiles for
                            // launch_tc_gemm, 256-row tiles for launch_tc_gemm_pair)
  const int32_t *n_mtiles;  // grouped modes: device count of M-tiles
  int b_rows_per_expert;    // unused (B is K-block tiled: see launch_repack_btiles)
  // TC_X_FUSED column regions (multiples of 256): [0, r_end) router logits,
  // [r_end, z_end) z, [z_end, ...) shared gate/up interleaved in blocks of 128.
  int r_end, z_end, n_routed, l;
  float *logits; int ld_logits;
  __nv_bfloat16 *z; int ld_z;
  __nv_bfloat16 *out; int ld_out;   // H, O, y, or Ucat (+ column offset for shared)
  int out_col0;
  int relu2;           // squared-ReLU experts: TC_EXPERT_GU and the shared
                       // region of TC_X_FUSED write relu(acc)^2 (no gate/up
                       // interleave); n_cols2 bounds their output columns
  int n_cols2;
  // Backward-only options (all zero in the forward):
  int raw;             // TC_EXPERT_GU and the shared region of TC_X_FUSED write
                       // the accumulator as is (bf16 gate/up pre-activations)
  __nv_bfloat16 *out2; int ld_out2;  // TC_X_FUSED shared region, with raw
  float *out_f32;      // TC_OUT / TC_EXPERT_DOWN: fp32 output [rows][ld_out]
  __nv_bfloat16 *out_h; int ld_h;  // TC_EXPERT_GU with raw: the hidden h as well
  // E4M3 operands (TC_EXPERT_GU / TC_EXPERT_DOWN with b_scale set): A is
  // E4M3 [rows][Kdim] with one scale per row in a_scale, B is the E4M3 weight
  // tiled in 256-row x 128-byte blocks (launch_quantize_e4m3_tiles) and
  // b_scale [expert][b_scale_ld] holds each weight row's scale; the MMA is
  // kind::f8f6f4 over 128-element K-blocks.
  const float *a_scale;
  const float *b_scale; int b_scale_ld;
  // NVFP4 operands (a_sf and b_sf set as well as the row scales): A is packed
  // E2M1 [rows][Kdim / 2], B the packed weight tiled in 256-row x 128-byte
  // blocks (launch_quantize_nvfp4_tiles); a_sf holds the E4M3 block scales of
  // A by M-tile of the tile table and K-block (2 KB each), b_sf those of B by
  // expert, N-tile and K-block (4 KB each), in the layout the MMA reads from
  // TMEM (see launch_quantize_nvfp4_tiles); the MMA is kind::mxf4nvf4 over
  // 256-element K-blocks.
  const uint8_t *a_sf, *b_sf;
  // TC_WGRAD: dW = A^T B with A [tokens][M] and B [tokens][N] the token-major
  // (row-major, tokens on rows) matrices themselves, read MN-major through
  // {64, 64} boxes; group g reduces over token rows [k_start[g], k_start[g] +
  // k_len[g]) (multiples of 64; k_len null: up to k_start[g + 1]; dense:
  // k_start null and rows [0, Kdim), rows past the maps' end read as zero);
  // n_tiles_n counts 256-column tiles of B.
  int wg_kind, groups;
  const int32_t *k_start, *k_len;
  int wg_d, wg_l, wg_m, wg_ns, wg_ms, wg_n, wg_npad, wg_lpad;  // layer sizes for the destinations
  float *g_router, *g_down, *g_up, *g_gate, *g_upx, *g_out, *g_sgate, *g_sup, *g_sout;
  // Forward bf16 outputs (z, H, O, y; not the fp32 router logits): with
  // tma_out set, an epilogue warp whose 32 rows are all valid stages each
  // 32 x 32 block in shared memory and writes it with one TMA store through
  // the launch's output tensor map (launch_tc_gemm's tmapOut); other warps
  // store directly.
  int tma_out;
  // Launch with programmatic stream serialization (the kernel may start while
  // the previous kernel of the stream drains; it waits for it before touching
  // global memory).  Only for a launch that directly follows another kernel
  // on the same stream.
  int pdl;
  int32_t *status;
  // Split reduction (dense pair launches only: TC_OUT, and TC_X_FUSED over the
  // router and z columns): k_split > 1 cuts the K-blocks into k_split slices of
  // consecutive K-blocks, each tile-slice a work item of its own, so that a
  // launch with few output tiles still fills the GPU.  Each item writes its
  // fp32 partial to part [k_split][M][n_tiles_n * 256]; launch_splitk_reduce
  // then sums the slices in slice order and applies the mode's output step.
  int k_split;         // at most kMaxKSplit
  float *part;
};
constexpr int kMaxKSplit = 16;

// The output step of a split launch: out = sum over slices of p.part, in
// slice order (fp32), then by mode: TC_OUT bf16 y; TC_X_FUSED fp32 router
// logits and bf16 z.  pdl: launched right after the split GEMM on s.
cudaError_t launch_splitk_reduce(const TcParams &p, cudaStream_t s, bool pdl);

// B operands of the tcgen05 GEMMs are stored K-block tiled: for each group
// (expert, or the whole matrix), N-tile n of 256 rows and K-block kb of 64
// columns, one contiguous 256 x 64 bf16 block (32 KB), so that every TMA
// load of B reads one contiguous range.  Rows past rows_per_group are zero.
// src: [groups][rows_per_group][cols] row-major; dst holds
// groups * ceil(rows_per_group/256) * (cols/64) blocks.
inline int64_t btile_rows(int groups, int rows_per_group, int cols) {
  return static_cast<int64_t>(groups) * ((rows_per_group + 255) / 256) * (cols / 64) * 256;
}
cudaError_t launch_repack_btiles(const __nv_bfloat16 *src, int groups, int rows_per_group,
                                 int cols, __nv_bfloat16 *dst, cudaStream_t s);

// E4M3 expert weights (fp8_weights.cu): src [groups][rows][cols] bf16 ->
// per-row power-of-two scales [groups][rows] and E4M3 codes stored in blocks
// of 256 rows x 128 bytes (per group, 256-row tile n and 128-column block kb:
// one contiguous block; padding rows zero).  cols % 128 == 0.  The same byte
// count as btile_rows(groups, rows_per_group, cols) * 64.
cudaError_t launch_quantize_e4m3_tiles(const __nv_bfloat16 *src, int groups, int rows_per_group,
                                       int cols, float *scales, uint8_t *dst, cudaStream_t s);

// E4M3 activations: row r of dst [rows][cols] (bytes) and scales[r] from the
// bf16 row src[gather ? gather[r] / K : r] (row stride cols): the smallest
// power-of-two scale with max |row| <= 448 scale, then each element's E4M3
// code, rounded to nearest even and saturating (the weights' rule).  One warp
// per row.  cols % 8 == 0.
cudaError_t launch_quantize_rows_e4m3(const __nv_bfloat16 *src, const int32_t *gather, int K,
                                      int rows, int cols, uint8_t *dst, float *scales,
                                      cudaStream_t s, bool pdl = false);

// NVFP4 expert weights (fp4_quant.cu): src [groups][rows_per_group][cols]
// bf16 -> packed E2M1 codes in 256-row x 128-byte blocks per (group, 256-row
// tile, 256-element K-block), E4M3 block scales in 4 KB per such block (two
// 128-row halves x four 64-element slices x one 512-byte atom: row r0 + 32 r1
// at bytes 16 r0 + 4 r1 .. + 3), and the power-of-two row scales [groups]
// [rows_per_group].  Padding rows, columns and scales are zero.  cols % 32 == 0.
size_t nvfp4_weight_code_bytes(int groups, int rows_per_group, int cols);
size_t nvfp4_weight_sf_bytes(int groups, int rows_per_group, int cols);
cudaError_t launch_quantize_nvfp4_tiles(const __nv_bfloat16 *src, int groups, int rows_per_group,
                                        int cols, float *scales, uint8_t *codes, uint8_t *sf,
                                        cudaStream_t s);

// NVFP4 activations, one block per M-tile of the table (tiles, device count
// n_tiles, grid max_tiles): tile row p reads the bf16 row src[gather ?
// gather[p] / K : p] (row stride cols) and writes the packed codes row p of
// codes [rows][cols / 2], scales[p] and, per K-block, the tile's four 512-byte
// block-scale atoms (sf: nvfp4_act_sf_bytes(max_tiles, cols) bytes; scales of
// blocks past cols are zero; the atoms' rows past the tile's expert are not
// written).
size_t nvfp4_act_sf_bytes(int max_tiles, int cols);
cudaError_t launch_quantize_act_nvfp4(const __nv_bfloat16 *src, const int32_t *gather, int K,
                                      const TileEntry *tiles, const int32_t *n_tiles,
                                      int max_tiles, int cols, uint8_t *codes, float *scales,
                                      uint8_t *sf, cudaStream_t s, bool pdl = false);

// Encodes a 2-D byte tensor map (rows x cols bytes, row stride in bytes)
// with a {128, box_rows} box and 128-byte swizzle (E4M3 GEMM operands).
// Host only.
int make_tmap_u8(void *tmap_out, const void *base, int64_t rows, int64_t cols,
                 int64_t row_stride_bytes, int box_rows);

// Encodes a 2-D bf16 K-major tensor map (rows x cols, row stride in
// elements) with a {64, box_rows} box and 128-byte swizzle.  Host only.
int make_tmap_bf16(void *tmap_out /*CUtensorMap, 64 B*/, const void *base, int64_t rows,
                   int64_t cols, int64_t row_stride_elems, int box_rows);

// Encodes a 2-D bf16 tensor map of an output matrix (rows x cols, row stride
// in elements) with a {32, 32} box and 64-byte swizzle, for the GEMM
// epilogue's TMA stores.  Host only.
int make_tmap_bf16_out(void *tmap_out /*CUtensorMap, 64 B*/, const void *base, int64_t rows,
                       int64_t cols, int64_t row_stride_elems);

// ---- backward (backward_kernels.cu)
// fp32 CUDA-core GEMM with arbitrary strides: C[g](i, j) (+)= sum_k
// A[g](i, k) B[g](j, k), X[g](r, k) at X + g*sX_g + r*sX_r + k*sX_k; k runs
// over [0, K), or over [k_off[g], k_off[g+1]) when k_off (device) is set.
struct SimtGemm {
  const float *A; long long sA_g, sA_r, sA_k;
  const float *B; long long sB_g, sB_r, sB_k;
  float *C; long long sC_g, ldc;
  int M, N, K;
  const int32_t *k_off;
  int accumulate;
};
cudaError_t simt_gemm(const SimtGemm &g, int groups, cudaStream_t s);
// C[r][c] (+)= sum_k A[r][k] W[e*sW_e + c*sW_r + k*sW_k], e = row_expert[r].
cudaError_t simt_rowexpert(const float *A, int lda, const float *W, long long sW_e, long long sW_r,
                           long long sW_k, const int32_t *row_expert, float *C, int ldc, int M,
                           int Ncols, int Kdim, bool accumulate, cudaStream_t s);
// From pre-activations a (gate; unused for squared ReLU), b (up) and the
// hidden gradient dh (may be null: h only): h, da, db (each may be null).
template <typename TI, typename TO>
cudaError_t launch_act_backward(const TI *a, const TI *b, int ldab, const float *dh, int lddh,
                                TO *h, int ldh, TO *da, TO *db, int ldd, int rows, int n,
                                bool relu2, cudaStream_t s);
// Per token: ds[t][k] = g_k (du_t . O[pos] - sum_j g_j du_t . O[pos_j]) and
// DO[pos(t,k)] = g_k du_t.
template <typename TO>
cudaError_t launch_slot_grad(const float *du, int lddu, const TO *O, int l, const int32_t *pos,
                             const float *gates, int T, int K, float *ds, TO *DO, cudaStream_t s);
// out[t][:n] = sum_k D[pos(t,k)][:n], slot order.
template <typename TI, typename TO>
cudaError_t launch_gather_sum(const TI *D, int ldD, const int32_t *pos, int T, int K, int n, TO *out,
                              int ldo, cudaStream_t s);
// out[t][e] = ds of the slot that selected e, 0 for unselected e (e < N).
template <typename TO>
cudaError_t launch_scatter_ds(const float *ds, const int32_t *ids, int T, int K, int N, TO *out,
                              int ldo, cudaStream_t s);
// db[e] = sum of ds over expert e's pairs, token order.
cudaError_t launch_bias_grad(const float *ds, const int32_t *offsets, const int32_t *perm, int N,
                             float *db, cudaStream_t s);

// Zeroes the padding rows [ends[e], offsets[e + 1]) of every expert (a padded
// dispatch order, see SegPad) in up to four bf16 row-major matrices ptr[i]
// with cols[i] columns (a multiple of 8); null entries are skipped.
struct PadRowsArgs {
  void *ptr[4];
  int cols[4];
};
cudaError_t launch_zero_pad_rows(const int32_t *offsets, const int32_t *ends, int N,
                                 const PadRowsArgs &a, cudaStream_t s);

// bf16: gate/up pre-activations AB [rows][ldab] in the GEMM's 128-interleaved
// layout (squared ReLU: plain up) and the hidden gradient dh [rows][lddh]
// (TD = float or bf16) -> dAB [rows][lddab] in the same layout; n hidden
// units per row (n, ldab, lddh, lddab multiples of 8).
template <typename TD>
cudaError_t launch_act_backward_rows(const __nv_bfloat16 *AB, int ldab, const TD *dh, int lddh,
                                     __nv_bfloat16 *dAB, int lddab, int rows, int n, bool relu2,
                                     cudaStream_t s);
// dst[c][col(r)] = src[r][c]; col(r) = r, or r + shift[row_expert[r]];
// `batch` independent matrices, src / dst advanced by src_batch / dst_batch.
cudaError_t launch_transpose_bf16(const __nv_bfloat16 *src, int lds, int R, int C,
                                  const int32_t *row_expert, const int32_t *shift,
                                  __nv_bfloat16 *dst, long long ldd, cudaStream_t s,
                                  int batch = 1, long long src_batch = 0,
                                  long long dst_batch = 0);
// Failure-detection self-test (see lmoe_selftest_wait_timeout).
cudaError_t launch_wait_selftest(int32_t *status, long long limit_ns, cudaStream_t s);

// tmapA32: with E4M3 operands (p.b_scale set), the same A matrix with a
// {128, 32} box, used for tiles of at most 32 token rows.
// tmapOut: with p.tma_out set (forward bf16 modes only), the bf16 output
// matrix's map from make_tmap_bf16_out (z for TC_X_FUSED).
cudaError_t launch_tc_gemm(const void *tmapA, const void *tmapB, const TcParams &p,
                           int num_sms, int max_ctas, cudaStream_t s,
                           const void *tmapA32 = nullptr, const void *tmapOut = nullptr);

// The forward's bf16 GEMMs (TC_X_FUSED, TC_EXPERT_GU, TC_EXPERT_DOWN, TC_OUT;
// bf16 weights, no backward options) on CTA pairs: 256 x 256 output tiles,
// tcgen05.mma.cta_group::2.  tmapA: A with a {64, 128} box (as for
// launch_tc_gemm); tmapB2: the K-block-tiled B with a {64, 128} box (each CTA
// loads half of a 256-row block); grouped modes read 256-row M-tiles
// (p.tiles / p.n_mtiles from launch_dispatch's second table).  At most
// max_pairs clusters of two CTAs are launched.
cudaError_t launch_tc_gemm_pair(const void *tmapA, const void *tmapB2, const TcParams &p,
                                int max_pairs, cudaStream_t s, const void *tmapOut = nullptr);

}  // namespace lmoe

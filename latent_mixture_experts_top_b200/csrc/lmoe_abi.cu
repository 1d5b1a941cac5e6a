// lmoe_abi.cu -- the C ABI declared in include/lmoe.h.
//
// One handle = one LatentMoE layer on one device: validated hyper-parameters
// (Latent-MoE README, "Usage": d, m, n_experts, top_k, alpha, n_shared,
// variant), repacked weight copies, a workspace sized for max_tokens, and the
// TMA tensor maps of every operand whose address is fixed.  lmoe_forward
// enqueues the whole layer on the caller's stream without allocating or
// synchronising.
#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#include <algorithm>
#include <new>

#include "../../include/lmoe.h"
#include "kernels.h"

using namespace lmoe;

namespace {

constexpr int kTileM = 128;   // grouped-GEMM M-tile (tcgen05 M)
constexpr int kTileN = 256;   // tcgen05 N per tile

struct alignas(64) TensorMap64 {
  unsigned char bytes[128];   // CUtensorMap is 128 bytes, 64-byte aligned
};

struct Workspace {
  float *logits = nullptr;
  int32_t *ids = nullptr;
  float *gates = nullptr;
  int32_t *chunk_counts = nullptr;
  int32_t *offsets = nullptr;
  int32_t *perm = nullptr, *pos = nullptr, *row_expert = nullptr;
  TileEntry *tiles = nullptr;     // 128-row M-tiles (single-CTA GEMMs)
  int32_t *n_tiles = nullptr;
  TileEntry *tiles2 = nullptr;    // 256-row M-tiles (CTA-pair GEMMs)
  int32_t *n_tiles2 = nullptr;
  void *z = nullptr, *zp = nullptr, *H = nullptr, *O = nullptr, *ucat = nullptr;
  void *x_stage = nullptr, *y_stage = nullptr;
  void *x_stage2 = nullptr, *y_stage2 = nullptr;  // lmoe_forward_host_batches' second set
  int32_t *status = nullptr;
  int32_t *arrivals = nullptr;  // fused routing: the last-block counter (zero between launches)
  int32_t *seg_end = nullptr;   // training: the end of each expert's rows in the padded order
  float *part = nullptr;        // bf16: fp32 partials of split dense GEMMs (kPartFloats)
  // E4M3 / NVFP4 routed experts: the expert GEMMs' A operands with row scales
  uint8_t *zq = nullptr, *hq = nullptr;  // [TK][l], [TK][m] (NVFP4: packed, half the bytes)
  float *zq_scale = nullptr, *hq_scale = nullptr;  // [TK]
  uint8_t *zq_sf = nullptr, *hq_sf = nullptr;  // NVFP4 block scales, by M-tile and K-block
  // expert parallelism: M-tile tables of the received rows (128- and 256-row)
  TileEntry *ep_tiles = nullptr, *ep_tiles2 = nullptr;
  int32_t *ep_n_tiles = nullptr, *ep_n_tiles2 = nullptr;
};

// Backward workspace (handles created with training = 1), sized for Tmax.
struct BwdWorkspace {
  void *a = nullptr, *b = nullptr;      // [TK][m] expert pre-activations (gate, up)
  float *dU = nullptr;                  // [T][ky] dy . [W_up | S_o]
  float *ds = nullptr;                  // [TK] router-logit gradient per slot
  void *DO = nullptr;                   // [TK][l] expert-output gradient (permuted)
  float *dH = nullptr;  // fp32 [TK][m]; bf16 mode: the hidden gradient, bf16 [Kp][m]
  void *dA = nullptr, *dB = nullptr;    // [TK][m]
  float *dZp = nullptr;                 // [TK][l]
  float *dz = nullptr;                  // [T][l]
  void *as = nullptr, *bs = nullptr;    // [T][ns ms] shared pre-activations
  void *das = nullptr, *dbs = nullptr;  // [T][ns ms]
  float *dsfull = nullptr;              // [T][N']
  // bf16 mode only
  void *AB = nullptr;      // [TK][gu_rows] expert gate/up pre-activations (GEMM layout)
  void *ABs = nullptr;     // [T][sh_rows]  shared gate/up pre-activations (W_x layout)
  void *dAB = nullptr;     // [TK][gu_rows]
  void *dXcat = nullptr;   // [T][nx_rows] = [dS (router) | dz | shared dAB], W_x columns
  // Rows of the per-pair buffers in the backward's padded dispatch order
  // (each expert's rows start at a multiple of 64; see backward_bf16).
  int64_t Kp = 0;
};

}  // namespace

// lmoe_forward_host's pipeline: at most this many chunks, of at least this
// many tokens each
constexpr int kHostChunks = 4, kHostChunkTokens = 2048;
// Split reductions of the dense pair GEMMs (the x-GEMM's router and z columns,
// the output GEMM) when their output tiles fill fewer than half of the CTA
// pairs (few tokens): at most kMaxSplit slices of at least kMinSplitKb
// K-blocks each, the partials of one launch within kPartFloats.
constexpr int kMaxSplit = kMaxKSplit, kMinSplitKb = 4;
// The shared experts' gate/up GEMM overlaps the routing on a side stream when
// it takes at most this many K-block waves on its capped CTA pairs (README
// acc: 6 waves x 32 K-blocks; the prefill layer's 35 x 64 runs first instead).
constexpr int kSideKbWaves = 1024;
// Calls of at least this many tokens permute z with a positions-only scatter
// and a destination-major row copy instead of the scatter's own copy: beside
// the side-stream shared GEMM (README acc) the two launches end sooner; at
// decode the extra launch costs more than it saves.
constexpr int kRowCopyTokens = 1024;
constexpr size_t kPartFloats = static_cast<size_t>(96) * 256 * 256;  // 24 MiB

struct lmoe_layer {
  lmoe_config cfg;
  int d = 0, l = 0, m = 0, N = 0, K = 0, ns = 0, ms = 0, Tmax = 0;
  int bf16 = 0;
  int relu2 = 0;      // squared-ReLU experts (two matrices)
  int fp8 = 0;        // quantised routed experts (weights and the activations they multiply)
  int fp4 = 0;        // ... in NVFP4 (else E4M3)
  size_t esize = 4;
  int device = 0, num_sms = 0;
  bool loaded = false;
  int max_tiles = 0, max_tiles2 = 0;
  // Expert parallelism: ep_world ranks share the N routed experts; this
  // handle holds NE = N / ep_world of them (NE = N without it), experts
  // [ep_rank * NE, (ep_rank + 1) * NE).  R_max: rows lmoe_ep_experts may
  // receive (ep_world * Tmax * K); h_rows: rows of the H workspace.
  int ep_world = 1, ep_rank = 0, NE = 0;
  int ep_T = -1;  // tokens of the last lmoe_ep_dispatch (its combine must match)
  // Routing in two launches (top-K' + histogram + scan, then scatter + the
  // permutation of z) when the shapes allow; else four (see run_route).
  bool fused_route = false;
  int route_chunk = kDispatchChunk;  // tokens per dispatch chunk of the path taken
  int route_shares = 1;  // blocks per dispatch chunk that split the permutation copies
  int64_t R_max = 0, h_rows = 0;
  int max_tiles_ep = 0, max_tiles2_ep = 0;
  // bf16 layout of the stacked x-matrix: [W_r | pad][W_down | pad][shared rows | pad]
  int n_pad = 0, l_pad = 0, sh_rows = 0, nx_rows = 0;
  int gu_rows = 0;    // B rows per expert of the expert up GEMM: 2m (SwiGLU) or m
  int ky = 0;  // l + n_s * m_s, the reduction length of the last GEMM
  // weights (handle-owned)
  void *w_router = nullptr;  // f32 path: [N][d]
  float *b_router = nullptr;
  void *w_x = nullptr;       // bf16 path: [nx_rows][d]
  void *w_down = nullptr;    // f32 path: [l][d]
  void *w_gu = nullptr;      // bf16: [N][2m][l] interleaved by 128; f32: unused
  void *w_gate = nullptr, *w_upx = nullptr;  // f32 path: [N][m][l]
  void *w_out = nullptr;     // [N][l][m]
  void *s_gate = nullptr, *s_up = nullptr;   // f32 path: [ns][ms][d]
  void *w_y = nullptr;       // [d][l + ns ms] = [W_up | S_o(0) | S_o(1) ...]
  Workspace ws;
  BwdWorkspace bw;
  bool training = false;
  // profiling: a ring of event sets (LMOE_NUM_STAGES + 1 per forward)
  int prof_slots = 0;
  int64_t prof_count = 0;     // forwards recorded since profiling was enabled
  cudaEvent_t *ev = nullptr;  // [prof_slots][LMOE_NUM_STAGES + 1]
  int64_t launches = 0;
  // bf16: the shared experts' gate/up GEMM runs on a side stream, forked after
  // the router/down GEMM and joined before the output GEMM.
  cudaStream_t side = nullptr;
  cudaEvent_t ev_fork = nullptr, ev_join = nullptr;
  // lmoe_forward_host: copy streams and per-chunk events of its pipeline
  cudaStream_t h2d = nullptr, d2h = nullptr;
  cudaEvent_t ev_start = nullptr, ev_in[kHostChunks] = {}, ev_out[kHostChunks] = {};
  // lmoe_forward_host_batches, per staging set: forward done, copy out done
  cudaEvent_t ev_done[2] = {}, ev_yfree[2] = {};
  TensorMap64 tm_wx, tm_wgu, tm_wo, tm_wy, tm_zp, tm_h, tm_ucat;
  TensorMap64 tm_out_z, tm_out_h, tm_out_o;  // epilogue TMA stores: z, H, O
  // B operands of the CTA-pair GEMMs: the same tiled matrices, {64, 128} boxes
  TensorMap64 tm_wx2, tm_wo2, tm_wy2;
  TensorMap64 tm_zq, tm_zq32, tm_hq, tm_hq32;  // E4M3 activations ({128, 128}, {128, 32})
  // E4M3 / NVFP4 expert weights (256-row x 128-byte blocks) and their row
  // scales; NVFP4 block scales (4 KB per 256-row tile and K-block)
  uint8_t *w_gu8 = nullptr, *w_o8 = nullptr;
  float *gu_scale = nullptr, *o_scale = nullptr;
  uint8_t *gu_sf = nullptr, *o_sf = nullptr;
  // bf16 training: transposed weights (K-block tiled) and backward maps
  void *w_yT = nullptr;   // [ky][d]
  void *w_oT = nullptr;   // [N][m][l]
  void *w_guT = nullptr;  // [N][l][gu_rows]
  void *w_xT = nullptr;   // [d][nx_rows]
  TensorMap64 tm_wyT, tm_woT, tm_wguT, tm_wxT, tm_DO, tm_dAB, tm_dXcat;
  // weight-gradient operands read MN-major ({64, 64} boxes of the token-major
  // matrices in the padded order)
  TensorMap64 tm_DOmn, tm_Hmn, tm_dABmn, tm_zpmn;
  TensorMap64 tm_dH_out;  // the hidden gradient's store map (bf16 in the dH buffer)
};

namespace {

int cuda_err(cudaError_t e) { return e == cudaSuccess ? LMOE_OK : LMOE_ERR_CUDA; }

// Keeps the caller's current device and switches to the handle's.
struct DeviceGuard {
  int prev = -1;
  bool ok = true;
  explicit DeviceGuard(int dev) {
    if (cudaGetDevice(&prev) != cudaSuccess) { ok = false; return; }
    if (prev != dev && cudaSetDevice(dev) != cudaSuccess) ok = false;
  }
  ~DeviceGuard() {
    int cur = -1;
    if (prev >= 0 && cudaGetDevice(&cur) == cudaSuccess && cur != prev) cudaSetDevice(prev);
  }
};

template <typename T>
bool dalloc(T **p, size_t bytes) {
  if (bytes == 0) bytes = 16;
  return cudaMalloc(reinterpret_cast<void **>(p), bytes) == cudaSuccess;
}

void free_all(lmoe_layer *h) {
  void *ptrs[] = {h->w_router, h->b_router, h->w_x, h->w_down, h->w_gu, h->w_gate, h->w_upx,
                  h->w_out, h->s_gate, h->s_up, h->w_y, h->ws.logits, h->ws.ids, h->ws.gates,
                  h->ws.chunk_counts, h->ws.offsets, h->ws.perm, h->ws.pos, h->ws.row_expert,
                  h->ws.tiles, h->ws.n_tiles, h->ws.tiles2, h->ws.n_tiles2, h->ws.z, h->ws.zp, h->ws.H, h->ws.O, h->ws.ucat,
                  h->ws.x_stage, h->ws.y_stage, h->ws.x_stage2, h->ws.y_stage2, h->ws.status, h->bw.a, h->bw.b, h->bw.dU,
                  h->bw.ds, h->bw.DO, h->bw.dH, h->bw.dA, h->bw.dB, h->bw.dZp, h->bw.dz,
                  h->bw.as, h->bw.bs, h->bw.das, h->bw.dbs, h->bw.dsfull, h->bw.AB,
                  h->bw.ABs, h->bw.dAB, h->bw.dXcat, h->ws.seg_end,
                  h->w_yT, h->w_oT, h->w_guT, h->w_xT, h->w_gu8,
                  h->w_o8, h->gu_scale, h->o_scale, h->gu_sf, h->o_sf, h->ws.zq_sf, h->ws.hq_sf,
                  h->ws.ep_tiles, h->ws.ep_tiles2,
                  h->ws.ep_n_tiles, h->ws.ep_n_tiles2, h->ws.arrivals, h->ws.zq, h->ws.hq,
                  h->ws.zq_scale, h->ws.hq_scale, h->ws.part};
  for (void *p : ptrs)
    if (p) cudaFree(p);
  if (h->ev_fork) cudaEventDestroy(h->ev_fork);
  if (h->ev_join) cudaEventDestroy(h->ev_join);
  if (h->side) cudaStreamDestroy(h->side);
  h->ev_fork = h->ev_join = nullptr;
  h->side = nullptr;
  for (int i = 0; i < kHostChunks; ++i) {
    if (h->ev_in[i]) cudaEventDestroy(h->ev_in[i]);
    if (h->ev_out[i]) cudaEventDestroy(h->ev_out[i]);
    h->ev_in[i] = h->ev_out[i] = nullptr;
  }
  for (int i = 0; i < 2; ++i) {
    if (h->ev_done[i]) cudaEventDestroy(h->ev_done[i]);
    if (h->ev_yfree[i]) cudaEventDestroy(h->ev_yfree[i]);
    h->ev_done[i] = h->ev_yfree[i] = nullptr;
  }
  if (h->ev_start) cudaEventDestroy(h->ev_start);
  if (h->h2d) cudaStreamDestroy(h->h2d);
  if (h->d2h) cudaStreamDestroy(h->d2h);
  h->ev_start = nullptr;
  h->h2d = h->d2h = nullptr;
}

int validate(const lmoe_config *c, lmoe_layer *h) {
  if (c->d <= 0 || c->m <= 0 || c->alpha <= 0 || c->max_tokens <= 0 || c->n_shared < 0)
    return LMOE_ERR_INVALID_CONFIG;
  if (c->variant != LMOE_EFF && c->variant != LMOE_ACC) return LMOE_ERR_INVALID_CONFIG;
  if (c->dtype != LMOE_F32 && c->dtype != LMOE_BF16) return LMOE_ERR_INVALID_CONFIG;
  if (c->activation != LMOE_SWIGLU && c->activation != LMOE_RELU2) return LMOE_ERR_INVALID_CONFIG;
  if (c->d % c->alpha) return LMOE_ERR_INVALID_CONFIG;
  if (c->n_shared > 0 && c->m_shared <= 0) return LMOE_ERR_INVALID_CONFIG;
  const int64_t N = c->n_routed_override > 0 ? c->n_routed_override
                                             : static_cast<int64_t>(c->alpha) * c->n_experts;
  const int64_t K = c->top_k_override > 0
                        ? c->top_k_override
                        : (c->variant == LMOE_ACC ? static_cast<int64_t>(c->alpha) * c->top_k
                                                  : c->top_k);
  if (N < 1 || K < 1 || K > N) return LMOE_ERR_INVALID_CONFIG;
  if (N > 1024) return LMOE_ERR_UNSUPPORTED;
  const int W = c->ep_world > 1 ? c->ep_world : 1;
  if (c->ep_world < 0 || c->ep_rank < 0 || c->ep_rank >= W) return LMOE_ERR_INVALID_CONFIG;
  if (W > 1) {
    if (N % W) return LMOE_ERR_INVALID_CONFIG;
    if (c->dtype != LMOE_BF16 || c->weight_format != LMOE_WEIGHTS_BF16 || c->training)
      return LMOE_ERR_UNSUPPORTED;
  }
  h->ep_world = W;
  h->ep_rank = c->ep_rank;
  h->NE = static_cast<int>(N / W);
  h->d = c->d;
  h->l = c->d / c->alpha;
  h->m = c->m;
  h->N = static_cast<int>(N);
  h->K = static_cast<int>(K);
  h->ns = c->n_shared;
  h->ms = c->n_shared > 0 ? c->m_shared : 0;
  h->Tmax = c->max_tokens;
  h->bf16 = c->dtype == LMOE_BF16;
  h->relu2 = c->activation == LMOE_RELU2;
  if (c->weight_format != LMOE_WEIGHTS_BF16 && c->weight_format != LMOE_WEIGHTS_FP8 &&
      c->weight_format != LMOE_WEIGHTS_NVFP4)
    return LMOE_ERR_INVALID_CONFIG;
  h->fp8 = c->weight_format != LMOE_WEIGHTS_BF16;
  h->fp4 = c->weight_format == LMOE_WEIGHTS_NVFP4;
  if (h->fp8 && (c->dtype != LMOE_BF16 || c->training)) return LMOE_ERR_UNSUPPORTED;
  // E4M3 GEMMs run 128-element K-blocks: l and m must be multiples of 128
  // (NVFP4, 256-element K-blocks, reads a ragged last one as zeros)
  if (h->fp8 && ((c->d / c->alpha) % 128 || c->m % 128)) return LMOE_ERR_UNSUPPORTED;
  h->esize = h->bf16 ? 2 : 4;
  h->ky = h->l + h->ns * h->ms;
  if (static_cast<int64_t>(h->Tmax) * h->K * W > INT32_MAX / 2) return LMOE_ERR_UNSUPPORTED;
  h->R_max = W > 1 ? static_cast<int64_t>(W) * h->Tmax * h->K : 0;
  h->h_rows = std::max(static_cast<int64_t>(h->Tmax) * h->K, h->R_max);
  if (h->bf16) {
    const int mq = h->relu2 ? 64 : 128;  // SwiGLU tiles pair 128 gate with 128 up columns
    if (h->d % 64 || h->l % 64 || h->m % mq || (h->ns > 0 && h->ms % mq) || h->N % 32)
      return LMOE_ERR_UNSUPPORTED;
  } else {
    if (h->l % 4 || h->ky % 4) return LMOE_ERR_UNSUPPORTED;
  }
  return LMOE_OK;
}

int make_map(TensorMap64 *dst, const void *base, int64_t rows, int64_t cols, int64_t stride,
             int box_rows) {
  return make_tmap_bf16(dst->bytes, base, rows, cols, stride, box_rows) == 0 ? LMOE_OK
                                                                             : LMOE_ERR_CUDA;
}

// Device-to-device 2-D copy in elements of size es.
cudaError_t copy2d(void *dst, size_t dpitch_el, const void *src, size_t spitch_el,
                   size_t width_el, size_t height, size_t es, cudaStream_t s) {
  if (width_el == 0 || height == 0) return cudaSuccess;
  return cudaMemcpy2DAsync(dst, dpitch_el * es, src, spitch_el * es, width_el * es, height,
                           cudaMemcpyDeviceToDevice, s);
}

char *off(void *base, size_t elems, size_t es) { return static_cast<char *>(base) + elems * es; }

}  // namespace

extern "C" {

// The kernels move activations, weights and gradients with 16-byte vectors
// and TMA, so every such array must start on a 16-byte boundary; the calls
// check this before launching anything.
static bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

const char *lmoe_strerror(int code) {
  switch (code) {
    case LMOE_OK: return "ok";
    case LMOE_ERR_INVALID_CONFIG: return "invalid configuration or argument";
    case LMOE_ERR_NULL_ARG: return "required pointer is NULL";
    case LMOE_ERR_NOT_LOADED: return "weights not loaded";
    case LMOE_ERR_TOO_MANY_TOKENS: return "token count outside [0, max_tokens]";
    case LMOE_ERR_CUDA: return "CUDA call failed";
    case LMOE_ERR_DEVICE_TIMEOUT: return "a device-side bounded wait ran out";
    case LMOE_ERR_UNSUPPORTED: return "shape not supported by this build";
    case LMOE_ERR_OUT_OF_MEMORY: return "device allocation failed";
    case LMOE_ERR_MISALIGNED: return "device array not 16-byte aligned";
    default: return "unknown status";
  }
}

int lmoe_create(const lmoe_config *cfg, lmoe_handle *out) {
  if (!cfg || !out) return LMOE_ERR_NULL_ARG;
  *out = nullptr;
  lmoe_layer *h = new (std::nothrow) lmoe_layer();
  if (!h) return LMOE_ERR_OUT_OF_MEMORY;
  h->cfg = *cfg;
  int rc = validate(cfg, h);
  if (rc != LMOE_OK) { delete h; return rc; }
  if (cudaGetDevice(&h->device) != cudaSuccess ||
      cudaDeviceGetAttribute(&h->num_sms, cudaDevAttrMultiProcessorCount, h->device) !=
          cudaSuccess) {
    delete h;
    return LMOE_ERR_CUDA;
  }
  const size_t T = h->Tmax, TK = static_cast<size_t>(h->Tmax) * h->K, es = h->esize;
  const size_t N = h->N, d = h->d, l = h->l, m = h->m;
  // bf16 training handles: the per-pair buffers hold the backward's padded
  // dispatch order (each expert's rows start at a multiple of 64)
  const bool padded = cfg->training != 0 && h->bf16;
  h->bw.Kp = padded ? static_cast<int64_t>((TK + 63) / 64 * 64 + 64 * N) : 0;
  const size_t TKr = padded ? static_cast<size_t>(h->bw.Kp) : TK;
  if (padded) h->h_rows = std::max(h->h_rows, static_cast<int64_t>(TKr));
  h->max_tiles = static_cast<int>(TK / kTileM + N + 1);
  h->max_tiles2 = static_cast<int>(TK / (2 * kTileM) + N + 1);
  h->n_pad = (h->N + kTileN - 1) / kTileN * kTileN;
  h->l_pad = (h->l + kTileN - 1) / kTileN * kTileN;
  h->sh_rows = h->relu2 ? (h->ns * h->ms + kTileN - 1) / kTileN * kTileN : 2 * h->ns * h->ms;
  h->nx_rows = h->n_pad + h->l_pad + h->sh_rows;
  h->gu_rows = h->relu2 ? h->m : 2 * h->m;
  h->fused_route = fused_route_ok(h->N, h->K, kFusedChunk);
  h->route_chunk = h->fused_route ? kFusedChunk : kDispatchChunk;
  {  // blocks per chunk for the permutation copies: about four per SM in all
    const int nc = dispatch_chunks(h->Tmax, kFusedChunk);
    h->route_shares = std::max(1, std::min(64, (4 * h->num_sms + nc - 1) / nc));
  }
  Workspace &w = h->ws;
  bool ok = dalloc(&w.logits, T * N * 4) && dalloc(&w.ids, TK * 4) && dalloc(&w.gates, TK * 4) &&
            dalloc(&w.chunk_counts, dispatch_count_elems(h->Tmax, h->route_chunk, h->N) * 4) &&
            dalloc(&w.offsets, (N + 1) * 4) && dalloc(&w.perm, TKr * 4) &&
            dalloc(&w.pos, TK * 4) && dalloc(&w.row_expert, TKr * 4) &&
            dalloc(&w.tiles, static_cast<size_t>(h->max_tiles) * sizeof(TileEntry)) &&
            dalloc(&w.n_tiles, 16) &&
            dalloc(&w.tiles2, static_cast<size_t>(h->max_tiles2) * sizeof(TileEntry)) &&
            dalloc(&w.n_tiles2, 16) && dalloc(&w.z, T * l * es) && dalloc(&w.zp, TKr * l * es) &&
            dalloc(&w.H, static_cast<size_t>(h->h_rows) * m * es) && dalloc(&w.O, TKr * l * es) &&
            dalloc(&w.ucat, T * h->ky * es) && dalloc(&w.x_stage, T * d * es) &&
            dalloc(&w.y_stage, T * d * es) && dalloc(&w.x_stage2, T * d * es) &&
            dalloc(&w.y_stage2, T * d * es) && dalloc(&w.status, 16) && dalloc(&w.arrivals, 16);
  if (ok && h->bf16) ok = dalloc(&w.part, kPartFloats * 4);
  if (ok) {  // weights
    if (h->bf16) {
      // K-block-tiled B operands (see launch_repack_btiles)
      ok = dalloc(&h->w_x, btile_rows(1, h->nx_rows, h->d) * 64 * es) &&
           dalloc(&h->w_y, btile_rows(1, h->d, h->ky) * 64 * es);
      if (ok && h->fp4)
        ok = dalloc(&h->w_gu8, nvfp4_weight_code_bytes(h->N, h->gu_rows, h->l)) &&
             dalloc(&h->w_o8, nvfp4_weight_code_bytes(h->N, h->l, h->m)) &&
             dalloc(&h->gu_sf, nvfp4_weight_sf_bytes(h->N, h->gu_rows, h->l)) &&
             dalloc(&h->o_sf, nvfp4_weight_sf_bytes(h->N, h->l, h->m)) &&
             dalloc(&h->gu_scale, N * h->gu_rows * 4) && dalloc(&h->o_scale, N * l * 4) &&
             dalloc(&w.zq, TK * l / 2) && dalloc(&w.hq, TK * m / 2) &&
             dalloc(&w.zq_scale, TK * 4) && dalloc(&w.hq_scale, TK * 4) &&
             dalloc(&w.zq_sf, nvfp4_act_sf_bytes(h->max_tiles, h->l)) &&
             dalloc(&w.hq_sf, nvfp4_act_sf_bytes(h->max_tiles, h->m));
      else if (ok && h->fp8)
        ok = dalloc(&h->w_gu8, btile_rows(h->N, h->gu_rows, h->l) * 64) &&
             dalloc(&h->w_o8, btile_rows(h->N, h->l, h->m) * 64) &&
             dalloc(&h->gu_scale, N * h->gu_rows * 4) && dalloc(&h->o_scale, N * l * 4) &&
             dalloc(&w.zq, TK * l) && dalloc(&w.hq, TK * m) && dalloc(&w.zq_scale, TK * 4) &&
             dalloc(&w.hq_scale, TK * 4);
      else if (ok)
        ok = dalloc(&h->w_gu, btile_rows(h->NE, h->gu_rows, h->l) * 64 * es) &&
             dalloc(&h->w_out, btile_rows(h->NE, h->l, h->m) * 64 * es);
      if (ok && h->ep_world > 1) {
        h->max_tiles_ep = static_cast<int>(h->R_max / kTileM + static_cast<int64_t>(h->ep_world) * h->NE + 1);
        h->max_tiles2_ep =
            static_cast<int>(h->R_max / (2 * kTileM) + static_cast<int64_t>(h->ep_world) * h->NE + 1);
        ok = dalloc(&w.ep_tiles, static_cast<size_t>(h->max_tiles_ep) * sizeof(TileEntry)) &&
             dalloc(&w.ep_tiles2, static_cast<size_t>(h->max_tiles2_ep) * sizeof(TileEntry)) &&
             dalloc(&w.ep_n_tiles, 16) && dalloc(&w.ep_n_tiles2, 16);
      }
    } else {
      ok = dalloc(&h->w_router, N * d * es) && dalloc(&h->w_down, l * d * es) &&
           (h->relu2 || dalloc(&h->w_gate, N * m * l * es)) &&
           dalloc(&h->w_upx, N * m * l * es) && dalloc(&h->w_out, N * l * m * es) &&
           (h->relu2 || dalloc(&h->s_gate, static_cast<size_t>(h->ns) * h->ms * d * es)) &&
           dalloc(&h->s_up, static_cast<size_t>(h->ns) * h->ms * d * es) &&
           dalloc(&h->w_y, d * h->ky * es);
    }
    if (ok && cfg->has_router_bias) ok = dalloc(&h->b_router, N * 4);
  }
  h->training = cfg->training != 0;
  if (ok && h->training) {
    BwdWorkspace &b = h->bw;
    const size_t nsms = static_cast<size_t>(h->ns) * h->ms;
    ok = dalloc(&b.a, TK * m * es) && dalloc(&b.b, TK * m * es) &&
         dalloc(&b.dU, T * h->ky * 4) && dalloc(&b.ds, TK * 4) && dalloc(&b.DO, TKr * l * es) &&
         dalloc(&b.dH, std::max(TK * m * 4, TKr * m * 2)) && dalloc(&b.dA, TK * m * es) && dalloc(&b.dB, TK * m * es) &&
         dalloc(&b.dZp, TKr * l * 4) && dalloc(&b.dz, T * l * 4) && dalloc(&b.as, T * nsms * es) &&
         dalloc(&b.bs, T * nsms * es) && dalloc(&b.das, T * nsms * es) &&
         dalloc(&b.dbs, T * nsms * es) && dalloc(&b.dsfull, T * N * 4);
    if (ok && h->bf16) {
      const size_t gu = h->gu_rows, nx = h->nx_rows;
      ok = dalloc(&b.AB, TKr * gu * 2) && dalloc(&b.ABs, T * h->sh_rows * 2) &&
           dalloc(&b.dAB, TKr * gu * 2) && dalloc(&b.dXcat, T * nx * 2) &&
           dalloc(&w.seg_end, N * 4) &&
           dalloc(&h->w_yT, btile_rows(1, h->ky, h->d) * 64 * 2) &&
           dalloc(&h->w_oT, btile_rows(h->N, h->m, h->l) * 64 * 2) &&
           dalloc(&h->w_guT, btile_rows(h->N, h->l, h->gu_rows) * 64 * 2) &&
           dalloc(&h->w_xT, btile_rows(1, h->d, h->nx_rows) * 64 * 2);
    }
  }
  if (!ok) {
    cudaGetLastError();
    free_all(h);
    delete h;
    return LMOE_ERR_OUT_OF_MEMORY;
  }
  if (cudaMemset(w.status, 0, 16) != cudaSuccess || cudaMemset(w.n_tiles, 0, 16) != cudaSuccess ||
      cudaMemset(w.arrivals, 0, 16) != cudaSuccess ||
      cudaMemset(w.n_tiles2, 0, 16) != cudaSuccess ||
      cudaMemset(w.ucat, 0, T * h->ky * es) != cudaSuccess) {
    free_all(h);
    delete h;
    return LMOE_ERR_CUDA;
  }
  if (h->bf16) {
    rc = make_map(&h->tm_zp, w.zp, static_cast<int64_t>(TKr), h->l, h->l, kTileM);
    if (rc == LMOE_OK) rc = make_map(&h->tm_h, w.H, h->h_rows, h->m, h->m, kTileM);
    if (rc == LMOE_OK) rc = make_map(&h->tm_ucat, w.ucat, h->Tmax, h->ky, h->ky, kTileM);
    if (rc == LMOE_OK &&
        (make_tmap_bf16_out(h->tm_out_z.bytes, w.z, h->Tmax, h->l, h->l) != 0 ||
         make_tmap_bf16_out(h->tm_out_h.bytes, w.H, h->h_rows, h->m, h->m) != 0 ||
         make_tmap_bf16_out(h->tm_out_o.bytes, w.O, static_cast<int64_t>(TKr), h->l, h->l) != 0))
      rc = LMOE_ERR_CUDA;
    // B operands: [tiled rows][64], one {64, 256} box per K-block tile
    if (rc == LMOE_OK)
      rc = make_map(&h->tm_wx, h->w_x, btile_rows(1, h->nx_rows, h->d), 64, 64, kTileN);
    if (rc == LMOE_OK)
      rc = make_map(&h->tm_wx2, h->w_x, btile_rows(1, h->nx_rows, h->d), 64, 64, kTileN / 2);
    if (rc == LMOE_OK && h->fp8) {
      // E4M3 / NVFP4 operands, 128-byte swizzle: A rows {128, 128} (and
      // {128, 32} for tiles of at most 32 rows); the weights in 256-row x
      // 128-byte blocks.  NVFP4 rows hold half as many bytes.
      const int64_t gu8_rows = h->fp4 ? static_cast<int64_t>(
                                            nvfp4_weight_code_bytes(h->N, h->gu_rows, h->l) / 128)
                                      : btile_rows(h->N, h->gu_rows, h->l) / 2;
      const int64_t o8_rows = h->fp4 ? static_cast<int64_t>(
                                           nvfp4_weight_code_bytes(h->N, h->l, h->m) / 128)
                                     : btile_rows(h->N, h->l, h->m) / 2;
      const int lb = h->fp4 ? h->l / 2 : h->l, mb = h->fp4 ? h->m / 2 : h->m;  // row bytes
      if (make_tmap_u8(h->tm_zq.bytes, w.zq, static_cast<int64_t>(TK), lb, lb, kTileM) != 0 ||
          make_tmap_u8(h->tm_zq32.bytes, w.zq, static_cast<int64_t>(TK), lb, lb, 32) != 0 ||
          make_tmap_u8(h->tm_hq.bytes, w.hq, static_cast<int64_t>(TK), mb, mb, kTileM) != 0 ||
          make_tmap_u8(h->tm_hq32.bytes, w.hq, static_cast<int64_t>(TK), mb, mb, 32) != 0 ||
          make_tmap_u8(h->tm_wgu.bytes, h->w_gu8, gu8_rows, 128, 128, kTileN) != 0 ||
          make_tmap_u8(h->tm_wo.bytes, h->w_o8, o8_rows, 128, 128, kTileN) != 0)
        rc = LMOE_ERR_CUDA;
    } else {
      if (rc == LMOE_OK)
        rc = make_map(&h->tm_wgu, h->w_gu, btile_rows(h->NE, h->gu_rows, h->l), 64, 64, kTileN);
      if (rc == LMOE_OK)
        rc = make_map(&h->tm_wo, h->w_out, btile_rows(h->NE, h->l, h->m), 64, 64, kTileN);
      if (rc == LMOE_OK)
        rc = make_map(&h->tm_wo2, h->w_out, btile_rows(h->NE, h->l, h->m), 64, 64, kTileN / 2);
    }
    if (rc == LMOE_OK)
      rc = make_map(&h->tm_wy, h->w_y, btile_rows(1, h->d, h->ky), 64, 64, kTileN);
    if (rc == LMOE_OK)
      rc = make_map(&h->tm_wy2, h->w_y, btile_rows(1, h->d, h->ky), 64, 64, kTileN / 2);
    if (rc == LMOE_OK && h->training) {
      BwdWorkspace &b = h->bw;
      const int64_t rows = static_cast<int64_t>(TKr);
      const int gu = h->gu_rows, nx = h->nx_rows;
      // A operands of the K-major backward GEMMs ({64, 128} boxes)
      rc = make_map(&h->tm_DO, b.DO, rows, h->l, h->l, kTileM);
      if (rc == LMOE_OK) rc = make_map(&h->tm_dAB, b.dAB, rows, gu, gu, kTileM);
      if (rc == LMOE_OK) rc = make_map(&h->tm_dXcat, b.dXcat, h->Tmax, nx, nx, kTileM);
      // transposed weights, K-block tiled ({64, 256} boxes)
      if (rc == LMOE_OK) rc = make_map(&h->tm_wyT, h->w_yT, btile_rows(1, h->ky, h->d), 64, 64, kTileN);
      if (rc == LMOE_OK) rc = make_map(&h->tm_woT, h->w_oT, btile_rows(h->N, h->m, h->l), 64, 64, kTileN);
      if (rc == LMOE_OK)
        rc = make_map(&h->tm_wguT, h->w_guT, btile_rows(h->N, h->l, gu), 64, 64, kTileN);
      if (rc == LMOE_OK) rc = make_map(&h->tm_wxT, h->w_xT, btile_rows(1, h->d, nx), 64, 64, kTileN);
      // expert weight-gradient operands, read MN-major: {64, 64} boxes of the
      // token-major matrices (the dense ones' maps are made per call, with
      // exactly T rows)
      if (rc == LMOE_OK) rc = make_map(&h->tm_DOmn, b.DO, rows, h->l, h->l, 64);
      if (rc == LMOE_OK) rc = make_map(&h->tm_Hmn, w.H, rows, h->m, h->m, 64);
      if (rc == LMOE_OK) rc = make_map(&h->tm_dABmn, b.dAB, rows, gu, gu, 64);
      if (rc == LMOE_OK) rc = make_map(&h->tm_zpmn, w.zp, rows, h->l, h->l, 64);
      // bf16 mode keeps the hidden gradient dH in bf16 [rows][m] inside the
      // (fp32-sized) dH buffer
      if (rc == LMOE_OK && make_tmap_bf16_out(h->tm_dH_out.bytes, b.dH, rows, h->m, h->m) != 0)
        rc = LMOE_ERR_CUDA;
    }
    if (rc == LMOE_OK &&
        (cudaStreamCreateWithFlags(&h->side, cudaStreamNonBlocking) != cudaSuccess ||
         cudaEventCreateWithFlags(&h->ev_fork, cudaEventDisableTiming) != cudaSuccess ||
         cudaEventCreateWithFlags(&h->ev_join, cudaEventDisableTiming) != cudaSuccess))
      rc = LMOE_ERR_CUDA;
    if (rc != LMOE_OK) {
      free_all(h);
      delete h;
      return rc;
    }
  }
  bool st_ok = cudaStreamCreateWithFlags(&h->h2d, cudaStreamNonBlocking) == cudaSuccess &&
               cudaStreamCreateWithFlags(&h->d2h, cudaStreamNonBlocking) == cudaSuccess &&
               cudaEventCreateWithFlags(&h->ev_start, cudaEventDisableTiming) == cudaSuccess;
  for (int i = 0; st_ok && i < kHostChunks; ++i)
    st_ok = cudaEventCreateWithFlags(&h->ev_in[i], cudaEventDisableTiming) == cudaSuccess &&
            cudaEventCreateWithFlags(&h->ev_out[i], cudaEventDisableTiming) == cudaSuccess;
  for (int i = 0; st_ok && i < 2; ++i)
    st_ok = cudaEventCreateWithFlags(&h->ev_done[i], cudaEventDisableTiming) == cudaSuccess &&
            cudaEventCreateWithFlags(&h->ev_yfree[i], cudaEventDisableTiming) == cudaSuccess;
  if (!st_ok) {
    free_all(h);
    delete h;
    return LMOE_ERR_CUDA;
  }
  *out = h;
  return LMOE_OK;
}

int lmoe_load_weights(lmoe_handle h, const lmoe_weights *wt, void *stream) {
  if (!h || !wt) return LMOE_ERR_NULL_ARG;
  if (!wt->w_router || !wt->w_down || !wt->w_up || !wt->w_upx || !wt->w_out)
    return LMOE_ERR_NULL_ARG;
  if (!h->relu2 && !wt->w_gate) return LMOE_ERR_NULL_ARG;
  if (h->ns > 0 && (!wt->s_up || !wt->s_out || (!h->relu2 && !wt->s_gate)))
    return LMOE_ERR_NULL_ARG;
  if (h->cfg.has_router_bias && !wt->b_router) return LMOE_ERR_NULL_ARG;
  {
    const void *used[] = {wt->w_router, wt->w_down, wt->w_up, wt->w_upx, wt->w_out,
                          h->relu2 ? nullptr : wt->w_gate,
                          h->ns > 0 ? wt->s_up : nullptr, h->ns > 0 ? wt->s_out : nullptr,
                          (h->ns > 0 && !h->relu2) ? wt->s_gate : nullptr};
    for (const void *q : used)
      if (q && !aligned16(q)) return LMOE_ERR_MISALIGNED;
  }
  DeviceGuard g(h->device);
  if (!g.ok) return LMOE_ERR_CUDA;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const size_t es = h->esize, N = h->N, d = h->d, l = h->l, m = h->m, ns = h->ns, ms = h->ms;
  const size_t ky = h->ky;
  cudaError_t e = cudaSuccess;
  auto cp = [&](void *dst, const void *src, size_t bytes) {
    if (e == cudaSuccess && bytes) e = cudaMemcpyAsync(dst, src, bytes, cudaMemcpyDeviceToDevice, s);
  };
  if (h->cfg.has_router_bias) cp(h->b_router, wt->b_router, N * 4);
  if (!h->bf16) {
    // fp32: the CUDA-core kernels read the natural layouts; W_y = [W_up | S_o(0) | ...]
    if (e == cudaSuccess) e = copy2d(h->w_y, ky, wt->w_up, l, l, d, es, s);
    for (size_t j = 0; j < ns && e == cudaSuccess; ++j)
      e = copy2d(off(h->w_y, l + j * ms, es), ky,
                 off(const_cast<void *>(wt->s_out), j * d * ms, es), ms, ms, d, es, s);
    cp(h->w_out, wt->w_out, N * l * m * es);
    cp(h->w_router, wt->w_router, N * d * es);
    cp(h->w_down, wt->w_down, l * d * es);
    if (!h->relu2) cp(h->w_gate, wt->w_gate, N * m * l * es);
    cp(h->w_upx, wt->w_upx, N * m * l * es);
    if (!h->relu2) cp(h->s_gate, wt->s_gate, ns * ms * d * es);
    cp(h->s_up, wt->s_up, ns * ms * d * es);
    if (e != cudaSuccess) return LMOE_ERR_CUDA;
    h->loaded = true;
    return LMOE_OK;
  }
  // bf16: assemble each B operand row-major in a temporary, then repack it
  // K-block tiled into the handle's buffer.
  void *tx = nullptr, *tgu = nullptr, *ty = nullptr;
  const size_t NE = h->NE;
  const size_t bx = static_cast<size_t>(h->nx_rows) * d * es, bgu = NE * 2 * m * l * es,
               by = d * ky * es;
  if (!dalloc(&tx, bx) || (!h->relu2 && !dalloc(&tgu, bgu)) || !dalloc(&ty, by)) {
    if (tx) cudaFree(tx);
    if (tgu) cudaFree(tgu);
    cudaGetLastError();
    return LMOE_ERR_OUT_OF_MEMORY;
  }
  // W_y = [W_up | S_o(0) | S_o(1) ...]  ([d][l + ns ms])
  if (e == cudaSuccess) e = copy2d(ty, ky, wt->w_up, l, l, d, es, s);
  for (size_t j = 0; j < ns && e == cudaSuccess; ++j)
    e = copy2d(off(ty, l + j * ms, es), ky, off(const_cast<void *>(wt->s_out), j * d * ms, es),
               ms, ms, d, es, s);
  // Stacked x-matrix: rows [0,N) W_r, [n_pad, n_pad+l) W_down, then for each
  // block b of 128 shared hidden units: 128 gate rows followed by the 128
  // matching up rows.  Padding rows are zero.
  if (e == cudaSuccess) e = cudaMemsetAsync(tx, 0, bx, s);
  cp(tx, wt->w_router, N * d * es);
  cp(off(tx, static_cast<size_t>(h->n_pad) * d, es), wt->w_down, l * d * es);
  const size_t sh0 = static_cast<size_t>(h->n_pad + h->l_pad);
  if (h->relu2) {  // shared up rows, in expert order (padding rows stay zero)
    cp(off(tx, sh0 * d, es), wt->s_up, ns * ms * d * es);
  }
  for (size_t b = 0; !h->relu2 && b < ns * ms / 128; ++b) {
    cp(off(tx, (sh0 + 256 * b) * d, es), off(const_cast<void *>(wt->s_gate), 128 * b * d, es),
       128 * d * es);
    cp(off(tx, (sh0 + 256 * b + 128) * d, es), off(const_cast<void *>(wt->s_up), 128 * b * d, es),
       128 * d * es);
  }
  // Expert gate/up: per expert, blocks of 128 gate rows then 128 up rows.
  for (size_t b = 0; !h->relu2 && b < m / 128 && e == cudaSuccess; ++b) {
    e = copy2d(off(tgu, 256 * b * l, es), 2 * m * l,
               off(const_cast<void *>(wt->w_gate), 128 * b * l, es), m * l, 128 * l, NE, es, s);
    if (e == cudaSuccess)
      e = copy2d(off(tgu, (256 * b + 128) * l, es), 2 * m * l,
                 off(const_cast<void *>(wt->w_upx), 128 * b * l, es), m * l, 128 * l, NE, es, s);
  }
  using bf = __nv_bfloat16;
  if (e == cudaSuccess)
    e = launch_repack_btiles(static_cast<const bf *>(tx), 1, h->nx_rows, h->d,
                             static_cast<bf *>(h->w_x), s);
  if (h->fp4) {  // NVFP4 codes, block scales and row scales in GEMM tiles
    if (e == cudaSuccess)
      e = launch_quantize_nvfp4_tiles(static_cast<const bf *>(h->relu2 ? wt->w_upx : tgu), h->N,
                                      h->gu_rows, h->l, h->gu_scale, h->w_gu8, h->gu_sf, s);
    if (e == cudaSuccess)
      e = launch_quantize_nvfp4_tiles(static_cast<const bf *>(wt->w_out), h->N, h->l, h->m,
                                      h->o_scale, h->w_o8, h->o_sf, s);
  } else if (h->fp8) {  // E4M3 codes + row scales, tiled like the bf16 weights
    if (e == cudaSuccess)
      e = launch_quantize_e4m3_tiles(static_cast<const bf *>(h->relu2 ? wt->w_upx : tgu), h->N,
                                     h->gu_rows, h->l, h->gu_scale, h->w_gu8, s);
    if (e == cudaSuccess)
      e = launch_quantize_e4m3_tiles(static_cast<const bf *>(wt->w_out), h->N, h->l, h->m,
                                     h->o_scale, h->w_o8, s);
  } else {
    if (e == cudaSuccess)  // expert up rows: interleaved gate/up, or the up-projection itself
      e = launch_repack_btiles(static_cast<const bf *>(h->relu2 ? wt->w_upx : tgu), h->NE,
                               h->gu_rows, h->l, static_cast<bf *>(h->w_gu), s);
    if (e == cudaSuccess)
      e = launch_repack_btiles(static_cast<const bf *>(wt->w_out), h->NE, h->l, h->m,
                               static_cast<bf *>(h->w_out), s);
  }
  if (e == cudaSuccess)
    e = launch_repack_btiles(static_cast<const bf *>(ty), 1, h->d, h->ky,
                             static_cast<bf *>(h->w_y), s);
  if (e == cudaSuccess && h->training) {
    // Backward: the transposed matrices, built in one scratch buffer and
    // K-block tiled like the forward's.
    const size_t big = std::max({static_cast<size_t>(h->nx_rows) * d, d * ky,
                                 N * m * l, N * static_cast<size_t>(h->gu_rows) * l});
    void *tt = nullptr;
    if (!dalloc(&tt, big * es)) e = cudaErrorMemoryAllocation;
    bf *t16 = static_cast<bf *>(tt);
    const bf *gu_src = static_cast<const bf *>(h->relu2 ? wt->w_upx : tgu);
    if (e == cudaSuccess)  // [W_up | S_o]^T: [ky][d]
      e = launch_transpose_bf16(static_cast<const bf *>(ty), static_cast<int>(ky), static_cast<int>(d),
                                static_cast<int>(ky), nullptr, nullptr, t16, static_cast<long long>(d), s);
    if (e == cudaSuccess)
      e = launch_repack_btiles(t16, 1, h->ky, h->d, static_cast<bf *>(h->w_yT), s);
    if (e == cudaSuccess)  // W_o[e]^T: [m][l] per expert
      e = launch_transpose_bf16(static_cast<const bf *>(wt->w_out), h->m, h->l, h->m, nullptr,
                                nullptr, t16, h->l, s, h->N, static_cast<long long>(l * m),
                                static_cast<long long>(m * l));
    if (e == cudaSuccess)
      e = launch_repack_btiles(t16, h->N, h->m, h->l, static_cast<bf *>(h->w_oT), s);
    if (e == cudaSuccess)  // W_gu[e]^T: [l][gu_rows] per expert
      e = launch_transpose_bf16(gu_src, h->l, h->gu_rows, h->l, nullptr, nullptr, t16,
                                h->gu_rows, s, h->N, static_cast<long long>(h->gu_rows) * l,
                                static_cast<long long>(h->gu_rows) * l);
    if (e == cudaSuccess)
      e = launch_repack_btiles(t16, h->N, h->l, h->gu_rows, static_cast<bf *>(h->w_guT), s);
    if (e == cudaSuccess)  // W_x^T: [d][nx_rows]
      e = launch_transpose_bf16(static_cast<const bf *>(tx), h->d, h->nx_rows, h->d, nullptr,
                                nullptr, t16, h->nx_rows, s);
    if (e == cudaSuccess)
      e = launch_repack_btiles(t16, 1, h->d, h->nx_rows, static_cast<bf *>(h->w_xT), s);
    const cudaError_t es3 = cudaStreamSynchronize(s);
    if (tt) cudaFree(tt);
    if (e == cudaSuccess) e = es3;
  }
  // the temporaries are freed once the repacks have run
  const cudaError_t es2 = cudaStreamSynchronize(s);
  cudaFree(tx);
  if (tgu) cudaFree(tgu);
  cudaFree(ty);
  if (e == cudaSuccess) e = es2;
  if (e != cudaSuccess) return LMOE_ERR_CUDA;
  h->loaded = true;
  return LMOE_OK;
}

static void mark(lmoe_layer *h, int i, cudaStream_t s) {
  if (h->prof_slots > 0) {
    const int64_t slot = h->prof_count % h->prof_slots;
    cudaEventRecord(h->ev[slot * (LMOE_NUM_STAGES + 1) + i], s);
  }
}

// Slices for a dense launch of `tiles` output tiles over nkb K-blocks, M rows
// and `cols` output columns on `slots` CTAs (or CTA pairs): 1 (no split) once
// the tiles fill half of the slots; otherwise enough slices to fill them,
// each non-empty.  A split launch runs on single CTAs when its tokens fit one
// 128-row M-tile (a pair's 256-row MMA would be mostly empty rows).  Calls
// of kHostChunkTokens tokens or more never split, so that lmoe_forward_host's
// chunks take the same path (and give the same bits) as one call over all
// their tokens.
static int split_for(int tiles, int nkb, int M, int cols, int slots) {
  if (M >= kHostChunkTokens || tiles <= 0 || 2 * tiles > slots) return 1;
  int ks = std::min(std::min(slots / tiles, kMaxSplit), nkb / kMinSplitKb);
  while (ks > 1 && static_cast<size_t>(ks) * M * cols > kPartFloats) --ks;
  if (ks < 2) return 1;
  const int per = (nkb + ks - 1) / ks;
  return (nkb + per - 1) / per;
}

static int check_call(lmoe_handle h, int32_t T) {
  if (!h) return LMOE_ERR_NULL_ARG;
  if (!h->loaded) return LMOE_ERR_NOT_LOADED;
  if (T < 0 || T > h->Tmax) return LMOE_ERR_TOO_MANY_TOKENS;
  return LMOE_OK;
}

// Router logits (+ z and shared hidden when full) and the routing steps.
// shared_raw (bf16 backward only): the shared experts' gate/up GEMM writes its
// raw pre-activations there ([T][sh_rows], W_x's shared-row layout) instead
// of the hidden.
// permute_dst: also write the z rows in dispatch order there (full only).
static cudaError_t run_route(lmoe_layer *h, const void *x, int T, bool full, cudaStream_t s,
                             void *shared_raw = nullptr, bool marks = true,
                             void *permute_dst = nullptr, SegPad seg = kNoPad) {
  Workspace &w = h->ws;
  cudaError_t e = cudaSuccess;
  if (seg.pad > 1) {  // padded order: its padding rows keep perm = -1
    e = cudaMemsetAsync(w.perm, 0xFF, static_cast<size_t>(h->bw.Kp) * 4, s);
    if (e != cudaSuccess) return e;
  }
  if (h->bf16) {
    TensorMap64 tm_x;
    if (make_map(&tm_x, x, T, h->d, h->d, kTileM) != LMOE_OK) return cudaErrorInvalidValue;
    TcParams p = {};
    p.mode = TC_X_FUSED;
    p.M = T;
    p.Kdim = h->d;
    p.n_tile_base = 0;
    p.n_tiles_n = (full ? h->n_pad + h->l_pad : h->n_pad) / kTileN;
    p.r_end = h->n_pad;
    p.z_end = h->n_pad + h->l_pad;
    p.n_routed = h->N;
    p.l = h->l;
    p.logits = w.logits;
    p.ld_logits = h->N;
    p.z = static_cast<__nv_bfloat16 *>(w.z);
    p.ld_z = h->l;
    p.out = static_cast<__nv_bfloat16 *>(w.ucat);
    p.ld_out = h->ky;
    p.out_col0 = h->l;
    p.relu2 = h->relu2;
    p.n_cols2 = h->ns * h->ms;
    p.status = w.status;
    p.tma_out = 1;  // z through TMA stores (the logits are stored directly)
    const int m_tiles = (T + kTileM - 1) / kTileM;
    const int m_tiles2 = (T + 2 * kTileM - 1) / (2 * kTileM);
    // few tokens: split the reduction (partials, then launch_splitk_reduce)
    const bool one_mtile = m_tiles == 1;
    const int xs = split_for((one_mtile ? m_tiles : m_tiles2) * p.n_tiles_n, h->d / 64, T,
                             p.n_tiles_n * kTileN, one_mtile ? h->num_sms : h->num_sms / 2);
    if (xs > 1) {
      p.k_split = xs;
      p.part = w.part;
    }
    if (xs > 1 && one_mtile) {
      p.tma_out = 0;
      e = launch_tc_gemm(tm_x.bytes, h->tm_wx.bytes, p, h->num_sms, p.n_tiles_n * xs, s);
    } else {
      e = launch_tc_gemm_pair(tm_x.bytes, h->tm_wx2.bytes, p, m_tiles2 * p.n_tiles_n * xs, s,
                              h->tm_out_z.bytes);
    }
    h->launches += 1;
    const int shared_tiles_n = (h->nx_rows - h->n_pad - h->l_pad) / kTileN;
    if (e == cudaSuccess && full && shared_tiles_n > 0) {
      // Shared experts' gate/up (the shared column range of the same matrix),
      // normally on the side stream, where it overlaps the routing kernels (a
      // long one runs first instead, below); the output GEMM joins it.  The
      // backward's raw variant runs on the single-CTA kernel.
      TcParams q = p;
      q.k_split = 0;
      q.part = nullptr;
      q.n_tile_base = (h->n_pad + h->l_pad) / kTileN;
      q.n_tiles_n = shared_tiles_n;
      // direct stores: the smaller shared-memory footprint lets the routing
      // kernels run beside this launch's CTAs.  The paired launch is capped at
      // num_sms * 2 / 5 CTA pairs (59 pairs, 118 of 148 SMs; each pair loops
      // over its tiles), so that the routing kernels find free SMs.
      q.tma_out = 0;
      if (shared_raw) {
        q.raw = 1;
        q.out2 = static_cast<__nv_bfloat16 *>(shared_raw);
        q.ld_out2 = h->sh_rows;
      }
      // A long shared GEMM (more than kSideKbWaves K-block waves on its capped
      // pairs) would outlast the routing and hold SMs into the persistent
      // gate/up GEMM, whose CTAs there would start late: it then runs first,
      // on the main stream and every SM.
      const int cap = std::max(1, h->num_sms * 2 / 5), shared_tiles = m_tiles2 * shared_tiles_n;
      const bool side = shared_raw || (shared_tiles + cap - 1) / cap * (h->d / 64) <= kSideKbWaves;
      if (side) {
        e = cudaEventRecord(h->ev_fork, s);
        if (e == cudaSuccess) e = cudaStreamWaitEvent(h->side, h->ev_fork, 0);
        if (e == cudaSuccess)
          e = shared_raw ? launch_tc_gemm(tm_x.bytes, h->tm_wx.bytes, q, h->num_sms,
                                          m_tiles * shared_tiles_n, h->side)
                         : launch_tc_gemm_pair(tm_x.bytes, h->tm_wx2.bytes, q,
                                               std::min(shared_tiles, cap), h->side);
        if (e == cudaSuccess) e = cudaEventRecord(h->ev_join, h->side);
      } else {
        e = launch_tc_gemm_pair(tm_x.bytes, h->tm_wx2.bytes, q, shared_tiles, s);
        if (e == cudaSuccess) e = cudaEventRecord(h->ev_join, s);
      }
      h->launches += 1;
    }
    if (e == cudaSuccess && xs > 1) {
      e = launch_splitk_reduce(p, s, false);
      h->launches += 1;
    }
  } else {
    e = simt_linear(static_cast<const float *>(x), h->d, static_cast<const float *>(h->w_router),
                    h->d, w.logits, h->N, T, h->N, h->d, s);
    h->launches += 1;
    if (e == cudaSuccess && full) {  // fp32: z and the shared hidden belong to stage 0 too
      e = simt_linear(static_cast<const float *>(x), h->d, static_cast<const float *>(h->w_down),
                      h->d, static_cast<float *>(w.z), h->l, T, h->l, h->d, s);
      h->launches += 1;
      if (e == cudaSuccess && h->ns > 0) {
        const float *xf = static_cast<const float *>(x);
        float *hs = static_cast<float *>(w.ucat) + h->l;
        e = h->relu2 ? simt_relu2(xf, h->d, static_cast<const float *>(h->s_up), h->ms, nullptr,
                                  hs, h->ky, T, h->ns * h->ms, h->d, s)
                     : simt_swiglu(xf, h->d, static_cast<const float *>(h->s_gate),
                                   static_cast<const float *>(h->s_up), h->ms, nullptr, hs, h->ky,
                                   T, h->ns * h->ms, h->d, s);
        h->launches += 1;
      }
    }
  }
  if (e != cudaSuccess) return e;
  if (full && marks) mark(h, 1, s);
  const int rb = h->l * static_cast<int>(h->esize);
  if (h->fused_route) {
    // programmatic launches: each follows the previous kernel of the stream
    // (bf16: the router GEMM; fp32: the CUDA-core router) and waits for it on
    // the device before touching memory
    e = launch_route_select(w.logits, h->N, h->b_router, T, h->N, h->K, w.ids, w.gates,
                            w.chunk_counts, kFusedChunk, w.arrivals, w.offsets, w.tiles,
                            w.n_tiles, kTileM, h->max_tiles, w.tiles2, w.n_tiles2, 2 * kTileM,
                            h->max_tiles2, s, true, seg);
    h->launches += 1;
    if (e != cudaSuccess) return e;
    if (full && marks) mark(h, 2, s);
    // From kRowCopyTokens tokens on, the scatter writes positions only and a
    // destination-major copy (one warp per permuted row) fills permute_dst;
    // below, the scatter also copies the rows (one launch less).
    const bool row_copy = permute_dst && T >= kRowCopyTokens;
    const bool fused_copy = permute_dst && !row_copy;
    e = launch_scatter_permute(w.ids, T, h->K, h->N, w.chunk_counts, kFusedChunk, w.offsets,
                               w.perm, w.pos, w.row_expert, fused_copy ? w.z : nullptr, rb,
                               fused_copy ? permute_dst : nullptr, h->route_shares, s, true);
    h->launches += 1;
    if (e != cudaSuccess) return e;
    if (full && marks) mark(h, 3, s);
    if (row_copy) {
      e = launch_permute_rows(w.z, w.perm, h->K, T * h->K, rb, permute_dst, s);
      h->launches += 1;
      if (e != cudaSuccess) return e;
    }
    if (full && marks) mark(h, 4, s);  // empty stage when the scatter copied the rows
    return e;
  }
  // top-K' also builds the dispatch histogram (into the zeroed count matrix)
  e = cudaMemsetAsync(w.chunk_counts, 0, dispatch_count_elems(T, kDispatchChunk, h->N) * 4, s);
  if (e != cudaSuccess) return e;
  e = launch_topk(w.logits, h->N, h->b_router, T, h->N, h->K, w.ids, w.gates, w.chunk_counts,
                  kDispatchChunk, s);
  h->launches += 1;
  if (e != cudaSuccess) return e;
  if (full && marks) mark(h, 2, s);
  e = launch_dispatch(w.ids, T, h->K, h->N, w.chunk_counts, kDispatchChunk, true, w.offsets,
                      w.perm, w.pos, w.row_expert, w.tiles, w.n_tiles, kTileM, h->max_tiles, s,
                      w.tiles2, w.n_tiles2, 2 * kTileM, h->max_tiles2, false, seg);
  h->launches += 2;
  if (e != cudaSuccess) return e;
  if (full && marks) mark(h, 3, s);
  if (permute_dst) {
    e = launch_permute_rows(w.z, w.perm, h->K, T * h->K, rb, permute_dst, s);
    h->launches += 1;
    if (e != cudaSuccess) return e;
    if (full && marks) mark(h, 4, s);
  }
  return e;
}

int lmoe_route(lmoe_handle h, const void *x, int32_t T, int32_t *ids, float *gates,
               int32_t *offsets, int32_t *perm, void *stream) {
  int rc = check_call(h, T);
  if (rc != LMOE_OK) return rc;
  if (T > 0 && !x) return LMOE_ERR_NULL_ARG;
  if (T > 0 && !aligned16(x)) return LMOE_ERR_MISALIGNED;
  DeviceGuard g(h->device);
  if (!g.ok) return LMOE_ERR_CUDA;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  Workspace &w = h->ws;
  cudaError_t e = cudaSuccess;
  if (T > 0) {
    e = run_route(h, x, T, false, s);
  } else {
    e = cudaMemsetAsync(w.offsets, 0, (h->N + 1) * sizeof(int32_t), s);
  }
  const size_t TK = static_cast<size_t>(T) * h->K;
  if (e == cudaSuccess && ids && TK)
    e = cudaMemcpyAsync(ids, w.ids, TK * 4, cudaMemcpyDeviceToDevice, s);
  if (e == cudaSuccess && gates && TK)
    e = cudaMemcpyAsync(gates, w.gates, TK * 4, cudaMemcpyDeviceToDevice, s);
  if (e == cudaSuccess && offsets)
    e = cudaMemcpyAsync(offsets, w.offsets, (h->N + 1) * 4, cudaMemcpyDeviceToDevice, s);
  if (e == cudaSuccess && perm && TK)
    e = cudaMemcpyAsync(perm, w.perm, TK * 4, cudaMemcpyDeviceToDevice, s);
  return cuda_err(e);
}

// bf16 expert GEMMs over grouped rows: A rows through tm_a ({64, 128} boxes;
// tm_a32: {64, 32} boxes, E4M3 weights only), the M-tile tables (128-row
// tiles, and 256-row tiles for the pair down GEMM), H in the workspace, and
// the expert outputs through the store map tm_o.  pair_down: the down GEMM
// runs on CTA pairs.  stage_gu / stage_down: profiling marks after each.
// pdl: the gate/up launch directly follows another kernel on s (the down
// GEMM always follows the gate/up GEMM).  a_rows: rows of A (and of H, O).
// E4M3 experts: A is the E4M3 copy of the rows (tm_a over zq), H is
// quantised to hq between the two GEMMs.
static cudaError_t run_experts_bf16(lmoe_layer *h, const TensorMap64 &tm_a,
                                    const TensorMap64 &tm_a32, const TileEntry *tiles,
                                    const int32_t *n_tiles, const TileEntry *tiles2,
                                    const int32_t *n_tiles2, bool pair_down, void *O,
                                    const TensorMap64 &tm_o, cudaStream_t s, bool marks,
                                    bool pdl, int a_rows) {
  Workspace &w = h->ws;
  TcParams p = {};
  p.mode = TC_EXPERT_GU;
  p.Kdim = h->l;
  p.n_tiles_n = (h->gu_rows + kTileN - 1) / kTileN;
  p.relu2 = h->relu2;
  p.n_cols2 = h->m;
  p.tiles = tiles;
  p.n_mtiles = n_tiles;
  if (h->fp8) {
    p.a_scale = h->ws.zq_scale;
    p.b_scale = h->gu_scale;
    p.b_scale_ld = h->gu_rows;
    if (h->fp4) {
      p.a_sf = h->ws.zq_sf;
      p.b_sf = h->gu_sf;
    }
  }
  p.b_rows_per_expert = h->gu_rows;
  p.out = static_cast<__nv_bfloat16 *>(w.H);
  p.ld_out = h->m;
  p.status = w.status;
  // Single-CTA tiles of 128 rows: measured at least as fast as CTA pairs for
  // the gate/up GEMM (K = l is short, the SwiGLU epilogue is the heavier)
  // and much faster when experts hold few tokens.
  p.tma_out = 1;
  p.pdl = pdl && !marks ? 1 : 0;
  cudaError_t e = launch_tc_gemm(tm_a.bytes, h->tm_wgu.bytes, p, h->num_sms, h->num_sms, s,
                                 tm_a32.bytes, h->tm_out_h.bytes);
  h->launches += 1;
  if (e != cudaSuccess) return e;
  if (h->fp4) {  // H rows -> NVFP4 codes and scales, the down GEMM's A operand
    e = launch_quantize_act_nvfp4(static_cast<const __nv_bfloat16 *>(w.H), nullptr, 1, tiles,
                                  n_tiles, h->max_tiles, h->m, w.hq, w.hq_scale, w.hq_sf, s,
                                  !marks);
    h->launches += 1;
    if (e != cudaSuccess) return e;
  } else if (h->fp8) {  // H rows -> E4M3 with row scales, the down GEMM's A operand
    e = launch_quantize_rows_e4m3(static_cast<const __nv_bfloat16 *>(w.H), nullptr, 1, a_rows,
                                  h->m, w.hq, w.hq_scale, s, !marks);
    h->launches += 1;
    if (e != cudaSuccess) return e;
  }
  if (marks) mark(h, 5, s);
  TcParams pd = {};
  pd.mode = TC_EXPERT_DOWN;
  pd.Kdim = h->m;
  pd.n_tiles_n = (h->l + kTileN - 1) / kTileN;
  pd.tiles = tiles;
  pd.n_mtiles = n_tiles;
  pd.b_rows_per_expert = h->l;
  pd.out = static_cast<__nv_bfloat16 *>(O);
  pd.ld_out = h->l;
  pd.status = w.status;
  if (h->fp8) {
    pd.a_scale = w.hq_scale;
    pd.b_scale = h->o_scale;
    pd.b_scale_ld = h->l;
    if (h->fp4) {
      pd.a_sf = w.hq_sf;
      pd.b_sf = h->o_sf;
    }
  }
  pd.tma_out = 1;
  pd.pdl = marks ? 0 : 1;
  if (pair_down) {
    pd.tiles = tiles2;
    pd.n_mtiles = n_tiles2;
    e = launch_tc_gemm_pair(h->tm_h.bytes, h->tm_wo2.bytes, pd, h->num_sms, s, tm_o.bytes);
  } else {
    e = launch_tc_gemm(h->fp8 ? h->tm_hq.bytes : h->tm_h.bytes, h->tm_wo.bytes, pd, h->num_sms,
                       h->num_sms, s, h->tm_hq32.bytes, tm_o.bytes);
  }
  h->launches += 1;
  if (e == cudaSuccess && marks) mark(h, 6, s);
  return e;
}

// bf16: u = the gate-weighted combine of the expert outputs O (dispatch
// order) into Ucat's first l columns, then y = [u | shared hidden] W_y^T
// once the side stream's shared gate/up GEMM has joined.
// pdl: the combine directly follows another kernel on s.
static cudaError_t run_combine_out_bf16(lmoe_layer *h, const void *O, void *y, int T,
                                        cudaStream_t s, bool marks, bool pdl) {
  Workspace &w = h->ws;
  cudaError_t e =
      launch_combine(O, w.pos, w.gates, T, h->K, h->l, w.ucat, h->ky, true, s, pdl && !marks);
  h->launches += 1;
  if (e != cudaSuccess) return e;
  if (marks) mark(h, 7, s);
  e = cudaStreamWaitEvent(s, h->ev_join, 0);  // shared hidden ready
  if (e != cudaSuccess) return e;
  TcParams q = {};
  q.mode = TC_OUT;
  q.M = T;
  q.Kdim = h->ky;
  q.n_tiles_n = (h->d + kTileN - 1) / kTileN;
  q.out = static_cast<__nv_bfloat16 *>(y);
  q.ld_out = h->d;
  q.status = w.status;
  // y through TMA stores when its address allows a tensor map (16-byte aligned)
  TensorMap64 tm_y;
  q.tma_out = make_tmap_bf16_out(tm_y.bytes, y, T, h->d, h->d) == 0 ? 1 : 0;
  const int tiles2 = (T + 2 * kTileM - 1) / (2 * kTileM) * q.n_tiles_n;
  // few tokens: split the reduction (partials, then launch_splitk_reduce)
  const bool one_mtile = T <= kTileM;
  const int ys = split_for(one_mtile ? q.n_tiles_n : tiles2, h->ky / 64, T,
                           q.n_tiles_n * kTileN, one_mtile ? h->num_sms : h->num_sms / 2);
  if (ys > 1) {
    q.k_split = ys;
    q.part = w.part;
    q.tma_out = 0;
  }
  if (ys > 1 && one_mtile)
    e = launch_tc_gemm(h->tm_ucat.bytes, h->tm_wy.bytes, q, h->num_sms, q.n_tiles_n * ys, s);
  else
    e = launch_tc_gemm_pair(h->tm_ucat.bytes, h->tm_wy2.bytes, q, tiles2 * ys, s, tm_y.bytes);
  h->launches += 1;
  if (e == cudaSuccess && ys > 1) {
    e = launch_splitk_reduce(q, s, true);
    h->launches += 1;
  }
  return e;
}

static int forward_impl(lmoe_layer *h, const void *x, void *y, int T, cudaStream_t s) {
  Workspace &w = h->ws;
  const int TK = T * h->K;
  mark(h, 0, s);
  // the experts' rows: permuted z (bf16, fp32), or its E4M3 copy with row
  // scales, gathered straight from z through perm
  cudaError_t e = run_route(h, x, T, true, s, nullptr, true, h->fp8 ? nullptr : w.zp);
  if (e != cudaSuccess) return LMOE_ERR_CUDA;
  if (h->fp4) {
    e = launch_quantize_act_nvfp4(static_cast<const __nv_bfloat16 *>(w.z), w.perm, h->K, w.tiles,
                                  w.n_tiles, h->max_tiles, h->l, w.zq, w.zq_scale, w.zq_sf, s,
                                  h->prof_slots == 0);
    h->launches += 1;
    if (e != cudaSuccess) return LMOE_ERR_CUDA;
    mark(h, 4, s);
  } else if (h->fp8) {
    e = launch_quantize_rows_e4m3(static_cast<const __nv_bfloat16 *>(w.z), w.perm, h->K, TK, h->l,
                                  w.zq, w.zq_scale, s, h->prof_slots == 0);
    h->launches += 1;
    if (e != cudaSuccess) return LMOE_ERR_CUDA;
    mark(h, 4, s);
  }
  if (h->bf16) {
    // CTA pairs (256-row M-tiles) for the down GEMM when experts average at
    // least 256 rows: the long reduction (K = m) then gains from the smaller
    // per-SM operand feed; with fewer rows the pair's half-empty tiles cost
    // more than that.
    const bool pair_down = !h->fp8 && static_cast<int64_t>(T) * h->K >= 256LL * h->N;
    const bool marks = h->prof_slots > 0;
    e = run_experts_bf16(h, h->fp8 ? h->tm_zq : h->tm_zp, h->tm_zq32, w.tiles, w.n_tiles,
                         w.tiles2, w.n_tiles2, pair_down, w.O, h->tm_out_o, s, marks, true, TK);
    if (e == cudaSuccess) e = run_combine_out_bf16(h, w.O, y, T, s, marks, true);
  } else {
    float *zpf = static_cast<float *>(w.zp);
    float *Hf = static_cast<float *>(w.H), *Of = static_cast<float *>(w.O);
    float *uf = static_cast<float *>(w.ucat);
    e = h->relu2 ? simt_relu2(zpf, h->l, static_cast<const float *>(h->w_upx), h->m,
                              w.row_expert, Hf, h->m, TK, h->m, h->l, s)
                 : simt_swiglu(zpf, h->l, static_cast<const float *>(h->w_gate),
                               static_cast<const float *>(h->w_upx), h->m, w.row_expert, Hf,
                               h->m, TK, h->m, h->l, s);
    h->launches += 1;
    mark(h, 5, s);
    if (e == cudaSuccess)
      e = simt_expert_down(Hf, h->m, static_cast<const float *>(h->w_out), w.row_expert, Of, h->l,
                           TK, h->l, h->m, s);
    h->launches += 1;
    mark(h, 6, s);
    if (e == cudaSuccess) e = launch_combine(Of, w.pos, w.gates, T, h->K, h->l, uf, h->ky, false, s);
    h->launches += 1;
    mark(h, 7, s);
    if (e == cudaSuccess)
      e = simt_linear(uf, h->ky, static_cast<const float *>(h->w_y), h->ky,
                      static_cast<float *>(y), h->d, T, h->d, h->ky, s);
    h->launches += 1;
  }
  if (e != cudaSuccess) return LMOE_ERR_CUDA;
  mark(h, 8, s);
  if (h->prof_slots > 0) ++h->prof_count;
  return LMOE_OK;
}

int lmoe_forward(lmoe_handle h, const void *x, void *y, int32_t T, void *stream) {
  int rc = check_call(h, T);
  if (rc != LMOE_OK) return rc;
  if (h->ep_world > 1) return LMOE_ERR_UNSUPPORTED;  // this rank holds a slice of the experts
  if (T == 0) return LMOE_OK;
  if (!x || !y) return LMOE_ERR_NULL_ARG;
  if (!aligned16(x) || !aligned16(y)) return LMOE_ERR_MISALIGNED;
  DeviceGuard g(h->device);
  if (!g.ok) return LMOE_ERR_CUDA;
  return forward_impl(h, x, y, T, static_cast<cudaStream_t>(stream));
}

// ---- expert parallelism (see the declarations of lmoe_ep_*)
static int check_ep(lmoe_handle h, int32_t T) {
  const int rc = check_call(h, T);
  if (rc != LMOE_OK) return rc;
  return h->ep_world > 1 ? LMOE_OK : LMOE_ERR_UNSUPPORTED;
}

int lmoe_ep_dispatch(lmoe_handle h, const void *x, int32_t T, void *send_rows,
                     int32_t *expert_counts, void *stream) {
  int rc = check_ep(h, T);
  if (rc != LMOE_OK) return rc;
  if (!expert_counts || (T > 0 && (!x || !send_rows))) return LMOE_ERR_NULL_ARG;
  if (T > 0 && (!aligned16(x) || !aligned16(send_rows))) return LMOE_ERR_MISALIGNED;
  DeviceGuard g(h->device);
  if (!g.ok) return LMOE_ERR_CUDA;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  Workspace &w = h->ws;
  h->ep_T = T;
  if (T == 0) return cuda_err(cudaMemsetAsync(expert_counts, 0, h->N * sizeof(int32_t), s));
  // routing over all N' experts, z, and the shared hidden (side stream)
  // (z rows in dispatch order: expert-grouped, hence destination-rank grouped)
  cudaError_t e = run_route(h, x, T, true, s, nullptr, false, send_rows);
  if (e == cudaSuccess) e = launch_counts_from_offsets(w.offsets, h->N, expert_counts, s);
  h->launches += 1;
  return cuda_err(e);
}

int lmoe_ep_experts(lmoe_handle h, const void *recv_rows, const int32_t *recv_counts, int32_t R,
                    void *out_rows, void *stream) {
  if (!h) return LMOE_ERR_NULL_ARG;
  if (!h->loaded) return LMOE_ERR_NOT_LOADED;
  if (h->ep_world <= 1) return LMOE_ERR_UNSUPPORTED;
  if (R < 0 || R > h->R_max) return LMOE_ERR_TOO_MANY_TOKENS;
  if (!recv_counts || (R > 0 && (!recv_rows || !out_rows))) return LMOE_ERR_NULL_ARG;
  if (R > 0 && (!aligned16(recv_rows) || !aligned16(out_rows))) return LMOE_ERR_MISALIGNED;
  if (R == 0) return LMOE_OK;
  DeviceGuard g(h->device);
  if (!g.ok) return LMOE_ERR_CUDA;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  Workspace &w = h->ws;
  TensorMap64 tm_a, tm_o;
  if (make_map(&tm_a, recv_rows, R, h->l, h->l, kTileM) != LMOE_OK ||
      make_tmap_bf16_out(tm_o.bytes, out_rows, R, h->l, h->l) != 0)
    return LMOE_ERR_CUDA;
  // tile tables of the received rows; rows past R (counts that sum to more)
  // are clipped, so no tile reaches past the caller's buffers
  cudaError_t e = launch_ep_tiles(recv_counts, h->ep_world, h->NE, R, w.ep_tiles, w.ep_n_tiles,
                                  kTileM, h->max_tiles_ep, w.ep_tiles2, w.ep_n_tiles2, 2 * kTileM,
                                  h->max_tiles2_ep, s);
  h->launches += 1;
  const bool pair_down = static_cast<int64_t>(R) >= 256LL * h->NE;
  if (e == cudaSuccess)
    e = run_experts_bf16(h, tm_a, tm_a, w.ep_tiles, w.ep_n_tiles, w.ep_tiles2, w.ep_n_tiles2,
                         pair_down, out_rows, tm_o, s, false, true, R);
  return cuda_err(e);
}

int lmoe_ep_combine(lmoe_handle h, const void *back_rows, void *y, int32_t T, void *stream) {
  int rc = check_ep(h, T);
  if (rc != LMOE_OK) return rc;
  if (T != h->ep_T) return LMOE_ERR_INVALID_CONFIG;  // not the dispatched batch
  if (T == 0) return LMOE_OK;
  if (!back_rows || !y) return LMOE_ERR_NULL_ARG;
  if (!aligned16(back_rows) || !aligned16(y)) return LMOE_ERR_MISALIGNED;
  DeviceGuard g(h->device);
  if (!g.ok) return LMOE_ERR_CUDA;
  return cuda_err(run_combine_out_bf16(h, back_rows, y, T, static_cast<cudaStream_t>(stream),
                                       false, false));
}

// ---- backward (see the declaration of lmoe_backward): fp32 mode on CUDA cores.
static SimtGemm sg_dense(const float *A, long long sA_r, long long sA_k, const float *B,
                         long long sB_r, long long sB_k, float *C, long long ldc, int M, int N,
                         int K, bool accumulate) {
  SimtGemm q = {};
  q.A = A; q.sA_r = sA_r; q.sA_k = sA_k;
  q.B = B; q.sB_r = sB_r; q.sB_k = sB_k;
  q.C = C; q.ldc = ldc;
  q.M = M; q.N = N; q.K = K;
  q.accumulate = accumulate ? 1 : 0;
  return q;
}

static cudaError_t backward_f32(lmoe_layer *h, const float *x, const float *dy, float *dx,
                                const lmoe_grads *g, int T, cudaStream_t s) {
  Workspace &w = h->ws;
  BwdWorkspace &b = h->bw;
  const int d = h->d, l = h->l, m = h->m, N = h->N, K = h->K, ky = h->ky;
  const int nsms = h->ns * h->ms, TK = T * K;
  const bool relu2 = h->relu2 != 0;
  const float *Wr = static_cast<const float *>(h->w_router);
  const float *Wd = static_cast<const float *>(h->w_down);
  const float *Wg = static_cast<const float *>(h->w_gate);
  const float *Wu = static_cast<const float *>(h->w_upx);
  const float *Wo = static_cast<const float *>(h->w_out);
  const float *Sg = static_cast<const float *>(h->s_gate);
  const float *Su = static_cast<const float *>(h->s_up);
  const float *Wy = static_cast<const float *>(h->w_y);
  float *zp = static_cast<float *>(w.zp), *H = static_cast<float *>(w.H);
  float *O = static_cast<float *>(w.O), *ucat = static_cast<float *>(w.ucat);
  float *A_ = static_cast<float *>(b.a), *B_ = static_cast<float *>(b.b);
  float *DO = static_cast<float *>(b.DO), *dA = static_cast<float *>(b.dA);
  float *dB = static_cast<float *>(b.dB);
  float *as = static_cast<float *>(b.as), *bs = static_cast<float *>(b.bs);
  float *das = static_cast<float *>(b.das), *dbs = static_cast<float *>(b.dbs);
  int64_t &L = h->launches;
#define LMOE_TRY(...) do { cudaError_t e_ = (__VA_ARGS__); ++L; if (e_ != cudaSuccess) return e_; } while (0)
  // forward activations: routing, z, shared hidden, expert pre-activations, H, O, u
  cudaError_t e = run_route(h, x, T, true, s);
  if (e != cudaSuccess) return e;
  LMOE_TRY(launch_permute_rows(w.z, w.perm, K, TK, l * 4, w.zp, s));
  if (!relu2) LMOE_TRY(simt_rowexpert(zp, l, Wg, 1LL * m * l, l, 1, w.row_expert, A_, m, TK, m, l, false, s));
  LMOE_TRY(simt_rowexpert(zp, l, Wu, 1LL * m * l, l, 1, w.row_expert, B_, m, TK, m, l, false, s));
  LMOE_TRY(launch_act_backward<float, float>(A_, B_, m, nullptr, 0, H, m, nullptr, nullptr, 0, TK,
                                             m, relu2, s));
  LMOE_TRY(simt_expert_down(H, m, Wo, w.row_expert, O, l, TK, l, m, s));
  LMOE_TRY(launch_combine(O, w.pos, w.gates, T, K, l, ucat, ky, false, s));
  // du | dh_s = dy . [W_up | S_o]   (C[t][c] = sum_i dy[t][i] W_y[i][c])
  LMOE_TRY(simt_gemm(sg_dense(dy, d, 1, Wy, 1, ky, b.dU, ky, T, ky, d, false), 1, s));
  // gate gradients and the expert-output gradients
  LMOE_TRY(launch_slot_grad<float>(b.dU, ky, O, l, w.pos, w.gates, T, K, b.ds, DO, s));
  // dH[p][c] = sum_j DO[p][j] W_o[e][j][c]
  LMOE_TRY(simt_rowexpert(DO, l, Wo, 1LL * l * m, 1, m, w.row_expert, b.dH, m, TK, m, l, false, s));
  LMOE_TRY(launch_act_backward<float, float>(A_, B_, m, b.dH, m, nullptr, 0, dA, dB, m, TK, m,
                                             relu2, s));
  // dZp[p][j] = sum_c dA[p][c] W_g[e][c][j] + dB[p][c] W_u[e][c][j]
  if (!relu2) LMOE_TRY(simt_rowexpert(dA, m, Wg, 1LL * m * l, 1, l, w.row_expert, b.dZp, l, TK, l, m, false, s));
  LMOE_TRY(simt_rowexpert(dB, m, Wu, 1LL * m * l, 1, l, w.row_expert, b.dZp, l, TK, l, m, !relu2, s));
  LMOE_TRY(launch_gather_sum<float, float>(b.dZp, l, w.pos, T, K, l, b.dz, l, s));
  // shared experts: pre-activations and their gradients (dh_s = dU[:, l:])
  if (nsms > 0) {
    if (!relu2) LMOE_TRY(simt_gemm(sg_dense(x, d, 1, Sg, d, 1, as, nsms, T, nsms, d, false), 1, s));
    LMOE_TRY(simt_gemm(sg_dense(x, d, 1, Su, d, 1, bs, nsms, T, nsms, d, false), 1, s));
    LMOE_TRY(launch_act_backward<float, float>(as, bs, nsms, b.dU + l, ky, nullptr, 0, das, dbs,
                                               nsms, T, nsms, relu2, s));
  }
  LMOE_TRY(launch_scatter_ds<float>(b.ds, w.ids, T, K, N, b.dsfull, N, s));
  // dx = dz W_down + dS W_r + da_s S_g + db_s S_u
  LMOE_TRY(simt_gemm(sg_dense(b.dz, l, 1, Wd, 1, d, dx, d, T, d, l, false), 1, s));
  LMOE_TRY(simt_gemm(sg_dense(b.dsfull, N, 1, Wr, 1, d, dx, d, T, d, N, true), 1, s));
  if (nsms > 0) {
    if (!relu2) LMOE_TRY(simt_gemm(sg_dense(das, nsms, 1, Sg, 1, d, dx, d, T, d, nsms, true), 1, s));
    LMOE_TRY(simt_gemm(sg_dense(dbs, nsms, 1, Su, 1, d, dx, d, T, d, nsms, true), 1, s));
  }
  // weight gradients, dense: K runs over the T tokens in order
  LMOE_TRY(simt_gemm(sg_dense(dy, 1, d, ucat, 1, ky, g->w_up, l, d, l, T, false), 1, s));
  if (nsms > 0) {
    SimtGemm q = sg_dense(dy, 1, d, ucat + l, 1, ky, g->s_out, h->ms, d, h->ms, T, false);
    q.sB_g = h->ms;
    q.sC_g = 1LL * d * h->ms;
    LMOE_TRY(simt_gemm(q, h->ns, s));
    if (!relu2) LMOE_TRY(simt_gemm(sg_dense(das, 1, nsms, x, 1, d, g->s_gate, d, nsms, d, T, false), 1, s));
    LMOE_TRY(simt_gemm(sg_dense(dbs, 1, nsms, x, 1, d, g->s_up, d, nsms, d, T, false), 1, s));
  }
  LMOE_TRY(simt_gemm(sg_dense(b.dz, 1, l, x, 1, d, g->w_down, d, l, d, T, false), 1, s));
  LMOE_TRY(simt_gemm(sg_dense(b.dsfull, 1, N, x, 1, d, g->w_router, d, N, d, T, false), 1, s));
  if (g->b_router) LMOE_TRY(launch_bias_grad(b.ds, w.offsets, w.perm, N, g->b_router, s));
  // weight gradients, grouped: K runs over expert e's permuted rows
  {
    SimtGemm q = sg_dense(DO, 1, l, H, 1, m, g->w_out, m, l, m, 0, false);
    q.k_off = w.offsets;
    q.sC_g = 1LL * l * m;
    LMOE_TRY(simt_gemm(q, N, s));
    q = sg_dense(dB, 1, m, zp, 1, l, g->w_upx, l, m, l, 0, false);
    q.k_off = w.offsets;
    q.sC_g = 1LL * m * l;
    LMOE_TRY(simt_gemm(q, N, s));
    if (!relu2) {
      q.A = dA;
      q.C = g->w_gate;
      LMOE_TRY(simt_gemm(q, N, s));
    }
  }
#undef LMOE_TRY
  return cudaSuccess;
}

// ---- backward, bf16 mode: every contraction on the tcgen05 GEMM.
static cudaError_t backward_bf16(lmoe_layer *h, const void *x, const void *dy, void *dx,
                                 const lmoe_grads *g, int T, cudaStream_t s) {
  using bf = __nv_bfloat16;
  Workspace &w = h->ws;
  BwdWorkspace &b = h->bw;
  const int d = h->d, l = h->l, m = h->m, N = h->N, K = h->K, ky = h->ky;
  const int nx = h->nx_rows, gu = h->gu_rows;
  const int n_pad = h->n_pad, l_pad = h->l_pad;
  const bool relu2 = h->relu2 != 0;
  bf *ucat = static_cast<bf *>(w.ucat), *dXcat = static_cast<bf *>(b.dXcat);
  int64_t &L = h->launches;
  auto gemm = [&](const TensorMap64 &ta, const TensorMap64 &tb, const TcParams &p, int tiles) {
    ++L;
    return launch_tc_gemm(ta.bytes, tb.bytes, p, h->num_sms, tiles, s);
  };
#define LMOE_TRY(...) do { cudaError_t e_ = (__VA_ARGS__); if (e_ != cudaSuccess) return e_; } while (0)
  TensorMap64 tm_x, tm_dy;
  if (make_map(&tm_x, x, T, d, d, kTileM) != LMOE_OK ||
      make_map(&tm_dy, dy, T, d, d, kTileM) != LMOE_OK)
    return cudaErrorInvalidValue;
  const int m_tiles_T = (T + kTileM - 1) / kTileM;
  // ---- forward activations, in the padded dispatch order: each expert's rows
  // start at a multiple of 64 (so that the weight gradients can read each
  // expert's rows of the token-major matrices as whole 64-row K-blocks), the
  // padding rows of zp are zeros
  const SegPad seg = {64, w.seg_end};
  LMOE_TRY(run_route(h, x, T, true, s, b.ABs, true, nullptr, seg));
  ++L;
  LMOE_TRY(launch_permute_rows(w.z, w.perm, K, static_cast<int>(b.Kp), l * 2, w.zp, s));
  {
    TcParams p = {};  // expert gate/up pre-activations AB
    p.mode = TC_EXPERT_GU; p.Kdim = l; p.n_tiles_n = (gu + kTileN - 1) / kTileN; p.raw = 1;
    p.relu2 = h->relu2; p.n_cols2 = m;
    p.tiles = w.tiles; p.n_mtiles = w.n_tiles;
    p.out = static_cast<bf *>(b.AB); p.ld_out = gu;
    p.out_h = static_cast<bf *>(w.H); p.ld_h = m;  // and the hidden
    p.status = w.status;
    LMOE_TRY(gemm(h->tm_zp, h->tm_wgu, p, h->num_sms));
  }
  {
    TcParams p = {};  // expert outputs O
    p.mode = TC_EXPERT_DOWN; p.Kdim = m; p.n_tiles_n = (l + kTileN - 1) / kTileN;
    p.tiles = w.tiles; p.n_mtiles = w.n_tiles;
    p.out = static_cast<bf *>(w.O); p.ld_out = l; p.status = w.status;
    LMOE_TRY(gemm(h->tm_h, h->tm_wo, p, h->num_sms));
  }
  ++L;
  LMOE_TRY(launch_combine(w.O, w.pos, w.gates, T, K, l, w.ucat, ky, true, s));  // u
  LMOE_TRY(cudaStreamWaitEvent(s, h->ev_join, 0));  // shared pre-activations ready
  // ---- dU = dy [W_up | S_o]  (fp32 [T][ky])
  {
    TcParams p = {};
    p.mode = TC_OUT; p.M = T; p.Kdim = d; p.n_tiles_n = (ky + kTileN - 1) / kTileN;
    p.out_f32 = b.dU; p.ld_out = ky; p.status = w.status;
    LMOE_TRY(gemm(tm_dy, h->tm_wyT, p, m_tiles_T * p.n_tiles_n));
  }
  // shared experts: pre-activation gradients into dXcat's shared columns
  const int nsms = h->ns * h->ms;
  if (nsms > 0) {
    ++L;
    LMOE_TRY(launch_act_backward_rows<float>(static_cast<bf *>(b.ABs), h->sh_rows, b.dU + l, ky,
                                             dXcat + n_pad + l_pad, nx, T, nsms, relu2, s));
  }
  // ---- gates, expert-output gradients, expert backward
  ++L;
  LMOE_TRY(launch_slot_grad<bf>(b.dU, ky, static_cast<bf *>(w.O), l, w.pos, w.gates, T, K, b.ds,
                                static_cast<bf *>(b.DO), s));
  {
    // dH = DO W_o[e] (bf16, through the forward epilogue's TMA stores), then the
    // activation backward dAB from dH and the recomputed AB, element-wise: as a
    // kernel of its own it keeps far more loads in flight than the GEMM's
    // eight epilogue warps could
    TcParams p = {};
    p.mode = TC_EXPERT_DOWN; p.Kdim = l; p.n_tiles_n = (m + kTileN - 1) / kTileN;
    p.tiles = w.tiles; p.n_mtiles = w.n_tiles;
    p.out = reinterpret_cast<bf *>(b.dH); p.ld_out = m; p.status = w.status; p.tma_out = 1;
    ++L;
    LMOE_TRY(launch_tc_gemm(h->tm_DO.bytes, h->tm_woT.bytes, p, h->num_sms, h->num_sms, s,
                            nullptr, h->tm_dH_out.bytes));
    ++L;
    LMOE_TRY(launch_act_backward_rows<bf>(static_cast<const bf *>(b.AB), gu,
                                          reinterpret_cast<const bf *>(b.dH), m,
                                          static_cast<bf *>(b.dAB), gu, static_cast<int>(b.Kp), m,
                                          relu2, s));
  }
  {
    TcParams p = {};  // dZp = dAB W_gu[e]  (fp32 [TK][l])
    p.mode = TC_EXPERT_DOWN; p.Kdim = gu; p.n_tiles_n = (l + kTileN - 1) / kTileN;
    p.tiles = w.tiles; p.n_mtiles = w.n_tiles;
    p.out_f32 = b.dZp; p.ld_out = l; p.status = w.status;
    LMOE_TRY(gemm(h->tm_dAB, h->tm_wguT, p, h->num_sms));
  }
  // ---- dXcat = [dS | dz | shared dAB] in W_x's row order, padding zeroed
  L += 2;
  LMOE_TRY(launch_gather_sum<float, bf>(b.dZp, l, w.pos, T, K, l, dXcat + n_pad, nx, s));
  LMOE_TRY(launch_scatter_ds<bf>(b.ds, w.ids, T, K, N, dXcat, nx, s));
  auto zero_cols = [&](bf *base, int64_t ld, int64_t c0, int64_t c1, int rows) {
    if (c1 <= c0 || rows <= 0) return cudaSuccess;
    return cudaMemset2DAsync(base + c0, ld * 2, 0, (c1 - c0) * 2, rows, s);
  };
  LMOE_TRY(zero_cols(dXcat, nx, N, n_pad, T));
  LMOE_TRY(zero_cols(dXcat, nx, n_pad + l, n_pad + l_pad, T));
  LMOE_TRY(zero_cols(dXcat, nx, n_pad + l_pad + (relu2 ? nsms : 2 * nsms), nx, T));
  {
    TcParams p = {};  // dx = dXcat W_x
    p.mode = TC_OUT; p.M = T; p.Kdim = nx; p.n_tiles_n = (d + kTileN - 1) / kTileN;
    p.out = static_cast<bf *>(dx); p.ld_out = d; p.status = w.status;
    LMOE_TRY(gemm(h->tm_dXcat, h->tm_wxT, p, m_tiles_T * p.n_tiles_n));
  }
  // ---- weight gradients: A^T B straight from the token-major matrices
  // (read MN-major), K running over tokens
  auto fill_sizes = [&](TcParams &p) {
    p.wg_d = d; p.wg_l = l; p.wg_m = m; p.wg_ns = h->ns; p.wg_ms = h->ms; p.wg_n = N;
    p.wg_npad = n_pad; p.wg_lpad = l_pad; p.relu2 = h->relu2; p.status = w.status;
    p.g_router = g->w_router; p.g_down = g->w_down; p.g_up = g->w_up; p.g_gate = g->w_gate;
    p.g_upx = g->w_upx; p.g_out = g->w_out; p.g_sgate = g->s_gate; p.g_sup = g->s_up;
    p.g_sout = g->s_out;
  };
  {
    // dense: the maps hold exactly T rows, so a ragged last K-block reads zeros
    TensorMap64 tm_dy_mn, tm_ucat_mn, tm_dX_mn, tm_x_mn;
    if (make_map(&tm_dy_mn, dy, T, d, d, 64) != LMOE_OK ||
        make_map(&tm_ucat_mn, ucat, T, ky, ky, 64) != LMOE_OK ||
        make_map(&tm_dX_mn, dXcat, T, nx, nx, 64) != LMOE_OK ||
        make_map(&tm_x_mn, x, T, d, d, 64) != LMOE_OK)
      return cudaErrorInvalidValue;
    const int Tp = (T + 63) / 64 * 64;  // whole K-blocks; rows from T on read as zeros
    TcParams p = {};  // [dW_up | dS_o] = dy^T [u | h_s]
    p.mode = TC_WGRAD; p.wg_kind = WG_Y; p.groups = 1; p.M = d; p.Kdim = Tp;
    p.n_tiles_n = (ky + kTileN - 1) / kTileN;
    fill_sizes(p);
    LMOE_TRY(gemm(tm_dy_mn, tm_ucat_mn, p, (d + kTileM - 1) / kTileM * p.n_tiles_n));
    TcParams q = {};  // [dW_r ; dW_down ; dS_g / dS_u] = dXcat^T x
    q.mode = TC_WGRAD; q.wg_kind = WG_X; q.groups = 1; q.M = nx; q.Kdim = Tp;
    q.n_tiles_n = (d + kTileN - 1) / kTileN;
    fill_sizes(q);
    LMOE_TRY(gemm(tm_dX_mn, tm_x_mn, q, (nx + kTileM - 1) / kTileM * q.n_tiles_n));
  }
  if (g->b_router) {
    ++L;
    LMOE_TRY(launch_bias_grad(b.ds, w.offsets, w.perm, N, g->b_router, s));
  }
  // grouped: expert e reduces over its padded rows [offsets[e], offsets[e + 1]),
  // whose padding rows must be zero in both operands (zp's already are)
  {
    ++L;
    PadRowsArgs pr = {};
    pr.ptr[0] = b.DO; pr.cols[0] = l;
    pr.ptr[1] = w.H; pr.cols[1] = m;
    pr.ptr[2] = b.dAB; pr.cols[2] = gu;
    LMOE_TRY(launch_zero_pad_rows(w.offsets, w.seg_end, N, pr, s));
  }
  {
    TcParams p = {};  // dW_o[e] = DO_e^T H_e
    p.mode = TC_WGRAD; p.wg_kind = WG_O; p.groups = N; p.M = l; p.Kdim = 64;
    p.k_start = w.offsets; p.k_len = nullptr;
    p.n_tiles_n = (m + kTileN - 1) / kTileN;
    fill_sizes(p);
    LMOE_TRY(gemm(h->tm_DOmn, h->tm_Hmn, p, N * ((l + kTileM - 1) / kTileM) * p.n_tiles_n));
  }
  {
    TcParams p = {};  // [dW_g ; dW_u][e] = dAB_e^T zp_e
    p.mode = TC_WGRAD; p.wg_kind = WG_GU; p.groups = N; p.M = gu; p.Kdim = 64;
    p.k_start = w.offsets; p.k_len = nullptr;
    p.n_tiles_n = (l + kTileN - 1) / kTileN;
    fill_sizes(p);
    LMOE_TRY(gemm(h->tm_dABmn, h->tm_zpmn, p, N * ((gu + kTileM - 1) / kTileM) * p.n_tiles_n));
  }
#undef LMOE_TRY
  return cudaSuccess;
}

int lmoe_backward(lmoe_handle h, const void *x, const void *dy, void *dx, const lmoe_grads *g,
                  int32_t T, void *stream) {
  int rc = check_call(h, T);
  if (rc != LMOE_OK) return rc;
  if (!h->training) return LMOE_ERR_UNSUPPORTED;
  if (!g || !g->w_router || !g->w_down || !g->w_up || !g->w_upx || !g->w_out)
    return LMOE_ERR_NULL_ARG;
  if (!h->relu2 && !g->w_gate) return LMOE_ERR_NULL_ARG;
  if (h->cfg.has_router_bias && !g->b_router) return LMOE_ERR_NULL_ARG;
  if (h->ns > 0 && (!g->s_up || !g->s_out || (!h->relu2 && !g->s_gate))) return LMOE_ERR_NULL_ARG;
  if (T > 0 && (!x || !dy || !dx)) return LMOE_ERR_NULL_ARG;
  if (T > 0 && (!aligned16(x) || !aligned16(dy) || !aligned16(dx))) return LMOE_ERR_MISALIGNED;
  {
    const float *used[] = {g->w_router, g->w_down, g->w_up, g->w_upx, g->w_out,
                           h->relu2 ? nullptr : g->w_gate,
                           h->ns > 0 ? g->s_up : nullptr, h->ns > 0 ? g->s_out : nullptr,
                           (h->ns > 0 && !h->relu2) ? g->s_gate : nullptr};
    for (const float *q : used)
      if (q && !aligned16(q)) return LMOE_ERR_MISALIGNED;
  }
  DeviceGuard guard(h->device);
  if (!guard.ok) return LMOE_ERR_CUDA;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const size_t N = h->N, d = h->d, l = h->l, m = h->m, nsms = static_cast<size_t>(h->ns) * h->ms;
  if (T == 0) {  // no tokens: every gradient is zero
    cudaError_t e = cudaSuccess;
    auto z = [&](float *p, size_t n) { if (p && e == cudaSuccess) e = cudaMemsetAsync(p, 0, n * 4, s); };
    z(g->w_router, N * d); z(g->b_router, N); z(g->w_down, l * d); z(g->w_up, d * l);
    z(g->w_gate, N * m * l); z(g->w_upx, N * m * l); z(g->w_out, N * l * m);
    z(g->s_gate, nsms * d); z(g->s_up, nsms * d); z(g->s_out, d * nsms);
    return cuda_err(e);
  }
  if (h->bf16) return cuda_err(backward_bf16(h, x, dy, dx, g, T, s));
  return cuda_err(backward_f32(h, static_cast<const float *>(x), static_cast<const float *>(dy),
                               static_cast<float *>(dx), g, T, s));
}

int lmoe_forward_host(lmoe_handle h, const void *x_host, void *y_host, int32_t T, void *stream) {
  int rc = check_call(h, T);
  if (rc != LMOE_OK) return rc;
  if (h->ep_world > 1) return LMOE_ERR_UNSUPPORTED;
  if (T == 0) return LMOE_OK;
  if (!x_host || !y_host) return LMOE_ERR_NULL_ARG;
  DeviceGuard g(h->device);
  if (!g.ok) return LMOE_ERR_CUDA;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  // A pipeline over token chunks: chunk c's copy in (h2d stream), its forward
  // (the caller's stream) and its copy out (d2h stream) run while the other
  // chunks copy or compute.  Every token's output is computed exactly as in
  // one call (the layer is row-wise in the tokens), only the order of work
  // changes.  Chunks of at least kHostChunkTokens tokens, at most kHostChunks.
  const int n_chunks = std::max(1, std::min(kHostChunks, T / kHostChunkTokens));
  const size_t row_bytes = static_cast<size_t>(h->d) * h->esize;
  const uint8_t *xh = static_cast<const uint8_t *>(x_host);
  uint8_t *yh = static_cast<uint8_t *>(y_host);
  uint8_t *xd = static_cast<uint8_t *>(h->ws.x_stage), *yd = static_cast<uint8_t *>(h->ws.y_stage);
  // the copies start after the work already queued on the caller's stream
  if (cudaEventRecord(h->ev_start, s) != cudaSuccess ||
      cudaStreamWaitEvent(h->h2d, h->ev_start, 0) != cudaSuccess)
    return LMOE_ERR_CUDA;
  for (int c = 0; c < n_chunks; ++c) {
    const int t0 = static_cast<int>(static_cast<int64_t>(T) * c / n_chunks);
    const int t1 = static_cast<int>(static_cast<int64_t>(T) * (c + 1) / n_chunks);
    const size_t off = static_cast<size_t>(t0) * row_bytes, bytes = (t1 - t0) * row_bytes;
    if (cudaMemcpyAsync(xd + off, xh + off, bytes, cudaMemcpyHostToDevice, h->h2d) != cudaSuccess ||
        cudaEventRecord(h->ev_in[c], h->h2d) != cudaSuccess ||
        cudaStreamWaitEvent(s, h->ev_in[c], 0) != cudaSuccess)
      return LMOE_ERR_CUDA;
    rc = forward_impl(h, xd + off, yd + off, t1 - t0, s);
    if (rc != LMOE_OK) return rc;
    if (cudaEventRecord(h->ev_out[c], s) != cudaSuccess ||
        cudaStreamWaitEvent(h->d2h, h->ev_out[c], 0) != cudaSuccess ||
        cudaMemcpyAsync(yh + off, yd + off, bytes, cudaMemcpyDeviceToHost, h->d2h) != cudaSuccess)
      return LMOE_ERR_CUDA;
  }
  if (cudaStreamSynchronize(h->d2h) != cudaSuccess) return LMOE_ERR_CUDA;
  return cuda_err(cudaStreamSynchronize(s));
}

int lmoe_forward_host_batches(lmoe_handle h, int32_t n_batches, const void *const *x_hosts,
                              void *const *y_hosts, int32_t T, void *stream) {
  int rc = check_call(h, T);
  if (rc != LMOE_OK) return rc;
  if (h->ep_world > 1) return LMOE_ERR_UNSUPPORTED;
  if (n_batches < 0) return LMOE_ERR_INVALID_CONFIG;
  if (n_batches == 0 || T == 0) return LMOE_OK;
  if (!x_hosts || !y_hosts) return LMOE_ERR_NULL_ARG;
  for (int b = 0; b < n_batches; ++b)
    if (!x_hosts[b] || !y_hosts[b]) return LMOE_ERR_NULL_ARG;
  DeviceGuard g(h->device);
  if (!g.ok) return LMOE_ERR_CUDA;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  // Batch b uses staging set b % 2: its copy in (h2d stream) overlaps batch
  // b - 1's forward (the caller's stream), and its copy out (d2h stream) the
  // forward of batch b + 1.  A set is refilled only after batch b - 2's
  // forward has read x from it (ev_done) and its copy out has read y
  // (ev_yfree).
  const size_t bytes = static_cast<size_t>(T) * h->d * h->esize;
  void *xd[2] = {h->ws.x_stage, h->ws.x_stage2}, *yd[2] = {h->ws.y_stage, h->ws.y_stage2};
  // the copies start after the work already queued on the caller's stream
  if (cudaEventRecord(h->ev_start, s) != cudaSuccess ||
      cudaStreamWaitEvent(h->h2d, h->ev_start, 0) != cudaSuccess)
    return LMOE_ERR_CUDA;
  for (int b = 0; b < n_batches; ++b) {
    const int k = b & 1;
    if (b >= 2 && cudaStreamWaitEvent(h->h2d, h->ev_done[k], 0) != cudaSuccess)
      return LMOE_ERR_CUDA;
    if (cudaMemcpyAsync(xd[k], x_hosts[b], bytes, cudaMemcpyHostToDevice, h->h2d) != cudaSuccess ||
        cudaEventRecord(h->ev_in[k], h->h2d) != cudaSuccess ||
        cudaStreamWaitEvent(s, h->ev_in[k], 0) != cudaSuccess)
      return LMOE_ERR_CUDA;
    if (b >= 2 && cudaStreamWaitEvent(s, h->ev_yfree[k], 0) != cudaSuccess) return LMOE_ERR_CUDA;
    rc = forward_impl(h, xd[k], yd[k], T, s);
    if (rc != LMOE_OK) return rc;
    if (cudaEventRecord(h->ev_done[k], s) != cudaSuccess ||
        cudaStreamWaitEvent(h->d2h, h->ev_done[k], 0) != cudaSuccess ||
        cudaMemcpyAsync(y_hosts[b], yd[k], bytes, cudaMemcpyDeviceToHost, h->d2h) != cudaSuccess ||
        cudaEventRecord(h->ev_yfree[k], h->d2h) != cudaSuccess)
      return LMOE_ERR_CUDA;
  }
  if (cudaStreamSynchronize(h->d2h) != cudaSuccess) return LMOE_ERR_CUDA;
  return cuda_err(cudaStreamSynchronize(s));
}

int lmoe_get_dims(lmoe_handle h, int32_t *l, int32_t *n_routed, int32_t *k_active) {
  if (!h) return LMOE_ERR_NULL_ARG;
  if (l) *l = h->l;
  if (n_routed) *n_routed = h->N;
  if (k_active) *k_active = h->K;
  return LMOE_OK;
}

int lmoe_device_status(lmoe_handle h, void *stream) {
  if (!h) return LMOE_ERR_NULL_ARG;
  DeviceGuard g(h->device);
  if (!g.ok) return LMOE_ERR_CUDA;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(s) != cudaSuccess) return LMOE_ERR_CUDA;
  int32_t st = 0;
  if (cudaMemcpy(&st, h->ws.status, sizeof(st), cudaMemcpyDeviceToHost) != cudaSuccess)
    return LMOE_ERR_CUDA;
  if (st != 0) {
    cudaMemset(h->ws.status, 0, sizeof(st));
    return LMOE_ERR_DEVICE_TIMEOUT;
  }
  return LMOE_OK;
}

int lmoe_selftest_wait_timeout(lmoe_handle h, int64_t limit_ns, void *stream) {
  if (!h) return LMOE_ERR_NULL_ARG;
  if (limit_ns <= 0 || limit_ns > 2000000000LL) return LMOE_ERR_INVALID_CONFIG;
  DeviceGuard g(h->device);
  if (!g.ok) return LMOE_ERR_CUDA;
  return cuda_err(launch_wait_selftest(h->ws.status, limit_ns, static_cast<cudaStream_t>(stream)));
}

int lmoe_debug_buffer(lmoe_handle h, int32_t which, void **dev_ptr, int64_t *numel) {
  if (!h || !dev_ptr || !numel) return LMOE_ERR_NULL_ARG;
  const int64_t T = h->Tmax, TK = static_cast<int64_t>(h->Tmax) * h->K;
  const Workspace &w = h->ws;
  switch (which) {
    case 0: *dev_ptr = w.logits; *numel = T * h->N; break;
    case 1: *dev_ptr = w.z; *numel = T * h->l; break;
    case 2: *dev_ptr = w.zp; *numel = TK * h->l; break;
    case 3: *dev_ptr = w.H; *numel = TK * h->m; break;
    case 4: *dev_ptr = w.O; *numel = TK * h->l; break;
    case 5: *dev_ptr = w.ucat; *numel = T * h->ky; break;
    case 6: *dev_ptr = w.ids; *numel = TK; break;
    case 7: *dev_ptr = w.gates; *numel = TK; break;
    case 8: *dev_ptr = w.offsets; *numel = h->N + 1; break;
    case 9: *dev_ptr = w.perm; *numel = TK; break;
    case 10: *dev_ptr = w.pos; *numel = TK; break;
    case 11: *dev_ptr = w.n_tiles; *numel = 1; break;
    case 12: case 13: case 14: case 15: {
      if (!h->fp8) return LMOE_ERR_INVALID_CONFIG;
      const int64_t gu_bytes = h->fp4 ? static_cast<int64_t>(
                                            nvfp4_weight_code_bytes(h->N, h->gu_rows, h->l))
                                      : btile_rows(h->N, h->gu_rows, h->l) * 64;
      const int64_t o_bytes = h->fp4 ? static_cast<int64_t>(nvfp4_weight_code_bytes(h->N, h->l, h->m))
                                     : btile_rows(h->N, h->l, h->m) * 64;
      if (which == 12) { *dev_ptr = h->w_gu8; *numel = gu_bytes; }
      if (which == 13) { *dev_ptr = h->gu_scale; *numel = static_cast<int64_t>(h->N) * h->gu_rows; }
      if (which == 14) { *dev_ptr = h->w_o8; *numel = o_bytes; }
      if (which == 15) { *dev_ptr = h->o_scale; *numel = static_cast<int64_t>(h->N) * h->l; }
      break;
    }
    case 16: case 17: case 18: case 19: {
      if (!h->fp8) return LMOE_ERR_INVALID_CONFIG;
      const int64_t div = h->fp4 ? 2 : 1;  // packed NVFP4 rows
      if (which == 16) { *dev_ptr = w.zq; *numel = TK * h->l / div; }
      if (which == 17) { *dev_ptr = w.zq_scale; *numel = TK; }
      if (which == 18) { *dev_ptr = w.hq; *numel = TK * h->m / div; }
      if (which == 19) { *dev_ptr = w.hq_scale; *numel = TK; }
      break;
    }
    case 20: case 21: case 22: case 23:
      if (!h->fp4) return LMOE_ERR_INVALID_CONFIG;
      if (which == 20) {
        *dev_ptr = h->gu_sf;
        *numel = static_cast<int64_t>(nvfp4_weight_sf_bytes(h->N, h->gu_rows, h->l));
      }
      if (which == 21) {
        *dev_ptr = h->o_sf;
        *numel = static_cast<int64_t>(nvfp4_weight_sf_bytes(h->N, h->l, h->m));
      }
      if (which == 22) {
        *dev_ptr = w.zq_sf;
        *numel = static_cast<int64_t>(nvfp4_act_sf_bytes(h->max_tiles, h->l));
      }
      if (which == 23) {
        *dev_ptr = w.hq_sf;
        *numel = static_cast<int64_t>(nvfp4_act_sf_bytes(h->max_tiles, h->m));
      }
      break;
    default: return LMOE_ERR_INVALID_CONFIG;
  }
  return LMOE_OK;
}

static void free_events(lmoe_layer *h) {
  if (!h->ev) return;
  for (int64_t i = 0; i < static_cast<int64_t>(h->prof_slots) * (LMOE_NUM_STAGES + 1); ++i)
    if (h->ev[i]) cudaEventDestroy(h->ev[i]);
  free(h->ev);
  h->ev = nullptr;
  h->prof_slots = 0;
}

int lmoe_profile(lmoe_handle h, int32_t slots) {
  if (!h) return LMOE_ERR_NULL_ARG;
  if (slots < 0) return LMOE_ERR_INVALID_CONFIG;
  DeviceGuard g(h->device);
  if (!g.ok) return LMOE_ERR_CUDA;
  free_events(h);
  h->prof_count = 0;
  if (slots == 0) return LMOE_OK;
  const int64_t n = static_cast<int64_t>(slots) * (LMOE_NUM_STAGES + 1);
  h->ev = static_cast<cudaEvent_t *>(calloc(static_cast<size_t>(n), sizeof(cudaEvent_t)));
  if (!h->ev) return LMOE_ERR_OUT_OF_MEMORY;
  h->prof_slots = slots;
  for (int64_t i = 0; i < n; ++i)
    if (cudaEventCreate(&h->ev[i]) != cudaSuccess) {
      free_events(h);
      return LMOE_ERR_CUDA;
    }
  return LMOE_OK;
}

int lmoe_stage_times(lmoe_handle h, float *ms, int32_t n, int32_t *n_forwards,
                     int64_t *launches) {
  if (!h) return LMOE_ERR_NULL_ARG;
  if (launches) *launches = h->launches;
  const int64_t recs = h->prof_slots > 0
                           ? (h->prof_count < h->prof_slots ? h->prof_count : h->prof_slots)
                           : 0;
  if (n_forwards) *n_forwards = static_cast<int32_t>(recs);
  if (!ms || n <= 0) return LMOE_OK;
  for (int i = 0; i < n; ++i) ms[i] = 0.0f;
  DeviceGuard g(h->device);
  if (!g.ok) return LMOE_ERR_CUDA;
  for (int64_t r = 0; r < recs; ++r) {
    cudaEvent_t *e = h->ev + r * (LMOE_NUM_STAGES + 1);
    if (cudaEventSynchronize(e[LMOE_NUM_STAGES]) != cudaSuccess) return LMOE_ERR_CUDA;
    for (int i = 0; i < n && i < LMOE_NUM_STAGES; ++i) {
      float t = 0.0f;
      if (cudaEventElapsedTime(&t, e[i], e[i + 1]) != cudaSuccess) return LMOE_ERR_CUDA;
      ms[i] += t;
    }
  }
  return LMOE_OK;
}

int lmoe_destroy(lmoe_handle h) {
  if (!h) return LMOE_OK;
  {
    DeviceGuard g(h->device);
    cudaDeviceSynchronize();
    free_all(h);
    free_events(h);
  }
  delete h;
  return LMOE_OK;
}

}  // extern "C"

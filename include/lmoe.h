/*
 * lmoe.h -- C ABI of the B200 (sm_100a) LatentMoE layer forward.
 *
 * The layer (sources: "LatentMoE: NVIDIA's Latent Mixture of Experts
 * Explained Through Equations, Architecture, Code and..." -- Figures 3, 6, 8
 * and 9 and the LatentMoE code module; the Latent-MoE GitHub README --
 * "Usage" and the eff / acc variants):
 *
 *   s   = x W_r^T (+ b_r)                 router on the full-width token x
 *   ids = top-K'(s), ties -> lower index   slot order = logit descending
 *   g   = softmax(s) at ids, renormalised to sum to 1 over the K' slots
 *   z   = x W_down^T                       d -> l = d / alpha, no bias
 *   u   = sum_k g_k E_{ids_k}(z),          E(v) = W_o (silu(W_g v) * (W_u v))
 *   y   = u W_up^T + sum_j S_j(x),         S_j: shared SwiGLU experts at width d
 *
 * Sizes: N' = alpha * n_experts, K' = alpha * top_k ("acc") or top_k ("eff"),
 * unless overridden.  y excludes the residual connection.
 *
 * Conventions for every call below:
 *   - Return value: LMOE_OK (0) or a negative LMOE_ERR_* code; no exceptions
 *     cross this boundary.  lmoe_strerror() names a code.
 *   - Pointers named *_dev / device pointers are CUDA device memory on the
 *     handle's device; *_host pointers are host memory (pinned or pageable).
 *     The caller owns every buffer it passes; the handle owns its weight
 *     copies and workspace (sized once at lmoe_create from max_tokens;
 *     lmoe_forward allocates nothing).
 *   - Matrices are row-major in nn.Linear [out][in] layout.
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *     stream).  Calls are asynchronous on it unless stated; one stream at a
 *     time per handle (the workspace is shared by all calls of a handle).
 *   - Errors found on the host are returned before anything is enqueued.
 *     Errors found on the device (a bounded wait that ran out) are recorded
 *     in a sticky status word that lmoe_device_status() reads.
 */
#ifndef LMOE_H
#define LMOE_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Variants of the Latent-MoE README: "eff" keeps K' = K, "acc" scales K' = alpha K. */
typedef enum { LMOE_EFF = 0, LMOE_ACC = 1 } lmoe_variant;

/* Element type of x, y and every weight.  LMOE_F32 runs fp32 CUDA-core
 * kernels end to end; LMOE_BF16 runs bf16 tensor-core (tcgen05) GEMMs with
 * fp32 accumulation and bf16 intermediates (z, expert hidden, expert out,
 * combined u, shared hidden). */
typedef enum { LMOE_F32 = 0, LMOE_BF16 = 1 } lmoe_dtype;

/* Expert activation.  LMOE_SWIGLU: E(v) = W_o (silu(W_g v) * (W_u v)), three
 * matrices.  LMOE_RELU2: E(v) = W_o (relu(W_u v))^2, two matrices -- the
 * Expert class of the article's code module, the activation its 95B running
 * example uses.  Shared experts use the same. */
typedef enum { LMOE_SWIGLU = 0, LMOE_RELU2 = 1 } lmoe_activation;

/* Element type of the routed experts in LMOE_BF16 mode.
 * LMOE_WEIGHTS_FP8: the expert GEMMs run in E4M3 on both operands
 * (tcgen05 kind::f8f6f4, fp32 accumulation), for the weight-streaming decode
 * regime ("LatentMoE Explained" puts an expert at about 22 MB in FP8; the
 * pages give no scaling recipe, this is the one chosen).  W_g, W_u and W_o
 * are stored as E4M3 with one power-of-two scale per weight row (the smallest
 * that brings the row's largest magnitude within 448); each token's z and
 * each expert's hidden vector are quantised the same way, per row, before
 * they are multiplied.  The layer then computes exactly with those quantised
 * operands.  Needs l and m multiples of 128.  Not with training = 1, not
 * with expert parallelism.
 * LMOE_WEIGHTS_NVFP4: the same with NVFP4 on both operands (the pages say
 * the shipped models were pretrained in NVFP4; the format is NVIDIA's
 * published one): E2M1 codes, one E4M3 scale per 16 consecutive elements of
 * a row, and a second-level power-of-two scale per row (the smallest with
 * the row's largest magnitude within 6 * 448).  Block scale b =
 * E4M3(block max / (6 s_row)), code = E2M1(x * rcp) with rcp = 1 / (b s_row)
 * rounded once, all in IEEE single precision, rounding to nearest even with
 * saturation.  The
 * expert GEMMs run tcgen05 kind::mxf4nvf4 (the tensor cores apply the block
 * scales, fp32 accumulation).  Same limits as LMOE_WEIGHTS_FP8. */
typedef enum {
  LMOE_WEIGHTS_BF16 = 0,
  LMOE_WEIGHTS_FP8 = 1,
  LMOE_WEIGHTS_NVFP4 = 2
} lmoe_weight_format;

enum {
  LMOE_OK = 0,
  LMOE_ERR_INVALID_CONFIG = -1,  /* d % alpha != 0, K' outside [1, N'], sizes <= 0 */
  LMOE_ERR_NULL_ARG = -2,        /* a required pointer is NULL */
  LMOE_ERR_NOT_LOADED = -3,      /* route/forward before lmoe_load_weights */
  LMOE_ERR_TOO_MANY_TOKENS = -4, /* T > max_tokens or T < 0 */
  LMOE_ERR_CUDA = -5,            /* a CUDA runtime / driver call failed */
  LMOE_ERR_DEVICE_TIMEOUT = -6,  /* a kernel's bounded wait ran out (status word) */
  LMOE_ERR_UNSUPPORTED = -7,     /* valid layer, but a shape this build does not tile */
  LMOE_ERR_OUT_OF_MEMORY = -8,   /* workspace or weight allocation failed */
  LMOE_ERR_MISALIGNED = -9       /* a device array does not start on a 16-byte
                                    boundary (cudaMalloc and torch allocations
                                    always do); refused before any launch */
};

/* Layer hyper-parameters.  Field names follow LatentMoEConfig of the
 * Latent-MoE README ("Usage"): d, m, n_experts (N), top_k (K), alpha,
 * n_shared, variant.  Additions: m_shared (shared-expert width), dtype,
 * n_routed_override / top_k_override (0 = derive N' and K' from the variant),
 * has_router_bias, max_tokens (workspace size; forward never allocates).
 * LMOE_BF16 additionally needs d, l, m_shared*n_shared to be multiples of 64,
 * N' a multiple of 32, and m, m_shared multiples of 128 (SwiGLU) or of 64
 * (squared ReLU); every mode needs N' <= 1024 (else LMOE_ERR_UNSUPPORTED). */
typedef struct {
  int32_t d, m, n_experts, top_k, alpha, n_shared, m_shared;
  int32_t variant;           /* lmoe_variant */
  int32_t dtype;             /* lmoe_dtype */
  int32_t n_routed_override; /* N' if > 0 */
  int32_t top_k_override;    /* K' if > 0 */
  int32_t has_router_bias;   /* 1: a float32 bias [N'] is added to the logits */
  int32_t max_tokens;        /* largest T any later call may pass */
  int32_t activation;        /* lmoe_activation */
  int32_t training;          /* 1: lmoe_backward is available (the handle
                                keeps the extra weight layouts and workspace
                                the backward needs); 0: forward only */
  int32_t weight_format;     /* lmoe_weight_format (bf16 dtype only) */
  int32_t ep_rank;           /* expert parallelism: this rank, in [0, ep_world) */
  int32_t ep_world;          /* ranks the N' routed experts are split over; 0 or
                                1 = no expert parallelism (see lmoe_ep_dispatch) */
} lmoe_config;

typedef struct lmoe_layer *lmoe_handle;

/* Device pointers to the caller's weights, element type = cfg.dtype (the
 * router bias is always float32), nn.Linear [out][in] row-major, each used
 * matrix starting on a 16-byte boundary (else LMOE_ERR_MISALIGNED):
 *   w_router [N'][d], b_router [N'] or NULL, w_down [l][d], w_up [d][l],
 *   w_gate [N'][m][l], w_upx [N'][m][l], w_out [N'][l][m],
 *   s_gate [n_s][m_s][d], s_up [n_s][m_s][d], s_out [n_s][d][m_s]
 * (s_* may be NULL when n_shared == 0; w_gate and s_gate are unused, and may
 * be NULL, for LMOE_RELU2, where w_upx / s_up are the up-projections). */
typedef struct {
  const void *w_router;
  const float *b_router;
  const void *w_down, *w_up;
  const void *w_gate, *w_upx, *w_out;
  const void *s_gate, *s_up, *s_out;
} lmoe_weights;

/* Validates *cfg, derives l, N', K', allocates the handle's workspace for
 * cfg->max_tokens tokens on the current CUDA device, and returns the handle
 * in *out.  Synchronous.  Errors: NULL_ARG, INVALID_CONFIG, UNSUPPORTED,
 * OUT_OF_MEMORY, CUDA. */
int lmoe_create(const lmoe_config *cfg, lmoe_handle *out);

/* Copies the weights into handle-owned device memory, repacked for the
 * kernels (bf16: router, W_down and the shared gate/up rows stacked into one
 * matrix over x; expert gate/up rows interleaved in blocks of 128; W_up and
 * the shared down-projections concatenated along their input dimension; and
 * every such matrix stored K-block tiled, one contiguous 256 x 64 block per
 * tile).  bf16 uses temporary device buffers and synchronises `stream`
 * before returning; fp32 is asynchronous (the caller's buffers may be freed
 * once `stream` has passed this call).  Errors: NULL_ARG, MISALIGNED,
 * OUT_OF_MEMORY, CUDA. */
int lmoe_load_weights(lmoe_handle h, const lmoe_weights *w, void *stream);

/* Routing only (router GEMM, softmax / top-K' / renormalise, dispatch).
 * x_dev [T][d]; outputs (device, any may be NULL):
 *   ids [T][K'] int32, slot order = logit descending, ties -> lower index;
 *   gates [T][K'] float32, summing to 1 per token;
 *   offsets [N'+1] int32, offsets[e] = number of (token, slot) pairs routed
 *     to experts < e (exclusive scan of the per-expert histogram);
 *   perm [T*K'] int32: perm[offsets[e] + r] = t*K' + k for the r-th token
 *     (ascending t) that chose expert e, in slot k.
 * x_dev starts on a 16-byte boundary.  T == 0 is allowed (offsets all 0).
 * Errors: NULL_ARG, NOT_LOADED, TOO_MANY_TOKENS, MISALIGNED, CUDA. */
int lmoe_route(lmoe_handle h, const void *x_dev, int32_t T, int32_t *ids,
               float *gates, int32_t *offsets, int32_t *perm, void *stream);

/* The layer forward: y_dev [T][d] = layer(x_dev [T][d]), element type
 * cfg.dtype.  x and y must not overlap and must start on 16-byte boundaries
 * (the kernels move them with 16-byte vectors and TMA).  Graph-capturable:
 * no host sync, no allocation.  T == 0 is a no-op.  The output is
 * deterministic for a given T.  A call of fewer than 2048 tokens whose dense
 * GEMMs (router and down-projection, output projection) have too few output
 * tiles to fill the GPU splits their reductions into slices summed in a fixed
 * order, so its y may differ from a larger call's y for the same tokens by
 * fp32 summation order (the routing is unaffected unless two scores tie to
 * within that rounding).  Errors: NULL_ARG, NOT_LOADED, TOO_MANY_TOKENS,
 * MISALIGNED, CUDA. */
int lmoe_forward(lmoe_handle h, const void *x_dev, void *y_dev, int32_t T, void *stream);

/* End-to-end variant with HOST buffers: copies x_host to a handle-owned
 * device staging buffer, runs the forward, copies y back to y_host, and
 * synchronises `stream` before returning.  For T >= 4096 the tokens are
 * split into up to 4 chunks of at least 2048: a chunk's copy in, forward and
 * copy out overlap the other chunks' (two handle-owned copy streams; the
 * forwards run on `stream` in order).  Each token's output is the one a
 * single lmoe_forward call over all T tokens computes, bit for bit (chunks
 * are never small enough to split their reductions).  Pinned host memory
 * gives full copy bandwidth and
 * the overlap.  Errors: as lmoe_forward. */
int lmoe_forward_host(lmoe_handle h, const void *x_host, void *y_host, int32_t T,
                      void *stream);

/* A sequence of host batches, for serving: n_batches independent forwards
 * of T tokens each, batch b from x_hosts[b] ([T][d], host memory) into
 * y_hosts[b] (caller-owned, [T][d]).  Batch b's copy in runs while batch
 * b - 1 computes and its copy out while batch b + 1 computes, through two
 * handle-owned device staging sets (allocated by lmoe_create; each holds
 * max_tokens * d elements of x and as many of y) and the two copy streams
 * of lmoe_forward_host; the forwards run on `stream` in batch order.  Each y is
 * the one lmoe_forward computes for that batch, bit for bit.  Returns after
 * `stream` and the copies have finished; pinned host memory gives the
 * overlap.  The arrays may repeat a buffer (the copies of one stream run in
 * batch order), but no y buffer may overlap an x buffer.  No counterpart in
 * the pages (host I/O around the layer).
 * Errors: NULL_ARG (a NULL array or entry with n_batches, T > 0),
 * INVALID_CONFIG (n_batches < 0), UNSUPPORTED (expert-parallel handle), and
 * those of lmoe_forward. */
int lmoe_forward_host_batches(lmoe_handle h, int32_t n_batches, const void *const *x_hosts,
                              void *const *y_hosts, int32_t T, void *stream);

/* Derived sizes: l = d / alpha, N', K'.  Any output pointer may be NULL. */
int lmoe_get_dims(lmoe_handle h, int32_t *l, int32_t *n_routed, int32_t *k_active);

/* Synchronises `stream`, then returns and clears the handle's sticky
 * device-side status (LMOE_OK or LMOE_ERR_DEVICE_TIMEOUT), or LMOE_ERR_CUDA
 * if the stream reports an error. */
int lmoe_device_status(lmoe_handle h, void *stream);

/* Failure-detection self-test.  Launches one warp that waits on an mbarrier
 * nothing ever completes, with the same bounded wait the GEMM kernels use
 * for every pipeline barrier, but limited to limit_ns (1 .. 2e9); when the
 * wait runs out the kernel records a timeout in the handle's status word and
 * returns, so the next lmoe_device_status gives LMOE_ERR_DEVICE_TIMEOUT and
 * the context stays usable.  It does not fault or hang the GPU.  No
 * counterpart in the pages (test infrastructure for the status word).
 * Errors: NULL_ARG, INVALID_CONFIG (limit out of range), CUDA. */
int lmoe_selftest_wait_timeout(lmoe_handle h, int64_t limit_ns, void *stream);

/* Test and profiling hook: the device address and element count of one of
 * the handle's intermediate buffers after the last call on the stream
 * (which: 0 logits f32 [T][N'], 1 z [T][l], 2 permuted z [T*K'][l],
 * 3 expert hidden [T*K'][m], 4 expert out [T*K'][l], 5 [u | shared hidden]
 * [T][l + n_s m_s], 6 ids, 7 gates, 8 offsets, 9 perm, 10 pos [T*K'] (inverse
 * of perm), 11 number of 128-row expert tiles; with LMOE_WEIGHTS_FP8 also
 * 12 gate/up E4M3 codes and 14 W_o E4M3 codes (bytes, in 256 x 128 blocks:
 * expert, 256-row tile, 128-column block, row, column), 13 gate/up row scales
 * [N'][2m, gate and up rows interleaved in blocks of 128; m rows of W_u for
 * squared ReLU] and 15 W_o row scales [N'][l], f32; 16 the E4M3 codes of the
 * experts' input rows [T*K'][l] (z in dispatch order) and 17 their row scales
 * [T*K'] f32; 18 the E4M3 codes of the expert hidden rows [T*K'][m] and 19
 * their row scales [T*K'] f32).  With LMOE_WEIGHTS_NVFP4 the same ids hold
 * the NVFP4 counterparts -- 12 / 14 the packed E2M1 weight codes (two per
 * byte, element 2i in the low nibble of byte i) in 256-row x 128-byte blocks
 * (expert, 256-row tile, 256-element K-block, row, byte), 13 / 15 the row
 * scales, 16 / 18 the packed activation codes [T*K'][l / 2] and [T*K'][m / 2],
 * 17 / 19 their row scales -- and also 20 / 21 the weights' E4M3 block scales
 * (bytes; per expert, 256-row tile and K-block 4 KB: for each 128-row half
 * and each 64-element slice of the K-block a 512-byte atom in which row
 * r0 + 32 r1 (r0 < 32, r1 < 4) holds its four scales at bytes 16 r0 + 4 r1
 * .. + 3) and 22 / 23 the activations' block scales (per 128-row tile of
 * debug buffer 11's count, in dispatch order of the experts, and K-block
 * 2 KB: the four slices' atoms of the tile's rows).  Errors: NULL_ARG,
 * INVALID_CONFIG (unknown `which`). */
int lmoe_debug_buffer(lmoe_handle h, int32_t which, void **dev_ptr, int64_t *numel);

/* Profiling hook.  slots > 0: every later lmoe_forward on this handle also
 * records CUDA events on its stream before the first stage and after each
 * stage (stages, in order: 0 router + W_down GEMM over x, 1 top-K', 2
 * dispatch, 3 permute z, 4 expert gate/up GEMM, 5 expert down GEMM, 6
 * combine, 7 output GEMM; the fp32 mode maps its kernels onto the same
 * indices; the bf16 shared experts' gate/up GEMM runs on a side stream during
 * stages 1-3 and is not timed separately), into a ring of `slots` event sets
 * created here (never in the forward).  slots == 0 turns profiling off.
 * Errors: NULL_ARG, CUDA. */
#define LMOE_NUM_STAGES 8
int lmoe_profile(lmoe_handle h, int32_t slots);

/* Per-stage milliseconds summed over the profiled forwards still in the ring
 * (the last min(count, slots) since lmoe_profile); waits for their events.
 * ms[i] for i < min(n, LMOE_NUM_STAGES) (ms may be NULL); *n_forwards = how
 * many forwards were summed; *launches = kernel launches this handle has made
 * in total.  Any output may be NULL.  Errors: NULL_ARG, CUDA. */
int lmoe_stage_times(lmoe_handle h, float *ms, int32_t n, int32_t *n_forwards,
                     int64_t *launches);

/* ---- Expert parallelism ("Shaping Latent MoE", Figure 6: the routed experts
 * sit between W_down and W_up, so the tokens cross between devices in the
 * latent width l; "LatentMoE Explained", Figure 12 and the passage on the
 * all-to-all that runs twice per expert layer).
 *
 * A handle created with ep_world = W > 1 and ep_rank = r holds the router,
 * W_down, W_up and the shared experts (replicated on every rank) and the
 * routed experts [r * N'/W, (r+1) * N'/W) only: in lmoe_load_weights,
 * w_gate / w_upx / w_out then point at those N'/W experts ([N'/W][m][l],
 * [N'/W][m][l], [N'/W][l][m]).  N' must be a multiple of W; bf16 dtype,
 * bf16 expert weights, no training.  lmoe_forward and lmoe_backward return
 * LMOE_ERR_UNSUPPORTED on such a handle; lmoe_route works.  One forward of
 * the layer on rank r is, in order on one stream:
 *
 *   1. lmoe_ep_dispatch(x [T][d]) -> send rows + expert counts
 *   2. (caller) exchange: every rank sends its rows for rank q's experts to
 *      rank q -- counts first, then the rows (an all-to-all with splits) --
 *      so that rank q receives, source rank by source rank, the rows for its
 *      experts;
 *   3. lmoe_ep_experts(received rows) -> expert outputs, same row order
 *   4. (caller) exchange back: the outputs return to their source ranks in
 *      the order they were sent;
 *   5. lmoe_ep_combine(returned rows) -> y [T][d].
 *
 * The exchanged rows are l wide (not d): z rows go out, expert-output rows
 * come back.  Steps 1 and 5 must use the same handle, with no other call on
 * it in between: the routing (ids, gates, positions) and the shared experts'
 * hidden of step 1 stay in the handle's workspace for step 5.  Step 3 uses
 * its own workspace, so it may run between them on the same stream. */

/* Step 1.  Routes x_dev [T][d] over all N' experts and writes
 * send_rows_dev [T*K'][l] (bf16): row p is z of the token in dispatch
 * position p (lmoe_route's perm order: experts ascending, tokens ascending
 * within an expert), so the rows for rank q are the contiguous range of
 * experts [q N'/W, (q+1) N'/W); and expert_counts_dev [N'] int32, the
 * number of rows per expert.  Rows past the T*K' actually routed are not
 * written.  x and send_rows start on 16-byte boundaries.  Errors: NULL_ARG,
 * NOT_LOADED, TOO_MANY_TOKENS, MISALIGNED, UNSUPPORTED (not an
 * expert-parallel handle), CUDA. */
int lmoe_ep_dispatch(lmoe_handle h, const void *x_dev, int32_t T, void *send_rows_dev,
                     int32_t *expert_counts_dev, void *stream);

/* Step 3.  recv_rows_dev [R][l] (bf16): the rows received from every source
 * rank s = 0..W-1 in turn, each source's rows grouped by this rank's local
 * experts in order (exactly what step 1's send rows give after the
 * exchange); recv_counts_dev [W][N'/W] int32 on the device: rows from source
 * s for local expert e.  Writes out_rows_dev [R][l] (bf16), row i =
 * E_e(row i) for the row's expert e, the latent expert l -> m -> l ("LatentMoE
 * Explained", Figure 9), not yet gate-weighted.  R = the sum of
 * recv_counts, at most W * max_tokens * K'.  Buffers start on 16-byte
 * boundaries.  Errors: NULL_ARG, NOT_LOADED, TOO_MANY_TOKENS (R out of
 * range), MISALIGNED, UNSUPPORTED, CUDA. */
int lmoe_ep_experts(lmoe_handle h, const void *recv_rows_dev, const int32_t *recv_counts_dev,
                    int32_t R, void *out_rows_dev, void *stream);

/* Step 5.  back_rows_dev [T*K'][l] (bf16): the expert outputs returned to
 * this rank, in the order of step 1's send rows.  Combines them with the
 * gates of step 1 in slot order and writes y_dev [T][d] = u W_up^T + the
 * shared experts of x (T must equal step 1's).  Buffers start on 16-byte
 * boundaries.  Errors: NULL_ARG, NOT_LOADED, TOO_MANY_TOKENS, MISALIGNED,
 * UNSUPPORTED, CUDA. */
int lmoe_ep_combine(lmoe_handle h, const void *back_rows_dev, void *y_dev, int32_t T,
                    void *stream);

/* Dispatch without allocation.  The paper has no counterpart to this call:
 * it exists for callers that may not call cudaMalloc where they need the
 * dispatch -- for instance a serving loop whose device memory is entirely
 * reserved up front by its own pool allocator, or a plugin whose host
 * framework forbids allocation inside its execute callback.
 *
 * Given ids [T][k_active] int32 on the device (as lmoe_route produces them:
 * every id in [0, n_routed), no id twice in a row), writes offsets
 * [n_routed+1] and perm [T*k_active] exactly as lmoe_route does,
 * asynchronously on `stream`.  Other ids are tolerated without any
 * out-of-bounds access: a pair whose id lies outside [0, n_routed) is
 * skipped (not counted in offsets, not placed in perm), so offsets[n_routed]
 * is the number of pairs placed and perm from that index on holds -1; a row
 * that names one expert twice places both pairs at one position of that
 * expert's range, and the position left over holds -1.
 * It needs no handle and calls no cudaMalloc, cudaFree or allocating
 * routine: its scratch (about 3 MiB) is one fixed file-scope device array
 * that every GPU loading this library holds until the process exits.
 *   - Limits: T <= LMOE_NOALLOC_MAX_TOKENS, T*k_active <=
 *     LMOE_NOALLOC_MAX_PAIRS (else LMOE_ERR_TOO_MANY_TOKENS), n_routed <=
 *     LMOE_NOALLOC_MAX_EXPERTS (else LMOE_ERR_UNSUPPORTED); k_active outside
 *     [1, n_routed] or T < 0 gives LMOE_ERR_INVALID_CONFIG; NULL offsets, or
 *     NULL ids / perm with T > 0, gives LMOE_ERR_NULL_ARG.
 *   - The first call on each device looks up the array's device address
 *     (cudaGetSymbolAddress, with that device current); make that first call
 *     before any stream capture.  The address is kept until the process
 *     exits, so do not call this after cudaDeviceReset on that device.
 *   - All calls on a device share the one array, and it keeps the last
 *     call's contents (each call rewrites every word it reads).  Calls that
 *     overlap on the GPU -- on different streams, or from different threads
 *     -- race on it and give wrong results; serialise them.
 * Errors: as listed above, and LMOE_ERR_CUDA. */
#define LMOE_NOALLOC_MAX_TOKENS 65536
#define LMOE_NOALLOC_MAX_PAIRS 262144
#define LMOE_NOALLOC_MAX_EXPERTS 1024
int lmoe_dispatch_noalloc(const int32_t *ids, int32_t T, int32_t k_active, int32_t n_routed,
                          int32_t *offsets, int32_t *perm, void *stream);

/* Weight gradients of one lmoe_backward call: float32 device arrays in the
 * layouts of lmoe_weights (w_router [N'][d], b_router [N'], w_down [l][d],
 * w_up [d][l], w_gate / w_upx [N'][m][l], w_out [N'][l][m], s_gate / s_up
 * [n_s][m_s][d], s_out [n_s][d][m_s]), caller-owned, overwritten (not
 * accumulated).  b_router is required only with has_router_bias; w_gate and
 * s_gate are unused (may be NULL) for LMOE_RELU2; s_* may be NULL when
 * n_shared == 0. */
typedef struct {
  float *w_router, *b_router, *w_down, *w_up;
  float *w_gate, *w_upx, *w_out;
  float *s_gate, *s_up, *s_out;
} lmoe_grads;

/* The layer backward: for the cotangent dy_dev [T][d] of y = layer(x_dev),
 * writes dx_dev [T][d] (element type cfg.dtype) and the weight gradients
 * *grads -- what loss.backward() computes for this layer in the Latent-MoE
 * README's Usage example.  The pages print no gradient formulas: it is the
 * chain rule through the forward ("LatentMoE Explained": Figure 3 router,
 * Figure 6 W_down / W_up, Figure 9 latent expert, the LatentMoE code
 * module's softmax / top-K / renormalise and slot loop); the top-K
 * selection is piecewise constant, so the router's gradient flows through
 * the renormalised gates of the selected experts only.  Stateless: the call
 * recomputes the forward activations it needs from x_dev (same routing as
 * lmoe_forward).  Weight gradients sum the T tokens in a fixed order
 * (deterministic).  Needs a handle created with training = 1.  No host
 * sync; T == 0 writes zero gradients.  x, dy and dx must not overlap; they
 * and the gradient arrays (b_router excepted) start on 16-byte boundaries.
 * Errors: NULL_ARG, NOT_LOADED, TOO_MANY_TOKENS, UNSUPPORTED (handle without
 * training), MISALIGNED, CUDA. */
int lmoe_backward(lmoe_handle h, const void *x_dev, const void *dy_dev, void *dx_dev,
                  const lmoe_grads *grads, int32_t T, void *stream);

/* Human-readable name of a status code (static string). */
const char *lmoe_strerror(int code);

/* Frees the handle and everything it owns (synchronises the device first).
 * NULL is a no-op. */
int lmoe_destroy(lmoe_handle h);

#ifdef __cplusplus
}
#endif

#endif /* LMOE_H */

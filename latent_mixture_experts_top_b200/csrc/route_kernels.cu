// route_kernels.cu -- routing, dispatch, permutation and combine kernels.
//
// Sources: "LatentMoE Explained" (Towards AI), Figure 3 (router: one score
// per expert, softmax, top-K), the LatentMoE code module (top-K of the
// softmax, the selected weights renormalised to sum to one, and a slot loop
// that masks, expert by expert, the tokens that chose it and adds the gated
// expert output to theirs).  The pages' masked loop is
// replaced by a histogram -> exclusive scan -> stable scatter that yields the
// same grouping (experts in index order, tokens ascending within an expert)
// in three launches and no host synchronisation.
#include <cuda_bf16.h>
#include <stdint.h>

#include "common.cuh"
#include "kernels.h"

namespace lmoe {
namespace {

constexpr unsigned kFull = 0xFFFFFFFFu;

// Order-preserving map of a float to an unsigned key (larger float -> larger key).
__device__ __forceinline__ uint32_t float_key(float v) {
  const uint32_t u = __float_as_uint(v);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
__device__ __forceinline__ float key_float(uint32_t k) {
  return __uint_as_float((k & 0x80000000u) ? (k & 0x7FFFFFFFu) : ~k);
}

// ---------------------------------------------------------------- top-K'
// One warp per token.  Lane j holds experts e = 32 i + j (i < VPL) as 32-bit
// order-preserving keys of their logits.  The selection order is by key
// descending, and equal keys go to the lower expert index.  Gates: g_k =
// e^{s_k - s_0} / sum_j e^{s_j - s_0}, which equals softmax(s) at the selected
// experts renormalised to sum to one (the softmax denominator cancels).
//
// Each of the K' rounds takes the warp maximum of the candidate keys (one
// REDUX), then the smallest expert index holding that maximum (a second
// REDUX), and removes exactly that candidate.  With wbuf (64 entries of this
// warp's shared memory) and K' <= 32 the rounds run over a short candidate
// list: tau, the K'-th largest of the 32 lane maxima, is at most the K'-th
// largest key (those K' maxima are K' distinct keys), so every key of the
// top-K' is >= tau; when at most 64 keys reach tau they are gathered, two per
// lane, and the rounds take their maximum from two registers instead of VPL.
// Otherwise the rounds run over all VPL keys of each lane.  Both give the
// same selection.  The chosen expert of each slot is counted in hist[e]
// (shared memory) when hist is given, else in gcount[e * gstride] (global)
// when gcount is given.
__device__ __forceinline__ bool key_before(uint32_t ka, uint32_t ea, uint32_t kb, uint32_t eb) {
  return ka > kb || (ka == kb && ea < eb);
}

template <int VPL>
__device__ __forceinline__ void select_token(const float *__restrict__ logits, int ld,
                                             const float *__restrict__ bias, int N, int K, int t,
                                             int32_t *__restrict__ ids, float *__restrict__ gates,
                                             int *hist, int32_t *gcount, int gstride,
                                             uint2 *wbuf = nullptr) {
  const int lane = threadIdx.x & 31;
  const float *row = logits + static_cast<size_t>(t) * ld;
  uint32_t key[VPL];
#pragma unroll
  for (int i = 0; i < VPL; ++i) {
    const int e = i * 32 + lane;
    key[i] = e < N ? float_key(row[e] + (bias ? bias[e] : 0.0f)) : 0u;
  }
  int32_t *ids_row = ids + static_cast<size_t>(t) * K;
  float *g_row = gates + static_cast<size_t>(t) * K;
  // the lane of slot k (k < 32) keeps its key and expert
  uint32_t slot_key = 0u, slot_e = 0u;
  bool short_list = false;
  if (wbuf && K <= 32) {
    uint32_t lm = key[0];
#pragma unroll
    for (int i = 1; i < VPL; ++i) lm = max(lm, key[i]);
    // bitonic sort of the lane maxima, descending (lane 0 the largest)
    uint32_t v = lm;
#pragma unroll
    for (int k = 2; k <= 32; k <<= 1) {
#pragma unroll
      for (int j = k >> 1; j > 0; j >>= 1) {
        const uint32_t o = __shfl_xor_sync(kFull, v, j);
        v = (((lane & k) == 0) == ((lane & j) == 0)) ? max(v, o) : min(v, o);
      }
    }
    const uint32_t tau = __shfl_sync(kFull, v, K - 1);  // > 0: K <= N keys are real
    int c = 0;
#pragma unroll
    for (int i = 0; i < VPL; ++i) c += key[i] >= tau ? 1 : 0;
    const int total = static_cast<int>(__reduce_add_sync(kFull, static_cast<uint32_t>(c)));
    if (total <= 64) {
      short_list = true;
      int pos = c;
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const int y = __shfl_up_sync(kFull, pos, off);
        if (lane >= off) pos += y;
      }
      pos -= c;  // exclusive prefix: this lane's first entry
#pragma unroll
      for (int i = 0; i < VPL; ++i)
        if (key[i] >= tau) wbuf[pos++] = make_uint2(key[i], static_cast<uint32_t>(i * 32 + lane));
      __syncwarp();
      // two candidates per lane, a before b; empty entries: key 0
      uint2 a = lane < total ? wbuf[lane] : make_uint2(0u, 0xFFFFFFFFu);
      uint2 b = lane + 32 < total ? wbuf[lane + 32] : make_uint2(0u, 0xFFFFFFFFu);
      __syncwarp();  // wbuf may be refilled by the warp's next token
      if (key_before(b.x, b.y, a.x, a.y)) {
        const uint2 tmp = a;
        a = b;
        b = tmp;
      }
      for (int k = 0; k < K; ++k) {
        const uint32_t wm = __reduce_max_sync(kFull, a.x);
        const uint32_t e = __reduce_min_sync(kFull, a.x == wm ? a.y : 0xFFFFFFFFu);
        if (a.y == e) {  // the one lane that held it
          a = b;
          b = make_uint2(0u, 0xFFFFFFFFu);
        }
        if (lane == k) {
          slot_key = wm;
          slot_e = e;
        }
      }
    }
  }
  if (!short_list) {
    for (int k = 0; k < K; ++k) {
      uint32_t m = key[0];
#pragma unroll
      for (int i = 1; i < VPL; ++i) m = max(m, key[i]);
      const uint32_t wm = __reduce_max_sync(kFull, m);
      uint32_t cand = 0xFFFFFFFFu;
#pragma unroll
      for (int i = VPL - 1; i >= 0; --i)
        if (key[i] == wm) cand = static_cast<uint32_t>(i * 32 + lane);
      const uint32_t e = __reduce_min_sync(kFull, cand);
#pragma unroll
      for (int i = 0; i < VPL; ++i)
        if (static_cast<uint32_t>(i * 32 + lane) == e) key[i] = 0u;
      if ((k & 31) == lane) {  // slots past 32 go straight to memory
        if (k < 32) {
          slot_key = wm;
          slot_e = e;
        } else {
          ids_row[k] = static_cast<int32_t>(e);
          g_row[k] = key_float(wm);
          if (hist) atomicAdd(hist + e, 1);
          else if (gcount) atomicAdd(gcount + static_cast<size_t>(e) * gstride, 1);
        }
      }
    }
  }
  const float s0 = key_float(__shfl_sync(kFull, slot_key, 0));
  const bool mine = lane < K;
  const float ex = mine ? expf(key_float(slot_key) - s0) : 0.0f;
  float sum = ex;
  for (int k = lane + 32; k < K; k += 32) sum += expf(g_row[k] - s0);
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) sum += __shfl_xor_sync(kFull, sum, off);
  if (mine) {
    ids_row[lane] = static_cast<int32_t>(slot_e);
    g_row[lane] = ex / sum;
    if (hist) atomicAdd(hist + slot_e, 1);
    else if (gcount) atomicAdd(gcount + static_cast<size_t>(slot_e) * gstride, 1);
  }
  for (int k = lane + 32; k < K; k += 32) g_row[k] = expf(g_row[k] - s0) / sum;
}

// topk_kernel: one warp per token.  If `counts` is given ([N][n_chunks],
// zeroed), it also builds the per-chunk expert histogram of the dispatch
// (chunk = `chunk` tokens).
template <int VPL>
__global__ void __launch_bounds__(256) topk_kernel(const float *__restrict__ logits, int ld,
                                                   const float *__restrict__ bias, int T, int N,
                                                   int K, int32_t *__restrict__ ids,
                                                   float *__restrict__ gates,
                                                   int32_t *__restrict__ counts, int n_chunks,
                                                   int chunk) {
  const int t = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  if (t >= T) return;
  select_token<VPL>(logits, ld, bias, N, K, t, ids, gates, nullptr,
                    counts ? counts + t / chunk : nullptr, (n_chunks + 3) & ~3);
}

// ---------------------------------------------------------------- dispatch
// Count matrix layout: counts[e][c] (expert-major), c = token chunk, row
// stride n_chunks rounded up to a multiple of 4 (16-byte rows).
// Phase 1 (when the top-K kernel did not count): per-chunk expert histogram.
// check_ids: ids come from the caller, not from the top-K kernel, so an id
// outside [0, N) is skipped instead of indexing the histogram with it.
__global__ void __launch_bounds__(256) dispatch_count_kernel(const int32_t *__restrict__ ids,
                                                             int T, int K, int N,
                                                             int32_t *__restrict__ counts,
                                                             int n_chunks, int chunk,
                                                             int check_ids) {
  extern __shared__ int32_t cnt[];  // [N]
  for (int e = threadIdx.x; e < N; e += blockDim.x) cnt[e] = 0;
  __syncthreads();
  const int t0 = blockIdx.x * chunk;
  const int tn = min(chunk, T - t0);
  const int32_t *base = ids + static_cast<size_t>(t0) * K;
  for (int i = threadIdx.x; i < tn * K; i += blockDim.x) {
    const int e = base[i];
    if (!check_ids || static_cast<unsigned>(e) < static_cast<unsigned>(N)) atomicAdd(&cnt[e], 1);
  }
  __syncthreads();
  const int ncp = (n_chunks + 3) & ~3;
  for (int e = threadIdx.x; e < N; e += blockDim.x)
    counts[static_cast<size_t>(e) * ncp + blockIdx.x] = cnt[e];
}

// Inclusive scan across a block of up to 1024 threads; returns the exclusive
// prefix and writes the total to *total.
__device__ int block_exclusive_scan(int v, int *warp_sums, int *total) {
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5, nw = (blockDim.x + 31) >> 5;
  int x = v;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const int y = __shfl_up_sync(kFull, x, off);
    if (lane >= off) x += y;
  }
  if (lane == 31) warp_sums[w] = x;
  __syncthreads();
  if (w == 0) {
    int s = lane < nw ? warp_sums[lane] : 0;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int y = __shfl_up_sync(kFull, s, off);
      if (lane >= off) s += y;
    }
    if (lane < nw) warp_sums[lane] = s;  // inclusive warp prefix
  }
  __syncthreads();
  const int before = (w > 0 ? warp_sums[w - 1] : 0) + x - v;
  *total = warp_sums[nw - 1];
  __syncthreads();
  return before;
}

// Phase 2 (one block of 256 threads, each owning up to four experts -- a block
// small enough to run beside a GEMM CTA on the same SM): each thread scans the
// chunk counts of its experts (in place: counts[e][c] becomes the number of
// pairs of expert e in chunks before c); the expert totals are then scanned
// into offsets and the table of tile_m-row M-tiles is written, and, when
// tiles2 is given, a second table of tile_m2-row M-tiles (the CTA-pair GEMM's).
constexpr int kScanThreads = 256, kScanPerThread = 4;  // N <= 1024

__device__ int scan_expert_row(int32_t *counts, int e, int n_chunks) {
  // The row is contiguous (row stride n_chunks rounded up to 4): 16-byte
  // loads, eight in flight at a time.
  const int ncp = (n_chunks + 3) & ~3;
  int4 *row = reinterpret_cast<int4 *>(counts + static_cast<size_t>(e) * ncp);
  const int nv = ncp / 4;
  int tot = 0;
  for (int v0 = 0; v0 < nv; v0 += 8) {
    int4 q[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) q[j] = v0 + j < nv ? __ldcg(row + v0 + j) : make_int4(0, 0, 0, 0);
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      if (v0 + j >= nv) break;
      const int c = 4 * (v0 + j);
      int4 o;
      o.x = tot; tot += c + 0 < n_chunks ? q[j].x : 0;
      o.y = tot; tot += c + 1 < n_chunks ? q[j].y : 0;
      o.z = tot; tot += c + 2 < n_chunks ? q[j].z : 0;
      o.w = tot; tot += c + 3 < n_chunks ? q[j].w : 0;
      row[v0 + j] = o;
    }
  }
  return tot;
}

// Writes the table entries of expert e's M-tiles (tile_m rows each, the last
// one ragged) from index tstart on.
__device__ void write_tiles(TileEntry *tiles, int tstart, int max_tiles, int e, int off, int tot,
                            int tile_m) {
  const int mt = (tot + tile_m - 1) / tile_m;
  for (int j = 0; j < mt; ++j) {
    const int idx = tstart + j;
    if (idx < max_tiles) {
      TileEntry te;
      te.row0 = off + j * tile_m;
      te.row_end = off + tot;
      te.expert = e;
      te.pad = 0;
      tiles[idx] = te;
    }
  }
}

// Phase 2 body, run by one block of kScanThreads threads.
// Offsets and tile tables from the expert totals of this thread's experts
// e0 .. e0+3 (all threads of the block call it).  seg.pad > 1: each expert's
// rows start at a multiple of seg.pad (offsets[e] is the padded start,
// offsets[N] the padded total, seg.ends[e] = offsets[e] + the expert's count);
// the tile tables cover the real rows only.
__device__ void offsets_and_tables(const int (&tot)[kScanPerThread], int e0, int N, SegPad seg,
                                   int32_t *__restrict__ offsets, TileEntry *__restrict__ tiles,
                                   int32_t *__restrict__ n_tiles, int tile_m, int max_tiles,
                                   TileEntry *__restrict__ tiles2, int32_t *__restrict__ n_tiles2,
                                   int tile_m2, int max_tiles2) {
  __shared__ int warp_sums[32];
  int span[kScanPerThread], mt[kScanPerThread], mt2[kScanPerThread];
  int my_span = 0, my_mt = 0, my_mt2 = 0;
#pragma unroll
  for (int i = 0; i < kScanPerThread; ++i) {
    span[i] = seg.pad > 1 ? (tot[i] + seg.pad - 1) / seg.pad * seg.pad : tot[i];
    mt[i] = (tot[i] + tile_m - 1) / tile_m;
    mt2[i] = tiles2 ? (tot[i] + tile_m2 - 1) / tile_m2 : 0;
    my_span += span[i];
    my_mt += mt[i];
    my_mt2 += mt2[i];
  }
  int all = 0, all_tiles = 0, all_tiles2 = 0;
  int off = block_exclusive_scan(my_span, warp_sums, &all);
  int tstart = block_exclusive_scan(my_mt, warp_sums, &all_tiles);
  int tstart2 = block_exclusive_scan(my_mt2, warp_sums, &all_tiles2);
#pragma unroll
  for (int i = 0; i < kScanPerThread; ++i) {
    const int e = e0 + i;
    if (e < N) {
      offsets[e] = off;
      if (seg.ends) seg.ends[e] = off + tot[i];
      write_tiles(tiles, tstart, max_tiles, e, off, tot[i], tile_m);
      if (tiles2) write_tiles(tiles2, tstart2, max_tiles2, e, off, tot[i], tile_m2);
    }
    off += span[i];
    tstart += mt[i];
    tstart2 += mt2[i];
  }
  if (threadIdx.x == 0) {
    offsets[N] = all;
    *n_tiles = min(all_tiles, max_tiles);
    if (tiles2) *n_tiles2 = min(all_tiles2, max_tiles2);
  }
}

__device__ void scan_and_tables(int32_t *__restrict__ counts, int n_chunks, int N, SegPad seg,
                                int32_t *__restrict__ offsets, TileEntry *__restrict__ tiles,
                                int32_t *__restrict__ n_tiles, int tile_m, int max_tiles,
                                TileEntry *__restrict__ tiles2, int32_t *__restrict__ n_tiles2,
                                int tile_m2, int max_tiles2) {
  const int e0 = threadIdx.x * kScanPerThread;  // experts e0 .. e0+3
  int tot[kScanPerThread];
#pragma unroll
  for (int i = 0; i < kScanPerThread; ++i) {
    const int e = e0 + i;
    tot[i] = e < N ? scan_expert_row(counts, e, n_chunks) : 0;
  }
  offsets_and_tables(tot, e0, N, seg, offsets, tiles, n_tiles, tile_m, max_tiles, tiles2,
                     n_tiles2, tile_m2, max_tiles2);
}

__global__ void __launch_bounds__(kScanThreads) dispatch_scan_kernel(
    int32_t *__restrict__ counts, int n_chunks, int N, SegPad seg, int32_t *__restrict__ offsets,
    TileEntry *__restrict__ tiles, int32_t *__restrict__ n_tiles, int tile_m, int max_tiles,
    TileEntry *__restrict__ tiles2, int32_t *__restrict__ n_tiles2, int tile_m2,
    int max_tiles2) {
  scan_and_tables(counts, n_chunks, N, seg, offsets, tiles, n_tiles, tile_m, max_tiles, tiles2,
                  n_tiles2, tile_m2, max_tiles2);
}

// ---------------------------------------------------------------- fused routing
// Phase 2 for the fused routing launch: each row of the count matrix becomes
// the exclusive prefix of its chunk counts, as in scan_and_tables, and the
// row's total goes to totals[e].  The rows are independent, so the loads of
// several rows are issued before any row is scanned: the scan costs a few
// dependent memory round trips instead of two per row.
//
// Short rows (at most 8 vectors, 32 chunks): one row per thread, the whole
// row in registers, scanned serially.
__device__ __forceinline__ int scan_row_thread(int4 *row, int nv, int n_chunks) {
  int4 q[8];
#pragma unroll
  for (int v = 0; v < 8; ++v) q[v] = v < nv ? __ldcg(row + v) : make_int4(0, 0, 0, 0);
  int run = 0;
#pragma unroll
  for (int v = 0; v < 8; ++v) {
    if (v >= nv) break;
    const int c = 4 * v;
    int4 o;
    o.x = run; run += c + 0 < n_chunks ? q[v].x : 0;
    o.y = run; run += c + 1 < n_chunks ? q[v].y : 0;
    o.z = run; run += c + 2 < n_chunks ? q[v].z : 0;
    o.w = run; run += c + 3 < n_chunks ? q[v].w : 0;
    row[v] = o;
  }
  return run;
}

// Longer rows: one warp per row, R rows per warp at a time.  Lane j holds the
// PER consecutive vectors j*PER .. j*PER+PER-1 of each of its rows (entries
// past n_chunks are row padding and count as zero); the warp scans the lanes'
// sums, and each lane writes its run's prefixes.
template <int PER, int R>
__device__ __forceinline__ void scan_rows_warp(int32_t *__restrict__ counts, int ncp,
                                               int n_chunks, int N, int *totals) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nwarps = blockDim.x >> 5;
  const int nv = ncp / 4;
  for (int e0 = warp * R; e0 < N; e0 += nwarps * R) {
    int4 q[R][PER];
    int sum[R], incl[R];
#pragma unroll
    for (int r = 0; r < R; ++r) {
      const bool on = e0 + r < N;
      const int4 *row = reinterpret_cast<const int4 *>(counts + static_cast<size_t>(on ? e0 + r : 0) * ncp);
#pragma unroll
      for (int i = 0; i < PER; ++i) {
        const int v = lane * PER + i;
        q[r][i] = on && v < nv ? __ldcg(row + v) : make_int4(0, 0, 0, 0);
      }
    }
#pragma unroll
    for (int r = 0; r < R; ++r) {
      int s = 0;
#pragma unroll
      for (int i = 0; i < PER; ++i) {
        const int c = 4 * (lane * PER + i);
        s += (c + 0 < n_chunks ? q[r][i].x : 0) + (c + 1 < n_chunks ? q[r][i].y : 0) +
             (c + 2 < n_chunks ? q[r][i].z : 0) + (c + 3 < n_chunks ? q[r][i].w : 0);
      }
      sum[r] = s;
      incl[r] = s;
    }
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
#pragma unroll
      for (int r = 0; r < R; ++r) {
        const int y = __shfl_up_sync(kFull, incl[r], off);
        if (lane >= off) incl[r] += y;
      }
    }
#pragma unroll
    for (int r = 0; r < R; ++r) {
      const int e = e0 + r;
      if (e >= N) break;  // the same for every lane
      int4 *row = reinterpret_cast<int4 *>(counts + static_cast<size_t>(e) * ncp);
      int run = incl[r] - sum[r];
#pragma unroll
      for (int i = 0; i < PER; ++i) {
        const int v = lane * PER + i;
        if (v >= nv) break;
        const int c = 4 * v;
        int4 o;
        o.x = run; run += c + 0 < n_chunks ? q[r][i].x : 0;
        o.y = run; run += c + 1 < n_chunks ? q[r][i].y : 0;
        o.z = run; run += c + 2 < n_chunks ? q[r][i].z : 0;
        o.w = run; run += c + 3 < n_chunks ? q[r][i].w : 0;
        row[v] = o;
      }
      if (lane == 31) totals[e] = incl[r];
    }
  }
}

// Rows of any length: one warp per row, each lane a contiguous run of vectors
// read twice (once for its sum, once for the prefixes).
__device__ void scan_rows_warp_any(int32_t *__restrict__ counts, int ncp, int n_chunks, int N,
                                   int *totals) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nwarps = blockDim.x >> 5;
  const int nv = ncp / 4;
  const int per = (nv + 31) / 32;
  for (int e = warp; e < N; e += nwarps) {
    int4 *row = reinterpret_cast<int4 *>(counts + static_cast<size_t>(e) * ncp);
    const int v0 = lane * per, v1 = min(nv, v0 + per);
    int sum = 0;
    for (int v = v0; v < v1; ++v) {
      const int4 q = __ldcg(row + v);
      const int c = 4 * v;
      sum += (c + 0 < n_chunks ? q.x : 0) + (c + 1 < n_chunks ? q.y : 0) +
             (c + 2 < n_chunks ? q.z : 0) + (c + 3 < n_chunks ? q.w : 0);
    }
    int incl = sum;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int y = __shfl_up_sync(kFull, incl, off);
      if (lane >= off) incl += y;
    }
    int run = incl - sum;
    for (int v = v0; v < v1; ++v) {
      const int4 q = __ldcg(row + v);
      const int c = 4 * v;
      int4 o;
      o.x = run; run += c + 0 < n_chunks ? q.x : 0;
      o.y = run; run += c + 1 < n_chunks ? q.y : 0;
      o.z = run; run += c + 2 < n_chunks ? q.z : 0;
      o.w = run; run += c + 3 < n_chunks ? q.w : 0;
      row[v] = o;
    }
    if (lane == 31) totals[e] = incl;
  }
}

// Phase 2 of the fused launch (any number of warps, N <= 1024): the row scans
// above by row length, then the block-wide scans of offsets and tile starts.
__device__ void scan_and_tables_warps(int32_t *__restrict__ counts, int n_chunks, int N,
                                      SegPad seg, int32_t *__restrict__ offsets,
                                      TileEntry *__restrict__ tiles,
                                      int32_t *__restrict__ n_tiles, int tile_m, int max_tiles,
                                      TileEntry *__restrict__ tiles2,
                                      int32_t *__restrict__ n_tiles2, int tile_m2,
                                      int max_tiles2) {
  __shared__ int totals[1024];
  const int ncp = (n_chunks + 3) & ~3;
  const int nv = ncp / 4;  // int4 vectors per row
  if (nv <= 8) {
    for (int e = threadIdx.x; e < N; e += blockDim.x)
      totals[e] = scan_row_thread(reinterpret_cast<int4 *>(counts + static_cast<size_t>(e) * ncp),
                                  nv, n_chunks);
  } else if (nv <= 32) {
    scan_rows_warp<1, 4>(counts, ncp, n_chunks, N, totals);
  } else if (nv <= 64) {
    scan_rows_warp<2, 4>(counts, ncp, n_chunks, N, totals);
  } else if (nv <= 128) {
    scan_rows_warp<4, 2>(counts, ncp, n_chunks, N, totals);
  } else {
    scan_rows_warp_any(counts, ncp, n_chunks, N, totals);
  }
  __syncthreads();
  // experts e0 .. e0+3 per thread, as in scan_and_tables
  const int e0 = threadIdx.x * kScanPerThread;
  int tot[kScanPerThread];
#pragma unroll
  for (int i = 0; i < kScanPerThread; ++i) {
    const int e = e0 + i;
    tot[i] = e < N ? totals[e] : 0;
  }
  offsets_and_tables(tot, e0, N, seg, offsets, tiles, n_tiles, tile_m, max_tiles, tiles2,
                     n_tiles2, tile_m2, max_tiles2);
}

// Top-K', dispatch histogram and scan in one launch.  Block c takes the
// chunk of `chunk` tokens starting at c * chunk, one warp per token (the
// selection is a chain of dependent warp reductions, so every token runs in
// its own warp at once), and counts the chosen experts in shared memory,
// which becomes column c of the count matrix (every entry written: no
// clearing needed).  The block that arrives last on the arrival counter (after a
// fence, so it sees every column) runs the scan of phase 2 and resets the
// counter to zero for the next launch.
template <int VPL>
__global__ void __launch_bounds__(1024) route_select_kernel(
    const float *__restrict__ logits, int ld, const float *__restrict__ bias, int T, int N, int K,
    int32_t *__restrict__ ids, float *__restrict__ gates, int32_t *__restrict__ counts,
    int n_chunks, int chunk, int32_t *__restrict__ arrivals, int32_t *__restrict__ offsets,
    TileEntry *__restrict__ tiles, int32_t *__restrict__ n_tiles, int tile_m, int max_tiles,
    TileEntry *__restrict__ tiles2, int32_t *__restrict__ n_tiles2, int tile_m2,
    int max_tiles2, SegPad seg) {
  __shared__ int hist[1024];
  __shared__ uint2 cand[32][64];  // each warp's top-K' candidate list
  __shared__ int is_last;
  const int warp = threadIdx.x >> 5, nwarps = blockDim.x >> 5;
  for (int e = threadIdx.x; e < N; e += blockDim.x) hist[e] = 0;
  griddep_wait();
  __syncthreads();
  const int t0 = blockIdx.x * chunk, t1 = min(T, t0 + chunk);
  for (int t = t0 + warp; t < t1; t += nwarps)  // one pass: nwarps == chunk
    select_token<VPL>(logits, ld, bias, N, K, t, ids, gates, hist, nullptr, 0, cand[warp]);
  __syncthreads();
  const int ncp = (n_chunks + 3) & ~3;
  for (int e = threadIdx.x; e < N; e += blockDim.x)
    counts[static_cast<size_t>(e) * ncp + blockIdx.x] = hist[e];
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) is_last = atomicAdd(arrivals, 1) == static_cast<int>(gridDim.x) - 1;
  __syncthreads();
  if (!is_last) return;
  __threadfence();
  scan_and_tables_warps(counts, n_chunks, N, seg, offsets, tiles, n_tiles, tile_m, max_tiles,
                        tiles2, n_tiles2, tile_m2, max_tiles2);
  if (threadIdx.x == 0) *arrivals = 0;
}

// Stable scatter and row permutation in one launch.  Block (c, share) with
// c = blockIdx.x / S: chunk c's first chunk/32 warps place its (token, slot)
// pairs exactly as dispatch_scatter_kernel does (share 0 also writes perm,
// pos and row_expert); then every warp of the block copies the source rows of
// the share's pairs (pair i of the chunk with i % S == share) to their
// permuted rows, 16 bytes per lane.  src == nullptr: positions only.
__global__ void __launch_bounds__(256) scatter_permute_kernel(
    const int32_t *__restrict__ ids, int T, int K, int N, const int32_t *__restrict__ counts,
    int n_chunks, int chunk, const int32_t *__restrict__ offsets, int32_t *__restrict__ perm,
    int32_t *__restrict__ pos, int32_t *__restrict__ row_expert, const uint4 *__restrict__ src,
    int vecs_per_row, uint4 *__restrict__ dst, int S) {
  extern __shared__ uint32_t sm[];
  const int W = chunk >> 5;
  uint32_t *mask = sm;                                            // [W][N]
  int32_t *wbase = reinterpret_cast<int32_t *>(sm + W * N);      // [W][N]
  int32_t *ppos = reinterpret_cast<int32_t *>(sm + 2 * W * N);   // [chunk][K]
  const int c = blockIdx.x / S, share = blockIdx.x - c * S;
  for (int i = threadIdx.x; i < W * N; i += blockDim.x) mask[i] = 0u;
  griddep_wait();
  __syncthreads();
  const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int t = c * chunk + threadIdx.x;
  const bool tok = threadIdx.x < chunk && t < T;
  const int32_t *my_ids = ids + static_cast<size_t>(t) * K;
  if (tok)
    for (int k = 0; k < K; ++k) atomicOr(&mask[w * N + my_ids[k]], 1u << lane);
  __syncthreads();
  for (int e = threadIdx.x; e < N; e += blockDim.x) {
    int run = 0;
    for (int ww = 0; ww < W; ++ww) {
      wbase[ww * N + e] = run;
      run += __popc(mask[ww * N + e]);
    }
  }
  __syncthreads();
  if (tok) {
    const uint32_t lt = (1u << lane) - 1u;
    const int ncp = (n_chunks + 3) & ~3;
    for (int k0 = 0; k0 < K; k0 += 8) {  // eight slots' loads in flight, then the stores
      int ev[8], base[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) ev[j] = k0 + j < K ? my_ids[k0 + j] : 0;
#pragma unroll
      for (int j = 0; j < 8; ++j)
        base[j] = k0 + j < K ? offsets[ev[j]] + counts[static_cast<size_t>(ev[j]) * ncp + c] : 0;
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const int k = k0 + j;
        if (k >= K) break;
        const int e = ev[j];
        const int p = base[j] + wbase[w * N + e] + __popc(mask[w * N + e] & lt);
        ppos[threadIdx.x * K + k] = p;
        if (share == 0) {
          const int flat = t * K + k;
          perm[p] = flat;
          pos[flat] = p;
          row_expert[p] = e;
        }
      }
    }
  }
  if (!src) return;
  __syncthreads();
  // The share's pairs are i = share, share + S, ...; item j = (its q-th pair,
  // vector v) with q = j / vecs_per_row: consecutive threads copy consecutive
  // 16-byte vectors of a row, four items in flight per thread (eight measured
  // slower).
  const int npairs = min(chunk, T - c * chunk) * K;
  const int my_pairs = npairs > share ? (npairs - share + S - 1) / S : 0;
  const int items = my_pairs * vecs_per_row;
  for (int j0 = threadIdx.x; j0 < items; j0 += 4 * blockDim.x) {
    uint4 v[4];
    int64_t dst_at[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int j = j0 + u * blockDim.x;
      dst_at[u] = -1;
      if (j < items) {
        const int q = j / vecs_per_row, vv = j - q * vecs_per_row;
        const int i = share + q * S;
        v[u] = src[static_cast<size_t>(c * chunk + i / K) * vecs_per_row + vv];
        dst_at[u] = static_cast<int64_t>(ppos[i]) * vecs_per_row + vv;
      }
    }
#pragma unroll
    for (int u = 0; u < 4; ++u)
      if (dst_at[u] >= 0) dst[dst_at[u]] = v[u];
  }
}

// Phase 3: stable scatter, one block per chunk, one warp per 32 tokens.  A
// per-warp bitmask per expert gives each (token, slot) its rank among the
// warp's tokens that chose the same expert (a token picks an expert at most
// once); the per-warp counts are scanned across the block's warps, and the
// chunk's base comes from phase 2.  Tokens therefore land in ascending order.
// check_ids: as in phase 1, pairs whose id lies outside [0, N) are skipped.
__global__ void __launch_bounds__(256) dispatch_scatter_kernel(
    const int32_t *__restrict__ ids, int T, int K, int N, const int32_t *__restrict__ counts,
    int n_chunks, int chunk, const int32_t *__restrict__ offsets, int32_t *__restrict__ perm,
    int32_t *__restrict__ pos, int32_t *__restrict__ row_expert, int check_ids) {
  extern __shared__ uint32_t sm[];
  const int W = blockDim.x >> 5;
  uint32_t *mask = sm;                                        // [W][N]
  int32_t *wbase = reinterpret_cast<int32_t *>(sm + W * N);  // [W][N]
  for (int i = threadIdx.x; i < W * N; i += blockDim.x) mask[i] = 0u;
  __syncthreads();
  const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int t = blockIdx.x * chunk + threadIdx.x;
  const bool valid = t < T;
  const int32_t *my_ids = ids + static_cast<size_t>(t) * K;
  if (valid)
    for (int k = 0; k < K; ++k) {
      const int e = my_ids[k];
      if (!check_ids || static_cast<unsigned>(e) < static_cast<unsigned>(N))
        atomicOr(&mask[w * N + e], 1u << lane);
    }
  __syncthreads();
  for (int e = threadIdx.x; e < N; e += blockDim.x) {
    int run = 0;
    for (int ww = 0; ww < W; ++ww) {
      wbase[ww * N + e] = run;
      run += __popc(mask[ww * N + e]);
    }
  }
  __syncthreads();
  if (!valid) return;
  const uint32_t lt = (1u << lane) - 1u;
  for (int k = 0; k < K; ++k) {
    const int e = my_ids[k];
    if (check_ids && static_cast<unsigned>(e) >= static_cast<unsigned>(N)) continue;
    const int p = offsets[e] + counts[static_cast<size_t>(e) * ((n_chunks + 3) & ~3) + blockIdx.x] +
                  wbase[w * N + e] + __popc(mask[w * N + e] & lt);
    const int flat = t * K + k;
    perm[p] = flat;
    pos[flat] = p;
    row_expert[p] = e;
  }
}

// ---------------------------------------------------------------- expert parallelism
// As write_tiles, for rows [off, off + tot) of which only those below R
// exist: a tile starting at or past R gets an empty range (row_end = row0:
// the GEMMs store nothing for it), the others end at min(row_end, R).
__device__ void write_tiles_clipped(TileEntry *tiles, int tstart, int max_tiles, int e, int off,
                                    int tot, int tile_m, int R) {
  const int mt = (tot + tile_m - 1) / tile_m;
  for (int j = 0; j < mt; ++j) {
    const int idx = tstart + j;
    if (idx < max_tiles) {
      TileEntry te;
      te.row0 = min(off + j * tile_m, R);
      te.row_end = min(off + tot, R);
      te.expert = e;
      te.pad = 0;
      tiles[idx] = te;
    }
  }
}

// Receiving side of the expert-parallel exchange: one block, thread e owns
// local expert e.  Segment (s, e) -- the rows source s sent for expert e --
// starts at the sum of every earlier source's rows plus source s's rows for
// experts before e.  Tiles are numbered expert by expert, sources in order
// within an expert.
__global__ void __launch_bounds__(1024) ep_tiles_kernel(
    const int32_t *__restrict__ recv_counts, int W, int NL, int R, TileEntry *__restrict__ tiles,
    int32_t *__restrict__ n_tiles, int tile_m, int max_tiles, TileEntry *__restrict__ tiles2,
    int32_t *__restrict__ n_tiles2, int tile_m2, int max_tiles2) {
  __shared__ int warp_sums[32];
  const int e = threadIdx.x;
  const bool mine = e < NL;
  // count of segment (s, e): clipped to non-negative; rows past R are dropped
  // below, so inconsistent counts cannot send a tile past the buffers
  auto count = [&](int s) {
    return mine ? max(0, recv_counts[static_cast<size_t>(s) * NL + e]) : 0;
  };
  int my_t = 0, my_t2 = 0;
  for (int s = 0; s < W; ++s) {
    const int c = count(s);
    my_t += (c + tile_m - 1) / tile_m;
    my_t2 += (c + tile_m2 - 1) / tile_m2;
  }
  int all_t = 0, all_t2 = 0;
  int t_at = block_exclusive_scan(my_t, warp_sums, &all_t);
  int t2_at = block_exclusive_scan(my_t2, warp_sums, &all_t2);
  int base = 0;  // rows of the sources before s
  for (int s = 0; s < W; ++s) {
    const int c = count(s);
    int src_rows = 0;
    const int r0 = base + block_exclusive_scan(c, warp_sums, &src_rows);
    if (mine) {
      write_tiles_clipped(tiles, t_at, max_tiles, e, r0, c, tile_m, R);
      write_tiles_clipped(tiles2, t2_at, max_tiles2, e, r0, c, tile_m2, R);
    }
    t_at += (c + tile_m - 1) / tile_m;
    t2_at += (c + tile_m2 - 1) / tile_m2;
    base += src_rows;
  }
  if (threadIdx.x == 0) {
    *n_tiles = min(all_t, max_tiles);
    *n_tiles2 = min(all_t2, max_tiles2);
  }
}

__global__ void counts_from_offsets_kernel(const int32_t *__restrict__ offsets, int N,
                                           int32_t *__restrict__ counts) {
  const int e = blockIdx.x * blockDim.x + threadIdx.x;
  if (e < N) counts[e] = offsets[e + 1] - offsets[e];
}

// ---------------------------------------------------------------- permute
__global__ void __launch_bounds__(256) permute_rows_kernel(const uint4 *__restrict__ src,
                                                           const int32_t *__restrict__ perm,
                                                           int K, int rows, int vecs_per_row,
                                                           uint4 *__restrict__ dst) {
  const int r = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (r >= rows) return;
  const int flat = perm[r];
  uint4 *d = dst + static_cast<size_t>(r) * vecs_per_row;
  if (flat < 0) {  // a padding row of a padded dispatch order: zeros
    for (int v = lane; v < vecs_per_row; v += 32) d[v] = make_uint4(0, 0, 0, 0);
    return;
  }
  const uint4 *s = src + static_cast<size_t>(flat / K) * vecs_per_row;
  for (int v = lane; v < vecs_per_row; v += 32) d[v] = s[v];
}

// ---------------------------------------------------------------- combine
template <typename Tio>
__device__ __forceinline__ void accum_vec(float *acc, const uint4 &raw, float g);
template <>
__device__ __forceinline__ void accum_vec<__nv_bfloat16>(float *acc, const uint4 &raw, float g) {
  const __nv_bfloat162 *h = reinterpret_cast<const __nv_bfloat162 *>(&raw);
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const float2 f = __bfloat1622float2(h[j]);
    acc[2 * j] = fmaf(g, f.x, acc[2 * j]);
    acc[2 * j + 1] = fmaf(g, f.y, acc[2 * j + 1]);
  }
}
template <>
__device__ __forceinline__ void accum_vec<float>(float *acc, const uint4 &raw, float g) {
  const float *f = reinterpret_cast<const float *>(&raw);
#pragma unroll
  for (int j = 0; j < 4; ++j) acc[j] = fmaf(g, f[j], acc[j]);
}
template <typename Tio>
__device__ __forceinline__ uint4 pack_vec(const float *acc);
template <>
__device__ __forceinline__ uint4 pack_vec<__nv_bfloat16>(const float *acc) {
  uint4 r;
  r.x = pack_bf16x2(acc[0], acc[1]);
  r.y = pack_bf16x2(acc[2], acc[3]);
  r.z = pack_bf16x2(acc[4], acc[5]);
  r.w = pack_bf16x2(acc[6], acc[7]);
  return r;
}
template <>
__device__ __forceinline__ uint4 pack_vec<float>(const float *acc) {
  uint4 r;
  r.x = __float_as_uint(acc[0]);
  r.y = __float_as_uint(acc[1]);
  r.z = __float_as_uint(acc[2]);
  r.w = __float_as_uint(acc[3]);
  return r;
}

// One warp per (token, 32 vectors of its row): a row of l elements takes
// ceil(l / (32 V)) warps, so that every vector of every token has its loads in
// flight at once; 16-byte vectors; the K' slots are summed in slot order
// 0..K'-1 in fp32 (eight slots' loads in flight, then accumulated in order).
// (At most 64 registers: 32 warps per SM.)
template <typename Tio>
__global__ void __launch_bounds__(256, 4) combine_kernel(const Tio *__restrict__ O,
                                                      const int32_t *__restrict__ pos,
                                                      const float *__restrict__ gates, int T,
                                                      int K, int l, Tio *__restrict__ u, int ldu) {
  constexpr int V = 16 / sizeof(Tio);
  const int nvec = l / V;
  const int wpt = (nvec + 31) / 32;  // warps per token
  const int gw = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  griddep_wait();
  const int t = gw / wpt;
  if (t >= T) return;
  const int vi = (gw - t * wpt) * 32 + lane;
  const bool active = vi < nvec;
  float acc[V];
#pragma unroll
  for (int j = 0; j < V; ++j) acc[j] = 0.0f;
  for (int k0 = 0; k0 < K; k0 += 32) {
    const int kk = k0 + lane;
    const int my_p = kk < K ? pos[static_cast<size_t>(t) * K + kk] : 0;
    const float my_g = kk < K ? gates[static_cast<size_t>(t) * K + kk] : 0.0f;
    const int kn = min(32, K - k0);
    for (int k1 = 0; k1 < kn; k1 += 8) {
      uint4 raw[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const int p = __shfl_sync(kFull, my_p, (k1 + j) & 31);
        if (active && k1 + j < kn)
          raw[j] = __ldcs(reinterpret_cast<const uint4 *>(O + static_cast<size_t>(p) * l + vi * V));
      }
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const float g = __shfl_sync(kFull, my_g, (k1 + j) & 31);
        if (active && k1 + j < kn) accum_vec<Tio>(acc, raw[j], g);
      }
    }
  }
  if (active)
    *reinterpret_cast<uint4 *>(u + static_cast<size_t>(t) * ldu + vi * V) = pack_vec<Tio>(acc);
}

// One 16-byte vector per thread: dst vector v -> (group, n-tile, k-block,
// row, chunk), copied from the row-major source or zero past the group's rows.
__global__ void __launch_bounds__(256) repack_btiles_kernel(const uint4 *__restrict__ src,
                                                            int rows_per_group, int cols, int nt,
                                                            int kb_count, int64_t n_vec,
                                                            uint4 *__restrict__ dst) {
  const int64_t v = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (v >= n_vec) return;
  const int c8 = static_cast<int>(v & 7);
  const int r = static_cast<int>((v >> 3) & 255);
  const int64_t blk = v >> 11;  // 256 rows x 8 vectors per block
  const int kb = static_cast<int>(blk % kb_count);
  const int64_t gn = blk / kb_count;
  const int n = static_cast<int>(gn % nt);
  const int64_t g = gn / nt;
  const int srow = n * 256 + r;
  uint4 val = make_uint4(0u, 0u, 0u, 0u);
  if (srow < rows_per_group)
    val = src[((g * rows_per_group + srow) * cols + kb * 64) / 8 + c8];
  dst[v] = val;
}

}  // namespace

cudaError_t launch_repack_btiles(const __nv_bfloat16 *src, int groups, int rows_per_group,
                                 int cols, __nv_bfloat16 *dst, cudaStream_t s) {
  if (cols % 64 || groups <= 0 || rows_per_group <= 0) return cudaErrorInvalidValue;
  const int nt = (rows_per_group + 255) / 256, kbc = cols / 64;
  const int64_t n_vec = static_cast<int64_t>(groups) * nt * kbc * 256 * 8;
  const int64_t blocks = (n_vec + 255) / 256;
  repack_btiles_kernel<<<static_cast<unsigned>(blocks), 256, 0, s>>>(
      reinterpret_cast<const uint4 *>(src), rows_per_group, cols, nt, kbc, n_vec,
      reinterpret_cast<uint4 *>(dst));
  return cudaGetLastError();
}

cudaError_t launch_topk(const float *logits, int ld, const float *bias, int T, int N, int K,
                        int32_t *ids, float *gates, int32_t *counts, int chunk, cudaStream_t s) {
  if (T <= 0) return cudaSuccess;
  const int blocks = (T + 7) / 8;
  const int vpl = (N + 31) / 32;
  const int nc = dispatch_chunks(T, chunk);
#define LMOE_TOPK(V)                                                                        \
  topk_kernel<V><<<blocks, 256, 0, s>>>(logits, ld, bias, T, N, K, ids, gates, counts, nc, \
                                        chunk)
  if (vpl <= 1) LMOE_TOPK(1);
  else if (vpl <= 2) LMOE_TOPK(2);
  else if (vpl <= 4) LMOE_TOPK(4);
  else if (vpl <= 8) LMOE_TOPK(8);
  else if (vpl <= 16) LMOE_TOPK(16);
  else if (vpl <= 32) LMOE_TOPK(32);
  else return cudaErrorInvalidValue;
#undef LMOE_TOPK
  return cudaGetLastError();
}

cudaError_t launch_dispatch(const int32_t *ids, int T, int K, int N, int32_t *chunk_counts,
                            int chunk, bool counts_ready, int32_t *offsets, int32_t *perm,
                            int32_t *pos, int32_t *row_expert, TileEntry *tiles,
                            int32_t *n_tiles, int tile_m, int max_tiles, cudaStream_t s,
                            TileEntry *tiles2, int32_t *n_tiles2, int tile_m2, int max_tiles2,
                            bool check_ids, SegPad seg) {
  if (N > 1024 || chunk % 32 || chunk < 32 || chunk > 256) return cudaErrorInvalidValue;
  if (seg.pad < 1 || (seg.pad > 1 && !seg.ends)) return cudaErrorInvalidValue;
  const int nc = dispatch_chunks(T, chunk);
  if (nc > 0 && !counts_ready) {
    dispatch_count_kernel<<<nc, 256, N * sizeof(int32_t), s>>>(ids, T, K, N, chunk_counts, nc,
                                                               chunk, check_ids ? 1 : 0);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  if (tiles2 && (!n_tiles2 || tile_m2 <= 0)) return cudaErrorInvalidValue;
  dispatch_scan_kernel<<<1, kScanThreads, 0, s>>>(chunk_counts, nc, N, seg, offsets, tiles,
                                                   n_tiles, tile_m, max_tiles, tiles2, n_tiles2,
                                                   tile_m2, max_tiles2);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess || nc == 0) return e;
  const int warps = chunk / 32;
  const size_t smem = 2 * static_cast<size_t>(warps) * N * sizeof(uint32_t);
  if (smem > 48 * 1024) {
    e = cudaFuncSetAttribute(dispatch_scatter_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(smem));
    if (e != cudaSuccess) return e;
  }
  dispatch_scatter_kernel<<<nc, 32 * warps, smem, s>>>(ids, T, K, N, chunk_counts, nc, chunk,
                                                       offsets, perm, pos, row_expert,
                                                       check_ids ? 1 : 0);
  return cudaGetLastError();
}

cudaError_t launch_ep_tiles(const int32_t *recv_counts, int W, int NL, int R, TileEntry *tiles,
                            int32_t *n_tiles, int tile_m, int max_tiles, TileEntry *tiles2,
                            int32_t *n_tiles2, int tile_m2, int max_tiles2, cudaStream_t s) {
  if (W < 1 || NL < 1 || NL > 1024 || static_cast<int64_t>(W) * NL > 65536 || tile_m <= 0 ||
      tile_m2 <= 0)
    return cudaErrorInvalidValue;
  const int threads = (NL + 31) / 32 * 32;
  ep_tiles_kernel<<<1, threads, 0, s>>>(recv_counts, W, NL, R, tiles, n_tiles, tile_m,
                                        max_tiles, tiles2, n_tiles2, tile_m2, max_tiles2);
  return cudaGetLastError();
}

cudaError_t launch_counts_from_offsets(const int32_t *offsets, int N, int32_t *counts,
                                       cudaStream_t s) {
  if (N <= 0) return cudaSuccess;
  counts_from_offsets_kernel<<<(N + 255) / 256, 256, 0, s>>>(offsets, N, counts);
  return cudaGetLastError();
}

bool fused_route_ok(int N, int K, int chunk) {
  // route_select_kernel: one warp per token of a chunk (at most 1024 threads);
  // scatter_permute_kernel: chunk * K positions in shared memory
  return N <= 1024 && chunk == 32 && chunk * K <= 4096;
}

cudaError_t launch_route_select(const float *logits, int ld, const float *bias, int T, int N,
                                int K, int32_t *ids, float *gates, int32_t *counts, int chunk,
                                int32_t *arrivals, int32_t *offsets, TileEntry *tiles,
                                int32_t *n_tiles, int tile_m, int max_tiles, TileEntry *tiles2,
                                int32_t *n_tiles2, int tile_m2, int max_tiles2, cudaStream_t s,
                                bool pdl, SegPad seg) {
  if (T <= 0) return cudaSuccess;
  if (!fused_route_ok(N, K, chunk) || !tiles2 || !n_tiles2 || tile_m2 <= 0)
    return cudaErrorInvalidValue;
  if (seg.pad < 1 || (seg.pad > 1 && !seg.ends)) return cudaErrorInvalidValue;
  const int nc = dispatch_chunks(T, chunk);
  const int vpl = (N + 31) / 32;
  cudaError_t e;
#define LMOE_ROUTE(V)                                                                            \
  e = launch_ex(route_select_kernel<V>, dim3(nc), dim3(32 * chunk), 0, s, pdl, logits, ld, bias, T, N, \
                K, ids, gates, counts, nc, chunk, arrivals, offsets, tiles, n_tiles, tile_m,     \
                max_tiles, tiles2, n_tiles2, tile_m2, max_tiles2, seg)
  if (vpl <= 1) LMOE_ROUTE(1);
  else if (vpl <= 2) LMOE_ROUTE(2);
  else if (vpl <= 4) LMOE_ROUTE(4);
  else if (vpl <= 8) LMOE_ROUTE(8);
  else if (vpl <= 16) LMOE_ROUTE(16);
  else LMOE_ROUTE(32);
#undef LMOE_ROUTE
  return e != cudaSuccess ? e : cudaGetLastError();
}

cudaError_t launch_scatter_permute(const int32_t *ids, int T, int K, int N, const int32_t *counts,
                                   int chunk, const int32_t *offsets, int32_t *perm, int32_t *pos,
                                   int32_t *row_expert, const void *src, int row_bytes, void *dst,
                                   int shares, cudaStream_t s, bool pdl) {
  if (T <= 0) return cudaSuccess;
  if (!fused_route_ok(N, K, chunk) || shares < 1) return cudaErrorInvalidValue;
  if (src && (row_bytes % 16 || !dst)) return cudaErrorInvalidValue;
  const int nc = dispatch_chunks(T, chunk);
  const int W = chunk / 32;
  const size_t smem = (2 * static_cast<size_t>(W) * N + static_cast<size_t>(chunk) * K) * 4;
  const int S = src ? shares : 1;
  const cudaError_t e = launch_ex(scatter_permute_kernel, dim3(nc * S), dim3(256), smem, s, pdl,
                                  ids, T, K, N, counts, nc, chunk, offsets, perm, pos, row_expert,
                                  static_cast<const uint4 *>(src), row_bytes / 16,
                                  static_cast<uint4 *>(dst), S);
  return e != cudaSuccess ? e : cudaGetLastError();
}

cudaError_t launch_permute_rows(const void *src, const int32_t *perm, int K, int rows,
                                int row_bytes, void *dst, cudaStream_t s) {
  if (rows <= 0) return cudaSuccess;
  if (row_bytes % 16) return cudaErrorInvalidValue;
  const int blocks = (rows + 7) / 8;
  permute_rows_kernel<<<blocks, 256, 0, s>>>(static_cast<const uint4 *>(src), perm, K, rows,
                                             row_bytes / 16, static_cast<uint4 *>(dst));
  return cudaGetLastError();
}

cudaError_t launch_combine(const void *O, const int32_t *pos, const float *gates, int T, int K,
                           int l, void *u, int ldu, bool is_bf16, cudaStream_t s, bool pdl) {
  if (T <= 0) return cudaSuccess;
  const int nvec = l / (is_bf16 ? 8 : 4);
  const int64_t warps = static_cast<int64_t>(T) * ((nvec + 31) / 32);
  const int blocks = static_cast<int>((warps + 7) / 8);
  if (is_bf16) {
    if (l % 8 || ldu % 8) return cudaErrorInvalidValue;
    const cudaError_t e = launch_ex(combine_kernel<__nv_bfloat16>, dim3(blocks), dim3(256), 0, s,
                                    pdl, static_cast<const __nv_bfloat16 *>(O), pos, gates, T, K,
                                    l, static_cast<__nv_bfloat16 *>(u), ldu);
    if (e != cudaSuccess) return e;
  } else {
    if (l % 4 || ldu % 4) return cudaErrorInvalidValue;
    const cudaError_t e = launch_ex(combine_kernel<float>, dim3(blocks), dim3(256), 0, s, pdl,
                                    static_cast<const float *>(O), pos, gates, T, K, l,
                                    static_cast<float *>(u), ldu);
    if (e != cudaSuccess) return e;
  }
  return cudaGetLastError();
}

}  // namespace lmoe

// dispatch_noalloc.cu -- lmoe_dispatch_noalloc, the by-expert dispatch for
// callers that cannot allocate device memory.
//
// Some callers may not call cudaMalloc at the point where they need the
// dispatch.  Examples: a serving loop whose device memory is entirely
// reserved up front by its own pool allocator (an extra cudaMalloc would fail
// or stall the device), or a plugin whose host framework forbids allocation
// inside its execute callback.  lmoe_route needs a handle, and the handle's
// workspace is allocated by lmoe_create.  This entry point instead runs the
// same three dispatch kernels (histogram, scan, stable scatter) with their
// scratch -- the per-chunk count matrix, the inverse permutation, the
// per-row expert and the M-tile table -- carved out of one fixed-size
// file-scope __device__ array.  Every GPU that loads this library holds that
// array (about 3 MiB) until the process exits.
#include <cuda_runtime.h>
#include <stdint.h>

#include <mutex>

#include "../../include/lmoe.h"
#include "kernels.h"

namespace lmoe {
namespace {

constexpr int kMaxTokens = LMOE_NOALLOC_MAX_TOKENS;
constexpr int kMaxPairs = LMOE_NOALLOC_MAX_PAIRS;
constexpr int kMaxExperts = LMOE_NOALLOC_MAX_EXPERTS;
constexpr int kTileRows = 128;
constexpr int kChunk = 256;  // tokens per histogram chunk (fewer chunks: smaller scratch)
constexpr int kMaxTiles = kMaxPairs / kTileRows + kMaxExperts + 1;

constexpr size_t round256(size_t b) { return (b + 255) / 256 * 256; }
constexpr size_t kCountsBytes =
    round256(static_cast<size_t>(((kMaxTokens + kChunk - 1) / kChunk + 3) / 4 * 4) *
             kMaxExperts * sizeof(int32_t));
constexpr size_t kPosBytes = round256(static_cast<size_t>(kMaxPairs) * sizeof(int32_t));
constexpr size_t kTilesBytes = round256(static_cast<size_t>(kMaxTiles) * sizeof(TileEntry));
constexpr size_t kOffPos = kCountsBytes;
constexpr size_t kOffRowExpert = kOffPos + kPosBytes;
constexpr size_t kOffTiles = kOffRowExpert + kPosBytes;
constexpr size_t kOffNTiles = kOffTiles + kTilesBytes;
constexpr size_t kScratchBytes = kOffNTiles + 256;

// The shared scratch.  In host code this name is only a stand-in for the
// symbol; its device address comes from cudaGetSymbolAddress below.
static __device__ __align__(256) unsigned char g_dispatch_scratch[kScratchBytes];

// Device address of g_dispatch_scratch, looked up once per device with that
// device current (the first call on the device does it) and kept for the
// life of the process: after a cudaDeviceReset the module may load at another
// address, so the entry point must not be called after a reset.
constexpr int kMaxDevices = 64;
std::mutex g_mutex;
void *g_scratch_addr[kMaxDevices] = {};

int scratch_address(int device, unsigned char **out) {
  if (device < 0 || device >= kMaxDevices) return LMOE_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_mutex);
  if (!g_scratch_addr[device]) {
    void *p = nullptr;
    if (cudaGetSymbolAddress(&p, g_dispatch_scratch) != cudaSuccess || !p) {
      cudaGetLastError();
      return LMOE_ERR_CUDA;
    }
    g_scratch_addr[device] = p;
  }
  *out = static_cast<unsigned char *>(g_scratch_addr[device]);
  return LMOE_OK;
}

}  // namespace
}  // namespace lmoe

extern "C" int lmoe_dispatch_noalloc(const int32_t *ids, int32_t T, int32_t k_active,
                                     int32_t n_routed, int32_t *offsets, int32_t *perm,
                                     void *stream) {
  using namespace lmoe;
  if (!offsets) return LMOE_ERR_NULL_ARG;
  if (T < 0 || k_active < 1 || n_routed < 1 || k_active > n_routed)
    return LMOE_ERR_INVALID_CONFIG;
  if (T > kMaxTokens || static_cast<int64_t>(T) * k_active > kMaxPairs)
    return LMOE_ERR_TOO_MANY_TOKENS;
  if (n_routed > kMaxExperts) return LMOE_ERR_UNSUPPORTED;
  if (T > 0 && (!ids || !perm)) return LMOE_ERR_NULL_ARG;
  int device = -1;
  if (cudaGetDevice(&device) != cudaSuccess) return LMOE_ERR_CUDA;
  unsigned char *base = nullptr;
  const int rc = scratch_address(device, &base);
  if (rc != LMOE_OK) return rc;
  // Every scratch word the kernels read is written earlier in the same call
  // (counts for every chunk and expert, then the scan), so nothing carried
  // over from a previous call needs clearing.
  int32_t *counts = reinterpret_cast<int32_t *>(base);
  int32_t *pos = reinterpret_cast<int32_t *>(base + kOffPos);
  int32_t *row_expert = reinterpret_cast<int32_t *>(base + kOffRowExpert);
  TileEntry *tiles = reinterpret_cast<TileEntry *>(base + kOffTiles);
  int32_t *n_tiles = reinterpret_cast<int32_t *>(base + kOffNTiles);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  // The ids come from the caller: the kernels skip any outside [0, n_routed)
  // (check_ids), and perm starts as -1 so that the entries such pairs would
  // have filled are defined.
  cudaError_t e = cudaSuccess;
  if (T > 0)
    e = cudaMemsetAsync(perm, 0xFF, static_cast<size_t>(T) * k_active * sizeof(int32_t), s);
  if (e == cudaSuccess)
    e = launch_dispatch(ids, T, k_active, n_routed, counts, kChunk, false, offsets, perm, pos,
                        row_expert, tiles, n_tiles, kTileRows, kMaxTiles, s, nullptr, nullptr,
                        0, 0, /*check_ids=*/true);
  return e == cudaSuccess ? LMOE_OK : LMOE_ERR_CUDA;
}

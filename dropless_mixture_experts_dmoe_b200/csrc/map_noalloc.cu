// map_noalloc.cu -- dmoe_sparse_map_noalloc: the routing + sparse-map call without a
// caller-provided workspace.
//
// Who needs it: code that may not allocate device memory at the point where it builds the
// sparse map -- for example a plugin inside a host application that owns every device
// allocation (and hands the plugin only its inputs and outputs), or a latency-critical loop
// that must not call cudaMalloc because it can synchronise the device and its cost is
// unbounded.  Such a caller cannot obtain the per-tile histogram workspace that
// dmoe_sparse_map requires.
//
// How: the scratch lives in a fixed-size array in device global memory that is part of the
// library image (every GPU that loads the library holds it until the process exits).  Host
// code cannot use the array's name as a device address, so the address is looked up once
// per device with cudaGetSymbolAddress and then passed to the same three map kernels that
// dmoe_sparse_map launches.  This entry point performs no allocation of any kind.
#include <mutex>

#include "common.cuh"
#include "kernels.h"

namespace {

// Capacity of the static scratch in int32 words: the per-tile histograms (ceil(T/64) * E), one
// counter, one status word per tile and the scan's per-segment totals (ceil(T/32768) * E)
// must fit (1 MiB; e.g. T <= 65152 tokens at E = 256, T <= 16256 at E = 1024).
constexpr size_t kNoAllocScratchInts = DMOE_NOALLOC_SCRATCH_BYTES / sizeof(int32_t);

static __device__ __align__(256) int32_t g_map_scratch[kNoAllocScratchInts];

constexpr int kMaxDevices = 64;
std::mutex g_setup_mutex;
int32_t *g_scratch_ptr[kMaxDevices] = {};

// Device address of g_map_scratch on the current device (looked up on first use).
int scratch_for_current_device(int32_t **out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return DMOE_ERR_DEVICE;
  std::lock_guard<std::mutex> lock(g_setup_mutex);
  if (!g_scratch_ptr[dev]) {
    void *p = nullptr;
    if (cudaGetSymbolAddress(&p, g_map_scratch) != cudaSuccess || p == nullptr)
      return DMOE_ERR_LAUNCH;
    g_scratch_ptr[dev] = static_cast<int32_t *>(p);
  }
  *out = g_scratch_ptr[dev];
  return DMOE_OK;
}

inline int rc_of(cudaError_t e) { return e == cudaSuccess ? DMOE_OK : DMOE_ERR_LAUNCH; }

}  // namespace

extern "C" int dmoe_sparse_map_noalloc(const dmoe_dims *dims, const void *logits,
                                       const dmoe_map *map, void *stream) {
  // Same host checks as dmoe_sparse_map, minus the workspace, plus the static capacity.
  const size_t ws_need = dmoe_workspace_bytes(dims, DMOE_WS_MAP);
  if (!dims) return DMOE_ERR_NULL;
  if (ws_need == 0) {  // invalid dims: let the regular entry point report the exact code
    dmoe_map empty = {};
    return dmoe_sparse_map(dims, logits, map ? map : &empty, nullptr, 0, stream);
  }
  if (dims->flags & DMOE_ROUTE_TOKEN_ROUNDING) return DMOE_ERR_SHAPE;  // needs its own scratch
  if (!map || !map->top_experts || !map->tokens_per_expert || !map->bins || !map->padded_bins ||
      !map->indices || !map->bin_ids || !map->dest_row || !map->block_expert ||
      !map->num_blocks || !map->status || (logits && !map->weights))
    return DMOE_ERR_NULL;
  const int T = dims->T, E = dims->num_experts, k = dims->top_k;
  if (dmoe::map_workspace_ints(T, E) > kNoAllocScratchInts) return DMOE_ERR_WORKSPACE;
  const uintptr_t a = reinterpret_cast<uintptr_t>(logits) |
                      reinterpret_cast<uintptr_t>(map->top_experts) |
                      (logits ? reinterpret_cast<uintptr_t>(map->weights) : 0);
  if (a & 15u) return DMOE_ERR_ALIGN;
  int dev = 0, major = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
      major != 10)
    return DMOE_ERR_DEVICE;
  int32_t *scratch = nullptr;
  int rc = scratch_for_current_device(&scratch);
  if (rc) return rc;

  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const long long n = (long long)T * k;
  const int nblk_cap =
      (int)((n + (long long)(DMOE_BLOCKING - 1) * E) / DMOE_BLOCKING);
  // The histogram kernel writes every (tile, expert) entry and every tile status word of the
  // scratch it later reads and zeroes the counter after them, so nothing left over from an
  // earlier call is ever read; the scan kernel stores the call's status word.
  const bool renorm = (dims->flags & DMOE_ROUTE_RENORMALIZE) != 0;
  if ((rc = rc_of(dmoe::launch_route_hist(static_cast<const uint16_t *>(logits), T, E, k, renorm,
                                          map->top_experts, map->weights, scratch, st))))
    return rc;
  if ((rc = rc_of(dmoe::launch_map_scan(T, E, scratch, map->tokens_per_expert, map->bins,
                                        map->padded_bins, map->num_blocks, map->status, st))))
    return rc;
  return rc_of(dmoe::launch_map_scatter(T, E, k, nblk_cap, map->top_experts, scratch, map->bins,
                                        map->padded_bins, map->indices, map->bin_ids,
                                        map->dest_row, map->block_expert, st));
}

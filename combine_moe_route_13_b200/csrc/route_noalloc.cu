// moe_route_topk_noalloc: the route step for callers that cannot allocate
// device memory.
//
// moe_route_topk needs a caller-provided workspace for its per-block expert
// histograms. Some callers have no way to obtain one: code running inside
// another framework's memory pool that forbids foreign cudaMalloc calls, or
// plug-ins that are handed only the input and output buffers. This variant
// keeps that scratch in a fixed device array that is part of the library
// image instead: the loader reserves it on every GPU where the library's
// kernels are loaded, and it stays reserved until the process exits.
//
// The device array's name is only a host-side handle in host code; its device
// address is looked up once per device with cudaGetSymbolAddress and cached.
#include <algorithm>
#include <mutex>

#include "moe_internal.h"

namespace moe {
namespace {

constexpr size_t NOALLOC_SCRATCH_BYTES = MOE_NOALLOC_SCRATCH_BYTES;
static_assert(NOALLOC_SCRATCH_BYTES % 256 == 0, "scratch size must keep 256-byte alignment");

// Per-block expert histograms of the route kernels ([blocks, E] int32).
static __device__ __align__(256) int32_t g_route_scratch[NOALLOC_SCRATCH_BYTES / 4];

constexpr int MAX_DEVICES = 64;
std::mutex g_mu;
int32_t* g_scratch_ptr[MAX_DEVICES] = {};

// Device address of g_route_scratch on the current device (looked up once).
cudaError_t scratch_on_current_device(int32_t** out) {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= MAX_DEVICES) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_mu);
  if (!g_scratch_ptr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_route_scratch);
    if (e != cudaSuccess) return e;
    g_scratch_ptr[dev] = static_cast<int32_t*>(p);
  }
  *out = g_scratch_ptr[dev];
  return cudaSuccess;
}

}  // namespace
}  // namespace moe

using namespace moe;

extern "C" moe_status_t moe_route_topk_noalloc(
    const moe_config_t* cfg, const float* logits, int32_t* topk_idx, float* topk_w,
    int32_t* expert_counts, int32_t* overflow, int32_t* expert_offsets, int32_t* segment_offsets,
    int32_t* token_slot, int32_t* row_src, int32_t* totals, void* stream) {
  moe_status_t st = validate(cfg, false);
  if (st != MOE_OK) return st;
  if (!expert_counts || !overflow || !expert_offsets || !segment_offsets || !totals)
    return MOE_ERR_INVALID_ARG;
  if (cfg->T > 0 && (!logits || !topk_idx || !topk_w || !token_slot)) return MOE_ERR_INVALID_ARG;
  const int64_t R = max_rows(*cfg);
  if (R > 0 && !row_src) return MOE_ERR_INVALID_ARG;
  const int64_t need = std::max<int64_t>(route_blocks(cfg->T), 1) * cfg->E * 4;
  if (need > (int64_t)NOALLOC_SCRATCH_BYTES) return MOE_ERR_WORKSPACE;
  int32_t* scratch = nullptr;
  if (scratch_on_current_device(&scratch) != cudaSuccess) return MOE_ERR_CUDA;
  const cudaError_t e = launch_route(*cfg, logits, topk_idx, topk_w, expert_counts, overflow,
                                     expert_offsets, segment_offsets, token_slot, row_src, totals,
                                     scratch, R, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

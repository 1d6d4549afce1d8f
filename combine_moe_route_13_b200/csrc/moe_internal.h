// Internal declarations shared by the CUDA sources of libmoe.so.
#pragma once

#include <algorithm>
#include <cstddef>
#include <cstdint>
#include <utility>

#include <cuda_runtime.h>

#include "../../include/moe.h"

namespace moe {

// Tokens handled by one block of the route's top-K kernel (the unit of the
// per-block expert histograms; the block's expert bitmap has tb/32 words per
// expert): the smallest of 32, 64, 128 that keeps the blocks within one wave
// of two 1024-thread blocks per SM (296 on the 148 SMs), else 128, so that a
// small batch still spreads over the SMs instead of leaving most of them idle
// (a batch of 1,024 tokens is 32 blocks of 32 tokens, not 8 of 128).
inline int route_tb(int64_t T) { return T <= 32 * 296 ? 32 : (T <= 64 * 296 ? 64 : 128); }
inline int64_t route_blocks(int64_t T) { return (T + route_tb(T) - 1) / route_tb(T); }
constexpr int MAX_E = 1024;
constexpr int MAX_K = 32;
// Rows per ready counter of the overlapped combine (the GEMM half-tile height).
constexpr int READY_ROWS = 128;
// Bound of every wait in the kernels (ns).
constexpr unsigned long long WAIT_LIMIT_NS = 2000000000ull;

inline int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }
inline size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

inline int act_size(int32_t act) { return act == MOE_F32 ? 4 : 2; }

// Byte offsets of every region in a workspace. The first 256 bytes hold the
// status word (uint32 at offset 0).
struct WsLayout {
  size_t status = 0;
  size_t blk_cnt = 0;      // [nblk, E] int32: per-block histograms, then bases
  size_t route_end = 0;    // bytes needed by moe_route_topk
  size_t topk_idx = 0, topk_w = 0, counts = 0, overflow = 0, offsets = 0;
  size_t segoff = 0, totals = 0, slot = 0, row_src = 0, row_ready = 0, logits = 0;
  size_t xp = 0, h = 0, y = 0;
  size_t xs = 0, hs = 0;   // fp8 scales (the fp8 codes xq, hq reuse the xp, h regions)
  size_t total = 0;        // bytes needed by moe_layer_forward
};

WsLayout ws_layout(const moe_config_t& c);

// Programmatic dependent launch. Every kernel of the layer is launched with
// programmatic stream serialization, so its launch and on-chip prologue may
// overlap the tail of the kernel before it in the stream. Each such kernel
// calls pdl_wait() before its first global-memory access (read or write: the
// previous kernel may still be reading a buffer this one overwrites) and
// pdl_trigger() to let its own successor launch early.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                       cudaStream_t s, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

// Grid of a kernel whose blocks stride over `work` items (tokens, rows): the
// blocks that are resident on the device at once, capped at `work`, so that
// the kernel's dependency wait (pdl_wait) runs once per block instead of once
// per item. Measured on the skewed dispatch (16,384 tokens): 26.6 us with one
// block per token, 22.5 us striding.
template <typename... KArgs>
int resident_grid(void (*kernel)(KArgs...), int threads, int64_t work) {
  int dev = 0, sms = 0, per = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
      cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per, kernel, threads, 0) != cudaSuccess ||
      sms < 1 || per < 1)
    return (int)std::max<int64_t>(1, std::min<int64_t>(work, 148 * 8));
  return (int)std::max<int64_t>(1, std::min<int64_t>(work, (int64_t)sms * per));
}

// Bounds-checked build (-DMOE_CHECK_BOUNDS, relocatable device code: the
// library variant libmoe_check.so). MOE_CHECK(c) checks an internal index
// invariant of a kernel (a decoded tile, a TMEM column, a shared-memory
// staging offset, a table index); a failed check counts itself and records
// the first failing source line in g_moe_bounds (read with
// moe_debug_bounds_failures), and the guarded access is skipped where the
// kernel uses MOE_CHECKED(c) as its condition. In the release build both
// compile to nothing (MOE_CHECKED(c) is true).
#if defined(MOE_CHECK_BOUNDS) && defined(__CUDACC__)
extern __device__ unsigned int g_moe_bounds[2];   // failures, first failing line
__device__ __forceinline__ void moe_bounds_fail(unsigned line) {
  if (atomicAdd(&g_moe_bounds[0], 1u) == 0u) atomicExch(&g_moe_bounds[1], line);
}
#define MOE_CHECK(c)                                       \
  do {                                                     \
    if (!(c)) ::moe::moe_bounds_fail((unsigned)__LINE__);  \
  } while (0)
#define MOE_CHECKED(c) ((c) ? true : (::moe::moe_bounds_fail((unsigned)__LINE__), false))
#else
#define MOE_CHECK(c) ((void)0)
#define MOE_CHECKED(c) true
#endif

#ifdef __CUDACC__
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}
#endif
// Rows of xp, h, y and row_src: the routed rows, then (n_shared = 1) the
// shared expert's T rows from shared_row0.
int64_t max_rows(const moe_config_t& c);
int64_t routed_rows(const moe_config_t& c);   // min(T*K, E*C) + E*(A-1)
int64_t shared_row0(const moe_config_t& c);   // roundup(routed_rows, 128) with a shared expert
moe_status_t validate(const moe_config_t* c, bool need_mlp);

// ---- launchers (return cudaGetLastError() of their launches) ----
// row_ready (optional): ceil(R_max / READY_ROWS) counters zeroed for the
// overlapped combine.
cudaError_t launch_route(const moe_config_t& c, const float* logits, int32_t* topk_idx,
                         float* topk_w, int32_t* counts, int32_t* overflow, int32_t* offsets,
                         int32_t* segoff, int32_t* slot, int32_t* row_src, int32_t* totals,
                         int32_t* blk_cnt, int64_t R_max, cudaStream_t s,
                         uint32_t* row_ready = nullptr, const float* sel_bias = nullptr);

// sh_row0 >= 0: also copy x[t] to xp[sh_row0 + t] (the shared expert's rows).
cudaError_t launch_dispatch(const moe_config_t& c, const void* x, const int32_t* slot, void* xp,
                            int64_t sh_row0, cudaStream_t s);

// sh_row0 >= 0: add y[sh_row0 + t] with weight 1 after the routed terms.
cudaError_t launch_combine(const moe_config_t& c, const void* y, const int32_t* slot,
                           const float* w, int64_t sh_row0, void* out, cudaStream_t s);

// Combine that waits, token by token, for the ready counters of its rows to
// reach `target` instead of for the previous kernel to finish.
cudaError_t launch_combine_wait(const moe_config_t& c, const void* y, const int32_t* slot,
                                const float* w, int64_t sh_row0, const uint32_t* row_ready,
                                uint32_t target, unsigned long long timeout_ns, uint32_t* status,
                                void* out, cudaStream_t s);

// fp32 CUDA-core grouped SwiGLU (gate/up then down); with a shared expert
// its rows [shared_row0, +T) of xp are included.
cudaError_t launch_mlp_f32(const moe_config_t& c, const float* xp, const int32_t* offsets,
                           const int32_t* counts, const float* w_gu, const float* w_d, float* h,
                           float* y, int64_t R_max, cudaStream_t s);

// bf16 tcgen05 grouped SwiGLU (gate/up then down). Returns a moe status.
// With a shared expert, its T rows are one more group of the same GEMMs; its
// gate/up input rows come from x_shared ([T,H], e.g. the layer input) when
// given, else from xp's rows [shared_row0, +T).
// row_ready (optional): the down GEMM adds 1 to the counter of a 128-row
// block each time it has stored one of the block's N tiles (release), so
// a block is final when its counter reaches ceil(H / 256).
moe_status_t launch_mlp_bf16_tc(const moe_config_t& c, const void* xp, const int32_t* offsets,
                                const int32_t* counts, const void* w_gu, const void* w_d,
                                void* h, void* y, int64_t R_max, uint32_t* status,
                                cudaStream_t s, uint32_t* row_ready = nullptr,
                                const void* x_shared = nullptr);

// Tile signalling of an expert-parallel owner's grouped GEMMs ("Mixture-of-
// Experts acceleration through overlap": the GEMM consumes rows as they arrive
// and publishes output tiles through flags the consumer polls).
//   Gate/up (arrive != nullptr): before a CTA loads its rows of a tile, it
//   waits until every sender owning some of those rows has raised its
//   DISPATCH flag of this step (acquire at system scope, bounded by wait_ns;
//   a wait that runs out records MOE_ERR_TIMEOUT and ends the kernel).
//   Down (yready != nullptr): each stored 128-row x 256-column tile adds 1 to
//   its block's counter in bank (step & 1) of yready (release at system
//   scope), so that a block is final when its counter reaches ceil(H / 256).
//   remote_first: tiles holding rows of other senders run before the tiles
//   that hold only this owner's own rows (the outputs other ranks read
//   first), each set in the usual (expert, N tile, M tile) order.
// The step number is `epoch`, or one past *counter when epoch is 0.
struct EpTiles {
  const uint32_t* arrive = nullptr;   // [W] this owner's DISPATCH flags, by sender
  const int32_t* split = nullptr;     // [E_local][W+1]: sender s's first row within each local
                                      // expert's rows; [W] = the expert's received rows
  const uint32_t* counter = nullptr;
  uint32_t epoch = 0;
  int W = 0, rank = 0;
  int remote_first = 0;
  unsigned long long wait_ns = 0;
  uint32_t* yready = nullptr;         // [2][ready_blocks]
  int ready_blocks = 0;
};

// One or both launches (modes: bit 0 gate/up, bit 1 down) of the bf16 grouped
// GEMM of launch_mlp_bf16_tc over an expert-parallel owner's local experts
// (no shared group), tile-signalled by `t`.
moe_status_t launch_mlp_bf16_tc_ep(const moe_config_t& c, int modes, const void* xr,
                                   const int32_t* offsets, const int32_t* counts,
                                   const void* w_gu, const void* w_d, void* h, void* y,
                                   int64_t R_max, uint32_t* status, cudaStream_t s,
                                   const EpTiles& t);

// The shared expert alone, bf16 on tcgen05: h[T,F] = silu(x Wg^T) * (x Wu^T),
// y[T,H] = h Wd^T for the T rows of x, with w_gu_sh [2F,H] and w_d_sh [H,F]
// (one expert). Same kernels and arithmetic as the shared group of
// launch_mlp_bf16_tc.
moe_status_t launch_shared_mlp_bf16_tc(const moe_config_t& c, const void* x, const void* w_gu_sh,
                                       const void* w_d_sh, void* h, void* y, uint32_t* status,
                                       cudaStream_t s);

// Router projection logits[T,E] = x[T,H] w_g[E,H]^T (fp32 out): tcgen05 for
// bf16, FFMA for fp32.
moe_status_t launch_router_logits_tc(const moe_config_t& c, const void* x, const void* w_g,
                                     float* logits, uint32_t* status, cudaStream_t s);
cudaError_t launch_router_f32(const moe_config_t& c, const float* x, const float* w_g,
                              float* logits, cudaStream_t s);

// ---- fp8 block-scaled path ----
moe_status_t validate_fp8(const moe_config_t* c);
cudaError_t launch_quantize_fp8(const void* src, int64_t rows, int64_t cols, uint8_t* q,
                                uint8_t* sf, cudaStream_t s);
cudaError_t launch_dispatch_fp8(const moe_config_t& c, const void* x, const int32_t* slot,
                                uint8_t* xq, uint8_t* xs, cudaStream_t s);
moe_status_t launch_mlp_fp8(const moe_config_t& c, const uint8_t* xq, const uint8_t* xs,
                            const int32_t* offsets, const int32_t* counts, const uint8_t* wq_gu,
                            const uint8_t* ws_gu, const uint8_t* wq_d, const uint8_t* ws_d,
                            uint8_t* hq, uint8_t* hs, void* y, int64_t R_max, uint32_t* status,
                            cudaStream_t s);

// Shared memory of launch_mlp_fp8_ep's kernels over c's E experts (two_sets:
// with the remote-first order's tables).
size_t fp8_ep_smem_bytes(const moe_config_t& c, bool two_sets);

// One or both launches (modes: bit 0 gate/up, bit 1 down) of the fp8 grouped
// GEMM of launch_mlp_fp8 over an expert-parallel owner's local experts (no
// shared group), tile-signalled by `t` as launch_mlp_bf16_tc_ep.
moe_status_t launch_mlp_fp8_ep(const moe_config_t& c, int modes, const uint8_t* xq,
                               const uint8_t* xs, const int32_t* offsets, const int32_t* counts,
                               const uint8_t* wq_gu, const uint8_t* ws_gu, const uint8_t* wq_d,
                               const uint8_t* ws_d, uint8_t* hq, uint8_t* hs, void* y,
                               int64_t R_max, uint32_t* status, cudaStream_t s,
                               const EpTiles& t);

// Ready-counter target of the down GEMM (its number of N tiles).
inline uint32_t ready_target(const moe_config_t& c) { return (uint32_t)ceil_div(c.H, 256); }

}  // namespace moe

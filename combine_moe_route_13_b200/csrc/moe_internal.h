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

// Ready-counter target of the down GEMM (its number of N tiles).
inline uint32_t ready_target(const moe_config_t& c) { return (uint32_t)ceil_div(c.H, 256); }

}  // namespace moe

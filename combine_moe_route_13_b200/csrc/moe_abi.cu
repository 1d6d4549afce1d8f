// extern "C" entry points of libmoe.so: argument validation, workspace layout
// and the launch order of the layer. Every entry point only launches kernels
// on the caller's stream; none allocates, frees or synchronises (except
// moe_get_device_status, which exists to synchronise).
#include <algorithm>
#include <climits>
#include <cmath>

#include "fp8_util.cuh"
#include "moe_internal.h"

namespace moe {

int64_t routed_rows(const moe_config_t& c) {
  return std::min<int64_t>((int64_t)c.T * c.K, (int64_t)c.E * c.capacity) +
         (int64_t)c.E * (c.row_align - 1);
}

int64_t shared_row0(const moe_config_t& c) {
  const int64_t r = routed_rows(c);
  return c.n_shared ? ceil_div(r, READY_ROWS) * READY_ROWS : r;
}

int64_t max_rows(const moe_config_t& c) { return shared_row0(c) + (int64_t)c.n_shared * c.T; }

// First shared-expert row for the kernels, or -1 without a shared expert.
static int64_t sh_row0_or_none(const moe_config_t& c) { return c.n_shared ? shared_row0(c) : -1; }

static moe_status_t basic_checks(const moe_config_t* c) {
  if (!c) return MOE_ERR_INVALID_ARG;
  if (c->T < 0 || c->H < 1 || c->E < 1 || c->K < 1 || c->F < 1 || c->S < 1) return MOE_ERR_INVALID_ARG;
  if (c->K > c->E || c->E % c->S != 0 || c->capacity < 0 || c->row_align < 1)
    return MOE_ERR_INVALID_ARG;
  if (c->act_dtype != MOE_F32 && c->act_dtype != MOE_BF16) return MOE_ERR_INVALID_ARG;
  if (c->n_shared != 0 && c->n_shared != 1) return MOE_ERR_INVALID_ARG;
  if (c->E > MAX_E || c->K > MAX_K || c->row_align > 1024) return MOE_ERR_UNSUPPORTED;
  if ((int64_t)c->T * c->K > INT_MAX / 2) return MOE_ERR_UNSUPPORTED;
  if (max_rows(*c) > INT_MAX / 2) return MOE_ERR_UNSUPPORTED;
  return MOE_OK;
}

moe_status_t validate(const moe_config_t* c, bool need_mlp) {
  moe_status_t st = basic_checks(c);
  if (st != MOE_OK) return st;
  const int sz = act_size(c->act_dtype);
  if (((int64_t)c->H * sz) % 16 != 0 || ((int64_t)c->F * sz) % 16 != 0) return MOE_ERR_UNSUPPORTED;
  if (need_mlp && c->act_dtype == MOE_BF16) {
    if (c->H % 64 != 0 || c->F % 64 != 0) return MOE_ERR_UNSUPPORTED;
    const int64_t ew = (int64_t)c->E + c->n_shared;   // experts in the weight arrays
    if (ew * 2 * c->F > INT_MAX / 2 || ew * c->H > INT_MAX / 2) return MOE_ERR_UNSUPPORTED;
  }
  if (need_mlp && c->act_dtype == MOE_F32 && ceil_div(max_rows(*c), 32) + c->E + 1 > 65535)
    return MOE_ERR_UNSUPPORTED;
  return MOE_OK;
}

moe_status_t validate_fp8(const moe_config_t* c) {
  moe_status_t st = validate(c, true);
  if (st != MOE_OK) return st;
  if (c->act_dtype != MOE_BF16 || c->H % 256 != 0 || c->F % FP8_BLOCK != 0 ||
      c->row_align % 128 != 0 || c->E > 512)
    return MOE_ERR_UNSUPPORTED;
  return MOE_OK;
}

WsLayout ws_layout(const moe_config_t& c) {
  WsLayout L;
  const int64_t nblk = route_blocks(c.T);
  const int64_t TK = (int64_t)c.T * c.K;
  const int64_t R = max_rows(c);
  const size_t as = act_size(c.act_dtype);
  size_t p = 256;   // status word region
  L.blk_cnt = p;   p += align256((size_t)std::max<int64_t>(nblk, 1) * c.E * 4);
  L.route_end = p;
  L.topk_idx = p;  p += align256((size_t)TK * 4);
  L.topk_w = p;    p += align256((size_t)TK * 4);
  L.counts = p;    p += align256((size_t)c.E * 4);
  L.overflow = p;  p += align256((size_t)c.E * 4);
  L.offsets = p;   p += align256((size_t)(c.E + 1) * 4);
  L.segoff = p;    p += align256((size_t)(c.S + 1) * 4);
  L.totals = p;    p += align256(16);
  L.slot = p;      p += align256((size_t)TK * 4);
  L.row_src = p;   p += align256((size_t)R * 4);
  L.row_ready = p; p += align256((size_t)ceil_div(R, READY_ROWS) * 4);
  L.logits = p;    p += align256((size_t)c.T * c.E * 4);
  L.xp = p;        p += align256((size_t)R * c.H * as);
  L.h = p;         p += align256((size_t)R * c.F * as);
  L.y = p;         p += align256((size_t)R * c.H * as);
  if (c.H % FP8_BLOCK == 0 && c.F % FP8_BLOCK == 0) {   // scales of the fp8 variant
    L.xs = p;      p += align256((size_t)sf_bytes(R, c.H));
    L.hs = p;      p += align256((size_t)sf_bytes(R, c.F));
  }
  L.total = p;
  return L;
}

static bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

static moe_status_t cuda_status(cudaError_t e) { return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA; }

}  // namespace moe

using namespace moe;

#ifdef MOE_CHECK_BOUNDS
namespace moe {
__device__ unsigned int g_moe_bounds[2] = {0u, 0u};
}
#endif

extern "C" {

moe_status_t moe_debug_bounds_failures(uint32_t* failures, uint32_t* first_line, int32_t reset) {
#ifdef MOE_CHECK_BOUNDS
  if (!failures || !first_line) return MOE_ERR_INVALID_ARG;
  unsigned int v[2] = {0u, 0u};
  if (cudaDeviceSynchronize() != cudaSuccess ||
      cudaMemcpyFromSymbol(v, moe::g_moe_bounds, sizeof(v)) != cudaSuccess)
    return MOE_ERR_CUDA;
  *failures = v[0];
  *first_line = v[1];
  if (reset) {
    const unsigned int z[2] = {0u, 0u};
    if (cudaMemcpyToSymbol(moe::g_moe_bounds, z, sizeof(z)) != cudaSuccess) return MOE_ERR_CUDA;
  }
  return MOE_OK;
#else
  (void)failures;
  (void)first_line;
  (void)reset;
  return MOE_ERR_UNSUPPORTED;
#endif
}

int32_t moe_version(void) { return 1 * 10000 + 2 * 100 + 0; }   // 1.2: tile-signalled moe_ep.h

const char* moe_status_string(moe_status_t s) {
  switch (s) {
    case MOE_OK: return "ok";
    case MOE_ERR_INVALID_ARG: return "invalid argument";
    case MOE_ERR_UNSUPPORTED: return "unsupported configuration";
    case MOE_ERR_WORKSPACE: return "workspace missing, misaligned or too small";
    case MOE_ERR_CUDA: return "CUDA runtime error";
    case MOE_ERR_TIMEOUT: return "a bounded wait inside a kernel gave up";
    case MOE_ERR_DEVICE_INPUT: return "a device-side table held an out-of-range value";
  }
  return "unknown status";
}

int32_t moe_capacity(int32_t T, int32_t K, int32_t E, double cf) {
  if (T < 0 || K < 1 || E < 1) return -1;
  if (cf < 0) return T;
  const double c = std::ceil(cf * (double)T * (double)K / (double)E);
  if (!(c <= (double)INT_MAX)) return -1;
  return (int32_t)c;
}

int64_t moe_max_rows(const moe_config_t* cfg) {
  if (basic_checks(cfg) != MOE_OK) return -1;
  return max_rows(*cfg);
}

moe_status_t moe_check_config(const moe_config_t* cfg) { return validate(cfg, true); }

size_t moe_route_workspace_bytes(const moe_config_t* cfg) {
  if (basic_checks(cfg) != MOE_OK) return 0;
  return ws_layout(*cfg).route_end;
}

size_t moe_workspace_bytes(const moe_config_t* cfg, uint32_t flags) {
  (void)flags;
  if (basic_checks(cfg) != MOE_OK) return 0;
  return ws_layout(*cfg).total;
}

moe_status_t moe_workspace_init(void* ws, size_t ws_bytes, void* stream) {
  if (!ws || ws_bytes < 256 || (reinterpret_cast<uintptr_t>(ws) & 255u)) return MOE_ERR_WORKSPACE;
  return cuda_status(cudaMemsetAsync(ws, 0, 4, static_cast<cudaStream_t>(stream)));
}

moe_status_t moe_route_topk_biased(const moe_config_t* cfg, const float* logits,
                                   const float* sel_bias, int32_t* topk_idx, float* topk_w,
                                   int32_t* expert_counts, int32_t* overflow,
                                   int32_t* expert_offsets, int32_t* segment_offsets,
                                   int32_t* token_slot, int32_t* row_src, int32_t* totals,
                                   void* ws, size_t ws_bytes, void* stream) {
  moe_status_t st = validate(cfg, false);
  if (st != MOE_OK) return st;
  if (!expert_counts || !overflow || !expert_offsets || !segment_offsets || !totals)
    return MOE_ERR_INVALID_ARG;
  if (cfg->T > 0 && (!logits || !topk_idx || !topk_w || !token_slot)) return MOE_ERR_INVALID_ARG;
  const int64_t R = max_rows(*cfg);
  if (R > 0 && !row_src) return MOE_ERR_INVALID_ARG;
  const WsLayout L = ws_layout(*cfg);
  if (!ws || (reinterpret_cast<uintptr_t>(ws) & 255u) || ws_bytes < L.route_end)
    return MOE_ERR_WORKSPACE;
  int32_t* blk = reinterpret_cast<int32_t*>(static_cast<char*>(ws) + L.blk_cnt);
  return cuda_status(launch_route(*cfg, logits, topk_idx, topk_w, expert_counts, overflow,
                                  expert_offsets, segment_offsets, token_slot, row_src, totals,
                                  blk, R, static_cast<cudaStream_t>(stream), nullptr, sel_bias));
}

moe_status_t moe_route_topk(const moe_config_t* cfg, const float* logits, int32_t* topk_idx,
                            float* topk_w, int32_t* expert_counts, int32_t* overflow,
                            int32_t* expert_offsets, int32_t* segment_offsets,
                            int32_t* token_slot, int32_t* row_src, int32_t* totals, void* ws,
                            size_t ws_bytes, void* stream) {
  return moe_route_topk_biased(cfg, logits, nullptr, topk_idx, topk_w, expert_counts, overflow,
                               expert_offsets, segment_offsets, token_slot, row_src, totals, ws,
                               ws_bytes, stream);
}

moe_status_t moe_router_logits(const moe_config_t* cfg, const void* x, const void* w_g,
                               float* logits, void* ws, size_t ws_bytes, void* stream) {
  moe_status_t st = validate(cfg, true);
  if (st != MOE_OK) return st;
  if (cfg->T == 0) return MOE_OK;
  if (!x || !w_g || !logits) return MOE_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(w_g)) return MOE_ERR_INVALID_ARG;
  if (!ws || (reinterpret_cast<uintptr_t>(ws) & 255u) || ws_bytes < 256) return MOE_ERR_WORKSPACE;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (cfg->act_dtype == MOE_F32)
    return cuda_status(launch_router_f32(*cfg, static_cast<const float*>(x),
                                         static_cast<const float*>(w_g), logits, s));
  return launch_router_logits_tc(*cfg, x, w_g, logits, static_cast<uint32_t*>(ws), s);
}

moe_status_t moe_dispatch(const moe_config_t* cfg, const void* x, const int32_t* token_slot,
                          void* xp, void* stream) {
  moe_status_t st = validate(cfg, false);
  if (st != MOE_OK) return st;
  if (cfg->T == 0) return MOE_OK;
  if (!x || !token_slot || !xp) return MOE_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(xp)) return MOE_ERR_INVALID_ARG;
  return cuda_status(launch_dispatch(*cfg, x, token_slot, xp, sh_row0_or_none(*cfg),
                                     static_cast<cudaStream_t>(stream)));
}

moe_status_t moe_expert_mlp(const moe_config_t* cfg, const void* xp,
                            const int32_t* expert_offsets, const int32_t* expert_counts,
                            const void* w_gu, const void* w_d, void* h, void* y, void* ws,
                            size_t ws_bytes, void* stream) {
  moe_status_t st = validate(cfg, true);
  if (st != MOE_OK) return st;
  const int64_t R = max_rows(*cfg);
  if (R == 0) return MOE_OK;
  if (!xp || !expert_offsets || !expert_counts || !w_gu || !w_d || !h || !y)
    return MOE_ERR_INVALID_ARG;
  if (!aligned16(xp) || !aligned16(w_gu) || !aligned16(w_d) || !aligned16(h) || !aligned16(y))
    return MOE_ERR_INVALID_ARG;
  if (!ws || (reinterpret_cast<uintptr_t>(ws) & 255u) || ws_bytes < 256) return MOE_ERR_WORKSPACE;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (cfg->act_dtype == MOE_F32)
    return cuda_status(launch_mlp_f32(*cfg, static_cast<const float*>(xp), expert_offsets,
                                      expert_counts, static_cast<const float*>(w_gu),
                                      static_cast<const float*>(w_d), static_cast<float*>(h),
                                      static_cast<float*>(y), R, s));
  return launch_mlp_bf16_tc(*cfg, xp, expert_offsets, expert_counts, w_gu, w_d, h, y, R,
                            static_cast<uint32_t*>(ws), s);
}

moe_status_t moe_combine(const moe_config_t* cfg, const void* y, const int32_t* token_slot,
                         const float* topk_w, void* out, void* stream) {
  moe_status_t st = validate(cfg, false);
  if (st != MOE_OK) return st;
  if (cfg->T == 0) return MOE_OK;
  if (!y || !token_slot || !topk_w || !out) return MOE_ERR_INVALID_ARG;
  if (!aligned16(y) || !aligned16(out)) return MOE_ERR_INVALID_ARG;
  return cuda_status(launch_combine(*cfg, y, token_slot, topk_w, sh_row0_or_none(*cfg), out,
                                    static_cast<cudaStream_t>(stream)));
}

moe_status_t moe_combine_wait(const moe_config_t* cfg, const void* y, const int32_t* token_slot,
                              const float* topk_w, const uint32_t* row_ready,
                              uint32_t ready_target, void* out, uint32_t timeout_us, void* ws,
                              size_t ws_bytes, void* stream) {
  moe_status_t st = validate(cfg, false);
  if (st != MOE_OK) return st;
  if (cfg->row_align % READY_ROWS != 0) return MOE_ERR_UNSUPPORTED;
  if (cfg->T == 0) return MOE_OK;
  if (!y || !token_slot || !topk_w || !row_ready || !out) return MOE_ERR_INVALID_ARG;
  if (!aligned16(y) || !aligned16(out)) return MOE_ERR_INVALID_ARG;
  if (!ws || (reinterpret_cast<uintptr_t>(ws) & 255u) || ws_bytes < 256) return MOE_ERR_WORKSPACE;
  return cuda_status(launch_combine_wait(*cfg, y, token_slot, topk_w, sh_row0_or_none(*cfg),
                                         row_ready, ready_target,
                                         (unsigned long long)timeout_us * 1000ull,
                                         static_cast<uint32_t*>(ws), out,
                                         static_cast<cudaStream_t>(stream)));
}

}  // extern "C"

namespace moe {

// The layer from router logits (written by the caller, or by the router
// projection when x_for_router is set), with an optional selection bias.
static moe_status_t layer_forward(const moe_config_t* cfg, const float* logits,
                                  const float* sel_bias, const void* x, const void* w_g,
                                  const void* w_gu, const void* w_d, void* out, uint32_t flags,
                                  void* ws, size_t ws_bytes, moe_layer_aux_t* aux, void* stream) {
  moe_status_t st = validate(cfg, true);
  if (st != MOE_OK) return st;
  if ((flags & ~MOE_FLAG_OVERLAP) != 0u) return MOE_ERR_UNSUPPORTED;
  const bool overlap = (flags & MOE_FLAG_OVERLAP) != 0u;
  if (overlap && (cfg->act_dtype != MOE_BF16 || cfg->row_align % READY_ROWS != 0))
    return MOE_ERR_UNSUPPORTED;
  if (cfg->T > 0 && (!(logits || w_g) || !x || !out)) return MOE_ERR_INVALID_ARG;
  if (!w_gu || !w_d) return MOE_ERR_INVALID_ARG;
  const WsLayout L = ws_layout(*cfg);
  if (!ws || (reinterpret_cast<uintptr_t>(ws) & 255u) || ws_bytes < L.total) return MOE_ERR_WORKSPACE;
  char* b = static_cast<char*>(ws);
  moe_layer_aux_t a = {};
  a.topk_idx = reinterpret_cast<int32_t*>(b + L.topk_idx);
  a.topk_w = reinterpret_cast<float*>(b + L.topk_w);
  a.expert_counts = reinterpret_cast<int32_t*>(b + L.counts);
  a.overflow = reinterpret_cast<int32_t*>(b + L.overflow);
  a.expert_offsets = reinterpret_cast<int32_t*>(b + L.offsets);
  a.segment_offsets = reinterpret_cast<int32_t*>(b + L.segoff);
  a.totals = reinterpret_cast<int32_t*>(b + L.totals);
  a.token_slot = reinterpret_cast<int32_t*>(b + L.slot);
  a.row_src = reinterpret_cast<int32_t*>(b + L.row_src);
  a.xp = b + L.xp;
  a.h = b + L.h;
  a.y = b + L.y;
  a.logits = reinterpret_cast<float*>(b + L.logits);
  if (aux) *aux = a;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (w_g) {   // router projection into the workspace
    st = moe_router_logits(cfg, x, w_g, a.logits, ws, ws_bytes, stream);
    if (st != MOE_OK) return st;
    logits = a.logits;
  }
  // Overlapped: the route also zeroes the ready counters, the down GEMM
  // publishes them and the combine consumes them while the GEMM finishes.
  uint32_t* ready = overlap ? reinterpret_cast<uint32_t*>(b + L.row_ready) : nullptr;
  uint32_t* status = static_cast<uint32_t*>(ws);
  const int64_t R = max_rows(*cfg);
  st = cuda_status(launch_route(*cfg, logits, a.topk_idx, a.topk_w, a.expert_counts, a.overflow,
                                a.expert_offsets, a.segment_offsets, a.token_slot, a.row_src,
                                a.totals, reinterpret_cast<int32_t*>(b + L.blk_cnt), R, s, ready,
                                sel_bias));
  if (st != MOE_OK) return st;
  if (cfg->T == 0) return MOE_OK;
  if (!aligned16(x) || !aligned16(out) || !aligned16(w_gu) || !aligned16(w_d))
    return MOE_ERR_INVALID_ARG;
  // bf16: the shared expert's gate/up GEMM reads x itself, so the dispatch
  // copies only the routed rows
  const bool bf16 = cfg->act_dtype == MOE_BF16;
  const int64_t sh = sh_row0_or_none(*cfg);
  st = cuda_status(launch_dispatch(*cfg, x, a.token_slot, a.xp, bf16 ? -1 : sh, s));
  if (st != MOE_OK) return st;
  if (bf16)
    st = launch_mlp_bf16_tc(*cfg, a.xp, a.expert_offsets, a.expert_counts, w_gu, w_d, a.h, a.y,
                            R, status, s, ready, cfg->n_shared ? x : nullptr);
  else
    st = cuda_status(launch_mlp_f32(*cfg, static_cast<const float*>(a.xp), a.expert_offsets,
                                    a.expert_counts, static_cast<const float*>(w_gu),
                                    static_cast<const float*>(w_d), static_cast<float*>(a.h),
                                    static_cast<float*>(a.y), R, s));
  if (st != MOE_OK) return st;
  if (!overlap)
    return cuda_status(launch_combine(*cfg, a.y, a.token_slot, a.topk_w, sh, out, s));
  return cuda_status(launch_combine_wait(*cfg, a.y, a.token_slot, a.topk_w, sh, ready,
                                         ready_target(*cfg), WAIT_LIMIT_NS, status, out, s));
}

}  // namespace moe

extern "C" {

moe_status_t moe_layer_forward(const moe_config_t* cfg, const float* logits, const void* x,
                               const void* w_gu, const void* w_d, void* out, uint32_t flags,
                               void* ws, size_t ws_bytes, moe_layer_aux_t* aux, void* stream) {
  if (cfg && cfg->T > 0 && !logits) return MOE_ERR_INVALID_ARG;
  return layer_forward(cfg, logits, nullptr, x, nullptr, w_gu, w_d, out, flags, ws, ws_bytes, aux,
                       stream);
}

moe_status_t moe_layer_forward_x(const moe_config_t* cfg, const void* x, const void* w_g,
                                 const float* sel_bias, const void* w_gu, const void* w_d,
                                 void* out, uint32_t flags, void* ws, size_t ws_bytes,
                                 moe_layer_aux_t* aux, void* stream) {
  if (!w_g) return MOE_ERR_INVALID_ARG;
  return layer_forward(cfg, nullptr, sel_bias, x, w_g, w_gu, w_d, out, flags, ws, ws_bytes, aux,
                       stream);
}

int64_t moe_fp8_scale_bytes(int64_t rows, int64_t cols) {
  if (rows < 0 || cols <= 0 || cols % FP8_BLOCK != 0) return -1;
  return sf_bytes(rows, cols);
}

moe_status_t moe_quantize_fp8(const void* src, int64_t rows, int64_t cols, uint8_t* codes,
                              uint8_t* scales, void* stream) {
  if (rows < 0 || cols <= 0 || cols % FP8_BLOCK != 0) return MOE_ERR_INVALID_ARG;
  if (rows > INT_MAX || cols > (int64_t)INT_MAX / 2) return MOE_ERR_UNSUPPORTED;
  if (rows == 0) return MOE_OK;
  if (!src || !codes || !scales || !aligned16(src) || !aligned16(codes) || !aligned16(scales))
    return MOE_ERR_INVALID_ARG;
  return cuda_status(
      launch_quantize_fp8(src, rows, cols, codes, scales, static_cast<cudaStream_t>(stream)));
}

moe_status_t moe_dispatch_fp8(const moe_config_t* cfg, const void* x, const int32_t* token_slot,
                              uint8_t* xq, uint8_t* xs, void* stream) {
  moe_status_t st = validate_fp8(cfg);
  if (st != MOE_OK) return st;
  if (cfg->T == 0) return MOE_OK;
  if (!x || !token_slot || !xq || !xs) return MOE_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(xq) || !aligned16(xs)) return MOE_ERR_INVALID_ARG;
  return cuda_status(
      launch_dispatch_fp8(*cfg, x, token_slot, xq, xs, static_cast<cudaStream_t>(stream)));
}

moe_status_t moe_expert_mlp_fp8(const moe_config_t* cfg, const uint8_t* xq, const uint8_t* xs,
                                const int32_t* expert_offsets, const int32_t* expert_counts,
                                const uint8_t* wq_gu, const uint8_t* ws_gu, const uint8_t* wq_d,
                                const uint8_t* ws_d, uint8_t* hq, uint8_t* hs, void* y, void* ws,
                                size_t ws_bytes, void* stream) {
  moe_status_t st = validate_fp8(cfg);
  if (st != MOE_OK) return st;
  const int64_t R = max_rows(*cfg);
  if (R == 0) return MOE_OK;
  if (!xq || !xs || !expert_offsets || !expert_counts || !wq_gu || !ws_gu || !wq_d || !ws_d ||
      !hq || !hs || !y)
    return MOE_ERR_INVALID_ARG;
  for (const void* p : {(const void*)xq, (const void*)xs, (const void*)wq_gu, (const void*)ws_gu,
                        (const void*)wq_d, (const void*)ws_d, (const void*)hq, (const void*)hs,
                        (const void*)y})
    if (!aligned16(p)) return MOE_ERR_INVALID_ARG;
  if (!ws || (reinterpret_cast<uintptr_t>(ws) & 255u) || ws_bytes < 256) return MOE_ERR_WORKSPACE;
  return launch_mlp_fp8(*cfg, xq, xs, expert_offsets, expert_counts, wq_gu, ws_gu, wq_d, ws_d, hq,
                        hs, y, R, static_cast<uint32_t*>(ws), static_cast<cudaStream_t>(stream));
}

moe_status_t moe_layer_forward_fp8(const moe_config_t* cfg, const float* logits, const void* x,
                                   const uint8_t* wq_gu, const uint8_t* ws_gu,
                                   const uint8_t* wq_d, const uint8_t* ws_d, void* out,
                                   uint32_t flags, void* ws, size_t ws_bytes,
                                   moe_layer_aux_t* aux, void* stream) {
  moe_status_t st = validate_fp8(cfg);
  if (st != MOE_OK) return st;
  if (flags != MOE_FLAG_NONE) return MOE_ERR_UNSUPPORTED;
  if (cfg->T > 0 && (!logits || !x || !out)) return MOE_ERR_INVALID_ARG;
  if (!wq_gu || !ws_gu || !wq_d || !ws_d) return MOE_ERR_INVALID_ARG;
  const WsLayout L = ws_layout(*cfg);
  if (!ws || (reinterpret_cast<uintptr_t>(ws) & 255u) || ws_bytes < L.total) return MOE_ERR_WORKSPACE;
  char* b = static_cast<char*>(ws);
  moe_layer_aux_t a = {};
  a.topk_idx = reinterpret_cast<int32_t*>(b + L.topk_idx);
  a.topk_w = reinterpret_cast<float*>(b + L.topk_w);
  a.expert_counts = reinterpret_cast<int32_t*>(b + L.counts);
  a.overflow = reinterpret_cast<int32_t*>(b + L.overflow);
  a.expert_offsets = reinterpret_cast<int32_t*>(b + L.offsets);
  a.segment_offsets = reinterpret_cast<int32_t*>(b + L.segoff);
  a.totals = reinterpret_cast<int32_t*>(b + L.totals);
  a.token_slot = reinterpret_cast<int32_t*>(b + L.slot);
  a.row_src = reinterpret_cast<int32_t*>(b + L.row_src);
  a.y = b + L.y;
  a.xq = reinterpret_cast<uint8_t*>(b + L.xp);
  a.xs = reinterpret_cast<uint8_t*>(b + L.xs);
  a.hq = reinterpret_cast<uint8_t*>(b + L.h);
  a.hs = reinterpret_cast<uint8_t*>(b + L.hs);
  if (aux) *aux = a;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int64_t R = max_rows(*cfg);
  st = cuda_status(launch_route(*cfg, logits, a.topk_idx, a.topk_w, a.expert_counts, a.overflow,
                                a.expert_offsets, a.segment_offsets, a.token_slot, a.row_src,
                                a.totals, reinterpret_cast<int32_t*>(b + L.blk_cnt), R, s));
  if (st != MOE_OK || cfg->T == 0) return st;
  if (!aligned16(x) || !aligned16(out) || !aligned16(wq_gu) || !aligned16(ws_gu) ||
      !aligned16(wq_d) || !aligned16(ws_d))
    return MOE_ERR_INVALID_ARG;
  st = cuda_status(launch_dispatch_fp8(*cfg, x, a.token_slot, a.xq, a.xs, s));
  if (st != MOE_OK) return st;
  st = launch_mlp_fp8(*cfg, a.xq, a.xs, a.expert_offsets, a.expert_counts, wq_gu, ws_gu, wq_d,
                      ws_d, a.hq, a.hs, a.y, R, static_cast<uint32_t*>(ws), s);
  if (st != MOE_OK) return st;
  return cuda_status(
      launch_combine(*cfg, a.y, a.token_slot, a.topk_w, sh_row0_or_none(*cfg), out, s));
}

moe_status_t moe_get_device_status(void* ws, moe_status_t* status, void* stream) {
  if (!ws || !status) return MOE_ERR_INVALID_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint32_t v = 0;
  if (cudaMemcpyAsync(&v, ws, 4, cudaMemcpyDeviceToHost, s) != cudaSuccess) return MOE_ERR_CUDA;
  if (cudaStreamSynchronize(s) != cudaSuccess) return MOE_ERR_CUDA;
  *status = static_cast<moe_status_t>(v);
  if (cudaMemsetAsync(ws, 0, 4, s) != cudaSuccess) return MOE_ERR_CUDA;
  return MOE_OK;
}

}  // extern "C"

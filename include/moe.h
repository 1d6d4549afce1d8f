/*
 * moe.h -- C ABI of libmoe.so: the single-GPU MoE expert layer on B200 (sm_100a).
 *
 *   route (top-K + softmax weights, histogram, capacity/overflow, owner-aligned
 *   offsets, permutation) -> dispatch -> grouped SwiGLU expert MLP -> combine
 *
 * The operations follow the pages this library is built from:
 *   - "Efficient and portable Mixture-of-Experts communication" (pplx-kernels):
 *     "Introductie" (router distribution, top-K, weighted average of expert
 *     outputs), "Dispatch" (pack tokens per expert, record the return address),
 *     "Combine" (gather 16-bit expert outputs, weighted average at the receiver).
 *   - "Enabling trillion-parameter models on AWS EFA": "Диспетчеризация и
 *     комбинирование" (count tokens per expert with shared-memory atomics in a
 *     block, cumulative sum -> offsets, pack contiguously), "MoE all-to-all через
 *     EFA" (grouped GEMM between dispatch and combine).
 *   - "MoE Expert Parallel Benchmark", Step 2: overflow = max(assigned - capacity, 0),
 *     effective tokens = sum(assigned - overflow).
 *   - "Mixture-of-Experts acceleration through overlap": remote-owner-aligned
 *     layout (each tile belongs to exactly one owner segment).
 *
 * Conventions for every entry point
 *   - Pointers named as device buffers are CUDA device pointers to row-major,
 *     contiguous data on the current device. The caller owns and allocates all
 *     of them; the library never allocates or frees device memory and keeps no
 *     per-call state on the host.
 *   - `stream` is a cudaStream_t passed as void* (NULL = the legacy default
 *     stream). Every call is asynchronous on that stream and never synchronises
 *     the host, except moe_get_device_status.
 *   - The return value reports argument, configuration, workspace and launch
 *     errors, detected before or at launch. Errors found by a kernel while it
 *     runs (a bounded wait that gave up, an expert id out of range in a
 *     caller-supplied table) are recorded in the workspace's status word and
 *     read with moe_get_device_status.
 *   - Shapes the kernels do not support return MOE_ERR_UNSUPPORTED; nothing is
 *     ever computed another way.
 *   - token_slot tables passed by the caller (moe_dispatch, moe_dispatch_fp8,
 *     moe_combine, moe_combine_wait): an entry that is negative or not below the
 *     routed rows min(T*K, E*C) + E*(A-1) is treated as a dropped assignment;
 *     nothing is written or read for it.
 *
 * Symbols: T tokens, H hidden size, E experts, K experts per token, F SwiGLU
 * width, S owner segments, C capacity per expert, A row alignment, R_max rows
 * of the dispatch buffer (moe_max_rows).
 *
 * Shared expert (n_shared = 1): an expert that every token uses with weight 1
 * next to its K routed experts (the shared experts whose multiplication the EFA
 * page runs while the dispatch transfers are in flight, "Диспетчеризация и
 * комбинирование"; the sum of routed and shared output is this library's
 * reading). It is stored as expert E of the weight arrays (w_gu and w_d hold
 * E + 1 experts, the shared one last, same F) and owns the T rows
 * [R_sh, R_sh + T) of xp, h and y, one per token in token order, where
 * R_sh = roundup(min(T*K, E*C) + E*(A-1), 128). Routing never selects it.
 */
#ifndef MOE_H
#define MOE_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  MOE_OK = 0,
  MOE_ERR_INVALID_ARG = 1,   /* null pointer, negative size, inconsistent config */
  MOE_ERR_UNSUPPORTED = 2,   /* valid config the kernels do not implement */
  MOE_ERR_WORKSPACE = 3,     /* workspace missing, misaligned or too small */
  MOE_ERR_CUDA = 4,          /* a CUDA runtime call or launch failed */
  MOE_ERR_TIMEOUT = 5,       /* device status: a bounded wait in a kernel gave up */
  MOE_ERR_DEVICE_INPUT = 6   /* device status: a caller table held an out-of-range id */
} moe_status_t;

typedef enum { MOE_F32 = 0, MOE_BF16 = 1 } moe_dtype_t;

/* Layer configuration. Limits: T >= 0; H >= 1; 1 <= E <= 1024; 1 <= K <= min(E, 32);
 * n_shared is 0 or 1 (a shared expert, see above);
 * F >= 1; S >= 1 and E % S == 0 (owner segment s holds experts [s*E/S, (s+1)*E/S));
 * capacity >= 0 (the per-expert limit C, see moe_capacity); 1 <= row_align <= 1024
 * (every expert's rows start at a multiple of A inside the dispatch buffer);
 * act_dtype is the dtype of x, the weights, xp, h, y and out.
 * Rows must be 16-byte multiples: H*sizeof(act) % 16 == 0, F*sizeof(act) % 16 == 0.
 * The bf16 expert MLP (tensor cores) also needs H % 64 == 0 and F % 64 == 0. */
typedef struct {
  int32_t T, H, E, K, F, S;
  int32_t capacity;
  int32_t row_align;
  int32_t act_dtype;
  int32_t n_shared;
} moe_config_t;

/* Pointers into the workspace where moe_layer_forward keeps the intermediates.
 * Filled by moe_layer_forward (host-side writes only) so that a caller can read
 * the route outputs, the dispatch buffer and the expert outputs afterwards. */
typedef struct {
  int32_t *topk_idx, *expert_counts, *overflow, *expert_offsets, *segment_offsets;
  int32_t *token_slot, *row_src, *totals;
  float *topk_w;
  void *xp, *h, *y;
  float *logits;   /* [T,E]: the router projection's output (moe_layer_forward_x only) */
  uint8_t *xq, *xs, *hq, *hs;   /* fp8 payload and its scales (moe_layer_forward_fp8 only) */
} moe_layer_aux_t;

#define MOE_FLAG_NONE 0u
/* moe_layer_forward: overlap the combine with the down GEMM through per-block
 * ready counters (see moe_combine_wait). bf16 only; row_align % 128 == 0. */
#define MOE_FLAG_OVERLAP 1u

/* C = ceil(cf * T * K / E), computed in double precision; cf < 0 means no limit
 * and returns T (a token picks an expert at most once). Returns -1 if T < 0,
 * K < 1 or E < 1. ("MoE Expert Parallel Benchmark", Step 2, fixes capacity as the
 * per-expert, per-step limit; the capacity-factor formula is this library's
 * reading.) */
int32_t moe_capacity(int32_t T, int32_t K, int32_t E, double cf);

/* R_max = min(T*K, E*C) + E*(A-1): rows of the dispatch buffer xp (and of h, y
 * and row_src). Every kept assignment gets one row and each expert adds at most
 * A-1 rows of alignment padding (a fixed worst-case bound, as the pplx-kernels
 * page sizes its receive buffers, "Draagbare kernels"). With n_shared = 1,
 * R_max = R_sh + T (the shared expert's rows follow). Returns -1 for an
 * invalid config. */
int64_t moe_max_rows(const moe_config_t* cfg);

/* MOE_OK if cfg is valid and supported, else the status moe_layer_forward
 * would return for it. */
moe_status_t moe_check_config(const moe_config_t* cfg);

/* Bytes of workspace needed by moe_route_topk (per-block histograms and the
 * status word). */
size_t moe_route_workspace_bytes(const moe_config_t* cfg);

/* Bytes of workspace needed by moe_layer_forward: the route workspace plus
 * every intermediate (route outputs, xp, h, y), each 256-byte aligned. */
size_t moe_workspace_bytes(const moe_config_t* cfg, uint32_t flags);

/* Zero the workspace's status word (and nothing else). Call once after
 * allocating a workspace; asynchronous on `stream`. */
moe_status_t moe_workspace_init(void* ws, size_t ws_bytes, void* stream);

/* Route: steps "top-K + weights", "histogram + capacity + overflow" and
 * "owner-aligned offsets + permutation".
 * Defining passages: the pplx-kernels page, "Introductie" (each token's router
 * distribution picks its top-K experts, whose outputs are averaged with the
 * router's weights); the EFA page, "Диспетчеризация и комбинирование" (tokens
 * per expert counted with shared-memory atomics inside a block, a cumulative
 * sum turned into offsets, tokens packed contiguously per destination);
 * "MoE Expert Parallel Benchmark", Step 2 (overflow = max(assigned - capacity,
 * 0), effective tokens = sum of assigned - overflow); "Mixture-of-Experts
 * acceleration through overlap" (the buffer ordered by owner, every tile
 * inside one owner's rows).
 *   logits          [T,E] fp32, device, read only. Any bias is already added.
 *   topk_idx        [T,K] int32 out: experts by (logit descending, index ascending).
 *   topk_w          [T,K] fp32 out: softmax over the K selected logits.
 *   expert_counts   [E]   int32 out: assignments per expert (the histogram).
 *   overflow        [E]   int32 out: max(count - C, 0).
 *   expert_offsets  [E+1] int32 out: off[0]=0, off[e+1]=off[e]+roundup(min(count,C), A).
 *   segment_offsets [S+1] int32 out: off[s*E/S].
 *   token_slot      [T,K] int32 out: row of (t,k) in xp, or -1 if it overflowed.
 *                   The first C assignments of each expert in token order are kept.
 *   row_src         [R_max] int32 out: t*K+k for each kept row, -1 on padding rows,
 *                   T*K+t on the shared expert's row of token t (n_shared = 1).
 *   totals          [4]   int32 out: {T*K, effective N, total overflow, R = off[E]}.
 *   ws, ws_bytes    workspace of at least moe_route_workspace_bytes(cfg) bytes,
 *                   256-byte aligned; contents need not be initialised except the
 *                   status word (moe_workspace_init).
 * All outputs are written in full; the results are deterministic. */
moe_status_t moe_route_topk(const moe_config_t* cfg, const float* logits,
                            int32_t* topk_idx, float* topk_w, int32_t* expert_counts,
                            int32_t* overflow, int32_t* expert_offsets,
                            int32_t* segment_offsets, int32_t* token_slot,
                            int32_t* row_src, int32_t* totals,
                            void* ws, size_t ws_bytes, void* stream);

/* moe_route_topk with a selection-only bias. Experts are selected by the fp32 sum
 * logits[t,e] + sel_bias[e], in the same order (larger first, then lower index);
 * the weights are the softmax over the selected experts' unbiased logits. This is
 * the bias-for-selection routing of DeepSeek-style routers, written with this
 * library's weight rule. sel_bias: [E] fp32 device, or NULL (then identical to
 * moe_route_topk). Other arguments as moe_route_topk. */
moe_status_t moe_route_topk_biased(const moe_config_t* cfg, const float* logits,
                                   const float* sel_bias, int32_t* topk_idx, float* topk_w,
                                   int32_t* expert_counts, int32_t* overflow,
                                   int32_t* expert_offsets, int32_t* segment_offsets,
                                   int32_t* token_slot, int32_t* row_src, int32_t* totals,
                                   void* ws, size_t ws_bytes, void* stream);

/* Router projection: the small linear layer in front of the route ("Introductie"
 * of the pplx-kernels page; the EFA page's introduction):
 *   logits[t,e] = sum_h x[t,h] * w_g[e,h], fp32 accumulation, stored as fp32.
 *   x [T,H] act, w_g [E,H] act, logits [T,E] fp32 out (device).
 *   ws: any workspace with a status word (at least 256 bytes).
 * bf16 runs on the tcgen05 tensor cores (a one-group instance of the grouped
 * GEMM), fp32 on CUDA cores (FFMA). Same shape limits as moe_expert_mlp. */
moe_status_t moe_router_logits(const moe_config_t* cfg, const void* x, const void* w_g,
                               float* logits, void* ws, size_t ws_bytes, void* stream);

/* Bytes of the fixed device scratch area used by moe_route_topk_noalloc. */
#define MOE_NOALLOC_SCRATCH_BYTES (1u << 20)

/* moe_route_topk for callers that cannot allocate device memory (no counterpart
 * on the pages; an addition of this library).
 * Some callers cannot call cudaMalloc or hand out a workspace: code that runs
 * inside another framework's allocator, plug-ins that receive only their input
 * and output buffers, or code paths where an allocation could fail at a bad
 * moment. This entry point takes the same arguments as moe_route_topk without
 * ws/ws_bytes and produces identical results. Its scratch (the per-block expert
 * histograms, ceil(T/b) * E * 4 bytes, b the tokens of a route block: 32 for
 * T <= 9472, 64 for T <= 18944, else 128) lives in a fixed device array of
 * MOE_NOALLOC_SCRATCH_BYTES (1 MiB) inside the library, which every GPU that
 * loads the library holds until the process exits.
 *   - It calls no cudaMalloc, cudaFree or allocating library routine.
 *   - Configurations needing more scratch than 1 MiB (ceil(T/b) * E > 262144)
 *     return MOE_ERR_WORKSPACE and launch nothing.
 *   - The first call on a device looks up the array's device address
 *     (cudaGetSymbolAddress) and caches it; make that first call before any
 *     stream capture on that device. The cached address belongs to that
 *     device's current context: after cudaDeviceReset (which unloads the
 *     library's kernels and their array) it is stale, so do not call this
 *     entry point again in a process that has reset the device.
 *   - Every call shares the one array, which keeps the last call's contents;
 *     the kernels write every scratch entry before reading it, so nothing needs
 *     to start at zero. Calls whose kernels overlap on the GPU (different
 *     streams, or threads without ordering between them) race on the array and
 *     give wrong results: serialise them. */
moe_status_t moe_route_topk_noalloc(const moe_config_t* cfg, const float* logits,
                                    int32_t* topk_idx, float* topk_w, int32_t* expert_counts,
                                    int32_t* overflow, int32_t* expert_offsets,
                                    int32_t* segment_offsets, int32_t* token_slot,
                                    int32_t* row_src, int32_t* totals, void* stream);

/* Dispatch ("Dispatch" of the pplx-kernels page): xp[token_slot[t,k]] = x[t],
 * a bit copy, for every (t,k) with token_slot >= 0, and xp[R_sh + t] = x[t]
 * when n_shared = 1.
 *   x          [T,H] act, device, read only.
 *   token_slot [T,K] int32 from moe_route_topk.
 *   xp         [R_max,H] act out; rows no slot points at are not written. */
moe_status_t moe_dispatch(const moe_config_t* cfg, const void* x, const int32_t* token_slot,
                          void* xp, void* stream);

/* Grouped SwiGLU expert MLP (the EFA page, "MoE all-to-all через EFA": the
 * experts' grouped GEMM runs between dispatch and combine on the packed rows;
 * the DistributedMoE README, "Результаты экспериментов": one grouped GEMM
 * instead of many small per-expert GEMMs; the SwiGLU form of the expert is this
 * library's reading, the pages give none). For every expert e and every row r in
 * [off_e, off_e + min(count_e, C)):
 *   h[r] = silu(xp[r] Wg_e^T) * (xp[r] Wu_e^T)   (fp32 accumulate, rounded to act)
 *   y[r] = h[r] W_d,e^T                          (fp32 accumulate, rounded to act)
 *   xp             [R_max,H] act.
 *   expert_offsets [E+1] int32, expert_counts [E] int32 (raw counts; the kept
 *                  count min(count, C) is derived on the device).
 *   w_gu           [E+n_shared,2F,H] act: rows 0..F-1 are Wg_e, rows F..2F-1 are Wu_e.
 *   w_d            [E+n_shared,H,F] act.
 *   With n_shared = 1 the shared expert E also maps rows [R_sh, R_sh + T).
 *   h              [R_max,F] act out (scratch for the second GEMM), y [R_max,H] act out.
 *   Rows outside every expert's kept range hold unspecified values afterwards
 *   (an expert's alignment padding rows may be written; no reader uses them).
 *   ws, ws_bytes   any workspace with a status word (at least 256 bytes).
 * bf16 runs on tcgen05 tensor cores (TMA-fed persistent grouped GEMM); fp32 runs
 * on a CUDA-core FFMA grouped GEMM (fp32 inputs, no TF32). */
moe_status_t moe_expert_mlp(const moe_config_t* cfg, const void* xp,
                            const int32_t* expert_offsets, const int32_t* expert_counts,
                            const void* w_gu, const void* w_d, void* h, void* y,
                            void* ws, size_t ws_bytes, void* stream);

/* Combine ("Combine" of the pplx-kernels page): out[t] = sum over k in order of
 * topk_w[t,k] * y[token_slot[t,k]] for slots >= 0, plus y[R_sh + t] when
 * n_shared = 1, fp32 accumulation, rounded once to act. Dropped assignments
 * contribute zero (no renormalisation); a token with every assignment dropped
 * gets zeros (or its shared expert's output alone).
 *   y [R_max,H] act, token_slot [T,K] int32, topk_w [T,K] fp32, out [T,H] act. */
moe_status_t moe_combine(const moe_config_t* cfg, const void* y, const int32_t* token_slot,
                         const float* topk_w, void* out, void* stream);

/* The combine as the consumer of a tile-signalled overlap ("Mixture-of-Experts
 * acceleration through overlap": the GEMM publishes tile-ready flags in its
 * epilogue and a separate kernel starts on each tile as soon as its flag is set).
 * Same result as moe_combine. Before reading the rows of token t, the kernel
 * waits until row_ready[slot / 128] >= ready_target for every kept slot of t,
 * and for its shared row R_sh + t when n_shared = 1 (acquire loads). moe_expert_mlp's down GEMM, run by moe_layer_forward with
 * MOE_FLAG_OVERLAP, adds 1 to a block's counter per stored 256-column tile
 * (release), so the target there is ceil(H / 256). The kernel does not wait for
 * the previous kernel in the stream, so token_slot and topk_w must already be
 * final when it starts; only the rows of y are waited for.
 *   row_ready   [ceil(R_max / 128)] uint32, device.
 *   timeout_us  bound of all waits; on expiry the kernel records MOE_ERR_TIMEOUT
 *               in the workspace's status word (moe_get_device_status), stops
 *               waiting everywhere and leaves the affected rows of out unwritten.
 *   ws          a workspace holding the status word (at least 256 bytes).
 * Requires row_align % 128 == 0 (every 128-row block belongs to one expert). */
moe_status_t moe_combine_wait(const moe_config_t* cfg, const void* y, const int32_t* token_slot,
                              const float* topk_w, const uint32_t* row_ready,
                              uint32_t ready_target, void* out, uint32_t timeout_us, void* ws,
                              size_t ws_bytes, void* stream);

/* The whole layer on `stream`: route -> dispatch -> expert MLP -> combine (the
 * cycle of the pplx-kernels page, "Introductie", "Dispatch" and "Combine", and
 * of the EFA page, "MoE all-to-all через EFA": dispatch to the experts, the
 * experts' grouped GEMM, combine back to token order by weighted average), with
 * every intermediate in the workspace (moe_workspace_bytes). `aux` may be NULL;
 * otherwise it receives the workspace pointers of the intermediates. No host
 * synchronisation: the per-expert counts stay on the device. With n_shared = 1 and
 * bf16, the shared expert's GEMM reads its rows straight from x, so the shared
 * rows of xp are not written. flags: MOE_FLAG_NONE,
 * or MOE_FLAG_OVERLAP (the combine overlaps the down GEMM; bf16 with
 * row_align % 128 == 0, else MOE_ERR_UNSUPPORTED; identical results). */
moe_status_t moe_layer_forward(const moe_config_t* cfg, const float* logits, const void* x,
                               const void* w_gu, const void* w_d, void* out,
                               uint32_t flags, void* ws, size_t ws_bytes,
                               moe_layer_aux_t* aux, void* stream);

/* The layer from hidden states: moe_router_logits (into the workspace) ->
 * moe_route_topk_biased -> dispatch -> expert MLP -> combine. w_g [E,H] act;
 * sel_bias [E] fp32 or NULL. flags: MOE_FLAG_NONE or MOE_FLAG_OVERLAP, as for
 * moe_layer_forward. aux->logits receives the logits' workspace address. */
moe_status_t moe_layer_forward_x(const moe_config_t* cfg, const void* x, const void* w_g,
                                 const float* sel_bias, const void* w_gu, const void* w_d,
                                 void* out, uint32_t flags, void* ws, size_t ws_bytes,
                                 moe_layer_aux_t* aux, void* stream);

/* ---------------------------------------------------------------------------
 * fp8 block-scaled variant ("Enabling trillion-parameter models on AWS EFA",
 * "Оценка": fp8 with block scaling for the dispatch, bf16 for the combine; the
 * pplx-kernels page, "Dispatch": tokens travel with their block scale factors).
 *
 * Format (the pages fix neither block shape nor scale encoding; this is the
 * library's reading): e4m3 codes (round to nearest even); one scale per 128
 * consecutive elements of a row along the contraction dimension; the scale is a
 * power of two 2^p stored as the byte p + 127 (UE8M0), p the smallest integer
 * >= -127 with max|block| <= 448 * 2^p.
 * Scale layout (what the tensor cores read): with KG = ceil(cols / 512), for each
 * block of 128 rows and each group of four 128-element k blocks a 512-byte chunk
 * at ((r / 128) * KG + kb / 4) * 512; row r's scale for k block kb is byte
 * 16*(r % 32) + 4*((r % 128) / 32) + kb % 4 of it. A [rows, cols] matrix has
 * moe_fp8_scale_bytes(rows, cols) bytes of scales; bytes of rows (or k blocks)
 * past the matrix are never written.
 * The whole fp8 path requires bf16 activations, H % 256 == 0, F % 128 == 0,
 * row_align % 128 == 0 and E <= 512 (else MOE_ERR_UNSUPPORTED). A shared expert
 * (n_shared = 1) works as in the bf16 path: its weights are the last of the
 * quantised arrays and its rows [R_sh, R_sh + T) of xq / hq / y are the tokens.
 * ------------------------------------------------------------------------- */

/* ceil(rows / 128) * ceil(cols / 512) * 512, or -1 if rows < 0 or cols is not a
 * positive multiple of 128. */
int64_t moe_fp8_scale_bytes(int64_t rows, int64_t cols);

/* Block-quantise a [rows, cols] bf16 matrix (device, row-major; cols % 128 == 0):
 * codes [rows, cols] e4m3 bytes, scales in the layout above. Used once for the
 * expert weights: w_gu as [E*2F, H] and w_d as [E*H, F]. */
moe_status_t moe_quantize_fp8(const void* src, int64_t rows, int64_t cols, uint8_t* codes,
                              uint8_t* scales, void* stream);

/* Dispatch with the fp8 payload: each token row of x [T,H] bf16 is quantised once
 * and its codes and scales written to every kept row token_slot[t,k] of
 * xq [R_max,H] (e4m3) and xs (moe_fp8_scale_bytes(R_max, H) bytes), and to its
 * shared-expert row R_sh + t when n_shared = 1. Rows no slot points at are not
 * written. */
moe_status_t moe_dispatch_fp8(const moe_config_t* cfg, const void* x, const int32_t* token_slot,
                              uint8_t* xq, uint8_t* xs, void* stream);

/* Grouped SwiGLU on the fp8 payload (tcgen05 block-scaled MMA, fp32 accumulate):
 * for every expert e and kept row r,
 *   h[r] = silu(xq[r] Wg_e^T) * (xq[r] Wu_e^T), quantised to hq[r] (e4m3) and hs
 *          (scales of the [R_max, F] matrix) from its fp32 value,
 *   y[r] = hq[r] W_d,e^T rounded to bf16,
 * with every operand taken as scale * e4m3 value. wq_gu [E',2F,H] e4m3 with scales
 * ws_gu of the [E'*2F, H] matrix; wq_d [E',H,F] with ws_d of [E'*H, F] (from
 * moe_quantize_fp8), E' = E + n_shared. y [R_max,H] bf16. ws: any workspace with
 * a status word. A caller offsets table whose expert leaves [0, R_max) or starts
 * off a multiple of 128 skips that expert and records MOE_ERR_DEVICE_INPUT. */
moe_status_t moe_expert_mlp_fp8(const moe_config_t* cfg, const uint8_t* xq, const uint8_t* xs,
                                const int32_t* expert_offsets, const int32_t* expert_counts,
                                const uint8_t* wq_gu, const uint8_t* ws_gu, const uint8_t* wq_d,
                                const uint8_t* ws_d, uint8_t* hq, uint8_t* hs, void* y, void* ws,
                                size_t ws_bytes, void* stream);

/* The whole layer with the fp8 payload: route -> moe_dispatch_fp8 ->
 * moe_expert_mlp_fp8 -> moe_combine (bf16), intermediates in the workspace
 * (moe_workspace_bytes). flags must be MOE_FLAG_NONE. aux (optional) also gets
 * xq, xs, hq, hs. */
moe_status_t moe_layer_forward_fp8(const moe_config_t* cfg, const float* logits, const void* x,
                                   const uint8_t* wq_gu, const uint8_t* ws_gu,
                                   const uint8_t* wq_d, const uint8_t* ws_d, void* out,
                                   uint32_t flags, void* ws, size_t ws_bytes,
                                   moe_layer_aux_t* aux, void* stream);

/* Synchronise `stream`, read the workspace's status word into *status and reset
 * it to MOE_OK. Returns MOE_ERR_CUDA if the synchronisation or copy failed. */
moe_status_t moe_get_device_status(void* ws, moe_status_t* status, void* stream);

/* Debugging aid (no counterpart on the pages). In the bounds-checked build of
 * the library (libmoe_check.so, compiled with -DMOE_CHECK_BOUNDS) every kernel
 * checks its internal index invariants (decoded tiles, TMEM columns,
 * shared-memory staging offsets, table indices); a failed check is counted
 * and skips the access it guards instead of stopping the kernel. This call
 * synchronises the device and returns the count and the source line of the
 * first failure on the current device, then zeroes them when reset != 0. The
 * release build returns MOE_ERR_UNSUPPORTED. */
moe_status_t moe_debug_bounds_failures(uint32_t* failures, uint32_t* first_line, int32_t reset);

/* Static text for a status code. */
const char* moe_status_string(moe_status_t status);

/* Library version as major*10000 + minor*100 + patch (1.1.0: the
 * expert-parallel entry points of moe_ep.h added; 1.2.0: their tile-signalled
 * form, moe_ep_t.flags). */
int32_t moe_version(void);

#ifdef __cplusplus
}
#endif

#endif /* MOE_H */

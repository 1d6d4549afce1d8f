/*
 * moe_ep.h -- C ABI of libmoe.so, expert-parallel part: the MoE layer split over
 * W ranks (one GPU each), rank d owning the experts [d*E/W, (d+1)*E/W).
 *
 * What the pages fix and what this interface does with it:
 *   - "Enabling trillion-parameter models on AWS EFA", "Буферы отправки и
 *     получения": the dispatch first exchanges the token counts per expert;
 *     from them each sender knows where its rows go and each receiver at which
 *     offset every sender's rows arrive. Inside a node the receive buffers are
 *     mapped into the peers, which write into them directly; the combine reads
 *     the expert outputs back and takes the weighted average.
 *   - "Efficient and portable Mixture-of-Experts communication", "Draagbare
 *     kernels": send and receive halves, each pair with its own symmetric
 *     buffers; a fixed bound on what a rank sends bounds what it receives per
 *     local expert and sender, so every sender derives a unique destination
 *     address without synchronising with the other senders; the receive layout
 *     is the one the expert GEMM needs.
 *   - "Mixture-of-Experts acceleration through overlap": the rows bound for
 *     one owner are contiguous (remote-owner-aligned layout); readiness is
 *     signalled by flags that the consumer polls.
 *
 * The layer per rank, in four steps (moe_ep_layer_forward runs all four):
 *   1. moe_ep_route: the one-rank route (moe_route_topk) of this rank's T tokens
 *      over all E experts, with capacity C enforced on this rank's batch; then
 *      its E counts are written into every rank's counts table (row = this
 *      rank) and each rank's COUNTS flag for this rank is set to `epoch`.
 *   2. moe_ep_dispatch: wait until every rank's counts of this epoch are here;
 *      derive the layout (below); write each kept token row straight into its
 *      owner's receive buffer xr; when every row is written, set each owner's
 *      DISPATCH flag for this rank.
 *   3. moe_ep_expert_mlp: with a shared expert, first its SwiGLU on this rank's
 *      own tokens (x), which needs nothing from the peers and so runs while
 *      their rows are in flight (the pages multiply the shared experts while
 *      the dispatch transfers are pending: EFA page, "Диспетчеризация и
 *      комбинирование"; pplx-kernels page, "Draagbare kernels"); then wait
 *      for every rank's DISPATCH flag; run the grouped SwiGLU (the tcgen05
 *      kernel of moe_expert_mlp) over the local experts' received rows into y;
 *      set every rank's Y flag for this rank.
 *   4. moe_ep_combine: wait for every rank's Y flag; out[t] = sum over kept k,
 *      in k order, of w[t,k] * (the owner's y row of that assignment), read
 *      from the owner's memory, plus (n_shared = 1) the rank's own shared-expert
 *      row with weight 1; fp32 accumulation, one rounding (as moe_combine).
 *   Every rank's out equals moe_layer_forward of its own tokens over all E
 *   experts (and the shared expert, if any): the same rows meet the same
 *   weights in the same order.
 *
 * Layout. kept[s][e] = min(count of rank s for expert e, C). On owner d, local
 * expert j (e = d*E/W + j) receives recv_counts[j] = sum_s kept[s][e] rows from
 * recv_offsets[j] on (an exclusive scan over j, each count rounded up to A),
 * rank 0's block first, then rank 1's, ...; each block in the sender's row
 * order (token order). Rank s writes its kept row of (t,k) to row
 * send_dst_row[e] + (token_slot[t,k] - expert_offsets[e]) of owner(e)'s xr,
 * with send_dst_row[e] = recv_offsets_owner[j] + sum_{s' < s} kept[s'][e].
 * The receive buffers hold R_recv = min(W*T*min(K, E/W), (E/W)*W*C) + (E/W)*(A-1)
 * rows (moe_ep_recv_rows).
 *
 * Memory. Each rank allocates one symmetric region of moe_ep_symmetric_bytes
 * (counts table [W][E] int32, flags [3][W] uint32, ready counters
 * [2][ceil(R_recv/128)] uint32, xr [R_recv][H], y [R_recv][H])
 * that its peers write into (counts, flags, xr) and read from (y), and a private
 * workspace of moe_ep_workspace_bytes (status word, route outputs, layout, h,
 * and with a shared expert its h and y for this rank's tokens).
 * `sym` is this rank's region as a pointer of this process; `peers` is a DEVICE
 * array of W pointers: peers[r] = rank r's region as mapped into this process
 * (peers[rank] = sym). Regions are zeroed once with moe_ep_symmetric_init on
 * every rank, followed by a barrier of the caller's (e.g. torch.distributed),
 * before the first step. moe_ep_sym_alloc and the moe_ipc_* calls below give a
 * region that another process can map (CUDA IPC; no multicast objects).
 *
 * Steps and reuse. `epoch` is the step number: 1 for the first step, one more
 * for each further step, the same on all ranks. epoch = 0 asks for the step
 * counter kept in the private workspace instead: the step's number is then one
 * past the counter, and the Y wait of moe_ep_combine (the step's last wait)
 * advances the counter, so that a step captured in a CUDA graph can be
 * replayed (every rank must then run its four steps in order, every step).
 * moe_ep_workspace_init zeroes the counter and the status word.
 * No barrier is needed between steps. A rank starts step e+1 (writing peers'
 * counts and xr) only after its combine of step e has seen every owner's Y
 * flag of step e, and an owner sets that flag after its GEMM of step e, the
 * last reader of its counts and xr of step e. An owner overwrites its y in step
 * e+1 only after every rank's DISPATCH flag of step e+1, which each rank sets
 * after its combine of step e, the reader of that y. (The combine reads the
 * owners' y in place.)
 *
 * Errors. Arguments: return codes as in moe.h. Every wait on a peer's flag is
 * bounded by timeout_us (0 = 2 s); one that runs out records MOE_ERR_TIMEOUT in
 * the status word (moe_get_device_status on the private workspace), and the
 * later waits then give up at once; the rank writes nothing more into its
 * peers' memory (no counts, rows or flags) and reads nothing more from it, so
 * its peers time out too instead of waiting. Its combine then leaves `out`
 * untouched (whatever the caller's buffer held before the step); its other
 * outputs of such a step are unspecified, and the group must be set up again
 * (moe_ep_workspace_init, moe_ep_symmetric_init and a barrier on every rank)
 * before its next step. A row whose computed destination falls outside the
 * receive buffer is not written and records MOE_ERR_DEVICE_INPUT.
 *
 * Limits: everything moe_expert_mlp supports for bf16 (tcgen05) plus
 * E % W == 0, S % W == 0, 1 <= W <= 64; fp32 activations use the CUDA-core
 * grouped GEMM and take no shared expert. Else MOE_ERR_UNSUPPORTED (or
 * INVALID_ARG).
 */
#ifndef MOE_EP_H
#define MOE_EP_H

#include "moe.h"

#ifdef __cplusplus
extern "C" {
#endif

/* Tile signalling ("Mixture-of-Experts acceleration through overlap": a
 * persistent GEMM that consumes rows as they arrive and publishes its output
 * tiles through flags that the consumer polls; remote-first tile order).
 * MOE_EP_TILE_SIGNAL (bf16 activations: the bf16 and the fp8 layer; row_align
 *   % 128 == 0; else MOE_ERR_UNSUPPORTED):
 *   - moe_ep_expert_mlp does not wait for every sender before its grouped
 *     GEMM: each CTA of the gate/up GEMM waits, before it loads its 128 rows of
 *     a tile, only for the DISPATCH flags of the senders whose rows those are
 *     (inside a local expert the senders' blocks follow in rank order). Before
 *     the down GEMM it waits for every sender (an owner overwrites y only after
 *     every rank's combine of the previous step has read it), and the down GEMM
 *     publishes each 128-row block of y through a ready counter in the
 *     symmetric region (one more per stored 256-column tile, released at
 *     system scope; two banks, by step parity).
 *   - moe_ep_combine does not wait for every owner's Y flag first: a token is
 *     combined as soon as the ready counters of its kept rows' blocks on their
 *     owners reach ceil(H/256). The Y flags are waited for after the combine
 *     (they still order the next step's writes into the peers).
 *   Results are bit for bit those of the untagged layer.
 * MOE_EP_REMOTE_FIRST (with MOE_EP_TILE_SIGNAL): the owner's GEMMs run the
 *   tiles that hold other senders' rows first and the tiles holding only its
 *   own rows last, so that the rows other ranks read are finished first. */
#define MOE_EP_TILE_SIGNAL 1u
#define MOE_EP_REMOTE_FIRST 2u

typedef struct {
  int32_t world;        /* W ranks */
  int32_t rank;         /* this rank, 0 <= rank < W */
  uint32_t epoch;       /* step number (>= 1, the same on every rank), or 0: the device-resident step counter */
  uint32_t timeout_us;  /* bound of each wait on a peer's flag; 0 = 2 000 000 */
  uint32_t flags;       /* MOE_EP_TILE_SIGNAL | MOE_EP_REMOTE_FIRST, or 0; the same on every rank */
} moe_ep_t;

/* Where the layer keeps its per-rank intermediates (host-side pointer values
 * into the caller's private workspace and symmetric region). */
typedef struct {
  int32_t *topk_idx, *expert_counts, *overflow, *expert_offsets, *segment_offsets;
  int32_t *token_slot, *row_src, *totals;
  float *topk_w;
  int32_t *counts_all;     /* [W][E]: every rank's expert counts (symmetric region) */
  uint32_t *flags;         /* [3][W]: COUNTS, DISPATCH, Y flags, by sender (symmetric) */
  int32_t *send_dst_row;   /* [E]: first row of this rank's block in owner(e)'s xr */
  int32_t *recv_offsets;   /* [E/W + 1]: local experts' first rows in xr, then the end */
  int32_t *recv_counts;    /* [E/W]: rows each local expert received */
  void *xr, *h, *y;        /* [R_recv][H] (symmetric), [R_recv][F] (private), [R_recv][H] (symmetric) */
  void *h_shared, *y_shared;   /* [T][F], [T][H] (private): the shared expert on this rank's tokens; NULL without one */
  uint8_t *xq, *xs;        /* fp8 layer: codes [R_recv][H] and scales, inside xr's region (symmetric) */
  uint8_t *hq, *hs;        /* fp8 layer: codes [R_recv][F] and scales, inside h's region (private) */
  int32_t *recv_split;     /* [E/W][W+1]: first row of sender s's block inside each local
                              expert's rows, and [W] = the rows it received (private) */
  uint32_t *y_ready;       /* [2][ceil(R_recv/128)]: ready counters of y's 128-row blocks,
                              bank (step & 1) (symmetric; MOE_EP_TILE_SIGNAL) */
} moe_ep_aux_t;

/* R_recv (see above); -1 for an invalid config or world. */
int64_t moe_ep_recv_rows(const moe_config_t* cfg, int32_t world);
/* Bytes of the symmetric region / of the private workspace; 0 if invalid. */
size_t moe_ep_symmetric_bytes(const moe_config_t* cfg, int32_t world);
size_t moe_ep_workspace_bytes(const moe_config_t* cfg, int32_t world);
/* MOE_OK if cfg and ep describe a supported expert-parallel layer. */
moe_status_t moe_ep_check(const moe_config_t* cfg, const moe_ep_t* ep);
/* Fill *aux from sym and ws (host only, no device work). */
moe_status_t moe_ep_aux(const moe_config_t* cfg, const moe_ep_t* ep, void* sym, void* ws,
                        moe_ep_aux_t* aux);
/* Zero the status word and the step counter of a private workspace
 * (stream-ordered); once, before the first step. */
moe_status_t moe_ep_workspace_init(const moe_config_t* cfg, int32_t world, void* ws,
                                   size_t ws_bytes, void* stream);
/* Zero the counts table and flags of this rank's region (stream-ordered). */
moe_status_t moe_ep_symmetric_init(const moe_config_t* cfg, int32_t world, void* sym,
                                   size_t sym_bytes, void* stream);

/* The four steps and the whole layer (see above). logits [T][E] fp32, x [T][H]
 * act; w_gu_local [E/W + n_shared][2F][H], w_d_local [E/W + n_shared][H][F]:
 * this rank's experts in ascending order, then the shared expert; out [T][H]
 * act. All device pointers, 16-byte aligned. moe_ep_expert_mlp reads x only
 * for the shared expert (NULL allowed when n_shared = 0). */
moe_status_t moe_ep_route(const moe_config_t* cfg, const moe_ep_t* ep, const float* logits,
                          void* sym, void* const* peers, void* ws, size_t ws_bytes, void* stream);
moe_status_t moe_ep_dispatch(const moe_config_t* cfg, const moe_ep_t* ep, const void* x,
                             void* sym, void* const* peers, void* ws, size_t ws_bytes,
                             void* stream);
moe_status_t moe_ep_expert_mlp(const moe_config_t* cfg, const moe_ep_t* ep, const void* x,
                               const void* w_gu_local, const void* w_d_local, void* sym,
                               void* const* peers, void* ws, size_t ws_bytes, void* stream);
moe_status_t moe_ep_combine(const moe_config_t* cfg, const moe_ep_t* ep, void* sym,
                            void* const* peers, void* out, void* ws, size_t ws_bytes,
                            void* stream);
moe_status_t moe_ep_layer_forward(const moe_config_t* cfg, const moe_ep_t* ep,
                                  const float* logits, const void* x, const void* w_gu_local,
                                  const void* w_d_local, void* sym, void* const* peers,
                                  void* out, moe_ep_aux_t* aux, void* ws, size_t ws_bytes,
                                  void* stream);

/* fp8 payload (the pages' production precision for the dispatch, with a bf16
 * combine: EFA page, "Оценка"; block scale factors travel beside the tokens:
 * pplx-kernels page, "Dispatch"). The route and the combine are the bf16
 * layer's (moe_ep_route, moe_ep_combine).
 *   moe_ep_dispatch_fp8: as moe_ep_dispatch, but each kept token row is
 *     quantised once (e4m3 codes, one UE8M0 scale per 128 values, the format
 *     and scale layout of moe_dispatch_fp8 in moe.h) and its codes and scales
 *     are written into the owner's xq / xs (the bytes crossing to a peer halve).
 *   moe_ep_expert_mlp_fp8: as moe_ep_expert_mlp with the block-scaled fp8
 *     grouped GEMMs of moe_expert_mlp_fp8 on the local experts (h quantised
 *     to fp8 in the gate/up epilogue, y in bf16). wq_gu_local [E/W][2F][H] and
 *     wq_d_local [E/W][H][F] are codes of this rank's experts, ws_gu_local /
 *     ws_d_local their scales in the blocked layout (for the experts of rank d,
 *     the contiguous slice of moe_quantize_fp8's scales of all experts that
 *     starts at chunk row d*(E/W)*2F/128, resp. d*(E/W)*H/128).
 *   With MOE_EP_TILE_SIGNAL the fp8 gate/up GEMM waits per CTA for the
 *     senders of its rows (their codes and scale chunks) and the fp8 down GEMM
 *     publishes y's 128-row blocks through the same ready counters as the bf16
 *     layer; MOE_EP_REMOTE_FIRST orders its tiles the same way.
 * Limits: those of moe_layer_forward_fp8 on each rank's local experts
 * (bf16 activations, H % 256 == 0, F % 128 == 0, A % 128 == 0); with
 * MOE_EP_REMOTE_FIRST the order's tables (two ints per local expert) must fit
 * the fp8 GEMM's shared memory beside its stages (about 340 local experts
 * with 256-row tiles); else MOE_ERR_UNSUPPORTED. A shared expert (n_shared
 * = 1) is run by every rank on its own tokens, as in the bf16 layer. */
moe_status_t moe_ep_dispatch_fp8(const moe_config_t* cfg, const moe_ep_t* ep, const void* x,
                                 void* sym, void* const* peers, void* ws, size_t ws_bytes,
                                 void* stream);
moe_status_t moe_ep_expert_mlp_fp8(const moe_config_t* cfg, const moe_ep_t* ep,
                                   const uint8_t* wq_gu_local, const uint8_t* ws_gu_local,
                                   const uint8_t* wq_d_local, const uint8_t* ws_d_local,
                                   void* sym, void* const* peers, void* ws, size_t ws_bytes,
                                   void* stream);
moe_status_t moe_ep_layer_forward_fp8(const moe_config_t* cfg, const moe_ep_t* ep,
                                      const float* logits, const void* x,
                                      const uint8_t* wq_gu_local, const uint8_t* ws_gu_local,
                                      const uint8_t* wq_d_local, const uint8_t* ws_d_local,
                                      void* sym, void* const* peers, void* out,
                                      moe_ep_aux_t* aux, void* ws, size_t ws_bytes,
                                      void* stream);

/* Setup (not the hot path): a symmetric region another process can map.
 * moe_ep_sym_alloc: cudaMalloc of `bytes` on the current device (its own
 * allocation, so that an IPC handle covers exactly it); moe_ep_sym_free frees it.
 * moe_ipc_get_handle writes the 64-byte CUDA IPC handle of such a region;
 * moe_ipc_open maps a peer's region into this process (*ptr), moe_ipc_close
 * unmaps it. Return MOE_ERR_CUDA when the runtime call fails. */
moe_status_t moe_ep_sym_alloc(size_t bytes, void** ptr);
moe_status_t moe_ep_sym_free(void* ptr);
moe_status_t moe_ipc_get_handle(void* ptr, uint8_t handle[64]);
moe_status_t moe_ipc_open(const uint8_t handle[64], void** ptr);
moe_status_t moe_ipc_close(void* ptr);

#ifdef __cplusplus
}
#endif

#endif /* MOE_EP_H */

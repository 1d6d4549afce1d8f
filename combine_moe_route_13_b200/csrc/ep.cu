// Expert parallelism: the layer split over W ranks, rank d owning the experts
// [d*E/W, (d+1)*E/W), with every exchange done by this library's kernels
// over peer memory (plain loads and stores through peer pointers; no
// multicast objects, no library collectives).
//
// Follows:
//  - "Enabling trillion-parameter models on AWS EFA", "Буферы отправки и
//    получения": counts per expert are exchanged first; from them senders
//    find where their rows go and receivers where each sender's rows land.
//    Inside a node the receive buffers are mapped into the peers, which write
//    into them directly.
//  - "Efficient and portable Mixture-of-Experts communication", "Draagbare
//    kernels": send halves that never block, receive halves that wait for
//    their data; a fixed per-sender bound gives every sender a unique
//    destination address with no synchronisation among senders; the received
//    rows are already in the expert GEMM's layout.
//  - "Mixture-of-Experts acceleration through overlap": flags published by
//    the producer and polled by the consumer.
//
// Kernels, in the order of a step on one rank:
//   publish   every rank's counts table gets this rank's E counts; COUNTS flag
//   plan      wait for all COUNTS flags; kept = min(count, C); scans give
//             send_dst_row[E], recv_offsets[E/W+1], recv_counts[E/W]
//   dispatch  blocks stride over tokens: a row is read once and written to
//             the owners of its kept experts
//   signal    every owner's DISPATCH flag for this rank, after the dispatch
//   (shared)  with a shared expert: its GEMM on this rank's own tokens, which
//             needs nothing from the peers and overlaps their dispatch
//   wait      one thread: all DISPATCH flags (then the grouped GEMM of
//             moe_expert_mlp over the local experts)
//   signal    every rank's Y flag for this rank, after the GEMM
//   wait      all Y flags
//   combine   blocks stride over tokens: the owners' y rows of a token's kept
//             assignments, read in place, weighted sum in k order, plus the
//             rank's own shared-expert row with weight 1
// Flags hold the step number (epoch) and are compared as "reached", so they
// are never reset. The step number is the caller's, or (epoch 0) one past a
// step counter in the workspace that the last wait of every step advances, so
// that a captured step can be replayed. Every wait is bounded; see moe_ep.h
// for the error rules.
#include <algorithm>
#include <climits>
#include <cstring>

#include "fp8_util.cuh"
#include "moe_internal.h"
#include "vec_util.cuh"
#include "../../include/moe_ep.h"

namespace moe {
namespace {

constexpr int EP_THREADS = 128;
constexpr int EP_UNROLL = 4;
constexpr int MAX_W = 64;
constexpr int PLAN_THREADS = 1024;   // >= MAX_E: one thread per expert
enum : int { FLAG_COUNTS = 0, FLAG_DISPATCH = 1, FLAG_Y = 2, NUM_FLAGS = 3 };

struct SymLayout {
  size_t counts = 0, flags = 0, yready = 0, xr = 0, y = 0, total = 0;
};

struct EpWs {
  size_t blk_cnt = 0, topk_idx = 0, topk_w = 0, counts = 0, overflow = 0, offsets = 0;
  size_t segoff = 0, totals = 0, slot = 0, row_src = 0;
  size_t send_dst = 0, recv_off = 0, recv_cnt = 0, split = 0, epoch = 0, h = 0, h_sh = 0, y_sh = 0;
  size_t x_sh = 0;   // fp8 layer with a shared expert: this rank's quantised tokens
  size_t total = 0;
};

int64_t recv_rows(const moe_config_t& c, int W) {
  const int64_t El = c.E / W;
  return std::min<int64_t>((int64_t)W * c.T * std::min<int64_t>(c.K, El),
                           El * W * (int64_t)c.capacity) +
         El * (c.row_align - 1);
}

// 128-row blocks of a receive buffer: the ready counters of one bank.
int64_t ready_blocks(const moe_config_t& c, int W) { return ceil_div(recv_rows(c, W), READY_ROWS); }

// The grouped GEMM's view of a rank: its E/W local experts, each with up to
// W*C received rows, R_recv rows in all (max_rows of this config = R_recv).
moe_config_t local_cfg(const moe_config_t& c, int W) {
  moe_config_t l = c;
  l.T = W * c.T;
  l.E = c.E / W;
  l.K = std::min(c.K, c.E / W);
  l.S = 1;
  l.capacity = W * c.capacity;
  l.n_shared = 0;
  return l;
}

// Bytes of an fp8 payload of `rows` rows of `cols` values: the codes, then (from
// the next 256-byte boundary) the scale bytes; 0 where cols is not a multiple
// of the scale block. The fp8 layer keeps xq/xs in the xr region and hq/hs in
// the h region.
size_t fp8_bytes(int64_t rows, int64_t cols) {
  if (cols % FP8_BLOCK != 0) return 0;
  return align256((size_t)rows * cols) + (size_t)sf_bytes(rows, cols);
}

SymLayout sym_layout(const moe_config_t& c, int W) {
  SymLayout L;
  const int64_t R = recv_rows(c, W);
  const size_t as = act_size(c.act_dtype);
  size_t p = 0;
  L.counts = p; p += align256((size_t)W * c.E * 4);
  L.flags = p;  p += align256((size_t)NUM_FLAGS * W * 4);
  L.yready = p; p += align256((size_t)2 * ready_blocks(c, W) * 4);
  L.xr = p;     p += align256(std::max<size_t>((size_t)R * c.H * as, fp8_bytes(R, c.H)));
  L.y = p;      p += align256((size_t)R * c.H * as);
  L.total = p;
  return L;
}

EpWs ep_ws_layout(const moe_config_t& c, int W) {
  EpWs L;
  const int64_t nblk = route_blocks(c.T);
  const int64_t TK = (int64_t)c.T * c.K;
  const int El = c.E / W;
  size_t p = 256;   // status word
  L.blk_cnt = p;   p += align256((size_t)std::max<int64_t>(nblk, 1) * c.E * 4);
  L.topk_idx = p;  p += align256((size_t)TK * 4);
  L.topk_w = p;    p += align256((size_t)TK * 4);
  L.counts = p;    p += align256((size_t)c.E * 4);
  L.overflow = p;  p += align256((size_t)c.E * 4);
  L.offsets = p;   p += align256((size_t)(c.E + 1) * 4);
  L.segoff = p;    p += align256((size_t)(c.S + 1) * 4);
  L.totals = p;    p += align256(16);
  L.slot = p;      p += align256((size_t)TK * 4);
  L.row_src = p;   p += align256((size_t)routed_rows(c) * 4);
  L.send_dst = p;  p += align256((size_t)c.E * 4);
  L.recv_off = p;  p += align256((size_t)(El + 1) * 4);
  L.recv_cnt = p;  p += align256((size_t)El * 4);
  L.split = p;     p += align256((size_t)El * (W + 1) * 4);
  L.epoch = p;     p += 256;   // the device-resident step counter
  L.h = p;         p += align256(std::max<size_t>((size_t)recv_rows(c, W) * c.F * act_size(c.act_dtype),
                                                 fp8_bytes(recv_rows(c, W), c.F)));
  if (c.n_shared) {   // the shared expert's h and y for this rank's own tokens
    L.h_sh = p;    p += align256(std::max<size_t>((size_t)c.T * c.F * act_size(c.act_dtype),
                                                  fp8_bytes(c.T, c.F)));
    L.y_sh = p;    p += align256((size_t)c.T * c.H * act_size(c.act_dtype));
    L.x_sh = p;    p += align256(fp8_bytes(c.T, c.H));   // codes + scales (fp8 layer)
  }
  L.total = p;
  return L;
}

moe_status_t ep_validate(const moe_config_t* c, const moe_ep_t* ep) {
  if (!c || !ep) return MOE_ERR_INVALID_ARG;
  moe_status_t st = validate(c, true);
  if (st != MOE_OK) return st;
  const int W = ep->world;
  if (W < 1 || ep->rank < 0 || ep->rank >= W) return MOE_ERR_INVALID_ARG;
  if (W > MAX_W) return MOE_ERR_UNSUPPORTED;
  if (c->E % W != 0 || c->S % W != 0) return MOE_ERR_INVALID_ARG;
  if ((int64_t)W * c->T > INT_MAX / 2 || (int64_t)W * c->capacity > INT_MAX / 2)
    return MOE_ERR_UNSUPPORTED;
  if (recv_rows(*c, W) > INT_MAX / 2) return MOE_ERR_UNSUPPORTED;
  if (ep->flags & ~(MOE_EP_TILE_SIGNAL | MOE_EP_REMOTE_FIRST)) return MOE_ERR_INVALID_ARG;
  if ((ep->flags & MOE_EP_REMOTE_FIRST) && !(ep->flags & MOE_EP_TILE_SIGNAL))
    return MOE_ERR_INVALID_ARG;
  if ((ep->flags & MOE_EP_TILE_SIGNAL) &&
      (c->act_dtype != MOE_BF16 || c->row_align % READY_ROWS != 0))
    return MOE_ERR_UNSUPPORTED;
  const moe_config_t l = local_cfg(*c, W);
  return validate(&l, true);
}

// The fp8 expert-parallel layer: the fp8 grouped GEMM's limits on each rank's
// local experts (and on its shared expert); with the remote-first order its
// tables must fit the kernel's shared memory too.
moe_status_t ep_validate_fp8(const moe_config_t* c, const moe_ep_t* ep) {
  moe_status_t st = ep_validate(c, ep);
  if (st != MOE_OK) return st;
  const moe_config_t l = local_cfg(*c, ep->world);
  if ((ep->flags & MOE_EP_REMOTE_FIRST) && fp8_ep_smem_bytes(l, true) > 227 * 1024)
    return MOE_ERR_UNSUPPORTED;
  return validate_fp8(&l);
}

moe_status_t ws_check(const moe_config_t& c, int W, const void* ws, size_t ws_bytes) {
  if (!ws || (reinterpret_cast<uintptr_t>(ws) & 255u) || ws_bytes < ep_ws_layout(c, W).total)
    return MOE_ERR_WORKSPACE;
  return MOE_OK;
}

moe_status_t cuda_st(cudaError_t e) { return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA; }

unsigned long long timeout_ns(const moe_ep_t& ep) {
  return ep.timeout_us ? (unsigned long long)ep.timeout_us * 1000ull : WAIT_LIMIT_NS;
}

// ---------------------------------------------------------------------------
// device side

__device__ __forceinline__ uint32_t ld_acquire_sys(const uint32_t* p) {
  uint32_t v;
  asm volatile("ld.acquire.sys.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

__device__ __forceinline__ void st_release_sys(uint32_t* p, uint32_t v) {
  asm volatile("st.release.sys.global.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

__device__ __forceinline__ unsigned long long ep_globaltimer() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ bool reached(uint32_t v, uint32_t epoch) {
  return (int32_t)(v - epoch) >= 0;
}

// This step's number: the caller's (value > 0), or one past the rank's
// device-resident step counter (value 0), which the Y wait of the combine
// advances at the end of every step, so that a captured step can be replayed.
struct Epoch {
  uint32_t value;
  const uint32_t* counter;
};

__device__ __forceinline__ uint32_t step_epoch(const Epoch& e) {
  return e.value ? e.value : *(volatile const uint32_t*)e.counter + 1u;
}

__device__ __forceinline__ uint32_t* peer_flags(void* const* peers, int d, size_t flags_off) {
  return reinterpret_cast<uint32_t*>(static_cast<char*>(peers[d]) + flags_off);
}

// One thread: wait until flags[0..W) have reached `epoch` (acquire). Gives up
// after timeout_ns, or at once when an earlier wait of this rank gave up,
// recording MOE_ERR_TIMEOUT.
__device__ bool wait_all(const uint32_t* flags, int W, uint32_t epoch,
                         unsigned long long timeout_ns, uint32_t* status) {
  const unsigned long long t0 = ep_globaltimer();
  for (int s = 0; s < W; ++s) {
    unsigned sleep_ns = 32;
    while (!reached(ld_acquire_sys(flags + s), epoch)) {
      if (*(volatile uint32_t*)status == (uint32_t)MOE_ERR_TIMEOUT ||
          ep_globaltimer() - t0 > timeout_ns) {
        atomicCAS(status, 0u, (uint32_t)MOE_ERR_TIMEOUT);
        return false;
      }
      __nanosleep(sleep_ns);
      if (sleep_ns < 2048) sleep_ns *= 2;
    }
  }
  return true;
}

__device__ __forceinline__ bool timed_out(const uint32_t* status) {
  return *(volatile const uint32_t*)status == (uint32_t)MOE_ERR_TIMEOUT;
}

// Block d writes this rank's counts into rank d's table, then sets rank d's
// COUNTS flag for this rank (release, after a system-scope fence that orders
// the whole block's writes before it). A rank that has timed out writes
// nothing into its peers' memory.
__global__ void ep_publish_kernel(const int32_t* __restrict__ counts, int E, int W, int rank,
                                  void* const* __restrict__ peers, size_t counts_off,
                                  size_t flags_off, Epoch epoch, const uint32_t* status) {
  __shared__ int s_skip;
  pdl_wait();
  pdl_trigger();
  if (threadIdx.x == 0) s_skip = timed_out(status);
  __syncthreads();
  if (s_skip) return;   // the same decision for every thread of the block
  const int d = blockIdx.x;
  int32_t* dst = reinterpret_cast<int32_t*>(static_cast<char*>(peers[d]) + counts_off) +
                 (size_t)rank * E;
  for (int e = threadIdx.x; e < E; e += blockDim.x) dst[e] = counts[e];
  __syncthreads();
  if (threadIdx.x == 0) {
    __threadfence_system();
    st_release_sys(peer_flags(peers, d, flags_off) + FLAG_COUNTS * W + rank, step_epoch(epoch));
  }
}

// One thread per expert e. tot = sum over senders of kept[s][e], pre = the
// part of it from senders before this rank; the aligned totals are scanned
// over all experts and each owner's scan restarts at its first expert.
__global__ void __launch_bounds__(PLAN_THREADS)
ep_plan_kernel(const int32_t* __restrict__ counts_all, const uint32_t* flags, int E, int W,
               int rank, int C, int A, Epoch epoch, unsigned long long timeout_ns,
               uint32_t* status, int32_t* __restrict__ send_dst, int32_t* __restrict__ recv_off,
               int32_t* __restrict__ recv_cnt, int32_t* __restrict__ split) {
  __shared__ long long s_scan[PLAN_THREADS];
  __shared__ int s_ok;
  pdl_wait();
  pdl_trigger();
  if (threadIdx.x == 0)
    s_ok = wait_all(flags + FLAG_COUNTS * W, W, step_epoch(epoch), timeout_ns, status);
  __syncthreads();
  const int e = threadIdx.x;
  const int El = E / W;
  MOE_CHECK(E <= PLAN_THREADS && W <= MAX_W);
  long long tot = 0, pre = 0;
  // a local expert's row split by sender: its senders' blocks in rank order
  int32_t* sp = (e < E && e / El == rank) ? split + (size_t)(e - rank * El) * (W + 1) : nullptr;
  if (e < E) {
    for (int s = 0; s < W; ++s) {
      if (sp) sp[s] = (int32_t)tot;
      // written by the peers: read from L2, never from a stale L1 line
      const int c = s_ok ? min(max(__ldcg(counts_all + (size_t)s * E + e), 0), C) : 0;
      tot += c;
      if (s < rank) pre += c;
    }
    if (sp) sp[W] = (int32_t)tot;
  }
  const long long aligned = (tot + A - 1) / A * A;
  s_scan[e] = e < E ? aligned : 0;
  __syncthreads();
  for (int off = 1; off < PLAN_THREADS; off <<= 1) {
    const long long v = e >= off ? s_scan[e - off] : 0;
    __syncthreads();
    s_scan[e] += v;
    __syncthreads();
  }
  if (e < E) {
    const int d = e / El;
    const int first = d * El;
    const long long first_excl = first == 0 ? 0 : s_scan[first - 1];
    const long long base = s_scan[e] - aligned - first_excl;
    // after a timeout every count reads as 0: nothing is sent or computed
    send_dst[e] = (int32_t)(base + pre);
    if (d == rank) {
      recv_off[e - first] = (int32_t)base;
      recv_cnt[e - first] = (int32_t)tot;
      if (e == first + El - 1) recv_off[El] = (int32_t)(s_scan[e] - first_excl);
    }
  }
}

// Blocks stride over the tokens (a grid of the blocks resident at once). The
// peer table is staged in shared memory once per block; for each token warp 0
// loads its slots, experts and their layout entries and packs the
// destinations of the kept assignments (k order); the row is read once and
// stored to each destination. After a timeout of this rank nothing is written.
// The DISPATCH flags are raised by ep_signal_kernel once this grid has
// finished (its stores are then complete and visible to the signalling grid).
__global__ void __launch_bounds__(EP_THREADS)
ep_dispatch_kernel(const uint4* __restrict__ x, const int32_t* __restrict__ topk_idx,
                   const int32_t* __restrict__ token_slot, const int32_t* __restrict__ offsets,
                   const int32_t* __restrict__ send_dst, void* const* __restrict__ peers,
                   size_t xr_off, int T, int K, int E, int El, int W, int row_vecs, int slot_end,
                   long long n_recv, uint32_t* status) {
  __shared__ uint4* s_dst[MAX_K];
  __shared__ char* s_peer[MAX_W];
  __shared__ int s_n, s_skip;
  pdl_wait();
  pdl_trigger();
  if (threadIdx.x < W) s_peer[threadIdx.x] = static_cast<char*>(peers[threadIdx.x]);
  if (threadIdx.x == 0) s_skip = timed_out(status);
  __syncthreads();
  if (s_skip) return;   // the same decision for every thread of the block
  const int k = threadIdx.x;
  for (int t = blockIdx.x; t < T; t += gridDim.x) {
    __syncthreads();   // the previous token's readers of s_dst and s_n are done
    if (k < 32) {
      uint4* dp = nullptr;
      if (k < K) {
        const int sl = token_slot[(size_t)t * K + k];
        const int e = topk_idx[(size_t)t * K + k];
        if (sl >= 0 && sl < slot_end) {
          const long long row =
              (e >= 0 && e < E) ? (long long)send_dst[e] + (sl - offsets[e]) : -1;
          if (row >= 0 && row < n_recv && MOE_CHECKED(e / El < W))
            dp = reinterpret_cast<uint4*>(s_peer[e / El] + xr_off) + row * row_vecs;
          else
            atomicCAS(status, 0u, (uint32_t)MOE_ERR_DEVICE_INPUT);
        }
      }
      const unsigned m = __ballot_sync(0xffffffffu, dp != nullptr);
      if (dp) s_dst[__popc(m & ((1u << k) - 1u))] = dp;
      if (k == 0) s_n = __popc(m);
    }
    __syncthreads();
    const int n = s_n;
    if (n == 0) continue;   // every assignment of this token overflowed
    const uint4* src = x + (size_t)t * row_vecs;
    for (int v0 = threadIdx.x; v0 < row_vecs; v0 += EP_THREADS * EP_UNROLL) {
      uint4 dv[EP_UNROLL];
#pragma unroll
      for (int u = 0; u < EP_UNROLL; ++u) {
        const int v = v0 + u * EP_THREADS;
        if (v < row_vecs) dv[u] = __ldcs(src + v);
      }
      for (int j = 0; j < n; ++j) {
        uint4* dst = s_dst[j];
#pragma unroll
        for (int u = 0; u < EP_UNROLL; ++u) {
          const int v = v0 + u * EP_THREADS;
          if (v < row_vecs) dst[v] = dv[u];
        }
      }
    }
  }
}

// The fp8 form of ep_dispatch_kernel: each kept token row is read once and
// quantised once, with the arithmetic of the one-rank fp8 dispatch (e4m3 codes,
// one UE8M0 scale per 128 values: a half-warp's 16 threads cover one block),
// and its codes and scale bytes are stored to each destination row of the
// owners' xq / xs.
__global__ void __launch_bounds__(EP_THREADS)
ep_dispatch_fp8_kernel(const uint4* __restrict__ x, const int32_t* __restrict__ topk_idx,
                       const int32_t* __restrict__ token_slot, const int32_t* __restrict__ offsets,
                       const int32_t* __restrict__ send_dst, void* const* __restrict__ peers,
                       size_t xq_off, size_t xs_off, int T, int K, int E, int El, int W,
                       int row_vecs, int slot_end, long long n_recv, uint32_t* status) {
  __shared__ char* s_base[MAX_K];
  __shared__ long long s_row[MAX_K];
  __shared__ char* s_peer[MAX_W];
  __shared__ int s_n, s_skip;
  pdl_wait();
  pdl_trigger();
  if (threadIdx.x < W) s_peer[threadIdx.x] = static_cast<char*>(peers[threadIdx.x]);
  if (threadIdx.x == 0) s_skip = timed_out(status);
  __syncthreads();
  if (s_skip) return;   // the same decision for every thread of the block
  const int k = threadIdx.x;
  const int64_t H = (int64_t)row_vecs * 8;
  const int KB = row_vecs / 16;
  for (int t = blockIdx.x; t < T; t += gridDim.x) {
    __syncthreads();   // the previous token's readers of s_base, s_row, s_n are done
    if (k < 32) {
      long long row = -1;
      int d = 0;
      if (k < K) {
        const int sl = token_slot[(size_t)t * K + k];
        const int e = topk_idx[(size_t)t * K + k];
        if (sl >= 0 && sl < slot_end) {
          row = (e >= 0 && e < E) ? (long long)send_dst[e] + (sl - offsets[e]) : -1;
          if (row < 0 || row >= n_recv) {
            atomicCAS(status, 0u, (uint32_t)MOE_ERR_DEVICE_INPUT);
            row = -1;
          }
          d = row >= 0 ? e / El : 0;
        }
      }
      const unsigned m = __ballot_sync(0xffffffffu, row >= 0);
      if (row >= 0) {
        const int pos = __popc(m & ((1u << k) - 1u));
        s_base[pos] = s_peer[d];
        s_row[pos] = row;
      }
      if (k == 0) s_n = __popc(m);
    }
    __syncthreads();
    const int n = s_n;
    if (n == 0) continue;   // every assignment of this token overflowed
    const uint4* src = x + (size_t)t * row_vecs;
    // row_vecs is a multiple of 16 and v0 of 128: a half-warp is all valid or all not
    for (int v0 = 0; v0 < row_vecs; v0 += EP_THREADS) {
      const int v = v0 + (int)threadIdx.x;
      const bool valid = v < row_vecs;
      float f[8];
      if (valid) {
        unpack_bf16x8(__ldcs(src + v), f);
      } else {
#pragma unroll
        for (int i = 0; i < 8; ++i) f[i] = 0.f;
      }
      float amax = 0.f;
#pragma unroll
      for (int i = 0; i < 8; ++i) amax = fmaxf(amax, fabsf(f[i]));
#pragma unroll
      for (int o = 1; o < 16; o <<= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
      if (!valid) continue;
      const int p = fp8_scale_exp(amax);
      const float inv = fp8_inv_scale(p);
      uint2 c;
      c.x = fp8x2(f[0] * inv, f[1] * inv) | (fp8x2(f[2] * inv, f[3] * inv) << 16);
      c.y = fp8x2(f[4] * inv, f[5] * inv) | (fp8x2(f[6] * inv, f[7] * inv) << 16);
      const uint8_t sbyte = (uint8_t)(p + 127);
      const int kb = v / 16;
      for (int j = 0; j < n; ++j) {
        char* base = s_base[j];
        const long long r = s_row[j];
        *reinterpret_cast<uint2*>(base + xq_off + r * H + (int64_t)v * 8) = c;
        if ((threadIdx.x & 15) == 0) base[xs_off + sf_offset(r, kb, KB)] = (char)sbyte;
      }
    }
  }
}

// advance (the last wait of a step): then move the rank's step counter on
// (device-resident numbering only).
__global__ void ep_wait_kernel(const uint32_t* flags, int W, Epoch epoch,
                               unsigned long long timeout_ns, uint32_t* status, uint32_t* advance) {
  pdl_wait();
  pdl_trigger();
  if (threadIdx.x == 0) {
    const uint32_t e = step_epoch(epoch);
    wait_all(flags, W, e, timeout_ns, status);
    if (advance && !epoch.value) *advance = e;
  }
}

// Before the down GEMM of a tile-signalled step: wait for every sender's
// DISPATCH flag (each is raised after that rank's combine of the previous
// step, the last reader of this owner's y and of the other bank of its ready
// counters), then zero that other bank, which the next step counts into.
__global__ void ep_wait_zero_kernel(const uint32_t* flags, int W, Epoch epoch,
                                    unsigned long long timeout_ns, uint32_t* status,
                                    uint32_t* yready, int nblk) {
  __shared__ int s_ok;
  pdl_wait();
  pdl_trigger();
  const uint32_t e = step_epoch(epoch);
  if (threadIdx.x == 0) s_ok = wait_all(flags, W, e, timeout_ns, status);
  __syncthreads();
  if (!s_ok) return;
  uint32_t* other = yready + (size_t)((e + 1u) & 1u) * nblk;
  for (int i = threadIdx.x; i < nblk; i += blockDim.x) other[i] = 0u;
}

// After the dispatch or the grouped GEMM (pdl_wait: that grid has finished and
// its stores are visible to this one): every rank's flag `which` for this rank,
// released at system scope after a system fence. Not after a timeout.
__global__ void ep_signal_kernel(void* const* __restrict__ peers, size_t flags_off, int which,
                                 int W, int rank, Epoch epoch, const uint32_t* status) {
  pdl_wait();
  pdl_trigger();
  const int d = threadIdx.x;
  if (d < W && !timed_out(status)) {
    __threadfence_system();
    st_release_sys(peer_flags(peers, d, flags_off) + which * W + rank, step_epoch(epoch));
  }
}

// out[t] = sum over kept k (k order) of w[t,k] * y_owner[row], fp32 FMA from
// 0, one rounding: the arithmetic of the one-rank combine, with the rows read
// in place from their owners. After a timeout of this rank nothing is read
// from the peers and `out` is left as it was.
// ready_target > 0 (tile signalling): before a token is combined, each kept
// row's 128-row block must have reached ready_target in its owner's ready
// counters (bank = step & 1; acquire at system scope, all waits bounded by one
// deadline); a token whose wait runs out is not written, nor is any later one.
template <bool BF16>
__global__ void __launch_bounds__(EP_THREADS)
ep_combine_kernel(const int32_t* __restrict__ topk_idx, const int32_t* __restrict__ token_slot,
                  const float* __restrict__ topk_w, const int32_t* __restrict__ offsets,
                  const int32_t* __restrict__ send_dst, void* const* __restrict__ peers,
                  size_t y_off, const uint4* __restrict__ y_sh, uint4* __restrict__ out, int T,
                  int K, int E, int El, int W, int row_vecs, int slot_end, long long n_recv,
                  uint32_t* status, size_t ready_off, int ready_nblk, uint32_t ready_target,
                  Epoch epoch, unsigned long long timeout_ns) {
  __shared__ const uint4* s_src[MAX_K];
  __shared__ float s_w[MAX_K];
  __shared__ char* s_peer[MAX_W];
  __shared__ int s_n, s_skip;
  pdl_wait();
  pdl_trigger();
  if (threadIdx.x < W) s_peer[threadIdx.x] = static_cast<char*>(peers[threadIdx.x]);
  if (threadIdx.x == 0) s_skip = timed_out(status);
  __syncthreads();
  if (s_skip) return;   // the same decision for every thread of the block
  constexpr int LANES = BF16 ? 8 : 4;
  const int k = threadIdx.x;
  const size_t bank = ready_target ? (size_t)(step_epoch(epoch) & 1u) * ready_nblk : 0;
  const unsigned long long deadline = ep_globaltimer() + timeout_ns;
  for (int t = blockIdx.x; t < T; t += gridDim.x) {
    __syncthreads();   // s_peer staged; the previous token's readers of s_src, s_w, s_n done
    if (k < 32) {      // warp 0 packs the kept assignments, k order
      const uint4* sp = nullptr;
      const uint32_t* ready = nullptr;
      float wt = 0.f;
      if (k < K) {
        const int sl = token_slot[(size_t)t * K + k];
        const int e = topk_idx[(size_t)t * K + k];
        wt = topk_w[(size_t)t * K + k];
        if (sl >= 0 && sl < slot_end) {
          const long long row =
              (e >= 0 && e < E) ? (long long)send_dst[e] + (sl - offsets[e]) : -1;
          if (row >= 0 && row < n_recv) {
            sp = reinterpret_cast<const uint4*>(s_peer[e / El] + y_off) + row * row_vecs;
            if (ready_target)
              ready = reinterpret_cast<const uint32_t*>(s_peer[e / El] + ready_off) + bank +
                      row / READY_ROWS;
          } else {
            atomicCAS(status, 0u, (uint32_t)MOE_ERR_DEVICE_INPUT);
          }
        }
      }
      // each lane waits for its own row's block on its owner
      bool ok = true;
      if (ready) {
        unsigned ns = 32;
        while (ld_acquire_sys(ready) < ready_target) {
          if (timed_out(status) || ep_globaltimer() > deadline) {
            atomicCAS(status, 0u, (uint32_t)MOE_ERR_TIMEOUT);
            ok = false;
            break;
          }
          __nanosleep(ns);
          if (ns < 1024) ns *= 2;
        }
      }
      const bool all_ok = __all_sync(0xffffffffu, ok);
      const unsigned m = __ballot_sync(0xffffffffu, sp != nullptr);
      if (sp) {
        const int pos = __popc(m & ((1u << k) - 1u));
        s_src[pos] = sp;
        s_w[pos] = wt;
      }
      if (k == 0) {
        s_n = __popc(m);
        s_skip = !all_ok;
      }
    }
    __syncthreads();
    if (s_skip) return;   // a wait ran out: this token and the rest stay unwritten
    const int n = s_n;
    uint4* dst = out + (size_t)t * row_vecs;
    for (int v0 = threadIdx.x; v0 < row_vecs; v0 += EP_THREADS * 2) {
      float acc[2][LANES];
#pragma unroll
      for (int u = 0; u < 2; ++u)
#pragma unroll
        for (int i = 0; i < LANES; ++i) acc[u][i] = 0.f;
      for (int kk = 0; kk < n; kk += 4) {
        uint4 d[4][2];
#pragma unroll
        for (int j = 0; j < 4; ++j)
#pragma unroll
          for (int u = 0; u < 2; ++u) {
            const int v = v0 + u * EP_THREADS;
            // rows written by another kernel, possibly on another GPU: read via L2
            d[j][u] = (kk + j < n && v < row_vecs) ? __ldcg(s_src[kk + j] + v)
                                                  : make_uint4(0u, 0u, 0u, 0u);
          }
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          if (kk + j >= n) continue;
          const float wk = s_w[kk + j];
#pragma unroll
          for (int u = 0; u < 2; ++u) {
            if (BF16) {
              float f[8];
              unpack_bf16x8(d[j][u], f);
#pragma unroll
              for (int i = 0; i < 8; ++i) acc[u][i] = fmaf(wk, f[i], acc[u][i]);
            } else {
              acc[u][0] = fmaf(wk, __uint_as_float(d[j][u].x), acc[u][0]);
              acc[u][1] = fmaf(wk, __uint_as_float(d[j][u].y), acc[u][1]);
              acc[u][2] = fmaf(wk, __uint_as_float(d[j][u].z), acc[u][2]);
              acc[u][3] = fmaf(wk, __uint_as_float(d[j][u].w), acc[u][3]);
            }
          }
        }
      }
      if (y_sh) {   // the shared expert's row, weight 1, after the routed terms
#pragma unroll
        for (int u = 0; u < 2; ++u) {
          const int v = v0 + u * EP_THREADS;
          if (v >= row_vecs) continue;
          const uint4 q = __ldg(y_sh + (size_t)t * row_vecs + v);
          if (BF16) {
            float f[8];
            unpack_bf16x8(q, f);
#pragma unroll
            for (int i = 0; i < 8; ++i) acc[u][i] += f[i];
          } else {
            acc[u][0] += __uint_as_float(q.x);
            acc[u][1] += __uint_as_float(q.y);
            acc[u][2] += __uint_as_float(q.z);
            acc[u][3] += __uint_as_float(q.w);
          }
        }
      }
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        const int v = v0 + u * EP_THREADS;
        if (v >= row_vecs) continue;
        uint4 o;
        if (BF16) {
          o.x = pack_bf16x2(acc[u][0], acc[u][1]);
          o.y = pack_bf16x2(acc[u][2], acc[u][3]);
          o.z = pack_bf16x2(acc[u][4], acc[u][5]);
          o.w = pack_bf16x2(acc[u][6], acc[u][7]);
        } else {
          o.x = __float_as_uint(acc[u][0]);
          o.y = __float_as_uint(acc[u][1]);
          o.z = __float_as_uint(acc[u][2]);
          o.w = __float_as_uint(acc[u][3]);
        }
        __stcs(dst + v, o);
      }
    }
  }
}

// ---------------------------------------------------------------------------
// host side

struct Ptrs {
  int32_t *topk_idx, *counts, *overflow, *offsets, *segoff, *slot, *row_src, *totals, *blk;
  float* topk_w;
  int32_t *send_dst, *recv_off, *recv_cnt, *split;
  uint32_t *status, *epoch;
  char *h, *h_sh, *y_sh, *x_sh;   // h_sh / y_sh / x_sh: nullptr without a shared expert
};

Ptrs ws_ptrs(const moe_config_t& c, int W, void* ws) {
  const EpWs L = ep_ws_layout(c, W);
  char* b = static_cast<char*>(ws);
  Ptrs p;
  p.status = reinterpret_cast<uint32_t*>(b);
  p.blk = reinterpret_cast<int32_t*>(b + L.blk_cnt);
  p.topk_idx = reinterpret_cast<int32_t*>(b + L.topk_idx);
  p.topk_w = reinterpret_cast<float*>(b + L.topk_w);
  p.counts = reinterpret_cast<int32_t*>(b + L.counts);
  p.overflow = reinterpret_cast<int32_t*>(b + L.overflow);
  p.offsets = reinterpret_cast<int32_t*>(b + L.offsets);
  p.segoff = reinterpret_cast<int32_t*>(b + L.segoff);
  p.totals = reinterpret_cast<int32_t*>(b + L.totals);
  p.slot = reinterpret_cast<int32_t*>(b + L.slot);
  p.row_src = reinterpret_cast<int32_t*>(b + L.row_src);
  p.send_dst = reinterpret_cast<int32_t*>(b + L.send_dst);
  p.recv_off = reinterpret_cast<int32_t*>(b + L.recv_off);
  p.recv_cnt = reinterpret_cast<int32_t*>(b + L.recv_cnt);
  p.split = reinterpret_cast<int32_t*>(b + L.split);
  p.epoch = reinterpret_cast<uint32_t*>(b + L.epoch);
  p.h = b + L.h;
  p.h_sh = c.n_shared ? b + L.h_sh : nullptr;
  p.y_sh = c.n_shared ? b + L.y_sh : nullptr;
  p.x_sh = c.n_shared ? b + L.x_sh : nullptr;
  return p;
}

moe_status_t common_checks(const moe_config_t* cfg, const moe_ep_t* ep, const void* sym,
                           void* const* peers, const void* ws, size_t ws_bytes) {
  moe_status_t st = ep_validate(cfg, ep);
  if (st != MOE_OK) return st;
  if (!sym || !peers) return MOE_ERR_INVALID_ARG;
  if (reinterpret_cast<uintptr_t>(sym) & 255u) return MOE_ERR_INVALID_ARG;
  return ws_check(*cfg, ep->world, ws, ws_bytes);
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace
}  // namespace moe

using namespace moe;

extern "C" {

int64_t moe_ep_recv_rows(const moe_config_t* cfg, int32_t world) {
  moe_ep_t ep = {world, 0, 1u, 0u};
  if (ep_validate(cfg, &ep) != MOE_OK) return -1;
  return recv_rows(*cfg, world);
}

size_t moe_ep_symmetric_bytes(const moe_config_t* cfg, int32_t world) {
  moe_ep_t ep = {world, 0, 1u, 0u};
  if (ep_validate(cfg, &ep) != MOE_OK) return 0;
  return sym_layout(*cfg, world).total;
}

size_t moe_ep_workspace_bytes(const moe_config_t* cfg, int32_t world) {
  moe_ep_t ep = {world, 0, 1u, 0u};
  if (ep_validate(cfg, &ep) != MOE_OK) return 0;
  return ep_ws_layout(*cfg, world).total;
}

moe_status_t moe_ep_check(const moe_config_t* cfg, const moe_ep_t* ep) {
  moe_status_t st = ep_validate(cfg, ep);
  if (st != MOE_OK) return st;
  return MOE_OK;
}

moe_status_t moe_ep_aux(const moe_config_t* cfg, const moe_ep_t* ep, void* sym, void* ws,
                        moe_ep_aux_t* aux) {
  moe_status_t st = ep_validate(cfg, ep);
  if (st != MOE_OK) return st;
  if (!sym || !ws || !aux) return MOE_ERR_INVALID_ARG;
  const Ptrs p = ws_ptrs(*cfg, ep->world, ws);
  const SymLayout S = sym_layout(*cfg, ep->world);
  char* sb = static_cast<char*>(sym);
  moe_ep_aux_t a = {};
  a.topk_idx = p.topk_idx;
  a.expert_counts = p.counts;
  a.overflow = p.overflow;
  a.expert_offsets = p.offsets;
  a.segment_offsets = p.segoff;
  a.token_slot = p.slot;
  a.row_src = p.row_src;
  a.totals = p.totals;
  a.topk_w = p.topk_w;
  a.counts_all = reinterpret_cast<int32_t*>(sb + S.counts);
  a.flags = reinterpret_cast<uint32_t*>(sb + S.flags);
  a.send_dst_row = p.send_dst;
  a.recv_offsets = p.recv_off;
  a.recv_counts = p.recv_cnt;
  a.xr = sb + S.xr;
  a.h = p.h;
  a.y = sb + S.y;
  a.h_shared = p.h_sh;
  a.y_shared = p.y_sh;
  a.recv_split = p.split;
  a.y_ready = reinterpret_cast<uint32_t*>(sb + S.yready);
  if (cfg->H % FP8_BLOCK == 0 && cfg->F % FP8_BLOCK == 0) {   // the fp8 layer's payload
    const int64_t R = recv_rows(*cfg, ep->world);
    a.xq = reinterpret_cast<uint8_t*>(sb + S.xr);
    a.xs = reinterpret_cast<uint8_t*>(sb + S.xr + align256((size_t)R * cfg->H));
    a.hq = reinterpret_cast<uint8_t*>(p.h);
    a.hs = reinterpret_cast<uint8_t*>(p.h + align256((size_t)R * cfg->F));
  }
  *aux = a;
  return MOE_OK;
}

moe_status_t moe_ep_workspace_init(const moe_config_t* cfg, int32_t world, void* ws,
                                   size_t ws_bytes, void* stream) {
  moe_ep_t ep = {world, 0, 1u, 0u};
  moe_status_t st = ep_validate(cfg, &ep);
  if (st != MOE_OK) return st;
  if ((st = ws_check(*cfg, world, ws, ws_bytes)) != MOE_OK) return st;
  const EpWs L = ep_ws_layout(*cfg, world);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if ((st = cuda_st(cudaMemsetAsync(ws, 0, 4, s))) != MOE_OK) return st;   // status word
  return cuda_st(cudaMemsetAsync(static_cast<char*>(ws) + L.epoch, 0, 4, s));   // step counter
}

moe_status_t moe_ep_symmetric_init(const moe_config_t* cfg, int32_t world, void* sym,
                                   size_t sym_bytes, void* stream) {
  moe_ep_t ep = {world, 0, 1u, 0u};
  moe_status_t st = ep_validate(cfg, &ep);
  if (st != MOE_OK) return st;
  const SymLayout S = sym_layout(*cfg, world);
  if (!sym || (reinterpret_cast<uintptr_t>(sym) & 255u)) return MOE_ERR_INVALID_ARG;
  if (sym_bytes < S.total) return MOE_ERR_WORKSPACE;
  return cuda_st(cudaMemsetAsync(sym, 0, S.xr, static_cast<cudaStream_t>(stream)));
}

moe_status_t moe_ep_route(const moe_config_t* cfg, const moe_ep_t* ep, const float* logits,
                          void* sym, void* const* peers, void* ws, size_t ws_bytes,
                          void* stream) {
  moe_status_t st = common_checks(cfg, ep, sym, peers, ws, ws_bytes);
  if (st != MOE_OK) return st;
  if (cfg->T > 0 && !logits) return MOE_ERR_INVALID_ARG;
  const moe_config_t& c = *cfg;
  const int W = ep->world;
  const Ptrs p = ws_ptrs(c, W, ws);
  const SymLayout S = sym_layout(c, W);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  st = cuda_st(launch_route(c, logits, p.topk_idx, p.topk_w, p.counts, p.overflow, p.offsets,
                            p.segoff, p.slot, p.row_src, p.totals, p.blk, routed_rows(c), s));
  if (st != MOE_OK) return st;
  return cuda_st(launch_pdl(ep_publish_kernel, dim3(W), dim3(256), 0, s,
                            (const int32_t*)p.counts, c.E, W, ep->rank, peers, S.counts, S.flags,
                            Epoch{ep->epoch, p.epoch}, (const uint32_t*)p.status));
}

moe_status_t moe_ep_dispatch(const moe_config_t* cfg, const moe_ep_t* ep, const void* x,
                             void* sym, void* const* peers, void* ws, size_t ws_bytes,
                             void* stream) {
  moe_status_t st = common_checks(cfg, ep, sym, peers, ws, ws_bytes);
  if (st != MOE_OK) return st;
  if (cfg->T > 0 && (!x || !aligned16(x))) return MOE_ERR_INVALID_ARG;
  const moe_config_t& c = *cfg;
  const int W = ep->world;
  const Ptrs p = ws_ptrs(c, W, ws);
  const SymLayout S = sym_layout(c, W);
  char* sb = static_cast<char*>(sym);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  st = cuda_st(launch_pdl(ep_plan_kernel, dim3(1), dim3(PLAN_THREADS), 0, s,
                          (const int32_t*)(sb + S.counts), (const uint32_t*)(sb + S.flags), c.E,
                          W, ep->rank, c.capacity, c.row_align, Epoch{ep->epoch, p.epoch},
                          timeout_ns(*ep),
                          p.status, p.send_dst, p.recv_off, p.recv_cnt, p.split));
  if (st != MOE_OK) return st;
  const int row_vecs = (int)((int64_t)c.H * act_size(c.act_dtype) / 16);
  if (c.T > 0) {
    st = cuda_st(launch_pdl(ep_dispatch_kernel,
                            dim3(resident_grid(ep_dispatch_kernel, EP_THREADS, c.T)),
                            dim3(EP_THREADS), 0, s, static_cast<const uint4*>(x),
                            (const int32_t*)p.topk_idx, (const int32_t*)p.slot,
                            (const int32_t*)p.offsets, (const int32_t*)p.send_dst, peers, S.xr,
                            c.T, c.K, c.E, c.E / W, W, row_vecs, (int)routed_rows(c),
                            (long long)recv_rows(c, W), p.status));
    if (st != MOE_OK) return st;
  }
  return cuda_st(launch_pdl(ep_signal_kernel, dim3(1), dim3(MAX_W), 0, s, peers, S.flags,
                            (int)FLAG_DISPATCH, W, ep->rank, Epoch{ep->epoch, p.epoch},
                            (const uint32_t*)p.status));
}

moe_status_t moe_ep_expert_mlp(const moe_config_t* cfg, const moe_ep_t* ep, const void* x,
                               const void* w_gu_local, const void* w_d_local, void* sym,
                               void* const* peers, void* ws, size_t ws_bytes, void* stream) {
  moe_status_t st = common_checks(cfg, ep, sym, peers, ws, ws_bytes);
  if (st != MOE_OK) return st;
  if (!w_gu_local || !w_d_local || !aligned16(w_gu_local) || !aligned16(w_d_local))
    return MOE_ERR_INVALID_ARG;
  if (cfg->n_shared && cfg->T > 0 && (!x || !aligned16(x))) return MOE_ERR_INVALID_ARG;
  const moe_config_t& c = *cfg;
  const int W = ep->world;
  const Ptrs p = ws_ptrs(c, W, ws);
  const SymLayout S = sym_layout(c, W);
  char* sb = static_cast<char*>(sym);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (c.n_shared) {
    // the shared expert on this rank's own tokens first: it needs nothing from
    // the peers, so it runs while their rows are still arriving
    const int El = c.E / W;
    const size_t as = act_size(c.act_dtype);
    const char* wg = static_cast<const char*>(w_gu_local) + (size_t)El * 2 * c.F * c.H * as;
    const char* wd = static_cast<const char*>(w_d_local) + (size_t)El * c.H * c.F * as;
    if (c.act_dtype == MOE_BF16) {
      st = launch_shared_mlp_bf16_tc(c, x, wg, wd, p.h_sh, p.y_sh, p.status, s);
    } else if (c.T > 0) {
      // the CUDA-core grouped SwiGLU with no routed group: its shared group is
      // rows [0, T) of x, with expert 0 of the shared expert's weights
      moe_config_t l = c;
      l.E = 0;
      l.K = 1;
      l.S = 1;
      l.capacity = 0;
      l.row_align = 1;
      l.n_shared = 1;
      st = cuda_st(launch_mlp_f32(l, static_cast<const float*>(x), nullptr, nullptr,
                                  reinterpret_cast<const float*>(wg),
                                  reinterpret_cast<const float*>(wd),
                                  reinterpret_cast<float*>(p.h_sh),
                                  reinterpret_cast<float*>(p.y_sh), c.T, s));
    }
    if (st != MOE_OK) return st;
  }
  const moe_config_t l = local_cfg(c, W);
  const int64_t R = recv_rows(c, W);
  const uint32_t* dispatch_flags = (const uint32_t*)(sb + S.flags) + FLAG_DISPATCH * W;
  if (ep->flags & MOE_EP_TILE_SIGNAL) {
    // gate/up: each CTA waits only for the senders of its rows; then every
    // sender (y and the other ready bank are free), then down, publishing y's
    // blocks as they are stored
    EpTiles t;
    t.arrive = dispatch_flags;
    t.split = p.split;
    t.counter = p.epoch;
    t.epoch = ep->epoch;
    t.W = W;
    t.rank = ep->rank;
    t.remote_first = (ep->flags & MOE_EP_REMOTE_FIRST) ? 1 : 0;
    t.wait_ns = timeout_ns(*ep);
    st = launch_mlp_bf16_tc_ep(l, 1, sb + S.xr, p.recv_off, p.recv_cnt, w_gu_local, w_d_local,
                               p.h, sb + S.y, R, p.status, s, t);
    if (st != MOE_OK) return st;
    const int nblk = (int)ready_blocks(c, W);
    st = cuda_st(launch_pdl(ep_wait_zero_kernel, dim3(1), dim3(1024), 0, s, dispatch_flags, W,
                            Epoch{ep->epoch, p.epoch}, timeout_ns(*ep), p.status,
                            reinterpret_cast<uint32_t*>(sb + S.yready), nblk));
    if (st != MOE_OK) return st;
    t.arrive = nullptr;
    t.yready = reinterpret_cast<uint32_t*>(sb + S.yready);
    t.ready_blocks = nblk;
    st = launch_mlp_bf16_tc_ep(l, 2, sb + S.xr, p.recv_off, p.recv_cnt, w_gu_local, w_d_local,
                               p.h, sb + S.y, R, p.status, s, t);
    if (st != MOE_OK) return st;
    return cuda_st(launch_pdl(ep_signal_kernel, dim3(1), dim3(MAX_W), 0, s, peers, S.flags,
                              (int)FLAG_Y, W, ep->rank, Epoch{ep->epoch, p.epoch},
                              (const uint32_t*)p.status));
  }
  st = cuda_st(launch_pdl(ep_wait_kernel, dim3(1), dim3(32), 0, s, dispatch_flags, W,
                          Epoch{ep->epoch, p.epoch}, timeout_ns(*ep), p.status,
                          (uint32_t*)nullptr));
  if (st != MOE_OK) return st;
  if (c.act_dtype == MOE_BF16)
    st = launch_mlp_bf16_tc(l, sb + S.xr, p.recv_off, p.recv_cnt, w_gu_local, w_d_local, p.h,
                            sb + S.y, R, p.status, s);
  else
    st = cuda_st(launch_mlp_f32(l, reinterpret_cast<const float*>(sb + S.xr), p.recv_off,
                                p.recv_cnt, static_cast<const float*>(w_gu_local),
                                static_cast<const float*>(w_d_local),
                                reinterpret_cast<float*>(p.h), reinterpret_cast<float*>(sb + S.y),
                                R, s));
  if (st != MOE_OK) return st;
  return cuda_st(launch_pdl(ep_signal_kernel, dim3(1), dim3(MAX_W), 0, s, peers, S.flags,
                            (int)FLAG_Y, W, ep->rank, Epoch{ep->epoch, p.epoch},
                            (const uint32_t*)p.status));
}

moe_status_t moe_ep_combine(const moe_config_t* cfg, const moe_ep_t* ep, void* sym,
                            void* const* peers, void* out, void* ws, size_t ws_bytes,
                            void* stream) {
  moe_status_t st = common_checks(cfg, ep, sym, peers, ws, ws_bytes);
  if (st != MOE_OK) return st;
  if (cfg->T > 0 && (!out || !aligned16(out))) return MOE_ERR_INVALID_ARG;
  const moe_config_t& c = *cfg;
  const int W = ep->world;
  const Ptrs p = ws_ptrs(c, W, ws);
  const SymLayout S = sym_layout(c, W);
  char* sb = static_cast<char*>(sym);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const bool tiles = (ep->flags & MOE_EP_TILE_SIGNAL) != 0;
  auto y_wait = [&]() {   // the step's last wait moves the step counter on
    return cuda_st(launch_pdl(ep_wait_kernel, dim3(1), dim3(32), 0, s,
                              (const uint32_t*)(sb + S.flags) + FLAG_Y * W, W,
                              Epoch{ep->epoch, p.epoch}, timeout_ns(*ep), p.status, p.epoch));
  };
  if (!tiles) {
    st = y_wait();
    if (st != MOE_OK || c.T == 0) return st;
  }
  if (c.T > 0) {
    const int row_vecs = (int)((int64_t)c.H * act_size(c.act_dtype) / 16);
    auto kernel = c.act_dtype == MOE_BF16 ? ep_combine_kernel<true> : ep_combine_kernel<false>;
    st = cuda_st(launch_pdl(kernel, dim3(resident_grid(kernel, EP_THREADS, c.T)),
                            dim3(EP_THREADS), 0, s, (const int32_t*)p.topk_idx,
                            (const int32_t*)p.slot, (const float*)p.topk_w,
                            (const int32_t*)p.offsets, (const int32_t*)p.send_dst, peers, S.y,
                            reinterpret_cast<const uint4*>(p.y_sh), static_cast<uint4*>(out),
                            c.T, c.K, c.E, c.E / W, W, row_vecs,
                            (int)routed_rows(c), (long long)recv_rows(c, W), p.status, S.yready,
                            (int)ready_blocks(c, W), tiles ? ready_target(c) : 0u,
                            Epoch{ep->epoch, p.epoch}, timeout_ns(*ep)));
    if (st != MOE_OK) return st;
  }
  // tile signalling: the Y flags still order the next step's writes into the peers
  return tiles ? y_wait() : MOE_OK;
}

moe_status_t moe_ep_layer_forward(const moe_config_t* cfg, const moe_ep_t* ep,
                                  const float* logits, const void* x, const void* w_gu_local,
                                  const void* w_d_local, void* sym, void* const* peers,
                                  void* out, moe_ep_aux_t* aux, void* ws, size_t ws_bytes,
                                  void* stream) {
  moe_status_t st = common_checks(cfg, ep, sym, peers, ws, ws_bytes);
  if (st != MOE_OK) return st;
  if (aux && (st = moe_ep_aux(cfg, ep, sym, ws, aux)) != MOE_OK) return st;
  if ((st = moe_ep_route(cfg, ep, logits, sym, peers, ws, ws_bytes, stream)) != MOE_OK) return st;
  if ((st = moe_ep_dispatch(cfg, ep, x, sym, peers, ws, ws_bytes, stream)) != MOE_OK) return st;
  if ((st = moe_ep_expert_mlp(cfg, ep, x, w_gu_local, w_d_local, sym, peers, ws, ws_bytes,
                              stream)) != MOE_OK)
    return st;
  return moe_ep_combine(cfg, ep, sym, peers, out, ws, ws_bytes, stream);
}

moe_status_t moe_ep_dispatch_fp8(const moe_config_t* cfg, const moe_ep_t* ep, const void* x,
                                 void* sym, void* const* peers, void* ws, size_t ws_bytes,
                                 void* stream) {
  moe_status_t st = ep_validate_fp8(cfg, ep);
  if (st != MOE_OK) return st;
  if ((st = common_checks(cfg, ep, sym, peers, ws, ws_bytes)) != MOE_OK) return st;
  if (cfg->T > 0 && (!x || !aligned16(x))) return MOE_ERR_INVALID_ARG;
  const moe_config_t& c = *cfg;
  const int W = ep->world;
  const Ptrs p = ws_ptrs(c, W, ws);
  const SymLayout S = sym_layout(c, W);
  const int64_t R = recv_rows(c, W);
  char* sb = static_cast<char*>(sym);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  st = cuda_st(launch_pdl(ep_plan_kernel, dim3(1), dim3(PLAN_THREADS), 0, s,
                          (const int32_t*)(sb + S.counts), (const uint32_t*)(sb + S.flags), c.E,
                          W, ep->rank, c.capacity, c.row_align, Epoch{ep->epoch, p.epoch},
                          timeout_ns(*ep),
                          p.status, p.send_dst, p.recv_off, p.recv_cnt, p.split));
  if (st != MOE_OK) return st;
  if (c.T > 0) {
    st = cuda_st(launch_pdl(ep_dispatch_fp8_kernel,
                            dim3(resident_grid(ep_dispatch_fp8_kernel, EP_THREADS, c.T)),
                            dim3(EP_THREADS), 0, s, static_cast<const uint4*>(x),
                            (const int32_t*)p.topk_idx, (const int32_t*)p.slot,
                            (const int32_t*)p.offsets, (const int32_t*)p.send_dst, peers, S.xr,
                            S.xr + align256((size_t)R * c.H), c.T, c.K, c.E, c.E / W, W,
                            c.H / 8, (int)routed_rows(c), (long long)R, p.status));
    if (st != MOE_OK) return st;
  }
  st = cuda_st(launch_pdl(ep_signal_kernel, dim3(1), dim3(MAX_W), 0, s, peers, S.flags,
                          (int)FLAG_DISPATCH, W, ep->rank, Epoch{ep->epoch, p.epoch},
                          (const uint32_t*)p.status));
  if (st != MOE_OK || !c.n_shared || c.T == 0) return st;
  // the shared expert's input: this rank's own token rows, quantised with the
  // dispatch's arithmetic (codes and blocked scales, rows from 0), after the
  // flags so that the peers' transfers are not held up by it
  uint8_t* xq_sh = reinterpret_cast<uint8_t*>(p.x_sh);
  return cuda_st(launch_quantize_fp8(x, c.T, c.H, xq_sh, xq_sh + align256((size_t)c.T * c.H), s));
}

moe_status_t moe_ep_expert_mlp_fp8(const moe_config_t* cfg, const moe_ep_t* ep,
                                   const uint8_t* wq_gu_local, const uint8_t* ws_gu_local,
                                   const uint8_t* wq_d_local, const uint8_t* ws_d_local,
                                   void* sym, void* const* peers, void* ws, size_t ws_bytes,
                                   void* stream) {
  moe_status_t st = ep_validate_fp8(cfg, ep);
  if (st != MOE_OK) return st;
  if ((st = common_checks(cfg, ep, sym, peers, ws, ws_bytes)) != MOE_OK) return st;
  for (const void* w : {(const void*)wq_gu_local, (const void*)ws_gu_local,
                        (const void*)wq_d_local, (const void*)ws_d_local})
    if (!w || !aligned16(w)) return MOE_ERR_INVALID_ARG;
  const moe_config_t& c = *cfg;
  const int W = ep->world;
  const Ptrs p = ws_ptrs(c, W, ws);
  const SymLayout S = sym_layout(c, W);
  const int64_t R = recv_rows(c, W);
  char* sb = static_cast<char*>(sym);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (c.n_shared && c.T > 0) {
    // the shared expert on this rank's own tokens first (codes and scales of
    // the last local expert; it needs nothing from the peers)
    const int El = c.E / W;
    const int64_t kg_gu = ceil_div(c.H / FP8_BLOCK, 4), kg_d = ceil_div(c.F / FP8_BLOCK, 4);
    moe_config_t l = c;
    l.E = 0;
    l.K = 1;
    l.S = 1;
    l.capacity = 0;
    l.row_align = 128;
    l.n_shared = 1;
    const uint8_t* xq_sh = reinterpret_cast<const uint8_t*>(p.x_sh);
    uint8_t* hq_sh = reinterpret_cast<uint8_t*>(p.h_sh);
    st = launch_mlp_fp8(
        l, xq_sh, xq_sh + align256((size_t)c.T * c.H), nullptr, nullptr,
        wq_gu_local + (size_t)El * 2 * c.F * c.H,
        ws_gu_local + (size_t)El * 2 * c.F / 128 * kg_gu * SF_CHUNK,
        wq_d_local + (size_t)El * c.H * c.F, ws_d_local + (size_t)El * c.H / 128 * kg_d * SF_CHUNK,
        hq_sh, hq_sh + align256((size_t)c.T * c.F), p.y_sh, c.T, p.status, s);
    if (st != MOE_OK) return st;
  }
  const uint32_t* dispatch_flags = (const uint32_t*)(sb + S.flags) + FLAG_DISPATCH * W;
  const moe_config_t l = local_cfg(c, W);
  const uint8_t* xq = reinterpret_cast<const uint8_t*>(sb + S.xr);
  const uint8_t* xs = xq + align256((size_t)R * c.H);
  uint8_t* hq = reinterpret_cast<uint8_t*>(p.h);
  uint8_t* hs = hq + align256((size_t)R * c.F);
  if (ep->flags & MOE_EP_TILE_SIGNAL) {
    // as the bf16 layer: gate/up waits per CTA for the senders of its rows
    // (codes and scale chunks), then every sender (y and the other ready bank
    // are free), then down, publishing y's blocks as they are stored
    EpTiles t;
    t.arrive = dispatch_flags;
    t.split = p.split;
    t.counter = p.epoch;
    t.epoch = ep->epoch;
    t.W = W;
    t.rank = ep->rank;
    t.remote_first = (ep->flags & MOE_EP_REMOTE_FIRST) ? 1 : 0;
    t.wait_ns = timeout_ns(*ep);
    st = launch_mlp_fp8_ep(l, 1, xq, xs, p.recv_off, p.recv_cnt, wq_gu_local, ws_gu_local,
                           wq_d_local, ws_d_local, hq, hs, sb + S.y, R, p.status, s, t);
    if (st != MOE_OK) return st;
    const int nblk = (int)ready_blocks(c, W);
    st = cuda_st(launch_pdl(ep_wait_zero_kernel, dim3(1), dim3(1024), 0, s, dispatch_flags, W,
                            Epoch{ep->epoch, p.epoch}, timeout_ns(*ep), p.status,
                            reinterpret_cast<uint32_t*>(sb + S.yready), nblk));
    if (st != MOE_OK) return st;
    t.arrive = nullptr;
    t.yready = reinterpret_cast<uint32_t*>(sb + S.yready);
    t.ready_blocks = nblk;
    st = launch_mlp_fp8_ep(l, 2, xq, xs, p.recv_off, p.recv_cnt, wq_gu_local, ws_gu_local,
                           wq_d_local, ws_d_local, hq, hs, sb + S.y, R, p.status, s, t);
    if (st != MOE_OK) return st;
    return cuda_st(launch_pdl(ep_signal_kernel, dim3(1), dim3(MAX_W), 0, s, peers, S.flags,
                              (int)FLAG_Y, W, ep->rank, Epoch{ep->epoch, p.epoch},
                              (const uint32_t*)p.status));
  }
  st = cuda_st(launch_pdl(ep_wait_kernel, dim3(1), dim3(32), 0, s, dispatch_flags, W,
                          Epoch{ep->epoch, p.epoch}, timeout_ns(*ep), p.status,
                          (uint32_t*)nullptr));
  if (st != MOE_OK) return st;
  st = launch_mlp_fp8(l, xq, xs, p.recv_off, p.recv_cnt, wq_gu_local, ws_gu_local, wq_d_local,
                      ws_d_local, hq, hs, sb + S.y, R, p.status, s);
  if (st != MOE_OK) return st;
  return cuda_st(launch_pdl(ep_signal_kernel, dim3(1), dim3(MAX_W), 0, s, peers, S.flags,
                            (int)FLAG_Y, W, ep->rank, Epoch{ep->epoch, p.epoch},
                            (const uint32_t*)p.status));
}

moe_status_t moe_ep_layer_forward_fp8(const moe_config_t* cfg, const moe_ep_t* ep,
                                      const float* logits, const void* x,
                                      const uint8_t* wq_gu_local, const uint8_t* ws_gu_local,
                                      const uint8_t* wq_d_local, const uint8_t* ws_d_local,
                                      void* sym, void* const* peers, void* out,
                                      moe_ep_aux_t* aux, void* ws, size_t ws_bytes,
                                      void* stream) {
  moe_status_t st = ep_validate_fp8(cfg, ep);
  if (st != MOE_OK) return st;
  if ((st = common_checks(cfg, ep, sym, peers, ws, ws_bytes)) != MOE_OK) return st;
  if (aux && (st = moe_ep_aux(cfg, ep, sym, ws, aux)) != MOE_OK) return st;
  if ((st = moe_ep_route(cfg, ep, logits, sym, peers, ws, ws_bytes, stream)) != MOE_OK) return st;
  if ((st = moe_ep_dispatch_fp8(cfg, ep, x, sym, peers, ws, ws_bytes, stream)) != MOE_OK)
    return st;
  if ((st = moe_ep_expert_mlp_fp8(cfg, ep, wq_gu_local, ws_gu_local, wq_d_local, ws_d_local, sym,
                                  peers, ws, ws_bytes, stream)) != MOE_OK)
    return st;
  return moe_ep_combine(cfg, ep, sym, peers, out, ws, ws_bytes, stream);
}

moe_status_t moe_ep_sym_alloc(size_t bytes, void** ptr) {
  if (!ptr || bytes == 0) return MOE_ERR_INVALID_ARG;
  return cuda_st(cudaMalloc(ptr, bytes));
}

moe_status_t moe_ep_sym_free(void* ptr) { return cuda_st(cudaFree(ptr)); }

moe_status_t moe_ipc_get_handle(void* ptr, uint8_t handle[64]) {
  static_assert(sizeof(cudaIpcMemHandle_t) == 64, "CUDA IPC handles are 64 bytes");
  if (!ptr || !handle) return MOE_ERR_INVALID_ARG;
  cudaIpcMemHandle_t h;
  if (cudaIpcGetMemHandle(&h, ptr) != cudaSuccess) return MOE_ERR_CUDA;
  std::memcpy(handle, &h, sizeof(h));
  return MOE_OK;
}

moe_status_t moe_ipc_open(const uint8_t handle[64], void** ptr) {
  if (!handle || !ptr) return MOE_ERR_INVALID_ARG;
  cudaIpcMemHandle_t h;
  std::memcpy(&h, handle, sizeof(h));
  return cuda_st(cudaIpcOpenMemHandle(ptr, h, cudaIpcMemLazyEnablePeerAccess));
}

moe_status_t moe_ipc_close(void* ptr) {
  if (!ptr) return MOE_ERR_INVALID_ARG;
  return cuda_st(cudaIpcCloseMemHandle(ptr));
}

}  // extern "C"

// Dispatch (scatter of token rows into the expert-grouped buffer) and combine
// (weighted gather-sum back to token order).
//
// Dispatch follows the pplx-kernels page ("Dispatch"): every token row is
// copied to the rows its experts own in the grouped-GEMM input. Combine
// follows its "Combine" section and the EFA page's receiver-side accumulation
// ("Диспетчеризация и комбинирование"): a token's K expert outputs are read
// back and summed with the router weights.
//
// Both are pure HBM streams. Each block strides over token rows (the grid is
// the blocks resident at once, so the PDL dependency wait runs once per
// block); each thread moves 16-byte vectors (8 bf16 or 4 fp32), several per
// iteration so that enough loads are in flight. A dispatched row is read once and written K times;
// a combined row reads its K expert rows and is written once. A shared
// expert adds one row per token to both (its copy of x, its output row).
#include <algorithm>

#include <cuda_bf16.h>

#include "moe_internal.h"
#include "vec_util.cuh"

namespace moe {
namespace {

constexpr int DC_THREADS = 128;
constexpr int DC_UNROLL = 4;

__device__ __forceinline__ uint4 ld_stream(const uint4* p) { return __ldcs(p); }

__global__ void __launch_bounds__(DC_THREADS)
dispatch_kernel(const uint4* __restrict__ x, const int32_t* __restrict__ token_slot,
                uint4* __restrict__ xp, int T, int K, int row_vecs, long long sh_row0,
                int slot_end) {
  __shared__ int s_slot[MAX_K + 1];
  // the shared expert's row of a token is one more destination
  const int KD = sh_row0 >= 0 ? K + 1 : K;
  MOE_CHECK(KD <= MAX_K + 1 && K <= DC_THREADS);
  pdl_wait();
  pdl_trigger();
  for (int t = blockIdx.x; t < T; t += gridDim.x) {
    __syncthreads();   // the previous token's readers of s_slot are done
    bool kept = false;
    if (threadIdx.x < K) {
      int s = token_slot[(size_t)t * K + threadIdx.x];
      if (s >= slot_end) s = -1;   // outside the grouped buffer: treated as dropped
      s_slot[threadIdx.x] = s;
      kept = s >= 0;
    } else if (threadIdx.x == K && KD > K) {
      s_slot[K] = (int)(sh_row0 + t);
      kept = true;
    }
    if (!__syncthreads_or(kept)) continue;   // every assignment overflowed: nothing to copy
    const uint4* src = x + (size_t)t * row_vecs;
    for (int v0 = threadIdx.x; v0 < row_vecs; v0 += DC_THREADS * DC_UNROLL) {
      uint4 d[DC_UNROLL];
#pragma unroll
      for (int u = 0; u < DC_UNROLL; ++u) {
        const int v = v0 + u * DC_THREADS;
        if (v < row_vecs) d[u] = ld_stream(src + v);
      }
      for (int k = 0; k < KD; ++k) {
        const int s = s_slot[k];
        if (s < 0) continue;
        uint4* dst = xp + (size_t)s * row_vecs;
#pragma unroll
        for (int u = 0; u < DC_UNROLL; ++u) {
          const int v = v0 + u * DC_THREADS;
          if (v < row_vecs) dst[v] = d[u];
        }
      }
    }
  }
}

template <bool BF16>
using Acc = float[2][BF16 ? 8 : 4];   // the two 16-byte vectors a thread accumulates

// acc += row (weight 1): the shared expert's term, after the routed ones.
// COHERENT: plain loads, for rows written while the kernel runs.
template <bool BF16, bool COHERENT>
__device__ __forceinline__ void add_row(const uint4* row, int v0, int row_vecs, Acc<BF16>& acc) {
#pragma unroll
  for (int u = 0; u < 2; ++u) {
    const int v = v0 + u * DC_THREADS;
    if (v >= row_vecs) continue;
    const uint4 d = COHERENT ? row[v] : __ldg(row + v);
    if (BF16) {
      float f[8];
      unpack_bf16x8(d, f);
#pragma unroll
      for (int i = 0; i < 8; ++i) acc[u][i] += f[i];
    } else {
      acc[u][0] += __uint_as_float(d.x);
      acc[u][1] += __uint_as_float(d.y);
      acc[u][2] += __uint_as_float(d.z);
      acc[u][3] += __uint_as_float(d.w);
    }
  }
}

// Round the accumulators once to the activation dtype and store them.
template <bool BF16>
__device__ __forceinline__ void store_acc(uint4* dst, int v0, int row_vecs, const Acc<BF16>& acc) {
#pragma unroll
  for (int u = 0; u < 2; ++u) {
    const int v = v0 + u * DC_THREADS;
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

// out[t] = sum_k w[t,k] * y[slot[t,k]] with fp32 accumulation in k order,
// plus y[sh_row0 + t] when sh_row0 >= 0 (the shared expert). Warp 0 first packs
// the token's kept assignments (in k order), so the gather loops over kept rows
// only: with heavy overflow most of a token's K slots are dropped.
template <bool BF16>
__global__ void __launch_bounds__(DC_THREADS)
combine_kernel(const uint4* __restrict__ y, const int32_t* __restrict__ token_slot,
               const float* __restrict__ topk_w, uint4* __restrict__ out, int T, int K,
               int row_vecs, long long sh_row0, int slot_end) {
  __shared__ int s_slot[MAX_K];
  __shared__ float s_w[MAX_K];
  __shared__ int s_n;
  pdl_wait();
  pdl_trigger();
  constexpr int LANES = BF16 ? 8 : 4;
  for (int t = blockIdx.x; t < T; t += gridDim.x) {
    __syncthreads();          // the previous token's readers of s_slot, s_w, s_n are done
    if (threadIdx.x < 32) {   // warp 0 packs the kept assignments, in k order
      int sl = -1;
      float wt = 0.f;
      if ((int)threadIdx.x < K) {
        sl = token_slot[(size_t)t * K + threadIdx.x];
        wt = topk_w[(size_t)t * K + threadIdx.x];
      }
      const bool keep = sl >= 0 && sl < slot_end;   // outside the grouped buffer: dropped
      const unsigned m = __ballot_sync(0xffffffffu, keep);
      if (keep) {
        const int pos = __popc(m & ((1u << threadIdx.x) - 1u));
        s_slot[pos] = sl;
        s_w[pos] = wt;
      }
      if (threadIdx.x == 0) s_n = __popc(m);
    }
    __syncthreads();
    const int n = s_n;   // from here on: the kept rows only
    uint4* dst = out + (size_t)t * row_vecs;
    for (int v0 = threadIdx.x; v0 < row_vecs; v0 += DC_THREADS * 2) {
      Acc<BF16> acc;
#pragma unroll
      for (int u = 0; u < 2; ++u)
#pragma unroll
        for (int i = 0; i < LANES; ++i) acc[u][i] = 0.f;
      // groups of 4 experts: issue the loads, then accumulate in k order
      for (int k = 0; k < n; k += 4) {
        uint4 d[4][2];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const int s = (k + j < n) ? s_slot[k + j] : -1;
#pragma unroll
          for (int u = 0; u < 2; ++u) {
            const int v = v0 + u * DC_THREADS;
            if (s >= 0 && v < row_vecs) d[j][u] = __ldg(y + (size_t)s * row_vecs + v);
            else d[j][u] = make_uint4(0u, 0u, 0u, 0u);
          }
        }
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          if (k + j >= n) continue;
          const float wk = s_w[k + j];
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
      if (sh_row0 >= 0) add_row<BF16, false>(y + (size_t)(sh_row0 + t) * row_vecs, v0, row_vecs, acc);
      store_acc<BF16>(dst, v0, row_vecs, acc);
    }
  }
}

__device__ __forceinline__ uint32_t ld_acquire(const uint32_t* p) {
  uint32_t v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

__device__ __forceinline__ unsigned long long globaltimer() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// The consumer half of the tile-signalled overlap ("Mixture-of-Experts
// acceleration through overlap": tile-ready flags published by the GEMM,
// consumed by a separate kernel as soon as they are set). Same arithmetic as
// combine_kernel, but instead of waiting for the previous kernel to finish, a
// token waits until the ready counter of the 128-row block of each of its
// kept rows has reached `target` (acquire). The wait is bounded: after
// `timeout_ns`, or once any block has given up, the block records
// MOE_ERR_TIMEOUT and leaves its token's output unwritten.
template <bool BF16>
__global__ void __launch_bounds__(DC_THREADS)
combine_wait_kernel(const uint4* __restrict__ y, const int32_t* __restrict__ token_slot,
                    const float* __restrict__ topk_w, uint4* __restrict__ out, int K,
                    int row_vecs, long long sh_row0, int slot_end, const uint32_t* row_ready,
                    uint32_t target,
                    unsigned long long timeout_ns, uint32_t* status) {
  __shared__ int s_slot[MAX_K + 1];
  __shared__ float s_w[MAX_K];
  __shared__ int s_ok, s_n;
  pdl_trigger();   // no griddepcontrol.wait: the ready counters carry the dependency
  const int t = blockIdx.x;
  if (threadIdx.x < 32) {   // warp 0 packs the kept assignments (k order), shared row last
    int sl = -1;
    float wt = 0.f;
    if ((int)threadIdx.x < K) {
      sl = token_slot[(size_t)t * K + threadIdx.x];
      wt = topk_w[(size_t)t * K + threadIdx.x];
    }
    const bool keep = sl >= 0 && sl < slot_end;   // outside the grouped buffer: dropped
    const unsigned m = __ballot_sync(0xffffffffu, keep);
    if (keep) {
      const int pos = __popc(m & ((1u << threadIdx.x) - 1u));
      s_slot[pos] = sl;
      s_w[pos] = wt;
    }
    if (threadIdx.x == 0) {
      s_n = __popc(m);
      if (sh_row0 >= 0) s_slot[s_n] = (int)(sh_row0 + t);
    }
  }
  __syncthreads();
  K = s_n;                                   // from here on: the kept rows only
  const int KW = sh_row0 >= 0 ? K + 1 : K;   // rows to wait for, the shared one last
  if (threadIdx.x == 0) {
    int ok = 1;
    const unsigned long long t0 = globaltimer();
    for (int k = 0; k < KW && ok; ++k) {
      const int sl = s_slot[k];
      if (sl < 0) continue;
      const uint32_t* flag = row_ready + sl / READY_ROWS;
      unsigned sleep_ns = 32;
      while (ld_acquire(flag) < target) {
        if (*(volatile uint32_t*)status != 0u || globaltimer() - t0 > timeout_ns) {
          atomicCAS(status, 0u, (uint32_t)MOE_ERR_TIMEOUT);
          ok = 0;
          break;
        }
        __nanosleep(sleep_ns);
        if (sleep_ns < 2048) sleep_ns *= 2;
      }
    }
    s_ok = ok;
  }
  __syncthreads();
  if (!s_ok) return;
  constexpr int LANES = BF16 ? 8 : 4;
  uint4* dst = out + (size_t)t * row_vecs;
  for (int v0 = threadIdx.x; v0 < row_vecs; v0 += DC_THREADS * 2) {
    Acc<BF16> acc;
#pragma unroll
    for (int u = 0; u < 2; ++u)
#pragma unroll
      for (int i = 0; i < LANES; ++i) acc[u][i] = 0.f;
    for (int k = 0; k < K; k += 4) {
      uint4 d[4][2];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int sl = (k + j < K) ? s_slot[k + j] : -1;
#pragma unroll
        for (int u = 0; u < 2; ++u) {
          const int v = v0 + u * DC_THREADS;
          // coherent loads: these rows were written while this kernel ran
          if (sl >= 0 && v < row_vecs) d[j][u] = y[(size_t)sl * row_vecs + v];
          else d[j][u] = make_uint4(0u, 0u, 0u, 0u);
        }
      }
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        if (k + j >= K || s_slot[k + j] < 0) continue;
        const float wk = s_w[k + j];
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
    if (sh_row0 >= 0) add_row<BF16, true>(y + (size_t)(sh_row0 + t) * row_vecs, v0, row_vecs, acc);
    store_acc<BF16>(dst, v0, row_vecs, acc);
  }
}

}  // namespace

cudaError_t launch_dispatch(const moe_config_t& c, const void* x, const int32_t* slot, void* xp,
                            int64_t sh_row0, cudaStream_t s) {
  if (c.T == 0) return cudaSuccess;
  const int row_vecs = (int)((int64_t)c.H * act_size(c.act_dtype) / 16);
  return launch_pdl(dispatch_kernel, dim3(resident_grid(dispatch_kernel, DC_THREADS, c.T)),
                    dim3(DC_THREADS), 0, s, static_cast<const uint4*>(x), slot,
                    static_cast<uint4*>(xp), c.T, c.K, row_vecs, (long long)sh_row0,
                    (int)routed_rows(c));
}

cudaError_t launch_combine(const moe_config_t& c, const void* y, const int32_t* slot,
                           const float* w, int64_t sh_row0, void* out, cudaStream_t s) {
  if (c.T == 0) return cudaSuccess;
  const int row_vecs = (int)((int64_t)c.H * act_size(c.act_dtype) / 16);
  auto kernel = c.act_dtype == MOE_BF16 ? combine_kernel<true> : combine_kernel<false>;
  return launch_pdl(kernel, dim3(resident_grid(kernel, DC_THREADS, c.T)), dim3(DC_THREADS), 0, s,
                    static_cast<const uint4*>(y), slot, w, static_cast<uint4*>(out), c.T, c.K,
                    row_vecs, (long long)sh_row0, (int)routed_rows(c));
}

cudaError_t launch_combine_wait(const moe_config_t& c, const void* y, const int32_t* slot,
                                const float* w, int64_t sh_row0, const uint32_t* row_ready,
                                uint32_t target, unsigned long long timeout_ns, uint32_t* status,
                                void* out, cudaStream_t s) {
  if (c.T == 0) return cudaSuccess;
  const int row_vecs = (int)((int64_t)c.H * act_size(c.act_dtype) / 16);
  auto kernel = c.act_dtype == MOE_BF16 ? combine_wait_kernel<true> : combine_wait_kernel<false>;
  return launch_pdl(kernel, dim3(c.T), dim3(DC_THREADS), 0, s, static_cast<const uint4*>(y), slot,
                    w, static_cast<uint4*>(out), c.K, row_vecs, (long long)sh_row0,
                    (int)routed_rows(c), row_ready,
                    target, timeout_ns, status);
}

}  // namespace moe

// Route: top-K with softmax weights, the expert histogram, capacity/overflow,
// owner-aligned offsets and the token-order permutation.
//
// "Enabling trillion-parameter models on AWS EFA", "Диспетчеризация и
// комбинирование": the dispatch counts tokens per expert with shared-memory
// atomics inside a block and turns the counts into packing offsets with a
// cumulative sum. Here every block of ROUTE_TB tokens builds a bitmap
// [expert][token-in-block] in shared memory with atomicOr; popcounts of the
// bitmap give both the block's histogram and, for each assignment, its rank
// among the block's earlier tokens of the same expert. A scan over blocks then
// gives each assignment its rank among all earlier tokens of its expert, so
// the permutation is deterministic and in token order (the pplx-kernels page,
// "Dispatch", notes that its own packing order is not).
//
// Three launches, no host synchronisation:
//   route_topk_kernel  one warp per token: K rounds of a warp arg-max over the
//                      token's E logits, softmax over the K winners, bitmap.
//   route_scan_kernel  one block: per-expert scan over blocks, counts,
//                      capacity/overflow ("MoE Expert Parallel Benchmark",
//                      Step 2), aligned exclusive scan over experts, segments.
//   route_slot_kernel  every assignment: slot = off[e] + rank if rank < C,
//                      else -1; row_src back-map; padding rows of row_src = -1.
#include <algorithm>
#include <cfloat>
#include <climits>
#include <cmath>

#include "moe_internal.h"

namespace moe {
namespace {

constexpr int WORDS = ROUTE_TB / 32;   // bitmap words per expert

struct Cand {
  float v;
  int i;   // INT_MAX: no candidate
};

// Total order of the selection: larger logit first, then lower expert index.
__device__ __forceinline__ bool better(const Cand& a, const Cand& b) {
  if (a.i == INT_MAX) return false;
  if (b.i == INT_MAX) return true;
  return a.v > b.v || (a.v == b.v && a.i < b.i);
}

template <int VPL>
__global__ void __launch_bounds__(ROUTE_THREADS)
route_topk_kernel(const float* __restrict__ logits, int T, int E, int K,
                  int32_t* __restrict__ topk_idx, float* __restrict__ topk_w,
                  int32_t* __restrict__ local_rank, int32_t* __restrict__ blk_cnt) {
  extern __shared__ uint32_t smem_u[];
  uint32_t* bitmap = smem_u;                                   // [E][WORDS]
  int32_t* idx_s = reinterpret_cast<int32_t*>(smem_u + E * WORDS);  // [ROUTE_TB][K]

  const int tb0 = blockIdx.x * ROUTE_TB;
  const int ntok = min(ROUTE_TB, T - tb0);
  for (int i = threadIdx.x; i < E * WORDS; i += blockDim.x) bitmap[i] = 0u;
  __syncthreads();

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nwarps = blockDim.x >> 5;
  for (int tl = warp; tl < ntok; tl += nwarps) {
    const int t = tb0 + tl;
    const float* row = logits + (size_t)t * E;
    float v[VPL];
    uint32_t taken = 0u;
#pragma unroll
    for (int j = 0; j < VPL; ++j) {
      const int e = lane + 32 * j;
      if (e < E) {
        v[j] = __ldg(row + e);
      } else {
        v[j] = 0.f;
        taken |= 1u << j;
      }
    }
    float my_v = 0.f, v0 = 0.f;
    int my_i = 0;
    for (int k = 0; k < K; ++k) {
      Cand c{0.f, INT_MAX};
#pragma unroll
      for (int j = 0; j < VPL; ++j) {
        // elements of a lane are visited in increasing index order, so a
        // strict '>' keeps the lowest index among equal logits
        if (!((taken >> j) & 1u) && (c.i == INT_MAX || v[j] > c.v)) {
          c.v = v[j];
          c.i = lane + 32 * j;
        }
      }
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) {
        Cand o;
        o.v = __shfl_xor_sync(0xffffffffu, c.v, off);
        o.i = __shfl_xor_sync(0xffffffffu, c.i, off);
        if (better(o, c)) c = o;
      }
      if (k == 0) v0 = c.v;
      if (lane == k) {
        my_v = c.v;
        my_i = c.i;
      }
      if ((c.i & 31) == lane) taken |= 1u << (c.i >> 5);
    }
    // softmax over the K selected logits, shifted by the largest one
    const float ex = (lane < K) ? expf(my_v - v0) : 0.f;
    float sum = ex;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, off);
    if (lane < K) {
      topk_idx[(size_t)t * K + lane] = my_i;
      topk_w[(size_t)t * K + lane] = ex / sum;
      idx_s[tl * K + lane] = my_i;
      atomicOr(&bitmap[my_i * WORDS + (tl >> 5)], 1u << (tl & 31));
    }
  }
  __syncthreads();

  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    int c = 0;
#pragma unroll
    for (int q = 0; q < WORDS; ++q) c += __popc(bitmap[e * WORDS + q]);
    blk_cnt[(size_t)blockIdx.x * E + e] = c;
  }
  for (int i = threadIdx.x; i < ntok * K; i += blockDim.x) {
    const int tl = i / K;
    const uint32_t* bm = bitmap + idx_s[i] * WORDS;
    const int w = tl >> 5;
    int r = __popc(bm[w] & ((1u << (tl & 31)) - 1u));
    for (int q = 0; q < w; ++q) r += __popc(bm[q]);
    local_rank[(size_t)tb0 * K + i] = r;
  }
}

// Block-wide exclusive scan for blockDim.x == 1024 (32 warps).
__device__ __forceinline__ int block_excl_scan_1024(int v, int* warp_tmp, int& total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int incl = v;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const int o = __shfl_up_sync(0xffffffffu, incl, off);
    if (lane >= off) incl += o;
  }
  if (lane == 31) warp_tmp[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    int w = warp_tmp[lane];
    int wi = w;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int o = __shfl_up_sync(0xffffffffu, wi, off);
      if (lane >= off) wi += o;
    }
    warp_tmp[lane] = wi - w;       // exclusive prefix of warp totals
    if (lane == 31) warp_tmp[32] = wi;
  }
  __syncthreads();
  const int res = warp_tmp[warp] + incl - v;
  total = warp_tmp[32];
  __syncthreads();
  return res;
}

__global__ void __launch_bounds__(1024)
route_scan_kernel(int nblk, int E, int S, int C, int A, int TK, int32_t* __restrict__ blk_cnt,
                  int32_t* __restrict__ counts, int32_t* __restrict__ overflow,
                  int32_t* __restrict__ offsets, int32_t* __restrict__ segoff,
                  int32_t* __restrict__ totals) {
  __shared__ int warp_tmp[33];
  __shared__ int off_s[MAX_E + 1];
  const int e = threadIdx.x;
  int cnt = 0;
  if (e < E) {
    // per-expert exclusive scan over the blocks, in place
#pragma unroll 8
    for (int b = 0; b < nblk; ++b) {
      const size_t p = (size_t)b * E + e;
      const int c = blk_cnt[p];
      blk_cnt[p] = cnt;
      cnt += c;
    }
  }
  const int kept = min(cnt, C);
  const int ov = cnt - kept;
  const int padded = (e < E) ? (kept + A - 1) / A * A : 0;
  int sum_pad, sum_kept, sum_ov;
  const int excl = block_excl_scan_1024(padded, warp_tmp, sum_pad);
  block_excl_scan_1024(e < E ? kept : 0, warp_tmp, sum_kept);
  block_excl_scan_1024(e < E ? ov : 0, warp_tmp, sum_ov);
  if (e < E) {
    counts[e] = cnt;
    overflow[e] = ov;
    offsets[e] = excl;
    off_s[e] = excl;
  }
  if (e == 0) {
    offsets[E] = sum_pad;
    off_s[E] = sum_pad;
    totals[0] = TK;
    totals[1] = sum_kept;
    totals[2] = sum_ov;
    totals[3] = sum_pad;
  }
  __syncthreads();
  const int per = E / S;
  for (int q = e; q <= S; q += blockDim.x) segoff[q] = off_s[q * per];
}

__global__ void __launch_bounds__(256)
route_slot_kernel(int T, int K, int E, int C, int64_t R_max,
                  const int32_t* __restrict__ topk_idx, const int32_t* __restrict__ blk_base,
                  const int32_t* __restrict__ offsets, const int32_t* __restrict__ counts,
                  int32_t* __restrict__ slot, int32_t* __restrict__ row_src) {
  __shared__ int off_s[MAX_E + 1];
  __shared__ int kept_s[MAX_E];
  for (int e = threadIdx.x; e <= E; e += blockDim.x) {
    off_s[e] = offsets[e];
    if (e < E) kept_s[e] = min(counts[e], C);
  }
  __syncthreads();
  const int64_t TK = (int64_t)T * K;
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < TK; i += stride) {
    const int t = (int)(i / K);
    const int e = topk_idx[i];
    const int pos = blk_base[(size_t)(t / ROUTE_TB) * E + e] + slot[i];
    int s = -1;
    if (pos < C) {
      s = off_s[e] + pos;
      row_src[s] = (int32_t)i;
    }
    slot[i] = s;
  }
  // rows no assignment fills: each expert's alignment padding and the tail
  const int R = off_s[E];
  for (int64_t r = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; r < R_max; r += stride) {
    bool pad = true;
    if (r < R) {
      int lo = 0, hi = E;   // largest e with off_s[e] <= r
      while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (off_s[mid] <= r) lo = mid; else hi = mid;
      }
      pad = (r - off_s[lo]) >= kept_s[lo];
    }
    if (pad) row_src[r] = -1;
  }
}

template <int VPL>
void launch_topk(int nblk, size_t smem, cudaStream_t s, const float* logits, int T, int E, int K,
                 int32_t* idx, float* w, int32_t* rank, int32_t* blk) {
  route_topk_kernel<VPL><<<nblk, ROUTE_THREADS, smem, s>>>(logits, T, E, K, idx, w, rank, blk);
}

}  // namespace

cudaError_t launch_route(const moe_config_t& c, const float* logits, int32_t* topk_idx,
                         float* topk_w, int32_t* counts, int32_t* overflow, int32_t* offsets,
                         int32_t* segoff, int32_t* slot, int32_t* row_src, int32_t* totals,
                         int32_t* blk_cnt, int64_t R_max, cudaStream_t s) {
  const int nblk = (int)ceil_div(c.T, ROUTE_TB);
  if (nblk > 0) {
    const size_t smem = (size_t)c.E * WORDS * 4 + (size_t)ROUTE_TB * c.K * 4;
    const int vpl = (int)ceil_div(c.E, 32);
    if (vpl <= 1) launch_topk<1>(nblk, smem, s, logits, c.T, c.E, c.K, topk_idx, topk_w, slot, blk_cnt);
    else if (vpl <= 2) launch_topk<2>(nblk, smem, s, logits, c.T, c.E, c.K, topk_idx, topk_w, slot, blk_cnt);
    else if (vpl <= 4) launch_topk<4>(nblk, smem, s, logits, c.T, c.E, c.K, topk_idx, topk_w, slot, blk_cnt);
    else if (vpl <= 8) launch_topk<8>(nblk, smem, s, logits, c.T, c.E, c.K, topk_idx, topk_w, slot, blk_cnt);
    else if (vpl <= 16) launch_topk<16>(nblk, smem, s, logits, c.T, c.E, c.K, topk_idx, topk_w, slot, blk_cnt);
    else launch_topk<32>(nblk, smem, s, logits, c.T, c.E, c.K, topk_idx, topk_w, slot, blk_cnt);
  }
  route_scan_kernel<<<1, 1024, 0, s>>>(nblk, c.E, c.S, c.capacity, c.row_align, c.T * c.K,
                                       blk_cnt, counts, overflow, offsets, segoff, totals);
  const int64_t work = std::max<int64_t>((int64_t)c.T * c.K, R_max);
  int grid = (int)std::min<int64_t>(std::max<int64_t>(ceil_div(work, 256), 1), 148 * 8);
  route_slot_kernel<<<grid, 256, 0, s>>>(c.T, c.K, c.E, c.capacity, R_max, topk_idx, blk_cnt,
                                         offsets, counts, slot, row_src);
  return cudaGetLastError();
}

}  // namespace moe

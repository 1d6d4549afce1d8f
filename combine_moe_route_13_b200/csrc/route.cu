// Route: top-K with softmax weights, the expert histogram, capacity/overflow,
// owner-aligned offsets and the token-order permutation.
//
// "Enabling trillion-parameter models on AWS EFA", "Диспетчеризация и
// комбинирование": the dispatch counts tokens per expert with shared-memory
// atomics inside a block and turns the counts into packing offsets with a
// cumulative sum. Here every block of tb tokens (32, 64 or 128, by batch
// size) builds a bitmap
// [expert][token-in-block] in shared memory with atomicOr; popcounts of the
// bitmap give both the block's histogram and, for each assignment, its rank
// among the block's earlier tokens of the same expert. A scan over blocks then
// gives each assignment its rank among all earlier tokens of its expert, so
// the permutation is deterministic and in token order (the pplx-kernels page,
// "Dispatch", notes that its own packing order is not).
//
// Three launches, no host synchronisation:
//   route_topk_kernel  one warp per token (4-8 tokens per warp, the next
//                      token's logits loaded while the current one is ranked):
//                      K rounds of a warp arg-max over the token's E logits
//                      (two redux.sync reductions per round on an
//                      order-preserving integer key), softmax over the K
//                      winners, bitmap, per-block counts [E][blocks].
//   route_scan_kernel  one warp per expert: exclusive scan of the expert's
//                      per-block counts (one coalesced row), its total count
//                      and overflow ("MoE Expert Parallel Benchmark", Step 2).
//   route_slot_kernel  every block first scans the aligned kept counts over
//                      the experts (block 0 stores the offsets, segment
//                      offsets and totals); then every assignment gets
//                      slot = off[e] + rank if rank < C, else -1, the row_src
//                      back-map; row_src padding rows get -1 and the shared
//                      expert's rows (if any) T*K + t.
#include <algorithm>
#include <cfloat>
#include <climits>
#include <cmath>

#include "moe_internal.h"

namespace moe {
namespace {

// Order-preserving map of a float to uint32 (larger float -> larger key);
// -0.0 is first folded into +0.0 so that the two compare equal, as floats do.
// Keys of finite values and of -inf are > 0.
__device__ __forceinline__ uint32_t order_key(float v) {
  const uint32_t b = __float_as_uint(v + 0.0f);
  return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}

__device__ __forceinline__ float key_value(uint32_t k) {
  return __uint_as_float((k & 0x80000000u) ? (k & 0x7FFFFFFFu) : ~k);
}

template <int VPL>
__device__ __forceinline__ void load_logits(const float* __restrict__ row, int E, int lane,
                                            float (&v)[VPL]) {
#pragma unroll
  for (int j = 0; j < VPL; ++j) {
    const int e = lane + 32 * j;
    v[j] = (e < E) ? __ldg(row + e) : 0.f;
  }
}

template <int VPL, int THREADS, bool BIAS>
__global__ void __launch_bounds__(THREADS)
route_topk_kernel(const float* __restrict__ logits, const float* __restrict__ sel_bias, int T,
                  int E, int K, int tb, int32_t* __restrict__ topk_idx, float* __restrict__ topk_w,
                  int32_t* __restrict__ local_rank, int32_t* __restrict__ blk_cnt) {
  extern __shared__ uint32_t smem_u[];
  const int WORDS = tb / 32;                                   // bitmap words per expert
  uint32_t* bitmap = smem_u;                                   // [E][WORDS]
  int32_t* idx_s = reinterpret_cast<int32_t*>(smem_u + E * WORDS);  // [tb][K]

  const int tb0 = blockIdx.x * tb;
  const int ntok = min(tb, T - tb0);
  for (int i = threadIdx.x; i < E * WORDS; i += blockDim.x) bitmap[i] = 0u;
  pdl_wait();
  pdl_trigger();
  __syncthreads();

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  constexpr int NWARPS = THREADS / 32;
  uint32_t invalid = 0u;   // bit j: element lane + 32 j does not exist
#pragma unroll
  for (int j = 0; j < VPL; ++j)
    if (lane + 32 * j >= E) invalid |= 1u << j;
  float bias[VPL];   // selection-only bias of this lane's experts
#pragma unroll
  for (int j = 0; j < VPL; ++j) bias[j] = (BIAS && lane + 32 * j < E) ? sel_bias[lane + 32 * j] : 0.f;
  float nxt[VPL];
  if (warp < ntok) load_logits<VPL>(logits + (size_t)(tb0 + warp) * E, E, lane, nxt);
  for (int tl = warp; tl < ntok; tl += NWARPS) {
    const int t = tb0 + tl;
    float v[VPL];
#pragma unroll
    for (int j = 0; j < VPL; ++j) v[j] = nxt[j];
    if (tl + NWARPS < ntok) load_logits<VPL>(logits + (size_t)(t + NWARPS) * E, E, lane, nxt);
    uint32_t taken = invalid;
    uint32_t key[VPL];
#pragma unroll
    for (int j = 0; j < VPL; ++j) key[j] = order_key(BIAS ? v[j] + bias[j] : v[j]);
    float my_v = 0.f, v0 = 0.f;
    int my_i = 0;
    for (int k = 0; k < K; ++k) {
      // this lane's best remaining element: elements are visited in increasing
      // index order, so a strict '>' keeps the lowest index among equal keys
      uint32_t best = 0u;
      int bi = INT_MAX;
#pragma unroll
      for (int j = 0; j < VPL; ++j) {
        if (!((taken >> j) & 1u) && key[j] > best) {
          best = key[j];
          bi = lane + 32 * j;
        }
      }
      // the warp's largest key, then the lowest index holding it
      const uint32_t m = __reduce_max_sync(0xffffffffu, best);
      const int win = __reduce_min_sync(0xffffffffu, best == m ? bi : INT_MAX);
      float wv;
      if (BIAS) {   // the winner's unbiased logit, from the lane that holds it
        float cand = 0.f;
#pragma unroll
        for (int j = 0; j < VPL; ++j)
          if (j == (win >> 5)) cand = v[j];
        wv = __shfl_sync(0xffffffffu, cand, win & 31);
      } else {
        wv = key_value(m);
      }
      if (k == 0) v0 = wv;
      if (lane == k) {
        my_v = wv;
        my_i = win;
      }
      if ((win & 31) == lane) taken |= 1u << (win >> 5);
    }
    // softmax over the K selected logits, shifted by the largest one (the
    // first winner unless a selection bias reordered them)
    if (BIAS)
      v0 = key_value(__reduce_max_sync(0xffffffffu, lane < K ? order_key(my_v) : 0u));
    const float ex = (lane < K) ? expf(my_v - v0) : 0.f;
    float sum = ex;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, off);
    if (lane < K) {
      topk_idx[(size_t)t * K + lane] = my_i;
      topk_w[(size_t)t * K + lane] = ex / sum;
      idx_s[tl * K + lane] = my_i;
      if (MOE_CHECKED(my_i >= 0 && my_i < E && tl < tb))
        atomicOr(&bitmap[my_i * WORDS + (tl >> 5)], 1u << (tl & 31));
    }
  }
  __syncthreads();

  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    int c = 0;
#pragma unroll
    for (int q = 0; q < WORDS; ++q) c += __popc(bitmap[e * WORDS + q]);
    blk_cnt[(size_t)e * gridDim.x + blockIdx.x] = c;
  }
  for (int i = threadIdx.x; i < ntok * K; i += blockDim.x) {
    const int tl = i / K;
    MOE_CHECK(idx_s[i] >= 0 && idx_s[i] < E);
    const uint32_t* bm = bitmap + idx_s[i] * WORDS;
    const int w = tl >> 5;
    int r = __popc(bm[w] & ((1u << (tl & 31)) - 1u));
    for (int q = 0; q < w; ++q) r += __popc(bm[q]);
    local_rank[(size_t)tb0 * K + i] = r;
  }
}

// One warp per expert: exclusive scan, in place, of the expert's per-block
// counts (row e of [E][nblk]), its total count and its overflow. Loads of
// eight 32-block chunks are issued before they are scanned.
__global__ void __launch_bounds__(1024)
route_scan_kernel(int nblk, int E, int C, int32_t* __restrict__ blk_cnt,
                  int32_t* __restrict__ counts, int32_t* __restrict__ overflow) {
  pdl_wait();
  pdl_trigger();
  const int e = blockIdx.x * 32 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (e >= E) return;
  int32_t* row = blk_cnt + (size_t)e * nblk;
  constexpr int G = 8;
  int carry = 0;
  for (int c0 = 0; c0 < nblk; c0 += 32 * G) {
    int v[G];
#pragma unroll
    for (int g = 0; g < G; ++g) {
      const int b = c0 + g * 32 + lane;
      v[g] = (b < nblk) ? row[b] : 0;
    }
#pragma unroll
    for (int g = 0; g < G; ++g) {
      int incl = v[g];
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const int o = __shfl_up_sync(0xffffffffu, incl, off);
        if (lane >= off) incl += o;
      }
      const int b = c0 + g * 32 + lane;
      if (b < nblk) row[b] = carry + incl - v[g];
      carry += __shfl_sync(0xffffffffu, incl, 31);
    }
  }
  if (lane == 0) {
    counts[e] = carry;
    overflow[e] = max(carry - C, 0);
  }
}

// Exclusive scan of the experts' aligned kept counts, done by every block of
// route_slot_kernel into shared memory (E <= 1024, 256 threads, 4 per thread).
__device__ __forceinline__ void expert_offsets_smem(int E, int C, int A,
                                                    const int32_t* __restrict__ counts,
                                                    int* off_s, int* kept_s, int* warp_tmp,
                                                    int& sum_kept) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int e0 = threadIdx.x * 4;
  int pad[4], kp[4], local = 0, lk = 0;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int e = e0 + i;
    kp[i] = (e < E) ? min(counts[e], C) : 0;
    pad[i] = (kp[i] + A - 1) / A * A;
    local += pad[i];
    lk += kp[i];
  }
  int incl = local, inck = lk;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const int o = __shfl_up_sync(0xffffffffu, incl, off);
    const int ok = __shfl_up_sync(0xffffffffu, inck, off);
    if (lane >= off) {
      incl += o;
      inck += ok;
    }
  }
  if (lane == 31) {
    warp_tmp[warp] = incl;
    warp_tmp[8 + warp] = inck;
  }
  __syncthreads();
  int base = 0, tot = 0, totk = 0;
  for (int w = 0; w < 8; ++w) {
    if (w < warp) base += warp_tmp[w];
    tot += warp_tmp[w];
    totk += warp_tmp[8 + w];
  }
  int run = base + incl - local;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int e = e0 + i;
    if (e < E) {
      off_s[e] = run;
      kept_s[e] = kp[i];
    }
    run += pad[i];
  }
  if (threadIdx.x == 0) off_s[E] = tot;
  sum_kept = totk;
  __syncthreads();
}

__global__ void __launch_bounds__(256)
route_slot_kernel(int T, int K, int E, int S, int C, int A, int nblk, int tb, int64_t R_max,
                  int64_t R_sh,
                  const int32_t* __restrict__ topk_idx, const int32_t* __restrict__ blk_base,
                  const int32_t* __restrict__ counts, int32_t* __restrict__ offsets,
                  int32_t* __restrict__ segoff, int32_t* __restrict__ totals,
                  int32_t* __restrict__ slot, int32_t* __restrict__ row_src,
                  uint32_t* __restrict__ row_ready, int64_t n_ready) {
  __shared__ int off_s[MAX_E + 1];
  __shared__ int kept_s[MAX_E];
  __shared__ int warp_tmp[16];
  pdl_wait();
  pdl_trigger();
  int sum_kept;
  expert_offsets_smem(E, C, A, counts, off_s, kept_s, warp_tmp, sum_kept);
  const int64_t TK = (int64_t)T * K;
  if (blockIdx.x == 0) {
    for (int e = threadIdx.x; e <= E; e += blockDim.x) offsets[e] = off_s[e];
    const int per = E / S;
    for (int q = threadIdx.x; q <= S; q += blockDim.x) segoff[q] = off_s[q * per];
    if (threadIdx.x == 0) {
      totals[0] = (int32_t)TK;
      totals[1] = sum_kept;
      totals[2] = (int32_t)TK - sum_kept;
      totals[3] = off_s[E];
    }
  }
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n_ready; i += stride)
    row_ready[i] = 0u;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < TK; i += stride) {
    const int t = (int)(i / K);
    const int e = topk_idx[i];
    const int pos = blk_base[(size_t)e * nblk + t / tb] + slot[i];
    int s = -1;
    if (pos < C) {
      s = off_s[e] + pos;
      row_src[s] = (int32_t)i;
    }
    slot[i] = s;
  }
  // rows no assignment fills: each expert's alignment padding and the tail;
  // from R_sh on, the shared expert's rows (one per token, id T*K + t)
  const int R = off_s[E];
  for (int64_t r = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; r < R_max; r += stride) {
    if (r >= R_sh) {
      row_src[r] = (int32_t)(TK + (r - R_sh));
      continue;
    }
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
cudaError_t launch_topk(int nblk, size_t smem, cudaStream_t s, const float* logits,
                        const float* sel_bias, int T, int E, int K, int tb, int32_t* idx, float* w,
                        int32_t* rank, int32_t* blk) {
  // 32 warps (4 tokens each) while the register budget allows: 16 warps for
  // E > 256, 8 for E > 512
  constexpr int THREADS = VPL >= 32 ? 256 : (VPL >= 16 ? 512 : 1024);
  if (sel_bias)
    return launch_pdl(route_topk_kernel<VPL, THREADS, true>, dim3(nblk), dim3(THREADS), smem, s,
                      logits, sel_bias, T, E, K, tb, idx, w, rank, blk);
  return launch_pdl(route_topk_kernel<VPL, THREADS, false>, dim3(nblk), dim3(THREADS), smem, s,
                    logits, sel_bias, T, E, K, tb, idx, w, rank, blk);
}

}  // namespace

cudaError_t launch_route(const moe_config_t& c, const float* logits, int32_t* topk_idx,
                         float* topk_w, int32_t* counts, int32_t* overflow, int32_t* offsets,
                         int32_t* segoff, int32_t* slot, int32_t* row_src, int32_t* totals,
                         int32_t* blk_cnt, int64_t R_max, cudaStream_t s,
                         uint32_t* row_ready, const float* sel_bias) {
  const int tb = route_tb(c.T);
  const int nblk = (int)route_blocks(c.T);
  const int64_t n_ready = row_ready ? ceil_div(R_max, READY_ROWS) : 0;
  if (nblk > 0) {
    const size_t smem = (size_t)c.E * (tb / 32) * 4 + (size_t)tb * c.K * 4;
    const int vpl = (int)ceil_div(c.E, 32);
    cudaError_t e;
    if (vpl <= 1) e = launch_topk<1>(nblk, smem, s, logits, sel_bias, c.T, c.E, c.K, tb, topk_idx, topk_w, slot, blk_cnt);
    else if (vpl <= 2) e = launch_topk<2>(nblk, smem, s, logits, sel_bias, c.T, c.E, c.K, tb, topk_idx, topk_w, slot, blk_cnt);
    else if (vpl <= 4) e = launch_topk<4>(nblk, smem, s, logits, sel_bias, c.T, c.E, c.K, tb, topk_idx, topk_w, slot, blk_cnt);
    else if (vpl <= 8) e = launch_topk<8>(nblk, smem, s, logits, sel_bias, c.T, c.E, c.K, tb, topk_idx, topk_w, slot, blk_cnt);
    else if (vpl <= 16) e = launch_topk<16>(nblk, smem, s, logits, sel_bias, c.T, c.E, c.K, tb, topk_idx, topk_w, slot, blk_cnt);
    else e = launch_topk<32>(nblk, smem, s, logits, sel_bias, c.T, c.E, c.K, tb, topk_idx, topk_w, slot, blk_cnt);
    if (e != cudaSuccess) return e;
  }
  cudaError_t e = launch_pdl(route_scan_kernel, dim3((unsigned)ceil_div(c.E, 32)), dim3(1024), 0, s,
                             nblk, c.E, c.capacity, blk_cnt, counts, overflow);
  if (e != cudaSuccess) return e;
  const int64_t work = std::max<int64_t>((int64_t)c.T * c.K, R_max);
  int grid = (int)std::min<int64_t>(std::max<int64_t>(ceil_div(work, 256), 1), 148 * 8);
  return launch_pdl(route_slot_kernel, dim3(grid), dim3(256), 0, s, c.T, c.K, c.E, c.S, c.capacity,
                    c.row_align, nblk, tb, R_max, shared_row0(c), (const int32_t*)topk_idx, (const int32_t*)blk_cnt,
                    (const int32_t*)counts, offsets, segoff, totals, slot, row_src, row_ready,
                    n_ready);
}

}  // namespace moe

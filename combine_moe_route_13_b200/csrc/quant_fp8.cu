// fp8 block quantisation: the dispatch with an fp8 payload, and the same
// quantisation of a whole matrix (expert weights, prepared once).
//
// Dispatch with fp8 follows the pplx-kernels page ("Dispatch": token rows are
// sent together with their block scale factors) and the EFA page ("Оценка":
// fp8 with block scaling for the dispatch, bf16 for the combine): the token row
// is read once as bf16, quantised once, and its codes and scales written to
// each of its kept rows.
//
// Blocks of 128 threads stride over the source rows. Thread t handles 16
// consecutive values (two 16-byte vectors of bf16, both loaded before either is
// used); the 8 threads of a warp's eighth cover one 128-element scale block,
// whose amax is a 3-step xor-shuffle reduction, and a warp covers four scale
// blocks: the four scale bytes a row's 512-value chunk owns are adjacent in the
// blocked layout (one UE8M0 byte per 32-k part of the MMA, see fp8_util.cuh),
// so lane 0 gathers them and stores one 4-byte word. Codes leave as 16-byte
// stores (2 KB per block iteration and destination).
#include <algorithm>

#include "fp8_util.cuh"
#include "moe_internal.h"

namespace moe {
namespace {

constexpr int QT = 128;

__device__ __forceinline__ void bf16x8_to_float(const uint4& q, float (&f)[8]) {
  const uint32_t w[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    f[2 * i] = __uint_as_float(w[i] << 16);
    f[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
  }
}

// DISPATCH: destinations are the kept slots of token row `row` (and its
// shared-expert row when sh_row0 >= 0); otherwise the destination is the row
// itself. Blocks stride over the rows (a grid of the blocks resident at once).
template <bool DISPATCH>
__global__ void __launch_bounds__(QT)
quant_rows_kernel(const uint4* __restrict__ src, int64_t rows, int row_vecs, int KB,
                  const int32_t* __restrict__ token_slot, int K, uint8_t* __restrict__ q,
                  uint8_t* __restrict__ sf, int slot_end, long long sh_row0) {
  __shared__ int s_dst[MAX_K + 1];
  __shared__ int s_n;
  pdl_wait();
  pdl_trigger();
  const int64_t H = (int64_t)row_vecs * 8;
  const int lane = threadIdx.x & 31;
  for (int64_t row = blockIdx.x; row < rows; row += gridDim.x) {
    if (DISPATCH) {
      __syncthreads();   // the previous row's readers of s_dst and s_n are done
      if (threadIdx.x < 32) {   // warp 0 packs the kept destinations, k order
        int s = -1;
        if (lane < K) s = token_slot[row * K + lane];
        const bool keep = s >= 0 && s < slot_end;   // others are dropped
        const unsigned m = __ballot_sync(0xffffffffu, keep);
        if (keep) s_dst[__popc(m & ((1u << lane) - 1u))] = s;
        if (lane == 0) {
          int n = __popc(m);
          if (sh_row0 >= 0) s_dst[n++] = (int)(sh_row0 + row);   // the shared expert's row
          s_n = n;
        }
      }
      __syncthreads();
      if (s_n == 0) continue;   // every assignment of this token overflowed
    }
    const int nd = DISPATCH ? s_n : 1;
    const uint4* x = src + row * row_vecs;
    // 16 values (two vectors) per thread, 2048 per block iteration; H is a
    // multiple of 128, so an 8-thread scale block is all valid or all not
    for (int v0 = 0; v0 < row_vecs; v0 += 2 * QT) {
      const int v = v0 + 2 * (int)threadIdx.x;   // this thread's first vector
      const bool valid = v < row_vecs;
      float f[16];
      if (valid) {
        const uint4 a = __ldcs(x + v), b = __ldcs(x + v + 1);
        float fa[8], fb[8];
        bf16x8_to_float(a, fa);
        bf16x8_to_float(b, fb);
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          f[i] = fa[i];
          f[8 + i] = fb[i];
        }
      } else {
#pragma unroll
        for (int i = 0; i < 16; ++i) f[i] = 0.f;
      }
      float amax = 0.f;
#pragma unroll
      for (int i = 0; i < 16; ++i) amax = fmaxf(amax, fabsf(f[i]));
#pragma unroll
      for (int o = 1; o < 8; o <<= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
      const int p = fp8_scale_exp(amax);
      const float inv = fp8_inv_scale(p);
      uint4 c;
      c.x = fp8x2(f[0] * inv, f[1] * inv) | (fp8x2(f[2] * inv, f[3] * inv) << 16);
      c.y = fp8x2(f[4] * inv, f[5] * inv) | (fp8x2(f[6] * inv, f[7] * inv) << 16);
      c.z = fp8x2(f[8] * inv, f[9] * inv) | (fp8x2(f[10] * inv, f[11] * inv) << 16);
      c.w = fp8x2(f[12] * inv, f[13] * inv) | (fp8x2(f[14] * inv, f[15] * inv) << 16);
      // the warp's four scale bytes (scale blocks kb0 .. kb0+3) into one word
      const uint32_t sb = (uint32_t)(p + 127);
      const uint32_t word = __shfl_sync(0xffffffffu, sb, 0) | (__shfl_sync(0xffffffffu, sb, 8) << 8) |
                            (__shfl_sync(0xffffffffu, sb, 16) << 16) |
                            (__shfl_sync(0xffffffffu, sb, 24) << 24);
      const int kb0 = (v - 2 * lane) / 16;   // the warp's first scale block
      for (int d = 0; d < nd; ++d) {
        const int64_t r = DISPATCH ? (int64_t)s_dst[d] : row;
        if (valid) *reinterpret_cast<uint4*>(q + r * H + (int64_t)v * 8) = c;
        // a warp's first scale block is valid whenever any of its lanes is
        if (lane == 0 && kb0 < KB && MOE_CHECKED(kb0 % 4 == 0))
          *reinterpret_cast<uint32_t*>(sf + sf_offset(r, kb0, KB)) = word;
      }
    }
  }
}

}  // namespace

cudaError_t launch_quantize_fp8(const void* src, int64_t rows, int64_t cols, uint8_t* q,
                                uint8_t* sf, cudaStream_t s) {
  if (rows == 0) return cudaSuccess;
  return launch_pdl(quant_rows_kernel<false>,
                    dim3(resident_grid(quant_rows_kernel<false>, QT, rows)), dim3(QT), 0, s,
                    static_cast<const uint4*>(src), rows, (int)(cols / 8),
                    (int)(cols / FP8_BLOCK), (const int32_t*)nullptr, 0, q, sf, 0, -1LL);
}

cudaError_t launch_dispatch_fp8(const moe_config_t& c, const void* x, const int32_t* slot,
                                uint8_t* xq, uint8_t* xs, cudaStream_t s) {
  if (c.T == 0) return cudaSuccess;
  return launch_pdl(quant_rows_kernel<true>,
                    dim3(resident_grid(quant_rows_kernel<true>, QT, c.T)), dim3(QT), 0, s,
                    static_cast<const uint4*>(x), (int64_t)c.T, c.H / 8, c.H / FP8_BLOCK, slot,
                    c.K, xq, xs, (int)routed_rows(c),
                    c.n_shared ? (long long)shared_row0(c) : -1LL);
}

}  // namespace moe

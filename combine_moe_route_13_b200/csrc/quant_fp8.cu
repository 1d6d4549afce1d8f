// fp8 block quantisation: the dispatch with an fp8 payload, and the same
// quantisation of a whole matrix (expert weights, prepared once).
//
// Dispatch with fp8 follows the pplx-kernels page ("Dispatch": token rows are
// sent together with their block scale factors) and the EFA page ("Оценка":
// fp8 with block scaling for the dispatch, bf16 for the combine): the token row
// is read once as bf16, quantised once, and its codes and scales written to
// each of its kept rows.
//
// Blocks of 128 threads stride over the source rows. Thread t handles the 16-byte
// vector v = v0 + t (8 bf16); the 16 threads of a half-warp cover one
// 128-element scale block, whose amax is a 4-step xor-shuffle reduction inside
// the half-warp. Codes leave as 8-byte stores (coalesced, 1 KB per block
// iteration); the half-warp's first thread stores the block's scale byte.
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
  for (int64_t row = blockIdx.x; row < rows; row += gridDim.x) {
    if (DISPATCH) {
      __syncthreads();   // the previous row's readers of s_dst and s_n are done
      if (threadIdx.x == 0) {
        int n = 0;
        for (int k = 0; k < K; ++k) {
          const int s = token_slot[row * K + k];
          if (s >= 0 && s < slot_end) s_dst[n++] = s;   // others are dropped
        }
        if (sh_row0 >= 0) s_dst[n++] = (int)(sh_row0 + row);   // the shared expert's row
        s_n = n;
      }
      __syncthreads();
      if (s_n == 0) continue;   // every assignment of this token overflowed
    }
    const int nd = DISPATCH ? s_n : 1;
    const uint4* x = src + row * row_vecs;
    // row_vecs is a multiple of 16 and v0 of 128: a half-warp is all valid or all not
    for (int v0 = 0; v0 < row_vecs; v0 += QT) {
      const int v = v0 + (int)threadIdx.x;
      const bool valid = v < row_vecs;
      float f[8];
      if (valid) {
        bf16x8_to_float(__ldcs(x + v), f);
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
      for (int d = 0; d < nd; ++d) {
        const int64_t r = DISPATCH ? (int64_t)s_dst[d] : row;
        *reinterpret_cast<uint2*>(q + r * H + (int64_t)v * 8) = c;
        if ((threadIdx.x & 15) == 0) sf[sf_offset(r, kb, KB)] = sbyte;
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

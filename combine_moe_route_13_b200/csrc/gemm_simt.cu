// fp32 grouped SwiGLU expert MLP on CUDA cores (FFMA, fp32 inputs, no TF32).
//
// The grouped GEMM of the pplx-kernels and EFA pages ("MoE all-to-all через
// EFA": the grouped GEMM multiplies the packed tokens with their expert's
// weights) for the fp32 activation dtype. Tensor cores would round fp32
// inputs to TF32, which the fp32 tolerance (1e-5 of the output's maximum)
// does not allow, so this path uses plain FMA.
//
// Each block computes a BM x BN tile of one expert: grid.y enumerates the
// experts' M tiles (an upper bound; surplus blocks exit), grid.x the N tiles.
// A shared expert (sh_rows > 0) is group E: rows [sh_row0, sh_row0 + sh_rows)
// with the weights of expert E.
// GATE_UP: out = silu(A Wg^T) * (A Wu^T) with Wg, Wu the two halves of w_gu[e];
// otherwise out = A W^T.
#include <algorithm>

#include "moe_internal.h"

namespace moe {
namespace {

constexpr int BM = 32, BN = 64, BK = 16, NT = 256;

template <bool GATE_UP>
__global__ void __launch_bounds__(NT)
simt_grouped_gemm(const float* __restrict__ A, int Kdim, const float* __restrict__ W,
                  int w_rows_per_expert, int up_off, int N_out, float* __restrict__ out,
                  const int32_t* __restrict__ offsets, const int32_t* __restrict__ counts, int E,
                  int C, int sh_rows, long long sh_row0) {
  __shared__ int mt_prefix[MAX_E + 2];
  __shared__ float As[BK][BM + 1];
  __shared__ float Bg[BK][BN + 1];
  __shared__ float Bu[GATE_UP ? BK : 1][BN + 1];
  // M tiles of each expert and their prefix (serial: E is small on this path)
  const int G = sh_rows > 0 ? E + 1 : E;   // groups
  if (threadIdx.x == 0) {
    int p = 0;
    for (int e = 0; e < G; ++e) {
      mt_prefix[e] = p;
      p += ((e < E ? min(counts[e], C) : sh_rows) + BM - 1) / BM;
    }
    mt_prefix[G] = p;
  }
  __syncthreads();
  const int mt = blockIdx.y;
  if (mt >= mt_prefix[G]) return;
  int lo = 0, hi = G;     // group e with mt_prefix[e] <= mt < mt_prefix[e+1]
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (mt_prefix[mid] <= mt) lo = mid; else hi = mid;
  }
  const int e = lo;   // experts without tiles never satisfy the strict upper bound
  const int kept = e < E ? min(counts[e], C) : sh_rows;
  const int r0 = (mt - mt_prefix[e]) * BM;          // first row inside the expert
  const int rows = min(BM, kept - r0);
  const int64_t row_base = (e < E ? (int64_t)offsets[e] : (int64_t)sh_row0) + r0;
  const int n0 = blockIdx.x * BN;
  const float* We = W + (int64_t)e * w_rows_per_expert * Kdim;

  const int ty = threadIdx.x / 16, tx = threadIdx.x % 16;   // rows ty*2+{0,1}, cols tx*4+{0..3}
  float accg[2][4] = {}, accu[2][4] = {};
  for (int k0 = 0; k0 < Kdim; k0 += BK) {
    for (int i = threadIdx.x; i < BM * BK; i += NT) {
      const int r = i / BK, kk = i % BK;
      As[kk][r] = (r < rows && k0 + kk < Kdim) ? A[(row_base + r) * Kdim + k0 + kk] : 0.f;
    }
    for (int i = threadIdx.x; i < BN * BK; i += NT) {
      const int n = i / BK, kk = i % BK;
      const bool ok = (n0 + n < N_out) && (k0 + kk < Kdim);
      Bg[kk][n] = ok ? We[(int64_t)(n0 + n) * Kdim + k0 + kk] : 0.f;
      if (GATE_UP) Bu[kk][n] = ok ? We[(int64_t)(up_off + n0 + n) * Kdim + k0 + kk] : 0.f;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < BK; ++kk) {
      const float a0 = As[kk][ty * 2], a1 = As[kk][ty * 2 + 1];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const float bg = Bg[kk][tx * 4 + j];
        accg[0][j] = fmaf(a0, bg, accg[0][j]);
        accg[1][j] = fmaf(a1, bg, accg[1][j]);
        if (GATE_UP) {
          const float bu = Bu[kk][tx * 4 + j];
          accu[0][j] = fmaf(a0, bu, accu[0][j]);
          accu[1][j] = fmaf(a1, bu, accu[1][j]);
        }
      }
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    const int r = ty * 2 + i;
    if (r >= rows) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int n = n0 + tx * 4 + j;
      if (n >= N_out) continue;
      float v;
      if (GATE_UP) {
        const float g = accg[i][j];
        v = g / (1.f + expf(-g)) * accu[i][j];
      } else {
        v = accg[i][j];
      }
      out[(row_base + r) * N_out + n] = v;
    }
  }
}

// Router projection for fp32 activations: one thread per logit, FFMA over H.
__global__ void __launch_bounds__(256)
router_logits_f32(const float* __restrict__ x, const float* __restrict__ w_g,
                  float* __restrict__ logits, int T, int H, int E) {
  pdl_wait();
  pdl_trigger();
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= (int64_t)T * E) return;
  const int t = (int)(i / E), e = (int)(i % E);
  const float* xr = x + (int64_t)t * H;
  const float* wr = w_g + (int64_t)e * H;
  float acc = 0.f;
  for (int h = 0; h < H; ++h) acc = fmaf(xr[h], wr[h], acc);
  logits[i] = acc;
}

}  // namespace

cudaError_t launch_router_f32(const moe_config_t& c, const float* x, const float* w_g,
                              float* logits, cudaStream_t s) {
  const int64_t n = (int64_t)c.T * c.E;
  if (n == 0) return cudaSuccess;
  return launch_pdl(router_logits_f32, dim3((unsigned)ceil_div(n, 256)), dim3(256), 0, s, x, w_g,
                    logits, c.T, c.H, c.E);
}

cudaError_t launch_mlp_f32(const moe_config_t& c, const float* xp, const int32_t* offsets,
                           const int32_t* counts, const float* w_gu, const float* w_d, float* h,
                           float* y, int64_t R_max, cudaStream_t s) {
  const int64_t mt_bound = ceil_div(R_max, BM) + c.E + 1;   // >= sum_e ceil(kept_e / BM)
  const int sh_rows = c.n_shared ? c.T : 0;
  const long long sh_row0 = c.n_shared ? shared_row0(c) : 0;
  if (mt_bound == 0 || mt_bound > 65535) return mt_bound == 0 ? cudaSuccess : cudaErrorInvalidValue;
  dim3 g1((unsigned)ceil_div(c.F, BN), (unsigned)mt_bound);
  simt_grouped_gemm<true><<<g1, NT, 0, s>>>(xp, c.H, w_gu, 2 * c.F, c.F, c.F, h, offsets, counts,
                                            c.E, c.capacity, sh_rows, sh_row0);
  dim3 g2((unsigned)ceil_div(c.H, BN), (unsigned)mt_bound);
  simt_grouped_gemm<false><<<g2, NT, 0, s>>>(h, c.F, w_d, c.H, 0, c.H, y, offsets, counts, c.E,
                                             c.capacity, sh_rows, sh_row0);
  return cudaGetLastError();
}

}  // namespace moe

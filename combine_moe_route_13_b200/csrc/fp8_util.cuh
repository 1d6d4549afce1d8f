// fp8 block scaling shared by the quantising kernels (dispatch, weight
// quantisation, the gate/up GEMM's epilogue).
//
// Format (the fp8 block-scaled payload of "Enabling trillion-parameter models
// on AWS EFA", "Оценка", and the scale factors the pplx-kernels page sends
// beside the tokens, "Dispatch"): e4m3 values; one scale per 128 consecutive
// elements of a row; the scale is a power of two 2^p stored as the byte p + 127
// (UE8M0), p the smallest integer >= -127 with amax <= 448 * 2^p.
//
// Scale bytes live in the layout the block-scaled MMA reads after a
// tcgen05.cp of 32 rows x 16 bytes: for each block of 128 rows and each group
// of four 128-element k blocks a 512-byte chunk; row r's scale for k block kb
// is byte 16*(r%32) + 4*((r%128)/32) + kb%4 of chunk (r/128, kb/4). One chunk
// copy serves four k blocks: the MMA selects the byte with its scale-factor id.
#pragma once

#include <cstdint>

#include <cuda_fp8.h>

namespace moe {

constexpr int FP8_BLOCK = 128;     // elements per scale
constexpr int SF_CHUNK = 512;      // scale bytes of 128 rows x four k blocks

// Byte offset of row r's scale for k block kb (KB k blocks per row).
__host__ __device__ __forceinline__ int64_t sf_offset(int64_t r, int kb, int KB) {
  const int KG = (KB + 3) / 4;
  return ((r / 128) * KG + kb / 4) * SF_CHUNK + 16 * (r % 32) + 4 * ((r % 128) / 32) + kb % 4;
}

// Bytes of scales for a [rows, cols] matrix.
__host__ __device__ __forceinline__ int64_t sf_bytes(int64_t rows, int64_t cols) {
  return ((rows + 127) / 128) * ((cols / FP8_BLOCK + 3) / 4) * SF_CHUNK;
}

#ifdef __CUDACC__
// Smallest p >= -127 with amax <= 448 * 2^p, from the bits of a non-negative
// finite amax: amax = f * 2^x, f in [0.5, 1); 448 = 0.875 * 2^9, so p = x - 9
// when f <= 0.875 (mantissa field <= 0x600000), else x - 8. Zero and
// subnormal amax (below 2^-126) give -127.
__device__ __forceinline__ int fp8_scale_exp(float amax) {
  const uint32_t b = __float_as_uint(amax);
  const int ex = (int)((b >> 23) & 0xFFu);
  if (ex == 0) return -127;
  const int x = ex - 126;
  const int p = (b & 0x7FFFFFu) <= 0x600000u ? x - 9 : x - 8;
  return p < -127 ? -127 : p;
}

// 2^-p as a float, for p in [-127, 126] (always true for a finite fp32 amax).
__device__ __forceinline__ float fp8_inv_scale(int p) {
  return __uint_as_float((uint32_t)(127 - p) << 23);
}

// Two values (already divided by the scale, |v| <= 448) to two e4m3 codes,
// round to nearest even; a in the low byte.
__device__ __forceinline__ uint32_t fp8x2(float a, float b) {
  return (uint32_t)__nv_cvt_float2_to_fp8x2(make_float2(a, b), __NV_SATFINITE, __NV_E4M3);
}
#endif

}  // namespace moe

// 16-byte vector helpers shared by the row-streaming kernels (dispatch,
// combine and their expert-parallel forms).
#pragma once

#include <cstdint>

#include <cuda_bf16.h>

namespace moe {

// Eight bf16 values of a 16-byte vector, widened exactly to fp32.
__device__ __forceinline__ void unpack_bf16x8(const uint4& q, float (&f)[8]) {
  const uint32_t w[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    f[2 * i] = __uint_as_float(w[i] << 16);
    f[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
  }
}

// Two fp32 values rounded to bf16 (nearest even), packed low first.
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  const __nv_bfloat162 b = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&b);
}

}  // namespace moe

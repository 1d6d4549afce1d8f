// Tile scheduling and expert-parallel tile signalling shared by the grouped
// GEMMs (bf16 and fp8): the device-side tile order (with the remote-first
// split of the overlap page's producer, "Mixture-of-Experts acceleration
// through overlap"), the per-sender arrival wait of a tile-signalled owner's
// gate/up producer, and the system-scope release of its ready counters.
#pragma once

#include "moe_internal.h"
#include "tc_ptx.cuh"

namespace moe {
namespace tc {

// Tile t -> (group, m tile, n tile). The tiles come in two sets: first every
// group's M tiles outside [ml0[e], ml0[e] + nl[e]), then those inside (nl = 0
// everywhere puts every tile in the first set). In each set a group owns a
// contiguous range, n-major then m inside; P is the prefix of the groups' M
// tiles and PB the prefix of nl, so the first set's prefix is P - PB.
__device__ __forceinline__ void decode_tile(int tile, int NT, const int* P, const int* PB,
                                            const int* ml0, int G, int& e, int& m, int& n) {
  const int totalA = (P[G] - PB[G]) * NT;
  int lo = 0, hi = G;
  if (tile < totalA) {
    const int g = tile / NT;   // P[lo] - PB[lo] <= g < P[hi] - PB[hi]
    while (hi - lo > 1) {
      const int mid = (lo + hi) >> 1;
      if (P[mid] - PB[mid] <= g) lo = mid; else hi = mid;
    }
    e = lo;
    const int base = P[e] - PB[e];
    const int mt = (P[e + 1] - PB[e + 1]) - base;
    const int local = tile - NT * base;
    n = local / mt;
    const int mm = local - n * mt;
    m = mm < ml0[e] ? mm : mm + (PB[e + 1] - PB[e]);
  } else {
    const int t2 = tile - totalA;
    const int g = t2 / NT;     // PB[lo] <= g < PB[hi]
    while (hi - lo > 1) {
      const int mid = (lo + hi) >> 1;
      if (PB[mid] <= g) lo = mid; else hi = mid;
    }
    e = lo;
    const int nl = PB[e + 1] - PB[e];
    const int local = t2 - NT * PB[e];
    n = local / nl;
    m = ml0[e] + (local - n * nl);
  }
}

__device__ __forceinline__ uint32_t ld_acquire_sys_u32(const uint32_t* p) {
  uint32_t v;
  asm volatile("ld.acquire.sys.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

__device__ __forceinline__ void red_release_add_sys(uint32_t* p, uint32_t v) {
  asm volatile("red.release.sys.global.add.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

// Raise the abort flag of the other CTA of the pair (its shared memory).
__device__ __forceinline__ void abort_peer_cta(uint32_t abort_local, uint32_t peer) {
  asm volatile("st.shared::cluster.u32 [%0], %1;" ::"r"(map_to_rank(abort_local, peer)), "r"(1u)
               : "memory");
}

// Wait until the flag has reached `epoch` (acquire at system scope). Gives up
// when the CTA aborts, when an earlier wait of this step gave up (the status
// word holds MOE_ERR_TIMEOUT), or after limit_ns, recording MOE_ERR_TIMEOUT
// and raising the abort flag.
static __device__ __noinline__ bool wait_arrival(const uint32_t* flag, uint32_t epoch,
                                          volatile int* abort_flag, uint32_t* status,
                                          unsigned long long limit_ns) {
  if ((int32_t)(ld_acquire_sys_u32(flag) - epoch) >= 0) return true;
  const unsigned long long t0 = globaltimer();
  unsigned ns = 64;
  while (true) {
    if (*abort_flag) return false;
    if ((int32_t)(ld_acquire_sys_u32(flag) - epoch) >= 0) return true;
    if (*(volatile uint32_t*)status == (uint32_t)MOE_ERR_TIMEOUT || globaltimer() - t0 > limit_ns) {
      atomicCAS(status, 0u, (uint32_t)MOE_ERR_TIMEOUT);
      *abort_flag = 1;
      return false;
    }
    __nanosleep(ns);
    if (ns < 1024) ns *= 2;
  }
}

}  // namespace tc
}  // namespace moe

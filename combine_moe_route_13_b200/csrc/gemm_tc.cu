// bf16 grouped SwiGLU expert MLP on the sm_100a tensor cores (tcgen05 + TMEM + TMA).
//
// The grouped GEMM between dispatch and combine ("Enabling trillion-parameter
// models on AWS EFA", "MoE all-to-all через EFA"; the DistributedMoE README,
// "Результаты экспериментов": one grouped GEMM instead of many small ones),
// written as a persistent kernel that walks every expert's tiles without a
// relaunch (the producer of "Mixture-of-Experts acceleration through
// overlap"). With the row alignment A = 128 every M tile lies inside one
// expert, hence inside one owner segment (the remote-owner-aligned layout of
// the same page); with any other A a tile starts at its expert's first row and
// rows past the expert's end are computed but never stored.
//
// Two launches:
//   MODE 0: [g | u] = xp W_gu[e]^T  (N = 128 gate + 128 up columns, one MMA of
//           N = 256), epilogue h = silu(g) * u rounded to bf16.
//   MODE 1: y = h W_d[e]^T (N = 256 columns), epilogue rounds to bf16.
//
// Per CTA (one per SM, persistent, static round-robin over tiles):
//   warp 0     TMA producer: A box [128 rows x 64 k] and two B boxes
//              [128 rows x 64 k], 128-byte swizzle, into a 4-stage ring.
//   warp 1     MMA issuer: 4 x tcgen05.mma (M=128, N=256, K=16) per stage,
//              fp32 accumulators in TMEM, two 256-column buffers so that the
//              epilogue of one tile overlaps the MMAs of the next.
//   warps 2-5  epilogue: tcgen05.ld rows from TMEM (each warp owns the 32
//              TMEM lanes of its sub-partition), SwiGLU / rounding, stores.
// Tile order: expert-major, then N tile, then M tile, so that the CTAs running
// at the same time share an expert's rows of xp and each weight slab in L2.
//
// Every wait on an mbarrier is bounded (globaltimer deadline). On expiry the
// kernel records MOE_ERR_TIMEOUT in the status word, all roles leave their
// loops, in-flight copies and MMAs are drained (again with a bound) and TMEM
// is freed before the CTA exits.
#include <algorithm>
#include <mutex>

#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_bf16.h>

#include "moe_internal.h"

namespace moe {
namespace tc {

constexpr int BM = 128;                     // tile rows = TMEM lanes
constexpr int BK = 64;                      // k per stage: one 128-byte swizzle row of bf16
constexpr int UMMA_N = 256;                 // N of one MMA
constexpr int STAGES = 4;
constexpr int A_BYTES = BM * BK * 2;        // 16 KB
constexpr int B_HALF_BYTES = 128 * BK * 2;  // 16 KB
constexpr int STAGE_BYTES = A_BYTES + 2 * B_HALF_BYTES;
constexpr int NUM_THREADS = 192;
constexpr uint32_t TMEM_COLS = 512;
constexpr unsigned long long WAIT_NS = 2000000000ull;   // 2 s
constexpr unsigned long long DRAIN_NS = 200000000ull;   // 0.2 s

// Instruction descriptor of tcgen05.mma.kind::f16: D fp32 (bits 4-5 = 1),
// A bf16 (bits 7-9 = 1), B bf16 (bits 10-12 = 1), both K-major (bits 15, 16 = 0),
// N >> 3 at bits 17-22, M >> 4 at bits 24-28.
constexpr uint32_t IDESC = (1u << 4) | (1u << 7) | (1u << 10) |
                           ((uint32_t)(UMMA_N >> 3) << 17) | ((uint32_t)(BM >> 4) << 24);

struct Ctl {
  uint64_t full[STAGES];
  uint64_t empty[STAGES];
  uint64_t tfull[2];
  uint64_t tempty[2];
  uint64_t drain;
  uint32_t tmem_base;
  int abort;
  int wsum[8];
};

size_t smem_bytes(int E) {
  return 1024 + (size_t)STAGES * STAGE_BYTES + sizeof(Ctl) + (size_t)(3 * E + 1) * 4;
}

// ---------------------------------------------------------------- PTX helpers

__device__ __forceinline__ uint32_t saddr(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

__device__ __forceinline__ void mbar_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
               : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}\n"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0u;
}

__device__ __forceinline__ unsigned long long globaltimer() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// Wait for the phase of `bar` with parity `parity`. Gives up when the CTA's
// abort flag is raised or after `limit_ns`; a timeout raises the flag and
// records MOE_ERR_TIMEOUT.
__device__ __noinline__ bool wait_phase(uint32_t bar, uint32_t parity, volatile int* abort_flag,
                                        uint32_t* status, unsigned long long limit_ns) {
  if (mbar_try_wait(bar, parity)) return true;
  const unsigned long long t0 = globaltimer();
  for (uint32_t it = 1;; ++it) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((it & 31u) == 0u) {
      if (*abort_flag) return false;
      if (globaltimer() - t0 > limit_ns || it > (1u << 30)) {
        *abort_flag = 1;
        atomicCAS(status, 0u, (uint32_t)MOE_ERR_TIMEOUT);
        return false;
      }
    }
  }
}

__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* map, int x, int y,
                                            uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3}], [%4];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(bar)
      : "memory");
}

__device__ __forceinline__ void prefetch_map(const CUtensorMap* map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

__device__ __forceinline__ void tmem_alloc(uint32_t dst, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst),
               "r"(ncols)
               : "memory");
}

__device__ __forceinline__ void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
               : "memory");
}

__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}

__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// Arrive once on `bar` when every tcgen05 operation this thread issued so far
// has completed.
__device__ __forceinline__ void tc_commit(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                   bar)
               : "memory");
}

__device__ __forceinline__ void tc_mma(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                       uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(IDESC), "r"(accumulate)
      : "memory");
}

// 32 consecutive fp32 columns of this thread's TMEM lane.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
      "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]),
        "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]),
        "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
}

__device__ __forceinline__ void tmem_ld_wait() {
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// Shared-memory matrix descriptor for a K-major tile written by TMA with the
// 128-byte swizzle: rows of 128 bytes, 8-row groups 1024 bytes apart (stride
// byte offset), leading byte offset unused (1), descriptor version 1, layout
// type 2 = SWIZZLE_128B. The tile base must be 1024-byte aligned; advancing k
// by 16 bf16 inside the swizzle row adds 32 bytes (2 in the >>4 address field).
__device__ __forceinline__ uint64_t sw128_desc(uint32_t smem_addr) {
  uint64_t d = (uint64_t)((smem_addr >> 4) & 0x3FFFu);
  d |= (uint64_t)1u << 16;
  d |= (uint64_t)(1024u >> 4) << 32;
  d |= (uint64_t)1u << 46;
  d |= (uint64_t)2u << 61;
  return d;
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  const __nv_bfloat162 b = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&b);
}

__device__ __forceinline__ float silu_mul(uint32_t g_bits, uint32_t u_bits) {
  const float g = __uint_as_float(g_bits);
  return g / (1.0f + __expf(-g)) * __uint_as_float(u_bits);
}

// Tile t -> (expert, m tile, n tile). Expert e owns tiles [NT*P[e], NT*P[e+1])
// where P is the prefix of its M-tile counts; inside, n-major then m.
__device__ __forceinline__ void decode_tile(int tile, int NT, const int* P, int E, int& e, int& m,
                                            int& n) {
  const int g = tile / NT;
  int lo = 0, hi = E;   // P[lo] <= g < P[hi]
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (P[mid] <= g) lo = mid; else hi = mid;
  }
  e = lo;
  const int mt = P[e + 1] - P[e];
  const int local = tile - NT * P[e];
  n = local / mt;
  m = local - n * mt;
}

template <int MODE>
__global__ void __launch_bounds__(NUM_THREADS, 1)
tc_grouped_gemm(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                __nv_bfloat16* __restrict__ out, int N_out, int Kdim, int b_rows_per_expert,
                int b_second_off, const int32_t* __restrict__ offsets,
                const int32_t* __restrict__ counts, int E, int C, long long R_max,
                uint32_t* __restrict__ status) {
  constexpr int BN_OUT = (MODE == 0) ? 128 : 256;   // output columns per tile
  constexpr int N_STEP = BN_OUT;                     // weight rows per n tile
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = saddr(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* smem = smem_raw + (base - raw);
  Ctl* ctl = reinterpret_cast<Ctl*>(smem + STAGES * STAGE_BYTES);
  int* P = reinterpret_cast<int*>(ctl + 1);   // [E+1] M-tile prefix
  int* row_off = P + (E + 1);                 // [E]
  int* kept_s = row_off + E;                  // [E]

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int NT = (N_out + BN_OUT - 1) / BN_OUT;
  const int KB = Kdim / BK;
  volatile int* abort_flag = &ctl->abort;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(saddr(&ctl->full[s]), 1);
      mbar_init(saddr(&ctl->empty[s]), 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(saddr(&ctl->tfull[b]), 1);
      mbar_init(saddr(&ctl->tempty[b]), 4);
    }
    mbar_init(saddr(&ctl->drain), 1);
    ctl->abort = 0;
    fence_mbar_init();
    prefetch_map(&tmA);
    prefetch_map(&tmB);
  }
  if (warp == 1) {
    tmem_alloc(saddr(&ctl->tmem_base), TMEM_COLS);
    tmem_relinquish();
  }
  {  // per-expert kept rows, first row and M-tile prefix (block scan)
    const int chunk = (E + NUM_THREADS - 1) / NUM_THREADS;
    const int e0 = threadIdx.x * chunk;
    int local = 0;
    for (int i = 0; i < chunk; ++i) {
      const int e = e0 + i;
      if (e < E) {
        const int k = max(0, min(counts[e], C));
        kept_s[e] = k;
        row_off[e] = offsets[e];
        local += (k + BM - 1) / BM;
      }
    }
    int incl = local;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int o = __shfl_up_sync(0xffffffffu, incl, off);
      if (lane >= off) incl += o;
    }
    if (lane == 31) ctl->wsum[warp] = incl;
    __syncthreads();
    int run = incl - local;
    for (int w = 0; w < warp; ++w) run += ctl->wsum[w];
    for (int i = 0; i < chunk; ++i) {
      const int e = e0 + i;
      if (e < E) {
        P[e] = run;
        run += (kept_s[e] + BM - 1) / BM;
      }
    }
    if (threadIdx.x == NUM_THREADS - 1) P[E] = run;
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = ctl->tmem_base;
  const int total = P[E] * NT;

  if (warp == 0) {
    if (lane == 0) {  // ------------------------------------------------ TMA producer
      int it = 0;
      for (int tile = blockIdx.x; tile < total; tile += gridDim.x) {
        int e, m, n;
        decode_tile(tile, NT, P, E, e, m, n);
        const int a_row = row_off[e] + m * BM;
        const int b_row0 = e * b_rows_per_expert + n * N_STEP;
        const int b_row1 = b_row0 + b_second_off;
        bool ok = true;
        for (int kb = 0; kb < KB; ++kb, ++it) {
          const int s = it % STAGES;
          const uint32_t ph = (uint32_t)(it / STAGES) & 1u;
          if (!wait_phase(saddr(&ctl->empty[s]), ph ^ 1u, abort_flag, status, WAIT_NS)) {
            ok = false;
            break;
          }
          const uint32_t sa = base + s * STAGE_BYTES;
          const uint32_t fb = saddr(&ctl->full[s]);
          mbar_expect_tx(fb, STAGE_BYTES);
          tma_load_2d(sa, &tmA, kb * BK, a_row, fb);
          tma_load_2d(sa + A_BYTES, &tmB, kb * BK, b_row0, fb);
          tma_load_2d(sa + A_BYTES + B_HALF_BYTES, &tmB, kb * BK, b_row1, fb);
        }
        if (!ok) break;
      }
      // the copies of the last STAGES stages must land before the CTA exits
      for (int i = max(0, it - STAGES); i < it; ++i)
        wait_phase(saddr(&ctl->full[i % STAGES]), (uint32_t)(i / STAGES) & 1u, abort_flag, status,
                   DRAIN_NS);
    }
  } else if (warp == 1) {
    if (lane == 0) {  // ------------------------------------------------ MMA issuer
      int it = 0, tcount = 0;
      for (int tile = blockIdx.x; tile < total; tile += gridDim.x, ++tcount) {
        const int b = tcount & 1;
        const uint32_t tph = (uint32_t)(tcount >> 1) & 1u;
        if (!wait_phase(saddr(&ctl->tempty[b]), tph ^ 1u, abort_flag, status, WAIT_NS)) break;
        tc_fence_after();
        const uint32_t d = tmem + (uint32_t)(b * UMMA_N);
        bool ok = true;
        for (int kb = 0; kb < KB; ++kb, ++it) {
          const int s = it % STAGES;
          const uint32_t ph = (uint32_t)(it / STAGES) & 1u;
          if (!wait_phase(saddr(&ctl->full[s]), ph, abort_flag, status, WAIT_NS)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sa = base + s * STAGE_BYTES;
          const uint64_t ad = sw128_desc(sa);
          const uint64_t bd = sw128_desc(sa + A_BYTES);
#pragma unroll
          for (int j = 0; j < BK / 16; ++j)
            tc_mma(d, ad + (uint64_t)(2 * j), bd + (uint64_t)(2 * j), (kb | j) != 0 ? 1u : 0u);
          tc_commit(saddr(&ctl->empty[s]));
        }
        if (!ok) break;
        tc_commit(saddr(&ctl->tfull[b]));
      }
      // every MMA this thread issued must finish before TMEM is released
      tc_commit(saddr(&ctl->drain));
      wait_phase(saddr(&ctl->drain), 0u, abort_flag, status, DRAIN_NS);
    }
  } else {  // -------------------------------------------------------- epilogue
    const int q = warp & 3;                 // TMEM sub-partition of this warp
    const int r_in = q * 32 + lane;         // tile row handled by this thread
    int tcount = 0;
    for (int tile = blockIdx.x; tile < total; tile += gridDim.x, ++tcount) {
      int e, m, n;
      decode_tile(tile, NT, P, E, e, m, n);
      const int rows = min(BM, kept_s[e] - m * BM);
      const long long grow = (long long)row_off[e] + m * BM + r_in;
      const int b = tcount & 1;
      const uint32_t tph = (uint32_t)(tcount >> 1) & 1u;
      int ok = 1;
      if (lane == 0) ok = wait_phase(saddr(&ctl->tfull[b]), tph, abort_flag, status, WAIT_NS);
      __syncwarp();
      ok = __shfl_sync(0xffffffffu, ok, 0);
      if (!ok) break;
      tc_fence_after();
      bool row_ok = r_in < rows;
      if (row_ok && (grow < 0 || grow >= R_max)) {   // inconsistent offsets from the caller
        atomicCAS(status, 0u, (uint32_t)MOE_ERR_DEVICE_INPUT);
        row_ok = false;
      }
      __nv_bfloat16* orow = out + (row_ok ? grow : 0) * (long long)N_out;
      const uint32_t t0 = tmem + ((uint32_t)(q * 32) << 16) + (uint32_t)(b * UMMA_N);
      if (MODE == 0) {
#pragma unroll 1
        for (int c = 0; c < 4; ++c) {
          uint32_t g[32], u[32];
          tmem_ld32(t0 + (uint32_t)(c * 32), g);
          tmem_ld32(t0 + 128u + (uint32_t)(c * 32), u);
          tmem_ld_wait();
          const int col = n * BN_OUT + c * 32;
          if (row_ok && col < N_out) {
            uint4* dst = reinterpret_cast<uint4*>(orow + col);
#pragma unroll
            for (int v = 0; v < 4; ++v) {
              uint4 o;
              o.x = pack_bf16x2(silu_mul(g[8 * v + 0], u[8 * v + 0]), silu_mul(g[8 * v + 1], u[8 * v + 1]));
              o.y = pack_bf16x2(silu_mul(g[8 * v + 2], u[8 * v + 2]), silu_mul(g[8 * v + 3], u[8 * v + 3]));
              o.z = pack_bf16x2(silu_mul(g[8 * v + 4], u[8 * v + 4]), silu_mul(g[8 * v + 5], u[8 * v + 5]));
              o.w = pack_bf16x2(silu_mul(g[8 * v + 6], u[8 * v + 6]), silu_mul(g[8 * v + 7], u[8 * v + 7]));
              dst[v] = o;
            }
          }
        }
      } else {
#pragma unroll 1
        for (int c = 0; c < 8; ++c) {
          uint32_t a[32];
          tmem_ld32(t0 + (uint32_t)(c * 32), a);
          tmem_ld_wait();
          const int col = n * BN_OUT + c * 32;
          if (row_ok && col < N_out) {
            uint4* dst = reinterpret_cast<uint4*>(orow + col);
#pragma unroll
            for (int v = 0; v < 4; ++v) {
              uint4 o;
              o.x = pack_bf16x2(__uint_as_float(a[8 * v + 0]), __uint_as_float(a[8 * v + 1]));
              o.y = pack_bf16x2(__uint_as_float(a[8 * v + 2]), __uint_as_float(a[8 * v + 3]));
              o.z = pack_bf16x2(__uint_as_float(a[8 * v + 4]), __uint_as_float(a[8 * v + 5]));
              o.w = pack_bf16x2(__uint_as_float(a[8 * v + 6]), __uint_as_float(a[8 * v + 7]));
              dst[v] = o;
            }
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(saddr(&ctl->tempty[b]));
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, TMEM_COLS);
  }
}

// ------------------------------------------------------------------ host side

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// 2-D bf16 map over a row-major [rows, cols] matrix, box 64 cols x 128 rows,
// 128-byte swizzle; reads outside the matrix return zeros.
bool make_map(CUtensorMap* map, const void* base, uint64_t cols, uint64_t rows) {
  PFN_cuTensorMapEncodeTiled_v12000 enc = encode_fn();
  if (!enc) return false;
  const cuuint64_t dims[2] = {cols, rows};
  const cuuint64_t strides[1] = {cols * 2};
  const cuuint32_t box[2] = {64, 128};
  const cuuint32_t estr[2] = {1, 1};
  return enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box,
             estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

int sm_count() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 0;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
  return n;
}

}  // namespace tc

moe_status_t launch_mlp_bf16_tc(const moe_config_t& c, const void* xp, const int32_t* offsets,
                                const int32_t* counts, const void* w_gu, const void* w_d,
                                void* h, void* y, int64_t R_max, uint32_t* status,
                                cudaStream_t s) {
  using namespace tc;
  if (R_max == 0) return MOE_OK;
  CUtensorMap mx, mwgu, mh, mwd;
  if (!make_map(&mx, xp, (uint64_t)c.H, (uint64_t)R_max) ||
      !make_map(&mwgu, w_gu, (uint64_t)c.H, (uint64_t)c.E * 2 * c.F) ||
      !make_map(&mh, h, (uint64_t)c.F, (uint64_t)R_max) ||
      !make_map(&mwd, w_d, (uint64_t)c.F, (uint64_t)c.E * c.H))
    return MOE_ERR_CUDA;
  const int sms = sm_count();
  if (sms <= 0) return MOE_ERR_CUDA;
  const size_t smem = smem_bytes(c.E);
  if (cudaFuncSetAttribute(tc_grouped_gemm<0>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)smem) != cudaSuccess ||
      cudaFuncSetAttribute(tc_grouped_gemm<1>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)smem) != cudaSuccess)
    return MOE_ERR_CUDA;
  const int64_t mt_bound = ceil_div(R_max, BM) + c.E;   // >= sum_e ceil(kept_e / BM)
  const int64_t t0 = mt_bound * ceil_div(c.F, 128), t1 = mt_bound * ceil_div(c.H, 256);
  const int g0 = (int)std::min<int64_t>(sms, t0), g1 = (int)std::min<int64_t>(sms, t1);
  tc_grouped_gemm<0><<<g0, NUM_THREADS, smem, s>>>(
      mx, mwgu, static_cast<__nv_bfloat16*>(h), c.F, c.H, 2 * c.F, c.F, offsets, counts, c.E,
      c.capacity, (long long)R_max, status);
  tc_grouped_gemm<1><<<g1, NUM_THREADS, smem, s>>>(
      mh, mwd, static_cast<__nv_bfloat16*>(y), c.H, c.F, c.H, 128, offsets, counts, c.E,
      c.capacity, (long long)R_max, status);
  return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

}  // namespace moe

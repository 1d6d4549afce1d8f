// bf16 grouped SwiGLU expert MLP on the sm_100a tensor cores (tcgen05 + TMEM + TMA).
//
// The grouped GEMM between dispatch and combine ("Enabling trillion-parameter
// models on AWS EFA", "MoE all-to-all через EFA"; the DistributedMoE README,
// "Результаты экспериментов": one grouped GEMM instead of many small ones),
// written as a persistent kernel that walks every expert's tiles without a
// relaunch (the producer of "Mixture-of-Experts acceleration through
// overlap"). With the row alignment A = 128 every 128-row half tile lies inside
// one expert, hence inside one owner segment (the remote-owner-aligned layout
// of the same page); with any other A a tile starts at its expert's first row
// and rows past the expert's end are computed but never stored.
//
// Two launches:
//   MODE 0: [g | u] = xp W_gu[e]^T  (N = 128 gate + 128 up columns, one MMA of
//           N = 256), epilogue h = silu(g) * u rounded to bf16.
//   MODE 1: y = h W_d[e]^T (N = 256 columns), epilogue rounds to bf16.
//
// CG = 2 (used): a cluster of two CTAs on two SMs shares one
// tcgen05.mma.cta_group::2 of M = 256, N = 256. Each CTA loads its own 128 rows
// of A and its own 128 rows (half of N) of B, so a CTA moves 32 KB per k step
// instead of 48 KB and six stages fit in shared memory. Each CTA's TMEM holds
// the 128 x 256 fp32 accumulator of its own rows. CG = 1: one CTA, M = 128,
// both B halves loaded by the CTA, four stages.
//
// Roles per CTA (one CTA per SM, persistent, static round-robin over tiles):
//   warp 0     TMA producer (128-byte swizzled boxes [64 k x 128 rows]);
//   warp 1     MMA issuer (one thread of the cluster's first CTA) and TMEM
//              allocation; two 256-column accumulators so that the epilogue
//              of one tile overlaps the MMAs of the next;
//   warps 2-5  epilogue: tcgen05.ld of its TMEM sub-partition's 32 lanes,
//              SwiGLU / rounding, then a 128 x 64 box staged in shared memory
//              (128-byte swizzle) and written by a TMA store; half tiles that
//              end inside an expert's last rows are stored row by row instead.
// Barriers: the producers of both CTAs signal the leader's "full" barrier;
// the leader's commits signal "empty" and "TMEM full" in both CTAs; both
// CTAs' epilogues signal the leader's "TMEM empty".
// Tile order: expert-major, then N tile, then M tile, so that the clusters
// running at the same time share an expert's rows of xp and each weight slab
// in L2.
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
#include "tc_ptx.cuh"
#include "tile_sched.cuh"

namespace moe {
namespace tc {

constexpr int BM = 128;                     // rows per CTA = TMEM lanes
constexpr int BK = 64;                      // k per stage: one 128-byte swizzle row of bf16
constexpr int UMMA_N = 256;                 // N of one MMA
constexpr int BOX_BYTES = 128 * BK * 2;     // one TMA box: 128 rows x 64 k, 16 KB
constexpr int NUM_THREADS = 192;
constexpr uint32_t TMEM_COLS = 512;
constexpr unsigned long long WAIT_NS = 2000000000ull;   // 2 s
constexpr unsigned long long DRAIN_NS = 200000000ull;   // 0.2 s

template <int CG>
struct Cfg {
  static constexpr int B_BOXES = 3 - CG;                    // B boxes loaded per CTA
  static constexpr int STAGE_BYTES = BOX_BYTES * (1 + B_BOXES);
  static constexpr int STAGES = CG == 2 ? 6 : 4;
  static constexpr int TILE_ROWS = BM * CG;                 // rows per tile (per cluster)
  // Instruction descriptor of tcgen05.mma.kind::f16: D fp32 (bits 4-5 = 1),
  // A bf16 (bits 7-9 = 1), B bf16 (bits 10-12 = 1), both K-major (bits 15,
  // 16 = 0), N >> 3 at bits 17-22, M >> 4 at bits 24-28 (M = 128 per CTA).
  static constexpr uint32_t IDESC = (1u << 4) | (1u << 7) | (1u << 10) |
                                    ((uint32_t)(UMMA_N >> 3) << 17) |
                                    ((uint32_t)((BM * CG) >> 4) << 24);
};

constexpr int MAX_STAGES = 6;

struct Ctl {
  uint64_t full[MAX_STAGES];
  uint64_t empty[MAX_STAGES];
  uint64_t tfull[2];
  uint64_t tempty[2];
  uint64_t drain;
  uint32_t tmem_base;
  int abort;
  int wsum[8];
};

constexpr int STAGING_BYTES = 128 * 64 * 2;   // one 128-row x 64-column bf16 output box

template <int CG>
size_t smem_bytes(int E) {
  return 1024 + (size_t)Cfg<CG>::STAGES * Cfg<CG>::STAGE_BYTES + STAGING_BYTES + sizeof(Ctl) +
         (size_t)(6 * E + 8) * 4;
}

// silu(g) * u = g * u / (1 + exp(-g)), with the fast exponential and the fast
// reciprocal-multiply division (the result is rounded to bf16 next). For very
// negative g the denominator overflows to inf and the quotient is 0, which is
// silu's limit.
__device__ __forceinline__ float silu_mul(uint32_t g_bits, uint32_t u_bits) {
  const float g = __uint_as_float(g_bits);
  return __fdividef(g * __uint_as_float(u_bits), 1.0f + __expf(-g));
}

// Exclusive prefix of `v` over the block's threads (all threads call it);
// wsum: one int per warp of shared memory. Returns the prefix; *total the sum.
__device__ __forceinline__ int block_exclusive(int v, int* wsum, int warp, int lane, int* total) {
  int incl = v;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const int o = __shfl_up_sync(0xffffffffu, incl, off);
    if (lane >= off) incl += o;
  }
  if (lane == 31) wsum[warp] = incl;
  __syncthreads();
  int run = incl - v, tot = 0;
  for (int w = 0; w < NUM_THREADS / 32; ++w) {
    if (w < warp) run += wsum[w];
    tot += wsum[w];
  }
  __syncthreads();   // wsum may be reused
  *total = tot;
  return run;
}

template <int MODE, int CG>
__global__ void __launch_bounds__(NUM_THREADS, 1)
tc_grouped_gemm(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                const __grid_constant__ CUtensorMap tmOut, const __grid_constant__ CUtensorMap tmA2,
                void* __restrict__ out_v, int N_out, int Kdim, int b_rows_per_expert,
                int b_second_off, const int32_t* __restrict__ offsets,
                const int32_t* __restrict__ counts, int E, int C, long long R_max,
                uint32_t* __restrict__ status, uint32_t* __restrict__ row_ready,
                int dense_rows, int sh_rows, int sh_a_row, int sh_out_row, const EpTiles ept) {
  using CF = Cfg<CG>;
  constexpr int STAGES = CF::STAGES;
  constexpr int BN_OUT = (MODE == 0) ? 128 : 256;   // output columns per tile
  __nv_bfloat16* __restrict__ out = static_cast<__nv_bfloat16*>(out_v);
  constexpr int N_STEP = BN_OUT;                     // weight rows per n tile
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = saddr(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* smem = smem_raw + (base - raw);
  const uint32_t staging = base + STAGES * CF::STAGE_BYTES;   // epilogue output box
  Ctl* ctl = reinterpret_cast<Ctl*>(smem + STAGES * CF::STAGE_BYTES + STAGING_BYTES);
  // Groups: the E routed experts, then (sh_rows > 0) the shared expert, whose
  // sh_rows rows are read from tmA2 at row sh_a_row and written at sh_out_row.
  const int G = sh_rows > 0 ? E + 1 : E;
  int* P = reinterpret_cast<int*>(ctl + 1);   // [G+1] M-tile prefix
  int* PB = P + (G + 1);                      // [G+1] prefix of the tiles ordered last
  int* row_off = PB + (G + 1);                // [G+1] first output row of each group, and its end
  int* kept_s = row_off + (G + 1);            // [G]
  int* ml0 = kept_s + G;                      // [G] first M tile ordered last

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = (CG == 2) ? cluster_ctarank() : 0u;   // position in the pair
  const bool leader = rank == 0;
  const int cluster_id = blockIdx.x / CG, n_clusters = gridDim.x / CG;
  const int NT = (N_out + BN_OUT - 1) / BN_OUT;
  const int KB = Kdim / BK;
  volatile int* abort_flag = &ctl->abort;
  // drains wait for copies and MMAs already issued even after an abort (bounded
  // by DRAIN_NS): shared memory and TMEM must not be released under them
  volatile int no_abort = 0;
  // With arrival waits (tile-signalled gate/up) one CTA of a pair may hold its
  // loads back for as long as a sender is late (up to ept.wait_ns), and every
  // other wait of the pair (the leader's MMA on the stage barriers, the
  // epilogues, the leader's final drain of stage barriers that count the peer's
  // copies) must outlast that.
  const bool arrivals = MODE == 0 && ept.arrive != nullptr;
  const unsigned long long wait_ns =
      arrivals ? (ept.wait_ns + DRAIN_NS > WAIT_NS ? ept.wait_ns + DRAIN_NS : WAIT_NS) : WAIT_NS;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(saddr(&ctl->full[s]), 1);
      mbar_init(saddr(&ctl->empty[s]), 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(saddr(&ctl->tfull[b]), 1);
      mbar_init(saddr(&ctl->tempty[b]), 4 * CG);
    }
    mbar_init(saddr(&ctl->drain), 1);
    ctl->abort = 0;
    fence_mbar_init();
    prefetch_map(&tmA);
    prefetch_map(&tmB);
    prefetch_map(&tmOut);
    if (G > E) prefetch_map(&tmA2);
  }
  if (warp == 1) {
    tmem_alloc<CG>(saddr(&ctl->tmem_base), TMEM_COLS);
    tmem_relinquish<CG>();
  }
  pdl_wait();      // everything above touched only this CTA's shared memory and TMEM
  pdl_trigger();
  // this step's number (tile-signalled expert-parallel GEMMs only)
  const uint32_t step = ept.epoch ? ept.epoch
                                  : (ept.counter ? *(volatile const uint32_t*)ept.counter + 1u : 0u);
  {  // per-group kept rows, first row and M-tile prefix (block scans)
    const int chunk = (G + NUM_THREADS - 1) / NUM_THREADS;
    const int e0 = threadIdx.x * chunk;
    int local = 0, localB = 0;
    for (int i = 0; i < chunk; ++i) {
      const int e = e0 + i;
      if (e < G) {
        // dense_rows > 0: one group of dense_rows rows starting at row 0
        int k = dense_rows > 0 ? dense_rows
                : e < E        ? max(0, min(counts[e], C))
                               : sh_rows;
        const int off = dense_rows > 0 ? 0 : (e < E ? offsets[e] : sh_out_row);
        // a caller table whose rows leave the buffer empties the expert
        if (k > 0 && (off < 0 || (long long)off + k > R_max)) {
          atomicCAS(status, 0u, (uint32_t)MOE_ERR_DEVICE_INPUT);
          k = 0;
        }
        kept_s[e] = k;
        row_off[e] = off;
        const int mt = (k + CF::TILE_ROWS - 1) / CF::TILE_ROWS;
        local += mt;
        // remote-first order: the M tiles whose rows are all this owner's own
        // (one contiguous block of the expert's rows) are ordered last
        int first_local = 0, n_local = 0;
        if (ept.remote_first && ept.split != nullptr && e < E && k > 0) {
          const int* sp = ept.split + (size_t)e * (ept.W + 1);
          const int lo = min(max(sp[ept.rank], 0), k), hi = min(max(sp[ept.rank + 1], lo), k);
          const int m_lo = (lo + CF::TILE_ROWS - 1) / CF::TILE_ROWS;
          const int m_hi = hi >= k ? mt : hi / CF::TILE_ROWS;
          if (m_hi > m_lo) {
            first_local = m_lo;
            n_local = m_hi - m_lo;
          }
        }
        ml0[e] = first_local;
        PB[e] = n_local;   // replaced by its prefix below
        localB += n_local;
      }
    }
    int tot = 0, totB = 0;
    int run = block_exclusive(local, ctl->wsum, warp, lane, &tot);
    int runB = block_exclusive(localB, ctl->wsum, warp, lane, &totB);
    for (int i = 0; i < chunk; ++i) {
      const int e = e0 + i;
      if (e < G) {
        P[e] = run;
        run += (kept_s[e] + CF::TILE_ROWS - 1) / CF::TILE_ROWS;
        const int n_local = PB[e];
        PB[e] = runB;
        runB += n_local;
      }
    }
    if (threadIdx.x == NUM_THREADS - 1) {
      P[G] = tot;
      PB[G] = totB;
      row_off[G] = dense_rows > 0 ? dense_rows : (G > E ? sh_out_row + sh_rows : offsets[E]);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (CG == 2) cluster_sync();   // both CTAs' barriers exist before anyone signals them
  tc_fence_after();
  const uint32_t tmem = ctl->tmem_base;
  const int total = P[G] * NT;

  if (warp == 0) {
    if (lane == 0) {  // ------------------------------------------------ TMA producer
      int it = 0;
      uint64_t seen = 0;   // senders whose DISPATCH flag of this step has been seen
      bool ok = true;
      for (int tile = cluster_id; tile < total; tile += n_clusters) {
        int e, m, n;
        decode_tile(tile, NT, P, PB, ml0, G, e, m, n);
        MOE_CHECK(e >= 0 && e < G && n >= 0 && n < NT && m >= 0 &&
                  m * CF::TILE_ROWS < max(kept_s[e], 1));
        const bool shared_group = e >= E;
        const CUtensorMap* mapA = shared_group ? &tmA2 : &tmA;
        const int a_row = (shared_group ? sh_a_row : row_off[e]) + m * CF::TILE_ROWS + (int)rank * BM;
        const int b_row0 = e * b_rows_per_expert + n * N_STEP;
        if (MODE == 0 && ept.arrive != nullptr && !shared_group) {
          // this CTA's rows of the tile: wait for every sender that owns some of them
          const int lo = m * CF::TILE_ROWS + (int)rank * BM;
          const int hi = min(lo + BM, kept_s[e]);
          const int* sp = ept.split + (size_t)e * (ept.W + 1);
          bool waited = false;
          for (int s = 0; s < ept.W && ok && lo < hi; ++s) {
            if ((seen >> s) & 1ull) continue;
            const int a = sp[s], b = sp[s + 1];
            if (b > a && a < hi && b > lo) {
              ok = wait_arrival(ept.arrive + s, step, abort_flag, status, ept.wait_ns);
              seen |= 1ull << s;
              waited = true;
            }
          }
          if (!ok) {
            if (CG == 2) abort_peer_cta(saddr(&ctl->abort), rank ^ 1u);
            break;
          }
          // the rows were written by the peers' generic stores: order the
          // acquire above before this CTA's TMA (async proxy) reads them
          if (waited) fence_proxy_async_global();
        }
        for (int kb = 0; kb < KB; ++kb, ++it) {
          const int s = it % STAGES;
          const uint32_t ph = (uint32_t)(it / STAGES) & 1u;
          if (!wait_phase(saddr(&ctl->empty[s]), ph ^ 1u, abort_flag, status, wait_ns)) {
            ok = false;
            break;
          }
          const uint32_t sa = base + s * CF::STAGE_BYTES;
          MOE_CHECK(s >= 0 && s < STAGES && a_row >= 0);
          const uint32_t fb_local = saddr(&ctl->full[s]);
          const uint32_t fb = (CG == 2) ? map_to_rank(fb_local, 0) : fb_local;
          if (leader) mbar_expect_tx(fb_local, CF::STAGE_BYTES * CG);
          tma_load_2d<CG>(sa, mapA, kb * BK, a_row, fb);
          if (CG == 2) {
            tma_load_2d<CG>(sa + BOX_BYTES, &tmB, kb * BK, b_row0 + (int)rank * b_second_off, fb);
          } else {
            tma_load_2d<CG>(sa + BOX_BYTES, &tmB, kb * BK, b_row0, fb);
            tma_load_2d<CG>(sa + 2 * BOX_BYTES, &tmB, kb * BK, b_row0 + b_second_off, fb);
          }
        }
        if (!ok) break;
      }
      (void)seen;
      // the copies of the last STAGES stages must land before the CTA exits
      // (the leader's barriers also count the peer's copies, which a pair CTA
      // waiting for a late sender issues only then: with arrival waits the
      // drain allows for that, unless the pair has aborted, when only this
      // CTA's own copies, already issued, are left to land)
      if (leader)
        for (int i = max(0, it - STAGES); i < it; ++i) {
          const uint32_t fb = saddr(&ctl->full[i % STAGES]);
          const uint32_t ph = (uint32_t)(i / STAGES) & 1u;
          if (!arrivals || !wait_phase(fb, ph, abort_flag, status, wait_ns))
            wait_phase(fb, ph, &no_abort, status, DRAIN_NS);
        }
    }
  } else if (warp == 1) {
    if (lane == 0 && leader) {  // ---------------------------------------- MMA issuer
      int it = 0, tcount = 0;
      for (int tile = cluster_id; tile < total; tile += n_clusters, ++tcount) {
        const int b = tcount & 1;
        const uint32_t tph = (uint32_t)(tcount >> 1) & 1u;
        if (!wait_phase(saddr(&ctl->tempty[b]), tph ^ 1u, abort_flag, status, wait_ns)) break;
        tc_fence_after();
        MOE_CHECK(b * UMMA_N + UMMA_N <= (int)TMEM_COLS);
        const uint32_t d = tmem + (uint32_t)(b * UMMA_N);
        bool ok = true;
        for (int kb = 0; kb < KB; ++kb, ++it) {
          const int s = it % STAGES;
          const uint32_t ph = (uint32_t)(it / STAGES) & 1u;
          if (!wait_phase(saddr(&ctl->full[s]), ph, abort_flag, status, wait_ns)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sa = base + s * CF::STAGE_BYTES;
          const uint64_t ad = sw128_desc(sa);
          const uint64_t bd = sw128_desc(sa + BOX_BYTES);
#pragma unroll
          for (int j = 0; j < BK / 16; ++j)
            tc_mma<CG>(d, ad + (uint64_t)(2 * j), bd + (uint64_t)(2 * j), CF::IDESC,
                       (kb | j) != 0 ? 1u : 0u);
          tc_commit<CG>(saddr(&ctl->empty[s]));
        }
        if (!ok) break;
        tc_commit<CG>(saddr(&ctl->tfull[b]));
      }
      // every MMA this thread issued must finish before TMEM is released
      tc_commit<CG>(saddr(&ctl->drain));
      wait_phase(saddr(&ctl->drain), 0u, &no_abort, status, DRAIN_NS);
    }
  } else {  // -------------------------------------------------------- epilogue
    const int q = warp & 3;                 // TMEM sub-partition of this warp
    const int r_in = q * 32 + lane;         // row of this CTA's half tile
    const uint32_t tempty0 = saddr(&ctl->tempty[0]);
    const uint32_t tempty_leader0 = (CG == 2) ? map_to_rank(tempty0, 0) : tempty0;
    int tcount = 0;
    for (int tile = cluster_id; tile < total; tile += n_clusters, ++tcount) {
      int e, m, n;
      decode_tile(tile, NT, P, PB, ml0, G, e, m, n);
      MOE_CHECK(e >= 0 && e < G && n >= 0 && n < NT && m >= 0 &&
                m * CF::TILE_ROWS < max(kept_s[e], 1) && r_in < BM);
      const int first = m * CF::TILE_ROWS + (int)rank * BM;   // first row of this half tile
      const int rows = min(BM, kept_s[e] - first);
      const long long grow = (long long)row_off[e] + first + r_in;
      const int b = tcount & 1;
      const uint32_t tph = (uint32_t)(tcount >> 1) & 1u;
      int ok = 1;
      if (lane == 0) ok = wait_phase(saddr(&ctl->tfull[b]), tph, abort_flag, status, wait_ns);
      __syncwarp();
      ok = __shfl_sync(0xffffffffu, ok, 0);
      if (!ok) break;
      tc_fence_after();
      bool row_ok = r_in < rows;
      if (row_ok && (grow < 0 || grow >= R_max)) {   // inconsistent offsets from the caller
        atomicCAS(status, 0u, (uint32_t)MOE_ERR_DEVICE_INPUT);
        row_ok = false;
      }
      // A half tile whose 128 rows all lie inside its expert's row range
      // (alignment padding included, which no reader uses) leaves through a
      // staged TMA store; otherwise each thread stores its own row if valid.
      const long long row0 = (long long)row_off[e] + first;
      const bool staged = MODE != 2 && rows > 0 && row0 >= 0 && row0 + BM <= row_off[e + 1] &&
                          row0 + BM <= R_max;
      __nv_bfloat16* orow = out + (row_ok ? grow : 0) * (long long)N_out;
      const uint32_t t0 = tmem + ((uint32_t)(q * 32) << 16) + (uint32_t)(b * UMMA_N);
      constexpr int CHUNKS = (MODE == 0) ? 2 : 4;   // 64 output columns each
      if (MODE == 2) {   // router logits: fp32 out, any number of columns
        float* lrow = static_cast<float*>(out_v) + (row_ok ? grow : 0) * (long long)N_out;
#pragma unroll 1
        for (int c = 0; c < 4; ++c) {
          uint32_t a[64];
          tmem_ld64(t0 + (uint32_t)(c * 64), a);
          tmem_ld_wait();
          const int col = n * BN_OUT + c * 64;
          if (!row_ok || col >= N_out) continue;
          if (col + 64 <= N_out && (N_out & 3) == 0) {
            float4* dst = reinterpret_cast<float4*>(lrow + col);
#pragma unroll
            for (int v = 0; v < 16; ++v)
              dst[v] = make_float4(__uint_as_float(a[4 * v]), __uint_as_float(a[4 * v + 1]),
                                   __uint_as_float(a[4 * v + 2]), __uint_as_float(a[4 * v + 3]));
          } else {
#pragma unroll
            for (int j = 0; j < 64; ++j)
              if (col + j < N_out) lrow[col + j] = __uint_as_float(a[j]);
          }
        }
      } else
#pragma unroll 1
      for (int c = 0; c < CHUNKS; ++c) {
        uint4 o[8];
        MOE_CHECK(c * 64 + 64 + (MODE == 0 ? 128 : 0) <= UMMA_N);
        if (MODE == 0) {   // gate in TMEM columns [c*64, +64), up in [128 + c*64, +64)
          uint32_t g[64], u[64];
          tmem_ld64(t0 + (uint32_t)(c * 64), g);
          tmem_ld64(t0 + 128u + (uint32_t)(c * 64), u);
          tmem_ld_wait();
#pragma unroll
          for (int v = 0; v < 8; ++v) {
            o[v].x = pack_bf16x2(silu_mul(g[8 * v + 0], u[8 * v + 0]), silu_mul(g[8 * v + 1], u[8 * v + 1]));
            o[v].y = pack_bf16x2(silu_mul(g[8 * v + 2], u[8 * v + 2]), silu_mul(g[8 * v + 3], u[8 * v + 3]));
            o[v].z = pack_bf16x2(silu_mul(g[8 * v + 4], u[8 * v + 4]), silu_mul(g[8 * v + 5], u[8 * v + 5]));
            o[v].w = pack_bf16x2(silu_mul(g[8 * v + 6], u[8 * v + 6]), silu_mul(g[8 * v + 7], u[8 * v + 7]));
          }
        } else {
          uint32_t a[64];
          tmem_ld64(t0 + (uint32_t)(c * 64), a);
          tmem_ld_wait();
#pragma unroll
          for (int v = 0; v < 8; ++v) {
            o[v].x = pack_bf16x2(__uint_as_float(a[8 * v + 0]), __uint_as_float(a[8 * v + 1]));
            o[v].y = pack_bf16x2(__uint_as_float(a[8 * v + 2]), __uint_as_float(a[8 * v + 3]));
            o[v].z = pack_bf16x2(__uint_as_float(a[8 * v + 4]), __uint_as_float(a[8 * v + 5]));
            o[v].w = pack_bf16x2(__uint_as_float(a[8 * v + 6]), __uint_as_float(a[8 * v + 7]));
          }
        }
        const int col = n * BN_OUT + c * 64;
        if (col >= N_out) continue;   // N_out % 64 == 0: a chunk is all in or all out
        if (staged) {
          if (threadIdx.x == 64) bulk_wait_read_all();   // the previous box has left smem
          epilogue_bar();
          MOE_CHECK((r_in + 1) * 128 <= STAGING_BYTES && col + 64 <= N_out);
          // row r_in of the box, 16-byte chunk v at position v ^ (r_in % 8):
          // the 128-byte swizzle the output tensor map uses
#pragma unroll
          for (int v = 0; v < 8; ++v) {
            const uint32_t a = staging + (uint32_t)(r_in * 128 + ((v ^ (r_in & 7)) << 4));
            asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(a), "r"(o[v].x),
                         "r"(o[v].y), "r"(o[v].z), "r"(o[v].w)
                         : "memory");
          }
          fence_proxy_async_smem();
          epilogue_bar();
          if (threadIdx.x == 64) {
            tma_store_2d(&tmOut, col, (int)row0, staging);
            bulk_commit();
          }
        } else if (row_ok) {
          uint4* dst = reinterpret_cast<uint4*>(orow + col);
#pragma unroll
          for (int v = 0; v < 8; ++v) dst[v] = o[v];
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        const uint32_t tb = tempty_leader0 + (uint32_t)(b * sizeof(uint64_t));
        if (CG == 2) mbar_arrive_cluster(tb); else mbar_arrive_local(tb);
      }
      if (MODE == 1 && ept.yready != nullptr && rows > 0) {
        // The same publication at system scope, into this step's bank of the
        // expert-parallel ready counters (read by the peers' combines).
        __threadfence_system();
        if (threadIdx.x == 64) {
          bulk_wait_all();
          fence_proxy_async_global();
        }
        epilogue_bar();
        if (threadIdx.x == 64 && MOE_CHECKED(row0 / READY_ROWS < ept.ready_blocks))
          red_release_add_sys(ept.yready + (size_t)(step & 1u) * ept.ready_blocks +
                                  row0 / READY_ROWS,
                              1u);
      } else if (row_ready != nullptr && rows > 0) {
        // Publish this half tile: its 128 rows (one ready block: the rows are
        // aligned to 128) have one more N tile stored. The staged TMA stores
        // are waited for by their issuing thread and every thread fences its
        // own stores before the barrier; the count is added with release.
        __threadfence();
        if (threadIdx.x == 64) {
          bulk_wait_all();
          fence_proxy_async_global();
        }
        epilogue_bar();
        if (threadIdx.x == 64 && MOE_CHECKED(row0 >= 0 && row0 < R_max))
          red_release_add(row_ready + (row0 / READY_ROWS), 1u);
      }
    }
    if (threadIdx.x == 64) bulk_wait_all();   // staged stores complete before the CTA exits
  }

  tc_fence_before();
  __syncthreads();
  if (CG == 2) cluster_sync();   // no CTA leaves while its peer may still signal it
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc<CG>(tmem, TMEM_COLS);
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

template <int MODE, int CG>
void fill_launch(cudaLaunchConfig_t& cfg, cudaLaunchAttribute* attr, int grid, size_t smem,
                 cudaStream_t s) {
  cfg = cudaLaunchConfig_t{};
  cfg.gridDim = dim3((unsigned)grid);
  cfg.blockDim = dim3(NUM_THREADS);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = CG;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
}

// Co-resident CTAs (CG = 1) or 2-CTA clusters (CG = 2) of tc_grouped_gemm<MODE, CG>
// with `smem` bytes of dynamic shared memory (its attribute must already allow
// that much).
template <int MODE, int CG>
int resident_units(size_t smem) {
  int dev = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    return 0;
  if (CG == 1) return sms;
  cudaLaunchConfig_t q;
  cudaLaunchAttribute attr[2];
  fill_launch<MODE, CG>(q, attr, sms & ~1, smem, nullptr);
  q.numAttrs = 1;   // the cluster shape only
  int clusters = 0;
  if (cudaOccupancyMaxActiveClusters(&clusters, tc_grouped_gemm<MODE, CG>, &q) != cudaSuccess)
    return 0;
  return clusters;
}

template <int CG>
moe_status_t launch_mlp(const moe_config_t& c, const void* xp, const int32_t* offsets,
                        const int32_t* counts, const void* w_gu, const void* w_d, void* h,
                        void* y, int64_t R_max, uint32_t* status, cudaStream_t s,
                        uint32_t* row_ready, const void* x_shared, int modes = 3,
                        const EpTiles& ept = EpTiles{}) {
  const int n_sh = c.n_shared ? 1 : 0;
  const int G = c.E + n_sh;   // routed experts + the shared expert (last in the weights)
  CUtensorMap mx, mwgu, mh, mwd, my, mxs;
  if (!make_map(&mx, xp, (uint64_t)c.H, (uint64_t)R_max) ||
      !make_map(&mwgu, w_gu, (uint64_t)c.H, (uint64_t)G * 2 * c.F) ||
      !make_map(&mh, h, (uint64_t)c.F, (uint64_t)R_max) ||
      !make_map(&mwd, w_d, (uint64_t)c.F, (uint64_t)G * c.H) ||
      !make_map(&my, y, (uint64_t)c.H, (uint64_t)R_max))
    return MOE_ERR_CUDA;
  // The shared expert's gate/up rows: the caller's x, or xp's shared rows.
  const int sh_rows = n_sh ? c.T : 0;
  const int sh_row0 = n_sh ? (int)shared_row0(c) : 0;
  int sh_a_row = sh_row0;
  mxs = mx;
  if (n_sh && x_shared) {
    if (!make_map(&mxs, x_shared, (uint64_t)c.H, (uint64_t)c.T)) return MOE_ERR_CUDA;
    sh_a_row = 0;
  }
  const size_t smem = smem_bytes<CG>(G);
  if (cudaFuncSetAttribute(tc_grouped_gemm<0, CG>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)smem) != cudaSuccess ||
      cudaFuncSetAttribute(tc_grouped_gemm<1, CG>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)smem) != cudaSuccess)
    return MOE_ERR_CUDA;
  const int units = resident_units<0, CG>(smem);
  if (units <= 0) return MOE_ERR_CUDA;
  const int64_t mt_bound = ceil_div(R_max, Cfg<CG>::TILE_ROWS) + G;  // >= sum over groups of M tiles
  const int64_t t0 = mt_bound * ceil_div(c.F, 128), t1 = mt_bound * ceil_div(c.H, 256);
  const int g0 = (int)std::min<int64_t>(units, t0) * CG;
  const int g1 = (int)std::min<int64_t>(units, t1) * CG;
  cudaLaunchConfig_t cfg;
  cudaLaunchAttribute attr[2];
  cudaError_t e = cudaSuccess;
  if (modes & 1) {
    fill_launch<0, CG>(cfg, attr, g0, smem, s);
    e = cudaLaunchKernelEx(&cfg, tc_grouped_gemm<0, CG>, mx, mwgu, mh, mxs, h, c.F, c.H, 2 * c.F,
                           c.F, offsets, counts, c.E, c.capacity, (long long)R_max, status,
                           (uint32_t*)nullptr, 0, sh_rows, sh_a_row, sh_row0, ept);
  }
  if (e == cudaSuccess && (modes & 2)) {
    fill_launch<1, CG>(cfg, attr, g1, smem, s);
    e = cudaLaunchKernelEx(&cfg, tc_grouped_gemm<1, CG>, mh, mwd, my, mh, y, c.H, c.F, c.H, 128,
                           offsets, counts, c.E, c.capacity, (long long)R_max, status, row_ready,
                           0, sh_rows, sh_row0, sh_row0, ept);
  }
  return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

// Router projection as one dense group: logits[T,E] = x[T,H] w_g[E,H]^T.
template <int CG>
moe_status_t launch_router(const moe_config_t& c, const void* x, const void* w_g, float* logits,
                           uint32_t* status, cudaStream_t s) {
  CUtensorMap mx, mg;
  if (!make_map(&mx, x, (uint64_t)c.H, (uint64_t)c.T) ||
      !make_map(&mg, w_g, (uint64_t)c.H, (uint64_t)c.E))
    return MOE_ERR_CUDA;
  const size_t smem = smem_bytes<CG>(1);
  if (cudaFuncSetAttribute(tc_grouped_gemm<2, CG>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)smem) != cudaSuccess)
    return MOE_ERR_CUDA;
  const int units = resident_units<2, CG>(smem);
  if (units <= 0) return MOE_ERR_CUDA;
  const int64_t tiles = ceil_div(c.T, Cfg<CG>::TILE_ROWS) * ceil_div(c.E, 256);
  const int grid = (int)std::min<int64_t>(units, tiles) * CG;
  cudaLaunchConfig_t cfg;
  cudaLaunchAttribute attr[2];
  fill_launch<2, CG>(cfg, attr, grid, smem, s);
  // the output map argument is unused in this mode (fp32 rows are stored directly)
  const cudaError_t e = cudaLaunchKernelEx(
      &cfg, tc_grouped_gemm<2, CG>, mx, mg, mx, mx, (void*)logits, c.E, c.H, 0, 128,
      (const int32_t*)nullptr, (const int32_t*)nullptr, 1, c.T, (long long)c.T, status,
      (uint32_t*)nullptr, c.T, 0, 0, 0, EpTiles{});
  return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

}  // namespace tc

moe_status_t launch_router_logits_tc(const moe_config_t& c, const void* x, const void* w_g,
                                     float* logits, uint32_t* status, cudaStream_t s) {
  if (c.T == 0) return MOE_OK;
  if (c.T >= 256) return tc::launch_router<2>(c, x, w_g, logits, status, s);
  return tc::launch_router<1>(c, x, w_g, logits, status, s);
}

moe_status_t launch_shared_mlp_bf16_tc(const moe_config_t& c, const void* x, const void* w_gu_sh,
                                       const void* w_d_sh, void* h, void* y, uint32_t* status,
                                       cudaStream_t s) {
  if (c.T == 0) return MOE_OK;
  // no routed groups (E = 0): the kernel's only group is the shared one, T rows
  // from row 0 of x, of h and of y, with the weights of expert 0 of w_gu_sh / w_d_sh
  moe_config_t l = c;
  l.E = 0;
  l.K = 1;
  l.S = 1;
  l.capacity = 0;
  l.row_align = 1;
  l.n_shared = 1;
  if (c.T >= 192)
    return tc::launch_mlp<2>(l, x, nullptr, nullptr, w_gu_sh, w_d_sh, h, y, c.T, status, s,
                             nullptr, x);
  return tc::launch_mlp<1>(l, x, nullptr, nullptr, w_gu_sh, w_d_sh, h, y, c.T, status, s, nullptr,
                           x);
}

moe_status_t launch_mlp_bf16_tc_ep(const moe_config_t& c, int modes, const void* xr,
                                   const int32_t* offsets, const int32_t* counts,
                                   const void* w_gu, const void* w_d, void* h, void* y,
                                   int64_t R_max, uint32_t* status, cudaStream_t s,
                                   const EpTiles& t) {
  if (R_max == 0) return MOE_OK;
  moe_config_t l = c;
  l.n_shared = 0;
  const int64_t rows_per_expert = std::min<int64_t>((int64_t)c.T * c.K, (int64_t)c.E * c.capacity) / c.E;
  if (rows_per_expert >= 192)
    return tc::launch_mlp<2>(l, xr, offsets, counts, w_gu, w_d, h, y, R_max, status, s, nullptr,
                             nullptr, modes, t);
  return tc::launch_mlp<1>(l, xr, offsets, counts, w_gu, w_d, h, y, R_max, status, s, nullptr,
                           nullptr, modes, t);
}

moe_status_t launch_mlp_bf16_tc(const moe_config_t& c, const void* xp, const int32_t* offsets,
                                const int32_t* counts, const void* w_gu, const void* w_d,
                                void* h, void* y, int64_t R_max, uint32_t* status,
                                cudaStream_t s, uint32_t* row_ready, const void* x_shared) {
  if (R_max == 0) return MOE_OK;
  // Tile shape from the expected rows per expert: 256-row pair tiles halve each
  // CTA's operand traffic but waste up to 255 padded rows per expert, so small
  // experts (decode-like batches) use 128-row single-CTA tiles.
  const int64_t rows_per_expert = std::min<int64_t>((int64_t)c.T * c.K, (int64_t)c.E * c.capacity) / c.E;
  if (rows_per_expert >= 192)
    return tc::launch_mlp<2>(c, xp, offsets, counts, w_gu, w_d, h, y, R_max, status, s,
                             row_ready, x_shared);
  return tc::launch_mlp<1>(c, xp, offsets, counts, w_gu, w_d, h, y, R_max, status, s, row_ready,
                           x_shared);
}

}  // namespace moe

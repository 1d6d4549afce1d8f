// fp8 block-scaled grouped SwiGLU expert MLP on the sm_100a tensor cores
// (tcgen05.mma kind::mxf8f6f4 with UE8M0 block scales, TMEM, TMA).
//
// The grouped GEMM between dispatch and combine ("Enabling trillion-parameter
// models on AWS EFA", "MoE all-to-all через EFA") fed by the fp8 block-scaled
// dispatch payload of the same page's evaluation ("Оценка"). Both operands are
// e4m3 with one power-of-two scale per 128 k values of a row (see
// fp8_util.cuh); the tensor cores apply the scales themselves, one per 32 k
// values, so the fp32 accumulator holds the exact sum of scaled products.
//
// Two launches, each a persistent grid of one CTA per SM walking the tiles of
// every expert (same tile order as the bf16 kernel: expert, N tile, M tile):
//   MODE 0: [g | u] = xq W_gu[e]^T (M = 128, N = 128 gate + 128 up columns),
//           epilogue h = silu(g) * u, quantised to e4m3 with one scale per
//           128 columns of a row (the tile's columns are exactly one scale
//           block), codes by TMA store, scales to their chunk.
//   MODE 1: y = hq W_d[e]^T (N = 256 columns), epilogue rounds to bf16.
//
// Per stage (128 k values = one 128-byte swizzle row of e4m3): TMA boxes of A
// (128 rows) and B (2 x 128 rows). A scale chunk covers four k blocks, so the
// three chunks of a k group (A, B rows 0-127, B rows 128-255; 512 bytes each,
// by bulk copy) ride with one stage in four: group 0 with the tile's first
// stage, group g > 0 three stages before it is used (with stage 4g - 3). The
// MMA thread moves them into TMEM with tcgen05.cp (32 rows x 16 bytes,
// replicated to the four lane quarters) when they arrive, into one of two
// scale slots, so that a copy's latency overlaps the previous group's MMAs;
// each K = 32 MMA of k block kb reads scale byte kb % 4 (its scale-factor id).
//
// TMEM: the 256-column fp32 accumulator at column 0 (single buffer) and two
// 12-column scale slots from column 256. To overlap one tile's epilogue with
// the next tile's MMAs despite the single accumulator, the epilogue first
// loads its whole row into registers and releases TMEM, then quantises /
// rounds and stores.
//
// Every mbarrier wait is bounded as in the bf16 kernel.
#include <algorithm>

#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_bf16.h>

#include "fp8_util.cuh"
#include "moe_internal.h"
#include "tc_ptx.cuh"
#include "tile_sched.cuh"

namespace moe {
namespace tc {
PFN_cuTensorMapEncodeTiled_v12000 encode_fn();
bool make_map(CUtensorMap* map, const void* base, uint64_t cols, uint64_t rows);
}  // namespace tc

namespace f8 {
using namespace tc;

constexpr int BM = 128;                         // rows per tile = TMEM lanes
constexpr int BK = 128;                         // k per stage (bytes of a swizzle row)
constexpr int UMMA_N = 256;
constexpr int A_BYTES = BM * BK;                // 16 KB
constexpr int B_HALF = 128 * BK;                // 16 KB
constexpr int SF_STAGE = 3 * SF_CHUNK;          // A, B rows 0-127, B rows 128-255
constexpr int MAX_STAGES = 6;
// CG = 1: one CTA per tile of 128 rows, loading A and both halves of B (four
// stages of 48 KB). CG = 2: a pair of CTAs on two SMs shares one
// tcgen05.mma.cta_group::2 of M = 256; each CTA loads its own 128 rows of A
// and its own half of B (32 KB per stage, six stages: half the operand bytes
// per k step and CTA, 1.5x the k steps of lookahead in the same shared
// memory), and the scale chunks of its A rows and of all 256 B rows (every
// CTA's TMEM holds the full B scales, as the one-CTA M = 128 MMA does).
template <int CG>
struct F8 {
  static constexpr int STAGES = CG == 2 ? 6 : 4;
  static constexpr int OPER_BYTES = A_BYTES + (CG == 2 ? 1 : 2) * B_HALF;
  static constexpr int TILE_ROWS = BM * CG;
};
// Threads: warp 0 TMA, warp 1 MMA, then the epilogue warps: eight for gate/up
// (two per TMEM lane quarter, each taking half of the tile's columns, so that
// a thread holds its 64 gate and 64 up accumulators in registers and TMEM is
// released before the SwiGLU and the quantisation run), four for down.
template <int MODE>
__host__ __device__ constexpr int epi_warps() { return MODE == 0 ? 8 : 4; }
template <int MODE>
__host__ __device__ constexpr int num_threads() { return 64 + 32 * epi_warps<MODE>(); }
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t SF_COL0 = 256;
constexpr uint32_t SF_COLS = 12;                // per scale slot: 4 (A) + 8 (B)
constexpr int STAGING_BYTES = 128 * 128;        // one 128-row x 128-byte output box
constexpr unsigned long long WAIT_NS = 2000000000ull;
constexpr unsigned long long DRAIN_NS = 200000000ull;

struct Ctl {
  uint64_t full[MAX_STAGES];
  uint64_t empty[MAX_STAGES];
  uint64_t tfull, tempty, drain;
  uint32_t tmem_base;
  int abort;
  int wsum[16];
  float amax[2][2][128];   // gate/up: [tile parity][column half][row] partial amax of h
};

// Shared memory of a launch over G groups; two_sets: the remote-first tile
// order's tables too (expert-parallel launches only: they would not fit at the
// 512-expert limit of the plain layer).
template <int CG>
size_t smem_bytes(int G, bool two_sets = false) {
  return 1024 + (size_t)F8<CG>::STAGES * (F8<CG>::OPER_BYTES + SF_STAGE) + STAGING_BYTES +
         sizeof(Ctl) + (size_t)(3 * G + 2 + (two_sets ? 2 * G + 1 : 0)) * 4;
}

// Instruction descriptor of tcgen05.mma.kind::mxf8f6f4.block_scale: B scale
// byte j (bits 4-5), A and B e4m3 (format 0 at bits 7-9, 10-12), both
// K-major, N >> 3 at bits 17-22, UE8M0 scales (bit 23), M >> 4 at bits 24-28,
// A scale byte j (bits 29-30), dense K = 32 (bit 31 = 0).
template <int CG>
__host__ __device__ constexpr uint32_t idesc_fp8(uint32_t j) {
  return (j << 4) | ((uint32_t)(UMMA_N >> 3) << 17) | (1u << 23) |
         ((uint32_t)((BM * CG) >> 4) << 24) | (j << 29);
}

// Global -> shared bulk copy (no tensor map), completion counted on `bar`.
__device__ __forceinline__ void bulk_load(uint32_t dst, const void* src, uint32_t bytes,
                                          uint32_t bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::
          "r"(dst),
      "l"(src), "r"(bytes), "r"(bar)
      : "memory");
}

// Shared-memory descriptor of a 32-row x 16-byte scale chunk: no swizzle,
// 8-row core matrices of 128 bytes stacked 128 bytes apart (stride byte
// offset); one core matrix wide, so the leading byte offset is not used.
__device__ __forceinline__ uint64_t sf_desc(uint32_t a) {
  uint64_t d = (uint64_t)((a >> 4) & 0x3FFFu);
  d |= (uint64_t)(128u >> 4) << 16;
  d |= (uint64_t)(128u >> 4) << 32;
  d |= (uint64_t)1u << 46;
  return d;
}

// 32 rows x 128 bits of shared memory into 4 TMEM columns, the same rows in
// each of the four 32-lane quarters. CG = 2 (issued by the pair's first CTA):
// each CTA's chunk at that shared-memory address into its own TMEM.
template <int CG>
__device__ __forceinline__ void sf_copy(uint32_t taddr, uint64_t sdesc) {
  if (CG == 2)
    asm volatile("tcgen05.cp.cta_group::2.32x128b.warpx4 [%0], %1;" ::"r"(taddr), "l"(sdesc)
                 : "memory");
  else
    asm volatile("tcgen05.cp.cta_group::1.32x128b.warpx4 [%0], %1;" ::"r"(taddr), "l"(sdesc)
                 : "memory");
}

template <int CG>
__device__ __forceinline__ void mma_fp8(uint32_t d, uint64_t ad, uint64_t bd, uint32_t idesc,
                                        uint32_t sfa, uint32_t sfb, uint32_t accumulate) {
  if (CG == 2)
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::2.kind::mxf8f6f4.block_scale [%0], %1, %2, %3, [%5], [%6], p;\n\t}\n" ::
            "r"(d),
        "l"(ad), "l"(bd), "r"(idesc), "r"(accumulate), "r"(sfa), "r"(sfb)
        : "memory");
  else
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::mxf8f6f4.block_scale [%0], %1, %2, %3, [%5], [%6], p;\n\t}\n" ::
            "r"(d),
        "l"(ad), "l"(bd), "r"(idesc), "r"(accumulate), "r"(sfa), "r"(sfb)
        : "memory");
}

__device__ __forceinline__ float silu_mul(uint32_t g_bits, uint32_t u_bits) {
  const float g = __uint_as_float(g_bits);
  return __fdividef(g * __uint_as_float(u_bits), 1.0f + __expf(-g));
}

// The k group whose scales ride with stage kb, or -1.
__device__ __forceinline__ int sf_group_of_stage(int kb, int KG) {
  if (kb == 0) return 0;
  if ((kb & 3) == 1 && (kb >> 2) + 1 < KG) return (kb >> 2) + 1;
  return -1;
}

// Tile -> (group, m tile, n tile), one set: group e owns tiles
// [NT*P[e], NT*P[e+1]), n-major then m.
__device__ __forceinline__ int decode_tile1(int tile, int NT, const int* P, int E, int& m, int& n) {
  const int g = tile / NT;
  int lo = 0, hi = E;
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (P[mid] <= g) lo = mid; else hi = mid;
  }
  const int mt = P[lo + 1] - P[lo];
  const int local = tile - NT * P[lo];
  n = local / mt;
  m = local - n * mt;
  return lo;
}

// Either order: with the remote-first tables (PB, ml0) the two-set order of
// the tile-signalled expert-parallel layer, else one set.
__device__ __forceinline__ int tile_of(int tile, int NT, const int* P, const int* PB,
                                       const int* ml0, int G, int& m, int& n) {
  if (PB == nullptr) return decode_tile1(tile, NT, P, G, m, n);
  int e;
  decode_tile(tile, NT, P, PB, ml0, G, e, m, n);
  return e;
}

// Write one 128-byte row of the output box into the staging buffer at the
// position the 128-byte swizzle of the output tensor map expects.
__device__ __forceinline__ void stage_row(uint32_t staging, int r, const uint4 (&o)[8]) {
#pragma unroll
  for (int v = 0; v < 8; ++v) {
    const uint32_t a = staging + (uint32_t)(r * 128 + ((v ^ (r & 7)) << 4));
    asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(a), "r"(o[v].x), "r"(o[v].y),
                 "r"(o[v].z), "r"(o[v].w)
                 : "memory");
  }
}

// Named barrier of the epilogue warps.
template <int MODE>
__device__ __forceinline__ void epi_bar() {
  asm volatile("bar.sync 1, %0;" ::"n"(32 * epi_warps<MODE>()) : "memory");
}

// Scale chunks (512 bytes: 128 rows x four k blocks) by tensor map (CG = 2):
// the scale buffer seen as [chunks][128] uint32, one chunk per box, so that
// both CTAs' copies count on the pair's first CTA's barrier like the
// operands (tmSFA, tmSFB); CG = 1 uses plain bulk copies from sfa / sfb.
template <int MODE, int CG>
__global__ void __launch_bounds__(num_threads<MODE>(), 1)
fp8_grouped_gemm(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                 const __grid_constant__ CUtensorMap tmOut, const __grid_constant__ CUtensorMap tmSFA,
                 const __grid_constant__ CUtensorMap tmSFB, const uint8_t* __restrict__ sfa,
                 const uint8_t* __restrict__ sfb, void* __restrict__ out_v,
                 uint8_t* __restrict__ out_sf, int N_out, int Kdim, int b_rows_per_expert,
                 int b_second_off, const int32_t* __restrict__ offsets,
                 const int32_t* __restrict__ counts, int E, int C, long long R_max,
                 uint32_t* __restrict__ status, int sh_rows, int sh_row0, const EpTiles ept) {
  using CF = F8<CG>;
  constexpr int STAGES = CF::STAGES;
  constexpr int OPER_BYTES = CF::OPER_BYTES;
  constexpr int BN_OUT = (MODE == 0) ? 128 : 256;   // output columns per tile
  constexpr int NUM_THREADS = num_threads<MODE>();
  constexpr int EPI_WARPS = epi_warps<MODE>();
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = saddr(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* smem = smem_raw + (base - raw);
  const uint32_t sf_smem = base + STAGES * OPER_BYTES;          // scale chunks of each stage
  const uint32_t staging = sf_smem + STAGES * SF_STAGE;         // 1024-aligned
  Ctl* ctl = reinterpret_cast<Ctl*>(smem + (staging - base) + STAGING_BYTES);
  // Groups: the E routed experts, then (sh_rows > 0) the shared expert: its
  // sh_rows rows start at sh_row0 and its weights are expert E's.
  const int G = sh_rows > 0 ? E + 1 : E;
  int* P = reinterpret_cast<int*>(ctl + 1);   // [G+1] M-tile prefix
  int* row_off = P + (G + 1);                 // [G+1] first row of each group, and its end
  int* kept_s = row_off + (G + 1);            // [G]
  // remote-first order (tile-signalled expert-parallel gate/up and down)
  const bool two_sets = ept.remote_first != 0 && ept.split != nullptr;
  int* PB = two_sets ? kept_s + G : nullptr;  // [G+1] prefix of the M tiles ordered last
  int* ml0 = two_sets ? PB + (G + 1) : nullptr;   // [G] first M tile ordered last

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = (CG == 2) ? cluster_ctarank() : 0u;   // position in the pair
  const bool leader = rank == 0;
  const int cta_group = blockIdx.x / CG, n_groups = gridDim.x / CG;
  const int NT = (N_out + BN_OUT - 1) / BN_OUT;
  const int KB = Kdim / BK;
  const int KG = (KB + 3) / 4;   // k groups (scale chunks per row block)
  volatile int* abort_flag = &ctl->abort;
  // drains wait for copies and MMAs already issued even after an abort (bounded
  // by DRAIN_NS): shared memory and TMEM must not be released under them
  volatile int no_abort = 0;
  // With arrival waits (tile-signalled gate/up) one CTA of a pair may hold its
  // loads back for as long as a sender is late (up to ept.wait_ns), and every
  // other wait of the pair must outlast that.
  const bool arrivals = MODE == 0 && ept.arrive != nullptr;
  const unsigned long long wait_ns =
      arrivals ? (ept.wait_ns + DRAIN_NS > WAIT_NS ? ept.wait_ns + DRAIN_NS : WAIT_NS) : WAIT_NS;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(saddr(&ctl->full[s]), 1);
      mbar_init(saddr(&ctl->empty[s]), 1);
    }
    mbar_init(saddr(&ctl->tfull), 1);
    mbar_init(saddr(&ctl->tempty), EPI_WARPS * CG);   // both CTAs' epilogues (on the first)
    mbar_init(saddr(&ctl->drain), 1);
    ctl->abort = 0;
    fence_mbar_init();
    prefetch_map(&tmA);
    prefetch_map(&tmB);
    prefetch_map(&tmOut);
    if (CG == 2) {
      prefetch_map(&tmSFA);
      prefetch_map(&tmSFB);
    }
  }
  if (warp == 1) {
    tmem_alloc<CG>(saddr(&ctl->tmem_base), TMEM_COLS);
    tmem_relinquish<CG>();
  }
  pdl_wait();
  pdl_trigger();
  // this step's number (tile-signalled expert-parallel GEMMs only)
  const uint32_t step = ept.epoch ? ept.epoch
                                  : (ept.counter ? *(volatile const uint32_t*)ept.counter + 1u : 0u);
  {  // per-group kept rows, first row and M-tile prefixes (block scans)
    const int chunk = (G + NUM_THREADS - 1) / NUM_THREADS;
    const int e0 = threadIdx.x * chunk;
    int local = 0, localB = 0;
    for (int i = 0; i < chunk; ++i) {
      const int e = e0 + i;
      if (e < G) {
        int k = e < E ? max(0, min(counts[e], C)) : sh_rows;
        const int off = e < E ? offsets[e] : sh_row0;
        // a caller table whose rows leave the buffer or start off a 128-row
        // block (the scale chunks are per 128 rows) empties the expert
        if (k > 0 && (off < 0 || (off & 127) != 0 || (long long)off + k > R_max)) {
          atomicCAS(status, 0u, (uint32_t)MOE_ERR_DEVICE_INPUT);
          k = 0;
        }
        kept_s[e] = k;
        row_off[e] = off;
        const int mt = (k + CF::TILE_ROWS - 1) / CF::TILE_ROWS;
        local += mt;
        if (two_sets) {
          // remote-first order: the M tiles whose rows are all this owner's
          // own (one contiguous block of the expert's rows) are ordered last
          int first_local = 0, n_local = 0;
          if (e < E && k > 0) {
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
    }
    // exclusive block prefix of v (all threads); *tot: the block's sum
    auto block_prefix = [&](int v, int* tot) {
      int incl = v;
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const int o = __shfl_up_sync(0xffffffffu, incl, off);
        if (lane >= off) incl += o;
      }
      if (lane == 31) ctl->wsum[warp] = incl;
      __syncthreads();
      int run = incl - v, t = 0;
      for (int w = 0; w < NUM_THREADS / 32; ++w) {
        if (w < warp) run += ctl->wsum[w];
        t += ctl->wsum[w];
      }
      __syncthreads();   // wsum is reused
      *tot = t;
      return run;
    };
    int tot = 0, totB = 0;
    int run = block_prefix(local, &tot);
    int runB = two_sets ? block_prefix(localB, &totB) : 0;
    for (int i = 0; i < chunk; ++i) {
      const int e = e0 + i;
      if (e < G) {
        P[e] = run;
        run += (kept_s[e] + CF::TILE_ROWS - 1) / CF::TILE_ROWS;
        if (two_sets) {
          const int n_local = PB[e];
          PB[e] = runB;
          runB += n_local;
        }
      }
    }
    if (threadIdx.x == NUM_THREADS - 1) {
      P[G] = tot;
      if (two_sets) PB[G] = totB;
      row_off[G] = G > E ? sh_row0 + sh_rows : offsets[E];
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
      for (int tile = cta_group; tile < total; tile += n_groups) {
        int m, n;
        const int e = tile_of(tile, NT, P, PB, ml0, G, m, n);
        MOE_CHECK(e >= 0 && e < G && n >= 0 && n < NT && m >= 0 &&
                  m * CF::TILE_ROWS < max(kept_s[e], 1));
        // this CTA's 128 rows of A (a multiple of 128)
        const int a_row = row_off[e] + m * CF::TILE_ROWS + (int)rank * BM;
        const int b_row0 = e * b_rows_per_expert + n * BN_OUT;
        const uint8_t* sa_rows = sfa + (size_t)(a_row / 128) * KG * SF_CHUNK;
        const uint8_t* sb0_rows = sfb + (size_t)(b_row0 / 128) * KG * SF_CHUNK;
        const uint8_t* sb1_rows = sfb + (size_t)((b_row0 + b_second_off) / 128) * KG * SF_CHUNK;
        bool ok = true;
        if (arrivals && e < E) {
          // this CTA's rows of the tile (codes and their scale chunk): wait for
          // every sender that owns some of them
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
          const uint32_t sa = base + s * OPER_BYTES;
          const uint32_t ss = sf_smem + s * SF_STAGE;
          const uint32_t fb_local = saddr(&ctl->full[s]);
          // the pair's copies all count on the first CTA's barrier
          const uint32_t fb = (CG == 2) ? map_to_rank(fb_local, 0) : fb_local;
          const int sg = sf_group_of_stage(kb, KG);
          if (leader) mbar_expect_tx(fb_local, (OPER_BYTES + (sg >= 0 ? SF_STAGE : 0)) * CG);
          MOE_CHECK(s >= 0 && s < STAGES && a_row >= 0);
          tma_load_2d<CG>(sa, &tmA, kb * BK, a_row, fb);
          if (CG == 2) {   // this CTA's half of B: gate rows or up rows (gate/up), 128 rows (down)
            tma_load_2d<CG>(sa + A_BYTES, &tmB, kb * BK, b_row0 + (int)rank * b_second_off, fb);
            if (sg >= 0) {
              tma_load_2d<CG>(ss, &tmSFA, 0, (a_row / 128) * KG + sg, fb);
              tma_load_2d<CG>(ss + SF_CHUNK, &tmSFB, 0, (b_row0 / 128) * KG + sg, fb);
              tma_load_2d<CG>(ss + 2 * SF_CHUNK, &tmSFB, 0,
                              ((b_row0 + b_second_off) / 128) * KG + sg, fb);
            }
          } else {
            tma_load_2d<CG>(sa + A_BYTES, &tmB, kb * BK, b_row0, fb);
            tma_load_2d<CG>(sa + A_BYTES + B_HALF, &tmB, kb * BK, b_row0 + b_second_off, fb);
            if (sg >= 0) {
              bulk_load(ss, sa_rows + (size_t)sg * SF_CHUNK, SF_CHUNK, fb);
              bulk_load(ss + SF_CHUNK, sb0_rows + (size_t)sg * SF_CHUNK, SF_CHUNK, fb);
              bulk_load(ss + 2 * SF_CHUNK, sb1_rows + (size_t)sg * SF_CHUNK, SF_CHUNK, fb);
            }
          }
        }
        if (!ok) break;
      }
      (void)seen;
      // the copies of the last STAGES stages land before the CTA exits (the
      // first CTA's barriers also count the peer's copies, which a pair CTA
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
    if (lane == 0 && leader) {  // ------------------------------------ MMA issuer
      int it = 0, tcount = 0;
      for (int tile = cta_group; tile < total; tile += n_groups, ++tcount) {
        if (!wait_phase(saddr(&ctl->tempty), ((uint32_t)tcount & 1u) ^ 1u, abort_flag, status,
                        wait_ns))
          break;
        tc_fence_after();
        bool ok = true;
        for (int kb = 0; kb < KB; ++kb, ++it) {
          const int s = it % STAGES;
          const uint32_t ph = (uint32_t)(it / STAGES) & 1u;
          if (!wait_phase(saddr(&ctl->full[s]), ph, abort_flag, status, wait_ns)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sa = base + s * OPER_BYTES;
          const uint32_t ss = sf_smem + s * SF_STAGE;
          const int sg = sf_group_of_stage(kb, KG);
          MOE_CHECK(SF_COL0 + 2 * SF_COLS <= TMEM_COLS && s >= 0 && s < STAGES);
          if (sg >= 0) {   // this stage brought the scales of k group sg
            const uint32_t slot = tmem + SF_COL0 + (uint32_t)(sg & 1) * SF_COLS;
            sf_copy<CG>(slot, sf_desc(ss));
            sf_copy<CG>(slot + 4, sf_desc(ss + SF_CHUNK));
            sf_copy<CG>(slot + 8, sf_desc(ss + 2 * SF_CHUNK));
          }
          const uint32_t cur = tmem + SF_COL0 + (uint32_t)((kb >> 2) & 1) * SF_COLS;
          const uint32_t sel = (uint32_t)(kb & 3);   // scale byte of this k block
          const uint32_t idesc = idesc_fp8<CG>(sel);
          const uint64_t ad = sw128_desc(sa);
          const uint64_t bd = sw128_desc(sa + A_BYTES);
#pragma unroll
          for (uint32_t j = 0; j < 4; ++j)
            mma_fp8<CG>(tmem, ad + 2 * j, bd + 2 * j, idesc, cur | (sel << 30),
                        (cur + 4) | (sel << 30), (kb | (int)j) != 0 ? 1u : 0u);
          tc_commit<CG>(saddr(&ctl->empty[s]));
        }
        if (!ok) break;
        tc_commit<CG>(saddr(&ctl->tfull));
      }
      tc_commit<CG>(saddr(&ctl->drain));
      wait_phase(saddr(&ctl->drain), 0u, &no_abort, status, DRAIN_NS);
    }
  } else {  // -------------------------------------------------------- epilogue
    const int q = warp & 3;                 // TMEM lane quarter of this warp
    const int r_in = q * 32 + lane;         // row of the tile
    const int half = (warp - 2) >> 2;       // gate/up: which 64 of the tile's 128 h columns
    const int KBo = N_out / FP8_BLOCK;      // scale blocks of an output row (MODE 0)
    // TMEM is released on the pair's first CTA's barrier
    const uint32_t tempty_lead = (CG == 2) ? map_to_rank(saddr(&ctl->tempty), 0)
                                           : saddr(&ctl->tempty);
    int tcount = 0;
    for (int tile = cta_group; tile < total; tile += n_groups, ++tcount) {
      int m, n;
      const int e = tile_of(tile, NT, P, PB, ml0, G, m, n);
      MOE_CHECK(e >= 0 && e < G && n >= 0 && n < NT && m >= 0 &&
                m * CF::TILE_ROWS < max(kept_s[e], 1) && r_in < BM);
      const int first = m * CF::TILE_ROWS + (int)rank * BM;   // this CTA's 128 rows
      const int rows = min(BM, kept_s[e] - first);
      const long long row0 = (long long)row_off[e] + first;
      const long long grow = row0 + r_in;
      int ok = 1;
      if (lane == 0) ok = wait_phase(saddr(&ctl->tfull), (uint32_t)tcount & 1u, abort_flag, status,
                                     wait_ns);
      __syncwarp();
      ok = __shfl_sync(0xffffffffu, ok, 0);
      if (!ok) break;
      tc_fence_after();
      bool row_ok = r_in < rows;
      if (row_ok && (grow < 0 || grow >= R_max)) {   // inconsistent offsets from the caller
        atomicCAS(status, 0u, (uint32_t)MOE_ERR_DEVICE_INPUT);
        row_ok = false;
      }
      // a 128-row tile inside its expert's row range (alignment padding
      // included) leaves through staged TMA stores, otherwise row by row
      const bool staged = rows > 0 && row0 >= 0 && row0 + BM <= row_off[e + 1] && row0 + BM <= R_max;
      const uint32_t t0 = tmem + ((uint32_t)(q * 32) << 16);
      if (MODE == 0) {
        // this thread's 64 gate and 64 up accumulators (columns 64*half of
        // each), loaded before anything is computed so that TMEM is released
        // as early as possible
        uint32_t g[64], u[64];
        const uint32_t cg = t0 + (uint32_t)(64 * half);
        tmem_ld32(cg, *reinterpret_cast<uint32_t(*)[32]>(g));
        tmem_ld32(cg + 32u, *reinterpret_cast<uint32_t(*)[32]>(g + 32));
        tmem_ld32(cg + 128u, *reinterpret_cast<uint32_t(*)[32]>(u));
        tmem_ld32(cg + 160u, *reinterpret_cast<uint32_t(*)[32]>(u + 32));
        tmem_ld_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) {   // TMEM free for the next tile
          if (CG == 2) mbar_arrive_cluster(tempty_lead); else mbar_arrive_local(tempty_lead);
        }
        float h[64];
        float amax = 0.f;
#pragma unroll
        for (int k = 0; k < 64; ++k) {
          h[k] = silu_mul(g[k], u[k]);
          amax = fmaxf(amax, fabsf(h[k]));
        }
        // the h block is the tile's 128 columns: amax over both halves of the row
        float* am = ctl->amax[tcount & 1][0];
        am[half * 128 + r_in] = amax;
        epi_bar<MODE>();
        amax = fmaxf(amax, am[(half ^ 1) * 128 + r_in]);
        const int p = fp8_scale_exp(amax);
        const float inv = fp8_inv_scale(p);
        uint4 o[4];
#pragma unroll
        for (int v = 0; v < 4; ++v) {
          const float* hv = h + 16 * v;
          o[v].x = fp8x2(hv[0] * inv, hv[1] * inv) | (fp8x2(hv[2] * inv, hv[3] * inv) << 16);
          o[v].y = fp8x2(hv[4] * inv, hv[5] * inv) | (fp8x2(hv[6] * inv, hv[7] * inv) << 16);
          o[v].z = fp8x2(hv[8] * inv, hv[9] * inv) | (fp8x2(hv[10] * inv, hv[11] * inv) << 16);
          o[v].w = fp8x2(hv[12] * inv, hv[13] * inv) | (fp8x2(hv[14] * inv, hv[15] * inv) << 16);
        }
        if (half == 0 && row_ok && MOE_CHECKED(n < KBo))
          out_sf[sf_offset(grow, n, KBo)] = (uint8_t)(p + 127);
        if (staged) {
          if (threadIdx.x == 64) bulk_wait_read_all();   // the previous box has left smem
          epi_bar<MODE>();
          // 16-byte chunks 4*half .. 4*half+3 of row r_in, at the 128-byte
          // swizzle's positions
#pragma unroll
          for (int v = 0; v < 4; ++v) {
            const int c = 4 * half + v;
            const uint32_t a = staging + (uint32_t)(r_in * 128 + ((c ^ (r_in & 7)) << 4));
            MOE_CHECK(r_in * 128 + 128 <= STAGING_BYTES);
            asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(a), "r"(o[v].x),
                         "r"(o[v].y), "r"(o[v].z), "r"(o[v].w)
                         : "memory");
          }
          fence_proxy_async_smem();
          epi_bar<MODE>();
          if (threadIdx.x == 64) {
            tma_store_2d(&tmOut, n * BN_OUT, (int)row0, staging);
            bulk_commit();
          }
        } else if (row_ok) {
          uint4* dst = reinterpret_cast<uint4*>(static_cast<uint8_t*>(out_v) + grow * N_out +
                                                (long long)n * BN_OUT + 64 * half);
#pragma unroll
          for (int v = 0; v < 4; ++v) dst[v] = o[v];
        }
      } else {
        uint32_t pk[128];   // 256 bf16 of this row
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          uint32_t a[64];
          tmem_ld64(t0 + (uint32_t)(c * 64), a);
          tmem_ld_wait();
#pragma unroll
          for (int k = 0; k < 32; ++k)
            pk[c * 32 + k] = pack_bf16x2(__uint_as_float(a[2 * k]), __uint_as_float(a[2 * k + 1]));
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) {
          if (CG == 2) mbar_arrive_cluster(tempty_lead); else mbar_arrive_local(tempty_lead);
        }
        __nv_bfloat16* orow = static_cast<__nv_bfloat16*>(out_v) + (row_ok ? grow : 0) * (long long)N_out;
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          const int col = n * BN_OUT + c * 64;
          if (col >= N_out) continue;   // N_out % 64 == 0: a chunk is all in or all out
          uint4 o[8];
#pragma unroll
          for (int v = 0; v < 8; ++v)
            o[v] = make_uint4(pk[c * 32 + 4 * v], pk[c * 32 + 4 * v + 1], pk[c * 32 + 4 * v + 2],
                              pk[c * 32 + 4 * v + 3]);
          if (staged) {
            if (threadIdx.x == 64) bulk_wait_read_all();
            epi_bar<MODE>();
            stage_row(staging, r_in, o);
            fence_proxy_async_smem();
            epi_bar<MODE>();
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
        if (ept.yready != nullptr && rows > 0) {
          // Publish this half tile at system scope, into this step's bank of
          // the expert-parallel ready counters (read by the peers' combines):
          // its 128 rows (one ready block) have one more N tile stored. The
          // staged stores are waited for by their issuing thread, every
          // thread fences its own stores, then one release add.
          __threadfence_system();
          if (threadIdx.x == 64) {
            bulk_wait_all();
            fence_proxy_async_global();
          }
          epi_bar<MODE>();
          if (threadIdx.x == 64 && MOE_CHECKED(row0 >= 0 && row0 / READY_ROWS < ept.ready_blocks))
            red_release_add_sys(ept.yready + (size_t)(step & 1u) * ept.ready_blocks +
                                    (size_t)(row0 / READY_ROWS),
                                1u);
        }
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

// 2-D uint8 map over a row-major [rows, cols] byte matrix: box 128 x 128,
// 128-byte swizzle, zeros outside.
bool make_map_u8(CUtensorMap* map, const void* base, uint64_t cols, uint64_t rows) {
  PFN_cuTensorMapEncodeTiled_v12000 enc = encode_fn();
  if (!enc) return false;
  const cuuint64_t dims[2] = {cols, rows};
  const cuuint64_t strides[1] = {cols};
  const cuuint32_t box[2] = {128, 128};
  const cuuint32_t estr[2] = {1, 1};
  return enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box,
             estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// The scale chunks of a blocked scale buffer ([rows/128][KG][512 bytes]) as a
// 2-D uint32 tensor [chunks][128]: one chunk per box, no swizzle.
bool make_map_sf(CUtensorMap* map, const void* base, int64_t rows, int64_t kdim) {
  PFN_cuTensorMapEncodeTiled_v12000 enc = encode_fn();
  if (!enc) return false;
  const int64_t chunks = ceil_div(rows, 128) * ceil_div(kdim / FP8_BLOCK, 4);
  const cuuint64_t dims[2] = {SF_CHUNK / 4, (cuuint64_t)chunks};
  const cuuint64_t strides[1] = {SF_CHUNK};
  const cuuint32_t box[2] = {SF_CHUNK / 4, 1};
  const cuuint32_t estr[2] = {1, 1};
  return enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT32, 2, const_cast<void*>(base), dims, strides, box,
             estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int MODE, int CG>
cudaError_t launch_one(int grid, size_t smem, cudaStream_t s, const CUtensorMap& a,
                       const CUtensorMap& b, const CUtensorMap& o, const CUtensorMap& msfa,
                       const CUtensorMap& msfb, const uint8_t* sfa, const uint8_t* sfb, void* out,
                       uint8_t* out_sf, int N_out, int Kdim, int b_rows, int b_second,
                       const int32_t* offsets, const int32_t* counts, int E, int C,
                       long long R_max, uint32_t* status, int sh_rows, int sh_row0,
                       const EpTiles& ept) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)grid);
  cfg.blockDim = dim3(num_threads<MODE>());
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  attr[1].id = cudaLaunchAttributeClusterDimension;
  attr[1].val.clusterDim.x = CG;
  attr[1].val.clusterDim.y = 1;
  attr[1].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  return cudaLaunchKernelEx(&cfg, fp8_grouped_gemm<MODE, CG>, a, b, o, msfa, msfb, sfa, sfb, out,
                            out_sf, N_out, Kdim, b_rows, b_second, offsets, counts, E, C, R_max,
                            status, sh_rows, sh_row0, ept);
}

// Co-resident CTAs (CG = 1) or CTA pairs (CG = 2) of one launch.
template <int MODE, int CG>
int resident_groups(size_t smem) {
  int dev = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    return 0;
  if (CG == 1) return sms;
  cudaLaunchConfig_t q = {};
  q.gridDim = dim3((unsigned)(sms & ~1));
  q.blockDim = dim3(num_threads<MODE>());
  q.dynamicSmemBytes = smem;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  q.attrs = attr;
  q.numAttrs = 1;
  int clusters = 0;
  if (cudaOccupancyMaxActiveClusters(&clusters, fp8_grouped_gemm<MODE, CG>, &q) != cudaSuccess)
    return 0;
  return clusters;
}

template <int CG>
moe_status_t launch_mlp(const moe_config_t& c, const uint8_t* xq, const uint8_t* xs,
                        const int32_t* offsets, const int32_t* counts, const uint8_t* wq_gu,
                        const uint8_t* ws_gu, const uint8_t* wq_d, const uint8_t* ws_d,
                        uint8_t* hq, uint8_t* hs, void* y, int64_t R_max, uint32_t* status,
                        cudaStream_t s, int modes = 3, const EpTiles& ept = EpTiles{}) {
  const int n_sh = c.n_shared ? 1 : 0;
  const int G = c.E + n_sh;   // routed experts + the shared expert (last in the weights)
  CUtensorMap mx, mwgu, mh, mwd, my, sx, sgu, shh, sd;
  if (!make_map_u8(&mx, xq, (uint64_t)c.H, (uint64_t)R_max) ||
      !make_map_u8(&mwgu, wq_gu, (uint64_t)c.H, (uint64_t)G * 2 * c.F) ||
      !make_map_u8(&mh, hq, (uint64_t)c.F, (uint64_t)R_max) ||
      !make_map_u8(&mwd, wq_d, (uint64_t)c.F, (uint64_t)G * c.H) ||
      !tc::make_map(&my, y, (uint64_t)c.H, (uint64_t)R_max))
    return MOE_ERR_CUDA;
  if (CG == 2) {
    if (!make_map_sf(&sx, xs, R_max, c.H) || !make_map_sf(&sgu, ws_gu, (int64_t)G * 2 * c.F, c.H) ||
        !make_map_sf(&shh, hs, R_max, c.F) || !make_map_sf(&sd, ws_d, (int64_t)G * c.H, c.F))
      return MOE_ERR_CUDA;
  } else {   // not read by the one-CTA kernel
    sx = sgu = shh = sd = mx;
  }
  const int sh_rows = n_sh ? c.T : 0;
  const int sh_row0 = n_sh ? (int)shared_row0(c) : 0;
  const size_t smem = smem_bytes<CG>(G, ept.remote_first != 0 && ept.split != nullptr);
  if (cudaFuncSetAttribute(fp8_grouped_gemm<0, CG>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)smem) != cudaSuccess ||
      cudaFuncSetAttribute(fp8_grouped_gemm<1, CG>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)smem) != cudaSuccess)
    return MOE_ERR_CUDA;
  const int u0 = resident_groups<0, CG>(smem), u1 = resident_groups<1, CG>(smem);
  if (u0 <= 0 || u1 <= 0) return MOE_ERR_CUDA;
  const int64_t mt_bound = ceil_div(R_max, F8<CG>::TILE_ROWS) + G;   // >= sum of M tiles
  const int g0 = (int)std::min<int64_t>(u0, mt_bound * ceil_div(c.F, 128)) * CG;
  const int g1 = (int)std::min<int64_t>(u1, mt_bound * ceil_div(c.H, 256)) * CG;
  // gate/up: the arrival waits only; down: the ready-counter publication only
  EpTiles t0 = ept, t1 = ept;
  t0.yready = nullptr;
  t1.arrive = nullptr;
  cudaError_t e = cudaSuccess;
  if (modes & 1)
    e = launch_one<0, CG>(g0, smem, s, mx, mwgu, mh, sx, sgu, xs, ws_gu, hq, hs, c.F, c.H, 2 * c.F,
                          c.F, offsets, counts, c.E, c.capacity, (long long)R_max, status,
                          sh_rows, sh_row0, t0);
  if (e == cudaSuccess && (modes & 2))
    e = launch_one<1, CG>(g1, smem, s, mh, mwd, my, shh, sd, hs, ws_d, y, nullptr, c.H, c.F, c.H,
                          128, offsets, counts, c.E, c.capacity, (long long)R_max, status,
                          sh_rows, sh_row0, t1);
  return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

}  // namespace f8

moe_status_t launch_mlp_fp8(const moe_config_t& c, const uint8_t* xq, const uint8_t* xs,
                            const int32_t* offsets, const int32_t* counts, const uint8_t* wq_gu,
                            const uint8_t* ws_gu, const uint8_t* wq_d, const uint8_t* ws_d,
                            uint8_t* hq, uint8_t* hs, void* y, int64_t R_max, uint32_t* status,
                            cudaStream_t s) {
  if (R_max == 0) return MOE_OK;
  // 256-row CTA-pair tiles halve each CTA's operand bytes per k step; small
  // experts (decode-like batches) keep 128-row one-CTA tiles, whose padding
  // is half as large (as in the bf16 grouped GEMM)
  const int64_t rows_per_expert =
      c.E > 0 ? std::min<int64_t>((int64_t)c.T * c.K, (int64_t)c.E * c.capacity) / c.E : c.T;
  if (rows_per_expert >= 192)
    return f8::launch_mlp<2>(c, xq, xs, offsets, counts, wq_gu, ws_gu, wq_d, ws_d, hq, hs, y,
                             R_max, status, s);
  return f8::launch_mlp<1>(c, xq, xs, offsets, counts, wq_gu, ws_gu, wq_d, ws_d, hq, hs, y, R_max,
                           status, s);
}

size_t fp8_ep_smem_bytes(const moe_config_t& c, bool two_sets) {
  const int64_t rows_per_expert =
      c.E > 0 ? std::min<int64_t>((int64_t)c.T * c.K, (int64_t)c.E * c.capacity) / c.E : c.T;
  return rows_per_expert >= 192 ? f8::smem_bytes<2>(c.E, two_sets)
                                : f8::smem_bytes<1>(c.E, two_sets);
}

moe_status_t launch_mlp_fp8_ep(const moe_config_t& c, int modes, const uint8_t* xq,
                               const uint8_t* xs, const int32_t* offsets, const int32_t* counts,
                               const uint8_t* wq_gu, const uint8_t* ws_gu, const uint8_t* wq_d,
                               const uint8_t* ws_d, uint8_t* hq, uint8_t* hs, void* y,
                               int64_t R_max, uint32_t* status, cudaStream_t s,
                               const EpTiles& t) {
  if (R_max == 0) return MOE_OK;
  moe_config_t l = c;
  l.n_shared = 0;
  const int64_t rows_per_expert =
      c.E > 0 ? std::min<int64_t>((int64_t)c.T * c.K, (int64_t)c.E * c.capacity) / c.E : c.T;
  if (rows_per_expert >= 192)
    return f8::launch_mlp<2>(l, xq, xs, offsets, counts, wq_gu, ws_gu, wq_d, ws_d, hq, hs, y,
                             R_max, status, s, modes, t);
  return f8::launch_mlp<1>(l, xq, xs, offsets, counts, wq_gu, ws_gu, wq_d, ws_d, hq, hs, y, R_max,
                           status, s, modes, t);
}

}  // namespace moe

// gemm.cu — persistent 2D x 3D NVFP4 block-scaled grouped GEMM for sm_100a (tcgen05 + TMEM).
//
// The operation is the grouped GEMM of "NVFP4 MegaMoE Kernel Rewrite — CuTeDSL" (section "The
// Reference Kernel: ScaledGroupedGemmKernel"): A(tokens, K) x B(experts, N, K) -> C(tokens, N),
// tokens bucketed per expert, E2M1 operands with one E4M3 scale per 16 elements, FP32
// accumulation.  The pages' kernel is a 7-warp CuTeDSL design; this one is written directly in
// PTX for sm_100a:
//
//   warp 0      TMA producer: A and B tiles (cp.async.bulk.tensor, 128-byte swizzle) into a
//               4-stage shared-memory ring
//   warp 3      scale producer: the pre-tiled scale atoms (cp.async.bulk) into a ring of their
//               own, ahead of the A/B ring
//   warp 1      MMA issuer (whole warp, elect.sync): tcgen05.mma.kind::mxf4nvf4.block_scale
//               (M=128, N=256, K=64) into a TMEM accumulator; it issues nothing else, because
//               the tensor pipe runs its instructions one after another and scale copies in that
//               stream cost as much as the MMAs themselves
//   warp 2      owns the tensor-memory allocation (512 columns)
//   warps 4..11 epilogue (176 registers each, setmaxnreg): tcgen05.ld of the accumulator (warp w
//               reads lanes 32*(w%4)..+31), then one of the fused epilogues below
//   warps 12..15 scale-factor warps: each stage's scale atoms go from the scale ring to the
//               tensor-memory layout the MMA reads, by ld.shared + tcgen05.st, one warp per
//               lane quadrant, as soon as the stage's tensor-memory columns are free
//
// Epilogues (the MODE template parameter):
//   PLAIN_F32 / PLAIN_BF16  C = acc / (gs_a * gs_b[e])
//   L1  SwiGLU + NVFP4 re-quantization in registers ("May 24, 2026 — Session Start Plan",
//       section 5 "NVFP4-1.1"): W1 is stored gate/up interleaved in 16-row blocks, so the
//       256-row B tile holds gate and up rows of the same 128 h features and each epilogue
//       thread finds matching gate and up values 16 accumulator columns apart.
//   L2  routing weight + scatter: each row's weighted output is stored to its slot's row of an
//       FP32 [T*k][H] buffer; a combine kernel then sums each token's k rows in a fixed order
//       (no atomics: FP32 reductions into a shared accumulator were the bottleneck).
//
// Tile scheduler: each expert's 128-padded row segment gives (rows/128) M-tiles; tiles are
// numbered expert by expert with the N-tile outer and the M-tile inner, so CTAs running at the
// same time share B (weight) tiles through L2.  CTAs take tiles with a static stride.  The
// segment offsets are read on the device: no host sync between routing and the GEMM.
//
// Every mbarrier wait is bounded (NVFP4_WAIT_TIMEOUT_NS).  A wait that runs out raises a CTA-wide
// abort flag: the producer waits (bounded) for its copies in flight, the MMA warp drains its
// MMAs, the tensor memory is freed and the kernel reports NVFP4_DEVERR_TIMEOUT.
#include <cudaTypedefs.h>

#include <mutex>

#include "common.cuh"
#include "launch.h"

namespace nvfp4 {
namespace {

constexpr int BM = 128;
constexpr int BK_BYTES = 128;  // 256 FP4 elements per stage along K
constexpr int A_BYTES = BM * BK_BYTES;                // 16 KB
constexpr uint32_t TMEM_COLS = 512;
constexpr int NUM_THREADS = 512;  // 4 role warps + 8 epilogue warps + 4 scale-factor warps
constexpr int EPI_WARP0 = 4;
constexpr int EPI_WARPS = 8;
constexpr int SF_WARP0 = EPI_WARP0 + EPI_WARPS;
// Register budgets per warpgroup (the block is launched with 128 per thread): the two epilogue
// warpgroups hold a whole 128-column accumulator slice in registers; the producer / MMA group
// and the scale-factor group need few.
constexpr uint32_t REGS_EPI = 176, REGS_OTHER = 80;
static_assert(2 * REGS_EPI + 2 * REGS_OTHER == 4 * 128, "register budgets exceed the launch's");
constexpr int MAX_E = 256;

// L2_ROWS:   each weighted row is stored to its slot's row of an FP32 [S][H] buffer; the rows
//            are exchanged between the lanes of an octet by register shuffles so that a warp
//            writes 4 rows x 128 bytes per store instruction.  A combine kernel then sums each
//            token's k slot rows in slot order (deterministic).
// L2_ATOMIC: each weighted row is added into its token's row of an FP32 [T][H] accumulator
//            (red.global.add.v4.f32, 4 rows x 128 bytes per warp instruction) instead of stored
//            to its slot's row;
//            tiles run N-slice by N-slice so the accumulator slice being added into (T x 256
//            floats) stays in L2.  No staging buffer: 4 stages.  The sum order of a token's
//            slots is not fixed.
enum Mode { PLAIN_F32 = 0, PLAIN_BF16 = 1, L1_SWIGLU = 2, L2_ROWS = 3, L2_ATOMIC = 4 };
template <int MODE>
__host__ __device__ constexpr bool is_l2() {
  return MODE == L2_ROWS || MODE == L2_ATOMIC;
}
// Tiles numbered N-slice by N-slice (all experts' M-tiles of N-slice 0, then of N-slice 1, ...)
// rather than expert by expert.
template <int MODE>
__host__ __device__ constexpr bool slice_major() { return MODE == L2_ATOMIC; }

// Average routed rows per expert from which the FFN's L2 adds into token rows (scatter-add)
// instead of writing slot rows and combining them
constexpr int kL2AtomicMinRowsPerExpert = 32;

// Tile width (N) per epilogue.  256 columns fill tensor memory with one accumulator; 128 leave
// room for two, so the epilogue of one tile overlaps the MMAs of the next.
constexpr int kL1TileN = 256;
constexpr int kL2TileN = 256;
template <int MODE>
constexpr int tile_n() {
  return MODE == L1_SWIGLU ? kL1TileN : is_l2<MODE>() ? kL2TileN : 256;
}

// Tile shape: M = 128 rows per CTA, N = 256 columns, K = 256 per stage.  One MMA instruction
// has a fixed cost, so the widest N moves the most weight bytes per instruction; one 256-column
// accumulator and the per-stage scale columns fill tensor memory.
//
// CTAS = 2 runs the pair form (cta_group::2) on a cluster of 2 CTAs: a 256 x 256 tile, each CTA
// holding 128 rows of A and 128 rows (N) of B per stage, so each SM moves 2/3 of the operand
// bytes of a 128 x 256 tile for the same MMA work.  The even CTA (the leader) issues the MMAs;
// both CTAs run producer, scale-factor and epilogue warps.
// SFV: elements per block scale: 16 (NVFP4: E4M3 scales, 4 per row per 64 of K) or 32 (MXFP4:
// UE8M0 scales, 2 per row per 64 of K).  The scales come in atoms of 128 rows x 4 scale columns
// (512 bytes), so one atom covers 4 * SFV elements of K and a 256-element stage takes NA atoms.
template <int MODE, int CTAS, int SFV = 16>
struct TileCfg {
  static_assert(SFV == 16 || SFV == 32, "NVFP4 or MXFP4 block scales");
  static constexpr int NA = 256 / (4 * SFV);               // scale atoms per stage along K
  static constexpr int SFA_BYTES = NA * 512;               // 128 rows x NA atoms
  static constexpr int SFA_COLS = 4 * NA;                  // tensor-memory columns of SFA
  static constexpr int BN = tile_n<MODE>();
  static_assert(BN == 128 || BN == 256, "tile width");
  static_assert(CTAS == 1 || BN == 256, "pair tiles are 256 columns wide");
  static constexpr int B_ROWS = BN / CTAS;                 // B rows (N) per CTA per stage
  static constexpr int B_BYTES = B_ROWS * BK_BYTES;
  static constexpr int SFB_BYTES = (BN / 128) * NA * 512;  // scales of all BN rows of B
  // A/B ring: STAGES slots of AB_BYTES.  Scale atoms have a ring of their own (SF_STAGES slots of
  // SF_BYTES), filled ahead of the A/B ring by a separate producer warp, so a stage's scales are
  // already in shared memory when its tensor-memory columns become free.
  static constexpr int AB_BYTES = A_BYTES + B_BYTES;
  static constexpr int SF_BYTES = SFA_BYTES + SFB_BYTES;
  static constexpr int SF_STAGES = 4;
  static constexpr int EPI_STAGE_BYTES = 0;  // no epilogue staging buffer
  static constexpr uint32_t SFB_COLS = (BN / 128) * 4 * NA;  // scale columns of B per stage
  static constexpr int STAGES_SMEM =
      (216 * 1024 - EPI_STAGE_BYTES - SF_STAGES * SF_BYTES) / AB_BYTES;
  static constexpr int STAGES_TMEM = (TMEM_COLS - BN) / (SFA_COLS + SFB_COLS);
  static constexpr int STAGES = STAGES_SMEM < STAGES_TMEM ? STAGES_SMEM : STAGES_TMEM;
  static constexpr int SF_OFFSET = STAGES * AB_BYTES;
  static constexpr int EPI_OFFSET = SF_OFFSET + SF_STAGES * SF_BYTES;
  static constexpr int SMEM_BYTES = EPI_OFFSET + EPI_STAGE_BYTES + 1024;
  static constexpr int ACC_BUFS = 2 * BN + STAGES * (SFA_COLS + SFB_COLS) <= TMEM_COLS ? 2 : 1;
  static constexpr uint32_t TM_SFA = ACC_BUFS * BN;        // SFA_COLS columns per stage
  static constexpr uint32_t TM_SFB = TM_SFA + STAGES * SFA_COLS;
  static constexpr uint32_t IDESC =
      SFV == 16 ? idesc_nvf4(BN, 128 * CTAS) : idesc_mxf4(BN, 128 * CTAS);
  static_assert(AB_BYTES % 1024 == 0, "stages must keep 1024-byte alignment (128B swizzle)");
  static_assert(SF_BYTES % 16 == 0, "bulk copies need 16-byte alignment");
  static_assert(TM_SFB + STAGES * SFB_COLS <= TMEM_COLS, "tensor memory budget");
};

struct GemmArgs {
  const uint8_t* sfa;
  const uint8_t* sfb;
  const float* gs_a;
  const float* gs_b;
  const int32_t* offs;
  int E;
  int N;         // rows per expert in B (2I for L1)
  int K;         // reduction length (elements)
  int n_tiles;   // N-tiles per expert
  int64_t R_max;
  void* out;     // PLAIN: [R_max][N]
  const float* gs_h;  // L1
  uint8_t* h;         // L1: [R_max][I/2]
  uint8_t* sfh;       // L1
  int I;              // L1
  float* h32;         // L1 (optional): FP32 h before quantization [R_max][I]
  uint32_t* h_stats;  // L1 (optional): amax bits of |h|, saturated and underflowed block scales
  const int32_t* row_slot;   // L2 (required), L1 (optional: skip padding rows)
  const float* row_w;        // L2
  float* ys;                 // L2: weighted expert outputs per slot [S][H]; L2_ATOMIC: [T][H]
  int S;                     // L2: slots (T*k)
  int k;                     // L2_ATOMIC: slots per token (token = slot / k)
  int32_t* status;
  int64_t out_rows;          // PLAIN: rows of `out`; rows at or past it are not stored
  int k_splits;              // PLAIN_F32: each tile's K is cut into this many ranges
  int64_t split_stride;      // PLAIN_F32, k_splits > 1: floats between two ranges' outputs
};

struct Tile {
  int e, m0, nt;
};

// Tile t -> (expert, first row, N-tile).  Each expert's segment gives ceil(rows / (128*CTAS))
// M-tiles of 128*CTAS rows.
template <int CTAS, bool SLICE_MAJOR = false>
__device__ __forceinline__ Tile decode_tile(int t, const int* tile_start, const int* seg, int E,
                                            int n_tiles) {
  if constexpr (SLICE_MAJOR) {
    // tile_start holds the prefix of M-tiles per expert; one N-slice has tile_start[E] tiles
    const int per_slice = tile_start[E];
    Tile r;
    r.nt = t / per_slice;
    const int u = t - r.nt * per_slice;
    int lo = 0, hi = E;  // tile_start[lo] <= u < tile_start[hi]
    while (hi - lo > 1) {
      const int mid = (lo + hi) >> 1;
      if (tile_start[mid] <= u) lo = mid;
      else hi = mid;
    }
    r.e = lo;
    r.m0 = seg[lo] + (u - tile_start[lo]) * (BM * CTAS);
    return r;
  }
  int lo = 0, hi = E;  // tile_start[lo] <= t < tile_start[hi]
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (tile_start[mid] <= t) lo = mid;
    else hi = mid;
  }
  const int local = t - tile_start[lo];
  const int mt_cnt = (((seg[lo + 1] - seg[lo]) >> 7) + CTAS - 1) / CTAS;
  Tile r;
  r.e = lo;
  r.nt = local / mt_cnt;
  r.m0 = seg[lo] + (local - r.nt * mt_cnt) * (BM * CTAS);
  return r;
}

template <int MODE, int CTAS, int SFV>
__global__ void __launch_bounds__(NUM_THREADS, 1)
    grouped_gemm_kernel(const __grid_constant__ CUtensorMap tm_a,
                        const __grid_constant__ CUtensorMap tm_b, const GemmArgs args) {
  using C = TileCfg<MODE, CTAS, SFV>;
  constexpr int NA = C::NA;
  constexpr int STAGES = C::STAGES;
  constexpr int BN = C::BN;
  constexpr int ACC_BUFS = C::ACC_BUFS;
  constexpr bool PAIR = CTAS == 2;
  extern __shared__ uint8_t smem_raw[];
  // A/B landed (a pair: both CTAs') and the stage's scales in tensor memory (all CTAs'
  // scale-factor warps): one barrier, so that the MMA warp waits once per stage
  __shared__ __align__(8) uint64_t bar_full[STAGES];
  __shared__ __align__(8) uint64_t bar_empty[STAGES];  // MMAs done with the stage
  __shared__ __align__(8) uint64_t bar_sfin[C::SF_STAGES];     // scale atoms landed in a slot
  __shared__ __align__(8) uint64_t bar_sfempty[C::SF_STAGES];  // scale slot copied out
  __shared__ __align__(8) uint64_t bar_acc_full[ACC_BUFS];
  __shared__ __align__(8) uint64_t bar_acc_empty[ACC_BUFS];
  __shared__ __align__(8) uint64_t bar_drain;
  __shared__ uint32_t tmem_slot;
  __shared__ int seg[MAX_E + 1];
  __shared__ int tile_start[MAX_E + 1];
  __shared__ int warp_sums[NUM_THREADS / 32];
  __shared__ int bad_offsets;
  __shared__ volatile int abort_flag;

  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int E = args.E;
  const uint32_t rank = PAIR ? cluster_ctarank() : 0u;  // 0 = leader
  const int cluster_id = blockIdx.x / CTAS, num_clusters = gridDim.x / CTAS;
  // shared::cluster address of this CTA's barrier `bar` in the leader / in the other CTA
  auto at_leader = [&](const uint64_t* bar) {
    return PAIR ? mapa_shared(smem_u32(bar), 0u) : smem_u32(bar);
  };
  auto at_peer = [&](const uint64_t* bar) { return mapa_shared(smem_u32(bar), rank ^ 1u); };

  // ---- scheduler table: tiles per expert, exclusive scan over experts
  if (tid == 0) {
    bad_offsets = 0;
    abort_flag = 0;
  }
  // E + 1 segment starts; no offsets = one dense segment of R_max rows (E = 1)
  for (int i = tid; i <= E; i += NUM_THREADS)
    seg[i] = args.offs != nullptr ? __ldg(args.offs + i) : (i == 0 ? 0 : (int)args.R_max);
  __syncthreads();
  int my_tiles = 0;
  if (tid < E) {
    const int lo = seg[tid], hi = seg[tid + 1];
    if (lo < 0 || hi < lo || (lo & 127) || (hi & 127) || hi > args.R_max) bad_offsets = 1;
    else
      my_tiles = ((((hi - lo) >> 7) + CTAS - 1) / CTAS) * (slice_major<MODE>() ? 1 : args.n_tiles);
  }
  int incl = my_tiles;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int v = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += v;
  }
  if (lane == 31) warp_sums[warp] = incl;
  __syncthreads();
  if (tid == 0) {
    int run = 0;
    for (int w = 0; w < NUM_THREADS / 32; ++w) {
      const int c = warp_sums[w];
      warp_sums[w] = run;
      run += c;
    }
  }
  __syncthreads();
  const int excl = warp_sums[warp] + incl - my_tiles;
  if (tid < E) tile_start[tid] = excl;
  if (tid == E - 1) tile_start[E] = excl + my_tiles;

  // ---- barriers and tensor memory
  if (tid == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(smem_u32(&bar_full[s]), 1 + 4 * CTAS);  // producer + scale-factor warps
      mbar_init(smem_u32(&bar_empty[s]), 1);
    }
    for (int j = 0; j < C::SF_STAGES; ++j) {
      mbar_init(smem_u32(&bar_sfin[j]), 1);
      mbar_init(smem_u32(&bar_sfempty[j]), 4);
    }
    for (int b = 0; b < ACC_BUFS; ++b) {
      mbar_init(smem_u32(&bar_acc_full[b]), 1);
      mbar_init(smem_u32(&bar_acc_empty[b]), EPI_WARPS * CTAS);
    }
    mbar_init(smem_u32(&bar_drain), 1);
    fence_mbar_init();
  }
  if (warp == 2) {
    if constexpr (PAIR) {
      tmem_alloc_pair(smem_u32(&tmem_slot), TMEM_COLS);
      tmem_relinquish_pair();
    } else {
      tmem_alloc(smem_u32(&tmem_slot), TMEM_COLS);
      tmem_relinquish();
    }
  }
  tc_fence_before();
  __syncthreads();
  if constexpr (PAIR) cluster_sync();  // the peer's barriers are initialised before any remote use
  tc_fence_after();
  const uint32_t tmem = tmem_slot;
  // PLAIN_F32 may cut each tile's K into KS ranges (split-K, for a dense product with fewer
  // tiles than SMs): work item t is K range t % KS of tile t / KS.  KS is 1 in every other mode.
  const int KS = MODE == PLAIN_F32 ? args.k_splits : 1;
  const int total =
      bad_offsets ? 0 : tile_start[E] * KS * (slice_major<MODE>() ? args.n_tiles : 1);
  if (tid == 0 && bad_offsets && blockIdx.x == 0) report(args.status, NVFP4_DEVERR_BAD_OFFSETS);

  const int K = args.K;
  const int nk = (K + 255) / 256;  // stages along K
  const int atoms_k = K / (4 * SFV);  // scale atoms along K (64 or 128 elements each)
  const int mma_k = K / 64;           // K = 64 MMA steps
  // stages [lo, hi) of work item t (the host keeps KS <= nk, so no range is empty)
  auto k_range = [&](int t, int& lo, int& hi) {
    const int ks = t % KS;
    lo = ks * nk / KS;
    hi = (ks + 1) * nk / KS;
  };

  // Roles by warpgroup (4 warps each).  setmaxnreg is executed by a whole warpgroup at the top
  // of its own branch: warpgroups 0 (producer, MMA) and 3 (scale factors) give registers to
  // warpgroups 1 and 2 (epilogue).
  if (warp < EPI_WARP0) {
    regs_release_to<REGS_OTHER>();
    if (warp == 0) {
      // =========================== TMA producer ===========================
      if (lane == 0) {
        prefetch_tmap(&tm_a);
        prefetch_tmap(&tm_b);
        uint32_t it = 0;
        bool ok = true;
        for (int t = cluster_id; t < total && ok; t += num_clusters) {
          const Tile tl = decode_tile<CTAS, slice_major<MODE>()>(t / KS, tile_start, seg, E,
                                                                args.n_tiles);
          const int m_cta = tl.m0 + BM * rank;  // this CTA's rows
          // B rows of this N-tile: BN consecutive rows (for L1: 16-row gate blocks each followed by
          // the 16 matching up rows); a pair's CTA r loads rows B_ROWS*r .. B_ROWS*r + B_ROWS-1
          const int b_row0 = tl.e * args.N + tl.nt * BN;
          int kb_lo, kb_hi;
          k_range(t, kb_lo, kb_hi);
          for (int kb = kb_lo; kb < kb_hi; ++kb, ++it) {
            const int s = it % STAGES;
            const uint32_t ph = (it / STAGES) & 1u;
            if (!mbar_wait_bounded(smem_u32(&bar_empty[s]), ph ^ 1u, &abort_flag)) {
              ok = false;
              break;
            }
            uint8_t* st = smem + s * C::AB_BYTES;
            const uint32_t sA = smem_u32(st), sB = sA + A_BYTES;
            if constexpr (PAIR) {
              const uint32_t full = at_leader(&bar_full[s]);
              if (rank == 0) mbar_arrive_expect_tx(smem_u32(&bar_full[s]), 2 * (A_BYTES + C::B_BYTES));
              tma_load_2d_pair(sA, &tm_a, full, kb * BK_BYTES, m_cta);
              tma_load_2d_pair(sB, &tm_b, full, kb * BK_BYTES, b_row0 + C::B_ROWS * (int)rank);
            } else {
              const uint32_t full = smem_u32(&bar_full[s]);
              mbar_arrive_expect_tx(full, A_BYTES + C::B_BYTES);
              tma_load_2d(sA, &tm_a, full, kb * BK_BYTES, m_cta);
  #pragma unroll
              for (int j = 0; j < BN / 128; ++j)
                tma_load_2d(sB + j * 128 * BK_BYTES, &tm_b, full, kb * BK_BYTES, b_row0 + 128 * j);
            }
          }
        }
        if (!ok) {
          // let the copies already issued land before the CTA can exit
          volatile int never = 0;
          const uint32_t first = it > (uint32_t)STAGES ? it - STAGES : 0u;
          for (uint32_t j = first; j < it && !PAIR; ++j)
            mbar_wait_bounded(smem_u32(&bar_full[j % STAGES]), (j / STAGES) & 1u, &never,
                              NVFP4_WAIT_TIMEOUT_NS / 4);
          if (PAIR) {  // this CTA's A/B boxes complete on the leader's barrier: give them time
            const uint64_t t0 = global_timer_ns();
            while (global_timer_ns() - t0 < 2000000ull) {
            }
          }
        }
      }
      __syncwarp();
    } else if (warp == 3) {
      // =========================== scale producer ===========================
      // Scale atoms of every stage (this CTA's 128 A rows, all BN rows of B) into the scale ring;
      // it runs ahead of the A/B producer by up to SF_STAGES stages.
      if (lane == 0) {
        uint32_t it = 0;
        bool ok = true;
        for (int t = cluster_id; t < total && ok; t += num_clusters) {
          const Tile tl = decode_tile<CTAS, slice_major<MODE>()>(t / KS, tile_start, seg, E,
                                                                args.n_tiles);
          const int m_cta = tl.m0 + BM * rank;
          // a pair's second half past the expert's segment computes rows it never writes; its
          // scale atoms are taken from the first half so that every read stays inside the tensor
          const int a_blk = (m_cta < seg[tl.e + 1] ? m_cta : tl.m0) >> 7;
          const int b_blk = (tl.e * args.N + tl.nt * BN) >> 7;
          int kb_lo, kb_hi;
          k_range(t, kb_lo, kb_hi);
          for (int kb = kb_lo; kb < kb_hi; ++kb, ++it) {
            const int j = it % C::SF_STAGES;
            const uint32_t ph = (it / C::SF_STAGES) & 1u;
            if (!mbar_wait_bounded(smem_u32(&bar_sfempty[j]), ph ^ 1u, &abort_flag)) {
              ok = false;
              break;
            }
            const int natoms = min(NA, atoms_k - kb * NA);
            const uint32_t sSFA = smem_u32(smem + C::SF_OFFSET + j * C::SF_BYTES);
            const uint32_t sf_bar = smem_u32(&bar_sfin[j]);
            mbar_arrive_expect_tx(sf_bar, natoms * 512 * (1 + BN / 128));
            bulk_load(sSFA, args.sfa + ((int64_t)a_blk * atoms_k + kb * NA) * 512, natoms * 512,
                      sf_bar);
#pragma unroll
            for (int jj = 0; jj < BN / 128; ++jj) {
              const int64_t b_atom = (int64_t)(b_blk + jj) * atoms_k + kb * NA;
              bulk_load(sSFA + C::SFA_BYTES + jj * NA * 512, args.sfb + b_atom * 512,
                        natoms * 512, sf_bar);
            }
          }
        }
        if (!ok) {  // let the copies already issued land before the CTA can exit
          volatile int never = 0;
          const uint32_t first = it > (uint32_t)C::SF_STAGES ? it - C::SF_STAGES : 0u;
          for (uint32_t j = first; j < it; ++j)
            mbar_wait_bounded(smem_u32(&bar_sfin[j % C::SF_STAGES]), (j / C::SF_STAGES) & 1u,
                              &never, NVFP4_WAIT_TIMEOUT_NS / 4);
        }
      }
      __syncwarp();
    } else if (warp == 1) {
      // =========================== MMA issuer (the leader's, for a pair) ===========================
      // The whole warp runs the loop; elect.sync picks the issuing lane.  Waits are agreed across
      // the warp so that every lane leaves the loop together.
      if (rank == 0) {
        // Descriptors of stage 0; stage s adds s * AB_BYTES / 16 to the start-address field
        // (bits [0,14) hold address >> 4, and every stage address fits, so the add never carries).
        const uint32_t s0 = smem_u32(smem);
        const uint64_t a_desc0 = smem_desc(s0, 16, 1024, 2);
        const uint64_t b_desc0 = smem_desc(s0 + A_BYTES, 16, 1024, 2);
        uint32_t it = 0, tile_it = 0;
        bool ok = true;
        // MMA a (K = 64) of a stage: NVFP4 reads the 4 scales of each row from column
        // group a; MXFP4 reads 2 scales, from column group a/2 at byte 2*(a%2)
        auto mma = [&](uint32_t d, uint64_t ad, uint64_t bd, uint32_t t_sfa, uint32_t t_sfb,
                       int a, uint32_t acc) {
          if constexpr (SFV == 16) {
            const uint32_t sfa = t_sfa + a * 4, sfb = t_sfb + a * (BN / 32);
            if constexpr (PAIR) tc_mma_nvf4_pair_warp(d, ad, bd, C::IDESC, sfa, sfb, acc);
            else tc_mma_nvf4_warp(d, ad, bd, C::IDESC, sfa, sfb, acc);
          } else {
            const uint32_t byte = 2u * static_cast<uint32_t>(a & 1);
            const uint32_t sfa = (t_sfa + (a >> 1) * 4) | (byte << 30);
            const uint32_t sfb = (t_sfb + (a >> 1) * (BN / 32)) | (byte << 30);
            const uint32_t idesc = idesc_sf_byte(C::IDESC, byte);
            if constexpr (PAIR) tc_mma_mxf4_pair_warp(d, ad, bd, idesc, sfa, sfb, acc);
            else tc_mma_mxf4_warp(d, ad, bd, idesc, sfa, sfb, acc);
          }
        };
        auto commit_all = [&](const uint64_t* bar) {  // arrive on `bar` of every CTA
          if constexpr (PAIR) {
            tc_commit_pair_warp(smem_u32(bar));
            tc_commit_pair_warp(at_peer(bar));
          } else {
            tc_commit_warp(smem_u32(bar));
          }
        };
        auto wait_all = [&](const uint64_t* bar, uint32_t parity) {
          return __all_sync(0xffffffffu, mbar_wait_bounded(smem_u32(bar), parity, &abort_flag));
        };
        for (int t = cluster_id; t < total && ok; t += num_clusters, ++tile_it) {
          const int b = tile_it % ACC_BUFS;
          if (!wait_all(&bar_acc_empty[b], ((tile_it / ACC_BUFS) & 1u) ^ 1u)) {
            ok = false;
            break;
          }
          const uint32_t d_tmem = tmem + b * BN;
          int kb_lo, kb_hi;
          k_range(t, kb_lo, kb_hi);
          // The tensor pipe keeps almost no queue ahead of the issuing warp, so a wait between
          // two stages adds to every stage (measured: 128 cycles per MMA with no waits, ~160 with
          // one wait per 4 MMAs).  Each stage's one barrier is therefore waited for while the
          // previous stage's MMAs still run: the first stage of a tile here, every later one
          // between the last two MMAs of the stage before it.
          auto stage_ready = [&](uint32_t j) {
            return wait_all(&bar_full[j % STAGES], (j / STAGES) & 1u);
          };
          if (kb_lo < kb_hi && !stage_ready(it)) {
            ok = false;
            break;
          }
          for (int kb = kb_lo; kb < kb_hi; ++kb, ++it) {
            const int s = it % STAGES;
            tc_fence_after();
            const uint64_t so = static_cast<uint64_t>(s) * (C::AB_BYTES >> 4);
            const uint32_t t_sfa = tmem + C::TM_SFA + s * C::SFA_COLS;
            const uint32_t t_sfb = tmem + C::TM_SFB + s * C::SFB_COLS;
            const uint32_t first = kb == kb_lo ? 0u : 1u;
            // scales of this stage are already in tensor memory (scale-factor warps)
            const int n_mma = min(4, mma_k - kb * 4);
            const bool more = kb + 1 < kb_hi;
            if (n_mma == 4) {
  #pragma unroll
              for (int a = 0; a < 3; ++a)
                mma(d_tmem, a_desc0 + so + 2 * a, b_desc0 + so + 2 * a, t_sfa, t_sfb, a,
                    a == 0 ? first : 1u);
              if (more && !stage_ready(it + 1)) ok = false;
              mma(d_tmem, a_desc0 + so + 6, b_desc0 + so + 6, t_sfa, t_sfb, 3, 1u);
            } else {
              for (int a = 0; a < n_mma; ++a)
                mma(d_tmem, a_desc0 + so + 2 * a, b_desc0 + so + 2 * a, t_sfa, t_sfb, a,
                    a == 0 ? first : 1u);
              if (more && !stage_ready(it + 1)) ok = false;
            }
            commit_all(&bar_empty[s]);
            if (!ok) break;
          }
          if (!ok) break;
          commit_all(&bar_acc_full[b]);
        }
        // all MMAs issued by this warp complete before tensor memory is freed
        if constexpr (PAIR) tc_commit_pair_warp(smem_u32(&bar_drain));
        else tc_commit_warp(smem_u32(&bar_drain));
        volatile int never = 0;
        mbar_wait_bounded(smem_u32(&bar_drain), 0, &never);
      }
      __syncwarp();
  }
  } else if (warp >= SF_WARP0) {
    regs_release_to<REGS_OTHER>();
    // =========================== scale-factor warps ===========================
    // warp (SF_WARP0 + q) writes lane quadrant q of each stage's scale-factor columns
    const uint32_t lane_base = static_cast<uint32_t>((warp & 3) * 32) << 16;
    uint32_t it = 0;
    bool ok = true;
    for (int t = cluster_id; t < total && ok; t += num_clusters) {
      int kb_lo, kb_hi;
      k_range(t, kb_lo, kb_hi);
      for (int kb = kb_lo; kb < kb_hi; ++kb, ++it) {
        const int s = it % STAGES;
        const uint32_t ph = (it / STAGES) & 1u;
        const int j = it % C::SF_STAGES;
        // the stage's scales are in the scale ring, and its tensor-memory columns are free once
        // the MMAs of the stage's previous use have completed (the A/B producer waits the same)
        if (!mbar_wait_bounded(smem_u32(&bar_sfin[j]), (it / C::SF_STAGES) & 1u, &abort_flag) ||
            !mbar_wait_bounded(smem_u32(&bar_empty[s]), ph ^ 1u, &abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint8_t* st = smem + C::SF_OFFSET + j * C::SF_BYTES;
        sf_rows128_to_tmem<NA>(tmem + lane_base + C::TM_SFA + s * C::SFA_COLS, st, lane);
        if constexpr (BN == 256)
          sf_rows256_to_tmem<NA>(tmem + lane_base + C::TM_SFB + s * C::SFB_COLS,
                                 st + C::SFA_BYTES, lane);
        else
          sf_rows128_to_tmem<NA>(tmem + lane_base + C::TM_SFB + s * C::SFB_COLS,
                                 st + C::SFA_BYTES, lane);
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(smem_u32(&bar_sfempty[j]));
          if constexpr (PAIR) mbar_arrive_cluster(at_leader(&bar_full[s]));
          else mbar_arrive(smem_u32(&bar_full[s]));
        }
      }
    }
  } else {
    regs_raise_to<REGS_EPI>();
    // =========================== epilogue ===========================
    // Two warps per tensor-memory lane quadrant (a warp may only read lanes 32*(warp%4)..+31);
    // `half` splits the tile's columns between them.
    const int q = warp & 3;
    const int half = (warp - EPI_WARP0) >> 2;
    uint32_t tile_it = 0;
    for (int t = cluster_id; t < total; t += num_clusters, ++tile_it) {
      const Tile tl = decode_tile<CTAS, slice_major<MODE>()>(t / KS, tile_start, seg, E,
                                                                args.n_tiles);
      const int b = tile_it % ACC_BUFS;
      // Everything the epilogue reads besides the accumulator (row map, routing weight, global
      // scales) is fetched before waiting for it, so that these loads do not hold up handing
      // tensor memory back to the MMA warp.
      const int m_cta = tl.m0 + BM * rank;
      const bool rows_valid = m_cta < seg[tl.e + 1];  // false: a pair's half past the segment
      // MXFP4 has no global scales: its block scales carry the whole range
      const float alpha =
          SFV == 32 ? 1.0f : 1.0f / (__ldg(args.gs_a) * __ldg(args.gs_b + tl.e));
      const int64_t row = m_cta + q * 32 + lane;
      // rows of the row map that are padding produce nothing; skip groups of 32 of them
      int slot = rows_valid ? 0 : -1;
      if (MODE == L1_SWIGLU || is_l2<MODE>()) {
        if (rows_valid && args.row_slot != nullptr) slot = __ldg(args.row_slot + row);
      }
      const float row_weight = (is_l2<MODE>() && slot >= 0) ? __ldg(args.row_w + row) : 0.0f;
      const float gs_h = MODE == L1_SWIGLU ? __ldg(args.gs_h) : 0.0f;
      if (!mbar_wait_bounded(smem_u32(&bar_acc_full[b]), (tile_it / ACC_BUFS) & 1u, &abort_flag))
        break;
      tc_fence_after();
      const uint32_t t_row = tmem + b * BN + (static_cast<uint32_t>(q * 32) << 16);
      const bool live = __any_sync(0xffffffffu, slot >= 0);
      bool released = false;  // accumulator buffer b handed back to the MMA warp
      auto release = [&] {
        tc_fence_before();
        __syncwarp();
        if (lane == 0) {
          if constexpr (PAIR) mbar_arrive_cluster(at_leader(&bar_acc_empty[b]));
          else mbar_arrive(smem_u32(&bar_acc_empty[b]));
        }
        released = true;
      };

      if (MODE == L1_SWIGLU) {
        if (live) {
          const int I = args.I;
          constexpr int n_chunks = BN / 128;  // 64-column chunks per warp
          uint8_t* hrow = args.h + row * (I / 2) + tl.nt * (BN / 4);
          // the warp's whole accumulator slice into registers, then tensor memory goes back to
          // the MMA warp and the next tile's MMAs overlap this epilogue
          uint32_t v[n_chunks][2][32];
#pragma unroll
          for (int cc = 0; cc < n_chunks; ++cc) {
            tmem_ld32(t_row + 64 * (half * n_chunks + cc), v[cc][0]);
            tmem_ld32(t_row + 64 * (half * n_chunks + cc) + 32, v[cc][1]);
          }
          tmem_wait_ld();
          release();
          uint32_t sfw = 0u;
          // what the epilogue learns about h on real rows (padding rows compute garbage)
          const bool real = slot >= 0;
          float h_max = 0.0f;
          uint32_t n_sat = 0u, n_under = 0u;
#pragma unroll
          for (int cc = 0; cc < n_chunks; ++cc) {
            // h features 32c..32c+31 of the tile live in accumulator columns 64c..64c+63 as two
            // 32-column blocks, each 16 gate columns followed by the 16 matching up columns
            const int c = half * n_chunks + cc;
            float hv[32];
#pragma unroll
            for (int i = 0; i < 16; ++i) {
              // h = silu(g) * u = g * u / (1 + e^-g), g and u de-scaled by alpha
              const float g0 = __uint_as_float(v[cc][0][i]) * alpha;
              const float u0 = __uint_as_float(v[cc][0][16 + i]) * alpha;
              const float g1 = __uint_as_float(v[cc][1][i]) * alpha;
              const float u1 = __uint_as_float(v[cc][1][16 + i]) * alpha;
              hv[i] = __fdividef(g0 * u0, 1.0f + __expf(-g0));
              hv[16 + i] = __fdividef(g1 * u1, 1.0f + __expf(-g1));
            }
            uint32_t packed[4];
#pragma unroll
            for (int bb = 0; bb < 2; ++bb) {
              float amax = 0.0f;
#pragma unroll
              for (int i = 0; i < 16; ++i) amax = fmaxf(amax, fabsf(hv[16 * bb + i]));
              float rcp, sc;
              const uint32_t sb = nvfp4_block_scale(amax, gs_h, rcp, sc);
              packed[2 * bb] = nvfp4_pack8(hv + 16 * bb, rcp);
              packed[2 * bb + 1] = nvfp4_pack8(hv + 16 * bb + 8, rcp);
              sfw |= sb << (8 * (2 * cc + bb));  // this warp's scale columns, in order
              h_max = fmaxf(h_max, amax);
              n_sat += sc > 448.0f ? 1u : 0u;
              n_under += (amax > 0.0f && sb == 0u) ? 1u : 0u;
            }
            *reinterpret_cast<uint4*>(hrow + 16 * c) =
                make_uint4(packed[0], packed[1], packed[2], packed[3]);
            if (args.h32 != nullptr && real) {
              float4* dst =
                  reinterpret_cast<float4*>(args.h32 + row * I + tl.nt * (BN / 2) + 32 * c);
#pragma unroll
              for (int q4 = 0; q4 < 8; ++q4)
                dst[q4] = make_float4(hv[4 * q4], hv[4 * q4 + 1], hv[4 * q4 + 2], hv[4 * q4 + 3]);
            }
          }
          if (args.h_stats != nullptr) {
            // |h| >= 0, so the float bits order like the values; one atomic per warp and tile
            const uint32_t hb = __reduce_max_sync(0xffffffffu, real ? __float_as_uint(h_max) : 0u);
            const uint32_t ns = __reduce_add_sync(0xffffffffu, real ? n_sat : 0u);
            const uint32_t nu = __reduce_add_sync(0xffffffffu, real ? n_under : 0u);
            if (lane == 0) {
              if (hb) atomicMax(args.h_stats, hb);
              if (ns) atomicAdd(args.h_stats + 1, ns);
              if (nu) atomicAdd(args.h_stats + 2, nu);
            }
          }
          // this warp's 2 * n_chunks scale columns are consecutive bytes of one 4-byte group of
          // the tiled layout
          const int sc0 = tl.nt * (BN / 32) + half * (BN / 64);
          uint8_t* sfp = args.sfh + sf_offset(row, sc0, I / 16);
          if constexpr (n_chunks == 2) *reinterpret_cast<uint32_t*>(sfp) = sfw;
          else *reinterpret_cast<uint16_t*>(sfp) = static_cast<uint16_t>(sfw);
        }
      } else if (is_l2<MODE>()) {
        // this row's weighted expert output goes to its slot's row of ys (L2_ROWS; the combine
        // kernel then sums a token's k slot rows) or is added into its token's row (L2_ATOMIC)
        if (live) {
          if (slot >= args.S) {
            report(args.status, NVFP4_DEVERR_BAD_INDEX);
            slot = -1;
          }
          const float scale = alpha * (slot >= 0 ? row_weight : 0.0f);
          const int H = args.N;
          const int c_lo = (BN / 64) * half;
          // the warp's whole slice (BN/2 columns) is read from tensor memory first; then the
          // accumulator goes back to the MMA warp and the stores overlap the next tile's MMAs.
          // No shared-memory staging.  Each lane holds 32 consecutive values of its own row
          // per 32-column chunk (8 pieces of 4); the 8 lanes of an octet transpose those pieces
          // among themselves with register shuffles (three exchange rounds), after which lane c
          // holds piece c of each of the octet's 8 rows.  Every vector store (L2_ROWS: the
          // slot's row) or reduction (L2_ATOMIC: the token's row) of the warp then covers
          // 4 rows x 128 contiguous bytes, the shape the SM -> L2 path takes fastest (about
          // 1.7x the rate of 16 rows x 32 bytes).
          const int tok = slot < 0 ? -1 : MODE == L2_ATOMIC ? slot / args.k : slot;
          int tok_r[8];  // the tokens of the octet's 8 rows
#pragma unroll
          for (int i = 0; i < 8; ++i) tok_r[i] = __shfl_sync(0xffffffffu, tok, (lane & ~7) | i);
          const int piece = lane & 7;
          uint32_t v[BN / 64][32];
#pragma unroll
          for (int j = 0; j < BN / 64; ++j) tmem_ld32(t_row + 32 * (c_lo + j), v[j]);
          tmem_wait_ld();
          release();
#pragma unroll
          for (int j = 0; j < BN / 64; ++j) {
#pragma unroll
            for (int i = 0; i < 32; ++i)
              v[j][i] = __float_as_uint(__uint_as_float(v[j][i]) * scale);
            // round m: a lane with lane bit m set keeps the pieces whose index has bit m set
            // and takes its partner's pieces with bit m set in place of its own with bit m clear;
            // the partner does the converse
#pragma unroll
            for (int m = 4; m >= 1; m >>= 1) {
              const bool hi = (lane & m) != 0;
#pragma unroll
              for (int j0 = 0; j0 < 8; ++j0) {
                if (j0 & m) continue;
                const int j1 = j0 | m;
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                  const uint32_t snd = hi ? v[j][4 * j0 + e] : v[j][4 * j1 + e];
                  const uint32_t rcv = __shfl_xor_sync(0xffffffffu, snd, m);
                  if (hi) v[j][4 * j0 + e] = rcv;
                  else v[j][4 * j1 + e] = rcv;
                }
              }
            }
            const int64_t col = (int64_t)tl.nt * BN + 32 * (c_lo + j) + 4 * piece;
#pragma unroll
            for (int i = 0; i < 8; ++i) {
              if (tok_r[i] < 0) continue;
              const float4 val =
                  make_float4(__uint_as_float(v[j][4 * i]), __uint_as_float(v[j][4 * i + 1]),
                              __uint_as_float(v[j][4 * i + 2]), __uint_as_float(v[j][4 * i + 3]));
              float* dst = args.ys + (int64_t)tok_r[i] * H + col;
              if constexpr (MODE == L2_ATOMIC) red_add_v4(dst, val);
              else *reinterpret_cast<float4*>(dst) = val;
            }
          }
        }
      } else if (rows_valid) {
        const int N = args.N;
        auto emit = [&](int c, const uint32_t (&v)[32]) {
          if (row >= args.out_rows) return;
          const int64_t col = (int64_t)tl.nt * BN + 32 * c;
          if (MODE == PLAIN_F32) {
            float* base = static_cast<float*>(args.out) + (int64_t)(t % KS) * args.split_stride;
            float4* o = reinterpret_cast<float4*>(base + row * N + col);
#pragma unroll
            for (int i = 0; i < 8; ++i)
              o[i] = make_float4(__uint_as_float(v[4 * i]) * alpha,
                                 __uint_as_float(v[4 * i + 1]) * alpha,
                                 __uint_as_float(v[4 * i + 2]) * alpha,
                                 __uint_as_float(v[4 * i + 3]) * alpha);
          } else {
            uint4* o = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(args.out) + row * N + col);
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              uint32_t wds[4];
#pragma unroll
              for (int j = 0; j < 4; ++j) {
                const __nv_bfloat162 p = __floats2bfloat162_rn(
                    __uint_as_float(v[8 * i + 2 * j]) * alpha,
                    __uint_as_float(v[8 * i + 2 * j + 1]) * alpha);
                wds[j] = *reinterpret_cast<const uint32_t*>(&p);
              }
              o[i] = make_uint4(wds[0], wds[1], wds[2], wds[3]);
            }
          }
        };
        const int c_lo = (BN / 64) * half;
        uint32_t v[BN / 64][32];
#pragma unroll
        for (int j = 0; j < BN / 64; ++j) tmem_ld32(t_row + 32 * (c_lo + j), v[j]);
        tmem_wait_ld();
        release();
#pragma unroll
        for (int j = 0; j < BN / 64; ++j) emit(c_lo + j, v[j]);
      }
      if (!released) release();
    }
  }

  __syncwarp();
  tc_fence_before();
  __syncthreads();
  // a pair: the leader's MMAs (which write both CTAs' tensor memory) are drained and no remote
  // arrival or copy is still headed for the other CTA before either frees or exits
  if constexpr (PAIR) cluster_sync();
  tc_fence_after();
  if (warp == 2) {
    if constexpr (PAIR) tmem_dealloc_pair(tmem, TMEM_COLS);
    else tmem_dealloc(tmem, TMEM_COLS);
  }
  if (tid == 0 && abort_flag) report(args.status, NVFP4_DEVERR_TIMEOUT);
}

// ------------------------------------------------------------------------------ host side

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault,
                                         &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// 2D byte tensor [rows][row_bytes], box 128 bytes x box_rows rows, 128-byte swizzle.
bool make_map(CUtensorMap* m, const void* base, uint64_t row_bytes, uint64_t rows,
              uint32_t box_rows = 128) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {row_bytes, rows};
  cuuint64_t strides[1] = {row_bytes};
  cuuint32_t box[2] = {128, box_rows};
  cuuint32_t estr[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

int num_sms() {
  int dev = 0, n = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
  return n > 0 ? n : 148;
}

// Pair tiles (CTAS = 2) from this many 128-row blocks of capacity per expert on average.  A pair
// tile covers 256 rows, so an expert with an odd number of blocks computes a half tile that
// nobody writes; with ~2.5 blocks per expert that waste (about 20%) outweighs the pair's smaller
// operand traffic, with 16 blocks per expert the pair is ahead.
constexpr int kPairMinBlocksPerExpert = 8;
// At most this many K ranges per tile of a dense product.
constexpr int kMaxKSplits = 16;

template <int MODE, int CTAS, int SFV>
nvfp4_status_t launch_cfg(const CUtensorMap& ma, const CUtensorMap& mb, const GemmArgs& args,
                          cudaStream_t s) {
  constexpr int smem = TileCfg<MODE, CTAS, SFV>::SMEM_BYTES;
  auto kernel = grouped_gemm_kernel<MODE, CTAS, SFV>;
  if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) !=
      cudaSuccess)
    return check_launch("cudaFuncSetAttribute");
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[1];
  cfg.blockDim = dim3(NUM_THREADS);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  if (CTAS == 1) {
    cfg.gridDim = dim3(num_sms());
  } else {
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = CTAS;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cfg.gridDim = dim3(num_sms());
    int clusters = 0;  // persistent: as many pairs as can be resident at once
    if (cudaOccupancyMaxActiveClusters(&clusters, kernel, &cfg) != cudaSuccess || clusters <= 0) {
      (void)cudaGetLastError();
      clusters = num_sms() / CTAS;
    }
    cfg.gridDim = dim3(clusters * CTAS);
  }
  if (cudaLaunchKernelEx(&cfg, kernel, ma, mb, args) != cudaSuccess)
    return check_launch("grouped_gemm_kernel");
  return check_launch("grouped_gemm_kernel");
}

template <int MODE, int SFV = 16>
nvfp4_status_t launch(const uint8_t* a, const uint8_t* b, int64_t b_rows, GemmArgs args,
                      cudaStream_t s) {
  CUtensorMap ma, mb;
  if (!make_map(&ma, a, args.K / 2, args.R_max) || !make_map(&mb, b, args.K / 2, b_rows)) {
    set_last_error("cuTensorMapEncodeTiled failed");
    return NVFP4_ERR_CUDA;
  }
  if constexpr (TileCfg<MODE, 1>::BN == 256) {
    if (args.R_max >= (int64_t)kPairMinBlocksPerExpert * BM * args.E)
      return launch_cfg<MODE, 2, SFV>(ma, mb, args, s);
  }
  return launch_cfg<MODE, 1, SFV>(ma, mb, args, s);
}

// out[t] = sum over the token's slots j (in order, skipping dropped ones) of ys[t*k + j]; FP32
// adds in a fixed order, so the output is bitwise reproducible.  8 columns per thread.
__global__ void combine_kernel(const float* __restrict__ ys, const int32_t* __restrict__ dst_row,
                               int T, int k, int H, float* __restrict__ out_f32,
                               __nv_bfloat16* __restrict__ out_bf16) {
  const int n8 = H / 8;
  const int64_t total = (int64_t)T * n8;
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < total;
       i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t t = i / n8;
    const int c = static_cast<int>(i - t * n8) * 8;
    float4 a = make_float4(0.f, 0.f, 0.f, 0.f), b = a;
    for (int j = 0; j < k; ++j) {
      if (__ldg(dst_row + t * k + j) < 0) continue;
      const float4* p = reinterpret_cast<const float4*>(ys + (t * k + j) * H + c);
      const float4 p0 = __ldg(p), p1 = __ldg(p + 1);
      a.x += p0.x; a.y += p0.y; a.z += p0.z; a.w += p0.w;
      b.x += p1.x; b.y += p1.y; b.z += p1.z; b.w += p1.w;
    }
    if (out_f32 != nullptr) {
      float4* o = reinterpret_cast<float4*>(out_f32 + t * H + c);
      o[0] = a;
      o[1] = b;
    }
    if (out_bf16 != nullptr) {
      const __nv_bfloat162 q0 = __floats2bfloat162_rn(a.x, a.y), q1 = __floats2bfloat162_rn(a.z, a.w),
                           q2 = __floats2bfloat162_rn(b.x, b.y), q3 = __floats2bfloat162_rn(b.z, b.w);
      uint4 o;
      o.x = *reinterpret_cast<const uint32_t*>(&q0);
      o.y = *reinterpret_cast<const uint32_t*>(&q1);
      o.z = *reinterpret_cast<const uint32_t*>(&q2);
      o.w = *reinterpret_cast<const uint32_t*>(&q3);
      *reinterpret_cast<uint4*>(out_bf16 + t * H + c) = o;
    }
  }
}

// out[i] = bf16(acc[i]) (round to nearest even), 8 elements per thread.
__global__ void __launch_bounds__(256) to_bf16_kernel(const float* __restrict__ acc, int64_t n8,
                                                      __nv_bfloat16* __restrict__ out) {
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n8;
       i += (int64_t)gridDim.x * blockDim.x) {
    const float4* p = reinterpret_cast<const float4*>(acc + 8 * i);
    const float4 a = __ldg(p), b = __ldg(p + 1);
    const __nv_bfloat162 q0 = __floats2bfloat162_rn(a.x, a.y), q1 = __floats2bfloat162_rn(a.z, a.w),
                         q2 = __floats2bfloat162_rn(b.x, b.y), q3 = __floats2bfloat162_rn(b.z, b.w);
    uint4 o;
    o.x = *reinterpret_cast<const uint32_t*>(&q0);
    o.y = *reinterpret_cast<const uint32_t*>(&q1);
    o.z = *reinterpret_cast<const uint32_t*>(&q2);
    o.w = *reinterpret_cast<const uint32_t*>(&q3);
    reinterpret_cast<uint4*>(out)[i] = o;
  }
}

// out[i] = bf16 of the sum over the K ranges r = 0 .. ks-1 of part[r * n + i], added in that
// order (reproducible).  4 consecutive outputs per thread, all ks loads in flight at once.
__global__ void __launch_bounds__(256) splitk_reduce_kernel(const float* __restrict__ part, int ks,
                                                            int64_t n,
                                                            __nv_bfloat16* __restrict__ out) {
  for (int64_t i = (blockIdx.x * (int64_t)blockDim.x + threadIdx.x) * 4; i < n;
       i += (int64_t)gridDim.x * blockDim.x * 4) {
    float4 p[kMaxKSplits];
#pragma unroll
    for (int r = 0; r < kMaxKSplits; ++r)
      if (r < ks) p[r] = __ldg(reinterpret_cast<const float4*>(part + r * n + i));
    float4 a = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int r = 0; r < kMaxKSplits; ++r) {
      if (r < ks) {
        a.x += p[r].x; a.y += p[r].y; a.z += p[r].z; a.w += p[r].w;
      }
    }
    const __nv_bfloat162 q0 = __floats2bfloat162_rn(a.x, a.y), q1 = __floats2bfloat162_rn(a.z, a.w);
    uint2 o;
    o.x = *reinterpret_cast<const uint32_t*>(&q0);
    o.y = *reinterpret_cast<const uint32_t*>(&q1);
    *reinterpret_cast<uint2*>(out + i) = o;
  }
}

bool ok_ptr(const void* p) { return p != nullptr && aligned16(p); }

}  // namespace

// K ranges of a dense product: split while the tiles fill at most half of the SMs and the
// caller's partial-sum buffer holds them; each range keeps at least one 256-element stage.
int dense_k_splits(int64_t M, int N, int K, int sms, int64_t part_floats) {
  const int64_t Mp = round_up(M, 128);
  const int64_t tiles = (Mp / BM) * (N / TileCfg<PLAIN_F32, 1>::BN);
  if (M <= 0 || tiles <= 0 || Mp >= (int64_t)kPairMinBlocksPerExpert * BM || tiles * 2 > sms)
    return 1;
  int64_t ks = sms / tiles;
  ks = ks < kMaxKSplits ? ks : kMaxKSplits;
  const int64_t nk = (K + 255) / 256;
  ks = ks < nk ? ks : nk;
  const int64_t fit = part_floats / (M * (int64_t)N);
  ks = ks < fit ? ks : fit;
  return ks >= 2 ? static_cast<int>(ks) : 1;
}

int device_sms() { return num_sms(); }

// FP32 partial products of a dense C = A B^T over ks K ranges, plane r = range r, M rows of N
// floats each, for a consumer that finishes the sum itself.  ks comes from dense_k_splits (so
// ks <= K/256 and the rows stay below the pair-tile threshold).
nvfp4_status_t gemm_dense_parts(const uint8_t* a, const uint8_t* sfa, const float* gs_a,
                                const uint8_t* b, const uint8_t* sfb, const float* gs_b,
                                int64_t M, int N, int K, int ks, float* part, int32_t* status,
                                cudaStream_t s) {
  if (M == 0) return NVFP4_OK;
  GemmArgs g{};
  g.sfa = sfa; g.sfb = sfb; g.gs_a = gs_a; g.gs_b = gs_b; g.offs = nullptr;
  g.E = 1; g.N = N; g.K = K; g.n_tiles = N / TileCfg<PLAIN_F32, 1>::BN; g.R_max = round_up(M, 128);
  g.out_rows = M; g.status = status; g.out = part; g.k_splits = ks;
  g.split_stride = M * (int64_t)N;
  return launch<PLAIN_F32>(a, b, N, g, s);
}

// Dense C = A B^T for A NVFP4 [round_up(M, 128)][K] (rows past M are padding that is never
// stored) and B NVFP4 [N][K]: one segment, no offsets.  With K splits the ranges' FP32 partial
// products go to `part` and splitk_reduce_kernel adds them; otherwise the bf16 result is stored
// straight from the epilogue.
nvfp4_status_t gemm_dense(const uint8_t* a, const uint8_t* sfa, const float* gs_a,
                          const uint8_t* b, const uint8_t* sfb, const float* gs_b, int64_t M, int N,
                          int K, void* out_bf16, float* part, int64_t part_floats, int32_t* status,
                          cudaStream_t s) {
  if (M == 0) return NVFP4_OK;
  const int64_t Mp = round_up(M, 128);
  const int ks = dense_k_splits(M, N, K, num_sms(), part != nullptr ? part_floats : 0);
  GemmArgs g{};
  g.sfa = sfa; g.sfb = sfb; g.gs_a = gs_a; g.gs_b = gs_b; g.offs = nullptr;
  g.E = 1; g.N = N; g.K = K; g.n_tiles = N / TileCfg<PLAIN_F32, 1>::BN; g.R_max = Mp;
  g.out_rows = M; g.status = status;
  if (ks == 1) {
    g.out = out_bf16;
    g.k_splits = 1;
    return launch<PLAIN_BF16>(a, b, N, g, s);
  }
  g.out = part;
  g.k_splits = ks;
  g.split_stride = M * (int64_t)N;
  nvfp4_status_t st = launch<PLAIN_F32>(a, b, N, g, s);
  if (st != NVFP4_OK) return st;
  const int64_t n = M * (int64_t)N;
  const int64_t want = (n / 4 + 255) / 256;
  splitk_reduce_kernel<<<(unsigned)(want < 148 * 8 ? want : 148 * 8), 256, 0, s>>>(
      part, ks, n, static_cast<__nv_bfloat16*>(out_bf16));
  return check_launch("splitk_reduce_kernel");
}

nvfp4_status_t gemm_plain(const uint8_t* a, const uint8_t* sfa, const float* gs_a, const uint8_t* b,
                          const uint8_t* sfb, const float* gs_b, const int32_t* offs, int E, int N,
                          int K, int64_t R_max, void* out, int out_dtype, int32_t* status,
                          cudaStream_t s) {
  GemmArgs g{};
  g.sfa = sfa; g.sfb = sfb; g.gs_a = gs_a; g.gs_b = gs_b; g.offs = offs;
  g.E = E; g.N = N; g.K = K; g.n_tiles = N / TileCfg<PLAIN_F32, 1>::BN; g.R_max = R_max; g.out = out;
  g.status = status; g.out_rows = R_max; g.k_splits = 1;
  const int64_t b_rows = (int64_t)E * N;
  return out_dtype == 0 ? launch<PLAIN_F32>(a, b, b_rows, g, s) : launch<PLAIN_BF16>(a, b, b_rows, g, s);
}

nvfp4_status_t gemm_l1(const uint8_t* a, const uint8_t* sfa, const float* gs_a, const uint8_t* w1,
                       const uint8_t* sfw1, const float* gs_w1, const int32_t* offs,
                       const int32_t* row_slot, int E, int H, int I, int64_t R_max,
                       const float* gs_h, uint8_t* h, uint8_t* sfh, float* h32,
                       uint32_t* h_stats, int32_t* status, cudaStream_t s) {
  GemmArgs g{};
  g.sfa = sfa; g.sfb = sfw1; g.gs_a = gs_a; g.gs_b = gs_w1; g.offs = offs;
  g.E = E; g.N = 2 * I; g.K = H; g.n_tiles = 2 * I / TileCfg<L1_SWIGLU, 1>::BN; g.R_max = R_max;
  g.gs_h = gs_h; g.h = h; g.sfh = sfh; g.I = I; g.row_slot = row_slot; g.status = status;
  g.h32 = h32; g.h_stats = h_stats;
  g.out_rows = R_max; g.k_splits = 1;
  return launch<L1_SWIGLU>(a, w1, (int64_t)E * 2 * I, g, s);
}

nvfp4_status_t gemm_l2(const uint8_t* h, const uint8_t* sfh, const float* gs_h, const uint8_t* w2,
                       const uint8_t* sfw2, const float* gs_w2, const int32_t* offs,
                       const int32_t* row_slot, const float* row_w, const int32_t* dst_row, int E,
                       int H, int I, int T, int k, int64_t R_max, float* ys, float* out_f32,
                       void* out_bf16, bool atomic, int32_t* status, cudaStream_t s) {
  if (T == 0) return NVFP4_OK;
  GemmArgs g{};
  g.sfa = sfh; g.sfb = sfw2; g.gs_a = gs_h; g.gs_b = gs_w2; g.offs = offs;
  g.E = E; g.N = H; g.K = I; g.R_max = R_max; g.n_tiles = H / TileCfg<L2_ROWS, 1>::BN;
  g.row_slot = row_slot; g.row_w = row_w; g.ys = ys; g.S = T * k; g.k = k; g.status = status;
  g.out_rows = R_max; g.k_splits = 1;
  if (atomic) {
    // the token rows are summed in place: in out_f32 when the caller wants it, else in ys
    float* acc = out_f32 != nullptr ? out_f32 : ys;
    const int64_t n = (int64_t)T * H;
    if (cudaMemsetAsync(acc, 0, n * sizeof(float), s) != cudaSuccess)
      return check_launch("cudaMemsetAsync(accumulator)");
    g.ys = acc;
    nvfp4_status_t st = launch<L2_ATOMIC>(h, w2, (int64_t)E * H, g, s);
    if (st != NVFP4_OK || out_bf16 == nullptr) return st;
    const int64_t want = (n / 8 + 255) / 256;
    to_bf16_kernel<<<(unsigned)(want < 148 * 16 ? want : 148 * 16), 256, 0, s>>>(
        acc, n / 8, static_cast<__nv_bfloat16*>(out_bf16));
    return check_launch("to_bf16_kernel");
  }
  nvfp4_status_t st = launch<L2_ROWS>(h, w2, (int64_t)E * H, g, s);
  if (st != NVFP4_OK) return st;
  const int64_t n = (int64_t)T * H / 8;
  const int64_t want = (n + 255) / 256;
  combine_kernel<<<(unsigned)(want < 148 * 16 ? want : 148 * 16), 256, 0, s>>>(
      ys, dst_row, T, k, H, out_f32, static_cast<__nv_bfloat16*>(out_bf16));
  return check_launch("combine_kernel");
}

// The L2 form for a batch: slot rows summed in slot order (deterministic) for few rows per expert
// or on request; otherwise added into token rows as they are produced (no per-slot round trip).
bool l2_use_atomic(int T, int k, int E, bool deterministic) {
  return !deterministic && (int64_t)T * k >= (int64_t)kL2AtomicMinRowsPerExpert * E;
}

}  // namespace nvfp4

using namespace nvfp4;

extern "C" nvfp4_status_t nvfp4_grouped_gemm(const uint8_t* a, const uint8_t* sfa,
                                             const float* gs_a, const uint8_t* b,
                                             const uint8_t* sfb, const float* gs_b,
                                             const int32_t* offs, int E, int N, int K,
                                             int64_t R_max, void* out, int out_dtype,
                                             int32_t* dev_status, nvfp4_stream_t stream) {
  if (E < 1 || E > MAX_E || N <= 0 || K <= 0 || R_max < 0) return NVFP4_ERR_INVALID_ARG;
  if (K % 64 || N % TileCfg<PLAIN_F32, 1>::BN || R_max % 128) return NVFP4_ERR_UNSUPPORTED_SHAPE;
  if (out_dtype != 0 && out_dtype != 1) return NVFP4_ERR_INVALID_ARG;
  if (!gs_a || !gs_b || !offs) return NVFP4_ERR_INVALID_ARG;
  if (R_max == 0) return NVFP4_OK;
  if (!ok_ptr(a) || !ok_ptr(sfa) || !ok_ptr(b) || !ok_ptr(sfb) || !ok_ptr(out))
    return (a && sfa && b && sfb && out) ? NVFP4_ERR_MISALIGNED : NVFP4_ERR_INVALID_ARG;
  return gemm_plain(a, sfa, gs_a, b, sfb, gs_b, offs, E, N, K, R_max, out, out_dtype, dev_status,
                    reinterpret_cast<cudaStream_t>(stream));
}

extern "C" nvfp4_status_t mxfp4_grouped_gemm(const uint8_t* a, const uint8_t* sfa,
                                             const uint8_t* b, const uint8_t* sfb,
                                             const int32_t* offs, int E, int N, int K,
                                             int64_t R_max, void* out, int out_dtype,
                                             int32_t* dev_status, nvfp4_stream_t stream) {
  if (E < 1 || E > MAX_E || N <= 0 || K <= 0 || R_max < 0) return NVFP4_ERR_INVALID_ARG;
  if (K % 128 || N % TileCfg<PLAIN_F32, 1, 32>::BN || R_max % 128)
    return NVFP4_ERR_UNSUPPORTED_SHAPE;
  if (out_dtype != 0 && out_dtype != 1) return NVFP4_ERR_INVALID_ARG;
  if (!offs) return NVFP4_ERR_INVALID_ARG;
  if (R_max == 0) return NVFP4_OK;
  if (!ok_ptr(a) || !ok_ptr(sfa) || !ok_ptr(b) || !ok_ptr(sfb) || !ok_ptr(out))
    return (a && sfa && b && sfb && out) ? NVFP4_ERR_MISALIGNED : NVFP4_ERR_INVALID_ARG;
  GemmArgs g{};
  g.sfa = sfa; g.sfb = sfb; g.gs_a = nullptr; g.gs_b = nullptr; g.offs = offs;
  g.E = E; g.N = N; g.K = K; g.n_tiles = N / TileCfg<PLAIN_F32, 1, 32>::BN; g.R_max = R_max;
  g.out = out; g.status = dev_status; g.out_rows = R_max; g.k_splits = 1;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const int64_t b_rows = (int64_t)E * N;
  return out_dtype == 0 ? launch<PLAIN_F32, 32>(a, b, b_rows, g, s)
                        : launch<PLAIN_BF16, 32>(a, b, b_rows, g, s);
}

namespace {
nvfp4_status_t l1_checked(const uint8_t* a, const uint8_t* sfa, const float* gs_a,
                          const uint8_t* w1, const uint8_t* sfw1, const float* gs_w1,
                          const int32_t* offs, const int32_t* row_slot, int E, int H, int I,
                          int64_t R_max, const float* gs_h, uint8_t* h, uint8_t* sfh, float* h32,
                          uint32_t* h_stats, int32_t* dev_status, nvfp4_stream_t stream) {
  if (E < 1 || E > MAX_E || H <= 0 || I <= 0 || R_max < 0) return NVFP4_ERR_INVALID_ARG;
  if (H % 64 || I % 64 || (2 * I) % TileCfg<L1_SWIGLU, 1>::BN || R_max % 128)
    return NVFP4_ERR_UNSUPPORTED_SHAPE;
  if (!gs_a || !gs_w1 || !offs || !gs_h) return NVFP4_ERR_INVALID_ARG;
  if (R_max == 0) return NVFP4_OK;
  if (!ok_ptr(a) || !ok_ptr(sfa) || !ok_ptr(w1) || !ok_ptr(sfw1) || !ok_ptr(h) || !ok_ptr(sfh))
    return (a && sfa && w1 && sfw1 && h && sfh) ? NVFP4_ERR_MISALIGNED : NVFP4_ERR_INVALID_ARG;
  if (reinterpret_cast<uintptr_t>(row_slot) & 3u) return NVFP4_ERR_MISALIGNED;
  if ((h32 && !aligned16(h32)) || (reinterpret_cast<uintptr_t>(h_stats) & 3u))
    return NVFP4_ERR_MISALIGNED;
  return gemm_l1(a, sfa, gs_a, w1, sfw1, gs_w1, offs, row_slot, E, H, I, R_max, gs_h, h, sfh, h32,
                 h_stats, dev_status, reinterpret_cast<cudaStream_t>(stream));
}
}  // namespace

extern "C" nvfp4_status_t moe_grouped_gemm_l1_swiglu_q(
    const uint8_t* a, const uint8_t* sfa, const float* gs_a, const uint8_t* w1,
    const uint8_t* sfw1, const float* gs_w1, const int32_t* offs, const int32_t* row_slot, int E,
    int H, int I, int64_t R_max, const float* gs_h, uint8_t* h, uint8_t* sfh, int32_t* dev_status,
    nvfp4_stream_t stream) {
  return l1_checked(a, sfa, gs_a, w1, sfw1, gs_w1, offs, row_slot, E, H, I, R_max, gs_h, h, sfh,
                    nullptr, nullptr, dev_status, stream);
}

extern "C" nvfp4_status_t moe_grouped_gemm_l1_swiglu_q_stats(
    const uint8_t* a, const uint8_t* sfa, const float* gs_a, const uint8_t* w1,
    const uint8_t* sfw1, const float* gs_w1, const int32_t* offs, const int32_t* row_slot, int E,
    int H, int I, int64_t R_max, const float* gs_h, uint8_t* h, uint8_t* sfh, float* h32,
    uint32_t* h_stats, int32_t* dev_status, nvfp4_stream_t stream) {
  return l1_checked(a, sfa, gs_a, w1, sfw1, gs_w1, offs, row_slot, E, H, I, R_max, gs_h, h, sfh,
                    h32, h_stats, dev_status, stream);
}

extern "C" nvfp4_status_t moe_grouped_gemm_l2_scatter(
    const uint8_t* h, const uint8_t* sfh, const float* gs_h, const uint8_t* w2,
    const uint8_t* sfw2, const float* gs_w2, const int32_t* offs, const int32_t* row_slot,
    const float* row_w, const int32_t* dst_row, int E, int H, int I, int T, int k, int64_t R_max,
    float* ys_ws, float* out_f32, void* out_bf16, int32_t* dev_status, nvfp4_stream_t stream) {
  if (E < 1 || E > MAX_E || H <= 0 || I <= 0 || T < 0 || k < 1 || R_max < 0)
    return NVFP4_ERR_INVALID_ARG;
  if (H % TileCfg<L2_ROWS, 1>::BN || I % 64 || R_max % 128) return NVFP4_ERR_UNSUPPORTED_SHAPE;
  if (!gs_h || !gs_w2 || !offs || !row_slot || !row_w || !dst_row || (!out_f32 && !out_bf16))
    return NVFP4_ERR_INVALID_ARG;
  if (T == 0 || R_max == 0) return NVFP4_OK;
  if (!ok_ptr(h) || !ok_ptr(sfh) || !ok_ptr(w2) || !ok_ptr(sfw2) || !ok_ptr(ys_ws) ||
      (out_f32 && !aligned16(out_f32)) || (out_bf16 && !aligned16(out_bf16)))
    return (h && sfh && w2 && sfw2 && ys_ws) ? NVFP4_ERR_MISALIGNED : NVFP4_ERR_INVALID_ARG;
  return gemm_l2(h, sfh, gs_h, w2, sfw2, gs_w2, offs, row_slot, row_w, dst_row, E, H, I, T, k,
                 R_max, ys_ws, out_f32, out_bf16, false, dev_status,
                 reinterpret_cast<cudaStream_t>(stream));
}

extern "C" nvfp4_status_t moe_grouped_gemm_l2_scatter_add(
    const uint8_t* h, const uint8_t* sfh, const float* gs_h, const uint8_t* w2,
    const uint8_t* sfw2, const float* gs_w2, const int32_t* offs, const int32_t* row_slot,
    const float* row_w, const int32_t* dst_row, int E, int H, int I, int T, int k, int64_t R_max,
    float* acc, void* out_bf16, int32_t* dev_status, nvfp4_stream_t stream) {
  if (E < 1 || E > MAX_E || H <= 0 || I <= 0 || T < 0 || k < 1 || R_max < 0)
    return NVFP4_ERR_INVALID_ARG;
  if (H % TileCfg<L2_ATOMIC, 1>::BN || I % 64 || R_max % 128) return NVFP4_ERR_UNSUPPORTED_SHAPE;
  if (!gs_h || !gs_w2 || !offs || !row_slot || !row_w || !dst_row || !acc)
    return NVFP4_ERR_INVALID_ARG;
  if (T == 0 || R_max == 0) return NVFP4_OK;
  if (!ok_ptr(h) || !ok_ptr(sfh) || !ok_ptr(w2) || !ok_ptr(sfw2) || !aligned16(acc) ||
      (out_bf16 && !aligned16(out_bf16)))
    return (h && sfh && w2 && sfw2) ? NVFP4_ERR_MISALIGNED : NVFP4_ERR_INVALID_ARG;
  return gemm_l2(h, sfh, gs_h, w2, sfw2, gs_w2, offs, row_slot, row_w, dst_row, E, H, I, T, k,
                 R_max, nullptr, acc, out_bf16, true, dev_status,
                 reinterpret_cast<cudaStream_t>(stream));
}

extern "C" int moe_ffn_l2_form(int T, int k, int E, int flags) {
  return l2_use_atomic(T, k, E, (flags & NVFP4_FFN_DETERMINISTIC) != 0) ? 1 : 0;
}

// ------------------------------------------------------------------------------ no-alloc variant
// The FP32 per-slot buffer of moe_grouped_gemm_l2_scatter_noalloc: one static array per device
// that loads the library.  Host code must not pass its name to a kernel (on the host it is only a
// stand-in symbol); its device address comes from cudaGetSymbolAddress, looked up once per device.
static __device__ __align__(256) float g_l2_noalloc_acc[NVFP4_L2_NOALLOC_MAX_ELEMS];

namespace {
constexpr int kMaxDevices = 64;

float* l2_noalloc_scratch() {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
    set_last_error("moe_grouped_gemm_l2_scatter_noalloc: no usable current device");
    return nullptr;
  }
  static std::mutex mu;
  static float* addr[kMaxDevices] = {};
  std::lock_guard<std::mutex> lock(mu);
  if (addr[dev] == nullptr) {
    void* p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_l2_noalloc_acc);
    if (e != cudaSuccess || p == nullptr) {
      check_launch("cudaGetSymbolAddress(g_l2_noalloc_acc)");
      return nullptr;
    }
    addr[dev] = static_cast<float*>(p);
  }
  return addr[dev];
}
}  // namespace

extern "C" nvfp4_status_t moe_grouped_gemm_l2_scatter_noalloc(
    const uint8_t* h, const uint8_t* sfh, const float* gs_h, const uint8_t* w2,
    const uint8_t* sfw2, const float* gs_w2, const int32_t* offs, const int32_t* row_slot,
    const float* row_w, const int32_t* dst_row, int E, int H, int I, int T, int k, int64_t R_max,
    void* out_bf16, int32_t* dev_status, nvfp4_stream_t stream) {
  if (E < 1 || E > MAX_E || H <= 0 || I <= 0 || T < 0 || k < 1 || R_max < 0)
    return NVFP4_ERR_INVALID_ARG;
  if (H % TileCfg<L2_ROWS, 1>::BN || I % 64 || R_max % 128) return NVFP4_ERR_UNSUPPORTED_SHAPE;
  if (!gs_h || !gs_w2 || !offs || !row_slot || !row_w || !dst_row || !out_bf16)
    return NVFP4_ERR_INVALID_ARG;
  if ((int64_t)T * k * H > NVFP4_L2_NOALLOC_MAX_ELEMS) {
    set_last_error("moe_grouped_gemm_l2_scatter_noalloc: T*k*H exceeds the static FP32 scratch "
                   "(NVFP4_L2_NOALLOC_MAX_ELEMS floats)");
    return NVFP4_ERR_WORKSPACE_TOO_SMALL;
  }
  if (T == 0 || R_max == 0) return NVFP4_OK;
  if (!ok_ptr(h) || !ok_ptr(sfh) || !ok_ptr(w2) || !ok_ptr(sfw2) || !aligned16(out_bf16))
    return (h && sfh && w2 && sfw2) ? NVFP4_ERR_MISALIGNED : NVFP4_ERR_INVALID_ARG;
  float* ys = l2_noalloc_scratch();
  if (ys == nullptr) return NVFP4_ERR_CUDA;
  return gemm_l2(h, sfh, gs_h, w2, sfw2, gs_w2, offs, row_slot, row_w, dst_row, E, H, I, T, k,
                 R_max, ys, nullptr, out_bf16, false, dev_status,
                 reinterpret_cast<cudaStream_t>(stream));
}

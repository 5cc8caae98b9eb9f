// Grouped expert GEMMs on the 5th-generation tensor cores (tcgen05, sm_100a).
//
// "Expert Parallel (EP)", Communication Pattern step 3 (each rank runs its local
// experts on the tokens it received); "Worked Example: Tracing a Token Through
// Expert Parallelism", Step 3 (two-layer FFN per expert).  Here every expert of
// every virtual rank runs in one persistent launch over the rank-major buffer.
//
// out[row, :] = epilogue( A[row, :] . B[g]^T ) for the rows of group g
//   A  bf16 [rows, K] row-major (K-major), rows of group g contiguous at
//      [group_offsets[g], group_offsets[g+1]);
//   B  bf16 [G, N, K] (K-major), one [N, K] matrix per group.
//
// Two kernels share this file.  grouped_gemm_pair_kernel (the default for 256-wide
// N tiles) runs 256 x 256 output tiles on a cluster of two CTAs with
// tcgen05.mma.cta_group::2; grouped_gemm_kernel runs 128 x BN tiles (BN = 256/128/64)
// on one CTA and serves the narrower N tiles.  In both, the tile list is
// expert-major, then N block, then M tile fastest, so the CTAs that run at the
// same time share each weight tile through L2 and stream every weight from HBM
// about once.  Each CTA derives the per-expert M-tile prefix from the group offsets
// (a block scan at launch): the host never learns the counts, so the grid is sized
// for the worst case and the CTAs take tiles from a device counter.  Empty experts
// own no tiles, so their weights are never read.
//
// One-CTA kernel: one CTA per SM, 6 warps:
//   warp 0      TMA producer: A tile [128 x 64] and B tile [BN x 64] per K step
//               into a STAGES-deep shared-memory ring (128-byte swizzle).
//   warp 1      allocates 2*BN TMEM columns; one lane issues tcgen05.mma
//               (M=128, N=BN, K=16, bf16 in, fp32 accumulate) into one of two
//               TMEM accumulators and commits to mbarriers.
//   warps 2-5   epilogue: tcgen05.ld the accumulator (warp w owns TMEM lanes
//               32*(w%4)..+31 = tile rows), apply the activation, round to bf16
//               and store the rows that belong to the group (rows past the group
//               end belong to the next expert and are dropped).
// The two accumulators let the epilogue of tile i overlap the MMAs of tile i+1.
//
// Every mbarrier wait is bounded (about 2 s of SM clock cycles): on expiry the
// kernel writes MOE_ERR_TIMEOUT to the status word, raises a CTA-wide abort flag
// so the other roles stop waiting, frees its TMEM and returns.
#include <stdio.h>
#include <stdlib.h>

#include "tc_common.cuh"

namespace moe {

namespace {


struct GemmArgs {
  CUtensorMap tmap_a;
  CUtensorMap tmap_b;
  const int32_t* group_offsets;   // the kernel derives the M tiles from these
  int32_t G, N, K, dense_rows;
  bf16* out;
  float* outf;               // EPI_PAIRSUM_F32 output
  int32_t ldo;
  int32_t* status;
  int32_t* counter;          // tile counter, zero at launch
};

// The CTA-pair kernel runs up to kMaxPhases GEMMs ("phases") in one persistent
// launch: tiles are numbered phase after phase and taken in that order.  A
// phase may depend on an earlier one (the down projection reads the activation
// rows the gate_up phase writes): its tile waits, before its first A load, until
// every tile of the matching 256-row band of the earlier phase has been stored.
constexpr int kMaxPhases = 4;
struct PhaseArgs {
  CUtensorMap tmap_a;        // A [rows, K], 128-row box
  CUtensorMap tmap_a64;      // the same A with a 64-row box (M = 128 remainder tiles)
  CUtensorMap tmap_a32;      // the same A with a 32-row box (skinny remainder tiles)
  CUtensorMap tmap_b;        // B [G, N, K]
  bf16* out;
  float* outf;               // EPI_PAIRSUM_F32 output
  int32_t ldo, N, K, epi;
  int32_t dense_rows;        // > 0: one dense group of this many rows; 0: the expert groups
  int32_t dep;               // phase whose band must be complete before A is read, or -1
  int32_t signal;            // 1: the epilogue counts stored tiles per band in done[]
  int32_t done_base;         // first done[] slot of this phase's bands (signal or dep source)
  bf16* const* sc_base;      // EPI_STORE: row i to sc_base[sc_rank[i]] + sc_row[i] * ldo, or null
  const int32_t* sc_rank;
  const int32_t* sc_row;
  int32_t sc_P, sc_rows;
};
struct PairArgs {
  PhaseArgs ph[kMaxPhases];
  const int32_t* group_offsets;   // [G + 1] (grouped phases); the kernel derives the M tiles
  int32_t G, nph;
  int32_t skinny;            // 1: groups of <= 64 rows run as skinny (weights-as-M) tiles
  int32_t fold;              // > 0: a single-band group of 257..256 + fold rows runs as one
                             //    folded tile (fold = 32 or 64, the largest remainder)
  int32_t fold_m256;         // 1: a folded remainder is one M = 256 product per K slice (needs
                             //    the gate/up exchange buffer in shared memory)
  int32_t* status;
  int32_t* counter;          // tile counter, zero at launch
  int32_t* done;             // band completion counts, zero at launch
  int32_t scatter;           // 1: a phase stores rows into other ranks' buffers (sc_base)
};

// Where output row `orow` of a scattering phase goes: the owning rank's buffer and row
// (rank and row checked against the table; a bad one stores nothing).
__device__ __forceinline__ void scatter_dst(const PhaseArgs& P, bool& valid, bf16*& o, int64_t& orow) {
  if (!valid) return;
  const int s = __ldg(P.sc_rank + orow), row = __ldg(P.sc_row + orow);
  if ((unsigned)s >= (unsigned)P.sc_P || (unsigned)row >= (unsigned)P.sc_rows) {
    valid = false;
    return;
  }
  o = P.sc_base[s];
  orow = row;
}

template <int BN>
struct GemmCfg {
  static constexpr int kStages = BN == 256 ? 4 : BN == 128 ? 6 : 8;
  static constexpr int kABytes = kTileM * kTileK * 2;
  static constexpr int kBBytes = BN * kTileK * 2;
  static constexpr int kStageBytes = kABytes + kBBytes;
  static constexpr int kTmemCols = 2 * BN;
  static constexpr uint32_t kIdesc = make_idesc(kTileM, BN);
  static size_t smem_bytes(int G) {
    return 1024 + (size_t)kStages * kStageBytes + kCtrlBytes + 2 * (size_t)(G + 1) * sizeof(int);
  }
};

// Per-group M tiles and their prefix, from the group offsets in shared memory:
// mt[g] = first tile of group g, mt[G] = all tiles.  Each thread sums a run of
// consecutive groups, a block scan of the run totals gives each run's first tile.
// Called by every thread of the block (it holds block barriers); wsum holds one int
// per warp.
template <int BN, int EPI>
__global__ void __launch_bounds__(kGemmThreads, 1) grouped_gemm_kernel(const __grid_constant__ GemmArgs p) {
  using C = GemmCfg<BN>;
  constexpr int S = C::kStages;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + ((1024u - (raw_addr & 1023u)) & 1023u);
  uint8_t* a_smem = smem;
  uint8_t* b_smem = smem + S * C::kABytes;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + S * C::kStageBytes);
  // bars: full[S], empty[S], tmem_full[2], tmem_empty[2], qfull[Q], qempty[Q]
  volatile int* tq = reinterpret_cast<volatile int*>(bars + 2 * S + 4 + 2 * kTileQ);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(const_cast<int*>(tq) + kTileQ);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  int* wsum = const_cast<int*>(abort_flag) + 1;                 // [kGemmThreads / 32]
  int* mt = reinterpret_cast<int*>(smem + S * C::kStageBytes + kCtrlBytes);
  const bool dense = p.group_offsets == nullptr;
  const int G = dense ? 1 : p.G;
  int* off = mt + (G + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t full0 = smem_u32(bars), empty0 = smem_u32(bars + S);
  const uint32_t tfull0 = smem_u32(bars + 2 * S), tempty0 = smem_u32(bars + 2 * S + 2);
  const uint32_t qfull0 = smem_u32(bars + 2 * S + 4), qempty0 = smem_u32(bars + 2 * S + 4 + kTileQ);

  if (threadIdx.x == 0) {
    for (int i = 0; i < S; ++i) {
      mbar_init(full0 + 8 * i, 1);
      mbar_init(empty0 + 8 * i, 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(tfull0 + 8 * i, 1);
      mbar_init(tempty0 + 8 * i, 4);
    }
    for (int i = 0; i < kTileQ; ++i) {
      mbar_init(qfull0 + 8 * i, 1);
      mbar_init(qempty0 + 8 * i, 5);         // MMA issuer + 4 epilogue warps
    }
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    prefetch_tmap(&p.tmap_a);
    prefetch_tmap(&p.tmap_b);
  }
  if (dense) {
    if (threadIdx.x == 0) {
      mt[0] = 0; mt[1] = (p.dense_rows + kTileM - 1) / kTileM;
      off[0] = 0; off[1] = p.dense_rows;
    }
  } else {
    for (int i = threadIdx.x; i <= G; i += blockDim.x) off[i] = p.group_offsets[i];
    __syncthreads();
    group_tile_prefix(off, G, mt, wsum, [](int rows) { return (rows + kTileM - 1) / kTileM; });
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(tmem_slot)),
                 "r"(C::kTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  const int nb = p.N / BN;
  const int total = mt[G] * nb;
  const int ksteps = p.K / kTileK;

  const uint32_t qempty_sched = map_to_cta(qempty0, 0);
  if (warp == 0) {
    if (lane == 0) {
      // ---------------- TMA producer (and tile scheduler) ----------------
      int stage = 0;
      uint32_t phase = 0;
      int next = atomicAdd(p.counter, 1);
      for (int qi = 0;; ++qi) {
        const int tile = tq_post<false>(p.counter, next, total, qi, qfull0, qempty0, tq, abort_flag, p.status);
        if (tile < 0) break;
        int g, m, n;
        decode_tile(tile, mt, G, nb, g, m, n);
        const int row0 = off[g] + m * kTileM;
        bool ok = true;
        for (int kb = 0; kb < ksteps; ++kb) {
          if (!mbar_wait(empty0 + 8 * stage, phase ^ 1u, abort_flag, p.status)) { ok = false; break; }
          const uint32_t fb = full0 + 8 * stage;
          mbar_arrive_expect_tx(fb, C::kStageBytes);
          tma_load_2d(smem_u32(a_smem + stage * C::kABytes), &p.tmap_a, fb, kb * kTileK, row0);
          tma_load_3d(smem_u32(b_smem + stage * C::kBBytes), &p.tmap_b, fb, kb * kTileK, n * BN, g);
          if (++stage == S) { stage = 0; phase ^= 1u; }
        }
        if (!ok) break;
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ---------------- MMA issuer ----------------
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      for (int qi = 0;; ++qi) {
        const int tile = tq_take<false>(qi, qfull0, qempty_sched, tq, abort_flag, p.status);
        if (tile < 0) break;
        if (!mbar_wait(tempty0 + 8 * acc, acc_phase ^ 1u, abort_flag, p.status)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + (uint32_t)(acc * BN);
        bool ok = true;
        for (int kb = 0; kb < ksteps; ++kb) {
          if (!mbar_wait(full0 + 8 * stage, phase, abort_flag, p.status)) { ok = false; break; }
          tc_fence_after();
          const uint64_t ad = sw128_desc(smem_u32(a_smem + stage * C::kABytes));
          const uint64_t bd = sw128_desc(smem_u32(b_smem + stage * C::kBBytes));
#pragma unroll
          for (int kk = 0; kk < kTileK / 16; ++kk)   // +32 bytes per K=16 slice
            tc_mma(d_tmem, ad + 2 * kk, bd + 2 * kk, C::kIdesc, (kb | kk) != 0);
          tc_commit(empty0 + 8 * stage);
          if (++stage == S) { stage = 0; phase ^= 1u; }
        }
        if (!ok) break;
        tc_commit(tfull0 + 8 * acc);
        acc ^= 1;
        if (acc == 0) acc_phase ^= 1u;
      }
    }
  } else {
    // ---------------- epilogue (warps 2..5) ----------------
    const int q = warp & 3;
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int qi = 0;; ++qi) {
      const int tile = tq_take<true>(qi, qfull0, qempty_sched, tq, abort_flag, p.status);
      if (__any_sync(0xffffffffu, tile < 0)) break;
      int g, m, n;
      decode_tile(tile, mt, G, nb, g, m, n);
      const int row0 = off[g] + m * kTileM;
      const int rows_valid = min(kTileM, off[g + 1] - row0);
      bool ok = true;
      if (lane == 0) ok = mbar_wait(tfull0 + 8 * acc, acc_phase, abort_flag, p.status);
      if (!__all_sync(0xffffffffu, ok)) break;     // keep the warp converged for tcgen05.ld
      tc_fence_after();
      const int r = q * 32 + lane;
      const bool valid = r < rows_valid;
      const uint32_t tb = tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)(acc * BN);
      const bool paired = EPI == EPI_SWIGLU || EPI == EPI_PAIRSUM_F32;
      epilogue_row<EPI>(p.out, p.outf, p.ldo, tb, 0, paired ? BN / 2 : BN, (int64_t)row0 + r,
                        paired ? n * (BN / 2) : n * BN, valid);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(tempty0 + 8 * acc);
      acc ^= 1;
      if (acc == 0) acc_phase ^= 1u;
    }
  }

  __syncwarp();                 // reconverge lane 0 of warps 0/1 with its warp
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base),
                 "r"(C::kTmemCols)
                 : "memory");
  }
}

// ---------------------------------------------------------------------------
// CTA-pair kernel: 256 x 256 output tiles on a cluster of 2 CTAs
// ---------------------------------------------------------------------------
// tcgen05.mma.cta_group::2 with M = 256, N = 256: CTA r of the pair holds A rows
// [row0 + 128 r, +128) and B rows [n0 + 128 r, +128) of every K step in its own
// shared memory, and its TMEM holds accumulator rows 128 r .. 128 r + 127 (all 256
// columns).  Per CTA and K step that is 16 KB of A + 16 KB of B for 128 x 256 x 64
// MACs, two thirds of the operand traffic of the one-CTA 128 x 256 tile.
// The last M tile of a group with at most 128 rows left runs as M = 128 instead
// (each CTA holds 64 A rows and still its 128 B rows): it costs half a full tile,
// which matters when groups hold a few hundred rows (e.g. 256 +- 18 rows per
// expert: a second full 256-row tile for 16 spill-over rows would waste a third
// of the tensor work).  Its accumulator uses the 2-CTA M = 128 layout: the CTA's
// row i sits in TMEM lane i for tile columns [0, 128) and in lane 64 + i for
// columns [128, 256), both at TMEM columns 0..127 — so each 128-column half of
// the B tile must carry matching gate/up (or hi/mid) columns, as packed.
//   warp 0 (both CTAs)   TMA producer: waits its own `empty` slot, loads its halves;
//                        the bytes complete on the leader's `full` barrier, whose
//                        expected byte count the leader posts for both CTAs.
//   warp 1 (leader)      issues the pair MMAs and commits to `empty` / `tmem_full`
//                        in both CTAs; warp 1 of both CTAs allocates the TMEM.
//   warps 2-5 (both)     epilogue of the CTA's 128 rows, then one arrive per warp
//                        on the leader's `tmem_empty` (8 arrivals per phase).
// Every wait is bounded as in the one-CTA kernel.
struct PairCfg {
  static constexpr int BN = 256;
  static constexpr int kStages = 6;
  static constexpr int kABytes = kTileM * kTileK * 2;            // this CTA's A half
  static constexpr int kBBytes = (BN / 2) * kTileK * 2;          // this CTA's B half
  static constexpr int kRemRows = 32;                           // folded rows per CTA (box)
  static constexpr int kRemBytes = kRemRows * kTileK * 2;        // this CTA's folded rows
  static constexpr int kStageBytes = kABytes + kBBytes + kRemBytes;
  static constexpr int kTmemCols = 2 * BN;
  static constexpr uint32_t kIdesc = make_idesc(2 * kTileM, BN);
  static constexpr uint32_t kIdescHalf = make_idesc(kTileM, BN);
  // gate/up exchange of a folded remainder's SwiGLU epilogue: 64 slab rows x 16 columns,
  // then its two mbarriers
  static constexpr int kFoldXBytes = 64 * 16 * 4 + 16;
  static size_t smem_bytes(int G, bool fold_x) {
    const size_t base = 1024 + (size_t)kStages * kStageBytes + kCtrlBytes + 2 * (size_t)(G + 1) * sizeof(int);
    return fold_x ? ((base + 15) & ~(size_t)15) + kFoldXBytes : base;
  }
};
// Largest remainder folded into a single-band group's tile (rows beyond 256): the
// remainder box holds kRemRows rows per CTA.
constexpr int kFoldMax = 2 * PairCfg::kRemRows;

// Where a pair tile sits: phase, group, M tile (256 rows), N block, its first row,
// the group's end row, and its band slot (the M tile's index across the phase).
struct PairTile {
  int ph, g, m, n, base, end, band;
};

// Shape of a pair tile from the rows it has left:
//   > 128 rows: M = 256 (128 rows per CTA), TK_FULL;
//   65..128 rows: M = 128 (64 rows per CTA), TK_HALF;
//   a group of at most 64 rows in all (a decode-sized batch), when enabled: TK_SKINNY,
//     the weights on the M side (M = 128: 64 weight rows per CTA, twice) and the rows
//     on the N side, N = rows rounded up to 32 (N/2 rows per CTA; a multiple of 32 is
//     a valid N for every 2-CTA MMA shape), for 2N/256 of an M = 128 tile's MMA work;
//   with folding enabled, a single-band group of 257..256 + fold rows in all: TK_FOLD,
//     the M = 256 tile of the first 256 rows plus, on every K step and from the same
//     weight slab in shared memory, the product of the remainder rows (weights as M,
//     rows as N).  The remainder then costs one small MMA per K16 slice instead of a
//     second tile that streams the whole weight panel again for a few rows (on
//     deepseek_v3's routing, 256 +- 18 rows per expert, half the experts have one).
//     Measured per tile on deepseek_v3: a folded K step 879-905 cycles against 613-630
//     for a full tile (1.44 full tiles), an M = 128 tile 614-623 (1.0).  The folded tile
//     falls behind when other tiles of its group share its weight tiles through L2
//     (the last band of larger groups, small_e8_d2048: 0.503 vs 0.475 ms), so only
//     single-band groups fold; with the one-product remainder a limit of 64 rows was
//     1.9 % faster than 32 on deepseek_v3's launch (6.94-7.03 vs 7.05-7.25 ms, one box).
// ns: the skinny (or folded) product's N, the row count rounded up to 32.
enum TileKind { TK_FULL = 0, TK_HALF = 1, TK_SKINNY = 2, TK_FOLD = 3 };
__device__ __forceinline__ int tile_kind(const PairTile& t, int skinny, int fold, int& ns) {
  const int left = t.end - t.base;
  ns = 0;
  if (fold > 0 && t.m == 0 && left > 2 * kTileM && left <= 2 * kTileM + fold) {
    ns = (left - 2 * kTileM + 31) & ~31;
    return TK_FOLD;
  }
  if (left > kTileM) return TK_FULL;
  if (!skinny || left > kTileM / 2 || t.m != 0) return TK_HALF;
  ns = (left + 31) & ~31;
  return TK_SKINNY;
}

// M tiles of a group of `rows` rows: 256 rows each; with folding, a group of 257..
// 256 + fold rows is one tile.
__device__ __forceinline__ int pair_mtiles(int rows, int fold) {
  if (rows <= 0) return 0;
  if (fold > 0 && rows > 2 * kTileM && rows <= 2 * kTileM + fold) return 1;
  return (rows + 2 * kTileM - 1) / (2 * kTileM);
}

__device__ __forceinline__ void decode_pair_tile(int tile, const int* pstart, int nph, const int* mt,
                                                 const int* off, int G, const int* dmt,
                                                 const int* doff, const PairArgs& p, PairTile& t) {
  int ph = 0;
  while (ph + 1 < nph && tile >= pstart[ph + 1]) ++ph;
  const int nb = p.ph[ph].N / PairCfg::BN;
  const bool dense = p.ph[ph].dense_rows > 0;
  const int* pm = dense ? dmt + 2 * ph : mt;
  const int* po = dense ? doff + 2 * ph : off;
  decode_tile(tile - pstart[ph], pm, dense ? 1 : G, nb, t.g, t.m, t.n);
  t.ph = ph;
  t.base = po[t.g] + t.m * 2 * kTileM;
  t.end = po[t.g + 1];
  t.band = pm[t.g] + t.m;
}

// Epilogue of a skinny product (a skinny tile, or the remainder of a folded one).  The
// accumulators hold weights-rows x tile-rows: in CTA r, TMEM lane i (i < 64) has
// weight row i of the CTA's slab for tile rows [0, ns/2), lane 64 + i the same weight
// row for tile rows [ns/2, ns), at columns tb.. (first 64 slab rows) and tb + 32..
// (second 64).  Warp q reads lanes 32q..32q+31.  The tile rows start at row `rbase`.
// The slab's rows are, per 256-wide N block n: SwiGLU / router pairs: the first and
// second factor of outputs n*128 + 64r + i; plain outputs: columns n*256 + 128r + i
// and + 64.  One output element per store (a warp writes 32 consecutive columns).
constexpr int kSkinnyHi = 32;     // TMEM column offset of the second 64 slab rows' product
__device__ __noinline__ void epilogue_skinny(int epi, bf16* out, float* outf, int ldo, uint32_t tb,
                                                const PairTile& t, int rbase, int rank, int q,
                                                int lane, int ns) {
  uint32_t r0[32], r1[32];
  tmem_ld32(tb, r0);
  tmem_ld32(tb + kSkinnyHi, r1);
  tmem_ld_wait();
  const int i = (q & 1) * 32 + lane;
  const int nh = ns >> 1;
  const int j0 = (q >> 1) * nh;                    // first tile row of this lane half
  const bool paired = epi == EPI_SWIGLU || epi == EPI_PAIRSUM_F32;
  const int col = paired ? t.n * 128 + rank * 64 + i : t.n * 256 + rank * 128 + i;
#pragma unroll
  for (int c = 0; c < 32; ++c) {
    if (c >= nh) break;
    const int64_t row = (int64_t)rbase + j0 + c;
    if (row >= t.end) break;
    const float a = __uint_as_float(r0[c]), b = __uint_as_float(r1[c]);
    if (epi == EPI_SWIGLU) {
      out[row * ldo + col] = __float2bfloat16_rn(silu_f(a) * b);
    } else if (epi == EPI_PAIRSUM_F32) {
      outf[row * ldo + col] = a + b;
    } else if (epi == EPI_GELU) {
      out[row * ldo + col] = __float2bfloat16_rn(gelu_f(a));
      out[row * ldo + col + 64] = __float2bfloat16_rn(gelu_f(b));
    } else {
      out[row * ldo + col] = __float2bfloat16_rn(a);
      out[row * ldo + col + 64] = __float2bfloat16_rn(b);
    }
  }
}

// Epilogue of a folded remainder computed as ONE M = 256 product per K slice (weights as
// M, the remainder rows as N = ns): in CTA r, TMEM lane m (0..127) holds slab row m of
// the CTA and columns 0..ns-1 the remainder rows 0..ns-1, which start at row `rbase`.
// Slab row m is, per 256-wide N block n: paired (SwiGLU / router pairs) the first
// factor of output n*128 + 64r + m (m < 64) or the second factor of output
// n*128 + 64r + m - 64; plain: output n*256 + 128r + m.  Paired, the warps holding the
// second factors (lane quarters 2, 3) pass them through shared memory (xbuf: 64 rows x
// 16 columns of fp32) to the warps holding the first (quarters 0, 1), 16 columns at a
// time, handing the buffer over on two mbarriers (xfull: 2 arrivals by the second-factor
// warps; xempty: 2 by the first-factor warps) with bounded waits.  `xk` counts the
// hand-overs so far (the same in every epilogue warp).  One element per store (a warp
// writes 32 consecutive output columns of a row).  Returns false if a wait gave up.
// Out of line, like epilogue_skinny: both run on few tiles, and inlined they made the main
// epilogue's code slower.
__device__ __noinline__ bool epilogue_fold256(int epi, bf16* out, float* outf, int ldo, uint32_t tb,
                                                 const PairTile& t, int rbase, int rank, int q, int lane,
                                                 int ns, float* xbuf, uint32_t xfull, uint32_t xempty,
                                                 uint32_t& xk, volatile int* abort_flag, int32_t* status) {
  const bool paired = epi == EPI_SWIGLU || epi == EPI_PAIRSUM_F32;
  for (int c0 = 0; c0 < ns; c0 += 16) {
    uint32_t v[16];
    __syncwarp();          // tcgen05.ld is warp-collective: reconverge after the masked stores
    tmem_ld16(tb + c0, v);
    tmem_ld_wait();
    if (!paired) {
      const int col = t.n * 256 + rank * 128 + q * 32 + lane;
#pragma unroll
      for (int c = 0; c < 16; ++c) {
        const int64_t row = (int64_t)rbase + c0 + c;
        if (c0 + c < ns && row < t.end) {
          const float x = __uint_as_float(v[c]);
          out[row * ldo + col] = __float2bfloat16_rn(epi == EPI_GELU ? gelu_f(x) : x);
        }
      }
      continue;
    }
    const int i = (q & 1) * 32 + lane;              // output among the CTA's 64
    float4* xr = reinterpret_cast<float4*>(xbuf + i * 16);
    const uint32_t par = xk & 1u;
    ++xk;
    bool ok = true;
    if (q >= 2) {
      if (lane == 0) ok = mbar_wait(xempty, par ^ 1u, abort_flag, status);
      if (!__all_sync(0xffffffffu, ok)) return false;
#pragma unroll
      for (int j = 0; j < 4; ++j)
        xr[j] = make_float4(__uint_as_float(v[4 * j]), __uint_as_float(v[4 * j + 1]),
                            __uint_as_float(v[4 * j + 2]), __uint_as_float(v[4 * j + 3]));
      __syncwarp();
      if (lane == 0) mbar_arrive(xfull);
    } else {
      if (lane == 0) ok = mbar_wait(xfull, par, abort_flag, status);
      if (!__all_sync(0xffffffffu, ok)) return false;
      float u[16];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const float4 f = xr[j];
        u[4 * j] = f.x; u[4 * j + 1] = f.y; u[4 * j + 2] = f.z; u[4 * j + 3] = f.w;
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(xempty);           // xbuf may be rewritten
      const int col = t.n * 128 + rank * 64 + i;
#pragma unroll
      for (int c = 0; c < 16; ++c) {
        const int64_t row = (int64_t)rbase + c0 + c;
        if (c0 + c < ns && row < t.end) {
          const float g = __uint_as_float(v[c]);
          if (epi == EPI_SWIGLU) out[row * ldo + col] = __float2bfloat16_rn(silu_f(g) * u[c]);
          else outf[row * ldo + col] = g + u[c];
        }
      }
    }
  }
  return true;
}

// Bounded wait (cycle count) until *cnt >= need, read with acquire semantics.
__device__ __noinline__ bool wait_count(const int32_t* cnt, int need, volatile int* abort_flag,
                                        int32_t* status) {
  const long long t0 = clock64();
  for (uint32_t it = 0;; ++it) {
    int v;
    asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(cnt) : "memory");
    if (v >= need) return true;
    if (*abort_flag) return false;
    if (clock64() - t0 > kWaitLimitCycles) {
      *abort_flag = 1;
      if (status != nullptr) atomicCAS(status, 0, (int32_t)MOE_ERR_TIMEOUT);
      return false;
    }
    __nanosleep(64);
  }
}

// TMEM of a pair CTA: two 256-column accumulators (buffers 0 and 1), each tracked as
// two regions: its head (columns 0..63) and its tail (64..255).  A tile with its main
// accumulator in buffer b occupies b's head and (unless skinny: its products fit in the
// head) b's tail; a folded tile also puts its remainder product in the OTHER buffer's
// head.  The MMA issuer waits, per region, until the region's previous occupant has
// been read out; the epilogue releases each region as soon as it has read it, a
// folded tile's remainder first and a main accumulator's head before its tail, so a
// folded tile waits only for the first part of the previous tile's epilogue.
// Barrier index of a region: head of b = b, tail of b = 2 + b.
__global__ void __launch_bounds__(kGemmThreads, 1) grouped_gemm_pair_kernel(const __grid_constant__ PairArgs p) {
  // launched as a programmatic dependent of the previous kernel on the stream: wait until
  // that kernel has completed and its writes are visible (a no-op otherwise)
  asm volatile("griddepcontrol.wait;" ::: "memory");
  using C = PairCfg;
  constexpr int S = C::kStages, BN = C::BN;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + ((1024u - (raw_addr & 1023u)) & 1023u);
  uint8_t* a_smem = smem;
  uint8_t* b_smem = smem + S * C::kABytes;
  uint8_t* r_smem = smem + S * (C::kABytes + C::kBBytes);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + S * C::kStageBytes);
  // bars: full[S], empty[S], tmem_full[2], tmem_free[4], qfull[Q], qempty[Q]
  volatile int* tq = reinterpret_cast<volatile int*>(bars + 2 * S + 6 + 2 * kTileQ);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(const_cast<int*>(tq) + kTileQ);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  int* pstart = reinterpret_cast<int*>(tmem_slot + 2);          // [kMaxPhases + 1]
  int* dmt = pstart + kMaxPhases + 1;                           // [kMaxPhases][2]
  int* doff = dmt + 2 * kMaxPhases;                             // [kMaxPhases][2]
  int* wsum = doff + 2 * kMaxPhases;                            // [kGemmThreads / 32]
  int* any_fold = wsum + kGemmThreads / 32;                     // 1: some group folds
  int* mt = reinterpret_cast<int*>(smem + S * C::kStageBytes + kCtrlBytes);
  const int G = p.G > 0 ? p.G : 1;
  int* off = mt + (G + 1);
  // gate/up exchange of folded remainders and its two mbarriers (present when p.fold_m256)
  float* xbuf = reinterpret_cast<float*>((reinterpret_cast<uintptr_t>(off + (G + 1)) + 15) & ~(uintptr_t)15);
  const uint32_t xfull = smem_u32(xbuf + 64 * 16), xempty = xfull + 8;
  const int nph = p.nph;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;
  const uint32_t full0 = smem_u32(bars), empty0 = smem_u32(bars + S);
  const uint32_t tfull0 = smem_u32(bars + 2 * S), tfree0 = smem_u32(bars + 2 * S + 2);
  const uint32_t qfull0 = smem_u32(bars + 2 * S + 6), qempty0 = smem_u32(bars + 2 * S + 6 + kTileQ);

  if (threadIdx.x == 0) {
    for (int i = 0; i < S; ++i) {
      mbar_init(full0 + 8 * i, 1);
      mbar_init(empty0 + 8 * i, 1);
    }
    for (int i = 0; i < 2; ++i) mbar_init(tfull0 + 8 * i, 1);
    for (int i = 0; i < 4; ++i) mbar_init(tfree0 + 8 * i, 8);     // 4 epilogue warps x 2 CTAs
    if (p.fold_m256) {
      mbar_init(xfull, 2);                 // the two second-factor warps of this CTA
      mbar_init(xempty, 2);                // the two first-factor warps
    }
    for (int i = 0; i < kTileQ; ++i) {
      mbar_init(qfull0 + 8 * i, 1);
      // leader: MMA issuer + 4 epilogue warps; peer: producer + 4 epilogue warps
      mbar_init(qempty0 + 8 * i, 10);
    }
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    for (int ph = 0; ph < nph; ++ph) {
      prefetch_tmap(&p.ph[ph].tmap_a);
      prefetch_tmap(&p.ph[ph].tmap_a64);
      prefetch_tmap(&p.ph[ph].tmap_a32);
      prefetch_tmap(&p.ph[ph].tmap_b);
      const int rows = p.ph[ph].dense_rows;
      dmt[2 * ph] = 0; dmt[2 * ph + 1] = pair_mtiles(rows, p.fold);
      doff[2 * ph] = 0; doff[2 * ph + 1] = rows;
    }
  }
  if (p.group_offsets != nullptr) {
    for (int i = threadIdx.x; i <= G; i += blockDim.x) off[i] = p.group_offsets[i];
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(tmem_slot)),
                 "r"(C::kTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
  }
  __syncthreads();
  if (threadIdx.x == 0) *any_fold = 0;
  if (p.group_offsets != nullptr) {
    const int fold = p.fold;
    group_tile_prefix(off, G, mt, wsum, [fold](int rows) { return pair_mtiles(rows, fold); });
    if (fold) {
      for (int g = threadIdx.x; g < G; g += blockDim.x) {
        const int rows = off[g + 1] - off[g];
        if (rows > 2 * kTileM && rows <= 2 * kTileM + fold) atomicOr(any_fold, 1);
      }
    }
  }
  if (threadIdx.x == 0) {          // tile numbering: phase after phase
    int acc_t = 0;
    for (int ph = 0; ph < nph; ++ph) {
      pstart[ph] = acc_t;
      const int mtiles = p.ph[ph].dense_rows > 0 ? dmt[2 * ph + 1] : mt[G];
      acc_t += mtiles * (p.ph[ph].N / BN);
    }
    pstart[nph] = acc_t;
  }
  tc_fence_before();
  cluster_sync();               // barriers of both CTAs initialised, TMEM allocated
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const int total = pstart[nph];
  const uint32_t qempty_sched = map_to_cta(qempty0, 0);

  if (warp == 0) {
    if (lane == 0) {
      // ---------------- TMA producer (both CTAs; the leader's also schedules) ----------------
      const uint32_t full0_leader = map_to_cta(full0, 0);
      int stage = 0;
      uint32_t phase = 0;
      int next = leader ? atomicAdd(p.counter, 1) : 0;
      const long long ti0 = instr_clock();
      for (int qi = 0;; ++qi) {
        const int tile = leader
            ? tq_post<true>(p.counter, next, total, qi, qfull0, qempty0, tq, abort_flag, p.status)
            : tq_take<false>(qi, qfull0, qempty_sched, tq, abort_flag, p.status);
        if (tile < 0) {
          // no tile left for this CTA: the next kernel on the stream may start launching
          // (it waits for this grid's completion before it reads anything)
          asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
          break;
        }
        PairTile t;
        decode_pair_tile(tile, pstart, nph, mt, off, G, dmt, doff, p, t);
        const PhaseArgs& P = p.ph[t.ph];
        int ns;
        const int kind = tile_kind(t, p.skinny, p.fold, ns);
        const bool m256 = kind == TK_FULL || kind == TK_FOLD;
        // rows of A this CTA loads: 128 (full), its 64 (half), or its ns/2 of a 32-row box
        const int arow = t.base + (int)rank * (m256 ? kTileM : kind == TK_HALF ? kTileM / 2 : ns / 2);
        const CUtensorMap* amap = m256 ? &P.tmap_a : kind == TK_HALF ? &P.tmap_a64 : &P.tmap_a32;
        const int abytes = m256 ? C::kABytes : kind == TK_HALF ? C::kABytes / 2 : C::kABytes / 4;
        // a folded tile also loads its remainder rows: this CTA's ns/2 of a 32-row box
        const bool fold = kind == TK_FOLD;
        const int rrow = t.base + 2 * kTileM + (int)rank * (ns / 2);
        const uint32_t stage_tx = 2u * (uint32_t)(abytes + C::kBBytes + (fold ? C::kRemBytes : 0));
        const int brow = t.n * BN + (int)rank * (BN / 2);
        if (P.dep >= 0) {
          // A rows of this band are written by phase P.dep: wait until all of its
          // N blocks (8 epilogue warps each) are stored, then order those generic-proxy
          // stores before this thread's TMA (async-proxy) reads
          const PhaseArgs& Q = p.ph[P.dep];
          if (!wait_count(p.done + Q.done_base + t.band, 8 * (Q.N / BN), abort_flag, p.status)) break;
          asm volatile("fence.proxy.async.global;" ::: "memory");
        }
        const int ksteps = P.K / kTileK;
        bool ok = true;
        for (int kb = 0; kb < ksteps; ++kb) {
          const long long tw = instr_clock();
          if (!mbar_wait(empty0 + 8 * stage, phase ^ 1u, abort_flag, p.status)) { ok = false; break; }
          instr_add(IS_PROD_WAIT, instr_clock() - tw);
          if (leader) mbar_arrive_expect_tx(full0 + 8 * stage, stage_tx);
          const uint32_t fb = full0_leader + 8 * stage;
          tma_load_2d_pair(smem_u32(a_smem + stage * C::kABytes), amap, fb, kb * kTileK, arow);
          tma_load_3d_pair(smem_u32(b_smem + stage * C::kBBytes), &P.tmap_b, fb, kb * kTileK, brow,
                           P.dense_rows > 0 ? 0 : t.g);
          if (fold)
            tma_load_2d_pair(smem_u32(r_smem + stage * C::kRemBytes), &P.tmap_a32, fb, kb * kTileK, rrow);
          if (++stage == S) { stage = 0; phase ^= 1u; }
        }
        if (!ok) break;
      }
      instr_add(IS_PROD_TOTAL, instr_clock() - ti0);
    }
  } else if (warp == 1) {
    if (lane == 0 && leader) {
      // ---------------- MMA issuer (leader CTA) ----------------
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t freeph = 0;       // bit i: parity of the next wait on TMEM region i
      const long long ti0 = instr_clock();
      for (int qi = 0;; ++qi) {
        const int tile = tq_take<false>(qi, qfull0, qempty_sched, tq, abort_flag, p.status);
        if (tile < 0) break;
        PairTile t;
        decode_pair_tile(tile, pstart, nph, mt, off, G, dmt, doff, p, t);
        int ns;
        const int kind = tile_kind(t, p.skinny, p.fold, ns);
        const uint32_t idesc = kind == TK_FULL || kind == TK_FOLD ? C::kIdesc
                               : kind == TK_HALF ? C::kIdescHalf : make_idesc(kTileM, ns);
        const uint32_t idesc_s = make_idesc(kTileM, ns);        // skinny / folded remainder
        const uint32_t idesc_f = make_idesc(2 * kTileM, ns);    // folded remainder, M = 256 form
        const int ksteps = p.ph[t.ph].K / kTileK;
        // the TMEM regions this tile writes: this buffer's head, its tail unless skinny,
        // the other buffer's head if folded
        const uint32_t need = (1u << acc) | (kind != TK_SKINNY ? 4u << acc : 0u) |
                              (kind == TK_FOLD ? 1u << (acc ^ 1) : 0u);
        bool ok = true;
        const long long tw = instr_clock();
        for (int i = 0; i < 4 && ok; ++i) {
          if (!((need >> i) & 1u)) continue;
          ok = mbar_wait(tfree0 + 8 * i, ((freeph >> i) & 1u) ^ 1u, abort_flag, p.status);
          freeph ^= 1u << i;
        }
        if (!ok) break;
        const long long tk0 = instr_clock();
        instr_add(IS_MMA_WAIT_ACC, tk0 - tw);
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + (uint32_t)(acc * BN);
        // skinny products (and a folded remainder, in the other buffer's head): the
        // first 64 weight rows into columns [0, ns/2), the second 64 into [32, 32 + ns/2)
        const uint32_t s_tmem = kind == TK_FOLD ? tmem_base + (uint32_t)((acc ^ 1) * BN) : d_tmem;
        for (int kb = 0; kb < ksteps; ++kb) {
          const long long tf = instr_clock();
          if (!mbar_wait(full0 + 8 * stage, phase, abort_flag, p.status)) { ok = false; break; }
          instr_add(IS_MMA_WAIT_FULL, instr_clock() - tf);
          tc_fence_after();
          const uint64_t ad = sw128_desc(smem_u32(a_smem + stage * C::kABytes));
          const uint64_t bd = sw128_desc(smem_u32(b_smem + stage * C::kBBytes));
          const uint64_t bd_hi = sw128_desc(smem_u32(b_smem + stage * C::kBBytes + C::kBBytes / 2));
          if (kind == TK_SKINNY) {
            // weights as the M operand (each CTA's B slab as two 64-row halves), rows as N
#pragma unroll
            for (int kk = 0; kk < kTileK / 16; ++kk) {
              tc_mma_pair(s_tmem, bd + 2 * kk, ad + 2 * kk, idesc_s, (kb | kk) != 0);
              tc_mma_pair(s_tmem + kSkinnyHi, bd_hi + 2 * kk, ad + 2 * kk, idesc_s, (kb | kk) != 0);
            }
          } else if (kind == TK_FOLD) {
            const uint64_t rd = sw128_desc(smem_u32(r_smem + stage * C::kRemBytes));
            if (p.fold_m256) {
              // the remainder as one M = 256 product: both CTAs' whole weight slabs as M
#pragma unroll
              for (int kk = 0; kk < kTileK / 16; ++kk) {
                tc_mma_pair(d_tmem, ad + 2 * kk, bd + 2 * kk, idesc, (kb | kk) != 0);
                tc_mma_pair(s_tmem, bd + 2 * kk, rd + 2 * kk, idesc_f, (kb | kk) != 0);
              }
            } else {
#pragma unroll
              for (int kk = 0; kk < kTileK / 16; ++kk) {
                tc_mma_pair(d_tmem, ad + 2 * kk, bd + 2 * kk, idesc, (kb | kk) != 0);
                tc_mma_pair(s_tmem, bd + 2 * kk, rd + 2 * kk, idesc_s, (kb | kk) != 0);
                tc_mma_pair(s_tmem + kSkinnyHi, bd_hi + 2 * kk, rd + 2 * kk, idesc_s, (kb | kk) != 0);
              }
            }
          } else {
#pragma unroll
            for (int kk = 0; kk < kTileK / 16; ++kk)
              tc_mma_pair(d_tmem, ad + 2 * kk, bd + 2 * kk, idesc, (kb | kk) != 0);
          }
          tc_commit_pair_both(empty0 + 8 * stage);
          if (++stage == S) { stage = 0; phase ^= 1u; }
        }
        if (!ok) break;
        {
          const int ki = kind == TK_FULL ? 0 : kind == TK_HALF ? 1 : kind == TK_FOLD ? 2 : 3;
          instr_add(IS_FULL_N + 2 * ki, 1);
          instr_add(IS_FULL_CYC + 2 * ki, instr_clock() - tk0);
          instr_add(IS_FULL_K + ki, ksteps);
          instr_add(IS_KSTEPS, ksteps);
        }
        tc_commit_pair_both(tfull0 + 8 * acc);
        acc ^= 1;
      }
      instr_add(IS_MMA_TOTAL, instr_clock() - ti0);
    }
  } else {
    // ---------------- epilogue (warps 2..5 of both CTAs) ----------------
    const int q = warp & 3;
    const uint32_t tfree_leader = map_to_cta(tfree0, 0);
    int acc = 0;
    uint32_t acc_phase = 0;
    uint32_t xk = 0;             // gate/up hand-overs of folded remainders so far
    const bool instr_epi = warp == 2 && lane == 0;
    const long long ti0 = instr_clock();
    // release TMEM region i: this warp has read all of its columns
    auto release = [&](int i) {
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(tfree_leader + 8 * i);
    };
    for (int qi = 0;; ++qi) {
      const int tile = tq_take<true>(qi, qfull0, qempty_sched, tq, abort_flag, p.status);
      if (__any_sync(0xffffffffu, tile < 0)) break;
      PairTile t;
      decode_pair_tile(tile, pstart, nph, mt, off, G, dmt, doff, p, t);
      const PhaseArgs& P = p.ph[t.ph];
      int ns;
      const int kind = tile_kind(t, p.skinny, p.fold, ns);
      bool ok = true;
      const long long tw = instr_clock();
      if (lane == 0) ok = mbar_wait(tfull0 + 8 * acc, acc_phase, abort_flag, p.status);
      if (instr_epi) instr_add(IS_EPI_WAIT, instr_clock() - tw);
      if (!__all_sync(0xffffffffu, ok)) break;
      tc_fence_after();
      const bool paired = P.epi == EPI_SWIGLU || P.epi == EPI_PAIRSUM_F32;
      const uint32_t lanes = (uint32_t)(q * 32) << 16;
      const uint32_t tb = tmem_base + lanes + (uint32_t)(acc * BN);
      if (kind == TK_FOLD) {
        // the remainder rows (after the first 256), from the other buffer's head
        const uint32_t tr = tmem_base + lanes + (uint32_t)((acc ^ 1) * BN);
        if (p.fold_m256) {
          if (!epilogue_fold256(P.epi, P.out, P.outf, P.ldo, tr, t, t.base + 2 * kTileM, (int)rank, q, lane, ns,
                                xbuf, xfull, xempty, xk, abort_flag, p.status))
            break;
        } else
          epilogue_skinny(P.epi, P.out, P.outf, P.ldo, tr, t, t.base + 2 * kTileM, (int)rank, q, lane, ns);
        release(acc ^ 1);
      }
      if (kind == TK_SKINNY) {
        epilogue_skinny(P.epi, P.out, P.outf, P.ldo, tb, t, t.base, (int)rank, q, lane, ns);
        release(acc);
      } else if (kind != TK_HALF) {
        // M = 256: this CTA's 128 rows in TMEM lanes 0..127, all 256 columns; output
        // columns [0, 64) read the head (and, paired, columns 64..127)
        const int row0 = t.base + (int)rank * kTileM;
        const int r = q * 32 + lane;
        const int col0 = paired ? t.n * (BN / 2) : t.n * BN;
        bool valid = r < min(t.end - row0, kTileM);
        bf16* o = P.out;
        int64_t orow = (int64_t)row0 + r;
        if (P.sc_base != nullptr) scatter_dst(P, valid, o, orow);
        if (*any_fold) {
          // the head (TMEM columns 0..63) is released as soon as it is in registers: a
          // folded tile that follows puts its remainder there
          epilogue_head_rt(P.epi, o, P.outf, P.ldo, tb, orow, col0, valid, [&] { release(acc); });
        } else {
          // no folded tile waits for a head: loads and stores interleaved, 32 columns at a time
          epilogue_row_rt(P.epi, o, P.outf, P.ldo, tb, 0, 64, orow, col0, valid);
          release(acc);
        }
        epilogue_row_rt(P.epi, o, P.outf, P.ldo, tb, 64, paired ? BN / 2 : BN, orow, col0, valid);
        release(2 + acc);
      } else {
        // M = 128: this CTA's 64 rows; lanes 0..63 hold tile columns [0, 128) and
        // lanes 64..127 columns [128, 256), each in TMEM columns 0..127
        const int row0 = t.base + (int)rank * (kTileM / 2);
        const int r = (q & 1) * 32 + lane, ch = q >> 1;
        const int col0 = paired ? t.n * (BN / 2) + ch * (BN / 4) : t.n * BN + ch * (BN / 2);
        bool valid = r < t.end - row0;
        bf16* o = P.out;
        int64_t orow = (int64_t)row0 + r;
        if (P.sc_base != nullptr) scatter_dst(P, valid, o, orow);
        epilogue_row_rt(P.epi, o, P.outf, P.ldo, tb, 0, paired ? BN / 4 : 64, orow, col0, valid);
        release(acc);
        if (!paired) epilogue_row_rt(P.epi, o, P.outf, P.ldo, tb, 64, BN / 2, orow, col0, valid);
        release(2 + acc);
      }
      if (P.signal) {
        // count this warp's stores of the band for the phase that reads them back
        asm volatile("fence.proxy.async.global;" ::: "memory");
        __threadfence();
        __syncwarp();
        if (lane == 0) atomicAdd(p.done + P.done_base + t.band, 1);
      }
      __syncwarp();
      acc ^= 1;
      if (acc == 0) acc_phase ^= 1u;
    }
    // rows stored into other ranks' memory are visible system-wide before the kernel
    // ends (the caller raises the ranks' flags after it)
    if (p.scatter) __threadfence_system();
    if (instr_epi) instr_add(IS_EPI_TOTAL, instr_clock() - ti0);
  }

  // Neither CTA leaves (or frees TMEM) while the pair's MMAs may still touch it.
  __syncwarp();                 // reconverge lane 0 of warps 0/1 with its warp
  tc_fence_before();
  cluster_sync();
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem_base),
                 "r"(C::kTmemCols)
                 : "memory");
  }
}

// ---------------------------------------------------------------------------
// Host side
// ---------------------------------------------------------------------------

bool make_map_2d(CUtensorMap* m, const void* base, uint64_t inner, uint64_t outer, uint32_t box_outer) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {inner * 2};
  cuuint32_t box[2] = {(cuuint32_t)kTileK, box_outer};
  cuuint32_t estr[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool make_map_3d(CUtensorMap* m, const void* base, uint64_t K, uint64_t N, uint64_t G, uint32_t box_n) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {K, N, G};
  cuuint64_t strides[2] = {K * 2, N * K * 2};
  cuuint32_t box[3] = {(cuuint32_t)kTileK, box_n, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

cudaError_t launch_tc_pair(const PairArgs& a, int clusters, cudaStream_t s) {
  const size_t smem = PairCfg::smem_bytes(a.group_offsets ? a.G : 1, a.fold_m256 != 0);
  auto kern = grouped_gemm_pair_kernel;
  cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (err != cudaSuccess) return err;
  cudaLaunchConfig_t cfg;
  memset(&cfg, 0, sizeof(cfg));
  cfg.gridDim = dim3(2 * clusters, 1, 1);
  cfg.blockDim = dim3(kGemmThreads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  // programmatic dependent launch: the grid may be scheduled while the previous kernel
  // finishes (the kernel's first instruction waits for that kernel's completion)
  // (MOE_PDL=0 in the environment: plain stream order; read at each call, for comparison)
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  const char* pdl_env = getenv("MOE_PDL");
  cfg.attrs = attr;
  cfg.numAttrs = (pdl_env && pdl_env[0] == '0') ? 1 : 2;
  err = cudaLaunchKernelEx(&cfg, kern, a);
  if (err != cudaSuccess) return err;
  return cudaGetLastError();
}

template <int BN, int EPI>
cudaError_t launch_tc(const GemmArgs& a, int grid, cudaStream_t s) {
  using C = GemmCfg<BN>;
  const size_t smem = C::smem_bytes(a.group_offsets ? a.G : 1);
  auto kern = grouped_gemm_kernel<BN, EPI>;
  cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (err != cudaSuccess) return err;
  kern<<<grid, kGemmThreads, smem, s>>>(a);
  return cudaGetLastError();
}

}  // namespace

int sm_count() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 148;
  static int cache[64] = {0};
  if (dev < 64 && cache[dev]) return cache[dev];
  int n = 148;
  cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
  if (dev < 64) cache[dev] = n;
  return n;
}

// Largest dynamic shared memory a block may opt in to on this device.
int smem_optin() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 232448;
  static int cache[64] = {0};
  if (dev < 64 && cache[dev]) return cache[dev];
  int n = 232448;
  cudaDeviceGetAttribute(&n, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
  if (dev < 64) cache[dev] = n;
  return n;
}

int64_t pair_band_bound(const GemmProblem& p) {
  // 256-row bands of a phase: ceil(rows / 256) for a dense group; for the expert
  // groups at most rows / 256 + G (each group adds at most one partial band)
  if (p.group_offsets == nullptr) return (p.dense_rows + 2 * kTileM - 1) / (2 * kTileM);
  return p.a_rows / (2 * kTileM) + p.G;
}

int64_t pair_done_slots(const GemmProblem* probs, int n) {
  int64_t slots = 0;
  for (int i = 0; i < n; ++i)
    for (int j = i + 1; j < n; ++j)
      if (probs[j].dep == i) { slots += pair_band_bound(probs[i]); break; }
  return slots;
}

cudaError_t launch_grouped_pair(const GemmProblem* probs, int n, int32_t* counter, int32_t* done,
                                cudaStream_t s) {
  if (n < 1 || n > kMaxPhases || counter == nullptr) return cudaErrorInvalidValue;
  PairArgs a;
  memset(&a, 0, sizeof(a));
  a.nph = n;
  {
    // MOE_GEMM_SKINNY=0 runs groups of <= 64 rows as M = 128 tiles too; MOE_GEMM_FOLD=0
    // runs a group's remainder of <= 64 rows past a full band as its own M = 128 tile
    const char* env = getenv("MOE_GEMM_SKINNY");
    a.skinny = (env && env[0] == '0') ? 0 : 1;
    env = getenv("MOE_GEMM_FOLD");
    const bool fold_on = !(env && env[0] == '0');
    // MOE_GEMM_FOLD256=0 runs a folded remainder as two M = 128 products per K slice
    env = getenv("MOE_GEMM_FOLD256");
    a.fold_m256 = (fold_on && !(env && env[0] == '0')) ? 1 : 0;
    // the largest folded remainder: kFoldMax rows with the one-product form
    // (MOE_GEMM_FOLD_MAX=32 for 32), 32 with the two-product form
    env = getenv("MOE_GEMM_FOLD_MAX");
    const int fmax = (env && atoi(env) == 32) ? 32 : kFoldMax;
    a.fold = fold_on ? (a.fold_m256 ? fmax : 32) : 0;
  }
  a.status = probs[0].status;
  a.counter = counter;
  a.done = done;
  int64_t tiles = 0, slot = 0;
  for (int i = 0; i < n; ++i) {
    const GemmProblem& p = probs[i];
    PhaseArgs& P = a.ph[i];
    if (p.tile_n != 256 || p.N % 256 != 0 || p.K % kTileK != 0) return cudaErrorInvalidValue;
    if (!make_map_2d(&P.tmap_a, p.A, (uint64_t)p.K, (uint64_t)p.a_rows, kTileM) ||
        !make_map_2d(&P.tmap_a64, p.A, (uint64_t)p.K, (uint64_t)p.a_rows, kTileM / 2) ||
        !make_map_2d(&P.tmap_a32, p.A, (uint64_t)p.K, (uint64_t)p.a_rows, kTileM / 4))
      return cudaErrorInvalidValue;
    // each CTA of a pair loads its 128-row half of the 256-row B tile
    if (!make_map_3d(&P.tmap_b, p.B, (uint64_t)p.K, (uint64_t)p.N, (uint64_t)p.G, 128))
      return cudaErrorInvalidValue;
    if (p.group_offsets != nullptr) {
      if (a.group_offsets != nullptr && (a.group_offsets != p.group_offsets || a.G != p.G))
        return cudaErrorInvalidValue;          // grouped phases share one grouping
      a.group_offsets = p.group_offsets;
      a.G = p.G;
      P.dense_rows = 0;
    } else {
      if (p.dense_rows <= 0) return cudaErrorInvalidValue;
      P.dense_rows = p.dense_rows;
    }
    P.out = p.out;
    P.outf = p.outf;
    P.ldo = p.ldo;
    P.N = p.N;
    P.K = p.K;
    P.epi = p.epi;
    P.dep = p.dep;
    if (p.sc_base != nullptr) {
      if (p.epi != EPI_STORE || p.sc_rank == nullptr || p.sc_row == nullptr || p.sc_P < 1)
        return cudaErrorInvalidValue;
      P.sc_base = p.sc_base;
      P.sc_rank = p.sc_rank;
      P.sc_row = p.sc_row;
      P.sc_P = p.sc_P;
      P.sc_rows = p.sc_rows;
      a.scatter = 1;
    }
    P.signal = 0;
    P.done_base = 0;
    if (p.dep >= 0) {
      // the phase read back must come first, share this phase's row tiling and count its bands
      if (p.dep >= i || done == nullptr) return cudaErrorInvalidValue;
      const GemmProblem& q = probs[p.dep];
      if ((q.group_offsets == nullptr) != (p.group_offsets == nullptr) ||
          (p.group_offsets == nullptr && q.dense_rows != p.dense_rows))
        return cudaErrorInvalidValue;
      PhaseArgs& Q = a.ph[p.dep];
      if (!Q.signal) {
        Q.signal = 1;
        Q.done_base = (int32_t)slot;
        slot += pair_band_bound(q);
      }
    }
    tiles += (p.max_tiles > 0 ? p.max_tiles : 1);
  }
  // a scattering launch runs only M = 256 and M = 128 tiles (the skinny and folded
  // epilogues write rows of their own)
  if (a.scatter) {
    a.skinny = 0;
    a.fold = 0;
    a.fold_m256 = 0;
  }
  // the M = 256 fold needs its exchange buffer next to the ring (room for about 700 groups)
  if (a.fold_m256 && PairCfg::smem_bytes(a.group_offsets ? a.G : 1, true) > (size_t)smem_optin()) {
    a.fold_m256 = 0;
    if (a.fold > 32) a.fold = 32;
  }
  const int64_t pairs = sm_count() / 2;
  const int clusters = (int)(tiles < pairs ? tiles : pairs);
  return launch_tc_pair(a, clusters, s);
}

cudaError_t launch_grouped_gemm(const GemmProblem& p, cudaStream_t s) {
  GemmArgs a;
  memset(&a, 0, sizeof(a));
  const int BN = p.tile_n;
  if (!make_map_2d(&a.tmap_a, p.A, (uint64_t)p.K, (uint64_t)p.a_rows, kTileM)) return cudaErrorInvalidValue;
  // each CTA of a pair loads its 128-row half of the 256-row B tile
  const uint32_t b_box = p.pair ? (uint32_t)(BN / 2) : (uint32_t)BN;
  if (!make_map_3d(&a.tmap_b, p.B, (uint64_t)p.K, (uint64_t)p.N, (uint64_t)p.G, b_box))
    return cudaErrorInvalidValue;
  a.group_offsets = p.group_offsets;
  a.G = p.G;
  a.N = p.N;
  a.K = p.K;
  a.dense_rows = p.dense_rows;
  a.out = p.out;
  a.outf = p.outf;
  a.ldo = p.ldo;
  a.status = p.status;
  a.counter = p.counter;
  if (p.counter == nullptr) return cudaErrorInvalidValue;
  const int64_t tiles = p.max_tiles > 0 ? p.max_tiles : 1;
  if (p.pair) {                 // 256 x 256 tiles on CTA pairs: a one-phase pair launch
    GemmProblem q = p;
    q.dep = -1;
    return launch_grouped_pair(&q, 1, p.counter, nullptr, s);
  }
  const int grid = (int)(tiles < sm_count() ? tiles : sm_count());
  if (BN == 256) {
    if (p.epi == EPI_SWIGLU) return launch_tc<256, EPI_SWIGLU>(a, grid, s);
    if (p.epi == EPI_GELU) return launch_tc<256, EPI_GELU>(a, grid, s);
    if (p.epi == EPI_PAIRSUM_F32) return launch_tc<256, EPI_PAIRSUM_F32>(a, grid, s);
    return launch_tc<256, EPI_STORE>(a, grid, s);
  }
  if (BN == 128) {
    if (p.epi == EPI_GELU) return launch_tc<128, EPI_GELU>(a, grid, s);
    if (p.epi == EPI_STORE) return launch_tc<128, EPI_STORE>(a, grid, s);
    return cudaErrorInvalidValue;
  }
  if (BN == 64) {
    if (p.epi == EPI_GELU) return launch_tc<64, EPI_GELU>(a, grid, s);
    if (p.epi == EPI_STORE) return launch_tc<64, EPI_STORE>(a, grid, s);
  }
  return cudaErrorInvalidValue;
}

// The pair and one-CTA kernels' cycle counters (instrumented builds; else not supported).
cudaError_t instr_read_pair(unsigned long long* host, int n) { return instr_read_tu(host, n); }

}  // namespace moe

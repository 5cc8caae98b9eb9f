// Grouped expert GEMM with MXFP8 operands on the 5th-generation tensor cores:
// tcgen05.mma.cta_group::2.kind::mxf8f6f4.block_scale, E4M3 A and B, one E8M0 scale
// per 32 K, 256 x 256 output tiles on a cluster of two CTAs.
//
// torchtitan issue 5554 (shared-expert overlap) lists MXFP8 routed experts as an
// option; "Expert Parallel (EP)", Communication Pattern step 3 and "Worked Example:
// Tracing a Token Through Expert Parallelism", Step 3 fix what runs: each expert's
// two-layer FFN over its rows of the rank-major buffer.  The format is OCP MX v1.0
// MXFP8 (E4M3): out[row, :] = epilogue( sum_k qa[row,k] 2^sa[row,k/32] qb[n,k] 2^sb[n,k/32] ),
// accumulated in fp32 by the tensor cores (the scaled products are exact).
//
// Operands (K-major E4M3 bytes):
//   A   [rows, K]; rows of group g at [off[g], off[g+1]); M tiles of 256 rows per group,
//       numbered across groups (tile t = tiles of the groups before g + m).
//   B   [G, N, K]; N tiles of 256 rows.
// Scales are stored "blocked": for tile t, K step s (128 K), block h (128 rows) a
// 512-byte block holding row m's four scales (K blocks 4s..4s+3) at byte
// 16 (m % 32) + 4 (m / 32) + j, the order tcgen05.cp .32x128b.warpx4 spreads over TMEM
// (row m in lane m % 32 of every lane quarter, column m / 32, byte j).  B has two blocks
// per tile and K step, at ((t * ksteps + s) * 2 + h) * 512 (mx_sf_offset); A has three,
// at ((t * ksteps + s) * 3 + h) * 512 (mx_sfa_offset), the third for a folded tile's
// remainder rows; so CTA h of a pair loads its A block and both B blocks of a K step with
// one TMA copy each.  A's blocks come from the row quantiser (the dispatch), which knows
// each row's tile, and from this kernel's own epilogue for the down projection's A (the
// activation): the up projection and the down projection tile the same groups the same
// way, so the epilogue of up tile t writes the scales of down tile t.
//
// The last tile of a group with at most 128 rows left runs as M = 128 (64 rows per CTA):
// its A scales use the same blocks (rows 0..63 of each), B's scales go to lane quarters
// 0-1 (rows 0..127) and 2-3 (rows 128..255), and the accumulator holds the CTA's row i in
// lane i for tile columns [0, 128) and in lane 64 + i for [128, 256).
//
// With folding (FOLD), a group of 257..256 + fold rows runs as ONE tile: per K step the
// M = 256 product of its first 256 rows and an M = 256 product of the pair's weight slabs
// (as M, their scales each CTA's own B block) with the remainder rows (as N = 32 or 64,
// their scales the third A block, read by both CTAs) into TMEM columns 320.., released on
// a barrier of its own.  The epilogue quantises a remainder row's activation across the
// 32 lanes of a warp (one weight row, i.e. one output, per lane); SwiGLU's up factors
// (lane quarters 2-3) reach the gate warps through shared memory on two mbarrier pairs.
//
// A CTA pair, 10 warps per CTA:
//   warp 0      TMA producer (lane 0, both CTAs): this CTA's 128 A rows, its 128 B rows,
//               its A scale block and both B scale blocks of each K step (and a folded
//               tile's remainder rows and scale blocks) into a 6-stage ring (5 with
//               folding); the bytes complete on the leader's `full` barrier.
//   warp 1      TMEM (512 columns, both CTAs); in the leader, lane 0 copies the stage's
//               scale blocks into TMEM (tcgen05.cp) and issues four M=256 N=256 K=32
//               block-scaled MMAs (and four remainder MMAs), scale byte j selected per
//               MMA; commits free the stage in both CTAs and hand the accumulator to the
//               epilogue.
//   warps 2-9   epilogue: warp w reads lanes 32 (w % 4) .. of TMEM, columns
//               128 ((w - 2) / 4) .. + 127, all into registers, then releases the
//               accumulator (16 arrivals on the leader) before its math and stores.
// The accumulator needs 256 TMEM columns and the scales 20, so there is one
// accumulator: the early release keeps the tensor cores' wait per tile to the TMEM
// read.  The scale columns are rewritten every K step: tcgen05 operations issued by one
// thread run in order, so a step's copy lands after the previous step's MMAs read theirs.
// Every wait is bounded and reports MOE_ERR_TIMEOUT.
#include <cuda_fp8.h>

#include "tc_common.cuh"

namespace moe {

namespace {

constexpr int kMxThreads = 320;
constexpr int kMxTileM = 256;

struct MxArgs {
  CUtensorMap tmap_a;        // E4M3 [rows, K], box 128 x 128 rows
  CUtensorMap tmap_a64;      // the same, box 128 x 64 rows (half tiles)
  CUtensorMap tmap_a32;      // the same, box 128 x 32 rows (a folded tile's remainder rows)
  CUtensorMap tmap_b;        // E4M3 [G, N, K], box 128 x 128 x 1
  CUtensorMap tmap_sfa;      // A scale blocks as [bytes / 256, 256], box 256 x 2 (one block)
  CUtensorMap tmap_sfb;      // B scale blocks, box 256 x 4 (both halves of a K step)
  CUtensorMap tmap_sfb1;     // B scale blocks, box 256 x 2 (one half)
  const int32_t* group_offsets;
  int32_t G, N, K;
  bf16* out;                 // EPI_STORE: bf16 [rows, ldo]
  int32_t ldo;
  uint8_t* q_out;            // EPI_SWIGLU / EPI_GELU: E4M3 activation [rows, ldo]
  uint8_t* q_sf;             //   and its scale blocks (ldo / 128 K steps)
  int32_t half;              // run a group's last <= 128 rows as an M = 128 tile
  int32_t fold;              // > 0: a group of 257..256 + fold rows runs as one folded tile
  int32_t* status;
  int32_t* counter;          // tile counter, zero at launch
};

// Shared memory per stage: this CTA's A and B halves and the scale blocks; with folding
// (kFold) also a folded tile's remainder rows (a 32-row box), their scale block and this
// CTA's own B scale block (the remainder product's A scales), in 5 stages instead of 6.
template <bool kFold>
struct MxCfgT {
  static constexpr int BN = 256;
  static constexpr int KS = 128;                     // K elements (bytes) per stage
  static constexpr int kStages = kFold ? 5 : 6;
  static constexpr int kABytes = 128 * KS;           // this CTA's 128 A rows
  static constexpr int kBBytes = 128 * KS;           // this CTA's 128 B rows
  static constexpr int kRemBytes = kFold ? 32 * KS : 0;
  static constexpr int kSfaBytes = 512;
  static constexpr int kSfbBytes = 1024;
  static constexpr int kSfoBytes = kFold ? 512 : 0;  // own B block (remainder product's A scales)
  static constexpr int kSfrBytes = kFold ? 512 : 0;  // remainder rows' scales
  static constexpr int kStageBytes =
      kABytes + kBBytes + kRemBytes + kSfaBytes + kSfbBytes + kSfoBytes + kSfrBytes;
  static constexpr int kTmemCols = 512;
  // scale columns after the accumulator, then the remainder product's accumulator
  static constexpr int kSfaCol = 256, kSfbCol = 260, kSsfaCol = 268, kSsfbCol = 272, kRemCol = 320;
  static constexpr int kCtrl = 512;
  // gate/up exchange of a folded remainder: per column half, 64 outputs x 32 columns fp32,
  // then 4 mbarriers
  static constexpr int kXBytes = kFold ? 2 * 64 * 32 * 4 + 32 : 0;
  static size_t smem_bytes(int G) {
    const size_t base = 1024 + (size_t)kStages * kStageBytes + kCtrl + 2 * (size_t)(G + 1) * sizeof(int);
    return ((base + 15) & ~(size_t)15) + kXBytes;
  }
};
using MxCfg = MxCfgT<false>;

// Block-scaled instruction descriptor, kind::mxf8f6f4: E4M3 A and B, K-major, E8M0 scales
// (bit 23), scale byte `j` of A and of B (bits 29-30 and 4-5).
__host__ __device__ constexpr uint32_t mx_idesc(int M, int N, int j) {
  return ((uint32_t)j << 4) | ((uint32_t)(N >> 3) << 17) | (1u << 23) | ((uint32_t)(M >> 4) << 24) |
         ((uint32_t)j << 29);
}

// Shared-memory descriptor of a 512-byte scale block for tcgen05.cp: no swizzle,
// 8-row core matrices of 16-byte rows placed 128 bytes apart.
__device__ __forceinline__ uint64_t sf_desc(uint32_t saddr) {
  return (uint64_t)((saddr & 0x3FFFFu) >> 4) | ((uint64_t)(128 >> 4) << 32) | ((uint64_t)1 << 46);
}

__device__ __forceinline__ void tc_cp_sf_pair(uint32_t taddr, uint64_t sdesc) {
  asm volatile("tcgen05.cp.cta_group::2.32x128b.warpx4 [%0], %1;" ::"r"(taddr), "l"(sdesc) : "memory");
}

__device__ __forceinline__ void tc_mma_mx_pair(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                               uint32_t idesc, uint32_t accumulate, uint32_t sfa,
                                               uint32_t sfb) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::mxf8f6f4.block_scale [%0], %1, %2, %3, [%5], [%6], p;\n\t}" ::"r"(
          d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(sfa), "r"(sfb)
      : "memory");
}

// Byte offset of B's scale (row m of half h, K block j) of tile t's K step s: two blocks
// (halves of 128 rows) per tile and K step.
__host__ __device__ __forceinline__ size_t mx_sf_offset(int64_t t, int ksteps, int s, int h, int m, int j) {
  return (size_t)((t * ksteps + s) * 2 + h) * 512 + 16 * (m & 31) + 4 * (m >> 5) + j;
}
// The same for A: three blocks per tile and K step, the third for a folded tile's
// remainder rows (rows 256.. of the group, m = row - 256).
__host__ __device__ __forceinline__ size_t mx_sfa_offset(int64_t t, int ksteps, int s, int h, int m, int j) {
  return (size_t)((t * ksteps + s) * 3 + h) * 512 + 16 * (m & 31) + 4 * (m >> 5) + j;
}

// M tiles of a group of `rows` rows: 256 rows each, a group of 257..256 + fold rows one.
__device__ __forceinline__ int mx_mtiles(int rows, int fold) {
  if (fold > 0 && rows > kMxTileM && rows <= kMxTileM + fold) return 1;
  return (rows + kMxTileM - 1) / kMxTileM;
}
// Whether tile m of a group of `rows` rows is folded; ns: the remainder's N (rows past
// 256 rounded up to 32).
__device__ __forceinline__ bool mx_is_fold(int rows, int m, int fold, int& ns) {
  ns = 0;
  if (fold > 0 && m == 0 && rows > kMxTileM && rows <= kMxTileM + fold) {
    ns = (rows - kMxTileM + 31) & ~31;
    return true;
  }
  return false;
}

// M tile m of a group of `rows` rows is a half tile (M = 128: 64 rows per CTA) when at
// most 128 rows are left for it and half tiles are enabled; otherwise M = 256.
__device__ __forceinline__ bool mx_is_half(int rows, int m, int half) {
  return half && rows - m * kMxTileM <= 128;
}

// Scale-block place of row `rr` of a group of `rows` rows: tile offset dt (from the
// group's first tile), block h and row m in it.
__device__ __forceinline__ void mx_a_place(int rows, int rr, int half, int fold, int& dt, int& h, int& m) {
  int ns;
  if (mx_is_fold(rows, 0, fold, ns)) {
    dt = 0;
    if (rr < kMxTileM) { h = rr >> 7; m = rr & 127; }
    else { h = 2; m = rr - kMxTileM; }
    return;
  }
  dt = rr / kMxTileM;
  const int within = rr % kMxTileM;
  if (mx_is_half(rows, dt, half)) { h = within >> 6; m = within & 63; }
  else { h = within >> 7; m = within & 127; }
}

// 64 rows of 16 bytes: rows 0..31 into lane quarters 0 and 1, rows 32..63 into quarters 2
// and 3 (the scale layout of B for an M = 128 pair MMA; measured: the ::02_13 form gives
// wrong products there).
__device__ __forceinline__ void tc_cp_sf_pair_64(uint32_t taddr, uint64_t sdesc) {
  asm volatile("tcgen05.cp.cta_group::2.64x128b.warpx2::01_23 [%0], %1;" ::"r"(taddr), "l"(sdesc) : "memory");
}

// E8M0 exponent of a block from its largest magnitude: floor(log2 amax) - 8, clamped to
// [-127, 127] (-127 for a zero block; a subnormal amax also lands on -127).
__device__ __forceinline__ int mx_exponent(float amax) {
  const int e = (int)((__float_as_uint(amax) >> 23) & 0xFFu) - 127 - 8;
  return e < -127 ? -127 : (e > 127 ? 127 : e);
}

// Quantise 32 values: E4M3 bytes of v * 2^-s (round to nearest even, saturated) into
// dst (32 bytes, 16-byte aligned); returns the scale byte s + 127.
__device__ __forceinline__ uint8_t mx_quant32(const float (&v)[32], uint8_t* dst) {
  float amax = 0.f;
#pragma unroll
  for (int i = 0; i < 32; ++i) amax = fmaxf(amax, fabsf(v[i]));
  const int s = mx_exponent(amax);
  const float inv = __uint_as_float((uint32_t)(127 - s) << 23);
  uint4 out[2];
  uint16_t* o = reinterpret_cast<uint16_t*>(out);
#pragma unroll
  for (int i = 0; i < 16; ++i)
    o[i] = (uint16_t)__nv_cvt_float2_to_fp8x2(make_float2(v[2 * i] * inv, v[2 * i + 1] * inv), __NV_SATFINITE,
                                              __NV_E4M3);
  uint4* d = reinterpret_cast<uint4*>(dst);
  d[0] = out[0];
  d[1] = out[1];
  return (uint8_t)(s + 127);
}

__device__ __forceinline__ void store32(bf16* dst, const uint32_t (&v)[32]) {
  float f[32];
#pragma unroll
  for (int i = 0; i < 32; ++i) f[i] = __uint_as_float(v[i]);
  store_row32(dst, f);
}
__device__ __forceinline__ uint8_t quant_swiglu32(const uint32_t (&gate)[32], const uint32_t (&up)[32],
                                                  uint8_t* dst) {
  float f[32];
#pragma unroll
  for (int i = 0; i < 32; ++i) f[i] = silu_f(__uint_as_float(gate[i])) * __uint_as_float(up[i]);
  return mx_quant32(f, dst);
}
__device__ __forceinline__ uint8_t quant_gelu32(const uint32_t (&v)[32], uint8_t* dst) {
  float f[32];
#pragma unroll
  for (int i = 0; i < 32; ++i) f[i] = gelu_f(__uint_as_float(v[i]));
  return mx_quant32(f, dst);
}

// Quantises, along the 32 lanes of a warp (32 consecutive outputs of one row), the value
// v of this lane: returns the E4M3 byte, and the block's scale byte through `sc`.
__device__ __forceinline__ uint8_t mx_quant_lanes(float v, uint8_t& sc) {
  float amax = fabsf(v);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
  const int s = mx_exponent(amax);
  const float inv = __uint_as_float((uint32_t)(127 - s) << 23);
  sc = (uint8_t)(s + 127);
  return (uint8_t)__nv_cvt_float_to_fp8(v * inv, __NV_SATFINITE, __NV_E4M3);
}

template <int EPI, bool FOLD>
__global__ void __launch_bounds__(kMxThreads, 1) grouped_gemm_mx_kernel(const __grid_constant__ MxArgs p) {
  using C = MxCfgT<FOLD>;
  constexpr int S = C::kStages, BN = C::BN;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + ((1024u - (raw_addr & 1023u)) & 1023u);
  uint8_t* a_smem = smem;
  uint8_t* b_smem = smem + S * C::kABytes;
  uint8_t* r_smem = smem + S * (C::kABytes + C::kBBytes);
  uint8_t* sfa_smem = r_smem + S * C::kRemBytes;
  uint8_t* sfb_smem = sfa_smem + S * C::kSfaBytes;
  uint8_t* sfo_smem = sfb_smem + S * C::kSfbBytes;
  uint8_t* sfr_smem = sfo_smem + S * C::kSfoBytes;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + S * C::kStageBytes);
  // bars: full[S], empty[S], tmem_full, tmem_empty, tmem_empty_rem, qfull[Q], qempty[Q]
  volatile int* tq = reinterpret_cast<volatile int*>(bars + 2 * S + 3 + 2 * kTileQ);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(const_cast<int*>(tq) + kTileQ);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  int* wsum = const_cast<int*>(abort_flag) + 1;                 // [kMxThreads / 32]
  int* mt = reinterpret_cast<int*>(smem + S * C::kStageBytes + C::kCtrl);
  const int G = p.G;
  int* off = mt + (G + 1);
  // gate/up exchange of folded remainders: xbuf[h] = 64 outputs x 32 columns, then
  // xfull[h], xempty[h] (FOLD only)
  float* xbuf = reinterpret_cast<float*>((reinterpret_cast<uintptr_t>(off + (G + 1)) + 15) & ~(uintptr_t)15);
  const uint32_t xbar0 = smem_u32(xbuf + 2 * 64 * 32);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;
  const uint32_t full0 = smem_u32(bars), empty0 = smem_u32(bars + S);
  const uint32_t tfull = smem_u32(bars + 2 * S), tempty = smem_u32(bars + 2 * S + 1);
  // the remainder accumulator is released on its own, after the main one
  const uint32_t tempty_rem = smem_u32(bars + 2 * S + 2);
  const uint32_t qfull0 = smem_u32(bars + 2 * S + 3), qempty0 = smem_u32(bars + 2 * S + 3 + kTileQ);
  const int fold = FOLD ? p.fold : 0;

  if (threadIdx.x == 0) {
    for (int i = 0; i < S; ++i) {
      mbar_init(full0 + 8 * i, 1);
      mbar_init(empty0 + 8 * i, 1);
    }
    mbar_init(tfull, 1);
    mbar_init(tempty, 16);                   // 8 epilogue warps x 2 CTAs
    mbar_init(tempty_rem, 16);
    for (int i = 0; i < kTileQ; ++i) {
      mbar_init(qfull0 + 8 * i, 1);
      // leader: MMA issuer + 8 epilogue warps; peer: producer + 8 epilogue warps
      mbar_init(qempty0 + 8 * i, 18);
    }
    if (FOLD) {
      for (int i = 0; i < 4; ++i) mbar_init(xbar0 + 8 * i, 2);   // xfull[2]: up warps; xempty[2]: gate warps
    }
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    prefetch_tmap(&p.tmap_a);
    prefetch_tmap(&p.tmap_a64);
    prefetch_tmap(&p.tmap_b);
    prefetch_tmap(&p.tmap_sfa);
    prefetch_tmap(&p.tmap_sfb);
    if (FOLD) {
      prefetch_tmap(&p.tmap_a32);
      prefetch_tmap(&p.tmap_sfb1);
    }
  }
  for (int i = threadIdx.x; i <= G; i += blockDim.x) off[i] = p.group_offsets[i];
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(tmem_slot)),
                 "r"(C::kTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
  }
  __syncthreads();
  group_tile_prefix(off, G, mt, wsum, [fold](int rows) { return mx_mtiles(rows, fold); });
  tc_fence_before();
  cluster_sync();               // barriers of both CTAs initialised, TMEM allocated
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  const int nb = p.N / BN;
  const int total = mt[G] * nb;
  const int ksteps = p.K / C::KS;
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
        if (tile < 0) break;
        int g, m, n;
        decode_tile(tile, mt, G, nb, g, m, n);
        const int rows = off[g + 1] - off[g];
        int ns;
        const bool fd = FOLD && mx_is_fold(rows, m, fold, ns);
        const bool hf = !fd && mx_is_half(rows, m, p.half);
        const int arow = off[g] + m * kMxTileM + (int)rank * (hf ? 64 : 128);
        const CUtensorMap* amap = hf ? &p.tmap_a64 : &p.tmap_a;
        const uint32_t stage_tx =
            fd ? 2u * (uint32_t)C::kStageBytes
               : 2u * (uint32_t)(C::kABytes + C::kBBytes + C::kSfaBytes + C::kSfbBytes - (hf ? C::kABytes / 2 : 0));
        const int brow = n * BN + (int)rank * 128;
        const int rrow = off[g] + kMxTileM + (int)rank * (ns / 2);
        const int64_t ta = (int64_t)mt[g] + m;              // A's tile (scale blocks)
        const int64_t tb = (int64_t)g * nb + n;              // B's tile
        bool ok = true;
        for (int kb = 0; kb < ksteps; ++kb) {
          const long long tw = instr_clock();
          if (!mbar_wait(empty0 + 8 * stage, phase ^ 1u, abort_flag, p.status)) { ok = false; break; }
          instr_add(IS_PROD_WAIT, instr_clock() - tw);
          if (leader) mbar_arrive_expect_tx(full0 + 8 * stage, stage_tx);
          const uint32_t fb = full0_leader + 8 * stage;
          tma_load_2d_pair(smem_u32(a_smem + stage * C::kABytes), amap, fb, kb * C::KS, arow);
          tma_load_3d_pair(smem_u32(b_smem + stage * C::kBBytes), &p.tmap_b, fb, kb * C::KS, brow, g);
          tma_load_2d_pair(smem_u32(sfa_smem + stage * C::kSfaBytes), &p.tmap_sfa, fb, 0,
                           (int)(((ta * ksteps + kb) * 3 + rank) * 2));
          tma_load_2d_pair(smem_u32(sfb_smem + stage * C::kSfbBytes), &p.tmap_sfb, fb, 0,
                           (int)((tb * ksteps + kb) * 4));
          if (FOLD && fd) {
            // the remainder rows (this CTA's ns/2 of a 32-row box), their scale block
            // (the third block, the same in both CTAs) and this CTA's own B scale block
            tma_load_2d_pair(smem_u32(r_smem + stage * C::kRemBytes), &p.tmap_a32, fb, kb * C::KS, rrow);
            tma_load_2d_pair(smem_u32(sfr_smem + stage * C::kSfrBytes), &p.tmap_sfa, fb, 0,
                             (int)(((ta * ksteps + kb) * 3 + 2) * 2));
            tma_load_2d_pair(smem_u32(sfo_smem + stage * C::kSfoBytes), &p.tmap_sfb1, fb, 0,
                             (int)(((tb * ksteps + kb) * 2 + rank) * 2));
          }
          if (++stage == S) { stage = 0; phase ^= 1u; }
        }
        if (!ok) break;
      }
      instr_add(IS_PROD_TOTAL, instr_clock() - ti0);
    }
  } else if (warp == 1) {
    if (lane == 0 && leader) {
      // ---------------- scale copies and block-scaled pair MMAs (leader CTA) ----------------
      const uint32_t t_sfa = tmem_base + C::kSfaCol, t_sfb = tmem_base + C::kSfbCol;
      const uint32_t t_ssfa = tmem_base + C::kSsfaCol, t_ssfb = tmem_base + C::kSsfbCol;
      const uint32_t t_rem = tmem_base + C::kRemCol;
      int stage = 0;
      uint32_t phase = 0;
      uint32_t acc_phase = 0, rem_phase = 0;
      const long long ti0 = instr_clock();
      for (int qi = 0;; ++qi) {
        const int tile = tq_take<false>(qi, qfull0, qempty_sched, tq, abort_flag, p.status);
        if (tile < 0) break;
        int g, m, n;
        decode_tile(tile, mt, G, nb, g, m, n);
        const int rows = off[g + 1] - off[g];
        int ns;
        const bool fd = FOLD && mx_is_fold(rows, m, fold, ns);
        const bool hf = !fd && mx_is_half(rows, m, p.half);
        const long long tw = instr_clock();
        if (!mbar_wait(tempty, acc_phase ^ 1u, abort_flag, p.status)) break;
        acc_phase ^= 1u;
        if (fd) {                              // the previous folded tile's remainder is read out
          if (!mbar_wait(tempty_rem, rem_phase ^ 1u, abort_flag, p.status)) break;
          rem_phase ^= 1u;
        }
        const long long tk0 = instr_clock();
        instr_add(IS_MMA_WAIT_ACC, tk0 - tw);
        tc_fence_after();
        bool ok = true;
        for (int kb = 0; kb < ksteps; ++kb) {
          const long long tf = instr_clock();
          if (!mbar_wait(full0 + 8 * stage, phase, abort_flag, p.status)) { ok = false; break; }
          instr_add(IS_MMA_WAIT_FULL, instr_clock() - tf);
          tc_fence_after();
          const uint32_t sa = smem_u32(sfa_smem + stage * C::kSfaBytes);
          const uint32_t sb = smem_u32(sfb_smem + stage * C::kSfbBytes);
          tc_cp_sf_pair(t_sfa, sf_desc(sa));
          if (!hf) {
            // M = 256: B's scales for rows n (0..255) in lane n % 32 of every quarter, column n / 32
            tc_cp_sf_pair(t_sfb, sf_desc(sb));              // B rows 0..127 of the tile
            tc_cp_sf_pair(t_sfb + 4, sf_desc(sb + 512));    // B rows 128..255
          } else {
            // M = 128: rows 0..127 in lane quarters 0 and 1, rows 128..255 in quarters 2 and 3
            tc_cp_sf_pair_64(t_sfb, sf_desc(sb));
          }
          if (FOLD && fd) {
            // remainder product: this CTA's weight slab as M (its own B block as A scales),
            // the remainder rows as N (their block, rows n in lane n % 32, column n / 32)
            tc_cp_sf_pair(t_ssfa, sf_desc(smem_u32(sfo_smem + stage * C::kSfoBytes)));
            tc_cp_sf_pair(t_ssfb, sf_desc(smem_u32(sfr_smem + stage * C::kSfrBytes)));
          }
          const uint64_t ad = sw128_desc(smem_u32(a_smem + stage * C::kABytes));
          const uint64_t bd = sw128_desc(smem_u32(b_smem + stage * C::kBBytes));
          const int mm = hf ? kMxTileM / 2 : kMxTileM;
#pragma unroll
          for (int j = 0; j < 4; ++j)          // K = 32 per MMA: +32 bytes
            tc_mma_mx_pair(tmem_base, ad + 2 * j, bd + 2 * j, mx_idesc(mm, BN, j), (kb | j) != 0,
                           t_sfa | ((uint32_t)j << 30), t_sfb | ((uint32_t)j << 30));
          if (FOLD && fd) {
            const uint64_t rd = sw128_desc(smem_u32(r_smem + stage * C::kRemBytes));
#pragma unroll
            for (int j = 0; j < 4; ++j)
              tc_mma_mx_pair(t_rem, bd + 2 * j, rd + 2 * j, mx_idesc(kMxTileM, ns, j), (kb | j) != 0,
                             t_ssfa | ((uint32_t)j << 30), t_ssfb | ((uint32_t)j << 30));
          }
          tc_commit_pair_both(empty0 + 8 * stage);
          if (++stage == S) { stage = 0; phase ^= 1u; }
        }
        if (!ok) break;
        {
          const int ki = fd ? 2 : hf ? 1 : 0;
          instr_add(IS_FULL_N + 2 * ki, 1);
          instr_add(IS_FULL_CYC + 2 * ki, instr_clock() - tk0);
          instr_add(IS_FULL_K + ki, ksteps);
          instr_add(IS_KSTEPS, ksteps);
        }
        tc_commit_pair_both(tfull);
      }
      instr_add(IS_MMA_TOTAL, instr_clock() - ti0);
    }
  } else {
    // ---------------- epilogue (warps 2..9 of both CTAs) ----------------
    const int q = warp & 3;                 // TMEM lane quarter this warp may read
    const int h = (warp - 2) >> 2;          // column half: TMEM columns 128 h .. 128 h + 127
    const uint32_t tempty_leader = map_to_cta(tempty, 0);
    const uint32_t tempty_rem_leader = map_to_cta(tempty_rem, 0);
    uint32_t acc_phase = 0;
    uint32_t xk = 0;                        // gate/up hand-overs of folded remainders so far
    const bool instr_epi = warp == 2 && lane == 0;
    const long long ti0 = instr_clock();
    for (int qi = 0;; ++qi) {
      const int tile = tq_take<true>(qi, qfull0, qempty_sched, tq, abort_flag, p.status);
      if (__any_sync(0xffffffffu, tile < 0)) break;
      int g, m, n;
      decode_tile(tile, mt, G, nb, g, m, n);
      bool ok = true;
      const long long tw = instr_clock();
      if (lane == 0) ok = mbar_wait(tfull, acc_phase, abort_flag, p.status);
      if (instr_epi) instr_add(IS_EPI_WAIT, instr_clock() - tw);
      if (!__all_sync(0xffffffffu, ok)) break;
      acc_phase ^= 1u;
      tc_fence_after();
      const int grows = off[g + 1] - off[g];
      int ns;
      const bool fd = FOLD && mx_is_fold(grows, m, fold, ns);
      const bool hf = !fd && mx_is_half(grows, m, p.half);
      // M = 256: this CTA's rows 0..127 in lanes 0..127, tile columns 0..255; this warp takes
      //   columns 128 h .. + 127 of lanes 32 q ...
      // M = 128: this CTA's rows 0..63 in lanes 0..63 for tile columns [0, 128) and in lanes
      //   64..127 for [128, 256), at TMEM columns 0..127; this warp takes 64 of them (SwiGLU:
      //   32 gate and the matching 32 up columns).
      // Folded: also the remainder product, CTA's weight row 32 q + lane x remainder rows
      //   [h ns / 2, (h + 1) ns / 2) at TMEM columns kRemCol + ...
      const uint32_t tl = tmem_base + ((uint32_t)(q * 32) << 16);
      uint32_t v0[32], v1[32], v2[32], v3[32];
      if (!hf) {
        tmem_ld32(tl + h * 128, v0);
        tmem_ld32(tl + h * 128 + 32, v1);
        tmem_ld32(tl + h * 128 + 64, v2);
        tmem_ld32(tl + h * 128 + 96, v3);
      } else if (EPI == EPI_SWIGLU) {
        tmem_ld32(tl + h * 32, v0);
        tmem_ld32(tl + 64 + h * 32, v2);
      } else {
        tmem_ld32(tl + h * 64, v0);
        tmem_ld32(tl + h * 64 + 32, v1);
      }
      tmem_ld_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(tempty_leader);      // the accumulator may be reused
      const int r = hf ? (q & 1) * 32 + lane : q * 32 + lane;
      const int64_t row = (int64_t)off[g] + m * kMxTileM + (int)rank * (hf ? 64 : 128) + r;
      // the activation's scales go to the down projection's tile mt[g] + m (the same
      // tiling), CTA half `rank`, row r
      const int qk = p.ldo / C::KS;
      const int64_t t = (int64_t)mt[g] + m;
      if (row >= off[g + 1]) {
        // a row past the group's end: nothing to store
      } else if (!hf) {
        if (EPI == EPI_STORE) {
          bf16* dst = p.out + row * p.ldo + n * BN + h * 128;
          store32(dst, v0);
          store32(dst + 32, v1);
          store32(dst + 64, v2);
          store32(dst + 96, v3);
        } else if (EPI == EPI_SWIGLU) {
          // [gate 64 | up 64] -> outputs n*128 + 64h + [0, 64): K step n, blocks 2h, 2h + 1
          uint8_t* dst = p.q_out + row * p.ldo + n * 128 + h * 64;
          const uint32_t s0 = quant_swiglu32(v0, v2, dst), s1 = quant_swiglu32(v1, v3, dst + 32);
          *reinterpret_cast<uint16_t*>(p.q_sf + mx_sfa_offset(t, qk, n, (int)rank, r, 2 * h)) =
              (uint16_t)(s0 | (s1 << 8));
        } else {
          // GELU: outputs n*256 + 128h + [0, 128): K step 2n + h, blocks 0..3
          uint8_t* dst = p.q_out + row * p.ldo + n * BN + h * 128;
          const int s = 2 * n + h;
          const uint32_t s0 = quant_gelu32(v0, dst), s1 = quant_gelu32(v1, dst + 32);
          const uint32_t s2 = quant_gelu32(v2, dst + 64), s3 = quant_gelu32(v3, dst + 96);
          *reinterpret_cast<uint32_t*>(p.q_sf + mx_sfa_offset(t, qk, s, (int)rank, r, 0)) =
              s0 | (s1 << 8) | (s2 << 16) | (s3 << 24);
        }
      } else {
        const int cq = q >> 1;               // tile columns 128 cq .. 128 cq + 127
        if (EPI == EPI_STORE) {
          bf16* dst = p.out + row * p.ldo + n * BN + cq * 128 + h * 64;
          store32(dst, v0);
          store32(dst + 32, v1);
        } else if (EPI == EPI_SWIGLU) {
          // outputs n*128 + 64 cq + 32 h + [0, 32): K step n, block 2 cq + h
          uint8_t* dst = p.q_out + row * p.ldo + n * 128 + cq * 64 + h * 32;
          p.q_sf[mx_sfa_offset(t, qk, n, (int)rank, r, 2 * cq + h)] = quant_swiglu32(v0, v2, dst);
        } else {
          // outputs n*256 + 128 cq + 64 h + [0, 64): K step 2n + cq, blocks 2h, 2h + 1
          uint8_t* dst = p.q_out + row * p.ldo + n * BN + cq * 128 + h * 64;
          const int s = 2 * n + cq;
          const uint32_t s0 = quant_gelu32(v0, dst), s1 = quant_gelu32(v1, dst + 32);
          *reinterpret_cast<uint16_t*>(p.q_sf + mx_sfa_offset(t, qk, s, (int)rank, r, 2 * h)) =
              (uint16_t)(s0 | (s1 << 8));
        }
      }
      __syncwarp();
      if (FOLD && fd) {
        uint32_t ra[16], rb[16];
        tc_fence_after();
        tmem_ld16(tl + C::kRemCol + h * (ns / 2), ra);
        if (ns == 64) tmem_ld16(tl + C::kRemCol + h * 32 + 16, rb);
        tmem_ld_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive_cluster(tempty_rem_leader);   // the remainder may be reused
        // The remainder: rows rbase + c, c in [h ns / 2, (h + 1) ns / 2) (local cc), and the
        // CTA's weight row wm = 32 q + lane, i.e. per 256-wide N block n: paired, the gate
        // (wm < 64) or up (wm >= 64) factor of output n*128 + 64 rank + wm % 64; plain,
        // output n*256 + 128 rank + wm.  Stores go one element per lane (a warp writes 32
        // consecutive outputs of a row); the activation is quantised across the warp's
        // 32 lanes, one block per remainder row.
        const int64_t rbase = (int64_t)off[g] + kMxTileM;
        const int nh = ns / 2;
        const int c0 = h * nh;
        if (EPI == EPI_STORE) {
          const int col = n * BN + (int)rank * 128 + q * 32 + lane;
#pragma unroll
          for (int cc = 0; cc < 32; ++cc) {
            if (cc < nh && rbase + c0 + cc < off[g + 1])
              p.out[(rbase + c0 + cc) * p.ldo + col] = __float2bfloat16_rn(__uint_as_float(cc < 16 ? ra[cc] : rb[cc - 16]));
          }
        } else if (EPI == EPI_GELU) {
          const int col = n * BN + (int)rank * 128 + q * 32 + lane;
          const int ks = col / C::KS, jb = (col / 32) & 3;
#pragma unroll
          for (int cc = 0; cc < 32; ++cc) {
            if (cc < nh && rbase + c0 + cc < off[g + 1]) {       // warp-uniform
              uint8_t sc;
              const uint8_t qv = mx_quant_lanes(gelu_f(__uint_as_float(cc < 16 ? ra[cc] : rb[cc - 16])), sc);
              p.q_out[(rbase + c0 + cc) * p.ldo + col] = qv;
              if (lane == 0) p.q_sf[mx_sfa_offset(t, qk, ks, 2, c0 + cc, jb)] = sc;
            }
          }
        } else {
          // SwiGLU: the up factors (quarters 2, 3) pass through xbuf[h] to the gate warps
          float* xb = xbuf + h * (64 * 32);
          const uint32_t xfull = xbar0 + 8 * h, xempty = xbar0 + 16 + 8 * h;
          const int i = (q & 1) * 32 + lane;                // output among the CTA's 64
          const uint32_t par = xk & 1u;
          ++xk;
          bool xok = true;
          if (q >= 2) {
            if (lane == 0) xok = mbar_wait(xempty, par ^ 1u, abort_flag, p.status);
            if (!__all_sync(0xffffffffu, xok)) break;
#pragma unroll
            for (int cc = 0; cc < 32; ++cc)
              if (cc < nh) xb[cc * 64 + i] = __uint_as_float(cc < 16 ? ra[cc] : rb[cc - 16]);
            __syncwarp();
            if (lane == 0) mbar_arrive(xfull);
          } else {
            if (lane == 0) xok = mbar_wait(xfull, par, abort_flag, p.status);
            if (!__all_sync(0xffffffffu, xok)) break;
            float u[32];
#pragma unroll
            for (int cc = 0; cc < 32; ++cc) u[cc] = cc < nh ? xb[cc * 64 + i] : 0.f;
            __syncwarp();
            if (lane == 0) mbar_arrive(xempty);              // xbuf[h] may be rewritten
            const int col = n * 128 + (int)rank * 64 + i;    // a 32-block: lanes 0..31 of this warp
            const int ks = col / C::KS, jb = (col / 32) & 3;
#pragma unroll
            for (int cc = 0; cc < 32; ++cc) {
              if (cc < nh && rbase + c0 + cc < off[g + 1]) {     // warp-uniform
                uint8_t sc;
                const uint8_t qv = mx_quant_lanes(silu_f(__uint_as_float(cc < 16 ? ra[cc] : rb[cc - 16])) * u[cc], sc);
                p.q_out[(rbase + c0 + cc) * p.ldo + col] = qv;
                if (lane == 0) p.q_sf[mx_sfa_offset(t, qk, ks, 2, c0 + cc, jb)] = sc;
              }
            }
          }
        }
        __syncwarp();
      }
    }
    if (instr_epi) instr_add(IS_EPI_TOTAL, instr_clock() - ti0);
  }

  // Neither CTA leaves (or frees TMEM) while the pair's MMAs may still touch it.
  __syncwarp();
  tc_fence_before();
  cluster_sync();
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem_base),
                 "r"(C::kTmemCols)
                 : "memory");
  }
}

bool make_map_u8(CUtensorMap* m, const void* base, int rank, const uint64_t* dims, uint32_t box_outer) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t d[3] = {dims[0], dims[1], rank > 2 ? dims[2] : 1};
  cuuint64_t strides[2] = {dims[0], dims[0] * dims[1]};
  cuuint32_t box[3] = {(cuuint32_t)MxCfg::KS, box_outer, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, rank, const_cast<void*>(base), d, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Scale blocks viewed as rows of 256 bytes; a box of `box_rows` rows (2: one block, 4: two).
bool make_map_sf(CUtensorMap* m, const void* base, size_t bytes, uint32_t box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn || bytes % 256 != 0 || bytes == 0) return false;
  cuuint64_t d[2] = {256, bytes / 256};
  cuuint64_t strides[1] = {256};
  cuuint32_t box[2] = {256, box_rows};
  cuuint32_t estr[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), d, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int EPI, bool FOLD>
cudaError_t launch_mx(const MxArgs& a, int clusters, cudaStream_t s) {
  const size_t smem = MxCfgT<FOLD>::smem_bytes(a.G);
  auto kern = grouped_gemm_mx_kernel<EPI, FOLD>;
  cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (err != cudaSuccess) return err;
  cudaLaunchConfig_t cfg;
  memset(&cfg, 0, sizeof(cfg));
  cfg.gridDim = dim3(2 * clusters, 1, 1);
  cfg.blockDim = dim3(kMxThreads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  err = cudaLaunchKernelEx(&cfg, kern, a);
  if (err != cudaSuccess) return err;
  return cudaGetLastError();
}

// B's scale blocks from row-major scales [G * N, K/32] (N % 256 == 0): one thread per
// (row, K step) moves the row's four scales as one word.  Tile t of B is rows
// [256 t, 256 t + 256) of the stacked [G * N] rows.
__global__ void __launch_bounds__(256)
mx_block_scales_kernel(const uint32_t* __restrict__ rowmajor, uint8_t* __restrict__ blocked, int64_t rows,
                       int ksteps) {
  const int64_t n = rows * ksteps;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t row = i / ksteps;
    const int s = (int)(i % ksteps);
    const int64_t t = row / kMxTileM;
    const int h = (int)((row / 128) & 1), m = (int)(row % 128);
    *reinterpret_cast<uint32_t*>(blocked + mx_sf_offset(t, ksteps, s, h, m, 0)) = __ldg(rowmajor + i);
  }
}

// Rows of A -> E4M3 rows with A's scale blocks.  One warp per row: the row's group (binary
// search of the offsets), its M tile and place in it, then 32-element blocks lane-strided.
// Row r's bf16 source is x[r] (x_perm), or, with src, x[src[r] / k]: the dispatch itself
// ("Expert Parallel (EP)", Communication Pattern step 2: each chosen expert gets a copy
// of the token), so the bf16 x_perm is never written.
__global__ void __launch_bounds__(256)
mx_quant_a_kernel(const bf16* __restrict__ x, const int32_t* __restrict__ src, int k,
                  const int32_t* __restrict__ group_offsets, int G, int K, int half, int fold,
                  uint8_t* __restrict__ q, uint8_t* __restrict__ sf) {
  extern __shared__ int sh[];
  int* mt = sh;                 // [G + 1]
  int* off = sh + (G + 1);      // [G + 1]
  int* wsum = off + (G + 1);    // [8]
  for (int i = threadIdx.x; i <= G; i += blockDim.x) off[i] = group_offsets[i];
  __syncthreads();
  group_tile_prefix(off, G, mt, wsum, [fold](int rows) { return mx_mtiles(rows, fold); });
  const int lane = threadIdx.x & 31;
  const int warps = (int)(gridDim.x * blockDim.x) >> 5;
  const int nblk = K / 32, ksteps = K / MxCfg::KS;
  const int rows = off[G];
  for (int r = (int)((blockIdx.x * blockDim.x + threadIdx.x) >> 5); r < rows; r += warps) {
    int lo = 0, hi = G;           // off[lo] <= r < off[hi]
    while (hi - lo > 1) {
      const int mid = (lo + hi) >> 1;
      if (off[mid] <= r) lo = mid; else hi = mid;
    }
    const int rr = r - off[lo];
    int dt, h, m;
    mx_a_place(off[lo + 1] - off[lo], rr, half, fold, dt, h, m);
    const int64_t t = (int64_t)mt[lo] + dt;
    const bf16* xr = x + (src != nullptr ? (int64_t)(__ldg(src + r) / k) : (int64_t)r) * K;
    // lane b takes block b (coalesced); the four blocks of a K step sit in four
    // consecutive lanes (nblk % 4 == 0), whose scales go out as one word
    for (int b0 = 0; b0 < nblk; b0 += 32) {
      const int b = b0 + lane;
      const bool ok = b < nblk;
      uint32_t sc = 0;
      if (ok) {
        const uint4* xs = reinterpret_cast<const uint4*>(xr + b * 32);
        float v[32];
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          const uint4 u = __ldg(xs + c);
          const __nv_bfloat162* hh = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const float2 f = __bfloat1622float2(hh[i]);
            v[8 * c + 2 * i] = f.x;
            v[8 * c + 2 * i + 1] = f.y;
          }
        }
        sc = mx_quant32(v, q + (int64_t)r * K + b * 32);
      }
      const uint32_t s1 = __shfl_down_sync(0xffffffffu, sc, 1);
      const uint32_t s2 = __shfl_down_sync(0xffffffffu, sc, 2);
      const uint32_t s3 = __shfl_down_sync(0xffffffffu, sc, 3);
      if (ok && (lane & 3) == 0)
        *reinterpret_cast<uint32_t*>(sf + mx_sfa_offset(t, ksteps, b >> 2, h, m, 0)) =
            sc | (s1 << 8) | (s2 << 16) | (s3 << 24);
    }
  }
}

}  // namespace

size_t mx_sf_bytes(int64_t tiles, int K) { return (size_t)tiles * (K / MxCfg::KS) * 1024; }
size_t mx_sfa_bytes(int64_t tiles, int K) { return (size_t)tiles * (K / MxCfg::KS) * 1536; }

cudaError_t launch_mx_block_scales(const uint8_t* rowmajor, uint8_t* blocked, int64_t rows, int K,
                                   cudaStream_t s) {
  if (rows % kMxTileM != 0 || K % MxCfg::KS != 0) return cudaErrorInvalidValue;
  const int64_t n = rows * (K / MxCfg::KS);
  if (n == 0) return cudaSuccess;
  int64_t grid = (n + 255) / 256;
  if (grid > 8 * (int64_t)sm_count()) grid = 8 * (int64_t)sm_count();
  mx_block_scales_kernel<<<(int)grid, 256, 0, s>>>(reinterpret_cast<const uint32_t*>(rowmajor), blocked, rows,
                                                   K / MxCfg::KS);
  return cudaGetLastError();
}

cudaError_t launch_mx_quant_a(const bf16* x, const int32_t* src, int k, int64_t rows,
                              const int32_t* group_offsets, int G, int K, int half_tiles, int fold, uint8_t* q,
                              uint8_t* sf, cudaStream_t s) {
  if (K % MxCfg::KS != 0 || G <= 0) return cudaErrorInvalidValue;
  if (rows == 0) return cudaSuccess;
  const size_t smem = (2 * (size_t)(G + 1) + 8) * sizeof(int);
  if (smem > 48 * 1024) return cudaErrorInvalidValue;
  int64_t grid = (rows + 7) / 8;                 // 8 rows (warps) per block
  if (grid > 4 * (int64_t)sm_count()) grid = 4 * (int64_t)sm_count();
  mx_quant_a_kernel<<<(int)grid, 256, smem, s>>>(x, src, k, group_offsets, G, K, half_tiles, fold, q, sf);
  return cudaGetLastError();
}

cudaError_t launch_grouped_mx(const MxProblem& p, cudaStream_t s) {
  if (p.N % MxCfg::BN != 0 || p.K % MxCfg::KS != 0 || p.counter == nullptr || p.group_offsets == nullptr ||
      p.G <= 0)
    return cudaErrorInvalidValue;
  if (p.epi != EPI_STORE && (p.ldo % MxCfg::KS != 0 || p.q_out == nullptr || p.q_sf == nullptr))
    return cudaErrorInvalidValue;
  const int64_t tiles_m = p.a_rows / kMxTileM + p.G;      // at least the sum of ceil(rows_g / 256)
  MxArgs a;
  memset(&a, 0, sizeof(a));
  const uint64_t da[2] = {(uint64_t)p.K, (uint64_t)p.a_rows};
  const uint64_t db[3] = {(uint64_t)p.K, (uint64_t)p.N, (uint64_t)p.G};
  const size_t sfb_bytes = mx_sf_bytes((int64_t)p.G * (p.N / MxCfg::BN), p.K);
  if (!make_map_u8(&a.tmap_a, p.A, 2, da, 128) || !make_map_u8(&a.tmap_a64, p.A, 2, da, 64) ||
      !make_map_u8(&a.tmap_a32, p.A, 2, da, 32) || !make_map_u8(&a.tmap_b, p.B, 3, db, 128) ||
      !make_map_sf(&a.tmap_sfa, p.sa, mx_sfa_bytes(tiles_m, p.K), 2) ||
      !make_map_sf(&a.tmap_sfb, p.sb, sfb_bytes, 4) || !make_map_sf(&a.tmap_sfb1, p.sb, sfb_bytes, 2))
    return cudaErrorInvalidValue;
  a.group_offsets = p.group_offsets;
  a.G = p.G;
  a.N = p.N;
  a.K = p.K;
  a.out = p.out;
  a.ldo = p.ldo;
  a.q_out = p.q_out;
  a.q_sf = p.q_sf;
  a.half = p.half_tiles;
  a.fold = p.fold;
  a.status = p.status;
  a.counter = p.counter;
  const int64_t tiles = tiles_m * (int64_t)(p.N / MxCfg::BN);
  const int pairs = sm_count() / 2;
  const int clusters = (int)(tiles < pairs ? (tiles > 0 ? tiles : 1) : pairs);
  if (p.fold > 0) {
    if (p.epi == EPI_SWIGLU) return launch_mx<EPI_SWIGLU, true>(a, clusters, s);
    if (p.epi == EPI_GELU) return launch_mx<EPI_GELU, true>(a, clusters, s);
    return launch_mx<EPI_STORE, true>(a, clusters, s);
  }
  if (p.epi == EPI_SWIGLU) return launch_mx<EPI_SWIGLU, false>(a, clusters, s);
  if (p.epi == EPI_GELU) return launch_mx<EPI_GELU, false>(a, clusters, s);
  return launch_mx<EPI_STORE, false>(a, clusters, s);
}

// The MXFP8 kernel's cycle counters (instrumented builds; else not supported).
cudaError_t instr_read_mx(unsigned long long* host, int n) { return instr_read_tu(host, n); }

}  // namespace moe

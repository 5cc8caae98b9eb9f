// Grouped expert GEMM with MXFP8 operands on the 5th-generation tensor cores:
// tcgen05.mma.kind::mxf8f6f4.block_scale, E4M3 A and B, one E8M0 scale per 32 K.
//
// torchtitan issue 5554 (shared-expert overlap) lists MXFP8 routed experts as an
// option; "Expert Parallel (EP)", Communication Pattern step 3 and "Worked Example:
// Tracing a Token Through Expert Parallelism", Step 3 fix what runs: each expert's
// two-layer FFN over its rows of the rank-major buffer.  The format is OCP MX v1.0
// MXFP8 (E4M3): out[row, :] = epilogue( sum_k qa[row,k] 2^sa[row,k/32] qb[n,k] 2^sb[n,k/32] ),
// accumulated in fp32 by the tensor cores (the scaled products are exact).
//
//   A   E4M3 [rows, K] (K-major) with its scales sa [rows, K/32] (row-major bytes,
//       s + 127), from moe_mxfp8_quantize; rows of group g at [off[g], off[g+1]);
//   B   E4M3 [G, N, K] (K-major) with its scales pre-arranged in the tensor cores'
//       block order: for group g, 128-row block n and 128-deep K step s, 512 bytes at
//       ((g * N/128 + n) * K/128 + s) * 512, row r's four scales (K blocks 4s..4s+3)
//       at byte 16 (r % 32) + 4 (r / 32).
//
// One CTA per SM, 128 x 128 output tiles, 6 warps as in the bf16 one-CTA kernel:
//   warp 0      producer: every lane gathers four rows' scale words of the A tile
//               into the 512-byte block order (one 16-byte store per lane), then lane 0
//               posts the stage's expected bytes and issues the A and B tile loads (TMA,
//               128 rows x 128 bytes, 128-byte swizzle) and B's 512-byte scale block
//               (bulk copy) into a 6-stage ring;
//   warp 1      allocates 512 TMEM columns (two 128-column accumulators, A and B scale
//               columns at 256 and 260); one lane copies the stage's scale blocks into
//               TMEM (tcgen05.cp 32x128b, broadcast to the four lane quarters) and issues
//               four M=128 N=128 K=32 block-scaled MMAs, scale block j selected by the
//               scale-id fields; commits free the stage and hand over the accumulator;
//   warps 2-5   epilogue (tcgen05.ld, activation, bf16 rows masked at the group end).
// The scale columns are rewritten every stage: tcgen05 operations of one thread run in
// issue order, so a stage's copy lands after the previous stage's MMAs have read theirs.
// Every wait is bounded and reports MOE_ERR_TIMEOUT.  The accumulators and scale columns
// need 264 TMEM columns, so the tile is 128 wide: two 256-wide accumulators would fill TMEM.
#include "tc_common.cuh"

namespace moe {

namespace {

struct MxArgs {
  CUtensorMap tmap_a;        // E4M3 [rows, K], box 128 x 128 bytes
  CUtensorMap tmap_b;        // E4M3 [G, N, K], box 128 x 128 x 1
  const uint32_t* sa;        // A scales as 32-bit words: [rows, K/128] (four K blocks each)
  const uint8_t* sb;         // B scales, block order (see above)
  const int32_t* group_offsets;
  int32_t G, N, K, a_rows;
  bf16* out;
  int32_t ldo;
  int32_t* status;
  int32_t* counter;          // tile counter, zero at launch
};

struct MxCfg {
  static constexpr int BN = 128;
  static constexpr int KS = 128;                     // K elements (bytes) per stage
  static constexpr int kStages = 6;
  static constexpr int kABytes = kTileM * KS;        // 16 KB
  static constexpr int kBBytes = BN * KS;            // 16 KB
  static constexpr int kSfBytes = 512;
  static constexpr int kStageBytes = kABytes + kBBytes + 2 * kSfBytes;
  static constexpr int kTmemCols = 512;
  static constexpr int kSfaCol = 256, kSfbCol = 260;
  static size_t smem_bytes(int G) {
    return 1024 + (size_t)kStages * kStageBytes + kCtrlBytes + 2 * (size_t)(G + 1) * sizeof(int);
  }
};

// Block-scaled instruction descriptor, kind::mxf8f6f4: E4M3 A and B, K-major, E8M0 scales,
// scale block `j` of A and of B (bits 29-30 and 4-5).
__host__ __device__ constexpr uint32_t mx_idesc(int M, int N, int j) {
  return ((uint32_t)j << 4) | ((uint32_t)(N >> 3) << 17) | (1u << 23) | ((uint32_t)(M >> 4) << 24) |
         ((uint32_t)j << 29);
}

// Shared-memory descriptor of a 512-byte scale block for tcgen05.cp: no swizzle,
// K-major, 8-row core matrices of 16 bytes placed 128 bytes apart.
__device__ __forceinline__ uint64_t sf_desc(uint32_t saddr) {
  return (uint64_t)((saddr & 0x3FFFFu) >> 4) | ((uint64_t)(128 >> 4) << 32) | ((uint64_t)1 << 46);
}

__device__ __forceinline__ void tc_cp_sf(uint32_t taddr, uint64_t sdesc) {
  asm volatile("tcgen05.cp.cta_group::1.32x128b.warpx4 [%0], %1;" ::"r"(taddr), "l"(sdesc) : "memory");
}

__device__ __forceinline__ void tc_mma_mx(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                          uint32_t accumulate, uint32_t sfa, uint32_t sfb) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::mxf8f6f4.block_scale [%0], %1, %2, %3, [%5], [%6], p;\n\t}" ::"r"(
          d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(sfa), "r"(sfb)
      : "memory");
}

__device__ __forceinline__ void bulk_load(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(bar)
      : "memory");
}

template <int EPI>
__global__ void __launch_bounds__(kGemmThreads, 1) grouped_gemm_mx_kernel(const __grid_constant__ MxArgs p) {
  using C = MxCfg;
  constexpr int S = C::kStages, BN = C::BN;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + ((1024u - (raw_addr & 1023u)) & 1023u);
  uint8_t* a_smem = smem;
  uint8_t* b_smem = smem + S * C::kABytes;
  uint8_t* sfa_smem = smem + S * (C::kABytes + C::kBBytes);
  uint8_t* sfb_smem = sfa_smem + S * C::kSfBytes;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + S * C::kStageBytes);
  // bars: full[S], empty[S], tmem_full[2], tmem_empty[2], qfull[Q], qempty[Q]
  volatile int* tq = reinterpret_cast<volatile int*>(bars + 2 * S + 4 + 2 * kTileQ);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(const_cast<int*>(tq) + kTileQ);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  int* wsum = const_cast<int*>(abort_flag) + 1;
  int* mt = reinterpret_cast<int*>(smem + S * C::kStageBytes + kCtrlBytes);
  const int G = p.G;
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
  for (int i = threadIdx.x; i <= G; i += blockDim.x) off[i] = p.group_offsets[i];
  __syncthreads();
  group_tile_prefix(off, G, mt, wsum, [](int rows) { return (rows + kTileM - 1) / kTileM; });
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
  const int ksteps = p.K / C::KS;
  const uint32_t qempty_sched = qempty0;

  if (warp == 0) {
    // ---------------- producer: scale gather (all lanes), TMA and bulk copies (lane 0) ----------------
    int stage = 0;
    uint32_t phase = 0;
    int next = 0;
    if (lane == 0) next = atomicAdd(p.counter, 1);
    for (int qi = 0;; ++qi) {
      int tile = 0;
      if (lane == 0) tile = tq_post<false>(p.counter, next, total, qi, qfull0, qempty0, tq, abort_flag, p.status);
      tile = __shfl_sync(0xffffffffu, tile, 0);
      if (tile < 0) break;
      int g, m, n;
      decode_tile(tile, mt, G, nb, g, m, n);
      const int row0 = off[g] + m * kTileM;
      const uint8_t* sb_tile = p.sb + ((size_t)g * nb + n) * ksteps * C::kSfBytes;
      bool ok = true;
      for (int kb = 0; kb < ksteps; ++kb) {
        int w = 1;
        if (lane == 0) w = mbar_wait(empty0 + 8 * stage, phase ^ 1u, abort_flag, p.status) ? 1 : 0;
        if (!__shfl_sync(0xffffffffu, w, 0)) { ok = false; break; }
        // this lane's rows lane, lane + 32, lane + 64, lane + 96: one word each (the four
        // scales of the stage's K blocks); rows past the tensor take scale 0 (2^-127)
        uint4 v;
        uint32_t* vw = reinterpret_cast<uint32_t*>(&v);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const int r = row0 + lane + 32 * j;
          vw[j] = r < p.a_rows ? __ldg(p.sa + (size_t)r * ksteps + kb) : 0u;
        }
        *reinterpret_cast<uint4*>(sfa_smem + stage * C::kSfBytes + 16 * lane) = v;
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        __syncwarp();
        if (lane == 0) {
          const uint32_t fb = full0 + 8 * stage;
          mbar_arrive_expect_tx(fb, C::kABytes + C::kBBytes + C::kSfBytes);
          tma_load_2d(smem_u32(a_smem + stage * C::kABytes), &p.tmap_a, fb, kb * C::KS, row0);
          tma_load_3d(smem_u32(b_smem + stage * C::kBBytes), &p.tmap_b, fb, kb * C::KS, n * BN, g);
          bulk_load(smem_u32(sfb_smem + stage * C::kSfBytes), sb_tile + (size_t)kb * C::kSfBytes,
                    C::kSfBytes, fb);
        }
        if (++stage == S) { stage = 0; phase ^= 1u; }
      }
      if (!ok) break;
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ---------------- scale copies and block-scaled MMAs ----------------
      const uint32_t t_sfa = tmem_base + C::kSfaCol, t_sfb = tmem_base + C::kSfbCol;
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
          tc_cp_sf(t_sfa, sf_desc(smem_u32(sfa_smem + stage * C::kSfBytes)));
          tc_cp_sf(t_sfb, sf_desc(smem_u32(sfb_smem + stage * C::kSfBytes)));
          const uint64_t ad = sw128_desc(smem_u32(a_smem + stage * C::kABytes));
          const uint64_t bd = sw128_desc(smem_u32(b_smem + stage * C::kBBytes));
#pragma unroll
          for (int j = 0; j < 4; ++j)          // K = 32 per MMA: +32 bytes
            tc_mma_mx(d_tmem, ad + 2 * j, bd + 2 * j, mx_idesc(kTileM, BN, j), (kb | j) != 0,
                      t_sfa | ((uint32_t)j << 30), t_sfb | ((uint32_t)j << 30));
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
      if (!__all_sync(0xffffffffu, ok)) break;
      tc_fence_after();
      const int r = q * 32 + lane;
      const uint32_t tb = tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)(acc * BN);
      const bool paired = EPI == EPI_SWIGLU;
      epilogue_row<EPI>(p.out, nullptr, p.ldo, tb, 0, paired ? BN / 2 : BN, (int64_t)row0 + r,
                        paired ? n * (BN / 2) : n * BN, r < rows_valid);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(tempty0 + 8 * acc);
      acc ^= 1;
      if (acc == 0) acc_phase ^= 1u;
    }
  }

  __syncwarp();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base),
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

template <int EPI>
cudaError_t launch_mx(const MxArgs& a, int grid, cudaStream_t s) {
  const size_t smem = MxCfg::smem_bytes(a.G);
  auto kern = grouped_gemm_mx_kernel<EPI>;
  cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (err != cudaSuccess) return err;
  kern<<<grid, kGemmThreads, smem, s>>>(a);
  return cudaGetLastError();
}

// Scale blocks of a B operand in the order above, from row-major scales [G * N, K/32]:
// one thread per (row, K step) writes the row's four scales as one word.
__global__ void __launch_bounds__(256)
mx_block_scales_kernel(const uint32_t* __restrict__ rowmajor, uint32_t* __restrict__ blocked, int64_t rows,
                       int ksteps) {
  const int64_t n = rows * ksteps;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t row = i / ksteps;
    const int kb = (int)(i % ksteps);
    const int64_t blk = row / 128;
    const int r = (int)(row % 128);
    // block (blk, kb) holds 128 words; row r's word at (16 (r % 32) + 4 (r / 32)) / 4
    blocked[(blk * ksteps + kb) * 128 + 4 * (r % 32) + r / 32] = __ldg(rowmajor + i);
  }
}

}  // namespace

cudaError_t launch_mx_block_scales(const uint8_t* rowmajor, uint8_t* blocked, int64_t rows, int K,
                                   cudaStream_t s) {
  if (rows % 128 != 0 || K % 128 != 0) return cudaErrorInvalidValue;
  const int64_t n = rows * (K / 128);
  if (n == 0) return cudaSuccess;
  int64_t grid = (n + 255) / 256;
  if (grid > 8 * (int64_t)sm_count()) grid = 8 * (int64_t)sm_count();
  mx_block_scales_kernel<<<(int)grid, 256, 0, s>>>(reinterpret_cast<const uint32_t*>(rowmajor),
                                                   reinterpret_cast<uint32_t*>(blocked), rows, K / 128);
  return cudaGetLastError();
}

cudaError_t launch_grouped_mx(const MxProblem& p, cudaStream_t s) {
  if (p.N % MxCfg::BN != 0 || p.K % MxCfg::KS != 0 || p.counter == nullptr || p.group_offsets == nullptr)
    return cudaErrorInvalidValue;
  MxArgs a;
  memset(&a, 0, sizeof(a));
  const uint64_t da[2] = {(uint64_t)p.K, (uint64_t)p.a_rows};
  const uint64_t db[3] = {(uint64_t)p.K, (uint64_t)p.N, (uint64_t)p.G};
  if (!make_map_u8(&a.tmap_a, p.A, 2, da, kTileM) || !make_map_u8(&a.tmap_b, p.B, 3, db, MxCfg::BN))
    return cudaErrorInvalidValue;
  a.sa = reinterpret_cast<const uint32_t*>(p.sa);
  a.sb = p.sb;
  a.group_offsets = p.group_offsets;
  a.G = p.G;
  a.N = p.N;
  a.K = p.K;
  a.a_rows = (int32_t)p.a_rows;
  a.out = p.out;
  a.ldo = p.ldo;
  a.status = p.status;
  a.counter = p.counter;
  const int64_t tiles = (p.a_rows / kTileM + p.G) * (int64_t)(p.N / MxCfg::BN);
  const int grid = (int)(tiles < sm_count() ? (tiles > 0 ? tiles : 1) : sm_count());
  if (p.epi == EPI_SWIGLU) return launch_mx<EPI_SWIGLU>(a, grid, s);
  if (p.epi == EPI_GELU) return launch_mx<EPI_GELU>(a, grid, s);
  return launch_mx<EPI_STORE>(a, grid, s);
}

}  // namespace moe

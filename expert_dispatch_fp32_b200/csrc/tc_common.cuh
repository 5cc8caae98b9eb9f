// Helpers shared by the tcgen05 GEMM kernels (grouped_gemm.cu, grouped_gemm_mx.cu): PTX
// wrappers for mbarriers, TMA, tcgen05 and clusters, the dynamic tile queue, the tile
// order, the epilogue row writers and the host-side tensor-map encoder.  Every
// translation unit that includes this gets its own copy (anonymous namespace).
#pragma once

#include <stdio.h>
#include <stdlib.h>

#include "moe_internal.cuh"

namespace moe {
namespace {

constexpr long long kWaitLimitCycles = 4000000000ll;   // 2 s at 2 GHz (4 s at 1 GHz)
constexpr int kGemmThreads = 192;
constexpr int kCtrlBytes = 512;     // barriers, tile queue, TMEM slot, abort flag

// ---------------------------------------------------------------------------
// Cycle counters of an instrumented build (-DMOE_INSTRUMENT; compiled out otherwise):
// per CTA, kInstrSlots 64-bit sums of SM cycles (clock64), each slot written by one
// thread of its CTA only, read back with moe_instr_read.  They show where a GEMM
// launch's MMA issuer, producer and epilogue spend their cycles, per tile kind.
// ---------------------------------------------------------------------------
constexpr int kInstrSlots = 24;
constexpr int kInstrCtas = 160;     // >= one CTA per SM
enum InstrSlot {
  IS_MMA_TOTAL = 0,   // MMA issuer: the whole tile loop
  IS_MMA_WAIT_ACC,    //   waiting for its accumulator (TMEM) to be drained
  IS_MMA_WAIT_FULL,   //   waiting for a filled stage
  IS_FULL_N,          // tiles of each kind and the issuer's cycles from their first to
  IS_FULL_CYC,        //   their last K step (stage waits included)
  IS_HALF_N,
  IS_HALF_CYC,
  IS_FOLD_N,
  IS_FOLD_CYC,
  IS_SKINNY_N,
  IS_SKINNY_CYC,
  IS_KSTEPS,          // K steps issued
  IS_PROD_WAIT,       // producer (lane 0 of warp 0, both CTAs): waiting for a free stage
  IS_PROD_TOTAL,
  IS_EPI_WAIT,        // first epilogue warp (lane 0): waiting for a full accumulator
  IS_EPI_TOTAL,
  IS_FULL_K,          // K steps of full, M = 128, folded and skinny tiles
  IS_HALF_K,
  IS_FOLD_K,
  IS_SKINNY_K,
};
#ifdef MOE_INSTRUMENT
__device__ unsigned long long g_instr[kInstrCtas * kInstrSlots];
__device__ __forceinline__ long long instr_clock() { return clock64(); }
__device__ __forceinline__ void instr_add(int slot, long long v) {
  if (blockIdx.x < kInstrCtas) g_instr[blockIdx.x * kInstrSlots + slot] += (unsigned long long)v;
}
// Copies this translation unit's counters to host[] (n values at most) and zeroes them.
inline cudaError_t instr_read_tu(unsigned long long* host, int n) {
  const size_t bytes = sizeof(unsigned long long) * (size_t)(n < kInstrCtas * kInstrSlots ? n : kInstrCtas * kInstrSlots);
  cudaError_t e = cudaMemcpyFromSymbol(host, g_instr, bytes);
  if (e != cudaSuccess) return e;
  void* d = nullptr;
  e = cudaGetSymbolAddress(&d, g_instr);
  if (e != cudaSuccess) return e;
  return cudaMemset(d, 0, sizeof(unsigned long long) * kInstrCtas * kInstrSlots);
}
#else
__device__ __forceinline__ long long instr_clock() { return 0; }
__device__ __forceinline__ void instr_add(int, long long) {}
inline cudaError_t instr_read_tu(unsigned long long*, int) { return cudaErrorNotSupported; }
#endif

// ---------------------------------------------------------------------------
// PTX wrappers
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
               : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}
// Same, with cluster-scope acquire (the phase was completed by arrivals that
// release writes made from the other CTA of the cluster).
__device__ __forceinline__ bool mbar_try_wait_cluster(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}

// Wait for phase `parity` of `bar`; false if the wait gave up.  The limit is
// counted in SM clock cycles (clock64 is a cheap register read; %globaltimer is
// not, and reading it on every missed first try stretched the pipeline's
// barrier round trips enough to idle the tensor cores a quarter of the time).
template <bool kCluster>
__device__ __noinline__ bool mbar_wait_slow(uint32_t bar, uint32_t parity, volatile int* abort_flag,
                                            int32_t* status) {
  const long long t0 = clock64();
  for (uint32_t it = 1;; ++it) {
    if (kCluster ? mbar_try_wait_cluster(bar, parity) : mbar_try_wait(bar, parity)) return true;
    if ((it & 63u) == 0) {
      if (*abort_flag) return false;
      if (clock64() - t0 > kWaitLimitCycles) {
        *abort_flag = 1;
        if (status != nullptr) atomicCAS(status, 0, (int32_t)MOE_ERR_TIMEOUT);
        return false;
      }
    }
  }
}
template <bool kCluster = false>
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, volatile int* abort_flag,
                                          int32_t* status) {
  if (kCluster ? mbar_try_wait_cluster(bar, parity) : mbar_try_wait(bar, parity)) return true;
  return mbar_wait_slow<kCluster>(bar, parity, abort_flag, status);
}

__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* map, uint32_t bar,
                                            int c0, int c1) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4}], [%2];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(c0), "r"(c1)
      : "memory");
}
__device__ __forceinline__ void tma_load_3d(uint32_t dst, const CUtensorMap* map, uint32_t bar,
                                            int c0, int c1, int c2) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5}], [%2];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(c0), "r"(c1), "r"(c2)
      : "memory");
}
__device__ __forceinline__ void prefetch_tmap(const CUtensorMap* map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_commit(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                   bar)
               : "memory");
}
__device__ __forceinline__ void tc_mma(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                       uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}
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
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
}
__device__ __forceinline__ void tmem_ld_wait() {
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// ---- CTA-pair (cluster of 2) forms ----
__device__ __forceinline__ uint32_t cluster_ctarank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
__device__ __forceinline__ void cluster_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
// Shared address of the same object in CTA `rank` of the cluster.
__device__ __forceinline__ uint32_t map_to_cta(uint32_t addr, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(addr), "r"(rank));
  return r;
}
__device__ __forceinline__ void mbar_arrive_cluster(uint32_t cluster_addr) {
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr)
               : "memory");
}
__device__ __forceinline__ void st_cluster_u32(uint32_t cluster_addr, int v) {
  asm volatile("st.shared::cluster.u32 [%0], %1;" ::"r"(cluster_addr), "r"(v) : "memory");
}

// ---- Dynamic tile scheduler ----
// One thread (the TMA producer of the CTA, or of the pair's leader) takes tile
// indices in order from a global counter and posts each into a ring of kTileQ
// shared-memory slots; every other role of the CTA (and of the peer CTA of a
// pair, whose slot is written through the cluster window) reads the slot, then
// arrives on the scheduler's `qempty` barrier so the slot can be reused.  A
// posted -1 ends every role.  Taking tiles in order as CTAs become free keeps
// tiles of very different cost (a 256-row tile next to a 128-row remainder)
// balanced across the SMs, and makes the tiles that share a weight tile (the M
// tiles of one expert and N block, consecutive in the order) start within a
// fraction of a tile of each other, so that weight tile is read from HBM once.
constexpr int kTileQ = 8;

template <bool kPair>
__device__ __forceinline__ int tq_post(int32_t* counter, int& next, int total, int qi, uint32_t qfull0,
                                       uint32_t qempty0, volatile int* tq,
                                       volatile int* abort_flag, int32_t* status) {
  const int slot = qi % kTileQ;
  const uint32_t ph = (uint32_t)(qi / kTileQ) & 1u;
  if (!mbar_wait<true>(qempty0 + 8 * slot, ph ^ 1u, abort_flag, status)) return -2;
  // `next` was taken one tile ahead, so the atomic's round trip overlaps the
  // previous tile's loads instead of stalling the pipeline at the tile edge
  int tile = next;
  if (tile >= total) tile = -1;
  else next = atomicAdd(counter, 1);
  tq[slot] = tile;
  if (kPair) st_cluster_u32(map_to_cta(smem_u32((const void*)(tq + slot)), 1), tile);
  mbar_arrive(qfull0 + 8 * slot);
  if (kPair) mbar_arrive_cluster(map_to_cta(qfull0 + 8 * slot, 1));
  return tile;
}

// Consumer side.  kWarp: the whole (converged) warp calls, every lane reads, and
// lane 0 releases the slot after a __syncwarp; otherwise one thread calls and
// releases.  The slot is released on the scheduler's barrier at `qempty_sched`
// (a shared::cluster address).  Returns -2 if the wait gave up.
template <bool kWarp>
__device__ __forceinline__ int tq_take(int qi, uint32_t qfull0, uint32_t qempty_sched,
                                       const volatile int* tq, volatile int* abort_flag,
                                       int32_t* status) {
  const int slot = qi % kTileQ;
  const uint32_t ph = (uint32_t)(qi / kTileQ) & 1u;
  int tile = -2;
  if (!kWarp || (threadIdx.x & 31) == 0) {      // one lane polls; the others wait in the shuffle
    if (mbar_wait<true>(qfull0 + 8 * slot, ph, abort_flag, status)) {
      tile = tq[slot];
      mbar_arrive_cluster(qempty_sched + 8 * slot);
    }
  }
  if (kWarp) tile = __shfl_sync(0xffffffffu, tile, 0);
  return tile;
}

// Loads into this CTA's shared memory whose bytes complete on `leader_bar`, the
// shared::cluster address (from mapa) of the barrier in the pair's leader CTA.
__device__ __forceinline__ void tma_load_2d_pair(uint32_t dst, const CUtensorMap* map,
                                                 uint32_t leader_bar, int c0, int c1) {
  asm volatile(
      "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4}], [%2];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(leader_bar), "r"(c0), "r"(c1)
      : "memory");
}
__device__ __forceinline__ void tma_load_3d_pair(uint32_t dst, const CUtensorMap* map,
                                                 uint32_t leader_bar, int c0, int c1, int c2) {
  asm volatile(
      "cp.async.bulk.tensor.3d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5}], [%2];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(leader_bar), "r"(c0), "r"(c1), "r"(c2)
      : "memory");
}
__device__ __forceinline__ void tc_mma_pair(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                            uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// Arrive once on the barrier at this shared offset in both CTAs of the pair when
// all tcgen05 operations issued so far by this thread have completed.
__device__ __forceinline__ void tc_commit_pair_both(uint32_t bar) {
  const uint16_t mask = 0x3;
  asm volatile(
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;" ::"r"(bar),
      "h"(mask)
      : "memory");
}

// Shared-memory matrix descriptor: K-major operand, 128-byte swizzle, rows of
// 128 bytes, 8-row core groups 1024 bytes apart (SBO), sm_100 descriptor version 1.
__device__ __forceinline__ uint64_t sw128_desc(uint32_t saddr) {
  return (uint64_t)((saddr & 0x3FFFFu) >> 4) | ((uint64_t)1 << 16) | ((uint64_t)(1024 >> 4) << 32) |
         ((uint64_t)1 << 46) | ((uint64_t)2 << 61);
}
// Instruction descriptor, kind::f16: fp32 accumulator, bf16 A and B, both K-major.
__host__ __device__ constexpr uint32_t make_idesc(int M, int N) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(N >> 3) << 17) |
         ((uint32_t)(M >> 4) << 24);
}

// Tile order: group-major; inside a group, M tiles in bands of kBandM, then N
// block, then M tile fastest inside the band.  Tiles that run at the same time
// share each weight tile (B) through L2, and a band's A rows (kBandM tiles of
// rows x K) stay in L2 while every N block of the band reads them, so a group of
// many rows (a dense shared expert, or one expert taking most tokens) reads A
// from HBM about once instead of once per N block.  Groups of at most kBandM
// tiles (the usual case) are plain N-major, M fastest.
constexpr int kBandM = 8;

__device__ __forceinline__ void decode_tile(int tile, const int* mt, int G, int nb, int& g,
                                            int& m, int& n) {
  int lo = 0, hi = G;                      // mt[lo]*nb <= tile < mt[hi]*nb
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (mt[mid] * nb <= tile) lo = mid; else hi = mid;
  }
  g = lo;
  const int mtiles = mt[g + 1] - mt[g];
  const int local = tile - mt[g] * nb;
  const int band = local / (kBandM * nb);
  const int in_full = mtiles / kBandM;             // full bands
  const int bw = band < in_full ? kBandM : mtiles - in_full * kBandM;
  const int rem = local - band * kBandM * nb;
  n = rem / bw;
  m = band * kBandM + (rem - n * bw);
}

// SiLU with the fast exp and divide intrinsics (a few ulp of fp32): its result is rounded to
// bf16 (or quantised) next, and the exact form kept the epilogue on the critical path of
// short-K launches.  g -> -inf gives g / inf = -0, the limit.
__device__ __forceinline__ float silu_f(float g) { return __fdividef(g, 1.0f + __expf(-g)); }
__device__ __forceinline__ float gelu_f(float h) {
  return 0.5f * h * (1.0f + erff(h * 0.70710678118654752f));
}

__device__ __forceinline__ void store_row32(bf16* dst, const float (&v)[32]) {
  uint4* d = reinterpret_cast<uint4*>(dst);
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    uint4 t;
    __nv_bfloat162* h = reinterpret_cast<__nv_bfloat162*>(&t);
#pragma unroll
    for (int i = 0; i < 4; ++i) h[i] = __floats2bfloat162_rn(v[q * 8 + 2 * i], v[q * 8 + 2 * i + 1]);
    d[q] = t;
  }
}

__device__ __forceinline__ void store_row32_f32(float* dst, const float (&v)[32]) {
  float4* d = reinterpret_cast<float4*>(dst);
#pragma unroll
  for (int q = 0; q < 8; ++q) d[q] = make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
}

// Epilogue of one output row: this thread's TMEM columns at `tb` hold accumulator
// values of row `row` (`valid` false: read, store nothing); output columns
// col0 + [cb, ce) are done (a range, so a caller can release the TMEM columns read so
// far before doing the rest).
//   EPI_SWIGLU / EPI_PAIRSUM_F32: every 128 columns are [first 64 | second 64] of
//     64 outputs (packed gate/up or router hi/mid groups); output column
//     col0 + 64 * group + c = silu(first) * second, or first + second in fp32
//     (output columns [0, 64) read TMEM columns [0, 128)).
//   EPI_STORE / EPI_GELU: output column col0 + c = value (or its GELU), TMEM column c.
// tcgen05.ld is warp-collective, so every lane runs the loads.
template <int EPI>
__device__ __forceinline__ void epilogue_row(bf16* out, float* outf, int ldo, uint32_t tb, int cb,
                                             int ce, int64_t row, int col0, bool valid) {
  if (EPI == EPI_SWIGLU || EPI == EPI_PAIRSUM_F32) {
#pragma unroll 1
    for (int c = cb; c < ce; c += 32) {
      const int tc = (c >> 6) * 128 + (c & 63);
      uint32_t a[32], b[32];
      __syncwarp();        // tcgen05.ld is warp-collective: reconverge after the masked stores
      tmem_ld32(tb + tc, a);
      tmem_ld32(tb + tc + 64, b);
      tmem_ld_wait();
      float v[32];
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        const float x = __uint_as_float(a[i]), y = __uint_as_float(b[i]);
        v[i] = (EPI == EPI_SWIGLU) ? silu_f(x) * y : x + y;
      }
      if (valid) {
        if (EPI == EPI_SWIGLU) store_row32(out + row * ldo + col0 + c, v);
        else store_row32_f32(outf + row * ldo + col0 + c, v);
      }
    }
  } else {
#pragma unroll 1
    for (int c = cb; c < ce; c += 32) {
      uint32_t h[32];
      __syncwarp();        // tcgen05.ld is warp-collective: reconverge after the masked stores
      tmem_ld32(tb + c, h);
      tmem_ld_wait();
      float v[32];
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        const float x = __uint_as_float(h[i]);
        v[i] = (EPI == EPI_GELU) ? gelu_f(x) : x;
      }
      if (valid) store_row32(out + row * ldo + col0 + c, v);
    }
  }
}

// Runtime choice of the epilogue (the phases of one launch differ).
__device__ __forceinline__ void epilogue_row_rt(int epi, bf16* out, float* outf, int ldo, uint32_t tb,
                                                int cb, int ce, int64_t row, int col0, bool valid) {
  switch (epi) {
    case EPI_SWIGLU: epilogue_row<EPI_SWIGLU>(out, outf, ldo, tb, cb, ce, row, col0, valid); break;
    case EPI_GELU: epilogue_row<EPI_GELU>(out, outf, ldo, tb, cb, ce, row, col0, valid); break;
    case EPI_PAIRSUM_F32: epilogue_row<EPI_PAIRSUM_F32>(out, outf, ldo, tb, cb, ce, row, col0, valid); break;
    default: epilogue_row<EPI_STORE>(out, outf, ldo, tb, cb, ce, row, col0, valid); break;
  }
}

// 32 output columns at dst from accumulator values a (and b, paired).
template <int EPI>
__device__ __forceinline__ void epilogue_cols32(bf16* out, float* outf, int64_t off, const uint32_t (&a)[32],
                                                const uint32_t (&b)[32]) {
  float v[32];
#pragma unroll
  for (int i = 0; i < 32; ++i) {
    const float x = __uint_as_float(a[i]);
    if (EPI == EPI_SWIGLU) v[i] = silu_f(x) * __uint_as_float(b[i]);
    else if (EPI == EPI_PAIRSUM_F32) v[i] = x + __uint_as_float(b[i]);
    else if (EPI == EPI_GELU) v[i] = gelu_f(x);
    else v[i] = x;
  }
  if (EPI == EPI_PAIRSUM_F32) store_row32_f32(outf + off, v);
  else store_row32(out + off, v);
}

// The first 64 output columns of a row (TMEM columns 0..63, and 64..127 for a paired
// epilogue) with the TMEM reads done before `release` runs: the columns' region may be
// reused as soon as they are in registers, before the math and the stores.
template <int EPI, class Release>
__device__ __forceinline__ void epilogue_head(bf16* out, float* outf, int ldo, uint32_t tb, int64_t row,
                                              int col0, bool valid, Release release) {
  constexpr bool kPaired = EPI == EPI_SWIGLU || EPI == EPI_PAIRSUM_F32;
  uint32_t a0[32], a1[32], b0[32], b1[32];
  tmem_ld32(tb, a0);
  tmem_ld32(tb + 32, a1);
  if (kPaired) {
    tmem_ld32(tb + 64, b0);
    tmem_ld32(tb + 96, b1);
  }
  tmem_ld_wait();
  release();
  if (valid) {
    epilogue_cols32<EPI>(out, outf, row * ldo + col0, a0, b0);
    epilogue_cols32<EPI>(out, outf, row * ldo + col0 + 32, a1, b1);
  }
  __syncwarp();          // the caller's next tcgen05.ld needs the whole warp converged
}
template <class Release>
__device__ __forceinline__ void epilogue_head_rt(int epi, bf16* out, float* outf, int ldo, uint32_t tb,
                                                 int64_t row, int col0, bool valid, Release release) {
  switch (epi) {
    case EPI_SWIGLU: epilogue_head<EPI_SWIGLU>(out, outf, ldo, tb, row, col0, valid, release); break;
    case EPI_GELU: epilogue_head<EPI_GELU>(out, outf, ldo, tb, row, col0, valid, release); break;
    case EPI_PAIRSUM_F32: epilogue_head<EPI_PAIRSUM_F32>(out, outf, ldo, tb, row, col0, valid, release); break;
    default: epilogue_head<EPI_STORE>(out, outf, ldo, tb, row, col0, valid, release); break;
  }
}

template <class TilesFn>
__device__ void group_tile_prefix(const int* off, int G, int* mt, int* wsum, TilesFn tiles) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int per = (G + (int)blockDim.x - 1) / (int)blockDim.x;
  const int g0 = min(G, (int)threadIdx.x * per), g1 = min(G, g0 + per);
  int run = 0;
  for (int g = g0; g < g1; ++g) run += tiles(off[g + 1] - off[g]);
  int inc = run;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int v = __shfl_up_sync(0xffffffffu, inc, o);
    if (lane >= o) inc += v;
  }
  if (lane == 31) wsum[warp] = inc;
  __syncthreads();
  int before = 0;
  for (int w = 0; w < warp; ++w) before += wsum[w];
  int pre = before + inc - run;
  for (int g = g0; g < g1; ++g) {
    mt[g] = pre;
    pre += tiles(off[g + 1] - off[g]);
  }
  if (threadIdx.x == blockDim.x - 1) mt[G] = before + inc;
  __syncthreads();
}


typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = []() -> EncodeTiledFn {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return nullptr;
    return reinterpret_cast<EncodeTiledFn>(ptr);
  }();
  return fn;
}

}  // namespace
}  // namespace moe

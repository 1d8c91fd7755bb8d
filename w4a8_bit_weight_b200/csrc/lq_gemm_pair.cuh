// lq_gemm_pair.cuh -- W4A8 GEMM on CTA pairs (tcgen05 cta_group::2) for
// large token counts.
//
// A cluster of two CTAs on two SMs computes one tile of 256 weight rows x 256
// tokens with tcgen05.mma.cta_group::2 (M = 256, N = 256, K = 32 per
// instruction):
//   * each CTA expands ITS 128 weight rows into ITS tensor memory (the MMA's
//     A operand, one TMEM lane per row, as in the one-CTA kernels);
//   * each CTA loads HALF of the tokens (128) into its shared memory (the
//     MMA's B operand is split by N across the pair), so every activation
//     byte fetched serves 256 weight rows;
//   * each CTA's TMEM holds the int32 accumulators of its 128 weight rows for
//     all 256 tokens;
//   * one thread of the even CTA issues every MMA for both SMs: 128 cycles of
//     tensor work per SM per instruction, enough to hide the issue cost.
// Stages carry 256 K (four groups of 64) and come in two rings: weight
// stages (packed codes, scales, offsets) are released as soon as the
// expansion warps have read them, activation stages when the MMAs that read
// them complete -- so refilling weights never waits for the tensor core and
// expansion stays off the activation refill path.  The accumulator is single:
// the epilogue warps of both CTAs hand it back as soon as it sits in their
// registers as packed bf16, before any global store.
//
// When the tiles leave the last round at most half full, that round's tiles
// are cut into halves of 128 tokens (N = 128 MMAs), one half per pair.
//
// Activation stage i and TMEM weight slot i are filled and drained together,
// so one barrier pair covers both.  Hand-offs between the two CTAs:
//   activations landed   -> both CTAs' activation copies complete their bytes on
//                           the even CTA's full[stage] (the pair form of TMA)
//   expansion done       -> arrive on the even CTA's full[stage] (remote for odd)
//   stage consumed       -> tcgen05.commit multicast to empty[stage] of both CTAs
//   tile finished        -> tcgen05.commit multicast to accfull of both CTAs
//   accumulator loaded   -> arrive on the even CTA's accempty (remote for odd)
// No TMA load uses cluster multicast: each CTA loads its own data.
//
// Warp roles (608 threads):
//   warp 0        TMA producer of weight stages
//   warp 1        TMEM allocation (both CTAs); MMA issue (even CTA)
//   warps 2-9     expansion: two groups of four warps, alternate K-blocks
//   warps 10-17   epilogue: two warps per TMEM lane quarter, 128 tokens each
//   warp 18       TMA producer of activation stages
#pragma once

#include <cuda_bf16.h>

#include "lq_device.cuh"
#include "lq_gemm_kernel.cuh"

namespace lq {

constexpr int kQBT = 256;                     // tokens per tile (MMA N)
constexpr int kQBN = 256;                     // weight rows per tile (MMA M, 128 per CTA)
constexpr int kQBK = 256;                     // K per stage
constexpr int kQXStages = 4;                  // activation ring
constexpr int kQWStages = 5;                  // weight ring
constexpr int kQSlots = kQXStages;            // TMEM A slots, paired with activation stages
constexpr int kQExpGroups = 2;
constexpr int kQEpiWarp0 = 2 + 4 * kQExpGroups;
constexpr int kQXProdWarp = kQEpiWarp0 + 8;
constexpr int kQThreads = 32 * (kQXProdWarp + 1);
constexpr int kQXSub = 128 * 128;             // one 128-token x 128-K SW128 sub-tile
constexpr int kQXBytes = 2 * kQXSub;          // 32 KB: this CTA's 128 tokens x 256 K
constexpr int kQWBytes = 128 * kQBK / 2;      // 16 KB: 128 rows x 256 codes, 128-byte rows (SW128)
constexpr int kQSABytes = (kQBK / 64) * 128;  // 4 groups x 128 rows
constexpr int kQWStage = kQWBytes + 2 * kQSABytes;  // 17 KB, keeps the 1024-byte alignment
constexpr uint32_t kQTxX = 2 * kQXBytes;      // both CTAs' activations land on the even CTA's barrier
constexpr uint32_t kQTxW = kQWStage;
constexpr int kQAccCols = kQBT;               // one accumulator
constexpr int kQSlotCols = kQBK / 4;          // 64 TMEM columns per expanded stage
constexpr int kQXRing = kQXStages * kQXBytes;
constexpr int kQWRing = kQWStages * kQWStage;
constexpr int kQBarBytes = 512;
constexpr int kQSmemBytes = kQXRing + kQWRing + kQBarBytes + 1024;
static_assert(kQWStage % 1024 == 0, "weight stage alignment");
static_assert(kQAccCols + kQSlots * kQSlotCols <= 512, "TMEM budget");
static_assert(kQSmemBytes <= 232448, "shared memory budget");
static_assert(kQSlots % kQExpGroups == 0, "slots per expansion group");

__device__ __forceinline__ void tmem_alloc_pair(uint32_t* dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(dst_smem)),
               "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish_pair() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc_pair(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
// D[256 x N] (+)= A[256 x 32] * B[N x 32]^T over the CTA pair (int8 -> int32).
__device__ __forceinline__ void mma_i8_ts_pair(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                               uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::i8 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// Arrives on the mbarrier at this shared-memory offset in every CTA of
// `cta_mask` once all prior tcgen05 operations of the pair have completed.
__device__ __forceinline__ void tc_commit_pair_mc(uint64_t* bar, uint16_t cta_mask) {
  asm volatile(
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;" ::"r"(
          smem_u32(bar)),
      "h"(cta_mask)
      : "memory");
}
__device__ __forceinline__ uint32_t idesc_i8_pair(int n) {
  return (2u << 4) | (1u << 7) | (1u << 10) | (uint32_t(n >> 3) << 17) | (uint32_t(kQBN >> 4) << 24);
}

// A pair's share of the tiles: whole tiles cid, cid + ncl, ...  When the last
// round would leave at least half of the pairs idle, its tiles are cut into
// token halves instead (an N = 128 pair MMA costs half an N = 256 one), one
// half per pair, so that round takes half as long.
struct PairWork {
  int nwhole, nunits, tail_tile, tail_half;
  __device__ __forceinline__ PairWork(int cid, int ncl, int tiles, bool may_split) {
    const int rounds = tiles / ncl, rem = tiles - rounds * ncl;
    const bool split = may_split && rem > 0 && 2 * rem <= ncl;
    nwhole = split ? rounds : (cid < tiles ? (tiles - 1 - cid) / ncl + 1 : 0);
    nunits = nwhole + ((split && cid < 2 * rem) ? 1 : 0);
    tail_tile = rounds * ncl + (cid >> 1);
    tail_half = cid & 1;
  }
  __device__ __forceinline__ int tile(int k, int cid, int ncl) const { return k < nwhole ? cid + k * ncl : tail_tile; }
  // -1: the whole tile; 0 / 1: that half of its 256 tokens
  __device__ __forceinline__ int half(int k) const { return k < nwhole ? -1 : tail_half; }
};

// Arrive on the even CTA's copy of `bar` (local arrive on the even CTA).
__device__ __forceinline__ void arrive_on_leader(uint64_t* bar, uint32_t crank) {
  if (crank == 0)
    mbar_arrive(bar);
  else
    mbar_arrive_remote(mapa_shared(smem_u32(bar), 0));
}

// Tensor load into this CTA's shared memory whose completed bytes are counted
// on an mbarrier of either CTA of the pair (`bar_cluster` is a shared::cluster
// address, e.g. from mapa).  Plain (non-multicast) copy.
__device__ __forceinline__ void tma_load_2d_pair(void* dst, const CUtensorMap* map, uint32_t bar_cluster, int c0,
                                                 int c1, uint64_t cache_hint) {
  asm volatile(
      "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
      " [%0], [%1, {%3, %4}], [%2], %5;" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(bar_cluster), "r"(c0), "r"(c1), "l"(cache_hint)
      : "memory");
}

// One elected lane waits; the decision is shared with the warp.
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, volatile int* abort_flag, bool cluster) {
  bool ok = true;
  if ((threadIdx.x & 31) == 0) ok = cluster ? mbar_wait_cluster(bar, parity, abort_flag) : mbar_wait(bar, parity, abort_flag);
  return __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
}

template <bool OUT_I32, bool SWI = false>
__global__ void __launch_bounds__(kQThreads, 1)
    w4a8_gemm_pair_kernel(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_w,
                          const __grid_constant__ CUtensorMap tm_s, const __grid_constant__ CUtensorMap tm_a,
                          const GemmArgs p) {
  constexpr int SX = kQXStages, SW = kQWStages;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* xring = smem;                 // SX x [2][128 tokens][128 B], SW128
  uint8_t* wring = smem + kQXRing;       // SW x ([128 rows][128 B] SW128 | s [4][128] | a [4][128])
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + kQXRing + kQWRing);  // [SX], used on the even CTA
  uint64_t* empty = full + SX;           // [SX]
  uint64_t* wfull = empty + SX;
  uint64_t* wempty = wfull + SW;
  uint64_t* accfull = wempty + SW;
  uint64_t* accempty = accfull + 1;
  uint64_t* drain = accempty + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const bool leader = (lane == 0);
  const uint32_t crank = cluster_ctarank();
  const bool even = (crank == 0);

  if (threadIdx.x == 0) {
    for (int s = 0; s < SX; ++s) {
      mbar_init(&full[s], 1 + 8);  // even producer's expect-tx + four expansion warps of each CTA
      mbar_init(&empty[s], 1);
    }
    for (int s = 0; s < SW; ++s) {
      mbar_init(&wfull[s], 1);
      mbar_init(&wempty[s], 4);  // the four warps of the expansion group that read it
    }
    mbar_init(accfull, 1);
    mbar_init(accempty, 16);     // eight epilogue warps of each CTA
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
    tma_prefetch_desc(&tm_x);
    tma_prefetch_desc(&tm_w);
    tma_prefetch_desc(&tm_s);
    tma_prefetch_desc(&tm_a);
  }
  if (warp == 1) {
    tmem_alloc_pair(tmem_slot, 512);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  // both CTAs' barriers exist before any remote arrive or multicast commit
  cluster_arrive();
  cluster_wait();

  const int KS = p.K / kQBK;                 // stages per tile
  const int tiles_m = p.tiles_m;
  const int tiles = (int)(p.U);             // host passes the tile count in U
  const int cid = blockIdx.x >> 1;
  const int ncl = gridDim.x >> 1;
  // Grouped GEMM (m_off set): the tiles are the token tiles of all groups (a
  // bound) times the weight tiles of one group; every role finds a tile's
  // group from the offsets (read after the grid dependency wait) and skips
  // tiles past the last group's rows, so all roles step through the same
  // tiles.  The last round is not split in token halves then.
  const bool grouped = (p.m_off != nullptr);
  const PairWork pw(cid, ncl, tiles, !grouped);
  // first token row, end row, first (stacked) weight row and scale offset of a
  // tile; false: no rows (grouped only).  Called by whole warps.
  auto geo = [&](int tile, int& xrow0, int& mend, int& wrow0, int& scoff) -> bool {
    const int tm = tile % tiles_m, tn = tile / tiles_m;
    if (!grouped) {
      xrow0 = tm * kQBT;
      mend = p.M;
      wrow0 = tn * kQBN;
      scoff = 0;
      return true;
    }
    const int ge = find_group_tile(p.m_off, p.groups, p.M, kQBT, tm, xrow0, mend);
    if (ge < 0) return false;
    wrow0 = ge * p.N + tn * kQBN;
    scoff = ge * p.N;
    return true;
  };
  int nvalid = pw.nunits;
  if (grouped && warp >= 2 && warp < kQEpiWarp0) {
    griddep_wait();
    nvalid = 0;
    for (int k = 0; k < pw.nunits; ++k) {
      int a0, a1, a2, a3;
      if (geo(pw.tile(k, cid, ncl), a0, a1, a2, a3)) ++nvalid;
    }
  }
  const int total = nvalid * KS;            // K-blocks this CTA takes part in

  if (warp == 0) {
    // ---------------------------------------------------- weight producer
    // weights depend on nothing the preceding kernel writes: no dependency wait
    uint64_t pol = 0;
    if (leader) pol = l2_policy_evict_first();
    if (grouped) griddep_wait();  // which weights: from the offsets
    uint32_t issued = 0, issued_par = 0;
    int it = 0;
    for (int k = 0; k < pw.nunits; ++k) {
      const int tile = pw.tile(k, cid, ncl);
      int xr0, me, wr0, so;
      if (!geo(tile, xr0, me, wr0, so)) continue;
      const int wrow = wr0 + (int)crank * 128;
      for (int kb = 0; kb < KS; ++kb, ++it) {
        const int w = it % SW;
        const uint32_t use = (uint32_t)(it / SW);
        if (it >= SW && !warp_wait(&wempty[w], (use & 1u) ^ 1u, abort_flag, false)) goto wprod_done;
        if (leader) {
          uint8_t* wb = wring + w * kQWStage;
          mbar_arrive_expect_tx(&wfull[w], kQTxW);
          tma_load_2d(wb, &tm_w, &wfull[w], kb * (kQBK / 2), wrow, pol);
          tma_load_2d(wb + kQWBytes, &tm_s, &wfull[w], wrow, kb * 4, pol);
          tma_load_2d(wb + kQWBytes + kQSABytes, &tm_a, &wfull[w], wrow, kb * 4, pol);
        }
        issued |= 1u << w;
        issued_par = (issued_par & ~(1u << w)) | ((use & 1u) << w);
      }
    }
  wprod_done:
    if (leader && *abort_flag)
      for (int s = 0; s < SW; ++s)
        if (issued & (1u << s)) {
          const unsigned long long t0w = globaltimer();
          while (!mbar_try_wait(smem_u32(&wfull[s]), (issued_par >> s) & 1u) && globaltimer() - t0w < 100000000ull) {
          }
        }
  } else if (warp == kQXProdWarp) {
    // ------------------------------------------------ activation producer
    uint64_t pol = 0;
    if (leader) pol = l2_policy_evict_last();
    griddep_wait();  // activations may be the output of the preceding kernel
    const uint32_t full_even = mapa_shared(smem_u32(full), 0);
    bool issued = false;
    int it = 0;
    for (int k = 0; k < pw.nunits; ++k) {
      const int tile = pw.tile(k, cid, ncl), half = pw.half(k);
      int xr0, me, wr0, so;
      if (!geo(tile, xr0, me, wr0, so)) continue;
      // B is split by N across the pair: 128 tokens per CTA, 64 for a half tile
      // (the 128-row box then carries 64 rows the MMA does not read)
      const int xrow = xr0 + (half < 0 ? (int)crank * 128 : half * 128 + (int)crank * 64);
      for (int kb = 0; kb < KS; ++kb, ++it) {
        const int x = it % SX;
        const uint32_t use = (uint32_t)(it / SX);
        if (it >= SX && !warp_wait(&empty[x], (use & 1u) ^ 1u, abort_flag, false)) goto xprod_done;
        if (leader) {
          uint8_t* xb = xring + x * kQXBytes;
          const uint32_t bar = full_even + (uint32_t)(x * 8);
          if (even) mbar_arrive_expect_tx(&full[x], kQTxX);
          tma_load_2d_pair(xb, &tm_x, bar, kb * kQBK, xrow, pol);
          tma_load_2d_pair(xb + kQXSub, &tm_x, bar, kb * kQBK + 128, xrow, pol);
        }
        issued = true;
      }
    }
  xprod_done:
    // The copies complete on the even CTA's barrier, whose phase also needs the
    // expansion warps: after an abort, give any copy in flight a fixed 200 us
    // to land before this CTA's shared memory is released.
    if (leader && issued && *abort_flag) {
      const unsigned long long t0w = globaltimer();
      while (globaltimer() - t0w < 200000ull) {
      }
    }
  } else if (warp == 1) {
    if (even) {
      // ------------------------------------------------- MMA issuer (even CTA)
      bool any = false;
      int it = 0, j = 0;
      if (grouped) griddep_wait();
      for (int k = 0; k < pw.nunits; ++k) {
        if (grouped) {
          int a0, a1, a2, a3;
          if (!geo(pw.tile(k, cid, ncl), a0, a1, a2, a3)) continue;
        }
        const uint32_t idesc = idesc_i8_pair(pw.half(k) < 0 ? kQBT : kQBT / 2);
        // the single accumulator is free once both CTAs' epilogues have loaded it
        if (!warp_wait(accempty, ((uint32_t)j & 1u) ^ 1u, abort_flag, true)) goto mma_done;
        tc_fence_after();
        for (int kb = 0; kb < KS; ++kb, ++it) {
          const int x = it % SX;
          if (!warp_wait(&full[x], (uint32_t)(it / SX) & 1u, abort_flag, true)) goto mma_done;
          if (leader) {
            tc_fence_after();
            const uint32_t xs = smem_u32(xring + x * kQXBytes);
            const uint32_t a_col = tmem_base + kQAccCols + x * kQSlotCols;
#pragma unroll
            for (int jj = 0; jj < kQBK / 32; ++jj) {
              const uint64_t bdesc = smem_desc_k_sw128(xs + (jj >> 2) * kQXSub) + (uint64_t)(2 * (jj & 3));
              mma_i8_ts_pair(tmem_base, a_col + jj * 8, bdesc, idesc, (kb > 0 || jj > 0) ? 1u : 0u);
            }
            tc_commit_pair_mc(&empty[x], 0x3);
          }
          any = true;
        }
        if (leader) tc_commit_pair_mc(accfull, 0x3);
        __syncwarp();
        ++j;
      }
      griddep_launch_dependents();
    mma_done:
      if (leader && any) {
        tc_commit_pair_mc(drain, 0x1);
        const uint32_t a = smem_u32(drain);
        const unsigned long long t0w = globaltimer();
        while (!mbar_try_wait(a, 0) && globaltimer() - t0w < 100000000ull) {
        }
      }
    }
  } else if (warp < kQEpiWarp0) {
    // ------------------------------------------------------ expansion warps
    const int sub = warp & 3;
    const int grp = (warp - 2) >> 2;
    const int r = sub * 32 + lane;
    const uint32_t t_lane = tmem_base + ((uint32_t)(sub * 32) << 16);
    const int sw = r & 7;                // 128-byte swizzle of this row's 16-byte chunks
    for (int it = grp; it < total; it += kQExpGroups) {
      const int w = it % SW, slot = it % SX;
      if (!__all_sync(0xffffffffu, mbar_wait(&wfull[w], (uint32_t)(it / SW) & 1u, abort_flag) &&
                                       mbar_wait(&empty[slot], ((uint32_t)(it / SX) & 1u) ^ 1u, abort_flag)))
        goto exp_done;
      tc_fence_after();
      const uint8_t* wb = wring + w * kQWStage;
      const uint8_t* ss = wb + kQWBytes;
      const uint32_t wrow = smem_u32(wb) + r * (kQBK / 2);
      uint32_t v0[32], v1[32];
#pragma unroll
      for (int h = 0; h < 2; ++h) {        // 128 K per half: groups 2h, 2h+1
        const uint32_t s0 = ss[(2 * h) * 128 + r], s1 = ss[(2 * h + 1) * 128 + r];
        const uint32_t a0 = (uint32_t)ss[kQSABytes + (2 * h) * 128 + r] * 0x01010101u;
        const uint32_t a1 = (uint32_t)ss[kQSABytes + (2 * h + 1) * 128 + r] * 0x01010101u;
        uint32_t* v = h ? v1 : v0;
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          const uint4 q = lds128(wrow + (((4 * h + c) ^ sw) << 4));
          const uint32_t s = c < 2 ? s0 : s1;
          const uint32_t a4 = c < 2 ? a0 : a1;
          lqq_expand_word(q.x, s, a4, v[8 * c + 0], v[8 * c + 1]);
          lqq_expand_word(q.y, s, a4, v[8 * c + 2], v[8 * c + 3]);
          lqq_expand_word(q.z, s, a4, v[8 * c + 4], v[8 * c + 5]);
          lqq_expand_word(q.w, s, a4, v[8 * c + 6], v[8 * c + 7]);
        }
      }
      // the weight stage has been read: the producer may refill it
      __syncwarp();
      if (lane == 0) mbar_arrive(&wempty[w]);
      tmem_st_32x32b_x32(t_lane + kQAccCols + slot * kQSlotCols, v0);
      tmem_st_32x32b_x32(t_lane + kQAccCols + slot * kQSlotCols + 32, v1);
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) arrive_on_leader(&full[slot], crank);
    }
  exp_done:;
  } else {
    // ------------------------------------------------------- epilogue warps
    const int sub = warp & 3;
    const int e = (warp - kQEpiWarp0) >> 2;   // tokens [128e, 128e + 128) of the tile
    const int r = sub * 32 + lane;
    const uint32_t t_lane = tmem_base + ((uint32_t)(sub * 32) << 16);
    griddep_wait();
    int j = 0;
    for (int k = 0; k < pw.nunits; ++k) {
      const int tile = pw.tile(k, cid, ncl), half = pw.half(k);
      int xr0, mend, wr0, scoff;
      if (!geo(tile, xr0, mend, wr0, scoff)) continue;
      const int tn = tile / tiles_m;
      const int n = tn * kQBN + (int)crank * 128 + r;  // output column (within the group)
      const bool n_ok = n < p.N;
      // a half tile's 128 tokens are accumulator columns 0-127: the second
      // pair of warps only hands the accumulator back
      const int mb = xr0 + (half < 0 ? e * 128 : half * 128);
      const int jj = j++;
      if (half >= 0 && e == 1) {
        if (!warp_wait(accfull, (uint32_t)jj & 1u, abort_flag, false)) goto epi_done;
        tc_fence_after();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) arrive_on_leader(accempty, crank);
        continue;
      }
      // scales are loaded before the accumulator is ready, off the hand-back path
      const float sc = (!OUT_I32 && n_ok) ? __ldg(p.s_c + scoff + n) : 0.0f;
      float sx4[4];  // s_x of tokens mb + 32c + lane
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const int m = mb + 32 * c + lane;
        sx4[c] = (!OUT_I32 && m < mend) ? ld_dep(p.s_x + m) : 0.0f;
      }
      if (!warp_wait(accfull, (uint32_t)jj & 1u, abort_flag, false)) goto epi_done;
      tc_fence_after();
      if constexpr (OUT_I32) {
#pragma unroll 1
        for (int cc = 0; cc < 4; ++cc) {
          uint32_t v[32];
          tmem_ld_32x32b_x32(t_lane + e * 128 + cc * 32, v);
          tmem_ld_wait();
          if (cc == 3) {
            tc_fence_before();
            __syncwarp();
            if (lane == 0) arrive_on_leader(accempty, crank);
          }
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            const int m = mb + cc * 32 + i;
            if (m < mend && n_ok) reinterpret_cast<int32_t*>(p.out)[(size_t)m * p.N + n] = (int32_t)v[i];
          }
        }
      } else if constexpr (SWI) {
        // SwiGLU of the interleaved gate/up rows (swiglu_pair): this lane's
        // output of each token pair (the even token in even lanes, the odd one
        // in odd lanes) as bf16 in registers first, the accumulator handed back
        // before any global store.
        uint32_t pk[32];  // pk[q / 2]: outputs of token pairs q (low half) and q + 1 (high half)
#pragma unroll
        for (int cc = 0; cc < 8; ++cc) {
          uint32_t v[16];
          tmem_ld_32x32b_x16(t_lane + e * 128 + cc * 16, v);
          const float sxl = sx4[cc >> 1];
          tmem_ld_wait();
#pragma unroll
          for (int i = 0; i < 16; i += 2) {
            const int src = (cc & 1) * 16 + i;
            const float y0 = __fmul_rn(__int2float_rn((int32_t)v[i]), __fmul_rn(__shfl_sync(0xffffffffu, sxl, src), sc));
            const float y1 =
                __fmul_rn(__int2float_rn((int32_t)v[i + 1]), __fmul_rn(__shfl_sync(0xffffffffu, sxl, src + 1), sc));
            const uint32_t b = __bfloat16_as_ushort(__float2bfloat16_rn(swiglu_pair(y0, y1)));
            const int q = 8 * cc + i / 2;  // token pair of the warp's 128
            if (q & 1)
              pk[q >> 1] |= b << 16;
            else
              pk[q >> 1] = b;
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) arrive_on_leader(accempty, crank);
        const bool odd = lane & 1;
        const int ld = p.N >> 1;
        const bool pair_ok = n_ok;  // N is a multiple of 16: a gate row and its up row are both valid or not
        __nv_bfloat16* o = reinterpret_cast<__nv_bfloat16*>(p.out) + (n >> 1);
#pragma unroll
        for (int q = 0; q < 64; ++q) {
          const int m = mb + 2 * q + (odd ? 1 : 0);
          const uint32_t h = (q & 1) ? (pk[q >> 1] >> 16) : (pk[q >> 1] & 0xFFFFu);
          if (m < mend && pair_ok) o[(size_t)m * ld] = __ushort_as_bfloat16((unsigned short)h);
        }
      } else {
        // All four chunks to packed bf16 in registers first, so the accumulator
        // goes back to the MMA warp before any global store is issued.
        uint32_t pk[64];  // pk[q] = bf16 pair for tokens (2q, 2q+1) of this warp's 128
#pragma unroll
        for (int cc = 0; cc < 8; ++cc) {
          uint32_t v[16];
          tmem_ld_32x32b_x16(t_lane + e * 128 + cc * 16, v);
          const float sxl = sx4[cc >> 1];
          tmem_ld_wait();
#pragma unroll
          for (int i = 0; i < 16; i += 2) {
            const int src = (cc & 1) * 16 + i;
            const float s0 = __fmul_rn(__shfl_sync(0xffffffffu, sxl, src), sc);
            const float s1 = __fmul_rn(__shfl_sync(0xffffffffu, sxl, src + 1), sc);
            const float y0 = __fmul_rn(__int2float_rn((int32_t)v[i]), s0);
            const float y1 = __fmul_rn(__int2float_rn((int32_t)v[i + 1]), s1);
            const __nv_bfloat162 h = __floats2bfloat162_rn(y0, y1);
            pk[8 * cc + i / 2] = *reinterpret_cast<const uint32_t*>(&h);
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) arrive_on_leader(accempty, crank);
        // Stores: lanes 2j and 2j+1 swap halves so that each lane writes the two
        // adjacent columns (n, n+1) of one token as one 4-byte word -- even
        // lanes the even token of a pair, odd lanes the odd token.
        const bool odd = lane & 1;
        const int n0 = n & ~1;
        const bool n0_ok = n0 < p.N;  // N is a multiple of 16, so n0 + 1 < N too
#pragma unroll
        for (int q = 0; q < 64; ++q) {
          const uint32_t mine = pk[q];
          const uint32_t other = __shfl_xor_sync(0xffffffffu, mine, 1);
          // even lane: (its token i at n, partner's token i at n+1); odd lane: token i+1
          const uint32_t lo = odd ? (other >> 16) : (mine & 0xFFFFu);
          const uint32_t hi = odd ? (mine >> 16) : (other & 0xFFFFu);
          const int m = mb + 2 * q + (odd ? 1 : 0);
          if (m < mend && n0_ok)
            *reinterpret_cast<uint32_t*>(reinterpret_cast<__nv_bfloat16*>(p.out) + (size_t)m * p.N + n0) =
                lo | (hi << 16);
        }
      }
    }
  epi_done:;
  }

  // ---------------------------------------------------------------- teardown
  // The even CTA's MMAs read the odd CTA's shared and tensor memory: neither
  // CTA leaves before the pair is done.
  __syncwarp();
  tc_fence_before();
  cluster_arrive();
  cluster_wait();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, 512);
  }
}

}  // namespace lq

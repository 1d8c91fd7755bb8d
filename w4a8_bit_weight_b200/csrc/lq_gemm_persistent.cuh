// lq_gemm_persistent.cuh -- persistent W4A8 GEMM for many tiles (prefill).
//
// Same operand placement and stage format as lq_gemm_kernel.cuh (weights
// expanded into TMEM as the MMA's A operand, 128 weight rows x 128 tokens
// per tile, K-blocks of 128), organized for throughput when there are at
// least as many tiles as SMs:
//   * one CTA per SM loops over tiles blockIdx.x, blockIdx.x + gridDim.x, ...
//     (token tiles fastest, so the CTAs in flight share weight tiles in L2);
//   * two TMEM accumulators (2 x 128 columns) alternate between tiles, so the
//     epilogue of tile j overlaps the mainloop of tile j+1;
//   * kPExpGroups groups of four expansion warps; group g expands the stages
//     of K-blocks g, g + kPExpGroups, ...  Expanding one stage (load, IMAD +
//     XOR, tcgen05.st, wait for the store) takes longer than the 256 cycles
//     of tensor work per stage, so several stages are expanded at once.
//
// Warp roles (64 + 128 * kPExpGroups + 128 threads):
//   warp 0        TMA producer (one elected lane issues)
//   warp 1        TMEM allocation, tcgen05.mma issue (one elected lane)
//   warps 2..     LiquidQuant expansion into the TMEM A slot of the stage
//   last 4 warps  epilogue: TMEM accumulators -> scales -> bf16 stores
#pragma once

#include <cuda_bf16.h>

#include "lq_device.cuh"
#include "lq_gemm_kernel.cuh"

namespace lq {

constexpr int kPBT = 128;                 // tokens per tile
constexpr int kPStages = 8;
constexpr int kPExpGroups = 4;
constexpr int kPEpiWarp0 = 2 + 4 * kPExpGroups;
constexpr int kPThreads = 32 * (kPEpiWarp0 + 4);
static_assert(kPStages % kPExpGroups == 0, "stages per expansion group");
constexpr int kPXBytes = kPBT * kBlockK;  // 16 KB
constexpr int kPWBytes = kBlockN * kBlockK / 2;
constexpr int kPSABytes = 2 * kBlockN;
constexpr int kPStageBytes = round_up_c(kPXBytes + kPWBytes + 2 * kPSABytes, 1024);
constexpr uint32_t kPTxBytes = kPXBytes + kPWBytes + 2 * kPSABytes;
constexpr int kPAccCols = 2 * kPBT;       // two accumulators
constexpr int kPBarBytes = 512;
constexpr int kPSmemBytes = kPStages * kPStageBytes + kPBarBytes + 1024;
static_assert(kPAccCols + kPStages * 32 <= 512, "TMEM budget");
static_assert(kPSmemBytes <= 232448, "shared memory budget");

template <bool OUT_I32>
__global__ void __launch_bounds__(kPThreads, 1)
    w4a8_gemm_persistent_kernel(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_w,
                                const __grid_constant__ CUtensorMap tm_s, const __grid_constant__ CUtensorMap tm_a,
                                const GemmArgs p) {
  constexpr int S = kPStages;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + S * kPStageBytes);
  uint64_t* afull = full + S;
  uint64_t* empty = afull + S;
  uint64_t* accfull = empty + S;   // [2]
  uint64_t* accempty = accfull + 2;  // [2]
  uint64_t* drain = accempty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const bool leader = (lane == 0);

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&afull[s], 4);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&accfull[b], 1);
      mbar_init(&accempty[b], 4);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
    tma_prefetch_desc(&tm_x);
    tma_prefetch_desc(&tm_w);
    tma_prefetch_desc(&tm_s);
    tma_prefetch_desc(&tm_a);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  const int KB = p.KB;
  const int tiles = (int)(p.U / KB);
  const int first_tile = blockIdx.x;
  const int stride = gridDim.x;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    uint64_t pol_stream = 0, pol_keep = 0;
    if (leader) {
      pol_stream = l2_policy_evict_first();
      pol_keep = l2_policy_evict_last();
    }
    const int P = first_tile < tiles ? min(S, KB) : 0;
    {
      const int tn0 = first_tile / p.tiles_m, tm0 = first_tile % p.tiles_m;
      if (leader) {
        for (int i = 0; i < P; ++i) {
          uint8_t* sb = smem + i * kPStageBytes;
          mbar_arrive_expect_tx(&full[i], kPTxBytes);
          tma_load_2d(sb + kPXBytes, &tm_w, &full[i], i * (kBlockK / 2), tn0 * kBlockN, pol_stream);
          tma_load_2d(sb + kPXBytes + kPWBytes, &tm_s, &full[i], tn0 * kBlockN, i * 2, pol_stream);
          tma_load_2d(sb + kPXBytes + kPWBytes + kPSABytes, &tm_a, &full[i], tn0 * kBlockN, i * 2, pol_stream);
        }
      }
      griddep_wait();
      if (leader)
        for (int i = 0; i < P; ++i)
          tma_load_2d(smem + i * kPStageBytes, &tm_x, &full[i], i * kBlockK, tm0 * kPBT, pol_keep);
      __syncwarp();
    }
    int stage = 0;
    uint32_t phase = 0;
    uint32_t issued = P >= 32 ? 0xffffffffu : ((1u << P) - 1u), issued_par = 0;
    int it = 0;
    for (int tile = first_tile; tile < tiles; tile += stride) {
      const int tile_m = tile % p.tiles_m, tile_n = tile / p.tiles_m;
      for (int kb = 0; kb < KB; ++kb, ++it) {
        if (it >= P) {
          if (!__all_sync(0xffffffffu, mbar_wait(&empty[stage], phase ^ 1u, abort_flag))) goto producer_done;
          if (leader) {
            uint8_t* sb = smem + stage * kPStageBytes;
            mbar_arrive_expect_tx(&full[stage], kPTxBytes);
            tma_load_2d(sb, &tm_x, &full[stage], kb * kBlockK, tile_m * kPBT, pol_keep);
            tma_load_2d(sb + kPXBytes, &tm_w, &full[stage], kb * (kBlockK / 2), tile_n * kBlockN, pol_stream);
            tma_load_2d(sb + kPXBytes + kPWBytes, &tm_s, &full[stage], tile_n * kBlockN, kb * 2, pol_stream);
            tma_load_2d(sb + kPXBytes + kPWBytes + kPSABytes, &tm_a, &full[stage], tile_n * kBlockN, kb * 2,
                        pol_stream);
          }
          issued |= 1u << stage;
          issued_par = (issued_par & ~(1u << stage)) | (phase << stage);
        }
        if (++stage == S) {
          stage = 0;
          phase ^= 1u;
        }
      }
    }
  producer_done:
    if (leader && *abort_flag) {
      for (int s = 0; s < S; ++s)
        if (issued & (1u << s)) {
          const uint32_t a = smem_u32(&full[s]);
          const unsigned long long t0w = globaltimer();
          while (!mbar_try_wait(a, (issued_par >> s) & 1u) && globaltimer() - t0w < 100000000ull) {
          }
        }
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------- MMA issuer
    constexpr uint32_t idesc = idesc_i8(kPBT);
    int stage = 0;
    uint32_t phase = 0;
    bool any = false;
    int j = 0;
    for (int tile = first_tile; tile < tiles; tile += stride, ++j) {
      const int b = j & 1;
      const uint32_t use_par = (uint32_t)(j >> 1) & 1u;
      if (!__all_sync(0xffffffffu, mbar_wait(&accempty[b], use_par ^ 1u, abort_flag))) goto mma_done;
      tc_fence_after();
      const uint32_t d_tmem = tmem_base + b * kPBT;
      for (int kb = 0; kb < KB; ++kb) {
        if (!__all_sync(0xffffffffu, mbar_wait(&afull[stage], phase, abort_flag))) goto mma_done;
        tc_fence_after();
        if (leader) {
          const uint64_t bdesc = smem_desc_k_sw128(smem_u32(smem + stage * kPStageBytes));
          const uint32_t a_col = tmem_base + kPAccCols + stage * 32;
#pragma unroll
          for (int jj = 0; jj < kBlockK / 32; ++jj)
            mma_i8_ts(d_tmem, a_col + jj * 8, bdesc + (uint64_t)(2 * jj), idesc, (kb > 0 || jj > 0) ? 1u : 0u);
          tc_commit(&empty[stage]);
        }
        __syncwarp();
        any = true;
        if (++stage == S) {
          stage = 0;
          phase ^= 1u;
        }
      }
      if (leader) tc_commit(&accfull[b]);
      __syncwarp();
    }
    griddep_launch_dependents();
  mma_done:
    if (leader && any) {
      tc_commit(drain);
      const uint32_t a = smem_u32(drain);
      const unsigned long long t0w = globaltimer();
      while (!mbar_try_wait(a, 0) && globaltimer() - t0w < 100000000ull) {
      }
    }
  } else if (warp < kPEpiWarp0) {
    // ------------------------------------------------------ expansion warps
    const int sub = warp & 3;
    const int grp = (warp - 2) >> 2;     // this group expands K-blocks grp, grp + G, ...
    const int r = sub * 32 + lane;       // weight row = TMEM lane
    const uint32_t t_lane = tmem_base + ((uint32_t)(sub * 32) << 16);
    const int sw = (r >> 1) & 3;
    int ntiles = 0;
    for (int tile = first_tile; tile < tiles; tile += stride) ++ntiles;
    const int total = ntiles * KB;
    for (int it = grp; it < total; it += kPExpGroups) {
      const int stage = it % S;
      const uint32_t phase = (uint32_t)(it / S) & 1u;
      if (!__all_sync(0xffffffffu, mbar_wait(&full[stage], phase, abort_flag))) goto exp_done;
      tc_fence_after();
      const uint8_t* sb = smem + stage * kPStageBytes;
      const uint8_t* ss = sb + kPXBytes + kPWBytes;
      const uint32_t s0 = ss[r], s1 = ss[kBlockN + r];
      const uint32_t a0 = (uint32_t)ss[kPSABytes + r] * 0x01010101u;
      const uint32_t a1 = (uint32_t)ss[kPSABytes + kBlockN + r] * 0x01010101u;
      const uint32_t wrow = smem_u32(sb + kPXBytes) + r * (kBlockK / 2);
      uint32_t v[32];
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const uint4 q = lds128(wrow + ((c ^ sw) << 4));
        const uint32_t s = c < 2 ? s0 : s1;
        const uint32_t a4 = c < 2 ? a0 : a1;
        lqq_expand_word(q.x, s, a4, v[8 * c + 0], v[8 * c + 1]);
        lqq_expand_word(q.y, s, a4, v[8 * c + 2], v[8 * c + 3]);
        lqq_expand_word(q.z, s, a4, v[8 * c + 4], v[8 * c + 5]);
        lqq_expand_word(q.w, s, a4, v[8 * c + 6], v[8 * c + 7]);
      }
      tmem_st_32x32b_x32(t_lane + kPAccCols + stage * 32, v);
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&afull[stage]);
    }
  exp_done:;
  } else {
    // ------------------------------------------------------- epilogue warps
    const int sub = warp & 3;
    const int r = sub * 32 + lane;
    const uint32_t t_lane = tmem_base + ((uint32_t)(sub * 32) << 16);
    griddep_wait();  // scales and the output may belong to the preceding kernel
    int j = 0;
    for (int tile = first_tile; tile < tiles; tile += stride, ++j) {
      const int b = j & 1;
      const uint32_t use_par = (uint32_t)(j >> 1) & 1u;
      if (!__all_sync(0xffffffffu, mbar_wait(&accfull[b], use_par, abort_flag))) goto epi_done;
      tc_fence_after();
      const int tile_m = tile % p.tiles_m, tile_n = tile / p.tiles_m;
      const int n = tile_n * kBlockN + r;
      const int m0 = tile_m * kPBT;
      const bool n_ok = n < p.N;
      const float sc = (!OUT_I32 && n_ok) ? __ldg(p.s_c + n) : 0.0f;
#pragma unroll 1
      for (int cc = 0; cc < kPBT / 32; ++cc) {
        uint32_t v[32];
        tmem_ld_32x32b_x32(t_lane + b * kPBT + cc * 32, v);
        tmem_ld_wait();
        if (cc == kPBT / 32 - 1) {
          // the whole accumulator is in registers: hand it back to the MMA warp
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&accempty[b]);
        }
        const int mb = m0 + cc * 32;
        float sxl = 0.0f;
        if (!OUT_I32 && mb + lane < p.M) sxl = ld_dep(p.s_x + mb + lane);
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          const int m = mb + i;
          if constexpr (OUT_I32) {
            if (m < p.M && n_ok) reinterpret_cast<int32_t*>(p.out)[(size_t)m * p.N + n] = (int32_t)v[i];
          } else {
            const float sx = __shfl_sync(0xffffffffu, sxl, i);
            if (m < p.M && n_ok) {
              const float y = __fmul_rn(__int2float_rn((int32_t)v[i]), __fmul_rn(sx, sc));
              reinterpret_cast<__nv_bfloat16*>(p.out)[(size_t)m * p.N + n] = __float2bfloat16_rn(y);
            }
          }
        }
      }
    }
  epi_done:;
  }

  // ---------------------------------------------------------------- teardown
  __syncwarp();
  tc_fence_before();
  cta_barrier_unaligned();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem_base, 512);
  }
}

}  // namespace lq

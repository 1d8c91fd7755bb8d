// lq_gemm_kernel.cuh -- the W4A8 GEMM for sm_100a.
//
// Operand placement (swap-AB): the 128 weight rows of a tile are the MMA's M
// side and live in TENSOR MEMORY as the A operand; the tokens are the MMA's N
// side (16..256) and come from shared memory as the B operand.  This is the
// B200 counterpart of the paper's "dequantize in registers and feed the MMA
// directly" (ImFP, review page referee summary): the expanded INT8 weights
// go registers -> TMEM with tcgen05.st and never touch shared memory, so
// shared-memory bandwidth is left to the activation tiles and the packed
// weights.
//
// Warp roles (192 threads, one CTA per SM):
//   warp 0     TMA producer: packed u4 weights, u8 scale/offset tiles and
//              int8 activation tiles into a ring of shared-memory stages.
//   warp 1     allocates TMEM; one thread issues tcgen05.mma kind::i8.
//   warps 2-5  LiquidQuant expansion (one weight row per thread, one IMAD +
//              one XOR per four weights) into the TMEM A slot of the stage,
//              then the epilogue: int32 accumulators -> scales -> bf16.
//
// Schedule (stream-K): the M x N x K work is cut into units of one tile x one
// K-block of 128; CTA c takes units [c*U/G, (c+1)*U/G).  A tile whose units
// all belong to one CTA is written directly; a tile shared by several CTAs is
// summed in an int32 workspace with atomic adds, and the CTA that arrives last
// (atomic ticket) applies the epilogue and restores the workspace and the
// ticket to zero.  Integer sums are order-independent, so the result is
// bit-identical either way.
#pragma once

#include <cuda_bf16.h>

#include "lq_device.cuh"

namespace lq {

constexpr int kBlockN = 128;        // weight rows per tile (MMA M)
constexpr int kBlockK = 128;        // K per pipeline stage (two groups of 64)
constexpr int kGemmThreads = 192;
constexpr int kTmemCols = 512;

__host__ __device__ constexpr int round_up_c(int x, int a) { return (x + a - 1) / a * a; }

template <int BT>
struct GemmCfg {
  static_assert(BT == 16 || BT == 32 || BT == 64 || BT == 128 || BT == 256, "tokens per tile");
  static constexpr int kStages = BT == 256 ? 5 : 8;
  static constexpr int kXBytes = BT * kBlockK;             // int8 activation tile, 128-byte rows
  static constexpr int kWBytes = kBlockN * kBlockK / 2;    // packed u4 weight tile, 64-byte rows
  static constexpr int kSABytes = 2 * kBlockN;             // 2 groups x 128 rows of u8
  static constexpr int kStageBytes = round_up_c(kXBytes + kWBytes + 2 * kSABytes, 1024);
  static constexpr uint32_t kTxBytes = kXBytes + kWBytes + 2 * kSABytes;
  static constexpr int kAccCols = BT < 32 ? 32 : BT;      // int32 accumulator columns
  static constexpr int kBarBytes = 256;
  // at least 120 KB so that two CTAs never share an SM (each holds 512 TMEM columns)
  static constexpr int kSmemBytes =
      round_up_c(kStages * kStageBytes + kBarBytes, 1024) + 1024 > 122880
          ? round_up_c(kStages * kStageBytes + kBarBytes, 1024) + 1024
          : 122880;
  static_assert(kAccCols + kStages * 32 <= kTmemCols, "TMEM budget");
  static_assert(3 * kStages * 8 + 4 * 8 + 16 <= kBarBytes, "barrier area");
};

struct GemmArgs {
  const float* s_x;
  const float* s_c;
  void* out;             // bf16 [M, N] or int32 [M, N]
  int32_t* ws;           // [tiles][BT][128] int32, zero between calls
  unsigned int* ticket;  // [tiles], zero between calls
  int M, N, K;
  int tiles_m, KB;
  long long U;           // units = tiles * KB
};

__device__ __forceinline__ long long cta_of_unit(long long u, long long U, long long G) {
  return ((u + 1) * G + U - 1) / U - 1;
}

// Bounded barrier among the four epilogue warps (an mbarrier with count 4),
// so that a warp that gave up a wait can never strand the others.
__device__ __forceinline__ bool group_sync(uint64_t* bar, uint32_t& phase, volatile int* abort_flag) {
  __syncwarp();
  if ((threadIdx.x & 31) == 0) mbar_arrive(bar);
  const bool ok = __all_sync(0xffffffffu, mbar_wait(bar, phase, abort_flag));
  phase ^= 1u;
  return ok;
}

template <bool OUT_I32>
__device__ __forceinline__ void store_out(const GemmArgs& p, int m, int n, int32_t acc, float sc) {
  if constexpr (OUT_I32) {
    reinterpret_cast<int32_t*>(p.out)[(size_t)m * p.N + n] = acc;
  } else {
    const float scale = __fmul_rn(__ldg(p.s_x + m), sc);
    const float y = __fmul_rn(__int2float_rn(acc), scale);
    reinterpret_cast<__nv_bfloat16*>(p.out)[(size_t)m * p.N + n] = __float2bfloat16_rn(y);
  }
}

template <int BT, bool OUT_I32>
__global__ void __launch_bounds__(kGemmThreads, 1)
    w4a8_gemm_kernel(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_w,
                     const __grid_constant__ CUtensorMap tm_s, const __grid_constant__ CUtensorMap tm_a,
                     const GemmArgs p) {
  using C = GemmCfg<BT>;
  constexpr int S = C::kStages;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + S * C::kStageBytes);
  uint64_t* afull = full + S;
  uint64_t* empty = afull + S;
  uint64_t* accfull = empty + S;
  uint64_t* drain = accfull + 1;
  uint64_t* grp = drain + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(grp + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  volatile int* last_flag = reinterpret_cast<volatile int*>(tmem_slot + 2);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&afull[s], 4);
      mbar_init(&empty[s], 1);
    }
    mbar_init(accfull, 1);
    mbar_init(drain, 1);
    mbar_init(grp, 4);
    *abort_flag = 0;
    *last_flag = 0;
    fence_mbar_init();
    tma_prefetch_desc(&tm_x);
    tma_prefetch_desc(&tm_w);
    tma_prefetch_desc(&tm_s);
    tma_prefetch_desc(&tm_a);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  const long long U = p.U;
  const long long G = gridDim.x;
  const long long u_begin = (long long)blockIdx.x * U / G;
  const long long u_end = ((long long)blockIdx.x + 1) * U / G;
  const int KB = p.KB;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      const uint64_t pol_stream = l2_policy_evict_first();  // weights: read once
      const uint64_t pol_keep = l2_policy_evict_last();     // activations: re-read per weight tile
      int stage = 0;
      uint32_t phase = 0;
      uint32_t issued = 0, issued_par = 0;  // per stage: load in flight, its phase parity
      for (long long u = u_begin; u < u_end;) {
        const int t = (int)(u / KB);
        const int kb0 = (int)(u % KB);
        const int kb1 = (int)min((long long)KB, kb0 + (u_end - u));
        const int tile_m = t % p.tiles_m, tile_n = t / p.tiles_m;
        for (int kb = kb0; kb < kb1; ++kb) {
          if (!mbar_wait(&empty[stage], phase ^ 1u, abort_flag)) goto producer_done;
          uint8_t* sb = smem + stage * C::kStageBytes;
          mbar_arrive_expect_tx(&full[stage], C::kTxBytes);
          tma_load_2d(sb, &tm_x, &full[stage], kb * kBlockK, tile_m * BT, pol_keep);
          tma_load_2d(sb + C::kXBytes, &tm_w, &full[stage], kb * (kBlockK / 2), tile_n * kBlockN, pol_stream);
          tma_load_2d(sb + C::kXBytes + C::kWBytes, &tm_s, &full[stage], tile_n * kBlockN, kb * 2, pol_stream);
          tma_load_2d(sb + C::kXBytes + C::kWBytes + C::kSABytes, &tm_a, &full[stage], tile_n * kBlockN, kb * 2,
                      pol_stream);
          issued |= 1u << stage;
          issued_par = (issued_par & ~(1u << stage)) | (phase << stage);
          if (++stage == S) {
            stage = 0;
            phase ^= 1u;
          }
        }
        u += kb1 - kb0;
      }
    producer_done:
      if (*abort_flag) {
        // never leave a bulk copy in flight into shared memory that is about to be released
        for (int s = 0; s < S; ++s)
          if (issued & (1u << s)) {
            const uint32_t a = smem_u32(&full[s]);
            const unsigned long long t0 = globaltimer();
            while (!mbar_try_wait(a, (issued_par >> s) & 1u) && globaltimer() - t0 < 100000000ull) {
            }
          }
      }
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------- MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_i8(BT);
      int stage = 0;
      uint32_t phase = 0;
      bool any = false;
      for (long long u = u_begin; u < u_end;) {
        const int kb0 = (int)(u % KB);
        const int kb1 = (int)min((long long)KB, kb0 + (u_end - u));
        for (int kb = kb0; kb < kb1; ++kb) {
          if (!mbar_wait(&afull[stage], phase, abort_flag)) goto mma_done;
          tc_fence_after();
          const uint64_t bdesc = smem_desc_k_sw128(smem_u32(smem + stage * C::kStageBytes));
          const uint32_t a_col = tmem_base + C::kAccCols + stage * 32;
#pragma unroll
          for (int j = 0; j < kBlockK / 32; ++j)
            mma_i8_ts(tmem_base, a_col + j * 8, bdesc + (uint64_t)(2 * j), idesc, (kb > kb0 || j > 0) ? 1u : 0u);
          tc_commit(&empty[stage]);
          any = true;
          if (++stage == S) {
            stage = 0;
            phase ^= 1u;
          }
        }
        tc_commit(accfull);
        u += kb1 - kb0;
      }
    mma_done:
      if (any) {
        // all issued MMAs have finished before TMEM is released
        tc_commit(drain);
        const uint32_t a = smem_u32(drain);
        const unsigned long long t0 = globaltimer();
        while (!mbar_try_wait(a, 0) && globaltimer() - t0 < 100000000ull) {
        }
      }
    }
  } else {
    // ------------------------------------------- expansion + epilogue warps
    const int sub = warp & 3;           // TMEM sub-partition this warp may access
    const int r = sub * 32 + lane;      // weight row of the tile = TMEM lane
    const uint32_t t_lane = tmem_base + ((uint32_t)(sub * 32) << 16);
    const int sw = (r >> 1) & 3;        // 64-byte swizzle of this row's 16-byte chunks
    int stage = 0;
    uint32_t phase = 0, acc_phase = 0, grp_phase = 0;
    for (long long u = u_begin; u < u_end;) {
      const int t = (int)(u / KB);
      const int kb0 = (int)(u % KB);
      const int kb1 = (int)min((long long)KB, kb0 + (u_end - u));
      const int tile_m = t % p.tiles_m, tile_n = t / p.tiles_m;
      for (int kb = kb0; kb < kb1; ++kb) {
        // warp-uniform decision: every lane waits, all continue only if all saw the phase
        if (!__all_sync(0xffffffffu, mbar_wait(&full[stage], phase, abort_flag))) goto epi_done;
        tc_fence_after();
        const uint8_t* sb = smem + stage * C::kStageBytes;
        const uint8_t* ss = sb + C::kXBytes + C::kWBytes;
        const uint8_t* sa = ss + C::kSABytes;
        const uint32_t s0 = ss[r], s1 = ss[kBlockN + r];
        const uint32_t a0 = (uint32_t)sa[r] * 0x01010101u, a1 = (uint32_t)sa[kBlockN + r] * 0x01010101u;
        const uint32_t wrow = smem_u32(sb + C::kXBytes) + r * (kBlockK / 2);
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
        tmem_st_32x32b_x32(t_lane + C::kAccCols + stage * 32, v);
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&afull[stage]);
        if (++stage == S) {
          stage = 0;
          phase ^= 1u;
        }
      }

      // ------------------------------------------------------- epilogue
      if (!__all_sync(0xffffffffu, mbar_wait(accfull, acc_phase, abort_flag))) goto epi_done;
      acc_phase ^= 1u;
      tc_fence_after();
      {
        const int n = tile_n * kBlockN + r;
        const int m0 = tile_m * BT;
        const bool n_ok = n < p.N;
        const float sc = (!OUT_I32 && n_ok) ? __ldg(p.s_c + n) : 0.0f;
        const bool whole = (kb0 == 0 && kb1 == KB);
        int32_t* ws_tile = p.ws + (size_t)t * BT * kBlockN;
        constexpr int CH = BT < 32 ? BT : 32;
#pragma unroll 1
        for (int cc = 0; cc < BT / CH; ++cc) {
          uint32_t v[32];
          if constexpr (CH == 16) {
            uint32_t v16[16];
            tmem_ld_32x32b_x16(t_lane + cc * CH, v16);
            tmem_ld_wait();
#pragma unroll
            for (int i = 0; i < 16; ++i) v[i] = v16[i];
          } else {
            tmem_ld_32x32b_x32(t_lane + cc * CH, v);
            tmem_ld_wait();
          }
#pragma unroll
          for (int i = 0; i < CH; ++i) {
            const int ml = cc * CH + i;
            const int m = m0 + ml;
            if (m < p.M) {
              if (whole) {
                if (n_ok) store_out<OUT_I32>(p, m, n, (int32_t)v[i], sc);
              } else {
                atomicAdd(ws_tile + ml * kBlockN + r, (int32_t)v[i]);
              }
            }
          }
        }
        tc_fence_before();
        if (!whole) {
          __threadfence();
          if (!group_sync(grp, grp_phase, abort_flag)) goto epi_done;
          if (warp == 2 && lane == 0) {
            const long long first = cta_of_unit((long long)t * KB, U, G);
            const long long last = cta_of_unit((long long)t * KB + KB - 1, U, G);
            const unsigned contributors = (unsigned)(last - first + 1);
            const unsigned prev = atomicAdd(p.ticket + t, 1u);
            *last_flag = (prev == contributors - 1) ? 1 : 0;
          }
          if (!group_sync(grp, grp_phase, abort_flag)) goto epi_done;
          if (*last_flag) {
            __threadfence();
            for (int ml = 0; ml < BT; ++ml) {
              const int m = m0 + ml;
              if (m >= p.M) break;
              int32_t* cell = ws_tile + ml * kBlockN + r;
              const int32_t acc = __ldcg(cell);
              *cell = 0;
              if (n_ok) store_out<OUT_I32>(p, m, n, acc, sc);
            }
            if (warp == 2 && lane == 0) p.ticket[t] = 0u;
          }
        }
      }
      u += kb1 - kb0;
    }
  epi_done:;
  }

  // ---------------------------------------------------------------- teardown
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem_base, kTmemCols);
  }
}

}  // namespace lq

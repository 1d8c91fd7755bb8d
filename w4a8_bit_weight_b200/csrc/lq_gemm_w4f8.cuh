// lq_gemm_w4f8.cuh -- the W4 x FP8 variant (FireQ page, abstract: INT4
// weights with channel-wise scaling, FP8 activations with one scale for the
// tensor), sm_100a.
//
// Quantization (readings, shared with the oracle's definitions):
//   weights      s_w[n] = amax_n / 7, q = clamp(rint(w * (7 / amax_n)), -7, 7),
//                stored as u = q + 8 in the LiquidQuant nibble layout (word j
//                of a row holds codes 8j..8j+7, byte b = u[8j+b] | u[8j+4+b] << 4);
//   activations  one scale for the tensor, s_x = amax / 448 (448: the largest
//                finite e4m3 value), codes e4m3(x * (448 / amax)) rounded to
//                nearest even and saturated;
//   GEMM         out[m,n] = bf16(acc * (s_x * s_w[n])), acc = sum_k e4m3(x) * q
//                accumulated in fp32 by the tensor core.
//
// The GEMM is deliberately plain: one CTA per 128-row x BT-token tile, a
// ring of stages, warp 0 loads (TMA), warps 2-5 turn each weight row's
// INT4 codes into e4m3 bytes (every integer in [-7, 7] is an e4m3 value, so
// this is exact) and write them as a 128-byte-swizzled A tile in shared
// memory, warp 1 issues tcgen05.mma kind::f8f6f4 with both operands in
// shared memory and fp32 accumulators in tensor memory; warps 2-5 apply the
// scales.  Every wait is bounded, as in the W4A8 kernels.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp8.h>

#include "lq_device.cuh"
#include "lq_quant_kernels.cuh"

namespace lq {

// ----------------------------------------------------------- quantizers
constexpr int kW4Threads = 128;

// one block per weight row
__global__ void __launch_bounds__(kW4Threads) quantize_weights_w4_kernel(const uint16_t* __restrict__ W, int K,
                                                                         uint8_t* __restrict__ qw4,
                                                                         float* __restrict__ s_w) {
  __shared__ float red[32];
  const int n = blockIdx.x;
  const uint16_t* row = W + (size_t)n * K;
  float amax = 0.0f;
  for (int k = threadIdx.x * 8; k < K; k += kW4Threads * 8) {
    const uint4 v = *reinterpret_cast<const uint4*>(row + k);
    const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      amax = fmaxf(amax, fabsf(bf16_bits_to_f32(w4[i] & 0xFFFFu)));
      amax = fmaxf(amax, fabsf(bf16_bits_to_f32(w4[i] >> 16)));
    }
  }
  amax = block_max<kW4Threads>(amax, red);
  const bool zero = (amax == 0.0f);
  const float inv = zero ? 0.0f : __fdiv_rn(7.0f, amax);
  if (threadIdx.x == 0) s_w[n] = zero ? 1.0f : __fdiv_rn(amax, 7.0f);
  uint32_t* out = reinterpret_cast<uint32_t*>(qw4 + (size_t)n * (K / 2));
  for (int k = threadIdx.x * 8; k < K; k += kW4Threads * 8) {
    const uint4 v = *reinterpret_cast<const uint4*>(row + k);
    const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
    uint32_t u[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const uint32_t h = (i & 1) ? (w4[i >> 1] >> 16) : (w4[i >> 1] & 0xFFFFu);
      const int q = zero ? 0 : min(7, max(-7, __float2int_rn(__fmul_rn(bf16_bits_to_f32(h), inv))));
      u[i] = (uint32_t)(q + 8);
    }
    uint32_t word = 0u;
#pragma unroll
    for (int b = 0; b < 4; ++b) word |= (u[b] | (u[b + 4] << 4)) << (8 * b);
    out[k / 8] = word;
  }
}

// Activation quantization, three launches: the tensor's amax (atomic max of
// the non-negative float bits, kept in s_x's word, zeroed by the host), the
// codes, then s_x = amax / 448 written over it.
__global__ void __launch_bounds__(kQuantActThreads) act_f8_amax_kernel(const uint16_t* __restrict__ X, int K,
                                                                       unsigned int* amax_bits) {
  __shared__ float red[32];
  const uint16_t* row = X + (size_t)blockIdx.x * K;
  float amax = 0.0f;
  for (int k = threadIdx.x * 8; k < K; k += kQuantActThreads * 8) {
    const uint4 v = ld_dep(reinterpret_cast<const uint4*>(row + k));
    const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      amax = fmaxf(amax, fabsf(bf16_bits_to_f32(w4[i] & 0xFFFFu)));
      amax = fmaxf(amax, fabsf(bf16_bits_to_f32(w4[i] >> 16)));
    }
  }
  amax = block_max<kQuantActThreads>(amax, red);
  if (threadIdx.x == 0) atomicMax(amax_bits, __float_as_uint(amax));
}

__global__ void __launch_bounds__(kQuantActThreads) act_f8_codes_kernel(const uint16_t* __restrict__ X, int K,
                                                                        const unsigned int* amax_bits,
                                                                        uint8_t* __restrict__ x_f8) {
  const float amax = __uint_as_float(ld_dep(amax_bits));
  const float inv = amax == 0.0f ? 0.0f : __fdiv_rn(448.0f, amax);
  const uint16_t* row = X + (size_t)blockIdx.x * K;
  uint8_t* out = x_f8 + (size_t)blockIdx.x * K;
  for (int k = threadIdx.x * 8; k < K; k += kQuantActThreads * 8) {
    const uint4 v = ld_dep(reinterpret_cast<const uint4*>(row + k));
    const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
    uint32_t o[2] = {0u, 0u};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float2 f = make_float2(__fmul_rn(bf16_bits_to_f32(w4[i] & 0xFFFFu), inv),
                                   __fmul_rn(bf16_bits_to_f32(w4[i] >> 16), inv));
      const uint32_t c2 = (uint32_t)__nv_cvt_float2_to_fp8x2(f, __NV_SATFINITE, __NV_E4M3);
      o[i >> 1] |= (c2 & 0xFFFFu) << (16 * (i & 1));
    }
    *reinterpret_cast<uint2*>(out + k) = make_uint2(o[0], o[1]);
  }
}

__global__ void act_f8_scale_kernel(float* s_x) {
  const float amax = __uint_as_float(*reinterpret_cast<const unsigned int*>(s_x));
  *s_x = amax == 0.0f ? 1.0f : __fdiv_rn(amax, 448.0f);
}

// ------------------------------------------------------------------ GEMM
constexpr int kF8Threads = 192;
constexpr int kF8Stages = 4;

template <int BT>
struct F8Cfg {
  static_assert(BT == 16 || BT == 128, "tokens per tile");
  static constexpr int S = kF8Stages;
  static constexpr int kXBytes = BT * 128;          // e4m3 activations, 128-byte rows, SW128
  static constexpr int kABytes = 128 * 128;         // e4m3 weights, SW128
  static constexpr int kWBytes = 128 * 64;          // packed INT4 codes, 64-byte rows, SW64
  static constexpr int kXRing = S * kXBytes;
  static constexpr int kARing = S * kABytes;
  static constexpr int kWRing = S * kWBytes;
  static constexpr int kBarOff = kXRing + kARing + kWRing;
  static constexpr int kSmemBytes = kBarOff + 256 + 1024;  // barriers and flags, alignment slack
  static constexpr int kAccCols = BT < 32 ? 32 : BT;
  static constexpr int kTmemCols = kAccCols <= 32 ? 32 : (kAccCols <= 64 ? 64 : 128);
  static_assert(kSmemBytes <= 232448, "shared memory budget");
  static_assert(3 * S * 8 + 16 + 12 <= 256, "barrier area");
};

struct F8Args {
  const float* s_x;  // one scale for the activation tensor
  const float* s_w;  // [N]
  __nv_bfloat16* out;
  int M, N, K, tiles_m;
};

// kind::f8f6f4 instruction descriptor: fp32 D, e4m3 A and B, both K-major,
// M = 128, N = n.
__host__ __device__ constexpr uint32_t idesc_f8(int n) {
  return (1u << 4)                        // D format: f32
         | (0u << 7) | (0u << 10)         // A, B: e4m3
         | (uint32_t(n >> 3) << 17) | (uint32_t(128 >> 4) << 24);
}

__device__ __forceinline__ void mma_f8_ss(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                          uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Eight INT4 codes of one packed word (code k at byte k % 4, high nibble for
// k >= 4) as eight e4m3 bytes, codes 0-3 in `lo`, 4-7 in `hi`.
__device__ __forceinline__ void w4_word_to_e4m3(uint32_t w, uint32_t& lo, uint32_t& hi) {
  uint32_t r[2] = {0u, 0u};
#pragma unroll
  for (int h = 0; h < 2; ++h) {
#pragma unroll
    for (int p = 0; p < 2; ++p) {
      const int b0 = 2 * p, b1 = 2 * p + 1;
      const float f0 = (float)((int)((w >> (8 * b0 + 4 * h)) & 15u) - 8);
      const float f1 = (float)((int)((w >> (8 * b1 + 4 * h)) & 15u) - 8);
      const uint32_t c2 = (uint32_t)__nv_cvt_float2_to_fp8x2(make_float2(f0, f1), __NV_SATFINITE, __NV_E4M3);
      r[h] |= (c2 & 0xFFFFu) << (16 * p);
    }
  }
  lo = r[0];
  hi = r[1];
}

template <int BT>
__global__ void __launch_bounds__(kF8Threads, 1)
    w4f8_gemm_kernel(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_w,
                     const F8Args p) {
  using C = F8Cfg<BT>;
  constexpr int S = C::S;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* xring = smem;
  uint8_t* aring = smem + C::kXRing;
  uint8_t* wring = aring + C::kARing;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::kBarOff);  // [S] weights and activations landed
  uint64_t* afull = full + S;                                        // [S] A tile written
  uint64_t* empty = afull + S;                                       // [S] MMAs of the stage done
  uint64_t* accfull = empty + S;
  uint64_t* drain = accfull + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int KB = p.K / 128;
  const int tile_m = blockIdx.x % p.tiles_m, tile_n = blockIdx.x / p.tiles_m;

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&afull[s], 4);
      mbar_init(&empty[s], 1);
    }
    mbar_init(accfull, 1);
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
    tma_prefetch_desc(&tm_x);
    tma_prefetch_desc(&tm_w);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, C::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  griddep_launch_dependents();

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      const uint64_t pol_stream = l2_policy_evict_first();
      const uint64_t pol_keep = l2_policy_evict_last();
      griddep_wait();  // activations and s_x may come from the preceding kernels
      uint32_t issued = 0, issued_par = 0;
      for (int it = 0; it < KB; ++it) {
        const int st = it % S;
        if (it >= S && !mbar_wait(&empty[st], (uint32_t)(it / S - 1) & 1u, abort_flag)) break;
        mbar_arrive_expect_tx(&full[st], (uint32_t)(C::kXBytes + C::kWBytes));
        tma_load_2d(wring + st * C::kWBytes, &tm_w, &full[st], it * 64, tile_n * 128, pol_stream);
        tma_load_2d(xring + st * C::kXBytes, &tm_x, &full[st], it * 128, tile_m * BT, pol_keep);
        issued |= 1u << st;
        issued_par = (issued_par & ~(1u << st)) | (((uint32_t)(it / S) & 1u) << st);
      }
      if (*abort_flag) {
        // no bulk copy may still be writing this CTA's shared memory when it leaves
        const unsigned long long t0w = globaltimer();
        for (int st = 0; st < S; ++st)
          if (issued & (1u << st))
            while (!mbar_try_wait(smem_u32(&full[st]), (issued_par >> st) & 1u) && globaltimer() - t0w < 100000000ull) {
            }
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ---------------------------------------------------------- MMA issuer
    bool any = false;
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_f8(BT);
      for (int it = 0; it < KB; ++it) {
        const int st = it % S;
        if (!mbar_wait(&afull[st], (uint32_t)(it / S) & 1u, abort_flag)) break;
        tc_fence_after();
        const uint64_t adesc = smem_desc_k_sw128(smem_u32(aring + st * C::kABytes));
        const uint64_t bdesc = smem_desc_k_sw128(smem_u32(xring + st * C::kXBytes));
#pragma unroll
        for (int j = 0; j < 4; ++j)
          mma_f8_ss(tmem_base, adesc + (uint64_t)(2 * j), bdesc + (uint64_t)(2 * j), idesc, (it > 0 || j > 0) ? 1u : 0u);
        tc_commit(&empty[st]);
        any = true;
      }
      if (any && !*abort_flag) tc_commit(accfull);
      if (any) {
        // all issued MMAs have finished before TMEM is released
        tc_commit(drain);
        const unsigned long long t0w = globaltimer();
        while (!mbar_try_wait(smem_u32(drain), 0) && globaltimer() - t0w < 100000000ull) {
        }
      }
    }
    __syncwarp();
  } else {
    // ----------------------------------- INT4 -> e4m3 expansion, then epilogue
    const int sub = warp & 3;
    const int r = sub * 32 + lane;  // weight row of the tile = TMEM lane
    const uint32_t t_lane = tmem_base + ((uint32_t)(sub * 32) << 16);
    const int sw = (r >> 1) & 3;    // 64-byte swizzle of the packed row's 16-byte chunks
    bool ok = true;
    for (int it = 0; it < KB && ok; ++it) {
      const int st = it % S;
      // the stage's loads have landed; its A tile is free (the stage was
      // refilled only after the MMAs that read it completed)
      if (!__all_sync(0xffffffffu, mbar_wait(&full[st], (uint32_t)(it / S) & 1u, abort_flag))) {
        ok = false;
        break;
      }
      const uint32_t wrow = smem_u32(wring + st * C::kWBytes) + r * 64;
      uint32_t v[32];
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const uint4 q = lds128(wrow + ((c ^ sw) << 4));
        const uint32_t w4[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) w4_word_to_e4m3(w4[i], v[8 * c + 2 * i], v[8 * c + 2 * i + 1]);
      }
      uint8_t* orow = aring + st * C::kABytes + r * 128;
#pragma unroll
      for (int c = 0; c < 8; ++c)
        *reinterpret_cast<uint4*>(orow + ((c ^ (r & 7)) << 4)) = make_uint4(v[4 * c], v[4 * c + 1], v[4 * c + 2], v[4 * c + 3]);
      fence_proxy_async_smem();  // read by the tensor core through the async proxy
      __syncwarp();
      if (lane == 0) mbar_arrive(&afull[st]);
    }
    if (ok && __all_sync(0xffffffffu, mbar_wait(accfull, 0, abort_flag))) {
      tc_fence_after();
      griddep_wait();
      const int n = tile_n * 128 + r;
      const bool n_ok = n < p.N;
      const float scale = n_ok ? __fmul_rn(ld_dep(p.s_x), __ldg(p.s_w + n)) : 0.0f;
      const int m0 = tile_m * BT;
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
        if (n_ok) {
#pragma unroll
          for (int i = 0; i < CH; ++i) {
            const int m = m0 + cc * CH + i;
            if (m < p.M) p.out[(size_t)m * p.N + n] = __float2bfloat16_rn(__fmul_rn(__uint_as_float(v[i]), scale));
          }
        }
      }
    }
  }

  // ---------------------------------------------------------------- teardown
  __syncwarp();
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, C::kTmemCols);
  }
}

}  // namespace lq

// lq_gemm_w4f8.cuh -- quantizers of the W4 x FP8 variant (FireQ page,
// abstract: INT4 weights with channel-wise scaling, FP8 activations with one
// scale for the tensor), sm_100a.
//
// Quantization (readings, shared with the oracle's definitions):
//   weights      s_w[n] = amax_n / 7, q = clamp(rint(w * (7 / amax_n)), -7, 7),
//                stored as u = q + 8 in the LiquidQuant nibble layout (word j
//                of a row holds codes 8j..8j+7, byte b = u[8j+b] | u[8j+4+b] << 4);
//   activations  one scale for the tensor, s_x = amax / 448 (448: the largest
//                finite e4m3 value), codes e4m3(x * (448 / amax)) rounded to
//                nearest even and saturated.
// The GEMM, out[m,n] = bf16(acc * (s_x * s_w[n])) with acc = sum_k e4m3(x) * q
// accumulated in fp32 by the tensor core, is the tile kernel's KIND 1
// (lq_gemm_kernel.cuh).
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

}  // namespace lq

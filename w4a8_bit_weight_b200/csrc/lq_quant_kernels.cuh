// lq_quant_kernels.cuh -- LiquidQuant weight quantization (offline), per-token
// activation quantization, and the INT8 expansion written to global memory.
//
// Every float decision is one IEEE binary32 operation with an explicit
// rounding intrinsic (no contraction, no fast-math), so the integer codes are
// bit-identical to a plain C implementation of the same formulas.
#pragma once

#include <cuda_bf16.h>

#include "lq_device.cuh"

namespace lq {

__device__ __forceinline__ float bf16_bits_to_f32(uint32_t h) { return __uint_as_float(h << 16); }

// Block-wide max of non-negative floats; every thread gets the result.
template <int THREADS>
__device__ __forceinline__ float block_max(float v, float* red) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (lane == 0) red[warp] = v;
  __syncthreads();
  if (warp == 0) {
    v = lane < THREADS / 32 ? red[lane] : 0.0f;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    if (lane == 0) red[0] = v;
  }
  __syncthreads();
  v = red[0];
  __syncthreads();
  return v;
}

// ---------------------------------------------------------------------------
// Weight quantization.  One CTA per output channel n (row of W).
//   Level 1: amax over the row; Q_i8 = clamp(rint(w * (119/amax)), -119, 119);
//            s_c = amax / 119 (zero row: s_c = 1, codes 0).
//   Level 2: per group of 64: mn, R = max - mn, s = max(1, round(R/15)),
//            a = 128 + mn, Q_u4 = min(15, round_half_up((Q - mn) / s)).
// One thread per group; the row is re-read from L1/L2 for the second pass.
// ---------------------------------------------------------------------------
constexpr int kQuantWThreads = 128;

__global__ void __launch_bounds__(kQuantWThreads) quantize_weights_kernel(
    const uint16_t* __restrict__ W, int N, int K, uint8_t* __restrict__ qw, uint8_t* __restrict__ s_u8,
    uint8_t* __restrict__ a_u8, float* __restrict__ s_c) {
  __shared__ float red[32];
  const int n = blockIdx.x;
  const uint16_t* row = W + (size_t)n * K;

  float amax = 0.0f;
  for (int k = threadIdx.x * 8; k < K; k += kQuantWThreads * 8) {
    const uint4 v = *reinterpret_cast<const uint4*>(row + k);
    const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      amax = fmaxf(amax, fabsf(bf16_bits_to_f32(w4[i] & 0xFFFFu)));
      amax = fmaxf(amax, fabsf(bf16_bits_to_f32(w4[i] >> 16)));
    }
  }
  amax = block_max<kQuantWThreads>(amax, red);
  const bool zero = (amax == 0.0f);
  const float inv = zero ? 0.0f : __fdiv_rn(119.0f, amax);
  if (threadIdx.x == 0) s_c[n] = zero ? 1.0f : __fdiv_rn(amax, 119.0f);

  const int ngroups = K / 64;
  for (int g = threadIdx.x; g < ngroups; g += kQuantWThreads) {
    int8_t q[64];
    int mn = 127, mx = -128;
    const uint4* src = reinterpret_cast<const uint4*>(row + g * 64);
#pragma unroll
    for (int c = 0; c < 8; ++c) {
      const uint4 v = src[c];
      const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const uint32_t h = (i & 1) ? (w4[i >> 1] >> 16) : (w4[i >> 1] & 0xFFFFu);
        int v8 = 0;
        if (!zero) {
          v8 = __float2int_rn(__fmul_rn(bf16_bits_to_f32(h), inv));
          v8 = min(119, max(-119, v8));
        }
        q[c * 8 + i] = (int8_t)v8;
        mn = min(mn, v8);
        mx = max(mx, v8);
      }
    }
    const int R = mx - mn;
    const int s = max(1, (2 * R + 15) / 30);
    const int a = 128 + mn;
    uint32_t words[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      uint32_t wv = 0;
#pragma unroll
      for (int b = 0; b < 4; ++b) {
        const int lo = min(15, (2 * (q[8 * j + b] - mn) + s) / (2 * s));
        const int hi = min(15, (2 * (q[8 * j + 4 + b] - mn) + s) / (2 * s));
        wv |= (uint32_t)(lo | (hi << 4)) << (8 * b);
      }
      words[j] = wv;
    }
    uint4* dst = reinterpret_cast<uint4*>(qw + (size_t)n * (K / 2) + g * 32);
    dst[0] = make_uint4(words[0], words[1], words[2], words[3]);
    dst[1] = make_uint4(words[4], words[5], words[6], words[7]);
    s_u8[(size_t)g * N + n] = (uint8_t)s;
    a_u8[(size_t)g * N + n] = (uint8_t)a;
  }
}

// ---------------------------------------------------------------------------
// Per-token symmetric INT8: one CTA per token row.  amax over the row, then
// x_q = clamp(rint(x * (127/amax)), -127, 127), s_x = amax / 127 (zero row:
// s_x = 1, codes 0).  16-byte loads of 8 bf16, 8-byte stores of 8 int8.
// ---------------------------------------------------------------------------
constexpr int kQuantActThreads = 256;

__device__ __forceinline__ uint32_t quant_pair_i8(uint32_t two_bf16, float inv) {
  int a = __float2int_rn(__fmul_rn(bf16_bits_to_f32(two_bf16 & 0xFFFFu), inv));
  int b = __float2int_rn(__fmul_rn(bf16_bits_to_f32(two_bf16 >> 16), inv));
  a = min(127, max(-127, a));
  b = min(127, max(-127, b));
  return (uint32_t)(a & 0xFF) | ((uint32_t)(b & 0xFF) << 8);
}

__global__ void __launch_bounds__(kQuantActThreads) quantize_act_kernel(const uint16_t* __restrict__ X,
                                                                        int K, int8_t* __restrict__ x_q,
                                                                        float* __restrict__ s_x) {
  __shared__ float red[32];
  griddep_launch_dependents();  // the GEMM that follows may start streaming its weights
  griddep_wait();               // X may be the output of the preceding kernel
  const int m = blockIdx.x;
  const uint16_t* row = X + (size_t)m * K;
  // The first kActHold chunks of 8 values per thread (K <= 16384) stay in
  // registers between the two passes; longer rows read the rest twice.
  constexpr int kActHold = 8;
  constexpr int kStep = kQuantActThreads * 8;
  auto row_max = [](const uint4& v, float a) {
    const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      a = fmaxf(a, fabsf(bf16_bits_to_f32(w4[i] & 0xFFFFu)));
      a = fmaxf(a, fabsf(bf16_bits_to_f32(w4[i] >> 16)));
    }
    return a;
  };
  uint4 hold[kActHold];
  float amax = 0.0f;
#pragma unroll
  for (int i = 0; i < kActHold; ++i) {
    const int k = threadIdx.x * 8 + i * kStep;
    hold[i] = k < K ? ld_dep(reinterpret_cast<const uint4*>(row + k)) : make_uint4(0u, 0u, 0u, 0u);
    amax = row_max(hold[i], amax);
  }
  for (int k = threadIdx.x * 8 + kActHold * kStep; k < K; k += kStep)
    amax = row_max(ld_dep(reinterpret_cast<const uint4*>(row + k)), amax);
  amax = block_max<kQuantActThreads>(amax, red);
  const bool zero = (amax == 0.0f);
  const float inv = zero ? 0.0f : __fdiv_rn(127.0f, amax);
  if (threadIdx.x == 0) s_x[m] = zero ? 1.0f : __fdiv_rn(amax, 127.0f);
  int8_t* out = x_q + (size_t)m * K;
  auto quant8 = [&](const uint4& v, int k) {
    uint2 o;
    o.x = quant_pair_i8(v.x, inv) | (quant_pair_i8(v.y, inv) << 16);
    o.y = quant_pair_i8(v.z, inv) | (quant_pair_i8(v.w, inv) << 16);
    *reinterpret_cast<uint2*>(out + k) = o;
  };
#pragma unroll
  for (int i = 0; i < kActHold; ++i) {
    const int k = threadIdx.x * 8 + i * kStep;
    if (k < K) quant8(hold[i], k);
  }
  for (int k = threadIdx.x * 8 + kActHold * kStep; k < K; k += kStep)
    quant8(ld_dep(reinterpret_cast<const uint4*>(row + k)), k);
}

// ---------------------------------------------------------------------------
// INT8 expansion to global memory, with the GEMM's own word routine.  One
// thread per packed 32-bit word (8 codes).
// ---------------------------------------------------------------------------
__global__ void dequant_weights_kernel(const uint32_t* __restrict__ qw, const uint8_t* __restrict__ s_u8,
                                       const uint8_t* __restrict__ a_u8, int N, int K,
                                       uint32_t* __restrict__ w_i8) {
  const long long words_per_row = K / 8;
  const long long idx = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= (long long)N * words_per_row) return;
  const int n = (int)(idx / words_per_row);
  const int j = (int)(idx % words_per_row);
  const int g = (j * 8) / 64;
  const uint32_t s = s_u8[(size_t)g * N + n];
  const uint32_t a4 = (uint32_t)a_u8[(size_t)g * N + n] * 0x01010101u;
  uint32_t lo, hi;
  lqq_expand_word(qw[idx], s, a4, lo, hi);
  w_i8[2 * idx] = lo;
  w_i8[2 * idx + 1] = hi;
}

}  // namespace lq

/*
 * lq_oracle.c -- plain, slow CPU oracle for the LiquidQuant W4A8 GEMM.
 *
 * TEST INFRASTRUCTURE ONLY.  This file is the independent reference that the
 * CUDA path is checked against.  Only the test suite, the smoke check and the
 * CPU-baseline leg of the benchmark may load it.  It shares no code, header,
 * table or constant with the CUDA library, and the library never calls it.
 *
 * Source of the method: "LiquidGEMM: Hardware-Efficient W4A8 GEMM Kernel for
 * High-Performance LLM Serving" (arXiv 2509.01229), as summarised on its
 * pith.science review page: the referee-report summary, the "What carries the
 * argument" section, major comment 3, minor comments 1-2, the circularity
 * rationale (Section 4, Eqs. 7, 9-12) and the free-parameter ledger (group
 * size 64).  The page does not print the equations themselves; every step
 * below states the reading taken where the text leaves it open.
 *
 * Arithmetic rules (chosen so the GPU can take every rounding decision in the
 * same precision):
 *   - floating point is IEEE binary32, one operation at a time; build with
 *     -ffp-contract=off and without -ffast-math;
 *   - round-to-integer of a float uses nearbyintf (round half to even);
 *   - integer rounding of a ratio of non-negative integers is round half up,
 *     written with integer division only.
 *
 * Functions return 0 on success and a negative code when an invariant that the
 * paper proves (the UINT8 range before the XOR, the int32 accumulator range)
 * does not hold, so a test can see the failure instead of a crash.
 *
 * Parity pins: every function here is pinned by the CPU tests in
 * tests/test_oracle_*.py against brute force, closed forms, invariants and
 * library routines (see those files).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define ORC_OK 0
#define ORC_ERR_ARG (-1)
#define ORC_ERR_UINT8_RANGE (-2) /* q*s + a left [0,255] before the XOR */
#define ORC_ERR_INT32_RANGE (-3) /* the exact sum does not fit int32 */

/* ---------------------------------------------------------------------- */
/* bf16 <-> fp32                                                           */
/* ---------------------------------------------------------------------- */

/* bf16 is the top half of an fp32 bit pattern: widening is exact. */
static float bf16_to_f32(uint16_t h) {
  uint32_t u = (uint32_t)h << 16;
  float f;
  memcpy(&f, &u, sizeof f);
  return f;
}

/* fp32 -> bf16, round to nearest, ties to even (NaN stays a quiet NaN). */
static uint16_t f32_to_bf16_rne(float f) {
  uint32_t u;
  memcpy(&u, &f, sizeof u);
  if ((u & 0x7F800000u) == 0x7F800000u && (u & 0x007FFFFFu) != 0u)
    return (uint16_t)((u >> 16) | 0x0040u);
  uint32_t lsb = (u >> 16) & 1u;
  u += 0x7FFFu + lsb;
  return (uint16_t)(u >> 16);
}

uint16_t lq_oracle_f32_to_bf16(float f) { return f32_to_bf16_rne(f); }
float lq_oracle_bf16_to_f32(uint16_t h) { return bf16_to_f32(h); }

static int clampi(int v, int lo, int hi) { return v < lo ? lo : (v > hi ? hi : v); }

int lq_oracle_num_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}

/* Threads the parallel loops use from now on (n >= 1); for timing the oracle
   on one core beside all of them. */
void lq_oracle_set_num_threads(int n) {
#ifdef _OPENMP
  if (n >= 1) omp_set_num_threads(n);
#else
  (void)n;
#endif
}

/* ---------------------------------------------------------------------- */
/* LiquidQuant level 1: per-channel symmetric INT8 in the protective range  */
/* [-119, 119] (review page: referee summary and circularity rationale,     */
/* "Q_i8 in [-119,119]", range adopted from QServe).                       */
/*   amax_n = max_k |W[n,k]|                                                */
/*   Q_i8[n,k] = clamp(rint(W[n,k] * (119 / amax_n)), -119, 119)            */
/*   s_c[n] = amax_n / 119                                                  */
/* Reading: the scale is amax/119; a zero row gets s_c = 1 and codes 0.     */
/* ---------------------------------------------------------------------- */
int lq_oracle_quantize_channels(const uint16_t* W, int N, int K, int8_t* q_i8, float* s_c) {
  if (!W || !q_i8 || !s_c || N < 0 || K < 0) return ORC_ERR_ARG;
  for (int n = 0; n < N; ++n) {
    const uint16_t* row = W + (size_t)n * K;
    float amax = 0.0f;
    for (int k = 0; k < K; ++k) {
      float a = fabsf(bf16_to_f32(row[k]));
      if (a > amax) amax = a;
    }
    if (amax == 0.0f) {
      s_c[n] = 1.0f;
      for (int k = 0; k < K; ++k) q_i8[(size_t)n * K + k] = 0;
      continue;
    }
    float inv = 119.0f / amax;
    for (int k = 0; k < K; ++k) {
      float t = bf16_to_f32(row[k]) * inv;
      int q = (int)nearbyintf(t);
      q_i8[(size_t)n * K + k] = (int8_t)clampi(q, -119, 119);
    }
    s_c[n] = amax / 119.0f;
  }
  return ORC_OK;
}

/* ---------------------------------------------------------------------- */
/* LiquidQuant level 2: each group of G consecutive INT8 values along K is  */
/* shifted into UINT8 by its minimum and quantized to UINT4 with an integer */
/* UINT8 scale (review page: referee summary, major comment 3 and minor     */
/* comment 2 -- round to nearest, s_u8 the rounded integer scale, at most   */
/* 16; "a = 2^7 + min(Q_i8)" from "What carries the argument").             */
/*   mn = min Q_i8, R = max Q_i8 - mn           (Q_u8 = Q_i8 - mn in [0,R]) */
/*   s_u8 = max(1, round(R / 15))               (= floor((2R + 15) / 30))   */
/*   Q_u4 = min(15, round(Q_u8 / s_u8))         (= floor((2Q_u8 + s)/(2s))) */
/*   a    = 128 + mn                                                         */
/* Packed layout (this library's own format): row n of qw has K/2 bytes;    */
/* the 32-bit little-endian word j of a row holds codes k = 8j..8j+7, with  */
/* byte b (0..3) = Q_u4[8j+b] | Q_u4[8j+4+b] << 4.  s_u8 and a_u8 are       */
/* stored [K/G][N], N contiguous.                                           */
/* ---------------------------------------------------------------------- */
int lq_oracle_quantize_groups(const int8_t* q_i8, int N, int K, int G, uint8_t* qw, uint8_t* s_u8,
                              uint8_t* a_u8) {
  if (!q_i8 || !qw || !s_u8 || !a_u8 || N < 0 || K < 0 || G <= 0 || K % G != 0 || K % 8 != 0)
    return ORC_ERR_ARG;
  int ngroups = K / G;
  uint8_t* codes = (uint8_t*)malloc((size_t)K);
  if (!codes) return ORC_ERR_ARG;
  for (int n = 0; n < N; ++n) {
    const int8_t* row = q_i8 + (size_t)n * K;
    for (int g = 0; g < ngroups; ++g) {
      int mn = 127, mx = -128;
      for (int i = 0; i < G; ++i) {
        int v = row[g * G + i];
        if (v < mn) mn = v;
        if (v > mx) mx = v;
      }
      int R = mx - mn;
      int s = (2 * R + 15) / 30;
      if (s < 1) s = 1;
      int a = 128 + mn;
      for (int i = 0; i < G; ++i) {
        int u = row[g * G + i] - mn; /* Q_u8, in [0, R] */
        int q = (2 * u + s) / (2 * s);
        if (q > 15) q = 15;
        codes[g * G + i] = (uint8_t)q;
      }
      s_u8[(size_t)g * N + n] = (uint8_t)s;
      a_u8[(size_t)g * N + n] = (uint8_t)a;
    }
    uint8_t* prow = qw + (size_t)n * (K / 2);
    for (int j = 0; j < K / 8; ++j)
      for (int b = 0; b < 4; ++b)
        prow[4 * j + b] = (uint8_t)(codes[8 * j + b] | (codes[8 * j + 4 + b] << 4));
  }
  free(codes);
  return ORC_OK;
}

/* Both levels, in the order the method applies them. */
int lq_oracle_quantize_weights(const uint16_t* W, int N, int K, int G, uint8_t* qw, uint8_t* s_u8,
                               uint8_t* a_u8, float* s_c, int8_t* q_i8_out) {
  if (N < 0 || K < 0) return ORC_ERR_ARG;
  int8_t* q = q_i8_out ? q_i8_out : (int8_t*)malloc((size_t)N * K + 1);
  if (!q) return ORC_ERR_ARG;
  int rc = lq_oracle_quantize_channels(W, N, K, q, s_c);
  if (rc == ORC_OK) rc = lq_oracle_quantize_groups(q, N, K, G, qw, s_u8, a_u8);
  if (!q_i8_out) free(q);
  return rc;
}

/* ---------------------------------------------------------------------- */
/* LiquidQuant dequantization (review page: "What carries the argument",   */
/* Eq. 12 in the circularity rationale):                                    */
/*   v = Q_u4 * s_u8 + a    (must stay in [0,255]: the UINT8 range proof)   */
/*   Q_i8_hat = int8(v XOR 0x80)                                            */
/* ---------------------------------------------------------------------- */
static int unpack_code(const uint8_t* prow, int k) {
  int j = k / 8, r = k % 8;
  uint8_t byte = prow[4 * j + (r & 3)];
  return r < 4 ? (byte & 0x0F) : (byte >> 4);
}

static int dequant_one(int q, int s, int a, int8_t* out) {
  int v = q * s + a;
  if (v < 0 || v > 255) return ORC_ERR_UINT8_RANGE;
  *out = (int8_t)(uint8_t)((unsigned)v ^ 0x80u);
  return ORC_OK;
}

int lq_oracle_dequant(const uint8_t* qw, const uint8_t* s_u8, const uint8_t* a_u8, int N, int K, int G,
                      int8_t* w_i8) {
  if (!qw || !s_u8 || !a_u8 || !w_i8 || N < 0 || K < 0 || G <= 0 || K % G != 0 || K % 8 != 0)
    return ORC_ERR_ARG;
  for (int n = 0; n < N; ++n) {
    const uint8_t* prow = qw + (size_t)n * (K / 2);
    for (int k = 0; k < K; ++k) {
      int g = k / G;
      int rc = dequant_one(unpack_code(prow, k), s_u8[(size_t)g * N + n], a_u8[(size_t)g * N + n],
                           &w_i8[(size_t)n * K + k]);
      if (rc) return rc;
    }
  }
  return ORC_OK;
}

/* ---------------------------------------------------------------------- */
/* Per-token symmetric INT8 activations (the review page's "8-bit           */
/* activations"; per-token symmetric is this library's reading):           */
/*   amax_m = max_k |X[m,k]|, x_q = clamp(rint(X * (127/amax_m)), -127, 127) */
/*   s_x[m] = amax_m / 127; a zero row gets s_x = 1 and codes 0.            */
/* ---------------------------------------------------------------------- */
int lq_oracle_quantize_act(const uint16_t* X, int M, int K, int8_t* x_q, float* s_x) {
  if (!X || !x_q || !s_x || M < 0 || K < 0) return ORC_ERR_ARG;
  for (int m = 0; m < M; ++m) {
    const uint16_t* row = X + (size_t)m * K;
    float amax = 0.0f;
    for (int k = 0; k < K; ++k) {
      float a = fabsf(bf16_to_f32(row[k]));
      if (a > amax) amax = a;
    }
    if (amax == 0.0f) {
      s_x[m] = 1.0f;
      for (int k = 0; k < K; ++k) x_q[(size_t)m * K + k] = 0;
      continue;
    }
    float inv = 127.0f / amax;
    for (int k = 0; k < K; ++k) {
      int q = (int)nearbyintf(bf16_to_f32(row[k]) * inv);
      x_q[(size_t)m * K + k] = (int8_t)clampi(q, -127, 127);
    }
    s_x[m] = amax / 127.0f;
  }
  return ORC_OK;
}

/* ---------------------------------------------------------------------- */
/* INT8 x INT8 -> int32 contraction (the GEMM loop nest over i, j, l of     */
/* Figure 2): acc[m,n] = sum_k x_q[m,k] * W_i8[n,k], summed exactly in      */
/* int64 and checked to fit int32.                                          */
/* ---------------------------------------------------------------------- */
int lq_oracle_gemm_i32(const int8_t* x_q, const int8_t* w_i8, int M, int N, int K, int32_t* acc) {
  if (!x_q || !w_i8 || !acc || M < 0 || N < 0 || K < 0) return ORC_ERR_ARG;
  int bad = 0;
#pragma omp parallel for schedule(static) reduction(| : bad)
  for (int m = 0; m < M; ++m) {
    const int8_t* xr = x_q + (size_t)m * K;
    for (int n = 0; n < N; ++n) {
      const int8_t* wr = w_i8 + (size_t)n * K;
      int64_t s = 0;
      for (int k = 0; k < K; ++k) s += (int64_t)xr[k] * (int64_t)wr[k];
      if (s < INT32_MIN || s > INT32_MAX) bad = 1;
      acc[(size_t)m * N + n] = (int32_t)s;
    }
  }
  return bad ? ORC_ERR_INT32_RANGE : ORC_OK;
}

/* ---------------------------------------------------------------------- */
/* Scale epilogue: y = float(acc) * (s_x[m] * s_c[n]), then bf16 round to   */
/* nearest even.  The pages give no epilogue; this is the per-token times   */
/* per-channel reading, with the product of the two scales taken first.     */
/* ---------------------------------------------------------------------- */
int lq_oracle_epilogue(const int32_t* acc, const float* s_x, const float* s_c, int M, int N,
                       uint16_t* out) {
  if (!acc || !s_x || !s_c || !out || M < 0 || N < 0) return ORC_ERR_ARG;
  for (int m = 0; m < M; ++m)
    for (int n = 0; n < N; ++n) {
      float scale = s_x[m] * s_c[n];
      float y = (float)acc[(size_t)m * N + n] * scale;
      out[(size_t)m * N + n] = f32_to_bf16_rne(y);
    }
  return ORC_OK;
}

/* ---------------------------------------------------------------------- */
/* SwiGLU epilogue of a gate/up pair (the FFN layers of the LiquidGEMM      */
/* review page's Fig. 12 caption are Llama-style gated layers; the pages    */
/* give no formula, the reading is the common one): the two projections of  */
/* the same input, each with the epilogue above in fp32 (not rounded to     */
/* bf16), then silu(gate) * up rounded once to bf16, with                   */
/*   silu(g) = g / (1 + exp(-g))    (IEEE fp32 steps, expf from libm).      */
/* The gate/up weights are one interleaved [2N, K] matrix quantized row by  */
/* row: row 2n is gate channel n, row 2n+1 up channel n (this library's     */
/* layout choice).  acc is [M, 2N], out [M, N].                             */
/* ---------------------------------------------------------------------- */
int lq_oracle_swiglu_epilogue(const int32_t* acc, const float* s_x, const float* s_c, int M, int N,
                              uint16_t* out) {
  if (!acc || !s_x || !s_c || !out || M < 0 || N < 0) return ORC_ERR_ARG;
  for (int m = 0; m < M; ++m)
    for (int n = 0; n < N; ++n) {
      const int32_t* row = acc + (size_t)m * 2 * N;
      float yg = (float)row[2 * n] * (s_x[m] * s_c[2 * n]);
      float yu = (float)row[2 * n + 1] * (s_x[m] * s_c[2 * n + 1]);
      float e = expf(-yg);
      float silu = yg / (1.0f + e);
      out[(size_t)m * N + n] = f32_to_bf16_rne(silu * yu);
    }
  return ORC_OK;
}

/* Whole W4A8 GEMM from already-quantized operands: dequant, contraction,
 * epilogue.  acc_out may be NULL. */
int lq_oracle_w4a8_gemm(const int8_t* x_q, const float* s_x, const uint8_t* qw, const uint8_t* s_u8,
                        const uint8_t* a_u8, const float* s_c, int M, int N, int K, int G,
                        uint16_t* out, int32_t* acc_out) {
  if (M < 0 || N < 0 || K < 0) return ORC_ERR_ARG;
  int8_t* w = (int8_t*)malloc((size_t)N * K + 1);
  int32_t* acc = acc_out ? acc_out : (int32_t*)malloc((size_t)M * N * sizeof(int32_t) + 4);
  int rc = (w && acc) ? ORC_OK : ORC_ERR_ARG;
  if (rc == ORC_OK) rc = lq_oracle_dequant(qw, s_u8, a_u8, N, K, G, w);
  if (rc == ORC_OK) rc = lq_oracle_gemm_i32(x_q, w, M, N, K, acc);
  if (rc == ORC_OK) rc = lq_oracle_epilogue(acc, s_x, s_c, M, N, out);
  free(w);
  if (!acc_out) free(acc);
  return rc;
}

/* The same result for a list of single outputs (m_idx[i], n_idx[i]); each
 * one dequantizes its weight row on the fly.  For shapes too large for the
 * full oracle.  acc_out may be NULL. */
int lq_oracle_w4a8_gemm_sampled(const int8_t* x_q, const float* s_x, const uint8_t* qw,
                                const uint8_t* s_u8, const uint8_t* a_u8, const float* s_c, int M,
                                int N, int K, int G, const int64_t* m_idx, const int64_t* n_idx,
                                int64_t count, uint16_t* out, int32_t* acc_out) {
  if (!x_q || !s_x || !qw || !s_u8 || !a_u8 || !s_c || !m_idx || !n_idx || !out || G <= 0 ||
      K % G != 0 || K % 8 != 0)
    return ORC_ERR_ARG;
  int bad = 0;
#pragma omp parallel for schedule(dynamic, 16) reduction(| : bad)
  for (int64_t i = 0; i < count; ++i) {
    int64_t m = m_idx[i], n = n_idx[i];
    if (m < 0 || m >= M || n < 0 || n >= N) {
      bad |= 1;
      continue;
    }
    const uint8_t* prow = qw + (size_t)n * (K / 2);
    const int8_t* xr = x_q + (size_t)m * K;
    int64_t s = 0;
    for (int k = 0; k < K; ++k) {
      int g = k / G;
      int8_t w;
      if (dequant_one(unpack_code(prow, k), s_u8[(size_t)g * N + n], a_u8[(size_t)g * N + n], &w)) {
        bad |= 2;
        break;
      }
      s += (int64_t)xr[k] * (int64_t)w;
    }
    if (s < INT32_MIN || s > INT32_MAX) bad |= 4;
    int32_t acc = (int32_t)s;
    if (acc_out) acc_out[i] = acc;
    float scale = s_x[m] * s_c[n];
    out[i] = f32_to_bf16_rne((float)acc * scale);
  }
  if (bad & 1) return ORC_ERR_ARG;
  if (bad & 2) return ORC_ERR_UINT8_RANGE;
  if (bad & 4) return ORC_ERR_INT32_RANGE;
  return ORC_OK;
}

/* ====================================================================== */
/* W4 x FP8 variant (FireQ page, abstract: INT4 weights with channel-wise  */
/* scaling, FP8 activations with a per-tensor scale).  The pages give no   */
/* formulas; the readings used here:                                       */
/*   weights:     s_w[n] = amax_n / 7, q = clamp(rint(w * (7 / amax_n)),   */
/*                -7, 7), stored as u = q + 8 in the LiquidQuant nibble    */
/*                layout; a zero row gets s_w = 1 and q = 0;               */
/*   activations: one scale for the tensor, s_x = amax / 448 (448 is the   */
/*                largest finite e4m3 value), codes e4m3(x * (448 / amax)) */
/*                rounded to nearest even and saturated to +-448; a zero   */
/*                tensor gets s_x = 1;                                     */
/*   GEMM:        acc[m,n] = sum_k e4m3(x)[m,k] * q[n,k], exact (every     */
/*                product and partial sum is a multiple of 2^-9 far below  */
/*                2^53 in magnitude, so double holds it exactly), then     */
/*                out = bf16((float)acc * (s_x * s_w[n])).                 */
/* ====================================================================== */

/* e4m3: 1 sign bit, 4 exponent bits (bias 7), 3 mantissa bits; exponent    */
/* field 0 is subnormal (m * 2^-9); S.1111.111 is NaN; no infinities; the   */
/* largest finite value is 1.75 * 2^8 = 448.                                 */
float lq_oracle_e4m3_to_f32(uint8_t c) {
  const int s = c >> 7, e = (c >> 3) & 15, m = c & 7;
  if (e == 15 && m == 7) return NAN;
  const float v = e == 0 ? ldexpf((float)m, -9) : ldexpf(1.0f + (float)m / 8.0f, e - 7);
  return s ? -v : v;
}

/* Round to nearest even, saturating finite values beyond 448 to 448. */
uint8_t lq_oracle_f32_to_e4m3(float x) {
  if (isnan(x)) return 0x7F;
  const uint8_t sign = signbit(x) ? 0x80 : 0x00;
  const float a = fabsf(x);
  if (a >= 448.0f) return sign | 0x7E;
  int e2;
  frexpf(a, &e2);               /* a = f * 2^e2, f in [0.5, 1): floor(log2 a) = e2 - 1 */
  int E = (a == 0.0f) ? 1 : (e2 - 1) + 7;
  if (E < 1) E = 1;             /* the subnormal range shares exponent field 1's quantum */
  const float quantum = ldexpf(1.0f, E - 7 - 3);
  const int n = (int)nearbyintf(a / quantum);  /* a / quantum is exact (power-of-two quantum) */
  /* n in [0, 16]: below 8 only in the subnormal range; 16 carries into the next binade */
  int code;
  if (n < 8)
    code = n;                       /* subnormal (E == 1 here) */
  else if (n == 16)
    code = ((E + 1) << 3);          /* E + 1 <= 15: a < 448 never rounds past 448 */
  else
    code = (E << 3) | (n - 8);
  return sign | (uint8_t)code;
}

int lq_oracle_quantize_weights_w4(const uint16_t* W, int N, int K, uint8_t* qw4, float* s_w) {
  if (!W || !qw4 || !s_w || N < 0 || K < 0 || K % 8 != 0) return ORC_ERR_ARG;
  for (int n = 0; n < N; ++n) {
    const uint16_t* row = W + (size_t)n * K;
    float amax = 0.0f;
    for (int k = 0; k < K; ++k) {
      float a = fabsf(bf16_to_f32(row[k]));
      if (a > amax) amax = a;
    }
    const float inv = amax == 0.0f ? 0.0f : 7.0f / amax;
    s_w[n] = amax == 0.0f ? 1.0f : amax / 7.0f;
    uint8_t* prow = qw4 + (size_t)n * (K / 2);
    memset(prow, 0, (size_t)K / 2);
    for (int k = 0; k < K; ++k) {
      const int q = amax == 0.0f ? 0 : clampi((int)nearbyintf(bf16_to_f32(row[k]) * inv), -7, 7);
      const int u = q + 8;
      const int j = k / 8, r = k % 8;       /* word j, code r: byte r%4, high nibble if r >= 4 */
      prow[4 * j + (r & 3)] |= (uint8_t)(r < 4 ? u : u << 4);
    }
  }
  return ORC_OK;
}

int lq_oracle_quantize_act_f8(const uint16_t* X, int M, int K, uint8_t* x_f8, float* s_x) {
  if (!X || !x_f8 || !s_x || M < 0 || K < 0) return ORC_ERR_ARG;
  float amax = 0.0f;
  for (size_t i = 0; i < (size_t)M * K; ++i) {
    float a = fabsf(bf16_to_f32(X[i]));
    if (a > amax) amax = a;
  }
  const float inv = amax == 0.0f ? 0.0f : 448.0f / amax;
  *s_x = amax == 0.0f ? 1.0f : amax / 448.0f;
  for (size_t i = 0; i < (size_t)M * K; ++i) x_f8[i] = lq_oracle_f32_to_e4m3(bf16_to_f32(X[i]) * inv);
  return ORC_OK;
}

int lq_oracle_w4f8_gemm(const uint8_t* x_f8, float s_x, const uint8_t* qw4, const float* s_w, int M, int N, int K,
                        uint16_t* out, double* acc_out) {
  if (!x_f8 || !qw4 || !s_w || !out || M < 0 || N < 0 || K < 0 || K % 8 != 0) return ORC_ERR_ARG;
  int bad = 0;
#pragma omp parallel for schedule(dynamic, 4) reduction(| : bad)
  for (int n = 0; n < N; ++n) {
    const uint8_t* prow = qw4 + (size_t)n * (K / 2);
    for (int m = 0; m < M; ++m) {
      const uint8_t* xr = x_f8 + (size_t)m * K;
      double s = 0.0;
      for (int k = 0; k < K; ++k) {
        const float xv = lq_oracle_e4m3_to_f32(xr[k]);
        if (isnan(xv)) bad |= 1;
        const int u = unpack_code(prow, k);
        s += (double)xv * (double)(u - 8);
      }
      if (acc_out) acc_out[(size_t)m * N + n] = s;
      out[(size_t)m * N + n] = f32_to_bf16_rne((float)s * (s_x * s_w[n]));
    }
  }
  return bad ? ORC_ERR_ARG : ORC_OK;
}

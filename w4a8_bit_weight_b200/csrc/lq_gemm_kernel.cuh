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
// Warp roles (192 threads):
//   warp 0     TMA producer: packed u4 weights, u8 scale/offset tiles and
//              int8 activation tiles into a ring of shared-memory stages.
//   warp 1     allocates TMEM; one thread issues tcgen05.mma kind::i8.
//   warps 2-5  LiquidQuant expansion (one weight row per thread, one IMAD +
//              one XOR per four weights) into the TMEM A slot of the stage,
//              then the epilogue: int32 accumulators -> scales -> bf16.
//
// Hand-offs: the weights of a K-block complete on its stage's weight barrier,
// the preloaded activation tiles on one barrier, a refilled activation tile
// on its stage's barrier (waited for by one expansion warp before its slot is
// reported ready).  The expansion warps publish how many blocks they have
// handed over; the MMA thread issues every block known to be ready as one
// run.  Stages and slots go back to the producer through MMA commits.
//
// Schedules (CS template parameter):
//   CS >= 1  split-K inside a thread-block cluster of CS CTAs: the cluster
//            owns one 128-row x BT-token tile, CTA rank r takes the r-th
//            slice of the K-blocks.  The partial sums are reduce-scattered
//            through distributed shared memory: each CTA owns one piece of
//            the tile (row quarters, token halves of them when CS = 8),
//            receives the other CTAs' partials of it by bulk copies, adds
//            them and writes that piece of the output.  CS = 1 is the plain
//            one-CTA-per-tile schedule.
//   CS == 0  stream-K over any grid: the M x N x K work is cut into units of
//            one tile x one K-block of 128; CTA c takes units
//            [c*U/G, (c+1)*U/G).  Tiles shared by several CTAs are summed in
//            an int32 workspace with atomic adds; the CTA that arrives last
//            (atomic ticket) applies the epilogue and restores the workspace
//            and the ticket to zero.
// Integer sums are order-independent, so every schedule gives bit-identical
// results.
//
// Programmatic dependent launch: every CTA lets the next kernel launch as soon
// as its prologue is done; the producer issues the weight loads of the first
// stages before griddepcontrol.wait (weights are never written by the kernel
// this launch overlaps), and the activation loads after it; the epilogue
// waits before it reads scales or writes the output.
//
// Also here: the grouped form (GemmArgs::m_off, one weight matrix per group
// of token rows, each cluster finding its group on the device), the fused
// activation quantization (FQ), the variants of the dequantization ablation
// (DQ), and the W4 x FP8 variant (KIND 1, FireQ page, abstract): symmetric
// INT4 weights expanded to e4m3 (w4_word_to_e4m3, exact), e4m3 activations
// with one scale for the tensor, tcgen05.mma kind::f8f6f4 into fp32
// accumulators.  The schedules, the pipeline and the reduce-scatter are the
// same; the partial sums are fp32, added in a fixed order, so every run of
// one schedule gives the same bits (different schedules may differ in the
// last place of the fp32 sums).
#pragma once

#include <cuda_bf16.h>

#include "lq_device.cuh"
#include "lq_quant_kernels.cuh"

namespace lq {

constexpr int kBlockN = 128;        // weight rows per tile (MMA M)
constexpr int kBlockK = 128;        // K per pipeline stage (two groups of 64)
// Expansion groups (template parameter EG): groups of four warps (one per
// TMEM sub-partition) take alternate K-blocks, so that one group's TMEM
// stores overlap the other's integer work; group 0 also runs the epilogue.
// Two groups pay where a 16-token decode CTA expands all of its preloaded
// K-blocks at once; where K-slices stream through the ring, the register cap
// of ten warps costs more than the overlap gains, and they keep one.  Stream-K
// and the fused quantization always keep one: a stream-K CTA runs several
// tiles through one accumulator, which the epilogue must have read before the
// next tile's first MMA (with one group the epilogue warps expanding the next
// tile's blocks themselves imply that order); the quantizing warps need more
// registers than two CTAs of ten warps could have.
__host__ __device__ constexpr int gemm_threads(int eg) { return 32 * (2 + 4 * eg); }
constexpr int kGemmThreads = gemm_threads(1);

__host__ __device__ constexpr int round_up_c(int x, int a) { return (x + a - 1) / a * a; }
__host__ __device__ constexpr int max_c(int a, int b) { return a > b ? a : b; }

// DQ selects the expansion for the ablation of the dequantization pipeline
// (the product path is DQ = 0): bit 0 = per-element expansion instead of the
// SWAR form; bit 1 = the expanded weights go to a shared-memory A tile per
// slot and the MMA reads both operands from shared memory (explicit
// pipeline), instead of tensor memory (implicit pipeline).
template <int BT, int CS, int DQ = 0>
struct GemmCfg {
  static_assert(BT == 16 || BT == 32 || BT == 64 || BT == 128 || BT == 256, "tokens per tile");
  static_assert(CS >= 0 && CS <= 8, "cluster size");
  // shared-memory stages: a ring of activation tiles and a ring of weight tiles
  // (32-token tiles in 8-CTA clusters keep to 7, so that two CTAs fit an SM;
  // 128-token tiles in clusters keep to 7 beside the split-K receive buffer)
  static constexpr int kStages =
      BT <= 32 ? (BT == 32 && CS == 8 ? 7 : 8) : BT == 64 ? 6 : (BT == 128 ? (CS >= 2 ? 7 : 8) : 5);
  static constexpr int kXBytes = BT * kBlockK;             // int8 activation tile, 128-byte rows (SW128)
  static constexpr int kWBytes = kBlockN * kBlockK / 2;    // packed u4 weight tile, 64-byte rows (SW64)
  static constexpr int kSABytes = 2 * kBlockN;             // 2 groups x 128 rows of u8
  static constexpr int kWStage = kWBytes + 2 * kSABytes;   // 8704 = 17 x 512: keeps the SW64 alignment
  static constexpr uint32_t kTxX = kXBytes;
  static constexpr uint32_t kTxW = kWStage;
  static constexpr int kAccCols = BT < 32 ? 32 : BT;      // int32 accumulator columns
  // TMEM A slots (one expanded K-block of 128 each, 32 columns), independent of
  // the number of shared-memory stages; small tiles keep to 256 columns so two
  // CTAs can share an SM
  static constexpr int kSlots = BT <= 64 ? (kStages < (256 - kAccCols) / 32 ? kStages : (256 - kAccCols) / 32)
                                         : kStages;
  static constexpr int kTmemCols = (kAccCols + kSlots * 32 <= 256) ? 256 : 512;
  // Cluster split-K is a reduce-scatter over token slices: CTA rank o owns
  // tokens [o kT, (o + 1) kT) of the tile for all 128 weight rows; every other
  // CTA sends it those columns of its partial sums straight from registers
  // (st.async into [source][row][kT] int32, counted on the owner's barrier).
  static constexpr int kT = CS >= 2 ? BT / CS : BT;                // tokens per owner
  static constexpr int kRedBytes = CS >= 2 ? (CS - 1) * kBlockN * kT * 4 : 0;  // received slices
  static constexpr int kXRing = kStages * kXBytes;
  static constexpr int kASmem = (DQ & 2) ? kSlots * kBlockN * kBlockK : 0;  // explicit pipeline: int8 A tiles, SW128
  static constexpr int kWRing = kStages * kWStage;
  // mbarriers and flags in the first 512 bytes; with fused activation
  // quantization, the cluster's partial row maxima [CS][16] and s_x [16]
  // after; the expansion warps' progress counters [4 EG] at byte 1088
  static constexpr int kBarBytes = 1152;
  static constexpr int kUsed = kXRing + kASmem + kWRing + kRedBytes + kBarBytes + 1024;  // + alignment slack
  // Shared memory also bounds how many CTAs share an SM: a 512-column CTA
  // takes at least 120 KB (one per SM), a 256-column CTA at least 80 KB (at
  // most two per SM), so co-resident CTAs never exceed the 512 TMEM columns.
  static constexpr int kSmemBytes = max_c(round_up_c(kUsed, 1024), kTmemCols == 512 ? 122880 : 81920);
  static_assert(kAccCols + kSlots * 32 <= kTmemCols, "TMEM budget");
  static_assert(kSmemBytes <= 232448, "shared memory budget");
  static_assert(kXBytes % 1024 == 0 && (kXRing + kASmem + kWRing + kRedBytes) % 8 == 0, "alignment");
  static_assert((3 * kStages + 2 * kSlots + 9) * 8 + 16 <= 512, "barrier area");
  // One K-block more than TMEM slots and no refills (a 16- or 32-token decode
  // CTA holding its whole K-slice): the extra block is expanded into the
  // shared memory of weight stages 0-1 (free by then) and multiplied with A
  // from shared memory, instead of waiting for slot 0 to be released.
  static_assert(kSlots < 2 || 128 * kBlockK <= 2 * kWStage, "overflow block fits two weight stages");
  static_assert(512 + 8 * 16 * 4 + 16 * 4 <= 1088 && 1088 + 4 * 2 * 4 <= kBarBytes,
                "fused-quantization and progress area");
  static_assert(CS < 2 || (kT >= 2 && kT % 2 == 0 && (kT == 2 || kT % 4 == 0)), "token slice: 2 or a multiple of 4");
};

struct GemmArgs {
  const uint16_t* x_bf16;  // fused activation quantization only: X [M, K] bf16
  const float* s_x;
  const float* s_c;
  void* out;             // bf16 [M, N] or int32 [M, N]
  int32_t* ws;           // stream-K only: [tiles][BT][128] int32, zero between calls
  unsigned int* ticket;  // stream-K only: [tiles], zero between calls
  int M, N, K;
  int tiles_m, KB;
  long long U;           // units = tiles * KB
  // grouped GEMM (one tile per cluster): group e multiplies token rows
  // [m_off[e], m_off[e+1]) by weight rows [e*N, (e+1)*N); tiles_m then bounds
  // the token tiles of all groups together
  const int* m_off = nullptr;
  int groups = 0;
};

// (tile, K-block) of a unit, stepped without divisions: an integer division
// costs a few hundred cycles, as much as the copy it would address.
struct UnitCursor {
  int kb, tile_m, tile_n;
  __device__ __forceinline__ UnitCursor(long long u, int KB, int tiles_m) {
    const int t = (int)(u / KB);
    kb = (int)(u - (long long)t * KB);
    tile_n = t / tiles_m;
    tile_m = t - tile_n * tiles_m;
  }
  // the cursor at K-block kb of tile t (32-bit arithmetic only)
  __device__ __forceinline__ static UnitCursor at(int t, int kb, int tiles_m) {
    UnitCursor c;
    c.kb = kb;
    c.tile_n = t / tiles_m;
    c.tile_m = t - c.tile_n * tiles_m;
    return c;
  }
  UnitCursor() = default;
  __device__ __forceinline__ void next(int KB, int tiles_m) {
    if (++kb == KB) {
      kb = 0;
      if (++tile_m == tiles_m) {
        tile_m = 0;
        ++tile_n;
      }
    }
  }
};

__device__ __forceinline__ long long cta_of_unit(long long u, long long U, long long G) {
  return ((u + 1) * G + U - 1) / U - 1;
}

// Grouped GEMM: the group of token tile j, the token tiles of all groups
// numbered in group order (ceil(rows / bt) tiles per group).  Called by a
// whole warp: each lane takes one group per step, an inclusive prefix sum of
// the tile counts (shuffles) and a ballot find the group.  Returns the group,
// or -1 past the last group's rows, and the tile's first row and the group's
// end row.  Offsets are read clamped to [0, M]: whatever they hold, no row
// outside the activations and the output is ever addressed.
__device__ __forceinline__ int find_group_tile(const int* m_off, int groups, int M, int bt, int j, int& row0,
                                               int& mend) {
  const int lane = threadIdx.x & 31;
  auto off_at = [&](int e) { return min(max(ld_dep(m_off + e), 0), M); };
  int ge = -1, before = 0, run = 0;
  for (int base = 0; base < groups && ge < 0; base += 32) {
    const int e = base + lane;
    int cnt = 0;
    if (e < groups) cnt = max(0, off_at(e + 1) - off_at(e) + bt - 1) / bt;
    int incl = cnt;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int v = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += v;
    }
    const unsigned hit = __ballot_sync(0xffffffffu, cnt > 0 && j >= run + incl - cnt && j < run + incl);
    if (hit) {
      const int l = __ffs(hit) - 1;
      ge = base + l;
      before = run + __shfl_sync(0xffffffffu, incl - cnt, l);
    }
    run += __shfl_sync(0xffffffffu, incl, 31);
  }
  if (ge >= 0) {
    row0 = off_at(ge) + (j - before) * bt;
    mend = off_at(ge + 1);
  }
  return ge;
}

// One lane polls the barrier; the decision is broadcast to the warp (cheaper
// than 32 lanes polling the same mbarrier).
__device__ __forceinline__ bool lane0_wait(uint64_t* bar, uint32_t parity, volatile int* abort_flag) {
  bool ok = true;
  if ((threadIdx.x & 31) == 0) ok = mbar_wait(bar, parity, abort_flag);
  return __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
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

// Four bf16 (two words, in order) -> four INT8 codes, one word: the same codes as
// quant_pair_i8 (rint(x * inv), then into [-127, 127]: the floor is applied
// before the saturating pack, which supplies the ceiling).
__device__ __forceinline__ uint32_t quant_quad_i8(uint32_t w01, uint32_t w23, float inv) {
  const int i0 = max(-127, __float2int_rn(__fmul_rn(__uint_as_float(w01 << 16), inv)));
  const int i1 = max(-127, __float2int_rn(__fmul_rn(__uint_as_float(w01 & 0xFFFF0000u), inv)));
  const int i2 = max(-127, __float2int_rn(__fmul_rn(__uint_as_float(w23 << 16), inv)));
  const int i3 = max(-127, __float2int_rn(__fmul_rn(__uint_as_float(w23 & 0xFFFF0000u), inv)));
  uint32_t hi, r;
  asm("cvt.pack.sat.s8.s32.b32 %0, %1, %2, 0;" : "=r"(hi) : "r"(i3), "r"(i2));
  asm("cvt.pack.sat.s8.s32.b32 %0, %1, %2, %3;" : "=r"(r) : "r"(i1), "r"(i0), "r"(hi));
  return r;
}

// Accumulator words: int32 sums (W4A8) or fp32 sums (W4 x FP8).
template <bool F8>
__device__ __forceinline__ float acc_f32(uint32_t v) {
  if constexpr (F8)
    return __uint_as_float(v);
  else
    return __int2float_rn((int32_t)v);
}
template <bool F8>
__device__ __forceinline__ uint32_t acc_add(uint32_t a, uint32_t b) {
  if constexpr (F8)
    return __float_as_uint(__fadd_rn(__uint_as_float(a), __uint_as_float(b)));
  else
    return a + b;
}
template <bool F8>
__device__ __forceinline__ void mma_ts_k(uint32_t d, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc, uint32_t acc) {
  if constexpr (F8)
    mma_f8_ts(d, a_tmem, b_desc, idesc, acc);
  else
    mma_i8_ts(d, a_tmem, b_desc, idesc, acc);
}
template <bool F8>
__device__ __forceinline__ void mma_ss_k(uint32_t d, uint64_t a_desc, uint64_t b_desc, uint32_t idesc, uint32_t acc) {
  if constexpr (F8)
    mma_f8_ss(d, a_desc, b_desc, idesc, acc);
  else
    mma_i8_ss(d, a_desc, b_desc, idesc, acc);
}

// Writes TC consecutive tokens [m_first, m_first + TC) of this thread's output
// column n from the accumulators v.  sx_lane holds s_x[m_first + lane] (lanes
// < TC).  The token scales are gathered first, so that the stores do not wait
// on one another.  Every lane of the warp must call it.
template <bool OUT_I32, int TC, bool F8 = false>
__device__ __forceinline__ void store_chunk(const GemmArgs& p, int m_first, int mend, int n, bool n_ok, const uint32_t* v,
                                            float sx_lane, float sc) {
  float scale[TC];
#pragma unroll
  for (int i = 0; i < TC; ++i) scale[i] = __fmul_rn(__shfl_sync(0xffffffffu, sx_lane, i), sc);
  if (!n_ok) return;
  const int mlim = mend - m_first;
  if constexpr (OUT_I32) {
    int32_t* o = reinterpret_cast<int32_t*>(p.out) + (size_t)m_first * p.N + n;
#pragma unroll
    for (int i = 0; i < TC; ++i)
      if (i < mlim) o[(size_t)i * p.N] = (int32_t)v[i];
  } else {
    __nv_bfloat16* o = reinterpret_cast<__nv_bfloat16*>(p.out) + (size_t)m_first * p.N + n;
#pragma unroll
    for (int i = 0; i < TC; ++i)
      if (i < mlim) o[(size_t)i * p.N] = __float2bfloat16_rn(__fmul_rn(acc_f32<F8>(v[i]), scale[i]));
  }
}

// SwiGLU epilogue of an interleaved gate/up pair: weight row 2j is gate
// channel j, row 2j + 1 up channel j, so the gate and up values of an output
// column sit in lanes 2i and 2i + 1 of a warp.  silu(g) = g / (1 + exp(-g))
// in IEEE fp32 steps (expf: CUDA's, within 2 ulp), one bf16 rounding.
__device__ __forceinline__ float silu_f32(float g) { return __fdiv_rn(g, __fadd_rn(1.0f, expf(-g))); }

// For a token pair (t, t + 1) whose fp32 values in this lane are y0, y1 (gate
// values in even lanes, up values in odd lanes): the even lane returns the
// output of token t, the odd lane that of token t + 1.  Every lane must call it.
__device__ __forceinline__ float swiglu_pair(float y0, float y1) {
  const bool odd = threadIdx.x & 1;
  const float other = __shfl_xor_sync(0xffffffffu, odd ? y0 : y1, 1);  // partner's value of this lane's token
  return odd ? __fmul_rn(silu_f32(other), y1) : __fmul_rn(silu_f32(y0), other);
}

// Writes TC tokens [m_first, m_first + TC) of output column n / 2 from the
// accumulators v of weight row n (SwiGLU; see swiglu_pair).  Every lane must call it.
template <int TC>
__device__ __forceinline__ void store_chunk_swiglu(const GemmArgs& p, int m_first, int mend, int n, bool n_ok,
                                                   const uint32_t* v, float sx_lane, float sc) {
  const bool odd = threadIdx.x & 1;
  const int ld = p.N >> 1;
  __nv_bfloat16* o = reinterpret_cast<__nv_bfloat16*>(p.out) + (size_t)m_first * ld + (n >> 1);
#pragma unroll
  for (int i = 0; i < TC; i += 2) {
    const float y0 = __fmul_rn(__int2float_rn((int32_t)v[i]), __fmul_rn(__shfl_sync(0xffffffffu, sx_lane, i), sc));
    const float y1 =
        __fmul_rn(__int2float_rn((int32_t)v[i + 1]), __fmul_rn(__shfl_sync(0xffffffffu, sx_lane, i + 1), sc));
    const float out = swiglu_pair(y0, y1);
    const int t = i + (odd ? 1 : 0);
    if (n_ok && m_first + t < mend) o[(size_t)t * ld] = __float2bfloat16_rn(out);
  }
}

// Output element from an accumulator and the token's scale s_x[m] (given).
template <bool OUT_I32>
__device__ __forceinline__ void store_out_sx(const GemmArgs& p, int m, int n, int32_t acc, float sx, float sc) {
  if constexpr (OUT_I32) {
    reinterpret_cast<int32_t*>(p.out)[(size_t)m * p.N + n] = acc;
  } else {
    const float y = __fmul_rn(__int2float_rn(acc), __fmul_rn(sx, sc));
    reinterpret_cast<__nv_bfloat16*>(p.out)[(size_t)m * p.N + n] = __float2bfloat16_rn(y);
  }
}

template <bool OUT_I32>
__device__ __forceinline__ void store_out(const GemmArgs& p, int m, int n, int32_t acc, float sc) {
  if constexpr (OUT_I32) {
    reinterpret_cast<int32_t*>(p.out)[(size_t)m * p.N + n] = acc;
  } else {
    const float scale = __fmul_rn(ld_dep(p.s_x + m), sc);
    const float y = __fmul_rn(__int2float_rn(acc), scale);
    reinterpret_cast<__nv_bfloat16*>(p.out)[(size_t)m * p.N + n] = __float2bfloat16_rn(y);
  }
}

// Reads CH accumulator columns [c0, c0+CH) of this warp's 32 TMEM lanes.
template <int CH>
__device__ __forceinline__ void tmem_load_cols(uint32_t taddr, uint32_t (&v)[32]) {
  if constexpr (CH == 16) {
    uint32_t v16[16];
    tmem_ld_32x32b_x16(taddr, v16);
    tmem_ld_wait();
#pragma unroll
    for (int i = 0; i < 16; ++i) v[i] = v16[i];
  } else {
    tmem_ld_32x32b_x32(taddr, v);
    tmem_ld_wait();
  }
}

// Reads W accumulator columns of this warp's 32 TMEM lanes and waits for them.
template <int W>
__device__ __forceinline__ void tmem_ld_cols(uint32_t taddr, uint32_t (&v)[W]) {
  static_assert(W == 2 || W == 4 || W == 8 || W == 16 || W == 32, "TMEM load width");
  if constexpr (W == 2) tmem_ld_32x32b_x2(taddr, v);
  if constexpr (W == 4) tmem_ld_32x32b_x4(taddr, v);
  if constexpr (W == 8) tmem_ld_32x32b_x8(taddr, v);
  if constexpr (W == 16) tmem_ld_32x32b_x16(taddr, v);
  if constexpr (W == 32) tmem_ld_32x32b_x32(taddr, v);
  tmem_ld_wait();
}

// CTAs that keep to 256 TMEM columns are meant to share an SM with a CTA of
// the next launch (programmatic dependent launch): registers are capped for two.
//
// FQ (fused activation quantization, 16-token tiles in a split-K cluster whose
// K-blocks all fit the preloaded stages): the activations arrive as bf16 and
// the expansion warps quantize them (per-token symmetric INT8, the same
// arithmetic as quantize_act_kernel) straight into the swizzled activation
// tiles; the row maxima are combined over the cluster through DSMEM.
//
// KIND 1 (W4 x FP8): the tensor maps carry e4m3 activations and the packed
// INT4 codes (no scale / offset tiles: tm_s and tm_a are never read); s_x is
// the tensor's one scale, s_c the channel scales s_w.
template <int BT, int CS, bool OUT_I32, bool FQ = false, int DQ = 0, int EG = 1, bool SWI = false, int KIND = 0>
__global__ void __launch_bounds__(gemm_threads(EG), GemmCfg<BT, CS, DQ>::kTmemCols == 256 ? 2 : 1)
    w4a8_gemm_kernel(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_x3,
                     const __grid_constant__ CUtensorMap tm_w, const __grid_constant__ CUtensorMap tm_s,
                     const __grid_constant__ CUtensorMap tm_a, const GemmArgs p) {
  using C = GemmCfg<BT, CS, DQ>;
  constexpr int kEG = EG;  // expansion groups of this variant
  static_assert(EG == 1 || (EG == 2 && !FQ && CS >= 1), "two expansion groups: cluster schedules, no fused quantization");
  static_assert(!SWI || (!OUT_I32 && !FQ && DQ == 0 && CS >= 1), "SwiGLU epilogue: bf16 output of cluster schedules");
  static_assert(!FQ || (BT == 16 && CS >= 2), "fused activation quantization: 16-token tiles, split-K clusters");
  static_assert(DQ == 0 || (!FQ && CS >= 1), "ablation variants: plain tile schedules only");
  static_assert(KIND == 0 || (KIND == 1 && !OUT_I32 && !FQ && DQ == 0 && !SWI && CS >= 1),
                "W4 x FP8: bf16 output of cluster schedules");
  constexpr bool F8 = (KIND == 1);
  // bytes a weight stage's loads complete (W4 x FP8 has no scale / offset tiles)
  constexpr uint32_t kTxW = F8 ? (uint32_t)C::kWBytes : C::kTxW;
  constexpr int S = C::kStages;
  constexpr int A = C::kSlots;
  // with as many TMEM slots as stages, block `it` uses stage and slot it % S:
  // one release (the slot's) frees both
  constexpr bool kJoint = (S == A);
  constexpr int CH = BT < 32 ? BT : 32;  // accumulator columns per TMEM load
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* xring = smem;                          // S x [BT][128] int8, SW128
  uint8_t* aring = smem + C::kXRing;              // explicit pipeline: A x [128][128] int8, SW128
  uint8_t* wring = aring + C::kASmem;             // S x ([128][64] packed, SW64 | s [2][128] | a [2][128])
  int32_t* red = reinterpret_cast<int32_t*>(wring + C::kWRing);  // [CS-1][BT][128]
  uint64_t* wfull = reinterpret_cast<uint64_t*>(wring + C::kWRing + C::kRedBytes);
  uint64_t* xfull = wfull + S;
  uint64_t* empty = xfull + S;
  uint64_t* afull = empty + S;    // [A]
  uint64_t* aempty = afull + A;   // [A]
  uint64_t* accfull = aempty + A;
  uint64_t* drain = accfull + 1;
  uint64_t* grp = drain + 1;
  uint64_t* redbar = grp + 1;
  uint64_t* xfirst = redbar + 1;  // the activation tiles of the first min(S, total) K-blocks, all at once
  uint64_t* amaxbar = xfirst + 1;  // FQ: the other CTAs' partial row maxima have landed
  uint64_t* ovfull = amaxbar + 1;  // the overflow K-block is expanded in shared memory
  uint64_t* drain2 = ovfull + 1;   // the second MMA issuer's MMAs have finished
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain2 + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  volatile int* last_flag = reinterpret_cast<volatile int*>(tmem_slot + 2);
  float* amx = reinterpret_cast<float*>(reinterpret_cast<uint8_t*>(wfull) + 512);  // FQ: [CS][16]
  float* sxs = amx + 8 * 16;                                                       // FQ: s_x [16]
  // blocks each expansion warp has reported ready (a hint for the MMA warp)
  volatile int* prog = reinterpret_cast<volatile int*>(reinterpret_cast<uint8_t*>(wfull) + 1088);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t crank = CS >= 2 ? cluster_ctarank() : 0u;

  // Grouped GEMM: this cluster's tile (token tile j over all groups, weight
  // tile tn of its group).  The row offsets may come from the preceding
  // kernel, so the dependency wait comes first.  Every warp finds the group
  // itself; a tile past the last group's rows leaves at once, before any
  // barrier, in every CTA of its cluster.
  int g_xrow = 0, g_mend = p.M, g_wrow = 0, g_scoff = 0;
  if (p.m_off != nullptr) {
    griddep_wait();
    const int t = (int)(blockIdx.x / (CS >= 1 ? CS : 1));
    const int j = t % p.tiles_m, tn = t / p.tiles_m;
    const int ge = find_group_tile(p.m_off, p.groups, p.M, BT, j, g_xrow, g_mend);
    if (ge < 0) return;
    g_wrow = ge * p.N + tn * kBlockN;
    g_scoff = ge * p.N;
  }
  const bool grouped = (p.m_off != nullptr);
  // first token row of token tile tm, first (stacked) weight row of weight tile tn
  auto xrow_of = [&](int tm) { return grouped ? g_xrow : tm * BT; };
  auto wrow_of = [&](int tn) { return grouped ? g_wrow : tn * kBlockN; };

  // this CTA's range of units (tile x K-block)
  const int KB = p.KB;
  long long u_begin, u_end;
  const long long U = p.U;
  const long long G = gridDim.x;
  // the tile and K-block of the first unit; a 64-bit division costs hundreds
  // of cycles, so cluster schedules (one tile per CTA) use 32-bit ones only
  int t_first, kb_first;
  if constexpr (CS >= 1) {
    t_first = (int)(blockIdx.x / CS);
    const int r = (int)(blockIdx.x % CS);
    kb_first = r * KB / CS;
    u_begin = (long long)t_first * KB + kb_first;
    u_end = (long long)t_first * KB + (r + 1) * KB / CS;
  } else {
    u_begin = (long long)blockIdx.x * U / G;
    u_end = ((long long)blockIdx.x + 1) * U / G;
    t_first = (int)(u_begin / KB);
    kb_first = (int)(u_begin - (long long)t_first * KB);
  }

  // the overflow K-block (see GemmCfg): one tile, exactly one block more than slots, no refills
  const bool ovf = !(DQ & 2) && CS >= 1 && A >= 2 && (int)(u_end - u_begin) == A + 1 && A + 1 <= S;

  // Two MMA issuers (decode): 16-token tiles whose K-blocks each have a TMEM
  // slot of their own (or the overflow block), so that no slot is reused and
  // nothing is refilled.  A single thread issues small-N MMAs at one per ~60
  // cycles; a second issuing warp overlaps with it.  The MMA warp takes the
  // even K-blocks into accumulator columns [0, 16), the producer warp, idle
  // once its loads are issued, the odd ones into [16, 32); the epilogue adds
  // the two.
  const int total_u = (int)(u_end - u_begin);
  const bool dual = BT == 16 && CS >= 1 && (DQ & 2) == 0 && total_u >= 2 && (total_u <= A || ovf);
  // Split-K clusters: whether this CTA's token slice holds any token of the tile
  // (the other CTAs send it partial sums only then).
  const int own_m0 = xrow_of(t_first % p.tiles_m);
  const bool own_valid = CS >= 2 && (int)crank * C::kT < min(BT, g_mend - own_m0);

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&wfull[s], 1);
      mbar_init(&xfull[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int s = 0; s < A; ++s) {
      mbar_init(&afull[s], 4);
      mbar_init(&aempty[s], 1);
    }
    mbar_init(accfull, dual ? 2 : 1);
    mbar_init(drain, 1);
    mbar_init(drain2, 1);
    mbar_init(grp, 4);
    // every CTA of a split-K cluster expects its piece from each of the others
    mbar_init(redbar, 1);
    if (CS >= 2) mbar_arrive_expect_tx(redbar, own_valid ? (uint32_t)C::kRedBytes : 0u);
    mbar_init(xfirst, FQ ? 4 : 1);  // FQ: the four quantizing warps
    mbar_init(amaxbar, 1);
    mbar_init(ovfull, 4);
    if (FQ) mbar_arrive_expect_tx(amaxbar, (uint32_t)(CS - 1) * 16 * 4);
    *abort_flag = 0;
    *last_flag = 0;
    for (int e = 0; e < 4 * kEG; ++e) prog[e] = 0;
    fence_mbar_init();
    if (!FQ) tma_prefetch_desc(CS >= 1 ? &tm_x3 : &tm_x);
    tma_prefetch_desc(&tm_w);
    if (!F8) {
      tma_prefetch_desc(&tm_s);
      tma_prefetch_desc(&tm_a);
    }
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, C::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  // The next kernel in the stream may launch now: its griddepcontrol.wait still
  // waits for this grid to complete, and meanwhile its CTAs, where they fit
  // beside this one, stream their weights.
  griddep_launch_dependents();
  // Cluster barrier, first half: this CTA's barriers are initialized.  The
  // second half is waited on only before a remote arrive (and at teardown).
  if constexpr (CS >= 2) cluster_arrive();
  bool cl_waited = false;


  // Producer and MMA warps run their loops with all 32 lanes (one lane issues),
  // so every warp stays converged up to the CTA barrier at teardown.
  const bool leader = (lane == 0);

  // The dual-issue form of the MMA loop (see `dual`): issuer i takes the
  // K-blocks b = i, i + 2, ... into accumulator columns [16 i, 16 i + 16).
  // Expansion finishes K-blocks in order, so a completed last block covers
  // every block before it; each slot is used once (phase 0).  Returns whether
  // this issuer has MMAs in flight (to be drained before TMEM is freed).
  auto dual_issue = [&](int i) -> bool {
    bool ok = true;
    if (leader) {
      constexpr uint32_t idesc = F8 ? idesc_f8(BT) : idesc_i8(BT);
      ok = mbar_wait(xfirst, 0, abort_flag);
      const int bl = ((total_u - 1 - i) & 1) ? total_u - 2 : total_u - 1;  // last block of this issuer
      if (ok && !(ovf && bl == A ? mbar_try_wait(smem_u32(ovfull), 0) : mbar_try_wait(smem_u32(&afull[bl]), 0)))
        for (int b = i; b <= bl && ok; b += 2)
          ok = (ovf && b == A) ? mbar_wait(ovfull, 0, abort_flag) : mbar_wait(&afull[b], 0, abort_flag);
      if (ok) {
        tc_fence_after();
        const uint32_t d = tmem_base + (uint32_t)(16 * i);
        for (int b = i; b < total_u; b += 2) {
          const uint64_t bdesc = smem_desc_k_sw128(smem_u32(xring + b * C::kXBytes));
          if (ovf && b == A) {
            // the overflow block: A from the weight stages it was expanded into
            const uint64_t adesc = smem_desc_k_sw128(smem_u32(wring));
#pragma unroll
            for (int j = 0; j < kBlockK / 32; ++j)
              mma_ss_k<F8>(d, adesc + (uint64_t)(2 * j), bdesc + (uint64_t)(2 * j), idesc, (b > i || j > 0) ? 1u : 0u);
          } else {
            const uint32_t a_col = tmem_base + C::kAccCols + b * 32;
#pragma unroll
            for (int j = 0; j < kBlockK / 32; ++j)
              mma_ts_k<F8>(d, a_col + j * 8, bdesc + (uint64_t)(2 * j), idesc, (b > i || j > 0) ? 1u : 0u);
          }
        }
        tc_commit(accfull);
      }
    }
    return __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
  };
  // waits (bounded) until this thread's issued MMAs have finished
  auto drain_mmas = [&](uint64_t* bar) {
    tc_commit(bar);
    const uint32_t a = smem_u32(bar);
    const unsigned long long t0w = globaltimer();
    while (!mbar_try_wait(a, 0) && globaltimer() - t0w < 100000000ull) {
    }
  };
  if (warp == 0) {
    // ------------------------------------------------------------ producer
    // Weight tiles depend on nothing the preceding kernel writes: the first
    // S of them are requested before griddepcontrol.wait; activation tiles
    // after it.  Weights and activations complete on separate barriers, so
    // the expansion never waits for activations.
    uint64_t pol_stream = 0, pol_keep = 0;
    if (leader) {
      pol_stream = l2_policy_evict_first();  // weights: read once
      pol_keep = l2_policy_evict_last();     // activations: re-read per weight tile
    }
    const int total = (int)(u_end - u_begin);
    const int P = min(S, total);
    const UnitCursor first = UnitCursor::at(t_first, kb_first, p.tiles_m);
    UnitCursor cw = first;  // after the prefetch: the unit of K-block P (every lane steps it)
    // first P K-blocks (they may span tiles in the stream-K schedule)
    for (int i = 0; i < P; ++i, cw.next(KB, p.tiles_m)) {
      if (leader) {
        uint8_t* wb = wring + i * C::kWStage;
        mbar_arrive_expect_tx(&wfull[i], kTxW);
        const int wr = wrow_of(cw.tile_n);
        tma_load_2d(wb, &tm_w, &wfull[i], cw.kb * (kBlockK / 2), wr, pol_stream);
        if (!F8) {
          tma_load_2d(wb + C::kWBytes, &tm_s, &wfull[i], wr, cw.kb * 2, pol_stream);
          tma_load_2d(wb + C::kWBytes + C::kSABytes, &tm_a, &wfull[i], wr, cw.kb * 2, pol_stream);
        }
      }
    }
    griddep_wait();
    if (leader && P > 0 && !FQ) {
      // one barrier for all of them: the MMA warp waits once
      if constexpr (CS >= 1) {
        // a cluster CTA's K-blocks are consecutive blocks of one tile: the first
        // S of them in one 3D box [block][token][128 bytes], which is the ring's
        // layout (blocks past the CTA's slice are loaded and not used; blocks
        // past K read as zero)
        mbar_arrive_expect_tx(xfirst, (uint32_t)S * C::kTxX);
        tma_load_3d(xring, &tm_x3, xfirst, 0, xrow_of(first.tile_m), first.kb, pol_keep);
      } else {
        mbar_arrive_expect_tx(xfirst, (uint32_t)P * C::kTxX);
        UnitCursor cx = first;
        for (int i = 0; i < P; ++i, cx.next(KB, p.tiles_m))
          tma_load_2d(xring + i * C::kXBytes, &tm_x, xfirst, cx.kb * kBlockK, xrow_of(cx.tile_m), pol_keep);
      }
    }
    __syncwarp();
    // xfull[s] serves the refills of stage s only: its k-th phase is the (k+1)-th use of the stage
    uint32_t issued = 0, issued_par = 0;
    {
      int stage = P % S;
      uint32_t phase = (uint32_t)(P / S) & 1u;
      for (int it = P; it < total; ++it, cw.next(KB, p.tiles_m)) {
        if (!lane0_wait(kJoint ? &aempty[stage] : &empty[stage], phase ^ 1u, abort_flag)) goto producer_done;
        if (leader) {
          const int kb = cw.kb, tile_m = cw.tile_m, tile_n = cw.tile_n;
          uint8_t* wb = wring + stage * C::kWStage;
          mbar_arrive_expect_tx(&wfull[stage], kTxW);
          const int wr = wrow_of(tile_n);
          tma_load_2d(wb, &tm_w, &wfull[stage], kb * (kBlockK / 2), wr, pol_stream);
          if (!F8) {
            tma_load_2d(wb + C::kWBytes, &tm_s, &wfull[stage], wr, kb * 2, pol_stream);
            tma_load_2d(wb + C::kWBytes + C::kSABytes, &tm_a, &wfull[stage], wr, kb * 2, pol_stream);
          }
          mbar_arrive_expect_tx(&xfull[stage], C::kTxX);
          tma_load_2d(xring + stage * C::kXBytes, &tm_x, &xfull[stage], kb * kBlockK, xrow_of(tile_m), pol_keep);
        }
        issued |= 1u << stage;
        issued_par = (issued_par & ~(1u << stage)) | ((phase ^ 1u) << stage);
        if (++stage == S) {
          stage = 0;
          phase ^= 1u;
        }
      }
    }
  producer_done:
    if (leader && *abort_flag) {
      // never leave a bulk copy in flight into shared memory that is about to be released
      const unsigned long long t0w = globaltimer();
      if (P > 0 && !FQ)
        while (!mbar_try_wait(smem_u32(xfirst), 0) && globaltimer() - t0w < 100000000ull) {
        }
      for (int s = 0; s < S; ++s) {
        // the last weight load into stage s: use (issued ? refill : first)
        if (s < P)
          while (!mbar_try_wait(smem_u32(&wfull[s]), ((issued >> s) & 1u) ? (((issued_par >> s) & 1u) ^ 1u) : 0u) &&
                 globaltimer() - t0w < 100000000ull) {
          }
        if (issued & (1u << s))
          while (!mbar_try_wait(smem_u32(&xfull[s]), (issued_par >> s) & 1u) && globaltimer() - t0w < 100000000ull) {
          }
      }
    }
    if (dual && dual_issue(1) && leader) drain_mmas(drain2);
  } else if (warp == 1 && dual) {
    // ------------------------------------------- MMA issuer (dual form)
    if (dual_issue(0) && leader) drain_mmas(drain);
  } else if (warp == 1) {
    // ---------------------------------------------------------- MMA issuer
    constexpr uint32_t idesc = F8 ? idesc_f8(BT) : idesc_i8(BT);
    // A wait costs about as much as a K-block of small MMAs, so the loop waits
    // as little as it can: once for all the preloaded activation tiles; the
    // activation tiles of later blocks are waited for by the expansion warps,
    // so that a completed slot means a block ready in full; expansion
    // finishes K-blocks in order, so a completed later block covers every
    // block before it.  Stages and slots are released only when a later
    // K-block will reuse them.
    const int total = (int)(u_end - u_begin);
    const int P = min(S, total);
    bool any = false, x_first_seen = false;
    int it = 0, ready = 0;  // K-blocks [0, ready) are known to be expanded
    for (long long u = u_begin; u < u_end;) {
      const int kb0 = u == u_begin ? kb_first : (int)(u % KB);
      const int kb1 = (int)min((long long)KB, kb0 + (u_end - u));
      for (int kb = kb0; kb < kb1;) {
        bool ok = true;
        int run = 1;  // K-blocks from `it` on that need no further wait
        if (leader) {
          const int slot = it % A;
          if (!x_first_seen) ok = mbar_wait(xfirst, 0, abort_flag);
          x_first_seen = true;
          if (ok && it >= ready) {
            // The expansion usually runs ahead.  Every expansion warp reports
            // the blocks it has handed over; the slowest report names the
            // furthest block that is likely complete, and one look at its slot
            // (whose previous block this warp has consumed: at most A - 1
            // ahead) covers every block before it.
            int rep_ = prog[0];
#pragma unroll
            for (int e = 1; e < 4 * kEG; ++e) rep_ = min(rep_, prog[e]);
            const int hi = min(min(rep_ - 1, it + A - 1), total - 1);
            // each group expands its blocks in order: its latest block covers
            // its earlier ones, so one look per group (blocks hi and hi - 1)
            if (hi > it && (!ovf || hi < A) && mbar_try_wait(smem_u32(&afull[hi % A]), (uint32_t)(hi / A) & 1u) &&
                (kEG == 1 ||
                 mbar_try_wait(smem_u32(&afull[(hi - 1) % A]), (uint32_t)((hi - 1) / A) & 1u))) {
              ready = hi + 1;
            } else {
              ok = (ovf && it == A) ? mbar_wait(ovfull, 0, abort_flag)
                                    : mbar_wait(&afull[slot], (uint32_t)(it / A) & 1u, abort_flag);
              ready = it + 1;
            }
            if (ok && ovf && ready == A && mbar_try_wait(smem_u32(ovfull), 0)) ready = A + 1;
          }
          run = min(ready - it, kb1 - kb);
        }
        run = __shfl_sync(0xffffffffu, ok ? run : 0, 0);
        if (run <= 0) goto mma_done;
        if (leader) {
          // the whole run back to back, one thread, no warp synchronization
          tc_fence_after();
          int stage = it % S, slot = it % A;
          // K-blocks whose stage (and slot) a later block reuses need release
          // commits, those whose slot only is reused need one, the rest none:
          // three loops, so that the last is a plain run of MMAs (measurably
          // faster to issue than one loop with the conditions inside)
          // the overflow block, if this run reaches it, goes last and separately
          const bool run_ovf = ovf && it + run == A + 1;
          const int run_ts = run - (run_ovf ? 1 : 0);
          const int r_both = min(run_ts, max(0, total - S - it));
          const int r_slot = min(run_ts, max(0, total - A - it));
          auto issue = [&](int r) {
            const uint64_t bdesc = smem_desc_k_sw128(smem_u32(xring + stage * C::kXBytes));
            if constexpr ((DQ & 2) != 0) {
              const uint64_t adesc = smem_desc_k_sw128(smem_u32(aring + slot * (kBlockN * kBlockK)));
#pragma unroll
              for (int j = 0; j < kBlockK / 32; ++j)
                mma_ss_k<F8>(tmem_base, adesc + (uint64_t)(2 * j), bdesc + (uint64_t)(2 * j), idesc,
                             (kb + r > kb0 || j > 0) ? 1u : 0u);
            } else {
              const uint32_t a_col = tmem_base + C::kAccCols + slot * 32;
#pragma unroll
              for (int j = 0; j < kBlockK / 32; ++j)
                mma_ts_k<F8>(tmem_base, a_col + j * 8, bdesc + (uint64_t)(2 * j), idesc,
                             (kb + r > kb0 || j > 0) ? 1u : 0u);
            }
          };
          int r = 0;
          for (; r < r_both; ++r) {
            issue(r);
            if constexpr (!kJoint) tc_commit(&empty[stage]);
            tc_commit(&aempty[slot]);
            if (++stage == S) stage = 0;
            if (++slot == A) slot = 0;
          }
          for (; r < r_slot; ++r) {
            issue(r);
            tc_commit(&aempty[slot]);
            if (++stage == S) stage = 0;
            if (++slot == A) slot = 0;
          }
          for (; r < run_ts; ++r) {
            issue(r);
            if (++stage == S) stage = 0;
            if (++slot == A) slot = 0;
          }
          if (run_ovf) {
            const uint64_t adesc = smem_desc_k_sw128(smem_u32(wring));
            const uint64_t bdesc = smem_desc_k_sw128(smem_u32(xring + stage * C::kXBytes));
#pragma unroll
            for (int j = 0; j < kBlockK / 32; ++j)
              mma_ss_k<F8>(tmem_base, adesc + (uint64_t)(2 * j), bdesc + (uint64_t)(2 * j), idesc, 1u);
          }
        }
        it += run;
        kb += run;
        any = true;
      }
      if (leader) tc_commit(accfull);
      __syncwarp();
      u += kb1 - kb0;
    }
  mma_done:
    if (leader && any) {
      // all issued MMAs have finished before TMEM is released
      tc_commit(drain);
      const uint32_t a = smem_u32(drain);
      const unsigned long long t0w = globaltimer();
      while (!mbar_try_wait(a, 0) && globaltimer() - t0w < 100000000ull) {
      }
    }
  } else {
    // ------------------------------------------- expansion + epilogue warps
    const int sub = warp & 3;           // TMEM sub-partition this warp may access
    const int egrp = (warp - 2) >> 2;   // expansion group: takes the K-blocks it_e with it_e % kEG == egrp
    const int r = sub * 32 + lane;      // weight row of the tile = TMEM lane
    const uint32_t t_lane = tmem_base + ((uint32_t)(sub * 32) << 16);
    const int sw = (r >> 1) & 3;        // 64-byte swizzle of this row's 16-byte chunks
    uint32_t acc_phase = 0, grp_phase = 0;
    bool waited_dep = false;
    // split-K: every epilogue warp reads this CTA's piece, so each must see all
    // of it arrive before the CTA may leave (the others' bulk copies write here)
    bool red_done = (CS < 2) || egrp != 0;  // group 0 runs the epilogue
    bool staged = false;  // this thread issued bulk copies from the staging rows
    int stage = 0, slot = 0;
    uint32_t sphase = 0, aphase = 0;

    // ------------------------------------------ fused activation quantization
    // (FQ) Quantizes this CTA's K-slice of the tile's activations into the
    // activation tiles.  Warp e = warp - 2 takes tokens e, e+4, e+8, e+12 (a
    // small batch spreads over all four warps; the cluster's partial maxima
    // are kept per warp, amx[src][4e + i] for token e + 4i), lane l the
    // 32 consecutive K of chunk l (a 128-K block is four chunks; the slice has
    // at most S blocks, so one chunk per lane at most).  Runs once the weight
    // blocks that have a slot of their own are expanded: the next block
    // waits for an MMA, and the MMAs wait for this.
    const int total_e = (int)(u_end - u_begin);
    bool x_done = !FQ || egrp != 0;
    auto fused_quantize = [&]() -> bool {
      x_done = true;
      griddep_wait();  // X may be the output of the preceding kernel
      waited_dep = true;
      cluster_wait();  // the other CTAs' barriers exist before any remote store
      cl_waited = true;
      const int e = warp - 2;
      const int nchunk = total_e * (kBlockK / 32);
      const int k0 = kb_first * kBlockK + lane * 32;  // this lane's first K
      const bool has = lane < nchunk;
      // the four tokens are independent: all loads first, then the reductions
      // and divisions side by side, so that no chain waits on another
      uint4 xv[4][4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int m = e + 4 * i;
        const bool ld = has && m < p.M;
        const uint4* src = reinterpret_cast<const uint4*>(p.x_bf16 + (size_t)(ld ? m : 0) * p.K + (ld ? k0 : 0));
#pragma unroll
        for (int c = 0; c < 4; ++c) xv[i][c] = ld ? ld_dep(src + c) : make_uint4(0u, 0u, 0u, 0u);
      }
      float pm[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        // max |x| on bf16 pairs: bf16 -> fp32 is exact and monotone, so the
        // maximum is the same as over the fp32 values
        __nv_bfloat162 m2 = __floats2bfloat162_rn(0.0f, 0.0f);
        if (e + 4 * i < p.M) {
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            const uint32_t w4[4] = {xv[i][c].x, xv[i][c].y, xv[i][c].z, xv[i][c].w};
#pragma unroll
            for (int j = 0; j < 4; ++j)
              m2 = __hmax2(m2, __habs2(*reinterpret_cast<const __nv_bfloat162*>(&w4[j])));
          }
        }
        const uint32_t mb = *reinterpret_cast<const uint32_t*>(&m2);
        pm[i] = fmaxf(bf16_bits_to_f32(mb & 0xFFFFu), bf16_bits_to_f32(mb >> 16));
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1)
#pragma unroll
        for (int i = 0; i < 4; ++i) pm[i] = fmaxf(pm[i], __shfl_xor_sync(0xffffffffu, pm[i], o));
      // pm[i]: this CTA's maximum of |X[4e + i, slice]|.  Partial maxima to the
      // other CTAs of the cluster (16 bytes each, counted on their barrier)
      // and to this CTA's own row.
      if (lane == 0) {
        *reinterpret_cast<float4*>(amx + crank * 16 + 4 * e) = make_float4(pm[0], pm[1], pm[2], pm[3]);
#pragma unroll
        for (int o = 0; o < CS; ++o)
          if (o != (int)crank)
            st_async_v4(mapa_shared(smem_u32(amx + crank * 16 + 4 * e), (uint32_t)o), __float_as_uint(pm[0]),
                        __float_as_uint(pm[1]), __float_as_uint(pm[2]), __float_as_uint(pm[3]),
                        mapa_shared(smem_u32(amaxbar), (uint32_t)o));
      }
      if (!__all_sync(0xffffffffu, mbar_wait_cluster(amaxbar, 0, abort_flag))) return false;
      // lane i < 4 finishes token 4e + i (row maximum over the cluster, the two
      // IEEE divisions) and hands 127/amax to the warp
      float inv_l = 0.0f;
      if (lane < 4) {
        const int m = e + 4 * lane;
        float a = lane == 0 ? pm[0] : lane == 1 ? pm[1] : lane == 2 ? pm[2] : pm[3];
#pragma unroll
        for (int o = 0; o < CS; ++o)
          if (o != (int)crank) a = fmaxf(a, amx[o * 16 + 4 * e + lane]);
        const bool zero = (a == 0.0f);
        inv_l = zero ? 0.0f : __fdiv_rn(127.0f, a);
        sxs[m] = zero ? 1.0f : __fdiv_rn(a, 127.0f);
      }
      float inv[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) inv[i] = __shfl_sync(0xffffffffu, inv_l, i);
      if (has) {
        // lane l: 32 codes of each token = two 16-byte chunks of its row in
        // block l / 4 (128-byte swizzle)
        uint8_t* blk = xring + (size_t)(lane >> 2) * C::kXBytes;
        const int ch = (lane & 3) * 2;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int m = e + 4 * i;
          uint32_t q[8] = {0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u};  // rows past the batch stay zero
          if (m < p.M) {
#pragma unroll
            for (int c = 0; c < 4; ++c) {
              q[2 * c] = quant_quad_i8(xv[i][c].x, xv[i][c].y, inv[i]);
              q[2 * c + 1] = quant_quad_i8(xv[i][c].z, xv[i][c].w, inv[i]);
            }
          }
          uint8_t* row = blk + m * 128;
          *reinterpret_cast<uint4*>(row + ((ch ^ (m & 7)) << 4)) = make_uint4(q[0], q[1], q[2], q[3]);
          *reinterpret_cast<uint4*>(row + (((ch + 1) ^ (m & 7)) << 4)) = make_uint4(q[4], q[5], q[6], q[7]);
        }
      }
      // the tensor core reads these tiles through the async proxy
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(xfirst);
      return true;
    };
    int it_e = 0;
    const int P_e = min(S, total_e);  // blocks from P_e on are refills of a stage
    // the first block that waits for an MMA (or the end; with the overflow
    // block in shared memory no block does)
    const int x_at = ovf ? total_e : min(A, total_e);

    for (long long u = u_begin; u < u_end;) {
      const int t = u == u_begin ? t_first : (int)(u / KB);
      const int kb0 = u == u_begin ? kb_first : (int)(u % KB);
      const int kb1 = (int)min((long long)KB, kb0 + (u_end - u));
      const int tile_m = t % p.tiles_m, tile_n = t / p.tiles_m;
      for (int kb = kb0; kb < kb1; ++kb, ++it_e) {
        if constexpr (FQ) {
          if (egrp == 0 && it_e == x_at && !fused_quantize()) goto epi_done;
        }
        if (it_e % kEG != egrp) {  // another group's block
          if (++stage == S) {
            stage = 0;
            sphase ^= 1u;
          }
          if (++slot == A) {
            slot = 0;
            aphase ^= 1u;
          }
          continue;
        }
        // the overflow block goes to shared memory: it needs weight stages 0-1,
        // which every warp has finished reading once blocks 0 and 1 are expanded
        const bool to_smem = ovf && it_e == A;
        // warp-uniform decision: every lane waits, all continue only if all saw the phase
        if (!__all_sync(0xffffffffu, mbar_wait(&wfull[stage], sphase, abort_flag) &&
                                         (to_smem ? mbar_wait(&afull[0], 0, abort_flag) &&
                                                        mbar_wait(&afull[1], 0, abort_flag)
                                                  : mbar_wait(&aempty[slot], aphase ^ 1u, abort_flag))))
          goto epi_done;
        tc_fence_after();
        const uint8_t* wb = wring + stage * C::kWStage;
        const uint32_t wrow = smem_u32(wb) + r * (kBlockK / 2);
        uint32_t v[32];
        if constexpr (F8) {
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            const uint4 q = lds128(wrow + ((c ^ sw) << 4));
            w4_word_to_e4m3(q.x, v[8 * c + 0], v[8 * c + 1]);
            w4_word_to_e4m3(q.y, v[8 * c + 2], v[8 * c + 3]);
            w4_word_to_e4m3(q.z, v[8 * c + 4], v[8 * c + 5]);
            w4_word_to_e4m3(q.w, v[8 * c + 6], v[8 * c + 7]);
          }
        } else {
          const uint8_t* ss = wb + C::kWBytes;
          const uint8_t* sa = ss + C::kSABytes;
          const uint32_t s0 = ss[r], s1 = ss[kBlockN + r];
          const uint32_t a0 = (uint32_t)sa[r] * 0x01010101u, a1 = (uint32_t)sa[kBlockN + r] * 0x01010101u;
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            const uint4 q = lds128(wrow + ((c ^ sw) << 4));
            const uint32_t s = c < 2 ? s0 : s1;
            const uint32_t a4 = c < 2 ? a0 : a1;
            if constexpr ((DQ & 1) != 0) {
              naive_expand_word(q.x, s, a4 & 0xFFu, v[8 * c + 0], v[8 * c + 1]);
              naive_expand_word(q.y, s, a4 & 0xFFu, v[8 * c + 2], v[8 * c + 3]);
              naive_expand_word(q.z, s, a4 & 0xFFu, v[8 * c + 4], v[8 * c + 5]);
              naive_expand_word(q.w, s, a4 & 0xFFu, v[8 * c + 6], v[8 * c + 7]);
            } else {
              lqq_expand_word(q.x, s, a4, v[8 * c + 0], v[8 * c + 1]);
              lqq_expand_word(q.y, s, a4, v[8 * c + 2], v[8 * c + 3]);
              lqq_expand_word(q.z, s, a4, v[8 * c + 4], v[8 * c + 5]);
              lqq_expand_word(q.w, s, a4, v[8 * c + 6], v[8 * c + 7]);
            }
          }
        }
        if (to_smem) {
          // row r of a 128-byte-swizzled K-major tile (the MMA's A descriptor)
          uint8_t* orow = wring + r * 128;
#pragma unroll
          for (int c = 0; c < 8; ++c)
            *reinterpret_cast<uint4*>(orow + ((c ^ (r & 7)) << 4)) = make_uint4(v[4 * c], v[4 * c + 1], v[4 * c + 2], v[4 * c + 3]);
          fence_proxy_async_smem();  // read by the tensor core through the async proxy
          __syncwarp();
          if (lane == 0) mbar_arrive(ovfull);
        } else {
          if constexpr ((DQ & 2) != 0) {
            // explicit pipeline: row r of the slot's 128-byte-swizzled A tile
            uint8_t* orow = aring + slot * (kBlockN * kBlockK) + r * 128;
#pragma unroll
            for (int c = 0; c < 8; ++c)
              *reinterpret_cast<uint4*>(orow + ((c ^ (r & 7)) << 4)) = make_uint4(v[4 * c], v[4 * c + 1], v[4 * c + 2], v[4 * c + 3]);
            fence_proxy_async_smem();  // read by the tensor core through the async proxy
          } else {
            tmem_st_32x32b_x32(t_lane + C::kAccCols + slot * 32, v);
            tmem_st_wait();
          }
          tc_fence_before();
          // a refilled block's activation tile: one warp sees it land before
          // the slot is reported ready (the MMA warp waits for the slot only)
          bool x_ok = true;
          if (sub == 2 && it_e >= P_e && lane == 0)  // the group's first warp
            x_ok = mbar_wait(&xfull[stage], (uint32_t)(it_e / S - 1) & 1u, abort_flag);
          __syncwarp();
          if (lane == 0 && x_ok) {
            mbar_arrive(&afull[slot]);
            prog[warp - 2] = it_e + 1;
          }
          if (!__shfl_sync(0xffffffffu, x_ok ? 1 : 0, 0)) goto epi_done;
        }
        if (++stage == S) {
          stage = 0;
          sphase ^= 1u;
        }
        if (++slot == A) {
          slot = 0;
          aphase ^= 1u;
        }
      }

      if constexpr (FQ) {
        if (!x_done && !fused_quantize()) goto epi_done;
      }
      if (egrp != 0) {  // the other expansion groups have no epilogue
        u += kb1 - kb0;
        continue;
      }
      // ------------------------------------------------------- epilogue
      if (!waited_dep) {
        griddep_wait();  // scales and the output may belong to the preceding kernel
        waited_dep = true;
      }
      // scales of this tile, loaded before the accumulator is ready: s_c of this
      // thread's row, s_x of token m0 + lane of the first column chunk
      const int n = tile_n * kBlockN + r;  // output column (within the group)
      const int m0 = xrow_of(tile_m);
      const int mend = g_mend;             // rows from here on are not this tile's
      const bool n_ok = n < p.N;
      const float sc = (!OUT_I32 && n_ok) ? __ldg(p.s_c + g_scoff + n) : 0.0f;
      // token scales, lane-distributed (token i of the chunk: lane i): direct
      // epilogues take the tile's tokens from m0, split-K clusters this CTA's
      // token slice from m0 + crank kT (registers j: tokens 32 j + lane)
      constexpr int SXC = CS >= 2 ? (C::kT < 32 ? C::kT : 32) : CH;
      constexpr int kSxRegs = CS >= 2 ? (C::kT + 31) / 32 : 1;
      const int sx0 = m0 + (CS >= 2 ? (int)crank * C::kT : 0);
      float sx_next = 0.0f;
      float sxr[kSxRegs];
#pragma unroll
      for (int j = 0; j < kSxRegs; ++j) sxr[j] = 0.0f;
      if constexpr (FQ) {
        // s_x from the quantizing warps (all four have arrived on xfirst)
        if (!__all_sync(0xffffffffu, mbar_wait(xfirst, 0, abort_flag))) goto epi_done;
      }
      if constexpr (!OUT_I32) {
        // W4 x FP8: one activation scale for the tensor
        auto sx_at = [&](int m) { return FQ ? sxs[m - m0] : ld_dep(p.s_x + (F8 ? 0 : m)); };
        if constexpr (CS >= 2) {
#pragma unroll
          for (int j = 0; j < kSxRegs; ++j) {
            const int i = 32 * j + lane;
            sxr[j] = (i < C::kT && sx0 + i < mend) ? sx_at(sx0 + i) : 0.0f;
          }
        } else {
          sx_next = (lane < SXC && sx0 + lane < mend) ? sx_at(sx0 + lane) : 0.0f;
        }
      }
      if (!__all_sync(0xffffffffu, mbar_wait(accfull, acc_phase, abort_flag))) goto epi_done;
      acc_phase ^= 1u;
      tc_fence_after();
      {
        const bool whole = (kb0 == 0 && kb1 == KB);
        if constexpr (CS >= 2) {
          // ------------------- cluster split-K: reduce-scatter over token slices
          // 1. the other CTAs' slices of this thread's row go straight from TMEM
          //    to their shared memory (st.async, counted on their redbar);
          // 2. this CTA's slice: its own partial sums plus the received ones,
          //    scaled and stored.
          constexpr int T = C::kT;
          constexpr int TCH = T < 32 ? T : 32;  // TMEM columns per load
          const int mvalid = min(BT, mend - m0);
          // the other CTAs' barriers are initialized once the whole cluster has arrived
          if (!cl_waited) {
            cluster_wait();
            cl_waited = true;
          }
          // Slice layout [source slot][row][T] int32; its 16-byte chunks are
          // rotated by the row (chunk q at q ^ (row mod T/4)) so that the
          // owner's 16-byte reads of consecutive rows fall in different banks.
          auto red_off = [&](int slot, int q4) -> int {  // int32 offset of chunk q4 (4 values) of row r
            constexpr int kC = T / 4;
            const int q = kC >= 2 ? (q4 ^ (r & (kC - 1))) : q4;
            return (slot * kBlockN + r) * T + 4 * q;
          };
          auto send = [&](int o, int c0, const uint32_t* v) {  // columns [c0, c0 + TCH) of slice o
            const int slot = (int)crank < o ? (int)crank : (int)crank - 1;
            const uint32_t bar = mapa_shared(smem_u32(redbar), (uint32_t)o);
            if constexpr (T == 2) {
              st_async_v2(mapa_shared(smem_u32(red + (slot * kBlockN + r) * 2), (uint32_t)o), v[0], v[1], bar);
            } else {
#pragma unroll
              for (int q = 0; q < TCH; q += 4)
                st_async_v4(mapa_shared(smem_u32(red + red_off(slot, (c0 + q) / 4)), (uint32_t)o), v[q], v[q + 1],
                            v[q + 2], v[q + 3], bar);
            }
          };
          uint32_t own16[BT == 16 ? T : 1];  // 16-token tiles: this CTA's slice, kept from the one load
          if constexpr (BT == 16) {
            uint32_t v[16];
            if (dual) {
              uint32_t w[32];
              tmem_ld_32x32b_x32(t_lane, w);
              tmem_ld_wait();
#pragma unroll
              for (int i = 0; i < 16; ++i) v[i] = acc_add<F8>(w[i], w[16 + i]);
            } else {
              tmem_ld_32x32b_x16(t_lane, v);
              tmem_ld_wait();
            }
#pragma unroll
            for (int o = 0; o < CS; ++o) {
              if (o == (int)crank) {
#pragma unroll
                for (int i = 0; i < T; ++i) own16[i] = v[o * T + i];
              } else if (o * T < mvalid) {
                send(o, 0, v + o * T);
              }
            }
          } else if constexpr ((CS - 1) * T <= 32) {
#pragma unroll
            for (int o = 0; o < CS; ++o) {
              if (o == (int)crank || o * T >= mvalid) continue;
#pragma unroll 1
              for (int c0 = 0; c0 < T; c0 += TCH) {
                uint32_t v[TCH];
                tmem_ld_cols<TCH>(t_lane + (uint32_t)(o * T + c0), v);
                send(o, c0, v);
              }
            }
          } else {
            // Large slices: per-thread remote stores would be thousands of
            // 16-byte messages, so each warp stages its 32 rows of every other
            // owner's slice in the free activation ring ([owner][row][T], the
            // receive layout) and sends each with one bulk copy.
            int32_t* stg = reinterpret_cast<int32_t*>(xring);
#pragma unroll
            for (int o = 0; o < CS; ++o) {
              if (o == (int)crank || o * T >= mvalid) continue;
#pragma unroll 1
              for (int c0 = 0; c0 < T; c0 += TCH) {
                uint32_t v[TCH];
                tmem_ld_cols<TCH>(t_lane + (uint32_t)(o * T + c0), v);
#pragma unroll
                for (int q = 0; q < TCH; q += 4)
                  *reinterpret_cast<uint4*>(stg + o * kBlockN * T + red_off(0, (c0 + q) / 4)) =
                      make_uint4(v[q], v[q + 1], v[q + 2], v[q + 3]);
              }
            }
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) {
#pragma unroll 1
              for (int o = 0; o < CS; ++o) {
                if (o == (int)crank || o * T >= mvalid) continue;
                const int slot = (int)crank < o ? (int)crank : (int)crank - 1;
                bulk_copy_s2s(mapa_shared(smem_u32(red + (slot * kBlockN + sub * 32) * T), (uint32_t)o),
                              stg + (o * kBlockN + sub * 32) * T, (uint32_t)(32 * T * 4),
                              mapa_shared(smem_u32(redbar), (uint32_t)o));
                staged = true;
              }
              bulk_commit();
            }
          }
          if (own_valid) {
            // every lane observes the completed bytes itself (cluster-scope acquire)
            if (!__all_sync(0xffffffffu, mbar_wait_cluster(redbar, 0, abort_flag))) goto epi_done;
          }
          red_done = true;
          if (own_valid) {
#pragma unroll 1
            for (int c0 = 0; c0 < T; c0 += TCH) {
              uint32_t acc[TCH];
              if constexpr (BT == 16) {
#pragma unroll
                for (int i = 0; i < TCH; ++i) acc[i] = own16[i];
              } else {
                tmem_ld_cols<TCH>(t_lane + (uint32_t)((int)crank * T + c0), acc);
              }
#pragma unroll
              for (int sidx = 0; sidx < CS - 1; ++sidx) {
                if constexpr (T == 2) {
                  const uint2 w2 = *reinterpret_cast<const uint2*>(red + (sidx * kBlockN + r) * 2);
                  acc[0] = acc_add<F8>(acc[0], w2.x);
                  acc[1] = acc_add<F8>(acc[1], w2.y);
                } else {
#pragma unroll
                  for (int q = 0; q < TCH; q += 4) {
                    const uint4 w4 = *reinterpret_cast<const uint4*>(red + red_off(sidx, (c0 + q) / 4));
                    acc[q] = acc_add<F8>(acc[q], w4.x);
                    acc[q + 1] = acc_add<F8>(acc[q + 1], w4.y);
                    acc[q + 2] = acc_add<F8>(acc[q + 2], w4.z);
                    acc[q + 3] = acc_add<F8>(acc[q + 3], w4.w);
                  }
                }
              }
              const float sx_chunk = (kSxRegs > 1 && c0 >= 32) ? sxr[kSxRegs - 1] : sxr[0];  // tokens c0 .. c0 + 31
              if constexpr (SWI) {
                store_chunk_swiglu<TCH>(p, sx0 + c0, mend, n, n_ok, acc, sx_chunk, sc);
              } else {
#pragma unroll
                for (int i = 0; i < TCH; ++i) {
                  const int ti = c0 + i;  // token of the slice
                  const int m = sx0 + ti;
                  float sxm = 0.0f;
                  if constexpr (!OUT_I32) sxm = __shfl_sync(0xffffffffu, sx_chunk, i);
                  if (m < mend && n_ok) {
                    if constexpr (OUT_I32) {
                      reinterpret_cast<int32_t*>(p.out)[(size_t)m * p.N + n] = (int32_t)acc[i];
                    } else {
                      const float y = __fmul_rn(acc_f32<F8>(acc[i]), __fmul_rn(sxm, sc));
                      reinterpret_cast<__nv_bfloat16*>(p.out)[(size_t)m * p.N + n] = __float2bfloat16_rn(y);
                    }
                  }
                }
              }
            }
          }
          // the staging rows are read by the bulk copies before this CTA may leave
          if (staged) bulk_wait_read();
          tc_fence_before();
        } else {
          int32_t* ws_tile = p.ws + (size_t)t * BT * kBlockN;
#pragma unroll 1
          for (int cc = 0; cc < BT / CH; ++cc) {
            const float sx_cur = sx_next;
            if (cc + 1 < BT / CH)
              sx_next = (!OUT_I32 && m0 + (cc + 1) * CH + lane < mend)
                            ? ld_dep(p.s_x + (F8 ? 0 : m0 + (cc + 1) * CH + lane))
                            : 0.0f;
            uint32_t v[32];
            if (dual) {
              // 16-token tile, two issuers: the sum of accumulator columns [0, 16) and [16, 32)
              tmem_ld_32x32b_x32(t_lane, v);
              tmem_ld_wait();
#pragma unroll
              for (int i = 0; i < 16; ++i) v[i] = acc_add<F8>(v[i], v[16 + i]);
            } else {
              tmem_load_cols<CH>(t_lane + cc * CH, v);
            }
            if (whole) {
              if constexpr (SWI)
                store_chunk_swiglu<CH>(p, m0 + cc * CH, mend, n, n_ok, v, sx_cur, sc);
              else
                store_chunk<OUT_I32, CH, F8>(p, m0 + cc * CH, mend, n, n_ok, v, sx_cur, sc);
            } else {
#pragma unroll
              for (int i = 0; i < CH; ++i) {
                const int ml = cc * CH + i;
                if (m0 + ml < p.M) atomicAdd(ws_tile + ml * kBlockN + r, (int32_t)v[i]);
              }
            }
          }
          tc_fence_before();
          if (CS == 0 && !whole) {
            // ------------------------------------- stream-K: last arriver finishes
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
              const int mrows = min(BT, p.M - m0);
#pragma unroll 1
              for (int mb = 0; mb < mrows; mb += 16) {
                int32_t vals[16];
#pragma unroll
                for (int i = 0; i < 16; ++i)
                  vals[i] = (mb + i < mrows) ? __ldcg(ws_tile + (mb + i) * kBlockN + r) : 0;
#pragma unroll
                for (int i = 0; i < 16; ++i)
                  if (mb + i < mrows) {
                    ws_tile[(mb + i) * kBlockN + r] = 0;
                    if (n_ok) store_out<OUT_I32>(p, m0 + mb + i, n, vals[i], sc);
                  }
              }
              if (warp == 2 && lane == 0) p.ticket[t] = 0u;
            }
          }
        }
      }
      u += kb1 - kb0;
    }
  epi_done:
    if (staged) bulk_wait_read();  // no bulk copy may still read the staging rows
    if (!red_done) {
      // owner on an error path: the other CTAs may still be writing into this
      // CTA's shared memory; wait (bounded) for their bytes before leaving
      const uint32_t a = smem_u32(redbar);
      const unsigned long long t0w = globaltimer();
      while (!mbar_try_wait_cluster(a, 0) && globaltimer() - t0w < 100000000ull) {
      }
    }
  }

  // ---------------------------------------------------------------- teardown
  __syncwarp();
  if constexpr (CS >= 2) {
    if (!cl_waited) cluster_wait();  // every thread completes the cluster barrier once
  }
  tc_fence_before();
  cta_barrier_unaligned();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem_base, C::kTmemCols);
  }
}

}  // namespace lq

/*
 * lq.h -- C ABI of the B200 (sm_100a) LiquidQuant W4A8 GEMM library.
 *
 * The method: "LiquidGEMM: Hardware-Efficient W4A8 GEMM Kernel for
 * High-Performance LLM Serving" (arXiv 2509.01229), as described on its
 * pith.science review page.  Weights go through two levels of quantization
 * (LiquidQuant, "LQQ"): per-channel symmetric INT8 in the protective range
 * [-119, 119], then group-wise UINT4 with an integer UINT8 scale s_u8 and an
 * offset a = 2^7 + min(Q_i8) per group of 64 along K.  Inside the GEMM each
 * 4-bit code is expanded back to INT8 with the overflow-free identity
 * Q_i8_hat = (Q_u4 * s_u8 + a) XOR 0x80, and the INT8 x INT8 product is
 * accumulated in int32 on the tensor cores.
 *
 * Conventions for every entry point
 *   - All pointers are DEVICE pointers unless stated otherwise.  The caller
 *     owns every buffer; the library never allocates or frees device memory.
 *   - Exception (zero-copy I/O): the bf16 activations X that a call reads
 *     (lq_quantize_act, lq_quantize_act_f8, lq_w4a8_linear*) and the outputs
 *     that a GEMM writes (`out` of every GEMM entry point) may also be host
 *     memory that the current device addresses at the same pointer: pinned
 *     with cudaHostAlloc, or registered with cudaHostRegister as mapped.  The
 *     kernels then read or write it over the host link directly, with no
 *     copy (for decode batches this is faster than a copy before and after:
 *     copy-engine transfers also end the programmatic-launch chain).  Any
 *     other host memory (pageable, or mapped at a different address) is
 *     refused with LQ_ERR_INVALID_ARG before anything is launched.  Weights,
 *     scales, int8 activations and workspaces must be device memory.
 *   - `stream` is a cudaStream_t passed as void* (NULL = the legacy default
 *     stream).  All work is enqueued asynchronously on it; nothing blocks the
 *     host except lq_get_device_error.
 *   - Arguments are validated before anything is launched; on any error
 *     nothing is launched and nothing is written.
 *   - Matrices are row-major.  Activations X and x_q are [M, K] (M tokens),
 *     weights W are [N, K] (nn.Linear layout, N output features), the output
 *     is [M, N].  bf16 buffers are passed as void*.
 *   - Only compute capability 10.0 devices (B200, sm_100a) are supported.
 *   - Inputs must be finite; non-finite values give unspecified codes but no
 *     fault.
 *
 * Packed weight format (this library's own; the paper's "dual-MMA packed
 * layout" is not given on the page):
 *   qw   uint8 [N, K/2]: in row n, little-endian 32-bit word j holds codes
 *        k = 8j..8j+7, byte b (0..3) = code[8j+b] | code[8j+4+b] << 4, so one
 *        AND yields codes 8j..8j+3 and one shift + AND yields 8j+4..8j+7,
 *        each already in byte order for a 4-wide SWAR expansion.
 *   s_u8 uint8 [K/64, N] and a_u8 uint8 [K/64, N]: per-group scale and
 *        offset, N contiguous.
 *   s_c  float [N]: per-channel scale of level 1 (amax / 119).
 */
#ifndef LQ_H
#define LQ_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define LQ_API __attribute__((visibility("default")))
#else
#define LQ_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum lq_status {
  LQ_OK = 0,
  LQ_ERR_INVALID_ARG = 1,       /* NULL pointer where data is needed, negative size */
  LQ_ERR_UNSUPPORTED_SHAPE = 2, /* a size rule below is broken */
  LQ_ERR_MISALIGNED = 3,        /* a pointer is not aligned as required */
  LQ_ERR_WORKSPACE = 4,         /* workspace missing or smaller than required */
  LQ_ERR_CUDA = 5,              /* a CUDA runtime or driver call failed */
  LQ_ERR_TIMEOUT = 6,           /* a device-side bounded wait gave up (reported by
                                   lq_get_device_error) */
  LQ_ERR_ARCH = 7               /* the current device is not compute capability 10.0 */
} lq_status;

/* Group size along K of the level-2 quantization (the paper's default). */
#define LQ_GROUP 64

/* Library version, major * 10000 + minor * 100 + patch. */
LQ_API int lq_version(void);

/* Human-readable name of a status code (static storage). */
LQ_API const char* lq_status_string(lq_status status);

/*
 * lq_quantize_weights -- offline LiquidQuant of a weight matrix (both levels).
 *   Level 1 (review page: referee summary and circularity rationale, the
 *   protective range "Q_i8 in [-119,119]"):
 *     amax_n = max_k |W[n,k]|;  Q_i8 = clamp(rint(W * (119 / amax_n)), -119, 119)
 *     s_c[n] = amax_n / 119;    a zero row gets s_c = 1 and codes 0.
 *   Level 2 (review page: referee summary; major comment 3 and minor comment 2
 *   on the integer scale; "What carries the argument" for the offset):
 *     per group of 64 along K: mn = min Q_i8, R = max Q_i8 - mn,
 *     s_u8 = max(1, round(R / 15)), a = 128 + mn,
 *     Q_u4 = min(15, round_half_up((Q_i8 - mn) / s_u8)).
 *   Rounding: float ops are single IEEE binary32 operations; rint is round to
 *   nearest even.
 *   W_bf16  [N, K] bf16, 16-byte aligned.
 *   qw      [N, K/2] uint8 out, 16-byte aligned.
 *   s_u8, a_u8 [K/64, N] uint8 out.   s_c [N] float out.
 *   group must be 64.  Requires N >= 1, K >= 64, K % 64 == 0.
 */
LQ_API lq_status lq_quantize_weights(const void* W_bf16, int N, int K, int group, uint8_t* qw,
                              uint8_t* s_u8, uint8_t* a_u8, float* s_c, void* stream);

/*
 * lq_quantize_act -- per-token symmetric INT8 activations (the review page's
 * "8-bit activations"; symmetric per token in [-127, 127] is this library's
 * reading):
 *   amax_m = max_k |X[m,k]|;  x_q = clamp(rint(X * (127 / amax_m)), -127, 127)
 *   s_x[m] = amax_m / 127;    a zero row gets s_x = 1 and codes 0.
 *   X_bf16 [M, K] bf16 and x_q [M, K] int8 out, both 16-byte aligned.
 *   s_x [M] float out.  Requires K % 16 == 0; M == 0 is a no-op.
 */
LQ_API lq_status lq_quantize_act(const void* X_bf16, int M, int K, int8_t* x_q, float* s_x, void* stream);

/*
 * lq_w4a8_gemm -- the W4A8 GEMM (review page: the abstract and referee
 * summary; the loop nest of Figure 2):
 *   W_hat[n,k] = int8((Q_u4[n,k] * s_u8[g,n] + a_u8[g,n]) XOR 0x80),  g = k / 64
 *   acc[m,n]   = sum_k x_q[m,k] * W_hat[n,k]          (exact, int32)
 *   out[m,n]   = bf16_rne(float(acc) * (s_x[m] * s_c[n]))
 *   x_q [M, K] int8, qw [N, K/2], s_u8/a_u8 [K/64, N] uint8: 16-byte aligned.
 *   s_x [M], s_c [N] float: 4-byte aligned.  out_bf16 [M, N] bf16 out.
 *   Requires group == 64, K % 128 == 0, 128 <= K <= 131072, N % 16 == 0,
 *   N >= 16; M == 0 is a no-op.
 *   workspace: device scratch of at least lq_w4a8_gemm_workspace_size(M,N,K)
 *   bytes (may be NULL when that is 0, which the automatic schedule always
 *   gives), 16-byte aligned, ZERO-FILLED by the caller before its first use.
 *   Each call leaves it zero-filled again, so it can be reused by later calls
 *   on the same stream without clearing; two calls in flight at the same time
 *   must not share one.  After a call that ended in LQ_ERR_TIMEOUT the caller
 *   must clear it again.
 *   Launch overlap: the GEMM and lq_quantize_act are launched as programmatic
 *   dependents of the preceding kernel in the stream (set LQ_PDL=0 in the
 *   environment to disable).  The GEMM starts streaming qw, s_u8 and a_u8
 *   before that kernel has finished, so those buffers must not be written by
 *   a kernel that itself triggers early launch (this library's weight
 *   quantizer does not); x_q, s_x, s_c and out are touched only after it has
 *   completed.  Each GEMM and lq_quantize_act in turn lets the next kernel in
 *   the stream launch as soon as its own CTAs have started: a kernel launched
 *   after it with programmatic stream serialization must wait for it
 *   (griddepcontrol.wait) before reading its output; other kernels are
 *   ordered as usual.
 */
LQ_API size_t lq_w4a8_gemm_workspace_size(int M, int N, int K);
LQ_API lq_status lq_w4a8_gemm(const int8_t* x_q, const float* s_x, const uint8_t* qw,
                       const uint8_t* s_u8, const uint8_t* a_u8, const float* s_c,
                       void* out_bf16, int M, int N, int K, int group, void* workspace,
                       size_t workspace_bytes, void* stream);

/* Schedules of lq_w4a8_gemm_ex. */
#define LQ_SCHED_AUTO 0       /* what lq_w4a8_gemm uses */
#define LQ_SCHED_TILES 1      /* one cluster of split_k CTAs per tile */
#define LQ_SCHED_PERSISTENT 2 /* grid CTAs loop over 128-token tiles */
#define LQ_SCHED_STREAMK 3    /* grid CTAs share the K-blocks of all tiles */
#define LQ_SCHED_PAIR 4       /* CTA pairs (tcgen05 cta_group::2) loop over 256 x 256 tiles */

/*
 * lq_w4a8_gemm_ex -- lq_w4a8_gemm with the schedule chosen by the caller
 * (tests and tuning).  Same result for every schedule (integer sums).
 *   block_t:  tokens per tile, one of 16, 32, 64, 128, 256; 0 = automatic
 *             (LQ_SCHED_PERSISTENT accepts only 0 or 128).
 *   schedule: LQ_SCHED_AUTO: block_t may be set, split_k and grid must be 0.
 *             LQ_SCHED_TILES: each tile of 128 weight rows x block_t tokens is
 *               computed by a thread-block cluster of split_k CTAs, each
 *               summing one slice of the K-blocks of 128; partial sums are
 *               reduced through distributed shared memory.  split_k is 1, 2,
 *               4 or 8 (8 only for block_t <= 32, 4 for block_t <= 128, 1
 *               for 256); 0 = automatic.  grid must be 0.
 *             LQ_SCHED_PERSISTENT: grid CTAs (0 = one per SM) loop over the
 *               tiles, overlapping each tile's epilogue with the next tile's
 *               main loop.  split_k must be 0.
 *             LQ_SCHED_PAIR: grid/2 clusters of two CTAs (0 = one CTA per SM)
 *               loop over tiles of 256 weight rows x 256 tokens; each MMA
 *               instruction spans both SMs of a pair.  Requires K % 256 == 0
 *               (else LQ_ERR_UNSUPPORTED_SHAPE); block_t must be 0 or 256;
 *               split_k must be 0.
 *             LQ_SCHED_STREAMK: the K-blocks of all tiles are spread evenly
 *               over grid CTAs (0 = one per SM; clamped to the number of
 *               K-blocks of work); tiles shared by several CTAs are reduced
 *               through the workspace.  split_k must be 0.
 *   out_i32:  when nonzero, out receives the int32 accumulators acc[m,n]
 *             instead of bf16 (bit-exact check of the contraction).
 * lq_w4a8_gemm_workspace_size_ex gives the workspace that schedule needs
 * (nonzero only for LQ_SCHED_STREAMK when tiles are shared).
 */
LQ_API size_t lq_w4a8_gemm_workspace_size_ex(int M, int N, int K, int block_t, int schedule, int split_k,
                                             int grid);
LQ_API lq_status lq_w4a8_gemm_ex(const int8_t* x_q, const float* s_x, const uint8_t* qw,
                                 const uint8_t* s_u8, const uint8_t* a_u8, const float* s_c, void* out,
                                 int M, int N, int K, int group, void* workspace, size_t workspace_bytes,
                                 int block_t, int schedule, int split_k, int grid, int out_i32,
                                 void* stream);

/* Paths of lq_w4a8_linear_ex. */
#define LQ_LINEAR_AUTO 0          /* what lq_w4a8_linear uses */
#define LQ_LINEAR_TWO_LAUNCHES 1  /* lq_quantize_act, then lq_w4a8_gemm */
#define LQ_LINEAR_FUSED 2         /* one launch; LQ_ERR_UNSUPPORTED_SHAPE where it does not apply */

/*
 * lq_w4a8_linear -- activation quantization and the GEMM in one call: the
 * result is bit-identical to lq_quantize_act(X) followed by lq_w4a8_gemm (the
 * same per-token INT8 codes and s_x, the same contraction and epilogue).
 *   X_bf16 [M, K] bf16 in, 16-byte aligned; qw, s_u8, a_u8, s_c and out_bf16
 *   as in lq_w4a8_gemm; same shape rules.
 *   The fused path applies to decode-sized batches (M <= 16) whose automatic
 *   schedule is a split-K cluster of 16-token tiles with each CTA's whole
 *   K-slice in shared memory (e.g. N = K = 4096): ONE launch, in which each
 *   CTA quantizes its K-slice of X itself and the cluster combines the row
 *   maxima through distributed shared memory; neither x_q nor s_x is written
 *   to memory and the workspace size is 0.  lq_w4a8_linear takes it for
 *   M <= 8 (on B200 at N = K = 4096 it is ahead of the two launches there and
 *   behind from M = 12, where each quantizing warp has more tokens); the
 *   other cases are the two launches, with x_q, s_x and the GEMM's workspace
 *   carved from `workspace`, which must hold
 *   lq_w4a8_linear_workspace_size(M, N, K) bytes, be 16-byte aligned and
 *   follow lq_w4a8_gemm's zero-fill rule (else LQ_ERR_WORKSPACE).
 *   lq_w4a8_linear_ex chooses the path (LQ_LINEAR_*; anything else is
 *   LQ_ERR_INVALID_ARG); its workspace size is lq_w4a8_linear_workspace_size_ex.
 *   Launch overlap as for lq_w4a8_gemm: X is read only after the preceding
 *   kernel in the stream has completed.
 *   The fused path is this library's (the pages quantize activations as a
 *   separate step); it changes when the work happens, not what is computed.
 */
LQ_API size_t lq_w4a8_linear_workspace_size(int M, int N, int K);
LQ_API lq_status lq_w4a8_linear(const void* X_bf16, const uint8_t* qw, const uint8_t* s_u8,
                                const uint8_t* a_u8, const float* s_c, void* out_bf16, int M, int N, int K,
                                int group, void* workspace, size_t workspace_bytes, void* stream);
LQ_API size_t lq_w4a8_linear_workspace_size_ex(int M, int N, int K, int path);
LQ_API lq_status lq_w4a8_linear_ex(const void* X_bf16, const uint8_t* qw, const uint8_t* s_u8,
                                   const uint8_t* a_u8, const float* s_c, void* out_bf16, int M, int N,
                                   int K, int group, void* workspace, size_t workspace_bytes, int path,
                                   void* stream);

/*
 * lq_w4a8_gemm_swiglu -- the gate/up pair of a gated FFN layer in one GEMM
 * with a fused SwiGLU epilogue (the FFN layers of the LiquidGEMM review page's
 * Fig. 12 caption; the pages do not write the gated FFN out, the reading is
 * the common one):
 *   out[m, j] = bf16( silu(y[m, 2j]) * y[m, 2j+1] ),
 *   y[m, n]   = float(acc[m, n]) * (s_x[m] * s_c[n])   (fp32, not rounded),
 *   silu(g)   = g / (1 + exp(-g))                        (fp32 steps).
 * The weights are one interleaved matrix of N = 2 * (FFN width) rows, row 2j
 * the gate channel j and row 2j + 1 the up channel j, quantized as usual by
 * lq_quantize_weights (per row, so interleaving changes no code).  Operands,
 * rules and workspace as lq_w4a8_gemm with this N; out_bf16 is [M, N/2]
 * (16-byte aligned).  The schedule is lq_w4a8_gemm's automatic one, a
 * persistent choice replaced by one cluster per tile (the SwiGLU epilogue
 * has no persistent or stream-K form).  exp is CUDA's expf (at most 2 ulp in
 * fp32), so an output may differ from a correctly rounded evaluation by one
 * bf16 ulp.
 */
LQ_API lq_status lq_w4a8_gemm_swiglu(const int8_t* x_q, const float* s_x, const uint8_t* qw, const uint8_t* s_u8,
                                     const uint8_t* a_u8, const float* s_c, void* out_bf16, int M, int N, int K,
                                     int group, void* workspace, size_t workspace_bytes, void* stream);
/* The same with the schedule chosen as in lq_w4a8_gemm_ex (test and
 * measurement use; LQ_SCHED_STREAMK and LQ_SCHED_PERSISTENT are refused with
 * LQ_ERR_UNSUPPORTED_SHAPE). */
LQ_API lq_status lq_w4a8_gemm_swiglu_ex(const int8_t* x_q, const float* s_x, const uint8_t* qw,
                                        const uint8_t* s_u8, const uint8_t* a_u8, const float* s_c, void* out_bf16,
                                        int M, int N, int K, int group, void* workspace, size_t workspace_bytes,
                                        int block_t, int schedule, int split_k, int grid, void* stream);

/*
 * lq_w4a8_gemm_i32 -- the contraction only: acc[m,n] as int32 [M, N] (16-byte
 * aligned), same operands, rules and workspace as lq_w4a8_gemm.
 */
LQ_API lq_status lq_w4a8_gemm_i32(const int8_t* x_q, const uint8_t* qw, const uint8_t* s_u8,
                           const uint8_t* a_u8, int32_t* acc, int M, int N, int K, int group,
                           void* workspace, size_t workspace_bytes, void* stream);

/*
 * lq_dequant_weights_i8 -- the in-kernel LiquidQuant expansion written out
 * (review page: "What carries the argument"; Eq. 12 in the circularity
 * rationale): w_i8[n,k] = int8((Q_u4 * s_u8 + a) XOR 0x80), [N, K] int8 out,
 * 16-byte aligned.  Uses the same device routine as the GEMM.  Requires
 * group == 64, K % 64 == 0, N >= 1.
 */
LQ_API lq_status lq_dequant_weights_i8(const uint8_t* qw, const uint8_t* s_u8, const uint8_t* a_u8, int N,
                                int K, int group, int8_t* w_i8, void* stream);

/*
 * lq_w4a8_gemm_noalloc -- lq_w4a8_gemm for callers that must not allocate
 * device memory where they launch the GEMM (a serving framework's enqueue
 * hook that owns all device memory, a latency-critical loop that cannot block
 * on the allocator or fail on out-of-memory mid-request).  The paper has no
 * counterpart; this is an interface convenience of this library.
 *   Same operands, layouts and result as lq_w4a8_gemm, computed with the
 *   stream-K schedule (one CTA per SM).  Its partial sums live in a 4 MiB
 *   scratch array inside the library image (held on every GPU that loads the
 *   library until the process exits) instead of a workspace; nothing is
 *   allocated and no workspace is passed.
 *   The scratch needed is ceil(M/bt) * ceil(N/128) * bt * 512 bytes plus a
 *   small tile counter area, bt being the automatic token-tile width (16, 32,
 *   64 or 128 tokens for M <= 16, 32, 64, larger); shapes that need more than
 *   the array return LQ_ERR_WORKSPACE without launching anything.
 *   The first call on each device looks up the array's device address
 *   (cudaGetSymbolAddress) with that device current; make that first call
 *   before any stream capture.  Every call clears the part of the array it
 *   uses (an asynchronous memset on `stream`) before the GEMM.
 *   All calls on a device share the one array: calls that can overlap on the
 *   GPU race and corrupt each other's results, so order them (e.g. issue
 *   them on one stream).
 */
LQ_API lq_status lq_w4a8_gemm_noalloc(const int8_t* x_q, const float* s_x, const uint8_t* qw,
                                      const uint8_t* s_u8, const uint8_t* a_u8, const float* s_c,
                                      void* out_bf16, int M, int N, int K, int group, void* stream);

/*
 * lq_plan_gemm -- TEST ONLY, touches no device: the schedule lq_w4a8_gemm_ex
 * would run for these arguments on a GPU with `sms` multiprocessors, all of
 * them reachable by clusters of every size (lq_plan_gemm_ex with
 * cluster_ctas = NULL).  On LQ_OK, plan[0..3] = schedule kind (LQ_SCHED_*),
 * token-tile width, CTAs per cluster (0 for stream-K, 2 for CTA pairs), grid
 * size.  Argument errors as in lq_w4a8_gemm_ex (M >= 1 here).
 */
LQ_API lq_status lq_plan_gemm(int M, int N, int K, int block_t, int schedule, int split_k, int grid, int sms,
                              int* plan);

/*
 * lq_plan_gemm_ex -- TEST ONLY, touches no device: lq_plan_gemm on a GPU
 * whose clusters of 2, 4 and 8 CTAs, two CTAs per SM, place at most
 * cluster_ctas[0], [1] and [2] CTAs at once (host array of 3 ints, each >= 1,
 * else LQ_ERR_INVALID_ARG; NULL: 2 x sms each).  The automatic schedule gives
 * streaming K-slices the widest split whose CTAs fit one wave of that
 * placement.  lq_device_cluster_ctas gives the current device's numbers, which
 * lq_w4a8_gemm_ex and the other GEMM calls use.
 */
LQ_API lq_status lq_plan_gemm_ex(int M, int N, int K, int block_t, int schedule, int split_k, int grid, int sms,
                                 const int* cluster_ctas, int* plan);

/*
 * lq_device_cluster_ctas -- how many CTAs of 2-, 4- and 8-CTA clusters the
 * current device holds at once with two CTAs per SM (cluster_ctas: host array
 * of 3 ints, written on LQ_OK).  A cluster's CTAs share one GPC, so slots
 * beyond a GPC's last whole cluster stay empty (B200, 148 SMs: 296, 284, 264).
 * The numbers come from the CUDA occupancy calculator at the first call of
 * any entry point on the device (2 x SMs where it cannot answer); no kernel
 * is launched.  LQ_ERR_INVALID_ARG for a NULL array, LQ_ERR_CUDA without a
 * device, LQ_ERR_ARCH on a device other than sm_100.
 */
LQ_API lq_status lq_device_cluster_ctas(int* cluster_ctas);

/*
 * lq_w4a8_gemm_ablation -- TEST AND MEASUREMENT ONLY: the pages' ablation of
 * the dequantization arithmetic (LQQ) and of the pipeline (explicit
 * coarse-grained, ExCP, vs implicit fine-grained, ImFP: LiquidGEMM Figs. 6
 * and 13, as the review page's figure list and referee summary describe
 * them), redone on sm_100 with four forms of the same tile kernel:
 *   LQ_ABL_IMPLICIT (0): the product kernel -- SWAR expansion (one IMAD and
 *     one XOR per four weights) into tensor memory, MMA with A from TMEM;
 *   LQ_ABL_NAIVE (1): that pipeline with the weights expanded one at a time
 *     (extract, IMAD, XOR, insert per weight);
 *   LQ_ABL_EXPLICIT (2): SWAR expansion written to a shared-memory A tile
 *     per slot (128-byte swizzle) and an MMA that reads both operands from
 *     shared memory;
 *   LQ_ABL_NAIVE_EXPLICIT (3): both.
 *   Same operands, result and errors as lq_w4a8_gemm_ex with the tile
 *   schedule; block_t must be 16 or 64 and split_k 4 (else
 *   LQ_ERR_UNSUPPORTED_SHAPE); out_i32 as in lq_w4a8_gemm_ex.  Every variant
 *   gives bit-identical results.
 */
#define LQ_ABL_IMPLICIT 0
#define LQ_ABL_NAIVE 1
#define LQ_ABL_EXPLICIT 2
#define LQ_ABL_NAIVE_EXPLICIT 3
LQ_API lq_status lq_w4a8_gemm_ablation(const int8_t* x_q, const float* s_x, const uint8_t* qw,
                                       const uint8_t* s_u8, const uint8_t* a_u8, const float* s_c, void* out,
                                       int M, int N, int K, int group, int variant, int block_t, int split_k,
                                       int out_i32, void* stream);

/*
 * lq_w4a8_grouped_gemm -- the W4A8 GEMM for a mixture-of-experts layer (one
 * weight matrix per group, or expert, each applied to its own run of token
 * rows): out[m, n] = bf16((sum_k x_q[m,k] * Q_hat[e*N + n, k]) * s_x[m] *
 * s_c[e*N + n]) for the rows m in [m_off[e], m_off[e+1]) of group e.  The
 * models the review page names for the accuracy study include the
 * mixture-of-experts Mixtral-8x7B ("What would settle it"); the grouped form
 * is this library's, not the paper's.
 *   x_q, s_x: [M, K] int8 and [M] fp32 from lq_quantize_act, the rows of
 *     each group contiguous and in group order (a router's sorted token
 *     copies).
 *   qw, s_u8, a_u8, s_c: the `groups` weight matrices stacked as one
 *     [groups * N, K] matrix and quantized in one lq_quantize_weights call
 *     (quantization is per row, so stacking changes nothing).
 *   m_off: DEVICE int32 [groups + 1], non-decreasing, m_off[0] = 0,
 *     m_off[groups] = M; it may be written by the kernel that precedes this
 *     one on the stream (it is read after the grid dependency wait).
 *     Empty groups are allowed.  Offsets that break these rules give
 *     undefined (but in-bounds) results.
 *   out_bf16: [M, N] bf16, row m for the group that owns m.
 *   Requires N % 128 == 0 (a weight tile never spans two groups), the GEMM's
 *   K and group rules, 1 <= groups <= LQ_MAX_GROUPS, 16-byte-aligned
 *   x_q, qw, s_u8, a_u8, out and 4-byte-aligned s_x, s_c, m_off.  No
 *   workspace.  Groups of more than 128 rows on average (with N % 256 == 0
 *   and K % 256 == 0) run on CTA pairs over 256 x 256 tiles; otherwise one
 *   thread-block cluster per 128-row weight tile and token tile (split-K
 *   inside the cluster for small token counts).  Tiles past the last group's
 *   rows are skipped.
 * lq_w4a8_grouped_gemm_ex adds block_t (0 = automatic, else 16, 32, 64 or 128
 *   for the tile kernel, or 256 for CTA pairs, which need N % 256 == 0 and
 *   K % 256 == 0), split_k (0 = automatic, else as in LQ_SCHED_TILES; none
 *   with 256) and out_i32 (int32 accumulators to `out`, s_x and s_c unused).
 */
#define LQ_MAX_GROUPS 1024
LQ_API lq_status lq_w4a8_grouped_gemm(const int8_t* x_q, const float* s_x, const uint8_t* qw,
                                      const uint8_t* s_u8, const uint8_t* a_u8, const float* s_c,
                                      const int* m_off, int groups, void* out_bf16, int M, int N, int K,
                                      int group, void* stream);
LQ_API lq_status lq_w4a8_grouped_gemm_ex(const int8_t* x_q, const float* s_x, const uint8_t* qw,
                                         const uint8_t* s_u8, const uint8_t* a_u8, const float* s_c,
                                         const int* m_off, int groups, void* out, int M, int N, int K,
                                         int group, int block_t, int split_k, int out_i32, void* stream);

/*
 * The W4 x FP8 variant (FireQ page, abstract: INT4 weights with channel-wise
 * scaling, FP8 activations with one scale for the tensor).  The pages give
 * no formulas; the readings:
 * lq_quantize_weights_w4 -- per-channel symmetric INT4: s_w[n] = amax_n / 7,
 *   q = clamp(rint(w * (7 / amax_n)), -7, 7) with IEEE fp32 operations,
 *   stored as q + 8 in the LiquidQuant nibble layout (qw4 [N, K/2]); a zero
 *   row gets s_w = 1 and q = 0.  K % 16 == 0; W and qw4 16-byte aligned.
 * lq_quantize_act_f8 -- FP8 e4m3 activations with one scale for the tensor:
 *   s_x[0] = amax / 448, x_f8 = e4m3(x * (448 / amax)), round to nearest
 *   even, saturated to +-448 (cvt ... satfinite); an all-zero or empty
 *   tensor gets s_x = 1.  Three launches and a 4-byte memset on `stream`
 *   (the tensor's maximum is gathered in s_x's word first).  K % 16 == 0.
 * lq_w4f8_gemm -- out[m,n] = bf16(acc * (s_x[0] * s_w[n])), acc the fp32
 *   sum over k of e4m3(x)[m,k] * q[n,k] computed by tcgen05.mma
 *   kind::f8f6f4 (the products are exact; the fp32 accumulation order is the
 *   tensor core's within a CTA's K-slice, and split-K partial sums are added
 *   in a fixed order, so repeated calls give identical bits).  The schedule
 *   is lq_w4a8_gemm's cluster form for 16-, 64- or 128-token tiles (M <= 16,
 *   <= 64, above): a cluster of CTAs per 128-row tile, split over K and
 *   reduce-scattered through distributed shared memory.  Shape and alignment
 *   rules as lq_w4a8_gemm (no group, no workspace).  Allocates nothing.
 */
LQ_API lq_status lq_quantize_weights_w4(const void* W_bf16, int N, int K, uint8_t* qw4, float* s_w, void* stream);
LQ_API lq_status lq_quantize_act_f8(const void* X_bf16, int M, int K, uint8_t* x_f8, float* s_x, void* stream);
LQ_API lq_status lq_w4f8_gemm(const uint8_t* x_f8, const float* s_x, const uint8_t* qw4, const float* s_w,
                              void* out_bf16, int M, int N, int K, void* stream);

/*
 * lq_device_addressable -- 1 if the current device can read and write `p`
 *   at that address (device or managed memory, or host memory mapped at the
 *   same address: the zero-copy rule above), else 0.  Launches nothing.
 */
LQ_API int lq_device_addressable(const void* p);

/*
 * lq_test_wait_timeout -- TEST ONLY: launches a one-CTA kernel whose first
 * warp waits on an mbarrier that nothing completes, with the GEMM kernels'
 * bounded wait: after the 2 s limit it raises the CTA's abort flag and
 * records LQ_ERR_TIMEOUT in the device error word; a second warp waiting on
 * another such barrier leaves as soon as the flag is up.  No fault, no trap:
 * the context stays usable, and lq_get_device_error then returns
 * LQ_ERR_TIMEOUT once.
 */
LQ_API lq_status lq_test_wait_timeout(void* stream);

/*
 * lq_get_device_error -- synchronizes `stream`, then reads and clears the
 * library's device error word.  Returns LQ_ERR_TIMEOUT if a kernel gave up a
 * bounded wait since the last call (its output is then undefined),
 * LQ_ERR_CUDA if the synchronization itself failed, else LQ_OK.
 */
LQ_API lq_status lq_get_device_error(void* stream);

#ifdef __cplusplus
}
#endif

#endif /* LQ_H */

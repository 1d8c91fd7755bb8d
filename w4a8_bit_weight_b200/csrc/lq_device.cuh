// lq_device.cuh -- device-side building blocks for sm_100a: mbarriers with
// bounded waits, TMA tile loads, tcgen05 (TMEM allocation, MMA, loads and
// stores), and the LiquidQuant 4-wide SWAR dequantization.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace lq {

// Device error word: 0 = none, else the first error code recorded since the
// host last read it (lq_get_device_error).
constexpr unsigned kErrTimeout = 6u;

// A single bounded wait never takes longer than this in a correct launch; a
// wait that does is treated as a fault: the kernel records kErrTimeout,
// unwinds and returns, leaving the context usable.
constexpr unsigned long long kWaitLimitNs = 2000000000ull;  // 2 s

// (this header is included by the library's single translation unit)
__device__ unsigned int g_error = 0;

__device__ __forceinline__ void record_error(unsigned code) { atomicCAS(&g_error, 0u, code); }

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ unsigned long long globaltimer() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// ---------------------------------------------------------------- mbarrier
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
               : "memory");
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

// Loads of data that the preceding kernel may write (activations, their
// scales, group row offsets), made after griddepcontrol.wait.  Under
// programmatic dependent launch that kernel is still running while this one
// is resident, so the non-coherent read-only path (whose data must not change
// during the kernel's lifetime) is not used for them: they are read through
// L2 (ld.global.cg).
template <typename T>
__device__ __forceinline__ T ld_dep(const T* ptr) {
  return __ldcg(ptr);
}

// Waits for the phase with the given parity to complete.  Gives up when the
// CTA-wide abort flag is raised by another role, or after kWaitLimitNs (then
// it raises the flag itself and records the error).  Returns false on give-up.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, volatile int* abort_flag) {
  const uint32_t a = smem_u32(bar);
  if (mbar_try_wait(a, parity)) return true;
  const unsigned long long t0 = globaltimer();
  while (true) {
    if (mbar_try_wait(a, parity)) return true;
    if (*abort_flag) return false;
    if (globaltimer() - t0 > kWaitLimitNs) {
      *abort_flag = 1;
      record_error(kErrTimeout);
      return false;
    }
  }
}

// Test of the bounded waits (no fault, no trap): warp 0 waits on a barrier
// that nothing completes and gives up after kWaitLimitNs, raising the CTA
// abort flag and recording kErrTimeout; warp 1 waits on another such barrier
// and must leave as soon as the flag is up, not after its own limit.
__global__ void wait_timeout_kernel() {
  __shared__ uint64_t bar[2];
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar[0], 1);
    mbar_init(&bar[1], 1);
    abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  if ((threadIdx.x & 31) == 0) mbar_wait(&bar[threadIdx.x >> 5], 0, &abort_flag);
  __syncthreads();
}

// Cluster-scope wait: also makes visible the shared-memory writes that other
// CTAs of the cluster released before arriving (remote arrive with .release).
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

__device__ __forceinline__ bool mbar_wait_cluster(uint64_t* bar, uint32_t parity, volatile int* abort_flag) {
  const uint32_t a = smem_u32(bar);
  if (mbar_try_wait_cluster(a, parity)) return true;
  const unsigned long long t0 = globaltimer();
  while (true) {
    if (mbar_try_wait_cluster(a, parity)) return true;
    if (*abort_flag) return false;
    if (globaltimer() - t0 > kWaitLimitNs) {
      *abort_flag = 1;
      record_error(kErrTimeout);
      return false;
    }
  }
}

// ------------------------------------------------- clusters and DSMEM
// Orders this thread's prior memory operations (shared::cluster stores
// included) before its later ones, at cluster scope.
__device__ __forceinline__ void fence_acq_rel_cluster() { asm volatile("fence.acq_rel.cluster;" ::: "memory"); }

__device__ __forceinline__ uint32_t cluster_ctarank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
// Cluster barrier in two halves: every thread of every CTA arrives once and
// waits once (each warp converged at both points).
__device__ __forceinline__ void cluster_arrive() {
  asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory");
}
__device__ __forceinline__ void cluster_wait() {
  asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory");
}
// Address of the same shared-memory variable in CTA `rank` of this cluster.
__device__ __forceinline__ uint32_t mapa_shared(uint32_t saddr, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(saddr), "r"(rank));
  return r;
}
__device__ __forceinline__ void st_cluster_u32(uint32_t caddr, uint32_t v) {
  asm volatile("st.shared::cluster.u32 [%0], %1;" ::"r"(caddr), "r"(v) : "memory");
}
// Bulk copy of `bytes` (a multiple of 16, both addresses 16-byte aligned) from
// this CTA's shared memory into another CTA's, counted on that CTA's mbarrier.
// The source must stay untouched until bulk_wait_read() returns.
__device__ __forceinline__ void bulk_copy_s2s(uint32_t dst_caddr, const void* src, uint32_t bytes, uint32_t bar_caddr) {
  asm volatile(
      "cp.async.bulk.shared::cluster.shared::cta.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst_caddr),
      "r"(smem_u32(src)), "r"(bytes), "r"(bar_caddr)
      : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
// Waits until every committed bulk copy of this thread has read its source.
__device__ __forceinline__ void bulk_wait_read() { asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory"); }
// Makes this thread's generic shared-memory writes visible to later async-proxy
// reads (bulk copies, TMA stores).
__device__ __forceinline__ void fence_proxy_async_smem() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

// 16-byte store into another CTA's shared memory whose bytes are counted on
// that CTA's mbarrier (complete_tx): no fence or arrive needed on this side.
__device__ __forceinline__ void st_async_v4(uint32_t caddr, uint32_t a, uint32_t b, uint32_t c, uint32_t d,
                                            uint32_t bar_caddr) {
  asm volatile("st.async.shared::cluster.mbarrier::complete_tx::bytes.v4.b32 [%0], {%1, %2, %3, %4}, [%5];" ::"r"(
                   caddr),
               "r"(a), "r"(b), "r"(c), "r"(d), "r"(bar_caddr)
               : "memory");
}
// 8-byte form of st_async_v4.
__device__ __forceinline__ void st_async_v2(uint32_t caddr, uint32_t a, uint32_t b, uint32_t bar_caddr) {
  asm volatile("st.async.shared::cluster.mbarrier::complete_tx::bytes.v2.b32 [%0], {%1, %2}, [%3];" ::"r"(caddr),
               "r"(a), "r"(b), "r"(bar_caddr)
               : "memory");
}
// Arrive on an mbarrier of another CTA of the cluster, releasing this
// thread's earlier writes at cluster scope.
__device__ __forceinline__ void mbar_arrive_remote(uint32_t caddr) {
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(caddr) : "memory");
}

// ------------------------------------ programmatic dependent launch (PDL)
// Blocks until the grids this launch depends on have completed and their
// memory is visible (returns at once when launched without the attribute).
__device__ __forceinline__ void griddep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
// Lets the next kernel in the stream start its prologue early.
__device__ __forceinline__ void griddep_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// -------------------------------------------------------------------- TMA
__device__ __forceinline__ void tma_prefetch_desc(const CUtensorMap* map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// 2D tiled bulk tensor load into this CTA's shared memory, completion
// reported as transaction bytes on `bar`.  c0 is the innermost coordinate.
__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, uint64_t* bar, int c0,
                                            int c1, uint64_t cache_hint) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
      " [%0], [%1, {%3, %4}], [%2], %5;" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(c0), "r"(c1), "l"(cache_hint)
      : "memory");
}

// 3D tiled bulk tensor load (c0 innermost), completion as transaction bytes on `bar`.
__device__ __forceinline__ void tma_load_3d(void* dst, const CUtensorMap* map, uint64_t* bar, int c0, int c1, int c2,
                                            uint64_t cache_hint) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
      " [%0], [%1, {%3, %4, %5}], [%2], %6;" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(c0), "r"(c1), "r"(c2), "l"(cache_hint)
      : "memory");
}

// L2 eviction-priority policies for the cache_hint operand.
__device__ __forceinline__ uint64_t l2_policy_evict_first() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
  return p;
}
__device__ __forceinline__ uint64_t l2_policy_evict_last() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(p));
  return p;
}

// ---------------------------------------------------------------- tcgen05
__device__ __forceinline__ void tmem_alloc(uint32_t* dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(dst_smem)),
               "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
// Arrives on `bar` once every tcgen05 operation this thread issued so far has
// completed.
__device__ __forceinline__ void tc_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                   smem_u32(bar))
               : "memory");
}

// D[128 x N] (+)= A[128 x 32] * B[N x 32]^T, int8 x int8 -> int32, with A in
// tensor memory and B described by a shared-memory matrix descriptor.
__device__ __forceinline__ void mma_i8_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                          uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::i8 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// The same with A also described by a shared-memory matrix descriptor.
__device__ __forceinline__ void mma_i8_ss(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                          uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::i8 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// kind::f8f6f4 (e4m3 A and B, fp32 D) with A in tensor memory / in shared memory.
__device__ __forceinline__ void mma_f8_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                          uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
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

// kind::f8f6f4 instruction descriptor: fp32 D, e4m3 A and B, both K-major,
// M = 128, N = n.
__host__ __device__ constexpr uint32_t idesc_f8(int n) {
  return (1u << 4)                        // D format: f32
         | (0u << 7) | (0u << 10)         // A, B: e4m3
         | (uint32_t(n >> 3) << 17) | (uint32_t(128 >> 4) << 24);
}

// Instruction descriptor for kind::i8: signed A and B, int32 D, both K-major,
// M = 128, N = n (multiple of 16, 16..256).
__host__ __device__ constexpr uint32_t idesc_i8(int n) {
  return (2u << 4)                          // D format: s32
         | (1u << 7)                        // A: signed 8-bit
         | (1u << 10)                       // B: signed 8-bit
         | (uint32_t(n >> 3) << 17)         // N / 8
         | (uint32_t(128 >> 4) << 24);      // M / 16
}

// Shared-memory matrix descriptor of a K-major operand tile stored with the
// 128-byte swizzle: rows of 128 bytes, 8-row atoms of 1024 bytes.  The tile
// base must be 1024-byte aligned; a K offset inside the 128-byte row is
// applied by advancing the start address.
__device__ __forceinline__ uint64_t smem_desc_k_sw128(uint32_t saddr) {
  return (uint64_t)((saddr & 0x3FFFFu) >> 4)  // start address / 16
         | (1ull << 16)                       // leading byte offset (unused for this layout)
         | ((uint64_t)(1024 >> 4) << 32)      // stride byte offset: 8 rows x 128 B
         | (1ull << 46)                       // descriptor version for tcgen05
         | (2ull << 61);                      // 128-byte swizzle
}

#define LQ_R8(i) "r"(v[i]), "r"(v[i + 1]), "r"(v[i + 2]), "r"(v[i + 3]), "r"(v[i + 4]), "r"(v[i + 5]), "r"(v[i + 6]), "r"(v[i + 7])
#define LQ_W8(i) "=r"(v[i]), "=r"(v[i + 1]), "=r"(v[i + 2]), "=r"(v[i + 3]), "=r"(v[i + 4]), "=r"(v[i + 5]), "=r"(v[i + 6]), "=r"(v[i + 7])

// Each thread of the warp writes 32 consecutive 32-bit columns of its own lane.
__device__ __forceinline__ void tmem_st_32x32b_x32(uint32_t taddr, const uint32_t (&v)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, "
      "%13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, "
      "%32};" ::"r"(taddr),
      LQ_R8(0), LQ_R8(8), LQ_R8(16), LQ_R8(24)
      : "memory");
}
__device__ __forceinline__ void tmem_st_32x32b_x16(uint32_t taddr, const uint32_t (&v)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, "
      "%14, %15, %16};" ::"r"(taddr),
      LQ_R8(0), LQ_R8(8)
      : "memory");
}
__device__ __forceinline__ void tmem_st_wait() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// Each thread of the warp reads 2 / 4 / 8 / 16 / 32 consecutive 32-bit columns of its lane.
__device__ __forceinline__ void tmem_ld_32x32b_x2(uint32_t taddr, uint32_t (&v)[2]) {
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x2.b32 {%0, %1}, [%2];" : "=r"(v[0]), "=r"(v[1]) : "r"(taddr) : "memory");
}
__device__ __forceinline__ void tmem_ld_32x32b_x4(uint32_t taddr, uint32_t (&v)[4]) {
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x4.b32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3])
               : "r"(taddr)
               : "memory");
}
__device__ __forceinline__ void tmem_ld_32x32b_x8(uint32_t taddr, uint32_t (&v)[8]) {
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
               : LQ_W8(0)
               : "r"(taddr)
               : "memory");
}
__device__ __forceinline__ void tmem_ld_32x32b_x16(uint32_t taddr, uint32_t (&v)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, "
      "%13, %14, %15}, [%16];"
      : LQ_W8(0), LQ_W8(8)
      : "r"(taddr)
      : "memory");
}
__device__ __forceinline__ void tmem_ld_32x32b_x32(uint32_t taddr, uint32_t (&v)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, "
      "%13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, "
      "%31}, [%32];"
      : LQ_W8(0), LQ_W8(8), LQ_W8(16), LQ_W8(24)
      : "r"(taddr)
      : "memory");
}
__device__ __forceinline__ void tmem_ld_wait() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }
// The same wait, with the loaded registers tied to it so that no use of them
// can be scheduled before the wait.
__device__ __forceinline__ void tmem_ld_wait_x16(uint32_t (&v)[16]) {
  asm volatile("tcgen05.wait::ld.sync.aligned;"
               : "+r"(v[0]), "+r"(v[1]), "+r"(v[2]), "+r"(v[3]), "+r"(v[4]), "+r"(v[5]), "+r"(v[6]), "+r"(v[7]),
                 "+r"(v[8]), "+r"(v[9]), "+r"(v[10]), "+r"(v[11]), "+r"(v[12]), "+r"(v[13]), "+r"(v[14]), "+r"(v[15])
               :
               : "memory");
}

#undef LQ_R8
#undef LQ_W8

// CTA-wide barrier that counts threads one by one (the non-.aligned form),
// correct even when the lanes of a warp arrive at different times.
__device__ __forceinline__ void cta_barrier_unaligned() { asm volatile("barrier.sync 0;" ::: "memory"); }

__device__ __forceinline__ uint4 lds128(uint32_t saddr) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "r"(saddr));
  return v;
}

// ------------------------------------------------- LiquidQuant expansion
// One packed 32-bit word holds eight 4-bit codes: bytes 0..3 low nibbles are
// codes k = 8j..8j+3, high nibbles k = 8j+4..8j+7.  Per four codes the
// expansion is one integer multiply-add and one XOR on the whole 32-bit word:
// every byte lane computes q * s + a <= 255 (the paper's UINT8 range
// guarantee), so no carry crosses a byte, and XOR 0x80 turns each UINT8
// lane into the two's-complement INT8 weight.  `a4` is a * 0x01010101.
__device__ __forceinline__ void lqq_expand_word(uint32_t w, uint32_t s, uint32_t a4, uint32_t& lo,
                                                uint32_t& hi) {
  lo = ((w & 0x0F0F0F0Fu) * s + a4) ^ 0x80808080u;
  hi = (((w >> 4) & 0x0F0F0F0Fu) * s + a4) ^ 0x80808080u;
}

__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
  uint32_t d;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
  return d;
}

// Eight symmetric INT4 codes of one packed word (u = q + 8, code k in byte
// k % 4, high nibble for k >= 4) as eight e4m3 bytes in code order: codes 0-3
// in `lo`, 4-7 in `hi`.  Every integer in [-8, 7] is an e4m3 value, so this
// is exact.  Byte permutes serve as 8-entry tables, indexed by a nibble's low
// three bits; a selector nibble with bit 3 set fills the byte with the top
// bit of the entry instead, and both tables keep that bit clear:
//   table P (e4m3 of 0..7), selectors u ^ 8: u >= 8 reads e4m3(u - 8),
//     u < 8 reads 0;
//   table N (e4m3 of -8..-1 without the sign bit), selectors u: u < 8 reads
//     |e4m3(u - 8)|, u >= 8 reads 0.
// The selectors of one 16-bit half are codes (0, 4, 1, 5) or (2, 6, 3, 7), so
// two more permutes put the bytes in code order; the sign (u < 8) is bit 3 of
// the code, negated and moved to bit 7 of its byte.
__device__ __forceinline__ void w4_word_to_e4m3(uint32_t w, uint32_t& lo, uint32_t& hi) {
  constexpr uint32_t kP0 = 0x44403800u, kP1 = 0x4E4C4A48u;  // e4m3(0..3), e4m3(4..7)
  constexpr uint32_t kN0 = 0x4A4C4E50u, kN1 = 0x38404448u;  // |e4m3(-8..-5)|, |e4m3(-4..-1)|
  const uint32_t wf = w ^ 0x88888888u;
  const uint32_t r0 = prmt(kP0, kP1, wf) | prmt(kN0, kN1, w);               // codes 0, 4, 1, 5
  const uint32_t r1 = prmt(kP0, kP1, wf >> 16) | prmt(kN0, kN1, w >> 16);   // codes 2, 6, 3, 7
  lo = prmt(r0, r1, 0x6420u) | (~(w << 4) & 0x80808080u);
  hi = prmt(r0, r1, 0x7531u) | (~w & 0x80808080u);
}

// The same eight values one at a time (nibble extract, IMAD, XOR, byte insert
// per weight): the per-element dequantization the SWAR form replaces, kept
// for the ablation of the expansion arithmetic.  a is the plain u8 offset.
__device__ __forceinline__ void naive_expand_word(uint32_t w, uint32_t s, uint32_t a, uint32_t& lo, uint32_t& hi) {
  uint32_t r0 = 0u, r1 = 0u;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const uint32_t q0 = (w >> (8 * i)) & 0xFu, q1 = (w >> (8 * i + 4)) & 0xFu;
    r0 |= (((q0 * s + a) ^ 0x80u) & 0xFFu) << (8 * i);
    r1 |= (((q1 * s + a) ^ 0x80u) & 0xFFu) << (8 * i);
  }
  lo = r0;
  hi = r1;
}

}  // namespace lq

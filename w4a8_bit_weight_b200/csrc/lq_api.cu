// lq_api.cu -- the C ABI (include/lq.h): argument validation, schedule choice,
// TMA descriptors and kernel launches.  All device code of the library is in
// this one translation unit.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>
#include <climits>
#include <cstdint>
#include <cstdlib>
#include <cstring>
#include <mutex>

#include "../../include/lq.h"
#include "lq_device.cuh"
#include "lq_gemm_kernel.cuh"
#include "lq_gemm_w4f8.cuh"
#include "lq_gemm_persistent.cuh"
#include "lq_gemm_pair.cuh"
#include "lq_quant_kernels.cuh"

namespace {

constexpr int kMaxDevices = 64;

// Filled once per device under g_mu; `ready` is published last (release) and
// read first (acquire), so a thread that sees it set sees the other fields.
struct DeviceInfo {
  std::atomic<bool> ready{false};
  bool sm100 = false;
  int sms = 0;
  int cluster_ctas[3] = {0, 0, 0};  // see cluster_fit
};
DeviceInfo g_dev[kMaxDevices];
std::mutex g_mu;

// An empty kernel that only the occupancy query below names (never launched).
__global__ void cluster_fit_probe_kernel() {}

// How many CTAs of c-CTA clusters the device holds at once when two CTAs share
// an SM.  A cluster's CTAs must sit in one GPC, so a GPC's slots beyond its
// last whole cluster stay empty: on B200 (148 SMs, 296 slots) clusters of 2, 4
// and 8 place 296, 284 and 264 CTAs.  The occupancy calculator answers for an
// empty 192-thread kernel whose shared memory admits exactly two CTAs per SM
// (as the tile kernel's does wherever two of its CTAs share an SM); if it
// cannot answer, 2 x sms.
int cluster_fit(int c, int sms) {
  constexpr int kSmem = 100 * 1024;  // two fit in an SM's 228 KB, three do not
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(c);
  cfg.blockDim = dim3(192);
  cfg.dynamicSmemBytes = kSmem;
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeClusterDimension;
  at[0].val.clusterDim.x = c;
  at[0].val.clusterDim.y = 1;
  at[0].val.clusterDim.z = 1;
  cfg.attrs = at;
  cfg.numAttrs = 1;
  int n = 0;
  if (cudaFuncSetAttribute(cluster_fit_probe_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmem) !=
          cudaSuccess ||
      cudaOccupancyMaxActiveClusters(&n, cluster_fit_probe_kernel, &cfg) != cudaSuccess || n <= 0) {
    (void)cudaGetLastError();
    return 2 * sms;
  }
  return std::min(2 * sms, n * c);
}

lq_status current_device(DeviceInfo** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return LQ_ERR_CUDA;
  DeviceInfo& d = g_dev[dev];
  if (!d.ready.load(std::memory_order_acquire)) {
    std::lock_guard<std::mutex> lk(g_mu);
    if (!d.ready.load(std::memory_order_relaxed)) {
      int major = 0, minor = 0, sms = 0;
      if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
          cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
          cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
        return LQ_ERR_CUDA;
      d.sm100 = (major == 10 && minor == 0);
      d.sms = sms;
      if (d.sm100)
        for (int i = 0; i < 3; ++i) d.cluster_ctas[i] = cluster_fit(2 << i, sms);
      d.ready.store(true, std::memory_order_release);
    }
  }
  *out = &d;
  return d.sm100 ? LQ_OK : LQ_ERR_ARCH;
}

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

// The bf16 activations a call reads and the outputs it writes may be host
// memory that the current device addresses directly (pinned with
// cudaHostAlloc, or registered with cudaHostRegister as mapped): the kernels
// then read or write it over the host link, with no copy.  Device and managed
// memory are addressable too.  Memory that CUDA does not know (pageable host
// memory) or host memory mapped at another address is refused before any
// launch.
bool device_addressable(const void* p) {
  cudaPointerAttributes a;
  if (cudaPointerGetAttributes(&a, p) != cudaSuccess) {
    (void)cudaGetLastError();
    return false;
  }
  switch (a.type) {
    case cudaMemoryTypeDevice:
    case cudaMemoryTypeManaged:
      return true;
    case cudaMemoryTypeHost:
      return a.devicePointer == p;
    default:
      return false;
  }
}

// ------------------------------------------------------------ tensor maps
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// 2D byte-element tensor [outer][inner] with `row_bytes` between rows.
bool make_map_u8(CUtensorMap* m, const void* base, uint64_t inner, uint64_t outer, uint64_t row_bytes,
                 uint32_t box_inner, uint32_t box_outer, CUtensorMapSwizzle sw) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  const cuuint64_t dims[2] = {inner, outer};
  const cuuint64_t strides[1] = {row_bytes};
  const cuuint32_t box[2] = {box_inner, box_outer};
  const cuuint32_t estr[2] = {1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// The activations of a split-K CTA's first `stages` K-blocks as one 3D box:
// x_q [M][K] viewed as [K/128 blocks][M tokens][128 bytes]; a box is `stages`
// blocks x bt tokens, which is the tile kernel's shared-memory ring layout.
bool make_map_x3(CUtensorMap* m, const void* x_q, int M, int K, int bt, int stages) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  const cuuint64_t dims[3] = {(cuuint64_t)lq::kBlockK, (cuuint64_t)M, (cuuint64_t)(K / lq::kBlockK)};
  const cuuint64_t strides[2] = {(cuuint64_t)K, (cuuint64_t)lq::kBlockK};
  const cuuint32_t box[3] = {(cuuint32_t)lq::kBlockK, (cuuint32_t)bt, (cuuint32_t)stages};
  const cuuint32_t estr[3] = {1, 1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void*>(x_q), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// ------------------------------------------------------------- schedule
enum SchedKind { kSchedAuto = 0, kSchedTiles = 1, kSchedPersistent = 2, kSchedStreamK = 3, kSchedPair = 4 };

struct Schedule {
  int kind = kSchedTiles;
  int bt = 0;        // tokens per tile
  int cs = 1;        // CTAs per tile in a cluster (split-K), 0 = stream-K
  int tiles_m = 0, tiles_n = 0, KB = 0;
  long long tiles = 0, U = 0;
  int grid = 0;
  bool split = false;  // stream-K: some tile is shared by several CTAs
  size_t ws_bytes = 0;
};

int auto_block_t(int M) {
  if (M <= 16) return 16;
  if (M <= 32) return 32;
  if (M <= 64) return 64;
  return 128;
}

bool valid_block_t(int bt) { return bt == 16 || bt == 32 || bt == 64 || bt == 128 || bt == 256; }

// largest cluster split instantiated for a tile width (shared-memory bound)
int max_split(int bt) { return bt <= 32 ? 8 : bt <= 128 ? 4 : 1; }

bool valid_split(int bt, int cs) { return (cs == 1 || cs == 2 || cs == 4 || cs == 8) && cs <= max_split(bt); }

bool pdl_enabled() {
  static const bool on = [] {
    const char* e = getenv("LQ_PDL");
    return !(e && e[0] == '0');
  }();
  return on;
}

bool valid_schedule(int M, int block_t, int schedule, int split_k, int grid) {
  if (block_t != 0 && !valid_block_t(block_t)) return false;
  if (split_k < 0 || grid < 0) return false;
  switch (schedule) {
    case kSchedAuto:
      return split_k == 0 && grid == 0;
    case kSchedTiles:
      return grid == 0 && (split_k == 0 || valid_split(block_t ? block_t : auto_block_t(M > 0 ? M : 1), split_k));
    case kSchedPersistent:
      return split_k == 0 && (block_t == 0 || block_t == lq::kPBT);
    case kSchedStreamK:
      return split_k == 0;
    case kSchedPair:
      return split_k == 0 && (block_t == 0 || block_t == lq::kQBT);
  }
  return false;
}

// shared-memory stages of the tile kernel for a token-tile size (one per
// preloaded K-block of 128)
int stages_of(int bt) {
  switch (bt) {
    case 16: return lq::GemmCfg<16, 1>::kStages;
    case 32: return lq::GemmCfg<32, 1>::kStages;
    case 64: return lq::GemmCfg<64, 1>::kStages;
    case 128: return lq::GemmCfg<128, 2>::kStages;
    default: return lq::GemmCfg<256, 1>::kStages;
  }
}

// whether two CTAs of the tile kernel fit one SM (shared memory and TMEM)
template <int BT, int CS>
bool fits_two_t() {
  using C = lq::GemmCfg<BT, CS>;
  return C::kTmemCols <= 256 && 2 * (C::kSmemBytes + 1024) <= 233472;
}
bool fits_two_per_sm(int bt, int cs) {
  switch (bt * 16 + cs) {
    case 16 * 16 + 2: return fits_two_t<16, 2>();
    case 16 * 16 + 4: return fits_two_t<16, 4>();
    case 16 * 16 + 8: return fits_two_t<16, 8>();
    case 32 * 16 + 2: return fits_two_t<32, 2>();
    case 32 * 16 + 4: return fits_two_t<32, 4>();
    case 32 * 16 + 8: return fits_two_t<32, 8>();
    case 64 * 16 + 2: return fits_two_t<64, 2>();
    case 64 * 16 + 4: return fits_two_t<64, 4>();
  }
  return false;
}

// CTAs of c-CTA clusters that fit at once, two per SM: from the device's table
// (cluster_fit) where there is one, else every SM counted
long long cluster_slots(int c, int sms, const int* cl) {
  const int i = c == 2 ? 0 : c == 4 ? 1 : c == 8 ? 2 : -1;
  return (cl != nullptr && i >= 0 && cl[i] > 0) ? std::min<long long>(cl[i], 2LL * sms) : 2LL * sms;
}

Schedule make_schedule(int M, int N, int K, int block_t, int schedule, int split_k, int grid, int sms,
                       const int* cl) {
  Schedule s;
  int kind = schedule;
  int bt = block_t ? block_t : auto_block_t(M);
  if (kind == kSchedAuto) {
    // more than 128 tokens and enough 256 x 256 tiles for half of the CTA
    // pairs: CTA pairs (a pair kernel tile costs about as much SM time as two
    // 128-token tiles of the persistent kernel, so it wins even when some
    // pairs stay idle); 128-token tiles too many to split K over two CTAs
    // each (so that a cluster schedule would give every CTA one whole tile):
    // persistent, whose 16 expansion warps per CTA are as fast there or
    // faster (measured on B200: 51.7 -> 49.1 us at 512 x 4096 x 14336, equal
    // at 128 x 14336 x 4096); otherwise one cluster per tile
    const long long t128 = (long long)((M + lq::kPBT - 1) / lq::kPBT) * ((N + lq::kBlockN - 1) / lq::kBlockN);
    const long long t256 = (long long)((M + lq::kQBT - 1) / lq::kQBT) * ((N + lq::kQBN - 1) / lq::kQBN);
    if (block_t == 0 && K % lq::kQBK == 0 && M > lq::kPBT && t256 >= sms / 4)
      kind = kSchedPair;
    else
      kind = (bt == lq::kPBT && 2 * t128 > sms) ? kSchedPersistent : kSchedTiles;
  }
  if (kind == kSchedPair) {
    s.kind = kind;
    s.bt = lq::kQBT;
    s.tiles_m = (M + lq::kQBT - 1) / lq::kQBT;
    s.tiles_n = (N + lq::kQBN - 1) / lq::kQBN;
    s.KB = K / lq::kBlockK;
    s.tiles = (long long)s.tiles_m * s.tiles_n;
    s.U = s.tiles;  // the pair kernel takes the tile count here
    long long pairs = grid > 0 ? (grid + 1) / 2 : sms / 2;
    if (pairs > s.tiles) pairs = s.tiles;
    if (pairs < 1) pairs = 1;
    s.cs = 2;
    s.grid = (int)(2 * pairs);
    return s;
  }
  if (kind == kSchedPersistent) bt = lq::kPBT;
  s.kind = kind;
  s.bt = bt;
  s.tiles_m = (M + s.bt - 1) / s.bt;
  s.tiles_n = (N + lq::kBlockN - 1) / lq::kBlockN;
  s.KB = K / lq::kBlockK;
  s.tiles = (long long)s.tiles_m * s.tiles_n;
  s.U = s.tiles * s.KB;
  if (kind == kSchedStreamK) {
    long long g = grid > 0 ? grid : sms;
    if (g > s.U) g = s.U;
    if (g > INT_MAX) g = INT_MAX;
    s.cs = 0;
    s.grid = (int)g;
    for (long long c = 1; c < g; ++c)
      if ((c * s.U / g) % s.KB != 0) {
        s.split = true;
        break;
      }
    if (s.split) {
      const size_t acc = (size_t)s.tiles * s.bt * lq::kBlockN * sizeof(int32_t);
      s.ws_bytes = acc + (((size_t)s.tiles * sizeof(unsigned) + 15) / 16) * 16;
    }
    return s;
  }
  if (kind == kSchedPersistent) {
    long long g = grid > 0 ? grid : sms;
    if (g > s.tiles) g = s.tiles;
    s.cs = 1;
    s.grid = (int)g;
    return s;
  }
  int cs = split_k;
  if (cs <= 0) {
    // one wave of one CTA per SM: as many CTAs per tile as fit, at least 4
    // K-blocks each.  That leaves room beside every CTA for one of the next
    // launch, which preloads its weights meanwhile.
    cs = 1;
    for (int c = max_split(s.bt); c >= 2; c /= 2)
      if (s.tiles * c <= sms && s.KB / c >= 4) {
        cs = c;
        break;
      }
    // When a CTA's K-slice is longer than its preloaded stages, the ring
    // streams the rest anyway and more CTAs stream faster: where two CTAs of
    // a wider split fit one SM, use that capacity -- as far as the device can
    // place clusters of that size.  One cluster more than fit starts a second
    // wave (measured on B200 at 16 x 4352 x 14336: 272 CTAs in 8-CTA
    // clusters, 18.3 us; 136 in 4-CTA clusters, 16.3 us; 16 x 4096 x 14336,
    // 256 CTAs in one wave, 11.5 us).
    if (s.KB / cs > stages_of(s.bt) && s.bt <= 64)
      for (int c = max_split(s.bt); c > cs; c /= 2)
        if (fits_two_per_sm(s.bt, c) && s.tiles * c <= cluster_slots(c, sms, cl) && s.KB / c >= 4) {
          cs = c;
          break;
        }
  }
  if (cs > s.KB) cs = 1;
  // 16-token tiles in 8-CTA clusters whose K-slices stream through the ring
  // run as 32-token tiles (the token tile count stays one): that
  // configuration has one TMEM slot per stage, so one commit per K-block
  // releases both (measured on B200: 12.2 -> 11.5 us at 16 x 4096 x 14336,
  // 11.9 -> 11.4 us at M = 1)
  if (block_t == 0 && split_k <= 0 && s.bt == 16 && cs == 8 && s.KB / cs > stages_of(16) && M <= 16) s.bt = 32;
  s.cs = cs;
  s.grid = (int)(s.tiles * cs);
  return s;
}

lq_status check_schedule_shape(const Schedule& s, int K) {
  if (s.kind == kSchedPair && K % lq::kQBK != 0) return LQ_ERR_UNSUPPORTED_SHAPE;
  return LQ_OK;
}

lq_status check_gemm_shape(int M, int N, int K, int group) {
  if (M < 0 || N < 0 || K < 0) return LQ_ERR_INVALID_ARG;
  if (group != LQ_GROUP) return LQ_ERR_UNSUPPORTED_SHAPE;
  if (K < lq::kBlockK || K % lq::kBlockK != 0 || K > 131072) return LQ_ERR_UNSUPPORTED_SHAPE;
  if (N < 16 || N % 16 != 0) return LQ_ERR_UNSUPPORTED_SHAPE;
  return LQ_OK;
}

template <typename Kern, typename... Args>
lq_status launch_ex(Kern kern, int grid, int block, int smem, int cluster, bool pdl, cudaStream_t st,
                    Args... args) {
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[2];
  int na = 0;
  if (cluster >= 2) {
    attr[na].id = cudaLaunchAttributeClusterDimension;
    attr[na].val.clusterDim.x = cluster;
    attr[na].val.clusterDim.y = 1;
    attr[na].val.clusterDim.z = 1;
    ++na;
  }
  if (pdl) {
    attr[na].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[na].val.programmaticStreamSerializationAllowed = 1;
    ++na;
  }
  cfg.gridDim = dim3(grid, 1, 1);
  cfg.blockDim = dim3(block, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cfg.attrs = attr;
  cfg.numAttrs = na;
  return cudaLaunchKernelEx(&cfg, kern, args...) == cudaSuccess ? LQ_OK : LQ_ERR_CUDA;
}

// The tile kernel's second activation map: for cluster schedules the 3D box of
// the first kStages K-blocks (make_map_x3), else a placeholder the kernel never
// reads.
template <int BT, int CS, int DQ>
bool make_tile_x3(CUtensorMap* tx3, const CUtensorMap& tx, const void* x_q, const lq::GemmArgs& a) {
  if constexpr (CS >= 1) {
    return make_map_x3(tx3, x_q, a.M, a.K, BT, lq::GemmCfg<BT, CS, DQ>::kStages);
  } else {
    *tx3 = tx;
    return true;
  }
}

// Output modes of the GEMM launches: bf16, int32 accumulators, or the SwiGLU
// of an interleaved gate/up pair (bf16, half the columns).
enum OutMode { kOutBf16 = 0, kOutI32 = 1, kOutSwiglu = 2 };

template <int BT, int CS, int OUT, int EG>
lq_status launch_gemm_tg(const Schedule& s, const CUtensorMap& tx, const void* x_q, const CUtensorMap& tw,
                         const CUtensorMap& ts, const CUtensorMap& ta, const lq::GemmArgs& a, cudaStream_t st) {
  using C = lq::GemmCfg<BT, CS>;
  auto kern = lq::w4a8_gemm_kernel<BT, CS, OUT == kOutI32, false, 0, EG, OUT == kOutSwiglu>;
  CUtensorMap tx3;
  if (!make_tile_x3<BT, CS, 0>(&tx3, tx, x_q, a)) return LQ_ERR_CUDA;
  // the attribute is per function and cheap; set it on every call so that any
  // device current at call time is covered
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemBytes) != cudaSuccess)
    return LQ_ERR_CUDA;
  return launch_ex(kern, s.grid, lq::gemm_threads(EG), C::kSmemBytes, CS, pdl_enabled(), st, tx, tx3, tw, ts, ta, a);
}

// Two expansion groups for 16-token cluster tiles whose CTAs preload every
// K-block of their slice (see gemm_threads in lq_gemm_kernel.cuh).
template <int BT, int CS, int OUT>
lq_status launch_gemm_t(const Schedule& s, const CUtensorMap& tx, const void* x_q, const CUtensorMap& tw,
                        const CUtensorMap& ts, const CUtensorMap& ta, const lq::GemmArgs& a, cudaStream_t st) {
  if constexpr (OUT == kOutSwiglu && CS == 0) {
    return LQ_ERR_UNSUPPORTED_SHAPE;  // the SwiGLU epilogue has no stream-K form
  } else {
    if constexpr (BT == 16 && CS >= 1) {
      if ((s.KB + CS - 1) / CS <= lq::GemmCfg<BT, CS>::kStages)
        return launch_gemm_tg<BT, CS, OUT, 2>(s, tx, x_q, tw, ts, ta, a, st);
    }
    return launch_gemm_tg<BT, CS, OUT, 1>(s, tx, x_q, tw, ts, ta, a, st);
  }
}

template <int BT, int OUT>
lq_status launch_gemm_bt(const Schedule& s, const CUtensorMap& tx, const void* x_q, const CUtensorMap& tw,
                         const CUtensorMap& ts, const CUtensorMap& ta, const lq::GemmArgs& a, cudaStream_t st) {
  switch (s.cs) {
    case 0: return launch_gemm_t<BT, 0, OUT>(s, tx, x_q, tw, ts, ta, a, st);
    case 1: return launch_gemm_t<BT, 1, OUT>(s, tx, x_q, tw, ts, ta, a, st);
    case 2:
      if constexpr (BT <= 128) return launch_gemm_t<BT, 2, OUT>(s, tx, x_q, tw, ts, ta, a, st);
      break;
    case 4:
      if constexpr (BT <= 128) return launch_gemm_t<BT, 4, OUT>(s, tx, x_q, tw, ts, ta, a, st);
      break;
    case 8:
      if constexpr (BT <= 32) return launch_gemm_t<BT, 8, OUT>(s, tx, x_q, tw, ts, ta, a, st);
      break;
  }
  return LQ_ERR_INVALID_ARG;
}

template <int OUT>
lq_status launch_gemm(const Schedule& s, const CUtensorMap& tx, const void* x_q, const CUtensorMap& tw,
                      const CUtensorMap& ts, const CUtensorMap& ta, const lq::GemmArgs& a, cudaStream_t st) {
  if (s.kind == kSchedPair) {
    auto kern = lq::w4a8_gemm_pair_kernel<OUT == kOutI32, OUT == kOutSwiglu>;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, lq::kQSmemBytes) != cudaSuccess)
      return LQ_ERR_CUDA;
    return launch_ex(kern, s.grid, lq::kQThreads, lq::kQSmemBytes, 2, pdl_enabled(), st, tx, tw, ts, ta, a);
  }
  if (s.kind == kSchedPersistent) {
    if constexpr (OUT == kOutSwiglu) return LQ_ERR_UNSUPPORTED_SHAPE;  // callers pick tiles instead
    auto kern = lq::w4a8_gemm_persistent_kernel<OUT == kOutI32>;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, lq::kPSmemBytes) != cudaSuccess)
      return LQ_ERR_CUDA;
    return launch_ex(kern, s.grid, lq::kPThreads, lq::kPSmemBytes, 1, pdl_enabled(), st, tx, tw, ts, ta, a);
  }
  switch (s.bt) {
    case 16: return launch_gemm_bt<16, OUT>(s, tx, x_q, tw, ts, ta, a, st);
    case 32: return launch_gemm_bt<32, OUT>(s, tx, x_q, tw, ts, ta, a, st);
    case 64: return launch_gemm_bt<64, OUT>(s, tx, x_q, tw, ts, ta, a, st);
    case 128: return launch_gemm_bt<128, OUT>(s, tx, x_q, tw, ts, ta, a, st);
    case 256: return launch_gemm_bt<256, OUT>(s, tx, x_q, tw, ts, ta, a, st);
  }
  return LQ_ERR_INVALID_ARG;
}

// The ablation of the dequantization pipeline (GemmCfg's DQ): the same tile
// kernel with per-element expansion (bit 0) and/or A expanded into shared
// memory (bit 1), for 16- and 64-token tiles in 4-CTA clusters.
template <int BT, int CS, bool I32, int DQ, int EG>
lq_status launch_abl_tg(const Schedule& s, const CUtensorMap& tx, const void* x_q, const CUtensorMap& tw,
                        const CUtensorMap& ts, const CUtensorMap& ta, const lq::GemmArgs& a, cudaStream_t st) {
  using C = lq::GemmCfg<BT, CS, DQ>;
  auto kern = lq::w4a8_gemm_kernel<BT, CS, I32, false, DQ, EG>;
  CUtensorMap tx3;
  if (!make_tile_x3<BT, CS, DQ>(&tx3, tx, x_q, a)) return LQ_ERR_CUDA;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemBytes) != cudaSuccess)
    return LQ_ERR_CUDA;
  return launch_ex(kern, s.grid, lq::gemm_threads(EG), C::kSmemBytes, CS, pdl_enabled(), st, tx, tx3, tw, ts, ta, a);
}

// the variants take the product kernel's expansion groups for the same shape
template <int BT, int CS, bool I32, int DQ>
lq_status launch_abl_t(const Schedule& s, const CUtensorMap& tx, const void* x_q, const CUtensorMap& tw,
                       const CUtensorMap& ts, const CUtensorMap& ta, const lq::GemmArgs& a, cudaStream_t st) {
  if constexpr (BT == 16) {
    if ((s.KB + CS - 1) / CS <= lq::GemmCfg<BT, CS, DQ>::kStages)
      return launch_abl_tg<BT, CS, I32, DQ, 2>(s, tx, x_q, tw, ts, ta, a, st);
  }
  return launch_abl_tg<BT, CS, I32, DQ, 1>(s, tx, x_q, tw, ts, ta, a, st);
}

template <bool I32>
lq_status launch_ablation(const Schedule& s, int dq, const CUtensorMap& tx, const void* x_q, const CUtensorMap& tw,
                          const CUtensorMap& ts, const CUtensorMap& ta, const lq::GemmArgs& a, cudaStream_t st) {
  if (dq == 0) return launch_gemm<I32 ? kOutI32 : kOutBf16>(s, tx, x_q, tw, ts, ta, a, st);
  if (s.kind != kSchedTiles || s.cs != 4) return LQ_ERR_UNSUPPORTED_SHAPE;
  switch (s.bt * 4 + dq) {
    case 16 * 4 + 1: return launch_abl_t<16, 4, I32, 1>(s, tx, x_q, tw, ts, ta, a, st);
    case 16 * 4 + 2: return launch_abl_t<16, 4, I32, 2>(s, tx, x_q, tw, ts, ta, a, st);
    case 16 * 4 + 3: return launch_abl_t<16, 4, I32, 3>(s, tx, x_q, tw, ts, ta, a, st);
    case 64 * 4 + 1: return launch_abl_t<64, 4, I32, 1>(s, tx, x_q, tw, ts, ta, a, st);
    case 64 * 4 + 2: return launch_abl_t<64, 4, I32, 2>(s, tx, x_q, tw, ts, ta, a, st);
    case 64 * 4 + 3: return launch_abl_t<64, 4, I32, 3>(s, tx, x_q, tw, ts, ta, a, st);
  }
  return LQ_ERR_UNSUPPORTED_SHAPE;
}

lq_status gemm_impl(const int8_t* x_q, const float* s_x, const uint8_t* qw, const uint8_t* s_u8,
                    const uint8_t* a_u8, const float* s_c, void* out, int M, int N, int K, int group,
                    void* workspace, size_t ws_bytes, int block_t, int schedule, int split_k, int grid,
                    bool out_i32, void* stream, int dq = 0, bool swiglu = false) {
  lq_status st = check_gemm_shape(M, N, K, group);
  if (st != LQ_OK) return st;
  if (!valid_schedule(M, block_t, schedule, split_k, grid)) return LQ_ERR_INVALID_ARG;
  if (M == 0) return LQ_OK;
  if (!x_q || !qw || !s_u8 || !a_u8 || !out || (!out_i32 && (!s_x || !s_c))) return LQ_ERR_INVALID_ARG;
  if (!aligned(x_q, 16) || !aligned(qw, 16) || !aligned(s_u8, 16) || !aligned(a_u8, 16) ||
      !aligned(out, 16) || (s_x && !aligned(s_x, 4)) || (s_c && !aligned(s_c, 4)))
    return LQ_ERR_MISALIGNED;
  DeviceInfo* dev = nullptr;
  st = current_device(&dev);
  if (st != LQ_OK) return st;
  if (!device_addressable(out)) return LQ_ERR_INVALID_ARG;
  Schedule s = make_schedule(M, N, K, block_t, schedule, split_k, grid, dev->sms, dev->cluster_ctas);
  if (swiglu) {
    // the SwiGLU epilogue runs on the tile kernel's cluster schedules and the
    // CTA-pair kernel: a persistent choice becomes one cluster per tile
    if (s.kind == kSchedStreamK || (s.kind == kSchedPersistent && schedule == kSchedPersistent))
      return LQ_ERR_UNSUPPORTED_SHAPE;
    if (s.kind == kSchedPersistent)
      s = make_schedule(M, N, K, lq::kPBT, kSchedTiles, 0, 0, dev->sms, dev->cluster_ctas);
  }
  st = check_schedule_shape(s, K);
  if (st != LQ_OK) return st;
  if (s.split) {
    if (!workspace || ws_bytes < s.ws_bytes) return LQ_ERR_WORKSPACE;
    if (!aligned(workspace, 16)) return LQ_ERR_MISALIGNED;
  }
  CUtensorMap tx, tw, ts, ta;
  // the pair kernel loads 128 tokens and 128 weight rows per CTA with 256 K per stage
  const bool pair = (s.kind == kSchedPair);
  const uint32_t x_rows = pair ? 128u : (uint32_t)s.bt;
  const uint32_t w_box = pair ? (uint32_t)lq::kQBK / 2 : (uint32_t)lq::kBlockK / 2;
  const uint32_t sa_groups = pair ? (uint32_t)lq::kQBK / LQ_GROUP : 2u;
  if (!make_map_u8(&tx, x_q, (uint64_t)K, (uint64_t)M, (uint64_t)K, lq::kBlockK, x_rows,
                   CU_TENSOR_MAP_SWIZZLE_128B) ||
      !make_map_u8(&tw, qw, (uint64_t)K / 2, (uint64_t)N, (uint64_t)K / 2, w_box, lq::kBlockN,
                   pair ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B) ||
      !make_map_u8(&ts, s_u8, (uint64_t)N, (uint64_t)K / LQ_GROUP, (uint64_t)N, lq::kBlockN, sa_groups,
                   CU_TENSOR_MAP_SWIZZLE_NONE) ||
      !make_map_u8(&ta, a_u8, (uint64_t)N, (uint64_t)K / LQ_GROUP, (uint64_t)N, lq::kBlockN, sa_groups,
                   CU_TENSOR_MAP_SWIZZLE_NONE))
    return LQ_ERR_CUDA;
  lq::GemmArgs a;
  a.x_bf16 = nullptr;
  a.s_x = s_x;
  a.s_c = s_c;
  a.out = out;
  a.ws = s.split ? static_cast<int32_t*>(workspace) : nullptr;
  a.ticket = s.split ? reinterpret_cast<unsigned int*>(static_cast<uint8_t*>(workspace) +
                                                        (size_t)s.tiles * s.bt * lq::kBlockN * 4)
                     : nullptr;
  a.M = M;
  a.N = N;
  a.K = K;
  a.tiles_m = s.tiles_m;
  a.KB = s.KB;
  a.U = s.U;
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  if (dq != 0)
    return out_i32 ? launch_ablation<true>(s, dq, tx, x_q, tw, ts, ta, a, cs)
                   : launch_ablation<false>(s, dq, tx, x_q, tw, ts, ta, a, cs);
  if (swiglu) return launch_gemm<kOutSwiglu>(s, tx, x_q, tw, ts, ta, a, cs);
  return out_i32 ? launch_gemm<kOutI32>(s, tx, x_q, tw, ts, ta, a, cs)
                 : launch_gemm<kOutBf16>(s, tx, x_q, tw, ts, ta, a, cs);
}

// ---------------------------------------- fused activation quantization
// One launch does act-quant + GEMM when the automatic schedule is a split-K
// cluster of 16-token tiles whose CTAs preload all of their K-blocks: every
// CTA then holds its whole K-slice of the activations and the row maxima can
// be combined over the cluster (see the FQ notes in lq_gemm_kernel.cuh).
bool fused_eligible(const Schedule& s, int M) {
  if (M < 1 || M > 16 || s.kind != kSchedTiles || s.bt != 16 || s.cs < 2) return false;
  const int per_cta = (s.KB + s.cs - 1) / s.cs;  // the largest K-slice, in K-blocks
  return per_cta <= lq::GemmCfg<16, 2>::kStages;
}

// The automatic choice: the four quantizing warps of a CTA take M/4 tokens
// each, so the fused launch wins only while M is small (measured on B200 at
// N = K = 4096: ahead up to M = 8, behind from M = 12).
constexpr int kFusedAutoMaxM = 8;

bool use_fused(const Schedule& s, int M, int path) {
  if (path == LQ_LINEAR_TWO_LAUNCHES) return false;
  if (!fused_eligible(s, M)) return false;
  return path == LQ_LINEAR_FUSED || M <= kFusedAutoMaxM;
}

template <int CS>
lq_status launch_fused_t(const Schedule& s, const CUtensorMap& tw, const CUtensorMap& ts, const CUtensorMap& ta,
                         const lq::GemmArgs& a, cudaStream_t st) {
  using C = lq::GemmCfg<16, CS>;
  auto kern = lq::w4a8_gemm_kernel<16, CS, false, true>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemBytes) != cudaSuccess)
    return LQ_ERR_CUDA;
  // no activation tensor maps: the weight map stands in for them (never used)
  return launch_ex(kern, s.grid, lq::gemm_threads(1), C::kSmemBytes, CS, pdl_enabled(), st, tw, tw, tw, ts, ta, a);
}

size_t align16(size_t b) { return (b + 15) / 16 * 16; }

}  // namespace

extern "C" {

size_t lq_w4a8_linear_workspace_size_ex(int M, int N, int K, int path) {
  if (check_gemm_shape(M, N, K, LQ_GROUP) != LQ_OK || M == 0) return 0;
  if (path < LQ_LINEAR_AUTO || path > LQ_LINEAR_FUSED) return 0;
  DeviceInfo* dev = nullptr;
  int sms = 148;
  const int* cl = nullptr;
  if (current_device(&dev) == LQ_OK) {
    sms = dev->sms;
    cl = dev->cluster_ctas;
  }
  const Schedule s = make_schedule(M, N, K, 0, 0, 0, 0, sms, cl);
  if (use_fused(s, M, path)) return 0;
  return align16((size_t)M * K) + align16((size_t)M * 4) + s.ws_bytes;
}

size_t lq_w4a8_linear_workspace_size(int M, int N, int K) {
  return lq_w4a8_linear_workspace_size_ex(M, N, K, LQ_LINEAR_AUTO);
}

lq_status lq_w4a8_linear(const void* X_bf16, const uint8_t* qw, const uint8_t* s_u8, const uint8_t* a_u8,
                         const float* s_c, void* out_bf16, int M, int N, int K, int group, void* workspace,
                         size_t workspace_bytes, void* stream) {
  return lq_w4a8_linear_ex(X_bf16, qw, s_u8, a_u8, s_c, out_bf16, M, N, K, group, workspace, workspace_bytes,
                           LQ_LINEAR_AUTO, stream);
}

lq_status lq_w4a8_linear_ex(const void* X_bf16, const uint8_t* qw, const uint8_t* s_u8, const uint8_t* a_u8,
                            const float* s_c, void* out_bf16, int M, int N, int K, int group, void* workspace,
                            size_t workspace_bytes, int path, void* stream) {
  lq_status st = check_gemm_shape(M, N, K, group);
  if (st != LQ_OK) return st;
  if (path < LQ_LINEAR_AUTO || path > LQ_LINEAR_FUSED) return LQ_ERR_INVALID_ARG;
  if (M == 0) return LQ_OK;
  if (!X_bf16 || !qw || !s_u8 || !a_u8 || !s_c || !out_bf16) return LQ_ERR_INVALID_ARG;
  if (!aligned(X_bf16, 16) || !aligned(qw, 16) || !aligned(s_u8, 16) || !aligned(a_u8, 16) ||
      !aligned(out_bf16, 16) || !aligned(s_c, 4))
    return LQ_ERR_MISALIGNED;
  DeviceInfo* dev = nullptr;
  st = current_device(&dev);
  if (st != LQ_OK) return st;
  if (!device_addressable(X_bf16) || !device_addressable(out_bf16)) return LQ_ERR_INVALID_ARG;
  const Schedule s = make_schedule(M, N, K, 0, 0, 0, 0, dev->sms, dev->cluster_ctas);
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  if (path == LQ_LINEAR_FUSED && !fused_eligible(s, M)) return LQ_ERR_UNSUPPORTED_SHAPE;
  if (!use_fused(s, M, path)) {
    // two launches: activations into the workspace, then the GEMM
    const size_t xq_bytes = align16((size_t)M * K), sx_bytes = align16((size_t)M * 4);
    if (!workspace || workspace_bytes < xq_bytes + sx_bytes + s.ws_bytes) return LQ_ERR_WORKSPACE;
    if (!aligned(workspace, 16)) return LQ_ERR_MISALIGNED;
    uint8_t* w = static_cast<uint8_t*>(workspace);
    int8_t* x_q = reinterpret_cast<int8_t*>(w);
    float* s_x = reinterpret_cast<float*>(w + xq_bytes);
    st = lq_quantize_act(X_bf16, M, K, x_q, s_x, stream);
    if (st != LQ_OK) return st;
    return gemm_impl(x_q, s_x, qw, s_u8, a_u8, s_c, out_bf16, M, N, K, group, w + xq_bytes + sx_bytes,
                     workspace_bytes - xq_bytes - sx_bytes, 0, 0, 0, 0, false, stream);
  }
  CUtensorMap tw, ts, ta;
  if (!make_map_u8(&tw, qw, (uint64_t)K / 2, (uint64_t)N, (uint64_t)K / 2, lq::kBlockK / 2, lq::kBlockN,
                   CU_TENSOR_MAP_SWIZZLE_64B) ||
      !make_map_u8(&ts, s_u8, (uint64_t)N, (uint64_t)K / LQ_GROUP, (uint64_t)N, lq::kBlockN, 2u,
                   CU_TENSOR_MAP_SWIZZLE_NONE) ||
      !make_map_u8(&ta, a_u8, (uint64_t)N, (uint64_t)K / LQ_GROUP, (uint64_t)N, lq::kBlockN, 2u,
                   CU_TENSOR_MAP_SWIZZLE_NONE))
    return LQ_ERR_CUDA;
  lq::GemmArgs a;
  a.x_bf16 = static_cast<const uint16_t*>(X_bf16);
  a.s_x = nullptr;
  a.s_c = s_c;
  a.out = out_bf16;
  a.ws = nullptr;
  a.ticket = nullptr;
  a.M = M;
  a.N = N;
  a.K = K;
  a.tiles_m = s.tiles_m;
  a.KB = s.KB;
  a.U = s.U;
  switch (s.cs) {
    case 2: return launch_fused_t<2>(s, tw, ts, ta, a, cs);
    case 4: return launch_fused_t<4>(s, tw, ts, ta, a, cs);
    case 8: return launch_fused_t<8>(s, tw, ts, ta, a, cs);
  }
  return LQ_ERR_INVALID_ARG;
}

}  // extern "C"

extern "C" {

int lq_version(void) { return 100; }

int lq_device_addressable(const void* p) {
  DeviceInfo* dev = nullptr;
  if (p == nullptr || current_device(&dev) != LQ_OK) return 0;
  return device_addressable(p) ? 1 : 0;
}

const char* lq_status_string(lq_status status) {
  switch (status) {
    case LQ_OK: return "LQ_OK";
    case LQ_ERR_INVALID_ARG: return "LQ_ERR_INVALID_ARG: invalid argument";
    case LQ_ERR_UNSUPPORTED_SHAPE: return "LQ_ERR_UNSUPPORTED_SHAPE: unsupported shape or group size";
    case LQ_ERR_MISALIGNED: return "LQ_ERR_MISALIGNED: pointer not aligned as required";
    case LQ_ERR_WORKSPACE: return "LQ_ERR_WORKSPACE: workspace missing or too small";
    case LQ_ERR_CUDA: return "LQ_ERR_CUDA: a CUDA call failed";
    case LQ_ERR_TIMEOUT: return "LQ_ERR_TIMEOUT: a device-side wait gave up";
    case LQ_ERR_ARCH: return "LQ_ERR_ARCH: device is not compute capability 10.0";
  }
  return "unknown lq_status";
}

lq_status lq_quantize_weights(const void* W_bf16, int N, int K, int group, uint8_t* qw, uint8_t* s_u8,
                              uint8_t* a_u8, float* s_c, void* stream) {
  if (N < 0 || K < 0) return LQ_ERR_INVALID_ARG;
  if (group != LQ_GROUP || K < LQ_GROUP || K % LQ_GROUP != 0 || N < 1) return LQ_ERR_UNSUPPORTED_SHAPE;
  if (!W_bf16 || !qw || !s_u8 || !a_u8 || !s_c) return LQ_ERR_INVALID_ARG;
  if (!aligned(W_bf16, 16) || !aligned(qw, 16) || !aligned(s_c, 4)) return LQ_ERR_MISALIGNED;
  DeviceInfo* dev = nullptr;
  lq_status st = current_device(&dev);
  if (st != LQ_OK) return st;
  lq::quantize_weights_kernel<<<N, lq::kQuantWThreads, 0, static_cast<cudaStream_t>(stream)>>>(
      static_cast<const uint16_t*>(W_bf16), N, K, qw, s_u8, a_u8, s_c);
  return cudaGetLastError() == cudaSuccess ? LQ_OK : LQ_ERR_CUDA;
}

lq_status lq_quantize_act(const void* X_bf16, int M, int K, int8_t* x_q, float* s_x, void* stream) {
  if (M < 0 || K < 0) return LQ_ERR_INVALID_ARG;
  if (K < 16 || K % 16 != 0) return LQ_ERR_UNSUPPORTED_SHAPE;
  if (M == 0) return LQ_OK;
  if (!X_bf16 || !x_q || !s_x) return LQ_ERR_INVALID_ARG;
  if (!aligned(X_bf16, 16) || !aligned(x_q, 16) || !aligned(s_x, 4)) return LQ_ERR_MISALIGNED;
  DeviceInfo* dev = nullptr;
  lq_status st = current_device(&dev);
  if (st != LQ_OK) return st;
  if (!device_addressable(X_bf16)) return LQ_ERR_INVALID_ARG;
  return launch_ex(lq::quantize_act_kernel, M, lq::kQuantActThreads, 0, 1, pdl_enabled(),
                   static_cast<cudaStream_t>(stream), static_cast<const uint16_t*>(X_bf16), K, x_q, s_x);
}

size_t lq_w4a8_gemm_workspace_size_ex(int M, int N, int K, int block_t, int schedule, int split_k, int grid) {
  if (check_gemm_shape(M, N, K, LQ_GROUP) != LQ_OK || M == 0) return 0;
  if (!valid_schedule(M, block_t, schedule, split_k, grid)) return 0;
  DeviceInfo* dev = nullptr;
  int sms = 148;
  const int* cl = nullptr;
  if (current_device(&dev) == LQ_OK) {
    sms = dev->sms;
    cl = dev->cluster_ctas;
  }
  return make_schedule(M, N, K, block_t, schedule, split_k, grid, sms, cl).ws_bytes;
}

size_t lq_w4a8_gemm_workspace_size(int M, int N, int K) {
  return lq_w4a8_gemm_workspace_size_ex(M, N, K, 0, 0, 0, 0);
}

lq_status lq_w4a8_gemm_ex(const int8_t* x_q, const float* s_x, const uint8_t* qw, const uint8_t* s_u8,
                          const uint8_t* a_u8, const float* s_c, void* out, int M, int N, int K, int group,
                          void* workspace, size_t workspace_bytes, int block_t, int schedule, int split_k,
                          int grid, int out_i32, void* stream) {
  return gemm_impl(x_q, s_x, qw, s_u8, a_u8, s_c, out, M, N, K, group, workspace, workspace_bytes, block_t,
                   schedule, split_k, grid, out_i32 != 0, stream);
}

lq_status lq_w4a8_gemm(const int8_t* x_q, const float* s_x, const uint8_t* qw, const uint8_t* s_u8,
                       const uint8_t* a_u8, const float* s_c, void* out_bf16, int M, int N, int K, int group,
                       void* workspace, size_t workspace_bytes, void* stream) {
  return gemm_impl(x_q, s_x, qw, s_u8, a_u8, s_c, out_bf16, M, N, K, group, workspace, workspace_bytes, 0, 0,
                   0, 0, false, stream);
}

lq_status lq_w4a8_gemm_swiglu(const int8_t* x_q, const float* s_x, const uint8_t* qw, const uint8_t* s_u8,
                              const uint8_t* a_u8, const float* s_c, void* out_bf16, int M, int N, int K, int group,
                              void* workspace, size_t workspace_bytes, void* stream) {
  return gemm_impl(x_q, s_x, qw, s_u8, a_u8, s_c, out_bf16, M, N, K, group, workspace, workspace_bytes, 0, 0, 0, 0,
                   false, stream, 0, true);
}

lq_status lq_w4a8_gemm_swiglu_ex(const int8_t* x_q, const float* s_x, const uint8_t* qw, const uint8_t* s_u8,
                                 const uint8_t* a_u8, const float* s_c, void* out_bf16, int M, int N, int K, int group,
                                 void* workspace, size_t workspace_bytes, int block_t, int schedule, int split_k,
                                 int grid, void* stream) {
  return gemm_impl(x_q, s_x, qw, s_u8, a_u8, s_c, out_bf16, M, N, K, group, workspace, workspace_bytes, block_t,
                   schedule, split_k, grid, false, stream, 0, true);
}

lq_status lq_w4a8_gemm_i32(const int8_t* x_q, const uint8_t* qw, const uint8_t* s_u8, const uint8_t* a_u8,
                           int32_t* acc, int M, int N, int K, int group, void* workspace,
                           size_t workspace_bytes, void* stream) {
  return gemm_impl(x_q, nullptr, qw, s_u8, a_u8, nullptr, acc, M, N, K, group, workspace, workspace_bytes, 0,
                   0, 0, 0, true, stream);
}

lq_status lq_plan_gemm_ex(int M, int N, int K, int block_t, int schedule, int split_k, int grid, int sms,
                          const int* cluster_ctas, int* plan) {
  if (!plan || sms < 1) return LQ_ERR_INVALID_ARG;
  if (cluster_ctas)
    for (int i = 0; i < 3; ++i)
      if (cluster_ctas[i] < 1) return LQ_ERR_INVALID_ARG;
  lq_status st = check_gemm_shape(M, N, K, LQ_GROUP);
  if (st != LQ_OK) return st;
  if (M < 1 || !valid_schedule(M, block_t, schedule, split_k, grid)) return LQ_ERR_INVALID_ARG;
  const Schedule s = make_schedule(M, N, K, block_t, schedule, split_k, grid, sms, cluster_ctas);
  st = check_schedule_shape(s, K);
  if (st != LQ_OK) return st;
  plan[0] = s.kind;
  plan[1] = s.bt;
  plan[2] = s.cs;
  plan[3] = s.grid;
  return LQ_OK;
}

lq_status lq_plan_gemm(int M, int N, int K, int block_t, int schedule, int split_k, int grid, int sms, int* plan) {
  return lq_plan_gemm_ex(M, N, K, block_t, schedule, split_k, grid, sms, nullptr, plan);
}

lq_status lq_device_cluster_ctas(int* cluster_ctas) {
  if (!cluster_ctas) return LQ_ERR_INVALID_ARG;
  DeviceInfo* dev = nullptr;
  const lq_status st = current_device(&dev);
  if (st != LQ_OK) return st;
  for (int i = 0; i < 3; ++i) cluster_ctas[i] = dev->cluster_ctas[i];
  return LQ_OK;
}

lq_status lq_w4a8_gemm_ablation(const int8_t* x_q, const float* s_x, const uint8_t* qw, const uint8_t* s_u8,
                                const uint8_t* a_u8, const float* s_c, void* out, int M, int N, int K, int group,
                                int variant, int block_t, int split_k, int out_i32, void* stream) {
  if (variant < LQ_ABL_IMPLICIT || variant > LQ_ABL_NAIVE_EXPLICIT) return LQ_ERR_INVALID_ARG;
  if ((block_t != 16 && block_t != 64) || split_k != 4) return LQ_ERR_UNSUPPORTED_SHAPE;
  return gemm_impl(x_q, s_x, qw, s_u8, a_u8, s_c, out, M, N, K, group, nullptr, 0, block_t, kSchedTiles, split_k,
                   0, out_i32 != 0, stream, variant);
}

lq_status lq_dequant_weights_i8(const uint8_t* qw, const uint8_t* s_u8, const uint8_t* a_u8, int N, int K,
                                int group, int8_t* w_i8, void* stream) {
  if (N < 0 || K < 0) return LQ_ERR_INVALID_ARG;
  if (group != LQ_GROUP || K < LQ_GROUP || K % LQ_GROUP != 0 || N < 1) return LQ_ERR_UNSUPPORTED_SHAPE;
  if (!qw || !s_u8 || !a_u8 || !w_i8) return LQ_ERR_INVALID_ARG;
  if (!aligned(qw, 16) || !aligned(w_i8, 16)) return LQ_ERR_MISALIGNED;
  DeviceInfo* dev = nullptr;
  lq_status st = current_device(&dev);
  if (st != LQ_OK) return st;
  const long long words = (long long)N * (K / 8);
  const int threads = 256;
  const long long blocks = (words + threads - 1) / threads;
  if (blocks > INT_MAX) return LQ_ERR_UNSUPPORTED_SHAPE;
  lq::dequant_weights_kernel<<<(int)blocks, threads, 0, static_cast<cudaStream_t>(stream)>>>(
      reinterpret_cast<const uint32_t*>(qw), s_u8, a_u8, N, K, reinterpret_cast<uint32_t*>(w_i8));
  return cudaGetLastError() == cudaSuccess ? LQ_OK : LQ_ERR_CUDA;
}

lq_status lq_test_wait_timeout(void* stream) {
  DeviceInfo* dev = nullptr;
  const lq_status st = current_device(&dev);
  if (st != LQ_OK) return st;
  lq::wait_timeout_kernel<<<1, 64, 0, static_cast<cudaStream_t>(stream)>>>();
  return cudaGetLastError() == cudaSuccess ? LQ_OK : LQ_ERR_CUDA;
}

lq_status lq_get_device_error(void* stream) {
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return LQ_ERR_CUDA;
  unsigned int code = 0;
  if (cudaMemcpyFromSymbol(&code, lq::g_error, sizeof code) != cudaSuccess) return LQ_ERR_CUDA;
  if (code != 0) {
    const unsigned int zero = 0;
    if (cudaMemcpyToSymbol(lq::g_error, &zero, sizeof zero) != cudaSuccess) return LQ_ERR_CUDA;
    return code == lq::kErrTimeout ? LQ_ERR_TIMEOUT : LQ_ERR_CUDA;
  }
  return LQ_OK;
}

}  // extern "C"

// ---------------------------------------------------------------------------
// Allocation-free GEMM.
//
// Some callers may not allocate device memory on the path that launches the
// GEMM: a serving framework's per-request enqueue hook (the framework owns all
// device memory and does not expect a library to call cudaMalloc there), or a
// latency-critical loop that must not block on the driver's allocator or fail
// on an out-of-memory error mid-request.  lq_w4a8_gemm_noalloc serves them: it
// runs the stream-K schedule with its int32 partial sums and tile tickets in
// the fixed array below instead of a caller-provided workspace.
//
// The array is part of the library image: every GPU on which the library is
// loaded holds these kNoAllocScratchBytes until the process exits.  All calls
// on a device share it, so two calls that overlap on the GPU (different
// streams, or one stream racing another) corrupt each other's sums; callers
// must order them, e.g. on a single stream.
// ---------------------------------------------------------------------------
namespace {

constexpr size_t kNoAllocScratchBytes = size_t(4) << 20;  // 4 MiB per device
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

// Device address of g_noalloc_scratch, resolved once per device.  In host code
// the array's name only stands for the symbol; kernels must be given this
// address.  The entries are atomics: a thread may read one while another
// publishes it under the mutex (acquire load, release store).
std::atomic<void*> g_noalloc_addr[kMaxDevices] = {};
std::mutex g_noalloc_mu;

lq_status noalloc_scratch(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return LQ_ERR_CUDA;
  void* p = g_noalloc_addr[dev].load(std::memory_order_acquire);
  if (!p) {
    std::lock_guard<std::mutex> lk(g_noalloc_mu);
    p = g_noalloc_addr[dev].load(std::memory_order_relaxed);
    if (!p) {
      if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) return LQ_ERR_CUDA;
      g_noalloc_addr[dev].store(p, std::memory_order_release);
    }
  }
  *out = p;
  return LQ_OK;
}

}  // namespace

extern "C" {

lq_status lq_w4a8_gemm_noalloc(const int8_t* x_q, const float* s_x, const uint8_t* qw, const uint8_t* s_u8,
                               const uint8_t* a_u8, const float* s_c, void* out_bf16, int M, int N, int K,
                               int group, void* stream) {
  lq_status st = check_gemm_shape(M, N, K, group);
  if (st != LQ_OK) return st;
  if (M == 0) return LQ_OK;
  if (!x_q || !qw || !s_u8 || !a_u8 || !out_bf16 || !s_x || !s_c) return LQ_ERR_INVALID_ARG;
  DeviceInfo* dev = nullptr;
  st = current_device(&dev);
  if (st != LQ_OK) return st;
  const Schedule s = make_schedule(M, N, K, 0, kSchedStreamK, 0, 0, dev->sms, dev->cluster_ctas);
  if (s.ws_bytes > kNoAllocScratchBytes) return LQ_ERR_WORKSPACE;
  void* scratch = nullptr;
  st = noalloc_scratch(&scratch);
  if (st != LQ_OK) return st;
  // the partial sums and tickets start from zero on every call, whatever an
  // earlier (possibly failed) call left behind
  if (s.ws_bytes != 0 &&
      cudaMemsetAsync(scratch, 0, s.ws_bytes, static_cast<cudaStream_t>(stream)) != cudaSuccess)
    return LQ_ERR_CUDA;
  return gemm_impl(x_q, s_x, qw, s_u8, a_u8, s_c, out_bf16, M, N, K, group, scratch, kNoAllocScratchBytes, 0,
                   kSchedStreamK, 0, 0, false, stream);
}

}  // extern "C"

// ------------------------------------------------------------ grouped GEMM
// Mixture-of-experts layers: every group (expert) has its own N x K weights,
// stacked as one [groups * N, K] matrix quantized in one call, and its own
// contiguous run of token rows.  One cluster per tile, as in the tile
// schedule; the token tiles of all groups are enumerated from a bound that
// needs no device data, and each cluster finds its group from the row
// offsets on the device.
namespace {

lq_status grouped_impl(const int8_t* x_q, const float* s_x, const uint8_t* qw, const uint8_t* s_u8,
                       const uint8_t* a_u8, const float* s_c, const int* m_off, int groups, void* out, int M, int N,
                       int K, int group, int block_t, int split_k, bool out_i32, void* stream) {
  lq_status st = check_gemm_shape(M, N, K, group);
  if (st != LQ_OK) return st;
  if (N % lq::kBlockN != 0) return LQ_ERR_UNSUPPORTED_SHAPE;  // a weight tile never spans two groups
  if (groups < 1 || groups > LQ_MAX_GROUPS || (long long)groups * N > INT_MAX) return LQ_ERR_INVALID_ARG;
  if (block_t != 0 && !valid_block_t(block_t)) return LQ_ERR_INVALID_ARG;
  if (split_k < 0 || (block_t == 256 && split_k > 0)) return LQ_ERR_INVALID_ARG;
  // 256-token tiles are the CTA-pair kernel's (256 weight rows, 256 K per stage)
  if (block_t == 256 && (N % lq::kQBN != 0 || K % lq::kQBK != 0)) return LQ_ERR_UNSUPPORTED_SHAPE;
  if (M == 0) return LQ_OK;
  if (!x_q || !qw || !s_u8 || !a_u8 || !out || !m_off || (!out_i32 && (!s_x || !s_c))) return LQ_ERR_INVALID_ARG;
  if (!aligned(x_q, 16) || !aligned(qw, 16) || !aligned(s_u8, 16) || !aligned(a_u8, 16) || !aligned(out, 16) ||
      !aligned(m_off, 4) || (s_x && !aligned(s_x, 4)) || (s_c && !aligned(s_c, 4)))
    return LQ_ERR_MISALIGNED;
  // CTA pairs when the groups average more than 128 rows and the shape allows
  // 256 x 256 tiles; else the tile kernel, its token tile from the mean rows
  // per group.  The token tiles of all groups number at most
  // sum(ceil(M_e / bt)) <= (M + groups (bt - 1)) / bt, and at most M.
  const bool pair = block_t == 256 || (block_t == 0 && split_k == 0 && N % lq::kQBN == 0 &&
                                       K % lq::kQBK == 0 && (long long)M > (long long)groups * lq::kPBT);
  const int bt = pair ? lq::kQBT : block_t ? block_t : auto_block_t((M + groups - 1) / groups);
  if (split_k > 0 && !valid_split(bt, split_k)) return LQ_ERR_INVALID_ARG;
  DeviceInfo* dev = nullptr;
  st = current_device(&dev);
  if (st != LQ_OK) return st;
  if (!device_addressable(out)) return LQ_ERR_INVALID_ARG;
  const long long tm_bound = std::min<long long>(((long long)M + (long long)groups * (bt - 1)) / bt, M);
  if (tm_bound * bt > INT_MAX) return LQ_ERR_UNSUPPORTED_SHAPE;
  const Schedule s =
      pair ? make_schedule((int)(tm_bound * bt), N, K, 0, kSchedPair, 0, 0, dev->sms, dev->cluster_ctas)
           : make_schedule((int)(tm_bound * bt), N, K, bt, kSchedTiles, split_k, 0, dev->sms, dev->cluster_ctas);
  const int NT = groups * N;
  // the pair kernel loads 128 tokens and 128 weight rows per CTA with 256 K per stage
  const uint32_t x_rows = pair ? 128u : (uint32_t)bt;
  const uint32_t w_box = pair ? (uint32_t)lq::kQBK / 2 : (uint32_t)lq::kBlockK / 2;
  const uint32_t sa_groups = pair ? (uint32_t)lq::kQBK / LQ_GROUP : 2u;
  CUtensorMap tx, tw, ts, ta;
  if (!make_map_u8(&tx, x_q, (uint64_t)K, (uint64_t)M, (uint64_t)K, lq::kBlockK, x_rows,
                   CU_TENSOR_MAP_SWIZZLE_128B) ||
      !make_map_u8(&tw, qw, (uint64_t)K / 2, (uint64_t)NT, (uint64_t)K / 2, w_box, lq::kBlockN,
                   pair ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B) ||
      !make_map_u8(&ts, s_u8, (uint64_t)NT, (uint64_t)K / LQ_GROUP, (uint64_t)NT, lq::kBlockN, sa_groups,
                   CU_TENSOR_MAP_SWIZZLE_NONE) ||
      !make_map_u8(&ta, a_u8, (uint64_t)NT, (uint64_t)K / LQ_GROUP, (uint64_t)NT, lq::kBlockN, sa_groups,
                   CU_TENSOR_MAP_SWIZZLE_NONE))
    return LQ_ERR_CUDA;
  lq::GemmArgs a;
  a.x_bf16 = nullptr;
  a.s_x = s_x;
  a.s_c = s_c;
  a.out = out;
  a.ws = nullptr;
  a.ticket = nullptr;
  a.M = M;
  a.N = N;
  a.K = K;
  a.tiles_m = s.tiles_m;
  a.KB = s.KB;
  a.U = s.U;
  a.m_off = m_off;
  a.groups = groups;
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  return out_i32 ? launch_gemm<kOutI32>(s, tx, x_q, tw, ts, ta, a, cs)
                 : launch_gemm<kOutBf16>(s, tx, x_q, tw, ts, ta, a, cs);
}

}  // namespace

extern "C" {

lq_status lq_w4a8_grouped_gemm_ex(const int8_t* x_q, const float* s_x, const uint8_t* qw, const uint8_t* s_u8,
                                  const uint8_t* a_u8, const float* s_c, const int* m_off, int groups, void* out,
                                  int M, int N, int K, int group, int block_t, int split_k, int out_i32,
                                  void* stream) {
  return grouped_impl(x_q, s_x, qw, s_u8, a_u8, s_c, m_off, groups, out, M, N, K, group, block_t, split_k,
                      out_i32 != 0, stream);
}

lq_status lq_w4a8_grouped_gemm(const int8_t* x_q, const float* s_x, const uint8_t* qw, const uint8_t* s_u8,
                               const uint8_t* a_u8, const float* s_c, const int* m_off, int groups, void* out_bf16,
                               int M, int N, int K, int group, void* stream) {
  return grouped_impl(x_q, s_x, qw, s_u8, a_u8, s_c, m_off, groups, out_bf16, M, N, K, group, 0, 0, false, stream);
}

}  // extern "C"

// ------------------------------------------------------------ W4 x FP8
namespace {

// The tile kernel's KIND 1 on its cluster schedules: 16-, 64- or 128-token
// tiles, the split and the expansion groups chosen as for W4A8.  The weight
// map stands in for the scale / offset maps, which KIND 1 never reads.
template <int BT, int CS, int EG>
lq_status launch_f8_tg(const Schedule& s, const CUtensorMap& tx, const void* x_f8, const CUtensorMap& tw,
                       const lq::GemmArgs& a, cudaStream_t st) {
  using C = lq::GemmCfg<BT, CS>;
  auto kern = lq::w4a8_gemm_kernel<BT, CS, false, false, 0, EG, false, 1>;
  CUtensorMap tx3;
  if (!make_tile_x3<BT, CS, 0>(&tx3, tx, x_f8, a)) return LQ_ERR_CUDA;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemBytes) != cudaSuccess)
    return LQ_ERR_CUDA;
  return launch_ex(kern, s.grid, lq::gemm_threads(EG), C::kSmemBytes, CS, pdl_enabled(), st, tx, tx3, tw, tw, tw, a);
}

template <int BT, int CS>
lq_status launch_f8_t(const Schedule& s, const CUtensorMap& tx, const void* x_f8, const CUtensorMap& tw,
                      const lq::GemmArgs& a, cudaStream_t st) {
  if constexpr (BT == 16) {
    if ((s.KB + CS - 1) / CS <= lq::GemmCfg<BT, CS>::kStages) return launch_f8_tg<BT, CS, 2>(s, tx, x_f8, tw, a, st);
  }
  return launch_f8_tg<BT, CS, 1>(s, tx, x_f8, tw, a, st);
}

template <int BT>
lq_status launch_f8_bt(const Schedule& s, const CUtensorMap& tx, const void* x_f8, const CUtensorMap& tw,
                       const lq::GemmArgs& a, cudaStream_t st) {
  switch (s.cs) {
    case 1: return launch_f8_t<BT, 1>(s, tx, x_f8, tw, a, st);
    case 2: return launch_f8_t<BT, 2>(s, tx, x_f8, tw, a, st);
    case 4: return launch_f8_t<BT, 4>(s, tx, x_f8, tw, a, st);
    case 8:
      if constexpr (BT <= 32) return launch_f8_t<BT, 8>(s, tx, x_f8, tw, a, st);
      break;
  }
  return LQ_ERR_INVALID_ARG;
}

lq_status w4f8_impl(const uint8_t* x_f8, const float* s_x, const uint8_t* qw4, const float* s_w, void* out, int M,
                    int N, int K, int sms, const int* cl, cudaStream_t st) {
  const int bt = M <= 16 ? 16 : M <= 64 ? 64 : 128;
  const Schedule s = make_schedule(M, N, K, bt, kSchedTiles, 0, 0, sms, cl);
  if (s.tiles * s.cs > INT_MAX) return LQ_ERR_UNSUPPORTED_SHAPE;
  CUtensorMap tx, tw;
  if (!make_map_u8(&tx, x_f8, (uint64_t)K, (uint64_t)M, (uint64_t)K, lq::kBlockK, (uint32_t)bt,
                   CU_TENSOR_MAP_SWIZZLE_128B) ||
      !make_map_u8(&tw, qw4, (uint64_t)K / 2, (uint64_t)N, (uint64_t)K / 2, lq::kBlockK / 2, lq::kBlockN,
                   CU_TENSOR_MAP_SWIZZLE_64B))
    return LQ_ERR_CUDA;
  lq::GemmArgs a;
  a.x_bf16 = nullptr;
  a.s_x = s_x;
  a.s_c = s_w;
  a.out = out;
  a.ws = nullptr;
  a.ticket = nullptr;
  a.M = M;
  a.N = N;
  a.K = K;
  a.tiles_m = s.tiles_m;
  a.KB = s.KB;
  a.U = s.U;
  switch (bt) {
    case 16: return launch_f8_bt<16>(s, tx, x_f8, tw, a, st);
    case 64: return launch_f8_bt<64>(s, tx, x_f8, tw, a, st);
    default: return launch_f8_bt<128>(s, tx, x_f8, tw, a, st);
  }
}

}  // namespace

extern "C" {

lq_status lq_quantize_weights_w4(const void* W_bf16, int N, int K, uint8_t* qw4, float* s_w, void* stream) {
  if (N < 0 || K < 0) return LQ_ERR_INVALID_ARG;
  if (K < 16 || K % 16 != 0) return LQ_ERR_UNSUPPORTED_SHAPE;
  if (N == 0) return LQ_OK;
  if (!W_bf16 || !qw4 || !s_w) return LQ_ERR_INVALID_ARG;
  if (!aligned(W_bf16, 16) || !aligned(qw4, 16) || !aligned(s_w, 4)) return LQ_ERR_MISALIGNED;
  DeviceInfo* dev = nullptr;
  const lq_status st = current_device(&dev);
  if (st != LQ_OK) return st;
  lq::quantize_weights_w4_kernel<<<N, lq::kW4Threads, 0, static_cast<cudaStream_t>(stream)>>>(
      static_cast<const uint16_t*>(W_bf16), K, qw4, s_w);
  return cudaGetLastError() == cudaSuccess ? LQ_OK : LQ_ERR_CUDA;
}

lq_status lq_quantize_act_f8(const void* X_bf16, int M, int K, uint8_t* x_f8, float* s_x, void* stream) {
  if (M < 0 || K < 0) return LQ_ERR_INVALID_ARG;
  if (K < 16 || K % 16 != 0) return LQ_ERR_UNSUPPORTED_SHAPE;
  if (!s_x || (M > 0 && (!X_bf16 || !x_f8))) return LQ_ERR_INVALID_ARG;
  if ((M > 0 && (!aligned(X_bf16, 16) || !aligned(x_f8, 16))) || !aligned(s_x, 4)) return LQ_ERR_MISALIGNED;
  DeviceInfo* dev = nullptr;
  const lq_status st = current_device(&dev);
  if (st != LQ_OK) return st;
  if (M > 0 && !device_addressable(X_bf16)) return LQ_ERR_INVALID_ARG;
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  // the tensor's amax in s_x's word, the codes, then s_x itself (an empty tensor gets s_x = 1)
  if (cudaMemsetAsync(s_x, 0, sizeof(float), cs) != cudaSuccess) return LQ_ERR_CUDA;
  unsigned int* amax_bits = reinterpret_cast<unsigned int*>(s_x);
  if (M > 0) {
    lq::act_f8_amax_kernel<<<M, lq::kQuantActThreads, 0, cs>>>(static_cast<const uint16_t*>(X_bf16), K, amax_bits);
    lq::act_f8_codes_kernel<<<M, lq::kQuantActThreads, 0, cs>>>(static_cast<const uint16_t*>(X_bf16), K, amax_bits,
                                                                 x_f8);
  }
  lq::act_f8_scale_kernel<<<1, 1, 0, cs>>>(s_x);
  return cudaGetLastError() == cudaSuccess ? LQ_OK : LQ_ERR_CUDA;
}

lq_status lq_w4f8_gemm(const uint8_t* x_f8, const float* s_x, const uint8_t* qw4, const float* s_w, void* out_bf16,
                       int M, int N, int K, void* stream) {
  lq_status st = check_gemm_shape(M, N, K, LQ_GROUP);
  if (st != LQ_OK) return st;
  if (M == 0) return LQ_OK;
  if (!x_f8 || !s_x || !qw4 || !s_w || !out_bf16) return LQ_ERR_INVALID_ARG;
  if (!aligned(x_f8, 16) || !aligned(qw4, 16) || !aligned(out_bf16, 16) || !aligned(s_x, 4) || !aligned(s_w, 4))
    return LQ_ERR_MISALIGNED;
  DeviceInfo* dev = nullptr;
  st = current_device(&dev);
  if (st != LQ_OK) return st;
  if (!device_addressable(out_bf16)) return LQ_ERR_INVALID_ARG;
  return w4f8_impl(x_f8, s_x, qw4, s_w, out_bf16, M, N, K, dev->sms, dev->cluster_ctas,
                   static_cast<cudaStream_t>(stream));
}

}  // extern "C"

// libqlora.so — C ABI (include/qlora.h) over the sm_100a kernels in
// codec.cuh and gemm.cuh. Host side: argument checks, the default code
// tables, TMA tensor-map encoding, workspace carving and the launch order of
// the forward and backward passes. Single translation unit.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <utility>
#include <atomic>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>
#include <new>
#include <vector>

#include "qlora.h"
#include "codec.cuh"
#include "gemm.cuh"
#include "skinny.cuh"
#include "smallm.cuh"
#include "adamw.cuh"
#include "ptx.cuh"

using namespace qlora;

namespace {

constexpr int kMaxDevices = 64;

// ------------------------------------------------------------ utilities --
inline bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
inline int64_t cdiv(int64_t a, int64_t b) { return (a + b - 1) / b; }
inline size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

struct DeviceInfo {
  bool init = false;
  bool sm100 = false;
  int sms = 0;
};
std::mutex g_mu;
DeviceInfo g_dev[kMaxDevices];
std::atomic<uint64_t> g_launches{0};
// Injected allocation failures: after g_inject_skip more allocations
// succeed, the next g_inject_fail fail.
std::mutex g_inject_mu;
int g_inject_skip = 0, g_inject_fail = 0;

// True when this allocation is to fail (consumes one injected failure).
bool inject_alloc_failure() {
  std::lock_guard<std::mutex> lock(g_inject_mu);
  if (g_inject_fail <= 0) return false;
  if (g_inject_skip > 0) {
    --g_inject_skip;
    return false;
  }
  --g_inject_fail;
  return true;
}
thread_local cudaEvent_t t_trace_start = nullptr;
thread_local cudaEvent_t t_trace_stop = nullptr;
// Compute type of the call in progress on this thread (set by the entry
// points for the duration of one call): fp16 operands and outputs when true,
// else bf16. Every launch of the call reads it.
thread_local bool t_f16 = false;
struct DtypeScope {
  explicit DtypeScope(bool f16) { t_f16 = f16; }
  ~DtypeScope() { t_f16 = false; }
  DtypeScope(const DtypeScope &) = delete;
  DtypeScope &operator=(const DtypeScope &) = delete;
};


qlora_status device_info(DeviceInfo *out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return QLORA_ERR_CUDA;
  std::lock_guard<std::mutex> lk(g_mu);
  DeviceInfo &d = g_dev[dev];
  if (!d.init) {
    int major = 0, minor = 0, sms = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
      return QLORA_ERR_CUDA;
    d.sm100 = (major == 10 && minor == 0);
    d.sms = sms;
    d.init = true;
  }
  *out = d;
  return d.sm100 ? QLORA_OK : QLORA_ERR_UNSUPPORTED;
}

// Code tables: finite and strictly ascending; the NF4 table holds 0.0f.
qlora_status check_tables(const float *nf4, const float *t8) {
  if (nf4 != nullptr) {
    bool zero = false;
    for (int i = 0; i < 16; ++i) {
      if (!std::isfinite(nf4[i])) return QLORA_ERR_TABLE;
      if (i > 0 && !(nf4[i] > nf4[i - 1])) return QLORA_ERR_TABLE;
      if (nf4[i] == 0.0f) zero = true;
    }
    if (!zero) return QLORA_ERR_TABLE;
  }
  if (t8 != nullptr) {
    for (int i = 0; i < 256; ++i) {
      if (!std::isfinite(t8[i])) return QLORA_ERR_TABLE;
      if (i > 0 && !(t8[i] > t8[i - 1])) return QLORA_ERR_TABLE;
    }
  }
  return QLORA_OK;
}

CodecTables make_tables(const float *nf4, const float *t8) {
  CodecTables t;
  std::memset(&t, 0, sizeof t);
  if (nf4) std::memcpy(t.nf4, nf4, sizeof t.nf4);
  if (t8) std::memcpy(t.t8, t8, sizeof t.t8);
  return t;
}

// Bucket table of the exact bucketed encode (see BucketTable): false when
// a midpoint lies outside [-1, 1] (the buckets cover only the range of
// x = w / c) or two midpoints fall inside one bucket; the binary search is
// used then. Host float arithmetic here is IEEE binary32 with the same
// operation order as the device (sum then halve; one fused multiply-add for
// the bucket).
bool build_buckets(const float *L, BucketTable *bt) {
  for (int i = 0; i < 15; ++i) {
    const float m = (L[i] + L[i + 1]) * 0.5f;
    if (!(m >= -1.0f && m <= 1.0f)) return false;
  }
  auto bucket = [](float x) {  // same arithmetic as nf4_code_bucket (|x| <= 1): (RNE(128 x + 128)) / 8
    const float y = std::fmaf(x, 128.0f, 128.0f + kBucketMagic);
    uint32_t a, b;
    std::memcpy(&a, &y, 4);
    std::memcpy(&b, &kBucketMagic, 4);
    return static_cast<int>((a - b) >> 3);
  };
  int jm[15], jp[15], inside[33] = {0};
  for (int j = 0; j < 33; ++j) bt->thr[j] = 2.0f;
  for (int i = 0; i < 15; ++i) {
    const float m = (L[i] + L[i + 1]) * 0.5f;
    jm[i] = bucket(m);
    jp[i] = bucket(std::nextafter(m, 2.0f));
    if (jm[i] == jp[i]) {
      if (inside[jm[i]]++) return false;
      bt->thr[jm[i]] = m;
    }
  }
  for (int j = 0; j < 33; ++j) {
    unsigned int c = 0;
    for (int i = 0; i < 15; ++i) c += (jp[i] < j || (jp[i] == j && jm[i] < j)) ? 1u : 0u;
    bt->cand[j] = c;
  }
  return true;
}

// Bucket table of the double-quantization encode (see DqBucketTable):
// false when a midpoint lies outside [2^-100, 1] or two share a bucket
// (the binary search is used then). Same fp32 arithmetic as the device.
bool build_dq_buckets(const float *t8, DqBucketTable *bt) {
  auto bucket = [](float x) {  // RNE(256 x) for x in [0, 1], as the kernel computes it
    const float y = std::fmaf(x, 256.0f, kBucketMagic);
    uint32_t a, b;
    std::memcpy(&a, &y, 4);
    std::memcpy(&b, &kBucketMagic, 4);
    return static_cast<int>(a - b);
  };
  int jm[255], jp[255], inside[257] = {0};
  for (int j = 0; j < 258; ++j) {
    bt->thr[j] = 2.0f;
    bt->cand[j] = 0u;
  }
  for (int i = 0; i < 255; ++i) {
    const float m = (t8[i] + t8[i + 1]) * 0.5f;
    if (!(m >= 0x1p-100f && m <= 1.0f)) return false;
    jm[i] = bucket(m);
    jp[i] = bucket(std::nextafter(m, 2.0f));
    if (jm[i] == jp[i]) {
      if (inside[jm[i]]++) return false;
      bt->thr[jm[i]] = m;
    }
  }
  // midpoint i lies below every x of bucket j from j = jp[i] on when it is the
  // last value of bucket jm[i] < jp[i], else from jp[i] + 1: count by prefix sum
  unsigned int from[258] = {0};
  for (int i = 0; i < 255; ++i) {
    const int j0 = jm[i] < jp[i] ? jp[i] : jp[i] + 1;
    ++from[j0 < 257 ? j0 : 257];
  }
  unsigned int c = 0;
  for (int j = 0; j < 257; ++j) {
    c += from[j];
    bt->cand[j] = c;
  }
  return true;
}

// The 8-bit bucket table of t8 (rebuilt only when t8 differs from this
// thread's last one); false when t8 needs the binary search instead.
bool dq_buckets(const float *t8, const DqBucketTable **out) {
  thread_local float last_t8[256];
  thread_local DqBucketTable bt;
  thread_local bool have_last = false, bucketed = false;
  if (!have_last || std::memcmp(last_t8, t8, sizeof last_t8) != 0) {
    std::memcpy(last_t8, t8, sizeof last_t8);
    bucketed = build_dq_buckets(t8, &bt);
    have_last = true;
  }
  *out = &bt;
  return bucketed;
}

// Every kernel is launched with programmatic stream serialization: it may
// start (prologue only) while the previous kernel in the stream finishes,
// and waits for it (griddepcontrol.wait) before touching its outputs.
template <typename... KArgs, typename... Args>
qlora_status launch_pdl(void (*kernel)(KArgs...), int grid, int block, size_t smem, cudaStream_t stream,
                        Args &&...args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(block);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  const cudaError_t e = cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
  g_launches.fetch_add(1, std::memory_order_relaxed);
  return e == cudaSuccess ? QLORA_OK : QLORA_ERR_CUDA;
}

// CTAs of `kernel` (block threads, static shared memory only) resident per
// SM, asked of the runtime once per kernel and device.
template <auto Kernel>
int resident_per_sm(int block) {
  static std::once_flag once[kMaxDevices];
  static int cached[kMaxDevices];
  int dev = 0;
  cudaGetDevice(&dev);
  std::call_once(once[dev], [&] {
    int n = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, Kernel, block, 0) != cudaSuccess || n < 1) n = 1;
    cached[dev] = n;
    cudaGetLastError();
  });
  return cached[dev];
}

int grid_for(int64_t work_items, int per_cta, int sms, int waves) {
  const int64_t want = cdiv(work_items, per_cta);
  const int64_t cap = static_cast<int64_t>(sms) * waves;
  return static_cast<int>(want < 1 ? 1 : (want < cap ? want : cap));
}

// ------------------------------------------------------------ TMA maps --
using EncodeTiledFn = CUresult (*)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                   const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                   const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// 2-D row-major tensor [outer, inner] with row pitch `row_bytes`; box
// {box_inner, box_outer}; out-of-range elements read as zero.
enum MapType { MAP_BF16, MAP_U8, MAP_F32 };

enum MapSwizzle { SW_NONE, SW_64B, SW_128B };

bool make_map(CUtensorMap *map, const void *base, MapType type, uint64_t inner, uint64_t outer,
              uint64_t row_bytes, uint32_t box_inner, uint32_t box_outer, MapSwizzle swz) {
  EncodeTiledFn fn = encode_fn();
  if (fn == nullptr) return false;
  const CUtensorMapDataType dt = type == MAP_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16
                                 : type == MAP_U8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8
                                                  : CU_TENSOR_MAP_DATA_TYPE_FLOAT32;
  const cuuint64_t dims[2] = {inner, outer};
  const cuuint64_t strides[1] = {row_bytes};
  const cuuint32_t box[2] = {box_inner, box_outer};
  const cuuint32_t estr[2] = {1, 1};
  const CUresult r = fn(map, dt, 2,
                        const_cast<void *>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                        swz == SW_128B ? CU_TENSOR_MAP_SWIZZLE_128B
                        : swz == SW_64B ? CU_TENSOR_MAP_SWIZZLE_64B
                                        : CU_TENSOR_MAP_SWIZZLE_NONE,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// bf16 operand [outer rows, inner] read as K-major tiles (box {64, box_rows})
bool map_kmajor(CUtensorMap *m, const void *p, int64_t inner, int64_t outer, uint32_t box_rows) {
  return make_map(m, p, MAP_BF16, inner, outer, inner * 2, 64, box_rows, SW_128B);
}
// bf16 operand [outer rows, inner] read as MN-major 64x64 chunks
bool map_mnmajor(CUtensorMap *m, const void *p, int64_t inner, int64_t outer) {
  return make_map(m, p, MAP_BF16, inner, outer, inner * 2, 64, 64, SW_128B);
}

// Token operand T [tokens, kdim] bf16 viewed as {64, tokens, kdim/64} (k
// within a 64-block, token, block): box {64, box_rows, bkb} lands as bkb
// consecutive K-major 128-byte-swizzled [box_rows][64] tiles.
bool map_tokens_3d(CUtensorMap *map, const void *T, int64_t tokens, int64_t kdim, uint32_t box_rows, uint32_t bkb) {
  EncodeTiledFn fn = encode_fn();
  if (fn == nullptr) return false;
  const cuuint64_t dims[3] = {64, static_cast<cuuint64_t>(tokens), static_cast<cuuint64_t>(kdim / 64)};
  const cuuint64_t strides[2] = {static_cast<cuuint64_t>(kdim) * 2, 128};
  const cuuint32_t box[3] = {64, box_rows, bkb};
  const cuuint32_t estr[3] = {1, 1, 1};
  const CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(T), dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// X [M, K] bf16 viewed as {64, K/64, M} (k within a block, block, token):
// box {64, 4, tokens} = four quantization blocks of K for every token row.
bool map_x_blocks(CUtensorMap *map, const void *X, int64_t M, int64_t K, uint32_t tokens) {
  EncodeTiledFn fn = encode_fn();
  if (fn == nullptr) return false;
  const cuuint64_t dims[3] = {64, static_cast<cuuint64_t>(K / 64), static_cast<cuuint64_t>(M)};
  const cuuint64_t strides[2] = {128, static_cast<cuuint64_t>(K) * 2};
  const cuuint32_t box[3] = {64, 4, tokens};
  const cuuint32_t estr[3] = {1, 1, 1};
  const CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(X), dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// ------------------------------------------------------- GEMM launcher --
template <class C>
qlora_status launch_gemm(const GemmArgs &args, int sms, int pair_slots, cudaStream_t stream) {
  static std::once_flag once[kMaxDevices];
  int dev = 0;
  cudaGetDevice(&dev);
  cudaError_t attr_err = cudaSuccess;
  std::call_once(once[dev], [&] {
    attr_err = cudaFuncSetAttribute(qgemm_kernel<C>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    C::SMEM_BYTES);
  });
  if (attr_err != cudaSuccess) return QLORA_ERR_CUDA;
  const int row_tiles = (args.rows + C::TILE_ROWS - 1) / C::TILE_ROWS;
  const int col_tiles = (args.cols + C::TILE_COLS - 1) / C::TILE_COLS;
  const int tiles = args.full_tiles + (row_tiles * col_tiles - args.full_tiles) *
                                          (args.tail_subtiles > 1 ? args.tail_subtiles : args.tail_splits);
  if constexpr (!C::PAIR) {
    const int grid = tiles < sms ? tiles : sms;
    return launch_pdl(qgemm_kernel<C>, grid, C::THREADS, C::SMEM_BYTES, stream, args);
  } else {
    // persistent: one cluster of two CTAs per resident pair slot, at most one per tile
    const int clusters = std::min(tiles, pair_slots);
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(2 * clusters);
    cfg.blockDim = dim3(C::THREADS);
    cfg.dynamicSmemBytes = C::SMEM_BYTES;
    cfg.stream = stream;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    attr[1].id = cudaLaunchAttributeClusterDimension;
    attr[1].val.clusterDim.x = 2;
    attr[1].val.clusterDim.y = 1;
    attr[1].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    const cudaError_t e = cudaLaunchKernelEx(&cfg, qgemm_kernel<C>, args);
    g_launches.fetch_add(1, std::memory_order_relaxed);
    return e == cudaSuccess ? QLORA_OK : QLORA_ERR_CUDA;
  }
}

// Clusters of two CTAs of pair variant C that can be resident at once on
// this device (asked of the runtime once per device; 0 if none or on error).
template <class C>
int resident_pairs() {
  static std::once_flag once[kMaxDevices];
  static int cached[kMaxDevices];
  int dev = 0;
  cudaGetDevice(&dev);
  std::call_once(once[dev], [&] {
    int n = 0;
    if (cudaFuncSetAttribute(qgemm_kernel<C>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES) ==
        cudaSuccess) {
      cudaLaunchConfig_t cfg = {};
      cfg.gridDim = dim3(2);
      cfg.blockDim = dim3(C::THREADS);
      cfg.dynamicSmemBytes = C::SMEM_BYTES;
      cudaLaunchAttribute at[1];
      at[0].id = cudaLaunchAttributeClusterDimension;
      at[0].val.clusterDim.x = 2;
      at[0].val.clusterDim.y = 1;
      at[0].val.clusterDim.z = 1;
      cfg.attrs = at;
      cfg.numAttrs = 1;
      if (cudaOccupancyMaxActiveClusters(&n, reinterpret_cast<const void *>(qgemm_kernel<C>), &cfg) != cudaSuccess)
        n = 0;
    }
    cudaGetLastError();
    cached[dev] = n;
  });
  return cached[dev];
}

// Block constants c' = t8[q] * S, block-major [K/64][N] fp32 (GEMM operand
// staging), decoded once per call by extra CTAs of the first skinny launch.

// Layer sizes shared by forward and backward.
struct Shape {
  int64_t M, N, K;
  int r;
};

// One counter per output tile of any GEMM of the call (tiles are at least
// 128 x 32).
int64_t counters_needed(const Shape &s) {
  // 128-row halves of the 256-row pair tiles included
  const int64_t rows = std::max(std::max(cdiv(s.M, 128), 2 * cdiv(s.N, 256)), 2 * cdiv(s.K, 256));
  return rows * std::max<int64_t>(1, cdiv(s.M, 32));
}

// ------------------------------------------------------- skinny GEMMs --
// out[rows, r] (or its transpose) = scale * sum_k Aop[row, k] Bop[j, k],
// the K range split across CTAs; the last CTA of a tile reduces.
enum SkinnyKind { SK_XA, SK_G, SK_DA, SK_DB };

int rank_tile(int r) { return r <= 64 ? 64 : (r <= 128 ? 128 : 256); }

// Ring depth per rank tile: 4 stages of 24 KB (r <= 64) or 3 of 32 KB
// (r <= 128) keep two CTAs on an SM; r <= 256 uses 4 stages of 48 KB.
// (Rings of about 192 KB per CTA, one CTA per SM, measured no faster.)
constexpr int skinny_stages(int bn) { return bn == 64 ? 4 : (bn == 128 ? 3 : 4); }

// One skinny-GEMM variant: its shared-memory opt-in and how many clusters
// of 2, 4 and 8 CTAs can be resident at once (asked of the runtime once per
// device).
template <int BN, bool AMN, bool BMN>
struct SkinnyVariant {
  using C = SkinnyCfg<BN, AMN, BMN, skinny_stages(BN)>;
  static qlora_status prepare(int (&max_clusters)[4], int *per_sm) {
    static std::once_flag once[kMaxDevices];
    static cudaError_t err[kMaxDevices];
    static int cached[kMaxDevices][4];
    static int resident[kMaxDevices];
    int dev = 0;
    cudaGetDevice(&dev);
    std::call_once(once[dev], [&] {
      err[dev] = cudaFuncSetAttribute(skinny_kernel<C>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES);
      // ask for the largest shared-memory carveout, so that two CTAs of
      // about 100 KB share an SM and the occupancy queries below count them
      if (err[dev] == cudaSuccess)
        err[dev] = cudaFuncSetAttribute(skinny_kernel<C>, cudaFuncAttributePreferredSharedMemoryCarveout,
                                        static_cast<int>(cudaSharedmemCarveoutMaxShared));
      int n1 = 0;
      if (err[dev] != cudaSuccess ||
          cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n1, skinny_kernel<C>, C::THREADS, C::SMEM_BYTES) !=
              cudaSuccess ||
          n1 < 1)
        n1 = 1;
      resident[dev] = n1;
      cached[dev][0] = 0;
      for (int l = 1; l <= 3; ++l) {
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(1u << l);
        cfg.blockDim = dim3(C::THREADS);
        cfg.dynamicSmemBytes = C::SMEM_BYTES;
        cudaLaunchAttribute at[1];
        at[0].id = cudaLaunchAttributeClusterDimension;
        at[0].val.clusterDim.x = 1u << l;
        at[0].val.clusterDim.y = 1;
        at[0].val.clusterDim.z = 1;
        cfg.attrs = at;
        cfg.numAttrs = 1;
        int n = 0;
        if (err[dev] != cudaSuccess ||
            cudaOccupancyMaxActiveClusters(&n, reinterpret_cast<const void *>(skinny_kernel<C>), &cfg) !=
                cudaSuccess)
          n = 0;
        cached[dev][l] = n;
      }
      cudaGetLastError();  // an unsupported cluster size only means "not that one"
    });
    for (int l = 0; l < 4; ++l) max_clusters[l] = cached[dev][l];
    *per_sm = resident[dev];
    return err[dev] == cudaSuccess ? QLORA_OK : QLORA_ERR_CUDA;
  }
};

struct SkinnyPlan {
  int rows, kblocks, splits, bn;
  int per_sm;  // resident CTAs per SM
};

// Split K over a cluster of 2, 4 or 8 CTAs per 128-row tile: the largest
// split whose clusters for all row tiles are resident at once (one wave),
// else one CTA per tile.
template <bool AMN, bool BMN>
qlora_status plan_skinny_v(int64_t rows, int64_t kdim, int r, SkinnyPlan *p) {
  p->rows = static_cast<int>(rows);
  p->kblocks = static_cast<int>(cdiv(kdim, 64));
  p->bn = rank_tile(r);
  int maxc[4];
  const qlora_status st = p->bn == 64    ? SkinnyVariant<64, AMN, BMN>::prepare(maxc, &p->per_sm)
                          : p->bn == 128 ? SkinnyVariant<128, AMN, BMN>::prepare(maxc, &p->per_sm)
                                         : SkinnyVariant<256, AMN, BMN>::prepare(maxc, &p->per_sm);
  const int row_tiles = static_cast<int>(cdiv(rows, 128));
  p->splits = 1;
  for (int l = 3; l >= 1; --l)
    if ((1 << l) <= p->kblocks && row_tiles <= maxc[l]) {
      p->splits = 1 << l;
      break;
    }
  return st;
}

template <int BN, bool AMN, bool BMN>
qlora_status run_skinny_bn(const SkinnyArgs &a, int grid, cudaStream_t st) {
  using C = typename SkinnyVariant<BN, AMN, BMN>::C;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(C::THREADS);
  cfg.dynamicSmemBytes = C::SMEM_BYTES;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  attr[1].id = cudaLaunchAttributeClusterDimension;
  attr[1].val.clusterDim.x = a.splits;
  attr[1].val.clusterDim.y = 1;
  attr[1].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = a.splits > 1 ? 2 : 1;
  const cudaError_t e = cudaLaunchKernelEx(&cfg, skinny_kernel<C>, a);
  g_launches.fetch_add(1, std::memory_order_relaxed);
  return e == cudaSuccess ? QLORA_OK : QLORA_ERR_CUDA;
}

template <bool AMN, bool BMN>
qlora_status run_skinny(const SkinnyArgs &a, int bn, int grid, cudaStream_t st) {
  if (bn == 64) return run_skinny_bn<64, AMN, BMN>(a, grid, st);
  if (bn == 128) return run_skinny_bn<128, AMN, BMN>(a, grid, st);
  return run_skinny_bn<256, AMN, BMN>(a, grid, st);
}


// kind: SK_XA   Aop = X [M,K] (K-major),   Bop = A  [K,r] (MN-major), rows = M, kdim = K
//       SK_G    Aop = dY [M,N] (K-major),  Bop = B  [r,N] (K-major),  rows = M, kdim = N
//       SK_DA   Aop = X^T (MN-major),      Bop = Gs [M,r] (MN-major), rows = K, kdim = M
//       SK_DB   Aop = dY^T (MN-major),     Bop = XA [M,r] (MN-major), rows = N, kdim = M
struct OutSpec {
  void *out;
  int64_t ld;
  float scale;
  void *out2;
  int64_t ld2;
  float scale2;
  bool transpose;
};

// One product's operands and output.
struct SkinnyOperands {
  const void *aop;
  int64_t a_inner, a_outer;
  const void *bop;
  int64_t b_inner, b_outer;
  int64_t rows, kdim;
  OutSpec o;
};

// Launch one or two products of the same kind (same operand layouts and
// reduction length) as one grid.
qlora_status skinny_launch(SkinnyKind kind, const SkinnyOperands *ops, int nprob, int r, int sms,
                           cudaStream_t st, unsigned int *zero_words, int nzero, bool early,
                           bool late = false) {
  int row_tiles[2] = {0, 0};
  for (int i = 0; i < nprob; ++i) row_tiles[i] = static_cast<int>(cdiv(ops[i].rows, 128));
  // the split is chosen for all row tiles of the launch together
  SkinnyPlan p;
  const int64_t plan_rows = static_cast<int64_t>(row_tiles[0] + row_tiles[1]) * 128;
  qlora_status pst = kind == SK_XA  ? plan_skinny_v<false, true>(plan_rows, ops[0].kdim, r, &p)
                     : kind == SK_G ? plan_skinny_v<false, false>(plan_rows, ops[0].kdim, r, &p)
                                    : plan_skinny_v<true, true>(plan_rows, ops[0].kdim, r, &p);
  if (pst != QLORA_OK) return pst;
  SkinnyArgs a;
  std::memset(&a, 0, sizeof a);
  for (int i = 0; i < nprob; ++i) {
    const SkinnyOperands &op = ops[i];
    SkinnyProblem &P = a.prob[i];
    bool ok = true;
    switch (kind) {
      case SK_XA:
        ok = map_kmajor(&P.tm_a, op.aop, op.a_inner, op.a_outer, 128) &&
             map_mnmajor(&P.tm_b, op.bop, op.b_inner, op.b_outer);
        break;
      case SK_G:
        ok = map_kmajor(&P.tm_a, op.aop, op.a_inner, op.a_outer, 128) &&
             map_kmajor(&P.tm_b, op.bop, op.b_inner, op.b_outer, p.bn);
        break;
      case SK_DA:
      case SK_DB:
        ok = map_mnmajor(&P.tm_a, op.aop, op.a_inner, op.a_outer) &&
             map_mnmajor(&P.tm_b, op.bop, op.b_inner, op.b_outer);
        break;
    }
    if (!ok) return QLORA_ERR_CUDA;
    P.out = op.o.out;
    P.out_ld = op.o.ld;
    P.out_scale = op.o.scale;
    P.out2 = op.o.out2;
    P.out2_ld = op.o.ld2;
    P.out2_scale = op.o.scale2;
    P.transpose = op.o.transpose ? 1 : 0;
    P.rows = static_cast<int>(op.rows);
    P.cols = r;
    P.kblocks = static_cast<int>(cdiv(op.kdim, 64));
  }
  a.splits = p.splits;
  a.prob0_ctas = row_tiles[0] * p.splits;
  a.zero_words = zero_words;
  a.nzero = nzero;
  a.early = early ? 1 : 0;
  a.late = late ? 1 : 0;
  a.f16 = t_f16 ? 1 : 0;
  const int grid = (row_tiles[0] + row_tiles[1]) * p.splits;
  switch (kind) {
    case SK_XA: return run_skinny<false, true>(a, p.bn, grid, st);
    case SK_G: return run_skinny<false, false>(a, p.bn, grid, st);
    default: return run_skinny<true, true>(a, p.bn, grid, st);
  }
}

qlora_status skinny(SkinnyKind kind, const void *aop, int64_t a_inner, int64_t a_outer, const void *bop,
                    int64_t b_inner, int64_t b_outer, int64_t rows, int64_t kdim, int r, const OutSpec &o,
                    int sms, cudaStream_t st, unsigned int *zero_words = nullptr, int nzero = 0,
                    bool early = false) {
  const SkinnyOperands op{aop, a_inner, a_outer, bop, b_inner, b_outer, rows, kdim, o};
  return skinny_launch(kind, &op, 1, r, sms, st, zero_words, nzero, early);
}

// -------------------------------------------------------- fused GEMMs --
// The pair variants of the fused GEMM (256 weight rows x 256 tokens per
// cluster of two CTAs): six token stages of one K block of 128 tokens (one
// 16 KB TMA box each), dequantized-weight stages of one K block (16 KB) and
// packed-code slots of 4 K blocks (18 KB).
constexpr int kPairBkb = 1, kPairSb = 6, kPairSa = 4, kPairSp = 2, kPairNpw = 8;
using FwdPairCfg = GemmCfg<256, A_DEQ_K, L2_A_MN, kPairBkb, kPairSb, kPairSa, kPairSp, kPairNpw, true>;
using BwdPairCfg = GemmCfg<256, A_DEQ_MN, L2_A_K, kPairBkb, kPairSb, kPairSa, kPairSp, kPairNpw, true>;
// Two 256-token sub-tiles per job (512 tokens per tile, each CTA loading 256
// of them): four token stages of one K block (32 KB boxes; finer stages than
// two of two blocks hide a refill behind three stages of MMAs, 2-3 % faster
// on the 7B shapes), 3 dequantized-weight stages, 2 packed-code slots (212 KB
// of shared memory).
constexpr int kPair2Bkb = 1, kPair2Sb = 4, kPair2Sa = 3, kPair2Sp = 2, kPair2Npw = 8;
using FwdPair2Cfg = GemmCfg<256, A_DEQ_K, L2_A_MN, kPair2Bkb, kPair2Sb, kPair2Sa, kPair2Sp, kPair2Npw, true, 2>;
using BwdPair2Cfg = GemmCfg<256, A_DEQ_MN, L2_A_K, kPair2Bkb, kPair2Sb, kPair2Sa, kPair2Sp, kPair2Npw, true, 2>;
// token counts from which a tile holds two 256-token sub-tiles
constexpr int64_t kTwoSubtileTokens = 1024;
// K blocks per token stage of the one-CTA variants: 32-token tiles take 4
// (a 16 KB box), the 256-token fallback 1 (a 32 KB box).
constexpr int single_bkb(int bn) { return bn == 32 ? 4 : 1; }

// Resident pair slots for the fused GEMMs on this device (both variants have
// the same shared memory and threads), 0 if the runtime reports none.
int fused_pair_slots(int sms) {
  const int n = std::min(std::min(resident_pairs<FwdPairCfg>(), resident_pairs<BwdPairCfg>()),
                         std::min(resident_pairs<FwdPair2Cfg>(), resident_pairs<BwdPair2Cfg>()));
  return std::min(n, sms / 2);
}

struct FusedPlan {
  int bn;
  int full_tiles, tail_splits, tail_subtiles;  // whole tiles first, then the rest split (see GemmArgs)
  bool pair;      // 256-row tiles over a cluster of two CTAs
  int ntt;        // token sub-tiles of bn tokens per tile (pairs: 1 or 2)
  int slots;      // persistent units: CTAs (one-CTA tiles) or clusters (pairs)
  size_t part_bytes;
  // tokens one CTA loads per K block (the token operand's TMA box height)
  uint32_t cta_tokens() const { return static_cast<uint32_t>(bn * ntt / (pair ? 2 : 1)); }
};

// Token tile: 32 tokens (one CTA per 128 weight rows) for a few tokens;
// otherwise 256 tokens on CTA pairs (256 weight rows), when the device can
// hold them, else on single CTAs; from kTwoSubtileTokens tokens on, two
// 256-token sub-tiles per tile. The persistent units (CTAs or pairs) run
// whole rounds of whole tiles; the tiles of a last, partial round are split
// so that the round fills the grid: by token sub-tile (two units of 256
// tokens over the whole K, disjoint outputs) when the tiles hold two and
// half the grid or more is idle, else over K (fp32 partials summed by the
// last split) when there are fewer tiles than units.
FusedPlan plan_fused(int64_t M, int64_t rows, int64_t kblocks, int sms, int pair_slots) {
  FusedPlan p;
  p.bn = M <= 32 ? 32 : 256;
  p.pair = M > 32 && pair_slots > 0;
  p.ntt = p.pair && M >= kTwoSubtileTokens ? 2 : 1;
  p.slots = p.pair ? pair_slots : sms;
  const int64_t tile_rows = p.pair ? 256 : 128;
  const int64_t tile_cols = static_cast<int64_t>(p.bn) * p.ntt;
  const int64_t tiles = cdiv(rows, tile_rows) * cdiv(M, tile_cols);
  const int64_t full = (tiles / p.slots) * p.slots;  // whole rounds
  const int64_t tail = tiles - full;
  p.tail_subtiles = 1;
  if (full > 0 && tail > 0 && p.ntt > 1 && tail * p.ntt <= p.slots) {
    p.full_tiles = static_cast<int>(full);
    p.tail_splits = 1;
    p.tail_subtiles = p.ntt;
    p.part_bytes = 0;
    return p;
  }
  // split K only when the tiles do not fill one round (the fp32 partials of
  // whole rounds of large tiles cost more than the imbalance they remove)
  int64_t splits = (tail > 0 && full == 0) ? p.slots / tail : 1;
  // a split runs at least 4 K blocks (1 on the memory-bound 32-token tiles)
  const int64_t min_kb = p.bn == 32 ? 1 : 4;
  if (splits > kblocks / min_kb) splits = kblocks / min_kb;
  if (splits < 2) splits = 1;
  p.full_tiles = static_cast<int>(splits > 1 ? full : tiles);
  p.tail_splits = static_cast<int>(splits);
  p.part_bytes = splits > 1 ? align256(static_cast<size_t>(splits) * tail * tile_rows * p.ntt * cdiv(p.bn, 32) * 32 * 4)
                            : 0;
  return p;
}

// Partial bytes of the plan the call will run on this device.
size_t fused_part_bound(int64_t M, int64_t rows, int64_t kblocks, int sms) {
  return plan_fused(M, rows, kblocks, sms, fused_pair_slots(sms)).part_bytes;
}

template <int BN, int AS, int L2>
qlora_status run_fused_bn(const GemmArgs &a, int sms, cudaStream_t st) {
  // rings: token stages (SB), dequantized weight tiles (SA), packed codes + constants (SP);
  // a few tokens leave the tensor core idle, so that variant runs 12 dequant warps
  // (P slots hold 4 K blocks each; the few-token variant streams the packed
  // weight from DRAM, so its P ring is deeper)
  constexpr int SB = BN > 64 ? 4 : 2, SA = BN > 64 ? 3 : 6, SP = BN > 64 ? 2 : 4, NPW = BN > 64 ? 8 : 12;
  return launch_gemm<GemmCfg<BN, AS, L2, single_bkb(BN), SB, SA, SP, NPW, false>>(a, sms, 0, st);
}

template <class C>
qlora_status run_fused_pair(const GemmArgs &a, int sms, int slots, cudaStream_t st) {
  return launch_gemm<C>(a, sms, slots, st);
}

// ---------------------------------------------------- few-token forward --
// Used for M <= 16 tokens: bands of 256 rows x chunks of 256 K split evenly
// over a persistent grid of one CTA per SM. The X A kernel launched just
// before it (and overlapping it) holds `busy_sms` SMs; leaving those out
// keeps every CTA of the stream starting at once.
constexpr int kSmallmMaxTokens = 16;

struct SmallmPlan {
  int nt, grid, units, kc, bands;
  size_t part_bytes;
};

SmallmPlan plan_smallm(int64_t M, int64_t N, int64_t K, int sms, int busy_sms) {
  SmallmPlan p;
  p.nt = static_cast<int>(cdiv(M, 8));
  p.bands = static_cast<int>(cdiv(N, SmallmCfg<1>::BAND));
  p.kc = static_cast<int>(cdiv(K, 256));
  p.units = p.bands * p.kc;
  const int avail = std::max(1, sms - busy_sms);
  // at least two units per CTA: a band then spans half as many CTAs, whose
  // serial reduction at the end costs more on small weights than the
  // parallelism it buys (4096 x 4096 at 16 tokens: 20.5 us against 26.8)
  p.grid = std::min(std::max(1, p.units / 2), avail);
  // two partial slots per CTA: its pieces of the bands shared with other CTAs
  p.part_bytes = align256(static_cast<size_t>(p.grid) * 2 * SmallmCfg<1>::WARPS * p.nt * 32 * 16);
  return p;
}

int skinny_ctas(int64_t rows, int64_t kdim, int r) {
  SkinnyPlan p;
  if (plan_skinny_v<false, true>(rows, kdim, r, &p) != QLORA_OK) return 8;
  return static_cast<int>(cdiv(rows, 128)) * p.splits;
}

template <int NT, bool F16>
qlora_status run_smallm_nt(const SmallmArgs &a, int grid, cudaStream_t st) {
  using C = SmallmCfg<NT>;
  static std::once_flag once[kMaxDevices];
  int dev = 0;
  cudaGetDevice(&dev);
  cudaError_t attr_err = cudaSuccess;
  std::call_once(once[dev], [&] {
    attr_err =
        cudaFuncSetAttribute(smallm_kernel<NT, F16>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES);
  });
  if (attr_err != cudaSuccess) return QLORA_ERR_CUDA;
  return launch_pdl(smallm_kernel<NT, F16>, grid, C::THREADS, C::SMEM_BYTES, st, a);
}

qlora_status run_smallm(const SmallmArgs &a, const SmallmPlan &p, cudaStream_t st) {
  if (t_f16) return p.nt == 1 ? run_smallm_nt<1, true>(a, p.grid, st) : run_smallm_nt<2, true>(a, p.grid, st);
  return p.nt == 1 ? run_smallm_nt<1, false>(a, p.grid, st) : run_smallm_nt<2, false>(a, p.grid, st);
}

// Workspace carve-up: [tile counters][bf16 M x r][bf16 M x r (backward)][fp32 partials]
struct WsLayout {
  size_t counters, mr, part, total;
  int64_t ncounters;
};

WsLayout ws_layout(const Shape &s, int sms, bool backward) {
  WsLayout w;
  w.ncounters = counters_needed(s);
  w.counters = align256(static_cast<size_t>(w.ncounters) * 4);
  w.mr = align256(static_cast<size_t>(s.M) * s.r * 2);
  if (!backward) {
    w.part = s.M <= kSmallmMaxTokens ? plan_smallm(s.M, s.N, s.K, sms, 0).part_bytes
                                     : fused_part_bound(s.M, s.N, s.K / 64, sms);
    w.total = w.counters + w.mr + w.part;
  } else {
    // the skinny GEMMs reduce their split-K partials in shared memory
    const size_t part = fused_part_bound(s.M, s.K, s.N / 64, sms);   // dX split-K
    w.part = part;
    w.total = w.counters + 2 * w.mr + w.part;
  }
  return w;
}

size_t fwd_ws_bytes(const Shape &s, int sms) { return ws_layout(s, sms, false).total; }
size_t bwd_ws_bytes(const Shape &s, int sms) { return ws_layout(s, sms, true).total; }

void trace_begin(cudaStream_t s) {
  if (t_trace_start && t_trace_stop) cudaEventRecord(t_trace_start, s);
}
void trace_end(cudaStream_t s) {
  if (t_trace_start && t_trace_stop) cudaEventRecord(t_trace_stop, s);
}

// Self-test of the failure path: one thread waits on an mbarrier phase that
// nothing completes. mbar_wait gives up after kWaitTimeoutNs, raises the
// abort flag and bit 0 of the device error word, and the kernel returns; no
// trap, no fault, the context stays usable.
__global__ void selftest_wait_kernel() {
  __shared__ __align__(8) unsigned long long bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    abort_flag = 0;
    mbar_init(smem_u32(&bar), 1);
    fence_barrier_init();
    mbar_wait(smem_u32(&bar), 0u, &abort_flag);
  }
}

qlora_status check_linear(const uint8_t *packed, const uint8_t *q, const float *scale2, const float *nf4,
                          const float *t8, const Shape &s, float alpha) {
  if (!packed || !q || !scale2 || !nf4 || !t8) return QLORA_ERR_NULL;
  if (s.M < 1 || s.N < 64 || s.K < 64 || s.N % 64 || s.K % 64) return QLORA_ERR_SHAPE;
  if (s.M > (int64_t(1) << 30) || s.N > (int64_t(1) << 30) || s.K > (int64_t(1) << 30))
    return QLORA_ERR_SHAPE;
  if (s.r < 1 || s.r > QLORA_MAX_RANK || s.r % 8) return QLORA_ERR_RANGE;
  if (!std::isfinite(alpha)) return QLORA_ERR_RANGE;
  if (!aligned16(packed) || !aligned16(q) || !aligned16(scale2)) return QLORA_ERR_ALIGN;
  return check_tables(nf4, t8);
}

}  // namespace

// ====================================================================== ABI
extern "C" {

const char *qlora_status_string(qlora_status s) {
  switch (s) {
    case QLORA_OK: return "QLORA_OK";
    case QLORA_ERR_NULL: return "QLORA_ERR_NULL";
    case QLORA_ERR_SHAPE: return "QLORA_ERR_SHAPE";
    case QLORA_ERR_ALIGN: return "QLORA_ERR_ALIGN";
    case QLORA_ERR_RANGE: return "QLORA_ERR_RANGE";
    case QLORA_ERR_CUDA: return "QLORA_ERR_CUDA";
    case QLORA_ERR_UNSUPPORTED: return "QLORA_ERR_UNSUPPORTED";
    case QLORA_ERR_WORKSPACE: return "QLORA_ERR_WORKSPACE";
    case QLORA_ERR_TABLE: return "QLORA_ERR_TABLE";
  }
  return "QLORA_ERR_UNKNOWN";
}

int qlora_abi_version(void) { return QLORA_ABI_VERSION; }

// Standard-normal quantile by Newton's method on the CDF written with erfc
// (double precision), from z = 0: z <- z - (Phi(z) - p) / phi(z).
static double normal_quantile(double p) {
  double z = 0.0;
  for (int it = 0; it < 100; ++it) {
    const double cdf = 0.5 * std::erfc(-z / std::sqrt(2.0));
    const double pdf = std::exp(-0.5 * z * z) / std::sqrt(2.0 * M_PI);
    const double step = (cdf - p) / pdf;
    z -= step;
    if (std::fabs(step) < 1e-17 * (1.0 + std::fabs(z))) break;
  }
  return z;
}

void qlora_nf4_levels(float out[16]) {
  if (out == nullptr) return;
  const double delta = 0.5 * ((1.0 - 1.0 / 30.0) + (1.0 - 1.0 / 32.0));
  const double zmax = normal_quantile(delta);
  for (int i = 0; i < 7; ++i) out[i] = static_cast<float>(-normal_quantile(delta + i * (0.5 - delta) / 7.0) / zmax);
  out[7] = 0.0f;
  for (int j = 0; j < 8; ++j) out[15 - j] = static_cast<float>(normal_quantile(delta + j * (0.5 - delta) / 8.0) / zmax);
}

void qlora_dq_levels(float out[256]) {
  if (out == nullptr) return;
  for (int k = 0; k < 256; ++k) out[k] = static_cast<float>(k) / 255.0f;
}

void qlora_int4_levels(float out[16]) {
  if (out == nullptr) return;
  for (int i = 0; i < 16; ++i) out[i] = static_cast<float>(static_cast<double>(i - 8) / 7.0);
}

void qlora_fp4_levels(float out[16]) {
  if (out == nullptr) return;
  // E2M1: sign, 2 exponent bits (bias 1), 1 mantissa bit; +0 once; 8 pads the table
  static const double v[16] = {-6.0, -4.0, -3.0, -2.0, -1.5, -1.0, -0.5, 0.0,
                               0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0, 8.0};
  for (int i = 0; i < 16; ++i) out[i] = static_cast<float>(v[i] / 6.0);
}

void qlora_dq_signed_levels(float out[256]) {
  if (out == nullptr) return;
  for (int k = 0; k < 256; ++k) out[k] = static_cast<float>((2.0 * k - 255.0) / 255.0);
}

void qlora_dq_dynamic_levels(float out[256]) {
  if (out == nullptr) return;
  out[0] = 0.0f;
  for (int k = 1; k < 256; ++k) {
    const int j = 255 - k;  // j = 0 is the largest level, 1
    out[k] = static_cast<float>(std::ldexp(1.0 - (j % 32) / 64.0, -(j / 32)));
  }
}

size_t qlora_workspace_bytes(int64_t M, int64_t N, int64_t K, int r) {
  if (M < 1 || N < 64 || K < 64 || N % 64 || K % 64 || r < 1 || r > QLORA_MAX_RANK || r % 8) return 0;
  DeviceInfo d;
  int sms = 148;
  if (device_info(&d) == QLORA_OK) sms = d.sms;
  const Shape s{M, N, K, r};
  const size_t f = fwd_ws_bytes(s, sms), b = bwd_ws_bytes(s, sms);
  return f > b ? f : b;
}

qlora_status qlora_quantize_nf4(const qlora_bf16 *W, int64_t N, int64_t K, const float nf4[16], uint8_t *packed,
                                float *absmax, qlora_stream_t stream) {
  if (!W || !nf4 || !packed || !absmax) return QLORA_ERR_NULL;
  if (N < 1 || K < 64 || K % 64) return QLORA_ERR_SHAPE;
  if (!aligned16(W) || !aligned16(packed) || !aligned16(absmax)) return QLORA_ERR_ALIGN;
  qlora_status st = check_tables(nf4, nullptr);
  if (st != QLORA_OK) return st;
  DeviceInfo d;
  if ((st = device_info(&d)) != QLORA_OK) return st;
  const int64_t nblocks = N * (K / 64);
  BucketTable bt;
  const bool bucketed = build_buckets(nf4, &bt);
  // 32-byte loads when W allows them
  const bool v8 = (reinterpret_cast<uintptr_t>(W) & 31u) == 0;
  auto kernel = bucketed ? (v8 ? quantize_nf4_kernel<true, true> : quantize_nf4_kernel<true, false>)
                         : (v8 ? quantize_nf4_kernel<false, true> : quantize_nf4_kernel<false, false>);
  // one resident wave (a grid-stride loop covers the rest); 512 32-byte units per CTA pass
  const int grid = grid_for(nblocks * 4, 512, d.sms,
                            bucketed ? resident_per_sm<quantize_nf4_kernel<true, true>>(256)
                                     : resident_per_sm<quantize_nf4_kernel<false, true>>(256));
  return launch_pdl(kernel, grid, 256, 0,
                    static_cast<cudaStream_t>(stream), reinterpret_cast<const uint4 *>(W), nblocks,
                    reinterpret_cast<uint32_t *>(packed), absmax, make_tables(nf4, nullptr), bt);
}

// threads per CTA of the one-pass quantize (each takes 1024 / this many
// 16-weight units of a group)
constexpr int kQuantizeDqThreads = 512;

qlora_status qlora_quantize_dq(const qlora_bf16 *W, int64_t N, int64_t K, const float nf4[16], const float t8[256],
                               uint8_t *packed, uint8_t *q, float *scale2, float *absmax, qlora_stream_t stream) {
  if (!W || !nf4 || !t8 || !packed || !q || !scale2) return QLORA_ERR_NULL;
  if (N < 1 || K < 64 || K % 64) return QLORA_ERR_SHAPE;
  if (!aligned16(W) || !aligned16(packed) || !aligned16(q) || !aligned16(scale2) || (absmax && !aligned16(absmax)))
    return QLORA_ERR_ALIGN;
  qlora_status st = check_tables(nf4, t8);
  if (st != QLORA_OK) return st;
  DeviceInfo d;
  if ((st = device_info(&d)) != QLORA_OK) return st;
  const int64_t nblocks = N * (K / 64);
  BucketTable bt;
  const bool bucketed = build_buckets(nf4, &bt);
  const DqBucketTable *dbt = nullptr;
  const bool dq_bucketed = dq_buckets(t8, &dbt);
  const bool v8 = (reinterpret_cast<uintptr_t>(W) & 31u) == 0;
  using KFn = void (*)(const uint4 *, int64_t, uint32_t *, uint8_t *, float *, float *, const CodecTables,
                       const BucketTable, const DqBucketTable);
  constexpr int QT = kQuantizeDqThreads;
  static const KFn table[8] = {
      quantize_dq_kernel<false, false, false, QT>, quantize_dq_kernel<false, false, true, QT>,
      quantize_dq_kernel<false, true, false, QT>,  quantize_dq_kernel<false, true, true, QT>,
      quantize_dq_kernel<true, false, false, QT>,  quantize_dq_kernel<true, false, true, QT>,
      quantize_dq_kernel<true, true, false, QT>,   quantize_dq_kernel<true, true, true, QT>};
  const KFn kernel = table[(bucketed ? 4 : 0) + (v8 ? 2 : 0) + (dq_bucketed ? 1 : 0)];
  // one group (256 blocks) per CTA pass, one resident wave
  const int64_t ng = cdiv(nblocks, 256);
  const int grid = grid_for(ng, 1, d.sms, resident_per_sm<quantize_dq_kernel<true, true, true, QT>>(QT));
  return launch_pdl(kernel, grid, QT, 0, static_cast<cudaStream_t>(stream), reinterpret_cast<const uint4 *>(W),
                    nblocks, reinterpret_cast<uint32_t *>(packed), q, scale2, absmax, make_tables(nf4, t8), bt,
                    *dbt);
}

qlora_status qlora_double_quant(const float *absmax, int64_t nb, const float t8[256], uint8_t *q, float *scale2,
                                qlora_stream_t stream) {
  if (!absmax || !t8 || !q || !scale2) return QLORA_ERR_NULL;
  if (nb < 1) return QLORA_ERR_SHAPE;
  if (!aligned16(absmax) || !aligned16(q) || !aligned16(scale2)) return QLORA_ERR_ALIGN;
  qlora_status st = check_tables(nullptr, t8);
  if (st != QLORA_OK) return st;
  DeviceInfo d;
  if ((st = device_info(&d)) != QLORA_OK) return st;
  const DqBucketTable *btp = nullptr;
  const bool bucketed = dq_buckets(t8, &btp);
  const DqBucketTable &bt = *btp;
  static DqBucketTable no_buckets;
  // one group per warp; at most two CTAs per SM (each fills its own table),
  // warps with more groups load the next one ahead
  const int64_t ng = cdiv(nb, 256);
  const int grid = grid_for(ng, 8, d.sms, 2);
  return bucketed ? launch_pdl(double_quant_kernel<true>, grid, 256, 0, static_cast<cudaStream_t>(stream), absmax,
                               nb, q, scale2, make_tables(nullptr, t8), bt)
                  : launch_pdl(double_quant_kernel<false>, grid, 256, 0, static_cast<cudaStream_t>(stream), absmax,
                               nb, q, scale2, make_tables(nullptr, t8), no_buckets);
}

qlora_status qlora_dequant(const uint8_t *packed, const uint8_t *q, const float *scale2, int64_t N, int64_t K,
                           const float nf4[16], const float t8[256], qlora_bf16 *W_out, qlora_stream_t stream) {
  if (!packed || !q || !scale2 || !nf4 || !t8 || !W_out) return QLORA_ERR_NULL;
  if (N < 1 || K < 64 || K % 64) return QLORA_ERR_SHAPE;
  if (!aligned16(packed) || !aligned16(q) || !aligned16(scale2) || !aligned16(W_out)) return QLORA_ERR_ALIGN;
  qlora_status st = check_tables(nf4, t8);
  if (st != QLORA_OK) return st;
  DeviceInfo d;
  if ((st = device_info(&d)) != QLORA_OK) return st;
  const int64_t nblocks = N * K / 64;
  const int grid = grid_for(nblocks, 256, d.sms, resident_per_sm<dequant_kernel>(256));
  return launch_pdl(dequant_kernel, grid, 256, 0, static_cast<cudaStream_t>(stream),
                    reinterpret_cast<const uint4 *>(packed), q, scale2, nblocks, reinterpret_cast<uint4 *>(W_out),
                    make_tables(nf4, t8), t_f16 ? 1 : 0);
}

qlora_status qlora_linear_fwd(const uint8_t *packed, const uint8_t *q, const float *scale2, const float nf4[16],
                              const float t8[256], int64_t M, int64_t N, int64_t K, const qlora_bf16 *X,
                              const qlora_bf16 *A, const qlora_bf16 *B, int r, float alpha, qlora_bf16 *Y,
                              qlora_bf16 *XA_out, void *workspace, size_t workspace_bytes,
                              qlora_stream_t stream) {
  const Shape s{M, N, K, r};
  qlora_status st = check_linear(packed, q, scale2, nf4, t8, s, alpha);
  if (st != QLORA_OK) return st;
  if (!X || !A || !B || !Y) return QLORA_ERR_NULL;
  if (!aligned16(X) || !aligned16(A) || !aligned16(B) || !aligned16(Y) || (XA_out && !aligned16(XA_out)) ||
      !aligned16(workspace))
    return QLORA_ERR_ALIGN;
  DeviceInfo d;
  if ((st = device_info(&d)) != QLORA_OK) return st;
  if (!workspace || workspace_bytes < fwd_ws_bytes(s, d.sms)) return QLORA_ERR_WORKSPACE;
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  const float scl = alpha / static_cast<float>(r);

  const WsLayout w = ws_layout(s, d.sms, false);
  uint8_t *ws = static_cast<uint8_t *>(workspace);
  unsigned int *counters = reinterpret_cast<unsigned int *>(ws);
  qlora_bf16 *xas = reinterpret_cast<qlora_bf16 *>(ws + w.counters);
  float *part = reinterpret_cast<float *>(ws + w.counters + w.mr);

  if (M <= kSmallmMaxTokens) {
    // Few tokens: XA (which also zeroes the band counters), then one pass over
    // the packed weight that dequantizes in registers.
    const SmallmPlan sp = plan_smallm(M, N, K, d.sms, skinny_ctas(M, K, r));
    OutSpec o{xas, r, scl, XA_out, r, 1.0f, false};
    st = skinny(SK_XA, X, K, M, A, r, K, M, K, r, o, d.sms, cs, counters, sp.bands);
    if (st != QLORA_OK) return st;
    SmallmArgs a;
    std::memset(&a, 0, sizeof a);
    if (!map_x_blocks(&a.tm_x, X, M, K, static_cast<uint32_t>(8 * sp.nt)) ||
        !make_map(&a.tm_w, packed, MAP_U8, K / 2, N, K / 2, 128, SmallmCfg<1>::BAND, SW_128B))
      return QLORA_ERR_CUDA;
    a.q = q;
    a.scale2 = scale2;
    a.B = B;
    a.xas = xas;
    a.Y = Y;
    a.part = part;
    a.counters = counters;
    a.N = N;
    a.K = K;
    a.M = static_cast<int>(M);
    a.r = r;
    a.kc = sp.kc;
    a.units = sp.units;
    a.tabs = make_tables(nf4, t8);
    trace_begin(cs);
    st = run_smallm(a, sp, cs);
    trace_end(cs);
    return st;
  }

  // 1) XA = X A -> XA_out = bf16(XA) (if wanted), xas = bf16(s XA); the same
  //    launch zeroes the split-K tile counters. The GEMM after it decodes
  //    the block constants itself and waits for this launch only before its
  //    low-rank K-steps and its counters, so its main loop overlaps it.
  {
    OutSpec o{xas, r, scl, XA_out, r, 1.0f, false};
    st = skinny(SK_XA, X, K, M, A, r, K, M, K, r, o, d.sms, cs, counters, static_cast<int>(w.ncounters), false);
    if (st != QLORA_OK) return st;
  }

  // 2) Y^T[n, m] = W'[n, :] . X[m, :] + B^T[n, :] . xas[m, :]
  const FusedPlan fp = plan_fused(M, N, K / 64, d.sms, fused_pair_slots(d.sms));
  const uint32_t b_rows = fp.cta_tokens();
  const uint32_t bkb = static_cast<uint32_t>(!fp.pair ? single_bkb(fp.bn) : fp.ntt == 2 ? kPair2Bkb : kPairBkb);
  GemmArgs a;
  std::memset(&a, 0, sizeof a);
  if (!map_tokens_3d(&a.tm_b, X, M, K, b_rows, bkb) ||
      !make_map(&a.tm_pk, packed, MAP_U8, K / 2, N, K / 2, 128, 128, SW_128B) ||
      !map_mnmajor(&a.tm_a2, B, N, r) || !map_kmajor(&a.tm_b2, xas, r, M, b_rows))
    return QLORA_ERR_CUDA;
  a.rows = static_cast<int>(N);
  a.cols = static_cast<int>(M);
  a.kblocks = static_cast<int>(K / 64);
  a.full_tiles = fp.full_tiles;
  a.tail_splits = fp.tail_splits;
  a.tail_subtiles = fp.tail_subtiles;
  a.lora_kblocks = static_cast<int>(cdiv(r, 64));
  a.out = Y;
  a.out_ld = N;
  a.part = part;
  a.counters = counters;
  std::memcpy(a.nf4, nf4, sizeof a.nf4);
  std::memcpy(a.t8, t8, sizeof a.t8);
  a.q = q;
  a.scale2 = scale2;
  a.wkb = K / 64;
  a.f16 = t_f16 ? 1 : 0;
  trace_begin(cs);
  st = fp.pair ? (fp.ntt == 2 ? run_fused_pair<FwdPair2Cfg>(a, d.sms, fp.slots, cs)
                              : run_fused_pair<FwdPairCfg>(a, d.sms, fp.slots, cs))
       : fp.bn == 32 ? run_fused_bn<32, A_DEQ_K, L2_A_MN>(a, d.sms, cs)
                     : run_fused_bn<256, A_DEQ_K, L2_A_MN>(a, d.sms, cs);
  trace_end(cs);
  return st;
}

qlora_status qlora_linear_bwd(const uint8_t *packed, const uint8_t *q, const float *scale2, const float nf4[16],
                              const float t8[256], int64_t M, int64_t N, int64_t K, const qlora_bf16 *X,
                              const qlora_bf16 *dY, const qlora_bf16 *A, const qlora_bf16 *B, const qlora_bf16 *XA,
                              int r, float alpha, qlora_bf16 *dX, qlora_bf16 *dA, qlora_bf16 *dB, void *workspace,
                              size_t workspace_bytes, qlora_stream_t stream) {
  const Shape s{M, N, K, r};
  qlora_status st = check_linear(packed, q, scale2, nf4, t8, s, alpha);
  if (st != QLORA_OK) return st;
  if (!X || !dY || !A || !B || !dX || !dA || !dB) return QLORA_ERR_NULL;
  if (!aligned16(X) || !aligned16(dY) || !aligned16(A) || !aligned16(B) || (XA && !aligned16(XA)) ||
      !aligned16(dX) || !aligned16(dA) || !aligned16(dB) || !aligned16(workspace))
    return QLORA_ERR_ALIGN;
  DeviceInfo d;
  if ((st = device_info(&d)) != QLORA_OK) return st;
  if (!workspace || workspace_bytes < bwd_ws_bytes(s, d.sms)) return QLORA_ERR_WORKSPACE;
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  const float scl = alpha / static_cast<float>(r);

  const WsLayout w = ws_layout(s, d.sms, true);
  uint8_t *ws = static_cast<uint8_t *>(workspace);
  unsigned int *counters = reinterpret_cast<unsigned int *>(ws);
  qlora_bf16 *gs = reinterpret_cast<qlora_bf16 *>(ws + w.counters);
  qlora_bf16 *xa_ws = reinterpret_cast<qlora_bf16 *>(ws + w.counters + w.mr);
  float *part = reinterpret_cast<float *>(ws + w.counters + 2 * w.mr);

  // 1) Gs = bf16(s * dY B^T); the same launch zeroes the tile counters
  //    (first kernel of the call: it waits before loading)
  {
    OutSpec o{gs, r, scl, nullptr, 0, 0.0f, false};
    st = skinny(SK_G, dY, N, M, B, N, r, M, N, r, o, d.sms, cs, counters, static_cast<int>(w.ncounters), false);
    if (st != QLORA_OK) return st;
  }

  // XA for dB, recomputed when the forward did not save it (X and A are
  // inputs, Gs just before is not an operand)
  const qlora_bf16 *xa = XA;
  if (xa == nullptr) {
    OutSpec o{xa_ws, r, 1.0f, nullptr, 0, 0.0f, false};
    st = skinny(SK_XA, X, K, M, A, r, K, M, K, r, o, d.sms, cs, nullptr, 0, true);
    if (st != QLORA_OK) return st;
    xa = xa_ws;
  }

  // 2) dX^T[k, m] = W'^T[k, :] . dY[m, :] + A[k, :] . Gs[m, :]
  const FusedPlan fp = plan_fused(M, K, N / 64, d.sms, fused_pair_slots(d.sms));
  const uint32_t b_rows = fp.cta_tokens();
  const uint32_t bkb = static_cast<uint32_t>(!fp.pair ? single_bkb(fp.bn) : fp.ntt == 2 ? kPair2Bkb : kPairBkb);
  GemmArgs a;
  std::memset(&a, 0, sizeof a);
  if (!map_tokens_3d(&a.tm_b, dY, M, N, b_rows, bkb) ||
      !make_map(&a.tm_pk, packed, MAP_U8, K / 2, N, K / 2, 64, 256, SW_64B) ||
      !map_kmajor(&a.tm_a2, A, r, K, 128) || !map_kmajor(&a.tm_b2, gs, r, M, b_rows))
    return QLORA_ERR_CUDA;
  a.rows = static_cast<int>(K);
  a.cols = static_cast<int>(M);
  a.kblocks = static_cast<int>(N / 64);
  a.full_tiles = fp.full_tiles;
  a.tail_splits = fp.tail_splits;
  a.tail_subtiles = fp.tail_subtiles;
  a.lora_kblocks = static_cast<int>(cdiv(r, 64));
  a.out = dX;
  a.out_ld = K;
  a.part = part;
  a.counters = counters;
  std::memcpy(a.nf4, nf4, sizeof a.nf4);
  std::memcpy(a.t8, t8, sizeof a.t8);
  a.q = q;
  a.scale2 = scale2;
  a.wkb = K / 64;
  a.f16 = t_f16 ? 1 : 0;
  trace_begin(cs);
  st = fp.pair ? (fp.ntt == 2 ? run_fused_pair<BwdPair2Cfg>(a, d.sms, fp.slots, cs)
                              : run_fused_pair<BwdPairCfg>(a, d.sms, fp.slots, cs))
       : fp.bn == 32 ? run_fused_bn<32, A_DEQ_MN, L2_A_K>(a, d.sms, cs)
                     : run_fused_bn<256, A_DEQ_MN, L2_A_K>(a, d.sms, cs);
  trace_end(cs);
  if (st != QLORA_OK) return st;

  // 3) dA = X^T Gs ([K, r]) and dB = s XA^T dY ([r, N], from dB^T[n, j]) in one
  //    launch. Every operand was written at least two kernels back: this
  //    launch can only start once every dX CTA has passed its own wait for
  //    those kernels, so they are complete; and the dX GEMM neither reads dA,
  //    dB nor writes anything read here. So the launch runs "late": its CTAs
  //    compute on the SMs the dX GEMM's last wave leaves idle and wait for it
  //    only before exiting (the call still ends after dX is written).
  const SkinnyOperands ops[2] = {
      {X, K, M, gs, r, M, K, M, OutSpec{dA, r, 1.0f, nullptr, 0, 0.0f, false}},
      {dY, N, M, xa, r, M, N, M, OutSpec{dB, N, scl, nullptr, 0, 0.0f, true}}};
  return skinny_launch(SK_DA, ops, 2, r, d.sms, cs, nullptr, 0, true, true);
}

qlora_status qlora_dequant_dt(const uint8_t *packed, const uint8_t *q, const float *scale2, int64_t N, int64_t K,
                              const float nf4[16], const float t8[256], qlora_dtype dtype, void *W_out,
                              qlora_stream_t stream) {
  if (dtype != QLORA_BF16 && dtype != QLORA_F16) return QLORA_ERR_RANGE;
  DtypeScope scope(dtype == QLORA_F16);
  return qlora_dequant(packed, q, scale2, N, K, nf4, t8, static_cast<qlora_bf16 *>(W_out), stream);
}

qlora_status qlora_linear_fwd_dt(const uint8_t *packed, const uint8_t *q, const float *scale2, const float nf4[16],
                                 const float t8[256], qlora_dtype dtype, int64_t M, int64_t N, int64_t K,
                                 const void *X, const void *A, const void *B, int r, float alpha, void *Y,
                                 void *XA_out, void *workspace, size_t workspace_bytes, qlora_stream_t stream) {
  if (dtype != QLORA_BF16 && dtype != QLORA_F16) return QLORA_ERR_RANGE;
  DtypeScope scope(dtype == QLORA_F16);
  return qlora_linear_fwd(packed, q, scale2, nf4, t8, M, N, K, static_cast<const qlora_bf16 *>(X),
                          static_cast<const qlora_bf16 *>(A), static_cast<const qlora_bf16 *>(B), r, alpha,
                          static_cast<qlora_bf16 *>(Y), static_cast<qlora_bf16 *>(XA_out), workspace,
                          workspace_bytes, stream);
}

qlora_status qlora_linear_bwd_dt(const uint8_t *packed, const uint8_t *q, const float *scale2, const float nf4[16],
                                 const float t8[256], qlora_dtype dtype, int64_t M, int64_t N, int64_t K,
                                 const void *X, const void *dY, const void *A, const void *B, const void *XA, int r,
                                 float alpha, void *dX, void *dA, void *dB, void *workspace, size_t workspace_bytes,
                                 qlora_stream_t stream) {
  if (dtype != QLORA_BF16 && dtype != QLORA_F16) return QLORA_ERR_RANGE;
  DtypeScope scope(dtype == QLORA_F16);
  return qlora_linear_bwd(packed, q, scale2, nf4, t8, M, N, K, static_cast<const qlora_bf16 *>(X),
                          static_cast<const qlora_bf16 *>(dY), static_cast<const qlora_bf16 *>(A),
                          static_cast<const qlora_bf16 *>(B), static_cast<const qlora_bf16 *>(XA), r, alpha,
                          static_cast<qlora_bf16 *>(dX), static_cast<qlora_bf16 *>(dA), static_cast<qlora_bf16 *>(dB),
                          workspace, workspace_bytes, stream);
}

}  // extern "C"

// Scratch of qlora_linear_fwd_noalloc: a fixed array in device global memory,
// one per GPU that loads the library, shared by every call on that GPU.
static __device__ __align__(256) unsigned char g_noalloc_scratch[QLORA_NOALLOC_SCRATCH_BYTES];

namespace {
void *g_noalloc_ptr[kMaxDevices] = {};

// Device address of g_noalloc_scratch on the current device, looked up once
// per device with that device current (the host-side symbol is only a
// stand-in and must never reach a kernel).
qlora_status noalloc_scratch(void **out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return QLORA_ERR_CUDA;
  std::lock_guard<std::mutex> lk(g_mu);
  if (g_noalloc_ptr[dev] == nullptr) {
    void *p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) return QLORA_ERR_CUDA;
    g_noalloc_ptr[dev] = p;
  }
  *out = g_noalloc_ptr[dev];
  return QLORA_OK;
}
}  // namespace

extern "C" {

qlora_status qlora_linear_fwd_noalloc(const uint8_t *packed, const uint8_t *q, const float *scale2,
                                      const float nf4[16], const float t8[256], int64_t M, int64_t N, int64_t K,
                                      const qlora_bf16 *X, const qlora_bf16 *A, const qlora_bf16 *B, int r,
                                      float alpha, qlora_bf16 *Y, qlora_bf16 *XA_out, qlora_stream_t stream) {
  const Shape s{M, N, K, r};
  qlora_status st = check_linear(packed, q, scale2, nf4, t8, s, alpha);
  if (st != QLORA_OK) return st;
  DeviceInfo d;
  if ((st = device_info(&d)) != QLORA_OK) return st;
  if (fwd_ws_bytes(s, d.sms) > QLORA_NOALLOC_SCRATCH_BYTES) return QLORA_ERR_WORKSPACE;
  void *scratch = nullptr;
  if ((st = noalloc_scratch(&scratch)) != QLORA_OK) return st;
  return qlora_linear_fwd(packed, q, scale2, nf4, t8, M, N, K, X, A, B, r, alpha, Y, XA_out, scratch,
                          QLORA_NOALLOC_SCRATCH_BYTES, stream);
}

void qlora_set_trace_events(void *start, void *stop) {
  t_trace_start = static_cast<cudaEvent_t>(start);
  t_trace_stop = static_cast<cudaEvent_t>(stop);
}

uint64_t qlora_launch_count(void) { return g_launches.load(std::memory_order_relaxed); }

int qlora_debug_fail_allocs(int skip, int n) {
  std::lock_guard<std::mutex> lock(g_inject_mu);
  const int pending = g_inject_fail;
  g_inject_skip = std::max(skip, 0);
  g_inject_fail = std::max(n, 0);
  return pending;
}

qlora_status qlora_selftest_bounded_wait(qlora_stream_t stream) {
  qlora_status st;
  DeviceInfo d;
  if ((st = device_info(&d)) != QLORA_OK) return st;
  selftest_wait_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>();
  g_launches.fetch_add(1, std::memory_order_relaxed);
  return cudaGetLastError() == cudaSuccess ? QLORA_OK : QLORA_ERR_CUDA;
}

uint32_t qlora_device_error(int clear) {
  unsigned int v = 0;
  if (cudaDeviceSynchronize() != cudaSuccess) return 0xFFFFFFFFu;
  if (cudaMemcpyFromSymbol(&v, g_error_word, sizeof v) != cudaSuccess) return 0xFFFFFFFFu;
  if (clear) {
    const unsigned int z = 0;
    if (cudaMemcpyToSymbol(g_error_word, &z, sizeof z) != cudaSuccess) return 0xFFFFFFFFu;
  }
  return v;
}

}  // extern "C"

// ------------------------------------------------ decoder-block chains --
namespace {

// The library's extra streams and fork/join events of this host thread on
// one device (created on first use, kept for the thread's life).
struct BlockStreams {
  bool init = false;
  cudaStream_t side[QLORA_BLOCK_STREAMS - 1] = {};
  cudaEvent_t fork = nullptr;
  cudaEvent_t join[QLORA_BLOCK_STREAMS - 1] = {};
};
thread_local BlockStreams t_block[kMaxDevices];

cudaError_t make_event(cudaEvent_t *e) {
  if (inject_alloc_failure()) return cudaErrorMemoryAllocation;
  return cudaEventCreateWithFlags(e, cudaEventDisableTiming);
}

cudaError_t make_stream(cudaStream_t *s) {
  if (inject_alloc_failure()) return cudaErrorMemoryAllocation;
  return cudaStreamCreateWithFlags(s, cudaStreamNonBlocking);
}

// Destroys whatever a failed first-use setup had created, so that the next
// call starts from nothing.
void release_block_streams(BlockStreams &b) {
  if (b.fork) cudaEventDestroy(b.fork);
  for (int i = 0; i < QLORA_BLOCK_STREAMS - 1; ++i) {
    if (b.side[i]) cudaStreamDestroy(b.side[i]);
    if (b.join[i]) cudaEventDestroy(b.join[i]);
  }
  b = BlockStreams{};
}

qlora_status block_streams(BlockStreams **out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return QLORA_ERR_CUDA;
  BlockStreams &b = t_block[dev];
  if (!b.init) {
    bool ok = make_event(&b.fork) == cudaSuccess;
    for (int i = 0; ok && i < QLORA_BLOCK_STREAMS - 1; ++i)
      ok = make_stream(&b.side[i]) == cudaSuccess && make_event(&b.join[i]) == cudaSuccess;
    if (!ok) {
      cudaGetLastError();
      release_block_streams(b);
      return QLORA_ERR_CUDA;
    }
    b.init = true;
  }
  *out = &b;
  return QLORA_OK;
}

size_t block_slice_bytes(int n, const qlora_linear_desc *desc, int64_t M, int r) {
  size_t m = 0;
  for (int i = 0; i < n; ++i) m = std::max(m, align256(qlora_workspace_bytes(M, desc[i].N, desc[i].K, r)));
  return m;
}

template <class Fn>
qlora_status run_block(int n, const qlora_linear_desc *desc, int64_t M, int r, void *workspace,
                       size_t workspace_bytes, cudaStream_t main, Fn &&one) {
  if (n < 1 || !desc) return n < 1 ? QLORA_ERR_SHAPE : QLORA_ERR_NULL;
  const size_t slice = block_slice_bytes(n, desc, M, r);
  if (slice == 0) return QLORA_ERR_SHAPE;
  const int ns = std::min(n, QLORA_BLOCK_STREAMS);
  if (!workspace || workspace_bytes < slice * ns) return QLORA_ERR_WORKSPACE;
  if (!aligned16(workspace)) return QLORA_ERR_ALIGN;
  BlockStreams *b = nullptr;
  qlora_status st = block_streams(&b);
  if (st != QLORA_OK) return st;
  // fork: the side streams start after everything queued on `main`
  if (cudaEventRecord(b->fork, main) != cudaSuccess) return QLORA_ERR_CUDA;
  for (int j = 1; j < ns; ++j)
    if (cudaStreamWaitEvent(b->side[j - 1], b->fork, 0) != cudaSuccess) return QLORA_ERR_CUDA;
  qlora_status first_err = QLORA_OK;
  for (int i = 0; i < n && first_err == QLORA_OK; ++i) {
    const int j = i % ns;
    cudaStream_t s = j == 0 ? main : b->side[j - 1];
    first_err = one(desc[i], static_cast<uint8_t *>(workspace) + slice * j, slice, s);
  }
  // join: `main` continues after every side stream's work (also on error,
  // so nothing launched is left outside the caller's stream order)
  for (int j = 1; j < ns; ++j)
    if (cudaEventRecord(b->join[j - 1], b->side[j - 1]) != cudaSuccess ||
        cudaStreamWaitEvent(main, b->join[j - 1], 0) != cudaSuccess)
      return QLORA_ERR_CUDA;
  return first_err;
}

}  // namespace

extern "C" {

size_t qlora_block_workspace_bytes(int n, const qlora_linear_desc *desc, int64_t M, int r) {
  if (n < 1 || !desc) return 0;
  return block_slice_bytes(n, desc, M, r) * static_cast<size_t>(std::min(n, QLORA_BLOCK_STREAMS));
}

qlora_status qlora_block_fwd(int n, const qlora_linear_desc *desc, const float nf4[16], const float t8[256],
                             qlora_dtype dtype, int64_t M, int r, float alpha, int save_xa, void *workspace,
                             size_t workspace_bytes, qlora_stream_t stream) {
  if (dtype != QLORA_BF16 && dtype != QLORA_F16) return QLORA_ERR_RANGE;
  return run_block(n, desc, M, r, workspace, workspace_bytes, static_cast<cudaStream_t>(stream),
                   [&](const qlora_linear_desc &d, void *ws, size_t wsb, cudaStream_t s) {
                     return qlora_linear_fwd_dt(d.packed, d.q, d.scale2, nf4, t8, dtype, M, d.N, d.K, d.X, d.A,
                                                d.B, r, alpha, d.Y, save_xa ? d.XA : nullptr, ws, wsb, s);
                   });
}

qlora_status qlora_block_bwd(int n, const qlora_linear_desc *desc, const float nf4[16], const float t8[256],
                             qlora_dtype dtype, int64_t M, int r, float alpha, int save_xa, void *workspace,
                             size_t workspace_bytes, qlora_stream_t stream) {
  if (dtype != QLORA_BF16 && dtype != QLORA_F16) return QLORA_ERR_RANGE;
  return run_block(n, desc, M, r, workspace, workspace_bytes, static_cast<cudaStream_t>(stream),
                   [&](const qlora_linear_desc &d, void *ws, size_t wsb, cudaStream_t s) {
                     return qlora_linear_bwd_dt(d.packed, d.q, d.scale2, nf4, t8, dtype, M, d.N, d.K, d.X, d.dY,
                                                d.A, d.B, save_xa ? d.XA : nullptr, r, alpha, d.dX, d.dA, d.dB,
                                                ws, wsb, s);
                   });
}

}  // extern "C"

// ------------------------------------------------------- paged AdamW --
struct qlora_paged_adamw {
  int device = 0;
  std::vector<int64_t> offset;  // nseg + 1 element offsets
  int64_t total = 0;            // elements (each of master, m, v holds `total` floats)
  int64_t stride = 0;           // floats between master, m and v (total rounded up to 64)
  float *state = nullptr;       // managed: master | m | v
  size_t bytes = 0;
  size_t reserve = 0;
  int where = 0;                // 0: device, 1: host
  bool hints = false;           // the device takes prefetch and placement hints
};

namespace {

// Page the state to `to` (0: device, 1: host) with placement hints and an
// asynchronous prefetch on `st`.
qlora_status adamw_place(qlora_paged_adamw *o, int to, cudaStream_t st) {
  if (o->hints) {
    const int loc = to == 1 ? cudaCpuDeviceId : o->device;
    if (cudaMemAdvise(o->state, o->bytes, cudaMemAdviseSetPreferredLocation, loc) != cudaSuccess ||
        (to == 1 && cudaMemAdvise(o->state, o->bytes, cudaMemAdviseSetAccessedBy, o->device) != cudaSuccess) ||
        cudaMemPrefetchAsync(o->state, o->bytes, loc, st) != cudaSuccess)
      return QLORA_ERR_CUDA;
  }
  o->where = to;
  return QLORA_OK;
}

// One launch per kAdamwMaxSegs segments; `init` selects the start kernel.
qlora_status adamw_launch(qlora_paged_adamw *o, void *const *params, const void *const *grads, bool init,
                          const AdamwHyper &h, cudaStream_t st) {
  DeviceInfo d;
  qlora_status status = device_info(&d);
  if (status != QLORA_OK) return status;
  const int nseg = static_cast<int>(o->offset.size()) - 1;
  for (int s0 = 0; s0 < nseg; s0 += kAdamwMaxSegs) {
    const int n = std::min(kAdamwMaxSegs, nseg - s0);
    AdamwSegs segs;
    std::memset(&segs, 0, sizeof segs);
    for (int i = 0; i < n; ++i) {
      segs.param[i] = params[s0 + i];
      segs.grad[i] = grads ? grads[s0 + i] : nullptr;
      segs.offset[i] = o->offset[s0 + i] - o->offset[s0];
    }
    segs.offset[n] = o->offset[s0 + n] - o->offset[s0];
    segs.nseg = n;
    const int64_t base = o->offset[s0];
    float *master = o->state + base, *m = o->state + o->stride + base, *v = o->state + 2 * o->stride + base;
    const int grid = grid_for(segs.offset[n], 256 * 4, d.sms, 8);
    status = init ? launch_pdl(adamw_init_kernel, grid, 256, 0, st, segs, master, m, v, h.f16)
                  : launch_pdl(adamw_kernel, grid, 256, 0, st, segs, master, m, v, h);
    if (status != QLORA_OK) return status;
  }
  return QLORA_OK;
}

bool finite_nonneg(float x) { return std::isfinite(x) && x >= 0.0f; }

}  // namespace

extern "C" {

int qlora_paged_adamw_placement(size_t free_bytes, size_t state_bytes, size_t reserve_bytes, int current) {
  if (current == 0) return free_bytes < reserve_bytes ? 1 : 0;
  return free_bytes >= state_bytes + reserve_bytes ? 0 : 1;
}

qlora_status qlora_paged_adamw_create(int nseg, const int64_t *counts, qlora_paged_adamw **out) {
  if (!counts || !out) return QLORA_ERR_NULL;
  *out = nullptr;
  if (nseg < 1) return QLORA_ERR_SHAPE;
  auto *o = new (std::nothrow) qlora_paged_adamw();
  if (!o) return QLORA_ERR_CUDA;
  try {
    o->offset.resize(static_cast<size_t>(nseg) + 1);
  } catch (const std::bad_alloc &) {
    delete o;
    return QLORA_ERR_CUDA;
  }
  o->offset[0] = 0;
  for (int i = 0; i < nseg; ++i) {
    if (counts[i] < 1) {
      delete o;
      return QLORA_ERR_SHAPE;
    }
    o->offset[i + 1] = o->offset[i] + counts[i];
  }
  o->total = o->offset[nseg];
  o->stride = (o->total + 63) / 64 * 64;
  o->bytes = static_cast<size_t>(o->stride) * 3 * sizeof(float);
  DeviceInfo d;
  const qlora_status st = device_info(&d);
  if (st != QLORA_OK) {
    delete o;
    return st;
  }
  cudaGetDevice(&o->device);
  int cma = 0;
  cudaDeviceGetAttribute(&cma, cudaDevAttrConcurrentManagedAccess, o->device);
  o->hints = cma != 0;
  void *p = nullptr;
  if (inject_alloc_failure() || cudaMallocManaged(&p, o->bytes, cudaMemAttachGlobal) != cudaSuccess) {
    cudaGetLastError();
    delete o;
    return QLORA_ERR_CUDA;
  }
  o->state = static_cast<float *>(p);
  *out = o;
  return QLORA_OK;
}

void qlora_paged_adamw_destroy(qlora_paged_adamw *opt) {
  if (!opt) return;
  if (opt->state) {
    cudaDeviceSynchronize();
    cudaFree(opt->state);
  }
  delete opt;
}

qlora_status qlora_paged_adamw_set_reserve(qlora_paged_adamw *opt, size_t reserve_bytes) {
  if (!opt) return QLORA_ERR_NULL;
  opt->reserve = reserve_bytes;
  return QLORA_OK;
}

int qlora_paged_adamw_location(const qlora_paged_adamw *opt) { return opt ? opt->where : -1; }

size_t qlora_paged_adamw_state_bytes(const qlora_paged_adamw *opt) { return opt ? opt->bytes : 0; }

qlora_status qlora_paged_adamw_state(const qlora_paged_adamw *opt, float **master, float **m, float **v) {
  if (!opt || !master || !m || !v) return QLORA_ERR_NULL;
  *master = opt->state;
  *m = opt->state + opt->stride;
  *v = opt->state + 2 * opt->stride;
  return QLORA_OK;
}

qlora_status qlora_paged_adamw_init(qlora_paged_adamw *opt, void *const *params, qlora_dtype dtype,
                                    qlora_stream_t stream) {
  if (!opt || !params) return QLORA_ERR_NULL;
  if (dtype != QLORA_BF16 && dtype != QLORA_F16) return QLORA_ERR_RANGE;
  const size_t nseg = opt->offset.size() - 1;
  for (size_t i = 0; i < nseg; ++i) {
    if (!params[i]) return QLORA_ERR_NULL;
    if (reinterpret_cast<uintptr_t>(params[i]) & 1u) return QLORA_ERR_ALIGN;
  }
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  qlora_status status = adamw_place(opt, 0, st);
  if (status != QLORA_OK) return status;
  AdamwHyper h;
  std::memset(&h, 0, sizeof h);
  h.f16 = dtype == QLORA_F16 ? 1 : 0;
  return adamw_launch(opt, params, nullptr, true, h, st);
}

qlora_status qlora_paged_adamw_step(qlora_paged_adamw *opt, void *const *params, const void *const *grads,
                                    qlora_dtype dtype, int64_t t, float lr, float beta1, float beta2, float eps,
                                    float weight_decay, qlora_stream_t stream) {
  if (!opt || !params || !grads) return QLORA_ERR_NULL;
  if (dtype != QLORA_BF16 && dtype != QLORA_F16) return QLORA_ERR_RANGE;
  if (t < 1 || !finite_nonneg(lr) || !finite_nonneg(beta1) || beta1 >= 1.0f || !finite_nonneg(beta2) ||
      beta2 >= 1.0f || !(std::isfinite(eps) && eps > 0.0f) || !finite_nonneg(weight_decay))
    return QLORA_ERR_RANGE;
  const size_t nseg = opt->offset.size() - 1;
  for (size_t i = 0; i < nseg; ++i) {
    if (!params[i] || !grads[i]) return QLORA_ERR_NULL;
    if ((reinterpret_cast<uintptr_t>(params[i]) | reinterpret_cast<uintptr_t>(grads[i])) & 1u)
      return QLORA_ERR_ALIGN;
  }
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  size_t free_b = 0, total_b = 0;
  if (cudaMemGetInfo(&free_b, &total_b) != cudaSuccess) return QLORA_ERR_CUDA;
  const int to = qlora_paged_adamw_placement(free_b, opt->bytes, opt->reserve, opt->where);
  qlora_status status = QLORA_OK;
  if (to != opt->where && (status = adamw_place(opt, to, st)) != QLORA_OK) return status;
  AdamwHyper h;
  h.lr = lr;
  h.b1 = beta1;
  h.b2 = beta2;
  h.eps = eps;
  h.wd = weight_decay;
  h.bc1 = static_cast<float>(1.0 - std::pow(static_cast<double>(beta1), static_cast<double>(t)));
  h.bc2 = static_cast<float>(1.0 - std::pow(static_cast<double>(beta2), static_cast<double>(t)));
  h.f16 = dtype == QLORA_F16 ? 1 : 0;
  if (!(h.bc1 > 0.0f) || !(h.bc2 > 0.0f)) return QLORA_ERR_RANGE;  // beta^t rounds to 1 only for beta = 1
  return adamw_launch(opt, params, grads, false, h, st);
}

}  // extern "C"

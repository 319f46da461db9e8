// C ABI of the W4A8 library: argument validation, schedule selection, tensor
// map encoding and kernel launches. Declarations and the contract of every
// entry point are in include/w4a8.h.
#include <cuda.h>
#include <cuda_runtime.h>

#include <mutex>
#include <utility>

#include "chain.cuh"
#include "gemm.cuh"
#include "kv4_attention.cuh"
#include "pack.cuh"
#include "quantize_act.cuh"
#include "quantize_weights.cuh"
#include "selftest.cuh"
#include "w4a8.h"

namespace w4a8 {

__device__ int g_device_error = 0;

namespace {

constexpr int kMaxDevices = 64;
constexpr int64_t kMaxK = 65536;
// Activation quantizers with at most this many rows (one CTA per row) release
// the next kernel before their dependency wait (see quantize_act.cuh).
constexpr int64_t kEarlyReleaseRows = 64;

struct DeviceInfo {
  bool ready = false;
  int sms = 0;
  int* err = nullptr;  // device address of g_device_error
};
DeviceInfo g_dev[kMaxDevices];
std::mutex g_dev_mu;

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
EncodeTiledFn g_encode = nullptr;

w4a8_status_t cuda_status(cudaError_t e) {
  if (e == cudaSuccess) return W4A8_OK;
  (void)cudaGetLastError();
  return W4A8_ERR_CUDA;
}

w4a8_status_t launch_status() { return cuda_status(cudaGetLastError()); }

// Per-device facts, fetched once with that device current.
w4a8_status_t device_info(DeviceInfo** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return cuda_status(cudaErrorInvalidDevice);
  if (dev < 0 || dev >= kMaxDevices) return W4A8_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_dev_mu);
  DeviceInfo& d = g_dev[dev];
  if (!d.ready) {
    if (cudaDeviceGetAttribute(&d.sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return launch_status();
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_device_error) != cudaSuccess) return launch_status();
    d.err = static_cast<int*>(p);
    if (g_encode == nullptr) {
      void* fn = nullptr;
      cudaDriverEntryPointQueryResult q;
      if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) != cudaSuccess ||
          q != cudaDriverEntryPointSuccess || fn == nullptr)
        return launch_status();
      g_encode = reinterpret_cast<EncodeTiledFn>(fn);
    }
    d.ready = true;
  }
  *out = &d;
  return W4A8_OK;
}

// Launches with programmatic stream serialization: the kernel may start
// while its predecessor in the stream finishes; it waits (griddepcontrol)
// before touching anything the predecessor writes.
// A cluster size above 1 launches thread-block clusters of that many CTAs
// along x.
template <typename... KArgs, typename... Args>
w4a8_status_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                         int cluster, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  int n = 1;
  if (cluster > 1) {
    attr[1].id = cudaLaunchAttributeClusterDimension;
    attr[1].val.clusterDim.x = static_cast<unsigned>(cluster);
    attr[1].val.clusterDim.y = 1;
    attr[1].val.clusterDim.z = 1;
    n = 2;
  }
  cfg.attrs = attr;
  cfg.numAttrs = n;
  return cuda_status(cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...));
}

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

int64_t packed_s1_offset(int64_t N, int64_t K) { return kHeaderBytes + (N / kTileN) * (K / kTileK) * kTileBytes; }
int64_t lut_table_offset(int64_t N, int64_t K) {
  return kHeaderBytes + (N / kTileN) * (K / kTileK) * kLutTileBytesPack;
}
int64_t lut3_table_offset(int64_t N, int64_t K) {
  return kHeaderBytes + (N / kTileN) * (K / kTileK) * kLut3TileBytesPack;
}

// ------------------------------------------------------------------ GEMM
// Resident CTAs per SM of a configuration (shared memory, threads and tensor
// memory permitting), computed once per device.
template <class C>
w4a8_status_t ctas_per_sm(int dev, int* out) {
  static int cache[kMaxDevices] = {};
  if (cache[dev] == 0) {
    if (cudaFuncSetAttribute(w4a8_gemm_kernel<C>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemBytes) !=
        cudaSuccess)
      return launch_status();
    int n = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, w4a8_gemm_kernel<C>, C::kThreads, C::kSmemBytes) !=
        cudaSuccess)
      return launch_status();
    n = n < 512 / C::kTmemCols ? n : 512 / C::kTmemCols;  // every resident CTA must get its TMEM
    cache[dev] = n > 0 ? n : 1;
  }
  *out = cache[dev];
  return W4A8_OK;
}

// Clusters of `split` CTAs of a configuration that can be resident at once
// (0 when a cluster of that size cannot be scheduled), computed once per
// device and size.
template <class C>
w4a8_status_t max_clusters(int dev, int split, int* out) {
  static int cache[kMaxDevices][C::kMaxSplit + 1] = {};
  if (split < 2 || split > C::kMaxSplit) {
    *out = 0;
    return W4A8_OK;
  }
  if (cache[dev][split] == 0) {
    int dummy = 0;
    w4a8_status_t st = ctas_per_sm<C>(dev, &dummy);  // sets the shared-memory attribute
    if (st != W4A8_OK) return st;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(split);
    cfg.blockDim = dim3(C::kThreads);
    cfg.dynamicSmemBytes = C::kSmemBytes;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = static_cast<unsigned>(split);
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, w4a8_gemm_kernel<C>, &cfg) != cudaSuccess) {
      (void)cudaGetLastError();
      n = 0;
    }
    cache[dev][split] = n > 0 ? n : -1;
  }
  *out = cache[dev][split] > 0 ? cache[dev][split] : 0;
  return W4A8_OK;
}

// The activation tensor map: int8 codes as [M, K] bytes, loaded as 128-byte
// rows with the 128-byte swizzle the MMA descriptor expects; or (W4A4) the
// packed 4-bit codes as [M, K / 2] bytes, loaded as plain 64-byte rows that
// the kernel expands in shared memory.
template <class C>
w4a8_status_t launch_gemm_cfg(const void* act, int64_t M, int64_t K, GemmArgs args, int grid,
                              cudaStream_t stream) {
  if (args.split > C::kMaxSplit) return W4A8_ERR_INVALID_ARG;
  CUtensorMap map;
  if constexpr (C::kLut) {
    // fp16 activations [M, K]: 64-value (128-byte) spans, 128-byte swizzle
    const cuuint64_t dims[2] = {static_cast<cuuint64_t>(K), static_cast<cuuint64_t>(M)};
    const cuuint64_t strides[1] = {static_cast<cuuint64_t>(2 * K)};
    const cuuint32_t box[2] = {64u, static_cast<cuuint32_t>(C::BN)};
    const cuuint32_t estr[2] = {1u, 1u};
    if (g_encode(&map, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, const_cast<void*>(act), dims, strides, box, estr,
                 CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                 CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return W4A8_ERR_CUDA;
    return launch_pdl(w4a8_gemm_kernel<C>, dim3(grid), dim3(C::kThreads), C::kSmemBytes, stream, args.split, map,
                      args);
  }
  const int64_t row_bytes = args.a4 ? K / 2 : K;
  const cuuint64_t dims[2] = {static_cast<cuuint64_t>(row_bytes), static_cast<cuuint64_t>(M)};
  const cuuint64_t strides[1] = {static_cast<cuuint64_t>(row_bytes)};
  const cuuint32_t box[2] = {args.a4 ? 64u : 128u, static_cast<cuuint32_t>(C::BN)};
  const cuuint32_t estr[2] = {1u, 1u};
  if (g_encode(&map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(act), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, args.a4 ? CU_TENSOR_MAP_SWIZZLE_NONE : CU_TENSOR_MAP_SWIZZLE_128B,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return W4A8_ERR_CUDA;
  return launch_pdl(w4a8_gemm_kernel<C>, dim3(grid), dim3(C::kThreads), C::kSmemBytes, stream, args.split, map,
                    args);
}

// Tile configurations: tokens per tile, k-blocks per chunk, weight and
// activation ring slots, TMEM ring slots, dequantizer groups, accumulator
// buffers, MMA issuers.
using Cfg16 = GemmCfg<16, 3, 4, 4, 2, 2, 2>;
using Cfg32 = GemmCfg<32, 3, 4, 4, 2, 2, 2>;
using Cfg64 = GemmCfg<64, 2, 6, 6, 2, 2, 2>;
// lookup-table weights against fp16 activations (decode tile sizes; larger M
// uses several 32-token tiles): one k-block per chunk and a third
// dequantizer group (the table lookups, not the weight bytes, limit it)
using CfgL16 = GemmCfg<16, 1, 12, 6, 3, 2, 2, 1>;
using CfgL32 = GemmCfg<32, 1, 6, 6, 3, 2, 2, 1>;
// the same with 3-bit indices in bit planes
using CfgL3_16 = GemmCfg<16, 1, 12, 6, 3, 2, 2, 3>;
using CfgL3_32 = GemmCfg<32, 1, 6, 6, 3, 2, 2, 3>;
using Cfg128 = GemmCfg<128, 4, 2, 2, 1, 2, 2>;

size_t ws_counter_bytes(int64_t M, int64_t N) {
  const int64_t tiles = (N / kTileN) * ((M + 15) / 16);  // the most tiles any block_m gives
  return static_cast<size_t>((tiles * 4 + 255) / 256 * 256);
}

// Activation quantizers (one CTA per token), dispatched on the row length;
// BITS = 8 writes int8 codes, 4 packed 4-bit codes.
template <int BITS>
w4a8_status_t launch_quantize_dynamic(const __half* a, int64_t M, int64_t K, void* codes, __half* s, int32_t* rowsum,
                                      cudaStream_t st) {
  const dim3 grid(static_cast<unsigned>(M));
  const int64_t nvec = K / 8;
  const int early = M <= kEarlyReleaseRows ? 1 : 0;
  if (nvec <= 128)
    return launch_pdl(quantize_act_kernel<128, 1, BITS>, grid, dim3(128), 0, st, 1, a, K, codes, s, rowsum, early);
  if (nvec <= 256)
    return launch_pdl(quantize_act_kernel<256, 1, BITS>, grid, dim3(256), 0, st, 1, a, K, codes, s, rowsum, early);
  if (nvec <= 512)
    return launch_pdl(quantize_act_kernel<256, 2, BITS>, grid, dim3(256), 0, st, 1, a, K, codes, s, rowsum, early);
  if (nvec <= 1024)
    return launch_pdl(quantize_act_kernel<256, 4, BITS>, grid, dim3(256), 0, st, 1, a, K, codes, s, rowsum, early);
  if (nvec <= 2048)
    return launch_pdl(quantize_act_kernel<256, 8, BITS>, grid, dim3(256), 0, st, 1, a, K, codes, s, rowsum, early);
  if (nvec <= 4096)
    return launch_pdl(quantize_act_kernel<512, 8, BITS>, grid, dim3(512), 0, st, 1, a, K, codes, s, rowsum, early);
  return launch_pdl(quantize_act_kernel<1024, 8, BITS>, grid, dim3(1024), 0, st, 1, a, K, codes, s, rowsum, early);
}

template <int BITS>
w4a8_status_t launch_quantize_static(const __half* a, int64_t M, int64_t K, const __half* sc, void* codes,
                                     __half* so, int32_t* rowsum, cudaStream_t st) {
  const dim3 grid(static_cast<unsigned>(M));
  const int64_t nvec = K / 8;
  const int early = M <= kEarlyReleaseRows ? 1 : 0;
  if (nvec <= 128)
    return launch_pdl(quantize_act_static_kernel<128, 1, BITS>, grid, dim3(128), 0, st, 1, a, K, sc, codes, so,
                      rowsum, early);
  if (nvec <= 512)
    return launch_pdl(quantize_act_static_kernel<256, 2, BITS>, grid, dim3(256), 0, st, 1, a, K, sc, codes, so,
                      rowsum, early);
  if (nvec <= 2048)
    return launch_pdl(quantize_act_static_kernel<256, 8, BITS>, grid, dim3(256), 0, st, 1, a, K, sc, codes, so,
                      rowsum, early);
  return launch_pdl(quantize_act_static_kernel<1024, 8, BITS>, grid, dim3(1024), 0, st, 1, a, K, sc, codes, so,
                    rowsum, early);
}

w4a8_status_t check_quantize_args(const void* A, int64_t M, int64_t K, const void* codes, const void* sA,
                                  const void* rowsum) {
  if (M < 0 || K < 0) return W4A8_ERR_INVALID_ARG;
  if (K == 0 || K % 8 != 0 || K > kMaxK || M > INT32_MAX) return W4A8_ERR_UNSUPPORTED_SHAPE;
  if (M == 0) return W4A8_OK;
  if (A == nullptr || codes == nullptr || sA == nullptr) return W4A8_ERR_INVALID_ARG;
  if (!aligned(A, 16) || !aligned(codes, 16) || !aligned(sA, 2) || !aligned(rowsum, 4)) return W4A8_ERR_MISALIGNED;
  return W4A8_OK;
}

}  // namespace

// Host-side checks shared by every GEMM entry point: options, shape limits,
// pointers and alignment. W4A8_OK with M == 0 or N == 0 means "nothing to do".
w4a8_status_t check_gemm_args(const void* A8, const void* sA, const int32_t* rowsum, const void* packed, int64_t M,
                              int64_t N, int64_t K, const void* Y, const int32_t* acc, const void* ws,
                              const w4a8_gemm_opts_t& o, int lut) {
  if (o.reserved != 0 || o.schedule < 0 || o.schedule > 3 || o.max_ctas < 0) return W4A8_ERR_INVALID_ARG;
  if (!(o.block_m == 0 || o.block_m == 16 || o.block_m == 32 || o.block_m == 64 || o.block_m == 128))
    return W4A8_ERR_INVALID_ARG;
  if (lut && o.block_m > 32) return W4A8_ERR_INVALID_ARG;
  if (M < 0 || N < 0 || K < 0) return W4A8_ERR_INVALID_ARG;
  if (K == 0 || K % kTileK != 0 || K > kMaxK || N % kTileN != 0) return W4A8_ERR_UNSUPPORTED_SHAPE;
  if (M > INT32_MAX || N > INT32_MAX || (N > 0 && M > (int64_t(1) << 62) / N)) return W4A8_ERR_UNSUPPORTED_SHAPE;
  if (M == 0 || N == 0) return W4A8_OK;
  if ((Y == nullptr) == (acc == nullptr)) return W4A8_ERR_INVALID_ARG;
  if (A8 == nullptr || packed == nullptr || (!lut && (rowsum == nullptr || (acc == nullptr && sA == nullptr))))
    return W4A8_ERR_INVALID_ARG;
  if (!aligned(A8, 16) || !aligned(packed, 16) || !aligned(Y, 16) || !aligned(acc, 16) || !aligned(sA, 2) ||
      !aligned(rowsum, 4) || !aligned(ws, 256))
    return W4A8_ERR_MISALIGNED;
  return W4A8_OK;
}

// A8: the int8 activation codes [M, K], or with a4 the packed 4-bit codes
// [M, K / 2] (W4A4).
w4a8_status_t gemm_impl(const void* A8, const void* sA, const int32_t* rowsum, const void* packed, int64_t M,
                        int64_t N, int64_t K, void* Y, int32_t* acc, void* ws, size_t ws_bytes,
                        const w4a8_gemm_opts_t* opts, cudaStream_t stream, int a4 = 0, int lut = 0) {
  w4a8_gemm_opts_t o = {0, 0, 0, 0};
  if (opts != nullptr) o = *opts;
  {
    const w4a8_status_t v = check_gemm_args(A8, sA, rowsum, packed, M, N, K, Y, acc, ws, o, lut);
    if (v != W4A8_OK || M == 0 || N == 0) return v;
  }
  DeviceInfo* dev = nullptr;
  w4a8_status_t st = device_info(&dev);
  if (st != W4A8_OK) return st;

  // Tokens per tile: the smallest of 16 / 32 that holds M up to 32 tokens;
  // up to 64 tokens, two 32-token tiles when every tile then still gets a
  // cluster of two or more CTAs (the k-range split reduced on chip), else one
  // 64-token tile; up to 128 tokens, four 32-token tiles as whole tiles when
  // they fit one wave (one 128-token tile per channel tile would leave most
  // SMs idle: measured, 128 tokens, 4096 x 4096: 12.2 -> 10.8 us; 4096 x
  // 14336: 30.4 -> 25.8 us); beyond, 128.
  const int n_tiles = static_cast<int>(N / kTileN);
  int bn = o.block_m;
  bool whole_small = false;  // 32-token tiles chosen for 65-128 tokens: no stream-K
  if (bn == 0) {
    if (M <= 16) {
      bn = 16;
    } else if (M <= 32 || lut) {
      bn = 32;
    } else if (M <= 64) {
      bn = 2 * (2 * static_cast<int64_t>(n_tiles)) <= dev->sms ? 32 : 64;
    } else if (M <= 128 && 4 * static_cast<int64_t>(n_tiles) <= dev->sms) {
      bn = 32;
      whole_small = true;
    } else {
      bn = 128;
    }
  }
  const int m_tiles = static_cast<int>((M + bn - 1) / bn);
  const int64_t num_tiles64 = static_cast<int64_t>(n_tiles) * m_tiles;
  if (num_tiles64 > INT32_MAX) return W4A8_ERR_UNSUPPORTED_SHAPE;
  const int num_tiles = static_cast<int>(num_tiles64);
  const int KB = static_cast<int>(K / kTileK);
  int dev_id = 0;
  cudaGetDevice(&dev_id);
  int per_sm = 1;
  if (lut == 3) {
    st = bn == 16 ? ctas_per_sm<CfgL3_16>(dev_id, &per_sm) : ctas_per_sm<CfgL3_32>(dev_id, &per_sm);
  } else if (lut) {
    st = bn == 16 ? ctas_per_sm<CfgL16>(dev_id, &per_sm) : ctas_per_sm<CfgL32>(dev_id, &per_sm);
  } else {
    switch (bn) {
      case 16: st = ctas_per_sm<Cfg16>(dev_id, &per_sm); break;
      case 32: st = ctas_per_sm<Cfg32>(dev_id, &per_sm); break;
      case 64: st = ctas_per_sm<Cfg64>(dev_id, &per_sm); break;
      default: st = ctas_per_sm<Cfg128>(dev_id, &per_sm); break;
    }
  }
  if (st != W4A8_OK) return st;
  int max_ctas = dev->sms * per_sm;
  if (o.max_ctas > 0 && o.max_ctas < max_ctas) max_ctas = o.max_ctas;

  // Cluster split: the largest split (<= 4, <= KB) whose clusters can all
  // be resident with one tile each. Chosen automatically when the tiles
  // fill at most half of the SMs (each tile then gets two or more CTAs).
  int split = 1;
  if (bn <= 32 && (o.schedule == 3 || (o.schedule == 0 && o.max_ctas == 0 && 2 * num_tiles <= dev->sms))) {
    for (int S = 4; S >= 2 && split == 1; --S) {
      if (S > KB) continue;
      int nclu = 0;
      if (lut == 3) {
        st = bn == 16 ? max_clusters<CfgL3_16>(dev_id, S, &nclu) : max_clusters<CfgL3_32>(dev_id, S, &nclu);
      } else if (lut) {
        st = bn == 16 ? max_clusters<CfgL16>(dev_id, S, &nclu) : max_clusters<CfgL32>(dev_id, S, &nclu);
      } else {
        st = bn == 16 ? max_clusters<Cfg16>(dev_id, S, &nclu) : max_clusters<Cfg32>(dev_id, S, &nclu);
      }
      if (st != W4A8_OK) return st;
      if (num_tiles <= nclu && num_tiles * S <= max_ctas) split = S;
    }
  }
  if (o.schedule == 3 && split == 1) return W4A8_ERR_UNSUPPORTED_SHAPE;

  const size_t need_ws = ws_counter_bytes(M, N) + static_cast<size_t>(M) * N * 4;
  if (a4) {
    // W4A4: expand the packed codes once into the workspace's scratch tail,
    // then run the int8 GEMM on them (expanding inside the GEMM repeats the
    // work for every output tile and, with one producer warp, limits the
    // activation rate). Without room for the tail the GEMM expands them
    // itself.
    // The expanded codes occupy the LAST M * K bytes of the workspace (from a
    // 256-byte boundary): a workspace sized for (M, N, K) then serves every
    // smaller shape without its scratch ever touching a zero-filled prefix.
    const size_t codes = static_cast<size_t>(M) * K;
    const size_t tail = ws_bytes >= codes ? (ws_bytes - codes) / 256 * 256 : 0;
    if (ws != nullptr && ws_bytes >= codes && tail >= need_ws) {
      int8_t* A8x = static_cast<int8_t*>(ws) + tail;
      const int64_t units = static_cast<int64_t>(codes / 16);
      const int64_t blocks = (units + 255) / 256;
      const int grid_x = static_cast<int>(blocks < 8L * dev->sms ? blocks : 8L * dev->sms);
      st = launch_pdl(expand_act4_kernel, dim3(grid_x), dim3(256), 0, stream, 1, static_cast<const uint2*>(A8),
                      units, reinterpret_cast<uint4*>(A8x));
      if (st != W4A8_OK) return st;
      return gemm_impl(A8x, sA, rowsum, packed, M, N, K, Y, acc, ws, tail, opts, stream, 0);
    }
  }
  const bool ws_ok = ws != nullptr && ws_bytes >= need_ws;
  // Tiles split stream-K (the rest go whole, round robin): everything when
  // the tiles do not fill one wave, else the tiles beyond the full waves, so
  // that every CTA gets the same number of k-blocks.
  int sk_tiles = 0;
  if (split > 1) {
    sk_tiles = 0;
  } else if (o.schedule == 2) {
    if (!ws_ok) return W4A8_ERR_WORKSPACE;
    sk_tiles = num_tiles;
  } else if (o.schedule == 0 && ws_ok && bn <= 32 && !whole_small) {
    // Token tiles of up to 32: with fewer tiles than CTAs (and no cluster
    // split) every tile is split over all CTAs, partial sums reduced through
    // the workspace. With at least a wave of tiles, the tiles of the last,
    // partial wave are split that way only when whole tiles would leave the
    // CTAs idle for more than about 20 k-blocks each on average (measured
    // break-even against the cost of the partial-sum reduction). Token tiles
    // of 64 and more always go whole: their partial tiles (64 x 128 int32
    // sums and up, one global atomic per element) measured slower than idle
    // CTAs on every such shape.
    if (num_tiles < max_ctas) {
      sk_tiles = num_tiles;
    } else {
      const int64_t rem = num_tiles % max_ctas;
      const int64_t idle_kb = rem == 0 ? 0 : (max_ctas - rem) * static_cast<int64_t>(KB) / max_ctas;
      sk_tiles = idle_kb > 20 ? static_cast<int>(rem) : 0;
    }
  }
  int grid;
  if (split > 1) {
    grid = num_tiles * split;
  } else if (sk_tiles == num_tiles) {
    const int64_t units = static_cast<int64_t>(num_tiles) * KB;
    grid = static_cast<int>(units < max_ctas ? units : max_ctas);
  } else {
    grid = num_tiles < max_ctas ? num_tiles : max_ctas;
  }

  GemmArgs a;
  a.tiles = static_cast<const uint8_t*>(packed) + kHeaderBytes;
  a.s1 = lut ? nullptr : reinterpret_cast<const __half*>(static_cast<const uint8_t*>(packed) + packed_s1_offset(N, K));
  a.lut_table = lut == 3 ? reinterpret_cast<const __half*>(static_cast<const uint8_t*>(packed) + lut3_table_offset(N, K))
                : lut ? reinterpret_cast<const __half*>(static_cast<const uint8_t*>(packed) + lut_table_offset(N, K))
                      : nullptr;
  a.sA = static_cast<const __half*>(sA);
  a.rowsum = rowsum;
  a.Y = static_cast<__half*>(Y);
  a.acc_out = acc;
  a.ws_cnt = sk_tiles > 0 ? static_cast<int32_t*>(ws) : nullptr;
  a.ws_acc = sk_tiles > 0 ? reinterpret_cast<int32_t*>(static_cast<uint8_t*>(ws) + ws_counter_bytes(M, N)) : nullptr;
  a.err = dev->err;
  a.M = static_cast<int>(M);
  a.N = static_cast<int>(N);
  a.KB = KB;
  a.m_tiles = m_tiles;
  a.num_tiles = num_tiles;
  a.sk_tiles = sk_tiles;
  a.split = split;
  // bands of 16 token tiles (16 x 128 tokens of activation rows shared in L2
  // by the CTAs of a wave) when the activation codes exceed ~a quarter of L2
  a.band = static_cast<int64_t>(M) * K > (int64_t(32) << 20) ? 16 : 0;
  a.a4 = a4;
  if (lut) {
    a.sA = nullptr;
    a.rowsum = nullptr;
    if (lut == 3)
      return bn == 16 ? launch_gemm_cfg<CfgL3_16>(A8, M, K, a, grid, stream)
                      : launch_gemm_cfg<CfgL3_32>(A8, M, K, a, grid, stream);
    return bn == 16 ? launch_gemm_cfg<CfgL16>(A8, M, K, a, grid, stream)
                    : launch_gemm_cfg<CfgL32>(A8, M, K, a, grid, stream);
  }
  switch (bn) {
    case 16: return launch_gemm_cfg<Cfg16>(A8, M, K, a, grid, stream);
    case 32: return launch_gemm_cfg<Cfg32>(A8, M, K, a, grid, stream);
    case 64: return launch_gemm_cfg<Cfg64>(A8, M, K, a, grid, stream);
    default: return launch_gemm_cfg<Cfg128>(A8, M, K, a, grid, stream);
  }
}


// ------------------------------------------------------------- GEMM chain
using CfgChain = GemmCfg<kChainMaxM, 3, 4, 4, 2, 2, 2>;

// Per-link split and workspace layout of a chain on a device with `sms` SMs:
// counters (done[n], ready[n], exits) first, then per link with split > 1
// its tickets and partial sums, each from a 256-byte boundary.
struct ChainPlan {
  int split[kChainMaxLinks];
  int seg0[kChainMaxLinks];
  size_t ticket_off[kChainMaxLinks];
  size_t part_off[kChainMaxLinks];
  size_t total;
};

size_t round256u(size_t x) { return (x + 255) / 256 * 256; }

void chain_plan(const w4a8_chain_link_t* links, int n, int sms, ChainPlan* p) {
  size_t off = round256u(static_cast<size_t>(2 * n + 1) * 4);
  int seg = 0;
  for (int j = 0; j < n; ++j) {
    const int T = static_cast<int>(links[j].N / kTileN), KB = static_cast<int>(links[j].K / kTileK);
    int S = 1;
    for (int s2 = 4; s2 >= 2; --s2)
      if (T * s2 <= sms && s2 <= KB) {
        S = s2;
        break;
      }
    p->split[j] = S;
    p->seg0[j] = seg;
    seg += T * S;
    p->ticket_off[j] = p->part_off[j] = 0;
    if (S > 1) {
      p->ticket_off[j] = off;
      off += round256u(static_cast<size_t>(T) * 4);
      p->part_off[j] = off;
      off += round256u(static_cast<size_t>(T) * S * static_cast<size_t>(links[j].M) * kTileN * 4);
    }
  }
  p->total = off;
}

w4a8_status_t check_chain_links(const w4a8_chain_link_t* links, int32_t n) {
  if (links == nullptr || n < 1 || n > kChainMaxLinks) return W4A8_ERR_INVALID_ARG;
  for (int j = 0; j < n; ++j) {
    const w4a8_chain_link_t& L = links[j];
    if (L.M < 1 || L.N < 1 || L.K < 1) return W4A8_ERR_INVALID_ARG;
    if (L.M > kChainMaxM || L.N % kTileN != 0 || L.N > INT32_MAX || L.K % kTileK != 0 || L.K > kMaxK)
      return W4A8_ERR_UNSUPPORTED_SHAPE;
    if (L.A == nullptr || L.packed == nullptr || L.A8 == nullptr || L.sA == nullptr || L.rowsum == nullptr ||
        L.Y == nullptr)
      return W4A8_ERR_INVALID_ARG;
    if (!aligned(L.A, 16) || !aligned(L.packed, 16) || !aligned(L.A8, 16) || !aligned(L.Y, 16) ||
        !aligned(L.sA, 2) || !aligned(L.rowsum, 4))
      return W4A8_ERR_MISALIGNED;
  }
  return W4A8_OK;
}

w4a8_status_t chain_sms(int* sms) {
  DeviceInfo* dev = nullptr;
  const w4a8_status_t st = device_info(&dev);
  if (st != W4A8_OK) return st;
  *sms = dev->sms;
  return W4A8_OK;
}

// ------------------------------------------------------------ 4-bit KV cache
constexpr int64_t kKvMaxLen = int64_t(1) << 24;

int64_t kv_splits(int64_t Lmax) { return (Lmax + kKvChunk - 1) / kKvChunk; }
int kv_heads_per_cta(int64_t G) { return G % 4 == 0 ? 4 : G % 2 == 0 ? 2 : 1; }
int64_t round256(int64_t x) { return (x + 255) / 256 * 256; }

// Shape check of the attention call; 0 = fine.
w4a8_status_t check_kv_shape(int64_t B, int64_t Hq, int64_t Hkv, int64_t Lmax, int32_t D) {
  if (B < 0 || Hq < 0 || Hkv < 0 || Lmax < 0) return W4A8_ERR_INVALID_ARG;
  if (D != kKvD || Hkv == 0 || Lmax == 0 || Hq % Hkv != 0 || Lmax > kKvMaxLen || B > 65535 || Hq > 65536)
    return W4A8_ERR_UNSUPPORTED_SHAPE;
  if (Hq > 0 && Hkv * ((Hq / Hkv) / kv_heads_per_cta(Hq / Hkv)) > 65535) return W4A8_ERR_UNSUPPORTED_SHAPE;
  return W4A8_OK;
}


w4a8_status_t kv_quantize_launch(const void* X, int64_t n, const int32_t* pos, int64_t H, int64_t Lmax,
                                 uint8_t* codes, uint32_t* params, cudaStream_t stream) {
  DeviceInfo* dev = nullptr;
  w4a8_status_t st = device_info(&dev);
  if (st != W4A8_OK) return st;
  KvQuantArgs a;
  a.x = static_cast<const __half*>(X);
  a.n = n;
  a.codes = codes;
  a.params = params;
  a.pos = pos;
  a.H = H;
  a.Lmax = Lmax;
  a.err = dev->err;
  const int64_t blocks = (n + kKvWarps - 1) / kKvWarps;
  const int64_t cap = static_cast<int64_t>(dev->sms) * 8;
  return launch_pdl(kv4_quantize_kernel, dim3(static_cast<unsigned>(blocks < cap ? blocks : cap)), dim3(kKvThreads),
                    0, stream, 1, a);
}

}  // namespace w4a8

using namespace w4a8;

extern "C" {

const char* w4a8_status_string(int status) {
  switch (status) {
    case W4A8_OK: return "W4A8_OK";
    case W4A8_ERR_INVALID_ARG: return "W4A8_ERR_INVALID_ARG";
    case W4A8_ERR_UNSUPPORTED_SHAPE: return "W4A8_ERR_UNSUPPORTED_SHAPE";
    case W4A8_ERR_MISALIGNED: return "W4A8_ERR_MISALIGNED";
    case W4A8_ERR_WORKSPACE: return "W4A8_ERR_WORKSPACE";
    case W4A8_ERR_CUDA: return "W4A8_ERR_CUDA";
    case W4A8_ERR_DEVICE: return "W4A8_ERR_DEVICE";
    default: return "W4A8_ERR_UNKNOWN";
  }
}

int w4a8_version(void) { return 100; }

w4a8_status_t w4a8_quantize_act(const void* A, int64_t M, int64_t K, int8_t* A8, void* sA, int32_t* rowsum,
                                w4a8_stream_t stream) {
  const w4a8_status_t st = check_quantize_args(A, M, K, A8, sA, rowsum);
  if (st != W4A8_OK || M == 0) return st;
  return launch_quantize_dynamic<8>(static_cast<const __half*>(A), M, K, A8, static_cast<__half*>(sA), rowsum,
                                    reinterpret_cast<cudaStream_t>(stream));
}

w4a8_status_t w4a8_quantize_act_static(const void* A, int64_t M, int64_t K, const void* s, int8_t* A8, void* sA,
                                       int32_t* rowsum, w4a8_stream_t stream) {
  const w4a8_status_t st = check_quantize_args(A, M, K, A8, sA, rowsum);
  if (st != W4A8_OK || M == 0) return st;
  if (s == nullptr) return W4A8_ERR_INVALID_ARG;
  if (!aligned(s, 2)) return W4A8_ERR_MISALIGNED;
  return launch_quantize_static<8>(static_cast<const __half*>(A), M, K, static_cast<const __half*>(s), A8,
                                   static_cast<__half*>(sA), rowsum, reinterpret_cast<cudaStream_t>(stream));
}

w4a8_status_t w4a4_quantize_act(const void* A, int64_t M, int64_t K, uint8_t* A4, void* sA, int32_t* rowsum,
                                w4a8_stream_t stream) {
  const w4a8_status_t st = check_quantize_args(A, M, K, A4, sA, rowsum);
  if (st != W4A8_OK || M == 0) return st;
  return launch_quantize_dynamic<4>(static_cast<const __half*>(A), M, K, A4, static_cast<__half*>(sA), rowsum,
                                    reinterpret_cast<cudaStream_t>(stream));
}

w4a8_status_t w4a4_quantize_act_static(const void* A, int64_t M, int64_t K, const void* s, uint8_t* A4, void* sA,
                                       int32_t* rowsum, w4a8_stream_t stream) {
  const w4a8_status_t st = check_quantize_args(A, M, K, A4, sA, rowsum);
  if (st != W4A8_OK || M == 0) return st;
  if (s == nullptr) return W4A8_ERR_INVALID_ARG;
  if (!aligned(s, 2)) return W4A8_ERR_MISALIGNED;
  return launch_quantize_static<4>(static_cast<const __half*>(A), M, K, static_cast<const __half*>(s), A4,
                                   static_cast<__half*>(sA), rowsum, reinterpret_cast<cudaStream_t>(stream));
}

w4a8_status_t w4a8_quantize_weights(const float* W, int64_t N, int64_t K, int32_t group, uint8_t* q, uint8_t* z,
                                    uint8_t* s2, void* s1, w4a8_stream_t stream) {
  if (N < 0 || K < 0) return W4A8_ERR_INVALID_ARG;
  if (group != 128 || K == 0 || K % 128 != 0 || K > kMaxK || N > INT32_MAX) return W4A8_ERR_UNSUPPORTED_SHAPE;
  if (N == 0) return W4A8_OK;
  if (W == nullptr || q == nullptr || z == nullptr || s2 == nullptr || s1 == nullptr) return W4A8_ERR_INVALID_ARG;
  if (!aligned(W, 16) || !aligned(q, 16) || !aligned(s1, 2)) return W4A8_ERR_MISALIGNED;
  quantize_weights_kernel<256><<<static_cast<int>(N), 256, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
      W, K, q, z, s2, static_cast<__half*>(s1));
  return launch_status();
}

size_t w4a8_packed_bytes(int64_t N, int64_t K, int32_t group) {
  if (group != 128 || N <= 0 || K <= 0 || N % 128 != 0 || K % 128 != 0 || K > kMaxK) return 0;
  return static_cast<size_t>(packed_s1_offset(N, K) + (2 * N + 15) / 16 * 16);
}

w4a8_status_t w4a8_pack_weights(const uint8_t* q, const uint8_t* z, const uint8_t* s2, const void* s1, int64_t N,
                                int64_t K, int32_t group, void* packed, size_t packed_bytes,
                                w4a8_stream_t stream) {
  if (N < 0 || K < 0) return W4A8_ERR_INVALID_ARG;
  if (group != 128 || N == 0 || K == 0 || N % 128 != 0 || K % 128 != 0 || K > kMaxK)
    return W4A8_ERR_UNSUPPORTED_SHAPE;
  if (q == nullptr || z == nullptr || s2 == nullptr || s1 == nullptr || packed == nullptr)
    return W4A8_ERR_INVALID_ARG;
  if (!aligned(q, 16) || !aligned(s1, 2) || !aligned(packed, 16)) return W4A8_ERR_MISALIGNED;
  if (packed_bytes < w4a8_packed_bytes(N, K, group)) return W4A8_ERR_INVALID_ARG;
  DeviceInfo* dev = nullptr;
  if (const w4a8_status_t e = device_info(&dev); e != W4A8_OK) return e;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  uint8_t* blob = static_cast<uint8_t*>(packed);
  const int64_t chunks = N * (K / 32);
  const int64_t blocks1 = (chunks + 255) / 256;
  pack_codes_kernel<<<static_cast<int>(blocks1 < 65535 * 16 ? blocks1 : 65535 * 16), 256, 0, st>>>(
      q, N, K, blob + kHeaderBytes, dev->err);
  if (cudaPeekAtLastError() != cudaSuccess) return launch_status();
  const int64_t metas = N * (K / 128);
  const int64_t blocks2 = (metas + 255) / 256;
  pack_meta_kernel<<<static_cast<int>(blocks2 < 65535 ? blocks2 : 65535), 256, 0, st>>>(
      z, s2, static_cast<const __half*>(s1), N, K, blob, packed_s1_offset(N, K), dev->err);
  return launch_status();
}

size_t w4a8_gemm_workspace_bytes(int64_t M, int64_t N, int64_t K) {
  (void)K;
  if (M <= 0 || N <= 0) return 0;
  return ws_counter_bytes(M, N) + static_cast<size_t>(M) * N * 4;
}

size_t w4a4_gemm_workspace_bytes(int64_t M, int64_t N, int64_t K) {
  const size_t base = w4a8_gemm_workspace_bytes(M, N, K);
  if (base == 0 || K <= 0) return base;
  return (base + 255) / 256 * 256 + static_cast<size_t>(M) * K;
}

w4a8_status_t w4a8_gemm(const int8_t* A8, const void* sA, const int32_t* rowsum, const void* packed, int64_t M,
                        int64_t N, int64_t K, void* Y, void* workspace, size_t workspace_bytes, w4a8_stream_t stream) {
  return gemm_impl(A8, sA, rowsum, packed, M, N, K, Y, nullptr, workspace, workspace_bytes, nullptr,
                   reinterpret_cast<cudaStream_t>(stream));
}

w4a8_status_t w4a8_gemm_debug_acc(const int8_t* A8, const int32_t* rowsum, const void* packed, int64_t M, int64_t N,
                                  int64_t K, int32_t* acc, void* workspace, size_t workspace_bytes,
                                  w4a8_stream_t stream) {
  return gemm_impl(A8, nullptr, rowsum, packed, M, N, K, nullptr, acc, workspace, workspace_bytes, nullptr,
                   reinterpret_cast<cudaStream_t>(stream));
}

w4a8_status_t w4a8_gemm_ex(const int8_t* A8, const void* sA, const int32_t* rowsum, const void* packed, int64_t M,
                           int64_t N, int64_t K, void* Y, int32_t* acc, void* workspace, size_t workspace_bytes,
                           const w4a8_gemm_opts_t* opts, w4a8_stream_t stream) {
  return gemm_impl(A8, sA, rowsum, packed, M, N, K, Y, acc, workspace, workspace_bytes, opts,
                   reinterpret_cast<cudaStream_t>(stream));
}

w4a8_status_t w4a4_gemm(const uint8_t* A4, const void* sA, const int32_t* rowsum, const void* packed, int64_t M,
                        int64_t N, int64_t K, void* Y, void* workspace, size_t workspace_bytes, w4a8_stream_t stream) {
  return gemm_impl(A4, sA, rowsum, packed, M, N, K, Y, nullptr, workspace, workspace_bytes, nullptr,
                   reinterpret_cast<cudaStream_t>(stream), 1);
}

w4a8_status_t w4a4_gemm_ex(const uint8_t* A4, const void* sA, const int32_t* rowsum, const void* packed, int64_t M,
                           int64_t N, int64_t K, void* Y, int32_t* acc, void* workspace, size_t workspace_bytes,
                           const w4a8_gemm_opts_t* opts, w4a8_stream_t stream) {
  return gemm_impl(A4, sA, rowsum, packed, M, N, K, Y, acc, workspace, workspace_bytes, opts,
                   reinterpret_cast<cudaStream_t>(stream), 1);
}

size_t w4lut_packed_bytes(int64_t N, int64_t K, int32_t group) {
  if (group != 128 || N <= 0 || K <= 0 || N % 128 != 0 || K % 128 != 0 || K > kMaxK) return 0;
  return static_cast<size_t>(lut_table_offset(N, K) + 64);
}

w4a8_status_t w4lut_pack_weights(const uint8_t* q, const void* s, const void* table, int64_t N, int64_t K,
                                 int32_t group, void* packed, size_t packed_bytes, w4a8_stream_t stream) {
  if (N < 0 || K < 0) return W4A8_ERR_INVALID_ARG;
  if (group != 128 || N == 0 || K == 0 || N % 128 != 0 || K % 128 != 0 || K > kMaxK)
    return W4A8_ERR_UNSUPPORTED_SHAPE;
  if (q == nullptr || s == nullptr || table == nullptr || packed == nullptr) return W4A8_ERR_INVALID_ARG;
  if (!aligned(q, 16) || !aligned(s, 2) || !aligned(table, 2) || !aligned(packed, 16)) return W4A8_ERR_MISALIGNED;
  if (packed_bytes < w4lut_packed_bytes(N, K, group)) return W4A8_ERR_INVALID_ARG;
  DeviceInfo* dev = nullptr;
  if (const w4a8_status_t e = device_info(&dev); e != W4A8_OK) return e;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  uint8_t* blob = static_cast<uint8_t*>(packed);
  const int64_t chunks = N * (K / 32);
  const int64_t blocks1 = (chunks + 255) / 256;
  lut_pack_codes_kernel<<<static_cast<int>(blocks1 < 65535 * 16 ? blocks1 : 65535 * 16), 256, 0, st>>>(
      q, N, K, blob + kHeaderBytes, dev->err);
  if (cudaPeekAtLastError() != cudaSuccess) return launch_status();
  const int64_t metas = N * (K / 128);
  const int64_t blocks2 = (metas + 255) / 256;
  lut_pack_meta_kernel<<<static_cast<int>(blocks2 < 65535 ? blocks2 : 65535), 256, 0, st>>>(
      static_cast<const __half*>(s), static_cast<const __half*>(table), N, K, blob, lut_table_offset(N, K));
  return launch_status();
}

w4a8_status_t w4lut_gemm(const void* A, const void* packed, int64_t M, int64_t N, int64_t K, void* Y,
                         void* workspace, size_t workspace_bytes, w4a8_stream_t stream) {
  return gemm_impl(A, nullptr, nullptr, packed, M, N, K, Y, nullptr, workspace, workspace_bytes, nullptr,
                   reinterpret_cast<cudaStream_t>(stream), 0, 1);
}

w4a8_status_t w4lut_gemm_ex(const void* A, const void* packed, int64_t M, int64_t N, int64_t K, void* Y, float* acc,
                            void* workspace, size_t workspace_bytes, const w4a8_gemm_opts_t* opts,
                            w4a8_stream_t stream) {
  return gemm_impl(A, nullptr, nullptr, packed, M, N, K, Y, reinterpret_cast<int32_t*>(acc), workspace,
                   workspace_bytes, opts, reinterpret_cast<cudaStream_t>(stream), 0, 1);
}

size_t w4lut3_packed_bytes(int64_t N, int64_t K, int32_t group) {
  if (group != 128 || N <= 0 || K <= 0 || N % 128 != 0 || K % 128 != 0 || K > kMaxK) return 0;
  return static_cast<size_t>(lut3_table_offset(N, K) + 64);
}

w4a8_status_t w4lut3_pack_weights(const uint8_t* q, const void* s, const void* table, int64_t N, int64_t K,
                                  int32_t group, void* packed, size_t packed_bytes, w4a8_stream_t stream) {
  if (N < 0 || K < 0) return W4A8_ERR_INVALID_ARG;
  if (group != 128 || N == 0 || K == 0 || N % 128 != 0 || K % 128 != 0 || K > kMaxK)
    return W4A8_ERR_UNSUPPORTED_SHAPE;
  if (q == nullptr || s == nullptr || table == nullptr || packed == nullptr) return W4A8_ERR_INVALID_ARG;
  if (!aligned(s, 2) || !aligned(table, 2) || !aligned(packed, 16)) return W4A8_ERR_MISALIGNED;
  if (packed_bytes < w4lut3_packed_bytes(N, K, group)) return W4A8_ERR_INVALID_ARG;
  DeviceInfo* dev = nullptr;
  if (const w4a8_status_t e = device_info(&dev); e != W4A8_OK) return e;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  uint8_t* blob = static_cast<uint8_t*>(packed);
  const int64_t warps = N * (K / 128);
  const int64_t blocks1 = (warps + 7) / 8;
  lut3_pack_codes_kernel<<<static_cast<int>(blocks1 < 65535 * 16 ? blocks1 : 65535 * 16), 256, 0, st>>>(
      q, N, K, blob + kHeaderBytes, dev->err);
  if (cudaPeekAtLastError() != cudaSuccess) return launch_status();
  const int64_t metas = N * (K / 128);
  const int64_t blocks2 = (metas + 255) / 256;
  lut3_pack_meta_kernel<<<static_cast<int>(blocks2 < 65535 ? blocks2 : 65535), 256, 0, st>>>(
      static_cast<const __half*>(s), static_cast<const __half*>(table), N, K, blob, lut3_table_offset(N, K));
  return launch_status();
}

w4a8_status_t w4lut3_gemm(const void* A, const void* packed, int64_t M, int64_t N, int64_t K, void* Y,
                          void* workspace, size_t workspace_bytes, w4a8_stream_t stream) {
  return gemm_impl(A, nullptr, nullptr, packed, M, N, K, Y, nullptr, workspace, workspace_bytes, nullptr,
                   reinterpret_cast<cudaStream_t>(stream), 0, 3);
}

w4a8_status_t w4lut3_gemm_ex(const void* A, const void* packed, int64_t M, int64_t N, int64_t K, void* Y,
                             float* acc, void* workspace, size_t workspace_bytes, const w4a8_gemm_opts_t* opts,
                             w4a8_stream_t stream) {
  return gemm_impl(A, nullptr, nullptr, packed, M, N, K, Y, reinterpret_cast<int32_t*>(acc), workspace,
                   workspace_bytes, opts, reinterpret_cast<cudaStream_t>(stream), 0, 3);
}

w4a8_status_t w4a8_get_device_error(w4a8_stream_t stream, int32_t* code) {
  if (code == nullptr) return W4A8_ERR_INVALID_ARG;
  DeviceInfo* dev = nullptr;
  w4a8_status_t st = device_info(&dev);
  if (st != W4A8_OK) return st;
  if (cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess) return launch_status();
  int v = 0;
  if (cudaMemcpy(&v, dev->err, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) return launch_status();
  *code = v;
  return W4A8_OK;
}

w4a8_status_t w4a8_clear_device_error(w4a8_stream_t stream) {
  DeviceInfo* dev = nullptr;
  w4a8_status_t st = device_info(&dev);
  if (st != W4A8_OK) return st;
  return cuda_status(cudaMemsetAsync(dev->err, 0, sizeof(int), reinterpret_cast<cudaStream_t>(stream)));
}

w4a8_status_t w4a8_selftest_bounded_wait(int64_t limit_ns, w4a8_stream_t stream) {
  DeviceInfo* dev = nullptr;
  w4a8_status_t st = device_info(&dev);
  if (st != W4A8_OK) return st;
  const int64_t lo = 1000, hi = static_cast<int64_t>(kWaitLimitNs);
  const int64_t lim = limit_ns < lo ? lo : limit_ns > hi ? hi : limit_ns;
  bounded_wait_selftest_kernel<<<1, 32, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
      dev->err, static_cast<uint64_t>(lim), W4A8_DEVERR_SELFTEST_WAIT);
  return launch_status();
}

// ------------------------------------------------- allocation-free GEMM
// Scratch for w4a8_gemm_noalloc: a file-scope device array instead of a
// caller workspace. In host code `g_noalloc_scratch` only names the symbol;
// its device address comes from cudaGetSymbolAddress, once per device.
static __device__ __align__(256) uint8_t g_noalloc_scratch[W4A8_NOALLOC_SCRATCH_BYTES];
static void* g_noalloc_addr[64] = {};
static std::mutex g_noalloc_mu;

w4a8_status_t w4a8_gemm_noalloc(const int8_t* A8, const void* sA, const int32_t* rowsum, const void* packed,
                                int64_t M, int64_t N, int64_t K, void* Y, w4a8_stream_t stream) {
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  // every argument check comes before the scratch is touched: a rejected
  // call must not clear the array under an earlier call still running on it
  const w4a8_gemm_opts_t o = {0, 0, 0, 0};
  const w4a8_status_t v = check_gemm_args(A8, sA, rowsum, packed, M, N, K, Y, nullptr, nullptr, o, 0);
  if (v != W4A8_OK || M == 0 || N == 0) return v;
  const size_t need = w4a8_gemm_workspace_bytes(M, N, K);
  if (need > W4A8_NOALLOC_SCRATCH_BYTES) return W4A8_ERR_WORKSPACE;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return cuda_status(cudaErrorInvalidDevice);
  void* scratch = nullptr;
  {
    std::lock_guard<std::mutex> lock(g_noalloc_mu);
    if (g_noalloc_addr[dev] == nullptr) {
      void* p = nullptr;
      if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr)
        return cuda_status(cudaErrorInvalidSymbol);
      g_noalloc_addr[dev] = p;
    }
    scratch = g_noalloc_addr[dev];
  }
  // the split-k tickets and partial sums must start at zero
  if (cudaMemsetAsync(scratch, 0, need, st) != cudaSuccess) return launch_status();
  return gemm_impl(A8, sA, rowsum, packed, M, N, K, Y, nullptr, scratch, need, nullptr, st);
}


size_t w4a8_chain_workspace_bytes(const w4a8_chain_link_t* links, int32_t n_links) {
  if (check_chain_links(links, n_links) != W4A8_OK) return 0;
  int sms = 0;
  if (chain_sms(&sms) != W4A8_OK) return 0;
  ChainPlan p;
  chain_plan(links, n_links, sms, &p);
  return p.total;
}

w4a8_status_t w4a8_chain(const w4a8_chain_link_t* links, int32_t n_links, void* workspace, size_t workspace_bytes,
                         w4a8_stream_t stream) {
  w4a8_status_t st = check_chain_links(links, n_links);
  if (st != W4A8_OK) return st;
  if (workspace != nullptr && !aligned(workspace, 256)) return W4A8_ERR_MISALIGNED;
  DeviceInfo* dev = nullptr;
  st = device_info(&dev);
  if (st != W4A8_OK) return st;
  int dev_id = 0;
  cudaGetDevice(&dev_id);
  ChainPlan p;
  chain_plan(links, n_links, dev->sms, &p);
  if (workspace == nullptr || workspace_bytes < p.total) return W4A8_ERR_WORKSPACE;
  {
    static int attr_set[kMaxDevices] = {};
    if (!attr_set[dev_id]) {
      if (cudaFuncSetAttribute(w4a8_chain_kernel<CfgChain>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               CfgChain::kSmemBytes) != cudaSuccess)
        return launch_status();
      attr_set[dev_id] = 1;
    }
  }
  ChainMaps maps;
  ChainArgs a;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  a.n_links = n_links;
  a.done = reinterpret_cast<int32_t*>(ws);
  a.ready = a.done + n_links;
  a.exits = a.ready + n_links;
  a.err = dev->err;
  for (int j = 0; j < n_links; ++j) {
    const w4a8_chain_link_t& L = links[j];
    ChainLink& c = a.link[j];
    c.tiles = static_cast<const uint8_t*>(L.packed) + kHeaderBytes;
    c.s1 = reinterpret_cast<const __half*>(static_cast<const uint8_t*>(L.packed) + packed_s1_offset(L.N, L.K));
    c.A = static_cast<const __half*>(L.A);
    c.A8 = L.A8;
    c.sA = static_cast<__half*>(L.sA);
    c.rowsum = L.rowsum;
    c.Y = static_cast<__half*>(L.Y);
    c.M = static_cast<int>(L.M);
    c.N = static_cast<int>(L.N);
    c.KB = static_cast<int>(L.K / kTileK);
    c.num_tiles = static_cast<int>(L.N / kTileN);
    c.split = p.split[j];
    c.seg0 = p.seg0[j];
    c.ticket = p.split[j] > 1 ? reinterpret_cast<int32_t*>(ws + p.ticket_off[j]) : nullptr;
    c.part = p.split[j] > 1 ? reinterpret_cast<int32_t*>(ws + p.part_off[j]) : nullptr;
    // the link's int8 codes, read as 128-byte rows with the 128-byte swizzle
    const cuuint64_t dims[2] = {static_cast<cuuint64_t>(L.K), static_cast<cuuint64_t>(L.M)};
    const cuuint64_t strides[1] = {static_cast<cuuint64_t>(L.K)};
    const cuuint32_t box[2] = {128u, static_cast<cuuint32_t>(CfgChain::BN)};
    const cuuint32_t estr[2] = {1u, 1u};
    if (g_encode(&maps.m[j], CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, L.A8, dims, strides, box, estr,
                 CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                 CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return W4A8_ERR_CUDA;
  }
  return launch_pdl(w4a8_chain_kernel<CfgChain>, dim3(dev->sms), dim3(CfgChain::kThreads), CfgChain::kSmemBytes,
                    reinterpret_cast<cudaStream_t>(stream), 1, maps, a);
}

w4a8_status_t w4kv_quantize(const void* X, int64_t n, int32_t D, uint8_t* codes, uint32_t* params,
                            w4a8_stream_t stream) {
  if (n < 0) return W4A8_ERR_INVALID_ARG;
  if (D != kKvD) return W4A8_ERR_UNSUPPORTED_SHAPE;
  if (n == 0) return W4A8_OK;
  if (X == nullptr || codes == nullptr || params == nullptr) return W4A8_ERR_INVALID_ARG;
  if (!aligned(X, 16) || !aligned(codes, 16) || !aligned(params, 4)) return W4A8_ERR_MISALIGNED;
  return kv_quantize_launch(X, n, nullptr, 1, 1, codes, params, reinterpret_cast<cudaStream_t>(stream));
}

w4a8_status_t w4kv_append(const void* K_new, const void* V_new, const int32_t* positions, int64_t B, int64_t Hkv,
                          int64_t Lmax, int32_t D, uint8_t* k_codes, uint32_t* k_params, uint8_t* v_codes,
                          uint32_t* v_params, w4a8_stream_t stream) {
  if (B < 0 || Hkv < 0 || Lmax < 0) return W4A8_ERR_INVALID_ARG;
  if (D != kKvD || Lmax > kKvMaxLen) return W4A8_ERR_UNSUPPORTED_SHAPE;
  if (B == 0 || Hkv == 0) return W4A8_OK;
  if (Lmax == 0) return W4A8_ERR_UNSUPPORTED_SHAPE;
  if (K_new == nullptr || V_new == nullptr || positions == nullptr || k_codes == nullptr || k_params == nullptr ||
      v_codes == nullptr || v_params == nullptr)
    return W4A8_ERR_INVALID_ARG;
  if (!aligned(K_new, 16) || !aligned(V_new, 16) || !aligned(positions, 4) || !aligned(k_codes, 16) ||
      !aligned(v_codes, 16) || !aligned(k_params, 4) || !aligned(v_params, 4))
    return W4A8_ERR_MISALIGNED;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const w4a8_status_t s1 = kv_quantize_launch(K_new, B * Hkv, positions, Hkv, Lmax, k_codes, k_params, st);
  if (s1 != W4A8_OK) return s1;
  return kv_quantize_launch(V_new, B * Hkv, positions, Hkv, Lmax, v_codes, v_params, st);
}

}  // extern "C"

// The attention kernel (partial results per chunk), then the merge. The
// attention kernel's dynamic shared memory is above the 48 KB default: raised
// once per (device, instantiation).
template <int GC>
w4a8_status_t kv_decode_launch(dim3 grid, dim3 merge_grid, cudaStream_t s, const KvAttnArgs& a) {
  static bool done[kMaxDevices] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return launch_status();
  if (!done[dev]) {
    // four CTAs per SM: the whole unified L1 / shared array as shared memory
    if (cudaFuncSetAttribute(kv4_decode_kernel<GC>, cudaFuncAttributeMaxDynamicSharedMemorySize, KvSmem::kBytes) !=
            cudaSuccess ||
        cudaFuncSetAttribute(kv4_decode_kernel<GC>, cudaFuncAttributePreferredSharedMemoryCarveout,
                             cudaSharedmemCarveoutMaxShared) != cudaSuccess)
      return launch_status();
    done[dev] = true;
  }
  const w4a8_status_t st = launch_pdl(kv4_decode_kernel<GC>, grid, dim3(kKvAttnThreads), KvSmem::kBytes, s, 1, a);
  if (st != W4A8_OK) return st;
  return launch_pdl(kv4_merge_kernel, merge_grid, dim3(kKvD), 0, s, 1, a);
}

extern "C" {

size_t w4kv_attention_workspace_bytes(int64_t B, int64_t Hq, int64_t Hkv, int64_t Lmax, int32_t D) {
  if (check_kv_shape(B, Hq, Hkv, Lmax, D) != W4A8_OK) return 0;
  return static_cast<size_t>(round256(B * Hq * kv_splits(Lmax) * kKvPartStride * 4));
}

w4a8_status_t w4kv_attention_decode(const void* q, const uint8_t* k_codes, const uint32_t* k_params,
                                    const uint8_t* v_codes, const uint32_t* v_params, const int32_t* seq_lens,
                                    int64_t B, int64_t Hq, int64_t Hkv, int64_t Lmax, int32_t D, float scale,
                                    void* out, void* workspace, size_t workspace_bytes, w4a8_stream_t stream) {
  const w4a8_status_t shape = check_kv_shape(B, Hq, Hkv, Lmax, D);
  if (shape != W4A8_OK) return shape;
  if (B == 0 || Hq == 0) return W4A8_OK;
  if (q == nullptr || k_codes == nullptr || k_params == nullptr || v_codes == nullptr || v_params == nullptr ||
      seq_lens == nullptr || out == nullptr)
    return W4A8_ERR_INVALID_ARG;
  if (!aligned(q, 16) || !aligned(k_codes, 16) || !aligned(v_codes, 16) || !aligned(k_params, 4) ||
      !aligned(v_params, 4) || !aligned(seq_lens, 4) || !aligned(out, 16) || !aligned(workspace, 256))
    return W4A8_ERR_MISALIGNED;
  if (workspace == nullptr || workspace_bytes < w4kv_attention_workspace_bytes(B, Hq, Hkv, Lmax, D))
    return W4A8_ERR_WORKSPACE;
  DeviceInfo* dev = nullptr;
  w4a8_status_t st = device_info(&dev);
  if (st != W4A8_OK) return st;
  const int64_t G = Hq / Hkv;
  const int gc = kv_heads_per_cta(G);
  KvAttnArgs a;
  a.q = static_cast<const __half*>(q);
  a.kc = k_codes;
  a.kp = k_params;
  a.vc = v_codes;
  a.vp = v_params;
  a.seq_lens = seq_lens;
  a.out = static_cast<__half*>(out);
  a.part = static_cast<float*>(workspace);
  a.B = static_cast<int>(B);
  a.groups = static_cast<int>(G / gc);
  a.Hq = static_cast<int>(Hq);
  a.Hkv = static_cast<int>(Hkv);
  a.nsplit = static_cast<int>(kv_splits(Lmax));
  a.Lmax = Lmax;
  a.scale = scale;
  a.err = dev->err;
  // one CTA per (chunk, head group, sequence)
  const dim3 grid(static_cast<unsigned>(a.nsplit), static_cast<unsigned>(Hkv * (G / gc)), static_cast<unsigned>(B));
  const dim3 merge_grid(static_cast<unsigned>(Hq), static_cast<unsigned>(B));
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  switch (gc) {
    case 4: return kv_decode_launch<4>(grid, merge_grid, s, a);
    case 2: return kv_decode_launch<2>(grid, merge_grid, s, a);
    default: return kv_decode_launch<1>(grid, merge_grid, s, a);
  }
}

}  // extern "C"

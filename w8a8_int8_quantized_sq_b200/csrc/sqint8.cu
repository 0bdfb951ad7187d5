// sqint8.cu -- host side of the C ABI declared in include/sqint8.h:
// argument checks, launch planning, tensor-map encoding and kernel launches.
// The library's own device memory is one error word plus the fixed scratch
// array of w8a8_scaled_mm_noalloc (end of this file); nothing else.
#include <atomic>
#include <cstdlib>
#include <mutex>

#include "../../include/sqint8.h"
#include "gemm.cuh"
#include "gemm2.cuh"
#include "gemm3.cuh"
#include "gemv.cuh"
#include "peak.cuh"
#include "quant.cuh"

using namespace sq;

namespace {

constexpr int64_t kMaxK = 131072;  // K * 127 * 127 < 2^31
// Every workspace starts with this many bytes of stream-K arrival counters
// (one 32-bit word per tile).  Nothing else is ever written there, so the
// region stays zero across calls of different operations and sizes that
// share one workspace.  Split-K scratch and converted weights follow it.
constexpr size_t kCounterBytes = 65536;
constexpr int64_t kMaxCounterTiles = static_cast<int64_t>(kCounterBytes / 4);

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// K-major 2-D operand: rows of `inner` elements, box of box_inner x box_rows,
// 128-byte swizzle, out-of-bounds rows read as zero.
bool make_map(CUtensorMap* m, const void* ptr, bool bf16, uint64_t inner, uint64_t rows,
              uint32_t box_inner, uint32_t box_rows,
              CUtensorMapSwizzle swz = CU_TENSOR_MAP_SWIZZLE_128B) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  const uint64_t esz = bf16 ? 2 : 1;
  cuuint64_t dims[2] = {inner, rows};
  cuuint64_t strides[1] = {inner * esz};
  cuuint32_t box[2] = {box_inner, box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(m, bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_UINT8, 2,
                   const_cast<void*>(ptr), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                   swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

int num_sms() {
  static std::atomic<int> cache[64];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 0;
  if (dev < 0 || dev >= 64) return 0;
  int v = cache[dev].load(std::memory_order_relaxed);
  if (v > 0) return v;
  if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
  cache[dev].store(v, std::memory_order_relaxed);
  return v;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

size_t align256(size_t v) { return (v + 255) & ~static_cast<size_t>(255); }

sq_status check_mnk(int64_t M, int64_t N, int64_t K) {
  if (M < 0 || N <= 0 || K <= 0) return SQ_ERR_SHAPE;
  if (N % 16 || K % 128 || K > kMaxK) return SQ_ERR_SHAPE;
  if (M > (1ll << 31) - 1 || N > (1ll << 31) - 1) return SQ_ERR_SHAPE;
  return SQ_OK;
}

sq_status launch_status() {
  return cudaGetLastError() == cudaSuccess ? SQ_OK : SQ_ERR_CUDA;
}

// ---------------------------------------------------------------- planning
enum GemmKind {
  GK_I8_SCALE = 0, GK_I8_I32 = 1, GK_GS128 = 2, GK_BF16 = 3, GK_W8A16_CONV = 4,
  GK_PG128 = 5,        // per-group activations x gs128 weights
  GK_FP8BLK = 6,       // E4M3 per-group activations x [128, 128] block weights
  GK_W8A16G_CONV = 7   // group-wise W8A16, reconstructed on load (M <= 32)
};

// One 128 x 128 tile per CTA, a fresh accumulator per 128-wide K block.
bool block_scaled(GemmKind k) { return k == GK_GS128 || k == GK_PG128 || k == GK_FP8BLK; }

struct GemmPlan {
  bool pair;  // CTA-pair kernel (256 x 256 tiles per cluster of two)
  bool pair3; // block-scaled CTA-pair kernel (256 x 128 tiles, a K block at a time)
  bool swap;
  int bn;
  bool stream_k;
  int grid;
  int tiles_r, tiles_c;
  int kb_total;
  long long total_iters;
  int splits;       // swapped: K parts per tile with whole splits, 0 for stream-K ranges
  int csplit;       // > 1: whole splits combined inside a cluster of csplit CTAs
  size_t ws_bytes;  // counter region + stream-K slots (0: no workspace)
};

// The CTA-pair kernel serves the large-token W8A8 shapes unless the
// environment variable SQ_GEMM_PAIR is set to 0 (then one CTA per 128 x 256
// tile is used, e.g. for comparisons).
bool pair_enabled() {
  static const bool on = [] {
    const char* e = getenv("SQ_GEMM_PAIR");
    return !(e && e[0] == '0');
  }();
  return on;
}

// Width of the block-scaled pair tiles' MMA N (the B rows of a pair tile).
// 256-wide tiles halve the accumulator round trips per multiply-add, but a
// shape with fewer than three waves of them over the SM pairs loses more to
// the partly filled last wave: M=8192 N=34816 K=5120 measured 2.46 ms (gs128)
// and 1.82 ms (FP8) at 256 against 2.64 and 2.06 at 128; M=2048 N=5120
// K=5120 measured 110 / 93 us at 128 against 120 / 97 at 256.
// SQ_BLK_PAIR_N=128 or 256 overrides the choice (for comparisons).
int blk_pair_bn(int64_t rows256, int64_t cols, int sms) {
  static const int forced = [] {
    const char* e = getenv("SQ_BLK_PAIR_N");
    if (!e) return 0;
    return e[0] == '1' ? 128 : (e[0] == '2' ? 256 : 0);
  }();
  if (forced) return forced;
  const int64_t tiles256 = ((rows256 + 255) / 256) * ((cols + 255) / 256);
  return tiles256 < 3 * (sms / 2) ? 128 : 256;
}

// sq_set_overlap: GEMM launches become programmatic dependents of the
// preceding kernel on the stream (they request weights before that kernel
// ends).  The setting belongs to the host thread that made it: calls from
// other threads keep the default.
thread_local int t_overlap = 0;
bool overlap_on() { return t_overlap != 0; }

GemmPlan plan_gemm(GemmKind kind, int64_t M, int64_t N, int64_t K, int sms) {
  GemmPlan p{};
  const bool i8 = kind != GK_BF16 && kind != GK_W8A16_CONV && kind != GK_W8A16G_CONV;
  p.kb_total = static_cast<int>(K / (i8 ? 128 : 64));
  if (!block_scaled(kind) && M <= 32) {
    p.swap = true;
    p.bn = M <= 16 ? 16 : 32;
    p.tiles_r = static_cast<int>((N + 127) / 128);
    p.tiles_c = 1;
    p.stream_k = true;
    p.total_iters = static_cast<long long>(p.tiles_r) * p.kb_total;
    const int whole = p.tiles_r <= sms ? sms / p.tiles_r : 0;
    if (whole > 0 && p.kb_total / whole <= 24) {
      // short K ranges: whole splits, so every CTA owns one contiguous K range
      // of one tile and runs a single epilogue (stream-K ranges with
      // G = tiles * splits); long ranges use every SM instead
      const int splits = whole > p.kb_total ? p.kb_total : whole;
      p.grid = p.tiles_r * splits;
      p.splits = splits;
      // W8A8: a tile's splits form one cluster and add their parts in
      // distributed shared memory (rank 0 holds splits - 1 parts of
      // 128 x bn words beside its operand ring)
      const int max_split = p.bn == 16 ? 8 : 5;
      if ((kind == GK_I8_SCALE || kind == GK_I8_I32) && splits >= 2 && splits <= max_split)
        p.csplit = splits;
    } else {
      p.grid = sms;
    }
    p.ws_bytes = kCounterBytes + static_cast<size_t>(p.grid) * 2 * 128 * p.bn * 4;
  } else if ((kind == GK_GS128 || kind == GK_FP8BLK) && pair_enabled()) {
    // gs128: A = weights (256 channels per pair tile), B = tokens (128);
    // FP8: A = tokens (256), B = weights (128 channels = one weight block)
    p.pair3 = true;
    p.swap = kind == GK_GS128;
    p.bn = blk_pair_bn(p.swap ? N : M, p.swap ? M : N, sms);
    p.tiles_r = static_cast<int>(((p.swap ? N : M) + 255) / 256);
    p.tiles_c = static_cast<int>(((p.swap ? M : N) + p.bn - 1) / p.bn);
    p.stream_k = false;
    p.total_iters = static_cast<long long>(p.tiles_r) * p.tiles_c * p.kb_total;
    p.grid = 0;  // decided at launch from the active-cluster limit
    p.ws_bytes = 0;
  } else if ((kind == GK_I8_SCALE || kind == GK_I8_I32 || kind == GK_BF16) && pair_enabled()) {
    p.pair = true;
    p.swap = false;
    p.bn = 256;
    p.tiles_r = static_cast<int>((M + 255) / 256);
    p.tiles_c = static_cast<int>((N + 255) / 256);
    p.stream_k = false;
    p.total_iters = static_cast<long long>(p.tiles_r) * p.tiles_c * p.kb_total;
    p.grid = 0;  // decided at launch from the active-cluster limit
    p.ws_bytes = 0;
  } else {
    p.swap = false;
    p.bn = block_scaled(kind) ? 128 : 256;
    p.tiles_r = static_cast<int>((M + 127) / 128);
    p.tiles_c = static_cast<int>((N + p.bn - 1) / p.bn);
    p.stream_k = false;
    const long long tiles = static_cast<long long>(p.tiles_r) * p.tiles_c;
    p.total_iters = tiles * p.kb_total;
    p.grid = static_cast<int>(tiles < sms ? tiles : sms);
    p.ws_bytes = 0;
  }
  return p;
}

// Whether `clusters` clusters of `size` CTAs of this kernel can all be
// resident at once (checked once per device, kernel and size).
template <class Cfg>
bool clusters_fit(int size, int clusters, int smem) {
  static std::atomic<int> cap[64][9];
  int dev = 0;
  if (size < 2 || size > 8 || cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64)
    return false;
  int c = cap[dev][size].load(std::memory_order_acquire);
  if (c == 0) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(size);
    cfg.blockDim = dim3(Cfg::THREADS);
    cfg.dynamicSmemBytes = smem;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = size;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaOccupancyMaxActiveClusters(&c, gemm_kernel<Cfg>, &cfg) != cudaSuccess || c <= 0) {
      cudaGetLastError();
      c = -1;
    }
    cap[dev][size].store(c, std::memory_order_release);
  }
  return c >= clusters;
}

template <class Cfg>
sq_status launch_gemm(const CUtensorMap& a, const CUtensorMap& b, GemmArgs g, int grid,
                      cudaStream_t st, bool pdl) {
  g.pdl = pdl ? 1 : 0;
  // cluster split-K needs room for the parts and every cluster resident at once;
  // otherwise the tile's parts meet in the workspace
  if (g.csplit > 1 && (Cfg::BLK || Cfg::CONV ||
                       Cfg::smem_bytes(g.kb_total, g.csplit) > 232448))
    g.csplit = 0;
  const int smem = Cfg::smem_bytes(g.kb_total, g.csplit);
  if (smem > 232448) return SQ_ERR_SHAPE;
  // Raise the kernel's dynamic shared-memory limit once per device (and only
  // upwards), so steady-state launches make no attribute call.
  static std::atomic<int> smem_set[64];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return SQ_ERR_CUDA;
  if (smem_set[dev].load(std::memory_order_acquire) < smem) {
    if (cudaFuncSetAttribute(gemm_kernel<Cfg>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             smem) != cudaSuccess)
      return SQ_ERR_CUDA;
    int cur = smem_set[dev].load();
    while (cur < smem && !smem_set[dev].compare_exchange_weak(cur, smem)) {
    }
  }
  if (g.csplit > 1 && !clusters_fit<Cfg>(g.csplit, grid / g.csplit, smem)) {
    g.csplit = 0;
    return launch_gemm<Cfg>(a, b, g, grid, st, pdl);
  }
  if (!pdl && g.csplit <= 1) {
    gemm_kernel<Cfg><<<grid, Cfg::THREADS, smem, st>>>(a, b, g);
    return launch_status();
  }
  // programmatic dependent launch: the kernel may start while the preceding
  // kernel on the stream runs; it requests only weights before griddep_wait.
  // Cluster split-K: the csplit CTAs of a tile are one cluster.
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(Cfg::THREADS);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  int na = 0;
  if (pdl) {
    attr[na].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[na].val.programmaticStreamSerializationAllowed = 1;
    ++na;
  }
  if (g.csplit > 1) {
    attr[na].id = cudaLaunchAttributeClusterDimension;
    attr[na].val.clusterDim.x = g.csplit;
    attr[na].val.clusterDim.y = 1;
    attr[na].val.clusterDim.z = 1;
    ++na;
  }
  cfg.attrs = attr;
  cfg.numAttrs = na;
  if (cudaLaunchKernelEx(&cfg, gemm_kernel<Cfg>, a, b, g) != cudaSuccess) return SQ_ERR_CUDA;
  return launch_status();
}

template <class Cfg>
sq_status launch_gemm2(const CUtensorMap& a, const CUtensorMap& b, const GemmArgs& g,
                       cudaStream_t st, bool pdl) {
  const int smem = Cfg::smem_bytes();
  static std::atomic<int> max_clusters[64];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return SQ_ERR_CUDA;
  cudaLaunchConfig_t cfg = {};
  cfg.blockDim = dim3(Cfg::THREADS);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 2 : 1;
  int mc = max_clusters[dev].load(std::memory_order_acquire);
  if (mc <= 0) {
    if (cudaFuncSetAttribute(gemm2_kernel<Cfg>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             smem) != cudaSuccess)
      return SQ_ERR_CUDA;
    cfg.gridDim = dim3(2);
    if (cudaOccupancyMaxActiveClusters(&mc, gemm2_kernel<Cfg>, &cfg) != cudaSuccess || mc <= 0)
      return SQ_ERR_CUDA;
    max_clusters[dev].store(mc, std::memory_order_release);
  }
  const int clusters = g.num_tiles < mc ? g.num_tiles : mc;
  cfg.gridDim = dim3(2 * clusters);
  if (cudaLaunchKernelEx(&cfg, gemm2_kernel<Cfg>, a, b, g) != cudaSuccess) return SQ_ERR_CUDA;
  return launch_status();
}

template <class Cfg>
sq_status launch_gemm3(const CUtensorMap& a, const CUtensorMap& b, const GemmArgs& g,
                       cudaStream_t st, bool pdl) {
  const int smem = Cfg::smem_bytes();
  static std::atomic<int> max_clusters[64];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return SQ_ERR_CUDA;
  cudaLaunchConfig_t cfg = {};
  cfg.blockDim = dim3(Cfg::THREADS);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 2 : 1;
  int mc = max_clusters[dev].load(std::memory_order_acquire);
  if (mc <= 0) {
    if (cudaFuncSetAttribute(gemm3_kernel<Cfg>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             smem) != cudaSuccess)
      return SQ_ERR_CUDA;
    cfg.gridDim = dim3(2);
    if (cudaOccupancyMaxActiveClusters(&mc, gemm3_kernel<Cfg>, &cfg) != cudaSuccess || mc <= 0)
      return SQ_ERR_CUDA;
    max_clusters[dev].store(mc, std::memory_order_release);
  }
  const int clusters = g.num_tiles < mc ? g.num_tiles : mc;
  cfg.gridDim = dim3(2 * clusters);
  if (cudaLaunchKernelEx(&cfg, gemm3_kernel<Cfg>, a, b, g) != cudaSuccess) return SQ_ERR_CUDA;
  return launch_status();
}

// act: q_a int8 [M,K] or x bf16 [M,K]; wt: q_w int8 [N,K] or bf16 [N,K].
sq_status run_gemm(GemmKind kind, const void* act, const void* wt, const float* s_tok,
                   const float* s_ch, const float* s_blk, void* out, int64_t M, int64_t N,
                   int64_t K, void* ws, size_t ws_bytes, cudaStream_t st, bool pdl = false,
                   const float* s_a = nullptr) {
  const int sms = num_sms();
  if (sms <= 0) return SQ_ERR_CUDA;
  const GemmPlan p = plan_gemm(kind, M, N, K, sms);
  if (p.stream_k && static_cast<int64_t>(p.tiles_r) * p.tiles_c > kMaxCounterTiles)
    return SQ_ERR_SHAPE;
  if (p.ws_bytes > 0 && (!ws || ws_bytes < p.ws_bytes)) return SQ_ERR_WORKSPACE;
  if (ws && !aligned16(ws)) return SQ_ERR_ALIGN;
  const bool conv = kind == GK_W8A16_CONV || kind == GK_W8A16G_CONV;
  const bool bf16 = kind == GK_BF16 || conv;
  const uint32_t kbe = bf16 ? 64 : 128;
  CUtensorMap ta, tb;
  const void* a_ptr = p.swap ? wt : act;
  const void* b_ptr = p.swap ? act : wt;
  const uint64_t a_rows = static_cast<uint64_t>(p.swap ? N : M);
  const uint64_t b_rows = static_cast<uint64_t>(p.swap ? M : N);
  if (conv) {
    if (!p.swap) return SQ_ERR_SHAPE;
    // raw int8 weight rows, 128 bytes (two 64-element K blocks) per row per box
    if (!make_map(&ta, a_ptr, false, static_cast<uint64_t>(K), a_rows, 128, 128))
      return SQ_ERR_CUDA;
  } else if (!make_map(&ta, a_ptr, bf16, static_cast<uint64_t>(K), a_rows, kbe, 128)) {
    return SQ_ERR_CUDA;
  }
  // the pair kernels stage half of the tile's B rows in each CTA
  if (!make_map(&tb, b_ptr, bf16, static_cast<uint64_t>(K), b_rows, kbe,
                p.pair ? 128 : (p.pair3 ? p.bn / 2 : p.bn)))
    return SQ_ERR_CUDA;

  GemmArgs g{};
  g.R = static_cast<int>(p.swap ? N : M);
  g.C = static_cast<int>(p.swap ? M : N);
  g.kb_total = p.kb_total;
  g.tiles_r = p.tiles_r;
  g.tiles_c = p.tiles_c;
  g.num_tiles = p.tiles_r * p.tiles_c;
  g.stream_k = p.stream_k ? 1 : 0;
  g.total_iters = p.total_iters;
  g.M = static_cast<int>(M);
  g.N = static_cast<int>(N);
  g.s_tok = s_tok;
  g.s_ch = s_ch;
  g.s_blk = s_blk;
  g.s_a = s_a;
  g.out = out;
  g.ws_cnt = p.ws_bytes ? static_cast<unsigned int*>(ws) : nullptr;
  g.ws = p.ws_bytes ? reinterpret_cast<uint32_t*>(static_cast<uint8_t*>(ws) + kCounterBytes)
                    : nullptr;
  g.csplit = p.csplit;

  if (p.pair3) {
    if (p.bn == 256) {
      if (kind == GK_GS128) return launch_gemm3<Gemm3Cfg<EPI_GS128, 256, true>>(ta, tb, g, st, pdl);
      return launch_gemm3<Gemm3Cfg<EPI_FP8BLK, 256, false>>(ta, tb, g, st, pdl);
    }
    if (kind == GK_GS128) return launch_gemm3<Gemm3Cfg<EPI_GS128, 128, false>>(ta, tb, g, st, pdl);
    return launch_gemm3<Gemm3Cfg<EPI_FP8BLK, 128, false>>(ta, tb, g, st, pdl);
  }
  if (p.pair) {
    if (kind == GK_I8_SCALE) return launch_gemm2<Gemm2Cfg<EPI_SCALE, 6>>(ta, tb, g, st, pdl);
    if (kind == GK_BF16)
      return launch_gemm2<Gemm2Cfg<EPI_SCALE, 6, false>>(ta, tb, g, st, pdl);
    return launch_gemm2<Gemm2Cfg<EPI_I32, 6>>(ta, tb, g, st, pdl);
  }
  switch (kind) {
    case GK_I8_SCALE:
      if (p.swap && p.bn == 16)
        return launch_gemm<GemmCfg<true, 16, 8, true, EPI_SCALE>>(ta, tb, g, p.grid, st, pdl);
      if (p.swap)
        return launch_gemm<GemmCfg<true, 32, 8, true, EPI_SCALE>>(ta, tb, g, p.grid, st, pdl);
      return launch_gemm<GemmCfg<true, 256, 4, false, EPI_SCALE>>(ta, tb, g, p.grid, st, pdl);
    case GK_I8_I32:
      if (p.swap && p.bn == 16)
        return launch_gemm<GemmCfg<true, 16, 8, true, EPI_I32>>(ta, tb, g, p.grid, st, pdl);
      if (p.swap)
        return launch_gemm<GemmCfg<true, 32, 8, true, EPI_I32>>(ta, tb, g, p.grid, st, pdl);
      return launch_gemm<GemmCfg<true, 256, 4, false, EPI_I32>>(ta, tb, g, p.grid, st, pdl);
    case GK_GS128:
      return launch_gemm<GemmCfg<true, 128, 4, false, EPI_GS128>>(ta, tb, g, p.grid, st, pdl);
    case GK_PG128:
      return launch_gemm<GemmCfg<true, 128, 4, false, EPI_PG128>>(ta, tb, g, p.grid, st, pdl);
    case GK_FP8BLK:
      return launch_gemm<GemmCfg<true, 128, 4, false, EPI_FP8BLK>>(ta, tb, g, p.grid, st, pdl);
    case GK_W8A16G_CONV:
      if (p.bn == 16)
        return launch_gemm<GemmCfg<false, 16, 3, true, EPI_W16G, true, 5>>(ta, tb, g, p.grid,
                                                                          st, pdl);
      return launch_gemm<GemmCfg<false, 32, 2, true, EPI_W16G, true, 5>>(ta, tb, g, p.grid, st,
                                                                        pdl);
    case GK_BF16:
      // bf16 weight copies exist only for M > 32 (no swapped schedule)
      if (p.swap) return SQ_ERR_SHAPE;
      return launch_gemm<GemmCfg<false, 256, 4, false, EPI_SCALE>>(ta, tb, g, p.grid, st, pdl);
    case GK_W8A16_CONV:
      if (p.bn == 16)
        return launch_gemm<GemmCfg<false, 16, 3, true, EPI_SCALE, true, 5>>(ta, tb, g, p.grid,
                                                                           st, pdl);
      return launch_gemm<GemmCfg<false, 32, 2, true, EPI_SCALE, true, 5>>(ta, tb, g, p.grid, st,
                                                                         pdl);
  }
  return SQ_ERR_SHAPE;
}

// A single token with per-channel scales: the CUDA-core matrix-vector kernel,
// rows dealt round-robin to at most one CTA per SM, when its threads and
// shared-memory stages fit.
bool gemv_plan(int64_t M, int64_t N, int64_t K, int sms, GemvLayout* lo, int* grid) {
  if (M != 1 || sms <= 0) return false;
  const int g = N < sms ? static_cast<int>(N) : sms;
  const GemvLayout l = gemv_layout(N, K, g);
  if (l.S < 2) return false;
  if (lo) *lo = l;
  if (grid) *grid = g;
  return true;
}

sq_status launch_gemv(const void* x, const int8_t* q_w, const float* s_ch, void* y, int64_t N,
                      int64_t K, const GemvLayout& l, int grid, cudaStream_t st, bool pdl) {
  static std::atomic<int> smem_set[64];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return SQ_ERR_CUDA;
  if (smem_set[dev].load(std::memory_order_acquire) < l.smem) {
    if (cudaFuncSetAttribute(w8a16_gemv_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             l.smem) != cudaSuccess)
      return SQ_ERR_CUDA;
    int cur = smem_set[dev].load();
    while (cur < l.smem && !smem_set[dev].compare_exchange_weak(cur, l.smem)) {
    }
  }
  const __nv_bfloat16* xb = static_cast<const __nv_bfloat16*>(x);
  __nv_bfloat16* yb = static_cast<__nv_bfloat16*>(y);
  const int n = static_cast<int>(N), k = static_cast<int>(K);
  if (!pdl) {
    w8a16_gemv_kernel<<<grid, l.nwc * 32 + 32, l.smem, st>>>(xb, q_w, s_ch, yb, n, k, l);
    return launch_status();
  }
  // programmatic dependent launch: the weight stream starts while the
  // preceding kernel runs; the token is read after griddep_wait
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(l.nwc * 32 + 32);
  cfg.dynamicSmemBytes = l.smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (cudaLaunchKernelEx(&cfg, w8a16_gemv_kernel, xb, q_w, s_ch, yb, n, k, l) != cudaSuccess)
    return SQ_ERR_CUDA;
  return launch_status();
}

// W8A16 workspace.  M <= 32 (dequant on load): [counter region][stream-K
// slots] (a single token on the matrix-vector kernel leaves it unused).
// Larger M: [counter region][bf16 weights N x K].
size_t w8a16_ws_bytes(int64_t M, int64_t N, int64_t K, int sms, size_t* w_off) {
  if (M <= 32) {
    if (w_off) *w_off = 0;
    return plan_gemm(GK_W8A16_CONV, M, N, K, sms).ws_bytes;  // same plan for GK_W8A16G_CONV
  }
  const GemmPlan p = plan_gemm(GK_BF16, M, N, K, sms);
  const size_t off = align256(p.ws_bytes > kCounterBytes ? p.ws_bytes : kCounterBytes);
  if (w_off) *w_off = off;
  return off + static_cast<size_t>(N) * static_cast<size_t>(K) * 2;
}

template <int TPR, bool HAS_VEC>
sq_status launch_quant(const void* x, const float* vec, int8_t* q, float* scales, int64_t nseg,
                       int64_t K, int64_t group, cudaStream_t st) {
  constexpr int SEGS = 256 / TPR;
  const int64_t blocks = (nseg + SEGS - 1) / SEGS;
  if (blocks > 2147483647ll) return SQ_ERR_SHAPE;
  quant_rows_kernel<TPR, HAS_VEC><<<static_cast<unsigned>(blocks), 256, 0, st>>>(
      static_cast<const __nv_bfloat16*>(x), vec, q, scales, nseg, static_cast<int>(K),
      static_cast<int>(group));
  return launch_status();
}

template <int TPR, int CH, int G, int MODE>
sq_status launch_quant_stream(const void* x, const float* vec, int8_t* q, float* scales,
                              int64_t rows, int64_t K, cudaStream_t st, float eps,
                              float* r_out) {
  const size_t row_bytes = static_cast<size_t>(K) * 2;
  // ring depth: about 100 KB of rows per block (two blocks per SM), at least
  // two rows per group so one is in flight while the other is processed
  int S = static_cast<int>((100u << 10) / (G * row_bytes));
  S = S < 2 ? 2 : (S > 8 ? 8 : S);
  const size_t smem = 1024 + static_cast<size_t>(G) * S * row_bytes;
  if (smem > 232448) return SQ_ERR_SHAPE;
  const int sms = num_sms();
  if (sms <= 0) return SQ_ERR_CUDA;
  int64_t blocks = (rows + G - 1) / G;
  if (blocks > 2 * sms) blocks = 2 * sms;
  auto kern = vec ? quant_stream_kernel<TPR, CH, G, true, MODE>
                  : quant_stream_kernel<TPR, CH, G, false, MODE>;
  static std::atomic<int> smem_set[64];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return SQ_ERR_CUDA;
  const int flag = vec ? 2 : 1;
  if ((smem_set[dev].load() & flag) == 0) {
    if (cudaFuncSetAttribute(quant_stream_kernel<TPR, CH, G, true, MODE>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, 232448) != cudaSuccess ||
        cudaFuncSetAttribute(quant_stream_kernel<TPR, CH, G, false, MODE>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, 232448) != cudaSuccess)
      return SQ_ERR_CUDA;
    smem_set[dev].fetch_or(3);
  }
  kern<<<static_cast<unsigned>(blocks), TPR * G, smem, st>>>(
      static_cast<const __nv_bfloat16*>(x), vec, q, scales, rows, static_cast<int>(K), S, eps,
      r_out);
  return launch_status();
}

template <int TPR, int G, int MODE>
sq_status launch_quant_stream_ch(int ch, const void* x, const float* vec, int8_t* q,
                                 float* scales, int64_t rows, int64_t K, cudaStream_t st,
                                 float eps, float* r_out) {
  switch (ch) {
    case 1: return launch_quant_stream<TPR, 1, G, MODE>(x, vec, q, scales, rows, K, st, eps, r_out);
    case 2: return launch_quant_stream<TPR, 2, G, MODE>(x, vec, q, scales, rows, K, st, eps, r_out);
    case 3: return launch_quant_stream<TPR, 3, G, MODE>(x, vec, q, scales, rows, K, st, eps, r_out);
    case 4: return launch_quant_stream<TPR, 4, G, MODE>(x, vec, q, scales, rows, K, st, eps, r_out);
    case 5: return launch_quant_stream<TPR, 5, G, MODE>(x, vec, q, scales, rows, K, st, eps, r_out);
    default: return launch_quant_stream<TPR, 6, G, MODE>(x, vec, q, scales, rows, K, st, eps, r_out);
  }
}

// Largest K the streaming kernel takes (256 threads x 6 chunks x 16 columns).
constexpr int64_t kMaxStreamK = 256 * 16 * 6;

// One row of K elements (K <= kMaxStreamK) per step: the streaming kernel with
// the fewest threads per row that keeps at most 6 chunks of 16 columns (and
// their 1/s factors) per thread.  MODE: QM_* bits (norm, 128-wide groups, FP8).
template <int MODE = 0>
sq_status quant_per_row(const void* x, const float* vec, int8_t* q, float* scales, int64_t rows,
                        int64_t K, cudaStream_t st, float eps = 0.0f, float* r_out = nullptr) {
  const int64_t c64 = (K + 1023) / 1024, c128 = (K + 2047) / 2048, c256 = (K + 4095) / 4096;
  if (c64 <= 6)
    return launch_quant_stream_ch<64, 4, MODE>(static_cast<int>(c64), x, vec, q, scales, rows, K,
                                               st, eps, r_out);
  if (c128 <= 6)
    return launch_quant_stream_ch<128, 1, MODE>(static_cast<int>(c128), x, vec, q, scales, rows,
                                                K, st, eps, r_out);
  return launch_quant_stream_ch<256, 1, MODE>(static_cast<int>(c256), x, vec, q, scales, rows, K,
                                              st, eps, r_out);
}

sq_status quant_rows(const void* x, const float* vec, int8_t* q, float* scales, int64_t nseg,
                     int64_t K, int64_t group, cudaStream_t st) {
  if (nseg == 0) return SQ_OK;
  if (group == K && K <= kMaxStreamK) return quant_per_row(x, vec, q, scales, nseg, K, st);
  if (group == 128) {
    return vec ? launch_quant<8, true>(x, vec, q, scales, nseg, K, group, st)
               : launch_quant<8, false>(x, vec, q, scales, nseg, K, group, st);
  }
  if (nseg >= 2048) {
    return vec ? launch_quant<32, true>(x, vec, q, scales, nseg, K, group, st)
               : launch_quant<32, false>(x, vec, q, scales, nseg, K, group, st);
  }
  return vec ? launch_quant<256, true>(x, vec, q, scales, nseg, K, group, st)
             : launch_quant<256, false>(x, vec, q, scales, nseg, K, group, st);
}

}  // namespace

extern "C" {

const char* sq_status_string(sq_status s) {
  switch (s) {
    case SQ_OK: return "ok";
    case SQ_ERR_NULL: return "null pointer";
    case SQ_ERR_SHAPE: return "unsupported shape";
    case SQ_ERR_ALIGN: return "pointer not 16-byte aligned";
    case SQ_ERR_WORKSPACE: return "workspace missing or too small";
    case SQ_ERR_CUDA: return "CUDA error";
    case SQ_ERR_TIMEOUT: return "kernel wait timed out";
  }
  return "unknown status";
}

sq_status sq_quant_per_token(const void* x_bf16, const float* inv_smooth, int8_t* q_i8,
                             float* s_tok, int64_t M, int64_t K, void* stream) {
  if (M < 0 || K <= 0 || K % 128 || K > kMaxK) return SQ_ERR_SHAPE;
  if (M == 0) return SQ_OK;
  if (!x_bf16 || !q_i8 || !s_tok) return SQ_ERR_NULL;
  if (!aligned16(x_bf16) || !aligned16(q_i8) || !aligned16(s_tok) ||
      (inv_smooth && !aligned16(inv_smooth)))
    return SQ_ERR_ALIGN;
  return quant_rows(x_bf16, inv_smooth, q_i8, s_tok, M, K, K, static_cast<cudaStream_t>(stream));
}

sq_status sq_quant_weight(const void* w_bf16, const float* smooth, int8_t* q_w, float* scales,
                          int64_t N, int64_t K, int64_t group, void* stream) {
  if (N < 0 || K <= 0 || K % 128 || K > kMaxK || (group != 0 && group != 128))
    return SQ_ERR_SHAPE;
  if (N == 0) return SQ_OK;
  if (!w_bf16 || !q_w || !scales) return SQ_ERR_NULL;
  if (!aligned16(w_bf16) || !aligned16(q_w) || !aligned16(scales) || (smooth && !aligned16(smooth)))
    return SQ_ERR_ALIGN;
  const int64_t g = group ? group : K;
  return quant_rows(w_bf16, smooth, q_w, scales, N * (K / g), K, g,
                    static_cast<cudaStream_t>(stream));
}

sq_status sq_smooth_factors(const void* x_bf16, int64_t M, const void* w_bf16, int64_t N,
                            int64_t K, double cap, double floor_, float* s_out,
                            float* inv_s_out, void* stream) {
  if (M <= 0 || N <= 0 || K <= 0 || K % 128 || K > kMaxK) return SQ_ERR_SHAPE;
  if (!x_bf16 || !w_bf16 || !s_out || !inv_s_out) return SQ_ERR_NULL;
  if (!aligned16(x_bf16) || !aligned16(w_bf16) || !aligned16(s_out) || !aligned16(inv_s_out))
    return SQ_ERR_ALIGN;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (cudaMemsetAsync(s_out, 0, K * 4, st) != cudaSuccess) return SQ_ERR_CUDA;
  if (cudaMemsetAsync(inv_s_out, 0, K * 4, st) != cudaSuccess) return SQ_ERR_CUDA;
  const int rpb = 64;
  const unsigned gx = static_cast<unsigned>((K / 8 + 255) / 256);
  dim3 gxm(gx, static_cast<unsigned>((M + rpb - 1) / rpb));
  colmax_kernel<<<gxm, 256, 0, st>>>(static_cast<const __nv_bfloat16*>(x_bf16), M,
                                     static_cast<int>(K), rpb,
                                     reinterpret_cast<unsigned int*>(s_out));
  dim3 gwn(gx, static_cast<unsigned>((N + rpb - 1) / rpb));
  colmax_kernel<<<gwn, 256, 0, st>>>(static_cast<const __nv_bfloat16*>(w_bf16), N,
                                     static_cast<int>(K), rpb,
                                     reinterpret_cast<unsigned int*>(inv_s_out));
  smooth_finalize_kernel<<<static_cast<unsigned>((K + 255) / 256), 256, 0, st>>>(
      s_out, inv_s_out, static_cast<int>(K), cap, floor_);
  return launch_status();
}

size_t sq_workspace_bytes(int op, int64_t M, int64_t N, int64_t K) {
  if (check_mnk(M, N, K) != SQ_OK) return 0;
  const int sms = num_sms();
  if (sms <= 0) return 0;
  switch (op) {
    case SQ_OP_W8A8: return plan_gemm(GK_I8_SCALE, M, N, K, sms).ws_bytes;
    case SQ_OP_W8A8_I32: return plan_gemm(GK_I8_I32, M, N, K, sms).ws_bytes;
    case SQ_OP_GS128: return plan_gemm(GK_GS128, M, N, K, sms).ws_bytes;
    case SQ_OP_W8A16: return w8a16_ws_bytes(M, N, K, sms, nullptr);
    case SQ_OP_PG128: return plan_gemm(GK_PG128, M, N, K, sms).ws_bytes;
    case SQ_OP_FP8BLK: return plan_gemm(GK_FP8BLK, M, N, K, sms).ws_bytes;
    case SQ_OP_W8A16_GROUP: return w8a16_ws_bytes(M, N, K, sms, nullptr);
  }
  return 0;
}

sq_status sq_describe_plan(int op, int64_t M, int64_t N, int64_t K, int sms,
                           sq_plan_info* out) {
  if (!out) return SQ_ERR_NULL;
  const sq_status s = check_mnk(M, N, K);
  if (s != SQ_OK) return s;
  if (sms <= 0) return SQ_ERR_SHAPE;
  GemmKind kind;
  switch (op) {
    case SQ_OP_W8A8: kind = GK_I8_SCALE; break;
    case SQ_OP_W8A8_I32: kind = GK_I8_I32; break;
    case SQ_OP_GS128: kind = GK_GS128; break;
    case SQ_OP_W8A16: kind = M <= 32 ? GK_W8A16_CONV : GK_BF16; break;
    case SQ_OP_PG128: kind = GK_PG128; break;
    case SQ_OP_FP8BLK: kind = GK_FP8BLK; break;
    case SQ_OP_W8A16_GROUP: kind = M <= 32 ? GK_W8A16G_CONV : GK_BF16; break;
    default: return SQ_ERR_SHAPE;
  }
  const GemmPlan p = plan_gemm(kind, M, N, K, sms);
  const int tiles = p.tiles_r * p.tiles_c;
  sq_plan_info r{};
  GemvLayout gl{};
  int ggrid = 0;
  if (op == SQ_OP_W8A16 && gemv_plan(M, N, K, sms, &gl, &ggrid)) {
    r.kernel = 5;
    r.grid = ggrid;
    r.tile_m = 1;
    r.tile_n = gl.rows_max;
    r.splits = 1;
  } else if (p.pair) {
    r.kernel = 0;
    r.grid = 2 * (tiles < sms / 2 ? tiles : sms / 2);
    r.tile_m = 256;
    r.tile_n = 256;
    r.splits = 1;
  } else if (p.pair3) {
    r.kernel = 4;
    r.grid = 2 * (tiles < sms / 2 ? tiles : sms / 2);
    r.tile_m = p.swap ? p.bn : 256;
    r.tile_n = p.swap ? 256 : p.bn;
    r.splits = 1;
  } else if (!p.swap) {
    r.kernel = 1;
    r.grid = p.grid;
    r.tile_m = 128;
    r.tile_n = p.bn;
    r.splits = 1;
  } else {
    r.kernel = p.csplit > 1 ? 3 : 2;
    r.grid = p.grid;
    r.tile_m = p.bn;
    r.tile_n = 128;
    r.splits = p.splits;
  }
  r.workspace_bytes = (op == SQ_OP_W8A16 || op == SQ_OP_W8A16_GROUP)
                          ? w8a16_ws_bytes(M, N, K, sms, nullptr)
                          : p.ws_bytes;
  *out = r;
  return SQ_OK;
}

sq_status w8a8_scaled_mm(const int8_t* q_a, const float* s_tok, const int8_t* q_w,
                         const float* s_ch, void* y_bf16, int64_t M, int64_t N, int64_t K,
                         void* workspace, size_t ws_bytes, void* stream) {
  sq_status s = check_mnk(M, N, K);
  if (s != SQ_OK) return s;
  if (M == 0) return SQ_OK;
  if (!q_a || !s_tok || !q_w || !s_ch || !y_bf16) return SQ_ERR_NULL;
  if (!aligned16(q_a) || !aligned16(s_tok) || !aligned16(q_w) || !aligned16(s_ch) ||
      !aligned16(y_bf16))
    return SQ_ERR_ALIGN;
  return run_gemm(GK_I8_SCALE, q_a, q_w, s_tok, s_ch, nullptr, y_bf16, M, N, K, workspace,
                  ws_bytes, static_cast<cudaStream_t>(stream), overlap_on());
}

sq_status sq_w8a8_linear(const void* x_bf16, const float* inv_smooth, const int8_t* q_w,
                         const float* s_ch, void* y_bf16, int8_t* q_a, float* s_tok, int64_t M,
                         int64_t N, int64_t K, void* workspace, size_t ws_bytes, void* stream) {
  sq_status s = check_mnk(M, N, K);
  if (s != SQ_OK) return s;
  if (M == 0) return SQ_OK;
  if (!x_bf16 || !q_w || !s_ch || !y_bf16 || !q_a || !s_tok) return SQ_ERR_NULL;
  if (!aligned16(x_bf16) || !aligned16(q_w) || !aligned16(s_ch) || !aligned16(y_bf16) ||
      !aligned16(q_a) || !aligned16(s_tok) || (inv_smooth && !aligned16(inv_smooth)))
    return SQ_ERR_ALIGN;
  const int sms = num_sms();
  if (sms <= 0) return SQ_ERR_CUDA;
  const GemmPlan p = plan_gemm(GK_I8_SCALE, M, N, K, sms);
  if (p.ws_bytes > 0 && (!workspace || ws_bytes < p.ws_bytes)) return SQ_ERR_WORKSPACE;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  s = quant_rows(x_bf16, inv_smooth, q_a, s_tok, M, K, K, st);
  if (s != SQ_OK) return s;
  return run_gemm(GK_I8_SCALE, q_a, q_w, s_tok, s_ch, nullptr, y_bf16, M, N, K, workspace,
                  ws_bytes, st, /*pdl=*/true);
}

sq_status w8a8_mm_i32(const int8_t* q_a, const int8_t* q_w, int32_t* acc, int64_t M, int64_t N,
                      int64_t K, void* workspace, size_t ws_bytes, void* stream) {
  sq_status s = check_mnk(M, N, K);
  if (s != SQ_OK) return s;
  if (M == 0) return SQ_OK;
  if (!q_a || !q_w || !acc) return SQ_ERR_NULL;
  if (!aligned16(q_a) || !aligned16(q_w) || !aligned16(acc)) return SQ_ERR_ALIGN;
  return run_gemm(GK_I8_I32, q_a, q_w, nullptr, nullptr, nullptr, acc, M, N, K, workspace,
                  ws_bytes, static_cast<cudaStream_t>(stream), overlap_on());
}

sq_status w8a8_gs128_mm(const int8_t* q_a, const float* s_tok, const int8_t* q_w,
                        const float* s_blk, void* y_bf16, int64_t M, int64_t N, int64_t K,
                        void* workspace, size_t ws_bytes, void* stream) {
  sq_status s = check_mnk(M, N, K);
  if (s != SQ_OK) return s;
  if (M == 0) return SQ_OK;
  if (!q_a || !s_tok || !q_w || !s_blk || !y_bf16) return SQ_ERR_NULL;
  if (!aligned16(q_a) || !aligned16(s_tok) || !aligned16(q_w) || !aligned16(s_blk) ||
      !aligned16(y_bf16))
    return SQ_ERR_ALIGN;
  return run_gemm(GK_GS128, q_a, q_w, s_tok, nullptr, s_blk, y_bf16, M, N, K, workspace,
                  ws_bytes, static_cast<cudaStream_t>(stream), overlap_on());
}

sq_status w8a16_mm(const void* x_bf16, const int8_t* q_w, const float* s_ch, void* y_bf16,
                   int64_t M, int64_t N, int64_t K, void* workspace, size_t ws_bytes,
                   void* stream) {
  sq_status s = check_mnk(M, N, K);
  if (s != SQ_OK) return s;
  if (M == 0) return SQ_OK;
  if (!x_bf16 || !q_w || !s_ch || !y_bf16) return SQ_ERR_NULL;
  if (!aligned16(x_bf16) || !aligned16(q_w) || !aligned16(s_ch) || !aligned16(y_bf16))
    return SQ_ERR_ALIGN;
  const int sms = num_sms();
  if (sms <= 0) return SQ_ERR_CUDA;
  size_t w_off = 0;
  const size_t need = w8a16_ws_bytes(M, N, K, sms, &w_off);
  if (!workspace || ws_bytes < need) return SQ_ERR_WORKSPACE;
  if (!aligned16(workspace)) return SQ_ERR_ALIGN;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  GemvLayout gl{};
  int ggrid = 0;
  if (gemv_plan(M, N, K, sms, &gl, &ggrid))  // one token: a matrix-vector product
    return launch_gemv(x_bf16, q_w, s_ch, y_bf16, N, K, gl, ggrid, st, overlap_on());
  if (M <= 32)  // weight-read bound: int8 weights are converted on load, in the GEMM
    return run_gemm(GK_W8A16_CONV, x_bf16, q_w, nullptr, s_ch, nullptr, y_bf16, M, N, K,
                    workspace, ws_bytes, st, overlap_on());
  __nv_bfloat16* wb = reinterpret_cast<__nv_bfloat16*>(static_cast<uint8_t*>(workspace) + w_off);
  const int64_t n16 = N * K / 16;
  const int64_t blocks = (n16 + 255) / 256 < 4 * sms ? (n16 + 255) / 256 : 4 * sms;
  i8_to_bf16_kernel<<<static_cast<unsigned>(blocks), 256, 0, st>>>(q_w, wb, n16);
  if (launch_status() != SQ_OK) return SQ_ERR_CUDA;
  // never a programmatic launch here: its weights come from the kernel just before
  return run_gemm(GK_BF16, x_bf16, wb, nullptr, s_ch, nullptr, y_bf16, M, N, K, workspace,
                  w_off, st);
}

// ---------------------------------------------------------------------------
// Fused RMSNorm + fold + quantisation, per-group activations, group-wise
// W8A16 and FP8 block scaling.

sq_status sq_fold_norm_weight(const void* w_norm_bf16, int zero_centered,
                              const float* inv_smooth, float* gamma, int64_t K, void* stream) {
  if (K <= 0 || K > kMaxK) return SQ_ERR_SHAPE;
  if (!w_norm_bf16 || !gamma) return SQ_ERR_NULL;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  fold_norm_weight_kernel<<<static_cast<unsigned>((K + 255) / 256), 256, 0, st>>>(
      static_cast<const __nv_bfloat16*>(w_norm_bf16), zero_centered, inv_smooth, gamma,
      static_cast<int>(K));
  return launch_status();
}

sq_status sq_rmsnorm_quant(const void* h_bf16, const float* gamma, float eps, int64_t group,
                           int8_t* q_i8, float* scales, float* inv_rms, int64_t M, int64_t K,
                           void* stream) {
  if (M < 0 || K <= 0 || K % 128 || K > kMaxStreamK) return SQ_ERR_SHAPE;
  if (group != 0 && group != K && group != 128) return SQ_ERR_SHAPE;
  if (!(eps > 0.0f) || !(eps < 3.4e38f)) return SQ_ERR_SHAPE;
  if (M == 0) return SQ_OK;
  if (!h_bf16 || !gamma || !q_i8 || !scales) return SQ_ERR_NULL;
  if (!aligned16(h_bf16) || !aligned16(gamma) || !aligned16(q_i8) || !aligned16(scales))
    return SQ_ERR_ALIGN;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (group == 128 && K != 128)
    return quant_per_row<QM_NORM | QM_GROUP>(h_bf16, gamma, q_i8, scales, M, K, st, eps, inv_rms);
  return quant_per_row<QM_NORM>(h_bf16, gamma, q_i8, scales, M, K, st, eps, inv_rms);
}

sq_status sq_quant_per_group(const void* x_bf16, const float* inv_smooth, int8_t* q_i8,
                             float* s_a, int64_t M, int64_t K, void* stream) {
  if (M < 0 || K <= 0 || K % 128 || K > kMaxK) return SQ_ERR_SHAPE;
  if (M == 0) return SQ_OK;
  if (!x_bf16 || !q_i8 || !s_a) return SQ_ERR_NULL;
  if (!aligned16(x_bf16) || !aligned16(q_i8) || !aligned16(s_a) ||
      (inv_smooth && !aligned16(inv_smooth)))
    return SQ_ERR_ALIGN;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (K <= kMaxStreamK)
    return quant_per_row<QM_GROUP>(x_bf16, inv_smooth, q_i8, s_a, M, K, st);
  return quant_rows(x_bf16, inv_smooth, q_i8, s_a, M * (K / 128), K, 128, st);
}

sq_status sq_quant_fp8_per_group(const void* x_bf16, const float* inv_smooth, uint8_t* q_e4m3,
                                 float* s_a, int64_t M, int64_t K, void* stream) {
  if (M < 0 || K <= 0 || K % 128 || K > kMaxStreamK) return SQ_ERR_SHAPE;
  if (M == 0) return SQ_OK;
  if (!x_bf16 || !q_e4m3 || !s_a) return SQ_ERR_NULL;
  if (!aligned16(x_bf16) || !aligned16(q_e4m3) || !aligned16(s_a) ||
      (inv_smooth && !aligned16(inv_smooth)))
    return SQ_ERR_ALIGN;
  return quant_per_row<QM_GROUP | QM_FP8>(x_bf16, inv_smooth, reinterpret_cast<int8_t*>(q_e4m3),
                                          s_a, M, K, static_cast<cudaStream_t>(stream));
}

sq_status sq_quant_fp8_block(const void* w_bf16, const float* smooth, uint8_t* q_e4m3,
                             float* s_w, int64_t N, int64_t K, void* stream) {
  if (N < 0 || K <= 0 || K % 128 || N % 128 || K > kMaxK) return SQ_ERR_SHAPE;
  if (N == 0) return SQ_OK;
  if (!w_bf16 || !q_e4m3 || !s_w) return SQ_ERR_NULL;
  if (!aligned16(w_bf16) || !aligned16(q_e4m3) || !aligned16(s_w) || (smooth && !aligned16(smooth)))
    return SQ_ERR_ALIGN;
  if (N / 128 > 65535) return SQ_ERR_SHAPE;
  dim3 grid(static_cast<unsigned>(K / 128), static_cast<unsigned>(N / 128));
  fp8_block_quant_kernel<<<grid, 256, 0, static_cast<cudaStream_t>(stream)>>>(
      static_cast<const __nv_bfloat16*>(w_bf16), smooth, q_e4m3, s_w, static_cast<int>(K));
  return launch_status();
}

sq_status w8a8_pg128_mm(const int8_t* q_a, const float* s_a, const int8_t* q_w,
                        const float* s_blk, void* y_bf16, int64_t M, int64_t N, int64_t K,
                        void* workspace, size_t ws_bytes, void* stream) {
  sq_status s = check_mnk(M, N, K);
  if (s != SQ_OK) return s;
  if (M == 0) return SQ_OK;
  if (!q_a || !s_a || !q_w || !s_blk || !y_bf16) return SQ_ERR_NULL;
  if (!aligned16(q_a) || !aligned16(s_a) || !aligned16(q_w) || !aligned16(s_blk) ||
      !aligned16(y_bf16))
    return SQ_ERR_ALIGN;
  return run_gemm(GK_PG128, q_a, q_w, nullptr, nullptr, s_blk, y_bf16, M, N, K, workspace,
                  ws_bytes, static_cast<cudaStream_t>(stream), overlap_on(), s_a);
}

sq_status fp8_block_mm(const uint8_t* q_a, const float* s_a, const uint8_t* q_w,
                       const float* s_w, void* y_bf16, int64_t M, int64_t N, int64_t K,
                       void* workspace, size_t ws_bytes, void* stream) {
  sq_status s = check_mnk(M, N, K);
  if (s != SQ_OK) return s;
  if (N % 128) return SQ_ERR_SHAPE;
  if (M == 0) return SQ_OK;
  if (!q_a || !s_a || !q_w || !s_w || !y_bf16) return SQ_ERR_NULL;
  if (!aligned16(q_a) || !aligned16(s_a) || !aligned16(q_w) || !aligned16(s_w) ||
      !aligned16(y_bf16))
    return SQ_ERR_ALIGN;
  return run_gemm(GK_FP8BLK, q_a, q_w, nullptr, nullptr, s_w, y_bf16, M, N, K, workspace,
                  ws_bytes, static_cast<cudaStream_t>(stream), overlap_on(), s_a);
}

sq_status w8a16_group_mm(const void* x_bf16, const int8_t* q_w, const float* s_grp,
                         void* y_bf16, int64_t M, int64_t N, int64_t K, void* workspace,
                         size_t ws_bytes, void* stream) {
  sq_status s = check_mnk(M, N, K);
  if (s != SQ_OK) return s;
  if (M == 0) return SQ_OK;
  if (!x_bf16 || !q_w || !s_grp || !y_bf16) return SQ_ERR_NULL;
  if (!aligned16(x_bf16) || !aligned16(q_w) || !aligned16(s_grp) || !aligned16(y_bf16))
    return SQ_ERR_ALIGN;
  const int sms = num_sms();
  if (sms <= 0) return SQ_ERR_CUDA;
  size_t w_off = 0;
  const size_t need = w8a16_ws_bytes(M, N, K, sms, &w_off);
  if (!workspace || ws_bytes < need) return SQ_ERR_WORKSPACE;
  if (!aligned16(workspace)) return SQ_ERR_ALIGN;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (M <= 32)  // weight-read bound: group-scaled reconstruction on load, in the GEMM
    return run_gemm(GK_W8A16G_CONV, x_bf16, q_w, nullptr, nullptr, s_grp, y_bf16, M, N, K,
                    workspace, ws_bytes, st, overlap_on());
  __nv_bfloat16* wb = reinterpret_cast<__nv_bfloat16*>(static_cast<uint8_t*>(workspace) + w_off);
  const int64_t n16 = N * K / 16;
  const int64_t blocks = (n16 + 255) / 256 < 4 * sms ? (n16 + 255) / 256 : 4 * sms;
  i8_to_bf16_group_kernel<<<static_cast<unsigned>(blocks), 256, 0, st>>>(q_w, s_grp, wb, n16,
                                                                         static_cast<int>(K));
  if (launch_status() != SQ_OK) return SQ_ERR_CUDA;
  // the reconstructed weights carry the scales: the epilogue stores the sums as they are
  return run_gemm(GK_BF16, x_bf16, wb, nullptr, nullptr, nullptr, y_bf16, M, N, K, workspace,
                  w_off, st);
}

sq_status sq_mma_peak(int kind, int iters, void* stream, double* ops_per_launch) {
  if (!ops_per_launch) return SQ_ERR_NULL;
  if (kind < 0 || kind > 2 || iters < 2 || iters > (1 << 24)) return SQ_ERR_SHAPE;
  const int sms = num_sms();
  if (sms < 2) return SQ_ERR_CUDA;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return SQ_ERR_CUDA;
  const int smem = 32768 + 1024;
  cudaLaunchConfig_t cfg = {};
  cfg.blockDim = dim3(128);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = static_cast<cudaStream_t>(stream);
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  auto kern = kind == PEAK_I8 ? mma_peak_kernel<PEAK_I8>
              : kind == PEAK_F8 ? mma_peak_kernel<PEAK_F8> : mma_peak_kernel<PEAK_BF16>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
    return SQ_ERR_CUDA;
  cfg.gridDim = dim3(2);
  int mc = 0;
  if (cudaOccupancyMaxActiveClusters(&mc, kern, &cfg) != cudaSuccess || mc <= 0) return SQ_ERR_CUDA;
  const int clusters = mc < sms / 2 ? mc : sms / 2;  // one pair per two SMs, all resident
  cfg.gridDim = dim3(2 * clusters);
  if (cudaLaunchKernelEx(&cfg, kern, iters) != cudaSuccess) return SQ_ERR_CUDA;
  // M = 256, N = 256 and K = 32 (8-bit) or 16 (bf16) elements per MMA; 2 ops per MAC
  const double k = kind == PEAK_BF16 ? 16.0 : 32.0;
  *ops_per_launch = 2.0 * 256.0 * 256.0 * k * iters * clusters;
  return launch_status();
}

sq_status sq_set_overlap(int enable) {
  t_overlap = enable ? 1 : 0;
  return SQ_OK;
}

sq_status sq_selftest_wait_timeout(int64_t limit_cycles, int* gave_up, void* stream) {
  if (!gave_up) return SQ_ERR_NULL;
  if (limit_cycles <= 0 || limit_cycles > kWaitLimitCycles) return SQ_ERR_SHAPE;
  wait_timeout_selftest_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(limit_cycles,
                                                                               gave_up);
  return launch_status();
}

sq_status sq_check_device_error(int reset) {
  if (cudaDeviceSynchronize() != cudaSuccess) return SQ_ERR_CUDA;
  unsigned int w = 0;
  if (cudaMemcpyFromSymbol(&w, g_error_word, sizeof(w)) != cudaSuccess) return SQ_ERR_CUDA;
  if (reset && w) {
    const unsigned int z = 0;
    if (cudaMemcpyToSymbol(g_error_word, &z, sizeof(z)) != cudaSuccess) return SQ_ERR_CUDA;
  }
  return (w & kErrTimeout) ? SQ_ERR_TIMEOUT : SQ_OK;
}

}  // extern "C"

// ---------------------------------------------------------------------------
// W8A8 GEMM for callers that cannot allocate device memory.
//
// Some callers of this library cannot call cudaMalloc: a plugin whose host
// framework owns every byte of device memory and hands it only the layer's
// inputs and outputs, or a latency-critical serving thread where cudaMalloc
// would synchronise the device and stall other streams.  For the small-token
// (M <= 32) split-K schedule, the only operation here that needs scratch, this
// entry point uses a fixed array in the library's own device memory instead
// of a caller-provided workspace.  The array is a file-scope static, so every
// GPU that loads the library holds it until the process exits.

namespace {
// Counter region (64 KiB) + stream-K partial slots for up to 148 CTAs at the
// widest small-M tile (2 slots x 128 rows x 32 columns x 4 bytes per CTA).
constexpr size_t kNoAllocScratchBytes = 5u << 20;  // 5 MiB
}  // namespace

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

namespace {
// Device address of g_noalloc_scratch for the current device, looked up once
// per device (with that device current) and cached.  In host code the
// symbol's name is only a host-side stand-in, never a device address.
void* noalloc_scratch_address() {
  static std::mutex mu;
  static void* addr[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
  std::lock_guard<std::mutex> lock(mu);
  if (!addr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess) return nullptr;
    addr[dev] = p;
  }
  return addr[dev];
}
}  // namespace

extern "C" sq_status w8a8_scaled_mm_noalloc(const int8_t* q_a, const float* s_tok,
                                            const int8_t* q_w, const float* s_ch, void* y_bf16,
                                            int64_t M, int64_t N, int64_t K, void* stream) {
  sq_status s = check_mnk(M, N, K);
  if (s != SQ_OK) return s;
  if (M == 0) return SQ_OK;
  if (!q_a || !s_tok || !q_w || !s_ch || !y_bf16) return SQ_ERR_NULL;
  if (!aligned16(q_a) || !aligned16(s_tok) || !aligned16(q_w) || !aligned16(s_ch) ||
      !aligned16(y_bf16))
    return SQ_ERR_ALIGN;
  const int sms = num_sms();
  if (sms <= 0) return SQ_ERR_CUDA;
  const GemmPlan p = plan_gemm(GK_I8_SCALE, M, N, K, sms);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (p.ws_bytes == 0)  // large M: this schedule needs no scratch at all
    return run_gemm(GK_I8_SCALE, q_a, q_w, s_tok, s_ch, nullptr, y_bf16, M, N, K, nullptr, 0,
                    st);
  if (p.ws_bytes > kNoAllocScratchBytes) return SQ_ERR_WORKSPACE;
  if (static_cast<int64_t>(p.tiles_r) * p.tiles_c > kMaxCounterTiles) return SQ_ERR_SHAPE;
  void* scratch = noalloc_scratch_address();
  if (!scratch) return SQ_ERR_CUDA;
  // The array keeps whatever the previous call left; the arrival counters
  // must start at zero, so clear the ones this call uses.
  if (cudaMemsetAsync(scratch, 0, static_cast<size_t>(p.tiles_r) * p.tiles_c * 4, st) !=
      cudaSuccess)
    return SQ_ERR_CUDA;
  return run_gemm(GK_I8_SCALE, q_a, q_w, s_tok, s_ch, nullptr, y_bf16, M, N, K, scratch,
                  kNoAllocScratchBytes, st);
}

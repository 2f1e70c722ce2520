// aria_q.cu -- the C ABI of libaria_q.so (declared in include/aria_q.h):
// host-side validation, tensor-map encoding, tile / split planning and
// launches of the sm_100a kernels. One translation unit, so the device
// status word is a single symbol without relocatable device code.
#include <cuda.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>

#include "aria_q.h"
#include "ptx.cuh"
#include "qgemm.cuh"
#include "quant_kernels.cuh"
#include "smallm.cuh"

#define ARIA_API extern "C" __attribute__((visibility("default")))

namespace {

thread_local char g_msg[512] = "";

aria_status fail(aria_status s, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_msg, sizeof(g_msg), fmt, ap);
  va_end(ap);
  return s;
}

aria_status cuda_fail(cudaError_t e, const char* what) {
  return fail(ARIA_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

constexpr int64_t kMaxDim = (int64_t{1} << 31) - 1;

// ------------------------------------------------------------ tensor maps ---
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

// 2-D row-major tensor [rows, cols] of `esize`-byte elements; box {bc, br}.
aria_status make_map(CUtensorMap* m, const void* base, CUtensorMapDataType dt, int esize,
                     int64_t rows, int64_t cols, int bc, int br, CUtensorMapSwizzle sw) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return fail(ARIA_ERR_CUDA, "cuTensorMapEncodeTiled unavailable");
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(cols * esize)};
  cuuint32_t box[2] = {static_cast<cuuint32_t>(bc), static_cast<cuuint32_t>(br)};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(m, dt, 2, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(ARIA_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", (int)r);
  return ARIA_OK;
}

// ---------------------------------------------------------- device facts ---
struct DevInfo {
  int sms = 148;
  int smem_optin = 232448;
};

constexpr int kMaxDevices = 64;

int current_device() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) dev = 0;
  return dev;
}

DevInfo dev_info() {
  static DevInfo info[kMaxDevices];
  static bool done[kMaxDevices] = {};
  static std::mutex mu;
  const int dev = current_device();
  std::lock_guard<std::mutex> g(mu);
  if (dev >= 0 && dev < kMaxDevices && !done[dev]) {
    cudaDeviceGetAttribute(&info[dev].sms, cudaDevAttrMultiProcessorCount, dev);
    cudaDeviceGetAttribute(&info[dev].smem_optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
    done[dev] = true;
  }
  return (dev >= 0 && dev < kMaxDevices) ? info[dev] : DevInfo{};
}

// ----------------------------------------------------------------- GEMM ---
struct Plan {
  aria::GemmParams p;
  dim3 grid;
  int threads;
  size_t smem;
};

aria_status plan_gemm(int kind, int64_t M, int64_t N, int64_t K, Plan* out) {
  using namespace aria;
  const DevInfo di = dev_info();
  GemmParams p{};
  p.M = static_cast<int>(M);
  p.N = static_cast<int>(N);
  p.K = static_cast<int>(K);
  const int unitK = kind == kQ4 ? 256 : (kind == kF16 ? 64 : 128);
  p.units = static_cast<int>((K + unitK - 1) / unitK);

  // Token tile: up to 256. W8A8 at M <= 512 uses narrower tiles (<= 160):
  // more output tiles fill the SMs, and without a dequant stage the per-tile
  // cost of a narrower MMA is small (measured: 15-25 % faster at M = 432).
  int max_bn = 256;
  if ((kind == kW8A8 || kind == kS32 || kind == kF16) && M <= 512) max_bn = 160;
#if defined(ARIA_MAX_BN)
  max_bn = ARIA_MAX_BN;  // tuning builds only
#endif
  auto tile_for = [&](int mt_try, int* bn_out) {  // token tile for mt_try token tiles
    int b = static_cast<int>((M + mt_try - 1) / mt_try);
    b = (b + 15) / 16 * 16;
    *bn_out = b;
    return static_cast<int>((M + b - 1) / b);
  };
  int bn = 0;
  int mt = tile_for(static_cast<int>((M + max_bn - 1) / max_bn), &bn);
  const int nt = static_cast<int>((N + kTileN - 1) / kTileN);
  // q8/q4 with a few hundred tokens: the dequant work per K block is the
  // same for any token tile, and a split-K launch costs several us of
  // cluster reduction. Measured at M = 432 (d = 1536 linears): prefer the
  // token tile that fills the most SMs (at least two thirds) without split-K;
  // otherwise one tile narrower than the widest when K is short (fewer
  // ranks to reduce), the widest when K is long (less K per rank).
  bool dq_policy = (kind == kQ8 || kind == kQ4) && M >= 128 && M <= 512;
#if defined(ARIA_MAX_BN)
  dq_policy = false;  // tuning builds pin the tile
#endif
  if (dq_policy) {
    const int mt0 = mt;
    int best_mt = 0, best_tiles = 0;
    for (int m_try = mt0; m_try <= mt0 + 2; ++m_try) {
      int b = 0;
      const int m_eff = tile_for(m_try, &b);
      const int64_t t = static_cast<int64_t>(nt) * m_eff;
      if (t <= di.sms && 3 * t >= 2 * static_cast<int64_t>(di.sms) && t > best_tiles) {
        best_tiles = static_cast<int>(t);
        best_mt = m_try;
      }
    }
    if (best_mt == 0) best_mt = K <= 2048 ? mt0 + 1 : mt0;
    mt = tile_for(best_mt, &bn);
  }
  // Many tokens (several tiles per CTA): the persistent CTAs take the tiles
  // round-robin, so the slowest CTA does ceil(tiles / SMs) of them. Pick the
  // token tile (a multiple of 16 in [128, 256]) that minimises that count
  // times the tile's width plus a fixed per-tile cost (16 token-columns'
  // worth), e.g. 176 instead of 256 for N = 1536 at M = 4096: 288 tiles in
  // two nearly full waves instead of 192 in two waves of which one is 30 %
  // full.
  bool wave_policy = M > 512;
#if defined(ARIA_MAX_BN)
  wave_policy = false;  // tuning builds pin the tile
#endif
  if (wave_policy) {
    int64_t best_cost = -1;
    for (int b = 256; b >= 128; b -= 16) {
      const int64_t m_t = (M + b - 1) / b;
      const int64_t waves = (static_cast<int64_t>(nt) * m_t + di.sms - 1) / di.sms;
      const int64_t cost = waves * (b + 16);
      if (best_cost < 0 || cost < best_cost) {
        best_cost = cost;
        bn = b;
        mt = static_cast<int>(m_t);
      }
    }
  }
  // W8A8 with few weight-row tiles and a short K: the narrowest token tile
  // that still leaves at least two thirds of the SMs busy without split-K
  // (measured at M = 432, N = K = 1536: 48-token tiles 6.8 us against 9.3 us
  // for 144-token tiles in 3-way split-K clusters; at K = 6144 the split
  // stays faster)
  bool narrow_policy = kind == kW8A8 && M <= 512 && K <= 2048 && static_cast<int64_t>(nt) * mt < di.sms;
#if defined(ARIA_MAX_BN)
  narrow_policy = false;  // tuning builds pin the tile
#endif
  if (narrow_policy) {
    for (int b = bn - 16; b >= 48; b -= 16) {
      const int64_t m_t = (M + b - 1) / b;
      const int64_t t = static_cast<int64_t>(nt) * m_t;
      if (t > di.sms) break;
      if (3 * t >= 2 * static_cast<int64_t>(di.sms)) {
        bn = b;
        mt = static_cast<int>(m_t);
        break;
      }
    }
  }
  p.BN = bn;
  const int64_t tiles = static_cast<int64_t>(nt) * mt;
  if (tiles > (int64_t{1} << 30)) return fail(ARIA_ERR_UNSUPPORTED, "too many tiles");
  p.tiles_n = nt;
  p.tiles = static_cast<int>(tiles);

  // split-K upper bound; the launcher lowers it until the clusters fit in one wave
  int splits = 1;
  if (tiles < di.sms) splits = static_cast<int>(std::min<int64_t>(8, di.sms / tiles));
  splits = std::max(1, std::min(splits, p.units));
#if defined(ARIA_FORCE_SPLITS)
  splits = std::max(1, std::min(std::min(ARIA_FORCE_SPLITS, p.units), static_cast<int>(di.sms / tiles)));  // tuning builds only
#endif
  p.splits = splits;

  const bool dq = (kind == kQ8 || kind == kQ4);
  // q8/q4 with one tile per CTA (every split-K CTA has one too): the A
  // operand lives in tensor memory, so a stage holds only the activation
  // tile; the ring depth stays <= 8 (8 A slots of 32 TMEM columns)
  const bool ta = dq && tiles <= di.sms;
  p.tmem_a = ta ? 1 : 0;
  const uint32_t a_tile = ta ? 0u : kATile;
  const uint32_t out_bytes = kind == kS32 ? 4 : 2;
  const uint32_t epi_warps = dq ? 4 : 8;
  const uint32_t stage_bytes = epi_warps * 2 * kEpiRows * 32 * out_bytes;  // 2 store boxes per warp
  const uint32_t sxd_bytes = 2 * aria::kTileBnMax * 4;  // W8A8 token scales, two m-tiles
  p.x_stage = static_cast<uint32_t>(bn) * 128u;
  p.raw_stage = kind == kQ8 ? kATile : (kind == kQ4 ? kATile + kQ4ScaleTile : 0);
  p.raw_stage = (p.raw_stage + 1023u) & ~1023u;
  const int64_t budget = static_cast<int64_t>(di.smem_optin) - 1024 - 512 - stage_bytes - sxd_bytes;
  // stage ring: one A tile + one X tile per stage (one MMA commit each);
  // q8/q4 also keep a ring of raw packed weight tiles for the dequant warps
  int nr = 0, na = 0, nx = 0;
  const int64_t st_bytes = a_tile + p.x_stage;
  int k_max = 8;
#if defined(ARIA_MAX_STAGES)
  k_max = ARIA_MAX_STAGES;  // tuning builds only
#endif
  for (int k = k_max; k >= 2 && na == 0; --k) {
    if (!dq) {
      if (k * st_bytes <= budget) na = k;
      continue;
    }
    for (int r = 4; r >= 2; --r)
      if (k * st_bytes + static_cast<int64_t>(r) * p.raw_stage <= budget) {
        na = k;
        nr = r;
        break;
      }
  }
  if (na == 0) return fail(ARIA_ERR_UNSUPPORTED, "tile does not fit in shared memory");
  nx = na;
  p.n_raw = nr;
  p.n_a = na;
  p.n_x = nx;
  p.off_raw = 0;
  p.off_a = p.off_raw + nr * p.raw_stage;
  p.off_x = p.off_a + na * a_tile;
  p.off_stage = p.off_x + nx * p.x_stage;
  p.off_sxd = p.off_stage + stage_bytes;
  p.off_bar = p.off_sxd + sxd_bytes;
  // the split-K partial tile (BN rows x 512 B) overlays the stage rings
  if (static_cast<uint32_t>(bn) * 512u > p.off_stage) p.splits = splits = 1;
  // warps 0..3 help with the last tile's epilogue when their store boxes (and
  // W8A8 token scales) fit in the activation ring
  const uint64_t helper_bytes = 8ull * kEpiRows * 32 * out_bytes + 4ull * kTileBnMax;
  p.helpers = static_cast<uint64_t>(nx) * p.x_stage >= helper_bytes ? 1 : 0;
  const uint32_t nbar = 2 * (nr + na) + 6;  // raw, stage, 2 acc_full, 2 acc_empty, mma_drain, acc_last
  const size_t smem = 1024 + p.off_bar + nbar * 8 + 16;
  if (smem > static_cast<size_t>(di.smem_optin)) return fail(ARIA_ERR_UNSUPPORTED, "shared memory plan too large");

  out->p = p;
  out->grid = dim3(static_cast<unsigned>(std::min<int64_t>(tiles, di.sms)), 1, 1);
  out->threads = 384;
  out->smem = smem;
  return ARIA_OK;
}

// Trace builds: each GEMM launch gets the next trace row block (see
// ARIA_STAMP); 0 otherwise.
#ifdef ARIA_TRACE
std::atomic<int> g_trace_launches{0};
int next_trace_launch() { return g_trace_launches.fetch_add(1); }
#else
int next_trace_launch() { return 0; }
#endif

// programmatic dependent launch: the kernel may start while the previous
// kernel in the stream drains; it waits (griddepcontrol.wait) before reading
// anything that kernel may write (the GEMM's packed weights are the one
// exception, see the stream-order note of aria_qgemm in the header)
void set_pdl(cudaLaunchConfig_t& cfg, cudaLaunchAttribute* attr) {
  attr[cfg.numAttrs].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[cfg.numAttrs].val.programmaticStreamSerializationAllowed = 1;
  cfg.numAttrs++;
  cfg.attrs = attr;
}

// how many clusters of `size` CTAs of this kernel can be resident at once on
// the current device (cached per device, size and shared-memory footprint;
// queried outside any capture on first use)
template <int KIND>
int max_clusters(int size, int threads, size_t smem) {
  static std::mutex mu;
  static int cache_dev[64], cache_size[64], cache_n[64];
  static size_t cache_smem[64];
  static int used = 0;
  const int dev = current_device();
  std::lock_guard<std::mutex> g(mu);
  for (int i = 0; i < used; ++i)
    if (cache_dev[i] == dev && cache_size[i] == size && cache_smem[i] == smem) return cache_n[i];
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(size, 1, 1);
  cfg.blockDim = dim3(threads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = size;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, aria::qgemm_kernel<KIND>, &cfg) != cudaSuccess) {
    cudaGetLastError();
    n = 0;
  }
  if (used < 64) {
    cache_dev[used] = dev;
    cache_size[used] = size;
    cache_smem[used] = smem;
    cache_n[used] = n;
    ++used;
  }
  return n;
}

// Raise a kernel's dynamic shared-memory limit to the device's opt-in
// maximum, once per kernel and device (the attribute is per device).
template <typename F>
aria_status opt_in_smem(F* kfn, bool (&done)[kMaxDevices], std::mutex& mu) {
  const int dev = current_device();
  if (dev < 0 || dev >= kMaxDevices) return fail(ARIA_ERR_UNSUPPORTED, "device index %d", dev);
  std::lock_guard<std::mutex> g(mu);
  if (done[dev]) return ARIA_OK;
  cudaError_t e = cudaFuncSetAttribute(kfn, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       dev_info().smem_optin);
  if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute");
  done[dev] = true;
  return ARIA_OK;
}

template <int KIND>
aria_status launch_gemm(const Plan& pl, const CUtensorMap& tw, const CUtensorMap& ts,
                        const CUtensorMap& tx, cudaStream_t st) {
  auto kfn = aria::qgemm_kernel<KIND>;
  static bool attr_done[kMaxDevices] = {};
  static std::mutex attr_mu;
  aria_status as = opt_in_smem(kfn, attr_done, attr_mu);
  if (as != ARIA_OK) return as;
  aria::GemmParams prm = pl.p;
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = pl.grid;
  cfg.blockDim = dim3(pl.threads, 1, 1);
  cfg.dynamicSmemBytes = pl.smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  cfg.numAttrs = 0;
  // largest split whose clusters are all co-resident (one wave)
  while (prm.splits > 1 && max_clusters<KIND>(prm.splits, pl.threads, pl.smem) < prm.tiles) --prm.splits;
  if (prm.splits > 1) {
    cfg.gridDim = dim3(prm.splits, prm.tiles, 1);
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = prm.splits;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.numAttrs = 1;
    cfg.attrs = attr;
  }
  set_pdl(cfg, attr);
  prm.trace_launch = next_trace_launch();
  cudaError_t e = cudaLaunchKernelEx(&cfg, kfn, tw, ts, tx, prm);
  if (e != cudaSuccess) return cuda_fail(e, "qgemm launch");
  return ARIA_OK;
}

// ------------------------------------------------------------- few tokens ---
// Plan of the few-token weight-only GEMM (smallm_kernel): the smallest
// cluster size S (K split) that keeps each warp's activation chunks in
// registers and the activations read per CTA at or below 32 KB, with the
// rows divided over as many clusters as the SMs hold. False when no plan
// fits (then the tensor-core kernel runs).
struct SmallPlan {
  aria::SmallParams p;
  int grid = 0, tb = 1, ch = 8;
  size_t smem = 0;
};

constexpr int64_t kSmallMaxTokens = 16;
constexpr size_t kSmallSmemBudget = 110 * 1024;  // two CTAs per SM

template <int KIND, int TB, int CH, int GP>
int small_max_clusters(int size, size_t smem) {
  static std::mutex mu;
  static int cache_dev[64], cache_size[64], cache_n[64];
  static size_t cache_smem[64];
  static int used = 0;
  const int dev = current_device();
  std::lock_guard<std::mutex> g(mu);
  for (int i = 0; i < used; ++i)
    if (cache_dev[i] == dev && cache_size[i] == size && cache_smem[i] == smem) return cache_n[i];
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(size, 1, 1);
  cfg.blockDim = dim3(aria::kSmThreads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = size;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, aria::smallm_kernel<KIND, TB, CH, GP>, &cfg) != cudaSuccess) {
    cudaGetLastError();
    n = 0;
  }
  if (used < 64) {
    cache_dev[used] = dev;
    cache_size[used] = size;
    cache_smem[used] = smem;
    cache_n[used] = n;
    ++used;
  }
  return n;
}

// shared-memory layout of a plan with `clusters` clusters of S CTAs
bool small_layout(int kind, int64_t M, int64_t N, int64_t K, int S, int clusters, int tb, int gp,
                  aria::SmallParams* p, size_t* smem) {
  using namespace aria;
  const int num = kind == kF16 ? 2 : 1, den = kind == kQ4 ? 2 : 1;
  p->S = S;
  p->kslice = static_cast<int>(K / S);
  p->rows_base = static_cast<int>(N / clusters);
  p->rows_rem = static_cast<int>(N % clusters);
  const int rmax = p->rows_base + (p->rows_rem ? 1 : 0);
  p->r_pad = (rmax + 15) / 16 * 16;
  const uint32_t slice = static_cast<uint32_t>(p->kslice) * num / den;
  p->wrow = slice + 16;
  auto up = [](uint64_t v, uint64_t a) { return (v + a - 1) / a * a; };
  uint64_t off = up(static_cast<uint64_t>(rmax) * p->wrow, 128);
  p->off_sc = static_cast<uint32_t>(off);
  if (kind == kQ4) off = up(off + static_cast<uint64_t>(rmax) * (p->kslice / 16), 128);
  p->off_red = static_cast<uint32_t>(off);
  off += static_cast<uint64_t>(kSmWarps) * tb * 8 * sm_red_stride(gp) * 4;
  p->off_part = static_cast<uint32_t>(up(off, 128));
  off = p->off_part + (S > 1 ? static_cast<uint64_t>(tb) * 8 * (p->r_pad + 4) * 4 : 0);
  p->off_bar = static_cast<uint32_t>(up(off, 16));
  p->off_sw = p->off_bar + 16;  // q8 channel scales of the rows
  *smem = p->off_sw + static_cast<uint64_t>(rmax) * 4;
  (void)M;
  return *smem <= kSmallSmemBudget;
}

template <int KIND, int TB, int CH, int GP>
bool plan_small_t(int64_t M, int64_t N, int64_t K, SmallPlan* out) {
  using namespace aria;
  const DevInfo di = dev_info();
  const int unit = KIND == kQ4 ? 256 : 64;
  if (K % unit) return false;
  int best_s = 0;
  for (int S = 1; S <= 8; ++S) {
    if (K % (static_cast<int64_t>(S) * unit)) continue;
    const int64_t kslice = K / S;
    if ((kslice / 64 + kSmWarps - 1) / kSmWarps > CH) continue;  // activation chunks in registers
    best_s = S;
    if (M * kslice * 2 <= 32768) break;  // activations read per CTA: small enough
  }
  if (best_s == 0) return false;
  const int S = best_s;
  int clusters = static_cast<int>(std::min<int64_t>(di.sms / S, N));
  SmallParams p{};
  size_t smem = 0;
  if (!small_layout(KIND, M, N, K, S, clusters, TB, GP, &p, &smem)) return false;
  if (S > 1) {
    const int fit = small_max_clusters<KIND, TB, CH, GP>(S, smem);
    if (fit < 1) return false;
    if (fit < clusters) {
      clusters = fit;
      if (!small_layout(KIND, M, N, K, S, clusters, TB, GP, &p, &smem)) return false;
    }
  }
  p.M = static_cast<int>(M);
  p.N = static_cast<int>(N);
  p.K = static_cast<int>(K);
  out->p = p;
  out->grid = clusters * S;
  out->tb = TB;
  out->ch = CH;
  out->smem = smem;
  return true;
}

bool plan_small(int kind, int64_t M, int64_t N, int64_t K, SmallPlan* out) {
  using namespace aria;
  if (M > kSmallMaxTokens) return false;
  const bool two = M > 8;
  switch (kind) {
    case kQ8: return two ? plan_small_t<kQ8, 2, 4, 2>(M, N, K, out) : plan_small_t<kQ8, 1, 6, 4>(M, N, K, out);
    case kQ4: return two ? plan_small_t<kQ4, 2, 4, 2>(M, N, K, out) : plan_small_t<kQ4, 1, 6, 4>(M, N, K, out);
    case kF16: return two ? plan_small_t<kF16, 2, 4, 2>(M, N, K, out) : plan_small_t<kF16, 1, 6, 4>(M, N, K, out);
  }
  return false;
}

template <int KIND, int TB, int CH, int GP>
aria_status launch_small_t(const SmallPlan& pl, cudaStream_t st) {
  auto kfn = aria::smallm_kernel<KIND, TB, CH, GP>;
  static bool attr_done[kMaxDevices] = {};
  static std::mutex attr_mu;
  aria_status as = opt_in_smem(kfn, attr_done, attr_mu);
  if (as != ARIA_OK) return as;
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(static_cast<unsigned>(pl.grid), 1, 1);
  cfg.blockDim = dim3(aria::kSmThreads, 1, 1);
  cfg.dynamicSmemBytes = pl.smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  cfg.numAttrs = 0;
  if (pl.p.S > 1) {
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = pl.p.S;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.numAttrs = 1;
    cfg.attrs = attr;
  }
  set_pdl(cfg, attr);
  aria::SmallParams sp = pl.p;
  sp.trace_launch = next_trace_launch();
  cudaError_t e = cudaLaunchKernelEx(&cfg, kfn, sp);
  if (e != cudaSuccess) return cuda_fail(e, "few-token GEMM launch");
  return ARIA_OK;
}

aria_status launch_small(int kind, const SmallPlan& pl, cudaStream_t st) {
  using namespace aria;
  const bool two = pl.tb == 2;
  switch (kind) {
    case kQ8: return two ? launch_small_t<kQ8, 2, 4, 2>(pl, st) : launch_small_t<kQ8, 1, 6, 4>(pl, st);
    case kQ4: return two ? launch_small_t<kQ4, 2, 4, 2>(pl, st) : launch_small_t<kQ4, 1, 6, 4>(pl, st);
    case kF16: return two ? launch_small_t<kF16, 2, 4, 2>(pl, st) : launch_small_t<kF16, 1, 6, 4>(pl, st);
  }
  return fail(ARIA_ERR_INVALID_ARG, "unknown kind");
}

aria_status check_gemm_shape(int64_t M, int64_t N, int64_t K) {
  if (M < 1 || N < 1 || K < 1 || M > kMaxDim || N > kMaxDim || K > kMaxDim)
    return fail(ARIA_ERR_INVALID_ARG, "sizes must be positive and < 2^31 (M=%lld N=%lld K=%lld)",
                (long long)M, (long long)N, (long long)K);
  if (N < 16 || N % 16) return fail(ARIA_ERR_UNSUPPORTED, "N must be a positive multiple of 16");
  if (K < 16 || K % 16) return fail(ARIA_ERR_UNSUPPORTED, "K must be a positive multiple of 16");
  return ARIA_OK;
}

}  // namespace

// ================================================================= ABI ===

ARIA_API const char* aria_status_string(aria_status s) {
  switch (s) {
    case ARIA_OK: return "ARIA_OK";
    case ARIA_ERR_INVALID_ARG: return "ARIA_ERR_INVALID_ARG";
    case ARIA_ERR_UNSUPPORTED: return "ARIA_ERR_UNSUPPORTED";
    case ARIA_ERR_MISALIGNED: return "ARIA_ERR_MISALIGNED";
    case ARIA_ERR_CUDA: return "ARIA_ERR_CUDA";
    case ARIA_ERR_TIMEOUT: return "ARIA_ERR_TIMEOUT";
  }
  return "ARIA_ERR_UNKNOWN";
}

ARIA_API const char* aria_last_error_message(void) { return g_msg; }

ARIA_API aria_status aria_qpack_size(aria_format fmt, int group, int64_t N, int64_t K,
                                     size_t* wq_bytes, size_t* scale_bytes) {
  if (!wq_bytes || !scale_bytes) return fail(ARIA_ERR_INVALID_ARG, "NULL output pointer");
  if (N < 1 || K < 1 || N > kMaxDim || K > kMaxDim)
    return fail(ARIA_ERR_INVALID_ARG, "N and K must be in [1, 2^31)");
  if (fmt == ARIA_FMT_Q8 || fmt == ARIA_FMT_W8A8) {
    if (group != 0) return fail(ARIA_ERR_UNSUPPORTED, "q8 scales are per output channel: group must be 0");
    *wq_bytes = static_cast<size_t>(N) * K;
    *scale_bytes = static_cast<size_t>(N) * 4;
    return ARIA_OK;
  }
  if (fmt == ARIA_FMT_F16)
    return fail(ARIA_ERR_UNSUPPORTED, "fp16 weights are used as they are, not packed");
  if (fmt == ARIA_FMT_Q4) {
    if (group != 32) return fail(ARIA_ERR_UNSUPPORTED, "q4 supports group = 32 only");
    if (K % 32) return fail(ARIA_ERR_UNSUPPORTED, "q4 needs K % 32 == 0");
    *wq_bytes = static_cast<size_t>(N) * (K / 2);
    *scale_bytes = static_cast<size_t>(N) * (K / 32) * 2;
    return ARIA_OK;
  }
  return fail(ARIA_ERR_INVALID_ARG, "unknown format %d", (int)fmt);
}

ARIA_API aria_status aria_qpack(aria_format fmt, int group, const void* W, int64_t N, int64_t K,
                                void* Wq, void* scales, void* stream) {
  size_t wb = 0, sb = 0;
  aria_status s = aria_qpack_size(fmt, group, N, K, &wb, &sb);
  if (s != ARIA_OK) return s;
  if (!W || !Wq || !scales) return fail(ARIA_ERR_INVALID_ARG, "NULL device pointer");
  if (!aligned16(W) || !aligned16(Wq) || !aligned16(scales))
    return fail(ARIA_ERR_MISALIGNED, "device pointers must be 16-byte aligned");
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  cudaLaunchConfig_t cfg{};
  cudaLaunchAttribute attr[1];
  cfg.stream = st;
  set_pdl(cfg, attr);
  cudaError_t e;
  if (fmt == ARIA_FMT_Q4) {
    const int64_t nchunk = N * (K / 8);
    const int64_t blocks = std::min<int64_t>((nchunk + 255) / 256, int64_t{dev_info().sms} * 16);
    cfg.gridDim = dim3(static_cast<unsigned>(blocks));
    cfg.blockDim = dim3(256);
    e = cudaLaunchKernelEx(&cfg, aria::pack_q4_kernel, static_cast<const __half*>(W), nchunk,
                           static_cast<uint32_t*>(Wq), static_cast<__half*>(scales));
  } else {
    if (K % 16) return fail(ARIA_ERR_UNSUPPORTED, "q8 needs K % 16 == 0");
    cfg.gridDim = dim3(static_cast<unsigned>(N));
    cfg.blockDim = dim3(aria::kRowThreads);
    e = cudaLaunchKernelEx(&cfg, aria::row_quant_i8_kernel, static_cast<const __half*>(W),
                           static_cast<int>(K), static_cast<int8_t*>(Wq), static_cast<float*>(scales),
                           false);
  }
  if (e != cudaSuccess) return cuda_fail(e, "pack launch");
  return ARIA_OK;
}

ARIA_API aria_status aria_act_quant(const void* X, int64_t M, int64_t K, int8_t* Xq, float* sx,
                                    void* stream) {
  if (!X || !Xq || !sx) return fail(ARIA_ERR_INVALID_ARG, "NULL device pointer");
  if (M < 1 || K < 1 || M > kMaxDim || K > kMaxDim)
    return fail(ARIA_ERR_INVALID_ARG, "M and K must be in [1, 2^31)");
  if (K % 16) return fail(ARIA_ERR_UNSUPPORTED, "K must be a multiple of 16");
  if (!aligned16(X) || !aligned16(Xq) || !aligned16(sx))
    return fail(ARIA_ERR_MISALIGNED, "device pointers must be 16-byte aligned");
  cudaLaunchConfig_t cfg{};
  cudaLaunchAttribute attr[1];
  cfg.stream = static_cast<cudaStream_t>(stream);
  cfg.gridDim = dim3(static_cast<unsigned>(M));
  cfg.blockDim = dim3(aria::kRowThreads);
  set_pdl(cfg, attr);
  cudaError_t e = cudaLaunchKernelEx(&cfg, aria::row_quant_i8_kernel, static_cast<const __half*>(X),
                                     static_cast<int>(K), Xq, sx, true);
  if (e != cudaSuccess) return cuda_fail(e, "act_quant launch");
  return ARIA_OK;
}

// Workspace of the fused W8A8 call: [0, 256) the grid barrier {arrivals,
// generation}; then the token scales fp32 [M]; then the codes int8 [M,K], at
// 256-byte aligned offsets (TMA reads the codes).
struct FusedWs {
  unsigned* gbar;
  float* sx;
  int8_t* xq;
};

constexpr size_t kWsHeader = 256;

size_t fused_ws_bytes(int64_t M, int64_t K) {
  const size_t sx = (static_cast<size_t>(M) * 4 + 255) / 256 * 256;
  return kWsHeader + sx + static_cast<size_t>(M) * static_cast<size_t>(K);
}

FusedWs fused_ws(void* ws, int64_t M) {
  uint8_t* b = static_cast<uint8_t*>(ws);
  const size_t sx = (static_cast<size_t>(M) * 4 + 255) / 256 * 256;
  return FusedWs{reinterpret_cast<unsigned*>(b), reinterpret_cast<float*>(b + kWsHeader),
                 reinterpret_cast<int8_t*>(b + kWsHeader + sx)};
}

// the failure-detection self-test's settings of a launch (defaults: none)
struct SelfTest {
  uint64_t wait_ns = 0;
  int drop_first_stage = 0;
};

static aria_status qgemm_impl(int kind, int64_t M, int64_t N, int64_t K, const void* X,
                              const float* sx, const void* Wq, const void* scales,
                              const void* bias, const float* steer, float alpha,
                              const float* alpha_dev, void* Y, cudaStream_t st,
                              const void* xf16 = nullptr, const FusedWs* ws = nullptr,
                              const SelfTest& selftest = SelfTest{}) {
  using namespace aria;
  aria_status s = check_gemm_shape(M, N, K);
  if (s != ARIA_OK) return s;
  if (kind == kQ4 && K % 256) return fail(ARIA_ERR_UNSUPPORTED, "q4 GEMM needs K % 256 == 0");
  // exact int32 accumulation: |acc| <= K * 127^2 must stay below 2^31
  if ((kind == kW8A8 || kind == kS32) && K * 127 * 127 > INT32_MAX)
    return fail(ARIA_ERR_UNSUPPORTED, "int8 GEMM needs K * 127^2 < 2^31 (K <= %lld), got K=%lld",
                (long long)(INT32_MAX / (127 * 127)), (long long)K);
  // a handful of tokens: the weight-streaming kernel, when its plan fits
  SmallPlan sp;
  if (!xf16 && !selftest.drop_first_stage && plan_small(kind, M, N, K, &sp)) {
    sp.p.W = static_cast<const uint8_t*>(Wq);
    sp.p.Wsc = kind == kQ4 ? static_cast<const __half*>(scales) : nullptr;
    sp.p.sw = kind == kQ8 ? static_cast<const float*>(scales) : nullptr;
    sp.p.X = static_cast<const __half*>(X);
    sp.p.bias = static_cast<const __half*>(bias);
    sp.p.steer = (steer && (alpha_dev || alpha != 0.0f)) ? steer : nullptr;
    sp.p.alpha = sp.p.steer ? alpha : 0.0f;
    sp.p.alpha_dev = sp.p.steer ? alpha_dev : nullptr;
    sp.p.Y = static_cast<__half*>(Y);
    return launch_small(kind, sp, st);
  }
  Plan pl;
  if ((s = plan_gemm(kind, M, N, K, &pl)) != ARIA_OK) return s;
  CUtensorMap tw, ts, tx;
  std::memset(&ts, 0, sizeof(ts));
  const int bn = pl.p.BN;
  if (kind == kQ4) {
    if ((s = make_map(&tw, Wq, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, N, K / 2, 128, 128,
                      CU_TENSOR_MAP_SWIZZLE_128B)) != ARIA_OK) return s;
    if ((s = make_map(&ts, scales, CU_TENSOR_MAP_DATA_TYPE_UINT16, 2, N, K / 32, 8, 128,
                      CU_TENSOR_MAP_SWIZZLE_NONE)) != ARIA_OK) return s;
  } else if (kind == kF16) {
    if ((s = make_map(&tw, Wq, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, N, K, 64, 128,
                      CU_TENSOR_MAP_SWIZZLE_128B)) != ARIA_OK) return s;
  } else {
    if ((s = make_map(&tw, Wq, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, N, K, 128, 128,
                      CU_TENSOR_MAP_SWIZZLE_128B)) != ARIA_OK) return s;
  }
  if (kind == kQ8 || kind == kQ4 || kind == kF16) {
    if ((s = make_map(&tx, X, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, M, K, 64, bn,
                      CU_TENSOR_MAP_SWIZZLE_128B)) != ARIA_OK) return s;
  } else {
    if ((s = make_map(&tx, X, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, M, K, 128, bn,
                      CU_TENSOR_MAP_SWIZZLE_128B)) != ARIA_OK) return s;
  }
  pl.p.sw = static_cast<const float*>((kind == kQ4 || kind == kF16) ? nullptr : scales);
  pl.p.sx = sx;
  pl.p.bias = static_cast<const __half*>(bias);
  // skip, not "+ 0*v": a host alpha of 0 drops the vector here; a device
  // alpha is tested in the kernel
  pl.p.steer = (steer && (alpha_dev || alpha != 0.0f)) ? steer : nullptr;
  pl.p.alpha = pl.p.steer ? alpha : 0.0f;
  pl.p.alpha_dev = pl.p.steer ? alpha_dev : nullptr;
  pl.p.Y = Y;
  pl.p.wait_ns = selftest.wait_ns;
  pl.p.drop_first_stage = selftest.drop_first_stage;
  if (xf16) {  // W8A8 with the activation quantisation in this launch
    pl.p.xf16 = static_cast<const __half*>(xf16);
    pl.p.xq_ws = ws->xq;
    pl.p.sx_ws = ws->sx;
    pl.p.gbar = ws->gbar;
    pl.p.sx = ws->sx;
  }
  switch (kind) {
    case kQ8: return launch_gemm<kQ8>(pl, tw, tw, tx, st);
    case kQ4: return launch_gemm<kQ4>(pl, tw, ts, tx, st);
    case kW8A8: return launch_gemm<kW8A8>(pl, tw, tw, tx, st);
    case kS32: return launch_gemm<kS32>(pl, tw, tw, tx, st);
    case kF16: return launch_gemm<kF16>(pl, tw, tw, tx, st);
  }
  return fail(ARIA_ERR_INVALID_ARG, "unknown kind");
}

// argument checks shared by aria_qgemm and aria_qgemm_steer_dev; sets *kind
static aria_status check_qgemm_args(aria_format fmt, int group, const void* X, const float* sx,
                                    const void* Wq, const void* scales, const void* bias,
                                    const float* steer_vec, const void* Y, int* kind) {
  if (!X || !Wq || !Y) return fail(ARIA_ERR_INVALID_ARG, "NULL device pointer");
  if (fmt == ARIA_FMT_Q8 || fmt == ARIA_FMT_W8A8) {
    if (group != 0) return fail(ARIA_ERR_UNSUPPORTED, "q8 scales are per output channel: group must be 0");
    *kind = fmt == ARIA_FMT_Q8 ? aria::kQ8 : aria::kW8A8;
  } else if (fmt == ARIA_FMT_Q4) {
    if (group != 32) return fail(ARIA_ERR_UNSUPPORTED, "q4 supports group = 32 only");
    *kind = aria::kQ4;
  } else if (fmt == ARIA_FMT_F16) {
    if (group != 0) return fail(ARIA_ERR_UNSUPPORTED, "fp16 weights have no groups: group must be 0");
    *kind = aria::kF16;
  } else {
    return fail(ARIA_ERR_INVALID_ARG, "unknown format %d", (int)fmt);
  }
  if (*kind == aria::kF16) {
    if (scales) return fail(ARIA_ERR_INVALID_ARG, "fp16 weights take no scales (pass NULL)");
  } else if (!scales) {
    return fail(ARIA_ERR_INVALID_ARG, "NULL device pointer");
  }
  if (*kind == aria::kW8A8 && !sx) return fail(ARIA_ERR_INVALID_ARG, "W8A8 needs sx");
  if (*kind != aria::kW8A8 && sx) return fail(ARIA_ERR_INVALID_ARG, "sx is for W8A8 only");
  for (const void* q : {X, static_cast<const void*>(sx), Wq, scales, bias,
                        static_cast<const void*>(steer_vec), Y})
    if (q && !aligned16(q)) return fail(ARIA_ERR_MISALIGNED, "device pointers must be 16-byte aligned");
  return ARIA_OK;
}

ARIA_API aria_status aria_qgemm(aria_format fmt, int group, int64_t M, int64_t N, int64_t K,
                                const void* X, const float* sx, const void* Wq, const void* scales,
                                const void* bias, const float* steer_vec, float alpha, void* Y,
                                void* stream) {
  int kind = 0;
  aria_status s = check_qgemm_args(fmt, group, X, sx, Wq, scales, bias, steer_vec, Y, &kind);
  if (s != ARIA_OK) return s;
  return qgemm_impl(kind, M, N, K, X, sx, Wq, scales, bias, steer_vec, alpha, nullptr, Y,
                    static_cast<cudaStream_t>(stream));
}

ARIA_API aria_status aria_qgemm_steer_dev(aria_format fmt, int group, int64_t M, int64_t N,
                                          int64_t K, const void* X, const float* sx,
                                          const void* Wq, const void* scales, const void* bias,
                                          const float* steer_vec, const float* alpha_dev, void* Y,
                                          void* stream) {
  int kind = 0;
  aria_status s = check_qgemm_args(fmt, group, X, sx, Wq, scales, bias, steer_vec, Y, &kind);
  if (s != ARIA_OK) return s;
  if (steer_vec && !alpha_dev)
    return fail(ARIA_ERR_INVALID_ARG, "a steering vector needs a device alpha");
  if (alpha_dev && (reinterpret_cast<uintptr_t>(alpha_dev) & 3u))
    return fail(ARIA_ERR_MISALIGNED, "alpha_dev must be 4-byte aligned");
  return qgemm_impl(kind, M, N, K, X, sx, Wq, scales, bias, steer_vec, 0.0f, alpha_dev, Y,
                    static_cast<cudaStream_t>(stream));
}

ARIA_API aria_status aria_w8a8_workspace_size(int64_t M, int64_t K, size_t* bytes) {
  if (!bytes) return fail(ARIA_ERR_INVALID_ARG, "NULL output pointer");
  if (M < 1 || K < 1 || M > kMaxDim || K > kMaxDim)
    return fail(ARIA_ERR_INVALID_ARG, "M and K must be in [1, 2^31)");
  *bytes = fused_ws_bytes(M, K);
  return ARIA_OK;
}

ARIA_API aria_status aria_qgemm_w8a8_fused(int64_t M, int64_t N, int64_t K, const void* X,
                                           const void* Wq, const float* sw, const void* bias,
                                           const float* steer_vec, float alpha,
                                           const float* alpha_dev, void* Y, void* workspace,
                                           size_t workspace_bytes, void* stream) {
  if (!X || !Wq || !sw || !Y || !workspace) return fail(ARIA_ERR_INVALID_ARG, "NULL device pointer");
  for (const void* q : {X, static_cast<const void*>(Wq), static_cast<const void*>(sw), bias,
                        static_cast<const void*>(steer_vec), static_cast<const void*>(Y)})
    if (q && !aligned16(q)) return fail(ARIA_ERR_MISALIGNED, "device pointers must be 16-byte aligned");
  if (reinterpret_cast<uintptr_t>(workspace) & 255u)
    return fail(ARIA_ERR_MISALIGNED, "the workspace must be 256-byte aligned");
  if (alpha_dev && (reinterpret_cast<uintptr_t>(alpha_dev) & 3u))
    return fail(ARIA_ERR_MISALIGNED, "alpha_dev must be 4-byte aligned");
  aria_status s = check_gemm_shape(M, N, K);
  if (s != ARIA_OK) return s;
  if (workspace_bytes < fused_ws_bytes(M, K))
    return fail(ARIA_ERR_INVALID_ARG, "workspace of %zu bytes, %zu needed", workspace_bytes,
                fused_ws_bytes(M, K));
  const FusedWs ws = fused_ws(workspace, M);
  return qgemm_impl(aria::kW8A8, M, N, K, ws.xq, ws.sx, Wq, sw, bias, steer_vec, alpha, alpha_dev, Y,
                    static_cast<cudaStream_t>(stream), X, &ws);
}

// ------------------------------------------------- no-allocation variant ---
// Scratch of aria_qgemm_w8a8_fused_noalloc: a file-scope device array that
// every GPU loading this library holds until the process exits. Host code
// must not pass the symbol itself to a kernel (on the host it names a
// stand-in, not device memory): its device address comes from
// cudaGetSymbolAddress, once per device, with that device current.
constexpr size_t kNoAllocScratchBytes = size_t{32} << 20;  // 32 MiB
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

static aria_status noalloc_scratch(void** out) {
  static void* addr[kMaxDevices] = {};
  static std::mutex mu;
  const int dev = current_device();
  if (dev < 0 || dev >= kMaxDevices) return fail(ARIA_ERR_UNSUPPORTED, "device index %d", dev);
  std::lock_guard<std::mutex> g(mu);
  if (!addr[dev]) {
    void* p = nullptr;
    cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress of the static scratch");
    addr[dev] = p;
  }
  *out = addr[dev];
  return ARIA_OK;
}

ARIA_API aria_status aria_qgemm_w8a8_fused_noalloc(int64_t M, int64_t N, int64_t K, const void* X,
                                                   const void* Wq, const float* sw, const void* bias,
                                                   const float* steer_vec, float alpha,
                                                   const float* alpha_dev, void* Y, void* stream) {
  if (!X || !Wq || !sw || !Y) return fail(ARIA_ERR_INVALID_ARG, "NULL device pointer");
  for (const void* q : {X, static_cast<const void*>(Wq), static_cast<const void*>(sw), bias,
                        static_cast<const void*>(steer_vec), static_cast<const void*>(Y)})
    if (q && !aligned16(q)) return fail(ARIA_ERR_MISALIGNED, "device pointers must be 16-byte aligned");
  if (alpha_dev && (reinterpret_cast<uintptr_t>(alpha_dev) & 3u))
    return fail(ARIA_ERR_MISALIGNED, "alpha_dev must be 4-byte aligned");
  aria_status s = check_gemm_shape(M, N, K);
  if (s != ARIA_OK) return s;
  const size_t need = fused_ws_bytes(M, K);
  if (need > kNoAllocScratchBytes)
    return fail(ARIA_ERR_UNSUPPORTED,
                "M=%lld K=%lld needs %zu bytes of scratch; the static scratch holds %zu "
                "(256 + 4*M rounded up to 256 + M*K must fit)",
                (long long)M, (long long)K, need, kNoAllocScratchBytes);
  void* scratch = nullptr;
  if ((s = noalloc_scratch(&scratch)) != ARIA_OK) return s;
  // the grid barrier's words must start at zero; the array keeps whatever
  // the last call left (a call that gave up leaves them non-zero)
  cudaError_t e = cudaMemsetAsync(scratch, 0, kWsHeader, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "clearing the static scratch's barrier");
  const FusedWs ws = fused_ws(scratch, M);
  return qgemm_impl(aria::kW8A8, M, N, K, ws.xq, ws.sx, Wq, sw, bias, steer_vec, alpha, alpha_dev, Y,
                    static_cast<cudaStream_t>(stream), X, &ws);
}

ARIA_API aria_status aria_qgemm_s32(int64_t M, int64_t N, int64_t K, const int8_t* Xq,
                                    const int8_t* Wq, int32_t* C, void* stream) {
  if (!Xq || !Wq || !C) return fail(ARIA_ERR_INVALID_ARG, "NULL device pointer");
  if (!aligned16(Xq) || !aligned16(Wq) || !aligned16(C))
    return fail(ARIA_ERR_MISALIGNED, "device pointers must be 16-byte aligned");
  return qgemm_impl(aria::kS32, M, N, K, Xq, nullptr, Wq, Wq, nullptr, nullptr, 0.0f, nullptr, C,
                    static_cast<cudaStream_t>(stream));
}

ARIA_API aria_status aria_selftest_bounded_wait(int64_t M, int64_t N, int64_t K, const int8_t* Xq,
                                               const float* sx, const int8_t* Wq, const float* sw,
                                               void* Y, uint32_t wait_limit_us, void* stream) {
  if (!Xq || !sx || !Wq || !sw || !Y) return fail(ARIA_ERR_INVALID_ARG, "NULL device pointer");
  for (const void* q : {static_cast<const void*>(Xq), static_cast<const void*>(sx),
                        static_cast<const void*>(Wq), static_cast<const void*>(sw),
                        static_cast<const void*>(Y)})
    if (!aligned16(q)) return fail(ARIA_ERR_MISALIGNED, "device pointers must be 16-byte aligned");
  if (wait_limit_us < 1 || wait_limit_us > 4000000u)
    return fail(ARIA_ERR_INVALID_ARG, "wait_limit_us must be in [1, 4e6]");
  SelfTest t;
  t.wait_ns = static_cast<uint64_t>(wait_limit_us) * 1000u;
  t.drop_first_stage = 1;
  return qgemm_impl(aria::kW8A8, M, N, K, Xq, sx, Wq, sw, nullptr, nullptr, 0.0f, nullptr, Y,
                    static_cast<cudaStream_t>(stream), nullptr, nullptr, t);
}

ARIA_API aria_status aria_device_status(void* stream) {
  cudaError_t e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "stream synchronize");
  unsigned v = 0, site = 0, zero = 0;
  if ((e = cudaMemcpyFromSymbol(&v, aria::g_status, sizeof(v))) != cudaSuccess)
    return cuda_fail(e, "read status word");
  if (v) {
    cudaMemcpyFromSymbol(&site, aria::g_wait_site, sizeof(site));
    cudaMemcpyToSymbol(aria::g_status, &zero, sizeof(zero));
    return fail(ARIA_ERR_TIMEOUT, "a bounded wait ran out in a kernel (site %u)", site);
  }
  return ARIA_OK;
}

#ifdef ARIA_TRACE
// trace builds only: copy the per-CTA phase stamps to host memory
ARIA_API int aria_trace_read(void* host, size_t bytes) {
  return static_cast<int>(cudaMemcpyFromSymbol(host, aria::g_trace, bytes));
}
ARIA_API int aria_trace_clear(void) {
  static long long zero[8192 * 24];
  g_trace_launches = 0;
  return static_cast<int>(cudaMemcpyToSymbol(aria::g_trace, zero, sizeof(zero)));
}
#endif

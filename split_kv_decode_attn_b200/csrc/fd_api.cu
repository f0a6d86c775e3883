// fd_api.cu — host side of libfd.so: argument checks, the split-count
// planner, TMA tensor-map encoding and kernel launches on the caller's
// stream.  See include/fd.h for the contract of every entry point.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>

#include "../../include/fd.h"
#include "fd_kernels.cuh"

namespace {

constexpr int kMaxSplits = 1024;
constexpr int kMaxDevices = 64;

// ---------------------------------------------------------------- planner

// Cost model of one call, in microseconds, used to pick the split count.
// It models device time: the constants were fitted to split-count sweeps
// measured on B200 from CUDA-graph replays (free of the host's launch work):
// 36 bf16 shapes (the CodeLlama-34B head shape at B = 1 and L = 512..128K,
// B = 2..40 at L = 2K..64K, G = 4, the varlen, paged and peaked workloads)
// and 12 fp8 shapes (B = 1, 4, 16 and the three workloads).  On a fresh
// sweep of 54 shapes the pick is the fastest measured split count or within
// 4.6 % of it; the mean regret is 0.7 %.
//
// A CTA streams its tokens at a rate of its own (the tile loop's latency,
// independent of the element type), unless the device's HBM bandwidth,
// shared by the CTAs in flight, is lower:
//   kHbmGBs            streaming rate of the whole device
//   kCtaTokPerUs       tokens per microsecond of one CTA
//   kCtaDeepTokPerUs   the same for a bf16 D = 128 grid of at most one CTA
//                      per SM, which runs the deeper ring
//   kCtaFp8TokPerUs    the same for an fp8 cache, two CTAs per SM
//   kCtaFp8DeepTokPerUs  an fp8 CTA alone on its SM (grid <= SMs), with eight
//                      consumer warps
//   kCtaPagedTokPerUs  alone on an SM when pages hold fewer than 64 tokens
//                      (one TMA box per page instead of one per tile) ...
//   kCtaPagedSharedTokPerUs  ... and two to an SM (bf16 or fp8)
//   kCtaFixedUs        per-CTA fixed cost within a wave
//   kCombineUs         device time added by a call with several splits (the
//                      combine kernel after its dependency) ...
//   kCombinePer32Us    ... plus this per 32 splits merged (one L2 round trip
//                      per batch of 32 partial rows)
struct PlanModel {
  static constexpr double kHbmGBs = 6500.0;
  static constexpr double kCtaTokPerUs = 90.0;
  static constexpr double kCtaDeepTokPerUs = 100.0;
  static constexpr double kCtaFp8TokPerUs = 100.0;
  static constexpr double kCtaFp8DeepTokPerUs = 180.0;
  static constexpr double kCtaPagedTokPerUs = 50.0;
  static constexpr double kCtaPagedSharedTokPerUs = 80.0;
  static constexpr double kCtaFixedUs = 0.3;
  static constexpr double kCombineUs = 1.0;
  static constexpr double kCombinePer32Us = 2.0;
};

// How a call cuts the history: T = ceil(max_len / 64) tiles into S = min(S
// requested, T) splits (1 when T = 0); split s covers the tiles
// [floor(s T / S), floor((s + 1) T / S)) of every sequence, so the splits
// differ by at most one tile and the largest has ceil(T / S).
struct Chunking {
  int tiles;      // T
  int splits;     // S, the effective split count
  int max_tiles;  // ceil(T / S)
};

Chunking chunking(int max_len, int num_splits) {
  const int T = max_len > 0 ? static_cast<int>((static_cast<long long>(max_len) + fd::kTile - 1) /
                                                fd::kTile)
                            : 0;
  const int S = T == 0 ? 1 : std::min(num_splits, T);
  return Chunking{T, S, T == 0 ? 0 : (T + S - 1) / S};
}

// Splits that hold tokens of a sequence of n tokens (the kernels' rule).
int split_parts(const Chunking& c, long long n) {
  const long long m = (n + fd::kTile - 1) / fd::kTile;
  if (m <= 0) return 0;
  const long long p = (m * c.splits + c.tiles - 1) / c.tiles;
  return static_cast<int>(std::min<long long>(p, c.splits));
}

// What the model needs to know of a problem besides its lengths.
struct PlanShape {
  int num_sms;
  int B;
  int Hkv;
  double token_bytes;  // K + V bytes of one token of one KV head
  bool small_pages;    // pages of fewer than 64 tokens
  bool deep_ring;      // D = 128: a grid of <= num_sms CTAs gets the deep ring
  bool fp8;            // fp8 E4M3 cache
};

// Time of one wave of k CTAs of `tokens` tokens each, in a grid of
// `grid` CTAs.  CTAs are spread over the SMs first one per SM, then two.
double wave_time_us(const PlanShape& ps, double tokens, double k, double grid) {
  const double hbm_tok = PlanModel::kHbmGBs * 1e3 / (k * ps.token_bytes);
  double own = PlanModel::kCtaTokPerUs;
  if (ps.small_pages)
    own = k <= ps.num_sms ? PlanModel::kCtaPagedTokPerUs : PlanModel::kCtaPagedSharedTokPerUs;
  else if (ps.fp8)
    own = ps.deep_ring && grid <= ps.num_sms ? PlanModel::kCtaFp8DeepTokPerUs
                                             : PlanModel::kCtaFp8TokPerUs;
  else if (ps.deep_ring && grid <= ps.num_sms) own = PlanModel::kCtaDeepTokPerUs;
  return tokens / std::min(hbm_tok, own) + PlanModel::kCtaFixedUs;
}

// Time of one call whose split kernel runs n_ctas non-empty CTAs over
// `tokens` KV-head tokens, the largest CTA holding max_cta of them.  The
// larger of two estimates: waves of CTAs of the mean size, and the largest
// CTA on its own (which decides the end when lengths differ).
double model_time_us(const PlanShape& ps, double n_ctas, double tokens, double max_cta,
                     int s_eff) {
  if (n_ctas <= 0) return PlanModel::kCtaFixedUs;
  const double slots = static_cast<double>(ps.num_sms) * fd::kCtasPerSm;
  const double grid = static_cast<double>(ps.B) * ps.Hkv * s_eff;
  const double mean = tokens / n_ctas;
  const double full_waves = std::floor(n_ctas / slots);
  const double rem = n_ctas - full_waves * slots;
  double waves = 0.0;
  if (full_waves > 0) waves += full_waves * wave_time_us(ps, mean, slots, grid);
  if (rem > 0) waves += wave_time_us(ps, mean, rem, grid);
  const double longest = wave_time_us(ps, max_cta, std::min(n_ctas, slots), grid);
  double t = std::max(waves, longest);
  if (s_eff > 1) t += PlanModel::kCombineUs + PlanModel::kCombinePer32Us * std::ceil(s_eff / 32.0);
  return t;
}

// The model for a batch whose sequences all hold max_len tokens.
double model_time_uniform(const PlanShape& ps, int B, int max_len, int S) {
  const Chunking c = chunking(max_len, S);
  const double units = static_cast<double>(B) * ps.Hkv;
  return model_time_us(ps, units * c.splits, units * max_len,
                       std::min<double>(static_cast<double>(c.max_tiles) * fd::kTile, max_len),
                       c.splits);
}

// The model for given per-sequence lengths (clamped to [0, max_len]).
double model_time_lengths(const PlanShape& ps, int B, int max_len, const int32_t* lens, int S) {
  const Chunking c = chunking(max_len, S);
  const double largest = static_cast<double>(c.max_tiles) * fd::kTile;
  double n_ctas = 0.0, tokens = 0.0, max_tok = 0.0;
  for (int b = 0; b < B; ++b) {
    const double n = std::min<double>(std::max<int32_t>(lens[b], 0), max_len);
    n_ctas += split_parts(c, static_cast<long long>(n));
    tokens += n;
    max_tok = std::max(max_tok, std::min(n, largest));
  }
  return model_time_us(ps, n_ctas * ps.Hkv, tokens * ps.Hkv, max_tok, c.splits);
}

bool is_pow2(int x) { return x > 0 && (x & (x - 1)) == 0; }

int ilog2(int x) {
  int r = 0;
  while ((1 << r) < x) ++r;
  return r;
}

fd_status check_shape(int B, int Hq, int Hkv, int D, int max_len, int block_size) {
  if (B < 1 || B > 65535 || Hq < 1 || Hkv < 1 || Hkv > 65535 || max_len < 0 || block_size < 0)
    return FD_ERR_INVALID_ARGUMENT;
  if (Hq % Hkv != 0) return FD_ERR_INVALID_ARGUMENT;
  if (D != 64 && D != 128) return FD_ERR_UNSUPPORTED;
  const int G = Hq / Hkv;
  if (G != 1 && G != 2 && G != 4 && G != 8 && G != 16) return FD_ERR_UNSUPPORTED;
  if (block_size != 0 && (!is_pow2(block_size) || block_size < 8 || block_size > 256))
    return FD_ERR_UNSUPPORTED;
  return FD_OK;
}

// --------------------------------------------------------- device queries

struct DeviceInfo {
  std::atomic<int> sms{0};
  std::atomic<int> sm100{-1};
};
DeviceInfo g_dev[kMaxDevices];

fd_status current_device(int* dev) {
  if (cudaGetDevice(dev) != cudaSuccess) return FD_ERR_CUDA;
  if (*dev < 0 || *dev >= kMaxDevices) return FD_ERR_CUDA;
  return FD_OK;
}

fd_status device_sms(int dev, int* sms) {
  int v = g_dev[dev].sms.load();
  if (v == 0) {
    if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
      return FD_ERR_CUDA;
    g_dev[dev].sms.store(v);
  }
  *sms = v;
  return FD_OK;
}

fd_status device_is_sm100(int dev) {
  int v = g_dev[dev].sm100.load();
  if (v < 0) {
    int major = 0, minor = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess)
      return FD_ERR_CUDA;
    v = (major == 10 && minor == 0) ? 1 : 0;
    g_dev[dev].sm100.store(v);
  }
  return v ? FD_OK : FD_ERR_UNSUPPORTED;
}

// Unique id of the calling thread's current CUDA context, or 0 when it cannot
// be read.  A device reset destroys the primary context; the next runtime
// call creates a new one, with a new id, in which the module is loaded again:
// device symbols may then sit at other addresses and function attributes are
// back at their defaults.  Per-device set-up is therefore keyed by this id.
unsigned long long current_context_id() {
  static PFN_cuCtxGetCurrent_v4000 get_current = nullptr;
  static PFN_cuCtxGetId_v12000 get_id = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q{};
    if (cudaGetDriverEntryPointByVersion("cuCtxGetCurrent", &p, 4000, cudaEnableDefault, &q) ==
            cudaSuccess && q == cudaDriverEntryPointSuccess)
      get_current = reinterpret_cast<PFN_cuCtxGetCurrent_v4000>(p);
    p = nullptr;
    if (cudaGetDriverEntryPointByVersion("cuCtxGetId", &p, 12000, cudaEnableDefault, &q) ==
            cudaSuccess && q == cudaDriverEntryPointSuccess)
      get_id = reinterpret_cast<PFN_cuCtxGetId_v12000>(p);
  });
  if (!get_current || !get_id) return 0;
  CUcontext ctx = nullptr;
  if (get_current(&ctx) != CUDA_SUCCESS || !ctx) return 0;
  unsigned long long id = 0;
  return get_id(ctx, &id) == CUDA_SUCCESS ? id : 0;
}

// ------------------------------------------------------------ tensor maps

PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
std::once_flag g_encode_once;

fd_status encoder(PFN_cuTensorMapEncodeTiled_v12000* fn) {
  std::call_once(g_encode_once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q{};
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000,
                                         cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  *fn = g_encode;
  return g_encode ? FD_OK : FD_ERR_CUDA;
}

// 5-D view {64 columns, head, row, column half, plane} of a bf16 cache, box
// {64, 1, box_rows, D/64, 1}: one copy brings both 64-column halves of
// box_rows rows of one KV head, landing as [half][row][64] with the 128-byte
// swizzle.  The strides place heads, rows and planes for each layout:
//   HND contiguous [B, Hkv, L, D]     HND paged [pages, Hkv, bs, D]
//   NHD contiguous [B, L, Hkv, D]     NHD paged [pages, bs, Hkv, D]
// A plane is a sequence (contiguous) or a page (paged).  Coordinates outside
// the view read zeros.
fd_status make_cache_map(CUtensorMap* tm, const void* base, int D, int Hkv, long long rows,
                         long long planes, int layout, int box_rows, bool fp8) {
  PFN_cuTensorMapEncodeTiled_v12000 enc;
  if (encoder(&enc) != FD_OK) return FD_ERR_CUDA;
  // An fp8 row of 128 entries is one 128-byte swizzle row; a bf16 row of D
  // entries is D/64 of them.
  const int elem = fp8 ? 1 : 2;
  const int inner = 128 / elem;
  const cuuint64_t row_bytes = static_cast<cuuint64_t>(D) * elem;
  const cuuint64_t head_stride =
      layout == FD_LAYOUT_HND ? static_cast<cuuint64_t>(rows) * row_bytes : row_bytes;
  const cuuint64_t row_stride =
      layout == FD_LAYOUT_HND ? row_bytes : static_cast<cuuint64_t>(Hkv) * row_bytes;
  const cuuint64_t plane_stride = static_cast<cuuint64_t>(Hkv) * rows * row_bytes;
  const int halves = static_cast<int>(row_bytes / 128);
  cuuint64_t dims[5] = {static_cast<cuuint64_t>(inner), static_cast<cuuint64_t>(Hkv),
                        static_cast<cuuint64_t>(rows), static_cast<cuuint64_t>(halves),
                        static_cast<cuuint64_t>(planes)};
  cuuint64_t strides[4] = {head_stride, row_stride, 128, plane_stride};
  cuuint32_t box[5] = {static_cast<cuuint32_t>(inner), 1, static_cast<cuuint32_t>(box_rows),
                       static_cast<cuuint32_t>(halves), 1};
  cuuint32_t estr[5] = {1, 1, 1, 1, 1};
  CUresult r = enc(tm, fp8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 5,
                   const_cast<void*>(base), dims,
                   strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                   CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? FD_OK : FD_ERR_CUDA;
}

// A tensor map depends only on its base address, shape, layout, box and
// device, so each host thread keeps the last few it encoded: a decode loop
// that reuses its cache buffers pays for the encoding once.
struct MapKey {
  const void* base;
  long long rows, planes;
  int D, Hkv, layout, box_rows, dev;
  bool fp8;
  bool operator==(const MapKey& o) const {
    return base == o.base && rows == o.rows && planes == o.planes && D == o.D && Hkv == o.Hkv &&
           layout == o.layout && box_rows == o.box_rows && dev == o.dev && fp8 == o.fp8;
  }
};

fd_status cached_cache_map(CUtensorMap* tm, const MapKey& key) {
  constexpr int kEntries = 16;
  struct Entry {
    MapKey key;
    CUtensorMap map;
    bool used;
  };
  thread_local Entry entries[kEntries] = {};
  thread_local int next = 0;
  for (int i = 0; i < kEntries; ++i) {
    if (entries[i].used && entries[i].key == key) {
      *tm = entries[i].map;
      return FD_OK;
    }
  }
  const fd_status st = make_cache_map(tm, key.base, key.D, key.Hkv, key.rows, key.planes,
                                      key.layout, key.box_rows, key.fp8);
  if (st != FD_OK) return st;
  entries[next] = Entry{key, *tm, true};
  next = (next + 1) % kEntries;
  return FD_OK;
}

// --------------------------------------------------------------- launches

// How a split CTA holds its SM (D = 128; D = 64 always shares):
//   kShared     two CTAs per SM: four consumer warps; bf16 3 stages (96 KB),
//               fp8 6 stages of 16 KB (96 KB)
//   kDeepLong   one CTA per SM (grid <= SMs), splits of more than 64 tiles:
//               eight consumer warps; bf16 4 stages (128 KB), fp8 8 (128 KB)
//   kDeepShort  one CTA per SM, splits of at most 64 tiles: eight consumer
//               warps; bf16 6 stages (192 KB), fp8 12 (192 KB)
// Measured on one B200 with the CodeLlama-34B heads at S = 16 (interleaved
// runs, eager us): bf16 6 stages against 4, 32K 22.55 vs 23.18, 64K 40.67 vs
// 41.53; but 128K 79.6 vs 77.8 and 256K 150.0 vs 149.3.  fp8 at S = 18 (one
// CTA per SM) against S = 32 (two per SM on most SMs): 32K 15.0 vs 15.55,
// 64K 24.1 vs 24.75, 128K 43.3 vs 45.4, 256K 79.9 vs 82.7.  The sparse
// decode (32 KB scan stages) keeps 4 stages at one CTA per SM.
enum Ring { kShared = 0, kDeepLong = 1, kDeepShort = 2 };
constexpr int kDeepShortMaxTiles = 64;

template <int D, bool FP8, int RING, bool SPARSE>
constexpr int split_stages() {
  if (FP8) return RING == kShared ? 6 : (RING == kDeepShort ? 12 : 8);
  if (D != 128) return 6;
  if (RING == kShared) return 3;
  return (RING == kDeepShort && !SPARSE) ? 6 : 4;
}

template <int RING>
constexpr int split_consumer_warps() {
  return RING == kShared ? fd::kConsumerWarps : fd::kWideConsumerWarps;
}

template <int D, int NB, int MODE, bool PAGED, bool FP8 = false, int RING = kShared,
          bool SPARSE = false>
fd_status launch_split(const CUtensorMap& tk, const CUtensorMap& tv, const CUtensorMap& tc,
                       const fd::SplitArgs& a, int n_splits, int Hkv, int B,
                       cudaStream_t stream) {
  constexpr int STAGES = split_stages<D, FP8, RING, SPARSE>();
  constexpr int CW = split_consumer_warps<RING>();
  using L = fd::SplitSmem<D, NB, STAGES, FP8, SPARSE, CW>;
  auto kern = fd::fd_split_kernel<D, NB, MODE, PAGED, STAGES, FP8, SPARSE, CW>;
  // The shared-memory opt-in belongs to the device's context; remember the
  // context in which each device got it (0: not yet, or the id is unknown).
  static std::atomic<unsigned long long> attr_ctx[kMaxDevices];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return FD_ERR_CUDA;
  const unsigned long long ctx = current_context_id();
  if (ctx == 0 || attr_ctx[dev].load() != ctx) {
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             L::kDynamicBytes) != cudaSuccess)
      return FD_ERR_CUDA;
    attr_ctx[dev].store(ctx);
  }
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(static_cast<unsigned>(n_splits), static_cast<unsigned>(Hkv),
                     static_cast<unsigned>(B));
  cfg.blockDim = dim3(fd::split_threads<CW>());
  cfg.dynamicSmemBytes = L::kDynamicBytes;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (cudaLaunchKernelEx(&cfg, kern, tk, tv, tc, a) != cudaSuccess) return FD_ERR_CUDA;
  return FD_OK;
}

// The fp8 split kernel on tcgen05 (D = 128, G in {2, 4, 8}, one CTA per SM).
template <bool PAGED, int STAGES, int G>
fd_status launch_split_tc(const CUtensorMap& tk, const CUtensorMap& tv, const fd::SplitArgs& a,
                          int n_splits, int Hkv, int B, cudaStream_t stream) {
  using L = fd::TcSmem<STAGES>;
  auto kern = fd::fd_split_tc_kernel<PAGED, STAGES, G>;
  static std::atomic<unsigned long long> attr_ctx[kMaxDevices];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return FD_ERR_CUDA;
  const unsigned long long ctx = current_context_id();
  if (ctx == 0 || attr_ctx[dev].load() != ctx) {
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             L::kDynamicBytes) != cudaSuccess)
      return FD_ERR_CUDA;
    attr_ctx[dev].store(ctx);
  }
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(static_cast<unsigned>(n_splits), static_cast<unsigned>(Hkv),
                     static_cast<unsigned>(B));
  cfg.blockDim = dim3(fd::kTcThreads);
  cfg.dynamicSmemBytes = L::kDynamicBytes;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (cudaLaunchKernelEx(&cfg, kern, tk, tv, a) != cudaSuccess) return FD_ERR_CUDA;
  return FD_OK;
}

template <int D>
fd_status launch_combine(const fd::SplitArgs& a, int B, cudaStream_t stream) {
  cudaLaunchConfig_t cfg{};
  const int rows = B * a.Hq;
  cfg.gridDim = dim3(static_cast<unsigned>((rows + fd::kCombineWarps - 1) / fd::kCombineWarps));
  cfg.blockDim = dim3(fd::kCombineWarps * 32);
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (cudaLaunchKernelEx(&cfg, fd::fd_combine_kernel<D>, a, B) != cudaSuccess) return FD_ERR_CUDA;
  return FD_OK;
}

// Launches the split kernel and, with several splits, the combine kernel.
// ring: how the CTAs hold their SMs (Ring; bf16, D = 128 only).
// sparse: the low-bit scan and top-delta selection run first (contiguous
// bf16 caches only).
template <int D, int NB, int MODE, bool PAGED, bool FP8 = false>
fd_status launch_call(const CUtensorMap& tk, const CUtensorMap& tv, const CUtensorMap& tc,
                      const fd::SplitArgs& a, int n_splits, int Hkv, int B, int ring,
                      bool sparse, cudaStream_t s) {
  fd_status r = FD_ERR_UNSUPPORTED;
  if constexpr (!PAGED && !FP8) {
    if (sparse) {
      if constexpr (D == 128) {
        r = ring != kShared
                ? launch_split<D, NB, MODE, PAGED, FP8, kDeepLong, true>(tk, tv, tc, a, n_splits, Hkv, B, s)
                : launch_split<D, NB, MODE, PAGED, FP8, kShared, true>(tk, tv, tc, a, n_splits, Hkv, B, s);
        if (r == FD_OK && n_splits > 1) r = launch_combine<D>(a, B, s);
      }
      return r;
    }
  }
  if (sparse) return FD_ERR_UNSUPPORTED;
  if constexpr (D == 128) {
    if (ring == kDeepShort)
      r = launch_split<D, NB, MODE, PAGED, FP8, kDeepShort>(tk, tv, tc, a, n_splits, Hkv, B, s);
    else if (ring == kDeepLong)
      r = launch_split<D, NB, MODE, PAGED, FP8, kDeepLong>(tk, tv, tc, a, n_splits, Hkv, B, s);
    else
      r = launch_split<D, NB, MODE, PAGED, FP8, kShared>(tk, tv, tc, a, n_splits, Hkv, B, s);
  } else {
    (void)ring;
    r = launch_split<D, NB, MODE, PAGED, FP8, kShared>(tk, tv, tc, a, n_splits, Hkv, B, s);
  }
  if (r == FD_OK && n_splits > 1) r = launch_combine<D>(a, B, s);
  return r;
}

// fp8 caches (D = 128).  mma.sync: codes converted to f16 in registers, f16
// contraction, bf16(p) residuals not needed.  tcgen05: the tcgen05 kernel
// where it applies (G in {2, 4, 8}, one CTA per SM).
template <bool PAGED>
fd_status dispatch_split_fp8(int G, const CUtensorMap& tk, const CUtensorMap& tv,
                             const fd::SplitArgs& a, int n_splits, int Hkv, int B, int ring,
                             bool tcgen05, cudaStream_t s) {
  if (tcgen05 && (G == 2 || G == 4 || G == 8) && ring != kShared) {
    // One CTA per SM: the tcgen05 kernel, with the rings of the mma.sync one.
    constexpr int kShort = split_stages<128, true, kDeepShort, false>();
    constexpr int kLong = split_stages<128, true, kDeepLong, false>();
    fd_status r;
    if (G == 8)
      r = ring == kDeepShort ? launch_split_tc<PAGED, kShort, 8>(tk, tv, a, n_splits, Hkv, B, s)
                             : launch_split_tc<PAGED, kLong, 8>(tk, tv, a, n_splits, Hkv, B, s);
    else if (G == 4)
      r = ring == kDeepShort ? launch_split_tc<PAGED, kShort, 4>(tk, tv, a, n_splits, Hkv, B, s)
                             : launch_split_tc<PAGED, kLong, 4>(tk, tv, a, n_splits, Hkv, B, s);
    else
      r = ring == kDeepShort ? launch_split_tc<PAGED, kShort, 2>(tk, tv, a, n_splits, Hkv, B, s)
                             : launch_split_tc<PAGED, kLong, 2>(tk, tv, a, n_splits, Hkv, B, s);
    if (r == FD_OK && n_splits > 1) r = launch_combine<128>(a, B, s);
    return r;
  }
  if (G <= 8)
    return launch_call<128, 1, fd::kHi, PAGED, true>(tk, tv, tk, a, n_splits, Hkv, B, ring,
                                                     false, s);
  return launch_call<128, 2, fd::kHi, PAGED, true>(tk, tv, tk, a, n_splits, Hkv, B, ring,
                                                   false, s);
}

template <int D, bool PAGED>
fd_status dispatch_split(int G, const CUtensorMap& tk, const CUtensorMap& tv,
                         const CUtensorMap& tc, const fd::SplitArgs& a, int n_splits, int Hkv,
                         int B, int ring, bool sparse, cudaStream_t s) {
  if (G <= 4)
    return launch_call<D, 1, fd::kDup, PAGED>(tk, tv, tc, a, n_splits, Hkv, B, ring, sparse, s);
  if (G == 8)
    return launch_call<D, 1, fd::kHiLo, PAGED>(tk, tv, tc, a, n_splits, Hkv, B, ring, sparse, s);
  return launch_call<D, 2, fd::kHiLo, PAGED>(tk, tv, tc, a, n_splits, Hkv, B, ring, sparse, s);
}

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

size_t round256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

// The split count with the lowest modelled time; a larger count must win by
// more than 2 % (fewer splits mean fewer partials to merge).  Counts beyond
// two CTAs per SM slot, from the batch's units alone, only add waves, so the
// search stops there.
template <class Model>
int pick_splits(int max_len, long long units, int slots, Model model) {
  const long long tiles = (static_cast<long long>(max_len) + fd::kTile - 1) / fd::kTile;
  if (tiles <= 1) return 1;
  const long long fill = (2LL * slots + units - 1) / std::max(units, 1LL);
  const int s_max = static_cast<int>(std::min<long long>(std::min<long long>(tiles, kMaxSplits),
                                                         std::max(fill, 1LL)));
  int best = 1;
  double best_t = model(1);
  for (int S = 2; S <= s_max; ++S) {
    const double t = model(S);
    if (t < best_t * 0.98) {
      best_t = t;
      best = S;
    }
  }
  return best;
}

// Tiles each split CTA of a contiguous cache pulls into L2 before it waits on
// the previous grid, one TMA prefetch per tile (the prefetch overlaps the
// previous call's combine and the launch between the calls).
// bf16: a quarter of the split's tiles, at least 2, with the tiles of the
// CTAs resident at once (one or two per SM) kept to 64 MB of the 126 MB L2.
// Swept on B200 over 2..16 tiles for the CodeLlama-34B heads at 16K..256K
// tokens and S = 16 (one CTA per SM) and 32 (two): the best depth grows with
// the split (16K: 4, 32K: 8, 64K and longer: 12..16 at S = 16; 2, 4, 6..8,
// 8 at S = 32), and a fixed 4 cost 0.9 us at 32K, 1.4 us at 64K and 2.8 us
// at 128K.
// fp8 (half the bytes per tile, twice the CTAs): half the split's tiles, at
// most 4, which the same sweep kept.
int prefetch_tiles(int max_tiles, long long grid, int sms, bool deep, bool fp8, int D) {
  if (fp8) return std::min(4, std::max(1, max_tiles / 2));
  const long long resident = std::min<long long>(grid, deep ? sms : 2LL * sms);
  const long long tile_bytes = 2LL * fd::kTile * D * 2;      // K + V tiles, bf16
  const long long cap = std::max<long long>(2, (64LL << 20) / (std::max(resident, 1LL) * tile_bytes));
  return static_cast<int>(std::min<long long>(std::min<long long>(max_tiles, std::max(2, max_tiles / 4)),
                                              std::min<long long>(cap, 16)));
}

// Inputs of the sparse decode (null for the dense one).
struct SparseArgs {
  const int8_t* k8;
  const float* k8_scale;
  uint8_t* kept;
  float delta;
};

// One decode call.  The result goes to `out` (bf16) or, for a partial over a
// shard of the history, to `out_f32` (fp32); exactly one of them is set.
fd_status decode_impl(const fd_problem* p, const void* q, const void* k_cache,
                      const void* v_cache, const int32_t* seqlens, const int32_t* block_table,
                      float scale, int num_splits, void* out, float* out_f32, float* lse,
                      void* workspace, size_t workspace_bytes, fd_stream_t stream,
                      const SparseArgs* sp = nullptr) {
  // ---- host-side checks: nothing is launched for an invalid call
  if (!p || !q || !k_cache || !v_cache || (!out == !out_f32)) return FD_ERR_INVALID_ARGUMENT;
  const fd_status st = check_shape(p->B, p->Hq, p->Hkv, p->D, p->max_len, p->block_size);
  if (st != FD_OK) return st;
  const bool paged = p->block_size != 0;
  if (paged != (block_table != nullptr)) return FD_ERR_INVALID_ARGUMENT;
  if (paged) {
    if (p->num_blocks < 1 || p->max_blocks_per_seq < 1) return FD_ERR_INVALID_ARGUMENT;
    if (static_cast<long long>(p->max_blocks_per_seq) * p->block_size < p->max_len)
      return FD_ERR_INVALID_ARGUMENT;
  }
  if (p->kv_layout != FD_LAYOUT_HND && p->kv_layout != FD_LAYOUT_NHD) return FD_ERR_INVALID_ARGUMENT;
  if (p->kv_dtype != FD_KV_BF16 && p->kv_dtype != FD_KV_FP8_E4M3) return FD_ERR_INVALID_ARGUMENT;
  if (p->fp8_mma != FD_FP8_MMA_SYNC && p->fp8_mma != FD_FP8_MMA_TCGEN05) return FD_ERR_INVALID_ARGUMENT;
  const bool fp8 = p->kv_dtype == FD_KV_FP8_E4M3;
  if (fp8) {
    if (p->D != 128) return FD_ERR_UNSUPPORTED;
    if (!std::isfinite(p->k_scale) || !(p->k_scale > 0.f) || !std::isfinite(p->v_scale) ||
        !(p->v_scale > 0.f))
      return FD_ERR_INVALID_ARGUMENT;
  }
  if (!std::isfinite(scale) || !(scale > 0.f)) return FD_ERR_INVALID_ARGUMENT;
  if (num_splits < 1 || num_splits > kMaxSplits) return FD_ERR_INVALID_ARGUMENT;
  if (!aligned(q, 16) || !aligned(k_cache, 16) || !aligned(v_cache, 16) || !aligned(out, 16) ||
      !aligned(out_f32, 16) ||
      !aligned(lse, 4) || !aligned(workspace, 16) || !aligned(seqlens, 4) ||
      !aligned(block_table, 4))
    return FD_ERR_INVALID_ARGUMENT;
  if (sp) {
    if (paged || fp8 || p->D != 128 || p->kv_layout != FD_LAYOUT_HND) return FD_ERR_UNSUPPORTED;
    if (!sp->k8 || !sp->k8_scale || !aligned(sp->k8, 16) || !aligned(sp->k8_scale, 4) ||
        std::isnan(sp->delta) || sp->delta < 0.f)
      return FD_ERR_INVALID_ARGUMENT;
    if (chunking(p->max_len, num_splits).max_tiles > fd::kMaxSparseTiles)
      return FD_ERR_INVALID_ARGUMENT;
  }

  const int B = p->B, Hq = p->Hq, Hkv = p->Hkv, D = p->D, G = Hq / Hkv;
  const Chunking chunks = chunking(p->max_len, num_splits);
  const int n_splits = chunks.splits;
  float* part_o = nullptr;
  float* part_lse = nullptr;
  if (n_splits > 1) {
    const size_t need = fd_workspace_bytes(B, Hq, D, n_splits);
    if (!workspace || workspace_bytes < need) return FD_ERR_WORKSPACE;
    const size_t rows = static_cast<size_t>(B) * Hq * n_splits;
    char* w = static_cast<char*>(workspace);
    part_o = reinterpret_cast<float*>(w);
    part_lse = reinterpret_cast<float*>(w + round256(rows * D * 4));
  }

  int dev = 0;
  if (current_device(&dev) != FD_OK) return FD_ERR_CUDA;
  const fd_status arch = device_is_sm100(dev);
  if (arch != FD_OK) return arch;

  // ---- tensor maps over the caches
  CUtensorMap tk, tv;
  const int layout = p->kv_layout;
  const long long rows = paged ? p->block_size : (p->max_len > 0 ? p->max_len : 1);
  const long long planes = paged ? p->num_blocks : B;
  const int box_rows = paged ? std::min(p->block_size, fd::kTile) : fd::kTile;
  if (cached_cache_map(&tk, MapKey{k_cache, rows, planes, D, Hkv, layout, box_rows, dev, fp8}) != FD_OK ||
      cached_cache_map(&tv, MapKey{v_cache, rows, planes, D, Hkv, layout, box_rows, dev, fp8}) != FD_OK)
    return FD_ERR_CUDA;
  // Sparse: the int8 key codes, read kScanTilesPerStage blocks per box (one
  // 128-byte row per token, as an fp8 cache).
  CUtensorMap tc{};
  if (sp && cached_cache_map(&tc, MapKey{sp->k8, rows, planes, D, Hkv, layout,
                                         fd::kScanTilesPerStage * fd::kTile, dev, true}) != FD_OK)
    return FD_ERR_CUDA;

  fd::SplitArgs a{};
  a.q = static_cast<const __nv_bfloat16*>(q);
  a.seqlens = seqlens;
  a.block_table = block_table;
  a.out = static_cast<__nv_bfloat16*>(out);
  a.out_f32 = out_f32;
  a.lse = lse;
  a.part_o = part_o;
  a.part_lse = part_lse;
  a.Hq = Hq;
  a.Hkv = Hkv;
  a.G = G;
  a.max_len = p->max_len;
  a.block_size = paged ? p->block_size : 0;
  a.log2_block_size = paged ? ilog2(p->block_size) : 0;
  a.log2_box_rows = ilog2(box_rows);
  a.max_blocks_per_seq = paged ? p->max_blocks_per_seq : 0;
  a.tiles = chunks.tiles;
  a.n_splits = n_splits;
  a.tile_q = chunks.tiles / n_splits;
  a.tile_r = chunks.tiles % n_splits;
  a.scale_log2 = scale * (fp8 ? p->k_scale : 1.f) * 1.4426950408889634074f;
  a.v_scale = fp8 ? p->v_scale : 1.f;
  a.scale = scale;
  if (sp) {
    a.k8 = sp->k8;
    a.k8_scale = sp->k8_scale;
    a.kept_out = sp->kept;
    a.n_blocks = (p->max_len + fd::kTile - 1) / fd::kTile;
    a.delta = sp->delta;
  }

  int sms = 0;
  if (device_sms(dev, &sms) != FD_OK) return FD_ERR_CUDA;
  const long long grid = static_cast<long long>(B) * Hkv * n_splits;
  const bool deep = grid <= sms;
  const int ring = !deep ? kShared : chunks.max_tiles <= kDeepShortMaxTiles ? kDeepShort : kDeepLong;
  a.prefetch_tiles = (paged || sp) ? 0 : prefetch_tiles(chunks.max_tiles, grid, sms, deep, fp8, D);

  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  fd_status r;
  const bool tcgen05 = p->fp8_mma == FD_FP8_MMA_TCGEN05;
  if (fp8)
    r = paged ? dispatch_split_fp8<true>(G, tk, tv, a, n_splits, Hkv, B, ring, tcgen05, s)
              : dispatch_split_fp8<false>(G, tk, tv, a, n_splits, Hkv, B, ring, tcgen05, s);
  else if (D == 128)
    r = paged ? dispatch_split<128, true>(G, tk, tv, tk, a, n_splits, Hkv, B, ring, false, s)
              : dispatch_split<128, false>(G, tk, tv, sp ? tc : tk, a, n_splits, Hkv, B, ring,
                                           sp != nullptr, s);
  else
    r = paged ? dispatch_split<64, true>(G, tk, tv, tk, a, n_splits, Hkv, B, ring, false, s)
              : dispatch_split<64, false>(G, tk, tv, tk, a, n_splits, Hkv, B, ring, false, s);
  return r;
}

// The planner over every input it uses.  elem_bytes: bytes of one cache
// element; seqlens: host lengths or null (every sequence holds max_len).
int plan_impl(int num_sms, int B, int Hkv, int D, int max_len, int block_size, int elem_bytes,
              const int32_t* seqlens) {
  // Two CTAs per slot from the batch alone: no split (this also bounds the
  // planning cost for large batches).
  if (static_cast<long long>(B) * Hkv >= 2LL * num_sms * fd::kCtasPerSm) return 1;
  const PlanShape ps{num_sms, B, Hkv, 2.0 * D * elem_bytes,
                     block_size > 0 && block_size < fd::kTile, D == 128, elem_bytes == 1};
  const long long units = static_cast<long long>(B) * Hkv;
  const int slots = num_sms * fd::kCtasPerSm;
  if (seqlens)
    return pick_splits(max_len, units, slots, [&](int S) {
      return model_time_lengths(ps, B, max_len, seqlens, S);
    });
  return pick_splits(max_len, units, slots,
                     [&](int S) { return model_time_uniform(ps, B, max_len, S); });
}

}  // namespace

extern "C" {

const char* fd_status_string(fd_status status) {
  switch (status) {
    case FD_OK: return "FD_OK";
    case FD_ERR_INVALID_ARGUMENT: return "FD_ERR_INVALID_ARGUMENT";
    case FD_ERR_UNSUPPORTED: return "FD_ERR_UNSUPPORTED";
    case FD_ERR_WORKSPACE: return "FD_ERR_WORKSPACE";
    case FD_ERR_CUDA: return "FD_ERR_CUDA";
    case FD_ERR_DEVICE_TIMEOUT: return "FD_ERR_DEVICE_TIMEOUT";
  }
  return "FD_ERR_UNKNOWN";
}

int fd_split_chunk(int max_len, int num_splits) {
  if (max_len < 0 || num_splits < 1 || num_splits > kMaxSplits) return FD_ERR_INVALID_ARGUMENT;
  return std::max(1, chunking(max_len, num_splits).max_tiles) * fd::kTile;
}

int fd_effective_splits(int max_len, int num_splits) {
  if (max_len < 0 || num_splits < 1 || num_splits > kMaxSplits) return FD_ERR_INVALID_ARGUMENT;
  return chunking(max_len, num_splits).splits;
}

int fd_plan_sm(int num_sms, int B, int Hq, int Hkv, int D, int max_len, int block_size) {
  if (num_sms < 1) return FD_ERR_INVALID_ARGUMENT;
  const fd_status st = check_shape(B, Hq, Hkv, D, max_len, block_size);
  if (st != FD_OK) return st;
  return plan_impl(num_sms, B, Hkv, D, max_len, block_size, 2, nullptr);
}

int fd_plan_seqlens(int num_sms, int B, int Hq, int Hkv, int D, int max_len, int block_size,
                    const int32_t* seqlens) {
  const fd_status st = check_shape(B, Hq, Hkv, D, max_len, block_size);
  if (st != FD_OK) return st;
  if (!seqlens) return FD_ERR_INVALID_ARGUMENT;
  if (num_sms < 1) {
    int dev = 0;
    if (current_device(&dev) != FD_OK || device_sms(dev, &num_sms) != FD_OK) return FD_ERR_CUDA;
  }
  return plan_impl(num_sms, B, Hkv, D, max_len, block_size, 2, seqlens);
}

int fd_plan_problem(int num_sms, const fd_problem* p, const int32_t* seqlens) {
  if (!p) return FD_ERR_INVALID_ARGUMENT;
  const fd_status st = check_shape(p->B, p->Hq, p->Hkv, p->D, p->max_len, p->block_size);
  if (st != FD_OK) return st;
  if (p->kv_dtype != FD_KV_BF16 && p->kv_dtype != FD_KV_FP8_E4M3) return FD_ERR_INVALID_ARGUMENT;
  if (p->kv_dtype == FD_KV_FP8_E4M3 && p->D != 128) return FD_ERR_UNSUPPORTED;
  if (num_sms < 1) {
    int dev = 0;
    if (current_device(&dev) != FD_OK || device_sms(dev, &num_sms) != FD_OK) return FD_ERR_CUDA;
  }
  return plan_impl(num_sms, p->B, p->Hkv, p->D, p->max_len, p->block_size,
                   p->kv_dtype == FD_KV_FP8_E4M3 ? 1 : 2, seqlens);
}

int fd_plan(int B, int Hq, int Hkv, int D, int max_len, int block_size) {
  const fd_status st = check_shape(B, Hq, Hkv, D, max_len, block_size);
  if (st != FD_OK) return st;
  int dev = 0, sms = 0;
  if (current_device(&dev) != FD_OK || device_sms(dev, &sms) != FD_OK) return FD_ERR_CUDA;
  return fd_plan_sm(sms, B, Hq, Hkv, D, max_len, block_size);
}

size_t fd_workspace_bytes(int B, int Hq, int D, int num_splits) {
  if (B < 1 || Hq < 1 || D < 1 || num_splits < 1 || num_splits > kMaxSplits) return 0;
  if (num_splits == 1) return 0;
  const size_t rows = static_cast<size_t>(B) * Hq * num_splits;
  return round256(rows * D * sizeof(float)) + round256(rows * sizeof(float));
}

fd_status fd_decode(const fd_problem* p, const void* q, const void* k_cache,
                    const void* v_cache, const int32_t* seqlens, const int32_t* block_table,
                    float scale, int num_splits, void* out, float* lse, void* workspace,
                    size_t workspace_bytes, fd_stream_t stream) {
  if (!out) return FD_ERR_INVALID_ARGUMENT;
  return decode_impl(p, q, k_cache, v_cache, seqlens, block_table, scale, num_splits, out,
                     nullptr, lse, workspace, workspace_bytes, stream);
}

fd_status fd_decode_partial(const fd_problem* p, const void* q, const void* k_cache,
                            const void* v_cache, const int32_t* seqlens,
                            const int32_t* block_table, float scale, int num_splits,
                            float* out_f32, float* lse, void* workspace, size_t workspace_bytes,
                            fd_stream_t stream) {
  if (!out_f32 || !lse) return FD_ERR_INVALID_ARGUMENT;
  return decode_impl(p, q, k_cache, v_cache, seqlens, block_table, scale, num_splits, nullptr,
                     out_f32, lse, workspace, workspace_bytes, stream);
}

fd_status fd_quantize_keys(const fd_problem* p, const void* k_cache, const int32_t* seqlens,
                           int8_t* k8, float* k8_scale, fd_stream_t stream) {
  if (!p || !k_cache || !k8 || !k8_scale) return FD_ERR_INVALID_ARGUMENT;
  const fd_status st = check_shape(p->B, p->Hq, p->Hkv, p->D, p->max_len, p->block_size);
  if (st != FD_OK) return st;
  if (p->block_size != 0 || p->kv_layout != FD_LAYOUT_HND || p->kv_dtype != FD_KV_BF16)
    return FD_ERR_UNSUPPORTED;
  if (!aligned(k_cache, 16) || !aligned(k8, 16) || !aligned(k8_scale, 4) || !aligned(seqlens, 4))
    return FD_ERR_INVALID_ARGUMENT;
  if (p->max_len == 0) return FD_OK;
  int dev = 0;
  if (current_device(&dev) != FD_OK) return FD_ERR_CUDA;
  const fd_status arch = device_is_sm100(dev);
  if (arch != FD_OK) return arch;
  const int n_blocks = (p->max_len + fd::kTile - 1) / fd::kTile;
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(static_cast<unsigned>(n_blocks), static_cast<unsigned>(p->Hkv),
                     static_cast<unsigned>(p->B));
  cfg.blockDim = dim3(128);
  cfg.stream = reinterpret_cast<cudaStream_t>(stream);
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  const __nv_bfloat16* k = static_cast<const __nv_bfloat16*>(k_cache);
  const cudaError_t e =
      p->D == 128 ? cudaLaunchKernelEx(&cfg, fd::fd_quantize_keys_kernel<128>, k, seqlens, p->Hkv,
                                       p->max_len, n_blocks, k8, k8_scale)
                  : cudaLaunchKernelEx(&cfg, fd::fd_quantize_keys_kernel<64>, k, seqlens, p->Hkv,
                                       p->max_len, n_blocks, k8, k8_scale);
  return e == cudaSuccess ? FD_OK : FD_ERR_CUDA;
}

fd_status fd_decode_sparse(const fd_problem* p, const void* q, const void* k_cache,
                           const void* v_cache, const int8_t* k8, const float* k8_scale,
                           const int32_t* seqlens, float scale, float delta, int num_splits,
                           void* out, float* lse, uint8_t* kept, void* workspace,
                           size_t workspace_bytes, fd_stream_t stream) {
  if (!out) return FD_ERR_INVALID_ARGUMENT;
  const SparseArgs sp{k8, k8_scale, kept, delta};
  return decode_impl(p, q, k_cache, v_cache, seqlens, nullptr, scale, num_splits, out, nullptr,
                     lse, workspace, workspace_bytes, stream, &sp);
}

fd_status fd_combine(int R, int B, int Hq, int D, const float* part_o, const float* part_lse,
                     void* out, float* lse, fd_stream_t stream) {
  const size_t rows = static_cast<size_t>(B > 0 ? B : 0) * static_cast<size_t>(Hq > 0 ? Hq : 0);
  return fd_combine_strided(R, B, Hq, D, part_o, rows * static_cast<size_t>(D > 0 ? D : 0),
                            part_lse, rows, out, lse, stream);
}

fd_status fd_combine_strided(int R, int B, int Hq, int D, const float* part_o, size_t o_stride,
                             const float* part_lse, size_t lse_stride, void* out, float* lse,
                             fd_stream_t stream) {
  if (R < 1 || R > kMaxSplits || B < 1 || Hq < 1 || !part_o || !part_lse || !out)
    return FD_ERR_INVALID_ARGUMENT;
  if (D != 64 && D != 128) return FD_ERR_UNSUPPORTED;
  if (!aligned(part_o, 16) || !aligned(part_lse, 4) || !aligned(out, 16) || !aligned(lse, 4))
    return FD_ERR_INVALID_ARGUMENT;
  const long long rows = static_cast<long long>(B) * Hq;
  if (rows > (1ll << 30)) return FD_ERR_INVALID_ARGUMENT;
  // Every part starts 16 bytes aligned and holds its rows; lse entries of a
  // part do not overlap the next part's.
  if (o_stride % 4 != 0 || o_stride < static_cast<size_t>(rows) * D ||
      lse_stride < static_cast<size_t>(rows))
    return FD_ERR_INVALID_ARGUMENT;
  int dev = 0;
  if (current_device(&dev) != FD_OK) return FD_ERR_CUDA;
  const fd_status arch = device_is_sm100(dev);
  if (arch != FD_OK) return arch;
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(static_cast<unsigned>((rows + fd::kCombineWarps - 1) / fd::kCombineWarps));
  cfg.blockDim = dim3(fd::kCombineWarps * 32);
  cfg.stream = reinterpret_cast<cudaStream_t>(stream);
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  __nv_bfloat16* o = static_cast<__nv_bfloat16*>(out);
  const int r = static_cast<int>(rows);
  const cudaError_t e = D == 128
      ? cudaLaunchKernelEx(&cfg, fd::fd_merge_kernel<128>, part_o, part_lse, R, r, o_stride,
                           lse_stride, o, lse)
      : cudaLaunchKernelEx(&cfg, fd::fd_merge_kernel<64>, part_o, part_lse, R, r, o_stride,
                           lse_stride, o, lse);
  return e == cudaSuccess ? FD_OK : FD_ERR_CUDA;
}

// Scratch of fd_decode_static_workspace: a file-scope device array, so that
// callers who cannot allocate device memory still get a workspace.
static __device__ __align__(256) unsigned char g_static_workspace[FD_STATIC_WORKSPACE_BYTES];

fd_status fd_decode_static_workspace(const fd_problem* p, const void* q, const void* k_cache,
                                     const void* v_cache, const int32_t* seqlens,
                                     const int32_t* block_table, float scale, int num_splits,
                                     void* out, float* lse, fd_stream_t stream) {
  // Host-side checks first: an oversized request launches nothing.
  if (!p || num_splits < 1 || num_splits > kMaxSplits) return FD_ERR_INVALID_ARGUMENT;
  const fd_status st = check_shape(p->B, p->Hq, p->Hkv, p->D, p->max_len, p->block_size);
  if (st != FD_OK) return st;
  const int n_splits = chunking(p->max_len, num_splits).splits;
  const size_t need = n_splits > 1 ? fd_workspace_bytes(p->B, p->Hq, p->D, n_splits) : 0;
  if (need > FD_STATIC_WORKSPACE_BYTES) return FD_ERR_WORKSPACE;

  // Set-up, once per device (and again after a device reset, which gives the
  // device a new context), with that device current: the host-side name of
  // the array is not a device address; ask the runtime for the real one.
  struct StaticSlot {
    std::mutex m;
    unsigned long long ctx = 0;
    void* ptr = nullptr;
  };
  static StaticSlot slots[kMaxDevices];
  int dev = 0;
  if (current_device(&dev) != FD_OK) return FD_ERR_CUDA;
  void* ws = nullptr;
  {
    StaticSlot& sl = slots[dev];
    std::lock_guard<std::mutex> lock(sl.m);
    const unsigned long long ctx = current_context_id();
    if (ctx != 0 && sl.ptr && sl.ctx == ctx) {
      ws = sl.ptr;
    } else {
      if (cudaGetSymbolAddress(&ws, g_static_workspace) != cudaSuccess || !ws)
        return FD_ERR_CUDA;
      sl.ptr = ws;
      sl.ctx = current_context_id();  // the lookup makes the context current if it was not
    }
  }
  return fd_decode(p, q, k_cache, v_cache, seqlens, block_table, scale, num_splits, out, lse, ws,
                   FD_STATIC_WORKSPACE_BYTES, stream);
}

fd_status fd_selftest_device_timeout(unsigned int limit_us, fd_stream_t stream) {
  if (limit_us == 0 || limit_us > 5000000u) return FD_ERR_INVALID_ARGUMENT;
  int dev = 0;
  if (current_device(&dev) != FD_OK) return FD_ERR_CUDA;
  fd::fd_wait_selftest_kernel<<<1, 32, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
      static_cast<unsigned long long>(limit_us) * 1000ull);
  return cudaGetLastError() == cudaSuccess ? FD_OK : FD_ERR_CUDA;
}

fd_status fd_check_device_error(fd_stream_t stream) {
  if (cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess)
    return FD_ERR_CUDA;
  unsigned int word = 0;
  if (cudaMemcpyFromSymbol(&word, fd::g_error_word, sizeof word) != cudaSuccess)
    return FD_ERR_CUDA;
  if (word) {
    const unsigned int zero = 0;
    if (cudaMemcpyToSymbol(fd::g_error_word, &zero, sizeof zero) != cudaSuccess)
      return FD_ERR_CUDA;
    return FD_ERR_DEVICE_TIMEOUT;
  }
  return FD_OK;
}

}  // extern "C"

// C-ABI entry points of libsfp8.so (declared in include/sfp8.h): argument
// validation, tile planning, TMA descriptor encoding and kernel launches.
// The kernels are in the .cuh files included below; this is the only
// translation unit of the library.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdint>
#include <cstring>
#include <algorithm>
#include <atomic>
#include <mutex>
#include <vector>

#include "sfp8.h"
#include "device_common.cuh"
#include "quantize_rowwise.cuh"
#include "quantize_tensorwise.cuh"
#include "sparse24_pack.cuh"
#include "prepare_weight24.cuh"
#include "sparse_linear.cuh"
#include "sparse_linear_pair.cuh"

namespace sfp8 {
namespace {

constexpr int kMaxDevices = 64;

struct DeviceInfo {
  bool probed = false;
  bool is_sm100 = false;
  int index = 0;
  int num_sms = 0;
  bool smem_attr_set[40] = {};   // (BN, KS, RA, FQ) instantiations
  int pair_clusters[4] = {};     // co-resident pairs of the pair kernel by (KS, WT) (0: unknown)
  int tw_blocks[12] = {};        // co-resident CTAs per SM of the tensor-wise quantiser (0: unknown)
  long long l2_bytes = 0;
};

std::mutex g_mutex;
DeviceInfo g_devices[kMaxDevices];

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
EncodeTiledFn g_encode = nullptr;

sfp8_status current_device(DeviceInfo** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return SFP8_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return SFP8_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_mutex);
  DeviceInfo& d = g_devices[dev];
  if (!d.probed) {
    int major = 0, minor = 0, sms = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
      return SFP8_ERR_CUDA;
    int l2 = 0;
    if (cudaDeviceGetAttribute(&l2, cudaDevAttrL2CacheSize, dev) != cudaSuccess) return SFP8_ERR_CUDA;
    d.is_sm100 = (major == 10 && minor == 0);
    d.index = dev;
    d.num_sms = sms;
    d.l2_bytes = l2;
    d.probed = true;
  }
  if (!d.is_sm100) return SFP8_ERR_ARCH;
  *out = &d;
  return SFP8_OK;
}

sfp8_status get_encoder(EncodeTiledFn* fn) {
  std::lock_guard<std::mutex> lock(g_mutex);
  if (g_encode == nullptr) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) !=
            cudaSuccess ||
        q != cudaDriverEntryPointSuccess || p == nullptr)
      return SFP8_ERR_CUDA;
    g_encode = reinterpret_cast<EncodeTiledFn>(p);
  }
  *fn = g_encode;
  return SFP8_OK;
}

inline bool aligned(const void* p, uintptr_t a) {
  return (reinterpret_cast<uintptr_t>(p) % a) == 0;
}

inline sfp8_status launch_status() {
  return cudaGetLastError() == cudaSuccess ? SFP8_OK : SFP8_ERR_CUDA;
}

inline int elem_size(sfp8_dtype t) {
  switch (t) {
    case SFP8_BF16:
    case SFP8_F16:
      return 2;
    case SFP8_F32:
      return 4;
    case SFP8_E4M3:
    case SFP8_E5M2:
      return 1;
  }
  return 0;
}

inline bool is_fp8(sfp8_dtype t) { return t == SFP8_E4M3 || t == SFP8_E5M2; }
inline bool is_wide(sfp8_dtype t) { return t == SFP8_BF16 || t == SFP8_F16 || t == SFP8_F32; }

// Launch with programmatic stream serialisation: the kernel may start while
// the previous grid on the stream finishes; it waits for it (griddepcontrol)
// before touching memory.
template <typename Kernel, typename... Args>
sfp8_status launch_dependent(Kernel kern, dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                             Args... args) {
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (cudaLaunchKernelEx(&cfg, kern, args...) != cudaSuccess) {
    cudaGetLastError();
    return SFP8_ERR_CUDA;
  }
  return SFP8_OK;
}

constexpr int kSmemLimit = 232448;                 // 227 KB: largest dynamic smem per CTA

// ------------------------------------------------------------------ quantise

// Row count from which the streaming quantiser is used (below it, a few
// register-tile blocks finish sooner).
constexpr int64_t kQuantStreamMinRows = 256;
constexpr int kQuantRingSlots = 24;         // <= kQuantMaxSlots
constexpr int kQuantSlotsPerConsumer = 1;   // consumers <= kQuantMaxConsumers

// q2 (a second copy of the codes) is honoured by the register-tile path
// only, which every caller that passes it reaches (fewer than 256 rows of at
// most 4096 vectors).
template <typename T, int kFmt>
sfp8_status launch_quantize(const void* x, int64_t rows, int64_t cols, int64_t ld, void* q,
                            float* scales, cudaStream_t st, void* q2 = nullptr) {
  const T* xp = static_cast<const T*>(x);
  uint8_t* qp = static_cast<uint8_t*>(q);
  if (q2 != nullptr && (rows >= kQuantStreamMinRows || cols / InputTraits<T>::kPerVec > 4096))
    return SFP8_ERR_UNSUPPORTED_SHAPE;   // not reached by the callers
  if (cols == 0) {
    const int64_t blocks = (rows + 255) / 256;
    return launch_dependent(quantize_empty_rows_kernel<kFmt>, dim3(static_cast<unsigned>(blocks)),
                            dim3(256), 0, st, rows, scales);
  }
  constexpr int P = InputTraits<T>::kPerVec;
  const int64_t nvec = cols / P;
  // Many rows of up to 16 KB: the streaming kernel (one CTA per SM, a ring
  // of row buffers filled by bulk copies; measured faster than the register
  // tiles up to 16 KB rows, slower beyond).
  const int64_t row_bytes = cols * static_cast<int64_t>(sizeof(T));
  if (rows >= kQuantStreamMinRows && row_bytes <= 16 * 1024) {
    DeviceInfo* dev = nullptr;
    sfp8_status s = current_device(&dev);
    if (s != SFP8_OK) return s;
    // Ring: up to 192 KB of rows in flight; every consumer warp owns
    // slots / consumers ring slots (a whole number).
    int slots = static_cast<int>((192 * 1024) / row_bytes);
    if (slots > kQuantRingSlots) slots = kQuantRingSlots;
    int consumers = slots / kQuantSlotsPerConsumer;
    if (consumers < 1) consumers = 1;
    slots = consumers * kQuantSlotsPerConsumer;
    const int smem = static_cast<int>(slots * row_bytes) + 1024;
    auto kern = quantize_rowwise_stream_kernel<T, kFmt>;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemLimit) !=
        cudaSuccess)
      return SFP8_ERR_CUDA;
    const int64_t grid = rows < dev->num_sms ? rows : dev->num_sms;
    return launch_dependent(kern, dim3(static_cast<unsigned>(grid)), dim3(kQuantThreads),
                            static_cast<size_t>(smem), st, xp, rows, cols, ld, qp, scales, slots,
                            consumers);
  }
  // Rows in registers.  Few rows (a decode step): as many threads per row as
  // the row has vectors (up to 512), so each thread converts one to eight
  // vectors and the call is short.  Many long rows: one warp per row up to
  // 512 vectors (16 per lane: 8 KB of bf16 in flight per warp), then 4 and
  // 16 warps per row (the 16-warp tile holds 8 vectors per thread: 16 would
  // not fit 512 threads' registers).
  auto launch = [&](auto kern, int tpr) {
    const int threads = tpr > 256 ? tpr : 256;
    const int64_t per_block = threads / tpr;
    const int64_t blocks = (rows + per_block - 1) / per_block;
    return launch_dependent(kern, dim3(static_cast<unsigned>(blocks)), dim3(threads), 0, st, xp,
                            rows, cols, ld, qp, scales, static_cast<uint8_t*>(q2));
  };
  if (rows < kQuantStreamMinRows) {
    if (nvec <= 32) return launch(quantize_rowwise_kernel<T, kFmt, 32, 1>, 32);
    if (nvec <= 128) return launch(quantize_rowwise_kernel<T, kFmt, 128, 1>, 128);
    if (nvec <= 512) return launch(quantize_rowwise_kernel<T, kFmt, 512, 1>, 512);
    if (nvec <= 1024) return launch(quantize_rowwise_kernel<T, kFmt, 512, 2>, 512);
    if (nvec <= 2048) return launch(quantize_rowwise_kernel<T, kFmt, 512, 4>, 512);
    if (nvec <= 4096) return launch(quantize_rowwise_kernel<T, kFmt, 512, 8>, 512);
  } else {
    if (nvec <= 32 * 4) return launch(quantize_rowwise_kernel<T, kFmt, 32, 4>, 32);
    if (nvec <= 32 * 16) return launch(quantize_rowwise_kernel<T, kFmt, 32, 16>, 32);
    if (nvec <= 128 * 16) return launch(quantize_rowwise_kernel<T, kFmt, 128, 16>, 128);
    if (nvec <= 512 * 8) return launch(quantize_rowwise_kernel<T, kFmt, 512, 8>, 512);
  }
  return launch_dependent(quantize_rowwise_long_kernel<T, kFmt>,
                          dim3(static_cast<unsigned>(rows)), dim3(1024), 0, st, xp, rows, cols,
                          ld, qp, scales);
}

template <typename T>
sfp8_status launch_quantize_fmt(const void* x, int64_t rows, int64_t cols, int64_t ld, void* q,
                                sfp8_dtype q_dtype, float* scales, cudaStream_t st,
                                void* q2 = nullptr) {
  if (q_dtype == SFP8_E4M3)
    return launch_quantize<T, SFP8_E4M3>(x, rows, cols, ld, q, scales, st, q2);
  return launch_quantize<T, SFP8_E5M2>(x, rows, cols, ld, q, scales, st, q2);
}

// ------------------------------------------------------------------ tensor-wise quantise

// Upper bound on co-resident CTAs per SM of the tensor-wise kernel (2048
// threads per SM / kTwThreads); sizes the partials of the reduction mode.
constexpr int kTwMaxBlocksPerSm = 2048 / kTwThreads;

size_t tensorwise_workspace_bytes(int num_sms, sfp8_amax_mode mode) {
  size_t b = kTwSyncWords * sizeof(unsigned int);
  if (mode == SFP8_AMAX_REDUCE) b += sizeof(float) * static_cast<size_t>(num_sms) * kTwMaxBlocksPerSm;
  return b;
}

template <typename T, int kFmt, bool kAtomic>
sfp8_status launch_tensorwise_cfg(DeviceInfo* dev, int slot, const void* x, int64_t numel,
                                  void* q, float* scale, void* workspace, cudaStream_t st) {
  auto kern = quantize_tensorwise_kernel<T, kFmt, kAtomic>;
  {
    std::lock_guard<std::mutex> lock(g_mutex);
    if (dev->tw_blocks[slot] == 0) {
      int per_sm = 0;
      if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kTwThreads, 0) !=
              cudaSuccess || per_sm < 1) {
        cudaGetLastError();
        return SFP8_ERR_CUDA;
      }
      dev->tw_blocks[slot] = per_sm < kTwMaxBlocksPerSm ? per_sm : kTwMaxBlocksPerSm;
    }
  }
  constexpr int P = InputTraits<T>::kPerVec;
  constexpr int64_t kTile = static_cast<int64_t>(kTwThreads) * kTwUnroll;
  const int64_t nvec = numel / P;
  const int64_t tiles = (nvec + kTile - 1) / kTile;
  const int64_t max_grid = static_cast<int64_t>(dev->tw_blocks[slot]) * dev->num_sms;
  int64_t grid = tiles < max_grid ? tiles : max_grid;
  if (grid < 1) grid = 1;
  const int64_t per_cta = tiles > 0 ? (tiles + grid - 1) / grid : 0;
  if (per_cta > 0) grid = (tiles + per_cta - 1) / per_cta;
  // Tiles per run that sweep 1 marks to stay in L2: half the L2 over all runs.
  const int64_t tile_bytes = kTile * 16;
  int64_t keep = dev->l2_bytes / 2 / (grid * tile_bytes);
  if (keep < 1) keep = 1;
  unsigned int* sync = static_cast<unsigned int*>(workspace);
  float* partials = reinterpret_cast<float*>(sync + kTwSyncWords);
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(static_cast<unsigned>(grid));
  cfg.blockDim = dim3(kTwThreads);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = st;
  // Cooperative: every CTA is resident at once (the kernel's grid barrier
  // needs that), or the launch fails.
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (cudaLaunchKernelEx(&cfg, kern, static_cast<const T*>(x), numel, static_cast<uint8_t*>(q),
                         scale, sync, partials, per_cta, keep) != cudaSuccess) {
    cudaGetLastError();
    return SFP8_ERR_CUDA;
  }
  return SFP8_OK;
}

template <typename T>
sfp8_status launch_tensorwise(DeviceInfo* dev, int dslot, const void* x, int64_t numel,
                              void* q, sfp8_dtype q_dtype, float* scale, sfp8_amax_mode mode,
                              void* workspace, cudaStream_t st) {
  const int slot = dslot * 4 + (q_dtype == SFP8_E5M2 ? 2 : 0) + (mode == SFP8_AMAX_ATOMIC ? 1 : 0);
  if (q_dtype == SFP8_E4M3) {
    if (mode == SFP8_AMAX_ATOMIC)
      return launch_tensorwise_cfg<T, SFP8_E4M3, true>(dev, slot, x, numel, q, scale, workspace, st);
    return launch_tensorwise_cfg<T, SFP8_E4M3, false>(dev, slot, x, numel, q, scale, workspace, st);
  }
  if (mode == SFP8_AMAX_ATOMIC)
    return launch_tensorwise_cfg<T, SFP8_E5M2, true>(dev, slot, x, numel, q, scale, workspace, st);
  return launch_tensorwise_cfg<T, SFP8_E5M2, false>(dev, slot, x, numel, q, scale, workspace, st);
}

// ------------------------------------------------------------------ linear plan

constexpr long long kResidentActMax = 96 * 1024;   // resident activation slice limit
constexpr int kPlanProducers = 4;                  // producer warps used

struct LinearPlan {
  int pair;             // 1: the CTA-pair kernel
  int wt;               // pair kernel: weight tiles (128 rows) per CTA
  int bn;
  int ks;               // k steps per pipeline stage
  int ra;               // 1: activation resident in shared memory (one token tile)
  int stages;
  int producers;
  int stage_bytes;
  int ra_bytes;
  int smem_bytes;
  int whole_tiles;      // 1: each CTA takes whole tiles; 0: stream-K
  int grid;
  int m_tiles;
  int k_steps;
  int units;            // stages per tile
  long long n_tiles;
  long long tiles;
  long long iters;
  size_t partial_bytes;
  size_t counter_bytes;
};

int choose_bn(int64_t m) {
  if (m <= 16) return 16;
  if (m <= 32) return 32;
  if (m <= 64) return 64;
  if (m <= 128) return 128;
  return 128;
}

// Producer warps for a ring of `stages` stages.  Producer w issues stages
// i = w (mod P) into ring slot i mod stages and waits on the slot's
// phase parity; with no more producers than slots, a producer is never two
// phases ahead of a slot, so the parity it waits on is unambiguous.
int producers_for(int stages) { return stages < kPlanProducers ? stages : kPlanProducers; }

// Token count from which the CTA-pair kernel is used; from
// kPairSmallMinTokens it is used when its tiles keep enough SMs busy.
constexpr int64_t kPairMinTokens = 512;
constexpr int64_t kPairSmallMinTokens = 64;
// k steps per pipeline stage of the CTA-pair kernel (when k allows).
constexpr int kPairStepsPerStage = 2;
// Weight tiles per CTA of the CTA-pair kernel (when there are enough tiles
// and k is long enough).
constexpr int kPairWeightTiles = 2;
constexpr int kPairTwoTileMinSteps = 64;   // k >= 8192

// A work split of the GEMM (an "algorithm"): everything else in a plan
// follows from it and the shape.
struct LinearChoice {
  int pair;    // 1: the CTA-pair kernel
  int bn;      // tokens per tile
  int ks;      // k steps per pipeline stage
  int wt;      // pair kernel: weight tiles per CTA (1 or 2); 1 otherwise
  int whole;   // one-CTA kernel: 1 whole tiles per CTA, 0 stream-K; 1 for pairs
  bool operator==(const LinearChoice& o) const {
    return pair == o.pair && bn == o.bn && ks == o.ks && wt == o.wt && whole == o.whole;
  }
};

// Pair tile width from the token count: the fewest tiles of at most
// kPairMaxTokens, split evenly (rounded up to the pair MMA's N granularity
// of 32).
int pair_bn_for(int64_t m) {
  const int64_t mt = (m + kPairMaxTokens - 1) / kPairMaxTokens;
  return static_cast<int>(((m + mt - 1) / mt + 31) / 32 * 32);
}

// The built-in rule.
LinearChoice default_choice(int64_t m, int64_t n, int64_t k, int num_sms) {
  LinearChoice c{};
  const int k_steps = static_cast<int>(k / kStepK);
  const long long n_tiles = (n + kTileN - 1) / kTileN;
  if (m >= kPairMinTokens) {
    c.pair = 1;
    c.bn = pair_bn_for(m);
    const int m_tiles = static_cast<int>((m + c.bn - 1) / c.bn);
    c.ks = (kPairStepsPerStage == 2 && k_steps % 2 == 0) ? 2 : 1;
    // Two weight tiles per CTA (512-row pair tiles) halve the activation
    // bytes per MMA, when that still leaves a tile for every pair.
    // The accumulators of a two-tile CTA are single-buffered (the epilogue
    // stalls the MMAs once per tile), so this pays off only for long k.
    const long long groups2 = (n_tiles + 3) / 4;
    c.wt = (kPairWeightTiles == 2 && k_steps >= kPairTwoTileMinSteps &&
            groups2 * m_tiles >= num_sms / 2) ? 2 : 1;
    c.whole = 1;
    return c;
  }
  // 64..511 tokens: CTA pairs when their tiles keep at least 60 % of the
  // pairs busy -- the widest token tile first (fewest re-reads of the
  // weight), and at each width two weight tiles per CTA before one (each
  // activation byte feeds twice the MMAs).  Measured in steady state: m=128,
  // 192 on pair tiles of one token tile 13.8 / 15.3 us against 16.9 / 23.5
  // us on the one-CTA kernel (k=4096, n=14336).
  if (m >= kPairSmallMinTokens) {
    const int bn0 = pair_bn_for(m);
    for (int bn = bn0; bn >= (bn0 < 128 ? bn0 : 128); bn -= 32) {
      for (int wt = 2; wt >= 1; --wt) {
        const long long pairs = ((n_tiles + 2 * wt - 1) / (2 * wt)) * ((m + bn - 1) / bn);
        if (pairs * 10 >= 6LL * (num_sms / 2)) {
          c.pair = 1;
          c.bn = bn;
          c.ks = (k_steps % 2 == 0) ? 2 : 1;
          c.wt = wt;
          c.whole = 1;
          return c;
        }
      }
    }
  }
  c.pair = 0;
  c.wt = 1;
  // Several k steps per stage (20-50 KB): the stages are consumed in order,
  // and fewer, larger copies keep more bytes in flight per SM than many
  // small ones (measured on B200: the feed rate per SM grows with the copy
  // size at a fixed shared-memory ring).
  auto ks_for = [&](int bn) {
    return (bn <= 32 && k_steps % 4 == 0) ? 4 : (bn <= 128 && k_steps % 2 == 0) ? 2 : 1;
  };
  // Whole tiles (no split-K fix-up) with the widest token tile that keeps
  // three quarters of the SMs busy: narrower tiles re-read the weight from L2
  // once per token tile, which costs less than idle SMs or a split.
  for (int bn = choose_bn(m); bn >= 16; bn /= 2) {
    const long long tiles = n_tiles * ((m + bn - 1) / bn);
    if (tiles * 4 >= 3LL * num_sms) {
      c.bn = bn;
      c.ks = ks_for(bn);
      c.whole = 1;
      return c;
    }
  }
  // Too few tiles even at 16 tokens: split the k range over the SMs when
  // each tile has enough of it (64 k steps or more; measured: m=16, n=4096,
  // k=14336 is fastest split, k=4096 on 32 whole tiles).
  c.bn = choose_bn(m);
  c.ks = ks_for(c.bn);
  c.whole = k_steps >= 64 ? 0 : 1;
  return c;
}

// The plan of a choice (any choice from linear_choices is valid).
LinearPlan plan_from_choice(int64_t m, int64_t n, int64_t k, int num_sms, const LinearChoice& c) {
  LinearPlan pl{};
  pl.bn = c.bn;
  pl.ks = c.ks;
  pl.m_tiles = static_cast<int>((m + pl.bn - 1) / pl.bn);
  pl.k_steps = static_cast<int>(k / kStepK);
  pl.units = pl.k_steps / pl.ks;
  pl.n_tiles = (n + kTileN - 1) / kTileN;
  if (c.pair) {
    pl.pair = 1;
    pl.wt = c.wt;
    pl.tiles = ((pl.n_tiles + 2 * pl.wt - 1) / (2 * pl.wt)) * pl.m_tiles;
    pl.iters = pl.tiles * pl.units;
    pl.whole_tiles = 1;
    pl.stage_bytes = pl.ks * (pl.wt * kWTileBytes + (pl.bn / 2) * kStepK);
    pl.stages = kSmemBudget / pl.stage_bytes;
    if (pl.stages > PairCfg<1, 1>::kMaxStages) pl.stages = PairCfg<1, 1>::kMaxStages;
    pl.producers = producers_for(pl.stages);
    pl.smem_bytes = pair_smem_bytes(pl.stages, pl.stage_bytes);
    // The grid (pairs) is set at launch from the co-resident cluster count.
    pl.grid = 2 * static_cast<int>(pl.tiles < num_sms / 2 ? pl.tiles : num_sms / 2);
    return pl;
  }
  pl.wt = 1;
  pl.tiles = pl.n_tiles * pl.m_tiles;
  pl.iters = pl.tiles * pl.units;
  pl.whole_tiles = c.whole;
  // One token tile: keep the CTA's whole activation slice in shared memory
  // (one copy) when it is small; every stage is then one weight copy.
  const long long a_slice = static_cast<long long>(pl.bn) * k;
  pl.ra = (pl.m_tiles == 1 && pl.bn <= 32 && a_slice <= kResidentActMax &&
           pl.k_steps <= 256) ? 1 : 0;
  pl.ra_bytes = pl.ra ? static_cast<int>(a_slice) : 0;
  pl.stage_bytes = pl.ks * kWTileBytes + (pl.ra ? 0 : pl.ks * pl.bn * kStepK);
  const int budget = kSmemBudget - pl.ra_bytes;
  pl.stages = budget / pl.stage_bytes;
  if (pl.stages > 16) pl.stages = 16;
  pl.producers = producers_for(pl.stages);
  pl.smem_bytes = linear_smem_bytes(pl.ra_bytes, pl.stages, pl.stage_bytes);
  if (pl.whole_tiles) {
    pl.grid = static_cast<int>(pl.tiles < num_sms ? pl.tiles : num_sms);
    pl.partial_bytes = 0;
    pl.counter_bytes = 0;
  } else {
    pl.grid = static_cast<int>(pl.iters < num_sms ? pl.iters : num_sms);
    if (pl.grid < 1) pl.grid = 1;
    pl.partial_bytes = static_cast<size_t>(pl.grid) * 2 * pl.bn * kTileN * sizeof(float);
    pl.partial_bytes = (pl.partial_bytes + 255) & ~static_cast<size_t>(255);
    pl.counter_bytes = static_cast<size_t>(pl.tiles) * 4 * sizeof(unsigned int);
  }
  return pl;
}

constexpr int kMaxLinearChoices = 64;

// Every work split offered for a shape: index 0 is the built-in rule, then
// (without repeats) the one-CTA kernel at each tile width up to about twice
// the token count, k steps per stage and whole-tile / stream-K split, and
// the CTA-pair kernel at tile widths up to the token count rounded up to 32
// (128..224 from 256 tokens), one or two k steps per stage, one or two
// weight tiles per CTA.
int linear_choices(int64_t m, int64_t n, int64_t k, int num_sms, LinearChoice* out) {
  int count = 0;
  auto add = [&](const LinearChoice& c) {
    for (int i = 0; i < count; ++i)
      if (out[i] == c) return;
    if (count < kMaxLinearChoices) out[count++] = c;
  };
  add(default_choice(m, n, k, num_sms));
  const int k_steps = static_cast<int>(k / kStepK);
  for (int bn : {16, 32, 64, 128}) {
    if (bn > 16 && bn >= 2 * m) continue;
    for (int ks : {1, 2, 4}) {
      if (k_steps % ks != 0 || (ks == 4 && bn > 32)) continue;
      for (int whole : {1, 0}) add(LinearChoice{0, bn, ks, 1, whole});
    }
  }
  {
    // CTA pairs at every token count: from 256 tokens the tile widths
    // 128..224; below, the widths up to the token count rounded up to 32
    const int m32 = static_cast<int>((m + 31) / 32 * 32);
    for (int bn : {pair_bn_for(m), 32, 64, 96, 128, 160, 192, 224}) {
      if (bn > kPairMaxTokens || bn > m32 || (m >= 256 && bn < 128)) continue;
      for (int ks : {1, 2}) {
        if (k_steps % ks != 0) continue;
        for (int wt : {1, 2}) add(LinearChoice{1, bn, ks, wt, 1});
      }
    }
  }
  return count;
}

// Shape-keyed choices set by sfp8_sparse_linear_set_algo, per device.
struct AlgoEntry {
  int64_t m, n, k;
  int algo;
  LinearChoice choice;
};
std::mutex g_algo_mutex;
std::vector<AlgoEntry> g_algo_table[kMaxDevices];
std::atomic<int> g_algo_entries{0};   // entries over all devices: 0 skips the lock

bool lookup_algo(int dev, int64_t m, int64_t n, int64_t k, AlgoEntry* e) {
  if (g_algo_entries.load(std::memory_order_acquire) == 0) return false;
  std::lock_guard<std::mutex> lock(g_algo_mutex);
  for (const AlgoEntry& a : g_algo_table[dev])
    if (a.m == m && a.n == n && a.k == k) {
      *e = a;
      return true;
    }
  return false;
}

// The plan used by sfp8_sparse_linear on device `dev`: the table's choice
// for this shape, else the built-in rule.
LinearPlan make_plan(int dev, int64_t m, int64_t n, int64_t k, int num_sms) {
  AlgoEntry e;
  if (dev >= 0 && dev < kMaxDevices && lookup_algo(dev, m, n, k, &e)) return plan_from_choice(m, n, k, num_sms, e.choice);
  return plan_from_choice(m, n, k, num_sms, default_choice(m, n, k, num_sms));
}

template <int BN, int KS, bool RA, bool FQ = false>
sfp8_status launch_linear_cfg(DeviceInfo* dev, const CUtensorMap& ta, const CUtensorMap& ty,
                              const LinearParams& prm, int smem_bytes, cudaStream_t st) {
  auto kern = sparse_linear_kernel<BN, KS, RA, FQ>;
  const int slot =
      FQ ? 32 + (KS == 1 ? 0 : KS == 2 ? 1 : 2)
         : ((BN == 16 ? 0 : BN == 32 ? 1 : BN == 64 ? 2 : BN == 128 ? 3 : 4) * 3 +
            (KS == 1 ? 0 : KS == 2 ? 1 : 2)) * 2 + (RA ? 1 : 0);
  {
    std::lock_guard<std::mutex> lock(g_mutex);
    if (!dev->smem_attr_set[slot]) {
      if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               kSmemLimit) != cudaSuccess)
        return SFP8_ERR_CUDA;
      dev->smem_attr_set[slot] = true;
    }
  }
  return launch_dependent(kern, dim3(prm.grid), dim3(linear_threads(FQ)), smem_bytes, st, ta, ty,
                          prm);
}

// Weight map for the pair kernel with two weight tiles per CTA: the packed
// buffer as (256 B, 40, k steps, tiles), so that a box (256, 40, KS, 2) is
// KS k steps of two consecutive tiles, landing as [tile][k step][10 KB].
sfp8_status encode_weight_4d(CUtensorMap* map, const void* packed, uint64_t n_tiles,
                             uint64_t k_steps, uint32_t box_steps) {
  EncodeTiledFn enc = nullptr;
  sfp8_status s = get_encoder(&enc);
  if (s != SFP8_OK) return s;
  cuuint64_t dims[4] = {256, kWTileBytes / 256, k_steps, n_tiles};
  cuuint64_t strides[3] = {256, kWTileBytes, k_steps * kWTileBytes};
  cuuint32_t box[4] = {256, kWTileBytes / 256, box_steps, 2};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 4, const_cast<void*>(packed), dims,
                   strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? SFP8_OK : SFP8_ERR_CUDA;
}

// Weight map for the pair kernel: the packed buffer as (256 B, 40, tiles x
// k steps) bytes, so that a box (256, 40, KS) is KS consecutive 10 KB packed
// tiles, landing in shared memory exactly as stored (no swizzle).
sfp8_status encode_weight_3d(CUtensorMap* map, const void* packed, uint64_t n_tiles,
                             uint64_t k_steps, uint32_t box_steps) {
  EncodeTiledFn enc = nullptr;
  sfp8_status s = get_encoder(&enc);
  if (s != SFP8_OK) return s;
  cuuint64_t dims[3] = {256, kWTileBytes / 256, n_tiles * k_steps};
  cuuint64_t strides[2] = {256, kWTileBytes};
  cuuint32_t box[3] = {256, kWTileBytes / 256, box_steps};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void*>(packed), dims,
                   strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? SFP8_OK : SFP8_ERR_CUDA;
}

// Activation map: dims (128 bytes of k, rows, k steps) with strides (k, 128),
// so that one box of (128, rows, steps) lands as [step][row][128 B] -- one
// 128B-swizzled BN x 128 B tile per k step, as the MMA reads it.
sfp8_status encode_act_3d(CUtensorMap* map, const void* base, uint64_t m, uint64_t k,
                          uint32_t box_rows, uint32_t box_steps) {
  EncodeTiledFn enc = nullptr;
  sfp8_status s = get_encoder(&enc);
  if (s != SFP8_OK) return s;
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(kStepK), m, k / kStepK};
  cuuint64_t strides[2] = {k, static_cast<cuuint64_t>(kStepK)};
  cuuint32_t box[3] = {static_cast<cuuint32_t>(kStepK), box_rows, box_steps};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void*>(base), dims, strides,
                   box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? SFP8_OK : SFP8_ERR_CUDA;
}


// Output map: y [m, n] bf16 row-major, box 128 columns x box_rows rows.
sfp8_status encode_y_2d(CUtensorMap* map, void* y, uint64_t m, uint64_t n, uint32_t box_rows) {
  EncodeTiledFn enc = nullptr;
  sfp8_status s = get_encoder(&enc);
  if (s != SFP8_OK) return s;
  cuuint64_t dims[2] = {n, m};
  cuuint64_t strides[1] = {n * 2};
  cuuint32_t box[2] = {static_cast<cuuint32_t>(kTileN), box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, y, dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                   CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? SFP8_OK : SFP8_ERR_CUDA;
}


// Whether x [m rows of ld_x elements, k used] shares bytes with a_q [m, k],
// s_a [m] or y [m, n] bf16 (host arithmetic on the addresses; sizes that do
// not fit are left to the size checks that follow).  The quantiser reads x
// while it writes a_q and s_a, and the fused GEMM reads x in every CTA while
// some CTAs already write.
bool outputs_overlap_input(const void* x, sfp8_dtype x_dtype, int64_t ld_x, int64_t m,
                                  int64_t k, const void* a_q, const void* s_a, const void* y,
                                  int64_t n) {
  const int64_t lim = int64_t(1) << 31;
  if (x == nullptr || m <= 0 || k <= 0 || m >= lim || k >= lim || n < 0 || n >= lim) return false;
  int64_t span = 0;
  if (__builtin_mul_overflow(m - 1, ld_x, &span) || __builtin_add_overflow(span, k, &span) ||
      __builtin_mul_overflow(span, static_cast<int64_t>(elem_size(x_dtype)), &span))
    return false;
  const uintptr_t xb = reinterpret_cast<uintptr_t>(x);
  const uintptr_t xe = xb + static_cast<uintptr_t>(span);
  auto hits = [&](const void* p, int64_t bytes) {
    if (p == nullptr || bytes <= 0) return false;
    const uintptr_t b = reinterpret_cast<uintptr_t>(p);
    return b < xe && xb < b + static_cast<uintptr_t>(bytes);
  };
  return hits(a_q, m * k) || hits(s_a, 4 * m) || hits(y, 2 * m * n);
}

// The activation that the one-call forward reads (for the overlap check).
struct XSpan {
  const void* x;
  sfp8_dtype dtype;
  int64_t ld;
};

// Validation shared by the sparse-linear entry points (everything except the
// workspace); on success fills *plan for the current device.  With `xs`
// (the one-call forward), outputs sharing bytes with x are refused too.
sfp8_status validate_linear(const void* a_q, sfp8_dtype a_dtype, const float* s_a, int64_t m,
                            const void* packed, sfp8_dtype w_dtype, const float* s_w, int64_t n,
                            int64_t k, const void* bias, const void* y, DeviceInfo** dev,
                            LinearPlan* plan, bool* empty, const XSpan* xs = nullptr) {
  *empty = false;
  if (!is_fp8(a_dtype) || !is_fp8(w_dtype)) return SFP8_ERR_UNSUPPORTED_DTYPE;
  if (m < 0 || n < 0 || k < 0) return SFP8_ERR_INVALID_ARG;
  if (k == 0 || k % kStepK != 0) return SFP8_ERR_UNSUPPORTED_SHAPE;
  if (m >= (int64_t(1) << 31) || n >= (int64_t(1) << 31) || k >= (int64_t(1) << 31))
    return SFP8_ERR_UNSUPPORTED_SHAPE;
  if (m == 0 || n == 0) {
    *empty = true;
    return SFP8_OK;
  }
  if (a_q == nullptr || s_a == nullptr || packed == nullptr || s_w == nullptr || y == nullptr)
    return SFP8_ERR_INVALID_ARG;
  if (!aligned(a_q, 16) || !aligned(packed, 16) || !aligned(s_a, 4) || !aligned(s_w, 4) ||
      !aligned(y, 2) || (bias != nullptr && !aligned(bias, 2)))
    return SFP8_ERR_MISALIGNED;
  if (xs != nullptr && outputs_overlap_input(xs->x, xs->dtype, xs->ld, m, k, a_q, s_a, y, n))
    return SFP8_ERR_INVALID_ARG;
  sfp8_status s = current_device(dev);
  if (s != SFP8_OK) return s;
  *plan = make_plan((*dev)->index, m, n, k, (*dev)->num_sms);
  return SFP8_OK;
}

// Token tiles per band of the pair kernel's tile order (pair_tile_coords):
// keep one operand resident in L2 while the other streams through once.  With
// half the L2 as the budget: an activation that fits is kept whole (one band:
// every weight group read once); else a weight that fits is kept (bands of one
// token tile: the activation read once); else bands of as many token tiles as
// fit, so the activation is read once and the weight once per band.
int pair_band(const DeviceInfo* dev, const LinearPlan& pl, int64_t m, int64_t n, int64_t k) {
  const long long budget = static_cast<long long>(dev->l2_bytes) / 2;
  const long long a_bytes = static_cast<long long>(m) * k;
  const long long w_bytes = static_cast<long long>(sfp8_compressed_bytes(n, k));
  if (a_bytes <= budget) return pl.m_tiles;
  if (w_bytes <= budget) return 1;
  const long long per_tile = static_cast<long long>(pl.bn) * k;
  long long band = budget / (per_tile > 0 ? per_tile : 1);
  if (band < 1) band = 1;
  if (band > pl.m_tiles) band = pl.m_tiles;
  return static_cast<int>(band);
}

// CTA-pair GEMM: both maps, the co-resident pair count (queried once per
// device), launch with programmatic stream serialisation.
template <int KS, int WT>
sfp8_status launch_pair_cfg(DeviceInfo* dev, const LinearPlan& pl, const void* a_q,
                            sfp8_dtype a_dtype, const float* s_a, int64_t m, const void* packed,
                            sfp8_dtype w_dtype, const float* s_w, int64_t n, int64_t k,
                            const void* bias, void* y, cudaStream_t st) {
  using Cfg = PairCfg<KS, WT>;
  auto kern = sparse_linear_pair_kernel<KS, WT>;
  constexpr int slot = (KS - 1) * 2 + (WT - 1);
  {
    std::lock_guard<std::mutex> lock(g_mutex);
    if (dev->pair_clusters[slot] == 0) {
      if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemLimit) !=
          cudaSuccess)
        return SFP8_ERR_CUDA;
      cudaLaunchConfig_t qc{};
      qc.gridDim = dim3(2 * (dev->num_sms / 2));
      qc.blockDim = dim3(Cfg::kThreads);
      qc.dynamicSmemBytes = kSmemLimit;
      cudaLaunchAttribute ca[1];
      ca[0].id = cudaLaunchAttributeClusterDimension;
      ca[0].val.clusterDim.x = 2;
      ca[0].val.clusterDim.y = 1;
      ca[0].val.clusterDim.z = 1;
      qc.attrs = ca;
      qc.numAttrs = 1;
      int clusters = 0;
      if (cudaOccupancyMaxActiveClusters(&clusters, kern, &qc) != cudaSuccess || clusters < 1) {
        cudaGetLastError();
        return SFP8_ERR_CUDA;
      }
      dev->pair_clusters[slot] = clusters;
    }
  }
  CUtensorMap tw2, tw, ta;
  sfp8_status s = encode_weight_3d(&tw, packed, static_cast<uint64_t>(pl.n_tiles),
                                   static_cast<uint64_t>(pl.k_steps), KS);
  if (s != SFP8_OK) return s;
  if (WT == 2) {
    s = encode_weight_4d(&tw2, packed, static_cast<uint64_t>(pl.n_tiles),
                         static_cast<uint64_t>(pl.k_steps), KS);
    if (s != SFP8_OK) return s;
  } else {
    tw2 = tw;
  }
  s = encode_act_3d(&ta, a_q, static_cast<uint64_t>(m), static_cast<uint64_t>(k),
                    static_cast<uint32_t>(pl.bn / 2), KS);
  if (s != SFP8_OK) return s;
  const long long max_pairs = dev->pair_clusters[slot];
  const int pairs = static_cast<int>(pl.tiles < max_pairs ? pl.tiles : max_pairs);
  PairParams prm{};
  prm.s_a = s_a;
  prm.s_w = s_w;
  prm.bias = static_cast<const __nv_bfloat16*>(bias);
  prm.y = static_cast<__nv_bfloat16*>(y);
  prm.m = static_cast<int>(m);
  prm.n = static_cast<int>(n);
  prm.k = static_cast<int>(k);
  prm.n_tiles = static_cast<int>(pl.n_tiles);
  prm.n_groups = static_cast<int>((pl.n_tiles + 2 * WT - 1) / (2 * WT));
  prm.bn = pl.bn;
  prm.m_tiles = pl.m_tiles;
  prm.k_steps = pl.k_steps;
  prm.units = pl.units;
  prm.tiles = static_cast<int>(pl.tiles);
  prm.band = pair_band(dev, pl, m, n, k);
  prm.pairs = pairs;
  prm.stages = pl.stages;
  prm.stage_bytes = pl.stage_bytes;
  prm.producers = pl.producers;
  prm.idesc = make_idesc_f8f6f4(w_dtype == SFP8_E5M2 ? 1u : 0u, a_dtype == SFP8_E5M2 ? 1u : 0u,
                                kPairTileN, static_cast<uint32_t>(pl.bn), true);
  return launch_dependent(kern, dim3(2 * pairs), dim3(Cfg::kThreads), pl.smem_bytes, st, tw2,
                          tw, ta, prm);
}

sfp8_status launch_pair(DeviceInfo* dev, const LinearPlan& pl, const void* a_q,
                        sfp8_dtype a_dtype, const float* s_a, int64_t m, const void* packed,
                        sfp8_dtype w_dtype, const float* s_w, int64_t n, int64_t k,
                        const void* bias, void* y, cudaStream_t st) {
  switch (pl.ks * 2 + pl.wt) {
    case 1 * 2 + 1:
      return launch_pair_cfg<1, 1>(dev, pl, a_q, a_dtype, s_a, m, packed, w_dtype, s_w, n, k,
                                   bias, y, st);
    case 1 * 2 + 2:
      return launch_pair_cfg<1, 2>(dev, pl, a_q, a_dtype, s_a, m, packed, w_dtype, s_w, n, k,
                                   bias, y, st);
    case 2 * 2 + 1:
      return launch_pair_cfg<2, 1>(dev, pl, a_q, a_dtype, s_a, m, packed, w_dtype, s_w, n, k,
                                   bias, y, st);
    case 2 * 2 + 2:
      return launch_pair_cfg<2, 2>(dev, pl, a_q, a_dtype, s_a, m, packed, w_dtype, s_w, n, k,
                                   bias, y, st);
    default:
      return SFP8_ERR_UNSUPPORTED_SHAPE;   // no such plan is made
  }
}

// The activation quantisation of a fused launch (the GEMM quantises x itself).
struct FusedQuant {
  const void* x;
  sfp8_dtype x_dtype;
  int64_t ld_x;
  void* a_q;      // written
  float* s_a;     // written
};

// Whether the GEMM of a plan can quantise the activation itself: one CTA
// kernel with the activation resident in one 16-token tile.
bool fusable(const LinearPlan& pl, int64_t m) {
  return !pl.pair && pl.ra && pl.bn == kFusedMaxTokens && pl.m_tiles == 1 &&
         m <= kFusedMaxTokens;
}

// Encodes the activation map and launches the GEMM for a validated plan
// (with `fq`, a fusable plan: the GEMM quantises x into a_q itself).
sfp8_status launch_linear(DeviceInfo* dev, const LinearPlan& pl, const void* a_q,
                          sfp8_dtype a_dtype, const float* s_a, int64_t m, const void* packed,
                          sfp8_dtype w_dtype, const float* s_w, int64_t n, int64_t k,
                          const void* bias, void* y, float* partials, unsigned int* counters,
                          cudaStream_t st, const void* a_map = nullptr, int64_t a_map_rows = 0,
                          const FusedQuant* fq = nullptr) {
  if (pl.pair)
    return launch_pair(dev, pl, a_q, a_dtype, s_a, m, packed, w_dtype, s_w, n, k, bias, y, st);
  // The activation map reads a_q's m rows, or a_map_rows rows of a_map (a
  // copy padded to the token tile: whole rows instead of out-of-range fill).
  // A fused launch loads no codes and gets no map.
  CUtensorMap ta;
  std::memset(&ta, 0, sizeof(ta));
  sfp8_status s = SFP8_OK;
  if (fq == nullptr) {
    s = encode_act_3d(&ta, a_map != nullptr ? a_map : a_q,
                      static_cast<uint64_t>(a_map != nullptr ? a_map_rows : m),
                      static_cast<uint64_t>(k), static_cast<uint32_t>(pl.bn),
                      static_cast<uint32_t>(pl.ra ? pl.k_steps : pl.ks));
    if (s != SFP8_OK) return s;
  }
  LinearParams prm{};
  prm.packed = static_cast<const uint8_t*>(packed);
  prm.s_a = s_a;
  prm.s_w = s_w;
  prm.bias = static_cast<const __nv_bfloat16*>(bias);
  prm.y = static_cast<__nv_bfloat16*>(y);
  prm.partials = partials;
  prm.counters = counters;
  prm.m = static_cast<int>(m);
  prm.n = static_cast<int>(n);
  prm.k = static_cast<int>(k);
  prm.m_tiles = pl.m_tiles;
  prm.k_steps = pl.k_steps;
  prm.units = pl.units;
  prm.tiles = pl.tiles;
  prm.iters = pl.iters;
  prm.grid = pl.grid;
  prm.whole_tiles = pl.whole_tiles;
  prm.stages = pl.stages;
  prm.ra_bytes = pl.ra_bytes;
  prm.producers = pl.producers;
  // MMA A operand = weight, B operand = activation.
  prm.idesc = make_idesc_f8f6f4(w_dtype == SFP8_E5M2 ? 1u : 0u, a_dtype == SFP8_E5M2 ? 1u : 0u,
                                kTileN, static_cast<uint32_t>(pl.bn), true);
  // y through one TMA store per CTA when each CTA takes one whole tile and
  // the resident activation's region can stage it (rows of y 16-byte
  // aligned); otherwise plain stores.  The unused map is a copy of ta.
  CUtensorMap ty = ta;
  prm.tma_store = 0;
  if (pl.ra && pl.whole_tiles && pl.tiles <= pl.grid && n % 8 == 0 && aligned(y, 16) &&
      static_cast<long long>(pl.bn) * kTileN * 2 <= pl.ra_bytes) {
    s = encode_y_2d(&ty, y, static_cast<uint64_t>(m), static_cast<uint64_t>(n),
                    static_cast<uint32_t>(pl.bn));
    if (s != SFP8_OK) return s;
    prm.tma_store = 1;
  }
  const int sm = pl.smem_bytes;
  if (fq != nullptr) {
    if (!fusable(pl, m)) return SFP8_ERR_UNSUPPORTED_SHAPE;
    prm.x = fq->x;
    prm.ld_x = fq->ld_x;
    prm.x_dtype = fq->x_dtype;
    prm.a_fmt = a_dtype;
    prm.a_q_out = static_cast<uint8_t*>(fq->a_q);
    prm.s_a_out = fq->s_a;
    switch (pl.ks) {
      case 1: return launch_linear_cfg<16, 1, true, true>(dev, ta, ty, prm, sm, st);
      case 2: return launch_linear_cfg<16, 2, true, true>(dev, ta, ty, prm, sm, st);
      case 4: return launch_linear_cfg<16, 4, true, true>(dev, ta, ty, prm, sm, st);
      default: return SFP8_ERR_UNSUPPORTED_SHAPE;   // no such plan is made
    }
  }
  if (pl.ra) {
    switch (pl.bn * 8 + pl.ks) {
      case 16 * 8 + 1: return launch_linear_cfg<16, 1, true>(dev, ta, ty, prm, sm, st);
      case 16 * 8 + 2: return launch_linear_cfg<16, 2, true>(dev, ta, ty, prm, sm, st);
      case 16 * 8 + 4: return launch_linear_cfg<16, 4, true>(dev, ta, ty, prm, sm, st);
      case 32 * 8 + 1: return launch_linear_cfg<32, 1, true>(dev, ta, ty, prm, sm, st);
      case 32 * 8 + 2: return launch_linear_cfg<32, 2, true>(dev, ta, ty, prm, sm, st);
      case 32 * 8 + 4: return launch_linear_cfg<32, 4, true>(dev, ta, ty, prm, sm, st);
      default: return SFP8_ERR_UNSUPPORTED_SHAPE;   // no such plan is made
    }
  }
  switch (pl.bn * 8 + pl.ks) {
    case 16 * 8 + 1: return launch_linear_cfg<16, 1, false>(dev, ta, ty, prm, sm, st);
    case 16 * 8 + 2: return launch_linear_cfg<16, 2, false>(dev, ta, ty, prm, sm, st);
    case 16 * 8 + 4: return launch_linear_cfg<16, 4, false>(dev, ta, ty, prm, sm, st);
    case 32 * 8 + 1: return launch_linear_cfg<32, 1, false>(dev, ta, ty, prm, sm, st);
    case 32 * 8 + 2: return launch_linear_cfg<32, 2, false>(dev, ta, ty, prm, sm, st);
    case 32 * 8 + 4: return launch_linear_cfg<32, 4, false>(dev, ta, ty, prm, sm, st);
    case 64 * 8 + 1: return launch_linear_cfg<64, 1, false>(dev, ta, ty, prm, sm, st);
    case 64 * 8 + 2: return launch_linear_cfg<64, 2, false>(dev, ta, ty, prm, sm, st);
    case 128 * 8 + 1: return launch_linear_cfg<128, 1, false>(dev, ta, ty, prm, sm, st);
    case 128 * 8 + 2: return launch_linear_cfg<128, 2, false>(dev, ta, ty, prm, sm, st);
    default: return SFP8_ERR_UNSUPPORTED_SHAPE;   // no such plan is made
  }
}

// Workspace of the one-call forward: the GEMM's split-K scratch, then --
// with the activation resident and fewer tokens than the tile -- a staging
// copy of the codes padded to the token tile (256-byte aligned), which the
// GEMM reads as whole rows (rows past m are never stored, whatever they hold).
size_t quant_workspace_need(const LinearPlan& pl, int64_t m, int64_t k, bool* pad,
                            size_t* pad_off) {
  size_t need = pl.partial_bytes + pl.counter_bytes;
  *pad = false;
  *pad_off = 0;
  if (!pl.pair && pl.ra && m < pl.bn) {
    *pad = true;
    *pad_off = (need + 255) & ~static_cast<size_t>(255);
    need = *pad_off + static_cast<size_t>(pl.bn) * static_cast<size_t>(k);
  }
  return need;
}

// sfp8_quantize_rowwise with an optional second copy of the codes (q2).
sfp8_status quantize_rowwise_impl(const void* x, sfp8_dtype x_dtype, int64_t rows, int64_t cols,
                                  int64_t ld_x, void* q, sfp8_dtype q_dtype, float* scales,
                                  void* stream, void* q2) {
  if (!is_wide(x_dtype) || !is_fp8(q_dtype)) return SFP8_ERR_UNSUPPORTED_DTYPE;
  if (rows < 0 || cols < 0 || ld_x < cols) return SFP8_ERR_INVALID_ARG;
  if (cols % 16 != 0) return SFP8_ERR_UNSUPPORTED_SHAPE;
  if (rows >= (int64_t(1) << 31) / 8) return SFP8_ERR_UNSUPPORTED_SHAPE;
  if (rows == 0) return SFP8_OK;
  if (scales == nullptr || (cols > 0 && (x == nullptr || q == nullptr)))
    return SFP8_ERR_INVALID_ARG;
  const int es = elem_size(x_dtype);
  if (cols > 0 && (!aligned(x, 16) || !aligned(q, 16) || (ld_x * es) % 16 != 0))
    return SFP8_ERR_MISALIGNED;
  if (!aligned(scales, 4) || (q2 != nullptr && !aligned(q2, 16))) return SFP8_ERR_MISALIGNED;
  DeviceInfo* dev = nullptr;
  sfp8_status s = current_device(&dev);
  if (s != SFP8_OK) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  switch (x_dtype) {
    case SFP8_BF16:
      return launch_quantize_fmt<__nv_bfloat16>(x, rows, cols, ld_x, q, q_dtype, scales, st, q2);
    case SFP8_F16:
      return launch_quantize_fmt<__half>(x, rows, cols, ld_x, q, q_dtype, scales, st, q2);
    default:
      return launch_quantize_fmt<float>(x, rows, cols, ld_x, q, q_dtype, scales, st, q2);
  }
}

}  // namespace
}  // namespace sfp8

namespace sfp8 {
namespace {

// Self-test of the failure path: one thread waits, with the bounded wait of
// every pipeline in this library, on an mbarrier that nothing arrives on.
// After kWaitLimitCycles the wait gives up, records SFP8_DEVICE_TIMEOUT in
// the status word and the kernel returns; nothing is left in flight.
__global__ void selftest_wait_timeout_kernel() {
  __shared__ __align__(8) uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(smem_u32(&bar), 1);
    abort_flag = 0;
    fence_barrier_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) mbar_wait(smem_u32(&bar), 0, &abort_flag);
}

}  // namespace
}  // namespace sfp8

using namespace sfp8;

extern "C" {

const char* sfp8_status_string(sfp8_status s) {
  switch (s) {
    case SFP8_OK: return "ok";
    case SFP8_ERR_INVALID_ARG: return "invalid argument";
    case SFP8_ERR_UNSUPPORTED_SHAPE: return "unsupported shape";
    case SFP8_ERR_MISALIGNED: return "misaligned pointer or stride";
    case SFP8_ERR_UNSUPPORTED_DTYPE: return "unsupported dtype";
    case SFP8_ERR_ARCH: return "current device is not sm_100";
    case SFP8_ERR_WORKSPACE: return "workspace missing or too small";
    case SFP8_ERR_CUDA: return "CUDA error";
    case SFP8_ERR_TIMEOUT: return "device-side wait timed out";
    case SFP8_ERR_DEVICE_CHECK: return "device-side check failed";
  }
  return "unknown status";
}

int sfp8_layout_version(void) { return SFP8_LAYOUT_VERSION; }

int64_t sfp8_padded_rows(int64_t n) {
  if (n < 0) return -1;
  return ((n + kTileN - 1) / kTileN) * kTileN;
}

size_t sfp8_compressed_bytes(int64_t n, int64_t k) {
  if (n < 0 || k < 0) return 0;
  return static_cast<size_t>(sfp8_padded_rows(n)) * static_cast<size_t>(k) * 5 / 8;
}

size_t sfp8_compressed_values_bytes(int64_t n, int64_t k) {
  if (n < 0 || k < 0) return 0;
  return static_cast<size_t>(sfp8_padded_rows(n)) * static_cast<size_t>(k) / 2;
}

size_t sfp8_compressed_meta_bytes(int64_t n, int64_t k) {
  if (n < 0 || k < 0) return 0;
  return static_cast<size_t>(sfp8_padded_rows(n)) * static_cast<size_t>(k) / 8;
}

sfp8_status sfp8_quantize_rowwise(const void* x, sfp8_dtype x_dtype, int64_t rows, int64_t cols,
                                  int64_t ld_x, void* q, sfp8_dtype q_dtype, float* scales,
                                  void* stream) {
  return quantize_rowwise_impl(x, x_dtype, rows, cols, ld_x, q, q_dtype, scales, stream, nullptr);
}

size_t sfp8_quantize_tensorwise_workspace_bytes(sfp8_amax_mode mode) {
  if (mode != SFP8_AMAX_REDUCE && mode != SFP8_AMAX_ATOMIC) return 0;
  int dev = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    return 0;
  return tensorwise_workspace_bytes(sms, mode);
}

sfp8_status sfp8_quantize_tensorwise(const void* x, sfp8_dtype x_dtype, int64_t numel, void* q,
                                     sfp8_dtype q_dtype, float* scale, sfp8_amax_mode mode,
                                     void* workspace, size_t workspace_bytes, void* stream) {
  if (!is_wide(x_dtype) || !is_fp8(q_dtype)) return SFP8_ERR_UNSUPPORTED_DTYPE;
  if (mode != SFP8_AMAX_REDUCE && mode != SFP8_AMAX_ATOMIC) return SFP8_ERR_INVALID_ARG;
  if (numel < 0) return SFP8_ERR_INVALID_ARG;
  if (numel >= (int64_t(1) << 40)) return SFP8_ERR_UNSUPPORTED_SHAPE;
  if (scale == nullptr || workspace == nullptr || (numel > 0 && (x == nullptr || q == nullptr)))
    return SFP8_ERR_INVALID_ARG;
  if ((numel > 0 && (!aligned(x, 16) || !aligned(q, 16))) || !aligned(scale, 4) ||
      !aligned(workspace, 16))
    return SFP8_ERR_MISALIGNED;
  DeviceInfo* dev = nullptr;
  sfp8_status s = current_device(&dev);
  if (s != SFP8_OK) return s;
  if (workspace_bytes < tensorwise_workspace_bytes(dev->num_sms, mode)) return SFP8_ERR_WORKSPACE;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  switch (x_dtype) {
    case SFP8_BF16:
      return launch_tensorwise<__nv_bfloat16>(dev, 0, x, numel, q, q_dtype, scale, mode, workspace, st);
    case SFP8_F16:
      return launch_tensorwise<__half>(dev, 1, x, numel, q, q_dtype, scale, mode, workspace, st);
    default:
      return launch_tensorwise<float>(dev, 2, x, numel, q, q_dtype, scale, mode, workspace, st);
  }
}

sfp8_status sfp8_prune_24(const void* w, sfp8_dtype dtype, int64_t rows, int64_t cols,
                          int64_t ld, void* out, void* stream) {
  if (!is_wide(dtype)) return SFP8_ERR_UNSUPPORTED_DTYPE;
  if (rows < 0 || cols < 0 || ld < cols) return SFP8_ERR_INVALID_ARG;
  if (cols % 16 != 0) return SFP8_ERR_UNSUPPORTED_SHAPE;
  if (rows == 0 || cols == 0) return SFP8_OK;
  if (w == nullptr || out == nullptr) return SFP8_ERR_INVALID_ARG;
  const int es = elem_size(dtype);
  if (!aligned(w, 16) || !aligned(out, 16) || (ld * es) % 16 != 0) return SFP8_ERR_MISALIGNED;
  if (w == out && ld != cols) return SFP8_ERR_INVALID_ARG;
  DeviceInfo* dev = nullptr;
  sfp8_status s = current_device(&dev);
  if (s != SFP8_OK) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int64_t vecs = rows * (cols * es / 16);
  int64_t blocks = (vecs + 255) / 256;
  const int64_t cap = static_cast<int64_t>(dev->num_sms) * 16;
  if (blocks > cap) blocks = cap;
  if (es == 2) {
    prune24_kernel<uint16_t><<<static_cast<unsigned>(blocks), 256, 0, st>>>(
        static_cast<const uint16_t*>(w), rows, cols, ld, static_cast<uint16_t*>(out));
  } else {
    prune24_kernel<uint32_t><<<static_cast<unsigned>(blocks), 256, 0, st>>>(
        static_cast<const uint32_t*>(w), rows, cols, ld, static_cast<uint32_t*>(out));
  }
  return launch_status();
}

sfp8_status sfp8_compress_24(const void* w_q, sfp8_dtype w_dtype, int64_t n, int64_t k,
                             void* packed, void* stream) {
  if (!is_fp8(w_dtype)) return SFP8_ERR_UNSUPPORTED_DTYPE;
  if (n < 0 || k < 0) return SFP8_ERR_INVALID_ARG;
  if (k % kStepK != 0 || k == 0) return SFP8_ERR_UNSUPPORTED_SHAPE;
  if (n == 0) return SFP8_OK;
  if (k / kStepK > 65535 || sfp8_padded_rows(n) / kTileN > 65535) return SFP8_ERR_UNSUPPORTED_SHAPE;
  if (w_q == nullptr || packed == nullptr) return SFP8_ERR_INVALID_ARG;
  if (!aligned(w_q, 16) || !aligned(packed, 16)) return SFP8_ERR_MISALIGNED;
  DeviceInfo* dev = nullptr;
  sfp8_status s = current_device(&dev);
  if (s != SFP8_OK) return s;
  dim3 grid(static_cast<unsigned>((k / kStepK + kCompressTiles - 1) / kCompressTiles),
            static_cast<unsigned>(sfp8_padded_rows(n) / kTileN));
  compress24_kernel<<<grid, 512, 0, static_cast<cudaStream_t>(stream)>>>(
      static_cast<const uint8_t*>(w_q), n, k, static_cast<uint8_t*>(packed));
  return launch_status();
}

extern "C++" {
namespace {

template <typename T>
sfp8_status launch_prepare(const void* w, int64_t n, int64_t k, int64_t ld, sfp8_dtype q_dtype,
                           void* packed, float* s_w, int sms, cudaStream_t st) {
  const int64_t n_pad = sfp8_padded_rows(n);
  auto kernel = q_dtype == SFP8_E4M3 ? prepare_weight24_kernel<T, SFP8_E4M3>
                                     : prepare_weight24_kernel<T, SFP8_E5M2>;
  // A grid-stride kernel: at most the co-resident blocks.  Rows longer than
  // one register segment are re-read in sweep 2, so their rows in flight
  // (one per warp) are also held to ~48 MB, well inside L2.
  int occ = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, kernel, 32 * kPrepWarps, 0) !=
          cudaSuccess || occ < 1)
    occ = 1;
  int64_t blocks = static_cast<int64_t>(occ) * sms;
  const int64_t row_bytes = k * static_cast<int64_t>(sizeof(T));
  if (row_bytes > 8192)
    blocks = std::min<int64_t>(blocks, std::max<int64_t>(sms, (48ll << 20) / (row_bytes * kPrepWarps)));
  blocks = std::min<int64_t>(blocks, n_pad / kPrepWarps);
  kernel<<<static_cast<unsigned>(blocks), 32 * kPrepWarps, 0, st>>>(
      static_cast<const T*>(w), n, k, ld, static_cast<uint8_t*>(packed), s_w, n_pad);
  return launch_status();
}

}  // namespace
}  // extern "C++"

sfp8_status sfp8_prepare_weight_24(const void* w, sfp8_dtype w_dtype, int64_t n, int64_t k,
                                   int64_t ld_w, sfp8_dtype q_dtype, void* packed, float* s_w,
                                   void* stream) {
  if (!is_fp8(q_dtype)) return SFP8_ERR_UNSUPPORTED_DTYPE;
  if (w_dtype != SFP8_BF16 && w_dtype != SFP8_F16 && w_dtype != SFP8_F32)
    return SFP8_ERR_UNSUPPORTED_DTYPE;
  if (n < 0 || k < 0 || ld_w < k) return SFP8_ERR_INVALID_ARG;
  if (k % kStepK != 0 || k == 0) return SFP8_ERR_UNSUPPORTED_SHAPE;
  if (n == 0) return SFP8_OK;
  if (w == nullptr || packed == nullptr || s_w == nullptr) return SFP8_ERR_INVALID_ARG;
  const int64_t esize = w_dtype == SFP8_F32 ? 4 : 2;
  if (!aligned(w, 16) || (ld_w * esize) % 16 != 0 || !aligned(packed, 16) || !aligned(s_w, 4))
    return SFP8_ERR_MISALIGNED;
  DeviceInfo* dev = nullptr;
  sfp8_status s = current_device(&dev);
  if (s != SFP8_OK) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  switch (w_dtype) {
    case SFP8_BF16:
      return launch_prepare<__nv_bfloat16>(w, n, k, ld_w, q_dtype, packed, s_w, dev->num_sms, st);
    case SFP8_F16:
      return launch_prepare<__half>(w, n, k, ld_w, q_dtype, packed, s_w, dev->num_sms, st);
    default:
      return launch_prepare<float>(w, n, k, ld_w, q_dtype, packed, s_w, dev->num_sms, st);
  }
}

sfp8_status sfp8_decompress_24(const void* packed, int64_t n, int64_t k, void* w_q,
                               void* stream) {
  if (n < 0 || k < 0) return SFP8_ERR_INVALID_ARG;
  if (k % kStepK != 0 || k == 0) return SFP8_ERR_UNSUPPORTED_SHAPE;
  if (n == 0) return SFP8_OK;
  if (k / kStepK > 65535 || sfp8_padded_rows(n) / kTileN > 65535) return SFP8_ERR_UNSUPPORTED_SHAPE;
  if (w_q == nullptr || packed == nullptr) return SFP8_ERR_INVALID_ARG;
  if (!aligned(w_q, 16) || !aligned(packed, 16)) return SFP8_ERR_MISALIGNED;
  DeviceInfo* dev = nullptr;
  sfp8_status s = current_device(&dev);
  if (s != SFP8_OK) return s;
  dim3 grid(static_cast<unsigned>(k / kStepK), static_cast<unsigned>(sfp8_padded_rows(n) / kTileN));
  decompress24_kernel<<<grid, 512, 0, static_cast<cudaStream_t>(stream)>>>(
      static_cast<const uint8_t*>(packed), n, k, static_cast<uint8_t*>(w_q));
  return launch_status();
}

size_t sfp8_sparse_linear_workspace_bytes(int64_t m, int64_t n, int64_t k) {
  if (m <= 0 || n <= 0 || k <= 0 || k % kStepK != 0) return 0;
  int dev = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    return 0;
  const LinearPlan pl = make_plan(dev, m, n, k, sms);
  return pl.partial_bytes + pl.counter_bytes;
}

sfp8_status sfp8_workspace_clear(void* workspace, size_t workspace_bytes, void* stream) {
  if (workspace_bytes == 0) return SFP8_OK;
  if (workspace == nullptr) return SFP8_ERR_INVALID_ARG;
  return cudaMemsetAsync(workspace, 0, workspace_bytes, static_cast<cudaStream_t>(stream)) ==
                 cudaSuccess
             ? SFP8_OK
             : SFP8_ERR_CUDA;
}

sfp8_status sfp8_sparse_linear(const void* a_q, sfp8_dtype a_dtype, const float* s_a, int64_t m,
                               const void* packed, sfp8_dtype w_dtype, const float* s_w,
                               int64_t n, int64_t k, const void* bias, void* y, void* workspace,
                               size_t workspace_bytes, void* stream) {
  DeviceInfo* dev = nullptr;
  LinearPlan pl{};
  bool empty = false;
  sfp8_status s = validate_linear(a_q, a_dtype, s_a, m, packed, w_dtype, s_w, n, k, bias, y,
                                  &dev, &pl, &empty);
  if (s != SFP8_OK || empty) return s;
  const size_t need = pl.partial_bytes + pl.counter_bytes;
  if (need > 0 && (workspace == nullptr || workspace_bytes < need)) return SFP8_ERR_WORKSPACE;
  if (workspace != nullptr && !aligned(workspace, 16)) return SFP8_ERR_MISALIGNED;
  float* partials = static_cast<float*>(workspace);
  unsigned int* counters = need > 0 ? reinterpret_cast<unsigned int*>(
                                          static_cast<uint8_t*>(workspace) + pl.partial_bytes)
                                    : nullptr;
  return launch_linear(dev, pl, a_q, a_dtype, s_a, m, packed, w_dtype, s_w, n, k, bias, y,
                       partials, counters, static_cast<cudaStream_t>(stream));
}

// ---- work-split selection ("algorithms")

// Shape check shared by the algorithm entry points (no pointers involved).
static bool algo_shape_ok(int64_t m, int64_t n, int64_t k) {
  return m > 0 && n > 0 && k > 0 && k % kStepK == 0 && m < (int64_t(1) << 31) &&
         n < (int64_t(1) << 31) && k < (int64_t(1) << 31);
}

int sfp8_sparse_linear_plan_count(int64_t m, int64_t n, int64_t k, int num_sms) {
  if (!algo_shape_ok(m, n, k) || num_sms < 2) return 0;
  LinearChoice ch[kMaxLinearChoices];
  return linear_choices(m, n, k, num_sms, ch);
}

sfp8_status sfp8_sparse_linear_plan_info(int64_t m, int64_t n, int64_t k, int num_sms, int algo,
                                         int64_t* info) {
  if (info == nullptr || !algo_shape_ok(m, n, k) || num_sms < 2) return SFP8_ERR_INVALID_ARG;
  LinearChoice ch[kMaxLinearChoices];
  const int count = linear_choices(m, n, k, num_sms, ch);
  if (algo < 0 || algo >= count) return SFP8_ERR_INVALID_ARG;
  const LinearPlan pl = plan_from_choice(m, n, k, num_sms, ch[algo]);
  const int64_t v[12] = {pl.pair, pl.bn, pl.ks, pl.wt, pl.whole_tiles, pl.ra, pl.stages,
                         pl.grid, pl.producers, pl.smem_bytes,
                         static_cast<int64_t>(pl.partial_bytes + pl.counter_bytes), pl.m_tiles};
  for (int i = 0; i < 12; ++i) info[i] = v[i];
  return SFP8_OK;
}

int sfp8_sparse_linear_algo_count(int64_t m, int64_t n, int64_t k) {
  if (!algo_shape_ok(m, n, k)) return 0;
  DeviceInfo* dev = nullptr;
  if (current_device(&dev) != SFP8_OK) return 0;
  LinearChoice ch[kMaxLinearChoices];
  return linear_choices(m, n, k, dev->num_sms, ch);
}

sfp8_status sfp8_sparse_linear_algo_info(int64_t m, int64_t n, int64_t k, int algo,
                                         int32_t* info) {
  if (info == nullptr || !algo_shape_ok(m, n, k)) return SFP8_ERR_INVALID_ARG;
  DeviceInfo* dev = nullptr;
  sfp8_status s = current_device(&dev);
  if (s != SFP8_OK) return s;
  LinearChoice ch[kMaxLinearChoices];
  const int count = linear_choices(m, n, k, dev->num_sms, ch);
  if (algo < 0 || algo >= count) return SFP8_ERR_INVALID_ARG;
  const LinearPlan pl = plan_from_choice(m, n, k, dev->num_sms, ch[algo]);
  info[0] = pl.pair;
  info[1] = pl.bn;
  info[2] = pl.ks;
  info[3] = pl.wt;
  info[4] = pl.whole_tiles;
  info[5] = pl.ra;
  info[6] = pl.stages;
  info[7] = pl.grid;
  return SFP8_OK;
}

size_t sfp8_sparse_linear_algo_workspace_bytes(int64_t m, int64_t n, int64_t k, int algo) {
  if (!algo_shape_ok(m, n, k)) return 0;
  DeviceInfo* dev = nullptr;
  if (current_device(&dev) != SFP8_OK) return 0;
  LinearChoice ch[kMaxLinearChoices];
  const int count = linear_choices(m, n, k, dev->num_sms, ch);
  if (algo < 0 || algo >= count) return 0;
  const LinearPlan pl = plan_from_choice(m, n, k, dev->num_sms, ch[algo]);
  return pl.partial_bytes + pl.counter_bytes;
}

size_t sfp8_sparse_linear_search_workspace_bytes(int64_t m, int64_t n, int64_t k) {
  if (!algo_shape_ok(m, n, k)) return 0;
  DeviceInfo* dev = nullptr;
  if (current_device(&dev) != SFP8_OK) return 0;
  LinearChoice ch[kMaxLinearChoices];
  const int count = linear_choices(m, n, k, dev->num_sms, ch);
  size_t most = 0;
  for (int i = 0; i < count; ++i) {
    const LinearPlan pl = plan_from_choice(m, n, k, dev->num_sms, ch[i]);
    most = std::max(most, pl.partial_bytes + pl.counter_bytes);
  }
  return most;
}

sfp8_status sfp8_sparse_linear_algo(const void* a_q, sfp8_dtype a_dtype, const float* s_a,
                                    int64_t m, const void* packed, sfp8_dtype w_dtype,
                                    const float* s_w, int64_t n, int64_t k, const void* bias,
                                    void* y, int algo, void* workspace, size_t workspace_bytes,
                                    void* stream) {
  DeviceInfo* dev = nullptr;
  LinearPlan pl{};
  bool empty = false;
  sfp8_status s = validate_linear(a_q, a_dtype, s_a, m, packed, w_dtype, s_w, n, k, bias, y,
                                  &dev, &pl, &empty);
  if (s != SFP8_OK || empty) return s;
  LinearChoice ch[kMaxLinearChoices];
  const int count = linear_choices(m, n, k, dev->num_sms, ch);
  if (algo < 0 || algo >= count) return SFP8_ERR_INVALID_ARG;
  pl = plan_from_choice(m, n, k, dev->num_sms, ch[algo]);
  const size_t need = pl.partial_bytes + pl.counter_bytes;
  if (need > 0 && (workspace == nullptr || workspace_bytes < need)) return SFP8_ERR_WORKSPACE;
  if (workspace != nullptr && !aligned(workspace, 16)) return SFP8_ERR_MISALIGNED;
  float* partials = static_cast<float*>(workspace);
  unsigned int* counters = need > 0 ? reinterpret_cast<unsigned int*>(
                                          static_cast<uint8_t*>(workspace) + pl.partial_bytes)
                                    : nullptr;
  return launch_linear(dev, pl, a_q, a_dtype, s_a, m, packed, w_dtype, s_w, n, k, bias, y,
                       partials, counters, static_cast<cudaStream_t>(stream));
}

sfp8_status sfp8_sparse_linear_set_algo(int64_t m, int64_t n, int64_t k, int algo) {
  if (!algo_shape_ok(m, n, k)) return SFP8_ERR_INVALID_ARG;
  DeviceInfo* dev = nullptr;
  sfp8_status s = current_device(&dev);
  if (s != SFP8_OK) return s;
  LinearChoice ch[kMaxLinearChoices];
  const int count = linear_choices(m, n, k, dev->num_sms, ch);
  if (algo >= count) return SFP8_ERR_INVALID_ARG;
  std::lock_guard<std::mutex> lock(g_algo_mutex);
  std::vector<AlgoEntry>& t = g_algo_table[dev->index];
  const size_t before = t.size();
  t.erase(std::remove_if(t.begin(), t.end(),
                         [&](const AlgoEntry& a) { return a.m == m && a.n == n && a.k == k; }),
          t.end());
  if (algo > 0) t.push_back(AlgoEntry{m, n, k, algo, ch[algo]});
  g_algo_entries.fetch_add(static_cast<int>(t.size()) - static_cast<int>(before),
                           std::memory_order_release);
  return SFP8_OK;
}

int sfp8_sparse_linear_get_algo(int64_t m, int64_t n, int64_t k) {
  int dev = 0;
  if (!algo_shape_ok(m, n, k) || cudaGetDevice(&dev) != cudaSuccess || dev < 0 ||
      dev >= kMaxDevices)
    return 0;
  AlgoEntry e;
  return lookup_algo(dev, m, n, k, &e) ? e.algo : 0;
}

sfp8_status sfp8_sparse_linear_search(const void* a_q, sfp8_dtype a_dtype, const float* s_a,
                                      int64_t m, const void* packed, sfp8_dtype w_dtype,
                                      const float* s_w, int64_t n, int64_t k, const void* bias,
                                      void* y, void* workspace, size_t workspace_bytes,
                                      void* flush, size_t flush_bytes, int reps,
                                      int* best_algo, float* times_us, int times_len,
                                      void* stream) {
  if (best_algo == nullptr || reps < 1 || reps > 64 || (flush == nullptr && flush_bytes > 0) ||
      (times_us == nullptr && times_len > 0) || times_len < 0)
    return SFP8_ERR_INVALID_ARG;
  DeviceInfo* dev = nullptr;
  LinearPlan pl{};
  bool empty = false;
  sfp8_status s = validate_linear(a_q, a_dtype, s_a, m, packed, w_dtype, s_w, n, k, bias, y,
                                  &dev, &pl, &empty);
  if (s != SFP8_OK) return s;
  if (empty) return SFP8_ERR_INVALID_ARG;
  LinearChoice ch[kMaxLinearChoices];
  const int count = linear_choices(m, n, k, dev->num_sms, ch);
  size_t need = 0;
  for (int i = 0; i < count; ++i) {
    const LinearPlan p = plan_from_choice(m, n, k, dev->num_sms, ch[i]);
    need = std::max(need, p.partial_bytes + p.counter_bytes);
  }
  if (need > 0 && (workspace == nullptr || workspace_bytes < need)) return SFP8_ERR_WORKSPACE;
  if (workspace != nullptr && !aligned(workspace, 16)) return SFP8_ERR_MISALIGNED;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  cudaEvent_t ev[128];
  int made = 0;
  for (; made < 2 * reps; ++made)
    if (cudaEventCreate(&ev[made]) != cudaSuccess) break;
  auto finish = [&](sfp8_status r) {
    for (int i = 0; i < made; ++i) cudaEventDestroy(ev[i]);
    if (r != SFP8_OK) cudaGetLastError();
    return r;
  };
  if (made < 2 * reps) return finish(SFP8_ERR_CUDA);
  int best = 0;
  float best_t = 0.0f;
  float ts[64];
  for (int a = 0; a < count; ++a) {
    const LinearPlan p = plan_from_choice(m, n, k, dev->num_sms, ch[a]);
    const size_t w = p.partial_bytes + p.counter_bytes;
    float* partials = static_cast<float*>(workspace);
    unsigned int* counters = w > 0 ? reinterpret_cast<unsigned int*>(
                                         static_cast<uint8_t*>(workspace) + p.partial_bytes)
                                   : nullptr;
    // counters must start at zero: another split's partials may lie there
    if (w > 0 && cudaMemsetAsync(workspace, 0, w, st) != cudaSuccess)
      return finish(SFP8_ERR_CUDA);
    s = launch_linear(dev, p, a_q, a_dtype, s_a, m, packed, w_dtype, s_w, n, k, bias, y,
                      partials, counters, st);   // warm-up
    if (s != SFP8_OK) return finish(s);
    for (int r = 0; r < reps; ++r) {
      if (flush_bytes > 0 && cudaMemsetAsync(flush, r & 0xff, flush_bytes, st) != cudaSuccess)
        return finish(SFP8_ERR_CUDA);
      if (cudaEventRecord(ev[2 * r], st) != cudaSuccess) return finish(SFP8_ERR_CUDA);
      s = launch_linear(dev, p, a_q, a_dtype, s_a, m, packed, w_dtype, s_w, n, k, bias, y,
                        partials, counters, st);
      if (s != SFP8_OK) return finish(s);
      if (cudaEventRecord(ev[2 * r + 1], st) != cudaSuccess) return finish(SFP8_ERR_CUDA);
    }
    if (cudaEventSynchronize(ev[2 * reps - 1]) != cudaSuccess) return finish(SFP8_ERR_CUDA);
    for (int r = 0; r < reps; ++r) {
      if (cudaEventElapsedTime(&ts[r], ev[2 * r], ev[2 * r + 1]) != cudaSuccess)
        return finish(SFP8_ERR_CUDA);
    }
    std::sort(ts, ts + reps);
    const float med = ts[reps / 2] * 1000.0f;
    if (a < times_len) times_us[a] = med;
    if (a == 0 || med < best_t) {
      best = a;
      best_t = med;
    }
  }
  *best_algo = best;
  return finish(SFP8_OK);
}

size_t sfp8_sparse_linear_quant_workspace_bytes(int64_t m, int64_t n, int64_t k) {
  if (m <= 0 || n <= 0 || k <= 0 || k % kStepK != 0) return 0;
  int dev = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    return 0;
  const LinearPlan pl = make_plan(dev, m, n, k, sms);
  bool pad = false;
  size_t pad_off = 0;
  return quant_workspace_need(pl, m, k, &pad, &pad_off);
}

// How the one-call forward runs the activation quantisation.
enum QuantMode { kQuantAuto = 0, kQuantFused = 1, kQuantChained = 2 };

// The built-in choice for a fusable plan: the chain.  Measured on B200
// (k = 4096, n = 14336, e4m3, graphs of 100 steps rotating 8 weight copies):
// fused 10.3 / 11.5 / 15.4 us per step at 1 / 4 / 16 tokens against 8.5 /
// 8.5 / 8.9 us chained.  No MMA of the fused kernel can start before its
// CTA has the amax of every row, i.e. two dependent passes over x (issued
// while the weight stream already fills the memory system) and up to 64 K
// conversions per CTA; the chain's small quantiser grid runs that critical
// path once, ahead of the GEMM's weight stream.
constexpr bool kFuseWhenPossible = false;

static sfp8_status quant_linear(const void* x, sfp8_dtype x_dtype, int64_t ld_x,
                                sfp8_dtype a_dtype,
                         void* a_q, float* s_a, int64_t m, const void* packed,
                         sfp8_dtype w_dtype, const float* s_w, int64_t n, int64_t k,
                         const void* bias, void* y, void* workspace, size_t workspace_bytes,
                         void* stream, QuantMode mode) {
  if (!is_wide(x_dtype)) return SFP8_ERR_UNSUPPORTED_DTYPE;
  if (ld_x < k) return SFP8_ERR_INVALID_ARG;
  DeviceInfo* dev = nullptr;
  LinearPlan pl{};
  bool empty = false;
  const XSpan xs{x, x_dtype, ld_x};
  sfp8_status s = validate_linear(a_q, a_dtype, s_a, m, packed, w_dtype, s_w, n, k, bias, y,
                                  &dev, &pl, &empty, &xs);
  if (s != SFP8_OK) return s;
  if (m > 0 && x == nullptr) return SFP8_ERR_INVALID_ARG;
  const int es = elem_size(x_dtype);
  if (m > 0 && (!aligned(x, 16) || (ld_x * es) % 16 != 0)) return SFP8_ERR_MISALIGNED;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (empty) {
    // n == 0 still quantises the activation; m == 0 does nothing
    if (m == 0) return SFP8_OK;
    return sfp8_quantize_rowwise(x, x_dtype, m, k, ld_x, a_q, a_dtype, s_a, stream);
  }
  const bool can_fuse = fusable(pl, m);
  if (mode == kQuantFused && !can_fuse) return SFP8_ERR_UNSUPPORTED_SHAPE;
  const bool fuse = mode == kQuantFused || (mode == kQuantAuto && can_fuse && kFuseWhenPossible);
  bool pad = false;
  size_t pad_off = 0;
  size_t need = quant_workspace_need(pl, m, k, &pad, &pad_off);
  if (fuse) {
    need = pl.partial_bytes + pl.counter_bytes;   // no staged copy of the codes
    pad = false;
  }
  if (need > 0 && (workspace == nullptr || workspace_bytes < need)) return SFP8_ERR_WORKSPACE;
  if (workspace != nullptr && !aligned(workspace, 16)) return SFP8_ERR_MISALIGNED;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  float* partials = reinterpret_cast<float*>(ws);
  unsigned int* counters = pl.counter_bytes > 0
                               ? reinterpret_cast<unsigned int*>(ws + pl.partial_bytes)
                               : nullptr;
  if (fuse) {
    const FusedQuant fq{x, x_dtype, ld_x, a_q, s_a};
    return launch_linear(dev, pl, a_q, a_dtype, s_a, m, packed, w_dtype, s_w, n, k, bias, y,
                         partials, counters, st, nullptr, 0, &fq);
  }
  uint8_t* staged = pad ? ws + pad_off : nullptr;
  s = quantize_rowwise_impl(x, x_dtype, m, k, ld_x, a_q, a_dtype, s_a, stream, staged);
  if (s != SFP8_OK) return s;
  return launch_linear(dev, pl, a_q, a_dtype, s_a, m, packed, w_dtype, s_w, n, k, bias, y,
                       partials, counters, st, staged, pad ? pl.bn : 0);
}

sfp8_status sfp8_sparse_linear_quant(const void* x, sfp8_dtype x_dtype, int64_t ld_x,
                                     sfp8_dtype a_dtype, void* a_q, float* s_a, int64_t m,
                                     const void* packed, sfp8_dtype w_dtype, const float* s_w,
                                     int64_t n, int64_t k, const void* bias, void* y,
                                     void* workspace, size_t workspace_bytes, void* stream) {
  return quant_linear(x, x_dtype, ld_x, a_dtype, a_q, s_a, m, packed, w_dtype, s_w, n, k, bias,
                      y, workspace, workspace_bytes, stream, kQuantAuto);
}

sfp8_status sfp8_sparse_linear_quant_fused(const void* x, sfp8_dtype x_dtype, int64_t ld_x,
                                           sfp8_dtype a_dtype, void* a_q, float* s_a, int64_t m,
                                           const void* packed, sfp8_dtype w_dtype,
                                           const float* s_w, int64_t n, int64_t k,
                                           const void* bias, void* y, void* workspace,
                                           size_t workspace_bytes, void* stream) {
  return quant_linear(x, x_dtype, ld_x, a_dtype, a_q, s_a, m, packed, w_dtype, s_w, n, k, bias,
                      y, workspace, workspace_bytes, stream, kQuantFused);
}

sfp8_status sfp8_sparse_linear_quant_chained(const void* x, sfp8_dtype x_dtype, int64_t ld_x,
                                             sfp8_dtype a_dtype, void* a_q, float* s_a,
                                             int64_t m, const void* packed, sfp8_dtype w_dtype,
                                             const float* s_w, int64_t n, int64_t k,
                                             const void* bias, void* y, void* workspace,
                                             size_t workspace_bytes, void* stream) {
  return quant_linear(x, x_dtype, ld_x, a_dtype, a_q, s_a, m, packed, w_dtype, s_w, n, k, bias,
                      y, workspace, workspace_bytes, stream, kQuantChained);
}

int sfp8_sparse_linear_quant_fusable(int64_t m, int64_t n, int64_t k) {
  if (m <= 0 || n <= 0 || k <= 0 || k % kStepK != 0) return 0;
  int dev = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    return 0;
  const LinearPlan pl = make_plan(dev, m, n, k, sms);
  return fusable(pl, m) ? 1 : 0;
}

sfp8_status sfp8_selftest_timeout(void* stream) {
  DeviceInfo* dev = nullptr;
  sfp8_status s = current_device(&dev);
  if (s != SFP8_OK) return s;
  selftest_wait_timeout_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>();
  return launch_status();
}

sfp8_status sfp8_sparse_linear_quant_host(const void* x_host, void* x_dev, sfp8_dtype x_dtype,
                                          sfp8_dtype a_dtype, void* a_q, float* s_a, int64_t m,
                                          const void* packed, sfp8_dtype w_dtype,
                                          const float* s_w, int64_t n, int64_t k,
                                          const void* bias, void* y_dev, void* y_host,
                                          void* workspace, size_t workspace_bytes,
                                          void* stream) {
  if (!is_wide(x_dtype)) return SFP8_ERR_UNSUPPORTED_DTYPE;
  DeviceInfo* dev = nullptr;
  LinearPlan pl{};
  bool empty = false;
  sfp8_status s = validate_linear(a_q, a_dtype, s_a, m, packed, w_dtype, s_w, n, k, bias, y_dev,
                                  &dev, &pl, &empty);
  if (s != SFP8_OK) return s;
  if (m == 0) return SFP8_OK;
  if (x_host == nullptr || x_dev == nullptr || (n > 0 && y_host == nullptr))
    return SFP8_ERR_INVALID_ARG;
  if (!aligned(x_dev, 16)) return SFP8_ERR_MISALIGNED;
  if (!empty) {
    bool pad = false;
    size_t pad_off = 0;
    const size_t need = quant_workspace_need(pl, m, k, &pad, &pad_off);
    if (need > 0 && (workspace == nullptr || workspace_bytes < need)) return SFP8_ERR_WORKSPACE;
    if (workspace != nullptr && !aligned(workspace, 16)) return SFP8_ERR_MISALIGNED;
  }
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const size_t x_bytes = static_cast<size_t>(m) * static_cast<size_t>(k) * elem_size(x_dtype);
  if (cudaMemcpyAsync(x_dev, x_host, x_bytes, cudaMemcpyHostToDevice, st) != cudaSuccess) {
    cudaGetLastError();
    return SFP8_ERR_CUDA;
  }
  s = sfp8_sparse_linear_quant(x_dev, x_dtype, k, a_dtype, a_q, s_a, m, packed, w_dtype, s_w, n,
                               k, bias, y_dev, workspace, workspace_bytes, stream);
  if (s != SFP8_OK || n == 0) return s;
  const size_t y_bytes = static_cast<size_t>(m) * static_cast<size_t>(n) * 2;
  if (cudaMemcpyAsync(y_host, y_dev, y_bytes, cudaMemcpyDeviceToHost, st) != cudaSuccess) {
    cudaGetLastError();
    return SFP8_ERR_CUDA;
  }
  return SFP8_OK;
}

sfp8_status sfp8_last_device_status(void) {
  uint32_t flags = 0;
  return sfp8_read_device_status(&flags, 0);
}

sfp8_status sfp8_read_device_status(uint32_t* flags, int clear) {
  if (flags == nullptr) return SFP8_ERR_INVALID_ARG;
  if (cudaDeviceSynchronize() != cudaSuccess) return SFP8_ERR_CUDA;
  unsigned int v = 0;
  if (cudaMemcpyFromSymbol(&v, g_device_status, sizeof(v)) != cudaSuccess) return SFP8_ERR_CUDA;
  if (clear) {
    const unsigned int zero = 0;
    if (cudaMemcpyToSymbol(g_device_status, &zero, sizeof(zero)) != cudaSuccess)
      return SFP8_ERR_CUDA;
  }
  *flags = v;
  if (v & SFP8_DEVICE_TIMEOUT) return SFP8_ERR_TIMEOUT;
  if (v & SFP8_DEVICE_CHECK_FAIL) return SFP8_ERR_DEVICE_CHECK;
  return SFP8_OK;
}

}  // extern "C"

// ---------------------------------------------------------------------------
// Sparse linear for callers that cannot allocate device memory.
//
// Some callers of this library run where no device allocation may happen at
// call time: code that is replayed inside a pre-built CUDA graph, allocators
// that forbid cudaMalloc after start-up, or hosts that hand the library only
// its inputs and outputs.  For them the split-K scratch (partial sums and
// per-tile counters) lives in a fixed buffer compiled into the library: one
// copy per device that loads it, kept until the process exits.
// ---------------------------------------------------------------------------

namespace {

constexpr size_t kNoAllocScratchBytes = SFP8_NOALLOC_SCRATCH_BYTES;

// In host code this name is only a stand-in; the device address is looked
// up once per device with cudaGetSymbolAddress.
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

std::mutex g_noalloc_mutex;
void* g_noalloc_ptr[sfp8::kMaxDevices] = {};

// Device address of the scratch buffer for the current device (set-up on
// the first call per device).
sfp8_status noalloc_scratch(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= sfp8::kMaxDevices)
    return SFP8_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_noalloc_mutex);
  if (g_noalloc_ptr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) {
      cudaGetLastError();
      return SFP8_ERR_CUDA;
    }
    g_noalloc_ptr[dev] = p;
  }
  *out = g_noalloc_ptr[dev];
  return SFP8_OK;
}

}  // namespace

extern "C" sfp8_status sfp8_sparse_linear_noalloc(const void* a_q, sfp8_dtype a_dtype,
                                                  const float* s_a, int64_t m,
                                                  const void* packed, sfp8_dtype w_dtype,
                                                  const float* s_w, int64_t n, int64_t k,
                                                  const void* bias, void* y, void* stream) {
  DeviceInfo* dev = nullptr;
  LinearPlan pl{};
  bool empty = false;
  sfp8_status s = validate_linear(a_q, a_dtype, s_a, m, packed, w_dtype, s_w, n, k, bias, y,
                                  &dev, &pl, &empty);
  if (s != SFP8_OK || empty) return s;
  if (pl.partial_bytes + pl.counter_bytes > kNoAllocScratchBytes) return SFP8_ERR_WORKSPACE;
  void* scratch = nullptr;
  s = noalloc_scratch(&scratch);
  if (s != SFP8_OK) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint8_t* counters = static_cast<uint8_t*>(scratch) + pl.partial_bytes;
  // The buffer keeps whatever the previous call left; the counters must
  // start at zero (the partial sums are always written before being read).
  if (pl.counter_bytes > 0 &&
      cudaMemsetAsync(counters, 0, pl.counter_bytes, st) != cudaSuccess)
    return SFP8_ERR_CUDA;
  return launch_linear(dev, pl, a_q, a_dtype, s_a, m, packed, w_dtype, s_w, n, k, bias, y,
                       static_cast<float*>(scratch), reinterpret_cast<unsigned int*>(counters),
                       st);
}

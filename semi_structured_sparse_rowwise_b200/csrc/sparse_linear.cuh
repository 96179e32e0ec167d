// Row-wise scaled 2:4 sparse FP8 GEMM for sm_100a.
//
// Page "Add CUTLASS-based row-wise scaled sparse FP8 kernel" (pytorch/ao pull
// request 1671), item 1: the linear with a 2:4 sparse FP8 weight and an FP8
// activation, each scaled per row; the four e4m3/e5m2 instantiations of the
// file table in issue 3516 are one kernel here, the operand formats being
// fields of the run-time instruction descriptor.
//
//     y[m, n] = bf16_RNE(acc[n, m] * s_a[m] * s_w[n] + bias[n])
//
// The sm_100 sparse MMA takes its 2:4 operand on the M side, so the weight is
// the MMA's A operand (128 weight rows per tile) and the activation its B
// operand (BN tokens per tile): the kernel computes y^T = W_sp . A_q^T.  The
// fp32 accumulator sits in tensor memory with lane = weight row n and column
// = token m, so in the epilogue the 32 lanes of a warp hold 32 consecutive
// n of one token and store a contiguous run of y.
//
// Structure (one CTA per SM, persistent):
//   warps 0-3   producers: per stage of KS 128-wide k steps, ONE contiguous
//               bulk copy of KS packed weight tiles (each 8 KB of kept values,
//               stored pre-swizzled in the 64B-swizzle form the MMA reads,
//               followed by its 2 KB of index metadata), and one 3-D TMA copy
//               of the KS activation tiles (BN x 128 B each, 128B swizzle).
//               Up to four producer warps issue, each owning every P-th
//               stage: an issuing thread keeps about one copy in flight, so
//               copies must come from several warps to overlap.
//               With a single token tile (decode) the CTA's whole activation
//               slice is loaded once instead (one 3-D TMA copy) and a stage is
//               just the weight copy; the weight beyond the first ring fill
//               is prefetched into L2 at the start.
//   warp 4      MMA issuer: per k step, copies the metadata block into tensor
//               memory (tcgen05.cp 128x128b) and issues two 128 x BN x 64
//               sparse MMAs; frees the stage with tcgen05.commit.  The whole
//               warp walks the loop and one elected lane issues.
//   warps 5-8   epilogue: tensor memory -> registers -> scale/bias/bf16 ->
//               global, or split-K partials to the workspace.
// Work split, chosen by the host:
//   whole tiles  CTA c takes tiles c, c + grid, ...: no partial sums.
//   stream-K     the (tile, stage) iterations are divided evenly over the
//                CTAs.  A tile split between CTAs is finished by its last
//                part: if every other part has already published its fp32
//                partial (a counter read with acquire semantics), straight
//                from its registers; otherwise it publishes its own and the
//                release/acquire counter update picks the finisher.  Parts
//                are always added in CTA order, so results are bit-identical
//                run to run whichever part finishes.
//
// Fused activation quantisation (FQ, one token tile of at most 16 tokens):
// instead of loading codes that the row-wise quantiser wrote, every CTA
// quantises the activation itself -- warps 5-12 read the m rows of x, reduce
// each row's amax, and write its codes (the quantiser's own quotient and
// conversion, so the same bits) straight into the resident activation's
// swizzled shared-memory tile.  The producers stream the weight meanwhile;
// the MMA warp waits for the codes.  The codes and scales also go to global
// memory, each k step of the codes written by one CTA.
//
// Every wait is bounded (device_common.cuh): on a timeout the CTA records
// SFP8_DEVICE_TIMEOUT, lets its copies in flight land, drains its MMAs,
// frees its tensor memory and returns.
#pragma once

#include <cuda_bf16.h>

#include "device_common.cuh"
#include "quantize_rowwise.cuh"

namespace sfp8 {

constexpr int kTileN = 128;     // weight rows per tile (MMA M)
constexpr int kStepK = 128;     // logical k per k step
constexpr int kWValBytes = kTileN * kStepK / 2;       // 8192: kept values of a tile
constexpr int kWMetaBytes = kTileN * kStepK / 8;      // 2048: index metadata of a tile
constexpr int kWTileBytes = kWValBytes + kWMetaBytes;  // 10240: packed tile
constexpr int kProducerWarps = 4;                       // warps issuing copies (max)
constexpr int kMmaWarp = kProducerWarps;                // one warp issuing MMAs
constexpr int kEpiWarp0 = kProducerWarps + 1;           // four epilogue warps
constexpr int kGemmThreads = 32 * (kProducerWarps + 5);
constexpr int kEpiThreads = 128;
constexpr int kSmemBudget = 225 * 1024;
// Fused quantisation: the four epilogue warps and four more quantise.
constexpr int kFusedQuantWarps = 8;
constexpr int kFusedQuantThreads = 32 * kFusedQuantWarps;
constexpr int kFusedMaxTokens = 16;
constexpr uint32_t kQuantBarrier = 2;   // named barrier of the quantiser warps
__host__ __device__ constexpr int linear_threads(bool fq) {
  return kGemmThreads + (fq ? kFusedQuantThreads - kEpiThreads : 0);
}

__host__ __device__ constexpr int pow2_at_least(int v) {
  int p = 32;
  while (p < v) p <<= 1;
  return p;
}

template <int BN, int KS, bool RA>
struct LinearCfg {
  static_assert(BN % 16 == 0 && BN >= 16 && BN <= 256, "BN must be 16..256, multiple of 16");
  static_assert(KS == 1 || KS == 2 || KS == 4, "1, 2 or 4 k steps per stage");
  static constexpr int kATileBytes = BN * kStepK;                 // one k step of activation
  // RA: the activation is resident for the whole k range, not per stage
  static constexpr int kStageBytes = KS * kWTileBytes + (RA ? 0 : KS * kATileBytes);
  static constexpr int kNumAcc = (2 * BN + 4 * KS <= 512) ? 2 : 1;
  static constexpr int kMetaCol = kNumAcc * BN;
  static constexpr int kTmemCols = pow2_at_least(kNumAcc * BN + 4 * KS);
  static constexpr int kMaxStages = 16;
  static constexpr int kBarrierBytes = 1024;
  static_assert(kStageBytes % 1024 == 0, "stages must stay 1024-byte aligned");
};

// Shared memory of a launch: align slack + resident activation + stages +
// barriers.
__host__ __device__ constexpr int linear_smem_bytes(int ra_bytes, int stages, int stage_bytes) {
  return 1024 + ra_bytes + stages * stage_bytes + 1024;
}

struct LinearParams {
  const uint8_t* packed;    // compressed weight, 10 KB tiles (layout version 3)
  const float* s_a;
  const float* s_w;
  const __nv_bfloat16* bias;
  __nv_bfloat16* y;
  float* partials;          // [grid][2][BN][128] fp32 (stream-K only)
  unsigned int* counters;   // [tiles][4]: one per tile and lane quadrant (stream-K only)
  int m, n, k;
  int m_tiles;              // ceil(m / BN)
  int k_steps;              // k / 128
  int units;                // stages per tile: k_steps / KS
  long long tiles;          // n_tiles * m_tiles
  long long iters;          // tiles * units
  int grid;
  int whole_tiles;          // 1: CTA c takes tiles c, c + grid, ...; 0: stream-K
  int stages;               // shared-memory pipeline depth (<= kMaxStages)
  int ra_bytes;             // resident activation bytes (BN * k) or 0
  int producers;            // producer warps issuing copies (1..kProducerWarps)
  int tma_store;            // 1: y through a TMA store from shared memory (one tile per CTA,
                            // resident activation: its region stages the tile)
  uint32_t idesc;
  // fused quantisation only
  const void* x;            // activation [m][ld_x], x_dtype
  long long ld_x;           // row stride of x in elements
  int x_dtype;              // SFP8_BF16 / SFP8_F16 / SFP8_F32
  int a_fmt;                // SFP8_E4M3 / SFP8_E5M2
  uint8_t* a_q_out;         // codes [m][k], written (k step t by CTA t mod grid)
  float* s_a_out;           // row scales [m], written by CTA 0
};

// The work of one CTA, one tile segment [u0, u1) (in stages) at a time.  All
// three roles walk it identically.
struct SegmentWalker {
  long long it, end;
  int units;
  int grid;
  bool whole;
  __device__ SegmentWalker(const LinearParams& p, int cta) {
    units = p.units;
    grid = p.grid;
    whole = p.whole_tiles != 0;
    if (whole) {
      it = cta;               // next tile
      end = p.tiles;
    } else {
      it = static_cast<long long>(cta) * p.iters / p.grid;
      end = static_cast<long long>(cta + 1) * p.iters / p.grid;
    }
  }
  __device__ bool next(long long& tile, int& u0, int& u1) {
    if (it >= end) return false;
    if (whole) {
      tile = it;
      u0 = 0;
      u1 = units;
      it += grid;
      return true;
    }
    tile = it / units;
    u0 = static_cast<int>(it % units);
    const long long left = end - it;
    u1 = static_cast<int>(left < units - u0 ? u0 + left : units);
    it += u1 - u0;
    return true;
  }
};

// Stream-K: CTA owning iteration i (the inverse of the even split).
__device__ __forceinline__ int cta_of_iter(long long i, const LinearParams& p) {
  return static_cast<int>(((i + 1) * p.grid - 1) / p.iters);
}

// Stream-K: partial-sum slot of CTA `cc` for `tile`: slot 0 holds the part of
// the tile its range starts in, slot 1 the part of the tile its range ends in.
template <int BN>
__device__ __forceinline__ const float* partial_slot(const LinearParams& p, int cc,
                                                     long long tile) {
  const long long start = static_cast<long long>(cc) * p.iters / p.grid;
  const int slot = (start / p.units == tile) ? 0 : 1;
  return p.partials + (static_cast<long long>(cc) * 2 + slot) * (BN * kTileN);
}

// Epilogue of one 16-column chunk: y = acc * (s_a * s_w) + bias.
__device__ __forceinline__ void store_chunk(const LinearParams& p, const float (&acc)[16],
                                            const float (&sa)[16], int n, int m0, float sw,
                                            float bias) {
  if (n >= p.n) return;
#pragma unroll
  for (int j = 0; j < 16; ++j) {
    const int m = m0 + j;
    if (m < p.m) {
      const float v = fmaf(acc[j], sa[j] * sw, bias);
      p.y[static_cast<long long>(m) * p.n + n] = __float2bfloat16_rn(v);
    }
  }
}

template <bool FQ = false>
__device__ __forceinline__ void load_sa(const LinearParams& p, int m0, float (&sa)[16],
                                        const float* sa_sm = nullptr) {
#pragma unroll
  for (int j = 0; j < 16; ++j) {
    if constexpr (FQ)
      sa[j] = (m0 + j < p.m) ? sa_sm[m0 + j] : 0.0f;
    else
      sa[j] = (m0 + j < p.m) ? __ldg(p.s_a + m0 + j) : 0.0f;
  }
}

// Fused quantisation of the m <= 16 rows of x by the kFusedQuantThreads
// quantiser threads (index qt): per row, amax = max |x| over the row, s =
// max(amax, 1e-12) / FP8_MAX, codes = satfinite RNE(x / s) -- exactly the
// arithmetic of quantize_rowwise_kernel.  The rows are spread over all
// threads (256 / R threads per row, R the row count rounded up to a power of
// two); x is read twice (amax, then codes; the second read hits L2).  Codes
// land in `ra` as the tile [k step][16 rows][128 B] with the 128-byte swizzle
// (16-byte chunk c of row r at chunk c ^ (r mod 8)); rows past m get zero
// codes.  `red` is shared scratch of kFusedQuantWarps floats.
template <typename T, int kFmt>
__device__ __forceinline__ void fused_quantize(const LinearParams& p, int qt, uint8_t* ra,
                                               float* sa_sm, float* red) {
  using Tr = InputTraits<T>;
  constexpr int P = Tr::kPerVec;      // elements per 16-byte vector
  constexpr int NV = 16 / P;          // vectors per 16 codes
  constexpr int kTileBytes = kFusedMaxTokens * kStepK;
  const int rows_p2 = p.m <= 1 ? 1 : p.m <= 2 ? 2 : p.m <= 4 ? 4 : p.m <= 8 ? 8 : 16;
  const int tpr = kFusedQuantThreads / rows_p2;
  const int row = qt / tpr;
  const int sub = qt % tpr;
  const bool live = row < p.m;
  const T* xr = static_cast<const T*>(p.x) + static_cast<long long>(live ? row : 0) * p.ld_x;
  float amax = 0.0f;
  if (live) {
    const int nvec = p.k / P;
#pragma unroll 8
    for (int v = sub; v < nvec; v += tpr)
      amax = Tr::abs_max(__ldg(reinterpret_cast<const uint4*>(xr + static_cast<long long>(v) * P)),
                         amax);
  }
  for (int o = (tpr < 32 ? tpr : 32) / 2; o > 0; o >>= 1)
    amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
  if (tpr > 32) {
    const int w = qt / 32;
    if (qt % 32 == 0) red[w] = amax;
    named_barrier_sync(kQuantBarrier, kFusedQuantThreads);
    const int wpr = tpr / 32;
    const int first = (w / wpr) * wpr;
    float mx = red[first];
    for (int i = 1; i < wpr; ++i) mx = fmaxf(mx, red[first + i]);
    amax = mx;
  }
  const float s = __fdiv_rn(fmaxf(amax, kGuardAmax), Fp8Out<kFmt>::kMax);
  const float r = __frcp_rn(s);
  if (live && sub == 0) {
    sa_sm[row] = s;
    if (blockIdx.x == 0) p.s_a_out[row] = s;
  }
  const int nchunk = p.k / 16;
  const int rsw = row % 8;
  uint8_t* ra_row = ra + (row / 8) * 1024 + rsw * 128;
  uint8_t* q_row = p.a_q_out + static_cast<long long>(live ? row : 0) * p.k;
#pragma unroll 4
  for (int j = sub; j < nchunk; j += tpr) {
    uint4 out = make_uint4(0u, 0u, 0u, 0u);
    const int ks = j / 8;
    if (live) {
      uint4 v[NV];
#pragma unroll
      for (int i = 0; i < NV; ++i)
        v[i] = __ldg(reinterpret_cast<const uint4*>(xr + static_cast<long long>(j) * 16 + i * P));
      uint32_t w[4];
#pragma unroll
      for (int i = 0; i < NV; ++i) {
        float f[P];
        Tr::to_float(v[i], f);
        uint32_t ww[P / 4];
        quantize_vec<kFmt, P>(f, s, r, ww);
#pragma unroll
        for (int t = 0; t < P / 4; ++t) w[i * (P / 4) + t] = ww[t];
      }
      out = make_uint4(w[0], w[1], w[2], w[3]);
      if (ks % p.grid == static_cast<int>(blockIdx.x))
        *reinterpret_cast<uint4*>(q_row + static_cast<long long>(j) * 16) = out;
    }
    *reinterpret_cast<uint4*>(ra_row + ks * kTileBytes + (((j % 8) ^ rsw) * 16)) = out;
  }
  // rows that no thread group covers (fewer rows than the tile): zero codes
  const int rest = (kFusedMaxTokens - rows_p2) * nchunk;
  for (int idx = qt; idx < rest; idx += kFusedQuantThreads) {
    const int r2 = rows_p2 + idx / nchunk;
    const int j = idx % nchunk;
    *reinterpret_cast<uint4*>(ra + (j / 8) * kTileBytes + (r2 / 8) * 1024 + (r2 % 8) * 128 +
                              (((j % 8) ^ (r2 % 8)) * 16)) = make_uint4(0u, 0u, 0u, 0u);
  }
}

// The quantiser threads' part of the fused kernel: codes and scales for the
// input type and code format of the call, made visible to the MMAs (async
// proxy) and signalled on `ra_bar`.
__device__ __forceinline__ void fused_quantize_all(const LinearParams& p, int qt, uint8_t* ra,
                                                   float* sa_sm, float* red, uint64_t* ra_bar) {
  const bool e5 = p.a_fmt == SFP8_E5M2;
  if (p.x_dtype == SFP8_BF16) {
    if (e5) fused_quantize<__nv_bfloat16, SFP8_E5M2>(p, qt, ra, sa_sm, red);
    else fused_quantize<__nv_bfloat16, SFP8_E4M3>(p, qt, ra, sa_sm, red);
  } else if (p.x_dtype == SFP8_F16) {
    if (e5) fused_quantize<__half, SFP8_E5M2>(p, qt, ra, sa_sm, red);
    else fused_quantize<__half, SFP8_E4M3>(p, qt, ra, sa_sm, red);
  } else {
    if (e5) fused_quantize<float, SFP8_E5M2>(p, qt, ra, sa_sm, red);
    else fused_quantize<float, SFP8_E4M3>(p, qt, ra, sa_sm, red);
  }
  fence_proxy_async_smem();
  named_barrier_sync(kQuantBarrier, kFusedQuantThreads);
  if (qt == 0) mbar_arrive(smem_u32(ra_bar));
}

template <int BN, int KS, bool RA, bool FQ = false>
__global__ void __launch_bounds__(linear_threads(FQ), 1)
    sparse_linear_kernel(const __grid_constant__ CUtensorMap tm_a,
                         const __grid_constant__ CUtensorMap tm_y, const LinearParams p) {
  static_assert(!FQ || (RA && BN == kFusedMaxTokens), "fused quantisation: one 16-token tile");
  using Cfg = LinearCfg<BN, KS, RA>;
  const int S = p.stages;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t* ra_base = smem;                       // resident activation (RA)
  uint8_t* stage_base = smem + p.ra_bytes;
  uint64_t* bars = reinterpret_cast<uint64_t*>(stage_base + S * Cfg::kStageBytes);
  constexpr int SM = Cfg::kMaxStages;
  uint64_t* full_bar = bars;                  // [S]
  uint64_t* empty_bar = bars + SM;            // [S]
  uint64_t* accf_bar = bars + 2 * SM;         // [2]
  uint64_t* acce_bar = bars + 2 * SM + 2;     // [2]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * SM + 4);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(bars + 2 * SM + 5);
  uint64_t* drain_bar = bars + 2 * SM + 6;
  uint64_t* ra_bar = bars + 2 * SM + 7;
  float* sa_sm = reinterpret_cast<float*>(bars + 2 * SM + 8);      // [16] (FQ)
  float* q_red = reinterpret_cast<float*>(bars + 2 * SM + 16);     // [8] (FQ)

  const int warp = threadIdx.x / 32;
  const int lane = threadIdx.x % 32;
  const int cta = blockIdx.x;
  // Dependent kernels of this library may launch right away: each of them
  // waits (griddepcontrol.wait) for this grid to complete before it reads or
  // writes anything this grid uses, so an early trigger only lets their
  // launch and their own weight prefetch overlap this grid's tail.
  grid_dependents_launch();

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(smem_u32(&full_bar[s]), 1);
      mbar_init(smem_u32(&empty_bar[s]), 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(smem_u32(&accf_bar[b]), 1);
      mbar_init(smem_u32(&acce_bar[b]), kEpiThreads / 32);
    }
    mbar_init(smem_u32(drain_bar), 1);
    mbar_init(smem_u32(ra_bar), 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (!FQ && warp == 0 && lane == 0) tma_prefetch_desc(&tm_a);
  if (warp == kMmaWarp) {
    tmem_alloc(smem_u32(tmem_slot), Cfg::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp < kProducerWarps) {
    // ------------------------------------------------------------ producers
    // Lane 0 of producer warp w < P issues the copies of stages i with
    // i % P == w.
    // no more producers than ring slots (see the host plan)
    const int P = p.producers < S ? p.producers : S;
    const int pw = warp;
    if (lane == 0 && pw < P) {
      // A weight tile is read once when there is one token tile (decode:
      // keep it from displacing anything); otherwise every token tile reuses
      // it, so it must stay in L2.
      const uint64_t pol_w = p.m_tiles == 1 ? l2_policy_evict_first() : l2_policy_evict_normal();
      const uint64_t pol_a = l2_policy_evict_last();
      auto issue_weight = [&](int stage, long long tile, int u) {
        const int nt = static_cast<int>(tile / p.m_tiles);
        uint8_t* st = stage_base + stage * Cfg::kStageBytes;
        const uint32_t fb = smem_u32(&full_bar[stage]);
        mbar_arrive_expect_tx(fb, Cfg::kStageBytes);
        bulk_load(smem_u32(st),
                  p.packed + (static_cast<long long>(nt) * p.k_steps + u * KS) * kWTileBytes,
                  KS * kWTileBytes, fb, pol_w);
      };
      auto issue_act = [&](int stage, long long tile, int u) {
        const int mt = static_cast<int>(tile % p.m_tiles);
        uint8_t* st = stage_base + stage * Cfg::kStageBytes + KS * kWTileBytes;
        tma_load_3d(smem_u32(st), &tm_a, 0, mt * BN, u * KS, smem_u32(&full_bar[stage]), pol_a);
      };
      // The weight does not depend on the preceding kernel: fill the first
      // stages with weight tiles before waiting for the activation.
      long long pre_count = 0;
      {
        SegmentWalker pre(p, cta);
        long long t2;
        int a0, a1;
        while (pre_count < S && pre.next(t2, a0, a1))
          for (int u = a0; u < a1 && pre_count < S; ++u) {
            if (pre_count % P == pw) issue_weight(static_cast<int>(pre_count), t2, u);
            ++pre_count;
          }
      }
      if (pw == 0 && p.m_tiles == 1) {
        // One token tile: everything past the stages just filled is read
        // once, by this CTA.  Ask L2 to fetch it now, so that HBM keeps
        // streaming while the ring waits for the activation.
        const uint64_t pol_pf = l2_policy_evict_normal();
        SegmentWalker pf(p, cta);
        long long t3;
        int b0, b1;
        long long seen = 0;
        while (pf.next(t3, b0, b1)) {
          const int nt3 = static_cast<int>(t3 / p.m_tiles);
          int s0 = b0;
          if (seen < pre_count) {
            const long long skip = pre_count - seen < b1 - b0 ? pre_count - seen : b1 - b0;
            s0 = b0 + static_cast<int>(skip);
          }
          seen += b1 - b0;
          if (s0 < b1) {
            // a hint: at most the next 16 MB of the segment
            long long bytes = static_cast<long long>(b1 - s0) * KS * kWTileBytes;
            if (bytes > (16ll << 20)) bytes = 16ll << 20;
            l2_prefetch_bulk(
                p.packed + (static_cast<long long>(nt3) * p.k_steps + s0 * KS) * kWTileBytes,
                static_cast<uint32_t>(bytes), pol_pf);
          }
        }
      }
      if (RA && !FQ && pw == P - 1) {
        // The whole activation slice of this CTA, [k steps][BN rows][128 B],
        // in one copy by the warp that issued the fewest prefetch copies.
        grid_dependency_wait();
        mbar_arrive_expect_tx(smem_u32(ra_bar), p.ra_bytes);
        tma_load_3d(smem_u32(ra_base), &tm_a, 0, 0, 0, smem_u32(ra_bar), pol_a);
      } else {
        grid_dependency_wait();
      }
      SegmentWalker walk(p, cta);
      long long tile;
      int u0, u1;
      long long i = 0;              // stage sequence number
      bool ok = true;
      while (ok && walk.next(tile, u0, u1)) {
        for (int u = u0; u < u1; ++u, ++i) {
          if (i % P != pw) continue;
          const int stage = static_cast<int>(i % S);
          if (i >= pre_count) {
            const uint32_t phase = static_cast<uint32_t>((i / S) & 1);
            if (!mbar_wait(smem_u32(&empty_bar[stage]), phase ^ 1u, abort_flag)) {
              ok = false;
              break;
            }
            issue_weight(stage, tile, u);
          }
          if (!RA) issue_act(stage, tile, u);
        }
      }
      if (!ok) {
        // Let this lane's copies already issued land before the CTA exits.
        const long long issued = i;      // stages up to (not incl.) i were considered
        long long first = issued > S ? issued - S : 0;
        for (long long t = first; t < issued; ++t) {
          if (t % P != pw) continue;
          const int s2 = static_cast<int>(t % S);
          const uint32_t ph = static_cast<uint32_t>((t / S) & 1);
          volatile int no_abort = 0;
          mbar_wait(smem_u32(&full_bar[s2]), ph, &no_abort);
        }
        if (RA && !FQ && pw == P - 1) {
          volatile int no_abort = 0;
          mbar_wait(smem_u32(ra_bar), 0, &no_abort);
        }
      }
    }
  } else if (warp == kMmaWarp) {
    // ------------------------------------------------------------ MMA issuer
    // The whole warp walks the loop (converged, so its operands stay
    // warp-uniform); one elected lane issues each tcgen05 operation.
    {
      grid_dependency_wait();   // start the wait limits only once inputs exist
      SegmentWalker walk(p, cta);
      long long tile;
      int u0, u1;
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      const uint32_t e_tmem = tmem_base + Cfg::kMetaCol;
      bool ok = true;
      if (RA) ok = mbar_wait_warp(smem_u32(ra_bar), 0, abort_flag);
      // Whether the full barrier of `stage` was already seen complete (each
      // stage tests the next one's right after its first MMA, so that the
      // barrier's latency overlaps queued tensor work).
      bool ready = false;
      while (ok && walk.next(tile, u0, u1)) {
        if (!mbar_wait_warp(smem_u32(&acce_bar[acc]), acc_phase ^ 1u, abort_flag)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + acc * BN;
        for (int u = u0; u < u1; ++u) {
          if (!ready && !mbar_wait_warp(smem_u32(&full_bar[stage]), phase, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const int next_stage = stage + 1 == S ? 0 : stage + 1;
          const uint32_t next_phase = stage + 1 == S ? phase ^ 1u : phase;
          const uint32_t st = smem_u32(stage_base + stage * Cfg::kStageBytes);
#pragma unroll
          for (int j = 0; j < KS; ++j) {
            const uint32_t w_addr = st + j * kWTileBytes;
            const uint32_t e_addr = w_addr + kWValBytes;
            const uint32_t a_addr =
                RA ? smem_u32(ra_base) + (u * KS + j) * Cfg::kATileBytes
                   : st + KS * kWTileBytes + j * Cfg::kATileBytes;
            // metadata: 128 rows x 16 bytes, no swizzle, 8-row groups 128 B apart;
            // k steps j and j + 1 (consecutive tiles, kWTileBytes apart) in one
            // 128 x 256-bit copy
            if constexpr (KS == 1) {
              tc_cp_128x128b_w(e_tmem, smem_desc(e_addr, 0, 128, kNoSwizzle));
            } else if (j % 2 == 0) {
              tc_cp_128x256b_w(e_tmem + 4 * j, smem_desc(e_addr, kWTileBytes, 128, kNoSwizzle));
            }
#pragma unroll
            for (int h = 0; h < 2; ++h) {
              // weight: 128 rows x 64 B (64B swizzle, 8-row atoms 512 B apart);
              // each MMA consumes 32 B of every row (64 logical k).
              const uint64_t adesc = smem_desc(w_addr + 32 * h, 16, 512, kSwizzle64);
              // activation: BN rows x 128 B (128B swizzle, atoms 1024 B apart);
              // each MMA consumes 64 B of every row.
              const uint64_t bdesc = smem_desc(a_addr + 64 * h, 16, 1024, kSwizzle128);
              mma_sp_f8f6f4_w(d_tmem, adesc, bdesc, e_tmem + 4 * j + 2 * h, p.idesc,
                              (u > u0 || j > 0 || h > 0) ? 1u : 0u);
              if (j == 0 && h == 0)
                ready = mbar_test_warp(smem_u32(&full_bar[next_stage]), next_phase);
            }
          }
          tc_commit_w(smem_u32(&empty_bar[stage]));
          stage = next_stage;
          phase = next_phase;
        }
        if (!ok) break;
        tc_commit_w(smem_u32(&accf_bar[acc]));
        if (Cfg::kNumAcc == 2) {
          acc ^= 1;
          if (acc == 0) acc_phase ^= 1u;
        } else {
          acc_phase ^= 1u;
        }
      }
      // Every MMA issued must have finished before tensor memory is freed.
      tc_commit_w(smem_u32(drain_bar));
      volatile int no_abort = 0;
      mbar_wait_warp(smem_u32(drain_bar), 0, &no_abort);
    }
  } else if (FQ && warp >= kEpiWarp0 + 4) {
    // ------------------------------------------------------------ quantiser only
    grid_dependency_wait();
    fused_quantize_all(p, threadIdx.x - 32 * kEpiWarp0, ra_base, sa_sm, q_red, ra_bar);
  } else {
    // ------------------------------------------------------------ epilogue
    // Each of the four warps owns 32 weight rows (its tensor-memory lane
    // quadrant) and finishes them on its own, split-K fix-up included, so no
    // barrier spans the four warps.
    grid_dependency_wait();
    if constexpr (FQ)
      fused_quantize_all(p, threadIdx.x - 32 * kEpiWarp0, ra_base, sa_sm, q_red, ra_bar);
    const int q = warp % 4;
    SegmentWalker walk(p, cta);
    long long tile;
    int u0, u1;
    int acc = 0;
    uint32_t acc_phase = 0;
    long long first_tile = -1;
    while (walk.next(tile, u0, u1)) {
      if (first_tile < 0) first_tile = tile;
      const int nt = static_cast<int>(tile / p.m_tiles);
      const int mt = static_cast<int>(tile % p.m_tiles);
      const int n_local = q * 32 + lane;
      const int n = nt * kTileN + n_local;
      const bool whole = (u0 == 0 && u1 == p.units);
      // Everything the epilogue needs besides the accumulator, loaded before
      // waiting for it.
      const float sw = (n < p.n) ? __ldg(p.s_w + n) : 0.0f;
      const float bv = (p.bias != nullptr && n < p.n) ? __bfloat162float(p.bias[n]) : 0.0f;
      float sa0[16];
      load_sa<FQ>(p, mt * BN, sa0, sa_sm);
      int c_first = cta, c_last = cta;
      unsigned int parts = 1;
      unsigned int* counter = p.counters + tile * 4 + q;
      if (!whole) {
        const long long it0 = tile * p.units;
        c_first = cta_of_iter(it0, p);
        c_last = cta_of_iter(it0 + p.units - 1, p);
        parts = static_cast<unsigned int>(c_last - c_first + 1);
      }
      int ok = 1;
      if (lane == 0) ok = mbar_wait(smem_u32(&accf_bar[acc]), acc_phase, abort_flag) ? 1 : 0;
      ok = __shfl_sync(0xffffffffu, ok, 0);
      if (!ok) break;
      // Split tile: finish it here if every other part has already arrived.
      bool finish_now = false;
      if (!whole) {
        unsigned int arrived = 0;
        if (lane == 0) arrived = load_acquire_gpu(counter);
        finish_now = __shfl_sync(0xffffffffu, arrived, 0) + 1 == parts;
      }
      tc_fence_after();
      const int slot = (tile == first_tile) ? 0 : 1;
      float* part = p.partials + (static_cast<long long>(cta) * 2 + slot) * (BN * kTileN);
      const uint32_t t_row = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + acc * BN;
#pragma unroll 1
      for (int c = 0; c < BN / 16; ++c) {
        uint32_t r[16];
        tmem_ld_32x32b_x16(t_row + c * 16, r);
        float sa[16];
        if (c == 0) {
#pragma unroll
          for (int j = 0; j < 16; ++j) sa[j] = sa0[j];
        } else {
          load_sa<FQ>(p, mt * BN + c * 16, sa, sa_sm);
        }
        tmem_ld_wait();
        float v[16];
#pragma unroll
        for (int j = 0; j < 16; ++j) v[j] = __uint_as_float(r[j]);
        if (whole && p.tma_store) {
          // stage the bf16 tile [BN tokens][128 rows] in the resident
          // activation's region, free once the tile's MMAs have completed
          __nv_bfloat16* stg = reinterpret_cast<__nv_bfloat16*>(ra_base);
#pragma unroll
          for (int j = 0; j < 16; ++j)
            stg[(c * 16 + j) * kTileN + n_local] = __float2bfloat16_rn(fmaf(v[j], sa[j] * sw, bv));
        } else if (whole) {
          store_chunk(p, v, sa, n, mt * BN + c * 16, sw, bv);
        } else if (finish_now) {
          float sum[16];
#pragma unroll
          for (int j = 0; j < 16; ++j) sum[j] = 0.0f;
          for (int cc = c_first; cc <= c_last; ++cc) {
            if (cc == cta) {
#pragma unroll
              for (int j = 0; j < 16; ++j) sum[j] += v[j];
            } else {
              const float* src = partial_slot<BN>(p, cc, tile) + c * 16 * kTileN + n_local;
              float a[16];
#pragma unroll
              for (int j = 0; j < 16; ++j) a[j] = __ldcg(src + j * kTileN);
#pragma unroll
              for (int j = 0; j < 16; ++j) sum[j] += a[j];
            }
          }
          store_chunk(p, sum, sa, n, mt * BN + c * 16, sw, bv);
        } else {
#pragma unroll
          for (int j = 0; j < 16; ++j) part[(c * 16 + j) * kTileN + n_local] = v[j];
        }
      }
      if (whole && p.tma_store) {
        // one bulk tensor store of the tile; rows past m and columns past n
        // are clipped by the tensor map
        fence_proxy_async_smem();
        named_barrier_sync(1, kEpiThreads);
        if (warp == kEpiWarp0 && lane == 0) {
          tma_store_2d(&tm_y, smem_u32(ra_base), nt * kTileN, mt * BN);
          bulk_commit_group();
          bulk_wait_group_0();
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&acce_bar[acc]));
      if (Cfg::kNumAcc == 2) {
        acc ^= 1;
        if (acc == 0) acc_phase ^= 1u;
      } else {
        acc_phase ^= 1u;
      }
      if (finish_now) {
        if (lane == 0) *counter = 0u;   // every other part has counted already
      } else if (!whole) {
        // The counter update is a release/acquire atomic: it orders this
        // warp's part (stores ordered across the warp by __syncwarp) before
        // the count and, for the last part, every other part before the
        // loads below.
        __syncwarp();
        unsigned int last = 0;
        if (lane == 0) last = (atomic_add_acq_rel_gpu(counter, 1u) + 1 == parts) ? 1u : 0u;
        last = __shfl_sync(0xffffffffu, last, 0);
        if (last) {
          __syncwarp();
#pragma unroll 1
          for (int c = 0; c < BN / 16; ++c) {
            float sa[16];
            load_sa<FQ>(p, mt * BN + c * 16, sa, sa_sm);
            float v[16];
#pragma unroll
            for (int j = 0; j < 16; ++j) v[j] = 0.0f;
            int cc = c_first;
            // two parts per round trip; additions stay in CTA order
            for (; cc + 1 <= c_last; cc += 2) {
              const float* s0 = partial_slot<BN>(p, cc, tile) + c * 16 * kTileN + n_local;
              const float* s1 = partial_slot<BN>(p, cc + 1, tile) + c * 16 * kTileN + n_local;
              float a0[16], a1[16];
#pragma unroll
              for (int j = 0; j < 16; ++j) {
                a0[j] = __ldcg(s0 + j * kTileN);
                a1[j] = __ldcg(s1 + j * kTileN);
              }
#pragma unroll
              for (int j = 0; j < 16; ++j) v[j] = (v[j] + a0[j]) + a1[j];
            }
            if (cc <= c_last) {
              const float* s0 = partial_slot<BN>(p, cc, tile) + c * 16 * kTileN + n_local;
#pragma unroll
              for (int j = 0; j < 16; ++j) v[j] += __ldcg(s0 + j * kTileN);
            }
            store_chunk(p, v, sa, n, mt * BN + c * 16, sw, bv);
          }
          if (lane == 0) *counter = 0u;
        }
      }
    }
  }

  // ------------------------------------------------------------ teardown
  __syncthreads();
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem_base, Cfg::kTmemCols);
  }
}

}  // namespace sfp8

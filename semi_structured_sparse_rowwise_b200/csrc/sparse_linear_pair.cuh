// Row-wise scaled 2:4 sparse FP8 GEMM on CTA pairs (cta_group::2), for many
// tokens (prefill).
//
// Same operation as sparse_linear.cuh (page "Add CUTLASS-based row-wise
// scaled sparse FP8 kernel", pytorch/ao pull request 1671, item 1):
//
//     y[m, n] = bf16_RNE(acc[n, m] * s_a[m] * s_w[n] + bias[n])
//
// A tile is 256 weight rows x BN tokens (BN a multiple of 32, at most 224,
// chosen per call to split the tokens evenly), computed by a cluster of two
// CTAs on two SMs with one tcgen05.mma.sp of M = 256, N = BN per 64 logical
// k.  CTA r of the pair holds weight rows [128 r, 128 r + 128) of the tile
// and tokens [r BN/2, (r + 1) BN/2) of it in its own shared memory; the MMA
// reads the A half of each CTA and both B halves, and writes each CTA's
// 128-lane half of the accumulator into that CTA's tensor memory (column c =
// token c of the tile).  Against one CTA computing 128 x BN alone, every SM
// loads and reads half the activation bytes per MMA, which is what lets the
// sparse tensor pipe run at its full rate: a lone CTA's MMA is bound by
// shared-memory reads (the activation operand of a sparse MMA is twice as
// long as its weight operand).  BN <= 224 leaves room in the 512 tensor-
// memory columns for two accumulators and the metadata, so the epilogue of a
// tile overlaps the MMAs of the next.  (The pair form of the sparse FP8 MMA
// takes N in steps of 32.)
//
// Roles (both CTAs unless noted):
//   warps 0-3   producers: per stage, one TMA copy of the CTA's packed
//               weight tiles (a 3-D or 4-D view of the 10 KB tiles) and one
//               of its activation tiles; all copies of a stage, both CTAs',
//               complete on the stage barrier of rank 0, which rank 0 arms
//               with the byte count of the pair.
//   warp 4      rank 0: the MMA issuer (metadata copies and MMAs for the pair,
//               commits multicast to both CTAs' barriers), the whole warp
//               walking the loop and one elected lane issuing.  Rank 1: only
//               allocates and frees tensor memory with rank 0.
//   warps 5-    epilogue: two warps per tensor-memory lane quadrant (and
//               weight slot), each taking every other 16-column chunk of the
//               accumulator: tensor memory -> registers -> scale/bias/bf16
//               -> global.
// Work split: tile t -> (weight group, token tile) in bands of token tiles
// (pair_tile_coords), pair p takes tiles p, p + pairs, ...  No split-K.  Tensor memory: accumulator b at columns
// [224 b, 224 b + BN), metadata of the stage's k steps at 448.
//
// Every wait is bounded (device_common.cuh); a timed-out CTA records
// SFP8_DEVICE_TIMEOUT and runs to the final cluster barrier, which both CTAs
// always reach.
#pragma once

#include <cuda_bf16.h>

#include "device_common.cuh"
#include "sparse_linear.cuh"

namespace sfp8 {

constexpr int kPairTileN = 256;        // weight rows per pair and weight slot (MMA M)
constexpr int kPairMaxTokens = 224;    // largest BN: 2 x 224 + metadata <= 512
constexpr int kPairLoadWarps = kProducerWarps;
constexpr int kPairMmaWarp = kPairLoadWarps;
constexpr int kPairEpiWarp0 = kPairMmaWarp + 1;
constexpr int kPairTmemCols = 512;
constexpr int kPairMetaCol = 2 * kPairMaxTokens;  // after the two accumulators

// KS k steps per stage; WT weight tiles (128 rows each) per CTA.
//   WT = 1: pair tile 256 x BN, two accumulators (double buffer).
//   WT = 2: pair tile 512 x BN, one accumulator per weight slot (single
//           buffer): each activation byte loaded feeds twice the MMAs.
template <int KS, int WT>
struct PairCfg {
  static_assert(KS == 1 || KS == 2, "1 or 2 k steps per stage");
  static_assert(WT == 1 || WT == 2, "1 or 2 weight tiles per CTA");
  static constexpr int kWBytes = KS * WT * kWTileBytes;
  static constexpr int kMaxStages = 16;
  static constexpr int kEpiWarps = 8 * WT;       // two per lane quadrant and slot
  static constexpr int kThreads = 32 * (kPairLoadWarps + 1 + kEpiWarps);
  static_assert(kPairMetaCol + 4 * KS * WT <= kPairTmemCols, "metadata columns must fit");
  // Shared memory of one stage for BN tokens per tile (a multiple of 1024).
  __host__ __device__ static constexpr int stage_bytes(int bn) {
    return KS * (WT * kWTileBytes + (bn / 2) * kStepK);
  }
};

__host__ __device__ constexpr int pair_smem_bytes(int stages, int stage_bytes) {
  return 1024 + stages * stage_bytes + 1024;
}

struct PairParams {
  const float* s_a;
  const float* s_w;
  const __nv_bfloat16* bias;
  __nv_bfloat16* y;
  int m, n, k;
  int n_tiles;      // 128-row weight tiles (ceil(n / 128))
  int n_groups;     // ceil(n_tiles / (2 WT)): weight-tile groups of a pair tile
  int bn;           // tokens per tile (multiple of 32, <= kPairMaxTokens)
  int m_tiles;      // ceil(m / bn)
  int k_steps;      // k / 128
  int units;        // stages per tile: k_steps / KS
  int tiles;        // n_groups * m_tiles
  int band;         // token tiles per band of the tile order (see pair_tile_coords)
  int pairs;        // gridDim.x / 2
  int stages;
  int stage_bytes;  // PairCfg<KS>::stage_bytes(bn)
  int producers;
  uint32_t idesc;
};

// Tile t -> (weight group g, token tile mt).  Tiles run in bands of p.band
// token tiles; within a band the token tile varies fastest, so the band's
// activation rows are reused by every weight group while they sit in L2 and
// each weight group is read once per band.  p.band = m_tiles is one band
// (every weight group read once); p.band = 1 runs every weight group over one
// token tile before the next (the weight stays in L2, the activation is read
// once).  The host picks the band from the operand sizes and the L2 size.
__device__ __forceinline__ void pair_tile_coords(const PairParams& p, int t, int& g, int& mt) {
  const int per_band = p.band * p.n_groups;
  const int b = t / per_band;
  const int r = t - b * per_band;
  const int m0 = b * p.band;
  const int bsize = p.m_tiles - m0 < p.band ? p.m_tiles - m0 : p.band;
  g = r / bsize;
  mt = m0 + (r - g * bsize);
}

__device__ __forceinline__ void load_sa_pair(const PairParams& p, int m0, float (&sa)[16]) {
#pragma unroll
  for (int j = 0; j < 16; ++j) sa[j] = (m0 + j < p.m) ? __ldg(p.s_a + m0 + j) : 0.0f;
}

template <int KS, int WT>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(PairCfg<KS, WT>::kThreads, 1)
    sparse_linear_pair_kernel(const __grid_constant__ CUtensorMap tm_w2,
                              const __grid_constant__ CUtensorMap tm_w,
                              const __grid_constant__ CUtensorMap tm_a, const PairParams p) {
  using Cfg = PairCfg<KS, WT>;
  const int S = p.stages;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t* stage_base = smem;
  const int SB = p.stage_bytes;
  uint64_t* bars = reinterpret_cast<uint64_t*>(stage_base + S * SB);
  constexpr int SM = Cfg::kMaxStages;
  uint64_t* full_bar = bars;                // [S], used on rank 0
  uint64_t* empty_bar = bars + SM;          // [S]
  uint64_t* accf_bar = bars + 2 * SM;       // [2] (WT = 2 uses [0])
  uint64_t* acce_bar = bars + 2 * SM + 2;   // [2], rank 0
  uint64_t* drain_bar = bars + 2 * SM + 4;  // rank 0
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * SM + 5);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(bars + 2 * SM + 6);

  const int warp = threadIdx.x / 32;
  const int lane = threadIdx.x % 32;
  const uint32_t rank = cluster_ctarank();
  const int pair = blockIdx.x / 2;
  // Same contract as the one-CTA kernel: dependents wait for this grid's
  // completion before touching anything it uses.
  grid_dependents_launch();

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(smem_u32(&full_bar[s]), 1);
      mbar_init(smem_u32(&empty_bar[s]), 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(smem_u32(&accf_bar[b]), 1);
      // every epilogue warp of both CTAs releases the accumulator(s)
      mbar_init(smem_u32(&acce_bar[b]), 2 * Cfg::kEpiWarps);
    }
    mbar_init(smem_u32(drain_bar), 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    if (WT == 2) tma_prefetch_desc(&tm_w2);
    tma_prefetch_desc(&tm_w);
    tma_prefetch_desc(&tm_a);
  }
  if (warp == kPairMmaWarp) {
    tmem_alloc_pair(smem_u32(tmem_slot), kPairTmemCols);
    tmem_relinquish_pair();
  }
  // Both CTAs' barriers exist before either CTA signals the other's.
  tc_fence_before();
  cluster_sync();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp < kPairLoadWarps) {
    // ------------------------------------------------------------ producers
    // no more producers than ring slots (see the host plan)
    const int P = p.producers < S ? p.producers : S;
    const int pw = warp;
    if (lane == 0 && pw < P) {
      const uint64_t pol_w = l2_policy_evict_normal();
      const uint64_t pol_a = l2_policy_evict_last();
      auto full_of = [&](int stage) { return map_to_cta(smem_u32(&full_bar[stage]), 0); };
      auto issue_weight = [&](int stage, int tile, int u) {
        // CTA r holds weight tiles (2 WT) g + WT r + h, h < WT, of group g.
        int g, mt_unused;
        pair_tile_coords(p, tile, g, mt_unused);
        const int nt0 = 2 * WT * g + WT * static_cast<int>(rank);
        const uint32_t dst = smem_u32(stage_base + stage * SB);
        // Rank 0 expects both CTAs' bytes of the stage.
        if (rank == 0) mbar_arrive_expect_tx(smem_u32(&full_bar[stage]), 2 * SB);
        if (WT == 2 && nt0 + 1 < p.n_tiles) {
          // both tiles in one copy: box (256, 40, KS, 2) -> [h][j][10 KB]
          tma_load_4d_pair(dst, &tm_w2, 0, 0, u * KS, nt0, full_of(stage), pol_w);
        } else {
#pragma unroll
          for (int h = 0; h < WT; ++h) {
            // Tiles past the end (a ragged last group) re-read the last tile;
            // their rows are >= n and never stored.
            int nt = nt0 + h;
            if (nt >= p.n_tiles) nt = p.n_tiles - 1;
            tma_load_3d_pair(dst + h * KS * kWTileBytes, &tm_w, 0, 0, nt * p.k_steps + u * KS,
                             full_of(stage), pol_w);
          }
        }
      };
      auto issue_act = [&](int stage, int tile, int u) {
        int g_unused, mt;
        pair_tile_coords(p, tile, g_unused, mt);
        tma_load_3d_pair(smem_u32(stage_base + stage * SB + Cfg::kWBytes), &tm_a, 0,
                         mt * p.bn + static_cast<int>(rank) * (p.bn / 2), u * KS,
                         full_of(stage), pol_a);
      };
      // Weights do not depend on the preceding kernel: fill the first stages
      // before waiting for it.
      long long pre_count = 0;
      for (int t = pair; t < p.tiles && pre_count < S; t += p.pairs)
        for (int u = 0; u < p.units && pre_count < S; ++u) {
          if (pre_count % P == pw) issue_weight(static_cast<int>(pre_count), t, u);
          ++pre_count;
        }
      grid_dependency_wait();
      long long i = 0;
      bool ok = true;
      for (int t = pair; ok && t < p.tiles; t += p.pairs) {
        for (int u = 0; u < p.units; ++u, ++i) {
          if (i % P != pw) continue;
          const int stage = static_cast<int>(i % S);
          if (i >= pre_count) {
            // A ring slot is reused once the MMAs of its previous use are done.
            const uint32_t phase = static_cast<uint32_t>((i / S) & 1);
            if (!mbar_wait(smem_u32(&empty_bar[stage]), phase ^ 1u, abort_flag)) {
              ok = false;
              break;
            }
            issue_weight(stage, t, u);
          }
          issue_act(stage, t, u);
        }
      }
      if (!ok && rank == 0) {
        // Let the stages this lane armed complete before the pair exits.
        const long long issued = i;
        const long long first = issued > S ? issued - S : 0;
        for (long long t2 = first; t2 < issued; ++t2) {
          if (t2 % P != pw) continue;
          volatile int no_abort = 0;
          mbar_wait(smem_u32(&full_bar[t2 % S]), static_cast<uint32_t>((t2 / S) & 1), &no_abort);
        }
      }
    }
  } else if (warp == kPairMmaWarp) {
    // ------------------------------------------------------------ MMA issuer
    // The whole warp walks the loop (converged, so its operands stay
    // warp-uniform); one elected lane issues each tcgen05 operation.
    if (rank == 0) {
      grid_dependency_wait();
      const uint32_t e_tmem = tmem_base + kPairMetaCol;
      int stage = 0;
      uint32_t phase = 0;
      const int a_tile_bytes = (p.bn / 2) * kStepK;
      int acc = 0;              // WT = 1: accumulator buffer of this tile
      uint32_t acc_phase = 0;
      bool ok = true;
      // Whether the full barrier of `stage` was already seen complete: each
      // stage tests the next one's barrier right after its first MMA, so the
      // barrier's latency overlaps queued tensor work instead of draining
      // the pipe between stages.
      bool ready = false;
      for (int t = pair; ok && t < p.tiles; t += p.pairs) {
        // The accumulator(s) are free once every epilogue warp of the pair
        // has read the tile that last used them.
        if (!mbar_wait_cluster_warp(smem_u32(&acce_bar[acc]), acc_phase ^ 1u, abort_flag)) break;
        tc_fence_after();
        for (int u = 0; u < p.units; ++u) {
          if (!ready && !mbar_wait_warp(smem_u32(&full_bar[stage]), phase, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const int next_stage = stage + 1 == S ? 0 : stage + 1;
          const uint32_t next_phase = stage + 1 == S ? phase ^ 1u : phase;
          const uint32_t st = smem_u32(stage_base + stage * SB);
#pragma unroll
          for (int j = 0; j < KS; ++j) {
            const uint32_t a_addr = st + Cfg::kWBytes + j * a_tile_bytes;
#pragma unroll
            for (int h = 0; h < WT; ++h) {
              // weight slot h, k step j: [h][j][10 KB]
              const uint32_t w_addr = st + (h * KS + j) * kWTileBytes;
              const uint32_t e_col = e_tmem + 4 * (h * KS + j);
              const uint32_t d_tmem = tmem_base + (WT == 1 ? acc : h) * kPairMaxTokens;
              // metadata of k steps j and j + 1 of this slot (consecutive tiles)
              // in one 128 x 256-bit copy
              if constexpr (KS == 1) {
                tc_cp_128x128b_pair_w(e_col, smem_desc(w_addr + kWValBytes, 0, 128, kNoSwizzle));
              } else if (j % 2 == 0) {
                tc_cp_128x256b_pair_w(e_col, smem_desc(w_addr + kWValBytes, kWTileBytes, 128,
                                                       kNoSwizzle));
              }
#pragma unroll
              for (int kh = 0; kh < 2; ++kh) {
                const uint64_t adesc = smem_desc(w_addr + 32 * kh, 16, 512, kSwizzle64);
                const uint64_t bdesc = smem_desc(a_addr + 64 * kh, 16, 1024, kSwizzle128);
                mma_sp_f8f6f4_pair_w(d_tmem, adesc, bdesc, e_col + 2 * kh, p.idesc,
                                     (u > 0 || j > 0 || kh > 0) ? 1u : 0u);
                if (j == 0 && h == 0 && kh == 0)
                  ready = mbar_test_warp(smem_u32(&full_bar[next_stage]), next_phase);
              }
            }
          }
          tc_commit_pair_mc_w(smem_u32(&empty_bar[stage]), 0x3);
          stage = next_stage;
          phase = next_phase;
        }
        if (!ok) break;
        tc_commit_pair_mc_w(smem_u32(&accf_bar[acc]), 0x3);
        if (WT == 1) {
          acc ^= 1;
          if (acc == 0) acc_phase ^= 1u;
        } else {
          acc_phase ^= 1u;
        }
      }
      tc_commit_pair_mc_w(smem_u32(drain_bar), 0x1);
      volatile int no_abort = 0;
      mbar_wait_warp(smem_u32(drain_bar), 0, &no_abort);
    }
  } else {
    // ------------------------------------------------------------ epilogue
    grid_dependency_wait();
    const int e = warp - kPairEpiWarp0;      // 0 .. 8 WT - 1
    const int q = warp % 4;                   // tensor-memory lane quadrant
    const int half = (e / 4) % 2;             // 16-column chunks half, half + 2, ...
    const int slot = e / 8;                   // weight slot (WT = 2)
    uint32_t acce_leader[2];
    for (int b = 0; b < 2; ++b) acce_leader[b] = map_to_cta(smem_u32(&acce_bar[b]), 0);
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int t = pair; t < p.tiles; t += p.pairs) {
      int g, mt;
      pair_tile_coords(p, t, g, mt);
      const int nt = 2 * WT * g + WT * static_cast<int>(rank) + slot;
      const int n = nt * kTileN + q * 32 + lane;
      const float sw = (n < p.n) ? __ldg(p.s_w + n) : 0.0f;
      const float bv = (p.bias != nullptr && n < p.n) ? __bfloat162float(p.bias[n]) : 0.0f;
      int ok = 1;
      if (lane == 0) ok = mbar_wait(smem_u32(&accf_bar[acc]), acc_phase, abort_flag) ? 1 : 0;
      ok = __shfl_sync(0xffffffffu, ok, 0);
      if (!ok) break;
      tc_fence_after();
      const uint32_t t_row = tmem_base + (static_cast<uint32_t>(q * 32) << 16) +
                             static_cast<uint32_t>((WT == 1 ? acc : slot) * kPairMaxTokens);
      const int m_tile0 = mt * p.bn;
#pragma unroll 1
      for (int c = half; c < p.bn / 16; c += 2) {
        uint32_t r[16];
        tmem_ld_32x32b_x16(t_row + c * 16, r);
        float sa[16];
        load_sa_pair(p, m_tile0 + c * 16, sa);
        tmem_ld_wait();
        if (n < p.n) {
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            const int m = m_tile0 + c * 16 + j;
            if (m < p.m)
              p.y[static_cast<long long>(m) * p.n + n] =
                  __float2bfloat16_rn(fmaf(__uint_as_float(r[j]), sa[j] * sw, bv));
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(acce_leader[acc]);
      if (WT == 1) {
        acc ^= 1;
        if (acc == 0) acc_phase ^= 1u;
      } else {
        acc_phase ^= 1u;
      }
    }
  }

  // ------------------------------------------------------------ teardown
  // Both CTAs are done with every tensor-memory access of the pair (rank 0's
  // MMAs have drained) before the pair frees it.
  tc_fence_before();
  cluster_sync();
  tc_fence_after();
  if (warp == kPairMmaWarp) tmem_dealloc_pair(tmem_base, kPairTmemCols);
}

}  // namespace sfp8

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
//   warp 0      TMA producer: per 128-wide k step, the compressed weight tile
//               (128 x 64 B, 64B swizzle), its 2 KB metadata tile (bulk copy)
//               and the activation tile (BN x 128 B, 128B swizzle) into one
//               stage of a multi-stage shared-memory ring.
//   warp 1      MMA issuer: copies the metadata tile into tensor memory
//               (tcgen05.cp 128x128b) and issues two 128 x BN x 64 sparse
//               MMAs per stage; frees the stage with tcgen05.commit.
//   warps 2-5   epilogue: tensor memory -> registers -> scale/bias/bf16 ->
//               global, or split-K partials to the workspace.
// Work split: the (tile, k step) iterations are divided evenly over the
// CTAs (stream-K).  A CTA whose range covers a tile's whole K finishes it
// directly; otherwise each part writes an fp32 partial and the last part to
// arrive (a per-tile counter) adds all parts in a fixed order and finishes
// the tile, so results do not depend on arrival order.
//
// Every wait is bounded (device_common.cuh): on a timeout the CTA records
// SFP8_DEVICE_TIMEOUT, lets its copies in flight land, frees its tensor
// memory and returns.
#pragma once

#include <cuda_bf16.h>

#include "device_common.cuh"

namespace sfp8 {

constexpr int kTileN = 128;     // weight rows per tile (MMA M)
constexpr int kStepK = 128;     // logical k per pipeline stage
constexpr int kMetaTileBytes = kTileN * kStepK / 8;   // 2048
constexpr int kWTileBytes = kTileN * kStepK / 2;      // 8192
constexpr int kGemmThreads = 192;
constexpr int kEpiThreads = 128;
constexpr int kSmemBudget = 225 * 1024;

__host__ __device__ constexpr int pow2_at_least(int v) {
  int p = 32;
  while (p < v) p <<= 1;
  return p;
}

template <int BN>
struct LinearCfg {
  static_assert(BN % 16 == 0 && BN >= 16 && BN <= 256, "BN must be 16..256, multiple of 16");
  static constexpr int kATileBytes = BN * kStepK;
  static constexpr int kStageBytes = kWTileBytes + kMetaTileBytes + kATileBytes;
  static constexpr int kNumAcc = (2 * BN + 4 <= 512) ? 2 : 1;
  static constexpr int kMetaCol = kNumAcc * BN;
  static constexpr int kTmemCols = pow2_at_least(kNumAcc * BN + 4);
  static constexpr int kBarrierBytes = 1024;
  static constexpr int kStagesMax = 16;
  static constexpr int kStages =
      ((kSmemBudget - kBarrierBytes - 1024) / kStageBytes) < kStagesMax
          ? ((kSmemBudget - kBarrierBytes - 1024) / kStageBytes)
          : kStagesMax;
  static constexpr int kSmemBytes = 1024 /*align slack*/ + kStages * kStageBytes + kBarrierBytes;
  static_assert(kStageBytes % 1024 == 0, "stages must stay 1024-byte aligned");
  static_assert(kStages >= 2, "need at least two stages");
};

struct LinearParams {
  const uint8_t* meta;
  const float* s_a;
  const float* s_w;
  const __nv_bfloat16* bias;
  __nv_bfloat16* y;
  float* partials;          // [grid][2][BN][128] fp32
  unsigned int* counters;   // [tiles][4]: one per tile and lane quadrant
  int m, n, k;
  int m_tiles;              // ceil(m / BN)
  int k_steps;              // k / 128
  long long tiles;          // n_tiles * m_tiles
  long long iters;          // tiles * k_steps
  int grid;
  uint32_t idesc;
};

// The contiguous range of (tile, k step) iterations owned by a CTA, walked
// one tile segment at a time.  All three roles walk it identically.
struct SegmentWalker {
  long long it, end;
  int k_steps;
  __device__ SegmentWalker(const LinearParams& p, int cta) {
    it = static_cast<long long>(cta) * p.iters / p.grid;
    end = static_cast<long long>(cta + 1) * p.iters / p.grid;
    k_steps = p.k_steps;
  }
  __device__ bool next(long long& tile, int& kb0, int& kb1) {
    if (it >= end) return false;
    tile = it / k_steps;
    kb0 = static_cast<int>(it % k_steps);
    const long long left = end - it;
    kb1 = static_cast<int>(left < k_steps - kb0 ? kb0 + left : k_steps);
    it += kb1 - kb0;
    return true;
  }
};

// CTA owning iteration i (the inverse of the even split).
__device__ __forceinline__ int cta_of_iter(long long i, const LinearParams& p) {
  return static_cast<int>(((i + 1) * p.grid - 1) / p.iters);
}

template <int BN>
__device__ __forceinline__ void tile_coords(const LinearParams& p, long long tile, int& nt,
                                            int& mt) {
  nt = static_cast<int>(tile / p.m_tiles);
  mt = static_cast<int>(tile % p.m_tiles);
}

// Epilogue for one 16-column chunk held in registers: y = acc*s_a*s_w + bias.
template <int BN>
__device__ __forceinline__ void store_chunk(const LinearParams& p, const float (&acc)[16],
                                            int n, int m0, float sw, float bias) {
  if (n >= p.n) return;
#pragma unroll
  for (int j = 0; j < 16; ++j) {
    const int m = m0 + j;
    if (m < p.m) {
      const float sa = __ldg(p.s_a + m);
      const float v = fmaf(acc[j], sa * sw, bias);
      p.y[static_cast<long long>(m) * p.n + n] = __float2bfloat16_rn(v);
    }
  }
}

template <int BN>
__global__ void __launch_bounds__(kGemmThreads, 1)
    sparse_linear_kernel(const __grid_constant__ CUtensorMap tm_w,
                         const __grid_constant__ CUtensorMap tm_a, const LinearParams p) {
  using Cfg = LinearCfg<BN>;
  constexpr int S = Cfg::kStages;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t* stage_base = smem;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + S * Cfg::kStageBytes);
  uint64_t* full_bar = bars;                  // [S]
  uint64_t* empty_bar = bars + S;             // [S]
  uint64_t* accf_bar = bars + 2 * S;          // [2]
  uint64_t* acce_bar = bars + 2 * S + 2;      // [2]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * S + 4);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(bars + 2 * S + 5);
  uint64_t* drain_bar = bars + 2 * S + 6;

  const int warp = threadIdx.x / 32;
  const int lane = threadIdx.x % 32;
  const int cta = blockIdx.x;

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
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tm_w);
    tma_prefetch_desc(&tm_a);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), Cfg::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      const uint64_t pol_w = l2_policy_evict_first();
      const uint64_t pol_a = l2_policy_evict_last();
      SegmentWalker walk(p, cta);
      long long tile;
      int kb0, kb1;
      int stage = 0;
      uint32_t phase = 0;
      long long issued = 0;
      // The weight does not depend on the preceding kernel: fill the first
      // stages with weight tiles before waiting for the activation.
      SegmentWalker pre(p, cta);
      int pre_stage = 0;
      long long pre_count = 0;
      {
        long long t2;
        int a0, a1;
        while (pre_count < S && pre.next(t2, a0, a1)) {
          int nt, mt;
          tile_coords<BN>(p, t2, nt, mt);
          for (int kb = a0; kb < a1 && pre_count < S; ++kb) {
            uint8_t* st = stage_base + pre_stage * Cfg::kStageBytes;
            const uint32_t fb = smem_u32(&full_bar[pre_stage]);
            mbar_arrive_expect_tx(fb, Cfg::kStageBytes);
            tma_load_2d(smem_u32(st), &tm_w, kb * (kStepK / 2), nt * kTileN, fb, pol_w);
            bulk_load(smem_u32(st + kWTileBytes),
                      p.meta + (static_cast<long long>(nt) * p.k_steps + kb) * kMetaTileBytes,
                      kMetaTileBytes, fb, pol_w);
            ++pre_stage;
            ++pre_count;
          }
        }
      }
      grid_dependency_wait();
      bool ok = true;
      while (ok && walk.next(tile, kb0, kb1)) {
        int nt, mt;
        tile_coords<BN>(p, tile, nt, mt);
        for (int kb = kb0; kb < kb1; ++kb) {
          uint8_t* st = stage_base + stage * Cfg::kStageBytes;
          const uint32_t fb = smem_u32(&full_bar[stage]);
          if (issued >= pre_count) {
            if (!mbar_wait(smem_u32(&empty_bar[stage]), phase ^ 1u, abort_flag)) {
              ok = false;
              break;
            }
            mbar_arrive_expect_tx(fb, Cfg::kStageBytes);
            tma_load_2d(smem_u32(st), &tm_w, kb * (kStepK / 2), nt * kTileN, fb, pol_w);
            bulk_load(smem_u32(st + kWTileBytes),
                      p.meta + (static_cast<long long>(nt) * p.k_steps + kb) * kMetaTileBytes,
                      kMetaTileBytes, fb, pol_w);
          }
          tma_load_2d(smem_u32(st + kWTileBytes + kMetaTileBytes), &tm_a, kb * kStepK,
                      mt * BN, fb, pol_a);
          ++issued;
          if (++stage == S) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      if (!ok) {
        // Let the copies already issued land before the CTA exits.  Stage s
        // was last filled by one of the last min(S, issued) iterations.
        long long first = issued > S ? issued - S : 0;
        for (long long i = first; i < issued; ++i) {
          const int s = static_cast<int>(i % S);
          const uint32_t ph = static_cast<uint32_t>((i / S) & 1);
          volatile int no_abort = 0;
          mbar_wait(smem_u32(&full_bar[s]), ph, &no_abort);
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      SegmentWalker walk(p, cta);
      long long tile;
      int kb0, kb1;
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      const uint32_t e_tmem = tmem_base + Cfg::kMetaCol;
      bool ok = true;
      while (ok && walk.next(tile, kb0, kb1)) {
        if (!mbar_wait(smem_u32(&acce_bar[acc]), acc_phase ^ 1u, abort_flag)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + acc * BN;
        for (int kb = kb0; kb < kb1; ++kb) {
          if (!mbar_wait(smem_u32(&full_bar[stage]), phase, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t st = smem_u32(stage_base + stage * Cfg::kStageBytes);
          const uint32_t w_addr = st;
          const uint32_t e_addr = st + kWTileBytes;
          const uint32_t a_addr = st + kWTileBytes + kMetaTileBytes;
          // metadata: 128 rows x 16 bytes, no swizzle, 8-row groups 128 B apart
          tc_cp_128x128b(e_tmem, smem_desc(e_addr, 0, 128, kNoSwizzle));
#pragma unroll
          for (int j = 0; j < 2; ++j) {
            // weight: 128 rows x 64 B (64B swizzle, 8-row atoms 512 B apart);
            // each MMA consumes 32 B of every row (64 logical k).
            const uint64_t adesc = smem_desc(w_addr + 32 * j, 16, 512, kSwizzle64);
            // activation: BN rows x 128 B (128B swizzle, atoms 1024 B apart);
            // each MMA consumes 64 B of every row.
            const uint64_t bdesc = smem_desc(a_addr + 64 * j, 16, 1024, kSwizzle128);
            mma_sp_f8f6f4(d_tmem, adesc, bdesc, e_tmem + 2 * j, p.idesc,
                          (kb > kb0 || j > 0) ? 1u : 0u);
          }
          tc_commit(smem_u32(&empty_bar[stage]));
          if (++stage == S) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        tc_commit(smem_u32(&accf_bar[acc]));
        if (Cfg::kNumAcc == 2) {
          acc ^= 1;
          if (acc == 0) acc_phase ^= 1u;
        } else {
          acc_phase ^= 1u;
        }
      }
      // Every MMA issued must have finished before tensor memory is freed.
      tc_commit(smem_u32(drain_bar));
      volatile int no_abort = 0;
      mbar_wait(smem_u32(drain_bar), 0, &no_abort);
    }
  } else {
    // ------------------------------------------------------------ epilogue
    // Each of the four warps owns 32 weight rows (its tensor-memory lane
    // quadrant) and finishes them on its own, split-K fix-up included, so no
    // barrier spans the four warps.
    grid_dependency_wait();
    const int q = warp % 4;
    SegmentWalker walk(p, cta);
    long long tile;
    int kb0, kb1;
    int acc = 0;
    uint32_t acc_phase = 0;
    long long first_tile = -1;
    while (walk.next(tile, kb0, kb1)) {
      if (first_tile < 0) first_tile = tile;
      int ok = 1;
      if (lane == 0) ok = mbar_wait(smem_u32(&accf_bar[acc]), acc_phase, abort_flag) ? 1 : 0;
      ok = __shfl_sync(0xffffffffu, ok, 0);
      if (!ok) break;
      tc_fence_after();
      int nt, mt;
      tile_coords<BN>(p, tile, nt, mt);
      const int n_local = q * 32 + lane;
      const int n = nt * kTileN + n_local;
      const bool whole = (kb0 == 0 && kb1 == p.k_steps);
      const float sw = (n < p.n) ? __ldg(p.s_w + n) : 0.0f;
      const float bv = (p.bias != nullptr && n < p.n) ? __bfloat162float(p.bias[n]) : 0.0f;
      const int slot = (tile == first_tile) ? 0 : 1;
      float* part = p.partials + (static_cast<long long>(cta) * 2 + slot) * (BN * kTileN);
      const uint32_t t_row = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + acc * BN;
#pragma unroll 1
      for (int c = 0; c < BN / 16; ++c) {
        uint32_t r[16];
        tmem_ld_32x32b_x16(t_row + c * 16, r);
        tmem_ld_wait();
        float v[16];
#pragma unroll
        for (int j = 0; j < 16; ++j) v[j] = __uint_as_float(r[j]);
        if (whole) {
          store_chunk<BN>(p, v, n, mt * BN + c * 16, sw, bv);
        } else {
#pragma unroll
          for (int j = 0; j < 16; ++j) part[(c * 16 + j) * kTileN + n_local] = v[j];
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
      if (!whole) {
        // Publish this warp's part of the split tile; the last part to
        // arrive (per tile and quadrant) adds all parts in CTA order.
        __threadfence();
        __syncwarp();
        const long long it0 = tile * p.k_steps;
        const int c_first = cta_of_iter(it0, p);
        const int c_last = cta_of_iter(it0 + p.k_steps - 1, p);
        unsigned int last = 0;
        if (lane == 0) {
          const unsigned int parts = static_cast<unsigned int>(c_last - c_first + 1);
          const unsigned int prev = atomicAdd(p.counters + tile * 4 + q, 1u);
          last = (prev + 1 == parts) ? 1u : 0u;
        }
        last = __shfl_sync(0xffffffffu, last, 0);
        if (last) {
          __threadfence();
#pragma unroll 1
          for (int c = 0; c < BN / 16; ++c) {
            float v[16];
#pragma unroll
            for (int j = 0; j < 16; ++j) v[j] = 0.0f;
            for (int cc = c_first; cc <= c_last; ++cc) {
              const long long cc_start = static_cast<long long>(cc) * p.iters / p.grid;
              const int cc_slot = (cc_start / p.k_steps == tile) ? 0 : 1;
              const float* src =
                  p.partials + (static_cast<long long>(cc) * 2 + cc_slot) * (BN * kTileN);
#pragma unroll
              for (int j = 0; j < 16; ++j) v[j] += __ldcg(src + (c * 16 + j) * kTileN + n_local);
            }
            store_chunk<BN>(p, v, n, mt * BN + c * 16, sw, bv);
          }
          if (lane == 0) p.counters[tile * 4 + q] = 0u;
        }
      }
    }
  }

  // ------------------------------------------------------------ teardown
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, Cfg::kTmemCols);
  }
}

}  // namespace sfp8

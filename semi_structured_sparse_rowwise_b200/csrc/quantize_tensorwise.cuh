// Tensor-wise FP8 quantisation: one scale for the whole tensor (page
// "[float8nocompile] Add alternate Triton kernels for FP8 conversion which
// use atomic_max-based algo instead of reduction-based algo", pytorch/ao pull
// request 1455, Summary).  The conversion rule is the row-wise one of
// quantize_rowwise.cuh with the whole tensor as the group:
//
//     amax = max over all elements |x|,  s = max(amax, 1e-12f) / FP8_MAX,
//     q    = cvt.rn.satfinite(x / s)     (x / s the correctly rounded quotient)
//
// The page finds the global amax in one of two ways: every block writes its
// partial maximum to a buffer that a second step reduces (deterministic), or
// every block folds its partial maximum into one shared word with an atomic
// max (no buffer sized by the block count).  Both are built here, as a mode
// of one kernel; a maximum is exact and independent of order, so the two
// give the same bits.
//
// One launch does both sweeps.  The grid is cooperative (all CTAs
// co-resident); CTA b owns a contiguous run of tiles (kTwThreads * kTwUnroll
// 16-byte vectors each).  Sweep 1 reads the run front to back, kTwBatch
// tiles per step, folding |x| into a CTA maximum and keeping the last
// step's tiles in registers.  The CTA then publishes its maximum (a partials
// slot, or an atomic max on the float's bits -- |x| >= 0, so the unsigned
// order of the bits is the float order) and arrives on a grid barrier in the
// workspace.  The last CTA to arrive computes the global amax (all its
// threads reduce the partials), clears what must start at zero for the next
// call and opens the barrier by bumping a generation word.  Sweep 2 converts
// the kept tiles from registers, then the rest of the run back to front, so
// that the most recently read tiles -- the ones most likely still in L2 --
// are re-read first.  The barrier wait is bounded (kWaitLimitCycles); on
// expiry the CTA records SFP8_DEVICE_TIMEOUT and converts nothing.
#pragma once

#include "quantize_rowwise.cuh"

namespace sfp8 {

constexpr int kTwThreads = 512;
constexpr int kTwUnroll = 4;       // 16-byte vectors per thread per tile
constexpr int kTwBatch = 1;        // tiles per step of either sweep (2 measured no faster)
constexpr int kTwSyncWords = 16;   // workspace header: barrier and amax words (64 bytes)

// Workspace words.  kTwArrived and kTwAtomicAmax are zero between calls
// (each call leaves them zero); kTwGeneration counts calls.
constexpr int kTwArrived = 0;
constexpr int kTwGeneration = 1;
constexpr int kTwAtomicAmax = 2;
constexpr int kTwResult = 3;

__device__ __forceinline__ uint4 ld_nc_hint(const void* p, uint64_t policy) {
  uint4 v;
  asm volatile("ld.global.nc.L2::cache_hint.v4.u32 {%0, %1, %2, %3}, [%4], %5;"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p), "l"(policy));
  return v;
}

__device__ __forceinline__ void store_release_gpu(unsigned int* addr, unsigned int v) {
  asm volatile("st.release.gpu.global.u32 [%0], %1;" ::"l"(addr), "r"(v) : "memory");
}

template <typename T>
__device__ __forceinline__ float load_scalar(const T* p);
template <>
__device__ __forceinline__ float load_scalar<__nv_bfloat16>(const __nv_bfloat16* p) {
  return __bfloat162float(*p);
}
template <>
__device__ __forceinline__ float load_scalar<__half>(const __half* p) {
  return __half2float(*p);
}
template <>
__device__ __forceinline__ float load_scalar<float>(const float* p) {
  return *p;
}

template <int kPerVec>
__device__ __forceinline__ void store_codes_streaming(uint8_t* dst, const uint32_t (&w)[kPerVec / 4]) {
  if constexpr (kPerVec == 8) {
    __stcs(reinterpret_cast<uint2*>(dst), make_uint2(w[0], w[1]));
  } else {
    __stcs(reinterpret_cast<unsigned int*>(dst), w[0]);
  }
}

// x: numel elements, 16-byte aligned; q: numel codes, 16-byte aligned.
// sync: kTwSyncWords words of workspace; partials: gridDim.x floats (the
// reduction mode only).  keep_tiles: tiles at the end of every CTA's run
// that sweep 1 reads with an evict-normal L2 policy (the rest evict-first,
// so the kept tiles outlive them in L2 until sweep 2 reads them first).
template <typename T, int kFmt, bool kAtomic>
__global__ void __launch_bounds__(kTwThreads)
    quantize_tensorwise_kernel(const T* __restrict__ x, int64_t numel, uint8_t* __restrict__ q,
                               float* __restrict__ scale, unsigned int* sync,
                               float* partials, int64_t tiles_per_cta, int64_t keep_tiles) {
  using Tr = InputTraits<T>;
  constexpr int P = Tr::kPerVec;
  constexpr int64_t kTile = static_cast<int64_t>(kTwThreads) * kTwUnroll;
  __shared__ float red[kTwThreads / 32];
  __shared__ float g_amax;
  __shared__ int failed;

  const int warp = threadIdx.x / 32;
  const int lane = threadIdx.x % 32;
  unsigned int gen = 0;
  // The generation is read before this CTA arrives, so the barrier cannot
  // have opened yet for this call.
  if (threadIdx.x == 0) gen = load_acquire_gpu(&sync[kTwGeneration]);

  const int64_t nvec = numel / P;
  const int64_t tiles = (nvec + kTile - 1) / kTile;
  const int64_t t_begin = static_cast<int64_t>(blockIdx.x) * tiles_per_cta;
  const int64_t t_end = t_begin + tiles_per_cta < tiles ? t_begin + tiles_per_cta : tiles;
  const int tail = static_cast<int>(numel - nvec * P);
  const bool tail_cta = blockIdx.x == gridDim.x - 1;

  // ---- sweep 1: CTA maximum, kTwBatch tiles per step (their loads all in
  // flight at once); the last step's tiles stay in registers
  const uint64_t pol_first = l2_policy_evict_first();
  const uint64_t pol_keep = l2_policy_evict_normal();
  uint4 v[kTwBatch * kTwUnroll];
  float amax = 0.0f;
  int64_t t_last = t_begin;           // first tile of the last step
  for (int64_t t = t_begin; t < t_end; t += kTwBatch) {
    t_last = t;
#pragma unroll
    for (int j = 0; j < kTwBatch; ++j) {
      const int64_t tt = t + j;
      const uint64_t pol = (t_end - tt) <= keep_tiles ? pol_keep : pol_first;
#pragma unroll
      for (int u = 0; u < kTwUnroll; ++u) {
        const int64_t vi = tt * kTile + u * kTwThreads + threadIdx.x;
        if (tt < t_end && vi < nvec) v[j * kTwUnroll + u] = ld_nc_hint(x + vi * P, pol);
      }
    }
#pragma unroll
    for (int j = 0; j < kTwBatch; ++j) {
      const int64_t tt = t + j;
#pragma unroll
      for (int u = 0; u < kTwUnroll; ++u) {
        const int64_t vi = tt * kTile + u * kTwThreads + threadIdx.x;
        if (tt < t_end && vi < nvec) amax = Tr::abs_max(v[j * kTwUnroll + u], amax);
      }
    }
  }
  if (tail_cta && threadIdx.x < tail)
    amax = fmaxf(amax, fabsf(load_scalar(x + nvec * P + threadIdx.x)));
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
  if (lane == 0) red[warp] = amax;
  __syncthreads();

  // ---- publish and arrive (warp 0, lane 0), then wait or finish the amax
  __shared__ unsigned int s_prev;
  if (warp == 0) {
    float m = lane < kTwThreads / 32 ? red[lane] : 0.0f;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    if (lane == 0) {
      if constexpr (kAtomic) {
        if (m > 0.0f) atomicMax(&sync[kTwAtomicAmax], __float_as_uint(m));
      } else {
        partials[blockIdx.x] = m;
      }
      // release: this CTA's partial (or atomic) before its arrival
      s_prev = atomic_add_acq_rel_gpu(&sync[kTwArrived], 1u);
    }
  }
  // orders lane 0's acquire (on the arrival) before every thread's loads below
  __syncthreads();
  const bool last = s_prev == gridDim.x - 1;
  if (last) {
    // Last to arrive: every other CTA's partial is visible.  The whole CTA
    // reduces the partials (each thread at most a few loads, issued together).
    float gm = 0.0f;
    if constexpr (kAtomic) {
      if (threadIdx.x == 0) gm = __uint_as_float(atomicExch(&sync[kTwAtomicAmax], 0u));
    } else {
      for (unsigned int i = threadIdx.x; i < gridDim.x; i += kTwThreads)
        gm = fmaxf(gm, __ldcg(&partials[i]));
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) gm = fmaxf(gm, __shfl_xor_sync(0xffffffffu, gm, o));
    if (lane == 0) red[warp] = gm;
    __syncthreads();
    if (warp == 0) {
      gm = lane < kTwThreads / 32 ? red[lane] : 0.0f;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) gm = fmaxf(gm, __shfl_xor_sync(0xffffffffu, gm, o));
      if (lane == 0) {
        sync[kTwResult] = __float_as_uint(gm);
        sync[kTwArrived] = 0u;
        store_release_gpu(&sync[kTwGeneration], gen + 1u);
        g_amax = gm;
        failed = 0;
      }
    }
  } else if (threadIdx.x == 0) {
    int fail = 0;
    const long long t0 = clock64();
    while (load_acquire_gpu(&sync[kTwGeneration]) == gen) {
      if (clock64() - t0 > kWaitLimitCycles) {
        report_device_error(SFP8_DEVICE_TIMEOUT);
        fail = 1;
        break;
      }
    }
    if (!fail) g_amax = __uint_as_float(__ldcg(&sync[kTwResult]));
    failed = fail;
  }
  __syncthreads();
  if (failed) return;

  // ---- sweep 2: convert, kept tiles first, then back to front
  const float s = __fdiv_rn(fmaxf(g_amax, kGuardAmax), Fp8Out<kFmt>::kMax);
  const float r = __frcp_rn(s);
  if (blockIdx.x == 0 && threadIdx.x == 0) *scale = s;
  auto convert = [&](const uint4& vec, int64_t vi) {
    float f[P];
    Tr::to_float(vec, f);
    uint32_t w[P / 4];
    quantize_vec<kFmt, P>(f, s, r, w);
    store_codes_streaming<P>(q + vi * P, w);
  };
  if (t_end > t_begin) {
#pragma unroll
    for (int j = 0; j < kTwBatch; ++j) {
      const int64_t tt = t_last + j;
#pragma unroll
      for (int u = 0; u < kTwUnroll; ++u) {
        const int64_t vi = tt * kTile + u * kTwThreads + threadIdx.x;
        if (tt < t_end && vi < nvec) convert(v[j * kTwUnroll + u], vi);
      }
    }
  }
  for (int64_t t = t_last - 1; t >= t_begin; t -= kTwBatch) {
#pragma unroll
    for (int j = 0; j < kTwBatch; ++j) {
      const int64_t tt = t - j;
#pragma unroll
      for (int u = 0; u < kTwUnroll; ++u) {
        const int64_t vi = tt * kTile + u * kTwThreads + threadIdx.x;
        if (tt >= t_begin && vi < nvec) v[j * kTwUnroll + u] = ld_nc_hint(x + vi * P, pol_first);
      }
    }
#pragma unroll
    for (int j = 0; j < kTwBatch; ++j) {
      const int64_t tt = t - j;
#pragma unroll
      for (int u = 0; u < kTwUnroll; ++u) {
        const int64_t vi = tt * kTile + u * kTwThreads + threadIdx.x;
        if (tt >= t_begin && vi < nvec) convert(v[j * kTwUnroll + u], vi);
      }
    }
  }
  if (tail_cta && threadIdx.x < tail) {
    const int64_t i = nvec * P + threadIdx.x;
    const float t = quotient_rn(load_scalar(x + i), s, r);
    q[i] = static_cast<uint8_t>(cvt_pair<kFmt>(t, 0.0f) & 0xffu);
  }
}

}  // namespace sfp8

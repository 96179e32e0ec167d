// Dynamic row-wise FP8 quantisation (page "Add CUTLASS-based row-wise
// scaled sparse FP8 kernel", pytorch/ao pull request 1671: the row-wise
// scaling of its title and item 1, the dynamic-activation path of item 4).
//
// Per row: amax = max |x| (fp32), s = max(amax, 1e-12f) / FP8_MAX (IEEE fp32
// division), q = cvt.rn.satfinite(x / s) where x / s is the correctly rounded
// fp32 quotient.  One HBM read of x: each group of TPR threads holds its
// whole row in registers (CHUNKS 16-byte vectors per thread), reduces the row
// amax with warp shuffles (and shared memory across warps when TPR > 32),
// then converts from the registers.  Rows too long for the register tile use
// a two-sweep variant that re-reads the row (from L2).
//
// The quotient without a division per element: t0 = x * r with r = RN(1/s)
// (the correctly rounded reciprocal), then two residual corrections with
// fused multiply-adds, e = x - t * s (exact in one fma) and t' = RN(t + e * r)
// -- Markstein's division method (P. Markstein, "Computation of elementary
// functions on the IBM RISC System/6000 processor", IBM J. Res. Develop.
// 34(1), 1990): the first correction makes t faithful, and from a faithful
// quotient and the correctly rounded reciprocal the second returns the
// correctly rounded quotient x / s whenever the residual does not underflow.
// It underflows only for quotients far below the smallest FP8 step, which
// round to a zero code either way; the sign of a zero quotient is x's.  So
// the codes are exactly those of the IEEE quotient (checked on the B200 for
// every finite bf16 and fp16 x against the scale of every finite bf16 and
// fp16 row amax, both formats, and for random fp32 x), with no branch and no
// division per element.  For 16-bit inputs the multiplies and fused
// multiply-adds run two values at a time on sm_100's packed fp32x2
// instructions.
//
// The kernels are launched as programmatic dependents: they let their own
// dependents (the GEMM) launch at once, then wait for the preceding grid to
// complete before reading x or writing q and the scales -- the preceding
// grid may be the GEMM of the previous call that still reads them.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp8.h>

#include "device_common.cuh"

namespace sfp8 {

template <typename T>
struct InputTraits;
// Per input type: widening of one 16-byte vector to floats, and the vector's
// max |value| folded into a running amax.  The 16-bit types take the max on
// packed pairs (exact: the max of the values, widened once).
template <>
struct InputTraits<__nv_bfloat16> {
  static constexpr int kPerVec = 8;
  __device__ static void to_float(const uint4& v, float (&f)[8]) {
    const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&v);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      float2 t = __bfloat1622float2(h[i]);
      f[2 * i] = t.x;
      f[2 * i + 1] = t.y;
    }
  }
  __device__ static float abs_max(const uint4& v, float amax) {
    const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&v);
    const __nv_bfloat162 m = __hmax2(__hmax2(__habs2(h[0]), __habs2(h[1])),
                                     __hmax2(__habs2(h[2]), __habs2(h[3])));
    return fmaxf(amax, fmaxf(__low2float(m), __high2float(m)));
  }
};
template <>
struct InputTraits<__half> {
  static constexpr int kPerVec = 8;
  __device__ static void to_float(const uint4& v, float (&f)[8]) {
    const __half2* h = reinterpret_cast<const __half2*>(&v);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      float2 t = __half22float2(h[i]);
      f[2 * i] = t.x;
      f[2 * i + 1] = t.y;
    }
  }
  __device__ static float abs_max(const uint4& v, float amax) {
    const __half2* h = reinterpret_cast<const __half2*>(&v);
    const __half2 m = __hmax2(__hmax2(__habs2(h[0]), __habs2(h[1])),
                              __hmax2(__habs2(h[2]), __habs2(h[3])));
    return fmaxf(amax, fmaxf(__low2float(m), __high2float(m)));
  }
};
template <>
struct InputTraits<float> {
  static constexpr int kPerVec = 4;
  __device__ static void to_float(const uint4& v, float (&f)[4]) {
    f[0] = __uint_as_float(v.x);
    f[1] = __uint_as_float(v.y);
    f[2] = __uint_as_float(v.z);
    f[3] = __uint_as_float(v.w);
  }
  __device__ static float abs_max(const uint4& v, float amax) {
    return fmaxf(fmaxf(amax, fmaxf(fabsf(__uint_as_float(v.x)), fabsf(__uint_as_float(v.y)))),
                 fmaxf(fabsf(__uint_as_float(v.z)), fabsf(__uint_as_float(v.w))));
  }
};

template <int kFmt>
struct Fp8Out;
template <>
struct Fp8Out<SFP8_E4M3> {
  static constexpr float kMax = 448.0f;
  static constexpr __nv_fp8_interpretation_t kInterp = __NV_E4M3;
};
template <>
struct Fp8Out<SFP8_E5M2> {
  static constexpr float kMax = 57344.0f;
  static constexpr __nv_fp8_interpretation_t kInterp = __NV_E5M2;
};

constexpr float kGuardAmax = 1e-12f;

// Two floats -> two FP8 codes (RNE, satfinite), first in the low byte.
template <int kFmt>
__device__ __forceinline__ uint32_t cvt_pair(float lo, float hi) {
  float2 v = make_float2(lo, hi);
  return static_cast<uint32_t>(
      __nv_cvt_float2_to_fp8x2(v, __NV_SATFINITE, Fp8Out<kFmt>::kInterp));
}

// RN(x / s) from r = RN(1/s) by two residual corrections (see above); a zero
// x gives a zero of x's sign.
__device__ __forceinline__ float quotient_rn(float x, float s, float r) {
  const float t0 = __fmul_rn(x, r);
  const float t1 = __fmaf_rn(__fmaf_rn(-t0, s, x), r, t0);
  const float t2 = __fmaf_rn(__fmaf_rn(-t1, s, x), r, t1);
  return copysignf(t2, x);
}

// The same quotient for two values at once, on the packed fp32x2 pipe of
// sm_100 (each lane an IEEE round-to-nearest multiply or fused multiply-add,
// so the results are those of quotient_rn bit for bit).  fma(t, -s, x)
// equals fma(-t, s, x) exactly (negation is exact).
__device__ __forceinline__ float2 quotient_rn2(float2 x, float2 s2n, float2 r2) {
  const float2 t0 = __fmul2_rn(x, r2);
  const float2 t1 = __ffma2_rn(__ffma2_rn(t0, s2n, x), r2, t0);
  const float2 t2 = __ffma2_rn(__ffma2_rn(t1, s2n, x), r2, t1);
  return make_float2(copysignf(t2.x, x.x), copysignf(t2.y, x.y));
}

// Quantises one 16-byte input vector (already widened to floats) into
// kPerVec codes packed little-endian; s is the row scale, r = RN(1/s).
template <int kFmt, int kPerVec>
__device__ __forceinline__ void quantize_vec(const float (&f)[kPerVec], float s, float r,
                                             uint32_t (&out)[kPerVec / 4]) {
  if constexpr (kPerVec == 8) {
    // 16-bit inputs (issue-bound): the packed quotient
    const float2 s2n = make_float2(-s, -s);
    const float2 r2 = make_float2(r, r);
#pragma unroll
    for (int w = 0; w < kPerVec / 4; ++w) {
      const float2 a = quotient_rn2(make_float2(f[4 * w], f[4 * w + 1]), s2n, r2);
      const float2 b = quotient_rn2(make_float2(f[4 * w + 2], f[4 * w + 3]), s2n, r2);
      out[w] = cvt_pair<kFmt>(a.x, a.y) | (cvt_pair<kFmt>(b.x, b.y) << 16);
    }
  } else {
    // fp32 inputs (bound by HBM; measured faster with the scalar form)
#pragma unroll
    for (int w = 0; w < kPerVec / 4; ++w) {
      float t[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) t[i] = quotient_rn(f[4 * w + i], s, r);
      out[w] = cvt_pair<kFmt>(t[0], t[1]) | (cvt_pair<kFmt>(t[2], t[3]) << 16);
    }
  }
}

template <int kPerVec>
__device__ __forceinline__ void store_codes(uint8_t* dst, const uint32_t (&w)[kPerVec / 4]) {
  if constexpr (kPerVec == 8) {
    *reinterpret_cast<uint2*>(dst) = make_uint2(w[0], w[1]);
  } else {
    *reinterpret_cast<uint32_t*>(dst) = w[0];
  }
}

// Max over the TPR threads of a row group (TPR a power of two); `red` is
// shared scratch of blockDim/32 floats.
template <int TPR>
__device__ __forceinline__ float row_group_max(float v, float* red) {
#pragma unroll
  for (int o = (TPR < 32 ? TPR : 32) / 2; o > 0; o >>= 1)
    v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  if constexpr (TPR > 32) {
    const int warp = threadIdx.x / 32;
    const int lane = threadIdx.x % 32;
    constexpr int kWarps = TPR / 32;
    if (lane == 0) red[warp] = v;
    __syncthreads();
    const int first = (warp / kWarps) * kWarps;
    float m = red[first];
#pragma unroll
    for (int i = 1; i < kWarps; ++i) m = fmaxf(m, red[first + i]);
    __syncthreads();
    v = m;
  }
  return v;
}

// Register-resident row quantiser: blockDim = max(TPR, 256) threads,
// blockDim / TPR rows per block.  q2, when not null, receives a second copy
// of the codes (same row stride).
template <typename T, int kFmt, int TPR, int CHUNKS>
__global__ void __launch_bounds__(TPR > 256 ? TPR : 256)
    quantize_rowwise_kernel(const T* __restrict__ x, int64_t rows, int64_t cols,
                            int64_t ld, uint8_t* __restrict__ q, float* __restrict__ scales,
                            uint8_t* __restrict__ q2) {
  grid_dependents_launch();
  grid_dependency_wait();
  using Tr = InputTraits<T>;
  constexpr int P = Tr::kPerVec;
  __shared__ float red[32];
  const int rows_per_block = blockDim.x / TPR;
  const int64_t row = static_cast<int64_t>(blockIdx.x) * rows_per_block + threadIdx.x / TPR;
  const int t = threadIdx.x % TPR;
  const bool row_ok = row < rows;
  const int64_t nvec = cols / P;
  const T* xr = x + (row_ok ? row : 0) * ld;

  uint4 v[CHUNKS];
  float amax = 0.0f;
#pragma unroll
  for (int c = 0; c < CHUNKS; ++c) {
    const int64_t vi = static_cast<int64_t>(c) * TPR + t;
    if (row_ok && vi < nvec) {
      v[c] = __ldg(reinterpret_cast<const uint4*>(xr + vi * P));
      amax = Tr::abs_max(v[c], amax);
    }
  }
  amax = row_group_max<TPR>(amax, red);
  const float s = __fdiv_rn(fmaxf(amax, kGuardAmax), Fp8Out<kFmt>::kMax);
  const float r = __frcp_rn(s);
  if (!row_ok) return;
  if (t == 0) scales[row] = s;
  uint8_t* qr = q + row * cols;
  uint8_t* qr2 = q2 != nullptr ? q2 + row * cols : nullptr;
#pragma unroll
  for (int c = 0; c < CHUNKS; ++c) {
    const int64_t vi = static_cast<int64_t>(c) * TPR + t;
    if (vi < nvec) {
      float f[P];
      Tr::to_float(v[c], f);
      uint32_t w[P / 4];
      quantize_vec<kFmt, P>(f, s, r, w);
      store_codes<P>(qr + vi * P, w);
      if (qr2 != nullptr) store_codes<P>(qr2 + vi * P, w);
    }
  }
}

// Streaming quantiser for rows of up to 48 KB: one persistent CTA per SM.
// Lane 0 of warp 0 streams the CTA's rows (rows b, b + grid, ...) into a
// ring of `slots` shared-memory row buffers, one bulk copy per row; consumer
// warp c (of `consumers`) owns ring slots c, c + consumers, ... (slots is a
// multiple of consumers, so every slot has one consumer and no wait can run
// two phases ahead).  A consumer reads its row from shared memory twice
// (amax, then convert) and writes the codes straight to global memory.  The
// ring keeps slots x row bytes in flight per SM whatever the registers.
constexpr int kQuantMaxConsumers = 24;
constexpr int kQuantMaxSlots = 24;
constexpr int kQuantThreads = 32 * (1 + kQuantMaxConsumers);

template <typename T, int kFmt>
__global__ void __launch_bounds__(kQuantThreads, 1)
    quantize_rowwise_stream_kernel(const T* __restrict__ x, int64_t rows, int64_t cols,
                                   int64_t ld, uint8_t* __restrict__ q,
                                   float* __restrict__ scales, int slots, int consumers) {
  grid_dependents_launch();
  using Tr = InputTraits<T>;
  constexpr int P = Tr::kPerVec;
  extern __shared__ __align__(128) uint8_t qsmem[];
  const int row_bytes = static_cast<int>(cols) * static_cast<int>(sizeof(T));
  uint64_t* full = reinterpret_cast<uint64_t*>(qsmem + static_cast<size_t>(slots) * row_bytes);
  uint64_t* empty = full + kQuantMaxSlots;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(empty + kQuantMaxSlots);
  const int warp = threadIdx.x / 32;
  const int lane = threadIdx.x % 32;
  if (threadIdx.x == 0) {
    for (int i = 0; i < slots; ++i) {
      mbar_init(smem_u32(&full[i]), 1);
      mbar_init(smem_u32(&empty[i]), 1);
    }
    *abort_flag = 0;
    fence_barrier_init();
  }
  __syncthreads();
  grid_dependency_wait();
  const int64_t my_rows = rows > blockIdx.x ? (rows - 1 - blockIdx.x) / gridDim.x + 1 : 0;
  if (warp == 0) {
    if (lane == 0) {
      const uint64_t pol = l2_policy_evict_first();
      for (int64_t j = 0; j < my_rows; ++j) {
        const int slot = static_cast<int>(j % slots);
        if (j >= slots &&
            !mbar_wait(smem_u32(&empty[slot]), static_cast<uint32_t>(((j / slots) - 1) & 1),
                       abort_flag))
          break;
        const int64_t row = blockIdx.x + j * gridDim.x;
        mbar_arrive_expect_tx(smem_u32(&full[slot]), row_bytes);
        bulk_load(smem_u32(qsmem + static_cast<size_t>(slot) * row_bytes), x + row * ld,
                  row_bytes, smem_u32(&full[slot]), pol);
      }
    }
  } else if (warp - 1 < consumers) {
    const int c = warp - 1;
    const int nvec = static_cast<int>(cols) / P;
    for (int64_t j = c; j < my_rows; j += consumers) {
      const int slot = static_cast<int>(j % slots);
      // every lane waits: the barrier's completion is what makes the copied
      // row visible to the lane that reads it
      const bool ok =
          mbar_wait(smem_u32(&full[slot]), static_cast<uint32_t>((j / slots) & 1), abort_flag);
      if (!__all_sync(0xffffffffu, ok)) break;
      const uint4* src = reinterpret_cast<const uint4*>(qsmem + static_cast<size_t>(slot) * row_bytes);
      float amax = 0.0f;
      for (int vi = lane; vi < nvec; vi += 32) amax = Tr::abs_max(src[vi], amax);
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
      const float s = __fdiv_rn(fmaxf(amax, kGuardAmax), Fp8Out<kFmt>::kMax);
      const float r = __frcp_rn(s);
      const int64_t row = blockIdx.x + j * gridDim.x;
      if (lane == 0) scales[row] = s;
      uint8_t* qr = q + row * cols;
      for (int vi = lane; vi < nvec; vi += 32) {
        float f[P];
        Tr::to_float(src[vi], f);
        uint32_t w[P / 4];
        quantize_vec<kFmt, P>(f, s, r, w);
        store_codes<P>(qr + static_cast<int64_t>(vi) * P, w);
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&empty[slot]));
    }
  }
}

// Long rows: one block of 1024 threads per row, two sweeps over the row.
template <typename T, int kFmt>
__global__ void __launch_bounds__(1024)
    quantize_rowwise_long_kernel(const T* __restrict__ x, int64_t rows, int64_t cols,
                                 int64_t ld, uint8_t* __restrict__ q,
                                 float* __restrict__ scales) {
  grid_dependents_launch();
  grid_dependency_wait();
  using Tr = InputTraits<T>;
  constexpr int P = Tr::kPerVec;
  __shared__ float red[32];
  const int64_t row = blockIdx.x;
  const T* xr = x + row * ld;
  const int64_t nvec = cols / P;
  float amax = 0.0f;
  for (int64_t vi = threadIdx.x; vi < nvec; vi += blockDim.x) {
    amax = Tr::abs_max(__ldg(reinterpret_cast<const uint4*>(xr + vi * P)), amax);
  }
  amax = row_group_max<1024>(amax, red);
  const float s = __fdiv_rn(fmaxf(amax, kGuardAmax), Fp8Out<kFmt>::kMax);
  const float r = __frcp_rn(s);
  if (threadIdx.x == 0) scales[row] = s;
  uint8_t* qr = q + row * cols;
  for (int64_t vi = threadIdx.x; vi < nvec; vi += blockDim.x) {
    uint4 v = __ldg(reinterpret_cast<const uint4*>(xr + vi * P));
    float f[P];
    Tr::to_float(v, f);
    uint32_t w[P / 4];
    quantize_vec<kFmt, P>(f, s, r, w);
    store_codes<P>(qr + vi * P, w);
  }
}

// cols == 0: only the guard scale is written.
template <int kFmt>
__global__ void quantize_empty_rows_kernel(int64_t rows, float* __restrict__ scales) {
  grid_dependents_launch();
  grid_dependency_wait();
  const int64_t r = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (r < rows) scales[r] = __fdiv_rn(kGuardAmax, Fp8Out<kFmt>::kMax);
}

}  // namespace sfp8

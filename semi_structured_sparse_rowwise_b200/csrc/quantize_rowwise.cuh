// Dynamic row-wise FP8 quantisation (page "Add CUTLASS-based row-wise
// scaled sparse FP8 kernel", pytorch/ao pull request 1671: the row-wise
// scaling of its title and item 1, the dynamic-activation path of item 4).
//
// Per row: amax = max |x| (fp32), s = max(amax, 1e-12f) / FP8_MAX (IEEE fp32
// division), q = cvt.rn.satfinite(x / s) with an IEEE fp32 division per
// element.  One HBM read of x: each group of TPR threads holds its whole row
// in registers (CHUNKS 16-byte vectors per thread), reduces the row amax
// with warp shuffles (and shared memory across warps when TPR > 32), then
// converts from the registers.  Rows too long for the register tile use a
// two-sweep variant that re-reads the row (from L2).
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

// Quantises one 16-byte input vector (already widened to floats) into
// kPerVec codes packed little-endian.
template <int kFmt, int kPerVec>
__device__ __forceinline__ void quantize_vec(const float (&f)[kPerVec], float s,
                                             uint32_t (&out)[kPerVec / 4]) {
#pragma unroll
  for (int w = 0; w < kPerVec / 4; ++w) {
    const float a = __fdiv_rn(f[4 * w + 0], s);
    const float b = __fdiv_rn(f[4 * w + 1], s);
    const float c = __fdiv_rn(f[4 * w + 2], s);
    const float d = __fdiv_rn(f[4 * w + 3], s);
    out[w] = cvt_pair<kFmt>(a, b) | (cvt_pair<kFmt>(c, d) << 16);
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
// blockDim / TPR rows per block.
template <typename T, int kFmt, int TPR, int CHUNKS>
__global__ void __launch_bounds__(TPR > 256 ? TPR : 256)
    quantize_rowwise_kernel(const T* __restrict__ x, int64_t rows, int64_t cols,
                            int64_t ld, uint8_t* __restrict__ q, float* __restrict__ scales) {
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
      float f[P];
      Tr::to_float(v[c], f);
#pragma unroll
      for (int i = 0; i < P; ++i) amax = fmaxf(amax, fabsf(f[i]));
    }
  }
  amax = row_group_max<TPR>(amax, red);
  const float s = __fdiv_rn(fmaxf(amax, kGuardAmax), Fp8Out<kFmt>::kMax);
  if (!row_ok) return;
  if (t == 0) scales[row] = s;
  uint8_t* qr = q + row * cols;
#pragma unroll
  for (int c = 0; c < CHUNKS; ++c) {
    const int64_t vi = static_cast<int64_t>(c) * TPR + t;
    if (vi < nvec) {
      float f[P];
      Tr::to_float(v[c], f);
      uint32_t w[P / 4];
      quantize_vec<kFmt, P>(f, s, w);
      store_codes<P>(qr + vi * P, w);
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
    uint4 v = __ldg(reinterpret_cast<const uint4*>(xr + vi * P));
    float f[P];
    Tr::to_float(v, f);
#pragma unroll
    for (int i = 0; i < P; ++i) amax = fmaxf(amax, fabsf(f[i]));
  }
  amax = row_group_max<1024>(amax, red);
  const float s = __fdiv_rn(fmaxf(amax, kGuardAmax), Fp8Out<kFmt>::kMax);
  if (threadIdx.x == 0) scales[row] = s;
  uint8_t* qr = q + row * cols;
  for (int64_t vi = threadIdx.x; vi < nvec; vi += blockDim.x) {
    uint4 v = __ldg(reinterpret_cast<const uint4*>(xr + vi * P));
    float f[P];
    Tr::to_float(v, f);
    uint32_t w[P / 4];
    quantize_vec<kFmt, P>(f, s, w);
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

// 2:4 pruning, compression and decompression kernels.
//
// Page "Add CUTLASS-based row-wise scaled sparse FP8 kernel" (pytorch/ao pull
// request 1671): item 1's converter of FP8 data to the compressed 2:4 format,
// with item 3's rule that -0.0 counts as zero.  The selection is integer-only:
// for finite FP8 codes (and finite bf16/fp16/fp32 bit patterns) the value of
// `bits & ~sign` grows with |value|, and -0.0 has magnitude bits 0.
//
// In a group with magnitudes m0..m3, element j is kept iff fewer than two
// elements beat it, where i beats j when m_i > m_j, or m_i == m_j and i < j
// (ties to the lower index).
//
// Compressed layout (version 3), for an [n, k] weight, n_pad = ceil(n/128)*128:
// one buffer of 10240-byte tiles, tile t = nt*(k/128) + kt (weight rows
// 128nt.., k columns 128kt..) at byte 10240*t:
//   bytes 0..8191: kept values; row r at 64*r holds the row's 64 kept codes
//   (two per group, lower index first) as four 16-byte chunks, chunk c stored
//   at position c ^ ((r >> 1) & 3) -- the 64-byte swizzle that the tensor
//   core's shared-memory descriptor expects.
//   bytes 8192..10239: index metadata; row r at 8192 + 16*r, byte b = nibbles
//   of groups 2b (bits 0..3) and 2b+1 (bits 4..7) of the tile's 32 groups --
//   exactly the 128-lane x 128-bit block the GEMM copies into tensor memory.
//   Padding rows: 0x00 values, nibble 0x4.
// A pipeline stage of the GEMM is therefore one contiguous copy.
#pragma once

#include "device_common.cuh"

namespace sfp8 {

// Keep mask (bit j set = element j kept) from four magnitudes.
__device__ __forceinline__ uint32_t keep_mask4(uint32_t m0, uint32_t m1, uint32_t m2,
                                               uint32_t m3) {
  // beats[i][j]: i beats j
  const uint32_t b01 = m0 >= m1, b02 = m0 >= m2, b03 = m0 >= m3;  // i < j: ties to i
  const uint32_t b12 = m1 >= m2, b13 = m1 >= m3, b23 = m2 >= m3;
  // number of elements beating j
  const uint32_t r0 = (1 - b01) + (1 - b02) + (1 - b03);
  const uint32_t r1 = b01 + (1 - b12) + (1 - b13);
  const uint32_t r2 = b02 + b12 + (1 - b23);
  const uint32_t r3 = b03 + b13 + b23;
  return (r0 < 2 ? 1u : 0u) | (r1 < 2 ? 2u : 0u) | (r2 < 2 ? 4u : 0u) | (r3 < 2 ? 8u : 0u);
}

// Kept indices i0 < i1 from a 4-bit mask with exactly two bits set.
__device__ __forceinline__ void kept_indices(uint32_t mask, uint32_t& i0, uint32_t& i1) {
  i0 = __ffs(mask) - 1;
  i1 = __ffs(mask & (mask - 1)) - 1;
}

// ---------------------------------------------------------------- prune

template <typename Bits>
struct PruneTraits;
template <>
struct PruneTraits<uint16_t> {
  static constexpr uint32_t kMag = 0x7FFFu;
};
template <>
struct PruneTraits<uint32_t> {
  static constexpr uint32_t kMag = 0x7FFFFFFFu;
};

// One 16-byte vector per thread: 2 groups of 16-bit elements or 1 group of
// 32-bit elements.  Dropped elements become +0.0 (all bits zero).
template <typename Bits>
__global__ void prune24_kernel(const Bits* __restrict__ w, int64_t rows, int64_t cols,
                               int64_t ld, Bits* __restrict__ out) {
  constexpr int kPer = 16 / sizeof(Bits);
  const int64_t vec_per_row = cols / kPer;
  const int64_t total = rows * vec_per_row;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < total;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t r = i / vec_per_row;
    const int64_t c = (i % vec_per_row) * kPer;
    uint4 v = *reinterpret_cast<const uint4*>(w + r * ld + c);
    Bits e[kPer];
    *reinterpret_cast<uint4*>(e) = v;
#pragma unroll
    for (int g = 0; g < kPer / 4; ++g) {
      const uint32_t M = PruneTraits<Bits>::kMag;
      const uint32_t keep = keep_mask4(e[4 * g] & M, e[4 * g + 1] & M, e[4 * g + 2] & M,
                                       e[4 * g + 3] & M);
#pragma unroll
      for (int j = 0; j < 4; ++j)
        if (!((keep >> j) & 1)) e[4 * g + j] = 0;
    }
    *reinterpret_cast<uint4*>(out + r * cols + c) = *reinterpret_cast<uint4*>(e);
  }
}

// ---------------------------------------------------------------- compress

// The rank rule on a 4-code group, four bytes at a time.  With magnitudes
// m_i = code_i & 0x7F (7 bits), the byte (0x80 | m_x) - m_y needs no borrow and
// has its top bit set iff m_x >= m_y.  Two such subtractions per pair of groups
// give the six comparisons of each group (i beats j for i < j iff m_i >= m_j),
// and a 64-entry table indexed by those six bits gives the byte selector of the
// two kept codes and their index nibble.
//
// Table index bits: 0: m0>=m1, 1: m0>=m2, 2: m0>=m3, 3: m1>=m2, 4: m1>=m3, 5: m2>=m3.
// Entry for the first group of a pair:  byte selector i0 | i1 << 4 in bits 0..7,
//   nibble in bits 16..19.
// Entry for the second group: byte selector (4 + i0) | (4 + i1) << 4 in bits 8..15,
//   nibble in bits 20..23.
__device__ __forceinline__ void group_select_entries(uint32_t idx, uint32_t& first,
                                                     uint32_t& second) {
  const uint32_t b01 = idx & 1, b02 = (idx >> 1) & 1, b03 = (idx >> 2) & 1;
  const uint32_t b12 = (idx >> 3) & 1, b13 = (idx >> 4) & 1, b23 = (idx >> 5) & 1;
  const uint32_t beaten0 = (1 - b01) + (1 - b02) + (1 - b03);
  const uint32_t beaten1 = b01 + (1 - b12) + (1 - b13);
  const uint32_t beaten2 = b02 + b12 + (1 - b23);
  const uint32_t beaten3 = b03 + b13 + b23;
  const uint32_t keep = (beaten0 < 2 ? 1u : 0u) | (beaten1 < 2 ? 2u : 0u) |
                        (beaten2 < 2 ? 4u : 0u) | (beaten3 < 2 ? 8u : 0u);
  uint32_t i0 = 0, i1 = 1;
  if (__popc(keep) == 2) kept_indices(keep, i0, i1);   // always, for real comparisons
  const uint32_t nib = i0 | (i1 << 2);
  first = i0 | (i1 << 4) | (nib << 16);
  second = ((4 + i0) << 8) | ((4 + i1) << 12) | (nib << 20);
}

// Top bits of the four bytes of d, gathered into bits 28..31 (byte 0's in bit
// 28).  The partial products land on distinct bit positions, so nothing carries.
__device__ __forceinline__ uint32_t byte_signs_high(uint32_t d) {
  return (d & 0x80808080u) * 0x00204081u;
}

// Block = 512 threads = 128 rows x 4 threads; blockIdx.x covers kCompressTiles
// k tiles, blockIdx.y = row tile.  For each of its k tiles a thread turns 32
// input codes (8 groups) into 16 value bytes and 4 metadata bytes; all its
// loads are issued before the first group is selected.
constexpr int kCompressTiles = 2;

__global__ void __launch_bounds__(512)
    compress24_kernel(const uint8_t* __restrict__ wq, int64_t n, int64_t k,
                      uint8_t* __restrict__ packed) {
  __shared__ uint32_t tab_first[64], tab_second[64];
  if (threadIdx.x < 64) group_select_entries(threadIdx.x, tab_first[threadIdx.x],
                                             tab_second[threadIdx.x]);
  __syncthreads();
  const int r = threadIdx.x / 4;   // row inside the tile
  const int j = threadIdx.x % 4;   // 32-code chunk inside the 128-wide k tile
  const int64_t nt = blockIdx.y;
  const int64_t row = nt * 128 + r;
  const int64_t ktiles = k / 128;
  const int64_t kt0 = static_cast<int64_t>(blockIdx.x) * kCompressTiles;
  uint32_t in[kCompressTiles][8];
#pragma unroll
  for (int t = 0; t < kCompressTiles; ++t) {
    if (row < n && kt0 + t < ktiles) {
      const uint8_t* src = wq + row * k + (kt0 + t) * 128 + 32 * j;
      *reinterpret_cast<uint4*>(&in[t][0]) = __ldg(reinterpret_cast<const uint4*>(src));
      *reinterpret_cast<uint4*>(&in[t][4]) = __ldg(reinterpret_cast<const uint4*>(src + 16));
    } else {
#pragma unroll
      for (int g = 0; g < 8; ++g) in[t][g] = 0;   // all-zero groups select (0, 1): nibble 0x4
    }
  }
#pragma unroll
  for (int t = 0; t < kCompressTiles; ++t) {
    if (kt0 + t >= ktiles) break;
    uint32_t vout[4];
    uint32_t mout = 0;
#pragma unroll
    for (int p = 0; p < 4; ++p) {
      const uint32_t wa = in[t][2 * p], wb = in[t][2 * p + 1];
      const uint32_t la = wa & 0x7F7F7F7Fu, lb = wb & 0x7F7F7F7Fu;
      const uint32_t ha = wa | 0x80808080u, hb = wb | 0x80808080u;
      // bytes (m0>=m1, m0>=m2, m0>=m3, m1>=m2) of each group
      const uint32_t da = __byte_perm(ha, 0, 0x1000) - __byte_perm(la, 0, 0x2321);
      const uint32_t db = __byte_perm(hb, 0, 0x1000) - __byte_perm(lb, 0, 0x2321);
      // bytes (a: m1>=m3, m2>=m3; b: m1>=m3, m2>=m3)
      const uint32_t d2 = __byte_perm(ha, hb, 0x6521) - __byte_perm(la, lb, 0x7733);
      const uint32_t s2 = byte_signs_high(d2) >> 24;   // bits 4..7
      const uint32_t ia = (byte_signs_high(da) >> 28) | (s2 & 0x30u);
      const uint32_t ib = (byte_signs_high(db) >> 28) | ((s2 >> 2) & 0x30u);
      const uint32_t e = tab_first[ia] | tab_second[ib];
      vout[p] = __byte_perm(wa, wb, e & 0xFFFFu);
      mout |= (e >> 16) << (8 * p);
    }
    uint8_t* tile = packed + (nt * ktiles + kt0 + t) * 10240;
    *reinterpret_cast<uint4*>(tile + 64 * r + 16 * (j ^ ((r >> 1) & 3))) =
        make_uint4(vout[0], vout[1], vout[2], vout[3]);
    *reinterpret_cast<uint32_t*>(tile + 8192 + 16 * r + 4 * j) = mout;
  }
}

// Inverse: same thread mapping, n real rows only.
__global__ void __launch_bounds__(512)
    decompress24_kernel(const uint8_t* __restrict__ packed, int64_t n, int64_t k,
                        uint8_t* __restrict__ wq) {
  const int r = threadIdx.x / 4;
  const int j = threadIdx.x % 4;
  const int64_t kt = blockIdx.x;
  const int64_t nt = blockIdx.y;
  const int64_t row = nt * 128 + r;
  if (row >= n) return;
  const int64_t ktiles = k / 128;
  const uint8_t* tile = packed + (nt * ktiles + kt) * 10240;
  const uint4 vv = *reinterpret_cast<const uint4*>(tile + 64 * r + 16 * (j ^ ((r >> 1) & 3)));
  const uint32_t mm = *reinterpret_cast<const uint32_t*>(tile + 8192 + 16 * r + 4 * j);
  const uint32_t vw[4] = {vv.x, vv.y, vv.z, vv.w};
  uint32_t out[8];
  bool bad = false;
#pragma unroll
  for (int g = 0; g < 8; ++g) {
    const uint32_t nib = (mm >> (4 * g)) & 0xF;
    const uint32_t i0 = nib & 3, i1 = nib >> 2;
    if (i0 >= i1) bad = true;
    const uint32_t v0 = (vw[g / 2] >> (16 * (g % 2))) & 0xFF;
    const uint32_t v1 = (vw[g / 2] >> (16 * (g % 2) + 8)) & 0xFF;
    out[g] = (v0 << (8 * i0)) | (i1 > i0 ? (v1 << (8 * i1)) : 0);
  }
  if (bad) report_device_error(SFP8_DEVICE_CHECK_FAIL);
  uint8_t* dst = wq + row * k + kt * 128 + 32 * j;
  *reinterpret_cast<uint4*>(dst) = make_uint4(out[0], out[1], out[2], out[3]);
  *reinterpret_cast<uint4*>(dst + 16) = make_uint4(out[4], out[5], out[6], out[7]);
}

}  // namespace sfp8

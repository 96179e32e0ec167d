// One-pass weight preparation: 2:4 magnitude prune, row-wise FP8
// quantisation and compression into the GEMM's tile layout.
//
// Page "Add CUTLASS-based row-wise scaled sparse FP8 kernel" (pytorch/ao
// pull request 1671): item 4 prepares the weight once, when the layer is
// quantised -- row-wise FP8 codes with one scale per output row, then item
// 1's conversion to the compressed 2:4 format.  The output is bit for bit
// that of the three separate steps (prune24_kernel, then the row-wise
// quantiser, then compress24_kernel):
//
//   * the prune keeps, per group of four, the two largest |w| (ties to the
//     lower index) -- always including the group's largest, so the pruned
//     row's amax is the input row's amax and one pass over the row gives the
//     scale before anything is pruned;
//   * only the two kept values are quantised (a dropped +0.0 is code 0x00);
//   * the compressor's selection on the four codes keeps the same two slots
//     unless a kept value quantised to a zero code; then the rank rule runs
//     on the codes (dropped slots 0x00), as the separate compressor would.
//
// One warp per weight row: the row's amax first, then the row's 64 value
// bytes and 16 metadata bytes of every k tile (the kernel below says how the
// row is held).  Rows n .. n_pad-1 of the last tile get the compressor's
// padding.
#pragma once

#include "quantize_rowwise.cuh"
#include "sparse24_pack.cuh"

namespace sfp8 {

// Per input type: the four magnitudes of a group (integer patterns that grow
// with |value| for finite inputs, -0.0 -> 0) and the two kept values widened
// to floats.  A group is 4 elements = kGroupWords 32-bit words.
template <typename T>
struct PrepGroup;
template <>
struct PrepGroup<__nv_bfloat16> {
  static constexpr int kGroupWords = 2;
  __device__ static void mags(const uint32_t* w, uint32_t (&m)[4]) {
    m[0] = w[0] & 0x7FFFu;
    m[1] = (w[0] >> 16) & 0x7FFFu;
    m[2] = w[1] & 0x7FFFu;
    m[3] = (w[1] >> 16) & 0x7FFFu;
  }
  // e: the prune-table entry (bits 0..15 gather the kept elements' bytes)
  __device__ static void kept(const uint32_t* w, uint32_t e, float& f0, float& f1) {
    const uint32_t p = __byte_perm(w[0], w[1], e);
    f0 = __uint_as_float(p << 16);
    f1 = __uint_as_float(p & 0xFFFF0000u);
  }
};
template <>
struct PrepGroup<__half> {
  static constexpr int kGroupWords = 2;
  __device__ static void mags(const uint32_t* w, uint32_t (&m)[4]) {
    PrepGroup<__nv_bfloat16>::mags(w, m);
  }
  __device__ static void kept(const uint32_t* w, uint32_t e, float& f0, float& f1) {
    const uint32_t p = __byte_perm(w[0], w[1], e);
    const __half2 h = *reinterpret_cast<const __half2*>(&p);
    f0 = __low2float(h);
    f1 = __high2float(h);
  }
};
template <>
struct PrepGroup<float> {
  static constexpr int kGroupWords = 4;
  __device__ static void mags(const uint32_t* w, uint32_t (&m)[4]) {
#pragma unroll
    for (int i = 0; i < 4; ++i) m[i] = w[i] & 0x7FFFFFFFu;
  }
  __device__ static void kept(const uint32_t* w, uint32_t e, float& f0, float& f1) {
    const uint32_t i0 = (e >> 20) & 3u, i1 = (e >> 22) & 3u;   // i0 in {0, 1, 2}, i1 in {1, 2, 3}
    f0 = __uint_as_float(i0 == 0 ? w[0] : (i0 == 1 ? w[1] : w[2]));
    f1 = __uint_as_float(i1 == 3 ? w[3] : (i1 == 2 ? w[2] : w[1]));
  }
};

// Prune table: for the six comparison bits of a group (bit order of
// group_select_entries), the byte selector that gathers the two kept 16-bit
// elements of the group's 8 bytes (bits 0..15), the index nibble (bits
// 16..19), i0 (bits 20..21) and i1 (bits 22..23).
__device__ __forceinline__ uint32_t prune_entry(uint32_t idx) {
  uint32_t first, second;
  group_select_entries(idx, first, second);
  const uint32_t i0 = first & 3u, i1 = (first >> 4) & 3u;
  const uint32_t sel16 = (0x10u + 0x22u * i0) | ((0x10u + 0x22u * i1) << 8);
  return sel16 | (first & 0xF0000u) | (i0 << 20) | (i1 << 22);
}

constexpr int kPrepWarps = 8;   // rows in flight per block (one per warp)

// A kept value became a zero code: the compressor's selection on the four
// codes of every group of the chunk (dropped slots hold 0x00).  Rare, and
// kept out of line so that the unrolled chunk loop stays small in the
// instruction cache.
__device__ __noinline__ void reselect_on_codes(uint32_t (&vals)[4], uint32_t& meta) {
  for (int g = 0; g < 8; ++g) {
    const uint32_t half = (vals[g / 2] >> (16 * (g % 2))) & 0xFFFFu;
    const uint32_t nib = (meta >> (4 * g)) & 0xFu;
    const uint32_t i0 = nib & 3u, i1 = nib >> 2;
    // the group's four codes as one word: c0 at byte i0, c1 at byte i1
    const uint32_t word = ((half & 0xFFu) << (8 * i0)) | ((half >> 8) << (8 * i1));
    const uint32_t keep = keep_mask4(word & 0x7Fu, (word >> 8) & 0x7Fu, (word >> 16) & 0x7Fu,
                                     (word >> 24) & 0x7Fu);
    uint32_t j0, j1;
    kept_indices(keep, j0, j1);
    const uint32_t v = ((word >> (8 * j0)) & 0xFFu) | (((word >> (8 * j1)) & 0xFFu) << 8);
    vals[g / 2] = (vals[g / 2] & ~(0xFFFFu << (16 * (g % 2)))) | (v << (16 * (g % 2)));
    meta = (meta & ~(0xFu << (4 * g))) | ((j0 | (j1 << 2)) << (4 * g));
  }
}

// Quantises and compresses one 32-element chunk (8 groups) held in `in`.
template <typename T, int kFmt>
__device__ __forceinline__ void prepare_chunk(const uint32_t* in, const uint32_t* tab, float s,
                                              float rcp, uint32_t (&vals)[4], uint32_t& meta) {
  using G = PrepGroup<T>;
  vals[0] = vals[1] = vals[2] = vals[3] = 0;
  meta = 0;
  bool zero_code = false;
#pragma unroll
  for (int g = 0; g < 8; ++g) {
    const uint32_t* gw = &in[g * G::kGroupWords];
    uint32_t m[4];
    G::mags(gw, m);
    const uint32_t idx = (m[0] >= m[1] ? 1u : 0u) | (m[0] >= m[2] ? 2u : 0u) |
                         (m[0] >= m[3] ? 4u : 0u) | (m[1] >= m[2] ? 8u : 0u) |
                         (m[1] >= m[3] ? 16u : 0u) | (m[2] >= m[3] ? 32u : 0u);
    const uint32_t e = tab[idx];
    float f0, f1;
    G::kept(gw, e, f0, f1);
    const float2 t = quotient_rn2(make_float2(f0, f1), make_float2(-s, -s), make_float2(rcp, rcp));
    const uint32_t codes = cvt_pair<kFmt>(t.x, t.y);
    zero_code = zero_code || (codes & 0x7Fu) == 0 || (codes & 0x7F00u) == 0;
    vals[g / 2] |= codes << (16 * (g % 2));
    meta |= ((e >> 16) & 0xFu) << (4 * g);
  }
  if (zero_code) reselect_on_codes(vals, meta);
}

// A row is taken in segments of 32 x kCpl chunks of 32 elements; lane l holds
// chunks l, l + 32, ... of the segment in registers.  Sweep 1 loads every
// segment (the amax) and keeps the last one; sweep 2 converts that one from
// registers and reloads the others (from L2).  A row of one segment (k <= 4096
// for 16-bit inputs, <= 2048 for fp32) is read from memory once.
template <typename T, int kFmt>
__global__ void __launch_bounds__(32 * kPrepWarps)
    prepare_weight24_kernel(const T* __restrict__ w, int64_t n, int64_t k, int64_t ld,
                            uint8_t* __restrict__ packed, float* __restrict__ s_w,
                            int64_t n_pad) {
  using Tr = InputTraits<T>;
  constexpr int P = Tr::kPerVec;                        // elements per 16-byte vector
  constexpr int kChunkVecs = 32 / P;                    // vectors per 32-element chunk
  constexpr int kChunkWords = 4 * kChunkVecs;
  constexpr int kCpl = 64 / kChunkWords;                // chunks per lane per segment
  constexpr int kSegChunks = 32 * kCpl;
  __shared__ uint32_t tab[64];
  if (threadIdx.x < 64) tab[threadIdx.x] = prune_entry(threadIdx.x);
  __syncthreads();
  const int warp = threadIdx.x / 32;
  const int lane = threadIdx.x % 32;
  const int64_t ktiles = k / 128;
  const int64_t chunks = k / 32;
  const int64_t segs = (chunks + kSegChunks - 1) / kSegChunks;
  for (int64_t row = static_cast<int64_t>(blockIdx.x) * kPrepWarps + warp; row < n_pad;
       row += static_cast<int64_t>(gridDim.x) * kPrepWarps) {
    const int64_t nt = row / 128;
    const int r = static_cast<int>(row % 128);
    uint8_t* tile_row = packed + nt * ktiles * 10240;
    const int vslot = 16 * (r >> 1 & 3);                  // swizzle of this row's value chunks
    if (row >= n) {   // padding rows: zero values, indices (0, 1) everywhere
      for (int64_t c = lane; c < chunks; c += 32) {
        uint8_t* tile = tile_row + (c / 4) * 10240;
        const int j = static_cast<int>(c % 4);
        *reinterpret_cast<uint4*>(tile + 64 * r + (16 * j ^ vslot)) = make_uint4(0, 0, 0, 0);
        *reinterpret_cast<uint32_t*>(tile + 8192 + 16 * r + 4 * j) = 0x44444444u;
      }
      continue;
    }
    const T* wr = w + row * ld;
    uint32_t in[kCpl][kChunkWords];
    auto load_segment = [&](int64_t seg) {
#pragma unroll
      for (int i = 0; i < kCpl; ++i) {
        const int64_t c = seg * kSegChunks + 32 * i + lane;
        if (c < chunks) {
#pragma unroll
          for (int v = 0; v < kChunkVecs; ++v)
            *reinterpret_cast<uint4*>(&in[i][4 * v]) =
                __ldg(reinterpret_cast<const uint4*>(wr + c * 32 + v * P));
        }
      }
    };
    // sweep 1: the row's amax (that of the pruned row, see above)
    float amax = 0.0f;
    for (int64_t seg = 0; seg < segs; ++seg) {
      load_segment(seg);
#pragma unroll
      for (int i = 0; i < kCpl; ++i) {
        if (seg * kSegChunks + 32 * i + lane < chunks) {
#pragma unroll
          for (int v = 0; v < kChunkVecs; ++v)
            amax = Tr::abs_max(*reinterpret_cast<const uint4*>(&in[i][4 * v]), amax);
        }
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
    const float s = __fdiv_rn(fmaxf(amax, kGuardAmax), Fp8Out<kFmt>::kMax);
    const float rcp = __frcp_rn(s);
    if (lane == 0) s_w[row] = s;
    // sweep 2: the last segment first (still in registers), then the others
    for (int64_t t = 0; t < segs; ++t) {
      const int64_t seg = (segs - 1 + t) % segs;
      if (t > 0) load_segment(seg);
#pragma unroll
      for (int i = 0; i < kCpl; ++i) {
        const int64_t c = seg * kSegChunks + 32 * i + lane;   // k columns 32c .. 32c+31
        if (c < chunks) {
          uint32_t vals[4], meta;
          prepare_chunk<T, kFmt>(in[i], tab, s, rcp, vals, meta);
          uint8_t* tile = tile_row + (c / 4) * 10240;
          const int j = static_cast<int>(c % 4);
          *reinterpret_cast<uint4*>(tile + 64 * r + (16 * j ^ vslot)) =
              make_uint4(vals[0], vals[1], vals[2], vals[3]);
          *reinterpret_cast<uint32_t*>(tile + 8192 + 16 * r + 4 * j) = meta;
        }
      }
    }
  }
}

}  // namespace sfp8

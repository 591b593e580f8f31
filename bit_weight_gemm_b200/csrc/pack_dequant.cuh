// pack_dequant.cuh - bit packing of weight codes and exact dequantisation.
//
// Both kernels are elementwise and bound by HBM bandwidth: one thread owns a
// few consecutive packed words, reads their codes (or writes their weights)
// with 128-bit accesses, and consecutive threads touch consecutive memory.
//
// Format (see bonsai.h): in a word, weight i sits in pair p = i/2 of half
// h = i%2.  Binary: bit 16h + 15 - p, set for t = -1.  Ternary: a 2-bit field
// whose high bit (16h + 15 - 2p) is the sign and low bit the magnitude.
// Shifting a word left by p (binary) or 2p (ternary) moves pair p's bits to
// bits 15 and 31 (binary), or 14-15 and 30-31 (ternary), where they are the
// sign and exponent-LSB bits of two FP16 values.
#pragma once

#include "ptx.cuh"

namespace bonsai {

constexpr int kGroup = 128;

__device__ unsigned int g_pack_bad_code = 0;

// Packs 16 ternary codes (one 16-byte load) into one word.  Returns false if
// any code is outside {-1, 0, +1}.
__device__ __forceinline__ bool pack_ternary_word(uint4 v, uint32_t& word) {
  const uint32_t b[4] = {v.x, v.y, v.z, v.w};
  uint32_t w = 0;
  bool ok = true;
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    const uint32_t code = (b[i >> 2] >> (8 * (i & 3))) & 0xFFu;  // int8 as a byte
    ok &= (((code + 1u) & 0xFFu) <= 2u);                          // -1, 0, +1 only
    const int low_bit = 16 * (i & 1) + 14 - 2 * (i >> 1);
    w |= (code & 3u) << low_bit;  // 0 -> 00, +1 -> 01, -1 (0xFF) -> 11
  }
  word = w;
  return ok;
}

// Packs 32 binary codes (two 16-byte loads) into one word.
__device__ __forceinline__ bool pack_binary_word(uint4 lo, uint4 hi, uint32_t& word) {
  const uint32_t b[8] = {lo.x, lo.y, lo.z, lo.w, hi.x, hi.y, hi.z, hi.w};
  uint32_t w = 0;
  bool ok = true;
#pragma unroll
  for (int i = 0; i < 32; ++i) {
    const uint32_t code = (b[i >> 2] >> (8 * (i & 3))) & 0xFFu;
    ok &= (code == 0x01u) | (code == 0xFFu);  // +1 or -1
    const int bit = 16 * (i & 1) + 15 - (i >> 1);
    w |= (code >> 7) << bit;  // the sign bit of the int8: set for -1
  }
  word = w;
  return ok;
}

// Each thread packs 4 consecutive words and writes them with one 16-byte
// store.  total_words is a multiple of 4 because K is a multiple of 128.
template <int MODE>
__global__ void __launch_bounds__(256) pack_kernel(const int8_t* __restrict__ codes, uint32_t* __restrict__ packed,
                                                   int64_t total_words) {
  constexpr int kPerWord = MODE == BONSAI_BINARY ? 32 : 16;
  const int64_t quads = total_words / 4;
  bool ok = true;
  for (int64_t q = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; q < quads; q += (int64_t)gridDim.x * blockDim.x) {
    const uint4* src = reinterpret_cast<const uint4*>(codes + q * 4 * kPerWord);
    uint32_t w[4];
    if (MODE == BONSAI_BINARY) {
      uint4 v[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) v[i] = __ldg(src + i);
#pragma unroll
      for (int i = 0; i < 4; ++i) ok &= pack_binary_word(v[2 * i], v[2 * i + 1], w[i]);
    } else {
      uint4 v[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) v[i] = __ldg(src + i);
#pragma unroll
      for (int i = 0; i < 4; ++i) ok &= pack_ternary_word(v[i], w[i]);
    }
    reinterpret_cast<uint4*>(packed)[q] = make_uint4(w[0], w[1], w[2], w[3]);
  }
  if (!__all_sync(0xffffffffu, ok) && lane_id() == 0) atomicOr(&g_pack_bad_code, 1u);
}

// Exact dequantisation.  Each thread expands one packed word: 16 (ternary)
// or 32 (binary) FP16 weights, 32 or 64 contiguous bytes.  The code becomes
// an exact FP16 t (ternary: the shifted field is 2t, halved exactly; binary:
// the sign bit over 1.0) and one IEEE FP16 multiply by the scale gives
// t * s with the product's sign-of-zero and NaN rules.
template <int MODE>
__global__ void __launch_bounds__(256) dequant_kernel(const uint32_t* __restrict__ packed,
                                                      const uint16_t* __restrict__ scales, uint16_t* __restrict__ w,
                                                      int64_t N, int64_t K) {
  constexpr int kPerWord = MODE == BONSAI_BINARY ? 32 : 16;
  const int64_t words_per_row = K / kPerWord;
  const int64_t groups = K / kGroup;
  const int64_t total = N * words_per_row;
  for (int64_t idx = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; idx < total;
       idx += (int64_t)gridDim.x * blockDim.x) {
    const int64_t n = idx / words_per_row;
    const int64_t j = idx - n * words_per_row;
    const uint32_t word = __ldg(packed + idx);
    const uint32_t s = __ldg(scales + n * groups + (j * kPerWord) / kGroup);
    const uint32_t s2 = s | (s << 16);
    uint32_t v[kPerWord / 2];
    if (MODE == BONSAI_BINARY) {
#pragma unroll
      for (int p = 0; p < 16; ++p) {
        const uint32_t t = ((word << p) & 0x80008000u) | 0x3C003C00u;  // +-1.0 pair
        v[p] = hmul2_bits(t, s2);
      }
    } else {
#pragma unroll
      for (int p = 0; p < 8; ++p) {
        const uint32_t two_t = (word << (2 * p)) & 0xC000C000u;  // {0, +-2.0} pair (-0 for the non-code)
        v[p] = hmul2_bits(hmul2_bits(two_t, 0x38003800u), s2);  // * 0.5 (exact), then * s
      }
    }
    uint4* dst = reinterpret_cast<uint4*>(w + n * K + j * kPerWord);
#pragma unroll
    for (int i = 0; i < kPerWord / 8; ++i) dst[i] = make_uint4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
  }
}

}  // namespace bonsai

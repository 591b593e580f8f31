// pack_dequant.cuh - bit packing of weight codes and exact dequantisation, for
// the binary and INT2 formats (below), the 4-bit group-affine weights and the
// base-3 ternary format (their sections further down), with the decode
// helpers the GEMM converters share.
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

// Packing works on four codes (one 32-bit register of int8) at a time.  A
// byte permute splits the even- and odd-indexed codes (they go to the low and
// high 16-bit halves of the word); a mask leaves each code's field at bits
// 8j of its byte j; one multiply then gathers the four fields into the top
// byte of the product in reverse order (field j at bit 30 - 2j, or 27 - j for
// one-bit fields), the order the layout wants: the multiplier's other terms
// land below bit 24 on bits no other term touches, so nothing carries.
constexpr uint32_t kGather2 = 0x40100401u;  // 2^30 + 2^20 + 2^10 + 1
constexpr uint32_t kGather1 = 0x08040201u;  // 2^27 + 2^18 + 2^9 + 1

// Nonzero bits for the bytes of x that are not -1, 0 or +1: a valid code is
// the sign extension of its two low bits, and those bits are not 10.
__device__ __forceinline__ uint32_t ternary_bad_bytes(uint32_t x) {
  const uint32_t f = x & 0x03030303u;
  const uint32_t hi = f & 0x02020202u;
  return ((f | (hi * 0x7Eu)) ^ x) | (hi & ~(f << 1));
}

// Packs 16 ternary codes (one 16-byte load) into one word; `bad` collects
// nonzero bits if any code is outside {-1, 0, +1}.
__device__ __forceinline__ uint32_t pack_ternary_word(uint4 v, uint32_t& bad) {
  const uint32_t e_lo = __byte_perm(v.x, v.y, 0x6420), e_hi = __byte_perm(v.z, v.w, 0x6420);  // codes 0,2,..,14
  const uint32_t o_lo = __byte_perm(v.x, v.y, 0x7531), o_hi = __byte_perm(v.z, v.w, 0x7531);  // codes 1,3,..,15
  bad |= ternary_bad_bytes(e_lo) | ternary_bad_bytes(e_hi) | ternary_bad_bytes(o_lo) | ternary_bad_bytes(o_hi);
  const uint32_t pe_lo = (e_lo & 0x03030303u) * kGather2, pe_hi = (e_hi & 0x03030303u) * kGather2;
  const uint32_t po_lo = (o_lo & 0x03030303u) * kGather2, po_hi = (o_hi & 0x03030303u) * kGather2;
  // even codes 0..6 -> bits 15..8, 8..14 -> 7..0; odd codes 1..7 -> 31..24, 9..15 -> 23..16
  return ((pe_lo >> 16) & 0x0000FF00u) | (pe_hi >> 24) | (po_lo & 0xFF000000u) | ((po_hi >> 8) & 0x00FF0000u);
}

// Packs 32 binary codes (two 16-byte loads) into one word: the sign bit of
// each int8 (set for -1) is its bit; `bad` collects nonzero bits for codes
// other than +1 and -1 (a valid byte is 0x01 with its sign bit spread over
// bits 1-7).
__device__ __forceinline__ uint32_t pack_binary_word(uint4 lo, uint4 hi, uint32_t& bad) {
  const uint32_t b[8] = {lo.x, lo.y, lo.z, lo.w, hi.x, hi.y, hi.z, hi.w};
  uint32_t w = 0;
#pragma unroll
  for (int g = 0; g < 4; ++g) {  // codes 8g .. 8g+7
    const uint32_t e = __byte_perm(b[2 * g], b[2 * g + 1], 0x6420);  // codes 8g, 8g+2, 8g+4, 8g+6
    const uint32_t o = __byte_perm(b[2 * g], b[2 * g + 1], 0x7531);
    const uint32_t se = (e >> 7) & 0x01010101u, so = (o >> 7) & 0x01010101u;
    bad |= ((e ^ 0x01010101u) ^ (se * 0xFEu)) | ((o ^ 0x01010101u) ^ (so * 0xFEu));
    w |= (((se * kGather1) >> 24) & 0xFu) << (12 - 4 * g);  // even codes: bits 15..0
    w |= (((so * kGather1) >> 24) & 0xFu) << (28 - 4 * g);  // odd codes: bits 31..16
  }
  return w;
}

// Each thread packs 4 consecutive words per step (one 16-byte store), with
// eight 16-byte loads in flight: two steps for ternary codes (4 loads a
// step), one for binary (8; as four 32-byte loads when WIDE, the codes then
// 32-byte aligned).  total_words is a multiple of 4 because K is a multiple
// of 128.
template <int MODE, bool WIDE = false>
__global__ void __launch_bounds__(256) pack_kernel(const int8_t* __restrict__ codes, uint32_t* __restrict__ packed,
                                                   int64_t total_words) {
  constexpr int kPerWord = MODE == BONSAI_BINARY ? 32 : 16;
  constexpr int kLoads = kPerWord / 4;  // 16-byte loads per 4 words
  constexpr int kSteps = 8 / kLoads;
  const int64_t quads = total_words / 4;
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  uint32_t bad = 0;
  for (int64_t q = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; q < quads; q += kSteps * stride) {
    uint4 v[kSteps][kLoads];
#pragma unroll
    for (int h = 0; h < kSteps; ++h) {
      const int64_t qh = q + h * stride < quads ? q + h * stride : q;
      const uint4* src = reinterpret_cast<const uint4*>(codes + qh * 4 * kPerWord);
      if constexpr (WIDE) {
#pragma unroll
        for (int i = 0; i < kLoads; i += 2) ldg_32b(src + i, v[h][i], v[h][i + 1]);
      } else {
#pragma unroll
        for (int i = 0; i < kLoads; ++i) v[h][i] = __ldg(src + i);
      }
    }
#pragma unroll
    for (int h = 0; h < kSteps; ++h) {
      uint32_t w[4];
#pragma unroll
      for (int i = 0; i < 4; ++i)
        w[i] = MODE == BONSAI_BINARY ? pack_binary_word(v[h][2 * i], v[h][2 * i + 1], bad)
                                     : pack_ternary_word(v[h][i], bad);
      if (h == 0 || q + h * stride < quads)
        reinterpret_cast<uint4*>(packed)[q + h * stride] = make_uint4(w[0], w[1], w[2], w[3]);
    }
  }
  if (!__all_sync(0xffffffffu, bad == 0) && lane_id() == 0) atomicOr(&g_pack_bad_code, 1u);
}

// Exact dequantisation.  Each thread expands one packed word: 16 (ternary)
// or 32 (binary) FP16 weights, 32 or 64 contiguous bytes.  The code becomes an exact FP16 t (ternary: the shifted field is 2t,
// halved exactly; binary: the sign bit over 1.0) and one IEEE FP16 multiply
// by the scale gives t * s with the product's sign-of-zero and NaN rules.
// WIDE: dst is 32-byte aligned and written 32 bytes a store.
template <int MODE, bool WIDE>
__device__ __forceinline__ void dequant_word(uint32_t word, uint32_t s2, uint16_t* dst) {
  constexpr int kPerWord = MODE == BONSAI_BINARY ? 32 : 16;
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
  uint4* out = reinterpret_cast<uint4*>(dst);
  if constexpr (WIDE) {
#pragma unroll
    for (int i = 0; i < kPerWord / 8; i += 2)
      stg_32b(out + i, make_uint4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]),
              make_uint4(v[4 * i + 4], v[4 * i + 5], v[4 * i + 6], v[4 * i + 7]));
  } else {
#pragma unroll
    for (int i = 0; i < kPerWord / 8; ++i) out[i] = make_uint4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
  }
}

template <int MODE, bool WIDE>
__global__ void __launch_bounds__(256) dequant_kernel(const uint32_t* __restrict__ packed,
                                                      const uint16_t* __restrict__ scales, uint16_t* __restrict__ w,
                                                      int64_t N, int64_t K) {
  constexpr int kPerWord = MODE == BONSAI_BINARY ? 32 : 16;
  const int64_t words_per_row = K / kPerWord;
  const int64_t groups = K / kGroup;
  const int64_t total = N * words_per_row;
  for (int64_t idx = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; idx < total;
       idx += (int64_t)gridDim.x * blockDim.x) {
    const int64_t n = idx / words_per_row, j = idx - n * words_per_row;
    const uint32_t s = __ldg(scales + n * groups + (j * kPerWord) / kGroup);
    dequant_word<MODE, WIDE>(__ldg(packed + idx), s | (s << 16), w + n * K + j * kPerWord);
  }
}

// ------------------------------------ 4-bit group-affine weights (HQQ) --
// (bonsai.h.)  q in 0..15, 8 per word: weight i of a word at bit 16 (i%2) +
// 4 (i/2), so (word >> 4p) & 0x000F000F holds weights 2p and 2p+1 in the
// two halves; FP16 scale s and zero z per 64 weights along K;
// w = fp16(fp16(q - z) * s).
constexpr int kModeHqq4 = 4;  // kernel template mode of this format
constexpr int kHqqGroup = 64;
constexpr uint32_t kF16x2_1024 = 0x64006400u;

// Weights 2p, 2p+1 of a word as the exact FP16 pair (q0, q1): the nibbles
// under FP16's exponent of 1024, minus 1024.
__device__ __forceinline__ uint32_t hqq4_q_pair(uint32_t word, int p) {
  const uint32_t magic = ((word >> (4 * p)) & 0x000F000Fu) | kF16x2_1024;  // (1024 + q0, 1024 + q1)
  uint32_t q;
  asm("sub.rn.f16x2 %0, %1, %2;" : "=r"(q) : "r"(magic), "r"(kF16x2_1024));
  return q;
}

// fp16(fp16(q - z) * s) for a pair, with z2 / s2 the group's zero / scale in
// both halves: two IEEE FP16 operations, as the format defines.
__device__ __forceinline__ uint32_t hqq4_w_pair(uint32_t q2, uint32_t z2, uint32_t s2) {
  uint32_t d;
  asm("sub.rn.f16x2 %0, %1, %2;" : "=r"(d) : "r"(q2), "r"(z2));
  return hmul2_bits(d, s2);
}

// Each thread packs 4 words (32 values, two 16-byte loads, one 16-byte store).
__global__ void __launch_bounds__(256) pack_hqq4_kernel(const uint8_t* __restrict__ q, uint32_t* __restrict__ packed,
                                                        int64_t total_words) {
  const int64_t quads = total_words / 4;
  bool ok = true;
  for (int64_t t = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; t < quads; t += (int64_t)gridDim.x * blockDim.x) {
    const uint4* src = reinterpret_cast<const uint4*>(q + t * 32);
    const uint4 a = __ldg(src), b = __ldg(src + 1);
    const uint32_t v[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
    uint32_t w[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      uint32_t word = 0;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const uint32_t value = (v[2 * j + (i >> 2)] >> (8 * (i & 3))) & 0xFFu;
        ok &= value <= 15u;
        word |= (value & 15u) << (16 * (i & 1) + 4 * (i >> 1));
      }
      w[j] = word;
    }
    reinterpret_cast<uint4*>(packed)[t] = make_uint4(w[0], w[1], w[2], w[3]);
  }
  if (!__all_sync(0xffffffffu, ok) && lane_id() == 0) atomicOr(&g_pack_bad_code, 1u);
}

// Exact dequantisation: one thread per word (8 weights, one 16-byte store).
__global__ void __launch_bounds__(256) dequant_hqq4_kernel(const uint32_t* __restrict__ packed,
                                                           const uint16_t* __restrict__ scales,
                                                           const uint16_t* __restrict__ zeros,
                                                           uint16_t* __restrict__ w, int64_t N, int64_t K) {
  const int64_t words_per_row = K / 8, groups = K / kHqqGroup;
  const int64_t total = N * words_per_row;
  for (int64_t idx = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; idx < total;
       idx += (int64_t)gridDim.x * blockDim.x) {
    const int64_t n = idx / words_per_row, j = idx - n * words_per_row;
    const uint32_t word = __ldg(packed + idx);
    const int64_t g = n * groups + (8 * j) / kHqqGroup;
    const uint32_t s = __ldg(scales + g), z = __ldg(zeros + g);
    const uint32_t s2 = s | (s << 16), z2 = z | (z << 16);
    uint32_t v[4];
#pragma unroll
    for (int p = 0; p < 4; ++p) v[p] = hqq4_w_pair(hqq4_q_pair(word, p), z2, s2);
    *reinterpret_cast<uint4*>(w + n * K + 8 * j) = make_uint4(v[0], v[1], v[2], v[3]);
  }
}

// ------------------------------------------------- base-3 ternary format --
// (bonsai.h.)  A group's byte j holds the trits at group positions j, j+26,
// j+52, j+78, j+104 as y = ceil(256 v / 243), v their base-3 number
// (digits t+1, most significant first).  y / 256 is v / 243 plus less than
// 1/243, so multiplying y by 3 puts the next digit in bits 8-9 and leaves
// the rest of the fraction in the low byte, exactly, five times.  Two bytes
// j and j+1 side by side as 16-bit lanes step together; their same digit is
// the pair of neighbouring weights (26 i + j, 26 i + j + 1).
constexpr int kB3GroupBytes = 26;
constexpr int kB3BlockGroups = 4;
constexpr int kB3BlockBytes = 112;  // 4 x 26 bytes + 8 zero bytes
constexpr uint32_t kB3Minus1025 = 0xE401E401u;  // FP16 -1025 in both halves

// Bytes 2p and 2p+1 of the group's (aligned) words as the 16-bit lanes of one
// register.
__device__ __forceinline__ uint32_t b3_byte_pair(const uint32_t* w, int p) {
  return __byte_perm(w[p >> 1], 0u, (p & 1) ? 0x4342u : 0x4140u);
}

// Steps a byte pair to its next digit pair and returns (t0, t1) as FP16:
// the digits d land under FP16's exponent of 1024 (byte 0x64 above them)
// and 1024 + d - 1025 = t exactly.
__device__ __forceinline__ uint32_t b3_next_t_pair(uint32_t& y) {
  const uint32_t t3 = y * 3u;
  y = t3 & 0x00FF00FFu;
  const uint32_t magic = __byte_perm(t3, 0x64646464u, 0x4341u);  // (1024 + d0, 1024 + d1)
  uint32_t t;
  asm("add.rn.f16x2 %0, %1, %2;" : "=r"(t) : "r"(magic), "r"(kB3Minus1025));
  return t;
}

// Loads the 26 bytes of group slot r (0..3) of a row's block as 7 words
// aligned to the group's first byte (slots 1 and 3 start 2 bytes into a word).
__device__ __forceinline__ void b3_group_words(const uint32_t* block, int r, uint32_t* w) {
  const int w0 = (kB3GroupBytes * r) >> 2;
  uint32_t raw[8];
#pragma unroll
  for (int k = 0; k < 8; ++k) raw[k] = block[w0 + k];
  const bool odd = (r & 1) != 0;
#pragma unroll
  for (int k = 0; k < 7; ++k) w[k] = odd ? __funnelshift_r(raw[k], raw[k + 1], 16) : raw[k];
}

// Packs the codes of group slot r of one row's block b into bytes
// 26r .. 26r+25 of the block's 112 (zeros for a slot past the row's groups;
// bytes 104..111 are zero).  One thread per slot, so consecutive threads read
// consecutive 128-byte groups with 16-byte loads.  A warp's 32 slots are 8
// whole blocks (896 contiguous bytes): the threads leave their 26 bytes in a
// shared-memory copy of them, and the warp writes it out in 16-byte stores.
// WIDE: the codes are 32-byte aligned and read 32 bytes a load.
template <bool WIDE>
__global__ void __launch_bounds__(256) pack_b3_kernel(const int8_t* __restrict__ codes, uint32_t* __restrict__ packed,
                                                      int64_t N, int64_t K) {
  constexpr int kWarpBlocks = 32 / kB3BlockGroups;
  constexpr int kWarpBytes = kWarpBlocks * kB3BlockBytes;
  __shared__ alignas(16) uint8_t stage_all[8][kWarpBytes];
  const int64_t groups = K / kGroup;
  const int64_t blocks_per_row = (groups + kB3BlockGroups - 1) / kB3BlockGroups;
  const int64_t total = N * blocks_per_row * kB3BlockGroups;  // slots, a multiple of 32 / kWarpBlocks
  const int lane = threadIdx.x & 31;
  uint8_t* stage = stage_all[threadIdx.x >> 5];
  bool ok = true;
  // Warp-uniform loop over runs of 32 slots.
  for (int64_t base = (blockIdx.x * (int64_t)blockDim.x + threadIdx.x) - lane; base < total;
       base += (int64_t)gridDim.x * blockDim.x) {
    const int64_t idx = base + lane;
    const int r = lane % kB3BlockGroups;
    uint16_t* dst = reinterpret_cast<uint16_t*>(stage + (lane / kB3BlockGroups) * kB3BlockBytes + kB3GroupBytes * r);
    const int64_t blk = idx / kB3BlockGroups;  // n * blocks_per_row + b
    const int64_t n = blk / blocks_per_row;
    const int64_t g = (blk - n * blocks_per_row) * kB3BlockGroups + r;
    if (idx < total && g < groups) {
      const uint4* src = reinterpret_cast<const uint4*>(codes + n * K + g * kGroup);
      uint4 q4[8];
      if constexpr (WIDE) {
#pragma unroll
        for (int i = 0; i < 8; i += 2) ldg_32b(src + i, q4[i], q4[i + 1]);
      } else {
#pragma unroll
        for (int i = 0; i < 8; ++i) q4[i] = __ldg(src + i);
      }
      uint32_t c[32];
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        c[4 * i] = q4[i].x;
        c[4 * i + 1] = q4[i].y;
        c[4 * i + 2] = q4[i].z;
        c[4 * i + 3] = q4[i].w;
      }
#pragma unroll
      for (int h = 0; h < kB3GroupBytes / 2; ++h) {
        uint32_t pair = 0;
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const int j = 2 * h + e;  // byte j holds codes j, 26 + j, 52 + j, 78 + j, 104 + j
          uint32_t v = 0;
#pragma unroll
          for (int i = 0; i < 5; ++i) {
            const int k = 26 * i + j;
            uint32_t q = 0;  // positions past the group: digit 0
            if (k < kGroup) {
              q = ((c[k >> 2] >> (8 * (k & 3))) + 1u) & 0xFFu;  // t + 1 for t in {-1, 0, +1}
              ok &= q <= 2u;
            }
            v = 3u * v + q;
          }
          pair |= (((256u * v + 242u) / 243u) & 0xFFu) << (8 * e);  // ceil(256 v / 243)
        }
        dst[h] = static_cast<uint16_t>(pair);
      }
    } else {
#pragma unroll
      for (int h = 0; h < kB3GroupBytes / 2; ++h) dst[h] = 0;
    }
    if (r == kB3BlockGroups - 1)
      *reinterpret_cast<uint2*>(stage + (lane / kB3BlockGroups) * kB3BlockBytes + kB3GroupBytes * kB3BlockGroups) =
          make_uint2(0u, 0u);
    __syncwarp();
    // The run's whole blocks (all 8 but at the very end), 16 bytes a thread.
    const int64_t left = (total - base) / kB3BlockGroups;
    const int chunks = (left < kWarpBlocks ? static_cast<int>(left) : kWarpBlocks) * (kB3BlockBytes / 16);
    uint4* out = reinterpret_cast<uint4*>(reinterpret_cast<uint8_t*>(packed) + base / kB3BlockGroups * kB3BlockBytes);
    for (int c16 = lane; c16 < chunks; c16 += 32) out[c16] = reinterpret_cast<const uint4*>(stage)[c16];
    __syncwarp();
  }
  if (!__all_sync(0xffffffffu, ok) && lane_id() == 0) atomicOr(&g_pack_bad_code, 1u);
}

// Exact dequantisation of the base-3 format: one thread per (row, group);
// t comes out of the digit step as an exact FP16 -1, +0 or +1 and one IEEE
// FP16 multiply by the scale gives t * s.
__global__ void __launch_bounds__(256) dequant_b3_kernel(const uint32_t* __restrict__ packed,
                                                         const uint16_t* __restrict__ scales,
                                                         uint16_t* __restrict__ w, int64_t N, int64_t K) {
  const int64_t groups = K / kGroup;
  const int64_t row_words = (groups + kB3BlockGroups - 1) / kB3BlockGroups * (kB3BlockBytes / 4);
  const int64_t total = N * groups;
  for (int64_t idx = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; idx < total;
       idx += (int64_t)gridDim.x * blockDim.x) {
    const int64_t n = idx / groups, g = idx - n * groups;
    const uint32_t* block = packed + n * row_words + g / kB3BlockGroups * (kB3BlockBytes / 4);
    uint32_t words[7];
    b3_group_words(block, static_cast<int>(g % kB3BlockGroups), words);
    const uint32_t s = __ldg(scales + n * groups + g);
    const uint32_t s2 = s | (s << 16);
    uint32_t y[13];
#pragma unroll
    for (int p = 0; p < 13; ++p) y[p] = b3_byte_pair(words, p);
    uint32_t* dst = reinterpret_cast<uint32_t*>(w + n * K + g * kGroup);  // FP16 pairs: weights 2c, 2c+1
#pragma unroll
    for (int i = 0; i < 5; ++i)
#pragma unroll
      for (int p = 0; p < 13; ++p) {
        const int c = 13 * i + p;
        if (c < kGroup / 2) dst[c] = hmul2_bits(b3_next_t_pair(y[p]), s2);
      }
  }
}

}  // namespace bonsai

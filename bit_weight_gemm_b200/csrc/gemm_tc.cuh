// gemm_tc.cuh - fused dequantise + GEMM on the 5th-generation tensor cores.
//
// out[m,n] = sum_k A[m,k] * w[n,k],  w[n,k] = s[n,k/128] * t[n,k]  (binary,
// ternary INT2, ternary base-3), or w = fp16(fp16(q - z) * s) with a scale
// and zero per 64 weights (4-bit group-affine).
//
// A CTA computes a tile of 128 weight rows x BLOCK_T tokens over a range of
// 128-wide K groups, as D^T = W * A^T, so that the weights are the MMA's M
// side and can be fed from tensor memory.  Three rings decouple the stages:
//
//   act ring   (warp 0)  TMA of the activation tile per group: BLOCK_T rows
//                        x 128 FP16 as two 128-byte-swizzled K slices.
//   word ring  (warp 2)  TMA of the 128 rows' packed words, 128 bytes of
//                        each row per stage (8 binary, 4 INT2 or 2 4-bit
//                        groups) with 128-byte swizzling, so that the
//                        converters' 16-byte reads are free of bank conflicts
//                        and each request moves a whole 128-byte line; or one
//                        unswizzled 112-byte base-3 block (4 groups).
//   TMEM ring  (warps 3-18, four per TMEM lane quadrant, taking groups in
//                        turn) converters: each thread owns one weight row,
//                        turns the group's words into FP16 weights (binary:
//                        sign bit over s; ternary INT2: the shifted 2-bit
//                        field is 2t, times s; base-3: digits stepped out of
//                        two bytes at a time, t, times s; 4-bit: the nibble
//                        pair under FP16's 1024, minus 1024, minus z, times
//                        s) and writes them to a TMEM stage with tcgen05.st.
//   warp 1               allocates TMEM; one thread issues
//                        tcgen05.mma.kind::f16 (M=128, N=BLOCK_T, K=16) x 8
//                        per group, A from TMEM, B from shared memory, FP32
//                        accumulator in TMEM; tcgen05.commit releases the
//                        act and TMEM stages.
//
// Launches use programmatic dependent launch: a CTA sets up its barriers and
// tensor memory while the previous kernel in the stream finishes, and waits
// for that kernel's completion before its first global-memory access.
//
// Epilogue, one CTA per tile (ksplit = 1): the converters read the
// accumulator (tcgen05.ld), scale by 1/2 (INT2, which converts 2ts; exact)
// or 1,
// round once to FP16 into a shared-memory tile, and one TMA store writes it.
// Split K (ksplit > 1, small M): the ksplit CTAs of a cluster share a tile;
// each leaves its FP32 partial in shared memory and, after a cluster
// barrier, each reduces a slice of the tile from all partials over
// distributed shared memory (16-byte loads) in a fixed order, rounds once
// and stores it.  Accumulation is spread over several TMEM accumulators so
// that narrow MMAs do not queue behind one accumulator.
//
// Weights are formed exactly: |t| <= 1 and s is FP16, so s*t (and 2*s*t for
// |s| < 32768) is an FP16 value, and the 4-bit weight is by definition the
// FP16 result of its two FP16 operations; products and the sum run in FP32.
#pragma once

#include "pack_dequant.cuh"
#include "ptx.cuh"

namespace bonsai {

__host__ __device__ constexpr int largest_divisor_at_most(int n, int cap) {
  int d = cap < n ? cap : n;
  while (n % d != 0) --d;
  return d;
}

__host__ __device__ constexpr int pow2_at_least(int x) {
  int p = 32;
  while (p < x) p *= 2;
  return p;
}

// One CTA per SM: a CTA owns all 512 TMEM columns and most of shared memory.
// (Two CTAs per SM with 128-token tiles, 256 TMEM columns each, measured 15%
// slower on the M=4608 workload.)
template <int MODE, int BLOCK_T>
struct GemmTile {
  static constexpr int kRows = 128;  // weight rows per tile (MMA M)
  static constexpr bool kB3 = MODE == BONSAI_TERNARY_B3;
  // Words a converter holds per group: 4 binary, 8 INT2, 7 base-3 (26 bytes).
  static constexpr bool kHqq = MODE == kModeHqq4;
  static constexpr int kWordsPerGroup = MODE == BONSAI_BINARY ? 4 : (kB3 ? 7 : (kHqq ? 16 : 8));
  static constexpr int kSliceBytes = BLOCK_T * 128;       // BLOCK_T rows x 64 FP16
  static constexpr int kActStageBytes = 2 * kSliceBytes;  // 128 K per stage
  // Tiles wider than one MMA (352 tokens) run as two halves of kMmaN tokens:
  // two MMAs per K step into two accumulators (the second at TMEM column
  // kHalfCol, 64-aligned), and TMA boxes of kMmaN rows (a box has at most
  // 256).
  static constexpr int kHalves = BLOCK_T > 256 ? 2 : 1;
  static constexpr int kMmaN = BLOCK_T / kHalves;
  static constexpr int kHalfCol = kHalves == 2 ? (kMmaN + 63) / 64 * 64 : 0;
  static constexpr int kHalfBytes = kMmaN * 128;  // one half of a K slice
  // Activation stages: as many as fit next to the word ring and the scales,
  // so that narrow tiles keep a split-K CTA's whole K range in flight.
  static constexpr int kActStages =
      BLOCK_T > 256 ? 2 : (BLOCK_T > 128 ? 3 : (BLOCK_T == 128 ? 4 : (96 * 1024) / kActStageBytes));
  // A word stage is 128 bytes of every row: 4 ternary or 8 binary groups,
  // one TMA box with 128-byte swizzling.
  // Base-3: one 112-byte block (4 groups) of every row per stage, without
  // swizzling (a 112-byte box is not a 128-byte swizzle span).
  static constexpr int kWGroups = kB3 ? kB3BlockGroups : 32 / kWordsPerGroup;
  static constexpr int kWRowBytes = kB3 ? kB3BlockBytes : 128;
  static constexpr int kWStageBytes = kRows * kWRowBytes;
  // Split-K ranges of base-3 weights start on block boundaries (TMA copies
  // start on 16-byte boundaries).
  static constexpr int kGroupAlign = kB3 ? kB3BlockGroups : 1;
  // Small token tiles are bandwidth-bound: enough word stages to keep every
  // load of a split-K CTA in flight at once.
  static constexpr int kWStages = BLOCK_T > 128 ? 2 : 4;
  // The tile's scales, staged once per CTA when 128 x groups x 2 bytes fit.
  // (4-bit group-affine weights keep scale and zero pairs in registers.)
  static constexpr int kScaleBytes = (BLOCK_T >= 256 || kHqq) ? 0 : 32768;
  // Converter warps: four per TMEM lane quadrant.  (Five per quadrant on
  // narrow tiles measured 2-5% slower.)  Two-half tiles leave room for two
  // TMEM stages only, and a quadrant may have no more warps than stages
  // (below); a group is then ~1400 cycles of MMAs, ample for two.
  static constexpr int kConvWarps = kHalves == 2 ? 8 : 16;
  static constexpr int kWarpsPerQuad = kConvWarps / 4;
  // Epilogue: the quadrant's warps split the token columns, 8 at least each:
  // the most warps (up to kWarpsPerQuad) that divide BLOCK_T / 8.
  static constexpr int kEpiWarpsPerQuad = largest_divisor_at_most(BLOCK_T / 8, kWarpsPerQuad);
  // Two MMA-issuing threads (alternate groups, separate accumulators) and
  // two activation producers for tiles of up to 128 tokens, where one thread
  // issuing every MMA and polling every barrier is the serial limit.  A
  // 256-token accumulator fills half of TMEM, so those tiles keep one.
  static constexpr int kMmaThreads = BLOCK_T <= 128 ? 2 : 1;
  static constexpr int kActWarpB = 3 + kConvWarps;  // second activation producer
  static constexpr int kMmaWarpB = 4 + kConvWarps;  // second MMA issuer (idle when kMmaThreads == 1)
  static constexpr int kThreads = 32 * (5 + kConvWarps);
  // Successive MMAs rotate over kAccs accumulators [a*BLOCK_T, (a+1)*BLOCK_T):
  // with narrow tiles an MMA is a few cycles of work, so a chain of MMAs into
  // one accumulator would run at the accumulate latency instead.
  static constexpr int kAccs = (kMmaThreads == 2 || BLOCK_T <= 32) ? 2 : 1;
  static constexpr int kACol0 = kHalves == 2 ? 2 * kHalfCol
                                : (kAccs * BLOCK_T < 64 ? 64 : kAccs * BLOCK_T);  // converted-weight stages follow
  // TMEM stages of converted weights, 64 columns each: all that is left
  // after the accumulators.  A stage is reused only after the MMAs that read
  // it completed, so the number of stages is the number of groups in flight
  // between the converters and the tensor core.
  static constexpr int kTmemCols = 512;
  static constexpr int kTStagesFit = (kTmemCols - kACol0) / 64;
  // With two MMA-issuing warps the stage count has the parity of
  // kWarpsPerQuad (one stage is left unused otherwise); see the assertion below.
  static constexpr int kTStages =
      (kMmaThreads == 2 && (kTStagesFit - kWarpsPerQuad) % 2 != 0) ? kTStagesFit - 1 : kTStagesFit;
  static constexpr int kActOff = 0;
  static constexpr int kWOff = kActStages * kActStageBytes;
  static constexpr int kScaleOff = kWOff + kWStages * kWStageBytes;
  static constexpr int kBarOff = kScaleOff + kScaleBytes;
  static constexpr int kNumBars = 2 * kActStages + 2 * kTStages + 2 * kWStages + 2;
  static constexpr int kMiscOff = kBarOff + kNumBars * 8;
  static constexpr int kSmemNeeded = kMiscOff + 16 + 1024;  // + slack to align the base to 1024
  // A second CTA could not get its 512 TMEM columns, so shared memory keeps
  // it off the SM.
  static constexpr int kSmemBytes = kSmemNeeded < 116 * 1024 ? 116 * 1024 : kSmemNeeded;

  static constexpr float kOutScale = MODE == BONSAI_TERNARY_INT2 ? 0.5f : 1.0f;  // INT2 converts to 2ts
  static_assert(kMmaN % 16 == 0 && kMmaN >= 16 && kMmaN <= 256 && kMmaN * kHalves == BLOCK_T, "MMA N for M=128");
  static_assert(kHalves == 1 || (kAccs == 1 && kHalfCol >= kMmaN && kHalfBytes % 1024 == 0), "two-half tiles");
  static_assert(kSliceBytes % 1024 == 0, "swizzle atoms need 1024-byte alignment");
  static_assert(kACol0 + kTStages * 64 <= kTmemCols && kTStages >= 2, "TMEM budget");
  // Parity waits on a TMEM stage are unambiguous only if the converter is at
  // most one use ahead of the MMAs: when a converter waits for the MMAs of
  // group i - TS (stage reuse), those of group i - 2TS must be done.  Its own
  // previous wait (group i - kWarpsPerQuad) saw group i - kWarpsPerQuad - TS
  // done, which covers i - 2TS if kWarpsPerQuad <= TS and, with two MMA warps
  // taking alternate groups, if both groups were issued by the same warp
  // (whose commit covers all its earlier MMAs): TS - kWarpsPerQuad even.
  static_assert(kWarpsPerQuad <= kTStages, "converter warps per quadrant <= TMEM stages");
  // Converter warps reading each full word stage: every one of them, or (4-bit
  // weights: 2 groups per stage) the four warps of each of its groups.
  static constexpr int kWReaders = 4 * (kWGroups < kWarpsPerQuad ? kWGroups : kWarpsPerQuad);
  static_assert(kWGroups % kWarpsPerQuad == 0 || kWarpsPerQuad % kWGroups == 0, "whole groups of readers");
  static_assert(kMmaThreads == 1 || (kTStages - kWarpsPerQuad) % 2 == 0, "same MMA warp for groups i-q-TS, i-2TS");
  static_assert(kSmemBytes <= 227 * 1024, "shared memory per CTA");
  static_assert(kActStages >= 2, "activation ring depth");
  // Parity waits are unambiguous only for a waiter that meets every phase of
  // a barrier, or whose skipped phases are known complete.  Two MMA warps take
  // alternate groups: with an even number of stages each of them (and each of
  // the two activation producers) keeps to its own stages.  With one MMA warp
  // the stages are released in order, which covers the producers' skips.
  static_assert(kMmaThreads == 1 || kActStages % 2 == 0, "alternate groups keep to their own stages");
  static_assert(BLOCK_T * kRows * 2 <= kActStages * kActStageBytes, "output tile fits the act ring");
  static_assert(kRows * BLOCK_T * 4 <= kActStages * kActStageBytes, "partial fits the act ring");
};

// Converts one group of this thread's row (4 binary or 8 ternary words)
// into FP16 products and writes them to 64 TMEM columns at `taddr`.
template <int MODE>
__device__ __forceinline__ void convert_group(const uint32_t* words, uint32_t s2, uint32_t taddr) {
  if (MODE == BONSAI_BINARY) {
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      uint32_t v[16];
#pragma unroll
      for (int p = 0; p < 16; ++p) v[p] = ((words[j] << p) & 0x80008000u) ^ s2;  // (+-s, +-s)
      tmem_store_8(taddr + j * 16, v);
      tmem_store_8(taddr + j * 16 + 8, v + 8);
    }
  } else {
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      uint32_t v[8];
#pragma unroll
      for (int p = 0; p < 8; ++p) v[p] = hmul2_bits((words[j] << (2 * p)) & 0xC000C000u, s2);  // (2ts, 2ts)
      tmem_store_8(taddr + j * 8, v);
    }
  }
}

// Base-3: the group's 26 bytes (7 words from b3_group_words) -> 64 TMEM
// columns of FP16 pairs t*s; column 13 i + p holds digit i of byte pair p,
// i.e. the weights 26 i + 2p and 26 i + 2p + 1.
__device__ __forceinline__ void convert_group_b3(const uint32_t* words, uint32_t s2, uint32_t taddr) {
  uint32_t y[13];
#pragma unroll
  for (int p = 0; p < 13; ++p) y[p] = b3_byte_pair(words, p);
  uint32_t v[8];
#pragma unroll
  for (int i = 0; i < 5; ++i)
#pragma unroll
    for (int p = 0; p < 13; ++p) {
      const int c = 13 * i + p;
      if (c < 64) {
        v[c & 7] = hmul2_bits(b3_next_t_pair(y[p]), s2);
        if ((c & 7) == 7) tmem_store_8(taddr + (c - 7), v);
      }
    }
}

// First word (uint32 x coordinate of the packed-weight tensor map) of the
// word stage that starts at group g0.
template <int MODE>
__device__ __forceinline__ int word_stage_x(int g0) {
  if (MODE == BONSAI_TERNARY_B3) return g0 / kB3BlockGroups * (kB3BlockBytes / 4);
  return g0 * (MODE == BONSAI_BINARY ? 4 : (MODE == kModeHqq4 ? 16 : 8));
}

// 4-bit group-affine: the group's 16 words (K 0..63 in words 0-7 with the
// first scale and zero, 64..127 in words 8-15 with the second) -> 64 TMEM
// columns of FP16 pairs fp16(fp16(q - z) * s); column 4 j + p holds weights
// 2p, 2p+1 of word j.  s_pair / z_pair hold the two groups' values.
__device__ __forceinline__ void convert_group_hqq4(const uint32_t* words, uint32_t s_pair, uint32_t z_pair,
                                                   uint32_t taddr) {
  const uint32_t s_lo = __byte_perm(s_pair, 0u, 0x1010u), s_hi = __byte_perm(s_pair, 0u, 0x3232u);
  const uint32_t z_lo = __byte_perm(z_pair, 0u, 0x1010u), z_hi = __byte_perm(z_pair, 0u, 0x3232u);
  uint32_t v[8];
#pragma unroll
  for (int j = 0; j < 16; ++j)
#pragma unroll
    for (int p = 0; p < 4; ++p) {
      const int c = 4 * j + p;
      v[c & 7] = hqq4_w_pair(hqq4_q_pair(words[j], p), j < 8 ? z_lo : z_hi, j < 8 ? s_lo : s_hi);
      if ((c & 7) == 7) tmem_store_8(taddr + (c - 7), v);
    }
}

// Boundary z of a split of `groups` into `ks` ranges, on multiples of ALIGN
// (nearest); the caller keeps ks <= groups / ALIGN so that no range is empty.
template <int ALIGN>
__host__ __device__ __forceinline__ int split_bound(int z, int groups, int ks) {
  if (z >= ks) return groups;
  const int x = static_cast<int>(static_cast<int64_t>(z) * groups / ks);
  const int r = (x + ALIGN / 2) / ALIGN * ALIGN;
  return r < groups ? r : groups;
}

// A wait the whole warp agrees on: every lane waits, and the warp goes on
// only if all lanes saw the phase complete.
__device__ __forceinline__ bool warp_wait(uint32_t bar, uint32_t parity, volatile int* abort_flag,
                                          uint64_t limit_ns) {
  const bool ok = wait_phase(bar, parity, abort_flag, limit_ns);
  return __all_sync(0xffffffffu, ok);
}

// warp_wait with the blocking loop inlined (see wait_phase_inlined).
__device__ __forceinline__ bool warp_wait_inlined(uint32_t bar, uint32_t parity, volatile int* abort_flag,
                                                  uint64_t limit_ns) {
  const bool ok = wait_phase_inlined(bar, parity, abort_flag, limit_ns);
  return __all_sync(0xffffffffu, ok);
}

// Reads 8 columns of this thread's lane from each of the NACC accumulators
// (BLOCK_T columns apart) and adds the first `used` of them in a fixed order
// (an accumulator no MMA wrote holds nothing meaningful).
template <int NACC, int BLOCK_T>
__device__ __forceinline__ void sum_accumulators(uint32_t taddr, int used, float* acc) {
  uint32_t v[NACC][8];
#pragma unroll
  for (int a = 0; a < NACC; ++a) tmem_load_8(taddr + a * BLOCK_T, v[a]);
  tmem_load_wait();
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    float x = __uint_as_float(v[0][j]);
#pragma unroll
    for (int a = 1; a < NACC; ++a)
      if (a < used) x += __uint_as_float(v[a][j]);
    acc[j] = x;
  }
}

struct GemmArgs {
  const uint16_t* scales;
  const uint16_t* zeros;  // 4-bit group-affine weights only
  uint16_t* out;
  int M, N, K;
  int ksplit;     // CTAs along K sharing one tile (the cluster size along z)
  int tma_store;  // 1: write the tile with one TMA store (needs N % 8 == 0)
  int scale_box;  // > 0: groups per row in the scale TMA box (the tile's scales arrive with one copy)
  uint64_t wait_limit_ns;
};

template <int MODE, int BLOCK_T>
__global__ void __launch_bounds__(GemmTile<MODE, BLOCK_T>::kThreads, 1)
    lowbit_gemm_kernel(const __grid_constant__ CUtensorMap tmap_act, const __grid_constant__ CUtensorMap tmap_w,
                       const __grid_constant__ CUtensorMap tmap_out, const __grid_constant__ CUtensorMap tmap_s,
                       const GemmArgs args) {
  using T = GemmTile<MODE, BLOCK_T>;
  constexpr int AS = T::kActStages, TS = T::kTStages, WS = T::kWStages;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + T::kBarOff);
  const uint32_t act_full0 = smem_addr(bars);                     // TMA bytes of act stage landed
  const uint32_t act_empty0 = smem_addr(bars + AS);               // MMAs reading act stage done
  const uint32_t t_ready0 = smem_addr(bars + 2 * AS);             // converted weights in TMEM stage (4 warps)
  const uint32_t t_free0 = smem_addr(bars + 2 * AS + TS);         // MMAs reading TMEM stage done
  const uint32_t w_full0 = smem_addr(bars + 2 * AS + 2 * TS);     // TMA bytes of word stage landed
  const uint32_t w_empty0 = smem_addr(bars + 2 * AS + 2 * TS + WS);  // converters read word stage
  const uint32_t dfull = smem_addr(bars + 2 * AS + 2 * TS + 2 * WS);  // accumulator final
  const uint32_t s_full = smem_addr(bars + 2 * AS + 2 * TS + 2 * WS + 1);  // scale tile landed
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + T::kMiscOff);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + T::kMiscOff + 4);

  // Broadcast from lane 0 so that the compiler treats the warp index, and so
  // every role branch below, as warp-uniform: the tcgen05 and TMA operands
  // derived from it can then live in uniform registers.
  const int warp = __shfl_sync(0xffffffffu, static_cast<int>(threadIdx.x >> 5), 0);
  const int lane = threadIdx.x & 31;
  const int n0 = blockIdx.x * T::kRows;
  const int m0 = blockIdx.y * BLOCK_T;
  const int groups = args.K / kGroup;
  const int g_begin = split_bound<T::kGroupAlign>(static_cast<int>(blockIdx.z), groups, args.ksplit);
  const int g_end = split_bound<T::kGroupAlign>(static_cast<int>(blockIdx.z) + 1, groups, args.ksplit);
  const int ng = g_end - g_begin;
  const uint64_t limit = args.wait_limit_ns;

  if (threadIdx.x == 0) {
    for (int s = 0; s < AS; ++s) {
      mbar_init(act_full0 + 8 * s, 1);
      mbar_init(act_empty0 + 8 * s, 1);
    }
    for (int s = 0; s < TS; ++s) {
      mbar_init(t_ready0 + 8 * s, 4);  // one converter warp per TMEM lane quadrant
      mbar_init(t_free0 + 8 * s, 1);
    }
    for (int s = 0; s < WS; ++s) {
      mbar_init(w_full0 + 8 * s, 1);
      mbar_init(w_empty0 + 8 * s, T::kWReaders);  // the converter warps that read each full stage
    }
    mbar_init(dfull, T::kMmaThreads);
    mbar_init(s_full, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_map(&tmap_act);
    tma_prefetch_map(&tmap_w);
    tma_prefetch_map(&tmap_out);
    if (args.scale_box > 0) tma_prefetch_map(&tmap_s);
  }
  if (warp == 2 && lane == 0) {
    // The CTA's packed words and scales into L2 while the preceding grid may
    // still run (they are read-only here; the copies into shared memory
    // follow griddep_wait).
    const int nw = (ng + T::kWGroups - 1) / T::kWGroups;
    for (int i = 0; i < nw; ++i) tma_prefetch_l2_2d(&tmap_w, word_stage_x<MODE>(g_begin + i * T::kWGroups), n0);
    if (args.scale_box > 0) tma_prefetch_l2_2d(&tmap_s, g_begin & ~7, n0);
  }
  if (warp == 1) {
    tmem_alloc(smem_addr(tmem_slot), T::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tmem = __shfl_sync(0xffffffffu, *tmem_slot, 0);  // warp-uniform (see above)
  // The next launch in the stream may start its own prologue now; it waits
  // (griddep_wait) for this grid to finish before touching global memory.
  // Only now, with this CTA's tensor memory held: a dependent CTA placed on
  // this SM may then block in its own allocation until this CTA frees its
  // columns, but never the other way round (this CTA waits on nothing the
  // dependent holds), so the two cannot deadlock.
  if (threadIdx.x == 0) griddep_launch_dependents();
  // Everything above touched only this CTA's own resources; global memory
  // (activations, weights, scales, output) only after the preceding grid in
  // the stream has completed.
  griddep_wait();

  // Producer and MMA loops run warp-uniformly: every lane of the warp takes
  // the same path and waits, and one elected lane issues each TMA, arrive,
  // MMA or commit (see the *_elected wrappers).
  if (warp == 0 || warp == T::kActWarpB) {
    // ------------------------------------- activation producers (2, alternate groups)
    const int first = warp == 0 ? 0 : 1;
    int issued = 0;
    for (int i = first; i < ng; i += 2) {
      const int s = i % AS;
      if (!warp_wait(act_empty0 + 8 * s, ((i / AS) & 1) ^ 1, abort_flag, limit)) break;
      const uint32_t full = act_full0 + 8 * s;
      mbar_arrive_expect_tx_elected(full, T::kActStageBytes);
      const uint32_t dst = smem_addr(smem + T::kActOff + s * T::kActStageBytes);
      const int k = (g_begin + i) * kGroup;
#pragma unroll
      for (int h = 0; h < T::kHalves; ++h) {  // rows m0 + h * kMmaN .. of each K slice
        tma_load_2d_elected(dst + h * T::kHalfBytes, &tmap_act, full, k, m0 + h * T::kMmaN);
        tma_load_2d_elected(dst + T::kSliceBytes + h * T::kHalfBytes, &tmap_act, full, k + 64, m0 + h * T::kMmaN);
      }
      issued = i + 1;
    }
    if (*abort_flag) {  // let copies in flight land before the CTA's memory goes away
      for (int i = first; i < issued; i += 2) {
        const uint64_t t0 = global_timer_ns();
        while (!mbar_try_wait(act_full0 + 8 * (i % AS), (i / AS) & 1) && global_timer_ns() - t0 < limit) {
        }
      }
    }
  } else if (warp == 2) {
    // ------------------------------------------------ packed-word producer
    if (args.scale_box > 0) {
      // The tile's scales: 128 rows x scale_box groups from an 8-aligned
      // group column (TMA needs 16-byte aligned starts).
      mbar_arrive_expect_tx_elected(s_full, static_cast<uint32_t>(args.scale_box) * T::kRows * 2);
      tma_load_2d_elected(smem_addr(smem + T::kScaleOff), &tmap_s, s_full, g_begin & ~7, n0);
    }
    int issued = 0;
    const int nw = (ng + T::kWGroups - 1) / T::kWGroups;
    for (int i = 0; i < nw; ++i) {
      const int s = i % WS;
      if (!warp_wait(w_empty0 + 8 * s, ((i / WS) & 1) ^ 1, abort_flag, limit)) break;
      const uint32_t full = w_full0 + 8 * s;
      mbar_arrive_expect_tx_elected(full, T::kWStageBytes);
      tma_load_2d_elected(smem_addr(smem + T::kWOff + s * T::kWStageBytes), &tmap_w, full,
                          word_stage_x<MODE>(g_begin + i * T::kWGroups), n0);
      issued = i + 1;
    }
    if (*abort_flag) {
      for (int i = issued > WS ? issued - WS : 0; i < issued; ++i) {
        const uint64_t t0 = global_timer_ns();
        while (!mbar_try_wait(w_full0 + 8 * (i % WS), (i / WS) & 1) && global_timer_ns() - t0 < limit) {
        }
      }
      if (args.scale_box > 0) {  // the scale tile's copy, which the converters may not have waited for
        const uint64_t t0 = global_timer_ns();
        while (!mbar_try_wait(s_full, 0) && global_timer_ns() - t0 < limit) {
        }
      }
    }
  } else if (warp == 1 || warp == T::kMmaWarpB) {
    // ------------------------------------------------------- MMA issuers
    constexpr int P = T::kMmaThreads;
    constexpr int kOwnAccs = T::kAccs / P;  // accumulators per issuing warp
    const int first = warp == 1 ? 0 : 1;
    if (first < P) {
      constexpr uint32_t idesc = f16_instr_desc(128, T::kMmaN);
      // Descriptor of act stage 0; other stages and K steps add their byte
      // offset >> 4 to the start-address field (no carry: shared memory
      // addresses stay below 256 KB).
      const uint64_t desc0 = sw128_kmajor_desc(smem_addr(smem + T::kActOff));
      int step = 0;  // this warp's MMA count
      for (int i = first; i < ng; i += P) {
        const int sa = i % AS, st = i % TS;
        if (!warp_wait(act_full0 + 8 * sa, (i / AS) & 1, abort_flag, limit)) break;
        if (!warp_wait(t_ready0 + 8 * st, (i / TS) & 1, abort_flag, limit)) break;
        tc_fence_after_sync();
        const uint64_t desc_s = desc0 + static_cast<uint64_t>((sa * T::kActStageBytes) >> 4);
        const uint32_t a_cols = tmem + T::kACol0 + st * 64;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint64_t bdesc = desc_s + static_cast<uint64_t>(((kk >> 2) * T::kSliceBytes + (kk & 3) * 32) >> 4);
          const int acc = (step % kOwnAccs) * P + first;
#pragma unroll
          for (int h = 0; h < T::kHalves; ++h)  // half h: tokens h * kMmaN .., accumulator at column h * kHalfCol
            mma_f16_tmem_a_elected(tmem + acc * BLOCK_T + h * T::kHalfCol, a_cols + kk * 8,
                                   bdesc + static_cast<uint64_t>((h * T::kHalfBytes) >> 4), idesc,
                                   step >= kOwnAccs ? 1u : 0u);
          ++step;
        }
        mma_commit_elected(act_empty0 + 8 * sa);
        mma_commit_elected(t_free0 + 8 * st);
      }
      mma_commit_elected(dfull);  // also on abort: lets this warp see its MMAs drain
      if (*abort_flag) {
        const uint64_t t0 = global_timer_ns();
        while (!mbar_try_wait(dfull, 0) && global_timer_ns() - t0 < limit) {
        }
      }
    }
  } else {
    // ------------------------------------------------ converters, epilogue
    // The warps of a TMEM lane quadrant take groups in turn, so that one's
    // barrier waits and latencies overlap the others' conversion.
    const int quad = warp & 3;  // a warp may only touch TMEM lanes 32*(warp%4) .. +31
    const int turn = (warp - 3) >> 2;  // 0 .. kWarpsPerQuad-1
    const int row = quad * 32 + lane;
    const int n = n0 + row;
    const uint32_t lane_base = static_cast<uint32_t>(quad * 32) << 16;
    const uint16_t* srow = args.scales + static_cast<size_t>(n) * groups + g_begin;
    const bool row_ok = n < args.N;
    // Scales: the whole tile's in shared memory when they fit, by one TMA
    // (scale_box > 0) or by batched loads; else two groups ahead in registers.
    const bool by_tma = args.scale_box > 0;
    const bool staged = by_tma || (T::kScaleBytes > 0 && T::kRows * ng * 2 <= T::kScaleBytes);
    const int s_stride = by_tma ? args.scale_box : ng;  // groups per row in the staged tile
    const int s_first = by_tma ? g_begin - (g_begin & ~7) : 0;
    uint16_t* sstage = reinterpret_cast<uint16_t*>(smem + T::kScaleOff);
    if (!by_tma && staged) {
      const int ct = threadIdx.x - 96;  // 0 .. 32 * kConvWarps - 1 over the converter warps
      constexpr int kBatch = 8;         // independent loads in flight per thread
      for (int e0 = ct; e0 < T::kRows * ng; e0 += kBatch * 32 * T::kConvWarps) {
        uint16_t v[kBatch];
#pragma unroll
        for (int u = 0; u < kBatch; ++u) {
          const int e = e0 + u * 32 * T::kConvWarps;
          const int r = e / ng, g = e - (e / ng) * ng;
          v[u] = (e < T::kRows * ng && n0 + r < args.N)
                     ? __ldg(args.scales + static_cast<size_t>(n0 + r) * groups + g_begin + g)
                     : uint16_t(0);
        }
#pragma unroll
        for (int u = 0; u < kBatch; ++u)
          if (e0 + u * 32 * T::kConvWarps < T::kRows * ng) sstage[e0 + u * 32 * T::kConvWarps] = v[u];
      }
      named_barrier_sync(2, 32 * T::kConvWarps);
    }
    uint32_t sq0 = 0, sq1 = 0, zq0 = 0, zq1 = 0;
    bool ok = !by_tma || warp_wait(s_full, 0, abort_flag, limit);
    constexpr int kStep = T::kWarpsPerQuad;
    // Scale (4-bit weights: the group's two scales, and two zeros) of group i.
    const uint32_t* srow2 =
        T::kHqq ? reinterpret_cast<const uint32_t*>(args.scales) + static_cast<size_t>(n) * groups + g_begin : nullptr;
    const uint32_t* zrow2 =
        T::kHqq ? reinterpret_cast<const uint32_t*>(args.zeros) + static_cast<size_t>(n) * groups + g_begin : nullptr;
    auto scale_at = [&](int i) -> uint32_t {
      if (!row_ok || i >= ng) return 0u;
      if constexpr (T::kHqq) return __ldg(srow2 + i);
      return __ldg(srow + i);
    };
    auto zero_at = [&](int i) -> uint32_t {
      if constexpr (T::kHqq) return (row_ok && i < ng) ? __ldg(zrow2 + i) : 0u;
      return 0u;
    };
    if (!staged) {
      sq0 = scale_at(turn);
      sq1 = scale_at(turn + kStep);
      zq0 = zero_at(turn);
      zq1 = zero_at(turn + kStep);
    }
    for (int i = turn; ok && i < ng; i += kStep) {
      const int wj = i / T::kWGroups;  // word stage of this group
      const int sw = wj % WS, st = i % TS;
      uint32_t sc, zc = 0;
      if (staged) {
        sc = sstage[row * s_stride + s_first + i];
      } else {
        sc = sq0;
        sq0 = sq1;
        sq1 = scale_at(i + 2 * kStep);
        zc = zq0;
        zq0 = zq1;
        zq1 = zero_at(i + 2 * kStep);
      }
      ok = warp_wait(w_full0 + 8 * sw, (wj / WS) & 1, abort_flag, limit) &&
           warp_wait(t_free0 + 8 * st, ((i / TS) & 1) ^ 1, abort_flag, limit);
      if (!ok) break;
      tc_fence_after_sync();  // the MMAs that read this TMEM stage are done
      const uint8_t* wstage = smem + T::kWOff + sw * T::kWStageBytes;
      // 128-byte swizzle: 16-byte chunk c of row r sits at chunk c ^ (r % 8).
      const int pos = i % T::kWGroups;
      const uint8_t* wrow = wstage + row * T::kWRowBytes;
      uint32_t words[T::kWordsPerGroup];
      if constexpr (T::kB3) {
        b3_group_words(reinterpret_cast<const uint32_t*>(wrow), pos, words);
      } else if constexpr (T::kHqq) {
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          const uint4 q = *reinterpret_cast<const uint4*>(wrow + 16 * ((4 * pos + c) ^ (row & 7)));
          words[4 * c] = q.x;
          words[4 * c + 1] = q.y;
          words[4 * c + 2] = q.z;
          words[4 * c + 3] = q.w;
        }
      } else if (MODE == BONSAI_BINARY) {
        const uint4 q = *reinterpret_cast<const uint4*>(wrow + 16 * (pos ^ (row & 7)));
        words[0] = q.x;
        words[1] = q.y;
        words[2] = q.z;
        words[3] = q.w;
      } else {
        const uint4 q0 = *reinterpret_cast<const uint4*>(wrow + 16 * ((2 * pos) ^ (row & 7)));
        const uint4 q1 = *reinterpret_cast<const uint4*>(wrow + 16 * ((2 * pos + 1) ^ (row & 7)));
        words[0] = q0.x;
        words[1] = q0.y;
        words[2] = q0.z;
        words[3] = q0.w;
        words[4] = q1.x;
        words[5] = q1.y;
        words[6] = q1.z;
        words[7] = q1.w;
      }
      __syncwarp();
      // Release the word stage after this warp's last group in it.  The
      // stage's readers (kWReaders) each have a group in every full stage;
      // only the CTA's last stage, which is never refilled, may lack some
      // readers' arrivals.
      const int stage_end = (wj + 1) * T::kWGroups < ng ? (wj + 1) * T::kWGroups : ng;
      if (lane == 0 && i + kStep >= stage_end) mbar_arrive(w_empty0 + 8 * sw);
      if constexpr (T::kB3)
        convert_group_b3(words, sc | (sc << 16), tmem + lane_base + T::kACol0 + st * 64);
      else if constexpr (T::kHqq)
        convert_group_hqq4(words, sc, zc, tmem + lane_base + T::kACol0 + st * 64);
      else
        convert_group<MODE>(words, sc | (sc << 16), tmem + lane_base + T::kACol0 + st * 64);
      tmem_store_wait();
      tc_fence_before_sync();
      __syncwarp();
      if (lane == 0) mbar_arrive(t_ready0 + 8 * st);
    }
    if (ok) ok = warp_wait(dfull, 0, abort_flag, limit);
    if (ok) tc_fence_after_sync();
    constexpr int kEpiCols = BLOCK_T / T::kEpiWarpsPerQuad;  // token columns per epilogue warp
    // With two issuing threads and a single group, the second accumulator is unused.
    const int used_accs = (T::kMmaThreads == 2 && ng < 2) ? 1 : T::kAccs;
    const bool epi = turn < T::kEpiWarpsPerQuad;
    const int c_begin = turn * kEpiCols;
    // TMEM column of token column c (8-column runs never straddle the halves).
    auto acc_col = [](int c) { return c < T::kMmaN ? c : c - T::kMmaN + T::kHalfCol; };
    if (args.ksplit == 1) {
      // FP16 tile [BLOCK_T tokens][128 rows] in the (now idle) act ring.
      uint16_t* tile = reinterpret_cast<uint16_t*>(smem + T::kActOff);
      if (ok && epi) {
#pragma unroll 1
        for (int c = 0; c < kEpiCols; c += 8) {
          float acc[8];
          sum_accumulators<T::kAccs, BLOCK_T>(tmem + lane_base + acc_col(c_begin + c), used_accs, acc);
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            const __half h = __float2half_rn(acc[j] * T::kOutScale);
            tile[(c_begin + c + j) * T::kRows + row] = __half_as_ushort(h);
          }
        }
      }
      fence_proxy_async_smem();
      named_barrier_sync(1, 32 * T::kConvWarps);
      if (*abort_flag == 0) {
        if (args.tma_store) {
          if (warp == 3 && lane == 0) {
            // Halves that start past the last token are not stored (a store
            // box starts inside the tensor).
#pragma unroll
            for (int h = 0; h < T::kHalves; ++h)
              if (h == 0 || m0 + h * T::kMmaN < args.M)
                tma_store_2d(&tmap_out, smem_addr(tile) + h * T::kMmaN * T::kRows * 2, n0, m0 + h * T::kMmaN);
            bulk_commit_group();
            bulk_wait_group_read0();
          }
        } else {
          const int ct = threadIdx.x - 96;  // 0 .. 32 * kConvWarps - 1 over the converter warps
          for (int e = ct; e < BLOCK_T * T::kRows; e += 32 * T::kConvWarps) {
            const int m = m0 + e / T::kRows, nn = n0 + e % T::kRows;
            if (m < args.M && nn < args.N) args.out[static_cast<size_t>(m) * args.N + nn] = tile[e];
          }
        }
      }
    } else if (ok && epi) {
      // FP32 partial [BLOCK_T tokens][128 rows] in the act ring.
      float* part = reinterpret_cast<float*>(smem + T::kActOff);
#pragma unroll 1
      for (int c = 0; c < kEpiCols; c += 8) {
        float acc[8];
        sum_accumulators<T::kAccs, BLOCK_T>(tmem + lane_base + acc_col(c_begin + c), used_accs, acc);
#pragma unroll
        for (int j = 0; j < 8; ++j) part[(c_begin + c + j) * T::kRows + row] = acc[j];
      }
    }
  }

  if (args.ksplit > 1) {
    __syncwarp();
    cluster_sync();  // every partial of the cluster is written
    if (*abort_flag == 0) {
      // This CTA's share of the tile, in runs of 4 consecutive rows of one
      // token: 16-byte loads from every CTA's partial, added in rank order.
      const uint32_t part = smem_addr(smem + T::kActOff);
      const int rank = static_cast<int>(cluster_ctarank());
      constexpr int Q = T::kRows * BLOCK_T / 4;
      const int q_begin = rank * Q / args.ksplit, q_end = (rank + 1) * Q / args.ksplit;
      for (int q = q_begin + threadIdx.x; q < q_end; q += T::kThreads) {
        const int m = (4 * q) / T::kRows, r = (4 * q) % T::kRows;
        const uint32_t local = part + 16u * static_cast<uint32_t>(q);
        float4 v[8];
#pragma unroll
        for (int j = 0; j < 8; ++j)
          if (j < args.ksplit) v[j] = ld_dsmem_f32x4(map_to_rank(local, j));
        float4 sum = v[0];
#pragma unroll
        for (int j = 1; j < 8; ++j)
          if (j < args.ksplit) {
            sum.x += v[j].x;
            sum.y += v[j].y;
            sum.z += v[j].z;
            sum.w += v[j].w;
          }
        const int gm = m0 + m;
        if (gm < args.M) {
          const float vals[4] = {sum.x, sum.y, sum.z, sum.w};
          uint16_t* dst = args.out + static_cast<size_t>(gm) * args.N + n0 + r;
#pragma unroll
          for (int j = 0; j < 4; ++j)
            if (n0 + r + j < args.N) dst[j] = __half_as_ushort(__float2half_rn(vals[j] * T::kOutScale));
        }
      }
    }
    cluster_sync();  // no CTA leaves while another still reads its partial
  }

  tc_fence_before_sync();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after_sync();
    tmem_dealloc(tmem, T::kTmemCols);
  }
}

// Bounded-wait self-test: waits on a barrier no one arrives at.
__global__ void wait_timeout_selftest_kernel(uint64_t limit_ns) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(smem_addr(&bar), 1);
    abort_flag = 0;
    fence_barrier_init();
  }
  __syncthreads();
  wait_phase(smem_addr(&bar), 0, &abort_flag, limit_ns);
}

}  // namespace bonsai

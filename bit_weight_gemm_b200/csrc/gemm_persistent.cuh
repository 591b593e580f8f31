// gemm_persistent.cuh - the large-M form of the fused dequantise + GEMM:
// one persistent CTA per SM walks a list of 128-row x BLOCK_T-token output
// tiles (BLOCK_T = 256, or 192 where 256-token tiles leave a wave part-empty).
//
// Same arithmetic, operand layout and stages as lowbit_gemm_kernel (see
// gemm_tc.cuh): converters turn packed words into exact FP16 products in
// tensor memory, one thread issues tcgen05.mma (M=128 weight rows, N=BLOCK_T
// tokens, K=16) with A from TMEM and B (activations) from shared memory, and
// the FP32 sum is rounded once to FP16.  What changes is the tile boundary.
// With one tile per CTA, each tile paid for its own start (first activation
// and word copies, first conversion) and its own end (accumulator read-out,
// output store, CTA exit) with the tensor core idle, about a quarter of the
// time at K = 3072.  Here the rings run on across tiles:
//
//   - the activation and word producers and the converters count groups over
//     the CTA's whole tile list, so the next tile's copies and conversions
//     start while the current tile's last MMAs run;
//   - at a tile's end each converter warp first converts its first group of
//     the next tile when that TMEM stage is already free, then reads its
//     64 x 32-lane share of the accumulator into registers and releases the
//     accumulator (acc_empty); the MMA warp starts the next tile on that
//     barrier while the converters round and store the finished tile from
//     registers.
//
// The tensor core thus idles at a tile boundary only for the read-out of the
// accumulator.  Requirements (checked by the host): more tiles than fit in one
// wave, and K a multiple of 128 x max(4, groups in one word stage) (512 for
// INT2, base-3 and 4-bit weights, 1024 binary), so that word stages never
// straddle two tiles and every converter warp keeps its TMEM stage.
#pragma once

#include "gemm_tc.cuh"

namespace bonsai {

template <int MODE, int BLOCK_T>
struct PersistTile {
  static constexpr int kBlockT = BLOCK_T;  // tokens per tile (MMA N)
  static constexpr int kRows = 128;    // weight rows per tile (MMA M)
  static constexpr bool kB3 = MODE == BONSAI_TERNARY_B3;
  static constexpr bool kHqq = MODE == kModeHqq4;
  static constexpr int kWordsPerGroup = MODE == BONSAI_BINARY ? 4 : (kB3 ? 7 : (kHqq ? 16 : 8));  // held per group
  static constexpr int kWGroups = kB3 ? kB3BlockGroups : 32 / kWordsPerGroup;  // groups per word stage
  static constexpr int kWRowBytes = kB3 ? kB3BlockBytes : 128;                  // bytes of a row per stage
  static constexpr int kSliceBytes = kBlockT * 128;     // BLOCK_T rows x 64 FP16
  static constexpr int kActStageBytes = 2 * kSliceBytes;
  static constexpr int kActStages = 3;
  static constexpr int kWStageBytes = kRows * kWRowBytes;
  static constexpr int kWStages = 2;
  static constexpr int kConvWarps = 16;  // four per TMEM lane quadrant
  static constexpr int kWarpsPerQuad = 4;
  static constexpr int kThreads = 32 * (3 + kConvWarps);
  static constexpr int kACol0 = kBlockT;  // one accumulator, then the converted-weight stages
  static constexpr int kTmemCols = 512;
  static constexpr int kTStages = 4;
  static constexpr int kEpiCols = kBlockT / kWarpsPerQuad;  // accumulator columns per converter warp
  static constexpr int kActOff = 0;
  static constexpr int kWOff = kActStages * kActStageBytes;
  static constexpr int kBarOff = kWOff + kWStages * kWStageBytes;
  static constexpr int kNumBars = 2 * kActStages + 2 * kTStages + 2 * kWStages + 2;
  static constexpr int kMiscOff = kBarOff + kNumBars * 8;
  static constexpr int kSmemBytes = kMiscOff + 16 + 1024;  // + slack to align the base to 1024
  static constexpr float kOutScale = MODE == BONSAI_TERNARY_INT2 ? 0.5f : 1.0f;  // INT2 converts to 2ts
  // A converter warp takes the groups i = turn (mod 4) of every tile and
  // TMEM stage c % 4 of the running group count c: with four stages and
  // every tile's group count a multiple of four, warp `turn` always uses
  // stage `turn`, and its first group of a tile reuses the stage of the
  // previous tile's group ng - 4 + turn.
  static_assert(kTStages == 4 && kWarpsPerQuad == 4, "stage ownership by turn");
  static_assert(kACol0 + kTStages * 64 <= kTmemCols, "TMEM budget");
  static_assert(kBlockT % 64 == 0 && kBlockT <= 256 && kSliceBytes % 1024 == 0, "tile width");
  // Converter warps reading each word stage: all 16, or (4-bit weights, 2
  // groups per stage) the 4 warps of each of its groups.
  static constexpr int kWReaders = 4 * (kWGroups < kWarpsPerQuad ? kWGroups : kWarpsPerQuad);
  static_assert(kEpiCols % 16 == 0, "read-out in 16-column batches");
  static_assert(kSmemBytes <= 227 * 1024, "shared memory per CTA");
};

struct PersistArgs {
  const uint16_t* scales;
  const uint16_t* zeros;  // 4-bit group-affine weights only
  uint16_t* out;
  int M, N, K;
  int tiles_n;  // 128-row tiles along N; tile tau covers rows (tau % tiles_n) and tokens (tau / tiles_n)
  int tiles;    // tiles_n x BLOCK_T-token tiles along M
  uint64_t wait_limit_ns;
};

template <int MODE, int BLOCK_T>
__global__ void __launch_bounds__(PersistTile<MODE, BLOCK_T>::kThreads, 1)
    lowbit_gemm_persistent_kernel(const __grid_constant__ CUtensorMap tmap_act,
                                  const __grid_constant__ CUtensorMap tmap_w, const PersistArgs args) {
  using T = PersistTile<MODE, BLOCK_T>;
  constexpr int AS = T::kActStages, TS = T::kTStages, WS = T::kWStages;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + T::kBarOff);
  const uint32_t act_full0 = smem_addr(bars);
  const uint32_t act_empty0 = smem_addr(bars + AS);
  const uint32_t t_ready0 = smem_addr(bars + 2 * AS);
  const uint32_t t_free0 = smem_addr(bars + 2 * AS + TS);
  const uint32_t w_full0 = smem_addr(bars + 2 * AS + 2 * TS);
  const uint32_t w_empty0 = smem_addr(bars + 2 * AS + 2 * TS + WS);
  const uint32_t acc_full = smem_addr(bars + 2 * AS + 2 * TS + 2 * WS);       // tile's last MMA done
  const uint32_t acc_empty = smem_addr(bars + 2 * AS + 2 * TS + 2 * WS + 1);  // accumulator read out
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + T::kMiscOff);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + T::kMiscOff + 4);

  const int warp = __shfl_sync(0xffffffffu, static_cast<int>(threadIdx.x >> 5), 0);
  const int lane = threadIdx.x & 31;
  const int groups = args.K / kGroup;  // per tile
  const int ntiles = args.tiles > static_cast<int>(blockIdx.x)
                         ? (args.tiles - static_cast<int>(blockIdx.x) + static_cast<int>(gridDim.x) - 1) /
                               static_cast<int>(gridDim.x)
                         : 0;
  const uint64_t limit = args.wait_limit_ns;
  // Tile `it` of this CTA: rows n0 .. n0+127, tokens m0 .. m0+255.
  auto tile_n0 = [&](int it) { return ((blockIdx.x + it * gridDim.x) % args.tiles_n) * T::kRows; };
  auto tile_m0 = [&](int it) { return static_cast<int>((blockIdx.x + it * gridDim.x) / args.tiles_n) * T::kBlockT; };

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
      mbar_init(w_empty0 + 8 * s, T::kWReaders);
    }
    mbar_init(acc_full, 1);
    mbar_init(acc_empty, T::kConvWarps);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_map(&tmap_act);
    tma_prefetch_map(&tmap_w);
  }
  if (warp == 1) {
    tmem_alloc(smem_addr(tmem_slot), T::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tmem = __shfl_sync(0xffffffffu, *tmem_slot, 0);
  // Dependents may launch once this CTA holds its tensor memory (see
  // lowbit_gemm_kernel: a dependent CTA may wait for these columns, never the
  // reverse).
  if (threadIdx.x == 0) griddep_launch_dependents();
  griddep_wait();

  if (warp == 0) {
    // ------------------------------------------------ activation producer
    int last = -1;  // running index of the latest copy
    bool ok = true;
    for (int it = 0; ok && it < ntiles; ++it) {
      const int m0 = tile_m0(it);
      for (int i = 0; i < groups; ++i) {
        const int c = it * groups + i;
        const int s = c % AS;
        if (!(ok = warp_wait(act_empty0 + 8 * s, ((c / AS) & 1) ^ 1, abort_flag, limit))) break;
        const uint32_t full = act_full0 + 8 * s;
        mbar_arrive_expect_tx_elected(full, T::kActStageBytes);
        const uint32_t dst = smem_addr(smem + T::kActOff + s * T::kActStageBytes);
        tma_load_2d_elected(dst, &tmap_act, full, i * kGroup, m0);
        tma_load_2d_elected(dst + T::kSliceBytes, &tmap_act, full, i * kGroup + 64, m0);
        last = c;
      }
    }
    if (*abort_flag) {  // copies still in flight are among the last AS running groups
      for (int c = last; c >= 0 && c > last - AS; --c) {
        const uint64_t t0 = global_timer_ns();
        while (!mbar_try_wait(act_full0 + 8 * (c % AS), (c / AS) & 1) && global_timer_ns() - t0 < limit) {
        }
      }
    }
  } else if (warp == 2) {
    // ------------------------------------------------ packed-word producer
    const int nw = groups / T::kWGroups;  // word stages per tile
    int last = -1;
    bool ok = true;
    for (int it = 0; ok && it < ntiles; ++it) {
      const int n0 = tile_n0(it);
      for (int j = 0; j < nw; ++j) {
        const int wc = it * nw + j;
        const int s = wc % WS;
        if (!(ok = warp_wait(w_empty0 + 8 * s, ((wc / WS) & 1) ^ 1, abort_flag, limit))) break;
        const uint32_t full = w_full0 + 8 * s;
        mbar_arrive_expect_tx_elected(full, T::kWStageBytes);
        tma_load_2d_elected(smem_addr(smem + T::kWOff + s * T::kWStageBytes), &tmap_w, full,
                            word_stage_x<MODE>(j * T::kWGroups), n0);
        last = wc;
      }
    }
    if (*abort_flag) {
      for (int wc = last; wc >= 0 && wc > last - WS; --wc) {
        const uint64_t t0 = global_timer_ns();
        while (!mbar_try_wait(w_full0 + 8 * (wc % WS), (wc / WS) & 1) && global_timer_ns() - t0 < limit) {
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------- MMA issuer
    constexpr uint32_t idesc = f16_instr_desc(128, T::kBlockT);
    const uint64_t desc0 = sw128_kmajor_desc(smem_addr(smem + T::kActOff));
    int done_tiles = 0;  // acc_full commits so far
    bool ok = true;
    for (int it = 0; ok && it < ntiles; ++it) {
      // The converters have read the previous tile's accumulator.
      if (!(ok = warp_wait(acc_empty, (it & 1) ^ 1, abort_flag, limit))) break;
      tc_fence_after_sync();
      for (int i = 0; i < groups; ++i) {
        const int c = it * groups + i;
        const int sa = c % AS, st = c % TS;
        if (!(ok = warp_wait(act_full0 + 8 * sa, (c / AS) & 1, abort_flag, limit))) break;
        if (!(ok = warp_wait(t_ready0 + 8 * st, (c / TS) & 1, abort_flag, limit))) break;
        tc_fence_after_sync();
        const uint64_t desc_s = desc0 + static_cast<uint64_t>((sa * T::kActStageBytes) >> 4);
        const uint32_t a_cols = tmem + T::kACol0 + st * 64;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint64_t bdesc = desc_s + static_cast<uint64_t>(((kk >> 2) * T::kSliceBytes + (kk & 3) * 32) >> 4);
          mma_f16_tmem_a_elected(tmem, a_cols + kk * 8, bdesc, idesc, (i | kk) != 0 ? 1u : 0u);
        }
        mma_commit_elected(act_empty0 + 8 * sa);
        mma_commit_elected(t_free0 + 8 * st);
      }
      if (!ok) break;
      mma_commit_elected(acc_full);
      ++done_tiles;
    }
    if (*abort_flag) {  // let the MMAs already issued drain before TMEM is freed
      mma_commit_elected(acc_full);
      const uint64_t t0 = global_timer_ns();
      while (!mbar_try_wait(acc_full, done_tiles & 1) && global_timer_ns() - t0 < limit) {
      }
    }
  } else if (warp >= 3 && warp < 3 + T::kConvWarps) {
    // --------------------------------------- converters and read-out
    const int quad = warp & 3;         // TMEM lanes 32*quad .. +31
    const int turn = (warp - 3) >> 2;  // groups i = turn (mod 4); TMEM stage `turn`
    const int row = quad * 32 + lane;
    const uint32_t lane_base = static_cast<uint32_t>(quad * 32) << 16;
    const int nw = groups / T::kWGroups;
    const int c_begin = turn * T::kEpiCols;  // this warp's accumulator columns (tokens)
    // The stage of a tile's first group `turn` is freed by the previous
    // tile's group ng - 4 + turn; only for turn 3 is that the last group, so
    // the other warps convert first and read out afterwards.
    const bool convert_first = turn < TS - 1;
    bool ok = true;

    // The group's scale (4-bit weights: its two scales, and the two zeros).
    auto scale_of = [&](int it, int i) -> uint32_t {
      const int n = tile_n0(it) + row;
      if (it >= ntiles || n >= args.N) return 0u;
      if constexpr (T::kHqq)
        return __ldg(reinterpret_cast<const uint32_t*>(args.scales) + static_cast<size_t>(n) * groups + i);
      return static_cast<uint32_t>(__ldg(args.scales + static_cast<size_t>(n) * groups + i));
    };
    auto zero_of = [&](int it, int i) -> uint32_t {
      if constexpr (T::kHqq) {
        const int n = tile_n0(it) + row;
        if (it >= ntiles || n >= args.N) return 0u;
        return __ldg(reinterpret_cast<const uint32_t*>(args.zeros) + static_cast<size_t>(n) * groups + i);
      }
      return 0u;
    };

    // Convert group i of tile it (running index c) into TMEM stage `turn`.
    auto convert = [&](int it, int i, uint32_t sc, uint32_t zc) -> bool {
      const int c = it * groups + i;
      const int wc = it * nw + i / T::kWGroups;
      const int sw = wc % WS;
      if (!warp_wait(w_full0 + 8 * sw, (wc / WS) & 1, abort_flag, limit)) return false;
      if (!warp_wait(t_free0 + 8 * turn, ((c / TS) & 1) ^ 1, abort_flag, limit)) return false;
      tc_fence_after_sync();
      const uint8_t* wrow = smem + T::kWOff + sw * T::kWStageBytes + row * T::kWRowBytes;
      const int pos = i % T::kWGroups;
      uint32_t words[T::kWordsPerGroup];
      if constexpr (T::kB3) {
        b3_group_words(reinterpret_cast<const uint32_t*>(wrow), pos, words);
      } else if constexpr (T::kHqq) {
#pragma unroll
        for (int q4 = 0; q4 < 4; ++q4) {
          const uint4 q = *reinterpret_cast<const uint4*>(wrow + 16 * ((4 * pos + q4) ^ (row & 7)));
          words[4 * q4] = q.x;
          words[4 * q4 + 1] = q.y;
          words[4 * q4 + 2] = q.z;
          words[4 * q4 + 3] = q.w;
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
      // Each reader has kWGroups / 4 groups of a word stage (or one, when a
      // stage holds fewer groups than a quadrant has warps); release after the last.
      if (lane == 0 && pos + T::kWarpsPerQuad >= T::kWGroups) mbar_arrive(w_empty0 + 8 * sw);
      if constexpr (T::kB3)
        convert_group_b3(words, sc | (sc << 16), tmem + lane_base + T::kACol0 + turn * 64);
      else if constexpr (T::kHqq)
        convert_group_hqq4(words, sc, zc, tmem + lane_base + T::kACol0 + turn * 64);
      else
        convert_group<MODE>(words, sc | (sc << 16), tmem + lane_base + T::kACol0 + turn * 64);
      tmem_store_wait();
      tc_fence_before_sync();
      __syncwarp();
      if (lane == 0) mbar_arrive(t_ready0 + 8 * turn);
      return true;
    };

    // Read this warp's share of tile it's accumulator, release it, then round
    // and store: row n, tokens m0 + c_begin .. + kEpiCols - 1.
    auto read_out = [&](int it) -> bool {
      if (!warp_wait(acc_full, it & 1, abort_flag, limit)) return false;
      tc_fence_after_sync();
      uint32_t h[T::kEpiCols / 2];  // FP16 pairs (token 2j, 2j+1)
#pragma unroll
      for (int b = 0; b < T::kEpiCols; b += 16) {
        uint32_t v[16];
        tmem_load_16(tmem + lane_base + c_begin + b, v);
        tmem_load_wait();
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const __half lo = __float2half_rn(__uint_as_float(v[2 * j]) * T::kOutScale);
          const __half hi = __float2half_rn(__uint_as_float(v[2 * j + 1]) * T::kOutScale);
          h[b / 2 + j] = static_cast<uint32_t>(__half_as_ushort(lo)) |
                         (static_cast<uint32_t>(__half_as_ushort(hi)) << 16);
        }
      }
      tc_fence_before_sync();
      __syncwarp();
      if (lane == 0) mbar_arrive(acc_empty);
      const int n = tile_n0(it) + row;
      const int m_first = tile_m0(it) + c_begin;
      if (n < args.N && *abort_flag == 0) {
        uint16_t* dst = args.out + static_cast<size_t>(m_first) * args.N + n;
        const int rows_left = args.M - m_first;  // tokens of this warp's 64 that exist
#pragma unroll
        for (int j = 0; j < T::kEpiCols / 2; ++j) {
          if (2 * j < rows_left) *dst = static_cast<uint16_t>(h[j]);
          dst += args.N;
          if (2 * j + 1 < rows_left) *dst = static_cast<uint16_t>(h[j] >> 16);
          dst += args.N;
        }
      }
      return true;
    };

    uint32_t sc_next = scale_of(0, turn), zc_next = zero_of(0, turn);
    for (int it = 0; ok && it < ntiles; ++it) {
      for (int i = turn; i < groups; i += T::kWarpsPerQuad) {
        const uint32_t sc = sc_next, zc = zc_next;
        const bool last_of_tile = i + T::kWarpsPerQuad >= groups;
        sc_next = last_of_tile ? scale_of(it + 1, turn) : scale_of(it, i + T::kWarpsPerQuad);
        zc_next = last_of_tile ? zero_of(it + 1, turn) : zero_of(it, i + T::kWarpsPerQuad);
        const bool first_of_tile = i == turn && it > 0;
        if (first_of_tile && !convert_first && !(ok = read_out(it - 1))) break;
        if (!(ok = convert(it, i, sc, zc))) break;
        if (first_of_tile && convert_first && !(ok = read_out(it - 1))) break;
      }
    }
    if (ok && ntiles > 0) read_out(ntiles - 1);
  }

  tc_fence_before_sync();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after_sync();
    tmem_dealloc(tmem, T::kTmemCols);
  }
}

}  // namespace bonsai

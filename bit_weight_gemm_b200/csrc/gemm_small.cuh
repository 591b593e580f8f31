// gemm_small.cuh - the bandwidth-bound form of the fused dequantise + GEMM:
// up to 16 tokens, where the packed weights are the whole cost.
//
// Same product as lowbit_gemm_kernel (gemm_tc.cuh): D^T = W * A^T with the
// weights as the MMA's M side, fed from tensor memory, tcgen05.mma kind::f16
// (M=128 weight rows, N=16 tokens, K=16) accumulating in FP32.  What changes
// is where the time goes.  At 16 tokens a launch streams 7.5 MB of packed
// weights and does little else, so the kernel is built around three facts
// measured on B200:
//
//  - Weights do not depend on the previous kernel in the stream, activations
//    do.  A CTA copies its whole slice of packed words into shared memory as
//    soon as it starts, before griddepcontrol.wait, and converts the first
//    groups into tensor memory while the previous kernel may still run on
//    other SMs.  (A kernel that allocates tensor memory gets one CTA per SM,
//    so a launch's CTAs start as the previous launch's leave their SMs.)  The
//    caller's side of this: packed and scales must not be written by the
//    kernel launched just before on the same stream.
//  - The scale is applied after the MMA.  Converting a group is then a shift
//    and a mask per pair of weights (INT2: the field is 2t; binary: the sign
//    over 1.0; base-3: the digit step), a third fewer instructions than with
//    the FP16 multiply, and the conversion is issue-bound.  Each TMEM stage
//    carries its own 16-column FP32 accumulator: the MMAs of one group write
//    it (the first with accumulate off), and the converter warp that owns the
//    stage reads it back before converting its next group into the stage,
//    adding s_g * D_g into registers.
//  - Equal work per CTA in one wave: the launch is tiles x ksplit CTAs, every
//    CTA holding the same number of 128-wide groups (at most 24).  With no
//    split on at most half the SMs, the next launch's CTAs start on the other
//    half while this one runs; otherwise ksplit is the largest split (up to
//    5) whose clusters all fit on the GPU at once.  The ksplit
//    CTAs of a tile form a cluster: ranks 1.. push their FP32 partial tile
//    into rank 0's shared memory with st.async, counted on rank 0's mbarrier,
//    and leave; rank 0 adds the partials in rank order (deterministic),
//    rounds once to FP16 and stores.
//
// Warps: 0 allocates TMEM and copies (words before the wait, activations
// after); 1..24 convert, six per TMEM lane quadrant: warp `turn` of a
// quadrant owns TMEM stage `turn` and takes the groups i = turn (mod 6) of the
// CTA's range.  The MMAs of a group are issued by one of the four warps that
// converted it (quadrant (turn + k) mod 4 for the turn's k-th group), once all four
// have: a single issuing thread sustains one M=128, N=16 MMA per ~30 cycles,
// so the six turns issue concurrently instead of queueing behind one warp.
//
// Numerics: the products a * t (t in {-1,0,+1}, or 2t for INT2) are exact in
// FP32, each group's sum is FP32, s_g * D_g is one FP32 rounding per group and
// the group sums add in FP32; one rounding to FP16 at the end.  Relative to
// sum_k |a_k w_k| this stays within a few units of 2^-24 per group added.
#pragma once

#include "gemm_tc.cuh"

namespace bonsai {

template <int MODE>
struct SmallTile {
  static constexpr int kBlockT = 16;  // tokens (MMA N)
  static constexpr int kRows = 128;   // weight rows (MMA M)
  static constexpr bool kB3 = MODE == BONSAI_TERNARY_B3;
  static constexpr int kWordsPerGroup = MODE == BONSAI_BINARY ? 4 : (kB3 ? 7 : 8);  // held per group
  static constexpr int kWGroups = kB3 ? kB3BlockGroups : 32 / kWordsPerGroup;        // groups per word stage
  static constexpr int kWRowBytes = kB3 ? kB3BlockBytes : 128;
  static constexpr int kWStageBytes = kRows * kWRowBytes;
  static constexpr int kGroupAlign = kB3 ? kB3BlockGroups : 1;
  static constexpr int kMaxGroups = 24;  // groups per CTA: the whole slice stays in shared memory
  static constexpr int kWStages = (kMaxGroups + kWGroups - 1) / kWGroups;
  static constexpr int kSliceBytes = kBlockT * 128;         // 16 rows x 64 FP16, one SW128 K slice
  static constexpr int kActGroupBytes = 2 * kSliceBytes;    // one group's activations
  static constexpr int kTurns = 6;                          // converter warps per quadrant = TMEM stages
  static constexpr int kConvWarps = 4 * kTurns;
  static constexpr int kThreads = 32 * (1 + kConvWarps);
  static constexpr int kTmemCols = 512;
  static constexpr int kAccCol0 = 64 * kTurns;  // stage t: weights at 64t, accumulator at kAccCol0 + 16t
  static constexpr int kGranules = kBlockT * kRows / 4;  // 4 consecutive rows of one token
  static constexpr int kMaxSplit = 5;                     // CTAs per cluster
  static constexpr int kRecvBytes = (kMaxSplit - 1) * kGranules * 16;  // rank 0 receives the other ranks' partials
  static constexpr int kWOff = 0;
  static constexpr int kActOff = kWOff + kWStages * kWStageBytes;
  static constexpr int kRecvOff = kActOff + kMaxGroups * kActGroupBytes;
  static constexpr int kBarOff = kRecvOff + kRecvBytes;
  static constexpr int kNumBars = kWStages + kMaxGroups + 2 * kTurns + 1;
  static constexpr int kMiscOff = kBarOff + kNumBars * 8;
  static constexpr int kSmemBytes = kMiscOff + 32 + 1024;  // + slack to align the base to 1024
  static constexpr float kOutScale = MODE == BONSAI_TERNARY_INT2 ? 0.5f : 1.0f;  // INT2 converts to 2t

  static_assert(kAccCol0 + 16 * kTurns <= kTmemCols, "TMEM budget");
  static_assert(kActOff % 1024 == 0 && kSliceBytes % 1024 == 0, "SW128 atoms are 1024-byte aligned");
  static_assert(kTurns * kBlockT * kRows * 4 <= kWStages * kWStageBytes + kMaxGroups * kActGroupBytes,
                "turn partials fit the word and activation areas");
  static_assert(kSmemBytes <= 227 * 1024, "shared memory per CTA");
  static_assert(kMaxGroups % kTurns == 0, "whole turns");
};

struct SmallArgs {
  const uint16_t* scales;
  uint16_t* out;
  int M, N, K;
  int ksplit;  // CTAs per tile along K (the cluster size along z)
  uint64_t wait_limit_ns;
};

// One group of this thread's row, without the scale, into 64 TMEM columns:
// INT2 gives the pairs (2t, 2t), binary (t, t) as +-1.0, base-3 (t, t).
template <int MODE>
__device__ __forceinline__ void convert_group_unscaled(const uint32_t* words, uint32_t taddr) {
  if (MODE == BONSAI_BINARY) {
    // One logic instruction per pair besides the shift: the sign bits under
    // the sign mask, or'ed with 1.0's exponent (both masks kept in registers).
    const uint32_t sign = 0x80008000u, one = 0x3C003C00u;
#pragma unroll
    for (int c = 0; c < 8; ++c) {
      uint32_t v[8];
#pragma unroll
      for (int p = 0; p < 8; ++p) v[p] = and_or(words[c >> 1] << (8 * (c & 1) + p), sign, one);
      tmem_store_8(taddr + c * 8, v);
    }
  } else if (MODE == BONSAI_TERNARY_B3) {
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
          v[c & 7] = b3_next_t_pair(y[p]);
          if ((c & 7) == 7) tmem_store_8(taddr + (c - 7), v);
        }
      }
  } else {
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      uint32_t v[8];
#pragma unroll
      for (int p = 0; p < 8; ++p) v[p] = (words[j] << (2 * p)) & 0xC000C000u;
      tmem_store_8(taddr + j * 8, v);
    }
  }
}

template <int MODE>
__global__ void __launch_bounds__(SmallTile<MODE>::kThreads, 1)
    lowbit_gemm_small_kernel(const __grid_constant__ CUtensorMap tmap_act, const __grid_constant__ CUtensorMap tmap_w,
                             const SmallArgs args) {
  using T = SmallTile<MODE>;
  constexpr int BT = T::kBlockT;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + T::kBarOff);
  const uint32_t w_full0 = smem_addr(bars);                                      // word stage landed
  const uint32_t a_full0 = smem_addr(bars + T::kWStages);                        // group's activations landed
  const uint32_t t_ready0 = smem_addr(bars + T::kWStages + T::kMaxGroups);       // stage converted (4 warps)
  const uint32_t t_free0 = t_ready0 + 8 * T::kTurns;                             // stage's MMAs done
  const uint32_t recv_bar = t_free0 + 8 * T::kTurns;                             // peers' partials landed
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + T::kMiscOff);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + T::kMiscOff + 4);
  // Uses of each TMEM stage whose MMAs were issued (read on the abort path).
  volatile int* issued_uses = reinterpret_cast<volatile int*>(smem + T::kMiscOff + 8);

  const int warp = __shfl_sync(0xffffffffu, static_cast<int>(threadIdx.x >> 5), 0);
  const int lane = threadIdx.x & 31;
  const int n0 = blockIdx.x * T::kRows;
  const int groups = args.K / kGroup;
  const int ks = args.ksplit;
  const int rank = static_cast<int>(blockIdx.z);  // = rank in the cluster (cluster dims 1 x 1 x ks)
  const int g_begin = split_bound<T::kGroupAlign>(rank, groups, ks);
  const int g_end = split_bound<T::kGroupAlign>(rank + 1, groups, ks);
  const int ng = g_end - g_begin;  // 1 .. kMaxGroups (checked by the host)
  const int n_wstages = (ng + T::kWGroups - 1) / T::kWGroups;
  const uint64_t limit = args.wait_limit_ns;

  // ---------------------------------------------- set-up, before the wait
  if (warp == 0) {
    if (lane == 0) {
      for (int s = 0; s < T::kWStages; ++s) mbar_init(w_full0 + 8 * s, 1);
      for (int i = 0; i < T::kMaxGroups; ++i) mbar_init(a_full0 + 8 * i, 1);
      for (int t = 0; t < T::kTurns; ++t) {
        mbar_init(t_ready0 + 8 * t, 4);  // one converter warp per lane quadrant
        mbar_init(t_free0 + 8 * t, 1);
      }
      mbar_init(recv_bar, 1);
      *abort_flag = 0;
      for (int t = 0; t < T::kTurns; ++t) issued_uses[t] = 0;
      fence_barrier_init();
      // The one phase of rank 0's recv_bar: this arrival plus the other ranks' partials.
      if (ks > 1 && rank == 0) mbar_arrive_expect_tx(recv_bar, static_cast<uint32_t>((ks - 1) * T::kGranules * 16));
      tma_prefetch_map(&tmap_w);
      tma_prefetch_map(&tmap_act);
    }
    __syncwarp();
    // The CTA's packed words: read-only here and, by the calling convention,
    // not written by the preceding kernel, so they are copied before the wait.
    for (int s = 0; s < n_wstages; ++s) {
      mbar_arrive_expect_tx_elected(w_full0 + 8 * s, T::kWStageBytes);
      tma_load_2d_elected(smem_addr(smem + T::kWOff + s * T::kWStageBytes), &tmap_w, w_full0 + 8 * s,
                          word_stage_x<MODE>(g_begin + s * T::kWGroups), n0);
    }
    // The activations into L2 meanwhile (a prefetch never returns stale data:
    // L2 is where the previous kernel's writes land); copied after the wait.
    if (lane == 0)
      for (int i = 0; i < ng; ++i) {
        tma_prefetch_l2_2d(&tmap_act, (g_begin + i) * kGroup, 0);
        tma_prefetch_l2_2d(&tmap_act, (g_begin + i) * kGroup + 64, 0);
      }
    tmem_alloc(smem_addr(tmem_slot), T::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tmem = __shfl_sync(0xffffffffu, *tmem_slot, 0);
  // Rank 0's receive barrier is armed: the other ranks wait on this phase of
  // the cluster barrier just before they send (rank 0 never waits on it).
  if (ks > 1) cluster_arrive();
  // Dependents may launch now that this CTA holds its tensor memory.
  if (threadIdx.x == 0) griddep_launch_dependents();

  int a_issued = 0;
  if (warp == 0) {
    // --------------------------------------------- activations, after the wait
    griddep_wait();
    for (int i = 0; i < ng; ++i) {
      const uint32_t full = a_full0 + 8 * i;
      const uint32_t dst = smem_addr(smem + T::kActOff + i * T::kActGroupBytes);
      const int k = (g_begin + i) * kGroup;
      mbar_arrive_expect_tx_elected(full, T::kActGroupBytes);
      tma_load_2d_elected(dst, &tmap_act, full, k, 0);
      tma_load_2d_elected(dst + T::kSliceBytes, &tmap_act, full, k + 64, 0);
      a_issued = i + 1;
    }
  } else {
    // ---------------------------------------------------------- converters
    const int quad = warp & 3;
    const int turn = (warp - 1) >> 2;  // 0 .. kTurns-1: owns TMEM stage `turn`
    const int row = quad * 32 + lane;
    const int n = n0 + row;
    const uint32_t lane_base = static_cast<uint32_t>(quad * 32) << 16;
    const uint32_t w_cols = tmem + lane_base + 64 * turn;
    const uint32_t d_cols = tmem + lane_base + T::kAccCol0 + 16 * turn;
    // This warp's groups are turn, turn + 3, ...: at most kMaxGroups / kTurns.
    constexpr int kMine = T::kMaxGroups / T::kTurns;
    float sc[kMine];
    const uint16_t* srow = args.scales + static_cast<size_t>(n < args.N ? n : 0) * groups + g_begin;
#pragma unroll
    for (int k = 0; k < kMine; ++k) {
      const int i = turn + k * T::kTurns;
      sc[k] = (n < args.N && i < ng) ? __half2float(__ushort_as_half(__ldg(srow + i))) : 0.0f;
    }
    float sums[BT];
#pragma unroll
    for (int c = 0; c < BT; ++c) sums[c] = 0.0f;
    bool ok = true;
    // Adds s * D of this stage's finished group (its use `use`) into sums.
    auto fold = [&](int use, float s) -> bool {
      if (!warp_wait_inlined(t_free0 + 8 * turn, use & 1, abort_flag, limit)) return false;
      tc_fence_after_sync();
      uint32_t v[16];
      tmem_load_16(d_cols, v);
      tmem_load_wait();
#pragma unroll
      for (int c = 0; c < BT; ++c) sums[c] = fmaf(s, __uint_as_float(v[c]), sums[c]);
      return true;
    };
#pragma unroll
    for (int k = 0; k < kMine; ++k) {
      const int i = turn + k * T::kTurns;
      if (!ok || i >= ng) break;
      if (k > 0 && !(ok = fold(k - 1, sc[k - 1]))) break;
      const int wj = i / T::kWGroups, pos = i % T::kWGroups;
      if (!(ok = warp_wait_inlined(w_full0 + 8 * wj, 0, abort_flag, limit))) break;
      const uint8_t* wrow = smem + T::kWOff + wj * T::kWStageBytes + row * T::kWRowBytes;
      uint32_t words[T::kWordsPerGroup];
      if constexpr (T::kB3) {
        b3_group_words(reinterpret_cast<const uint32_t*>(wrow), pos, words);
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
      convert_group_unscaled<MODE>(words, w_cols);
      tmem_store_wait();
      tc_fence_before_sync();
      __syncwarp();
      if (lane == 0) mbar_arrive(t_ready0 + 8 * turn);
      if (quad == ((turn + k) & 3)) {
        // This warp issues the group's MMAs once all four quadrants have
        // converted it and its activations have landed.
        if (!(ok = warp_wait_inlined(t_ready0 + 8 * turn, k & 1, abort_flag, limit) &&
                   warp_wait_inlined(a_full0 + 8 * i, 0, abort_flag, limit)))
          break;
        tc_fence_after_sync();
        constexpr uint32_t idesc = f16_instr_desc(128, BT);
        mma8_f16_tmem_a_elected<T::kSliceBytes>(
            tmem + T::kAccCol0 + 16 * turn, tmem + 64 * turn,
            sw128_kmajor_desc(smem_addr(smem + T::kActOff + i * T::kActGroupBytes)), idesc);
        mma_commit_elected(t_free0 + 8 * turn);
        if (lane == 0) issued_uses[turn] = k + 1;
      }
    }
    // The last group of this stage.
    const int mine = ng > turn ? (ng - turn + T::kTurns - 1) / T::kTurns : 0;
    if (ok && mine > 0) {
#pragma unroll
      for (int k = 1; k <= kMine; ++k)
        if (k == mine) ok = fold(k - 1, sc[k - 1]);
    }

    // ------------------------------------------------------------ epilogue
    // Every converter has seen the MMAs of its stage complete, so after this
    // barrier every MMA is done and the word and activation areas are free.
    named_barrier_sync(1, 32 * T::kConvWarps);
    griddep_wait();  // (already satisfied) before the first global write
    float* part = reinterpret_cast<float*>(smem + T::kWOff);  // [turn][token][row]
#pragma unroll
    for (int c = 0; c < BT; ++c) part[(turn * BT + c) * T::kRows + row] = sums[c];
    named_barrier_sync(1, 32 * T::kConvWarps);
    const int ct = threadIdx.x - 32;  // 0 .. 32 * kConvWarps - 1
    // This CTA's partial of granule g (rows r4..r4+3 of token m), the turns
    // added in order.
    auto own = [&](int g) -> float4 {
      const int m = g / (T::kRows / 4), r4 = (g % (T::kRows / 4)) * 4;
      float4 p = *reinterpret_cast<const float4*>(part + m * T::kRows + r4);
#pragma unroll
      for (int t = 1; t < T::kTurns; ++t) {
        const float4 q = *reinterpret_cast<const float4*>(part + (t * BT + m) * T::kRows + r4);
        p.x += q.x;
        p.y += q.y;
        p.z += q.z;
        p.w += q.w;
      }
      return p;
    };
    const bool aborted = __shfl_sync(0xffffffffu, *abort_flag, 0) != 0;  // warp-uniform
    if (ks == 1 || rank == 0) {
      // ------------------------ the tile's owner: add the peers' partials in rank order, round, store
      bool ok2 = !aborted;
      if (ks > 1 && ok2) {
        const uint64_t t0 = global_timer_ns();
        while (!mbar_try_wait_cluster(recv_bar, 0)) {
          if (*abort_flag || global_timer_ns() - t0 > limit) {
            *abort_flag = 1;
            atomicOr(&g_device_error, kErrBitTimeout);
            ok2 = false;
            break;
          }
        }
      }
      if (ok2) {
        for (int g = ct; g < T::kGranules; g += 32 * T::kConvWarps) {
          float4 p = own(g);
          for (int c = 1; c < ks; ++c) {
            const float4 v = *reinterpret_cast<const float4*>(smem + T::kRecvOff + ((c - 1) * T::kGranules + g) * 16);
            p.x += v.x;
            p.y += v.y;
            p.z += v.z;
            p.w += v.w;
          }
          const int m = g / (T::kRows / 4), r4 = (g % (T::kRows / 4)) * 4;
          if (m < args.M) {
            uint16_t* dst = args.out + static_cast<size_t>(m) * args.N + n0 + r4;
            const float vals[4] = {p.x, p.y, p.z, p.w};
#pragma unroll
            for (int j = 0; j < 4; ++j)
              if (n0 + r4 + j < args.N) dst[j] = __half_as_ushort(__float2half_rn(vals[j] * T::kOutScale));
          }
        }
      }
    } else if (!aborted) {
      // ------------------------ the other ranks: push the partial into rank 0's receive slot
      cluster_wait();  // rank 0's receive barrier is initialised
      const uint32_t dst0 = map_to_rank(smem_addr(smem + T::kRecvOff) + (rank - 1) * T::kGranules * 16, 0);
      const uint32_t bar0 = map_to_rank(recv_bar, 0);
      for (int g = ct; g < T::kGranules; g += 32 * T::kConvWarps) st_async_f32x4(dst0 + g * 16, own(g), bar0);
    }
  }

  // ------------------------------------------------------------- teardown
  if (*abort_flag) {
    if (ks > 1 && rank == 0 && threadIdx.x == 32) {
      // Partials already on their way land before this CTA's memory goes away.
      const uint64_t t0 = global_timer_ns();
      while (!mbar_try_wait_cluster(recv_bar, 0) && global_timer_ns() - t0 < limit) {
      }
    }
    if (warp == 0) {  // copies in flight land before the CTA's memory goes away
      for (int s = 0; s < n_wstages; ++s) {
        const uint64_t t0 = global_timer_ns();
        while (!mbar_try_wait(w_full0 + 8 * s, 0) && global_timer_ns() - t0 < limit) {
        }
      }
      for (int i = 0; i < a_issued; ++i) {
        const uint64_t t0 = global_timer_ns();
        while (!mbar_try_wait(a_full0 + 8 * i, 0) && global_timer_ns() - t0 < limit) {
        }
      }
      // MMAs issued but never waited for: the last use of each stage whose
      // MMAs were issued completes after all earlier ones of that stage.
      for (int t = 0; t < T::kTurns; ++t) {
        const int u = issued_uses[t];
        if (u == 0) continue;
        const uint64_t t0 = global_timer_ns();
        while (!mbar_try_wait(t_free0 + 8 * t, (u - 1) & 1) && global_timer_ns() - t0 < limit) {
        }
      }
    }
  }
  tc_fence_before_sync();
  __syncthreads();
  if (warp == 0) {
    __syncwarp();
    tc_fence_after_sync();
    tmem_dealloc(tmem, T::kTmemCols);
  }
}

}  // namespace bonsai

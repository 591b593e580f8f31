// gemm_batch.cuh - many independent layers of up to 16 tokens in one
// persistent launch: the bandwidth-bound regime without a launch per layer.
//
// Same product and numerics as lowbit_gemm_small_kernel (gemm_small.cuh):
// D^T = W * A^T with the weights as the MMA's M side, fed from tensor memory,
// tcgen05.mma kind::f16 (M=128 weight rows, N=16 tokens, K=16), the group's
// scale applied after the MMA (each TMEM stage has its own 16-column FP32
// accumulator; s_g * D_g is added into registers), one rounding to FP16.
//
// What changes is the schedule.  At 16 tokens a layer is 7-8 MB of packed
// weights streamed once, about 1.2 us at HBM speed, while a launch of its
// own costs several microseconds of start, dependency release, activation
// latency and reduction that the stream cannot hide (a kernel that allocates
// tensor memory takes a whole SM, so consecutive launches do not overlap).
// Here one CTA per SM walks a list of units, a unit being one layer's
// 128-row tile over the whole of K, and the rings run on across units and
// layers.  The CTA's word stages (four groups of each of the 128 rows: 128
// bytes INT2, 64 binary, one 112-byte block base-3) are dealt out in turn:
// stage wc goes to slot and turn wc mod T (T = 5),
// so every barrier of a slot serves the same warps, phase after phase.
//
//   warp 0     TMA of each stage's packed words into its slot, issued before
//              griddepcontrol.wait: weights are read-only and, by the
//              calling convention, not written by the kernel launched just
//              before.
//   warp 1     TMA of the stage's activations (16 x 128 FP16 per group, rows
//              past M read as zeros) into the same slot, after the wait.
//   converters four warps per turn, one per TMEM lane quadrant: each group of
//              the turn's stage is converted unscaled into the turn's TMEM
//              stage, and one of the four warps (in rotation) issues its 8
//              MMAs.  At a unit's end each converter thread leaves its row's
//              16 partial sums in shared memory.
//   epilogue   two warps add the turns' partials of a unit in turn order,
//              round once and store the 16 x 128 outputs, while the
//              converters go on with the next unit.
//
// No split of K, so no reduction between CTAs and no scratch memory; the
// host cuts the unit list into one contiguous range per CTA with nearly equal
// numbers of groups.
#pragma once

#include "gemm_small.cuh"

namespace bonsai {

constexpr int kBatchMaxLayers = 96;  // layers per launch (larger batches take several launches)
constexpr int kBatchMaxCtas = 160;

struct BatchLayer {
  const uint16_t* scales;  // FP16 [N, K/128]
  uint16_t* out;           // FP16 [M, N]
  int M, N, K;
  int unit0;  // first unit (128-row tile) of this layer in the launch's unit list
};

// Kernel parameter block (kept under the 32 KB parameter limit).
struct BatchParams {
  CUtensorMap act[kBatchMaxLayers];  // FP16 [M, K], boxes of 16 rows x 64
  CUtensorMap w[kBatchMaxLayers];    // packed words [N, row words], boxes of one word stage x 128 rows
  BatchLayer layer[kBatchMaxLayers];
  int count;  // layers
  int units;  // units of all layers
  uint64_t wait_limit_ns;
  int cta_unit0[kBatchMaxCtas + 1];  // CTA c takes units cta_unit0[c] .. cta_unit0[c+1]-1
};
static_assert(sizeof(BatchParams) <= 32000, "kernel parameter space");

template <int MODE>
struct BatchTile {
  static constexpr int kBlockT = 16;  // tokens (MMA N)
  static constexpr int kRows = 128;   // weight rows (MMA M)
  static constexpr bool kB3 = MODE == BONSAI_TERNARY_B3;
  static constexpr int kWordsPerGroup = MODE == BONSAI_BINARY ? 4 : (kB3 ? 7 : 8);  // held per group
  static constexpr int kWGroups = 4;                                                  // groups per word stage
  static constexpr int kWRowBytes = kB3 ? kB3BlockBytes : 16 * kWordsPerGroup;  // binary: 64 (64-byte swizzle)
  static constexpr int kWStageBytes = kRows * kWRowBytes;
  static constexpr int kSliceBytes = kBlockT * 128;       // 16 rows x 64 FP16, one SW128 K slice
  static constexpr int kActGroupBytes = 2 * kSliceBytes;  // one group's activations
  // A turn's slot: one word stage and the activations of its groups.
  static constexpr int kSlotBytes = kWStageBytes + kWGroups * kActGroupBytes;
  // Turns (converter warps per lane quadrant = slots = TMEM stages), as many
  // as shared memory holds: 5 (32 KB slots; 30 KB base-3, 24 KB binary).
  // Warps are what hide the hand-over latencies: binary weights in 8-group
  // stages, with room for 4 turns only, ran 43% longer per layer than INT2.
  static constexpr int kTurns = 5;
  static constexpr int kConvWarp0 = 2;
  static constexpr int kConvWarps = 4 * kTurns;
  static constexpr int kEpiWarp0 = kConvWarp0 + kConvWarps;
  static constexpr int kEpiWarps = 2;  // one thread per two weight rows (registers: 768 threads, 80 each)
  static constexpr int kThreads = 32 * (kEpiWarp0 + kEpiWarps);
  static constexpr int kTmemCols = 512;
  static constexpr int kAccCol0 = 64 * kTurns;  // stage t: weights at 64t, accumulator at kAccCol0 + 16t
  static constexpr int kPartBytes = kTurns * kBlockT * kRows * 4;  // [turn][token][row] FP32
  static constexpr int kSlotOff = 0;
  static constexpr int kPartOff = kSlotOff + kTurns * kSlotBytes;
  static constexpr int kBarOff = kPartOff + kPartBytes;
  static constexpr int kNumBars = 6 * kTurns + 2;
  static constexpr int kMiscOff = kBarOff + kNumBars * 8;
  static constexpr int kSmemBytes = kMiscOff + 64 + 1024;  // + slack to align the base to 1024
  static constexpr float kOutScale = MODE == BONSAI_TERNARY_INT2 ? 0.5f : 1.0f;  // INT2 converts to 2t

  static_assert(kAccCol0 + 16 * kTurns <= kTmemCols, "TMEM budget");
  static_assert(kSlotBytes % 1024 == 0 && kWStageBytes % 1024 == 0, "SW128 stages and atoms are 1024-byte aligned");
  static_assert(kSmemBytes <= 227 * 1024, "shared memory per CTA");
  static_assert(kThreads <= 1024, "threads per CTA");
  static_assert(8 + 4 * kTurns + 8 <= 64, "misc words");
};

template <int MODE>
__global__ void __launch_bounds__(BatchTile<MODE>::kThreads, 1)
    lowbit_gemm_batch_kernel(const __grid_constant__ BatchParams params) {
  using T = BatchTile<MODE>;
  constexpr int TT = T::kTurns, BT = T::kBlockT, WG = T::kWGroups;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + T::kBarOff);
  // Per turn (slot) t, each barrier at base + 8t:
  const uint32_t w_full0 = smem_addr(bars);     // the slot's word stage landed
  const uint32_t w_empty0 = w_full0 + 8 * TT;   // its four converter warps hold the words
  const uint32_t a_full0 = w_empty0 + 8 * TT;   // the stage's activations landed
  const uint32_t a_empty0 = a_full0 + 8 * TT;   // the stage's MMAs are done with them
  const uint32_t t_ready0 = a_empty0 + 8 * TT;  // TMEM stage converted (4 warps)
  const uint32_t t_free0 = t_ready0 + 8 * TT;   // TMEM stage's MMAs done
  const uint32_t part_full = t_free0 + 8 * TT;  // every converter left its unit partial
  const uint32_t part_free = part_full + 8;     // the epilogue has read them
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + T::kMiscOff);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + T::kMiscOff + 4);
  // Uses of each TMEM stage whose MMAs were issued, then the latest word and
  // activation stages issued (read on the abort path).
  volatile int* issued_uses = reinterpret_cast<volatile int*>(smem + T::kMiscOff + 8);
  volatile int* last_w = reinterpret_cast<volatile int*>(smem + T::kMiscOff + 8 + 4 * TT);
  volatile int* last_a = last_w + 1;

  const int warp = __shfl_sync(0xffffffffu, static_cast<int>(threadIdx.x >> 5), 0);
  const int lane = threadIdx.x & 31;
  const int u_begin = params.cta_unit0[blockIdx.x];
  const int u_end = params.cta_unit0[blockIdx.x + 1];
  const uint64_t limit = params.wait_limit_ns;
  // Layer of unit u: layers' units are consecutive, so a cursor only moves on.
  auto advance = [&](int u, int p) {
    while (p + 1 < params.count && params.layer[p + 1].unit0 <= u) ++p;
    return p;
  };
  auto slot = [&](int t) { return smem + T::kSlotOff + t * T::kSlotBytes; };

  // -------------------------------------------------------------- set-up
  if (warp == 0) {
    if (lane == 0) {
      for (int t = 0; t < TT; ++t) {
        mbar_init(w_full0 + 8 * t, 1);
        mbar_init(w_empty0 + 8 * t, 4);
        mbar_init(a_full0 + 8 * t, 1);
        mbar_init(a_empty0 + 8 * t, 1);
        mbar_init(t_ready0 + 8 * t, 4);
        mbar_init(t_free0 + 8 * t, 1);
        issued_uses[t] = 0;
      }
      mbar_init(part_full, 32 * T::kConvWarps);
      mbar_init(part_free, 32 * T::kEpiWarps);
      *abort_flag = 0;
      *last_w = -1;
      *last_a = -1;
      fence_barrier_init();
    }
    __syncwarp();
    tmem_alloc(smem_addr(tmem_slot), T::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tmem = __shfl_sync(0xffffffffu, *tmem_slot, 0);
  // Dependents may launch now that this CTA holds its tensor memory.
  if (threadIdx.x == 0) griddep_launch_dependents();

  // Every ring runs over the CTA's running word-stage count wc: stage wc goes
  // to slot wc mod TT and is converted by turn wc mod TT, so each barrier of
  // a slot is used by the same warps, every phase in order, and its parity
  // waits are unambiguous.
  if (warp == 0) {
    // ------------------------------------- packed-word producer (no wait)
    int p = 0, wc = 0;
    bool ok = true;
    for (int u = u_begin; ok && u < u_end; ++u) {
      p = advance(u, p);
      const int n0 = (u - params.layer[p].unit0) * T::kRows;
      const int nws = (params.layer[p].K / kGroup + WG - 1) / WG;
      for (int j = 0; j < nws; ++j, ++wc) {
        const int t = wc % TT;
        if (!(ok = warp_wait_inlined(w_empty0 + 8 * t, ((wc / TT) & 1) ^ 1, abort_flag, limit))) break;
        mbar_arrive_expect_tx_elected(w_full0 + 8 * t, T::kWStageBytes);
        tma_load_2d_elected(smem_addr(slot(t)), &params.w[p], w_full0 + 8 * t, word_stage_x<MODE>(j * WG), n0);
        if (lane == 0) *last_w = wc;
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------- activation producer
    if (lane == 0 && u_begin < u_end) {  // the first unit's activations into L2 meanwhile
      const int p0 = advance(u_begin, 0);
      const int g0 = params.layer[p0].K / kGroup;
      for (int i = 0; i < g0 && i < 16; ++i) {
        tma_prefetch_l2_2d(&params.act[p0], i * kGroup, 0);
        tma_prefetch_l2_2d(&params.act[p0], i * kGroup + 64, 0);
      }
    }
    griddep_wait();
    int p = 0, wc = 0;
    bool ok = true;
    for (int u = u_begin; ok && u < u_end; ++u) {
      p = advance(u, p);
      const int groups = params.layer[p].K / kGroup;
      const int nws = (groups + WG - 1) / WG;
      for (int j = 0; j < nws; ++j, ++wc) {
        const int t = wc % TT;
        const int gs = groups - j * WG < WG ? groups - j * WG : WG;  // groups in this stage
        if (!(ok = warp_wait_inlined(a_empty0 + 8 * t, ((wc / TT) & 1) ^ 1, abort_flag, limit))) break;
        const uint32_t full = a_full0 + 8 * t;
        const uint32_t dst = smem_addr(slot(t) + T::kWStageBytes);
        mbar_arrive_expect_tx_elected(full, static_cast<uint32_t>(gs * T::kActGroupBytes));
        for (int g = 0; g < gs; ++g) {
          const int k = (j * WG + g) * kGroup;
          tma_load_2d_elected(dst + g * T::kActGroupBytes, &params.act[p], full, k, 0);
          tma_load_2d_elected(dst + g * T::kActGroupBytes + T::kSliceBytes, &params.act[p], full, k + 64, 0);
        }
        if (lane == 0) *last_a = wc;
      }
    }
  } else if (warp < T::kEpiWarp0) {
    // ---------------------------------------------------------- converters
    const int quad = warp & 3;                     // TMEM lanes 32*quad .. +31
    const int turn = (warp - T::kConvWarp0) >> 2;  // owns slot and TMEM stage `turn`
    const int row = quad * 32 + lane;
    const uint32_t lane_base = static_cast<uint32_t>(quad * 32) << 16;
    const uint32_t w_cols = tmem + lane_base + 64 * turn;
    const uint32_t d_cols = tmem + lane_base + T::kAccCol0 + 16 * turn;
    const uint8_t* wslot = slot(turn) + row * T::kWRowBytes;
    const uint32_t act_slot = smem_addr(slot(turn) + T::kWStageBytes);
    float* part = reinterpret_cast<float*>(smem + T::kPartOff);
    float sums[BT];
    // Adds s * D of this stage's use k (its MMAs' completion) into sums.
    auto fold = [&](int k, float s) -> bool {
      if (!warp_wait_inlined(t_free0 + 8 * turn, k & 1, abort_flag, limit)) return false;
      tc_fence_after_sync();
      uint32_t v[16];
      tmem_load_16(d_cols, v);
      tmem_load_wait();
#pragma unroll
      for (int m = 0; m < BT; ++m) sums[m] = fmaf(s, __uint_as_float(v[m]), sums[m]);
      return true;
    };
    // wc0: running word-stage count at the unit's start; ks: stages this turn
    // has taken (its k-th stage is phase k of its slot's barriers).
    int p = 0, wc0 = 0, use = 0, ks = 0, ul = 0;
    float s_pend = 0.0f;
    bool ok = true;
    // The stage's scales of this row, FP16 pairs: groups 2i, 2i+1 in sv[i].
    constexpr int kSv = WG / 2;
    static_assert(kSv == 2, "a stage's scales are one 8-byte load");
    auto scale_of = [&](const uint32_t* sv, int pos) -> float {
      uint32_t h = sv[0];
#pragma unroll
      for (int i = 1; i < kSv; ++i)
        if ((pos >> 1) == i) h = sv[i];
      return __half2float(__ushort_as_half(static_cast<uint16_t>((pos & 1) ? h >> 16 : h)));
    };
    for (int u = u_begin; ok && u < u_end; ++u, ++ul) {
      p = advance(u, p);
      const int n = (u - params.layer[p].unit0) * T::kRows + row;
      const int groups = params.layer[p].K / kGroup;
      const int nws = (groups + WG - 1) / WG;
      const bool row_in = n < params.layer[p].N;
      const uint16_t* srow = params.layer[p].scales + static_cast<size_t>(row_in ? n : 0) * groups;
      // Whole stages of scales are one aligned vector load when every row
      // starts on a stage boundary (the scale array is 16-byte aligned).
      const bool vec_scales = groups % WG == 0;
#pragma unroll
      for (int m = 0; m < BT; ++m) sums[m] = 0.0f;
      bool pend = false;
      for (int j = ((turn - wc0) % TT + TT) % TT; ok && j < nws; j += TT, ++ks) {
        const uint32_t ph = ks & 1;
        const int gs = groups - j * WG < WG ? groups - j * WG : WG;
        uint32_t sv[kSv];
#pragma unroll
        for (int i = 0; i < kSv; ++i) sv[i] = 0u;
        if (row_in) {
          if (vec_scales) {
            const uint2 q = __ldg(reinterpret_cast<const uint2*>(srow + j * WG));
            sv[0] = q.x;
            sv[1] = q.y;
          } else {
#pragma unroll
            for (int g = 0; g < WG; ++g)
              if (g < gs) sv[g >> 1] |= static_cast<uint32_t>(__ldg(srow + j * WG + g)) << (16 * (g & 1));
          }
        }
        if (!(ok = warp_wait_inlined(w_full0 + 8 * turn, ph, abort_flag, limit))) break;
        for (int pos = 0; pos < gs; ++pos) {
          const float s_cur = scale_of(sv, pos);
          if (pend && !(ok = fold(use - 1, s_pend))) break;
          uint32_t words[T::kWordsPerGroup];
          if constexpr (T::kB3) {
            b3_group_words(reinterpret_cast<const uint32_t*>(wslot), pos, words);
          } else if (MODE == BONSAI_BINARY) {  // 64-byte rows, 64-byte swizzle
            const uint4 q = *reinterpret_cast<const uint4*>(wslot + 16 * (pos ^ ((row >> 1) & 3)));
            words[0] = q.x;
            words[1] = q.y;
            words[2] = q.z;
            words[3] = q.w;
          } else {
            const uint4 q0 = *reinterpret_cast<const uint4*>(wslot + 16 * ((2 * pos) ^ (row & 7)));
            const uint4 q1 = *reinterpret_cast<const uint4*>(wslot + 16 * ((2 * pos + 1) ^ (row & 7)));
            words[0] = q0.x;
            words[1] = q0.y;
            words[2] = q0.z;
            words[3] = q0.w;
            words[4] = q1.x;
            words[5] = q1.y;
            words[6] = q1.z;
            words[7] = q1.w;
          }
          const bool last = pos == gs - 1;
          if (last) {  // the stage's words are in registers: release the slot's word half
            __syncwarp();
            if (lane == 0) mbar_arrive(w_empty0 + 8 * turn);
          }
          convert_group_unscaled<MODE>(words, w_cols);
          tmem_store_wait();
          tc_fence_before_sync();
          __syncwarp();
          if (lane == 0) mbar_arrive(t_ready0 + 8 * turn);
          if (quad == ((turn + use) & 3)) {
            // This warp issues the group's MMAs once all four quadrants have
            // converted it and the stage's activations have landed.
            if (!(ok = warp_wait_inlined(t_ready0 + 8 * turn, use & 1, abort_flag, limit) &&
                       warp_wait_inlined(a_full0 + 8 * turn, ph, abort_flag, limit)))
              break;
            tc_fence_after_sync();
            constexpr uint32_t idesc = f16_instr_desc(128, BT);
            mma8_f16_tmem_a_elected<T::kSliceBytes>(tmem + T::kAccCol0 + 16 * turn, tmem + 64 * turn,
                                                    sw128_kmajor_desc(act_slot + pos * T::kActGroupBytes), idesc);
            // The stage's earlier groups' MMAs completed before this group was
            // converted (folds), so this commit releases its activations.
            // The awaited barrier last: its arrival follows the release.
            if (last) mma_commit_elected(a_empty0 + 8 * turn);
            mma_commit_elected(t_free0 + 8 * turn);
            if (lane == 0) issued_uses[turn] = use + 1;
          }
          s_pend = s_cur;
          pend = true;
          ++use;
        }
      }
      if (ok && pend) ok = fold(use - 1, s_pend);
      if (!ok) break;
      // The unit's partial: the previous unit's must have been read.
      if (ul > 0 && !(ok = warp_wait_inlined(part_free, (ul - 1) & 1, abort_flag, limit))) break;
#pragma unroll
      for (int m = 0; m < BT; ++m) part[(turn * BT + m) * T::kRows + row] = sums[m];
      mbar_arrive(part_full);
      wc0 += nws;
    }
  } else {
    // ------------------------------------------------------------ epilogue
    constexpr int kRowsPerThread = T::kRows / (32 * T::kEpiWarps);
    const int row0 = (warp - T::kEpiWarp0) * 32 + lane;
    const float* part = reinterpret_cast<const float*>(smem + T::kPartOff);
    griddep_wait();  // before the first global write
    int p = 0, ul = 0;
    for (int u = u_begin; u < u_end; ++u, ++ul) {
      p = advance(u, p);
      if (!warp_wait_inlined(part_full, ul & 1, abort_flag, limit)) break;
      uint32_t h[kRowsPerThread][BT / 2];  // FP16 pairs (token 2j, 2j+1) of each row
#pragma unroll
      for (int r = 0; r < kRowsPerThread; ++r) {
        const int row = row0 + r * 32 * T::kEpiWarps;
#pragma unroll
        for (int m = 0; m < BT; m += 2) {
          float a0 = part[m * T::kRows + row], a1 = part[(m + 1) * T::kRows + row];
#pragma unroll
          for (int t = 1; t < TT; ++t) {
            a0 += part[(t * BT + m) * T::kRows + row];
            a1 += part[(t * BT + m + 1) * T::kRows + row];
          }
          h[r][m / 2] = static_cast<uint32_t>(__half_as_ushort(__float2half_rn(a0 * T::kOutScale))) |
                        (static_cast<uint32_t>(__half_as_ushort(__float2half_rn(a1 * T::kOutScale))) << 16);
        }
      }
      mbar_arrive(part_free);
      const BatchLayer& L = params.layer[p];
#pragma unroll
      for (int r = 0; r < kRowsPerThread; ++r) {
        const int n = (u - L.unit0) * T::kRows + row0 + r * 32 * T::kEpiWarps;
        if (n < L.N) {
          uint16_t* dst = L.out + n;
#pragma unroll
          for (int m = 0; m < BT; ++m)
            if (m < L.M) dst[static_cast<size_t>(m) * L.N] = static_cast<uint16_t>(h[r][m / 2] >> (16 * (m & 1)));
        }
      }
    }
  }

  // ------------------------------------------------------------- teardown
  tc_fence_before_sync();
  __syncthreads();
  if (*abort_flag && lane == 0) {
    // Copies and MMAs still in flight finish before the CTA's shared and
    // tensor memory go away (each wait bounded).
    if (warp == 0 || warp == 1) {
      const int last = warp == 0 ? *last_w : *last_a;
      const uint32_t full0 = warp == 0 ? w_full0 : a_full0;
      for (int wc = last; wc >= 0 && wc > last - TT; --wc) {
        const uint64_t t0 = global_timer_ns();
        while (!mbar_try_wait(full0 + 8 * (wc % TT), (wc / TT) & 1) && global_timer_ns() - t0 < limit) {
        }
      }
    } else if (warp == T::kConvWarp0) {
      // A stage has at most one use whose MMAs were issued and not waited for.
      for (int t = 0; t < TT; ++t) {
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

// gemm_tc.cuh - fused dequantise + GEMM on the 5th-generation tensor cores.
//
// out[m,n] = sum_k A[m,k] * w[n,k],  w[n,k] = s[n,k/128] * t[n,k].
//
// Tile = 128 weight rows x BLOCK_T tokens, computed as D^T = W * A^T so that
// the weights are the MMA's M side and can be fed from tensor memory:
//
//   warp 0      TMA producer: per 128-wide K group, the activation tile
//               (BLOCK_T x 128 FP16, two 128-byte-swizzled K slices) and the
//               packed words of the 128 weight rows land in a shared-memory
//               stage; one mbarrier counts the bytes.
//   warp 1      allocates tensor memory, then one thread issues
//               tcgen05.mma.kind::f16 (M=128, N=BLOCK_T, K=16) x 8 per group:
//               A = converted weights in TMEM, B = activations in SMEM,
//               D = FP32 accumulator in TMEM; tcgen05.commit frees the stage.
//   warps 2-5   converters: each thread owns one weight row (its TMEM lane),
//               turns the group's packed words into exact FP16 products
//               (binary: sign bit over s; ternary: the shifted 2-bit field is
//               2t, times s) and stores them into the stage's TMEM columns
//               with tcgen05.st.  After the last group they read the
//               accumulator back (tcgen05.ld), scale by 1 (binary) or 1/2
//               (ternary, exact), round once to FP16 and store out[m, n].
//
// Weights are multiplied exactly: |t| <= 1 and s is FP16, so s*t (and 2*s*t
// for |s| < 32768) is an FP16 value.  The sum runs in FP32 on the tensor
// cores and is rounded to FP16 once.
#pragma once

#include "pack_dequant.cuh"
#include "ptx.cuh"

namespace bonsai {

__host__ __device__ constexpr int pow2_at_least(int x) {
  int p = 32;
  while (p < x) p *= 2;
  return p;
}

template <int MODE, int BLOCK_T, int STAGES>
struct GemmTile {
  static constexpr int kRows = 128;                                 // weight rows per tile (MMA M)
  static constexpr int kWordsPerGroup = MODE == BONSAI_BINARY ? 4 : 8;
  static constexpr int kSliceBytes = BLOCK_T * 128;                 // BLOCK_T rows x 64 FP16
  static constexpr int kActStageBytes = 2 * kSliceBytes;            // 128 K per stage
  static constexpr int kWStageBytes = kRows * kWordsPerGroup * 4;
  static constexpr int kStageTx = kActStageBytes + kWStageBytes;
  static constexpr int kACol0 = BLOCK_T < 64 ? 64 : BLOCK_T;        // TMEM columns: [0,BLOCK_T) = D
  static constexpr int kTmemCols = pow2_at_least(kACol0 + STAGES * 64);
  static constexpr int kActOff = 0;
  static constexpr int kWOff = STAGES * kActStageBytes;
  static constexpr int kBarOff = kWOff + STAGES * kWStageBytes;
  static constexpr int kNumBars = 3 * STAGES + 1;
  static constexpr int kMiscOff = kBarOff + kNumBars * 8;
  static constexpr int kSmemNeeded = kMiscOff + 16 + 1024;          // + slack to align the base to 1024
  // Shared memory also caps how many CTAs share an SM, so that their tensor
  // memory allocations fit side by side (512 columns per SM, 228 KB of
  // shared memory per SM): 512 columns -> 1 CTA, 256 -> 2.
  static constexpr int kSmemFloor = kTmemCols == 512 ? 116 * 1024 : (kTmemCols == 256 ? 78 * 1024 : 0);
  static constexpr int kSmemBytes = kSmemNeeded > kSmemFloor ? kSmemNeeded : kSmemFloor;
  static constexpr float kOutScale = MODE == BONSAI_BINARY ? 1.0f : 0.5f;
  static_assert(BLOCK_T % 16 == 0 && BLOCK_T >= 16 && BLOCK_T <= 256, "MMA N for M=128");
  static_assert(kSliceBytes % 1024 == 0, "swizzle atoms need 1024-byte alignment");
  static_assert(kTmemCols <= 512, "tensor memory has 512 columns");
  static_assert(kSmemBytes <= 227 * 1024, "shared memory per CTA");
};

// Converts one group (128 weights) of this thread's row into FP16 products
// and writes them to 64 TMEM columns starting at `taddr`.
template <int MODE>
__device__ __forceinline__ void convert_group_to_tmem(const uint32_t* words, uint32_t s2, uint32_t taddr) {
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

// Waits that the whole warp agrees on: every lane waits, and the warp goes on
// only if all lanes saw the phase complete.
__device__ __forceinline__ bool warp_wait(uint32_t bar, uint32_t parity, volatile int* abort_flag,
                                          uint64_t limit_ns) {
  const bool ok = wait_phase(bar, parity, abort_flag, limit_ns);
  return __all_sync(0xffffffffu, ok);
}

template <int MODE, int BLOCK_T, int STAGES>
__global__ void __launch_bounds__(192, 1)
    lowbit_gemm_kernel(const __grid_constant__ CUtensorMap tmap_act, const __grid_constant__ CUtensorMap tmap_w,
                       const uint16_t* __restrict__ scales, uint16_t* __restrict__ out, int M, int N, int K,
                       uint64_t wait_limit_ns) {
  using T = GemmTile<MODE, BLOCK_T, STAGES>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + T::kBarOff);
  const uint32_t full0 = smem_addr(bars);                 // full[s]:  TMA bytes of stage s landed
  const uint32_t ready0 = smem_addr(bars + STAGES);       // ready[s]: converted weights in TMEM (4 warps)
  const uint32_t empty0 = smem_addr(bars + 2 * STAGES);   // empty[s]: MMAs reading stage s finished
  const uint32_t dfull = smem_addr(bars + 3 * STAGES);    // accumulator final
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + T::kMiscOff);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + T::kMiscOff + 4);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int n0 = blockIdx.x * T::kRows;
  const int m0 = blockIdx.y * BLOCK_T;
  const int groups = K / kGroup;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(full0 + 8 * s, 1);
      mbar_init(ready0 + 8 * s, 4);
      mbar_init(empty0 + 8 * s, 1);
    }
    mbar_init(dfull, 1);
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
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    // ---------------------------------------------------------- producer
    if (elect_one()) {
      int issued = 0;
      for (int g = 0; g < groups; ++g) {
        const int s = g % STAGES;
        const uint32_t ph = (g / STAGES) & 1;
        if (!wait_phase(empty0 + 8 * s, ph ^ 1, abort_flag, wait_limit_ns)) break;
        const uint32_t full = full0 + 8 * s;
        mbar_arrive_expect_tx(full, T::kStageTx);
        const uint32_t act = smem_addr(smem + T::kActOff + s * T::kActStageBytes);
        tma_load_2d(act, &tmap_act, full, g * kGroup, m0);
        tma_load_2d(act + T::kSliceBytes, &tmap_act, full, g * kGroup + 64, m0);
        tma_load_2d(smem_addr(smem + T::kWOff + s * T::kWStageBytes), &tmap_w, full, g * T::kWordsPerGroup, n0);
        issued = g + 1;
      }
      if (*abort_flag) {
        // Let copies already in flight land before the CTA's memory goes away.
        for (int g = issued - STAGES < 0 ? 0 : issued - STAGES; g < issued; ++g) {
          const uint64_t t0 = global_timer_ns();
          while (!mbar_try_wait(full0 + 8 * (g % STAGES), (g / STAGES) & 1) && global_timer_ns() - t0 < wait_limit_ns) {
          }
        }
      }
    }
  } else if (warp == 1) {
    // --------------------------------------------------------- MMA issuer
    if (elect_one()) {
      constexpr uint32_t idesc = f16_instr_desc(128, BLOCK_T);
      for (int g = 0; g < groups; ++g) {
        const int s = g % STAGES;
        const uint32_t ph = (g / STAGES) & 1;
        if (!wait_phase(full0 + 8 * s, ph, abort_flag, wait_limit_ns)) break;
        if (!wait_phase(ready0 + 8 * s, ph, abort_flag, wait_limit_ns)) break;
        tc_fence_after_sync();
        const uint32_t act = smem_addr(smem + T::kActOff + s * T::kActStageBytes);
        const uint32_t a_cols = tmem + T::kACol0 + s * 64;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint64_t bdesc = sw128_kmajor_desc(act + (kk >> 2) * T::kSliceBytes + (kk & 3) * 32);
          mma_f16_tmem_a(tmem, a_cols + kk * 8, bdesc, idesc, (g | kk) != 0 ? 1u : 0u);
        }
        mma_commit(empty0 + 8 * s);
      }
      mma_commit(dfull);  // also on abort: lets this thread see its MMAs drain
      if (*abort_flag) {
        const uint64_t t0 = global_timer_ns();
        while (!mbar_try_wait(dfull, 0) && global_timer_ns() - t0 < wait_limit_ns) {
        }
      }
    }
  } else {
    // ------------------------------------------------ converters + epilogue
    const int quad = warp & 3;  // a warp may only touch TMEM lanes 32*(warp%4) .. +31
    const int row = quad * 32 + lane;
    const int n = n0 + row;
    const uint32_t lane_base = static_cast<uint32_t>(quad * 32) << 16;
    const uint16_t* srow = scales + static_cast<size_t>(n) * groups;
    uint32_t s_next = n < N ? __ldg(srow) : 0u;
    bool ok = true;
    for (int g = 0; g < groups; ++g) {
      const int s = g % STAGES;
      const uint32_t ph = (g / STAGES) & 1;
      const uint32_t sc = s_next;
      if (g + 1 < groups && n < N) s_next = __ldg(srow + g + 1);
      ok = warp_wait(full0 + 8 * s, ph, abort_flag, wait_limit_ns) &&
           warp_wait(empty0 + 8 * s, ph ^ 1, abort_flag, wait_limit_ns);
      if (!ok) break;
      tc_fence_after_sync();  // the MMAs that read this stage's columns are done
      const uint4* src = reinterpret_cast<const uint4*>(smem + T::kWOff + s * T::kWStageBytes) +
                         row * (T::kWordsPerGroup / 4);
      uint32_t words[T::kWordsPerGroup];
#pragma unroll
      for (int i = 0; i < T::kWordsPerGroup / 4; ++i) {
        const uint4 q = src[i];
        words[4 * i] = q.x;
        words[4 * i + 1] = q.y;
        words[4 * i + 2] = q.z;
        words[4 * i + 3] = q.w;
      }
      convert_group_to_tmem<MODE>(words, sc | (sc << 16), tmem + lane_base + T::kACol0 + s * 64);
      tmem_store_wait();
      tc_fence_before_sync();
      __syncwarp();
      if (lane == 0) mbar_arrive(ready0 + 8 * s);
    }
    if (ok && warp_wait(dfull, 0, abort_flag, wait_limit_ns)) {
      tc_fence_after_sync();
#pragma unroll 1
      for (int c = 0; c < BLOCK_T; c += 16) {
        uint32_t v[16];
        tmem_load_16(tmem + lane_base + c, v);
        tmem_load_wait();
        if (n < N) {
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            const int m = m0 + c + j;
            if (m < M) {
              const __half h = __float2half_rn(__uint_as_float(v[j]) * T::kOutScale);
              out[static_cast<size_t>(m) * N + n] = __half_as_ushort(h);
            }
          }
        }
      }
    }
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

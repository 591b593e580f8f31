// ptx.cuh - thin inline-PTX wrappers for sm_100a: mbarriers, TMA tile loads,
// tensor-memory allocation, tcgen05 MMA / load / store, and bounded waits.
//
// Every mbarrier wait in the library goes through wait_phase(), which gives
// up after a time limit, records BONSAI_ERR_TIMEOUT in the device error word
// and raises the CTA's abort flag so the other warps stop too.  The one
// blocking instruction without a limit is tcgen05.alloc, which waits for free
// tensor-memory columns.  It cannot wait forever: every kernel allocates
// before it lets dependent grids launch (griddepcontrol.launch_dependents)
// and frees its columns before it exits, and a CTA holding columns waits only
// for grids launched before it, whose CTAs already hold theirs.
#pragma once

#include <cuda.h>
#include <cuda_fp16.h>
#include <stdint.h>

namespace bonsai {

// Device-wide error word, read and cleared by bonsai_get_device_error().
__device__ unsigned int g_device_error = 0;
constexpr unsigned kErrBitTimeout = 1u << 7;  // a bounded wait ran out

__device__ __forceinline__ uint32_t smem_addr(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint64_t global_timer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ uint32_t lane_id() { return threadIdx.x & 31u; }

__device__ __forceinline__ bool elect_one() {
  uint32_t pred = 0;
  asm volatile(
      "{\n"
      "  .reg .pred p;\n"
      "  elect.sync _|p, 0xffffffff;\n"
      "  selp.u32 %0, 1, 0, p;\n"
      "}\n"
      : "=r"(pred));
  return pred != 0;
}

// Warp-uniform issue.  The *_elected wrappers below are executed by a whole
// converged warp; one lane, chosen by elect.sync inside the instruction
// sequence (always the same lane for a full warp), issues the operation.  A
// loop that stays warp-uniform keeps its descriptors and addresses in the
// warp's uniform registers; the same loop run by one elected thread pays for
// moving them on every tcgen05.mma (about three times the issue cost).

// ------------------------------------------------------------- mbarrier --
__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_barrier_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.release.cta.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

// Counts `count` arrivals at once.
__device__ __forceinline__ void mbar_arrive_count(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.arrive.release.cta.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.release.cta.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
               : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx_elected(uint32_t bar, uint32_t bytes) {
  asm volatile(
      "{\n"
      "  .reg .pred e;\n"
      "  elect.sync _|e, 0xffffffff;\n"
      "  @e mbarrier.arrive.expect_tx.release.cta.shared::cta.b64 _, [%0], %1;\n"
      "}\n" ::"r"(bar),
      "r"(bytes)
      : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t done;
  asm volatile(
      "{\n"
      "  .reg .pred p;\n"
      "  mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n"
      "  selp.u32 %0, 1, 0, p;\n"
      "}\n"
      : "=r"(done)
      : "r"(bar), "r"(parity)
      : "memory");
  return done != 0;
}

// Non-blocking test: has the phase with the given parity completed?
__device__ __forceinline__ bool mbar_test_wait(uint32_t bar, uint32_t parity) {
  uint32_t done;
  asm volatile(
      "{\n"
      "  .reg .pred p;\n"
      "  mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n"
      "  selp.u32 %0, 1, 0, p;\n"
      "}\n"
      : "=r"(done)
      : "r"(bar), "r"(parity)
      : "memory");
  return done != 0;
}

// The blocking loop of a bounded wait.
__device__ __forceinline__ bool wait_phase_loop(uint32_t bar, uint32_t parity, volatile int* abort_flag,
                                                uint64_t limit_ns) {
  const uint64_t t0 = global_timer_ns();
  for (uint32_t i = 1;; ++i) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((i & 15u) == 0) {
      if (*abort_flag) return false;
      if (global_timer_ns() - t0 > limit_ns) {
        *abort_flag = 1;
        atomicOr(&g_device_error, kErrBitTimeout);
        return false;
      }
    }
  }
}

// The blocking part of wait_phase, kept out of line.
__device__ __noinline__ bool wait_phase_slow(uint32_t bar, uint32_t parity, volatile int* abort_flag,
                                             uint64_t limit_ns) {
  return wait_phase_loop(bar, parity, abort_flag, limit_ns);
}

// Waits until the phase with the given parity of barrier `bar` completes.
// Returns false (without waiting further) when the CTA's abort flag is up or
// when `limit_ns` has passed; in the latter case it records the timeout.
// A phase that has already completed costs one non-blocking test.
__device__ __forceinline__ bool wait_phase(uint32_t bar, uint32_t parity, volatile int* abort_flag,
                                           uint64_t limit_ns) {
  if (mbar_test_wait(bar, parity)) return true;
  return wait_phase_slow(bar, parity, abort_flag, limit_ns);
}

// The same wait with its loop inlined, for kernels whose waits mostly block
// (the batched small-M kernel: a call per wait measured 8% of its time).
__device__ __forceinline__ bool wait_phase_inlined(uint32_t bar, uint32_t parity, volatile int* abort_flag,
                                                   uint64_t limit_ns) {
  if (mbar_test_wait(bar, parity)) return true;
  return wait_phase_loop(bar, parity, abort_flag, limit_ns);
}

// ------------------------------------------- programmatic dependent launch --
// Blocks until every grid this one depends on has completed and its memory
// writes are visible (a no-op when the launch has no such dependency).
__device__ __forceinline__ void griddep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

// Lets the next grid in the stream be scheduled once every CTA of this grid
// has issued this (or exited).
__device__ __forceinline__ void griddep_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// ------------------------------------------------------------------ TMA --
__device__ __forceinline__ void tma_prefetch_map(const CUtensorMap* map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// Asks the TMA unit to bring a 2-D box into L2 (no shared-memory write, no
// completion to wait for).  L2 is the device's point of coherence, so a
// prefetch can never make a later load see stale data.
__device__ __forceinline__ void tma_prefetch_l2_2d(const CUtensorMap* map, int32_t x, int32_t y) {
  asm volatile("cp.async.bulk.prefetch.tensor.2d.L2.global.tile [%0, {%1, %2}];" ::"l"(
                   reinterpret_cast<uint64_t>(map)),
               "r"(x), "r"(y)
               : "memory");
}

// 2-D tiled bulk copy global -> shared, completing `bar` with the bytes.
// x is the innermost (contiguous) coordinate in elements, y the row.
__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* map, uint32_t bar, int32_t x,
                                            int32_t y) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4}], [%2];" ::"r"(
          dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(x), "r"(y)
      : "memory");
}

__device__ __forceinline__ void tma_load_2d_elected(uint32_t dst, const CUtensorMap* map, uint32_t bar, int32_t x,
                                                    int32_t y) {
  asm volatile(
      "{\n"
      "  .reg .pred e;\n"
      "  elect.sync _|e, 0xffffffff;\n"
      "  @e cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4}], [%2];\n"
      "}\n" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(x), "r"(y)
      : "memory");
}

// 2-D tiled bulk copy shared -> global (out-of-range rows and columns of the
// box are not written), tracked by the issuing thread's bulk group.
__device__ __forceinline__ void tma_store_2d(const CUtensorMap* map, uint32_t src, int32_t x, int32_t y) {
  asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%2, %3}], [%1];" ::"l"(
                   reinterpret_cast<uint64_t>(map)),
               "r"(src), "r"(x), "r"(y)
               : "memory");
}

__device__ __forceinline__ void bulk_commit_group() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }

// Waits until every committed bulk store has finished reading shared memory.
__device__ __forceinline__ void bulk_wait_group_read0() {
  asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
}

// Makes this thread's generic-proxy shared-memory writes visible to the
// async proxy (TMA) before a later bulk copy reads them.
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// Barrier among `count` threads (a multiple of 32) on hardware barrier `id`.
__device__ __forceinline__ void named_barrier_sync(uint32_t id, uint32_t count) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(count) : "memory");
}

// ------------------------------------------------------------- clusters --
// Every thread of every CTA of the cluster arrives, then waits for all.
__device__ __forceinline__ void cluster_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// The two halves of cluster_sync, for work in between.
__device__ __forceinline__ void cluster_arrive() {
  asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory");
}

__device__ __forceinline__ void cluster_wait() { asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory"); }

// Stores 16 bytes into another CTA's shared memory (cluster addresses from
// map_to_rank) and counts them on that CTA's mbarrier as transaction bytes.
__device__ __forceinline__ void st_async_f32x4(uint32_t cluster_addr, float4 v, uint32_t cluster_bar) {
  asm volatile("st.async.shared::cluster.mbarrier::complete_tx::bytes.v4.f32 [%0], {%1, %2, %3, %4}, [%5];" ::"r"(
                   cluster_addr),
               "f"(v.x), "f"(v.y), "f"(v.z), "f"(v.w), "r"(cluster_bar)
               : "memory");
}

// try_wait with acquire at cluster scope: the phase's completion also makes
// the data that other CTAs of the cluster delivered with it visible.
__device__ __forceinline__ bool mbar_try_wait_cluster(uint32_t bar, uint32_t parity) {
  uint32_t done;
  asm volatile(
      "{\n"
      "  .reg .pred p;\n"
      "  mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n"
      "  selp.u32 %0, 1, 0, p;\n"
      "}\n"
      : "=r"(done)
      : "r"(bar), "r"(parity)
      : "memory");
  return done != 0;
}

__device__ __forceinline__ uint32_t cluster_ctarank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}

// Address of the same shared-memory location in CTA `rank` of the cluster.
__device__ __forceinline__ uint32_t map_to_rank(uint32_t saddr, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(saddr), "r"(rank));
  return r;
}

__device__ __forceinline__ float4 ld_dsmem_f32x4(uint32_t cluster_addr) {
  float4 v;
  asm volatile("ld.shared::cluster.v4.f32 {%0, %1, %2, %3}, [%4];"
               : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
               : "r"(cluster_addr)
               : "memory");
  return v;
}

__device__ __forceinline__ float ld_dsmem_f32(uint32_t cluster_addr) {
  float v;
  asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(cluster_addr) : "memory");
  return v;
}

// ------------------------------------------------------ tensor memory --
__device__ __forceinline__ void tmem_alloc(uint32_t dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst_smem), "r"(ncols)
               : "memory");
}

__device__ __forceinline__ void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}

__device__ __forceinline__ void tc_fence_before_sync() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}

__device__ __forceinline__ void tc_fence_after_sync() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// D[tmem] (+)= A[tmem] * B[smem]^T, kind::f16 (FP16 inputs, FP32 accumulator).
__device__ __forceinline__ void mma_f16_tmem_a(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                               uint32_t accumulate) {
  asm volatile(
      "{\n"
      "  .reg .pred p;\n"
      "  setp.ne.b32 p, %4, 0;\n"
      "  tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n"
      "}\n" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

__device__ __forceinline__ void mma_f16_tmem_a_elected(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc,
                                                       uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n"
      "  .reg .pred p, e;\n"
      "  setp.ne.b32 p, %4, 0;\n"
      "  elect.sync _|e, 0xffffffff;\n"
      "  @e tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n"
      "}\n" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// The 8 MMAs of one 128-wide K group (K=16 each), issued by one elected
// lane: A from TMEM columns a_tmem + 8kk, B from SW128 K slices of SLICE
// bytes (descriptor start addresses advance by 32 bytes within a slice and by
// SLICE bytes between the two).  The first MMA overwrites D.
template <int SLICE>
__device__ __forceinline__ void mma8_f16_tmem_a_elected(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc,
                                                        uint32_t idesc) {
  static_assert(SLICE % 16 == 0 && SLICE / 16 + 6 < (1 << 14), "descriptor start-address offsets");
  asm volatile(
      "{\n"
      "  .reg .pred e, f, t;\n"
      "  .reg .b64 b1, b2, b3, b4, b5, b6, b7;\n"
      "  .reg .b32 a1, a2, a3, a4, a5, a6, a7;\n"
      "  setp.ne.b32 f, %3, %3;\n"
      "  setp.eq.b32 t, %3, %3;\n"
      "  add.s64 b1, %2, 2;\n"
      "  add.s64 b2, %2, 4;\n"
      "  add.s64 b3, %2, 6;\n"
      "  add.s64 b4, %2, %4;\n"
      "  add.s64 b5, %2, %5;\n"
      "  add.s64 b6, %2, %6;\n"
      "  add.s64 b7, %2, %7;\n"
      "  add.u32 a1, %1, 8;\n"
      "  add.u32 a2, %1, 16;\n"
      "  add.u32 a3, %1, 24;\n"
      "  add.u32 a4, %1, 32;\n"
      "  add.u32 a5, %1, 40;\n"
      "  add.u32 a6, %1, 48;\n"
      "  add.u32 a7, %1, 56;\n"
      "  elect.sync _|e, 0xffffffff;\n"
      "  @e tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, f;\n"
      "  @e tcgen05.mma.cta_group::1.kind::f16 [%0], [a1], b1, %3, t;\n"
      "  @e tcgen05.mma.cta_group::1.kind::f16 [%0], [a2], b2, %3, t;\n"
      "  @e tcgen05.mma.cta_group::1.kind::f16 [%0], [a3], b3, %3, t;\n"
      "  @e tcgen05.mma.cta_group::1.kind::f16 [%0], [a4], b4, %3, t;\n"
      "  @e tcgen05.mma.cta_group::1.kind::f16 [%0], [a5], b5, %3, t;\n"
      "  @e tcgen05.mma.cta_group::1.kind::f16 [%0], [a6], b6, %3, t;\n"
      "  @e tcgen05.mma.cta_group::1.kind::f16 [%0], [a7], b7, %3, t;\n"
      "}\n" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "n"(SLICE / 16), "n"(SLICE / 16 + 2), "n"(SLICE / 16 + 4),
      "n"(SLICE / 16 + 6)
      : "memory");
}

// The elected lane (the one that issued the MMAs) commits.
__device__ __forceinline__ void mma_commit_elected(uint32_t bar) {
  asm volatile(
      "{\n"
      "  .reg .pred e;\n"
      "  elect.sync _|e, 0xffffffff;\n"
      "  @e tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];\n"
      "}\n" ::"r"(bar)
      : "memory");
}

// Arrive once on `bar` when every tcgen05 operation this thread issued so
// far has completed.
__device__ __forceinline__ void mma_commit(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
               : "memory");
}

// Each thread of the warp writes 8 consecutive 32-bit columns of its lane.
__device__ __forceinline__ void tmem_store_8(uint32_t taddr, const uint32_t* v) {
  asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"r"(taddr),
               "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7])
               : "memory");
}

__device__ __forceinline__ void tmem_store_wait() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// Each thread of the warp reads 8 consecutive 32-bit columns of its lane.
__device__ __forceinline__ void tmem_load_8(uint32_t taddr, uint32_t* v) {
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
               : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7])
               : "r"(taddr)
               : "memory");
}

// Each thread of the warp reads 16 consecutive 32-bit columns of its lane.
__device__ __forceinline__ void tmem_load_16(uint32_t taddr, uint32_t* v) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
      "%15}, [%16];"
      : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7]),
        "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), "=r"(v[14]), "=r"(v[15])
      : "r"(taddr)
      : "memory");
}

__device__ __forceinline__ void tmem_load_wait() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

// --------------------------------------------------------- descriptors --
// Shared-memory matrix descriptor for a K-major operand tile written by TMA
// with 128-byte swizzling: rows of 128 bytes, 8-row groups 1024 bytes apart.
// Fields: start address >> 4 in bits 0-13, leading byte offset >> 4 in bits
// 16-29 (unused for this layout), stride byte offset >> 4 in bits 32-45,
// version 1 in bits 46-47, swizzle mode 2 (128B) in bits 61-63.
__device__ __forceinline__ uint64_t sw128_kmajor_desc(uint32_t saddr) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((saddr & 0x3FFFFu) >> 4);
  d |= static_cast<uint64_t>(1u) << 16;
  d |= static_cast<uint64_t>(1024u >> 4) << 32;
  d |= static_cast<uint64_t>(1u) << 46;
  d |= static_cast<uint64_t>(2u) << 61;
  return d;
}

// Instruction descriptor, kind::f16: FP32 accumulator (bits 4-5 = 1), A and B
// FP16 (bits 7-9, 10-12 = 0), both K-major (bits 15, 16 = 0), N >> 3 in bits
// 17-22, M >> 4 in bits 24-28.
__host__ __device__ constexpr uint32_t f16_instr_desc(int m, int n) {
  return (1u << 4) | (static_cast<uint32_t>(n >> 3) << 17) | (static_cast<uint32_t>(m >> 4) << 24);
}

// ------------------------------------------------------- global loads ---
// One 32-byte read-only load (the address 32-byte aligned) as two uint4.
__device__ __forceinline__ void ldg_32b(const void* p, uint4& lo, uint4& hi) {
  asm volatile("ld.global.nc.v8.u32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
               : "=r"(lo.x), "=r"(lo.y), "=r"(lo.z), "=r"(lo.w), "=r"(hi.x), "=r"(hi.y), "=r"(hi.z), "=r"(hi.w)
               : "l"(reinterpret_cast<uint64_t>(p)));
}

// One 32-byte store (the address 32-byte aligned) of two uint4.
__device__ __forceinline__ void stg_32b(void* p, const uint4& lo, const uint4& hi) {
  asm volatile("st.global.v8.u32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"l"(reinterpret_cast<uint64_t>(p)),
               "r"(lo.x), "r"(lo.y), "r"(lo.z), "r"(lo.w), "r"(hi.x), "r"(hi.y), "r"(hi.z), "r"(hi.w)
               : "memory");
}

// ------------------------------------------------------------ bit ops ---
// (a & b) | c in one three-input logic instruction, b and c in registers.
__device__ __forceinline__ uint32_t and_or(uint32_t a, uint32_t b, uint32_t c) {
  uint32_t d;
  asm("lop3.b32 %0, %1, %2, %3, 0xEA;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
  return d;
}

// ------------------------------------------------------------- f16x2 ---
__device__ __forceinline__ uint32_t hmul2_bits(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("mul.rn.f16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}

}  // namespace bonsai

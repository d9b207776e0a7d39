// Thin inline-PTX wrappers for sm_100a: mbarriers, cp.async, TMA tiled loads,
// tcgen05 (TMEM allocation, UMMA issue, commit, TMEM loads) and fences.
// Every wait in this file is bounded.  A pipeline wait gives up after the
// CTA's limit (WaitCtl::limit_ns of %globaltimer time, kWaitLimitNs unless the
// caller asked for another) or as soon as the CTA's abort word is set; a drain
// wait on the abort path has its own limit, kDrainLimitNs.
#pragma once

#include <cstdint>
#include <cuda.h>

namespace subm3d {

constexpr uint64_t kWaitLimitNs = 2000000000ull;   // 2 s: default limit of a pipeline wait
constexpr uint64_t kDrainLimitNs = 1000000000ull;  // 1 s: limit of one drain wait

// Per-CTA wait control, in shared memory.  The first pipeline wait that runs
// out of time sets `abort`; from then on every pipeline wait of the CTA
// returns false at once, each role leaves its loop, drains what it has issued
// (mbar_drain) and the CTA exits through its normal teardown.
struct WaitCtl {
  int abort;
  int pad;
  unsigned long long limit_ns;
};

// Called by one thread before the CTA's first __syncthreads.
__device__ __forceinline__ void wait_ctl_init(WaitCtl* w, uint64_t limit_ns) {
  w->abort = 0;
  w->pad = 0;
  w->limit_ns = limit_ns;
}

__device__ __forceinline__ bool wait_aborted(const WaitCtl* w) {
  return *reinterpret_cast<const volatile int*>(&w->abort) != 0;
}

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint64_t globaltimer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// ----------------------------------------------------------------- mbarrier --

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}

__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar))
               : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(
                   smem_u32(bar)),
               "r"(bytes)
               : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// One bounded-suspension poll: the thread sleeps at most about `hint_ns`
// (or until the phase completes) before the call returns.
__device__ __forceinline__ bool mbar_try_wait_hint(uint64_t* bar, uint32_t parity,
                                                   uint32_t hint_ns) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity), "r"(hint_ns)
      : "memory");
  return ok != 0;
}

// Suspension per poll of the slow paths: a quarter of the limit, between
// 256 ns and 100 us, so that a limit is noticed within about a quarter of itself.
__device__ __forceinline__ uint32_t poll_hint_ns(uint64_t limit_ns) {
  const uint64_t q = limit_ns / 4;
  return static_cast<uint32_t>(q < 256 ? 256 : (q > 100000 ? 100000 : q));
}

// Slow path of mbar_wait, kept out of line so that the many wait sites of a
// warp-specialised kernel share one copy of the polling loop.  The abort word
// and the clock are checked after every poll.
static __device__ __noinline__ bool mbar_wait_slow(uint64_t* bar, uint32_t parity, WaitCtl* w) {
  volatile WaitCtl* vw = w;
  const uint64_t limit = vw->limit_ns;
  const uint32_t hint = poll_hint_ns(limit);
  const uint64_t t0 = globaltimer_ns();
  for (;;) {
    if (mbar_try_wait_hint(bar, parity, hint)) return true;
    if (vw->abort) return false;
    if (globaltimer_ns() - t0 > limit) {
      vw->abort = 1;
      return false;
    }
  }
}

// Waits for the phase of `bar` with the given parity to complete.  Returns
// false (and sets the abort word) when the wait exceeds the CTA's limit, or
// returns false at once when another role of the CTA has already set it.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, WaitCtl* w) {
  if (mbar_try_wait(bar, parity)) return true;
  return mbar_wait_slow(bar, parity, w);
}

// Abort path: waits for the phase of `bar` with the given parity to complete,
// whatever the abort word says, for at most kDrainLimitNs.  A role calls it
// for each asynchronous operation it issued (a TMA or bulk copy into shared
// memory, a tcgen05.commit after its MMAs) before the CTA frees its tensor
// memory and exits, so that nothing still writes shared or tensor memory the
// CTA no longer owns.  Returns false if the limit ran out.
static __device__ __noinline__ bool mbar_drain(uint64_t* bar, uint32_t parity) {
  const uint64_t t0 = globaltimer_ns();
  for (;;) {
    if (mbar_try_wait_hint(bar, parity, 100000)) return true;
    if (globaltimer_ns() - t0 > kDrainLimitNs) return false;
  }
}

__device__ __forceinline__ void sts_u32(uint32_t addr, uint32_t v) {
  asm volatile("st.shared.u32 [%0], %1;" ::"r"(addr), "r"(v) : "memory");
}

__device__ __forceinline__ void sts_u16(uint32_t addr, uint16_t v) {
  asm volatile("st.shared.u16 [%0], %1;" ::"r"(addr), "h"(v) : "memory");
}

__device__ __forceinline__ uint4 lds_16(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "r"(addr)
               : "memory");
  return v;
}

// ----------------------------------------------------------------- cp.async --

// 16-byte global->shared copy; src_bytes = 0 writes 16 zero bytes.
__device__ __forceinline__ void cp_async_16(uint32_t dst, const void* src, uint32_t src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src),
               "r"(src_bytes)
               : "memory");
}

// Waits until every cp.async copy this thread issued has landed.
__device__ __forceinline__ void cp_async_wait_all() {
  asm volatile("cp.async.wait_all;" ::: "memory");
}

// Arrive on `bar` once all cp.async copies this thread issued so far have
// landed.  .noinc: the arrival is one of the barrier's expected arrivals.
__device__ __forceinline__ void cp_async_mbar_arrive_noinc(uint64_t* bar) {
  asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(smem_u32(bar))
               : "memory");
}

// Makes this thread's generic-proxy shared-memory writes visible to the async
// proxy (tensor core operand reads, TMA).
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// --------------------------------------------------------------------- TMA --

__device__ __forceinline__ void tma_prefetch_desc(const CUtensorMap* map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// 3-D tiled TMA load into this CTA's shared memory, completing on `bar`.
__device__ __forceinline__ void tma_load_3d(uint32_t dst, const CUtensorMap* map, uint64_t* bar,
                                            int32_t c0, int32_t c1, int32_t c2) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5}], [%2];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(c0), "r"(c1), "r"(c2)
      : "memory");
}

// 1-D bulk copy global -> this CTA's shared memory (16-byte aligned, size a
// multiple of 16), completing on `bar`.
__device__ __forceinline__ void bulk_load(uint32_t dst, const void* src, uint32_t bytes,
                                          uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          dst),
      "l"(src), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

// ----------------------------------------------------------------- tcgen05 --

__device__ __forceinline__ void tmem_alloc(uint32_t* dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                   smem_u32(dst_smem)),
               "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// D[tmem] (+)= A[smem] * B[smem]^T, kind::f16 (bf16 inputs, fp32 accumulate).
__device__ __forceinline__ void umma_bf16(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                          uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Arrive once on `bar` when all tcgen05 operations this thread issued so far complete.
__device__ __forceinline__ void umma_commit(uint64_t* bar) {
  asm volatile(
      "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
          smem_u32(bar))
      : "memory");
}

// Each thread of the warp reads 32 consecutive fp32 columns of its TMEM lane.
__device__ __forceinline__ void tmem_ld_32x32b_x32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
      "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]),
        "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]),
        "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
}
__device__ __forceinline__ void tmem_ld_wait() {
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// Shared-memory matrix descriptor for a K-major operand in a swizzled layout
// with rows of `row_bytes` (128, 64 or 32) and 8-row atoms stacked along M/N
// (stride 8 * row_bytes); layout codes 2 (128 B), 4 (64 B), 6 (32 B).
__device__ __forceinline__ uint64_t smem_desc_sw(uint32_t saddr, uint32_t row_bytes) {
  const uint32_t layout = row_bytes == 128 ? 2u : (row_bytes == 64 ? 4u : 6u);
  uint64_t d = 0;
  d |= static_cast<uint64_t>((saddr & 0x3FFFFu) >> 4);
  d |= static_cast<uint64_t>(1u) << 16;
  d |= static_cast<uint64_t>((8u * row_bytes) >> 4) << 32;
  d |= static_cast<uint64_t>(1u) << 46;
  d |= static_cast<uint64_t>(layout) << 61;
  return d;
}

// Descriptor of an MN-major operand in the 128-byte swizzle layout: rows of
// 128 bytes (64 consecutive M or N elements) at consecutive K, 8 rows per
// 1024-byte swizzle atom, atoms `sbo` bytes apart along K and `lbo` bytes apart
// along M/N (the canonical ((8,n),(8,k)):((1,LBO),(8,SBO)) layout in 16-byte
// units); layout type 2 at [61,64), version 1 at [46,48), base offset 0.
__device__ __forceinline__ uint64_t smem_desc_mn_sw128(uint32_t saddr, uint32_t lbo,
                                                       uint32_t sbo) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((saddr & 0x3FFFFu) >> 4);
  d |= static_cast<uint64_t>((lbo >> 4) & 0x3FFFu) << 16;
  d |= static_cast<uint64_t>((sbo >> 4) & 0x3FFFu) << 32;
  d |= static_cast<uint64_t>(1u) << 46;
  d |= static_cast<uint64_t>(2u) << 61;
  return d;
}

// Instruction descriptor, kind::f16: fp32 accumulator (bits [4,6) = 1), bf16 A
// and B ([7,10) = 1, [10,13) = 1), both K-major (bits 15, 16 = 0), N >> 3 at
// [17,23), M >> 4 at [24,29).
__host__ __device__ constexpr uint32_t idesc_bf16_f32(uint32_t m, uint32_t n) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((n >> 3) << 17) | ((m >> 4) << 24);
}

// The same with both operands MN-major (A: bit 15, B: bit 16).
__host__ __device__ constexpr uint32_t idesc_bf16_f32_mn(uint32_t m, uint32_t n) {
  return idesc_bf16_f32(m, n) | (1u << 15) | (1u << 16);
}

// ------------------------------------------------------------- abort path --

// A TMA producer's drain: load m of the producer went to ring slot m % slots and
// completes the phase of parity (m / slots) & 1 of full[slot]; the last
// min(issued, slots) loads are the only ones that can still be in flight.
__device__ __forceinline__ void drain_ring(uint64_t* full, int slots, int64_t issued) {
  const int64_t first = issued > slots ? issued - slots : 0;
  for (int64_t m = first; m < issued; ++m)
    mbar_drain(&full[m % slots], static_cast<uint32_t>((m / slots) & 1));
}

// The MMA issuer's drain: tcgen05.commit tracks every tcgen05 operation the
// thread issued before it, so one commit to `bar` (a count-1 barrier used for
// nothing else) and a wait for its first phase cover all of them.
__device__ __forceinline__ void drain_mma(uint64_t* bar) {
  umma_commit(bar);
  mbar_drain(bar, 0);
}

}  // namespace subm3d

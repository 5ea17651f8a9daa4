// Thin inline-PTX wrappers for sm_100a: mbarriers with bounded waits, TMA
// (tensor and bulk copies, stores), tcgen05 across a CTA pair (TMEM
// allocation, MMAs, scale copies, loads), warp-level MMAs, clusters and the
// NVFP4 conversion instructions.
#pragma once

#include <cstdint>
#include <cuda_bf16.h>
#include <cuda_fp16.h>

namespace svdq {

// ------------------------------------------------------------ status word --
// One per device: SVDQ_ERR_TIMEOUT and the id of the wait that expired.
__device__ unsigned int g_status_code = 0;
__device__ unsigned int g_status_where = 0;

__device__ __forceinline__ void record_timeout(unsigned int where) {
  if (atomicCAS(&g_status_code, 0u, 5u) == 0u) atomicExch(&g_status_where, where);
}

// ------------------------------------------------------------------ misc --
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint64_t globaltimer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// ------------------------------------------------------------- mbarriers --
__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count));
}

__device__ __forceinline__ void fence_barrier_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

// Longest time (ns) one try_wait may keep the thread suspended in hardware
// before it returns false; waiters sleep instead of spinning, and the bounded
// waits below still look at the clock between calls.
constexpr uint32_t kSuspendHintNs = 1000000;

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity), "n"(kSuspendHintNs)
      : "memory");
  return ok != 0;
}

// Bounded wait for the phase with the given parity.  Returns false (and
// records a timeout with id `where`) when `timeout_ns` elapses first.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, uint64_t timeout_ns,
                                          unsigned int where) {
#pragma unroll 1
  for (int i = 0; i < 32; ++i)
    if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
#pragma unroll 1
  while (true) {
    if (mbar_try_wait(bar, parity)) return true;
    if (globaltimer_ns() - t0 > timeout_ns) {
      record_timeout(where);
      return false;
    }
  }
}

// ------------------------------------------- programmatic dependent launch --
// The layer's kernels are launched with the programmatic stream-serialisation
// attribute: a grid may be scheduled while the kernel ahead of it in the
// stream still runs, once every CTA of that kernel has issued
// griddep_launch_dependents() (or exited).  griddep_wait() returns when the
// kernel ahead has completed and its memory writes are visible; every thread
// waits before it touches global memory the kernel ahead may write or read
// (L2 prefetches excepted: L2 is the device's point of coherence, so a
// prefetch can fetch a line early but never a stale one).  Without such a
// predecessor the wait returns at once.
__device__ __forceinline__ void griddep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

__device__ __forceinline__ void griddep_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// ------------------------------------------------------------------- TMA --

__device__ __forceinline__ void prefetch_tmap(const void* tmap) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(tmap) : "memory");
}

// Generic-proxy writes to shared memory -> visible to the async proxy
// (tensor cores, TMA).
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// --------------------------------------------------------------- tcgen05 --

__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}

__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

__device__ __forceinline__ void tmem_ld_wait() {
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// 32 lanes x 32 bit, 32 consecutive columns: thread t gets lane (base + t).
__device__ __forceinline__ void tmem_ld_32x32b_x32(uint32_t taddr, uint32_t* v) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
      "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
      : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]),
        "=r"(v[7]), "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]),
        "=r"(v[14]), "=r"(v[15]), "=r"(v[16]), "=r"(v[17]), "=r"(v[18]), "=r"(v[19]), "=r"(v[20]),
        "=r"(v[21]), "=r"(v[22]), "=r"(v[23]), "=r"(v[24]), "=r"(v[25]), "=r"(v[26]), "=r"(v[27]),
        "=r"(v[28]), "=r"(v[29]), "=r"(v[30]), "=r"(v[31])
      : "r"(taddr));
}

// Named barrier over `count` threads (ids 1..15; id 0 is __syncthreads).
__device__ __forceinline__ void named_bar_sync(uint32_t id, uint32_t count) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(count) : "memory");
}

// Shared-memory matrix descriptor (sm100 format, version 1).
//   layout: 0 = no swizzle (8 x 16 B core matrices), 2 = 128-byte swizzle.
//   lbo/sbo: leading / stride byte offsets (multiples of 16).
__device__ __forceinline__ uint64_t make_sdesc(uint32_t saddr, uint32_t lbo, uint32_t sbo,
                                               uint32_t layout) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((saddr >> 4) & 0x3FFF);
  d |= static_cast<uint64_t>((lbo >> 4) & 0x3FFF) << 16;
  d |= static_cast<uint64_t>((sbo >> 4) & 0x3FFF) << 32;
  d |= static_cast<uint64_t>(1) << 46;  // descriptor version for sm100
  d |= static_cast<uint64_t>(layout & 7) << 61;
  return d;
}

// ------------------------------------------------------ single CTA (1-SM) --

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

// ----------------------------------------------------- CTA-pair (2-SM) --

__device__ __forceinline__ void tmem_alloc_pair(uint32_t dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst_smem),
               "r"(ncols)
               : "memory");
}

__device__ __forceinline__ void tmem_relinquish_pair() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_dealloc_pair(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
               : "memory");
}

// Arrive on an mbarrier given by its shared::cluster address (release at
// cluster scope: prior writes of this thread are visible to the waiter).
__device__ __forceinline__ void mbar_arrive_cluster(uint32_t bar_cluster) {
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(bar_cluster)
               : "memory");
}

// Arrive on a (possibly remote) mbarrier with release at CTA scope.  For a
// hand-off of tensor memory (tcgen05.wait::ld, tcgen05.fence::before_thread_sync,
// this arrive; the waiter's tcgen05.fence::after_thread_sync) no generic
// memory has to be published, and the cluster-scope release above waits for
// every earlier global store of the thread to complete: under a heavily
// loaded L2 that took about 0.6 us per arrive on B200.
__device__ __forceinline__ void mbar_arrive_remote(uint32_t bar_cluster) {
  asm volatile("mbarrier.arrive.release.cta.shared::cluster.b64 _, [%0];" ::"r"(bar_cluster) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait_cluster(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2, %3;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity), "n"(kSuspendHintNs)
      : "memory");
  return ok != 0;
}

// Bounded wait (acquire at cluster scope) for barriers that threads of the
// peer CTA arrive on.
__device__ __forceinline__ bool mbar_wait_cluster(uint32_t bar, uint32_t parity, uint64_t timeout_ns,
                                                  unsigned int where) {
#pragma unroll 1
  for (int i = 0; i < 32; ++i)
    if (mbar_try_wait_cluster(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
#pragma unroll 1
  while (true) {
    if (mbar_try_wait_cluster(bar, parity)) return true;
    if (globaltimer_ns() - t0 > timeout_ns) {
      record_timeout(where);
      return false;
    }
  }
}

// ------------------------------------------------- warp-wide issue (elect) --
// Issue loops run with the whole warp converged and let elect.sync pick the
// single lane that executes the instruction: this keeps the loop's values on
// the warp-uniform path (a loop run by one lane inside a divergent branch
// issues tcgen05 MMAs at well under half their rate).
#define SVDQ_ELECT_BEGIN "{\n\t.reg .pred e;\n\t.reg .b32 rx;\n\telect.sync rx|e, 0xffffffff;\n\t"
#define SVDQ_ELECT_END "\n\t}"

__device__ __forceinline__ void e_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile(SVDQ_ELECT_BEGIN "@e mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" SVDQ_ELECT_END ::"r"(bar),
               "r"(bytes)
               : "memory");
}

__device__ __forceinline__ void e_tma_load_2d(uint32_t dst, const void* tmap, uint32_t bar, int x, int y) {
  asm volatile(SVDQ_ELECT_BEGIN
               "@e cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes"
               " [%0], [%1, {%2, %3}], [%4];" SVDQ_ELECT_END ::"r"(dst),
               "l"(tmap), "r"(x), "r"(y), "r"(bar)
               : "memory");
}

// TMA load into this CTA's shared memory whose completion bytes go to the
// mbarrier at `bar_cluster` (a shared::cluster address, possibly the peer's).
__device__ __forceinline__ void e_tma_load_2d_pair(uint32_t dst, const void* tmap, uint32_t bar_cluster, int x,
                                                   int y) {
  asm volatile(SVDQ_ELECT_BEGIN
               "@e cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
               " [%0], [%1, {%2, %3}], [%4];" SVDQ_ELECT_END ::"r"(dst),
               "l"(tmap), "r"(x), "r"(y), "r"(bar_cluster)
               : "memory");
}

// Prefetch a 2-D box of a tensor into L2 (no shared memory, no barrier).
__device__ __forceinline__ void e_tma_prefetch_2d(const void* tmap, int x, int y) {
  asm volatile(SVDQ_ELECT_BEGIN "@e cp.async.bulk.prefetch.tensor.2d.L2.global.tile [%0, {%1, %2}];" SVDQ_ELECT_END ::"l"(
                   tmap),
               "r"(x), "r"(y)
               : "memory");
}

// Prefetch a 3-D box of a tensor into L2.
__device__ __forceinline__ void e_tma_prefetch_3d(const void* tmap, int x, int y, int z) {
  asm volatile(SVDQ_ELECT_BEGIN "@e cp.async.bulk.prefetch.tensor.3d.L2.global.tile [%0, {%1, %2, %3}];" SVDQ_ELECT_END ::"l"(
                   tmap),
               "r"(x), "r"(y), "r"(z)
               : "memory");
}

// Untiled bulk copy global -> shared (16-byte aligned, size multiple of 16).
__device__ __forceinline__ void e_bulk_load(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar) {
  asm volatile(SVDQ_ELECT_BEGIN
               "@e cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" SVDQ_ELECT_END ::
                   "r"(dst),
               "l"(src), "r"(bytes), "r"(bar)
               : "memory");
}

// One CTA's MMA: D (tmem) (+)= A x B, bf16 operands, fp32 accumulator.
__device__ __forceinline__ void e_mma_bf16(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                           uint32_t accumulate) {
  asm volatile(SVDQ_ELECT_BEGIN ".reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
               "@e tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;" SVDQ_ELECT_END ::"r"(d_tmem),
               "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
               : "memory");
}

// One CTA's block-scaled FP4 MMA (E2M1 operands, UE4M3 scale per 16 along K,
// scale factors read from tmem).
__device__ __forceinline__ void e_mma_nvf4(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                           uint32_t sfa_tmem, uint32_t sfb_tmem, uint32_t accumulate) {
  asm volatile(SVDQ_ELECT_BEGIN ".reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
               "@e tcgen05.mma.cta_group::1.kind::mxf4nvf4.block_scale.block16 [%0], %1, %2, %3, [%5], [%6], p;" SVDQ_ELECT_END ::
                   "r"(d_tmem),
               "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(sfa_tmem), "r"(sfb_tmem)
               : "memory");
}

// Arrive once on this CTA's mbarrier when all prior tcgen05 ops of this
// thread are complete.
__device__ __forceinline__ void e_commit(uint32_t bar) {
  asm volatile(SVDQ_ELECT_BEGIN "@e tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" SVDQ_ELECT_END ::
                   "r"(bar)
               : "memory");
}

__device__ __forceinline__ void e_arrive(uint32_t bar) {
  asm volatile(SVDQ_ELECT_BEGIN "@e mbarrier.arrive.shared::cta.b64 _, [%0];" SVDQ_ELECT_END ::"r"(bar) : "memory");
}

// Copy 32 rows x 128 bits from shared memory into tensor memory, replicated
// into the four 32-lane quadrants (one CTA).
__device__ __forceinline__ void e_tmem_cp_32x128b_warpx4(uint32_t taddr, uint64_t sdesc) {
  asm volatile(SVDQ_ELECT_BEGIN "@e tcgen05.cp.cta_group::1.32x128b.warpx4 [%0], %1;" SVDQ_ELECT_END ::"r"(taddr),
               "l"(sdesc)
               : "memory");
}

__device__ __forceinline__ void e_tma_load_3d(uint32_t dst, const void* tmap, uint32_t bar, int x, int y, int z) {
  asm volatile(SVDQ_ELECT_BEGIN
               "@e cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes"
               " [%0], [%1, {%2, %3, %4}], [%5];" SVDQ_ELECT_END ::"r"(dst),
               "l"(tmap), "r"(x), "r"(y), "r"(z), "r"(bar)
               : "memory");
}

// MMAs across the CTA pair (issued by the even CTA): A rows split by CTA,
// B columns split by CTA, D rows in each CTA's own tensor memory.
__device__ __forceinline__ void e_mma_bf16_pair(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                                uint32_t accumulate) {
  asm volatile(SVDQ_ELECT_BEGIN ".reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
               "@e tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;" SVDQ_ELECT_END ::"r"(d_tmem),
               "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
               : "memory");
}

// D (tmem) (+)= (A * SFA) x (B * SFB): FP4 E2M1 operands, UE4M3 scale per
// 16 elements along K (scale factors read from tmem).
__device__ __forceinline__ void e_mma_nvf4_pair(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                                uint32_t sfa_tmem, uint32_t sfb_tmem, uint32_t accumulate) {
  asm volatile(SVDQ_ELECT_BEGIN ".reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
               "@e tcgen05.mma.cta_group::2.kind::mxf4nvf4.block_scale.block16 [%0], %1, %2, %3, [%5], [%6], p;" SVDQ_ELECT_END ::
                   "r"(d_tmem),
               "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(sfa_tmem), "r"(sfb_tmem)
               : "memory");
}

// Arrive once on the mbarrier at the same shared-memory offset in both CTAs
// of the pair when all prior tcgen05 ops of this thread are complete.
__device__ __forceinline__ void e_commit_pair_both(uint32_t bar) {
  asm volatile(SVDQ_ELECT_BEGIN
               "@e tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64"
               " [%0], %1;" SVDQ_ELECT_END ::"r"(bar),
               "h"(static_cast<uint16_t>(3))
               : "memory");
}

// Retire `bytes` expected transaction bytes of an mbarrier's current phase
// as if they had arrived (one elected lane; no arrival is counted).
__device__ __forceinline__ void e_mbar_complete_tx(uint32_t bar, uint32_t bytes) {
  asm volatile(SVDQ_ELECT_BEGIN "@e mbarrier.complete_tx.shared::cta.b64 [%0], %1;" SVDQ_ELECT_END ::"r"(bar),
               "r"(bytes)
               : "memory");
}

// Store a 32-bit value to a shared::cluster address (possibly the peer CTA's).
__device__ __forceinline__ void st_dsmem_u32(uint32_t addr, uint32_t v) {
  asm volatile("st.shared::cluster.u32 [%0], %1;" ::"r"(addr), "r"(v) : "memory");
}

// Warp-uniform bounded waits: every lane polls, lane 0's outcome decides for
// the whole warp (a warp that issues through elect.sync must stay converged).
__device__ __forceinline__ bool warp_wait(uint32_t bar, uint32_t parity, uint64_t timeout_ns, unsigned int where) {
  const bool ok = mbar_wait(bar, parity, timeout_ns, where);
  return __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
}

__device__ __forceinline__ bool warp_wait_cluster(uint32_t bar, uint32_t parity, uint64_t timeout_ns,
                                                  unsigned int where) {
  const bool ok = mbar_wait_cluster(bar, parity, timeout_ns, where);
  return __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
}

__device__ __forceinline__ bool warp_flag(const volatile int* flag) {
  return __shfl_sync(0xffffffffu, *flag, 0) != 0;
}

__device__ __forceinline__ void e_tma_load_3d_pair(uint32_t dst, const void* tmap, uint32_t bar_cluster, int x,
                                                   int y, int z) {
  asm volatile(SVDQ_ELECT_BEGIN
               "@e cp.async.bulk.tensor.3d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
               " [%0], [%1, {%2, %3, %4}], [%5];" SVDQ_ELECT_END ::"r"(dst),
               "l"(tmap), "r"(x), "r"(y), "r"(z), "r"(bar_cluster)
               : "memory");
}

// Copy 32 rows x 128 bits from shared memory into tensor memory, replicated
// into the four 32-lane quadrants, in both CTAs of the pair (each from its
// own shared memory at the same offset).
__device__ __forceinline__ void e_tmem_cp_pair_32x128b_warpx4(uint32_t taddr, uint64_t sdesc) {
  asm volatile(SVDQ_ELECT_BEGIN "@e tcgen05.cp.cta_group::2.32x128b.warpx4 [%0], %1;" SVDQ_ELECT_END ::"r"(taddr),
               "l"(sdesc)
               : "memory");
}

// TMA store of a 2-D box from shared memory (bulk-group completion).
__device__ __forceinline__ void tma_store_2d(const void* tmap, uint32_t src, int x, int y) {
  asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%2, %3}], [%1];" ::"l"(tmap), "r"(src),
               "r"(x), "r"(y)
               : "memory");
}

// Untiled bulk copy shared -> global (bulk-group completion; 16-byte aligned,
// size a multiple of 16).
__device__ __forceinline__ void bulk_store(void* gdst, uint32_t ssrc, uint32_t bytes) {
  asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;" ::"l"(gdst), "r"(ssrc), "r"(bytes)
               : "memory");
}

__device__ __forceinline__ void bulk_commit_group() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }

// Wait until at most N bulk groups of this thread still read shared memory.
template <int N>
__device__ __forceinline__ void bulk_wait_group_read() {
  asm volatile("cp.async.bulk.wait_group.read %0;" ::"n"(N) : "memory");
}

template <int N>
__device__ __forceinline__ void bulk_wait_group() {
  asm volatile("cp.async.bulk.wait_group %0;" ::"n"(N) : "memory");
}

// ------------------------------------------------- warp-level MMA (mma.sync) --
// Four 8x8 b16 matrices from shared memory; lane i supplies the row address of
// matrix i / 8 (row i % 8).
__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_trans(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                              uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
// D (16x8 fp32) = A (16x16 bf16, row) * B (16x8 bf16, col) + C
__device__ __forceinline__ void mma_bf16_16816(float* d, const uint32_t* a, uint32_t b0, uint32_t b1,
                                               const float* c) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%10, %11, %12, %13};"
      : "=f"(d[0]), "=f"(d[1]), "=f"(d[2]), "=f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1), "f"(c[0]), "f"(c[1]), "f"(c[2]),
        "f"(c[3]));
}

// ------------------------------------------------------------- clusters --
__device__ __forceinline__ uint32_t cluster_ctarank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}

__device__ __forceinline__ void cluster_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::
                   : "memory");
}

// Four fp32 values from a shared::cluster address (possibly another CTA's).
__device__ __forceinline__ float4 ld_dsmem_f32x4(uint32_t addr) {
  float4 v;
  asm volatile("ld.shared::cluster.v4.f32 {%0, %1, %2, %3}, [%4];"
               : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
               : "r"(addr)
               : "memory");
  return v;
}

__device__ __forceinline__ uint32_t cluster_id_x() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%clusterid.x;" : "=r"(r));
  return r;
}

__device__ __forceinline__ void tmem_ld_32x32b_x16(uint32_t taddr, uint32_t* v) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15}, [%16];"
      : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7]),
        "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), "=r"(v[14]), "=r"(v[15])
      : "r"(taddr));
}

__device__ __forceinline__ uint32_t map_shared_rank(uint32_t saddr, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(saddr), "r"(rank));
  return r;
}

// ------------------------------------------------------- NVFP4 convert --
// fp32 -> E4M3 (round to nearest even, saturating); returns the byte.
__device__ __forceinline__ uint32_t cvt_e4m3_satfinite(float x) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(0.0f), "f"(x));
  return r & 0xFFu;
}

// E4M3 byte -> fp32 (exact).
__device__ __forceinline__ float e4m3_to_f32(uint32_t code) {
  uint32_t h2;
  uint16_t c = static_cast<uint16_t>(code & 0xFFu);
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h2) : "h"(c));
  return __half2float(__ushort_as_half(static_cast<unsigned short>(h2 & 0xFFFFu)));
}

// Eight fp32 values -> eight E2M1 codes packed little-endian into 32 bits:
// element i in bits [4i, 4i+4).  Round to nearest even, saturating to 6.
__device__ __forceinline__ uint32_t cvt_e2m1x8(const float* v) {
  uint32_t out;
  asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b0, %2, %1;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b1, %4, %3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b2, %6, %5;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b3, %8, %7;\n\t"
      "mov.b32 %0, {b0, b1, b2, b3};\n\t}"
      : "=r"(out)
      : "f"(v[0]), "f"(v[1]), "f"(v[2]), "f"(v[3]), "f"(v[4]), "f"(v[5]), "f"(v[6]), "f"(v[7]));
  return out;
}

}  // namespace svdq

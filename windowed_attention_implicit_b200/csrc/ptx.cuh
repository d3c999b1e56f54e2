// ptx.cuh -- inline-PTX building blocks for sm_100a: mbarriers with bounded
// waits, TMA tensor copies, tcgen05 tensor-core MMAs, tensor memory (TMEM)
// allocation / loads / stores and the shared-memory matrix descriptors.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <stdint.h>

namespace rib {

// ---------------------------------------------------------------- status word
// g_status[0]: first error code recorded by any kernel (0 = none)
// g_status[1]: site code of the wait that gave up
__device__ int g_status[2];

enum WaitSite : int {
  SITE_DEBUG = 1,
  SITE_FWD_PRODUCER = 10, SITE_FWD_MMA = 11, SITE_FWD_SOFTMAX = 12, SITE_FWD_DRAIN = 13,
  SITE_BWD_PRODUCER = 20, SITE_BWD_MMA = 21, SITE_BWD_COMPUTE = 22, SITE_BWD_DRAIN = 23,
  SITE_COPY = 30, SITE_CLA = 40,
};

constexpr int kErrTimeout = -6;

__device__ __forceinline__ void record_error(int code, int site) {
  if (atomicCAS(&g_status[0], 0, code) == 0) atomicExch(&g_status[1], site);
}

// ---------------------------------------------------------------- debug guards
// In the debug build (RIB_DEBUG, librib_debug.so) every global access that
// does not go through a TMA tensor map is tested first: an element index at
// or beyond its buffer's extent (derived from the call's shapes) records
// RIB_ERR_BOUNDS with the site, the index and the extent, and the access is
// skipped.  In the release build rib_guard is `true` and compiles away.
constexpr int kErrBounds = -8;
enum GuardSite : int {
  G_FWD_OUT = 100, G_FWD_LSE, G_FWD_GATE, G_FWD_OUT_GATED,
  G_TF32_OUT = 110, G_TF32_LSE,
  G_BWD_DQKV = 120, G_BWD_DKP_PART, G_BWD_DQ_ACC, G_BWD_PRE_IN, G_BWD_PRE_OUT,
  G_BWD_PRE_ZERO, G_DQ_FIN_IN, G_DQ_FIN_OUT, G_POSGRAD_IN, G_POSGRAD_OUT,
  G_POS_W = 140, G_POS_OUT, G_MLP_IN, G_MLP_PART, G_MLP_OUT,
  G_CLA_W = 150, G_CLA_GATE, G_CLA_IN, G_CLA_OUT, G_CLA_PART, G_CLA_RED,
  G_SELFTEST = 190,
};
#ifdef RIB_DEBUG
// [0] element index, [1] extent of the first access a guard refused
__device__ unsigned long long g_guard_info[2];
__device__ __noinline__ bool rib_guard_fail(unsigned long long idx, unsigned long long n,
                                            int site) {
  if (atomicCAS(&g_status[0], 0, kErrBounds) == 0) {
    atomicExch(&g_status[1], site);
    atomicExch(&g_guard_info[0], idx);
    atomicExch(&g_guard_info[1], n);
  }
  return false;
}
__device__ __forceinline__ bool rib_guard(unsigned long long idx, unsigned long long n,
                                          int site) {
  return idx < n ? true : rib_guard_fail(idx, n, site);
}
#else
__device__ __forceinline__ constexpr bool rib_guard(unsigned long long, unsigned long long,
                                                    int) {
  return true;
}
#endif

__device__ __forceinline__ uint64_t globaltimer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// ---------------------------------------------------------------- mbarrier
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count)
               : "memory");
}

__device__ __forceinline__ void fence_mbarrier_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.release.cta.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar))
               : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.release.cta.shared::cta.b64 _, [%0], %1;" ::"r"(
                   smem_u32(bar)),
               "r"(bytes)
               : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.acquire.cta.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// The same test, but the thread may sleep in it for up to `hint_ns` until
// the phase completes, instead of returning at once: waiting warps then give
// their issue slots to the warps that have work.
__device__ __forceinline__ bool mbar_try_wait_sleep(uint64_t* bar, uint32_t parity,
                                                    uint32_t hint_ns) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.acquire.cta.shared::cta.b64 p, [%1], %2, %3;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity), "r"(hint_ns)
      : "memory");
  return ok != 0;
}

// Bounded wait for the phase with the given parity to complete.  Gives up
// when `abort` (a shared flag of the CTA) is set by another thread, or when
// `limit_ns` elapses; in the latter case it records RIB_ERR_TIMEOUT with the
// site code and raises the CTA's abort flag.  Returns true on success.
// The retry loop polls only the barrier: the abort flag and the (slow to
// read) global timer are checked once every 64 tries, so a waiter resumes
// within a few cycles of the phase completing.
// With `sleep_ns` > 0 each retry may sleep that long (mbar_try_wait_sleep).
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, volatile int* abort,
                                          uint64_t limit_ns, int site, uint32_t sleep_ns = 0) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  for (uint32_t it = 1;; ++it) {
    if (sleep_ns ? mbar_try_wait_sleep(bar, parity, sleep_ns) : mbar_try_wait(bar, parity))
      return true;
    if ((it & 63u) == 0) {
      if (*abort) return false;
      if (globaltimer_ns() - t0 > limit_ns) {
        record_error(kErrTimeout, site);
        *abort = 1;
        return false;
      }
    }
  }
}

// Release store / acquire load of a shared-memory int (a flag or counter
// that one thread publishes to the rest of the CTA).
__device__ __forceinline__ void st_release_shared(int* p, int v) {
  asm volatile("st.release.cta.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(p)), "r"(v) : "memory");
}
__device__ __forceinline__ int ld_acquire_shared(const int* p) {
  int v;
  asm volatile("ld.acquire.cta.shared::cta.b32 %0, [%1];" : "=r"(v) : "r"(smem_u32(p)) : "memory");
  return v;
}

// ---------------------------------------------------------------- TMA
__device__ __forceinline__ void tma_prefetch_desc(const CUtensorMap* map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

__device__ __forceinline__ void tma_load_4d(void* dst, const CUtensorMap* map, uint64_t* bar,
                                            int c0, int c1, int c2, int c3) {
  asm volatile(
      "cp.async.bulk.tensor.4d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5, %6}], [%2];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(c0), "r"(c1), "r"(c2),
      "r"(c3)
      : "memory");
}

__device__ __forceinline__ void tma_load_5d(void* dst, const CUtensorMap* map, uint64_t* bar,
                                            int c0, int c1, int c2, int c3, int c4) {
  asm volatile(
      "cp.async.bulk.tensor.5d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5, %6, %7}], [%2];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(c0), "r"(c1), "r"(c2),
      "r"(c3), "r"(c4)
      : "memory");
}

__device__ __forceinline__ void tma_store_4d(const CUtensorMap* map, const void* src, int c0,
                                             int c1, int c2, int c3) {
  asm volatile(
      "cp.async.bulk.tensor.4d.global.shared::cta.tile.bulk_group [%0, {%2, %3, %4, %5}], [%1];" ::
          "l"(reinterpret_cast<uint64_t>(map)),
      "r"(smem_u32(src)), "r"(c0), "r"(c1), "r"(c2), "r"(c3)
      : "memory");
}

__device__ __forceinline__ void tma_store_commit() {
  asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}

// Waits until every committed bulk store has finished reading shared memory.
__device__ __forceinline__ void tma_store_wait_read_all() {
  asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
}

// Waits until every committed bulk store is complete (writes visible).
__device__ __forceinline__ void tma_store_wait_all() {
  asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
}

// Adds `bytes` (multiple of 16) fp32 values from shared memory into global
// memory with one bulk asynchronous reduction (both addresses 16-byte aligned).
__device__ __forceinline__ void bulk_reduce_add_f32(float* gdst, const void* ssrc, uint32_t bytes) {
  asm volatile(
      "cp.reduce.async.bulk.global.shared::cta.bulk_group.add.f32 [%0], [%1], %2;" ::"l"(gdst),
      "r"(smem_u32(ssrc)), "r"(bytes)
      : "memory");
}

// Named barrier for `count` threads (a multiple of 32) of the CTA.
__device__ __forceinline__ void named_bar_sync(int id, int count) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(count) : "memory");
}

// Orders this thread's generic-proxy shared-memory writes before later
// async-proxy accesses (TMA stores, tensor-core operand reads).
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// ---------------------------------------------------------------- tcgen05
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

// D[tmem] (+)= A[smem desc] * B[smem desc]^T, kind::f16 (bf16 in, fp32
// accumulate), issued by one elected lane of a converged warp.  The
// whole warp executes the call with warp-uniform operands: issued this way a
// thread sustains one MMA per ~43 cycles (M=128, N=48) against ~90 cycles
// when a single lane issues from a divergent branch, where the operands are
// not known to be uniform.
__device__ __forceinline__ void umma_ss_elect(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                              uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p, e;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "elect.sync _|e, 0xffffffff;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// STEPS MMAs D (+)= A_k B_k^T, k = 0..STEPS-1 (STEPS = 6 or 8), issued by
// one elected lane of a converged warp: A_k = tensor memory at a_tmem + 8k
// (16 bf16 columns per step), B_k = b_desc advanced by k * b_step
// (descriptor units of 16 bytes).  `first_acc` = 0 makes the first MMA
// overwrite D.  One election and no per-step descriptor arithmetic keep the
// issuing warp's instruction count low while it shares its scheduler with
// busy warps.
#define RIB_TS_STEP                                                   \
  "add.s32 a, a, 8;\n\t add.s64 b, b, %3;\n\t"                    \
  "@e tcgen05.mma.cta_group::1.kind::f16 [%0], [a], b, %4, t;\n\t"
template <int STEPS>
__device__ __forceinline__ void umma_ts_chain_elect(uint32_t d_tmem, uint32_t a_tmem,
                                                    uint64_t b_desc, uint32_t b_step,
                                                    uint32_t idesc, uint32_t first_acc) {
  static_assert(STEPS == 6 || STEPS == 8, "chains of 6 or 8 K-steps");
  if constexpr (STEPS == 8) {
    asm volatile(
        "{\n\t.reg .pred p, e, t;\n\t.reg .b64 b;\n\t.reg .b32 a;\n\t"
        "setp.ne.b32 p, %5, 0;\n\t"
        "setp.eq.b32 t, %4, %4;\n\t"
        "elect.sync _|e, 0xffffffff;\n\t"
        "mov.b32 a, %1;\n\t mov.b64 b, %2;\n\t"
        "@e tcgen05.mma.cta_group::1.kind::f16 [%0], [a], b, %4, p;\n\t"
        RIB_TS_STEP RIB_TS_STEP RIB_TS_STEP RIB_TS_STEP RIB_TS_STEP RIB_TS_STEP RIB_TS_STEP
        "}" ::"r"(d_tmem), "r"(a_tmem), "l"(b_desc), "l"(static_cast<uint64_t>(b_step)),
        "r"(idesc), "r"(first_acc)
        : "memory");
  } else {
    asm volatile(
        "{\n\t.reg .pred p, e, t;\n\t.reg .b64 b;\n\t.reg .b32 a;\n\t"
        "setp.ne.b32 p, %5, 0;\n\t"
        "setp.eq.b32 t, %4, %4;\n\t"
        "elect.sync _|e, 0xffffffff;\n\t"
        "mov.b32 a, %1;\n\t mov.b64 b, %2;\n\t"
        "@e tcgen05.mma.cta_group::1.kind::f16 [%0], [a], b, %4, p;\n\t"
        RIB_TS_STEP RIB_TS_STEP RIB_TS_STEP RIB_TS_STEP RIB_TS_STEP
        "}" ::"r"(d_tmem), "r"(a_tmem), "l"(b_desc), "l"(static_cast<uint64_t>(b_step)),
        "r"(idesc), "r"(first_acc)
        : "memory");
  }
}
#undef RIB_TS_STEP

__device__ __forceinline__ void umma_ts8_elect(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc,
                                               uint32_t b_step, uint32_t idesc,
                                               uint32_t first_acc) {
  umma_ts_chain_elect<8>(d_tmem, a_tmem, b_desc, b_step, idesc, first_acc);
}

// The same with A from shared memory: A_k = a_desc + k * a_step.
__device__ __forceinline__ void umma_ss8_elect(uint32_t d_tmem, uint64_t a_desc, uint32_t a_step,
                                               uint64_t b_desc, uint32_t b_step, uint32_t idesc,
                                               uint32_t first_acc) {
  asm volatile(
      "{\n\t.reg .pred p, e, t;\n\t.reg .b64 a, b, sa, sb;\n\t"
      "setp.ne.b32 p, %6, 0;\n\t"
      "setp.eq.b32 t, %5, %5;\n\t"
      "cvt.u64.u32 sa, %2;\n\t cvt.u64.u32 sb, %4;\n\t"
      "elect.sync _|e, 0xffffffff;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %3, %5, p;\n\t"
      "add.s64 a, %1, sa;\n\t add.s64 b, %3, sb;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], a, b, %5, t;\n\t"
      "add.s64 a, a, sa;\n\t add.s64 b, b, sb;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], a, b, %5, t;\n\t"
      "add.s64 a, a, sa;\n\t add.s64 b, b, sb;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], a, b, %5, t;\n\t"
      "add.s64 a, a, sa;\n\t add.s64 b, b, sb;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], a, b, %5, t;\n\t"
      "add.s64 a, a, sa;\n\t add.s64 b, b, sb;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], a, b, %5, t;\n\t"
      "add.s64 a, a, sa;\n\t add.s64 b, b, sb;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], a, b, %5, t;\n\t"
      "add.s64 a, a, sa;\n\t add.s64 b, b, sb;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], a, b, %5, t;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "r"(a_step), "l"(b_desc), "r"(b_step), "r"(idesc), "r"(first_acc)
      : "memory");
}

// The score chain of the augmented product, D = A0 B0^T + A1 B1^T + A2 B2^T
// (two content K-steps, one positional), issued by one elected lane.  With
// `three` = 0 only the first two MMAs are issued.
__device__ __forceinline__ void umma_ss3_elect(uint32_t d_tmem, uint64_t a0, uint64_t b0,
                                               uint64_t a1, uint64_t b1, uint64_t a2, uint64_t b2,
                                               uint32_t idesc, uint32_t three) {
  asm volatile(
      "{\n\t.reg .pred f, t, e, q;\n\t"
      "setp.ne.b32 f, %7, %7;\n\t"
      "setp.eq.b32 t, %7, %7;\n\t"
      "elect.sync _|e, 0xffffffff;\n\t"
      "setp.ne.and.b32 q, %8, 0, e;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %7, f;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], %3, %4, %7, t;\n\t"
      "@q tcgen05.mma.cta_group::1.kind::f16 [%0], %5, %6, %7, t;\n\t}" ::"r"(d_tmem),
      "l"(a0), "l"(b0), "l"(a1), "l"(b1), "l"(a2), "l"(b2), "r"(idesc), "r"(three)
      : "memory");
}

// tcgen05.commit from one elected lane of a converged warp: arrives once on
// `bar` when every MMA that lane issued with the *_elect calls above has
// completed.
__device__ __forceinline__ void umma_commit_elect(uint64_t* bar) {
  asm volatile(
      "{\n\t.reg .pred e;\n\t"
      "elect.sync _|e, 0xffffffff;\n\t"
      "@e tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];\n\t}" ::"r"(
          smem_u32(bar))
      : "memory");
}

// Register reallocation between warpgroups (all four warps of a warpgroup
// execute the same instruction).  The block's launch budget (threads x
// registers per thread at launch) must cover the sum of the new counts, or
// the increase would wait for registers that never come.
template <int N>
__device__ __forceinline__ void regs_inc() {
  asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(N));
}
template <int N>
__device__ __forceinline__ void regs_dec() {
  asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(N));
}

__device__ __forceinline__ void tmem_wait_ld() {
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_wait_st() {
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_st_x8(uint32_t taddr, const uint32_t (&r)[8]) {
  asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};"
               :: "r"(taddr), "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7])
               : "memory");
}

__device__ __forceinline__ void tmem_ld_x16(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
               : "r"(taddr));
}

__device__ __forceinline__ void tmem_st_x16(uint32_t taddr, const uint32_t (&r)[16]) {
  asm volatile("tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};"
               :: "r"(taddr), "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
               : "memory");
}

__device__ __forceinline__ void tmem_ld_x32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
               : "r"(taddr));
}

__device__ __forceinline__ void tmem_st_x32(uint32_t taddr, const uint32_t (&r)[32]) {
  asm volatile("tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};"
               :: "r"(taddr), "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]), "r"(r[16]), "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]), "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31])
               : "memory");
}


// Ties the registers of a finished tcgen05.ld to the preceding wait::ld so
// that no consumer is scheduled above it.
__device__ __forceinline__ void reg_fence_x8(uint32_t (&r)[8]) {
  asm volatile("" : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]), "+r"(r[6]), "+r"(r[7]));
}

// Ties the registers of a finished tcgen05.ld to the preceding wait::ld so
// that no consumer is scheduled above it.
__device__ __forceinline__ void reg_fence_x16(uint32_t (&r)[16]) {
  asm volatile("" : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]), "+r"(r[6]), "+r"(r[7]), "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]), "+r"(r[12]), "+r"(r[13]), "+r"(r[14]), "+r"(r[15]));
}

// Ties the registers of a finished tcgen05.ld to the preceding wait::ld so
// that no consumer is scheduled above it.
__device__ __forceinline__ void reg_fence_x32(uint32_t (&r)[32]) {
  asm volatile("" : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]), "+r"(r[6]), "+r"(r[7]), "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]), "+r"(r[12]), "+r"(r[13]), "+r"(r[14]), "+r"(r[15]), "+r"(r[16]), "+r"(r[17]), "+r"(r[18]), "+r"(r[19]), "+r"(r[20]), "+r"(r[21]), "+r"(r[22]), "+r"(r[23]), "+r"(r[24]), "+r"(r[25]), "+r"(r[26]), "+r"(r[27]), "+r"(r[28]), "+r"(r[29]), "+r"(r[30]), "+r"(r[31]));
}

// Shared-memory matrix descriptor of tcgen05.mma (sm_100 format):
// start address, leading / stride byte offsets (all >> 4), version 1 at
// bits 46-47, base offset 0, layout type at bits 61-63.
// kLayoutSW128B32: 128-byte rows whose 32-byte granules are XORed with the
// row index mod 4 (a 4-row atom); the layout an MN-major tf32 operand needs.
enum : uint32_t {
  kLayoutNone = 0, kLayoutSW128B32 = 1, kLayoutSW128 = 2, kLayoutSW64 = 4, kLayoutSW32 = 6
};

__device__ __forceinline__ uint64_t make_sdesc(uint32_t saddr, uint32_t lbo_bytes,
                                               uint32_t sbo_bytes, uint32_t layout) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((saddr >> 4) & 0x3FFFu);
  d |= static_cast<uint64_t>((lbo_bytes >> 4) & 0x3FFFu) << 16;
  d |= static_cast<uint64_t>((sbo_bytes >> 4) & 0x3FFFu) << 32;
  d |= static_cast<uint64_t>(1) << 46;
  d |= static_cast<uint64_t>(layout & 7u) << 61;
  return d;
}

// Instruction descriptor of tcgen05.mma kind::f16 with bf16 A/B and fp32 D.
// a_mn / b_mn select MN-major (transposed) operands.
__host__ __device__ constexpr uint32_t make_idesc_bf16(int M, int N, bool a_mn, bool b_mn) {
  return (1u << 4)                                 // D format: f32
         | (1u << 7)                               // A format: bf16
         | (1u << 10)                              // B format: bf16
         | ((a_mn ? 1u : 0u) << 15) | ((b_mn ? 1u : 0u) << 16) |
         (static_cast<uint32_t>(N >> 3) << 17) | (static_cast<uint32_t>(M >> 4) << 24);
}

// Instruction descriptor of tcgen05.mma kind::tf32: fp32 operands in shared
// or tensor memory read as tf32 (10 explicit mantissa bits), fp32 D.
__host__ __device__ constexpr uint32_t make_idesc_tf32(int M, int N, bool a_mn, bool b_mn) {
  return (1u << 4)                                 // D format: f32
         | (2u << 7)                               // A format: tf32
         | (2u << 10)                              // B format: tf32
         | ((a_mn ? 1u : 0u) << 15) | ((b_mn ? 1u : 0u) << 16) |
         (static_cast<uint32_t>(N >> 3) << 17) | (static_cast<uint32_t>(M >> 4) << 24);
}

// D[tmem] (+)= A[smem desc] * B[smem desc]^T, kind::tf32 (K = 8 per MMA),
// issued by one elected lane of a converged warp.
__device__ __forceinline__ void umma_tf32_ss_elect(uint32_t d_tmem, uint64_t a_desc,
                                                   uint64_t b_desc, uint32_t idesc,
                                                   uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p, e;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "elect.sync _|e, 0xffffffff;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::tf32 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// D[tmem] (+)= A[tmem] * B[smem desc]^T, kind::tf32 (A: 8 fp32 columns per MMA),
// issued by one elected lane of a converged warp.
__device__ __forceinline__ void umma_tf32_ts_elect(uint32_t d_tmem, uint32_t a_tmem,
                                                   uint64_t b_desc, uint32_t idesc,
                                                   uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p, e;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "elect.sync _|e, 0xffffffff;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::tf32 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// fp32 -> tf32 (round to nearest, ties away from zero), kept in an fp32
// register with the 13 low mantissa bits zero.
__device__ __forceinline__ float round_tf32(float x) {
  uint32_t r;
  asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(r) : "f"(x));
  return __uint_as_float(r);
}

__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

// One 32-byte global store per thread (a whole sector); ptr 32-byte aligned.
__device__ __forceinline__ void st_global_v8(void* ptr, uint32_t a0, uint32_t a1, uint32_t a2,
                                             uint32_t a3, uint32_t a4, uint32_t a5, uint32_t a6,
                                             uint32_t a7) {
  asm volatile("st.global.v8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"l"(ptr), "r"(a0),
               "r"(a1), "r"(a2), "r"(a3), "r"(a4), "r"(a5), "r"(a6), "r"(a7)
               : "memory");
}

// One thread's 64-byte row (32 bf16 channels of a token, or 16 fp32
// values): with v8 (a 32-byte aligned row) two whole 32-byte sectors, else
// four 16-byte stores.  When a warp's 32 rows lie far apart, a 16-byte
// store per lane half-fills 32 sectors at once.
__device__ __forceinline__ void store_row64(void* dst, const uint32_t (&w)[16], bool v8) {
  if (v8) {
    st_global_v8(dst, w[0], w[1], w[2], w[3], w[4], w[5], w[6], w[7]);
    st_global_v8(static_cast<uint8_t*>(dst) + 32, w[8], w[9], w[10], w[11], w[12], w[13], w[14],
                 w[15]);
  } else {
    uint4* d = static_cast<uint4*>(dst);
#pragma unroll
    for (int q = 0; q < 4; ++q) d[q] = make_uint4(w[4 * q], w[4 * q + 1], w[4 * q + 2], w[4 * q + 3]);
  }
}

// ---------------------------------------------------------------- packed fp32
// Two fp32 values in one 64-bit register pair (low = first).
__device__ __forceinline__ uint64_t pk2(float lo, float hi) {
  return static_cast<uint64_t>(__float_as_uint(lo)) |
         (static_cast<uint64_t>(__float_as_uint(hi)) << 32);
}
__device__ __forceinline__ float lo2(uint64_t v) { return __uint_as_float(static_cast<uint32_t>(v)); }
__device__ __forceinline__ float hi2(uint64_t v) {
  return __uint_as_float(static_cast<uint32_t>(v >> 32));
}
__device__ __forceinline__ uint64_t ffma2(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}
__device__ __forceinline__ uint64_t fadd2(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ uint64_t fmul2(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

// 2^x for two packed x <= 8 on the FMA pipe (no MUFU).
// Cody-Waite reduction: n = round(x) via the 1.5*2^23 rounding constant,
// f = x - n in [-1/2, 1/2] (exact); 2^f from the degree-3 polynomial that
// minimises the maximum relative error on [-1/2, 1/2] (Remez exchange,
// csrc/fit_exp2_poly.py: 7.5e-5); 2^n is added to the exponent field.
// x is clamped at -125 so the exponent stays normal (2^-125 is negligible
// wherever this feeds a bf16 softmax numerator).
constexpr float kExp2C0 = 0.9999280571937561f;
constexpr float kExp2C1 = 0.6932609677314758f;
constexpr float kExp2C2 = 0.2426111251115799f;
constexpr float kExp2C3 = 0.0551716685295105f;
constexpr float kRoundMagic = 12582912.0f;  // 1.5 * 2^23

__device__ __forceinline__ uint64_t exp2_fma2(uint64_t x2) {
  const float xl = fmaxf(lo2(x2), -125.f), xh = fmaxf(hi2(x2), -125.f);
  const uint64_t xc = pk2(xl, xh);
  const uint64_t t = fadd2(xc, pk2(kRoundMagic, kRoundMagic));
  const uint64_t nf = fadd2(t, pk2(-kRoundMagic, -kRoundMagic));
  const uint64_t f = ffma2(nf, pk2(-1.f, -1.f), xc);
  uint64_t p = ffma2(pk2(kExp2C3, kExp2C3), f, pk2(kExp2C2, kExp2C2));
  p = ffma2(p, f, pk2(kExp2C1, kExp2C1));
  p = ffma2(p, f, pk2(kExp2C0, kExp2C0));
  const uint32_t rl = static_cast<uint32_t>(p) + (static_cast<uint32_t>(t) << 23);
  const uint32_t rh = static_cast<uint32_t>(p >> 32) + (static_cast<uint32_t>(t >> 32) << 23);
  return static_cast<uint64_t>(rl) | (static_cast<uint64_t>(rh) << 32);
}

template <typename T>
__device__ __forceinline__ T* align1024(uint8_t* p) {
  const uint32_t a = smem_u32(p);
  return reinterpret_cast<T*>(p + ((1024u - (a & 1023u)) & 1023u));
}

// Tests two barriers at once (both phases complete?): the two tests are in
// flight together, so a warp that finds both ready pays one round trip.
__device__ __forceinline__ bool mbar_try_wait2(uint64_t* bar0, uint32_t parity0, uint64_t* bar1,
                                               uint32_t parity1) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "mbarrier.try_wait.parity.acquire.cta.shared::cta.b64 p, [%1], %2;\n\t"
      "mbarrier.try_wait.parity.acquire.cta.shared::cta.b64 q, [%3], %4;\n\t"
      "and.pred p, p, q;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar0)), "r"(parity0), "r"(smem_u32(bar1)), "r"(parity1)
      : "memory");
  return ok != 0;
}

// Warp-uniform bounded wait: the warp proceeds only if every lane saw the
// phase complete, so no warp-collective tcgen05 op runs on a partial warp.
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, volatile int* abort,
                                          uint64_t limit, int site, uint32_t sleep_ns = 0) {
  const bool ok = mbar_wait(bar, parity, abort, limit, site, sleep_ns);
  return __all_sync(0xffffffffu, ok);
}

// warp_wait on two barriers; when both phases are already complete (the
// common case where it is used) the warp pays one test instead of two.
__device__ __forceinline__ bool warp_wait2(uint64_t* bar0, uint32_t parity0, uint64_t* bar1,
                                           uint32_t parity1, volatile int* abort, uint64_t limit,
                                           int site) {
  const bool ok = mbar_try_wait2(bar0, parity0, bar1, parity1) ||
                  (mbar_wait(bar0, parity0, abort, limit, site) &&
                   mbar_wait(bar1, parity1, abort, limit, site));
  return __all_sync(0xffffffffu, ok);
}

}  // namespace rib

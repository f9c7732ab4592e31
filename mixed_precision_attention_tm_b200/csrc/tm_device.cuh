// tm_device.cuh -- sm_100a device primitives used by the libtm kernels:
// mbarriers with bounded waits, TMA tile loads, tcgen05 (TMEM allocation,
// MMA issue/commit, TMEM loads/stores) and the device error word.
//
// Every wait in this library is bounded: after TM_WAIT_LIMIT_NS of global
// time a wait gives up, records TM_DEVERR_TIMEOUT in the device error word
// and returns false, and the caller unwinds without touching further
// pipeline state.
#pragma once

#include <cuda.h>
#include <cuda_fp16.h>
#include <stdint.h>

#define TM_DEVERR_TIMEOUT 1u
#define TM_DEVERR_SEQLEN 2u

#ifndef TM_WAIT_LIMIT_NS
#define TM_WAIT_LIMIT_NS 2000000000ull   // 2 s
#endif

// Optional event tracing (compiled out unless TM_TRACE is defined): one
// traced CTA records (event id, SM clock) pairs per role into a device buffer
// that tm_debug_trace_read copies out.  Used to read pipeline timelines.
#ifdef TM_TRACE
#define TM_TRACE_ROLES 4
#define TM_TRACE_EVENTS 4096
static __device__ unsigned long long g_tm_trace[TM_TRACE_ROLES][TM_TRACE_EVENTS];
static __device__ unsigned int g_tm_trace_block;
#define TM_TRACE_DECL unsigned int tm_trace_n = 0;
#define TM_TRACE_EV(role, ev)                                                                   \
  do {                                                                                          \
    if (blockIdx.x == g_tm_trace_block && tm_trace_n < TM_TRACE_EVENTS) {                        \
      long long tm_c;                                                                           \
      asm volatile("mov.u64 %0, %%clock64;" : "=l"(tm_c));                                     \
      g_tm_trace[role][tm_trace_n++] = (static_cast<unsigned long long>(ev) << 56) |             \
                                       (static_cast<unsigned long long>(tm_c) & 0xFFFFFFFFFFFFFFull); \
    }                                                                                           \
  } while (0)
#else
#define TM_TRACE_DECL
#define TM_TRACE_EV(role, ev) \
  do {                        \
  } while (0)
#endif

namespace tmk {

// Defined in tm_api.cu (relocatable device code is not used, so each
// translation unit that needs the word receives its address as a kernel
// argument instead of naming the symbol).
struct DevErr {
  unsigned int* word;
};

__device__ __forceinline__ void dev_error(const DevErr& e, unsigned int bits) {
  if (e.word) atomicOr(e.word, bits);
}

__device__ __forceinline__ uint64_t global_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// ---------------------------------------------------------------- mbarrier
__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count));
}

__device__ __forceinline__ void fence_barrier_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void fence_async_shared() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
               : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.b32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}

// Waits until the phase with the given parity has completed.  Gives up (and
// reports) after limit_ns of global time, or early when *abort becomes
// non-zero.
#if defined(TM_TRACE) || defined(TM_TIMEOUT_INFO)
// First timed-out wait of a launch (TM_TRACE or TM_TIMEOUT_INFO builds):
// block, barrier offset within the block's shared window, parity, thread.
static __device__ unsigned int g_tm_timeout_info[5];
#endif
__device__ __forceinline__ bool mbar_wait_limit(uint32_t bar, uint32_t parity, const DevErr& err,
                                                volatile int* abort, uint64_t limit_ns) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = global_ns();
  while (true) {
    if (mbar_try_wait(bar, parity)) return true;
    if (*abort) return false;
    if (global_ns() - t0 > limit_ns) {
#if defined(TM_TRACE) || defined(TM_TIMEOUT_INFO)
      if (atomicCAS(&g_tm_timeout_info[0], 0u, 1u) == 0u) {
        g_tm_timeout_info[1] = blockIdx.x;
        g_tm_timeout_info[2] = bar;
        g_tm_timeout_info[3] = parity;
        g_tm_timeout_info[4] = threadIdx.x;
      }
#endif
      dev_error(err, TM_DEVERR_TIMEOUT);
      *abort = 1;
      return false;
    }
  }
}

__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, const DevErr& err,
                                          volatile int* abort) {
  return mbar_wait_limit(bar, parity, err, abort, TM_WAIT_LIMIT_NS);
}

__device__ __forceinline__ bool mbar_test_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.b32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}

// Spinning wait for a single latency-critical thread (the MMA issuer): polls
// with the non-suspending test_wait; same time limit and abort rules as
// mbar_wait.
__device__ __forceinline__ bool mbar_spin(uint32_t bar, uint32_t parity, const DevErr& err,
                                          volatile int* abort) {
  for (int i = 0; i < 256; ++i)
    if (mbar_test_wait(bar, parity)) return true;
  const uint64_t t0 = global_ns();
  while (true) {
    for (int i = 0; i < 256; ++i)
      if (mbar_test_wait(bar, parity)) return true;
    if (*abort) return false;
    if (global_ns() - t0 > TM_WAIT_LIMIT_NS) {
      dev_error(err, TM_DEVERR_TIMEOUT);
      *abort = 1;
      return false;
    }
  }
}

// True in exactly one lane of a converged warp (elect.sync: the same lane
// every time for a full mask, so the tcgen05 operations it issues and their
// commits come from one thread).
__device__ __forceinline__ bool elect_one() {
  uint32_t pred;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "elect.sync _|p, 0xffffffff;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(pred));
  return pred != 0;
}

// Warp-cooperative wait: lane 0 polls, the other lanes wait at __syncwarp and
// then confirm with one try_wait each (so every lane observes the phase with
// acquire semantics).  Keeps 31 of 32 threads off the shared-memory barrier
// while a warp waits.  Must be called by all 32 lanes of a converged warp.
__device__ __forceinline__ bool mbar_wait_warp(uint32_t bar, uint32_t parity, const DevErr& err,
                                               volatile int* abort) {
  bool ok = true;
  if ((threadIdx.x & 31) == 0) ok = mbar_wait(bar, parity, err, abort);
  ok = __shfl_sync(0xffffffffu, ok, 0);
  if (ok && (threadIdx.x & 31) != 0) {
    while (!mbar_try_wait(bar, parity)) {
    }
  }
  __syncwarp();
  return ok;
}

// ---------------------------------------------------------------- TMA
__device__ __forceinline__ void tma_load_3d(uint32_t dst, const CUtensorMap* map, uint32_t bar,
                                            int32_t c0, int32_t c1, int32_t c2) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5}], [%2];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(c0), "r"(c1), "r"(c2)
      : "memory");
}

// Same load with an L2 cache policy (from createpolicy).
__device__ __forceinline__ void tma_load_3d_hint(uint32_t dst, const CUtensorMap* map, uint32_t bar,
                                                 int32_t c0, int32_t c1, int32_t c2, uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes.L2::cache_hint"
      " [%0], [%1, {%3, %4, %5}], [%2], %6;" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(c0), "r"(c1), "r"(c2), "l"(policy)
      : "memory");
}

// Brings a tensor tile into L2 ahead of its shared-memory load (no completion).
__device__ __forceinline__ void tma_prefetch_l2_3d(const CUtensorMap* map, int32_t c0, int32_t c1, int32_t c2) {
  asm volatile("cp.async.bulk.prefetch.tensor.3d.L2.global.tile [%0, {%1, %2, %3}];" ::"l"(
                   reinterpret_cast<uint64_t>(map)),
               "r"(c0), "r"(c1), "r"(c2)
               : "memory");
}

__device__ __forceinline__ uint64_t l2_policy_evict_last() {
  uint64_t pol;
  asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(pol));
  return pol;
}
__device__ __forceinline__ uint64_t l2_policy_evict_first() {
  uint64_t pol;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
  return pol;
}

__device__ __forceinline__ void prefetch_tmap(const CUtensorMap* map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// ---------------------------------------------------------------- tcgen05
__device__ __forceinline__ void tmem_alloc(uint32_t dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst_smem),
               "r"(ncols));
}
__device__ __forceinline__ void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols));
}
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
// Arrives once on `bar` when every tcgen05 operation issued so far by this
// thread has completed.
__device__ __forceinline__ void tc_commit(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                   bar)
               : "memory");
}

// D(tmem) (+)= A(smem desc) * B(smem desc), kind::f16 (fp16 in, fp32 acc)
__device__ __forceinline__ void mma_f16_ss(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                           uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate));
}
// D(tmem) (+)= A(tmem) * B(smem desc), kind::f16
__device__ __forceinline__ void mma_f16_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc,
                                           uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate));
}
// D(tmem, s32) (+)= A(smem desc, s8) * B(smem desc, s8), kind::i8
__device__ __forceinline__ void mma_i8_ss(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                          uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::i8 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate));
}

// Groups of tcgen05.mma issued from one asm statement, with every
// descriptor formed before the first MMA.  Measured on B200: an MMA issued
// back to back after another from the same thread starts as that one
// finishes (M128 N128 K16 f16 or K32 i8: 64 SM cycles each), but each
// instruction the issuing thread executes between two MMAs delays the second
// one (descriptor arithmetic and a branch between MMAs raised the time per
// MMA to 70-107 cycles).  acc_first is the accumulate flag of the group's
// first MMA; the others accumulate.
template <int N>
__device__ __forceinline__ void mma_f16_ss_n(uint32_t d, const uint64_t* a, const uint64_t* b, uint32_t idesc,
                                             uint32_t acc_first);
template <int N>
__device__ __forceinline__ void mma_i8_ss_n(uint32_t d, const uint64_t* a, const uint64_t* b, uint32_t idesc,
                                            uint32_t acc_first);
template <int N>
__device__ __forceinline__ void mma_f8_ss_n(uint32_t d, const uint64_t* a, const uint64_t* b, uint32_t idesc,
                                            uint32_t acc_first);
// A from TMEM (a[i]: TMEM addresses), B from shared memory, kind::f16
template <int N>
__device__ __forceinline__ void mma_f16_ts_n(uint32_t d, const uint32_t* a, const uint64_t* b, uint32_t idesc,
                                             uint32_t acc_first);
template <>
__device__ __forceinline__ void mma_f16_ss_n<4>(uint32_t d, const uint64_t* a, const uint64_t* b, uint32_t idesc,
                                          uint32_t acc_first) {
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.b32 p, %10, 0;\n\t"
      "setp.ne.b32 q, %11, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %5, %9, p;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %2, %6, %9, q;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %3, %7, %9, q;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %4, %8, %9, q;\n\t}"
      ::"r"(d), "l"(a[0]), "l"(a[1]), "l"(a[2]), "l"(a[3]), "l"(b[0]), "l"(b[1]), "l"(b[2]), "l"(b[3]), "r"(idesc), "r"(acc_first), "r"(1u));
}
template <>
__device__ __forceinline__ void mma_f16_ss_n<8>(uint32_t d, const uint64_t* a, const uint64_t* b, uint32_t idesc,
                                          uint32_t acc_first) {
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.b32 p, %18, 0;\n\t"
      "setp.ne.b32 q, %19, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %9, %17, p;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %2, %10, %17, q;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %3, %11, %17, q;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %4, %12, %17, q;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %5, %13, %17, q;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %6, %14, %17, q;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %7, %15, %17, q;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %8, %16, %17, q;\n\t}"
      ::"r"(d), "l"(a[0]), "l"(a[1]), "l"(a[2]), "l"(a[3]), "l"(a[4]), "l"(a[5]), "l"(a[6]), "l"(a[7]), "l"(b[0]), "l"(b[1]), "l"(b[2]), "l"(b[3]), "l"(b[4]), "l"(b[5]), "l"(b[6]), "l"(b[7]), "r"(idesc), "r"(acc_first), "r"(1u));
}
template <>
__device__ __forceinline__ void mma_i8_ss_n<2>(uint32_t d, const uint64_t* a, const uint64_t* b, uint32_t idesc,
                                          uint32_t acc_first) {
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.b32 p, %6, 0;\n\t"
      "setp.ne.b32 q, %7, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::i8 [%0], %1, %3, %5, p;\n\t"
      "tcgen05.mma.cta_group::1.kind::i8 [%0], %2, %4, %5, q;\n\t}"
      ::"r"(d), "l"(a[0]), "l"(a[1]), "l"(b[0]), "l"(b[1]), "r"(idesc), "r"(acc_first), "r"(1u));
}
template <>
__device__ __forceinline__ void mma_i8_ss_n<4>(uint32_t d, const uint64_t* a, const uint64_t* b, uint32_t idesc,
                                          uint32_t acc_first) {
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.b32 p, %10, 0;\n\t"
      "setp.ne.b32 q, %11, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::i8 [%0], %1, %5, %9, p;\n\t"
      "tcgen05.mma.cta_group::1.kind::i8 [%0], %2, %6, %9, q;\n\t"
      "tcgen05.mma.cta_group::1.kind::i8 [%0], %3, %7, %9, q;\n\t"
      "tcgen05.mma.cta_group::1.kind::i8 [%0], %4, %8, %9, q;\n\t}"
      ::"r"(d), "l"(a[0]), "l"(a[1]), "l"(a[2]), "l"(a[3]), "l"(b[0]), "l"(b[1]), "l"(b[2]), "l"(b[3]), "r"(idesc), "r"(acc_first), "r"(1u));
}
// kind::f8f6f4 (E4M3 codes per the instruction descriptor), K = 32 per MMA
template <>
__device__ __forceinline__ void mma_f8_ss_n<4>(uint32_t d, const uint64_t* a, const uint64_t* b, uint32_t idesc,
                                         uint32_t acc_first) {
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.b32 p, %10, 0;\n\t"
      "setp.ne.b32 q, %11, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %1, %5, %9, p;\n\t"
      "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %2, %6, %9, q;\n\t"
      "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %3, %7, %9, q;\n\t"
      "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %4, %8, %9, q;\n\t}"
      ::"r"(d), "l"(a[0]), "l"(a[1]), "l"(a[2]), "l"(a[3]), "l"(b[0]), "l"(b[1]), "l"(b[2]), "l"(b[3]), "r"(idesc), "r"(acc_first), "r"(1u));
}
template <>
__device__ __forceinline__ void mma_f16_ts_n<4>(uint32_t d, const uint32_t* a, const uint64_t* b, uint32_t idesc,
                                          uint32_t acc_first) {
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.b32 p, %10, 0;\n\t"
      "setp.ne.b32 q, %11, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %5, %9, p;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%2], %6, %9, q;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%3], %7, %9, q;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%4], %8, %9, q;\n\t}"
      ::"r"(d), "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "l"(b[0]), "l"(b[1]), "l"(b[2]), "l"(b[3]), "r"(idesc), "r"(acc_first), "r"(1u));
}
template <>
__device__ __forceinline__ void mma_f16_ts_n<8>(uint32_t d, const uint32_t* a, const uint64_t* b, uint32_t idesc,
                                          uint32_t acc_first) {
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.b32 p, %18, 0;\n\t"
      "setp.ne.b32 q, %19, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %9, %17, p;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%2], %10, %17, q;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%3], %11, %17, q;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%4], %12, %17, q;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%5], %13, %17, q;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%6], %14, %17, q;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%7], %15, %17, q;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%8], %16, %17, q;\n\t}"
      ::"r"(d), "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(a[4]), "r"(a[5]), "r"(a[6]), "r"(a[7]), "l"(b[0]), "l"(b[1]), "l"(b[2]), "l"(b[3]), "l"(b[4]), "l"(b[5]), "l"(b[6]), "l"(b[7]), "r"(idesc), "r"(acc_first), "r"(1u));
}

// INT8 score tiles leave the tensor core as exact fp32 numbers, so that the
// softmax treats them like FP16 score tiles (only the scale differs) and
// needs no int32 -> fp32 conversion.  The accumulator starts at a seed: one
// kind::f16 MMA on constant operands writes the fp32 value 1.5 * 2^23 (bit
// pattern 0x4B400000); the kind::i8 MMAs add their s32 dot product acc to that
// bit pattern, which then reads as the fp32 number 1.5 * 2^23 + acc exactly
// (|acc| < 2^22: at most d * 127^2 = 2064512 here); a last kind::f16 MMA with
// accumulate adds -1.5 * 2^23 in fp32, leaving acc exactly (every operand,
// product and sum involved is an exactly representable fp32 value).
constexpr float kAccSeed = 12582912.0f;
// The constant operands: three no-swizzle core matrices (8 rows of 16
// bytes), each row one fp16 value v followed by seven zeros.  Read with zero
// leading and stride offsets, every 8 x 8 core matrix of a 128 x 16 operand
// is the block, so the operand holds v at k = 0 and 8 and 0 elsewhere:
// A = 2048 and B = +-3072 give K = 16 products 2 * 2048 * (+-3072) =
// +-1.5 * 2^23 in every element.
constexpr uint32_t kSeedRowA = 0x6800u;    // fp16 2048
constexpr uint32_t kSeedRowB = 0x6A00u;    // fp16 3072
constexpr uint32_t kSeedRowBn = 0xEA00u;   // fp16 -3072
constexpr int kSeedBytes = 384;            // A block, B block, -B block
// Written by the 32 lanes of one warp; the caller makes them visible to the
// tensor core (fence.proxy.async) before the CTA barrier.
__device__ __forceinline__ void seed_blocks_init(uint32_t* blk, int lane) {
#pragma unroll
  for (int i = lane; i < kSeedBytes / 4; i += 32) {
    const int word_in_row = i & 3, block = i >> 5;
    const uint32_t v = block == 0 ? kSeedRowA : (block == 1 ? kSeedRowB : kSeedRowBn);
    blk[i] = word_in_row == 0 ? v : 0u;
  }
}
// Descriptor of a seed block: no swizzle, zero leading and stride offsets.
__device__ __forceinline__ uint64_t seed_desc(uint32_t saddr) {
  return (static_cast<uint64_t>((saddr >> 4) & 0x3FFFu)) | (static_cast<uint64_t>(1) << 46);
}
// The INT8 QK^T of one score tile with an fp32 result: the seed MMA, N
// kind::i8 MMAs accumulating onto it and the unseed MMA, from one asm
// statement with every descriptor formed beforehand.  sd[0..2]: descriptors
// of the A, B and -B blocks.
template <int N>
__device__ __forceinline__ void mma_i8_exact_n(uint32_t d, const uint64_t* sd, uint32_t idesc_seed, const uint64_t* a,
                                               const uint64_t* b, uint32_t idesc);
template <>
__device__ __forceinline__ void mma_i8_exact_n<2>(uint32_t d, const uint64_t* sd, uint32_t idesc_seed,
                                                  const uint64_t* a, const uint64_t* b, uint32_t idesc) {
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.b32 p, %10, 0;\n\t"
      "setp.ne.b32 q, %11, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %4, p;\n\t"
      "tcgen05.mma.cta_group::1.kind::i8 [%0], %5, %7, %9, q;\n\t"
      "tcgen05.mma.cta_group::1.kind::i8 [%0], %6, %8, %9, q;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %3, %4, q;\n\t}"
      ::"r"(d), "l"(sd[0]), "l"(sd[1]), "l"(sd[2]), "r"(idesc_seed), "l"(a[0]), "l"(a[1]), "l"(b[0]), "l"(b[1]),
      "r"(idesc), "r"(0u), "r"(1u));
}
template <>
__device__ __forceinline__ void mma_i8_exact_n<4>(uint32_t d, const uint64_t* sd, uint32_t idesc_seed,
                                                  const uint64_t* a, const uint64_t* b, uint32_t idesc) {
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.b32 p, %14, 0;\n\t"
      "setp.ne.b32 q, %15, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %4, p;\n\t"
      "tcgen05.mma.cta_group::1.kind::i8 [%0], %5, %9, %13, q;\n\t"
      "tcgen05.mma.cta_group::1.kind::i8 [%0], %6, %10, %13, q;\n\t"
      "tcgen05.mma.cta_group::1.kind::i8 [%0], %7, %11, %13, q;\n\t"
      "tcgen05.mma.cta_group::1.kind::i8 [%0], %8, %12, %13, q;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %3, %4, q;\n\t}"
      ::"r"(d), "l"(sd[0]), "l"(sd[1]), "l"(sd[2]), "r"(idesc_seed), "l"(a[0]), "l"(a[1]), "l"(a[2]), "l"(a[3]),
      "l"(b[0]), "l"(b[1]), "l"(b[2]), "l"(b[3]), "r"(idesc), "r"(0u), "r"(1u));
}

// 32 lanes x 32 consecutive 32-bit columns: thread t of the warp receives
// columns [col, col+32) of TMEM lane (lane base of taddr) + t.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]),
        "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]),
        "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
}
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
      "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
      "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]),
      "r"(r[15]), "r"(r[16]), "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]),
      "r"(r[22]), "r"(r[23]), "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]),
      "r"(r[29]), "r"(r[30]), "r"(r[31])
      : "memory");
}
// Same as tmem_ld32 / tmem_st32 on 32 consecutive elements of a register
// array (the offset must be a compile-time constant after unrolling).
__device__ __forceinline__ void tmem_ld32p(uint32_t taddr, uint32_t* r) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]),
        "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]),
        "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
}
__device__ __forceinline__ void tmem_st32p(uint32_t taddr, const uint32_t* r) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
      "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
      "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]),
      "r"(r[15]), "r"(r[16]), "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]),
      "r"(r[22]), "r"(r[23]), "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]),
      "r"(r[29]), "r"(r[30]), "r"(r[31])
      : "memory");
}
// Marks 32 registers as (re)defined here, so that the compiler cannot move
// their uses above this point (used after tcgen05.wait::ld for registers
// filled by an asynchronous tcgen05.ld issued earlier).
__device__ __forceinline__ void reg_fence32(uint32_t* r) {
  asm volatile(""
               : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]), "+r"(r[6]),
                 "+r"(r[7]), "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]), "+r"(r[12]), "+r"(r[13]),
                 "+r"(r[14]), "+r"(r[15]), "+r"(r[16]), "+r"(r[17]), "+r"(r[18]), "+r"(r[19]),
                 "+r"(r[20]), "+r"(r[21]), "+r"(r[22]), "+r"(r[23]), "+r"(r[24]), "+r"(r[25]),
                 "+r"(r[26]), "+r"(r[27]), "+r"(r[28]), "+r"(r[29]), "+r"(r[30]), "+r"(r[31]));
}
__device__ __forceinline__ void tmem_wait_ld() {
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}
// Waits for this thread's TMEM loads into r[0, N) and then pins those
// registers: the empty asm statement "modifies" them after the wait, so the
// compiler cannot schedule a use of a loaded value ahead of the wait.
template <int N>
__device__ __forceinline__ void tmem_wait_ld_regs(uint32_t* r) {
  tmem_wait_ld();
#pragma unroll
  for (int c = 0; c < N / 32; ++c) reg_fence32(r + c * 32);
}
__device__ __forceinline__ void tmem_wait_st() {
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

// ---------------------------------------------------------------- descriptors
// Shared-memory matrix descriptor of tcgen05.mma (sm_100 format):
//  [0,14) start address >> 4, [16,30) leading-dimension byte offset >> 4,
//  [32,46) stride-dimension byte offset >> 4, [46,48) version = 1,
//  [49,52) base offset = 0 (1024-byte aligned atoms), [61,64) layout:
//  2 = 128-byte swizzle, 4 = 64-byte swizzle.
enum : uint32_t { kSwizzle128 = 2, kSwizzle64 = 4 };

__device__ __forceinline__ uint64_t smem_desc(uint32_t saddr, uint32_t lbo, uint32_t sbo,
                                              uint32_t layout) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((saddr >> 4) & 0x3FFFu);
  d |= static_cast<uint64_t>((lbo >> 4) & 0x3FFFu) << 16;
  d |= static_cast<uint64_t>((sbo >> 4) & 0x3FFFu) << 32;
  d |= static_cast<uint64_t>(1) << 46;
  d |= static_cast<uint64_t>(layout) << 61;
  return d;
}

// Instruction descriptor of tcgen05.mma kind::f16 / kind::i8:
//  [4,6) D format (1 = f32, 2 = s32), [7,10) A format, [10,13) B format
//  (f16: 0 = f16; i8: 1 = signed), bit 15 A major, bit 16 B major
//  (0 = K-major, 1 = MN-major), [17,23) N >> 3, [24,29) M >> 4.
__host__ __device__ constexpr uint32_t idesc_f16(int M, int N, bool b_mn_major) {
  return (1u << 4) | (0u << 7) | (0u << 10) | (0u << 15) | ((b_mn_major ? 1u : 0u) << 16) |
         (static_cast<uint32_t>(N >> 3) << 17) | (static_cast<uint32_t>(M >> 4) << 24);
}
__host__ __device__ constexpr uint32_t idesc_i8(int M, int N) {
  return (2u << 4) | (1u << 7) | (1u << 10) | (static_cast<uint32_t>(N >> 3) << 17) |
         (static_cast<uint32_t>(M >> 4) << 24);
}
// kind::f8f6f4 with E4M3 A and B (format code 0), f32 D, both K-major.
__host__ __device__ constexpr uint32_t idesc_f8_e4m3(int M, int N) {
  return (1u << 4) | (0u << 7) | (0u << 10) | (static_cast<uint32_t>(N >> 3) << 17) |
         (static_cast<uint32_t>(M >> 4) << 24);
}

// ---------------------------------------------------------------- misc
// Lazy online-softmax rescaling: a row's running max m is raised (and O and
// the row sum rescaled) only when a score exceeds it by more than this many
// powers of two.  P = 2^(s - m) then stays below 2^15, inside fp16's range
// (max 65504) at full relative precision, and the fp32 row sum and O
// accumulator are unaffected; a larger margin means fewer rescales.
constexpr float kLazyRescaleLog2 = 15.0f;

__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Warpgroup register reallocation (all four warps of the warpgroup execute it).
template <uint32_t N>
__device__ __forceinline__ void regs_inc() {
  asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(N));
}
template <uint32_t N>
__device__ __forceinline__ void regs_dec() {
  asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(N));
}

// Packed fp32 pairs (sm_100 f32x2 arithmetic: two lanes per instruction).
__device__ __forceinline__ uint64_t f2pack(float lo, float hi) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
  return r;
}
__device__ __forceinline__ void f2unpack(uint64_t v, float& lo, float& hi) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}
__device__ __forceinline__ uint64_t f2fma(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}
__device__ __forceinline__ uint64_t f2add(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ uint64_t f2mul(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}

// 2^y for y <= kLazyRescaleLog2 on the FMA pipe, two lanes at a time (f32x2).  y = n + f
// with n = rne(y) obtained by adding 1.5 * 2^23 (whose float ulp is 1), f in
// [-1/2, 1/2]; 2^f by a degree-3 minimax polynomial (relative error <= 7.5e-5
// on that interval, coefficients from a Remez fit); 2^n enters the exponent
// field with one integer shift-add per lane.  y is clamped at -125 so masked
// (-inf) scores give a normal ~2^-125, which rounds to 0 in fp16.
__device__ __forceinline__ void exp2_poly2(uint64_t y2, float& p0, float& p1) {
  float y0, y1;
  f2unpack(y2, y0, y1);
  y2 = f2pack(fmaxf(y0, -125.0f), fmaxf(y1, -125.0f));
  const uint64_t magic = f2pack(12582912.0f, 12582912.0f);
  const uint64_t nmagic = f2pack(-12582912.0f, -12582912.0f);
  const uint64_t t2 = f2add(y2, magic);
  const uint64_t n2 = f2add(t2, nmagic);
  const uint64_t f2 = f2fma(n2, f2pack(-1.0f, -1.0f), y2);
  uint64_t q = f2fma(f2pack(0.0551716685f, 0.0551716685f), f2, f2pack(0.2426111251f, 0.2426111251f));
  q = f2fma(q, f2, f2pack(0.6932609677f, 0.6932609677f));
  q = f2fma(q, f2, f2pack(0.9999280572f, 0.9999280572f));
  float q0, q1, t0, t1;
  f2unpack(q, q0, q1);
  f2unpack(t2, t0, t1);
  p0 = __int_as_float(__float_as_int(q0) + (__float_as_int(t0) << 23));
  p1 = __int_as_float(__float_as_int(q1) + (__float_as_int(t1) << 23));
}

__device__ __forceinline__ void st_global_stream_v4(void* ptr, uint4 v) {
  asm volatile("st.global.cs.v4.b32 [%0], {%1, %2, %3, %4};" ::"l"(ptr), "r"(v.x), "r"(v.y), "r"(v.z),
               "r"(v.w)
               : "memory");
}

__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}

// Maximum of N register values with 8 independent chains of 3-input maxima.
template <int N>
__device__ __forceinline__ float row_max(const float* x) {
  constexpr int NA = 8, PER = N / NA;
  float a[NA];
#pragma unroll
  for (int k = 0; k < NA; ++k) {
    a[k] = x[k];
    int t = 1;
#pragma unroll
    for (; t + 1 < PER; t += 2) a[k] = fmax3(a[k], x[k + NA * t], x[k + NA * (t + 1)]);
    if (t < PER) a[k] = fmaxf(a[k], x[k + NA * t]);
  }
  return fmaxf(fmax3(a[0], a[1], a[2]), fmax3(fmax3(a[3], a[4], a[5]), a[6], a[7]));
}

__device__ __forceinline__ void named_bar_sync(int id, int nthreads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}
// Arrives on named barrier `id` (expected count nthreads) without waiting;
// executed by whole warps.
__device__ __forceinline__ void named_bar_arrive(int id, int nthreads) {
  asm volatile("bar.arrive %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

__device__ __forceinline__ uint32_t pack_half2(float lo, float hi) {
  __half2 h = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&h);
}

// Sequence b's extent and the number of `tile`-row tiles of the sequences
// before it (the global index of its first tile).
struct SeqInfo {
  int64_t start;
  int64_t len;
  int64_t tile_base;
};

__device__ __forceinline__ SeqInfo seq_info(const int32_t* cu, int b, int64_t L, int tile) {
  SeqInfo s;
  if (cu == nullptr) {
    s.start = 0;
    s.len = L;
    s.tile_base = 0;
    return s;
  }
  int64_t base = 0;
  int32_t prev = cu[0];
  for (int i = 0; i < b; ++i) {
    const int32_t nxt = cu[i + 1];
    base += (static_cast<int64_t>(nxt - prev) + tile - 1) / tile;
    prev = nxt;
  }
  s.start = prev;
  s.len = static_cast<int64_t>(cu[b + 1]) - prev;
  s.tile_base = base;
  return s;
}

}  // namespace tmk

// Inline-PTX building blocks for sm_100a: mbarriers with bounded waits, TMA
// tile loads, and the 5th-generation tensor core (tcgen05: TMEM allocation,
// MMA issue/commit, TMEM loads).  Written from the PTX ISA's descriptions of
// these instructions.
#pragma once

#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <mutex>

namespace lsh {
namespace sm100 {

// Codes OR-ed into the device error word when a bounded wait gives up.
enum : unsigned int {
  kErrWaitProducer = 1u << 0,
  kErrWaitMma = 1u << 1,
  kErrWaitEpilogue = 1u << 2,
  kErrWaitDrain = 1u << 3,
};

// A bounded wait gives up after this long (ns of %globaltimer).
constexpr unsigned long long kWaitLimitNs = 2000000000ull;

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ unsigned long long globaltimer() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// ---- mbarrier ---------------------------------------------------------------
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}

__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
               "r"(bytes)
               : "memory");
}

// Adds `bytes` to the transaction count the current phase waits for.
__device__ __forceinline__ void mbar_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.expect_tx.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
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

// Like mbar_try_wait, but the thread may be suspended (without taking issue
// slots) until the phase completes or about `suspend_ns` have passed.
__device__ __forceinline__ bool mbar_try_wait_suspend(uint64_t* bar, uint32_t parity,
                                                      uint32_t suspend_ns) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity), "r"(suspend_ns)
      : "memory");
  return ok != 0;
}

// Wait until the phase of `bar` with parity `parity` has completed.  Each
// attempt suspends the thread for up to 0.5 ms, so waiting costs no issue
// slots.  Gives up (returns false) when *abort is set by another thread or
// after kWaitLimitNs; the caller then records an error and leaves its loop.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity,
                                          const volatile int* abort) {
  if (mbar_try_wait(bar, parity)) return true;
  const unsigned long long t0 = globaltimer();
  while (true) {
    if (mbar_try_wait_suspend(bar, parity, 500000u)) return true;
    if (*abort) return false;
    if (globaltimer() - t0 > kWaitLimitNs) return false;
  }
}

// mbar_wait with its own time limit: gives up once `limit_ns` of
// %globaltimer have passed (at once, without looking, when limit_ns is 0).
__device__ __forceinline__ bool mbar_wait_for(uint64_t* bar, uint32_t parity,
                                              const volatile int* abort,
                                              unsigned long long limit_ns) {
  if (limit_ns == 0) return false;
  if (mbar_try_wait(bar, parity)) return true;
  const unsigned long long t0 = globaltimer();
  while (true) {
    if (mbar_try_wait_suspend(bar, parity, 500000u)) return true;
    if (*abort) return false;
    if (globaltimer() - t0 > limit_ns) return false;
  }
}

// Non-blocking test of the phase with parity `parity`.
__device__ __forceinline__ bool mbar_test(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// Like mbar_wait, but spinning on test_wait: the waiter is never suspended,
// so it resumes as soon as the phase completes (at the cost of issue slots
// while it waits).  Same abort flag and time limit.
__device__ __forceinline__ bool mbar_wait_spin(uint64_t* bar, uint32_t parity,
                                               const volatile int* abort) {
  if (mbar_test(bar, parity)) return true;
  const unsigned long long t0 = globaltimer();
  for (uint32_t n = 1;; ++n) {
    if (mbar_test(bar, parity)) return true;
    if ((n & 1023u) == 0) {
      if (*abort) return false;
      if (globaltimer() - t0 > kWaitLimitNs) return false;
    }
  }
}

// Spins, as a whole converged warp, until the phases of all four barriers
// have completed (repeat a barrier to wait on fewer).  The four tests of a
// pass are independent, so their shared-memory round trips overlap instead of
// adding up; a warp vote gives every lane the same verdict.  A completed
// phase cannot complete again before the caller acts, so a lane that saw it
// early loses nothing by waiting for the vote.  Same abort flag and time
// limit as mbar_wait_spin.
__device__ __forceinline__ bool mbar_wait4_warp(uint64_t* b0, uint32_t p0, uint64_t* b1,
                                                uint32_t p1, uint64_t* b2, uint32_t p2,
                                                uint64_t* b3, uint32_t p3,
                                                const volatile int* abort) {
  unsigned long long t0 = 0;
  for (uint32_t n = 0;; ++n) {
    const bool d = mbar_test(b0, p0) & mbar_test(b1, p1) & mbar_test(b2, p2) & mbar_test(b3, p3);
    if (__all_sync(0xffffffffu, d)) return true;
    if (n == 0) t0 = globaltimer();
    if ((n & 1023u) == 1023u) {
      const bool stop = *abort || globaltimer() - t0 > kWaitLimitNs;
      if (__any_sync(0xffffffffu, stop)) return false;
    }
  }
}

// mbar_wait on four barriers in turn for a converged warp (repeat a barrier
// to wait on fewer): the warp sleeps instead of polling, and a vote gives
// every lane the same verdict.
__device__ __forceinline__ bool mbar_wait4_sleep(uint64_t* b0, uint32_t p0, uint64_t* b1,
                                                 uint32_t p1, uint64_t* b2, uint32_t p2,
                                                 uint64_t* b3, uint32_t p3,
                                                 const volatile int* abort) {
  const bool ok = mbar_wait(b0, p0, abort) && mbar_wait(b1, p1, abort) &&
                  mbar_wait(b2, p2, abort) && mbar_wait(b3, p3, abort);
  return __all_sync(0xffffffffu, ok);
}

// mbar_wait_spin over four barriers at once for a single thread (repeat a
// barrier to wait on fewer): the four tests of a pass are independent, so
// their round trips overlap.
__device__ __forceinline__ bool mbar_wait4_spin(uint64_t* b0, uint32_t p0, uint64_t* b1,
                                                uint32_t p1, uint64_t* b2, uint32_t p2,
                                                uint64_t* b3, uint32_t p3,
                                                const volatile int* abort) {
  unsigned long long t0 = 0;
  for (uint32_t n = 0;; ++n) {
    if (mbar_test(b0, p0) & mbar_test(b1, p1) & mbar_test(b2, p2) & mbar_test(b3, p3))
      return true;
    if (n == 0) t0 = globaltimer();
    if ((n & 1023u) == 1023u && (*abort || globaltimer() - t0 > kWaitLimitNs)) return false;
  }
}

// True in exactly one active lane of a converged warp.
__device__ __forceinline__ bool elect_one_sync() {
  uint32_t pred = 0;
  asm volatile(
      "{\n\t.reg .pred P;\n\t"
      "elect.sync _|P, %1;\n\t"
      "selp.b32 %0, 1, 0, P;\n\t}"
      : "=r"(pred)
      : "r"(0xffffffffu));
  return pred != 0;
}

// ---- fences -------------------------------------------------------------------
// Generic-proxy writes to shared memory -> visible to the async proxy (TMA,
// tensor core).
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void tc_fence_before_sync() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}

__device__ __forceinline__ void tc_fence_after_sync() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// ---- TMA ------------------------------------------------------------------------
__device__ __forceinline__ void tma_load_3d(void* dst, const CUtensorMap* map, uint64_t* bar,
                                            int x, int y, int z) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5}], [%2];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(x), "r"(y), "r"(z)
      : "memory");
}

// Four rows y0..y3 of a 2-D tensor map whose box is one row high, starting
// at column x (x * element size must be a multiple of 16 bytes), to four
// consecutive box-sized pieces of shared memory.  Rows outside the tensor
// read as zeros.
__device__ __forceinline__ void tma_gather4(void* dst, const CUtensorMap* map, uint64_t* bar,
                                            int x, int y0, int y1, int y2, int y3) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile::gather4.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5, %6, %7}], [%2];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(x), "r"(y0), "r"(y1), "r"(y2),
      "r"(y3)
      : "memory");
}

__device__ __forceinline__ void tma_prefetch_desc(const CUtensorMap* map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// ---- TMEM -------------------------------------------------------------------------
// Executed by one full warp.  Writes the TMEM base address to *dst (shared).
__device__ __forceinline__ void tmem_alloc(uint32_t* dst, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                   smem_u32(dst)),
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

// 32 lanes x 32 consecutive 32-bit columns: thread t gets lane (base + t),
// columns col..col+31 in r[0..31].
__device__ __forceinline__ void tmem_ld_32x32b_x32(uint32_t taddr, uint32_t* r) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
      "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
        "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]),
        "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
        "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]),
        "=r"(r[31])
      : "r"(taddr));
}

// Wait for this thread's outstanding tcgen05.ld; the register operands tie
// every use of the loaded values to after the wait.
__device__ __forceinline__ void tmem_ld_wait(uint32_t* r) {
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int i = 0; i < 32; ++i) asm volatile("" : "+r"(r[i]));
}

// 32 lanes x 16 consecutive 32-bit columns from registers: thread t writes
// lane (base + t), columns col..col+15 from r[0..15].
__device__ __forceinline__ void tmem_st_32x32b_x16(uint32_t taddr, const uint32_t* r) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
      "{%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
      "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]),
      "r"(r[15])
      : "memory");
}

// Wait until this thread's outstanding tcgen05.st have written tensor memory.
__device__ __forceinline__ void tmem_st_wait() {
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

// ---- MMA ----------------------------------------------------------------------------
// D[tmem] (+)= A[tmem] x B[smem]^T, kind::f16: A (bf16, M rows across the TMEM
// lanes, two K elements per 32-bit column) is read from tensor memory.
__device__ __forceinline__ void mma_bf16_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc,
                                            uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// D[tmem] (+)= A[smem] x B[smem]^T, kind::f16 (bf16 inputs, fp32 accumulate),
// one issuing thread.  accumulate == 0 overwrites D.
__device__ __forceinline__ void mma_bf16_ss(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                            uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// The mbarrier completes one arrival when every tcgen05.mma issued so far by
// this thread has finished.
__device__ __forceinline__ void mma_commit(uint64_t* bar) {
  asm volatile(
      "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
          smem_u32(bar))
      : "memory");
}

// Instruction descriptor of kind::f16: bf16 A and B, fp32 accumulator, both
// operands K-major, shape M x N.
__host__ __device__ constexpr uint32_t idesc_bf16_f32(int M, int N) {
  return (1u << 4)                          // D format: f32
         | (1u << 7)                        // A format: bf16
         | (1u << 10)                       // B format: bf16
         | ((uint32_t)(N >> 3) << 17)       // N / 8
         | ((uint32_t)(M >> 4) << 24);      // M / 16
}

// Shared-memory matrix descriptor, K-major, 128-byte swizzle: rows of 128
// bytes (64 bf16 of K), 8-row groups 1024 bytes apart, atoms 1024-aligned.
// Stepping K by 16 elements inside an atom advances the start address by 32 B.
__device__ __forceinline__ uint64_t sdesc_kmajor_sw128(uint32_t saddr) {
  return (uint64_t)((saddr & 0x3FFFFu) >> 4)   // start address
         | ((uint64_t)1 << 16)                 // leading byte offset (unused here)
         | ((uint64_t)(1024 >> 4) << 32)       // stride byte offset: 8 rows
         | ((uint64_t)1 << 46)                 // descriptor version (sm_100)
         | ((uint64_t)2 << 61);                // swizzle: 128 B
}

// Byte offset of element (row, k) in a K-major 128B-swizzled tile whose rows
// are 128 bytes of bf16 (k < 64): 16-byte chunk index XOR (row % 8).
__host__ __device__ __forceinline__ uint32_t sw128_offset(uint32_t row, uint32_t k) {
  return row * 128u + ((((k >> 3) ^ (row & 7u)) & 7u) << 4) + ((k & 7u) << 1);
}

// cuTensorMapEncodeTiled from the driver, resolved once (nullptr if absent).
inline PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
  static std::once_flag once;
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  std::call_once(once, [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &ptr, 12000,
                                         cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
  });
  return fn;
}

}  // namespace sm100
}  // namespace lsh

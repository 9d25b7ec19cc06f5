// Fifth-generation tensor core (tcgen05) and mbarrier helpers for sm_100a kernels: operand
// layout and descriptors of kind::tf32 MMAs from shared memory, bounded mbarrier waits, bulk
// copies without multicast, TMEM loads.  Each including translation unit gets its own copies
// (internal linkage).
#pragma once

#include <cuda_runtime.h>

#include <cstdint>

#include "internal.h"

namespace e3b {
namespace {

// Byte offset of element (row, k) of a K-major operand block with K columns, in the canonical
// no-swizzle layout: 8-row x 16-byte core matrices; the core matrices along K are LBO = 128 bytes
// apart (so one MMA K-step of 8 tf32 values spans 256 bytes), 8-row groups SBO = 32 K bytes apart.
__host__ __device__ constexpr uint32_t kmajor_off(int row, int k, int K) {
  return uint32_t((row >> 3) * (K * 32) + (k >> 2) * 128 + (row & 7) * 16 + (k & 3) * 4);
}

// Shared-memory matrix descriptor: start address, LBO, SBO (16-byte units), the descriptor
// version of this architecture (bit 46), no swizzle (bits 61-63 zero).
__device__ __forceinline__ uint64_t smem_desc(uint32_t saddr, int K) {
  const uint64_t lbo = 128u >> 4, sbo = uint64_t(K * 32) >> 4;
  return uint64_t((saddr >> 4) & 0x3FFFu) | (lbo << 16) | (sbo << 32) | (uint64_t(1) << 46);
}

// Instruction descriptor of kind::tf32: float32 accumulator (bits 4-5 = 1), A and B tf32 (bits
// 7-9 and 10-12 = 2), both K-major, N / 8 at bits 17-22, M / 16 at bits 24-28.
constexpr uint32_t idesc_tf32(int M, int N) {
  return (1u << 4) | (2u << 7) | (2u << 10) | (uint32_t(N >> 3) << 17) | (uint32_t(M >> 4) << 24);
}

__device__ __forceinline__ uint32_t saddr(const void* p) { return static_cast<uint32_t>(__cvta_generic_to_shared(p)); }

__device__ __forceinline__ float to_tf32(float x) {
  uint32_t r;
  asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(r) : "f"(x));
  return __uint_as_float(r);
}

__device__ __forceinline__ unsigned long long now_ns() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ void bar_init(uint64_t* b, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(saddr(b)), "r"(count) : "memory");
}

__device__ __forceinline__ bool bar_test(uint64_t* b, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(ok)
      : "r"(saddr(b)), "r"(parity)
      : "memory");
  return ok != 0;
}

// Bounded wait for phase `parity` of barrier b; false (E3_ERR_TIMEOUT recorded) after wait_ns.
__device__ __forceinline__ bool bar_wait(uint64_t* b, uint32_t parity, int* status, unsigned long long wait_ns) {
  if (bar_test(b, parity)) return true;
  const unsigned long long t0 = now_ns();
  while (!bar_test(b, parity)) {
    if (now_ns() - t0 > wait_ns) {
      atomicCAS(status, 0, int(E3_ERR_TIMEOUT));
      return false;
    }
  }
  return true;
}

__device__ __forceinline__ void bulk_copy(void* dst, const void* src, uint32_t bytes, uint64_t* b) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(saddr(b)), "r"(bytes) : "memory");
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                   saddr(dst)),
               "l"(src), "r"(bytes), "r"(saddr(b))
               : "memory");
}

__device__ __forceinline__ void mma_tf32(uint32_t tmem_d, uint64_t a, uint64_t b, uint32_t idesc, uint32_t accumulate) {
  const uint32_t mask = 0;  // no output lane disabled
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
      " tcgen05.mma.cta_group::1.kind::tf32 [%0], %1, %2, %3, {%5, %5, %5, %5}, p;\n}\n" ::"r"(tmem_d),
      "l"(a), "l"(b), "r"(idesc), "r"(accumulate), "r"(mask));
}

__device__ __forceinline__ void mma_commit(uint64_t* b) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(saddr(b))
               : "memory");
}

__device__ __forceinline__ void fence_before_sync() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void fence_after_sync() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// 32 consecutive accumulator columns of this thread's TMEM lane (the caller waits with
// tcgen05.wait::ld before reading v).
__device__ __forceinline__ void tmem_ld32_nowait(uint32_t taddr, uint32_t (&v)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
      "%15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
      : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7]), "=r"(v[8]),
        "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), "=r"(v[14]), "=r"(v[15]), "=r"(v[16]),
        "=r"(v[17]), "=r"(v[18]), "=r"(v[19]), "=r"(v[20]), "=r"(v[21]), "=r"(v[22]), "=r"(v[23]), "=r"(v[24]),
        "=r"(v[25]), "=r"(v[26]), "=r"(v[27]), "=r"(v[28]), "=r"(v[29]), "=r"(v[30]), "=r"(v[31])
      : "r"(taddr));
}

// The same wait by every lane of a warp, with one verdict for the warp: the lanes leave it
// converged (the TMEM loads that follow are warp-collective) and agree on a timeout.
// Lane 0 polls (32 lanes polling one barrier serialise in shared memory); once it has seen the
// phase complete, every lane tests it once more, which succeeds at once and gives each lane its
// own acquire of what the phase publishes (the phase cannot advance before this warp signals).
__device__ __forceinline__ bool warp_wait(uint64_t* b, uint32_t parity, int* status, unsigned long long wait_ns) {
  bool ok = true;
  if ((threadIdx.x & 31) == 0) ok = bar_wait(b, parity, status, wait_ns);
  ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
  if (ok) ok = bar_test(b, parity);
  return __all_sync(0xffffffffu, ok) != 0;
}

// The abort flag as one value for the whole warp.
__device__ __forceinline__ bool warp_aborted(volatile int* flag) { return __any_sync(0xffffffffu, *flag != 0) != 0; }

}  // namespace
}  // namespace e3b

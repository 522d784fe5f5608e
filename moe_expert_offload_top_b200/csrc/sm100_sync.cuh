// mbarrier helpers with bounded waits, shared by the sm_100a kernels that
// stage data through shared memory (TMA producers and their consumers).
//
// Every wait is bounded by an iteration cap and a %globaltimer cap: on timeout
// the waiting thread records `code` in the device error word and raises the
// CTA's abort flag, so all roles leave instead of waiting for ever.
#pragma once
#include "common.cuh"

namespace ftk {

constexpr long long WAIT_LIMIT = 1ll << 30;            // iteration cap of one wait
constexpr unsigned long long WAIT_NS = 2000000000ull;  // and its time cap: 2 s

FT_DEVICE uint32_t smem_u32(const void* p) { return (uint32_t)__cvta_generic_to_shared(p); }

FT_DEVICE void mbar_init(uint64_t* b, int count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(b)), "r"(count));
}
FT_DEVICE void mbar_expect_tx(uint64_t* b, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(b)), "r"(bytes)
               : "memory");
}
FT_DEVICE void mbar_arrive(uint64_t* b) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(b)) : "memory");
}
FT_DEVICE bool mbar_try(uint64_t* b, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(b)), "r"(parity)
      : "memory");
  return ok != 0;
}
FT_DEVICE unsigned long long global_ns() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}
// Bounded wait.  Returns false (after flagging) on timeout or when the CTA aborts.
FT_DEVICE bool mbar_wait(uint64_t* b, uint32_t parity, volatile int* abort_flag, int* err, int code,
                         unsigned long long limit_ns = WAIT_NS) {
  if (mbar_try(b, parity)) return true;
  const unsigned long long t0 = global_ns();
  for (long long i = 0; i < WAIT_LIMIT; ++i) {
    if (mbar_try(b, parity)) return true;
    if ((i & 255) == 255) {
      if (*abort_flag) return false;
      if (global_ns() - t0 > limit_ns) break;
    }
  }
  *abort_flag = 1;
  atomicExch(err, code);
  return false;
}
// Bounded wait used while draining: no flagging.
FT_DEVICE void mbar_drain(uint64_t* b, uint32_t parity) {
  const unsigned long long t0 = global_ns();
  for (long long i = 0; i < WAIT_LIMIT; ++i) {
    if (mbar_try(b, parity)) return;
    if ((i & 255) == 255 && global_ns() - t0 > WAIT_NS) return;
  }
}


}  // namespace ftk

// Device helpers shared by the sm_100a kernels of the routed-MoE layer.
#pragma once
#include <cuda_runtime.h>
#include <stdint.h>

#define FT_DEVICE __device__ __forceinline__

namespace ftk {

// bf16 halves of a 32-bit word -> two fp32 values (a bf16 is the top half of a float32).
FT_DEVICE float bf16lo(uint32_t w) { return __uint_as_float(w << 16); }
FT_DEVICE float bf16hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }
FT_DEVICE float bf16_to_f32(uint16_t b) { return __uint_as_float(((uint32_t)b) << 16); }

// fp32 -> bf16 bits, round to nearest even (finite inputs).
FT_DEVICE uint16_t f32_to_bf16(float f) {
  uint32_t u = __float_as_uint(f);
  u += 0x7FFFu + ((u >> 16) & 1u);
  return (uint16_t)(u >> 16);
}

// 16-byte streaming load of data read once per launch: bypasses L1 allocation.
FT_DEVICE uint4 ld_stream16(const void* p) {
  uint4 r;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "l"(p));
  return r;
}

FT_DEVICE float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xFFFFFFFFu, v, o);
  return v;
}

FT_DEVICE float silu(float a) { return a / (1.0f + expf(-a)); }

}  // namespace ftk

// Building blocks of the tensor-core decode GEMVs for packed weights (int4, NVFP4): every
// lane copies the bytes it reads itself into its own slots of a shared-memory ring with
// cp.async (16-byte copies, 32-bit shared addresses), a block maximum for the per-row
// input scales, and launches with dynamic shared memory and programmatic dependence.
#pragma once
#include "common.cuh"
#include "kernels.hpp"
#include "sm100_sync.cuh"

namespace ftk {
namespace ring {

FT_DEVICE void cp16s(uint32_t dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}
FT_DEVICE uint4 lds128(uint32_t a) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(a));
  return v;
}
FT_DEVICE uint32_t lds32(uint32_t a) {
  uint32_t v;
  asm volatile("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(a));
  return v;
}
FT_DEVICE void cp_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
FT_DEVICE void cp_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }
FT_DEVICE uint32_t word_of(const uint4& v, int j) { return j == 0 ? v.x : j == 1 ? v.y : j == 2 ? v.z : v.w; }

// Threads of the slicing kernels.
constexpr int kPrepThreads = 256;

// Block maximum of v over kPrepThreads threads (all call it).  Its barriers also order every
// read before it ahead of every write after it.
FT_DEVICE float block_max(float v, float* red) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xFFFFFFFFu, v, o));
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = v;
  __syncthreads();
  float m = 0.f;
  for (int i = 0; i < kPrepThreads / 32; ++i) m = fmaxf(m, red[i]);
  __syncthreads();
  return m;
}

// Binary exponent E of m > 0 (m = f * 2^E, 1 <= f < 2), 0 for m = 0.
FT_DEVICE int exponent_of(float m) { return m > 0.f ? ((int)((__float_as_uint(m) >> 23) & 0xFF) - 127) : 0; }

// Launches `kern` with `smem` bytes of dynamic shared memory; with `dependent`, as a
// programmatic dependent launch of the previous kernel on the stream.
template <typename... KArgs, typename... Args>
cudaError_t launch_ex(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s, bool dependent,
                      Args... args) {
  if (smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = dependent ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, kern, static_cast<KArgs>(args)...);
}

}  // namespace ring
}  // namespace ftk

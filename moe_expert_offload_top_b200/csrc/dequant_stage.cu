// Prefill with NVFP4 expert weights: the selected experts' NVFP4 blobs are expanded to
// bf16 in a staging arena, where the tcgen05 grouped GEMMs read them.
//
// Method ("FreeToken linux": the 4-bit release; "FreeToken's MoE memory handling"):
// every selected expert runs from its cache slot.  The NVFP4 weight of element (r, c)
// of a matrix is e2m1(r, c) * e4m3(r, c / 16) * g, with g the fp32 scale of the whole
// matrix.  The product of an e2m1 value (at most 2 significant bits) and an e4m3 scale
// (at most 4) has at most 6 significant bits and lies in bf16's range, so the staged
// bf16 value e2m1 * e4m3 is exact; g is applied to the GEMM's fp32 accumulator (the
// epilogue multiplies gate, up and down by their own g).  The tensor-core MMA then
// multiplies exact weights by the bf16 activations, as for bf16 stacks.
//
// Staged layout per expert: the bf16 blob layout (W_gate [I][H], W_up [I][H],
// W_down [H][I]), so the GEMMs' tensor maps address it as they address bf16 slots.
#include "decode_gemv.cuh"

namespace ftk {

namespace {

using namespace gemv;

// One thread per 32 elements (16 bytes of e2m1 codes, two e4m3 block scales).
__global__ void __launch_bounds__(256)
dequant_nvfp4_stage_kernel(const __grid_constant__ ExpertList list, int H, int I, uint16_t* __restrict__ stage,
                           float* __restrict__ gscale) {
  const size_t mat = (size_t)H * I;
  const size_t chunks = 3 * mat / 32;                 // per expert
  const size_t blob_elems = 3 * mat;                  // staged bf16 elements per expert
  const size_t total = chunks * (size_t)list.n;
  for (size_t idx = (size_t)blockIdx.x * blockDim.x + threadIdx.x; idx < total;
       idx += (size_t)gridDim.x * blockDim.x) {
    const int entry = (int)(idx / chunks);
    const size_t c = idx - (size_t)entry * chunks;
    const uint8_t* blob = list.blob[entry];
    const size_t e0 = c * 32;                         // first element, over the three matrices
    const size_t m = e0 / mat, off = e0 - m * mat;
    const uint4 q = __ldcs(reinterpret_cast<const uint4*>(blob + m * (mat / 2) + off / 2));
    const uint16_t sc2 = *reinterpret_cast<const uint16_t*>(blob + 3 * mat / 2 + m * (mat / 16) + off / 16);
    // the two 16-element block scales as f16, each broadcast to both halves of a pair
    uint32_t s2;
    asm("{ .reg .b16 t; cvt.u16.u32 t, %1; cvt.rn.f16x2.e4m3x2 %0, t; }" : "=r"(s2) : "r"((uint32_t)sc2));
    const uint32_t s_lo = __byte_perm(s2, 0, 0x1010), s_hi = __byte_perm(s2, 0, 0x3232);
    const uint32_t w[4] = {q.x, q.y, q.z, q.w};
    uint32_t out[16];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const uint32_t sp = i < 2 ? s_lo : s_hi;
#pragma unroll
      for (int b = 0; b < 4; ++b) {
        // two e2m1 codes -> f16 pair (exact), times the f16 scale pair (exact: at most 6
        // significant bits, within f16 range), -> two fp32 -> one bf16 pair (exact)
        uint32_t h2, p2, o;
        asm("{ .reg .b8 t; cvt.u8.u32 t, %1; cvt.rn.f16x2.e2m1x2 %0, t; }" : "=r"(h2) : "r"((w[i] >> (8 * b)) & 0xFFu));
        asm("mul.rn.f16x2 %0, %1, %2;" : "=r"(p2) : "r"(h2), "r"(sp));
        const float lo = __half2float(__ushort_as_half((unsigned short)(p2 & 0xFFFFu)));
        const float hi = __half2float(__ushort_as_half((unsigned short)(p2 >> 16)));
        asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(o) : "f"(hi), "f"(lo));
        out[4 * i + b] = o;
      }
    }
    uint4* dst = reinterpret_cast<uint4*>(stage + (size_t)entry * blob_elems + e0);
#pragma unroll
    for (int i = 0; i < 4; ++i) dst[i] = make_uint4(out[4 * i], out[4 * i + 1], out[4 * i + 2], out[4 * i + 3]);
    if (c == 0) {
      const float* gl = reinterpret_cast<const float*>(blob + 3 * mat / 2 + 3 * mat / 16);
      gscale[3 * entry] = gl[0];
      gscale[3 * entry + 1] = gl[1];
      gscale[3 * entry + 2] = gl[2];
    }
  }
}

}  // namespace

cudaError_t launch_dequant_nvfp4_stage(const ExpertList& list, int H, int I, void* stage, float* gscale, int num_sms,
                                       cudaStream_t s) {
  if (list.n <= 0) return cudaSuccess;
  if (H % 32 || I % 32) return cudaErrorInvalidValue;
  const long long total = (long long)list.n * (3LL * H * I / 32);
  long long blocks = (total + 255) / 256;
  const long long cap = 8LL * (num_sms > 0 ? num_sms : 148);
  if (blocks > cap) blocks = cap;
  dequant_nvfp4_stage_kernel<<<(unsigned)blocks, 256, 0, s>>>(list, H, I, static_cast<uint16_t*>(stage), gscale);
  return cudaGetLastError();
}

}  // namespace ftk

// K3 - SwiGLU expert FFN for decode-sized batches, reading every selected
// expert's weights from its cache slot, and K5 - the gate-weighted combine.
//
// Method ("FreeToken linux", "FreeToken's MoE memory handling"; "FreeToken
// gguf", the `offload` backend): each activated expert runs on the GPU from
// the slot that holds it.  Expert FFN (stated workloads): h = silu(W_gate x) *
// (W_up x), y = W_down h.  Output: out[t] = sum_j g[t,j] y[t,j] + shared(x_t).
//
// At decode sizes (a few tokens per expert) the FFN is a batch of
// matrix-vector products bound by HBM bandwidth: every weight byte is read
// exactly once per launch with 16-byte streaming loads, and the few token
// vectors of an expert are staged once per CTA in shared memory.
#include <cuda_fp16.h>

#include "common.cuh"
#include "kernels.hpp"

namespace ftk {

namespace {

enum { WT_F32 = 0, WT_BF16 = 1, WT_INT4 = 2, WT_NVFP4 = 3 };
enum { MODE_GATE_UP = 0, MODE_DOWN = 1 };

#ifndef FT_GEMV_WARPS
#define FT_GEMV_WARPS 4
#endif
#ifndef FT_GEMV_GU_RPW
#define FT_GEMV_GU_RPW 2
#endif
#ifndef FT_GEMV_D_RPW
#define FT_GEMV_D_RPW 4
#endif
#ifndef FT_GEMV_NT_MAX
#define FT_GEMV_NT_MAX 8
#endif
constexpr int kWarps = FT_GEMV_WARPS;   // warps per CTA
constexpr int kThreads = kWarps * 32;

// Elements held by one 16-byte weight load.
template <int WT> struct WTraits;
template <> struct WTraits<WT_F32>  { static constexpr int EL = 4; };
template <> struct WTraits<WT_BF16> { static constexpr int EL = 8; };
template <> struct WTraits<WT_INT4> { static constexpr int EL = 32; };
template <> struct WTraits<WT_NVFP4> { static constexpr int EL = 32; };

// Two e2m1 values of one byte -> fp32 (hardware conversion to f16x2, then widened).
FT_DEVICE void e2m1x2_to_f32(uint32_t byte, float& lo, float& hi) {
  uint32_t h2;
  asm("{ .reg .b8 t; cvt.u8.u32 t, %1; cvt.rn.f16x2.e2m1x2 %0, t; }" : "=r"(h2) : "r"(byte));
  lo = __half2float(__ushort_as_half((unsigned short)(h2 & 0xFFFFu)));
  hi = __half2float(__ushort_as_half((unsigned short)(h2 >> 16)));
}
// Two e4m3 values of a 16-bit word -> fp32.
FT_DEVICE void e4m3x2_to_f32(uint32_t two, float& lo, float& hi) {
  uint32_t h2;
  asm("{ .reg .b16 t; cvt.u16.u32 t, %1; cvt.rn.f16x2.e4m3x2 %0, t; }" : "=r"(h2) : "r"(two));
  lo = __half2float(__ushort_as_half((unsigned short)(h2 & 0xFFFFu)));
  hi = __half2float(__ushort_as_half((unsigned short)(h2 >> 16)));
}

// 16-byte weight load, read once per launch: evict-first in the caches.  Not
// volatile, so the compiler may hoist the loads of later iterations.
FT_DEVICE uint4 ldw(const uint8_t* p) { return __ldcs(reinterpret_cast<const uint4*>(p)); }


// Weights of one 16-byte chunk, group g of 8 elements (f32: 4 elements) -> fp32
// (int4: the raw integers; the group scale multiplies the chunk's partial sum).
template <int WT>
FT_DEVICE void wgroup(const uint4& c, int g, float* v) {
  const uint32_t w[4] = {c.x, c.y, c.z, c.w};
  if constexpr (WT == WT_F32) {
#pragma unroll
    for (int i = 0; i < 4; ++i) v[i] = __uint_as_float(w[i]);
  } else if constexpr (WT == WT_BF16) {
#pragma unroll
    for (int i = 0; i < 4; ++i) { v[2 * i] = bf16lo(w[i]); v[2 * i + 1] = bf16hi(w[i]); }
  } else {
#pragma unroll
    for (int n = 0; n < 8; ++n) v[n] = (float)(((int32_t)(w[g] << (28 - 4 * n))) >> 28);
  }
}

// Input elements [i, i + GE) of one token vector (GE = 4 for f32 weights, else 8):
// x is bf16 (gate/up of bf16/int4 stacks) or f32; h is f32.
template <int GE, bool BF16IN>
FT_DEVICE void ldin(const void* base, int i, float* v) {
  if constexpr (BF16IN) {
    const uint4 a = __ldg(reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(base) + i));
    const uint32_t u[4] = {a.x, a.y, a.z, a.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) { v[2 * j] = bf16lo(u[j]); v[2 * j + 1] = bf16hi(u[j]); }
  } else {
    const float* f = static_cast<const float*>(base) + i;
#pragma unroll
    for (int j = 0; j < GE; j += 4) {
      const float4 a = __ldg(reinterpret_cast<const float4*>(f + j));
      v[j] = a.x; v[j + 1] = a.y; v[j + 2] = a.z; v[j + 3] = a.w;
    }
  }
}

// Grouped GEMV.  Grid (ceil(rows / (kWarps*RPW)), list.n); warp w of CTA (bx, i)
// owns rows [(bx*kWarps + w)*RPW, +RPW) of list entry i and all of its pairs, NT
// at a time:
//   MODE_GATE_UP: rows of W_gate and W_up (I rows, K = H), input x[token(q)],
//                 output h[q][r] = silu(W_gate[r].x) * (W_up[r].x)
//   MODE_DOWN:    rows of W_down (H rows, K = I), input h[q], output y[q][r].
// Lane l reads 16-byte chunks l, l+32, ... of each row; token vectors come
// through L1 (every warp of the entry reads the same few).  No shared memory,
// no block barrier: warps stream independently.
template <int MODE, int WT, int NT, int RPW>
__global__ void __launch_bounds__(kThreads)
grouped_gemv_kernel(const void* __restrict__ xin, int T, int H, int I, int k,
                    const __grid_constant__ ExpertList list, const int* __restrict__ offsets,
                    const int* __restrict__ perm, float* __restrict__ hbuf,
                    float* __restrict__ ybuf) {
  constexpr int EL = WTraits<WT>::EL;
  constexpr bool GU = MODE == MODE_GATE_UP;
  constexpr int NM = GU ? 2 : 1;               // weight matrices per row
  constexpr int GE = WT == WT_F32 ? 4 : 8;     // elements per decode group
  constexpr int NG = EL / GE;                  // groups per chunk
  constexpr bool BF16IN = GU && WT != WT_F32;

  const int entry = blockIdx.y;
  const int e = list.expert[entry];
  const uint8_t* blob = list.blob[entry];
  const int K = GU ? H : I;
  const int rows = GU ? I : H;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int rbase = (blockIdx.x * kWarps + warp) * RPW;
  // Programmatic dependent launch: the down projection may be launched while this
  // gate/up grid runs; it waits for this grid's completion before it reads h.
  if (GU) asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  else asm volatile("griddepcontrol.wait;" ::: "memory");
  const int q0 = e >= 0 ? offsets[e] : T * k;
  const int q1 = e >= 0 ? offsets[e + 1] : T * k + T;
  if (q1 <= q0) return;
  if (rbase >= rows) return;

  const size_t mat = (size_t)H * I;
  const uint8_t* wmat[2];
  const uint16_t* smat[2] = {nullptr, nullptr};
  const uint8_t* fmat[2] = {nullptr, nullptr};   // nvfp4 e4m3 block scales
  float gmat[2] = {1.f, 1.f};                    // nvfp4 fp32 global scales
  if (WT == WT_NVFP4) {
    const uint8_t* sc = blob + 3 * mat / 2;
    const float* gl = reinterpret_cast<const float*>(blob + 3 * mat / 2 + 3 * mat / 16);
    if (GU) { wmat[0] = blob; wmat[1] = blob + mat / 2; fmat[0] = sc; fmat[1] = sc + mat / 16; gmat[0] = gl[0]; gmat[1] = gl[1]; }
    else { wmat[0] = blob + mat; wmat[1] = nullptr; fmat[0] = sc + 2 * (mat / 16); gmat[0] = gl[2]; }
  } else if (WT == WT_INT4) {
    const uint16_t* sc = reinterpret_cast<const uint16_t*>(blob + 3 * mat / 2);
    if (GU) { wmat[0] = blob; wmat[1] = blob + mat / 2; smat[0] = sc; smat[1] = sc + mat / 128; }
    else { wmat[0] = blob + mat; wmat[1] = nullptr; smat[0] = sc + 2 * (mat / 128); }
  } else {
    constexpr int es = WT == WT_F32 ? 4 : 2;
    if (GU) { wmat[0] = blob; wmat[1] = blob + mat * es; }
    else { wmat[0] = blob + 2 * mat * es; wmat[1] = nullptr; }
  }
  const size_t row_bytes = (WT == WT_INT4 || WT == WT_NVFP4) ? (size_t)K / 2 : (size_t)K * (WT == WT_F32 ? 4 : 2);
  bool rok[RPW];
#pragma unroll
  for (int r = 0; r < RPW; ++r) rok[r] = rbase + r < rows;

  for (int c = q0; c < q1; c += NT) {
    const int nt = min(NT, q1 - c);
    const void* in[NT];
#pragma unroll
    for (int t = 0; t < NT; ++t) {
      const int q = c + (t < nt ? t : 0);
      if (GU) {
        const int tok = e >= 0 ? perm[q] / k : q - T * k;
        in[t] = BF16IN ? (const void*)(static_cast<const uint16_t*>(xin) + (size_t)tok * H)
                       : (const void*)(static_cast<const float*>(xin) + (size_t)tok * H);
      } else {
        in[t] = hbuf + (size_t)q * I;
      }
    }
    float acc[RPW][NM][NT];
#pragma unroll
    for (int r = 0; r < RPW; ++r)
#pragma unroll
      for (int m = 0; m < NM; ++m)
#pragma unroll
        for (int t = 0; t < NT; ++t) acc[r][m][t] = 0.f;

#pragma unroll 2
    for (int kk = lane * EL; kk < K; kk += 32 * EL) {
      uint4 wc[RPW][NM];
      float sc[RPW][NM];
#pragma unroll
      for (int r = 0; r < RPW; ++r)
#pragma unroll
        for (int m = 0; m < NM; ++m) {
          const int rr = rok[r] ? rbase + r : rbase;
          wc[r][m] = ldw(wmat[m] + (size_t)rr * row_bytes +
                         ((WT == WT_INT4 || WT == WT_NVFP4) ? kk / 2 : kk * (WT == WT_F32 ? 4 : 2)));
          if (WT == WT_INT4) sc[r][m] = bf16_to_f32(__ldg(smat[m] + (size_t)rr * (K / 128) + kk / 128));
          if (WT == WT_NVFP4) {   // the chunk's two block scales, packed in sc as raw bits
            const uint16_t two = __ldg(reinterpret_cast<const unsigned short*>(fmat[m] + (size_t)rr * (K / 16) + kk / 16));
            sc[r][m] = __uint_as_float((uint32_t)two);
          }
        }
      float part[RPW][NM][NT];
#pragma unroll
      for (int r = 0; r < RPW; ++r)
#pragma unroll
        for (int m = 0; m < NM; ++m)
#pragma unroll
          for (int t = 0; t < NT; ++t) part[r][m][t] = 0.f;
      if constexpr (WT == WT_NVFP4) {
        // e2m1 bytes -> f16x2 by the hardware conversion -> fp32; partial sums per
        // 16-element block are scaled by that block's e4m3 scale.
        float pb[RPW][NM][NT][2];
#pragma unroll
        for (int r = 0; r < RPW; ++r)
#pragma unroll
          for (int m = 0; m < NM; ++m)
#pragma unroll
            for (int t = 0; t < NT; ++t) pb[r][m][t][0] = pb[r][m][t][1] = 0.f;
#pragma unroll
        for (int g = 0; g < 4; ++g) {
          float xv[NT][8];
#pragma unroll
          for (int t = 0; t < NT; ++t)
            if (t < nt) ldin<8, BF16IN>(in[t], kk + 8 * g, xv[t]);
#pragma unroll
          for (int r = 0; r < RPW; ++r)
#pragma unroll
            for (int m = 0; m < NM; ++m) {
              const uint32_t w = g == 0 ? wc[r][m].x : g == 1 ? wc[r][m].y : g == 2 ? wc[r][m].z : wc[r][m].w;
              float wv[8];
#pragma unroll
              for (int b = 0; b < 4; ++b) e2m1x2_to_f32((w >> (8 * b)) & 0xFFu, wv[2 * b], wv[2 * b + 1]);
#pragma unroll
              for (int t = 0; t < NT; ++t)
                if (t < nt) {
#pragma unroll
                  for (int j = 0; j < 8; ++j) pb[r][m][t][g >> 1] = fmaf(wv[j], xv[t][j], pb[r][m][t][g >> 1]);
                }
            }
        }
#pragma unroll
        for (int r = 0; r < RPW; ++r)
#pragma unroll
          for (int m = 0; m < NM; ++m) {
            float s0, s1;
            e4m3x2_to_f32(__float_as_uint(sc[r][m]), s0, s1);
#pragma unroll
            for (int t = 0; t < NT; ++t) part[r][m][t] = s0 * pb[r][m][t][0] + s1 * pb[r][m][t][1];
          }
      } else if constexpr (WT == WT_INT4) {
        // Packed dequant.  Nibbles n and n+4 of a word sit in the two 16-bit halves of
        // (w >> 4n) & 0x000F000F; xor with 0x4308 per half makes the bf16 128 + (q + 8)
        // (0x4300 is 128.0 in bf16, its last mantissa bit 1.0; xor 8 maps a 4-bit
        // two's-complement q to q + 8).  Widening to fp32 and one packed add of -136
        // give the pair (q_n, q_{n+4}) exactly; packed fp32 FMAs meet the matching x
        // pairs.  About 3 lane instructions per weight instead of 5.
        float2 acc2[RPW][NM][NT];
#pragma unroll
        for (int r = 0; r < RPW; ++r)
#pragma unroll
          for (int m = 0; m < NM; ++m)
#pragma unroll
            for (int t = 0; t < NT; ++t) acc2[r][m][t] = make_float2(0.f, 0.f);
        const float2 bias = make_float2(-136.f, -136.f);
#pragma unroll
        for (int g = 0; g < 4; ++g) {
          float2 xp[NT][4];
#pragma unroll
          for (int t = 0; t < NT; ++t)
            if (t < nt) {
              float xv[8];
              ldin<8, BF16IN>(in[t], kk + 8 * g, xv);
#pragma unroll
              for (int n = 0; n < 4; ++n) xp[t][n] = make_float2(xv[n], xv[n + 4]);
            }
#pragma unroll
          for (int r = 0; r < RPW; ++r)
#pragma unroll
            for (int m = 0; m < NM; ++m) {
              const uint32_t w = g == 0 ? wc[r][m].x : g == 1 ? wc[r][m].y : g == 2 ? wc[r][m].z : wc[r][m].w;
#pragma unroll
              for (int n = 0; n < 4; ++n) {
                const uint32_t v = ((w >> (4 * n)) & 0x000F000Fu) ^ 0x43084308u;
                const float2 q2 = __fadd2_rn(make_float2(bf16lo(v), bf16hi(v)), bias);
#pragma unroll
                for (int t = 0; t < NT; ++t)
                  if (t < nt) acc2[r][m][t] = __ffma2_rn(q2, xp[t][n], acc2[r][m][t]);
              }
            }
        }
#pragma unroll
        for (int r = 0; r < RPW; ++r)
#pragma unroll
          for (int m = 0; m < NM; ++m)
#pragma unroll
            for (int t = 0; t < NT; ++t) part[r][m][t] = acc2[r][m][t].x + acc2[r][m][t].y;
      } else {
#pragma unroll
      for (int g = 0; g < NG; ++g) {
        float wv[RPW][NM][GE];
#pragma unroll
        for (int r = 0; r < RPW; ++r)
#pragma unroll
          for (int m = 0; m < NM; ++m) wgroup<WT>(wc[r][m], g, wv[r][m]);
#pragma unroll
        for (int t = 0; t < NT; ++t) {
          if (t < nt) {
            float xv[GE];
            ldin<GE, BF16IN>(in[t], kk + g * GE, xv);
#pragma unroll
            for (int r = 0; r < RPW; ++r)
#pragma unroll
              for (int m = 0; m < NM; ++m)
#pragma unroll
                for (int j = 0; j < GE; ++j) part[r][m][t] = fmaf(wv[r][m][j], xv[j], part[r][m][t]);
          }
        }
      }
      }
#pragma unroll
      for (int r = 0; r < RPW; ++r)
#pragma unroll
        for (int m = 0; m < NM; ++m)
#pragma unroll
          for (int t = 0; t < NT; ++t)
            acc[r][m][t] = WT == WT_INT4 ? fmaf(sc[r][m], part[r][m][t], acc[r][m][t])
                                         : acc[r][m][t] + part[r][m][t];
    }
#pragma unroll
    for (int r = 0; r < RPW; ++r)
#pragma unroll
      for (int t = 0; t < NT; ++t) {
        const float a0 = warp_sum(acc[r][0][t]) * gmat[0];
        const float a1 = GU ? warp_sum(acc[r][NM - 1][t]) * gmat[NM - 1] : 0.f;
        if (lane == 0 && rok[r] && t < nt) {
          const int q = c + t;
          if (GU) hbuf[(size_t)q * I + rbase + r] = silu(a0) * a1;
          else ybuf[(size_t)q * H + rbase + r] = a0;
        }
      }
  }
}

// Launches `kern`; with `dependent`, as a programmatic dependent launch of the
// previous kernel on the stream (it may start before that kernel completes and must
// order itself with griddepcontrol.wait).
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, cudaStream_t s, bool dependent,
                       Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = 0;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = dependent ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, kern, static_cast<KArgs>(args)...);
}

template <int MODE, int WT, int RPW>
cudaError_t launch_gemv(int nt_max, dim3 grid, cudaStream_t s, const void* x, int T, int H, int I, int k,
                        const ExpertList& list, const int* offsets, const int* perm, float* h, float* y) {
#define FT_GEMV_CASE(NTV)                                                                  \
  {                                                                                        \
    return launch_pdl(grouped_gemv_kernel<MODE, WT, NTV, RPW>, grid, dim3(kThreads), s,    \
                      MODE == MODE_DOWN, x, T, H, I, k, list, offsets, perm, h, y);        \
  }
  if (nt_max <= 1) FT_GEMV_CASE(1)
  if (nt_max <= 2 || FT_GEMV_NT_MAX <= 2) FT_GEMV_CASE(2)
  if (nt_max <= 4 || FT_GEMV_NT_MAX <= 4) FT_GEMV_CASE(4)
  FT_GEMV_CASE(8)
#undef FT_GEMV_CASE
}

// out[t][r] = sum_j g[t][j] * y[inv[t*k+j]][r] (+ y[T*k+t][r]); 4 outputs per thread.
template <bool OUT_BF16>
__global__ void combine_kernel(const float* __restrict__ y, const float* __restrict__ gates,
                               const int* __restrict__ inv, int T, int H, int k, int has_shared,
                               void* __restrict__ out) {
  asm volatile("griddepcontrol.wait;" ::: "memory");
  const int per_tok = H / 4;
  const long long idx = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= (long long)T * per_tok) return;
  const int t = (int)(idx / per_tok), r = (int)(idx - (long long)t * per_tok) * 4;
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  for (int j = 0; j < k; ++j) {
    const float g = gates[(size_t)t * k + j];
    const float4 v = *reinterpret_cast<const float4*>(y + (size_t)inv[(size_t)t * k + j] * H + r);
    acc.x = fmaf(g, v.x, acc.x); acc.y = fmaf(g, v.y, acc.y);
    acc.z = fmaf(g, v.z, acc.z); acc.w = fmaf(g, v.w, acc.w);
  }
  if (has_shared) {
    const float4 v = *reinterpret_cast<const float4*>(y + ((size_t)T * k + t) * H + r);
    acc.x += v.x; acc.y += v.y; acc.z += v.z; acc.w += v.w;
  }
  if (OUT_BF16) {
    uint2 o;
    o.x = (uint32_t)f32_to_bf16(acc.x) | ((uint32_t)f32_to_bf16(acc.y) << 16);
    o.y = (uint32_t)f32_to_bf16(acc.z) | ((uint32_t)f32_to_bf16(acc.w) << 16);
    reinterpret_cast<uint2*>(out)[((size_t)t * H + r) / 4] = o;
  } else {
    reinterpret_cast<float4*>(out)[((size_t)t * H + r) / 4] = acc;
  }
}

}  // namespace

// Rows per warp for one matrix pass: enough rows that a warp streams about
// FT_GEMV_WARP_BYTES of weights (short rows need several), at most 8.
#ifndef FT_GEMV_WARP_BYTES
#define FT_GEMV_WARP_BYTES 16384
#endif
static int rows_per_warp(size_t row_bytes_all_matrices, int cap) {
  int r = 1;
  while (r < cap && (size_t)(2 * r) * row_bytes_all_matrices <= FT_GEMV_WARP_BYTES) r *= 2;
  return r;
}

template <int MODE, int WT>
static cudaError_t launch_pass(int nt, int rpw, int rows, cudaStream_t s, const void* x, int T, int H, int I, int k,
                               const ExpertList& list, const int* offsets, const int* perm, float* h, float* y) {
  auto grid = [&](int r) { return dim3((rows + kWarps * r - 1) / (kWarps * r), list.n); };
  switch (rpw) {
    case 1: return launch_gemv<MODE, WT, 1>(nt, grid(1), s, x, T, H, I, k, list, offsets, perm, h, y);
    case 2: return launch_gemv<MODE, WT, 2>(nt, grid(2), s, x, T, H, I, k, list, offsets, perm, h, y);
    case 4: return launch_gemv<MODE, WT, 4>(nt, grid(4), s, x, T, H, I, k, list, offsets, perm, h, y);
    default:
      // packed formats stop at 4 rows per warp (their dequant needs the registers)
      if constexpr (WT == WT_INT4 || WT == WT_NVFP4)
        return launch_gemv<MODE, WT, 4>(nt, grid(4), s, x, T, H, I, k, list, offsets, perm, h, y);
      else
        return launch_gemv<MODE, WT, 8>(nt, grid(8), s, x, T, H, I, k, list, offsets, perm, h, y);
  }
}

cudaError_t launch_ffn_decode(const void* x, int T, int H, int I, int k, int wdtype,
                              const ExpertList& list, int max_pairs_per_expert, const int* offsets,
                              const int* perm, float* h, float* y, cudaStream_t s,
                              cudaEvent_t between, int* err) {
  (void)err;
  if (list.n <= 0 || T <= 0) return cudaSuccess;
  int nt = max_pairs_per_expert < T ? max_pairs_per_expert : T;
  if (nt < 1) nt = 1;
  auto bytes_of = [&](int K) -> size_t {
    return wdtype == WT_F32 ? (size_t)K * 4 : wdtype == WT_BF16 ? (size_t)K * 2 : (size_t)K / 2;
  };
  const int cap = (wdtype == WT_INT4 || wdtype == WT_NVFP4) ? 4 : 8;
  const int r_gu = rows_per_warp(2 * bytes_of(H), cap);   // a gate row and an up row
  const int r_d = rows_per_warp(bytes_of(I), cap);
  cudaError_t e;
#define FT_FFN(WTV)                                                                                        \
  e = launch_pass<MODE_GATE_UP, WTV>(nt, r_gu, I, s, x, T, H, I, k, list, offsets, perm, h, y);            \
  if (e != cudaSuccess) return e;                                                                          \
  if (between) cudaEventRecord(between, s);                                                               \
  return launch_pass<MODE_DOWN, WTV>(nt, r_d, H, s, x, T, H, I, k, list, offsets, perm, h, y);
  if (wdtype == WT_F32) { FT_FFN(WT_F32) }
  if (wdtype == WT_BF16) { FT_FFN(WT_BF16) }
  if (wdtype == WT_NVFP4) { FT_FFN(WT_NVFP4) }
  FT_FFN(WT_INT4)
#undef FT_FFN
}

cudaError_t launch_combine(const float* y, const float* gates, const int* inv, int T, int H, int k,
                           bool has_shared, bool out_bf16, void* out, cudaStream_t s) {
  if (T <= 0) return cudaSuccess;
  const long long n = (long long)T * (H / 4);
  const int threads = 256;
  const unsigned blocks = (unsigned)((n + threads - 1) / threads);
  if (out_bf16)
    return launch_pdl(combine_kernel<true>, dim3(blocks), dim3(threads), s, true, y, gates, inv, T, H, k,
                      (int)has_shared, out);
  else
    return launch_pdl(combine_kernel<false>, dim3(blocks), dim3(threads), s, true, y, gates, inv, T, H, k,
                      (int)has_shared, out);
  return cudaGetLastError();
}

}  // namespace ftk

// Decode GEMV building blocks shared by the per-pass kernels and the fused decode
// FFN kernel: weight formats, 16-byte streaming loads, and the rows of one expert
// for all of its token pairs (gate/up + SwiGLU, or down).
//
// Method ("FreeToken linux", "FreeToken's MoE memory handling"): each activated
// expert runs from the cache slot that holds it; expert FFN h = silu(W_gate x) *
// (W_up x), y = W_down h.  At decode sizes this is a batch of matrix-vector
// products bound by HBM bandwidth: every weight byte is read once per launch.
#pragma once
#include <cuda_fp16.h>

#include "common.cuh"
#include "kernels.hpp"

namespace ftk {
namespace gemv {

enum { WT_F32 = 0, WT_BF16 = 1, WT_INT4 = 2, WT_NVFP4 = 3 };
enum { MODE_GATE_UP = 0, MODE_DOWN = 1 };

#ifndef FT_GEMV_WARPS
#define FT_GEMV_WARPS 4
#endif
#ifndef FT_GEMV_NT_MAX
#define FT_GEMV_NT_MAX 8
#endif
// K steps of a warp's rows unrolled, so that their 16-byte loads are in flight together.
#ifndef FT_GEMV_UNROLL
#define FT_GEMV_UNROLL 2
#endif
constexpr int kWarps = FT_GEMV_WARPS;   // warps per CTA
constexpr int kUnroll = FT_GEMV_UNROLL;
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
// x is bf16 (gate/up of bf16/int4 stacks) or f32; h is f32.  COH: the vector was
// written earlier in the same launch by another CTA, so it is read through L2
// (ld.global.cg) instead of the non-coherent path.
template <typename V>
FT_DEVICE V ldvec(const V* p, bool coh) { return coh ? __ldcg(p) : __ldg(p); }

template <int GE, bool BF16IN, bool COH = false>
FT_DEVICE void ldin(const void* base, int i, float* v) {
  if constexpr (BF16IN) {
    const uint4 a = ldvec(reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(base) + i), COH);
    const uint32_t u[4] = {a.x, a.y, a.z, a.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) { v[2 * j] = bf16lo(u[j]); v[2 * j + 1] = bf16hi(u[j]); }
  } else {
    const float* f = static_cast<const float*>(base) + i;
#pragma unroll
    for (int j = 0; j < GE; j += 4) {
      const float4 a = ldvec(reinterpret_cast<const float4*>(f + j), COH);
      v[j] = a.x; v[j + 1] = a.y; v[j + 2] = a.z; v[j + 3] = a.w;
    }
  }
}

// Rows of one list entry for all of its pairs, NT pairs at a time.  Warp w of the
// CTA owns rows [(rblock*kWarps + w)*RPW, +RPW):
//   MODE_GATE_UP: rows of W_gate and W_up (I rows, K = H), input x[token(q)],
//                 output h[q][r] = silu(W_gate[r].x) * (W_up[r].x)
//   MODE_DOWN:    rows of W_down (H rows, K = I), input h[q], output y[q][r].
// e is the entry's expert (-1: the shared expert, pairs T*k .. T*k+T-1) and blob its
// weights.  Lane l reads 16-byte chunks l, l+32, ... of each row; token vectors come
// through L1 (every warp of the entry reads the same few), or through L2 when COH.
// No shared memory and no block barrier: warps stream independently.
template <int MODE, int WT, int NT, int RPW, bool COH>
FT_DEVICE void gemv_rows(const void* __restrict__ xin, int T, int H, int I, int k, int e,
                         const uint8_t* __restrict__ blob, int rblock, const int* __restrict__ offsets,
                         const int* __restrict__ perm, float* __restrict__ hbuf, float* __restrict__ ybuf) {
  constexpr int EL = WTraits<WT>::EL;
  constexpr bool GU = MODE == MODE_GATE_UP;
  constexpr int NM = GU ? 2 : 1;               // weight matrices per row
  constexpr int GE = WT == WT_F32 ? 4 : 8;     // elements per decode group
  constexpr int NG = EL / GE;                  // groups per chunk
  constexpr bool BF16IN = GU && WT != WT_F32;

  const int K = GU ? H : I;
  const int rows = GU ? I : H;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int rbase = (rblock * kWarps + warp) * RPW;
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

    // One K step of this warp's rows: the 16-byte chunks (and scales) at element kk ...
    auto load_step = [&](int kk, uint4 (&wc)[RPW][NM], float (&sc)[RPW][NM]) {
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
    };
    // ... and their products with the token vectors, added to acc in K order.
    auto compute_step = [&](int kk, const uint4 (&wc)[RPW][NM], const float (&sc)[RPW][NM]) {
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
              if (t < nt) ldin<8, BF16IN, COH>(in[t], kk + 8 * g, xv[t]);
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
                ldin<8, BF16IN, COH>(in[t], kk + 8 * g, xv);
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
              ldin<GE, BF16IN, COH>(in[t], kk + g * GE, xv);
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
    };
    if constexpr (RPW == 1 && (WT == WT_BF16 || WT == WT_F32)) {
      // One row (pair) per warp, the short-list and long-row case: bound by DRAM latency,
      // so up to 8 K steps of loads are issued before the first is used (the summation
      // order, and so every output, is the same as in the loop below).
      constexpr int D = 8;
      for (int kb = lane * EL; kb < K; kb += D * 32 * EL) {
        uint4 wd[D][RPW][NM];
        float sd[D][RPW][NM];
#pragma unroll
        for (int u = 0; u < D; ++u)
          if (kb + u * 32 * EL < K) load_step(kb + u * 32 * EL, wd[u], sd[u]);
#pragma unroll
        for (int u = 0; u < D; ++u)
          if (kb + u * 32 * EL < K) compute_step(kb + u * 32 * EL, wd[u], sd[u]);
      }
    } else {
#pragma unroll kUnroll
      for (int kk = lane * EL; kk < K; kk += 32 * EL) {
        uint4 wc[RPW][NM];
        float sc[RPW][NM];
        load_step(kk, wc, sc);
        compute_step(kk, wc, sc);
      }
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

}  // namespace gemv
}  // namespace ftk

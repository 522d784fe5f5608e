// K1 - router logits and top-k gating.
//
// Method ("FreeToken linux", "FreeToken's MoE memory handling"): the router
// scores every routed expert and activates a few per token (6 of 256 in
// DeepSeek-V4-Flash).  Logits are fp32; the k largest are selected (ties to
// the lower expert index) and their gates are the softmax, or the sigmoid,
// of the selected logits normalised to sum to 1.
#include "common.cuh"
#include "decode_gemv.cuh"
#include "kernels.hpp"

namespace ftk {

namespace {

constexpr int kRouterThreads = 256;
constexpr int kRouterEPB = 2;   // experts per CTA
constexpr int kRouterTPB = 8;   // tokens per CTA

template <typename XT>
FT_DEVICE void load_x4(const XT* x, float v[4]);
template <>
FT_DEVICE void load_x4<float>(const float* x, float v[4]) {
  float4 a = *reinterpret_cast<const float4*>(x);
  v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
}
template <>
FT_DEVICE void load_x4<uint16_t>(const uint16_t* x, float v[4]) {
  uint2 a = *reinterpret_cast<const uint2*>(x);
  v[0] = bf16lo(a.x); v[1] = bf16hi(a.x); v[2] = bf16lo(a.y); v[3] = bf16hi(a.y);
}

// Grid (ceil(E/EPB), ceil(T/TPB)).  Thread i of the CTA owns elements
// [4i + 1024 m, 4i + 1024 m + 4) of the hidden axis; partial sums are reduced
// across the warp by butterfly and across the 8 warps in warp order, so the
// summation order is fixed for a given H.
template <typename XT>
__global__ void __launch_bounds__(kRouterThreads)
router_logits_kernel(const XT* __restrict__ x, const float* __restrict__ w, int T, int H, int E,
                     float* __restrict__ z) {
  __shared__ float part[kRouterThreads / 32][kRouterEPB][kRouterTPB];
  const int e0 = blockIdx.x * kRouterEPB, t0 = blockIdx.y * kRouterTPB;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  float acc[kRouterEPB][kRouterTPB];
#pragma unroll
  for (int i = 0; i < kRouterEPB; ++i)
#pragma unroll
    for (int t = 0; t < kRouterTPB; ++t) acc[i][t] = 0.f;
#pragma unroll 4
  for (int hh = threadIdx.x * 4; hh < H; hh += kRouterThreads * 4) {   // unrolled: loads in flight together
    float wv[kRouterEPB][4];
#pragma unroll
    for (int i = 0; i < kRouterEPB; ++i) {
      if (e0 + i < E) {
        float4 a = *reinterpret_cast<const float4*>(w + (size_t)(e0 + i) * H + hh);
        wv[i][0] = a.x; wv[i][1] = a.y; wv[i][2] = a.z; wv[i][3] = a.w;
      } else {
        wv[i][0] = wv[i][1] = wv[i][2] = wv[i][3] = 0.f;
      }
    }
#pragma unroll
    for (int t = 0; t < kRouterTPB; ++t) {
      if (t0 + t < T) {
        float xv[4];
        load_x4<XT>(x + (size_t)(t0 + t) * H + hh, xv);
#pragma unroll
        for (int i = 0; i < kRouterEPB; ++i)
#pragma unroll
          for (int c = 0; c < 4; ++c) acc[i][t] = fmaf(wv[i][c], xv[c], acc[i][t]);
      }
    }
  }
#pragma unroll
  for (int i = 0; i < kRouterEPB; ++i)
#pragma unroll
    for (int t = 0; t < kRouterTPB; ++t) {
      float v = warp_sum(acc[i][t]);
      if (lane == 0) part[warp][i][t] = v;
    }
  __syncthreads();
  if (threadIdx.x < kRouterEPB * kRouterTPB) {
    int i = threadIdx.x / kRouterTPB, t = threadIdx.x % kRouterTPB;
    if (e0 + i < E && t0 + t < T) {
      float s = 0.f;
      for (int wp = 0; wp < kRouterThreads / 32; ++wp) s += part[wp][i][t];
      z[(size_t)(t0 + t) * E + e0 + i] = s;
    }
  }
}

// One warp per token.  Lane l holds logits e = l + 32 m.  Each of the k rounds
// takes the warp-wide maximum (ties: lower index) among unselected experts.
__global__ void topk_gates_kernel(const float* __restrict__ z, int T, int E, int k, int gating,
                                  int* __restrict__ ids, float* __restrict__ gates) {
  constexpr int kPer = 8;   // E <= 256
  const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5, lane = threadIdx.x & 31;
  if (warp >= T) return;
  float v[kPer];
  bool taken[kPer];
#pragma unroll
  for (int m = 0; m < kPer; ++m) {
    int e = lane + 32 * m;
    v[m] = e < E ? z[(size_t)warp * E + e] : 0.f;
    taken[m] = !(e < E);
  }
  float zsel[16];
  int isel[16];
  for (int r = 0; r < k; ++r) {
    float best = 0.f;
    int bi = 0x7FFFFFFF;
#pragma unroll
    for (int m = 0; m < kPer; ++m) {
      int e = lane + 32 * m;
      if (!taken[m] && (bi == 0x7FFFFFFF || v[m] > best)) { best = v[m]; bi = e; }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      float ob = __shfl_xor_sync(0xFFFFFFFFu, best, o);
      int oi = __shfl_xor_sync(0xFFFFFFFFu, bi, o);
      bool better = (oi != 0x7FFFFFFF) &&
                    (bi == 0x7FFFFFFF || ob > best || (ob == best && oi < bi));
      if (better) { best = ob; bi = oi; }
    }
    zsel[r] = best;
    isel[r] = bi;
#pragma unroll
    for (int m = 0; m < kPer; ++m)
      if (lane + 32 * m == bi) taken[m] = true;
  }
  if (lane == 0) {
    float wsum = 0.f, wv[16];
    for (int r = 0; r < k; ++r) {
      float a = gating == 0 ? expf(zsel[r] - zsel[0]) : 1.0f / (1.0f + expf(-zsel[r]));
      wv[r] = a;
      wsum += a;
    }
    for (int r = 0; r < k; ++r) {
      ids[(size_t)warp * k + r] = isel[r];
      gates[(size_t)warp * k + r] = wv[r] / wsum;
    }
  }
}

// Many tokens: CTA tile of 64 tokens x 64 experts, K step 32 through shared
// memory, 256 threads each owning a 4 x 4 block of logits.  Each logit sums in two
// levels, in a fixed order: a fresh fp32 partial of the 32 products of a K step (fmaf
// in increasing H), added to the logit's accumulator step by step.  The error then grows
// with 32 + H/32 terms rather than H (at H = 7168 a single running sum missed the 2e-6
// relative bound against the float64 sum).
constexpr int RT = 64, RE = 64, RK = 32;
template <typename XT>
__global__ void __launch_bounds__(256)
router_logits_tiled_kernel(const XT* __restrict__ x, const float* __restrict__ w, int T, int H, int E,
                           float* __restrict__ z) {
  __shared__ float xs[RK][RT + 4];
  __shared__ float ws[RK][RE + 4];
  const int t0 = blockIdx.x * RT, e0 = blockIdx.y * RE;
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;   // 16 x 16 threads
  float acc[4][4] = {};
  for (int k0 = 0; k0 < H; k0 += RK) {
    // 64 x 32 of x and of w: 2048 elements each, 8 per thread
    for (int i = threadIdx.x; i < RT * RK; i += 256) {
      const int r = i / RK, c = i % RK;
      float xv = 0.f, wv = 0.f;
      if (t0 + r < T && k0 + c < H) {
        if constexpr (sizeof(XT) == 2) xv = bf16_to_f32(x[(size_t)(t0 + r) * H + k0 + c]);
        else xv = x[(size_t)(t0 + r) * H + k0 + c];
      }
      if (e0 + r < E && k0 + c < H) wv = w[(size_t)(e0 + r) * H + k0 + c];
      xs[c][r] = xv;
      ws[c][r] = wv;
    }
    __syncthreads();
    float part[4][4] = {};
#pragma unroll
    for (int c = 0; c < RK; ++c) {
      float a[4], b[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) { a[i] = xs[c][ty * 4 + i]; b[i] = ws[c][tx * 4 + i]; }
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) part[i][j] = fmaf(a[i], b[j], part[i][j]);
    }
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int j = 0; j < 4; ++j) acc[i][j] += part[i][j];
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int t = t0 + ty * 4 + i, e = e0 + tx * 4 + j;
      if (t < T && e < E) z[(size_t)t * E + e] = acc[i][j];
    }
}

// Many tokens, pipelined: the same 64 x 64 CTA tile, K steps of 32 elements through a
// 3-stage cp.async ring (x rows as stored, bf16 or fp32; router rows fp32).  Thread (tx, ty)
// = (tid % 16, tid / 16) owns logits (t0 + ty + 16 i, e0 + tx + 16 j), i, j < 4, so the 16
// lanes of a half-warp read 16 consecutive router rows; rows are padded by 16 bytes so that
// those 16-byte reads fall on distinct banks.  The two-level sum of router_logits_tiled_kernel
// (a partial per K step of 32, then the accumulator), bit for bit.  Needs H % 32 == 0 and
// 16-byte aligned x and w.  The launcher runs it for fp32 x; bf16 x goes to the tf32 kernel
// below (the template keeps both, so a bf16 instance stays a bit-exact fp32-pipe reference).
constexpr int PT = 64, PE = 64, PK = 32, PS = 3;
template <typename XT>
struct RouterPipe {
  static constexpr int kXRow = PK * (int)sizeof(XT) + 16;   // bytes of one x row in a stage
  static constexpr int kWRow = PK * 4 + 16;
  static constexpr int kStage = PT * kXRow + PE * kWRow;
  static constexpr int kBytes = PS * kStage;
};

template <typename XT>
__global__ void __launch_bounds__(256)
router_logits_pipe_kernel(const XT* __restrict__ x, const float* __restrict__ w, int T, int H, int E,
                          float* __restrict__ z) {
  using P = RouterPipe<XT>;
  extern __shared__ __align__(16) unsigned char rsm[];
  const int t0 = blockIdx.x * PT, e0 = blockIdx.y * PE;
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  const int nk = H / PK;
  const uint32_t base = (uint32_t)__cvta_generic_to_shared(rsm);
  // the 16-byte pieces this thread copies per stage: x rows (PK * sizeof(XT) / 16 pieces
  // each) and router rows (8 pieces each)
  constexpr int XP = PK * (int)sizeof(XT) / 16, WP = PK * 4 / 16;
  auto issue = [&](int ks, int st) {
    const uint32_t sx = base + st * P::kStage, sw = sx + PT * P::kXRow;
    for (int i = threadIdx.x; i < PT * XP; i += 256) {
      const int r = i / XP, c = i % XP;
      const XT* src = x + (size_t)min(t0 + r, T - 1) * H + (size_t)ks * PK + c * (16 / (int)sizeof(XT));
      asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(sx + r * P::kXRow + c * 16), "l"(src) : "memory");
    }
    for (int i = threadIdx.x; i < PE * WP; i += 256) {
      const int r = i / WP, c = i % WP;
      const float* src = w + (size_t)min(e0 + r, E - 1) * H + (size_t)ks * PK + c * 4;
      asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(sw + r * P::kWRow + c * 16), "l"(src) : "memory");
    }
  };
  float acc[4][4];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) acc[i][j] = 0.f;
  for (int s = 0; s < PS - 1; ++s) {
    if (s < nk) issue(s, s);
    asm volatile("cp.async.commit_group;" ::: "memory");
  }
  for (int ks = 0; ks < nk; ++ks) {
    asm volatile("cp.async.wait_group %0;" ::"n"(PS - 2) : "memory");
    __syncthreads();   // stage ks is in for every thread; stage ks - 1 is no longer read
    if (ks + PS - 1 < nk) issue(ks + PS - 1, (ks + PS - 1) % PS);
    asm volatile("cp.async.commit_group;" ::: "memory");
    const unsigned char* sx = rsm + (ks % PS) * P::kStage;
    const unsigned char* sw = sx + PT * P::kXRow;
    float part[4][4];
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int j = 0; j < 4; ++j) part[i][j] = 0.f;
#pragma unroll
    for (int kq = 0; kq < PK; kq += 4) {
      float a[4][4], b[4][4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const unsigned char* row = sx + (ty + 16 * i) * P::kXRow;
        if constexpr (sizeof(XT) == 2) {
          const uint2 v = *reinterpret_cast<const uint2*>(row + kq * 2);
          a[i][0] = bf16lo(v.x); a[i][1] = bf16hi(v.x); a[i][2] = bf16lo(v.y); a[i][3] = bf16hi(v.y);
        } else {
          const float4 v = *reinterpret_cast<const float4*>(row + kq * 4);
          a[i][0] = v.x; a[i][1] = v.y; a[i][2] = v.z; a[i][3] = v.w;
        }
      }
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const float4 v = *reinterpret_cast<const float4*>(sw + (tx + 16 * j) * P::kWRow + kq * 4);
        b[j][0] = v.x; b[j][1] = v.y; b[j][2] = v.z; b[j][3] = v.w;
      }
#pragma unroll
      for (int kk = 0; kk < 4; ++kk)
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
          for (int j = 0; j < 4; ++j) part[i][j] = fmaf(a[i][kk], b[j][kk], part[i][j]);
    }
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int j = 0; j < 4; ++j) acc[i][j] += part[i][j];
  }
  asm volatile("cp.async.wait_group 0;" ::: "memory");
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int t = t0 + ty + 16 * i, e = e0 + tx + 16 * j;
      if (t < T && e < E) z[(size_t)t * E + e] = acc[i][j];
    }
}

// Many tokens with bf16 x, on the tensor cores.  A bf16 value is exact in tf32, and an fp32
// router weight w splits into hi = tf32(w) (round to nearest, ties away) and lo = w - hi,
// exact in fp32, of which the MMA reads the top 11 significant bits: x w = x hi + x lo to
// within 2^-21 of |x w| (lo's truncation).  mma.sync.m16n8k8 (tf32 x tf32, exact products,
// fp32 accumulators) multiplies.  Each K step of 32 sums into a fresh partial (four k8 MMAs,
// hi then lo each), added to the logit's accumulator step by step: the two-level sum of the
// SIMT kernels, though not their rounding.  The CTA tile is 64 tokens x 64 experts, kTfWarps
// warps of (64 / (kTfWarps / 2)) x 32 (MT m16 x 4 n8 MMA tiles); the K steps stream through
// router_logits_pipe_kernel's 3-stage cp.async ring.  Fragments (m16n8k8, tf32), lane (g, t) = (lane / 4, lane % 4):
// a0 = A[g][t], a1 = A[g+8][t], a2 = A[g][t+4], a3 = A[g+8][t+4]; b0 = B[t][g], b1 = B[t+4][g];
// d0, d1 = D[g][2t], D[g][2t+1], d2, d3 = D[g+8][2t], D[g+8][2t+1]; A = x (tokens x k), B[k][n]
// = w[n][k].  Needs H % 32 == 0 and 16-byte aligned x and w.
FT_DEVICE void mma_tf32(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm("mma.sync.aligned.m16n8k8.row.col.f32.tf32.tf32.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
FT_DEVICE void tf32_split(float w, uint32_t& hi, uint32_t& lo) {
  asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(hi) : "f"(w));
  lo = __float_as_uint(w - __uint_as_float(hi));
}

#ifndef FT_ROUTER_TF32_WARPS
#define FT_ROUTER_TF32_WARPS 4
#endif
constexpr int kTfWarps = FT_ROUTER_TF32_WARPS;   // 4 or 8
constexpr int kTfMt = 8 / kTfWarps;              // m16 tiles per warp
__global__ void __launch_bounds__(32 * kTfWarps)
router_logits_tf32_kernel(const uint16_t* __restrict__ x, const float* __restrict__ w, int T, int H, int E,
                          float* __restrict__ z) {
  using P = RouterPipe<uint16_t>;
  extern __shared__ __align__(16) unsigned char rsm[];
  const int t0 = blockIdx.x * PT, e0 = blockIdx.y * PE;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
  const int wm = (warp >> 1) * 16 * kTfMt, wn = (warp & 1) * 32;   // the warp's tokens and experts in the tile
  const int nk = H / PK;
  const uint32_t base = (uint32_t)__cvta_generic_to_shared(rsm);
  constexpr int XP = PK * 2 / 16, WP = PK * 4 / 16;   // 16-byte pieces of an x row, a router row
  auto issue = [&](int ks, int st) {
    const uint32_t sx = base + st * P::kStage, sw = sx + PT * P::kXRow;
    for (int i = threadIdx.x; i < PT * XP; i += 32 * kTfWarps) {
      const int r = i / XP, c = i % XP;
      const uint16_t* src = x + (size_t)min(t0 + r, T - 1) * H + (size_t)ks * PK + c * 8;
      asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(sx + r * P::kXRow + c * 16), "l"(src) : "memory");
    }
    for (int i = threadIdx.x; i < PE * WP; i += 32 * kTfWarps) {
      const int r = i / WP, c = i % WP;
      const float* src = w + (size_t)min(e0 + r, E - 1) * H + (size_t)ks * PK + c * 4;
      asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(sw + r * P::kWRow + c * 16), "l"(src) : "memory");
    }
  };
  float acc[kTfMt][4][4];
#pragma unroll
  for (int i = 0; i < kTfMt; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) acc[i][j][0] = acc[i][j][1] = acc[i][j][2] = acc[i][j][3] = 0.f;
  for (int s = 0; s < PS - 1; ++s) {
    if (s < nk) issue(s, s);
    asm volatile("cp.async.commit_group;" ::: "memory");
  }
  for (int ks = 0; ks < nk; ++ks) {
    asm volatile("cp.async.wait_group %0;" ::"n"(PS - 2) : "memory");
    __syncthreads();   // stage ks is in for every thread; stage ks - 1 is no longer read
    if (ks + PS - 1 < nk) issue(ks + PS - 1, (ks + PS - 1) % PS);
    asm volatile("cp.async.commit_group;" ::: "memory");
    const unsigned char* sx = rsm + (ks % PS) * P::kStage;
    const unsigned char* sw = sx + PT * P::kXRow;
    float part[kTfMt][4][4];
#pragma unroll
    for (int i = 0; i < kTfMt; ++i)
#pragma unroll
      for (int j = 0; j < 4; ++j) part[i][j][0] = part[i][j][1] = part[i][j][2] = part[i][j][3] = 0.f;
#pragma unroll
    for (int k0 = 0; k0 < PK; k0 += 8) {
      uint32_t a[kTfMt][4];
#pragma unroll
      for (int i = 0; i < kTfMt; ++i) {
        const unsigned short* r0 = reinterpret_cast<const unsigned short*>(sx + (wm + 16 * i + g) * P::kXRow) + k0 + t;
        const unsigned short* r1 = reinterpret_cast<const unsigned short*>(sx + (wm + 16 * i + g + 8) * P::kXRow) + k0 + t;
        a[i][0] = (uint32_t)r0[0] << 16;
        a[i][1] = (uint32_t)r1[0] << 16;
        a[i][2] = (uint32_t)r0[4] << 16;
        a[i][3] = (uint32_t)r1[4] << 16;
      }
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const float* wr = reinterpret_cast<const float*>(sw + (wn + 8 * j + g) * P::kWRow) + k0 + t;
        uint32_t h0, l0, h1, l1;
        tf32_split(wr[0], h0, l0);
        tf32_split(wr[4], h1, l1);
#pragma unroll
        for (int i = 0; i < kTfMt; ++i) {
          mma_tf32(part[i][j], a[i], h0, h1);
          mma_tf32(part[i][j], a[i], l0, l1);
        }
      }
    }
#pragma unroll
    for (int i = 0; i < kTfMt; ++i)
#pragma unroll
      for (int j = 0; j < 4; ++j)
#pragma unroll
        for (int c = 0; c < 4; ++c) acc[i][j][c] += part[i][j][c];
  }
  asm volatile("cp.async.wait_group 0;" ::: "memory");
#pragma unroll
  for (int i = 0; i < kTfMt; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j)
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const int tok = t0 + wm + 16 * i + g + 8 * (c >> 1), e = e0 + wn + 8 * j + 2 * t + (c & 1);
        if (tok < T && e < E) z[(size_t)tok * E + e] = acc[i][j][c];
      }
}

// Decode routing in one launch: the router CTAs of router_logits_kernel write
// their logits; the last CTA to finish (a __threadfence + atomic ticket, no
// waiting) then runs top-k + gates for every token and the stable permutation
// of the T*k pairs, and resets the ticket for the next launch.
template <typename XT>
__global__ void __launch_bounds__(kRouterThreads)
route_decode_kernel(const XT* __restrict__ x, const float* __restrict__ w, int T, int H, int E, int k,
                    int gating, float* __restrict__ z, int* __restrict__ ids, float* __restrict__ gates,
                    int* __restrict__ counts, int* __restrict__ offsets, int* __restrict__ perm,
                    int* __restrict__ inv, int* __restrict__ ticket, int* __restrict__ box, int seq,
                    const int* __restrict__ err) {
  __shared__ float part[kRouterThreads / 32][kRouterEPB][kRouterTPB];
  __shared__ int last;
  __shared__ int s_cnt[256], s_base[256], s_wc[kRouterThreads / 32][256], s_wsum[kRouterThreads / 32];
  __shared__ int s_ids[64 * 16];
  const int e0 = blockIdx.x * kRouterEPB, t0 = blockIdx.y * kRouterTPB;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // Launched as a programmatic dependent of the previous kernel on the stream: the
  // router rows do not depend on it, so they are brought toward L2 first (one prefetch
  // per 128-byte line); everything the previous kernel may write or read (x, the
  // routing buffers, the ticket) is touched only after griddepcontrol.wait.
  for (int i = 0; i < kRouterEPB; ++i)
    if (e0 + i < E)
      for (int hh = threadIdx.x * 32; hh < H; hh += kRouterThreads * 32)
        asm volatile("prefetch.global.L2 [%0];" ::"l"(__cvta_generic_to_global(w + (size_t)(e0 + i) * H + hh)));
  asm volatile("griddepcontrol.wait;" ::: "memory");
  {  // ---- logits of this CTA's experts and tokens (as router_logits_kernel)
    float acc[kRouterEPB][kRouterTPB];
#pragma unroll
    for (int i = 0; i < kRouterEPB; ++i)
#pragma unroll
      for (int t = 0; t < kRouterTPB; ++t) acc[i][t] = 0.f;
#pragma unroll 4
    for (int hh = threadIdx.x * 4; hh < H; hh += kRouterThreads * 4) {   // unrolled: loads in flight together
      float wv[kRouterEPB][4];
#pragma unroll
      for (int i = 0; i < kRouterEPB; ++i) {
        if (e0 + i < E) {
          float4 a = *reinterpret_cast<const float4*>(w + (size_t)(e0 + i) * H + hh);
          wv[i][0] = a.x; wv[i][1] = a.y; wv[i][2] = a.z; wv[i][3] = a.w;
        } else {
          wv[i][0] = wv[i][1] = wv[i][2] = wv[i][3] = 0.f;
        }
      }
#pragma unroll
      for (int t = 0; t < kRouterTPB; ++t) {
        if (t0 + t < T) {
          float xv[4];
          load_x4<XT>(x + (size_t)(t0 + t) * H + hh, xv);
#pragma unroll
          for (int i = 0; i < kRouterEPB; ++i)
#pragma unroll
            for (int c = 0; c < 4; ++c) acc[i][t] = fmaf(wv[i][c], xv[c], acc[i][t]);
        }
      }
    }
#pragma unroll
    for (int i = 0; i < kRouterEPB; ++i)
#pragma unroll
      for (int t = 0; t < kRouterTPB; ++t) {
        if (t0 + t < T) {   // the same for the whole CTA: the shuffles stay warp-uniform
          float v = warp_sum(acc[i][t]);
          if (lane == 0) part[warp][i][t] = v;
        }
      }
    __syncthreads();
    if (threadIdx.x < kRouterEPB * kRouterTPB) {
      int i = threadIdx.x / kRouterTPB, t = threadIdx.x % kRouterTPB;
      if (e0 + i < E && t0 + t < T) {
        float sum = 0.f;
        for (int wp = 0; wp < kRouterThreads / 32; ++wp) sum += part[wp][i][t];
        z[(size_t)(t0 + t) * E + e0 + i] = sum;
      }
      __threadfence();   // the logit writers publish before the ticket
    }
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    const int nblocks = gridDim.x * gridDim.y;
    last = atomicAdd(ticket, 1) == nblocks - 1;
  }
  __syncthreads();
  if (!last) return;
  if (warp < T) __threadfence();   // the warps that read the logits
  // ---- top-k + gates: one warp per token, logits read through L2
  for (int t = warp; t < T; t += kRouterThreads / 32) {
    float v[8];
    bool taken[8];
#pragma unroll
    for (int m = 0; m < 8; ++m) {
      const int e = lane + 32 * m;
      v[m] = e < E ? __ldcg(z + (size_t)t * E + e) : 0.f;
      taken[m] = !(e < E);
    }
    float zsel[16];
    int isel[16];
    for (int r = 0; r < k; ++r) {
      float best = 0.f;
      int bi = 0x7FFFFFFF;
#pragma unroll
      for (int m = 0; m < 8; ++m) {
        const int e = lane + 32 * m;
        if (!taken[m] && (bi == 0x7FFFFFFF || v[m] > best)) { best = v[m]; bi = e; }
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        const float ob = __shfl_xor_sync(0xFFFFFFFFu, best, o);
        const int oi = __shfl_xor_sync(0xFFFFFFFFu, bi, o);
        const bool better = (oi != 0x7FFFFFFF) && (bi == 0x7FFFFFFF || ob > best || (ob == best && oi < bi));
        if (better) { best = ob; bi = oi; }
      }
      zsel[r] = best;
      isel[r] = bi;
#pragma unroll
      for (int m = 0; m < 8; ++m)
        if (lane + 32 * m == bi) taken[m] = true;
    }
    if (lane == 0) {
      float wsum = 0.f, wv[16];
      for (int r = 0; r < k; ++r) {
        const float a = gating == 0 ? expf(zsel[r] - zsel[0]) : 1.0f / (1.0f + expf(-zsel[r]));
        wv[r] = a;
        wsum += a;
      }
      for (int r = 0; r < k; ++r) {
        ids[(size_t)t * k + r] = isel[r];
        gates[(size_t)t * k + r] = wv[r] / wsum;
        s_ids[t * k + r] = isel[r];
      }
    }
  }
  // ---- stable counting sort of the n = T*k pairs by expert (n <= 1024)
  const int n = T * k;
  for (int e = threadIdx.x; e < E; e += kRouterThreads) s_cnt[e] = 0;
  __syncthreads();
  for (int p = threadIdx.x; p < n; p += kRouterThreads) atomicAdd(&s_cnt[s_ids[p]], 1);
  __syncthreads();
  {  // exclusive scan of the E <= 256 counts: one per thread, warp scans, then warp totals
    const int c = threadIdx.x < E ? s_cnt[threadIdx.x] : 0;
    int incl = c;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int v = __shfl_up_sync(0xFFFFFFFFu, incl, o);
      if (lane >= o) incl += v;
    }
    if (lane == 31) s_wsum[warp] = incl;
    __syncthreads();
    int before = 0;
    for (int w2 = 0; w2 < warp; ++w2) before += s_wsum[w2];
    if (threadIdx.x < E) {
      s_base[threadIdx.x] = before + incl - c;
      counts[threadIdx.x] = c;
      offsets[threadIdx.x] = before + incl - c;
    }
    if (threadIdx.x == 0) offsets[E] = n;
  }
  __syncthreads();
  const unsigned lt = (1u << lane) - 1u;
  if (n <= 32) {
    // one warp: a pair's place is its expert's base + its rank among equal keys
    if (warp == 0) {
      const int e = lane < n ? s_ids[lane] : -1;
      const unsigned mask = __match_any_sync(0xFFFFFFFFu, e);
      if (e >= 0) {
        const int q = s_base[e] + __popc(mask & lt);
        perm[q] = lane;
        inv[lane] = q;
      }
    }
  } else {
    for (int c = 0; c < n; c += kRouterThreads) {
      for (int i = threadIdx.x; i < (kRouterThreads / 32) * E; i += kRouterThreads) s_wc[i / E][i % E] = 0;
      __syncthreads();
      const int p = c + threadIdx.x;
      const int e = p < n ? s_ids[p] : -1;
      const unsigned mask = __match_any_sync(0xFFFFFFFFu, e);
      const int rank = __popc(mask & lt);
      if (e >= 0 && rank == 0) s_wc[warp][e] = __popc(mask);
      __syncthreads();
      if (e >= 0) {
        int before = 0;
        for (int w2 = 0; w2 < warp; ++w2) before += s_wc[w2][e];
        const int q = s_base[e] + before + rank;
        perm[q] = p;
        inv[p] = q;
      }
      __syncthreads();
      for (int ee = threadIdx.x; ee < E; ee += kRouterThreads) {
        int sum = 0;
        for (int w2 = 0; w2 < kRouterThreads / 32; ++w2) sum += s_wc[w2][ee];
        s_base[ee] += sum;
      }
      __syncthreads();
    }
  }
  if (box) {
    // publish to the host through mapped pinned memory: every word carries the call's
    // tag (seq, 1 .. 2^21-1) above a 10-bit value (an id, or the device error word), so
    // the host takes the words once all of them show the tag, whatever order they
    // arrive in; no system-scope fence is needed.
    const int tag = seq << 10;
    volatile int* vb = reinterpret_cast<volatile int*>(box);
    for (int p = threadIdx.x; p < n; p += kRouterThreads) vb[2 + p] = tag | s_ids[p];
    if (threadIdx.x == 0) vb[1] = tag | (*reinterpret_cast<const volatile int*>(err) & 0x3FF);
  }
  if (threadIdx.x == 0) *ticket = 0;
}

}  // namespace

cudaError_t launch_router_logits_tiled(const void* x, bool x_bf16, const float* w_router, int T, int H,
                                       int E, float* logits, cudaStream_t s) {
  if (T <= 0) return cudaSuccess;
  const bool aligned = ((reinterpret_cast<uintptr_t>(x) | reinterpret_cast<uintptr_t>(w_router)) & 15) == 0;
  if (H % PK == 0 && aligned) {
    dim3 pgrid((T + PT - 1) / PT, (E + PE - 1) / PE);
    if (x_bf16) {
      auto kern = router_logits_tf32_kernel;
      cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, RouterPipe<uint16_t>::kBytes);
      if (e != cudaSuccess) return e;
      kern<<<pgrid, 32 * kTfWarps, RouterPipe<uint16_t>::kBytes, s>>>(static_cast<const uint16_t*>(x), w_router, T, H, E,
                                                                       logits);
    } else {
      auto kern = router_logits_pipe_kernel<float>;
      cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, RouterPipe<float>::kBytes);
      if (e != cudaSuccess) return e;
      kern<<<pgrid, 256, RouterPipe<float>::kBytes, s>>>(static_cast<const float*>(x), w_router, T, H, E, logits);
    }
    return cudaGetLastError();
  }
  dim3 grid((T + RT - 1) / RT, (E + RE - 1) / RE);
  if (x_bf16)
    router_logits_tiled_kernel<uint16_t><<<grid, 256, 0, s>>>(static_cast<const uint16_t*>(x), w_router, T, H,
                                                              E, logits);
  else
    router_logits_tiled_kernel<float><<<grid, 256, 0, s>>>(static_cast<const float*>(x), w_router, T, H, E,
                                                           logits);
  return cudaGetLastError();
}

cudaError_t launch_route_decode(const void* x, bool x_bf16, const float* w_router, int T, int H, int E, int k,
                                int gating, float* logits, int* ids, float* gates, int* counts, int* offsets,
                                int* perm, int* inv, int* ticket, cudaStream_t s, int* box, int seq,
                                const int* err) {
  if (T <= 0) return cudaSuccess;
  if (T > 64 || E > 256 || k > 16) return cudaErrorInvalidValue;
  dim3 grid((E + kRouterEPB - 1) / kRouterEPB, (T + kRouterTPB - 1) / kRouterTPB);
  // programmatic dependent launch: may start while the previous kernel (the last forward's
  // combine) finishes; the kernel orders itself with griddepcontrol.wait
  if (x_bf16)
    return gemv::launch_pdl(route_decode_kernel<uint16_t>, grid, dim3(kRouterThreads), s, true,
                            static_cast<const uint16_t*>(x), w_router, T, H, E, k, gating, logits, ids, gates, counts,
                            offsets, perm, inv, ticket, box, seq, err);
  return gemv::launch_pdl(route_decode_kernel<float>, grid, dim3(kRouterThreads), s, true,
                          static_cast<const float*>(x), w_router, T, H, E, k, gating, logits, ids, gates, counts,
                          offsets, perm, inv, ticket, box, seq, err);
}

cudaError_t launch_router_logits(const void* x, bool x_bf16, const float* w_router, int T, int H,
                                 int E, float* logits, cudaStream_t s) {
  if (T <= 0) return cudaSuccess;
  dim3 grid((E + kRouterEPB - 1) / kRouterEPB, (T + kRouterTPB - 1) / kRouterTPB);
  if (x_bf16)
    router_logits_kernel<uint16_t><<<grid, kRouterThreads, 0, s>>>(
        static_cast<const uint16_t*>(x), w_router, T, H, E, logits);
  else
    router_logits_kernel<float><<<grid, kRouterThreads, 0, s>>>(static_cast<const float*>(x),
                                                               w_router, T, H, E, logits);
  return cudaGetLastError();
}

cudaError_t launch_topk_gates(const float* logits, int T, int E, int k, int gating, int* ids,
                              float* gates, cudaStream_t s) {
  if (T <= 0) return cudaSuccess;
  const int threads = 256, warps = threads / 32;
  topk_gates_kernel<<<(T + warps - 1) / warps, threads, 0, s>>>(logits, T, E, k, gating, ids,
                                                               gates);
  return cudaGetLastError();
}

}  // namespace ftk

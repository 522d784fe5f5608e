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
#include "common.cuh"
#include "kernels.hpp"

namespace ftk {

namespace {

enum { WT_F32 = 0, WT_BF16 = 1, WT_INT4 = 2 };
enum { MODE_GATE_UP = 0, MODE_DOWN = 1 };

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;

// Elements held by one 16-byte weight load.
template <int WT> struct WTraits;
template <> struct WTraits<WT_F32>  { static constexpr int EL = 4; };
template <> struct WTraits<WT_BF16> { static constexpr int EL = 8; };
template <> struct WTraits<WT_INT4> { static constexpr int EL = 32; };

// Shared-memory position of input element i.  For int4 the 32 elements of one
// lane's load are spread so that, for each of the load's four 8-element words,
// the 32 lanes read 32 consecutive 16-byte cells (no bank conflicts).
template <int WT>
FT_DEVICE int spos(int i) {
  if (WT != WT_INT4) return i;
  int blk = i >> 10, r = i & 1023;
  return (blk << 10) + (((r & 31) >> 3) << 8) + ((r >> 5) << 3) + (r & 7);
}

// Weight chunk -> EL fp32 values (int4: the raw integers; the group scale is
// applied to the chunk's partial sum).
template <int WT>
FT_DEVICE void decode_chunk(const uint4& c, float* v);
template <>
FT_DEVICE void decode_chunk<WT_F32>(const uint4& c, float* v) {
  v[0] = __uint_as_float(c.x); v[1] = __uint_as_float(c.y);
  v[2] = __uint_as_float(c.z); v[3] = __uint_as_float(c.w);
}
template <>
FT_DEVICE void decode_chunk<WT_BF16>(const uint4& c, float* v) {
  const uint32_t w[4] = {c.x, c.y, c.z, c.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) { v[2 * i] = bf16lo(w[i]); v[2 * i + 1] = bf16hi(w[i]); }
}
template <>
FT_DEVICE void decode_chunk<WT_INT4>(const uint4& c, float* v) {
  const uint32_t w[4] = {c.x, c.y, c.z, c.w};
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int n = 0; n < 8; ++n) v[8 * i + n] = (float)(((int32_t)(w[i] << (28 - 4 * n))) >> 28);
}

// Input element type in shared memory: x (f32 or bf16) for gate/up, h (f32) for down.
template <int MODE, int WT> struct InT { using T = float; };
template <> struct InT<MODE_GATE_UP, WT_BF16> { using T = uint16_t; };
template <> struct InT<MODE_GATE_UP, WT_INT4> { using T = uint16_t; };

FT_DEVICE float in_val(const float* p, int i) { return p[i]; }
FT_DEVICE float in_val(const uint16_t* p, int i) { return bf16_to_f32(p[i]); }

// Reads EL consecutive logical input elements starting at kk (a multiple of EL).
template <int WT, typename IT>
FT_DEVICE void load_in(const IT* s, int kk, float* v) {
  constexpr int EL = WTraits<WT>::EL;
  if constexpr (WT == WT_INT4) {
#pragma unroll
    for (int w = 0; w < 4; ++w) {
      const int base = spos<WT>(kk + 8 * w);   // 8 contiguous cells
      if constexpr (sizeof(IT) == 2) {
        uint4 a = *reinterpret_cast<const uint4*>(s + base);
        const uint32_t u[4] = {a.x, a.y, a.z, a.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) { v[8 * w + 2 * i] = bf16lo(u[i]); v[8 * w + 2 * i + 1] = bf16hi(u[i]); }
      } else {
        float4 a = *reinterpret_cast<const float4*>(s + base);
        float4 b = *reinterpret_cast<const float4*>(s + base + 4);
        v[8 * w + 0] = a.x; v[8 * w + 1] = a.y; v[8 * w + 2] = a.z; v[8 * w + 3] = a.w;
        v[8 * w + 4] = b.x; v[8 * w + 5] = b.y; v[8 * w + 6] = b.z; v[8 * w + 7] = b.w;
      }
    }
  } else if constexpr (sizeof(IT) == 2) {   // EL = 8 bf16
    uint4 a = *reinterpret_cast<const uint4*>(s + kk);
    const uint32_t u[4] = {a.x, a.y, a.z, a.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) { v[2 * i] = bf16lo(u[i]); v[2 * i + 1] = bf16hi(u[i]); }
  } else {
#pragma unroll
    for (int i = 0; i < EL; i += 4) {
      float4 a = *reinterpret_cast<const float4*>(s + kk + i);
      v[i] = a.x; v[i + 1] = a.y; v[i + 2] = a.z; v[i + 3] = a.w;
    }
  }
}

// Grouped GEMV.  Grid (ceil(rows / (kWarps*RPW)), list.n).  CTA (bx, i) handles
// rows [bx*kWarps*RPW, ...) of list entry i for up to NT of its pairs at a time:
//   MODE_GATE_UP: rows of W_gate and W_up (I rows, K = H), input x[token(q)],
//                 output h[q][r] = silu(W_gate[r].x) * (W_up[r].x)
//   MODE_DOWN:    rows of W_down (H rows, K = I), input h[q], output y[q][r].
template <int MODE, int WT, int NT, int RPW>
__global__ void __launch_bounds__(kThreads)
grouped_gemv_kernel(const void* __restrict__ xin, int T, int H, int I, int k,
                    const __grid_constant__ ExpertList list, const int* __restrict__ offsets,
                    const int* __restrict__ perm, float* __restrict__ hbuf,
                    float* __restrict__ ybuf) {
  using IT = typename InT<MODE, WT>::T;
  constexpr int EL = WTraits<WT>::EL;
  constexpr bool GU = MODE == MODE_GATE_UP;
  constexpr int NM = GU ? 2 : 1;    // weight matrices per row
  extern __shared__ __align__(16) unsigned char smem_raw[];
  IT* sx = reinterpret_cast<IT*>(smem_raw);

  const int entry = blockIdx.y;
  const int e = list.expert[entry];
  const uint8_t* blob = list.blob[entry];
  const int q0 = e >= 0 ? offsets[e] : T * k;
  const int q1 = e >= 0 ? offsets[e + 1] : T * k + T;
  if (q1 <= q0) return;
  const int K = GU ? H : I;
  const int rows = GU ? I : H;
  const int Kpad = WT == WT_INT4 ? ((K + 1023) & ~1023) : K;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int rbase = blockIdx.x * kWarps * RPW + warp * RPW;

  // weight matrix bases within the blob
  const size_t mat = (size_t)H * I;
  const uint8_t* wmat[2];
  const uint16_t* smat[2] = {nullptr, nullptr};
  if (WT == WT_INT4) {
    const uint16_t* sc = reinterpret_cast<const uint16_t*>(blob + 3 * mat / 2);
    if (GU) { wmat[0] = blob; wmat[1] = blob + mat / 2; smat[0] = sc; smat[1] = sc + mat / 128; }
    else { wmat[0] = blob + mat; wmat[1] = nullptr; smat[0] = sc + 2 * (mat / 128); }
  } else {
    constexpr int es = WT == WT_F32 ? 4 : 2;
    if (GU) { wmat[0] = blob; wmat[1] = blob + mat * es; }
    else { wmat[0] = blob + 2 * mat * es; wmat[1] = nullptr; }
  }
  const size_t row_bytes = WT == WT_INT4 ? (size_t)K / 2 : (size_t)K * (WT == WT_F32 ? 4 : 2);

  for (int c = q0; c < q1; c += NT) {
    const int nt = min(NT, q1 - c);
    // stage the inputs of pairs c .. c+nt-1
    for (int idx = threadIdx.x; idx < nt * K; idx += kThreads) {
      const int t = idx / K, i = idx - t * K;
      const int q = c + t;
      IT v;
      if (GU) {
        const int tok = e >= 0 ? perm[q] / k : q - T * k;
        v = reinterpret_cast<const IT*>(xin)[(size_t)tok * H + i];
      } else {
        v = reinterpret_cast<const IT*>(hbuf)[(size_t)q * I + i];
      }
      sx[t * Kpad + spos<WT>(i)] = v;
    }
    __syncthreads();
    float acc[RPW][NM][NT];
#pragma unroll
    for (int r = 0; r < RPW; ++r)
#pragma unroll
      for (int m = 0; m < NM; ++m)
#pragma unroll
        for (int t = 0; t < NT; ++t) acc[r][m][t] = 0.f;
    bool rok[RPW];
#pragma unroll
    for (int r = 0; r < RPW; ++r) rok[r] = rbase + r < rows;
#pragma unroll 2
    for (int kk = lane * EL; kk < K; kk += 32 * EL) {
      uint4 wc[RPW][NM];
#pragma unroll
      for (int r = 0; r < RPW; ++r)
#pragma unroll
        for (int m = 0; m < NM; ++m)
          wc[r][m] = rok[r] ? ld_stream16(wmat[m] + (size_t)(rbase + r) * row_bytes +
                                          (WT == WT_INT4 ? kk / 2 : kk * (WT == WT_F32 ? 4 : 2)))
                            : make_uint4(0, 0, 0, 0);
      float sc[RPW][NM];
      if (WT == WT_INT4) {
#pragma unroll
        for (int r = 0; r < RPW; ++r)
#pragma unroll
          for (int m = 0; m < NM; ++m)
            sc[r][m] = rok[r] ? bf16_to_f32(smat[m][(size_t)(rbase + r) * (K / 128) + kk / 128]) : 0.f;
      }
#pragma unroll
      for (int t = 0; t < NT; ++t) {
        if (t < nt) {
          float xv[EL];
          load_in<WT, IT>(sx + t * Kpad, kk, xv);
#pragma unroll
          for (int r = 0; r < RPW; ++r)
#pragma unroll
            for (int m = 0; m < NM; ++m) {
              float wv[EL];
              decode_chunk<WT>(wc[r][m], wv);
              float p = 0.f;
#pragma unroll
              for (int j = 0; j < EL; ++j) p = fmaf(wv[j], xv[j], p);
              if (WT == WT_INT4) acc[r][m][t] = fmaf(sc[r][m], p, acc[r][m][t]);
              else acc[r][m][t] += p;
            }
        }
      }
    }
#pragma unroll
    for (int r = 0; r < RPW; ++r)
#pragma unroll
      for (int t = 0; t < NT; ++t) {
        float a0 = warp_sum(acc[r][0][t]);
        float a1 = GU ? warp_sum(acc[r][NM - 1][t]) : 0.f;
        if (lane == 0 && rok[r] && t < nt) {
          const int q = c + t;
          if (GU) hbuf[(size_t)q * I + rbase + r] = silu(a0) * a1;
          else ybuf[(size_t)q * H + rbase + r] = a0;
        }
      }
    __syncthreads();
  }
}

template <int MODE, int WT, int RPW>
cudaError_t launch_gemv(int nt_max, dim3 grid, size_t smem, cudaStream_t s, const void* x, int T,
                        int H, int I, int k, const ExpertList& list, const int* offsets,
                        const int* perm, float* h, float* y) {
#define FT_GEMV_CASE(NTV)                                                                         \
  {                                                                                               \
    auto kern = grouped_gemv_kernel<MODE, WT, NTV, RPW>;                                          \
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,       \
                                         (int)smem);                                              \
    if (e != cudaSuccess) return e;                                                               \
    kern<<<grid, kThreads, smem, s>>>(x, T, H, I, k, list, offsets, perm, h, y);                  \
    return cudaGetLastError();                                                                    \
  }
  if (nt_max <= 1) FT_GEMV_CASE(1)
  if (nt_max <= 2) FT_GEMV_CASE(2)
  if (nt_max <= 4) FT_GEMV_CASE(4)
  FT_GEMV_CASE(8)
#undef FT_GEMV_CASE
}

// out[t][r] = sum_j g[t][j] * y[inv[t*k+j]][r] (+ y[T*k+t][r]); 4 outputs per thread.
template <bool OUT_BF16>
__global__ void combine_kernel(const float* __restrict__ y, const float* __restrict__ gates,
                               const int* __restrict__ inv, int T, int H, int k, int has_shared,
                               void* __restrict__ out) {
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

cudaError_t launch_ffn_decode(const void* x, int T, int H, int I, int k, int wdtype,
                              const ExpertList& list, int max_pairs_per_expert, const int* offsets,
                              const int* perm, float* h, float* y, cudaStream_t s,
                              cudaEvent_t between) {
  if (list.n <= 0 || T <= 0) return cudaSuccess;
  int nt = max_pairs_per_expert < T ? max_pairs_per_expert : T;
  if (nt < 1) nt = 1;
  const int NTcap = nt <= 1 ? 1 : nt <= 2 ? 2 : nt <= 4 ? 4 : 8;
  constexpr int RPW_GU = 2, RPW_D = 4;
  dim3 g1((I + kWarps * RPW_GU - 1) / (kWarps * RPW_GU), list.n);
  dim3 g2((H + kWarps * RPW_D - 1) / (kWarps * RPW_D), list.n);
  cudaError_t e;
  if (wdtype == WT_F32) {
    size_t s1 = (size_t)NTcap * H * 4, s2 = (size_t)NTcap * I * 4;
    e = launch_gemv<MODE_GATE_UP, WT_F32, RPW_GU>(nt, g1, s1, s, x, T, H, I, k, list, offsets, perm, h, y);
    if (e != cudaSuccess) return e;
    if (between) cudaEventRecord(between, s);
    return launch_gemv<MODE_DOWN, WT_F32, RPW_D>(nt, g2, s2, s, x, T, H, I, k, list, offsets, perm, h, y);
  } else if (wdtype == WT_BF16) {
    size_t s1 = (size_t)NTcap * H * 2, s2 = (size_t)NTcap * I * 4;
    e = launch_gemv<MODE_GATE_UP, WT_BF16, RPW_GU>(nt, g1, s1, s, x, T, H, I, k, list, offsets, perm, h, y);
    if (e != cudaSuccess) return e;
    if (between) cudaEventRecord(between, s);
    return launch_gemv<MODE_DOWN, WT_BF16, RPW_D>(nt, g2, s2, s, x, T, H, I, k, list, offsets, perm, h, y);
  } else {
    size_t s1 = (size_t)NTcap * ((H + 1023) & ~1023) * 2, s2 = (size_t)NTcap * ((I + 1023) & ~1023) * 4;
    e = launch_gemv<MODE_GATE_UP, WT_INT4, RPW_GU>(nt, g1, s1, s, x, T, H, I, k, list, offsets, perm, h, y);
    if (e != cudaSuccess) return e;
    if (between) cudaEventRecord(between, s);
    return launch_gemv<MODE_DOWN, WT_INT4, RPW_D>(nt, g2, s2, s, x, T, H, I, k, list, offsets, perm, h, y);
  }
}

cudaError_t launch_combine(const float* y, const float* gates, const int* inv, int T, int H, int k,
                           bool has_shared, bool out_bf16, void* out, cudaStream_t s) {
  if (T <= 0) return cudaSuccess;
  const long long n = (long long)T * (H / 4);
  const int threads = 256;
  const unsigned blocks = (unsigned)((n + threads - 1) / threads);
  if (out_bf16)
    combine_kernel<true><<<blocks, threads, 0, s>>>(y, gates, inv, T, H, k, has_shared, out);
  else
    combine_kernel<false><<<blocks, threads, 0, s>>>(y, gates, inv, T, H, k, has_shared, out);
  return cudaGetLastError();
}

}  // namespace ftk

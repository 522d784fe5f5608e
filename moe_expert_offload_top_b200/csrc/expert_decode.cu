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
// exactly once per launch with 16-byte streaming loads; the few token vectors
// of an expert come through L1.  These are the per-pass kernels (gate/up, down,
// combine as three launches); ffn_fused.cuh runs the three in one launch.
#include "decode_gemv.cuh"

namespace ftk {

namespace {

using namespace gemv;

// Grouped GEMV, one matrix pass.  Grid (ceil(rows / (kWarps*RPW)), list.n): CTA (bx, i)
// runs row block bx of list entry i (gemv_rows).
template <int MODE, int WT, int NT, int RPW>
__global__ void __launch_bounds__(kThreads)
grouped_gemv_kernel(const void* __restrict__ xin, int T, int H, int I, int k,
                    const __grid_constant__ ExpertList list, const int* __restrict__ offsets,
                    const int* __restrict__ perm, float* __restrict__ hbuf,
                    float* __restrict__ ybuf) {
  // Programmatic dependent launch: the down projection may be launched while this
  // gate/up grid runs; it waits for this grid's completion before it reads h.
  if (MODE == MODE_GATE_UP) asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  else asm volatile("griddepcontrol.wait;" ::: "memory");
  gemv_rows<MODE, WT, NT, RPW, false>(xin, T, H, I, k, list.expert[blockIdx.y], list.blob[blockIdx.y],
                                      blockIdx.x, offsets, perm, hbuf, ybuf);
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
  // the next forward's routing kernel may launch now (it waits for this grid itself)
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
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

// Which decode GEMV runs: the tensor-core kernels where their shapes allow, else the
// per-row GEMV on the fp32 pipes.  bf16 uses the tensor cores from 2 tokens on: with one
// token the per-row GEMV streams the weights faster (at dsv4flash shapes gate/up took 44.8
// against 50.7 us per launch), with 8 it is 2.6 times slower.
enum { kPathRows = 0, kPathInt4Mma = 1, kPathNvfp4Mma = 2, kPathBf16Mma = 3 };
static int decode_path(int wdtype, bool tensor, int H, int I, int T) {
  if (!tensor) return kPathRows;
  if (wdtype == WT_INT4) return kPathInt4Mma;
  if (wdtype == WT_NVFP4 && H % 128 == 0 && I % 128 == 0) return kPathNvfp4Mma;   // whole groups of 128
  if (wdtype == WT_BF16 && T >= 2 && H % 32 == 0 && I % 32 == 0) return kPathBf16Mma;
  return kPathRows;
}

int ffn_decode_kernels(int wdtype, bool int4_tensor, int H, int I, int T) {
  switch (decode_path(wdtype, int4_tensor, H, I, T)) {
    case kPathInt4Mma:
    case kPathNvfp4Mma:
      return 4;   // token slicing, gate/up, h slicing, down
    case kPathBf16Mma:
      return 3;   // gate/up, h split, down
    default:
      return 2;   // gate/up, down
  }
}

cudaError_t launch_ffn_decode(const void* x, int T, int H, int I, int k, int wdtype,
                              const ExpertList& list, int max_pairs_per_expert, const int* offsets,
                              const int* perm, float* h, float* y, cudaStream_t s,
                              cudaEvent_t between, int* err, bool int4_tensor, void* int4_xs) {
  (void)err;
  if (list.n <= 0 || T <= 0) return cudaSuccess;
  switch (decode_path(wdtype, int4_tensor, H, I, T)) {
    case kPathInt4Mma:
      return launch_ffn_int4_mma(x, T, H, I, k, list, offsets, perm, h, y, s, between, max_pairs_per_expert, int4_xs);
    case kPathNvfp4Mma:
      return launch_ffn_nvfp4_mma(x, T, H, I, k, list, offsets, perm, h, y, s, between, max_pairs_per_expert, int4_xs);
    case kPathBf16Mma:
      return launch_ffn_bf16_mma(x, T, H, I, k, list, offsets, perm, h, y, s, between, max_pairs_per_expert);
    default:
      break;
  }
  int nt = max_pairs_per_expert < T ? max_pairs_per_expert : T;
  if (nt < 1) nt = 1;
  auto bytes_of = [&](int K) -> size_t {
    return wdtype == WT_F32 ? (size_t)K * 4 : wdtype == WT_BF16 ? (size_t)K * 2 : (size_t)K / 2;
  };
  const int cap = (wdtype == WT_INT4 || wdtype == WT_NVFP4) ? 4 : 8;
  // Short lists (the experts copied in by this call, say) give few CTAs: fewer rows per
  // warp then, down to one, until the pass has at least two CTAs per SM.
  static const int sms = [] {
    int d = 0, n = 148;
    cudaGetDevice(&d);
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, d);
    return n > 0 ? n : 148;
  }();
  auto widen = [&](int r, int rows) {
    while (r > 1 && (long long)list.n * ((rows + kWarps * r - 1) / (kWarps * r)) < 2LL * sms) r >>= 1;
    return r;
  };
  const int r_gu = widen(rows_per_warp(2 * bytes_of(H), cap), I);   // a gate row and an up row
  const int r_d = widen(rows_per_warp(bytes_of(I), cap), H);
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

int ffn_fused_ctl_ints(int H) { return 2 + kMaxList + (H + 2 * kWarps - 1) / (2 * kWarps); }

#ifndef FT_FUSED_GU_CAP
#define FT_FUSED_GU_CAP 4
#endif
#ifndef FT_FUSED_D_CAP
#define FT_FUSED_D_CAP 8
#endif

cudaError_t launch_ffn_fused(const FusedParams& p, int wdtype, const ExpertList& list, int max_pairs_per_expert,
                             int num_sms, cudaStream_t s) {
  if (list.n <= 0 || p.T <= 0) return cudaSuccess;
  int nt = max_pairs_per_expert < p.T ? max_pairs_per_expert : p.T;
  if (nt < 1) nt = 1;
  auto bytes_of = [&](int K) -> size_t {
    return wdtype == WT_F32 ? (size_t)K * 4 : wdtype == WT_BF16 ? (size_t)K * 2 : (size_t)K / 2;
  };
  const bool packed = wdtype == WT_INT4 || wdtype == WT_NVFP4;
  const int rg = rows_per_warp(2 * bytes_of(p.H), FT_FUSED_GU_CAP);
  int rd = rows_per_warp(bytes_of(p.I), packed && FT_FUSED_D_CAP > 4 ? 4 : FT_FUSED_D_CAP);
  if (rd < 2) rd = 2;   // the counter block holds ceil(H / (2 * kWarps)) down row blocks
  switch (wdtype) {
    case WT_F32: return launch_ffn_fused_f32(nt, rg, rd, p, list, num_sms, s);
    case WT_BF16: return launch_ffn_fused_bf16(nt, rg, rd, p, list, num_sms, s);
    case WT_INT4: return launch_ffn_fused_int4(nt, rg, rd, p, list, num_sms, s);
    case WT_NVFP4: return launch_ffn_fused_nvfp4(nt, rg, rd, p, list, num_sms, s);
    default: return cudaErrorInvalidValue;
  }
}

namespace {
__global__ void hold_kernel(const volatile int* flag, int want, unsigned long long limit_ns) {
  unsigned long long t0, t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t0));
  for (unsigned it = 0; it < (1u << 24); ++it) {
    if (*flag >= want) return;
    __nanosleep(256);
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    if (t - t0 > limit_ns) return;
  }
}
}  // namespace

cudaError_t launch_hold(const volatile int* flag, int want, unsigned long long limit_ns, cudaStream_t s) {
  hold_kernel<<<1, 1, 0, s>>>(flag, want, limit_ns);
  return cudaGetLastError();
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

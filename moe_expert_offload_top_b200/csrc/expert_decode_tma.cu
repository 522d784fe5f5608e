// K3 (decode) fed by bulk copies: the expert weights stream from the cache
// slots into shared memory through the TMA engine, so each SM keeps ~100-190 KB
// of weight bytes in flight at almost no register cost, and the arithmetic
// reads them from shared memory.
//
// Method ("FreeToken linux", "FreeToken's MoE memory handling"): every selected
// expert runs from the slot that holds it; at decode sizes the expert FFN is a
// batch of matrix-vector products bound by HBM bandwidth.
//
// Work: the rows of every list entry are cut into row blocks of U = 8*RPWARP
// rows (gate/up: a row is the gate row and the up row), each row block into
// K slices that fit one stage.  The CTAs of the grid (one per SM) take balanced
// contiguous ranges of row blocks; the (row block, K slice) chunks of a CTA run
// through a 3-stage ring:
//   warp 8 lane 0  producer: per chunk, one cp.async.bulk per (row, matrix) of the
//                  slice (and its int4 scales), completing on the stage's barrier;
//   warps 0..7     consumers: warp w owns rows w, w+8, ... of the block, reads
//                  16-byte chunks of its rows from shared memory, the token
//                  vectors through L1, accumulates across the slices of the block
//                  in registers and stores h (SwiGLU) or y at the last slice.
// Every wait is bounded (sm100_sync.cuh).
#include "common.cuh"
#include "kernels.hpp"
#include "sm100_sync.cuh"

namespace ftk {

namespace {

enum { TWT_F32 = 0, TWT_BF16 = 1, TWT_INT4 = 2 };
constexpr int TG_CONSUMERS = 8;
constexpr int TG_THREADS = (TG_CONSUMERS + 1) * 32;
constexpr int TG_STAGES = 3;
constexpr int TG_STAGE_BYTES = 64 * 1024;

static __device__ int g_tma_gemv_err;   // error word when the caller passes none

struct TgSmem {
  uint64_t full[TG_STAGES], empty[TG_STAGES];
  int abort;
};

template <int WT> struct TgTraits;
template <> struct TgTraits<TWT_F32>  { static constexpr int EL = 4;  static constexpr int NUM = 4, DEN = 1; };
template <> struct TgTraits<TWT_BF16> { static constexpr int EL = 8;  static constexpr int NUM = 2, DEN = 1; };
template <> struct TgTraits<TWT_INT4> { static constexpr int EL = 32; static constexpr int NUM = 1, DEN = 2; };

FT_DEVICE void bulk_load(void* dst, const void* src, uint32_t bytes, uint64_t* bar, uint64_t policy) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint [%0], [%1], %2, [%3], %4;"
      ::"r"(smem_u32(dst)), "l"(src), "r"(bytes), "r"(smem_u32(bar)), "l"(policy)
      : "memory");
}

FT_DEVICE uint64_t evict_first_policy() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
  return p;
}

template <int WT>
FT_DEVICE void tg_group(const uint4& c, int g, float* v) {
  const uint32_t w[4] = {c.x, c.y, c.z, c.w};
  if constexpr (WT == TWT_F32) {
#pragma unroll
    for (int i = 0; i < 4; ++i) v[i] = __uint_as_float(w[i]);
  } else if constexpr (WT == TWT_BF16) {
#pragma unroll
    for (int i = 0; i < 4; ++i) { v[2 * i] = bf16lo(w[i]); v[2 * i + 1] = bf16hi(w[i]); }
  } else {
#pragma unroll
    for (int n = 0; n < 8; ++n) v[n] = (float)(((int32_t)(w[g] << (28 - 4 * n))) >> 28);
  }
}

template <int GE, bool BF16IN>
FT_DEVICE void tg_in(const void* base, int i, float* v) {
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

template <int MODE, int WT, int NT, int RPWARP>
__global__ void __launch_bounds__(TG_THREADS, 1)
gemv_tma_kernel(const void* __restrict__ xin, int T, int H, int I, int k, const __grid_constant__ ExpertList list,
                const int* __restrict__ offsets, const int* __restrict__ perm, float* __restrict__ hbuf,
                float* __restrict__ ybuf, int KC, int n_slices, int* err_word) {
  constexpr bool GU = MODE == 0;
  constexpr int NM = GU ? 2 : 1;
  constexpr int EL = TgTraits<WT>::EL;
  constexpr int GE = WT == TWT_F32 ? 4 : 8;
  constexpr int NG = EL / GE;
  constexpr bool BF16IN = GU && WT != TWT_F32;
  constexpr int U = 8 * RPWARP;
  extern __shared__ __align__(128) unsigned char tg_smem[];
  TgSmem* S = reinterpret_cast<TgSmem*>(tg_smem + TG_STAGES * TG_STAGE_BYTES);
  int* err = err_word ? err_word : &g_tma_gemv_err;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int K = GU ? H : I;
  const int rows = GU ? I : H;
  const int bpe = (rows + U - 1) / U;                 // row blocks per entry
  const int n_blocks = bpe * list.n;
  const int b0 = (int)((long long)n_blocks * blockIdx.x / gridDim.x);
  const int b1 = (int)((long long)n_blocks * (blockIdx.x + 1) / gridDim.x);
  const int n_chunks = (b1 - b0) * n_slices;
  const size_t mat = (size_t)H * I;
  // bytes per K element of one row of one matrix, as num/den; scales: 2 bytes per 128
  const size_t row_bytes = (size_t)K * TgTraits<WT>::NUM / TgTraits<WT>::DEN;
  const int kc_bytes = KC * TgTraits<WT>::NUM / TgTraits<WT>::DEN;   // one row slice in smem
  const int sc_bytes = WT == TWT_INT4 ? KC / 128 * 2 : 0;
  const int w_region = U * NM * kc_bytes;                               // weights of a stage

  if (threadIdx.x == 0) {
    for (int s = 0; s < TG_STAGES; ++s) { mbar_init(&S->full[s], 1); mbar_init(&S->empty[s], TG_CONSUMERS); }
    S->abort = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncthreads();
  volatile int* abort_flag = &S->abort;

  auto matrix_base = [&](const uint8_t* blob, int m, const uint8_t*& w, const uint16_t*& sc) {
    if (WT == TWT_INT4) {
      const uint16_t* s0 = reinterpret_cast<const uint16_t*>(blob + 3 * mat / 2);
      w = GU ? blob + (m ? mat / 2 : 0) : blob + mat;
      sc = GU ? s0 + (m ? mat / 128 : 0) : s0 + 2 * (mat / 128);
    } else {
      constexpr int es = WT == TWT_F32 ? 4 : 2;
      w = GU ? blob + (m ? mat * es : 0) : blob + 2 * mat * es;
      sc = nullptr;
    }
  };

  if (warp == TG_CONSUMERS) {
    if (lane == 0) {   // --------------------------------------------------- producer
      const uint64_t pol = evict_first_policy();
      int c = 0;
      for (; c < n_chunks && !*abort_flag; ++c) {
        const int s = c % TG_STAGES;
        if (!mbar_wait(&S->empty[s], ((c / TG_STAGES) & 1) ^ 1, abort_flag, err, 301)) break;
        const int blk = b0 + c / n_slices, sl = c - (c / n_slices) * n_slices;
        const int entry = blk / bpe;
        const int row0 = (blk - entry * bpe) * U;
        const int nrows = min(U, rows - row0);
        const int k0 = sl * KC;
        const int kc = min(KC, K - k0);
        const int kcb = kc * TgTraits<WT>::NUM / TgTraits<WT>::DEN;
        const int scb = WT == TWT_INT4 ? kc / 128 * 2 : 0;
        unsigned char* st = tg_smem + s * TG_STAGE_BYTES;
        mbar_expect_tx(&S->full[s], (uint32_t)(nrows * NM * (kcb + scb)));
        const uint8_t* blob = list.blob[entry];
        for (int m = 0; m < NM; ++m) {
          const uint8_t* wb;
          const uint16_t* sb;
          matrix_base(blob, m, wb, sb);
          for (int r = 0; r < nrows; ++r) {
            const uint8_t* src = wb + (size_t)(row0 + r) * row_bytes + (size_t)k0 * TgTraits<WT>::NUM / TgTraits<WT>::DEN;
            bulk_load(st + (m * U + r) * kc_bytes, src, (uint32_t)kcb, &S->full[s], pol);
            if (WT == TWT_INT4)
              bulk_load(st + w_region + (m * U + r) * sc_bytes, sb + (size_t)(row0 + r) * (K / 128) + k0 / 128,
                        (uint32_t)scb, &S->full[s], pol);
          }
        }
      }
      for (int j = c - TG_STAGES < 0 ? 0 : c - TG_STAGES; j < c; ++j)
        mbar_drain(&S->full[j % TG_STAGES], (j / TG_STAGES) & 1);
    }
  } else {               // --------------------------------------------------- consumers
    float acc[RPWARP][NM][NT];
    const void* in[NT];
    int q0 = 0, nt = 0;
    for (int c = 0; c < n_chunks && !*abort_flag; ++c) {
      const int s = c % TG_STAGES;
      const int blk = b0 + c / n_slices, sl = c - (c / n_slices) * n_slices;
      const int entry = blk / bpe;
      const int row0 = (blk - entry * bpe) * U;
      const int nrows = min(U, rows - row0);
      if (sl == 0) {      // new row block: token vectors of the entry, zero accumulators
        const int e = list.expert[entry];
        q0 = e >= 0 ? offsets[e] : T * k;
        const int q1 = e >= 0 ? offsets[e + 1] : T * k + T;
        nt = min(NT, q1 - q0);
#pragma unroll
        for (int t = 0; t < NT; ++t) {
          const int q = q0 + (t < nt ? t : 0);
          if (GU) {
            const int tok = e >= 0 ? perm[q] / k : q - T * k;
            in[t] = BF16IN ? (const void*)(static_cast<const uint16_t*>(xin) + (size_t)tok * H)
                           : (const void*)(static_cast<const float*>(xin) + (size_t)tok * H);
          } else {
            in[t] = hbuf + (size_t)q * I;
          }
        }
#pragma unroll
        for (int r = 0; r < RPWARP; ++r)
#pragma unroll
          for (int m = 0; m < NM; ++m)
#pragma unroll
            for (int t = 0; t < NT; ++t) acc[r][m][t] = 0.f;
      }
      if (!mbar_wait(&S->full[s], (c / TG_STAGES) & 1, abort_flag, err, 302)) break;
      const unsigned char* st = tg_smem + s * TG_STAGE_BYTES;
      const int k0 = sl * KC;
      const int kc = min(KC, K - k0);
#pragma unroll
      for (int j = 0; j < RPWARP; ++j) {
        const int r = warp + 8 * j;
        if (r < nrows) {
          for (int kk = lane * EL; kk < kc; kk += 32 * EL) {
            float part[NM][NT];
#pragma unroll
            for (int m = 0; m < NM; ++m)
#pragma unroll
              for (int t = 0; t < NT; ++t) part[m][t] = 0.f;
            uint4 wc[NM];
            float sc[NM];
#pragma unroll
            for (int m = 0; m < NM; ++m) {
              wc[m] = *reinterpret_cast<const uint4*>(st + (m * U + r) * kc_bytes +
                                                      kk * TgTraits<WT>::NUM / TgTraits<WT>::DEN);
              sc[m] = WT == TWT_INT4
                          ? bf16_to_f32(reinterpret_cast<const uint16_t*>(st + w_region + (m * U + r) * sc_bytes)[kk / 128])
                          : 1.f;
            }
            if constexpr (WT == TWT_INT4) {
              // Packed dequant: nibble pairs (n, n+4) of a word become the bf16x2 values
              // q + 136 with one mask/xor/or (0x4300 is 128.0 in bf16, whose last
              // mantissa bit is 1.0; xor 8 maps two's-complement q to q + 8), widen
              // exactly to fp32 pairs, lose the 136 exactly in one packed add, and meet
              // the matching x pairs in packed fp32 FMAs.
              float2 acc2[NM][NT];
#pragma unroll
              for (int m = 0; m < NM; ++m)
#pragma unroll
                for (int t = 0; t < NT; ++t) acc2[m][t] = make_float2(0.f, 0.f);
              const float2 bias = make_float2(-136.f, -136.f);
#pragma unroll
              for (int g = 0; g < 4; ++g) {
                float2 xp[NT][4];
#pragma unroll
                for (int t = 0; t < NT; ++t)
                  if (t < nt) {
                    const uint4 a = __ldg(reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(in[t]) + k0 + kk + 8 * g));
                    xp[t][0] = make_float2(bf16lo(a.x), bf16lo(a.z));
                    xp[t][1] = make_float2(bf16hi(a.x), bf16hi(a.z));
                    xp[t][2] = make_float2(bf16lo(a.y), bf16lo(a.w));
                    xp[t][3] = make_float2(bf16hi(a.y), bf16hi(a.w));
                  }
#pragma unroll
                for (int m = 0; m < NM; ++m) {
                  const uint32_t w = g == 0 ? wc[m].x : g == 1 ? wc[m].y : g == 2 ? wc[m].z : wc[m].w;
#pragma unroll
                  for (int n = 0; n < 4; ++n) {
                    const uint32_t v = ((w >> (4 * n)) & 0x000F000Fu) ^ 0x43084308u;
                    const float2 q2 = __fadd2_rn(make_float2(bf16lo(v), bf16hi(v)), bias);
#pragma unroll
                    for (int t = 0; t < NT; ++t)
                      if (t < nt) acc2[m][t] = __ffma2_rn(q2, xp[t][n], acc2[m][t]);
                  }
                }
              }
#pragma unroll
              for (int m = 0; m < NM; ++m)
#pragma unroll
                for (int t = 0; t < NT; ++t) part[m][t] = acc2[m][t].x + acc2[m][t].y;
            } else {
#pragma unroll
            for (int g = 0; g < NG; ++g) {
              float xv[NT][GE];
#pragma unroll
              for (int t = 0; t < NT; ++t)
                if (t < nt) tg_in<GE, BF16IN>(in[t], k0 + kk + g * GE, xv[t]);
#pragma unroll
              for (int m = 0; m < NM; ++m) {
                float wv[GE];
                tg_group<WT>(wc[m], g, wv);
#pragma unroll
                for (int t = 0; t < NT; ++t)
                  if (t < nt) {
#pragma unroll
                    for (int e2 = 0; e2 < GE; ++e2) part[m][t] = fmaf(wv[e2], xv[t][e2], part[m][t]);
                  }
              }
            }
            }
#pragma unroll
            for (int m = 0; m < NM; ++m)
#pragma unroll
              for (int t = 0; t < NT; ++t)
                acc[j][m][t] = WT == TWT_INT4 ? fmaf(sc[m], part[m][t], acc[j][m][t]) : acc[j][m][t] + part[m][t];
          }
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&S->empty[s]);
      if (sl == n_slices - 1) {   // the block's last slice: reduce and store
#pragma unroll
        for (int j = 0; j < RPWARP; ++j) {
          const int r = warp + 8 * j;
#pragma unroll
          for (int t = 0; t < NT; ++t) {
            const float a0 = warp_sum(acc[j][0][t]);
            const float a1 = GU ? warp_sum(acc[j][NM - 1][t]) : 0.f;
            if (lane == 0 && r < nrows && t < nt) {
              const int q = q0 + t;
              if (GU) hbuf[(size_t)q * I + row0 + r] = silu(a0) * a1;
              else ybuf[(size_t)q * H + row0 + r] = a0;
            }
          }
        }
      }
    }
  }
  __syncthreads();
}

template <int MODE, int WT, int RPWARP>
cudaError_t launch_tma(int nt, int grid, int KC, int n_slices, cudaStream_t s, const void* x, int T, int H, int I,
                       int k, const ExpertList& list, const int* offsets, const int* perm, float* h, float* y,
                       int* err) {
  const size_t smem = (size_t)TG_STAGES * TG_STAGE_BYTES + sizeof(TgSmem);
#define FT_TG_CASE(NTV)                                                                                     \
  {                                                                                                         \
    auto kern = gemv_tma_kernel<MODE, WT, NTV, RPWARP>;                                                     \
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);     \
    if (e != cudaSuccess) return e;                                                                         \
    kern<<<grid, TG_THREADS, smem, s>>>(x, T, H, I, k, list, offsets, perm, h, y, KC, n_slices, err);       \
    return cudaGetLastError();                                                                              \
  }
  if (nt <= 1) FT_TG_CASE(1)
  if (nt <= 2) FT_TG_CASE(2)
  if (nt <= 4) FT_TG_CASE(4)
  FT_TG_CASE(8)
#undef FT_TG_CASE
}

// Shape of one matrix pass: rows per warp (1, 2, 4 or 8) and K slice such that a stage
// (U rows x NM matrices x slice, plus int4 scales) fits TG_STAGE_BYTES.
template <int MODE, int WT>
cudaError_t launch_pass(int nt, int num_sms, cudaStream_t s, const void* x, int T, int H, int I, int k,
                        const ExpertList& list, const int* offsets, const int* perm, float* h, float* y,
                        int* err) {
  constexpr int NM = MODE == 0 ? 2 : 1;
  constexpr int EL = TgTraits<WT>::EL;
  const int K = MODE == 0 ? H : I;
  const int rows = MODE == 0 ? I : H;
  // bytes of one row of one matrix for `kc` K elements, plus its scales
  auto row_slice_bytes = [&](int kc) { return kc * TgTraits<WT>::NUM / TgTraits<WT>::DEN + (WT == TWT_INT4 ? kc / 64 : 0); };
  int rpw = 1;
  while (rpw < 8 && 8 * (rpw * 2) * NM * row_slice_bytes(K) <= TG_STAGE_BYTES && 8 * rpw * 2 <= rows) rpw *= 2;
  const int U = 8 * rpw;
  const int step = WT == TWT_INT4 ? 1024 : 32 * EL;   // K granularity: lane chunks (int4: 16-byte scale runs)
  // largest multiple of `step` whose stage (U rows x NM matrices x slice, with scales) fits
  const double per_elem = (double)TgTraits<WT>::NUM / TgTraits<WT>::DEN + (WT == TWT_INT4 ? 2.0 / 128 : 0.0);
  int KC = (int)((double)TG_STAGE_BYTES / (U * NM * per_elem));
  KC = (KC / step) * step;
  if (KC < step) KC = step;
  if (KC >= K) KC = K;
  const int n_slices = (K + KC - 1) / KC;
  const long long blocks = (long long)((rows + U - 1) / U) * list.n;
  const int grid = (int)(blocks < num_sms ? blocks : num_sms);
  switch (rpw) {
    case 1: return launch_tma<MODE, WT, 1>(nt, grid, KC, n_slices, s, x, T, H, I, k, list, offsets, perm, h, y, err);
    case 2: return launch_tma<MODE, WT, 2>(nt, grid, KC, n_slices, s, x, T, H, I, k, list, offsets, perm, h, y, err);
    case 4: return launch_tma<MODE, WT, 4>(nt, grid, KC, n_slices, s, x, T, H, I, k, list, offsets, perm, h, y, err);
    default: return launch_tma<MODE, WT, 8>(nt, grid, KC, n_slices, s, x, T, H, I, k, list, offsets, perm, h, y, err);
  }
}

}  // namespace

bool tma_gemv_supported(int H, int I, int wdtype) {
  // bulk copies need 16-byte aligned rows and slices
  if (wdtype == TWT_INT4) return H % 1024 == 0 && I % 1024 == 0;
  const int eb = wdtype == TWT_F32 ? 4 : 2;
  return (H * eb) % 16 == 0 && (I * eb) % 16 == 0;
}

cudaError_t launch_ffn_decode_tma(const void* x, int T, int H, int I, int k, int wdtype, const ExpertList& list,
                                  int nt, const int* offsets, const int* perm, float* h, float* y, int* err,
                                  int num_sms, cudaStream_t s, cudaEvent_t between) {
  if (list.n <= 0 || T <= 0) return cudaSuccess;
  cudaError_t e;
#define FT_TG_FFN(WTV)                                                                                 \
  e = launch_pass<0, WTV>(nt, num_sms, s, x, T, H, I, k, list, offsets, perm, h, y, err);              \
  if (e != cudaSuccess) return e;                                                                      \
  if (between) cudaEventRecord(between, s);                                                            \
  return launch_pass<1, WTV>(nt, num_sms, s, x, T, H, I, k, list, offsets, perm, h, y, err);
  if (wdtype == TWT_F32) { FT_TG_FFN(TWT_F32) }
  if (wdtype == TWT_BF16) { FT_TG_FFN(TWT_BF16) }
  FT_TG_FFN(TWT_INT4)
#undef FT_TG_FFN
}

}  // namespace ftk

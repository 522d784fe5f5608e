// K3 for decode with int4 (group-128) expert weights, on the tensor cores.
//
// Method ("FreeToken linux", "FreeToken's MoE memory handling"): each selected expert
// runs from its cache slot; h = silu(W_gate x) * (W_up x), y = W_down h, with int4
// weights w = q * s (q a two's-complement nibble, s the bf16 scale of 128 consecutive
// reduction-axis elements of one row; the low nibble of a byte holds the even element).
//
// Why tensor cores for a matrix-vector product.  On the FP32 pipes an int4 weight costs
// about five instructions (unpack, widen, offset, multiply-add), so the GEMV is bound by
// instruction issue, not by HBM.  Here the unpack is two instructions per weight pair
// and the multiply-adds go to mma.sync.m16n8k16 (bf16 in, fp32 accumulate), which also
// covers up to 8 tokens of an expert at once.  The operands stay in registers:
// tcgen05.mma would take the dequantised weights from shared memory, i.e. twice the
// HBM bytes again through shared memory, for an M of at most 8 tokens.
//
// Tile: a CTA owns 16 output rows of W_gate and W_up together, or 16*RT rows of W_down
// (RT row tiles share each input fragment and the offset MMAs), of one expert; its 4
// warps split the reduction axis into contiguous ranges of 128-element groups and their
// partial sums are added in warp order through shared memory.
//
// Fragments.  Lane (g, t) = (lane / 4, lane % 4).  For one 128-element group, lane
// (g, t) loads 16 bytes (32 nibbles, elements 32t .. 32t+31) of rows g and g+8.  Word j
// of that chunk holds elements k0 .. k0+7 (k0 = 32t + 8j); the pair (k0+n, k0+n+4) of
// nibbles n and n+4 becomes one bf16x2 register: ((w >> 4n) & 0x000F000F) ^ 0x43084308
// is the bf16 pair (136 + q).  The MMA's reduction index is a permutation of the
// physical one (the same for weights and inputs): MMA 2j takes pairs n = 0, 1, MMA 2j+1
// pairs n = 2, 3, and the input fragment is built from the same element pairs with
// byte permutes.  The offset 136 is removed per group by one more MMA against a
// constant fragment of -136, so each group's partial sum is sum(q x) exactly as far as
// fp32 accumulation goes; it is then scaled by the group's s and accumulated.
//
// Down projection: its input h is fp32.  The gate/up kernel stores each h value as two
// bf16 (hi = bf16(h), lo = bf16(h - hi)) in the same row of the h buffer, and the down
// kernel runs its MMAs on both, so h keeps 16 bits of mantissa (relative error 2^-17).
#include "decode_gemv.cuh"

namespace ftk {

namespace {

using namespace gemv;

constexpr int kQWarps = 4;
constexpr int kQThreads = 32 * kQWarps;
#ifndef FT_INT4_MMA_UNROLL
#define FT_INT4_MMA_UNROLL 2
#endif
#ifndef FT_INT4_MMA_DOWN_TILES
#define FT_INT4_MMA_DOWN_TILES 2
#endif
constexpr int kQUnroll = FT_INT4_MMA_UNROLL;         // 128-element groups of loads in flight
constexpr int kDownTiles = FT_INT4_MMA_DOWN_TILES;   // 16-row tiles per CTA in the down pass
constexpr uint32_t kNeg136x2 = 0xC308C308u;   // bf16 pair (-136, -136)

// d (16x8 f32) += A (16x16 bf16) * B (16x8 bf16).
FT_DEVICE void mma16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3, uint32_t b0,
                        uint32_t b1) {
  asm("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// Nibbles n and n+4 of w as the bf16 pair (136 + q_n, 136 + q_{n+4}).
FT_DEVICE uint32_t nib2(uint32_t w, int n) { return ((w >> (4 * n)) & 0x000F000Fu) ^ 0x43084308u; }

FT_DEVICE uint32_t word_of(const uint4& v, int j) { return j == 0 ? v.x : j == 1 ? v.y : j == 2 ? v.z : v.w; }

// Input pairs (e_n, e_{n+4}), n = 0..3, of 8 consecutive bf16 elements held in v.
FT_DEVICE void in_pairs(const uint4& v, uint32_t (&p)[4]) {
  p[0] = __byte_perm(v.x, v.z, 0x5410);
  p[1] = __byte_perm(v.x, v.z, 0x7632);
  p[2] = __byte_perm(v.y, v.w, 0x5410);
  p[3] = __byte_perm(v.y, v.w, 0x7632);
}

// MODE 0: gate/up + SwiGLU into h (bf16 hi/lo per value); MODE 1: down into y (f32).
// Grid (ceil(rows / (16 * tiles)), list.n), 128 threads.
template <int MODE>
__global__ void __launch_bounds__(kQThreads)
int4_mma_kernel(const uint16_t* __restrict__ x, int T, int H, int I, int k, const __grid_constant__ ExpertList list,
                const int* __restrict__ offsets, const int* __restrict__ perm, float* __restrict__ hbuf,
                float* __restrict__ ybuf) {
  constexpr bool GU = MODE == 0;
  constexpr int NM = GU ? 2 : kDownTiles;   // 16x(K) weight tiles per CTA: gate and up, or down row tiles
  __shared__ float red[kQWarps][NM][16][8];
  const int e = list.expert[blockIdx.y];
  const uint8_t* blob = list.blob[blockIdx.y];
  const int K = GU ? H : I, rows = GU ? I : H;
  const int row0 = blockIdx.x * (GU ? 16 : 16 * kDownTiles);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
  const size_t mat = (size_t)H * I;
  const uint16_t* sc = reinterpret_cast<const uint16_t*>(blob + 3 * mat / 2);
  const size_t row_bytes = (size_t)K / 2;
  const int nb = K / 128;                                       // scale groups per row
  // tile m: weight rows rA[m], rB[m] (this lane's g and g+8) of matrix wm[m], scales sm[m]
  const uint8_t* wm[NM];
  const uint16_t* sm[NM];
  int rA[NM], rB[NM];
  if constexpr (GU) {
    wm[0] = blob; wm[1] = blob + mat / 2;
    sm[0] = sc; sm[1] = sc + mat / 128;
    rA[0] = rA[1] = min(row0 + g, rows - 1);
    rB[0] = rB[1] = min(row0 + g + 8, rows - 1);
  } else {
#pragma unroll
    for (int m = 0; m < NM; ++m) {
      wm[m] = blob + mat;
      sm[m] = sc + 2 * (mat / 128);
      rA[m] = min(row0 + 16 * m + g, rows - 1);
      rB[m] = min(row0 + 16 * m + g + 8, rows - 1);
    }
  }
  const int b0 = warp * nb / kQWarps, b1 = (warp + 1) * nb / kQWarps;
  if (GU) asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  else asm volatile("griddepcontrol.wait;" ::: "memory");
  const int q0 = e >= 0 ? offsets[e] : T * k;
  const int q1 = e >= 0 ? offsets[e + 1] : T * k + T;
  if (q1 <= q0 || row0 >= rows) return;   // the same for the whole CTA

  for (int c0 = q0; c0 < q1; c0 += 8) {
    const int nt = min(8, q1 - c0);
    const bool colv = g < nt;                                   // this lane's input column
    const uint16_t* src = x;
    if (colv) {
      const int q = c0 + g;
      if constexpr (GU) {
        const int tok = e >= 0 ? perm[q] / k : q - T * k;
        src = x + (size_t)tok * H;
      } else {
        src = reinterpret_cast<const uint16_t*>(hbuf + (size_t)q * I);   // hi at [0, I), lo at [I, 2I)
      }
    }
    float acc[NM][4];
#pragma unroll
    for (int m = 0; m < NM; ++m) acc[m][0] = acc[m][1] = acc[m][2] = acc[m][3] = 0.f;

#pragma unroll kQUnroll
    for (int blk = b0; blk < b1; ++blk) {
      uint4 wa[NM], wb[NM];
      float s[NM][2];
#pragma unroll
      for (int m = 0; m < NM; ++m) {
        wa[m] = ldw(wm[m] + (size_t)rA[m] * row_bytes + (size_t)blk * 64 + t * 16);
        wb[m] = ldw(wm[m] + (size_t)rB[m] * row_bytes + (size_t)blk * 64 + t * 16);
        s[m][0] = bf16_to_f32(__ldg(sm[m] + (size_t)rA[m] * nb + blk));
        s[m][1] = bf16_to_f32(__ldg(sm[m] + (size_t)rB[m] * nb + blk));
      }
      constexpr int NS = GU ? 1 : 2;   // input parts: x, or h hi and lo
      uint4 xv[NS][4];
#pragma unroll
      for (int p = 0; p < NS; ++p)
#pragma unroll
        for (int j = 0; j < 4; ++j)
          xv[p][j] = colv ? __ldg(reinterpret_cast<const uint4*>(src + (size_t)p * I + (size_t)blk * 128 + 32 * t + 8 * j))
                          : make_uint4(0u, 0u, 0u, 0u);
      float d[NM][4], db[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int m = 0; m < NM; ++m) d[m][0] = d[m][1] = d[m][2] = d[m][3] = 0.f;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
#pragma unroll
        for (int p = 0; p < NS; ++p) {
          uint32_t b[4];
          in_pairs(xv[p][j], b);
#pragma unroll
          for (int m = 0; m < NM; ++m) {
            const uint32_t a = word_of(wa[m], j), c = word_of(wb[m], j);
            mma16816(d[m], nib2(a, 0), nib2(c, 0), nib2(a, 1), nib2(c, 1), b[0], b[1]);
            mma16816(d[m], nib2(a, 2), nib2(c, 2), nib2(a, 3), nib2(c, 3), b[2], b[3]);
          }
          mma16816(db, kNeg136x2, kNeg136x2, kNeg136x2, kNeg136x2, b[0], b[1]);
          mma16816(db, kNeg136x2, kNeg136x2, kNeg136x2, kNeg136x2, b[2], b[3]);
        }
      }
      // d: rows g (d[0], d[1]) and g+8 (d[2], d[3]), columns 2t and 2t+1
#pragma unroll
      for (int m = 0; m < NM; ++m) {
        acc[m][0] = fmaf(s[m][0], d[m][0] + db[0], acc[m][0]);
        acc[m][1] = fmaf(s[m][0], d[m][1] + db[1], acc[m][1]);
        acc[m][2] = fmaf(s[m][1], d[m][2] + db[2], acc[m][2]);
        acc[m][3] = fmaf(s[m][1], d[m][3] + db[3], acc[m][3]);
      }
    }
#pragma unroll
    for (int m = 0; m < NM; ++m) {
      red[warp][m][g][2 * t] = acc[m][0];
      red[warp][m][g][2 * t + 1] = acc[m][1];
      red[warp][m][g + 8][2 * t] = acc[m][2];
      red[warp][m][g + 8][2 * t + 1] = acc[m][3];
    }
    __syncthreads();
    {
      const int r = threadIdx.x >> 3, col = threadIdx.x & 7;   // 128 threads: one (row, column) of a tile
      if constexpr (GU) {
        const float gv = ((red[0][0][r][col] + red[1][0][r][col]) + red[2][0][r][col]) + red[3][0][r][col];
        const float uv = ((red[0][1][r][col] + red[1][1][r][col]) + red[2][1][r][col]) + red[3][1][r][col];
        if (col < nt && row0 + r < rows) {
          const int q = c0 + col;
          const float hv = silu(gv) * uv;
          const uint16_t hi = f32_to_bf16(hv);
          uint16_t* hrow = reinterpret_cast<uint16_t*>(hbuf + (size_t)q * I);
          hrow[row0 + r] = hi;
          hrow[I + row0 + r] = f32_to_bf16(hv - bf16_to_f32(hi));
        }
      } else {
#pragma unroll
        for (int m = 0; m < NM; ++m) {
          const float v = ((red[0][m][r][col] + red[1][m][r][col]) + red[2][m][r][col]) + red[3][m][r][col];
          const int row = row0 + 16 * m + r;
          if (col < nt && row < rows) ybuf[(size_t)(c0 + col) * H + row] = v;
        }
      }
    }
    __syncthreads();
  }
}

}  // namespace

cudaError_t launch_ffn_int4_mma(const void* x, int T, int H, int I, int k, const ExpertList& list, const int* offsets,
                                const int* perm, float* h, float* y, cudaStream_t s, cudaEvent_t between) {
  if (list.n <= 0 || T <= 0) return cudaSuccess;
  if (H % 128 || I % 128) return cudaErrorInvalidValue;
  const uint16_t* xb = static_cast<const uint16_t*>(x);
  cudaError_t e = launch_pdl(int4_mma_kernel<0>, dim3(I / 16, list.n), dim3(kQThreads), s, false, xb, T, H, I, k,
                             list, offsets, perm, h, y);
  if (e != cudaSuccess) return e;
  if (between) cudaEventRecord(between, s);
  const unsigned down_ctas = (unsigned)((H + 16 * kDownTiles - 1) / (16 * kDownTiles));
  return launch_pdl(int4_mma_kernel<1>, dim3(down_ctas, list.n), dim3(kQThreads), s, true, xb, T, H, I, k, list,
                    offsets, perm, h, y);
}

}  // namespace ftk

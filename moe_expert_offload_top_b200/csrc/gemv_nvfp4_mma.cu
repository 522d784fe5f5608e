// K3 for decode with NVFP4 expert weights, on the f16 tensor cores.
//
// Method ("FreeToken linux", "FreeToken's MoE memory handling"; the NVFP4 release): each
// selected expert runs from its cache slot; h = silu(W_gate x) * (W_up x), y = W_down h, with
// NVFP4 weights w = c * s * G: c an e2m1 code (the low nibble of a byte holds the even
// element), s the e4m3 scale of 16 consecutive reduction-axis elements of one row, G the fp32
// scale of the matrix.
//
// Operands.  cvt.rn.f16x2.e2m1x2 turns a code byte into an f16 pair and one mul.rn.f16x2 by
// the pair (s, s) makes c * s, exactly: the product has at most 5 significant bits and lies
// in f16's normal range (2^-10 <= |c s| <= 2688).  These are the A fragments of
// mma.sync.m16n8k16 (f16 x f16 into fp32 accumulators).  With the block scales inside A,
// the groups of a row sum in the accumulators with no per-group step.  The inputs are rows
// of f16 with a per-row power-of-two scale, x' = x * 2^(14 - E), E the binary exponent of
// the row's largest |x|, so |x'| < 2^15.  A bf16 x converts exactly (f16 holds its 8
// significant bits) wherever |x| >= 2^-28 of the row's largest; h (fp32) rounds to 11
// significant bits there, a relative error of at most 2^-11 per element.  The result is the
// accumulator times G * 2^(E - 14).
//
// Fragments (m16n8k16, 16-bit).  Lane (g, t) = (lane / 4, lane % 4) holds 16 bytes of weight
// rows g and g+8 per group of 128 reduction-axis elements: elements 32t .. 32t+31.  MMA j
// (0..7) takes elements 4j .. 4j+3 of each lane's chunk: code byte 2j (elements 4j, 4j+1)
// gives A register a0 (row g) / a1 (row g+8), byte 2j+1 gives a2 / a3.  The MMA's reduction
// index is therefore a permutation of the physical one, and the inputs, kept in their
// natural order, follow it: B registers b0, b1 of MMA j are input elements 32t + 4j ..
// 32t + 4j + 3 of column g.  Elements 32t .. 32t+15 have block scale 2t of the group and
// 32t+16 .. 32t+31 block scale 2t+1: MMAs 0-3 use the first, 4-7 the second.
//
// Memory pipeline: as in the int4 kernel.  Every lane copies its own 16 bytes of rows g and
// g+8 of each tile, and (lanes of a token column) the column's 64 bytes, into its own slots
// of a cp.async ring, S - 1 groups ahead; stages hold input bytes for the launch's columns
// only; the CTA's block scales are staged in shared memory once; the W warps of a CTA split
// the reduction axis (W = 4 for gate/up, 2 for down) and add their sums in warp order; both
// passes are programmatic dependents of the slicing kernel before them.
#include "decode_gemv.cuh"
#include "gemv_ring.cuh"

namespace ftk {

namespace {

using namespace gemv;
using namespace ring;

#ifndef FT_NVFP4_GU_WARPS
#define FT_NVFP4_GU_WARPS 4
#endif
#ifndef FT_NVFP4_DOWN_WARPS
#define FT_NVFP4_DOWN_WARPS 2
#endif
constexpr int kWarpsPerSm = 16;   // resident warps per SM: caps the registers
constexpr int kDownTiles = 2;     // 16-row tiles of a down CTA
constexpr int kNtok = 8;          // tokens (MMA columns) per pass

// d (16x8 f32) += A (16x16 f16) * B (16x8 f16).
FT_DEVICE void mma_f16(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3, uint32_t b0, uint32_t b1) {
  asm("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}
// The four code bytes of w as f16 pairs (byte b -> o[b]; its low nibble in the low half).
FT_DEVICE void e2m1x8_to_f16x2(uint32_t w, uint32_t (&o)[4]) {
  asm("{ .reg .b8 c0, c1, c2, c3;\n\t"
      "mov.b32 {c0, c1, c2, c3}, %4;\n\t"
      "cvt.rn.f16x2.e2m1x2 %0, c0;\n\t"
      "cvt.rn.f16x2.e2m1x2 %1, c1;\n\t"
      "cvt.rn.f16x2.e2m1x2 %2, c2;\n\t"
      "cvt.rn.f16x2.e2m1x2 %3, c3; }"
      : "=r"(o[0]), "=r"(o[1]), "=r"(o[2]), "=r"(o[3])
      : "r"(w));
}
FT_DEVICE uint32_t hmul2(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("mul.rn.f16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}
// The two e4m3 scales in each half of sw as f16 pairs: lo = (s0, s1) of the low half, hi of
// the high half.
FT_DEVICE void e4m3x4_to_f16x2(uint32_t sw, uint32_t& lo, uint32_t& hi) {
  asm("{ .reg .b16 l, h;\n\t"
      "mov.b32 {l, h}, %2;\n\t"
      "cvt.rn.f16x2.e4m3x2 %0, l;\n\t"
      "cvt.rn.f16x2.e4m3x2 %1, h; }"
      : "=r"(lo), "=r"(hi)
      : "r"(sw));
}
FT_DEVICE uint32_t dup_lo(uint32_t p) { return __byte_perm(p, 0, 0x1010); }   // (p.lo, p.lo)
FT_DEVICE uint32_t dup_hi(uint32_t p) { return __byte_perm(p, 0, 0x3232); }   // (p.hi, p.hi)

// ---------------------------------------------------------------- the inputs --
// A sliced row of K inputs: [K f16: x * 2^(14 - E)][f: float = 2^(E - 14)][12 bytes].
__host__ __device__ constexpr size_t f16_row_bytes(int K) { return 2 * (size_t)K + 16; }

// The T tokens of x (bf16 [T][H]) as f16 rows; grid T, kPrepThreads threads.
__global__ void __launch_bounds__(kPrepThreads) nvfp4_prep_x_kernel(const uint16_t* __restrict__ x, int H,
                                                                    unsigned char* __restrict__ xs) {
  __shared__ float red[kPrepThreads / 32];
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");   // the gate/up pass's weight copies
  const uint16_t* row = x + (size_t)blockIdx.x * H;
  unsigned char* out = xs + (size_t)blockIdx.x * f16_row_bytes(H);
  float m = 0.f;
  for (int i = threadIdx.x; i < H; i += kPrepThreads) m = fmaxf(m, fabsf(bf16_to_f32(row[i])));
  m = block_max(m, red);
  const int E = exponent_of(m);
  const float scale = ldexpf(1.f, 14 - E);   // exact, and so is v * scale
  __half* o = reinterpret_cast<__half*>(out);
  for (int i = threadIdx.x; i < H; i += kPrepThreads) o[i] = __float2half_rn(bf16_to_f32(row[i]) * scale);
  if (threadIdx.x == 0) *reinterpret_cast<float*>(out + 2 * (size_t)H) = ldexpf(1.f, E - 14);
}

// The h rows of the list's pairs (fp32 [rows][I] written by the gate/up pass) as f16 rows,
// in place: row q becomes [I f16][f] within its 4I bytes.  Grid (n_list, rows_max).
__global__ void __launch_bounds__(kPrepThreads) nvfp4_prep_h_kernel(const __grid_constant__ ExpertList list, int T,
                                                                    int k, int I, const int* __restrict__ offsets,
                                                                    float* __restrict__ hbuf) {
  __shared__ float red[kPrepThreads / 32];
  extern __shared__ float vals[];   // I floats
  asm volatile("griddepcontrol.wait;" ::: "memory");
  const int e = list.expert[blockIdx.x];
  const int q0 = e >= 0 ? offsets[e] : T * k;
  const int n = e >= 0 ? offsets[e + 1] - q0 : T;
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  if ((int)blockIdx.y >= n) return;   // the same for the whole CTA
  float* row = hbuf + (size_t)(q0 + blockIdx.y) * I;
  float m = 0.f;
  for (int i = threadIdx.x; i < I; i += kPrepThreads) {
    const float v = __ldcg(row + i);
    vals[i] = v;
    m = fmaxf(m, fabsf(v));
  }
  m = block_max(m, red);   // its barriers also order every read of the row before the writes
  const int E = exponent_of(m);
  const float scale = ldexpf(1.f, 14 - E);
  __half* o = reinterpret_cast<__half*>(row);
  for (int i = threadIdx.x; i < I; i += kPrepThreads) o[i] = __float2half_rn(vals[i] * scale);
  if (threadIdx.x == 0) *reinterpret_cast<float*>(reinterpret_cast<unsigned char*>(row) + 2 * (size_t)I) = ldexpf(1.f, E - 14);
}

// ------------------------------------------------------------------ the GEMV --
// Per CTA: per warp a ring of S stages (the warps' partial sums reuse its bytes once every
// warp has drained its ring), and the block scales of its rows.  A stage is 2 NM weight chunks x 32 lanes x 16 bytes (chunk-major), then the input
// bytes of ncols columns, 256 bytes each (128 f16 of the group): lane (g, t)'s piece u
// (elements 32t + 8u .. +7) at slot (4u + t) ^ (4 (g & 1)), so that the 8 lanes of a
// quarter-warp read 8 distinct bank groups.  The scales are words [nb][NM][8 g][4 t]: the
// bytes 2t, 2t+1 of the group's 8 block scales of row g, then of row g+8.
template <int NM, int S, int W>
struct Fp4Smem {
  __host__ __device__ static constexpr size_t wbytes() { return (size_t)2 * NM * 32 * 16; }
  __host__ __device__ static constexpr size_t stage_bytes(int ncols) { return wbytes() + (size_t)ncols * 256; }
  __host__ __device__ static constexpr size_t ring_bytes(int ncols) { return (size_t)W * S * stage_bytes(ncols); }
  __host__ __device__ static constexpr size_t red_bytes() { return (size_t)W * NM * 16 * 8 * sizeof(float); }
  __host__ __device__ static constexpr size_t scale_off(int ncols) {
    return ring_bytes(ncols) > red_bytes() ? ring_bytes(ncols) : red_bytes();
  }
  __host__ __device__ static constexpr size_t bytes(int nb, int ncols) {
    return scale_off(ncols) + (size_t)nb * NM * 32 * 4;
  }
};

// MODE 0: gate/up + SwiGLU into h (fp32, then sliced by nvfp4_prep_h_kernel); MODE 1: down
// into y.  xs: the f16 token rows (MODE 0).  ncols (1..8): token columns per pass, at least
// the most pairs of any listed expert for one pass per expert.  Grid (ceil(rows / rows per
// CTA), list.n), 32 W threads, Fp4Smem<NM, S, W>::bytes(K / 128, ncols) bytes of shared memory.
template <int MODE, int NM, int S, int W>
__global__ void __launch_bounds__(32 * W, kWarpsPerSm / W)
nvfp4_mma_kernel(const unsigned char* __restrict__ xs, int T, int H, int I, int k, const __grid_constant__ ExpertList list,
                 const int* __restrict__ offsets, const int* __restrict__ perm, float* __restrict__ hbuf,
                 float* __restrict__ ybuf, int ncols) {
  constexpr bool GU = MODE == 0;
  using L = Fp4Smem<NM, S, W>;
  extern __shared__ __align__(16) unsigned char smem[];
  float (*red)[NM][16][8] = reinterpret_cast<float (*)[NM][16][8]>(smem);   // over the ring
  uint32_t* ssc = reinterpret_cast<uint32_t*>(smem + L::scale_off(ncols));

  const int e = list.expert[blockIdx.y];
  const uint8_t* blob = list.blob[blockIdx.y];
  const int K = GU ? H : I, rows = GU ? I : H;
  const int rows_cta = GU ? 16 * (NM / 2) : 16 * NM;
  const int row0 = blockIdx.x * rows_cta;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
  const size_t mat = (size_t)H * I;
  const uint8_t* scb = blob + 3 * mat / 2;                                           // e4m3 block scales
  const float* gsc = reinterpret_cast<const float*>(blob + 3 * mat / 2 + 3 * mat / 16);   // matrix scales
  const size_t row_bytes = (size_t)K / 2;
  const int nb = K / 128;
  const size_t srow = f16_row_bytes(K);   // an input row (x rows; h rows are 4 I bytes apart)
  const int b0 = warp * nb / W, b1 = (warp + 1) * nb / W, nblk = b1 - b0;
  int rbase[NM];
  const uint8_t* wsrc[2 * NM];   // this lane's 16 bytes of rows g ([2m]) and g+8 ([2m+1]) of tile m, group b0
#pragma unroll
  for (int m = 0; m < NM; ++m) {
    const uint8_t* wm = GU ? blob + (m & 1) * (mat / 2) : blob + mat;
    rbase[m] = GU ? row0 + 16 * (m >> 1) : row0 + 16 * m;
    wsrc[2 * m] = wm + (size_t)min(rbase[m] + g, rows - 1) * row_bytes + t * 16 + (size_t)b0 * 64;
    wsrc[2 * m + 1] = wm + (size_t)min(rbase[m] + g + 8, rows - 1) * row_bytes + t * 16 + (size_t)b0 * 64;
  }
  const uint32_t sbytes = (uint32_t)L::stage_bytes(ncols);
  const uint32_t ring_w = smem_u32(smem) + (uint32_t)warp * S * sbytes + (uint32_t)lane * 16;
  const uint32_t ring_x = smem_u32(smem) + (uint32_t)warp * S * sbytes + (uint32_t)L::wbytes();
  const uint32_t ssc_s = smem_u32(ssc) + (uint32_t)(g * 4 + t) * 4;

  const int q0 = e >= 0 ? offsets[e] : T * k;
  const int q1 = e >= 0 ? offsets[e + 1] : T * k + T;
  if (GU) asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  if (q1 <= q0 || row0 >= rows) {
    asm volatile("griddepcontrol.wait;" ::: "memory");
    return;
  }
  // block scales of the CTA's rows
  for (int i = threadIdx.x; i < nb * NM * 32; i += 32 * W) {
    const int b = i / (NM * 32), m = (i / 32) % NM, gg = (i / 4) % 8, tt = i % 4;
    const uint8_t* sm_m = GU ? scb + (m & 1) * (mat / 16) : scb + 2 * (mat / 16);
    const int rb = GU ? row0 + 16 * (m >> 1) : row0 + 16 * m;
    const uint32_t s_g = *reinterpret_cast<const unsigned short*>(sm_m + (size_t)min(rb + gg, rows - 1) * (K / 16) + b * 8 + 2 * tt);
    const uint32_t s_g8 = *reinterpret_cast<const unsigned short*>(sm_m + (size_t)min(rb + gg + 8, rows - 1) * (K / 16) + b * 8 + 2 * tt);
    ssc[i] = s_g | (s_g8 << 16);
  }
  auto issue_w = [&](int i, uint32_t st_off) {
#pragma unroll
    for (int c = 0; c < 2 * NM; ++c) cp16s(ring_w + st_off + 512 * c, wsrc[c] + (size_t)i * 64);
  };
  // the input column of lane g, group b0 + i: its 64 bytes (elements 32t .. 32t+31)
  uint32_t xo[4];
#pragma unroll
  for (int u = 0; u < 4; ++u) xo[u] = (uint32_t)(g * 256 + 16 * ((4 * u + t) ^ (4 * (g & 1))));
  auto issue_x = [&](int i, uint32_t st_off, const unsigned char* src) {
    const unsigned char* p = src + (size_t)(b0 + i) * 256 + 64 * t;
#pragma unroll
    for (int u = 0; u < 4; ++u) cp16s(ring_x + st_off + xo[u], p + 16 * u);
  };

  bool first = true;
  for (int c0 = q0; c0 < q1; c0 += ncols) {
    const int nt = min(ncols, q1 - c0);
    const bool valid = g < nt;
#pragma unroll 1
    for (int i = 0; i < S - 1; ++i) {
      if (i < nblk) issue_w(i, i * sbytes);
      cp_commit();
    }
    // before this point: only the weights, scales and routing (ready before the kernel before)
    if (first) asm volatile("griddepcontrol.wait;" ::: "memory");
    first = false;
    const unsigned char* src = xs;
    if (valid) {
      const int q = c0 + g;
      if constexpr (GU) src = xs + (size_t)(e >= 0 ? perm[q] / k : q - T * k) * srow;
      else src = reinterpret_cast<const unsigned char*>(hbuf + (size_t)q * I);
    }
#pragma unroll 1
    for (int i = 0; i < S - 1; ++i) {
      if (valid && i < nblk) issue_x(i, i * sbytes, src);
      cp_commit();
    }
    __syncthreads();   // the scales are staged
    // lanes past the pass's columns read column 0 (copied by lanes 0-3); their MMA columns are
    // discarded
    const int gx = valid ? g : 0;
    uint32_t xr[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) xr[u] = ring_x + (uint32_t)(gx * 256 + 16 * ((4 * u + t) ^ (4 * (gx & 1))));

    float acc[NM][4];
#pragma unroll
    for (int m = 0; m < NM; ++m) acc[m][0] = acc[m][1] = acc[m][2] = acc[m][3] = 0.f;
    uint32_t st_off = 0, wst_off = (S - 1) * sbytes;
    const uint32_t ring_bytes = S * sbytes;
#pragma unroll 1
    for (int i = 0; i < nblk; ++i) {
      const int nx = i + S - 1;
      if (nx < nblk) {
        issue_w(nx, wst_off);
        if (valid) issue_x(nx, wst_off, src);
      }
      cp_commit();
      cp_wait<S - 1>();
      __syncwarp();   // lanes 0-3's input copies are complete for the lanes that read them
      uint4 xv[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) xv[u] = lds128(xr[u] + st_off);
      const uint32_t srow_s = ssc_s + (uint32_t)(b0 + i) * (NM * 128);
#pragma unroll
      for (int m = 0; m < NM; ++m) {
        const uint4 wg = lds128(ring_w + st_off + 512 * (2 * m)), wg8 = lds128(ring_w + st_off + 512 * (2 * m + 1));
        uint32_t sg, sg8;   // (s_2t, s_2t+1) of rows g and g+8
        e4m3x4_to_f16x2(lds32(srow_s + 128 * m), sg, sg8);
#pragma unroll
        for (int wd = 0; wd < 4; ++wd) {   // code word wd: MMAs 2 wd and 2 wd + 1
          const uint32_t spg = wd < 2 ? dup_lo(sg) : dup_hi(sg), spg8 = wd < 2 ? dup_lo(sg8) : dup_hi(sg8);
          uint32_t og[4], og8[4];
          e2m1x8_to_f16x2(word_of(wg, wd), og);
          e2m1x8_to_f16x2(word_of(wg8, wd), og8);
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            const int j = 2 * wd + h;
            const uint32_t bx0 = word_of(xv[j >> 1], 2 * (j & 1)), bx1 = word_of(xv[j >> 1], 2 * (j & 1) + 1);
            mma_f16(acc[m], hmul2(og[2 * h], spg), hmul2(og8[2 * h], spg8), hmul2(og[2 * h + 1], spg),
                    hmul2(og8[2 * h + 1], spg8), bx0, bx1);
          }
        }
      }
      st_off = st_off + sbytes == ring_bytes ? 0 : st_off + sbytes;
      wst_off = wst_off + sbytes == ring_bytes ? 0 : wst_off + sbytes;
    }
    cp_wait<0>();
    __syncthreads();   // every warp's ring is drained: the partial sums may overwrite it
    // acc: rows g (0, 1) and g+8 (2, 3), columns 2t and 2t+1
#pragma unroll
    for (int m = 0; m < NM; ++m) {
      red[warp][m][g][2 * t] = acc[m][0];
      red[warp][m][g][2 * t + 1] = acc[m][1];
      red[warp][m][g + 8][2 * t] = acc[m][2];
      red[warp][m][g + 8][2 * t + 1] = acc[m][3];
    }
    __syncthreads();
    for (int rc = threadIdx.x; rc < 128; rc += 32 * W) {
      const int r = rc >> 3, col = rc & 7;   // one (row, column) of a tile per thread
      auto wsum = [&](int m, int cc) {
        float v = red[0][m][r][cc];
#pragma unroll
        for (int w = 1; w < W; ++w) v += red[w][m][r][cc];
        return v;
      };
      if (col < nt) {
        const int q = c0 + col;
        // the column's input row: 2^(E - 14) after its f16 values
        const float f = GU ? *reinterpret_cast<const float*>(xs + (size_t)(e >= 0 ? perm[q] / k : q - T * k) * srow + 2 * (size_t)K)
                           : __ldcg(reinterpret_cast<const float*>(reinterpret_cast<const unsigned char*>(hbuf + (size_t)q * I) + 2 * (size_t)K));
        if constexpr (GU) {
          const float fg = f * gsc[0], fu = f * gsc[1];
#pragma unroll
          for (int p = 0; p < NM / 2; ++p) {
            const int row = rbase[2 * p] + r;
            if (row < rows) hbuf[(size_t)q * I + row] = silu(wsum(2 * p, col) * fg) * (wsum(2 * p + 1, col) * fu);
          }
        } else {
          const float fd = f * gsc[2];
#pragma unroll
          for (int m = 0; m < NM; ++m) {
            const int row = rbase[m] + r;
            if (row < rows) ybuf[(size_t)q * H + row] = wsum(m, col) * fd;
          }
        }
      }
    }
    __syncthreads();
  }
}

// Stages of the ring for a pass of ncols token columns: the most (up to 5) with which
// kWarpsPerSm / W CTAs fit on an SM (of its 228 KB, less 1 KB reserved per CTA).
template <int NM, int W>
int fp4_stages(int nb, int ncols) {
  constexpr size_t kBudget = 228 * 1024 / (kWarpsPerSm / W) - 1024;
  return Fp4Smem<NM, 5, W>::bytes(nb, ncols) <= kBudget   ? 5
         : Fp4Smem<NM, 4, W>::bytes(nb, ncols) <= kBudget ? 4
                                                          : 3;
}

template <int MODE, int NM, int W, typename... Args>
cudaError_t launch_fp4(int nb, int ncols, dim3 grid, cudaStream_t s, bool dependent, Args... args) {
  switch (fp4_stages<NM, W>(nb, ncols)) {
    case 5:
      return launch_ex(nvfp4_mma_kernel<MODE, NM, 5, W>, grid, dim3(32 * W), Fp4Smem<NM, 5, W>::bytes(nb, ncols), s,
                       dependent, args..., ncols);
    case 4:
      return launch_ex(nvfp4_mma_kernel<MODE, NM, 4, W>, grid, dim3(32 * W), Fp4Smem<NM, 4, W>::bytes(nb, ncols), s,
                       dependent, args..., ncols);
    default:
      return launch_ex(nvfp4_mma_kernel<MODE, NM, 3, W>, grid, dim3(32 * W), Fp4Smem<NM, 3, W>::bytes(nb, ncols), s,
                       dependent, args..., ncols);
  }
}
}  // namespace

cudaError_t launch_ffn_nvfp4_mma(const void* x, int T, int H, int I, int k, const ExpertList& list, const int* offsets,
                                 const int* perm, float* h, float* y, cudaStream_t s, cudaEvent_t between,
                                 int max_pairs_per_expert, void* xsliced) {
  if (list.n <= 0 || T <= 0) return cudaSuccess;
  if (H % 128 || I % 128) return cudaErrorInvalidValue;
  // the f16 tokens go to xsliced, or to the front of y (y is written only by the down pass,
  // after the gate/up pass has read them)
  unsigned char* xs = static_cast<unsigned char*>(xsliced ? xsliced : static_cast<void*>(y));
  int has_shared = 0;
  for (int i = 0; i < list.n; ++i) has_shared |= list.expert[i] < 0;
  int rows_max = max_pairs_per_expert < 1 ? T * k : max_pairs_per_expert;
  if (has_shared && T > rows_max) rows_max = T;
  const int ncols = rows_max < kNtok ? rows_max : kNtok;
  cudaError_t e = launch_ex(nvfp4_prep_x_kernel, dim3(T), dim3(kPrepThreads), 0, s, false,
                            static_cast<const uint16_t*>(x), H, xs);
  if (e != cudaSuccess) return e;
  e = launch_fp4<0, 2, FT_NVFP4_GU_WARPS>(H / 128, ncols, dim3(I / 16, list.n), s, true,
                                          static_cast<const unsigned char*>(xs), T, H, I, k, list, offsets, perm, h, y);
  if (e != cudaSuccess) return e;
  if (between) cudaEventRecord(between, s);
  e = launch_ex(nvfp4_prep_h_kernel, dim3(list.n, rows_max), dim3(kPrepThreads), (size_t)I * sizeof(float), s, true,
                list, T, k, I, offsets, h);
  if (e != cudaSuccess) return e;
  const unsigned down_ctas = (unsigned)((H + 16 * kDownTiles - 1) / (16 * kDownTiles));
  return launch_fp4<1, kDownTiles, FT_NVFP4_DOWN_WARPS>(I / 128, ncols, dim3(down_ctas, list.n), s, true,
                                                        static_cast<const unsigned char*>(xs), T, H, I, k, list,
                                                        offsets, perm, h, y);
}

}  // namespace ftk

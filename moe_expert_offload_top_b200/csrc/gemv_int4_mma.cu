// K3 for decode with int4 (group-128) expert weights, on the int8 tensor cores.
//
// Method ("FreeToken linux", "FreeToken's MoE memory handling"): each selected expert
// runs from its cache slot; h = silu(W_gate x) * (W_up x), y = W_down h, with int4
// weights w = q * s (q a two's-complement nibble, s the bf16 scale of 128 consecutive
// reduction-axis elements of one row; the low nibble of a byte holds the even element).
//
// Integer products, exact.  A nibble q moved into the high half of a byte reads, as a
// signed int8, 16 q: (w << 4) & 0xF0F0F0F0 gives the even elements of a 32-bit word and
// w & 0xF0F0F0F0 the odd ones, three instructions per eight weights and no offset to
// remove.  The inputs (the token x for gate/up, h for down) are written, once per launch,
// as 16-bit block fixed point: X = round(v * 2^(14 - E)) with E the exponent of the
// largest |v| of the row (|X| < 2^15; for a bf16 x every element within 2^7 of the
// largest is exact, and the error of any element is below 2^-15 of the largest), split
// into a signed high byte and an unsigned low byte, X = 256 hi + lo.
// mma.sync.m16n8k32 multiplies the 16 q bytes with the hi bytes (s8 x s8) and the lo bytes
// (s8 x u8) into int32 accumulators, exactly: each 128-element group gives
// S = 256 D_hi + D_lo = 16 sum(q X).  The group's partial is float(S) times its weight
// scale s, summed in fp32; the row's result is that sum times 2^(E - 14) / 16.
//
// Fragments (m16n8k32, 8-bit).  Lane (g, t) = (lane / 4, lane % 4) holds 16 bytes (32
// nibbles, elements 32t .. 32t+31) of weight rows g and g+8 per group.  Word j of that
// chunk is elements k0 .. k0+7 (k0 = 32t + 8j): its even elements form A register a0 (row
// g) / a1 (row g+8) and its odd elements a2 / a3 of MMA j.  The reduction index of the MMA
// is therefore a permutation of the physical one, and the inputs are stored in the same
// permutation: in every block of 8 elements, the even ones first, then the odd ones.
//
// Memory pipeline: every lane copies the bytes it uses itself (16 bytes of rows g and g+8
// of each tile; for the lanes of a token column, 32 + 32 bytes of its hi and lo bytes) into
// its own slots of a shared-memory ring with cp.async, S - 1 groups ahead.  A stage holds
// the weight chunks and the input bytes of only the columns the launch uses (ncols <= 8,
// the most pairs of one expert), so that at batch 1 nearly all of the ring is weights; S
// is chosen per launch so that the CTAs of 16 warps fit on an SM (the register limit).  Both
// passes copy their first weight groups before griddepcontrol.wait.  Scales of the CTA's
// rows are staged in shared memory once.  The W warps of a CTA split the reduction axis and
// add their partial sums in warp order: W = 4 for gate/up (16 rows of gate and of up per
// CTA), W = 1 for down (32 rows per one-warp CTA, so that at batch 1 the 8 x 224 CTAs of a
// top-8 forward at H = 7168 are resident at once).  Lanes past the pass's token columns read
// column 0's input bytes, so the loop has no branch on the column; their MMA columns are
// discarded.
#include "decode_gemv.cuh"
#include "gemv_ring.cuh"

namespace ftk {

namespace {

using namespace gemv;
using namespace ring;

#ifndef FT_INT4_WARPS_PER_SM
#define FT_INT4_WARPS_PER_SM 16
#endif
constexpr int kWarpsPerSm = FT_INT4_WARPS_PER_SM;   // resident warps per SM: caps the registers
#ifndef FT_INT4_GU_WARPS
#define FT_INT4_GU_WARPS 4
#endif
#ifndef FT_INT4_DOWN_WARPS
#define FT_INT4_DOWN_WARPS 1
#endif
#ifndef FT_INT4_DOWN_TILES
#define FT_INT4_DOWN_TILES 2
#endif
constexpr int kDownTiles = FT_INT4_DOWN_TILES;
constexpr int kNtok = 8;                 // tokens (MMA columns) per pass

// d (16x8 s32) += A (16x32 s8) * B (32x8, s8 or u8).
FT_DEVICE void mma_s8s8(int (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3, uint32_t b0, uint32_t b1) {
  asm("mma.sync.aligned.m16n8k32.row.col.s32.s8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
      : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}
FT_DEVICE void mma_s8u8(int (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3, uint32_t b0, uint32_t b1) {
  asm("mma.sync.aligned.m16n8k32.row.col.s32.s8.u8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
      : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// 16 q of the even / odd nibbles of w as four signed bytes.
FT_DEVICE uint32_t even16q(uint32_t w) { return (w << 4) & 0xF0F0F0F0u; }
FT_DEVICE uint32_t odd16q(uint32_t w) { return w & 0xF0F0F0F0u; }

// ---------------------------------------------------------------- the inputs --
// A sliced row of K inputs: [hi bytes: K][lo bytes: K][f: float = 2^(E - 14) / 16][12 bytes],
// bytes in the even-then-odd order of every block of 8 elements.
__host__ __device__ constexpr size_t sliced_row_bytes(int K) { return 2 * (size_t)K + 16; }

// Writes the 8 values v (elements 8b .. 8b+7 of a row) as bytes of X = round(v * scale):
// hi bytes (signed) and lo bytes (unsigned), even elements first.
FT_DEVICE void slice8(const float (&v)[8], float scale, unsigned char* hi, unsigned char* lo, int b) {
  uint32_t h[2] = {0u, 0u}, l[2] = {0u, 0u};
#pragma unroll
  for (int e = 0; e < 8; ++e) {
    int X = __float2int_rn(v[e] * scale);
    X = max(-32767, min(32767, X));
    const int pos = (e & 1) ? 4 + (e >> 1) : (e >> 1);   // even elements first, then odd
    h[pos >> 2] |= (uint32_t)((X >> 8) & 0xFF) << (8 * (pos & 3));
    l[pos >> 2] |= (uint32_t)(X & 0xFF) << (8 * (pos & 3));
  }
  *reinterpret_cast<uint2*>(hi + 8 * b) = make_uint2(h[0], h[1]);
  *reinterpret_cast<uint2*>(lo + 8 * b) = make_uint2(l[0], l[1]);
}

// The T tokens of x (bf16 [T][H]) as sliced rows; grid T, kPrepThreads threads.
__global__ void __launch_bounds__(kPrepThreads) int4_prep_x_kernel(const uint16_t* __restrict__ x, int H,
                                                                   unsigned char* __restrict__ xs) {
  __shared__ float red[kPrepThreads / 32];
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");   // the gate/up pass's weight copies
  const uint16_t* row = x + (size_t)blockIdx.x * H;
  unsigned char* out = xs + (size_t)blockIdx.x * sliced_row_bytes(H);
  float m = 0.f;
  for (int i = threadIdx.x; i < H; i += kPrepThreads) m = fmaxf(m, fabsf(bf16_to_f32(row[i])));
  m = block_max(m, red);
  // E = exponent of the largest |v|; the scale 2^(14 - E) is exact, so is v * scale
  const int E = exponent_of(m);
  const float scale = ldexpf(1.f, 14 - E);
  for (int b = threadIdx.x; b < H / 8; b += kPrepThreads) {
    const uint4 q = *reinterpret_cast<const uint4*>(row + 8 * b);
    const float v[8] = {bf16lo(q.x), bf16hi(q.x), bf16lo(q.y), bf16hi(q.y),
                        bf16lo(q.z), bf16hi(q.z), bf16lo(q.w), bf16hi(q.w)};
    slice8(v, scale, out, out + H, b);
  }
  if (threadIdx.x == 0) *reinterpret_cast<float*>(out + 2 * (size_t)H) = ldexpf(1.f, E - 14) * 0.0625f;
}

// The h rows of the list's pairs (fp32 [rows][I] written by the gate/up pass), sliced in
// place: row q becomes [hi I][lo I][f] within its 4I bytes.  Grid (n_list, rows_max).
__global__ void __launch_bounds__(kPrepThreads) int4_prep_h_kernel(const __grid_constant__ ExpertList list, int T,
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
  unsigned char* out = reinterpret_cast<unsigned char*>(row);
  for (int b = threadIdx.x; b < I / 8; b += kPrepThreads) {
    float v[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) v[i] = vals[8 * b + i];
    slice8(v, scale, out, out + I, b);
  }
  if (threadIdx.x == 0) *reinterpret_cast<float*>(out + 2 * (size_t)I) = ldexpf(1.f, E - 14) * 0.0625f;
}

// ------------------------------------------------------------------ the GEMV --
// Per CTA: per warp a ring of S stages, then the warps' partial sums, then the scales of
// its rows (per group and tile, the bf16 scales of rows g and g+8 in one word).  A stage is 2 NM weight chunks x 32 lanes x 16 bytes (chunk-major), then the
// input bytes of ncols columns, 256 bytes each: pieces 0-7 the 128 hi bytes of the group,
// 8-15 the lo bytes, piece p of column c at slot p ^ c so that the 8 columns' lanes read
// without bank conflicts.
template <int NM, int S, int W>
struct Int4Smem {
  __host__ __device__ static constexpr size_t wbytes() { return (size_t)2 * NM * 32 * 16; }
  __host__ __device__ static constexpr size_t stage_bytes(int ncols) { return wbytes() + (size_t)ncols * 256; }
  __host__ __device__ static constexpr size_t red_off(int ncols) { return (size_t)W * S * stage_bytes(ncols); }
  __host__ __device__ static constexpr size_t red_bytes() { return (size_t)W * NM * 16 * 8 * sizeof(float); }
  __host__ __device__ static constexpr size_t scale_off(int ncols) { return red_off(ncols) + red_bytes(); }
  __host__ __device__ static constexpr size_t bytes(int nb, int ncols) {
    return scale_off(ncols) + (size_t)NM * 16 * nb * 2;
  }
};

// MODE 0: gate/up + SwiGLU into h (fp32, sliced by int4_prep_h_kernel); MODE 1: down into y.
// xs: the sliced token rows (MODE 0).  ncols (1..8): token columns per pass, at least the
// most pairs of any listed expert for one pass per expert.  Grid (ceil(rows / rows per CTA),
// list.n), 128 threads, Int4Smem<NM, S>::bytes(K / 128, ncols) bytes of shared memory.
template <int MODE, int NM, int S, int W>
__global__ void __launch_bounds__(32 * W, kWarpsPerSm / W)
int4_i8_kernel(const unsigned char* __restrict__ xs, int T, int H, int I, int k, const __grid_constant__ ExpertList list,
               const int* __restrict__ offsets, const int* __restrict__ perm, float* __restrict__ hbuf,
               float* __restrict__ ybuf, int ncols) {
  constexpr bool GU = MODE == 0;
  using L = Int4Smem<NM, S, W>;
  extern __shared__ __align__(16) unsigned char smem[];
  float (*red)[NM][16][8] = reinterpret_cast<float (*)[NM][16][8]>(smem + L::red_off(ncols));
  uint32_t* ssc = reinterpret_cast<uint32_t*>(smem + L::scale_off(ncols));   // [nb][NM][8]: rows g | g+8 << 16

  const int e = list.expert[blockIdx.y];
  const uint8_t* blob = list.blob[blockIdx.y];
  const int K = GU ? H : I, rows = GU ? I : H;
  const int rows_cta = GU ? 16 * (NM / 2) : 16 * NM;
  const int row0 = blockIdx.x * rows_cta;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
  const size_t mat = (size_t)H * I;
  const uint16_t* sc = reinterpret_cast<const uint16_t*>(blob + 3 * mat / 2);
  const size_t row_bytes = (size_t)K / 2;
  const int nb = K / 128;
  const size_t srow = sliced_row_bytes(K);   // a sliced input row (x rows; h rows are 4 I bytes apart)
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
  // shared addresses: weight chunk c of stage st at ring_w + st * sbytes + 512 c; piece p of
  // input column c at ring_x + st * sbytes + 256 c + 16 (p ^ c)
  const uint32_t sbytes = (uint32_t)L::stage_bytes(ncols);
  const uint32_t ring_w = smem_u32(smem) + (uint32_t)warp * S * sbytes + (uint32_t)lane * 16;
  const uint32_t ring_x = smem_u32(smem) + (uint32_t)warp * S * sbytes + (uint32_t)L::wbytes();
  const uint32_t ssc_s = smem_u32(ssc) + (uint32_t)g * 4;

  const int q0 = e >= 0 ? offsets[e] : T * k;
  const int q1 = e >= 0 ? offsets[e + 1] : T * k + T;
  if (GU) asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  if (q1 <= q0 || row0 >= rows) {
    asm volatile("griddepcontrol.wait;" ::: "memory");
    return;
  }
  for (int i = threadIdx.x; i < nb * NM * 8; i += 32 * W) {
    const int b = i / (NM * 8), m = (i / 8) % NM, r = i % 8;
    const uint16_t* sm_m = GU ? sc + (m & 1) * (mat / 128) : sc + 2 * (mat / 128);
    const int rb = GU ? row0 + 16 * (m >> 1) : row0 + 16 * m;
    const uint32_t s_lo = __ldg(sm_m + (size_t)min(rb + r, rows - 1) * nb + b);
    const uint32_t s_hi = __ldg(sm_m + (size_t)min(rb + r + 8, rows - 1) * nb + b);
    ssc[i] = s_lo | (s_hi << 16);
  }
  auto issue_w = [&](int i, uint32_t st_off) {
#pragma unroll
    for (int c = 0; c < 2 * NM; ++c) cp16s(ring_w + st_off + 512 * c, wsrc[c] + (size_t)i * 64);
  };
  // the input column of lane g, group b0 + i: 32 hi bytes (elements 32t .. 32t+31), 32 lo bytes
  const uint32_t xo[4] = {(uint32_t)(g * 256 + 16 * ((2 * t) ^ g)), (uint32_t)(g * 256 + 16 * ((2 * t + 1) ^ g)),
                          (uint32_t)(g * 256 + 16 * ((8 + 2 * t) ^ g)), (uint32_t)(g * 256 + 16 * ((9 + 2 * t) ^ g))};
  auto issue_x = [&](int i, uint32_t st_off, const unsigned char* src) {
    const unsigned char* p = src + (size_t)(b0 + i) * 128 + 32 * t;
    cp16s(ring_x + st_off + xo[0], p);
    cp16s(ring_x + st_off + xo[1], p + 16);
    cp16s(ring_x + st_off + xo[2], p + K);
    cp16s(ring_x + st_off + xo[3], p + K + 16);
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
    const uint32_t xr0 = ring_x + gx * 256 + 16 * ((2 * t) ^ gx), xr1 = ring_x + gx * 256 + 16 * ((2 * t + 1) ^ gx);
    const uint32_t xr2 = ring_x + gx * 256 + 16 * ((8 + 2 * t) ^ gx), xr3 = ring_x + gx * 256 + 16 * ((9 + 2 * t) ^ gx);

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
      uint4 wv[2 * NM];
#pragma unroll
      for (int c = 0; c < 2 * NM; ++c) wv[c] = lds128(ring_w + st_off + 512 * c);
      const uint4 xh0 = lds128(xr0 + st_off), xh1 = lds128(xr1 + st_off);
      const uint4 xl0 = lds128(xr2 + st_off), xl1 = lds128(xr3 + st_off);
      int dh[NM][4], dl[NM][4];
#pragma unroll
      for (int m = 0; m < NM; ++m)
#pragma unroll
        for (int r = 0; r < 4; ++r) dh[m][r] = dl[m][r] = 0;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        // B of MMA j: this lane's 8 input bytes of word j (even elements, then odd ones)
        const uint4& xh = j < 2 ? xh0 : xh1;
        const uint4& xl = j < 2 ? xl0 : xl1;
        const uint32_t bh0 = word_of(xh, 2 * (j & 1)), bh1 = word_of(xh, 2 * (j & 1) + 1);
        const uint32_t bl0 = word_of(xl, 2 * (j & 1)), bl1 = word_of(xl, 2 * (j & 1) + 1);
#pragma unroll
        for (int m = 0; m < NM; ++m) {
          const uint32_t a = word_of(wv[2 * m], j), c = word_of(wv[2 * m + 1], j);
          const uint32_t a0 = even16q(a), a1 = even16q(c), a2 = odd16q(a), a3 = odd16q(c);
          mma_s8s8(dh[m], a0, a1, a2, a3, bh0, bh1);
          mma_s8u8(dl[m], a0, a1, a2, a3, bl0, bl1);
        }
      }
      // dh/dl: rows g (0, 1) and g+8 (2, 3), columns 2t and 2t+1
      const uint32_t srow_s = ssc_s + (uint32_t)(b0 + i) * (NM * 32);
#pragma unroll
      for (int m = 0; m < NM; ++m) {
        const uint32_t sp = lds32(srow_s + 32 * m);
        const float s0 = __uint_as_float(sp << 16), s1 = __uint_as_float(sp & 0xFFFF0000u);
        acc[m][0] = fmaf(s0, (float)(256 * dh[m][0] + dl[m][0]), acc[m][0]);
        acc[m][1] = fmaf(s0, (float)(256 * dh[m][1] + dl[m][1]), acc[m][1]);
        acc[m][2] = fmaf(s1, (float)(256 * dh[m][2] + dl[m][2]), acc[m][2]);
        acc[m][3] = fmaf(s1, (float)(256 * dh[m][3] + dl[m][3]), acc[m][3]);
      }
      st_off = st_off + sbytes == ring_bytes ? 0 : st_off + sbytes;
      wst_off = wst_off + sbytes == ring_bytes ? 0 : wst_off + sbytes;
    }
    cp_wait<0>();
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
        // the column's input row: 2^(E - 14) / 16 after its bytes
        const float f = GU ? *reinterpret_cast<const float*>(xs + (size_t)(e >= 0 ? perm[q] / k : q - T * k) * srow + 2 * (size_t)K)
                           : __ldcg(reinterpret_cast<const float*>(reinterpret_cast<const unsigned char*>(hbuf + (size_t)q * I) + 2 * (size_t)K));
        if constexpr (GU) {
#pragma unroll
          for (int p = 0; p < NM / 2; ++p) {
            const int row = rbase[2 * p] + r;
            if (row < rows) hbuf[(size_t)q * I + row] = silu(wsum(2 * p, col) * f) * (wsum(2 * p + 1, col) * f);
          }
        } else {
#pragma unroll
          for (int m = 0; m < NM; ++m) {
            const int row = rbase[m] + r;
            if (row < rows) ybuf[(size_t)q * H + row] = wsum(m, col) * f;
          }
        }
      }
    }
    __syncthreads();
  }
}

}  // namespace

size_t int4_sliced_x_bytes(int T, int H) { return (size_t)T * sliced_row_bytes(H); }

namespace {
// Stages of the ring for a pass of ncols token columns: the most (up to 5) with which
// kWarpsPerSm / W CTAs fit on an SM (of its 228 KB, less 1 KB reserved per CTA).
template <int NM, int W>
int int4_stages(int nb, int ncols) {
  constexpr size_t kBudget = 228 * 1024 / (kWarpsPerSm / W) - 1024;
  return Int4Smem<NM, 5, W>::bytes(nb, ncols) <= kBudget   ? 5
         : Int4Smem<NM, 4, W>::bytes(nb, ncols) <= kBudget ? 4
                                                           : 3;
}

template <int MODE, int NM, int W, typename... Args>
cudaError_t launch_i8(int nb, int ncols, dim3 grid, cudaStream_t s, bool dependent, Args... args) {
  switch (int4_stages<NM, W>(nb, ncols)) {
    case 5:
      return launch_ex(int4_i8_kernel<MODE, NM, 5, W>, grid, dim3(32 * W), Int4Smem<NM, 5, W>::bytes(nb, ncols), s,
                       dependent, args..., ncols);
    case 4:
      return launch_ex(int4_i8_kernel<MODE, NM, 4, W>, grid, dim3(32 * W), Int4Smem<NM, 4, W>::bytes(nb, ncols), s,
                       dependent, args..., ncols);
    default:
      return launch_ex(int4_i8_kernel<MODE, NM, 3, W>, grid, dim3(32 * W), Int4Smem<NM, 3, W>::bytes(nb, ncols), s,
                       dependent, args..., ncols);
  }
}
}  // namespace

cudaError_t launch_ffn_int4_mma(const void* x, int T, int H, int I, int k, const ExpertList& list, const int* offsets,
                                const int* perm, float* h, float* y, cudaStream_t s, cudaEvent_t between,
                                int max_pairs_per_expert, void* xsliced) {
  if (list.n <= 0 || T <= 0) return cudaSuccess;
  if (H % 128 || I % 128) return cudaErrorInvalidValue;
  // the sliced tokens go to xsliced, or to the front of y (y is written only by the down pass,
  // after the gate/up pass has read them)
  unsigned char* xs = static_cast<unsigned char*>(xsliced ? xsliced : static_cast<void*>(y));
  int has_shared = 0;
  for (int i = 0; i < list.n; ++i) has_shared |= list.expert[i] < 0;
  int rows_max = max_pairs_per_expert < 1 ? T * k : max_pairs_per_expert;
  if (has_shared && T > rows_max) rows_max = T;
  const int ncols = rows_max < kNtok ? rows_max : kNtok;
  cudaError_t e = launch_ex(int4_prep_x_kernel, dim3(T), dim3(kPrepThreads), 0, s, false,
                            static_cast<const uint16_t*>(x), H, xs);
  if (e != cudaSuccess) return e;
  e = launch_i8<0, 2, FT_INT4_GU_WARPS>(H / 128, ncols, dim3(I / 16, list.n), s, true,
                                       static_cast<const unsigned char*>(xs), T, H, I, k, list, offsets, perm, h, y);
  if (e != cudaSuccess) return e;
  if (between) cudaEventRecord(between, s);
  e = launch_ex(int4_prep_h_kernel, dim3(list.n, rows_max), dim3(kPrepThreads), (size_t)I * sizeof(float), s, true,
                list, T, k, I, offsets, h);
  if (e != cudaSuccess) return e;
  const unsigned down_ctas = (unsigned)((H + 16 * kDownTiles - 1) / (16 * kDownTiles));
  return launch_i8<1, kDownTiles, FT_INT4_DOWN_WARPS>(I / 128, ncols, dim3(down_ctas, list.n), s, true,
                                                     static_cast<const unsigned char*>(xs), T, H, I, k, list, offsets,
                                                     perm, h, y);
}

}  // namespace ftk

// K3 for decode with int4 (group-128) expert weights, on the tensor cores.
//
// Method ("FreeToken linux", "FreeToken's MoE memory handling"): each selected expert
// runs from its cache slot; h = silu(W_gate x) * (W_up x), y = W_down h, with int4
// weights w = q * s (q a two's-complement nibble, s the bf16 scale of 128 consecutive
// reduction-axis elements of one row; the low nibble of a byte holds the even element).
//
// Why tensor cores for a matrix-vector product.  On the FP32 pipes an int4 weight costs
// about five instructions (unpack, widen, offset, multiply-add), so the GEMV is bound by
// instruction issue, not by HBM.  Here the unpack is about one instruction per weight
// and the multiply-adds go to mma.sync.m16n8k16 (bf16 in, fp32 accumulate), which also
// covers up to 8 tokens of an expert at once.  The operands stay in registers:
// tcgen05.mma would take the dequantised weights from shared memory, i.e. twice the
// HBM bytes again through shared memory, for an M of at most 8 tokens.
//
// Tile: a CTA owns NM 16-row weight tiles of one expert: gate and up rows of the same
// 16 (or 32) h columns, or 16*NM consecutive rows of W_down.  Its 4 warps split the
// reduction axis into contiguous ranges of 128-element groups; their partial sums are
// added in warp order through shared memory.
//
// Memory pipeline.  Every lane copies the bytes it will itself use (its two rows of
// each tile, 16 bytes per row per group, and its 64 bytes of the input vector) into its
// own slots of a shared-memory ring with cp.async, S groups ahead of the group it
// computes, and reads them back with 16-byte shared loads: the loads in flight do not
// hold registers, and no barrier is needed (a thread's cp.async.wait_group covers its
// own copies).  The scales of the CTA's rows are staged in shared memory once.  The
// down pass copies its weights (and scales) before griddepcontrol.wait, so they stream
// while the gate/up grid finishes; only its inputs h wait for it.
//
// Fragments.  Lane (g, t) = (lane / 4, lane % 4).  For one 128-element group, lane
// (g, t) holds 16 bytes (32 nibbles, elements 32t .. 32t+31) of rows g and g+8.  Word j
// of that chunk holds elements k0 .. k0+7 (k0 = 32t + 8j); the pair (k0+n, k0+n+4) of
// nibbles n and n+4 becomes one bf16x2 register: ((w >> 4n) & 0x000F000F) ^ 0x43084308
// is the bf16 pair (136 + q).  This is the exponent-bias (magic number) integer-to-
// float conversion: the 4-bit integer is written into the low mantissa bits of a float
// whose exponent makes one mantissa step worth 1 (bf16 128.0 = 0x4300), and flipping
// bit 3 maps the two's-complement nibble q to q + 8, so the float reads 128 + q + 8
// (the conversion described for int4 -> fp16 by Kim et al., "Who Says Elephants Can't
// Run: Bringing Large Scale MoE Models into Cloud Scale Production", 2022, here with a
// bf16 exponent).  The MMA's reduction index is a permutation of the physical one (the
// same for weights and inputs): MMA 2j takes pairs n = 0, 1, MMA 2j+1 pairs n = 2, 3,
// and the input fragment is built from the same element pairs with byte permutes.  The
// offset 136 is removed per group by one MMA against a constant fragment of -136 (shared
// by the CTA's tiles), so each group's partial sum is sum(q x) as far as fp32
// accumulation goes; it is then scaled by the group's s and accumulated.
//
// Down projection: its input h is fp32.  The gate/up kernel stores each h value as two
// bf16 (hi = bf16(h), lo = bf16(h - hi)) in the same row of the h buffer, so h keeps 16
// bits of mantissa (relative error 2^-17).  The down MMAs take hi and lo as separate
// columns of the input fragment (columns 0-3: hi of up to 4 tokens, 4-7: their lo), so
// one MMA covers both, and the two columns are added at the end.
#include "decode_gemv.cuh"
#include "sm100_sync.cuh"

namespace ftk {

namespace {

using namespace gemv;

constexpr int kQWarps = 4;
constexpr int kQThreads = 32 * kQWarps;
#ifndef FT_INT4_STAGES
#define FT_INT4_STAGES 4
#endif
#ifndef FT_INT4_GU_TILES
#define FT_INT4_GU_TILES 2
#endif
#ifndef FT_INT4_DOWN_TILES
#define FT_INT4_DOWN_TILES 2
#endif
constexpr int kStages = FT_INT4_STAGES;          // groups of copies in flight per lane
constexpr int kGuTiles = FT_INT4_GU_TILES;       // gate/up: 16-row tiles per CTA (gate, up: even)
constexpr int kDownTiles = FT_INT4_DOWN_TILES;   // down: 16-row tiles per CTA
constexpr uint32_t kNeg136x2 = 0xC308C308u;      // bf16 pair (-136, -136)

// d (16x8 f32) = A (16x16 bf16) * B (16x8 bf16) + c.
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

// 16-byte asynchronous copy global -> shared; bytes = 0 writes zeros and reads nothing.
FT_DEVICE void cp16(void* dst, const void* src, uint32_t bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(smem_u32(dst)), "l"(src), "r"(bytes)
               : "memory");
}
FT_DEVICE void cp_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
FT_DEVICE void cp_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

// Shared-memory layout of one CTA (dynamic): the scales of its rows, the partial sums of
// its warps, and per warp a ring of kStages groups of (2 NM weight chunks + 4 input
// chunks) x 32 lanes x 16 bytes, stored chunk-major so that a warp's 16-byte shared
// accesses are contiguous.
template <int NM>
struct Int4Smem {
  static constexpr int kChunks = 2 * NM + 4;
  __host__ __device__ static constexpr size_t ring_off() { return 0; }
  __host__ __device__ static constexpr size_t ring_bytes() { return (size_t)kQWarps * kStages * kChunks * 32 * 16; }
  __host__ __device__ static constexpr size_t red_off() { return ring_bytes(); }
  __host__ __device__ static constexpr size_t red_bytes() { return (size_t)kQWarps * NM * 16 * 8 * sizeof(float); }
  __host__ __device__ static constexpr size_t scale_off() { return red_off() + red_bytes(); }
  __host__ __device__ static constexpr size_t bytes(int nb) { return scale_off() + (size_t)NM * 16 * nb * sizeof(uint16_t); }
};

// MODE 0: gate/up + SwiGLU into h (bf16 hi/lo per value); MODE 1: down into y (f32).
// Grid (ceil(rows / rows per CTA), list.n), 128 threads, Int4Smem<NM>::bytes(nb) of dynamic
// shared memory.
template <int MODE, int NM>
__global__ void __launch_bounds__(kQThreads)
int4_mma_kernel(const uint16_t* __restrict__ x, int T, int H, int I, int k, const __grid_constant__ ExpertList list,
                const int* __restrict__ offsets, const int* __restrict__ perm, float* __restrict__ hbuf,
                float* __restrict__ ybuf) {
  constexpr bool GU = MODE == 0;
  constexpr int NTOK = GU ? 8 : 4;          // tokens per pass (down: hi and lo take two columns each)
  using L = Int4Smem<NM>;
  extern __shared__ __align__(16) unsigned char smem[];
  uint4* ring = reinterpret_cast<uint4*>(smem + L::ring_off());
  float (*red)[NM][16][8] = reinterpret_cast<float (*)[NM][16][8]>(smem + L::red_off());
  uint16_t* ssc = reinterpret_cast<uint16_t*>(smem + L::scale_off());   // [NM][16][nb]

  const int e = list.expert[blockIdx.y];
  const uint8_t* blob = list.blob[blockIdx.y];
  const int K = GU ? H : I, rows = GU ? I : H;
  const int rows_cta = GU ? 16 * (NM / 2) : 16 * NM;
  const int row0 = blockIdx.x * rows_cta;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
  const size_t mat = (size_t)H * I;
  const uint16_t* sc = reinterpret_cast<const uint16_t*>(blob + 3 * mat / 2);
  const size_t row_bytes = (size_t)K / 2;
  const int nb = K / 128;                                       // scale groups per row
  // tile m: matrix wm[m], first row rbase[m]
  const uint8_t* wm[NM];
  int rbase[NM];
#pragma unroll
  for (int m = 0; m < NM; ++m) {
    wm[m] = GU ? blob + (m & 1) * (mat / 2) : blob + mat;
    rbase[m] = GU ? row0 + 16 * (m >> 1) : row0 + 16 * m;
  }
  const uint8_t* wsrcA[NM];   // this lane's rows g and g+8 of each tile (clamped to the matrix)
  const uint8_t* wsrcB[NM];
#pragma unroll
  for (int m = 0; m < NM; ++m) {
    wsrcA[m] = wm[m] + (size_t)min(rbase[m] + g, rows - 1) * row_bytes + t * 16;
    wsrcB[m] = wm[m] + (size_t)min(rbase[m] + g + 8, rows - 1) * row_bytes + t * 16;
  }
  const int b0 = warp * nb / kQWarps, b1 = (warp + 1) * nb / kQWarps, nblk = b1 - b0;
  uint4* myring = ring + (size_t)warp * kStages * L::kChunks * 32 + lane;   // chunk c of stage s: [(s*kChunks + c)*32]

  const int q0 = e >= 0 ? offsets[e] : T * k;   // offsets is written before this grid (routing)
  const int q1 = e >= 0 ? offsets[e + 1] : T * k + T;
  if (GU) asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  if (q1 <= q0 || row0 >= rows) {                // the same for the whole CTA
    if (!GU) asm volatile("griddepcontrol.wait;" ::: "memory");
    return;
  }

  // scales of the CTA's rows (rows past the matrix repeat its last row; never stored)
  for (int i = threadIdx.x; i < NM * 16 * nb; i += kQThreads) {
    const int m = i / (16 * nb), r = (i / nb) % 16, b = i % nb;
    const uint16_t* sm_m = GU ? sc + (m & 1) * (mat / 128) : sc + 2 * (mat / 128);
    const int rb = GU ? row0 + 16 * (m >> 1) : row0 + 16 * m;
    ssc[i] = __ldg(sm_m + (size_t)min(rb + r, rows - 1) * nb + b);
  }

  auto issue_w = [&](int i) {   // weight chunks of local group i into stage i % kStages
    uint4* st = myring + (size_t)(i % kStages) * L::kChunks * 32;
    const size_t off = (size_t)(b0 + i) * 64;
#pragma unroll
    for (int m = 0; m < NM; ++m) {
      cp16(st + (2 * m) * 32, wsrcA[m] + off, 16);
      cp16(st + (2 * m + 1) * 32, wsrcB[m] + off, 16);
    }
  };
  // input chunks: 64 bytes of this lane's column for local group i (zeros where the
  // column has no token)
  auto issue_x = [&](int i, const uint16_t* src, bool valid) {
    uint4* st = myring + (size_t)(i % kStages) * L::kChunks * 32 + 2 * NM * 32;
    const uint16_t* p = valid ? src + (size_t)(b0 + i) * 128 + 32 * t : x;
#pragma unroll
    for (int j = 0; j < 4; ++j) cp16(st + j * 32, valid ? p + 8 * j : x, valid ? 16u : 0u);
  };

  bool first_chunk = true;
  for (int c0 = q0; c0 < q1; c0 += NTOK) {
    const int nt = min(NTOK, q1 - c0);
    // this lane's input column: GU token g; down hi (g < 4) or lo (g >= 4) of token g % 4
    const int col_tok = GU ? g : (g & 3);
    const bool valid = col_tok < nt;
    // prologue: weight copies of the first kStages-1 groups (down: before waiting for the
    // gate/up grid, whose h it reads), then the inputs of those groups
#pragma unroll
    for (int i = 0; i < kStages - 1; ++i) {
      if (i < nblk) issue_w(i);
      cp_commit();
    }
    if (!GU && first_chunk) asm volatile("griddepcontrol.wait;" ::: "memory");
    first_chunk = false;
    const uint16_t* src = x;
    if (valid) {
      const int q = c0 + col_tok;
      if constexpr (GU) {
        const int tok = e >= 0 ? perm[q] / k : q - T * k;
        src = x + (size_t)tok * H;
      } else {
        src = reinterpret_cast<const uint16_t*>(hbuf + (size_t)q * I) + (g >> 2) * I;   // hi, or lo
      }
    }
#pragma unroll
    for (int i = 0; i < kStages - 1; ++i) {
      if (i < nblk) issue_x(i, src, valid);
      cp_commit();
    }
    __syncthreads();   // the scales are staged

    float acc[NM][4];
#pragma unroll
    for (int m = 0; m < NM; ++m) acc[m][0] = acc[m][1] = acc[m][2] = acc[m][3] = 0.f;

    for (int i = 0; i < nblk; ++i) {
      const int nx = i + kStages - 1;   // the group whose copies go out now
      if (nx < nblk) {
        issue_w(nx);
        issue_x(nx, src, valid);
      }
      cp_commit();
      cp_wait<kStages - 1>();           // group i has landed (this lane's copies)
      const uint4* st = myring + (size_t)(i % kStages) * L::kChunks * 32;
      uint4 wa[NM], wb[NM], xv[4];
#pragma unroll
      for (int m = 0; m < NM; ++m) { wa[m] = st[(2 * m) * 32]; wb[m] = st[(2 * m + 1) * 32]; }
#pragma unroll
      for (int j = 0; j < 4; ++j) xv[j] = st[(2 * NM + j) * 32];
      float d[NM][4], db[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int m = 0; m < NM; ++m) d[m][0] = d[m][1] = d[m][2] = d[m][3] = 0.f;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        uint32_t b[4];
        in_pairs(xv[j], b);
#pragma unroll
        for (int m = 0; m < NM; ++m) {
          const uint32_t a = word_of(wa[m], j), c = word_of(wb[m], j);
          mma16816(d[m], nib2(a, 0), nib2(c, 0), nib2(a, 1), nib2(c, 1), b[0], b[1]);
          mma16816(d[m], nib2(a, 2), nib2(c, 2), nib2(a, 3), nib2(c, 3), b[2], b[3]);
        }
        mma16816(db, kNeg136x2, kNeg136x2, kNeg136x2, kNeg136x2, b[0], b[1]);
        mma16816(db, kNeg136x2, kNeg136x2, kNeg136x2, kNeg136x2, b[2], b[3]);
      }
      // d: rows g (d[0], d[1]) and g+8 (d[2], d[3]), columns 2t and 2t+1
      const int blk = b0 + i;
#pragma unroll
      for (int m = 0; m < NM; ++m) {
        const float s0 = bf16_to_f32(ssc[(m * 16 + g) * nb + blk]);
        const float s1 = bf16_to_f32(ssc[(m * 16 + g + 8) * nb + blk]);
        acc[m][0] = fmaf(s0, d[m][0] + db[0], acc[m][0]);
        acc[m][1] = fmaf(s0, d[m][1] + db[1], acc[m][1]);
        acc[m][2] = fmaf(s1, d[m][2] + db[2], acc[m][2]);
        acc[m][3] = fmaf(s1, d[m][3] + db[3], acc[m][3]);
      }
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
    {
      const int r = threadIdx.x >> 3, col = threadIdx.x & 7;   // 128 threads: one (row, column) of a tile
      auto wsum = [&](int m, int cc) {
        return ((red[0][m][r][cc] + red[1][m][r][cc]) + red[2][m][r][cc]) + red[3][m][r][cc];
      };
      if constexpr (GU) {
#pragma unroll
        for (int p = 0; p < NM / 2; ++p) {
          const int row = rbase[2 * p] + r;
          if (col < nt && row < rows) {
            const float hv = silu(wsum(2 * p, col)) * wsum(2 * p + 1, col);
            const uint16_t hi = f32_to_bf16(hv);
            uint16_t* hrow = reinterpret_cast<uint16_t*>(hbuf + (size_t)(c0 + col) * I);
            hrow[row] = hi;
            hrow[I + row] = f32_to_bf16(hv - bf16_to_f32(hi));
          }
        }
      } else {
        if (col < nt) {
#pragma unroll
          for (int m = 0; m < NM; ++m) {
            const int row = rbase[m] + r;
            if (row < rows) ybuf[(size_t)(c0 + col) * H + row] = wsum(m, col) + wsum(m, col + 4);
          }
        }
      }
    }
    __syncthreads();
  }
}

template <typename... KArgs, typename... Args>
cudaError_t launch_smem(void (*kern)(KArgs...), dim3 grid, size_t smem, cudaStream_t s, bool dependent,
                        Args... args) {
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = dim3(kQThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = dependent ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, kern, static_cast<KArgs>(args)...);
}

}  // namespace

cudaError_t launch_ffn_int4_mma(const void* x, int T, int H, int I, int k, const ExpertList& list, const int* offsets,
                                const int* perm, float* h, float* y, cudaStream_t s, cudaEvent_t between,
                                int /*max_pairs_per_expert*/) {
  if (list.n <= 0 || T <= 0) return cudaSuccess;
  if (H % 128 || I % 128) return cudaErrorInvalidValue;
  const uint16_t* xb = static_cast<const uint16_t*>(x);
  const unsigned gu_ctas = (unsigned)((I + 16 * (kGuTiles / 2) - 1) / (16 * (kGuTiles / 2)));
  cudaError_t e = launch_smem(int4_mma_kernel<0, kGuTiles>, dim3(gu_ctas, list.n), Int4Smem<kGuTiles>::bytes(H / 128),
                              s, false, xb, T, H, I, k, list, offsets, perm, h, y);
  if (e != cudaSuccess) return e;
  if (between) cudaEventRecord(between, s);
  const unsigned down_ctas = (unsigned)((H + 16 * kDownTiles - 1) / (16 * kDownTiles));
  return launch_smem(int4_mma_kernel<1, kDownTiles>, dim3(down_ctas, list.n), Int4Smem<kDownTiles>::bytes(I / 128),
                     s, true, xb, T, H, I, k, list, offsets, perm, h, y);
}

}  // namespace ftk

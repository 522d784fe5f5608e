// K3 for decode with bf16 expert weights, on the bf16 tensor cores.
//
// Method ("FreeToken linux", "FreeToken's MoE memory handling"): each selected expert runs
// from its cache slot; h = silu(W_gate x) * (W_up x), y = W_down h.  At decode sizes every
// weight byte is read once per launch and the pass is bound by HBM: the kernel's job is to
// keep enough bytes in flight and issue little else.
//
// Operands.  The bf16 weight words are the A fragments of mma.sync.m16n8k16 as loaded (no
// conversion); the products are exact in the fp32 accumulators.  The gate/up pass reads the
// tokens x (bf16) as they are.  Between the passes a small kernel rewrites the h rows (fp32)
// in place as bf16 hi = bf16(h) and lo = bf16(h - hi) ([I hi][I lo] in the row's 4I bytes),
// and the down pass multiplies both: h keeps 16 significant bits (relative error at most
// 2^-17).
//
// Fragments (m16n8k16, 16-bit).  Lane (g, t) = (lane / 4, lane % 4) holds 16 bytes of weight
// rows g and g+8 per group of 32 reduction-axis elements: elements 8t .. 8t+7, as words w0..w3
// of two elements each.  MMA h (0, 1) takes words 2h and 2h+1: A registers a0 / a2 from row g,
// a1 / a3 from row g+8.  The MMA's reduction index is a permutation of the physical one, and
// the inputs, in their natural order, follow it: B registers b0, b1 of MMA h are input words
// 2h and 2h+1 of the lane's 16 bytes of column g (elements 8t + 4h .. 8t + 4h + 3).
//
// Memory pipeline: as the int4 and NVFP4 kernels (lane-private cp.async ring of S stages,
// input slots for the launch's token columns only, 4 warps per CTA for gate/up and 1 for
// down, partial sums added in warp order).  The down pass is a programmatic dependent of the
// h slicing, and copies its first weight groups before griddepcontrol.wait.
#include "decode_gemv.cuh"
#include "gemv_ring.cuh"

namespace ftk {

namespace {

using namespace gemv;
using namespace ring;

#ifndef FT_BF16MMA_GU_WARPS
#define FT_BF16MMA_GU_WARPS 4
#endif
#ifndef FT_BF16MMA_DOWN_WARPS
#define FT_BF16MMA_DOWN_WARPS 1
#endif
constexpr int kWarpsPerSm = 16;   // resident warps per SM: caps the registers
constexpr int kDownTiles = 2;     // 16-row tiles of a down CTA
constexpr int kNtok = 8;          // tokens (MMA columns) per pass
constexpr int kGroup = 32;        // reduction-axis elements per group (16 bytes per lane and row)

// d (16x8 f32) += A (16x16 bf16) * B (16x8 bf16).
FT_DEVICE void mma_bf16(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3, uint32_t b0, uint32_t b1) {
  asm("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// The h rows of the list's pairs (fp32 [rows][I] written by the gate/up pass), in place as
// [I bf16 hi][I bf16 lo] within the row's 4I bytes.  Grid (n_list, rows_max).
__global__ void __launch_bounds__(kPrepThreads) bf16_split_h_kernel(const __grid_constant__ ExpertList list, int T,
                                                                    int k, int I, const int* __restrict__ offsets,
                                                                    float* __restrict__ hbuf) {
  extern __shared__ float vals[];   // I floats
  asm volatile("griddepcontrol.wait;" ::: "memory");
  const int e = list.expert[blockIdx.x];
  const int q0 = e >= 0 ? offsets[e] : T * k;
  const int n = e >= 0 ? offsets[e + 1] - q0 : T;
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  if ((int)blockIdx.y >= n) return;   // the same for the whole CTA
  float* row = hbuf + (size_t)(q0 + blockIdx.y) * I;
  for (int i = threadIdx.x; i < I; i += kPrepThreads) vals[i] = __ldcg(row + i);
  __syncthreads();   // every read of the row before the writes
  uint16_t* hi = reinterpret_cast<uint16_t*>(row);
  uint16_t* lo = hi + I;
  for (int i = threadIdx.x; i < I; i += kPrepThreads) {
    const float v = vals[i];
    const uint16_t b = f32_to_bf16(v);
    hi[i] = b;
    lo[i] = f32_to_bf16(v - bf16_to_f32(b));
  }
}

// Per CTA: per warp a ring of S stages (the warps' partial sums reuse its bytes once every
// warp has drained its ring).  A stage is 2 NM weight chunks x 32 lanes x 16 bytes
// (chunk-major), then the input bytes of ncols columns: 64 bytes each (32 bf16) for gate/up,
// 128 for down (32 hi, then 32 lo), so that a quarter-warp's 8 lanes (columns g, g+1) read 8
// distinct bank groups (see xslot).
template <int MODE, int NM, int S, int W>
struct Bf16Smem {
  static constexpr int kPieces = MODE == 0 ? 4 : 8;   // 16-byte pieces of a column per group
  __host__ __device__ static constexpr size_t wbytes() { return (size_t)2 * NM * 32 * 16; }
  __host__ __device__ static constexpr size_t stage_bytes(int ncols) { return wbytes() + (size_t)ncols * kPieces * 16; }
  __host__ __device__ static constexpr size_t ring_bytes(int ncols) { return (size_t)W * S * stage_bytes(ncols); }
  __host__ __device__ static constexpr size_t red_bytes() { return (size_t)W * NM * 16 * 8 * sizeof(float); }
  __host__ __device__ static constexpr size_t bytes(int ncols) {
    return ring_bytes(ncols) > red_bytes() ? ring_bytes(ncols) : red_bytes();
  }
};

// MODE 0: gate/up + SwiGLU into h (fp32, then split by bf16_split_h_kernel); MODE 1: down into
// y.  x: the tokens (bf16 [T][H]).  ncols (1..8): token columns per pass, at least the most
// pairs of any listed expert for one pass per expert.  Grid (ceil(rows / rows per CTA),
// list.n), 32 W threads, Bf16Smem<MODE, NM, S, W>::bytes(ncols) bytes of shared memory.
template <int MODE, int NM, int S, int W>
__global__ void __launch_bounds__(32 * W, kWarpsPerSm / W)
bf16_mma_kernel(const uint16_t* __restrict__ x, int T, int H, int I, int k, const __grid_constant__ ExpertList list,
                const int* __restrict__ offsets, const int* __restrict__ perm, float* __restrict__ hbuf,
                float* __restrict__ ybuf, int ncols) {
  constexpr bool GU = MODE == 0;
  using L = Bf16Smem<MODE, NM, S, W>;
  extern __shared__ __align__(16) unsigned char smem[];
  float (*red)[NM][16][8] = reinterpret_cast<float (*)[NM][16][8]>(smem);   // over the ring

  const int e = list.expert[blockIdx.y];
  const uint8_t* blob = list.blob[blockIdx.y];
  const int K = GU ? H : I, rows = GU ? I : H;
  const int rows_cta = GU ? 16 * (NM / 2) : 16 * NM;
  const int row0 = blockIdx.x * rows_cta;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
  const size_t mat = (size_t)H * I;
  const size_t row_bytes = (size_t)K * 2;
  const int nb = K / kGroup;
  const int b0 = warp * nb / W, b1 = (warp + 1) * nb / W, nblk = b1 - b0;
  int rbase[NM];
  const uint8_t* wsrc[2 * NM];   // this lane's 16 bytes of rows g ([2m]) and g+8 ([2m+1]) of tile m, group b0
#pragma unroll
  for (int m = 0; m < NM; ++m) {
    const uint8_t* wm = GU ? blob + (m & 1) * (mat * 2) : blob + 2 * (mat * 2);
    rbase[m] = GU ? row0 + 16 * (m >> 1) : row0 + 16 * m;
    wsrc[2 * m] = wm + (size_t)min(rbase[m] + g, rows - 1) * row_bytes + t * 16 + (size_t)b0 * 64;
    wsrc[2 * m + 1] = wm + (size_t)min(rbase[m] + g + 8, rows - 1) * row_bytes + t * 16 + (size_t)b0 * 64;
  }
  const uint32_t sbytes = (uint32_t)L::stage_bytes(ncols);
  const uint32_t ring_w = smem_u32(smem) + (uint32_t)warp * S * sbytes + (uint32_t)lane * 16;
  const uint32_t ring_x = smem_u32(smem) + (uint32_t)warp * S * sbytes + (uint32_t)L::wbytes();
  constexpr uint32_t kColBytes = L::kPieces * 16;

  const int q0 = e >= 0 ? offsets[e] : T * k;
  const int q1 = e >= 0 ? offsets[e + 1] : T * k + T;
  if (GU) asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  if (q1 <= q0 || row0 >= rows) {
    if (!GU) asm volatile("griddepcontrol.wait;" ::: "memory");
    return;
  }
  auto issue_w = [&](int i, uint32_t st_off) {
#pragma unroll
    for (int c = 0; c < 2 * NM; ++c) cp16s(ring_w + st_off + 512 * c, wsrc[c] + (size_t)i * 64);
  };
  // the input column of lane g, group b0 + i: its 16 bytes (elements 8t .. 8t+7); down: of hi
  // and of lo.  Slot of part u (0 hi, 1 lo), piece t: (4u + t) ^ (4 (g & 1)) for down, t ^ 0
  // for gate/up (two 64-byte columns already fill a quarter-warp's 8 bank groups).
  auto xslot = [&](int gg, int u) {
    return (uint32_t)(gg * kColBytes + 16 * (GU ? t : ((4 * u + t) ^ (4 * (gg & 1)))));
  };
  const uint32_t xo0 = xslot(g, 0), xo1 = xslot(g, 1);
  auto issue_x = [&](int i, uint32_t st_off, const unsigned char* src) {
    const unsigned char* p = src + (size_t)(b0 + i) * 64 + 16 * t;
    cp16s(ring_x + st_off + xo0, p);
    if constexpr (!GU) cp16s(ring_x + st_off + xo1, p + 2 * (size_t)I);   // the lo half
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
    // down: before this point only the weights and the routing (ready before the kernel before)
    if (!GU && first) asm volatile("griddepcontrol.wait;" ::: "memory");
    first = false;
    const unsigned char* src = reinterpret_cast<const unsigned char*>(x);
    if (valid) {
      const int q = c0 + g;
      if constexpr (GU) src = reinterpret_cast<const unsigned char*>(x + (size_t)(e >= 0 ? perm[q] / k : q - T * k) * H);
      else src = reinterpret_cast<const unsigned char*>(hbuf + (size_t)q * I);
    }
#pragma unroll 1
    for (int i = 0; i < S - 1; ++i) {
      if (valid && i < nblk) issue_x(i, i * sbytes, src);
      cp_commit();
    }
    // lanes past the pass's columns read column 0 (copied by lanes 0-3); their MMA columns are
    // discarded
    const int gx = valid ? g : 0;
    const uint32_t xr0 = ring_x + xslot(gx, 0), xr1 = ring_x + xslot(gx, 1);

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
      const uint4 xh = lds128(xr0 + st_off);
      uint4 xl = make_uint4(0u, 0u, 0u, 0u);
      if constexpr (!GU) xl = lds128(xr1 + st_off);
#pragma unroll
      for (int m = 0; m < NM; ++m) {
        const uint4 wg = lds128(ring_w + st_off + 512 * (2 * m)), wg8 = lds128(ring_w + st_off + 512 * (2 * m + 1));
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const uint32_t a0 = word_of(wg, 2 * h), a1 = word_of(wg8, 2 * h);
          const uint32_t a2 = word_of(wg, 2 * h + 1), a3 = word_of(wg8, 2 * h + 1);
          mma_bf16(acc[m], a0, a1, a2, a3, word_of(xh, 2 * h), word_of(xh, 2 * h + 1));
          if constexpr (!GU) mma_bf16(acc[m], a0, a1, a2, a3, word_of(xl, 2 * h), word_of(xl, 2 * h + 1));
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
        if constexpr (GU) {
#pragma unroll
          for (int p = 0; p < NM / 2; ++p) {
            const int row = rbase[2 * p] + r;
            if (row < rows) hbuf[(size_t)q * I + row] = silu(wsum(2 * p, col)) * wsum(2 * p + 1, col);
          }
        } else {
#pragma unroll
          for (int m = 0; m < NM; ++m) {
            const int row = rbase[m] + r;
            if (row < rows) ybuf[(size_t)q * H + row] = wsum(m, col);
          }
        }
      }
    }
    __syncthreads();
  }
}

// Stages of the ring for a pass of ncols token columns: the most (up to 5) with which
// kWarpsPerSm / W CTAs fit on an SM (of its 228 KB, less 1 KB reserved per CTA).
template <int MODE, int NM, int W>
int bf16_stages(int ncols) {
  constexpr size_t kBudget = 228 * 1024 / (kWarpsPerSm / W) - 1024;
  return Bf16Smem<MODE, NM, 5, W>::bytes(ncols) <= kBudget   ? 5
         : Bf16Smem<MODE, NM, 4, W>::bytes(ncols) <= kBudget ? 4
                                                             : 3;
}

template <int MODE, int NM, int W, typename... Args>
cudaError_t launch_b16(int ncols, dim3 grid, cudaStream_t s, bool dependent, Args... args) {
  switch (bf16_stages<MODE, NM, W>(ncols)) {
    case 5:
      return launch_ex(bf16_mma_kernel<MODE, NM, 5, W>, grid, dim3(32 * W), Bf16Smem<MODE, NM, 5, W>::bytes(ncols), s,
                       dependent, args..., ncols);
    case 4:
      return launch_ex(bf16_mma_kernel<MODE, NM, 4, W>, grid, dim3(32 * W), Bf16Smem<MODE, NM, 4, W>::bytes(ncols), s,
                       dependent, args..., ncols);
    default:
      return launch_ex(bf16_mma_kernel<MODE, NM, 3, W>, grid, dim3(32 * W), Bf16Smem<MODE, NM, 3, W>::bytes(ncols), s,
                       dependent, args..., ncols);
  }
}
}  // namespace

cudaError_t launch_ffn_bf16_mma(const void* x, int T, int H, int I, int k, const ExpertList& list, const int* offsets,
                                const int* perm, float* h, float* y, cudaStream_t s, cudaEvent_t between,
                                int max_pairs_per_expert) {
  if (list.n <= 0 || T <= 0) return cudaSuccess;
  if (H % kGroup || I % kGroup) return cudaErrorInvalidValue;
  int has_shared = 0;
  for (int i = 0; i < list.n; ++i) has_shared |= list.expert[i] < 0;
  int rows_max = max_pairs_per_expert < 1 ? T * k : max_pairs_per_expert;
  if (has_shared && T > rows_max) rows_max = T;
  const int ncols = rows_max < kNtok ? rows_max : kNtok;
  cudaError_t e = launch_b16<0, 2, FT_BF16MMA_GU_WARPS>(ncols, dim3((I + 15) / 16, list.n), s, false,
                                                        static_cast<const uint16_t*>(x), T, H, I, k, list, offsets,
                                                        perm, h, y);
  if (e != cudaSuccess) return e;
  if (between) cudaEventRecord(between, s);
  e = launch_ex(bf16_split_h_kernel, dim3(list.n, rows_max), dim3(kPrepThreads), (size_t)I * sizeof(float), s, true,
                list, T, k, I, offsets, h);
  if (e != cudaSuccess) return e;
  const unsigned down_ctas = (unsigned)((H + 16 * kDownTiles - 1) / (16 * kDownTiles));
  return launch_b16<1, kDownTiles, FT_BF16MMA_DOWN_WARPS>(ncols, dim3(down_ctas, list.n), s, true,
                                                          static_cast<const uint16_t*>(x), T, H, I, k, list, offsets,
                                                          perm, h, y);
}

}  // namespace ftk

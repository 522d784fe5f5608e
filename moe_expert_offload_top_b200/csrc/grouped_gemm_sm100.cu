// K4 - grouped SwiGLU expert GEMMs for prefill on the 5th-generation tensor
// cores (tcgen05 + TMEM), fed by TMA from the expert-slot arena.
//
// Method ("FreeToken linux", "FreeToken's MoE memory handling"): in prefill
// many tokens reach each expert, and every selected expert runs from the slot
// that holds it while the next layer's experts are copied in.  Expert FFN
// (stated workloads): h = silu(A W_gate^T) * (A W_up^T) in bf16, y = h W_down^T
// in fp32, with A the expert's gathered token rows.
//
// One persistent kernel per GEMM, one CTA per SM:
//   warp 0  TMA producer: A tile [128 x 64] bf16 and the B tile per stage, no
//           multicast (every CTA loads its own tiles from this GPU's memory).
//           bf16 weights: B [256 x 64] bf16 with 128-byte swizzle, 4 stages.
//           NVFP4 weights: the B tile's packed e2m1 codes [256 x 32 bytes] and,
//           every fourth stage, its e4m3 block scales for the next 256 columns
//           [256 x 16 bytes], 3 stages.
//   warp 1  MMA issuer: tcgen05.mma.cta_group::1.kind::f16, M=128, N=256,
//           K=16, fp32 accumulators in TMEM, two accumulator buffers of 256
//           columns so the epilogue of one tile overlaps the next tile's MMAs.
//   warps 2-5  epilogue: tcgen05.ld 32x32b rows of the accumulator, SwiGLU
//           (gate/up) or plain (down), masked row stores to global memory.
//   warps 6-9  (NVFP4 only) expansion: each stage's codes times their block scales
//           become the bf16 B tile, written in the 128-byte-swizzled layout the MMA
//           reads, then handed to the MMA warp through the async proxy.  An e2m1
//           value (2 significant bits) times an e4m3 scale (4) has at most 6
//           significant bits and lies in bf16's range, so the operand is exact; the
//           fp32 scale of each matrix multiplies the accumulator in the epilogue.
// Tiles: per group (a selected expert or the shared expert) ceil(rows/128)
// M-tiles times the N-tiles of the output, N-major inside a group so that the
// M-tiles sharing one weight tile run back to back.  An M-tile may read rows
// of the next group; those rows are computed and never stored.
//
// Every wait on an mbarrier is bounded: on timeout the thread records an error
// code in *err, sets the CTA's abort flag, and all roles drain and leave; the
// TMEM columns are always released.
#include <cuda.h>
#include <cuda_fp16.h>

#include "common.cuh"
#include "kernels.hpp"
#include "sm100_sync.cuh"

namespace ftk {

namespace {

constexpr int BM = 128, BN = 256, BK = 64;
constexpr int A_BYTES = BM * BK * 2;      // 16 KB
constexpr int B_BYTES = BN * BK * 2;      // 32 KB
constexpr int TMEM_COLS = 512;            // two 128 x 256 fp32 accumulators
constexpr int MAX_STAGES = 4;

// Per weight format: pipeline stages, threads, and the raw bytes of a B tile's codes.
template <int WT> struct GemmCfg;
template <> struct GemmCfg<GW_BF16> {
  static constexpr int STAGES = 4, THREADS = 192, RAW = 0, SCALE_RING = 0;
};
template <> struct GemmCfg<GW_NVFP4> {
  static constexpr int STAGES = 3, THREADS = 320, RAW = BN * BK / 2;   // 8 KB of e2m1 codes
  static constexpr int SCALE_RING = 2 * BN * 16;                       // two blocks of 4 stages' scales
};
template <int WT> constexpr int stage_bytes() { return A_BYTES + B_BYTES + GemmCfg<WT>::RAW; }

struct GemmSmem {
  uint64_t full[MAX_STAGES], empty[MAX_STAGES], conv[MAX_STAGES], tfull[2], tempty[2];
  uint32_t tmem_base;
  int abort;
  int mt_start[kMaxList + 1];   // prefix of M-tiles over groups
  int row_start[kMaxList];
  int rows[kMaxList];
};

FT_DEVICE void tma_load_2d(void* dst, const CUtensorMap* map, uint64_t* bar, int c0, int c1) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4}], [%2];"
      ::"r"(smem_u32(dst)), "l"((uint64_t)map), "r"(smem_u32(bar)), "r"(c0), "r"(c1)
      : "memory");
}
FT_DEVICE void tma_load_3d(void* dst, const CUtensorMap* map, uint64_t* bar, int c0, int c1, int c2) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4, %5}], [%2];"
      ::"r"(smem_u32(dst)), "l"((uint64_t)map), "r"(smem_u32(bar)), "r"(c0), "r"(c1), "r"(c2)
      : "memory");
}

// Shared-memory matrix descriptor: K-major, 128-byte swizzle, 8-row groups 1024 B apart.
FT_DEVICE uint64_t smem_desc(uint32_t addr) {
  uint64_t d = 0;
  d |= (uint64_t)((addr >> 4) & 0x3FFF);          // start address
  d |= (uint64_t)1 << 16;                         // leading byte offset (unused with swizzle)
  d |= (uint64_t)(1024 >> 4) << 32;               // stride byte offset
  d |= (uint64_t)1 << 46;                         // descriptor version (sm_100)
  d |= (uint64_t)2 << 61;                         // swizzle: 128 B
  return d;
}

// Instruction descriptor: kind::f16, bf16 x bf16 -> f32, A and B K-major, M x N.
__host__ __device__ constexpr uint32_t idesc_bf16(int M, int N) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

FT_DEVICE void mma_bf16(uint32_t d_tmem, uint64_t a, uint64_t b, uint32_t idesc, uint32_t acc) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}"
      ::"r"(d_tmem), "l"(a), "l"(b), "r"(idesc), "r"(acc));
}
FT_DEVICE void mma_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];"
               ::"r"(smem_u32(bar)) : "memory");
}
FT_DEVICE void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
FT_DEVICE void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

FT_DEVICE void tmem_ld32(uint32_t taddr, float* v) {
  uint32_t r[32];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]),
        "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]),
        "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}

// Two e2m1 codes of `byte`, times the f16 pair `sp` (a block scale in both halves), as one
// bf16 pair: the e2m1 pair converts exactly to f16, the product is exact in f16 (at most
// 6 significant bits, magnitudes 2^-10 .. 2688), and each f16 converts exactly to bf16.
FT_DEVICE uint32_t e2m1x2_times(uint32_t byte, uint32_t sp) {
  uint32_t h2, p2, o;
  asm("{ .reg .b8 t; cvt.u8.u32 t, %1; cvt.rn.f16x2.e2m1x2 %0, t; }" : "=r"(h2) : "r"(byte));
  asm("mul.rn.f16x2 %0, %1, %2;" : "=r"(p2) : "r"(h2), "r"(sp));
  const float lo = __half2float(__ushort_as_half((unsigned short)(p2 & 0xFFFFu)));
  const float hi = __half2float(__ushort_as_half((unsigned short)(p2 >> 16)));
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(o) : "f"(hi), "f"(lo));
  return o;
}

// MODE 0: gate/up + SwiGLU (B = [W_gate rows n0..n0+127 ; W_up rows n0..n0+127], out = h bf16 [rows][I])
// MODE 1: down (B = W_down rows n0..n0+255, out = y f32 [rows][H])
// WT: GW_BF16 (B read as bf16 through tmBr / tmBs) or GW_NVFP4 (codes and scales through
// fp4's maps, expanded in shared memory; tmBr / tmBs unused).
template <int MODE, int WT>
__global__ void __launch_bounds__(GemmCfg<WT>::THREADS, 1)
grouped_gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmBr,
                    const __grid_constant__ CUtensorMap tmBs, const __grid_constant__ GemmGroups groups,
                    const __grid_constant__ GemmFp4 fp4, const int* __restrict__ offsets, int T, int k, int I,
                    int H, void* __restrict__ out, int* __restrict__ err) {
  constexpr int STAGES = GemmCfg<WT>::STAGES;
  constexpr int STAGE_BYTES = stage_bytes<WT>();
  constexpr bool FP4 = WT == GW_NVFP4;
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* base = (unsigned char*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  unsigned char* scale_ring = base + STAGES * STAGE_BYTES;   // NVFP4: [2][BN rows][16 bytes]
  GemmSmem* S = reinterpret_cast<GemmSmem*>(scale_ring + GemmCfg<WT>::SCALE_RING);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int K = MODE == 0 ? H : I;
  const int KB = K / BK;
  const int n_tiles = MODE == 0 ? I / (BN / 2) : H / BN;
  const int ld_out = MODE == 0 ? I : H;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&S->full[s], 1);
      mbar_init(&S->empty[s], 1);
      mbar_init(&S->conv[s], 128);
    }
    for (int b = 0; b < 2; ++b) { mbar_init(&S->tfull[b], 1); mbar_init(&S->tempty[b], 128); }
    S->abort = 0;
    int acc = 0;
    for (int g = 0; g < groups.n; ++g) {
      const int e = groups.expert[g];
      const int r0 = e >= 0 ? offsets[e] : T * k;
      const int nr = e >= 0 ? offsets[e + 1] - r0 : T;
      S->row_start[g] = r0;
      S->rows[g] = nr;
      S->mt_start[g] = acc;
      acc += (nr + BM - 1) / BM;
    }
    S->mt_start[groups.n] = acc;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  }
  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
                 ::"r"(smem_u32(&S->tmem_base)), "r"(TMEM_COLS));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = S->tmem_base;
  const int total_tiles = S->mt_start[groups.n] * n_tiles;
  volatile int* abort_flag = &S->abort;

  // tile -> (group, m-tile, n-tile)
  auto decode = [&](int t, int& g, int& m, int& n) {
    int lo = 0, hi = groups.n - 1;
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (S->mt_start[mid] * n_tiles <= t) lo = mid; else hi = mid - 1;
    }
    g = lo;
    const int local = t - S->mt_start[g] * n_tiles;
    const int mtg = S->mt_start[g + 1] - S->mt_start[g];
    n = local / mtg;
    m = local - n * mtg;
  };

  if (warp == 0) {
    if (lane == 0) {   // ---------------------------------------------- TMA producer
      int it = 0, sblk = 0;
      for (int t = blockIdx.x; t < total_tiles && !*abort_flag; t += gridDim.x) {
        int g, m, n;
        decode(t, g, m, n);
        const int row0 = S->row_start[g] + m * BM;
        const bool sh = groups.expert[g] < 0;
        const int z = groups.z[g];
        // B rows of the tile: gate rows n*128.. and up rows I + n*128.., or down rows n*256..
        const int br0 = MODE == 0 ? n * (BN / 2) : n * BN;
        const int br1 = MODE == 0 ? I + n * (BN / 2) : n * BN + BN / 2;
        bool stop = false;
        for (int kb = 0; kb < KB; ++kb, ++it) {
          const int s = it % STAGES;
          const uint32_t par = ((it / STAGES) & 1) ^ 1;
          if (!mbar_wait(&S->empty[s], par, abort_flag, err, 101)) { stop = true; break; }
          unsigned char* sa = base + s * STAGE_BYTES;
          unsigned char* sb = sa + A_BYTES;
          if constexpr (!FP4) {
            const CUtensorMap* mb = sh ? &tmBs : &tmBr;
            mbar_expect_tx(&S->full[s], A_BYTES + B_BYTES);
            tma_load_2d(sa, &tmA, &S->full[s], kb * BK, row0);
            if (MODE == 0) {   // boxes of 128 rows: gate rows, then up rows
              tma_load_3d(sb, mb, &S->full[s], kb * BK, br0, z);
              tma_load_3d(sb + B_BYTES / 2, mb, &S->full[s], kb * BK, br1, z);
            } else {           // one box of 256 down rows
              tma_load_3d(sb, mb, &S->full[s], kb * BK, br0, z);
            }
          } else {
            const CUtensorMap* mq = sh ? &fp4.q_shared[MODE] : &fp4.q_routed[MODE];
            const CUtensorMap* ms = sh ? &fp4.s_shared[MODE] : &fp4.s_routed[MODE];
            unsigned char* raw = sb + B_BYTES;
            const bool scales = (kb & 3) == 0;   // a new block of 4 stages' block scales
            mbar_expect_tx(&S->full[s], A_BYTES + GemmCfg<WT>::RAW + (scales ? BN * 16 : 0));
            tma_load_2d(sa, &tmA, &S->full[s], kb * BK, row0);
            tma_load_3d(raw, mq, &S->full[s], kb * (BK / 2), br0, z);
            tma_load_3d(raw + GemmCfg<WT>::RAW / 2, mq, &S->full[s], kb * (BK / 2), br1, z);
            if (scales) {
              unsigned char* sdst = scale_ring + (sblk & 1) * (BN * 16);
              tma_load_3d(sdst, ms, &S->full[s], (kb / 4) * 16, br0, z);
              tma_load_3d(sdst + BN / 2 * 16, ms, &S->full[s], (kb / 4) * 16, br1, z);
              ++sblk;
            }
          }
        }
        if (stop) break;
      }
      // drain: wait (bounded) until every issued stage has landed
      const int issued = it;
      for (int j = issued - STAGES < 0 ? 0 : issued - STAGES; j < issued; ++j) {
        mbar_drain(&S->full[j % STAGES], (j / STAGES) & 1);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {   // ---------------------------------------------- MMA issuer
      constexpr uint32_t idesc = idesc_bf16(BM, BN);
      int it = 0, tl = 0;
      for (int t = blockIdx.x; t < total_tiles && !*abort_flag; t += gridDim.x, ++tl) {
        const int b = tl & 1;
        if (!mbar_wait(&S->tempty[b], ((tl >> 1) & 1) ^ 1, abort_flag, err, 102)) break;
        tc_fence_after();
        const uint32_t d = tmem + b * BN;
        bool ok = true;
        for (int kb = 0; kb < KB; ++kb, ++it) {
          const int s = it % STAGES;
          if (!mbar_wait(&S->full[s], (it / STAGES) & 1, abort_flag, err, 103)) { ok = false; break; }
          if (FP4 && !mbar_wait(&S->conv[s], (it / STAGES) & 1, abort_flag, err, 106)) { ok = false; break; }
          tc_fence_after();
          const uint32_t sa = smem_u32(base + s * STAGE_BYTES);
          const uint32_t sb = sa + A_BYTES;
#pragma unroll
          for (int kk = 0; kk < BK / 16; ++kk)
            mma_bf16(d, smem_desc(sa + kk * 32), smem_desc(sb + kk * 32), idesc, (kb | kk) ? 1u : 0u);
          mma_commit(&S->empty[s]);
        }
        if (!ok) break;
        mma_commit(&S->tfull[b]);
      }
    }
  } else if (warp < 6) {   // ------------------------------------------ epilogue (warps 2..5)
    const int q = warp & 3;                   // TMEM lane quarter this warp may access
    const int r = q * 32 + lane;              // tile row of this thread
    int tl = 0;
    for (int t = blockIdx.x; t < total_tiles && !*abort_flag; t += gridDim.x, ++tl) {
      int g, m, n;
      decode(t, g, m, n);
      const int b = tl & 1;
      if (!mbar_wait(&S->tfull[b], (tl >> 1) & 1, abort_flag, err, 104)) break;
      tc_fence_after();
      const int valid = S->rows[g] - m * BM;
      const int row = S->row_start[g] + m * BM + r;
      const uint32_t tbase = tmem + ((uint32_t)(q * 32) << 16) + b * BN;
      // NVFP4: the fp32 scales of gate, up and down, stored in the expert's blob
      float sg = 1.f, su = 1.f, sd = 1.f;
      if constexpr (FP4) {
        const uint8_t* gb = (groups.expert[g] < 0 ? fp4.g_shared : fp4.g_routed) +
                            (size_t)groups.z[g] * fp4.blob + fp4.g_off;
        const float* gl = reinterpret_cast<const float*>(gb);
        sg = gl[0]; su = gl[1]; sd = gl[2];
      }
      if (MODE == 0) {
        uint16_t* hout = static_cast<uint16_t*>(out) + (size_t)row * ld_out + n * (BN / 2);
#pragma unroll 1
        for (int j = 0; j < BN / 2; j += 32) {
          float u[32], v[32];
          tmem_ld32(tbase + j, u);
          tmem_ld32(tbase + BN / 2 + j, v);
          if constexpr (FP4) {
#pragma unroll
            for (int i = 0; i < 32; ++i) { u[i] *= sg; v[i] *= su; }
          }
          if (r < valid) {
            uint32_t pk[16];
#pragma unroll
            for (int i = 0; i < 16; ++i) {
              const float h0 = silu(u[2 * i]) * v[2 * i], h1 = silu(u[2 * i + 1]) * v[2 * i + 1];
              pk[i] = (uint32_t)f32_to_bf16(h0) | ((uint32_t)f32_to_bf16(h1) << 16);
            }
            uint4* dst = reinterpret_cast<uint4*>(hout + j);
#pragma unroll
            for (int i = 0; i < 4; ++i) dst[i] = make_uint4(pk[4 * i], pk[4 * i + 1], pk[4 * i + 2], pk[4 * i + 3]);
          }
        }
      } else {
        float* yout = static_cast<float*>(out) + (size_t)row * ld_out + n * BN;
#pragma unroll 1
        for (int j = 0; j < BN; j += 32) {
          float v[32];
          tmem_ld32(tbase + j, v);
          if constexpr (FP4) {
#pragma unroll
            for (int i = 0; i < 32; ++i) v[i] *= sd;
          }
          if (r < valid) {
            float4* dst = reinterpret_cast<float4*>(yout + j);
#pragma unroll
            for (int i = 0; i < 8; ++i) dst[i] = make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
          }
        }
      }
      tc_fence_before();
      mbar_arrive(&S->tempty[b]);
    }
  } else if constexpr (FP4) {   // ---------------------------------- expansion (warps 6..9)
    // 512 items per stage: B row rr (0..255) and half hf (K elements 32 hf .. 32 hf + 31 of
    // the stage): 16 bytes of codes -> 64 bytes (four 16-byte chunks) of bf16, chunk c of
    // row rr stored at rr * 128 + ((c ^ (rr & 7)) * 16) (the 128-byte swizzle); a thread
    // takes items ct, ct + 128, ct + 256, ct + 384.
    const int ct = threadIdx.x - 192;
    int it = 0, sblk = 0;
    for (int t = blockIdx.x; t < total_tiles && !*abort_flag; t += gridDim.x) {
      bool stop = false;
      for (int kb = 0; kb < KB; ++kb, ++it) {
        const int s = it % STAGES;
        if (!mbar_wait(&S->full[s], (it / STAGES) & 1, abort_flag, err, 105)) { stop = true; break; }
        if ((kb & 3) == 0) ++sblk;
        const unsigned char* sblock = scale_ring + ((sblk - 1) & 1) * (BN * 16) + (kb & 3) * 4;
        unsigned char* sb = base + s * STAGE_BYTES + A_BYTES;
        const unsigned char* raw = sb + B_BYTES;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int item = ct + 128 * i;
          const int rr = item >> 1, hf = item & 1;
          const uint4 qv = *reinterpret_cast<const uint4*>(raw + rr * 32 + hf * 16);
          const uint32_t sc2 = *reinterpret_cast<const uint16_t*>(sblock + rr * 16 + hf * 2);
          uint32_t s2;   // the two 16-element block scales as f16, each in both halves of a pair
          asm("{ .reg .b16 t; cvt.u16.u32 t, %1; cvt.rn.f16x2.e4m3x2 %0, t; }" : "=r"(s2) : "r"(sc2));
          const uint32_t s_lo = __byte_perm(s2, 0, 0x1010), s_hi = __byte_perm(s2, 0, 0x3232);
          const uint32_t w[4] = {qv.x, qv.y, qv.z, qv.w};
#pragma unroll
          for (int j = 0; j < 4; ++j) {   // word j: elements 8j .. 8j+7 of the half -> chunk 4 hf + j
            const uint32_t sp = j < 2 ? s_lo : s_hi;
            uint4 o;
            o.x = e2m1x2_times(w[j] & 0xFFu, sp);
            o.y = e2m1x2_times((w[j] >> 8) & 0xFFu, sp);
            o.z = e2m1x2_times((w[j] >> 16) & 0xFFu, sp);
            o.w = e2m1x2_times(w[j] >> 24, sp);
            const int c = 4 * hf + j;
            *reinterpret_cast<uint4*>(sb + rr * 128 + ((c ^ (rr & 7)) * 16)) = o;
          }
        }
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");   // visible to the tensor cores
        mbar_arrive(&S->conv[s]);
      }
      if (stop) break;
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 0)
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(TMEM_COLS));
}

// Self-test of the bounded wait: one thread waits on an mbarrier that nothing
// arrives on; the wait must give up after limit_ns and leave code 199 in *err.
__global__ void wait_selftest_kernel(unsigned long long limit_ns, int* err) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    mbar_wait(&bar, 0, &abort_flag, err, 199, limit_ns);
  }
}

// A rows for the grouped GEMM: A[q] = x[perm[q] / k] (q < T*k), A[T*k + t] = x[t].
__global__ void gather_rows_kernel(const uint16_t* __restrict__ x, const int* __restrict__ perm, int T,
                                   int k, int H, int with_shared, uint16_t* __restrict__ A) {
  const int rows = T * k + (with_shared ? T : 0);
  const int per_row = H / 8;
  for (long long idx = (long long)blockIdx.x * blockDim.x + threadIdx.x; idx < (long long)rows * per_row;
       idx += (long long)gridDim.x * blockDim.x) {
    const int q = (int)(idx / per_row), c = (int)(idx - (long long)q * per_row);
    const int tok = q < T * k ? perm[q] / k : q - T * k;
    reinterpret_cast<uint4*>(A + (size_t)q * H)[c] = reinterpret_cast<const uint4*>(x + (size_t)tok * H)[c];
  }
}

}  // namespace

cudaError_t launch_wait_selftest(unsigned long long limit_ns, int* err, cudaStream_t s) {
  wait_selftest_kernel<<<1, 32, 0, s>>>(limit_ns, err);
  return cudaGetLastError();
}

size_t gemm_smem_bytes(int wt) {
  return wt == GW_NVFP4
             ? 1024 + GemmCfg<GW_NVFP4>::STAGES * stage_bytes<GW_NVFP4>() + GemmCfg<GW_NVFP4>::SCALE_RING + sizeof(GemmSmem)
             : 1024 + GemmCfg<GW_BF16>::STAGES * stage_bytes<GW_BF16>() + sizeof(GemmSmem);
}

cudaError_t launch_gather_rows(const void* x, const int* perm, int T, int k, int H, bool with_shared,
                               void* A, cudaStream_t s) {
  const int rows = T * k + (with_shared ? T : 0);
  if (rows <= 0) return cudaSuccess;
  const long long n = (long long)rows * (H / 8);
  const int threads = 256;
  long long blocks = (n + threads - 1) / threads;
  if (blocks > 148 * 16) blocks = 148 * 16;
  gather_rows_kernel<<<(unsigned)blocks, threads, 0, s>>>(static_cast<const uint16_t*>(x), perm, T, k, H,
                                                         with_shared ? 1 : 0, static_cast<uint16_t*>(A));
  return cudaGetLastError();
}

namespace {
template <int MODE, int WT>
cudaError_t launch_gemm_t(const GemmMaps& maps, const GemmGroups& groups, const GemmFp4& fp4, const int* offsets,
                          int T, int k, int I, int H, void* out, int* err, int grid, cudaStream_t s) {
  const size_t smem = gemm_smem_bytes(WT);
  cudaError_t e = cudaFuncSetAttribute(grouped_gemm_kernel<MODE, WT>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)smem);
  if (e != cudaSuccess) return e;
  const CUtensorMap& a = MODE == 0 ? maps.a_x : maps.a_h;
  const CUtensorMap& br = MODE == 0 ? maps.b1_routed : maps.b2_routed;
  const CUtensorMap& bs = MODE == 0 ? maps.b1_shared : maps.b2_shared;
  grouped_gemm_kernel<MODE, WT><<<grid, GemmCfg<WT>::THREADS, smem, s>>>(a, br, bs, groups, fp4, offsets, T, k, I, H,
                                                                         out, err);
  return cudaGetLastError();
}
}  // namespace

cudaError_t launch_grouped_gemm(int mode, const GemmMaps& maps, const GemmGroups& groups, const int* offsets,
                                int T, int k, int I, int H, void* out, int* err, int num_sms, cudaStream_t s,
                                const GemmFp4* fp4) {
  if (groups.n <= 0 || T <= 0) return cudaSuccess;
  // an upper bound of the tile count; CTAs beyond the real count exit at once
  const long long rows_max = (long long)T * k + T;
  const int n_tiles = mode == 0 ? I / (BN / 2) : H / BN;
  long long tiles_max = ((rows_max + BM - 1) / BM + groups.n) * n_tiles;
  int grid = num_sms;
  if (tiles_max < grid) grid = (int)tiles_max;
  static const GemmFp4 no_fp4 = {};
  if (fp4) {
    if (H % 256 || I % 256) return cudaErrorInvalidValue;
    return mode == 0 ? launch_gemm_t<0, GW_NVFP4>(maps, groups, *fp4, offsets, T, k, I, H, out, err, grid, s)
                     : launch_gemm_t<1, GW_NVFP4>(maps, groups, *fp4, offsets, T, k, I, H, out, err, grid, s);
  }
  return mode == 0 ? launch_gemm_t<0, GW_BF16>(maps, groups, no_fp4, offsets, T, k, I, H, out, err, grid, s)
                   : launch_gemm_t<1, GW_BF16>(maps, groups, no_fp4, offsets, T, k, I, H, out, err, grid, s);
}

}  // namespace ftk

// ------------------------------------------------------------------ host side --
namespace ftk {

namespace {
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  return fn;
}
}  // namespace

bool encode_map_2d(CUtensorMap* m, const void* base, uint64_t inner, uint64_t rows, uint64_t row_bytes,
                   uint32_t box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {inner, rows};
  cuuint64_t strides[1] = {row_bytes};
  cuuint32_t box[2] = {(cuuint32_t)BK, box_rows};
  cuuint32_t es[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool encode_map_3d(CUtensorMap* m, const void* base, uint64_t inner, uint64_t rows, uint64_t depth,
                   uint64_t row_bytes, uint64_t depth_bytes, uint32_t box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {inner, rows, depth};
  cuuint64_t strides[2] = {row_bytes, depth_bytes};
  cuuint32_t box[3] = {(cuuint32_t)BK, box_rows, 1};
  cuuint32_t es[3] = {1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool encode_map_u8_3d(CUtensorMap* m, const void* base, uint64_t inner, uint64_t rows, uint64_t depth,
                      uint64_t row_bytes, uint64_t depth_bytes, uint32_t box_inner, uint32_t box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {inner, rows, depth};
  cuuint64_t strides[2] = {row_bytes, depth_bytes};
  cuuint32_t box[3] = {box_inner, box_rows, 1};
  cuuint32_t es[3] = {1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void*>(base), dims, strides, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace ftk

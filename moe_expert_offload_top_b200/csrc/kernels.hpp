// Internal launch functions of the sm_100a kernels (host side).
#pragma once
#include <cuda.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

namespace ftk {

#ifndef FT_MAX_LIST
#define FT_MAX_LIST 257
#endif
constexpr int kMaxList = FT_MAX_LIST;   // routed experts of one layer + the shared expert

// Per-launch list of experts whose FFN runs: entry i reads its weights at blob[i];
// its token pairs are offsets[expert[i]] .. offsets[expert[i]+1] of the permutation,
// or, for expert[i] == -1 (the shared expert), the T pairs T*k .. T*k+T-1 = tokens 0..T-1.
struct ExpertList {
  int n;
  int expert[kMaxList];
  const uint8_t* blob[kMaxList];
};

// K1: z[t][e] = x[t] . W_r[e] (fp32), then top-k + gates.
cudaError_t launch_router_logits(const void* x, bool x_bf16, const float* w_router, int T, int H,
                                 int E, float* logits, cudaStream_t s);
cudaError_t launch_topk_gates(const float* logits, int T, int E, int k, int gating, int* ids,
                              float* gates, cudaStream_t s);
// K1+K2 for decode (T <= 64, E <= 256, k <= 16) in one launch: logits, top-k + gates and
// the stable permutation (the last router CTA does the second part).  *ticket must be 0
// before the launch; the kernel leaves it 0.  box (optional, mapped pinned host memory of
// 2 + T*k ints): the last CTA also writes seq << 10 | value to box[2 + p] (the ids, < 1024)
// and box[1] (the low 10 bits of *err), so the host can take the routing as soon as every
// word shows the tag; seq is in 1 .. 2^21 - 1.
cudaError_t launch_route_decode(const void* x, bool x_bf16, const float* w_router, int T, int H, int E, int k,
                                int gating, float* logits, int* ids, float* gates, int* counts, int* offsets,
                                int* perm, int* inv, int* ticket, cudaStream_t s, int* box = nullptr,
                                int seq = 0, const int* err = nullptr);
// K2: stable counting sort of the T*k pairs by expert.
// inv (optional): inv[t*k+j] = position of pair (t,j) in perm.
cudaError_t launch_permute(const int* ids, int T, int k, int E, int* counts, int* offsets,
                           int* perm, int* inv, cudaStream_t s);
// K3 (decode): per list entry, gate/up + SwiGLU of its tokens into h [pairs][I] fp32,
// then the down projection into y [pairs][H] fp32.  Pairs are positions in the
// permutation (routed) or T*k + t (shared expert).  `between` (optional) is recorded
// on s between the gate/up and the down passes.
// Packed and bf16 weights run on the tensor cores unless int4_tensor is false: int4 on the
// int8 ones (launch_ffn_int4_mma), NVFP4 on the f16 ones (launch_ffn_nvfp4_mma, H and I
// multiples of 128), bf16 on the bf16 ones (launch_ffn_bf16_mma, H and I multiples of 32, T >= 2).  The h rows of
// the list's pairs are then left as sliced inputs (see below), and int4_xs
// (int4_sliced_x_bytes(T, H) bytes) receives the sliced tokens, or, when null, the front of
// y does (before the down pass writes y).
cudaError_t launch_ffn_decode(const void* x, int T, int H, int I, int k, int wdtype,
                              const ExpertList& list, int max_pairs_per_expert, const int* offsets,
                              const int* perm, float* h, float* y, cudaStream_t s,
                              cudaEvent_t between = nullptr, int* err = nullptr, bool int4_tensor = true,
                              void* int4_xs = nullptr);
// K3 (decode) for int4 group-128 weights on the int8 tensor cores (gemv_int4_mma.cu); x bf16.
// The tokens and, after the gate/up pass, the h rows of the list's pairs are written as
// 16-bit block fixed point split into a signed and an unsigned byte per value (a sliced row:
// hi bytes, lo bytes, then a float), the tokens into xsliced (or the front of y when null), the
// h rows in place.  max_pairs_per_expert: the most pairs one entry owns.
cudaError_t launch_ffn_int4_mma(const void* x, int T, int H, int I, int k, const ExpertList& list, const int* offsets,
                                const int* perm, float* h, float* y, cudaStream_t s, cudaEvent_t between,
                                int max_pairs_per_expert, void* xsliced);
// Bytes of the sliced tokens of launch_ffn_int4_mma and launch_ffn_nvfp4_mma.
size_t int4_sliced_x_bytes(int T, int H);
// K3 (decode) for NVFP4 weights on the f16 tensor cores (gemv_nvfp4_mma.cu); x bf16.  The
// tokens and, after the gate/up pass, the h rows of the list's pairs are written as f16 rows
// with a per-row power-of-two scale (then a float: the scale's inverse), the tokens into
// xsliced (or the front of y when null), the h rows in place.
cudaError_t launch_ffn_nvfp4_mma(const void* x, int T, int H, int I, int k, const ExpertList& list, const int* offsets,
                                 const int* perm, float* h, float* y, cudaStream_t s, cudaEvent_t between,
                                 int max_pairs_per_expert, void* xsliced);
// K3 (decode) for bf16 weights on the bf16 tensor cores (gemv_bf16_mma.cu); x bf16.  After the
// gate/up pass the h rows of the list's pairs are rewritten in place as bf16 hi and lo halves.
cudaError_t launch_ffn_bf16_mma(const void* x, int T, int H, int I, int k, const ExpertList& list, const int* offsets,
                                const int* perm, float* h, float* y, cudaStream_t s, cudaEvent_t between,
                                int max_pairs_per_expert);
// Kernels one launch_ffn_decode call launches for these arguments.
int ffn_decode_kernels(int wdtype, bool int4_tensor, int H, int I, int T);
// K3 + K5 (decode) in one launch (ffn_fused.cuh): gate/up + SwiGLU into h, down into y
// and, with `combine`, out[t] = sum_j gates[t][j] * y[inv[t*k+j]] (+ shared) for the
// entries of `list`.  The combine of a launch covers every pair of the forward, so
// entries not in `list` must have written their y rows earlier on the stream.
// ctl: ffn_fused_ctl_ints(H) ints of device memory, zero before the first launch
// (every launch leaves them zero); launches that use one ctl must not overlap.
// A down item waits at most limit_ns for its entry's gate/up items and otherwise
// writes 111 to *err.
struct FusedParams {
  const void* x;
  const int* offsets;
  const int* perm;
  float* h;
  float* y;
  const float* gates;
  const int* inv;
  void* out;
  int* ctl;
  int* err;
  int T, H, I, k;
  int has_shared, combine, out_bf16;
  int wait_extra;   // tests only: down items wait for this many gate/up items more than exist
  unsigned long long limit_ns;
};
int ffn_fused_ctl_ints(int H);
cudaError_t launch_ffn_fused(const FusedParams& p, int wdtype, const ExpertList& list, int max_pairs_per_expert,
                             int num_sms, cudaStream_t s);
cudaError_t launch_ffn_fused_f32(int nt, int rg, int rd, const FusedParams& p, const ExpertList& list, int num_sms,
                                 cudaStream_t s);
cudaError_t launch_ffn_fused_bf16(int nt, int rg, int rd, const FusedParams& p, const ExpertList& list, int num_sms,
                                  cudaStream_t s);
cudaError_t launch_ffn_fused_int4(int nt, int rg, int rd, const FusedParams& p, const ExpertList& list, int num_sms,
                                  cudaStream_t s);
cudaError_t launch_ffn_fused_nvfp4(int nt, int rg, int rd, const FusedParams& p, const ExpertList& list,
                                   int num_sms, cudaStream_t s);
// One thread waits until *flag >= want (the host writes the flag through mapped pinned
// memory), at most limit_ns.  Holds the stream while the host queues the launches of
// a timed stage, so that CUDA events around them time the kernels and not the host.
cudaError_t launch_hold(const volatile int* flag, int want, unsigned long long limit_ns, cudaStream_t s);

// K5: out[t] = sum_j gates[t][j] * y[inv[t*k+j]] (ascending j) + y[T*k+t] if has_shared.
cudaError_t launch_combine(const float* y, const float* gates, const int* inv, int T, int H, int k,
                           bool has_shared, bool out_bf16, void* out, cudaStream_t s);

// K4 (prefill): groups of the grouped GEMM.  Group g = routed expert expert[g] (rows
// offsets[e] .. offsets[e+1] of the gathered A) whose weights are slot z[g] of the
// arena, or the shared expert (expert[g] = -1, rows T*k .. T*k+T-1, layer z[g] of the
// shared-expert area).
struct GemmGroups {
  int n;
  int expert[kMaxList];
  int z[kMaxList];
};

// TMA descriptors of the prefill GEMMs (encoded on the host when buffers move).
struct GemmMaps {
  CUtensorMap a_x;        // gathered token rows  [rows][H] bf16, box 64 x 128
  CUtensorMap a_h;        // SwiGLU output h      [rows][I] bf16, box 64 x 128
  CUtensorMap b1_routed;  // gate|up rows of slots [C][2I][H], box 64 x 128 x 1
  CUtensorMap b1_shared;  // gate|up rows of shared experts [L][2I][H]
  CUtensorMap b2_routed;  // down rows of slots [C][H][I], box 64 x 256 x 1
  CUtensorMap b2_shared;  // down rows of shared experts [L][H][I]
};

// Weight format of the prefill GEMMs.
enum { GW_BF16 = 0, GW_NVFP4 = 1 };
// NVFP4 slots for the prefill GEMMs, expanded to bf16 inside the GEMM: tensor maps over
// the packed e2m1 codes and the e4m3 block scales of the slot arena and of the shared
// experts (index 0: the gate|up rows [2I][H/2 or H/16], 1: the down rows [H][I/2 or I/16];
// uint8, boxes of 32 or 16 bytes x 128 rows), and where each blob's three fp32 matrix
// scales lie: g_routed + z * blob + g_off (slot z), or g_shared + layer * blob + g_off.
struct GemmFp4 {
  CUtensorMap q_routed[2], q_shared[2];
  CUtensorMap s_routed[2], s_shared[2];
  const uint8_t* g_routed;
  const uint8_t* g_shared;
  unsigned long long blob;
  unsigned long long g_off;
};

size_t gemm_smem_bytes(int wt);
// One CTA waits (bounded by limit_ns) on an mbarrier nobody arrives on; sets *err = 199.
cudaError_t launch_wait_selftest(unsigned long long limit_ns, int* err, cudaStream_t s);
// A[q] = x[perm[q] / k] for q < T*k; A[T*k + t] = x[t] when with_shared (bf16 rows of H).
cudaError_t launch_gather_rows(const void* x, const int* perm, int T, int k, int H, bool with_shared,
                               void* A, cudaStream_t s);
// mode 0: h = silu(A W_gate^T) * (A W_up^T) (bf16 [rows][I]); mode 1: y = h W_down^T (f32 [rows][H]).
// bf16 weights through maps.b*; with fp4 (H, I multiples of 256), NVFP4 weights expanded in
// the GEMM, whose epilogue applies each matrix's fp32 scale.  Bounded pipeline waits that give
// up write 101-106 to *err.
cudaError_t launch_grouped_gemm(int mode, const GemmMaps& maps, const GemmGroups& groups, const int* offsets,
                                int T, int k, int I, int H, void* out, int* err, int num_sms, cudaStream_t s,
                                const GemmFp4* fp4 = nullptr);
// uint8 3-D tensor map without swizzle (box box_inner bytes x box_rows rows x 1).
bool encode_map_u8_3d(CUtensorMap* m, const void* base, uint64_t inner, uint64_t rows, uint64_t depth,
                      uint64_t row_bytes, uint64_t depth_bytes, uint32_t box_inner, uint32_t box_rows);
// 2-D / 3-D bf16 tensor maps with 128-byte swizzle (box inner extent 64 elements).
bool encode_map_2d(CUtensorMap* m, const void* base, uint64_t inner, uint64_t rows, uint64_t row_bytes,
                   uint32_t box_rows);
bool encode_map_3d(CUtensorMap* m, const void* base, uint64_t inner, uint64_t rows, uint64_t depth,
                   uint64_t row_bytes, uint64_t depth_bytes, uint32_t box_rows);
// Router logits for many tokens: tiled SIMT fp32 GEMM (64 tokens x 64 experts per CTA).
cudaError_t launch_router_logits_tiled(const void* x, bool x_bf16, const float* w_router, int T, int H,
                                       int E, float* logits, cudaStream_t s);

}  // namespace ftk

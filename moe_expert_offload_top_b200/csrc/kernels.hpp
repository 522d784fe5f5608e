// Internal launch functions of the sm_100a kernels (host side).
#pragma once
#include <cuda_runtime.h>
#include <stdint.h>

namespace ftk {

constexpr int kMaxList = 257;   // routed experts of one layer + the shared expert

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
// K2: stable counting sort of the T*k pairs by expert.
// inv (optional): inv[t*k+j] = position of pair (t,j) in perm.
cudaError_t launch_permute(const int* ids, int T, int k, int E, int* counts, int* offsets,
                           int* perm, int* inv, cudaStream_t s);
// K3 (decode): per list entry, gate/up + SwiGLU of its tokens into h [pairs][I] fp32,
// then the down projection into y [pairs][H] fp32.  Pairs are positions in the
// permutation (routed) or T*k + t (shared expert).  `between` (optional) is recorded
// on s between the two launches.
cudaError_t launch_ffn_decode(const void* x, int T, int H, int I, int k, int wdtype,
                              const ExpertList& list, int max_pairs_per_expert, const int* offsets,
                              const int* perm, float* h, float* y, cudaStream_t s,
                              cudaEvent_t between = nullptr);
// K5: out[t] = sum_j gates[t][j] * y[inv[t*k+j]] (ascending j) + y[T*k+t] if has_shared.
cudaError_t launch_combine(const float* y, const float* gates, const int* inv, int T, int H, int k,
                           bool has_shared, bool out_bf16, void* out, cudaStream_t s);

}  // namespace ftk

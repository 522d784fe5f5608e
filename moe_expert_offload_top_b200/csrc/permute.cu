// K2 - token permutation by expert (a stable counting sort of the T*k
// (token, slot) pairs by their expert), so that each selected expert's
// weights are read once for all of its tokens.
#include "common.cuh"
#include "kernels.hpp"

namespace ftk {

namespace {

constexpr int kPermThreads = 1024;
constexpr int kPermWarps = kPermThreads / 32;

// One CTA.  Pass 1: histogram in shared memory.  Pass 2: exclusive scan.
// Pass 3: the pairs in chunks of 1024 (one per thread, in flat order); a
// pair's place is its expert's running base + the count of equal keys in
// lower warps of the chunk + its rank among equal keys in its own warp
// (__match_any_sync).  Positions are therefore in ascending flat index within
// each expert, whatever the thread timing.
__global__ void __launch_bounds__(kPermThreads)
permute_kernel(const int* __restrict__ ids, int n, int E, int* __restrict__ counts,
               int* __restrict__ offsets, int* __restrict__ perm, int* __restrict__ inv) {
  extern __shared__ int sm[];
  int* cnt = sm;                       // [E]
  int* base = cnt + E;                 // [E]
  int* wc = base + E;                  // [kPermWarps][E]
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  for (int e = tid; e < E; e += kPermThreads) cnt[e] = 0;
  __syncthreads();
  for (int p = tid; p < n; p += kPermThreads) {
    int e = ids[p];
    if (e >= 0 && e < E) atomicAdd(&cnt[e], 1);
  }
  __syncthreads();
  if (tid == 0) {
    int run = 0;
    for (int e = 0; e < E; ++e) { base[e] = run; run += cnt[e]; }
    offsets[E] = run;
  }
  __syncthreads();
  for (int e = tid; e < E; e += kPermThreads) { counts[e] = cnt[e]; offsets[e] = base[e]; }
  const unsigned lt = (1u << lane) - 1u;
  for (int c = 0; c < n; c += kPermThreads) {
    for (int i = tid; i < kPermWarps * E; i += kPermThreads) wc[i] = 0;
    __syncthreads();
    int p = c + tid;
    int e = p < n ? ids[p] : -1;
    if (e >= E) e = -1;
    unsigned mask = __match_any_sync(0xFFFFFFFFu, e);
    int rank = __popc(mask & lt);
    if (e >= 0 && rank == 0) wc[warp * E + e] = __popc(mask);
    __syncthreads();
    if (e >= 0) {
      int before = 0;
      for (int w = 0; w < warp; ++w) before += wc[w * E + e];
      int q = base[e] + before + rank;
      perm[q] = p;
      if (inv) inv[p] = q;
    }
    __syncthreads();
    for (int ee = tid; ee < E; ee += kPermThreads) {
      int s = 0;
      for (int w = 0; w < kPermWarps; ++w) s += wc[w * E + ee];
      base[ee] += s;
    }
    __syncthreads();
  }
}

// More than one chunk: one CTA per chunk of kPermThreads pairs, in a single launch with no
// scratch and no waiting between CTAs.  Each CTA counts every pair by expert (the totals,
// hence offsets) and, in the same pass, the pairs before its chunk (its per-expert prefix),
// all from L2; its chunk's pairs then take offsets[e] + prefix[e] + their rank in the chunk,
// ranked as in permute_kernel.  The positions, counts and offsets equal permute_kernel's.
__global__ void __launch_bounds__(kPermThreads)
permute_chunks_kernel(const int* __restrict__ ids, int n, int E, int* __restrict__ counts,
                      int* __restrict__ offsets, int* __restrict__ perm, int* __restrict__ inv) {
  extern __shared__ int sm[];
  int* cnt = sm;                       // [E] every pair
  int* pre = cnt + E;                  // [E] pairs before this chunk
  int* base = pre + E;                 // [E]
  int* wc = base + E;                  // [kPermWarps][E]
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int c = blockIdx.x * kPermThreads;
  for (int e = tid; e < E; e += kPermThreads) cnt[e] = pre[e] = 0;
  for (int i = tid; i < kPermWarps * E; i += kPermThreads) wc[i] = 0;
  __syncthreads();
  for (int p = tid; p < n; p += kPermThreads) {
    const int e = __ldg(ids + p);
    if (e >= 0 && e < E) {
      atomicAdd(&cnt[e], 1);
      if (p < c) atomicAdd(&pre[e], 1);
    }
  }
  __syncthreads();
  if (tid == 0) {
    int run = 0;
    for (int e = 0; e < E; ++e) { base[e] = run + pre[e]; run += cnt[e]; }
    if (blockIdx.x == 0) offsets[E] = run;
  }
  __syncthreads();
  if (blockIdx.x == 0)
    for (int e = tid; e < E; e += kPermThreads) { counts[e] = cnt[e]; offsets[e] = base[e]; }
  const unsigned lt = (1u << lane) - 1u;
  const int p = c + tid;
  int e = p < n ? __ldg(ids + p) : -1;
  if (e >= E) e = -1;
  const unsigned mask = __match_any_sync(0xFFFFFFFFu, e);
  const int rank = __popc(mask & lt);
  if (e >= 0 && rank == 0) wc[warp * E + e] = __popc(mask);
  __syncthreads();
  if (e >= 0) {
    int before = 0;
    for (int w = 0; w < warp; ++w) before += wc[w * E + e];
    const int q = base[e] + before + rank;
    perm[q] = p;
    if (inv) inv[p] = q;
  }
}

}  // namespace

cudaError_t launch_permute(const int* ids, int T, int k, int E, int* counts, int* offsets,
                           int* perm, int* inv, cudaStream_t s) {
  size_t smem = sizeof(int) * (size_t)(2 * E + kPermWarps * E);
  static bool attr_set = false;
  if (!attr_set) {
    cudaFuncSetAttribute(permute_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, 64 * 1024);
    attr_set = true;
  }
  const long long n = (long long)T * k;
  if (n > kPermThreads && n <= (long long)kPermThreads * 65535) {
    static bool chunks_attr_set = false;
    if (!chunks_attr_set) {
      cudaFuncSetAttribute(permute_chunks_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, 64 * 1024);
      chunks_attr_set = true;
    }
    const size_t smem_c = sizeof(int) * (size_t)(3 * E + kPermWarps * E);
    permute_chunks_kernel<<<(unsigned)((n + kPermThreads - 1) / kPermThreads), kPermThreads, smem_c, s>>>(
        ids, (int)n, E, counts, offsets, perm, inv);
    return cudaGetLastError();
  }
  permute_kernel<<<1, kPermThreads, smem, s>>>(ids, T * k, E, counts, offsets, perm, inv);
  return cudaGetLastError();
}

}  // namespace ftk

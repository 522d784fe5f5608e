// K3 + K5 for decode in one launch: gate/up + SwiGLU, the down projection and the
// gate-weighted combine of one forward.
//
// Method ("FreeToken linux", "FreeToken's MoE memory handling"): every selected
// expert runs from the cache slot that holds it, h = silu(W_gate x) * (W_up x),
// y = W_down h, and out[t] = sum_j g[t,j] y[t,j] (+ the shared expert's y).  The
// arithmetic of every output is that of the per-pass kernels (gemv_rows and the
// combine in ascending j); only the scheduling differs.
//
// Scheduling.  The work is a list of CTA-sized items taken in increasing order from
// an atomic counter: first every gate/up row block of every entry, then every down
// row block.  A down item of entry i waits for the count of entry i's finished
// gate/up items.  Since every gate/up item was taken before any down item, by a CTA
// that is running and never waits, the wait always ends (it is also bounded by time
// and records code 111 in the error word if it gives up).  The combine of down row
// block b is run by the CTA that finishes the last entry's item for block b (a fence
// plus an arrival count, no waiting).  The last CTA to leave zeroes the counters for
// the next launch.
//
// One launch replaces three and keeps the HBM weight stream going from the gate/up
// rows into the down rows; h and y move between CTAs through L2.
#pragma once
#include "decode_gemv.cuh"

namespace ftk {
namespace fused {

using namespace gemv;

// Layout of the counter block (ints).
constexpr int kCtlNext = 0;               // next work item
constexpr int kCtlDone = 1;               // CTAs that have left
constexpr int kCtlA = 2;                  // [kMaxList] finished gate/up items per entry
constexpr int kCtlC = 2 + kMaxList;       // [down row blocks] entries finished per block
constexpr int kErrFusedWait = 111;

FT_DEVICE int ld_acquire(const int* p) {
  int v;
  asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

FT_DEVICE unsigned long long globaltimer_ns() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// One thread waits until *p >= target.  Gives up after limit_ns (or 2^26 polls),
// writing `code` to *err.  Returns whether the count was reached.
FT_DEVICE bool wait_count(const int* p, int target, unsigned long long limit_ns, int* err, int code) {
  if (ld_acquire(p) >= target) return true;
  const unsigned long long t0 = globaltimer_ns();
  for (unsigned it = 0; it < (1u << 26); ++it) {
    __nanosleep(32);
    if (ld_acquire(p) >= target) return true;
    if ((it & 31) == 0 && globaltimer_ns() - t0 > limit_ns) break;
  }
  atomicExch(err, code);
  return false;
}

// out[t][r] for r in [r0, r1): sum over j ascending of g[t][j] * y[inv[t*k+j]][r], then
// + y[T*k+t][r] with a shared expert (the per-pass combine's order).  y was written in
// this launch by other CTAs: read through L2.
FT_DEVICE void combine_rows(const FusedParams& p, int r0, int r1) {
  const int nr = r1 - r0;
  for (int idx = threadIdx.x; idx < p.T * nr; idx += kThreads) {
    const int t = idx / nr, r = r0 + (idx - t * nr);
    float acc = 0.f;
    for (int j = 0; j < p.k; ++j) {
      const float g = p.gates[(size_t)t * p.k + j];
      acc = fmaf(g, __ldcg(p.y + (size_t)p.inv[(size_t)t * p.k + j] * p.H + r), acc);
    }
    if (p.has_shared) acc += __ldcg(p.y + ((size_t)p.T * p.k + t) * p.H + r);
    if (p.out_bf16) static_cast<uint16_t*>(p.out)[(size_t)t * p.H + r] = f32_to_bf16(acc);
    else static_cast<float*>(p.out)[(size_t)t * p.H + r] = acc;
  }
}

template <int WT, int NT, int RG, int RD>
__global__ void __launch_bounds__(kThreads)
ffn_decode_fused_kernel(const __grid_constant__ FusedParams p, const __grid_constant__ ExpertList list) {
  constexpr int kRowsA = kWarps * RG, kRowsB = kWarps * RD;
  const int nA = (p.I + kRowsA - 1) / kRowsA;
  const int nB = (p.H + kRowsB - 1) / kRowsB;
  const int totA = list.n * nA, tot = totA + list.n * nB;
  int* ctl = p.ctl;
  __shared__ int s_item, s_flag;
  if (threadIdx.x == 0) s_item = atomicAdd(ctl + kCtlNext, 1);
  __syncthreads();
  int item = s_item;
  while (item < tot) {
    int nxt = 0;
    if (threadIdx.x == 0) nxt = atomicAdd(ctl + kCtlNext, 1);   // in flight while this item runs
    if (item < totA) {
      const int entry = item / nA, b = item - entry * nA;
      gemv_rows<MODE_GATE_UP, WT, NT, RG, false>(p.x, p.T, p.H, p.I, p.k, list.expert[entry], list.blob[entry],
                                                 b, p.offsets, p.perm, p.h, p.y);
      __threadfence();
      __syncthreads();
      if (threadIdx.x == 0) atomicAdd(ctl + kCtlA + entry, 1);
    } else {
      const int j = item - totA, entry = j / nB, b = j - entry * nB;
      if (threadIdx.x == 0) wait_count(ctl + kCtlA + entry, nA + p.wait_extra, p.limit_ns, p.err, kErrFusedWait);
      __syncthreads();
      gemv_rows<MODE_DOWN, WT, NT, RD, true>(p.x, p.T, p.H, p.I, p.k, list.expert[entry], list.blob[entry], b,
                                             p.offsets, p.perm, p.h, p.y);
      if (p.combine) {
        __threadfence();
        __syncthreads();
        if (threadIdx.x == 0) s_flag = atomicAdd(ctl + kCtlC + b, 1) == list.n - 1;
        __syncthreads();
        if (s_flag) {
          __threadfence();
          combine_rows(p, b * kRowsB, min(p.H, (b + 1) * kRowsB));
        }
      }
    }
    if (threadIdx.x == 0) s_item = nxt;
    __syncthreads();
    item = s_item;
  }
  // The last CTA to leave zeroes the counters for the next launch on the stream.
  if (threadIdx.x == 0) {
    __threadfence();
    s_flag = atomicAdd(ctl + kCtlDone, 1) == (int)gridDim.x - 1;
  }
  __syncthreads();
  if (s_flag) {
    for (int i = threadIdx.x; i < list.n; i += kThreads) ctl[kCtlA + i] = 0;
    if (p.combine)
      for (int b = threadIdx.x; b < nB; b += kThreads) ctl[kCtlC + b] = 0;
    if (threadIdx.x == 0) {
      ctl[kCtlNext] = 0;
      ctl[kCtlDone] = 0;
    }
  }
}

template <int WT, int NT, int RG, int RD>
cudaError_t launch_inst(const FusedParams& p, const ExpertList& list, int num_sms, cudaStream_t s) {
  static const int per_sm = [] {
    int nb = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&nb, ffn_decode_fused_kernel<WT, NT, RG, RD>, kThreads, 0) !=
        cudaSuccess)
      cudaGetLastError();
    return nb > 0 ? nb : 1;
  }();
  const long long nA = (p.I + kWarps * RG - 1) / (kWarps * RG);
  const long long nB = (p.H + kWarps * RD - 1) / (kWarps * RD);
  const long long tot = (long long)list.n * (nA + nB);
  const long long cap = (long long)per_sm * (num_sms > 0 ? num_sms : 1);
  const unsigned grid = (unsigned)(tot < cap ? tot : cap);
  ffn_decode_fused_kernel<WT, NT, RG, RD><<<grid, kThreads, 0, s>>>(p, list);
  return cudaGetLastError();
}

template <int WT, int RG, int RD>
cudaError_t launch_nt(int nt, const FusedParams& p, const ExpertList& list, int num_sms, cudaStream_t s) {
  if (nt <= 1) return launch_inst<WT, 1, RG, RD>(p, list, num_sms, s);
  if (nt <= 2) return launch_inst<WT, 2, RG, RD>(p, list, num_sms, s);
  if (nt <= 4) return launch_inst<WT, 4, RG, RD>(p, list, num_sms, s);
  return launch_inst<WT, 8, RG, RD>(p, list, num_sms, s);
}

// Rows per warp: gate/up 1, 2 or 4; down 2, 4 or 8 (2 or 4 for the packed formats,
// whose dequant needs the registers).
template <int WT, int RG>
cudaError_t launch_rd(int nt, int rd, const FusedParams& p, const ExpertList& list, int num_sms, cudaStream_t s) {
  if (rd <= 2) return launch_nt<WT, RG, 2>(nt, p, list, num_sms, s);
  if constexpr (WT == WT_INT4 || WT == WT_NVFP4) {
    return launch_nt<WT, RG, 4>(nt, p, list, num_sms, s);
  } else {
    if (rd <= 4) return launch_nt<WT, RG, 4>(nt, p, list, num_sms, s);
    return launch_nt<WT, RG, 8>(nt, p, list, num_sms, s);
  }
}

template <int WT>
cudaError_t launch_wt(int nt, int rg, int rd, const FusedParams& p, const ExpertList& list, int num_sms,
                      cudaStream_t s) {
  if (rg <= 1) return launch_rd<WT, 1>(nt, rd, p, list, num_sms, s);
  if (rg <= 2) return launch_rd<WT, 2>(nt, rd, p, list, num_sms, s);
  return launch_rd<WT, 4>(nt, rd, p, list, num_sms, s);
}

}  // namespace fused
}  // namespace ftk

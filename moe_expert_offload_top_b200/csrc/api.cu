// C ABI of the routed-MoE layer stack over a shared LRU expert-slot cache.
//
// Method (FreeToken pages): the full routed-expert pool stays in pinned host
// memory; a fixed number of GPU expert slots, managed by one LRU shared by all
// MoE layers, hold recently used experts; a miss is copied over PCIe into a
// slot and kept ("FreeToken linux", "FreeToken's MoE memory handling";
// "FreeToken gguf", `offload` backend).  Prefill copies the next layer's
// experts while the current layer runs (whole-layer double buffering, same
// section).  The cache is resized at a safe point ("FreeToken RTX 5090",
// dynamic reconfiguration).
//
// Ordering (all CUDA work of a handle):
//   compute stream = the caller's stream of each forward; copies run on the
//   library's copy stream.  Before a slot is overwritten, the copy stream waits
//   for the event recorded after the last forward that read it (use ring).
//   Before a forward's kernels read a slot, the compute stream waits for the
//   event recorded after the slot's last fill (fill ring).  Both rings are
//   FIFO-ordered, so waiting on the newest relevant event covers older ones.
#include <algorithm>
#include <atomic>
#include <chrono>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <string>
#include <thread>
#include <vector>

#include "../../include/ftmoe.h"
#include "cache.hpp"
#include "kernels.hpp"

namespace {

thread_local std::string g_create_error;

}  // namespace

namespace ftk {
// Message for ft_last_error(NULL) from a step-level entry point.
void set_step_error(const std::string& msg) { g_create_error = msg; }
}  // namespace ftk

namespace {
constexpr int kRing = 128;

struct FillTiming {
  cudaEvent_t a, b;
};

// Stage boundaries of one timed forward, on its stream.
// Per-pass FFN: G0 | gate/up | G1 | down | D1 | combine | C1.  Fused FFN: F0 | launch | F1
// and, when split around the fill wait, F2 | launch | F3; C1 closes the forward.
// Split per-pass FFN (resident experts first): G0 | gate/up | G1 | down | DA, the fill wait,
// G2 | gate/up | G3 | down | D1 | combine | C1.
enum { SE_R0, SE_R1, SE_P0, SE_P1, SE_G0, SE_G1, SE_D1, SE_C1, SE_F0, SE_F1, SE_F2, SE_F3,
       SE_DA, SE_G2, SE_G3, SE_N };
struct StageEvents {
  cudaEvent_t ev[SE_N];
  double gu_bytes, d_bytes, flops, fused_bytes;
  int fused_launches;   // 0: per-pass kernels
  int split;            // per-pass kernels in two groups around the fill wait
};

}  // namespace

struct ft_moe {
  int device = 0;
  int E = 0, k = 0, H = 0, I = 0, wdtype = 0;
  int L = 1, gating = 0, has_shared = 0, prefill = 0;
  size_t blob = 0;
  uint8_t* pool = nullptr;
  size_t pool_bytes = 0;
  uint8_t* arena = nullptr;
  int C = 0;
  uint8_t* shared = nullptr;
  ftc::SlotLru lru;
  cudaStream_t copy = nullptr;

  cudaEvent_t use_ev[kRing];
  long long use_ev_call[kRing];
  cudaEvent_t fill_ev[kRing];
  long long fill_ev_batch[kRing];
  long long call = 0;
  long long fill_batches = 0;
  std::vector<long long> slot_last_use;    // last forward call that read the slot
  std::vector<long long> slot_fill_batch;  // last fill batch that wrote the slot
  long long copy_waited_use = -1;
  long long compute_waited_fill = -1;
  cudaStream_t last_stream = nullptr;
  bool has_last_stream = false;

  std::vector<FillTiming> timing_pending, timing_free;
  double h2d_seconds = 0.0;

  int cap_tokens = 0;
  float* d_logits = nullptr;
  int* d_ids = nullptr;
  float* d_gates = nullptr;
  int* d_counts = nullptr;
  int* d_offsets = nullptr;
  int* d_perm = nullptr;
  int* d_inv = nullptr;
  float* d_h = nullptr;
  void* d_xs = nullptr;           // int4 / NVFP4 stacks: the forward's tokens as sliced rows (tensor-core GEMV)
  float* d_y = nullptr;
  int* h_ids = nullptr;            // routing ids on the host: h_box + 2
  int* h_box = nullptr;            // mapped pinned {seq, device error word, ids[T*k]}
  int* d_box = nullptr;
  int route_seq = 0;
  int* d_err = nullptr;           // device-side error word (bounded waits that gave up)
  int* d_ticket = nullptr;        // arrival counter of the fused decode routing kernel
  int* h_err = nullptr;
  uint16_t* d_ax = nullptr;       // gathered token rows for the prefill GEMMs
  ftk::GemmMaps maps;
  bool maps_dirty = true;
  // NVFP4 prefill: the selected experts expanded to bf16 for the tcgen05 GEMMs
  ftk::GemmFp4 fp4 = {};          // NVFP4 stacks: maps over the slots' codes and block scales
  int num_sms = 148;
  int gemm_min_avg_pairs = 32;    // tcgen05 path when bf16 and T*k/|S| >= this
  int fused_routing = 1;          // one-launch routing for decode-sized calls
  int inject_copy_fail = 0;       // countdown to a simulated failed slot fill (0 = off)
  int inject_route_timeout = 0;   // countdown to a simulated routing-wait timeout
  int inject_fused_wait = 0;      // countdown to a fused decode FFN launch whose waits run out
  cudaEvent_t route_ev = nullptr;
  cudaEvent_t xs_ev = nullptr;    // orders a forward after the previous stream's work
  int last_T = 0;
  int fused_ffn = 0;              // decode FFN + combine as one launch (ffn_decode_fused_kernel)
  int int4_tensor = 1;            // int4 / NVFP4 decode GEMV on the tensor cores (mma.sync)
  int* d_ctl = nullptr;           // work counters of the fused decode FFN
  int* h_hold = nullptr;          // mapped pinned flag that releases hold_kernel (stage timing)
  int* d_hold = nullptr;
  int hold_seq = 0;

  ft_cache_stats_t st{};
  ft_perf_t perf{};
  bool stage_timing = false;
  std::vector<StageEvents> stage_pending, stage_free;
  bool trace_on = true;
  std::vector<ftc::Access> trace;
  int timeout_ms = 20000;
  std::string err;
  std::atomic<int> busy{0};
};

namespace {

int fail(ft_moe* h, int code, const std::string& msg) {
  if (h) h->err = msg;
  return code;
}

int cuda_fail(ft_moe* h, cudaError_t e, const char* what) {
  return fail(h, FT_ERR_CUDA, std::string(what) + ": " + cudaGetErrorString(e));
}

#define FT_CUDA(h, call)                                   \
  do {                                                     \
    cudaError_t _e = (call);                               \
    if (_e != cudaSuccess) return cuda_fail((h), _e, #call); \
  } while (0)

struct BusyGuard {
  ft_moe* h;
  bool ok;
  explicit BusyGuard(ft_moe* hh) : h(hh) { ok = h->busy.exchange(1) == 0; }
  ~BusyGuard() {
    if (ok) h->busy.store(0);
  }
};

// Host wait on an event, polling with a deadline.
int wait_event(ft_moe* h, cudaEvent_t ev, const char* what) {
  auto t0 = std::chrono::steady_clock::now();
  for (;;) {
    cudaError_t q = cudaEventQuery(ev);
    if (q == cudaSuccess) return FT_OK;
    if (q != cudaErrorNotReady) return cuda_fail(h, q, what);
    auto dt = std::chrono::steady_clock::now() - t0;
    if (std::chrono::duration_cast<std::chrono::milliseconds>(dt).count() > h->timeout_ms)
      return fail(h, FT_ERR_TIMEOUT, std::string("timed out waiting for ") + what);
  }
}

// Host wait for the fused routing kernel's mailbox (mapped pinned memory): every word
// box[1] (error word) and box[2 .. 2+n) (ids) carries the call's tag above a 10-bit
// value.  Returns once all of them show this call's tag, leaving the plain values in
// place.  Polls the routing event now and then to catch a failed kernel, and gives up
// after the handle's deadline.
int wait_box(ft_moe* h, int seq, int n) {
  volatile int* box = h->h_box;
  auto tagged = [&]() {
    if ((box[1] >> 10) != seq) return false;
    for (int p = 0; p < n; ++p)
      if ((box[2 + p] >> 10) != seq) return false;
    return true;
  };
  auto t0 = std::chrono::steady_clock::now();
  for (unsigned it = 1;; ++it) {
    if (tagged()) break;
    if ((it & 255) == 0) {
      const cudaError_t q = cudaEventQuery(h->route_ev);
      if (q == cudaSuccess) {
        if (tagged()) break;
        return fail(h, FT_ERR_CUDA, "routing kernel finished without publishing its ids");
      }
      if (q != cudaErrorNotReady) return cuda_fail(h, q, "routing ids");
      auto dt = std::chrono::steady_clock::now() - t0;
      if (std::chrono::duration_cast<std::chrono::milliseconds>(dt).count() > h->timeout_ms)
        return fail(h, FT_ERR_TIMEOUT, "timed out waiting for routing ids");
    }
  }
  std::atomic_thread_fence(std::memory_order_acquire);
  box[1] &= 0x3FF;
  for (int p = 0; p < n; ++p) box[2 + p] &= 0x3FF;
  return FT_OK;
}

// Tag of the next fused routing call's mailbox words: 1 .. 2^21 - 1, never 0.
int next_route_seq(ft_moe* h) {
  h->route_seq = h->route_seq % ((1 << 21) - 1) + 1;
  return h->route_seq;
}

void free_scratch(ft_moe* h) {
  cudaFree(h->d_logits); cudaFree(h->d_ids); cudaFree(h->d_gates); cudaFree(h->d_counts);
  cudaFree(h->d_offsets); cudaFree(h->d_perm); cudaFree(h->d_inv); cudaFree(h->d_h);
  cudaFree(h->d_y);
  cudaFree(h->d_xs);
  h->d_xs = nullptr;
  cudaFree(h->d_ax);
  h->d_ax = nullptr;
  h->maps_dirty = true;
  if (h->h_box) cudaFreeHost(h->h_box);
  h->d_logits = nullptr; h->d_ids = nullptr; h->d_gates = nullptr; h->d_counts = nullptr;
  h->d_offsets = nullptr; h->d_perm = nullptr; h->d_inv = nullptr; h->d_h = nullptr;
  h->d_y = nullptr; h->h_ids = nullptr; h->h_box = nullptr; h->d_box = nullptr;
  h->cap_tokens = 0;
}

int ensure_scratch(ft_moe* h, int T) {
  if (T <= h->cap_tokens) return FT_OK;
  // the old buffers may still be read by queued kernels
  if (h->has_last_stream) FT_CUDA(h, cudaStreamSynchronize(h->last_stream));
  free_scratch(h);
  const size_t pairs = (size_t)T * h->k, rows = pairs + T;
  bool ok = cudaMalloc(&h->d_logits, sizeof(float) * (size_t)T * h->E) == cudaSuccess &&
            cudaMalloc(&h->d_ids, sizeof(int) * pairs) == cudaSuccess &&
            cudaMalloc(&h->d_gates, sizeof(float) * pairs) == cudaSuccess &&
            cudaMalloc(&h->d_counts, sizeof(int) * h->E) == cudaSuccess &&
            cudaMalloc(&h->d_offsets, sizeof(int) * (h->E + 1)) == cudaSuccess &&
            cudaMalloc(&h->d_perm, sizeof(int) * pairs) == cudaSuccess &&
            cudaMalloc(&h->d_inv, sizeof(int) * pairs) == cudaSuccess &&
            cudaMalloc(&h->d_h, sizeof(float) * rows * h->I) == cudaSuccess &&
            cudaMalloc(&h->d_y, sizeof(float) * rows * h->H) == cudaSuccess &&
            cudaHostAlloc(&h->h_box, sizeof(int) * (2 + pairs), cudaHostAllocMapped) == cudaSuccess &&
            cudaHostGetDevicePointer(reinterpret_cast<void**>(&h->d_box), h->h_box, 0) == cudaSuccess &&
            ((h->wdtype != FT_W_BF16 && h->wdtype != FT_W_NVFP4) ||
             cudaMalloc(&h->d_ax, sizeof(uint16_t) * rows * h->H) == cudaSuccess) &&
            ((h->wdtype != FT_W_INT4_G128 && h->wdtype != FT_W_NVFP4) ||
             cudaMalloc(&h->d_xs, ftk::int4_sliced_x_bytes(T, h->H)) == cudaSuccess);
  if (!ok) {
    cudaGetLastError();
    free_scratch(h);
    return fail(h, FT_ERR_OOM, "scratch allocation failed");
  }
  memset(h->h_box, 0, sizeof(int) * (2 + pairs));   // tag 0: never a call's tag
  h->h_ids = h->h_box + 2;
  h->cap_tokens = T;
  return FT_OK;
}

int ensure_pool(ft_moe* h) {
  if (h->pool) return FT_OK;
  size_t bytes = (size_t)h->L * h->E * h->blob;
  if (cudaHostAlloc(&h->pool, bytes, cudaHostAllocPortable) != cudaSuccess) {
    cudaGetLastError();
    h->pool = nullptr;
    return fail(h, FT_ERR_OOM, "pinned pool allocation failed");
  }
  h->pool_bytes = bytes;
  return FT_OK;
}

void reset_cache_state(ft_moe* h) {
  h->lru.reset(h->L * h->E, h->C);
  h->slot_last_use.assign(h->C, -1);
  h->slot_fill_batch.assign(h->C, -1);
}

FillTiming get_timing(ft_moe* h) {
  if (!h->timing_free.empty()) {
    FillTiming t = h->timing_free.back();
    h->timing_free.pop_back();
    return t;
  }
  FillTiming t;
  cudaEventCreate(&t.a);
  cudaEventCreate(&t.b);
  return t;
}

// Adds finished fill intervals to h2d_seconds.  block: wait for all of them.
void harvest_timing(ft_moe* h, bool block) {
  std::vector<FillTiming> keep;
  for (auto& t : h->timing_pending) {
    if (block) cudaEventSynchronize(t.b);
    if (cudaEventQuery(t.b) == cudaSuccess) {
      float ms = 0.f;
      if (cudaEventElapsedTime(&ms, t.a, t.b) == cudaSuccess) h->h2d_seconds += ms * 1e-3;
      h->timing_free.push_back(t);
    } else {
      keep.push_back(t);
    }
  }
  h->timing_pending.swap(keep);
}

// Copies the experts of the missed accesses in recs[first..] into their slots.
int issue_fills(ft_moe* h, std::vector<ftc::Access>& recs, size_t first) {
  std::vector<int> slots;
  long long need_use = -1;
  for (size_t i = first; i < recs.size(); ++i)
    if (!recs[i].hit) {
      slots.push_back(recs[i].slot);
      need_use = std::max(need_use, h->slot_last_use[recs[i].slot]);
    }
  if (slots.empty()) return FT_OK;
  if (need_use > h->copy_waited_use) {
    const int r = (int)(need_use % kRing);
    FT_CUDA(h, cudaStreamWaitEvent(h->copy, h->use_ev[r], 0));
    h->copy_waited_use = h->use_ev_call[r];
  }
  FillTiming tm = get_timing(h);
  cudaEventRecord(tm.a, h->copy);
  for (size_t i = first; i < recs.size(); ++i) {
    if (recs[i].hit) continue;
    const ftc::Access& a = recs[i];
    const uint8_t* src = h->pool + ((size_t)a.layer * h->E + a.expert) * h->blob;
    uint8_t* dst = h->arena + (size_t)a.slot * h->blob;
    cudaError_t e;
    if (h->inject_copy_fail > 0 && --h->inject_copy_fail == 0)
      e = cudaErrorUnknown;   // injected on the host: the copy is not issued
    else
      e = cudaMemcpyAsync(dst, src, h->blob, cudaMemcpyHostToDevice, h->copy);
    if (e != cudaSuccess) {
      // roll back this and every later fill of the set to "not resident"
      for (size_t j = i; j < recs.size(); ++j)
        if (!recs[j].hit) h->lru.drop(recs[j].slot);
      h->timing_free.push_back(tm);
      // the copies issued before this one still land: their slots stay resident, so mark
      // them with a fill event that a later forward reading them waits on
      std::vector<int> issued;
      for (size_t j = first; j < i; ++j)
        if (!recs[j].hit) issued.push_back(recs[j].slot);
      if (!issued.empty()) {
        const long long b = h->fill_batches++;
        const int r = (int)(b % kRing);
        cudaEventRecord(h->fill_ev[r], h->copy);
        h->fill_ev_batch[r] = b;
        for (int s : issued) h->slot_fill_batch[s] = b;
      }
      return cuda_fail(h, e, "cudaMemcpyAsync (slot fill)");
    }
    h->st.h2d_bytes += (long long)h->blob;
  }
  cudaEventRecord(tm.b, h->copy);
  h->timing_pending.push_back(tm);
  if (h->timing_pending.size() > 64) harvest_timing(h, false);
  const long long b = h->fill_batches++;
  const int r = (int)(b % kRing);
  FT_CUDA(h, cudaEventRecord(h->fill_ev[r], h->copy));
  h->fill_ev_batch[r] = b;
  for (int s : slots) h->slot_fill_batch[s] = b;
  return FT_OK;
}

bool gemm_shapes_ok(const ft_moe* h) {
  // bf16: 256-column tiles of the outputs, 64-element K blocks; NVFP4 also reads its block
  // scales in 16-byte boxes (256 elements of K per row), so I must be a multiple of 256 too
  return (h->wdtype == FT_W_BF16 && h->H % 256 == 0 && h->I % 128 == 0) ||
         (h->wdtype == FT_W_NVFP4 && h->H % 256 == 0 && h->I % 256 == 0);
}

int ensure_maps(ft_moe* h) {
  if (!h->maps_dirty) return FT_OK;
  const uint64_t rows = (uint64_t)h->cap_tokens * (h->k + 1);
  const uint64_t H = h->H, I = h->I;
  bool ok = ftk::encode_map_2d(&h->maps.a_x, h->d_ax, H, rows, H * 2, 128) &&
            ftk::encode_map_2d(&h->maps.a_h, h->d_h, I, rows, I * 2, 128);
  if (ok && h->wdtype == FT_W_BF16) {
    ok = ftk::encode_map_3d(&h->maps.b1_routed, h->arena, H, 2 * I, h->C, H * 2, h->blob, 128) &&
         ftk::encode_map_3d(&h->maps.b2_routed, h->arena + 2 * I * H * 2, I, H, h->C, I * 2, h->blob, 256);
    if (ok && h->shared) {
      ok = ftk::encode_map_3d(&h->maps.b1_shared, h->shared, H, 2 * I, h->L, H * 2, h->blob, 128) &&
           ftk::encode_map_3d(&h->maps.b2_shared, h->shared + 2 * I * H * 2, I, H, h->L, I * 2, h->blob, 256);
    } else {
      h->maps.b1_shared = h->maps.b1_routed;
      h->maps.b2_shared = h->maps.b2_routed;
    }
  }
  if (ok && h->wdtype == FT_W_NVFP4) {
    // blob: codes Q_gate|Q_up [2I][H/2], Q_down [H][I/2]; block scales S_gate|S_up [2I][H/16],
    // S_down [H][I/16]; then the three fp32 matrix scales
    const uint64_t mat = H * I, q2 = mat, s1 = 3 * mat / 2, s2 = s1 + mat / 8;
    auto maps_over = [&](const uint8_t* b, uint64_t depth, CUtensorMap* q, CUtensorMap* sc) {
      return ftk::encode_map_u8_3d(&q[0], b, H / 2, 2 * I, depth, H / 2, h->blob, 32, 128) &&
             ftk::encode_map_u8_3d(&q[1], b + q2, I / 2, H, depth, I / 2, h->blob, 32, 128) &&
             ftk::encode_map_u8_3d(&sc[0], b + s1, H / 16, 2 * I, depth, H / 16, h->blob, 16, 128) &&
             ftk::encode_map_u8_3d(&sc[1], b + s2, I / 16, H, depth, I / 16, h->blob, 16, 128);
    };
    ok = maps_over(h->arena, h->C, h->fp4.q_routed, h->fp4.s_routed);
    if (ok && h->shared) {
      ok = maps_over(h->shared, h->L, h->fp4.q_shared, h->fp4.s_shared);
    } else {
      for (int i = 0; i < 2; ++i) { h->fp4.q_shared[i] = h->fp4.q_routed[i]; h->fp4.s_shared[i] = h->fp4.s_routed[i]; }
    }
    h->fp4.g_routed = h->arena;
    h->fp4.g_shared = h->shared ? h->shared : h->arena;
    h->fp4.blob = h->blob;
    h->fp4.g_off = 3 * mat / 2 + 3 * mat / 16;
  }
  if (!ok) return fail(h, FT_ERR_CUDA, "cuTensorMapEncodeTiled failed");
  h->maps_dirty = false;
  return FT_OK;
}

StageEvents* stage_begin(ft_moe* h) {
  if (!h->stage_timing) return nullptr;
  if (h->stage_free.empty()) {
    StageEvents se;
    for (int i = 0; i < SE_N; ++i) cudaEventCreate(&se.ev[i]);
    h->stage_free.push_back(se);
  }
  h->stage_pending.push_back(h->stage_free.back());
  h->stage_free.pop_back();
  StageEvents* se = &h->stage_pending.back();
  se->gu_bytes = se->d_bytes = se->flops = se->fused_bytes = 0.0;
  se->fused_launches = 0;
  se->split = 0;
  return se;
}

// While stage timing is on, the forward's stream is held by a one-thread kernel until
// the host has queued the launches of a stage, so the events around each launch time
// the kernel rather than the host issuing it.  The guard releases the hold on every path.
struct StageHold {
  ft_moe* h = nullptr;
  void begin(ft_moe* hh, StageEvents* se, cudaStream_t s) {
    if (!se || !hh->d_hold) return;
    h = hh;
    ++h->hold_seq;
    ftk::launch_hold(h->d_hold, h->hold_seq, 200000000ull, s);
  }
  void release() {
    if (h) *reinterpret_cast<volatile int*>(h->h_hold) = h->hold_seq;
    h = nullptr;
  }
  ~StageHold() { release(); }
};

void stage_mark(StageEvents* se, int which, cudaStream_t s) {
  if (se) cudaEventRecord(se->ev[which], s);
}

void harvest_stages(ft_moe* h, bool block) {
  std::vector<StageEvents> keep;
  for (auto& se : h->stage_pending) {
    if (block) cudaEventSynchronize(se.ev[SE_C1]);
    if (cudaEventQuery(se.ev[SE_C1]) != cudaSuccess) {
      keep.push_back(se);
      continue;
    }
    auto ms = [&](int a, int b) {
      float t = 0.f;
      cudaEventElapsedTime(&t, se.ev[a], se.ev[b]);
      return (double)t;
    };
    h->perf.router_ms += ms(SE_R0, SE_R1);
    h->perf.permute_ms += ms(SE_P0, SE_P1);
    if (se.fused_launches > 0) {
      h->perf.ffn_fused_ms += ms(SE_F0, SE_F1) + (se.fused_launches > 1 ? ms(SE_F2, SE_F3) : 0.0);
      h->perf.ffn_fused_bytes += se.fused_bytes;
      h->perf.ffn_fused_launches += se.fused_launches;
    } else {
      h->perf.ffn_gate_up_launches += se.split ? 2 : 1;
      if (se.split) {
        h->perf.ffn_gate_up_ms += ms(SE_G0, SE_G1) + ms(SE_G2, SE_G3);
        h->perf.ffn_down_ms += ms(SE_G1, SE_DA) + ms(SE_G3, SE_D1);
      } else {
        h->perf.ffn_gate_up_ms += ms(SE_G0, SE_G1);
        h->perf.ffn_down_ms += ms(SE_G1, SE_D1);
      }
      h->perf.combine_ms += ms(SE_D1, SE_C1);
      h->perf.ffn_gate_up_bytes += se.gu_bytes;
      h->perf.ffn_down_bytes += se.d_bytes;
    }
    h->perf.ffn_flops += se.flops;
    h->perf.timed_forwards++;
    h->stage_free.push_back(se);
  }
  h->stage_pending.swap(keep);
}

void account(ft_moe* h, const std::vector<ftc::Access>& recs, size_t first) {
  for (size_t i = first; i < recs.size(); ++i) {
    const ftc::Access& a = recs[i];
    if (a.kind == FT_ROUTED) {
      h->st.routed++;
      if (a.hit) h->st.hits++; else h->st.misses++;
    } else {
      h->st.prefetch++;
      if (a.hit) h->st.prefetch_hits++; else h->st.prefetch_misses++;
    }
    if (a.ev_layer >= 0) h->st.evictions++;
    if (h->trace_on) h->trace.push_back(a);
  }
}

std::vector<int> all_keys(const ft_moe* h, int layer) {
  std::vector<int> keys(h->E);
  for (int e = 0; e < h->E; ++e) keys[e] = layer * h->E + e;
  return keys;
}

}  // namespace

extern "C" {

const char* ft_version(void) { return "ftmoe 0.1 sm_100a"; }

ft_moe* ft_moe_create(int num_experts, int top_k, int hidden, int inter, int wdtype,
                      int cache_slots) {
  if (num_experts < 1 || num_experts > FT_MAX_EXPERTS || top_k < 1 || top_k > num_experts ||
      top_k > FT_MAX_TOPK || hidden < 8 || inter < 8 || hidden % 8 || inter % 8 ||
      wdtype < FT_W_F32 || wdtype > FT_W_NVFP4 || cache_slots < 1) {
    g_create_error = "ft_moe_create: invalid argument";
    return nullptr;
  }
  if (wdtype == FT_W_INT4_G128 && (hidden % 128 || inter % 128)) {
    g_create_error = "ft_moe_create: int4 needs hidden and inter multiples of 128";
    return nullptr;
  }
  if (wdtype == FT_W_NVFP4 && (hidden % 32 || inter % 32)) {
    g_create_error = "ft_moe_create: nvfp4 needs hidden and inter multiples of 32";
    return nullptr;
  }
  ft_moe* h = new ft_moe();
  cudaGetDevice(&h->device);
  h->E = num_experts; h->k = top_k; h->H = hidden; h->I = inter; h->wdtype = wdtype;
  h->C = cache_slots;
  const size_t n = 3ull * hidden * inter;
  h->blob = wdtype == FT_W_F32 ? 4 * n : wdtype == FT_W_BF16 ? 2 * n
            : wdtype == FT_W_NVFP4 ? n / 2 + n / 16 + 16 : n / 2 + 2 * (n / 128);
  if (cudaMalloc(&h->arena, (size_t)cache_slots * h->blob) != cudaSuccess) {
    cudaGetLastError();
    g_create_error = "ft_moe_create: slot arena allocation failed";
    delete h;
    return nullptr;
  }
  cudaStreamCreateWithFlags(&h->copy, cudaStreamNonBlocking);
  for (int i = 0; i < kRing; ++i) {
    cudaEventCreateWithFlags(&h->use_ev[i], cudaEventDisableTiming);
    cudaEventCreateWithFlags(&h->fill_ev[i], cudaEventDisableTiming);
    h->use_ev_call[i] = -1;
    h->fill_ev_batch[i] = -1;
  }
  cudaEventCreateWithFlags(&h->route_ev, cudaEventDisableTiming);
  cudaEventCreateWithFlags(&h->xs_ev, cudaEventDisableTiming);
  cudaMalloc(&h->d_err, sizeof(int));
  cudaMemset(h->d_err, 0, sizeof(int));
  cudaMalloc(&h->d_ticket, sizeof(int));
  cudaMemset(h->d_ticket, 0, sizeof(int));
  cudaHostAlloc(&h->h_err, sizeof(int), cudaHostAllocDefault);
  if (h->h_err) *h->h_err = 0;
  const size_t ctl_bytes = sizeof(int) * (size_t)ftk::ffn_fused_ctl_ints(hidden);
  cudaMalloc(&h->d_ctl, ctl_bytes);
  cudaMemset(h->d_ctl, 0, ctl_bytes);
  if (cudaHostAlloc(&h->h_hold, sizeof(int), cudaHostAllocMapped) == cudaSuccess) {
    *h->h_hold = 0;
    cudaHostGetDevicePointer(reinterpret_cast<void**>(&h->d_hold), h->h_hold, 0);
  }
  cudaDeviceGetAttribute(&h->num_sms, cudaDevAttrMultiProcessorCount, h->device);
  reset_cache_state(h);
  if (cudaGetLastError() != cudaSuccess) {
    g_create_error = "ft_moe_create: CUDA setup failed";
    ft_moe_destroy(h);
    return nullptr;
  }
  return h;
}

int ft_moe_set_layers(ft_moe* h, int num_layers, int gating, int has_shared_expert) {
  if (!h) return FT_ERR_INVALID;
  if (num_layers < 1 || (gating != FT_GATE_SOFTMAX && gating != FT_GATE_SIGMOID))
    return fail(h, FT_ERR_INVALID, "ft_moe_set_layers: invalid argument");
  BusyGuard g(h);
  if (!g.ok) return fail(h, FT_ERR_BUSY, "ft_moe_set_layers: forward in flight");
  cudaStreamSynchronize(h->copy);
  if (h->has_last_stream) cudaStreamSynchronize(h->last_stream);
  if (num_layers != h->L && h->pool) {
    cudaFreeHost(h->pool);
    h->pool = nullptr;
  }
  if (h->shared) {
    cudaFree(h->shared);
    h->shared = nullptr;
  }
  h->maps_dirty = true;
  h->L = num_layers;
  h->gating = gating;
  h->has_shared = has_shared_expert ? 1 : 0;
  int rc = ensure_pool(h);
  if (rc) return rc;
  if (h->has_shared) {
    if (cudaMalloc(&h->shared, (size_t)h->L * h->blob) != cudaSuccess) {
      cudaGetLastError();
      h->shared = nullptr;
      return fail(h, FT_ERR_OOM, "shared-expert allocation failed");
    }
    FT_CUDA(h, cudaMemset(h->shared, 0, (size_t)h->L * h->blob));
  }
  reset_cache_state(h);
  return FT_OK;
}

size_t ft_moe_blob_bytes(const ft_moe* h) { return h ? h->blob : 0; }

void* ft_moe_pool_ptr(ft_moe* h, int layer, int expert) {
  if (!h || layer < 0 || layer >= h->L || expert < 0 || expert >= h->E) return nullptr;
  if (ensure_pool(h) != FT_OK) return nullptr;
  return h->pool + ((size_t)layer * h->E + expert) * h->blob;
}

int ft_moe_set_shared(ft_moe* h, int layer, const void* host_blob) {
  if (!h) return FT_ERR_INVALID;
  if (!h->has_shared || !h->shared || layer < 0 || layer >= h->L || !host_blob)
    return fail(h, FT_ERR_INVALID, "ft_moe_set_shared: no shared expert or bad layer");
  FT_CUDA(h, cudaMemcpy(h->shared + (size_t)layer * h->blob, host_blob, h->blob,
                        cudaMemcpyHostToDevice));
  return FT_OK;
}

int ft_moe_set_mode(ft_moe* h, int prefill) {
  if (!h) return FT_ERR_INVALID;
  h->prefill = prefill ? 1 : 0;
  return FT_OK;
}

int ft_moe_reserve(ft_moe* h, int max_tokens) {
  if (!h || max_tokens < 0) return FT_ERR_INVALID;
  BusyGuard g(h);
  if (!g.ok) return fail(h, FT_ERR_BUSY, "ft_moe_reserve: forward in flight");
  return ensure_scratch(h, max_tokens);
}

int ft_moe_set_timeout_ms(ft_moe* h, int ms) {
  if (!h || ms < 1) return FT_ERR_INVALID;
  h->timeout_ms = ms;
  return FT_OK;
}

int ft_moe_forward(ft_moe* h, int layer, const void* x, int n_tokens, const float* router_w,
                   void* out, void* stream_) {
  if (!h) return FT_ERR_INVALID;
  if (layer < 0 || layer >= h->L || n_tokens < 0 || (n_tokens > 0 && (!x || !router_w || !out)))
    return fail(h, FT_ERR_INVALID, "ft_moe_forward: invalid argument");
  if (!h->pool) return fail(h, FT_ERR_INVALID, "ft_moe_forward: pool not allocated");
  if (n_tokens == 0) return FT_OK;
  BusyGuard g(h);
  if (!g.ok) return fail(h, FT_ERR_BUSY, "ft_moe_forward: another call in flight");
  cudaStream_t s = static_cast<cudaStream_t>(stream_);
  const int T = n_tokens, E = h->E, k = h->k;
  int rc = ensure_scratch(h, T);
  if (rc) return rc;
  // keep forwards of this handle ordered across streams: all work queued so far on the
  // previous stream completes before this call's first kernel
  if (h->has_last_stream && s != h->last_stream && h->call > 0) {
    FT_CUDA(h, cudaEventRecord(h->xs_ev, h->last_stream));
    FT_CUDA(h, cudaStreamWaitEvent(s, h->xs_ev, 0));
  }
  const bool xbf16 = h->wdtype != FT_W_F32;
  if (h->stage_pending.size() > 256) harvest_stages(h, false);
  StageEvents* se = stage_begin(h);
  StageHold hold;
  hold.begin(h, se, s);
  stage_mark(se, SE_R0, s);
  const bool fused_route = h->fused_routing && T <= 64 && E <= 256 && k <= 16;
  if (fused_route) {
    // logits, top-k/gates and the permutation in one launch
    // the kernel also publishes the ids and the error word to the host mailbox
    FT_CUDA(h, ftk::launch_route_decode(x, xbf16, router_w, T, h->H, E, k, h->gating, h->d_logits, h->d_ids,
                                        h->d_gates, h->d_counts, h->d_offsets, h->d_perm, h->d_inv,
                                        h->d_ticket, s, h->d_box, next_route_seq(h), h->d_err));
    stage_mark(se, SE_R1, s);
    FT_CUDA(h, cudaEventRecord(h->route_ev, s));
    stage_mark(se, SE_P0, s);
    stage_mark(se, SE_P1, s);
    h->perf.kernel_launches += 1;
  } else {
    if (T > 64)
      FT_CUDA(h, ftk::launch_router_logits_tiled(x, xbf16, router_w, T, h->H, E, h->d_logits, s));
    else
      FT_CUDA(h, ftk::launch_router_logits(x, xbf16, router_w, T, h->H, E, h->d_logits, s));
    FT_CUDA(h, ftk::launch_topk_gates(h->d_logits, T, E, k, h->gating, h->d_ids, h->d_gates, s));
    stage_mark(se, SE_R1, s);
    FT_CUDA(h, cudaMemcpyAsync(h->h_ids, h->d_ids, sizeof(int) * (size_t)T * k,
                               cudaMemcpyDeviceToHost, s));
    FT_CUDA(h, cudaMemcpyAsync(h->h_err, h->d_err, sizeof(int), cudaMemcpyDeviceToHost, s));
    FT_CUDA(h, cudaEventRecord(h->route_ev, s));
    stage_mark(se, SE_P0, s);
    FT_CUDA(h, ftk::launch_permute(h->d_ids, T, k, E, h->d_counts, h->d_offsets, h->d_perm,
                                   h->d_inv, s));
    stage_mark(se, SE_P1, s);
    h->perf.kernel_launches += 3;
  }
  h->perf.forwards++;
  hold.release();
  {
    auto w0 = std::chrono::steady_clock::now();
    if (h->inject_route_timeout > 0 && --h->inject_route_timeout == 0) {
      cudaEventSynchronize(h->route_ev);   // the work itself completes; only the report is injected
      return fail(h, FT_ERR_TIMEOUT, "timed out waiting for routing ids (injected)");
    }
    rc = fused_route ? wait_box(h, h->route_seq, T * k) : wait_event(h, h->route_ev, "routing ids");
    h->perf.host_wait_ms +=
        std::chrono::duration<double, std::milli>(std::chrono::steady_clock::now() - w0).count();
  }
  if (rc) return rc;
  const auto t_routed = std::chrono::steady_clock::now();   // the routing is on the host
  h->last_T = T;
  // A failure from here on leaves no kernel of this call running: the caller's stream is
  // drained first, so a following forward on another stream cannot race on the scratch.
  auto bail = [&](int code, const std::string& msg) {
    hold.release();
    cudaStreamSynchronize(s);
    return fail(h, code, msg);
  };
  // CUDA failures from here on also drain the caller's stream (through bail)
#define FT_CUDA_B(call)                                                                      \
  do {                                                                                       \
    cudaError_t _e = (call);                                                                 \
    if (_e != cudaSuccess) return bail(FT_ERR_CUDA, std::string(#call) + ": " + cudaGetErrorString(_e)); \
  } while (0)
  int* dev_err = fused_route ? h->h_box + 1 : h->h_err;
  if (*dev_err) {
    const int code = *dev_err;
    *dev_err = 0;
    cudaMemsetAsync(h->d_err, 0, sizeof(int), s);
    return bail(FT_ERR_DEVICE_CHECK,
                "a previous forward's kernel gave up waiting (code " + std::to_string(code) + ")");
  }

  // distinct selected experts, ascending, and the largest token count of one expert
  std::vector<int> cnt(E, 0);
  for (int i = 0; i < T * k; ++i) {
    const int e = h->h_ids[i];
    if (e < 0 || e >= E) return bail(FT_ERR_DEVICE_CHECK, "router produced an invalid expert id");
    cnt[e]++;
  }
  std::vector<int> S, keys;
  int max_pairs = 0;
  for (int e = 0; e < E; ++e)
    if (cnt[e]) {
      S.push_back(e);
      keys.push_back(layer * E + e);
      max_pairs = std::max(max_pairs, cnt[e]);
    }
  const bool pre0 = h->prefill && layer == 0;
  const bool pre_next = h->prefill && layer + 1 < h->L;
  if ((int)S.size() > h->C || ((pre0 || pre_next) && E > h->C))
    return bail(FT_ERR_CAPACITY, "cache has fewer slots than one step needs");

  const long long call = h->call;
  std::vector<ftc::Access> recs;
  if (pre0) {
    h->lru.access_set(all_keys(h, 0), E, (int)call, FT_PREFETCH, recs);
    rc = issue_fills(h, recs, 0);
    account(h, recs, 0);
    if (rc) return bail(rc, h->err);
  }
  const size_t first_routed = recs.size();
  h->lru.access_set(keys, E, (int)call, FT_ROUTED, recs);
  rc = issue_fills(h, recs, first_routed);
  account(h, recs, first_routed);
  if (rc) return bail(rc, h->err);

  // the kernels read the slots of S: wait for their newest fill
  ftk::ExpertList list;
  list.n = 0;
  long long entry_fill[ftk::kMaxList];
  long long need_fill = -1;
  for (size_t i = 0; i < S.size(); ++i) {
    const int slot = h->lru.slot_of(keys[i]);
    list.expert[list.n] = S[i];
    list.blob[list.n] = h->arena + (size_t)slot * h->blob;
    entry_fill[list.n] = h->slot_fill_batch[slot];
    list.n++;
    need_fill = std::max(need_fill, h->slot_fill_batch[slot]);
  }
  if (h->has_shared) {
    list.expert[list.n] = -1;
    list.blob[list.n] = h->shared + (size_t)layer * h->blob;
    entry_fill[list.n] = -1;
    list.n++;
  }
  const bool same_stream = h->has_last_stream && s == h->last_stream;
  const bool must_wait = need_fill > h->compute_waited_fill || (need_fill >= 0 && !same_stream);
  auto wait_fills = [&]() -> int {
    const int r = (int)(need_fill % kRing);
    FT_CUDA_B(cudaStreamWaitEvent(s, h->fill_ev[r], 0));
    h->compute_waited_fill = h->fill_ev_batch[r];
    return FT_OK;
  };
  const double xb = xbf16 ? 2.0 : 4.0;
  const size_t mat = (size_t)h->H * h->I;
  const double wmat = h->wdtype == FT_W_INT4_G128 ? mat / 2.0 + 2.0 * (mat / 128)
                      : h->wdtype == FT_W_NVFP4 ? mat / 2.0 + mat / 16.0
                                                : (double)mat * (h->wdtype == FT_W_F32 ? 4 : 2);
  const double pairs = (double)T * k + (h->has_shared ? T : 0);
  if (se) {
    // algorithmic bytes: every weight of the listed experts once, their inputs and outputs
    se->gu_bytes = list.n * 2.0 * wmat + pairs * (h->H * xb + h->I * 4.0);
    se->d_bytes = list.n * wmat + pairs * (h->I * 4.0 + h->H * 4.0);
    se->flops = pairs * 6.0 * mat;
  }
  // The slots of this call are read by the gate/up and down kernels only: use_ev marks
  // their end (the copy stream waits on it before overwriting a slot).  Recorded before
  // the combine, so that the next forward's routing kernel can follow the combine
  // directly (programmatic dependent launch).
  auto record_use = [&]() -> int {
    const int r = (int)(call % kRing);
    FT_CUDA_B(cudaEventRecord(h->use_ev[r], s));
    h->use_ev_call[r] = call;
    return FT_OK;
  };
  hold.begin(h, se, s);
  const bool use_gemm = gemm_shapes_ok(h) && (long long)T * k >= (long long)h->gemm_min_avg_pairs * (long long)S.size();
  // Decode path: entries whose slots this stream has already waited for (and the shared
  // expert) run while this call's misses are still being copied; the rest run after the
  // wait for the fills, followed by the combine.
  ftk::ExpertList ready, later;
  ready.n = later.n = 0;
  for (int i = 0; i < list.n; ++i) {
    const bool is_ready = entry_fill[i] < 0 || (same_stream && entry_fill[i] <= h->compute_waited_fill);
    ftk::ExpertList& dst = is_ready ? ready : later;
    dst.expert[dst.n] = list.expert[i];
    dst.blob[dst.n] = list.blob[i];
    dst.n++;
  }
  // (not while stage timing: its events then time each launch over the forward's whole list)
  const bool split = !use_gemm && ready.n > 0 && later.n > 0 && !se;
  if (!use_gemm && h->fused_ffn) {
    // one fused launch per group; the last one also runs the combine
    ftk::FusedParams fp{};
    fp.x = x; fp.offsets = h->d_offsets; fp.perm = h->d_perm; fp.h = h->d_h; fp.y = h->d_y;
    fp.gates = h->d_gates; fp.inv = h->d_inv; fp.out = out; fp.ctl = h->d_ctl; fp.err = h->d_err;
    fp.T = T; fp.H = h->H; fp.I = h->I; fp.k = k;
    fp.has_shared = h->has_shared != 0; fp.out_bf16 = xbf16 ? 1 : 0;
    fp.limit_ns = 2000000000ull;
    if (h->inject_fused_wait > 0 && --h->inject_fused_wait == 0) {
      fp.wait_extra = 1;          // a count nothing reaches: every down item's wait runs out
      fp.limit_ns = 1000000ull;   // after 1 ms, with code 111 in the error word
    }
    if (se) {   // weights of every listed expert once, x in, out back (h, y stay in L2)
      se->fused_bytes = list.n * 3.0 * wmat + (double)T * h->H * xb * 2.0;
    }
    if (split) {
      fp.combine = 0;
      stage_mark(se, SE_F0, s);
      FT_CUDA_B(ftk::launch_ffn_fused(fp, h->wdtype, ready, max_pairs, h->num_sms, s));
      stage_mark(se, SE_F1, s);
      rc = wait_fills();
      if (rc) return bail(rc, h->err);
      fp.combine = 1;
      stage_mark(se, SE_F2, s);
      FT_CUDA_B(ftk::launch_ffn_fused(fp, h->wdtype, later, max_pairs, h->num_sms, s));
      stage_mark(se, SE_F3, s);
      if (se) se->fused_launches = 2;
      h->perf.kernel_launches += 2;
    } else {
      if (must_wait) {
        rc = wait_fills();
        if (rc) return bail(rc, h->err);
      }
      fp.combine = 1;
      stage_mark(se, SE_F0, s);
      FT_CUDA_B(ftk::launch_ffn_fused(fp, h->wdtype, list, max_pairs, h->num_sms, s));
      stage_mark(se, SE_F1, s);
      if (se) se->fused_launches = 1;
      h->perf.kernel_launches += 1;
    }
    stage_mark(se, SE_C1, s);
    rc = record_use();
    if (rc) return bail(rc, h->err);
  } else {
    if (use_gemm) {
      if (must_wait) {
        rc = wait_fills();
        if (rc) return bail(rc, h->err);
      }
      // NVFP4 slots are expanded to bf16 inside the GEMMs (exact), bf16 slots read as they are
      const ftk::GemmFp4* fp4 = h->wdtype == FT_W_NVFP4 ? &h->fp4 : nullptr;
      rc = ensure_maps(h);
      if (rc) return bail(rc, h->err);
      ftk::GemmGroups groups;
      groups.n = list.n;
      for (int i = 0; i < list.n; ++i) {
        groups.expert[i] = list.expert[i];
        groups.z[i] = list.expert[i] >= 0 ? h->lru.slot_of(layer * E + list.expert[i]) : layer;
      }
      FT_CUDA_B(ftk::launch_gather_rows(x, h->d_perm, T, k, h->H, h->has_shared != 0, h->d_ax, s));
      h->perf.kernel_launches += 1;
      stage_mark(se, SE_G0, s);
      FT_CUDA_B(ftk::launch_grouped_gemm(0, h->maps, groups, h->d_offsets, T, k, h->I, h->H, h->d_h,
                                          h->d_err, h->num_sms, s, fp4));
      stage_mark(se, SE_G1, s);
      FT_CUDA_B(ftk::launch_grouped_gemm(1, h->maps, groups, h->d_offsets, T, k, h->I, h->H, h->d_y,
                                          h->d_err, h->num_sms, s, fp4));
      if (se) {   // bf16 h, and the weights of each listed expert read once (in their stored format)
        se->gu_bytes = list.n * 2.0 * wmat + pairs * (h->H * 2.0 + h->I * 2.0);
        se->d_bytes = list.n * wmat + pairs * (h->I * 2.0 + h->H * 4.0);
      }
    } else if (split) {
      // gate/up | G1 | down of the ready group, the wait, then gate/up | G3 | down of the rest
      stage_mark(se, SE_G0, s);
      FT_CUDA_B(ftk::launch_ffn_decode(x, T, h->H, h->I, k, h->wdtype, ready, max_pairs, h->d_offsets,
                                        h->d_perm, h->d_h, h->d_y, s, se ? se->ev[SE_G1] : nullptr, h->d_err,
                                        h->int4_tensor != 0, h->d_xs));
      stage_mark(se, SE_DA, s);
      rc = wait_fills();
      if (rc) return bail(rc, h->err);
      stage_mark(se, SE_G2, s);
      FT_CUDA_B(ftk::launch_ffn_decode(x, T, h->H, h->I, k, h->wdtype, later, max_pairs, h->d_offsets,
                                        h->d_perm, h->d_h, h->d_y, s, se ? se->ev[SE_G3] : nullptr, h->d_err,
                                        h->int4_tensor != 0, h->d_xs));
      if (se) se->split = 1;
      h->perf.kernel_launches += ftk::ffn_decode_kernels(h->wdtype, h->int4_tensor != 0, h->H, h->I, T);
    } else {
      if (must_wait) {
        rc = wait_fills();
        if (rc) return bail(rc, h->err);
      }
      stage_mark(se, SE_G0, s);
      FT_CUDA_B(ftk::launch_ffn_decode(x, T, h->H, h->I, k, h->wdtype, list, max_pairs, h->d_offsets,
                                        h->d_perm, h->d_h, h->d_y, s, se ? se->ev[SE_G1] : nullptr, h->d_err,
                                        h->int4_tensor != 0, h->d_xs));
    }
    stage_mark(se, SE_D1, s);
    rc = record_use();
    if (rc) return bail(rc, h->err);
    FT_CUDA_B(ftk::launch_combine(h->d_y, h->d_gates, h->d_inv, T, h->H, k, h->has_shared != 0,
                                   xbf16, out, s));
    stage_mark(se, SE_C1, s);
    // one FFN pass (the GEMMs: gate/up, down) and the combine
    h->perf.kernel_launches +=
        (use_gemm ? 2 : ftk::ffn_decode_kernels(h->wdtype, h->int4_tensor != 0, h->H, h->I, T)) + 1;
  }
  hold.release();
#undef FT_CUDA_B
  for (int key : keys) h->slot_last_use[h->lru.slot_of(key)] = call;
  h->perf.host_issue_ms +=
      std::chrono::duration<double, std::milli>(std::chrono::steady_clock::now() - t_routed).count();
  h->last_stream = s;
  h->has_last_stream = true;
  h->call++;

  if (pre_next) {
    const size_t first_pre = recs.size();
    h->lru.access_set(all_keys(h, layer + 1), E, (int)call, FT_PREFETCH, recs);
    rc = issue_fills(h, recs, first_pre);
    account(h, recs, first_pre);
    if (rc) return rc;
  }
  return FT_OK;
}

int ft_moe_sync(ft_moe* h) {
  if (!h) return FT_ERR_INVALID;
  FT_CUDA(h, cudaStreamSynchronize(h->copy));
  if (h->has_last_stream) FT_CUDA(h, cudaStreamSynchronize(h->last_stream));
  int code = 0;
  FT_CUDA(h, cudaMemcpy(&code, h->d_err, sizeof(int), cudaMemcpyDeviceToHost));
  if (code) {
    cudaMemset(h->d_err, 0, sizeof(int));
    return fail(h, FT_ERR_DEVICE_CHECK, "a kernel gave up waiting (code " + std::to_string(code) + ")");
  }
  return FT_OK;
}

int ft_moe_set_int4_tensor_cores(ft_moe* h, int enabled) {
  if (!h) return FT_ERR_INVALID;
  h->int4_tensor = enabled != 0;
  return FT_OK;
}

int ft_moe_set_fused_ffn(ft_moe* h, int enabled) {
  if (!h) return FT_ERR_INVALID;
  h->fused_ffn = enabled != 0;
  return FT_OK;
}

int ft_moe_set_fused_routing(ft_moe* h, int enabled) {
  if (!h) return FT_ERR_INVALID;
  h->fused_routing = enabled != 0;
  return FT_OK;
}

int ft_moe_debug_inject(ft_moe* h, int what, int countdown) {
  if (!h || countdown < 0) return FT_ERR_INVALID;
  if (what == FT_INJECT_COPY_FAIL) h->inject_copy_fail = countdown;
  else if (what == FT_INJECT_ROUTE_TIMEOUT) h->inject_route_timeout = countdown;
  else if (what == FT_INJECT_FUSED_WAIT) h->inject_fused_wait = countdown;
  else return fail(h, FT_ERR_INVALID, "ft_moe_debug_inject: unknown fault");
  return FT_OK;
}

int ft_debug_device_wait_selftest(int limit_us, void* stream) {
  if (limit_us < 1 || limit_us > 1000000) return FT_ERR_INVALID;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  int* err = nullptr;
  int code = 0;
  if (cudaMallocAsync(&err, sizeof(int), s) != cudaSuccess) return FT_ERR_OOM;
  cudaError_t e = cudaMemsetAsync(err, 0, sizeof(int), s);
  if (e == cudaSuccess) e = ftk::launch_wait_selftest((unsigned long long)limit_us * 1000ull, err, s);
  if (e == cudaSuccess) e = cudaMemcpyAsync(&code, err, sizeof(int), cudaMemcpyDeviceToHost, s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  cudaFreeAsync(err, s);
  cudaStreamSynchronize(s);
  if (e != cudaSuccess) return FT_ERR_CUDA;
  return code == 199 ? FT_ERR_DEVICE_CHECK : FT_OK;
}

int ft_moe_set_gemm_threshold(ft_moe* h, int min_avg_pairs) {
  if (!h || min_avg_pairs < 0) return FT_ERR_INVALID;
  h->gemm_min_avg_pairs = min_avg_pairs;
  return FT_OK;
}

int ft_moe_set_stage_timing(ft_moe* h, int enabled) {
  if (!h) return FT_ERR_INVALID;
  h->stage_timing = enabled != 0;
  return FT_OK;
}

int ft_moe_perf(ft_moe* h, ft_perf_t* out) {
  if (!h || !out) return FT_ERR_INVALID;
  harvest_stages(h, true);
  *out = h->perf;
  return FT_OK;
}

int ft_moe_reset_perf(ft_moe* h) {
  if (!h) return FT_ERR_INVALID;
  harvest_stages(h, true);
  h->perf = ft_perf_t{};
  return FT_OK;
}

int ft_moe_last_routing(const ft_moe* hc, int* ids, float* gates, int* n_tokens) {
  ft_moe* h = const_cast<ft_moe*>(hc);
  if (!h) return FT_ERR_INVALID;
  if (n_tokens) *n_tokens = h->last_T;
  if (h->last_T == 0) return FT_OK;
  if (h->has_last_stream) FT_CUDA(h, cudaStreamSynchronize(h->last_stream));
  const size_t n = (size_t)h->last_T * h->k;
  if (ids) FT_CUDA(h, cudaMemcpy(ids, h->d_ids, sizeof(int) * n, cudaMemcpyDeviceToHost));
  if (gates) FT_CUDA(h, cudaMemcpy(gates, h->d_gates, sizeof(float) * n, cudaMemcpyDeviceToHost));
  return FT_OK;
}

int ft_cache_resize(ft_moe* h, int slots) {
  if (!h) return FT_ERR_INVALID;
  if (slots < 1) return fail(h, FT_ERR_INVALID, "ft_cache_resize: slots must be >= 1");
  BusyGuard g(h);
  if (!g.ok) return fail(h, FT_ERR_BUSY, "ft_cache_resize: forward in flight");
  FT_CUDA(h, cudaStreamSynchronize(h->copy));
  if (h->has_last_stream) FT_CUDA(h, cudaStreamSynchronize(h->last_stream));
  if (slots == h->C) return FT_OK;
  uint8_t* na = nullptr;
  if (cudaMalloc(&na, (size_t)slots * h->blob) != cudaSuccess) {
    cudaGetLastError();
    return fail(h, FT_ERR_OOM, "ft_cache_resize: arena allocation failed");
  }
  std::vector<int> evicted;
  std::vector<std::pair<int, int>> moves;
  const int old_c = h->C;
  std::vector<int> old_key_of(old_c);
  for (int s2 = 0; s2 < old_c; ++s2) old_key_of[s2] = h->lru.key_of(s2);
  h->lru.resize(slots, evicted, moves);
  cudaError_t e = cudaSuccess;
  if (slots > old_c) {
    e = cudaMemcpyAsync(na, h->arena, (size_t)old_c * h->blob, cudaMemcpyDeviceToDevice, h->copy);
  } else {
    for (int s2 = 0; s2 < slots && e == cudaSuccess; ++s2)
      if (h->lru.key_of(s2) >= 0 && old_key_of[s2] == h->lru.key_of(s2))
        e = cudaMemcpyAsync(na + (size_t)s2 * h->blob, h->arena + (size_t)s2 * h->blob, h->blob,
                            cudaMemcpyDeviceToDevice, h->copy);
    for (auto& m : moves)
      if (e == cudaSuccess)
        e = cudaMemcpyAsync(na + (size_t)m.second * h->blob, h->arena + (size_t)m.first * h->blob,
                            h->blob, cudaMemcpyDeviceToDevice, h->copy);
  }
  if (e == cudaSuccess) e = cudaStreamSynchronize(h->copy);
  if (e != cudaSuccess) {
    cudaFree(na);
    reset_cache_state(h);   // contents unknown: start empty
    return cuda_fail(h, e, "ft_cache_resize copy");
  }
  cudaFree(h->arena);
  h->arena = na;
  h->C = slots;
  h->maps_dirty = true;
  h->st.evictions += (long long)evicted.size();
  h->slot_last_use.assign(slots, -1);
  h->slot_fill_batch.assign(slots, -1);
  return FT_OK;
}

int ft_cache_clear(ft_moe* h) {
  if (!h) return FT_ERR_INVALID;
  BusyGuard g(h);
  if (!g.ok) return fail(h, FT_ERR_BUSY, "ft_cache_clear: forward in flight");
  FT_CUDA(h, cudaStreamSynchronize(h->copy));
  if (h->has_last_stream) FT_CUDA(h, cudaStreamSynchronize(h->last_stream));
  reset_cache_state(h);
  return FT_OK;
}

int ft_cache_stats(const ft_moe* hc, ft_cache_stats_t* out) {
  ft_moe* h = const_cast<ft_moe*>(hc);
  if (!h || !out) return FT_ERR_INVALID;
  cudaStreamSynchronize(h->copy);
  harvest_timing(h, true);
  *out = h->st;
  out->h2d_seconds = h->h2d_seconds;
  out->resident = h->lru.size();
  out->capacity = h->C;
  return FT_OK;
}

int ft_cache_reset_stats(ft_moe* h) {
  if (!h) return FT_ERR_INVALID;
  cudaStreamSynchronize(h->copy);
  harvest_timing(h, true);
  h->st = ft_cache_stats_t{};
  h->h2d_seconds = 0.0;
  return FT_OK;
}

int ft_cache_trace(const ft_moe* h, ft_access_t* buf, int cap, int* n) {
  if (!h || !n || cap < 0 || (cap > 0 && !buf)) return FT_ERR_INVALID;
  *n = (int)h->trace.size();
  const int m = std::min(cap, *n);
  for (int i = 0; i < m; ++i) {
    const ftc::Access& a = h->trace[i];
    buf[i] = ft_access_t{a.call, a.layer, a.expert, a.kind, a.hit, a.slot, a.ev_layer, a.ev_expert};
  }
  return FT_OK;
}

int ft_cache_set_trace(ft_moe* h, int enabled) {
  if (!h) return FT_ERR_INVALID;
  h->trace_on = enabled != 0;
  if (!h->trace_on) h->trace.clear();
  return FT_OK;
}

int ft_cache_slot_of(const ft_moe* h, int layer, int expert) {
  if (!h || layer < 0 || layer >= h->L || expert < 0 || expert >= h->E) return -1;
  return h->lru.slot_of(layer * h->E + expert);
}

void* ft_cache_slot_ptr(ft_moe* h, int slot) {
  if (!h || slot < 0 || slot >= h->C) return nullptr;
  return h->arena + (size_t)slot * h->blob;
}

const char* ft_last_error(const ft_moe* h) {
  return h ? h->err.c_str() : g_create_error.c_str();
}

void ft_moe_destroy(ft_moe* h) {
  if (!h) return;
  if (h->copy) cudaStreamSynchronize(h->copy);
  if (h->has_last_stream) cudaStreamSynchronize(h->last_stream);
  harvest_timing(h, true);
  for (auto& t : h->timing_free) { cudaEventDestroy(t.a); cudaEventDestroy(t.b); }
  for (int i = 0; i < kRing; ++i) {
    if (h->use_ev[i]) cudaEventDestroy(h->use_ev[i]);
    if (h->fill_ev[i]) cudaEventDestroy(h->fill_ev[i]);
  }
  if (h->route_ev) cudaEventDestroy(h->route_ev);
  if (h->xs_ev) cudaEventDestroy(h->xs_ev);
  harvest_stages(h, true);
  for (auto& se : h->stage_free)
    for (int i = 0; i < SE_N; ++i) cudaEventDestroy(se.ev[i]);
  free_scratch(h);
  cudaFree(h->d_err);
  cudaFree(h->d_ticket);
  cudaFree(h->d_ctl);
  if (h->h_err) cudaFreeHost(h->h_err);
  if (h->h_hold) cudaFreeHost(h->h_hold);
  if (h->copy) cudaStreamDestroy(h->copy);
  cudaFree(h->arena);
  cudaFree(h->shared);
  if (h->pool) cudaFreeHost(h->pool);
  delete h;
}

// Static placement: the first `capacity` keys in (layer, expert) order are resident
// for good; every other access is a miss served without caching.
static int simulate_static(int num_layers, int num_experts, int capacity, const int* ops, int n_ops_ints,
                           ft_access_t* trace, int trace_cap, int* n_trace, ft_cache_stats_t* stats) {
  std::vector<ft_access_t> recs;
  ft_cache_stats_t st{};
  int cap = capacity;
  int i = 0;
  while (i < n_ops_ints) {
    if (ops[i] == 0) {
      if (i + 5 > n_ops_ints) return FT_ERR_INVALID;
      const int call = ops[i + 1], layer = ops[i + 2], kind = ops[i + 3], n = ops[i + 4];
      if (layer < 0 || layer >= num_layers || n < 0 || i + 5 + n > n_ops_ints) return FT_ERR_INVALID;
      std::vector<int> es(ops + i + 5, ops + i + 5 + n);
      std::sort(es.begin(), es.end());
      es.erase(std::unique(es.begin(), es.end()), es.end());
      for (int e : es) {
        if (e < 0 || e >= num_experts) return FT_ERR_INVALID;
        const int key = layer * num_experts + e;
        const int hit = key < cap;
        recs.push_back(ft_access_t{call, layer, e, kind, hit, hit ? key : -1, -1, -1});
        if (kind == FT_ROUTED) { st.routed++; if (hit) st.hits++; else st.misses++; }
        else { st.prefetch++; if (hit) st.prefetch_hits++; else st.prefetch_misses++; }
      }
      i += 5 + n;
    } else if (ops[i] == 1) {
      if (i + 2 > n_ops_ints || ops[i + 1] < 1) return FT_ERR_INVALID;
      cap = ops[i + 1];
      i += 2;
    } else {
      return FT_ERR_INVALID;
    }
  }
  *n_trace = (int)recs.size();
  for (int r = 0; r < std::min(trace_cap, *n_trace); ++r) trace[r] = recs[r];
  st.resident = std::min(cap, num_layers * num_experts);
  st.capacity = cap;
  if (stats) *stats = st;
  return FT_OK;
}

int ft_cache_simulate_policy(int policy, int num_layers, int num_experts, int capacity, const int* ops,
                             int n_ops_ints, ft_access_t* trace, int trace_cap, int* n_trace,
                             ft_cache_stats_t* stats, int* n_capacity_errors) {
  if (policy == FT_POLICY_LRU)
    return ft_cache_simulate(num_layers, num_experts, capacity, ops, n_ops_ints, trace, trace_cap, n_trace,
                             stats, n_capacity_errors);
  if (policy != FT_POLICY_STATIC || num_layers < 1 || num_experts < 1 || capacity < 1 || n_ops_ints < 0 ||
      (n_ops_ints > 0 && !ops) || !n_trace || trace_cap < 0 || (trace_cap > 0 && !trace))
    return FT_ERR_INVALID;
  if (n_capacity_errors) *n_capacity_errors = 0;
  return simulate_static(num_layers, num_experts, capacity, ops, n_ops_ints, trace, trace_cap, n_trace, stats);
}

int ft_probe_host_link(size_t bytes, int iters, double* h2d_gbs, double* d2h_gbs) {
  if (bytes < 1024 || iters < 1 || !h2d_gbs || !d2h_gbs) return FT_ERR_INVALID;
  void* hbuf = nullptr;
  void* dbuf = nullptr;
  cudaStream_t s = nullptr;
  cudaEvent_t a = nullptr, b = nullptr;
  int rc = FT_OK;
  if (cudaHostAlloc(&hbuf, bytes, cudaHostAllocDefault) != cudaSuccess ||
      cudaMalloc(&dbuf, bytes) != cudaSuccess) {
    cudaGetLastError();
    rc = FT_ERR_OOM;
  }
  if (rc == FT_OK) {
    memset(hbuf, 1, bytes);
    cudaStreamCreateWithFlags(&s, cudaStreamNonBlocking);
    cudaEventCreate(&a);
    cudaEventCreate(&b);
    for (int dir = 0; dir < 2 && rc == FT_OK; ++dir) {
      const cudaMemcpyKind kind = dir == 0 ? cudaMemcpyHostToDevice : cudaMemcpyDeviceToHost;
      void* dst = dir == 0 ? dbuf : hbuf;
      const void* src = dir == 0 ? hbuf : dbuf;
      cudaMemcpyAsync(dst, src, bytes, kind, s);            // warm-up
      cudaEventRecord(a, s);
      for (int it = 0; it < iters; ++it) cudaMemcpyAsync(dst, src, bytes, kind, s);
      cudaEventRecord(b, s);
      float ms = 0.f;
      if (cudaEventSynchronize(b) != cudaSuccess || cudaEventElapsedTime(&ms, a, b) != cudaSuccess || ms <= 0.f)
        rc = FT_ERR_CUDA;
      else
        *(dir == 0 ? h2d_gbs : d2h_gbs) = (double)bytes * iters / (ms * 1e-3) / 1e9;
    }
  }
  if (a) cudaEventDestroy(a);
  if (b) cudaEventDestroy(b);
  if (s) cudaStreamDestroy(s);
  if (dbuf) cudaFree(dbuf);
  if (hbuf) cudaFreeHost(hbuf);
  return rc;
}

int ft_probe_host_memory(size_t bytes, int threads, int iters, double* gbs) {
  if (bytes < 4096 || threads < 1 || threads > 256 || iters < 1 || !gbs) return FT_ERR_INVALID;
  std::vector<uint8_t> src, dst;
  try {
    src.assign(bytes, 1);
    dst.assign(bytes, 0);
  } catch (...) {
    return FT_ERR_OOM;
  }
  auto pass = [&]() {
    std::vector<std::thread> pool;
    const size_t per = (bytes + threads - 1) / threads;
    for (int t = 0; t < threads; ++t) {
      const size_t b0 = std::min(bytes, (size_t)t * per), b1 = std::min(bytes, b0 + per);
      if (b1 > b0) pool.emplace_back([&, b0, b1] { memcpy(dst.data() + b0, src.data() + b0, b1 - b0); });
    }
    for (auto& th : pool) th.join();
  };
  pass();   // warm-up: touches every page
  const auto t0 = std::chrono::steady_clock::now();
  for (int it = 0; it < iters; ++it) pass();
  const double sec = std::chrono::duration<double>(std::chrono::steady_clock::now() - t0).count();
  if (sec <= 0.0) return FT_ERR_INVALID;
  *gbs = (double)bytes * iters / sec / 1e9;
  return FT_OK;
}

int ft_cache_simulate(int num_layers, int num_experts, int capacity, const int* ops,
                      int n_ops_ints, ft_access_t* trace, int trace_cap, int* n_trace,
                      ft_cache_stats_t* stats, int* n_capacity_errors) {
  if (num_layers < 1 || num_experts < 1 || capacity < 1 || n_ops_ints < 0 ||
      (n_ops_ints > 0 && !ops) || !n_trace || trace_cap < 0 || (trace_cap > 0 && !trace))
    return FT_ERR_INVALID;
  ftc::SlotLru lru;
  lru.reset(num_layers * num_experts, capacity);
  std::vector<ftc::Access> recs;
  ft_cache_stats_t st{};
  int cap_err = 0;
  int i = 0;
  while (i < n_ops_ints) {
    if (ops[i] == 0) {
      if (i + 5 > n_ops_ints) return FT_ERR_INVALID;
      const int call = ops[i + 1], layer = ops[i + 2], kind = ops[i + 3], n = ops[i + 4];
      if (layer < 0 || layer >= num_layers || n < 0 || i + 5 + n > n_ops_ints ||
          (kind != FT_ROUTED && kind != FT_PREFETCH))
        return FT_ERR_INVALID;
      std::vector<int> keys;
      for (int j = 0; j < n; ++j) {
        const int e = ops[i + 5 + j];
        if (e < 0 || e >= num_experts) return FT_ERR_INVALID;
        keys.push_back(layer * num_experts + e);
      }
      std::sort(keys.begin(), keys.end());
      keys.erase(std::unique(keys.begin(), keys.end()), keys.end());
      const size_t first = recs.size();
      if (!lru.access_set(keys, num_experts, call, kind, recs)) {
        cap_err++;
      } else {
        for (size_t r = first; r < recs.size(); ++r) {
          const ftc::Access& a = recs[r];
          if (a.kind == FT_ROUTED) { st.routed++; if (a.hit) st.hits++; else st.misses++; }
          else { st.prefetch++; if (a.hit) st.prefetch_hits++; else st.prefetch_misses++; }
          if (a.ev_layer >= 0) st.evictions++;
        }
      }
      i += 5 + n;
    } else if (ops[i] == 1) {
      if (i + 2 > n_ops_ints || ops[i + 1] < 1) return FT_ERR_INVALID;
      std::vector<int> evicted;
      std::vector<std::pair<int, int>> moves;
      lru.resize(ops[i + 1], evicted, moves);
      st.evictions += (long long)evicted.size();
      i += 2;
    } else {
      return FT_ERR_INVALID;
    }
  }
  *n_trace = (int)recs.size();
  for (int r = 0; r < std::min(trace_cap, *n_trace); ++r) {
    const ftc::Access& a = recs[r];
    trace[r] = ft_access_t{a.call, a.layer, a.expert, a.kind, a.hit, a.slot, a.ev_layer, a.ev_expert};
  }
  st.resident = lru.size();
  st.capacity = lru.capacity();
  if (stats) *stats = st;
  if (n_capacity_errors) *n_capacity_errors = cap_err;
  return FT_OK;
}

// ------------------------------------------------------------ step level --

int ft_router_topk(const void* x, int x_is_bf16, const float* router_w, int T, int H, int E,
                   int top_k, int gating, float* logits, int* ids, float* gates, void* stream) {
  if (T < 0 || H < 4 || H % 4 || E < 1 || E > FT_MAX_EXPERTS || top_k < 1 || top_k > E ||
      top_k > FT_MAX_TOPK || (T > 0 && (!x || !router_w || !logits || !ids || !gates)))
    return FT_ERR_INVALID;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  // the forward's choice: the tiled router above 64 tokens
  const cudaError_t le = T > 64 ? ftk::launch_router_logits_tiled(x, x_is_bf16 != 0, router_w, T, H, E, logits, s)
                                : ftk::launch_router_logits(x, x_is_bf16 != 0, router_w, T, H, E, logits, s);
  if (le != cudaSuccess) return FT_ERR_CUDA;
  if (ftk::launch_topk_gates(logits, T, E, top_k, gating, ids, gates, s) != cudaSuccess)
    return FT_ERR_CUDA;
  return FT_OK;
}

int ft_route_decode(const void* x, int x_is_bf16, const float* router_w, int T, int H, int E, int top_k,
                    int gating, float* logits, int* ids, float* gates, int* counts, int* offsets, int* perm,
                    int* inv, int* ticket, void* stream) {
  if (T < 0 || T > 64 || H < 4 || H % 4 || E < 1 || E > FT_MAX_EXPERTS || top_k < 1 || top_k > E ||
      top_k > FT_MAX_TOPK || !ticket || !counts || !offsets ||
      (T > 0 && (!x || !router_w || !logits || !ids || !gates || !perm || !inv)))
    return FT_ERR_INVALID;
  return ftk::launch_route_decode(x, x_is_bf16 != 0, router_w, T, H, E, top_k, gating, logits, ids, gates,
                                  counts, offsets, perm, inv, ticket, static_cast<cudaStream_t>(stream)) ==
                 cudaSuccess
             ? FT_OK
             : FT_ERR_CUDA;
}

int ft_permute(const int* ids, int T, int top_k, int E, int* counts, int* offsets, int* perm,
               int* inv, void* stream) {
  if (T < 0 || top_k < 1 || E < 1 || E > FT_MAX_EXPERTS || !counts || !offsets ||
      (T > 0 && (!ids || !perm)))
    return FT_ERR_INVALID;
  return ftk::launch_permute(ids, T, top_k, E, counts, offsets, perm, inv,
                             static_cast<cudaStream_t>(stream)) == cudaSuccess
             ? FT_OK
             : FT_ERR_CUDA;
}

int ft_expert_ffn_decode(const void* x, int T, int H, int I, int top_k, int wdtype,
                         const void* const* blobs, const int* experts, int n_list,
                         int max_pairs_per_expert, const int* offsets, const int* perm, float* h,
                         float* y, void* stream) {
  if (T < 0 || H < 8 || I < 8 || H % 8 || I % 8 || top_k < 1 || n_list < 0 ||
      n_list > ftk::kMaxList || wdtype < FT_W_F32 || wdtype > FT_W_NVFP4 ||
      (wdtype == FT_W_INT4_G128 && (H % 128 || I % 128)) || (wdtype == FT_W_NVFP4 && (H % 32 || I % 32)) ||
      (n_list > 0 && (!blobs || !experts || !offsets || !perm || !h || !y || !x)))
    return FT_ERR_INVALID;
  ftk::ExpertList list;
  list.n = n_list;
  for (int i = 0; i < n_list; ++i) {
    if (experts[i] < -1 || experts[i] >= FT_MAX_EXPERTS || !blobs[i]) return FT_ERR_INVALID;
    list.expert[i] = experts[i];
    list.blob[i] = static_cast<const uint8_t*>(blobs[i]);
  }
  return ftk::launch_ffn_decode(x, T, H, I, top_k, wdtype, list, max_pairs_per_expert, offsets,
                                perm, h, y, static_cast<cudaStream_t>(stream), nullptr) == cudaSuccess
             ? FT_OK
             : FT_ERR_CUDA;
}

int ft_expert_ffn_prefill(const void* x, int T, int H, int I, int top_k, const void* weights, int n_slots,
                          const int* experts, const int* slots, int n_list, const int* offsets, const int* perm,
                          void* a_rows, void* h, float* y, int* err, void* stream) {
  auto bad = [](const char* why) {
    ftk::set_step_error(std::string("ft_expert_ffn_prefill: ") + why);
    return FT_ERR_INVALID;
  };
  if (T < 0 || top_k < 1 || n_list < 0 || n_list > ftk::kMaxList || n_slots < 1)
    return bad("invalid size");
  if (H < 256 || I < 128 || H % 256 || I % 128) return bad("H must be a multiple of 256 and I of 128");
  if (T == 0 || n_list == 0) return FT_OK;
  if (!x || !weights || !experts || !slots || !offsets || !perm || !a_rows || !h || !y || !err)
    return bad("null pointer");
  if (((uintptr_t)weights | (uintptr_t)a_rows | (uintptr_t)h) & 15) return bad("buffers must be 16-byte aligned");
  ftk::GemmGroups groups;
  groups.n = n_list;
  int n_shared = 0;
  for (int i = 0; i < n_list; ++i) {
    if (experts[i] < -1 || experts[i] >= FT_MAX_EXPERTS || slots[i] < 0 || slots[i] >= n_slots)
      return bad("bad expert list entry");
    n_shared += experts[i] < 0;
    groups.expert[i] = experts[i];
    groups.z[i] = slots[i];
  }
  if (n_shared > 1) return bad("more than one shared-expert entry");
  const uint64_t rows = (uint64_t)T * top_k + T;
  const uint64_t blob = 3ull * H * I * 2;
  const unsigned char* w = static_cast<const unsigned char*>(weights);
  ftk::GemmMaps m;
  bool ok = ftk::encode_map_2d(&m.a_x, a_rows, H, rows, (uint64_t)H * 2, 128) &&
            ftk::encode_map_2d(&m.a_h, h, I, rows, (uint64_t)I * 2, 128) &&
            ftk::encode_map_3d(&m.b1_routed, w, H, 2ull * I, n_slots, (uint64_t)H * 2, blob, 128) &&
            ftk::encode_map_3d(&m.b2_routed, w + 2ull * I * H * 2, I, H, n_slots, (uint64_t)I * 2, blob, 256);
  if (!ok) {
    ftk::set_step_error("ft_expert_ffn_prefill: cuTensorMapEncodeTiled failed");
    return FT_ERR_CUDA;
  }
  m.b1_shared = m.b1_routed;   // the shared expert is a slot of the same array
  m.b2_shared = m.b2_routed;
  int dev = 0, num_sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&num_sms, cudaDevAttrMultiProcessorCount, dev);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaError_t e = ftk::launch_gather_rows(x, perm, T, top_k, H, n_shared > 0, a_rows, s);
  if (e == cudaSuccess)
    e = ftk::launch_grouped_gemm(0, m, groups, offsets, T, top_k, I, H, h, err, num_sms, s);
  if (e == cudaSuccess)
    e = ftk::launch_grouped_gemm(1, m, groups, offsets, T, top_k, I, H, y, err, num_sms, s);
  if (e != cudaSuccess) {
    ftk::set_step_error(std::string("ft_expert_ffn_prefill: launch: ") + cudaGetErrorString(e));
    return FT_ERR_CUDA;
  }
  return FT_OK;
}

int ft_combine(const float* y, const float* gates, const int* inv, int T, int H, int top_k,
               int has_shared, int out_is_bf16, void* out, void* stream) {
  if (T < 0 || H < 4 || H % 4 || top_k < 1 || (T > 0 && (!y || !gates || !inv || !out)))
    return FT_ERR_INVALID;
  return ftk::launch_combine(y, gates, inv, T, H, top_k, has_shared != 0, out_is_bf16 != 0, out,
                             static_cast<cudaStream_t>(stream)) == cudaSuccess
             ? FT_OK
             : FT_ERR_CUDA;
}

}  // extern "C"

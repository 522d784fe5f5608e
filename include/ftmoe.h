/*
 * ftmoe.h - C ABI of a routed mixture-of-experts layer stack executed against
 * a shared LRU cache of expert slots in GPU memory (NVIDIA B200, sm_100a).
 *
 * The method (FreeToken pages):
 *  - The router activates a few experts per token, e.g. 6 of 256 routed
 *    experts ("FreeToken linux", section "FreeToken's MoE memory handling").
 *  - The full routed-expert pool lives in host memory and stays the reference
 *    copy.  Spare GPU memory holds expert slots.  One LRU policy, shared by
 *    every MoE layer, decides which experts the slots hold (same section;
 *    "FreeToken gguf", MoE backends, `offload`).
 *  - A missed expert is copied over PCIe into a slot and kept for reuse (same
 *    sections).  Executing misses on the CPU is not part of this library.
 *  - Prefill streams the next layer's experts while the current layer runs
 *    (whole-layer double buffering; "FreeToken linux", same section;
 *    "FreeToken RTX 5090", prefill and decode).
 *  - The cache can be resized at a safe point without a restart.  Capacity
 *    changes speed, never the result ("FreeToken RTX 5090", dynamic
 *    reconfiguration; "FreeToken linux", elastic cache resize).
 *
 * The pages give no API.  The names below follow their problem statement.
 *
 * Conventions for every entry point:
 *  - "device" pointers are CUDA global-memory addresses on the device that was
 *    current when the handle was created.  "host" pointers are CPU memory.
 *  - `stream` is a cudaStream_t passed as void* (NULL = the legacy default stream).
 *  - Calls returning int return an ft_status.  On error they leave a message
 *    in ft_last_error(h).
 *  - The caller owns x, router weights, out and all ft_* argument buffers.
 *    The library owns the pinned pool, the slot arena, shared-expert memory,
 *    scratch, its copy stream and its events.
 *  - A handle is not thread-safe: use one host thread per handle at a time.
 */
#ifndef FTMOE_H
#define FTMOE_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define FT_API __attribute__((visibility("default")))
#else
#define FT_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef struct ft_moe ft_moe; /* opaque; owned by the library */

enum ft_status {
  FT_OK = 0,
  FT_ERR_INVALID = 1,      /* bad argument or call order; nothing was changed */
  FT_ERR_OOM = 2,          /* device or pinned-host allocation failed */
  FT_ERR_CUDA = 3,         /* a CUDA call failed; cache state of the failed fills is rolled back */
  FT_ERR_CAPACITY = 4,     /* one step needs more distinct experts than there are slots */
  FT_ERR_BUSY = 5,         /* resize or destroy requested while a forward is in flight */
  FT_ERR_TIMEOUT = 6,      /* a host wait on the GPU passed its deadline */
  FT_ERR_DEVICE_CHECK = 7  /* a kernel's bounded wait gave up, or its own check failed (the message
                              gives the code from the device error word) */
};

enum ft_wdtype { FT_W_F32 = 0, FT_W_BF16 = 1, FT_W_INT4_G128 = 2, FT_W_NVFP4 = 3 };
enum ft_gating { FT_GATE_SOFTMAX = 0, FT_GATE_SIGMOID = 1 };
enum ft_access_kind { FT_ROUTED = 0, FT_PREFETCH = 1 };

/* Largest supported number of routed experts per layer. */
#define FT_MAX_EXPERTS 256
/* Largest supported top-k. */
#define FT_MAX_TOPK 16

/* Cache counters since creation (or since the last ft_cache_reset_stats). */
typedef struct {
  long long routed;           /* routed accesses: one per distinct expert per layer per forward */
  long long hits;             /* routed accesses found resident */
  long long misses;           /* routed accesses filled from the host pool */
  long long evictions;        /* entries dropped to make room (fills and shrinks) */
  long long prefetch;         /* prefetch accesses (prefill mode) */
  long long prefetch_hits;
  long long prefetch_misses;  /* prefetch accesses that copied an expert */
  long long h2d_bytes;        /* bytes copied host -> slot */
  double h2d_seconds;         /* copy-stream time of those copies, from CUDA events */
  int resident;               /* occupied slots */
  int capacity;               /* slots */
} ft_cache_stats_t;

/* One cache access, in the order the cache saw them. */
typedef struct {
  int call;       /* forward-call index of the handle, from 0 */
  int layer;
  int expert;
  int kind;       /* ft_access_kind */
  int hit;        /* 1 = resident already */
  int slot;       /* slot used */
  int ev_layer;   /* key evicted to make room, or -1 */
  int ev_expert;
} ft_access_t;

/* ------------------------------------------------------------------------ *
 * Cache-level API
 * ------------------------------------------------------------------------ */

/* Creates a stack description with `cache_slots` expert slots of one blob each.
 * Source: "FreeToken linux", "FreeToken's MoE memory handling" (the routed experts
 * live in host memory; a fixed share of GPU memory holds expert slots; e.g. 6 of 256
 * experts per token) and "FreeToken gguf", MoE backends (`offload`: the experts stay
 * in host memory and a GPU cache holds the hot ones).
 *   num_experts E (1..FT_MAX_EXPERTS), top_k k (1..min(E, FT_MAX_TOPK)),
 *   hidden H and inter I (SwiGLU intermediate): multiples of 8.  For
 *   FT_W_INT4_G128 they must be multiples of 128, for FT_W_NVFP4 of 32.  wdtype is an
 *   ft_wdtype.
 * The stack starts with 1 layer, softmax gating and no shared expert.  Call
 * ft_moe_set_layers before filling the pool.  Allocates the slot arena on the
 * current device; the pinned pool is allocated by ft_moe_set_layers.
 * Returns NULL on failure, with the reason in ft_last_error(NULL). */
FT_API ft_moe* ft_moe_create(int num_experts, int top_k, int hidden, int inter, int wdtype,
                      int cache_slots);

/* Source: "FreeToken linux", "FreeToken's MoE memory handling" (one cache shared by
 * every MoE layer of the model).
 * Sets the number of layers L, the gating (ft_gating) and whether each layer has one
 * always-on shared expert (gate weight 1).  (Re)allocates the pinned host pool of
 * L*E expert blobs (contents undefined until written) and the resident shared-expert
 * memory (zeroed).  The cache is emptied.  Not allowed while a forward is in flight. */
FT_API int ft_moe_set_layers(ft_moe* h, int num_layers, int gating, int has_shared_expert);

/* Bytes of one expert blob (the runtime layout below). */
FT_API size_t ft_moe_blob_bytes(const ft_moe* h);

/* Source: "FreeToken linux", "FreeToken's MoE memory handling" (the full routed-expert
 * pool stays in host memory as the reference copy; misses are copied from it) and
 * "FreeToken linux", setup (the weights are prepared once in the runtime layout).
 * Host address of routed expert (layer, expert) in the library-owned pinned pool,
 * or NULL for bad indices.  Blobs are contiguous in (layer, expert) order:
 * ft_moe_pool_ptr(h, l, e) = ft_moe_pool_ptr(h, 0, 0) + (l*E + e) * ft_moe_blob_bytes(h).  The caller writes the expert's blob there before the
 * first forward that can read it.  A blob already copied into a slot is not copied
 * again until evicted.
 * Runtime blob layout (row-major, K = reduction axis contiguous):
 *   f32 / bf16: W_gate [I][H], W_up [I][H], W_down [H][I].
 *   int4 g128:  packed W_gate [I][H/2], W_up [I][H/2], W_down [H][I/2] bytes.  Byte b
 *               of a row holds element 2b in its low nibble and 2b+1 in its high
 *               nibble, two's complement in [-8, 7].  Then the bf16 scales
 *               S_gate [I][H/128], S_up [I][H/128], S_down [H][I/128], one per 128
 *               consecutive K elements of a row.  w = q * s.
 *   nvfp4:      packed e2m1 W_gate [I][H/2], W_up [I][H/2], W_down [H][I/2] (same nibble
 *               order; code bit 3 sign, bits 2-1 exponent bias 1, bit 0 mantissa), then
 *               e4m3 block scales S_gate [I][H/16], S_up [I][H/16], S_down [H][I/16] (one
 *               byte per 16 consecutive K elements), then the fp32 global scales g_gate,
 *               g_up, g_down and 4 zero bytes.  w = e2m1(q) * e4m3(s) * g.  H and I must
 *               be multiples of 32.  Decode runs the streaming GEMV on these codes;
 *               prefill (the GEMM path) expands each weight tile exactly to bf16
 *               (e2m1 * e4m3) in shared memory inside the GEMM and applies g to its
 *               accumulators. */
FT_API void* ft_moe_pool_ptr(ft_moe* h, int layer, int expert);

/* Source: the stated DeepSeek-V4-Flash-shaped workloads (one always-on shared expert;
 * the pages name none, so it is kept resident and added with weight 1).
 * Copies the shared expert of `layer` (a host blob in the same layout) into resident
 * device memory.  Synchronous. */
FT_API int ft_moe_set_shared(ft_moe* h, int layer, const void* host_blob);

/* Source: "FreeToken linux", "FreeToken's MoE memory handling", and "FreeToken RTX
 * 5090", prefill and decode (whole-layer double buffering during prefill: the next
 * layer's experts stream in while the current layer computes).
 * Decode (0) or prefill (1) cache policy.  Prefill: a forward of layer 0 first
 * prefetches every expert of layer 0, and each forward of layer l issues the
 * prefetch of every expert of layer l+1 on the copy stream after its own routed
 * accesses, so the copy overlaps layer l's kernels. */
FT_API int ft_moe_set_mode(ft_moe* h, int prefill);

/* Grows the per-forward scratch for up to max_tokens tokens (forward grows it on
 * demand too, with a device synchronisation). */
FT_API int ft_moe_reserve(ft_moe* h, int max_tokens);

/* One MoE layer on n_tokens tokens.
 * Source: "FreeToken linux", "FreeToken's MoE memory handling" (the router picks a few
 * experts per token; each picked expert runs from the GPU slot that holds it, a missed
 * one being copied there over PCIe first; the outputs are mixed by the gate weights)
 * and "FreeToken RTX 5090", dynamic reconfiguration (capacity changes speed, never the
 * result: every forward computes the dense MoE layer exactly).
 *   x        device [n_tokens][H], float32 for FT_W_F32 stacks, bf16 otherwise.
 *   router_w device [E][H] float32.
 *   out      device [n_tokens][H], same type as x.
 *   stream   caller's stream; every kernel and the wait for slot fills run on it.
 * Steps: router logits (fp32) and top-k with normalised gates; one host read of
 * the selected expert ids (for up to 64 tokens the routing kernel writes them to mapped
 * pinned memory, otherwise a device-to-host copy; the host waits, with a deadline);
 * the LRU lookup and update over the distinct selected experts (hits in ascending
 * expert order first, then misses in ascending order, each taking the lowest free slot
 * or evicting the least recently used entry); copies of missed experts from the
 * pinned pool into their slots on the library's copy stream, each after the
 * kernels that last read the slot; token permutation by expert; the SwiGLU FFN of
 * every selected expert reading its weights from its slot (on the GEMV path the
 * experts already resident run before the wait for this call's copies); the
 * gate-weighted sum of the k outputs in ascending k order, plus the shared expert.
 * Returns FT_ERR_CAPACITY, before any state changes, if the distinct experts of
 * the call exceed the cache slots.  All forwards of a handle are ordered: a
 * forward on another stream first waits for the previous forward's kernels.  A forward
 * that fails after its first launch drains `stream` before returning, except on
 * FT_ERR_TIMEOUT, after which the caller should call ft_moe_sync before using the
 * handle on another stream. */
FT_API int ft_moe_forward(ft_moe* h, int layer, const void* x, int n_tokens, const float* router_w,
                   void* out, void* stream);

/* Waits for every forward and copy of the handle, then checks the device error word
 * that a kernel sets when one of its bounded waits gives up (FT_ERR_DEVICE_CHECK; the
 * word is cleared): codes 101-106 the prefill GEMM's pipeline waits, 111 the fused
 * decode FFN's wait for an expert's gate/up rows.  A forward also reports a word set
 * by an earlier forward. */
FT_API int ft_moe_sync(ft_moe* h);

/* Expert FFN path: bf16 stacks with H % 256 == 0 and I % 128 == 0, and nvfp4 stacks with
 * H % 256 == 0 and I % 256 == 0, use the tcgen05 grouped GEMMs when n_tokens * k >= min_avg_pairs * |S| (on average at least
 * min_avg_pairs tokens per selected expert; default 32), else the streaming GEMV.
 * Both compute the same function.  0 always selects the GEMMs where shapes allow. */
FT_API int ft_moe_set_gemm_threshold(ft_moe* h, int min_avg_pairs);

/* Routing launch shape for calls of up to 64 tokens: 1 (default) = one fused kernel
 * (ft_route_decode), 0 = router, top-k and permutation as three launches.  Same results. */
FT_API int ft_moe_set_fused_routing(ft_moe* h, int enabled);

/* Decode FFN launch shape (the GEMV path).  Either way the experts whose slots this
 * stream has already waited for run before the wait for this call's misses, and the rest
 * after it.  0 (default) = per group a gate/up and a down launch, then one combine;
 * 1 = per group one fused kernel that runs gate/up + SwiGLU, down and (in the last group)
 * the combine.  The per-output arithmetic is the same, so the outputs are bit-identical. */
FT_API int ft_moe_set_fused_ffn(ft_moe* h, int enabled);

/* Decode GEMV for int4, NVFP4 and bf16 weights (per-pass launch shape): 1 (default) = on the
 * tensor cores (mma.sync), 0 = fp32 multiply-adds on the CUDA cores.  int4: the int8 tensor
 * cores (m16n8k32: the nibbles as signed bytes 16 q, the inputs x and h as 16-bit block fixed
 * point in two bytes, exact int32 products per 128-element group, scaled and summed in fp32).
 * NVFP4 with H and I multiples of 128: the f16 tensor cores (m16n8k16: e2m1 code times e4m3
 * block scale formed exactly as f16, the inputs as f16 rows with a per-row power-of-two scale,
 * fp32 accumulators).  bf16 with H and I multiples of 32 and 2 or more tokens: the bf16 tensor
 * cores (m16n8k16: the weights as stored, x as stored, h as bf16 hi + lo halves, fp32
 * accumulators); one token runs on the fp32 pipes, which stream the weights faster there.  Other shapes
 * and formats use the fp32 pipes.  Both choices are within the stated bound of the oracle;
 * their outputs differ in the last bits.  ft_expert_ffn_decode always uses the tensor cores. */
FT_API int ft_moe_set_int4_tensor_cores(ft_moe* h, int enabled);

/* Host-side fault injection for tests of failure handling (no GPU fault is made).
 *   FT_INJECT_COPY_FAIL: the countdown-th slot fill from now is reported failed instead
 *     of being issued.  The forward returns FT_ERR_CUDA before launching its FFN; the
 *     entries of that fill and of the later fills of the same set become not resident
 *     (their accesses stay in the trace); the fills of the set issued before it stay
 *     resident, and a later forward that reads them waits for their copies.  The next
 *     forward works normally.
 *   FT_INJECT_ROUTE_TIMEOUT: the countdown-th routing wait reports FT_ERR_TIMEOUT (after
 *     the GPU work completes); the cache is unchanged.
 *   FT_INJECT_FUSED_WAIT: in the countdown-th fused decode FFN launch every down item
 *     waits for one gate/up item more than exist, so each of those device waits gives
 *     up after 1 ms and writes code 111 to the error word; the kernel still completes,
 *     and the next forward (or ft_moe_sync) reports FT_ERR_DEVICE_CHECK.
 * countdown 0 disarms. */
enum ft_inject { FT_INJECT_COPY_FAIL = 1, FT_INJECT_ROUTE_TIMEOUT = 2, FT_INJECT_FUSED_WAIT = 3 };
FT_API int ft_moe_debug_inject(ft_moe* h, int what, int countdown);

/* Runs one CTA that waits, with the same bounded wait the prefill GEMM kernels use, on a
 * barrier that nothing arrives on, for limit_us microseconds (1..1e6).  The wait gives up,
 * records the failure in an error word, and the kernel returns: FT_ERR_DEVICE_CHECK is the
 * expected result, and the context stays usable.  Allocates 4 bytes stream-ordered. */
FT_API int ft_debug_device_wait_selftest(int limit_us, void* stream);

/* Copies the routing of the last forward to host memory: ids [n_tokens][k] (expert
 * indices, by descending logit, ties to the lower index) and gates [n_tokens][k].
 * Either pointer may be NULL. */
FT_API int ft_moe_last_routing(const ft_moe* h, int* ids, float* gates, int* n_tokens);

/* Source: "FreeToken RTX 5090", dynamic reconfiguration, and "FreeToken linux", elastic
 * cache resize (the cache grows or shrinks at a safe point without a restart; a shrink
 * under memory pressure costs some speed, e.g. -7% from 58% to 40% of the model in the
 * cache demo of "this tool runs datacenter AI on your PC").
 * Changes the number of slots at a safe point: waits for all work of the handle,
 * then grows (entries keep slot and recency; new slots are free) or shrinks
 * (least recently used entries are evicted down to the new size; survivors in
 * slots >= slots are moved, most recent first, into the lowest free slots below
 * it, keeping recency).  Reallocates the arena and copies resident slots on the
 * device.  FT_ERR_BUSY if a forward is in flight on another thread. */
FT_API int ft_cache_resize(ft_moe* h, int slots);

/* Empties the cache at a safe point (waits for the handle's work): every slot becomes
 * free, capacity, counters and trace are kept. */
FT_API int ft_cache_clear(ft_moe* h);

/* Source: "FreeToken linux", performance (the miss rate of expert reads, e.g. 16% for
 * the shared LRU against 62% for a static split) and "FreeToken's MoE memory handling"
 * (the runtime measures the pinned-memory transfer bandwidth over PCIe).
 * Reads the counters (waits for the copy stream so h2d_seconds is complete). */
FT_API int ft_cache_stats(const ft_moe* h, ft_cache_stats_t* out);
FT_API int ft_cache_reset_stats(ft_moe* h);

/* Source: "FreeToken RTX 5090" (miss rates of the cache policies measured on the same
 * replayed routing traces).
 * Copies up to `cap` trace records, oldest first, into buf and sets *n to the
 * number recorded since the trace was last cleared (may exceed cap).  Tracing is
 * on by default; ft_cache_set_trace(h, 0) turns it off and clears it. */
FT_API int ft_cache_trace(const ft_moe* h, ft_access_t* buf, int cap, int* n);
FT_API int ft_cache_set_trace(ft_moe* h, int enabled);

/* Slot currently holding (layer, expert), or -1. */
FT_API int ft_cache_slot_of(const ft_moe* h, int layer, int expert);

/* Device address of slot s in the arena (valid until the next resize). */
FT_API void* ft_cache_slot_ptr(ft_moe* h, int slot);

/* Per-stage device time and launch counts of the handle's forwards.  Stage times are
 * summed CUDA-event intervals on the forward's stream, taken only while stage timing
 * is on; ffn_gate_up and ffn_down start after the wait for slot fills, so they hold
 * kernel time only.  *_bytes are the algorithmic bytes of those launches: the weight
 * bytes of every selected expert (and the shared expert) plus their input and output
 * vectors. */
typedef struct {
  long long forwards;
  long long kernel_launches;
  long long timed_forwards;
  double router_ms;        /* router logits + top-k/gates */
  double permute_ms;
  double ffn_gate_up_ms;   /* gate/up GEMV or GEMM + SwiGLU */
  double ffn_down_ms;
  double combine_ms;
  double ffn_gate_up_bytes;
  double ffn_down_bytes;
  double ffn_flops;        /* 2 * (3 * H * I) per (token, expert) pair */
  double host_wait_ms;     /* host time spent waiting for the routing ids */
  /* Fused decode FFN (gate/up + SwiGLU + down + combine in one launch, the default for
   * the GEMV path): kernel time, algorithmic bytes (the weights of every listed expert,
   * x in and out back) and launches.  A forward whose experts are partly still being
   * copied runs two launches (the resident experts first), so launches >= forwards. */
  double ffn_fused_ms;
  double ffn_fused_bytes;
  long long ffn_fused_launches;
  long long ffn_gate_up_launches;   /* per-pass gate/up launches (two where a forward is split) */
  double host_issue_ms;  /* host time from the routing's arrival to the last launch queued: the
                            LRU, the fills and the FFN launches (on the path of every forward) */
} ft_perf_t;

/* Stage timing holds the forward's stream with a one-thread kernel while the host queues
 * each stage, so the CUDA events around a launch time the kernel, not the host issuing
 * it; and every forward's FFN then runs after the wait for its fills (no split into
 * resident and copied experts), so each launch covers the forward's whole list.  For
 * measurement only: it serialises the host and the GPU. */
FT_API int ft_moe_set_stage_timing(ft_moe* h, int enabled);
/* Waits for the timed forwards and reads the counters. */
FT_API int ft_moe_perf(ft_moe* h, ft_perf_t* out);
FT_API int ft_moe_reset_perf(ft_moe* h);

/* Deadline of every host wait on the GPU, in milliseconds (default 20000). */
FT_API int ft_moe_set_timeout_ms(ft_moe* h, int ms);

/* The pages give no error reporting; this is the plainest completion of their API.
 * Message of the last failed call on h, or of the last failed ft_moe_create when
 * h is NULL (per host thread). */
FT_API const char* ft_last_error(const ft_moe* h);

/* The pages give no teardown; this is the plainest completion of their API.
 * Waits for the handle's work and frees everything it owns. */
FT_API void ft_moe_destroy(ft_moe* h);

/* Host-only replay of the cache policy (no GPU, no allocation on the device): runs the
 * library's own slot table over a script and reports what the cache would do.  For
 * capacity planning and for checking the policy without a GPU.
 * ops is a flat int array of records:
 *   {0, call, layer, kind, n, e_1 .. e_n}  one access set (distinct experts of one layer;
 *                                           any order, they are sorted first)
 *   {1, new_capacity}                      a resize at a safe point
 * A set larger than the capacity is skipped, changes nothing, and is counted in
 * *n_capacity_errors.  trace receives up to trace_cap records; *n_trace is the total.
 * stats (may be NULL) receives the counters (h2d fields zero).  Returns FT_ERR_INVALID
 * for a malformed script or out-of-range ids. */
FT_API int ft_cache_simulate(int num_layers, int num_experts, int capacity, const int* ops,
                             int n_ops_ints, ft_access_t* trace, int trace_cap, int* n_trace,
                             ft_cache_stats_t* stats, int* n_capacity_errors);

/* The same replay under another placement policy, to compare the shared LRU with the
 * static layer split the pages contrast it with ("FreeToken linux", performance: at
 * one RTX 5090 capacity the LRU missed 16% of expert reads where a static split missed
 * 62%; "this tool runs datacenter AI on your PC": static placement vs dynamic caching).
 *   FT_POLICY_LRU:    ft_cache_simulate.
 *   FT_POLICY_STATIC: the first `capacity` keys in (layer, expert) order stay resident for
 *                     good (slot = key); every other access is a miss that is served
 *                     without being cached (slot -1, nothing evicted).  A resize changes
 *                     which keys are resident.
 * Arguments and script format as for ft_cache_simulate. */
enum ft_policy { FT_POLICY_LRU = 0, FT_POLICY_STATIC = 1 };
FT_API int ft_cache_simulate_policy(int policy, int num_layers, int num_experts, int capacity,
                                    const int* ops, int n_ops_ints, ft_access_t* trace, int trace_cap,
                                    int* n_trace, ft_cache_stats_t* stats, int* n_capacity_errors);

/* Measures the host link the slot fills use ("FreeToken linux", setup: measure the
 * pinned-memory PCIe bandwidth on the machine rather than trusting the specification):
 * `iters` copies of `bytes` between pinned host memory and the current device, each way,
 * timed with CUDA events on a private stream.  Allocates and frees its own buffers. */
FT_API int ft_probe_host_link(size_t bytes, int iters, double* h2d_gbs, double* d2h_gbs);

/* Host memory copy bandwidth (no GPU): `iters` memcpy passes of `bytes` between two
 * host buffers, split over `threads` threads (1..256), timed with a steady clock.
 * *gbs = bytes * iters / seconds / 1e9 (copied bytes, not read + written).  With the
 * link probe it forms the bandwidth profile a CPU/GPU placement policy would read
 * ("FreeToken linux": the bandwidth check of the setup).  Allocates and frees its own
 * buffers; FT_ERR_OOM if they cannot be allocated. */
FT_API int ft_probe_host_memory(size_t bytes, int threads, int iters, double* gbs);

/* ------------------------------------------------------------------------ *
 * Step-level kernels.  Each runs one step of the forward on caller-owned device
 * buffers, on `stream`, without the cache.  They are the same kernels the
 * forward launches.  They allocate nothing, return after the launch, and report
 * launch errors only.
 * ------------------------------------------------------------------------ */

/* Router + gating ("FreeToken linux", MoE memory handling: a few experts per token).
 * z[t][e] = sum_h x[t][h] * router_w[e][h] in fp32.  ids[t][:] = the top_k experts
 * by z (descending, ties to the lower index).  gates[t][j] = softmax or sigmoid of
 * the selected logits, normalised over the k selected.
 *   x: [T][H] (x_is_bf16 ? bf16 : f32), router_w: [E][H] f32, logits: [T][E] f32
 *   (written), ids: [T][k] int32, gates: [T][k] f32.
 * Above 64 tokens the logits come from the forward's tiled router: each logit sums a partial
 * per 32 elements of H into its accumulator, in H order.  With H % 32 == 0 and 16-byte
 * aligned x and router_w the K steps stream through shared memory with cp.async: bf16 x on
 * the tf32 tensor cores (bf16 is exact in tf32; each router weight is split into tf32 hi + lo,
 * within 2^-21 of it), fp32 x on the fp32 pipes.  Otherwise a one-step kernel on the fp32
 * pipes computes the fp32-pipe sums, bit for bit. */
FT_API int ft_router_topk(const void* x, int x_is_bf16, const float* router_w, int T, int H, int E,
                   int top_k, int gating, float* logits, int* ids, float* gates, void* stream);

/* Router + gating + token permutation in one launch, for decode-sized batches (T <= 64):
 * the results of ft_router_topk followed by ft_permute (with inv), bit for bit the same
 * selection and order.  ticket: a device int that is 0 before the first call; every call
 * leaves it 0 again (one ticket per stream of calls). */
FT_API int ft_route_decode(const void* x, int x_is_bf16, const float* router_w, int T, int H, int E,
                           int top_k, int gating, float* logits, int* ids, float* gates, int* counts,
                           int* offsets, int* perm, int* inv, int* ticket, void* stream);

/* Token permutation by expert.  counts[e] = pairs routed to e; offsets = exclusive
 * prefix sum (E+1 entries); perm[q] = flat pair index t*k + j for q in expert-major
 * order, ascending token inside an expert (a stable counting sort); inv (optional,
 * may be NULL) is its inverse: inv[t*k + j] = q.
 *   ids: [T][k] int32 in [0, E).  counts: [E], offsets: [E+1], perm, inv: [T*k] int32.
 * One CTA; T*k up to 2^31. */
FT_API int ft_permute(const int* ids, int T, int top_k, int E, int* counts, int* offsets, int* perm,
               int* inv, void* stream);

/* SwiGLU FFN of a list of experts for decode-sized batches: every weight byte is
 * read once per launch.  blobs and experts are HOST arrays of n_list entries
 * (n_list <= FT_MAX_EXPERTS + 1); blobs[i] is the DEVICE address of entry i's blob
 * (runtime layout, see ft_moe_pool_ptr).  Entry i owns the pairs q in
 * [offsets[e], offsets[e+1]) with e = experts[i], whose token is perm[q] / k; or, for
 * experts[i] = -1 (a shared expert), the pairs q = T*k + t for every token t.
 *     h[q] = silu(W_gate x_t) * (W_up x_t)        (h: [T*k + T][I] f32, device)
 *     y[q] = W_down h[q]                          (y: [T*k + T][H] f32, device)
 *   x: [T][H] device, f32 for FT_W_F32, else bf16.  max_pairs_per_expert: the largest
 *   pair count of one entry (sizes the per-CTA token staging; larger values are
 *   processed in chunks of 8).  Rows of h / y that no entry owns are not written.
 *   FT_W_INT4_G128 (the int8 tensor-core GEMV): the tokens and, between the two passes,
 *   the entries' h rows are rewritten as 16-bit block fixed point (a signed and an
 *   unsigned byte per value, then a float scale), the tokens in the first
 *   T * (2H + 16) bytes of y before the down pass writes y, the h rows in place; so after
 *   the call h holds that form, not the fp32 values, and rows of y that no entry owns may
 *   hold those bytes.
 *   FT_W_BF16 with H and I multiples of 32 and T >= 2 (the bf16 tensor-core GEMV): between the passes
 *   the entries' h rows are rewritten in place as bf16 hi and lo halves ([I hi][I lo] in the
 *   row's 4I bytes, 16 significant bits); x is read as it is.
 *   FT_W_NVFP4 with H and I multiples of 128 (the f16 tensor-core GEMV): likewise, with the
 *   tokens and h rows rewritten as f16 with a per-row power-of-two scale (then a float, the
 *   scale's inverse), the tokens in the first T * (2H + 16) bytes of y.  h rounds to 11
 *   significant bits there (relative error at most 2^-11 per element); x is exact.  Other
 *   NVFP4 shapes run on the fp32 pipes and leave h in fp32. */
FT_API int ft_expert_ffn_decode(const void* x, int T, int H, int I, int top_k, int wdtype,
                         const void* const* blobs, const int* experts, int n_list,
                         int max_pairs_per_expert, const int* offsets, const int* perm, float* h,
                         float* y, void* stream);

/* SwiGLU FFN of a list of experts for prefill-sized batches, on the tcgen05 grouped GEMMs
 * that ft_moe_forward runs in prefill ("FreeToken linux", "FreeToken's MoE memory
 * handling": in prefill every selected expert runs from the slot that holds it, while
 * the next layer's experts are copied in).  bf16 weights; H % 256 == 0, I % 128 == 0.
 *   weights: DEVICE array of n_slots bf16 expert blobs (runtime layout, see
 *     ft_moe_pool_ptr), 3*H*I*2 bytes apart, 16-byte aligned.  experts, slots: HOST
 *     arrays of n_list entries (n_list <= FT_MAX_EXPERTS + 1): entry i is routed expert
 *     experts[i] (its pairs q in [offsets[e], offsets[e+1])) or, for experts[i] = -1 (at
 *     most one entry), a shared expert (pairs q = T*k + t for every token t); its weights
 *     are blob slots[i] (0 <= slots[i] < n_slots) of `weights`.
 *   x: [T][H] bf16.  offsets [E+1], perm [T*k]: as written by ft_permute.
 *   a_rows: [T*k + T][H] bf16 scratch (written: the gathered token row of every pair).
 *   h: [T*k + T][I] bf16 (written): h[q] = bf16(silu(W_gate x_t) * (W_up x_t)), fp32 accumulation.
 *   y: [T*k + T][H] f32 (written): y[q] = W_down h[q], fp32 accumulation.
 *   err: a DEVICE int, 0 before the call; a kernel whose bounded pipeline wait gives up
 *     writes 101-104 there (the outputs are then incomplete).
 * Rows that no entry owns are not written.  Allocates nothing (the tensor maps are built
 * on the host per call).  FT_ERR_INVALID (message in ft_last_error(NULL)) for bad sizes,
 * entries or alignment; FT_ERR_CUDA if a launch fails. */
FT_API int ft_expert_ffn_prefill(const void* x, int T, int H, int I, int top_k, const void* weights, int n_slots,
                                 const int* experts, const int* slots, int n_list, const int* offsets,
                                 const int* perm, void* a_rows, void* h, float* y, int* err, void* stream);

/* Gate-weighted combine: out[t] = sum_{j<k} gates[t][j] * y[inv[t*k+j]], summed in
 * ascending j in fp32, plus y[T*k + t] (weight 1) when has_shared.
 *   y: device f32 rows (see ft_expert_ffn_decode), gates: [T][k] f32, inv: [T*k] int32,
 *   out: [T][H], bf16 if out_is_bf16 else f32 (round to nearest even).  H % 4 == 0. */
FT_API int ft_combine(const float* y, const float* gates, const int* inv, int T, int H, int top_k,
               int has_shared, int out_is_bf16, void* out, void* stream);

/* Size, in floats, of the static device scratch of ft_expert_ffn_decode_noalloc
 * (12 MiB).  Every GPU that loads this library holds it until the process exits. */
#define FT_NOALLOC_SCRATCH_FLOATS (3u * 1024u * 1024u)

/* The decode expert FFN followed by the gate-weighted combine, allocating nothing.
 * No FreeToken page has a counterpart of this call: it exists for callers that may not
 * allocate device memory while they run, such as a serving engine that fixes its whole
 * device-memory plan at start-up and owns every byte after that, or a caller on a
 * latency-critical decode loop that cannot pay cudaMalloc's implicit device
 * synchronisation.  Such callers still pass every input and output buffer; only the
 * intermediate rows that ft_expert_ffn_decode takes as caller buffers (h, y) move into a
 * file-scope static device array of FT_NOALLOC_SCRATCH_FLOATS floats.
 * Computes out[t] = sum_j gates[t][j] * y[inv[t*k+j]] (+ the shared expert's y with
 * weight 1 when has_shared), with h and y as defined for ft_expert_ffn_decode;
 * arguments as for ft_expert_ffn_decode and ft_combine (out: [T][H], f32 for FT_W_F32,
 * else bf16).
 *  - Limit: (T*k + T) * (I + H) <= FT_NOALLOC_SCRATCH_FLOATS; larger sizes return
 *    FT_ERR_INVALID before any launch, with the reason in ft_last_error(NULL).
 *  - Calls no cudaMalloc, cudaFree or other allocating routine.  The first call on a
 *    device looks up the array's device address (cudaGetSymbolAddress, with that device
 *    current) and caches it; make that first call before any stream capture.
 *  - Every call on a device uses the same array, which keeps the last call's contents.
 *    Nothing in it needs to start at zero, because each call writes every row it reads,
 *    provided the list is complete: it must hold every expert that occurs in the routed
 *    ids (the rows of an expert missing from it would be read as left by an earlier call,
 *    possibly of another model), and exactly one entry -1 when has_shared is set (none
 *    otherwise; checked, FT_ERR_INVALID).  Calls whose kernels overlap on the GPU (other
 *    streams, other threads) race on the array: order them on one stream. */
FT_API int ft_expert_ffn_decode_noalloc(const void* x, int T, int H, int I, int top_k, int wdtype,
                                        const void* const* blobs, const int* experts, int n_list,
                                        int max_pairs_per_expert, const int* offsets, const int* perm,
                                        const float* gates, const int* inv, int has_shared, void* out,
                                        void* stream);

/* Version string of the library build. */
FT_API const char* ft_version(void);

#ifdef __cplusplus
}
#endif
#endif /* FTMOE_H */

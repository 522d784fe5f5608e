/*
 * Seeded synthetic inputs for the routed-MoE layer over a shared LRU expert
 * cache.  This file holds no arithmetic of the method itself: it only draws
 * numbers and writes them in the runtime expert-blob format.  Both the CPU
 * oracle and the CUDA path read what it writes.
 *
 * Generator: Philox-4x32-10 (Salmon, Moraes, Dror, Shaw, "Parallel random
 * numbers: as easy as 1, 2, 3", SC'11), keyed per tensor by splitmix64
 * (Steele, Lea, Flood, "Fast splittable pseudorandom number generators",
 * OOPSLA'14).  Normals by inversion of a 65536-cell quantile table with linear
 * interpolation inside each cell (normal_from_u32).  Value i of a tensor uses
 * counter i/4 and output lane i%4, so any slice of any tensor can be drawn on
 * its own, and host threads can fill the pool in parallel.
 *
 * Runtime expert blob (one expert, `wdtype` fixed per stack):
 *   f32 / bf16 : W_gate [I][H], W_up [I][H], W_down [H][I], row-major.
 *   int4 g128  : Q_gate [I][H/2], Q_up [I][H/2], Q_down [H][I/2] (bytes; byte b
 *                of a row holds element 2b in its low nibble and 2b+1 in its
 *                high nibble, two's complement in [-8,7]), then the bf16 scales
 *                S_gate [I][H/128], S_up [I][H/128], S_down [H][I/128], one per
 *                128 consecutive reduction-axis elements of a row.
 *   The int4 quantiser (data preparation, run once): s = bf16_rne(max|w|/7),
 *   q = 0 if s == 0 else clamp(rint(w/s), -8, 7) with ties to even.
 *   nvfp4      : Q_gate [I][H/2], Q_up [I][H/2], Q_down [H][I/2] (e2m1 nibbles, element
 *                2b in the low nibble of byte b), then e4m3 block scales S_gate [I][H/16],
 *                S_up [I][H/16], S_down [H][I/16] (one byte per 16 consecutive reduction-
 *                axis elements), then the fp32 global scales g_gate, g_up, g_down and 4
 *                zero bytes.  w = e2m1(q) * e4m3(s) * g.
 *   The nvfp4 quantiser: g = max|W| / (448 * 6) (1 if W is zero); per block of 16,
 *   s = e4m3_rne(max|w| / 6 / g); q = e2m1_rne(w / (s * g)) (0 if s = 0), both with
 *   ties to even and saturation (448, 6).
 */
#define _GNU_SOURCE
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef __AVX2__
#include <immintrin.h>
#endif

#define SYNTH_API __attribute__((visibility("default")))

enum { SYN_W_F32 = 0, SYN_W_BF16 = 1, SYN_W_INT4 = 2, SYN_W_NVFP4 = 3 };
enum {
  SYN_T_WGATE = 1, SYN_T_WUP = 2, SYN_T_WDOWN = 3, SYN_T_ROUTER = 4,
  SYN_T_SH_GATE = 5, SYN_T_SH_UP = 6, SYN_T_SH_DOWN = 7,
  SYN_T_TOKENS = 8, SYN_T_AR1 = 9
};

static inline uint64_t splitmix64(uint64_t z) {
  z += 0x9E3779B97F4A7C15ull;
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}

static inline void philox4x32_10(uint32_t c[4], uint32_t k0, uint32_t k1) {
  for (int r = 0; r < 10; ++r) {
    uint64_t p0 = (uint64_t)0xD2511F53u * c[0];
    uint64_t p1 = (uint64_t)0xCD9E8D57u * c[2];
    uint32_t hi0 = (uint32_t)(p0 >> 32), lo0 = (uint32_t)p0;
    uint32_t hi1 = (uint32_t)(p1 >> 32), lo1 = (uint32_t)p1;
    uint32_t n0 = hi1 ^ c[1] ^ k0, n2 = hi0 ^ c[3] ^ k1;
    c[0] = n0; c[1] = lo1; c[2] = n2; c[3] = lo0;
    k0 += 0x9E3779B9u; k1 += 0xBB67AE85u;
  }
}

static inline uint64_t tensor_key(uint64_t seed, int tensor, int layer, int expert) {
  uint64_t h = splitmix64(seed);
  h = splitmix64(h ^ (uint64_t)(uint32_t)tensor);
  h = splitmix64(h ^ ((uint64_t)(uint32_t)layer << 20));
  h = splitmix64(h ^ ((uint64_t)(uint32_t)expert << 40));
  return h;
}

/* Normal quantile table: Q[i] = Phi^{-1}((i + 0.5) / 65536), i = 0..65535, found by
 * bisection on Phi(z) = erfc(-z/sqrt(2))/2 in double precision. */
static float g_q[65536];
static pthread_once_t g_q_once = PTHREAD_ONCE_INIT;
static void init_quantiles(void) {
  for (int i = 0; i < 65536; ++i) {
    double p = (i + 0.5) / 65536.0, lo = -12.0, hi = 12.0;
    for (int it = 0; it < 80; ++it) {
      double mid = 0.5 * (lo + hi);
      if (0.5 * erfc(-mid / 1.4142135623730951) < p) lo = mid; else hi = mid;
    }
    g_q[i] = (float)(0.5 * (lo + hi));
  }
}

/* One standard normal from 32 random bits, by inversion: the top 16 bits pick a
 * cell of equal probability, the low 16 bits interpolate linearly between the
 * cell's quantile and its neighbour's.  Tails end at |z| = 4.42. */
static inline float normal_from_u32(uint32_t w) {
  int i = (int)(w >> 16);
  float f = ((float)(w & 0xFFFFu) + 0.5f) * (1.0f / 65536.0f) - 0.5f;
  int j = f >= 0.0f ? (i < 65535 ? i + 1 : i) : (i > 0 ? i - 1 : i);
  return g_q[i] + fabsf(f) * (g_q[j] - g_q[i]);
}

/* the four normals of counter block `blk` */
static inline void normal_block(uint64_t key, uint64_t blk, float out[4]) {
  uint32_t c[4] = {(uint32_t)blk, (uint32_t)(blk >> 32), 0u, 0u};
  philox4x32_10(c, (uint32_t)key, (uint32_t)(key >> 32));
  for (int l = 0; l < 4; ++l) out[l] = normal_from_u32(c[l]);
}

/* Philox over 16 consecutive counter blocks at once (lanes independent, so the
 * compiler can vectorise the rounds); out[4*b + l] = normal of lane l, block blk0+b. */
static inline void normal_blocks16(uint64_t key, uint64_t blk0, float out[64]) {
  uint32_t c0[16], c1[16], c2[16], c3[16];
  uint32_t k0 = (uint32_t)key, k1 = (uint32_t)(key >> 32);
  for (int b = 0; b < 16; ++b) {
    uint64_t blk = blk0 + (uint64_t)b;
    c0[b] = (uint32_t)blk; c1[b] = (uint32_t)(blk >> 32); c2[b] = 0u; c3[b] = 0u;
  }
#ifdef __AVX2__
  /* 8 lanes per vector: _mm256_mul_epu32 gives the full 64-bit products of the even
   * 32-bit lanes, so odd lanes are shifted down and multiplied separately. */
  for (int h = 0; h < 16; h += 8) {
    __m256i a0 = _mm256_loadu_si256((const __m256i*)(c0 + h)), a1 = _mm256_loadu_si256((const __m256i*)(c1 + h));
    __m256i a2 = _mm256_loadu_si256((const __m256i*)(c2 + h)), a3 = _mm256_loadu_si256((const __m256i*)(c3 + h));
    const __m256i m0 = _mm256_set1_epi32((int)0xD2511F53u), m1 = _mm256_set1_epi32((int)0xCD9E8D57u);
    const __m256i lo32 = _mm256_set1_epi64x(0xFFFFFFFFll);
    uint32_t kk0 = k0, kk1 = k1;
    for (int r = 0; r < 10; ++r) {
      __m256i pe0 = _mm256_mul_epu32(a0, m0), po0 = _mm256_mul_epu32(_mm256_srli_epi64(a0, 32), m0);
      __m256i pe1 = _mm256_mul_epu32(a2, m1), po1 = _mm256_mul_epu32(_mm256_srli_epi64(a2, 32), m1);
      __m256i hi0 = _mm256_or_si256(_mm256_srli_epi64(pe0, 32), _mm256_andnot_si256(lo32, po0));
      __m256i lo0 = _mm256_or_si256(_mm256_and_si256(pe0, lo32), _mm256_slli_epi64(po0, 32));
      __m256i hi1 = _mm256_or_si256(_mm256_srli_epi64(pe1, 32), _mm256_andnot_si256(lo32, po1));
      __m256i lo1 = _mm256_or_si256(_mm256_and_si256(pe1, lo32), _mm256_slli_epi64(po1, 32));
      __m256i n0 = _mm256_xor_si256(_mm256_xor_si256(hi1, a1), _mm256_set1_epi32((int)kk0));
      __m256i n2 = _mm256_xor_si256(_mm256_xor_si256(hi0, a3), _mm256_set1_epi32((int)kk1));
      a0 = n0; a1 = lo1; a2 = n2; a3 = lo0;
      kk0 += 0x9E3779B9u; kk1 += 0xBB67AE85u;
    }
    _mm256_storeu_si256((__m256i*)(c0 + h), a0); _mm256_storeu_si256((__m256i*)(c1 + h), a1);
    _mm256_storeu_si256((__m256i*)(c2 + h), a2); _mm256_storeu_si256((__m256i*)(c3 + h), a3);
  }
#else
  for (int r = 0; r < 10; ++r) {
    for (int b = 0; b < 16; ++b) {
      uint64_t p0 = (uint64_t)0xD2511F53u * c0[b];
      uint64_t p1 = (uint64_t)0xCD9E8D57u * c2[b];
      uint32_t n0 = (uint32_t)(p1 >> 32) ^ c1[b] ^ k0, n2 = (uint32_t)(p0 >> 32) ^ c3[b] ^ k1;
      c1[b] = (uint32_t)p1; c3[b] = (uint32_t)p0; c0[b] = n0; c2[b] = n2;
    }
    k0 += 0x9E3779B9u; k1 += 0xBB67AE85u;
  }
#endif
  for (int b = 0; b < 16; ++b) {
    out[4 * b + 0] = normal_from_u32(c0[b]);
    out[4 * b + 1] = normal_from_u32(c1[b]);
    out[4 * b + 2] = normal_from_u32(c2[b]);
    out[4 * b + 3] = normal_from_u32(c3[b]);
  }
}

/* dst[i] = sigma * N_i for i in [offset, offset+n) of tensor (seed,tensor,layer,expert) */
SYNTH_API void synth_normal_f32(uint64_t seed, int tensor, int layer, int expert,
                                uint64_t offset, uint64_t n, float sigma, float* dst) {
  pthread_once(&g_q_once, init_quantiles);
  uint64_t key = tensor_key(seed, tensor, layer, expert);
  uint64_t i = offset, end = offset + n;
  float blk[64];
  while (i < end) {
    uint64_t b0 = i >> 6 << 4;            /* 16 blocks = 64 values, aligned */
    normal_blocks16(key, b0, blk);
    uint64_t base = b0 << 2;
    for (uint64_t v = i - base; v < 64 && i < end; ++v, ++i) dst[i - offset] = sigma * blk[v];
  }
}

/* The bare Philox-4x32-10 bijection: out = Philox(ctr, key).  Exported so that the
 * published known-answer vectors can be checked against the generator's own rounds. */
SYNTH_API void synth_philox4x32_10(const uint32_t* ctr, const uint32_t* key, uint32_t* out) {
  uint32_t c[4] = {ctr[0], ctr[1], ctr[2], ctr[3]};
  philox4x32_10(c, key[0], key[1]);
  memcpy(out, c, sizeof c);
}

/* synth_normal_f32 computed one counter block at a time through the scalar rounds:
 * a check of the 16-block (vectorised) path, which must give the same bits. */
SYNTH_API void synth_normal_f32_scalar(uint64_t seed, int tensor, int layer, int expert,
                                       uint64_t offset, uint64_t n, float sigma, float* dst) {
  pthread_once(&g_q_once, init_quantiles);
  uint64_t key = tensor_key(seed, tensor, layer, expert);
  for (uint64_t i = offset; i < offset + n; ++i) {
    float blk[4];
    normal_block(key, i >> 2, blk);
    dst[i - offset] = sigma * blk[i & 3];
  }
}

static inline uint16_t bf16_rne(float f) {
  uint32_t u;
  memcpy(&u, &f, 4);
  u += 0x7FFFu + ((u >> 16) & 1u);
  return (uint16_t)(u >> 16);
}
static inline float bf16_to_f32(uint16_t b) {
  uint32_t u = (uint32_t)b << 16;
  float f;
  memcpy(&f, &u, 4);
  return f;
}

SYNTH_API void synth_round_bf16(const float* src, uint64_t n, uint16_t* dst) {
  for (uint64_t i = 0; i < n; ++i) dst[i] = bf16_rne(src[i]);
}

/* int4 g128 quantiser over `rows` rows of length K (K % 128 == 0). */
SYNTH_API void synth_quantise_int4(const float* w, int rows, int K, uint8_t* q, uint16_t* scales) {
  int groups = K / 128;
  for (int r = 0; r < rows; ++r) {
    const float* wr = w + (size_t)r * K;
    uint8_t* qr = q + (size_t)r * (K / 2);
    for (int g = 0; g < groups; ++g) {
      float amax = 0.0f;
      for (int j = 0; j < 128; ++j) { float a = fabsf(wr[g * 128 + j]); if (a > amax) amax = a; }
      uint16_t sb = bf16_rne(amax / 7.0f);
      scales[(size_t)r * groups + g] = sb;
      float s = bf16_to_f32(sb);
      int8_t qq[128];
      if (s != 0.0f) {
        for (int j = 0; j < 128; ++j) {
          float t = nearbyintf(wr[g * 128 + j] / s);
          t = t < -8.0f ? -8.0f : (t > 7.0f ? 7.0f : t);
          qq[j] = (int8_t)t;
        }
      } else {
        memset(qq, 0, sizeof(qq));
      }
      for (int j = 0; j < 128; j += 2)
        qr[(g * 128 + j) / 2] = (uint8_t)((qq[j] & 0xF) | ((qq[j + 1] & 0xF) << 4));
    }
  }
}

/* e2m1 (FP4) code of a real value: nearest of {0,.5,1,1.5,2,3,4,6} (ties to the even
 * mantissa), saturating at 6; bit 3 is the sign. */
static uint8_t e2m1_rne(float v) {
  static const float mag[8] = {0.f, 0.5f, 1.f, 1.5f, 2.f, 3.f, 4.f, 6.f};
  uint8_t sgn = v < 0.f ? 8 : 0;
  float a = fabsf(v);
  int best = 0;
  for (int c = 1; c < 8; ++c) {
    float d = fabsf(a - mag[c]), db = fabsf(a - mag[best]);
    if (d < db || (d == db && (c & 1) == 0)) best = c;
  }
  return (uint8_t)(sgn | best);
}

/* e4m3 (FP8, bias 7, no infinities, max 448) code of a non-negative value, round to
 * nearest even, saturating at 448. */
static uint8_t e4m3_rne(float v) {
  if (!(v > 0.f)) return 0;
  if (v >= 448.f) return 0x7E;
  int best = 0;
  float bestd = v;
  for (int c = 1; c <= 0x7E; ++c) {
    int e = c >> 3, m = c & 7;
    float val = e == 0 ? ldexpf((float)m, -9) : ldexpf(1.f + m / 8.f, e - 7);
    float d = fabsf(v - val);
    if (d < bestd || (d == bestd && (c & 1) == 0)) { best = c; bestd = d; }
  }
  return (uint8_t)best;
}

static float e4m3_value(uint8_t c) {
  int e = (c >> 3) & 15, m = c & 7;
  return e == 0 ? ldexpf((float)m, -9) : ldexpf(1.f + m / 8.f, e - 7);
}

/* nvfp4 quantiser for one matrix [rows][K] (K % 16 == 0) given its global scale g. */
SYNTH_API void synth_quantise_nvfp4_rows(const float* w, int rows, int K, float g, uint8_t* q, uint8_t* scales) {
  const float e2m1_mag[8] = {0.f, 0.5f, 1.f, 1.5f, 2.f, 3.f, 4.f, 6.f};
  (void)e2m1_mag;
  for (int r = 0; r < rows; ++r) {
    const float* wr = w + (size_t)r * K;
    for (int b = 0; b < K / 16; ++b) {
      float amax = 0.f;
      for (int j = 0; j < 16; ++j) { float a = fabsf(wr[b * 16 + j]); if (a > amax) amax = a; }
      uint8_t sc = e4m3_rne(amax / 6.0f / g);
      scales[(size_t)r * (K / 16) + b] = sc;
      float s = e4m3_value(sc) * g;
      for (int j = 0; j < 16; j += 2) {
        uint8_t c0 = s > 0.f ? e2m1_rne(wr[b * 16 + j] / s) : 0;
        uint8_t c1 = s > 0.f ? e2m1_rne(wr[b * 16 + j + 1] / s) : 0;
        q[(size_t)r * (K / 2) + (b * 16 + j) / 2] = (uint8_t)(c0 | (c1 << 4));
      }
    }
  }
}

/* One matrix [rows][cols] of tensor id `tensor` in the blob's element format. */
static void write_matrix(uint64_t seed, int tensor, int layer, int expert, int rows, int cols,
                         int wdtype, float sigma, uint8_t* dst_w, uint16_t* dst_s, float* scratch) {
  if (wdtype == SYN_W_F32) {
    synth_normal_f32(seed, tensor, layer, expert, 0, (uint64_t)rows * cols, sigma, (float*)dst_w);
  } else if (wdtype == SYN_W_BF16) {
    uint16_t* o = (uint16_t*)dst_w;
    for (int r = 0; r < rows; ++r) {
      synth_normal_f32(seed, tensor, layer, expert, (uint64_t)r * cols, cols, sigma, scratch);
      for (int c = 0; c < cols; ++c) o[(size_t)r * cols + c] = bf16_rne(scratch[c]);
    }
  } else {
    for (int r = 0; r < rows; ++r) {
      synth_normal_f32(seed, tensor, layer, expert, (uint64_t)r * cols, cols, sigma, scratch);
      synth_quantise_int4(scratch, 1, cols, dst_w + (size_t)r * (cols / 2), dst_s + (size_t)r * (cols / 128));
    }
  }
}

SYNTH_API uint64_t synth_blob_bytes(int H, int I, int wdtype) {
  uint64_t n = 3ull * H * I;
  if (wdtype == SYN_W_F32) return n * 4;
  if (wdtype == SYN_W_BF16) return n * 2;
  if (wdtype == SYN_W_NVFP4) return n / 2 + n / 16 + 16;
  return n / 2 + (n / 128) * 2;
}

/* nvfp4 matrix: two passes over the draws (the global scale needs the matrix maximum). */
static void write_matrix_nvfp4(uint64_t seed, int tensor, int layer, int expert, int rows, int cols, float sigma,
                               uint8_t* q, uint8_t* sc, float* g_out, float* scratch) {
  float amax = 0.f;
  for (int r = 0; r < rows; ++r) {
    synth_normal_f32(seed, tensor, layer, expert, (uint64_t)r * cols, cols, sigma, scratch);
    for (int c = 0; c < cols; ++c) { float a = fabsf(scratch[c]); if (a > amax) amax = a; }
  }
  float g = amax > 0.f ? amax / (448.0f * 6.0f) : 1.0f;
  *g_out = g;
  for (int r = 0; r < rows; ++r) {
    synth_normal_f32(seed, tensor, layer, expert, (uint64_t)r * cols, cols, sigma, scratch);
    synth_quantise_nvfp4_rows(scratch, 1, cols, g, q + (size_t)r * (cols / 2), sc + (size_t)r * (cols / 16));
  }
}

/* Writes one expert blob.  shared != 0 selects the always-on shared expert of `layer`. */
SYNTH_API int synth_expert_blob(uint64_t seed, int layer, int expert, int shared, int H, int I,
                                int wdtype, float sigma, uint8_t* dst) {
  int tg = shared ? SYN_T_SH_GATE : SYN_T_WGATE, tu = shared ? SYN_T_SH_UP : SYN_T_WUP,
      td = shared ? SYN_T_SH_DOWN : SYN_T_WDOWN;
  int ex = shared ? 0 : expert;
  if (wdtype == SYN_W_INT4 && ((H % 128) || (I % 128))) return -1;
  if (wdtype == SYN_W_NVFP4 && ((H % 32) || (I % 32))) return -1;
  float* scratch = (float*)malloc(sizeof(float) * (size_t)(H > I ? H : I));
  if (!scratch) return -2;
  uint64_t mat = (uint64_t)H * I;
  if (wdtype == SYN_W_NVFP4) {
    uint8_t* q = dst;
    uint8_t* sc = dst + 3 * mat / 2;
    float g[4] = {0.f, 0.f, 0.f, 0.f};
    write_matrix_nvfp4(seed, tg, layer, ex, I, H, sigma, q, sc, &g[0], scratch);
    write_matrix_nvfp4(seed, tu, layer, ex, I, H, sigma, q + mat / 2, sc + mat / 16, &g[1], scratch);
    write_matrix_nvfp4(seed, td, layer, ex, H, I, sigma, q + mat, sc + 2 * (mat / 16), &g[2], scratch);
    memcpy(dst + 3 * mat / 2 + 3 * mat / 16, g, 16);
    free(scratch);
    return 0;
  }
  if (wdtype == SYN_W_INT4) {
    uint8_t* q = dst;
    uint16_t* s = (uint16_t*)(dst + 3 * mat / 2);
    write_matrix(seed, tg, layer, ex, I, H, wdtype, sigma, q, s, scratch);
    write_matrix(seed, tu, layer, ex, I, H, wdtype, sigma, q + mat / 2, s + mat / 128, scratch);
    write_matrix(seed, td, layer, ex, H, I, wdtype, sigma, q + mat, s + 2 * (mat / 128), scratch);
  } else {
    size_t es = wdtype == SYN_W_F32 ? 4 : 2;
    write_matrix(seed, tg, layer, ex, I, H, wdtype, sigma, dst, NULL, scratch);
    write_matrix(seed, tu, layer, ex, I, H, wdtype, sigma, dst + mat * es, NULL, scratch);
    write_matrix(seed, td, layer, ex, H, I, wdtype, sigma, dst + 2 * mat * es, NULL, scratch);
  }
  free(scratch);
  return 0;
}

typedef struct {
  uint64_t seed; int L, E, H, I, wdtype; float sigma;
  uint8_t* base; uint64_t stride;   /* blob (l,e) at base + (l*E+e)*stride */
  int next; pthread_mutex_t mu; int err;
} pool_job;

static void* pool_worker(void* arg) {
  pool_job* j = (pool_job*)arg;
  for (;;) {
    pthread_mutex_lock(&j->mu);
    int id = j->next++;
    pthread_mutex_unlock(&j->mu);
    if (id >= j->L * j->E) break;
    int l = id / j->E, e = id % j->E;
    int rc = synth_expert_blob(j->seed, l, e, 0, j->H, j->I, j->wdtype, j->sigma,
                               j->base + (uint64_t)id * j->stride);
    if (rc) j->err = rc;
  }
  return NULL;
}

/* Fills all L*E routed-expert blobs with `nthreads` host threads. */
SYNTH_API int synth_fill_pool(uint64_t seed, int L, int E, int H, int I, int wdtype, float sigma,
                              uint8_t* base, uint64_t stride, int nthreads) {
  pool_job j = {seed, L, E, H, I, wdtype, sigma, base, stride, 0, PTHREAD_MUTEX_INITIALIZER, 0};
  if (nthreads < 1) nthreads = 1;
  if (nthreads > 256) nthreads = 256;
  pthread_t th[256];
  for (int t = 0; t < nthreads; ++t) pthread_create(&th[t], NULL, pool_worker, &j);
  for (int t = 0; t < nthreads; ++t) pthread_join(th[t], NULL);
  return j.err;
}

/* AR(1) chain: x_0 = eps_0, x_t = phi*x_{t-1} + sig*eps_t, eps ~ N(0, I_H) from tensor SYN_T_AR1
 * with layer = chain.  Writes T rows of H fp32 values. */
SYNTH_API void synth_ar1(uint64_t seed, int chain, int T, int H, float phi, float sig, float* dst) {
  float* eps = (float*)malloc(sizeof(float) * (size_t)H);
  for (int t = 0; t < T; ++t) {
    synth_normal_f32(seed, SYN_T_AR1, chain, 0, (uint64_t)t * H, H, 1.0f, eps);
    float* row = dst + (size_t)t * H;
    if (t == 0) memcpy(row, eps, sizeof(float) * (size_t)H);
    else for (int h = 0; h < H; ++h) row[h] = phi * dst[(size_t)(t - 1) * H + h] + sig * eps[h];
  }
  free(eps);
}

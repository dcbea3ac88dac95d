/*
 * Seeded synthetic inputs for the sparse MoE FFN layer.
 *
 * This file is the single source of input bits for both the CPU oracle and
 * the CUDA path: it holds no step of the layer's arithmetic (no router, no
 * selection, no expert projection, no quantisation), only random draws.
 *
 * Generator (counter based, so any element can be drawn independently and in
 * parallel):
 *   key    = splitmix64(seed ^ (tag << 56))         one well-mixed key per (seed, tensor)
 *   u64    = splitmix64(key ^ (idx >> 1))           one draw per index pair
 *   u1, u2 = ((u64 >> 32) + 0.5) / 2^32, ((u64 & 0xffffffff) + 0.5) / 2^32
 *   z      = sqrt(-2 ln u1) * (idx even ? cos(2 pi u2) : sin(2 pi u2))
 *   value  = bf16_rne((float)(z * sigma))   or the fp32 value for fp32 tensors
 * splitmix64 is Steele, Lea & Flood's SplitMix64 finaliser (OOPSLA 2014), and
 * the normal draw is the Box-Muller transform (Box & Muller 1958).
 *
 * idx is always the element's index in the LOGICAL tensor as the layer is
 * stated (x[T,H], Wr[H,E], Wg/Wu[E,H,I], Wd[E,I,H]), whatever layout the
 * caller stores it in, so a transposed store draws the same values.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

static inline uint64_t splitmix64(uint64_t z) {
  z += 0x9E3779B97F4A7C15ULL;
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ULL;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBULL;
  return z ^ (z >> 31);
}

static inline uint64_t gen_key(uint64_t seed, uint32_t tag) {
  return splitmix64(seed ^ ((uint64_t)tag << 56));
}

static inline float normal_at(uint64_t key, uint64_t idx) {
  uint64_t u = splitmix64(key ^ (idx >> 1));
  float u1 = ((float)(uint32_t)(u >> 32) + 0.5f) * 2.3283064365386963e-10f;
  float u2 = ((float)(uint32_t)(u & 0xffffffffu) + 0.5f) * 2.3283064365386963e-10f;
  /* (float)(2^32 - 1) + 0.5 rounds to 2^32, giving u == 1.0; clamp below 1. */
  if (u1 >= 1.0f) u1 = 0.99999994f;
  float r = sqrtf(-2.0f * logf(u1));
  float th = 6.2831853071795865f * u2;
  return (idx & 1) ? r * sinf(th) : r * cosf(th);
}

/* float -> bf16 bits, round to nearest even (inputs are finite). */
static inline uint16_t f32_to_bf16_rne(float f) {
  uint32_t b;
  memcpy(&b, &f, 4);
  uint32_t lsb = (b >> 16) & 1u;
  b += 0x7FFFu + lsb;
  return (uint16_t)(b >> 16);
}

/* ------------------------------------------------------------------------ */
/* Threaded 3-D draw: logical tensor [nb][R][C], stored as                    */
/*   transpose == 0:  out[b*bstride + r*C + c]                                */
/*   transpose == 1:  out[b*bstride + c*R + r]                                */
/* ------------------------------------------------------------------------ */
typedef struct {
  uint64_t key;
  float sigma;
  int64_t nb, R, C, bstride;
  int transpose, as_f32;
  void* out;
  int64_t lo, hi; /* range of (b, outer) rows this worker fills */
} job_t;

static void* worker(void* arg) {
  job_t* j = (job_t*)arg;
  int64_t outer = j->transpose ? j->C : j->R;
  int64_t inner = j->transpose ? j->R : j->C;
  for (int64_t row = j->lo; row < j->hi; ++row) {
    int64_t b = row / outer, o = row % outer;
    int64_t base = b * j->bstride + o * inner;
    for (int64_t in = 0; in < inner; ++in) {
      int64_t r = j->transpose ? in : o;
      int64_t c = j->transpose ? o : in;
      uint64_t idx = (uint64_t)((b * j->R + r) * j->C + c);
      float v = normal_at(j->key, idx) * j->sigma;
      if (j->as_f32)
        ((float*)j->out)[base + in] = v;
      else
        ((uint16_t*)j->out)[base + in] = f32_to_bf16_rne(v);
    }
  }
  return NULL;
}

static void run_jobs(job_t proto, int nthreads) {
  int64_t outer = proto.transpose ? proto.C : proto.R;
  int64_t rows = proto.nb * outer;
  if (nthreads < 1) nthreads = 1;
  if (nthreads > 256) nthreads = 256;
  if ((int64_t)nthreads > rows) nthreads = (int)(rows > 0 ? rows : 1);
  pthread_t th[256];
  job_t jobs[256];
  for (int t = 0; t < nthreads; ++t) {
    jobs[t] = proto;
    jobs[t].lo = rows * t / nthreads;
    jobs[t].hi = rows * (t + 1) / nthreads;
    pthread_create(&th[t], NULL, worker, &jobs[t]);
  }
  for (int t = 0; t < nthreads; ++t) pthread_join(th[t], NULL);
}

/* bf16 normal tensor; see the layout rule above. */
void gen_normal_bf16(uint64_t seed, uint32_t tag, float sigma, int64_t nb, int64_t R,
                     int64_t C, int transpose, int64_t bstride, uint16_t* out, int nthreads) {
  job_t p = {gen_key(seed, tag), sigma, nb, R, C, bstride, transpose, 0, out, 0, 0};
  run_jobs(p, nthreads);
}

/* fp32 normal tensor (no bf16 rounding), same index rule. */
void gen_normal_f32(uint64_t seed, uint32_t tag, float sigma, int64_t nb, int64_t R, int64_t C,
                    int transpose, int64_t bstride, float* out, int nthreads) {
  job_t p = {gen_key(seed, tag), sigma, nb, R, C, bstride, transpose, 1, out, 0, 0};
  run_jobs(p, nthreads);
}

/* Seeded Fisher-Yates permutation of 0..n-1 (Durstenfeld's in-place form):
 * for i = n-1 .. 1, swap perm[i] with perm[j], j = splitmix64(key ^ i) mod (i+1). */
void gen_permutation(uint64_t seed, uint32_t tag, int64_t n, int32_t* perm) {
  uint64_t key = gen_key(seed, tag);
  for (int64_t i = 0; i < n; ++i) perm[i] = (int32_t)i;
  for (int64_t i = n - 1; i > 0; --i) {
    int64_t j = (int64_t)(splitmix64(key ^ (uint64_t)i) % (uint64_t)(i + 1));
    int32_t t = perm[i];
    perm[i] = perm[j];
    perm[j] = t;
  }
}

/* The SplitMix64 finaliser itself, exposed so tests can pin it. */
uint64_t gen_splitmix64(uint64_t z) { return splitmix64(z); }

/* Raw 64-bit draws of one stream. */
void gen_raw_u64(uint64_t seed, uint32_t tag, int64_t n, uint64_t* out) {
  uint64_t key = gen_key(seed, tag);
  for (int64_t i = 0; i < n; ++i) out[i] = splitmix64(key ^ (uint64_t)i);
}

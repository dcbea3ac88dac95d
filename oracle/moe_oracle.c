/*
 * CPU oracle for the sparse MoE FFN layer forward.
 *
 * TEST INFRASTRUCTURE. Only tests/, __graft_entry__.smoke() and bench.py's
 * cpu_baseline leg may load, call or execute anything under oracle/. The
 * product path never does; it shares no code, header, table or helper with
 * this file.
 *
 * Plain, slow, obviously correct: every step is the definition written out,
 * in the order the pages state it. Threads only split independent outputs;
 * no summation is blocked, split or reordered.
 *
 * Precision (and why):
 *   - router logits: fp32, one accumulator per (token, expert), h ascending.
 *     The logits decide an integer (the top-k ids), so they are taken in the
 *     precision of the kernel that must match them. A bf16 x bf16 product is
 *     exact in fp32 (8 + 8 significand bits), so this is a fully specified
 *     function of the inputs.
 *   - routing weights: fp64 exp / sum, rounded once to fp32.
 *   - expert projections, SwiGLU and the weighted combine: fp64 accumulation,
 *     each output rounded once to fp32 at the end.
 *   - FP8: e4m3 codes and their fp32 scales are decided in fp32 (the kernel's
 *     precision); dequantised values are exact in fp64.
 *
 * Parity pins: every function here is checked in tests/ against something
 * other than itself (fp64 error bounds, brute force, library special cases,
 * closed forms, exhaustive codec tables).
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* ------------------------------------------------------------------------ */
/* small helpers                                                             */
/* ------------------------------------------------------------------------ */
static inline float bf16_widen(uint16_t b) {
  uint32_t u = (uint32_t)b << 16;
  float f;
  memcpy(&f, &u, 4);
  return f;
}

typedef void (*range_fn)(void* ctx, int64_t lo, int64_t hi);
typedef struct {
  range_fn fn;
  void* ctx;
  int64_t lo, hi;
} span_t;

static void* span_main(void* a) {
  span_t* s = (span_t*)a;
  s->fn(s->ctx, s->lo, s->hi);
  return NULL;
}

/* Split [0, n) into nthreads contiguous spans. */
static void parallel_for(int64_t n, int nthreads, range_fn fn, void* ctx) {
  if (nthreads < 1) nthreads = 1;
  if (nthreads > 256) nthreads = 256;
  if (n < nthreads) nthreads = (int)(n > 0 ? n : 1);
  pthread_t th[256];
  span_t sp[256];
  for (int t = 0; t < nthreads; ++t) {
    sp[t].fn = fn;
    sp[t].ctx = ctx;
    sp[t].lo = n * t / nthreads;
    sp[t].hi = n * (t + 1) / nthreads;
    pthread_create(&th[t], NULL, span_main, &sp[t]);
  }
  for (int t = 0; t < nthreads; ++t) pthread_join(th[t], NULL);
}

/* ------------------------------------------------------------------------ */
/* Router logits.                                                            */
/* "Mixture of Experts (MoE): a practical explanation" (lira-now.com), §5    */
/* "How the Router (Top-k Routing) works step by step", steps 1-2 and the    */
/* pseudocode's `logits = router(x)`: a linear layer from the token vector   */
/* to E scores. The bias (when the layer has one) is added to the score.     */
/*   logits[t, e] = (sum_h x[t, h] * Wr[h, e]) + bias[e]                      */
/* The logits decide integers (the selected experts), so the fp32 order of  */
/* the sum is fixed (the page states none): the h range is cut into         */
/* ROUTER_BLOCKS = 8 contiguous blocks, block b = [b*H/8, (b+1)*H/8) with   */
/* the bounds rounded down (H/8 each when 8 divides H); each block sum      */
/* starts at 0                                                               */
/* and adds its products h ascending, one fp32 add of the exact bf16 x bf16 */
/* product per term; the block sums are then added left to right:           */
/*   s = p_0;  s = s + p_1;  ...;  s = s + p_7;  logit = s + bias[e]        */
/* ------------------------------------------------------------------------ */
enum { ROUTER_BLOCKS = 8 };
typedef struct {
  const uint16_t *x, *wr;
  const float* bias;
  const int32_t* tokens;
  int64_t H, E;
  float* logits;
} logits_ctx;

static void logits_rows(void* p, int64_t lo, int64_t hi) {
  logits_ctx* c = (logits_ctx*)p;
  enum { EB = 16 }; /* experts computed side by side; each keeps its own h-ascending sum */
  for (int64_t r = lo; r < hi; ++r) {
    int64_t t = c->tokens ? c->tokens[r] : r;
    const uint16_t* xr = c->x + t * c->H;
    for (int64_t e0 = 0; e0 < c->E; e0 += EB) {
      int64_t ne = c->E - e0 < EB ? c->E - e0 : EB;
      float acc[EB];
      for (int b = 0; b < ROUTER_BLOCKS; ++b) {
        float part[EB];
        for (int j = 0; j < EB; ++j) part[j] = 0.0f;
        const int64_t h0 = b * c->H / ROUTER_BLOCKS, h1 = (b + 1) * c->H / ROUTER_BLOCKS;
        for (int64_t h = h0; h < h1; ++h) {
          float xv = bf16_widen(xr[h]);
          const uint16_t* wrow = c->wr + h * c->E + e0;
          for (int64_t j = 0; j < ne; ++j) part[j] += xv * bf16_widen(wrow[j]);
        }
        for (int j = 0; j < EB; ++j) acc[j] = b == 0 ? part[j] : acc[j] + part[j];
      }
      for (int64_t j = 0; j < ne; ++j)
        c->logits[r * c->E + e0 + j] = acc[j] + (c->bias ? c->bias[e0 + j] : 0.0f);
    }
  }
}

/* logits for rows tokens[0..nt) (or 0..nt when tokens == NULL) */
void oracle_router_logits(const uint16_t* x, const uint16_t* wr, const float* bias,
                          const int32_t* tokens, int64_t nt, int64_t H, int64_t E, float* logits,
                          int nthreads) {
  logits_ctx c = {x, wr, bias, tokens, H, E, logits};
  parallel_for(nt, nthreads, logits_rows, &c);
}

/* ------------------------------------------------------------------------ */
/* Softmax top-k with renormalised weights.                                  */
/* Same page, §5 steps 3-5 and the pseudocode's `probs = softmax(logits)`,   */
/* `values, indices = topk(probs, k)`, `weights = values / values.sum()`.    */
/* softmax is strictly increasing in the logit, so the k largest probs are   */
/* the k largest logits; ties (equal fp32 logits) go to the lower expert     */
/* index, and slot j holds the j-th largest. The full softmax denominator    */
/* cancels in the renormalisation, leaving                                   */
/*   w_j = exp(l_j - l_max) / sum_{i in selected} exp(l_i - l_max).          */
/* The toy layer's `+ 1e-9` in the denominator is not used: the denominator  */
/* is >= 1 because the top term is exp(0).                                   */
/* ------------------------------------------------------------------------ */
void oracle_topk(const float* logits, int64_t T, int64_t E, int k, int32_t* ids, float* w) {
  char* taken = (char*)malloc((size_t)E);
  double* ex = (double*)malloc(sizeof(double) * (size_t)k);
  for (int64_t t = 0; t < T; ++t) {
    const float* l = logits + t * E;
    memset(taken, 0, (size_t)E);
    for (int j = 0; j < k; ++j) {
      int64_t best = -1;
      for (int64_t e = 0; e < E; ++e) {
        if (taken[e]) continue;
        if (best < 0 || l[e] > l[best]) best = e; /* strict >: lower index wins ties */
      }
      taken[best] = 1;
      ids[t * k + j] = (int32_t)best;
    }
    double lmax = (double)l[ids[t * k]];
    double den = 0.0;
    for (int j = 0; j < k; ++j) {
      ex[j] = exp((double)l[ids[t * k + j]] - lmax);
      den += ex[j];
    }
    for (int j = 0; j < k; ++j) w[t * k + j] = (float)(ex[j] / den);
  }
  free(taken);
  free(ex);
}

/* ------------------------------------------------------------------------ */
/* Permutation by expert.                                                    */
/* "Experts backends" (HF Transformers docs), backend table, `grouped_mm`    */
/* row: the routed tokens are sorted by chosen expert so each expert's rows  */
/* are contiguous for one grouped GEMM. Order is expert-major, then token    */
/* ascending (a token holds each expert at most once), which makes the       */
/* result unique:                                                            */
/*   offsets[0] = 0, offsets[e+1] = offsets[e] + count[e]                    */
/*   row p in [offsets[e], offsets[e+1]) is (token, slot) pairs with expert  */
/*   e, in ascending token order; inv_perm[t*k + j] = p.                     */
/* ------------------------------------------------------------------------ */
void oracle_permute(const int32_t* ids, int64_t T, int64_t E, int k, int32_t* offsets,
                    int32_t* perm_token, int32_t* perm_slot, int32_t* inv_perm) {
  for (int64_t e = 0; e <= E; ++e) offsets[e] = 0;
  for (int64_t i = 0; i < T * k; ++i) offsets[ids[i] + 1] += 1;
  for (int64_t e = 0; e < E; ++e) offsets[e + 1] += offsets[e];
  int64_t p = 0;
  for (int64_t e = 0; e < E; ++e) {
    for (int64_t t = 0; t < T; ++t) {
      for (int j = 0; j < k; ++j) {
        if (ids[t * k + j] == e) {
          perm_token[p] = (int32_t)t;
          perm_slot[p] = j;
          inv_perm[t * k + j] = (int32_t)p;
          ++p;
        }
      }
    }
  }
}

/* ------------------------------------------------------------------------ */
/* Expert FFN: gated MLP, up/gate projection -> SwiGLU -> down projection.    */
/* "Experts backends", `deepgemm_megamoe` row and "SonicMoE" section: the     */
/* expert is a gated MLP (gate and up projections, SwiGLU, down projection). */
/* SiLU goes on the gate projection, the up projection stays linear:         */
/*   g_i = sum_h x_h Wg[e,h,i],  u_i = sum_h x_h Wu[e,h,i]                   */
/*   a_i = act(g_i) * u_i,       act = silu by default:                       */
/*                               silu(z) = z / (1 + exp(-z))                 */
/* The same page lists experts with other gated activations (silu, gelu or   */
/* relu: SwiGLU / GeGLU / ReGLU); act selects one:                           */
/*   ACT_SILU  z / (1 + exp(-z))                                             */
/*   ACT_GELU  z * Phi(z) = z/2 * (1 + erf(z / sqrt 2))   (the erf form, the */
/*             one the toy layer's nn.GELU() denotes by default)             */
/*   ACT_RELU  max(z, 0)                                                     */
/*   y_c = sum_i a_i Wd[e,i,c]                                               */
/* Weights arrive K-major: w13[e] = [Wg[e]^T ; Wu[e]^T] ([2I, H]) and        */
/* w2[e] = Wd[e]^T ([H, I]).                                                 */
/* ------------------------------------------------------------------------ */

enum { ACT_SILU = 1, ACT_GELU = 2, ACT_RELU = 3 };

static double gate_act(double z, int act) {
  if (act == ACT_GELU) return 0.5 * z * (1.0 + erf(z / sqrt(2.0)));
  if (act == ACT_RELU) return z > 0.0 ? z : 0.0;
  return z / (1.0 + exp(-z));
}

/* Up to GROUP rows are evaluated side by side so the fp64 sums vectorise
 * across rows; every (row, output) sum still runs over its index ascending. */
#define GROUP 8

/* a[n, I] (fp64) from fp64 activation rows xT[H][GROUP] (row r in column r) */
static void expert_hidden(const double* xT, int64_t n, const uint16_t* w13e, const double* w13e_d,
                          int64_t H, int64_t I, int act, double* a) {
  for (int64_t i = 0; i < I; ++i) {
    double g[GROUP], u[GROUP];
    for (int r = 0; r < GROUP; ++r) g[r] = u[r] = 0.0;
    for (int64_t h = 0; h < H; ++h) {
      double wg, wu;
      if (w13e_d) {
        wg = w13e_d[i * H + h];
        wu = w13e_d[(I + i) * H + h];
      } else {
        wg = (double)bf16_widen(w13e[i * H + h]);
        wu = (double)bf16_widen(w13e[(I + i) * H + h]);
      }
      const double* xh = xT + h * GROUP;
      for (int r = 0; r < GROUP; ++r) {
        g[r] += xh[r] * wg;
        u[r] += xh[r] * wu;
      }
    }
    for (int64_t r = 0; r < n; ++r) a[r * I + i] = gate_act(g[r], act) * u[r];
  }
}

/* y[n, H] (fp64) from fp64 hidden rows aT[I][GROUP] */
static void expert_out(const double* aT, int64_t n, const uint16_t* w2e, const double* w2e_d,
                       int64_t H, int64_t I, double* y) {
  for (int64_t c = 0; c < H; ++c) {
    double acc[GROUP];
    for (int r = 0; r < GROUP; ++r) acc[r] = 0.0;
    for (int64_t i = 0; i < I; ++i) {
      double wd = w2e_d ? w2e_d[c * I + i] : (double)bf16_widen(w2e[c * I + i]);
      const double* ai = aT + i * GROUP;
      for (int r = 0; r < GROUP; ++r) acc[r] += ai[r] * wd;
    }
    for (int64_t r = 0; r < n; ++r) y[r * H + c] = acc[r];
  }
}

/* transpose rows [n, C] into [C][GROUP], zero-padding missing rows */
static void to_cols(const double* rows, int64_t n, int64_t C, double* T) {
  for (int64_t c = 0; c < C; ++c)
    for (int r = 0; r < GROUP; ++r) T[c * GROUP + r] = r < n ? rows[r * C + c] : 0.0;
}

/* Exposed pieces, used by the tests to pin one GEMM stage at a time.
 * a_rows: [n, H] bf16 rows; out: [n, I] fp32 (each value rounded once). */
void oracle_expert_gated_rows(const uint16_t* a_rows, int64_t n, const uint16_t* w13e, int64_t H,
                              int64_t I, int act, float* out) {
  double* xr = (double*)malloc(sizeof(double) * (size_t)(GROUP * H));
  double* xT = (double*)malloc(sizeof(double) * (size_t)(GROUP * H));
  double* a = (double*)malloc(sizeof(double) * (size_t)(GROUP * I));
  for (int64_t r0 = 0; r0 < n; r0 += GROUP) {
    int64_t m = n - r0 < GROUP ? n - r0 : GROUP;
    for (int64_t i = 0; i < m * H; ++i) xr[i] = (double)bf16_widen(a_rows[r0 * H + i]);
    to_cols(xr, m, H, xT);
    expert_hidden(xT, m, w13e, NULL, H, I, act, a);
    for (int64_t i = 0; i < m * I; ++i) out[r0 * I + i] = (float)a[i];
  }
  free(xr);
  free(xT);
  free(a);
}

/* h_rows: [n, I] bf16 rows; out: [n, H] fp32 */
void oracle_expert_down_rows(const uint16_t* h_rows, int64_t n, const uint16_t* w2e, int64_t H,
                             int64_t I, float* out) {
  double* a = (double*)malloc(sizeof(double) * (size_t)(GROUP * I));
  double* aT = (double*)malloc(sizeof(double) * (size_t)(GROUP * I));
  double* y = (double*)malloc(sizeof(double) * (size_t)(GROUP * H));
  for (int64_t r0 = 0; r0 < n; r0 += GROUP) {
    int64_t m = n - r0 < GROUP ? n - r0 : GROUP;
    for (int64_t i = 0; i < m * I; ++i) a[i] = (double)bf16_widen(h_rows[r0 * I + i]);
    to_cols(a, m, I, aT);
    expert_out(aT, m, w2e, NULL, H, I, y);
    for (int64_t i = 0; i < m * H; ++i) out[r0 * H + i] = (float)y[i];
  }
  free(a);
  free(aT);
  free(y);
}

/* ------------------------------------------------------------------------ */
/* FP8 e4m3 (OCP E4M3FN: 1 sign, 4 exponent bits with bias 7, 3 mantissa    */
/* bits; no infinities; S.1111.111 is NaN; largest finite 448).              */
/* "Fine-grained FP8" (HF Transformers docs), opening list: weights are      */
/* quantised to 8 bits per 128 x 128 block, activations per token per group  */
/* of 128 input channels, dynamically.                                       */
/* ------------------------------------------------------------------------ */
double oracle_e4m3_decode(uint8_t q) {
  int s = q >> 7, ef = (q >> 3) & 15, m = q & 7;
  if (ef == 15 && m == 7) return NAN;
  double v = ef == 0 ? ldexp((double)m, -9) : ldexp(1.0 + m / 8.0, ef - 7);
  return s ? -v : v;
}

/* Round a finite float to the nearest e4m3 code, ties to even, saturating at
 * +-448 (values this layer encodes never exceed 448 * (1 + 2^-23)). */
uint8_t oracle_e4m3_encode(float f) {
  uint8_t s = signbit(f) ? 0x80 : 0;
  double a = fabs((double)f);
  if (a >= 464.0) return s | 0x7E; /* beyond the 448/480 midpoint: saturate */
  if (a < ldexp(1.0, -6)) {      /* subnormal range: multiples of 2^-9 */
    double m = rint(ldexp(a, 9)); /* default mode rounds ties to even */
    return s | (uint8_t)m;       /* m == 8 is the code of 2^-6, as wanted */
  }
  int ex;
  frexp(a, &ex); /* a = f * 2^ex, f in [0.5, 1) -> unbiased exponent ex-1 */
  int e = ex - 1;
  double m = rint((ldexp(a, -e) - 1.0) * 8.0);
  if (m == 8.0) {
    m = 0.0;
    e += 1;
  }
  if (e > 8) return s | 0x7E;
  return s | (uint8_t)(((e + 7) << 3) | (int)m);
}

/* amax / 448 in fp32 with IEEE division; an all-zero group gets scale 1.
 * With power-of-two scales ("Fine-grained FP8" / "Experts backends", UE8M0
 * scale format: scales stored as 8-bit exponents, float8_e8m0fnu), the scale
 * is the smallest power of two >= amax / 448 (that fp32 quotient, so no
 * scaled value exceeds 448), kept within the format's range 2^-127..2^127. */
enum { SCALE_F32 = 0, SCALE_UE8M0 = 1 };

static inline float group_scale(float amax, int fmt) {
  if (!(amax > 0.0f)) return 1.0f;
  const float r = amax / 448.0f;
  if (fmt != SCALE_UE8M0) return r;
  int e;
  const float m = frexpf(r, &e); /* r = m * 2^e, m in [0.5, 1) */
  int p2 = m == 0.5f ? e - 1 : e;  /* r is a power of two: 2^(e-1); else round up */
  if (p2 < -127) p2 = -127;
  if (p2 > 127) p2 = 127;
  return ldexpf(1.0f, p2);
}

/* Per row, per group of 128 consecutive columns: s = amax/448, q = e4m3(v/s).
 * vals: [rows, cols] fp32 (already widened); q: [rows, cols]; s: [rows, cols/128]. */
static void quant_groups_f32(const float* vals, int64_t rows, int64_t cols, uint8_t* q, float* s,
                             int fmt) {
  int64_t G = cols / 128;
  for (int64_t r = 0; r < rows; ++r) {
    for (int64_t g = 0; g < G; ++g) {
      const float* v = vals + r * cols + g * 128;
      float amax = 0.0f;
      for (int c = 0; c < 128; ++c) amax = fmaxf(amax, fabsf(v[c]));
      float sc = group_scale(amax, fmt);
      s[r * G + g] = sc;
      for (int c = 0; c < 128; ++c) q[r * cols + g * 128 + c] = oracle_e4m3_encode(v[c] / sc);
    }
  }
}

/* Activation quantisation of bf16 rows [rows, cols]. */
void oracle_quant_act_fp8(const uint16_t* x, int64_t rows, int64_t cols, uint8_t* q, float* s,
                          int fmt) {
  float* v = (float*)malloc(sizeof(float) * (size_t)cols);
  for (int64_t r = 0; r < rows; ++r) {
    for (int64_t c = 0; c < cols; ++c) v[c] = bf16_widen(x[r * cols + c]);
    quant_groups_f32(v, 1, cols, q + r * cols, s + r * (cols / 128), fmt);
  }
  free(v);
}

/* Weight quantisation of nb matrices of bf16 [rows, cols] in 128 x 128
 * blocks: q [nb, rows, cols], s [nb, rows/128, cols/128]. Blocks are
 * independent; threads take whole blocks. */
typedef struct {
  const uint16_t* w;
  int64_t rows, cols;
  uint8_t* q;
  float* s;
  int fmt;
} wq_ctx;

static void wq_blocks(void* p, int64_t lo, int64_t hi) {
  wq_ctx* c = (wq_ctx*)p;
  int64_t RB = c->rows / 128, CB = c->cols / 128, rows = c->rows, cols = c->cols;
  for (int64_t blk = lo; blk < hi; ++blk) {
    int64_t b = blk / (RB * CB), rb = (blk / CB) % RB, cb = blk % CB;
    const uint16_t* wb = c->w + b * rows * cols;
    float amax = 0.0f;
    for (int64_t r = rb * 128; r < rb * 128 + 128; ++r)
      for (int64_t cc = cb * 128; cc < cb * 128 + 128; ++cc)
        amax = fmaxf(amax, fabsf(bf16_widen(wb[r * cols + cc])));
    float sc = group_scale(amax, c->fmt);
    c->s[blk] = sc;
    for (int64_t r = rb * 128; r < rb * 128 + 128; ++r)
      for (int64_t cc = cb * 128; cc < cb * 128 + 128; ++cc)
        c->q[b * rows * cols + r * cols + cc] = oracle_e4m3_encode(bf16_widen(wb[r * cols + cc]) / sc);
  }
}

void oracle_quant_weight_fp8(const uint16_t* w, int64_t nb, int64_t rows, int64_t cols,
                             uint8_t* q, float* s, int fmt, int nthreads) {
  wq_ctx c = {w, rows, cols, q, s, fmt};
  parallel_for(nb * (rows / 128) * (cols / 128), nthreads, wq_blocks, &c);
}


/* ------------------------------------------------------------------------ */
/* FP4 e2m1 (OCP: 1 sign, 2 exponent bits with bias 1, 1 mantissa bit; no   */
/* infinities, no NaN; magnitudes 0, 0.5, 1, 1.5, 2, 3, 4, 6).               */
/* "Experts backends", "FP8 and FP4 quantized experts": FP4 expert weights   */
/* packed two per byte, with weight scales in the UE8M0 format (8-bit        */
/* exponents, float8_e8m0fnu). The pages give no block geometry for them;    */
/* the OCP microscaling block is taken: one scale per row per 32 consecutive */
/* elements along K. The scale is the smallest power of two >= amax / 6      */
/* (that fp32 quotient, so no scaled value exceeds 6), within 2^-127..2^127, */
/* 1 for an all-zero block, stored as its biased exponent (code = p + 127).  */
/* Byte c/2 of a row holds element c (c even) in its low four bits and      */
/* element c + 1 in its high four bits. Activations stay FP8 e4m3 with      */
/* power-of-two scales per (row, 128-group), as in the UE8M0 FP8 layer.     */
/* ------------------------------------------------------------------------ */
double oracle_e2m1_decode(uint8_t q) {
  int s = (q >> 3) & 1, ef = (q >> 1) & 3, m = q & 1;
  double v = ef == 0 ? 0.5 * m : ldexp(1.0 + 0.5 * m, ef - 1);
  return s ? -v : v;
}

/* Nearest e2m1 magnitude, ties to the even code (mantissa bit 0); beyond 6
 * saturates to 6. The sign is kept (a negative value that rounds to zero
 * gives the code of -0). */
uint8_t oracle_e2m1_encode(float f) {
  static const double mag[8] = {0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0};
  uint8_t s = signbit(f) ? 8 : 0;
  double a = fabs((double)f);
  if (a >= 6.0) return s | 7;
  int best = 0;
  for (int c = 1; c < 8; ++c) {
    double dc = fabs(a - mag[c]), db = fabs(a - mag[best]);
    if (dc < db || (dc == db && (c & 1) == 0)) best = c;
  }
  return s | (uint8_t)best;
}

static inline float fp4_block_scale(float amax) {
  if (!(amax > 0.0f)) return 1.0f;
  const float r = amax / 6.0f;
  int e;
  const float m = frexpf(r, &e); /* r = m * 2^e, m in [0.5, 1) */
  int p2 = m == 0.5f ? e - 1 : e;
  if (p2 < -127) p2 = -127;
  if (p2 > 127) p2 = 127;
  return ldexpf(1.0f, p2);
}

/* nb matrices of bf16 [rows, cols] -> q [nb, rows, cols/2] (packed codes),
 * sc [nb, rows, cols/32] (e8m0 codes). Rows are independent. */
typedef struct {
  const uint16_t* w;
  int64_t cols;
  uint8_t *q, *sc;
} wq4_ctx;

static void wq4_rows(void* p, int64_t lo, int64_t hi) {
  wq4_ctx* c = (wq4_ctx*)p;
  const int64_t cols = c->cols;
  for (int64_t r = lo; r < hi; ++r) {
    const uint16_t* wr = c->w + r * cols;
    for (int64_t b = 0; b < cols / 32; ++b) {
      float amax = 0.0f;
      for (int i = 0; i < 32; ++i) amax = fmaxf(amax, fabsf(bf16_widen(wr[b * 32 + i])));
      const float sc = fp4_block_scale(amax);
      int ex;
      frexpf(sc, &ex); /* sc = 2^(ex - 1) */
      c->sc[r * (cols / 32) + b] = (uint8_t)(ex - 1 + 127);
      for (int i = 0; i < 32; i += 2) {
        uint8_t lo4 = oracle_e2m1_encode(bf16_widen(wr[b * 32 + i]) / sc);
        uint8_t hi4 = oracle_e2m1_encode(bf16_widen(wr[b * 32 + i + 1]) / sc);
        c->q[r * (cols / 2) + (b * 32 + i) / 2] = (uint8_t)(lo4 | (hi4 << 4));
      }
    }
  }
}

void oracle_quant_weight_fp4(const uint16_t* w, int64_t nb, int64_t rows, int64_t cols,
                             uint8_t* q, uint8_t* sc, int nthreads) {
  wq4_ctx c = {w, cols, q, sc};
  parallel_for(nb * rows, nthreads, wq4_rows, &c);
}

/* ------------------------------------------------------------------------ */
/* The layer: the eager per-expert loop.                                     */
/* "Experts backends", backend table, `eager` row (loop over the selected    */
/* experts, project their tokens), and "Mixture of Experts (MoE): a          */
/* practical explanation" §13's toy layer: for each slot j, for each expert  */
/* e, the tokens whose slot-j expert is e get out += w[t, j] * expert_e(x_t). */
/* Per token the k contributions are summed in slot order j = 0..k-1.        */
/* Runs on a subset of tokens (each token's output depends on that token     */
/* only, §5 pseudocode's `y = sum_i weights_i * expert_i(x)`).               */
/* ------------------------------------------------------------------------ */
typedef struct {
  const uint16_t* x;
  int64_t H, I, E;
  int k;
  const int32_t* tokens;
  int64_t nt;
  /* bf16 weights, or e4m3 codes + fp32 block scales */
  const uint16_t *w13, *w2;
  const uint8_t *w13q, *w2q, *xq;
  const float *w13s, *w2s, *xs;
  int fp8;       /* quantised experts: FP8 activations, e4m3 or e2m1 weights */
  int scale_fmt; /* FP8 scales: fp32 or power-of-two (UE8M0) */
  int fp4;       /* weights: packed e2m1 codes with e8m0 scales per (row, 32) */
  const uint8_t *w13s8, *w2s8;
  int act;       /* gated activation of the expert MLP */
  /* work list: items of up to CHUNK (row, slot) pairs of one expert */
  int64_t* item_e;
  int64_t* item_start; /* into pairs */
  int64_t* item_len;
  int32_t* pair_row;
  int32_t* pair_slot;
  int64_t nitems;
  int64_t next;
  pthread_mutex_t mu;
  double* y; /* [nt, k, H]: expert output of (row, slot) */
} fwd_ctx;

static void dequant_fp8(const uint8_t* q, const float* s, int64_t rows, int64_t cols, double* out) {
  int64_t CB = cols / 128;
  for (int64_t r = 0; r < rows; ++r)
    for (int64_t c = 0; c < cols; ++c)
      out[r * cols + c] = oracle_e4m3_decode(q[r * cols + c]) * (double)s[(r / 128) * CB + c / 128];
}

static void dequant_fp4(const uint8_t* q, const uint8_t* sc, int64_t rows, int64_t cols,
                        double* out) {
  for (int64_t r = 0; r < rows; ++r)
    for (int64_t c = 0; c < cols; ++c) {
      uint8_t byte = q[r * (cols / 2) + c / 2];
      uint8_t code = (c & 1) ? (byte >> 4) : (byte & 15);
      out[r * cols + c] = oracle_e2m1_decode(code) * ldexp(1.0, (int)sc[r * (cols / 32) + c / 32] - 127);
    }
}

static void* fwd_worker(void* p) {
  fwd_ctx* c = (fwd_ctx*)p;
  int64_t H = c->H, I = c->I;
  double* xr = (double*)malloc(sizeof(double) * (size_t)(GROUP * H));
  double* xT = (double*)malloc(sizeof(double) * (size_t)(GROUP * H));
  double* a = (double*)malloc(sizeof(double) * (size_t)(GROUP * I));
  double* aT = (double*)malloc(sizeof(double) * (size_t)(GROUP * I));
  double* y = (double*)malloc(sizeof(double) * (size_t)(GROUP * H));
  float* af = (float*)malloc(sizeof(float) * (size_t)I);
  uint8_t* aq = (uint8_t*)malloc((size_t)I);
  float* as = (float*)malloc(sizeof(float) * (size_t)(I / 128 + 1));
  double *w13d = NULL, *w2d = NULL;
  int64_t cur_e = -1;
  if (c->fp8) {
    w13d = (double*)malloc(sizeof(double) * (size_t)(2 * I * H));
    w2d = (double*)malloc(sizeof(double) * (size_t)(H * I));
  }
  for (;;) {
    pthread_mutex_lock(&c->mu);
    int64_t it = c->next++;
    pthread_mutex_unlock(&c->mu);
    if (it >= c->nitems) break;
    int64_t e = c->item_e[it];
    const uint16_t* w13e = c->fp8 ? NULL : c->w13 + e * 2 * I * H;
    const uint16_t* w2e = c->fp8 ? NULL : c->w2 + e * H * I;
    if (c->fp8 && e != cur_e) {
      if (c->fp4) { /* w-hat = e2m1 code * 2^(e8m0 code - 127) of its (row, 32) block */
        dequant_fp4(c->w13q + e * 2 * I * (H / 2), c->w13s8 + e * 2 * I * (H / 32), 2 * I, H, w13d);
        dequant_fp4(c->w2q + e * H * (I / 2), c->w2s8 + e * H * (I / 32), H, I, w2d);
      } else { /* w-hat = e4m3 code * its block scale */
        dequant_fp8(c->w13q + e * 2 * I * H, c->w13s + e * (2 * I / 128) * (H / 128), 2 * I, H, w13d);
        dequant_fp8(c->w2q + e * H * I, c->w2s + e * (H / 128) * (I / 128), H, I, w2d);
      }
      cur_e = e;
    }
    for (int64_t g0 = 0; g0 < c->item_len[it]; g0 += GROUP) {
      int64_t n = c->item_len[it] - g0 < GROUP ? c->item_len[it] - g0 : GROUP;
      const int32_t* rows = c->pair_row + c->item_start[it] + g0;
      const int32_t* slots = c->pair_slot + c->item_start[it] + g0;
      for (int64_t r = 0; r < n; ++r) {
        int64_t t = c->tokens[rows[r]];
        for (int64_t h = 0; h < H; ++h) {
          if (c->fp8) /* x-hat = e4m3(x / s) * s per (token, 128-group) */
            xr[r * H + h] = oracle_e4m3_decode(c->xq[rows[r] * H + h]) *
                            (double)c->xs[rows[r] * (H / 128) + h / 128];
          else
            xr[r * H + h] = (double)bf16_widen(c->x[t * H + h]);
        }
      }
      to_cols(xr, n, H, xT);
      expert_hidden(xT, n, w13e, w13d, H, I, c->act, a);
      if (c->fp8) { /* the down projection's input is quantised per (row, 128-group) too */
        for (int64_t r = 0; r < n; ++r) {
          for (int64_t i = 0; i < I; ++i) af[i] = (float)a[r * I + i];
          quant_groups_f32(af, 1, I, aq, as, c->scale_fmt);
          for (int64_t i = 0; i < I; ++i) a[r * I + i] = oracle_e4m3_decode(aq[i]) * (double)as[i / 128];
        }
      }
      to_cols(a, n, I, aT);
      expert_out(aT, n, w2e, w2d, H, I, y);
      for (int64_t r = 0; r < n; ++r)
        memcpy(c->y + ((int64_t)rows[r] * c->k + slots[r]) * H, y + r * H, sizeof(double) * (size_t)H);
    }
  }
  free(xr);
  free(xT);
  free(a);
  free(aT);
  free(y);
  free(af);
  free(aq);
  free(as);
  free(w13d);
  free(w2d);
  return NULL;
}

/* The toy layer's (slot j, expert e) loops evaluate expert e on every token
 * whose slot-j choice is e. The same (token, slot) evaluations are made here,
 * grouped by expert so one expert's weights are read together; each is an
 * independent computation, and the k results of a token are then summed in
 * slot order j = 0..k-1. */
static void run_forward(fwd_ctx* c, const int32_t* ids, const float* topk_w, float* out,
                        int nthreads) {
  int64_t nt = c->nt, k = c->k, E = c->E, H = c->H;
  const int64_t CHUNK = 64;
  int64_t max_items = E + nt * k / CHUNK + 1;
  c->item_e = (int64_t*)malloc(sizeof(int64_t) * (size_t)max_items);
  c->item_start = (int64_t*)malloc(sizeof(int64_t) * (size_t)max_items);
  c->item_len = (int64_t*)malloc(sizeof(int64_t) * (size_t)max_items);
  c->pair_row = (int32_t*)malloc(sizeof(int32_t) * (size_t)(nt * k + 1));
  c->pair_slot = (int32_t*)malloc(sizeof(int32_t) * (size_t)(nt * k + 1));
  c->y = (double*)calloc((size_t)(nt * k * H), sizeof(double));
  int64_t p = 0, ni = 0;
  for (int64_t e = 0; e < E; ++e) {
    int64_t start = p;
    for (int64_t r = 0; r < nt; ++r)
      for (int64_t j = 0; j < k; ++j)
        if (ids[r * k + j] == e) {
          c->pair_row[p] = (int32_t)r;
          c->pair_slot[p] = (int32_t)j;
          ++p;
        }
    for (int64_t s0 = start; s0 < p; s0 += CHUNK) {
      c->item_e[ni] = e;
      c->item_start[ni] = s0;
      c->item_len[ni] = p - s0 < CHUNK ? p - s0 : CHUNK;
      ++ni;
    }
  }
  c->nitems = ni;
  c->next = 0;
  pthread_mutex_init(&c->mu, NULL);
  if (nthreads < 1) nthreads = 1;
  if (nthreads > 256) nthreads = 256;
  pthread_t th[256];
  for (int t = 0; t < nthreads; ++t) pthread_create(&th[t], NULL, fwd_worker, c);
  for (int t = 0; t < nthreads; ++t) pthread_join(th[t], NULL);
  pthread_mutex_destroy(&c->mu);
  /* weighted combine: out[t] = sum_{j ascending} w[t, j] * y[t, j] */
  for (int64_t r = 0; r < nt; ++r) {
    for (int64_t h = 0; h < H; ++h) {
      double acc = 0.0;
      for (int64_t j = 0; j < k; ++j) acc += (double)topk_w[r * k + j] * c->y[(r * k + j) * H + h];
      out[r * H + h] = (float)acc;
    }
  }
  free(c->item_e);
  free(c->item_start);
  free(c->item_len);
  free(c->pair_row);
  free(c->pair_slot);
  free(c->y);
}

/* Experts + combine for given routing (ids/w [nt, k]) of tokens[0..nt).
 * out: [nt, H] fp32. */
void oracle_experts_combine(const uint16_t* x, const int32_t* tokens, int64_t nt, int64_t H,
                            int64_t I, int64_t E, int k, const int32_t* ids, const float* topk_w,
                            const uint16_t* w13, const uint16_t* w2, int act, float* out,
                            int nthreads) {
  fwd_ctx c;
  memset(&c, 0, sizeof(c));
  c.act = act;
  c.x = x;
  c.H = H;
  c.I = I;
  c.E = E;
  c.k = k;
  c.tokens = tokens;
  c.nt = nt;
  c.w13 = w13;
  c.w2 = w2;
  run_forward(&c, ids, topk_w, out, nthreads);
}

/* FP8 experts + combine: x is quantised here per (token, 128-group), weights
 * are given as e4m3 codes with fp32 128 x 128 block scales. */
void oracle_experts_combine_fp8(const uint16_t* x, const int32_t* tokens, int64_t nt, int64_t H,
                                int64_t I, int64_t E, int k, const int32_t* ids,
                                const float* topk_w, const uint8_t* w13q, const float* w13s,
                                const uint8_t* w2q, const float* w2s, int act, int scale_fmt,
                                float* out, int nthreads) {
  uint8_t* xq = (uint8_t*)malloc((size_t)(nt * H));
  float* xs = (float*)malloc(sizeof(float) * (size_t)(nt * (H / 128)));
  uint16_t* xrows = (uint16_t*)malloc(sizeof(uint16_t) * (size_t)H);
  for (int64_t r = 0; r < nt; ++r) {
    memcpy(xrows, x + (int64_t)tokens[r] * H, sizeof(uint16_t) * (size_t)H);
    oracle_quant_act_fp8(xrows, 1, H, xq + r * H, xs + r * (H / 128), scale_fmt);
  }
  fwd_ctx c;
  memset(&c, 0, sizeof(c));
  c.x = x;
  c.H = H;
  c.I = I;
  c.E = E;
  c.k = k;
  c.tokens = tokens;
  c.nt = nt;
  c.w13q = w13q;
  c.w13s = w13s;
  c.w2q = w2q;
  c.w2s = w2s;
  c.xq = xq;
  c.xs = xs;
  c.fp8 = 1;
  c.scale_fmt = scale_fmt;
  c.act = act;
  run_forward(&c, ids, topk_w, out, nthreads);
  free(xq);
  free(xs);
  free(xrows);
}

/* FP4 experts + combine: x is quantised here per (token, 128-group) to e4m3
 * with power-of-two scales; weights are packed e2m1 codes with e8m0 scales
 * per (row, 32-element block); the down projection's input is re-quantised
 * the same way as x. */
void oracle_experts_combine_fp4(const uint16_t* x, const int32_t* tokens, int64_t nt, int64_t H,
                                int64_t I, int64_t E, int k, const int32_t* ids,
                                const float* topk_w, const uint8_t* w13q, const uint8_t* w13s,
                                const uint8_t* w2q, const uint8_t* w2s, int act, float* out,
                                int nthreads) {
  uint8_t* xq = (uint8_t*)malloc((size_t)(nt * H));
  float* xs = (float*)malloc(sizeof(float) * (size_t)(nt * (H / 128)));
  for (int64_t r = 0; r < nt; ++r)
    oracle_quant_act_fp8(x + (int64_t)tokens[r] * H, 1, H, xq + r * H, xs + r * (H / 128),
                         SCALE_UE8M0);
  fwd_ctx c;
  memset(&c, 0, sizeof(c));
  c.x = x;
  c.H = H;
  c.I = I;
  c.E = E;
  c.k = k;
  c.tokens = tokens;
  c.nt = nt;
  c.w13q = w13q;
  c.w13s8 = w13s;
  c.w2q = w2q;
  c.w2s8 = w2s;
  c.xq = xq;
  c.xs = xs;
  c.fp8 = 1;
  c.fp4 = 1;
  c.scale_fmt = SCALE_UE8M0;
  c.act = act;
  run_forward(&c, ids, topk_w, out, nthreads);
  free(xq);
  free(xs);
}

/* The whole layer with FP4 experts for tokens[0..nt) (see
 * oracle_experts_combine_fp4); ids_out / w_out / logits_out may be NULL. */
void oracle_moe_forward_fp4(const uint16_t* x, const int32_t* tokens, int64_t nt, int64_t H,
                            int64_t I, int64_t E, int k, const uint16_t* wr, const float* bias,
                            const uint8_t* w13q, const uint8_t* w13s, const uint8_t* w2q,
                            const uint8_t* w2s, int act, float* out, int32_t* ids_out,
                            float* w_out, float* logits_out, int nthreads) {
  float* logits = logits_out ? logits_out : (float*)malloc(sizeof(float) * (size_t)(nt * E));
  int32_t* ids = ids_out ? ids_out : (int32_t*)malloc(sizeof(int32_t) * (size_t)(nt * k));
  float* w = w_out ? w_out : (float*)malloc(sizeof(float) * (size_t)(nt * k));
  oracle_router_logits(x, wr, bias, tokens, nt, H, E, logits, nthreads);
  oracle_topk(logits, nt, E, k, ids, w);
  oracle_experts_combine_fp4(x, tokens, nt, H, I, E, k, ids, w, w13q, w13s, w2q, w2s, act, out,
                             nthreads);
  if (!logits_out) free(logits);
  if (!ids_out) free(ids);
  if (!w_out) free(w);
}

/* The whole layer for tokens[0..nt): logits -> top-k -> experts -> combine.
 * ids_out/w_out ([nt, k]) and logits_out ([nt, E]) may be NULL. */
void oracle_moe_forward(const uint16_t* x, const int32_t* tokens, int64_t nt, int64_t H, int64_t I,
                        int64_t E, int k, const uint16_t* wr, const float* bias,
                        const uint16_t* w13, const uint16_t* w2, const uint8_t* w13q,
                        const float* w13s, const uint8_t* w2q, const float* w2s, int act,
                        int scale_fmt, float* out, int32_t* ids_out, float* w_out,
                        float* logits_out, int nthreads) {
  float* logits = logits_out ? logits_out : (float*)malloc(sizeof(float) * (size_t)(nt * E));
  int32_t* ids = ids_out ? ids_out : (int32_t*)malloc(sizeof(int32_t) * (size_t)(nt * k));
  float* w = w_out ? w_out : (float*)malloc(sizeof(float) * (size_t)(nt * k));
  oracle_router_logits(x, wr, bias, tokens, nt, H, E, logits, nthreads);
  oracle_topk(logits, nt, E, k, ids, w);
  if (w13q)
    oracle_experts_combine_fp8(x, tokens, nt, H, I, E, k, ids, w, w13q, w13s, w2q, w2s, act,
                               scale_fmt, out, nthreads);
  else
    oracle_experts_combine(x, tokens, nt, H, I, E, k, ids, w, w13, w2, act, out, nthreads);
  if (!logits_out) free(logits);
  if (!ids_out) free(ids);
  if (!w_out) free(w);
}

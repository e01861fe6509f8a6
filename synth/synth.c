/*
 * Seeded synthetic inputs for the CSA lightning-indexer top-k step.
 *
 * This module is shared by the CUDA path's tests/benchmark and by the CPU
 * oracle's tests.  It holds none of the indexer's arithmetic: it only draws
 * numbers and stores them in the input formats (bf16, fp8 e4m3 + per-row fp32
 * scale, fp32).
 *
 * Random numbers: SplitMix64 (Steele, Lea, Flood, "Fast splittable
 * pseudorandom number generators", OOPSLA 2014), used counter-based: the n-th
 * output of a stream seeded with `key` is mix(key + (n+1)*GAMMA), so every
 * element is a pure function of (seed, tensor id, flat index) and any slice
 * can be generated on its own, in parallel, in any order.
 *
 * Normals: Box-Muller transform on two uniforms per element (host libm).
 * bf16: round-to-nearest-even from fp32.
 * fp8 e4m3: OCP 8-bit floating point specification (E4M3: bias 7, no
 * infinities, max finite 448, subnormal step 2^-9); round-to-nearest-even,
 * saturating to +-448.  Per-row scale = amax/448.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define GAMMA 0x9E3779B97F4A7C15ull

static inline uint64_t smix(uint64_t z) {
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}

/* n-th output of the SplitMix64 stream whose state starts at `key`. */
uint64_t synth_draw(uint64_t key, uint64_t n) { return smix(key + (n + 1) * GAMMA); }

/* Stream key for one tensor of one seeded workload. */
uint64_t synth_stream_key(uint64_t seed, uint32_t tensor_id) {
  return synth_draw(synth_draw(seed, 0x5EED), tensor_id);
}

static inline double u01_open_closed(uint64_t u) { /* (0, 1] */
  return (double)((u >> 11) + 1) * (1.0 / 9007199254740992.0);
}
static inline double u01(uint64_t u) { /* [0, 1) */
  return (double)(u >> 11) * (1.0 / 9007199254740992.0);
}
static inline int u_below(uint64_t u, uint32_t n) { /* multiply-shift, 0..n-1 */
  return (int)(((u >> 32) * (uint64_t)n) >> 32);
}

double synth_normal(uint64_t key, uint64_t i) {
  double a = u01_open_closed(synth_draw(key, 2 * i));
  double b = u01(synth_draw(key, 2 * i + 1));
  return sqrt(-2.0 * log(a)) * cos(6.283185307179586 * b);
}

uint16_t synth_f32_to_bf16(float x) {
  uint32_t u;
  memcpy(&u, &x, 4);
  if ((u & 0x7F800000u) == 0x7F800000u) return (uint16_t)(u >> 16); /* inf/nan: truncate */
  u += 0x7FFFu + ((u >> 16) & 1u);
  return (uint16_t)(u >> 16);
}

/* OCP E4M3 encode: round to nearest even, saturate to 448. */
uint8_t synth_f32_to_e4m3(float x) {
  uint8_t sign = (x < 0.0f || (x == 0.0f && signbit(x))) ? 0x80 : 0x00;
  double a = fabs((double)x);
  if (a != a) return 0x7F; /* NaN */
  if (a >= 448.0) return sign | 0x7E;
  if (a == 0.0) return sign;
  int e;
  frexp(a, &e);           /* a = f * 2^e, f in [0.5, 1) -> a in [2^(e-1), 2^e) */
  int E = e - 1;          /* a in [2^E, 2^(E+1)) */
  if (E < -6) {           /* subnormal range: step 2^-9 */
    double m = nearbyint(a * 512.0); /* default rounding mode: nearest-even */
    if (m >= 8.0) return sign | 0x08; /* rounds up to min normal 2^-6 */
    return sign | (uint8_t)m;
  }
  double frac = a / ldexp(1.0, E) - 1.0;      /* [0, 1) */
  double mq = nearbyint(frac * 8.0);          /* 0..8 */
  if (mq >= 8.0) { mq = 0.0; E += 1; }
  if (E > 8) return sign | 0x7E;
  uint8_t code = (uint8_t)(((E + 7) << 3) | (int)mq);
  if (code == 0x7F) code = 0x7E;              /* 480 would be NaN: saturate */
  return sign | code;
}

/* ---------------------------------------------------------------- threads */
typedef void (*row_fn)(void* ctx, int64_t r0, int64_t r1);
typedef struct { row_fn fn; void* ctx; int64_t r0, r1; } job_t;
static void* job_run(void* p) { job_t* j = (job_t*)p; j->fn(j->ctx, j->r0, j->r1); return NULL; }

static void parallel_rows(row_fn fn, void* ctx, int64_t rows, int nthreads) {
  if (nthreads < 1) nthreads = 1;
  if (nthreads > 256) nthreads = 256;
  if (rows < 4096 || nthreads == 1) { fn(ctx, 0, rows); return; }
  pthread_t th[256];
  job_t jobs[256];
  int64_t per = (rows + nthreads - 1) / nthreads;
  int n = 0;
  for (int i = 0; i < nthreads; ++i) {
    int64_t a = (int64_t)i * per, b = a + per;
    if (b > rows) b = rows;
    if (a >= b) break;
    jobs[n].fn = fn; jobs[n].ctx = ctx; jobs[n].r0 = a; jobs[n].r1 = b;
    pthread_create(&th[n], NULL, job_run, &jobs[n]);
    ++n;
  }
  for (int i = 0; i < n; ++i) pthread_join(th[i], NULL);
}

/* --------------------------------------------------------- row producers */
enum { KIND_GAUSS = 0, KIND_INT = 1 };
enum { FMT_BF16 = 0, FMT_E4M3 = 1 };

typedef struct {
  void* out; float* scale; int D; int kind; int fmt;
  uint64_t key; double sigma;
  int64_t row0; /* global index of out's first row (element counter base) */
  /* planted boost (kc only) */
  const uint8_t* boosted; const float* dir; int T; double boost;
} rows_ctx;

static void store_row(rows_ctx* c, int64_t r, const float* x) {
  int D = c->D;
  if (c->fmt == FMT_BF16) {
    uint16_t* o = (uint16_t*)c->out + r * D;
    for (int d = 0; d < D; ++d) o[d] = synth_f32_to_bf16(x[d]);
  } else {
    float amax = 0.0f;
    for (int d = 0; d < D; ++d) { float a = fabsf(x[d]); if (a > amax) amax = a; }
    float s = amax > 0.0f ? amax / 448.0f : 1.0f;
    c->scale[r] = s;
    uint8_t* o = (uint8_t*)c->out + r * D;
    for (int d = 0; d < D; ++d) o[d] = synth_f32_to_e4m3(x[d] / s);
  }
}

static void rows_work(void* p, int64_t r0, int64_t r1) {
  rows_ctx* c = (rows_ctx*)p;
  float x[1024];
  for (int64_t r = r0; r < r1; ++r) {
    const float* dir = NULL;
    if (c->boosted && c->boosted[r]) dir = c->dir + (r / c->T) * c->D;
    for (int d = 0; d < c->D; ++d) {
      uint64_t i = (uint64_t)(c->row0 + r) * c->D + d;
      double v;
      if (c->kind == KIND_GAUSS) v = synth_normal(c->key, i) * c->sigma;
      else v = (double)(u_below(synth_draw(c->key, i), 7) - 3);
      if (dir) v += c->boost * (double)dir[d];
      x[d] = (float)v;
    }
    store_row(c, r, x);
  }
}

/*
 * rows x D matrix.  kind 0: N(0,1)*sigma; kind 1: integers uniform in
 * {-3..3}.  fmt 0: bf16 into out (uint16); fmt 1: e4m3 into out (uint8) with
 * one fp32 scale per row into scale.
 */
int synth_matrix(void* out, float* scale, int64_t rows, int D, uint64_t seed,
                 uint32_t tensor_id, int kind, double sigma, int fmt, int nthreads) {
  if (D <= 0 || D > 1024 || rows < 0 || (fmt == FMT_E4M3 && !scale)) return -1;
  rows_ctx c;
  memset(&c, 0, sizeof c);
  c.out = out; c.scale = scale; c.D = D; c.kind = kind; c.fmt = fmt;
  c.key = synth_stream_key(seed, tensor_id); c.sigma = sigma;
  parallel_rows(rows_work, &c, rows, nthreads);
  return 0;
}

/*
 * Rows [row0, row0 + rows) of the matrix synth_matrix would make, written to
 * out (and scale) starting at their first element: the same values, for
 * callers that fill a large tensor piecewise or need a few rows only.
 */
int synth_matrix_range(void* out, float* scale, int64_t row0, int64_t rows, int D, uint64_t seed,
                       uint32_t tensor_id, int kind, double sigma, int fmt, int nthreads) {
  if (D <= 0 || D > 1024 || rows < 0 || row0 < 0 || (fmt == FMT_E4M3 && !scale)) return -1;
  rows_ctx c;
  memset(&c, 0, sizeof c);
  c.out = out; c.scale = scale; c.D = D; c.kind = kind; c.fmt = fmt;
  c.key = synth_stream_key(seed, tensor_id); c.sigma = sigma; c.row0 = row0;
  parallel_rows(rows_work, &c, rows, nthreads);
  return 0;
}

/*
 * Planted-boost key matrix [B*T, D]: every row is N(0,1)*sigma; in each
 * sequence b, n_boost = round(frac*T) rows chosen uniformly without
 * replacement (partial Fisher-Yates) get `boost * u_b` added, u_b a unit
 * vector drawn per sequence.  Values are summed in double, then stored.
 * boosted_out (optional, B*T bytes) receives the 0/1 choice per row.
 */
int synth_keys_planted(void* out, float* scale, int B, int T, int D, uint64_t seed,
                       uint32_t tensor_id, double sigma, double frac, double boost,
                       int fmt, int nthreads, uint8_t* boosted_out) {
  if (B <= 0 || T <= 0 || D <= 0 || D > 1024 || (fmt == FMT_E4M3 && !scale)) return -1;
  int64_t rows = (int64_t)B * T;
  uint8_t* boosted = (uint8_t*)calloc((size_t)rows, 1);
  float* dir = (float*)malloc(sizeof(float) * (size_t)B * D);
  int32_t* perm = (int32_t*)malloc(sizeof(int32_t) * (size_t)T);
  if (!boosted || !dir || !perm) { free(boosted); free(dir); free(perm); return -2; }
  uint64_t kdir = synth_stream_key(seed, tensor_id + 100);
  uint64_t kpick = synth_stream_key(seed, tensor_id + 200);
  int64_t nb = (int64_t)llround(frac * (double)T);
  if (nb > T) nb = T;
  for (int b = 0; b < B; ++b) {
    double nrm = 0.0, tmp[1024];
    for (int d = 0; d < D; ++d) { tmp[d] = synth_normal(kdir, (uint64_t)b * D + d); nrm += tmp[d] * tmp[d]; }
    nrm = sqrt(nrm);
    for (int d = 0; d < D; ++d) dir[(size_t)b * D + d] = (float)(tmp[d] / nrm);
    for (int s = 0; s < T; ++s) perm[s] = s;
    for (int64_t i = 0; i < nb; ++i) {
      uint64_t u = synth_draw(kpick, (uint64_t)b * T + i);
      int64_t j = i + (int64_t)(u % (uint64_t)(T - i));
      int32_t t = perm[i]; perm[i] = perm[j]; perm[j] = t;
      boosted[(int64_t)b * T + perm[i]] = 1;
    }
  }
  rows_ctx c;
  memset(&c, 0, sizeof c);
  c.out = out; c.scale = scale; c.D = D; c.kind = KIND_GAUSS; c.fmt = fmt;
  c.key = synth_stream_key(seed, tensor_id); c.sigma = sigma;
  c.boosted = boosted; c.dir = dir; c.T = T; c.boost = boost;
  parallel_rows(rows_work, &c, rows, nthreads);
  if (boosted_out) memcpy(boosted_out, boosted, (size_t)rows);
  free(boosted); free(dir); free(perm);
  return 0;
}

/* ---------------------------------------------------------------- weights */
typedef struct { float* out; uint64_t key; int kind; double scale; } w_ctx;

static void w_work(void* p, int64_t r0, int64_t r1) {
  w_ctx* c = (w_ctx*)p;
  for (int64_t i = r0; i < r1; ++i) {
    uint64_t u = synth_draw(c->key, (uint64_t)i);
    if (c->kind == 0) c->out[i] = (float)(u01(u) * c->scale);
    else c->out[i] = (float)ldexp(1.0, -u_below(u, 7));
  }
}

/* n fp32 weights.  kind 0: U(0,1)*scale; kind 1: 2^-j, j uniform in {0..6}. */
int synth_weights(float* out, int64_t n, uint64_t seed, uint32_t tensor_id, int kind,
                  double scale, int nthreads) {
  if (n < 0) return -1;
  w_ctx c = {out, synth_stream_key(seed, tensor_id), kind, scale};
  parallel_rows(w_work, &c, n, nthreads);
  return 0;
}

/* Uniform sample of `count` distinct integers from [lo, hi) (partial
 * Fisher-Yates over a counter stream), written sorted ascending. */
int synth_sample_rows(int64_t* out, int64_t count, int64_t lo, int64_t hi, uint64_t seed) {
  int64_t n = hi - lo;
  if (count < 0 || n < count) return -1;
  int64_t* p = (int64_t*)malloc(sizeof(int64_t) * (size_t)(n > 0 ? n : 1));
  if (!p) return -2;
  for (int64_t i = 0; i < n; ++i) p[i] = lo + i;
  uint64_t key = synth_stream_key(seed, 900);
  for (int64_t i = 0; i < count; ++i) {
    int64_t j = i + (int64_t)(synth_draw(key, (uint64_t)i) % (uint64_t)(n - i));
    int64_t t = p[i]; p[i] = p[j]; p[j] = t;
  }
  /* insertion sort of the chosen prefix (count is small) */
  for (int64_t i = 1; i < count; ++i) {
    int64_t v = p[i], j = i - 1;
    while (j >= 0 && p[j] > v) { p[j + 1] = p[j]; --j; }
    p[j + 1] = v;
  }
  memcpy(out, p, sizeof(int64_t) * (size_t)count);
  free(p);
  return 0;
}

/*
 * CPU oracle for the CSA lightning-indexer top-k step.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check and the
 * benchmark's CPU-baseline leg may load or call this file.  It shares no code,
 * header, table or helper with the CUDA library, and the library never calls
 * it.
 *
 * What it computes (StreamIndex, "Memory-Bounded Compressed Sparse Attention
 * via Streaming Top-k", abstract: a lightning indexer -- a learned scoring
 * projection over compressed keys -- scores the compressed keys and the top-k
 * are selected per query).  The scoring function is the DeepSeek-V3.2
 * lightning-indexer form, which the pages name only as that lineage:
 *
 *     I[b,t,s] = sum_h w[b,t,h] * ReLU( sum_d q[b,t,h,d] * kc[b,s,d] )
 *
 * Compressed key s covers tokens [s*m, s*m+m-1]; it is visible to query t iff
 * s*m+m-1 <= t (and s < T), so row t sees n(t) = min(T, floor((t+1)/m))
 * keys, namely s = 0..n(t)-1.  The row's result is its visible keys fully
 * sorted by (score descending, index ascending), truncated to k, padded with
 * index -1 / score -inf when n(t) < k.
 *
 * Key formats: bf16; fp8 E4M3 with a per-row fp32 scale; and MXFP4 (the
 * 4-bit indexer keys named by the V4.1-Flash deployment notes, "two-level
 * sparse attention", indexer_kv_dtype): OCP Microscaling FP4 -- E2M1 codes,
 * two per byte, with one E8M0 power-of-two scale per 32 consecutive values
 * along D; queries stay bf16 in that format.
 *
 * Arithmetic: every input value is widened exactly to double (bf16 -> double
 * is exact; e4m3 -> double is exact; an E2M1 code times its E8M0 block scale
 * is a power-of-two multiple of a 2-bit significand, exact in double; scales
 * and w are fp32, exact in double),
 * dot products are summed in d order, heads in h order, all in double.  The
 * reported score is the double result rounded to float.  Plain loops,
 * single-threaded, no SIMD intrinsics; qsort for the full sort.
 *
 * Parity pins (tests): hand-worked 4x4 cases, the matmul special cases, the
 * visible-pair closed form, the causal invariant, prefix monotonicity of
 * top-k, brute force over all k-subsets, head-permutation and power-of-two
 * scaling invariances, integer-exact inputs.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* bf16 bit pattern -> double (bf16 is the top half of an IEEE binary32). */
double oracle_bf16_value(uint16_t bits) {
  uint32_t u = (uint32_t)bits << 16;
  float f;
  memcpy(&f, &u, 4);
  return (double)f;
}

/* OCP FP8 E4M3: sign, 4 exponent bits (bias 7), 3 mantissa bits; exponent
 * field 0 is subnormal (m * 2^-9); S.1111.111 is NaN; no infinities. */
double oracle_e4m3_value(uint8_t bits) {
  int sign = bits >> 7, e = (bits >> 3) & 15, m = bits & 7;
  double v;
  if (e == 15 && m == 7) return NAN;
  if (e == 0) v = ldexp((double)m, -9);
  else v = ldexp(1.0 + m / 8.0, e - 7);
  return sign ? -v : v;
}

/* OCP MX FP4 E2M1, a 4-bit code: bit 3 sign, bits 2-1 exponent (bias 1),
 * bit 0 mantissa; exponent field 0 is subnormal (mantissa * 0.5).  The
 * magnitudes are 0, 0.5, 1, 1.5, 2, 3, 4, 6; there is no infinity or NaN. */
double oracle_e2m1_value(uint8_t code) {
  int sign = (code >> 3) & 1, e = (code >> 1) & 3, m = code & 1;
  double v = e == 0 ? 0.5 * m : ldexp(1.0 + 0.5 * m, e - 1);
  return sign ? -v : v;
}

/* OCP MX E8M0 block scale: 2^(bits - 127); 0xFF is NaN. */
double oracle_e8m0_value(uint8_t bits) {
  if (bits == 0xFF) return NAN;
  return ldexp(1.0, (int)bits - 127);
}

/* Number of keys visible to query t: key s is visible iff s*m+m-1 <= t. */
int64_t oracle_visible_count(int64_t t, int64_t T, int64_t m) {
  int64_t n = (t + 1) / m;
  return n < T ? n : T;
}

/* One indexer score in double from already-widened rows.
 * qT: D*H (d-major, i.e. the query row transposed), krow: D, wrow: H,
 * dot: H doubles of scratch.  Each head's dot product is summed over d in
 * increasing order; the loop runs the H independent sums side by side. */
static double score_rows(const double* qT, const double* krow, const double* wrow, int H, int D,
                         double* dot) {
  for (int h = 0; h < H; ++h) dot[h] = 0.0;
  for (int d = 0; d < D; ++d) {
    const double kd = krow[d];
    const double* qd = qT + (size_t)d * H;
    for (int h = 0; h < H; ++h) dot[h] += qd[h] * kd;
  }
  double acc = 0.0;
  for (int h = 0; h < H; ++h) {
    double r = dot[h] > 0.0 ? dot[h] : 0.0;
    acc += wrow[h] * r;
  }
  return acc;
}

typedef struct { double score; int64_t idx; } cand_t;

/* score descending, then index ascending */
static int cand_cmp(const void* pa, const void* pb) {
  const cand_t* a = (const cand_t*)pa;
  const cand_t* b = (const cand_t*)pb;
  if (a->score > b->score) return -1;
  if (a->score < b->score) return 1;
  return (a->idx > b->idx) - (a->idx < b->idx);
}

/* Widening of one query row / key row / weight row to double. */
typedef struct {
  int fmt; /* 0 bf16, 1 e4m3, 2 bf16 queries with MXFP4 keys */
  const void* q; const float* q_scale;
  const void* kc; const float* kc_scale;
  const float* w;
  int64_t B, S, T, H, D, m;
  const uint8_t* kc_mx; /* fmt 2: E8M0 block scales [B,T,D/32] */
} problem_t;

/* Value d of MXFP4 row r: codes [rows, D/2] bytes, value d in the low
 * nibble of byte d/2 when d is even and in the high nibble when d is odd;
 * scales [rows, D/32], block d/32. */
static double mxfp4_value(const uint8_t* codes, const uint8_t* scales, int64_t r, int64_t D, int64_t d) {
  uint8_t byte = codes[r * (D / 2) + d / 2];
  uint8_t code = (d & 1) ? (uint8_t)(byte >> 4) : (uint8_t)(byte & 15);
  return oracle_e2m1_value(code) * oracle_e8m0_value(scales[r * (D / 32) + d / 32]);
}

/* qrow receives the query's H x D values transposed to D x H. */
static void widen_query(const problem_t* p, int64_t b, int64_t t, double* qrow, double* wrow) {
  int64_t base = (b * p->S + t) * p->H;
  for (int64_t h = 0; h < p->H; ++h) {
    wrow[h] = (double)p->w[base + h];
    for (int64_t d = 0; d < p->D; ++d) {
      int64_t i = (base + h) * p->D + d;
      if (p->fmt != 1) qrow[d * p->H + h] = oracle_bf16_value(((const uint16_t*)p->q)[i]);
      else qrow[d * p->H + h] = oracle_e4m3_value(((const uint8_t*)p->q)[i]) * (double)p->q_scale[base + h];
    }
  }
}

static void widen_key(const problem_t* p, int64_t b, int64_t s, double* krow) {
  int64_t r = b * p->T + s;
  for (int64_t d = 0; d < p->D; ++d) {
    int64_t i = r * p->D + d;
    if (p->fmt == 0) krow[d] = oracle_bf16_value(((const uint16_t*)p->kc)[i]);
    else if (p->fmt == 2) krow[d] = mxfp4_value((const uint8_t*)p->kc, p->kc_mx, r, p->D, d);
    else krow[d] = oracle_e4m3_value(((const uint8_t*)p->kc)[i]) * (double)p->kc_scale[r];
  }
}

/*
 * Top-k for the listed rows.  rows[i] = b*S + t.  Outputs are [n_rows, k]:
 * out_idx (int32, -1 padded), out_score (float, -inf padded, may be NULL),
 * out_score64 (double, -inf padded, may be NULL).  Returns 0, or -1 on a bad
 * argument, -2 on allocation failure.
 */
static int topk_rows(const problem_t* p, int64_t k, const int64_t* rows, int64_t n_rows,
                     int32_t* out_idx, float* out_score, double* out_score64) {
  if (p->B <= 0 || p->S <= 0 || p->T <= 0 || p->H <= 0 || p->D <= 0 || p->m <= 0 || k <= 0) return -1;
  double* qrow = (double*)malloc(sizeof(double) * (size_t)(p->H * p->D));
  double* wrow = (double*)malloc(sizeof(double) * (size_t)p->H);
  double* krow = (double*)malloc(sizeof(double) * (size_t)p->D);
  double* dot = (double*)malloc(sizeof(double) * (size_t)p->H);
  cand_t* c = (cand_t*)malloc(sizeof(cand_t) * (size_t)p->T);
  if (!qrow || !wrow || !krow || !dot || !c) {
    free(qrow); free(wrow); free(krow); free(dot); free(c);
    return -2;
  }
  for (int64_t i = 0; i < n_rows; ++i) {
    int64_t r = rows[i];
    if (r < 0 || r >= p->B * p->S) { free(qrow); free(wrow); free(krow); free(dot); free(c); return -1; }
    int64_t b = r / p->S, t = r % p->S;
    int64_t n = oracle_visible_count(t, p->T, p->m);
    widen_query(p, b, t, qrow, wrow);
    for (int64_t s = 0; s < n; ++s) {
      widen_key(p, b, s, krow);
      c[s].score = score_rows(qrow, krow, wrow, (int)p->H, (int)p->D, dot);
      c[s].idx = s;
    }
    qsort(c, (size_t)n, sizeof(cand_t), cand_cmp);
    for (int64_t j = 0; j < k; ++j) {
      int64_t o = i * k + j;
      if (j < n) {
        out_idx[o] = (int32_t)c[j].idx;
        if (out_score) out_score[o] = (float)c[j].score;
        if (out_score64) out_score64[o] = c[j].score;
      } else {
        out_idx[o] = -1;
        if (out_score) out_score[o] = -INFINITY;
        if (out_score64) out_score64[o] = -INFINITY;
      }
    }
  }
  free(qrow); free(wrow); free(krow); free(dot); free(c);
  return 0;
}

/* bf16 q [B,S,H,D], bf16 kc [B,T,D], fp32 w [B,S,H]. */
int oracle_topk_bf16(const uint16_t* q, const uint16_t* kc, const float* w, int64_t B, int64_t S,
                     int64_t T, int64_t H, int64_t D, int64_t m, int64_t k, const int64_t* rows,
                     int64_t n_rows, int32_t* out_idx, float* out_score, double* out_score64) {
  problem_t p = {0, q, NULL, kc, NULL, w, B, S, T, H, D, m, NULL};
  return topk_rows(&p, k, rows, n_rows, out_idx, out_score, out_score64);
}

/* bf16 q [B,S,H,D]; MXFP4 kc: codes [B,T,D/2] bytes and E8M0 scales
 * [B,T,D/32] (D a multiple of 32). */
int oracle_topk_mxfp4(const uint16_t* q, const uint8_t* kc, const uint8_t* kc_mx_scale, const float* w,
                      int64_t B, int64_t S, int64_t T, int64_t H, int64_t D, int64_t m, int64_t k,
                      const int64_t* rows, int64_t n_rows, int32_t* out_idx, float* out_score,
                      double* out_score64) {
  if (D <= 0 || D % 32 != 0) return -1;
  problem_t p = {2, q, NULL, kc, NULL, w, B, S, T, H, D, m, kc_mx_scale};
  return topk_rows(&p, k, rows, n_rows, out_idx, out_score, out_score64);
}

/* The MXFP4 rows [rows, D] as doubles (D a multiple of 32). */
int oracle_mxfp4_decode(const uint8_t* codes, const uint8_t* scales, int64_t rows, int64_t D, double* out) {
  if (rows < 0 || D <= 0 || D % 32 != 0) return -1;
  for (int64_t r = 0; r < rows; ++r)
    for (int64_t d = 0; d < D; ++d) out[r * D + d] = mxfp4_value(codes, scales, r, D, d);
  return 0;
}

/* e4m3 q [B,S,H,D] with q_scale [B,S,H]; e4m3 kc [B,T,D] with kc_scale [B,T];
 * each value dequantised as code value * its row's scale. */
int oracle_topk_e4m3(const uint8_t* q, const float* q_scale, const uint8_t* kc,
                     const float* kc_scale, const float* w, int64_t B, int64_t S, int64_t T,
                     int64_t H, int64_t D, int64_t m, int64_t k, const int64_t* rows,
                     int64_t n_rows, int32_t* out_idx, float* out_score, double* out_score64) {
  problem_t p = {1, q, q_scale, kc, kc_scale, w, B, S, T, H, D, m, NULL};
  return topk_rows(&p, k, rows, n_rows, out_idx, out_score, out_score64);
}

/*
 * Two-stage indexer (the V4.1-Flash indexer as the deployment notes describe
 * it, "two-level sparse attention", indexer section: a cheap candidate stage
 * first picks blocks of compressed keys -- 2048 blocks of 8 -- then the best
 * keys among the candidates are kept).  The pages do not say how a block is
 * scored; this oracle takes the plainest reading:
 *   - block j of a sequence is keys jG .. jG+G-1 (nb = floor(T/G) blocks);
 *   - its pooled key is the mean of its G keys rounded once to bf16 (nearest
 *     even);
 *   - the coarse score of block j for query t is the indexer score of the
 *     pooled key; only complete visible blocks compete (jG+G-1 < n(t));
 *   - the best n_keep blocks by (coarse score desc, block index asc) are
 *     kept, all of them when fewer compete;
 *   - the candidates are the keys of the kept blocks plus the visible keys
 *     of the incomplete last block (n(t) mod G of them);
 *   - the result is the top-k of the candidates by (indexer score desc, key
 *     index asc), padded as the one-stage result.
 * With at most n_keep complete visible blocks, every visible key is a
 * candidate and the result is the one-stage top-k.
 */

/* Round to the nearest bf16 (ties to even), from double, for normal values. */
static double round_bf16(double x) {
  if (x == 0.0 || !isfinite(x)) return x;
  int e;
  frexp(x, &e);                 /* |x| = f * 2^e, f in [0.5, 1) */
  double u = ldexp(1.0, e - 8); /* one unit in the 8th significant bit */
  return nearbyint(x / u) * u;  /* default rounding mode: ties to even */
}

/* Pooled keys of sequence b: nb rows of D doubles (bf16 values). */
static void pooled_keys(const problem_t* p, int64_t b, int64_t G, int64_t nb, double* pool, double* krow) {
  for (int64_t j = 0; j < nb; ++j) {
    for (int64_t d = 0; d < p->D; ++d) pool[j * p->D + d] = 0.0;
    for (int64_t i = 0; i < G; ++i) {
      widen_key(p, b, j * G + i, krow);
      for (int64_t d = 0; d < p->D; ++d) pool[j * p->D + d] += krow[d];
    }
    for (int64_t d = 0; d < p->D; ++d) pool[j * p->D + d] = round_bf16(pool[j * p->D + d] / (double)G);
  }
}

int oracle_pool_keys_bf16(const uint16_t* kc, int64_t B, int64_t T, int64_t D, int64_t G, double* out) {
  if (B <= 0 || T <= 0 || D <= 0 || G <= 0) return -1;
  problem_t p = {0, NULL, NULL, kc, NULL, NULL, B, 1, T, 1, D, 1, NULL};
  double* krow = (double*)malloc(sizeof(double) * (size_t)D);
  if (!krow) return -2;
  int64_t nb = T / G;
  for (int64_t b = 0; b < B; ++b) pooled_keys(&p, b, G, nb, out + b * nb * D, krow);
  free(krow);
  return 0;
}

int oracle_topk_two_stage_bf16(const uint16_t* q, const uint16_t* kc, const float* w, int64_t B, int64_t S,
                               int64_t T, int64_t H, int64_t D, int64_t m, int64_t k, int64_t G,
                               int64_t n_keep, const int64_t* rows, int64_t n_rows, int32_t* out_idx,
                               float* out_score, double* out_score64) {
  if (B <= 0 || S <= 0 || T <= 0 || H <= 0 || D <= 0 || m <= 0 || k <= 0 || G <= 0 || n_keep <= 0) return -1;
  problem_t p = {0, q, NULL, kc, NULL, w, B, S, T, H, D, m, NULL};
  const int64_t nb = T / G;
  double* qrow = (double*)malloc(sizeof(double) * (size_t)(H * D));
  double* wrow = (double*)malloc(sizeof(double) * (size_t)H);
  double* krow = (double*)malloc(sizeof(double) * (size_t)D);
  double* dot = (double*)malloc(sizeof(double) * (size_t)H);
  double* pool = (double*)malloc(sizeof(double) * (size_t)((nb > 0 ? nb : 1) * D));
  cand_t* blk = (cand_t*)malloc(sizeof(cand_t) * (size_t)(nb > 0 ? nb : 1));
  cand_t* c = (cand_t*)malloc(sizeof(cand_t) * (size_t)T);
  int rc = 0;
  int64_t pooled_b = -1;
  if (!qrow || !wrow || !krow || !dot || !pool || !blk || !c) rc = -2;
  for (int64_t i = 0; rc == 0 && i < n_rows; ++i) {
    int64_t r = rows[i];
    if (r < 0 || r >= B * S) { rc = -1; break; }
    int64_t b = r / S, t = r % S;
    if (b != pooled_b) {
      pooled_keys(&p, b, G, nb, pool, krow);
      pooled_b = b;
    }
    int64_t n = oracle_visible_count(t, T, m);
    int64_t nbv = n / G;
    widen_query(&p, b, t, qrow, wrow);
    /* coarse stage over the complete visible blocks */
    for (int64_t j = 0; j < nbv; ++j) {
      blk[j].score = score_rows(qrow, pool + j * D, wrow, (int)H, (int)D, dot);
      blk[j].idx = j;
    }
    qsort(blk, (size_t)nbv, sizeof(cand_t), cand_cmp);
    int64_t kept = nbv < n_keep ? nbv : n_keep;
    /* fine stage over the kept blocks' keys and the incomplete block's visible keys */
    int64_t nc = 0;
    for (int64_t j = 0; j < kept; ++j)
      for (int64_t e = 0; e < G; ++e) c[nc++].idx = blk[j].idx * G + e;
    for (int64_t s = nbv * G; s < n; ++s) c[nc++].idx = s;
    for (int64_t x = 0; x < nc; ++x) {
      widen_key(&p, b, c[x].idx, krow);
      c[x].score = score_rows(qrow, krow, wrow, (int)H, (int)D, dot);
    }
    qsort(c, (size_t)nc, sizeof(cand_t), cand_cmp);
    for (int64_t j = 0; j < k; ++j) {
      int64_t o = i * k + j;
      if (j < nc) {
        out_idx[o] = (int32_t)c[j].idx;
        if (out_score) out_score[o] = (float)c[j].score;
        if (out_score64) out_score64[o] = c[j].score;
      } else {
        out_idx[o] = -1;
        if (out_score) out_score[o] = -INFINITY;
        if (out_score64) out_score64[o] = -INFINITY;
      }
    }
  }
  free(qrow); free(wrow); free(krow); free(dot); free(pool); free(blk); free(c);
  return rc;
}

/*
 * Sparse attention over the selected compressed entries: the consumer of the
 * indexer's top-k in the CSA pipeline (StreamIndex abstract: a sparse
 * attention kernel reads only the selected entries).  The pages give no
 * dimensions for it; the reading follows the DeepSeek-V3.2 lineage they
 * name: every head of query t attends over the compressed latents idx[t, j]
 * (index -1 = padding, skipped), each latent serving as key (all Dk values)
 * and as value (its first Dv values):
 *   o[t,h,:] = sum_j p_j kv[idx_j, :Dv],  p = softmax_j(scale * q[t,h,:] . kv[idx_j, :])
 * and lse[t,h] = log sum_j exp(scale * logit_j) (-inf and o = 0 when no
 * entry is valid).  fp64 throughout; the maximum logit is subtracted before
 * exponentiating.
 *   q [B,S,H,Dk] bf16, kv [B,T,Dk] bf16, idx [B,S,k] int32; out [B,S,H,Dv]
 *   and lse [B,S,H] double.  Returns 0, -1 on a bad argument or index.
 */
int oracle_sparse_attention_bf16(const uint16_t* q, const uint16_t* kv, const int32_t* idx, int64_t B,
                                 int64_t S, int64_t T, int64_t H, int64_t Dk, int64_t Dv, int64_t k,
                                 double scale, double* out, double* lse) {
  if (B <= 0 || S <= 0 || T <= 0 || H <= 0 || Dk <= 0 || Dv <= 0 || Dv > Dk || k <= 0) return -1;
  double* logit = (double*)malloc(sizeof(double) * (size_t)k);
  if (!logit) return -2;
  int rc = 0;
  for (int64_t b = 0; b < B && rc == 0; ++b)
    for (int64_t t = 0; t < S && rc == 0; ++t) {
      const int32_t* sel = idx + (b * S + t) * k;
      for (int64_t j = 0; j < k; ++j)
        if (sel[j] < -1 || sel[j] >= T) rc = -1;
      if (rc) break;
      for (int64_t h = 0; h < H; ++h) {
        const uint16_t* qh = q + ((b * S + t) * H + h) * Dk;
        double* o = out + ((b * S + t) * H + h) * Dv;
        double mx = -INFINITY;
        for (int64_t j = 0; j < k; ++j) {
          if (sel[j] < 0) continue;
          const uint16_t* kr = kv + (b * T + sel[j]) * Dk;
          double dot = 0.0;
          for (int64_t d = 0; d < Dk; ++d) dot += oracle_bf16_value(qh[d]) * oracle_bf16_value(kr[d]);
          logit[j] = scale * dot;
          if (logit[j] > mx) mx = logit[j];
        }
        for (int64_t d = 0; d < Dv; ++d) o[d] = 0.0;
        if (mx == -INFINITY) {
          lse[(b * S + t) * H + h] = -INFINITY;
          continue;
        }
        double den = 0.0;
        for (int64_t j = 0; j < k; ++j) {
          if (sel[j] < 0) continue;
          const double e = exp(logit[j] - mx);
          den += e;
          const uint16_t* vr = kv + (b * T + sel[j]) * Dk;
          for (int64_t d = 0; d < Dv; ++d) o[d] += e * oracle_bf16_value(vr[d]);
        }
        for (int64_t d = 0; d < Dv; ++d) o[d] /= den;
        lse[(b * S + t) * H + h] = mx + log(den);
      }
    }
  free(logit);
  return rc;
}

/* All T scores of one row (bf16 inputs) in double; invisible keys get NaN.
 * For brute-force and invariant tests on small inputs. */
int oracle_scores_bf16(const uint16_t* q, const uint16_t* kc, const float* w, int64_t B, int64_t S,
                       int64_t T, int64_t H, int64_t D, int64_t m, int64_t row, double* out) {
  problem_t p = {0, q, NULL, kc, NULL, w, B, S, T, H, D, m, NULL};
  if (row < 0 || row >= B * S) return -1;
  double* qrow = (double*)malloc(sizeof(double) * (size_t)(H * D));
  double* wrow = (double*)malloc(sizeof(double) * (size_t)H);
  double* krow = (double*)malloc(sizeof(double) * (size_t)D);
  double* dot = (double*)malloc(sizeof(double) * (size_t)H);
  if (!qrow || !wrow || !krow || !dot) { free(qrow); free(wrow); free(krow); free(dot); return -2; }
  int64_t b = row / S, t = row % S, n = oracle_visible_count(t, T, m);
  widen_query(&p, b, t, qrow, wrow);
  for (int64_t s = 0; s < T; ++s) {
    if (s < n) { widen_key(&p, b, s, krow); out[s] = score_rows(qrow, krow, wrow, (int)H, (int)D, dot); }
    else out[s] = NAN;
  }
  free(qrow); free(wrow); free(krow); free(dot);
  return 0;
}

/*
 * flashhead_oracle.c — TEST INFRASTRUCTURE, not part of the product.
 *
 * A plain, slow, obviously correct CPU restatement of the FlashHead head in float64 arithmetic.
 * Only the tests, the smoke check and the benchmark's CPU-baseline leg call it.  It shares no code,
 * header, table or helper with the CUDA library, and the CUDA library never calls it.
 *
 * Every stored value (fp32 or BF16) is widened exactly to double before use; all sums, logarithms
 * and exponentials are done in double.  Selection uses a full sort; arg-maxima use a linear scan
 * with the explicit tie rule.  Steps follow the pages in their order:
 *
 *   "FlashHead notes" = the reading-notes page "FlashHead: Efficient Drop-In Replacement for the
 *   Classification Head in Language Model Inference"; "FlashHead summary" = the paper-summary page
 *   of the same title.
 *
 *   1. Stage 1 scores s = C·h                      (FlashHead notes, overall architecture, Figure 1)
 *   2. p clusters: top-p (greedy) or Gumbel-top-p  (FlashHead notes, Module 2)
 *   3. candidates = tokens of the chosen clusters   (FlashHead notes, Module 1: dense C2T)
 *   4. exact logits z_t = E[t]·h                     (FlashHead notes, Eq. 1 and Figure 1 Stage 2)
 *   5. argmax (Eq. 2) or softmax(z/τ) draw (Eq. 3) over the candidates
 *   6. Monte Carlo marginal over N Stage-1 draws     (FlashHead notes, Module 4 and Eq. 7)
 *   7. dense head over all v tokens                  (FlashHead notes, Eq. 1–3)
 *
 * Readings where the pages are silent (they are the repository's specification):
 *   - clusters are ordered by (score desc, id asc), tokens by (logit desc, id asc);
 *   - the returned probe set is in ascending cluster id, candidates in slot order r*b + j;
 *   - sampling without replacement is realised as Gumbel-top-p, token sampling as Gumbel-max;
 *   - random numbers are Philox4x32-10 words with the counter layout of orc_draw_u32, mapped to
 *     u = ((x >> 9) + 0.5) * 2^-23 (exact in fp32 as well) and G = -log(-log u);
 *   - p(t|h,S) = 0 for a token outside the candidates of S; the standard error is the sample
 *     standard deviation (N-1 denominator) over sqrt(N).
 *
 * Parity pins live in tests/test_oracle_pins.py.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORC_F32 0
#define ORC_BF16 1

/* ------------------------------------------------------------------ stored values ---------- */

static double bf16_bits_to_double(uint16_t bits) {
  uint32_t w = (uint32_t)bits << 16;
  float f;
  memcpy(&f, &w, sizeof f);
  return (double)f;
}

/* Element i of a stored array (fp32 values or BF16 patterns), widened exactly. */
static double stored_at(const void* base, int dtype, int64_t i) {
  if (dtype == ORC_F32) return (double)((const float*)base)[i];
  return bf16_bits_to_double(((const uint16_t*)base)[i]);
}

/* INT4 centroid value (FlashHead notes, Module 3, selective quantisation of Stage 1):
   q in two's complement, low nibble = even column; value = q * scale of its 32-column group. */
static double int4_centroid_at(const uint8_t* q4, const uint16_t* scales, int64_t d, int64_t k,
                               int64_t j) {
  uint8_t byte = q4[k * (d / 2) + j / 2];
  int nib = (j % 2 == 0) ? (byte & 0xF) : (byte >> 4);
  int q = (nib >= 8) ? nib - 16 : nib;
  double scale = bf16_bits_to_double(scales[k * (d / 32) + j / 32]);
  return (double)q * scale;
}

/* ------------------------------------------------------------------ Philox4x32-10 ---------- */
/* Salmon, Moraes, Dror, Shaw, "Parallel random numbers: as easy as 1, 2, 3" (SC'11): ten rounds of
   the 4x32 Philox S-box; the round multipliers are 0xD2511F53 and 0xCD9E8D57, the key is bumped by
   the Weyl constants 0x9E3779B9 and 0xBB67AE85 between rounds. */

void orc_philox4x32_10(const uint32_t ctr_in[4], const uint32_t key_in[2], uint32_t out[4]) {
  uint32_t x0 = ctr_in[0], x1 = ctr_in[1], x2 = ctr_in[2], x3 = ctr_in[3];
  uint32_t k0 = key_in[0], k1 = key_in[1];
  for (int round = 0; round < 10; ++round) {
    if (round > 0) {
      k0 += 0x9E3779B9u;
      k1 += 0xBB67AE85u;
    }
    uint64_t prod_a = (uint64_t)0xD2511F53u * (uint64_t)x0;
    uint64_t prod_b = (uint64_t)0xCD9E8D57u * (uint64_t)x2;
    uint32_t hi_a = (uint32_t)(prod_a >> 32), lo_a = (uint32_t)prod_a;
    uint32_t hi_b = (uint32_t)(prod_b >> 32), lo_b = (uint32_t)prod_b;
    uint32_t y0 = hi_b ^ x1 ^ k0;
    uint32_t y1 = lo_b;
    uint32_t y2 = hi_a ^ x3 ^ k1;
    uint32_t y3 = lo_a;
    x0 = y0; x1 = y1; x2 = y2; x3 = y3;
  }
  out[0] = x0; out[1] = x1; out[2] = x2; out[3] = x3;
}

/* The repository's counter layout: key = (seed lo, seed hi); counter = (elem >> 2, row, step lo,
   (stream << 24) | (step hi & 0xFFFFFF)); the draw is output word (elem & 3). */
uint32_t orc_draw_u32(uint64_t seed, uint64_t step, uint32_t row, uint32_t stream, uint64_t elem) {
  uint32_t key[2] = {(uint32_t)seed, (uint32_t)(seed >> 32)};
  uint32_t ctr[4] = {(uint32_t)(elem >> 2), row, (uint32_t)step,
                     (stream << 24) | ((uint32_t)(step >> 32) & 0xFFFFFFu)};
  uint32_t out[4];
  orc_philox4x32_10(ctr, key, out);
  return out[elem & 3];
}

void orc_philox_words(uint64_t seed, uint64_t step, uint32_t row, uint32_t stream, int64_t n,
                      uint32_t* out) {
  for (int64_t e = 0; e < n; ++e) out[e] = orc_draw_u32(seed, step, row, stream, (uint64_t)e);
}

/* u = ((x >> 9) + 0.5) * 2^-23 lies strictly inside (0, 1) and has at most 24 significant bits, so
   an fp32 implementation can form it exactly too; G = -log(-log u) is a standard Gumbel variate.
   Both logarithms in double. */
double orc_uniform(uint32_t x) { return ((double)(x >> 9) + 0.5) * (1.0 / 8388608.0); }

double orc_gumbel(uint32_t x) { return -log(-log(orc_uniform(x))); }

/* ------------------------------------------------------------------ Stage 1 ---------------- */

/* s[q][k] = Σ_j C[k][j] · H[q][j]  (FlashHead notes, overall architecture: Stage 1 scores h against
   the c centroids).  s1_fmt 0 reads C; s1_fmt 1 reads the INT4 centroids and their BF16 scales. */
void orc_stage1_scores(const void* C, int dtype, const uint8_t* q4, const uint16_t* scales,
                       int s1_fmt, int64_t c, int64_t d, const void* H, int B, double* s) {
#pragma omp parallel for collapse(2) schedule(static)
  for (int q = 0; q < B; ++q) {
    for (int64_t k = 0; k < c; ++k) {
      double acc = 0.0;
      for (int64_t j = 0; j < d; ++j) {
        double ckj = (s1_fmt == 1) ? int4_centroid_at(q4, scales, d, k, j)
                                   : stored_at(C, dtype, k * d + j);
        acc += ckj * stored_at(H, dtype, (int64_t)q * d + j);
      }
      s[(int64_t)q * c + k] = acc;
    }
  }
}

/* key[q][k] = s[q][k] / τ + G(seed, step, q, stream, k)  (FlashHead notes, Module 2 sampling mode:
   softmax-scaled centroid logits; the Gumbel perturbation turns top-p into sampling without
   replacement). */
void orc_gumbel_keys(const double* s, int B, int64_t c, double tau, uint64_t seed, uint64_t step,
                     uint32_t stream, double* keys) {
  for (int q = 0; q < B; ++q)
    for (int64_t k = 0; k < c; ++k)
      keys[(int64_t)q * c + k] =
          s[(int64_t)q * c + k] / tau + orc_gumbel(orc_draw_u32(seed, step, (uint32_t)q, stream,
                                                                (uint64_t)k));
}

/* ------------------------------------------------------------------ selection -------------- */

typedef struct {
  double key;
  int64_t id;
} keyed_t;

/* (key desc, id asc); -0.0 and +0.0 compare equal under C's <, as required. */
static int cmp_key_desc_id_asc(const void* pa, const void* pb) {
  const keyed_t* a = (const keyed_t*)pa;
  const keyed_t* b = (const keyed_t*)pb;
  if (a->key > b->key) return -1;
  if (a->key < b->key) return 1;
  return (a->id < b->id) ? -1 : (a->id > b->id) ? 1 : 0;
}

static int cmp_i32_asc(const void* pa, const void* pb) {
  int32_t a = *(const int32_t*)pa, b = *(const int32_t*)pb;
  return (a > b) - (a < b);
}

/* Top-p of one row of keys by full sort (FlashHead notes, Module 2: the p clusters with the highest
   centroid logits).  sel receives the p ids in ascending order.  margin (if not NULL) receives
   key_(p) - key_(p+1) of the sorted keys (+inf when p == c). */
static void select_row(const double* keys, int64_t c, int p, int32_t* sel, double* margin,
                       keyed_t* scratch) {
  for (int64_t k = 0; k < c; ++k) {
    scratch[k].key = keys[k];
    scratch[k].id = k;
  }
  qsort(scratch, (size_t)c, sizeof(keyed_t), cmp_key_desc_id_asc);
  for (int r = 0; r < p; ++r) sel[r] = (int32_t)scratch[r].id;
  qsort(sel, (size_t)p, sizeof(int32_t), cmp_i32_asc);
  if (margin) *margin = (p < c) ? scratch[p - 1].key - scratch[p].key : INFINITY;
}

void orc_select_topp(const double* keys, int B, int64_t c, int p, int32_t* sel, double* margin) {
#pragma omp parallel
  {
    keyed_t* scratch = (keyed_t*)malloc(sizeof(keyed_t) * (size_t)c);
#pragma omp for schedule(static)
    for (int q = 0; q < B; ++q)
      select_row(keys + (int64_t)q * c, c, p, sel + (int64_t)q * p, margin ? margin + q : NULL,
                 scratch);
    free(scratch);
  }
}

/* ------------------------------------------------------------------ Stage 2 ---------------- */

/* Candidate slot r*b + j holds C2T[S[r]][j] (FlashHead notes, Module 1: a dense c×b C2T turns the
   gather into index arithmetic). */
void orc_gather(const int32_t* C2T, int64_t b, const int32_t* sel, int B, int p, int32_t* cand) {
  for (int q = 0; q < B; ++q)
    for (int r = 0; r < p; ++r)
      for (int64_t j = 0; j < b; ++j)
        cand[((int64_t)q * p + r) * b + j] = C2T[(int64_t)sel[(int64_t)q * p + r] * b + j];
}

/* z = E[t]·h for each listed token (FlashHead notes, Eq. 1 restricted to the candidates). */
static double row_dot(const void* E, int dtype, int64_t d, int64_t t, const void* H, int q) {
  double acc = 0.0;
  for (int64_t j = 0; j < d; ++j)
    acc += stored_at(E, dtype, t * d + j) * stored_at(H, dtype, (int64_t)q * d + j);
  return acc;
}

void orc_logits(const void* E, int dtype, int64_t d, const void* H, int B, const int32_t* cand,
                int64_t P, double* z) {
#pragma omp parallel for collapse(2) schedule(static)
  for (int q = 0; q < B; ++q)
    for (int64_t i = 0; i < P; ++i)
      z[(int64_t)q * P + i] = row_dot(E, dtype, d, cand[(int64_t)q * P + i], H, q);
}

/* Arg-max of val over n entries under (value desc, id asc) (FlashHead notes, Eq. 2).  Returns the
   winning position; *gap receives best - runner-up (+inf when n == 1). */
static int64_t argmax_pos(const double* val, const int32_t* ids, int64_t n, double* gap) {
  int64_t best = 0;
  for (int64_t i = 1; i < n; ++i)
    if (val[i] > val[best] || (val[i] == val[best] && ids[i] < ids[best])) best = i;
  double second = -INFINITY;
  for (int64_t i = 0; i < n; ++i)
    if (i != best && val[i] > second) second = val[i];
  if (gap) *gap = (n > 1) ? val[best] - second : INFINITY;
  return best;
}

/* The whole head for B queries.  sample == 0: greedy (Module 2 greedy mode, Eq. 2).  sample != 0:
   Stage 1 keys s/τ + G(seed, step, q, 0, k), Stage-2 keys z/τ + G(seed, step, q, 1, t) (Module 2
   sampling mode, Eq. 3).  Outputs (any may be NULL except tok):
     tok[B]                 chosen token ids
     sel[B*p]               probe sets, ascending
     cand[B*P], z[B*P]      candidate token ids in slot order and their exact logits
     dec[B*P]               decision keys (z for greedy, z/τ + G' for sampling)
     set_margin[B]          key_(p) - key_(p+1) of the Stage-1 keys
     tok_margin[B]          best - runner-up of the decision keys */
void orc_head(const void* E, const void* C, int dtype, const uint8_t* q4, const uint16_t* scales,
              int s1_fmt, const int32_t* C2T, int64_t v, int64_t d, int64_t c, int64_t b,
              const void* H, int B, int p, int sample, double tau, uint64_t seed, uint64_t step,
              int32_t* tok, int32_t* sel_out, int32_t* cand_out, double* z_out, double* dec_out,
              double* set_margin, double* tok_margin) {
  (void)v;
  int64_t P = (int64_t)p * b;
  double* s = (double*)malloc(sizeof(double) * (size_t)(B * c));
  double* keys = (double*)malloc(sizeof(double) * (size_t)(B * c));
  int32_t* sel = (int32_t*)malloc(sizeof(int32_t) * (size_t)(B * p));
  int32_t* cand = (int32_t*)malloc(sizeof(int32_t) * (size_t)(B * P));
  double* z = (double*)malloc(sizeof(double) * (size_t)(B * P));
  double* dec = (double*)malloc(sizeof(double) * (size_t)(B * P));

  orc_stage1_scores(C, dtype, q4, scales, s1_fmt, c, d, H, B, s);                 /* step 1 */
  if (sample)
    orc_gumbel_keys(s, B, c, tau, seed, step, 0u, keys);                           /* step 2 */
  else
    memcpy(keys, s, sizeof(double) * (size_t)(B * c));
  orc_select_topp(keys, B, c, p, sel, set_margin);
  orc_gather(C2T, b, sel, B, p, cand);                                             /* step 3 */
  orc_logits(E, dtype, d, H, B, cand, P, z);                                       /* step 4 */
  for (int q = 0; q < B; ++q) {                                                    /* step 5 */
    for (int64_t i = 0; i < P; ++i) {
      int64_t at = (int64_t)q * P + i;
      dec[at] = sample ? z[at] / tau + orc_gumbel(orc_draw_u32(seed, step, (uint32_t)q, 1u,
                                                               (uint64_t)cand[at]))
                       : z[at];
    }
    int64_t pos = argmax_pos(dec + (int64_t)q * P, cand + (int64_t)q * P, P,
                             tok_margin ? tok_margin + q : NULL);
    tok[q] = cand[(int64_t)q * P + pos];
  }
  if (sel_out) memcpy(sel_out, sel, sizeof(int32_t) * (size_t)(B * p));
  if (cand_out) memcpy(cand_out, cand, sizeof(int32_t) * (size_t)(B * P));
  if (z_out) memcpy(z_out, z, sizeof(double) * (size_t)(B * P));
  if (dec_out) memcpy(dec_out, dec, sizeof(double) * (size_t)(B * P));
  free(s); free(keys); free(sel); free(cand); free(z); free(dec);
}

/* ------------------------------------------------------------------ dense head ------------- */

/* z over all v tokens, then argmax or Gumbel-max with stream 1 keyed by token id (FlashHead notes,
   Eq. 1–3).  z_out (v per query) and tok_margin may be NULL. */
void orc_dense(const void* E, int dtype, int64_t v, int64_t d, const void* H, int B, int sample,
               double tau, uint64_t seed, uint64_t step, int32_t* tok, double* z_out,
               double* tok_margin) {
  int32_t* ids = (int32_t*)malloc(sizeof(int32_t) * (size_t)v);
  for (int64_t t = 0; t < v; ++t) ids[t] = (int32_t)t;
  double* z = (double*)malloc(sizeof(double) * (size_t)v);
  double* dec = (double*)malloc(sizeof(double) * (size_t)v);
  for (int q = 0; q < B; ++q) {
#pragma omp parallel for schedule(static)
    for (int64_t t = 0; t < v; ++t) {
      z[t] = row_dot(E, dtype, d, t, H, q);
      dec[t] = sample ? z[t] / tau + orc_gumbel(orc_draw_u32(seed, step, (uint32_t)q, 1u,
                                                              (uint64_t)t))
                      : z[t];
    }
    tok[q] = (int32_t)argmax_pos(dec, ids, v, tok_margin ? tok_margin + q : NULL);
    if (z_out) memcpy(z_out + (int64_t)q * v, z, sizeof(double) * (size_t)v);
  }
  free(ids); free(z); free(dec);
}

/* ------------------------------------------------------------------ Monte Carlo ------------ */

/* Marginal token probability (FlashHead notes, Module 4 and Eq. 7): for draws i = i0..i1-1,
   S_i = Gumbel-top-p of s/τ + G(seed, i, q, 2, k); the candidate set is the tokens of S_i; the
   conditional probability of target t is its softmax(z/τ) weight among the candidates, summed
   literally over the candidate tokens of that draw, or 0 when t is not a candidate.
   per_draw[(q*(i1-i0) + (i-i0))*T + j] receives p_i(targets[q*T + j]).
   mean/se over draws [i0, i1) are written when not NULL (se: sample sd over sqrt(count)). */
void orc_mc(const void* E, const void* C, int dtype, const uint8_t* q4, const uint16_t* scales,
            int s1_fmt, const int32_t* C2T, int64_t v, int64_t d, int64_t c, int64_t b,
            const void* H, int B, const int32_t* targets, int T, int p, double tau, int64_t i0,
            int64_t i1, uint64_t seed, double* per_draw, double* mean, double* se) {
  int64_t n = i1 - i0;
  double* s = (double*)malloc(sizeof(double) * (size_t)(B * c));
  orc_stage1_scores(C, dtype, q4, scales, s1_fmt, c, d, H, B, s);
  double* z = (double*)malloc(sizeof(double) * (size_t)v);
  double* pd = per_draw ? per_draw : (double*)malloc(sizeof(double) * (size_t)(B * n * T));
  for (int q = 0; q < B; ++q) {
#pragma omp parallel for schedule(static)
    for (int64_t t = 0; t < v; ++t) z[t] = row_dot(E, dtype, d, t, H, q);   /* S-independent */
#pragma omp parallel
    {
      double* keys = (double*)malloc(sizeof(double) * (size_t)c);
      keyed_t* scratch = (keyed_t*)malloc(sizeof(keyed_t) * (size_t)c);
      int32_t* sel = (int32_t*)malloc(sizeof(int32_t) * (size_t)p);
      unsigned char* is_cand = (unsigned char*)malloc((size_t)v);
#pragma omp for schedule(static)
      for (int64_t i = i0; i < i1; ++i) {
        for (int64_t k = 0; k < c; ++k)
          keys[k] = s[(int64_t)q * c + k] / tau +
                    orc_gumbel(orc_draw_u32(seed, (uint64_t)i, (uint32_t)q, 2u, (uint64_t)k));
        select_row(keys, c, p, sel, NULL, scratch);
        memset(is_cand, 0, (size_t)v);
        double m = -INFINITY;
        for (int r = 0; r < p; ++r)
          for (int64_t j = 0; j < b; ++j) {
            int32_t t = C2T[(int64_t)sel[r] * b + j];
            is_cand[t] = 1;
            if (z[t] / tau > m) m = z[t] / tau;
          }
        double denom = 0.0;
        for (int r = 0; r < p; ++r)
          for (int64_t j = 0; j < b; ++j) denom += exp(z[C2T[(int64_t)sel[r] * b + j]] / tau - m);
        for (int jt = 0; jt < T; ++jt) {
          int32_t t = targets[(int64_t)q * T + jt];
          pd[((int64_t)q * n + (i - i0)) * T + jt] = is_cand[t] ? exp(z[t] / tau - m) / denom : 0.0;
        }
      }
      free(keys); free(scratch); free(sel); free(is_cand);
    }
  }
  if (mean || se) {
    for (int q = 0; q < B; ++q)
      for (int jt = 0; jt < T; ++jt) {
        double sum = 0.0;
        for (int64_t i = 0; i < n; ++i) sum += pd[((int64_t)q * n + i) * T + jt];
        double mu = sum / (double)n;
        double ss = 0.0;
        for (int64_t i = 0; i < n; ++i) {
          double dlt = pd[((int64_t)q * n + i) * T + jt] - mu;
          ss += dlt * dlt;
        }
        if (mean) mean[q * T + jt] = mu;
        if (se) se[q * T + jt] = (n > 1) ? sqrt(ss / (double)(n - 1)) / sqrt((double)n) : 0.0;
      }
  }
  if (!per_draw) free(pd);
  free(s); free(z);
}

/* Threads for the next parallel regions (n >= 1; no effect without OpenMP). */
void orc_set_num_threads(int n) {
#ifdef _OPENMP
  extern void omp_set_num_threads(int);
  if (n >= 1) omp_set_num_threads(n);
#else
  (void)n;
#endif
}

/* Number of threads the OpenMP runtime will use (1 without OpenMP). */
int orc_num_threads(void) {
#ifdef _OPENMP
  extern int omp_get_max_threads(void);
  return omp_get_max_threads();
#else
  return 1;
#endif
}

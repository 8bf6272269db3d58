/*
 * fh_kmeans.h — C ABI of the FlashHead index builder: equal-size spherical k-means on B200.
 *
 * What it computes (FlashHead notes, Module 1 "equal-size spherical K-Means", Eq.4 and Eq.5, and
 * the implementation details: c clusters of exactly b = v/c tokens, up to 1000 iterations):
 *   Eq.4  minimise -sum_i cos(e_i, c_k(i)) over labelings with exactly b tokens per cluster;
 *   Eq.5  each centre is the L2-normalised mean of its members.
 * Following Dhillon & Modha's spherical k-means (which the notes cite), rows are compared by
 * direction: x_i = e_i / |e_i|, and Eq.5 averages the x_i.  One iteration is
 *   assignment  the equal-size labeling that maximises sum_i x_i . c_k(i) for the current centres,
 *               within v*eps of the optimum (an eps-scaled auction for the transportation
 *               problem, Bertsekas & Castanon 1989; every result carries prices that certify it);
 *   update      Eq.5, after which the objective of Eq.4 is -sum_k |sum_{i in k} x_i|.
 * The similarities x_i . c_k are computed on the tensor cores from the stored BF16 rows of E and
 * the centres rounded to BF16 (the precision the head's Stage 1 reads them in), accumulated in
 * fp32.  The run stops when an assignment repeats the previous labels or after `iters` iterations.
 *
 * The outputs are a FlashHead index: C (c x d unit rows) and C2T (c x b, row k = the tokens of
 * cluster k in ascending id order), ready for fh_index_load (include/flashhead.h).
 *
 * Conventions (as in flashhead.h).  Pointers marked "device" are CUDA device memory owned by the
 * caller.  Matrices are dense row-major; BF16 values are 16-bit patterns.  Unlike the head calls,
 * these calls SYNCHRONISE the stream: the auction reads back the number of unassigned tokens after
 * every round.  Argument errors are returned before any launch; a device-side finding (a zero row,
 * an init token out of range or repeated, labels that are not equal-size, a cluster whose members
 * sum to zero) returns FH_ERR_ARG with a message; exceeding max_rounds returns FH_ERR_TIMEOUT.
 * fh_last_error() describes the last failure.  The workspace is device scratch of
 * fh_kmeans_ws_bytes(v, d, c) bytes, 256-byte aligned; it holds the v x c fp32 similarity matrix.
 */
#ifndef FH_KMEANS_H
#define FH_KMEANS_H

#include "flashhead.h"

#ifdef __cplusplus
extern "C" {
#endif

/* Limits of the builder: 1 <= c <= FH_MAX_C, c divides v, v < 2^31, d a multiple of 8 up to
   FH_MAX_D, E in BF16; 1e-5 <= eps <= 0.25. */

typedef struct {
  const void* E;               /* device, v x d, BF16: the token embeddings */
  int32_t dtype;               /* must be FH_BF16 */
  int64_t v, d, c;             /* tokens, hidden size, clusters */
  int32_t iters;               /* iterations, >= 1 */
  float eps;                   /* auction tolerance of the last scaling phase */
  int64_t max_rounds;          /* bound on auction rounds over the call; 0 = 1<<22 */
  const int32_t* init_tokens;  /* device, c distinct token ids: initial centres c_k = x_init[k]
                                  (fh_kmeans_build only) */
  const uint16_t* C_in;        /* device, c x d BF16 centres to assign against
                                  (fh_kmeans_assign only) */
  const int32_t* labels_in;    /* device, v labels in [0, c), b per cluster (fh_kmeans_update only) */
  int32_t* labels;             /* device, v: out, cluster of each token (build, assign) */
  int32_t* C2T;                /* device, c x b: out, tokens of each cluster, ascending */
  float* C;                    /* device, c x d fp32: out, unit centres (build, update) */
  uint16_t* C_bf16;            /* device, c x d BF16 or NULL: out, C rounded to nearest even */
  double* objective;           /* device, iters doubles or NULL: Eq.4 after each update */
  float* prices;               /* device, c floats or NULL: out, prices of the last auction */
  int32_t iters_done;          /* out: updates performed */
  int64_t rounds;              /* out: auction rounds performed */
} fh_kmeans_args;

/* Device workspace bytes for v tokens of d columns in c clusters (0 when the sizes are invalid). */
size_t fh_kmeans_ws_bytes(int64_t v, int64_t d, int64_t c);

/* Equal-size spherical k-means from init_tokens: writes labels, C2T, C (and C_bf16, objective,
   prices when given), iters_done and rounds. */
fh_status fh_kmeans_build(fh_kmeans_args* args, void* ws, size_t ws_bytes, fh_stream stream);

/* The assignment half-step alone against the BF16 centres C_in: writes labels, C2T and prices
   (when given) and rounds.  The labels are equal-size and within v*eps of the best equal-size
   assignment for those centres; the prices certify it (every token's net value a_ik - price_k at
   its own cluster is within eps of its best net value). */
fh_status fh_kmeans_assign(fh_kmeans_args* args, void* ws, size_t ws_bytes, fh_stream stream);

/* The update half-step alone (Eq.5) for labels_in: writes C2T, C (and C_bf16, objective[0]). */
fh_status fh_kmeans_update(fh_kmeans_args* args, void* ws, size_t ws_bytes, fh_stream stream);

#ifdef __cplusplus
}
#endif

#endif /* FH_KMEANS_H */

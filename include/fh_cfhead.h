/*
 * fh_cfhead.h — C ABI of the coarse-fine LM head (CFHead) on B200 (sm_100a), a second workload of
 * the same library (libflashhead.so).
 *
 * What it computes (page "Fast LM Head via Coarse-Fine Decomposition and Tile-Wise Weight
 * Clustering", abstract): the head weights E ∈ R^{v×d} are represented offline by tile-wise k-means
 * as a compact codebook and an index map; at decode time coarse scores over the whole vocabulary are
 * computed from per-tile look-up tables and the streamed indices, and the exact product with the
 * original weights runs only on the top-k candidates.  The abstract fixes no parameter or layout;
 * this library reads it as follows:
 *   - the columns of E are cut into T = d / w tiles of w consecutive columns; tile t has a codebook
 *     Cb[t] of K <= 16 entries of w fp32 values, and every token u one 4-bit code I[u][t] < K per tile;
 *   - per query h: LUT[t][j] = Cb[t][j]·h[t·w .. t·w + w) (fp32, in column order);
 *   - coarse score ŝ_u = Σ_t LUT[t][I[u][t]] (fp32: four partial sums over the tiles t ≡ 0, 1, 2, 3
 *     (mod 4), each in tile order, then (s0 + s1) + (s2 + s3));
 *   - candidates = the k tokens with the largest coarse scores, ordered (score desc, token id asc);
 *   - exact logits z_u = E[u]·h (fp32 accumulation of BF16 products) for the candidates, and the
 *     token = arg-max of z (greedy) or of z/τ + G(seed, step, q, FH_RNG_STAGE2, u) (sampling: a
 *     softmax(z/τ) draw over the candidates by Gumbel-max), ties to the smaller token id.
 * The Philox stream, the Gumbel transform, the status codes, the stream and the ownership
 * conventions are those of flashhead.h.
 *
 * Index-map layout: uint32 words [T/8][v]; word (g, u) holds the codes of tiles 8g .. 8g+7 of token
 * u, tile 8g + j in bits 4j .. 4j+3 (so a warp reading 32 consecutive tokens of one word row reads
 * 128 contiguous bytes).
 */
#ifndef FH_CFHEAD_H
#define FH_CFHEAD_H

#include <stddef.h>
#include <stdint.h>

#include "flashhead.h"

#ifdef __cplusplus
extern "C" {
#endif

/* Limits of this build (k, the number of candidates, may be anything up to v). */
enum { FH_CF_MAX_K = 16 };

typedef struct fh_cf_index fh_cf_index;   /* opaque host-side handle */

/* Description of one coarse-fine index.  All pointers are device memory owned by the caller and must
   stay valid while the handle lives. */
typedef struct {
  int64_t v, d;              /* vocabulary and hidden size; d % (8*w) == 0, v < 2^24 */
  int32_t w;                 /* columns per tile, 1 <= w <= 64 */
  int32_t K;                 /* codebook entries per tile, 1 <= K <= FH_CF_MAX_K */
  const void* E;             /* device, v x d BF16 patterns (the original head weights) */
  const float* codebooks;    /* device, T x K x w fp32, T = d / w */
  const uint32_t* codes;     /* device, T/8 x v packed 4-bit codes (layout above) */
} fh_cf_desc;

/* Validate desc and create a handle (host metadata only; nothing is launched). */
fh_status fh_cf_load(const fh_cf_desc* desc, fh_cf_index** out);

/* Release a handle (host memory only).  NULL is ignored. */
void fh_cf_free(fh_cf_index* idx);

/* Device workspace bytes one fh_cf_head / fh_cf_coarse_scores call needs at batch B with k
   candidates (0 for invalid arguments).  256-byte aligned and zero-filled before first use; a call
   leaves it ready for the next call on the same stream.  fh_ws_status reads and clears its status
   word (its first 5120 bytes follow the same control-block convention as a FlashHead workspace). */
size_t fh_cf_workspace_bytes(const fh_cf_index* idx, int B, int k);

/* The coarse-fine head for B queries (1 <= B <= FH_MAX_BATCH, 1 <= k <= v).
   H: device, B x d BF16.  out_tok: device, B int32.  sample == 0: greedy; else tau > 0.
   dbg_cand: device B x k int32 or NULL — the candidate set of each query, in no particular order.
   dbg_coarse: device B x v fp32 or NULL — the coarse scores.  Asynchronous on `stream`. */
fh_status fh_cf_head(const fh_cf_index* idx, const void* H, int B, int k, int sample, float tau,
                     uint64_t seed, uint64_t step, int32_t* out_tok, void* ws, size_t ws_bytes,
                     fh_stream stream, int32_t* dbg_cand, float* dbg_coarse);

/* The coarse scores alone (the first step of fh_cf_head): out: device, B x v fp32. */
fh_status fh_cf_coarse_scores(const fh_cf_index* idx, const void* H, int B, float* out, void* ws,
                              size_t ws_bytes, fh_stream stream);

#ifdef __cplusplus
}
#endif

#endif /* FH_CFHEAD_H */

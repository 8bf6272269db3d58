/*
 * flashhead.h — C ABI of the FlashHead two-stage classification head on B200 (sm_100a).
 *
 * What the library computes.  The dense language-model head is z = E·h (E ∈ R^{v×d} token
 * embeddings, h ∈ R^d the last hidden vector, z ∈ R^v the logits; FlashHead notes, Eq. 1).
 * FlashHead replaces it by a retrieval in two stages (FlashHead notes, "overall architecture"
 * and Figure 1; FlashHead summary, Abstract and Figure 1):
 *   Stage 1  s = C·h over c unit-norm spherical-k-means centroids C ∈ R^{c×d}; keep p clusters —
 *            the p best for greedy decoding, or p drawn without replacement from softmax(s/τ)
 *            for sampling (FlashHead notes, Module 2 "multi-probe retrieval").
 *   Stage 2  gather the p·b token rows named by the dense equal-size cluster-to-token table
 *            C2T ∈ N^{c×b}, b = v/c (FlashHead notes, Module 1 "equal-size spherical k-means"),
 *            compute their exact logits and take the argmax (Eq. 2) or a softmax(z/τ) draw (Eq. 3).
 * Stage 1 may read INT4 centroids while Stage 2 stays BF16 (FlashHead notes, Module 3
 * "selective quantization").  A Monte Carlo driver estimates the marginal token probability
 * p̂(t|h) = (1/N) Σ_i p(t|h,S_i) over N independent Stage-1 draws S_i (FlashHead notes,
 * Module 4 and Eq. 7).  A dense head over all v rows is provided as the in-run comparison.
 * The index (C and C2T) is built offline from E by equal-size spherical k-means: see fh_kmeans.h.
 *
 * Citation names used in this header:
 *   "FlashHead notes"   — the reading-notes page "FlashHead: Efficient Drop-In Replacement for the
 *                         Classification Head in Language Model Inference" (method description,
 *                         Modules 1–4, Eq. 1–7, Figures 1–2, implementation details).
 *   "FlashHead summary" — the paper-summary page of the same title (Abstract, Figure 1, Tables 1–7).
 *
 * Conventions shared by every entry point.
 *   - Memory.  Every pointer argument named "device" is CUDA device memory owned by the caller;
 *     the library never frees it and never keeps it beyond the call, except the index buffers,
 *     which must outlive the fh_index handle.  Host pointers are said to be host pointers.
 *   - Layout.  Matrices are dense row-major with the stated shape, rows contiguous.  BF16 values
 *     are passed as their 16-bit patterns.  H holds B query rows of d elements each.
 *   - Streams.  fh_stream is a cudaStream_t (NULL = the legacy default stream).  Every compute
 *     entry point is asynchronous on that stream; only fh_index_load and fh_ws_status synchronise.
 *   - Errors.  Argument, shape and workspace errors are detected on the host before any launch and
 *     returned synchronously; nothing is launched then.  A CUDA launch error returns FH_ERR_CUDA.
 *     Device-side errors (a bounded wait that timed out, an index out of range met by a kernel)
 *     are recorded in the workspace status word and reported by fh_ws_status.  fh_last_error()
 *     returns a thread-local message describing the last non-FH_OK status of the calling thread.
 *   - Allocation.  No compute entry point allocates device memory: scratch space is the caller's
 *     workspace buffer, sized by fh_workspace_bytes.
 *   - Profiling.  Every entry point marks its host-side extent with an NVTX range of its own name
 *     (header-only NVTX v3: without an attached profiler a push or pop is a no-op call).
 *   - Tie rules.  Clusters are ordered by (score desc, cluster id asc), tokens by
 *     (logit desc, token id asc); -0.0 is treated as +0.0.  Inputs must be finite.
 *   - Random numbers.  Sampling uses Philox4x32-10 (Salmon, Moraes, Dror, Shaw, "Parallel random
 *     numbers: as easy as 1, 2, 3", SC'11) with key = (seed low 32 bits, seed high 32 bits) and
 *     counter = (elem >> 2, row, step low 32 bits, (stream << 24) | (step high 32 bits & 0xFFFFFF)),
 *     taking output word (elem & 3).  A draw x becomes u = ((x >> 9) + 0.5)·2^-23 ∈ (0,1), which is
 *     exact in fp32, and the Gumbel variate G = -log(-log u).  Streams: FH_RNG_STAGE1 (Stage-1
 *     keys, elem = cluster id), FH_RNG_STAGE2 (Stage-2 and dense-head keys, elem = token id),
 *     FH_RNG_MC (Monte Carlo draws, elem = cluster id, step = draw index).  row = the query's
 *     index within the batch.
 */
#ifndef FLASHHEAD_H
#define FLASHHEAD_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  FH_OK = 0,
  FH_ERR_ARG = 1,         /* NULL pointer, p outside [1, c], tau <= 0, B outside [1, FH_MAX_BATCH] ... */
  FH_ERR_SHAPE = 2,       /* v != c*b, d not a multiple of 8 (32 for INT4), sizes past the limits */
  FH_ERR_INDEX = 3,       /* C2T is not a permutation of 0..v-1 */
  FH_ERR_WORKSPACE = 4,   /* workspace NULL, too small or not 256-byte aligned */
  FH_ERR_CUDA = 5,        /* a CUDA runtime call or launch failed */
  FH_ERR_TIMEOUT = 6,     /* a bounded device-side wait gave up (reported by fh_ws_status) */
  FH_ERR_UNSUPPORTED = 7  /* a valid request this build has no kernel for */
} fh_status;

typedef enum { FH_F32 = 0, FH_BF16 = 1 } fh_dtype;

/* Stage-1 centroid format.  INT4_G32: symmetric 4-bit integers q ∈ [-8, 7] in two's complement,
   two per byte, the low nibble holding the even column; one BF16 scale per (row, group of 32
   consecutive columns); the centroid value is q·scale (FlashHead notes, Module 3). */
typedef enum { FH_STAGE1_DENSE = 0, FH_STAGE1_INT4_G32 = 1 } fh_stage1_fmt;

/* Operation selector for fh_workspace_bytes. */
typedef enum { FH_OP_GREEDY = 0, FH_OP_SAMPLE = 1, FH_OP_MC = 2, FH_OP_DENSE = 3 } fh_op;

/* Philox stream ids (see "Random numbers" above). */
enum { FH_RNG_STAGE1 = 0, FH_RNG_STAGE2 = 1, FH_RNG_MC = 2 };

/* Limits of this build. */
enum { FH_MAX_BATCH = 64, FH_MAX_C = 32768, FH_MAX_D = 8192 };

typedef void* fh_stream;            /* cudaStream_t */
typedef struct fh_index fh_index;   /* opaque host-side handle */

/* Description of one FlashHead index (FlashHead notes, Module 1 and "implementation details":
   centroid matrix C ∈ R^{c×d} plus the C2T map).  All pointers are device memory owned by the
   caller and must stay valid while the handle lives. */
typedef struct {
  int64_t v, d, c, b;        /* vocabulary, hidden size, clusters, tokens per cluster; v == c*b */
  int32_t dtype;             /* fh_dtype of E, C, E_perm and every H passed later */
  int32_t s1_fmt;            /* fh_stage1_fmt used by Stage 1 */
  const void* E;             /* device, v x d, dtype */
  const void* C;             /* device, c x d, dtype, unit rows; may be NULL iff s1_fmt == INT4_G32 */
  const int32_t* C2T;        /* device, c x b int32; row k lists the b token ids of cluster k */
  const uint8_t* C_q4;       /* device, c x d/2 bytes (INT4_G32 only, dtype must be BF16) */
  const uint16_t* C_scales;  /* device, c x d/32 BF16 patterns (INT4_G32 only) */
  void* E_perm;              /* device, v x d, dtype, or NULL.  When given, fh_index_load writes
                                the cluster-major copy E_perm[k*b + j] = E[C2T[k][j]] there, which
                                the batched tensor-core Stage 2 streams one cluster block at a time. */
} fh_index_desc;

/* Optional device outputs of one fused head call, for checking the intermediate results.
   Any field may be NULL.  sel: B x p cluster ids of S, ascending.  cand_tok: B x (p*b) token ids
   in slot order (slot r*b + j holds C2T[S[r]][j]).  cand_logit: B x (p*b) fp32 logits z of those
   tokens (the raw logits in both greedy and sampling mode). */
typedef struct {
  int32_t* sel;
  int32_t* cand_tok;
  float* cand_logit;
} fh_debug_out;

/* ---------------------------------------------------------------- index lifecycle ---------- */

/* Bytes of device scratch fh_index_load needs for validating C2T (v/8 rounded up, plus a header). */
size_t fh_index_load_ws_bytes(const fh_index_desc* desc);

/* Validate desc and create a handle.  Checks v == c*b, the size limits, d % 8 == 0 (d % 32 == 0 for
   INT4), pointer presence, and — on the device — that C2T lists every token id in [0, v) exactly once
   (FlashHead notes, Module 1: every cluster holds exactly b tokens, so C2T is a dense c×b tensor).
   Builds E_perm when desc->E_perm is non-NULL.  ws: device scratch of fh_index_load_ws_bytes bytes.
   Synchronises `stream`.  Returns FH_ERR_INDEX if C2T is not a permutation; *out is then NULL.
   The handle holds host metadata only (shapes and pointers). */
fh_status fh_index_load(const fh_index_desc* desc, void* ws, size_t ws_bytes, fh_stream stream,
                        fh_index** out);

/* Release a handle (host memory only).  NULL is ignored. */
void fh_index_free(fh_index* idx);

/* Device workspace bytes one call of `op` needs at batch B, probes p, T targets per query and N
   Monte Carlo draws (T and N are ignored unless op == FH_OP_MC).  Returns 0 for invalid arguments.
   Workspaces must be 256-byte aligned and zero-filled before their first use (the calls leave
   them ready for the next call).  A workspace may be reused by consecutive calls on the same
   stream; calls that overlap in time need separate workspaces. */
size_t fh_workspace_bytes(const fh_index* idx, int op, int B, int p, int T, int64_t N);

/* Read and clear the status word of a workspace (synchronises `stream`).  Returns FH_OK, or the
   device-side error a previous call recorded there (FH_ERR_TIMEOUT, FH_ERR_INDEX); after an error
   the workspace's control block is zeroed again so that it can be reused (its call generation moves
   past every tag a failed call may have left in the selection words). */
fh_status fh_ws_status(void* ws, fh_stream stream);

/* Thread-local description of the last error returned on this thread ("" if none). */
const char* fh_last_error(void);

/* ---------------------------------------------------------------- fused head calls --------- */

/* Greedy FlashHead head (FlashHead notes, Module 2 greedy mode and Eq. 2).
   H: device, B x d, dtype.  1 <= B <= FH_MAX_BATCH, 1 <= p <= c.
   For each query q: S_q = the p clusters with the largest s_q = C·h_q; candidates = the p·b tokens of
   S_q through C2T; out_tok[q] = argmax of their exact logits z_t = E[t]·h_q (fp32 accumulation).
   out_tok: device, B int32.  dbg: optional intermediate outputs, or NULL.
   Execution (all paths compute the same thing): B = 1 runs one persistent kernel; batches of 2 to 16
   stream the union of their probe sets once on the CUDA cores (Stage 1 on the tensor cores in BF16),
   and BF16 batches above 16 run both stages on the tensor cores, each needed E row read once for the
   whole batch (dbg->cand_tok or dbg->cand_logit force the per-query CUDA-core Stage 2 instead;
   dbg->sel alone does not).  The paths sum the fp32 logits in different orders, so their tokens can
   differ only where two candidates' logits are within that rounding (~1e-6 relative); each path is
   deterministic. */
fh_status fh_head_greedy(const fh_index* idx, const void* H, int B, int p, int32_t* out_tok,
                         void* ws, size_t ws_bytes, fh_stream stream, const fh_debug_out* dbg);

/* fh_head_greedy with host buffers, the call a host-side decode loop makes: copies H_host (host,
   B x d of the index's dtype; pinned memory keeps the copy asynchronous) to h_dev (device, the same
   size, 16-byte aligned), runs fh_head_greedy into tok_dev (device, B int32) and copies the tokens
   to tok_host (host, B int32).  All three steps are queued on `stream`; tok_host holds the tokens
   once the stream has synchronised.  The staging buffers h_dev and tok_dev belong to the caller and
   are overwritten; arguments are checked before anything is queued, with fh_head_greedy's codes. */
fh_status fh_head_greedy_host(const fh_index* idx, const void* H_host, int B, int p, int32_t* tok_host,
                              void* h_dev, int32_t* tok_dev, void* ws, size_t ws_bytes, fh_stream stream);

/* Sampling FlashHead head (FlashHead notes, Module 2 sampling mode and Eq. 3; FlashHead summary,
   Abstract item (3)).  Stage 1 draws p clusters without replacement from softmax(s_q/τ) as the top p of
   s_q/τ + G(seed, step, q, FH_RNG_STAGE1, k) (Gumbel-top-p); Stage 2 draws a token from
   softmax(z/τ) over the candidates as the argmax of z_t/τ + G(seed, step, q, FH_RNG_STAGE2, t)
   (Gumbel-max).  tau > 0.  Arguments otherwise as fh_head_greedy. */
fh_status fh_head_sample(const fh_index* idx, const void* H, int B, int p, float tau, uint64_t seed,
                         uint64_t step, int32_t* out_tok, void* ws, size_t ws_bytes,
                         fh_stream stream, const fh_debug_out* dbg);

/* Monte Carlo marginal token probability (FlashHead notes, Module 4 and Eq. 7).
   For each query q and draw i < N: S_i = Gumbel-top-p of s_q/τ + G(seed, i, q, FH_RNG_MC, k);
   p_i(t) = exp(z_t/τ) / Σ_{u ∈ cand(S_i)} exp(z_u/τ) if t's cluster is in S_i, else 0.
   targets: device, B x T int32 token ids.  out_mean, out_se: device, B x T fp64 —
   mean_i p_i(t) and its standard error sd_i(p_i(t))/sqrt(N) (sample sd, N-1 denominator; 0 if N==1).
   1 <= T <= 64, 1 <= N <= 2^24. */
fh_status fh_mc_token_prob(const fh_index* idx, const void* H, int B, const int32_t* targets, int T,
                           int p, float tau, int64_t N, uint64_t seed, double* out_mean,
                           double* out_se, void* ws, size_t ws_bytes, fh_stream stream);

/* The same estimate over the draws i0 .. i0 + N - 1 (draw i uses step i of the FH_RNG_MC stream), so
   that a long run can be split into ranges — on one device over time, or over several devices — and
   recomputed bit for bit: the sum over consecutive ranges of N_r·mean_r equals N·mean of the whole
   range (up to the rounding of the sums).  0 <= i0 <= 2^40; other arguments as fh_mc_token_prob,
   which is this call with i0 = 0. */
fh_status fh_mc_token_prob_range(const fh_index* idx, const void* H, int B, const int32_t* targets,
                                 int T, int p, float tau, int64_t i0, int64_t N, uint64_t seed,
                                 double* out_mean, double* out_se, void* ws, size_t ws_bytes,
                                 fh_stream stream);

/* Dense head over the whole vocabulary (FlashHead notes, Eq. 1–3): z = E·h_q for every token.
   sample == 0: out_tok[q] = argmax z; sample != 0: argmax of z_t/τ + G(seed, step, q, FH_RNG_STAGE2, t).
   out_logits: device B x v fp32 logits z, or NULL.  BF16 batches of 2 or more run on the tensor
   cores (one pass over E for the whole batch); batch 1 streams E on CUDA cores. */
fh_status fh_dense_head(const fh_index* idx, const void* H, int B, int sample, float tau,
                        uint64_t seed, uint64_t step, int32_t* out_tok, float* out_logits,
                        void* ws, size_t ws_bytes, fh_stream stream);

/* ---------------------------------------------------------------- single steps ------------- */
/* Each runs one step of the path on its own, for step-by-step checking; the fused calls above
   run the same device code. */

/* Stage-1 scores s = C·h_q (FlashHead notes, Figure 1 Stage 1), fp32.  out_s: device, B x c.
   Runs the kernel the fused heads run at batch B: batches of 2 or more on the tensor cores (BF16
   centroids directly, INT4 centroids dequantised to fp16 in shared memory), the CUDA-core Stage-1
   kernel at B = 1 and for fp32 indexes. */
fh_status fh_stage1_scores(const fh_index* idx, const void* H, int B, float* out_s,
                           void* ws, size_t ws_bytes, fh_stream stream);

/* Gumbel keys key[q][k] = s[q][k]/τ + G(seed, step, q, rng_stream, k), fp32.
   s, out_keys: device, B x c (may alias). */
fh_status fh_gumbel_keys(const float* s, int B, int64_t c, float tau, uint64_t seed, uint64_t step,
                         uint32_t rng_stream, float* out_keys, fh_stream stream);

/* Top-p selection (FlashHead notes, Module 2): for each of B rows of `keys` (device, B x c fp32),
   out_sel (device, B x p int32) = the ids of the p largest keys under (key desc, id asc), written in
   ascending id order. */
fh_status fh_select_topp(const float* keys, int B, int64_t c, int p, int32_t* out_sel,
                         fh_stream stream);

/* Candidate gather (FlashHead notes, Module 1: slot i → cluster S[i / b], row i mod b):
   out_cand[q][r*b + j] = C2T[sel[q][r]][j].  sel: device B x p; out_cand: device B x (p*b). */
fh_status fh_gather_candidates(const fh_index* idx, const int32_t* sel, int B, int p,
                               int32_t* out_cand, fh_stream stream);

/* Exact candidate logits out_z[q][i] = E[cand[q][i]]·h_q, fp32 accumulation.
   cand: device B x P int32 in [0, v); out_z: device B x P fp32. */
fh_status fh_candidate_logits(const fh_index* idx, const void* H, int B, const int32_t* cand,
                              int64_t P, float* out_z, fh_stream stream);

/* Raw Philox4x32-10 words: out[e] = word (e & 3) of Philox(key(seed), counter(e, row, step, rng_stream))
   for e in [0, n).  out: device, n uint32. */
fh_status fh_philox_u32(uint64_t seed, uint64_t step, uint32_t row, uint32_t rng_stream, int64_t n,
                        uint32_t* out, fh_stream stream);

/* ---------------------------------------------------------------- allocation-free call ----- */
/* No counterpart in the pages: an integration convenience of this library.
   Greedy head at batch 1 (the same computation and kernels as fh_head_greedy with B = 1) for callers
   that can neither allocate device memory nor lend a workspace — for example code inside a host
   framework that owns the whole device heap, or a decode loop that cannot afford cudaMalloc's
   implicit device synchronisation.  The call's scratch lives in a file-scope device array of
   FH_STATIC_SCRATCH_BYTES bytes that every GPU loading the library keeps until process exit.
   H: device, 1 x d; out_tok: device, 1 int32.  Allocates nothing: it calls no cudaMalloc/cudaFree
   and no allocating library routine.  Argument errors return before anything is queued.
   The array is used like a workspace: it starts zeroed, and every call leaves the words that must
   start at zero (histogram, arg-max, tickets) at zero again and tags the rest with its call
   generation.  The call first writes -1 to out_tok, so a call that fails on the device (a bounded
   wait that gave up) leaves -1 there; its error stays in the array's status word until
   fh_static_status reports it and zeroes the control block (until then later calls fail too).
   The first call on a device looks up the array's device address (cudaGetSymbolAddress, with that
   device current); make that first call before any stream capture.  Calls share the one array, so
   calls that overlap in time on the GPU (on different streams) race; serialise them.
   Returns FH_ERR_WORKSPACE with a message when the index needs more scratch than the array holds:
   4·(c + p) bytes plus about 530 KiB for c <= 16384 (the batch-1 kernel's word table), plus about
   7 KiB above; every index with c + p up to about 31,000 fits. */
enum { FH_STATIC_SCRATCH_BYTES = 655360 };
fh_status fh_head_greedy_static(const fh_index* idx, const void* H, int p, int32_t* out_tok,
                                fh_stream stream);

/* Read and clear the status word of the current device's static scratch (synchronises `stream`):
   FH_OK, or the device-side error of an earlier fh_head_greedy_static call (FH_ERR_TIMEOUT), after
   which the array's control block is zeroed again, as fh_ws_status does for a workspace. */
fh_status fh_static_status(fh_stream stream);

/* The device address and size of the current device's static scratch, for diagnostics and tests
   (writing to it while calls run races with them). */
fh_status fh_static_scratch(void** dev_ptr, size_t* bytes);

#ifdef __cplusplus
}
#endif

#endif /* FLASHHEAD_H */

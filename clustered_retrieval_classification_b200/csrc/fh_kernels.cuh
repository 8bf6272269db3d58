// fh_kernels.cuh — launch parameters of the FlashHead kernels and their host-side launchers.
// The launchers are defined in fh_kernels.cu; the C ABI in fh_api.cu validates arguments, lays out
// the caller's workspace and calls them.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace fh {

enum ElemKind : int { kF32 = 0, kBF16 = 1 };

constexpr int kMaxDevices = 64;  // per-device host caches (kernel attributes)

// Raise a kernel's dynamic shared-memory limit to `bytes` on the current device, once per
// (kernel, device) and size.
cudaError_t set_smem_attr(const void* kernel, size_t bytes);

// Stage 1: s[q][k] = C[k]·h_q (or the Gumbel key s/τ + G when sample != 0).
struct Stage1Params {
  const void* C;               // c x d (dense) — or null for INT4
  const uint8_t* q4;           // c x d/2 (INT4)
  const uint16_t* scales;      // c x d/32 (INT4)
  const void* H;               // B x d
  float* out;                  // B x c
  int64_t c, d;
  int B;
  int sample;
  float tau;
  uint64_t seed, step;
  uint32_t rng_stream;
  uint32_t* status;
  uint32_t* tickets_to_clear;  // reset to 0 by block (0,0) for the kernels that follow
  int n_tickets;
};

// Stage 2 over the candidates of each query, with the token decision fused in.
struct Stage2Params {
  const void* E;               // v x d (row source when E_perm is null)
  const void* E_perm;          // v x d cluster-major copy, or null
  const int32_t* C2T;          // c x b
  const void* H;               // B x d
  const float* keys;           // B x c Stage-1 keys (fused selection) — or null
  const int32_t* sel;          // B x p probe sets (when keys is null)
  int64_t v, d, c, b;
  int B, p;
  int sample;
  float tau;
  uint64_t seed, step;
  unsigned long long* part;    // gridDim.x x B partial arg-maxima
  uint32_t* tickets;           // B counters
  int32_t* out_tok;            // B
  int32_t* dbg_sel;            // B x p or null
  int32_t* dbg_tok;            // B x P or null
  float* dbg_logit;            // B x P or null
  uint32_t* status;
};

// Dense head over all v rows of E for each query.
struct DenseParams {
  const void* E;
  const void* H;
  int64_t v, d;
  int B;
  int sample;
  float tau;
  uint64_t seed, step;
  unsigned long long* part;    // gridDim.x x B
  uint32_t* tickets;           // B
  int32_t* out_tok;            // B (may be null)
  float* out_logits;           // B x v or null
  uint32_t* status;
};

// Monte Carlo marginal (per query: N draws of Gumbel-top-p over the Stage-1 scores).
struct McParams {
  const float* s;              // B x c Stage-1 scores
  const float* z;              // B x v logits
  const int32_t* C2T;          // c x b
  const int32_t* cluster_of;   // v: token → cluster
  const int32_t* targets;      // B x T
  float* zmax;                 // B: max_t z_t/τ
  double* Z;                   // B x c: Σ_{u in cluster} exp(z_u/τ - zmax)
  double* per_draw;            // B x N x T
  double* out_mean;            // B x T
  double* out_se;              // B x T
  int64_t v, c, b, N;
  int64_t i0;                  // first draw index (draw i uses Philox step i0 + i)
  int B, T, p;
  float tau;
  uint64_t seed;
  uint32_t* status;
};

// Tensor-core logits for a batch of queries with the mask and the decision fused (fh_tc.cu).
struct TcParams {
  int64_t rows, d;                 // A operand: rows x d (E, or its cluster-major copy)
  int B;                           // queries (<= 64)
  int64_t b;                       // rows per cluster (the mask granularity)
  const unsigned long long* qmask; // per cluster: bit q set when query q takes it (null: every row)
  const int32_t* row_tok;          // token of each A row (C2T in cluster-major order); null: the row
  int sample;
  float tau;
  uint64_t seed, step;
  unsigned long long* best;        // B packed arg-maxima (zero between calls)
  unsigned long long* ticket;      // arrival count (zero between calls)
  int32_t* out_tok;                // B, or null
  float* out_logits;               // B x rows indexed by token, or null
  float* out_keys;                 // B x rows: write the raw products (Stage-1 keys) instead
  int32_t* tile_list;              // the 128-row tiles some query takes, any order (null: every tile)
  int32_t* tile_count;             // their number (device word, written before the launch)
  uint32_t* status;
  int n_tiles, tile_rows, stages;  // set by the launcher
  int qrows, copies;               // query rows of one copy in the MMA's 128 rows, copies (launcher)
  int kbs;                         // K-blocks per pipeline stage (launcher)
};
// Batched Stage 2 over the union of the batch's probe sets (fh_kernels.cu): the listed clusters of
// the cluster-major copy, each row dotted with the queries whose mask bit is set.
struct UnionParams {
  const void* E_perm;              // v x d cluster-major copy
  const int32_t* C2T;              // c x b
  const void* H;                   // B x d
  int64_t v, d, c, b;
  int B;                           // <= 64
  const unsigned long long* qmask; // per cluster: bit q set when query q takes it
  const int32_t* cl_list;          // the clusters with a nonzero mask, each once, in any order
  const int32_t* cl_count;         // their number (device)
  int sample;
  float tau;
  uint64_t seed, step;
  unsigned long long* best;        // B packed arg-maxima (zero between calls)
  uint32_t* ticket;                // arrival count (zero between calls)
  int32_t* out_tok;                // B
  uint32_t* status;
};
bool union_supported(int elem, int64_t d, int64_t v, int64_t b, int B, int num_sms);
cudaError_t launch_union_rows(const UnionParams& prm, int elem, int num_sms, cudaStream_t st);
bool tc_supported(int elem, int64_t d, int B);
cudaError_t launch_tc_head(const void* A, const void* H, TcParams p, int num_sms, cudaStream_t st);
// qmask: c words, zero before the call; list/count (count zero before the call): the clusters some
// query selected, or with tile_flags (zero before the call) the tile_rows-row tiles of the
// cluster-major copy (rows rows, b per cluster) that hold one.
cudaError_t launch_build_qmask(const int32_t* sel, int B, int p, unsigned long long* qmask,
                               cudaStream_t st, int32_t* list = nullptr, int32_t* count = nullptr,
                               uint32_t* tile_flags = nullptr, int64_t b = 0, int64_t rows = 0,
                               int tile_rows = 128, bool overlap = false);
bool tc_int4_supported(int64_t d, int B, const void* scales);
// INT4 Stage-1 keys on the tensor cores: out_keys[q][k] = Σ_j q4[k][j]·scale[k][j/32]·h_q[j] (or the
// Gumbel key when sample != 0), dequantised to fp16 in shared memory (fh_tc.cu).
cudaError_t launch_tc_keys_int4(const uint8_t* q4, const uint16_t* scales, int64_t rows, int64_t d,
                                const void* H, int B, int sample, float tau, uint64_t seed,
                                uint64_t step, float* out_keys, uint32_t* status,
                                uint32_t* tickets_to_clear, int n_tickets, int num_sms,
                                cudaStream_t st);

// The batch-1 persistent head (fh_head1.cu).
constexpr int kHead1Bins = 1024;       // Stage-1 key histogram
constexpr int kHead1BucketCap = 64;    // tagged (cluster, key) words kept per histogram bin

struct Head1Params {
  const void* C;               // c x d (dense Stage 1) or null
  const uint8_t* q4;           // c x d/2 (INT4 Stage 1) or null
  const uint16_t* scales;      // c x d/32
  const void* H;               // 1 x d
  const void* E;               // v x d
  const void* E_perm;          // v x d cluster-major copy, or null
  const int32_t* C2T;          // c x b
  float* keys;                 // c: Stage-1 keys (workspace)
  int64_t c, d, b;
  int p;
  int sample;
  float tau;
  uint64_t seed, step;
  uint32_t* arrive;               // blocks done with the call (zero between calls)
  unsigned long long* best;       // the call's packed (key, ~token) maximum (zero between calls)
  uint32_t* hist;                 // kHead1Bins-bin key histogram (zero between calls)
  uint32_t* gen;                  // tag of the last completed call (a call tags its words gen+1)
  uint32_t* keys_ready;           // arrivals once the keys are written (grows by gridDim.x per use)
  unsigned long long* bucket;     // kHead1Bins x kHead1BucketCap tagged words (tag, cluster, key)
  int32_t* out_tok;
  int32_t* dbg_sel;            // p or null
  int32_t* dbg_tok;            // p*b or null
  float* dbg_logit;            // p*b or null
  uint32_t* status;
  int k1, k2;                  // ring slots per warp in Stage 1 / Stage 2 (set by the launcher)
  uint32_t ring_bytes;         // (set by the launcher)
};

// Threads per block of the persistent head for c clusters (0: not supported, use the batched path).
int head1_threads(int64_t c);
cudaError_t launch_head1(Head1Params prm, int elem, int int4, int num_sms, cudaStream_t st);

// ---- launchers (return cudaGetLastError() of the launch) ----
cudaError_t launch_stage1(const Stage1Params& prm, int elem, int int4, int num_sms,
                          cudaStream_t st, bool pdl_primary);
cudaError_t launch_gumbel_keys(const float* s, float* keys, int B, int64_t c, float tau,
                               uint64_t seed, uint64_t step, uint32_t rng_stream,
                               cudaStream_t st);
// zero / zero_bytes (optional, a multiple of 4): a region cleared on the way, for the next kernel; a
// call that passes one follows the Stage-1 kernel of the same head call and may overlap its tail.
cudaError_t launch_select(const float* keys, int32_t* sel, int B, int64_t c, int p,
                          cudaStream_t st, void* zero = nullptr, size_t zero_bytes = 0);
cudaError_t launch_stage2(const Stage2Params& prm, int elem, int num_sms, cudaStream_t st);
cudaError_t launch_dense(const DenseParams& prm, int elem, int num_sms, cudaStream_t st);
cudaError_t launch_gather(const int32_t* C2T, int64_t b, const int32_t* sel, int B, int p,
                          int32_t* cand, cudaStream_t st);
cudaError_t launch_cand_logits(const void* E, int elem, int64_t d, const void* H, int B,
                               const int32_t* cand, int64_t P, float* out_z, cudaStream_t st);
cudaError_t launch_philox(uint64_t seed, uint64_t step, uint32_t row, uint32_t rng_stream,
                          int64_t n, uint32_t* out, cudaStream_t st);
cudaError_t launch_validate_c2t(const int32_t* C2T, int64_t v, uint32_t* bitmap,
                                uint32_t* status, cudaStream_t st);
cudaError_t launch_build_perm(const void* E, const int32_t* C2T, int64_t v, int64_t d, int elem,
                              void* E_perm, cudaStream_t st);
cudaError_t launch_mc(const McParams& prm, int num_sms, cudaStream_t st);

// Number of Stage-2 blocks used per query for `rows` candidate rows.
int stage2_blocks(int64_t rows, int B, int num_sms);

}  // namespace fh

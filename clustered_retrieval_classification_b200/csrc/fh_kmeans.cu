// fh_kmeans.cu — the FlashHead index builder on the device: equal-size spherical k-means
// (FlashHead notes, Module 1, Eq.4 and Eq.5).  The arithmetic of every step lives in
// fh_kmeans_core.cuh; this file holds the kernels that run it, the device backend of the iteration
// loop and the C ABI of include/fh_kmeans.h.
//
// Kernels (one iteration of an auction round: bid, scan, scatter, resolve; then labels, update):
//   similarities   the tensor-core kernel of fh_tc.cu in key mode, 64 tokens per launch as the
//                  "queries" against the BF16 centres as rows: S[i][k] = e_i . c_k in fp32
//   k_km_bid       one warp per unassigned token: a coalesced pass over its row of S, best and
//                  second-best net value by shuffles, the bid and its slot in the cluster's inbox
//   k_km_scan      one block: start of each cluster's bids (exclusive prefix sum over c)
//   k_km_scatter   one thread per bid: bids grouped by cluster
//   k_km_resolve   one thread per cluster: the b best of kept + received bids (heap), price update
//   k_km_labels    one thread per cluster: labels and its C2T row, sorted
//   k_km_update    one block per cluster: Eq.5 over the columns, norm, fp32 and BF16 centre
// Nothing waits on another block: every kernel is a plain data-parallel pass, and the host ends an
// auction phase when the read-back count of unassigned tokens reaches zero (at most max_rounds).
#include <cuda_runtime.h>

#include <algorithm>
#include <cstdarg>
#include <cstdio>

#include "../../include/fh_kmeans.h"
#include "fh_kernels.cuh"
#include "fh_nvtx.cuh"
#include "fh_kmeans_core.cuh"

namespace fh {
fh_status report(fh_status st, const char* fmt, ...);  // fh_api.cu: sets fh_last_error()
}

namespace {

using namespace fhkm;

constexpr int kTokensPerLaunch = 64;   // queries per tensor-core launch
constexpr int kBidThreads = 256;       // 8 warps, one token each
constexpr int kScanThreads = 1024;
constexpr int kUpdateThreads = 256;
constexpr size_t kAlign = 256;

enum Counter { kNext = 0, kBadRows = 1, kChanged = 2, kBad = 3, kDegenerateCtr = 4, kTcStatus = 5 };

size_t up(size_t x) { return (x + kAlign - 1) / kAlign * kAlign; }

struct KmLayout {
  size_t ctr, S, inv, Cb, price, slot_bid, slot_tok, fill, cnt, off, inbox, U0, U1, bid_k, bid_beta,
      pos, prev, norms, total;
};

KmLayout km_layout(int64_t v, int64_t d, int64_t c) {
  KmLayout L{};
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t at = off;
    off = up(off + bytes);
    return at;
  };
  L.ctr = take(256);
  L.S = take((size_t)v * c * 4);
  L.inv = take((size_t)v * 4);
  L.Cb = take((size_t)c * d * 2);
  L.price = take((size_t)c * 4);
  L.slot_bid = take((size_t)v * 4);
  L.slot_tok = take((size_t)v * 4);
  L.fill = take((size_t)c * 4);
  L.cnt = take((size_t)c * 4);
  L.off = take((size_t)c * 4);
  L.inbox = take((size_t)v * 4);
  L.U0 = take((size_t)v * 4);
  L.U1 = take((size_t)v * 4);
  L.bid_k = take((size_t)v * 4);
  L.bid_beta = take((size_t)v * 4);
  L.pos = take((size_t)v * 4);
  L.prev = take((size_t)v * 4);
  L.norms = take((size_t)c * 4);
  L.total = off;
  return L;
}

unsigned blocks_for(int64_t items, int per_block) {
  return (unsigned)((items + per_block - 1) / per_block);
}

// ------------------------------------------------------------------ kernels ---------------

__global__ void k_km_row_norms(const uint16_t* E, int64_t v, int64_t d, float* inv,
                               uint32_t* bad_rows) {
  const int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
  if (i >= v) return;
  const float r = row_inv_norm(E + i * d, d);
  inv[i] = r;
  if (r == 0.f) fetch_add(bad_rows, 1u);
}

__global__ void k_km_init(const uint16_t* E, const float* inv, const int32_t* init, int64_t v,
                          int64_t d, float* C, uint16_t* Cb, int32_t* mark, uint32_t* bad) {
  __shared__ int32_t tok_s;
  const int k = blockIdx.x;
  if (threadIdx.x == 0) {
    tok_s = claim_init_token(init, k, v, mark);
    if (tok_s < 0) fetch_add(bad, 1u);
  }
  __syncthreads();
  const int32_t tok = tok_s;
  for (int64_t j = threadIdx.x; j < d; j += blockDim.x) {
    const float x = tok >= 0 ? unit_value(E, inv, tok, d, j) : 0.f;
    C[(int64_t)k * d + j] = x;
    Cb[(int64_t)k * d + j] = f32_to_bf16(x);
  }
}

__device__ __forceinline__ Top2 shfl_xor_top2(const Top2& t, int o) {
  Top2 r;
  r.v1 = __shfl_xor_sync(0xFFFFFFFFu, t.v1, o);
  r.a1 = __shfl_xor_sync(0xFFFFFFFFu, t.a1, o);
  r.v2 = __shfl_xor_sync(0xFFFFFFFFu, t.v2, o);
  r.k1 = __shfl_xor_sync(0xFFFFFFFFu, t.k1, o);
  return r;
}

__global__ void __launch_bounds__(kBidThreads) k_km_bid(Auction s, const float* S, const float* inv,
                                                        int64_t n, float eps) {
  const int64_t w = (blockIdx.x * (int64_t)blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (w >= n) return;  // uniform over the warp
  const int32_t i = s.U[w];
  Top2 t = lane_top2(S + (int64_t)i * s.c, inv[i], s.price, s.c, lane, 32);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) t = top2_merge(t, shfl_xor_top2(t, o));
  if (lane == 0) {
    const int k1 = (t.k1 >= 0 && t.k1 < s.c) ? t.k1 : 0;  // finite rows always give k1 < c
    s.bid_k[w] = k1;
    s.bid_beta[w] = bid_value(t, eps);
    s.pos[w] = fetch_add(&s.cnt[k1], 1);
  }
}

__global__ void __launch_bounds__(kScanThreads) k_km_scan(const int32_t* cnt, int32_t* off, int c) {
  __shared__ int32_t part[kScanThreads];
  const int t = threadIdx.x;
  const int per = (c + kScanThreads - 1) / kScanThreads;
  const int lo = min(c, t * per), hi = min(c, lo + per);
  int32_t sum = 0;
  for (int k = lo; k < hi; ++k) sum += cnt[k];
  part[t] = sum;
  __syncthreads();
  if (t < 32) {  // lane l turns partials [32l, 32l + 32) into exclusive sums, then adds its base
    int32_t run = 0;
    for (int j = 0; j < 32; ++j) {
      const int32_t x = part[t * 32 + j];
      part[t * 32 + j] = run;
      run += x;
    }
    int32_t incl = run;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int32_t y = __shfl_up_sync(0xFFFFFFFFu, incl, o);
      if (t >= o) incl += y;
    }
    const int32_t base = incl - run;
    for (int j = 0; j < 32; ++j) part[t * 32 + j] += base;
  }
  __syncthreads();
  int32_t run = part[t];
  for (int k = lo; k < hi; ++k) {
    off[k] = run;
    run += cnt[k];
  }
}

__global__ void k_km_scatter(Auction s, int64_t n) {
  const int64_t t = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
  if (t < n) scatter_bid(s, t);
}

__global__ void k_km_resolve(Auction s) {
  const int k = blockIdx.x * blockDim.x + threadIdx.x;
  if (k < s.c) resolve_cluster(k, s);
}

__global__ void k_km_iota(int32_t* U, int64_t v) {
  const int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
  if (i < v) U[i] = (int32_t)i;
}

__global__ void k_km_one_cluster(int32_t* slot_tok, int32_t* fill, int64_t v) {
  const int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
  if (i < v) slot_tok[i] = (int32_t)i;
  if (i == 0) fill[0] = (int32_t)v;
}

__global__ void k_km_slots(const int32_t* labels, int64_t v, int c, int64_t b, int32_t* fill,
                           int32_t* slot_tok, uint32_t* bad) {
  const int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
  if (i < v && !slot_from_label(i, labels, c, b, fill, slot_tok)) fetch_add(bad, 1u);
}

__global__ void k_km_labels(const int32_t* slot_tok, int c, int64_t b, int32_t* labels,
                            int32_t* C2T) {
  const int k = blockIdx.x * blockDim.x + threadIdx.x;
  if (k < c) write_cluster(k, slot_tok, b, labels, C2T);
}

__global__ void k_km_changes(const int32_t* labels, int32_t* prev, int64_t v, int first,
                             uint32_t* changed) {
  const int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
  if (i >= v) return;
  if (!first && labels[i] != prev[i]) fetch_add(changed, 1u);
  prev[i] = labels[i];
}

__global__ void __launch_bounds__(kUpdateThreads) k_km_update(const uint16_t* E, const float* inv,
                                                              const int32_t* C2T, int64_t d,
                                                              int64_t b, float* C, uint16_t* Cb,
                                                              float* norms, uint32_t* degenerate) {
  extern __shared__ float acc[];  // d columns of the member sum
  __shared__ float norm_s;
  const int k = blockIdx.x;
  const int32_t* members = C2T + (int64_t)k * b;
  for (int64_t j = threadIdx.x; j < d; j += blockDim.x) acc[j] = member_sum(E, inv, members, b, d, j);
  __syncthreads();
  if (threadIdx.x == 0) {
    const float n = column_norm(acc, d);
    norm_s = n;
    norms[k] = n;
    if (!(n > 0.f)) fetch_add(degenerate, 1u);
  }
  __syncthreads();
  const float n = norm_s;
  for (int64_t j = threadIdx.x; j < d; j += blockDim.x) {
    const float x = centre_value(acc[j], n);
    C[(int64_t)k * d + j] = x;
    Cb[(int64_t)k * d + j] = f32_to_bf16(x);
  }
}

__global__ void k_km_objective(const float* norms, int c, double* out) {
  __shared__ double part[kObjectiveParts];
  part[threadIdx.x] = objective_part(norms, c, threadIdx.x, kObjectiveParts);
  __syncthreads();
  if (threadIdx.x == 0) *out = objective_total(part, kObjectiveParts);
}

// ------------------------------------------------------------------ device backend --------

struct DeviceBackend {
  const uint16_t* E = nullptr;
  int64_t v = 0, d = 0, b = 0;
  int c = 0;
  const int32_t* init = nullptr;
  const uint16_t* C_score = nullptr;  // BF16 centres the similarities use
  const int32_t* labels_in = nullptr;
  int32_t* labels = nullptr;
  int32_t* C2T = nullptr;
  float* C = nullptr;
  uint16_t* Cb = nullptr;             // where the update writes the BF16 centres
  double* objective = nullptr;
  float *S = nullptr, *inv = nullptr, *norms = nullptr;
  int32_t* prev = nullptr;
  uint32_t* ctr = nullptr;
  Auction a{};
  int32_t* U[2] = {nullptr, nullptr};
  int cur = 0;
  int num_sms = 0;
  cudaStream_t st = nullptr;
  cudaError_t err = cudaSuccess;

  bool ok(cudaError_t e) {
    if (e != cudaSuccess && err == cudaSuccess) err = e;
    return e == cudaSuccess;
  }
  bool launched() { return ok(cudaGetLastError()); }

  // Reads counter `i` (after the work queued so far) and zeroes it.
  bool take(int i, int64_t* out) {
    uint32_t h = 0;
    if (!ok(cudaMemcpyAsync(&h, ctr + i, 4, cudaMemcpyDeviceToHost, st))) return false;
    if (!ok(cudaStreamSynchronize(st))) return false;
    *out = h;
    return ok(cudaMemsetAsync(ctr + i, 0, 4, st));
  }

  bool row_norms(int64_t* bad) {
    k_km_row_norms<<<blocks_for(v, 256), 256, 0, st>>>(E, v, d, inv, ctr + kBadRows);
    return launched() && take(kBadRows, bad);
  }

  bool init_centres(int64_t* bad) {
    if (!ok(cudaMemsetAsync(prev, 0xFF, (size_t)v * 4, st))) return false;
    k_km_init<<<c, 256, 0, st>>>(E, inv, init, v, d, C, Cb, prev, ctr + kBad);
    return launched() && take(kBad, bad);
  }

  bool similarities() {
    const int64_t Bq = std::min<int64_t>(kTokensPerLaunch, v);
    for (int64_t start = 0; start < v; start += kTokensPerLaunch) {
      const int64_t s0 = std::min(start, v - Bq);  // the last launch re-covers a few rows
      fh::TcParams tp = {};
      tp.rows = c;
      tp.d = d;
      tp.B = (int)Bq;
      tp.b = 1;
      tp.out_keys = S + s0 * c;
      tp.status = ctr + kTcStatus;
      if (!ok(fh::launch_tc_head(C_score, E + s0 * d, tp, num_sms, st))) return false;
    }
    return true;
  }

  bool zero_prices() { return ok(cudaMemsetAsync(a.price, 0, (size_t)c * 4, st)); }

  bool reset_phase() {
    if (!ok(cudaMemsetAsync(a.fill, 0, (size_t)c * 4, st))) return false;
    cur = 0;
    k_km_iota<<<blocks_for(v, 256), 256, 0, st>>>(U[0], v);
    return launched();
  }

  bool one_cluster() {
    k_km_one_cluster<<<blocks_for(v, 256), 256, 0, st>>>(a.slot_tok, a.fill, v);
    return launched();
  }

  bool round(int64_t n, float eps) {
    Auction s = a;
    s.U = U[cur];
    s.U_next = U[cur ^ 1];
    s.n_next = reinterpret_cast<int32_t*>(ctr + kNext);
    k_km_bid<<<blocks_for(n, kBidThreads / 32), kBidThreads, 0, st>>>(s, S, inv, n, eps);
    if (!launched()) return false;
    k_km_scan<<<1, kScanThreads, 0, st>>>(s.cnt, s.off, c);
    if (!launched()) return false;
    k_km_scatter<<<blocks_for(n, 256), 256, 0, st>>>(s, n);
    if (!launched()) return false;
    k_km_resolve<<<blocks_for(c, 128), 128, 0, st>>>(s);
    return launched();
  }

  bool next_count(int64_t* left) {
    if (!take(kNext, left)) return false;
    cur ^= 1;
    return true;
  }

  bool slots_from_labels(int64_t* bad) {
    if (!ok(cudaMemsetAsync(a.fill, 0, (size_t)c * 4, st))) return false;
    k_km_slots<<<blocks_for(v, 256), 256, 0, st>>>(labels_in, v, c, b, a.fill, a.slot_tok, ctr + kBad);
    return launched() && take(kBad, bad);
  }

  bool finish_labels(bool first, int64_t* changed) {
    k_km_labels<<<blocks_for(c, 128), 128, 0, st>>>(a.slot_tok, c, b, labels, C2T);
    if (!launched()) return false;
    k_km_changes<<<blocks_for(v, 256), 256, 0, st>>>(labels, prev, v, first ? 1 : 0, ctr + kChanged);
    return launched() && take(kChanged, changed);
  }

  bool update_centres(int t, int64_t* degenerate) {
    k_km_update<<<c, kUpdateThreads, (size_t)d * 4, st>>>(E, inv, C2T, d, b, C, Cb, norms,
                                                          ctr + kDegenerateCtr);
    if (!launched()) return false;
    if (objective) {
      k_km_objective<<<1, kObjectiveParts, 0, st>>>(norms, c, objective + t);
      if (!launched()) return false;
    }
    return take(kDegenerateCtr, degenerate);
  }
};

enum Op { kBuild, kAssign, kUpdate };

fh_status check_args(const fh_kmeans_args* A, Op op, void* ws, size_t ws_bytes) {
  if (!A) return fh::report(FH_ERR_ARG, "args is NULL");
  if (!A->E) return fh::report(FH_ERR_ARG, "E is NULL");
  if (A->dtype != FH_BF16) return fh::report(FH_ERR_UNSUPPORTED, "the builder clusters BF16 embeddings only");
  if (A->c < 1 || A->c > FH_MAX_C) return fh::report(FH_ERR_SHAPE, "c outside [1, %d]", (int)FH_MAX_C);
  if (A->v < 2 || A->v > 0x7FFFFFFF || A->v % A->c != 0)
    return fh::report(FH_ERR_SHAPE, "v must be in [2, 2^31) and a multiple of c");
  if (A->d < 8 || A->d > FH_MAX_D || A->d % 8 != 0)
    return fh::report(FH_ERR_SHAPE, "d must be a multiple of 8 in [8, %d]", (int)FH_MAX_D);
  if (op == kBuild && (A->iters < 1 || !A->init_tokens))
    return fh::report(FH_ERR_ARG, "iters < 1 or init_tokens is NULL");
  if (op == kAssign && !A->C_in) return fh::report(FH_ERR_ARG, "C_in is NULL");
  if (op == kUpdate && !A->labels_in) return fh::report(FH_ERR_ARG, "labels_in is NULL");
  if (op != kUpdate && !A->labels) return fh::report(FH_ERR_ARG, "labels is NULL");
  if (!A->C2T) return fh::report(FH_ERR_ARG, "C2T is NULL");
  if (op != kAssign && !A->C) return fh::report(FH_ERR_ARG, "C is NULL");
  if (op != kUpdate && !(A->eps >= 1e-5f && A->eps <= 0.25f))
    return fh::report(FH_ERR_ARG, "eps outside [1e-5, 0.25]");
  if (A->max_rounds < 0) return fh::report(FH_ERR_ARG, "max_rounds < 0");
  if (!fh::tc_supported(fh::kBF16, A->d, (int)std::min<int64_t>(kTokensPerLaunch, A->v)))
    return fh::report(FH_ERR_UNSUPPORTED, "no tensor-core similarity kernel for this shape or driver");
  if (!ws || (reinterpret_cast<uintptr_t>(ws) % kAlign) != 0)
    return fh::report(FH_ERR_WORKSPACE, "workspace NULL or not 256-byte aligned");
  if (ws_bytes < km_layout(A->v, A->d, A->c).total)
    return fh::report(FH_ERR_WORKSPACE, "workspace of %zu bytes is smaller than %zu", ws_bytes,
                      km_layout(A->v, A->d, A->c).total);
  const uintptr_t e = reinterpret_cast<uintptr_t>(A->E);
  const uintptr_t ci = reinterpret_cast<uintptr_t>(A->C_in);
  if ((e & 15u) || (op == kAssign && (ci & 15u)))
    return fh::report(FH_ERR_ARG, "E and C_in must be 16-byte aligned");
  return FH_OK;
}

fh_status run_op(fh_kmeans_args* A, Op op, void* ws, size_t ws_bytes, fh_stream stream) {
  fh_status r = check_args(A, op, ws, ws_bytes);
  if (r != FH_OK) return r;
  A->iters_done = 0;
  A->rounds = 0;
  const KmLayout L = km_layout(A->v, A->d, A->c);
  char* base = static_cast<char*>(ws);
  DeviceBackend be;
  be.st = static_cast<cudaStream_t>(stream);
  int dev = 0;
  if (!be.ok(cudaGetDevice(&dev)) ||
      !be.ok(cudaDeviceGetAttribute(&be.num_sms, cudaDevAttrMultiProcessorCount, dev)))
    return fh::report(FH_ERR_CUDA, "device query: %s", cudaGetErrorString(be.err));
  be.E = static_cast<const uint16_t*>(A->E);
  be.v = A->v;
  be.d = A->d;
  be.c = (int)A->c;
  be.b = A->v / A->c;
  be.init = A->init_tokens;
  be.labels_in = A->labels_in;
  be.labels = op == kUpdate ? reinterpret_cast<int32_t*>(base + L.prev) : A->labels;
  be.C2T = A->C2T;
  be.C = A->C;
  be.Cb = reinterpret_cast<uint16_t*>(base + L.Cb);
  be.C_score = op == kAssign ? A->C_in : be.Cb;
  be.objective = A->objective;
  be.S = reinterpret_cast<float*>(base + L.S);
  be.inv = reinterpret_cast<float*>(base + L.inv);
  be.norms = reinterpret_cast<float*>(base + L.norms);
  // update: the labels are rebuilt from labels_in into the prev region; changes are not counted
  be.prev = op == kUpdate ? reinterpret_cast<int32_t*>(base + L.U1) : reinterpret_cast<int32_t*>(base + L.prev);
  be.ctr = reinterpret_cast<uint32_t*>(base + L.ctr);
  be.a.v = A->v;
  be.a.c = (int)A->c;
  be.a.b = be.b;
  be.a.price = reinterpret_cast<float*>(base + L.price);
  be.a.slot_bid = reinterpret_cast<float*>(base + L.slot_bid);
  be.a.slot_tok = reinterpret_cast<int32_t*>(base + L.slot_tok);
  be.a.fill = reinterpret_cast<int32_t*>(base + L.fill);
  be.a.cnt = reinterpret_cast<int32_t*>(base + L.cnt);
  be.a.off = reinterpret_cast<int32_t*>(base + L.off);
  be.a.inbox = reinterpret_cast<int32_t*>(base + L.inbox);
  be.a.bid_k = reinterpret_cast<int32_t*>(base + L.bid_k);
  be.a.bid_beta = reinterpret_cast<float*>(base + L.bid_beta);
  be.a.pos = reinterpret_cast<int32_t*>(base + L.pos);
  be.U[0] = reinterpret_cast<int32_t*>(base + L.U0);
  be.U[1] = reinterpret_cast<int32_t*>(base + L.U1);
  if (!be.ok(cudaMemsetAsync(be.ctr, 0, 256, be.st)) ||
      !be.ok(cudaMemsetAsync(be.a.cnt, 0, (size_t)A->c * 4, be.st)))
    return fh::report(FH_ERR_CUDA, "workspace reset: %s", cudaGetErrorString(be.err));

  const Config cfg = make_config(A->v, A->d, A->c, op == kBuild ? A->iters : 1, A->eps, A->max_rounds);
  Progress pr;
  Outcome o = op == kBuild ? run(be, cfg, pr) : op == kAssign ? assign_only(be, cfg, pr) : update_only(be, cfg);
  A->rounds = pr.rounds;
  A->iters_done = op == kBuild ? pr.iters_done : (op == kUpdate && o == kDone ? 1 : 0);
  if (o == kBackend) return fh::report(FH_ERR_CUDA, "k-means step: %s", cudaGetErrorString(be.err));
  // outputs that are copies of workspace state
  if (o == kDone && op != kAssign && A->C_bf16 &&
      !be.ok(cudaMemcpyAsync(A->C_bf16, be.Cb, (size_t)A->c * A->d * 2, cudaMemcpyDeviceToDevice, be.st)))
    return fh::report(FH_ERR_CUDA, "copy of the BF16 centres: %s", cudaGetErrorString(be.err));
  if (o == kDone && op != kUpdate && A->prices &&
      !be.ok(cudaMemcpyAsync(A->prices, be.a.price, (size_t)A->c * 4, cudaMemcpyDeviceToDevice, be.st)))
    return fh::report(FH_ERR_CUDA, "copy of the prices: %s", cudaGetErrorString(be.err));
  int64_t tc_status = 0;
  if (!be.take(kTcStatus, &tc_status))
    return fh::report(FH_ERR_CUDA, "status read: %s", cudaGetErrorString(be.err));
  if (tc_status) return fh::report(FH_ERR_TIMEOUT, "a tensor-core similarity launch timed out");
  switch (o) {
    case kDone: return FH_OK;
    case kZeroRow: return fh::report(FH_ERR_ARG, "E has a zero or non-finite row");
    case kBadInit:
      return fh::report(FH_ERR_ARG, op == kUpdate ? "labels_in is not an equal-size labeling"
                                                  : "init_tokens out of range or repeated");
    case kDegenerate: return fh::report(FH_ERR_ARG, "a cluster's members sum to zero");
    case kRoundLimit: return fh::report(FH_ERR_TIMEOUT, "auction exceeded max_rounds");
    default: return fh::report(FH_ERR_CUDA, "k-means step failed");
  }
}

}  // namespace

extern "C" {

size_t fh_kmeans_ws_bytes(int64_t v, int64_t d, int64_t c) {
  if (c < 1 || c > FH_MAX_C || v < 2 || v > 0x7FFFFFFF || v % c != 0 || d < 8 || d > FH_MAX_D)
    return 0;
  return km_layout(v, d, c).total;
}

fh_status fh_kmeans_build(fh_kmeans_args* args, void* ws, size_t ws_bytes, fh_stream stream) {
  FH_NVTX_RANGE("fh_kmeans_build");
  return run_op(args, kBuild, ws, ws_bytes, stream);
}

fh_status fh_kmeans_assign(fh_kmeans_args* args, void* ws, size_t ws_bytes, fh_stream stream) {
  FH_NVTX_RANGE("fh_kmeans_assign");
  return run_op(args, kAssign, ws, ws_bytes, stream);
}

fh_status fh_kmeans_update(fh_kmeans_args* args, void* ws, size_t ws_bytes, fh_stream stream) {
  FH_NVTX_RANGE("fh_kmeans_update");
  return run_op(args, kUpdate, ws, ws_bytes, stream);
}

}  // extern "C"

// fh_kmeans_core.cuh — equal-size spherical k-means, the offline builder of a FlashHead index
// (FlashHead notes, Module 1 "equal-size spherical K-Means", Eq.4 and Eq.5; implementation details:
// c clusters of exactly b = v/c tokens, up to 1000 iterations).
//
// One iteration alternates two half-steps, each an exact or certified optimiser of Eq.4 on the
// unit rows x_i = e_i / |e_i| (spherical k-means after Dhillon & Modha, whom the notes cite):
//   assignment  labels maximising sum_i x_i . c_k(i) with exactly b tokens per cluster.  This is a
//               transportation problem; it is solved by the auction algorithm for transportation
//               problems (Bertsekas & Castanon, "The auction algorithm for the transportation
//               problem", Annals of OR 20, 1989) in its Jacobi form with epsilon scaling: every
//               unassigned token bids for its best cluster at net value a_ik - price_k, raising the
//               price by the gap to its second best plus eps; a cluster keeps its b highest bids
//               and its price becomes the lowest bid it keeps.  The result satisfies
//               eps-complementary slackness, hence is within v*eps of the optimum.
//   update      Eq.5: c_k = sum_{i in k} x_i / |sum_{i in k} x_i|, after which the objective of
//               Eq.4 equals -sum_k |sum_{i in k} x_i|.
//
// Every per-item step is a __host__ __device__ function and the iteration loop is a template over
// a backend, so that the device kernels (fh_kmeans.cu) and a host build of the same steps run the
// same arithmetic in the same order.  Floating point follows IEEE round-to-nearest everywhere
// (explicit fused multiply-adds, correctly rounded division and square root).
#pragma once

#include <math.h>
#include <stdint.h>
#include <string.h>

#if defined(__CUDACC__)
#define KM_HD __host__ __device__ __forceinline__
#else
#define KM_HD inline
#endif

namespace fhkm {

// ------------------------------------------------------------------ scalar helpers --------

KM_HD float bf16_to_f32(uint16_t h) {
#if defined(__CUDA_ARCH__)
  return __uint_as_float((uint32_t)h << 16);
#else
  uint32_t u = (uint32_t)h << 16;
  float f;
  memcpy(&f, &u, 4);
  return f;
#endif
}

// Round to nearest even; inputs are finite.
KM_HD uint16_t f32_to_bf16(float f) {
#if defined(__CUDA_ARCH__)
  uint32_t u = __float_as_uint(f);
#else
  uint32_t u;
  memcpy(&u, &f, 4);
#endif
  u += 0x7FFFu + ((u >> 16) & 1u);
  return (uint16_t)(u >> 16);
}

KM_HD float fma_rn(float a, float b, float c) { return fmaf(a, b, c); }

KM_HD float sqrt_rn(float x) {
#if defined(__CUDA_ARCH__)
  return __fsqrt_rn(x);
#else
  return sqrtf(x);
#endif
}

KM_HD float div_rn(float a, float b) {
#if defined(__CUDA_ARCH__)
  return __fdiv_rn(a, b);
#else
  return a / b;
#endif
}

// Counter increments: atomic in the device build, plain in the (sequential) host build.
KM_HD int32_t fetch_add(int32_t* p, int32_t x) {
#if defined(__CUDA_ARCH__)
  return atomicAdd(p, x);
#else
  const int32_t o = *p;
  *p = o + x;
  return o;
#endif
}

KM_HD uint32_t fetch_add(uint32_t* p, uint32_t x) {
#if defined(__CUDA_ARCH__)
  return atomicAdd(p, x);
#else
  const uint32_t o = *p;
  *p = o + x;
  return o;
#endif
}

KM_HD int32_t compare_swap(int32_t* p, int32_t expect, int32_t desired) {
#if defined(__CUDA_ARCH__)
  return atomicCAS(p, expect, desired);
#else
  const int32_t o = *p;
  if (o == expect) *p = desired;
  return o;
#endif
}

// ------------------------------------------------------------------ unit rows -------------

// 1/|e_i| for one BF16 row, accumulated in order of the columns; 0 for a zero row or one whose
// squared norm is not a finite float (both are rejected by the caller).
KM_HD float row_inv_norm(const uint16_t* e, int64_t d) {
  float ss = 0.f;
  for (int64_t j = 0; j < d; ++j) {
    const float x = bf16_to_f32(e[j]);
    ss = fma_rn(x, x, ss);
  }
  return (ss > 0.f && ss <= 3.0e38f) ? div_rn(1.f, sqrt_rn(ss)) : 0.f;
}

// Column j of the unit row x_tok (an initial centre).
KM_HD float unit_value(const uint16_t* E, const float* inv_norm, int32_t tok, int64_t d, int64_t j) {
  return bf16_to_f32(E[(int64_t)tok * d + j]) * inv_norm[tok];
}

// Checks one initial-centre token: in range and not taken by another centre (mark[] starts at -1).
// Returns the token, or -1 when it is rejected.
KM_HD int32_t claim_init_token(const int32_t* init, int k, int64_t v, int32_t* mark) {
  const int32_t tok = init[k];
  if (tok < 0 || (int64_t)tok >= v) return -1;
  return compare_swap(&mark[tok], -1, k) == -1 ? tok : -1;
}

// ------------------------------------------------------------------ bids ------------------

// Best net value v1 = a_ik1 - price_k1 (ties to the lower cluster id), its similarity a1, and the
// second best net value v2 over the other clusters.
struct Top2 {
  float v1, a1, v2;
  int k1;
};

KM_HD Top2 top2_init() {
  Top2 t;
  t.v1 = -INFINITY;
  t.a1 = 0.f;
  t.v2 = -INFINITY;
  t.k1 = 0x7FFFFFFF;
  return t;
}

KM_HD bool ahead(float va, int ka, float vb, int kb) { return va > vb || (va == vb && ka < kb); }

KM_HD void top2_add(Top2& t, float a, float net, int k) {
  if (ahead(net, k, t.v1, t.k1)) {
    t.v2 = t.v1;
    t.v1 = net;
    t.a1 = a;
    t.k1 = k;
  } else if (net > t.v2) {
    t.v2 = net;
  }
}

// Combines the results over two disjoint sets of clusters; exact, associative and commutative.
KM_HD Top2 top2_merge(const Top2& x, const Top2& y) {
  const bool y_first = ahead(y.v1, y.k1, x.v1, x.k1);
  Top2 r = y_first ? y : x;
  const float other = y_first ? x.v1 : y.v1;
  r.v2 = fmaxf(r.v2, other);
  return r;
}

// Lane `lane` of `lanes` scans clusters lane, lane + lanes, ... of one token's similarity row.
KM_HD Top2 lane_top2(const float* S_row, float inv_norm, const float* price, int c, int lane,
                     int lanes) {
  Top2 t = top2_init();
  for (int k = lane; k < c; k += lanes) {
    const float a = S_row[k] * inv_norm;
    top2_add(t, a, a - price[k], k);
  }
  return t;
}

// The bid a token places on its best cluster: a_ik1 - v2 + eps (needs c >= 2).
KM_HD float bid_value(const Top2& t, float eps) { return (t.a1 - t.v2) + eps; }

// ------------------------------------------------------------------ cluster resolution ----

// The kept bids of a cluster form a heap with the worst (lowest bid, then highest token id) at
// the root.
KM_HD bool worse(float ba, int32_t ta, float bb, int32_t tb) {
  return ba < bb || (ba == bb && ta > tb);
}

KM_HD void heap_swap(float* hb, int32_t* ht, int64_t i, int64_t j) {
  const float b = hb[i];
  hb[i] = hb[j];
  hb[j] = b;
  const int32_t t = ht[i];
  ht[i] = ht[j];
  ht[j] = t;
}

KM_HD void heap_up(float* hb, int32_t* ht, int64_t i) {
  while (i > 0) {
    const int64_t p = (i - 1) >> 1;
    if (!worse(hb[i], ht[i], hb[p], ht[p])) break;
    heap_swap(hb, ht, i, p);
    i = p;
  }
}

KM_HD void heap_down(float* hb, int32_t* ht, int64_t n, int64_t i) {
  for (;;) {
    const int64_t l = 2 * i + 1, r = l + 1;
    int64_t m = i;
    if (l < n && worse(hb[l], ht[l], hb[m], ht[m])) m = l;
    if (r < n && worse(hb[r], ht[r], hb[m], ht[m])) m = r;
    if (m == i) return;
    heap_swap(hb, ht, i, m);
    i = m;
  }
}

// Device state of the auction.  U lists the tokens without a cluster; entry t of bid_k,
// bid_beta and pos belongs to the token U[t].
struct Auction {
  int64_t v;
  int c;
  int64_t b;
  float* price;       // c
  float* slot_bid;    // c x b kept bids (heap per cluster)
  int32_t* slot_tok;  // c x b their tokens
  int32_t* fill;      // c kept bids per cluster
  int32_t* cnt;       // c bids received this round (zero between rounds)
  int32_t* off;       // c start of each cluster's bids in inbox
  int32_t* inbox;     // v positions t, grouped by cluster
  const int32_t* U;   // v tokens bidding this round
  int32_t* U_next;    // v tokens left without a cluster after it
  int32_t* n_next;    // 1 their number
  int32_t* bid_k;     // v
  float* bid_beta;    // v
  int32_t* pos;       // v position of the bid among its cluster's bids
};

// Merges the bids a cluster received this round into the bids it keeps; the b best stay, the
// others (evicted holders and rejected bidders) are listed for the next round.  The kept set is
// the b best of (kept before) + (received) whatever order the bids arrive in.
KM_HD void resolve_cluster(int k, const Auction& s) {
  const int32_t m = s.cnt[k];
  if (m == 0) return;
  s.cnt[k] = 0;
  float* hb = s.slot_bid + (int64_t)k * s.b;
  int32_t* ht = s.slot_tok + (int64_t)k * s.b;
  int64_t n = s.fill[k];
  const int32_t o = s.off[k];
  for (int32_t j = 0; j < m; ++j) {
    const int32_t t = s.inbox[o + j];
    const int32_t tok = s.U[t];
    const float beta = s.bid_beta[t];
    if (n < s.b) {
      hb[n] = beta;
      ht[n] = tok;
      heap_up(hb, ht, n);
      ++n;
    } else if (worse(hb[0], ht[0], beta, tok)) {
      const int32_t out = ht[0];
      hb[0] = beta;
      ht[0] = tok;
      heap_down(hb, ht, n, 0);
      s.U_next[fetch_add(s.n_next, 1)] = out;
    } else {
      s.U_next[fetch_add(s.n_next, 1)] = tok;
    }
  }
  s.fill[k] = (int32_t)n;
  if (n == s.b) s.price[k] = hb[0];
}

// Bidder t's entry in its cluster's group of the inbox.
KM_HD void scatter_bid(const Auction& s, int64_t t) {
  s.inbox[s.off[s.bid_k[t]] + s.pos[t]] = (int32_t)t;
}

// ------------------------------------------------------------------ C2T and Eq.5 ----------

KM_HD void sift_down_max(int32_t* a, int64_t i, int64_t len) {
  for (;;) {
    const int64_t l = 2 * i + 1, r = l + 1;
    int64_t m = i;
    if (l < len && a[l] > a[m]) m = l;
    if (r < len && a[r] > a[m]) m = r;
    if (m == i) return;
    const int32_t x = a[i];
    a[i] = a[m];
    a[m] = x;
    i = m;
  }
}

// Row k of C2T: the tokens cluster k keeps, in ascending id order (heap sort in place).
KM_HD void sort_ascending(int32_t* a, int64_t n) {
  for (int64_t i = n / 2 - 1; i >= 0; --i) sift_down_max(a, i, n);
  for (int64_t e = n - 1; e > 0; --e) {
    const int32_t x = a[0];
    a[0] = a[e];
    a[e] = x;
    sift_down_max(a, 0, e);
  }
}

// Labels and C2T row k from the tokens cluster k keeps.
KM_HD void write_cluster(int k, const int32_t* slot_tok, int64_t b, int32_t* labels, int32_t* C2T) {
  int32_t* row = C2T + (int64_t)k * b;
  for (int64_t m = 0; m < b; ++m) {
    const int32_t tok = slot_tok[(int64_t)k * b + m];
    labels[tok] = k;
    row[m] = tok;
  }
  sort_ascending(row, b);
}

// Given labels: token i joins the tokens its cluster keeps.  Returns false for a label out of
// range or a cluster past b tokens (the token is then dropped).
KM_HD bool slot_from_label(int64_t i, const int32_t* labels, int c, int64_t b, int32_t* fill,
                           int32_t* slot_tok) {
  const int32_t k = labels[i];
  if (k < 0 || k >= c) return false;
  const int32_t p = fetch_add(&fill[k], 1);
  if (p >= b) return false;
  slot_tok[(int64_t)k * b + p] = (int32_t)i;
  return true;
}

// Column j of sum_{i in k} x_i, the members taken in C2T order.
KM_HD float member_sum(const uint16_t* E, const float* inv_norm, const int32_t* members, int64_t b,
                       int64_t d, int64_t j) {
  float acc = 0.f;
  for (int64_t m = 0; m < b; ++m) {
    const int32_t tok = members[m];
    acc = fma_rn(bf16_to_f32(E[(int64_t)tok * d + j]), inv_norm[tok], acc);
  }
  return acc;
}

// |sum_{i in k} x_i| from its d columns, accumulated in column order.
KM_HD float column_norm(const float* acc, int64_t d) {
  float ss = 0.f;
  for (int64_t j = 0; j < d; ++j) ss = fma_rn(acc[j], acc[j], ss);
  return sqrt_rn(ss);
}

// Column j of the updated centre: the member sum over its norm (0 for a degenerate cluster).
KM_HD float centre_value(float acc, float norm) { return norm > 0.f ? div_rn(acc, norm) : 0.f; }

// Eq.4 after the update: -sum_k |sum_{i in k} x_i|, summed as `parts` strided partial sums.
KM_HD double objective_part(const float* norms, int c, int part, int parts) {
  double s = 0.0;
  for (int k = part; k < c; k += parts) s += (double)norms[k];
  return s;
}

KM_HD double objective_total(const double* parts, int n) {
  double s = 0.0;
  for (int t = 0; t < n; ++t) s += parts[t];
  return -s;
}

constexpr int kObjectiveParts = 256;

// ------------------------------------------------------------------ the iteration loop -----

struct Config {
  int64_t v, d;
  int c;
  int64_t b;
  int iters;
  float eps_first, eps_final, eps_ratio;
  int64_t max_rounds;
};

// Epsilon scaling: the first phase bids with eps = 0.25 (cosines lie in [-1, 1]), each later
// phase with eps / 8, down to the caller's eps.  max_rounds <= 0 takes 2^22 rounds.
inline Config make_config(int64_t v, int64_t d, int64_t c, int iters, float eps, int64_t max_rounds) {
  Config cfg;
  cfg.v = v;
  cfg.d = d;
  cfg.c = (int)c;
  cfg.b = v / c;
  cfg.iters = iters;
  cfg.eps_first = 0.25f;
  cfg.eps_final = eps;
  cfg.eps_ratio = 8.f;
  cfg.max_rounds = max_rounds > 0 ? max_rounds : (int64_t(1) << 22);
  return cfg;
}

enum Outcome { kDone = 0, kBadInit = 1, kZeroRow = 2, kDegenerate = 3, kRoundLimit = 4, kBackend = 5 };

struct Progress {
  int iters_done = 0;
  int64_t rounds = 0;
};

// Backend interface (every call returns false on a backend failure):
//   row_norms(&zero_rows)      1/|e_i| of every token; counts zero rows
//   init_centres(&bad)         c_k = x_{init[k]}; counts init tokens out of range or repeated
//   similarities()             S[i][k] = e_i . c_k with the BF16 centres
//   zero_prices(), reset_phase()   prices 0; no token assigned, every token listed to bid
//   one_cluster()              c == 1: every token in cluster 0
//   round(n, eps)              one Jacobi round for the n listed tokens
//   next_count(&n)             tokens left without a cluster; makes them the next list
//   slots_from_labels(&bad)    given labels: each cluster keeps its tokens; counts clusters whose
//                              size is not b and labels out of range
//   finish_labels(first, &changed)  labels and C2T from the kept bids; labels changed vs the last
//   update_centres(t, &degenerate)  Eq.5 and the objective of iteration t

// The equal-size assignment for the centres the backend scores with (prices start at 0).
template <class Backend>
Outcome auction(Backend& be, const Config& cfg, Progress& pr) {
  if (cfg.c == 1) return (be.zero_prices() && be.one_cluster()) ? kDone : kBackend;
  if (!be.zero_prices()) return kBackend;
  float eps = cfg.eps_first > cfg.eps_final ? cfg.eps_first : cfg.eps_final;
  for (;;) {
    if (!be.reset_phase()) return kBackend;
    int64_t left = cfg.v;
    while (left > 0) {
      if (++pr.rounds > cfg.max_rounds) return kRoundLimit;
      if (!be.round(left, eps)) return kBackend;
      if (!be.next_count(&left)) return kBackend;
    }
    if (eps <= cfg.eps_final) return kDone;
    eps = eps / cfg.eps_ratio;
    if (eps < cfg.eps_final) eps = cfg.eps_final;
  }
}

// The assignment half-step alone, for centres given by the caller.
template <class Backend>
Outcome assign_only(Backend& be, const Config& cfg, Progress& pr) {
  int64_t n = 0;
  if (!be.row_norms(&n)) return kBackend;
  if (n) return kZeroRow;
  if (cfg.c > 1 && !be.similarities()) return kBackend;  // one cluster needs no scores
  const Outcome o = auction(be, cfg, pr);
  if (o != kDone) return o;
  return be.finish_labels(true, &n) ? kDone : kBackend;
}

// The update half-step (Eq.5) alone, for labels given by the caller.
template <class Backend>
Outcome update_only(Backend& be, const Config& cfg) {
  int64_t n = 0;
  if (!be.row_norms(&n)) return kBackend;
  if (n) return kZeroRow;
  if (!be.slots_from_labels(&n)) return kBackend;
  if (n) return kBadInit;
  if (!be.finish_labels(true, &n)) return kBackend;
  if (!be.update_centres(0, &n)) return kBackend;
  return n ? kDegenerate : kDone;
}

// Equal-size spherical k-means from the initial centres c_k = x_{init[k]}: alternate the two
// half-steps until the labels repeat or `iters` iterations have run.
template <class Backend>
Outcome run(Backend& be, const Config& cfg, Progress& pr) {
  int64_t n = 0;
  if (!be.row_norms(&n)) return kBackend;
  if (n) return kZeroRow;
  if (!be.init_centres(&n)) return kBackend;
  if (n) return kBadInit;
  for (int t = 0; t < cfg.iters; ++t) {
    if (cfg.c > 1 && !be.similarities()) return kBackend;
    const Outcome o = auction(be, cfg, pr);
    if (o != kDone) return o;
    int64_t changed = 0;
    if (!be.finish_labels(t == 0, &changed)) return kBackend;
    if (t > 0 && changed == 0) break;  // a fixed point: the last update already used these labels
    if (!be.update_centres(t, &n)) return kBackend;
    if (n) return kDegenerate;
    pr.iters_done = t + 1;
  }
  return kDone;
}

}  // namespace fhkm

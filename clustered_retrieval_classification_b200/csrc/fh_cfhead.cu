// fh_cfhead.cu — the coarse-fine LM head (include/fh_cfhead.h): per-tile look-up tables, coarse
// scores over the vocabulary from the streamed 4-bit index map, exact top-k selection, exact logits of
// the k candidates and the token decision.
//
// Page "Fast LM Head via Coarse-Fine Decomposition and Tile-Wise Weight Clustering", abstract: a
// compact codebook and an index map from tile-wise k-means; full-vocabulary coarse scores through
// tile-wise LUTs and index streaming; exact GEMV on the top-k candidates only.
//
// Kernels, one call (grid.y = query):
//   k_cf_lut      LUT[q][t][j] = Cb[t][j]·h_q[t·w ..) (fp32, column order); zeroes the query's
//                 histogram and list counters for this call
//   k_cf_coarse   each block: the query's LUT into shared memory (one bulk copy), the bound
//                 R = Σ_t max_j |LUT[t][j]| (|ŝ| <= R) and from it the binning; then one thread per
//                 token: ŝ_u = Σ_t LUT[t][code] as four partial sums (tiles t mod 4), 32-bit code words
//                 read coalesced (one word row = 8 tiles of 32 consecutive tokens = 128 bytes) in
//                 batches of 16 with the next batch in flight; a 4096-bin histogram of the scores
//   k_cf_compact  each block: the boundary bin d* from the summed histogram (where the count from the
//                 top reaches k); its tokens above d* go to the candidate list, the boundary bin's
//                 (score, id) pairs to the boundary list (warp-aggregated appends)
//   k_cf_resolve  one block per query: the boundary pairs ranked exactly — radix passes on the score's
//                 order-preserving image, then on the token id among equal scores — and the `need`
//                 best appended to the candidate list
//   k_cf_exact    one warp per candidate row of E: the exact logit (fp32 accumulation of BF16
//                 products), the Gumbel term when sampling, a packed 64-bit arg-max; the last block of
//                 the query writes the token and resets the query's maximum and ticket
// Bins: the score times a power of two 2^-e (2^e > R, exact), 256 bins per binade of its magnitude over
// eight binades on each side of zero — a monotone integer function of the bit pattern, so a bin holds
// a contiguous range of scores.
#include <cuda_runtime.h>

#include <cstdarg>
#include <cstdio>
#include <new>

#include "../../include/fh_cfhead.h"
#include "fh_device.cuh"
#include "fh_kernels.cuh"
#include "fh_nvtx.cuh"

struct fh_cf_index {
  fh_cf_desc desc;
  int num_sms;
};

namespace fh {
fh_status report(fh_status st, const char* fmt, ...);  // fh_api.cu: sets fh_last_error()
}

namespace {

using namespace fh;

constexpr int kCfBins = 4096;
constexpr uint32_t kCfFineLo = 0x3B800000u;  // bit pattern of 2^-8
constexpr uint32_t kCfFine = 2046u;          // fine bins per sign
constexpr int kCfThreads = 256;
constexpr size_t kCfHeader = 5120;           // status word, tickets, maxima, list counters
constexpr size_t kCfTicketOff = 16, kCfBestOff = 1024, kCfCandCntOff = 1536, kCfBndCntOff = 1792;

__device__ __forceinline__ uint32_t cf_bin(float key, float scale) {
  const uint32_t u = __float_as_uint(key * scale);
  const uint32_t a = u & 0x7FFFFFFFu;
  const bool neg = (u >> 31) != 0u;
  if (a < kCfFineLo) return (neg && a != 0u) ? 2047u : 2048u;
  const uint32_t t = (a - kCfFineLo) >> 15;
  if (neg) return t >= kCfFine ? 0u : kCfFine - t;
  return t >= kCfFine ? 4095u : 2049u + t;
}

struct CfParams {
  const uint16_t* E;        // v x d BF16
  const float* cb;          // T x K x w
  const uint32_t* codes;    // T/8 x v
  const uint16_t* H;        // B x d BF16
  int64_t v, d;
  int w, K, T, k, B;
  int sample;
  float tau;
  uint64_t seed, step;
  float* lut;               // B x T x K
  float* scale;             // B
  uint32_t* hist;           // B x kCfBins
  float* coarse;            // B x v
  int32_t* cand;            // B x k
  unsigned long long* blist;  // B x v: (score image << 32) | token
  uint32_t* cand_cnt;       // B
  uint32_t* bnd_cnt;        // B
  uint32_t* tickets;        // B
  unsigned long long* best; // B
  int32_t* out_tok;         // B
  uint32_t* status;
};

// ------------------------------------------------------------------ look-up tables
// LUT[q][t][j] at (q·T + t)·16 + j: every tile takes 16 entries whatever K is (entries past K are
// zero), so the score loop addresses a tile's entries with compile-time offsets.
constexpr int kCfLutStride = FH_CF_MAX_K;
static_assert(kCfLutStride == 16, "4-bit codes index 16 entries");

__global__ void __launch_bounds__(kCfThreads) k_cf_lut(const CfParams p) {
  const int q = blockIdx.y;
  const int i = blockIdx.x * kCfThreads + threadIdx.x;
  if (blockIdx.x == 0) {  // this call's histogram and list counters start at zero
    for (int b = threadIdx.x; b < kCfBins; b += kCfThreads) p.hist[(size_t)q * kCfBins + b] = 0u;
    if (threadIdx.x == 0) {
      p.cand_cnt[q] = 0u;
      p.bnd_cnt[q] = 0u;
    }
  }
  if (i >= p.T * kCfLutStride) return;
  const int t = i / kCfLutStride, j = i % kCfLutStride;  // tile t, entry j (zero past K)
  float acc = 0.0f;
  if (j < p.K) {
    const float* c = p.cb + ((size_t)t * p.K + j) * p.w;
    const uint16_t* h = p.H + (size_t)q * p.d + (size_t)t * p.w;
    for (int e = 0; e < p.w; ++e) acc = fmaf(c[e], __uint_as_float((uint32_t)h[e] << 16), acc);
  }
  p.lut[(size_t)q * p.T * kCfLutStride + i] = acc;
}

// ------------------------------------------------------------------ coarse scores

constexpr int kCfWordsInFlight = 16;  // code words per batch; two batches are in flight

__global__ void __launch_bounds__(kCfThreads) k_cf_coarse(const CfParams p) {
  extern __shared__ __align__(16) float lut_s[];  // T x 16, then kCfBins histogram words
  __shared__ float red_s[kCfThreads / 32];
  __shared__ __align__(8) uint64_t lut_bar;
  const int q = blockIdx.y, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int TK = p.T * kCfLutStride;
  const int G8 = p.T / 8;
  const int64_t v = p.v;
  const int64_t u = (int64_t)blockIdx.x * kCfThreads + tid;  // one token per thread
  const uint32_t* col = p.codes + (u < v ? u : 0);
  // the query's look-up table in one bulk copy, while each thread requests its first word rows (the
  // barrier is initialised and made visible to the block before anyone waits on it)
  if (tid == 0) {
    mbar_init(&lut_bar, 1);
    fence_mbar_init();
  }
  __syncthreads();
  if (tid == 0) {
    mbar_arrive_expect_tx(&lut_bar, (uint32_t)TK * 4u);
    bulk_g2s(lut_s, p.lut + (size_t)q * TK, (uint32_t)TK * 4u, &lut_bar);
  }
  uint32_t wa[kCfWordsInFlight], wb[kCfWordsInFlight];
  auto load = [&](uint32_t (&w)[kCfWordsInFlight], int g0) {
#pragma unroll
    for (int g = 0; g < kCfWordsInFlight; ++g)
      w[g] = (g0 + g < G8 && u < v) ? __ldg(col + (size_t)(g0 + g) * v) : 0u;
  };
  load(wa, 0);
  uint32_t* hist_s = reinterpret_cast<uint32_t*>(lut_s + TK);
  for (int b = tid; b < kCfBins; b += kCfThreads) hist_s[b] = 0u;
  const bool lut_ok = mbar_wait(&lut_bar, 0u, p.status);
  if (!__syncthreads_and(lut_ok)) {  // (status recorded) the copy lands before the block leaves
    if (tid == 0) mbar_wait(&lut_bar, 0u, nullptr, 50000000ull);
    return;
  }
  // |ŝ_u| <= R = Σ_t max_j |LUT[t][j]| (fixed order: identical in every block)
  float part = 0.0f;
  for (int t = tid; t < p.T; t += kCfThreads) {
    float m = 0.0f;
    // entries in rotated order: the lanes of a warp read different banks
    for (int j = 0, jr = t % p.K; j < p.K; ++j, jr = (jr + 1 == p.K) ? 0 : jr + 1)
      m = fmaxf(m, fabsf(lut_s[t * kCfLutStride + jr]));
    part += m;
  }
  part = warp_sum(part);
  if (lane == 0) red_s[warp] = part;
  __syncthreads();
  float R = 0.0f;
#pragma unroll
  for (int w = 0; w < kCfThreads / 32; ++w) R += red_s[w];
  int e = 0;
  frexpf(R * 1.0625f + 1e-30f, &e);
  float scale = ldexpf(1.0f, -e);
  if (!(isfinite(scale) && scale > 0.0f)) scale = 1.0f;
  if (blockIdx.x == 0 && tid == 0) p.scale[q] = scale;

  if (u < v) {
    // Σ_t LUT[t][code] as four partial sums over the tiles t ≡ 0, 1, 2, 3 (mod 4), each in tile
    // order, then (s0 + s1) + (s2 + s3); the word batches alternate between two register sets so that
    // one is in flight while the other is summed
    float a0 = 0.0f, a1 = 0.0f, a2 = 0.0f, a3 = 0.0f;
    auto sum = [&](const uint32_t (&w)[kCfWordsInFlight], int g0) {
#pragma unroll
      for (int g = 0; g < kCfWordsInFlight; ++g) {
        if (g0 + g < G8) {
          const float* lt = lut_s + (size_t)(8 * (g0 + g)) * kCfLutStride;
          const uint32_t x = w[g];
          a0 += lt[0 * kCfLutStride + (x & 15u)];
          a1 += lt[1 * kCfLutStride + ((x >> 4) & 15u)];
          a2 += lt[2 * kCfLutStride + ((x >> 8) & 15u)];
          a3 += lt[3 * kCfLutStride + ((x >> 12) & 15u)];
          a0 += lt[4 * kCfLutStride + ((x >> 16) & 15u)];
          a1 += lt[5 * kCfLutStride + ((x >> 20) & 15u)];
          a2 += lt[6 * kCfLutStride + ((x >> 24) & 15u)];
          a3 += lt[7 * kCfLutStride + (x >> 28)];
        }
      }
    };
    for (int g0 = 0; g0 < G8; g0 += 2 * kCfWordsInFlight) {
      if (g0 + kCfWordsInFlight < G8) load(wb, g0 + kCfWordsInFlight);
      sum(wa, g0);
      if (g0 + 2 * kCfWordsInFlight < G8) load(wa, g0 + 2 * kCfWordsInFlight);
      if (g0 + kCfWordsInFlight < G8) sum(wb, g0 + kCfWordsInFlight);
    }
    const float acc = (a0 + a1) + (a2 + a3);
    p.coarse[(size_t)q * v + u] = acc;
    atomicAdd(&hist_s[cf_bin(acc, scale)], 1u);
  }
  __syncthreads();
  for (int b = tid; b < kCfBins; b += kCfThreads) {
    const uint32_t n = hist_s[b];
    if (n) atomicAdd(&p.hist[(size_t)q * kCfBins + b], n);
  }
}

// ------------------------------------------------------------------ boundary bin and compaction

// The boundary bin d* (where the count from the top first reaches k), the count above it and in it.
// Called by the whole block; ends with a __syncthreads.
struct CfBoundary {
  uint32_t dstar, above, m;
};

__device__ __forceinline__ CfBoundary cf_boundary(const uint32_t* hist, uint32_t k) {
  constexpr int HPT = kCfBins / kCfThreads;  // 16 consecutive bins per thread
  __shared__ unsigned long long wtot[kCfThreads / 32];
  __shared__ CfBoundary res;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  uint32_t hb[HPT], tot = 0;
#pragma unroll
  for (int u = 0; u < HPT; ++u) {
    hb[u] = hist[tid * HPT + u];
    tot += hb[u];
  }
  if (tid == 0) res = CfBoundary{0u, 0u, 0u};
  // keys in the bins above this thread's: suffix sum over the threads after it
  uint32_t incl = tot;  // inclusive prefix within the warp, from the top (lane 31 first)
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const uint32_t o = __shfl_down_sync(0xFFFFFFFFu, incl, off);
    if (lane + off < 32) incl += o;
  }
  if (lane == 0) wtot[warp] = incl;
  __syncthreads();
  uint32_t cum = incl - tot;
  for (int w2 = warp + 1; w2 < kCfThreads / 32; ++w2) cum += (uint32_t)wtot[w2];
#pragma unroll
  for (int u = HPT - 1; u >= 0; --u) {
    if (cum < k && cum + hb[u] >= k) res = CfBoundary{(uint32_t)(tid * HPT + u), cum, hb[u]};
    cum += hb[u];
  }
  __syncthreads();
  return res;
}

__global__ void __launch_bounds__(kCfThreads) k_cf_compact(const CfParams p) {
  __shared__ unsigned long long wsum[kCfThreads / 32];
  __shared__ uint32_t base_s[2];
  const int q = blockIdx.y, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const uint32_t k = (uint32_t)p.k;
  const bool all = (int64_t)k >= p.v;
  CfBoundary bd{0u, 0u, 0u};
  if (!all) bd = cf_boundary(p.hist + (size_t)q * kCfBins, k);
  const uint32_t need = all ? 0u : k - bd.above;
  const bool whole = need == bd.m;  // the boundary bin is taken whole
  const float scale = p.scale[q];
  const int64_t v = p.v;
  const int64_t u0 = v * blockIdx.x / gridDim.x, u1 = v * (blockIdx.x + 1) / gridDim.x;
  for (int64_t base = u0; base < u1; base += kCfThreads) {
    const int64_t u = base + tid;
    bool is_c = false, is_b = false;
    float s = 0.0f;
    if (u < u1) {
      s = p.coarse[(size_t)q * v + u];
      const uint32_t bn = all ? 0u : cf_bin(s, scale);
      is_c = all || bn > bd.dstar || (bn == bd.dstar && whole);
      is_b = !is_c && bn == bd.dstar;
    }
    // one block-wide exclusive scan of both flags (candidate count high, boundary count low), then
    // one append per list and chunk
    const unsigned long long mine = ((unsigned long long)is_c << 32) | (unsigned long long)is_b;
    unsigned long long incl = mine;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const unsigned long long o = __shfl_up_sync(0xFFFFFFFFu, incl, off);
      if (lane >= off) incl += o;
    }
    if (lane == 31) wsum[warp] = incl;
    __syncthreads();
    unsigned long long before = 0ull, total = 0ull;
#pragma unroll
    for (int w = 0; w < kCfThreads / 32; ++w) {
      before += w < warp ? wsum[w] : 0ull;
      total += wsum[w];
    }
    if (tid == 0) {
      const uint32_t nc = (uint32_t)(total >> 32), nb = (uint32_t)total;
      base_s[0] = nc ? atomicAdd(&p.cand_cnt[q], nc) : 0u;
      base_s[1] = nb ? atomicAdd(&p.bnd_cnt[q], nb) : 0u;
    }
    __syncthreads();
    const unsigned long long ex = before + incl - mine;
    if (is_c) {
      const uint32_t slot = base_s[0] + (uint32_t)(ex >> 32);
      if (slot < k) p.cand[(size_t)q * k + slot] = (int32_t)u;
      else set_status(p.status, kStatusIndex);
    }
    if (is_b) {
      const uint32_t slot = base_s[1] + (uint32_t)ex;
      p.blist[(size_t)q * v + slot] = ((unsigned long long)float_key(s) << 32) | (unsigned long long)u;
    }
    __syncthreads();  // wsum and base_s are reused by the next chunk
  }
}

// ------------------------------------------------------------------ exact boundary ranking

constexpr int kCfResolveThreads = 1024;

// In the block's shared histogram, the digit d where the count from the top (desc) or from the bottom
// (asc) first reaches `target`; returns d and the count strictly before it in that direction.
// The first digit, in the given order, at which the running count reaches `target`, and the count
// before it.  Warp 0: lane l sums the 8 digits at ordered positions 8l .. 8l+7, a warp scan finds the
// lane where the running count crosses `target`, and that lane walks its 8 digits.
__device__ __forceinline__ void cf_pick_digit(const uint32_t* h256, uint32_t target, bool desc,
                                              uint32_t* digit, uint32_t* before) {
  if (threadIdx.x < 32) {
    const int lane = threadIdx.x;
    uint32_t c[8], sum = 0;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int pos = 8 * lane + i;
      c[i] = h256[desc ? 255 - pos : pos];
      sum += c[i];
    }
    uint32_t incl = sum;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t y = __shfl_up_sync(0xFFFFFFFFu, incl, o);
      if (lane >= o) incl += y;
    }
    const uint32_t excl = incl - sum;
    if (excl < target && target <= incl) {
      uint32_t cum = excl;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        if (cum + c[i] >= target) {
          const int pos = 8 * lane + i;
          *digit = (uint32_t)(desc ? 255 - pos : pos);
          *before = cum;
          break;
        }
        cum += c[i];
      }
    }
  }
}

constexpr uint32_t kCfResolveStage = 12288;  // boundary entries staged in shared memory (96 KiB)

__global__ void __launch_bounds__(kCfResolveThreads) k_cf_resolve(const CfParams p) {
  extern __shared__ __align__(16) unsigned long long bl_s[];  // kCfResolveStage entries
  __shared__ uint32_t h256[256];
  __shared__ uint32_t digit_s, before_s;
  const int q = blockIdx.y, tid = threadIdx.x;
  const uint32_t k = (uint32_t)p.k;
  if ((int64_t)k >= p.v) return;
  const uint32_t have = p.cand_cnt[q];  // the certain candidates compacted so far
  const uint32_t m = p.bnd_cnt[q];
  if (have >= k || m == 0u) return;
  uint32_t need = k - have;
  // the boundary list, read once into shared memory when it fits (the passes below re-read it)
  const unsigned long long* bl = p.blist + (size_t)q * p.v;
  if (m <= kCfResolveStage) {
    for (uint32_t i = tid; i < m; i += kCfResolveThreads) bl_s[i] = bl[i];
    bl = bl_s;
    __syncthreads();
  }
  // 1. the exact threshold image T: 8-bit radix passes from the top of the score images
  uint32_t prefix = 0u, mask = 0u;
  for (int shift = 24; shift >= 0; shift -= 8) {
    for (int i = tid; i < 256; i += kCfResolveThreads) h256[i] = 0u;
    __syncthreads();
    for (uint32_t i = tid; i < m; i += kCfResolveThreads) {
      const uint32_t img = (uint32_t)(bl[i] >> 32);
      if ((img & mask) == prefix) atomicAdd(&h256[(img >> shift) & 255u], 1u);
    }
    __syncthreads();
    cf_pick_digit(h256, need, true, &digit_s, &before_s);
    __syncthreads();
    prefix |= digit_s << shift;
    mask |= 255u << shift;
    need -= before_s;
    __syncthreads();
  }
  // 2. among the scores equal to T, the `need` smallest token ids: radix passes from the bottom
  uint32_t iprefix = 0u, imask = 0u;
  for (int shift = 16; shift >= 0; shift -= 8) {
    for (int i = tid; i < 256; i += kCfResolveThreads) h256[i] = 0u;
    __syncthreads();
    for (uint32_t i = tid; i < m; i += kCfResolveThreads) {
      const unsigned long long e = bl[i];
      const uint32_t id = (uint32_t)e;
      if ((uint32_t)(e >> 32) == prefix && (id & imask) == iprefix)
        atomicAdd(&h256[(id >> shift) & 255u], 1u);
    }
    __syncthreads();
    cf_pick_digit(h256, need, false, &digit_s, &before_s);
    __syncthreads();
    iprefix |= digit_s << shift;
    imask |= 255u << shift;
    need -= before_s;
    __syncthreads();
  }
  // 3. append: scores above T, and the ids up to the last one taken at T (ids are distinct)
  for (uint32_t i = tid; i < m; i += kCfResolveThreads) {
    const unsigned long long e = bl[i];
    const uint32_t img = (uint32_t)(e >> 32), id = (uint32_t)e;
    if (img > prefix || (img == prefix && id <= iprefix)) {
      const uint32_t slot = atomicAdd(&p.cand_cnt[q], 1u);
      if (slot < k) p.cand[(size_t)q * k + slot] = (int32_t)id;
      else set_status(p.status, kStatusIndex);
    }
  }
}

// ------------------------------------------------------------------ exact logits and the decision

__global__ void __launch_bounds__(kCfThreads) k_cf_exact(const CfParams p) {
  extern __shared__ __align__(16) uint4 h_s[];  // the query, d / 8 chunks
  __shared__ unsigned long long wbest[kCfThreads / 32];
  __shared__ bool last_s;
  const int q = blockIdx.y, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int nch = (int)(p.d / 8);
  for (int i = tid; i < nch; i += kCfThreads) h_s[i] = reinterpret_cast<const uint4*>(p.H + (size_t)q * p.d)[i];
  __syncthreads();
  const int nwarps = gridDim.x * (kCfThreads / 32);
  unsigned long long best = 0ull;
  for (int r = blockIdx.x * (kCfThreads / 32) + warp; r < p.k; r += nwarps) {
    const uint32_t u = (uint32_t)p.cand[(size_t)q * p.k + r];
    const uint4* row = reinterpret_cast<const uint4*>(p.E + (size_t)u * p.d);
    float acc = 0.0f;
    for (int ch = lane; ch < nch; ch += 32) acc = dot8_bf16(ld_stream_v4(row + ch), h_s[ch], acc);
    const float z = warp_sum(acc);
    float val = z;
    if (p.sample) val = z / p.tau + gumbel_from_u32(philox_word(p.seed, p.step, (uint32_t)q, 1u, u));
    const unsigned long long pk = pack_best(val, u);
    best = pk > best ? pk : best;
  }
  if (lane == 0) wbest[warp] = best;
  __syncthreads();
  if (tid == 0) {
    unsigned long long bb = 0ull;
    for (int w = 0; w < kCfThreads / 32; ++w) bb = wbest[w] > bb ? wbest[w] : bb;
    if (bb) atomicMax(&p.best[q], bb);
    __threadfence();
    last_s = atomicAdd(&p.tickets[q], 1u) + 1u == gridDim.x;
  }
  __syncthreads();
  if (last_s && tid == 0) {
    __threadfence();
    const unsigned long long fin = atomicExch(&p.best[q], 0ull);
    p.out_tok[q] = fin ? (int32_t)best_id(fin) : -1;
    p.tickets[q] = 0u;
  }
}

// ------------------------------------------------------------------ host side

size_t up(size_t x) { return (x + 255) / 256 * 256; }

struct CfLayout {
  size_t lut, scale, hist, coarse, cand, blist, total;
};

CfLayout cf_layout(const fh_cf_index* idx, int B, int k) {
  const fh_cf_desc& D = idx->desc;
  const int64_t T = D.d / D.w;
  CfLayout L;
  size_t off = kCfHeader;
  auto take = [&](size_t bytes) {
    const size_t at = off;
    off = up(off + bytes);
    return at;
  };
  L.lut = take((size_t)B * T * kCfLutStride * 4);
  L.scale = take((size_t)B * 4);
  L.hist = take((size_t)B * kCfBins * 4);
  L.coarse = take((size_t)B * D.v * 4);
  L.cand = take((size_t)B * k * 4);
  L.blist = take((size_t)B * D.v * 8);
  L.total = off;
  return L;
}

fh_status cf_check(const fh_cf_index* idx, const void* H, int B, void* ws, size_t ws_bytes, int k) {
  if (!idx) return report(FH_ERR_ARG, "index handle is NULL");
  if (!H || (reinterpret_cast<uintptr_t>(H) & 15u))
    return report(FH_ERR_ARG, "H must be a 16-byte aligned device pointer");
  if (B < 1 || B > FH_MAX_BATCH) return report(FH_ERR_ARG, "B=%d outside [1, %d]", B, FH_MAX_BATCH);
  if (k < 1 || (int64_t)k > idx->desc.v) return report(FH_ERR_ARG, "k=%d outside [1, v]", k);
  if (!ws) return report(FH_ERR_WORKSPACE, "workspace is NULL");
  if (reinterpret_cast<uintptr_t>(ws) % 256) return report(FH_ERR_WORKSPACE, "workspace must be 256-byte aligned");
  const size_t need = cf_layout(idx, B, k).total;
  if (ws_bytes < need) return report(FH_ERR_WORKSPACE, "workspace has %zu bytes, %zu needed", ws_bytes, need);
  return FH_OK;
}

CfParams cf_params(const fh_cf_index* idx, const void* H, int B, int k, void* ws) {
  const fh_cf_desc& D = idx->desc;
  const CfLayout L = cf_layout(idx, B, k);
  char* base = static_cast<char*>(ws);
  CfParams p = {};
  p.E = static_cast<const uint16_t*>(D.E);
  p.cb = D.codebooks;
  p.codes = D.codes;
  p.H = static_cast<const uint16_t*>(H);
  p.v = D.v;
  p.d = D.d;
  p.w = D.w;
  p.K = D.K;
  p.T = (int)(D.d / D.w);
  p.k = k;
  p.B = B;
  p.lut = reinterpret_cast<float*>(base + L.lut);
  p.scale = reinterpret_cast<float*>(base + L.scale);
  p.hist = reinterpret_cast<uint32_t*>(base + L.hist);
  p.coarse = reinterpret_cast<float*>(base + L.coarse);
  p.cand = reinterpret_cast<int32_t*>(base + L.cand);
  p.blist = reinterpret_cast<unsigned long long*>(base + L.blist);
  p.cand_cnt = reinterpret_cast<uint32_t*>(base + kCfCandCntOff);
  p.bnd_cnt = reinterpret_cast<uint32_t*>(base + kCfBndCntOff);
  p.tickets = reinterpret_cast<uint32_t*>(base + kCfTicketOff);
  p.best = reinterpret_cast<unsigned long long*>(base + kCfBestOff);
  p.status = reinterpret_cast<uint32_t*>(base);
  return p;
}

fh_status cuda_err(cudaError_t e, const char* what) {
  return report(FH_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

// Blocks per query for the vocabulary-wide kernels: about two waves of 256-thread blocks in all.
int cf_blocks(const fh_cf_index* idx, int B, int64_t work_items) {
  int64_t g = (2 * (int64_t)idx->num_sms + B - 1) / B;
  const int64_t max_g = (work_items + kCfThreads - 1) / kCfThreads;
  if (g > max_g) g = max_g;
  return (int)(g < 1 ? 1 : g);
}

// The look-up tables and the coarse scores (with their histogram) of every query.
cudaError_t cf_launch_coarse(const fh_cf_index* idx, const CfParams& p, cudaStream_t st) {
  const int TK = p.T * kCfLutStride;
  k_cf_lut<<<dim3((TK + kCfThreads - 1) / kCfThreads, p.B), kCfThreads, 0, st>>>(p);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const size_t smem = (size_t)TK * 4 + (size_t)kCfBins * 4;
  e = set_smem_attr(reinterpret_cast<const void*>(k_cf_coarse), smem);
  if (e != cudaSuccess) return e;
  k_cf_coarse<<<dim3((unsigned)((p.v + kCfThreads - 1) / kCfThreads), p.B), kCfThreads, smem, st>>>(p);
  return cudaGetLastError();
}

}  // namespace

extern "C" {

fh_status fh_cf_load(const fh_cf_desc* desc, fh_cf_index** out) {
  if (out) *out = nullptr;
  if (!desc || !out) return report(FH_ERR_ARG, "desc or out is NULL");
  const fh_cf_desc& D = *desc;
  if (D.v < 1 || D.d < 1 || D.w < 1 || D.K < 1) return report(FH_ERR_SHAPE, "non-positive size");
  if (D.v >= (int64_t{1} << 24)) return report(FH_ERR_SHAPE, "v must be below 2^24");
  if (D.w > 64) return report(FH_ERR_SHAPE, "w=%d exceeds 64", D.w);
  if (D.K > FH_CF_MAX_K) return report(FH_ERR_SHAPE, "K=%d exceeds %d (4-bit codes)", D.K, FH_CF_MAX_K);
  if (D.d % (8 * (int64_t)D.w)) return report(FH_ERR_SHAPE, "d must be a multiple of 8 tiles (8*w)");
  if (D.d > FH_MAX_D) return report(FH_ERR_SHAPE, "d=%lld exceeds %d", (long long)D.d, FH_MAX_D);
  if ((D.d / D.w) * D.K > 32768) return report(FH_ERR_UNSUPPORTED, "T*K above 32768 look-up entries");
  if (!D.E || !D.codebooks || !D.codes) return report(FH_ERR_ARG, "E, codebooks and codes are required");
  if (reinterpret_cast<uintptr_t>(D.E) & 15u) return report(FH_ERR_ARG, "E must be 16-byte aligned");
  int dev = 0, sms = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (e != cudaSuccess) return cuda_err(e, "device query");
  fh_cf_index* idx = new (std::nothrow) fh_cf_index;
  if (!idx) return report(FH_ERR_ARG, "out of host memory");
  idx->desc = D;
  idx->num_sms = sms;
  *out = idx;
  return FH_OK;
}

void fh_cf_free(fh_cf_index* idx) { delete idx; }

size_t fh_cf_workspace_bytes(const fh_cf_index* idx, int B, int k) {
  if (!idx || B < 1 || B > FH_MAX_BATCH || k < 1 || (int64_t)k > idx->desc.v) return 0;
  return cf_layout(idx, B, k).total;
}

fh_status fh_cf_coarse_scores(const fh_cf_index* idx, const void* H, int B, float* out, void* ws,
                              size_t ws_bytes, fh_stream stream) {
  FH_NVTX_RANGE("fh_cf_coarse_scores");
  fh_status r = cf_check(idx, H, B, ws, ws_bytes, 1);
  if (r != FH_OK) return r;
  if (!out) return report(FH_ERR_ARG, "out is NULL");
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  CfParams p = cf_params(idx, H, B, 1, ws);
  p.coarse = out;
  cudaError_t e = cf_launch_coarse(idx, p, st);
  if (e != cudaSuccess) return cuda_err(e, "coarse-score launch");
  return FH_OK;
}

fh_status fh_cf_head(const fh_cf_index* idx, const void* H, int B, int k, int sample, float tau,
                     uint64_t seed, uint64_t step, int32_t* out_tok, void* ws, size_t ws_bytes,
                     fh_stream stream, int32_t* dbg_cand, float* dbg_coarse) {
  FH_NVTX_RANGE("fh_cf_head");
  fh_status r = cf_check(idx, H, B, ws, ws_bytes, k);
  if (r != FH_OK) return r;
  if (!out_tok) return report(FH_ERR_ARG, "out_tok is NULL");
  if (sample && !(tau > 0.0f)) return report(FH_ERR_ARG, "tau must be > 0");
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  CfParams p = cf_params(idx, H, B, k, ws);
  p.sample = sample;
  p.tau = tau;
  p.seed = seed;
  p.step = step;
  p.out_tok = out_tok;
  cudaError_t e = cf_launch_coarse(idx, p, st);
  if (e != cudaSuccess) return cuda_err(e, "coarse-score launch");
  k_cf_compact<<<dim3(cf_blocks(idx, B, p.v), B), kCfThreads, 0, st>>>(p);
  if ((e = cudaGetLastError()) != cudaSuccess) return cuda_err(e, "compaction launch");
  if ((e = set_smem_attr(reinterpret_cast<const void*>(k_cf_resolve), kCfResolveStage * 8u)) != cudaSuccess)
    return cuda_err(e, "resolve attribute");
  k_cf_resolve<<<dim3(1, B), kCfResolveThreads, kCfResolveStage * 8u, st>>>(p);
  if ((e = cudaGetLastError()) != cudaSuccess) return cuda_err(e, "boundary launch");
  if (dbg_coarse &&
      (e = cudaMemcpyAsync(dbg_coarse, p.coarse, (size_t)B * p.v * 4, cudaMemcpyDeviceToDevice, st)) != cudaSuccess)
    return cuda_err(e, "debug copy");
  if (dbg_cand &&
      (e = cudaMemcpyAsync(dbg_cand, p.cand, (size_t)B * k * 4, cudaMemcpyDeviceToDevice, st)) != cudaSuccess)
    return cuda_err(e, "debug copy");
  const int warps_per_block = kCfThreads / 32;
  int gx = (k + warps_per_block - 1) / warps_per_block;
  const int cap = (4 * idx->num_sms + B - 1) / B;
  if (gx > cap) gx = cap;
  const size_t smem = (size_t)p.d * 2;
  if ((e = set_smem_attr(reinterpret_cast<const void*>(k_cf_exact), smem)) != cudaSuccess)
    return cuda_err(e, "exact-logit attributes");
  k_cf_exact<<<dim3(gx, B), kCfThreads, smem, st>>>(p);
  if ((e = cudaGetLastError()) != cudaSuccess) return cuda_err(e, "exact-logit launch");
  return FH_OK;
}

}  // extern "C"

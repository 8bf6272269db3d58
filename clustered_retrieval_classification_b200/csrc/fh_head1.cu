// fh_head1.cu — the batch-1 FlashHead head as one persistent kernel (one block per SM).
//
// At batch 1 the whole call moves ~66 MB (Llama-shaped head), about 10 µs of HBM time on a B200, so
// every launch boundary and every serial step between the two bandwidth phases shows.  One kernel
// runs the whole path (FlashHead notes, overall architecture and Figure 1):
//
//   0. Prologue: one Stage-1 copy per warp (index data only) is issued at once; the kernel then waits
//      for the preceding kernel of the stream (programmatic dependent launch) before it reads h or
//      touches the workspace, so the centroid stream starts during the predecessor's tail; h is
//      requested before the rest of the first copies (a small load queues behind the bulk copies in
//      flight on its SM).
//   1. Stage 1: each block streams its share of centroid rows (C, or the INT4 nibbles) through
//      per-warp shared-memory rings, computes s = C·h (or the Gumbel key s/τ + G), and counts each key
//      in a block histogram.  The bins are a monotone integer function of the exactly scaled key
//      (key·2^-e with 2^e above the bound ‖h‖ of unit centroids, or ‖h‖/τ + 17 with the Gumbel term):
//      64 bins per binade of |key·2^-e| in [2^-8, 1) on each side of zero, so a key's bin and its
//      order inside the bin come from its bit pattern.
//   2. Exchange: the block adds its counts to the global histogram (one returning add per non-empty
//      bin, all in flight together), which gives every key a distinct position in its bin, and writes
//      one tagged word (call tag, cluster id, order inside the bin) per key at (bin, position).
//   3. Grid barrier = histogram poll: every block polls the summed histogram until its counts reach c
//      (bounded wait).  The scan of the counts gives the boundary bin d* holding the p-th key, the
//      number of keys above it, and for every rank of the Stage-2 list (bins from the top, positions
//      inside a bin, then the boundary bin's taken keys) the word that names its cluster.
//   4. Selection (FlashHead notes, Module 2): each block reads the words of the ranks its Stage-2
//      rows need — one round of loads — and, when it has boundary ranks, the boundary bin's words,
//      which it ranks exactly under (key desc, id asc).  A bin too full for the word table, or a
//      boundary bin that is not a fine bin, sends every block to the full selection instead (all keys
//      loaded, exact radix passes).
//   5. Stage 2 (FlashHead notes, Module 1 and Figure 1): the block streams its slice of the p·b
//      candidate rows (the cluster-major copy: a cluster is b contiguous rows), with the C2T rows of
//      its clusters copied first for the token ids, computes the exact logits and keeps the arg-max of
//      z (greedy, Eq. 2) or of z/τ + G' (sampling, Eq. 3).
//   6. Each block posts its best (value, token) as one packed 64-bit word to its slot and counts itself
//      in with a release add; block 0 waits for the G arrivals, reduces the slots, writes the token
//      and clears the histogram.
//
// Stage-2 slots follow the rank order; the arg-max does not depend on it, and the optional debug
// outputs are written in the canonical ascending order.
#include "fh_device.cuh"
#include "fh_kernels.cuh"
#include "fh_select.cuh"
#include "fh_stream.cuh"

namespace fh {

// Phase stamps for profiling builds (compile with -DFH_PHASE_TIMING; off in the library): thread 0 of
// every block records %globaltimer at the phase boundaries of the batch-1 head.
#ifdef FH_PHASE_TIMING
__device__ unsigned long long g_h1_stamps[512 * 16];
#define H1_STAMP(i)                                                                \
  do {                                                                             \
    if (threadIdx.x == 0) g_h1_stamps[blockIdx.x * 16 + (i)] = global_timer_ns();  \
  } while (0)
#else
#define H1_STAMP(i) \
  do {              \
  } while (0)
#endif

constexpr int kHistBins = kHead1Bins;
// Stage-1 rows each warp requests before the wait for the preceding kernel (the rest follow h).
#ifndef FH_H1_PRE_ROWS
#define FH_H1_PRE_ROWS 1
#endif
constexpr int kHead1PreRows = FH_H1_PRE_ROWS;
#ifndef FH_H1_S1_WARP_BYTES
#define FH_H1_S1_WARP_BYTES 12288
#endif
#ifndef FH_H1_S2_WARP_BYTES
#define FH_H1_S2_WARP_BYTES 8192
#endif
constexpr uint32_t kHead1Stage1WarpBytes = FH_H1_S1_WARP_BYTES;
constexpr uint32_t kHead1Stage2WarpBytes = FH_H1_S2_WARP_BYTES;
constexpr int kCap = kHead1BucketCap;
static_assert(kCap % 32 == 0 && kCap <= kSelCandMax && kCap <= 256, "bucket words are ranked by warps");

// ------------------------------------------------------------------ key binning
// x = key·scale with scale a power of two (exact for every |x| >= 2^-126), then, on each side of zero,
// 64 bins per binade of |x| over [2^-8, 2^(-8 + 510/64)): the fine bins 1..510 (negative keys) and
// 513..1022 (positive keys).  |x| < 2^-8 falls into the central bins 511 (negative) and 512 (zero and
// positive; -0 and +0 alike), larger |x| into the end bins 0 and 1023.  Every step is an integer
// operation on the bit pattern of x, so the bin is monotone in the key; inside a fine bin the low 17
// bits of |x|'s pattern order the keys exactly (distinct keys have distinct x).
constexpr uint32_t kFineLo = 0x3B800000u;  // bit pattern of 2^-8
constexpr uint32_t kFineBins = 510u;

struct Binning {
  float scale;
  __device__ __forceinline__ uint32_t operator()(float key) const {
    const uint32_t u = __float_as_uint(key * scale);
    const uint32_t a = u & 0x7FFFFFFFu;
    const bool neg = (u >> 31) != 0u;
    if (a < kFineLo) return (neg && a != 0u) ? 511u : 512u;
    const uint32_t t = (a - kFineLo) >> 17;
    if (neg) return t >= kFineBins ? 0u : 510u - t;
    return t >= kFineBins ? 1023u : 513u + t;
  }
  // The order of a key inside its fine bin (17 bits; larger = larger key).
  __device__ __forceinline__ uint32_t order_bits(float key) const {
    const uint32_t u = __float_as_uint(key * scale);
    const uint32_t off = ((u & 0x7FFFFFFFu) - kFineLo) & 0x1FFFFu;
    return (u >> 31) ? 0x1FFFFu - off : off;
  }
};

__device__ __forceinline__ bool fine_bin(uint32_t d) {
  return (d >= 1u && d <= 510u) || (d >= 513u && d <= 1022u);
}

// Every block computes the same ‖h‖ (same data, same reduction order) and from it the scale: the power
// of two 2^-e with 2^e > R, R bounding |key| (unit centroids: |s| <= ‖h‖, with a 1/16 margin for INT4
// centroids; sampling adds the Gumbel term, |G| <= 16.7 for the 23-bit uniforms).
__device__ __forceinline__ Binning make_binning(const float hnorm, int sample, float tau) {
  float r = hnorm * 1.0625f + 1e-30f;
  if (sample) r = r / tau + 17.0f;
  int e = 0;
  frexpf(r, &e);  // r = m·2^e, m in [0.5, 1)
  Binning bn;
  bn.scale = ldexpf(1.0f, -e);
  if (!(isfinite(bn.scale) && bn.scale > 0.0f)) bn.scale = 1.0f;
  return bn;
}

// Smallest order-preserving key image u with bin(value of u) >= d (d in [1, kHistBins)), found by a
// warp-wide 32-ary search over the images of finite floats; bin is monotone in u there, so a key is in
// a bin >= d exactly when its image is >= the returned edge.  Called by a whole warp.
__device__ __forceinline__ uint32_t bin_edge(const Binning& bin, uint32_t d) {
  const int lane = threadIdx.x & 31;
  uint32_t lo = 0x007FFFFFu, hi = 0xFF800000u;  // images of -inf and +inf
  if (bin(key_float(hi)) < d) return 0xFFFFFFFFu;  // no finite key reaches bin d
  if (bin(key_float(lo)) >= d) return lo;
  // invariant: bin(lo) < d <= bin(hi); each round shrinks hi - lo by a factor of ~32
  for (int round = 0; round < 12 && hi - lo > 1u; ++round) {
    const uint32_t step = (hi - lo) / 32u + 1u;
    const uint32_t u = min(hi, lo + step * (uint32_t)lane + step);
    const bool ge = bin(key_float(u)) >= d;
    const uint32_t mask = __ballot_sync(0xFFFFFFFFu, ge);  // lanes at and after the edge
    const int first = __ffs(mask) - 1;
    const uint32_t nhi = first >= 0 ? min(hi, lo + step * (uint32_t)first + step) : hi;
    const uint32_t nlo = first > 0 ? lo + step * (uint32_t)(first - 1) + step : lo;
    lo = nlo;
    hi = nhi;
  }
  return hi;
}

// HPT consecutive histogram bins (16- or 8-byte aligned) with one relaxed gpu-scope vector load.
template <int HPT>
__device__ __forceinline__ void load_bins_relaxed(const uint32_t* p, uint32_t (&hb)[HPT]) {
  if constexpr (HPT == 4) {
    asm volatile("ld.relaxed.gpu.global.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(hb[0]), "=r"(hb[1]), "=r"(hb[2]), "=r"(hb[3]) : "l"(p) : "memory");
  } else {
    asm volatile("ld.relaxed.gpu.global.v2.u32 {%0, %1}, [%2];" : "=r"(hb[0]), "=r"(hb[1]) : "l"(p) : "memory");
  }
}

__device__ __forceinline__ void st_relaxed_u64(unsigned long long* p, unsigned long long v) {
  asm volatile("st.relaxed.gpu.global.u64 [%0], %1;" ::"l"(p), "l"(v) : "memory");
}

// Poll a 64-bit word until its upper half equals `tag`, then return it (payload in the lower half).
// Bounded: after 0.5 s it records a timeout, clears `ok` and returns 0.
__device__ __forceinline__ unsigned long long poll_tagged(const unsigned long long* p, uint32_t tag,
                                                          uint32_t* status, bool& ok) {
  const uint64_t t0 = global_timer_ns();
  for (uint32_t it = 1;; ++it) {
    unsigned long long v;
    asm volatile("ld.relaxed.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
    if ((uint32_t)(v >> 32) == tag) return v;
    if ((it & 63u) == 0 && global_timer_ns() - t0 > 500000000ull) {
      set_status(status, kStatusTimeout);
      ok = false;
      return 0ull;
    }
  }
}

// Payload of a word: cluster id (bits 17..30) and the order inside the bin (bits 0..16).
__device__ __forceinline__ int word_id(unsigned long long w) { return (int)((uint32_t)(w >> 17) & 0x3FFFu); }

// Rank the m (<= 32*KP) boundary candidates under (key desc, id asc) and write the ids of the `need`
// best into out in rank order.  Every lane keeps KP candidates in registers (absent ones as 0, below
// every key); each warp ranks four candidates per pass, branch-free.
template <int KP>
__device__ __forceinline__ void rank_boundary(const uint32_t* cand_key, const int* cand_id, uint32_t m,
                                              uint32_t need, int* out, int lane, int warp, int nwarps) {
  uint32_t ck[KP];
  int cid[KP];
#pragma unroll
  for (int u = 0; u < KP; ++u) {
    const uint32_t q = (uint32_t)(lane + 32 * u);
    ck[u] = q < m ? cand_key[q] : 0u;
    cid[u] = q < m ? cand_id[q] : 0x7FFFFFFF;
  }
  for (uint32_t i0 = (uint32_t)warp * 4u; i0 < m; i0 += (uint32_t)nwarps * 4u) {
    uint32_t ki[4], rk[4];
    int ii[4];
#pragma unroll
    for (int t = 0; t < 4; ++t) {
      const uint32_t i = i0 + t;
      ki[t] = i < m ? cand_key[i] : 0xFFFFFFFFu;
      ii[t] = i < m ? cand_id[i] : 0;
      rk[t] = 0u;
    }
#pragma unroll
    for (int u = 0; u < KP; ++u)
#pragma unroll
      for (int t = 0; t < 4; ++t)
        rk[t] += (uint32_t)(ck[u] > ki[t]) + ((uint32_t)(ck[u] == ki[t]) & (uint32_t)(cid[u] < ii[t]));
#pragma unroll
    for (int t = 0; t < 4; ++t) {
      const uint32_t r = __reduce_add_sync(0xFFFFFFFFu, rk[t]);
      if (lane == 0 && i0 + t < m && r < need) out[r] = ii[t];
    }
  }
}

// ------------------------------------------------------------------ shared-memory layout

struct Head1Layout {
  uint32_t bars1, bars2, hs, sc, sel, hist, histg, ownk, ownp, rkid, asc, tokr, zr, ring, total;
};

__host__ __device__ inline uint32_t h1_align(uint32_t x, uint32_t a) { return (x + a - 1) / a * a; }

// Words of C2T copied per touched cluster: its b ids, widened to whole 16-byte chunks.
__host__ __device__ inline int h1_tok_words(int b) { return (b + 6 + 3) / 4 * 4; }

template <int NT>
__host__ __device__ inline Head1Layout head1_layout(uint32_t row2, int rows1_max, int nch4, int rmax,
                                                    int b, uint32_t ring_bytes) {
  // rows1_max: Stage-1 rows of the largest block (its own keys are kept); nch4: INT4 groups per row;
  // rmax: Stage-2 ranks (clusters) a block touches at most
  const int sc_rows = nch4 ? rows1_max : 0;
  Head1Layout L;
  L.bars1 = 0;
  L.bars2 = 1024;
  L.hs = 2048;
  L.sc = h1_align(L.hs + row2, 128);
  L.sel = h1_align(L.sc + (uint32_t)sc_rows * nch4 * 2u + 4u, 128);
  L.hist = h1_align(L.sel + (uint32_t)sizeof(SelectSmem<NT>), 16);
  L.histg = h1_align(L.hist + kHistBins * 4u, 16);
  L.ownk = h1_align(L.histg + kHistBins * 4u, 16);
  L.ownp = h1_align(L.ownk + (uint32_t)rows1_max * 4u, 16);
  L.rkid = h1_align(L.ownp + (uint32_t)rows1_max * 4u, 16);
  L.asc = h1_align(L.rkid + (uint32_t)rmax * 4u, 16);
  L.tokr = h1_align(L.asc + (uint32_t)rmax * 4u, 16);
  L.zr = h1_align(L.tokr + (uint32_t)rmax * (uint32_t)h1_tok_words(b) * 4u, 16);  // rmax * b >= its rows
  L.ring = h1_align(L.zr + (uint32_t)rmax * (uint32_t)b * 4u, 128);
  L.total = L.ring + ring_bytes;
  return L;
}

// ------------------------------------------------------------------ the kernel

template <int ELEM, int INT4_MCH, int NT, int KPT>
__global__ void __launch_bounds__(NT, 1) k_head1(const Head1Params prm) {
  extern __shared__ __align__(128) uint8_t smem[];
  constexpr int W = NT / 32;
  constexpr int HPT = kHistBins / NT;  // histogram bins per thread
  static_assert(HPT == 2 || HPT == 4, "bins per thread");
  __shared__ unsigned long long warp_best[W];
  __shared__ float red_s[W];
  __shared__ bool abort_s;
  __shared__ uint32_t dstar_s, above_s, total_s, m_s, edge_lo_s, edge_hi_s;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int G = gridDim.x, bid = blockIdx.x;
  const int64_t c = prm.c, d = prm.d;
  const int b = (int)prm.b;
  const uint32_t row2 = (uint32_t)(d * (ELEM == kBF16 ? 2 : 4));  // E row bytes
  const uint32_t row1 = INT4_MCH ? (uint32_t)(d / 2) : row2;       // Stage-1 row bytes
  const int nch2 = (int)(row2 / 16);
  const int nch4 = INT4_MCH ? (int)(d / 32) : 0;
  const int P = prm.p * b;
  // 32-bit splits (the launcher keeps v * gridDim.x below 2^31): 64-bit division is a long software
  // sequence on the GPU, and these sit on the path between the stages.
  const uint32_t uG = (uint32_t)G, uc = (uint32_t)c;
  const int rows1_max = (int)((uc + uG - 1u) / uG);
  const int rows2_max = (int)(((uint32_t)P + uG - 1u) / uG);
  const int rmax = (int)(rows2_max / b) + 2;
  const int tsw = h1_tok_words(b);
  const int K1 = prm.k1, K2 = prm.k2;
  const Head1Layout L = head1_layout<NT>(row2, rows1_max, nch4, rmax, b, prm.ring_bytes);
  uint64_t* bars1 = reinterpret_cast<uint64_t*>(smem + L.bars1);
  uint64_t* bars2 = reinterpret_cast<uint64_t*>(smem + L.bars2);
  uint64_t* tok_bar = &bars2[126];  // the C2T rows of the touched clusters
  uint64_t* key_bar = &bars2[127];  // the key copy of the full selection
  uint8_t* hs = smem + L.hs;
  uint16_t* sc_s = reinterpret_cast<uint16_t*>(smem + L.sc);
  SelectSmem<NT>& sm = *reinterpret_cast<SelectSmem<NT>*>(smem + L.sel);
  uint32_t* hist_s = reinterpret_cast<uint32_t*>(smem + L.hist);
  uint32_t* histg_s = reinterpret_cast<uint32_t*>(smem + L.histg);  // keys in bins above each bin
  float* own_keys = reinterpret_cast<float*>(smem + L.ownk);
  uint32_t* own_pos = reinterpret_cast<uint32_t*>(smem + L.ownp);
  int* rk_id = reinterpret_cast<int*>(smem + L.rkid);   // cluster of each touched rank
  int* asc_of = reinterpret_cast<int*>(smem + L.asc);   // its ascending position (debug outputs)
  int32_t* tokr = reinterpret_cast<int32_t*>(smem + L.tokr);
  uint8_t* ring = smem + L.ring;
  H1_STAMP(0);

  // ------------------------------------------------------------------ prologue
  const int64_t lo1 = uc * (uint32_t)bid / uG, hi1 = uc * (uint32_t)(bid + 1) / uG;
  const int nk = (int)(hi1 - lo1);
  uint32_t scv[4];  // INT4: this block's group scales, two per 32-bit word (loaded before any copy)
  const int nsc = INT4_MCH ? nk * nch4 : 0;
  const int sc_words = (nsc + 1) / 2;
  if constexpr (INT4_MCH > 0) {
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int w = tid + u * NT;
      if (w < sc_words) {
        const int64_t e = lo1 * nch4 + 2 * (int64_t)w;  // scales are read as pairs
        const uint32_t a = prm.scales[e];
        const uint32_t bb = (2 * w + 1 < nsc) ? prm.scales[e + 1] : 0u;
        scv[u] = a | (bb << 16);
      }
    }
  }
  if (tid < W * K1) mbar_init(&bars1[tid], 1);
  if (tid < W * K2) mbar_init(&bars2[tid], 1);
  if (tid == 0) {
    mbar_init(tok_bar, 1);
    mbar_init(key_bar, 1);
  }
  fence_mbar_init();
  __syncthreads();

  // Stage-1 rows of this warp: first1, first1 + W, ...; the first K1 are requested now (index data:
  // no dependence on the preceding kernel).
  const int64_t first1 = lo1 + warp;
  const int n1 = (first1 < hi1) ? (int)((hi1 - first1 + W - 1) / W) : 0;
  uint8_t* ring1 = ring + (size_t)warp * K1 * row1;
  uint64_t* b1 = bars1 + warp * K1;
  const uint8_t* src1 = INT4_MCH ? static_cast<const uint8_t*>(static_cast<const void*>(prm.q4))
                                 : static_cast<const uint8_t*>(prm.C);
  const int pre = min(K1, kHead1PreRows);
  if (lane < pre && lane < n1)
    issue_row(ring1 + (size_t)lane * row1, src1 + (size_t)(first1 + (int64_t)W * lane) * row1, row1,
              &b1[lane]);

  // h and the workspace may be written by the preceding kernel: wait for it (a no-op unless the
  // launch allowed programmatic overlap).  A small load queues behind the bulk copies the SM has in
  // flight, so h is requested before the rest of the first copies.
  pdl_wait_prior();
  uint4 hv[4];
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    const int ch = tid + u * NT;
    if (ch < nch2) hv[u] = __ldg(reinterpret_cast<const uint4*>(prm.H) + ch);
  }
  uint32_t tag = __ldcg(prm.gen) + 1u;  // this call's tag on its words (never 0)
  if (tag == 0u) tag = 1u;
  if (lane >= pre && lane < K1 && lane < n1)
    issue_row(ring1 + (size_t)lane * row1, src1 + (size_t)(first1 + (int64_t)W * lane) * row1, row1,
              &b1[lane]);
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    const int ch = tid + u * NT;
    if (ch < nch2) reinterpret_cast<uint4*>(hs)[ch] = hv[u];
  }
  if constexpr (INT4_MCH > 0) {
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int w = tid + u * NT;
      if (w < sc_words) reinterpret_cast<uint32_t*>(sc_s)[w] = scv[u];
    }
  }
  for (int i = tid; i < kHistBins; i += NT) hist_s[i] = 0u;
  __syncthreads();
  H1_STAMP(1);
  // ‖h‖ (fixed reduction order, identical in every block) and the key binning
  float hsq = 0.0f;
  for (int ch = tid; ch < nch2; ch += NT) {
    const uint4 v = reinterpret_cast<const uint4*>(hs)[ch];
    hsq = (ELEM == kBF16) ? dot8_bf16(v, v, hsq) : dot4_f32(v, v, hsq);
  }
  hsq = warp_sum(hsq);
  if (lane == 0) red_s[warp] = hsq;
  // INT4 rows are read as 32-bit words of 8 columns (four words share one group scale): lane l takes
  // the words l, l + 32, ..., so a row of any width keeps every lane busy but the last pass's, and
  // keeps the 8 columns of h of each of its words in registers (one conflict-free 16-byte load each).
  constexpr int kWpl = INT4_MCH ? 4 * INT4_MCH : 1;  // words per lane, at most
  const int nw4 = nch4 * 4;                            // words per INT4 row
  float hreg[kWpl][INT4_MCH ? 8 : 1];
  if constexpr (INT4_MCH > 0) {
    const uint32_t hs_a = smem_addr(hs);
#pragma unroll
    for (int i = 0; i < kWpl; ++i) {
      const int wd = lane + 32 * i;
      const uint4 v = wd < nw4 ? lds_v4(hs_a + 16u * (uint32_t)wd) : make_uint4(0u, 0u, 0u, 0u);
      hreg[i][0] = bf16_lo(v.x);
      hreg[i][1] = bf16_hi(v.x);
      hreg[i][2] = bf16_lo(v.y);
      hreg[i][3] = bf16_hi(v.y);
      hreg[i][4] = bf16_lo(v.z);
      hreg[i][5] = bf16_hi(v.z);
      hreg[i][6] = bf16_lo(v.w);
      hreg[i][7] = bf16_hi(v.w);
    }
  }
  __syncthreads();
  float hn2 = 0.0f;
#pragma unroll
  for (int w = 0; w < W; ++w) hn2 += red_s[w];
  const Binning bin = make_binning(sqrtf(hn2), prm.sample, prm.tau);
  const bool all = prm.p >= c;

  // ------------------------------------------------------------------ Stage 1
  // The score of the warp's row n stays in lane n (n1 <= 32: a block has at most NT rows) until the
  // stream is over; the keys are then formed and counted by all lanes at once.
  const uint32_t hs_addr = smem_addr(hs);
  float my_s = 0.0f;
  int n_done = 0;
  for (int n = 0, slot = 0, phase = 0; n < n1; ++n) {
    if (!mbar_wait(&b1[slot], (uint32_t)phase, prm.status)) {
      for (int m = n + 1; m < n1 && m < n + K1; ++m)
        mbar_wait(&b1[m % K1], (uint32_t)((m / K1) & 1), nullptr, 50000000ull);
      break;
    }
    const int k = (int)first1 + W * n;
    const uint32_t row_s = smem_addr(ring1 + (size_t)slot * row1);
    float s;
    if constexpr (INT4_MCH > 0) {
      float part = 0.0f;
      const uint16_t* scr = sc_s + (k - (int)lo1) * nch4;
      const uint32_t* roww = reinterpret_cast<const uint32_t*>(ring1 + (size_t)slot * row1);
#pragma unroll
      for (int i = 0; i < kWpl; ++i) {
        const int wd = lane + 32 * i;
        if (wd < nw4) {
          const uint32_t w = roww[wd];
          const float scale = __uint_as_float((uint32_t)scr[wd >> 2] << 16);
          part = fmaf(scale, int4_word_dot(w, hreg[i]), part);
        }
      }
      s = warp_sum(part);
    } else {
      s = warp_sum(row_dot_partial<ELEM>(row_s, hs_addr, nch2, lane));
    }
    __syncwarp();
    if (lane == 0 && n + K1 < n1) {
      fence_proxy_async_smem();
      issue_row(ring1 + (size_t)slot * row1, src1 + (size_t)(first1 + (int64_t)W * (n + K1)) * row1,
                row1, &b1[slot]);
    }
    my_s = lane == n ? s : my_s;
    n_done = n + 1;
    if (n == 0) H1_STAMP(13);
    if (++slot == K1) {
      slot = 0;
      phase ^= 1;
    }
  }
  H1_STAMP(14);
  if (lane < n_done) {
    const int k = (int)first1 + W * lane;
    float key = my_s;
    if (prm.sample)
      key = my_s / prm.tau + gumbel_from_u32(philox_word(prm.seed, prm.step, 0u, 0u, (uint32_t)k));
    prm.keys[k] = key;
    own_keys[k - (int)lo1] = key;
    if (!all) own_pos[k - (int)lo1] = atomicAdd(&hist_s[bin(key)], 1u);
  }
  __syncthreads();
  H1_STAMP(2);

  // ------------------------------------------------------------------ exchange and grid barrier
  uint32_t hb[HPT];
  uint32_t htot = 0, before = 0;
  if (!all) {
    // The block's first position in each non-empty bin: one returning add per bin, all in flight.
    {
      uint32_t cnt[HPT], base[HPT];
#pragma unroll
      for (int u = 0; u < HPT; ++u) cnt[u] = hist_s[tid + u * NT];
#pragma unroll
      for (int u = 0; u < HPT; ++u) base[u] = cnt[u] ? atomicAdd(prm.hist + tid + u * NT, cnt[u]) : 0u;
#pragma unroll
      for (int u = 0; u < HPT; ++u) hist_s[tid + u * NT] = base[u];
    }
    __syncthreads();
    // One word per key at (bin, position): (tag, cluster id, order inside the bin).
    if (tid < nk) {
      const float key = own_keys[tid];
      const uint32_t bn = bin(key);
      const uint32_t pos = hist_s[bn] + own_pos[tid];
      if (pos < (uint32_t)kCap)
        st_relaxed_u64(prm.bucket + (size_t)bn * kCap + pos,
                       ((unsigned long long)tag << 32) | ((unsigned long long)(lo1 + tid) << 17) |
                           bin.order_bits(key));
    }
    H1_STAMP(3);
    // The summed histogram is complete once its counts add up to c.  Every block polls it until then:
    // the poll is the grid barrier, and its last round already holds the counts the selection needs.
    for (int i = tid; i < 1025; i += NT) sm.selbits[i] = 0u;
    if (tid == 0) sm.cand_count = 0u;
    const uint64_t t0 = global_timer_ns();
    for (uint32_t it = 1;; ++it) {
      load_bins_relaxed<HPT>(prm.hist + tid * HPT, hb);
      htot = 0;
#pragma unroll
      for (int u = 0; u < HPT; ++u) htot += hb[u];
      const unsigned long long ex = block_scan2<NT>(0u, htot, sm, 0);
      before = (uint32_t)(ex & 0xFFFFFFFFull);
      if (tid == NT - 1) total_s = before + htot;
      if (tid == 0) abort_s = (it & 15u) == 0u && global_timer_ns() - t0 > 500000000ull;
      __syncthreads();
      if (total_s >= (uint32_t)c || abort_s) break;  // the same decision in every thread
      __syncthreads();                                 // total_s and the scan scratch are reused
    }
    if (total_s != (uint32_t)c) {  // a wait gave up somewhere: nothing below is valid
      if (tid == 0) set_status(prm.status, kStatusTimeout);
      return;
    }
  }
  // Every block of this grid is resident now: the next kernel of the stream may start its prologue
  // as blocks leave (it waits for this grid to complete before touching h or the workspace).
  pdl_launch_dependents();
  H1_STAMP(4);

  // ------------------------------------------------------------------ boundary bin
  if (tid == 0) {
    dstar_s = 0u;
    above_s = (uint32_t)c;
    m_s = 0u;
  }
  __syncthreads();
  if (!all) {
    uint32_t cum = total_s - before - htot;  // keys in bins above this thread's bins
#pragma unroll
    for (int u = HPT - 1; u >= 0; --u) {
      histg_s[tid * HPT + u] = cum;  // keys in bins above bin tid*HPT+u
      if (cum < (uint32_t)prm.p && cum + hb[u] >= (uint32_t)prm.p) {
        dstar_s = (uint32_t)(tid * HPT + u);
        above_s = cum;
        m_s = hb[u];
      }
      cum += hb[u];
    }
    __syncthreads();
  }
  const uint32_t dstar = dstar_s;
  const uint32_t above_n = above_s;
  const uint32_t need = (uint32_t)prm.p - min(above_n, (uint32_t)prm.p);
  const uint32_t m_total = m_s;
  bool fast = true;
  if (!all) {
    // every bin from d* up must fit the word table, and a partly taken boundary bin must be a fine
    // bin (its words then order the keys exactly)
    bool over = false;
#pragma unroll
    for (int u = 0; u < HPT; ++u) over |= (uint32_t)(tid * HPT + u) >= dstar && hb[u] > (uint32_t)kCap;
    over = __syncthreads_or(over);
    fast = !over && (need == m_total || fine_bin(dstar));
  }
  const uint8_t* E = static_cast<const uint8_t*>(prm.E);
  const uint8_t* Ep = static_cast<const uint8_t*>(prm.E_perm);
  const bool perm = Ep != nullptr;

  // This block's Stage-2 rows [r0, r1) of the rank-ordered list (row g: rank g / b, row g % b of
  // that cluster) and the ranks they touch.
  const int r0 = (int)((uint32_t)P * (uint32_t)bid / uG), r1 = (int)((uint32_t)P * (uint32_t)(bid + 1) / uG);
  const int rk0 = r0 / b, rk1 = (r1 > r0) ? (r1 - 1) / b + 1 : rk0;
  const int nrk = rk1 - rk0;
  const bool want_dbg = prm.dbg_sel || prm.dbg_tok || prm.dbg_logit;
  int* tab = reinterpret_cast<int*>(ring);  // debug: the whole list (ring free until Stage 2)

  if (all) {
    // every cluster is taken: rank r is cluster r
    if (tid < nrk) {
      rk_id[tid] = rk0 + tid;
      asc_of[tid] = rk0 + tid;
    }
    if (prm.dbg_sel && bid == 0)
      for (int q = tid; q < prm.p; q += NT) prm.dbg_sel[q] = q;
  } else if (fast) {
    // ---------------------------------------------------------------- selection from the words
    // Rank r < above_n lives in the bin t0 = the lowest t with (keys above t) <= r, at position
    // r - (keys above t0); ranks from above_n on are the boundary bin's taken keys.
    auto certain_word = [&](uint32_t r, bool& ok) {
      int lo = 0, hi = kHistBins - 1;
      while (lo < hi) {
        const int mid = (lo + hi) >> 1;
        if (histg_s[mid] <= r) hi = mid;
        else lo = mid + 1;
      }
      return word_id(poll_tagged(prm.bucket + (size_t)lo * kCap + (r - histg_s[lo]), tag, prm.status, ok));
    };
    const bool bnd_ranks = want_dbg || rk1 > (int)above_n;  // does this block need the boundary bin?
    bool ok = true;
    if (want_dbg) {
      for (uint32_t r = tid; r < above_n; r += NT) tab[r] = certain_word(r, ok);
    } else if (tid < nrk && (uint32_t)(rk0 + tid) < above_n) {
      rk_id[tid] = certain_word((uint32_t)(rk0 + tid), ok);
    }
    int* bsel = reinterpret_cast<int*>(sm.selbits);  // boundary ids in rank order (need <= kCap)
    if (bnd_ranks && need > 0u) {
      // the boundary words are read by the last kCap threads, so that their loads go out together
      // with the certain words of the first threads
      const unsigned long long* bw = prm.bucket + (size_t)dstar * kCap;
      const int bt = tid - (NT - kCap);
      if (need == m_total) {  // the whole bin is taken: any order will do, take the positions
        if (bt >= 0 && bt < (int)m_total) bsel[bt] = word_id(poll_tagged(bw + bt, tag, prm.status, ok));
      } else {
        uint32_t* ckey = reinterpret_cast<uint32_t*>(sm.cand_key);
        if (bt >= 0 && bt < (int)m_total) {
          const unsigned long long w = poll_tagged(bw + bt, tag, prm.status, ok);
          ckey[bt] = (uint32_t)(w & 0x1FFFFull) + 1u;  // 0 stays below every key
          sm.cand_id[bt] = word_id(w);
        }
        if (!__syncthreads_and(ok)) return;
        rank_boundary<kCap / 32>(ckey, sm.cand_id, m_total, need, bsel, lane, warp, W);
      }
    }
    if (!__syncthreads_and(ok)) return;
    if (want_dbg) {
      for (uint32_t r = above_n + tid; r < (uint32_t)prm.p; r += NT) tab[r] = bsel[r - above_n];
      __syncthreads();
      if (tid < nrk) rk_id[tid] = tab[rk0 + tid];
    } else if (tid < nrk && (uint32_t)(rk0 + tid) >= above_n) {
      rk_id[tid] = bsel[rk0 + tid - (int)above_n];
    }
    __syncthreads();
    if (want_dbg) {
      // canonical (ascending) positions of this block's clusters, and the probe set
      for (int t = warp; t < nrk; t += W) {
        const int x = rk_id[t];
        uint32_t cnt = 0;
        for (int q = lane; q < prm.p; q += 32) cnt += (uint32_t)(tab[q] < x);
        cnt = __reduce_add_sync(0xFFFFFFFFu, cnt);
        if (lane == 0) asc_of[t] = (int)cnt;
      }
      if (prm.dbg_sel && bid == 0) {
        for (int q = tid; q < prm.p; q += NT) {
          const int x = tab[q];
          uint32_t cnt = 0;
          for (int y = 0; y < prm.p; ++y) cnt += (uint32_t)(tab[y] < x);
          prm.dbg_sel[cnt] = x;
        }
      }
    }
  } else {
    // ---------------------------------------------------------------- full selection (crowded bin)
    // A bin from d* up holds more keys than the word table, or the boundary bin cannot order its keys
    // from the words: every block loads all keys and selects with the block-wide selector (exact radix
    // passes on the boundary bin).  The keys are visible once every block has arrived here.
    if (tid == 0) {
      asm volatile("fence.acq_rel.gpu;" ::: "memory");
      uint32_t old;
      asm volatile("atom.acq_rel.gpu.global.add.u32 %0, [%1], 1;" : "=r"(old) : "l"(prm.keys_ready) : "memory");
      const uint32_t target = (old / uG + 1u) * uG;
      const uint64_t t0 = global_timer_ns();
      abort_s = false;
      for (uint32_t it = 1;; ++it) {
        uint32_t v;
        asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(prm.keys_ready) : "memory");
        if ((int32_t)(v - target) >= 0) break;
        if ((it & 63u) == 0 && global_timer_ns() - t0 > 500000000ull) {
          set_status(prm.status, kStatusTimeout);
          abort_s = true;
          break;
        }
      }
    }
    __syncthreads();
    if (abort_s) return;
    const uint32_t keys_bytes = (uint32_t)((c * 4 + 15) / 16 * 16);
    float* keys_s = reinterpret_cast<float*>(ring);
    if (tid == 0) {
      asm volatile("fence.proxy.async;" ::: "memory");
      mbar_arrive_expect_tx(key_bar, keys_bytes);
      bulk_g2s(keys_s, prm.keys, keys_bytes, key_bar);
    }
    if (!mbar_wait(key_bar, 0u, prm.status)) return;
    uint32_t key[KPT];
    {
      const int kb = tid * KPT;
#pragma unroll
      for (int j = 0; j < KPT; ++j) key[j] = (kb + j < c) ? float_key(keys_s[kb + j]) : 0u;
    }
    SelState st;
    st.above = above_n;
    st.need = need;
    if (warp == 0) {
      const uint32_t e = (dstar == 0u) ? 1u : bin_edge(bin, dstar);
      if (lane == 0) edge_lo_s = e;
    } else if (warp == 1) {
      const uint32_t e = (dstar + 1u >= (uint32_t)kHistBins) ? 0xFFFFFFFFu : bin_edge(bin, dstar + 1u);
      if (lane == 0) edge_hi_s = e;
    }
    __syncthreads();
    const uint32_t elo = edge_lo_s, ehi = edge_hi_s;
    st.certain = 0u;
    st.boundary = 0u;
#pragma unroll
    for (int j = 0; j < KPT; ++j) {
      const uint32_t kj = key[j];
      const uint32_t real = (uint32_t)(kj != 0u);
      const uint32_t abv = (uint32_t)(kj >= ehi);
      st.certain |= (real & abv) << j;
      st.boundary |= (real & (uint32_t)(kj >= elo) & (abv ^ 1u)) << j;
    }
    const int base = tid * KPT;
    const uint32_t bsel = topp_resolve<NT, KPT>(key, st, sm);
    const uint32_t sel = st.certain | bsel;
    {
      const unsigned long long exc = block_scan2<NT>(__popc(st.certain), __popc(bsel), sm, 1);
      const unsigned long long exa = block_scan2<NT>(__popc(sel), 0u, sm, 2);
      int rc = (int)(exc >> 32), rb = (int)above_n + (int)(exc & 0xFFFFFFFFull);
      int a = (int)(exa >> 32);
      for (uint32_t bits = sel; bits; bits &= bits - 1, ++a) {
        const int j = __ffs(bits) - 1;
        int& r = (st.certain >> j & 1u) ? rc : rb;
        if (r >= rk0 && r < rk1) {
          rk_id[r - rk0] = base + j;
          asc_of[r - rk0] = a;
        }
        ++r;
        if (prm.dbg_sel && bid == 0) prm.dbg_sel[a] = base + j;
      }
    }
    __syncthreads();
  }
  H1_STAMP(5);

  // ------------------------------------------------------------------ Stage 2
  // This warp's first K2 candidate rows go out first (rows of the cluster-major copy are addressed by
  // cluster id alone), then the C2T rows of the touched clusters (one small copy each; b ids widened
  // to 16-byte chunks).  The logits are kept per row and turned into decision keys once the stream is
  // over, so the token ids never stand in front of a row.
  const int nr = r1 - r0;
  const int n2 = (warp < nr) ? (nr - warp + W - 1) / W : 0;
  uint8_t* ring2 = ring + (size_t)warp * K2 * row2;
  uint64_t* b2 = bars2 + warp * K2;
  float* zr = reinterpret_cast<float*>(smem + L.zr);  // logit of block row g - r0
  // The C2T copies go out from the last warp, one lane a cluster (warp 0 carries the block's other
  // serial work).
  auto issue_tok = [&]() {
    if (warp == W - 1 && nrk > 0) {
      uint32_t bytes = 0;
      for (int i = lane; i < nrk; i += 32) {
        const int e0 = rk_id[i] * b;
        bytes += (uint32_t)(((e0 + b + 3) & ~3) - (e0 & ~3)) * 4u;
      }
      bytes = __reduce_add_sync(0xFFFFFFFFu, bytes);
      if (lane == 0) mbar_arrive_expect_tx(tok_bar, bytes);
      __syncwarp();
      for (int i = lane; i < nrk; i += 32) {
        const int e0 = rk_id[i] * b;
        const int s0 = e0 & ~3;
        fence_proxy_async_smem();
        bulk_g2s(tokr + i * tsw, prm.C2T + s0, (uint32_t)(((e0 + b + 3) & ~3) - s0) * 4u, tok_bar);
      }
    }
  };
  auto token_of = [&](int q, int j) {  // rank q (global), row j of its cluster
    const int e0 = rk_id[q - rk0] * b;
    return tokr[(q - rk0) * tsw + (e0 & 3) + j];
  };
  if (!perm) {  // the rows are addressed through their token ids: wait for the C2T rows
    issue_tok();
    const bool ok = nrk == 0 || mbar_wait(tok_bar, 0u, prm.status);
    if (!__syncthreads_and(ok)) return;
  }
  auto issue2 = [&](int n) {
    const int slot = n % K2;
    const int g = r0 + warp + W * n;
    const int q = g / b, j = g - q * b;
    mbar_arrive_expect_tx(&b2[slot], row2);
    const uint8_t* src = perm ? Ep + ((size_t)rk_id[q - rk0] * b + j) * row2
                              : E + (size_t)token_of(q, j) * row2;
    bulk_g2s(ring2 + (size_t)slot * row2, src, row2, &b2[slot]);
  };
  if (lane < K2 && lane < n2) {
    fence_proxy_async_smem();  // the ring was last read by Stage 1 and the selection
    issue2(lane);
  }
  if (perm) {
    __syncwarp();
    issue_tok();
  }
  H1_STAMP(10);
  bool ok2 = true;
  for (int n = 0, slot = 0, phase = 0; n < n2; ++n) {
    if (!mbar_wait(&b2[slot], (uint32_t)phase, prm.status)) {
      for (int m = n + 1; m < n2 && m < n + K2; ++m)
        mbar_wait(&b2[m % K2], (uint32_t)((m / K2) & 1), nullptr, 50000000ull);
      ok2 = false;
      break;
    }
    if (n == 0) H1_STAMP(6);
    const int g = r0 + warp + W * n;
    const float z = warp_sum(row_dot_partial<ELEM>(smem_addr(ring2 + (size_t)slot * row2), hs_addr,
                                                   nch2, lane));
    __syncwarp();
    if (lane == 0) {
      if (n + K2 < n2) {
        fence_proxy_async_smem();
        issue2(n + K2);
      }
      zr[g - r0] = z;
    }
    if (++slot == K2) {
      slot = 0;
      phase ^= 1;
    }
  }
  // the decision keys of this warp's rows (lane l takes rows l, l + 32, ...) once the ids are in
  bool tok_ok = ok2;
  if (perm && n2 > 0 && ok2) {
    if (lane == 0) tok_ok = mbar_wait(tok_bar, 0u, prm.status);
    tok_ok = __shfl_sync(0xFFFFFFFFu, tok_ok, 0);
  }
  if (!tok_ok) {  // (status recorded) the C2T copies land before the block leaves
    if (perm && tid == 0 && nrk > 0) mbar_wait(tok_bar, 0u, nullptr, 50000000ull);
    return;
  }
  __syncwarp();
  unsigned long long best = 0ull;
  for (int n = lane; n < n2; n += 32) {
    const int g = r0 + warp + W * n;
    const int q = g / b, j = g - q * b;
    const uint32_t tok = (uint32_t)token_of(q, j);
    const float z = zr[g - r0];
    float val = z;
    if (prm.sample)
      val = z / prm.tau + gumbel_from_u32(philox_word(prm.seed, prm.step, 0u, 1u, tok));
    const unsigned long long pk = pack_best(val, tok);
    best = pk > best ? pk : best;
    if (want_dbg) {
      const int ai = asc_of[q - rk0] * b + j;
      if (prm.dbg_logit) prm.dbg_logit[ai] = z;
      if (prm.dbg_tok) prm.dbg_tok[ai] = (int32_t)tok;
    }
  }
  best = warp_max_u64(best);

  // ------------------------------------------------------------------ arg-max over the grid
  // Every block folds its best (value, ~token) into the call's maximum with one relaxed 64-bit max and
  // counts itself in with an acquire-release add; the block that arrives last reads the maximum,
  // writes the token and returns the maximum, the count and the histogram to zero for the next call.
  // No block waits for another here.
  if (lane == 0) warp_best[warp] = best;
  __syncthreads();
  H1_STAMP(7);
  if (tid == 0) {
    unsigned long long bb = 0ull;
    for (int w = 0; w < W; ++w) bb = warp_best[w] > bb ? warp_best[w] : bb;
    asm volatile("red.relaxed.gpu.global.max.u64 [%0], %1;" ::"l"(prm.best), "l"(bb) : "memory");
    uint32_t old;
    asm volatile("atom.acq_rel.gpu.global.add.u32 %0, [%1], 1;" : "=r"(old) : "l"(prm.arrive) : "memory");
    abort_s = old != uG - 1u;  // (not the last block)
  }
  __syncthreads();
  if (abort_s) return;
  H1_STAMP(8);
  for (int i = tid; i < kHistBins; i += NT) prm.hist[i] = 0u;
  if (tag == 0xFFFFFFFFu) {  // the tags wrap after this call: no older word may alias a new tag
#pragma unroll 1
    for (int i = tid; i < kHistBins * kCap; i += NT) prm.bucket[i] = 0ull;
  }
  if (tid == 0) {
    unsigned long long fin;
    asm volatile("ld.relaxed.gpu.global.u64 %0, [%1];" : "=l"(fin) : "l"(prm.best) : "memory");
    st_relaxed_u64(prm.best, 0ull);
    *prm.arrive = 0u;
    *prm.gen = tag;
    prm.out_tok[0] = (int32_t)best_id(fin);
  }
  H1_STAMP(9);
}

// ------------------------------------------------------------------ launcher

#ifdef FH_PHASE_TIMING
extern "C" int fh_probe_head1_stamps(unsigned long long* host, int n) {
  return (int)cudaMemcpyFromSymbol(host, g_h1_stamps, (size_t)n * 8);
}
#endif

int head1_threads(int64_t c) { return c <= 256 * 32 ? 256 : (c <= 512 * 32 ? 512 : 0); }

cudaError_t launch_head1(Head1Params prm, int elem, int int4, int num_sms, cudaStream_t st) {
  const int NT = head1_threads(prm.c);
  if (NT == 0 || prm.c > (1 << 14)) return cudaErrorInvalidValue;  // cluster ids travel in 14 bits
  const int W = NT / 32;
  const int G = num_sms;
  const uint32_t row2 = (uint32_t)(prm.d * (elem == kBF16 ? 2 : 4));
  const uint32_t row1 = int4 ? (uint32_t)(prm.d / 2) : row2;
  if (row2 / 16 > 4u * (uint32_t)NT) return cudaErrorInvalidValue;  // h: 4 chunks per thread
  const int nch4 = int4 ? (int)(prm.d / 32) : 0;
  const int64_t P = (int64_t)prm.p * prm.b;
  if ((prm.c * prm.b) * (int64_t)G >= (int64_t{1} << 31)) return cudaErrorInvalidValue;  // 32-bit splits
  const int rows1_max = (int)((prm.c + G - 1) / G);
  if (rows1_max > NT) return cudaErrorInvalidValue;  // one thread per own key
  if (int4 && (rows1_max * nch4 + 1) / 2 > 4 * NT) return cudaErrorInvalidValue;
  const int rows2_max = (int)((P + G - 1) / G);
  const int rmax = (int)(rows2_max / prm.b) + 2;
  if (rmax > NT) return cudaErrorInvalidValue;
  const int b = (int)prm.b;
  const uint32_t fixed = (NT == 256 ? head1_layout<256>(row2, rows1_max, nch4, rmax, b, 0)
                                    : head1_layout<512>(row2, rows1_max, nch4, rmax, b, 0)).total;
  const uint32_t budget = 220u * 1024u;
  const int kcap = (1024 / 8 - 2) / W;  // barriers per stage (the last two of bars2 are reserved)
  if (fixed + (uint32_t)W * (row2 > row1 ? row2 : row1) > budget) return cudaErrorInvalidValue;
  const uint32_t ring_bytes = (budget - fixed) / 128u * 128u;
  // Rows in flight per warp: about kHead1Stage1WarpBytes / kHead1Stage2WarpBytes of copies.  Fewer
  // bytes in flight than the ring holds make the first rows of each block land sooner and the blocks
  // finish closer together (measured at the Llama-3.2-1B shape: 12 KiB / 8 KiB per warp gave 20.6 µs
  // a call, 48 KiB / 24 KiB 22.2 µs, 16 KiB / 4 KiB 22.8 µs).
  auto slots = [&](uint32_t row, int64_t rows, uint32_t warp_bytes) {
    int64_t k = ring_bytes / ((uint64_t)W * row);
    const int64_t per_warp = (rows + W - 1) / W;
    const int64_t want = warp_bytes / row;
    if (k > want) k = want;
    if (k > per_warp) k = per_warp;
    if (k > kcap) k = kcap;
    return (int)(k < 1 ? 1 : k);
  };
  // the crowded-bin selection copies all keys into the ring, the debug outputs list the probe set there
  if (ring_bytes < (uint32_t)((prm.c * 4 + 15) / 16 * 16)) return cudaErrorInvalidValue;
  prm.k1 = slots(row1, rows1_max, kHead1Stage1WarpBytes);
  prm.k2 = slots(row2, rows2_max, kHead1Stage2WarpBytes);
  prm.ring_bytes = ring_bytes;
  const size_t smem = fixed + ring_bytes;

  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(G);
  cfg.blockDim = dim3(NT);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  // One block per SM.  The grid barrier needs every block resident: a programmatically overlapped
  // launch lets this grid's blocks start only as the preceding grid's blocks leave, and this grid lets
  // the next one start only after its own barrier, when all of its blocks are resident.
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  const int kpt = (int)((prm.c + NT - 1) / NT);
  cudaError_t e = cudaSuccess;
#define FH_H1(EL, M4, NTT, KP)                                                                     \
  do {                                                                                            \
    e = set_smem_attr(reinterpret_cast<const void*>(k_head1<EL, M4, NTT, KP>), smem);            \
    if (e != cudaSuccess) return e;                                                               \
    e = cudaLaunchKernelEx(&cfg, k_head1<EL, M4, NTT, KP>, prm);                                  \
  } while (0)
#define FH_H1_NT(EL, M4)                                  \
  do {                                                    \
    if (NT == 512) FH_H1(EL, M4, 512, 32);                \
    else if (kpt <= 8) FH_H1(EL, M4, 256, 8);             \
    else FH_H1(EL, M4, 256, 32);                          \
  } while (0)
  if (int4) {
    if (nch4 <= 32) FH_H1_NT(kBF16, 1);
    else if (nch4 <= 64) FH_H1_NT(kBF16, 2);
    else FH_H1_NT(kBF16, 4);
  } else if (elem == kBF16) {
    FH_H1_NT(kBF16, 0);
  } else {
    FH_H1_NT(kF32, 0);
  }
#undef FH_H1_NT
#undef FH_H1
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace fh

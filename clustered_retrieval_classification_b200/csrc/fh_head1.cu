// fh_head1.cu — the batch-1 FlashHead head as one persistent cooperative kernel (one block per SM).
//
// At batch 1 the whole call moves ~66 MB (Llama-shaped head), about 10 µs of HBM time on a B200, so
// every launch boundary and every serial step between the two bandwidth phases shows.  One kernel
// therefore runs the whole path (FlashHead notes, overall architecture and Figure 1):
//
//   1. Stage 1: each block loads h, then bulk-copies its share of centroid rows (C, or the INT4
//      nibbles) into its shared-memory ring at once, computes s = C·h (or the Gumbel key s/τ + G),
//      writes the keys, and counts each key in a 1024-bin block histogram.  The bins cover a range
//      fixed in advance from ‖h‖ (unit centroids give |s| <= ‖h‖; the Gumbel term lies in
//      [-2.9, 16.7]); keys outside are clamped into the end bins, so the binning is monotone for any
//      input and only its resolution depends on the range.  The block adds its counts to the global
//      histogram with returning release adds, which give every key a distinct position in its bin.
//   2. Grid barrier = histogram poll: every block polls the summed histogram until its counts reach c
//      (bounded wait); the last poll holds the counts, the boundary bin follows by a block scan.
//   3. Selection without a global list (FlashHead notes, Module 2): a certain cluster's rank in the
//      Stage-2 list is (keys in higher bins) + (its position in its bin); the block that scored it
//      writes its id at that rank as one 64-bit word tagged with the call's generation, and the
//      boundary bin's (key, id) pairs likewise.  Block 0 ranks the boundary bin exactly (warp rank,
//      or radix passes when crowded — then every block selects on all keys) and writes the ids it
//      selects at the remaining ranks.  Each block polls only the words of its own rows, all before
//      it issues any Stage-2 copy.
//   4. Stage 2 (FlashHead notes, Module 1 and Figure 1): the block streams its slice of the p·b
//      candidate rows, each together with the 16-byte C2T chunk holding its token id, computes the
//      exact logits and keeps the arg-max of z (greedy, Eq. 2) or of z/τ + G' (sampling, Eq. 3).
//   5. Each block folds its best (value, token) into one 64-bit atomicMax; the last block to arrive
//      writes the token and clears the histogram, the selection words and the maximum.
//
// No small global load waits behind the bulk copies: h and the INT4 scales are loaded before the
// Stage-1 copies, the rank words are polled before the Stage-2 copies, and token ids arrive inside the
// row copies.  Stage-2 slots follow the rank order; the arg-max does not depend on it, and the
// optional debug outputs are written in the canonical ascending order.
#include "fh_device.cuh"
#include "fh_kernels.cuh"
#include "fh_select.cuh"
#include "fh_stream.cuh"

namespace fh {

constexpr int kHistBins = 1024;
static_assert(kHead1BndMax == kSelCandMax, "boundary entries = ranked candidates");

struct Head1Layout {
  uint32_t bars1, bars2, hs, sc, sel, hist, ownk, ownp, rank_cl, asc, tokc, ring, total;
};

__host__ __device__ inline uint32_t h1_align(uint32_t x, uint32_t a) { return (x + a - 1) / a * a; }

template <int NT>
__host__ __device__ inline Head1Layout head1_layout(uint32_t row2, int rows1_max, int nch4, int rmax,
                                                    int slots2, uint32_t ring_bytes) {
  // rows1_max: Stage-1 rows of the largest block (its own keys are kept); nch4: INT4 groups per row
  const int sc_rows = nch4 ? rows1_max : 0;
  Head1Layout L;
  L.bars1 = 0;
  L.bars2 = 1024;
  L.hs = 2048;
  L.sc = h1_align(L.hs + row2, 128);
  L.sel = h1_align(L.sc + (uint32_t)sc_rows * nch4 * 2u + 4u, 128);
  L.hist = h1_align(L.sel + (uint32_t)sizeof(SelectSmem<NT>), 16);
  L.ownk = h1_align(L.hist + kHistBins * 4u, 16);
  L.ownp = h1_align(L.ownk + (uint32_t)rows1_max * 4u, 16);
  L.rank_cl = h1_align(L.ownp + (uint32_t)rows1_max * 4u, 16);
  L.asc = h1_align(L.rank_cl + 2u * (uint32_t)rmax * 4u, 16);
  L.tokc = h1_align(L.asc + 2u * (uint32_t)rmax * 4u, 16);
  L.ring = h1_align(L.tokc + (uint32_t)slots2 * 16u, 128);
  L.total = L.ring + ring_bytes;
  return L;
}

// Monotone binning of a key into [0, kHistBins): the same function in Stage 1 and in the selection.
struct Binning {
  float lo, scale;
  __device__ __forceinline__ uint32_t operator()(float x) const {
    const float t = (x - lo) * scale;
    return (uint32_t)min(kHistBins - 1, max(0, (int)t));
  }
};

// Smallest order-preserving key image u with bin(value of u) >= d (d in [1, kHistBins)), found by a
// warp-wide 32-ary search over the images of finite floats; bin is monotone in u there, so a key is in
// a bin >= d exactly when its image is >= the returned edge.  Called by a whole warp.
__device__ __forceinline__ uint32_t bin_edge_image(const Binning& bin, uint32_t d) {
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

// The same edge from the inverse of the binning, corrected by a few one-image steps; falls back to
// the warp search when the correction does not settle.  Called by a whole warp.
__device__ __forceinline__ uint32_t bin_edge(const Binning& bin, uint32_t d) {
  bool ok = false;
  uint32_t u = 0;
  if (bin.scale > 0.0f) {
    const float x0 = bin.lo + (float)d / bin.scale;
    if (isfinite(x0)) {
      u = float_key(x0);
      for (int it = 0; it < 16 && u < 0xFF800000u && bin(key_float(u)) < d; ++it) ++u;
      for (int it = 0; it < 16 && u > 0x00800000u && bin(key_float(u - 1u)) >= d; ++it) --u;
      ok = u > 0x00800000u && u <= 0xFF800000u && bin(key_float(u)) >= d &&
           bin(key_float(u - 1u)) < d;
    }
  }
  return ok ? u : bin_edge_image(bin, d);
}

// Every block computes the same ‖h‖ (same data, same reduction order) and from it the binning.
__device__ __forceinline__ Binning make_binning(const float hnorm, int sample, float tau) {
  Binning bn;
  const float r = hnorm * 1.0625f + 1e-30f;
  const float lo = sample ? -r / tau - 3.0f : -r;
  const float hi = sample ? r / tau + 17.0f : r;
  bn.lo = lo;
  bn.scale = (float)kHistBins / (hi - lo);
  if (!(isfinite(bn.scale) && bn.scale > 0.0f)) bn.scale = 0.0f;  // everything in bin 0
  return bn;
}

__device__ __forceinline__ uint32_t atom_add_release_u32(uint32_t* p, uint32_t v) {
  uint32_t old;
  asm volatile("atom.release.gpu.global.add.u32 %0, [%1], %2;" : "=r"(old) : "l"(p), "r"(v) : "memory");
  return old;
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

__device__ __forceinline__ unsigned long long ld_relaxed_u64(const unsigned long long* p) {
  unsigned long long v;
  asm volatile("ld.relaxed.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
  return v;
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

// Rank the m (<= 32*KP) boundary candidates under (key desc, id asc) and write the ids of the `need`
// best into bsel_rank in rank order.  Every lane keeps KP candidates in registers (absent ones as
// image 0, below every key); each warp ranks four candidates per pass, branch-free.
template <int KP>
__device__ __forceinline__ void rank_boundary(const float* cand_key, const int* cand_id, uint32_t m,
                                              uint32_t need, int* bsel_rank, int lane, int warp,
                                              int nwarps) {
  uint32_t ck[KP];
  int cid[KP];
#pragma unroll
  for (int u = 0; u < KP; ++u) {
    const uint32_t q = (uint32_t)(lane + 32 * u);
    ck[u] = q < m ? __float_as_uint(cand_key[q]) : 0u;
    cid[u] = q < m ? cand_id[q] : 0x7FFFFFFF;
  }
  for (uint32_t i0 = (uint32_t)warp * 4u; i0 < m; i0 += (uint32_t)nwarps * 4u) {
    uint32_t ki[4], rk[4];
    int ii[4];
#pragma unroll
    for (int t = 0; t < 4; ++t) {
      const uint32_t i = i0 + t;
      ki[t] = i < m ? __float_as_uint(cand_key[i]) : 0xFFFFFFFFu;
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
      if (lane == 0 && i0 + t < m && r < need) bsel_rank[r] = ii[t];
    }
  }
}

template <int ELEM, int INT4_MCH, int NT, int KPT>
__global__ void __launch_bounds__(NT, 1) k_head1(const Head1Params prm) {
  extern __shared__ __align__(128) uint8_t smem[];
  constexpr int W = NT / 32;
  __shared__ unsigned long long warp_best[W];
  __shared__ float red_s[W];
  __shared__ bool abort_s, last_s;
  __shared__ uint32_t dstar_s, above_s, total_s, edge_lo_s, edge_hi_s, m_s;
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
  const int K1 = prm.k1, K2 = prm.k2;
  const Head1Layout L = head1_layout<NT>(row2, rows1_max, nch4, rmax, W * K2, prm.ring_bytes);
  uint64_t* bars1 = reinterpret_cast<uint64_t*>(smem + L.bars1);
  uint64_t* bars2 = reinterpret_cast<uint64_t*>(smem + L.bars2);
  uint8_t* hs = smem + L.hs;
  uint16_t* sc_s = reinterpret_cast<uint16_t*>(smem + L.sc);
  SelectSmem<NT>& sm = *reinterpret_cast<SelectSmem<NT>*>(smem + L.sel);
  uint32_t* hist_s = reinterpret_cast<uint32_t*>(smem + L.hist);
  float* own_keys = reinterpret_cast<float*>(smem + L.ownk);
  uint32_t* own_pos = reinterpret_cast<uint32_t*>(smem + L.ownp);
  int* rank_cl = reinterpret_cast<int*>(smem + L.rank_cl);
  int* asc_of = reinterpret_cast<int*>(smem + L.asc);
  uint4* tokc = reinterpret_cast<uint4*>(smem + L.tokc);
  uint8_t* ring = smem + L.ring;

  // ------------------------------------------------------------------ prologue: h before any copy
  uint4 hv[4];
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    const int ch = tid + u * NT;
    if (ch < nch2) hv[u] = __ldg(reinterpret_cast<const uint4*>(prm.H) + ch);
  }
  const int64_t lo1 = uc * (uint32_t)bid / uG, hi1 = uc * (uint32_t)(bid + 1) / uG;
  // this call's tags on its selection entries: 32 bits on the certain ranks, 18 on the boundary bin
  const uint32_t tag = __ldcg(prm.gen) + 1u;
  const uint32_t tag_b = (tag & 0x3FFFFu) | (uint32_t)((tag & 0x3FFFFu) == 0u);
  uint32_t scv[4];  // INT4: this block's group scales, two per 32-bit word
  const int nsc = INT4_MCH ? (int)((hi1 - lo1) * nch4) : 0;
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
  uint64_t* bar_keys = &bars2[127];  // key copy of the full selection
  if (tid == 0) mbar_init(bar_keys, 1);
  fence_mbar_init();
  __syncthreads();

  // ------------------------------------------------------------------ Stage 1
  const int64_t first1 = lo1 + warp;
  const int n1 = (first1 < hi1) ? (int)((hi1 - first1 + W - 1) / W) : 0;
  uint8_t* ring1 = ring + (size_t)warp * K1 * row1;
  uint64_t* b1 = bars1 + warp * K1;
  const uint8_t* src1 = INT4_MCH ? static_cast<const uint8_t*>(static_cast<const void*>(prm.q4))
                                 : static_cast<const uint8_t*>(prm.C);
  if (lane < K1 && lane < n1)  // the first K1 rows of the warp, one lane each
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
  // ‖h‖ (fixed reduction order, identical in every block) and the key binning
  float hsq = 0.0f;
  for (int ch = tid; ch < nch2; ch += NT) {
    const uint4 v = reinterpret_cast<const uint4*>(hs)[ch];
    hsq = (ELEM == kBF16) ? dot8_bf16(v, v, hsq) : dot4_f32(v, v, hsq);
  }
  hsq = warp_sum(hsq);
  if (lane == 0) red_s[warp] = hsq;
  float hreg[INT4_MCH ? INT4_MCH : 1][INT4_MCH ? 32 : 1];
  if constexpr (INT4_MCH > 0) {
    const uint16_t* Hs = reinterpret_cast<const uint16_t*>(hs);
#pragma unroll
    for (int m = 0; m < INT4_MCH; ++m) {
      const int ch = lane + 32 * m;
#pragma unroll
      for (int e = 0; e < 32; ++e)
        hreg[m][e] = (ch < nch4) ? __uint_as_float((uint32_t)Hs[32 * ch + e] << 16) : 0.0f;
    }
  }
  __syncthreads();
  float hn2 = 0.0f;
#pragma unroll
  for (int w = 0; w < W; ++w) hn2 += red_s[w];
  const Binning bin = make_binning(sqrtf(hn2), prm.sample, prm.tau);

  const uint32_t hs_addr = smem_addr(hs);
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
#pragma unroll
      for (int m = 0; m < INT4_MCH; ++m) {
        const int ch = lane + 32 * m;
        if (ch < nch4) {
          const uint4 w = lds_v4(row_s + ch * 16);
          const float scale = __uint_as_float((uint32_t)sc_s[(k - (int)lo1) * nch4 + ch] << 16);
          part = fmaf(scale, int4_group_dot(w, hreg[m]), part);
        }
      }
      s = warp_sum(part);
    } else {
      s = warp_sum(row_dot_partial<ELEM>(row_s, hs_addr, nch2, lane));
    }
    __syncwarp();
    if (lane == 0) {
      if (n + K1 < n1) {
        fence_proxy_async_smem();
        issue_row(ring1 + (size_t)slot * row1, src1 + (size_t)(first1 + (int64_t)W * (n + K1)) * row1,
                  row1, &b1[slot]);
      }
      float key = s;
      if (prm.sample)
        key = s / prm.tau + gumbel_from_u32(philox_word(prm.seed, prm.step, 0u, 0u, (uint32_t)k));
      prm.keys[k] = key;
      own_keys[k - (int)lo1] = key;
      own_pos[k - (int)lo1] = atomicAdd(&hist_s[bin(key_float(float_key(key)))], 1u);
    }
    if (++slot == K1) {
      slot = 0;
      phase ^= 1;
    }
  }
  __syncthreads();
  // Add the block's counts to the global histogram.  The adds are releases (whoever sees a count also
  // sees the keys this block wrote), and each returns the block's first position in that bin, so every
  // key gets a distinct position among the keys of its bin.
  for (int i = tid; i < kHistBins; i += NT) {
    const uint32_t n = hist_s[i];
    if (n) hist_s[i] = atom_add_release_u32(&prm.hist[i], n);
  }

  // ------------------------------------------------------------------ histogram (grid barrier)
  // The summed histogram is complete once its counts add up to c.  Every block polls it until then:
  // the poll is the grid barrier, and its last round already holds the counts the selection needs.
  constexpr int HPT = kHistBins / NT;  // histogram bins per thread
  static_assert(HPT == 2 || HPT == 4, "bins per thread");
  uint32_t hb[HPT];
  uint32_t htot = 0, before = 0;
  for (int i = tid; i < 1025; i += NT) sm.selbits[i] = 0u;
  if (tid == 0) {  // (the polling loop's barriers order these before the boundary search)
    sm.cand_count = 0u;
    dstar_s = 0u;
    above_s = 0u;
  }
  {
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

  // ------------------------------------------------------------------ boundary bin
  uint32_t* histg_s = reinterpret_cast<uint32_t*>(ring);  // keys in bins above each bin
  const bool all = prm.p >= c;
  {
    uint32_t cum = total_s - before - htot;  // keys in bins above this thread's bins
#pragma unroll
    for (int u = HPT - 1; u >= 0; --u) {
      histg_s[tid * HPT + u] = cum;  // from here on: keys in bins above bin tid*HPT+u
      if (!all && cum < (uint32_t)prm.p && cum + hb[u] >= (uint32_t)prm.p) {
        dstar_s = (uint32_t)(tid * HPT + u);
        above_s = cum;
        m_s = hb[u];
      }
      cum += hb[u];
    }
    __syncthreads();
  }
  const uint32_t dstar = all ? 0u : dstar_s;
  const uint32_t above_n = all ? (uint32_t)c : above_s;
  const uint32_t need = (uint32_t)prm.p - above_n;
  const uint32_t m_total = all ? 0u : m_s;
  // Stage-2 rows of this block: its share of the certain rows [c0, c1) and of the boundary rows
  // [d0, d1) (global rows in list order: rank r = row / b, certain ranks first).  Local row l is
  // c0 + l below nc and d0 + (l - nc) above, so certain rows stream while the boundary is resolved.
  const int CR = (int)above_n * b, BR = (int)need * b;
  const int c0 = (int)((uint32_t)CR * (uint32_t)bid / uG), c1 = (int)((uint32_t)CR * (uint32_t)(bid + 1) / uG);
  const int d0 = CR + (int)((uint32_t)BR * (uint32_t)bid / uG);
  const int d1 = CR + (int)((uint32_t)BR * (uint32_t)(bid + 1) / uG);
  const int nc = c1 - c0, nr = nc + (d1 - d0);
  const int rc0 = c0 / b, rc1 = (c1 + b - 1) / b;  // certain ranks touched
  const int rb0 = d0 / b, rb1 = (d1 + b - 1) / b;  // boundary ranks touched
  int* rk_c = rank_cl;
  int* rk_b = rank_cl + rmax;
  int* asc_c = asc_of;
  int* asc_b = asc_of + rmax;
  const bool want_dbg = prm.dbg_sel || prm.dbg_tok || prm.dbg_logit;

  const uint8_t* E = static_cast<const uint8_t*>(prm.E);
  const uint8_t* Ep = static_cast<const uint8_t*>(prm.E_perm);
  const bool perm = Ep != nullptr;
  const int n2 = (warp < nr) ? (nr - warp + W - 1) / W : 0;
  uint8_t* ring2 = ring + (size_t)warp * K2 * row2;
  uint64_t* b2 = bars2 + warp * K2;
  uint4* tokc_w = tokc + warp * K2;
  auto global_row = [&](int l) { return l < nc ? c0 + l : d0 + (l - nc); };
  auto row_e = [&](int g) {  // flat C2T index (= row of the cluster-major copy) of global row g
    const int r = g / b;
    const int cl = (r < (int)above_n) ? rk_c[r - rc0] : rk_b[r - rb0];
    return cl * b + (g - r * b);
  };
  auto issue2 = [&](int n) {
    const int slot = n % K2;
    const int e = row_e(global_row(warp + W * n));
    const int32_t* chunk = prm.C2T + (e & ~3);  // 16-byte chunk holding the token id
    mbar_arrive_expect_tx(&b2[slot], row2 + 16u);
    bulk_g2s(&tokc_w[slot], chunk, 16u, &b2[slot]);
    const uint8_t* src = perm ? Ep + (size_t)e * row2 : E + (size_t)__ldg(prm.C2T + e) * row2;
    bulk_g2s(ring2 + (size_t)slot * row2, src, row2, &b2[slot]);
  };
  const bool fast = all || m_total <= (uint32_t)kSelCandMax;

  if (fast) {
    // ---------------------------------------------------------------- distributed selection
    // A cluster's rank in the Stage-2 list is (keys in higher bins) + (its position in its bin), known
    // to the block that scored it as soon as the histogram is: each block writes the ids of its
    // certain clusters at their ranks, and the (key, id) of its boundary-bin clusters at their
    // positions, each as one 64-bit word tagged with the call's tag.  Block 0 resolves the boundary
    // bin and writes the ranks it fills the same way.  Every block polls only the words its own rows
    // need, so no word is read by more than a few blocks: no counters, no fences, no hot spot.
    const int nk = (int)(hi1 - lo1);
    if (tid < nk) {
      const uint32_t img = float_key(own_keys[tid]);
      const uint32_t dg = bin(key_float(img));
      const uint32_t pos = hist_s[dg] + own_pos[tid];
      const unsigned long long tg = (unsigned long long)tag << 32;
      const uint32_t id = (uint32_t)(lo1 + tid);
      if (all || dg > dstar) {
        st_relaxed_u64(prm.order + histg_s[dg] + pos, tg | id);
      } else if (dg == dstar) {  // (18-bit tag, 14-bit id, key image)
        st_relaxed_u64(prm.bnd + pos, ((unsigned long long)tag_b << 46) |
                                      ((unsigned long long)id << 32) | img);
      }
    }
    // Poll tagged words (each thread at most one of `words`, all loads of a round in flight together);
    // false if a wait gave up (status set).
    auto poll_words = [&](const unsigned long long* words, int n, int* dst) {
      bool ok = true;
      for (int q = tid; q < n; q += NT) dst[q] = (int)(uint32_t)poll_tagged(words + q, tag, prm.status, ok);
      return ok;
    };
    // Every word this block needs is read before any of its Stage-2 copies is issued: a small load
    // issued behind a block's bulk copies waits until they have drained.
    if (need > 0u) {
      if (bid == 0) {
        // The resolver: reads the boundary bin's keys once, ranks them exactly, and writes the ids
        // of the `need` best at ranks above_n .. p - 1, tagged like the certain ones.
        bool ok = true;
        {
          const uint32_t qa = (uint32_t)tid, qb = (uint32_t)(tid + NT);
          uint32_t pend = (qa < m_total ? 1u : 0u) | (qb < m_total ? 2u : 0u);
          const uint64_t t0 = global_timer_ns();
          for (uint32_t it = 1; pend; ++it) {
            unsigned long long v0 = 0ull, v1 = 0ull;
            if (pend & 1u) v0 = ld_relaxed_u64(prm.bnd + qa);
            if (pend & 2u) v1 = ld_relaxed_u64(prm.bnd + qb);
            if ((pend & 1u) && (uint32_t)(v0 >> 46) == tag_b) {
              sm.cand_key[qa] = __uint_as_float((uint32_t)v0);
              sm.cand_id[qa] = (int)((uint32_t)(v0 >> 32) & 0x3FFFu);
              pend &= ~1u;
            }
            if ((pend & 2u) && (uint32_t)(v1 >> 46) == tag_b) {
              sm.cand_key[qb] = __uint_as_float((uint32_t)v1);
              sm.cand_id[qb] = (int)((uint32_t)(v1 >> 32) & 0x3FFFu);
              pend &= ~2u;
            }
            if (pend && (it & 15u) == 0u && global_timer_ns() - t0 > 500000000ull) {
              set_status(prm.status, kStatusTimeout);
              ok = false;
              break;
            }
          }
        }
        if (!__syncthreads_and(ok)) return;
        int* bsel_rank = reinterpret_cast<int*>(sm.selbits);
        if (m_total <= 128u)
          rank_boundary<4>(sm.cand_key, sm.cand_id, m_total, need, bsel_rank, lane, warp, W);
        else
          rank_boundary<kSelCandMax / 32>(sm.cand_key, sm.cand_id, m_total, need, bsel_rank, lane, warp, W);
        __syncthreads();
        const unsigned long long tg = (unsigned long long)tag << 32;
        for (uint32_t r = tid; r < need; r += NT)
          st_relaxed_u64(prm.order + above_n + r, tg | (uint32_t)bsel_rank[r]);
      }
    }
    // the certain and the boundary ranks of this block's rows (the resolver reads back its own words)
    {
      bool ok = poll_words(prm.order + rc0, rc1 - rc0, rk_c);
      if (rb1 > rb0) ok = poll_words(prm.order + rb0, rb1 - rb0, rk_b) && ok;
      if (!__syncthreads_and(ok)) return;
    }
    if (want_dbg) {
      // canonical (ascending) positions: count the selected clusters below each of this block's
      bool ok = true;
      for (int q = tid; q < prm.p; q += NT) poll_tagged(prm.order + q, tag, prm.status, ok);
      if (!__syncthreads_and(ok)) return;
      auto sel_at = [&](int q) { return (int)(uint32_t)__ldcg(prm.order + q); };
      const int ncr = rc1 - rc0, nbr = rb1 - rb0;
      for (int t = warp; t < ncr + nbr; t += W) {
        const int x = t < ncr ? rk_c[t] : rk_b[t - ncr];
        uint32_t cnt = 0;
        for (int q = lane; q < prm.p; q += 32) cnt += (uint32_t)(sel_at(q) < x);
        cnt = __reduce_add_sync(0xFFFFFFFFu, cnt);
        if (lane == 0) {
          if (t < ncr) asc_c[t] = (int)cnt;
          else asc_b[t - ncr] = (int)cnt;
        }
      }
      if (prm.dbg_sel && bid == 0) {
        for (int q = tid; q < prm.p; q += NT) {
          const int x = sel_at(q);
          uint32_t cnt = 0;
          for (int y = 0; y < prm.p; ++y) cnt += (uint32_t)(sel_at(y) < x);
          prm.dbg_sel[cnt] = x;
        }
      }
      __syncthreads();
    }
    if (lane < K2 && lane < n2) {
      fence_proxy_async_smem();  // the ring was last read by Stage 1
      issue2(lane);
    }
  } else {
    // ---------------------------------------------------------------- full selection (crowded bin)
    // More than kSelCandMax keys share the boundary bin: every block loads all keys and selects
    // with the block-wide selector (exact radix passes on the boundary bin).
    const uint32_t keys_bytes = (uint32_t)((c * 4 + 15) / 16 * 16);
    float* keys_s = reinterpret_cast<float*>(ring + kHistBins * 4);
    // Every thread saw some of the release adds of the histogram: its acquire fence makes the keys
    // of those blocks visible, and the barrier passes that on to thread 0, which copies them.
    asm volatile("fence.acq_rel.gpu;" ::: "memory");
    __syncthreads();
    if (tid == 0) {
      asm volatile("fence.proxy.async;" ::: "memory");
      mbar_arrive_expect_tx(bar_keys, keys_bytes);
      bulk_g2s(keys_s, prm.keys, keys_bytes, bar_keys);
    }
    if (!mbar_wait(bar_keys, 0u, prm.status)) return;
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
        if (st.certain >> j & 1u) {
          if (rc >= rc0 && rc < rc1) {
            rk_c[rc - rc0] = base + j;
            asc_c[rc - rc0] = a;
          }
          ++rc;
        } else {
          if (rb >= rb0 && rb < rb1) {
            rk_b[rb - rb0] = base + j;
            asc_b[rb - rb0] = a;
          }
          ++rb;
        }
        if (prm.dbg_sel && bid == 0) prm.dbg_sel[a] = base + j;
      }
    }
    __syncthreads();
    if (lane < K2 && lane < n2) {
      fence_proxy_async_smem();  // the ring was last read by the key copy
      issue2(lane);
    }
  }
  __syncthreads();
  // ------------------------------------------------------------------ Stage 2
  unsigned long long best = 0ull;
  for (int n = 0, slot = 0, phase = 0; n < n2; ++n) {
    if (!mbar_wait(&b2[slot], (uint32_t)phase, prm.status)) {
      for (int m = n + 1; m < n2 && m < n + K2; ++m)
        mbar_wait(&b2[m % K2], (uint32_t)((m / K2) & 1), nullptr, 50000000ull);
      break;
    }
    const int g = global_row(warp + W * n);
    const float z = warp_sum(row_dot_partial<ELEM>(smem_addr(ring2 + (size_t)slot * row2), hs_addr,
                                                   nch2, lane));
    __syncwarp();
    if (lane == 0) {
      const int q = g / b;
      const int e = row_e(g);
      const uint4 ch = tokc_w[slot];
      const uint32_t q4i = (uint32_t)(e & 3);
      const uint32_t tok = q4i == 0 ? ch.x : q4i == 1 ? ch.y : q4i == 2 ? ch.z : ch.w;
      if (n + K2 < n2) {
        fence_proxy_async_smem();
        issue2(n + K2);
      }
      float val = z;
      if (prm.sample)
        val = z / prm.tau + gumbel_from_u32(philox_word(prm.seed, prm.step, 0u, 1u, tok));
      const unsigned long long pk = pack_best(val, tok);
      best = pk > best ? pk : best;
      if (want_dbg) {
        const int ai = ((q < (int)above_n) ? asc_c[q - rc0] : asc_b[q - rb0]) * b + (g - q * b);
        if (prm.dbg_logit) prm.dbg_logit[ai] = z;
        if (prm.dbg_tok) prm.dbg_tok[ai] = (int32_t)tok;
      }
    }
    if (++slot == K2) {
      slot = 0;
      phase ^= 1;
    }
  }

  // ------------------------------------------------------------------ arg-max over the grid
  if (lane == 0) warp_best[warp] = best;
  __syncthreads();
  if (tid == 0) {
    unsigned long long bb = 0ull;
    for (int w = 0; w < W; ++w) bb = warp_best[w] > bb ? warp_best[w] : bb;
    if (bb) atomicMax(prm.best, bb);
    __threadfence();
    const unsigned long long t = atomicAdd(prm.ticket, 1ull);
    last_s = ((t + 1) % (unsigned long long)G) == 0ull;
  }
  __syncthreads();
  if (last_s) {
    __threadfence();
    for (int i = tid; i < kHistBins; i += NT) prm.hist[i] = 0u;
    if (fast) {  // the next call starts from zeroed entries (the tags already tell calls apart)
      for (uint32_t q = tid; q < (uint32_t)prm.p; q += NT) prm.order[q] = 0ull;
      for (uint32_t q = tid; q < m_total; q += NT) prm.bnd[q] = 0ull;
    }
    if (tid == 0) *prm.gen = tag;
    if (tid == 0) {
      const unsigned long long fin = atomicAdd(prm.best, 0ull);
      prm.out_tok[0] = (int32_t)best_id(fin);
      atomicExch(prm.best, 0ull);
    }
  }
}

// ------------------------------------------------------------------ launcher

int head1_threads(int64_t c) { return c <= 256 * 32 ? 256 : (c <= 512 * 32 ? 512 : 0); }

cudaError_t launch_head1(Head1Params prm, int elem, int int4, int num_sms, cudaStream_t st) {
  const int NT = head1_threads(prm.c);
  if (NT == 0) return cudaErrorInvalidValue;
  const int W = NT / 32;
  const int G = num_sms;
  const uint32_t row2 = (uint32_t)(prm.d * (elem == kBF16 ? 2 : 4));
  const uint32_t row1 = int4 ? (uint32_t)(prm.d / 2) : row2;
  if (row2 / 16 > 4u * (uint32_t)NT) return cudaErrorInvalidValue;  // h: 4 chunks per thread
  const int nch4 = int4 ? (int)(prm.d / 32) : 0;
  const int64_t P = (int64_t)prm.p * prm.b;
  if ((prm.c * prm.b) * (int64_t)G >= (int64_t{1} << 31)) return cudaErrorInvalidValue;  // 32-bit splits
  const int rows1_max = (int)((prm.c + G - 1) / G);
  if (int4 && (rows1_max * nch4 + 1) / 2 > 4 * NT) return cudaErrorInvalidValue;
  const int rows2_max = (int)((P + G - 1) / G);
  const int rmax = (int)(rows2_max / prm.b) + 2;
  auto fixed_for = [&](int k2) {
    return (NT == 256 ? head1_layout<256>(row2, rows1_max, nch4, rmax, W * k2, 0)
                      : head1_layout<512>(row2, rows1_max, nch4, rmax, W * k2, 0)).total;
  };
  const uint32_t budget = 220u * 1024u;
  const int kcap = (1024 / 8 - 1) / W;  // barriers per stage (the last one of bars2 is the key copy's)
  const uint32_t fixed = fixed_for(kcap);
  if (fixed + (uint32_t)W * (row2 > row1 ? row2 : row1) > budget) return cudaErrorInvalidValue;
  const uint32_t ring_bytes = (budget - fixed) / 128u * 128u;
  auto slots = [&](uint32_t row, int64_t rows) {
    int64_t k = ring_bytes / ((uint64_t)W * row);
    const int64_t per_warp = (rows + W - 1) / W;
    if (k > per_warp) k = per_warp;
    if (k > kcap) k = kcap;
    return (int)(k < 1 ? 1 : k);
  };
  if (ring_bytes < (uint32_t)((prm.c * 4 + 15) / 16 * 16) + 4096u) return cudaErrorInvalidValue;
  prm.k1 = slots(row1, rows1_max);
  prm.k2 = slots(row2, rows2_max);
  prm.ring_bytes = ring_bytes;
  const size_t smem = fixed_for(prm.k2) + ring_bytes;

  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(G);
  cfg.blockDim = dim3(NT);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
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

// fh_select.cuh — block-wide exact top-p selection over up to NT*KPT keys (KPT <= 32).
//
// FlashHead notes, Module 2 ("multi-probe retrieval"): greedy decoding keeps the p clusters with the
// highest centroid logits; sampling keeps the top p of the Gumbel-perturbed logits.  Order is
// (key desc, id asc) with -0.0 == +0.0, so the selected set is unique.
//
// Thread t holds the keys of ids [t*KPT, t*KPT + KPT) as order-preserving uint32 images in registers;
// ids >= n hold the image 0, below every finite key, and are never counted.  Per-key work is a few
// 32-bit instructions per pass, because at batch 1 one block sweeps all c keys and the selection sits
// on the critical path between the two bandwidth phases.
//
//   topp_bin:     min / max; one 256-bin histogram over the value range [min, max] with
//                 digit(x) = min(255, ⌊(x-min)·256/(max-min)⌋), monotone in x; the boundary bin d* is
//                 where the count from the top first reaches p.  Keys above d* are selected for sure
//                 ("certain"); keys in d* are the boundary set; need = p - #certain of them are taken.
//   topp_resolve: picks exactly `need` boundary keys — by ranking each boundary key against the others
//                 under (key desc, id asc) when there are at most kSelCandMax of them, otherwise by four
//                 8-bit radix passes (exact threshold key T) and an id-ordered scan of the keys equal
//                 to T.
//   block_scan2:  exclusive prefix sums of two per-thread counts (one packed 64-bit scan), used to
//                 place selected ids in ascending id order.
#pragma once

#include "fh_device.cuh"

namespace fh {

constexpr int kSelCandMax = 512;

template <int NT>
struct SelectSmem {
  uint32_t hist[256];
  uint32_t selbits[1025];            // boundary keys chosen by topp_resolve, by id (c <= 32768)
  float cand_key[kSelCandMax];
  int cand_id[kSelCandMax];
  unsigned long long wscan[3][NT / 32];
  uint32_t wcnt[NT / 32];
  uint32_t wmin[NT / 32], wmax[NT / 32];
  uint32_t cand_count;
  int found_bin;
  uint32_t found_above;
};

struct SelState {
  uint32_t certain;   // this thread's keys above the boundary bin (selected)
  uint32_t boundary;  // this thread's keys in the boundary bin
  uint32_t above;     // block-wide number of certain keys
  uint32_t need;      // boundary keys to take: p - above
};

// Warp 0: among the 256 bins, the bin where the count from the top first reaches `target`
// (Σ hist >= target >= 1).  Writes the bin and the count above it.
template <int NT>
__device__ __forceinline__ void find_boundary_bin(SelectSmem<NT>& sm, uint32_t target) {
  const int lane = threadIdx.x & 31;
  const uint4 a = *reinterpret_cast<const uint4*>(&sm.hist[lane * 8]);
  const uint4 b = *reinterpret_cast<const uint4*>(&sm.hist[lane * 8 + 4]);
  const uint32_t h[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
  const uint32_t tot = a.x + a.y + a.z + a.w + b.x + b.y + b.z + b.w;
  uint32_t suf = tot;  // Σ over lanes >= lane
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const uint32_t o = __shfl_down_sync(0xFFFFFFFFu, suf, off);
    if (lane + off < 32) suf += o;
  }
  uint32_t cum = suf - tot;
#pragma unroll
  for (int i = 7; i >= 0; --i) {
    if (cum < target && cum + h[i] >= target) {
      sm.found_bin = lane * 8 + i;
      sm.found_above = cum;
    }
    cum += h[i];
  }
}

// Exclusive prefix sums over the block of two counts per thread (a in the high word, b in the low
// word of the result).  Uses wscan[slot]; one __syncthreads.
template <int NT>
__device__ __forceinline__ unsigned long long block_scan2(uint32_t a, uint32_t b, SelectSmem<NT>& sm,
                                                          int slot) {
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  const unsigned long long v = ((unsigned long long)a << 32) | b;
  unsigned long long incl = v;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const unsigned long long o = __shfl_up_sync(0xFFFFFFFFu, incl, off);
    if (lane >= off) incl += o;
  }
  if (lane == 31) sm.wscan[slot][wid] = incl;
  __syncthreads();
  unsigned long long before = 0ull;
#pragma unroll
  for (int w = 0; w < NT / 32; ++w)
    if (w < wid) before += sm.wscan[slot][w];
  return before + incl - v;
}

// Load helper: order-preserving images of row[base .. base+KPT) (0 beyond n).
template <int KPT>
__device__ __forceinline__ void load_key_images(const float* row, int n, uint32_t (&key)[KPT]) {
  const int base = threadIdx.x * KPT;
  if (base + KPT <= n && (reinterpret_cast<uintptr_t>(row + base) & 15u) == 0) {
#pragma unroll
    for (int j = 0; j < KPT; j += 4) {
      const float4 f = __ldcg(reinterpret_cast<const float4*>(row + base + j));
      key[j] = float_key(f.x);
      key[j + 1] = float_key(f.y);
      key[j + 2] = float_key(f.z);
      key[j + 3] = float_key(f.w);
    }
  } else {
#pragma unroll
    for (int j = 0; j < KPT; ++j) key[j] = (base + j < n) ? float_key(__ldcg(row + base + j)) : 0u;
  }
}

// Phase 1: boundary bin.  Ends with a __syncthreads.
template <int NT, int KPT>
__device__ __forceinline__ SelState topp_bin(const uint32_t (&key)[KPT], int n, int p,
                                             SelectSmem<NT>& sm) {
  static_assert(KPT <= 32, "masks are 32 bits");
  const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
  SelState st;
  uint32_t real = 0;
#pragma unroll
  for (int j = 0; j < KPT; ++j) real |= (key[j] != 0u ? 1u : 0u) << j;
  if (p >= n) {  // everything is selected
    st.certain = real;
    st.boundary = 0u;
    st.above = (uint32_t)n;
    st.need = 0u;
    return st;
  }
  uint32_t mn = 0xFFFFFFFFu, mx = 0u;
#pragma unroll
  for (int j = 0; j < KPT; ++j) {
    mn = min(mn, key[j] ? key[j] : 0xFFFFFFFFu);
    mx = max(mx, key[j]);
  }
  mn = __reduce_min_sync(0xFFFFFFFFu, mn);
  mx = __reduce_max_sync(0xFFFFFFFFu, mx);
  if (lane == 0) {
    sm.wmin[wid] = mn;
    sm.wmax[wid] = mx;
  }
  for (int i = tid; i < 256; i += NT) sm.hist[i] = 0u;
  for (int i = tid; i < 1025; i += NT) sm.selbits[i] = 0u;
  if (tid == 0) sm.cand_count = 0u;
  __syncthreads();
  mn = 0xFFFFFFFFu;
  mx = 0u;
#pragma unroll
  for (int w = 0; w < NT / 32; ++w) {
    mn = min(mn, sm.wmin[w]);
    mx = max(mx, sm.wmax[w]);
  }
  if (mn == mx) {  // all keys equal: the boundary set is everything
    st.certain = 0u;
    st.boundary = real;
    st.above = 0u;
    st.need = (uint32_t)p;
    return st;
  }
  const float lo = key_float(mn);
  const float range = key_float(mx) - lo;
  const float scale = 256.0f / range;
  if (!(isfinite(range) && isfinite(scale) && scale > 0.0f)) {
    st.certain = 0u;
    st.boundary = real;
    st.above = 0u;
    st.need = (uint32_t)p;
    return st;
  }
  uint32_t dig[KPT];
#pragma unroll
  for (int j = 0; j < KPT; ++j) {
    dig[j] = (uint32_t)min(255, (int)((key_float(key[j]) - lo) * scale));
    if (key[j]) atomicAdd(&sm.hist[dig[j]], 1u);
  }
  __syncthreads();
  if (wid == 0) find_boundary_bin(sm, (uint32_t)p);
  __syncthreads();
  const uint32_t dstar = (uint32_t)sm.found_bin;
  st.above = sm.found_above;
  st.need = (uint32_t)p - st.above;
  st.certain = 0u;
  st.boundary = 0u;
#pragma unroll
  for (int j = 0; j < KPT; ++j) {
    st.certain |= (key[j] && dig[j] > dstar ? 1u : 0u) << j;
    st.boundary |= (key[j] && dig[j] == dstar ? 1u : 0u) << j;
  }
  return st;
}

// Phase 2: the boundary keys taken (a mask over this thread's keys).  Ends with a __syncthreads.
template <int NT, int KPT>
__device__ __forceinline__ uint32_t topp_resolve(const uint32_t (&key)[KPT], const SelState& st,
                                                 SelectSmem<NT>& sm) {
  const int tid = threadIdx.x, wid = tid >> 5;
  const int base = tid * KPT;
  if (st.need == 0u) return 0u;
  // block-wide size of the boundary set (every thread computes the same value)
  uint32_t m_local = __popc(st.boundary);
  m_local = __reduce_add_sync(0xFFFFFFFFu, m_local);
  if ((tid & 31) == 0) sm.wcnt[wid] = m_local;
  __syncthreads();
  uint32_t m = 0;
#pragma unroll
  for (int w = 0; w < NT / 32; ++w) m += sm.wcnt[w];
  if (m == st.need) {
    __syncthreads();
    return st.boundary;
  }
  if (m <= (uint32_t)kSelCandMax) {
    // rank each boundary key against the others under (key desc, id asc): candidates are compacted
    // to shared memory, every lane keeps up to kSelCandMax/32 of them in registers, and each warp
    // ranks a share of the candidates with one comparison sweep and one warp reduction apiece.
    // compaction: one shared atomic per warp, then predicated stores at scanned positions
    const int lane = tid & 31;
    const uint32_t nb = __popc(st.boundary);
    uint32_t incl = nb;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const uint32_t o = __shfl_up_sync(0xFFFFFFFFu, incl, off);
      incl += (lane >= off) ? o : 0u;
    }
    const uint32_t wtot = __shfl_sync(0xFFFFFFFFu, incl, 31);
    uint32_t wbase = 0;
    if (lane == 0 && wtot) wbase = atomicAdd(&sm.cand_count, wtot);
    uint32_t pos = __shfl_sync(0xFFFFFFFFu, wbase, 0) + incl - nb;
#pragma unroll
    for (int j = 0; j < KPT; ++j) {  // static indices keep key[] in registers
      const uint32_t bit = st.boundary >> j & 1u;
      if (bit) {
        sm.cand_key[pos] = __uint_as_float(key[j]);  // the image itself orders correctly as uint32
        sm.cand_id[pos] = base + j;
      }
      pos += bit;
    }
    __syncthreads();
    // rank each boundary key against the others under (key desc, id asc): every lane keeps up to
    // kSelCandMax/32 candidates in registers (absent ones as image 0, which no key equals or is below),
    // and each warp ranks a share of the candidates with one branch-free sweep and a warp reduction.
    constexpr int kPer = kSelCandMax / 32;
    uint32_t ck[kPer];
    int cid[kPer];
#pragma unroll
    for (int u = 0; u < kPer; ++u) {
      const uint32_t q = (uint32_t)(lane + 32 * u);
      ck[u] = q < m ? __float_as_uint(sm.cand_key[q]) : 0u;
      cid[u] = q < m ? sm.cand_id[q] : 0x7FFFFFFF;
    }
    for (uint32_t i = wid; i < m; i += NT / 32) {
      const uint32_t ki = __float_as_uint(sm.cand_key[i]);
      const int ii = sm.cand_id[i];
      uint32_t rank = 0;
#pragma unroll
      for (int u = 0; u < kPer; ++u)
        rank += (uint32_t)(ck[u] > ki) + ((uint32_t)(ck[u] == ki) & (uint32_t)(cid[u] < ii));
      rank = __reduce_add_sync(0xFFFFFFFFu, rank);
      if (lane == 0 && rank < st.need) atomicOr(&sm.selbits[ii >> 5], 1u << (ii & 31));
    }
    __syncthreads();
  } else {
    // radix passes over the boundary keys' images → exact threshold key T
    uint32_t prefix = 0, pmask = 0, rem = st.need;
    for (int shift = 24; shift >= 0; shift -= 8) {
      for (int i = tid; i < 256; i += NT) sm.hist[i] = 0u;
      __syncthreads();
#pragma unroll
      for (int j = 0; j < KPT; ++j)
        if ((st.boundary >> j & 1u) && (key[j] & pmask) == prefix)
          atomicAdd(&sm.hist[(key[j] >> shift) & 255u], 1u);
      __syncthreads();
      if (wid == 0) find_boundary_bin(sm, rem);
      __syncthreads();
      prefix |= (uint32_t)sm.found_bin << shift;
      pmask |= 255u << shift;
      rem -= sm.found_above;
    }
    uint32_t gt = 0, eq = 0;
#pragma unroll
    for (int j = 0; j < KPT; ++j) {
      gt |= ((st.boundary >> j & 1u) && key[j] > prefix ? 1u : 0u) << j;
      eq |= ((st.boundary >> j & 1u) && key[j] == prefix ? 1u : 0u) << j;
    }
    // the `rem` lowest ids among the keys equal to T
    const unsigned long long ex = block_scan2<NT>(0u, __popc(eq), sm, 1);
    uint32_t eq_before = (uint32_t)(ex & 0xFFFFFFFFull);
    uint32_t take = gt;
    for (uint32_t bits = eq; bits; bits &= bits - 1) {
      const int j = __ffs(bits) - 1;
      if (eq_before < rem) take |= 1u << j;
      ++eq_before;
    }
    __syncthreads();
    return take;
  }
  // read back this thread's bits (ids base .. base+KPT-1 may straddle two words)
  const uint32_t lo = sm.selbits[base >> 5], hi = sm.selbits[(base >> 5) + 1];
  const uint32_t mine = __funnelshift_r(lo, hi, base & 31) & (KPT == 32 ? 0xFFFFFFFFu : ((1u << KPT) - 1u));
  return mine & st.boundary;
}

// Full top-p: returns this thread's selected mask; when out_ids is not null the p selected ids are
// written there in ascending order.  Ends with a __syncthreads.
template <int NT, int KPT>
__device__ __forceinline__ uint32_t block_select_topp(const uint32_t (&key)[KPT], int n, int p,
                                                      SelectSmem<NT>& sm, int* out_ids) {
  const SelState st = topp_bin<NT, KPT>(key, n, p, sm);
  const uint32_t sel = st.certain | topp_resolve<NT, KPT>(key, st, sm);
  if (out_ids) {
    const unsigned long long ex = block_scan2<NT>(0u, __popc(sel), sm, 0);
    uint32_t pos = (uint32_t)(ex & 0xFFFFFFFFull);
    const int base = threadIdx.x * KPT;
    for (uint32_t bits = sel; bits; bits &= bits - 1) out_ids[pos++] = base + __ffs(bits) - 1;
  }
  __syncthreads();
  return sel;
}

}  // namespace fh

// fh_select.cuh — block-wide exact top-p selection over up to NT*KPT keys.
//
// FlashHead notes, Module 2 ("multi-probe retrieval"): greedy decoding keeps the p clusters with the
// highest centroid logits; sampling keeps the top p of the Gumbel-perturbed logits.  Order is
// (key desc, id asc) with -0.0 == +0.0, so the selected set is unique.
//
// Algorithm (one thread block; thread t holds the keys of ids [t*KPT, t*KPT + KPT) in registers):
//   1. min / max of the keys (order-preserving uint32 images, warp reductions).
//   2. One 256-bin histogram over the value range [min, max]:  digit(x) = min(255, ⌊(x-min)·256/(max-min)⌋)
//      is monotone non-decreasing in x, so all keys of bins above the boundary bin d* are selected and
//      none below it.  d* is the bin where the count from the top first reaches p.
//   3. The boundary bin is resolved exactly: with at most kSelCandMax members, by ranking each member
//      against the others under (key desc, id asc); otherwise by four 8-bit radix passes over the
//      uint32 images of its members, which yield the exact threshold key T and how many keys equal to
//      T are taken (the lowest ids).
//   4. One block-wide exclusive scan of packed (#greater, #equal) counts gives each selected key its
//      position in ascending id order.
// Everything is deterministic; no step depends on the order in which shared-memory atomics land.
#pragma once

#include "fh_device.cuh"

namespace fh {

constexpr int kSelCandMax = 512;

template <int NT>
struct SelectSmem {
  uint32_t hist[256];
  float cand_key[kSelCandMax];
  int cand_id[kSelCandMax];
  uint8_t cand_sel[kSelCandMax];
  unsigned long long warp_scan[NT / 32];
  uint32_t wmin[NT / 32];
  uint32_t wmax[NT / 32];
  uint32_t kmin, kmax;
  uint32_t cand_count;
  int found_bin;
  uint32_t found_above;
};

// Warp 0: among 256 bins, find the bin where the count from the top first reaches `target`.
// Writes the bin and the count of all bins above it.  Requires Σ hist >= target >= 1.
template <int NT>
__device__ __forceinline__ void find_boundary_bin(SelectSmem<NT>& sm, uint32_t target) {
  const int lane = threadIdx.x & 31;
  uint32_t h[8];
  uint32_t tot = 0;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    h[i] = sm.hist[lane * 8 + i];
    tot += h[i];
  }
  uint32_t suf = tot;  // Σ over lanes >= lane
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    uint32_t o = __shfl_down_sync(0xFFFFFFFFu, suf, off);
    if (lane + off < 32) suf += o;
  }
  uint32_t cum = suf - tot;  // count in bins of higher lanes
#pragma unroll
  for (int i = 7; i >= 0; --i) {
    if (cum < target && cum + h[i] >= target) {
      sm.found_bin = lane * 8 + i;
      sm.found_above = cum;
    }
    cum += h[i];
  }
}

// Block-wide exclusive prefix sum of one 64-bit value per thread.
template <int NT>
__device__ __forceinline__ unsigned long long block_exclusive_scan_u64(unsigned long long v,
                                                                        SelectSmem<NT>& sm) {
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  unsigned long long incl = v;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    unsigned long long o = __shfl_up_sync(0xFFFFFFFFu, incl, off);
    if (lane >= off) incl += o;
  }
  if (lane == 31) sm.warp_scan[wid] = incl;
  __syncthreads();
  if (wid == 0) {
    unsigned long long w = (lane < NT / 32) ? sm.warp_scan[lane] : 0ull;
    unsigned long long wi = w;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      unsigned long long o = __shfl_up_sync(0xFFFFFFFFu, wi, off);
      if (lane >= off) wi += o;
    }
    if (lane < NT / 32) sm.warp_scan[lane] = wi - w;
  }
  __syncthreads();
  return incl - v + sm.warp_scan[wid];
}

// Top-p of the keys x (thread t holds ids t*KPT + j, valid when < n).  Returns a bit mask over j of
// this thread's selected keys.  When out_ids is not null, the p selected ids are written there in
// ascending order (out_ids may be shared or global memory).  All threads of the block must call it
// with the same n and p, 1 <= p <= n <= NT*KPT.  Ends with a __syncthreads().
template <int NT, int KPT>
__device__ uint64_t block_select_topp(const float (&x)[KPT], int n, int p, SelectSmem<NT>& sm,
                                      int* out_ids) {
  static_assert(KPT <= 64, "KPT must fit a 64-bit mask");
  const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
  const int base = tid * KPT;

  uint32_t key[KPT];
  uint64_t valid = 0;
#pragma unroll
  for (int j = 0; j < KPT; ++j) {
    const bool ok = base + j < n;
    key[j] = ok ? float_key(x[j]) : 0u;
    if (ok) valid |= 1ull << j;
  }

  uint64_t gt = 0, eq = 0;  // classes: selected outright / tied at the threshold
  uint32_t rem_eq = 0;      // how many of the tied keys are taken (lowest ids first)

  if (p >= n) {
    gt = valid;
  } else {
    // ---- 1. min / max
    uint32_t mn = 0xFFFFFFFFu, mx = 0u;
#pragma unroll
    for (int j = 0; j < KPT; ++j)
      if (valid >> j & 1ull) {
        mn = min(mn, key[j]);
        mx = max(mx, key[j]);
      }
    mn = __reduce_min_sync(0xFFFFFFFFu, mn);
    mx = __reduce_max_sync(0xFFFFFFFFu, mx);
    if (lane == 0) {
      sm.wmin[wid] = mn;
      sm.wmax[wid] = mx;
    }
    for (int i = tid; i < 256; i += NT) sm.hist[i] = 0u;
    if (tid == 0) sm.cand_count = 0u;
    __syncthreads();
    if (wid == 0) {
      uint32_t a = (lane < NT / 32) ? sm.wmin[lane] : 0xFFFFFFFFu;
      uint32_t b = (lane < NT / 32) ? sm.wmax[lane] : 0u;
      a = __reduce_min_sync(0xFFFFFFFFu, a);
      b = __reduce_max_sync(0xFFFFFFFFu, b);
      if (lane == 0) {
        sm.kmin = a;
        sm.kmax = b;
      }
    }
    __syncthreads();
    const uint32_t kmin = sm.kmin, kmax = sm.kmax;

    if (kmin == kmax) {
      eq = valid;  // all keys equal: the p lowest ids
      rem_eq = (uint32_t)p;
    } else {
      const float lo = key_float(kmin), hi = key_float(kmax);
      const float range = hi - lo;
      const float scale = 256.0f / range;
      const bool binned = isfinite(range) && isfinite(scale) && scale > 0.0f;
      uint32_t digit_mask = 0;  // keys in the boundary bin (all keys when not binned)
      uint32_t cand_pos[KPT];
      uint32_t rem = (uint32_t)p;
      int dstar = 0;
      uint64_t in_bin = 0;
      if (binned) {
        uint32_t dig[KPT];
#pragma unroll
        for (int j = 0; j < KPT; ++j) {
          const float xv = key_float(key[j]);
          dig[j] = (uint32_t)min(255, (int)((xv - lo) * scale));
          if (valid >> j & 1ull) atomicAdd(&sm.hist[dig[j]], 1u);
        }
        __syncthreads();
        if (wid == 0) find_boundary_bin(sm, (uint32_t)p);
        __syncthreads();
        dstar = sm.found_bin;
        rem = (uint32_t)p - sm.found_above;
#pragma unroll
        for (int j = 0; j < KPT; ++j)
          if (valid >> j & 1ull) {
            if ((int)dig[j] > dstar) gt |= 1ull << j;
            else if ((int)dig[j] == dstar) in_bin |= 1ull << j;
          }
        (void)digit_mask;
      } else {
        in_bin = valid;
      }
      const uint32_t m = binned ? sm.hist[dstar] : (uint32_t)n;
      if (binned && m <= (uint32_t)kSelCandMax) {
        // ---- 3a. rank the boundary bin's members
#pragma unroll
        for (int j = 0; j < KPT; ++j)
          if (in_bin >> j & 1ull) {
            const uint32_t pos = atomicAdd(&sm.cand_count, 1u);
            cand_pos[j] = pos;
            sm.cand_key[pos] = key_float(key[j]);
            sm.cand_id[pos] = base + j;
          }
        __syncthreads();
        for (uint32_t i = tid; i < m; i += NT) {
          const float ki = sm.cand_key[i];
          const int ii = sm.cand_id[i];
          uint32_t rank = 0;
          for (uint32_t jj = 0; jj < m; ++jj) {
            const float kj = sm.cand_key[jj];
            rank += (kj > ki) || (kj == ki && sm.cand_id[jj] < ii);
          }
          sm.cand_sel[i] = rank < rem ? 1 : 0;
        }
        __syncthreads();
#pragma unroll
        for (int j = 0; j < KPT; ++j)
          if ((in_bin >> j & 1ull) && sm.cand_sel[cand_pos[j]]) gt |= 1ull << j;
      } else {
        // ---- 3b. radix passes over the members' uint32 images
        uint32_t prefix = 0, pmask = 0;
        for (int shift = 24; shift >= 0; shift -= 8) {
          for (int i = tid; i < 256; i += NT) sm.hist[i] = 0u;
          __syncthreads();
#pragma unroll
          for (int j = 0; j < KPT; ++j)
            if ((in_bin >> j & 1ull) && (key[j] & pmask) == prefix)
              atomicAdd(&sm.hist[(key[j] >> shift) & 255u], 1u);
          __syncthreads();
          if (wid == 0) find_boundary_bin(sm, rem);
          __syncthreads();
          prefix |= (uint32_t)sm.found_bin << shift;
          pmask |= 255u << shift;
          rem -= sm.found_above;
          __syncthreads();
        }
#pragma unroll
        for (int j = 0; j < KPT; ++j)
          if (in_bin >> j & 1ull) {
            if (key[j] > prefix) gt |= 1ull << j;
            else if (key[j] == prefix) eq |= 1ull << j;
          }
        rem_eq = rem;
      }
    }
  }

  // ---- 4. positions in ascending id order
  unsigned long long local =
      ((unsigned long long)__popcll(gt) << 32) | (unsigned long long)__popcll(eq);
  unsigned long long excl = block_exclusive_scan_u64<NT>(local, sm);
  uint32_t gt_before = (uint32_t)(excl >> 32), eq_before = (uint32_t)(excl & 0xFFFFFFFFull);
  uint64_t selected = 0;
#pragma unroll
  for (int j = 0; j < KPT; ++j) {
    if (gt >> j & 1ull) {
      if (out_ids) out_ids[gt_before + min(eq_before, rem_eq)] = base + j;
      selected |= 1ull << j;
      ++gt_before;
    } else if (eq >> j & 1ull) {
      if (eq_before < rem_eq) {
        if (out_ids) out_ids[gt_before + eq_before] = base + j;
        selected |= 1ull << j;
      }
      ++eq_before;
    }
  }
  __syncthreads();
  return selected;
}

}  // namespace fh

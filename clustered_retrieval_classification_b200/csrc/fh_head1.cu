// fh_head1.cu — the batch-1 FlashHead head as one persistent cooperative kernel (one block per SM).
//
// At batch 1 the whole call moves ~66 MB (Llama-shaped head), about 10 µs of HBM time on a B200, so
// every launch boundary and every serial step between the two bandwidth phases shows.  One kernel
// therefore runs the whole path (FlashHead notes, overall architecture and Figure 1):
//
//   1. Stage 1: every block bulk-copies its share of centroid rows (C, or the INT4 nibbles) into its
//      shared-memory ring at once, computes s = C·h (or the Gumbel key s/τ + G) and writes the keys.
//   2. Grid barrier (self-resetting arrival counter + generation word, bounded wait).
//   3. Selection, redundantly in every block (FlashHead notes, Module 2): topp_bin finds the boundary
//      bin; the clusters above it are certain, so their Stage-2 rows are issued right away, and the
//      boundary bin is resolved (topp_resolve) while those copies are in flight.
//   4. Stage 2 (FlashHead notes, Module 1 and Figure 1): the block streams its slice of the p·b
//      candidate rows (cluster-major copy E_perm when present, else E through C2T), computes the exact
//      logits and keeps the arg-max of z (greedy, Eq. 2) or of z/τ + G' (sampling, Eq. 3).
//   5. Each block folds its best (value, token) into one 64-bit atomicMax; the last block to arrive
//      writes the token and resets the call's counters.
//
// Slots of Stage 2 are ordered "certain clusters by ascending id, then the boundary clusters taken, by
// ascending id"; the arg-max does not depend on the order, and the optional debug outputs are written
// in the canonical ascending order.
#include "fh_device.cuh"
#include "fh_kernels.cuh"
#include "fh_select.cuh"
#include "fh_stream.cuh"

namespace fh {

struct Head1Layout {
  uint32_t bars1, bars2, hs, sc, sel, rank_cl, asc, tok, ring, total;
};

__host__ __device__ inline uint32_t h1_align(uint32_t x, uint32_t a) { return (x + a - 1) / a * a; }

template <int NT>
__host__ __device__ inline Head1Layout head1_layout(uint32_t row2, int rows1_max, int nch4,
                                                    int rmax, int rows2_max, uint32_t ring_bytes) {
  Head1Layout L;
  L.bars1 = 0;
  L.bars2 = 1024;
  L.hs = 2048;
  L.sc = h1_align(L.hs + row2, 128);
  L.sel = h1_align(L.sc + (uint32_t)rows1_max * nch4 * 2u, 128);
  L.rank_cl = h1_align(L.sel + (uint32_t)sizeof(SelectSmem<NT>), 16);
  L.asc = h1_align(L.rank_cl + (uint32_t)rmax * 4u, 16);
  L.tok = h1_align(L.asc + (uint32_t)rmax * 4u, 16);
  L.ring = h1_align(L.tok + (uint32_t)rows2_max * 4u, 128);
  L.total = L.ring + ring_bytes;
  return L;
}

// Wait for the whole grid.  Returns false if the wait timed out (status set).
__device__ __forceinline__ bool grid_barrier(uint32_t* count, uint32_t* gen, uint32_t nblocks,
                                             uint32_t* status, bool* abort_s) {
  __syncthreads();
  if (threadIdx.x == 0) {
    bool ok = true;
    const uint32_t g0 = *reinterpret_cast<volatile uint32_t*>(gen);
    __threadfence();
    const uint32_t arrived = atomicAdd(count, 1u);
    if (arrived == nblocks - 1) {
      *reinterpret_cast<volatile uint32_t*>(count) = 0u;
      __threadfence();
      atomicAdd(gen, 1u);
    } else {
      const uint64_t t0 = global_timer_ns();
      uint32_t it = 0;
      while (*reinterpret_cast<volatile uint32_t*>(gen) == g0) {
        if ((++it & 255u) == 0 && global_timer_ns() - t0 > 500000000ull) {
          set_status(status, kStatusTimeout);
          ok = false;
          break;
        }
      }
    }
    __threadfence();
    *abort_s = !ok;
  }
  __syncthreads();
  return !*abort_s;
}

template <int ELEM, int INT4_MCH, int NT, int KPT>
__global__ void __launch_bounds__(NT, 1) k_head1(const Head1Params prm) {
  extern __shared__ __align__(128) uint8_t smem[];
  constexpr int W = NT / 32;
  __shared__ unsigned long long warp_best[W];
  __shared__ bool abort_s;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int G = gridDim.x, bid = blockIdx.x;
  const int64_t c = prm.c, d = prm.d, b = prm.b;
  const uint32_t row2 = (uint32_t)(d * (ELEM == kBF16 ? 2 : 4));   // E row bytes
  const uint32_t row1 = INT4_MCH ? (uint32_t)(d / 2) : row2;        // stage-1 row bytes
  const int nch2 = (int)(row2 / 16);
  const int nch4 = INT4_MCH ? (int)(d / 32) : 0;
  const int64_t P = (int64_t)prm.p * b;
  const int rows1_max = (int)((c + G - 1) / G);
  const int rows2_max = (int)((P + G - 1) / G);
  const int rmax = (int)(rows2_max / b) + 2;
  const Head1Layout L =
      head1_layout<NT>(row2, INT4_MCH ? rows1_max : 0, nch4, rmax, rows2_max, prm.ring_bytes);
  uint64_t* bars1 = reinterpret_cast<uint64_t*>(smem + L.bars1);
  uint64_t* bars2 = reinterpret_cast<uint64_t*>(smem + L.bars2);
  uint8_t* hs = smem + L.hs;
  uint16_t* sc_s = reinterpret_cast<uint16_t*>(smem + L.sc);
  SelectSmem<NT>& sm = *reinterpret_cast<SelectSmem<NT>*>(smem + L.sel);
  int* rank_cl = reinterpret_cast<int*>(smem + L.rank_cl);
  int* asc_of = reinterpret_cast<int*>(smem + L.asc);
  int32_t* tok_s = reinterpret_cast<int32_t*>(smem + L.tok);
  uint8_t* ring = smem + L.ring;
  const int K1 = prm.k1, K2 = prm.k2;

  if (tid < W * K1) mbar_init(&bars1[tid], 1);
  if (tid < W * K2) mbar_init(&bars2[tid], 1);
  fence_mbar_init();
  __syncthreads();

  // ------------------------------------------------------------------ Stage 1
  const int64_t lo1 = c * bid / G, hi1 = c * (bid + 1) / G;
  const int64_t first1 = lo1 + warp;
  const int64_t n1 = (first1 < hi1) ? (hi1 - first1 + W - 1) / W : 0;
  uint8_t* ring1 = ring + (size_t)warp * K1 * row1;
  uint64_t* b1 = bars1 + warp * K1;
  const uint8_t* src1 = INT4_MCH ? static_cast<const uint8_t*>(static_cast<const void*>(prm.q4))
                                 : static_cast<const uint8_t*>(prm.C);
  if (lane == 0)
    for (int n = 0; n < K1 && n < n1; ++n)
      issue_row(ring1 + (size_t)n * row1, src1 + (size_t)(first1 + (int64_t)W * n) * row1, row1, &b1[n]);
  block_copy_g2s(hs, static_cast<const uint8_t*>(prm.H), (int)row2);
  float hreg[INT4_MCH ? INT4_MCH : 1][INT4_MCH ? 32 : 1];
  if constexpr (INT4_MCH > 0) {
    for (int64_t i = tid; i < (hi1 - lo1) * nch4; i += NT) sc_s[i] = prm.scales[lo1 * nch4 + i];
    const uint16_t* Hh = static_cast<const uint16_t*>(prm.H);
#pragma unroll
    for (int m = 0; m < (INT4_MCH ? INT4_MCH : 1); ++m) {
      const int ch = lane + 32 * m;
#pragma unroll
      for (int e = 0; e < (INT4_MCH ? 32 : 1); ++e)
        hreg[m][e] = (ch < nch4) ? __uint_as_float((uint32_t)Hh[32 * ch + e] << 16) : 0.0f;
    }
  }
  __syncthreads();
  const uint32_t hs_addr = smem_addr(hs);
  for (int64_t n = 0; n < n1; ++n) {
    const int slot = (int)(n % K1);
    if (!mbar_wait(&b1[slot], (uint32_t)((n / K1) & 1), prm.status)) {
      for (int64_t m = n + 1; m < n1 && m < n + K1; ++m)
        mbar_wait(&b1[m % K1], (uint32_t)((m / K1) & 1), nullptr, 50000000ull);
      break;
    }
    const int64_t k = first1 + (int64_t)W * n;
    const uint32_t row_s = smem_addr(ring1 + (size_t)slot * row1);
    float s;
    if constexpr (INT4_MCH > 0) {
      float part = 0.0f;
#pragma unroll
      for (int m = 0; m < (INT4_MCH ? INT4_MCH : 1); ++m) {
        const int ch = lane + 32 * m;
        if (ch < nch4) {
          const uint4 w = lds_v4(row_s + ch * 16);
          const float scale = __uint_as_float((uint32_t)sc_s[(k - lo1) * nch4 + ch] << 16);
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
    }
  }

  // ------------------------------------------------------------------ grid barrier
  if (!grid_barrier(prm.bar_count, prm.bar_gen, (uint32_t)G, prm.status, &abort_s)) return;

  // ------------------------------------------------------------------ selection
  uint32_t key[KPT];
  load_key_images<KPT>(prm.keys, (int)c, key);
  const SelState st = topp_bin<NT, KPT>(key, (int)c, prm.p, sm);
  const int base = tid * KPT;
  const int64_t s0 = P * bid / G, s1 = P * (bid + 1) / G;
  const int64_t r0 = s0 / b, r1 = (s1 + b - 1) / b;   // ranks this block touches
  const int64_t certain_rows = (int64_t)st.above * b;
  {
    const unsigned long long ex = block_scan2<NT>(__popc(st.certain), 0u, sm, 0);
    int64_t r = (int64_t)(ex >> 32);
    for (uint32_t bits = st.certain; bits; bits &= bits - 1, ++r)
      if (r >= r0 && r < r1) rank_cl[r - r0] = base + __ffs(bits) - 1;
  }
  __syncthreads();
  const uint8_t* E = static_cast<const uint8_t*>(prm.E);
  const uint8_t* Ep = static_cast<const uint8_t*>(prm.E_perm);
  const bool perm = Ep != nullptr;
  const int64_t first2 = s0 + warp;
  const int64_t n2 = (first2 < s1) ? (s1 - first2 + W - 1) / W : 0;
  uint8_t* ring2 = ring + (size_t)warp * K2 * row2;
  uint64_t* b2 = bars2 + warp * K2;
  auto row_src = [&](int64_t i) -> const uint8_t* {
    const int64_t cl = rank_cl[i / b - r0];
    if (perm) return Ep + (size_t)(cl * b + i % b) * row2;
    return E + (size_t)tok_s[i - s0] * row2;
  };
  // certain rows: tokens, then (cluster-major copy) the first copies of each warp
  for (int64_t i = s0 + tid; i < s1 && i < certain_rows; i += NT)
    tok_s[i - s0] = prm.C2T[(int64_t)rank_cl[i / b - r0] * b + i % b];
  int issued = 0;
  if (lane == 0) fence_proxy_async_smem();  // the ring was last read by Stage 1
  if (perm && lane == 0)
    for (int n = 0; n < K2 && n < n2; ++n) {
      const int64_t i = first2 + (int64_t)W * n;
      if (i >= certain_rows) break;
      issue_row(ring2 + (size_t)n * row2, row_src(i), row2, &b2[n]);
      issued = n + 1;
    }
  // resolve the boundary bin while those copies fly
  const uint32_t bsel = topp_resolve<NT, KPT>(key, st, sm);
  {
    const unsigned long long ex = block_scan2<NT>(__popc(bsel), 0u, sm, 1);
    int64_t r = (int64_t)st.above + (int64_t)(ex >> 32);
    for (uint32_t bits = bsel; bits; bits &= bits - 1, ++r)
      if (r >= r0 && r < r1) rank_cl[r - r0] = base + __ffs(bits) - 1;
  }
  const bool want_dbg = prm.dbg_sel || prm.dbg_tok || prm.dbg_logit;
  if (want_dbg) {  // ascending rank of every selected cluster, for the canonical debug order
    const uint32_t sel = st.certain | bsel;
    const unsigned long long ex = block_scan2<NT>(__popc(sel), 0u, sm, 2);
    int64_t a = (int64_t)(ex >> 32);
    const unsigned long long exc = block_scan2<NT>(__popc(st.certain), __popc(bsel), sm, 0);
    int64_t rc = (int64_t)(exc >> 32), rb = (int64_t)st.above + (int64_t)(exc & 0xFFFFFFFFull);
    for (uint32_t bits = sel; bits; bits &= bits - 1, ++a) {
      const int j = __ffs(bits) - 1;
      const int64_t r = (st.certain >> j & 1u) ? rc++ : rb++;
      if (r >= r0 && r < r1) asc_of[r - r0] = (int)a;
      if (prm.dbg_sel && bid == 0) prm.dbg_sel[a] = base + j;
    }
  }
  __syncthreads();
  for (int64_t i = (certain_rows > s0 ? certain_rows : s0) + tid; i < s1; i += NT)
    tok_s[i - s0] = prm.C2T[(int64_t)rank_cl[i / b - r0] * b + i % b];
  __syncthreads();
  if (lane == 0)
    for (int n = issued; n < K2 && n < n2; ++n)
      issue_row(ring2 + (size_t)n * row2, row_src(first2 + (int64_t)W * n), row2, &b2[n]);

  // ------------------------------------------------------------------ Stage 2
  unsigned long long best = 0ull;
  for (int64_t n = 0; n < n2; ++n) {
    const int slot = (int)(n % K2);
    if (!mbar_wait(&b2[slot], (uint32_t)((n / K2) & 1), prm.status)) {
      for (int64_t m = n + 1; m < n2 && m < n + K2; ++m)
        mbar_wait(&b2[m % K2], (uint32_t)((m / K2) & 1), nullptr, 50000000ull);
      break;
    }
    const int64_t i = first2 + (int64_t)W * n;
    const float z = warp_sum(row_dot_partial<ELEM>(smem_addr(ring2 + (size_t)slot * row2), hs_addr,
                                                   nch2, lane));
    __syncwarp();
    if (lane == 0) {
      if (n + K2 < n2) {
        fence_proxy_async_smem();
        issue_row(ring2 + (size_t)slot * row2, row_src(first2 + (int64_t)W * (n + K2)), row2,
                  &b2[slot]);
      }
      const uint32_t tok = (uint32_t)tok_s[i - s0];
      float val = z;
      if (prm.sample)
        val = z / prm.tau + gumbel_from_u32(philox_word(prm.seed, prm.step, 0u, 1u, tok));
      const unsigned long long pk = pack_best(val, tok);
      best = pk > best ? pk : best;
      if (want_dbg) {
        const int64_t ai = (int64_t)asc_of[i / b - r0] * b + i % b;
        if (prm.dbg_logit) prm.dbg_logit[ai] = z;
        if (prm.dbg_tok) prm.dbg_tok[ai] = (int32_t)tok;
      }
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
    const uint32_t t = atomicAdd(prm.ticket, 1u);
    if (t == (uint32_t)G - 1) {
      __threadfence();
      const unsigned long long fin = atomicAdd(prm.best, 0ull);
      prm.out_tok[0] = (int32_t)best_id(fin);
      *prm.best = 0ull;
      *prm.ticket = 0u;
      __threadfence();
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
  const int nch4 = int4 ? (int)(prm.d / 32) : 0;
  const int64_t P = (int64_t)prm.p * prm.b;
  const int rows1_max = (int)((prm.c + G - 1) / G);
  const int rows2_max = (int)((P + G - 1) / G);
  const int rmax = (int)(rows2_max / prm.b) + 2;
  const uint32_t fixed = (NT == 256 ? head1_layout<256>(row2, int4 ? rows1_max : 0, nch4, rmax,
                                                        rows2_max, 0)
                                    : head1_layout<512>(row2, int4 ? rows1_max : 0, nch4, rmax,
                                                        rows2_max, 0)).total;
  const uint32_t budget = 220u * 1024u;
  if (fixed + (uint32_t)W * row2 > budget) return cudaErrorInvalidValue;
  const uint32_t ring_bytes = (budget - fixed) / 128u * 128u;
  auto slots = [&](uint32_t row, int64_t rows) {
    int64_t k = ring_bytes / ((uint64_t)W * row);
    const int64_t per_warp = (rows + W - 1) / W;
    if (k > per_warp) k = per_warp;
    if (k > 1024 / 8 / W) k = 1024 / 8 / W;
    return (int)(k < 1 ? 1 : k);
  };
  prm.k1 = slots(row1, rows1_max);
  prm.k2 = slots(row2, rows2_max);
  prm.ring_bytes = ring_bytes;
  const size_t smem = fixed + ring_bytes;

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
    static bool attr_set = false;                                                                 \
    if (!attr_set) {                                                                              \
      e = cudaFuncSetAttribute(k_head1<EL, M4, NTT, KP>,                                          \
                               cudaFuncAttributeMaxDynamicSharedMemorySize, 227 * 1024);          \
      if (e != cudaSuccess) return e;                                                             \
      attr_set = true;                                                                            \
    }                                                                                             \
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

// fh_kernels.cu — CUDA-core streaming kernels of the FlashHead head (sm_100a).
//
// Every kernel that reads rows of C or E streams them through shared memory with bulk copies
// (cp.async.bulk on the TMA engine): each warp owns a private ring of K row slots, one mbarrier per
// slot, and keeps K rows in flight while it computes the dot product of the previous one with the
// query vector(s) held in shared memory.  Rows are the unit of work, so a C2T-indexed gather costs
// the same as a contiguous stream: every row is 4 KiB of contiguous HBM at the Llama-shaped head.
//
// Kernels:
//   k_stage1<E,QB>   s = C·h for QB queries per block; optional Gumbel-key epilogue   (Stage 1)
//   k_stage1_int4<M> the same from INT4 centroids with BF16 group scales, one query    (Stage 1, INT4)
//   k_stage1_int4_mq<M,QB> INT4 for QB queries per block, each group decoded once      (Stage 1, INT4)
//   k_select<KPT>    top-p per query                                                    (selection)
//   k_build_qmask    per-cluster bit masks of the queries that selected it, and the list of
//                    the clusters (or 128-row tiles) some query selected                (batched Stage 2)
//   k_union_rows<E>  the union of a batch's probe sets, each row read once for the batch (batched Stage 2)
//   k_rows<E,MODE,KPT> candidates (fused selection or given sets) or all rows (dense):
//                    dot, arg-max / Gumbel-max, partial results, last-block reduction   (Stage 2, dense)
// The batch-1 head is one persistent kernel (fh_head1.cu); batched BF16 heads run on the tensor
// cores (fh_tc.cu).
//   k_gather, k_cand_logits, k_gumbel_keys, k_philox                                    (single steps)
//   k_validate_c2t, k_build_perm                                                        (index load)
//   k_mc_*                                                                              (Monte Carlo)
#include <mutex>
#include <utility>
#include <unordered_map>

#include "fh_kernels.cuh"
#include "fh_device.cuh"
#include "fh_select.cuh"
#include "fh_stream.cuh"

namespace fh {

constexpr int kWarps = 8;
constexpr int kThreads = kWarps * 32;

// ============================================================================ Stage 1 (dense C)

template <int ELEM, int QB>
__global__ void __launch_bounds__(kThreads) k_stage1(const Stage1Params prm, int K) {
  extern __shared__ __align__(128) uint8_t smem[];
  pdl_launch_dependents();
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  if (blockIdx.x == 0 && blockIdx.y == 0 && tid < prm.n_tickets) prm.tickets_to_clear[tid] = 0u;

  const uint32_t row_bytes = (uint32_t)(prm.d * (ELEM == kBF16 ? 2 : 4));
  const int nch = (int)(row_bytes / 16);
  const int q0 = blockIdx.y * QB;
  const int nq = min(QB, prm.B - q0);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem);
  uint8_t* hs = smem + 1024;
  uint8_t* ring = hs + (size_t)QB * row_bytes;

  if (tid < kWarps * K) mbar_init(&bars[tid], 1);
  fence_mbar_init();
  for (int q = 0; q < nq; ++q)
    block_copy_g2s(hs + (size_t)q * row_bytes,
                   static_cast<const uint8_t*>(prm.H) + (size_t)(q0 + q) * row_bytes, row_bytes);
  __syncthreads();

  const int64_t lo = prm.c * blockIdx.x / gridDim.x;
  const int64_t hi = prm.c * (blockIdx.x + 1) / gridDim.x;
  const uint8_t* C = static_cast<const uint8_t*>(prm.C);
  const uint32_t hs_addr = smem_addr(hs);
  auto src = [&](int64_t k) { return C + (size_t)k * row_bytes; };
  auto body = [&](int64_t k, uint32_t row_s) {
    float part[QB];
    if constexpr (QB == 1) part[0] = row_dot_partial<ELEM>(row_s, hs_addr, nch, lane);
    else row_dot_partial_multi<ELEM, QB>(row_s, hs_addr, row_bytes, nch, nq, lane, part);
#pragma unroll
    for (int q = 0; q < QB; ++q) {
      if (q < nq) {
        const float s = warp_sum(part[q]);
        if (lane == 0) {
          float out = s;
          if (prm.sample)
            out = s / prm.tau + gumbel_from_u32(philox_word(prm.seed, prm.step, (uint32_t)(q0 + q),
                                                            prm.rng_stream, (uint32_t)k));
          prm.out[(size_t)(q0 + q) * prm.c + k] = out;
        }
      }
    }
  };
  warp_stream_rows(lo + warp, hi, kWarps, lane, ring + (size_t)warp * K * row_bytes, bars + warp * K,
                   K, row_bytes, src, body, prm.status);
}

// ============================================================================ Stage 1 (INT4 C)
// One query per blockIdx.y.  Lane l handles the 16-byte chunks l, l+32, ... of a row (one chunk =
// one 32-column group), so its slice of h lives in registers as fp32.  A nibble n decodes to
// q = (n ^ 8) - 8 through the float pattern 0x4B000000 | (n ^ 8) = 2^23 + (n ^ 8), exactly.

template <int MCH>
__global__ void __launch_bounds__(kThreads) k_stage1_int4(const Stage1Params prm, int K,
                                                          int rows_max) {
  extern __shared__ __align__(128) uint8_t smem[];
  pdl_launch_dependents();
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  if (blockIdx.x == 0 && blockIdx.y == 0 && tid < prm.n_tickets) prm.tickets_to_clear[tid] = 0u;

  const int q = blockIdx.y;
  const int64_t d = prm.d;
  const uint32_t row_bytes = (uint32_t)(d / 2);
  const int nch = (int)(d / 32);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem);
  uint16_t* sc_s = reinterpret_cast<uint16_t*>(smem + 1024);
  uint8_t* ring = smem + 1024 + (((size_t)rows_max * nch * 2 + 127) / 128) * 128;

  const int64_t lo = prm.c * blockIdx.x / gridDim.x;
  const int64_t hi = prm.c * (blockIdx.x + 1) / gridDim.x;
  if (tid < kWarps * K) mbar_init(&bars[tid], 1);
  fence_mbar_init();
  // the block's scales, row-major (hi-lo) x nch
  for (int64_t i = tid; i < (hi - lo) * nch; i += kThreads) sc_s[i] = prm.scales[lo * nch + i];
  // this lane's slice of h
  float hreg[MCH][32];
  const uint4* H = reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(prm.H) + (size_t)q * d);
#pragma unroll
  for (int m = 0; m < MCH; ++m) {
    const int ch = lane + 32 * m;
#pragma unroll
    for (int i = 0; i < 4; ++i) {  // the group's 32 columns: four 16-byte loads
      const uint4 v = (ch < nch) ? __ldg(H + 4 * ch + i) : make_uint4(0u, 0u, 0u, 0u);
      hreg[m][8 * i + 0] = bf16_lo(v.x);
      hreg[m][8 * i + 1] = bf16_hi(v.x);
      hreg[m][8 * i + 2] = bf16_lo(v.y);
      hreg[m][8 * i + 3] = bf16_hi(v.y);
      hreg[m][8 * i + 4] = bf16_lo(v.z);
      hreg[m][8 * i + 5] = bf16_hi(v.z);
      hreg[m][8 * i + 6] = bf16_lo(v.w);
      hreg[m][8 * i + 7] = bf16_hi(v.w);
    }
  }
  __syncthreads();

  auto src = [&](int64_t k) { return prm.q4 + (size_t)k * row_bytes; };
  auto body = [&](int64_t k, uint32_t row_s) {
    float part = 0.0f;
#pragma unroll
    for (int m = 0; m < MCH; ++m) {
      const int ch = lane + 32 * m;
      if (ch < nch) {
        const uint4 w = lds_v4(row_s + ch * 16);
        const float scale = __uint_as_float((uint32_t)sc_s[(k - lo) * nch + ch] << 16);
        part = fmaf(scale, int4_group_dot(w, hreg[m]), part);
      }
    }
    const float s = warp_sum(part);
    if (lane == 0) {
      float out = s;
      if (prm.sample)
        out = s / prm.tau +
              gumbel_from_u32(philox_word(prm.seed, prm.step, (uint32_t)q, prm.rng_stream, (uint32_t)k));
      prm.out[(size_t)q * prm.c + k] = out;
    }
  };
  warp_stream_rows(lo + warp, hi, kWarps, lane, ring + (size_t)warp * K * row_bytes, bars + warp * K,
                   K, row_bytes, src, body, prm.status);
}

// Several queries per block: each INT4 row is read and each group decoded once for QB queries.  The
// queries' h sit in shared memory as fp32, transposed so that the 32 lanes (32 consecutive groups)
// read consecutive 16-byte chunks: hT[q][e/4][group][e%4] for column 32*group + e.
template <int MCH, int QB>
__global__ void __launch_bounds__(kThreads) k_stage1_int4_mq(const Stage1Params prm, int K,
                                                             int rows_max) {
  extern __shared__ __align__(128) uint8_t smem[];
  pdl_launch_dependents();
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  if (blockIdx.x == 0 && blockIdx.y == 0 && tid < prm.n_tickets) prm.tickets_to_clear[tid] = 0u;

  const int q0 = blockIdx.y * QB;
  const int nq = min(QB, prm.B - q0);
  const int64_t d = prm.d;
  const uint32_t row_bytes = (uint32_t)(d / 2);
  const int nch = (int)(d / 32);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem);
  uint16_t* sc_s = reinterpret_cast<uint16_t*>(smem + 1024);
  float* hT = reinterpret_cast<float*>(smem + 1024 + (((size_t)rows_max * nch * 2 + 127) / 128) * 128);
  uint8_t* ring = reinterpret_cast<uint8_t*>(hT + (size_t)QB * d);

  const int64_t lo = prm.c * blockIdx.x / gridDim.x;
  const int64_t hi = prm.c * (blockIdx.x + 1) / gridDim.x;
  if (tid < kWarps * K) mbar_init(&bars[tid], 1);
  fence_mbar_init();
  for (int64_t i = tid; i < (hi - lo) * nch; i += kThreads) sc_s[i] = prm.scales[lo * nch + i];
  const uint16_t* H = static_cast<const uint16_t*>(prm.H);
  for (int64_t i = tid; i < (int64_t)QB * d; i += kThreads) {
    const int q = (int)(i / d), col = (int)(i % d);
    const int ch = col >> 5, e = col & 31;
    hT[(((size_t)q * 8 + (e >> 2)) * nch + ch) * 4 + (e & 3)] =
        q < nq ? __uint_as_float((uint32_t)H[(size_t)(q0 + q) * d + col] << 16) : 0.0f;
  }
  __syncthreads();
  const uint32_t hT_addr = smem_addr(hT);

  auto src = [&](int64_t k) { return prm.q4 + (size_t)k * row_bytes; };
  auto body = [&](int64_t k, uint32_t row_s) {
    float acc[QB];
#pragma unroll
    for (int q = 0; q < QB; ++q) acc[q] = 0.0f;
#pragma unroll
    for (int m = 0; m < MCH; ++m) {
      const int ch = lane + 32 * m;
      if (ch < nch) {
        float dq[32];
        int4_decode32(lds_v4(row_s + ch * 16), dq);
        const float scale = __uint_as_float((uint32_t)sc_s[(k - lo) * nch + ch] << 16);
#pragma unroll
        for (int q = 0; q < QB; ++q) {
          float g = 0.0f;
#pragma unroll
          for (int e4 = 0; e4 < 8; ++e4) {
            const uint4 hv = lds_v4(hT_addr + (uint32_t)((((size_t)q * 8 + e4) * nch + ch) * 16));
            g = fmaf(dq[4 * e4 + 0], __uint_as_float(hv.x), g);
            g = fmaf(dq[4 * e4 + 1], __uint_as_float(hv.y), g);
            g = fmaf(dq[4 * e4 + 2], __uint_as_float(hv.z), g);
            g = fmaf(dq[4 * e4 + 3], __uint_as_float(hv.w), g);
          }
          acc[q] = fmaf(scale, g, acc[q]);
        }
      }
    }
#pragma unroll
    for (int q = 0; q < QB; ++q) {
      const float s = warp_sum(acc[q]);
      if (lane == 0 && q < nq) {
        float out = s;
        if (prm.sample)
          out = s / prm.tau + gumbel_from_u32(philox_word(prm.seed, prm.step, (uint32_t)(q0 + q),
                                                          prm.rng_stream, (uint32_t)k));
        prm.out[(size_t)(q0 + q) * prm.c + k] = out;
      }
    }
  };
  warp_stream_rows(lo + warp, hi, kWarps, lane, ring + (size_t)warp * K * row_bytes, bars + warp * K,
                   K, row_bytes, src, body, prm.status);
}

// ============================================================================ single steps

__global__ void k_gumbel_keys(const float* s, float* keys, int B, int64_t c, float tau, uint64_t seed,
                              uint64_t step, uint32_t rng_stream) {
  const int64_t n = (int64_t)B * c;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n;
       i += (int64_t)gridDim.x * blockDim.x) {
    const int q = (int)(i / c);
    const uint32_t k = (uint32_t)(i % c);
    keys[i] = s[i] / tau + gumbel_from_u32(philox_word(seed, step, (uint32_t)q, rng_stream, k));
  }
}

__global__ void k_philox(uint64_t seed, uint64_t step, uint32_t row, uint32_t rng_stream, int64_t n,
                         uint32_t* out) {
  for (int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e < n;
       e += (int64_t)gridDim.x * blockDim.x)
    out[e] = philox_word(seed, step, row, rng_stream, (uint32_t)e);
}

__global__ void k_gather(const int32_t* C2T, int64_t b, const int32_t* sel, int B, int p,
                         int32_t* cand) {
  const int64_t P = (int64_t)p * b;
  const int64_t n = (int64_t)B * P;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n;
       i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t q = i / P, slot = i % P;
    cand[i] = C2T[(int64_t)sel[q * p + slot / b] * b + slot % b];
  }
}

// One warp per candidate: z = E[tok]·h_q with 16-byte loads straight from global memory.
template <int ELEM>
__global__ void k_cand_logits(const void* E, int64_t d, const void* H, int B, const int32_t* cand,
                              int64_t P, float* out_z) {
  const int lane = threadIdx.x & 31;
  const int64_t warp = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int64_t nwarps = ((int64_t)gridDim.x * blockDim.x) >> 5;
  const int64_t row_bytes = d * (ELEM == kBF16 ? 2 : 4);
  const int nch = (int)(row_bytes / 16);
  for (int64_t i = warp; i < (int64_t)B * P; i += nwarps) {
    const int64_t q = i / P;
    const uint8_t* row = static_cast<const uint8_t*>(E) + (size_t)cand[i] * row_bytes;
    const uint8_t* h = static_cast<const uint8_t*>(H) + (size_t)q * row_bytes;
    float acc = 0.0f;
    for (int ch = lane; ch < nch; ch += 32) {
      const uint4 a = ld_stream_v4(row + ch * 16);
      const uint4 b = __ldg(reinterpret_cast<const uint4*>(h) + ch);
      acc = (ELEM == kBF16) ? dot8_bf16(a, b, acc) : dot4_f32(a, b, acc);
    }
    acc = warp_sum(acc);
    if (lane == 0) out_z[i] = acc;
  }
}

// ============================================================================ selection kernel

// zero / zero_words (optional): a region the blocks clear for the kernel that follows (the query
// masks of a batched Stage 2), which saves it a separate memset.
template <int NT, int KPT>
__global__ void __launch_bounds__(NT) k_select(const float* keys, int32_t* sel, int64_t c, int p,
                                               uint32_t* zero, int zero_words) {
  __shared__ SelectSmem<NT> sm;
  const int q = blockIdx.x;
  pdl_launch_dependents();
  // the cleared region was last read by an earlier call, which had finished before this call began
  for (int i = q * NT + (int)threadIdx.x; i < zero_words; i += (int)gridDim.x * NT) zero[i] = 0u;
  pdl_wait_prior();  // the keys
  uint32_t key[KPT];
  load_key_images<KPT>(keys + (size_t)q * c, (int)c, key);
  block_select_topp<NT, KPT>(key, (int)c, p, sm, sel + (size_t)q * p);
}

// ============================================================================ Stage 2 (batched)
// Candidates of query blockIdx.y from the given probe sets; dot, decision key, running arg-max, partial
// results per block and a last-block reduction per query.

struct RowsSmemLayout {
  uint32_t bars, hs, ring, sel, tok, total;
};

__host__ __device__ inline uint32_t align_up(uint32_t x, uint32_t a) { return (x + a - 1) / a * a; }

__host__ __device__ inline RowsSmemLayout rows_layout(uint32_t row_bytes, int K, int p, int rows_max) {
  RowsSmemLayout L;
  L.bars = 0;
  L.hs = 1024;
  L.ring = align_up(L.hs + row_bytes, 128);
  L.sel = align_up(L.ring + (uint32_t)kWarps * K * row_bytes, 16);
  L.tok = align_up(L.sel + (uint32_t)p * 4u, 16);
  L.total = align_up(L.tok + (uint32_t)rows_max * 4u, 128);
  return L;
}

template <int ELEM>
__global__ void __launch_bounds__(kThreads) k_rows(const Stage2Params prm, int K, int rows_max) {
  extern __shared__ __align__(128) uint8_t smem[];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int q = blockIdx.y;
  const uint32_t row_bytes = (uint32_t)(prm.d * (ELEM == kBF16 ? 2 : 4));
  const int nch = (int)(row_bytes / 16);
  const RowsSmemLayout L = rows_layout(row_bytes, K, prm.p, rows_max);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L.bars);
  uint8_t* hs = smem + L.hs;
  uint8_t* ring = smem + L.ring;
  int* sel_s = reinterpret_cast<int*>(smem + L.sel);
  int32_t* tok_s = reinterpret_cast<int32_t*>(smem + L.tok);
  __shared__ unsigned long long warp_best[kWarps];
  __shared__ bool is_last;

  if (tid < kWarps * K) mbar_init(&bars[tid], 1);
  fence_mbar_init();
  block_copy_g2s(hs, static_cast<const uint8_t*>(prm.H) + (size_t)q * row_bytes, row_bytes);
  for (int r = tid; r < prm.p; r += kThreads) sel_s[r] = prm.sel[(size_t)q * prm.p + r];
  __syncthreads();

  const int64_t b = prm.b;
  const int64_t P = (int64_t)prm.p * b;
  const int64_t lo = P * blockIdx.x / gridDim.x;
  const int64_t hi = P * (blockIdx.x + 1) / gridDim.x;
  const uint8_t* E = static_cast<const uint8_t*>(prm.E);
  const uint8_t* Ep = static_cast<const uint8_t*>(prm.E_perm);
  const bool perm = Ep != nullptr;
  auto src = [&](int64_t i) -> const uint8_t* {
    if (perm) return Ep + (size_t)((int64_t)sel_s[i / b] * b + i % b) * row_bytes;
    return E + (size_t)tok_s[i - lo] * row_bytes;
  };
  const int64_t first = lo + warp;
  int64_t nw = (first < hi) ? (hi - first + kWarps - 1) / kWarps : 0;
  uint8_t* ring_w = ring + (size_t)warp * K * row_bytes;
  uint64_t* bars_w = bars + warp * K;
  // With the cluster-major copy the first rows are issued before the token ids are loaded.
  if (perm && lane == 0)
    for (int n = 0; n < K && n < nw; ++n)
      issue_row(ring_w + (size_t)n * row_bytes, src(first + (int64_t)kWarps * n), row_bytes, &bars_w[n]);
  for (int64_t i = lo + tid; i < hi; i += kThreads)
    tok_s[i - lo] = prm.C2T[(int64_t)sel_s[i / b] * b + i % b];
  __syncthreads();
  if (!perm && lane == 0)
    for (int n = 0; n < K && n < nw; ++n)
      issue_row(ring_w + (size_t)n * row_bytes, src(first + (int64_t)kWarps * n), row_bytes, &bars_w[n]);

  const uint32_t hs_addr = smem_addr(hs);
  unsigned long long best = 0ull;
  for (int64_t n = 0; n < nw; ++n) {
    const int slot = (int)(n % K);
    if (!mbar_wait(&bars_w[slot], (uint32_t)((n / K) & 1), prm.status)) {
      for (int64_t m = n + 1; m < nw && m < n + K; ++m)
        mbar_wait(&bars_w[m % K], (uint32_t)((m / K) & 1), nullptr, 50000000ull);
      break;
    }
    const int64_t i = first + (int64_t)kWarps * n;
    const float z =
        warp_sum(row_dot_partial<ELEM>(smem_addr(ring_w + (size_t)slot * row_bytes), hs_addr, nch, lane));
    __syncwarp();
    if (lane == 0) {
      if (n + K < nw) {
        fence_proxy_async_smem();
        issue_row(ring_w + (size_t)slot * row_bytes, src(first + (int64_t)kWarps * (n + K)), row_bytes,
                  &bars_w[slot]);
      }
      const uint32_t tok = (uint32_t)tok_s[i - lo];
      float val = z;
      if (prm.sample)
        val = z / prm.tau + gumbel_from_u32(philox_word(prm.seed, prm.step, (uint32_t)q, 1u, tok));
      const unsigned long long pk = pack_best(val, tok);
      best = pk > best ? pk : best;
      if (prm.dbg_logit) prm.dbg_logit[(size_t)q * P + i] = z;
      if (prm.dbg_tok) prm.dbg_tok[(size_t)q * P + i] = (int32_t)tok;
    }
  }

  if (lane == 0) warp_best[warp] = best;
  __syncthreads();
  if (tid == 0) {
    unsigned long long bb = 0ull;
    for (int w = 0; w < kWarps; ++w) bb = warp_best[w] > bb ? warp_best[w] : bb;
    prm.part[(size_t)q * gridDim.x + blockIdx.x] = bb;
    __threadfence();
    const uint32_t t = atomicAdd(&prm.tickets[q], 1u);
    is_last = (t == gridDim.x - 1);
  }
  __syncthreads();
  if (is_last && warp == 0) {
    __threadfence();
    unsigned long long bb = 0ull;
    for (uint32_t g = lane; g < gridDim.x; g += 32) {
      const unsigned long long v = __ldcg(&prm.part[(size_t)q * gridDim.x + g]);
      bb = v > bb ? v : bb;
    }
    bb = warp_max_u64(bb);
    if (lane == 0) {
      if (prm.out_tok) prm.out_tok[q] = (int32_t)best_id(bb);
      prm.tickets[q] = 0u;
    }
  }
}

// ============================================================================ Stage 2 (union of the batch)
// Batched Stage 2 over the union of the probe sets (FlashHead notes, Figure 1 Stage 2, for a batch):
// the clusters some query selected, listed once each (in the order k_build_qmask found them), are
// streamed once as whole rows of the cluster-major copy; every row is dotted with the queries whose probe set holds its cluster (the
// cluster's query mask) and folded into those queries' running arg-max.  All B query vectors stay in
// shared memory; block b takes the union's rows [R·b/G, R·(b+1)/G), R = (listed clusters)·b.

struct UnionSmemLayout {
  uint32_t bars, hs, ring, tok, msk, cls, total;
};

__host__ __device__ inline UnionSmemLayout union_layout(uint32_t row_bytes, int B, int NW, int K,
                                                        int rows_max, int cl_max) {
  UnionSmemLayout L;
  L.bars = 0;  // NW * K ring barriers and the query vectors' barrier (NW * K < 128)
  L.hs = 1024;
  L.ring = align_up(L.hs + (uint32_t)B * row_bytes, 128);
  L.tok = align_up(L.ring + (uint32_t)NW * K * row_bytes, 16);
  L.msk = align_up(L.tok + (uint32_t)rows_max * 4u, 16);
  L.cls = align_up(L.msk + (uint32_t)cl_max * 8u, 16);
  L.total = align_up(L.cls + (uint32_t)cl_max * 4u, 128);
  return L;
}

// Lane-partial dot products of a row held in registers (chunk lane + 32·j in ra[j], the first RCH
// chunks of the lane) with one or two staged query vectors: the same four chains, in the same order,
// as row_dot_partial, so the sums are bit-identical to it.
template <int ELEM, int RCH>
__device__ __forceinline__ float cached_dot_partial(const uint4 (&ra)[RCH], uint32_t h_s, int nch, int lane) {
  float a0 = 0.0f, a1 = 0.0f, a2 = 0.0f, a3 = 0.0f;
#pragma unroll
  for (int j = 0; j < RCH; ++j) {
    const int ch = lane + 32 * j;
    if (ch < nch) {
      const uint4 h = lds_v4(h_s + ch * 16);
      if (ELEM == kBF16) {
        a0 = fma2_bf16(ra[j].x, h.x, a0);
        a1 = fma2_bf16(ra[j].y, h.y, a1);
        a2 = fma2_bf16(ra[j].z, h.z, a2);
        a3 = fma2_bf16(ra[j].w, h.w, a3);
      } else {
        a0 = fmaf(__uint_as_float(ra[j].x), __uint_as_float(h.x), a0);
        a1 = fmaf(__uint_as_float(ra[j].y), __uint_as_float(h.y), a1);
        a2 = fmaf(__uint_as_float(ra[j].z), __uint_as_float(h.z), a2);
        a3 = fmaf(__uint_as_float(ra[j].w), __uint_as_float(h.w), a3);
      }
    }
  }
  return (a0 + a1) + (a2 + a3);
}

template <int ELEM, int RCH>
__device__ __forceinline__ void cached_dot2_partial(const uint4 (&ra)[RCH], uint32_t h0, uint32_t h1, int nch,
                                                    int lane, float& z0, float& z1) {
  float a0 = 0.0f, a1 = 0.0f, a2 = 0.0f, a3 = 0.0f, b0 = 0.0f, b1 = 0.0f, b2 = 0.0f, b3 = 0.0f;
#pragma unroll
  for (int j = 0; j < RCH; ++j) {
    const int ch = lane + 32 * j;
    if (ch < nch) {
      const uint4 x = lds_v4(h0 + ch * 16), y = lds_v4(h1 + ch * 16);
      if (ELEM == kBF16) {
        a0 = fma2_bf16(ra[j].x, x.x, a0);
        a1 = fma2_bf16(ra[j].y, x.y, a1);
        a2 = fma2_bf16(ra[j].z, x.z, a2);
        a3 = fma2_bf16(ra[j].w, x.w, a3);
        b0 = fma2_bf16(ra[j].x, y.x, b0);
        b1 = fma2_bf16(ra[j].y, y.y, b1);
        b2 = fma2_bf16(ra[j].z, y.z, b2);
        b3 = fma2_bf16(ra[j].w, y.w, b3);
      } else {
        a0 = fmaf(__uint_as_float(ra[j].x), __uint_as_float(x.x), a0);
        a1 = fmaf(__uint_as_float(ra[j].y), __uint_as_float(x.y), a1);
        a2 = fmaf(__uint_as_float(ra[j].z), __uint_as_float(x.z), a2);
        a3 = fmaf(__uint_as_float(ra[j].w), __uint_as_float(x.w), a3);
        b0 = fmaf(__uint_as_float(ra[j].x), __uint_as_float(y.x), b0);
        b1 = fmaf(__uint_as_float(ra[j].y), __uint_as_float(y.y), b1);
        b2 = fmaf(__uint_as_float(ra[j].z), __uint_as_float(y.z), b2);
        b3 = fmaf(__uint_as_float(ra[j].w), __uint_as_float(y.w), b3);
      }
    }
  }
  z0 = (a0 + a1) + (a2 + a3);
  z1 = (b0 + b1) + (b2 + b3);
}

// Two warp sums with their shuffles interleaved (each the same butterfly as warp_sum).
__device__ __forceinline__ void warp_sum2(float& x, float& y) {
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) {
    const float tx = __shfl_xor_sync(0xFFFFFFFFu, x, off);
    const float ty = __shfl_xor_sync(0xFFFFFFFFu, y, off);
    x += tx;
    y += ty;
  }
}

template <int ELEM, int NW, int RCH>
__global__ void __launch_bounds__(NW * 32, 1) k_union_rows(const UnionParams prm, int K, int rows_max, int cl_max) {
  extern __shared__ __align__(128) uint8_t smem[];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const uint32_t row_bytes = (uint32_t)(prm.d * (ELEM == kBF16 ? 2 : 4));
  const int nch = (int)(row_bytes / 16);
  const UnionSmemLayout L = union_layout(row_bytes, prm.B, NW, K, rows_max, cl_max);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L.bars);
  uint8_t* hs = smem + L.hs;
  uint8_t* ring = smem + L.ring;
  int32_t* tok_s = reinterpret_cast<int32_t*>(smem + L.tok);
  unsigned long long* msk_s = reinterpret_cast<unsigned long long*>(smem + L.msk);
  int32_t* cl_s = reinterpret_cast<int32_t*>(smem + L.cls);  // the block's listed clusters
  __shared__ unsigned long long blk_best[NW][64];
  __shared__ bool is_last;

  uint64_t* hbar = bars + NW * K;  // the query vectors
  if (tid < NW * K + 1) mbar_init(&bars[tid], 1);
  fence_mbar_init();
  __syncthreads();
  // The query vectors are inputs of the whole call, complete before its first kernel began, so they
  // are requested before the wait for the mask builder, which may still be running.
  if (tid == 0) issue_row(hs, prm.H, (uint32_t)prm.B * row_bytes, hbar);
  pdl_wait_prior();

  // 32-bit row arithmetic: the union has at most v < 2^31 rows
  const uint32_t b = (uint32_t)prm.b;
  const int n_cl = __ldcg(prm.cl_count);
  const int64_t R = (int64_t)n_cl * b;
  const uint32_t lo = (uint32_t)(R * blockIdx.x / gridDim.x), hi = (uint32_t)(R * (blockIdx.x + 1) / gridDim.x);
  const uint32_t c_lo = lo / b;  // first listed cluster this block touches
  const uint32_t c_hi = hi > lo ? (hi - 1) / b + 1 : c_lo;
  const uint8_t* Ep = static_cast<const uint8_t*>(prm.E_perm);
  auto src = [&](uint32_t i) -> const uint8_t* {
    const uint32_t ci = i / b;
    return Ep + ((size_t)cl_s[ci - c_lo] * b + (i - ci * b)) * row_bytes;
  };
  const uint32_t first = lo + warp;
  const int nw = (first < hi) ? (int)((hi - first + NW - 1) / NW) : 0;
  uint8_t* ring_w = ring + (size_t)warp * K * row_bytes;
  uint64_t* bars_w = bars + warp * K;

  for (uint32_t ci = c_lo + tid; ci < c_hi; ci += NW * 32) cl_s[ci - c_lo] = __ldcg(prm.cl_list + ci);
  __syncthreads();
  // the first rows, then the token ids and the cluster masks
  if (lane == 0)
    for (int n = 0; n < K && n < nw; ++n)
      issue_row(ring_w + (size_t)n * row_bytes, src(first + (uint32_t)(NW * n)), row_bytes, &bars_w[n]);
  for (uint32_t i = lo + tid; i < hi; i += NW * 32) {
    const uint32_t ci = i / b;
    tok_s[i - lo] = __ldg(prm.C2T + (size_t)cl_s[ci - c_lo] * b + (i - ci * b));
  }
  for (uint32_t ci = c_lo + tid; ci < c_hi; ci += NW * 32) msk_s[ci - c_lo] = __ldcg(prm.qmask + cl_s[ci - c_lo]);
  const bool h_ok = mbar_wait(hbar, 0u, prm.status);
  if (!__syncthreads_and(h_ok)) {  // (status recorded) the rows already requested land first
    if (lane == 0)
      for (int n = 0; n < K && n < nw; ++n) mbar_wait(&bars_w[n], 0u, nullptr, 50000000ull);
    return;
  }

  const uint32_t hs_addr = smem_addr(hs);
  unsigned long long best0 = 0ull, best1 = 0ull;  // queries lane and lane + 32
  // Sampling: the row's Gumbel terms are drawn before its dot products, lane l for queries l and
  // l + 32 of the cluster's mask, all lanes at once (rather than one lane per (row, query) after the
  // sum), so the draws overlap the products.
  float g0 = 0.0f, g1 = 0.0f;
  auto draw = [&](unsigned long long mk, uint32_t tok) {
    if (mk >> lane & 1ull)
      g0 = gumbel_from_u32(philox_word(prm.seed, prm.step, (uint32_t)lane, 1u, tok));
    if (mk >> (lane + 32) & 1ull)
      g1 = gumbel_from_u32(philox_word(prm.seed, prm.step, (uint32_t)(lane + 32), 1u, tok));
  };
  auto fold = [&](int q, float z, uint32_t tok) {
    if (lane == (q & 31)) {
      float val = z;
      if (prm.sample) val = z / prm.tau + (q < 32 ? g0 : g1);
      const unsigned long long pk = pack_best(val, tok);
      if (q < 32) best0 = pk > best0 ? pk : best0;
      else best1 = pk > best1 ? pk : best1;
    }
  };
  auto refill = [&](int n, int slot) {  // the slot's next row, once every lane is done reading it
    __syncwarp();
    if (lane == 0 && n + K < nw) {
      fence_proxy_async_smem();
      issue_row(ring_w + (size_t)slot * row_bytes, src(first + (uint32_t)(NW * (n + K))), row_bytes,
                &bars_w[slot]);
    }
  };
  for (int n = 0; n < nw; ++n) {
    const int slot = (int)(n % K);
    if (!mbar_wait(&bars_w[slot], (uint32_t)((n / K) & 1), prm.status)) {
      for (int m = n + 1; m < nw && m < n + K; ++m)
        mbar_wait(&bars_w[m % K], (uint32_t)((m / K) & 1), nullptr, 50000000ull);
      break;
    }
    const uint32_t i = first + (uint32_t)(NW * n);
    const uint32_t row_s = smem_addr(ring_w + (size_t)slot * row_bytes);
    const uint32_t tok = (uint32_t)tok_s[i - lo];
    unsigned long long mk = msk_s[i / b - c_lo];
    if (prm.sample) draw(mk, tok);
    if constexpr (RCH > 0) {
      // the row into registers, its slot refilled at once, then the cluster's queries two at a time
      uint4 ra[RCH];
#pragma unroll
      for (int j = 0; j < RCH; ++j) {
        const int ch = lane + 32 * j;
        ra[j] = ch < nch ? lds_v4(row_s + ch * 16) : make_uint4(0u, 0u, 0u, 0u);
      }
#pragma unroll
      for (int j = 0; j < RCH; ++j)  // the loads have returned before the slot is handed back
        asm volatile("" : "+r"(ra[j].x), "+r"(ra[j].y), "+r"(ra[j].z), "+r"(ra[j].w));
      refill(n, slot);
      while (mk) {  // the same queries in every lane
        const int q0 = __ffsll((long long)mk) - 1;
        mk &= mk - 1;
        if (mk) {
          const int q1 = __ffsll((long long)mk) - 1;
          mk &= mk - 1;
          float z0, z1;
          cached_dot2_partial<ELEM, RCH>(ra, hs_addr + (uint32_t)q0 * row_bytes, hs_addr + (uint32_t)q1 * row_bytes,
                                         nch, lane, z0, z1);
          warp_sum2(z0, z1);
          fold(q0, z0, tok);
          fold(q1, z1, tok);
        } else {
          fold(q0, warp_sum(cached_dot_partial<ELEM, RCH>(ra, hs_addr + (uint32_t)q0 * row_bytes, nch, lane)), tok);
        }
      }
    } else {
      while (mk) {  // the same queries in every lane
        const int q = __ffsll((long long)mk) - 1;
        mk &= mk - 1;
        fold(q, warp_sum(row_dot_partial<ELEM>(row_s, hs_addr + (uint32_t)q * row_bytes, nch, lane)), tok);
      }
      refill(n, slot);
    }
  }

  blk_best[warp][lane] = best0;
  blk_best[warp][lane + 32] = best1;
  __syncthreads();
  if (tid < prm.B) {
    unsigned long long bb = 0ull;
    for (int w = 0; w < NW; ++w) bb = blk_best[w][tid] > bb ? blk_best[w][tid] : bb;
    if (bb) atomicMax(prm.best + tid, bb);
  }
  __threadfence();
  __syncthreads();
  if (tid == 0) is_last = atomicAdd(prm.ticket, 1u) + 1u == gridDim.x;
  __syncthreads();
  if (is_last) {  // every other block has added its maxima: publish, and leave zeros for the next call
    __threadfence();
    if (tid < prm.B) {
      const unsigned long long fin = atomicExch(prm.best + tid, 0ull);
      prm.out_tok[tid] = fin ? (int32_t)best_id(fin) : -1;
    }
    if (tid == 0) atomicExch(prm.ticket, 0u);
  }
}

// Dense head: the same kernel over all rows; logits optionally written out.
template <int ELEM>
__global__ void __launch_bounds__(kThreads) k_dense(const DenseParams prm, int K) {
  extern __shared__ __align__(128) uint8_t smem[];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int q = blockIdx.y;
  const uint32_t row_bytes = (uint32_t)(prm.d * (ELEM == kBF16 ? 2 : 4));
  const int nch = (int)(row_bytes / 16);
  const RowsSmemLayout L = rows_layout(row_bytes, K, 0, 0);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L.bars);
  uint8_t* hs = smem + L.hs;
  uint8_t* ring = smem + L.ring;
  __shared__ unsigned long long warp_best[kWarps];
  __shared__ bool is_last;
  if (tid < kWarps * K) mbar_init(&bars[tid], 1);
  fence_mbar_init();
  block_copy_g2s(hs, static_cast<const uint8_t*>(prm.H) + (size_t)q * row_bytes, row_bytes);
  __syncthreads();

  const int64_t lo = prm.v * blockIdx.x / gridDim.x;
  const int64_t hi = prm.v * (blockIdx.x + 1) / gridDim.x;
  const uint8_t* E = static_cast<const uint8_t*>(prm.E);
  const uint32_t hs_addr = smem_addr(hs);
  unsigned long long best = 0ull;
  auto src = [&](int64_t t) { return E + (size_t)t * row_bytes; };
  auto body = [&](int64_t t, uint32_t row_s) {
    const float z = warp_sum(row_dot_partial<ELEM>(row_s, hs_addr, nch, lane));
    if (lane == 0) {
      float val = z;
      if (prm.sample)
        val = z / prm.tau + gumbel_from_u32(philox_word(prm.seed, prm.step, (uint32_t)q, 1u, (uint32_t)t));
      const unsigned long long pk = pack_best(val, (uint32_t)t);
      best = pk > best ? pk : best;
      if (prm.out_logits) prm.out_logits[(size_t)q * prm.v + t] = z;
    }
  };
  warp_stream_rows(lo + warp, hi, kWarps, lane, ring + (size_t)warp * K * row_bytes, bars + warp * K,
                   K, row_bytes, src, body, prm.status);

  if (lane == 0) warp_best[warp] = best;
  __syncthreads();
  if (tid == 0) {
    unsigned long long bb = 0ull;
    for (int w = 0; w < kWarps; ++w) bb = warp_best[w] > bb ? warp_best[w] : bb;
    prm.part[(size_t)q * gridDim.x + blockIdx.x] = bb;
    __threadfence();
    const uint32_t t = atomicAdd(&prm.tickets[q], 1u);
    is_last = (t == gridDim.x - 1);
  }
  __syncthreads();
  if (is_last && warp == 0) {
    __threadfence();
    unsigned long long bb = 0ull;
    for (uint32_t g = lane; g < gridDim.x; g += 32) {
      const unsigned long long v = __ldcg(&prm.part[(size_t)q * gridDim.x + g]);
      bb = v > bb ? v : bb;
    }
    bb = warp_max_u64(bb);
    if (lane == 0) {
      if (prm.out_tok) prm.out_tok[q] = (int32_t)best_id(bb);
      prm.tickets[q] = 0u;
    }
  }
}

// ============================================================================ index load

__global__ void k_validate_c2t(const int32_t* C2T, int64_t v, uint32_t* bitmap, uint32_t* status) {
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < v;
       i += (int64_t)gridDim.x * blockDim.x) {
    const int32_t t = C2T[i];
    if (t < 0 || (int64_t)t >= v) {
      set_status(status, kStatusIndex);
      continue;
    }
    const uint32_t bit = 1u << (t & 31);
    const uint32_t old = atomicOr(&bitmap[t >> 5], bit);
    if (old & bit) set_status(status, kStatusIndex);
  }
}

__global__ void k_build_perm(const uint8_t* E, const int32_t* C2T, int64_t v, int64_t row_bytes,
                             uint8_t* E_perm) {
  const int lane = threadIdx.x & 31;
  const int64_t warp = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int64_t nwarps = ((int64_t)gridDim.x * blockDim.x) >> 5;
  for (int64_t r = warp; r < v; r += nwarps) {
    const uint4* s = reinterpret_cast<const uint4*>(E + (size_t)C2T[r] * row_bytes);
    uint4* d = reinterpret_cast<uint4*>(E_perm + (size_t)r * row_bytes);
    for (int64_t ch = lane; ch < row_bytes / 16; ch += 32) d[ch] = s[ch];
  }
}

// ============================================================================ Monte Carlo
// FlashHead notes, Module 4 and Eq. 7.  The candidates of a draw are whole clusters, so the softmax
// denominator over cand(S_i) equals Σ_{k∈S_i} Z_k with Z_k = Σ_{u∈cluster k} exp(z_u/τ - zmax):
// the S-independent part is computed once per query and each draw only selects and sums.

__global__ void k_mc_cluster_of(const int32_t* C2T, int64_t v, int64_t b, int32_t* cluster_of) {
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < v;
       i += (int64_t)gridDim.x * blockDim.x)
    cluster_of[C2T[i]] = (int32_t)(i / b);
}

__global__ void k_mc_zmax(const float* z, int64_t v, float tau, float* zmax) {
  __shared__ float red[32];
  const int q = blockIdx.x;
  float m = -INFINITY;
  for (int64_t t = threadIdx.x; t < v; t += blockDim.x) m = fmaxf(m, z[(size_t)q * v + t] / tau);
  for (int off = 16; off > 0; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, off));
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = m;
  __syncthreads();
  if (threadIdx.x < 32) {
    m = (threadIdx.x < blockDim.x / 32) ? red[threadIdx.x] : -INFINITY;
    for (int off = 16; off > 0; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, off));
    if (threadIdx.x == 0) zmax[q] = m;
  }
}

// Z[q][k] = Σ_{u in cluster k} exp(z_u/τ - zmax_q): one warp per (query, cluster), lane j takes the
// cluster's rows j, j+32, ... and a fixed shuffle tree sums them (deterministic).
__global__ void k_mc_partition(const float* z, const int32_t* C2T, int64_t v, int64_t c, int64_t b,
                               float tau, const float* zmax, double* Z, int B) {
  const int lane = threadIdx.x & 31;
  const int64_t nw = ((int64_t)gridDim.x * blockDim.x) >> 5;
  for (int64_t i = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5; i < (int64_t)B * c; i += nw) {
    const int64_t q = i / c, k = i % c;
    const double m = (double)zmax[q];
    double acc = 0.0;
    for (int64_t j = lane; j < b; j += 32)
      acc += exp((double)z[(size_t)q * v + C2T[k * b + j]] / (double)tau - m);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(0xFFFFFFFFu, acc, off);
    if (lane == 0) Z[i] = acc;
  }
}

constexpr int kMcThreads = 512;

template <int KPT>
__global__ void __launch_bounds__(kMcThreads) k_mc_draws(const McParams prm) {
  __shared__ SelectSmem<kMcThreads> sm;
  __shared__ double red[kMcThreads / 32];
  __shared__ double denom_s;
  __shared__ int32_t tcl[64];     // cluster of each target
  __shared__ double tnum[64];     // exp(z_t/τ - zmax)
  __shared__ uint8_t tsel[64];
  const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
  const int q = blockIdx.y;
  const int64_t c = prm.c;
  const int base = tid * KPT;
  const double m = (double)prm.zmax[q];
  for (int j = tid; j < prm.T; j += kMcThreads) {
    const int32_t t = prm.targets[(size_t)q * prm.T + j];
    if (t < 0 || (int64_t)t >= prm.v) {  // out-of-range target: reported, probability 0
      set_status(prm.status, kStatusIndex);
      tcl[j] = -1;
      tnum[j] = 0.0;
      continue;
    }
    tcl[j] = prm.cluster_of[t];
    tnum[j] = exp((double)prm.z[(size_t)q * prm.v + t] / (double)prm.tau - m);
  }
  float sdiv[KPT];
#pragma unroll
  for (int j = 0; j < KPT; ++j)
    sdiv[j] = (base + j < c) ? prm.s[(size_t)q * c + base + j] / prm.tau : 0.0f;
  __syncthreads();

  const int64_t lo = prm.N * blockIdx.x / gridDim.x;
  const int64_t hi = prm.N * (blockIdx.x + 1) / gridDim.x;
  for (int64_t i = lo; i < hi; ++i) {
    uint32_t key[KPT];
#pragma unroll
    for (int g = 0; g < KPT / 4; ++g) {
      const uint4 w = philox_block(prm.seed, (uint64_t)(prm.i0 + i), (uint32_t)q, 2u, (uint32_t)((base >> 2) + g));
      const uint32_t wv[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int j = 4 * g + e;
        key[j] = (base + j < c) ? float_key(sdiv[j] + gumbel_from_u32(wv[e])) : 0u;
      }
    }
    const uint32_t mine = block_select_topp<kMcThreads, KPT>(key, (int)c, prm.p, sm, nullptr);
    double acc = 0.0;
    for (uint32_t bits = mine; bits; bits &= bits - 1)
      acc += prm.Z[(size_t)q * c + base + __ffs(bits) - 1];
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(0xFFFFFFFFu, acc, off);
    if (lane == 0) red[wid] = acc;
    for (int j = 0; j < prm.T; ++j) {
      const int k = tcl[j];
      if (k >= base && k < base + KPT) tsel[j] = (mine >> (k - base)) & 1u ? 1 : 0;
    }
    __syncthreads();
    if (tid == 0) {
      double dsum = 0.0;
      for (int w = 0; w < kMcThreads / 32; ++w) dsum += red[w];
      denom_s = dsum;
    }
    __syncthreads();
    for (int j = tid; j < prm.T; j += kMcThreads)
      prm.per_draw[((size_t)q * prm.N + i) * prm.T + j] = (tcl[j] >= 0 && tsel[j]) ? tnum[j] / denom_s : 0.0;
    __syncthreads();
  }
}

__global__ void k_mc_reduce(const double* per_draw, int64_t N, int T, int B, double* mean,
                            double* se) {
  const int lane = threadIdx.x & 31;
  const int w = (int)(((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5);
  if (w >= B * T) return;
  const int q = w / T, j = w % T;
  double s = 0.0;
  for (int64_t i = lane; i < N; i += 32) s += per_draw[((size_t)q * N + i) * T + j];
  for (int off = 16; off > 0; off >>= 1) s += __shfl_xor_sync(0xFFFFFFFFu, s, off);
  const double mu = s / (double)N;
  double ss = 0.0;
  for (int64_t i = lane; i < N; i += 32) {
    const double dl = per_draw[((size_t)q * N + i) * T + j] - mu;
    ss += dl * dl;
  }
  for (int off = 16; off > 0; off >>= 1) ss += __shfl_xor_sync(0xFFFFFFFFu, ss, off);
  if (lane == 0) {
    mean[w] = mu;
    se[w] = (N > 1) ? sqrt(ss / (double)(N - 1)) / sqrt((double)N) : 0.0;
  }
}

// ============================================================================ launchers

// Ring slots per warp for rows of row_bytes within `budget` bytes of ring: at least 1, at most 16 (the
// kernels keep kWarps x 16 mbarriers in their first 1024 bytes of shared memory).
static int ring_slots(uint32_t row_bytes, uint32_t budget) {
  int k = (int)(budget / ((uint32_t)kWarps * row_bytes));
  return k < 1 ? 1 : (k > 16 ? 16 : k);
}

// Raise a kernel's dynamic shared-memory limit to `bytes`, remembering the limits already set so
// that repeated launches skip the driver call.
template <typename Kern>
static cudaError_t set_smem(Kern kern, size_t bytes) {
  return set_smem_attr(reinterpret_cast<const void*>(kern), bytes);
}

// Launch `kern` with programmatic stream serialisation when `overlap` is set: its blocks may be
// scheduled once every block of the preceding kernel has signalled launch_dependents, and the kernel
// waits (pdl_wait_prior) before it reads anything that kernel wrote.  Only for launches that follow
// another kernel of the same call on the stream.
template <typename... KArgs, typename... Args>
static cudaError_t launch_k(bool overlap, void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem,
                            cudaStream_t st, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = overlap ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
}

cudaError_t set_smem_attr(const void* kernel, size_t bytes) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  static std::mutex mu;
  static std::unordered_map<const void*, size_t> limit[kMaxDevices];
  std::lock_guard<std::mutex> lock(mu);
  auto it = limit[dev].find(kernel);
  if (it != limit[dev].end() && it->second >= bytes) return cudaSuccess;
  e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
  if (e == cudaSuccess) limit[dev][kernel] = bytes;
  return e;
}

cudaError_t launch_stage1(const Stage1Params& prm, int elem, int int4, int num_sms,
                          cudaStream_t st, bool pdl_primary) {
  (void)pdl_primary;
  if (int4) {
    const uint32_t row_bytes = (uint32_t)(prm.d / 2);
    const int K = ring_slots(row_bytes, 96 * 1024);
    const int G = num_sms;
    const int rows_max = (int)((prm.c + G - 1) / G);
    const int nch = (int)(prm.d / 32);
    const size_t smem = 1024 + (((size_t)rows_max * nch * 2 + 127) / 128) * 128 +
                        (size_t)kWarps * K * row_bytes;
    cudaError_t e;
    if (prm.B > 1) {  // eight queries per block
      constexpr int QB = 8;
      const size_t smem_mq = 1024 + (((size_t)rows_max * nch * 2 + 127) / 128) * 128 +
                             (size_t)QB * prm.d * 4 + (size_t)kWarps * K * row_bytes;
      dim3 grid_mq(G, (prm.B + QB - 1) / QB);
#define FH_S1Q(M)                                                                   \
  do {                                                                              \
    if ((e = set_smem(k_stage1_int4_mq<M, QB>, smem_mq)) != cudaSuccess) return e;  \
    k_stage1_int4_mq<M, QB><<<grid_mq, kThreads, smem_mq, st>>>(prm, K, rows_max);  \
  } while (0)
      if (nch <= 32) FH_S1Q(1);
      else if (nch <= 64) FH_S1Q(2);
      else FH_S1Q(4);
#undef FH_S1Q
      return cudaGetLastError();
    }
    dim3 grid(G, prm.B);
    if (nch <= 32) {
      if ((e = set_smem(k_stage1_int4<1>, smem)) != cudaSuccess) return e;
      k_stage1_int4<1><<<grid, kThreads, smem, st>>>(prm, K, rows_max);
    } else if (nch <= 64) {
      if ((e = set_smem(k_stage1_int4<2>, smem)) != cudaSuccess) return e;
      k_stage1_int4<2><<<grid, kThreads, smem, st>>>(prm, K, rows_max);
    } else {
      if ((e = set_smem(k_stage1_int4<4>, smem)) != cudaSuccess) return e;
      k_stage1_int4<4><<<grid, kThreads, smem, st>>>(prm, K, rows_max);
    }
    return cudaGetLastError();
  }
  const uint32_t row_bytes = (uint32_t)(prm.d * (elem == kBF16 ? 2 : 4));
  const int K = ring_slots(row_bytes, 160 * 1024);
  const int QB = prm.B == 1 ? 1 : 4;
  const size_t smem = 1024 + (size_t)QB * row_bytes + (size_t)kWarps * K * row_bytes;
  dim3 grid(num_sms, (prm.B + QB - 1) / QB);
  cudaError_t e;
#define FH_S1(EL, Q)                                                          \
  do {                                                                        \
    if ((e = set_smem(k_stage1<EL, Q>, smem)) != cudaSuccess) return e;       \
    k_stage1<EL, Q><<<grid, kThreads, smem, st>>>(prm, K);                    \
  } while (0)
  if (elem == kBF16) {
    if (QB == 1) FH_S1(kBF16, 1); else FH_S1(kBF16, 4);
  } else {
    if (QB == 1) FH_S1(kF32, 1); else FH_S1(kF32, 4);
  }
#undef FH_S1
  return cudaGetLastError();
}

cudaError_t launch_gumbel_keys(const float* s, float* keys, int B, int64_t c, float tau,
                               uint64_t seed, uint64_t step, uint32_t rng_stream, cudaStream_t st) {
  const int64_t n = (int64_t)B * c;
  const int blocks = (int)((n + 255) / 256 < 4096 ? (n + 255) / 256 : 4096);
  k_gumbel_keys<<<blocks, 256, 0, st>>>(s, keys, B, c, tau, seed, step, rng_stream);
  return cudaGetLastError();
}

cudaError_t launch_select(const float* keys, int32_t* sel, int B, int64_t c, int p, cudaStream_t st,
                          void* zero, size_t zero_bytes) {
  uint32_t* z = static_cast<uint32_t*>(zero);
  const int zw = zero ? (int)(zero_bytes / 4) : 0;  // a few hundred KB at most
  // a selection that clears the masks is the batched head's, right after its Stage-1 kernel
  const bool ov = zero != nullptr;
  if (c <= 512 * 4) return launch_k(ov, k_select<512, 4>, B, 512, 0, st, keys, sel, c, p, z, zw);
  if (c <= 512 * 8) return launch_k(ov, k_select<512, 8>, B, 512, 0, st, keys, sel, c, p, z, zw);
  if (c <= 512 * 16) return launch_k(ov, k_select<512, 16>, B, 512, 0, st, keys, sel, c, p, z, zw);
  if (c <= 512 * 32) return launch_k(ov, k_select<512, 32>, B, 512, 0, st, keys, sel, c, p, z, zw);
  return launch_k(ov, k_select<1024, 32>, B, 1024, 0, st, keys, sel, c, p, z, zw);
}

// List slots for the lanes that claim one: one returning add per converged group of lanes (rather
// than one per lane, which serialises on the counter's address), each claimant's slot ranked by lane.
// Returns -1 to the others.
__device__ __forceinline__ int32_t claim_slot(int32_t* count, bool need) {
  const unsigned act = __activemask();
  const unsigned m = __ballot_sync(act, need);
  if (m == 0u) return -1;
  const int lane = threadIdx.x & 31, leader = __ffs(m) - 1;
  int32_t base = 0;
  if (lane == leader) base = atomicAdd(count, __popc(m));
  base = __shfl_sync(act, base, leader);
  return need ? base + __popc(m & ((1u << lane) - 1u)) : -1;
}

// qmask[cluster] |= 1 << q for every cluster in query q's probe set (qmask zeroed beforehand).
// list (optional, with *count zeroed like qmask): the clusters with a nonzero mask, each appended once
// by the query that sets its first bit (in no particular order).
// Bit q of qmask[k]: query q selected cluster k.  The first selection of a cluster lists it (the
// union Stage 2) or, with tile_flags, lists every tile_rows-row tile of the cluster-major copy it
// overlaps that no earlier cluster listed (the tensor-core Stage 2; any order will do).
__global__ void k_build_qmask(const int32_t* __restrict__ sel, int B, int p, unsigned long long* qmask,
                              int32_t* list, int32_t* count, uint32_t* tile_flags, int64_t b,
                              int64_t rows, int tile_rows) {
  pdl_launch_dependents();
  pdl_wait_prior();  // the probe sets and the cleared masks
  const int64_t n = (int64_t)B * p;
  // a cluster of b rows overlaps at most this many tiles
  const int64_t span = tile_flags ? (b - 1 + tile_rows - 1) / tile_rows + 1 : 1;
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x) {
    const int32_t k = __ldcg(sel + i);
    const unsigned long long old = atomicOr(qmask + k, 1ull << (uint32_t)(i / p));
    if (!list) continue;
    const bool first = old == 0ull;
    if (!tile_flags) {
      const int32_t s = claim_slot(count, first);
      if (first) list[s] = k;
    } else {
      const int64_t r0 = (int64_t)k * b, r1 = (r0 + b < rows ? r0 + b : rows) - 1;
      for (int64_t j = 0; j < span; ++j) {
        const int64_t t = r0 / tile_rows + j;
        const bool mine = first && t <= r1 / tile_rows && atomicExch(tile_flags + t, 1u) == 0u;
        const int32_t s = claim_slot(count, mine);
        if (mine) list[s] = (int32_t)t;
      }
    }
  }
}

cudaError_t launch_build_qmask(const int32_t* sel, int B, int p, unsigned long long* qmask,
                               cudaStream_t st, int32_t* list, int32_t* count, uint32_t* tile_flags,
                               int64_t b, int64_t rows, int tile_rows, bool overlap) {
  const int64_t n = (int64_t)B * p;
  const int blocks = (int)((n + 255) / 256 < 1024 ? (n + 255) / 256 : 1024);
  return launch_k(overlap, k_build_qmask, blocks, 256, 0, st, sel, B, p, qmask, list, count, tile_flags, b,
                  rows, tile_rows);
}

int stage2_blocks(int64_t rows, int B, int num_sms) {
  int64_t g = (B == 1) ? num_sms : (2 * (int64_t)num_sms + B - 1) / B;
  const int64_t max_g = (rows + 7) / 8;  // at least ~8 rows per block
  if (g > max_g) g = max_g;
  return (int)(g < 1 ? 1 : g);
}

cudaError_t launch_stage2(const Stage2Params& prm, int elem, int num_sms, cudaStream_t st) {
  const uint32_t row_bytes = (uint32_t)(prm.d * (elem == kBF16 ? 2 : 4));
  const int K = ring_slots(row_bytes, 128 * 1024);
  const int64_t P = (int64_t)prm.p * prm.b;
  const int G = stage2_blocks(P, prm.B, num_sms);
  const int rows_max = (int)((P + G - 1) / G);
  const RowsSmemLayout L = rows_layout(row_bytes, K, prm.p, rows_max);
  const size_t smem = L.total;
  cudaError_t e;
  if (elem == kBF16) {
    if ((e = set_smem(k_rows<kBF16>, smem)) != cudaSuccess) return e;
    k_rows<kBF16><<<dim3(G, prm.B), kThreads, smem, st>>>(prm, K, rows_max);
  } else {
    if ((e = set_smem(k_rows<kF32>, smem)) != cudaSuccess) return e;
    k_rows<kF32><<<dim3(G, prm.B), kThreads, smem, st>>>(prm, K, rows_max);
  }
  return cudaGetLastError();
}

// Warps and ring slots of the union kernel at batch B: the most warps (16, 12, 8) for which a ring
// of two slots each fits beside the query vectors, with as many slots as fit, within the opt-in
// shared memory of a block less the kernel's static arrays; 0 slots: the query vectors leave no room
// for a ring of two.  More warps beat more rows in flight (Llama shape, greedy, µs a call at 8 / 12 /
// 16 queries: 16 warps × 2 slots 69.2 / 84.2 / 99.5; the split with the most rows in flight, 8 × 5,
// 8 × 5 and 12 × 3, 90.5 / 113.3 / 109.6).
#ifndef FH_UNION_SMEM_CAP
#define FH_UNION_SMEM_CAP (227u * 1024u)
#endif
#ifndef FH_UNION_WARPS
#define FH_UNION_WARPS 0  // 16, 12 or 8 to fix the warp count
#endif
static int union_slots(uint32_t row_bytes, int B, int rows_max, int cl_max, int* nw, size_t* smem) {
  for (int NW : {16, 12, 8}) {
    if (FH_UNION_WARPS != 0 && NW != FH_UNION_WARPS) continue;
    const uint32_t cap = FH_UNION_SMEM_CAP - (uint32_t)NW * 64u * 8u - 128u;  // blk_best, is_last
    for (int K = 128 / NW - 1; K >= 2; --K) {
      const UnionSmemLayout L = union_layout(row_bytes, B, NW, K, rows_max, cl_max);
      if (L.total <= cap) {
        *nw = NW;
        *smem = L.total;
        return K;
      }
    }
  }
  return 0;
}

bool union_supported(int elem, int64_t d, int64_t v, int64_t b, int B, int num_sms) {
  if (B < 1 || B > 64) return false;
  const uint32_t row_bytes = (uint32_t)(d * (elem == kBF16 ? 2 : 4));
  const int rows_max = (int)((v + num_sms - 1) / num_sms);
  size_t smem = 0;
  int nw = 0;
  return union_slots(row_bytes, B, rows_max, (int)(rows_max / b + 2), &nw, &smem) >= 2;
}

cudaError_t launch_union_rows(const UnionParams& prm, int elem, int num_sms, cudaStream_t st) {
  const uint32_t row_bytes = (uint32_t)(prm.d * (elem == kBF16 ? 2 : 4));
  const int G = num_sms;
  const int rows_max = (int)((prm.v + G - 1) / G);  // the union has at most v rows
  const int cl_max = (int)(rows_max / prm.b + 2);
  size_t smem = 0;
  int NW = 0;
  const int K = union_slots(row_bytes, prm.B, rows_max, cl_max, &NW, &smem);
  if (K < 2) return cudaErrorInvalidValue;
  // rows of up to 256 16-byte chunks (4 KB) are held in registers, 8 chunks a lane
  const bool cached = row_bytes <= 256u * 16u;
  cudaError_t e;
#define FH_UN(EL, W, R)                                                                      \
  do {                                                                                       \
    if ((e = set_smem(k_union_rows<EL, W, R>, smem)) != cudaSuccess) return e;               \
    e = launch_k(true, k_union_rows<EL, W, R>, G, W * 32, smem, st, prm, K, rows_max, cl_max); \
  } while (0)
#define FH_UN_W(EL, R)                 \
  do {                                 \
    if (NW == 16) FH_UN(EL, 16, R);    \
    else if (NW == 12) FH_UN(EL, 12, R); \
    else FH_UN(EL, 8, R);              \
  } while (0)
  if (elem == kBF16) {
    if (cached) FH_UN_W(kBF16, 8); else FH_UN_W(kBF16, 0);
  } else {
    if (cached) FH_UN_W(kF32, 8); else FH_UN_W(kF32, 0);
  }
#undef FH_UN_W
#undef FH_UN
  return e;
}

cudaError_t launch_dense(const DenseParams& prm, int elem, int num_sms, cudaStream_t st) {
  const uint32_t row_bytes = (uint32_t)(prm.d * (elem == kBF16 ? 2 : 4));
  const int K = ring_slots(row_bytes, 128 * 1024);
  const int G = stage2_blocks(prm.v, prm.B, num_sms);
  const RowsSmemLayout L = rows_layout(row_bytes, K, 0, 0);
  const size_t smem = L.total;
  cudaError_t e;
  if (elem == kBF16) {
    if ((e = set_smem(k_dense<kBF16>, smem)) != cudaSuccess) return e;
    k_dense<kBF16><<<dim3(G, prm.B), kThreads, smem, st>>>(prm, K);
  } else {
    if ((e = set_smem(k_dense<kF32>, smem)) != cudaSuccess) return e;
    k_dense<kF32><<<dim3(G, prm.B), kThreads, smem, st>>>(prm, K);
  }
  return cudaGetLastError();
}

cudaError_t launch_gather(const int32_t* C2T, int64_t b, const int32_t* sel, int B, int p,
                          int32_t* cand, cudaStream_t st) {
  const int64_t n = (int64_t)B * p * b;
  const int blocks = (int)((n + 255) / 256 < 4096 ? (n + 255) / 256 : 4096);
  k_gather<<<blocks, 256, 0, st>>>(C2T, b, sel, B, p, cand);
  return cudaGetLastError();
}

cudaError_t launch_cand_logits(const void* E, int elem, int64_t d, const void* H, int B,
                               const int32_t* cand, int64_t P, float* out_z, cudaStream_t st) {
  const int64_t warps = (int64_t)B * P;
  const int blocks = (int)((warps * 32 + 255) / 256 < 8192 ? (warps * 32 + 255) / 256 : 8192);
  if (elem == kBF16) k_cand_logits<kBF16><<<blocks, 256, 0, st>>>(E, d, H, B, cand, P, out_z);
  else k_cand_logits<kF32><<<blocks, 256, 0, st>>>(E, d, H, B, cand, P, out_z);
  return cudaGetLastError();
}

cudaError_t launch_philox(uint64_t seed, uint64_t step, uint32_t row, uint32_t rng_stream, int64_t n,
                          uint32_t* out, cudaStream_t st) {
  const int blocks = (int)((n + 255) / 256 < 4096 ? (n + 255) / 256 : 4096);
  k_philox<<<blocks, 256, 0, st>>>(seed, step, row, rng_stream, n, out);
  return cudaGetLastError();
}

cudaError_t launch_validate_c2t(const int32_t* C2T, int64_t v, uint32_t* bitmap, uint32_t* status,
                                cudaStream_t st) {
  const int blocks = (int)((v + 255) / 256 < 4096 ? (v + 255) / 256 : 4096);
  k_validate_c2t<<<blocks, 256, 0, st>>>(C2T, v, bitmap, status);
  return cudaGetLastError();
}

cudaError_t launch_build_perm(const void* E, const int32_t* C2T, int64_t v, int64_t d, int elem,
                              void* E_perm, cudaStream_t st) {
  const int64_t row_bytes = d * (elem == kBF16 ? 2 : 4);
  k_build_perm<<<1184, 256, 0, st>>>(static_cast<const uint8_t*>(E), C2T, v, row_bytes,
                                     static_cast<uint8_t*>(E_perm));
  return cudaGetLastError();
}

cudaError_t launch_mc(const McParams& prm, int num_sms, cudaStream_t st) {
  cudaError_t e;
  k_mc_cluster_of<<<1024, 256, 0, st>>>(prm.C2T, prm.v, prm.b, const_cast<int32_t*>(prm.cluster_of));
  k_mc_zmax<<<prm.B, 1024, 0, st>>>(prm.z, prm.v, prm.tau, prm.zmax);
  k_mc_partition<<<4 * num_sms, 256, 0, st>>>(prm.z, prm.C2T, prm.v, prm.c, prm.b, prm.tau, prm.zmax,
                                               prm.Z, prm.B);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  int64_t gd = (4 * (int64_t)num_sms + prm.B - 1) / prm.B;
  if (gd > prm.N) gd = prm.N;
  dim3 grid((unsigned)gd, prm.B);
#define FH_MC(KP) k_mc_draws<KP><<<grid, kMcThreads, 0, st>>>(prm)
  if (prm.c <= kMcThreads * 4) FH_MC(4);
  else if (prm.c <= kMcThreads * 8) FH_MC(8);
  else if (prm.c <= kMcThreads * 12) FH_MC(12);
  else if (prm.c <= kMcThreads * 16) FH_MC(16);
  else if (prm.c <= kMcThreads * 20) FH_MC(20);
  else if (prm.c <= kMcThreads * 24) FH_MC(24);
  else FH_MC(32);
#undef FH_MC
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  const int warps = prm.B * prm.T;
  k_mc_reduce<<<(warps * 32 + 255) / 256, 256, 0, st>>>(prm.per_draw, prm.N, prm.T, prm.B,
                                                       prm.out_mean, prm.out_se);
  return cudaGetLastError();
}

}  // namespace fh

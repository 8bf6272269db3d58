// fh_tc.cu — tensor-core logits for a batch of queries: Z = A · Hᵀ over 128-row tiles of A with
// tcgen05.mma (BF16 in, FP32 accumulators in tensor memory), the per-query candidate mask and the
// token decision fused into the epilogue.
//
// Used where the head is a dense contraction: the batched dense head (A = E, every row a candidate)
// and batched FlashHead Stage 2 (A = the cluster-major copy of E; a row takes part for query q when
// q's probe set holds the row's cluster — FlashHead notes, Module 1 and Figure 1, and Eq. 2/3 for the
// decision).  Stage 2 lists the clusters some query selected and gathers them, 128 rows (whole
// clusters) per tile, so every needed row is read once for all queries; the epilogue masks each
// (row, query) pair by whether the query selected the row's cluster.
//
// One persistent CTA per SM, 8 warps with fixed roles:
//   warp 0      TMA producer: K-blocks of 64 columns of the A tile (128 rows) and of H (N rows),
//               128-byte swizzled, into a ring of S shared-memory stages;
//   warp 1      MMA issuer: four 128 x N x 16 tcgen05.mma per stage into one of two TMEM accumulators;
//   warp 2      allocates and frees the tensor memory (two accumulators, each in one half);
//   warps 4..7  epilogue: each reads its 32 TMEM lanes (rows) of the finished accumulator, applies the
//               mask (and the Gumbel term when sampling), and reduces the arg-max of every query.
// The two accumulators let the epilogue of one tile overlap the MMAs of the next.  Every wait is
// bounded: on a timeout the CTA records it, drains its own copies and MMAs, frees TMEM and leaves.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <mutex>  // std::call_once

#include "fh_device.cuh"
#include "fh_kernels.cuh"
#include "fh_stream.cuh"

namespace fh {
namespace {

constexpr int kTcKB = 64;          // K elements per stage: one 128-byte swizzle atom per row
constexpr int kTcThreads = 256;
constexpr uint32_t kTcSmemBudget = 200u * 1024u;

// ------------------------------------------------------------------ tcgen05 / TMA primitives

// Shared-memory matrix descriptor of a K-major operand in the 128-byte swizzled layout: rows of 128 B,
// 8-row groups 1024 B apart (stride byte offset 64 in 16-byte units, leading offset unused = 1),
// descriptor version 1, layout type 2 (SWIZZLE_128B).
__device__ __forceinline__ uint64_t sw128_desc(uint32_t saddr) {
  return (uint64_t)((saddr & 0x3FFFFu) >> 4) | ((uint64_t)1 << 16) | ((uint64_t)64 << 32) |
         ((uint64_t)1 << 46) | ((uint64_t)2 << 61);
}

// Instruction descriptor of kind::f16: FP32 accumulator, BF16 A and B, both K-major, M x N.
template <int N>
__host__ __device__ constexpr uint32_t idesc_bf16(int M) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}
static_assert(idesc_bf16<128>(128) == ((1u << 4) | (1u << 7) | (1u << 10) | (16u << 17) | (8u << 24)), "idesc");

__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, int x, int y,
                                            uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];"
      ::"r"(smem_addr(dst)), "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(smem_addr(bar))
      : "memory");
}

__device__ __forceinline__ void mma_bf16(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                         uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, {%5, %6, %7, %8}, p;\n\t}\n"
      ::"r"(d_tmem), "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(0u), "r"(0u), "r"(0u), "r"(0u)
      : "memory");
}

// Arrive (once) on `bar` when every tcgen05 operation this thread issued so far has completed.
__device__ __forceinline__ void mma_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];"
               ::"r"(smem_addr(bar)) : "memory");
}

__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// 32 lanes x 16 columns of 32-bit accumulators: thread t of the warp gets lane (taddr.lane + t).
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, "
      "%13, %14, %15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
}
__device__ __forceinline__ void tmem_ld_wait() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

// Bounded wait for phase `parity` of `bar`; gives up when another role set *abort or after 0.5 s
// (then it records the timeout and sets *abort itself).
__device__ __forceinline__ bool tc_wait(uint64_t* bar, uint32_t parity, volatile int* abort,
                                        uint32_t* status) {
  uint64_t t0 = 0;
  for (uint32_t it = 1;; ++it) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((it & 255u) == 0) {
      if (*abort) return false;
      const uint64_t now = global_timer_ns();
      if (t0 == 0) {
        t0 = now;
      } else if (now - t0 > 500000000ull) {
        set_status(status, kStatusTimeout);
        *abort = 1;
        return false;
      }
    }
  }
}

// ------------------------------------------------------------------ the kernel
//
// D = H · E_tileᵀ: the MMA's M side is the queries (H padded to 128 rows with zeros), its N side the
// 128 rows of an E tile, so tensor-memory lane q holds query q and column r row r of the tile.  Each
// epilogue thread owns one query and reduces its arg-max along its own columns: no cross-lane work.

constexpr int kTcRows = 128;                       // E rows per tile (the MMA's N)
constexpr int kTcWave = 512 / kTcRows;             // tiles whose accumulators fit tensor memory

template <int S, bool SAMPLE>
struct TcLayout {
  static constexpr uint32_t kBlk = 128u * 128u;    // one K-block of H or of an E tile: 128 rows x 128 B
  static constexpr uint32_t kHOff = S * kBlk;      // S stages of E blocks, then 2 of H blocks
  static constexpr uint32_t kRowOff = kHOff + 2 * kBlk;            // tile rows: token, mask
  static constexpr uint32_t kClOff = kRowOff + kTcRows * 12u;        // the wave's cluster ids
  static constexpr uint32_t kGumOff = kClOff + kTcWave * 16u * 4u;  // sampling: 4 warps x 32 x 32 G
  static constexpr uint32_t kPairOff = kGumOff + (SAMPLE ? 4u * 32u * 32u * 4u : 0u);  // and pairs
  static constexpr uint32_t kBars = kPairOff + (SAMPLE ? 4u * 64u * 4u : 0u) + 64u;
  static constexpr uint32_t kDyn = kBars + 1024u + 1024u;          // + barriers, + alignment slack
};

// KEYS: write the products (Stage-1 keys) instead of reducing an arg-max; SAMPLE: add the Gumbel
// term.  Separate instantiations keep each epilogue's code out of the other modes' instruction stream.
template <int S, bool KEYS, bool SAMPLE>
__global__ void __launch_bounds__(kTcThreads, 1)
    k_tc_head(const __grid_constant__ CUtensorMap tmE, const __grid_constant__ CUtensorMap tmH,
              const TcParams a) {
  using Lay = TcLayout<S, SAMPLE>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023u) & ~uintptr_t(1023));
  uint32_t* tok_s = reinterpret_cast<uint32_t*>(smem + Lay::kRowOff);                     // 128
  unsigned long long* msk_s = reinterpret_cast<unsigned long long*>(smem + Lay::kRowOff + 512u);  // 128
  int32_t* wave_cl = reinterpret_cast<int32_t*>(smem + Lay::kClOff);  // kTcWave x gpt
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + Lay::kBars);
  uint64_t* empty = full + S;
  uint64_t* hfull = empty + S;     // H block landed
  uint64_t* hempty = hfull + 2;    // H block no longer read
  uint64_t* tfull = hempty + 2;    // a wave's accumulators are final (MMA -> epilogue)
  uint64_t* tempty = tfull + 1;    // and have been read (epilogue -> MMA)
  uint64_t* drain = tempty + 1;    // last commit of the MMA issuer
  __shared__ uint32_t tmem_base_s;
  __shared__ int abort_s;
  __shared__ bool last_s;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int G = gridDim.x;
  const int KB = (int)((a.d + kTcKB - 1) / kTcKB);
  // This CTA's tiles: bid, bid + G, ..., processed in waves of kTcWave tiles whose accumulators all
  // live in tensor memory at once, so each H block is read once per wave.  In gather mode tile t is
  // the gpt clusters gpt*t .. gpt*t + gpt - 1 of the selected-cluster list (b rows each).
  const int gpt = a.cl_list ? (int)(kTcRows / a.b) : 0;
  const int n_cl = a.cl_list ? __ldg(a.cl_count) : 0;
  // listed mode: the contiguous tiles some query takes, tile_list[0 .. *tile_count)
  const int n_list = a.cl_list ? (n_cl + gpt - 1) / gpt : (a.tile_list ? __ldg(a.tile_count) : a.n_tiles);
  const int my_tiles = n_list > (int)blockIdx.x ? (n_list - (int)blockIdx.x + G - 1) / G : 0;
  const int n_waves = (my_tiles + kTcWave - 1) / kTcWave;
  auto tile_at = [&](int j) {
    const int e = (int)blockIdx.x + j * G;
    return a.tile_list ? __ldg(a.tile_list + e) : e;
  };

  if (tid == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&hfull[i], 1);
      mbar_init(&hempty[i], 1);
    }
    mbar_init(tfull, 1);
    mbar_init(tempty, 4);
    mbar_init(drain, 1);
    abort_s = 0;
  }
  if (warp == 2) {  // all 512 columns: kTcWave accumulators of 128 lanes (queries) x 128 rows, FP32
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
                 ::"r"(smem_addr(&tmem_base_s)), "r"(512u) : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  {  // H buffers: TMA writes only the first Bpad rows; the rest must read as zeros in the MMA
    uint4* hz = reinterpret_cast<uint4*>(smem + Lay::kHOff);
    for (int i = tid; i < (int)(2 * Lay::kBlk / 16); i += kTcThreads) hz[i] = make_uint4(0u, 0u, 0u, 0u);
    fence_proxy_async_smem();
  }
  fence_mbar_init();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base_s;
  const uint32_t h_bytes = (uint32_t)((a.B + 15) / 16 * 16) * 128u;  // the H box: Bpad rows

  if (warp == 0) {
    // ---------------------------------------------------------------- TMA producer
    int it = 0, hit = 0;
    bool ok = true;
    for (int w = 0; w < n_waves && ok; ++w) {
      const int j0 = w * kTcWave, nt = min(kTcWave, my_tiles - j0);
      if (gpt) {  // the wave's cluster ids, read once by the whole warp (no load in the issue loop)
        for (int i = lane; i < nt * gpt; i += 32) {
          const int slot = tile_at(j0 + i / gpt) * gpt + i % gpt;
          wave_cl[i] = slot < n_cl ? __ldg(a.cl_list + slot) : -1;
        }
        __syncwarp();
      }
      if (lane == 0) {
        for (int kb = 0; kb < KB && ok; ++kb, ++hit) {
          const int hs = hit & 1;
          if (!tc_wait(&hempty[hs], (uint32_t)(((hit >> 1) & 1) ^ 1), &abort_s, a.status)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&hfull[hs], h_bytes);  // rows past B (up to Bpad) read as zeros
          tma_load_2d(smem + Lay::kHOff + hs * Lay::kBlk, &tmH, kb * kTcKB, 0, &hfull[hs]);
          for (int j = 0; j < nt; ++j, ++it) {
            const int s = it % S;
            if (!tc_wait(&empty[s], (uint32_t)(((it / S) & 1) ^ 1), &abort_s, a.status)) {
              ok = false;
              break;
            }
            uint8_t* dst = smem + (size_t)s * Lay::kBlk;
            const int t = tile_at(j0 + j);
            if (gpt) {  // one box of b rows per listed cluster; the rows of absent ones stay unread
              const int nc = min(gpt, n_cl - t * gpt);
              mbar_arrive_expect_tx(&full[s], (uint32_t)nc * (uint32_t)a.b * 128u);
              for (int i = 0; i < nc; ++i)
                tma_load_2d(dst + (size_t)i * a.b * 128u, &tmE, kb * kTcKB, wave_cl[j * gpt + i] * (int)a.b,
                            &full[s]);
            } else {
              mbar_arrive_expect_tx(&full[s], Lay::kBlk);
              tma_load_2d(dst, &tmE, kb * kTcKB, t * kTcRows, &full[s]);
            }
          }
        }
      }
      ok = __shfl_sync(0xFFFFFFFFu, ok, 0);
      // the next wave rewrites the cluster ids only after lane 0 issued every load of this one
      __syncwarp();
    }
    if (lane == 0) {
      // leave no copy in flight: the last loads have landed (at once when all went well)
      for (int j = max(0, it - S); j < it; ++j)
        mbar_wait(&full[j % S], (uint32_t)((j / S) & 1), nullptr, 50000000ull);
      for (int j = max(0, hit - 2); j < hit; ++j)
        mbar_wait(&hfull[j & 1], (uint32_t)((j >> 1) & 1), nullptr, 50000000ull);
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16<kTcRows>(128);  // M = 128 queries, N = 128 rows
      const uint32_t sbase = smem_addr(smem);
      int it = 0, hit = 0;
      bool ok = true, issued = false;
      for (int w = 0; w < n_waves && ok; ++w) {
        const int nt = min(kTcWave, my_tiles - w * kTcWave);
        if (!tc_wait(tempty, (uint32_t)((w & 1) ^ 1), &abort_s, a.status)) break;
        tc_fence_after();
        for (int kb = 0; kb < KB && ok; ++kb, ++hit) {
          const int hs = hit & 1;
          if (!tc_wait(&hfull[hs], (uint32_t)((hit >> 1) & 1), &abort_s, a.status)) {
            ok = false;
            break;
          }
          const uint32_t ha = sbase + Lay::kHOff + (uint32_t)hs * Lay::kBlk;
          for (int j = 0; j < nt; ++j, ++it) {
            const int s = it % S;
            if (!tc_wait(&full[s], (uint32_t)((it / S) & 1), &abort_s, a.status)) {
              ok = false;
              break;
            }
            // (TMA writes and MMA reads are both async-proxy operations ordered by the barrier)
            const uint32_t ea = sbase + (uint32_t)s * Lay::kBlk;
            const uint32_t d_tmem = tmem + (uint32_t)(j * kTcRows);
#pragma unroll
            for (int k = 0; k < kTcKB / 16; ++k)  // 16 BF16 = 32 bytes along K per instruction
              mma_bf16(d_tmem, sw128_desc(ha + 32u * k), sw128_desc(ea + 32u * k), idesc,
                       (uint32_t)((kb | k) != 0));
            mma_commit(&empty[s]);  // the E stage is free once these MMAs have read it
            issued = true;
          }
          if (ok) mma_commit(&hempty[hs]);
        }
        if (ok) mma_commit(tfull);
      }
      if (issued) {  // every MMA has completed before the tensor memory is freed
        mma_commit(drain);
        mbar_wait(drain, 0u, nullptr, 50000000ull);
      }
    }
  } else if (warp >= 4) {
    // ---------------------------------------------------------------- epilogue: one query per thread
    const int et = tid - 128;             // 0..127: this thread's query and its tile-row duty
    const int q = et;                     // lane q of tensor memory (warp quarter = warp % 4)
    const bool q_live = q < a.B;          // lanes past the batch take no row but join every warp step
    uint32_t bk = 0u, bt = 0xFFFFFFFFu;   // best key image and its token
    auto group_sync = [] { asm volatile("bar.sync 1, 128;" ::: "memory"); };
    for (int w = 0; w < n_waves; ++w) {
      const int j0 = w * kTcWave, nt = min(kTcWave, my_tiles - j0);
      if (!tc_wait(tfull, (uint32_t)(w & 1), &abort_s, a.status)) break;
      tc_fence_after();
      for (int j = 0; j < nt; ++j) {
        const int t = tile_at(j0 + j);
        {  // the tile's rows: token and query mask (0: no query takes the row, or no row)
          const int r = et;
          int64_t row, cl;
          bool valid;
          if (a.cl_list) {
            const int slot = t * gpt + r / (int)a.b;
            valid = slot < n_cl;
            cl = valid ? __ldg(a.cl_list + slot) : 0;
            row = cl * a.b + r % (int)a.b;
          } else {
            row = (int64_t)t * kTcRows + r;
            valid = row < a.rows;
            cl = a.qmask ? row / a.b : 0;
          }
          tok_s[r] = valid ? (a.row_tok ? (uint32_t)__ldg(a.row_tok + row) : (uint32_t)row) : 0u;
          msk_s[r] = valid ? (a.qmask ? __ldg(a.qmask + cl) : ~0ull) : 0ull;
        }
        group_sync();
        const uint32_t tbase = tmem + ((uint32_t)(32 * (warp & 3)) << 16) + (uint32_t)(j * kTcRows);
        const int64_t row0 = (int64_t)t * kTcRows;  // contiguous mode: first row of the tile
        for (int c0 = 0; c0 < kTcRows; c0 += 32) {
          uint32_t v[32];
          tmem_ld16(tbase + (uint32_t)c0, *reinterpret_cast<uint32_t(*)[16]>(v));
          tmem_ld16(tbase + (uint32_t)c0 + 16u, *reinterpret_cast<uint32_t(*)[16]>(v + 16));
          tmem_ld_wait();
          if constexpr (KEYS) {  // Stage-1 keys (contiguous rows): s[q][row] or s/τ + G(q, stream 0, row)
#pragma unroll
            for (int i = 0; i < 32; ++i) {
              const int64_t row = row0 + c0 + i;
              if (q < a.B && row < a.rows) {
                const float z = __uint_as_float(v[i]);
                a.out_keys[(int64_t)q * a.rows + row] =
                    SAMPLE ? z / a.tau + gumbel_from_u32(philox_word(a.seed, a.step, (uint32_t)q, 0u, (uint32_t)row)) : z;
              }
            }
            continue;
          }
          if constexpr (!SAMPLE) {
            if (!q_live) continue;  // (uniform per warp when B is a multiple of 32)
          }
          float* gum = nullptr;
          if constexpr (SAMPLE) {
            // The Gumbel terms G(q, 1, token) of the (row, query) pairs this warp takes in the chunk,
            // spread evenly over the lanes: a row is taken by few of the warp's 32 queries, so one
            // evaluation per row and lane would leave most lanes idle.  Lane i lists row i's takers
            // (a ballot), a scan gives each row its first pair, and pair k goes to lane k % 32.
            uint32_t* bal_s = reinterpret_cast<uint32_t*>(smem + Lay::kPairOff) + (warp & 3) * 64;
            gum = reinterpret_cast<float*>(smem + Lay::kGumOff) + (warp & 3) * 1024;
            uint32_t my_bal = 0u;
#pragma unroll
            for (int i = 0; i < 32; ++i) {
              const uint32_t bi = __ballot_sync(0xFFFFFFFFu, q_live && ((msk_s[c0 + i] >> q) & 1ull));
              if (lane == i) my_bal = bi;
            }
            const uint32_t my_cnt = __popc(my_bal);
            uint32_t incl = my_cnt;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
              const uint32_t y = __shfl_up_sync(0xFFFFFFFFu, incl, o);
              if (lane >= o) incl += y;
            }
            bal_s[lane] = my_bal;
            bal_s[32 + lane] = incl - my_cnt;  // the row's first pair
            const uint32_t pairs = __shfl_sync(0xFFFFFFFFu, incl, 31);
            __syncwarp();
            for (uint32_t k = (uint32_t)lane; k < pairs; k += 32u) {
              int i = 0;  // the last row whose first pair is <= k
#pragma unroll
              for (int step = 16; step > 0; step >>= 1)
                if (i + step < 32 && bal_s[32 + i + step] <= k) i += step;
              const uint32_t ql = __fns(bal_s[i], 0u, (int)(k - bal_s[32 + i]) + 1);
              const uint32_t qq = (uint32_t)(32 * (warp & 3)) + ql;
              gum[i * 32 + (int)ql] = gumbel_from_u32(philox_word(a.seed, a.step, qq, 1u, tok_s[c0 + i]));
            }
            __syncwarp();
          }
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            const unsigned long long mk = msk_s[c0 + i];
            if (!q_live || !((mk >> q) & 1ull)) continue;
            const uint32_t tk = tok_s[c0 + i];
            const float z = __uint_as_float(v[i]);
            if (a.out_logits) a.out_logits[(int64_t)q * a.rows + tk] = z;
            float val = z;
            if constexpr (SAMPLE) val = z / a.tau + gum[i * 32 + lane];
            const uint32_t key = float_key(val);
            if (key > bk || (key == bk && tk < bt)) {
              bk = key;
              bt = tk;
            }
          }
          if constexpr (SAMPLE) __syncwarp();  // the warp's G buffer is rewritten for the next chunk
        }
        group_sync();  // the tile rows are rewritten for the next tile
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(tempty);  // the next wave may overwrite the accumulators
    }
    if (!KEYS && q < a.B && bk) atomicMax(a.best + q, ((unsigned long long)bk << 32) | (unsigned long long)(~bt));
  }

  // ------------------------------------------------------------------ teardown and the grid arg-max
  tc_fence_before();
  __syncthreads();
  if (warp == 2) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(512u) : "memory");
  }
  if constexpr (KEYS) return;  // Stage-1 keys: nothing to reduce
  __threadfence();
  __syncthreads();
  if (tid == 0) {
    const unsigned long long tk = atomicAdd(a.ticket, 1ull);
    last_s = tk + 1ull == (unsigned long long)G;
  }
  __syncthreads();
  if (last_s) {  // every other CTA has added its maxima: publish, and leave zeros for the next call
    __threadfence();
    if (tid < a.B) {
      const unsigned long long fin = atomicExch(a.best + tid, 0ull);
      if (a.out_tok) a.out_tok[tid] = fin ? (int32_t)best_id(fin) : -1;
    }
    if (tid == 0) atomicExch(a.ticket, 0ull);
  }
}

// The 128-row tiles of which some query takes a cluster, in ascending order; one block.
__global__ void __launch_bounds__(1024) k_selected_tiles(const unsigned long long* __restrict__ qmask,
                                                         int64_t rows, int64_t b, int n_tiles,
                                                         int32_t* list, int32_t* count) {
  __shared__ int base_s;
  __shared__ int wsum[32];
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  if (threadIdx.x == 0) base_s = 0;
  __syncthreads();
  for (int t0 = 0; t0 < n_tiles; t0 += blockDim.x) {
    const int t = t0 + (int)threadIdx.x;
    bool act = false;
    if (t < n_tiles) {
      const int64_t r0 = (int64_t)t * kTcRows, r1 = min(r0 + kTcRows, rows) - 1;
      for (int64_t cl = r0 / b; cl <= r1 / b && !act; ++cl) act = qmask[cl] != 0ull;
    }
    const unsigned bal = __ballot_sync(0xFFFFFFFFu, act);
    if (lane == 0) wsum[wid] = __popc(bal);
    __syncthreads();
    int before = 0, total = 0;
    for (int i = 0; i < (int)(blockDim.x >> 5); ++i) {
      before += i < wid ? wsum[i] : 0;
      total += wsum[i];
    }
    if (act) list[base_s + before + __popc(bal & ((1u << lane) - 1u))] = t;
    __syncthreads();
    if (threadIdx.x == 0) base_s += total;
    __syncthreads();
  }
  if (threadIdx.x == 0) *count = base_s;
}

// The clusters some query takes (nonzero mask), in ascending order; one block.
__global__ void __launch_bounds__(1024) k_selected_clusters(const unsigned long long* __restrict__ qmask,
                                                            int64_t c, int32_t* list, int32_t* count) {
  __shared__ int base_s;
  __shared__ int wsum[32];
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  if (threadIdx.x == 0) base_s = 0;
  __syncthreads();
  for (int64_t k0 = 0; k0 < c; k0 += blockDim.x) {
    const int64_t k = k0 + threadIdx.x;
    const bool act = k < c && qmask[k] != 0ull;
    const unsigned bal = __ballot_sync(0xFFFFFFFFu, act);
    if (lane == 0) wsum[wid] = __popc(bal);
    __syncthreads();
    int before = 0, total = 0;
    for (int i = 0; i < (int)(blockDim.x >> 5); ++i) {
      before += i < wid ? wsum[i] : 0;
      total += wsum[i];
    }
    if (act) list[base_s + before + __popc(bal & ((1u << lane) - 1u))] = (int32_t)k;
    __syncthreads();
    if (threadIdx.x == 0) base_s += total;
    __syncthreads();
  }
  if (threadIdx.x == 0) *count = base_s;
}

// ------------------------------------------------------------------ host side

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q = cudaDriverEntryPointSymbolNotFound;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// 2-D BF16 map over `rows` rows of `d` elements (row stride d*2 bytes), boxes of 64 x box_rows,
// 128-byte swizzle; rows past the end read as zeros.
bool make_map(CUtensorMap* m, const void* base, int64_t d, int64_t rows, uint32_t box_rows) {
  PFN_cuTensorMapEncodeTiled_v12000 fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {(cuuint64_t)d, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)d * 2u};
  cuuint32_t box[2] = {(cuuint32_t)kTcKB, box_rows};
  cuuint32_t estr[2] = {1u, 1u};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

cudaError_t launch_kernel(const CUtensorMap& mE, const CUtensorMap& mH, const TcParams& p, int num_sms,
                          cudaStream_t st) {
  constexpr int S = (int)((kTcSmemBudget - 2u * 16384u - 4096u) / 16384u);
  const bool keys = p.out_keys != nullptr, sample = p.sample != 0;
  auto kern = keys ? (sample ? k_tc_head<S, true, true> : k_tc_head<S, true, false>)
                   : (sample ? k_tc_head<S, false, true> : k_tc_head<S, false, false>);
  const uint32_t dyn = sample ? TcLayout<S, true>::kDyn : TcLayout<S, false>::kDyn;
  cudaError_t e = set_smem_attr(reinterpret_cast<const void*>(kern), dyn);
  if (e != cudaSuccess) return e;
  // every SM when the tiles are listed on the device; otherwise no more CTAs than tiles
  const int grid = (p.cl_list || p.tile_list || p.n_tiles >= num_sms) ? num_sms : p.n_tiles;
  kern<<<grid, kTcThreads, dyn, st>>>(mE, mH, p);
  return cudaGetLastError();
}

}  // namespace

bool tc_supported(int elem, int64_t d, int B) {
  return elem == kBF16 && d % 8 == 0 && B >= 1 && B <= 64 && encode_fn() != nullptr;
}

cudaError_t launch_tc_head(const void* A, const void* H, TcParams p, int num_sms, cudaStream_t st) {
  if (p.B < 1 || p.B > 64 || p.rows < 1 || (p.qmask && p.b < 1)) return cudaErrorInvalidValue;
  if (p.out_keys && (p.qmask || p.cl_list)) return cudaErrorInvalidValue;
  p.n_tiles = (int)((p.rows + kTcRows - 1) / kTcRows);
  uint32_t box = kTcRows;
  if (p.tile_list) {  // the selected tiles, listed on the device (the kernel reads their count)
    if (!p.qmask || p.cl_list) return cudaErrorInvalidValue;
    k_selected_tiles<<<1, 1024, 0, st>>>(p.qmask, p.rows, p.b, p.n_tiles, p.tile_list, p.tile_count);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  if (p.cl_list) {  // the selected clusters, listed on the device (the kernel reads their count)
    if (p.b < 8 || kTcRows % p.b != 0) return cudaErrorInvalidValue;  // whole 8-row swizzle atoms per box
    k_selected_clusters<<<1, 1024, 0, st>>>(p.qmask, p.rows / p.b, p.cl_list, p.cl_count);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    box = (uint32_t)p.b;
  }
  CUtensorMap mE, mH;
  if (!make_map(&mE, A, p.d, p.rows, box) || !make_map(&mH, H, p.d, p.B, (uint32_t)((p.B + 15) / 16 * 16)))
    return cudaErrorInvalidValue;
  return launch_kernel(mE, mH, p, num_sms, st);
}

}  // namespace fh

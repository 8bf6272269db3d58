// fh_tc.cu — tensor-core logits for a batch of queries: Z = A · Hᵀ over 128-row tiles of A with
// tcgen05.mma (BF16 in, FP32 accumulators in tensor memory), the per-query candidate mask and the
// token decision fused into the epilogue.
//
// Used where the head is a dense contraction: the batched dense head (A = E, every row a candidate)
// and batched FlashHead Stage 2 (A = the cluster-major copy of E; a row takes part for query q when
// q's probe set holds the row's cluster — FlashHead notes, Module 1 and Figure 1, and Eq. 2/3 for the
// decision) at large batches.  Stage 2 lists the 128-row tiles that hold a cluster some query
// selected and streams them, so every needed row is read once for all queries; the epilogue masks
// each (row, query) pair by whether the query selected the row's cluster.  Stage-1 keys (A = C, or
// the INT4 centroids dequantised in shared memory) use the same pipeline.
//
// One persistent CTA per SM, 8 warps with fixed roles:
//   warp 0      TMA producer: per stage one K-block (64 columns) of H (Bpad rows) and of each A tile
//               of the current wave (128 or 64 rows), 128-byte swizzled;
//   warp 1      MMA issuer: four 128 x R x 16 tcgen05.mma per tile and stage into the wave's half of
//               tensor memory;
//   warp 2      allocates and frees the tensor memory (two halves of 256 columns);
//   warps 4..7  epilogue: thread q reads TMEM lane q (query q) of the finished wave, applies the mask
//               (and the Gumbel term when sampling), and reduces the query's arg-max.
// The two halves let the epilogue of one wave overlap the MMAs of the next.  Every wait is bounded:
// on a timeout the CTA records it, drains its own copies and MMAs, frees TMEM and leaves.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <cuda_fp16.h>

#include <mutex>  // std::call_once

#include "fh_device.cuh"
#include "fh_kernels.cuh"
#include "fh_stream.cuh"

namespace fh {
namespace {

constexpr int kTcKB = 64;          // K elements per stage: one 128-byte swizzle atom per row
constexpr int kTcThreads = 256;
// The tensor-core head: warps 0-3 (TMA producer, MMA issuer, tensor-memory owner, spare) and eight
// epilogue warps, two on each quarter of the tensor-memory lanes, reading 16-row chunks.
constexpr int kTcEpiWarps = 8;
constexpr int kTcHeadThreads = 128 + 32 * kTcEpiWarps;
constexpr int kTcChunk = 16;
// K-blocks per pipeline stage: a stage then fetches a row's consecutive K-blocks together (the keys'
// 64-row tiles fetched 128 bytes of each row per stage: 20.5 µs for the Llama-shaped keys at one
// K-block per stage, 15.3 at two, 12.0 at four, no better at eight; the head modes' 128-row tiles
// gain ~3 % at two); fewer when two stages would not fit.
#ifndef FH_TC_KEYS_KBS
#define FH_TC_KEYS_KBS 4
#endif
#ifndef FH_TC_HEAD_KBS
#define FH_TC_HEAD_KBS 2
#endif

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
// D = H · E_tileᵀ: the MMA's M side is the queries (H padded to 128 rows), its N side the rows of an
// E tile (128; 64 for Stage-1 keys when that gives every SM a tile), so tensor-memory lane q holds
// query q and column r row r of the tile.  Each epilogue thread owns one query and reduces its
// arg-max along its own columns: no cross-lane work.
//
// Tiles go in waves of up to kTcWave whose accumulators fill one half of the 512 TMEM columns, so
// the epilogue of one wave overlaps the MMAs of the next.  A pipeline stage holds one K-block of H
// and the same K-block of every tile of the wave under one barrier pair, so the K-blocks in flight
// are bounded by the number of stages alone.  A stage's H block holds only the Bpad = ⌈B/16⌉·16
// rows the copy writes: the MMA's rows past Bpad read whatever follows in shared memory (inside the
// allocation, see tc_layout) and only produce accumulator lanes no thread reads.

constexpr int kTcRows = 128;                 // E rows per tile in the head modes
constexpr int kTcWave = 2;                   // tiles per wave (2 x 128 accumulator columns)
constexpr int kTcMaxStages = 16;
constexpr uint32_t kTcSmemMax = 226u * 1024u;

// Dynamic shared memory of the kernel: `stages` stages of (H block, E blocks of the wave), the tile
// rows (token, mask), the sampling scratch, the barriers.
struct TcLay {
  uint32_t h_bytes, e_bytes, sub_bytes, stage_bytes;  // one K-block: H, one E tile, H + the wave; a stage
  uint32_t row_off, gum_off, bar_off, dyn;
};
// Where the epilogue bounds the kernel, the queries fill the MMA's 128 rows: qrows = 32 or 64 rows
// (the batch, zero-padded) repeated copies = 128 / qrows times, so that every epilogue warp's
// tensor-memory lanes hold live queries (lane l: query l % qrows) and the warps holding copies of the
// same queries split a tile's rows between them.  Otherwise one copy of the batch padded to 16 rows
// (the MMA's rows past it read whatever follows in shared memory; their lanes are never read).
__host__ __device__ inline void tc_query_layout(int B, bool copies, int& qrows, int& ncopies) {
  qrows = copies ? (B <= 32 ? 32 : 64) : (B + 15) / 16 * 16;
  ncopies = copies ? 128 / qrows : 1;
}

// A stage holds kbs consecutive K-blocks, each laid out as [H][E tile 0][E tile 1 ...].
__host__ __device__ inline TcLay tc_layout(int qrows, int copies, int tile_rows, int wave, bool sample,
                                           int stages, int kbs) {
  TcLay L;
  L.h_bytes = (uint32_t)(qrows * copies) * 128u;  // multiple of 2048: E blocks stay 1024-aligned
  L.e_bytes = (uint32_t)tile_rows * 128u;
  L.sub_bytes = L.h_bytes + (uint32_t)wave * L.e_bytes;
  L.stage_bytes = (uint32_t)kbs * L.sub_bytes;
  L.row_off = (uint32_t)stages * L.stage_bytes;
  L.gum_off = L.row_off + (uint32_t)kTcRows * 12u;
  L.bar_off = L.gum_off + (sample ? (uint32_t)kTcEpiWarps * kTcChunk * 32u * 4u : 0u);  // G[row][lane] a warp
  const uint32_t end = L.bar_off + (uint32_t)(2 * kTcMaxStages + 8) * 8u;
  // the last K-block's H operand is read as 128 rows of 128 B
  const uint32_t h_end = (uint32_t)(stages > 0 ? stages - 1 : 0) * L.stage_bytes +
                         (uint32_t)(kbs - 1) * L.sub_bytes + 128u * 128u;
  L.dyn = (end > h_end ? end : h_end) + 1024u;  // + alignment slack
  return L;
}

// KEYS: write the products (Stage-1 keys) instead of reducing an arg-max; SAMPLE: add the Gumbel
// term.  Separate instantiations keep each epilogue's code out of the other modes' instruction stream.
template <bool KEYS, bool SAMPLE>
__global__ void __launch_bounds__(kTcHeadThreads, 1)
    k_tc_head(const __grid_constant__ CUtensorMap tmE, const __grid_constant__ CUtensorMap tmH,
              const TcParams a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023u) & ~uintptr_t(1023));
  constexpr int WT = KEYS ? 1 : kTcWave;
  const int R = a.tile_rows, S = a.stages;
  const int Bq = a.qrows, D = a.copies;  // query rows of one copy, copies
  const int KBS = a.kbs;                  // K-blocks per stage
  const TcLay Lay = tc_layout(Bq, D, R, WT, SAMPLE, S, KBS);
  uint32_t* tok_s = reinterpret_cast<uint32_t*>(smem + Lay.row_off);                     // 128
  unsigned long long* msk_s = reinterpret_cast<unsigned long long*>(smem + Lay.row_off + 512u);  // 128
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + Lay.bar_off);
  uint64_t* empty = full + kTcMaxStages;
  uint64_t* tfull = empty + kTcMaxStages;  // [2] a wave's accumulators are final (MMA -> epilogue)
  uint64_t* tempty = tfull + 2;            // [2] and have been read (epilogue -> MMA)
  uint64_t* drain = tempty + 2;            // last commit of the MMA issuer
  __shared__ uint32_t tmem_base_s;
  __shared__ int abort_s;
  __shared__ bool last_s;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int G = gridDim.x;
  const int KB = (int)((a.d + kTcKB - 1) / kTcKB);
  const int NG = (KB + KBS - 1) / KBS;  // stages a wave takes
  // This CTA's tiles: bid, bid + G, ... of every tile, or in listed mode of the contiguous tiles some
  // query takes, tile_list[0 .. *tile_count)
  const int n_list = a.tile_list ? __ldg(a.tile_count) : a.n_tiles;
  const int my_tiles = n_list > (int)blockIdx.x ? (n_list - (int)blockIdx.x + G - 1) / G : 0;
  const int n_waves = (my_tiles + WT - 1) / WT;
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
      mbar_init(&tfull[i], 1);
      mbar_init(&tempty[i], kTcEpiWarps);
    }
    mbar_init(drain, 1);
    abort_s = 0;
  }
  if (warp == 2) {  // all 512 columns: two halves of kTcWave accumulators (128 lanes x R rows, FP32)
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
                 ::"r"(smem_addr(&tmem_base_s)), "r"(512u) : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  fence_mbar_init();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base_s;

  if (warp == 0) {
    // ---------------------------------------------------------------- TMA producer
    int it = 0;
    bool ok = true;
    for (int w = 0; w < n_waves && ok; ++w) {
      const int j0 = w * WT, nt = min(WT, my_tiles - j0);
      if (lane == 0) {
        // the wave's E tiles go out before the query rows (the bytes that come from HBM first)
        static_assert(kTcWave == 2, "two tiles a wave");
        const int y0 = tile_at(j0) * R, y1 = nt > 1 ? tile_at(j0 + 1) * R : y0;
        const uint32_t kb_bytes = Lay.h_bytes + (uint32_t)nt * Lay.e_bytes;  // H rows past B read as zeros
        for (int g = 0; g < NG; ++g, ++it) {
          const int s = it % S;
          if (!tc_wait(&empty[s], (uint32_t)(((it / S) & 1) ^ 1), &abort_s, a.status)) {
            ok = false;
            break;
          }
          const int kb0 = g * KBS, kbn = min(KBS, KB - kb0);
          uint8_t* stg = smem + (size_t)s * Lay.stage_bytes;
          mbar_arrive_expect_tx(&full[s], (uint32_t)kbn * kb_bytes);
          for (int kk = 0; kk < kbn; ++kk) {  // a row's consecutive K-blocks go out together
            uint8_t* sub = stg + (size_t)kk * Lay.sub_bytes;
            tma_load_2d(sub + Lay.h_bytes, &tmE, (kb0 + kk) * kTcKB, y0, &full[s]);
            if (nt > 1) tma_load_2d(sub + Lay.h_bytes + Lay.e_bytes, &tmE, (kb0 + kk) * kTcKB, y1, &full[s]);
          }
          for (int kk = 0; kk < kbn; ++kk)
            for (int r = 0; r < D; ++r)
              tma_load_2d(stg + (size_t)kk * Lay.sub_bytes + (size_t)r * Bq * 128u, &tmH, (kb0 + kk) * kTcKB,
                          0, &full[s]);
        }
      }
      ok = __shfl_sync(0xFFFFFFFFu, ok, 0);
    }
    if (lane == 0) {
      // leave no copy in flight: the last loads have landed (at once when all went well)
      for (int j = max(0, it - S); j < it; ++j)
        mbar_wait(&full[j % S], (uint32_t)((j / S) & 1), nullptr, 50000000ull);
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      // kind::f16, FP32 accumulator, BF16 A and B, both K-major, M = 128 queries, N = R rows
      const uint32_t idesc = (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(R >> 3) << 17) | ((uint32_t)(128 >> 4) << 24);
      const uint32_t sbase = smem_addr(smem);
      int it = 0;
      bool ok = true, issued = false;
      for (int w = 0; w < n_waves && ok; ++w) {
        const int nt = min(WT, my_tiles - w * WT), acc = w & 1;
        if (!tc_wait(&tempty[acc], (uint32_t)(((w >> 1) & 1) ^ 1), &abort_s, a.status)) break;
        tc_fence_after();
        for (int g = 0; g < NG; ++g, ++it) {
          const int s = it % S;
          if (!tc_wait(&full[s], (uint32_t)((it / S) & 1), &abort_s, a.status)) {
            ok = false;
            break;
          }
          tc_fence_after();
          // (TMA writes and MMA reads are both async-proxy operations ordered by the barrier)
          const int kb0 = g * KBS, kbn = min(KBS, KB - kb0);
          for (int kk = 0; kk < kbn; ++kk) {
            const int kb = kb0 + kk;
            const uint32_t ha = sbase + (uint32_t)s * Lay.stage_bytes + (uint32_t)kk * Lay.sub_bytes;
            for (int j = 0; j < nt; ++j) {
              const uint32_t ea = ha + Lay.h_bytes + (uint32_t)j * Lay.e_bytes;
              const uint32_t d_tmem = tmem + (uint32_t)(acc * 256 + j * R);
#pragma unroll
              for (int k = 0; k < kTcKB / 16; ++k)  // 16 BF16 = 32 bytes along K per instruction
                mma_bf16(d_tmem, sw128_desc(ha + 32u * k), sw128_desc(ea + 32u * k), idesc,
                         (uint32_t)((kb | k) != 0));
            }
          }
          mma_commit(&empty[s]);  // the stage is free once these MMAs have read it
          issued = true;
        }
        if (ok) mma_commit(&tfull[acc]);
      }
      if (issued) {  // every MMA has completed before the tensor memory is freed
        mma_commit(drain);
        mbar_wait(drain, 0u, nullptr, 50000000ull);
      }
    }
  } else if (warp >= 4) {
    // ---------------------------------------------------------------- epilogue
    // Thread et reads lane el = et % 128 of tensor memory (its warp's quarter), which holds query
    // q = el % (128 / D) of copy el / (128 / D); with its half h = et / 128 that names one of 2·D slots,
    // and the 16-row chunks of a tile go round robin over the slots.
    const int et = tid - 128;                    // 0 .. 32·kTcEpiWarps - 1
    const int el = et & 127;                     // its lane of tensor memory
    const int qmod = 128 / D;                    // lanes per copy of the queries
    const int q = el & (qmod - 1);               // its query
    const int slot = el / qmod + D * (et >> 7);  // its chunks: slot, slot + 2·D, ...
    const bool q_live = q < a.B;                 // lanes past the batch take no row but join every warp step
    uint32_t bk = 0u, bt = 0xFFFFFFFFu;          // best key image and its token
    auto group_sync = [] { asm volatile("bar.sync 1, %0;" ::"n"(32 * kTcEpiWarps) : "memory"); };
    // A tile's rows: token and query mask (0: no query takes the row, or no row), staged by the first
    // 128 threads.  The next tile's are loaded into registers while the current tile is reduced.
    uint32_t tok_n = 0u;
    unsigned long long msk_n = 0ull;
    auto load_rows = [&](int jj) {
      const int64_t row = (int64_t)tile_at(jj) * kTcRows + et;
      const bool valid = row < a.rows;
      const int64_t cl = a.qmask ? row / a.b : 0;
      tok_n = valid ? (a.row_tok ? (uint32_t)__ldg(a.row_tok + row) : (uint32_t)row) : 0u;
      msk_n = valid ? (a.qmask ? __ldg(a.qmask + cl) : ~0ull) : 0ull;
    };
    if (!KEYS && my_tiles > 0 && et < 128) load_rows(0);
    for (int w = 0; w < n_waves; ++w) {
      const int j0 = w * WT, nt = min(WT, my_tiles - j0), acc = w & 1;
      if (!tc_wait(&tfull[acc], (uint32_t)((w >> 1) & 1), &abort_s, a.status)) break;
      tc_fence_after();
      for (int j = 0; j < nt; ++j) {
        const int t = tile_at(j0 + j);
        if constexpr (!KEYS) {
          if (et < 128) {
            tok_s[et] = tok_n;
            msk_s[et] = msk_n;
          }
          group_sync();
          if (et < 128 && j0 + j + 1 < my_tiles) load_rows(j0 + j + 1);
        }
        const uint32_t tbase = tmem + ((uint32_t)(32 * (warp & 3)) << 16) + (uint32_t)(acc * 256 + j * R);
        const int64_t row0 = (int64_t)t * R;  // contiguous mode: first row of the tile
        for (int c0 = kTcChunk * slot; c0 < R; c0 += kTcChunk * 2 * D) {
          uint32_t v[kTcChunk];
          tmem_ld16(tbase + (uint32_t)c0, v);
          tmem_ld_wait();
          if constexpr (KEYS) {  // Stage-1 keys (contiguous rows): s[q][row] or s/τ + G(q, stream 0, row)
            if (q < a.B) {
#pragma unroll
              for (int i = 0; i < kTcChunk; ++i) {
                const int64_t row = row0 + c0 + i;
                if (row < a.rows) {
                  const float z = __uint_as_float(v[i]);
                  a.out_keys[(int64_t)q * a.rows + row] =
                      SAMPLE ? z / a.tau + gumbel_from_u32(philox_word(a.seed, a.step, (uint32_t)q, 0u, (uint32_t)row)) : z;
                }
              }
            }
            continue;
          }
          // the chunk's rows this thread's query takes (bit i: row c0 + i), from the rows' query masks
          uint32_t tm = 0u;
#pragma unroll
          for (int i = 0; i < kTcChunk; ++i) tm |= (uint32_t)((msk_s[c0 + i] >> q) & 1ull) << i;
          if (!q_live) tm = 0u;
          if (__ballot_sync(0xFFFFFFFFu, tm != 0u) == 0u) continue;  // no lane takes a row of the chunk
          float* gum = nullptr;
          if constexpr (SAMPLE) {
            // the Gumbel terms G(q, 1, token) of the rows this thread takes, two at a time (two
            // independent Philox chains), in the warp's buffer at [row][lane]
            gum = reinterpret_cast<float*>(smem + Lay.gum_off) + (warp - 4) * (kTcChunk * 32);
            for (uint32_t rest = tm; rest != 0u;) {
              const int ia = __ffs(rest) - 1;
              rest &= rest - 1u;
              const int ib = rest ? __ffs(rest) - 1 : ia;
              if (rest) rest &= rest - 1u;
              const uint32_t wa = philox_word(a.seed, a.step, (uint32_t)q, 1u, tok_s[c0 + ia]);
              const uint32_t wb = philox_word(a.seed, a.step, (uint32_t)q, 1u, tok_s[c0 + ib]);
              gum[ia * 32 + lane] = gumbel_from_u32(wa);
              gum[ib * 32 + lane] = gumbel_from_u32(wb);
            }
          }
          // the decision over the chunk, branch-free: every row's loads are independent of the others'
#pragma unroll
          for (int i = 0; i < kTcChunk; ++i) {
            const bool take = (tm >> i) & 1u;
            const uint32_t tk = tok_s[c0 + i];
            const float z = __uint_as_float(v[i]);
            if (a.out_logits && take) a.out_logits[(int64_t)q * a.rows + tk] = z;
            float val = z;
            if constexpr (SAMPLE) val = z / a.tau + (take ? gum[i * 32 + lane] : 0.0f);
            const uint32_t key = float_key(val);
            const bool better = take && (key > bk || (key == bk && tk < bt));
            bk = better ? key : bk;
            bt = better ? tk : bt;
          }
        }
        if constexpr (!KEYS) group_sync();  // the tile rows are rewritten for the next tile
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&tempty[acc]);  // the MMAs may overwrite these accumulators
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

cudaError_t launch_kernel(const CUtensorMap& mE, const CUtensorMap& mH, TcParams p, int num_sms,
                          cudaStream_t st) {
  const bool keys = p.out_keys != nullptr, sample = p.sample != 0;
  const int wave = keys ? 1 : kTcWave;
  int S = 0;
  for (;;) {  // the most stages that fit at this many K-blocks a stage; fewer K-blocks if not two
    for (S = kTcMaxStages; S >= 2; --S)
      if (tc_layout(p.qrows, p.copies, p.tile_rows, wave, sample, S, p.kbs).dyn <= kTcSmemMax) break;
    if (S >= 2 || p.kbs <= 1) break;
    p.kbs /= 2;
  }
  if (S < 2) return cudaErrorInvalidValue;
  p.stages = S;
  auto kern = keys ? (sample ? k_tc_head<true, true> : k_tc_head<true, false>)
                   : (sample ? k_tc_head<false, true> : k_tc_head<false, false>);
  const uint32_t dyn = tc_layout(p.qrows, p.copies, p.tile_rows, wave, sample, S, p.kbs).dyn;
  cudaError_t e = set_smem_attr(reinterpret_cast<const void*>(kern), dyn);
  if (e != cudaSuccess) return e;
  // every SM when the tiles are listed on the device; otherwise no more CTAs than tiles
  const int grid = (p.tile_list || p.n_tiles >= num_sms) ? num_sms : p.n_tiles;
  kern<<<grid, kTcHeadThreads, dyn, st>>>(mE, mH, p);
  return cudaGetLastError();
}

// ------------------------------------------------------------------ INT4 Stage-1 keys
//
// Stage-1 keys from INT4 centroids (FlashHead notes, Module 3) for a batch of queries: the MMA's B
// operand (128 centroid rows per tile) is dequantised in shared memory — q·scale for the 4-bit q and
// the row's BF16 group scale, which is exact in fp16 (at most 11 significant bits) — and the queries
// are converted from BF16 to fp16 in place (exact for |h_j| in [2^-17, 65504]); kind::f16 MMAs with fp16
// operands and FP32 accumulators then give the keys.  One tile of 128 centroid rows per CTA pass.
// Warp roles: warp 0 loads (TMA: the query block of each K-block, the 32-byte nibble rows of the
// tile; one bulk copy for the tile's scales), warp 1 issues the MMAs, warp 2 owns 128 TMEM columns,
// warps 4..7 dequantise (thread t: row t of the tile) and finally read the accumulators (thread t:
// query t) and write the keys.

constexpr int kI4Stages = 4;
constexpr uint32_t kI4Blk = 128u * 128u;   // one K-block of fp16 operand: 128 rows x 128 B
constexpr uint32_t kI4Nib = 128u * 32u;    // one K-block of nibbles: 128 rows x 32 B

struct I4Layout {
  static constexpr uint32_t kH = 0;                                  // S query blocks (SW128)
  static constexpr uint32_t kOp = kH + kI4Stages * kI4Blk;           // S dequantised blocks (SW128)
  static constexpr uint32_t kNib = kOp + kI4Stages * kI4Blk;         // S nibble blocks
  static constexpr uint32_t kSc = kNib + kI4Stages * kI4Nib;         // the tile's scales
};

struct TcInt4Params {
  int64_t rows, d;            // c centroid rows of d columns
  int B;
  int sample;
  float tau;
  uint64_t seed, step;
  const uint16_t* scales;     // rows x d/32 BF16
  float* out_keys;            // B x rows
  uint32_t* status;
  uint32_t* tickets_to_clear;  // reset to 0 by block 0 for the kernels that follow
  int n_tickets;
  int n_tiles;
};

__device__ __forceinline__ uint16_t f32_to_f16_bits(float x) {
  return __half_as_ushort(__float2half_rn(x));
}

// BF16 -> fp16 for the 8 values of a 16-byte chunk (rounds to nearest when not exact).
__device__ __forceinline__ uint4 bf16x8_to_f16x8(uint4 v) {
  uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int i = 0; i < 4; ++i)
    w[i] = (uint32_t)f32_to_f16_bits(bf16_lo(w[i])) | ((uint32_t)f32_to_f16_bits(bf16_hi(w[i])) << 16);
  return make_uint4(w[0], w[1], w[2], w[3]);
}

template <bool SAMPLE>
__global__ void __launch_bounds__(kTcThreads, 1)
    k_tc_keys_int4(const __grid_constant__ CUtensorMap tmH, const __grid_constant__ CUtensorMap tmQ,
                   const TcInt4Params a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023u) & ~uintptr_t(1023));
  __shared__ uint64_t full_in[kI4Stages], dq_full[kI4Stages], op_empty[kI4Stages];
  __shared__ uint64_t sc_full, tfull, tempty, drain;
  __shared__ uint32_t tmem_base_s;
  __shared__ int abort_s;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int KB = (int)((a.d + kTcKB - 1) / kTcKB);
  const int G32 = (int)(a.d / 32);
  const uint32_t sc_row = (uint32_t)G32 * 2u;  // scale bytes per row
  const uint32_t h_bytes = (uint32_t)((a.B + 15) / 16 * 16) * 128u;
  if (tid == 0) {
    for (int s = 0; s < kI4Stages; ++s) {
      mbar_init(&full_in[s], 1);
      mbar_init(&dq_full[s], 4);
      mbar_init(&op_empty[s], 1);
    }
    mbar_init(&sc_full, 1);
    mbar_init(&tfull, 1);
    mbar_init(&tempty, 4);
    mbar_init(&drain, 1);
    abort_s = 0;
  }
  if (blockIdx.x == 0 && tid < a.n_tickets) a.tickets_to_clear[tid] = 0u;
  if (warp == 2) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
                 ::"r"(smem_addr(&tmem_base_s)), "r"(128u) : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  {  // query blocks: TMA writes only the first Bpad rows; the rest must read as zeros in the MMA
    uint4* hz = reinterpret_cast<uint4*>(smem + I4Layout::kH);
    for (int i = tid; i < (int)(kI4Stages * kI4Blk / 16); i += kTcThreads) hz[i] = make_uint4(0u, 0u, 0u, 0u);
    fence_proxy_async_smem();
  }
  fence_mbar_init();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base_s;
  const int my_tiles = a.n_tiles > (int)blockIdx.x ? (a.n_tiles - (int)blockIdx.x + (int)gridDim.x - 1) / (int)gridDim.x : 0;

  if (warp == 0) {
    // ---------------------------------------------------------------- loads
    if (lane == 0) {
      int it = 0, sc_n = 0;
      bool ok = true;
      for (int j = 0; j < my_tiles && ok; ++j) {
        const int t = (int)blockIdx.x + j * (int)gridDim.x;
        const int64_t r0 = (int64_t)t * 128;
        const int nrows = (int)min((int64_t)128, a.rows - r0);
        // the tile's scales: one bulk copy of whole 16-byte chunks (the ragged tail is read directly
        // by the dequantising threads), once the previous tile's dequantisation is over
        if (j > 0 && !tc_wait(&tempty, (uint32_t)((j - 1) & 1), &abort_s, a.status)) break;
        const uint32_t sc_bytes = (uint32_t)nrows * sc_row;
        const uint32_t sc16 = sc_bytes & ~15u;
        mbar_arrive_expect_tx(&sc_full, sc16);
        if (sc16) bulk_g2s(smem + I4Layout::kSc, reinterpret_cast<const uint8_t*>(a.scales) + (size_t)r0 * sc_row, sc16, &sc_full);
        ++sc_n;
        for (int kb = 0; kb < KB; ++kb, ++it) {
          const int s = it % kI4Stages;
          if (!tc_wait(&op_empty[s], (uint32_t)(((it / kI4Stages) & 1) ^ 1), &abort_s, a.status)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&full_in[s], h_bytes + kI4Nib);
          tma_load_2d(smem + I4Layout::kH + s * kI4Blk, &tmH, kb * kTcKB, 0, &full_in[s]);
          tma_load_2d(smem + I4Layout::kNib + s * kI4Nib, &tmQ, kb * 32, (int)r0, &full_in[s]);
        }
      }
      // leave no copy in flight
      for (int j = max(0, it - kI4Stages); j < it; ++j)
        mbar_wait(&full_in[j % kI4Stages], (uint32_t)((j / kI4Stages) & 1), nullptr, 50000000ull);
      if (sc_n) mbar_wait(&sc_full, (uint32_t)((sc_n - 1) & 1), nullptr, 50000000ull);
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc = (1u << 4) | ((uint32_t)(128 >> 3) << 17) | ((uint32_t)(128 >> 4) << 24);
      const uint32_t sbase = smem_addr(smem);
      int it = 0;
      bool ok = true, issued = false;
      for (int j = 0; j < my_tiles && ok; ++j) {
        if (j > 0 && !tc_wait(&tempty, (uint32_t)((j - 1) & 1), &abort_s, a.status)) break;
        tc_fence_after();
        for (int kb = 0; kb < KB; ++kb, ++it) {
          const int s = it % kI4Stages;
          if (!tc_wait(&dq_full[s], (uint32_t)((it / kI4Stages) & 1), &abort_s, a.status)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t ha = sbase + I4Layout::kH + (uint32_t)s * kI4Blk;
          const uint32_t ba = sbase + I4Layout::kOp + (uint32_t)s * kI4Blk;
#pragma unroll
          for (int k = 0; k < kTcKB / 16; ++k)
            mma_bf16(tmem, sw128_desc(ha + 32u * k), sw128_desc(ba + 32u * k), idesc, (uint32_t)((kb | k) != 0));
          mma_commit(&op_empty[s]);
          issued = true;
        }
        if (ok) mma_commit(&tfull);
      }
      if (issued) {
        mma_commit(&drain);
        mbar_wait(&drain, 0u, nullptr, 50000000ull);
      }
    }
  } else if (warp >= 4) {
    // ---------------------------------------------------------------- dequantise, then the keys
    const int et = tid - 128;  // this thread's tile row (dequantisation) and query (epilogue)
    int it = 0;
    for (int j = 0; j < my_tiles; ++j) {
      const int t = (int)blockIdx.x + j * (int)gridDim.x;
      const int64_t r0 = (int64_t)t * 128;
      const int nrows = (int)min((int64_t)128, a.rows - r0);
      if (!tc_wait(&sc_full, (uint32_t)(j & 1), &abort_s, a.status)) break;
      const uint16_t* sc_s = reinterpret_cast<const uint16_t*>(smem + I4Layout::kSc);
      // the row's scales (the bytes past the bulk copy's last whole chunk straight from memory)
      const uint32_t sc16 = ((uint32_t)nrows * sc_row) & ~15u;
      auto scale_at = [&](int g) {
        const uint32_t off = (uint32_t)et * sc_row + 2u * (uint32_t)g;
        uint16_t bits = 0;
        if (et < nrows) bits = off < sc16 ? sc_s[off / 2] : __ldg(a.scales + (size_t)(r0 + et) * G32 + g);
        return __uint_as_float((uint32_t)bits << 16);
      };
      bool ok = true;
      for (int kb = 0; kb < KB; ++kb, ++it) {
        const int s = it % kI4Stages;
        if (!tc_wait(&full_in[s], (uint32_t)((it / kI4Stages) & 1), &abort_s, a.status)) {
          ok = false;
          break;
        }
        // the query block: BF16 -> fp16 in place (threads split the Bpad x 8 chunks)
        uint8_t* hb = smem + I4Layout::kH + s * kI4Blk;
        for (int ch = et; ch < (int)(h_bytes / 16); ch += 128) {
          uint4* p = reinterpret_cast<uint4*>(hb + 16 * ch);
          *p = bf16x8_to_f16x8(*p);
        }
        // row et of the centroid tile: 64 nibbles -> 64 fp16 values, written 128-byte swizzled
        const uint8_t* nib = smem + I4Layout::kNib + s * kI4Nib + et * 32;
        uint8_t* op = smem + I4Layout::kOp + s * kI4Blk + (et >> 3) * 1024 + (et & 7) * 128;
        const int g0 = 2 * kb;
        const float sc0 = g0 < G32 ? scale_at(g0) : 0.0f, sc1 = g0 + 1 < G32 ? scale_at(g0 + 1) : 0.0f;
        const uint4 w0 = *reinterpret_cast<const uint4*>(nib), w1 = *reinterpret_cast<const uint4*>(nib + 16);
        const uint32_t words[8] = {w0.x, w0.y, w0.z, w0.w, w1.x, w1.y, w1.z, w1.w};
        const __half2 s2a = __half2half2(__float2half_rn(sc0)), s2b = __half2half2(__float2half_rn(sc1));
        const __half2 bias = __half2half2(__ushort_as_half((uint16_t)0x6408u));  // 1032 = 1024 + 8
#pragma unroll
        for (int c = 0; c < 8; ++c) {  // chunk c: columns 8c .. 8c+7 (one 32-bit word of nibbles)
          // nibble n of u is q_n + 8 (two's complement -> offset binary); fp16 0x6400 | b is 1024 + b,
          // so subtracting 1032 gives q exactly, and q times the fp16 scale is exact (<= 11 bits)
          const uint32_t u = words[c] ^ 0x88888888u, u4 = u >> 4;
          uint32_t out[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            // low half: the low nibble of byte e (column 2e); high half: its high nibble (column 2e+1)
            const uint32_t t = __byte_perm(u, u4, (uint32_t)(e | (e << 4) | ((4 + e) << 8) | ((4 + e) << 12)));
            const uint32_t x = (t & 0x000F000Fu) | 0x64006400u;
            const __half2 q = __hsub2(*reinterpret_cast<const __half2*>(&x), bias);
            const __half2 r = __hmul2(q, c < 4 ? s2a : s2b);
            out[e] = *reinterpret_cast<const uint32_t*>(&r);
          }
          *reinterpret_cast<uint4*>(op + ((c ^ (et & 7)) << 4)) = make_uint4(out[0], out[1], out[2], out[3]);
        }
        fence_proxy_async_smem();  // generic writes -> the tensor core's async reads
        __syncwarp();
        if (lane == 0) mbar_arrive(&dq_full[s]);
      }
      if (!ok) break;
      // the accumulators of this tile: lane q of TMEM = query q
      if (!tc_wait(&tfull, (uint32_t)(j & 1), &abort_s, a.status)) break;
      tc_fence_after();
      const int q = et;
      const uint32_t tbase = tmem + ((uint32_t)(32 * (warp & 3)) << 16);
      for (int c0 = 0; c0 < 128; c0 += 32) {
        uint32_t v[32];
        tmem_ld16(tbase + (uint32_t)c0, *reinterpret_cast<uint32_t(*)[16]>(v));
        tmem_ld16(tbase + (uint32_t)c0 + 16u, *reinterpret_cast<uint32_t(*)[16]>(v + 16));
        tmem_ld_wait();
        if (q < a.B) {
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            const int64_t row = r0 + c0 + i;
            if (row < a.rows) {
              const float z = __uint_as_float(v[i]);
              a.out_keys[(int64_t)q * a.rows + row] =
                  SAMPLE ? z / a.tau + gumbel_from_u32(philox_word(a.seed, a.step, (uint32_t)q, 0u, (uint32_t)row)) : z;
            }
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&tempty);  // the next tile may reuse the accumulators and scales
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 2) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(128u) : "memory");
  }
}

// 2-D maps of the INT4 Stage 1: the queries as fp16 (same bits as the BF16 map; the data is converted
// in shared memory) and the nibble rows (uint8, 32-byte boxes of 128 rows, no swizzle).
bool make_map_h16(CUtensorMap* m, const void* base, int64_t d, int64_t rows, uint32_t box_rows) {
  PFN_cuTensorMapEncodeTiled_v12000 fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {(cuuint64_t)d, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)d * 2u};
  cuuint32_t box[2] = {(cuuint32_t)kTcKB, box_rows};
  cuuint32_t estr[2] = {1u, 1u};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT16, 2, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool make_map_nib(CUtensorMap* m, const void* base, int64_t d, int64_t rows) {
  PFN_cuTensorMapEncodeTiled_v12000 fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {(cuuint64_t)(d / 2), (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)(d / 2)};
  cuuint32_t box[2] = {32u, 128u};
  cuuint32_t estr[2] = {1u, 1u};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

bool tc_int4_supported(int64_t d, int B, const void* scales) {
  return B >= 1 && B <= 64 && d % 32 == 0 && (reinterpret_cast<uintptr_t>(scales) & 15u) == 0 &&
         I4Layout::kSc + (size_t)128 * (d / 32) * 2 + 1024 <= 227 * 1024;
}

bool tc_supported(int elem, int64_t d, int B) {
  return elem == kBF16 && d % 8 == 0 && B >= 1 && B <= 64 && encode_fn() != nullptr;
}

cudaError_t launch_tc_head(const void* A, const void* H, TcParams p, int num_sms, cudaStream_t st) {
  if (p.B < 1 || p.B > 64 || p.rows < 1 || (p.qmask && p.b < 1)) return cudaErrorInvalidValue;
  if (p.out_keys && p.qmask) return cudaErrorInvalidValue;
  // Stage-1 keys of few rows take 64-row tiles when that gives every SM at most one
  p.tile_rows = (p.out_keys && (p.rows + 63) / 64 <= num_sms) ? 64 : kTcRows;
  p.n_tiles = (int)((p.rows + p.tile_rows - 1) / p.tile_rows);
  uint32_t box = (uint32_t)p.tile_rows;
  // listed tiles (the kernel reads their count on the device): filled by the query-mask builder
  if (p.tile_list && (!p.qmask || !p.tile_count)) return cudaErrorInvalidValue;
  CUtensorMap mE, mH;
  // copies of the queries where the epilogue bounds the kernel: the head modes, sampled keys of 16
  // queries or more, and keys of more than 32 queries (measured at the Llama-3.2-1B shape; below
  // that the keys' epilogue is light enough, and copies multiply the query bytes each stage brings
  // in: 64 KB of query rows beside 32 KB of centroid rows a stage.  Sampled head at 2 / 4 / 6 / 12
  // queries without copies 52.5 / 64.7 / 73.3 / 103.4 µs against 55.0 / 67.0 / 75.3 / 104.7 with
  // them; at 16, 120.9 against 119.5)
  tc_query_layout(p.B, !p.out_keys || (p.sample && p.B >= 16) || p.B > 32, p.qrows, p.copies);
  // K-blocks per stage: the keys' small tiles fetch a row's consecutive K-blocks together
  p.kbs = p.out_keys ? FH_TC_KEYS_KBS : FH_TC_HEAD_KBS;
  if (!make_map(&mE, A, p.d, p.rows, box) || !make_map(&mH, H, p.d, p.B, (uint32_t)p.qrows))
    return cudaErrorInvalidValue;
  return launch_kernel(mE, mH, p, num_sms, st);
}


cudaError_t launch_tc_keys_int4(const uint8_t* q4, const uint16_t* scales, int64_t rows, int64_t d,
                                const void* H, int B, int sample, float tau, uint64_t seed,
                                uint64_t step, float* out_keys, uint32_t* status,
                                uint32_t* tickets_to_clear, int n_tickets, int num_sms,
                                cudaStream_t st) {
  if (B < 1 || B > 64 || rows < 1 || d % 32 != 0 || n_tickets > kTcThreads) return cudaErrorInvalidValue;
  TcInt4Params p = {};
  p.rows = rows;
  p.d = d;
  p.B = B;
  p.sample = sample;
  p.tau = tau;
  p.seed = seed;
  p.step = step;
  p.scales = scales;
  p.out_keys = out_keys;
  p.status = status;
  p.tickets_to_clear = tickets_to_clear;
  p.n_tickets = tickets_to_clear ? n_tickets : 0;
  p.n_tiles = (int)((rows + 127) / 128);
  CUtensorMap mH, mQ;
  if (!make_map_h16(&mH, H, d, B, (uint32_t)((B + 15) / 16 * 16)) || !make_map_nib(&mQ, q4, d, rows))
    return cudaErrorInvalidValue;
  const size_t dyn = I4Layout::kSc + (size_t)128 * (d / 32) * 2 + 1024;
  if (dyn > 227 * 1024) return cudaErrorInvalidValue;
  auto kern = sample ? k_tc_keys_int4<true> : k_tc_keys_int4<false>;
  cudaError_t e = set_smem_attr(reinterpret_cast<const void*>(kern), dyn);
  if (e != cudaSuccess) return e;
  const int grid = p.n_tiles < num_sms ? p.n_tiles : num_sms;
  kern<<<grid, kTcThreads, dyn, st>>>(mH, mQ, p);
  return cudaGetLastError();
}

}  // namespace fh

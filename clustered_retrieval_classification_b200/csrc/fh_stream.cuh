// fh_stream.cuh — streaming building blocks shared by the FlashHead kernels: dot products of staged
// rows with staged query vectors, the per-warp bulk-copy ring, and the INT4 group dot product.
#pragma once

#include "fh_device.cuh"

namespace fh {

enum ElemSize : int { kElemF32 = 0, kElemBF16 = 1 };

__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// Lane-partial dot product of a staged row (shared address row_s) with a staged query vector
// (shared address h_s); nch = row bytes / 16.  ELEM: 1 = BF16, 0 = fp32.  Four partial sums, one per
// 32-bit word of a chunk, keep four FMA chains in flight; they are added at the end.
template <int ELEM>
__device__ __forceinline__ float row_dot_partial(uint32_t row_s, uint32_t h_s, int nch, int lane) {
  float a0 = 0.0f, a1 = 0.0f, a2 = 0.0f, a3 = 0.0f;
#pragma unroll 4
  for (int ch = lane; ch < nch; ch += 32) {
    const uint4 a = lds_v4(row_s + ch * 16);
    const uint4 h = lds_v4(h_s + ch * 16);
    if (ELEM == 1) {
      a0 = fma2_bf16(a.x, h.x, a0);
      a1 = fma2_bf16(a.y, h.y, a1);
      a2 = fma2_bf16(a.z, h.z, a2);
      a3 = fma2_bf16(a.w, h.w, a3);
    } else {
      a0 = fmaf(__uint_as_float(a.x), __uint_as_float(h.x), a0);
      a1 = fmaf(__uint_as_float(a.y), __uint_as_float(h.y), a1);
      a2 = fmaf(__uint_as_float(a.z), __uint_as_float(h.z), a2);
      a3 = fmaf(__uint_as_float(a.w), __uint_as_float(h.w), a3);
    }
  }
  return (a0 + a1) + (a2 + a3);
}

// Lane-partial dot products of one staged row with QB staged query vectors (QB rows of row bytes
// from h_s; the first nq are live): the row's chunk is read once for all queries, and the QB sums
// are independent FMA chains.
template <int ELEM, int QB>
__device__ __forceinline__ void row_dot_partial_multi(uint32_t row_s, uint32_t h_s, uint32_t row_bytes,
                                                      int nch, int nq, int lane, float (&acc)[QB]) {
#pragma unroll
  for (int q = 0; q < QB; ++q) acc[q] = 0.0f;
#pragma unroll 2
  for (int ch = lane; ch < nch; ch += 32) {
    const uint4 a = lds_v4(row_s + ch * 16);
    float af[8];
    if (ELEM != 1) {
      af[0] = __uint_as_float(a.x); af[1] = __uint_as_float(a.y);
      af[2] = __uint_as_float(a.z); af[3] = __uint_as_float(a.w);
    }
#pragma unroll
    for (int q = 0; q < QB; ++q) {
      if (q < nq) {
        const uint4 h = lds_v4(h_s + (uint32_t)q * row_bytes + ch * 16);
        if (ELEM == 1) {
          float t = acc[q];
          t = fma2_bf16(a.x, h.x, t);
          t = fma2_bf16(a.y, h.y, t);
          t = fma2_bf16(a.z, h.z, t);
          t = fma2_bf16(a.w, h.w, t);
          acc[q] = t;
        } else {
          float t = acc[q];
          t = fmaf(af[0], __uint_as_float(h.x), t); t = fmaf(af[1], __uint_as_float(h.y), t);
          t = fmaf(af[2], __uint_as_float(h.z), t); t = fmaf(af[3], __uint_as_float(h.w), t);
          acc[q] = t;
        }
      }
    }
  }
}

// Copy `bytes` (multiple of 16) from global to shared memory with 16-byte loads by the whole block.
__device__ __forceinline__ void block_copy_g2s(void* dst, const void* src, int bytes) {
  for (int i = threadIdx.x; i < bytes / 16; i += blockDim.x)
    reinterpret_cast<uint4*>(dst)[i] = __ldg(reinterpret_cast<const uint4*>(src) + i);
}

// Issue the bulk copy of one row into a ring slot, counting its bytes on the slot's barrier.
__device__ __forceinline__ void issue_row(uint8_t* slot_dst, const void* src, uint32_t bytes,
                                          uint64_t* bar) {
  mbar_arrive_expect_tx(bar, bytes);
  bulk_g2s(slot_dst, src, bytes, bar);
}

// The per-warp streaming loop.  Rows first, first+W, first+2W, ... below `hi` are brought into the
// warp's ring (K slots of row_bytes) and handed to body(row, shared address) in order.  src(row)
// gives the global address of a row.  Returns false if a wait timed out (status already set).
template <typename Src, typename Body>
__device__ __forceinline__ bool warp_stream_rows(int64_t first, int64_t hi, int W, int lane,
                                                 uint8_t* ring, uint64_t* bars, int K,
                                                 uint32_t row_bytes, const Src& src,
                                                 const Body& body, uint32_t* status) {
  if (first >= hi) return true;
  const int64_t nw = (hi - first + W - 1) / W;
  if (lane == 0) {
    for (int n = 0; n < K && n < nw; ++n) {
      mbar_arrive_expect_tx(&bars[n], row_bytes);
      bulk_g2s(ring + (size_t)n * row_bytes, src(first + (int64_t)W * n), row_bytes, &bars[n]);
    }
  }
  for (int64_t n = 0; n < nw; ++n) {
    const int slot = (int)(n % K);
    const uint32_t parity = (uint32_t)((n / K) & 1);
    if (!mbar_wait(&bars[slot], parity, status)) {
      // Give the copies still in flight a bounded chance to land before the block exits.
      for (int64_t m = n + 1; m < nw && m < n + K; ++m)
        mbar_wait(&bars[m % K], (uint32_t)((m / K) & 1), nullptr, 50000000ull);
      return false;
    }
    body(first + (int64_t)W * n, smem_addr(ring + (size_t)slot * row_bytes));
    __syncwarp();
    if (lane == 0 && n + K < nw) {
      fence_proxy_async_smem();
      mbar_arrive_expect_tx(&bars[slot], row_bytes);
      bulk_g2s(ring + (size_t)slot * row_bytes, src(first + (int64_t)W * (n + K)), row_bytes,
               &bars[slot]);
    }
  }
  return true;
}


// ---- INT4 Stage-1 rows: one 16-byte chunk = 32 nibbles = one 32-column group.
// A nibble n decodes to q = (n ^ 8) - 8 through the float pattern 0x4B000000 | (n ^ 8) = 2^23 + (n ^ 8).
__device__ __forceinline__ float int4_group_dot(const uint4 w, const float* hg) {
  const uint32_t words[4] = {w.x, w.y, w.z, w.w};
  float acc_e = 0.0f, acc_o = 0.0f;  // even and odd columns: two FMA chains, added at the end
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const uint32_t even = (words[i] & 0x0F0F0F0Fu) ^ 0x08080808u;         // columns 8i + 0,2,4,6
    const uint32_t odd = ((words[i] >> 4) & 0x0F0F0F0Fu) ^ 0x08080808u;   // columns 8i + 1,3,5,7
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float qe = __uint_as_float(__byte_perm(even, 0x4B000000u, 0x7440u + j)) - 8388616.0f;
      const float qo = __uint_as_float(__byte_perm(odd, 0x4B000000u, 0x7440u + j)) - 8388616.0f;
      acc_e = fmaf(qe, hg[8 * i + 2 * j], acc_e);
      acc_o = fmaf(qo, hg[8 * i + 2 * j + 1], acc_o);
    }
  }
  return acc_e + acc_o;
}

// One 32-bit word of an INT4 row: columns 0..7 of h (hw), low nibble = even column.
__device__ __forceinline__ float int4_word_dot(const uint32_t w, const float* hw) {
  const uint32_t even = (w & 0x0F0F0F0Fu) ^ 0x08080808u;
  const uint32_t odd = ((w >> 4) & 0x0F0F0F0Fu) ^ 0x08080808u;
  float acc_e = 0.0f, acc_o = 0.0f;
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const float qe = __uint_as_float(__byte_perm(even, 0x4B000000u, 0x7440u + j)) - 8388616.0f;
    const float qo = __uint_as_float(__byte_perm(odd, 0x4B000000u, 0x7440u + j)) - 8388616.0f;
    acc_e = fmaf(qe, hw[2 * j], acc_e);
    acc_o = fmaf(qo, hw[2 * j + 1], acc_o);
  }
  return acc_e + acc_o;
}

// The 32 values of one INT4 group (columns 0..31, low nibble = even column), decoded exactly.
__device__ __forceinline__ void int4_decode32(const uint4 w, float (&dq)[32]) {
  const uint32_t words[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const uint32_t even = (words[i] & 0x0F0F0F0Fu) ^ 0x08080808u;
    const uint32_t odd = ((words[i] >> 4) & 0x0F0F0F0Fu) ^ 0x08080808u;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      dq[8 * i + 2 * j] = __uint_as_float(__byte_perm(even, 0x4B000000u, 0x7440u + j)) - 8388616.0f;
      dq[8 * i + 2 * j + 1] = __uint_as_float(__byte_perm(odd, 0x4B000000u, 0x7440u + j)) - 8388616.0f;
    }
  }
}

}  // namespace fh

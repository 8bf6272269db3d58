// fh_device.cuh — device-side building blocks shared by the FlashHead kernels (sm_100a).
//
// Contents: BF16 widening and 8-wide dot products, the order-preserving float→uint32 key map used by
// every selection and arg-max, Philox4x32-10 and the Gumbel transform, shared-memory mbarriers and
// bulk (TMA engine) copies with bounded waits, and the workspace status word.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace fh {

// ------------------------------------------------------------------------------ status word
// Every workspace starts with a 32-bit status word that keeps the first device-side error of any
// call using it (values are fh_status codes) until fh_ws_status clears it.
enum : uint32_t { kStatusIndex = 3u, kStatusTimeout = 6u };

__device__ __forceinline__ void set_status(uint32_t* status, uint32_t code) {
  if (status) atomicCAS(status, 0u, code);
}

// ------------------------------------------------------------------------------ numbers

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

// acc += Σ_i a_i·b_i over the 8 BF16 values of two 16-byte chunks, in element order.
// c + a_lo·b_lo, then + a_hi·b_hi, for two pairs of BF16 patterns: the mixed-precision FMA multiplies
// the BF16 inputs and adds in FP32 with one rounding, as fmaf does on the inputs widened to FP32 (an
// exact widening), so the value is the same, without the two widening operations per element.
__device__ __forceinline__ float fma2_bf16(uint32_t a, uint32_t b, float c) {
  float r;
  asm("{\n\t.reg .b16 al, ah, bl, bh;\n\t.reg .f32 t;\n\t"
      "mov.b32 {al, ah}, %1;\n\tmov.b32 {bl, bh}, %2;\n\t"
      "fma.rn.f32.bf16 t, al, bl, %3;\n\tfma.rn.f32.bf16 %0, ah, bh, t;\n\t}"
      : "=f"(r)
      : "r"(a), "r"(b), "f"(c));
  return r;
}

__device__ __forceinline__ float dot8_bf16(const uint4& a, const uint4& b, float acc) {
  acc = fma2_bf16(a.x, b.x, acc);
  acc = fma2_bf16(a.y, b.y, acc);
  acc = fma2_bf16(a.z, b.z, acc);
  acc = fma2_bf16(a.w, b.w, acc);
  return acc;
}

// acc += Σ_i a_i·b_i over the 4 fp32 values of two 16-byte chunks, in element order.
__device__ __forceinline__ float dot4_f32(const uint4& a, const uint4& b, float acc) {
  acc = fmaf(__uint_as_float(a.x), __uint_as_float(b.x), acc);
  acc = fmaf(__uint_as_float(a.y), __uint_as_float(b.y), acc);
  acc = fmaf(__uint_as_float(a.z), __uint_as_float(b.z), acc);
  acc = fmaf(__uint_as_float(a.w), __uint_as_float(b.w), acc);
  return acc;
}

// Order-preserving map: a > b (as floats, -0 == +0) ⇔ key(a) > key(b) (as uint32).
__device__ __forceinline__ uint32_t float_key(float f) {
  uint32_t u = __float_as_uint(f);
  if (u == 0x80000000u) u = 0u;  // -0.0 → +0.0
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
__device__ __forceinline__ float key_float(uint32_t k) {
  uint32_t u = (k & 0x80000000u) ? (k & 0x7FFFFFFFu) : ~k;
  return __uint_as_float(u);
}

// Packed arg-max candidate: larger packed value = larger value, then smaller id.  0 = "none".
__device__ __forceinline__ unsigned long long pack_best(float val, uint32_t id) {
  return ((unsigned long long)float_key(val) << 32) | (unsigned long long)(~id);
}
__device__ __forceinline__ uint32_t best_id(unsigned long long packed) {
  return ~(uint32_t)(packed & 0xFFFFFFFFull);
}

__device__ __forceinline__ unsigned long long warp_max_u64(unsigned long long v) {
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) {
    unsigned long long o = __shfl_xor_sync(0xFFFFFFFFu, v, off);
    v = o > v ? o : v;
  }
  return v;
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xFFFFFFFFu, v, off);
  return v;
}

// ------------------------------------------------------------------------------ Philox4x32-10
// Salmon, Moraes, Dror, Shaw, SC'11.  Ten rounds; multipliers 0xD2511F53 / 0xCD9E8D57; key bumped by
// the Weyl constants 0x9E3779B9 / 0xBB67AE85 between rounds.
__device__ __forceinline__ uint4 philox4x32_10(uint4 ctr, uint32_t k0, uint32_t k1) {
#pragma unroll
  for (int r = 0; r < 10; ++r) {
    if (r) {
      k0 += 0x9E3779B9u;
      k1 += 0xBB67AE85u;
    }
    const uint32_t lo_a = 0xD2511F53u * ctr.x, hi_a = __umulhi(0xD2511F53u, ctr.x);
    const uint32_t lo_b = 0xCD9E8D57u * ctr.z, hi_b = __umulhi(0xCD9E8D57u, ctr.z);
    ctr = make_uint4(hi_b ^ ctr.y ^ k0, lo_b, hi_a ^ ctr.w ^ k1, lo_a);
  }
  return ctr;
}

// The four words of the block holding element group g = elem >> 2 (the library's counter layout:
// counter = (g, row, step lo, (stream << 24) | (step hi & 0xFFFFFF)), key = seed).
__device__ __forceinline__ uint4 philox_block(uint64_t seed, uint64_t step, uint32_t row,
                                              uint32_t stream, uint32_t group) {
  uint4 ctr = make_uint4(group, row, (uint32_t)step,
                         (stream << 24) | ((uint32_t)(step >> 32) & 0xFFFFFFu));
  return philox4x32_10(ctr, (uint32_t)seed, (uint32_t)(seed >> 32));
}

__device__ __forceinline__ uint32_t philox_word(uint64_t seed, uint64_t step, uint32_t row,
                                                uint32_t stream, uint32_t elem) {
  uint4 w = philox_block(seed, step, row, stream, elem >> 2);
  switch (elem & 3u) {
    case 0: return w.x;
    case 1: return w.y;
    case 2: return w.z;
    default: return w.w;
  }
}

// u = ((x >> 9) + 0.5)·2^-23 has at most 24 significant bits, so it is exact in fp32 and lies in
// (0, 1); G = -log(-log u) with CUDA's logf.
__device__ __forceinline__ float gumbel_from_u32(uint32_t x) {
  const float u = ((float)(x >> 9) + 0.5f) * 1.1920928955078125e-7f;
  return -logf(-logf(u));
}

// ------------------------------------------------------------------------------ memory

__device__ __forceinline__ uint4 ld_stream_v4(const void* p) {
  uint4 r;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "l"(p));
  return r;
}

__device__ __forceinline__ uint4 lds_v4(uint32_t saddr) {
  uint4 r;
  asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "r"(saddr));
  return r;
}

__device__ __forceinline__ uint32_t smem_addr(const void* p) {
  return (uint32_t)__cvta_generic_to_shared(p);
}

__device__ __forceinline__ uint64_t global_timer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
  return t;
}

// ------------------------------------------------------------------------------ mbarriers

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(bar)), "r"(count));
}

__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_addr(bar)),
               "r"(bytes)
               : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_addr(bar)) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_addr(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// Wait until phase `parity` of `bar` completes, for at most `limit_ns` nanoseconds.  On timeout the
// workspace status becomes FH_ERR_TIMEOUT and false is returned; the caller then stops its work.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, uint32_t* status,
                                          uint64_t limit_ns = 500000000ull) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = global_timer_ns();
  for (;;) {
    for (int i = 0; i < 64; ++i)
      if (mbar_try_wait(bar, parity)) return true;
    if (global_timer_ns() - t0 > limit_ns) {
      set_status(status, kStatusTimeout);
      return false;
    }
  }
}

// Bulk copy (TMA engine, no tensor map) of `bytes` from global memory into this CTA's shared memory;
// completion is counted on `bar` in bytes.  src, dst and bytes must be multiples of 16.
__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_addr(dst)),
      "l"(src), "r"(bytes), "r"(smem_addr(bar))
      : "memory");
}

// ------------------------------------------------------------------------------ PDL
// Programmatic dependent launch: the next kernel of the stream may start its prologue once every block
// of this kernel has called launch_dependents; wait_prior blocks until the preceding kernel finished
// and its writes are visible.  Both are no-ops when the launch did not request programmatic
// serialisation.
__device__ __forceinline__ void pdl_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}
__device__ __forceinline__ void pdl_wait_prior() {
  asm volatile("griddepcontrol.wait;" ::: "memory");
}

}  // namespace fh

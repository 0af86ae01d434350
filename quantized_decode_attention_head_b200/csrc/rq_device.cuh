// Device-side helpers: packed-format tables, tensor-core MMA, fragment
// transpose, mbarrier and bulk-copy primitives (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cstdint>

#include "rq_internal.h"

namespace rq {

// ----------------------------------------------------------- format tables
// Slot list of one lane ordered by (class, word, slot); entry i -> (word, slot).
// b = 2: slot classes 0,1,2,3,4,0,1,2 (slots 0-4 of a 16-bit half lie inside
//        an fp16 mantissa in place, 5-7 after a 10-bit shift);
// b = 4: classes 0,1,0,1; b = 3, 8: all class 0 (natural order).
__host__ __device__ constexpr int slot_word(int b, int W, int i) {
  return b == 2 ? (i < 6 * W ? (i % (2 * W)) / 2 : (i - 6 * W) % W)
       : b == 4 ? (i % (2 * W)) / 2
                : i / (codes_per_word(b) / 2);
}
__host__ __device__ constexpr int slot_pos(int b, int W, int i) {
  return b == 2 ? (i < 6 * W ? i / (2 * W) + 5 * ((i % (2 * W)) % 2) : 3 + (i - 6 * W) / W)
       : b == 4 ? i / (2 * W) + 2 * ((i % (2 * W)) % 2)
                : i % (codes_per_word(b) / 2);
}
// Slot-list index of the K pair (mb, kb, r) and of the V pair (mb, kb, r).
__host__ __device__ constexpr int k_pair_index(int D, int mb, int kb, int r) {
  return 4 * ((mb * 2 + (r & 1)) * (D / 32) + kb / 2) + (kb & 1) * 2 + (r >> 1);
}
__host__ __device__ constexpr int v_pair_index(int mb, int kb, int r) {
  return 4 * (mb * 2 + (r & 1)) + kb * 2 + (r >> 1);
}
// Byte offset of word w of a lane inside a code blob of W words per lane.
__host__ __device__ constexpr int word_offset(int W, int lane, int w) {
  return w < 4 * (W / 4) ? ((w / 4) * 32 + lane) * 16 + (w % 4) * 4
                         : (W / 4) * 512 + ((w - 4 * (W / 4)) * 32 + lane) * 4;
}

// Class of a slot: how many b-bit steps its codes sit above the lowest
// position from which they are read in place (fp16 mantissa = bits 0..9 of a
// 16-bit half).  b=2: slots 0..4 in place, 5..7 after a 10-bit shift;
// b=4: slots 0,1 in place, 2,3 after an 8-bit shift; b=3, 8: every slot is
// shifted down to bit 0 (class 0).
__host__ __device__ constexpr int slot_class(int b, int p) {
  return b == 2 ? (p < 5 ? p : p - 5) : b == 4 ? (p & 1) : 0;
}
// Class shared by the four pairs of quad q of a blob with W words per lane.
__host__ __device__ constexpr int quad_class(int b, int W, int q) { return slot_class(b, slot_pos(b, W, 4 * q)); }

// Pair of b-bit codes of slot p of word w as an fp16x2 of subnormals
// c * 2^(b*class - 24): the code bits become the fp16 mantissa with a zero
// exponent field, so the values are exact and need no offset removal.  The
// 2^(b*class) factor is undone by the per-quad scale.
template <int B>
__device__ __forceinline__ uint32_t extract_pair(const uint32_t* words, int w, int p) {
  constexpr uint32_t m = (1u << B) - 1u;
  constexpr uint32_t mm = m | (m << 16);
  if (B == 2) return p < 5 ? (words[w] & (mm << (2 * p))) : ((words[w] >> 10) & (mm << (2 * (p - 5))));
  if (B == 4) return p < 2 ? (words[w] & (mm << (4 * p))) : ((words[w] >> 8) & (mm << (4 * (p - 2))));
  if (B == 8) return p == 0 ? (words[w] & mm) : ((words[w] >> 8) & mm);
  return (words[w] >> (B * p)) & mm;
}

// ------------------------------------------------------------ tensor cores
// D = A(16x16 f16, row) * B(16x8 f16, col) + C, fp32 accumulate.
__device__ __forceinline__ void mma_f16(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 "
      "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};\n"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// Transpose an 8x8 b16 matrix held one row-pair per thread (m8n8 fragment).
__device__ __forceinline__ uint32_t movmatrix_trans(uint32_t x) {
  uint32_t y;
  asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;\n" : "=r"(y) : "r"(x));
  return y;
}

__device__ __forceinline__ uint32_t pack_half2(float lo, float hi) {
  __half2 h = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&h);
}

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;\n" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ float bf16_bits_to_float(uint32_t bits16) { return __uint_as_float(bits16 << 16); }

// ------------------------------------------------------ mbarrier / bulk copy
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;\n" ::"r"(smem_u32(bar)), "r"(count));
}
__device__ __forceinline__ void mbar_fence_init() {
  asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
}
__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;\n" ::"r"(smem_u32(bar)), "r"(bytes)
               : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];\n" ::"r"(smem_u32(bar)) : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}
__device__ __forceinline__ uint64_t global_timer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %globaltimer;\n" : "=l"(t));
  return t;
}
// Bounded wait: gives up after ~1 s and returns false.
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t* bar, uint32_t parity) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = global_timer_ns();
  while (true) {
    if (mbar_try_wait(bar, parity)) return true;
    if (global_timer_ns() - t0 > 1000000000ull) return false;
  }
}
// Orders this thread's earlier generic-proxy shared-memory accesses before
// later async-proxy (bulk copy) accesses of the same memory.
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;\n" ::: "memory");
}
// 1-D bulk copy global -> shared, completion counted on an mbarrier (bytes).
__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];\n" ::"r"(
          smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

}  // namespace rq

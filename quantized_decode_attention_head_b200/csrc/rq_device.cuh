// Device-side helpers: packed-format tables, integer tensor-core MMA,
// mbarrier and bulk-copy primitives (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cstdint>

#include "rq_internal.h"

namespace rq {

// ----------------------------------------------------------- format tables
// A lane of a code blob owns D/4 registers (rho, kh) of four bytes: the 8-bit
// A-operand fragments of the m16n8k32 integer MMA.  Row group rho has class
// j = rho mod C and both its registers come from source sigma = 2*(rho/C)+kh;
// the code of byte e sits at bits 8e + b*j .. 8e + b*j + b - 1 of the source,
// so masking the source word to those bits of every byte yields four codes
// scaled by 2^(b*j).  3-bit sources past the W words are assembled from the
// top bit pairs (bits 6, 7 of each byte) of three consecutive words.
__host__ __device__ constexpr int n_classes(int b) { return b == 2 ? 4 : b == 8 ? 1 : 2; }
__host__ __device__ constexpr int reg_class(int b, int rho) { return rho % n_classes(b); }
__host__ __device__ constexpr int reg_source(int b, int rho, int kh) { return 2 * (rho / n_classes(b)) + kh; }
__host__ __device__ constexpr uint32_t class_mask(int b, int j) {
  return (((1u << b) - 1u) * 0x01010101u) << (b * j);
}
// Byte offset of word w of a lane inside a code blob of W words per lane.
__host__ __device__ constexpr int word_offset(int W, int lane, int w) {
  return w < 4 * (W / 4) ? ((w / 4) * 32 + lane) * 16 + (w % 4) * 4
                         : (W / 4) * 512 + ((w - 4 * (W / 4)) * 32 + lane) * 4;
}

// Register (rho, kh) of a lane from its W code words (rho, kh compile-time
// after unrolling): four codes * 2^(b*j) as u8 bytes.
template <int B, int W>
__device__ __forceinline__ uint32_t code_reg(const uint32_t* words, int rho, int kh) {
  const int j = reg_class(B, rho), s = reg_source(B, rho, kh);
  if (B == 3 && s >= W) {
    const int q = s - W;
    const uint32_t f = ((words[3 * q] >> 6) & 0x03030303u) | ((words[3 * q + 1] >> 4) & 0x0C0C0C0Cu) |
                       ((words[3 * q + 2] >> 2) & 0x30303030u);
    return f & class_mask(3, j);
  }
  return words[s] & class_mask(B, j);
}

// Places code c (B bits) of byte e of register (rho, kh) into the lane's words.
template <int B, int W>
__device__ __forceinline__ void put_code(uint32_t* words, int rho, int kh, int e, uint32_t c) {
  const int j = reg_class(B, rho), s = reg_source(B, rho, kh);
  if (B == 3 && s >= W) {
    const int q = s - W;
#pragma unroll
    for (int k = 0; k < 3; ++k) {
      const int f = 3 * j + k;
      words[3 * q + f / 2] |= ((c >> k) & 1u) << (8 * e + 6 + (f & 1));
    }
  } else {
    words[s] |= c << (8 * e + B * j);
  }
}

// ------------------------------------------------------------ tensor cores
// D = A(16x32 u8, row) * B(32x8 s8 / u8, col) + C, s32 accumulate; every C
// element is the same value c.  Results are returned as raw 32-bit words.
// (The MMAs are pure register operations: not volatile, so the compiler may
// schedule them freely.)
__device__ __forceinline__ void imma_u8s8(uint32_t (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1,
                                          uint32_t c) {
  asm(
      "mma.sync.aligned.m16n8k32.row.col.s32.u8.s8.s32 "
      "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%10,%11,%12,%13};\n"
      : "=r"(d[0]), "=r"(d[1]), "=r"(d[2]), "=r"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1), "r"(c), "r"(c), "r"(c), "r"(c));
}
__device__ __forceinline__ void imma_u8u8(uint32_t (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1,
                                          uint32_t c) {
  asm(
      "mma.sync.aligned.m16n8k32.row.col.s32.u8.u8.s32 "
      "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%10,%11,%12,%13};\n"
      : "=r"(d[0]), "=r"(d[1]), "=r"(d[2]), "=r"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1), "r"(c), "r"(c), "r"(c), "r"(c));
}

// bf16 MMAs of the window path, fp32 accumulate in place:
// m16n8k16 (A a0..a3, B b0, b1) and m16n8k8 (A a0, a1, B b0).
__device__ __forceinline__ void mma_bf16_k16(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                             uint32_t b0, uint32_t b1) {
  asm(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 "
      "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};\n"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}
__device__ __forceinline__ void mma_bf16_k8(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t b0) {
  asm(
      "mma.sync.aligned.m16n8k8.row.col.f32.bf16.bf16.f32 "
      "{%0,%1,%2,%3}, {%4,%5}, {%6}, {%0,%1,%2,%3};\n"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(b0));
}
// Four 8x8 b16 matrices from shared memory; lanes 8i .. 8i + 7 address the
// rows of matrix i.  Plain: thread (g, t) receives row g, columns 2t, 2t + 1;
// .trans: rows 2t, 2t + 1 of column g.
__device__ __forceinline__ void ldsm_x4(uint32_t (&r)[4], uint32_t addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr)
               : "memory");
}
__device__ __forceinline__ void ldsm_x4_trans(uint32_t (&r)[4], uint32_t addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr)
               : "memory");
}
// (lo, hi) -> bf16x2 bits, each rounded to nearest even; lo in the low half.
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;\n" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;\n" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ float bf16_bits_to_float(uint32_t bits16) { return __uint_as_float(bits16 << 16); }

// ------------------------------------------- programmatic dependent launch
// Lets the next kernel of the stream be scheduled before this one ends.
__device__ __forceinline__ void griddep_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;\n" ::: "memory");
}
// Waits until every prerequisite grid has completed and its memory is visible
// (returns at once when the kernel was launched without the dependency).
__device__ __forceinline__ void griddep_wait() { asm volatile("griddepcontrol.wait;\n" ::: "memory"); }

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
// Bounded wait: gives up after limit_ns (default ~1 s) and returns false.
constexpr uint64_t kWaitLimitNs = 1000000000ull;
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t* bar, uint32_t parity, uint64_t limit_ns = kWaitLimitNs) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = global_timer_ns();
  while (true) {
    if (mbar_try_wait(bar, parity)) return true;
    if (global_timer_ns() - t0 > limit_ns) return false;
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

// L2 policy for data that a launch reads once (packed tile records): evicted
// first, so that the lines later launches reuse (window rows, workspace,
// kernel code) stay in L2.
__device__ __forceinline__ uint64_t l2_evict_first_policy() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;\n" : "=l"(p));
  return p;
}

// bulk_g2s with an L2 cache policy.
__device__ __forceinline__ void bulk_g2s_hint(void* dst, const void* src, uint32_t bytes, uint64_t* bar,
                                              uint64_t policy) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint [%0], [%1], %2, [%3], %4;\n" ::"r"(
          smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar)), "l"(policy)
      : "memory");
}

// Completion count of a device-scope counter, taken by one thread of a CTA
// after a CTA barrier: the acquire-release add publishes the CTA's earlier
// global writes (ordered before this thread by the barrier) to the CTA that
// takes the final count, and gives that CTA the others' writes, which its
// other threads read after the next barrier.  Returns the old value.
__device__ __forceinline__ uint32_t count_acq_rel(uint32_t* p) {
  uint32_t old;
  asm volatile("atom.acq_rel.gpu.global.add.u32 %0, [%1], 1;\n" : "=r"(old) : "l"(p) : "memory");
  return old;
}
// L2 prefetch of a global range (no completion to wait for); address and
// size multiples of 16 bytes.
__device__ __forceinline__ void l2_prefetch(const void* src, uint32_t bytes) {
  asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;\n" ::"l"(src), "r"(bytes) : "memory");
}

// When p: arms bar for `bytes` and starts the bulk copy src -> dst with an L2
// policy.  Both steps are predicated inside one asm block, so a caller that
// passes a lane-dependent p does not branch.
__device__ __forceinline__ void bulk_g2s_hint_if(bool p, void* dst, const void* src, uint32_t bytes, uint64_t* bar,
                                                 uint64_t policy) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %0, 0;\n"
      " @p mbarrier.arrive.expect_tx.shared::cta.b64 _, [%1], %2;\n"
      " @p cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint [%3], [%4], %2, [%1], %5;\n"
      "}\n" ::"r"((int)p),
      "r"(smem_u32(bar)), "r"(bytes), "r"(smem_u32(dst)), "l"(src), "l"(policy)
      : "memory");
}

}  // namespace rq

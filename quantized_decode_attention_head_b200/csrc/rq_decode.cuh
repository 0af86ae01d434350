// Split-K decode attention over the packed cache (sm_100a): device code and
// launch templates.  Each rq_decode_<D>x<G>.cu translation unit instantiates
// one (head_dim, GQA group) pair; rq_decode.cu holds the dispatchers.
#pragma once
//
//
// One CTA = one work item of one (layer, batch, kv-head) stream: a
// contiguous range of at most 128 packed tiles (items 0..n_splits-1), chunks
// of the bf16 sink + recent window (the next items, on the bf16 tensor
// cores), or, in a fused step before a tile flush, the pack-ahead of that
// tile.  Four warps process tiles; lane 0 of each streams the warp's own tile
// records into a private ring of shared-memory stages with 1-D bulk copies
// (cp.async.bulk, TMA engine) completing on mbarriers.  Each CTA merges its
// warps' partial softmax states (log-sum-exp) and publishes one partial; the
// last item of a stream to finish (or, past 16 items, of each group of 8,
// then of the groups) merges the partials and writes the output -- no second
// launch.  With an explicit split count, consecutive items form
// thread-block clusters whose first CTA merges the cluster through
// distributed shared memory.
//
// Per tile (32 tokens), with the G query heads that share the kv head:
//   q.K^T  : integer tensor-core MMA (mma.sync m16n8k32, u8 x s8 -> s32).
//            A = the packed K codes, masked in registers to one code class
//            per byte (a byte then reads code * 2^(b j), exact), B = q in
//            16-bit fixed point per head split into two s8 terms
//            (q_int = 256 q1 + q2, one column each).  One MMA per 32-channel
//            K group, so the group's fp16 scale and bf16 zero factor out of
//            the exact integer sum (InnerQ grouping):
//              score = sum_grp s_grp * sum_d q_d c_d + z_grp * sum_d q_d.
//   softmax: online, base 2, running max per head; P in 16-bit fixed point
//            relative to the running max, split into two u8 terms.
//   P.V    : MMA (u8 x u8 -> s32) with A = V codes (channel x token), B = P;
//            the V scale/zero are per channel for the whole tile:
//              o_d += s_d * sum_t p_t c_td + z_d * sum_t p_t,
//            where sum_t p_t comes from the same MMA with A = 1.
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include <cooperative_groups.h>

#include <cfloat>
#include <map>
#include <mutex>
#include <tuple>

#include "rq_device.cuh"
#include "rq_internal.h"
#include "rq_pack.cuh"

namespace rq {
namespace {

constexpr int NW = kDecodeConsumerWarps;
constexpr int kMaxStages = 8;                // per-warp ring depth limit
constexpr uint32_t kBiasBits = 0x4B400000u;  // bits of 1.5 * 2^23
constexpr float kBias = 12582912.0f;         // 1.5 * 2^23
constexpr float kPScale = 65535.0f;          // P in 16-bit fixed point: p_int = rint(p * 65535)
constexpr float kQMax = 32639.0f;            // q_int in [-32639, 32639] = 256 * q1 + q2, q1, q2 in s8
// normalized caches: q_int in [-8323072, 8323072] = 65536 q1 + 256 q2 + q3, all s8
constexpr float kQMax3 = 8323072.0f;

template <int D, int G>
struct Cfg {
  static constexpr int NG = D / 32;                  // K groups per token (one k32 MMA each)
  static constexpr int NB = (G + 3) / 4;             // 8-column blocks: 4 heads x 2 terms
  static constexpr int HB = G < 4 ? G : 4;           // heads per block
  static constexpr int PART = partial_floats(G, D);  // floats per partial state (16-byte multiple)
  static constexpr int KMW = NG;                     // K meta words converted per lane
  static constexpr int VMW = D / 32;                 // V meta words converted per lane
  static constexpr int KSTR = NG * 8 + 4;            // floats per gid row of the K scale scratch
  static constexpr int VSTR = (D / 8) * 2 + 4;       // floats per gid row of the V scale scratch
  static constexpr int SCRATCH = 8 * (KSTR + VSTR);  // floats per warp
};

// Per-warp state.  Thread (gid, tig) owns, in block nb, head 4nb + tig of the
// MMA results (columns 2 tig, 2 tig + 1 = the two terms of that head).
// QT = 2: q in 16-bit fixed point (two s8 terms); QT = 3: 24-bit (three s8
// terms, for caches whose K normalization factors are folded into q and
// widen its range): terms 1, 2 in qb, term 3 in qb3 (column 2 h, 2 h + 1 = 0).
template <int D, int G, int QT = 2>
struct WarpState {
  using C = Cfg<D, G>;
  uint32_t qb[C::NB][C::NG][2];  // q B-fragments: column n = 2 h + term, bytes = s8 terms
  uint32_t qb3[C::NB][C::NG][QT == 3 ? 2 : 1];  // third-term B-fragments (QT = 3)
  float2 qz[C::NB][C::NG];       // sum of q_int over group g (both halves) -- zero-point term
  float xs[C::NB];               // sq * softmax scale * log2(e)
  float m[C::NB], l[C::NB];      // running max (log2 units) and sum of p (x 65535)
  float2 o[C::NB][D / 16];       // .x channel 16 mb + gid, .y channel 16 mb + 8 + gid (x 65535)
  float kf[C::KMW], vf[C::VMW];  // class factors 2^(-b j) of the meta words this lane converts
};

// Packed fp32 pairs (FFMA2 / FMUL2 / FADD2 on sm_100): two lanes of
// arithmetic per instruction, each rounded as its scalar counterpart.
__device__ __forceinline__ float2 ffma2(float2 a, float2 b, float2 c) { return __ffma2_rn(a, b, c); }
__device__ __forceinline__ float2 fmul2(float2 a, float2 b) { return __fmul2_rn(a, b); }
__device__ __forceinline__ float2 fadd2(float2 a, float2 b) { return __fadd2_rn(a, b); }

// The two-term results (hi, lo) of rows gid and gid + 8 of one MMA -> the
// pair (256 hi + lo) of both rows in fp32: |256 hi + lo| < 2^31 is exact in
// int32, one rounding to fp32 per row.  (The alternative -- C = the bits of
// 1.5 * 2^23, so that the results read as floats, and packed subtractions --
// pairs registers of different rows and measured more instructions.)
__device__ __forceinline__ float2 combine_terms(const uint32_t (&c)[4]) {
  return make_float2((float)((int)c[0] * 256 + (int)c[1]), (float)((int)c[2] * 256 + (int)c[3]));
}

__device__ __forceinline__ float pow2i(int e) { return __int_as_float((e + 127) << 23); }

// q of the G heads -> per-head 16-bit fixed point (sq = max|q_h| / 32639)
// split into two s8 terms q_int = 256 q1 + q2, laid out as the k32 x n8
// B-fragments of the q.K^T MMA (column n = 2 * head + term).
template <int D, int G, int KB, int VB, int QT>
__device__ void setup_query(WarpState<D, G, QT>& st, const uint16_t* qh, const float* nrm, float scale_log2,
                            int lane) {
  using C = Cfg<D, G>;
  const int gid = lane >> 2, tig = lane & 3;
  const int hl = gid >> 1, tau = gid & 1;
#pragma unroll
  for (int nb = 0; nb < C::NB; ++nb) {
    const bool hv = hl < C::HB;
    const uint16_t* qp = qh + (size_t)(4 * nb + hl) * D;
    float qv[C::NG][8];
    float mx = 0.0f;
    int ps[C::NG];
#pragma unroll
    for (int g = 0; g < C::NG; ++g) {
      ps[g] = 0;
#pragma unroll
      for (int kh = 0; kh < 2; ++kh) {
        uint2 u = make_uint2(0u, 0u);
        if (hv) u = __ldg(reinterpret_cast<const uint2*>(qp + 32 * g + 16 * kh + 4 * tig));
        const uint32_t w[2] = {u.x, u.y};
        // K normalization folded into q for the packed tiles: q_d * n_d (exact, powers of two)
        const float4 nv = *reinterpret_cast<const float4*>(nrm + 32 * g + 16 * kh + 4 * tig);
        const float nn[4] = {nv.x, nv.y, nv.z, nv.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float x = bf16_bits_to_float(e & 1 ? w[e >> 1] >> 16 : w[e >> 1] & 0xFFFFu) * nn[e];
          qv[g][4 * kh + e] = x;
          mx = fmaxf(mx, fabsf(x));
        }
      }
    }
    // the four lanes of a quad hold all D channels of one head
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
    constexpr float QM = QT == 3 ? kQMax3 : kQMax;
    constexpr int QI = (int)QM;
    const float inv = mx > 0.0f ? QM / mx : 0.0f;
    const float sq = mx * (1.0f / QM);
#pragma unroll
    for (int g = 0; g < C::NG; ++g)
#pragma unroll
      for (int kh = 0; kh < 2; ++kh) {
        uint32_t packed = 0u, packed3 = 0u;
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          int qi = __float2int_rn(qv[g][4 * kh + e] * inv);
          qi = qi > QI ? QI : (qi < -QI ? -QI : qi);
          if constexpr (QT == 3) {
            // qi = 65536 q1 + 256 q2 + q3, every term in [-128, 127]
            const int q3 = ((qi + 128) & 0xFF) - 128;
            const int r = (qi - q3) >> 8;
            const int q2 = ((r + 128) & 0xFF) - 128;
            const int q1 = (r - q2) >> 8;
            packed |= ((uint32_t)(tau ? q2 : q1) & 0xFFu) << (8 * e);
            packed3 |= ((uint32_t)(tau ? 0 : q3) & 0xFFu) << (8 * e);
          } else {
            const int q1 = (qi + 128) >> 8;  // floor((qi + 128) / 256)
            const int q2 = qi - (q1 << 8);   // in [-128, 127]
            packed |= ((uint32_t)(tau ? q2 : q1) & 0xFFu) << (8 * e);
          }
          ps[g] += qi;  // exact: |sum| < 2^31
        }
        st.qb[nb][g][kh] = hv ? packed : 0u;
        if constexpr (QT == 3) st.qb3[nb][g][kh] = hv ? packed3 : 0u;
      }
    // zero-point term: sum of the SAME rounded q_int over each group, so the
    // code and zero terms together are exactly (s c + z) . q_int and the large
    // cancellation between them (z = group minimum) leaves no rounding residue
#pragma unroll
    for (int g = 0; g < C::NG; ++g) {
      ps[g] += __shfl_xor_sync(0xffffffffu, ps[g], 1);
      ps[g] += __shfl_xor_sync(0xffffffffu, ps[g], 2);
    }
    // the result columns of thread (gid, tig) belong to head 4nb + tig, whose
    // statistics live in lane 8 tig (gid = 2 tig, term 0)
    const float sq_c = __shfl_sync(0xffffffffu, sq, 8 * tig);
#pragma unroll
    for (int g = 0; g < C::NG; ++g) {
      const float z = (float)__shfl_sync(0xffffffffu, ps[g], 8 * tig);  // exact below 2^24 (QT = 2)
      st.qz[nb][g] = make_float2(z, z);
    }
    st.xs[nb] = sq_c * scale_log2;
    st.m[nb] = -INFINITY;
    st.l[nb] = 0.0f;
#pragma unroll
    for (int mb = 0; mb < D / 16; ++mb) st.o[nb][mb] = make_float2(0.0f, 0.0f);
  }
  // class factors of the metadata words this lane converts (see convert_meta)
#pragma unroll
  for (int k = 0; k < C::KMW; ++k) {
    const int w = C::KMW * lane + k, g = w / 32, i = (w % 32) % 4;
    st.kf[k] = pow2i(-KB * reg_class(KB, i * C::NG + g));
  }
#pragma unroll
  for (int k = 0; k < C::VMW; ++k) {
    const int w = C::VMW * lane + k, rho = w % (D / 8);
    st.vf[k] = pow2i(-VB * reg_class(VB, rho));
  }
}

template <int W>
__device__ __forceinline__ void load_words(uint32_t (&w)[W], const uint8_t* blob, int lane) {
#pragma unroll
  for (int c = 0; c < W / 4; ++c) {
    const uint4 u = *reinterpret_cast<const uint4*>(blob + word_offset(W, lane, 4 * c));
    w[4 * c] = u.x;
    w[4 * c + 1] = u.y;
    w[4 * c + 2] = u.z;
    w[4 * c + 3] = u.w;
  }
#pragma unroll
  for (int k = 4 * (W / 4); k < W; ++k) w[k] = *reinterpret_cast<const uint32_t*>(blob + word_offset(W, lane, k));
}

__device__ __forceinline__ float half_lo_to_float(uint32_t m) {
  return __half2float(__ushort_as_half((unsigned short)(m & 0xFFFFu)));
}

// Metadata of one tile -> scale * 2^(-b j) and zero floats in the warp's
// scratch, each entry converted once, stored per pair of MMA rows as
// (s_a, s_b, z_a, z_b) so that one 16-byte load gives the scale pair and the
// zero pair of a packed epilogue.  K: pair (i = 2 mb, 2 mb + 1) of group g
// for tokens gid + 8 i; V: pair (rho = 2 mb, 2 mb + 1) for channels
// 16 mb + gid and 16 mb + 8 + gid.
template <int D, int G, int KB, int VB, int QT>
__device__ __forceinline__ void convert_meta(const uint8_t* rec, const WarpState<D, G, QT>& st, float* ks, float* vs,
                                             int lane) {
  using C = Cfg<D, G>;
  const uint32_t* kmeta = reinterpret_cast<const uint32_t*>(rec + blob_bytes(KB, D));
  const uint32_t* vmeta = reinterpret_cast<const uint32_t*>(rec + blob_bytes(KB, D) + 4 * D + blob_bytes(VB, D));
  uint32_t km[C::KMW], vm[C::VMW];
  if constexpr (C::KMW == 4) {
    const uint4 u = *reinterpret_cast<const uint4*>(kmeta + 4 * lane);
    km[0] = u.x, km[1] = u.y, km[2] = u.z, km[3] = u.w;
  } else {
    const uint2 u = *reinterpret_cast<const uint2*>(kmeta + 2 * lane);
    km[0] = u.x, km[1] = u.y;
  }
  if constexpr (C::VMW == 4) {
    const uint4 u = *reinterpret_cast<const uint4*>(vmeta + 4 * lane);
    vm[0] = u.x, vm[1] = u.y, vm[2] = u.z, vm[3] = u.w;
  } else {
    const uint2 u = *reinterpret_cast<const uint2*>(vmeta + 2 * lane);
    vm[0] = u.x, vm[1] = u.y;
  }
  // consecutive words k, k + 1 form one row pair: (s_k, s_k+1, z_k, z_k+1)
  float kv[2 * C::KMW], vv[2 * C::VMW];
#pragma unroll
  for (int k = 0; k < C::KMW; k += 2) {
    const float2 sc = fmul2(make_float2(half_lo_to_float(km[k]), half_lo_to_float(km[k + 1])),
                            make_float2(st.kf[k], st.kf[k + 1]));
    kv[2 * k] = sc.x;
    kv[2 * k + 1] = sc.y;
    kv[2 * k + 2] = __uint_as_float(km[k] & 0xFFFF0000u);
    kv[2 * k + 3] = __uint_as_float(km[k + 1] & 0xFFFF0000u);
  }
#pragma unroll
  for (int k = 0; k < C::VMW; k += 2) {
    const float2 sc = fmul2(make_float2(half_lo_to_float(vm[k]), half_lo_to_float(vm[k + 1])),
                            make_float2(st.vf[k], st.vf[k + 1]));
    vv[2 * k] = sc.x;
    vv[2 * k + 1] = sc.y;
    vv[2 * k + 2] = __uint_as_float(vm[k] & 0xFFFF0000u);
    vv[2 * k + 3] = __uint_as_float(vm[k + 1] & 0xFFFF0000u);
  }
  // word w = KMW * lane + k: group w / 32, gid (w % 32) / 4, i = w % 4
  {
    const int w0 = C::KMW * lane;
    float* dst = ks + ((w0 % 32) / 4) * C::KSTR + ((w0 / 32) * 4 + (w0 % 4)) * 2;
#pragma unroll
    for (int c = 0; c < C::KMW / 2; ++c)
      *reinterpret_cast<float4*>(dst + 4 * c) = make_float4(kv[4 * c], kv[4 * c + 1], kv[4 * c + 2], kv[4 * c + 3]);
  }
  // word w = VMW * lane + k: gid w / (D/8), rho = w % (D/8)
  {
    const int w0 = C::VMW * lane;
    float* dst = vs + (w0 / (D / 8)) * C::VSTR + (w0 % (D / 8)) * 2;
#pragma unroll
    for (int c = 0; c < C::VMW / 2; ++c)
      *reinterpret_cast<float4*>(dst + 4 * c) = make_float4(vv[4 * c], vv[4 * c + 1], vv[4 * c + 2], vv[4 * c + 3]);
  }
}

// q.K^T of one tile: raw scores acc[nb][i] (units sq, without the softmax
// scale) for token gid + 8 i and head 4 nb + tig.  One k32 MMA per (token
// half, group); its two term columns combine exactly in int32, and the
// group's scale/zero apply to that exact integer sum.
// The epilogue runs on row pairs (tokens gid + 16 mb, gid + 16 mb + 8):
// acc2[nb][mb] = (score of the first, score of the second).
template <int D, int G, int KB, int QT>
__device__ __forceinline__ void qk_tile(const uint8_t* rec, const WarpState<D, G, QT>& st, const float* ks,
                                        float2 (&acc)[Cfg<D, G>::NB][2], int lane) {
  using C = Cfg<D, G>;
  constexpr int W = words_per_lane(KB, D);
  const int gid = lane >> 2;
  uint32_t kw[W];
  load_words<W>(kw, rec, lane);
#pragma unroll
  for (int nb = 0; nb < C::NB; ++nb)
#pragma unroll
    for (int mb = 0; mb < 2; ++mb) acc[nb][mb] = make_float2(0.0f, 0.0f);
#pragma unroll
  for (int g = 0; g < C::NG; ++g)
#pragma unroll
    for (int mb = 0; mb < 2; ++mb) {
      const float4 sz = *reinterpret_cast<const float4*>(ks + gid * C::KSTR + (g * 4 + 2 * mb) * 2);
      uint32_t a[4];
#pragma unroll
      for (int r = 0; r < 4; ++r) a[r] = code_reg<KB, W>(kw, (2 * mb + (r & 1)) * C::NG + g, r >> 1);
#pragma unroll
      for (int nb = 0; nb < C::NB; ++nb) {
        uint32_t c[4];
        float2 v;
        if constexpr (QT == 3) {
          // terms 1, 2 in one MMA, term 3 in another: 65536 t1 + (256 t2 + t3),
          // the bracket exact in int32, two roundings in fp32
          uint32_t c3[4];
          imma_u8s8(c, a, st.qb[nb][g][0], st.qb[nb][g][1], 0u);
          imma_u8s8(c3, a, st.qb3[nb][g][0], st.qb3[nb][g][1], 0u);
          v = make_float2(fmaf(65536.0f, (float)(int)c[0], (float)((int)c[1] * 256 + (int)c3[0])),
                          fmaf(65536.0f, (float)(int)c[2], (float)((int)c[3] * 256 + (int)c3[2])));
        } else {
          imma_u8s8(c, a, st.qb[nb][g][0], st.qb[nb][g][1], 0u);
          v = combine_terms(c);
        }
        acc[nb][mb] = ffma2(make_float2(sz.x, sz.y), v, ffma2(make_float2(sz.z, sz.w), st.qz[nb][g], acc[nb][mb]));
      }
    }
}

// Online softmax of one tile.  The probabilities are taken relative to the
// running maximum m (p <= 1, 16-bit fixed point p_int = rint(65535 p)); m
// moves -- and the state is rescaled -- only when a score of the tile exceeds
// it, which after the first tiles is rare.  Returns the P B-fragments pb
// (column n = 2 * head + term, term 0 = high byte).
template <int D, int G, int QT>
__device__ __forceinline__ void softmax_tile(WarpState<D, G, QT>& st, const float2 (&acc)[Cfg<D, G>::NB][2],
                                             uint32_t (&pb)[Cfg<D, G>::NB][2], int lane) {
  using C = Cfg<D, G>;
  const int gid = lane >> 2, tig = lane & 3;
  // x[nb][i]: token gid + 8 i (acc pairs hold tokens (gid + 16 mb, gid + 16 mb + 8))
  float x[C::NB][4];
  bool grow = false;
#pragma unroll
  for (int nb = 0; nb < C::NB; ++nb) {
    const float2 xs2 = make_float2(st.xs[nb], st.xs[nb]);
#pragma unroll
    for (int mb = 0; mb < 2; ++mb) {
      const float2 y = fmul2(acc[nb][mb], xs2);
      x[nb][2 * mb] = y.x;
      x[nb][2 * mb + 1] = y.y;
    }
    grow |= fmaxf(fmaxf(x[nb][0], x[nb][1]), fmaxf(x[nb][2], x[nb][3])) > st.m[nb];
  }
  if (__any_sync(0xffffffffu, grow)) {
#pragma unroll
    for (int nb = 0; nb < C::NB; ++nb) {
      float v = fmaxf(fmaxf(x[nb][0], x[nb][1]), fmaxf(x[nb][2], x[nb][3]));
      v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 4));
      v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 8));
      v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 16));
      const float mn = fmaxf(st.m[nb], v);
      const float alpha = ex2(st.m[nb] - mn);  // 0 while m = -inf
      st.m[nb] = mn;
      st.l[nb] *= alpha;
      const float2 a2 = make_float2(alpha, alpha);
#pragma unroll
      for (int mb = 0; mb < D / 16; ++mb) st.o[nb][mb] = fmul2(st.o[nb][mb], a2);
    }
  }
  const int hl = gid >> 1;
  const int src0 = 4 * tig + hl, src1 = 16 + 4 * tig + hl;
#pragma unroll
  for (int nb = 0; nb < C::NB; ++nb) {
    uint32_t y[4];
    const float2 m2 = make_float2(st.m[nb], st.m[nb]);
#pragma unroll
    for (int i = 0; i < 4; i += 2) {
      const float2 d = fadd2(make_float2(x[nb][i], x[nb][i + 1]), make_float2(-m2.x, -m2.y));
      const float2 p = ffma2(make_float2(ex2(d.x), ex2(d.y)), make_float2(kPScale, kPScale), make_float2(kBias, kBias));
      y[i] = __float_as_uint(p.x);
      y[i + 1] = __float_as_uint(p.y);
    }
    // low 16 bits of y = p_int; byte e of hi/lo = token gid + 8e
    const uint32_t u0 = __byte_perm(y[0], y[1], 0x5410), u1 = __byte_perm(y[2], y[3], 0x5410);
    const uint32_t hi = __byte_perm(u0, u1, 0x7531), lo = __byte_perm(u0, u1, 0x6420);
    // B element (k, n = gid): token 4 (k >> 4) + ((k >> 2) & 3) + 8 (k & 3),
    // held by lane 4 * gid_src + head with gid_src = tig (k < 16) or tig + 4
    const uint32_t h0 = __shfl_sync(0xffffffffu, hi, src0), l0 = __shfl_sync(0xffffffffu, lo, src0);
    const uint32_t h1 = __shfl_sync(0xffffffffu, hi, src1), l1 = __shfl_sync(0xffffffffu, lo, src1);
    const bool hv = hl < C::HB;
    pb[nb][0] = hv ? ((gid & 1) ? l0 : h0) : 0u;
    pb[nb][1] = hv ? ((gid & 1) ? l1 : h1) : 0u;
  }
}

// P.V of one tile into the running state.  One k32 MMA per 16 channels; the
// channel's scale/zero apply to the exact integer sum, and the zero term
// needs sum_t p_t, which one more MMA with A = 1 delivers in the same layout.
template <int D, int G, int VB, int QT>
__device__ __forceinline__ void pv_tile(const uint8_t* vrec, WarpState<D, G, QT>& st, const float* vs,
                                        const uint32_t (&pb)[Cfg<D, G>::NB][2], int lane) {
  using C = Cfg<D, G>;
  constexpr int W = words_per_lane(VB, D);
  const int gid = lane >> 2;
  float2 ps[C::NB];
  const uint32_t ones[4] = {0x01010101u, 0x01010101u, 0x01010101u, 0x01010101u};
#pragma unroll
  for (int nb = 0; nb < C::NB; ++nb) {
    uint32_t c[4];
    imma_u8u8(c, ones, pb[nb][0], pb[nb][1], kBiasBits);
    const float p = fmaf(256.0f, __uint_as_float(c[0]) - kBias, __uint_as_float(c[1]) - kBias);
    ps[nb] = make_float2(p, p);
    st.l[nb] += p;
  }
  uint32_t vw[W];
  load_words<W>(vw, vrec, lane);
#pragma unroll
  for (int mb = 0; mb < D / 16; ++mb) {
    const float4 sz = *reinterpret_cast<const float4*>(vs + gid * C::VSTR + 4 * mb);
    uint32_t a[4];
#pragma unroll
    for (int r = 0; r < 4; ++r) a[r] = code_reg<VB, W>(vw, 2 * mb + (r & 1), r >> 1);
#pragma unroll
    for (int nb = 0; nb < C::NB; ++nb) {
      uint32_t c[4];
      imma_u8u8(c, a, pb[nb][0], pb[nb][1], 0u);
      const float2 v = combine_terms(c);
      st.o[nb][mb] = ffma2(make_float2(sz.x, sz.y), v, ffma2(make_float2(sz.z, sz.w), ps[nb], st.o[nb][mb]));
    }
  }
}

__device__ __forceinline__ void raise_abort(volatile int* abort_flag, int* status) {
  *abort_flag = 1;
  atomicCAS(status, 0, kDeviceTimeout);
}

// Consumer warp w owns tiles w, w + NW, w + 2 NW, ... of the CTA's range and a
// private ring of `stages` shared-memory slots.  Lane 0 streams the warp's
// own tile records into the ring with 1-D bulk copies (TMA) and re-arms a
// slot as soon as the warp has read it, so the warp never waits on another
// warp and every warp keeps `stages` records in flight.
template <int D, int G, int KB, int VB, int QT>
__device__ void consume(WarpState<D, G, QT>& st, const uint16_t* qh, const float* nrm, float scale_log2, uint8_t* ring,
                        int stages,
                        int stage_bytes, uint64_t* bars, float* scratch, const uint8_t* src, int rec, int n_my,
                        int warp, int lane, volatile int* abort_flag, int* status) {
  using C = Cfg<D, G>;
  const int n_w = n_my > warp ? (n_my - warp + NW - 1) / NW : 0;
  // Packed tiles are written only by kernels that complete before a decode
  // launch may start (prefill, tile flush), never by the decode launch this
  // one may overlap, so the first records can be fetched before waiting on
  // it; the query, the window and the workspace are read after the wait.
  const uint64_t policy = l2_evict_first_policy();  // tile records are read once per launch
  if (lane == 0) {
    for (int j = 0; j < stages && j < n_w; ++j) {
      mbar_arrive_expect_tx(&bars[j], (uint32_t)rec);
      bulk_g2s_hint(ring + (size_t)j * stage_bytes, src + (int64_t)(warp + j * NW) * rec, (uint32_t)rec, &bars[j],
                    policy);
    }
  }
  griddep_wait();  // every earlier kernel of the stream has completed and its writes are visible
  setup_query<D, G, KB, VB, QT>(st, qh, nrm, scale_log2, lane);
  float* ks = scratch;
  float* vs = scratch + 8 * C::KSTR;
  const int VOFF = blob_bytes(KB, D) + 4 * D;
  int j = 0, slot = 0, parity = 0;  // ring position of tile j, advanced without division
  uint8_t* cur = ring;               // slot address of tile j
  const uint8_t* nsrc = src + (int64_t)(warp + stages * NW) * rec;  // record of tile j + stages
  bool ok = true;
  for (; j < n_w; ++j) {
    ok = __all_sync(0xffffffffu, mbar_wait_bounded(&bars[slot], (uint32_t)parity));
    if (!ok) break;
    convert_meta<D, G, KB, VB, QT>(cur, st, ks, vs, lane);
    __syncwarp();
    float2 acc[C::NB][2];
    qk_tile<D, G, KB, QT>(cur, st, ks, acc, lane);
    uint32_t pb[C::NB][2];
    softmax_tile<D, G, QT>(st, acc, pb, lane);
    pv_tile<D, G, VB, QT>(cur + VOFF, st, vs, pb, lane);
    // every lane has read the slot (its values are consumed): lane 0 re-arms
    // it for tile j + stages, as a predicated copy rather than a branch.  The
    // slot is only ever read through the generic proxy, so the refill (async
    // proxy) needs no proxy fence, only this ordering after the reads.
    __syncwarp();
    bulk_g2s_hint_if(lane == 0 && j + stages < n_w, cur, nsrc, (uint32_t)rec, &bars[slot], policy);
    nsrc += (int64_t)NW * rec;
    cur += stage_bytes;
    if (++slot == stages) {
      slot = 0;
      parity ^= 1;
      cur = ring;
    }
    if ((j & 3) == 3 && *abort_flag) {  // another warp gave up: stop within four tiles
      ok = false;
      break;
    }
  }
  if (!ok) {
    if (lane == 0) {
      raise_abort(abort_flag, status);
      // let the copies in flight land before the CTA exits
      for (int k = j; k < n_w && k < j + stages; ++k) (void)mbar_wait_bounded(&bars[k % stages], (k / stages) & 1);
    }
  }
}

template <int D, int G, int QT>
__device__ __forceinline__ void consume_dispatch(int kb, int vb, WarpState<D, G, QT>& st, const uint16_t* qh,
                                                 const float* nrm, float scale_log2, uint8_t* ring, int stages, int stage_bytes,
                                                 uint64_t* bars, float* scratch, const uint8_t* src, int rec,
                                                 int n_my, int warp, int lane, volatile int* abort_flag,
                                                 int* status) {
#define RQ_C(KBV, VBV)                                                                                       \
  consume<D, G, KBV, VBV, QT>(st, qh, nrm, scale_log2, ring, stages, stage_bytes, bars, scratch, src, rec, n_my, warp, \
                          lane, abort_flag, status)
#define RQ_V(KBV)                  \
  switch (vb) {                    \
    case 2: RQ_C(KBV, 2); break;   \
    case 3: RQ_C(KBV, 3); break;   \
    case 4: RQ_C(KBV, 4); break;   \
    default: RQ_C(KBV, 8); break;  \
  }
  switch (kb) {
    case 2: RQ_V(2) break;
    case 3: RQ_V(3) break;
    case 4: RQ_V(4) break;
    default: RQ_V(8) break;
  }
#undef RQ_V
#undef RQ_C
}

// Canonical partial of one warp in shared memory: o[G][D], m[G], l[G], with
// o and l back in units of p (the tile path keeps them x 65535).
template <int D, int G, int QT>
__device__ void dump_tile_state(const WarpState<D, G, QT>& st, float* slot, int lane) {
  using C = Cfg<D, G>;
  const int gid = lane >> 2, tig = lane & 3;
  constexpr float inv = 1.0f / kPScale;
#pragma unroll
  for (int nb = 0; nb < C::NB; ++nb) {
    const int h = 4 * nb + tig;
    if (tig < C::HB) {
#pragma unroll
      for (int mb = 0; mb < D / 16; ++mb) {
        slot[h * D + 16 * mb + gid] = st.o[nb][mb].x * inv;
        slot[h * D + 16 * mb + 8 + gid] = st.o[nb][mb].y * inv;
      }
      if (gid == 0) {
        slot[G * D + h] = st.m[nb];
        slot[G * D + G + h] = st.l[nb] * inv;
      }
    }
  }
}

// bf16 sink + recent window on the tensor cores.  The window is split into
// chunks of 32 tokens, a.win_chunks consecutive chunks per work item.
// For each chunk lane 0 of warp 0 stages its K and V rows in shared memory
// with a few 1-D bulk copies of contiguous rows (measured faster than one
// copy per row into padded, bank-conflict-free rows: the TMA engine is shared
// with the tile streams, and its per-copy cost outweighs the ldmatrix bank
// conflicts of 256-byte rows); warp w then takes tokens 8 w .. 8 w + 7 of the
// chunk for all G heads:
//   scores (heads x 8 tokens) = q (A, bf16 from the caller's rows, heads in
//     rows 0..G-1) . K^T (B, ldmatrix of the K rows), m16n8k16, fp32;
//   o^T (channels x heads) += V^T (A, ldmatrix.trans of the V rows) . P (B,
//     straight from the score fragments), m16n8k8, with P split into two
//     bf16 terms p = p_hi + p_lo (relative error 2^-17 instead of bf16's
//     2^-9), so that the products are exact and only the fp32 accumulation
//     rounds.
// Each warp keeps its own online-softmax state over its tokens; the warps'
// states are merged like the tile path's.
constexpr int kWinChunk = 32;
__host__ __device__ constexpr int window_row_stride(int D) { return 2 * D; }
// shared memory of a window item: two buffers of one K and one V chunk
__host__ __device__ constexpr int window_smem_bytes(int D) { return 2 * 2 * kWinChunk * window_row_stride(D); }

__host__ __device__ inline int window_tokens(int T, int S, int Tq) { return (T < S ? T : S) + (T - (T < S ? T : S) - Tq); }

// Lane 0 of a warp: the K and V rows of window tokens j0 .. j0 + cnt - 1
// into kbuf / vbuf (row t at t * window_row_stride(D)), counted on bar, with
// one bulk copy per contiguous run of rows (at most three: sink, ring, ring
// after its wrap) and one for the newest token of a fused append.
template <int D>
__device__ __forceinline__ void window_issue_chunk(const DecodeArgs& a, const uint8_t* win, uint8_t* kbuf,
                                                   uint8_t* vbuf, uint64_t* bar, int j0, int cnt,
                                                   const uint16_t* knew, const uint16_t* vnew, int lane) {
  constexpr int RB = 2 * D;
  if (lane != 0) return;
  const int S = a.g.S, ring = a.g.R + kTile;
  const int n_sink = a.T < S ? a.T : S;
  mbar_arrive_expect_tx(bar, (uint32_t)(cnt * RB * 2));
  const int n_cache = knew ? cnt - 1 : cnt;
  if (knew) {
    bulk_g2s(kbuf + (size_t)n_cache * RB, knew, (uint32_t)RB, bar);
    bulk_g2s(vbuf + (size_t)n_cache * RB, vnew, (uint32_t)RB, bar);
  }
  int t = 0;
  while (t < n_cache) {
    const int j = j0 + t;
    size_t row, v_off;
    int run;
    if (j < n_sink) {
      row = j;
      run = min(n_cache - t, n_sink - j);
      v_off = S;
    } else {
      const int slot = (a.Tq + (j - n_sink)) % ring;
      row = (size_t)2 * S + slot;
      run = min(n_cache - t, ring - slot);
      v_off = ring;
    }
    bulk_g2s(kbuf + (size_t)t * RB, win + row * RB, (uint32_t)(run * RB), bar);
    bulk_g2s(vbuf + (size_t)t * RB, win + (row + v_off) * RB, (uint32_t)(run * RB), bar);
    t += run;
  }
}

// L2 prefetch of the cache rows (K and V) of window tokens [j0, j1), by one
// thread: at most three contiguous runs (sink, ring, ring after its wrap).
// Issued before the wait on the previous kernel: a row that kernel still
// writes is updated in L2, which the later copies read.
template <int D>
__device__ void window_prefetch_l2(const DecodeArgs& a, const uint8_t* win, int j0, int j1) {
  constexpr int RB = 2 * D;
  const int S = a.g.S, ring = a.g.R + kTile;
  const int n_sink = a.T < S ? a.T : S;
  for (int j = j0; j < j1;) {
    size_t row, v_off;
    int run;
    if (j < n_sink) {
      row = j;
      run = min(j1, n_sink) - j;
      v_off = S;
    } else {
      const int slot = (a.Tq + (j - n_sink)) % ring;
      row = (size_t)2 * S + slot;
      run = min(j1 - j, ring - slot);
      v_off = ring;
    }
    l2_prefetch(win + row * RB, (uint32_t)(run * RB));
    l2_prefetch(win + (row + v_off) * RB, (uint32_t)(run * RB));
    j += run;
  }
}

template <int D, int G>
__device__ void window_item(const DecodeArgs& a, uint8_t* win, const uint16_t* qh, size_t knew_off, int witem,
                            uint8_t* scratch, uint64_t* bar, float* slot, int warp, int lane,
                            volatile int* abort_flag) {
  constexpr int RB = 2 * D, RS = window_row_stride(D);
  constexpr int KS = D / 16;  // k16 steps of q.K^T, m16 tiles of o^T
  const int tid = warp * 32 + lane, gid = lane >> 2, tig = lane & 3;
  const int n_tok = window_tokens(a.T, a.g.S, a.Tq);
  const int n_chunks = (n_tok + kWinChunk - 1) / kWinChunk;
  const int c0 = witem * a.win_chunks;
  const int c1 = min(c0 + a.win_chunks, n_chunks);
  constexpr int kBufBytes = 2 * kWinChunk * RS;  // one K and one V chunk
  // chunk c0 + k lands in buffer k % 2 on bar[k % 2]; the copy of the chunk
  // after next starts as soon as every warp has read a buffer
  auto issue = [&](int ch) {  // warp 0
    const int j0 = ch * kWinChunk;
    const int cnt = min(kWinChunk, n_tok - j0);
    const bool newest = a.k_new != nullptr && j0 + cnt == n_tok;
    const int bi = (ch - c0) & 1;
    uint8_t* kb = scratch + bi * kBufBytes;
    window_issue_chunk<D>(a, win, kb, kb + kWinChunk * RS, bar + bi, j0, cnt, newest ? a.k_new + knew_off : nullptr,
                          newest ? a.v_new + knew_off : nullptr, lane);
  };
  // (an item past the window's last chunk -- a padding item of a cluster --
  // issues nothing and leaves empty partial states).  The buffers overlap the
  // warp slots, which are written after the last chunk.
  if (warp == 0 && c0 < c1) {
    issue(c0);
    if (c0 + 1 < c1) issue(c0 + 1);
  }
  // q of head gid: bf16 A fragments (rows gid + 8 are empty), re-read from
  // L1 for every chunk rather than held in registers
  const uint32_t* qrow = reinterpret_cast<const uint32_t*>(qh + (gid < G ? gid : 0) * D) + tig;
  // running state: m, l of head gid (l summed over the quad at the end);
  // o[mt]: channels 16 mt + gid (+ 8) x heads 2 tig, 2 tig + 1
  float m = -INFINITY, l = 0.0f;
  float o[KS][4];
#pragma unroll
  for (int mt = 0; mt < KS; ++mt) o[mt][0] = o[mt][1] = o[mt][2] = o[mt][3] = 0.0f;
  const int n0 = 8 * warp;  // this warp's tokens in every chunk
  for (int ch = c0; ch < c1; ++ch) {
    const int j0 = ch * kWinChunk;
    const int cnt = min(kWinChunk, n_tok - j0);
    // a fused append delivers the newest token (window index n_tok - 1) itself
    const bool newest = a.k_new != nullptr && j0 + cnt == n_tok;
    const int bi = (ch - c0) & 1;
    const uint32_t parity = ((ch - c0) >> 1) & 1;
    uint8_t* kbuf = scratch + bi * kBufBytes;
    uint8_t* vbuf = kbuf + kWinChunk * RS;
    const bool ok = __all_sync(0xffffffffu, mbar_wait_bounded(bar + bi, parity));
    if (!__syncthreads_and(ok)) {
      if (tid == 0) {
        raise_abort(abort_flag, a.status);
        // let the copies in flight (this chunk and the next) land before the CTA exits
        (void)mbar_wait_bounded(bar + bi, parity);
        if (ch + 1 < c1) (void)mbar_wait_bounded(bar + (bi ^ 1), ((ch + 1 - c0) >> 1) & 1);
      }
      return;
    }
    if (newest && tid < 2 * (D / 8)) {
      // the appended token enters the cache (sink row, or its ring slot) for
      // later calls; no other work item of this call reads that row
      const int S = a.g.S, ring = a.g.R + kTile;
      const int n_sink = a.T < S ? a.T : S;
      const int j = n_tok - 1;
      size_t krow, vrow;
      if (j < n_sink) {
        krow = j;
        vrow = (size_t)S + j;
      } else {
        const int rs = (a.Tq + (j - n_sink)) % ring;
        krow = (size_t)2 * S + rs;
        vrow = (size_t)2 * S + ring + rs;
      }
      const int c = tid % (D / 8);
      const bool isv = tid >= D / 8;
      const uint4 x = reinterpret_cast<const uint4*>((isv ? vbuf : kbuf) + (size_t)(cnt - 1) * RS)[c];
      reinterpret_cast<uint4*>(win + (isv ? vrow : krow) * RB)[c] = x;
    }
    if (n0 < cnt) {  // warp-uniform
      if (n0 + 8 > cnt) {
        // rows past the window's end hold stale bytes: P is 0 there, but
        // 0 * NaN is not, so their V rows are zeroed first (this is the
        // window's last chunk: no later copy lands in this buffer)
        for (int i = lane; i < (n0 + 8 - cnt) * (RB / 16); i += 32) {
          const int t = cnt + i / (RB / 16);
          reinterpret_cast<uint4*>(vbuf + (size_t)t * RS)[i % (RB / 16)] = make_uint4(0u, 0u, 0u, 0u);
        }
        __syncwarp();
      }
      // scores: head gid (row) x tokens n0 + 2 tig, + 1 (columns), in two
      // accumulators over even and odd k-steps
      float s[2][4] = {{0.0f, 0.0f, 0.0f, 0.0f}, {0.0f, 0.0f, 0.0f, 0.0f}};
      const uint32_t krow = smem_u32(kbuf) + (n0 + (lane & 7)) * RS + (lane >> 3) * 16;
#pragma unroll 1
      for (int p = 0; p < KS / 2; ++p) {
        uint32_t b[4], qa[4];
        ldsm_x4(b, krow + p * 64);  // channels 32 p .. 32 p + 31: k-steps 2 p, 2 p + 1
#pragma unroll
        for (int i = 0; i < 4; ++i) qa[i] = gid < G ? __ldg(qrow + 16 * p + 4 * i) : 0u;
        mma_bf16_k16(s[0], qa[0], 0u, qa[1], 0u, b[0], b[1]);
        mma_bf16_k16(s[1], qa[2], 0u, qa[3], 0u, b[2], b[3]);
      }
      const int t0 = n0 + 2 * tig;
      const float x0 = t0 < cnt ? (s[0][0] + s[1][0]) * a.scale_log2 : -INFINITY;
      const float x1 = t0 + 1 < cnt ? (s[0][1] + s[1][1]) * a.scale_log2 : -INFINITY;
      float cm = fmaxf(x0, x1);  // token n0 is valid: finite after the quad max
      cm = fmaxf(cm, __shfl_xor_sync(0xffffffffu, cm, 1));
      cm = fmaxf(cm, __shfl_xor_sync(0xffffffffu, cm, 2));
      const float mn = fmaxf(m, cm);
      const float alpha = ex2(m - mn);  // 0 while m = -inf
      m = mn;
      const float p0 = ex2(x0 - mn), p1 = ex2(x1 - mn);
      l = fmaf(l, alpha, p0 + p1);
      // o columns are heads 2 tig, 2 tig + 1, whose state lives in lanes 8 tig, 8 tig + 4
      const float a0 = __shfl_sync(0xffffffffu, alpha, 8 * tig), a1 = __shfl_sync(0xffffffffu, alpha, 8 * tig + 4);
#pragma unroll
      for (int mt = 0; mt < KS; ++mt) {
        o[mt][0] *= a0;
        o[mt][1] *= a1;
        o[mt][2] *= a0;
        o[mt][3] *= a1;
      }
      // B fragment of P (tokens 2 tig, 2 tig + 1 of head gid) in two bf16 terms
      const uint32_t ph = pack_bf16x2(p0, p1);
      const uint32_t pl = pack_bf16x2(p0 - bf16_bits_to_float(ph & 0xFFFFu), p1 - bf16_bits_to_float(ph >> 16));
      const uint32_t vrow = smem_u32(vbuf) + (n0 + (lane & 7)) * RS + (lane >> 3) * 16;
#pragma unroll
      for (int p = 0; p < KS / 2; ++p) {
        uint32_t v[4];
        ldsm_x4_trans(v, vrow + p * 64);  // channels 32 p .. 32 p + 31: m-tiles 2 p, 2 p + 1
        mma_bf16_k8(o[2 * p], v[0], v[1], ph);
        mma_bf16_k8(o[2 * p + 1], v[2], v[3], ph);
        mma_bf16_k8(o[2 * p], v[0], v[1], pl);
        mma_bf16_k8(o[2 * p + 1], v[2], v[3], pl);
      }
    }
    if (ch + 2 < c1) {
      __syncthreads();  // every warp has finished reading this buffer
      if (warp == 0) {
        fence_proxy_async_smem();
        issue(ch + 2);
      }
    }
  }
  l += __shfl_xor_sync(0xffffffffu, l, 1);
  l += __shfl_xor_sync(0xffffffffu, l, 2);
  __syncthreads();  // every warp has read the chunk buffers, which the warp slots overlap
  // this warp's partial state of all G heads (m = -inf, l = 0, o = 0 when it
  // saw no token)
#pragma unroll
  for (int e = 0; e < 2; ++e) {
    const int h = 2 * tig + e;
    if (h < G) {
#pragma unroll
      for (int mt = 0; mt < KS; ++mt) {
        slot[h * D + 16 * mt + gid] = o[mt][e];
        slot[h * D + 16 * mt + 8 + gid] = o[mt][2 + e];
      }
    }
  }
  if (tig == 0 && gid < G) {
    slot[G * D + gid] = m;
    slot[G * D + G + gid] = l;
  }
}

// Pack-ahead item (a fused step whose next append completes a tile): the 32
// oldest ring tokens -- exactly the tile that append will flush -- are
// quantized and packed into tile slot a.pack_tile, which no item of this
// launch reads, so the next step needs no separate flush launch.  The rows
// it reads are not the one this launch's window item writes (n_recent >= 2).
// Warp 0 packs K, warp 1 V.  Leaves empty partial states in the warp slots.
template <int D, int G>
__device__ void pack_item(const DecodeArgs& a, const HeadDesc& hd, int b, uint8_t* area, float* merge, int tid) {
  using C = Cfg<D, G>;
  const int warp = tid >> 5, lane = tid & 31;
  TileSmem<D>& sm = *reinterpret_cast<TileSmem<D>*>(area);
  uint8_t* win = a.buf + hd.win_base + (int64_t)b * a.g.win_bytes;
  const int S = a.g.S, ring = a.g.R + kTile;
  griddep_wait();
  if (warp == 0) stage_kinv<D>(sm.kinv, stream_norm(a.buf, hd, a.g, b), lane);
  constexpr int kChunks = D / 8;
  for (int j = tid; j < kTile * kChunks; j += blockDim.x) {
    const int t = j / kChunks, c = j % kChunks;
    const int slot = (a.pack_pos + t - S) % ring;
    const uint4* krow = reinterpret_cast<const uint4*>(win + ((size_t)2 * S + slot) * D * 2);
    const uint4* vrow = reinterpret_cast<const uint4*>(win + ((size_t)2 * S + ring + slot) * D * 2);
    *reinterpret_cast<uint4*>(&sm.k.x[t][c * 4]) = __ldg(krow + c);
    *reinterpret_cast<uint4*>(&sm.v.x[t][c * 4]) = __ldg(vrow + c);
  }
  __syncthreads();
  uint8_t* rec = a.buf + hd.tile_base + (int64_t)b * hd.tile_stride + (int64_t)a.pack_tile * hd.rec_bytes;
  if (warp == 0) {
    pack_k_dispatch<D, true>(sm.k, sm.kinv, hd.k_bits, rec, lane, a.g.hybrid);
  } else if (warp == 1) {
    pack_v_dispatch<D>(sm.v, hd.v_bits, rec + blob_bytes(hd.k_bits, D) + 4 * D, lane, a.g.hybrid);
  }
  __syncthreads();  // the staged tile is dead; its memory becomes the warp slots
  float* slot = merge + warp * C::PART;
  for (int i = lane; i < G * D; i += 32) slot[i] = 0.0f;
  if (lane < G) {
    slot[G * D + lane] = -INFINITY;
    slot[G * D + G + lane] = 0.0f;
  }
}

// Final log-sum-exp merge of n partial states (o[G][D], m[G], l[G] each,
// stride PART floats) into the normalised output, for the slice of outputs
// owned by cluster rank `part` (of CL): one output per thread, all of its loads for
// up to 24 partials in flight at once (a stream of the long-context cache has
// 17 cluster partials, so one round trip to L2 covers them).
template <int D, int G, int CL>
__device__ void merge_outputs(const float* base, int n, float* outp, int part, int tid) {
  using C = Cfg<D, G>;
  constexpr int PER = (G * D + CL - 1) / CL;  // outputs of one CTA
  constexpr int U = 24;
  for (int idx = part * PER + tid; idx < (part + 1) * PER && idx < G * D; idx += kDecodeThreads) {
    const int hh = idx / D;
    float M = -INFINITY, O = 0.0f, L = 0.0f;
    for (int i0 = 0; i0 < n; i0 += U) {
      float ov[U], mv[U], lv[U];
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const bool ok = i0 + u < n;
        const float* pp = base + (size_t)(i0 + u) * C::PART;
        ov[u] = ok ? __ldcg(pp + idx) : 0.0f;
        mv[u] = ok ? __ldcg(pp + G * D + hh) : -INFINITY;
        lv[u] = ok ? __ldcg(pp + G * D + G + hh) : 0.0f;
      }
      float nm = M;
#pragma unroll
      for (int u = 0; u < U; ++u) nm = fmaxf(nm, mv[u]);
      if (nm == -INFINITY) continue;
      const float sc = ex2(M - nm);  // 0 while M = -inf
      O *= sc;
      L *= sc;
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const float f = ex2(mv[u] - nm);
        O = fmaf(ov[u], f, O);
        L = fmaf(lv[u], f, L);
      }
      M = nm;
    }
    outp[idx] = L > 0.0f ? O / L : 0.0f;
  }
}

// Merge of n partial states (stride PART floats) with four consecutive
// outputs of one head per thread and the loads of up to U partials in flight:
// into one more partial state at dst (outp null), or into the normalised
// outputs at outp.
template <int D, int G, int U>
__device__ void merge_quads(const float* base, int n, float* dst, float* outp, int tid) {
  using C = Cfg<D, G>;
  for (int qd = tid; qd < G * D / 4; qd += kDecodeThreads) {
    const int idx = 4 * qd, hh = idx / D;
    float M = -INFINITY, L = 0.0f;
    float4 O = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
    for (int i0 = 0; i0 < n; i0 += U) {
      float4 ov[U];
      float mv[U], lv[U];
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const bool ok = i0 + u < n;
        const float* pp = base + (size_t)(i0 + u) * C::PART;
        ov[u] = ok ? __ldcg(reinterpret_cast<const float4*>(pp + idx)) : make_float4(0.0f, 0.0f, 0.0f, 0.0f);
        mv[u] = ok ? __ldcg(pp + G * D + hh) : -INFINITY;
        lv[u] = ok ? __ldcg(pp + G * D + G + hh) : 0.0f;
      }
      float nm = M;
#pragma unroll
      for (int u = 0; u < U; ++u) nm = fmaxf(nm, mv[u]);
      if (nm == -INFINITY) continue;
      const float sc = ex2(M - nm);  // 0 while M = -inf
      O.x *= sc, O.y *= sc, O.z *= sc, O.w *= sc;
      L *= sc;
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const float f = ex2(mv[u] - nm);
        O.x = fmaf(ov[u].x, f, O.x), O.y = fmaf(ov[u].y, f, O.y);
        O.z = fmaf(ov[u].z, f, O.z), O.w = fmaf(ov[u].w, f, O.w);
        L = fmaf(lv[u], f, L);
      }
      M = nm;
    }
    if (outp != nullptr) {
      const bool any = L > 0.0f;
      *reinterpret_cast<float4*>(outp + idx) =
          make_float4(any ? O.x / L : 0.0f, any ? O.y / L : 0.0f, any ? O.z / L : 0.0f, any ? O.w / L : 0.0f);
    } else {
      *reinterpret_cast<float4*>(dst + idx) = O;
      if (idx % D == 0) {
        dst[G * D + hh] = M;
        dst[G * D + G + hh] = L;
      }
    }
  }
}

// Tile work item: the warps stream and process their tiles, then (after every
// stage read has completed, so the merge area may alias the stages) leave
// their partial states in the warp slots.
template <int D, int G, int QT>
__device__ __forceinline__ void tile_item(const DecodeArgs& a, const HeadDesc& hd, const uint16_t* qh,
                                          const float* nrm, uint8_t* area, uint8_t* smem, float* merge,
                                          uint64_t* bars, const uint8_t* src, int rec, int n_my, int warp, int lane,
                                          volatile int* abort_flag) {
  using C = Cfg<D, G>;
  WarpState<D, G, QT> st;
  consume_dispatch<D, G, QT>(hd.k_bits, hd.v_bits, st, qh, nrm, a.scale_log2,
                             area + (size_t)warp * a.stages * a.stage_bytes, a.stages, a.stage_bytes,
                             bars + warp * kMaxStages, reinterpret_cast<float*>(smem) + warp * C::SCRATCH, src, rec,
                             n_my, warp, lane, abort_flag, a.status);
  __syncthreads();
  if (!*abort_flag) dump_tile_state<D, G, QT>(st, merge + warp * C::PART, lane);
}

// CL = CTAs per thread-block cluster (kDecodeCluster, or 1: no cluster); the
// cluster shape is given at launch.
// QT: s8 terms of the fixed-point query (2, or 3 for K-normalized caches); a
// separate instantiation so that the 16-bit path keeps its register budget.
template <int D, int G, int CL, int QT>
__global__ void __launch_bounds__(kDecodeThreads, QT == 3 ? 3 : RQ_DECODE_MIN_BLOCKS) decode_kernel(DecodeArgs a) {
  using C = Cfg<D, G>;
  extern __shared__ __align__(128) uint8_t smem[];
  __shared__ uint64_t bars[NW * kMaxStages];
  __shared__ volatile int abort_flag;
  __shared__ int is_last;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int srel = blockIdx.y, item = blockIdx.x;
  const int NI = a.n_splits + a.n_win + a.n_pack;  // work items of this stream
  const int h = srel % a.g.Hkv, b = (srel / a.g.Hkv) % a.g.B, lrel = srel / (a.g.Hkv * a.g.B);
  const int l = a.layer0 + lrel;
  const HeadDesc hd = a.desc[l * a.g.Hkv + h];
  const uint16_t* qh = a.q + ((size_t)(lrel * a.g.B + b) * a.g.Hq + (size_t)h * G) * D;
  // dynamic shared memory: [per-warp scale scratch][stages | merge + window]
  uint8_t* area = smem + (size_t)NW * C::SCRATCH * 4;
  float* merge = reinterpret_cast<float*>(area);  // aliases the stages after the main loop

  // programmatic dependent launch: the next kernel of the stream may be
  // scheduled now; it waits below for this grid's memory before reading any
  // input, so only its launch and prologue overlap our tail
  griddep_launch_dependents();
  if (tid == 0) {
    abort_flag = 0;
    for (int s = 0; s < NW * kMaxStages; ++s) mbar_init(&bars[s], 1);
    mbar_fence_init();
  }
  __syncthreads();

  const bool tiles_item = item < a.n_splits;
  if (tiles_item) {
    const int t0 = (int)(((int64_t)item * a.n_tiles) / a.n_splits);
    const int t1 = (int)(((int64_t)(item + 1) * a.n_tiles) / a.n_splits);
    const int rec = hd.rec_bytes;
    const uint8_t* src = a.buf + hd.tile_base + (int64_t)b * hd.tile_stride + (int64_t)t0 * rec;
    const float* nrm = reinterpret_cast<const float*>(a.buf + hd.win_base + (int64_t)b * a.g.win_bytes +
                                                      window_rows_bytes(a.g.S, a.g.R, D));
    tile_item<D, G, QT>(a, hd, qh, nrm, area, smem, merge, bars, src, rec, t1 - t0, warp, lane, &abort_flag);
  } else if (a.n_pack && item == a.n_splits + a.n_win) {
    pack_item<D, G>(a, hd, b, area, merge, tid);
  } else {
    // 32-token chunks of the bf16 sink + recent window
    uint8_t* win = a.buf + hd.win_base + (int64_t)b * a.g.win_bytes;
    if (tid == 0) {
      const int n_tok = window_tokens(a.T, a.g.S, a.Tq);
      const int j0 = (item - a.n_splits) * a.win_chunks * kWinChunk;
      const int j1 = min(j0 + a.win_chunks * kWinChunk, n_tok);
      if (j0 < j1) window_prefetch_l2<D>(a, win, j0, j1);
    }
    griddep_wait();  // the window rows and the query may come from the previous kernel
    const size_t knew_off = ((size_t)(lrel * a.g.B + b) * a.g.Hkv + h) * D;
    // the chunk buffers start at the base of the dynamic shared memory (the
    // tile path's scale scratch is idle here) and end inside the merge area
    window_item<D, G>(a, win, qh, knew_off, item - a.n_splits, smem, &bars[0], merge + warp * C::PART, warp, lane,
                      &abort_flag);
  }
  __syncthreads();
  const bool valid = !abort_flag;

  // merge the warps' partial states into this item's partial (shared memory)
  float* mypart = merge + NW * C::PART;
  for (int idx = tid; idx < G * D; idx += blockDim.x) {
    const int hh = idx / D;
    float M = -INFINITY;
    if (valid) {
#pragma unroll
      for (int w = 0; w < NW; ++w) M = fmaxf(M, merge[w * C::PART + G * D + hh]);
    }
    float O = 0.0f, L = 0.0f;
    if (M != -INFINITY) {
#pragma unroll
      for (int w = 0; w < NW; ++w) {
        const float f = ex2(merge[w * C::PART + G * D + hh] - M);
        O = fmaf(merge[w * C::PART + idx], f, O);
        L = fmaf(merge[w * C::PART + G * D + G + hh], f, L);
      }
    }
    mypart[idx] = O;
    if (idx % D == 0) {
      mypart[G * D + hh] = M;
      mypart[G * D + G + hh] = L;
    }
  }
  // Level 1: the CL items of a thread-block cluster (consecutive items of one
  // stream) are merged by the cluster's first CTA straight from the others'
  // shared memory (CL = 1: the CTA stores its own partial).  Every CTA passes
  // both cluster barriers on every path (no early exit before them).
  namespace cg = cooperative_groups;
  float* ps = a.partials + (size_t)srel * partial_slots(NI) * C::PART;
  const int ncl = (int)gridDim.x / CL;
  int crank = 0;
  if constexpr (CL > 1) {
    cg::cluster_group cluster = cg::this_cluster();
    crank = (int)cluster.block_rank();
    cluster.sync();  // all partials of the cluster are in shared memory
    if (crank == 0) {
      const float* rp[CL];
#pragma unroll
      for (int r = 0; r < CL; ++r) rp[r] = cluster.map_shared_rank(mypart, r);
      float* cp = ps + (size_t)(item / CL) * C::PART;
      for (int idx = tid; idx < G * D; idx += blockDim.x) {
        const int hh = idx / D;
        float mv[CL];
        float M = -INFINITY;
#pragma unroll
        for (int r = 0; r < CL; ++r) {
          mv[r] = rp[r][G * D + hh];
          M = fmaxf(M, mv[r]);
        }
        float O = 0.0f, L = 0.0f;
        if (M != -INFINITY) {
#pragma unroll
          for (int r = 0; r < CL; ++r) {
            const float f = ex2(mv[r] - M);
            O = fmaf(rp[r][idx], f, O);
            L = fmaf(rp[r][G * D + G + hh], f, L);
          }
        }
        cp[idx] = O;
        if (idx % D == 0) {
          cp[G * D + hh] = M;
          cp[G * D + G + hh] = L;
        }
      }
    }
  } else {
    __syncthreads();  // the item partial is complete in shared memory
    float* cp = ps + (size_t)item * C::PART;
    for (int idx = tid; idx < C::PART; idx += blockDim.x) cp[idx] = mypart[idx];
    const int ngr = merge_groups(NI);
    if (ngr > 0) {
      // two levels: the last item of each group of kMergeGroup merges the
      // group into partial slot NI + group; the last group merger merges the
      // group partials into the output
      const int grp = item / kMergeGroup;
      const int gsize = min(kMergeGroup, NI - grp * kMergeGroup);
      __syncthreads();
      if (tid == 0) {
        uint32_t* gc = &a.counters[(size_t)srel * kCountersPerStream + 1 + grp];
        const int last_g = count_acq_rel(gc) == (unsigned)(gsize - 1);
        if (last_g) *gc = 0u;  // every item of the group has counted: reset for the next call
        is_last = last_g;
      }
      __syncthreads();
      if (!is_last) return;
      merge_quads<D, G, kMergeGroup>(ps + (size_t)grp * kMergeGroup * C::PART, gsize, ps + (size_t)(NI + grp) * C::PART,
                                     nullptr, tid);
      __syncthreads();
      if (tid == 0) is_last = count_acq_rel(&a.counters[(size_t)srel * kCountersPerStream]) == (unsigned)(ngr - 1);
      __syncthreads();
      if (!is_last) return;
      float* outp = a.out + ((size_t)(lrel * a.g.B + b) * a.g.Hq + (size_t)h * G) * D;
      merge_quads<D, G, 12>(ps + (size_t)NI * C::PART, ngr, nullptr, outp, tid);
      if (tid == 0) a.counters[(size_t)srel * kCountersPerStream] = 0u;
      return;
    }
  }
  // the first CTA publishes the cluster partial and learns whether its
  // cluster is the stream's last; it tells every CTA of the cluster
  if (crank == 0) {
    __syncthreads();
    if (tid == 0) {
      const int last = count_acq_rel(&a.counters[(size_t)srel * kCountersPerStream]) == (unsigned)(ncl - 1);
      if constexpr (CL > 1) {
        cg::cluster_group cluster = cg::this_cluster();
#pragma unroll
        for (int r = 0; r < CL; ++r) *cluster.map_shared_rank(&is_last, r) = last;
      } else {
        is_last = last;
      }
    }
  }
  if constexpr (CL > 1) {
    cg::this_cluster().sync();  // remote partial reads and the is_last stores are complete
  } else {
    __syncthreads();
  }
  if (!is_last) return;
  // Level 2: the CTAs of the last cluster merge the cluster partials, each a
  // slice of the outputs (CTAs other than the one that took the count
  // acquire the other clusters' partials with a fence of their own)
  if constexpr (CL > 1) __threadfence();
  float* outp = a.out + ((size_t)(lrel * a.g.B + b) * a.g.Hq + (size_t)h * G) * D;
  if constexpr (CL > 1) {
    merge_outputs<D, G, CL>(ps, ncl, outp, crank, tid);
  } else {
    merge_quads<D, G, kOneLevelItems>(ps, ncl, nullptr, outp, tid);
  }
  if (crank == 0 && tid == 0) a.counters[(size_t)srel * kCountersPerStream] = 0u;
}

// Host-side caches (per device) of the decode kernel's shared-memory
// attribute and of its resident capacity: both are fixed for a given
// (device, D, G, cluster, size), and querying them on every call costs more
// host time than a decode step.
std::mutex g_attr_mu;
std::map<std::tuple<int, int, int, int, int>, int> g_smem_set;       // (dev, D, G, CL, QT) -> largest size set
std::map<std::tuple<int, int, int, int, int, int>, int> g_resident;  // (dev, D, G, CL, QT, smem) -> CTAs

template <int D, int G, int CL, int QT>
cudaError_t ensure_smem(int smem) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  std::lock_guard<std::mutex> lock(g_attr_mu);
  int& cur = g_smem_set[std::make_tuple(dev, D, G, CL, QT)];
  if (cur >= smem) return cudaSuccess;
  e = cudaFuncSetAttribute(decode_kernel<D, G, CL, QT>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e == cudaSuccess) cur = smem;
  return e;
}

template <int D, int G, int CL, int QT>
cudaError_t launch_dgc(const DecodeArgs& a, int smem, cudaStream_t st) {
  cudaError_t e = ensure_smem<D, G, CL, QT>(smem);
  if (e != cudaSuccess) return e;
  const int streams = a.n_layers * a.g.B * a.g.Hkv;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(cluster_items(a.n_splits + a.n_win + a.n_pack, CL), streams, 1);
  cfg.blockDim = dim3(kDecodeThreads, 1, 1);
  cfg.dynamicSmemBytes = (size_t)smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = RQ_DECODE_PDL;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (CL > 1) {
    attr[1].id = cudaLaunchAttributeClusterDimension;
    attr[1].val.clusterDim.x = CL;
    attr[1].val.clusterDim.y = 1;
    attr[1].val.clusterDim.z = 1;
    cfg.numAttrs = 2;
  }
  e = cudaLaunchKernelEx(&cfg, decode_kernel<D, G, CL, QT>, a);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

template <int D, int G>
cudaError_t launch_dg(const DecodeArgs& a, int smem, cudaStream_t st) {
  const bool q3 = a.q_terms == 3;
  if (a.cluster == 1) return q3 ? launch_dgc<D, G, 1, 3>(a, smem, st) : launch_dgc<D, G, 1, 2>(a, smem, st);
  if (a.cluster == kDecodeCluster)
    return q3 ? launch_dgc<D, G, kDecodeCluster, 3>(a, smem, st) : launch_dgc<D, G, kDecodeCluster, 2>(a, smem, st);
  return cudaErrorInvalidValue;
}

// CTAs of the decode kernel that the device holds at once, in whole clusters.
template <int D, int G, int CL, int QT>
int resident_ctas_dgc(int smem) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return CL;
  {
    std::lock_guard<std::mutex> lock(g_attr_mu);
    auto it = g_resident.find(std::make_tuple(dev, D, G, CL, QT, smem));
    if (it != g_resident.end()) return it->second;
  }
  if (ensure_smem<D, G, CL, QT>(smem) != cudaSuccess) return CL;
  int n = 0;
  if (CL > 1) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(CL * 64, 1, 1);
    cfg.blockDim = dim3(kDecodeThreads, 1, 1);
    cfg.dynamicSmemBytes = (size_t)smem;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = CL;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaOccupancyMaxActiveClusters(&n, decode_kernel<D, G, CL, QT>, &cfg) != cudaSuccess || n < 1) return CL;
    n *= CL;
  } else {
    int per_sm = 0, sms = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, decode_kernel<D, G, CL, QT>, kDecodeThreads, smem) !=
            cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || per_sm < 1 || sms < 1)
      return 1;
    n = per_sm * sms;
  }
  std::lock_guard<std::mutex> lock(g_attr_mu);
  g_resident[std::make_tuple(dev, D, G, CL, QT, smem)] = n;
  return n;
}

template <int D, int G>
int resident_ctas_dg(int cluster, int smem, int q_terms) {
  if (q_terms == 3)
    return cluster == 1 ? resident_ctas_dgc<D, G, 1, 3>(smem) : resident_ctas_dgc<D, G, kDecodeCluster, 3>(smem);
  return cluster == 1 ? resident_ctas_dgc<D, G, 1, 2>(smem) : resident_ctas_dgc<D, G, kDecodeCluster, 2>(smem);
}

}  // namespace

// One (head_dim, GQA group) pair: launch and resident-CTA query (explicit
// specializations live in rq_decode_<D>x<G>.cu).
template <int D, int G>
cudaError_t launch_decode_dg(const DecodeArgs& a, int smem, cudaStream_t st);
template <int D, int G>
int decode_resident_ctas_dg(int cluster, int smem, int q_terms);

}  // namespace rq

#define RQ_DECODE_INSTANTIATE(DD, GG)                                                      \
  namespace rq {                                                                           \
  template <>                                                                              \
  cudaError_t launch_decode_dg<DD, GG>(const DecodeArgs& a, int smem, cudaStream_t st) {   \
    return launch_dg<DD, GG>(a, smem, st);                                                 \
  }                                                                                        \
  template <>                                                                              \
  int decode_resident_ctas_dg<DD, GG>(int cluster, int smem, int q_terms) {                \
    return resident_ctas_dg<DD, GG>(cluster, smem, q_terms);                               \
  }                                                                                        \
  }

// Quantize-and-pack of one 32-token tile (device code shared by the prefill,
// the append/flush and the decode kernels' pack-ahead item).
//
// InnerQ grouping ("InnerQ: Hardware-Aware Tuning-Free Quantization of KV
// Cache for Large Language Models", abstract / "Core claim"): K groups run
// along head_dim per token (32 channels), V groups along tokens per channel
// (the 32 tokens of a tile).  Asymmetric min/max quantization with an fp16
// scale and a bf16 zero; bit widths 2, 3, 4, 8 per (layer, kv-head).
//
// Every arithmetic step of the rounding rule is an IEEE fp32 operation with
// round-to-nearest-even (__fsub_rn, __fdiv_rn, __frcp_rn, __fmul_rn,
// __float2half_rn, __float2int_rn), so codes and scales are reproducible
// bit for bit on any IEEE machine.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "rq_device.cuh"
#include "rq_internal.h"

namespace rq {
namespace {

// One 32-token tile of K or V staged in shared memory (bf16 pairs, rows
// padded so that the lane-per-token and fragment-order reads hit distinct
// banks) and its group statistics: K -- 1/scale and zero per (token, group)
// at [t * D/32 + g]; V -- per channel at [d].
template <int D>
struct HalfTile {
  static constexpr int kStride = D / 2 + 4;  // words per staged row (16-byte aligned)
  uint32_t x[kTile][kStride];
  float r[D];
  float z[D];
};

// Append/flush: K and V tiles staged together (one warp packs each).
template <int D>
struct TileSmem {
  HalfTile<D> k, v;
  float kinv[D];  // 1 / n per channel (K normalization; powers of two)
};

// Stream's K normalization factors n[D] (fp32), stored after its window rows.
__device__ __forceinline__ float* stream_norm(uint8_t* buf, const HeadDesc& hd, const Geom& g, int b) {
  return reinterpret_cast<float*>(buf + hd.win_base + (int64_t)b * g.win_bytes + window_rows_bytes(g.S, g.R, g.D));
}

// 1 / n of the stream into shared memory (one warp).
template <int D>
__device__ __forceinline__ void stage_kinv(float* kinv, const float* nrm, int lane) {
  for (int d = lane; d < D; d += 32) kinv[d] = 1.0f / nrm[d];
}

__device__ __forceinline__ float lo_bf16(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float hi_bf16(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

// Hybrid option (InnerQ, technique (i): a symmetric or an asymmetric
// quantizer per group, chosen from the group's statistics; this library's
// rule): a group nearly centred on zero, |max + min| <= (max - min) / 8, is
// quantized on the symmetric interval [-M, M], M = max(|min|, |max|).
constexpr float kHybridTau = 0.125f;

// Scale/zero of one group from its min and max; returns the meta word and
// leaves in mn the zero the codes are taken from.  The extremes are real
// numbers: x + 0 turns a -0.0 extreme into +0.0, so the stored zero and scale
// do not depend on which of two equal zeros fminf / fmaxf returned.
template <int B>
__device__ __forceinline__ uint32_t group_params(float& mn, float mx, float& r, bool hybrid) {
  mn = __fadd_rn(mn, 0.0f);
  mx = __fadd_rn(mx, 0.0f);
  if (hybrid && fabsf(__fadd_rn(mx, mn)) <= __fmul_rn(__fsub_rn(mx, mn), kHybridTau)) {
    const float m = fmaxf(fabsf(mn), fabsf(mx));
    mn = __fadd_rn(-m, 0.0f);
    mx = m;
  }
  float s32 = __fdiv_rn(__fsub_rn(mx, mn), (float)((1 << B) - 1));
  s32 = fminf(s32, 65504.0f);
  const __half h = __float2half_rn(s32);
  const float s = __half2float(h);
  r = s > 0.0f ? __frcp_rn(s) : 0.0f;
  return (uint32_t)__half_as_ushort(h) | ((__float_as_uint(mn) >> 16) << 16);
}

template <int B>
__device__ __forceinline__ uint32_t code_of(float x, float z, float r) {
  int c = __float2int_rn(__fmul_rn(__fsub_rn(x, z), r));
  c = c < 0 ? 0 : c;
  c = c > (1 << B) - 1 ? (1 << B) - 1 : c;
  return (uint32_t)c;
}

// The same rule on two elements at once: c = min(rint((x - z) * r), 2^B - 1)
// with x - z and the product each one fp32 operation rounded to nearest
// (packed pairs), and rint done by adding 1.5 * 2^23: for 0 <= y < 2^22 the
// sum rounds to y's nearest integer (ties to even) + 1.5 * 2^23 exactly.
// x >= z holds for every element of its group (z is the group minimum, or
// -M), so y >= 0; y is clamped to 2^B - 1 before the rounding add (the clamp
// binds only for subnormal or saturated fp16 scales).  The clamp also keeps
// the multiply and the rounding add apart: a multiply feeding an add
// directly may be contracted into one fused multiply-add by the code
// generator -- on packed pairs even when both carry an explicit rounding
// modifier -- which would round the exact product once instead of twice and
// change the codes of products that round to a half-way point.
// Returns the sums' bit patterns, the code in the low byte.
constexpr float kRound = 12582912.0f;  // 1.5 * 2^23
template <int B>
__device__ __forceinline__ uint2 codes2(float2 x, float2 nz, float2 r) {
  constexpr float kTop = (float)((1 << B) - 1);
  const float2 y = __fmul2_rn(__fadd2_rn(x, nz), r);
  const float2 m = __fadd2_rn(make_float2(fminf(y.x, kTop), fminf(y.y, kTop)), make_float2(kRound, kRound));
  return make_uint2(__float_as_uint(m.x), __float_as_uint(m.y));
}

// Four codes (low bytes of the codes2 results) into the four bytes of one
// register, byte e = code e.
__device__ __forceinline__ uint32_t code_bytes(uint2 c01, uint2 c23) {
  return __byte_perm(__byte_perm(c01.x, c01.y, 0x0040), __byte_perm(c23.x, c23.y, 0x0040), 0x5410);
}

// Places register (rho, kh) -- byte e holding code e -- into the lane's words.
template <int B, int W>
__device__ __forceinline__ void put_reg(uint32_t* words, int rho, int kh, uint32_t reg) {
  const int j = reg_class(B, rho), sgm = reg_source(B, rho, kh);
  if (B == 3 && sgm >= W) {
#pragma unroll
    for (int e = 0; e < 4; ++e) put_code<B, W>(words, rho, kh, e, (reg >> (8 * e)) & 0xFFu);
  } else {
    words[sgm] |= reg << (B * j);
  }
}

__device__ __forceinline__ float2 bf16x2_to_float2(uint32_t w) { return make_float2(lo_bf16(w), hi_bf16(w)); }

// Minimum and maximum of a group of 32 bf16 values held as 16 pairs, compared
// as bf16x2 (exact: widening bf16 to fp32 keeps the order).
__device__ __forceinline__ void minmax_pairs(uint32_t& mnw, uint32_t& mxw, uint32_t w) {
  const __nv_bfloat162 a = *reinterpret_cast<const __nv_bfloat162*>(&w);
  __nv_bfloat162 lo = *reinterpret_cast<const __nv_bfloat162*>(&mnw), hi = *reinterpret_cast<const __nv_bfloat162*>(&mxw);
  lo = __hmin2(lo, a);
  hi = __hmax2(hi, a);
  mnw = *reinterpret_cast<const uint32_t*>(&lo);
  mxw = *reinterpret_cast<const uint32_t*>(&hi);
}
__device__ __forceinline__ float min_of_pair(uint32_t w) { return fminf(lo_bf16(w), hi_bf16(w)); }
__device__ __forceinline__ float max_of_pair(uint32_t w) { return fmaxf(lo_bf16(w), hi_bf16(w)); }

// KN: multiply by the K normalization factors 1/n (false: n = 1, skipped).
template <int D, int KB, bool KN>
__device__ void pack_k(HalfTile<D>& sm, const float* kinv, uint8_t* rec, int lane, bool hybrid) {
  constexpr int NG = D / 32;
  constexpr int W = words_per_lane(KB, D);
  // statistics: lane = token; 16-byte row reads (the padded row stride puts
  // the eight lanes of a phase on distinct banks)
  {
    const int t = lane;
#pragma unroll
    for (int grp = 0; grp < NG; ++grp) {
      float mn, mx;
      if constexpr (KN) {
        mn = INFINITY, mx = -INFINITY;
#pragma unroll
        for (int c4 = 0; c4 < 4; ++c4) {
          const uint4 u = *reinterpret_cast<const uint4*>(&sm.x[t][grp * 16 + 4 * c4]);
          const uint32_t w4[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            const int cw = grp * 16 + 4 * c4 + k;
            const float x0 = lo_bf16(w4[k]) * kinv[2 * cw], x1 = hi_bf16(w4[k]) * kinv[2 * cw + 1];
            mn = fminf(mn, fminf(x0, x1));
            mx = fmaxf(mx, fmaxf(x0, x1));
          }
        }
      } else {
        uint32_t mnw = sm.x[t][grp * 16], mxw = mnw;
#pragma unroll
        for (int c4 = 0; c4 < 4; ++c4) {
          const uint4 u = *reinterpret_cast<const uint4*>(&sm.x[t][grp * 16 + 4 * c4]);
          minmax_pairs(mnw, mxw, u.x);
          minmax_pairs(mnw, mxw, u.y);
          minmax_pairs(mnw, mxw, u.z);
          minmax_pairs(mnw, mxw, u.w);
        }
        mn = min_of_pair(mnw);
        mx = max_of_pair(mxw);
      }
      float r;
      const uint32_t meta = group_params<KB>(mn, mx, r, hybrid);
      sm.r[t * NG + grp] = r;
      sm.z[t * NG + grp] = mn;
      const int i = (t & 7) * 4 + (t >> 4) * 2 + ((t >> 3) & 1);
      reinterpret_cast<uint32_t*>(rec + blob_bytes(KB, D))[grp * 32 + i] = meta;
    }
  }
  __syncwarp();
  const int gid = lane >> 2, tig = lane & 3;
  uint32_t words[W];
#pragma unroll
  for (int w = 0; w < W; ++w) words[w] = 0;
  // register (rho, kh), byte e: token gid + 8i, channel 32g + 16kh + 4tig + e
#pragma unroll
  for (int rho = 0; rho < D / 8; ++rho) {
    const int i = rho / NG, g = rho % NG;
    const int t = gid + 8 * i;
    const float r1 = sm.r[t * NG + g], z1 = sm.z[t * NG + g];
    const float2 rr = make_float2(r1, r1), nz = make_float2(-z1, -z1);
#pragma unroll
    for (int kh = 0; kh < 2; ++kh) {
      const int d0 = 32 * g + 16 * kh + 4 * tig;
      const uint2 xw = *reinterpret_cast<const uint2*>(&sm.x[t][d0 / 2]);
      float2 x01 = bf16x2_to_float2(xw.x), x23 = bf16x2_to_float2(xw.y);
      if constexpr (KN) {
        x01 = __fmul2_rn(x01, make_float2(kinv[d0], kinv[d0 + 1]));
        x23 = __fmul2_rn(x23, make_float2(kinv[d0 + 2], kinv[d0 + 3]));
      }
      put_reg<KB, W>(words, rho, kh, code_bytes(codes2<KB>(x01, nz, rr), codes2<KB>(x23, nz, rr)));
    }
  }
#pragma unroll
  for (int c = 0; c < W / 4; ++c)
    *reinterpret_cast<uint4*>(rec + word_offset(W, lane, 4 * c)) =
        make_uint4(words[4 * c], words[4 * c + 1], words[4 * c + 2], words[4 * c + 3]);
#pragma unroll
  for (int w = 4 * (W / 4); w < W; ++w) *reinterpret_cast<uint32_t*>(rec + word_offset(W, lane, w)) = words[w];
}

template <int D, int VB>
__device__ void pack_v(HalfTile<D>& sm, uint8_t* vrec, int lane, bool hybrid) {
  constexpr int W = words_per_lane(VB, D);
  // statistics: each lane owns channel pairs (2w, 2w+1), compared as bf16x2
#pragma unroll
  for (int w = lane; w < D / 2; w += 32) {
    uint32_t mnw = sm.x[0][w], mxw = mnw;
#pragma unroll 8
    for (int t = 1; t < kTile; ++t) minmax_pairs(mnw, mxw, sm.x[t][w]);
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int d = 2 * w + h;
      float r, z = h ? hi_bf16(mnw) : lo_bf16(mnw);
      const uint32_t meta = group_params<VB>(z, h ? hi_bf16(mxw) : lo_bf16(mxw), r, hybrid);
      sm.r[d] = r;
      sm.z[d] = z;
      const int i = (d & 7) * (D / 8) + (d >> 4) * 2 + ((d >> 3) & 1);
      reinterpret_cast<uint32_t*>(vrec + blob_bytes(VB, D))[i] = meta;
    }
  }
  __syncwarp();
  const int gid = lane >> 2, tig = lane & 3;
  // channels 16 mb + 8 rh + gid have the parity of gid: pick that bf16 half of
  // a staged word into the high half of a float with one byte permute
  const uint32_t half_sel = (gid & 1) ? 0x3244u : 0x1044u;
  uint32_t words[W];
#pragma unroll
  for (int w = 0; w < W; ++w) words[w] = 0;
  // register (rho, kh), byte e: channel 16mb + 8rh + gid (rho = 2mb + rh),
  // token 4kh + tig + 8e
#pragma unroll
  for (int rho = 0; rho < D / 8; ++rho) {
    const int d = 16 * (rho / 2) + 8 * (rho % 2) + gid;
    const float r1 = sm.r[d], z1 = sm.z[d];
    const float2 rr = make_float2(r1, r1), nz = make_float2(-z1, -z1);
#pragma unroll
    for (int kh = 0; kh < 2; ++kh) {
      float xv[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) xv[e] = __uint_as_float(__byte_perm(sm.x[4 * kh + tig + 8 * e][d >> 1], 0u, half_sel));
      put_reg<VB, W>(words, rho, kh,
                     code_bytes(codes2<VB>(make_float2(xv[0], xv[1]), nz, rr), codes2<VB>(make_float2(xv[2], xv[3]), nz, rr)));
    }
  }
#pragma unroll
  for (int c = 0; c < W / 4; ++c)
    *reinterpret_cast<uint4*>(vrec + word_offset(W, lane, 4 * c)) =
        make_uint4(words[4 * c], words[4 * c + 1], words[4 * c + 2], words[4 * c + 3]);
#pragma unroll
  for (int w = 4 * (W / 4); w < W; ++w) *reinterpret_cast<uint32_t*>(vrec + word_offset(W, lane, w)) = words[w];
}

template <int D, bool KN>
__device__ __forceinline__ void pack_k_dispatch(HalfTile<D>& sm, const float* kinv, int kb, uint8_t* rec, int lane,
                                                bool hybrid) {
  switch (kb) {
    case 2: pack_k<D, 2, KN>(sm, kinv, rec, lane, hybrid); break;
    case 3: pack_k<D, 3, KN>(sm, kinv, rec, lane, hybrid); break;
    case 4: pack_k<D, 4, KN>(sm, kinv, rec, lane, hybrid); break;
    default: pack_k<D, 8, KN>(sm, kinv, rec, lane, hybrid); break;
  }
}

template <int D>
__device__ __forceinline__ void pack_v_dispatch(HalfTile<D>& sm, int vb, uint8_t* vrec, int lane, bool hybrid) {
  switch (vb) {
    case 2: pack_v<D, 2>(sm, vrec, lane, hybrid); break;
    case 3: pack_v<D, 3>(sm, vrec, lane, hybrid); break;
    case 4: pack_v<D, 4>(sm, vrec, lane, hybrid); break;
    default: pack_v<D, 8>(sm, vrec, lane, hybrid); break;
  }
}

}  // namespace
}  // namespace rq

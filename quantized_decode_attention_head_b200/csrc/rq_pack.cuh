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

// KN: multiply by the K normalization factors 1/n (false: n = 1, skipped).
template <int D, int KB, bool KN>
__device__ void pack_k(HalfTile<D>& sm, const float* kinv, uint8_t* rec, int lane, bool hybrid) {
  constexpr int NG = D / 32;
  constexpr int W = words_per_lane(KB, D);
  // statistics: lane = token, rotated word order spreads smem banks
  {
    const int t = lane;
#pragma unroll
    for (int grp = 0; grp < NG; ++grp) {
      float mn = INFINITY, mx = -INFINITY;
#pragma unroll
      for (int c = 0; c < 16; ++c) {
        const int cw = grp * 16 + ((c + (t >> 3)) & 15);
        const uint32_t w = sm.x[t][cw];
        const float x0 = KN ? lo_bf16(w) * kinv[2 * cw] : lo_bf16(w);
        const float x1 = KN ? hi_bf16(w) * kinv[2 * cw + 1] : hi_bf16(w);
        mn = fminf(mn, fminf(x0, x1));
        mx = fmaxf(mx, fmaxf(x0, x1));
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
  for (int rho = 0; rho < D / 8; ++rho)
#pragma unroll
    for (int kh = 0; kh < 2; ++kh)
#pragma unroll
      for (int e = 0; e < 4; e += 2) {
        const int i = rho / NG, g = rho % NG;
        const int t = gid + 8 * i, d0 = 32 * g + 16 * kh + 4 * tig + e;
        const uint32_t x = sm.x[t][d0 / 2];
        const float rr = sm.r[t * NG + g], z = sm.z[t * NG + g];
        put_code<KB, W>(words, rho, kh, e, code_of<KB>(KN ? lo_bf16(x) * kinv[d0] : lo_bf16(x), z, rr));
        put_code<KB, W>(words, rho, kh, e + 1, code_of<KB>(KN ? hi_bf16(x) * kinv[d0 + 1] : hi_bf16(x), z, rr));
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
  // statistics: each lane owns channel pairs (2w, 2w+1)
#pragma unroll
  for (int w = lane; w < D / 2; w += 32) {
    float mn0 = INFINITY, mx0 = -INFINITY, mn1 = INFINITY, mx1 = -INFINITY;
#pragma unroll 8
    for (int t = 0; t < kTile; ++t) {
      const uint32_t x = sm.x[t][w];
      mn0 = fminf(mn0, lo_bf16(x));
      mx0 = fmaxf(mx0, lo_bf16(x));
      mn1 = fminf(mn1, hi_bf16(x));
      mx1 = fmaxf(mx1, hi_bf16(x));
    }
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int d = 2 * w + h;
      float r, z = h ? mn1 : mn0;
      const uint32_t meta = group_params<VB>(z, h ? mx1 : mx0, r, hybrid);
      sm.r[d] = r;
      sm.z[d] = z;
      const int i = (d & 7) * (D / 8) + (d >> 4) * 2 + ((d >> 3) & 1);
      reinterpret_cast<uint32_t*>(vrec + blob_bytes(VB, D))[i] = meta;
    }
  }
  __syncwarp();
  const int gid = lane >> 2, tig = lane & 3;
  uint32_t words[W];
#pragma unroll
  for (int w = 0; w < W; ++w) words[w] = 0;
  // register (rho, kh), byte e: channel 16mb + 8rh + gid (rho = 2mb + rh),
  // token 4kh + tig + 8e
#pragma unroll
  for (int rho = 0; rho < D / 8; ++rho) {
    const int d = 16 * (rho / 2) + 8 * (rho % 2) + gid;
    const float rr = sm.r[d], z = sm.z[d];
#pragma unroll
    for (int kh = 0; kh < 2; ++kh)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const uint32_t x = sm.x[4 * kh + tig + 8 * e][d >> 1];
        put_code<VB, W>(words, rho, kh, e, code_of<VB>((d & 1) ? hi_bf16(x) : lo_bf16(x), z, rr));
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

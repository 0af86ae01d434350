// Split-K decode attention over the packed cache (sm_100a).
//
// One CTA = one work item of one (layer, batch, kv-head) stream: either a
// contiguous range of packed tiles (items 0..n_splits-1) or the bf16 sink +
// recent window (item n_splits).  Four consumer warps process tiles; a fifth
// warp streams tile records into a ring of shared-memory stages with 1-D bulk
// copies (cp.async.bulk, TMA engine) completing on mbarriers.  The last CTA
// of a stream to finish merges all items' partial softmax states
// (log-sum-exp) and writes the output -- no second launch.
//
// Per tile (32 tokens), with the G query heads that share the kv head:
//   q.K^T  : tensor-core MMA (m16n8k16, f16 in, f32 accumulate).  A = the
//            packed K codes unpacked in registers to fp16 subnormals c*2^-24
//            (exact), B = q scaled by 2^kq into fp16 range.  Each 32-channel
//            K group gets its own 8-column slot so its fp16 scale and bf16
//            zero factor out of the inner sum (InnerQ grouping):
//              score = sum_grp s_grp * sum_d q_d c_d + z_grp * sum_d q_d.
//   softmax: online, base 2, running max per head.
//   P.V    : MMA with A = V codes (channel x token), B = P (fp16), fp32
//            accumulate; the V scale/zero are per channel for the whole tile:
//              o_d += s_d * sum_t p_t c_td + z_d * sum_t p_t,
//            where sum_t p_t comes from the same MMA with A = 1.
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include <cfloat>

#include "rq_device.cuh"
#include "rq_internal.h"

namespace rq {
namespace {

constexpr int NW = kDecodeConsumerWarps;
constexpr int kStages = 8;  // multiple of NW: stage s is always consumed by warp s % NW
static_assert(kStages % NW == 0, "stage ownership");

template <int D, int G>
struct Cfg {
  static constexpr int NG = D / 32;      // K groups per token
  static constexpr int GPS = 8 / G;      // groups sharing one 8-column accumulator
  static constexpr int NSET = (NG + GPS - 1) / GPS;
  static constexpr int PART = G * D + 2 * G;  // floats per partial state
};

template <int D, int G>
struct WarpState {
  uint32_t qb[D / 16][2];          // q B-fragments (fp16, scaled by 2^kq)
  float kscale;                    // 2^(24 - kq)
  float qsum[Cfg<D, G>::NSET][2];  // sum of q over the thread's (group, head) columns
  float m[2], l[2];                // running max (log2 units) / sum per column parity
  float o[D / 16][4];              // P.V accumulators, out^T fragment layout
};

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}
__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

template <int D, int G>
__device__ void setup_query(WarpState<D, G>& st, const uint16_t* qh, int lane) {
  using C = Cfg<D, G>;
  const int gid = lane >> 2, tig = lane & 3;
  const int bh = gid % G;          // head of B column n = gid
  const int bgl = gid / G;         // group slot of B column n = gid
  uint32_t raw[D / 16][2];
  float mx = 0.0f;
#pragma unroll
  for (int kb = 0; kb < D / 16; ++kb)
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      raw[kb][j] = __ldg(reinterpret_cast<const uint32_t*>(qh + bh * D + 16 * kb + 8 * j + 2 * tig));
      mx = fmaxf(mx, fmaxf(fabsf(bf16_bits_to_float(raw[kb][j] & 0xFFFFu)), fabsf(bf16_bits_to_float(raw[kb][j] >> 16))));
    }
  mx = warp_max(mx);
  int kq = 0;
  if (mx > 0.0f) {
    const int e = (int)((__float_as_uint(mx) >> 23) & 0xFF) - 126;  // mx < 2^e
    kq = 15 - e;
    kq = kq > 100 ? 100 : (kq < -100 ? -100 : kq);
  }
  const float up = __int_as_float((kq + 127) << 23);
  st.kscale = __int_as_float((24 - kq + 127) << 23);
#pragma unroll
  for (int kb = 0; kb < D / 16; ++kb) {
    const bool valid = ((kb / 2) % C::GPS) == bgl;
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      const float lo = bf16_bits_to_float(raw[kb][j] & 0xFFFFu) * up;
      const float hi = bf16_bits_to_float(raw[kb][j] >> 16) * up;
      st.qb[kb][j] = valid ? pack_half2(lo, hi) : 0u;
    }
  }
#pragma unroll
  for (int s = 0; s < C::NSET; ++s)
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      const int n = 2 * tig + e;
      const int grp = s * C::GPS + n / G, h = n % G;
      float acc = 0.0f;
      if (grp < C::NG) {
        const uint4* p = reinterpret_cast<const uint4*>(qh + h * D + grp * 32);
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          const uint4 u = __ldg(p + c);
          const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
          for (int k = 0; k < 4; ++k) acc += bf16_bits_to_float(w[k] & 0xFFFFu) + bf16_bits_to_float(w[k] >> 16);
        }
      }
      st.qsum[s][e] = acc;
    }
  st.m[0] = st.m[1] = -INFINITY;
  st.l[0] = st.l[1] = 0.0f;
#pragma unroll
  for (int mb = 0; mb < D / 16; ++mb)
#pragma unroll
    for (int r = 0; r < 4; ++r) st.o[mb][r] = 0.0f;
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

// q.K^T of one tile -> logits x[mb][rr][e] (log2 units) for tokens
// 16mb + 8rr + gid and heads (2 tig + e) % G.
template <int D, int G, int KB>
__device__ __forceinline__ void qk_tile(const uint8_t* rec, const WarpState<D, G>& st, float scale_log2,
                                        float (&x)[2][2][2], int lane) {
  using C = Cfg<D, G>;
  constexpr int W = words_per_lane(KB, D);
  const int gid = lane >> 2, tig = lane & 3;
  uint32_t kw[W];
  load_words<W>(kw, rec, lane);
  float acc[C::NSET][2][4];
#pragma unroll
  for (int s = 0; s < C::NSET; ++s)
#pragma unroll
    for (int mb = 0; mb < 2; ++mb)
#pragma unroll
      for (int r = 0; r < 4; ++r) acc[s][mb][r] = 0.0f;
#pragma unroll
  for (int mb = 0; mb < 2; ++mb)
#pragma unroll
    for (int kb = 0; kb < D / 16; ++kb) {
      uint32_t a[4];
#pragma unroll
      for (int r = 0; r < 4; ++r) {
        const int idx = k_pair_index(D, mb, kb, r);
        a[r] = extract_pair<KB>(kw[slot_word(KB, W, idx)], slot_pos(KB, W, idx));
      }
      mma_f16(acc[(kb / 2) / C::GPS][mb], a, st.qb[kb][0], st.qb[kb][1]);
    }
  const uint32_t* kmeta = reinterpret_cast<const uint32_t*>(rec + blob_bytes(KB, D));
  float sc[2][2][2];
#pragma unroll
  for (int mb = 0; mb < 2; ++mb)
#pragma unroll
    for (int rr = 0; rr < 2; ++rr) sc[mb][rr][0] = sc[mb][rr][1] = 0.0f;
#pragma unroll
  for (int s = 0; s < C::NSET; ++s)
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      const int grp = s * C::GPS + (2 * tig + e) / G;
      if (grp < C::NG) {
        const uint4 mv = *reinterpret_cast<const uint4*>(kmeta + grp * 32 + gid * 4);
        const uint32_t mw[4] = {mv.x, mv.y, mv.z, mv.w};
#pragma unroll
        for (int mb = 0; mb < 2; ++mb)
#pragma unroll
          for (int rr = 0; rr < 2; ++rr) {
            const uint32_t m = mw[mb * 2 + rr];
            const float sk = __half2float(__ushort_as_half((unsigned short)(m & 0xFFFFu))) * st.kscale;
            const float z = __uint_as_float(m & 0xFFFF0000u);
            sc[mb][rr][e] = fmaf(sk, acc[s][mb][rr * 2 + e], fmaf(z, st.qsum[s][e], sc[mb][rr][e]));
          }
      }
    }
  // sum the group columns of each head across the quad of lanes sharing a row
#pragma unroll
  for (int mb = 0; mb < 2; ++mb)
#pragma unroll
    for (int rr = 0; rr < 2; ++rr) {
      float v0 = sc[mb][rr][0], v1 = sc[mb][rr][1];
      if (G == 1) {
        v0 += v1;
        v0 += __shfl_xor_sync(0xffffffffu, v0, 1);
        v0 += __shfl_xor_sync(0xffffffffu, v0, 2);
        v1 = v0;
      } else if (G == 2) {
        v0 += __shfl_xor_sync(0xffffffffu, v0, 1);
        v1 += __shfl_xor_sync(0xffffffffu, v1, 1);
        v0 += __shfl_xor_sync(0xffffffffu, v0, 2);
        v1 += __shfl_xor_sync(0xffffffffu, v1, 2);
      } else if (G == 4) {
        v0 += __shfl_xor_sync(0xffffffffu, v0, 2);
        v1 += __shfl_xor_sync(0xffffffffu, v1, 2);
      }
      x[mb][rr][0] = v0 * scale_log2;
      x[mb][rr][1] = v1 * scale_log2;
    }
}

// Online softmax update; returns P as PV B-fragments pb[kb][rr].
template <int D, int G>
__device__ __forceinline__ void softmax_tile(WarpState<D, G>& st, const float (&x)[2][2][2], uint32_t (&pb)[2][2]) {
  float tmax[2];
#pragma unroll
  for (int e = 0; e < 2; ++e) {
    float v = fmaxf(fmaxf(x[0][0][e], x[0][1][e]), fmaxf(x[1][0][e], x[1][1][e]));
    v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 4));
    v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 8));
    v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 16));
    tmax[e] = v;
  }
  const bool grow = tmax[0] > st.m[0] || tmax[1] > st.m[1];
  if (__any_sync(0xffffffffu, grow)) {
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      const float mn = fmaxf(st.m[e], tmax[e]);
      const float alpha = ex2(st.m[e] - mn);
      st.m[e] = mn;
      st.l[e] *= alpha;
#pragma unroll
      for (int mb = 0; mb < D / 16; ++mb) {
        st.o[mb][e] *= alpha;
        st.o[mb][2 + e] *= alpha;
      }
    }
  }
#pragma unroll
  for (int mb = 0; mb < 2; ++mb)
#pragma unroll
    for (int rr = 0; rr < 2; ++rr)
      pb[mb][rr] = movmatrix_trans(pack_half2(ex2(x[mb][rr][0] - st.m[0]), ex2(x[mb][rr][1] - st.m[1])));
}

template <int D, int G, int VB>
__device__ __forceinline__ void pv_tile(const uint8_t* vrec, WarpState<D, G>& st, const uint32_t (&pb)[2][2], int lane) {
  constexpr int W = words_per_lane(VB, D);
  const int gid = lane >> 2;
  uint32_t vw[W];
  load_words<W>(vw, vrec, lane);
  float acc[D / 16][4];
#pragma unroll
  for (int mb = 0; mb < D / 16; ++mb) {
    acc[mb][0] = acc[mb][1] = acc[mb][2] = acc[mb][3] = 0.0f;
#pragma unroll
    for (int kb = 0; kb < 2; ++kb) {
      uint32_t a[4];
#pragma unroll
      for (int r = 0; r < 4; ++r) {
        const int idx = v_pair_index(mb, kb, r);
        a[r] = extract_pair<VB>(vw[slot_word(VB, W, idx)], slot_pos(VB, W, idx));
      }
      mma_f16(acc[mb], a, pb[kb][0], pb[kb][1]);
    }
  }
  float ps[4] = {0.0f, 0.0f, 0.0f, 0.0f};
  const uint32_t ones[4] = {0x3C003C00u, 0x3C003C00u, 0x3C003C00u, 0x3C003C00u};
  mma_f16(ps, ones, pb[0][0], pb[0][1]);
  mma_f16(ps, ones, pb[1][0], pb[1][1]);
  const uint32_t* vmeta = reinterpret_cast<const uint32_t*>(vrec + blob_bytes(VB, D)) + gid * (D / 8);
  constexpr float k2p24 = 16777216.0f;
#pragma unroll
  for (int c = 0; c < D / 32; ++c) {
    const uint4 mv = *reinterpret_cast<const uint4*>(vmeta + 4 * c);
    const uint32_t mw[4] = {mv.x, mv.y, mv.z, mv.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int mb = 2 * c + j / 2, rr = j % 2;
      const float sv = __half2float(__ushort_as_half((unsigned short)(mw[j] & 0xFFFFu))) * k2p24;
      const float z = __uint_as_float(mw[j] & 0xFFFF0000u);
#pragma unroll
      for (int e = 0; e < 2; ++e)
        st.o[mb][rr * 2 + e] = fmaf(sv, acc[mb][rr * 2 + e], fmaf(z, ps[e], st.o[mb][rr * 2 + e]));
    }
  }
  st.l[0] += ps[0];
  st.l[1] += ps[1];
}

template <int D, int G, int KB, int VB>
__device__ __forceinline__ void process_tile(const uint8_t* rec, WarpState<D, G>& st, float scale_log2, int lane) {
  float x[2][2][2];
  qk_tile<D, G, KB>(rec, st, scale_log2, x, lane);
  uint32_t pb[2][2];
  softmax_tile<D, G>(st, x, pb);
  pv_tile<D, G, VB>(rec + blob_bytes(KB, D) + 4 * D, st, pb, lane);
}

template <int D, int G>
__device__ __forceinline__ void process_tile_dispatch(int kb, int vb, const uint8_t* rec, WarpState<D, G>& st,
                                                      float sl2, int lane) {
#define RQ_V(KBV)                                                         \
  switch (vb) {                                                           \
    case 2: process_tile<D, G, KBV, 2>(rec, st, sl2, lane); break;        \
    case 3: process_tile<D, G, KBV, 3>(rec, st, sl2, lane); break;        \
    case 4: process_tile<D, G, KBV, 4>(rec, st, sl2, lane); break;        \
    default: process_tile<D, G, KBV, 8>(rec, st, sl2, lane); break;       \
  }
  switch (kb) {
    case 2: RQ_V(2) break;
    case 3: RQ_V(3) break;
    case 4: RQ_V(4) break;
    default: RQ_V(8) break;
  }
#undef RQ_V
}

// Canonical partial of one warp in shared memory: o[G][D], m[G], l[G].
template <int D, int G>
__device__ void dump_tile_state(const WarpState<D, G>& st, float* slot, int lane) {
  const int gid = lane >> 2, tig = lane & 3;
#pragma unroll
  for (int e = 0; e < 2; ++e) {
    const int n = 2 * tig + e;
    if (n < G) {
#pragma unroll
      for (int mb = 0; mb < D / 16; ++mb)
#pragma unroll
        for (int rr = 0; rr < 2; ++rr) slot[n * D + 16 * mb + 8 * rr + gid] = st.o[mb][rr * 2 + e];
      if (gid == 0) {
        slot[G * D + n] = st.m[e];
        slot[G * D + G + n] = st.l[e];
      }
    }
  }
}

// bf16 sink + recent window on CUDA cores; lane = token for q.k, lane = channel for p.v.
template <int D, int G>
__device__ void window_warp(const DecodeArgs& a, const uint8_t* win, const float* qs, float* slot, int warp, int lane) {
  const int S = a.g.S, ring = a.g.R + kTile;
  const int n_sink = a.T < S ? a.T : S;
  const int n_tok = n_sink + (a.T - n_sink - a.Tq);
  float m[G], l[G], o[G][D / 32];
#pragma unroll
  for (int h = 0; h < G; ++h) {
    m[h] = -INFINITY;
    l[h] = 0.0f;
#pragma unroll
    for (int j = 0; j < D / 32; ++j) o[h][j] = 0.0f;
  }
  auto row_of = [&](int j, int kv) -> const uint16_t* {
    if (j < n_sink) return reinterpret_cast<const uint16_t*>(win + ((size_t)kv * S + j) * D * 2);
    const int slot_i = (a.Tq + (j - n_sink)) % ring;  // position S + Tq + (j - n_sink)
    return reinterpret_cast<const uint16_t*>(win + ((size_t)2 * S + (size_t)kv * ring + slot_i) * D * 2);
  };
  for (int c0 = warp * 32; c0 < n_tok; c0 += NW * 32) {
    const int j = c0 + lane;
    const bool valid = j < n_tok;
    float sc[G];
#pragma unroll
    for (int h = 0; h < G; ++h) sc[h] = 0.0f;
    if (valid) {
      const uint4* kr = reinterpret_cast<const uint4*>(row_of(j, 0));
#pragma unroll 4
      for (int c = 0; c < D / 8; ++c) {
        const uint4 u = __ldg(kr + c);
        const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const float k0 = bf16_bits_to_float(w[k] & 0xFFFFu), k1 = bf16_bits_to_float(w[k] >> 16);
#pragma unroll
          for (int h = 0; h < G; ++h) sc[h] = fmaf(qs[h * D + 8 * c + 2 * k], k0, fmaf(qs[h * D + 8 * c + 2 * k + 1], k1, sc[h]));
        }
      }
    }
    float p[G];
#pragma unroll
    for (int h = 0; h < G; ++h) {
      const float xv = valid ? sc[h] * a.scale_log2 : -INFINITY;
      const float mn = fmaxf(m[h], warp_max(xv));
      const float alpha = ex2(m[h] - mn);
      p[h] = valid ? ex2(xv - mn) : 0.0f;
      l[h] = l[h] * alpha + warp_sum(p[h]);
      m[h] = mn;
#pragma unroll
      for (int jj = 0; jj < D / 32; ++jj) o[h][jj] *= alpha;
    }
    const int cnt = min(32, n_tok - c0);
    for (int t = 0; t < cnt; ++t) {
      const uint16_t* vr = row_of(c0 + t, 1);
      float vv[D / 32];
#pragma unroll
      for (int jj = 0; jj < D / 32; ++jj) vv[jj] = bf16_bits_to_float(__ldg(vr + lane + 32 * jj));
#pragma unroll
      for (int h = 0; h < G; ++h) {
        const float pt = __shfl_sync(0xffffffffu, p[h], t);
#pragma unroll
        for (int jj = 0; jj < D / 32; ++jj) o[h][jj] = fmaf(pt, vv[jj], o[h][jj]);
      }
    }
  }
#pragma unroll
  for (int h = 0; h < G; ++h) {
#pragma unroll
    for (int jj = 0; jj < D / 32; ++jj) slot[h * D + lane + 32 * jj] = o[h][jj];
    if (lane == 0) {
      slot[G * D + h] = m[h];
      slot[G * D + G + h] = l[h];
    }
  }
}

__device__ __forceinline__ void raise_abort(volatile int* abort_flag, int* status) {
  *abort_flag = 1;
  atomicCAS(status, 0, kDeviceTimeout);
}

template <int D, int G>
__global__ void __launch_bounds__(kDecodeThreads) decode_kernel(DecodeArgs a) {
  using C = Cfg<D, G>;
  extern __shared__ __align__(128) uint8_t smem[];
  __shared__ uint64_t full_bar[kStages], empty_bar[kStages];
  __shared__ volatile int abort_flag;
  __shared__ int is_last;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int srel = blockIdx.y, item = blockIdx.x;
  const int NI = a.n_splits + 1;
  const int h = srel % a.g.Hkv, b = (srel / a.g.Hkv) % a.g.B, lrel = srel / (a.g.Hkv * a.g.B);
  const int l = a.layer0 + lrel;
  const HeadDesc hd = a.desc[l * a.g.Hkv + h];
  const uint16_t* qh = a.q + ((size_t)(lrel * a.g.B + b) * a.g.Hq + (size_t)h * G) * D;
  float* merge = reinterpret_cast<float*>(smem);  // aliases the stages after the main loop

  if (tid == 0) {
    abort_flag = 0;
#pragma unroll
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full_bar[s], 1);
      mbar_init(&empty_bar[s], 1);
    }
    mbar_fence_init();
  }
  __syncthreads();

  WarpState<D, G> st;
  const bool tiles_item = item < a.n_splits;
  if (tiles_item) {
    const int t0 = (int)(((int64_t)item * a.n_tiles) / a.n_splits);
    const int t1 = (int)(((int64_t)(item + 1) * a.n_tiles) / a.n_splits);
    const int n_my = t1 - t0;
    const int rec = hd.rec_bytes;
    const uint8_t* src = a.buf + hd.tile_base + (int64_t)b * hd.tile_stride + (int64_t)t0 * rec;
    if (warp == NW) {
      if (lane == 0) {
        int last_issue[kStages];
#pragma unroll
        for (int s = 0; s < kStages; ++s) last_issue[s] = -1;
        for (int i = 0; i < n_my; ++i) {
          const int s = i % kStages;
          if (i >= kStages && !mbar_wait_bounded(&empty_bar[s], ((i / kStages) - 1) & 1)) {
            raise_abort(&abort_flag, a.status);
            break;
          }
          if (abort_flag) break;
          mbar_arrive_expect_tx(&full_bar[s], (uint32_t)rec);
          bulk_g2s(smem + (size_t)s * a.stage_bytes, src + (int64_t)i * rec, (uint32_t)rec, &full_bar[s]);
          last_issue[s] = i;
        }
        if (abort_flag) {  // let copies in flight land before the CTA exits
          for (int s = 0; s < kStages; ++s)
            if (last_issue[s] >= 0) (void)mbar_wait_bounded(&full_bar[s], (last_issue[s] / kStages) & 1);
        }
      }
    } else {
      setup_query<D, G>(st, qh, lane);
      for (int i = warp; i < n_my; i += NW) {
        const int s = i % kStages;
        const bool ok = __all_sync(0xffffffffu, mbar_wait_bounded(&full_bar[s], (i / kStages) & 1));
        if (!ok) {
          if (lane == 0) raise_abort(&abort_flag, a.status);
          break;
        }
        process_tile_dispatch<D, G>(hd.k_bits, hd.v_bits, smem + (size_t)s * a.stage_bytes, st, a.scale_log2, lane);
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty_bar[s]);
        if (abort_flag) break;
      }
    }
  } else {
    // bf16 sink + recent window on CUDA cores
    float* qs = merge + NW * C::PART;
    for (int i = tid; i < G * D; i += blockDim.x) qs[i] = bf16_bits_to_float(qh[i]);
    __syncthreads();
    if (warp < NW) {
      const uint8_t* win = a.buf + hd.win_base + (int64_t)b * a.g.win_bytes;
      window_warp<D, G>(a, win, qs, merge + warp * C::PART, warp, lane);
    }
  }
  __syncthreads();  // every stage read has completed; merge may now alias the stages
  if (tiles_item && warp < NW && !abort_flag) dump_tile_state<D, G>(st, merge + warp * C::PART, lane);
  __syncthreads();
  if (abort_flag) return;

  // merge the four warps' partial states into this item's partial
  float* part = a.partials + ((size_t)srel * NI + item) * C::PART;
  for (int idx = tid; idx < G * D; idx += blockDim.x) {
    const int hh = idx / D;
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < NW; ++w) M = fmaxf(M, merge[w * C::PART + G * D + hh]);
    float O = 0.0f, L = 0.0f;
    if (M != -INFINITY) {
#pragma unroll
      for (int w = 0; w < NW; ++w) {
        const float f = ex2(merge[w * C::PART + G * D + hh] - M);
        O = fmaf(merge[w * C::PART + idx], f, O);
        L = fmaf(merge[w * C::PART + G * D + G + hh], f, L);
      }
    }
    part[idx] = O;
    if (idx % D == 0) {
      part[G * D + hh] = M;
      part[G * D + G + hh] = L;
    }
  }
  __threadfence();
  __syncthreads();
  if (tid == 0) is_last = (atomicAdd(&a.counters[srel], 1u) == (unsigned)(NI - 1));
  __syncthreads();
  if (!is_last) return;
  __threadfence();

  // last CTA of the stream: log-sum-exp combine over all items
  float* wts = merge;  // [NI][G] weights, then [G] 1/L
  const float* base = a.partials + (size_t)srel * NI * C::PART;
  for (int hh = warp; hh < G; hh += blockDim.x / 32) {
    float M = -INFINITY;
    for (int i = lane; i < NI; i += 32) M = fmaxf(M, __ldcg(base + (size_t)i * C::PART + G * D + hh));
    M = warp_max(M);
    float L = 0.0f;
    for (int i = lane; i < NI; i += 32) {
      const float mi = __ldcg(base + (size_t)i * C::PART + G * D + hh);
      const float f = (M == -INFINITY) ? 0.0f : ex2(mi - M);
      wts[i * G + hh] = f;
      L = fmaf(__ldcg(base + (size_t)i * C::PART + G * D + G + hh), f, L);
    }
    L = warp_sum(L);
    if (lane == 0) wts[NI * G + hh] = L > 0.0f ? 1.0f / L : 0.0f;
  }
  __syncthreads();
  float* outp = a.out + ((size_t)(lrel * a.g.B + b) * a.g.Hq + (size_t)h * G) * D;
  for (int idx = tid; idx < G * D; idx += blockDim.x) {
    const int hh = idx / D;
    float O = 0.0f;
    for (int i = 0; i < NI; ++i) O = fmaf(__ldcg(base + (size_t)i * C::PART + idx), wts[i * G + hh], O);
    outp[idx] = O * wts[NI * G + hh];
  }
  if (tid == 0) a.counters[srel] = 0u;
}

template <int D, int G>
cudaError_t launch_dg(const DecodeArgs& a, int smem, cudaStream_t st) {
  cudaError_t e = cudaFuncSetAttribute(decode_kernel<D, G>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  const int streams = a.n_layers * a.g.B * a.g.Hkv;
  dim3 grid(a.n_splits + 1, streams);
  decode_kernel<D, G><<<grid, kDecodeThreads, smem, st>>>(a);
  return cudaGetLastError();
}

}  // namespace

int decode_smem_bytes(int n_items, int stage_bytes, int G, int D) {
  const int part = G * D + 2 * G;
  int merge = (NW * part + G * D) * 4;
  const int wts = (n_items + 1) * G * 4;
  merge = merge > wts ? merge : wts;
  const int ring = kStages * stage_bytes;
  int need = ring > merge ? ring : merge;
  return (need + 127) / 128 * 128;
}

cudaError_t launch_decode(const DecodeArgs& a, int smem, cudaStream_t st) {
  const int D = a.g.D, G = a.g.G;
#define RQ_DG(DD, GG) \
  if (D == DD && G == GG) return launch_dg<DD, GG>(a, smem, st);
  RQ_DG(128, 1) RQ_DG(128, 2) RQ_DG(128, 4) RQ_DG(128, 8)
  RQ_DG(64, 1) RQ_DG(64, 2) RQ_DG(64, 4) RQ_DG(64, 8)
#undef RQ_DG
  return cudaErrorInvalidValue;
}

}  // namespace rq

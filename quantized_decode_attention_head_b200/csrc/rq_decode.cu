// Split-K decode attention over the packed cache (sm_100a).
//
// One CTA = one work item of one (layer, batch, kv-head) stream: either a
// contiguous range of packed tiles (items 0..n_splits-1) or the bf16 sink +
// recent window (items n_splits..).  Four warps process tiles; lane 0 of each
// streams the warp's own tile records into a private ring of shared-memory
// stages with 1-D bulk copies (cp.async.bulk, TMA engine) completing on
// mbarriers.  The last CTA
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
#include <mutex>

#include "rq_device.cuh"
#include "rq_internal.h"

namespace rq {
namespace {

constexpr int NW = kDecodeConsumerWarps;
constexpr int kMaxStages = 8;  // per-warp ring depth limit
constexpr float kRescaleSlack = 8.0f;

template <int D, int G>
struct Cfg {
  static constexpr int NG = D / 32;      // K groups per token
  static constexpr int GPS = 8 / G;      // groups sharing one 8-column accumulator
  static constexpr int NSET = (NG + GPS - 1) / GPS;
  static constexpr int PART = G * D + 2 * G;  // floats per partial state
};

template <int D, int G>
struct WarpState {
  static constexpr int KE = G == 1 ? 2 : 1;  // column parities with distinct K groups
  uint32_t qb[D / 16][2];                    // q B-fragments (fp16, scaled by 2^kq)
  float ksf[2][2][Cfg<D, G>::NSET][KE];      // 2^(24 - kq - b*class) * softmax scale * log2(e)
  float qsum[Cfg<D, G>::NSET][2];            // softmax-scaled sum of q over (group, head) columns
  float m[2], l[2];                          // running max (log2 units) / sum per column parity
  float o[D / 16][4];                        // P.V accumulators (x 2^-24), out^T fragment layout
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

__device__ __forceinline__ float pow2i(int e) { return __int_as_float((e + 127) << 23); }

template <int D, int G, int KB>
__device__ void setup_query(WarpState<D, G>& st, const uint16_t* qh, float scale_log2, int lane) {
  using C = Cfg<D, G>;
  constexpr int WK = words_per_lane(KB, D);
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
  const float up = pow2i(kq);
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
      st.qsum[s][e] = acc * scale_log2;
#pragma unroll
      for (int mb = 0; mb < 2; ++mb)
#pragma unroll
        for (int rr = 0; rr < 2; ++rr) {
          if (e < WarpState<D, G>::KE) {
            const int q = (mb * 2 + rr) * C::NG + (grp < C::NG ? grp : 0);
            st.ksf[mb][rr][s][e] = pow2i(24 - kq - KB * quad_class(KB, WK, q)) * scale_log2;
          }
        }
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

__device__ __forceinline__ float half_lo_to_float(uint32_t m) {
  return __half2float(__ushort_as_half((unsigned short)(m & 0xFFFFu)));
}

// q.K^T of one tile -> logits x[mb][rr][e] (log2 units, softmax scale applied)
// for tokens 16mb + 8rr + gid and heads (2 tig + e) % G.
template <int D, int G, int KB>
__device__ __forceinline__ void qk_tile(const uint8_t* rec, const WarpState<D, G>& st, float (&x)[2][2][2], int lane) {
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
        a[r] = extract_pair<KB>(kw, slot_word(KB, W, idx), slot_pos(KB, W, idx));
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
    for (int e = 0; e < WarpState<D, G>::KE; ++e) {
      // for G >= 2 both column parities of a thread share one K group
      const int grp = s * C::GPS + (2 * tig + e) / G;
      if (grp < C::NG) {
        const uint4 mv = *reinterpret_cast<const uint4*>(kmeta + grp * 32 + gid * 4);
        const uint32_t mw[4] = {mv.x, mv.y, mv.z, mv.w};
#pragma unroll
        for (int mb = 0; mb < 2; ++mb)
#pragma unroll
          for (int rr = 0; rr < 2; ++rr) {
            const uint32_t m = mw[mb * 2 + rr];
            const float sk = half_lo_to_float(m) * st.ksf[mb][rr][s][e];
            const float z = __uint_as_float(m & 0xFFFF0000u);
            if (G == 1) {
              sc[mb][rr][e] = fmaf(sk, acc[s][mb][rr * 2 + e], fmaf(z, st.qsum[s][e], sc[mb][rr][e]));
            } else {
              sc[mb][rr][0] = fmaf(sk, acc[s][mb][rr * 2], fmaf(z, st.qsum[s][0], sc[mb][rr][0]));
              sc[mb][rr][1] = fmaf(sk, acc[s][mb][rr * 2 + 1], fmaf(z, st.qsum[s][1], sc[mb][rr][1]));
            }
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
      x[mb][rr][0] = v0;
      x[mb][rr][1] = v1;
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
  // Lazy rescale: the reference max only moves when a score exceeds it by
  // more than kRescaleSlack (log2 units), so P <= 2^kRescaleSlack stays well
  // inside fp16 and o is rescaled only a handful of times per work item.
  const bool grow = tmax[0] > st.m[0] + kRescaleSlack || tmax[1] > st.m[1] + kRescaleSlack;
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
  // sum_t p_t * 2^-24 per column: A = the fp16 subnormal 2^-24, so every
  // accumulator below carries the same 2^-24 as the unpacked codes
  float ps[4] = {0.0f, 0.0f, 0.0f, 0.0f};
  const uint32_t tiny[4] = {0x00010001u, 0x00010001u, 0x00010001u, 0x00010001u};
  mma_f16(ps, tiny, pb[0][0], pb[0][1]);
  mma_f16(ps, tiny, pb[1][0], pb[1][1]);
  uint32_t vw[W];
  load_words<W>(vw, vrec, lane);
  const uint32_t* vmeta = reinterpret_cast<const uint32_t*>(vrec + blob_bytes(VB, D)) + gid * (D / 8);
#pragma unroll
  for (int c = 0; c < D / 32; ++c) {
    const uint4 mv = *reinterpret_cast<const uint4*>(vmeta + 4 * c);
    const uint32_t mw[4] = {mv.x, mv.y, mv.z, mv.w};
#pragma unroll
    for (int half = 0; half < 2; ++half) {
      const int mb = 2 * c + half;
      float acc[4] = {0.0f, 0.0f, 0.0f, 0.0f};
#pragma unroll
      for (int kb = 0; kb < 2; ++kb) {
        uint32_t a[4];
#pragma unroll
        for (int r = 0; r < 4; ++r) {
          const int idx = v_pair_index(mb, kb, r);
          a[r] = extract_pair<VB>(vw, slot_word(VB, W, idx), slot_pos(VB, W, idx));
        }
        mma_f16(acc, a, pb[kb][0], pb[kb][1]);
      }
#pragma unroll
      for (int rr = 0; rr < 2; ++rr) {
        const uint32_t m = mw[half * 2 + rr];
        const int cls = quad_class(VB, W, mb * 2 + rr);
        float sv = half_lo_to_float(m);
        if (cls) sv *= 1.0f / (float)(1 << (VB * cls));
        const float z = __uint_as_float(m & 0xFFFF0000u);
#pragma unroll
        for (int e = 0; e < 2; ++e)
          st.o[mb][rr * 2 + e] = fmaf(sv, acc[rr * 2 + e], fmaf(z, ps[e], st.o[mb][rr * 2 + e]));
      }
    }
  }
  st.l[0] += ps[0];
  st.l[1] += ps[1];
}

template <int D, int G, int KB>
__device__ __forceinline__ void score_tile(const uint8_t* rec, WarpState<D, G>& st, uint32_t (&pb)[2][2], int lane) {
  float x[2][2][2];
  qk_tile<D, G, KB>(rec, st, x, lane);
  softmax_tile<D, G>(st, x, pb);
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
template <int D, int G, int KB, int VB>
__device__ void consume(WarpState<D, G>& st, const uint16_t* qh, float scale_log2, uint8_t* ring, int stages,
                        int stage_bytes, uint64_t* bars, const uint8_t* src, int rec, int n_my, int warp, int lane,
                        volatile int* abort_flag, int* status) {
  const int n_w = n_my > warp ? (n_my - warp + NW - 1) / NW : 0;
  if (lane == 0) {
    for (int j = 0; j < stages && j < n_w; ++j) {
      mbar_arrive_expect_tx(&bars[j], (uint32_t)rec);
      bulk_g2s(ring + (size_t)j * stage_bytes, src + (int64_t)(warp + j * NW) * rec, (uint32_t)rec, &bars[j]);
    }
  }
  setup_query<D, G, KB>(st, qh, scale_log2, lane);
  // ring position of a tile: slot = j mod stages, parity = (j / stages) & 1,
  // advanced incrementally (no integer division in the loop)
  auto wait_slot = [&](int slot, int parity) -> bool {
    return __all_sync(0xffffffffu, mbar_wait_bounded(&bars[slot], (uint32_t)parity));
  };
  auto refill = [&](int j, int slot) {  // the warp has finished reading tile j's slot
    if (lane == 0 && j + stages < n_w) {
      fence_proxy_async_smem();  // generic-proxy reads of the slot precede the async refill
      mbar_arrive_expect_tx(&bars[slot], (uint32_t)rec);
      bulk_g2s(ring + (size_t)slot * stage_bytes, src + (int64_t)(warp + (j + stages) * NW) * rec, (uint32_t)rec,
               &bars[slot]);
    }
  };
  const int VOFF = blob_bytes(KB, D) + 4 * D;
  int j = 0;
  bool ok = true;
  if (n_w > 0) {
    // software pipeline: the scores of tile j + 1 are computed in the same
    // block as the P.V of tile j, so their MMA chains interleave
    uint32_t pb[2][2];
    int cs = 0;             // slot of tile j
    int ns = 1, nph = 0;    // slot and parity of tile j + 1
    if (ns == stages) {
      ns = 0;
      nph = 1;
    }
    ok = wait_slot(0, 0);
    if (ok) score_tile<D, G, KB>(ring, st, pb, lane);
    for (; ok && j + 1 < n_w; ++j) {
      ok = wait_slot(ns, nph);
      if (!ok) break;
      const uint8_t* cur = ring + (size_t)cs * stage_bytes;
      const uint8_t* nxt = ring + (size_t)ns * stage_bytes;
      float x[2][2][2];
      qk_tile<D, G, KB>(nxt, st, x, lane);
      pv_tile<D, G, VB>(cur + VOFF, st, pb, lane);
      softmax_tile<D, G>(st, x, pb);
      __syncwarp();
      refill(j, cs);
      cs = ns;
      if (++ns == stages) {
        ns = 0;
        nph ^= 1;
      }
      if (*abort_flag) {
        ok = false;
        break;
      }
    }
    if (ok) {
      pv_tile<D, G, VB>(ring + (size_t)cs * stage_bytes + VOFF, st, pb, lane);
      __syncwarp();
      ++j;
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

template <int D, int G>
__device__ __forceinline__ void consume_dispatch(int kb, int vb, WarpState<D, G>& st, const uint16_t* qh,
                                                 float scale_log2, uint8_t* ring, int stages, int stage_bytes,
                                                 uint64_t* bars, const uint8_t* src, int rec, int n_my, int warp,
                                                 int lane, volatile int* abort_flag, int* status) {
#define RQ_C(KBV, VBV)                                                                                           \
  consume<D, G, KBV, VBV>(st, qh, scale_log2, ring, stages, stage_bytes, bars, src, rec, n_my, warp, lane, abort_flag, \
                          status)
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
        for (int rr = 0; rr < 2; ++rr) slot[n * D + 16 * mb + 8 * rr + gid] = st.o[mb][rr * 2 + e] * 16777216.0f;
      if (gid == 0) {
        slot[G * D + n] = st.m[e];
        slot[G * D + G + n] = st.l[e] * 16777216.0f;
      }
    }
  }
}

// bf16 sink + recent window on CUDA cores.  The window is split into work
// items of 32 tokens.  Thread 0 stages the item's K and V rows in shared
// memory with at most six 1-D bulk copies (the rows of a chunk form at most
// three contiguous runs: sink, ring, ring after wrap); warp w then takes heads
// w, w + 4, ...: lane = token for q.k (K row words read in a lane-rotated
// order so the 32 rows hit 32 banks), lane = channel for p.v.
constexpr int kWinChunk = 32;

__host__ __device__ inline int window_tokens(int T, int S, int Tq) { return (T < S ? T : S) + (T - (T < S ? T : S) - Tq); }

template <int D>
__device__ __forceinline__ void window_issue_chunk(const DecodeArgs& a, const uint8_t* win, uint32_t* kbuf,
                                                   uint32_t* vbuf, uint64_t* bar, int j0, int cnt) {
  const int S = a.g.S, ring = a.g.R + kTile;
  const int n_sink = a.T < S ? a.T : S;
  mbar_arrive_expect_tx(bar, (uint32_t)(cnt * D * 2 * 2));
  int t = 0;
  while (t < cnt) {
    const int j = j0 + t;
    size_t row;  // K row inside the window block; its V row follows its block's K rows
    int run;
    size_t v_off;
    if (j < n_sink) {
      row = j;
      run = min(cnt - t, n_sink - j);
      v_off = S;
    } else {
      const int slot = (a.Tq + (j - n_sink)) % ring;
      row = (size_t)2 * S + slot;
      run = min(cnt - t, ring - slot);
      v_off = ring;
    }
    bulk_g2s(kbuf + (size_t)t * (D / 2), win + row * D * 2, (uint32_t)(run * D * 2), bar);
    bulk_g2s(vbuf + (size_t)t * (D / 2), win + (row + v_off) * D * 2, (uint32_t)(run * D * 2), bar);
    t += run;
  }
}

template <int D, int G>
__device__ void window_item(const DecodeArgs& a, const uint8_t* win, const uint16_t* qh, int chunk, float* scratch,
                            uint64_t* bar, float* slot, int warp, int lane, volatile int* abort_flag) {
  constexpr int RW = D / 2;  // words per bf16 row
  constexpr int HW = (G + NW - 1) / NW;
  const int tid = warp * 32 + lane;
  const int n_tok = window_tokens(a.T, a.g.S, a.Tq);
  const int j0 = chunk * kWinChunk;
  const int cnt = max(0, min(kWinChunk, n_tok - j0));
  float* qs = scratch;                                              // [G][D]
  uint32_t* kbuf = reinterpret_cast<uint32_t*>(qs + G * D);         // [32][RW]
  uint32_t* vbuf = kbuf + kWinChunk * RW;                           // [32][RW]
  if (tid == 0 && cnt > 0) window_issue_chunk<D>(a, win, kbuf, vbuf, bar, j0, cnt);
  for (int i = tid; i < G * D; i += NW * 32) qs[i] = bf16_bits_to_float(qh[i]);
  const bool ok = cnt == 0 || __all_sync(0xffffffffu, mbar_wait_bounded(bar, 0));
  if (!__syncthreads_and(ok)) {
    if (tid == 0) {
      raise_abort(abort_flag, a.status);
      (void)mbar_wait_bounded(bar, 0);  // let the copies land before the CTA exits
    }
    return;
  }
#pragma unroll
  for (int j = 0; j < HW; ++j) {
    const int h = warp + NW * j;
    float m = -INFINITY, l = 0.0f, o[D / 32];
#pragma unroll
    for (int c = 0; c < D / 32; ++c) o[c] = 0.0f;
    if (h < G && cnt > 0) {
      float acc = 0.0f;
      if (lane < cnt) {
#pragma unroll 8
        for (int w = 0; w < RW; ++w) {
          const int wr = (w + lane) & (RW - 1);
          const uint32_t kk = kbuf[lane * RW + wr];
          acc = fmaf(qs[h * D + 2 * wr], bf16_bits_to_float(kk & 0xFFFFu),
                     fmaf(qs[h * D + 2 * wr + 1], bf16_bits_to_float(kk >> 16), acc));
        }
      }
      const float x = lane < cnt ? acc * a.scale_log2 : -INFINITY;
      m = warp_max(x);
      const float p = ex2(x - m);
      l = warp_sum(p);
      for (int t = 0; t < cnt; ++t) {
        const float pt = __shfl_sync(0xffffffffu, p, t);
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
          const int d = lane + 32 * c;
          const uint32_t vv = vbuf[t * RW + d / 2];
          o[c] = fmaf(pt, (d & 1) ? bf16_bits_to_float(vv >> 16) : bf16_bits_to_float(vv & 0xFFFFu), o[c]);
        }
      }
    }
    if (h < G) {
#pragma unroll
      for (int c = 0; c < D / 32; ++c) slot[h * D + lane + 32 * c] = o[c];
      if (lane == 0) {
        slot[G * D + h] = m;
        slot[G * D + G + h] = l;
      }
    }
  }
  // heads of the other warps: empty partial states
  for (int h = 0; h < G; ++h) {
    if (h % NW == warp) continue;
#pragma unroll
    for (int c = 0; c < D / 32; ++c) slot[h * D + lane + 32 * c] = 0.0f;
    if (lane == 0) {
      slot[G * D + h] = -INFINITY;
      slot[G * D + G + h] = 0.0f;
    }
  }
}

// Log-sum-exp merge of n partial states (stride PART floats from `base`)
// into one: written to `dst` as a partial, or normalised into `outp`.  Each
// thread owns OPT outputs and loads the o, m and l of up to U partials for
// all of them at once (one round of independent loads per U partials).
template <int D, int G>
__device__ void combine_partials(const float* base, int n, float* dst, float* outp, int tid) {
  using C = Cfg<D, G>;
  constexpr int OPT = (G * D + kDecodeThreads - 1) / kDecodeThreads;
  constexpr int U = OPT >= 32 ? 1 : 32 / OPT;  // at most 96 values in flight per thread
  float M[OPT], L[OPT], O[OPT];
#pragma unroll
  for (int k = 0; k < OPT; ++k) {
    M[k] = -INFINITY;
    L[k] = 0.0f;
    O[k] = 0.0f;
  }
  for (int i0 = 0; i0 < n; i0 += U) {
    float ov[OPT][U], mv[OPT][U], lv[OPT][U];
#pragma unroll
    for (int k = 0; k < OPT; ++k) {
      const int idx = tid + k * kDecodeThreads;
      const int hh = idx < G * D ? idx / D : 0;
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const bool ok = idx < G * D && i0 + u < n;
        const float* pp = base + (size_t)(i0 + u) * C::PART;
        ov[k][u] = ok ? __ldcg(pp + idx) : 0.0f;
        mv[k][u] = ok ? __ldcg(pp + G * D + hh) : -INFINITY;
        lv[k][u] = ok ? __ldcg(pp + G * D + G + hh) : 0.0f;
      }
    }
#pragma unroll
    for (int k = 0; k < OPT; ++k) {
      float nm = M[k];
#pragma unroll
      for (int u = 0; u < U; ++u) nm = fmaxf(nm, mv[k][u]);
      if (nm == -INFINITY) continue;
      const float a = ex2(M[k] - nm);  // 0 when M was -inf
      O[k] *= a;
      L[k] *= a;
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const float f = ex2(mv[k][u] - nm);
        O[k] = fmaf(ov[k][u], f, O[k]);
        L[k] = fmaf(lv[k][u], f, L[k]);
      }
      M[k] = nm;
    }
  }
#pragma unroll
  for (int k = 0; k < OPT; ++k) {
    const int idx = tid + k * kDecodeThreads;
    if (idx >= G * D) continue;
    if (outp) {
      outp[idx] = L[k] > 0.0f ? O[k] / L[k] : 0.0f;
    } else {
      dst[idx] = O[k];
      if (idx % D == 0) {
        dst[G * D + idx / D] = M[k];
        dst[G * D + G + idx / D] = L[k];
      }
    }
  }
}

template <int D, int G>
__global__ void __launch_bounds__(kDecodeThreads, 3) decode_kernel(DecodeArgs a) {
  using C = Cfg<D, G>;
  extern __shared__ __align__(128) uint8_t smem[];
  __shared__ uint64_t bars[NW * kMaxStages];
  __shared__ volatile int abort_flag;
  __shared__ int is_last;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int srel = blockIdx.y, item = blockIdx.x;
  const int NI = a.n_splits + a.n_win;  // work items of this stream
  const int NG = (NI + kGroup - 1) / kGroup;
  const int h = srel % a.g.Hkv, b = (srel / a.g.Hkv) % a.g.B, lrel = srel / (a.g.Hkv * a.g.B);
  const int l = a.layer0 + lrel;
  const HeadDesc hd = a.desc[l * a.g.Hkv + h];
  const uint16_t* qh = a.q + ((size_t)(lrel * a.g.B + b) * a.g.Hq + (size_t)h * G) * D;
  float* merge = reinterpret_cast<float*>(smem);  // aliases the stages after the main loop

  if (tid == 0) {
    abort_flag = 0;
    for (int s = 0; s < NW * kMaxStages; ++s) mbar_init(&bars[s], 1);
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
    if (warp < NW)
      consume_dispatch<D, G>(hd.k_bits, hd.v_bits, st, qh, a.scale_log2,
                             smem + (size_t)warp * a.stages * a.stage_bytes, a.stages, a.stage_bytes,
                             bars + warp * kMaxStages, src, rec, n_my, warp, lane, &abort_flag, a.status);
  } else {
    // one 32-token chunk of the bf16 sink + recent window
    const uint8_t* win = a.buf + hd.win_base + (int64_t)b * a.g.win_bytes;
    window_item<D, G>(a, win, qh, item - a.n_splits, merge + NW * C::PART, &bars[0], merge + warp * C::PART, warp,
                      lane, &abort_flag);
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
  // two-level log-sum-exp combine: the last item of each group of kGroup
  // merges the group; the last group merges the group results into out.
  uint32_t* cnt = a.counters + (size_t)srel * kCountersPerStream;
  const int g = item / kGroup;
  const int gsize = min(kGroup, NI - g * kGroup);
  float* outp = a.out + ((size_t)(lrel * a.g.B + b) * a.g.Hq + (size_t)h * G) * D;
  float* gpart = a.partials + (size_t)a.n_streams * NI * C::PART + ((size_t)srel * NG + g) * C::PART;
  __threadfence();
  __syncthreads();
  if (tid == 0) is_last = (atomicAdd(&cnt[1 + g], 1u) == (unsigned)(gsize - 1));
  __syncthreads();
  if (!is_last) return;
  __threadfence();
  combine_partials<D, G>(a.partials + ((size_t)srel * NI + g * kGroup) * C::PART, gsize, gpart,
                         NG == 1 ? outp : nullptr, tid);
  if (tid == 0) cnt[1 + g] = 0u;
  if (NG == 1) return;
  __threadfence();
  __syncthreads();
  if (tid == 0) is_last = (atomicAdd(&cnt[0], 1u) == (unsigned)(NG - 1));
  __syncthreads();
  if (!is_last) return;
  __threadfence();
  combine_partials<D, G>(a.partials + (size_t)a.n_streams * NI * C::PART + (size_t)srel * NG * C::PART, NG,
                         nullptr, outp, tid);
  if (tid == 0) cnt[0] = 0u;
}

template <int D, int G>
cudaError_t launch_dg(const DecodeArgs& a, int smem, cudaStream_t st) {
  cudaError_t e = cudaFuncSetAttribute(decode_kernel<D, G>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  const int streams = a.n_layers * a.g.B * a.g.Hkv;
  dim3 grid(a.n_splits + a.n_win, streams);
  decode_kernel<D, G><<<grid, kDecodeThreads, smem, st>>>(a);
  return cudaGetLastError();
}

}  // namespace

int decode_smem_bytes(int n_items, int stages, int stage_bytes, int G, int D) {
  const int part = G * D + 2 * G;
  // merge slots + window scratch (q, one K and one V chunk)
  int merge = (NW * part + G * D) * 4 + 2 * kWinChunk * D * 2;
  const int ring = NW * stages * stage_bytes;
  int need = ring > merge ? ring : merge;
  return (need + 127) / 128 * 128;
}

template <int D, int G>
int occupancy_dg(int smem) {
  if (cudaFuncSetAttribute(decode_kernel<D, G>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
    return 1;
  int n = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, decode_kernel<D, G>, kDecodeThreads, smem) != cudaSuccess)
    return 1;
  return n > 0 ? n : 1;
}

int decode_occupancy(int D, int G, int smem) {
#define RQ_DG(DD, GG) \
  if (D == DD && G == GG) return occupancy_dg<DD, GG>(smem);
  RQ_DG(128, 1) RQ_DG(128, 2) RQ_DG(128, 4) RQ_DG(128, 8)
  RQ_DG(64, 1) RQ_DG(64, 2) RQ_DG(64, 4) RQ_DG(64, 8)
#undef RQ_DG
  return 1;
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

// ---------------------------------------------------------------------------
// Scratch for rq_decode_attention_noalloc: a file-scope device array, so that
// callers that must not allocate device memory (see include/rq.h) can still
// run the split-K decode.  Every device that loads this library holds it
// until the process exits.  Host code may only use the address returned by
// cudaGetSymbolAddress for the current device, never the array's name.
namespace rq {
namespace {
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_noalloc_mu;
void* g_noalloc_ptr[kMaxDevices] = {};
}  // namespace

cudaError_t noalloc_scratch(void** ptr) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  if (g_noalloc_ptr[dev] == nullptr) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);  // once per device, with that device current
    if (e != cudaSuccess) return e;
    g_noalloc_ptr[dev] = p;
  }
  *ptr = g_noalloc_ptr[dev];
  return cudaSuccess;
}
}  // namespace rq

// Quantize-and-pack kernels: prefill of whole tiles, window copy, and the
// decode-time append with tile flush.
//
// InnerQ grouping (arXiv 2602.23200, abstract / "Core claim"): K groups run
// along head_dim per token (32 channels), V groups along tokens per channel
// (the 32 tokens of a tile).  Asymmetric min/max quantization with an fp16
// scale and a bf16 zero; bit widths 2, 3, 4, 8 per (layer, kv-head).
//
// Every arithmetic step of the rounding rule is an IEEE fp32 operation with
// round-to-nearest-even (__fsub_rn, __fdiv_rn, __frcp_rn, __fmul_rn,
// __float2half_rn, __float2int_rn), so codes and scales are reproducible
// bit for bit on any IEEE machine.
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "rq_device.cuh"
#include "rq_internal.h"

namespace rq {
namespace {

constexpr int kQuantWarps = 4;

template <int D>
struct TileSmem {
  static constexpr int kStride = D / 2 + 4;  // words per staged row (16-byte aligned)
  uint32_t k[kTile][kStride];                // bf16 pairs
  uint32_t v[kTile][kStride];
  float kr[kTile][D / 32];  // 1 / scale per (token, group)
  float kz[kTile][D / 32];  // zero per (token, group)
  float vr[D];
  float vz[D];
  float kinv[D];  // 1 / n per channel (K normalization; powers of two)
};

// Stream's K normalization factors n[D] (fp32), stored after its window rows.
__device__ __forceinline__ float* stream_norm(uint8_t* buf, const HeadDesc& hd, const Geom& g, int b) {
  return reinterpret_cast<float*>(buf + hd.win_base + (int64_t)b * g.win_bytes + window_rows_bytes(g.S, g.R, g.D));
}

// 1 / n of the stream into shared memory (one warp).
template <int D>
__device__ __forceinline__ void stage_kinv(TileSmem<D>& sm, const float* nrm, int lane) {
  for (int d = lane; d < D; d += 32) sm.kinv[d] = 1.0f / nrm[d];
}

__device__ __forceinline__ float lo_bf16(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float hi_bf16(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

// Scale/zero of one group from its min and max; returns the meta word.
template <int B>
__device__ __forceinline__ uint32_t group_params(float mn, float mx, float& r) {
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

// Stage 32 rows of D bf16 (row t at rows[t]) into the smem tile (whole warp).
template <int D>
__device__ __forceinline__ void stage_rows(uint32_t (*dst)[TileSmem<D>::kStride], const uint16_t* const* rows,
                                           int lane) {
  constexpr int kChunks = D / 8;  // 16-byte chunks per row
#pragma unroll 4
  for (int j = lane; j < kTile * kChunks; j += 32) {
    const int t = j / kChunks, c = j % kChunks;
    const uint4 x = __ldg(reinterpret_cast<const uint4*>(rows[t]) + c);
    *reinterpret_cast<uint4*>(&dst[t][c * 4]) = x;
  }
}

template <int D, int KB>
__device__ void pack_k(TileSmem<D>& sm, uint8_t* rec, int lane) {
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
        const uint32_t w = sm.k[t][cw];
        const float x0 = lo_bf16(w) * sm.kinv[2 * cw], x1 = hi_bf16(w) * sm.kinv[2 * cw + 1];
        mn = fminf(mn, fminf(x0, x1));
        mx = fmaxf(mx, fmaxf(x0, x1));
      }
      float r;
      const uint32_t meta = group_params<KB>(mn, mx, r);
      sm.kr[t][grp] = r;
      sm.kz[t][grp] = mn;
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
        const uint32_t x = sm.k[t][d0 / 2];
        const float rr = sm.kr[t][g], z = sm.kz[t][g];
        put_code<KB, W>(words, rho, kh, e, code_of<KB>(lo_bf16(x) * sm.kinv[d0], z, rr));
        put_code<KB, W>(words, rho, kh, e + 1, code_of<KB>(hi_bf16(x) * sm.kinv[d0 + 1], z, rr));
      }
#pragma unroll
  for (int c = 0; c < W / 4; ++c)
    *reinterpret_cast<uint4*>(rec + word_offset(W, lane, 4 * c)) =
        make_uint4(words[4 * c], words[4 * c + 1], words[4 * c + 2], words[4 * c + 3]);
#pragma unroll
  for (int w = 4 * (W / 4); w < W; ++w) *reinterpret_cast<uint32_t*>(rec + word_offset(W, lane, w)) = words[w];
}

template <int D, int VB>
__device__ void pack_v(TileSmem<D>& sm, uint8_t* vrec, int lane) {
  constexpr int W = words_per_lane(VB, D);
  // statistics: each lane owns channel pairs (2w, 2w+1)
#pragma unroll
  for (int w = lane; w < D / 2; w += 32) {
    float mn0 = INFINITY, mx0 = -INFINITY, mn1 = INFINITY, mx1 = -INFINITY;
#pragma unroll 8
    for (int t = 0; t < kTile; ++t) {
      const uint32_t x = sm.v[t][w];
      mn0 = fminf(mn0, lo_bf16(x));
      mx0 = fmaxf(mx0, lo_bf16(x));
      mn1 = fminf(mn1, hi_bf16(x));
      mx1 = fmaxf(mx1, hi_bf16(x));
    }
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int d = 2 * w + h;
      float r;
      const uint32_t meta = group_params<VB>(h ? mn1 : mn0, h ? mx1 : mx0, r);
      sm.vr[d] = r;
      sm.vz[d] = h ? mn1 : mn0;
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
    const float rr = sm.vr[d], z = sm.vz[d];
#pragma unroll
    for (int kh = 0; kh < 2; ++kh)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const uint32_t x = sm.v[4 * kh + tig + 8 * e][d >> 1];
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

template <int D>
__device__ void quantize_staged_tile(TileSmem<D>& sm, int kb, int vb, uint8_t* rec, int lane) {
  switch (kb) {
    case 2: pack_k<D, 2>(sm, rec, lane); break;
    case 3: pack_k<D, 3>(sm, rec, lane); break;
    case 4: pack_k<D, 4>(sm, rec, lane); break;
    default: pack_k<D, 8>(sm, rec, lane); break;
  }
  uint8_t* vrec = rec + blob_bytes(kb, D) + 4 * D;
  switch (vb) {
    case 2: pack_v<D, 2>(sm, vrec, lane); break;
    case 3: pack_v<D, 3>(sm, vrec, lane); break;
    case 4: pack_v<D, 4>(sm, vrec, lane); break;
    default: pack_v<D, 8>(sm, vrec, lane); break;
  }
}

// grid (ceil(tiles / 4), L*B*Hkv); one warp per tile.
template <int D>
__global__ void __launch_bounds__(kQuantWarps * 32) quantize_tiles_kernel(QuantizeArgs a) {
  extern __shared__ __align__(16) uint8_t smem_raw[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n_tiles = a.Tq / kTile;
  const int tile = blockIdx.x * kQuantWarps + warp;
  if (tile >= n_tiles) return;
  const int s = blockIdx.y;
  const int h = s % a.g.Hkv, b = (s / a.g.Hkv) % a.g.B, l = s / (a.g.Hkv * a.g.B);
  const HeadDesc hd = a.desc[l * a.g.Hkv + h];
  TileSmem<D>& sm = reinterpret_cast<TileSmem<D>*>(smem_raw)[warp];
  const size_t row0 = ((size_t)s * a.T + a.g.S + (size_t)tile * kTile) * D;
  const uint16_t* krows[kTile];
  const uint16_t* vrows[kTile];
#pragma unroll
  for (int t = 0; t < kTile; ++t) {
    krows[t] = a.k + row0 + (size_t)t * D;
    vrows[t] = a.v + row0 + (size_t)t * D;
  }
  stage_rows<D>(sm.k, krows, lane);
  stage_rows<D>(sm.v, vrows, lane);
  stage_kinv<D>(sm, stream_norm(a.buf, hd, a.g, b), lane);
  __syncwarp();
  uint8_t* rec = a.buf + hd.tile_base + (int64_t)b * hd.tile_stride + (int64_t)tile * hd.rec_bytes;
  quantize_staged_tile<D>(sm, hd.k_bits, hd.v_bits, rec, lane);
}

// Copy sink tokens [0, min(S,T)) and recent tokens [S+Tq, T) into the window block.
__global__ void copy_window_kernel(QuantizeArgs a) {
  const int s = blockIdx.x;
  const int h = s % a.g.Hkv, b = (s / a.g.Hkv) % a.g.B, l = s / (a.g.Hkv * a.g.B);
  const HeadDesc hd = a.desc[l * a.g.Hkv + h];
  const int D = a.g.D, S = a.g.S, ring = a.g.R + kTile;
  uint8_t* win = a.buf + hd.win_base + (int64_t)b * a.g.win_bytes;
  const int n_sink = a.T < S ? a.T : S;
  const int rows = n_sink + (a.T - n_sink - a.Tq);
  const int chunks = D / 8;
  const size_t src0 = (size_t)s * a.T * D;
  for (int j = threadIdx.x; j < rows * chunks * 2; j += blockDim.x) {
    const int kv = j / (rows * chunks);
    const int rj = (j % (rows * chunks)) / chunks, c = j % chunks;
    int pos, dst_row;
    uint8_t* base;
    if (rj < n_sink) {
      pos = rj;
      dst_row = rj;
      base = win + (size_t)kv * S * D * 2;
    } else {
      pos = S + a.Tq + (rj - n_sink);
      dst_row = (pos - S) % ring;
      base = win + (size_t)2 * S * D * 2 + (size_t)kv * ring * D * 2;
    }
    const uint16_t* src = (kv ? a.v : a.k) + src0 + (size_t)pos * D;
    reinterpret_cast<uint4*>(base + (size_t)dst_row * D * 2)[c] = __ldg(reinterpret_cast<const uint4*>(src) + c);
  }
}

// grid (n_layers*B*Hkv); two warps per stream: warp 0 writes the token, and
// on a flush warp 0 quantizes and packs K while warp 1 does V.
template <int D>
__global__ void __launch_bounds__(64) append_kernel(AppendArgs a) {
  extern __shared__ __align__(16) uint8_t smem_raw[];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int srel = blockIdx.x;
  const int h = srel % a.g.Hkv, b = (srel / a.g.Hkv) % a.g.B, l = a.layer0 + srel / (a.g.Hkv * a.g.B);
  const HeadDesc hd = a.desc[l * a.g.Hkv + h];
  const int S = a.g.S, ring = a.g.R + kTile;
  uint8_t* win = a.buf + hd.win_base + (int64_t)b * a.g.win_bytes;
  uint8_t* kdst;
  uint8_t* vdst;
  if (a.T_old < S) {
    kdst = win + (size_t)a.T_old * D * 2;
    vdst = win + (size_t)(S + a.T_old) * D * 2;
  } else {
    const int slot = (a.T_old - S) % ring;
    kdst = win + ((size_t)2 * S + slot) * D * 2;
    vdst = win + ((size_t)2 * S + ring + slot) * D * 2;
  }
  constexpr int kChunks = D / 8;
  if (tid < kChunks) {
    reinterpret_cast<uint4*>(kdst)[tid] = __ldg(reinterpret_cast<const uint4*>(a.k_new + (size_t)srel * D) + tid);
  } else if (tid < 2 * kChunks) {
    reinterpret_cast<uint4*>(vdst)[tid - kChunks] =
        __ldg(reinterpret_cast<const uint4*>(a.v_new + (size_t)srel * D) + tid - kChunks);
  }
  if (!a.flush) return;
  __syncthreads();
  TileSmem<D>& sm = *reinterpret_cast<TileSmem<D>*>(smem_raw);
  const uint16_t* krows[kTile];
  const uint16_t* vrows[kTile];
#pragma unroll
  for (int t = 0; t < kTile; ++t) {
    const int slot = (a.flush_pos + t - S) % ring;
    krows[t] = reinterpret_cast<const uint16_t*>(win + ((size_t)2 * S + slot) * D * 2);
    vrows[t] = reinterpret_cast<const uint16_t*>(win + ((size_t)2 * S + ring + slot) * D * 2);
  }
  if (warp == 0) stage_kinv<D>(sm, stream_norm(a.buf, hd, a.g, b), lane);
  // rows were just written through global memory by this block: plain loads
#pragma unroll 4
  for (int j = tid; j < kTile * kChunks; j += 64) {
    const int t = j / kChunks, c = j % kChunks;
    *reinterpret_cast<uint4*>(&sm.k[t][c * 4]) = reinterpret_cast<const uint4*>(krows[t])[c];
    *reinterpret_cast<uint4*>(&sm.v[t][c * 4]) = reinterpret_cast<const uint4*>(vrows[t])[c];
  }
  __syncthreads();
  uint8_t* rec = a.buf + hd.tile_base + (int64_t)b * hd.tile_stride + (int64_t)a.flush_tile * hd.rec_bytes;
  if (warp == 0) {
    switch (hd.k_bits) {
      case 2: pack_k<D, 2>(sm, rec, lane); break;
      case 3: pack_k<D, 3>(sm, rec, lane); break;
      case 4: pack_k<D, 4>(sm, rec, lane); break;
      default: pack_k<D, 8>(sm, rec, lane); break;
    }
  } else {
    uint8_t* vrec = rec + blob_bytes(hd.k_bits, D) + 4 * D;
    switch (hd.v_bits) {
      case 2: pack_v<D, 2>(sm, vrec, lane); break;
      case 3: pack_v<D, 3>(sm, vrec, lane); break;
      case 4: pack_v<D, 4>(sm, vrec, lane); break;
      default: pack_v<D, 8>(sm, vrec, lane); break;
    }
  }
}

// Distortion measurement for calibration: for every (head, bit width), the
// sum of squared errors of quantizing and dequantizing the head's samples
// with the rule above (x_hat = c * s + z in fp64).  One warp per group at a
// time (lane = element); K groups are 32 channels of a token, V groups one
// channel over 32 tokens.  Accumulated in fp64 with one atomic per warp.
template <int B>
__device__ double group_sse(float x) {
  float mn = x, mx = x;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, o));
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  }
  float r;
  const uint32_t meta = group_params<B>(mn, mx, r);
  const double s = (double)__half2float(__ushort_as_half((unsigned short)(meta & 0xFFFFu)));
  const double z = (double)__uint_as_float(meta & 0xFFFF0000u);
  const double xh = __dadd_rn(__dmul_rn((double)code_of<B>(x, mn, r), s), z);
  const double e = (double)x - xh;
  return e * e;
}

__global__ void measure_sse_kernel(const uint16_t* x, int n_tokens, int head_dim, int role, int b, int bi,
                                   int n_bits, double* sse) {
  const int head = blockIdx.y;
  const int lane = threadIdx.x & 31;
  const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int n_warps = (gridDim.x * blockDim.x) >> 5;
  const int per_row = head_dim / 32;
  const long n_groups = role == 0 ? (long)n_tokens * per_row : (long)(n_tokens / kTile) * head_dim;
  const uint16_t* xh = x + (size_t)head * n_tokens * head_dim;
  double acc = 0.0;
  for (long gi = warp; gi < n_groups; gi += n_warps) {
    size_t idx;
    if (role == 0) {
      idx = (size_t)(gi / per_row) * head_dim + 32 * (gi % per_row) + lane;
    } else {
      idx = (size_t)(kTile * (gi / head_dim) + lane) * head_dim + gi % head_dim;
    }
    const float v = __uint_as_float((uint32_t)xh[idx] << 16);
    double e2;
    switch (b) {
      case 2: e2 = group_sse<2>(v); break;
      case 3: e2 = group_sse<3>(v); break;
      case 4: e2 = group_sse<4>(v); break;
      default: e2 = group_sse<8>(v); break;
    }
    acc += e2;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
  if (lane == 0) atomicAdd(&sse[(size_t)head * n_bits + bi], acc);
}

__global__ void scale_kernel(double* v, int n, double f) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i < n) v[i] *= f;
}

// K normalization factors of every stream: set to a constant (1 at cache
// initialisation and for prefills without normalization, 0 before a maximum).
__global__ void norm_fill_kernel(uint8_t* buf, const HeadDesc* desc, Geom g, float value) {
  const int s = blockIdx.x;
  const int h = s % g.Hkv, b = (s / g.Hkv) % g.B, l = s / (g.Hkv * g.B);
  const HeadDesc hd = desc[l * g.Hkv + h];
  float* n = stream_norm(buf, hd, g, b);
  for (int d = threadIdx.x; d < g.D; d += blockDim.x) n[d] = value;
}

// max over the prefill tokens of |K[t, d]| per stream and channel, as the
// bits of a non-negative float (ordered like unsigned integers)
__global__ void norm_max_kernel(QuantizeArgs a, int tokens_per_block) {
  const int s = blockIdx.y;
  const int h = s % a.g.Hkv, b = (s / a.g.Hkv) % a.g.B, l = s / (a.g.Hkv * a.g.B);
  const HeadDesc hd = a.desc[l * a.g.Hkv + h];
  const int D = a.g.D;
  const int t0 = blockIdx.x * tokens_per_block, t1 = min(a.T, t0 + tokens_per_block);
  const uint16_t* k = a.k + (size_t)s * a.T * D;
  for (int d = threadIdx.x; d < D; d += blockDim.x) {
    float m = 0.0f;
    for (int t = t0; t < t1; ++t) m = fmaxf(m, fabsf(__uint_as_float((uint32_t)k[(size_t)t * D + d] << 16)));
    atomicMax(reinterpret_cast<unsigned int*>(stream_norm(a.buf, hd, a.g, b)) + d, __float_as_uint(m));
  }
}

// maximum -> smallest power of two >= it (1 for a zero channel)
__global__ void norm_finalize_kernel(QuantizeArgs a) {
  const int s = blockIdx.x;
  const int h = s % a.g.Hkv, b = (s / a.g.Hkv) % a.g.B, l = s / (a.g.Hkv * a.g.B);
  const HeadDesc hd = a.desc[l * a.g.Hkv + h];
  float* n = stream_norm(a.buf, hd, a.g, b);
  for (int d = threadIdx.x; d < a.g.D; d += blockDim.x) {
    const float m = n[d];
    int e = 0;
    const float f = frexpf(m, &e);  // m = f * 2^e, f in [0.5, 1)
    n[d] = m > 0.0f ? ldexpf(1.0f, f == 0.5f ? e - 1 : e) : 1.0f;
  }
}

}  // namespace

cudaError_t launch_norm_reset(uint8_t* buf, const HeadDesc* desc, const Geom& g, cudaStream_t st) {
  norm_fill_kernel<<<g.L * g.B * g.Hkv, 128, 0, st>>>(buf, desc, g, 1.0f);
  return cudaGetLastError();
}

cudaError_t launch_quantize(const QuantizeArgs& a, cudaStream_t st) {
  const int streams = a.g.L * a.g.B * a.g.Hkv;
  // the prefill fixes the K normalization factors before any tile is packed
  if (a.k_norm && a.T > 0) {
    norm_fill_kernel<<<streams, 128, 0, st>>>(a.buf, a.desc, a.g, 0.0f);
    const int tpb = 1024;
    norm_max_kernel<<<dim3((a.T + tpb - 1) / tpb, streams), 128, 0, st>>>(a, tpb);
    norm_finalize_kernel<<<streams, 128, 0, st>>>(a);
  } else {
    norm_fill_kernel<<<streams, 128, 0, st>>>(a.buf, a.desc, a.g, 1.0f);
  }
  cudaError_t e0 = cudaGetLastError();
  if (e0 != cudaSuccess) return e0;
  const int n_tiles = a.Tq / kTile;
  if (n_tiles > 0) {
    dim3 grid((n_tiles + kQuantWarps - 1) / kQuantWarps, streams);
    if (a.g.D == 128) {
      const int smem = kQuantWarps * (int)sizeof(TileSmem<128>);
      cudaFuncSetAttribute(quantize_tiles_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
      quantize_tiles_kernel<128><<<grid, kQuantWarps * 32, smem, st>>>(a);
    } else {
      const int smem = kQuantWarps * (int)sizeof(TileSmem<64>);
      cudaFuncSetAttribute(quantize_tiles_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
      quantize_tiles_kernel<64><<<grid, kQuantWarps * 32, smem, st>>>(a);
    }
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  if (a.T > 0) copy_window_kernel<<<streams, 128, 0, st>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_append(const AppendArgs& a, cudaStream_t st) {
  const int streams = a.n_layers * a.g.B * a.g.Hkv;
  if (a.g.D == 128) {
    const int smem = a.flush ? (int)sizeof(TileSmem<128>) : 0;
    append_kernel<128><<<streams, 64, smem, st>>>(a);
  } else {
    const int smem = a.flush ? (int)sizeof(TileSmem<64>) : 0;
    append_kernel<64><<<streams, 64, smem, st>>>(a);
  }
  return cudaGetLastError();
}

cudaError_t launch_measure_distortion(const uint16_t* x, int n_heads, int n_tokens, int head_dim, int role,
                                      const int* bits, int n_bits, double* mse, cudaStream_t st) {
  cudaError_t e = cudaMemsetAsync(mse, 0, sizeof(double) * (size_t)n_heads * n_bits, st);
  if (e != cudaSuccess) return e;
  for (int bi = 0; bi < n_bits; ++bi) {
    measure_sse_kernel<<<dim3(64, n_heads), 256, 0, st>>>(x, n_tokens, head_dim, role, bits[bi], bi, n_bits, mse);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  const int n = n_heads * n_bits;
  scale_kernel<<<(n + 255) / 256, 256, 0, st>>>(mse, n, 1.0 / ((double)n_tokens * head_dim));
  return cudaGetLastError();
}

}  // namespace rq

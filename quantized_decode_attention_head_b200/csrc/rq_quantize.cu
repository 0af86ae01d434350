// Quantize-and-pack kernels: prefill of whole tiles, window copy, and the
// decode-time append with tile flush (the tile rule itself is in
// rq_pack.cuh).
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "rq_device.cuh"
#include "rq_internal.h"
#include "rq_pack.cuh"

namespace rq {
namespace {

constexpr int kQuantWarps = 4;

// Prefill: one warp stages and packs K, then V, through one half tile, so
// that five 4-warp CTAs fit an SM.
template <int D>
struct PrefillSmem {
  HalfTile<D> t;
  float kinv[D];
};

// 16-byte asynchronous copy global -> shared through L2 (not L1): no
// register holds the data, so a thread can have many in flight.
__device__ __forceinline__ void cp_async16(void* dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(smem_u32(dst)), "l"(src) : "memory");
}
// Waits until every cp.async copy of the executing thread has landed.
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;\n" ::: "memory"); }

// Stage 32 consecutive rows of D bf16 (row t at base + t * D) into the smem
// tile (whole warp): every 16-byte chunk of the lane is in flight at once
// (asynchronous copies, no register round trip -- measured 16 % faster on the
// long-context prefill and 21 % on Mistral-7B-b64 than loads through
// registers in batches of eight); returns when the lane's chunks have landed,
// and the caller's __syncwarp makes all of them visible to the warp.
template <int D>
__device__ __forceinline__ void stage_rows_contig(uint32_t (*dst)[HalfTile<D>::kStride], const uint16_t* base,
                                                  int lane) {
  constexpr int kChunks = D / 8;  // 16-byte chunks per row
  const uint4* src = reinterpret_cast<const uint4*>(base);
#pragma unroll
  for (int j = lane; j < kTile * kChunks; j += 32) cp_async16(&dst[j / kChunks][(j % kChunks) * 4], src + j);
  cp_async_wait_all();
}

// grid (ceil(tiles / 4), L*B*Hkv); one warp per tile: K rows staged and
// packed, then V rows through the same buffer.  KN: the cache normalizes K.
constexpr int kQuantMinBlocks = 5;
template <int D, bool KN>
__global__ void __launch_bounds__(kQuantWarps * 32, kQuantMinBlocks) quantize_tiles_kernel(QuantizeArgs a) {
  extern __shared__ __align__(16) uint8_t smem_raw[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n_tiles = a.Tq / kTile;
  const int tile = blockIdx.x * kQuantWarps + warp;
  if (tile >= n_tiles) return;
  const int s = blockIdx.y;
  const int h = s % a.g.Hkv, b = (s / a.g.Hkv) % a.g.B, l = s / (a.g.Hkv * a.g.B);
  const HeadDesc hd = a.desc[l * a.g.Hkv + h];
  PrefillSmem<D>& sm = reinterpret_cast<PrefillSmem<D>*>(smem_raw)[warp];
  const size_t row0 = ((size_t)s * a.T + a.g.S + (size_t)tile * kTile) * D;
  // the V rows are staged after the K rows are packed: start bringing them
  // into L2 now (Mistral-7B-b64 prefill 2.35 -> 2.18 ms)
  if (lane == 0) l2_prefetch(a.v + row0, (uint32_t)(kTile * D * 2));
  stage_rows_contig<D>(sm.t.x, a.k + row0, lane);
  if (KN) stage_kinv<D>(sm.kinv, stream_norm(a.buf, hd, a.g, b), lane);
  __syncwarp();
  uint8_t* rec = a.buf + hd.tile_base + (int64_t)b * hd.tile_stride + (int64_t)tile * hd.rec_bytes;
  pack_k_dispatch<D, KN>(sm.t, sm.kinv, hd.k_bits, rec, lane, a.g.hybrid);
  __syncwarp();  // every lane has read the K rows and statistics
  stage_rows_contig<D>(sm.t.x, a.v + row0, lane);
  __syncwarp();
  pack_v_dispatch<D>(sm.t, hd.v_bits, rec + blob_bytes(hd.k_bits, D) + 4 * D, lane, a.g.hybrid);
}

// Copy sink tokens [0, min(S,T)) and recent tokens [S+Tq, T) into the window
// block.  grid (streams, Y): the stream's 16-byte chunks (K and V rows) are
// spread over Y blocks, one or two chunks per thread, so that the copy is a
// few load latencies long rather than a chain of them.
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
  for (int j = blockIdx.y * blockDim.x + threadIdx.x; j < rows * chunks * 2; j += gridDim.y * blockDim.x) {
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
  if (warp == 0) stage_kinv<D>(sm.kinv, stream_norm(a.buf, hd, a.g, b), lane);
  // rows were just written through global memory by this block: plain loads
#pragma unroll 4
  for (int j = tid; j < kTile * kChunks; j += 64) {
    const int t = j / kChunks, c = j % kChunks;
    *reinterpret_cast<uint4*>(&sm.k.x[t][c * 4]) = reinterpret_cast<const uint4*>(krows[t])[c];
    *reinterpret_cast<uint4*>(&sm.v.x[t][c * 4]) = reinterpret_cast<const uint4*>(vrows[t])[c];
  }
  __syncthreads();
  uint8_t* rec = a.buf + hd.tile_base + (int64_t)b * hd.tile_stride + (int64_t)a.flush_tile * hd.rec_bytes;
  if (warp == 0) {
    pack_k_dispatch<D, true>(sm.k, sm.kinv, hd.k_bits, rec, lane, a.g.hybrid);
  } else {
    pack_v_dispatch<D>(sm.v, hd.v_bits, rec + blob_bytes(hd.k_bits, D) + 4 * D, lane, a.g.hybrid);
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
  const uint32_t meta = group_params<B>(mn, mx, r, false);
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

template <int D>
void launch_tiles(const QuantizeArgs& a, dim3 grid, cudaStream_t st) {
  const int smem = kQuantWarps * (int)sizeof(PrefillSmem<D>);
  if (a.k_norm) {
    cudaFuncSetAttribute(quantize_tiles_kernel<D, true>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    quantize_tiles_kernel<D, true><<<grid, kQuantWarps * 32, smem, st>>>(a);
  } else {
    cudaFuncSetAttribute(quantize_tiles_kernel<D, false>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    quantize_tiles_kernel<D, false><<<grid, kQuantWarps * 32, smem, st>>>(a);
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
  // (a cache without normalization keeps the factors of 1 that
  // rq_cache_init wrote: no launch)
  if (a.k_norm && a.T > 0) {
    norm_fill_kernel<<<streams, 128, 0, st>>>(a.buf, a.desc, a.g, 0.0f);
    const int tpb = 1024;
    norm_max_kernel<<<dim3((a.T + tpb - 1) / tpb, streams), 128, 0, st>>>(a, tpb);
    norm_finalize_kernel<<<streams, 128, 0, st>>>(a);
  } else if (a.k_norm) {
    norm_fill_kernel<<<streams, 128, 0, st>>>(a.buf, a.desc, a.g, 1.0f);
  }
  cudaError_t e0 = cudaGetLastError();
  if (e0 != cudaSuccess) return e0;
  const int n_tiles = a.Tq / kTile;
  if (n_tiles > 0) {
    dim3 grid((n_tiles + kQuantWarps - 1) / kQuantWarps, streams);
    if (a.g.D == 128) {
      launch_tiles<128>(a, grid, st);
    } else {
      launch_tiles<64>(a, grid, st);
    }
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  if (a.T > 0) {
    const int n_sink = a.T < a.g.S ? a.T : a.g.S;
    const int rows = n_sink + (a.T - n_sink - a.Tq);
    const int items = rows * (a.g.D / 8) * 2;
    int y = (items + 127) / 128;
    y = y < 1 ? 1 : (y > 65535 ? 65535 : y);  // the loop strides over any remainder
    copy_window_kernel<<<dim3(streams, y), 128, 0, st>>>(a);
  }
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

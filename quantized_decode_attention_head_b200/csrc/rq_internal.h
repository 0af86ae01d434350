// Internal declarations shared by the host library and the CUDA kernels.
// Not part of the public C ABI (include/rq.h).
#pragma once

#include <cstddef>
#include <cstdint>

#include <cuda_runtime.h>

namespace rq {

constexpr int kTile = 32;          // tokens per packed tile == group size
constexpr int kHeaderAlign = 256;  // alignment of every region of the cache buffer

// One descriptor per (layer, kv-head), stored at the start of the device buffer.
struct HeadDesc {
  int32_t k_bits;
  int32_t v_bits;
  int32_t rec_bytes;   // bytes of one packed tile record
  int32_t pad;
  int64_t tile_base;   // byte offset of batch element 0's tile records
  int64_t tile_stride; // bytes between batch elements (max_tiles * rec_bytes)
  int64_t win_base;    // byte offset of batch element 0's window block
};
static_assert(sizeof(HeadDesc) == 40, "HeadDesc layout");

struct Geom {
  int L, B, Hq, Hkv, D, G, S, R;
  int max_tiles;
  int hybrid;          // per-group symmetric / asymmetric choice (group_params)
  int64_t win_bytes;   // bytes of one stream's window block
};

// codes per 32-bit word for a bit width
__host__ __device__ constexpr int codes_per_word(int b) { return b == 2 ? 16 : b == 3 ? 10 : b == 4 ? 8 : 4; }
__host__ __device__ constexpr int words_per_lane(int b, int d) { return (d + codes_per_word(b) - 1) / codes_per_word(b); }
__host__ __device__ constexpr int blob_bytes(int b, int d) { return words_per_lane(b, d) * 128; }
__host__ __device__ constexpr int record_bytes(int kb, int vb, int d) {
  return blob_bytes(kb, d) + 4 * d + blob_bytes(vb, d) + 4 * d;
}

// Window block of one stream: [sink K][sink V][ring K][ring V] bf16 rows of D,
// then the per-channel K normalization factors n[D] (fp32).
__host__ __device__ inline int64_t window_rows_bytes(int S, int R, int D) {
  return (int64_t)(2 * S + 2 * (R + kTile)) * D * 2;
}
__host__ __device__ inline int64_t window_bytes(int S, int R, int D) { return window_rows_bytes(S, R, D) + 4 * D; }

// Quantized token count for T tokens (multiple of 32; recent window in [R, R+32)).
__host__ __device__ inline int quantized_tokens(int T, int S, int R) {
  return T >= S + R ? ((T - S - R) / kTile) * kTile : 0;
}

struct QuantizeArgs {
  Geom g;
  uint8_t* buf;
  const HeadDesc* desc;
  const uint16_t* k;   // [L][B][Hkv][T][D]
  const uint16_t* v;
  int T;
  int Tq;
  int k_norm;          // set n from the prefill (1) or to 1 (0)
};

struct AppendArgs {
  Geom g;
  uint8_t* buf;
  const HeadDesc* desc;
  const uint16_t* k_new;  // [nL][B][Hkv][D]
  const uint16_t* v_new;
  int layer0, n_layers;
  int T_old;              // length before the append
  int flush;              // 1: quantize ring positions [flush_pos, flush_pos+32) into tile flush_tile
  int flush_pos;
  int flush_tile;
};

struct DecodeArgs {
  Geom g;
  uint8_t* buf;
  const HeadDesc* desc;
  const uint16_t* q;      // [nL][B][Hq][D]
  float* out;             // [nL][B][Hq][D]
  float scale_log2;       // softmax scale * log2(e)
  int layer0, n_layers;
  int T, Tq, n_tiles;
  int n_splits;           // tile splits: items [0, n_splits)
  int n_win;              // bf16 window items (32 tokens each): items [n_splits, n_splits + n_win)
  int n_pack;             // 1: item n_splits + n_win packs the tile the next append completes
  int pack_pos;           // its first token (absolute position) and its tile slot
  int pack_tile;
  int n_streams;          // streams of this call
  int cluster;            // CTAs per thread-block cluster: kDecodeCluster or 1
  int q_terms;            // s8 terms of the fixed-point query: 2 (16 bits) or 3 (24 bits, K-normalized caches)
  int win_chunks;         // 32-token window chunks per window item
  int stages;             // per-warp ring depth (2..8)
  int stage_bytes;        // bytes per stage (max record size in the call)
  float* partials;        // [streams][n_splits+1][G*D + 2G]
  uint32_t* counters;     // [streams]
  int* status;            // workspace status word
  const uint16_t* k_new;  // fused append: the token added in this call, [nL][B][Hkv][D] (else null)
  const uint16_t* v_new;
};

// Split-K combine.  The automatic plan runs single-CTA items (cluster 1):
// each publishes its partial, and the last to finish merges them (two levels
// past kOneLevelItems items).  An explicit split count runs the items of a
// stream (tile splits, then window chunks) in thread-block clusters of
// `cluster` consecutive items (the grid padded with empty items to whole
// clusters); a cluster merges its items through distributed shared memory,
// and the CTAs of the last cluster of the stream to finish merge the cluster
// partials, each a slice of the outputs.  Per stream counter [0] counts
// finished items, groups or clusters.
#ifndef RQ_DECODE_CLUSTER
#define RQ_DECODE_CLUSTER 4
#endif
constexpr int kDecodeCluster = RQ_DECODE_CLUSTER;
// decode launches allow programmatic dependent launch (1) or not (0)
#ifndef RQ_DECODE_PDL
#define RQ_DECODE_PDL 1
#endif
constexpr int kCountersPerStream = 64;
constexpr int kMaxItems = 496;
// Most tiles per work item (32 per warp).  A warp keeps P in 16-bit fixed
// point relative to its running maximum; over many tokens that maximum sits
// far above most scores and the rounding of the small probabilities grows
// (measured on a 33K-token stream: 256 tiles per warp exceed max-abs 2e-3,
// 32 stay near a third of it).  Every plan splits a stream into items of at
// most this many tiles; calls that run in several waves use items of this
// size.
constexpr int kMaxTilesPerItem = 128;
inline int min_splits(int n_tiles) { return (n_tiles + kMaxTilesPerItem - 1) / kMaxTilesPerItem; }
__host__ __device__ inline int cluster_items(int items, int cluster) {
  return (items + cluster - 1) / cluster * cluster;
}

// Floats of one partial softmax state (o[G][D], m[G], l[G]), padded to a
// multiple of four so that every partial starts on a 16-byte boundary.
__host__ __device__ constexpr int partial_floats(int G, int D) { return (G * D + 2 * G + 3) / 4 * 4; }
// Single-CTA items (cluster 1) of a stream: up to kOneLevelItems, the last
// item to finish merges all partials into the output (one round of loads);
// beyond, they merge in groups of kMergeGroup: the last item of a group to
// finish merges the group into one more partial, the last group merger
// merges the group partials into the output.
constexpr int kMergeGroup = 8;
constexpr int kOneLevelItems = 16;
__host__ __device__ inline int merge_groups(int items) {
  return items > kOneLevelItems ? (items + kMergeGroup - 1) / kMergeGroup : 0;
}
// partial slots of one stream: one per item plus one per merge group
__host__ __device__ inline int partial_slots(int items) { return items + merge_groups(items); }

// Workspace layout (bytes): [status int32, pad to 256][kCountersPerStream u32
// counters per stream of the whole cache (L*B*Hkv): [0] items or groups
// merged, [1 + group] items of a merge group finished][partials of one call:
// [stream][partial_slots(items)][partial_floats(G, D)] = o, m, l (cluster
// partials use the first items' slots)].  The counter region is sized for
// every stream so calls with different layer arguments never overlap.
inline size_t ws_counter_offset() { return 256; }
inline size_t ws_partial_offset(int64_t all_streams) {
  return ws_counter_offset() + (size_t)all_streams * kCountersPerStream * 4;
}
inline size_t ws_total_bytes(int64_t all_streams, int64_t call_streams, int items, int G, int D) {
  return ws_partial_offset(all_streams) + (size_t)call_streams * partial_slots(items) * (size_t)partial_floats(G, D) * 4;
}
// bf16 window tokens of a T-token cache and the number of window work items
// of `per` chunks of 32 tokens each (at least one item).  A one-wave plan
// takes two chunks per item: both copies start at once, so an item waits for
// one round trip and the window items stay off the critical path (measured
// on the Llama-3-8B decode: 14.7 us at 2, 15.4 at 3, 17.5 at 4).  A plan of
// several waves takes the whole window in one item: its CTAs compete for
// slots, and fewer, longer window items cost less slot time; so does a
// one-wave plan whose tile items are long enough to hide it.
constexpr int kWinChunksOneWave = 2;
constexpr int kWinChunksWaves = 8;
// A one-wave plan whose tile items hold at least this many tiles (10 per
// warp) also takes the whole window in one item.
constexpr int kWholeWindowTiles = 40;
inline int window_items(int T, int S, int R, int per) {
  const int n_tok = T - quantized_tokens(T, S, R);
  const int chunks = (n_tok + kTile - 1) / kTile;
  const int n = (chunks + per - 1) / per;
  return n > 0 ? n : 1;
}

// Kernel launchers (rq_kernels.cu).  Return cudaGetLastError() after launch.
cudaError_t launch_quantize(const QuantizeArgs& a, cudaStream_t s);
// Sets every stream's K normalization factors to 1 (cache initialisation).
cudaError_t launch_norm_reset(uint8_t* buf, const HeadDesc* desc, const Geom& g, cudaStream_t s);
cudaError_t launch_append(const AppendArgs& a, cudaStream_t s);
// Mean squared quantization error per (head, bit width) of bf16 samples
// x [n_heads][n_tokens][head_dim]; role 0 = K groups, 1 = V groups.
cudaError_t launch_measure_distortion(const uint16_t* x, int n_heads, int n_tokens, int head_dim, int role,
                                      const int* bits, int n_bits, double* mse, cudaStream_t s);
cudaError_t launch_decode(const DecodeArgs& a, int smem_bytes, cudaStream_t s);
int decode_smem_bytes(int n_items, int stages, int stage_bytes, int G, int D);
// shared memory the non-ring roles of a decode CTA need (the rings may use it)
int decode_free_bytes(int G, int D);
// CTAs of the decode kernel resident on the device at once, in whole clusters
// of `cluster` CTAs
int decode_resident_ctas(int D, int G, int cluster, int smem_bytes, int q_terms);

// One-thread kernel whose bounded mbarrier wait runs out after limit_ns and
// records kDeviceTimeout in *status (self-test of the timeout path).
cudaError_t launch_wait_timeout_selftest(int* status, unsigned long long limit_ns, cudaStream_t s);

// Size of the device array behind rq_decode_attention_noalloc (bytes).
constexpr size_t kNoAllocScratchBytes = size_t(32) << 20;
// Address of that array on the current device (looked up once per device).
cudaError_t noalloc_scratch(void** ptr);

constexpr int kDecodeConsumerWarps = 4;
// CTAs per SM the decode kernel's registers are sized for, and the bytes of
// tile records in flight per warp
#ifndef RQ_DECODE_MIN_BLOCKS
#define RQ_DECODE_MIN_BLOCKS 4
#endif
#ifndef RQ_STAGE_BUDGET
#define RQ_STAGE_BUDGET 6144
#endif
constexpr int kDecodeThreads = kDecodeConsumerWarps * 32;
// per-warp ring depth: about 6 KB of records in flight per warp (2 to 8)
inline int decode_stages(int stage_bytes) {
  const int p = RQ_STAGE_BUDGET / stage_bytes;
  return p < 2 ? 2 : (p > 8 ? 8 : p);
}
constexpr int kDeviceTimeout = 7;  // == RQ_ERR_DEVICE_TIMEOUT

}  // namespace rq

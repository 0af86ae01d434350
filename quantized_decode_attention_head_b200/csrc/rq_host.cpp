// Host side of the C ABI: argument checks, the cache buffer layout, length
// bookkeeping and kernel launches.  See include/rq.h for the contract.
#include <cmath>
#include <cstring>
#include <new>
#include <vector>

#include <cuda_runtime.h>

#include "rq.h"
#include "rq_internal.h"

using rq::HeadDesc;

struct rq_cache {
  rq::Geom g;
  int max_tokens;
  std::vector<int> k_bits, v_bits;
  std::vector<HeadDesc> desc;  // host copy of the device header
  uint8_t* buf;
  size_t bytes;
  std::vector<int> length;  // tokens per layer
  // per layer: the length at which a fused step packed the tile that the
  // next append completes (-1: none), see rq_decode_step
  std::vector<int> packed_ahead;
  int sm_count;
  int k_norm;               // per-channel K normalization set by the prefill
};

namespace {

size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }
// Device arguments the kernels move in 16-byte vectors or bulk copies.
bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool valid_bits(int b) { return b == 2 || b == 3 || b == 4 || b == 8; }

rq_status check_config(const rq_cache_config* c) {
  if (!c || !c->k_bits || !c->v_bits) return RQ_ERR_INVALID_ARG;
  if (c->n_layers < 1 || c->batch < 1 || c->n_q_heads < 1 || c->n_kv_heads < 1 || c->n_sink < 0 ||
      c->n_recent < 0 || c->max_tokens < 0)
    return RQ_ERR_INVALID_ARG;
  if (c->head_dim != 64 && c->head_dim != 128) return RQ_ERR_UNSUPPORTED;
  if (c->group != rq::kTile) return RQ_ERR_UNSUPPORTED;
  if (c->n_q_heads % c->n_kv_heads != 0) return RQ_ERR_UNSUPPORTED;
  const int G = c->n_q_heads / c->n_kv_heads;
  if (G != 1 && G != 2 && G != 4 && G != 8) return RQ_ERR_UNSUPPORTED;
  for (int i = 0; i < c->n_layers * c->n_kv_heads; ++i)
    if (!valid_bits(c->k_bits[i]) || !valid_bits(c->v_bits[i])) return RQ_ERR_UNSUPPORTED;
  return RQ_OK;
}

// Computes the geometry, the per-(layer, kv-head) descriptors and the total size.
size_t layout(const rq_cache_config* c, rq::Geom& g, std::vector<HeadDesc>& desc) {
  g.L = c->n_layers;
  g.B = c->batch;
  g.Hq = c->n_q_heads;
  g.Hkv = c->n_kv_heads;
  g.D = c->head_dim;
  g.G = c->n_q_heads / c->n_kv_heads;
  g.S = c->n_sink;
  g.R = c->n_recent;
  g.max_tiles = rq::quantized_tokens(c->max_tokens, g.S, g.R) / rq::kTile;
  g.hybrid = c->hybrid ? 1 : 0;
  g.win_bytes = rq::window_bytes(g.S, g.R, g.D);
  const int nh = g.L * g.Hkv;
  desc.assign(nh, HeadDesc{});
  size_t off = align_up((size_t)nh * sizeof(HeadDesc), rq::kHeaderAlign);
  for (int i = 0; i < nh; ++i) {
    HeadDesc& d = desc[i];
    d.k_bits = c->k_bits[i];
    d.v_bits = c->v_bits[i];
    d.rec_bytes = rq::record_bytes(d.k_bits, d.v_bits, g.D);
    d.tile_base = (int64_t)off;
    d.tile_stride = (int64_t)g.max_tiles * d.rec_bytes;
    off = align_up(off + (size_t)g.B * d.tile_stride, rq::kHeaderAlign);
  }
  for (int i = 0; i < nh; ++i) {
    desc[i].win_base = (int64_t)off;
    off = align_up(off + (size_t)g.B * g.win_bytes, rq::kHeaderAlign);
  }
  return off;
}

bool layer_range(const rq_cache* c, int layer, int& l0, int& nl) {
  if (layer == -1) {
    l0 = 0;
    nl = c->g.L;
    for (int l = 1; l < c->g.L; ++l)
      if (c->length[l] != c->length[0]) return false;
    return true;
  }
  if (layer < 0 || layer >= c->g.L) return false;
  l0 = layer;
  nl = 1;
  return true;
}

// Largest record among the heads of layers [l0, l0 + nl).
int max_record(const rq_cache* c, int l0, int nl) {
  int r = 16;
  for (int l = l0; l < l0 + nl; ++l)
    for (int h = 0; h < c->g.Hkv; ++h) r = c->desc[l * c->g.Hkv + h].rec_bytes > r ? c->desc[l * c->g.Hkv + h].rec_bytes : r;
  return r;
}

// Tile splits per stream and cluster size of a decode call (auto mode):
// single-CTA items (no cluster barrier holds a slot, the cluster scheduler
// leaves no slot empty), merged by the last items to finish.  One wave when
// every stream gets at least two tile items of at most kMaxTilesPerItem tiles
// besides its window items; several waves of items of kMaxTilesPerItem tiles
// otherwise.  (Explicit split counts run in clusters of kDecodeCluster.)
int auto_splits(const rq_cache* c, int streams, int n_tiles, int stage_bytes, int n_win, int* cluster,
                bool* one_wave_plan = nullptr) {
  *cluster = 1;
  if (one_wave_plan) *one_wave_plan = false;
  if (n_tiles <= 0) return 0;
  const int smem = rq::decode_smem_bytes(2, rq::decode_stages(stage_bytes),
                                         stage_bytes, c->g.G, c->g.D);
  const long slots1 = rq::decode_resident_ctas(c->g.D, c->g.G, 1, smem, c->k_norm ? 3 : 2);
  const int need = rq::min_splits(n_tiles);
  const int max_by_work = n_tiles / 8 > need ? n_tiles / 8 : need;  // keep a CTA's pipeline busy
  long s;
  const long one_wave = slots1 / streams - n_win;
  if (one_wave >= 2 && one_wave >= need) {
    // one wave: each stream takes an equal share of the resident slots, so
    // every SM holds the same number of equally sized tile items
    s = one_wave;
    if (one_wave_plan) *one_wave_plan = true;
  } else {
    s = need;  // several waves
  }
  if (s > max_by_work) s = max_by_work;
  if (s > n_tiles) s = n_tiles;
  return (int)s;
}

// The last failing CUDA call of this thread (rq_last_cuda_error).
thread_local cudaError_t g_last_cuda_error = cudaSuccess;
void note_cuda_error(cudaError_t e) {
  if (e != cudaSuccess) g_last_cuda_error = e;
}

rq_status cuda_status(cudaError_t e) {
  note_cuda_error(e);
  return e == cudaSuccess ? RQ_OK : RQ_ERR_CUDA;
}

// Decode arguments for layers [l0, l0 + nl) of a cache holding T tokens, with
// the workspace checked and partitioned; the fused-append pointers are null.
rq_status fill_decode(const rq_cache* c, int l0, int nl, int T, const void* q, float* out, float softmax_scale,
                      int n_splits, void* workspace, size_t ws_bytes, rq::DecodeArgs& a, int& smem,
                      int n_pack = 0) {
  const int Tq = rq::quantized_tokens(T, c->g.S, c->g.R);
  const int n_tiles = Tq / rq::kTile;
  const int streams = nl * c->g.B * c->g.Hkv;
  if (streams > 65535) return RQ_ERR_UNSUPPORTED;
  const int stage_bytes = max_record(c, l0, nl);
  // window items of two chunks, unless the automatic plan runs in several
  // waves (then one item takes the whole window)
  int win_chunks = rq::kWinChunksOneWave;
  int n_win = rq::window_items(T, c->g.S, c->g.R, win_chunks);
  int cluster = rq::kDecodeCluster;  // explicit split counts run in clusters
  int splits = n_splits;
  if (n_splits == 0) {
    bool one_wave = false;
    splits = auto_splits(c, streams, n_tiles, stage_bytes, n_win + n_pack, &cluster, &one_wave);
    if (!one_wave && n_tiles > 0) {
      win_chunks = rq::kWinChunksWaves;
      n_win = rq::window_items(T, c->g.S, c->g.R, win_chunks);
    } else if (one_wave && splits > 0 && n_tiles / splits >= rq::kWholeWindowTiles) {
      // long tile items: one window item of the whole window finishes well
      // before them, and the slots it frees go to tile items
      win_chunks = rq::kWinChunksWaves;
      n_win = rq::window_items(T, c->g.S, c->g.R, win_chunks);
      splits = auto_splits(c, streams, n_tiles, stage_bytes, n_win + n_pack, &cluster, &one_wave);
    }
  }
  a.cluster = cluster;
  if (splits < rq::min_splits(n_tiles)) splits = rq::min_splits(n_tiles);  // at most kMaxTilesPerItem per item
  if (splits > n_tiles) splits = n_tiles;
  if (n_tiles > 0 && splits < 1) splits = 1;
  const int items = splits + n_win + n_pack;
  if (rq::cluster_items(items, cluster) > rq::kMaxItems) return RQ_ERR_UNSUPPORTED;
  const int64_t all_streams = (int64_t)c->g.L * c->g.B * c->g.Hkv;
  if (ws_bytes < rq::ws_total_bytes(all_streams, streams, items, c->g.G, c->g.D)) return RQ_ERR_WORKSPACE;
  a.g = c->g;
  a.buf = c->buf;
  a.desc = reinterpret_cast<const HeadDesc*>(c->buf);
  a.q = static_cast<const uint16_t*>(q);
  a.out = out;
  const float scale = softmax_scale > 0.0f ? softmax_scale : 1.0f / std::sqrt((float)c->g.D);
  a.scale_log2 = scale * 1.4426950408889634f;
  a.layer0 = l0;
  a.n_layers = nl;
  a.T = T;
  a.Tq = Tq;
  a.n_tiles = n_tiles;
  a.n_splits = splits;
  a.n_win = n_win;
  a.win_chunks = win_chunks;
  a.n_pack = n_pack;
  a.pack_pos = 0;
  a.pack_tile = 0;
  a.n_streams = streams;
  // K-normalized caches fold the channel factors into the query, which widens
  // its range: 24-bit fixed point there, 16-bit otherwise
  a.q_terms = c->k_norm ? 3 : 2;
  a.stages = rq::decode_stages(stage_bytes);
  a.stage_bytes = stage_bytes;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  a.status = reinterpret_cast<int*>(ws);
  a.counters = reinterpret_cast<uint32_t*>(ws + rq::ws_counter_offset());
  a.partials = reinterpret_cast<float*>(ws + rq::ws_partial_offset(all_streams));
  a.k_new = nullptr;
  a.v_new = nullptr;
  smem = rq::decode_smem_bytes(items, a.stages, stage_bytes, c->g.G, c->g.D);
  if (smem > 227 * 1024) return RQ_ERR_UNSUPPORTED;
  return RQ_OK;
}

}  // namespace

extern "C" {

const char* rq_status_string(rq_status s) {
  switch (s) {
    case RQ_OK: return "ok";
    case RQ_ERR_INVALID_ARG: return "invalid argument";
    case RQ_ERR_UNSUPPORTED: return "unsupported configuration";
    case RQ_ERR_INFEASIBLE_BUDGET: return "infeasible bit budget";
    case RQ_ERR_CAPACITY: return "capacity exceeded";
    case RQ_ERR_WORKSPACE: return "workspace too small";
    case RQ_ERR_CUDA: return "CUDA error";
    case RQ_ERR_DEVICE_TIMEOUT: return "device wait timed out";
  }
  return "unknown status";
}

const char* rq_last_cuda_error(void) {
  return g_last_cuda_error == cudaSuccess ? "no error" : cudaGetErrorString(g_last_cuda_error);
}

const char* rq_build_info(void) {
  return "librq: sm_100a; quantize/pack, append/flush, split-K mma.sync decode with bulk-copy pipeline";
}

rq_status rq_cache_bytes(const rq_cache_config* cfg, size_t* bytes) {
  if (!bytes) return RQ_ERR_INVALID_ARG;
  const rq_status st = check_config(cfg);
  if (st != RQ_OK) return st;
  rq::Geom g;
  std::vector<HeadDesc> desc;
  *bytes = layout(cfg, g, desc);
  return RQ_OK;
}

rq_status rq_cache_init(const rq_cache_config* cfg, void* dev_buf, size_t bytes, rq_cache** out,
                        cudaStream_t stream) {
  if (!out || !dev_buf) return RQ_ERR_INVALID_ARG;
  const rq_status st = check_config(cfg);
  if (st != RQ_OK) return st;
  if (reinterpret_cast<uintptr_t>(dev_buf) % rq::kHeaderAlign != 0) return RQ_ERR_INVALID_ARG;
  rq_cache* c = new (std::nothrow) rq_cache();
  if (!c) return RQ_ERR_INVALID_ARG;
  const size_t need = layout(cfg, c->g, c->desc);
  if (bytes < need) {
    delete c;
    return RQ_ERR_CAPACITY;
  }
  c->max_tokens = cfg->max_tokens;
  c->k_bits.assign(cfg->k_bits, cfg->k_bits + c->g.L * c->g.Hkv);
  c->v_bits.assign(cfg->v_bits, cfg->v_bits + c->g.L * c->g.Hkv);
  c->buf = static_cast<uint8_t*>(dev_buf);
  c->bytes = bytes;
  c->length.assign(c->g.L, 0);
  c->packed_ahead.assign(c->g.L, -1);
  int dev = 0;
  c->sm_count = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess && n > 0) c->sm_count = n;
  }
  c->k_norm = cfg->k_norm ? 1 : 0;
  // The header copy and the reset of the normalization factors (to 1: a cache
  // built by appends only) are queued on the caller's stream -- the stream on
  // which the buffer is valid (a stream-ordered allocator may hand out memory
  // whose previous users are still queued there) -- like every other call.
  // The copy's source is the handle's own descriptor vector, which lives as
  // long as the handle.
  cudaError_t e = cudaMemcpyAsync(c->buf, c->desc.data(), c->desc.size() * sizeof(HeadDesc), cudaMemcpyHostToDevice,
                                  stream);
  if (e == cudaSuccess) e = rq::launch_norm_reset(c->buf, reinterpret_cast<const HeadDesc*>(c->buf), c->g, stream);
  if (e != cudaSuccess) {
    note_cuda_error(e);
    delete c;
    return RQ_ERR_CUDA;
  }
  *out = c;
  return RQ_OK;
}

void rq_cache_destroy(rq_cache* cache) { delete cache; }

rq_status rq_cache_length(const rq_cache* c, int layer, int* tokens) {
  if (!c || !tokens || layer < 0 || layer >= c->g.L) return RQ_ERR_INVALID_ARG;
  *tokens = c->length[layer];
  return RQ_OK;
}

rq_status rq_cache_stream_layout(const rq_cache* c, int layer, int b, int kv_head, size_t* tile_offset,
                                 int* record_bytes, int* n_tiles, size_t* window_offset) {
  if (!c || layer < 0 || layer >= c->g.L || b < 0 || b >= c->g.B || kv_head < 0 || kv_head >= c->g.Hkv)
    return RQ_ERR_INVALID_ARG;
  const HeadDesc& d = c->desc[layer * c->g.Hkv + kv_head];
  if (tile_offset) *tile_offset = (size_t)(d.tile_base + (int64_t)b * d.tile_stride);
  if (record_bytes) *record_bytes = d.rec_bytes;
  if (n_tiles) *n_tiles = rq::quantized_tokens(c->length[layer], c->g.S, c->g.R) / rq::kTile;
  if (window_offset) *window_offset = (size_t)(d.win_base + (int64_t)b * c->g.win_bytes);
  return RQ_OK;
}

rq_status rq_quantize_kv(rq_cache* c, const void* k, const void* v, int n_tokens, cudaStream_t stream) {
  if (!c || n_tokens < 0 || (n_tokens > 0 && (!k || !v))) return RQ_ERR_INVALID_ARG;
  if (n_tokens > 0 && (!aligned16(k) || !aligned16(v))) return RQ_ERR_INVALID_ARG;
  if (n_tokens > c->max_tokens) return RQ_ERR_CAPACITY;
  rq::QuantizeArgs a;
  a.g = c->g;
  a.buf = c->buf;
  a.desc = reinterpret_cast<const HeadDesc*>(c->buf);
  a.k = static_cast<const uint16_t*>(k);
  a.v = static_cast<const uint16_t*>(v);
  a.T = n_tokens;
  a.Tq = rq::quantized_tokens(n_tokens, c->g.S, c->g.R);
  a.k_norm = c->k_norm;
  if (n_tokens > 0) {
    const rq_status st = cuda_status(rq::launch_quantize(a, stream));
    if (st != RQ_OK) return st;
  }
  for (int l = 0; l < c->g.L; ++l) {
    c->length[l] = n_tokens;
    c->packed_ahead[l] = -1;
  }
  return RQ_OK;
}

rq_status rq_append_token(rq_cache* c, int layer, const void* k_new, const void* v_new, cudaStream_t stream) {
  if (!c || !k_new || !v_new || !aligned16(k_new) || !aligned16(v_new)) return RQ_ERR_INVALID_ARG;
  int l0, nl;
  if (!layer_range(c, layer, l0, nl)) return RQ_ERR_INVALID_ARG;
  const int T_old = c->length[l0];
  if (T_old + 1 > c->max_tokens) return RQ_ERR_CAPACITY;
  rq::AppendArgs a;
  a.g = c->g;
  a.buf = c->buf;
  a.desc = reinterpret_cast<const HeadDesc*>(c->buf);
  a.k_new = static_cast<const uint16_t*>(k_new);
  a.v_new = static_cast<const uint16_t*>(v_new);
  a.layer0 = l0;
  a.n_layers = nl;
  a.T_old = T_old;
  const int S = c->g.S, R = c->g.R;
  const int Tq_old = rq::quantized_tokens(T_old, S, R);
  a.flush = (T_old >= S && (T_old - S - Tq_old) + 1 == R + rq::kTile) ? 1 : 0;
  a.flush_pos = S + Tq_old;
  a.flush_tile = Tq_old / rq::kTile;
  const rq_status st = cuda_status(rq::launch_append(a, stream));
  if (st != RQ_OK) return st;
  for (int l = l0; l < l0 + nl; ++l) c->length[l] = T_old + 1;
  return RQ_OK;
}

rq_status rq_decode_workspace_bytes(const rq_cache* c, int n_splits, size_t* bytes) {
  if (!c || !bytes || n_splits < 0) return RQ_ERR_INVALID_ARG;
  const int streams_layer = c->g.B * c->g.Hkv;
  const int max_tiles = c->g.max_tiles;
  int s = n_splits;
  const int rec = max_record(c, 0, c->g.L);
  const int nw = (c->g.S + c->g.R + 2 * rq::kTile - 1) / rq::kTile;  // most window items any length can need
  int cl = 0;
  const int a1 = auto_splits(c, streams_layer, max_tiles, rec, 1, &cl);
  const int a2 = auto_splits(c, streams_layer * c->g.L, max_tiles, rec, 1, &cl);
  if (s < a1) s = a1;
  if (s < a2) s = a2;
  if (s > rq::kMaxItems - nw) s = rq::kMaxItems - nw;
  const int64_t all = (int64_t)streams_layer * c->g.L;
  *bytes = rq::ws_total_bytes(all, all, s + nw + 1, c->g.G, c->g.D);  // + a pack-ahead item
  return RQ_OK;
}

rq_status rq_decode_workspace_init(void* workspace, size_t ws_bytes, cudaStream_t stream) {
  if (!workspace || !aligned16(workspace) || ws_bytes < rq::ws_counter_offset()) return RQ_ERR_INVALID_ARG;
  return cuda_status(cudaMemsetAsync(workspace, 0, ws_bytes, stream));
}

rq_status rq_selftest_device_timeout(void* workspace, size_t ws_bytes, unsigned long long limit_ns,
                                     cudaStream_t stream) {
  if (!workspace || !aligned16(workspace) || ws_bytes < rq::ws_counter_offset() || limit_ns > 1000000000ull)
    return RQ_ERR_INVALID_ARG;
  return cuda_status(rq::launch_wait_timeout_selftest(static_cast<int*>(workspace), limit_ns, stream));
}

rq_status rq_decode_read_status(const void* workspace, int* device_status) {
  if (!workspace || !device_status) return RQ_ERR_INVALID_ARG;
  return cuda_status(cudaMemcpy(device_status, workspace, sizeof(int), cudaMemcpyDeviceToHost));
}

rq_status rq_decode_attention(rq_cache* c, int layer, const void* q, float* out, float softmax_scale, int n_splits,
                              void* workspace, size_t ws_bytes, cudaStream_t stream) {
  if (!c || !q || !out || !workspace || n_splits < 0) return RQ_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(out) || !aligned16(workspace)) return RQ_ERR_INVALID_ARG;
  int l0, nl;
  if (!layer_range(c, layer, l0, nl)) return RQ_ERR_INVALID_ARG;
  rq::DecodeArgs a;
  int smem = 0;
  rq_status st = fill_decode(c, l0, nl, c->length[l0], q, out, softmax_scale, n_splits, workspace, ws_bytes, a, smem);
  if (st != RQ_OK) return st;
  return cuda_status(rq::launch_decode(a, smem, stream));
}

rq_status rq_decode_step(rq_cache* c, int layer, const void* q, const void* k_new, const void* v_new, float* out,
                         float softmax_scale, int n_splits, void* workspace, size_t ws_bytes, cudaStream_t stream) {
  if (!c || !q || !k_new || !v_new || !out || !workspace || n_splits < 0) return RQ_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k_new) || !aligned16(v_new) || !aligned16(out) || !aligned16(workspace))
    return RQ_ERR_INVALID_ARG;
  int l0, nl;
  if (!layer_range(c, layer, l0, nl)) return RQ_ERR_INVALID_ARG;
  const int T_old = c->length[l0];
  if (T_old + 1 > c->max_tokens) return RQ_ERR_CAPACITY;
  const int S = c->g.S, R = c->g.R;
  bool packed = true;  // the previous fused step packed the tile this append completes
  for (int l = l0; l < l0 + nl; ++l) packed = packed && c->packed_ahead[l] == T_old;
  if (rq::quantized_tokens(T_old + 1, S, R) != rq::quantized_tokens(T_old, S, R) && !packed) {
    // the append completes a tile that is not packed yet: quantize it first,
    // then decode (two launches)
    rq_status st = rq_append_token(c, layer, k_new, v_new, stream);
    if (st != RQ_OK) return st;
    return rq_decode_attention(c, layer, q, out, softmax_scale, n_splits, workspace, ws_bytes, stream);
  }
  // One launch: append (the window item writes the new token) + decode, and,
  // when the next append will complete a tile, that tile is packed ahead by
  // one more work item.  Its 32 tokens are the oldest of the ring, all
  // present now; with n_recent >= 2 the token appended here is not among them.
  const int T = T_old + 1;
  const int Tq = rq::quantized_tokens(T, S, R);
  int n_pack = (R >= 2 && T + 1 <= c->max_tokens && rq::quantized_tokens(T + 1, S, R) != Tq) ? 1 : 0;
  rq::DecodeArgs a;
  int smem = 0;
  rq_status st = fill_decode(c, l0, nl, T, q, out, softmax_scale, n_splits, workspace, ws_bytes, a, smem, n_pack);
  if (n_pack && (st == RQ_ERR_WORKSPACE || st == RQ_ERR_UNSUPPORTED)) {
    // no room for the extra item (a workspace sized without it, or an
    // explicit split count at the item limit): the next step flushes itself
    n_pack = 0;
    st = fill_decode(c, l0, nl, T, q, out, softmax_scale, n_splits, workspace, ws_bytes, a, smem, 0);
  }
  if (st != RQ_OK) return st;
  a.k_new = static_cast<const uint16_t*>(k_new);
  a.v_new = static_cast<const uint16_t*>(v_new);
  a.pack_pos = S + Tq;
  a.pack_tile = Tq / rq::kTile;
  if (packed && Tq != rq::quantized_tokens(T_old, S, R)) {
    // This launch reads the tile the previous decode launch packed ahead.  A
    // decode launch may start before its predecessor ends (programmatic
    // dependent launch) and fetches its first tile records before waiting on
    // it, so it must not follow the packing launch directly: a 4-byte memset
    // of the workspace's padding (bytes 4..7, unused) in between makes it a
    // plain stream dependency -- the packing launch completes first.  This
    // holds in stream capture too (a memset node, not a kernel edge).
    st = cuda_status(cudaMemsetAsync(static_cast<uint8_t*>(workspace) + 4, 0, 4, stream));
    if (st != RQ_OK) return st;
  }
  st = cuda_status(rq::launch_decode(a, smem, stream));
  if (st != RQ_OK) return st;
  for (int l = l0; l < l0 + nl; ++l) {
    c->length[l] = T;
    c->packed_ahead[l] = n_pack ? T : -1;
  }
  return RQ_OK;
}

}  // extern "C"

// Distortion of the library's quantizer on calibration samples (see include/rq.h).
extern "C" rq_status rq_measure_distortion(const void* x, int n_heads, int n_tokens, int head_dim, int role,
                                           const int* bits, int n_bits, double* mse, cudaStream_t stream) {
  if (!x || !bits || !mse || n_heads < 1 || n_tokens < 1 || n_bits < 1 || (role != 0 && role != 1))
    return RQ_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(x) & 1u) || (reinterpret_cast<uintptr_t>(mse) & 7u)) return RQ_ERR_INVALID_ARG;
  if (head_dim != 64 && head_dim != 128) return RQ_ERR_UNSUPPORTED;
  if (role == 1 && n_tokens % rq::kTile != 0) return RQ_ERR_INVALID_ARG;
  if (n_heads > 65535) return RQ_ERR_UNSUPPORTED;
  for (int i = 0; i < n_bits; ++i)
    if (!valid_bits(bits[i])) return RQ_ERR_UNSUPPORTED;
  return cuda_status(rq::launch_measure_distortion(static_cast<const uint16_t*>(x), n_heads, n_tokens, head_dim,
                                                   role, bits, n_bits, mse, stream));
}

// Decode without a caller-supplied workspace (see include/rq.h).  Uses the
// library's own device scratch array; allocates nothing.
extern "C" rq_status rq_decode_attention_noalloc(rq_cache* c, int layer, const void* q, float* out,
                                                  float softmax_scale, int n_splits, cudaStream_t stream) {
  if (!c || !q || !out || n_splits < 0 || !aligned16(q) || !aligned16(out)) return RQ_ERR_INVALID_ARG;
  int l0, nl;
  if (!layer_range(c, layer, l0, nl)) return RQ_ERR_INVALID_ARG;
  void* scratch = nullptr;
  if (cuda_status(rq::noalloc_scratch(&scratch)) != RQ_OK) return RQ_ERR_CUDA;
  rq::DecodeArgs a;
  int smem = 0;
  const int64_t all_streams = (int64_t)c->g.L * c->g.B * c->g.Hkv;
  rq_status st = fill_decode(c, l0, nl, c->length[l0], q, out, softmax_scale, n_splits, scratch,
                             rq::kNoAllocScratchBytes, a, smem);
  if (st == RQ_ERR_WORKSPACE) return RQ_ERR_WORKSPACE;  // more split partials than the fixed array holds
  if (st != RQ_OK) return st;
  // status word and completion counters must start at zero; the array keeps
  // whatever the previous call (on any stream) left in it
  if (cuda_status(cudaMemsetAsync(scratch, 0, rq::ws_partial_offset(all_streams), stream)) != RQ_OK) return RQ_ERR_CUDA;
  return cuda_status(rq::launch_decode(a, smem, stream));
}

// Status word of the scratch array behind rq_decode_attention_noalloc on the
// current device (see include/rq.h).
extern "C" rq_status rq_decode_noalloc_read_status(int* device_status) {
  if (!device_status) return RQ_ERR_INVALID_ARG;
  void* scratch = nullptr;
  if (cuda_status(rq::noalloc_scratch(&scratch)) != RQ_OK) return RQ_ERR_CUDA;
  return cuda_status(cudaMemcpy(device_status, scratch, sizeof(int), cudaMemcpyDeviceToHost));
}

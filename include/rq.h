/*
 * rq.h -- mixed-precision, group-wise quantized KV cache and decode attention
 * for NVIDIA B200 (sm_100a).  C ABI of librq.so.
 *
 * The operations follow three of the pages this library is built from:
 *
 *   RateQuant: Optimal Mixed-Precision KV Cache Quantization via
 *   Rate-Distortion Theory (arXiv 2605.06675v2) -- per-head bit allocation
 *   under an average-bit budget: distortion model D(b) = alpha*beta^-b (§3.1),
 *   reverse waterfilling (§3.1, App. B.1), integer allocation (§3.3, App. U),
 *   separate K and V budgets (§3.4).
 *
 *   InnerQ: Hardware-Aware Tuning-Free Quantization of KV Cache for Large
 *   Language Models (arXiv 2602.23200) -- groups along the inner dimension of
 *   the decode vector-matrix products (K: per token along head_dim; V: per
 *   channel along tokens), asymmetric per-group quantization, high-precision
 *   sink and recent windows, dequantization fused into decode attention
 *   (abstract; "Core claim"; Algorithm 1, decode-phase attention).
 *
 *   Spend Bits Where Queries Look (NOVA-KV, arXiv 2608.04074, review page)
 *   and Behavioral Capacity Certificates (arXiv 2609.37887, abstract) -- keys
 *   need more precision than values, hence separate K and V bit widths.
 *
 * Conventions
 *   - Every pointer named dev_* / k / v / q / out / workspace is DEVICE memory
 *     owned by the caller.  The library never allocates or frees device memory.
 *   - Device calls are asynchronous on the given stream; arguments are checked
 *     on the host first and nothing is launched when a check fails.  After a
 *     launch, a CUDA launch error is reported as RQ_ERR_CUDA.
 *   - bf16 tensors are passed as raw 16-bit patterns (const void*), row-major
 *     and contiguous; out is float32.
 *   - k, v, q, k_new, v_new, out and workspace start on a 16-byte boundary
 *     (the kernels move them in 16-byte vectors and bulk copies); a pointer
 *     that does not is rejected with RQ_ERR_INVALID_ARG before any launch.
 *   - Lengths are tracked on the host in the rq_cache handle, so no call reads
 *     device memory back (except the rq_*_read_status calls, which say so).
 *   - Device memory handed to the library is used on the stream given with
 *     the call; a buffer must be valid on that stream (a stream-ordered
 *     allocator such as PyTorch's hands out memory for its current stream).
 *   - A handle is not thread-safe; one handle per thread of control.
 *
 * Packed tile format (one record per 32-token tile of one (layer, batch,
 * kv-head) stream; all offsets in bytes; the format is this library's own):
 *   record = [K codes | K meta | V codes | V meta]
 *   codes  : 32 lanes x W words, W = ceil(D / cpw), cpw = 16, 10, 8, 4 codes
 *            per 32-bit word for b = 2, 3, 4, 8.  Lane L = 4*gid + tig owns
 *            D/4 registers of four bytes e = 0..3: the 8-bit A-operand
 *            fragments of the m16n8k32 integer tensor-core MMA.  Register
 *            (rho, kh), rho in 0..D/8-1, kh in 0..1, byte e holds the code of
 *              K: token gid + 8i, channel 32g + 16kh + 4tig + e, rho = i*D/32 + g
 *              V: channel 16mb + 8rh + gid, token 4kh + tig + 8e,  rho = 2mb + rh
 *            Row group rho has class j = rho mod C (C = 4, 2, 2, 1 for
 *            b = 2, 3, 4, 8) and source sigma = 2*(rho / C) + kh: the code
 *            sits at bits 8e + b*j .. 8e + b*j + b - 1 of word sigma, so the
 *            word masked to those bits of every byte reads code * 2^(b*j).
 *            b = 3, sigma >= W: source W + q is the top bit pair (bits 6, 7 of
 *            each byte) of words 3q, 3q+1, 3q+2; code bit k of class j, byte e
 *            is bit 8e + 6 + (f%2) of word 3q + f/2, f = 3j + k; unused top
 *            bits are zero.
 *            Word w of lane L lives at ((w/4)*32 + L)*16 + (w%4)*4 for
 *            w < 4*floor(W/4), else floor(W/4)*512 + ((w - 4 floor(W/4))*32 + L)*4.
 *   meta   : u32 = fp16 scale | bf16 zero << 16.  K: D/32 groups x 32 entries,
 *            entry i = token 16((i>>1)&1) + 8(i&1) + (i>>2).  V: D entries,
 *            entry i = channel 16*mb + 8*rr + gid, gid = i/(D/8),
 *            mb = (i%(D/8))/2, rr = i%2.
 *   Quantization rule per group (IEEE fp32, round to nearest even):
 *     max, min = the group's extremes, each + 0 (a -0.0 extreme becomes +0.0),
 *       replaced by M, -M + 0 for a centred group of a hybrid cache (config),
 *     s = fp16(min((max - min) / (2^b - 1), 65504)), z = min (bf16),
 *     c = clamp(rint((x - z) * (s > 0 ? 1/s : 0)), 0, 2^b - 1).
 *   Windows per stream: sink K [S][D], sink V [S][D], recent ring K [R+32][D],
 *   ring V [R+32][D] (bf16), then the K normalization factors n [D] (fp32,
 *   powers of two; all 1 unless k_norm); token position P >= S sits in ring slot
 *   (P - S) mod (R + 32).  With T tokens, Tq = 32*floor((T - S - R)/32) tokens
 *   (0 when T < S + R) are quantized; the rest stay bf16.
 */
#ifndef RQ_H_
#define RQ_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* cudaStream_t;

typedef enum {
  RQ_OK = 0,
  RQ_ERR_INVALID_ARG = 1,       /* null pointer, negative size, bad layer, ... */
  RQ_ERR_UNSUPPORTED = 2,       /* head_dim not 64/128, group != 32, bits not in {2,3,4,8}, G not in {1,2,4,8} */
  RQ_ERR_INFEASIBLE_BUDGET = 3, /* avg_bits outside [min S, max S] */
  RQ_ERR_CAPACITY = 4,          /* tokens would exceed max_tokens, or buffer too small */
  RQ_ERR_WORKSPACE = 5,         /* workspace too small */
  RQ_ERR_CUDA = 6,              /* a CUDA runtime call failed */
  RQ_ERR_DEVICE_TIMEOUT = 7     /* a kernel gave up waiting (see rq_decode_read_status) */
} rq_status;

/* Static, human-readable name of a status code.  Never NULL. */
const char* rq_status_string(rq_status s);

/* ---------------------------------------------------------------- allocation
 * rq_allocate_bits -- RateQuant per-head bit allocation (host only, pure).
 *   Continuous reverse waterfilling (§3.1, App. B.1): minimise
 *   sum_h w_h alpha_h beta_h^-b_h subject to sum_h b_h = n * avg_bits and
 *   min(S) <= b_h <= max(S); stationary point
 *   b_h = clip(log_beta_h(w_h alpha_h ln(beta_h) / lambda)).
 *   Integer allocation (§3.3, App. B.3, App. U): b_int[h] in S minimising the
 *   same objective with sum_h b_int[h] <= floor(n * avg_bits); greedy
 *   max-heap when S is contiguous, exact dynamic programme otherwise.  Among
 *   allocations of equal distortion (relative 1e-12) the lexicographically
 *   largest vector is returned.
 * Arguments: n heads (n >= 1); w, alpha, beta host arrays [n] with w > 0,
 *   alpha > 0, beta > 1; allowed host array [n_allowed] of distinct bit
 *   widths in 1..16; b_cont [n] (nullable) receives the continuous solution,
 *   b_int [n] the integer one; log_lambda (nullable) receives ln(lambda).
 * Errors: RQ_ERR_INVALID_ARG, RQ_ERR_INFEASIBLE_BUDGET.  Outputs untouched on
 *   error.  Memory: all host, caller-owned. */
rq_status rq_allocate_bits(int n, const double* w, const double* alpha, const double* beta,
                           double avg_bits, const int* allowed, int n_allowed,
                           double* b_cont, int* b_int, double* log_lambda);

/* ------------------------------------------------------ distortion calibration
 * RateQuant fits its distortion model D(b) = alpha * beta^-b per quantizer
 * from a small calibration set (§1 "Method"; §3.4, quantizer-agnostic
 * extensions, K and V on separate curves) and gives a head whose fit is poor
 * (R^2 < 0.96) the decay rate min(beta_fitted, beta_bar) (W.10); it caps
 * sensitivities at 5 times their mean before allocating (W.14).  A joint K/V
 * budget is one rq_allocate_bits call over the 2N (head, K|V) units with their
 * own (w, alpha, beta).
 *
 * rq_measure_distortion -- mean squared error, per head and bit width, of
 *   quantizing and dequantizing calibration samples with this library's rule
 *   (the same groups and rounding as rq_quantize_kv; x_hat = c * s + z in
 *   fp64).  x: device bf16 [n_heads][n_tokens][head_dim]; role 0 = K groups
 *   (32 channels of a token), 1 = V groups (one channel over 32 tokens;
 *   n_tokens a multiple of 32).  bits: host [n_bits] in {2,3,4,8}.  mse:
 *   device double [n_heads][n_bits], overwritten.
 * Errors: RQ_ERR_INVALID_ARG, RQ_ERR_UNSUPPORTED (head_dim, bits), RQ_ERR_CUDA. */
rq_status rq_measure_distortion(const void* x, int n_heads, int n_tokens, int head_dim, int role,
                                const int* bits, int n_bits, double* mse, cudaStream_t stream);

/* rq_fit_distortion -- host, pure.  Per head, the least-squares line through
 *   (b, ln mse) gives ln alpha - b ln beta and its R^2 (points with mse <= 0
 *   are left out); heads with R^2 < r2_min get beta = min(beta, beta_bar),
 *   beta_bar = mean fitted beta of the heads at or above r2_min (of all heads
 *   when none is).  mse: host [n_heads][n_bits]; outputs host [n_heads].
 * Errors: RQ_ERR_INVALID_ARG (fewer than two usable points for a head). */
rq_status rq_fit_distortion(int n_heads, const int* bits, int n_bits, const double* mse, double r2_min,
                            double* alpha, double* beta, double* r2);

/* rq_cap_weights -- host, pure: w_out[i] = min(w[i], factor * mean(w))
 *   (factor 5 in W.14).  w_out may alias w.  Errors: RQ_ERR_INVALID_ARG. */
rq_status rq_cap_weights(int n, const double* w, double factor, double* w_out);

/* --------------------------------------------------------------------- cache */
typedef struct {
  int n_layers;      /* L >= 1 */
  int batch;         /* B >= 1 */
  int n_q_heads;     /* Hq, multiple of n_kv_heads, Hq/Hkv in {1,2,4,8} */
  int n_kv_heads;    /* Hkv >= 1 */
  int head_dim;      /* D in {64, 128} */
  int group;         /* must be 32 (tokens per V group = channels per K group) */
  int n_sink;        /* S >= 0 bf16 sink tokens */
  int n_recent;      /* R >= 0 minimum bf16 recent tokens */
  int max_tokens;    /* capacity per sequence */
  const int* k_bits; /* host [L*Hkv] in {2,3,4,8}, index l*Hkv + h (copied) */
  const int* v_bits; /* host [L*Hkv] in {2,3,4,8} (copied) */
  int k_norm;        /* 1: per-channel K normalization (InnerQ abstract): rq_quantize_kv sets
                        n_d = smallest power of two >= max_t |K[t, d]| per stream and channel
                        over the prefill tokens, tiles hold K / n, queries are multiplied by n
                        for the quantized tokens; 0: n = 1.  Windows keep K as is. */
  int hybrid;        /* 1: symmetric or asymmetric quantizer per group (InnerQ abstract,
                        technique (i); this library's rule): a group with
                        |max + min| <= (max - min) / 8 (fp32) is quantized on [-M, M],
                        M = max(|min|, |max|), i.e. min := -M, max := M in the rule below;
                        other groups on [min, max].  The record format and the decode are
                        the same either way (every group stores its own scale and zero).
                        0: every group asymmetric. */
} rq_cache_config;

typedef struct rq_cache rq_cache; /* opaque host handle */

/* Device buffer size needed for cfg (header + tile records + windows). */
rq_status rq_cache_bytes(const rq_cache_config* cfg, size_t* bytes);

/* Bind a caller-owned device buffer (>= rq_cache_bytes, 256-byte aligned) to
 * a new host handle with length 0.  Queues, on `stream`, the copy of the
 * buffer's descriptor header and the reset of every stream's K normalization
 * factors to 1 (asynchronous like every other device call; later calls on
 * the same stream see them).  *out receives the handle.  (The call the pages'
 * problem statement implies has no stream; the buffer is stream-ordered
 * memory, so the stream is given here.) */
rq_status rq_cache_init(const rq_cache_config* cfg, void* dev_buf, size_t bytes, rq_cache** out,
                        cudaStream_t stream);

/* Free the host handle (never the device buffer).  NULL is ignored. */
void rq_cache_destroy(rq_cache* cache);

/* Current token count of a layer (all batch elements share it). */
rq_status rq_cache_length(const rq_cache* cache, int layer, int* tokens);

/* Where a stream's data lives inside the device buffer (byte offsets from the
 * buffer start): tile records (tile i at tile_offset + i*record_bytes, valid
 * for i < *n_tiles) and the window block (sink K, sink V, ring K, ring V). */
rq_status rq_cache_stream_layout(const rq_cache* cache, int layer, int b, int kv_head,
                                 size_t* tile_offset, int* record_bytes, int* n_tiles,
                                 size_t* window_offset);

/* ------------------------------------------------------------- quantize / pack
 * rq_quantize_kv -- prefill: quantize and pack a T-token prefix of every
 *   layer, replacing the cache contents (InnerQ groups, fp16 scale / bf16
 *   zero, per-(layer, kv-head) bits).  k, v: device bf16
 *   [L][B][Hkv][T][D] contiguous.  Tokens [0,S) go to the sink, Tq tokens to
 *   tiles, the rest to the recent ring.  n_tokens in [0, max_tokens].
 * Errors: RQ_ERR_INVALID_ARG, RQ_ERR_CAPACITY, RQ_ERR_CUDA. */
rq_status rq_quantize_kv(rq_cache* cache, const void* k, const void* v, int n_tokens,
                         cudaStream_t stream);

/* rq_append_token -- add one token per (batch, kv-head) to one layer
 *   (layer >= 0; k_new, v_new bf16 [B][Hkv][D]) or to all layers at once
 *   (layer = -1; [L][B][Hkv][D]; every layer must have the same length).
 *   The token enters the recent ring (or the sink while T < S); when the
 *   recent window reaches R + 32 tokens its oldest 32 are quantized into the
 *   next tile by the same rule as rq_quantize_kv.
 * Errors: RQ_ERR_INVALID_ARG, RQ_ERR_CAPACITY (length would pass max_tokens),
 *   RQ_ERR_CUDA. */
rq_status rq_append_token(rq_cache* cache, int layer, const void* k_new, const void* v_new,
                          cudaStream_t stream);

/* ---------------------------------------------------------- decode attention
 * Workspace (caller-owned device memory) holds split partials, per-stream
 * completion counters and a status word.  Size it with
 * rq_decode_workspace_bytes (valid for every layer argument and every split
 * count <= n_splits) and zero it once with rq_decode_workspace_init; every
 * successful rq_decode_attention leaves the counters at zero again.  Calls
 * that share a workspace must not overlap on the GPU. */
rq_status rq_decode_workspace_bytes(const rq_cache* cache, int n_splits, size_t* bytes);
rq_status rq_decode_workspace_init(void* workspace, size_t ws_bytes, cudaStream_t stream);

/* rq_decode_attention -- one decode step of grouped-query attention over the
 *   packed cache (InnerQ Algorithm 1, decode phase; the page's listing is cut
 *   off, so the standard softmax(q K^T * scale) V is computed).  Query head h
 *   reads kv head h / (Hq/Hkv).  Reads every cached token: bf16 sink, packed
 *   tiles (dequantized inside the dot products: per-group scale and zero
 *   factored out of the inner sums), bf16 recent window.  Split-K over tiles
 *   with a fused log-sum-exp combine.
 * q: device bf16 [B][Hq][D] (layer >= 0) or [L][B][Hq][D] (layer = -1).
 * out: device float32, same shape.  softmax_scale <= 0 selects 1/sqrt(D).
 * n_splits: tile splits per stream, 0 = automatic; capped to the tile count
 *   and raised to ceil(tiles / 128): an item holds at most 128 tiles, since
 *   each warp's probabilities are kept in 16-bit fixed point relative to its
 *   running maximum and their rounding grows over longer sequences.
 * Errors: RQ_ERR_INVALID_ARG, RQ_ERR_WORKSPACE, RQ_ERR_CUDA. */
rq_status rq_decode_attention(rq_cache* cache, int layer, const void* q, float* out,
                              float softmax_scale, int n_splits, void* workspace,
                              size_t ws_bytes, cudaStream_t stream);

/* rq_decode_step -- one serving step: rq_append_token(layer, k_new, v_new)
 *   followed by rq_decode_attention(layer, q, ...) over the cache that now
 *   includes the new token, with the same arguments, layouts, results and
 *   errors as those two calls (InnerQ Algorithm 1, decode phase: the current
 *   token's key and value join the high-precision recent window).  Both
 *   happen in one kernel launch: the window work item that owns the newest
 *   position reads the token from k_new / v_new and writes it into the
 *   cache.  When the NEXT append will complete a tile (its 32 tokens are the
 *   oldest of the recent window, all present already), one more work item of
 *   this launch quantizes and packs that tile into its slot, which nothing
 *   reads until then; the next rq_decode_step on the same layers then only
 *   advances the length past it.  A step whose append completes a tile that
 *   was not packed ahead -- the first step after rq_quantize_kv or
 *   rq_append_token, or any step when n_recent < 2 -- quantizes the tile
 *   first and decodes after (two launches).  Results are those of the two
 *   calls in every case.  Workspace: rq_decode_workspace_bytes includes the
 *   extra item; a workspace (or an explicit n_splits at the item limit) with
 *   no room for it makes the step skip the pack-ahead, and the next step
 *   flushes with two launches.  On an error nothing is launched and the length is
 *   unchanged; otherwise the length grows by one.  The pages have no
 *   separate counterpart: it is the two operations above, fused. */
rq_status rq_decode_step(rq_cache* cache, int layer, const void* q, const void* k_new, const void* v_new,
                         float* out, float softmax_scale, int n_splits, void* workspace, size_t ws_bytes,
                         cudaStream_t stream);

/* Blocking read of the workspace status word: 0 when every kernel that used
 * this workspace completed normally, otherwise RQ_ERR_DEVICE_TIMEOUT in the
 * low byte (a pipeline wait gave up after ~1 s and the kernel returned
 * without writing its outputs). */
rq_status rq_decode_read_status(const void* workspace, int* device_status);

/* rq_selftest_device_timeout -- exercises the device timeout path without a
 *   fault: one thread waits on an mbarrier that nothing completes, using the
 *   bounded wait of the decode pipeline with the given limit (limit_ns <= 1e9),
 *   gives up and records RQ_ERR_DEVICE_TIMEOUT in the workspace status word as
 *   a decode kernel would; rq_decode_read_status then reports it.  Clear the
 *   word again with rq_decode_workspace_init.  The pages have no counterpart.
 * Errors: RQ_ERR_INVALID_ARG (null or too small workspace, limit above 1 s),
 *   RQ_ERR_CUDA. */
rq_status rq_selftest_device_timeout(void* workspace, size_t ws_bytes, unsigned long long limit_ns,
                                     cudaStream_t stream);

/* rq_decode_attention_noalloc -- the same decode step as rq_decode_attention,
 *   for callers that cannot allocate device memory: code running where
 *   cudaMalloc is unavailable or forbidden (inside a custom allocator or
 *   memory pool that must not re-enter the CUDA allocator, a host runtime
 *   whose device memory is fully pre-reserved, or a plugin that may only use
 *   buffers handed to it).  The pages define no such call; it has no
 *   counterpart there.
 * Scratch: a fixed 32 MiB device array inside this library (status word,
 *   per-stream completion counters, split partials), held by every device
 *   that loads the library until the process exits.  The first call on a
 *   device looks the array's address up (cudaGetSymbolAddress) with that
 *   device current; make that first call before any stream capture.  Each
 *   call clears the status word and counters (cudaMemsetAsync on the given
 *   stream) before the kernel; no memory is allocated or freed.
 * All calls share the one array, which keeps the last call's contents: calls
 *   that overlap on the GPU (other streams, other threads, other handles)
 *   race and corrupt each other's results; serialise them.
 * Arguments as rq_decode_attention, minus the workspace.  The call returns
 *   before the kernel runs, so a pipeline wait that gives up on the device
 *   (the kernel then leaves out untouched) shows only in the array's status
 *   word: read it with rq_decode_noalloc_read_status.
 * n_splits = 0 takes the automatic plan.  No plan goes below ceil(tiles /
 *   128) splits (see rq_decode_attention), so a call is only as small as
 *   that: about (ceil(tiles / 128) + window items) * streams * (G*D + 2G) * 4
 *   bytes of partials, which a one-wave plan keeps far below the array and a
 *   call of very many streams (several waves) may exceed.
 * Errors: RQ_ERR_INVALID_ARG; RQ_ERR_WORKSPACE when the call's split
 *   partials exceed the array (nothing is launched) -- decode fewer layers
 *   per call; RQ_ERR_CUDA. */
rq_status rq_decode_attention_noalloc(rq_cache* cache, int layer, const void* q, float* out,
                                      float softmax_scale, int n_splits, cudaStream_t stream);

/* rq_decode_noalloc_read_status -- blocking read of the status word of the
 *   scratch array behind rq_decode_attention_noalloc on the current device
 *   (waits for the device's work queued before it): 0 when the last call on
 *   this device completed normally, RQ_ERR_DEVICE_TIMEOUT in the low byte
 *   when a pipeline wait of that call gave up.  Each call clears the word, so
 *   it reflects the LAST call made on the device (from any thread).
 * Errors: RQ_ERR_INVALID_ARG (null pointer), RQ_ERR_CUDA. */
rq_status rq_decode_noalloc_read_status(int* device_status);

/* Name of the last CUDA error a call of this thread reported as RQ_ERR_CUDA
 * ("no error" if none).  Static string, never NULL. */
const char* rq_last_cuda_error(void);

/* Library build description (static string). */
const char* rq_build_info(void);

#ifdef __cplusplus
}
#endif

#endif /* RQ_H_ */

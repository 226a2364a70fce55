/*
 * kvq -- decode attention over a low-bit quantized KV cache, for NVIDIA B200 (sm_100a).
 *
 * C ABI.  Every entry point takes plain pointers and sizes; device pointers
 * are CUDA global memory owned by the caller (the library never allocates or
 * frees them), host pointers are ordinary (preferably pinned) host memory.
 * All GPU work is enqueued asynchronously on the CUDA stream passed as
 * `stream` (a cudaStream_t cast to void*; NULL = legacy default stream).
 * Arguments are checked on the host before anything is launched; a rejected
 * call returns a non-zero kvq_status and enqueues nothing.  No C++ exception
 * crosses this boundary.  KVQ_ERR_CUDA reports a launch or copy error
 * reported by the CUDA runtime at enqueue time.
 *
 * Method sources (page title, section):
 *  [DQK] "Dual-QK: Sharp Queries and Flat Keys for Prunable 2-bit KV Caches"
 *        (paperlayer.ai summary of arXiv 2610.09827)
 *  [TQ]  "TurboQuant on Quantized Models: Solving Compound Quantization Error
 *        with Pre-RoPE Compression and KV Compaction" (tq-kv, Zenodo abstract)
 *  [SIQ] "Statistical Inference and Quality Measures of KV Cache Quantisations
 *        Inspired by TurboQuant" (gist.science explainer), scheme KQV
 *  [CQ]  "CASK-Q" (decentralizedcompute.company), Method
 */
#ifndef KVQ_H
#define KVQ_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define KVQ_API __attribute__((visibility("default")))
#else
#define KVQ_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  KVQ_OK = 0,
  KVQ_ERR_INVALID_ARG = 1, /* null pointer, negative size, misaligned pointer, bad flag   */
  KVQ_ERR_UNSUPPORTED = 2, /* a valid configuration this build does not implement          */
  KVQ_ERR_CAPACITY = 3,    /* offset + n_new > capacity, or max_len > capacity             */
  KVQ_ERR_WORKSPACE = 4,   /* workspace smaller than the matching *_workspace_bytes query */
  KVQ_ERR_CUDA = 5,        /* the CUDA runtime reported an error when enqueuing            */
  KVQ_ERR_TIMEOUT = 6      /* a bounded wait inside a kernel gave up (kvq_decode_status)   */
} kvq_status;

typedef enum { KVQ_F32 = 0, KVQ_BF16 = 1, KVQ_F16 = 2 } kvq_dtype;

/*
 * Packed cache descriptor.  Shapes: B = batch, H = kv_heads, d = head_dim,
 * N = capacity (tokens), g = 32 (group_size), P = 4 (prune_granule).
 * Supported: d = 128, g = 32, P = 4, k_bits, v_bits in {2, 4},
 * N a multiple of 128, every pointer 16-byte aligned.
 *
 * Byte layout (all little-endian; ownership: caller-allocated device memory
 * of the sizes kvq_cache_sizes reports).  Codes are stored in blocks of 128
 * tokens, T = N / 128 blocks per (sequence, head):
 *  k_codes  [B][H][T][d/P][128] words of P*k_bits bits (uint16 for INT4,
 *           uint8 for INT2): inside a block, one row per group of 4 channels
 *           (channel-major), so a decode step reads only the rows it keeps,
 *           and adjacent kept rows are adjacent in memory [DQK Sec. 3.3].
 *           Channel 4p+i of token n sits in bits [i*k_bits, (i+1)*k_bits) of
 *           word (n / 128, p, n % 128).
 *  k_scales [B][H][T][d/g][128] x {fp16 scale, fp16 zero} (4 bytes).
 *  k_ch0    [B][H][N] bf16, channel 0 of the rotated key (only when keep_ch0;
 *           NULL otherwise); code slot 0 of such keys is written as 0 and
 *           channel 0 is outside group 0's range [DQK Sec. 1, Sec. 3.3, App. C.3].
 *  v_codes  [B][H][T][d][16*v_bits] bytes: inside a block, one row per
 *           channel holding that channel's 128 codes in token order (token t
 *           at bits ((t mod (8/v_bits)) * v_bits) of byte t / (8/v_bits) of
 *           the row).  Each row is cut into 16-byte chunks (32 tokens for
 *           INT4, 64 for INT2); chunk i of channel c is stored at chunk
 *           position i XOR s(c), s(c) = (c >> 1) & 3 for INT4 and
 *           (c >> 2) & 1 for INT2, so that the rows of 8 consecutive
 *           channels begin in 8 different shared-memory bank groups when a
 *           block is staged on chip.
 *  v_scales [B][H][N][d/g] x {fp16 scale, fp16 zero}.
 * Dequantized element: x = scale * code + zero [DQK Sec. 3.3, App. B.2; CQ].
 */
typedef struct {
  int32_t batch, kv_heads, head_dim, capacity;
  int32_t k_bits, v_bits, group_size, prune_granule;
  int32_t rotate_k; /* 1: keys (and queries) pass through the orthonormal Walsh-Hadamard transform;
                       2: through the caller's dual transform pair t_query / t_key (below)       */
  int32_t keep_ch0; /* 1: rotated channel 0 of each key is kept in bf16, unquantized               */
  int32_t rotate_v; /* 1: values pass through the orthonormal Walsh-Hadamard transform before they
                       are quantized, and decode outputs are rotated back [DQK App. B.2]           */
  float v_clip;     /* value clipping ratio in (0, 1]: each value group's min and max are scaled
                       by it before scale and zero are formed, values beyond saturate; 1 = none  */
  void* k_codes;
  void* k_scales;
  void* k_ch0;
  void* v_codes;
  void* v_scales;
  /* bf16 token windows [DQK Sec. 3.3: the first 64 and the most recent 256
     tokens stay BF16; TQ: sink tokens preserved]; 0 and NULL = none.
     k_window, v_window: [B][H][sink_tokens + recent_tokens][d] bf16, sizes
     from kvq_window_bytes: the rotated key and the value (rotated when
     rotate_v) of token n, at slot n when n < sink_tokens, else at ring slot
     sink_tokens + (n - sink_tokens) % recent_tokens: an append writes its
     tokens n < sink_tokens and its last recent_tokens tokens (the end state of
     writing every token in order).
     A decode over seq_lens[b] = len takes tokens n < sink_tokens and
     n >= max(sink_tokens, len - recent_tokens) from the windows, scored over
     every channel (the channel mask applies to the coded tokens only), so the
     ring must hold the last recent_tokens appended: decode len equal to the
     tokens appended so far.  sink_tokens + recent_tokens <= min(capacity,
     2048) (larger: KVQ_ERR_UNSUPPORTED). */
  int32_t sink_tokens, recent_tokens;
  void* k_window;
  void* v_window;
  /* Dual transform pair [DQK Sec. 1, Sec. 3.1], used when rotate_k == 2 (NULL
     otherwise): per kv head an invertible d x d matrix T applied to queries
     and its inverse transpose applied to keys, so that (T q).(T^-T k) = q.k
     before quantization and pruning.  Both are caller-owned device fp32
     arrays [H][d][d], row-major, 16-byte aligned, read but never written; the
     library does not check that t_key is T^-T.  Each transformed channel i is
     sum_j A[i][j] x[j] over j = 0..d-1 in that order, fp64 products and sums
     each rounded once, rounded to fp32.  Keys, their bf16 window copies and
     channel 0 (keep_ch0) are taken after the transform; values are not
     affected. */
  const float* t_query;
  const float* t_key;
  /* Bucket-relative RoPE [DQK Sec. 3.4, App. C.4]; 0 and NULL = none (keys
     and queries are used as given).  With bucket_tokens = w > 0, keys and
     queries arrive before rotary embedding.  Token n belongs to bucket
     k = n / w with anchor k * w; its key is embedded at offset n mod w, then
     transformed (rotate_k) and quantized.  At decode and selection the query
     of sequence b sits at position L - 1 (L = seq_lens[b]) and is embedded at
     offset L - 1 - k * w for bucket k (possibly beyond w), then transformed;
     each bucket has its own channel mask and one softmax covers all buckets.
     Rotary embedding pairs channel i with i + d/2 at angle
     offset * rope_inv_freq[i] (fp64 angle, cos and sin; each product and sum
     rounded once), the row then rounded to fp32.
     Layout: bucket-major -- every array is laid out as the cache of batch
     B * (capacity / w) and capacity w, bucket k of sequence b being its
     sequence b * (capacity / w) + k (kvq_cache_sizes is unchanged).
     bf16 token windows combine with buckets: the windows stay per sequence
     and are placed by sequence positions, and a window token is scored with
     the query of the bucket it sits in.
     Requires w a multiple of 128 dividing capacity, B * capacity / w <= 65535,
     and sink_tokens, recent_tokens <= w (otherwise KVQ_ERR_UNSUPPORTED); an
     append must stay inside one bucket (otherwise KVQ_ERR_INVALID_ARG).
     rope_inv_freq: caller-owned device fp32 [d/2], 16-byte aligned. */
  int32_t bucket_tokens;
  const float* rope_inv_freq;
} kvq_cache;

/*
 * Sizes in bytes of the five cache arrays, in the order k_codes, k_scales,
 * k_ch0 (0 unless keep_ch0), v_codes, v_scales.  Pointer fields are ignored.
 */
KVQ_API kvq_status kvq_cache_sizes(const kvq_cache* cache, size_t bytes_out[5]);

/* Bytes of each of k_window and v_window (0 without windows or on bad arguments). */
KVQ_API size_t kvq_window_bytes(const kvq_cache* cache);

/*
 * Quantize and append n_new tokens per (sequence, kv head) at token positions
 * [offset, offset + n_new) of the cache; no other token's codes, scales or
 * zeros change, so earlier tokens are never re-quantized (incremental cache
 * [TQ]).  Value-code bytes that also hold tokens outside the range are read
 * and written back with those tokens' bits unchanged, so two appends to the
 * same sequence whose ranges touch the same 64-token window must not run
 * concurrently (on different streams without ordering).
 *  k_new, v_new: device [B][H][n_new][d] of `dtype`.
 * Keys: x = H_d k / sqrt(d) when rotate_k == 1 (fp64 butterflies in natural
 * Sylvester order, rounded to fp32) [DQK Sec. 1; SIQ KQV; TQ], x = t_key[h] k
 * when rotate_k == 2 (fp64 in-order sums, rounded to fp32); channel 0 to
 * bf16 when keep_ch0; then per token and per 32-channel group
 * scale = fp16((max - min) / L), zero = fp16(min), L = 2^bits - 1,
 * code = clamp(round_half_even((x - zero) / scale), 0, L) with IEEE fp32
 * subtract and divide [DQK Sec. 3.3].  Values: the same quantizer [DQK App.
 * B.2], after the same rotation when rotate_v, with min and max multiplied by
 * v_clip (fp32) before scale and zero are formed (keys are not clipped).
 * n_new == 0 is a no-op.
 */
KVQ_API kvq_status kvq_quantize_append(const kvq_cache* cache, const void* k_new, const void* v_new,
                                       kvq_dtype dtype, int32_t n_new, int32_t offset, void* stream);

/*
 * Dynamic query-channel pruning [DQK Sec. 3.2, App. C.2]: for each
 * (sequence b, kv head h) the energy of channel group p is
 * E[p] = sum over the G = q_heads/kv_heads query heads of head h and the 4
 * channels of group p of q_rot^2 (fp64, heads outer, channels inner);
 * the keep_groups largest energies are kept, equal energies keeping the
 * lower p.  mask_out[b*H + h] (device uint32) gets bit p set for a kept group.
 *  q: device [B][q_heads][d] of `dtype`, un-rotated (rotated here when
 *  rotate_k == 1, q_rot = t_query[h] q when rotate_k == 2).  Query head j
 *  belongs to kv head j / G.  keep_groups in [1, 32].
 */
KVQ_API kvq_status kvq_select_channels(const kvq_cache* cache, const void* q, kvq_dtype dtype, int32_t q_heads,
                                       int32_t keep_groups, uint32_t* mask_out, void* stream);

/*
 * The same selection for queries at known positions: without bucket-relative
 * RoPE identical to kvq_select_channels (seq_lens unused); with it, one mask
 * per bucket from the query embedded at that bucket's offset [DQK Sec. 3.4:
 * masks may differ across buckets], mask_out [B][capacity / w][H].
 *  seq_lens: device int32 [B], the query of sequence b at position
 *  seq_lens[b] - 1.  kvq_select_channels on a bucketed cache returns
 *  KVQ_ERR_INVALID_ARG (it has no positions).
 */
KVQ_API kvq_status kvq_select_channels_at(const kvq_cache* cache, const void* q, kvq_dtype dtype, int32_t q_heads,
                                          const int32_t* seq_lens, int32_t keep_groups, uint32_t* mask_out,
                                          void* stream);

/*
 * The status of the last split decode (kvq_decode_attention or
 * kvq_decode_partials) that used `workspace`: KVQ_OK, or KVQ_ERR_TIMEOUT when
 * one of its bounded waits gave up.  The split decode's roles hand tiles to
 * one another through shared-memory barriers, and every wait on one is
 * bounded (about a second); after a give-up the CTA lets its work in flight
 * land, writes NaN partials (so the affected outputs are NaN), sets a status
 * word in the workspace and returns, and the context stays usable.  Each
 * split decode clears the word before it starts.  This call copies the word
 * back on `stream` and synchronizes that stream.  q_heads and workspace_bytes
 * as given to the decode.
 */
KVQ_API kvq_status kvq_decode_status(const kvq_cache* cache, int32_t q_heads, const void* workspace,
                                     size_t workspace_bytes, void* stream);

/*
 * Test hook for the give-up path: the next split decode enqueued from the
 * calling host thread leaves tile `tile` of its first CTA unfilled (its ring
 * stage never completes), so the waits on that tile give up after about a
 * second and kvq_decode_status reports KVQ_ERR_TIMEOUT.  A negative tile
 * clears the hook.  Not for production use.
 */
KVQ_API void kvq_test_withhold_tile(int32_t tile);

/*
 * Bounds-checked debug build (libkvq_checked.so, compiled with
 * -DKVQ_BOUNDS_CHECK): the kernels compare the range of every cache-array,
 * partial and window access they check with the array's extent, skip an
 * access out of bounds and count it.  This call synchronizes the device and
 * returns the count since the last reset (clearing it when `reset` is not
 * 0); in the regular library it returns UINT32_MAX (no checks compiled in).
 */
KVQ_API uint32_t kvq_bounds_violations(int32_t reset);

/* Device workspace bytes kvq_decode_attention needs for these sizes (0 on bad arguments). */
KVQ_API size_t kvq_decode_workspace_bytes(const kvq_cache* cache, int32_t q_heads, int32_t max_len);

/*
 * Fused decode attention over the packed cache [DQK Sec. 3.2-3.4; TQ].
 * For each sequence b and query head j (kv head h = j / G):
 *  s_n = softmax_scale * sum over kept channels c of q_rot[c] * k_hat_n[c],
 *  o = sum_n softmax(s)_n * v_hat_n over n < seq_lens[b]
 *  (with rotate_v, v_hat_n is the rotated value and o is rotated back by the
 *  same orthonormal transform before it is written),
 * scored directly from the key codes (no dequantized key is written):
 * per group, scale * (q . codes) + zero * sum(q), plus q_rot[0] * k_ch0 when
 * channel 0 is kept.  Sequences are cut into 128-token tiles and the tiles
 * of all (sequence, kv head) pairs are spread evenly over the GPU's SMs, so a
 * sequence may be split between several of them; each piece keeps a running
 * max and sum, and a combine pass merges the pieces into one softmax over the
 * whole sequence [DQK Sec. 3.4].  Supported GQA group sizes
 * G = q_heads / kv_heads: 1, 2, 4, 8, 16 (others: KVQ_ERR_UNSUPPORTED).
 *  q:        device [B][q_heads][d] of `dtype`, un-rotated (with rotate_k == 2
 *            the workspace also holds the transformed fp32 query rows).
 *  seq_lens: device int32 [B]; entries are clamped to [0, max_len]; a
 *            sequence of length 0 gets a zero output.
 *  max_len:  host bound on seq_lens, 0 <= max_len <= capacity; sizes the grid.
 *  mask:     device uint32 [B][H] from kvq_select_channels, or NULL = every
 *            channel group ([B][capacity / w][H] from kvq_select_channels_at
 *            with bucket-relative RoPE).
 *  out:      device fp32 [B][q_heads][d].
 *  workspace: device scratch of at least kvq_decode_workspace_bytes bytes,
 *            owned by the caller; not read by later calls.
 */
KVQ_API kvq_status kvq_decode_attention(const kvq_cache* cache, const void* q, kvq_dtype dtype, int32_t q_heads,
                                        const int32_t* seq_lens, int32_t max_len, const uint32_t* mask,
                                        float softmax_scale, float* out, void* workspace, size_t workspace_bytes,
                                        void* stream);

/*
 * The two halves of kvq_decode_attention, for callers that time them apart
 * or schedule the combine separately.  kvq_decode_partials runs the split
 * decode kernel only and leaves, in `workspace`, one partial per piece of
 * sequence it scored: the piece's running max of the scores in base-2 units
 * (score * log2(e)), its sum of 2^(score - max), and the unnormalized sum of
 * 2^(score - max) * v_hat per channel, for every query head.  How pieces are
 * cut and laid out in the workspace is private to the library: only
 * kvq_decode_combine, called with the same cache, q_heads, seq_lens and
 * max_len and the same workspace, reads it back, and writes `out`
 * [B][q_heads][d].
 * Argument rules and statuses are those of kvq_decode_attention.
 */
KVQ_API kvq_status kvq_decode_partials(const kvq_cache* cache, const void* q, kvq_dtype dtype, int32_t q_heads,
                                       const int32_t* seq_lens, int32_t max_len, const uint32_t* mask,
                                       float softmax_scale, void* workspace, size_t workspace_bytes, void* stream);
KVQ_API kvq_status kvq_decode_combine(const kvq_cache* cache, int32_t q_heads, const int32_t* seq_lens,
                                      int32_t max_len, float* out, const void* workspace, size_t workspace_bytes,
                                      void* stream);

/*
 * kvq_decode_attention with the query-channel selection of
 * kvq_select_channels (kvq_select_channels_at with bucket-relative RoPE) done
 * inside the call, keeping `keep_groups` (1..32) channel groups per (sequence,
 * kv head) [DQK Sec. 3.2, App. C.2].  The selection reads the query rows the
 * decode prepares anyway: with bucket-relative RoPE each bucket's embedded and
 * transformed rows, with the caller's pair the transformed rows, so they are
 * computed once.  Masks and outputs are those of the two calls in sequence.
 * The masks stay in `workspace` (kvq_decode_workspace_bytes covers them).
 * keep_groups outside 1..32: KVQ_ERR_INVALID_ARG; the other rules are those of
 * kvq_decode_attention.  kvq_decode_partials_select is its split half (its
 * partials are combined by kvq_decode_combine).
 */
KVQ_API kvq_status kvq_decode_attention_select(const kvq_cache* cache, const void* q, kvq_dtype dtype,
                                               int32_t q_heads, const int32_t* seq_lens, int32_t max_len,
                                               int32_t keep_groups, float softmax_scale, float* out,
                                               void* workspace, size_t workspace_bytes, void* stream);
KVQ_API kvq_status kvq_decode_partials_select(const kvq_cache* cache, const void* q, kvq_dtype dtype,
                                              int32_t q_heads, const int32_t* seq_lens, int32_t max_len,
                                              int32_t keep_groups, float softmax_scale, void* workspace,
                                              size_t workspace_bytes, void* stream);

/*
 * kvq_decode_attention without a workspace argument, for callers that cannot
 * allocate device memory: an engine that owns every byte of device memory in
 * its own pool and has no allocator to lend across this C boundary, or a
 * decode loop that must never call cudaMalloc because it can synchronize the
 * device or fail under a fixed memory budget.  The pages have no counterpart
 * to this entry point; it is an interface convenience only.
 *
 * Same arguments, results and statuses as kvq_decode_attention, minus the
 * workspace.  The per-split partials live in a fixed 16 MiB device array
 * inside the library (every GPU that loads the library holds it until the
 * process exits); a call whose partials would not fit, i.e. whose
 * kvq_decode_workspace_bytes exceeds 16 MiB, returns KVQ_ERR_WORKSPACE and
 * enqueues nothing.  The call allocates nothing.  The first call on a device
 * looks up that array's device address (with the device current) and caches
 * it, so make that first call before any stream capture.  The cached address
 * belongs to the device's context of that first call: after cudaDeviceReset,
 * or any other teardown and re-creation of the context, it is stale, and this
 * entry point must not be called again in the process.  Every call shares
 * the array: calls that run concurrently on the GPU (different streams, or
 * different host threads, without ordering between them) race on it and give
 * undefined results.  Nothing in the array needs to start at zero: each call
 * writes every partial it reads back.
 */
KVQ_API kvq_status kvq_decode_attention_static(const kvq_cache* cache, const void* q, kvq_dtype dtype,
                                               int32_t q_heads, const int32_t* seq_lens, int32_t max_len,
                                               const uint32_t* mask, float softmax_scale, float* out,
                                               void* stream);

/* Device workspace bytes kvq_decode_step_host needs (0 on bad arguments). */
KVQ_API size_t kvq_decode_step_workspace_bytes(const kvq_cache* cache, kvq_dtype dtype, int32_t q_heads,
                                               int32_t max_len);

/*
 * One decode step from host buffers: copies q_host ([B][q_heads][d] of
 * `dtype`) into the device workspace, runs kvq_select_channels when
 * keep_groups < 32, then kvq_decode_attention, and copies the fp32 output to
 * out_host ([B][q_heads][d]).  Everything is enqueued on `stream`; out_host
 * is valid once the stream has been synchronized.  Host buffers should be
 * page-locked for the copies to run asynchronously.
 */
KVQ_API kvq_status kvq_decode_step_host(const kvq_cache* cache, const void* q_host, kvq_dtype dtype,
                                        int32_t q_heads, const int32_t* seq_lens, int32_t max_len,
                                        int32_t keep_groups, float softmax_scale, float* out_host,
                                        void* workspace, size_t workspace_bytes, void* stream);

/* Static description of a status code. */
KVQ_API const char* kvq_status_string(kvq_status status);

#ifdef __cplusplus
}
#endif

#endif /* KVQ_H */

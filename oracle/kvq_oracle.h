/*
 * CPU oracle for quantized-KV decode attention -- TEST INFRASTRUCTURE ONLY.
 *
 * Plain, slow, obviously-correct restatement of what the decode path computes,
 * written from the method's description and kept independent of the CUDA
 * library: it shares no header, helper, table or constant with it.  Only the
 * tests, the smoke check and the benchmark's CPU-baseline leg may call it.
 *
 * Sources (page title, section):
 *  - "Dual-QK: Sharp Queries and Flat Keys for Prunable 2-bit KV Caches"
 *    (paperlayer.ai summary of arXiv 2610.09827): Sec. 1 (Hadamard rotation,
 *    channel 0 in BF16, paired transforms that preserve q.k), Sec. 3.2
 *    (dynamic query-channel pruning with one shared mask), Sec. 3.3 (asymmetric
 *    per-token INT2 keys, channel-major key rows), Sec. 3.4 (one global softmax
 *    over segments), App. B.2 (per-token asymmetric values), App. C.2 (group-L2
 *    query energy summed over the GQA group), App. C.3 (channel 0 outside the
 *    range estimate).
 *  - "TurboQuant on Quantized Models ..." (tq-kv, Zenodo abstract): scoring
 *    without key decompression; incremental cache append.
 *  - "Statistical Inference and Quality Measures of KV Cache Quantisations
 *    Inspired by TurboQuant" (gist.science explainer), scheme KQV: WHT + plain
 *    n-bit scalar quantization of keys.
 *  - "CASK-Q" (decentralizedcompute.company), Method: scalar codes + FP16
 *    scales as the stored format.
 *  - Dual-QK App. B.2 and Sec. 3.3: values rotated (the Hadamard part of the
 *    rotation the pages take from OSCAR) and quantized with a 0.92 clipping
 *    ratio; the ratio scales the group's minimum and maximum before the scale
 *    and zero are formed (keys are not clipped).  The attention output then
 *    leaves the rotated basis through the same orthonormal transform.
 *  - Dual-QK Sec. 3.3 (the first 64 and the most recent 256 tokens remain
 *    BF16) and tq-kv's sink-token preservation: window tokens are kept as bf16
 *    copies of the rotated key and of the (rotated) value and scored in full
 *    (all channels), under the same softmax as the quantized tokens.
 *  - Dual-QK Sec. 1 and Sec. 3.1: a general dual transform pair, fixed per
 *    KV head.  Queries take an invertible d x d matrix T and keys its inverse
 *    transpose, so that (T q).(T^{-T} k) = q.k before quantization and
 *    pruning; both matrices are supplied by the caller (calibrating them is
 *    outside the decode path).  Each output is the fp64 sum over j = 0..d-1,
 *    in that order, of A[i][j] x[j] (product and sum each rounded once),
 *    rounded to fp32.
 *  - Dual-QK Sec. 3.4 and App. C.4: bucket-relative RoPE.  Token n belongs to
 *    bucket n / w (w = 2048 on the pages) with anchor w * (n / w); its key is
 *    stored rotary-embedded at its offset n mod w from the anchor, then taken
 *    through the key transform.  The query (at position len - 1, the last
 *    token appended) is embedded at its offset p - anchor for each bucket,
 *    which may exceed w, then taken through the query transform; each bucket
 *    selects its own channel mask from its own query, and one softmax covers
 *    every bucket.  Rotary embedding pairs channel i with i + d/2 and turns the
 *    pair by angle pos * inv_freq[i] (fp64 cos and sin), the caller supplying
 *    the model's inverse frequencies; the embedded row is rounded to fp32.
 *
 * Precision: FWHT in fp64 (natural Sylvester order), rotated values rounded
 * to fp32; quantization in fp32 with IEEE round-half-to-even; dequantization,
 * channel energies, scores and softmax in fp64.
 */
#ifndef KVQ_ORACLE_H
#define KVQ_ORACLE_H
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Packed cache as the oracle writes it (host memory, oracle-owned layout code). */
typedef struct {
  int32_t batch, kv_heads, head_dim, capacity;
  int32_t k_bits, v_bits; /* 2 or 4 */
  int32_t rotate_k; /* 0: none; 1: orthonormal Walsh-Hadamard on keys and queries; 2: the caller's pair */
  int32_t keep_ch0;
  int32_t rotate_v; /* 1: values pass through the orthonormal Walsh-Hadamard transform before quantization */
  float v_clip;     /* value clipping ratio in (0, 1]; 1 = no clipping                              */
  uint8_t* k_codes;   /* [B][Hkv][ceil(cap/128)][d/4][128] x (4*k_bits/8) bytes     */
  uint16_t* k_scales; /* [B][Hkv][ceil(cap/128)][d/32][128] x {fp16 scale, fp16 zero} */
  uint16_t* k_ch0;    /* [B][Hkv][cap] bf16, or NULL                        */
  uint8_t* v_codes;   /* [B][Hkv][ceil(cap/128)][d][128*v_bits/8]: per block of 128 tokens one
                         row per channel, 16-byte chunks swizzled by channel        */
  uint16_t* v_scales; /* [B][Hkv][cap][d/32] x {fp16 scale, fp16 zero}      */
  /* bf16 windows: token n < sink at slot n, token n >= sink at ring slot
     sink + (n - sink) % recent; at decode, tokens n < sink and
     n >= max(sink, len - recent) are taken from the window */
  int32_t sink, recent;
  uint16_t* k_win; /* [B][Hkv][sink + recent][d] bf16 rotated key, or NULL   */
  uint16_t* v_win; /* [B][Hkv][sink + recent][d] bf16 (rotated) value, or NULL */
  /* rotate_k == 2: per kv head, row-major d x d fp32 matrices, T for queries
     and T^{-T} for keys; NULL otherwise */
  const float* t_q; /* [Hkv][d][d] */
  const float* t_k; /* [Hkv][d][d] */
  /* bucket-relative RoPE: bucket width w (0 = keys and queries used as given,
     no rotary embedding) and the d/2 inverse frequencies */
  int32_t bucket_w;
  const float* rope_inv_freq; /* [d/2] */
} orc_cache;

typedef struct {
  int64_t k_elems, v_elems;     /* quantized elements written            */
  int64_t k_exempt, v_exempt;   /* elements within the near-tie window     */
  int64_t k_clamped, v_clamped; /* codes clamped into [0, L]               */
  int64_t groups_exempt;        /* groups whose fp16 scale/zero is near a tie */
} orc_stats;

/* in-place unnormalized Walsh-Hadamard butterflies, natural order, fp64 */
void orc_fwht(double* x, int32_t d);
/* out = fp32(FWHT(x) * (1/sqrt(d))) */
void orc_rotate(const float* x, int32_t d, float* out);

/* out[i] = fp32(sum_j A[i][j] * x[j]), fp64 products and sums in order j = 0..d-1 */
void orc_transform(const float* A, const float* x, int32_t d, float* out);

/* rotary embedding of one row at position pos: out[i] = x[i] cos - x[i+d/2] sin,
   out[i+d/2] = x[i+d/2] cos + x[i] sin, angle pos * inv_freq[i], fp64, rounded to fp32 */
void orc_rope(const float* x, int32_t d, const float* inv_freq, int64_t pos, float* out);

/* IEEE binary16 / bfloat16 round-to-nearest-even from fp32, and widening */
uint16_t orc_half_rn(float x);
double orc_half_value(uint16_t h);
uint16_t orc_bf16_rn(float x);
double orc_bf16_value(uint16_t h);

/*
 * Asymmetric quantization of one group of n values.  include[i] == 0 leaves
 * element i out of the range estimate and gives it code 0.  Writes fp16
 * scale/zero bits and codes; exempt[i] (may be NULL) flags near-tie elements;
 * returns 1 if the group's scale or zero is within the fp16 tie window.
 */
int32_t orc_quantize_group(const float* x, const uint8_t* include, int32_t n, int32_t bits, uint16_t* s16,
                           uint16_t* z16, uint8_t* codes, uint8_t* exempt, int64_t* clamped);
/* the same with a clipping ratio: min and max are multiplied by clip (fp32)
   before the scale and zero are formed; codes outside [0, L] clamp */
int32_t orc_quantize_group_clip(const float* x, const uint8_t* include, int32_t n, int32_t bits, float clip,
                                uint16_t* s16, uint16_t* z16, uint8_t* codes, uint8_t* exempt, int64_t* clamped);

/*
 * Quantize k_new/v_new ([B][Hkv][n_new][d] fp32 values) and write them at
 * tokens [offset, offset+n_new) of the cache.  k_row_exempt / v_row_exempt
 * ([B][Hkv][n_new], may be NULL) flag rows holding any exempt element.
 * Returns 0, or -1 on bad arguments.
 */
int32_t orc_quantize_append(const orc_cache* c, const float* k_new, const float* v_new, int32_t n_new,
                            int32_t offset, orc_stats* stats, uint8_t* k_row_exempt, uint8_t* v_row_exempt);

/* unpack the d codes of token n of (b, h): which = 0 for K, 1 for V */
void orc_unpack_codes(const orc_cache* c, int32_t b, int32_t h, int32_t n, int32_t which, uint8_t* codes);

/* dequantized K and V rows [n][d] of (b, h), tokens n0..n0+n-1, fp64 */
void orc_dequantize(const orc_cache* c, int32_t b, int32_t h, int32_t n0, int32_t n, double* khat, double* vhat);

/*
 * Channel selection: per (b, kv head) keep the `keep` channel groups of 4
 * with the largest query energy summed over the GQA group.  q is
 * [B][Hq][d] fp32 values (un-rotated; rotated here when rotate == 1, taken
 * through t_q[h] ([Hkv][d][d], the pair's query matrix) when rotate == 2).
 * mask[b*Hkv + h] bit p set = group p kept.  energy (may be NULL) receives
 * [B][Hkv][d/4] fp64 energies.
 */
void orc_select(const float* q, int32_t B, int32_t Hq, int32_t Hkv, int32_t d, int32_t rotate, const float* t_q,
                int32_t keep, uint32_t* mask, double* energy);

/*
 * Channel selection per bucket of a bucket-relative RoPE cache (bucket_w > 0):
 * mask[(b * nb + k) * Hkv + h], nb = ceil(capacity / bucket_w), from the query
 * embedded at offset (lens[b] - 1) - k * bucket_w and transformed like the
 * keys' partner; energy (may be NULL) [B][nb][Hkv][d/4].
 */
void orc_select_buckets(const orc_cache* c, const float* q, int32_t Hq, const int32_t* lens, int32_t keep,
                        uint32_t* mask, double* energy);

/*
 * Decode attention over the oracle cache for rows r = b*Hq + hq listed in
 * `rows` (all B*Hq rows when rows == NULL); with rotate_v the output is the
 * orthonormal Walsh-Hadamard transform (its own inverse) of the attention
 * over the rotated values.  Remaining arguments:
 * `rows` (all B*Hq rows when rows == NULL).  q as in orc_select; lens[b]
 * tokens of sequence b; mask NULL = all channels ([B][nb][Hkv], one per bucket,
 * with bucket-relative RoPE).  out[r][d] fp64 (row-major
 * in the order of `rows`).
 */
void orc_attention(const orc_cache* c, const float* q, int32_t Hq, const int32_t* lens, const uint32_t* mask,
                   double scale, const int32_t* rows, int32_t nrows, double* out);

/* (T q) . (T^{-T} k) in fp64 for a d x d row-major invertible T; returns NaN if T is singular */
double orc_dual_score(const double* T, int32_t d, const double* q, const double* k);

#ifdef __cplusplus
}
#endif
#endif

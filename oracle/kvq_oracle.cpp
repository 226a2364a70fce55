// CPU oracle for quantized-KV decode attention -- TEST INFRASTRUCTURE ONLY.
// See kvq_oracle.h for the sources each function follows.  Build with
// -ffp-contract=off and without fast-math: IEEE rounding of every fp32
// subtract and divide is part of what the oracle states.
#include "kvq_oracle.h"

#include <cfenv>
#include <cmath>
#include <algorithm>
#include <cstring>
#include <limits>
#include <vector>

namespace {

constexpr int kGroup = 32;   // quantization group: 32 channels (workload recipe)
constexpr int kGranule = 4;  // pruning granule: 4 channels (workload recipe)

// Round |x| to a binary format with `p` significand bits (implicit bit
// included), minimum normal exponent `emin` and maximum exponent `emax`,
// nearest-even.  Returns +-inf on overflow.
double round_format(double x, int p, int emin, int emax) {
  if (x == 0.0 || std::isnan(x) || std::isinf(x)) return x;
  double a = std::fabs(x);
  int e2;
  std::frexp(a, &e2);  // a = f * 2^e2, f in [0.5, 1)
  int E = e2 - 1;      // a in [2^E, 2^(E+1))
  int qexp = (E < emin ? emin : E) - (p - 1);
  double quantum = std::ldexp(1.0, qexp);
  double r = std::nearbyint(a / quantum) * quantum;  // default mode: nearest-even
  if (r >= std::ldexp(1.0, emax + 1)) r = std::numeric_limits<double>::infinity();
  return std::copysign(r, x);
}

// encode a value already representable in the format as its bit pattern
uint16_t encode_format(double r, int p, int emin, int bias, int ebits) {
  uint16_t sign = std::signbit(r) ? (uint16_t)(1u << 15) : 0;
  double a = std::fabs(r);
  const int mbits = p - 1;
  if (std::isinf(a)) return sign | (uint16_t)(((1u << ebits) - 1) << mbits);
  if (a == 0.0) return sign;
  if (a < std::ldexp(1.0, emin)) {  // subnormal: multiple of 2^(emin - mbits)
    return sign | (uint16_t)std::llround(a / std::ldexp(1.0, emin - mbits));
  }
  int e2;
  std::frexp(a, &e2);
  int E = e2 - 1;
  long m = std::llround(a / std::ldexp(1.0, E - mbits)) - (1L << mbits);
  return sign | (uint16_t)(((E + bias) << mbits) | m);
}

double decode_format(uint16_t h, int mbits, int emin, int bias, int ebits) {
  int sign = (h >> 15) & 1;
  int e = (h >> mbits) & ((1 << ebits) - 1);
  int m = h & ((1 << mbits) - 1);
  double v;
  if (e == 0)
    v = std::ldexp((double)m, emin - mbits);
  else if (e == (1 << ebits) - 1)
    v = m ? std::numeric_limits<double>::quiet_NaN() : std::numeric_limits<double>::infinity();
  else
    v = std::ldexp((double)((1 << mbits) | m), e - bias - mbits);
  return sign ? -v : v;
}

// |x| within rel of a midpoint between two neighbouring fp16 values
bool near_half_midpoint(float x, double rel) {
  double a = std::fabs((double)x);
  if (a == 0.0 || a > 65504.0) return false;
  int e2;
  std::frexp(a, &e2);
  int E = e2 - 1;
  double quantum = std::ldexp(1.0, (E < -14 ? -14 : E) - 10);
  double t = a / quantum;
  double frac = t - std::floor(t);
  return std::fabs(frac - 0.5) * quantum <= rel * a;
}

inline size_t bh_index(const orc_cache* c, int b, int h) { return (size_t)b * c->kv_heads + h; }

// --- layout: byte/element addresses of the packed cache --------------------
// Keys are stored in blocks of kBlock tokens.  Within a block, K codes are
// channel-major: one row of kBlock words per group of 4 channels; a token's 4
// codes share one 16-bit (INT4) or 8-bit (INT2) word, channel 4p+i in bits
// [i*bits, (i+1)*bits).  Key scale/zero pairs follow the same blocking with
// one row per 32-channel group.
constexpr int kBlock = 128;
inline size_t n_blocks(const orc_cache* c) { return (size_t)(c->capacity + kBlock - 1) / kBlock; }
inline size_t k_word_index(const orc_cache* c, int b, int h, int pg, int n) {
  const size_t blk = bh_index(c, b, h) * n_blocks(c) + n / kBlock;
  return (blk * (c->head_dim / kGranule) + pg) * kBlock + n % kBlock;
}
inline size_t k_scale_index(const orc_cache* c, int b, int h, int g, int n) {
  const size_t blk = bh_index(c, b, h) * n_blocks(c) + n / kBlock;
  return (blk * (c->head_dim / kGroup) + g) * kBlock + n % kBlock;
}
inline size_t ch0_index(const orc_cache* c, int b, int h, int n) {
  return bh_index(c, b, h) * (size_t)c->capacity + n;
}
// V codes: channel-major inside each block of kBlock tokens.  A block holds
// one row per channel; a row packs the block's kBlock codes of that channel in
// token order, little-endian (token t at bits ((t mod (8/bits)) * bits) of
// byte t / (8/bits)), and is split into 16-byte chunks.  Chunk i of channel
// ch is stored at chunk position i ^ chunk_swizzle(ch), so that the rows of 8
// consecutive channels touch 8 different 16-byte bank groups.
inline int v_row_bytes(const orc_cache* c) { return kBlock * c->v_bits / 8; }
inline int v_chunk_swizzle(const orc_cache* c, int ch) {
  return c->v_bits == 4 ? (ch >> 1) & 3 : (ch >> 2) & 1;
}
// byte holding the code of channel ch, token n of (b, h); *shift = its bit offset
inline size_t v_code_byte(const orc_cache* c, int b, int h, int ch, int n, int* shift) {
  const int per_byte = 8 / c->v_bits;
  const int tokens_per_chunk = 16 * per_byte;
  const int t = n % kBlock;
  const int chunk = (t / tokens_per_chunk) ^ v_chunk_swizzle(c, ch);
  const size_t blk = bh_index(c, b, h) * n_blocks(c) + n / kBlock;
  *shift = (t % per_byte) * c->v_bits;
  return (blk * c->head_dim + ch) * (size_t)v_row_bytes(c) + (size_t)chunk * 16 + (t % tokens_per_chunk) / per_byte;
}
inline size_t v_scale_index(const orc_cache* c, int b, int h, int n, int g) {
  return (bh_index(c, b, h) * (size_t)c->capacity + n) * (c->head_dim / kGroup) + g;
}

void store_k_word(const orc_cache* c, int b, int h, int pg, int n, uint32_t word) {
  size_t i = k_word_index(c, b, h, pg, n);
  if (c->k_bits == 4) {
    c->k_codes[2 * i] = (uint8_t)(word & 0xFF);
    c->k_codes[2 * i + 1] = (uint8_t)(word >> 8);
  } else {
    c->k_codes[i] = (uint8_t)word;
  }
}
uint32_t load_k_word(const orc_cache* c, int b, int h, int pg, int n) {
  size_t i = k_word_index(c, b, h, pg, n);
  if (c->k_bits == 4) return (uint32_t)c->k_codes[2 * i] | ((uint32_t)c->k_codes[2 * i + 1] << 8);
  return c->k_codes[i];
}

// bf16 window of a cache: sink + recent slots per (b, h)
inline long wsize(const orc_cache* c) { return (long)c->sink + c->recent; }
// slot written for token n by an append, or -1
inline long window_slot(const orc_cache* c, long n) {
  if (n < c->sink) return n;
  if (c->recent > 0) return c->sink + (n - c->sink) % c->recent;
  return -1;
}
// window row of token j when a decode of a length-len sequence reads it from
// the window (j < sink, or j among the last `recent` tokens), else NULL
inline const uint16_t* window_row(const orc_cache* c, const uint16_t* win, int b, int h, long j, long len) {
  const bool in = j < c->sink || (c->recent > 0 && j >= std::max((long)c->sink, len - c->recent));
  if (!in || !win) return nullptr;
  return win + (((size_t)b * c->kv_heads + h) * wsize(c) + window_slot(c, j)) * c->head_dim;
}

}  // namespace

extern "C" {
void orc_rope(const float* x, int32_t d, const float* inv_freq, int64_t pos, float* out);
void orc_transform(const float* A, const float* x, int32_t d, float* out);
void orc_rotate(const float* x, int32_t d, float* out);
}

namespace {

// A key (query = false) or query row as the cache scores it: rotary-embedded
// at `rel` when the cache uses bucket-relative RoPE, then taken through the
// key or query side of the cache's transform.
void prepare_row(const orc_cache* c, int h, const float* x, bool query, long rel, float* out) {
  const int d = c->head_dim;
  std::vector<float> e(x, x + d);
  if (c->bucket_w > 0) orc_rope(x, d, c->rope_inv_freq, rel, e.data());
  if (c->rotate_k == 2)
    orc_transform((query ? c->t_q : c->t_k) + (size_t)h * d * d, e.data(), d, out);
  else if (c->rotate_k)
    orc_rotate(e.data(), d, out);
  else
    for (int i = 0; i < d; ++i) out[i] = e[i];
}

inline int n_buckets(const orc_cache* c) { return c->bucket_w > 0 ? (c->capacity + c->bucket_w - 1) / c->bucket_w : 1; }

// keep the `keep` largest energies of the GQA group's rows qr [G][d]; equal
// energies rank the lower index first
uint32_t select_mask(const float* qr, int G, int d, int keep, double* energy) {
  const int npg = d / kGranule;
  std::vector<double> E(npg);
  for (int p = 0; p < npg; ++p) {
    double e = 0.0;
    for (int g = 0; g < G; ++g)
      for (int i = p * kGranule; i < (p + 1) * kGranule; ++i) {
        double v = (double)qr[(size_t)g * d + i];
        e += v * v;
      }
    E[p] = e;
    if (energy) energy[p] = e;
  }
  uint32_t m = 0;
  for (int p = 0; p < npg; ++p) {
    int rank = 0;
    for (int o = 0; o < npg; ++o)
      if (E[o] > E[p] || (E[o] == E[p] && o < p)) ++rank;
    if (rank < keep) m |= 1u << p;
  }
  return m;
}

}  // namespace

extern "C" {

void orc_rope(const float* x, int32_t d, const float* inv_freq, int64_t pos, float* out) {
  const int hd = d / 2;
  for (int i = 0; i < hd; ++i) {
    const double th = (double)pos * (double)inv_freq[i];
    const double cs = std::cos(th), sn = std::sin(th);
    const double a = x[i], b = x[i + hd];
    out[i] = (float)(a * cs - b * sn);
    out[i + hd] = (float)(b * cs + a * sn);
  }
}

void orc_fwht(double* x, int32_t d) {
  // Sylvester order: H[i][j] = (-1)^popcount(i & j); stage h pairs (i, i+h)
  for (int h = 1; h < d; h <<= 1)
    for (int i = 0; i < d; ++i)
      if ((i & h) == 0) {
        double a = x[i], b = x[i + h];
        x[i] = a + b;
        x[i + h] = a - b;
      }
}

void orc_transform(const float* A, const float* x, int32_t d, float* out) {
  for (int i = 0; i < d; ++i) {
    double acc = 0.0;
    for (int j = 0; j < d; ++j) acc += (double)A[(size_t)i * d + j] * (double)x[j];
    out[i] = (float)acc;
  }
}

void orc_rotate(const float* x, int32_t d, float* out) {
  std::vector<double> t(d);
  for (int i = 0; i < d; ++i) t[i] = (double)x[i];
  orc_fwht(t.data(), d);
  const double inv = 1.0 / std::sqrt((double)d);
  for (int i = 0; i < d; ++i) out[i] = (float)(t[i] * inv);
}

uint16_t orc_half_rn(float x) {
  double r = round_format((double)x, 11, -14, 15);
  return encode_format(r, 11, -14, 15, 5);
}
double orc_half_value(uint16_t h) { return decode_format(h, 10, -14, 15, 5); }
uint16_t orc_bf16_rn(float x) {
  double r = round_format((double)x, 8, -126, 127);
  return encode_format(r, 8, -126, 127, 8);
}
double orc_bf16_value(uint16_t h) { return decode_format(h, 7, -126, 127, 8); }

int32_t orc_quantize_group(const float* x, const uint8_t* include, int32_t n, int32_t bits, uint16_t* s16,
                           uint16_t* z16, uint8_t* codes, uint8_t* exempt, int64_t* clamped) {
  return orc_quantize_group_clip(x, include, n, bits, 1.0f, s16, z16, codes, exempt, clamped);
}

int32_t orc_quantize_group_clip(const float* x, const uint8_t* include, int32_t n, int32_t bits, float clip,
                                uint16_t* s16, uint16_t* z16, uint8_t* codes, uint8_t* exempt, int64_t* clamped) {
  const int L = (1 << bits) - 1;
  float mn = std::numeric_limits<float>::infinity(), mx = -std::numeric_limits<float>::infinity();
  for (int i = 0; i < n; ++i)
    if (!include || include[i]) {
      if (x[i] < mn) mn = x[i];
      if (x[i] > mx) mx = x[i];
    }
  // -0 and +0 compare equal; the extremes are taken as +0 so that the stored
  // scale and zero do not depend on which of the two came first.
  mn = mn + 0.0f;
  mx = mx + 0.0f;
  // clipping ratio: both ends of the range move toward zero by the same factor
  // (exact for clip = 1)
  mn = clip * mn;
  mx = clip * mx;
  // scale = (max - min) / L and zero = min, both computed in fp32 and stored
  // as fp16; values beyond the fp16 range saturate at +-65504.
  float range = mx - mn;
  float s32 = range / (float)L;
  if (s32 > 65504.0f) s32 = 65504.0f;
  float zsat = mn > 65504.0f ? 65504.0f : (mn < -65504.0f ? -65504.0f : mn);
  *s16 = orc_half_rn(s32);
  *z16 = orc_half_rn(zsat);
  const float sf = (float)orc_half_value(*s16);
  const float zf = (float)orc_half_value(*z16);
  int32_t group_exempt = (near_half_midpoint(s32, 1e-6) || near_half_midpoint(zsat, 1e-6)) ? 1 : 0;
  for (int i = 0; i < n; ++i) {
    if (exempt) exempt[i] = 0;
    if ((include && !include[i]) || sf == 0.0f) {
      codes[i] = 0;
      continue;
    }
    float v = (x[i] - zf) / sf;  // fp32 subtract, fp32 divide, each rounded once
    float r = std::nearbyint(v);
    int code = (int)r;
    if (code < 0 || code > L) {
      code = code < 0 ? 0 : L;
      if (clamped) ++*clamped;
    }
    codes[i] = (uint8_t)code;
    double fv = (double)v;
    if (exempt && std::fabs(fv - (std::floor(fv) + 0.5)) <= 1e-6 * std::fmax(std::fabs(fv), 1.0)) exempt[i] = 1;
  }
  return group_exempt;
}

int32_t orc_quantize_append(const orc_cache* c, const float* k_new, const float* v_new, int32_t n_new,
                            int32_t offset, orc_stats* stats, uint8_t* k_row_exempt, uint8_t* v_row_exempt) {
  const int d = c->head_dim;
  if (d % kGroup != 0 || n_new < 0 || offset < 0 || offset + n_new > c->capacity) return -1;
  if (c->rotate_k == 2 && !c->t_k) return -1;
  if (c->bucket_w < 0 || (c->bucket_w > 0 && !c->rope_inv_freq)) return -1;
  if ((c->k_bits != 2 && c->k_bits != 4) || (c->v_bits != 2 && c->v_bits != 4)) return -1;
  const int ngroups = d / kGroup, npg = d / kGranule;
  orc_stats total = {0, 0, 0, 0, 0, 0, 0};
  const int nbh = c->batch * c->kv_heads;
#pragma omp parallel for schedule(dynamic, 1)
  for (int bh = 0; bh < nbh; ++bh) {
    const int b = bh / c->kv_heads, h = bh % c->kv_heads;
    orc_stats st = {0, 0, 0, 0, 0, 0, 0};
    std::vector<float> xr(d);
    std::vector<uint8_t> incl(d), codes(d), ex(d);
    for (int t = 0; t < n_new; ++t) {
      const int n = offset + t;
      const size_t row = ((size_t)bh * n_new + t) * d;
      // ---- keys: rotate, optional channel 0 in bf16, quantize, pack ----
      prepare_row(c, h, k_new + row, false, c->bucket_w > 0 ? n % c->bucket_w : 0, xr.data());
      const long ws = window_slot(c, n);
      if (ws >= 0)
        for (int i = 0; i < d; ++i) c->k_win[(((size_t)b * c->kv_heads + h) * wsize(c) + ws) * d + i] = orc_bf16_rn(xr[i]);
      for (int i = 0; i < d; ++i) incl[i] = 1;
      if (c->keep_ch0) {
        c->k_ch0[ch0_index(c, b, h, n)] = orc_bf16_rn(xr[0]);
        incl[0] = 0;
      }
      int row_ex = 0;
      for (int g = 0; g < ngroups; ++g) {
        uint16_t s16, z16;
        int gex = orc_quantize_group(&xr[g * kGroup], &incl[g * kGroup], kGroup, c->k_bits, &s16, &z16,
                                     &codes[g * kGroup], &ex[g * kGroup], &st.k_clamped);
        size_t si = k_scale_index(c, b, h, g, n);
        c->k_scales[2 * si] = s16;
        c->k_scales[2 * si + 1] = z16;
        st.groups_exempt += gex;
        for (int i = 0; i < kGroup; ++i) {
          if (!incl[g * kGroup + i]) continue;
          st.k_elems++;
          if (gex || ex[g * kGroup + i]) {
            st.k_exempt++;
            row_ex = 1;
          }
        }
      }
      if (k_row_exempt) k_row_exempt[(size_t)bh * n_new + t] = (uint8_t)row_ex;
      for (int pg = 0; pg < npg; ++pg) {
        uint32_t word = 0;
        for (int i = 0; i < kGranule; ++i) word |= (uint32_t)codes[pg * kGranule + i] << (i * c->k_bits);
        store_k_word(c, b, h, pg, n, word);
      }
      // ---- values: optional rotation, quantize with the clipping ratio, pack
      // into the channel rows of the block ----
      if (c->rotate_v)
        orc_rotate(v_new + row, d, xr.data());
      else
        for (int i = 0; i < d; ++i) xr[i] = v_new[row + i];
      if (ws >= 0)
        for (int i = 0; i < d; ++i) c->v_win[(((size_t)b * c->kv_heads + h) * wsize(c) + ws) * d + i] = orc_bf16_rn(xr[i]);
      row_ex = 0;
      for (int g = 0; g < ngroups; ++g) {
        uint16_t s16, z16;
        int gex = orc_quantize_group_clip(&xr[g * kGroup], nullptr, kGroup, c->v_bits, c->v_clip, &s16, &z16,
                                          &codes[g * kGroup], &ex[g * kGroup], &st.v_clamped);
        size_t si = v_scale_index(c, b, h, n, g);
        c->v_scales[2 * si] = s16;
        c->v_scales[2 * si + 1] = z16;
        st.groups_exempt += gex;
        for (int i = 0; i < kGroup; ++i) {
          st.v_elems++;
          if (gex || ex[g * kGroup + i]) {
            st.v_exempt++;
            row_ex = 1;
          }
        }
      }
      if (v_row_exempt) v_row_exempt[(size_t)bh * n_new + t] = (uint8_t)row_ex;
      const uint32_t vmask = (1u << c->v_bits) - 1;
      for (int ch = 0; ch < d; ++ch) {
        int sh;
        const size_t i = v_code_byte(c, b, h, ch, n, &sh);
        // only this token's bits change; the byte's other tokens keep theirs
        c->v_codes[i] = (uint8_t)((c->v_codes[i] & ~(vmask << sh)) | ((uint32_t)codes[ch] << sh));
      }
    }
#pragma omp critical
    {
      total.k_elems += st.k_elems;
      total.v_elems += st.v_elems;
      total.k_exempt += st.k_exempt;
      total.v_exempt += st.v_exempt;
      total.k_clamped += st.k_clamped;
      total.v_clamped += st.v_clamped;
      total.groups_exempt += st.groups_exempt;
    }
  }
  if (stats) *stats = total;
  return 0;
}

void orc_unpack_codes(const orc_cache* c, int32_t b, int32_t h, int32_t n, int32_t which, uint8_t* codes) {
  const int d = c->head_dim;
  if (which == 0) {
    const uint32_t mask = (1u << c->k_bits) - 1;
    for (int pg = 0; pg < d / kGranule; ++pg) {
      uint32_t w = load_k_word(c, b, h, pg, n);
      for (int i = 0; i < kGranule; ++i) codes[pg * kGranule + i] = (uint8_t)((w >> (i * c->k_bits)) & mask);
    }
  } else {
    const uint32_t mask = (1u << c->v_bits) - 1;
    for (int ch = 0; ch < d; ++ch) {
      int sh;
      const size_t i = v_code_byte(c, b, h, ch, n, &sh);
      codes[ch] = (uint8_t)((c->v_codes[i] >> sh) & mask);
    }
  }
}

void orc_dequantize(const orc_cache* c, int32_t b, int32_t h, int32_t n0, int32_t n, double* khat, double* vhat) {
  const int d = c->head_dim;
  std::vector<uint8_t> codes(d);
  for (int t = 0; t < n; ++t) {
    const int tok = n0 + t;
    if (khat) {
      orc_unpack_codes(c, b, h, tok, 0, codes.data());
      for (int ch = 0; ch < d; ++ch) {
        if (c->keep_ch0 && ch == 0) {
          khat[(size_t)t * d] = orc_bf16_value(c->k_ch0[ch0_index(c, b, h, tok)]);
          continue;
        }
        size_t si = k_scale_index(c, b, h, ch / kGroup, tok);
        khat[(size_t)t * d + ch] =
            orc_half_value(c->k_scales[2 * si]) * codes[ch] + orc_half_value(c->k_scales[2 * si + 1]);
      }
    }
    if (vhat) {
      orc_unpack_codes(c, b, h, tok, 1, codes.data());
      for (int ch = 0; ch < d; ++ch) {
        size_t si = v_scale_index(c, b, h, tok, ch / kGroup);
        vhat[(size_t)t * d + ch] =
            orc_half_value(c->v_scales[2 * si]) * codes[ch] + orc_half_value(c->v_scales[2 * si + 1]);
      }
    }
  }
}

void orc_select(const float* q, int32_t B, int32_t Hq, int32_t Hkv, int32_t d, int32_t rotate, const float* t_q,
                int32_t keep, uint32_t* mask, double* energy) {
  const int G = Hq / Hkv, npg = d / kGranule;
  std::vector<float> qr((size_t)G * d);
  for (int b = 0; b < B; ++b)
    for (int hk = 0; hk < Hkv; ++hk) {
      for (int g = 0; g < G; ++g) {
        const float* qi = q + ((size_t)b * Hq + (size_t)hk * G + g) * d;
        if (rotate == 2)
          orc_transform(t_q + (size_t)hk * d * d, qi, d, &qr[(size_t)g * d]);
        else if (rotate)
          orc_rotate(qi, d, &qr[(size_t)g * d]);
        else
          for (int i = 0; i < d; ++i) qr[(size_t)g * d + i] = qi[i];
      }
      // energy of channel group p summed over the GQA group's query heads
      mask[(size_t)b * Hkv + hk] =
          select_mask(qr.data(), G, d, keep, energy ? energy + ((size_t)b * Hkv + hk) * npg : nullptr);
    }
}

void orc_select_buckets(const orc_cache* c, const float* q, int32_t Hq, const int32_t* lens, int32_t keep,
                        uint32_t* mask, double* energy) {
  const int d = c->head_dim, Hkv = c->kv_heads, G = Hq / Hkv, npg = d / kGranule, nb = n_buckets(c);
  std::vector<float> qr((size_t)G * d);
  for (int b = 0; b < c->batch; ++b)
    for (int k = 0; k < nb; ++k)
      for (int hk = 0; hk < Hkv; ++hk) {
        const long rel = (long)lens[b] - 1 - (long)k * c->bucket_w;  // query offset from bucket k's anchor
        for (int g = 0; g < G; ++g)
          prepare_row(c, hk, q + ((size_t)b * Hq + (size_t)hk * G + g) * d, true, rel, &qr[(size_t)g * d]);
        const size_t u = ((size_t)b * nb + k) * Hkv + hk;
        mask[u] = select_mask(qr.data(), G, d, keep, energy ? energy + u * npg : nullptr);
      }
}

void orc_attention(const orc_cache* c, const float* q, int32_t Hq, const int32_t* lens, const uint32_t* mask,
                   double scale, const int32_t* rows, int32_t nrows, double* out) {
  const int d = c->head_dim, G = Hq / c->kv_heads;
  const int total = rows ? nrows : c->batch * Hq;
#pragma omp parallel for schedule(dynamic, 1)
  for (int r = 0; r < total; ++r) {
    const int row = rows ? rows[r] : r;
    const int b = row / Hq, hq = row % Hq, hk = hq / G;
    double* o = out + (size_t)r * d;
    for (int ch = 0; ch < d; ++ch) o[ch] = 0.0;
    const int len = lens[b];
    if (len <= 0) continue;
    // the query as each bucket scores it (one bucket without bucket-relative RoPE)
    const int nb = n_buckets(c), used = c->bucket_w > 0 ? (len - 1) / c->bucket_w + 1 : 1;
    std::vector<float> qall((size_t)used * d);
    for (int k = 0; k < used; ++k)
      prepare_row(c, hk, q + (size_t)row * d, true, (long)len - 1 - (long)k * c->bucket_w, &qall[(size_t)k * d]);
    std::vector<double> s(len), khat(d), vhat(d);
    double smax = -std::numeric_limits<double>::infinity();
    for (int j = 0; j < len; ++j) {
      const int k = c->bucket_w > 0 ? j / c->bucket_w : 0;
      const float* qr = &qall[(size_t)k * d];
      const uint32_t m = mask ? mask[((size_t)b * nb + k) * c->kv_heads + hk] : 0xFFFFFFFFu;
      const uint16_t* kw = window_row(c, c->k_win, b, hk, j, len);
      double acc = 0.0;
      if (kw) {  // bf16 window token: every channel
        for (int ch = 0; ch < d; ++ch) acc += (double)qr[ch] * orc_bf16_value(kw[ch]);
      } else {
        orc_dequantize(c, b, hk, j, 1, khat.data(), nullptr);
        for (int ch = 0; ch < d; ++ch)
          if ((m >> (ch / kGranule)) & 1u) acc += (double)qr[ch] * khat[ch];
      }
      s[j] = scale * acc;
      if (s[j] > smax) smax = s[j];
    }
    // one softmax over every token of the sequence
    double l = 0.0;
    for (int j = 0; j < len; ++j) {
      s[j] = std::exp(s[j] - smax);
      l += s[j];
    }
    for (int j = 0; j < len; ++j) {
      const uint16_t* vw = window_row(c, c->v_win, b, hk, j, len);
      if (vw)
        for (int ch = 0; ch < d; ++ch) vhat[ch] = orc_bf16_value(vw[ch]);
      else
        orc_dequantize(c, b, hk, j, 1, nullptr, vhat.data());
      for (int ch = 0; ch < d; ++ch) o[ch] += s[j] * vhat[ch];
    }
    for (int ch = 0; ch < d; ++ch) o[ch] /= l;
    if (c->rotate_v) {
      // back from the rotated value basis: the orthonormal transform is its own inverse
      orc_fwht(o, d);
      const double inv = 1.0 / std::sqrt((double)d);
      for (int ch = 0; ch < d; ++ch) o[ch] *= inv;
    }
  }
}

double orc_dual_score(const double* T, int32_t d, const double* q, const double* k) {
  // q' = T q
  std::vector<double> qp(d, 0.0);
  for (int i = 0; i < d; ++i)
    for (int j = 0; j < d; ++j) qp[i] += T[(size_t)i * d + j] * q[j];
  // k' = T^{-T} k: solve T^T y = k by Gaussian elimination with partial pivoting
  std::vector<double> A((size_t)d * d), y(k, k + d);
  for (int i = 0; i < d; ++i)
    for (int j = 0; j < d; ++j) A[(size_t)i * d + j] = T[(size_t)j * d + i];
  for (int col = 0; col < d; ++col) {
    int piv = col;
    for (int r = col + 1; r < d; ++r)
      if (std::fabs(A[(size_t)r * d + col]) > std::fabs(A[(size_t)piv * d + col])) piv = r;
    if (A[(size_t)piv * d + col] == 0.0) return std::numeric_limits<double>::quiet_NaN();
    if (piv != col) {
      for (int j = 0; j < d; ++j) std::swap(A[(size_t)col * d + j], A[(size_t)piv * d + j]);
      std::swap(y[col], y[piv]);
    }
    for (int r = col + 1; r < d; ++r) {
      double f = A[(size_t)r * d + col] / A[(size_t)col * d + col];
      for (int j = col; j < d; ++j) A[(size_t)r * d + j] -= f * A[(size_t)col * d + j];
      y[r] -= f * y[col];
    }
  }
  for (int r = d - 1; r >= 0; --r) {
    double acc = y[r];
    for (int j = r + 1; j < d; ++j) acc -= A[(size_t)r * d + j] * y[j];
    y[r] = acc / A[(size_t)r * d + r];
  }
  double dot = 0.0;
  for (int i = 0; i < d; ++i) dot += qp[i] * y[i];
  return dot;
}

}  // extern "C"

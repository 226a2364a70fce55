// Fused rotate + quantize + pack + append kernel.
//
// One CTA handles the new tokens of one (sequence, kv head) that fall in one
// 64-token-aligned window of the cache; each of its 8 warps takes 8 tokens,
// four lanes per token, lane g of a token owning the 32 channels of
// quantization group g.  Keys: fp64 Walsh-Hadamard butterflies (Dual-QK
// summary Sec. 1; gist.science KQV scheme) or the kv head's key matrix of the
// caller's dual transform pair (Dual-QK Sec. 1, Sec. 3.1), optional bf16 channel 0 (Dual-QK
// Sec. 3.3, App. C.3), per-32-channel asymmetric quantization (Dual-QK
// Sec. 3.3).  Values: the same quantizer, optionally after the same rotation
// and with a clipping ratio on each group's range (Dual-QK App. B.2).
// Both code kinds are staged in shared memory and leave channel-major: key
// words one coalesced row per pruning group, value codes packed into each
// channel's row of the 128-token block.  Only tokens [offset, offset+n_new)
// change (tq-kv incremental cache); value-code words that also hold tokens
// outside that range are read, patched and written back by the one CTA whose
// window contains them.
#include "transform.cuh"

namespace kvq {
namespace {

constexpr int kAppendTile = 64;  // tokens per CTA window, aligned to absolute token positions
constexpr int kAppendWarps = 8;

// 3-input fp32 max / min (sm_100)
template <bool MAX>
__device__ __forceinline__ float mm3(float a, float b, float c) {
  float r;
  if (MAX)
    asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  else
    asm("min.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}
// max / min of v0, v[1..31] as a depth-4 tree
template <bool MAX>
__device__ __forceinline__ float reduce32(float v0, const float (&v)[32]) {
  float a[11];
  a[0] = mm3<MAX>(v0, v[1], v[2]);
#pragma unroll
  for (int i = 1; i < 10; ++i) a[i] = mm3<MAX>(v[3 * i], v[3 * i + 1], v[3 * i + 2]);
  a[10] = mm3<MAX>(v[30], v[31], v[31]);
  const float b0 = mm3<MAX>(a[0], a[1], a[2]), b1 = mm3<MAX>(a[3], a[4], a[5]);
  const float b2 = mm3<MAX>(a[6], a[7], a[8]), b3 = mm3<MAX>(a[9], a[10], a[10]);
  return mm3<MAX>(mm3<MAX>(b0, b1, b2), b3, b3);
}

// 1.5 * 2^23: for 0 <= q <= 2^22, q + kRoundMagic rounds q to the nearest
// integer (ties to even) and leaves it in the low significand bits
constexpr float kRoundMagic = 12582912.0f;
constexpr float kNear = 0.5f - 1e-5f;  // |q - round(q)| beyond this: next to a rounding boundary

// low bytes of four words -> one word, a in byte 0
__device__ __forceinline__ uint32_t pack_low_bytes(uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
  return __byte_perm(__byte_perm(a, b, 0x0040), __byte_perm(c, d, 0x0040), 0x5410);
}
// four codes (bytes 0..3 of x, each < 2^BITS) -> one BITS*4-bit word, byte 0 lowest
template <int BITS>
__device__ __forceinline__ uint32_t compress_codes(uint32_t x) {
  if (BITS == 4) {
    x |= x >> 4;  // byte 0: c0 | c1 << 4, byte 2: c2 | c3 << 4
    return __byte_perm(x, 0, 0x0020) & 0xFFFFu;
  } else {
    x |= x >> 6;  // byte 0: c0 | c1 << 2, byte 2: c2 | c3 << 2
    return (x | (x >> 12)) & 0xFFu;
  }
}

// Quantize one 32-channel group held by this lane (v[0..31]); skip0: element 0
// is kept out of the range and gets code 0; clip: the clipping ratio applied to
// the group's minimum and maximum.  Returns the fp16 (scale, zero) pair; byte j
// of packed[p] is the code of element 4p + j.
//
// The code is round_half_even((x - zero) / scale) clamped to [0, L], the
// quotient as IEEE fp32 division gives it.  It is formed as
// q = (x - zero) * rcp(scale) with a correctly rounded reciprocal and clamped
// to [0, L] (the bounds are integers, so clamp and round commute); q is then
// within 2^-22 * q < 4e-6 of the clamped IEEE quotient.  When an element's q
// lies within 1e-5 of a rounding boundary (k + 1/2) the group is coded again
// with the IEEE division for such elements, so every code is the division's.
template <int BITS>
__device__ __forceinline__ __half2 quantize_group32(const float (&v)[32], bool skip0, float clip,
                                                   uint32_t (&packed)[8]) {
  const float v0 = skip0 ? v[1] : v[0];
  // -0 and +0 are the same extreme; take it as +0 so the stored bits are unique;
  // then the clipping ratio scales both ends (exact for clip = 1)
  const float mn = __fmul_rn(clip, __fadd_rn(reduce32<false>(v0, v), 0.0f));
  const float mx = __fmul_rn(clip, __fadd_rn(reduce32<true>(v0, v), 0.0f));
  constexpr int L = (1 << BITS) - 1;
  const float s32 = fminf(__fdiv_rn(__fsub_rn(mx, mn), (float)L), 65504.0f);
  const float zc = fminf(fmaxf(mn, -65504.0f), 65504.0f);
  const __half s16 = __float2half_rn(s32), z16 = __float2half_rn(zc);
  const float sf = __half2float(s16), zf = __half2float(z16);
  const float rs = sf != 0.0f ? __frcp_rn(sf) : 0.0f;  // sf == 0: every code is 0
  float near[4] = {0.0f, 0.0f, 0.0f, 0.0f};
#pragma unroll
  for (int p = 0; p < 8; ++p) {
    uint32_t m[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float q = fminf(fmaxf(__fmul_rn(__fsub_rn(v[4 * p + j], zf), rs), 0.0f), (float)L);
      const float mq = __fadd_rn(q, kRoundMagic);
      const float d = fabsf(__fsub_rn(q, __fsub_rn(mq, kRoundMagic)));  // exact: |q - round(q)|
      near[j] = fmaxf(near[j], (p == 0 && j == 0 && skip0) ? 0.0f : d);
      m[j] = __float_as_uint(mq);
    }
    packed[p] = pack_low_bytes(m[0], m[1], m[2], m[3]);
  }
  if (mm3<true>(mm3<true>(near[0], near[1], near[2]), near[3], near[3]) > kNear) {
    // rare: code the group again, with the IEEE division next to a boundary
#pragma unroll
    for (int p = 0; p < 8; ++p) {
      uint32_t m[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const float d = __fsub_rn(v[4 * p + j], zf);
        float q = fminf(fmaxf(__fmul_rn(d, rs), 0.0f), (float)L);
        if (fabsf(__fsub_rn(q, rintf(q))) > kNear) q = fminf(fmaxf(rintf(__fdiv_rn(d, sf)), 0.0f), (float)L);
        m[j] = __float_as_uint(__fadd_rn(q, kRoundMagic));
      }
      packed[p] = pack_low_bytes(m[0], m[1], m[2], m[3]);
    }
  }
  if (skip0) packed[0] &= 0xFFFFFF00u;
  return __halves2half2(s16, z16);
}

// 32 consecutive input elements held raw: 64 bytes (16-bit types) or 128 (fp32)
template <typename In>
struct Raw32 {
  uint4 w[sizeof(In) * 2];
};
template <typename In>
__device__ __forceinline__ void load_raw(const In* p, Raw32<In>& r) {
#pragma unroll
  for (int j = 0; j < (int)sizeof(In) * 2; ++j) r.w[j] = reinterpret_cast<const uint4*>(p)[j];
}
__device__ __forceinline__ void widen2(uint32_t u, const __nv_bfloat16*, float& a, float& b) {
  a = __uint_as_float(u << 16);
  b = __uint_as_float(u & 0xFFFF0000u);
}
__device__ __forceinline__ void widen2(uint32_t u, const __half*, float& a, float& b) {
  const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&u));
  a = f.x;
  b = f.y;
}
// exact widening to fp32
template <typename In>
__device__ __forceinline__ void widen(const Raw32<In>& r, float (&f)[32]) {
  if constexpr (sizeof(In) == 4) {
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      f[4 * j] = __uint_as_float(r.w[j].x);
      f[4 * j + 1] = __uint_as_float(r.w[j].y);
      f[4 * j + 2] = __uint_as_float(r.w[j].z);
      f[4 * j + 3] = __uint_as_float(r.w[j].w);
    }
  } else {
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      widen2(r.w[j].x, (const In*)nullptr, f[8 * j], f[8 * j + 1]);
      widen2(r.w[j].y, (const In*)nullptr, f[8 * j + 2], f[8 * j + 3]);
      widen2(r.w[j].z, (const In*)nullptr, f[8 * j + 4], f[8 * j + 5]);
      widen2(r.w[j].w, (const In*)nullptr, f[8 * j + 6], f[8 * j + 7]);
    }
  }
}

// 4x4 byte transpose: out[j] byte k = byte j of in[k]
__device__ __forceinline__ void transpose_bytes4(const uint32_t (&in)[4], uint32_t (&out)[4]) {
  const uint32_t t0 = __byte_perm(in[0], in[1], 0x5140), t1 = __byte_perm(in[0], in[1], 0x7362);
  const uint32_t t2 = __byte_perm(in[2], in[3], 0x5140), t3 = __byte_perm(in[2], in[3], 0x7362);
  out[0] = __byte_perm(t0, t2, 0x5410);
  out[1] = __byte_perm(t0, t2, 0x7632);
  out[2] = __byte_perm(t1, t3, 0x5410);
  out[3] = __byte_perm(t1, t3, 0x7632);
}

// Orthonormal Walsh-Hadamard transform of one 128-channel row held by four
// lanes, lane g holding channels 32g .. 32g+31: butterflies in fp64, natural
// Sylvester order (stage h pairs channels i and i + h, i & h == 0, -> (a + b,
// a - b)); the stages below 32 stay inside the lane, 32 and 64 pair lanes g ^ 1
// and g ^ 2; then one fp64 multiply by 1/sqrt(128) and a round to fp32.  All
// 32 lanes of the warp take part.
__device__ __forceinline__ void rotate_row_4lanes(float (&v)[32], int g, double inv_sqrt_d) {
  double x[32];
#pragma unroll
  for (int i = 0; i < 32; ++i) x[i] = v[i];
#pragma unroll
  for (int hs = 1; hs < 32; hs <<= 1)
#pragma unroll
    for (int i = 0; i < 32; ++i)
      if ((i & hs) == 0) {
        const double u = x[i], w = x[i + hs];
        x[i] = __dadd_rn(u, w);
        x[i + hs] = __dsub_rn(u, w);
      }
#pragma unroll
  for (int m = 1; m <= 2; m <<= 1) {
    const bool upper = (g & m) != 0;
#pragma unroll
    for (int i = 0; i < 32; ++i) {
      // lower lane: x + o; upper lane: o - x = o + (-x), the same IEEE sum
      const double o = __shfl_xor_sync(kFull, x[i], m);
      x[i] = __dadd_rn(upper ? -x[i] : x[i], o);
    }
  }
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] = __double2float_rn(__dmul_rn(x[i], inv_sqrt_d));
}

// Key rows of the window's 64 tokens through the kv head's matrix A of the
// caller's transform pair, as one 64 x 128 x 128 product: channel i of token t
// is the fp64 sum over j = 0..127, in order, of A[i][j] x_tj, rounded to fp32.
// A product of two fp32 numbers is exact in fp64, so a fused multiply-add per
// step rounds once, as a rounded sum of the rounded product does: the result is
// that in-order sum bit for bit.  On entry lane (tt, g) holds channels
// 32g .. 32g+31 of token tt in v; on return the transformed ones.  Every thread
// of the block takes part.  Dynamic shared memory: A^T in fp64 as [j][i]
// (128 KB) and X^T in fp64 as [j][t] (64 KB), token t of row j at column
// (t + 8 (j / 32)) mod 64 so that the four lanes of a token store into
// distinct banks; the fp32 results then take X^T's space as rows [t][i].
constexpr int kPairYStride = kHeadDim + 4;  // floats per token row of the results
constexpr size_t kPairSmemBytes = sizeof(double) * kHeadDim * (kHeadDim + kAppendTile);

__device__ __forceinline__ void transform_rows_block(float (&v)[32], int g, int tt, const float* __restrict__ A,
                                                     double* __restrict__ sA, double* __restrict__ sX) {
  static_assert(kAppendWarps * 32 == 256 && kAppendTile == 64, "thread layout of the product");
#pragma unroll
  for (int r = 0; r < 32; ++r) sX[(32 * g + r) * kAppendTile + ((tt + 8 * g) & (kAppendTile - 1))] = (double)v[r];
  // A^T: thread e converts A[i][4q .. 4q+3], i = e mod 128 (consecutive threads,
  // consecutive i: conflict-free stores)
  const float4* A4 = reinterpret_cast<const float4*>(A);
#pragma unroll 4
  for (int e = threadIdx.x; e < kHeadDim * kHeadDim / 4; e += 256) {
    const int i = e & (kHeadDim - 1), q = e >> 7;
    const float4 m = __ldg(A4 + i * (kHeadDim / 4) + q);
    double* d = sA + 4 * q * kHeadDim + i;
    d[0] = (double)m.x;
    d[kHeadDim] = (double)m.y;
    d[2 * kHeadDim] = (double)m.z;
    d[3 * kHeadDim] = (double)m.w;
  }
  __syncthreads();
  // thread: tokens tb + 16 s (s < 4), channels 8 ib .. 8 ib + 7; a warp reads
  // two A^T addresses (broadcast) and 16 consecutive X^T entries per load
  const int tb = threadIdx.x & 15, ib = threadIdx.x >> 4;
  double acc[4][8];
#pragma unroll
  for (int s = 0; s < 4; ++s)
#pragma unroll
    for (int r = 0; r < 8; ++r) acc[s][r] = 0.0;
#pragma unroll 1
  for (int jg = 0; jg < 4; ++jg) {
    int xo[4];
#pragma unroll
    for (int s = 0; s < 4; ++s) xo[s] = (tb + 16 * s + 8 * jg) & (kAppendTile - 1);
#pragma unroll 4
    for (int j = 32 * jg; j < 32 * jg + 32; ++j) {
      const double2* ar = reinterpret_cast<const double2*>(sA + j * kHeadDim + 8 * ib);
      double a[8], x[4];
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const double2 p = ar[k];
        a[2 * k] = p.x;
        a[2 * k + 1] = p.y;
      }
#pragma unroll
      for (int s = 0; s < 4; ++s) x[s] = sX[j * kAppendTile + xo[s]];
#pragma unroll
      for (int s = 0; s < 4; ++s)
#pragma unroll
        for (int r = 0; r < 8; ++r) acc[s][r] = __fma_rn(a[r], x[s], acc[s][r]);
    }
  }
  __syncthreads();  // X^T is read: its space takes the results
  float* sY = reinterpret_cast<float*>(sX);
#pragma unroll
  for (int s = 0; s < 4; ++s)
#pragma unroll
    for (int h = 0; h < 2; ++h)
      *reinterpret_cast<float4*>(sY + (tb + 16 * s) * kPairYStride + 8 * ib + 4 * h) =
          make_float4(__double2float_rn(acc[s][4 * h]), __double2float_rn(acc[s][4 * h + 1]),
                      __double2float_rn(acc[s][4 * h + 2]), __double2float_rn(acc[s][4 * h + 3]));
  __syncthreads();
#pragma unroll
  for (int m = 0; m < 8; ++m) {
    const float4 o = *reinterpret_cast<const float4*>(sY + tt * kPairYStride + 32 * g + 4 * m);
    v[4 * m] = o.x;
    v[4 * m + 1] = o.y;
    v[4 * m + 2] = o.z;
    v[4 * m + 3] = o.w;
  }
}

// Rotary embedding of one key row held by four lanes as above, at position
// pos (Dual-QK Sec. 3.4, bucket-relative RoPE): channel i < 64 pairs with
// i + 64, held by lane group g ^ 2; angle pos * inv_freq[i mod 64] in fp64,
// x_i cos - x_{i+64} sin below, x_{i+64} cos + x_i sin above, each product and
// sum rounded once, then rounded to fp32.  All 32 lanes of the warp take part.
__device__ __forceinline__ void rope_row_4lanes(float (&v)[32], int g, int pos, const float* __restrict__ inv_freq) {
  const bool upper = g >= 2;
  const int f0 = 32 * (g & 1);
#pragma unroll
  for (int i = 0; i < 32; ++i) {
    const double other = (double)__shfl_xor_sync(kFull, v[i], 2);
    double sn, cs;
    sincos(__dmul_rn((double)pos, (double)__ldg(inv_freq + f0 + i)), &sn, &cs);
    const double own = __dmul_rn((double)v[i], cs), cross = __dmul_rn(other, sn);
    v[i] = __double2float_rn(upper ? __dadd_rn(own, cross) : __dsub_rn(own, cross));
  }
}

// bf16 (round to nearest even) copy of this lane's 32 channels into a window row
__device__ __forceinline__ void store_bf16_32(__nv_bfloat16* dst, const float (&v)[32]) {
  uint32_t w[16];
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    const __nv_bfloat162 p = __floats2bfloat162_rn(v[2 * i], v[2 * i + 1]);
    w[i] = *reinterpret_cast<const uint32_t*>(&p);
  }
  uint4* d = reinterpret_cast<uint4*>(dst);
#pragma unroll
  for (int i = 0; i < 4; ++i) d[i] = make_uint4(w[4 * i], w[4 * i + 1], w[4 * i + 2], w[4 * i + 3]);
}

// ROT & 3: 0 keys as given, 1 Walsh-Hadamard rotation, 2 the pair's key
// matrix tk[h] (192 KB of dynamic shared memory: one resident block); ROT & 4: keys first rotary-embedded at their token index in the
// view (the offset from their bucket's anchor), frequencies inv_freq
template <int KB, int VB, int ROT, bool CH0, bool ROTV, typename In>
__global__ void __launch_bounds__(kAppendWarps * 32, (ROT & 3) == 2 ? 1 : 3)
    k_quantize_append(AppendArgs a, const float* __restrict__ tk, const float* __restrict__ inv_freq) {
  constexpr int TPW = 32 / VB;            // value tokens per 32-bit word: 8 (INT4) or 16 (INT2)
  constexpr int WPR = kAppendTile / TPW;  // value words per channel in the window: 8 or 4
  // key words [pruning group][token], 16 bits a token (its KB * 4 low bits used)
  __shared__ __align__(16) uint16_t kw[kPruneGroups][kAppendTile + 2];
  // value codes [token][channel], one byte each; rows padded to 144 bytes so
  // that the 16-byte stores of the 8 tokens a quarter-warp holds fall on
  // distinct banks
  __shared__ __align__(16) uint8_t vcode[kAppendTile][kHeadDim + 16];
  // packed value words [word][channel]; rows padded by TPW words so that the
  // TPW-channel x WPR-word block a warp reads falls on distinct banks
  __shared__ __align__(16) uint32_t vword[WPR][kHeadDim + TPW];

  const CacheView& c = a.c;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int h = blockIdx.y, b = blockIdx.z;
  const int w0 = (a.offset / kAppendTile + blockIdx.x) * kAppendTile;  // absolute first token of the window
  const int lo = max(a.offset - w0, 0);                                // window tokens [lo, hi) are new
  const int hi = min(a.offset + a.n_new - w0, kAppendTile);
  const size_t bh = (size_t)b * c.H + h;
  const int tb0 = w0 % kKeyBlock;                                      // window start inside its block: 0 or 64
  const size_t unit_blk = bh * (size_t)(c.cap / kKeyBlock) + w0 / kKeyBlock;  // (unit, block) index
  // four lanes per token, lane group g = lane & 3 holding channels 32g .. 32g+31
  const int g = lane & 3;
  const int tt = warp * 8 + (lane >> 2);  // window token of this lane
  const bool active = tt >= lo && tt < hi;
  // input row of window token tt: (bh * n_new + w0 + tt - offset), never negative when active
  const size_t row = bh * a.n_new + (size_t)(w0 + (active ? tt : lo) - a.offset);
  const In* kin = static_cast<const In*>(a.k_new) + row * kHeadDim + 32 * g;
  const In* vin = static_cast<const In*>(a.v_new) + row * kHeadDim + 32 * g;

  Raw32<In> kraw, vraw;  // value loads issued together with the key loads
  if (active) {
    load_raw(kin, kraw);
    load_raw(vin, vraw);
  } else {
#pragma unroll
    for (int j = 0; j < (int)sizeof(In) * 2; ++j) kraw.w[j] = vraw.w[j] = make_uint4(0, 0, 0, 0);
  }
  float kx[32];
  widen(kraw, kx);

  // ---- key row: rotated, then quantized (keys are not clipped)
  if (ROT & 4) rope_row_4lanes(kx, g, w0 + tt, inv_freq);
  if ((ROT & 3) == 1) rotate_row_4lanes(kx, g, a.inv_sqrt_d);
  if ((ROT & 3) == 2) {
    extern __shared__ __align__(16) double pair_smem[];
    transform_rows_block(kx, g, tt, tk + (size_t)h * kPairElems, pair_smem, pair_smem + kHeadDim * kHeadDim);
  }
  // bf16 window copies (rotated key, then the value below) for tokens with a
  // window slot: every sink token, and of the later tokens only this append's
  // last `recent`, the ones that still own their ring slot when it ends (an
  // earlier token of the same append would race with them for the slot)
  // (positions count from the view's first token: a bucket's anchor with
  // bucket-relative RoPE, whose view's window rows are its sequence's)
  const int wn = c.pos_base + w0 + tt;
  const int wslot = active && (wn < c.sink || wn >= c.pos_base + a.offset + a.n_new - c.recent)
                        ? window_slot(c.sink, c.recent, wn) : -1;
  if (wslot >= 0 &&
      kvq_in_bounds((bh * (size_t)(c.sink + c.recent) + wslot) * kHeadDim + 32 * g, 32, c.win_elems()))
    store_bf16_32(c.kwin + (bh * (size_t)(c.sink + c.recent) + wslot) * kHeadDim + 32 * g, kx);
  uint32_t code[8];
  {
    const bool skip0 = CH0 && g == 0;
    const __half2 sz = quantize_group32<KB>(kx, skip0, 1.0f, code);
#pragma unroll
    for (int p = 0; p < 8; ++p) kw[8 * g + p][tt] = (uint16_t)compress_codes<KB>(code[p]);
    if (active) {
      const size_t ksi = (unit_blk * kGroups + g) * kKeyBlock + tb0 + tt;
      if (kvq_in_bounds(ksi, 1, c.ks_pairs())) c.ks[ksi] = sz;
      if (skip0 && kvq_in_bounds(bh * c.cap + w0 + tt, 1, c.rows())) c.k0[bh * c.cap + w0 + tt] = __float2bfloat16_rn(kx[0]);
    }
  }
  // ---- value row: optionally rotated, the same quantizer with the clipping
  // ratio; codes as bytes, scales token-major
  {
    float vx[32];
    widen(vraw, vx);
    if (ROTV) rotate_row_4lanes(vx, g, a.inv_sqrt_d);
    if (wslot >= 0 &&
        kvq_in_bounds((bh * (size_t)(c.sink + c.recent) + wslot) * kHeadDim + 32 * g, 32, c.win_elems()))
      store_bf16_32(c.vwin + (bh * (size_t)(c.sink + c.recent) + wslot) * kHeadDim + 32 * g, vx);
    const __half2 sz = quantize_group32<VB>(vx, false, c.v_clip, code);
    if (!active) {
#pragma unroll
      for (int p = 0; p < 8; ++p) code[p] = 0;  // tokens outside the append contribute zero bits
    } else if (kvq_in_bounds((bh * c.cap + w0 + tt) * kGroups + g, 1, c.ks_pairs())) {
      c.vs[(bh * c.cap + w0 + tt) * kGroups + g] = sz;
    }
    *reinterpret_cast<uint4*>(&vcode[tt][32 * g]) = make_uint4(code[0], code[1], code[2], code[3]);
    *reinterpret_cast<uint4*>(&vcode[tt][32 * g + 16]) = make_uint4(code[4], code[5], code[6], code[7]);
  }
  __syncthreads();

  // ---- key rows out: one pruning group's run per warp, two tokens a lane
  {
    const int t = 2 * lane;  // window tokens t, t + 1
    const bool a0 = t >= lo && t < hi, a1 = t + 1 >= lo && t + 1 < hi;
    for (int pg = warp; pg < kPruneGroups; pg += kAppendWarps) {
      const size_t idx = (unit_blk * kPruneGroups + pg) * kKeyBlock + tb0 + t;
      const uint32_t w2 = *reinterpret_cast<const uint32_t*>(&kw[pg][t]);  // token t in the low half
      if (!kvq_in_bounds(idx * (KB == 4 ? 2 : 1), KB == 4 ? 4 : 2, c.kc_bytes())) continue;
      if (KB == 4) {
        uint16_t* dst = reinterpret_cast<uint16_t*>(c.kc) + idx;
        if (a0 && a1)
          *reinterpret_cast<uint32_t*>(dst) = w2;
        else if (a0)
          dst[0] = (uint16_t)w2;
        else if (a1)
          dst[1] = (uint16_t)(w2 >> 16);
      } else {
        uint8_t* dst = c.kc + idx;
        const uint32_t b2 = (w2 & 0xFFu) | ((w2 >> 8) & 0xFF00u);
        if (a0 && a1)
          *reinterpret_cast<uint16_t*>(dst) = (uint16_t)b2;
        else if (a0)
          dst[0] = (uint8_t)b2;
        else if (a1)
          dst[1] = (uint8_t)(b2 >> 8);
      }
    }
  }

  // ---- value codes: each thread packs 4 channels x TPW tokens into 4 words
  // (token order, low bits first) with byte transposes
  if (threadIdx.x < 32 * WPR) {
    const int c4 = threadIdx.x & 31, w = threadIdx.x >> 5;  // channels 4 c4 .. 4 c4 + 3, word w
    uint32_t out[4] = {0u, 0u, 0u, 0u};
#pragma unroll
    for (int k = 0; k < TPW / 4; ++k) {
      uint32_t in[4], col[4];
#pragma unroll
      for (int r = 0; r < 4; ++r) in[r] = *reinterpret_cast<const uint32_t*>(&vcode[w * TPW + 4 * k + r][4 * c4]);
      transpose_bytes4(in, col);  // col[j]: channel 4 c4 + j, tokens 4k .. 4k + 3
#pragma unroll
      for (int j = 0; j < 4; ++j) out[j] |= compress_codes<VB>(col[j]) << (4 * VB * k);
    }
    *reinterpret_cast<uint4*>(&vword[w][4 * c4]) = make_uint4(out[0], out[1], out[2], out[3]);
  }
  __syncthreads();
  // ...and store them into the channel rows of the 128-token block
  constexpr int TPC = 16 * 8 / VB;  // tokens per 16-byte chunk: 32 or 64
  uint8_t* vblk = c.vc + unit_blk * (size_t)(kHeadDim * (kKeyBlock * VB / 8));
  for (int i = threadIdx.x; i < kHeadDim * WPR; i += blockDim.x) {
    const int ch = i / WPR, w = i % WPR;  // a warp: 32 / WPR channels, all their words
    const int t0 = w * TPW;               // first window token of the word
    const int a0 = max(lo - t0, 0), a1 = min(hi - t0, TPW);  // new tokens of this word: [a0, a1)
    if (a0 >= a1) continue;
    const int tb = tb0 + t0;  // ... inside the block
    const int chunk = (tb / TPC) ^ v_chunk_swizzle(VB, ch);
    uint32_t* dst =
        reinterpret_cast<uint32_t*>(vblk + ch * (kKeyBlock * VB / 8) + chunk * 16 + (tb % TPC) / (8 / VB));
    if (!kvq_in_bounds((size_t)(reinterpret_cast<uint8_t*>(dst) - c.vc), 4, c.vc_bytes())) continue;
    uint32_t word = vword[w][ch];
    if (a0 > 0 || a1 < TPW) {
      const uint32_t keep_lo = a0 * VB >= 32 ? ~0u : ((1u << (a0 * VB)) - 1u);
      const uint32_t keep_hi = a1 * VB >= 32 ? 0u : ~((1u << (a1 * VB)) - 1u);
      word |= *dst & (keep_lo | keep_hi);  // the other tokens' codes stay as they were
    }
    *dst = word;
  }
}

template <int KB, int VB, int ROT, bool CH0, bool ROTV>
cudaError_t launch_typed(const AppendArgs& a, const float* tk, const float* fr, cudaStream_t s) {
  const int first = a.offset / kAppendTile, last = (a.offset + a.n_new - 1) / kAppendTile;
  dim3 grid(last - first + 1, a.c.H, a.c.B);
  dim3 block(kAppendWarps * 32);
  auto kern = a.dtype == KVQ_F32 ? k_quantize_append<KB, VB, ROT, CH0, ROTV, float>
                                 : (a.dtype == KVQ_BF16 ? k_quantize_append<KB, VB, ROT, CH0, ROTV, __nv_bfloat16>
                                                        : k_quantize_append<KB, VB, ROT, CH0, ROTV, __half>);
  const size_t smem = (ROT & 3) == 2 ? kPairSmemBytes : 0;
  if (smem) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
  }
  kern<<<grid, block, smem, s>>>(a, tk, fr);
  return cudaGetLastError();
}

template <int KB, int VB, int ROT, bool ROTV>
cudaError_t launch_ch0(const AppendArgs& a, const float* tk, const float* fr, cudaStream_t s) {
  return a.c.keep_ch0 ? launch_typed<KB, VB, ROT, true, ROTV>(a, tk, fr, s)
                      : launch_typed<KB, VB, ROT, false, ROTV>(a, tk, fr, s);
}

template <int KB, int VB, bool ROTV>
cudaError_t launch_flags(const AppendArgs& a, const float* tk, const float* fr, cudaStream_t s) {
  switch (a.c.rotate + (fr ? 4 : 0)) {
    case 0: return launch_ch0<KB, VB, 0, ROTV>(a, tk, fr, s);
    case 1: return launch_ch0<KB, VB, 1, ROTV>(a, tk, fr, s);
    case 2: return launch_ch0<KB, VB, 2, ROTV>(a, tk, fr, s);
    case 4: return launch_ch0<KB, VB, 4, ROTV>(a, tk, fr, s);
    case 5: return launch_ch0<KB, VB, 5, ROTV>(a, tk, fr, s);
    default: return launch_ch0<KB, VB, 6, ROTV>(a, tk, fr, s);
  }
}

// value rotation is a template flag, so kernels without it stay as small as before
template <int KB, int VB>
cudaError_t launch_bits(const AppendArgs& a, const float* tk, const float* fr, cudaStream_t s) {
  return a.c.rotate_v ? launch_flags<KB, VB, true>(a, tk, fr, s) : launch_flags<KB, VB, false>(a, tk, fr, s);
}

}  // namespace

cudaError_t launch_append_ext(const AppendArgs& a, const float* tk, const float* fr, cudaStream_t s) {
  if (a.c.k_bits == 4 && a.c.v_bits == 4) return launch_bits<4, 4>(a, tk, fr, s);
  if (a.c.k_bits == 4) return launch_bits<4, 2>(a, tk, fr, s);
  if (a.c.v_bits == 4) return launch_bits<2, 4>(a, tk, fr, s);
  return launch_bits<2, 2>(a, tk, fr, s);
}

cudaError_t launch_append(const AppendArgs& a, cudaStream_t s) { return launch_append_ext(a, nullptr, nullptr, s); }

KVQ_BOUNDS_COUNTER(bounds_append)

}  // namespace kvq

// Split-sequence decode attention on the 5th-generation tensor cores (tcgen05).
//
// Same contract as the CUDA-core kernel (one CTA per (split, kv head,
// sequence); per-split running max / sum / accumulator out), for GQA groups
// of G = 4, 8 or 16 query heads.  Per 128-token tile:
//
//  1. one thread streams the raw tile into a shared-memory stage with 1-D bulk
//     async copies (only the key-code rows of kept channel groups, the key
//     scales, channel 0, the value codes and value scales), two stages deep;
//  2. all 256 threads turn the key codes into exact f16 integers (tile A,
//     K-major: token x channel);
//  3. one thread issues 8 UMMAs D_g[token][hi/lo x head] = A[token][ch in g]
//     . Q[hi/lo x head][ch in g], one f32 accumulator per 32-channel group g in
//     tensor memory, so each token's per-group key scale and zero are applied
//     exactly afterwards: score = sum_g s_g (D_hi + D_lo) + z_g sum_{c in g} q_c
//     (+ q_0 k_ch0).  No dequantized key exists anywhere (tq-kv abstract;
//     Dual-QK summary Sec. 3.2, 3.3).  q is split into f16 hi + lo parts, so
//     the product keeps ~22 bits of q;
//  4. thread (token, head half) reads its scores from tensor memory, the CTA
//     agrees on the tile max, and each thread forms p = 2^(s - m) and
//     P'[token][g x head] = p * value scale_g into tile B (f16), and keeps the
//     value zero-point term sum p * zero_g and the running sum in registers;
//  5. the value codes become exact f16 integers in tile A (now MN-major:
//     channel x token) and one thread issues 8 UMMAs
//     O[channel][g x head] = A[channel][token] . P'[token][g x head];
//  6. thread (channel, head half) adds O[channel][group(channel) x head] into
//     its rescaled register accumulator.
// The combine pass merges splits into one softmax (Dual-QK summary Sec. 3.4).
//
// The code -> f16 step emits channel pairs in a fixed interleaved order; the
// query operand (score) and the tensor-memory lane -> channel map (PV) use the
// same order, so nothing is reshuffled.  Every wait on an mbarrier is bounded;
// a CTA that gives up writes NaN partials instead of hanging.
#include "common.cuh"
#include "sm100.cuh"

namespace kvq {
namespace {

using namespace sm100;

constexpr int kTcThreads = 256;
constexpr int kTile = 128;

template <int G, int KB, int VB, bool CH0>
struct TcShape {
  static constexpr int NS = 2 * G < 16 ? 16 : 2 * G;  // score columns per group: hi, lo per head (+ zero pad)
  static constexpr int NO = 4 * G;        // PV columns: group x head
  static constexpr int HH = G / 2;        // heads per thread half
  static constexpr int TMEM_USED = 4 * NS + NO;
  static constexpr int TMEM_COLS = TMEM_USED <= 64 ? 64 : (TMEM_USED <= 128 ? 128 : 256);
  static constexpr int KW = KB == 4 ? 2 : 1;          // bytes per key-code word (one channel group of 4)
  static constexpr int KROW = kTile * KW;             // bytes per key-code row of a tile
  static constexpr int VROW = kHeadDim * VB / 8;      // bytes per value row
  // shared-memory layout (bytes)
  static constexpr int A_OFF = 0;                     // 128 x 128 f16 operand tile
  static constexpr int BQ_OFF = A_OFF + kTile * kHeadDim * 2;
  static constexpr int BP_OFF = BQ_OFF + NS * kHeadDim * 2;
  static constexpr int RAW_OFF = BP_OFF + NO * kTile * 2;
  static constexpr int R_KC = 0;
  static constexpr int R_KS = R_KC + kPruneGroups * KROW;
  static constexpr int R_K0 = R_KS + kGroups * kTile * 4;
  static constexpr int R_VC = R_K0 + (CH0 ? kTile * 2 : 0);
  static constexpr int R_VS = R_VC + kTile * VROW;
  static constexpr int RAW_BYTES = R_VS + kTile * kGroups * 4;
  static constexpr int MISC_OFF = RAW_OFF + 2 * RAW_BYTES;
  // misc: qsum[G][4] f32, q0[G] f32, two reduction arrays [2 halves][4 warps][8] f32,
  // 3 mbarriers, the tensor-memory address slot
  static constexpr int QSUM_OFF = MISC_OFF;
  static constexpr int Q0_OFF = QSUM_OFF + G * kGroups * 4;
  static constexpr int RED_OFF = Q0_OFF + G * 4;
  static constexpr int RED_BYTES = 2 * (2 * 4 * 8) * 4;
  static constexpr int BAR_OFF = ((RED_OFF + RED_BYTES + 7) / 8) * 8;
  static constexpr int SLOT_OFF = BAR_OFF + 3 * 8;
  static constexpr int SMEM_BYTES = SLOT_OFF + 16;
};

// Position, within its 8- (INT4) or 16-channel (INT2) block, that the code ->
// f16 conversion gives channel offset i.
template <int BITS>
__device__ __forceinline__ int pos_of(int i) {
  if (BITS == 4) return i < 4 ? 2 * i : 2 * (i - 4) + 1;
  return i < 8 ? 2 * i : 2 * (i - 8) + 1;
}
// Channel held at operand position p (inverse of pos_of over the whole row).
template <int BITS>
__device__ __forceinline__ int chan_of(int p) {
  if (BITS == 4) return (p & ~7) + ((p & 7) >> 1) + 4 * (p & 1);
  return (p & ~15) + ((p & 15) >> 1) + 8 * (p & 1);
}

// byte offset of element (row r, col k) in a no-swizzle K-major tile whose
// 8-row groups are 2048 B apart and whose 8-column chunks are 128 B apart
__device__ __forceinline__ uint32_t kmajor_off(int r, int k) {
  return (r & 7) * 16 + (k & 7) * 2 + (k >> 3) * 128 + (r >> 3) * 2048;
}
// byte offset of element (mn, k) in a no-swizzle MN-major tile: 8-element MN
// chunks 2048 B apart, 8-deep K groups 128 B apart
__device__ __forceinline__ uint32_t mnmajor_off(int mn, int k) {
  return (mn & 7) * 2 + (k & 7) * 16 + (mn >> 3) * 2048 + (k >> 3) * 128;
}

template <int G, int KB, int VB, bool CH0>
__device__ __forceinline__ void issue_tile_loads(const DecodeArgs& a, uint8_t* raw, uint32_t bar, size_t bh,
                                                 int n0, uint32_t msk) {
  using S = TcShape<G, KB, VB, CH0>;
  const CacheView& c = a.c;
  const int ntc = kTile;  // cap and n0 are multiples of the 128-token key block
  uint32_t bytes = 0;
  bytes += (uint32_t)__popc(msk) * ntc * S::KW;
  bytes += kGroups * ntc * 4;
  if (CH0 && (msk & 1u)) bytes += ntc * 2;
  bytes += ntc * S::VROW + ntc * 16;
  mbar_arrive_expect_tx(bar, bytes);
  const uint32_t dst = smem_addr(raw);
  for (int pg = 0; pg < kPruneGroups; ++pg)
    if ((msk >> pg) & 1u)
      bulk_g2s(dst + S::R_KC + pg * S::KROW, c.kc + key_word_index(bh, c.cap, pg, n0) * S::KW, ntc * S::KW, bar);
  // the block's 4 scale rows are contiguous
  bulk_g2s(dst + S::R_KS, c.ks + key_scale_index(bh, c.cap, 0, n0), kGroups * ntc * 4, bar);
  if (CH0 && (msk & 1u)) bulk_g2s(dst + S::R_K0, c.k0 + bh * c.cap + n0, ntc * 2, bar);
  bulk_g2s(dst + S::R_VC, c.vc + (bh * c.cap + n0) * S::VROW, ntc * S::VROW, bar);
  bulk_g2s(dst + S::R_VS, c.vs + (bh * c.cap + n0) * kGroups, ntc * 16, bar);
}

template <int G, int KB, int VB, bool CH0, typename In>
__global__ void __launch_bounds__(kTcThreads, 2) k_decode_split_tc(DecodeArgs a) {
  using S = TcShape<G, KB, VB, CH0>;
  constexpr int HH = S::HH;
  extern __shared__ __align__(1024) uint8_t smem[];
  const CacheView& c = a.c;
  const int split = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int len = min(max(a.seq_lens[b], 0), a.max_len);
  const int start = split * a.split_tokens;
  if (start >= len) return;
  const int end = min(start + a.split_tokens, len);
  const int ntiles = (end - start + kTile - 1) / kTile;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int half = tid >> 7;   // head half (epilogue / PV), also the channel half for key conversion
  const int j = tid & 127;     // token of the tile (conversion, score) == tensor-memory lane
  const size_t bh = (size_t)b * c.H + h;
  const uint32_t msk = a.mask ? a.mask[bh] : kFull;

  uint8_t* A = smem + S::A_OFF;
  uint8_t* BQ = smem + S::BQ_OFF;
  uint8_t* BP = smem + S::BP_OFF;
  uint8_t* raw0 = smem + S::RAW_OFF;
  float* qsum = reinterpret_cast<float*>(smem + S::QSUM_OFF);  // [G][4]
  float* q0s = reinterpret_cast<float*>(smem + S::Q0_OFF);     // [G]
  float* redm = reinterpret_cast<float*>(smem + S::RED_OFF);   // [2][4][8]
  float* reds = redm + 2 * 4 * 8;                              // [2][4][8]
  const uint32_t bar_full0 = smem_addr(smem + S::BAR_OFF);
  const uint32_t bar_mma = bar_full0 + 16;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + S::SLOT_OFF);

  if (tid == 0) {
    mbar_init(bar_full0, 1);
    mbar_init(bar_full0 + 8, 1);
    mbar_init(bar_mma, 1);
    mbar_fence_init();
  }
  if (warp == 0) {
    tmem_alloc(smem_addr(tmem_slot), S::TMEM_COLS);
    tmem_relinquish();
  }

  // ---- query operand: rotated q as f16 hi/lo rows at the converted channel order
  for (int i = tid; i < S::NS * kHeadDim * 2 / 16; i += kTcThreads)
    reinterpret_cast<uint4*>(BQ)[i] = make_uint4(0, 0, 0, 0);  // padding rows stay zero
  __syncthreads();
  for (int hq = warp; hq < G; hq += kTcThreads / 32) {
    const In* qrow = static_cast<const In*>(a.q) + ((size_t)b * a.Hq + (size_t)h * G + hq) * kHeadDim;
    float x[4];
    load_row_warp(qrow, c.rotate != 0, a.inv_sqrt_d, lane, x);
    const bool sel = (msk >> lane) & 1u;
    float part = 0.0f;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int ch = 4 * lane + i;
      float v = sel ? x[i] : 0.0f;
      if (CH0 && ch == 0) v = 0.0f;  // channel 0 is scored from its bf16 copy
      part += v;
      const __half hi = __float2half_rn(v);
      const __half lo = __float2half_rn(v - __half2float(hi));
      const int blk = KB == 4 ? 8 : 16;
      const int p = (ch / blk) * blk + pos_of<KB>(ch % blk);
      *reinterpret_cast<__half*>(BQ + kmajor_off(hq, p)) = hi;
      *reinterpret_cast<__half*>(BQ + kmajor_off(G + hq, p)) = lo;
    }
#pragma unroll
    for (int m = 1; m < 8; m <<= 1) part += __shfl_xor_sync(kFull, part, m);
    if ((lane & 7) == 0) qsum[hq * kGroups + (lane >> 3)] = part;
    if (lane == 0) q0s[hq] = (CH0 && sel) ? x[0] : 0.0f;
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t t_score = tmem;               // 4 groups x NS columns
  const uint32_t t_pv = tmem + 4 * S::NS;      // NO columns

  if (tid == 0) {
    issue_tile_loads<G, KB, VB, CH0>(a, raw0, bar_full0, bh, start, msk);
    if (ntiles > 1) issue_tile_loads<G, KB, VB, CH0>(a, raw0 + S::RAW_BYTES, bar_full0 + 8, bh, start + kTile, msk);
  }

  const uint32_t idesc_s = idesc_f16_f32(kTile, S::NS, 0, 0);
  const uint32_t idesc_o = idesc_f16_f32(kTile, S::NO, 1, 1);
  const uint32_t a_addr = smem_addr(A), bq_addr = smem_addr(BQ), bp_addr = smem_addr(BP);
  const uint32_t lane_base = (uint32_t)(32 * (warp & 3)) << 16;  // this warp's tensor-memory lanes

  float m_run[HH], l_acc[HH], o[HH], zacc[kGroups][HH];
#pragma unroll
  for (int i = 0; i < HH; ++i) {
    m_run[i] = -__int_as_float(0x7f800000);
    l_acc[i] = 0.0f;
    o[i] = 0.0f;
#pragma unroll
    for (int g = 0; g < kGroups; ++g) zacc[g][i] = 0.0f;
  }
  bool ok = true;
  uint32_t mma_phase = 0;

  for (int t = 0; t < ntiles; ++t) {
    const int stage = t & 1;
    uint8_t* raw = raw0 + stage * S::RAW_BYTES;
    const int n0 = start + t * kTile;
    ok &= mbar_wait(bar_full0 + 8 * stage, (t >> 1) & 1);

    // ---- 2. key codes -> f16 tile A (K-major), this thread: token j, channel half
    if (KB == 4) {
#pragma unroll
      for (int qq = 0; qq < 8; ++qq) {
        const int q = half * 8 + qq;  // block of 8 channels = groups 2q, 2q+1
        const bool s0 = (msk >> (2 * q)) & 1u, s1 = (msk >> (2 * q + 1)) & 1u;
        uint4 v = make_uint4(0, 0, 0, 0);
        if (s0 || s1) {
          const uint32_t w0 = s0 ? reinterpret_cast<const uint16_t*>(raw + S::R_KC + (2 * q) * S::KROW)[j] : 0u;
          const uint32_t w1 = s1 ? reinterpret_cast<const uint16_t*>(raw + S::R_KC + (2 * q + 1) * S::KROW)[j] : 0u;
          uint32_t r[4];
          codes4_to_f16(w0 | (w1 << 16), r);
          v = make_uint4(r[0], r[1], r[2], r[3]);
        }
        *reinterpret_cast<uint4*>(A + kmajor_off(j, 8 * q)) = v;
      }
    } else {
#pragma unroll
      for (int qq = 0; qq < 4; ++qq) {
        const int q = half * 4 + qq;  // block of 16 channels = groups 4q .. 4q+3
        const uint32_t sel4 = (msk >> (4 * q)) & 0xFu;
        uint4 v0 = make_uint4(0, 0, 0, 0), v1 = v0;
        if (sel4) {
          uint32_t x = 0;
#pragma unroll
          for (int i = 0; i < 4; ++i)
            if ((sel4 >> i) & 1u) x |= (uint32_t)(raw + S::R_KC + (4 * q + i) * S::KROW)[j] << (8 * i);
          uint32_t r[8];
          codes2_to_f16(x, r);
          v0 = make_uint4(r[0], r[1], r[2], r[3]);
          v1 = make_uint4(r[4], r[5], r[6], r[7]);
        }
        *reinterpret_cast<uint4*>(A + kmajor_off(j, 16 * q)) = v0;
        *reinterpret_cast<uint4*>(A + kmajor_off(j, 16 * q + 8)) = v1;
      }
    }
    fence_proxy_async();
    __syncthreads();

    // ---- 3. score UMMAs (one thread)
    if (tid == 0) {
      tc_fence_after();
#pragma unroll
      for (int g = 0; g < kGroups; ++g)
#pragma unroll
        for (int s = 0; s < 2; ++s) {
          const int ks = 2 * g + s;  // 16-channel step
          umma_f16(t_score + g * S::NS, smem_desc(a_addr + ks * 256, 128, 2048),
                   smem_desc(bq_addr + ks * 256, 128, 2048), idesc_s, s);
        }
      umma_commit(bar_mma);
    }
    // per-token scalars while the tensor core works
    const bool valid = n0 + j < end;
    float2 ksz[kGroups], vsz[kGroups];
#pragma unroll
    for (int g = 0; g < kGroups; ++g)
      ksz[g] = __half22float2(reinterpret_cast<const __half2*>(raw + S::R_KS + g * kTile * 4)[j]);
    {
      const uint4 vv = reinterpret_cast<const uint4*>(raw + S::R_VS)[j];
      vsz[0] = __half22float2(*reinterpret_cast<const __half2*>(&vv.x));
      vsz[1] = __half22float2(*reinterpret_cast<const __half2*>(&vv.y));
      vsz[2] = __half22float2(*reinterpret_cast<const __half2*>(&vv.z));
      vsz[3] = __half22float2(*reinterpret_cast<const __half2*>(&vv.w));
    }
    float k0v = 0.0f;
    if (CH0 && (msk & 1u)) k0v = __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(raw + S::R_K0)[j]);

    ok &= mbar_wait(bar_mma, mma_phase);
    mma_phase ^= 1;
    tc_fence_after();

    // ---- 4. scores of this thread's token for its head half
    float sc[HH];
#pragma unroll
    for (int i = 0; i < HH; ++i) sc[i] = 0.0f;
#pragma unroll
    for (int g = 0; g < kGroups; ++g) {
      uint32_t hi[HH], lo[HH];
      tmem_ld<HH>(t_score + lane_base + g * S::NS + half * HH, hi);
      tmem_ld<HH>(t_score + lane_base + g * S::NS + G + half * HH, lo);
      tmem_wait_ld();
#pragma unroll
      for (int i = 0; i < HH; ++i) {
        const float dot = __uint_as_float(hi[i]) + __uint_as_float(lo[i]);
        sc[i] = fmaf(ksz[g].x, dot, fmaf(ksz[g].y, qsum[(half * HH + i) * kGroups + g], sc[i]));
      }
    }
#pragma unroll
    for (int i = 0; i < HH; ++i) {
      if (CH0) sc[i] = fmaf(q0s[half * HH + i], k0v, sc[i]);
      sc[i] = valid ? sc[i] * a.scale_log2 : -__int_as_float(0x7f800000);
      const float mx = warp_max(sc[i]);
      if (lane == 0) redm[(half * 4 + (warp & 3)) * 8 + i] = mx;
    }
    tc_fence_before();
    __syncthreads();

    float alpha[HH];
    uint32_t pk[kGroups][HH];  // f16 bits of P' per group (packed later)
#pragma unroll
    for (int i = 0; i < HH; ++i) {
      float tmax = redm[(half * 4) * 8 + i];
#pragma unroll
      for (int w = 1; w < 4; ++w) tmax = fmaxf(tmax, redm[(half * 4 + w) * 8 + i]);
      const float m_new = fmaxf(m_run[i], tmax);
      alpha[i] = exp2f(m_run[i] - m_new);
      m_run[i] = m_new;
      const float p = valid ? exp2f(sc[i] - m_new) : 0.0f;
      l_acc[i] = fmaf(l_acc[i], alpha[i], p);
#pragma unroll
      for (int g = 0; g < kGroups; ++g) {
        zacc[g][i] = fmaf(zacc[g][i], alpha[i], p * vsz[g].y);
        pk[g][i] = __half_as_ushort(__float2half_rn(valid ? p * vsz[g].x : 0.0f));
      }
    }
    // P' row of this token: columns g*G + half*HH + i (contiguous per group)
#pragma unroll
    for (int g = 0; g < kGroups; ++g) {
      const int n = g * G + half * HH;
      if (HH == 2) {
        *reinterpret_cast<uint32_t*>(BP + mnmajor_off(n, j)) = pk[g][0] | (pk[g][1] << 16);
      } else {
#pragma unroll
        for (int i = 0; i < HH; i += 4) {
          uint2 v = make_uint2(pk[g][i] | (pk[g][i + 1] << 16), pk[g][i + 2] | (pk[g][i + 3] << 16));
          *reinterpret_cast<uint2*>(BP + mnmajor_off(n + i, j)) = v;
        }
      }
    }

    // ---- 5. value codes -> f16 tile A (MN-major: channel position x token)
    if (VB == 4) {
#pragma unroll
      for (int it = 0; it < 2; ++it) {
        const int k = 2 * half + it;                  // 16-byte chunk of the 64-byte row
        const int kk = k ^ ((j >> 1) & 3);            // rotate chunks across tokens: conflict-free reads
        const uint4 w = *reinterpret_cast<const uint4*>(raw + S::R_VC + j * S::VROW + kk * 16);
        const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          uint32_t r[4];
          codes4_to_f16(ws[i], r);
          *reinterpret_cast<uint4*>(A + mnmajor_off(8 * (4 * kk + i), j)) = make_uint4(r[0], r[1], r[2], r[3]);
        }
      }
    } else {
      const int k = half;                             // 16-byte chunk of the 32-byte row
      const int kk = k ^ ((j >> 2) & 1);
      const uint4 w = *reinterpret_cast<const uint4*>(raw + S::R_VC + j * S::VROW + kk * 16);
      const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        uint32_t r[8];
        codes2_to_f16(ws[i], r);
        const int p = 64 * kk + 16 * i;
        *reinterpret_cast<uint4*>(A + mnmajor_off(p, j)) = make_uint4(r[0], r[1], r[2], r[3]);
        *reinterpret_cast<uint4*>(A + mnmajor_off(p + 8, j)) = make_uint4(r[4], r[5], r[6], r[7]);
      }
    }
    fence_proxy_async();
    __syncthreads();

    // ---- PV UMMAs, and the raw stage is free for tile t + 2
    if (tid == 0) {
      tc_fence_after();
#pragma unroll
      for (int s = 0; s < kTile / 16; ++s)
        umma_f16(t_pv, smem_desc(a_addr + s * 256, 128, 2048), smem_desc(bp_addr + s * 256, 128, 2048), idesc_o,
                 s > 0 ? 1u : 0u);
      umma_commit(bar_mma);
      if (t + 2 < ntiles) issue_tile_loads<G, KB, VB, CH0>(a, raw, bar_full0 + 8 * stage, bh, n0 + 2 * kTile, msk);
    }
    ok &= mbar_wait(bar_mma, mma_phase);
    mma_phase ^= 1;
    tc_fence_after();

    // ---- 6. this thread's channel (lane) and group, its head half
    {
      uint32_t d[HH];
      tmem_ld<HH>(t_pv + lane_base + (warp & 3) * G + half * HH, d);
      tmem_wait_ld();
#pragma unroll
      for (int i = 0; i < HH; ++i) o[i] = fmaf(o[i], alpha[i], __uint_as_float(d[i]));
    }
    tc_fence_before();
  }

  // ---- reduce the per-token sums over the CTA's 128 tokens (per head half)
  __syncthreads();
#pragma unroll
  for (int i = 0; i < HH; ++i) {
    const float s = warp_sum(l_acc[i]);
    if (lane == 0) reds[(half * 4 + (warp & 3)) * 8 + i] = s;
  }
  __syncthreads();
  float lsum[HH];
#pragma unroll
  for (int i = 0; i < HH; ++i) {
    lsum[i] = 0.0f;
#pragma unroll
    for (int w = 0; w < 4; ++w) lsum[i] += reds[(half * 4 + w) * 8 + i];
  }
  // zero-point term of this thread's channel group: sum over tokens of p * zero_g
  const int g_own = warp & 3;
  float zsum[HH];
#pragma unroll
  for (int g = 0; g < kGroups; ++g) {
    __syncthreads();
#pragma unroll
    for (int i = 0; i < HH; ++i) {
      const float s = warp_sum(zacc[g][i]);
      if (lane == 0) redm[(half * 4 + (warp & 3)) * 8 + i] = s;
    }
    __syncthreads();
    if (g == g_own) {
#pragma unroll
      for (int i = 0; i < HH; ++i) {
        zsum[i] = 0.0f;
#pragma unroll
        for (int w = 0; w < 4; ++w) zsum[i] += redm[(half * 4 + w) * 8 + i];
      }
    }
  }

  // ---- partials: acc[channel] per head, (max, sum) per head
  const int ch = chan_of<VB>(j);
#pragma unroll
  for (int i = 0; i < HH; ++i) {
    const int hq = h * G + half * HH + i;
    const size_t pidx = ((size_t)b * a.Hq + hq) * a.max_splits + split;
    const float nan = __int_as_float(0x7fc00000);
    a.part_acc[pidx * kHeadDim + ch] = ok ? o[i] + zsum[i] : nan;
    if (j == 0) a.part_ml[pidx] = ok ? make_float2(m_run[i], lsum[i]) : make_float2(nan, nan);
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, S::TMEM_COLS);
  }
}

template <int G, int KB, int VB, bool CH0, typename In>
cudaError_t launch_tc_typed(const DecodeArgs& a, cudaStream_t s) {
  using S = TcShape<G, KB, VB, CH0>;
  static_assert(S::SMEM_BYTES <= 110 * 1024, "two CTAs per SM");
  auto kern = k_decode_split_tc<G, KB, VB, CH0, In>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, S::SMEM_BYTES);
  if (e != cudaSuccess) return e;
  dim3 grid(a.max_splits, a.c.H, a.c.B), block(kTcThreads);
  kern<<<grid, block, S::SMEM_BYTES, s>>>(a);
  return cudaGetLastError();
}

template <int G, int KB, int VB, bool CH0>
cudaError_t launch_tc_dtype(const DecodeArgs& a, cudaStream_t s) {
  switch (a.dtype) {
    case KVQ_F32: return launch_tc_typed<G, KB, VB, CH0, float>(a, s);
    case KVQ_BF16: return launch_tc_typed<G, KB, VB, CH0, __nv_bfloat16>(a, s);
    default: return launch_tc_typed<G, KB, VB, CH0, __half>(a, s);
  }
}

template <int KB, int VB, bool CH0>
cudaError_t launch_tc_g(const DecodeArgs& a, cudaStream_t s) {
  switch (a.Hq / a.c.H) {
    case 4: return launch_tc_dtype<4, KB, VB, CH0>(a, s);
    case 8: return launch_tc_dtype<8, KB, VB, CH0>(a, s);
    case 16: return launch_tc_dtype<16, KB, VB, CH0>(a, s);
    default: return cudaErrorInvalidValue;
  }
}

template <int KB, int VB>
cudaError_t launch_tc_bits(const DecodeArgs& a, cudaStream_t s) {
  return a.c.keep_ch0 ? launch_tc_g<KB, VB, true>(a, s) : launch_tc_g<KB, VB, false>(a, s);
}

}  // namespace

bool decode_tc_supported(int g) { return g == 4 || g == 8 || g == 16; }

cudaError_t launch_decode_split_tc(const DecodeArgs& a, cudaStream_t s) {
  if (a.c.k_bits == 4 && a.c.v_bits == 4) return launch_tc_bits<4, 4>(a, s);
  if (a.c.k_bits == 4) return launch_tc_bits<4, 2>(a, s);
  if (a.c.v_bits == 4) return launch_tc_bits<2, 4>(a, s);
  return launch_tc_bits<2, 2>(a, s);
}

}  // namespace kvq

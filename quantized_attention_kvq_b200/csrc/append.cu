// Fused rotate + quantize + pack + append kernel.
//
// One CTA handles the new tokens of one (sequence, kv head) that fall in one
// 64-token-aligned window of the cache; each of its 8 warps takes every 8th
// token, one 128-channel row at a time with lane l owning channels 4l..4l+3
// (= pruning group l).  Keys: fp64 Walsh-Hadamard butterflies (Dual-QK
// summary Sec. 1; gist.science KQV scheme), optional bf16 channel 0 (Dual-QK
// Sec. 3.3, App. C.3), per-32-channel asymmetric quantization (Dual-QK
// Sec. 3.3).  Values: the same quantizer without rotation (Dual-QK App. B.2).
// Both code kinds are staged in shared memory and leave channel-major: key
// words one coalesced row per pruning group, value codes packed into each
// channel's row of the 128-token block.  Only tokens [offset, offset+n_new)
// change (tq-kv incremental cache); value-code words that also hold tokens
// outside that range are read, patched and written back by the one CTA whose
// window contains them.
#include "common.cuh"

namespace kvq {
namespace {

constexpr int kAppendTile = 64;  // tokens per CTA window, aligned to absolute token positions
constexpr int kAppendWarps = 8;

// Quantize the 4 channels this lane holds; the 8 lanes of a group agree on
// (scale, zero).  skip0: channel 0 of this lane is kept out of the range and
// gets code 0.  Returns the lane's packed word (4 codes of BITS bits).
template <int BITS>
__device__ __forceinline__ uint32_t quantize_lane(const float x[4], bool skip0, __half2& sz) {
  float mn = __int_as_float(0x7f800000), mx = -__int_as_float(0x7f800000);
#pragma unroll
  for (int i = 0; i < 4; ++i)
    if (!(skip0 && i == 0)) {
      mn = fminf(mn, x[i]);
      mx = fmaxf(mx, x[i]);
    }
#pragma unroll
  for (int m = 1; m < 8; m <<= 1) {
    mn = fminf(mn, __shfl_xor_sync(kFull, mn, m));
    mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, m));
  }
  // -0 and +0 are the same extreme; take it as +0 so the stored bits are unique
  mn = __fadd_rn(mn, 0.0f);
  mx = __fadd_rn(mx, 0.0f);
  constexpr int L = (1 << BITS) - 1;
  float s32 = fminf(__fdiv_rn(__fsub_rn(mx, mn), (float)L), 65504.0f);
  float zc = fminf(fmaxf(mn, -65504.0f), 65504.0f);
  const __half s16 = __float2half_rn(s32), z16 = __float2half_rn(zc);
  sz = __halves2half2(s16, z16);
  const float sf = __half2float(s16), zf = __half2float(z16);
  uint32_t word = 0;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    int code = 0;
    if (!(skip0 && i == 0) && sf != 0.0f) {
      code = __float2int_rn(__fdiv_rn(__fsub_rn(x[i], zf), sf));  // IEEE fp32, ties to even
      code = min(max(code, 0), L);
    }
    word |= (uint32_t)code << (BITS * i);
  }
  return word;
}

template <int KB, int VB, bool ROT, bool CH0, typename In>
__global__ void __launch_bounds__(kAppendWarps * 32) k_quantize_append(AppendArgs a) {
  constexpr int TPW = 32 / VB;                  // value tokens per 32-bit word: 8 (INT4) or 16 (INT2)
  constexpr int WPR = kAppendTile / TPW;        // value words per channel in the window: 8 or 4
  __shared__ uint16_t kw[kPruneGroups][kAppendTile + 2];
  __shared__ __half2 ksz[kGroups][kAppendTile];
  __shared__ __nv_bfloat16 k0s[kAppendTile];
  __shared__ __align__(16) uint8_t vcode[kAppendTile][kHeadDim];  // [token][channel] value codes
  __shared__ uint32_t vword[kHeadDim][WPR + 1];                   // packed value words, padded rows

  const CacheView& c = a.c;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int h = blockIdx.y, b = blockIdx.z;
  const int w0 = (a.offset / kAppendTile + blockIdx.x) * kAppendTile;  // absolute first token of the window
  const int lo = max(a.offset - w0, 0);                                // window tokens [lo, hi) are new
  const int hi = min(a.offset + a.n_new - w0, kAppendTile);
  const size_t bh = (size_t)b * c.H + h;
  // input row of window token tt: (bh * n_new + w0 + tt - offset), never negative for tt >= lo
  const size_t row0 = bh * a.n_new + (w0 + lo - a.offset);
  const In* kin = static_cast<const In*>(a.k_new) + (row0 - lo) * kHeadDim;
  const In* vin = static_cast<const In*>(a.v_new) + (row0 - lo) * kHeadDim;

  // one-deep prefetch of the next row pair
  float kx[4], vx[4], kn[4], vn[4];
  int tt = lo + warp;
  if (tt < hi) {
    load4(kin + (size_t)tt * kHeadDim + 4 * lane, kn);
    load4(vin + (size_t)tt * kHeadDim + 4 * lane, vn);
  }
  for (; tt < hi; tt += kAppendWarps) {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      kx[i] = kn[i];
      vx[i] = vn[i];
    }
    const int nx = tt + kAppendWarps;
    if (nx < hi) {
      load4(kin + (size_t)nx * kHeadDim + 4 * lane, kn);
      load4(vin + (size_t)nx * kHeadDim + 4 * lane, vn);
    }
    const size_t n = (size_t)w0 + tt;

    // ---- key row
    if (ROT) rotate_row_warp(kx, a.inv_sqrt_d, lane);
    if (CH0 && lane == 0) k0s[tt] = __float2bfloat16_rn(kx[0]);
    __half2 sz;
    const uint32_t kword = quantize_lane<KB>(kx, CH0 && lane == 0, sz);
    kw[lane][tt] = (uint16_t)kword;
    if ((lane & 7) == 0) ksz[lane >> 3][tt] = sz;

    // ---- value row: codes of channels 4l..4l+3 as bytes; scales token-major, written directly
    const uint32_t vw = quantize_lane<VB>(vx, false, sz);
    constexpr uint32_t L = (1u << VB) - 1;
    *reinterpret_cast<uint32_t*>(&vcode[tt][4 * lane]) =
        (vw & L) | (((vw >> VB) & L) << 8) | (((vw >> (2 * VB)) & L) << 16) | (((vw >> (3 * VB)) & L) << 24);
    if ((lane & 7) == 0) c.vs[(bh * c.cap + n) * kGroups + (lane >> 3)] = sz;
  }
  __syncthreads();

  // ---- key rows out: channel-major, one coalesced run per pruning group
  const int ntok = hi - lo;
  for (int i = threadIdx.x; i < kPruneGroups * ntok; i += blockDim.x) {
    const int pg = i / ntok, t = lo + i % ntok;
    const size_t idx = key_word_index(bh, c.cap, pg, w0 + t);
    if (KB == 4)
      reinterpret_cast<uint16_t*>(c.kc)[idx] = kw[pg][t];
    else
      c.kc[idx] = (uint8_t)kw[pg][t];
  }
  for (int i = threadIdx.x; i < kGroups * ntok; i += blockDim.x) {
    const int g = i / ntok, t = lo + i % ntok;
    c.ks[key_scale_index(bh, c.cap, g, w0 + t)] = ksz[g][t];
  }
  if (CH0)
    for (int t = lo + threadIdx.x; t < hi; t += blockDim.x) c.k0[bh * c.cap + w0 + t] = k0s[t];

  // ---- value codes: pack each channel's window into words (token order, low bits first)
  for (int i = threadIdx.x; i < kHeadDim * WPR; i += blockDim.x) {
    const int ch = i % kHeadDim, w = i / kHeadDim;  // a warp: 32 channels of one word position
    uint32_t word = 0;
#pragma unroll
    for (int k = 0; k < TPW; ++k) {
      const int t = w * TPW + k;
      const uint32_t code = (t >= lo && t < hi) ? vcode[t][ch] : 0u;
      word |= code << (VB * k);
    }
    vword[ch][w] = word;
  }
  __syncthreads();
  // ...and store them into the channel rows of the 128-token block
  const int blk = w0 / kKeyBlock;
  const int tb0 = w0 % kKeyBlock;               // window start inside the block: 0 or 64
  constexpr int TPC = 16 * 8 / VB;              // tokens per 16-byte chunk: 32 or 64
  for (int i = threadIdx.x; i < kHeadDim * WPR; i += blockDim.x) {
    const int ch = i / WPR, w = i % WPR;        // a warp: 32 / WPR channels, all their words
    const int t0 = w * TPW;                     // first window token of the word
    const int tb = tb0 + t0;                    // ... inside the block
    const int chunk = (tb / TPC) ^ v_chunk_swizzle(VB, ch);
    uint32_t* dst = reinterpret_cast<uint32_t*>(c.vc + v_row_offset(bh, c.cap, blk, ch, VB) + chunk * 16 +
                                                (tb % TPC) / (8 / VB));
    const int a0 = max(lo - t0, 0), a1 = min(hi - t0, TPW);  // new tokens of this word: [a0, a1)
    if (a0 >= a1) continue;
    uint32_t word = vword[ch][w];
    if (a0 > 0 || a1 < TPW) {
      const uint32_t keep_lo = a0 * VB >= 32 ? ~0u : ((1u << (a0 * VB)) - 1u);
      const uint32_t keep_hi = a1 * VB >= 32 ? 0u : ~((1u << (a1 * VB)) - 1u);
      word |= *dst & (keep_lo | keep_hi);  // the other tokens' codes stay as they were
    }
    *dst = word;
  }
}

template <int KB, int VB, bool ROT, bool CH0>
cudaError_t launch_typed(const AppendArgs& a, cudaStream_t s) {
  const int first = a.offset / kAppendTile, last = (a.offset + a.n_new - 1) / kAppendTile;
  dim3 grid(last - first + 1, a.c.H, a.c.B);
  dim3 block(kAppendWarps * 32);
  switch (a.dtype) {
    case KVQ_F32: k_quantize_append<KB, VB, ROT, CH0, float><<<grid, block, 0, s>>>(a); break;
    case KVQ_BF16: k_quantize_append<KB, VB, ROT, CH0, __nv_bfloat16><<<grid, block, 0, s>>>(a); break;
    default: k_quantize_append<KB, VB, ROT, CH0, __half><<<grid, block, 0, s>>>(a); break;
  }
  return cudaGetLastError();
}

template <int KB, int VB>
cudaError_t launch_bits(const AppendArgs& a, cudaStream_t s) {
  const bool rot = a.c.rotate != 0, ch0 = a.c.keep_ch0 != 0;
  if (rot && ch0) return launch_typed<KB, VB, true, true>(a, s);
  if (rot) return launch_typed<KB, VB, true, false>(a, s);
  if (ch0) return launch_typed<KB, VB, false, true>(a, s);
  return launch_typed<KB, VB, false, false>(a, s);
}

}  // namespace

cudaError_t launch_append(const AppendArgs& a, cudaStream_t s) {
  if (a.c.k_bits == 4 && a.c.v_bits == 4) return launch_bits<4, 4>(a, s);
  if (a.c.k_bits == 4) return launch_bits<4, 2>(a, s);
  if (a.c.v_bits == 4) return launch_bits<2, 4>(a, s);
  return launch_bits<2, 2>(a, s);
}

}  // namespace kvq

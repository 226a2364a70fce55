// Fused rotate + quantize + pack + append kernel.
//
// One CTA handles a tile of 64 new tokens of one (sequence, kv head); each of
// its 8 warps takes every 8th token, one 128-channel row at a time with lane
// l owning channels 4l..4l+3 (= pruning group l).  Keys: fp64 Walsh-Hadamard
// butterflies (Dual-QK summary Sec. 1; gist.science KQV scheme), optional
// bf16 channel 0 (Dual-QK Sec. 3.3, App. C.3), per-32-channel asymmetric
// quantization (Dual-QK Sec. 3.3).  Values: the same quantizer without
// rotation (Dual-QK App. B.2).  Key code words are staged in shared memory and
// written channel-major so every row store is coalesced; value rows and their
// scales go straight out token-major.  Only tokens [offset, offset+n_new) are
// touched (tq-kv incremental cache).
#include "common.cuh"

namespace kvq {
namespace {

constexpr int kAppendTile = 64;
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
  __shared__ uint16_t kw[kPruneGroups][kAppendTile + 2];
  __shared__ __half2 ksz[kGroups][kAppendTile];
  __shared__ __nv_bfloat16 k0s[kAppendTile];

  const CacheView& c = a.c;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int h = blockIdx.y, b = blockIdx.z;
  const int t0 = blockIdx.x * kAppendTile;
  const int ntok = min(kAppendTile, a.n_new - t0);
  const size_t bh = (size_t)b * c.H + h;
  const In* kin = static_cast<const In*>(a.k_new) + (bh * a.n_new + t0) * kHeadDim;
  const In* vin = static_cast<const In*>(a.v_new) + (bh * a.n_new + t0) * kHeadDim;

  // one-deep prefetch of the next row pair
  float kx[4], vx[4], kn[4], vn[4];
  int tt = warp;
  if (tt < ntok) {
    load4(kin + (size_t)tt * kHeadDim + 4 * lane, kn);
    load4(vin + (size_t)tt * kHeadDim + 4 * lane, vn);
  }
  for (; tt < ntok; tt += kAppendWarps) {
#pragma unroll
    for (int i = 0; i < 4; ++i) { kx[i] = kn[i]; vx[i] = vn[i]; }
    const int nx = tt + kAppendWarps;
    if (nx < ntok) {
      load4(kin + (size_t)nx * kHeadDim + 4 * lane, kn);
      load4(vin + (size_t)nx * kHeadDim + 4 * lane, vn);
    }
    const size_t n = (size_t)a.offset + t0 + tt;

    // ---- key row
    if (ROT) rotate_row_warp(kx, a.inv_sqrt_d, lane);
    if (CH0 && lane == 0) k0s[tt] = __float2bfloat16_rn(kx[0]);
    __half2 sz;
    const uint32_t kword = quantize_lane<KB>(kx, CH0 && lane == 0, sz);
    kw[lane][tt] = (uint16_t)kword;
    if ((lane & 7) == 0) ksz[lane >> 3][tt] = sz;

    // ---- value row: token-major, written directly (coalesced 32/64 bytes)
    const uint32_t vword = quantize_lane<VB>(vx, false, sz);
    uint8_t* vrow = c.vc + (bh * c.cap + n) * (kHeadDim * VB / 8);
    if (VB == 4)
      reinterpret_cast<uint16_t*>(vrow)[lane] = (uint16_t)vword;
    else
      vrow[lane] = (uint8_t)vword;
    if ((lane & 7) == 0) c.vs[(bh * c.cap + n) * kGroups + (lane >> 3)] = sz;
  }
  __syncthreads();

  // ---- key rows out: channel-major, one coalesced run per pruning group
  const size_t n0 = (size_t)a.offset + t0;
  for (int i = threadIdx.x; i < kPruneGroups * ntok; i += blockDim.x) {
    const int pg = i / ntok, t = i - pg * ntok;
    const size_t idx = key_word_index(bh, c.cap, pg, (int)n0 + t);
    if (KB == 4)
      reinterpret_cast<uint16_t*>(c.kc)[idx] = kw[pg][t];
    else
      c.kc[idx] = (uint8_t)kw[pg][t];
  }
  for (int i = threadIdx.x; i < kGroups * ntok; i += blockDim.x) {
    const int g = i / ntok, t = i - g * ntok;
    c.ks[key_scale_index(bh, c.cap, g, (int)n0 + t)] = ksz[g][t];
  }
  if (CH0)
    for (int t = threadIdx.x; t < ntok; t += blockDim.x) c.k0[bh * c.cap + n0 + t] = k0s[t];
}

template <int KB, int VB, bool ROT, bool CH0>
cudaError_t launch_typed(const AppendArgs& a, cudaStream_t s) {
  dim3 grid((a.n_new + kAppendTile - 1) / kAppendTile, a.c.H, a.c.B);
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

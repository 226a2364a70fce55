// Bucket-relative RoPE decode (Dual-QK summary Sec. 3.4, App. C.4).  The cache
// is bucket-major, so bucket k of sequence b is sequence b * nb + k of a cache
// of batch B * nb and capacity w, and the split decode runs over that bucket
// batch unchanged.  Around it: k_bucket_q gives every bucket its own query
// (embedded at its offset from the bucket's anchor, then transformed like the
// keys' partner) and length; k_bucket_merge then folds the split decode's
// partials of all buckets of a sequence into one softmax.
#include "transform.cuh"

namespace kvq {
namespace {

constexpr int kBucketWarps = 4;
constexpr int kDecodeTile = 128;  // tokens per tile of the split decode

template <typename In>
__global__ void __launch_bounds__(kBucketWarps * 32)
    k_bucket_q(const In* __restrict__ q, int rotate, const float* __restrict__ tq, const float* __restrict__ fr,
               const int32_t* __restrict__ lens, int max_len, int rows, int Hq, int H, int w, int nb,
               double inv_sqrt_d, float* __restrict__ qb, int32_t* __restrict__ vlens) {
  const int lane = threadIdx.x & 31;
  const int r = blockIdx.x * kBucketWarps + (threadIdx.x >> 5);  // (b * nb + k) * Hq + query head
  if (r >= rows) return;  // whole warps leave together
  const int vb = r / Hq, hq = r - vb * Hq;
  const int b = vb / nb, k = vb - b * nb;
  const int L = min(max(lens[b], 0), max_len);
  if (hq == 0 && lane == 0) vlens[vb] = min(max(L - k * w, 0), w);
  float x[4];
  load4(q + ((size_t)b * Hq + hq) * kHeadDim + 4 * lane, x);
  rope_row_warp(x, lane, (long long)L - 1 - (long long)k * w, fr);
  if (rotate == 1) rotate_row_warp(x, inv_sqrt_d, lane);
  if (rotate == 2) transform_row_warp(x, tq + (size_t)(hq / (Hq / H)) * kPairElems, lane);
  reinterpret_cast<float4*>(qb + (size_t)r * kHeadDim)[lane] = make_float4(x[0], x[1], x[2], x[3]);
}

__device__ __forceinline__ int bucket_tiles(const DecodeArgs& v, int vb) {
  const int len = min(max(v.seq_lens[vb], 0), v.max_len);
  return (len + kDecodeTile - 1) / kDecodeTile;
}

// One CTA of 128 threads per (sequence, query head), thread = channel.  The
// split decode left, for bucket unit u = vb * H + h of n_t tiles starting at
// tile t_u of the flattened tile list, one partial per CTA c in
// [t_u / per, (t_u + n_t - 1) / per] (per = ceil(total tiles / ctas)) in slot
// (u + c) * ngrp + e for each of its ngrp epilogue groups e, row slot * G +
// the head's index in its group; an empty one has max -inf.  Maxima and sums
// are in the log2 domain of the decode.
__global__ void __launch_bounds__(kHeadDim) k_bucket_merge(DecodeArgs v, int nb, int ctas, int ngrp,
                                                           float* __restrict__ out) {
  const int row = blockIdx.x;  // b * Hq + query head
  const int b = row / v.Hq, hq = row - b * v.Hq;
  const int G = v.Hq / v.c.H;
  const int h = hq / G, hl = hq - h * G;
  const int chn = threadIdx.x;
  // tiles of the whole bucket batch and of the buckets before sequence b
  // (block-wide sums, each thread taking every 128th bucket sequence)
  const int2 tp = block_tile_prefix(v.c.B, b * nb, v.c.H, [&](int vb) { return bucket_tiles(v, vb); });
  const int total = tp.x, tb = tp.y;
  const int per = (total + ctas - 1) / ctas;
  const float NEG_INF = -__int_as_float(0x7f800000);
  float M = NEG_INF;
  {
    int t0 = tb;
    for (int k = 0; k < nb; ++k) {
      const int vb = b * nb + k, nt = bucket_tiles(v, vb);
      if (nt > 0) {
        const int u = vb * v.c.H + h, tu = t0 + h * nt;
        for (int sl = (u + tu / per) * ngrp; sl < (u + (tu + nt - 1) / per + 1) * ngrp; ++sl)
          M = fmaxf(M, v.part_ml[(size_t)sl * G + hl].x);
      }
      t0 += v.c.H * nt;
    }
  }
  float l = 0.0f, o = 0.0f;
  {
    int t0 = tb;
    for (int k = 0; k < nb; ++k) {
      const int vb = b * nb + k, nt = bucket_tiles(v, vb);
      if (nt > 0) {
        const int u = vb * v.c.H + h, tu = t0 + h * nt;
        for (int sl = (u + tu / per) * ngrp; sl < (u + (tu + nt - 1) / per + 1) * ngrp; ++sl) {
          const size_t r = (size_t)sl * G + hl;
          const float2 ml = v.part_ml[r];
          if (ml.x == NEG_INF) continue;
          const float e = exp2f(ml.x - M);
          l = fmaf(e, ml.y, l);
          o = fmaf(e, v.part_acc[r * kHeadDim + chn], o);
        }
      }
      t0 += v.c.H * nt;
    }
  }
  float res = l > 0.0f ? o / l : 0.0f;
  if (v.c.rotate_v) {
    // back from the rotated value basis (the orthonormal Walsh-Hadamard
    // transform is its own inverse), fp32 butterflies over the 128 channels
    __shared__ float x[kHeadDim];
    x[chn] = res;
    for (int hs = 1; hs < kHeadDim; hs <<= 1) {
      __syncthreads();
      const float mine = x[chn], other = x[chn ^ hs];
      __syncthreads();
      x[chn] = (chn & hs) ? other - mine : mine + other;
    }
    __syncthreads();
    res = x[chn] * (float)v.inv_sqrt_d;
  }
  out[(size_t)row * kHeadDim + chn] = res;
}

}  // namespace

cudaError_t launch_bucket_queries(const void* q, int dtype, int rotate, const float* tq, const float* fr,
                                  const int32_t* lens, int max_len, int B, int Hq, int H, int w, int nb,
                                  double inv_sqrt_d, float* qb, int32_t* vlens, cudaStream_t s) {
  const int rows = B * nb * Hq;
  const dim3 grid((rows + kBucketWarps - 1) / kBucketWarps), block(kBucketWarps * 32);
  switch (dtype) {
    case KVQ_F32:
      k_bucket_q<float><<<grid, block, 0, s>>>(static_cast<const float*>(q), rotate, tq, fr, lens, max_len, rows, Hq,
                                               H, w, nb, inv_sqrt_d, qb, vlens);
      break;
    case KVQ_BF16:
      k_bucket_q<__nv_bfloat16><<<grid, block, 0, s>>>(static_cast<const __nv_bfloat16*>(q), rotate, tq, fr, lens,
                                                       max_len, rows, Hq, H, w, nb, inv_sqrt_d, qb, vlens);
      break;
    default:
      k_bucket_q<__half><<<grid, block, 0, s>>>(static_cast<const __half*>(q), rotate, tq, fr, lens, max_len, rows,
                                                Hq, H, w, nb, inv_sqrt_d, qb, vlens);
      break;
  }
  return cudaGetLastError();
}

cudaError_t launch_bucket_merge(const DecodeArgs& v, int nb, int ctas, int ngrp, float* out, cudaStream_t s) {
  k_bucket_merge<<<(v.c.B / nb) * v.Hq, kHeadDim, 0, s>>>(v, nb, ctas, ngrp, out);
  return cudaGetLastError();
}

}  // namespace kvq

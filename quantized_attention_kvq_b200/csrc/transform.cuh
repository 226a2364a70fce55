// Caller-supplied dual transform pair (Dual-QK summary Sec. 1, Sec. 3.1): per
// kv head an invertible 128 x 128 matrix T on queries and its inverse
// transpose on keys, fp32 row-major, so that (T q).(T^-T k) = q.k before
// quantization and pruning.  Transformed channel i is the fp64 sum over
// j = 0..127, in that order, of A[i][j] x[j] (product and sum each rounded
// once), rounded to fp32.
#pragma once

#include "common.cuh"

namespace kvq {

constexpr size_t kPairElems = (size_t)kHeadDim * kHeadDim;  // one matrix

// One 128-channel row spread over a warp, lane l holding channels 4l .. 4l+3
// (the layout load_row_warp gives), replaced by A x.  Lane l reads rows
// 4l .. 4l+3 of A as float4s; channel j's value comes from lane j / 4.
__device__ __forceinline__ void transform_row_warp(float x[4], const float* __restrict__ A, int lane) {
  const float4* rows = reinterpret_cast<const float4*>(A) + (size_t)lane * 4 * (kHeadDim / 4);
  double acc[4] = {0.0, 0.0, 0.0, 0.0};
#pragma unroll 4
  for (int s = 0; s < 32; ++s) {
    double xs[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) xs[k] = (double)__shfl_sync(kFull, x[k], s);
#pragma unroll
    for (int r = 0; r < 4; ++r) {
      const float4 m = __ldg(rows + r * (kHeadDim / 4) + s);  // A[4l + r][4s .. 4s+3]
      acc[r] = __dadd_rn(acc[r], __dmul_rn((double)m.x, xs[0]));
      acc[r] = __dadd_rn(acc[r], __dmul_rn((double)m.y, xs[1]));
      acc[r] = __dadd_rn(acc[r], __dmul_rn((double)m.z, xs[2]));
      acc[r] = __dadd_rn(acc[r], __dmul_rn((double)m.w, xs[3]));
    }
  }
#pragma unroll
  for (int r = 0; r < 4; ++r) x[r] = __double2float_rn(acc[r]);
}

// Rotary embedding of one row spread over a warp (lane l holding channels
// 4l .. 4l+3) at position pos (Dual-QK Sec. 3.4, bucket-relative RoPE):
// channel i < 64 pairs with i + 64, held by lane l ^ 16; angle pos * inv_freq[i
// mod 64] in fp64, x_i cos - x_{i+64} sin below, x_{i+64} cos + x_i sin above,
// each product and sum rounded once, then rounded to fp32.
__device__ __forceinline__ void rope_row_warp(float x[4], int lane, long long pos,
                                              const float* __restrict__ inv_freq) {
  const bool upper = lane >= 16;
  const int f0 = 4 * (lane & 15);
#pragma unroll
  for (int r = 0; r < 4; ++r) {
    const double other = (double)__shfl_xor_sync(kFull, x[r], 16);
    double sn, cs;
    sincos(__dmul_rn((double)pos, (double)__ldg(inv_freq + f0 + r)), &sn, &cs);
    const double own = __dmul_rn((double)x[r], cs), cross = __dmul_rn(other, sn);
    x[r] = __double2float_rn(upper ? __dadd_rn(own, cross) : __dsub_rn(own, cross));
  }
}

// Channel selection with the pair's query matrices tq [H][128][128] (used
// when a.rotate == 2; may be NULL otherwise).
cudaError_t launch_select_pair(const SelectArgs& a, const float* tq, cudaStream_t s);
// The same per bucket of a bucket-relative RoPE cache: grid row B * nb, the
// query embedded at offset (seq_lens[b] - 1) - k * w for bucket k, masks
// [B][nb][H].
cudaError_t launch_select_buckets(const SelectArgs& a, const float* tq, const float* inv_freq,
                                  const int32_t* seq_lens, int w, int nb, cudaStream_t s);
// Append with the pair's key matrices tk [H][128][128] (used when
// a.c.rotate == 2; may be NULL otherwise) and, when inv_freq is not NULL, the
// keys rotary-embedded at their token index in the view before the transform.
cudaError_t launch_append_ext(const AppendArgs& a, const float* tk, const float* inv_freq, cudaStream_t s);

// Bucket-relative RoPE decode (bucket.cu).  The cache is bucket-major: bucket
// k of sequence b is sequence b * nb + k of a cache of batch B * nb and
// capacity w.  k_bucket_q writes, per (b, k, query head), the query embedded
// at offset L_b - 1 - k * w (L_b = seq_lens[b] clamped to [0, max_len]) and
// taken through the cache's query transform, as fp32 rows qb[B * nb][Hq][128],
// and the bucket's length vlens[b * nb + k] = clamp(L_b - k * w, 0, w).
cudaError_t launch_bucket_queries(const void* q, int dtype, int rotate, const float* tq, const float* inv_freq,
                                  const int32_t* seq_lens, int max_len, int B, int Hq, int H, int w, int nb,
                                  double inv_sqrt_d, float* qb, int32_t* vlens, cudaStream_t s);
// One softmax over every bucket: merges the split decode's partials of the
// nb bucket units of each sequence (v: the decode's arguments over the
// bucket batch) into out [B][Hq][128], rotated back when v.c.rotate_v.
cudaError_t launch_bucket_merge(const DecodeArgs& v, int nb, int ctas, int ngrp, float* out, cudaStream_t s);
// out[b][j] = tq[j / G] q[b][j] as fp32 rows, G = Hq / H, for the decode.
cudaError_t launch_transform_q(const void* q, int dtype, const float* tq, int B, int Hq, int H, float* out,
                               cudaStream_t s);

}  // namespace kvq

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

// Channel selection with the pair's query matrices tq [H][128][128] (used
// when a.rotate == 2; may be NULL otherwise).
cudaError_t launch_select_pair(const SelectArgs& a, const float* tq, cudaStream_t s);
// Append with the pair's key matrices tk [H][128][128] (used when
// a.c.rotate == 2; may be NULL otherwise).
cudaError_t launch_append_pair(const AppendArgs& a, const float* tk, cudaStream_t s);
// out[b][j] = tq[j / G] q[b][j] as fp32 rows, G = Hq / H, for the decode.
cudaError_t launch_transform_q(const void* q, int dtype, const float* tq, int B, int Hq, int H, float* out,
                               cudaStream_t s);

}  // namespace kvq

// Combine pass: merges the per-split (max, sum, acc) partials of one
// (sequence, query head) into a single softmax over the whole sequence
// (Dual-QK summary Sec. 3.4: segments scored differently still share one
// global softmax).  o = sum_s 2^(m_s - M) acc_s / sum_s 2^(m_s - M) l_s.
#include "common.cuh"

namespace kvq {
namespace {

__global__ void __launch_bounds__(kHeadDim) k_combine(DecodeArgs a) {
  const int row = blockIdx.x;  // b * Hq + query head
  const int b = row / a.Hq;
  const int ch = threadIdx.x;
  const int len = min(max(a.seq_lens[b], 0), a.max_len);
  const int nsplit = (len + a.split_tokens - 1) / a.split_tokens;
  const float2* ml = a.part_ml + (size_t)row * a.max_splits;
  const float* acc = a.part_acc + (size_t)row * a.max_splits * kHeadDim;
  float M = -__int_as_float(0x7f800000);
  for (int s = 0; s < nsplit; ++s) M = fmaxf(M, ml[s].x);
  float l = 0.0f, o = 0.0f;
  for (int s = 0; s < nsplit; ++s) {
    const float2 v = ml[s];
    const float w = exp2f(v.x - M);
    l = fmaf(w, v.y, l);
    o = fmaf(w, acc[(size_t)s * kHeadDim + ch], o);
  }
  a.out[(size_t)row * kHeadDim + ch] = nsplit > 0 ? o / l : 0.0f;
}

}  // namespace

cudaError_t launch_combine(const DecodeArgs& a, cudaStream_t s) {
  k_combine<<<a.c.B * a.Hq, kHeadDim, 0, s>>>(a);
  return cudaGetLastError();
}

}  // namespace kvq

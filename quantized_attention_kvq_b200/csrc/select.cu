// Query-channel selection (Dual-QK summary Sec. 3.2, App. C.2): one CTA per
// (sequence, kv head).  Its warps rotate the GQA group's query rows (or take
// them through the kv head's matrix of the caller's transform pair, after a
// rotary embedding at the query's offset from a bucket's anchor when the cache
// uses bucket-relative RoPE, one CTA per bucket then); warp 0
// then gives lane p the fp64 energy of channel group p (heads outer, channels
// inner, the order the mask is defined in), ranks the 32 energies across the
// warp (ties keep the lower group) and writes the kept-group bitmask.
#include "transform.cuh"

namespace kvq {
namespace {

constexpr int kSelectThreads = 128;
constexpr int kMaxG = 64;

template <typename In>
__global__ void __launch_bounds__(kSelectThreads) k_select(SelectArgs a, const float* __restrict__ tq,
                                                           const float* __restrict__ fr,
                                                           const int32_t* __restrict__ lens, int w, int nb) {
  __shared__ float4 qr[kMaxG][kPruneGroups];  // rotated query rows, 4 channels per entry
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // grid row b = sequence * nb + bucket (nb = 1 without bucket-relative RoPE)
  const int h = blockIdx.x, b = blockIdx.y;
  const int G = a.Hq / a.H;
  const int seq = b / nb;
  const In* q = static_cast<const In*>(a.q) + ((size_t)seq * a.Hq + (size_t)h * G) * kHeadDim;
  // the query's offset from this bucket's anchor
  const long long rel = fr ? (long long)max(lens[seq], 0) - 1 - (long long)(b - seq * nb) * w : 0;
  for (int j = warp; j < G; j += kSelectThreads / 32) {
    float x[4];
    load4(q + (size_t)j * kHeadDim + 4 * lane, x);
    if (fr) rope_row_warp(x, lane, rel, fr);
    if (a.rotate == 1) rotate_row_warp(x, a.inv_sqrt_d, lane);
    if (a.rotate == 2) transform_row_warp(x, tq + (size_t)h * kPairElems, lane);
    qr[j][lane] = make_float4(x[0], x[1], x[2], x[3]);
  }
  __syncthreads();
  if (warp != 0) return;
  double e = 0.0;
  for (int j = 0; j < G; ++j) {
    const float4 v = qr[j][lane];
    e = __dadd_rn(e, __dmul_rn((double)v.x, (double)v.x));
    e = __dadd_rn(e, __dmul_rn((double)v.y, (double)v.y));
    e = __dadd_rn(e, __dmul_rn((double)v.z, (double)v.z));
    e = __dadd_rn(e, __dmul_rn((double)v.w, (double)v.w));
  }
  int rank = 0;
#pragma unroll
  for (int o = 0; o < 32; ++o) {
    const double eo = __shfl_sync(kFull, e, o);
    rank += (eo > e || (eo == e && o < lane)) ? 1 : 0;
  }
  const uint32_t m = __ballot_sync(kFull, rank < a.keep);
  if (lane == 0) a.mask[(size_t)b * a.H + h] = m;
}

}  // namespace

cudaError_t launch_select_buckets(const SelectArgs& a, const float* tq, const float* fr, const int32_t* lens, int w,
                                  int nb, cudaStream_t s) {
  dim3 grid(a.H, a.B * nb), block(kSelectThreads);
  switch (a.dtype) {
    case KVQ_F32: k_select<float><<<grid, block, 0, s>>>(a, tq, fr, lens, w, nb); break;
    case KVQ_BF16: k_select<__nv_bfloat16><<<grid, block, 0, s>>>(a, tq, fr, lens, w, nb); break;
    default: k_select<__half><<<grid, block, 0, s>>>(a, tq, fr, lens, w, nb); break;
  }
  return cudaGetLastError();
}

cudaError_t launch_select_pair(const SelectArgs& a, const float* tq, cudaStream_t s) {
  return launch_select_buckets(a, tq, nullptr, nullptr, 0, 1, s);
}

cudaError_t launch_select(const SelectArgs& a, cudaStream_t s) { return launch_select_pair(a, nullptr, s); }

}  // namespace kvq

// Query side of the caller's dual transform pair for the decode: every query
// row is taken through its kv head's matrix T once, into fp32 rows that the
// split decode and the window pass then read as untransformed queries.  One
// warp per row.
#include "transform.cuh"

namespace kvq {
namespace {

constexpr int kTransformWarps = 4;

template <typename In>
__global__ void __launch_bounds__(kTransformWarps * 32) k_transform_q(const In* __restrict__ q,
                                                                      const float* __restrict__ tq, int rows, int Hq,
                                                                      int G, float* __restrict__ out) {
  const int lane = threadIdx.x & 31;
  const int r = blockIdx.x * kTransformWarps + (threadIdx.x >> 5);
  if (r >= rows) return;  // whole warps leave together
  const int h = (r % Hq) / G;
  float x[4];
  load_row_warp(q + (size_t)r * kHeadDim, false, 0.0, lane, x);
  transform_row_warp(x, tq + (size_t)h * kPairElems, lane);
  reinterpret_cast<float4*>(out + (size_t)r * kHeadDim)[lane] = make_float4(x[0], x[1], x[2], x[3]);
}

}  // namespace

cudaError_t launch_transform_q(const void* q, int dtype, const float* tq, int B, int Hq, int H, float* out,
                               cudaStream_t s) {
  const int rows = B * Hq, G = Hq / H;
  const dim3 grid((rows + kTransformWarps - 1) / kTransformWarps), block(kTransformWarps * 32);
  switch (dtype) {
    case KVQ_F32: k_transform_q<float><<<grid, block, 0, s>>>(static_cast<const float*>(q), tq, rows, Hq, G, out); break;
    case KVQ_BF16:
      k_transform_q<__nv_bfloat16><<<grid, block, 0, s>>>(static_cast<const __nv_bfloat16*>(q), tq, rows, Hq, G, out);
      break;
    default: k_transform_q<__half><<<grid, block, 0, s>>>(static_cast<const __half*>(q), tq, rows, Hq, G, out); break;
  }
  return cudaGetLastError();
}

}  // namespace kvq

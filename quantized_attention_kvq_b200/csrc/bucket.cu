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
constexpr int kMergeSlots = 1024;  // slots listed at once by the merge (a chunk of 128 buckets needs fewer)
constexpr int kMergeBatch = 16;   // slots whose loads the merge issues together

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
//
// The sequence's buckets are taken 128 at a time, thread k taking bucket k
// of the chunk: its tile count, then (block scan) its first tile, then its
// first and last slot and the max over them.  With the maximum of the whole
// sequence known, every thread walks the chunk's slot ranges from shared
// memory, so its loads do not wait on one another.
__global__ void __launch_bounds__(kHeadDim) k_bucket_merge(DecodeArgs v, int nb, int ctas, int ngrp,
                                                           float* __restrict__ out) {
  const int row = blockIdx.x;  // b * Hq + query head
  const int b = row / v.Hq, hq = row - b * v.Hq;
  const int G = v.Hq / v.c.H;
  const int h = hq / G, hl = hq - h * G;
  const int chn = threadIdx.x, lane = chn & 31, warp = chn >> 5;
  // tiles of the whole bucket batch and of the buckets before sequence b
  // (block-wide sums, each thread taking every 128th bucket sequence)
  const int2 tp = block_tile_prefix(v.c.B, b * nb, v.c.H, [&](int vb) { return bucket_tiles(v, vb); });
  const int total = tp.x;
  const int per = (total + ctas - 1) / ctas;
  const float NEG_INF = -__int_as_float(0x7f800000);
  __shared__ int s_first[kHeadDim], s_last[kHeadDim];  // slot range of each bucket of the chunk
  __shared__ int s_scan[4];
  __shared__ float s_max[4];

  // pass 1: the maximum over every slot of the sequence
  float M = NEG_INF;
  int t0 = tp.y;  // first tile of the chunk's first bucket sequence (its kv head 0 unit)
  for (int k0 = 0; k0 < nb; k0 += kHeadDim) {
    const int k = k0 + chn;
    const int vb = b * nb + k;
    const int nt = k < nb ? bucket_tiles(v, vb) : 0;
    // exclusive scan of H * nt over the chunk
    int x = v.c.H * nt;
#pragma unroll
    for (int m = 1; m < 32; m <<= 1) {
      const int y = __shfl_up_sync(kFull, x, m);
      if (lane >= m) x += y;
    }
    if (lane == 31) s_scan[warp] = x;
    __syncthreads();
    int before = 0;
    for (int w = 0; w < warp; ++w) before += s_scan[w];
    const int incl = x + before;
    const int chunk_sum = s_scan[0] + s_scan[1] + s_scan[2] + s_scan[3];
    const int tk = t0 + incl - v.c.H * nt;  // first tile of bucket sequence vb
    int f = 0, l = -1;
    float mk = NEG_INF;
    if (nt > 0) {
      const int u = vb * v.c.H + h, tu = tk + h * nt;
      f = (u + tu / per) * ngrp;
      l = (u + (tu + nt - 1) / per + 1) * ngrp - 1;
      for (int sl = f; sl <= l; ++sl) mk = fmaxf(mk, v.part_ml[(size_t)sl * G + hl].x);
    }
    s_first[chn] = f;
    s_last[chn] = l;
    mk = fmaxf(mk, __shfl_xor_sync(kFull, mk, 16));
    mk = fmaxf(mk, __shfl_xor_sync(kFull, mk, 8));
    mk = fmaxf(mk, __shfl_xor_sync(kFull, mk, 4));
    mk = fmaxf(mk, __shfl_xor_sync(kFull, mk, 2));
    mk = fmaxf(mk, __shfl_xor_sync(kFull, mk, 1));
    if (lane == 0) s_max[warp] = mk;
    __syncthreads();
    M = fmaxf(M, fmaxf(fmaxf(s_max[0], s_max[1]), fmaxf(s_max[2], s_max[3])));
    t0 += chunk_sum;
  }
  // the bf16 window tokens' partial of the unit, when the cache has windows
  const bool win = v.c.sink + v.c.recent > 0;
  const size_t rw = (size_t)(v.win_base + b * v.c.H + h) * G + hl;
  if (win) M = fmaxf(M, v.part_ml[rw].x);
  // pass 2: every slot's weight 2^(m - M), its sum and its channel.  A
  // chunk's slots are listed in shared memory first (at most 2 per CTA range
  // end per bucket plus one per `per` tiles, so under 1024), then walked
  // kMergeBatch at a time with their loads issued together.
  __shared__ int s_slot[kMergeSlots];
  float l = 0.0f, o = 0.0f;
  const int nchunks = (nb + kHeadDim - 1) / kHeadDim;
  t0 = tp.y;
  for (int c = 0; c < nchunks; ++c) {
    const int k = c * kHeadDim + chn;
    const int vb = b * nb + k;
    int f = 0, ll = -1;
    if (nchunks > 1) {
      // this chunk's slot ranges again (pass 1 kept only the last chunk's)
      const int nt = k < nb ? bucket_tiles(v, vb) : 0;
      int x = v.c.H * nt;
#pragma unroll
      for (int m = 1; m < 32; m <<= 1) {
        const int y = __shfl_up_sync(kFull, x, m);
        if (lane >= m) x += y;
      }
      __syncthreads();
      if (lane == 31) s_scan[warp] = x;
      __syncthreads();
      int before = 0;
      for (int w = 0; w < warp; ++w) before += s_scan[w];
      const int tk = t0 + x + before - v.c.H * nt;
      t0 += s_scan[0] + s_scan[1] + s_scan[2] + s_scan[3];
      if (nt > 0) {
        const int u = vb * v.c.H + h, tu = tk + h * nt;
        f = (u + tu / per) * ngrp;
        ll = (u + (tu + nt - 1) / per + 1) * ngrp - 1;
      }
    } else {
      f = s_first[chn];
      ll = s_last[chn];
    }
    // list the chunk's slots: exclusive scan of the per-bucket counts
    const int cnt = ll - f + 1;
    int x = cnt;
#pragma unroll
    for (int m = 1; m < 32; m <<= 1) {
      const int y = __shfl_up_sync(kFull, x, m);
      if (lane >= m) x += y;
    }
    __syncthreads();
    if (lane == 31) s_scan[warp] = x;
    __syncthreads();
    int base = x - cnt;
    for (int w = 0; w < warp; ++w) base += s_scan[w];
    const int n = min(s_scan[0] + s_scan[1] + s_scan[2] + s_scan[3], kMergeSlots);
    for (int i = 0; i < cnt && base + i < kMergeSlots; ++i) s_slot[base + i] = f + i;
    __syncthreads();
    for (int i0 = 0; i0 < n; i0 += kMergeBatch) {
      float2 ml[kMergeBatch];
      float ac[kMergeBatch];
#pragma unroll
      for (int j = 0; j < kMergeBatch; ++j) {
        const int i = min(i0 + j, n - 1);
        const size_t r = (size_t)s_slot[i] * G + hl;
        ml[j] = v.part_ml[r];
        ac[j] = v.part_acc[r * kHeadDim + chn];  // an empty slot's is not used
      }
#pragma unroll
      for (int j = 0; j < kMergeBatch; ++j) {
        const bool use = i0 + j < n && ml[j].x != NEG_INF;
        const float e = use ? exp2f(ml[j].x - M) : 0.0f;
        l = fmaf(e, use ? ml[j].y : 0.0f, l);
        o = use ? fmaf(e, ac[j], o) : o;
      }
    }
    __syncthreads();
  }
  if (win) {
    const float2 ml = v.part_ml[rw];
    if (ml.x != NEG_INF) {
      const float e = exp2f(ml.x - M);
      l = fmaf(e, ml.y, l);
      o = fmaf(e, v.part_acc[rw * kHeadDim + chn], o);
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

// Attention over the bf16 token windows (the first sink tokens and the most
// recent ones of each sequence, kept as bf16 rows of the rotated key and the
// value): one partial per (sequence, kv head) for the combine pass.
#include "common.cuh"

namespace kvq {
namespace {

// Attention over the bf16 window tokens of one unit (sequence b, kv head h):
// tokens n < sink and the last `recent` tokens, scored over every channel from
// the bf16 rotated keys (Dual-QK Sec. 3.3; tq-kv sink tokens), one partial
// (max and sum in base-2 units, unnormalized values) per query head at slot
// win_base + unit for the combine.  kWinThreads threads: thread = window token
// for the scores and weights; for the value sums kWinParts groups of 128
// threads (thread = channel) take contiguous quarters of the window, so a
// thread's chain of row loads is a quarter as long, and add up at the end.
constexpr int kWinParts = 4;
constexpr int kWinThreads = kWinParts * kHeadDim;
constexpr int kWinWarps = kWinThreads / 32;

template <int G, typename In>
__global__ void __launch_bounds__(kWinThreads) k_window(DecodeArgs a) {
  // q [G][128], weights [G][sink + recent], reductions [G][kWinWarps], slots
  // [sink + recent], value partial sums [kWinParts - 1][G][128]
  extern __shared__ float wsm[];
  const CacheView& c = a.c;
  const int u = blockIdx.x, b = u / c.H, h = u - b * c.H;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int WS = c.sink + c.recent;
  const int len = min(max(a.seq_lens[b], 0), a.max_len);
  const int n_sink = min(c.sink, len);
  const int r0 = c.recent > 0 ? max(c.sink, len - c.recent) : len;  // first recent token
  const int W = n_sink + max(len - r0, 0);                            // window tokens
  // with bucket-relative RoPE the window tokens take the query of the bucket
  // they sit in: the sinks bucket 0's, the recent tokens one of at most two
  // buckets' (the recent window is at most a bucket long)
  const bool bk = a.bucket_nb > 0;
  const int NQ = bk ? 3 : 1;
  int kbq[3] = {0, 0, 0};
  if (bk && len > 0) {
    kbq[1] = r0 / a.bucket_w;
    kbq[2] = (len - 1) / a.bucket_w;
  }
  float* qs = wsm;
  float* pw = qs + NQ * G * kHeadDim;
  float* red = pw + G * WS;
  int* slot = reinterpret_cast<int*>(red + G * kWinWarps);  // window slot of window token w
  float* osum = reinterpret_cast<float*>(slot + WS);
  const size_t row0 = (size_t)u * WS;
  for (int w = tid; w < W; w += kWinThreads)
    slot[w] = window_slot(c.sink, c.recent, w < n_sink ? w : r0 + (w - n_sink));
  // the query rows, rotated as the keys are (with buckets: each bucket's rows
  // as the decode prepared them), one warp per head
  for (int sg = warp; sg < NQ * G; sg += kWinWarps) {
    const int sq = sg / G, g = sg - sq * G;
    const size_t qrow = bk ? ((size_t)b * a.bucket_nb + kbq[sq]) * a.Hq + (size_t)h * G + g
                           : (size_t)b * a.Hq + (size_t)h * G + g;
    float x[4];
    load_row_warp(static_cast<const In*>(a.q) + qrow * kHeadDim, c.rotate != 0, a.inv_sqrt_d, lane, x);
#pragma unroll
    for (int i = 0; i < 4; ++i) qs[sg * kHeadDim + 4 * lane + i] = x[i];
  }
  __syncthreads();
  // scores (base-2 units) of every window token, all channels
  float mloc[G];
#pragma unroll
  for (int g = 0; g < G; ++g) mloc[g] = -__int_as_float(0x7f800000);
  for (int w = tid; w < W; w += kWinThreads) {
    // the whole bf16 key row in flight at once (16 independent 16-byte loads)
    const uint4* kr = reinterpret_cast<const uint4*>(c.kwin + (row0 + slot[w]) * kHeadDim);
    uint4 raw[kHeadDim / 8];
#pragma unroll
    for (int i = 0; i < kHeadDim / 8; ++i) raw[i] = kr[i];
    float acc[G];
#pragma unroll
    for (int g = 0; g < G; ++g) acc[g] = 0.0f;
    int sq = 0;  // the token's query set
    if (bk) {
      const int n = w < n_sink ? w : r0 + (w - n_sink);
      sq = n < c.sink ? 0 : (n / a.bucket_w == kbq[1] ? 1 : 2);
    }
    const float* qw = qs + sq * G * kHeadDim;
#pragma unroll
    for (int i8 = 0; i8 < kHeadDim / 8; ++i8) {
      const uint32_t pr[4] = {raw[i8].x, raw[i8].y, raw[i8].z, raw[i8].w};
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int cc = 8 * i8 + 2 * i;
        const float k0 = __uint_as_float(pr[i] << 16), k1 = __uint_as_float(pr[i] & 0xFFFF0000u);
#pragma unroll
        for (int g = 0; g < G; ++g)
          acc[g] = fmaf(qw[g * kHeadDim + cc + 1], k1, fmaf(qw[g * kHeadDim + cc], k0, acc[g]));
      }
    }
#pragma unroll
    for (int g = 0; g < G; ++g) {
      const float sc = acc[g] * a.scale_log2;
      pw[g * WS + w] = sc;
      mloc[g] = fmaxf(mloc[g], sc);
    }
  }
  // per head: the max, then weights 2^(s - max) and their sum
#pragma unroll
  for (int g = 0; g < G; ++g) {
    const float mx = warp_max(mloc[g]);
    if (lane == 0) red[g * kWinWarps + warp] = mx;
  }
  __syncthreads();
  float m[G], lsum[G];
#pragma unroll
  for (int g = 0; g < G; ++g) {
    float mx = red[g * kWinWarps];
    for (int i = 1; i < kWinWarps; ++i) mx = fmaxf(mx, red[g * kWinWarps + i]);
    m[g] = mx;
    lsum[g] = 0.0f;
  }
  __syncthreads();
  for (int w = tid; w < W; w += kWinThreads)
#pragma unroll
    for (int g = 0; g < G; ++g) {
      const float p = exp2f(pw[g * WS + w] - m[g]);
      pw[g * WS + w] = p;
      lsum[g] += p;
    }
#pragma unroll
  for (int g = 0; g < G; ++g) {
    const float sm = warp_sum(lsum[g]);
    if (lane == 0) red[g * kWinWarps + warp] = sm;
  }
  __syncthreads();
  // value sums: group part takes window tokens [w_lo, w_hi), thread = channel;
  // sixteen tokens' loads in flight before their multiply-adds
  const int part = tid / kHeadDim, ch = tid % kHeadDim;
  const int w_lo = part * W / kWinParts, w_hi = (part + 1) * W / kWinParts;
  float o[G];
#pragma unroll
  for (int g = 0; g < G; ++g) o[g] = 0.0f;
  constexpr int kBatch = 16;
  const __nv_bfloat16* vb = c.vwin + row0 * kHeadDim + ch;
  int w = w_lo;
  for (; w + kBatch <= w_hi; w += kBatch) {
    float v[kBatch];
#pragma unroll
    for (int i = 0; i < kBatch; ++i) v[i] = __bfloat162float(vb[(size_t)slot[w + i] * kHeadDim]);
#pragma unroll
    for (int i = 0; i < kBatch; ++i)
#pragma unroll
      for (int g = 0; g < G; ++g) o[g] = fmaf(pw[g * WS + w + i], v[i], o[g]);
  }
  for (; w < w_hi; ++w) {
    const float v = __bfloat162float(vb[(size_t)slot[w] * kHeadDim]);
#pragma unroll
    for (int g = 0; g < G; ++g) o[g] = fmaf(pw[g * WS + w], v, o[g]);
  }
  if (part > 0)
#pragma unroll
    for (int g = 0; g < G; ++g) osum[((part - 1) * G + g) * kHeadDim + ch] = o[g];
  __syncthreads();
  if (part == 0) {
#pragma unroll
    for (int g = 0; g < G; ++g) {
      float t = o[g];
      for (int q = 1; q < kWinParts; ++q) t += osum[((q - 1) * G + g) * kHeadDim + ch];
      const size_t r = (size_t)(a.win_base + u) * G + g;
      if (!kvq_in_bounds(r, 1, a.part_rows)) continue;
      a.part_acc[r * kHeadDim + ch] = t;
      if (ch == 0) {
        float l = 0.0f;
        for (int i = 0; i < kWinWarps; ++i) l += red[g * kWinWarps + i];
        a.part_ml[r] = W > 0 ? make_float2(m[g], l) : make_float2(-__int_as_float(0x7f800000), 0.0f);
      }
    }
  }
}

template <int G>
cudaError_t launch_window_g(const DecodeArgs& a, cudaStream_t s) {
  const int ws = a.c.sink + a.c.recent;
  const int nq = a.bucket_nb > 0 ? 3 : 1;  // query sets (bucket-relative RoPE: up to three buckets)
  const size_t smem =
      (size_t)(nq * G * kHeadDim + G * ws + G * kWinWarps + ws + (kWinParts - 1) * G * kHeadDim) * sizeof(float);
  auto kern = a.dtype == KVQ_F32 ? k_window<G, float> : (a.dtype == KVQ_BF16 ? k_window<G, __nv_bfloat16> : k_window<G, __half>);
  if (smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
  }
  kern<<<a.c.B * a.c.H, kWinThreads, smem, s>>>(a);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_window(const DecodeArgs& a, cudaStream_t s) {
  switch (a.Hq / a.c.H) {
    case 1: return launch_window_g<1>(a, s);
    case 2: return launch_window_g<2>(a, s);
    case 4: return launch_window_g<4>(a, s);
    case 8: return launch_window_g<8>(a, s);
    case 16: return launch_window_g<16>(a, s);
    default: return cudaErrorInvalidValue;
  }
}


KVQ_BOUNDS_COUNTER(bounds_window)

}  // namespace kvq

// Split-sequence decode attention over the packed cache, CUDA-core version.
//
// Grid (split, kv head, sequence); 128 threads.  A CTA owns the G query heads
// of one kv head and one split of the sequence (a multiple of 128 tokens) and
// walks it in tiles of 128 tokens:
//   score:  thread t takes token t of the tile and scores it for all G heads
//           straight from the key code words of the kept pruning groups:
//           per quant group g, s_g * sum(q * code) + z_g * sum(q), plus
//           q[0] * k_ch0 when channel 0 is kept (Dual-QK summary Sec. 3.2,
//           3.3; tq-kv abstract: no dequantized key is written anywhere);
//   softmax: running max / sum per head in the exp2 domain;
//   PV:     thread t takes channel t and accumulates p * (s_v * code + z_v).
// It writes (max, sum, acc[128]) per head; the combine pass merges splits
// into one softmax (Dual-QK Sec. 3.4).
#include "common.cuh"

namespace kvq {
namespace {

constexpr int kThreads = kDecodeTile;  // one token (score) / one channel (PV) per thread

template <typename In>
__device__ __forceinline__ const In* q_ptr(const DecodeArgs& a) { return static_cast<const In*>(a.q); }

template <int G, int KB, int VB, bool CH0, typename In>
__global__ void __launch_bounds__(kThreads) k_decode_split_simt(DecodeArgs a) {
  const CacheView& c = a.c;
  const int split = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int len = min(max(a.seq_lens[b], 0), a.max_len);
  const int start = split * a.split_tokens;
  if (start >= len) return;
  const int end = min(start + a.split_tokens, len);

  __shared__ float4 qs[G][kPruneGroups];  // rotated query, 4 channels per entry
  __shared__ float qsum[G][kGroups];      // sum of kept, quantized query channels per group
  __shared__ float q0s[G];                // q[0] when channel 0 is kept and selected, else 0
  __shared__ float ps[G][kDecodeTile];    // tile probabilities
  __shared__ float redm[G][kThreads / 32];
  __shared__ float reds[G][kThreads / 32];

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const size_t bh = (size_t)b * c.H + h;
  const uint32_t msk = a.mask ? a.mask[bh] : kFull;

  // ---- query preparation (one warp per head)
  for (int j = warp; j < G; j += kThreads / 32) {
    const In* qrow = q_ptr<In>(a) + ((size_t)b * a.Hq + (size_t)h * G + j) * kHeadDim;
    float x[4];
    load_row_warp(qrow, c.rotate != 0, a.inv_sqrt_d, lane, x);
    qs[j][lane] = make_float4(x[0], x[1], x[2], x[3]);
    const bool sel = (msk >> lane) & 1u;
    float part = 0.0f;
    if (sel) part = (CH0 && lane == 0 ? 0.0f : x[0]) + x[1] + x[2] + x[3];
#pragma unroll
    for (int m = 1; m < 8; m <<= 1) part += __shfl_xor_sync(kFull, part, m);
    if ((lane & 7) == 0) qsum[j][lane >> 3] = part;
    if (lane == 0) q0s[j] = (CH0 && sel) ? x[0] : 0.0f;
  }
  __syncthreads();

  float m_run[G], l_run[G], o[G];
#pragma unroll
  for (int j = 0; j < G; ++j) {
    m_run[j] = -__int_as_float(0x7f800000);
    l_run[j] = 0.0f;
    o[j] = 0.0f;
  }
  constexpr uint32_t LK = (1u << KB) - 1, LV = (1u << VB) - 1;

  for (int tile = start; tile < end; tile += kDecodeTile) {
    const int n = tile + tid;
    const bool valid = n < end;
    float sc[G];
    if (valid) {
      float acc[kGroups][G];
#pragma unroll
      for (int g = 0; g < kGroups; ++g)
#pragma unroll
        for (int j = 0; j < G; ++j) acc[g][j] = 0.0f;
#pragma unroll
      for (int g = 0; g < kGroups; ++g) {
#pragma unroll
        for (int pp = 0; pp < 8; ++pp) {
          const int pg = g * 8 + pp;
          if (!((msk >> pg) & 1u)) continue;  // CTA-uniform
          const size_t idx = key_word_index(bh, c.cap, pg, n);
          const uint32_t w = KB == 4 ? (uint32_t)reinterpret_cast<const uint16_t*>(c.kc)[idx] : (uint32_t)c.kc[idx];
          const float c0 = (float)(w & LK), c1 = (float)((w >> KB) & LK);
          const float c2 = (float)((w >> (2 * KB)) & LK), c3 = (float)((w >> (3 * KB)) & LK);
#pragma unroll
          for (int j = 0; j < G; ++j) {
            const float4 qv = qs[j][pg];
            acc[g][j] = fmaf(c0, qv.x, fmaf(c1, qv.y, fmaf(c2, qv.z, fmaf(c3, qv.w, acc[g][j]))));
          }
        }
      }
#pragma unroll
      for (int j = 0; j < G; ++j) sc[j] = 0.0f;
#pragma unroll
      for (int g = 0; g < kGroups; ++g) {
        const float2 sz = __half22float2(c.ks[key_scale_index(bh, c.cap, g, n)]);
#pragma unroll
        for (int j = 0; j < G; ++j) sc[j] = fmaf(sz.x, acc[g][j], fmaf(sz.y, qsum[j][g], sc[j]));
      }
      if (CH0 && (msk & 1u)) {
        const float k0 = __bfloat162float(c.k0[bh * c.cap + n]);
#pragma unroll
        for (int j = 0; j < G; ++j) sc[j] = fmaf(q0s[j], k0, sc[j]);
      }
#pragma unroll
      for (int j = 0; j < G; ++j) sc[j] *= a.scale_log2;
    } else {
#pragma unroll
      for (int j = 0; j < G; ++j) sc[j] = -__int_as_float(0x7f800000);
    }

    // ---- tile max, probabilities, running sums
#pragma unroll
    for (int j = 0; j < G; ++j) {
      const float mx = warp_max(sc[j]);
      if (lane == 0) redm[j][warp] = mx;
    }
    __syncthreads();
    float alpha[G];
#pragma unroll
    for (int j = 0; j < G; ++j) {
      float tmax = redm[j][0];
#pragma unroll
      for (int w = 1; w < kThreads / 32; ++w) tmax = fmaxf(tmax, redm[j][w]);
      const float m_new = fmaxf(m_run[j], tmax);
      const float p = valid ? exp2f(sc[j] - m_new) : 0.0f;
      ps[j][tid] = p;
      alpha[j] = exp2f(m_run[j] - m_new);
      m_run[j] = m_new;
      const float s = warp_sum(p);
      if (lane == 0) reds[j][warp] = s;
    }
    __syncthreads();
#pragma unroll
    for (int j = 0; j < G; ++j) {
      float s = reds[j][0];
#pragma unroll
      for (int w = 1; w < kThreads / 32; ++w) s += reds[j][w];
      l_run[j] = fmaf(l_run[j], alpha[j], s);
      o[j] *= alpha[j];
    }

    // ---- PV: thread tid owns channel tid
    const int ch = tid, g = ch >> 5;
    const int nv = min(kDecodeTile, end - tile);
    constexpr int per_byte = 8 / VB;
    for (int jj = 0; jj < nv; ++jj) {
      const size_t tok = bh * c.cap + tile + jj;
      const uint32_t byte = c.vc[tok * (kHeadDim * VB / 8) + ch / per_byte];
      const float code = (float)((byte >> ((ch % per_byte) * VB)) & LV);
      const float2 sz = __half22float2(c.vs[tok * kGroups + g]);
      const float vhat = fmaf(sz.x, code, sz.y);
#pragma unroll
      for (int j = 0; j < G; ++j) o[j] = fmaf(ps[j][jj], vhat, o[j]);
    }
    __syncthreads();  // ps and red buffers are rewritten by the next tile
  }

  // ---- partials
#pragma unroll
  for (int j = 0; j < G; ++j) {
    const size_t pidx = ((size_t)b * a.Hq + (size_t)h * G + j) * a.max_splits + split;
    a.part_acc[pidx * kHeadDim + tid] = o[j];
    if (tid == 0) a.part_ml[pidx] = make_float2(m_run[j], l_run[j]);
  }
}

template <int G, int KB, int VB, bool CH0>
cudaError_t launch_g(const DecodeArgs& a, cudaStream_t s) {
  dim3 grid(a.max_splits, a.c.H, a.c.B), block(kThreads);
  switch (a.dtype) {
    case KVQ_F32: k_decode_split_simt<G, KB, VB, CH0, float><<<grid, block, 0, s>>>(a); break;
    case KVQ_BF16: k_decode_split_simt<G, KB, VB, CH0, __nv_bfloat16><<<grid, block, 0, s>>>(a); break;
    default: k_decode_split_simt<G, KB, VB, CH0, __half><<<grid, block, 0, s>>>(a); break;
  }
  return cudaGetLastError();
}

template <int KB, int VB, bool CH0>
cudaError_t launch_flags(const DecodeArgs& a, cudaStream_t s) {
  switch (a.Hq / a.c.H) {
    case 1: return launch_g<1, KB, VB, CH0>(a, s);
    case 2: return launch_g<2, KB, VB, CH0>(a, s);
    case 4: return launch_g<4, KB, VB, CH0>(a, s);
    case 8: return launch_g<8, KB, VB, CH0>(a, s);
    case 16: return launch_g<16, KB, VB, CH0>(a, s);
    default: return cudaErrorInvalidValue;
  }
}

template <int KB, int VB>
cudaError_t launch_bits(const DecodeArgs& a, cudaStream_t s) {
  return a.c.keep_ch0 ? launch_flags<KB, VB, true>(a, s) : launch_flags<KB, VB, false>(a, s);
}

}  // namespace

cudaError_t launch_decode_split(const DecodeArgs& a, cudaStream_t s) {
  if (a.c.k_bits == 4 && a.c.v_bits == 4) return launch_bits<4, 4>(a, s);
  if (a.c.k_bits == 4) return launch_bits<4, 2>(a, s);
  if (a.c.v_bits == 4) return launch_bits<2, 4>(a, s);
  return launch_bits<2, 2>(a, s);
}

}  // namespace kvq

// Internal helpers shared by the kvq kernels (not part of the C ABI).
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "kvq.h"

namespace kvq {

constexpr int kHeadDim = 128;
constexpr int kGroup = 32;         // channels per quantization group
constexpr int kGroups = kHeadDim / kGroup;      // 4
constexpr int kGranule = 4;        // channels per pruning group
constexpr int kPruneGroups = kHeadDim / kGranule;  // 32
constexpr unsigned kFull = 0xFFFFFFFFu;

// ---------------------------------------------------------------- loads
// Four consecutive input elements as fp32 (exact widening).
__device__ __forceinline__ void load4(const float* p, float f[4]) {
  float4 v = *reinterpret_cast<const float4*>(p);
  f[0] = v.x; f[1] = v.y; f[2] = v.z; f[3] = v.w;
}
__device__ __forceinline__ void load4(const __nv_bfloat16* p, float f[4]) {
  uint2 v = *reinterpret_cast<const uint2*>(p);
  f[0] = __uint_as_float(v.x << 16);
  f[1] = __uint_as_float(v.x & 0xFFFF0000u);
  f[2] = __uint_as_float(v.y << 16);
  f[3] = __uint_as_float(v.y & 0xFFFF0000u);
}
__device__ __forceinline__ void load4(const __half* p, float f[4]) {
  uint2 v = *reinterpret_cast<const uint2*>(p);
  __half2 a = *reinterpret_cast<__half2*>(&v.x), b = *reinterpret_cast<__half2*>(&v.y);
  float2 fa = __half22float2(a), fb = __half22float2(b);
  f[0] = fa.x; f[1] = fa.y; f[2] = fb.x; f[3] = fb.y;
}

// ---------------------------------------------------------------- rotation
// Orthonormal Walsh-Hadamard transform of one 128-channel row held by a warp,
// lane l owning channels 4l..4l+3.  Butterflies in fp64, natural Sylvester
// order (stage h pairs channel i with i+h, i & h == 0, -> (a+b, a-b)), then one
// fp64 multiply by 1/sqrt(128) and a round to fp32.  Every fp64 add of bf16 or
// fp32 inputs is IEEE-rounded in the same order on every lane, so the fp32
// result is reproducible bit for bit.
__device__ __forceinline__ void rotate_row_warp(float x[4], double inv_sqrt_d, int lane) {
  double v0 = x[0], v1 = x[1], v2 = x[2], v3 = x[3];
  // h = 1: (0,1), (2,3)
  double a0 = __dadd_rn(v0, v1), a1 = __dsub_rn(v0, v1);
  double a2 = __dadd_rn(v2, v3), a3 = __dsub_rn(v2, v3);
  // h = 2: (0,2), (1,3)
  v0 = __dadd_rn(a0, a2); v2 = __dsub_rn(a0, a2);
  v1 = __dadd_rn(a1, a3); v3 = __dsub_rn(a1, a3);
  // h = 4 .. 64: partner lane l ^ m; the lower lane keeps a+b, the upper a-b
#pragma unroll
  for (int m = 1; m < 32; m <<= 1) {
    const bool upper = (lane & m) != 0;
    double o0 = __shfl_xor_sync(kFull, v0, m), o1 = __shfl_xor_sync(kFull, v1, m);
    double o2 = __shfl_xor_sync(kFull, v2, m), o3 = __shfl_xor_sync(kFull, v3, m);
    v0 = upper ? __dsub_rn(o0, v0) : __dadd_rn(v0, o0);
    v1 = upper ? __dsub_rn(o1, v1) : __dadd_rn(v1, o1);
    v2 = upper ? __dsub_rn(o2, v2) : __dadd_rn(v2, o2);
    v3 = upper ? __dsub_rn(o3, v3) : __dadd_rn(v3, o3);
  }
  x[0] = __double2float_rn(__dmul_rn(v0, inv_sqrt_d));
  x[1] = __double2float_rn(__dmul_rn(v1, inv_sqrt_d));
  x[2] = __double2float_rn(__dmul_rn(v2, inv_sqrt_d));
  x[3] = __double2float_rn(__dmul_rn(v3, inv_sqrt_d));
}

// Load one 128-channel row (4 channels per lane) and optionally rotate it.
template <typename In>
__device__ __forceinline__ void load_row_warp(const In* row, bool rotate, double inv_sqrt_d, int lane, float x[4]) {
  load4(row + 4 * lane, x);
  if (rotate) rotate_row_warp(x, inv_sqrt_d, lane);
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int m = 16; m > 0; m >>= 1) v = fmaxf(v, __shfl_xor_sync(kFull, v, m));
  return v;
}
// Tile counts over sequences [0, n) of a batch, by a 128-thread block:
// thread t takes sequences t, t + 128, ...; returns (sum over all, sum over
// sequences < before), each times `mult`, in every thread.
template <typename TilesOf>
__device__ __forceinline__ int2 block_tile_prefix(int n, int before, int mult, TilesOf tiles_of_seq) {
  __shared__ int red[2][4];
  int all = 0, pre = 0;
  for (int i = threadIdx.x; i < n; i += 128) {
    const int t = tiles_of_seq(i);
    all += t;
    if (i < before) pre += t;
  }
#pragma unroll
  for (int m = 16; m > 0; m >>= 1) {
    all += __shfl_xor_sync(0xFFFFFFFFu, all, m);
    pre += __shfl_xor_sync(0xFFFFFFFFu, pre, m);
  }
  if ((threadIdx.x & 31) == 0) {
    red[0][threadIdx.x >> 5] = all;
    red[1][threadIdx.x >> 5] = pre;
  }
  __syncthreads();
  const int2 r = make_int2(mult * (red[0][0] + red[0][1] + red[0][2] + red[0][3]),
                           mult * (red[1][0] + red[1][1] + red[1][2] + red[1][3]));
  __syncthreads();
  return r;
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int m = 16; m > 0; m >>= 1) v += __shfl_xor_sync(kFull, v, m);
  return v;
}

// ---------------------------------------------------------------- cache layout
// Keys are stored in blocks of kKeyBlock tokens; inside a block, one row of
// kKeyBlock code words per channel group of 4, then (separately) one row of
// kKeyBlock (scale, zero) pairs per 32-channel group.  Value codes use the
// same blocks with one row per channel (see v_code_byte).
constexpr int kKeyBlock = 128;
// index of the code word of (unit bh, channel group pg, token n)
__host__ __device__ __forceinline__ size_t key_word_index(size_t bh, int cap, int pg, int n) {
  return (((bh * (size_t)(cap / kKeyBlock) + n / kKeyBlock) * kPruneGroups + pg) * kKeyBlock) + n % kKeyBlock;
}
// index of the (scale, zero) pair of (unit bh, 32-channel group g, token n)
__host__ __device__ __forceinline__ size_t key_scale_index(size_t bh, int cap, int g, int n) {
  return (((bh * (size_t)(cap / kKeyBlock) + n / kKeyBlock) * kGroups + g) * kKeyBlock) + n % kKeyBlock;
}

// Value codes: per block of kKeyBlock tokens, one row per channel holding the
// block's codes in token order (little-endian inside a byte), cut into
// 16-byte chunks; chunk i of channel ch sits at chunk position
// i ^ v_chunk_swizzle(ch), so 8 consecutive channels' rows start in 8
// different shared-memory bank groups.
// bf16 window slot of token n (written by appends), or -1: slot n below the
// sink, else a ring of `recent` slots
__host__ __device__ __forceinline__ int window_slot(int sink, int recent, int n) {
  if (n < sink) return n;
  return recent > 0 ? sink + (n - sink) % recent : -1;
}
// whether a decode over a length-len sequence takes token n from the windows
__host__ __device__ __forceinline__ bool in_window(int sink, int recent, int n, int len) {
  return n < sink || (recent > 0 && n >= (sink > len - recent ? sink : len - recent));
}

__host__ __device__ __forceinline__ int v_chunk_swizzle(int v_bits, int ch) {
  return v_bits == 4 ? (ch >> 1) & 3 : (ch >> 2) & 1;
}
// byte offset of the row of (unit bh, block blk, channel ch)
__host__ __device__ __forceinline__ size_t v_row_offset(size_t bh, int cap, int blk, int ch, int v_bits) {
  return ((bh * (size_t)(cap / kKeyBlock) + blk) * kHeadDim + ch) * (size_t)(kKeyBlock * v_bits / 8);
}

// ---------------------------------------------------------------- launch plumbing
struct CacheView {
  int B, H, cap, k_bits, v_bits, rotate, keep_ch0, rotate_v;
  float v_clip;
  int sink, recent;                    // bf16 token windows (0, 0: none)
  int pos_base;                        // sequence position of the view's token 0 (a bucket's anchor)
  __nv_bfloat16* kwin;                 // [B][H][sink + recent][128]
  __nv_bfloat16* vwin;
  uint8_t* kc;
  __half2* ks;
  __nv_bfloat16* k0;
  uint8_t* vc;
  __half2* vs;
  // extents of the arrays (what kvq_cache_sizes reports), for the bounds checks
  __host__ __device__ size_t rows() const { return (size_t)B * H * cap; }
  __host__ __device__ size_t kc_bytes() const { return rows() * kPruneGroups * (k_bits == 4 ? 2 : 1); }
  __host__ __device__ size_t ks_pairs() const { return rows() * kGroups; }
  __host__ __device__ size_t vc_bytes() const { return rows() * (kHeadDim * v_bits / 8); }
  __host__ __device__ size_t win_elems() const { return (size_t)B * H * (sink + recent) * kHeadDim; }
};

// Debug build (-DKVQ_BOUNDS_CHECK): a checked access first compares its
// element range [idx, idx + n) with its buffer's extent; an access out of
// bounds is skipped and counted in this translation unit's counter, which the
// host reads through kvq_bounds_violations.  Without the flag the checks
// compile to nothing.
#ifdef KVQ_BOUNDS_CHECK
namespace {
__device__ unsigned int g_kvq_oob = 0;
}
__device__ __forceinline__ bool kvq_in_bounds(size_t idx, size_t n, size_t extent) {
  if (idx + n <= extent) return true;
  atomicAdd(&g_kvq_oob, 1u);
  return false;
}
#define KVQ_BOUNDS_COUNTER(fn)                                                          \
  unsigned fn(bool reset) {                                                             \
    unsigned v = 0;                                                                     \
    cudaMemcpyFromSymbol(&v, g_kvq_oob, sizeof(v));                                    \
    if (reset) {                                                                        \
      const unsigned z = 0;                                                             \
      cudaMemcpyToSymbol(g_kvq_oob, &z, sizeof(z));                                     \
    }                                                                                   \
    return v;                                                                           \
  }
#else
__device__ __forceinline__ bool kvq_in_bounds(size_t, size_t, size_t) { return true; }
#define KVQ_BOUNDS_COUNTER(fn) \
  unsigned fn(bool) { return 0; }
#endif
// per translation unit: its count of skipped accesses (optionally cleared)
unsigned bounds_append(bool reset);
unsigned bounds_decode(bool reset);
unsigned bounds_window(bool reset);

struct AppendArgs {
  CacheView c;
  const void* k_new;
  const void* v_new;
  int dtype, n_new, offset;
  double inv_sqrt_d;
};

struct SelectArgs {
  const void* q;
  int dtype, B, Hq, H, rotate, keep;
  double inv_sqrt_d;
  uint32_t* mask;
};

struct DecodeArgs {
  CacheView c;
  const void* q;
  int dtype, Hq;
  const int32_t* seq_lens;
  int max_len;
  const uint32_t* mask;
  float scale_log2;  // softmax_scale * log2(e): scores live in the exp2 domain
  double inv_sqrt_d;
  int win_base;     // first partial slot of the bf16 windows: one slot per unit after decode_slots
  float* part_acc;  // [decode_slots][G][128] unnormalized accumulators
  float2* part_ml;  // [decode_slots][G] (running max, running sum)
  float* out;       // [B][Hq][128]
  size_t part_rows;  // rows of part_acc / part_ml (for the bounds checks)
  int* status;      // device word: bit 0 set when a bounded wait of the split decode gave up
  // bucket-relative RoPE: sequence vb of the decode is bucket vb % bucket_nb of
  // sequence vb / bucket_nb, whose length is real_lens[] (clamped to
  // real_max_len); bucket_nb = 0 without buckets.  The bf16 windows are
  // placed by the real sequence's positions and length.
  int bucket_nb, bucket_w;
  const int32_t* real_lens;
  int real_max_len;
  int withheld_tile;  // test hook: CTA 0 never fills this tile's ring stage (-1: none)
};

cudaError_t launch_append(const AppendArgs& a, cudaStream_t s);
cudaError_t launch_select(const SelectArgs& a, cudaStream_t s);
// persistent tensor-core split decode (GQA groups of 1, 2, 4, 8 or 16 query
// heads) and its combine; partial slots: decode_groups(G) per (unit + CTA),
// decode_slots of them
bool decode_g_supported(int g);
int decode_groups(int G);
int decode_slots(int B, int H, int G);
cudaError_t launch_decode(const DecodeArgs& a, cudaStream_t s);
// attention over the bf16 window tokens of every unit: one partial per unit at win_base + unit
cudaError_t launch_window(const DecodeArgs& a, cudaStream_t s);
cudaError_t launch_combine(const DecodeArgs& a, cudaStream_t s);

// Checked split decode + combine into a caller-chosen scratch buffer of
// `workspace_bytes` bytes (the body of kvq_decode_attention).
kvq_status decode_into(const kvq_cache* c, const void* q, kvq_dtype dtype, int32_t q_heads, const int32_t* seq_lens,
                       int32_t max_len, const uint32_t* mask, float softmax_scale, float* out, void* workspace,
                       size_t workspace_bytes, cudaStream_t s);

}  // namespace kvq

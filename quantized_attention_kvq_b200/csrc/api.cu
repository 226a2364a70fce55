// C ABI of libkvq: argument checks, workspace carving and kernel launches.
// Every check happens on the host before anything is enqueued; no exception
// leaves this file.
#include <cmath>
#include <cstdint>
#include <mutex>

#include <nvtx3/nvToolsExt.h>

#include "transform.cuh"

namespace kvq {
namespace {

// One NVTX range per enqueueing ABI call (named after it), so that a
// timeline profiler shows which call enqueued which kernels.  NVTX is
// header-only and costs a branch when no tool is attached.
struct NvtxRange {
  explicit NvtxRange(const char* name) { nvtxRangePushA(name); }
  ~NvtxRange() { nvtxRangePop(); }
  NvtxRange(const NvtxRange&) = delete;
  NvtxRange& operator=(const NvtxRange&) = delete;
};

constexpr size_t kAlign = 256;

inline size_t round_up(size_t v, size_t a) { return (v + a - 1) / a * a; }
inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
inline size_t dtype_size(kvq_dtype t) { return t == KVQ_F32 ? 4 : 2; }
inline bool dtype_ok(int t) { return t == KVQ_F32 || t == KVQ_BF16 || t == KVQ_F16; }

// Shape/flag checks that do not look at pointers.
kvq_status check_shape(const kvq_cache* c) {
  if (!c) return KVQ_ERR_INVALID_ARG;
  if (c->batch < 1 || c->kv_heads < 1 || c->capacity < 1 || c->head_dim < 1) return KVQ_ERR_INVALID_ARG;
  if (c->rotate_k < 0 || c->rotate_k > 2 || (c->keep_ch0 != 0 && c->keep_ch0 != 1)) return KVQ_ERR_INVALID_ARG;
  if ((c->rotate_v != 0 && c->rotate_v != 1) || !(c->v_clip > 0.0f && c->v_clip <= 1.0f)) return KVQ_ERR_INVALID_ARG;
  if (c->sink_tokens < 0 || c->recent_tokens < 0 || (int64_t)c->sink_tokens + c->recent_tokens > c->capacity)
    return KVQ_ERR_INVALID_ARG;
  if (c->sink_tokens + c->recent_tokens > 2048) return KVQ_ERR_UNSUPPORTED;  // the window kernel's shared memory
  if (c->head_dim != kHeadDim || c->group_size != kGroup || c->prune_granule != kGranule) return KVQ_ERR_UNSUPPORTED;
  if ((c->k_bits != 2 && c->k_bits != 4) || (c->v_bits != 2 && c->v_bits != 4)) return KVQ_ERR_UNSUPPORTED;
  if (c->capacity % kKeyBlock != 0) return KVQ_ERR_UNSUPPORTED;
  if (c->bucket_tokens < 0) return KVQ_ERR_INVALID_ARG;
  // with bucket-relative RoPE the bf16 windows may touch at most three
  // buckets (the sinks the first, the recent tokens at most two)
  if (c->bucket_tokens > 0 && (c->bucket_tokens % kKeyBlock != 0 || c->capacity % c->bucket_tokens != 0 ||
                               c->sink_tokens > c->bucket_tokens || c->recent_tokens > c->bucket_tokens))
    return KVQ_ERR_UNSUPPORTED;
  // the selection runs one grid row per (sequence, bucket), the append one grid
  // layer per sequence: both at most 65535
  const int64_t rows = (int64_t)c->batch * (c->bucket_tokens > 0 ? c->capacity / c->bucket_tokens : 1);
  if (rows > 65535) return KVQ_ERR_UNSUPPORTED;
  return KVQ_OK;
}

// the caller's transform pair, when rotate_k selects it
bool pair_ok(const kvq_cache* c, bool query, bool key) {
  if (c->rotate_k != 2) return true;
  return (!query || (c->t_query && aligned16(c->t_query))) && (!key || (c->t_key && aligned16(c->t_key)));
}

kvq_status check_cache(const kvq_cache* c) {
  kvq_status st = check_shape(c);
  if (st != KVQ_OK) return st;
  if (!pair_ok(c, true, true)) return KVQ_ERR_INVALID_ARG;
  if (c->bucket_tokens > 0 && (!c->rope_inv_freq || !aligned16(c->rope_inv_freq))) return KVQ_ERR_INVALID_ARG;
  if (!c->k_codes || !c->k_scales || !c->v_codes || !c->v_scales || (c->keep_ch0 && !c->k_ch0))
    return KVQ_ERR_INVALID_ARG;
  if (!aligned16(c->k_codes) || !aligned16(c->k_scales) || !aligned16(c->v_codes) || !aligned16(c->v_scales) ||
      (c->keep_ch0 && !aligned16(c->k_ch0)))
    return KVQ_ERR_INVALID_ARG;
  if (c->sink_tokens + c->recent_tokens > 0 &&
      (!c->k_window || !c->v_window || !aligned16(c->k_window) || !aligned16(c->v_window)))
    return KVQ_ERR_INVALID_ARG;
  return KVQ_OK;
}

kvq_status check_heads(const kvq_cache* c, int32_t q_heads) {
  if (q_heads < 1 || q_heads % c->kv_heads != 0) return KVQ_ERR_INVALID_ARG;
  return KVQ_OK;
}

CacheView view(const kvq_cache* c) {
  CacheView v;
  v.B = c->batch;
  v.H = c->kv_heads;
  v.cap = c->capacity;
  v.k_bits = c->k_bits;
  v.v_bits = c->v_bits;
  v.rotate = c->rotate_k;
  v.keep_ch0 = c->keep_ch0;
  v.rotate_v = c->rotate_v;
  v.v_clip = c->v_clip;
  v.sink = c->sink_tokens;
  v.recent = c->recent_tokens;
  v.pos_base = 0;
  v.kwin = static_cast<__nv_bfloat16*>(c->k_window);
  v.vwin = static_cast<__nv_bfloat16*>(c->v_window);
  v.kc = static_cast<uint8_t*>(c->k_codes);
  v.ks = static_cast<__half2*>(c->k_scales);
  v.k0 = static_cast<__nv_bfloat16*>(c->k_ch0);
  v.vc = static_cast<uint8_t*>(c->v_codes);
  v.vs = static_cast<__half2*>(c->v_scales);
  return v;
}

double inv_sqrt_d() { return 1.0 / std::sqrt((double)kHeadDim); }

// Buckets of a bucket-relative RoPE cache (1 without): the arrays are those of
// a cache of batch B * nb and capacity bucket_tokens.
inline int n_buckets(const kvq_cache* c) { return c->bucket_tokens > 0 ? c->capacity / c->bucket_tokens : 1; }

// Bytes of the five arrays for `batch` sequences of `cap` tokens.
void array_bytes(const kvq_cache* c, size_t batch, size_t cap, size_t out[5]) {
  const size_t rows = batch * c->kv_heads * cap;
  out[0] = rows * kPruneGroups * (c->k_bits == 4 ? 2 : 1);
  out[1] = rows * kGroups * 4;
  out[2] = c->keep_ch0 ? rows * 2 : 0;
  out[3] = rows * (kHeadDim * c->v_bits / 8);
  out[4] = rows * kGroups * 4;
}

// The view of bucket sequence vb alone (batch 1, capacity bucket_tokens).
CacheView bucket_sequence_view(const kvq_cache* c, size_t vb) {
  CacheView v = view(c);
  size_t per[5];
  array_bytes(c, 1, c->bucket_tokens, per);
  v.B = 1;
  v.cap = c->bucket_tokens;
  v.kc = v.kc + vb * per[0];
  v.ks = reinterpret_cast<__half2*>(reinterpret_cast<char*>(v.ks) + vb * per[1]);
  if (v.k0) v.k0 = reinterpret_cast<__nv_bfloat16*>(reinterpret_cast<char*>(v.k0) + vb * per[2]);
  v.vc = v.vc + vb * per[3];
  v.vs = reinterpret_cast<__half2*>(reinterpret_cast<char*>(v.vs) + vb * per[4]);
  // the bf16 windows belong to the real sequence vb / nb, at its positions
  const int nb = n_buckets(c);
  v.pos_base = (int)(vb % nb) * c->bucket_tokens;
  const size_t win_seq = (size_t)c->kv_heads * (c->sink_tokens + c->recent_tokens) * kHeadDim;
  if (v.kwin) v.kwin += (vb / nb) * win_seq;
  if (v.vwin) v.vwin += (vb / nb) * win_seq;
  return v;
}

// Workspace of the decode: one partial row (128-channel accumulator, running
// max and sum) per (slot, query head of the GQA group), decode_slots slots;
// with the caller's transform pair, then the transformed fp32 query rows.
struct DecodePlan {
  size_t rows, acc_bytes, ml_offset, tq_offset, qb_offset, vl_offset, mask_offset, status_offset, bytes;
};

DecodePlan plan_decode(const kvq_cache* c, int32_t q_heads) {
  DecodePlan p;
  const int G = q_heads / c->kv_heads;
  const bool win = c->sink_tokens + c->recent_tokens > 0;  // one more partial per unit for the windows
  const int Bv = c->batch * n_buckets(c);  // the split decode runs over every bucket as a sequence
  const size_t rows = ((size_t)decode_slots(Bv, c->kv_heads, G) + (win ? c->batch * c->kv_heads : 0)) * G;
  p.rows = rows;
  p.acc_bytes = rows * kHeadDim * sizeof(float);
  p.ml_offset = round_up(p.acc_bytes, kAlign);
  p.tq_offset = p.ml_offset + round_up(rows * sizeof(float2), kAlign);
  p.bytes = p.tq_offset;
  if (c->rotate_k == 2) p.bytes += round_up((size_t)c->batch * q_heads * kHeadDim * sizeof(float), kAlign);
  // with buckets: each bucket's query rows and length
  p.qb_offset = p.bytes;
  if (c->bucket_tokens > 0) p.bytes += round_up((size_t)Bv * q_heads * kHeadDim * sizeof(float), kAlign);
  p.vl_offset = p.bytes;
  if (c->bucket_tokens > 0) p.bytes += round_up((size_t)Bv * sizeof(int32_t), kAlign);
  // the kept-group masks of a decode that selects channels itself
  p.mask_offset = p.bytes;
  p.bytes += round_up((size_t)Bv * c->kv_heads * sizeof(uint32_t), kAlign);
  // the split decode's status word (a wait gave up), cleared by each split
  p.status_offset = p.bytes;
  p.bytes += kAlign;
  return p;
}

// test hook: the tile the next split decode of this host thread withholds
thread_local int g_withheld_tile = -1;
int take_withheld_tile() {
  const int t = g_withheld_tile;
  g_withheld_tile = -1;
  return t;
}

kvq_status cuda_status(cudaError_t e) { return e == cudaSuccess ? KVQ_OK : KVQ_ERR_CUDA; }

// which halves of the decode to enqueue
enum { kRunSplit = 1, kRunCombine = 2 };

// The kept-group masks of a decode that selects its channels itself, from the
// query rows the decode prepares anyway: rows already transformed (fp32, no
// further rotation) when `rows` is not NULL, else the caller's queries.
kvq_status enqueue_select(const kvq_cache* c, const void* q, kvq_dtype dtype, int32_t q_heads, int32_t B,
                          const float* rows, int32_t keep_groups, uint32_t* mask, cudaStream_t s) {
  SelectArgs a;
  a.q = rows ? static_cast<const void*>(rows) : q;
  a.dtype = rows ? KVQ_F32 : dtype;
  a.B = B;
  a.Hq = q_heads;
  a.H = c->kv_heads;
  a.rotate = rows ? 0 : c->rotate_k;
  a.keep = keep_groups;
  a.inv_sqrt_d = inv_sqrt_d();
  a.mask = mask;
  return cuda_status(launch_select_pair(a, rows ? nullptr : c->t_query, s));
}

// Per device: a non-blocking side stream and two events for forking the
// window kernel off the caller's stream (created on first use, never freed).
struct SideStream {
  cudaStream_t stream = nullptr;
  cudaEvent_t fork = nullptr, join = nullptr;
};
constexpr int kMaxSideDevices = 64;
SideStream g_side[kMaxSideDevices];
std::mutex g_side_mutex;

kvq_status side_stream(SideStream** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxSideDevices) return KVQ_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_side_mutex);
  SideStream& ss = g_side[dev];
  if (!ss.stream) {
    if (cudaStreamCreateWithFlags(&ss.stream, cudaStreamNonBlocking) != cudaSuccess ||
        cudaEventCreateWithFlags(&ss.fork, cudaEventDisableTiming) != cudaSuccess ||
        cudaEventCreateWithFlags(&ss.join, cudaEventDisableTiming) != cudaSuccess)
      return KVQ_ERR_CUDA;
  }
  *out = &ss;
  return KVQ_OK;
}

// The window attention on the side stream: after everything enqueued on s so
// far, and before everything enqueued on s afterwards.  One fork at a time
// per device (the events are reused), which the mutex above orders.
kvq_status fork_window(const DecodeArgs& a, cudaStream_t s) {
  SideStream* ss = nullptr;
  kvq_status st = side_stream(&ss);
  if (st != KVQ_OK) return st;
  std::lock_guard<std::mutex> lock(g_side_mutex);
  if (cudaEventRecord(ss->fork, s) != cudaSuccess || cudaStreamWaitEvent(ss->stream, ss->fork, 0) != cudaSuccess)
    return KVQ_ERR_CUDA;
  if ((st = cuda_status(launch_window(a, ss->stream))) != KVQ_OK) return st;
  if (cudaEventRecord(ss->join, ss->stream) != cudaSuccess || cudaStreamWaitEvent(s, ss->join, 0) != cudaSuccess)
    return KVQ_ERR_CUDA;
  return KVQ_OK;
}

kvq_status enqueue_decode(const kvq_cache* c, const void* q, kvq_dtype dtype, int32_t q_heads,
                          const int32_t* seq_lens, int32_t max_len, const uint32_t* mask, float softmax_scale,
                          float* out, void* workspace, const DecodePlan& plan, cudaStream_t s,
                          int parts = kRunSplit | kRunCombine, int32_t keep_groups = kPruneGroups) {
  uint32_t* own_mask = reinterpret_cast<uint32_t*>(static_cast<char*>(workspace) + plan.mask_offset);
  const bool select = keep_groups < kPruneGroups;
  if (c->bucket_tokens > 0) {
    // every bucket is a sequence of the split decode, with its own query and
    // length; the merge makes one softmax of them
    const int nb = n_buckets(c), G = q_heads / c->kv_heads;
    char* ws = static_cast<char*>(workspace);
    DecodeArgs v;
    v.c = view(c);
    v.c.B = c->batch * nb;
    v.c.cap = c->bucket_tokens;
    v.c.rotate = 0;
    v.q = ws + plan.qb_offset;
    v.dtype = KVQ_F32;
    v.Hq = q_heads;
    v.seq_lens = reinterpret_cast<const int32_t*>(ws + plan.vl_offset);
    v.max_len = max_len < c->bucket_tokens ? max_len : c->bucket_tokens;
    v.mask = mask;
    v.scale_log2 = (float)((double)softmax_scale * 1.4426950408889634);  // log2(e)
    v.inv_sqrt_d = inv_sqrt_d();
    v.win_base = decode_slots(v.c.B, c->kv_heads, G);
    v.part_acc = reinterpret_cast<float*>(ws);
    v.part_ml = reinterpret_cast<float2*>(ws + plan.ml_offset);
    v.out = nullptr;
    v.part_rows = plan.rows;
    v.bucket_nb = nb;
    v.bucket_w = c->bucket_tokens;
    v.real_lens = seq_lens;
    v.real_max_len = max_len;
    v.status = reinterpret_cast<int*>(ws + plan.status_offset);
    v.withheld_tile = -1;
    if (parts & kRunSplit) {
      v.withheld_tile = take_withheld_tile();
      kvq_status st0 = cuda_status(cudaMemsetAsync(v.status, 0, sizeof(int), s));
      if (st0 != KVQ_OK) return st0;
      kvq_status st = cuda_status(launch_bucket_queries(
          q, dtype, c->rotate_k, c->t_query, c->rope_inv_freq, seq_lens, max_len, c->batch, q_heads, c->kv_heads,
          c->bucket_tokens, nb, inv_sqrt_d(), reinterpret_cast<float*>(ws + plan.qb_offset),
          reinterpret_cast<int32_t*>(ws + plan.vl_offset), s));
      if (st != KVQ_OK) return st;
      if (select) {
        // every bucket's query rows are embedded and transformed already
        st = enqueue_select(c, nullptr, KVQ_F32, q_heads, v.c.B, reinterpret_cast<const float*>(ws + plan.qb_offset),
                            keep_groups, own_mask, s);
        if (st != KVQ_OK) return st;
        v.mask = own_mask;
      }
      if (v.max_len > 0 && (st = cuda_status(launch_decode(v, s))) != KVQ_OK) return st;
      if (c->sink_tokens + c->recent_tokens > 0) {
        // the bf16 window tokens of each real sequence, scored with the query
        // rows of the buckets they sit in (already embedded and transformed)
        DecodeArgs aw = v;
        aw.c = view(c);
        aw.c.rotate = 0;
        aw.q = ws + plan.qb_offset;
        aw.dtype = KVQ_F32;
        aw.seq_lens = seq_lens;
        aw.max_len = max_len;
        if ((st = fork_window(aw, s)) != KVQ_OK) return st;
      }
    }
    if (parts & kRunCombine)
      return cuda_status(launch_bucket_merge(v, nb, decode_slots(0, 0, G) / decode_groups(G), decode_groups(G), out, s));
    return KVQ_OK;
  }
  DecodeArgs a;
  a.c = view(c);
  a.q = q;
  a.dtype = dtype;
  a.Hq = q_heads;
  a.seq_lens = seq_lens;
  a.max_len = max_len;
  a.mask = mask;
  a.scale_log2 = (float)((double)softmax_scale * 1.4426950408889634);  // log2(e)
  a.inv_sqrt_d = inv_sqrt_d();
  a.win_base = decode_slots(c->batch, c->kv_heads, q_heads / c->kv_heads);
  a.part_acc = static_cast<float*>(workspace);
  a.part_ml = reinterpret_cast<float2*>(static_cast<char*>(workspace) + plan.ml_offset);
  a.out = out;
  a.part_rows = plan.rows;
  a.bucket_nb = 0;
  a.bucket_w = 0;
  a.real_lens = nullptr;
  a.real_max_len = 0;
  a.status = reinterpret_cast<int*>(static_cast<char*>(workspace) + plan.status_offset);
  a.withheld_tile = -1;
  if (parts & kRunSplit) {
    a.withheld_tile = take_withheld_tile();
    kvq_status st = cuda_status(cudaMemsetAsync(a.status, 0, sizeof(int), s));
    if (st != KVQ_OK) return st;
  }
  if ((parts & kRunSplit) && c->rotate_k == 2) {
    // the kernels below read the transformed rows as untransformed fp32 queries
    float* qt = reinterpret_cast<float*>(static_cast<char*>(workspace) + plan.tq_offset);
    kvq_status st = cuda_status(launch_transform_q(q, dtype, c->t_query, c->batch, q_heads, c->kv_heads, qt, s));
    if (st != KVQ_OK) return st;
    a.q = qt;
    a.dtype = KVQ_F32;
    a.c.rotate = 0;
  }
  if ((parts & kRunSplit) && select) {
    kvq_status st = enqueue_select(c, q, dtype, q_heads, c->batch,
                                   c->rotate_k == 2 ? static_cast<const float*>(a.q) : nullptr, keep_groups, own_mask, s);
    if (st != KVQ_OK) return st;
    a.mask = own_mask;
  }
  if ((parts & kRunSplit) && max_len > 0) {
    kvq_status st = cuda_status(launch_decode(a, s));
    if (st != KVQ_OK) return st;
  }
  if ((parts & kRunSplit) && c->sink_tokens + c->recent_tokens > 0) {
    // the bf16 window attention is independent of the split decode: it runs on
    // a side stream forked after the split, so its CTAs take SMs as the split's
    // CTAs finish, and joins before the combine
    kvq_status st = fork_window(a, s);
    if (st != KVQ_OK) return st;
  }
  if (parts & kRunCombine) return cuda_status(launch_combine(a, s));
  return KVQ_OK;
}

kvq_status check_decode(const kvq_cache* c, const void* q, kvq_dtype dtype, int32_t q_heads,
                        const int32_t* seq_lens, int32_t max_len, float softmax_scale, const void* out,
                        const void* workspace, size_t workspace_bytes, bool need_q) {
  kvq_status st = check_cache(c);
  if (st != KVQ_OK) return st;
  if ((st = check_heads(c, q_heads)) != KVQ_OK) return st;
  if (!dtype_ok(dtype) || (need_q && (!q || !aligned16(q))) || !seq_lens || !out || !workspace ||
      !aligned16(workspace))
    return KVQ_ERR_INVALID_ARG;
  if (!std::isfinite(softmax_scale)) return KVQ_ERR_INVALID_ARG;
  if (max_len < 0) return KVQ_ERR_INVALID_ARG;
  if (max_len > c->capacity) return KVQ_ERR_CAPACITY;
  if (!decode_g_supported(q_heads / c->kv_heads)) return KVQ_ERR_UNSUPPORTED;
  if (workspace_bytes < plan_decode(c, q_heads).bytes) return KVQ_ERR_WORKSPACE;
  return KVQ_OK;
}

}  // namespace

kvq_status decode_into(const kvq_cache* c, const void* q, kvq_dtype dtype, int32_t q_heads, const int32_t* seq_lens,
                       int32_t max_len, const uint32_t* mask, float softmax_scale, float* out, void* workspace,
                       size_t workspace_bytes, cudaStream_t s) {
  kvq_status st = check_decode(c, q, dtype, q_heads, seq_lens, max_len, softmax_scale, out, workspace,
                               workspace_bytes, true);
  if (st != KVQ_OK) return st;
  return enqueue_decode(c, q, dtype, q_heads, seq_lens, max_len, mask, softmax_scale, out, workspace,
                        plan_decode(c, q_heads), s);
}

}  // namespace kvq

using namespace kvq;

extern "C" {

KVQ_API kvq_status kvq_cache_sizes(const kvq_cache* c, size_t bytes_out[5]) {
  kvq_status st = check_shape(c);
  if (st != KVQ_OK) return st;
  if (!bytes_out) return KVQ_ERR_INVALID_ARG;
  array_bytes(c, c->batch, c->capacity, bytes_out);
  return KVQ_OK;
}

KVQ_API size_t kvq_window_bytes(const kvq_cache* c) {
  if (check_shape(c) != KVQ_OK) return 0;
  return (size_t)c->batch * c->kv_heads * (size_t)(c->sink_tokens + c->recent_tokens) * kHeadDim * 2;
}

KVQ_API kvq_status kvq_quantize_append(const kvq_cache* c, const void* k_new, const void* v_new, kvq_dtype dtype,
                                       int32_t n_new, int32_t offset, void* stream) {
  NvtxRange range("kvq_quantize_append");
  kvq_status st = check_cache(c);
  if (st != KVQ_OK) return st;
  if (!dtype_ok(dtype) || n_new < 0 || offset < 0) return KVQ_ERR_INVALID_ARG;
  if ((int64_t)offset + n_new > c->capacity) return KVQ_ERR_CAPACITY;
  if (n_new == 0) return KVQ_OK;
  if (!k_new || !v_new || !aligned16(k_new) || !aligned16(v_new)) return KVQ_ERR_INVALID_ARG;
  if (c->bucket_tokens > 0) {
    // one launch per sequence into its bucket's sequence, keys embedded at
    // their offset from the bucket's anchor
    const int w = c->bucket_tokens, k = offset / w;
    if ((offset + n_new - 1) / w != k) return KVQ_ERR_INVALID_ARG;
    const size_t in_seq = (size_t)c->kv_heads * n_new * kHeadDim * dtype_size(dtype);
    for (int b = 0; b < c->batch; ++b) {
      AppendArgs a;
      a.c = bucket_sequence_view(c, (size_t)b * n_buckets(c) + k);
      a.k_new = static_cast<const char*>(k_new) + b * in_seq;
      a.v_new = static_cast<const char*>(v_new) + b * in_seq;
      a.dtype = dtype;
      a.n_new = n_new;
      a.offset = offset - k * w;
      a.inv_sqrt_d = inv_sqrt_d();
      kvq_status st = cuda_status(launch_append_ext(a, c->t_key, c->rope_inv_freq, static_cast<cudaStream_t>(stream)));
      if (st != KVQ_OK) return st;
    }
    return KVQ_OK;
  }
  AppendArgs a;
  a.c = view(c);
  a.k_new = k_new;
  a.v_new = v_new;
  a.dtype = dtype;
  a.n_new = n_new;
  a.offset = offset;
  a.inv_sqrt_d = inv_sqrt_d();
  return cuda_status(launch_append_ext(a, c->t_key, nullptr, static_cast<cudaStream_t>(stream)));
}

KVQ_API kvq_status kvq_select_channels_at(const kvq_cache* c, const void* q, kvq_dtype dtype, int32_t q_heads,
                                          const int32_t* seq_lens, int32_t keep_groups, uint32_t* mask_out,
                                          void* stream) {
  NvtxRange range("kvq_select_channels_at");
  kvq_status st = check_shape(c);
  if (st != KVQ_OK) return st;
  if ((st = check_heads(c, q_heads)) != KVQ_OK) return st;
  if (!dtype_ok(dtype) || !q || !mask_out || !aligned16(q) || !pair_ok(c, true, false)) return KVQ_ERR_INVALID_ARG;
  if (c->bucket_tokens > 0 && (!seq_lens || !c->rope_inv_freq || !aligned16(c->rope_inv_freq)))
    return KVQ_ERR_INVALID_ARG;
  if (keep_groups < 1 || keep_groups > kPruneGroups) return KVQ_ERR_INVALID_ARG;
  if (q_heads / c->kv_heads > 64) return KVQ_ERR_UNSUPPORTED;
  SelectArgs a;
  a.q = q;
  a.dtype = dtype;
  a.B = c->batch;
  a.Hq = q_heads;
  a.H = c->kv_heads;
  a.rotate = c->rotate_k;
  a.keep = keep_groups;
  a.inv_sqrt_d = inv_sqrt_d();
  a.mask = mask_out;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (c->bucket_tokens > 0)
    return cuda_status(
        launch_select_buckets(a, c->t_query, c->rope_inv_freq, seq_lens, c->bucket_tokens, n_buckets(c), s));
  return cuda_status(launch_select_pair(a, c->t_query, s));
}

KVQ_API kvq_status kvq_select_channels(const kvq_cache* c, const void* q, kvq_dtype dtype, int32_t q_heads,
                                       int32_t keep_groups, uint32_t* mask_out, void* stream) {
  NvtxRange range("kvq_select_channels");
  // bucket-relative RoPE needs the queries' positions: kvq_select_channels_at
  if (c && c->bucket_tokens != 0) return KVQ_ERR_INVALID_ARG;
  return kvq_select_channels_at(c, q, dtype, q_heads, nullptr, keep_groups, mask_out, stream);
}

KVQ_API kvq_status kvq_decode_status(const kvq_cache* c, int32_t q_heads, const void* workspace,
                                     size_t workspace_bytes, void* stream) {
  NvtxRange range("kvq_decode_status");
  if (check_shape(c) != KVQ_OK || check_heads(c, q_heads) != KVQ_OK || !workspace || !aligned16(workspace))
    return KVQ_ERR_INVALID_ARG;
  if (!decode_g_supported(q_heads / c->kv_heads)) return KVQ_ERR_UNSUPPORTED;
  const DecodePlan plan = plan_decode(c, q_heads);
  if (workspace_bytes < plan.bytes) return KVQ_ERR_WORKSPACE;
  int word = 0;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (cudaMemcpyAsync(&word, static_cast<const char*>(workspace) + plan.status_offset, sizeof(int),
                      cudaMemcpyDeviceToHost, s) != cudaSuccess ||
      cudaStreamSynchronize(s) != cudaSuccess)
    return KVQ_ERR_CUDA;
  return word ? KVQ_ERR_TIMEOUT : KVQ_OK;
}

KVQ_API void kvq_test_withhold_tile(int32_t tile) { kvq::g_withheld_tile = tile < 0 ? -1 : tile; }

KVQ_API uint32_t kvq_bounds_violations(int32_t reset) {
#ifdef KVQ_BOUNDS_CHECK
  if (cudaDeviceSynchronize() != cudaSuccess) return UINT32_MAX;
  const bool r = reset != 0;
  return kvq::bounds_append(r) + kvq::bounds_decode(r) + kvq::bounds_window(r);
#else
  (void)reset;
  return UINT32_MAX;  // this build has no bounds checks
#endif
}

KVQ_API size_t kvq_decode_workspace_bytes(const kvq_cache* c, int32_t q_heads, int32_t max_len) {
  if (check_shape(c) != KVQ_OK || check_heads(c, q_heads) != KVQ_OK) return 0;
  if (max_len < 0 || max_len > c->capacity) return 0;
  return plan_decode(c, q_heads).bytes;
}

KVQ_API kvq_status kvq_decode_attention(const kvq_cache* c, const void* q, kvq_dtype dtype, int32_t q_heads,
                                        const int32_t* seq_lens, int32_t max_len, const uint32_t* mask,
                                        float softmax_scale, float* out, void* workspace, size_t workspace_bytes,
                                        void* stream) {
  NvtxRange range("kvq_decode_attention");
  kvq_status st = check_decode(c, q, dtype, q_heads, seq_lens, max_len, softmax_scale, out, workspace,
                               workspace_bytes, true);
  if (st != KVQ_OK) return st;
  return enqueue_decode(c, q, dtype, q_heads, seq_lens, max_len, mask, softmax_scale, out, workspace,
                        plan_decode(c, q_heads), static_cast<cudaStream_t>(stream));
}

KVQ_API kvq_status kvq_decode_partials(const kvq_cache* c, const void* q, kvq_dtype dtype, int32_t q_heads,
                                       const int32_t* seq_lens, int32_t max_len, const uint32_t* mask,
                                       float softmax_scale, void* workspace, size_t workspace_bytes, void* stream) {
  NvtxRange range("kvq_decode_partials");
  kvq_status st = check_decode(c, q, dtype, q_heads, seq_lens, max_len, softmax_scale, workspace, workspace,
                               workspace_bytes, true);
  if (st != KVQ_OK) return st;
  return enqueue_decode(c, q, dtype, q_heads, seq_lens, max_len, mask, softmax_scale, nullptr, workspace,
                        plan_decode(c, q_heads), static_cast<cudaStream_t>(stream), kRunSplit);
}

KVQ_API kvq_status kvq_decode_attention_select(const kvq_cache* c, const void* q, kvq_dtype dtype, int32_t q_heads,
                                               const int32_t* seq_lens, int32_t max_len, int32_t keep_groups,
                                               float softmax_scale, float* out, void* workspace,
                                               size_t workspace_bytes, void* stream) {
  NvtxRange range("kvq_decode_attention_select");
  kvq_status st = check_decode(c, q, dtype, q_heads, seq_lens, max_len, softmax_scale, out, workspace,
                               workspace_bytes, true);
  if (st != KVQ_OK) return st;
  if (keep_groups < 1 || keep_groups > kPruneGroups) return KVQ_ERR_INVALID_ARG;
  return enqueue_decode(c, q, dtype, q_heads, seq_lens, max_len, nullptr, softmax_scale, out, workspace,
                        plan_decode(c, q_heads), static_cast<cudaStream_t>(stream), kRunSplit | kRunCombine,
                        keep_groups);
}

KVQ_API kvq_status kvq_decode_partials_select(const kvq_cache* c, const void* q, kvq_dtype dtype, int32_t q_heads,
                                              const int32_t* seq_lens, int32_t max_len, int32_t keep_groups,
                                              float softmax_scale, void* workspace, size_t workspace_bytes,
                                              void* stream) {
  NvtxRange range("kvq_decode_partials_select");
  kvq_status st = check_decode(c, q, dtype, q_heads, seq_lens, max_len, softmax_scale, workspace, workspace,
                               workspace_bytes, true);
  if (st != KVQ_OK) return st;
  if (keep_groups < 1 || keep_groups > kPruneGroups) return KVQ_ERR_INVALID_ARG;
  return enqueue_decode(c, q, dtype, q_heads, seq_lens, max_len, nullptr, softmax_scale, nullptr, workspace,
                        plan_decode(c, q_heads), static_cast<cudaStream_t>(stream), kRunSplit, keep_groups);
}

KVQ_API kvq_status kvq_decode_combine(const kvq_cache* c, int32_t q_heads, const int32_t* seq_lens, int32_t max_len,
                                      float* out, const void* workspace, size_t workspace_bytes, void* stream) {
  NvtxRange range("kvq_decode_combine");
  kvq_status st = check_decode(c, nullptr, KVQ_F32, q_heads, seq_lens, max_len, 1.0f, out, workspace,
                               workspace_bytes, false);
  if (st != KVQ_OK) return st;
  return enqueue_decode(c, nullptr, KVQ_F32, q_heads, seq_lens, max_len, nullptr, 1.0f, out,
                        const_cast<void*>(workspace), plan_decode(c, q_heads),
                        static_cast<cudaStream_t>(stream), kRunCombine);
}

KVQ_API size_t kvq_decode_step_workspace_bytes(const kvq_cache* c, kvq_dtype dtype, int32_t q_heads,
                                               int32_t max_len) {
  if (check_shape(c) != KVQ_OK || check_heads(c, q_heads) != KVQ_OK || !dtype_ok(dtype)) return 0;
  if (max_len < 0 || max_len > c->capacity) return 0;
  const size_t qb = (size_t)c->batch * q_heads * kHeadDim * dtype_size(dtype);
  const size_t mb = (size_t)c->batch * n_buckets(c) * c->kv_heads * sizeof(uint32_t);
  const size_t ob = (size_t)c->batch * q_heads * kHeadDim * sizeof(float);
  return round_up(qb, kAlign) + round_up(mb, kAlign) + round_up(ob, kAlign) + plan_decode(c, q_heads).bytes;
}

KVQ_API kvq_status kvq_decode_step_host(const kvq_cache* c, const void* q_host, kvq_dtype dtype, int32_t q_heads,
                                        const int32_t* seq_lens, int32_t max_len, int32_t keep_groups,
                                        float softmax_scale, float* out_host, void* workspace,
                                        size_t workspace_bytes, void* stream) {
  NvtxRange range("kvq_decode_step_host");
  kvq_status st = check_cache(c);
  if (st != KVQ_OK) return st;
  if ((st = check_heads(c, q_heads)) != KVQ_OK) return st;
  if (!dtype_ok(dtype) || !q_host || !out_host || !seq_lens || !workspace || !aligned16(workspace))
    return KVQ_ERR_INVALID_ARG;
  if (keep_groups < 1 || keep_groups > kPruneGroups || !std::isfinite(softmax_scale) || max_len < 0)
    return KVQ_ERR_INVALID_ARG;
  if (max_len > c->capacity) return KVQ_ERR_CAPACITY;
  if (!decode_g_supported(q_heads / c->kv_heads)) return KVQ_ERR_UNSUPPORTED;
  if (workspace_bytes < kvq_decode_step_workspace_bytes(c, dtype, q_heads, max_len)) return KVQ_ERR_WORKSPACE;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  char* ws = static_cast<char*>(workspace);
  const size_t qb = (size_t)c->batch * q_heads * kHeadDim * dtype_size(dtype);
  const size_t mb = (size_t)c->batch * n_buckets(c) * c->kv_heads * sizeof(uint32_t);
  const size_t ob = (size_t)c->batch * q_heads * kHeadDim * sizeof(float);
  void* q_dev = ws;
  uint32_t* mask_dev = reinterpret_cast<uint32_t*>(ws + round_up(qb, kAlign));
  float* out_dev = reinterpret_cast<float*>(ws + round_up(qb, kAlign) + round_up(mb, kAlign));
  void* dec_ws = ws + round_up(qb, kAlign) + round_up(mb, kAlign) + round_up(ob, kAlign);
  if ((st = cuda_status(cudaMemcpyAsync(q_dev, q_host, qb, cudaMemcpyHostToDevice, s))) != KVQ_OK) return st;
  const uint32_t* mask = nullptr;
  if (keep_groups < kPruneGroups) {
    st = kvq_select_channels_at(c, q_dev, dtype, q_heads, seq_lens, keep_groups, mask_dev, stream);
    if (st != KVQ_OK) return st;
    mask = mask_dev;
  }
  const DecodePlan plan = plan_decode(c, q_heads);
  st = enqueue_decode(c, q_dev, dtype, q_heads, seq_lens, max_len, mask, softmax_scale, out_dev, dec_ws, plan, s);
  if (st != KVQ_OK) return st;
  return cuda_status(cudaMemcpyAsync(out_host, out_dev, ob, cudaMemcpyDeviceToHost, s));
}

KVQ_API const char* kvq_status_string(kvq_status s) {
  switch (s) {
    case KVQ_OK: return "ok";
    case KVQ_ERR_INVALID_ARG: return "invalid argument";
    case KVQ_ERR_UNSUPPORTED: return "unsupported configuration";
    case KVQ_ERR_CAPACITY: return "cache capacity exceeded";
    case KVQ_ERR_WORKSPACE: return "workspace too small";
    case KVQ_ERR_CUDA: return "CUDA runtime error";
    case KVQ_ERR_TIMEOUT: return "a bounded wait in a kernel gave up";
  }
  return "unknown status";
}

}  // extern "C"

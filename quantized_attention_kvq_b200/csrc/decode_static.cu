// Decode attention for callers that cannot allocate device memory.
//
// Some callers cannot hand the library a workspace: an engine that owns every
// byte of device memory through its own pool and exposes no allocator across
// the C boundary, or a latency-critical decode loop that must never call
// cudaMalloc (it can synchronize the device and fail under a fixed memory
// budget).  kvq_decode_attention_static serves them: it runs the same split
// decode and combine kernels as kvq_decode_attention, but keeps the per-split
// partials in the fixed device array below instead of a caller workspace.
//
// The array is a file-scope __device__ symbol, so every GPU that loads the
// library holds kScratchBytes of it until the process exits.  Host code cannot
// use the symbol's name as a device address; the address is looked up once
// per device with cudaGetSymbolAddress, with that device current, on the
// first call made on it.
#include <nvtx3/nvToolsExt.h>
#include <mutex>

#include "common.cuh"

namespace kvq {
namespace {

constexpr size_t kScratchBytes = size_t(16) << 20;  // 16 MiB of split partials
constexpr int kMaxDevices = 64;

static __device__ __align__(256) unsigned char g_decode_scratch[kScratchBytes];

std::mutex g_scratch_mutex;
void* g_scratch_ptr[kMaxDevices] = {};

// Device address of g_decode_scratch on the current device (looked up once).
kvq_status scratch_for_current_device(void** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return KVQ_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_scratch_mutex);
  if (!g_scratch_ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_decode_scratch) != cudaSuccess || !p) return KVQ_ERR_CUDA;
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return KVQ_OK;
}

}  // namespace
}  // namespace kvq

extern "C" KVQ_API kvq_status kvq_decode_attention_static(const kvq_cache* cache, const void* q, kvq_dtype dtype,
                                                          int32_t q_heads, const int32_t* seq_lens, int32_t max_len,
                                                          const uint32_t* mask, float softmax_scale, float* out,
                                                          void* stream) {
  struct Range {  // NVTX range named after the call (header-only; a branch when no tool is attached)
    Range() { nvtxRangePushA("kvq_decode_attention_static"); }
    ~Range() { nvtxRangePop(); }
  } range;
  void* scratch = nullptr;
  kvq_status st = kvq::scratch_for_current_device(&scratch);
  if (st != KVQ_OK) return st;
  // sizes whose partials exceed the fixed array are rejected with
  // KVQ_ERR_WORKSPACE before anything is enqueued
  return kvq::decode_into(cache, q, dtype, q_heads, seq_lens, max_len, mask, softmax_scale, out, scratch,
                          kvq::kScratchBytes, static_cast<cudaStream_t>(stream));
}

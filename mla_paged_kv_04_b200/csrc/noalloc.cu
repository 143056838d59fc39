// Allocation-free variant of mla_decode_fwd (see mla_decode_fwd_noalloc in
// include/mla.h).
//
// Some callers cannot hand the library a workspace: code that runs while a
// CUDA graph is being captured (device allocation is not allowed there),
// plugins of inference engines whose enqueue step must not allocate, and
// servers that reserve all device memory up front for their own pool.  For
// them the split-KV workspace (status word + fp32 partial results) lives in a
// fixed-size array in device memory that belongs to this library.
//
// The array is a file-scope __device__ variable, so every GPU that loads the
// library keeps kNoAllocScratchBytes reserved until the process exits.  On the
// host its name is only a stand-in symbol, never a device address: the address
// is looked up once per device with cudaGetSymbolAddress (on the first call
// made while that device is current) and cached.  That first call should
// therefore happen before any stream capture begins.  All calls share the one
// array, so calls that may overlap on the GPU (different streams, different
// host threads) race on it; each call first clears the status word, which is
// the only part that must start at zero.
#include <cuda_runtime.h>

#include <mutex>

#include "../../include/mla.h"
#include "common.cuh"
#include "entry.cuh"

namespace {

constexpr size_t kNoAllocScratchBytes = MLA_NOALLOC_SCRATCH_BYTES;  // 64 MiB per device
constexpr int kMaxDevices = 64;

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

std::mutex g_mutex;
void* g_scratch_ptr[kMaxDevices] = {};

// Device address of this device's scratch array (looked up once per device).
mla_status_t scratch_for_current_device(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return MLA_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return MLA_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_mutex);
  if (g_scratch_ptr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) return MLA_ERR_CUDA;
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return MLA_OK;
}

}  // namespace

extern "C" {

mla_status_t mla_decode_fwd_noalloc(const void* q, const void* kv_cache, mla_kv_format_t fmt, int64_t num_blocks,
                                    const int32_t* block_table, int max_pages, const int32_t* cache_seqlens,
                                    int batch, int s_q, int h_q, float softmax_scale, int causal,
                                    const int32_t* sched, const int32_t* num_splits, int num_sm_parts, void* out,
                                    float* lse, void* stream) {
  // Every host-side check comes before anything is enqueued.
  mla_status_t st = mla::check_decode_args(q, kv_cache, fmt, num_blocks, block_table, max_pages, cache_seqlens,
                                           batch, s_q, h_q, softmax_scale, sched, num_splits, num_sm_parts, out, lse);
  if (st != MLA_OK) return st;
  if (mla::ws_bytes(batch, num_sm_parts, s_q * h_q) > kNoAllocScratchBytes) return MLA_ERR_WORKSPACE;
  if (!mla::current_device_supported()) return MLA_ERR_UNSUPPORTED;
  void* scratch = nullptr;
  st = scratch_for_current_device(&scratch);
  if (st != MLA_OK) return st;
  if (cudaMemsetAsync(scratch, 0, sizeof(int), static_cast<cudaStream_t>(stream)) != cudaSuccess)
    return MLA_ERR_CUDA;
  return mla::launch_decode_call(q, kv_cache, fmt, num_blocks, block_table, max_pages, cache_seqlens, batch, s_q,
                                 h_q, softmax_scale, causal, sched, num_splits, num_sm_parts, out, lse, scratch,
                                 stream);
}

mla_status_t mla_noalloc_last_device_status(void* stream) {
  void* scratch = nullptr;
  mla_status_t st = scratch_for_current_device(&scratch);
  if (st != MLA_OK) return st;
  return mla::read_device_status(scratch, stream);
}

}  // extern "C"

// C-ABI entry points (include/mla.h): argument validation, TMA descriptor
// creation, workspace carving and kernel launches.  No allocation happens
// here; every buffer belongs to the caller.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <atomic>
#include <cmath>
#include <cstdint>
#include <mutex>

#include "../../include/mla.h"
#include "append.cuh"
#include "common.cuh"
#include "entry.cuh"

namespace mla {
cudaError_t launch_metadata(const int32_t* seqlens, int uniform_len, int batch, int rtiles, int parts,
                            int32_t* sched, int32_t* num_splits, cudaStream_t stream);
int metadata_max_batch();
cudaError_t launch_combine(const CombineParams& p, int parts, cudaStream_t stream);
cudaError_t launch_decode_bf16(const CUtensorMap& tm_lat, const CUtensorMap& tm_rope, const DecodeParams& p,
                               int num_parts, cudaStream_t stream);
cudaError_t launch_decode_fp8(const CUtensorMap& tm_lat, const CUtensorMap& tm_scale, const CUtensorMap& tm_rope,
                              const DecodeParams& p, int num_parts, cudaStream_t stream);
cudaError_t launch_decode_sparse_fp8(const CUtensorMap& tm_lat, const CUtensorMap& tm_tail, const DecodeParams& p,
                                     int num_parts, cudaStream_t stream);
}  // namespace mla

using namespace mla;

namespace {

constexpr unsigned long long kDefaultTimeoutNs = 2000000000ull;  // 2 s per wait
constexpr int kMaxTopk = 1 << 24;  // sparse decode: entries per index list

// Limit of every bounded wait in the decode kernel (mla_set_wait_timeout_ns).
std::atomic<unsigned long long> g_timeout_ns{kDefaultTimeoutNs};
// Timestamp buffer of a trace build (mla_debug_set_trace_buffer), else null.
std::atomic<unsigned long long*> g_trace{nullptr};
// mla_debug_hold_at_tile: the flag (null = off) and the tile.
std::mutex g_hold_mutex;
const int* g_hold_flag = nullptr;
int g_hold_tile = -1;

bool aligned(const void* ptr, uintptr_t a) { return (reinterpret_cast<uintptr_t>(ptr) % a) == 0; }

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    cudaDriverEntryPointQueryResult q;
    void* f = nullptr;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(f);
  });
  return fn;
}

// True if the current device is an sm_100 part (the only target built).
bool device_supported() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return false;
  int major = 0, minor = 0;
  if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess) return false;
  if (cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess) return false;
  return major == 10 && minor == 0;
}

// 2-D tiled map over a [rows, width] row-major cache view.
bool make_map(CUtensorMap* map, CUtensorMapDataType dtype, const void* base, uint64_t width, uint64_t rows,
              uint64_t row_bytes, uint32_t box_w, uint32_t box_h, CUtensorMapSwizzle swz) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t gdim[2] = {width, rows};
  cuuint64_t gstride[1] = {row_bytes};
  cuuint32_t box[2] = {box_w, box_h};
  cuuint32_t estride[2] = {1, 1};
  return fn(map, dtype, 2, const_cast<void*>(base), gdim, gstride, box, estride, CU_TENSOR_MAP_INTERLEAVE_NONE, swz,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// batch >= 1, s_q >= 1, h_q >= 1; M = s_q * h_q <= 128 * kMaxRowTiles and
// batch * row_tiles(M) <= the schedule's batch limit.
mla_status_t check_shape(int batch, int s_q, int h_q) {
  if (batch < 1 || s_q < 1 || h_q < 1) return MLA_ERR_INVALID_ARG;
  const long long M = static_cast<long long>(s_q) * h_q;
  if (M > static_cast<long long>(kRows) * kMaxRowTiles) return MLA_ERR_UNSUPPORTED;
  if (static_cast<long long>(batch) * row_tiles(static_cast<int>(M)) > metadata_max_batch())
    return MLA_ERR_UNSUPPORTED;
  return MLA_OK;
}

}  // namespace

namespace mla {

// Synchronises the stream, then maps the status word at `word` (device) to
// an mla_status_t.
mla_status_t read_device_status(const void* word, void* stream) {
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return MLA_ERR_CUDA;
  int status = 0;
  if (cudaMemcpy(&status, word, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) return MLA_ERR_CUDA;
  switch (status) {
    case 0: return MLA_OK;
    case kStatusBadSchedule: return MLA_ERR_INVALID_ARG;
    case kStatusTimeout: return MLA_ERR_TIMEOUT;
    case kStatusBadBlock: return MLA_ERR_BAD_BLOCK_INDEX;
    default: return MLA_ERR_CUDA;
  }
}

}  // namespace mla

extern "C" {

const char* mla_status_string(mla_status_t s) {
  switch (s) {
    case MLA_OK: return "MLA_OK";
    case MLA_ERR_INVALID_ARG: return "MLA_ERR_INVALID_ARG";
    case MLA_ERR_UNSUPPORTED: return "MLA_ERR_UNSUPPORTED";
    case MLA_ERR_WORKSPACE: return "MLA_ERR_WORKSPACE";
    case MLA_ERR_CUDA: return "MLA_ERR_CUDA";
    case MLA_ERR_TIMEOUT: return "MLA_ERR_TIMEOUT";
    case MLA_ERR_BAD_BLOCK_INDEX: return "MLA_ERR_BAD_BLOCK_INDEX";
  }
  return "MLA_ERR_UNKNOWN";
}

int mla_default_num_sm_parts(int device) {
  int sms = 0;
  if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, device) != cudaSuccess) return -1;
  return sms / 2;
}

int mla_num_splits_len(int batch, int s_q, int h_q) {
  if (check_shape(batch, s_q, h_q) != MLA_OK) return 0;
  return batch * row_tiles(s_q * h_q) + 1;
}

size_t mla_metadata_size(int batch, int s_q, int h_q, int num_sm_parts) {
  if (check_shape(batch, s_q, h_q) != MLA_OK || num_sm_parts < 1) return 0;
  return sched_ints(batch * row_tiles(s_q * h_q), num_sm_parts) * sizeof(int32_t);
}

mla_status_t mla_get_metadata(const int32_t* cache_seqlens, int batch, int s_q, int h_q, int num_sm_parts,
                              int32_t* sched, int32_t* num_splits, void* stream) {
  if (!cache_seqlens || !sched || !num_splits) return MLA_ERR_INVALID_ARG;
  if (!aligned(cache_seqlens, 4) || !aligned(sched, 16) || !aligned(num_splits, 4)) return MLA_ERR_INVALID_ARG;
  if (num_sm_parts < 1 || num_sm_parts > 65535) return MLA_ERR_INVALID_ARG;
  mla_status_t st = check_shape(batch, s_q, h_q);
  if (st != MLA_OK) return st;
  const int rt = row_tiles(s_q * h_q);
  cudaError_t e = launch_metadata(cache_seqlens, 0, batch * rt, rt, num_sm_parts, sched, num_splits,
                                  static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? MLA_OK : MLA_ERR_CUDA;
}

size_t mla_workspace_size(int batch, int s_q, int h_q, int num_sm_parts) {
  if (check_shape(batch, s_q, h_q) != MLA_OK || num_sm_parts < 1) return 0;
  return ws_bytes(batch, num_sm_parts, s_q * h_q);
}

}  // extern "C"

namespace mla {

// Everything about a decode call the host can check, except the workspace
// and the device.
mla_status_t check_decode_args(const void* q, const void* kv_cache, mla_kv_format_t fmt, int64_t num_blocks,
                               const int32_t* block_table, int max_pages, const int32_t* cache_seqlens, int batch,
                               int s_q, int h_q, float softmax_scale, const int32_t* sched,
                               const int32_t* num_splits, int num_sm_parts, const void* out, const float* lse) {
  if (!q || !kv_cache || !block_table || !cache_seqlens || !sched || !num_splits || !out || !lse)
    return MLA_ERR_INVALID_ARG;
  if (!aligned(q, 16) || !aligned(kv_cache, 16) || !aligned(out, 16) || !aligned(block_table, 4) ||
      !aligned(cache_seqlens, 4) || !aligned(lse, 4) || !aligned(sched, 16) || !aligned(num_splits, 4))
    return MLA_ERR_INVALID_ARG;
  if (fmt != MLA_KV_BF16 && fmt != MLA_KV_FP8_656) return MLA_ERR_INVALID_ARG;
  if (num_blocks < 1 || num_blocks > (static_cast<int64_t>(1) << 31) / kPage) return MLA_ERR_INVALID_ARG;
  if (max_pages < 1 || num_sm_parts < 1 || num_sm_parts > 65535) return MLA_ERR_INVALID_ARG;
  if (!std::isfinite(softmax_scale)) return MLA_ERR_INVALID_ARG;
  return check_shape(batch, s_q, h_q);
}

bool current_device_supported() { return device_supported(); }

// Enqueues the decode and combine kernels of a call whose arguments passed
// check_decode_args and whose workspace holds ws_bytes(batch, parts, M).
mla_status_t launch_decode_call(const void* q, const void* kv_cache, mla_kv_format_t fmt, int64_t num_blocks,
                                const int32_t* block_table, int max_pages, const int32_t* cache_seqlens, int batch,
                                int s_q, int h_q, float softmax_scale, int causal, const int32_t* sched,
                                const int32_t* num_splits, int num_sm_parts, void* out, float* lse, void* workspace,
                                void* stream) {
  const int M = s_q * h_q;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  DecodeParams p{};
  p.q = static_cast<const uint16_t*>(q);
  p.block_table = block_table;
  p.seqlens = cache_seqlens;
  p.sched = sched;
  p.out = static_cast<uint16_t*>(out);
  p.lse = lse;
  p.lse_part = reinterpret_cast<float*>(ws + ws_lse_offset());
  p.o_part = reinterpret_cast<float*>(ws + ws_o_offset(batch, num_sm_parts, M));
  p.status = reinterpret_cast<int*>(ws);
  p.num_blocks = num_blocks;
  p.max_pages = max_pages;
  p.batch = batch;
  p.s_q = s_q;
  p.h_q = h_q;
  p.M = M;
  p.row_tiles = row_tiles(M);
  p.causal = causal ? 1 : 0;
  p.num_parts = num_sm_parts;
  p.scale_log2 = static_cast<float>(static_cast<double>(softmax_scale) * 1.4426950408889634);
  p.req_div = 1;
  p.req_batch = batch;
  p.q_wide = aligned(q, 32) ? 1 : 0;
  p.out_wide = (aligned(out, 32) && aligned(p.o_part, 32)) ? 1 : 0;
  p.timeout_ns = g_timeout_ns.load(std::memory_order_relaxed);
  p.trace = g_trace.load(std::memory_order_relaxed);
  {
    std::lock_guard<std::mutex> lock(g_hold_mutex);
    p.hold_flag = g_hold_flag;
    p.hold_tile = g_hold_tile;
  }

  const uint64_t rows = static_cast<uint64_t>(num_blocks) * kPage;
  CUtensorMap tm_a, tm_b, tm_c;
  cudaError_t e;
  if (fmt == MLA_KV_BF16) {
    if (!make_map(&tm_a, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, kv_cache, kDqk, rows, kDqk * 2, 64, kPage,
                  CU_TENSOR_MAP_SWIZZLE_128B) ||
        !make_map(&tm_b, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, kv_cache, kDqk, rows, kDqk * 2, 32, kPage,
                  CU_TENSOR_MAP_SWIZZLE_64B))
      return MLA_ERR_CUDA;
    e = launch_decode_bf16(tm_a, tm_b, p, num_sm_parts, s);
  } else {
    // raw bytes of a token: a latent half (256 B), the four scales (16 B), a RoPE half (64 B)
    if (!make_map(&tm_a, CU_TENSOR_MAP_DATA_TYPE_UINT8, kv_cache, kFp8TokenBytes, rows, kFp8TokenBytes, 256, kPage,
                  CU_TENSOR_MAP_SWIZZLE_NONE) ||
        !make_map(&tm_b, CU_TENSOR_MAP_DATA_TYPE_UINT8, kv_cache, kFp8TokenBytes, rows, kFp8TokenBytes, 16, kPage,
                  CU_TENSOR_MAP_SWIZZLE_NONE) ||
        !make_map(&tm_c, CU_TENSOR_MAP_DATA_TYPE_UINT8, kv_cache, kFp8TokenBytes, rows, kFp8TokenBytes, 64, kPage,
                  CU_TENSOR_MAP_SWIZZLE_NONE))
      return MLA_ERR_CUDA;
    e = launch_decode_fp8(tm_a, tm_b, tm_c, p, num_sm_parts, s);
  }
  if (e != cudaSuccess) return MLA_ERR_CUDA;

  CombineParams c{};
  c.sched = sched;
  c.num_splits = num_splits;
  c.lse_part = p.lse_part;
  c.o_part = p.o_part;
  c.out = p.out;
  c.lse = lse;
  c.batch = batch;
  c.M = M;
  c.row_tiles = row_tiles(M);
  c.num_parts = num_sm_parts;
  e = launch_combine(c, num_sm_parts, s);
  return e == cudaSuccess ? MLA_OK : MLA_ERR_CUDA;
}

}  // namespace mla

extern "C" {

mla_status_t mla_decode_fwd(const void* q, const void* kv_cache, mla_kv_format_t fmt, int64_t num_blocks,
                            const int32_t* block_table, int max_pages, const int32_t* cache_seqlens, int batch,
                            int s_q, int h_q, float softmax_scale, int causal, const int32_t* sched,
                            const int32_t* num_splits, int num_sm_parts, void* out, float* lse, void* workspace,
                            size_t workspace_bytes, void* stream) {
  if (!workspace || !aligned(workspace, 256)) return MLA_ERR_INVALID_ARG;
  mla_status_t st = check_decode_args(q, kv_cache, fmt, num_blocks, block_table, max_pages, cache_seqlens, batch,
                                      s_q, h_q, softmax_scale, sched, num_splits, num_sm_parts, out, lse);
  if (st != MLA_OK) return st;
  if (workspace_bytes < ws_bytes(batch, num_sm_parts, s_q * h_q)) return MLA_ERR_WORKSPACE;
  if (!device_supported()) return MLA_ERR_UNSUPPORTED;
  return launch_decode_call(q, kv_cache, fmt, num_blocks, block_table, max_pages, cache_seqlens, batch, s_q, h_q,
                            softmax_scale, causal, sched, num_splits, num_sm_parts, out, lse, workspace, stream);
}

int mla_sparse_num_splits_len(int batch, int s_q, int h_q) {
  if (batch < 1 || s_q < 1 || static_cast<long long>(batch) * s_q > (1 << 30)) return 0;
  return mla_num_splits_len(batch * s_q, 1, h_q);
}

size_t mla_sparse_metadata_size(int batch, int s_q, int h_q, int num_sm_parts) {
  if (batch < 1 || s_q < 1 || static_cast<long long>(batch) * s_q > (1 << 30)) return 0;
  return mla_metadata_size(batch * s_q, 1, h_q, num_sm_parts);
}

size_t mla_sparse_workspace_size(int batch, int s_q, int h_q, int num_sm_parts) {
  if (batch < 1 || s_q < 1 || static_cast<long long>(batch) * s_q > (1 << 30)) return 0;
  return mla_workspace_size(batch * s_q, 1, h_q, num_sm_parts);
}

mla_status_t mla_get_sparse_metadata(int batch, int s_q, int h_q, int topk, int num_sm_parts, int32_t* sched,
                                     int32_t* num_splits, void* stream) {
  if (!sched || !num_splits || !aligned(sched, 16) || !aligned(num_splits, 4)) return MLA_ERR_INVALID_ARG;
  if (num_sm_parts < 1 || num_sm_parts > 65535 || topk < 1 || topk > kMaxTopk) return MLA_ERR_INVALID_ARG;
  if (batch < 1 || s_q < 1) return MLA_ERR_INVALID_ARG;
  if (static_cast<long long>(batch) * s_q > (1 << 30)) return MLA_ERR_UNSUPPORTED;
  const int units = batch * s_q;
  mla_status_t st = check_shape(units, 1, h_q);
  if (st != MLA_OK) return st;
  const int rt = row_tiles(h_q);
  cudaError_t e = launch_metadata(nullptr, topk, units * rt, rt, num_sm_parts, sched, num_splits,
                                  static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? MLA_OK : MLA_ERR_CUDA;
}

mla_status_t mla_sparse_decode_fwd(const void* q, const void* kv_cache, int64_t num_blocks,
                                   const int32_t* block_table, int max_pages, const int32_t* cache_seqlens,
                                   const int32_t* indices, int topk, int batch, int s_q, int h_q, float softmax_scale,
                                   const int32_t* sched, const int32_t* num_splits, int num_sm_parts, void* out,
                                   float* lse, void* workspace, size_t workspace_bytes, void* stream) {
  if (!indices || !aligned(indices, 4) || topk < 1 || topk > kMaxTopk) return MLA_ERR_INVALID_ARG;
  if (!workspace || !aligned(workspace, 256)) return MLA_ERR_INVALID_ARG;
  if (batch < 1 || s_q < 1) return MLA_ERR_INVALID_ARG;
  if (static_cast<long long>(batch) * s_q > (1 << 30)) return MLA_ERR_UNSUPPORTED;
  const int units = batch * s_q;
  // the unit checks of a dense call with `units` requests of h_q rows
  mla_status_t st = check_decode_args(q, kv_cache, MLA_KV_FP8_656, num_blocks, block_table, max_pages,
                                      cache_seqlens, units, 1, h_q, softmax_scale, sched, num_splits, num_sm_parts,
                                      out, lse);
  if (st != MLA_OK) return st;
  if (workspace_bytes < ws_bytes(units, num_sm_parts, h_q)) return MLA_ERR_WORKSPACE;
  if (!device_supported()) return MLA_ERR_UNSUPPORTED;

  cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  DecodeParams p{};
  p.q = static_cast<const uint16_t*>(q);
  p.block_table = block_table;
  p.seqlens = cache_seqlens;
  p.sched = sched;
  p.out = static_cast<uint16_t*>(out);
  p.lse = lse;
  p.lse_part = reinterpret_cast<float*>(ws + ws_lse_offset());
  p.o_part = reinterpret_cast<float*>(ws + ws_o_offset(units, num_sm_parts, h_q));
  p.status = reinterpret_cast<int*>(ws);
  p.num_blocks = num_blocks;
  p.max_pages = max_pages;
  p.batch = units;
  p.s_q = 1;
  p.h_q = h_q;
  p.M = h_q;
  p.row_tiles = row_tiles(h_q);
  p.causal = 0;
  p.num_parts = num_sm_parts;
  p.scale_log2 = static_cast<float>(static_cast<double>(softmax_scale) * 1.4426950408889634);
  p.req_div = s_q;
  p.req_batch = batch;
  p.indices = indices;
  p.topk = topk;
  p.q_wide = aligned(q, 32) ? 1 : 0;
  p.out_wide = (aligned(out, 32) && aligned(p.o_part, 32)) ? 1 : 0;
  p.timeout_ns = g_timeout_ns.load(std::memory_order_relaxed);
  p.trace = g_trace.load(std::memory_order_relaxed);
  {
    std::lock_guard<std::mutex> lock(g_hold_mutex);
    p.hold_flag = g_hold_flag;
    p.hold_tile = g_hold_tile;
  }
  // one-row boxes for the TMA row gathers: this CTA's latent half (256 bytes)
  // and bytes [496, 656) of the token
  const uint64_t rows = static_cast<uint64_t>(num_blocks) * kPage;
  CUtensorMap tm_lat, tm_tail;
  if (!make_map(&tm_lat, CU_TENSOR_MAP_DATA_TYPE_UINT8, kv_cache, kFp8TokenBytes, rows, kFp8TokenBytes, 256, 1,
                CU_TENSOR_MAP_SWIZZLE_NONE) ||
      !make_map(&tm_tail, CU_TENSOR_MAP_DATA_TYPE_UINT8, kv_cache, kFp8TokenBytes, rows, kFp8TokenBytes, 160, 1,
                CU_TENSOR_MAP_SWIZZLE_NONE))
    return MLA_ERR_CUDA;
  cudaError_t e = launch_decode_sparse_fp8(tm_lat, tm_tail, p, num_sm_parts, s);
  if (e != cudaSuccess) return MLA_ERR_CUDA;
  CombineParams c{};
  c.sched = sched;
  c.num_splits = num_splits;
  c.lse_part = p.lse_part;
  c.o_part = p.o_part;
  c.out = p.out;
  c.lse = lse;
  c.batch = units;
  c.M = h_q;
  c.row_tiles = p.row_tiles;
  c.num_parts = num_sm_parts;
  e = launch_combine(c, num_sm_parts, s);
  return e == cudaSuccess ? MLA_OK : MLA_ERR_CUDA;
}

mla_status_t mla_kv_append(const void* kv_new, int batch, int s_new, const int32_t* cache_seqlens,
                           const int32_t* block_table, int max_pages, void* kv_cache, mla_kv_format_t fmt,
                           int64_t num_blocks, void* workspace, size_t workspace_bytes, void* stream) {
  if (!kv_new || !cache_seqlens || !block_table || !kv_cache || !workspace) return MLA_ERR_INVALID_ARG;
  if (!aligned(kv_new, 16) || !aligned(kv_cache, 16) || !aligned(block_table, 4) || !aligned(cache_seqlens, 4) ||
      !aligned(workspace, 4))
    return MLA_ERR_INVALID_ARG;
  if (fmt != MLA_KV_BF16 && fmt != MLA_KV_FP8_656) return MLA_ERR_INVALID_ARG;
  if (batch < 1 || s_new < 1 || max_pages < 1) return MLA_ERR_INVALID_ARG;
  if (num_blocks < 1 || num_blocks > (static_cast<int64_t>(1) << 31) / kPage) return MLA_ERR_INVALID_ARG;
  // one warp per token, eight per block: the grid stays below 2^31 blocks
  const long long tokens = static_cast<long long>(batch) * s_new;
  if (tokens > (static_cast<long long>(1) << 33)) return MLA_ERR_UNSUPPORTED;
  if (workspace_bytes < sizeof(int)) return MLA_ERR_WORKSPACE;
  if (!device_supported()) return MLA_ERR_UNSUPPORTED;
  AppendParams p{};
  p.kv_new = static_cast<const uint16_t*>(kv_new);
  p.block_table = block_table;
  p.seqlens = cache_seqlens;
  p.kv_cache = static_cast<uint8_t*>(kv_cache);
  p.status = static_cast<int*>(workspace);
  p.num_blocks = num_blocks;
  p.tokens = tokens;
  p.max_pages = max_pages;
  p.s_new = s_new;
  p.fp8 = fmt == MLA_KV_FP8_656 ? 1 : 0;
  return launch_append(p, static_cast<cudaStream_t>(stream)) == cudaSuccess ? MLA_OK : MLA_ERR_CUDA;
}

mla_status_t mla_last_device_status(const void* workspace, void* stream) {
  if (!workspace) return MLA_ERR_INVALID_ARG;
  return read_device_status(workspace, stream);
}

uint64_t mla_set_wait_timeout_ns(uint64_t ns) {
  return g_timeout_ns.exchange(ns == 0 ? kDefaultTimeoutNs : ns);
}

size_t mla_debug_trace_bytes(void) { return kTraceBytes; }

mla_status_t mla_debug_hold_at_tile(const int* flag, int tile) {
  if (flag != nullptr && !aligned(flag, 4)) return MLA_ERR_INVALID_ARG;
  std::lock_guard<std::mutex> lock(g_hold_mutex);
  g_hold_flag = (tile < 0) ? nullptr : flag;
  g_hold_tile = (flag == nullptr) ? -1 : tile;
  return MLA_OK;
}

mla_status_t mla_debug_set_trace_buffer(void* buffer, size_t bytes) {
#ifdef MLA_TRACE
  if (buffer != nullptr && (bytes < kTraceBytes || !aligned(buffer, 8))) return MLA_ERR_INVALID_ARG;
  g_trace.store(static_cast<unsigned long long*>(buffer));
  return MLA_OK;
#else
  (void)buffer;
  (void)bytes;
  return MLA_ERR_UNSUPPORTED;
#endif
}

mla_status_t mla_clear_device_status(void* workspace, void* stream) {
  if (!workspace) return MLA_ERR_INVALID_ARG;
  return cudaMemsetAsync(workspace, 0, sizeof(int), static_cast<cudaStream_t>(stream)) == cudaSuccess
             ? MLA_OK
             : MLA_ERR_CUDA;
}

}  // extern "C"

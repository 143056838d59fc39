// Host-side pieces shared by the C-ABI entry points (api.cu, noalloc.cu).
#pragma once

#include <cstdint>

#include "../../include/mla.h"

namespace mla {

// Every argument of a decode call the host can check, except the workspace
// and the device: MLA_OK, MLA_ERR_INVALID_ARG or MLA_ERR_UNSUPPORTED.
mla_status_t check_decode_args(const void* q, const void* kv_cache, mla_kv_format_t fmt, int64_t num_blocks,
                               const int32_t* block_table, int max_pages, const int32_t* cache_seqlens, int batch,
                               int s_q, int h_q, float softmax_scale, const int32_t* sched,
                               const int32_t* num_splits, int num_sm_parts, const void* out, const float* lse);

// True if the current device is an sm_100 part.
bool current_device_supported();

// Enqueues the decode and combine kernels of a call that passed
// check_decode_args, with a workspace of at least ws_bytes(batch, parts, M)
// bytes (256-byte aligned) whose status word the kernels report into.
mla_status_t launch_decode_call(const void* q, const void* kv_cache, mla_kv_format_t fmt, int64_t num_blocks,
                                const int32_t* block_table, int max_pages, const int32_t* cache_seqlens, int batch,
                                int s_q, int h_q, float softmax_scale, int causal, const int32_t* sched,
                                const int32_t* num_splits, int num_sm_parts, void* out, float* lse, void* workspace,
                                void* stream);

// Synchronises `stream`, then maps the device status word at `word` to an
// mla_status_t.
mla_status_t read_device_status(const void* word, void* stream);

}  // namespace mla

// Parameters and launcher of the cache-append kernel (append.cu), shared with
// the C-ABI layer (api.cu).
#pragma once

#include <cuda_runtime.h>

#include <cstdint>

namespace mla {

struct AppendParams {
  const uint16_t* kv_new;      // bf16 [batch, s_new, 576]
  const int32_t* block_table;  // [batch, max_pages]
  const int32_t* seqlens;      // [batch]: lengths after the append
  uint8_t* kv_cache;           // [num_blocks, 64, 1152 or 656 bytes]
  int* status;                 // workspace status word
  long long num_blocks;
  long long tokens;            // batch * s_new
  int max_pages;
  int s_new;
  int fp8;
};

cudaError_t launch_append(const AppendParams& p, cudaStream_t stream);

}  // namespace mla

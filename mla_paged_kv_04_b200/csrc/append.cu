// Cache append on sm_100a: new tokens into the paged KV cache.
//
// The step that fills what the decode kernel reads: token t of request b (of
// s_new new tokens, cache_seqlens[b] = L_b counting them) is token
// p = L_b - s_new + t of the request and goes to slot p % 64 of physical
// block block_table[b, p / 64].  BF16 rows are stored as they are; FP8 rows
// are quantised into the 656-byte layout (the size on the menfem.com DeepSeek
// page, "Key Contributions", with the RoPE slice kept in BF16): per 128-wide
// latent group, scale = amax / 448 and code = E4M3 round-to-nearest-even of
// x / scale with saturation, both divisions IEEE binary32; a group with
// amax 0 gets scale 0 and codes 0.
//
// One warp per new token.  The work is a row copy (1,152 bytes in; 1,152 or
// 656 bytes out), so the kernel is bound by HBM bandwidth and launch latency:
// every lane moves 16-byte words, and the FP8 path keeps its arithmetic
// (a max over 16 values, an 8-lane shuffle reduction, 16 divisions and
// conversions per lane) in registers.
#include <cuda_fp8.h>
#include <cuda_runtime.h>

#include "append.cuh"
#include "common.cuh"

namespace mla {

namespace {

constexpr int kAppendWarps = 8;  // tokens per block

__global__ void __launch_bounds__(kAppendWarps * 32) append_kernel(const AppendParams p) {
  const int lane = threadIdx.x & 31;
  const long long tok = static_cast<long long>(blockIdx.x) * kAppendWarps + (threadIdx.x >> 5);
  if (tok >= p.tokens) return;
  const int b = static_cast<int>(tok / p.s_new);
  const int t = static_cast<int>(tok % p.s_new);
  const int pos = p.seqlens[b] - p.s_new + t;
  if (pos < 0) {  // more new tokens than the request's length: reported as MLA_ERR_INVALID_ARG
    if (lane == 0) report_status(p.status, kStatusBadSchedule);
    return;
  }
  const int page = pos / kPage;
  const long long phys = page < p.max_pages ? p.block_table[static_cast<size_t>(b) * p.max_pages + page] : -1;
  if (phys < 0 || phys >= p.num_blocks) {
    if (lane == 0) report_status(p.status, kStatusBadBlock);
    return;
  }
  const size_t row = static_cast<size_t>(phys) * kPage + (pos % kPage);
  const uint4* src = reinterpret_cast<const uint4*>(p.kv_new + static_cast<size_t>(tok) * kDqk);
  if (!p.fp8) {
    uint4* dst = reinterpret_cast<uint4*>(p.kv_cache + row * (kDqk * 2));
    for (int i = lane; i < kDqk * 2 / 16; i += 32) dst[i] = __ldg(src + i);  // 72 words of 16 bytes
    return;
  }
  uint8_t* dst = p.kv_cache + row * kFp8TokenBytes;
  // Lane l quantises latent dims [16 l, 16 l + 16): group l / 8.
  const uint4 w0 = __ldg(src + 2 * lane), w1 = __ldg(src + 2 * lane + 1);
  const uint32_t w[8] = {w0.x, w0.y, w0.z, w0.w, w1.x, w1.y, w1.z, w1.w};
  float x[16];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    x[2 * i] = __uint_as_float(w[i] << 16);  // bf16 -> fp32 is exact
    x[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
  }
  float amax = 0.f;
#pragma unroll
  for (int i = 0; i < 16; ++i) amax = fmaxf(amax, fabsf(x[i]));
#pragma unroll
  for (int o = 1; o < 8; o <<= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
  const float scale = amax / 448.0f;  // IEEE binary32 division (no fast-math in this build)
  uint32_t c[4] = {0u, 0u, 0u, 0u};
  if (scale > 0.f) {
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      const uint32_t code = __nv_cvt_float_to_fp8(x[i] / scale, __NV_SATFINITE, __NV_E4M3);
      c[i >> 2] |= code << (8 * (i & 3));  // byte i of the 16 is dim 16 l + i
    }
  }
  *reinterpret_cast<uint4*>(dst + 16 * lane) = make_uint4(c[0], c[1], c[2], c[3]);
  if ((lane & 7) == 0) *reinterpret_cast<float*>(dst + kDv + 4 * (lane >> 3)) = scale;
  // RoPE: source bytes [1024, 1152) -> cache bytes [528, 656), eight 16-byte words
  if (lane < 8) *reinterpret_cast<uint4*>(dst + kDv + 16 + 16 * lane) = __ldg(src + 64 + lane);
}

}  // namespace

cudaError_t launch_append(const AppendParams& p, cudaStream_t stream) {
  const long long blocks = (p.tokens + kAppendWarps - 1) / kAppendWarps;
  append_kernel<<<static_cast<unsigned>(blocks), kAppendWarps * 32, 0, stream>>>(p);
  return cudaGetLastError();
}

}  // namespace mla

// Split-KV combine: merges the fp32 partial outputs of a split request.
//   lse = ln sum_s e^{lse_s},   out = sum_s e^{lse_s - lse} * o_s   (bf16 RNE)
// Splits with lse_s = -inf (no visible key, or a zero-page split) get no
// weight and their partial output is not read.  Each lane of a warp owns 16
// of the 512 output columns of one query row (four 16-byte loads per split).
#include <cuda_runtime.h>
#include <math_constants.h>

#include "common.cuh"

namespace mla {

constexpr int kCombineWarps = 8;
constexpr int kCombineRowsPerBlock = 32;

// grid.x walks the schedule's list of split requests (at most one per CTA
// pair), grid.y covers the query rows 32 at a time; eight warps per block,
// one query row per warp at a time.
__global__ void __launch_bounds__(32 * kCombineWarps) combine_kernel(const CombineParams p) {
  if (p.sched[0] != p.num_parts) return;  // reported by the decode kernel
  const int num_split_req = p.sched[5];
  if (static_cast<int>(blockIdx.x) >= num_split_req) return;
  const int parts = p.sched[0];
  const int b = p.sched[sched_split_list_offset(parts) + blockIdx.x];
  const int first = p.num_splits[b];
  const int nsplit = p.num_splits[b + 1] - first;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int rr = warp; rr < kCombineRowsPerBlock; rr += kCombineWarps) {
  const int r = blockIdx.y * kCombineRowsPerBlock + rr;
  if (r >= p.M) break;

  float m = -CUDART_INF_F;
  for (int s = lane; s < nsplit; s += 32) m = fmaxf(m, p.lse_part[static_cast<size_t>(first + s) * p.M + r]);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));

  float acc[16];
#pragma unroll
  for (int i = 0; i < 16; ++i) acc[i] = 0.f;
  float wsum = 0.f;
  if (m != -CUDART_INF_F) {
    for (int s = 0; s < nsplit; ++s) {
      const size_t row = static_cast<size_t>(first + s) * p.M + r;
      const float ls = p.lse_part[row];
      if (ls == -CUDART_INF_F) continue;
      const float w = expf(ls - m);
      wsum += w;
      const float4* src = reinterpret_cast<const float4*>(p.o_part + row * kDv) + lane * 4;
#pragma unroll
      for (int v = 0; v < 4; ++v) {
        float4 x = src[v];
        acc[4 * v + 0] += w * x.x;
        acc[4 * v + 1] += w * x.y;
        acc[4 * v + 2] += w * x.z;
        acc[4 * v + 3] += w * x.w;
      }
    }
  }
  const float inv = wsum > 0.f ? 1.f / wsum : 0.f;
  uint32_t packed[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    uint32_t r2;
    asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r2) : "f"(acc[2 * i + 1] * inv), "f"(acc[2 * i] * inv));
    packed[i] = r2;
  }
  uint4* dst = reinterpret_cast<uint4*>(p.out + (static_cast<size_t>(b) * p.M + r) * kDv + lane * 16);
  dst[0] = make_uint4(packed[0], packed[1], packed[2], packed[3]);
  dst[1] = make_uint4(packed[4], packed[5], packed[6], packed[7]);
  if (lane == 0) p.lse[static_cast<size_t>(b) * p.M + r] = wsum > 0.f ? m + logf(wsum) : -CUDART_INF_F;
  }
}

cudaError_t launch_combine(const CombineParams& p, int parts, cudaStream_t stream) {
  dim3 grid(parts, (p.M + kCombineRowsPerBlock - 1) / kCombineRowsPerBlock);
  combine_kernel<<<grid, 32 * kCombineWarps, 0, stream>>>(p);
  return cudaGetLastError();
}

}  // namespace mla

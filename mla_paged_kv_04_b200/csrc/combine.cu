// Split-KV combine: merges the fp32 partial outputs of a split request.
//   lse = ln sum_s e^{lse_s},   out = sum_s e^{lse_s - lse} * o_s   (bf16 RNE)
// Splits with lse_s = -inf (no visible key, or a zero-page split) get no
// weight and their partial output is not read.  Each lane of a warp owns 16
// of the 512 output columns of one query row (four 16-byte loads per split).
// Summation order: the splits in index order per lane, so the result does not
// depend on timing.
#include <cuda_runtime.h>
#include <math_constants.h>

#include "common.cuh"
#include "sm100.cuh"

namespace mla {

constexpr int kCombineWarps = 4;  // one query row per warp
constexpr int kCombineUnroll = 4;  // splits whose partial rows are in flight at once

// Merges row r of split virtual request vb (one warp).
__device__ __forceinline__ void combine_row(const CombineParams& p, int vb, int r, int mt, int lane) {
  const int b = vb / p.row_tiles, row0 = (vb - b * p.row_tiles) * kRows;
  const int first = p.num_splits[vb];
  const int nsplit = p.num_splits[vb + 1] - first;
  if (r >= mt || row0 + r >= p.M) return;

  float m = -CUDART_INF_F;
  for (int s = lane; s < nsplit; s += 32) m = fmaxf(m, p.lse_part[static_cast<size_t>(first + s) * mt + r]);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));

  float acc[16];
#pragma unroll
  for (int i = 0; i < 16; ++i) acc[i] = 0.f;
  float wsum = 0.f;  // this lane's splits; reduced over the warp below
  if (m != -CUDART_INF_F) {
    for (int s0 = 0; s0 < nsplit; s0 += 32) {
      float w = 0.f;
      if (s0 + lane < nsplit) {
        const float ls = p.lse_part[static_cast<size_t>(first + s0 + lane) * mt + r];
        w = (ls == -CUDART_INF_F) ? 0.f : expf(ls - m);
      }
      wsum += w;
      const int cnt = min(32, nsplit - s0);
      for (int k = 0; k < cnt; k += kCombineUnroll) {
        float wk[kCombineUnroll];
        float4 x[kCombineUnroll][4];
#pragma unroll
        for (int u = 0; u < kCombineUnroll; ++u) {
          wk[u] = __shfl_sync(0xffffffffu, w, (k + u) & 31);
          if (k + u >= cnt) wk[u] = 0.f;
          const float4* src =
              reinterpret_cast<const float4*>(p.o_part + (static_cast<size_t>(first + s0 + k + u) * mt + r) * kDv) +
              lane * 4;
#pragma unroll
          for (int v = 0; v < 4; ++v) x[u][v] = wk[u] != 0.f ? src[v] : make_float4(0.f, 0.f, 0.f, 0.f);
        }
#pragma unroll
        for (int u = 0; u < kCombineUnroll; ++u) {
#pragma unroll
          for (int v = 0; v < 4; ++v) {
            acc[4 * v + 0] += wk[u] * x[u][v].x;
            acc[4 * v + 1] += wk[u] * x[u][v].y;
            acc[4 * v + 2] += wk[u] * x[u][v].z;
            acc[4 * v + 3] += wk[u] * x[u][v].w;
          }
        }
      }
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) wsum += __shfl_xor_sync(0xffffffffu, wsum, o);
  const float inv = wsum > 0.f ? 1.f / wsum : 0.f;
  uint32_t packed[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    uint32_t r2;
    asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r2) : "f"(acc[2 * i + 1] * inv), "f"(acc[2 * i] * inv));
    packed[i] = r2;
  }
  const size_t orow = static_cast<size_t>(b) * p.M + row0 + r;
  uint4* dst = reinterpret_cast<uint4*>(p.out + orow * kDv + lane * 16);
  dst[0] = make_uint4(packed[0], packed[1], packed[2], packed[3]);
  dst[1] = make_uint4(packed[4], packed[5], packed[6], packed[7]);
  if (lane == 0) p.lse[orow] = wsum > 0.f ? m + logf(wsum) : -CUDART_INF_F;
}

// At most this many blocks: when no request is split (whole-request
// schedules) the kernel's cost is its launch and drain, which grows with the
// grid; otherwise blocks loop over the work.
constexpr int kCombineMaxBlocks = 4 * 148;

// One work unit per (split virtual request, group of kCombineWarps query
// rows), one row per warp; blocks take units blockIdx.x, blockIdx.x +
// gridDim.x, ...  Lane s holds split s's weight (in chunks of 32 splits); the
// partial rows of kCombineUnroll splits are loaded together so that their
// latencies overlap.
__global__ void __launch_bounds__(32 * kCombineWarps) combine_kernel(const CombineParams p) {
  pdl_wait();  // the decode kernel has completed
  // a schedule made for another CTA-pair count or batch: reported by the
  // decode kernel, nothing to merge
  if (p.sched[0] != p.num_parts || p.sched[3] != p.batch * p.row_tiles || p.sched[7] != p.row_tiles) return;
  const int num_split_req = p.sched[5];
  const int parts = p.sched[0];
  const int mt = rows_per_tile(p.M);  // partial rows per slot
  const int groups = (mt + kCombineWarps - 1) / kCombineWarps;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int unit = blockIdx.x; unit < num_split_req * groups; unit += gridDim.x) {
    const int vb = p.sched[sched_split_list_offset(parts) + unit / groups];  // virtual request
    const int r = (unit % groups) * kCombineWarps + warp;                     // row within the row tile
    combine_row(p, vb, r, mt, lane);
  }
}

cudaError_t launch_combine(const CombineParams& p, int parts, cudaStream_t stream) {
  cudaLaunchConfig_t cfg = {};
  const int units = parts * ((rows_per_tile(p.M) + kCombineWarps - 1) / kCombineWarps);  // upper bound
  cfg.gridDim = dim3(units < kCombineMaxBlocks ? units : kCombineMaxBlocks);
  cfg.blockDim = dim3(32 * kCombineWarps);
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;  // overlaps the decode kernel's tail
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, combine_kernel, p);
}

}  // namespace mla

// Split-KV schedule for variable-length batches, computed on the device by a
// single block (one thread per request, up to 1024) so that it stays on the
// caller's stream.
//
// Cost model: request b costs n_b + c units, n_b = ceil(L_b / 64) pages and
// c = kSplitOverheadPages.  The requests' cost intervals are laid end to end
// (exclusive prefix C_b) and the line [0, T) is cut into pieces of
// t = ceil(T / parts) units; piece k belongs to CTA pair ("part") k.  A
// request crossing a cut is split there: split s of request b covers the
// virtual range [max(C_b, k t), min(C_b + cost_b, (k + 1) t)) - C_b with
// k = floor(C_b / t) + s; the first c virtual units of a request stand for
// its fixed cost, so virtual position v maps to page clamp(v - c, 0, n_b).
// A split may therefore hold zero pages; the decode kernel then only writes
// lse = -inf for it and the combine kernel gives it no weight.
//
// Whole-request mode: part k serves the m = ceil(batch / parts) requests
// [k m, k m + m) whole (parts past the batch stay idle) and nothing is split,
// when the costliest part is at most kSplitPenaltyPages above t.  (m = 1
// when the batch fits the parts; m > 1 pays off for many equal requests,
// such as the sparse decode's lists, where the balanced cut would split
// nearly every request.)
//
// Requests with more than 128 query rows: everything above is over virtual
// requests v = b * row_tiles + tile, each with the length of request b, so
// "batch" below is the virtual batch and v's length is seqlens[v / row_tiles].
// With seqlens == nullptr every virtual request has the length uniform_len
// (the sparse decode: each query token attends to a list of topk entries).
#include <cuda_runtime.h>

#include "common.cuh"

namespace mla {

constexpr int kMetaThreads = 1024;
constexpr int kMaxBatch = 16384;

__device__ __forceinline__ int block_exclusive_scan(int v, int* warp_sums, int* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  const int nwarps = static_cast<int>(blockDim.x) >> 5;
  if (lane == 31) warp_sums[warp] = x;
  __syncthreads();
  if (warp == 0) {
    int w = (lane < nwarps) ? warp_sums[lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      int y = __shfl_up_sync(0xffffffffu, w, o);
      if (lane >= o) w += y;
    }
    warp_sums[lane] = w;  // inclusive
  }
  __syncthreads();
  int prefix = x - v + (warp > 0 ? warp_sums[warp - 1] : 0);
  *total = warp_sums[nwarps - 1];
  __syncthreads();
  return prefix;
}

__device__ __forceinline__ int block_max(int v, int* warp_sums) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int nwarps = static_cast<int>(blockDim.x) >> 5;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = max(v, __shfl_xor_sync(0xffffffffu, v, o));
  if (lane == 0) warp_sums[warp] = v;
  __syncthreads();
  int m = 0;
  for (int w = 0; w < nwarps; ++w) m = max(m, warp_sums[w]);
  __syncthreads();
  return m;
}

__global__ void __launch_bounds__(kMetaThreads) metadata_kernel(const int32_t* __restrict__ seqlens,
                                                                int uniform_len, int batch, int rtiles, int parts,
                                                                int overhead, int32_t* __restrict__ sched,
                                                                int32_t* __restrict__ num_splits) {
  // the decode kernel may begin launching (it waits for this grid to complete)
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  extern __shared__ int sm[];
  int* C = sm;                 // [batch + 1] cost prefix
  int* S = sm + batch + 1;     // [batch + 1] split prefix
  __shared__ int warp_sums[32];

  const int per = (batch + static_cast<int>(blockDim.x) - 1) / static_cast<int>(blockDim.x);
  const int b0 = threadIdx.x * per;
  const int b1 = min(batch, b0 + per);

  // 1. cost prefix
  int local = 0;
  for (int b = b0; b < b1; ++b) {
    int L = (seqlens ? max(seqlens[b / rtiles], 0) : uniform_len);
    local += (L + kPage - 1) / kPage + overhead;
  }
  int T;
  int run = block_exclusive_scan(local, warp_sums, &T);
  for (int b = b0; b < b1; ++b) {
    C[b] = run;
    int L = (seqlens ? max(seqlens[b / rtiles], 0) : uniform_len);
    run += (L + kPage - 1) / kPage + overhead;
  }
  if (threadIdx.x == 0) C[batch] = T;
  __syncthreads();
  int t = max(1, (T + parts - 1) / parts);

  // whole-request mode?  The costliest part when part k takes requests
  // [k m, k m + m) whole.
  const int m = (batch + parts - 1) / parts;
  int local_max = 0;
  for (int k = threadIdx.x; k < parts; k += blockDim.x)
    local_max = max(local_max, C[min((k + 1) * m, batch)] - C[min(k * m, batch)]);
  const int max_cost = block_max(local_max, warp_sums);
  if (max_cost <= t + kSplitPenaltyPages) {
    int32_t* part_first = sched + kSchedHeader;
    int32_t* items = sched + sched_items_offset(parts);
    for (int b = b0; b < b1; ++b) {
      const int L = (seqlens ? max(seqlens[b / rtiles], 0) : uniform_len);
      items[4 * b + 0] = b;
      items[4 * b + 1] = 0;
      items[4 * b + 2] = (L + kPage - 1) / kPage;
      items[4 * b + 3] = -1;
      num_splits[b] = b;
    }
    for (int k = threadIdx.x; k <= parts; k += blockDim.x) part_first[k] = min(k * m, batch);
    if (threadIdx.x == 0) {
      num_splits[batch] = batch;
      sched[0] = parts;
      sched[1] = batch;
      sched[2] = max_cost;
      sched[3] = batch;
      sched[4] = overhead;
      sched[5] = 0;
      sched[6] = 1;
      sched[7] = rtiles;
    }
    return;
  }

  // 2. splits per request and their prefix
  local = 0;
  for (int b = b0; b < b1; ++b) {
    int k0 = C[b] / t, k1 = (C[b + 1] - 1) / t;
    local += k1 - k0 + 1;
  }
  int I;
  run = block_exclusive_scan(local, warp_sums, &I);
  for (int b = b0; b < b1; ++b) {
    S[b] = run;
    int k0 = C[b] / t, k1 = (C[b + 1] - 1) / t;
    run += k1 - k0 + 1;
  }
  if (threadIdx.x == 0) S[batch] = I;
  __syncthreads();

  // 3. items, and the compact list of split requests
  int32_t* part_first = sched + kSchedHeader;
  int32_t* split_list = sched + sched_split_list_offset(parts);
  int32_t* items = sched + sched_items_offset(parts);
  local = 0;
  for (int b = b0; b < b1; ++b) local += ((C[b + 1] - 1) / t - C[b] / t) > 0;
  int nsplit_req;
  int split_pos = block_exclusive_scan(local, warp_sums, &nsplit_req);
  for (int b = b0; b < b1; ++b) {
    const int L = (seqlens ? max(seqlens[b / rtiles], 0) : uniform_len);
    const int n = (L + kPage - 1) / kPage;
    const int cb = C[b], cost = C[b + 1] - C[b];
    const int k0 = cb / t, k1 = (C[b + 1] - 1) / t;
    const int K = k1 - k0 + 1;
    for (int s = 0; s < K; ++s) {
      const int k = k0 + s;
      const int v0 = max(cb, k * t) - cb;
      const int v1 = min(cb + cost, (k + 1) * t) - cb;
      const int p0 = min(max(v0 - overhead, 0), n);
      const int p1 = min(max(v1 - overhead, 0), n);
      const int idx = S[b] + s;
      items[4 * idx + 0] = b;
      items[4 * idx + 1] = p0;
      items[4 * idx + 2] = p1;
      items[4 * idx + 3] = (K > 1) ? idx : -1;
    }
    if (K > 1) split_list[split_pos++] = b;
    num_splits[b] = S[b];
  }
  if (threadIdx.x == 0) {
    num_splits[batch] = I;
    sched[0] = parts;
    sched[1] = I;
    sched[2] = t;
    sched[3] = batch;
    sched[4] = overhead;
    sched[5] = nsplit_req;
    sched[6] = 0;
    sched[7] = rtiles;
  }

  // 4. first item of each part: the request holding virtual position k t
  for (int k = threadIdx.x; k <= parts; k += blockDim.x) {
    const long long pos = static_cast<long long>(k) * t;
    int first;
    if (k == parts || pos >= T) {
      first = I;
    } else {
      int lo = 0, hi = batch - 1;  // largest b with C[b] <= pos
      while (lo < hi) {
        int mid = (lo + hi + 1) >> 1;
        if (C[mid] <= pos) lo = mid; else hi = mid - 1;
      }
      first = S[lo] + (k - C[lo] / t);
    }
    part_first[k] = first;
  }
}

// `batch` is the virtual batch (requests * rtiles); seqlens == nullptr gives
// every virtual request the length uniform_len.
cudaError_t launch_metadata(const int32_t* seqlens, int uniform_len, int batch, int rtiles, int parts,
                            int32_t* sched, int32_t* num_splits, cudaStream_t stream) {
  const size_t smem = 2ull * (batch + 1) * sizeof(int);
  if (smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(metadata_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
    if (e != cudaSuccess) return e;
  }
  // one request per thread up to 1024 requests (whole warps): small batches
  // sync fewer warps in the block scans
  const int threads = batch >= kMetaThreads ? kMetaThreads : ((batch + 31) / 32) * 32;
  metadata_kernel<<<1, threads > 0 ? threads : 32, smem, stream>>>(seqlens, uniform_len, batch, rtiles, parts,
                                                                  kSplitOverheadPages, sched, num_splits);
  return cudaGetLastError();
}

int metadata_max_batch() { return kMaxBatch; }

}  // namespace mla

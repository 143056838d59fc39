// Shared definitions of the CUDA side: problem constants, the schedule
// layout written by the metadata kernel, kernel parameter blocks and the
// device-side error reporting.
#pragma once

#include <cstddef>
#include <cstdint>

namespace mla {

constexpr int kPage = 64;         // tokens per cache block
constexpr int kDqk = 576;         // key width: 512 latent + 64 RoPE
constexpr int kDv = 512;          // value width (the latent)
constexpr int kDRope = 64;
constexpr int kRows = 128;        // MMA M: query rows (s_q * h_q, padded) per work item
constexpr int kMaxRowTiles = 8;   // M = s_q * h_q <= 1024: up to 8 row tiles per request

// A request with M = s_q * h_q query rows is served as ceil(M / 128) row
// tiles; the schedule treats every (request, row tile) as a unit of its own
// ("virtual request" v = request * row_tiles + tile), so the tiles of one
// request run on different CTA pairs at about the same time and share its
// pages through L2.
__host__ __device__ inline int row_tiles(int M) { return (M + kRows - 1) / kRows; }
// Rows of a row tile's partial results in the workspace (the stride per slot).
__host__ __device__ inline int rows_per_tile(int M) { return M < kRows ? M : kRows; }
constexpr int kFp8TokenBytes = 656;

// Per-request fixed cost of the split-KV schedule, in units of one page.
// A split costs a partial-output write plus its read-back in the combine
// kernel (2 x 128 rows x 512 x 4 B, about 7 bf16 pages of traffic for a
// 128-row request); a smaller value splits more eagerly.
constexpr int kSplitOverheadPages = 4;
// A schedule that splits requests pays for it outside the page loop: the
// fp32 partial outputs go to memory and come back in the combine kernel, and
// a CTA pair that serves two items drains and refills its pipeline in
// between.  The schedule keeps requests whole (ceil(batch / parts) of them
// per CTA pair) unless that makes the longest part longer than the balanced
// cut by more than this many pages.
#ifndef MLA_SPLIT_PENALTY_PAGES
#define MLA_SPLIT_PENALTY_PAGES 16
#endif
constexpr int kSplitPenaltyPages = MLA_SPLIT_PENALTY_PAGES;

// Schedule buffer (int32) written by the metadata kernel, over the virtual
// requests (request, row tile) of the batch:
//   [0] num_parts  [1] total_items  [2] units per part  [3] virtual batch
//   (batch * row tiles)  [4] overhead   [5] number of split virtual requests
//   [6] 1 if whole requests (ceil(batch / parts) consecutive ones per
//   part, no split), else 0  [7] row tiles
//   [8, 8 + num_parts + 1)          first item index of each part
//   then num_parts ints             ids of the split requests (first [5] valid)
//   then (16-byte aligned) 4 ints per item: request b, first page, end page, slot
// Items are ordered by (request, split).  `slot` is the item's index when
// the request is split (its partial-output row block), -1 otherwise.
constexpr int kSchedHeader = 8;
__host__ __device__ inline int sched_split_list_offset(int parts) { return kSchedHeader + parts + 1; }
__host__ __device__ inline int sched_items_offset(int parts) {
  return (sched_split_list_offset(parts) + parts + 3) & ~3;
}
__host__ __device__ inline size_t sched_ints(int batch, int parts) {
  return static_cast<size_t>(sched_items_offset(parts)) +
         4ull * (static_cast<size_t>(batch) + static_cast<size_t>(parts));
}
__host__ __device__ inline int max_items(int batch, int parts) { return batch + parts; }

// Workspace: a 256-byte header (status word at offset 0), then fp32 partial
// lse [max_items][Mt] and fp32 partial outputs [max_items][Mt][512], with
// max_items over the virtual batch and Mt = rows_per_tile(M).
constexpr size_t kWsHeader = 256;
__host__ __device__ inline size_t ws_lse_offset() { return kWsHeader; }
__host__ __device__ inline size_t ws_o_offset(int batch, int parts, int M) {
  const int vb = batch * row_tiles(M);
  size_t lse_bytes = 4ull * static_cast<size_t>(max_items(vb, parts)) * static_cast<size_t>(rows_per_tile(M));
  return kWsHeader + ((lse_bytes + 255) / 256) * 256;
}
__host__ __device__ inline size_t ws_bytes(int batch, int parts, int M) {
  const int vb = batch * row_tiles(M);
  return ws_o_offset(batch, parts, M) +
         4ull * static_cast<size_t>(max_items(vb, parts)) * static_cast<size_t>(rows_per_tile(M)) * kDv;
}

struct DecodeParams {
  const uint16_t* q;            // bf16 [batch, M, 576]
  const int32_t* block_table;   // [batch, max_pages]
  const int32_t* seqlens;       // [batch]
  const int32_t* sched;         // schedule buffer
  uint16_t* out;                // bf16 [batch, M, 512]
  float* lse;                   // [batch, M]
  float* lse_part;              // [max_items, M]
  float* o_part;                // [max_items, M, 512]
  int* status;                  // workspace status word
  long long num_blocks;
  int max_pages;
  int batch;
  int s_q;
  int h_q;
  int M;                        // query rows per request (s_q * h_q)
  int row_tiles;                // ceil(M / 128)
  int causal;
  int num_parts;                // CTA pairs launched (must equal sched[0])
  float scale_log2;             // softmax_scale * log2(e)
  unsigned long long timeout_ns;
  unsigned long long* trace;    // per-tile timestamps (trace build only), else null
  const int* hold_flag;         // diagnostics (mla_debug_hold_at_tile): device flag, or null
  int hold_tile;                // the PV issuer's tile at which it waits for *hold_flag != 0
  int q_wide;                   // q is 32-byte aligned: 32-byte loads
  int out_wide;                 // out and the partials are 32-byte aligned: 32-byte stores
  // Units and requests.  Rows of q, out and lse are grouped in `batch` units
  // of M rows.  Dense decode: a unit is a request (req_div = 1).  Sparse
  // decode: a unit is one query token of a request (M = h_q, req_div = s_q),
  // and the block table and the lengths are indexed by unit / req_div.
  int req_div;
  int req_batch;                // rows of block_table and seqlens
  const int32_t* indices;       // sparse: [batch units, topk] positions in the request
  int topk;
};

// Per-tile timestamps of the decode kernel, recorded only by a library built
// with MLA_TRACE: trace[cta][role][tile][slot] holds the SM clock (clock64)
// when a role passed a fixed point of its loop, for the first kTraceCtas CTAs
// and their first kTraceTiles tiles.  Role kTraceCta, tile 0, also holds the
// global timer (ns) at kernel entry in slot 15, so that CTAs can be aligned.
constexpr int kTraceCtas = 4;
constexpr int kTraceRoles = 7;
constexpr int kTraceTiles = 128;
constexpr int kTraceSlots = 16;
enum : int {
  kTraceProducer = 0,  // 0 wait for a free stage, 1 copies issued
  kTraceQk = 1,        // 0 wait for the page, 1 page ready, 2 S free, 3 issued
  kTracePv = 2,        // 0 wait for P, 1 P ready, 2 issued
  kTraceSoftmax = 3,   // 0 wait for S, 1 S ready, 2 S loaded, 3 row max, 4 buffer
                       // credit, 5 sent, 6 first half in, 7 P formed, 8 reference
                       // chain, 9 P buffer free, 10 O rescaled, 11 P stored
  kTraceDequant = 4,   // 0 wait for raw bytes, 1 raw ready, 2 stage free, 3 done
  kTraceItem = 5,      // tile = item: 0 start, 1 Q stored, 2 epilogue start, 3 done,
                       // 4 final reference known, 5 row sums joined, 6 last PV done
  kTraceCta = 6,       // tile 0: 0 entry, 1 set up, 2 schedule readable, 3 roles
                       // done, 4 exit, 15 global timer at entry
};
constexpr size_t kTraceBytes =
    sizeof(unsigned long long) * kTraceCtas * kTraceRoles * kTraceTiles * kTraceSlots;

struct CombineParams {
  const int32_t* sched;         // schedule buffer (split-request list)
  const int32_t* num_splits;    // [batch + 1]
  const float* lse_part;
  const float* o_part;
  uint16_t* out;
  float* lse;
  int batch;
  int M;
  int row_tiles;
  int num_parts;
};

// Status codes as stored in the workspace status word (match mla_status_t).
constexpr int kStatusBadSchedule = 1;
constexpr int kStatusTimeout = 5;
constexpr int kStatusBadBlock = 6;

__device__ __forceinline__ void report_status(int* status, int code) {
  atomicCAS(status, 0, code);
}

}  // namespace mla

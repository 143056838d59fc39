// MLA decode over a paged KV cache on sm_100a.
//
// One CTA pair (a 2-CTA cluster) per part of the split-KV schedule, persistent
// over the part's work items (request, page range).
//
//   * The pair splits the 576 key dims: CTA r owns latent dims
//     [256 r, 256 r + 256) and RoPE dims [512 + 32 r, 512 + 32 r + 32).  Each
//     CTA gathers only its half of every 64-token page (block_table-driven TMA
//     loads, 36 KB per page half; the FP8 variant loads the raw 656-byte rows
//     and dequantises its half in shared memory), so KV crosses HBM once.
//   * Q (this CTA's 288 dims, up to 128 query rows = s_q * h_q) lives in tensor
//     memory and is the A operand of the partial S_r = Q_r K_r^T: tcgen05.mma,
//     M = 128, N = 64 tokens, K = 288, fp32 accumulation in tensor memory.
//   * Softmax exchange, factorised: exp2(x0 + x1 - M0 - M1) = exp2(x0 - M0) *
//     exp2(x1 - M1) with x_r = log2(e) * softmax_scale * S_r.  Each CTA
//     exponentiates its own partial logits against a lazy per-row reference
//     M_r and sends only those factors (fp16) and M_r to the peer through
//     distributed shared memory; P = (own fp32 factor) * (peer fp16 factor).
//     That halves the bytes on the CTA-pair link against shipping the fp32
//     partial S; each CTA normalises its own half of O with its own row sum.
//   * O_r += P V_r with V_r = this CTA's 256 latent dims of the same page (the
//     value is the first 512 dims of the key): M = 128, N = 256, K = 64, P read
//     from tensor memory, V as an MN-major operand of the same 128-byte-
//     swizzled tile the QK^T product reads as K-major.
//   * Epilogue: bf16 out + lse for an unsplit request, fp32 partials for a
//     split one (merged by the combine kernel).
//   * Sparse variant (FP8 cache): a unit is one query token, and its tiles are
//     64-entry slices of its index list instead of pages.  The producer is a
//     whole warp that maps the listed positions through the block table and
//     gathers the rows with TMA; a per-tile validity mask replaces the length
//     mask.
//
// Warp roles: warp 0 TMA producer, warp 1 QK^T issuer, warp 2 tensor-memory
// allocator, warp 3 PV issuer; warps 4-11 softmax in two warpgroups that take
// alternate tiles (warpgroup w the tiles g with g % 2 == w), thread (w, r)
// owning query row r (= tensor-memory lane r) and all 64 columns of its
// warpgroup's tiles; FP8 adds warps 12-15 for the dequantisation.  The
// ping-pong lets one warpgroup wait for its pair message while the other one
// exponentiates, and no barrier joins the two warpgroups inside a tile.  Each
// warpgroup raises its lazy reference to the other's latest published one,
// read without waiting (any reference is correct; the two converge within a
// tile or two).  The combined reference of the last consumed tile, which is
// the scale O is at, passes between them through an mbarrier-guarded slot, so
// O is rescaled exactly when that scale moves.  tcgen05.mma issue blocks for
// about the instruction's run time, so QK^T and PV get one issuing thread each
// (one thread for both would hold QK^T(j + 1) behind PV(j)), with their
// shared-memory descriptors precomputed.
//
// Every mbarrier wait is bounded (params.timeout_ns); a wait that runs out
// records MLA_ERR_TIMEOUT, raises a CTA-wide abort flag, and the CTA drains
// its copies and MMAs, frees tensor memory and exits.
#include <cuda.h>
#include <cuda_fp16.h>
#include <cuda_fp8.h>
#include <cuda_runtime.h>
#include <math_constants.h>

#include <atomic>

#include "common.cuh"
#include "sm100.cuh"

namespace mla {

namespace dk {
constexpr int kChunkBytes = kPage * 128;                 // 64 tokens x 64 dims bf16 (SW128)
constexpr int kRopeBytes = kPage * 64;                   // 64 tokens x 32 dims bf16 (SW64)
constexpr int kStageBytes = 4 * kChunkBytes + kRopeBytes;  // 36864: one page half
constexpr int kRawLatBytes = kPage * 256;               // FP8: this CTA's 256 latent codes per token
constexpr int kRawScaleBytes = kPage * 16;              // FP8: the 4 fp32 scales per token
constexpr int kRawRopeBytes = kPage * 64;               // FP8: this CTA's 32 RoPE bf16 per token
constexpr int kRawBytes = kRawLatBytes + kRawScaleBytes + kRawRopeBytes;  // 21504
// Sparse decode: the gather brings, per token, this CTA's latent half and
// bytes [496, 656) of the token (the last latent bytes, the four scales and
// both RoPE halves; 160 bytes keeps every group of four rows 128-byte
// aligned in shared memory).
constexpr int kTailX = 496;
constexpr int kTailBytes = 160;
constexpr int kRawSparseBytes = kRawLatBytes + kPage * kTailBytes;  // 26624
#ifndef MLA_FP8_RAW_STAGES
#define MLA_FP8_RAW_STAGES 2
#endif
#ifndef MLA_FP8_STAGES
#define MLA_FP8_STAGES 3
#endif
#ifndef MLA_BF16_STAGES
#define MLA_BF16_STAGES 5
#endif
#ifndef MLA_FP8_XBUFFERS
#define MLA_FP8_XBUFFERS 3
#endif
#ifndef MLA_BF16_XBUFFERS
#define MLA_BF16_XBUFFERS 2
#endif
// The sparse decode: the same pipeline depths as the dense FP8 path (four
// raw stages with two dequantised stages and two exchange buffers, or three
// raw stages with two dequantised ones, measured 6% slower: a dequantised
// stage is held from its dequant until P*V has read it, and two of them
// leave the dequant waiting).
#ifndef MLA_SPARSE_RAW_STAGES
#define MLA_SPARSE_RAW_STAGES 2
#endif
#ifndef MLA_SPARSE_STAGES
#define MLA_SPARSE_STAGES 3
#endif
#ifndef MLA_SPARSE_XBUFFERS
#define MLA_SPARSE_XBUFFERS 3
#endif
// Exchange message per tile: fp16 factors [8 chunks of 8 tokens][128 rows][16 B]
// + the fp32 reference of every row.
constexpr int kXERegionBytes = 8 * kRows * 16;          // 16384
constexpr int kXMsgBytes = kXERegionBytes + kRows * 4;  // 16896
constexpr int kXBufBytes = kXMsgBytes;
constexpr int kSoftmaxWarps = 8;
// FP8: one dequant warp per scheduler partition (a warpgroup).
constexpr int kDqWarps = 4;
// FP8 register split per warpgroup (512 threads launch with 128 registers
// each): control 64, softmax 176, dequant 96, and the softmax and dequant
// warpgroups at 64 for the common tail.  64 + 2 x 176 + 96 = 4 x 128: the
// softmax warpgroups' increase is exactly funded by the decreases.  (ptxas
// does not fit the dequant warpgroup's code below 96 registers.)
constexpr int kRegLaunchFp8 = 128;
constexpr int kRegCtl = 64;
constexpr int kRegSoftmax = 176;
constexpr int kRegDq = 96;
constexpr int kRegTail = 64;
// The sparse decode's control warpgroup runs the whole-warp gather (index
// and block-table reads, row shuffles): control 80, dequant 80.
constexpr int kRegCtlSparse = 80;
constexpr int kRegDqSparse = 80;
constexpr int kRegTailSparse = 80;
static_assert(kRegCtlSparse + 2 * kRegSoftmax + (kDqWarps / 4) * kRegDqSparse <= (3 + kDqWarps / 4) * kRegLaunchFp8,
              "register split exceeds the launch budget");
static_assert(kRegCtl + 2 * kRegSoftmax + (kDqWarps / 4) * kRegDq <= (3 + kDqWarps / 4) * kRegLaunchFp8,
              "register split exceeds the launch budget");
constexpr float kRescaleThreshold = 8.0f;  // log2 units: the lazy reference moves by more than a factor 256

template <bool kFp8, bool kSparse = false>
struct Cfg {
  // bf16 page-half stages
  static constexpr int kStages = kSparse ? MLA_SPARSE_STAGES : kFp8 ? MLA_FP8_STAGES : MLA_BF16_STAGES;
  // FP8: raw 656-byte-format stages, and the bytes of one
  static constexpr int kRawStages = kSparse ? MLA_SPARSE_RAW_STAGES : MLA_FP8_RAW_STAGES;
  static constexpr int kRawStageBytes = kSparse ? kRawSparseBytes : kRawBytes;
  // Pair-exchange receive buffers: tile g uses buffer g % kXBuffers, and the
  // peer writes tile g + kXBuffers's message into it only after this CTA has
  // read tile g's (a remote arrive on the peer's "buffer free" barrier).
  static constexpr int kXBuffers = kSparse ? MLA_SPARSE_XBUFFERS : kFp8 ? MLA_FP8_XBUFFERS : MLA_BF16_XBUFFERS;
  static constexpr int kThreads = kFp8 ? 384 + 32 * kDqWarps : 384;
  static constexpr int kFull = 0;
  static constexpr int kEmpty = kFull + kStages;
  static constexpr int kSFull = kEmpty + kStages;  // two: by tile parity
  static constexpr int kSFree = kSFull + 2;
  static constexpr int kPFull = kSFree + 1;    // two: one per P buffer (= per warpgroup)
  static constexpr int kPvDone = kPFull + 2;   // two: one per P buffer
  static constexpr int kQReady = kPvDone + 2;
  static constexpr int kXFull = kQReady + 1;  // two per buffer: tokens 0-31, tokens 32-63 + reference
  static constexpr int kDrain = kXFull + 2 * kXBuffers;  // two: QK^T and PV issuers
  static constexpr int kCChain = kDrain + 2;   // combined reference of tile g published
  static constexpr int kEpi = kCChain + 1;     // both warpgroups' row sums published
  static constexpr int kXFree = kEpi + 1;      // two: the peer has read this CTA's message in buffer i
  static constexpr int kRawFull = kXFree + kXBuffers;  // FP8 only
  static constexpr int kRawEmpty = kRawFull + kRawStages;
  static constexpr int kNumBars = kRawEmpty + kRawStages;
  static constexpr int kXOffset = kStages * kStageBytes;
  static constexpr int kRawOffset = kXOffset + kXBuffers * kXBufBytes;
  // Q's RoPE half-slice (128 rows x 32 dims bf16, SW64 K-major) is an SS operand
  static constexpr int kQRopeOffset = kRawOffset + (kFp8 ? kRawStages * kRawStageBytes : 0);
  // [wg][row] fp32: each warpgroup's latest lazy reference; [row] the
  // combined reference of the last consumed tile; [wg][row] the row-sum parts
  // at the item's final scale.  Then barriers, the abort flag, the tensor-
  // memory base and the slot where the peer CTA reports its abort flag.
  static constexpr int kRefSlotOffset = kQRopeOffset + kRows * 64;
  static constexpr int kCombSlotOffset = kRefSlotOffset + 2 * kRows * 4;
  static constexpr int kEpiOffset = kCombSlotOffset + kRows * 4;
  // Sparse decode: the validity mask of each raw stage and of each bf16
  // stage (bit t: token t of the tile is a key).
  static constexpr int kRawMaskOffset = kEpiOffset + 2 * kRows * 4;
  static constexpr int kStageMaskOffset = kRawMaskOffset + 8 * kRawStages;
  static constexpr int kBarOffset = kStageMaskOffset + 8 * kStages;
  // The dynamic shared memory base is 1024-byte aligned (the driver reserves
  // the first 1 KB of the window); the kernel checks it at entry.
  static constexpr int kSmemBytes = kBarOffset + kNumBars * 8 + 16;
  static_assert(kSmemBytes <= 232448, "shared memory budget");
};
// tensor-memory columns (512 allocated)
constexpr uint32_t kColO = 0;    // 256 fp32 columns: this CTA's half of O
constexpr uint32_t kColS = 256;  // 64 fp32 columns: partial S
constexpr uint32_t kColP = 320;  // 2 x 32 columns: P (packed bf16 pairs), double-buffered
constexpr uint32_t kColQ = 384;  // 128 columns: Q's 256 latent dims as packed bf16 pairs
}  // namespace dk

__device__ const int g_never_abort = 0;

// Per-tile timestamps (layout in common.cuh).  Only a library compiled with
// MLA_TRACE records them; the product build emits no code for TRACE.
#ifdef MLA_TRACE
__device__ __forceinline__ void trace_point(const DecodeParams& p, int role, uint32_t tile, int slot) {
  if (p.trace != nullptr && blockIdx.x < static_cast<unsigned>(kTraceCtas) && tile < static_cast<uint32_t>(kTraceTiles))
    p.trace[((static_cast<size_t>(blockIdx.x) * kTraceRoles + role) * kTraceTiles + tile) * kTraceSlots + slot] =
        clock64();
}
#define TRACE(role, tile, slot) trace_point(p, (role), static_cast<uint32_t>(tile), (slot))
#else
#define TRACE(role, tile, slot) ((void)0)
#endif

// Warp-uniform bounded wait.  Fast path: every lane tries the phase once (a
// completed phase, the common case, costs one warp-wide try).  Otherwise lane 0
// polls with the time limit, then every lane performs its own (immediately
// successful) acquire of the same phase.
template <bool kCluster = false>
__device__ __forceinline__ bool warp_wait(uint32_t bar, uint32_t parity, const volatile int* abort,
                                          uint64_t limit) {
  if (__all_sync(0xffffffffu, kCluster ? mbar_try_cluster(bar, parity) : mbar_try(bar, parity))) return true;
  int ok = 1;
  if ((threadIdx.x & 31) == 0) ok = mbar_wait<kCluster>(bar, parity, abort, limit);
  ok = __shfl_sync(0xffffffffu, ok, 0);
  if (ok) {
#pragma unroll 1
    for (int i = 0; i < (1 << 20); ++i)
      if (kCluster ? mbar_try_cluster(bar, parity) : mbar_try(bar, parity)) break;
  }
  return ok != 0;
}

// Diagnostics (mla_debug_hold_at_tile): wait, bounded like every other wait,
// until the host-visible flag becomes non-zero.  A test gives a flag that
// nothing sets, so the wait runs out with the pipeline full and the abort
// path (drain copies and MMAs, free tensor memory, report MLA_ERR_TIMEOUT)
// runs for real.
__device__ __forceinline__ bool hold_until_flag(const DecodeParams& p, const volatile int* abort_flag) {
  const volatile int* flag = p.hold_flag;
  const uint64_t t0 = globaltimer_ns();
#pragma unroll 1
  while (*flag == 0) {
    if (*abort_flag || globaltimer_ns() - t0 > p.timeout_ns) return false;
    __nanosleep(256);
  }
  return true;
}

__device__ __forceinline__ void raise_abort(const DecodeParams& p, volatile int* abort_flag) {
  report_status(p.status, kStatusTimeout);
  *abort_flag = 1;
}

// 16 E4M3 codes (one 16-byte raw unit) times an fp32 scale -> 16 bf16 (RNE),
// as 8 packed pairs in memory order.  e4m3 -> f16 is exact; the product is
// formed in fp32 (a packed pair of IEEE multiplies) and rounded once to bf16.
__device__ __forceinline__ void dequant16(const uint4 raw, float sc, uint32_t (&w)[8]) {
  const uint32_t in[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const __nv_fp8x2_storage_t pair = static_cast<__nv_fp8x2_storage_t>((in[i] >> (16 * h)) & 0xFFFFu);
      const __half2_raw hr = __nv_cvt_fp8x2_to_halfraw2(pair, __NV_E4M3);
      const float2 v = __fmul2_rn(make_float2(__half2float(__ushort_as_half(hr.x)), __half2float(__ushort_as_half(hr.y))),
                                  make_float2(sc, sc));
      w[2 * i + h] = pack_bf16x2(v.x, v.y);
    }
  }
}

// kSparse (FP8 only): each unit (a query token) attends to the tokens its
// index list names instead of a page range; the producer gathers their rows
// with TMA gathers and a per-tile validity mask replaces the length mask.
template <bool kFp8, bool kSparse>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(dk::Cfg<kFp8>::kThreads, 1)
    decode_kernel(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_b,
                  const __grid_constant__ CUtensorMap tm_c, const DecodeParams p) {
  using namespace dk;
  using C = Cfg<kFp8, kSparse>;
  static_assert(!kSparse || kFp8, "the sparse decode reads the 656-byte FP8 cache");
  constexpr int kCtlRegs = kSparse ? kRegCtlSparse : kRegCtl;
  constexpr int kDqRegs = kSparse ? kRegDqSparse : kRegDq;
  constexpr int kTailRegs = kSparse ? kRegTailSparse : kRegTail;
  constexpr int kStages = C::kStages;
  extern __shared__ uint8_t smem_raw[];
  TRACE(kTraceCta, 0, 0);
#ifdef MLA_TRACE
  if (threadIdx.x == 0 && p.trace != nullptr && blockIdx.x < static_cast<unsigned>(kTraceCtas))
    p.trace[(static_cast<size_t>(blockIdx.x) * kTraceRoles + kTraceCta) * kTraceTiles * kTraceSlots + 15] =
        globaltimer_ns();
#endif
  // The combine kernel may start launching now; it waits for this grid.
  pdl_launch_dependents();
  const uint32_t raw_addr = smem_u32(smem_raw);
  if (raw_addr & 1023u) {  // swizzled tiles need 1024-byte alignment
    pdl_wait();
    if (threadIdx.x == 0) report_status(p.status, kStatusBadSchedule);
    return;
  }
  const uint32_t base = raw_addr;
  uint8_t* sbase = smem_raw + (base - raw_addr);
  const uint32_t stage0 = base;
  const uint32_t xbuf0 = base + C::kXOffset;
  const uint32_t rawbuf0 = base + C::kRawOffset;
  const uint32_t bar0 = base + C::kBarOffset;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(sbase + C::kBarOffset + C::kNumBars * 8);
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(sbase + C::kBarOffset + C::kNumBars * 8 + 4);
#define BAR(i) (bar0 + 8u * static_cast<uint32_t>(i))

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const uint32_t peer = rank ^ 1u;
  const int part = static_cast<int>(cluster_id_x());

  if (threadIdx.x == 0) {
    for (int i = 0; i < kStages; ++i) {
      mbar_init(BAR(C::kFull + i), kFp8 ? kDqWarps : 1);  // FP8: every dequant warp arrives
      mbar_init(BAR(C::kEmpty + i), 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(BAR(C::kSFull + i), 1);
      mbar_init(BAR(C::kPFull + i), 4);  // the four warps of the consuming warpgroup
      mbar_init(BAR(C::kPvDone + i), 1);
      mbar_init(BAR(C::kDrain + i), 1);
    }
    mbar_init(BAR(C::kSFree), 4);
    mbar_init(BAR(C::kQReady), kSoftmaxWarps);
    for (int i = 0; i < 2 * C::kXBuffers; ++i) mbar_init(BAR(C::kXFull + i), 1);
    mbar_init(BAR(C::kCChain), 128);  // every thread of the consuming warpgroup
    mbar_init(BAR(C::kEpi), kSoftmaxWarps * 32);
    for (int i = 0; i < C::kXBuffers; ++i) mbar_init(BAR(C::kXFree + i), 4);  // the peer warpgroup's four warps
    for (int i = 0; i < C::kRawStages; ++i) {
      mbar_init(BAR(C::kRawFull + i), 1);
      mbar_init(BAR(C::kRawEmpty + i), kDqWarps);
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 2) {
    tmem_alloc(smem_u32(tmem_holder), 512);
    tmem_relinquish();
  }
  if (!kSparse && warp == 0 && lane == 0) {
    tma_prefetch_desc(&tm_a);
    tma_prefetch_desc(&tm_b);
    if (kFp8) tma_prefetch_desc(&tm_c);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;
  cluster_sync();  // the peer's barriers are initialised before any st.async reaches them
  if (threadIdx.x == 0) TRACE(kTraceCta, 0, 1);

  // While the schedule kernel finishes: start q and the block table towards
  // L2, spread over every thread of the grid, so that the first Q and
  // block-table reads after the wait do not go to DRAM.  A prefetch only
  // moves cache lines and cannot observe a value, so it is issued before the
  // wait whoever writes these tensors.
  {
    const size_t nthr = static_cast<size_t>(gridDim.x) * blockDim.x;
    const size_t tid = static_cast<size_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    const size_t qbytes = static_cast<size_t>(p.batch) * p.M * (kDqk * 2);
    const size_t btbytes = static_cast<size_t>(p.req_batch) * p.max_pages * 4;
    const uint8_t* qb = reinterpret_cast<const uint8_t*>(p.q);
    const uint8_t* btb = reinterpret_cast<const uint8_t*>(p.block_table);
    for (size_t o = tid * 128; o < qbytes; o += nthr * 128) prefetch_l2_line(qb + o);
    for (size_t o = tid * 128; o < btbytes; o += nthr * 128) prefetch_l2_line(btb + o);
  }
  // Everything above wrote only this CTA's own memories.  The schedule was
  // written by the previous kernel in the stream (mla_get_metadata), and the
  // workspace and outputs may still be read by the previous combine pass.
  pdl_wait();
  if (threadIdx.x == 0) TRACE(kTraceCta, 0, 2);
  // The header and this part's item range are read together (independent
  // loads, all inside the header of a buffer sized for p.num_parts); the range
  // is used only if the header matches this call.
  const int s_parts = p.sched[0], s_vbatch = p.sched[3], s_rtiles = p.sched[7];
  const int s_first = p.sched[kSchedHeader + part], s_end = p.sched[kSchedHeader + part + 1];
  const int32_t* items = p.sched + sched_items_offset(p.num_parts);
  int it_begin = 0, it_end = 0;
  if (s_parts != p.num_parts || s_vbatch != p.batch * p.row_tiles || s_rtiles != p.row_tiles) {
    // schedule made for another CTA-pair count or another batch: its request
    // ids and item slots may lie outside this call's tensors and workspace,
    // so do nothing and report it
    if (threadIdx.x == 0) report_status(p.status, kStatusBadSchedule);
  } else {
    it_begin = s_first;
    it_end = s_end;
  }

  // Register budget per warpgroup (FP8, constants above).  The only increase
  // is the softmax warpgroups' at their start, which the decreases exactly
  // fund; at the end every warpgroup is at kRegTail for the short common
  // tail.  (An increase anywhere else could take registers that a softmax
  // warpgroup still waits for: setmaxnreg.inc blocks until the pool can pay.)
  if (warp < 4) {
    if constexpr (kFp8) setmaxnreg_dec<kCtlRegs>();
  if (kSparse && warp == 0) {
    // ------------------------------------------------------------------ sparse gather (whole warp)
    // Tile j of an item is entries [64 j, 64 j + 64) of the unit's index
    // list.  Lane l resolves entries l and l + 32: it reads the position,
    // checks it against the request's length and maps it through the block
    // table to a row of the cache (viewed as [num_blocks * 64, 656] bytes).
    // These reads run ahead of the copies (see below).  The copies are TMA
    // gathers of four rows: lanes 0-15 bring the latent halves of tokens
    // 4l .. 4l + 3 (256 bytes each), lanes 16-31 their tails (bytes 496-655).
    // Entries that are not keys (padding, positions outside [0, L), pages that
    // map outside the cache, which are also reported) fetch row 0 instead and
    // keep their bit in the stage's mask clear; the dequant writes zeros for
    // them and the softmax masks their logits.
    uint64_t* raw_mask = reinterpret_cast<uint64_t*>(sbase + C::kRawMaskOffset);
    uint32_t g = 0;
    bool ok = true;
    for (int it = it_begin; it < it_end && ok; ++it) {
      const int vb = items[4 * it], p0 = items[4 * it + 1], p1 = items[4 * it + 2];
      const int u = vb / p.row_tiles;
      const int req = u / p.req_div;
      const int L = p.seqlens[req];
      const int32_t* bt = p.block_table + static_cast<size_t>(req) * p.max_pages;
      const int32_t* list = p.indices + static_cast<size_t>(u) * p.topk;
      if (lane == 0 && rank == 0 && p1 > p0) {
        const int row0 = (vb - u * p.row_tiles) * kRows;
        const uint8_t* qb = reinterpret_cast<const uint8_t*>(p.q) + (static_cast<size_t>(u) * p.M + row0) * (kDqk * 2);
        const uint32_t bytes = static_cast<uint32_t>(min(kRows, p.M - row0)) * (kDqk * 2);
        for (uint32_t o = 0; o < bytes; o += 16384u) prefetch_l2_bulk(qb + o, min(16384u, bytes - o));
      }
      // Each tile's rows take two dependent reads (its list entries, then the
      // block table): start this item's slice of the list and the request's
      // block-table row towards L2 now, so that those reads hit L2.  Only
      // whole 16-byte granules inside each array are prefetched.
      if (lane == 0 && p1 > p0) {
        auto prefetch_range = [](const int32_t* first, const int32_t* last) {
          const uintptr_t a0 = (reinterpret_cast<uintptr_t>(first) + 15u) & ~static_cast<uintptr_t>(15);
          const uintptr_t a1 = reinterpret_cast<uintptr_t>(last) & ~static_cast<uintptr_t>(15);
          for (uintptr_t a = a0; a < a1; a += 16384u)
            prefetch_l2_bulk(reinterpret_cast<const void*>(a), static_cast<uint32_t>(a1 - a < 16384u ? a1 - a : 16384u));
        };
        prefetch_range(list + p0 * kPage, list + min(p1 * kPage, p.topk));
        if (rank == 0) prefetch_range(bt, bt + min((max(L, 0) + kPage - 1) / kPage, p.max_pages));
      }
      // A tile's rows take two dependent reads: its list entries, then the
      // block-table entries they select.  Both are software-pipelined over
      // the tiles: while tile pg's gathers go out, the block-table reads of
      // tile pg + 2 and the list reads of tile pg + 3 are issued, and each
      // value is first used one tile after its read was issued.  Lane l
      // holds entries l and l + 32 of a tile.
      auto load_pos = [&](int pg, int (&pos)[2]) {
#pragma unroll
        for (int k = 0; k < 2; ++k) {
          const int e = pg * kPage + lane + 32 * k;
          pos[k] = (pg < p1 && e < p.topk) ? list[e] : -1;
        }
      };
      // -1 for a page outside the table (reported below if the entry is a key)
      auto load_blk = [&](const int (&pos)[2], int (&blk)[2]) {
#pragma unroll
        for (int k = 0; k < 2; ++k) {
          const int pgi = pos[k] / kPage;
          blk[k] = (pos[k] >= 0 && pos[k] < L && pgi < p.max_pages) ? bt[pgi] : -1;
        }
      };
      // cache rows (-1: not a key)
      auto rows_of = [&](const int (&pos)[2], const int (&blk)[2], int (&row)[2]) {
#pragma unroll
        for (int k = 0; k < 2; ++k) {
          row[k] = -1;
          if (pos[k] >= 0 && pos[k] < L) {
            if (blk[k] < 0 || blk[k] >= p.num_blocks) report_status(p.status, kStatusBadBlock);
            else row[k] = blk[k] * kPage + pos[k] % kPage;
          }
        }
      };
      int cur[2] = {-1, -1};
      int pos1[2] = {-1, -1}, blk1[2] = {-1, -1}, pos2[2] = {-1, -1};  // tiles pg + 1 and pg + 2
      if (p1 > p0) {
        int pos0[2], blk0[2];
        load_pos(p0, pos0);
        load_pos(p0 + 1, pos1);
        load_pos(p0 + 2, pos2);
        load_blk(pos0, blk0);
        load_blk(pos1, blk1);
        rows_of(pos0, blk0, cur);
      }
      for (int pg = p0; pg < p1; ++pg, ++g) {
        const uint32_t st = g % C::kRawStages;
        if (lane == 0) TRACE(kTraceProducer, g, 0);
        int waited = 1;
        if (lane == 0 && g >= static_cast<uint32_t>(C::kRawStages))
          waited = mbar_wait(BAR(C::kRawEmpty + st), ((g / C::kRawStages) & 1u) ^ 1u, abort_flag, p.timeout_ns);
        waited = __shfl_sync(0xffffffffu, waited, 0);
        if (!waited) {
          if (lane == 0) raise_abort(p, abort_flag);
          ok = false;
          break;
        }
        const uint32_t m0 = __ballot_sync(0xffffffffu, cur[0] >= 0), m1 = __ballot_sync(0xffffffffu, cur[1] >= 0);
        const uint32_t fb = BAR(C::kRawFull + st);
        if (lane == 0) {
          raw_mask[st] = (static_cast<uint64_t>(m1) << 32) | m0;
          mbar_arrive_expect_tx(fb, kRawSparseBytes);
        }
        __syncwarp();
        // rows of tokens 4q .. 4q + 3, q = lane % 16: token t sits in lane
        // t % 32, slot t / 32
        const int q4 = lane & 15;
        int rows[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int t = 4 * q4 + i;
          const int r0 = __shfl_sync(0xffffffffu, cur[0], t & 31);
          const int r1 = __shfl_sync(0xffffffffu, cur[1], t & 31);
          const int rr = t < 32 ? r0 : r1;
          rows[i] = rr < 0 ? 0 : rr;
        }
        const uint32_t dst = rawbuf0 + st * C::kRawStageBytes;
        if (lane < 16)
          tma_gather4(dst + q4 * 4 * 256, &tm_a, fb, static_cast<int>(rank) * 256, rows[0], rows[1], rows[2], rows[3]);
        else
          tma_gather4(dst + kRawLatBytes + q4 * 4 * kTailBytes, &tm_b, fb, kTailX, rows[0], rows[1], rows[2],
                      rows[3]);
        if (lane == 0) TRACE(kTraceProducer, g, 1);
        // tile pg + 1's rows from reads issued a tile ago; the reads of the
        // next two tiles go out
        rows_of(pos1, blk1, cur);
        load_blk(pos2, blk1);
#pragma unroll
        for (int k = 0; k < 2; ++k) pos1[k] = pos2[k];
        load_pos(pg + 3, pos2);
      }
    }
    // Never leave a copy landing in shared memory after the CTA exits.
    if (lane == 0)
      for (uint32_t k = (g > static_cast<uint32_t>(C::kRawStages) ? g - C::kRawStages : 0u); k < g; ++k)
        mbar_wait(BAR(C::kRawFull + k % C::kRawStages), (k / C::kRawStages) & 1u, &g_never_abort, 100000000ull);
  } else if (warp == 0) {
    // ------------------------------------------------------------------ TMA producer
    if (lane == 0) {
      // BF16: page halves straight into the MMA stages.  FP8: raw bytes into
      // the raw stages, for the dequant warps.
      constexpr int nst = kFp8 ? C::kRawStages : kStages;
      const int full0 = kFp8 ? C::kRawFull : C::kFull;
      const int empty0 = kFp8 ? C::kRawEmpty : C::kEmpty;
      uint32_t g = 0;
      bool ok = true;
      for (int it = it_begin; it < it_end && ok; ++it) {
        const int vb = items[4 * it], p0 = items[4 * it + 1], p1 = items[4 * it + 2];
        const int b = vb / p.row_tiles, row0 = (vb - b * p.row_tiles) * kRows;
        const int32_t* bt = p.block_table + static_cast<size_t>(b) * p.max_pages;
        // The block-table entries of the first nst pages, read together and
        // first of all: at a kernel's start every SM's memory pipe is busy and
        // a lone dependent load waits for microseconds.  Later entries are
        // read one page ahead (the wait for a free stage hides the load).
        // A page past the table's row reads as -1, a bad index.
        int32_t head[nst];
#pragma unroll
        for (int i = 0; i < nst; ++i) head[i] = (p0 + i < p1 && p0 + i < p.max_pages) ? bt[p0 + i] : -1;
        int32_t bt_next = -1;
        // This producer runs kStages pages ahead: start this item's Q rows
        // towards L2 now, so that the softmax warps' Q loads at the item
        // boundary do not wait on DRAM behind the page stream (rank 0 fetches
        // whole rows for both CTAs; q rows are contiguous, 1152 B each).
        if (rank == 0 && p1 > p0) {
          const uint8_t* qb =
              reinterpret_cast<const uint8_t*>(p.q) + (static_cast<size_t>(b) * p.M + row0) * (kDqk * 2);
          const uint32_t bytes = static_cast<uint32_t>(min(kRows, p.M - row0)) * (kDqk * 2);
          for (uint32_t o = 0; o < bytes; o += 16384u) prefetch_l2_bulk(qb + o, min(16384u, bytes - o));
        }
        for (int pg = p0; pg < p1; ++pg, ++g) {
          const uint32_t st = g % nst;
          TRACE(kTraceProducer, g, 0);
          // BF16, the CTA's first item: page 0 goes out with the Q loads, the
          // rest of the prefetch only once Q is in tensor memory.  At a
          // kernel's start every CTA loads Q and fills all its stages at
          // once; served in that order, Q and page 0 arrive first and the
          // tensor pipe starts earlier while the other pages stream in behind
          // them (uniform batch 103.4 -> 101.4 us).  FP8 keeps its raw stages
          // filling from the start: its dequant warps need them first (2%
          // slower with the same order).
          if (!kFp8 && it == it_begin && pg == p0 + 1 &&
              !mbar_wait(BAR(C::kQReady), 0, abort_flag, p.timeout_ns)) {
            raise_abort(p, abort_flag);
            ok = false;
            break;
          }
          if (g >= static_cast<uint32_t>(nst) &&
              !mbar_wait(BAR(empty0 + st), ((g / nst) & 1u) ^ 1u, abort_flag, p.timeout_ns)) {
            raise_abort(p, abort_flag);
            ok = false;
            break;
          }
          // A page past the block table's row (cache_seqlens larger than
          // 64 * max_pages) is treated like a bad block index.
          const int j = pg - p0;
          long long phys = bt_next;
#pragma unroll
          for (int i = 0; i < nst; ++i)
            if (j == i) phys = head[i];
          if (j + 1 >= nst && pg + 1 < p1) bt_next = (pg + 1 < p.max_pages) ? bt[pg + 1] : -1;
          if (phys < 0 || phys >= p.num_blocks) {
            report_status(p.status, kStatusBadBlock);
            phys = 0;
          }
          const int y = static_cast<int>(phys) * kPage;
          const uint32_t fb = BAR(full0 + st);
          if constexpr (kFp8) {
            const uint32_t dst = rawbuf0 + st * C::kRawStageBytes;
            mbar_arrive_expect_tx(fb, kRawBytes);
            tma_load_2d(dst, &tm_a, fb, static_cast<int>(rank) * 256, y);
            tma_load_2d(dst + kRawLatBytes, &tm_b, fb, 512, y);
            tma_load_2d(dst + kRawLatBytes + kRawScaleBytes, &tm_c, fb, 528 + static_cast<int>(rank) * 64, y);
          } else {
            const uint32_t dst = stage0 + st * kStageBytes;
            mbar_arrive_expect_tx(fb, kStageBytes);
#pragma unroll
            for (int c = 0; c < 4; ++c)
              tma_load_2d(dst + c * kChunkBytes, &tm_a, fb, static_cast<int>(rank) * 256 + c * 64, y);
            tma_load_2d(dst + 4 * kChunkBytes, &tm_b, fb, 512 + static_cast<int>(rank) * 32, y);
          }
          TRACE(kTraceProducer, g, 1);
        }
      }
      // Never leave a copy landing in shared memory after the CTA exits.
      for (uint32_t k = (g > static_cast<uint32_t>(nst) ? g - nst : 0u); k < g; ++k)
        mbar_wait(BAR(full0 + k % nst), (k / nst) & 1u, &g_never_abort, 100000000ull);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------------ QK^T issuer
    if (lane == 0) {
      constexpr uint32_t idesc_qk = idesc_bf16(128, 64, false, false);
      // The descriptor's address field is (shared address >> 4) in its low
      // bits, so a byte offset o within the window is added as o >> 4.
      const uint64_t d_lat = sdesc(stage0, 16, 1024, kSwizzle128);
      const uint64_t d_rope = sdesc(stage0 + 4 * kChunkBytes, 16, 512, kSwizzle64);
      const uint64_t d_qrope = sdesc(base + C::kQRopeOffset, 16, 512, kSwizzle64);
      uint32_t g = 0, nitem = 0;
      bool ok = true;
      for (int it = it_begin; it < it_end && ok; ++it) {
        const int n = items[4 * it + 2] - items[4 * it + 1];
        if (n <= 0) continue;
        if (!mbar_wait(BAR(C::kQReady), nitem & 1u, abort_flag, p.timeout_ns)) { ok = false; break; }
        ++nitem;
        for (int j = 0; j < n; ++j, ++g) {
          const uint32_t st = g % kStages;
          TRACE(kTraceQk, g, 0);
          if (!mbar_wait(BAR(C::kFull + st), (g / kStages) & 1u, abort_flag, p.timeout_ns)) { ok = false; break; }
          TRACE(kTraceQk, g, 1);
          if (g > 0 && !mbar_wait(BAR(C::kSFree), (g - 1) & 1u, abort_flag, p.timeout_ns)) { ok = false; break; }
          TRACE(kTraceQk, g, 2);
          tc_fence_after();
          const uint64_t so = static_cast<uint64_t>((st * kStageBytes) >> 4);
#pragma unroll
          for (int ks = 0; ks < 16; ++ks)
            mma_ts(tmem + kColS, tmem + kColQ + ks * 8, d_lat + so + (((ks >> 2) * kChunkBytes + (ks & 3) * 32) >> 4),
                   idesc_qk, ks > 0 ? 1u : 0u);
#pragma unroll
          for (int ks = 0; ks < 2; ++ks) mma_ss(tmem + kColS, d_qrope + 2 * ks, d_rope + so + 2 * ks, idesc_qk, 1u);
          tc_commit(BAR(C::kSFull + (g & 1u)));
          TRACE(kTraceQk, g, 3);
        }
      }
      if (!ok) raise_abort(p, abort_flag);
      // All issued MMAs complete before tensor memory is released.
      tc_commit(BAR(C::kDrain));
      mbar_wait(BAR(C::kDrain), 0, &g_never_abort, 100000000ull);
    }
  } else if (warp == 3) {
    // ------------------------------------------------------------------ PV issuer
    if (lane == 0) {
      constexpr uint32_t idesc_pv = idesc_bf16(128, 256, false, true);
      const uint64_t d_v = sdesc(stage0, 8192, 1024, kSwizzle128);
      uint32_t g = 0;
      bool ok = true;
      for (int it = it_begin; it < it_end && ok; ++it) {
        const int n = items[4 * it + 2] - items[4 * it + 1];
        for (int j = 0; j < n; ++j, ++g) {
          const uint32_t pb = g & 1u;
          TRACE(kTracePv, g, 0);
          if (p.hold_flag != nullptr && static_cast<int>(g) == p.hold_tile && !hold_until_flag(p, abort_flag)) {
            ok = false;
            break;
          }
          if (!mbar_wait(BAR(C::kPFull + pb), (g >> 1) & 1u, abort_flag, p.timeout_ns)) { ok = false; break; }
          TRACE(kTracePv, g, 1);
          tc_fence_after();
          const uint64_t so = static_cast<uint64_t>(((g % kStages) * kStageBytes) >> 4);
#pragma unroll
          for (int ks = 0; ks < 4; ++ks)
            mma_ts(tmem + kColO, tmem + kColP + pb * 32 + ks * 8, d_v + so + ks * (2048 >> 4), idesc_pv,
                   (j == 0 && ks == 0) ? 0u : 1u);
          tc_commit(BAR(C::kPvDone + pb));
          tc_commit(BAR(C::kEmpty + g % kStages));
          TRACE(kTracePv, g, 2);
        }
      }
      if (!ok) raise_abort(p, abort_flag);
      tc_commit(BAR(C::kDrain + 1));
      mbar_wait(BAR(C::kDrain + 1), 0, &g_never_abort, 100000000ull);
    }
  }
    __syncwarp();
    static_assert(kCtlRegs == kTailRegs, "the control warps stay at their budget for the tail");
  } else if (warp < 4 + kSoftmaxWarps) {
    // ------------------------------------------------------------------ softmax / epilogue
    if constexpr (kFp8) setmaxnreg_inc<kRegSoftmax>();
    const int wg = (warp - 4) >> 2;         // warpgroup: the tiles g with g % 2 == wg
    const int wq = warp & 3;                // tensor-memory lane quarter
    const int r = wq * 32 + lane;           // query row == tensor-memory lane
    const int wt = threadIdx.x - 128 * (1 + wg);  // 0..127 within the warpgroup
    const uint32_t trow = tmem + (static_cast<uint32_t>(wq * 32) << 16);
    const uint32_t xpeer = mapa_shared(xbuf0, peer);
    const uint32_t xbar_peer = mapa_shared(BAR(C::kXFull), peer);
    const uint32_t xfree_peer = mapa_shared(BAR(C::kXFree), peer);
    const uint8_t* xlocal = sbase + C::kXOffset;
    volatile float* ref_slot = reinterpret_cast<volatile float*>(sbase + C::kRefSlotOffset);
    ref_slot[wg * kRows + r] = -CUDART_INF_F;
    float* comb_slot = reinterpret_cast<float*>(sbase + C::kCombSlotOffset);
    float* epi_slot = reinterpret_cast<float*>(sbase + C::kEpiOffset);
    const float c_log2 = p.scale_log2;
    const float c_abs = fabsf(c_log2);
    const bool c_neg = c_log2 < 0.f;
    uint32_t g = 0;      // tile counter of this CTA (every tile, both warpgroups)
    uint32_t nitem = 0;  // items with at least one page
    bool ok = true;
    const int mt = rows_per_tile(p.M);  // partial-result rows per slot
    for (int it = it_begin; it < it_end && ok; ++it) {
      const int vb = items[4 * it], p0 = items[4 * it + 1], p1 = items[4 * it + 2], slot = items[4 * it + 3];
      const int b = vb / p.row_tiles, row0 = (vb - b * p.row_tiles) * kRows;
      const bool row_ok = row0 + r < p.M;   // this thread's row exists in the request
      const int qi = (row0 + r) / p.h_q;    // its query token
      const int L = p.seqlens[b / p.req_div];
      const int n = p1 - p0;
      const size_t orow = static_cast<size_t>(b) * p.M + row0 + r;
      if (n <= 0) {
        if (row_ok) {
          if (slot >= 0) {
            if (rank == 0 && wg == 0) p.lse_part[static_cast<size_t>(slot) * mt + r] = -CUDART_INF_F;
          } else {
            uint4* dst = reinterpret_cast<uint4*>(p.out + orow * kDv + rank * 256 + wg * 128);
            for (int v = 0; v < 16; ++v) dst[v] = make_uint4(0, 0, 0, 0);
            if (rank == 0 && wg == 0) p.lse[orow] = -CUDART_INF_F;
          }
        }
        continue;
      }
      if (wg == 0 && wt == 0) TRACE(kTraceItem, it - it_begin, 0);
      // Q -> tensor memory: this CTA's 256 latent dims as 128 packed bf16
      // pairs (warpgroup w writes columns [64 w, 64 w + 64)); the 32 RoPE dims
      // go to shared memory (SW64 K-major rows of 64 bytes), warpgroup 1.
      {
        const uint4* qrow = reinterpret_cast<const uint4*>(p.q + orow * kDqk);
        // all loads first, so their latencies overlap: 32-byte loads when q
        // is 32-byte aligned (rows are 1152 bytes, so then every row is),
        // else 16-byte ones
        uint32_t v[4][16];
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          const int e0 = static_cast<int>(rank) * 256 + (wg * 4 + c) * 32;
          if (p.q_wide) {
#pragma unroll
            for (int u = 0; u < 2; ++u) {
              if (row_ok) ld_global_v8(qrow + e0 / 8 + 2 * u, &v[c][8 * u]);
              else {
#pragma unroll
                for (int i = 0; i < 8; ++i) v[c][8 * u + i] = 0u;
              }
            }
          } else {
#pragma unroll
            for (int u = 0; u < 4; ++u) {
              const uint4 w = row_ok ? __ldg(qrow + e0 / 8 + u) : make_uint4(0, 0, 0, 0);
              v[c][4 * u + 0] = w.x;
              v[c][4 * u + 1] = w.y;
              v[c][4 * u + 2] = w.z;
              v[c][4 * u + 3] = w.w;
            }
          }
        }
#pragma unroll
        for (int c = 0; c < 4; ++c) tmem_st16(trow + kColQ + (wg * 4 + c) * 16, v[c]);
        if (wg == 1) {
          uint8_t* qr = sbase + C::kQRopeOffset + r * 64;
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const uint4 w = row_ok ? __ldg(qrow + (512 + static_cast<int>(rank) * 32) / 8 + u) : make_uint4(0, 0, 0, 0);
            *reinterpret_cast<uint4*>(qr + ((u ^ ((r >> 1) & 3)) << 4)) = w;
          }
          fence_proxy_async_smem();
        }
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(BAR(C::kQReady));
        if (wg == 0 && wt == 0) TRACE(kTraceItem, it - it_begin, 1);
      }
      const int vis = p.causal ? min(L, L - p.s_q + qi + 1) : L;
      // every row sees at least this many keys: tiles below it need no mask
      const int vis_all = p.causal ? max(0, L - p.s_q + 1) : L;
      const int last_page = (L - 1) / kPage;
      float ref_own = -CUDART_INF_F;  // this warpgroup's lazy reference of row r
      float l = 0.f;                  // this warpgroup's part of the row sum ...
      float m_l = -CUDART_INF_F;      // ... at this combined reference (log2 units)

#pragma unroll 1
      for (int j = wg ^ static_cast<int>(g & 1u); j < n; j += 2) {
        const uint32_t gg = g + static_cast<uint32_t>(j);
        const int pg = p0 + j;
        // ---------------------------------------------------------------- produce
        // read the partial logits of tile gg, fix the row's lazy reference,
        // exponentiate, send the fp16 factors (+ reference) to the peer CTA
        if (wt == 0) TRACE(kTraceSoftmax, gg, 0);
        if (!warp_wait(BAR(C::kSFull + (gg & 1u)), (gg >> 1) & 1u, abort_flag, p.timeout_ns)) { ok = false; break; }
        if (wt == 0) TRACE(kTraceSoftmax, gg, 1);
        tc_fence_after();
        uint32_t s[64];
        tmem_ld64(trow + kColS, s);
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(BAR(C::kSFree));
        if (wt == 0) TRACE(kTraceSoftmax, gg, 2);
        const int tok0 = pg * kPage;
        // Sparse decode: the tile's validity mask, written by the dequant warps
        // before they completed the stage's full barrier; acquiring that
        // (already completed) phase makes the write visible here.  The stage
        // is not refilled before this tile's P*V, so the mask stays put.
        uint64_t vmask = ~0ull;
        if constexpr (kSparse) {
          const uint32_t st = gg % kStages;
          if (!warp_wait(BAR(C::kFull + st), (gg / kStages) & 1u, abort_flag, p.timeout_ns)) { ok = false; break; }
          vmask = *reinterpret_cast<const volatile uint64_t*>(sbase + C::kStageMaskOffset + 8 * st);
        }
        const bool full_tile = kSparse ? (vmask == ~0ull) : (tok0 + kPage <= vis_all);
        float e[64];
        float tmax;
        {
          float a[4] = {-CUDART_INF_F, -CUDART_INF_F, -CUDART_INF_F, -CUDART_INF_F};
          if (full_tile) {
            // max of the raw products; the scale's sign decides max or min
            if (!c_neg) {
#pragma unroll
              for (int t = 0; t < 32; ++t)
                a[t & 3] = fmax3(a[t & 3], __uint_as_float(s[2 * t]), __uint_as_float(s[2 * t + 1]));
            } else {
#pragma unroll
              for (int t = 0; t < 32; ++t)
                a[t & 3] = fmax3(a[t & 3], -__uint_as_float(s[2 * t]), -__uint_as_float(s[2 * t + 1]));
            }
            tmax = fmaxf(fmaxf(a[0], a[1]), fmaxf(a[2], a[3])) * c_abs;
          } else {
#pragma unroll
            for (int t = 0; t < 64; ++t) {
              const bool key = kSparse ? ((vmask >> t) & 1ull) != 0 : (tok0 + t < vis);
              e[t] = key ? __uint_as_float(s[t]) * c_log2 : -CUDART_INF_F;
            }
#pragma unroll
            for (int t = 0; t < 32; ++t) a[t & 3] = fmax3(a[t & 3], e[2 * t], e[2 * t + 1]);
            tmax = fmaxf(fmaxf(a[0], a[1]), fmaxf(a[2], a[3]));
          }
        }
        // the reference: this warpgroup's last one, raised to the other
        // warpgroup's latest (read without waiting; any value works, and the
        // two converge after a tile or two)
        if (wt == 0) TRACE(kTraceSoftmax, gg, 3);
        const float prev = fmaxf(ref_own, ref_slot[(wg ^ 1) * kRows + r]);
        const float ref = (tmax > prev + kRescaleThreshold) ? tmax : prev;
        ref_own = ref;
        ref_slot[wg * kRows + r] = ref;
        const float msub = (ref == -CUDART_INF_F) ? 0.f : ref;
        constexpr uint32_t kXBuffers = C::kXBuffers;
        const uint32_t xb = gg % kXBuffers;
        if (wt == 0) {
          mbar_arrive_expect_tx(BAR(C::kXFull + 2 * xb), kXERegionBytes / 2);
          mbar_arrive_expect_tx(BAR(C::kXFull + 2 * xb + 1), kXMsgBytes - kXERegionBytes / 2);
        }
        // the peer has read tile gg - 2's message out of the same buffer
        if (gg >= static_cast<uint32_t>(kXBuffers) &&
            !warp_wait<true>(BAR(C::kXFree + xb), ((gg - kXBuffers) / kXBuffers) & 1u, abort_flag, p.timeout_ns)) {
          ok = false;
          break;
        }
        if (wt == 0) TRACE(kTraceSoftmax, gg, 4);
        {
          // Exponentiate and send in two halves of 32 tokens: the first half
          // crosses to the peer while the second is computed.
          const uint32_t rx = xpeer + xb * kXBufBytes;
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            const uint32_t rbar = xbar_peer + 8u * (2 * xb + h);
            if (full_tile) {
              // the exponent arguments in packed fp32 pairs (one FFMA2 per two)
              const float2 c2 = make_float2(c_log2, c_log2), nm2 = make_float2(-msub, -msub);
#pragma unroll
              for (int t = 32 * h; t < 32 * h + 32; t += 2) {
                const float2 x =
                    __ffma2_rn(make_float2(__uint_as_float(s[t]), __uint_as_float(s[t + 1])), c2, nm2);
                e[t] = ex2_approx(x.x);
                e[t + 1] = ex2_approx(x.y);
              }
            } else {
#pragma unroll
              for (int t = 32 * h; t < 32 * h + 32; ++t) e[t] = ex2_approx(e[t] - msub);
            }
#pragma unroll
            for (int c = 4 * h; c < 4 * h + 4; ++c)
              st_async_v4u(rx + (c * kRows + r) * 16, pack_f16x2(e[8 * c + 0], e[8 * c + 1]),
                           pack_f16x2(e[8 * c + 2], e[8 * c + 3]), pack_f16x2(e[8 * c + 4], e[8 * c + 5]),
                           pack_f16x2(e[8 * c + 6], e[8 * c + 7]), rbar);
          }
          st_async_b32(rx + kXERegionBytes + r * 4, __float_as_uint(ref), xbar_peer + 8u * (2 * xb + 1));
        }
        if (wt == 0) TRACE(kTraceSoftmax, gg, 5);
        // ---------------------------------------------------------------- consume
        // combine with the peer's factors into P, rescale O when the combined
        // reference moved, hand P to the PV MMA
        // The two halves of the peer's message complete separately: P of
        // tokens 0-31 is formed while tokens 32-63 (and the reference, which
        // P itself does not need) are still crossing.
        const uint8_t* xs = xlocal + xb * kXBufBytes;
        uint32_t pk[32];
        float2 rs2[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};  // row-sum partials, packed pairs
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          if (!warp_wait<true>(BAR(C::kXFull + 2 * xb + h), (gg / kXBuffers) & 1u, abort_flag, p.timeout_ns)) {
            ok = false;
            break;
          }
          if (wt == 0 && h == 0) TRACE(kTraceSoftmax, gg, 6);
#pragma unroll
          for (int c = 4 * h; c < 4 * h + 4; ++c) {
            const uint4 w = *reinterpret_cast<const uint4*>(xs + (c * kRows + r) * 16);
            const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              const float2 a = __fmul2_rn(make_float2(e[8 * c + 2 * q], e[8 * c + 2 * q + 1]), unpack_f16x2(ww[q]));
              rs2[q & 1] = __fadd2_rn(rs2[q & 1], a);
              pk[4 * c + q] = pack_bf16x2(a.x, a.y);
            }
          }
        }
        if (!ok) break;
        if (wt == 0) TRACE(kTraceSoftmax, gg, 7);
        const float m_new = ref + *reinterpret_cast<const float*>(xs + kXERegionBytes + r * 4);
        const float rowsum = (rs2[0].x + rs2[1].x) + (rs2[0].y + rs2[1].y);
        {
          // This warp is done with the peer's message: hand the buffer back
          // now, before the reference chain.  m_new and rowsum depend on every
          // value loaded from the buffer, and the arrive's address depends on
          // both through an opaque zero, so it issues only after those loads
          // have completed; a relaxed arrive is then enough to keep the peer's
          // next write behind them.
          uint32_t z;
          asm volatile("{\n .reg .b32 t;\n xor.b32 t, %1, %2;\n and.b32 %0, t, 0;\n}\n"
                       : "=r"(z) : "r"(__float_as_uint(m_new)), "r"(__float_as_uint(rowsum)));
          __syncwarp();
          if (lane == 0) mbar_arrive_remote_relaxed(xfree_peer + 8u * xb + z);
        }
        if (gg > 0 && !warp_wait(BAR(C::kCChain), (gg - 1u) & 1u, abort_flag, p.timeout_ns)) { ok = false; break; }
        if (wt == 0) TRACE(kTraceSoftmax, gg, 8);
        const float m_prev = j > 0 ? comb_slot[r] : -CUDART_INF_F;
        comb_slot[r] = m_new;
        mbar_arrive(BAR(C::kCChain));
        const uint32_t pb = gg & 1u;
        // P buffer pb was last read by PV(gg - 2)
        if (gg >= 2) {
          if (!warp_wait(BAR(C::kPvDone + pb), ((gg - 2) >> 1) & 1u, abort_flag, p.timeout_ns)) { ok = false; break; }
          tc_fence_after();
        }
        if (wt == 0) TRACE(kTraceSoftmax, gg, 9);
        const bool moved = m_new != m_prev;
        if (j > 0 && __any_sync(0xffffffffu, moved)) {
          // O must be stable: PV(gg - 1) done
          if (!warp_wait(BAR(C::kPvDone + (pb ^ 1u)), ((gg - 1) >> 1) & 1u, abort_flag, p.timeout_ns)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const float factor = moved ? ((m_prev == -CUDART_INF_F) ? 0.f : ex2_approx(m_prev - m_new)) : 1.f;
#pragma unroll 1
          for (int cc = 0; cc < 8; ++cc) {
            uint32_t o[32];
            const uint32_t col = kColO + cc * 32;
            tmem_ld32(trow + col, o);
#pragma unroll
            for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * factor);
            tmem_st16(trow + col, *reinterpret_cast<uint32_t(*)[16]>(&o[0]));
            tmem_st16(trow + col + 16, *reinterpret_cast<uint32_t(*)[16]>(&o[16]));
          }
        }
        if (wt == 0) TRACE(kTraceSoftmax, gg, 10);
        if (m_new != m_l) {
          l = (m_l == -CUDART_INF_F) ? 0.f : l * ex2_approx(m_l - m_new);
          m_l = m_new;
        }
        l += rowsum;
        if constexpr (!kFp8) {
          // Slots past the end of the request on its last page may hold NaN/Inf:
          // zero those V rows so that 0 * garbage cannot reach O.  (The FP8
          // dequant warps write zeros there themselves.)
          if (pg == last_page && (L & (kPage - 1))) {
            const int t0 = L & (kPage - 1);
            uint8_t* stg = sbase + (gg % kStages) * kStageBytes;
            for (int u = wt; u < (kPage - t0) * 32; u += 128) {
              const int row = t0 + (u >> 5), w = u & 31;
              *reinterpret_cast<uint4*>(stg + (w >> 3) * kChunkBytes + row * 128 + (w & 7) * 16) =
                  make_uint4(0, 0, 0, 0);
            }
            fence_proxy_async_smem();
          }
        }
        tmem_st16(trow + kColP + pb * 32, *reinterpret_cast<const uint32_t(*)[16]>(&pk[0]));
        tmem_st16(trow + kColP + pb * 32 + 16, *reinterpret_cast<const uint32_t(*)[16]>(&pk[16]));
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(BAR(C::kPFull + pb));
        if (wt == 0) TRACE(kTraceSoftmax, gg, 11);
      }
      if (!ok) break;
      // epilogue: both warpgroups' row sums at the combined reference of the
      // item's last tile, then this warpgroup's 128 columns of O
      if (wg == 0 && wt == 0) TRACE(kTraceItem, it - it_begin, 2);
      const uint32_t glast = g + static_cast<uint32_t>(n) - 1u;
      g += static_cast<uint32_t>(n);
      float m_fin = m_l;  // this warpgroup consumed the last tile
      if ((glast & 1u) != static_cast<uint32_t>(wg)) {
        if (!warp_wait(BAR(C::kCChain), glast & 1u, abort_flag, p.timeout_ns)) { ok = false; break; }
        m_fin = comb_slot[r];
      }
      if (wg == 0 && wt == 0) TRACE(kTraceItem, it - it_begin, 4);
      const float lw = (m_l == -CUDART_INF_F) ? 0.f : l * ex2_approx(m_l - m_fin);
      epi_slot[wg * kRows + r] = lw;
      ref_slot[wg * kRows + r] = -CUDART_INF_F;  // the next item starts afresh
      mbar_arrive(BAR(C::kEpi));
      if (!warp_wait(BAR(C::kEpi), nitem & 1u, abort_flag, p.timeout_ns)) { ok = false; break; }
      if (wg == 0 && wt == 0) TRACE(kTraceItem, it - it_begin, 5);
      ++nitem;
      const float lt = lw + epi_slot[(wg ^ 1) * kRows + r];
      if (!warp_wait(BAR(C::kPvDone + (glast & 1u)), (glast >> 1) & 1u, abort_flag, p.timeout_ns)) {
        ok = false;
        break;
      }
      if (wg == 0 && wt == 0) TRACE(kTraceItem, it - it_begin, 6);
      tc_fence_after();
      const float inv = lt > 0.f ? 1.f / lt : 0.f;
      const float lse_val = lt > 0.f ? (m_fin + __log2f(lt)) * 0.69314718055994531f : -CUDART_INF_F;
#pragma unroll 1
      for (int cc = 0; cc < 4; ++cc) {
        uint32_t o[32];
        const int col = wg * 128 + cc * 32;  // within this CTA's 256 columns
        tmem_ld32(trow + kColO + col, o);
        if (row_ok) {
          // Each thread writes its own row: 32-byte stores (a whole sector
          // per lane) when the buffers allow, else 16-byte ones.
          if (slot < 0) {
            uint16_t* dst = p.out + orow * kDv + rank * 256 + col;
#pragma unroll
            for (int h = 0; h < 2; ++h) {
              uint32_t w[8];
#pragma unroll
              for (int i = 0; i < 8; ++i)
                w[i] = pack_bf16x2(__uint_as_float(o[16 * h + 2 * i]) * inv, __uint_as_float(o[16 * h + 2 * i + 1]) * inv);
              if (p.out_wide) {
                st_global_v8(dst + 16 * h, w[0], w[1], w[2], w[3], w[4], w[5], w[6], w[7]);
              } else {
                uint4* d4 = reinterpret_cast<uint4*>(dst + 16 * h);
                d4[0] = make_uint4(w[0], w[1], w[2], w[3]);
                d4[1] = make_uint4(w[4], w[5], w[6], w[7]);
              }
            }
          } else {
            float* dst = p.o_part + (static_cast<size_t>(slot) * mt + r) * kDv + rank * 256 + col;
#pragma unroll
            for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * inv);
            if (p.out_wide) {
#pragma unroll
              for (int v = 0; v < 4; ++v)
                st_global_v8(dst + 8 * v, o[8 * v], o[8 * v + 1], o[8 * v + 2], o[8 * v + 3], o[8 * v + 4],
                             o[8 * v + 5], o[8 * v + 6], o[8 * v + 7]);
            } else {
              float4* d4 = reinterpret_cast<float4*>(dst);
#pragma unroll
              for (int v = 0; v < 8; ++v)
                d4[v] = make_float4(__uint_as_float(o[4 * v]), __uint_as_float(o[4 * v + 1]),
                                    __uint_as_float(o[4 * v + 2]), __uint_as_float(o[4 * v + 3]));
            }
          }
        }
      }
      if (row_ok && rank == 0 && wg == 0) {
        if (slot < 0) p.lse[orow] = lse_val;
        else p.lse_part[static_cast<size_t>(slot) * mt + r] = lse_val;
      }
      if (wg == 0 && wt == 0) TRACE(kTraceItem, it - it_begin, 3);
    }
    if (!ok) raise_abort(p, abort_flag);
    __syncwarp();
    if constexpr (kFp8) setmaxnreg_dec<kTailRegs>();
  } else if (kFp8) {
    // ------------------------------------------------------------------ FP8 dequant (warps 12-15)
    setmaxnreg_dec<kDqRegs>();
    // Raw 656-byte tokens -> this CTA's bf16 page half, in the same swizzled
    // layout the BF16 path gets from TMA.  Thread dt handles 16-code units
    // u = dt + 128 k: token u / 16, codes 16 (u % 16) .. +16 of the CTA's 256.
    constexpr int kDqThreads = 32 * kDqWarps;
    const int dt = threadIdx.x - 128 - kSoftmaxWarps * 32;
    uint32_t g = 0;
    bool ok = true;
    for (int it = it_begin; it < it_end && ok; ++it) {
      const int p0 = items[4 * it + 1], p1 = items[4 * it + 2];
      const int L = p.seqlens[items[4 * it] / p.row_tiles / p.req_div];
      const int last_page = (L - 1) / kPage;
      for (int pg = p0; pg < p1; ++pg, ++g) {
        const uint32_t rs = g % C::kRawStages, st = g % kStages;
        if (dt == 0) TRACE(kTraceDequant, g, 0);
        if (!warp_wait(BAR(C::kRawFull + rs), (g / C::kRawStages) & 1u, abort_flag, p.timeout_ns)) { ok = false; break; }
        if (dt == 0) TRACE(kTraceDequant, g, 1);
        if (g >= static_cast<uint32_t>(kStages) &&
            !warp_wait(BAR(C::kEmpty + st), ((g / kStages) & 1u) ^ 1u, abort_flag, p.timeout_ns)) { ok = false; break; }
        if (dt == 0) TRACE(kTraceDequant, g, 2);
        // Token t of the tile is a key: t below the request's length on its
        // last page, or (sparse) its bit in the mask the gather wrote.
        const int valid = (pg == last_page) ? L - pg * kPage : kPage;
        uint64_t tmask = 0;
        if constexpr (kSparse) tmask = *reinterpret_cast<const volatile uint64_t*>(sbase + C::kRawMaskOffset + 8 * rs);
        const uint8_t* rlat = sbase + C::kRawOffset + rs * C::kRawStageBytes;
        // where token t's scales and this CTA's RoPE half are: the dense copy
        // lays them out as [64][16] and [64][64]; the sparse gather brings
        // bytes 496-655 of each token as one 160-byte row
        const uint8_t* rscale = rlat + kRawLatBytes + (kSparse ? 512 - kTailX : 0);
        const uint8_t* rrope = kSparse ? rlat + kRawLatBytes + (528 - kTailX) + 64 * static_cast<int>(rank)
                                       : rlat + kRawLatBytes + kRawScaleBytes;
        constexpr int kScaleStride = kSparse ? kTailBytes : 16;
        constexpr int kRopeStride = kSparse ? kTailBytes : 64;
        uint8_t* dst = sbase + st * kStageBytes;
#pragma unroll 2
        for (int k = 0; k < 1024 / kDqThreads; ++k) {
          const int u = dt + kDqThreads * k;
          const int t = u >> 4, g16 = u & 15;
          uint32_t w[8];
          if (kSparse ? ((tmask >> t) & 1ull) != 0 : t < valid) {
            const uint4 codes = *reinterpret_cast<const uint4*>(rlat + t * 256 + g16 * 16);
            const float sc =
                *reinterpret_cast<const float*>(rscale + t * kScaleStride + 4 * (2 * static_cast<int>(rank) + (g16 >> 3)));
            dequant16(codes, sc, w);
          } else {
#pragma unroll
            for (int i = 0; i < 8; ++i) w[i] = 0u;
          }
          uint8_t* row = dst + (g16 >> 2) * kChunkBytes + t * 128;
          const int u0 = (g16 & 3) * 2;
          *reinterpret_cast<uint4*>(row + ((u0 ^ (t & 7)) << 4)) = make_uint4(w[0], w[1], w[2], w[3]);
          *reinterpret_cast<uint4*>(row + (((u0 + 1) ^ (t & 7)) << 4)) = make_uint4(w[4], w[5], w[6], w[7]);
        }
#pragma unroll
        for (int k = 0; k < 256 / kDqThreads; ++k) {
          const int u = dt + kDqThreads * k;
          const int t = u >> 2, w4 = u & 3;
          uint4 v = make_uint4(0, 0, 0, 0);
          if (kSparse ? ((tmask >> t) & 1ull) != 0 : t < valid)
            v = *reinterpret_cast<const uint4*>(rrope + t * kRopeStride + w4 * 16);
          *reinterpret_cast<uint4*>(dst + 4 * kChunkBytes + t * 64 + ((w4 ^ ((t >> 1) & 3)) << 4)) = v;
        }
        // sparse: the mask goes with the bf16 stage to the softmax warps
        if (kSparse && dt == 0) *reinterpret_cast<volatile uint64_t*>(sbase + C::kStageMaskOffset + 8 * st) = tmask;
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(BAR(C::kFull + st));
          mbar_arrive(BAR(C::kRawEmpty + rs));
        }
        if (dt == 0) TRACE(kTraceDequant, g, 3);
      }
    }
    if (!ok) raise_abort(p, abort_flag);
    __syncwarp();
    if constexpr (kDqRegs != kTailRegs) setmaxnreg_dec<kTailRegs>();
  }

  tc_fence_before();
  __syncthreads();
  if (threadIdx.x == 0) TRACE(kTraceCta, 0, 3);
  // Teardown.  In the normal path the peer has waited for every message this
  // CTA sent it, so no transfer is in flight and one cluster barrier suffices.
  // After an abort the peer may have stopped consuming, and distributed-
  // shared-memory stores or remote arrives issued here may still be on their
  // way to it.  Each CTA therefore tells the other whether it gave up; if
  // either did, both let such transfers land (they take about a microsecond;
  // the wait is 50 us) before a second cluster barrier, after which either
  // CTA may exit and release its shared memory.
  volatile int* peer_abort = reinterpret_cast<volatile int*>(sbase + C::kBarOffset + C::kNumBars * 8 + 8);
  if (threadIdx.x == 0)
    st_cluster_u32(mapa_shared(base + C::kBarOffset + C::kNumBars * 8 + 8, peer), static_cast<uint32_t>(*abort_flag));
  cluster_sync();
  if (*abort_flag != 0 || *peer_abort != 0) {
    if (threadIdx.x == 0) {
      const uint64_t t0 = globaltimer_ns();
#pragma unroll 1
      for (int i = 0; i < 1000 && globaltimer_ns() - t0 < 50000ull; ++i) __nanosleep(1000);
    }
    __syncthreads();
    cluster_sync();
  }
  if (threadIdx.x == 0) TRACE(kTraceCta, 0, 4);
  if (warp == 2) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
#undef BAR
}

template <bool kFp8, bool kSparse>
static cudaError_t launch_decode(const CUtensorMap& tm_a, const CUtensorMap& tm_b, const CUtensorMap& tm_c,
                                 const DecodeParams& p, int num_parts, cudaStream_t stream) {
  using C = dk::Cfg<kFp8, kSparse>;
  // The shared-memory opt-in is an attribute of the function on each device:
  // set it once per device (a bit per device below 64; devices above that set
  // it on every launch).  Racing host threads may both set it, which is
  // harmless.
  static std::atomic<unsigned long long> attr_done{0};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const unsigned long long bit = dev < 64 ? (1ull << dev) : 0ull;
  if (bit == 0 || (attr_done.load(std::memory_order_acquire) & bit) == 0) {
    e = cudaFuncSetAttribute(decode_kernel<kFp8, kSparse>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             C::kSmemBytes);
    if (e != cudaSuccess) return e;
    attr_done.fetch_or(bit, std::memory_order_acq_rel);
  }
  // Programmatic dependent launch: the CTAs start (barriers, tensor memory)
  // while the metadata kernel finishes, and wait in the kernel before
  // reading the schedule.
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2 * num_parts);
  cfg.blockDim = dim3(C::kThreads);
  cfg.dynamicSmemBytes = C::kSmemBytes;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, decode_kernel<kFp8, kSparse>, tm_a, tm_b, tm_c, p);
}

cudaError_t launch_decode_bf16(const CUtensorMap& tm_lat, const CUtensorMap& tm_rope, const DecodeParams& p,
                               int num_parts, cudaStream_t stream) {
  return launch_decode<false, false>(tm_lat, tm_rope, tm_rope, p, num_parts, stream);
}

cudaError_t launch_decode_fp8(const CUtensorMap& tm_lat, const CUtensorMap& tm_scale, const CUtensorMap& tm_rope,
                              const DecodeParams& p, int num_parts, cudaStream_t stream) {
  return launch_decode<true, false>(tm_lat, tm_scale, tm_rope, p, num_parts, stream);
}

// The sparse decode gathers rows: tm_lat has a (256 x 1)-byte box, tm_tail a
// (160 x 1)-byte one, both over the cache viewed as [num_blocks * 64, 656].
cudaError_t launch_decode_sparse_fp8(const CUtensorMap& tm_lat, const CUtensorMap& tm_tail, const DecodeParams& p,
                                     int num_parts, cudaStream_t stream) {
  return launch_decode<true, true>(tm_lat, tm_tail, tm_tail, p, num_parts, stream);
}

}  // namespace mla

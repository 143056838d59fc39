/*
 * mla.h — C ABI of the B200 (sm_100a) MLA paged-KV decoding library.
 *
 * Operation (FlashMLA, an MLA decoding kernel for batches of
 * variable-length sequences over a BF16 cache paged in 64-token blocks, as
 * the DeepSeek launch tweet on the 8bitnewsroom page describes it; MLA's
 * shared compressed latent KV with decoupled RoPE: Novita AI page, section
 * "Was ist MLA?" and its MHA/MQA/GQA/MLA table):
 *
 *   For request b with L = cache_seqlens[b] cached tokens, query token i in
 *   [0, s_q) and head h in [0, h_q):
 *     K_j   = key of token j: 576 values (512 latent + 64 RoPE), read from
 *             physical block block_table[b, j / 64], slot j % 64
 *     V_j   = K_j[0:512]           (the value is the latent part of the key)
 *     x_j   = softmax_scale * sum_{d<576} q[b,i,h,d] * K_j[d]
 *     visible keys: j < L, and with causal != 0 also j <= L - s_q + i
 *     lse[b,i,h]   = ln sum_j exp(x_j)                (natural log)
 *     out[b,i,h,:] = sum_j exp(x_j - lse) * V_j       (bf16, RNE)
 *   A row with no visible key gets out = 0 and lse = -inf.
 *
 * Cache formats:
 *   MLA_KV_BF16     kv_cache is bf16 [num_blocks, 64, 576] (1152 B/token).
 *   MLA_KV_FP8_656  kv_cache is uint8 [num_blocks, 64, 656] (656 B/token,
 *                   the size on the menfem.com DeepSeek page, "Key
 *                   Contributions"): bytes [0,512) E4M3 latent codes (OCP
 *                   FP8 E4M3), bytes [512,528) four little-endian fp32 scales
 *                   (scale g applies to latent dims [128g, 128g+128)), bytes
 *                   [528,656) the 64 RoPE values in bf16.  The kernel forms
 *                   code * scale in fp32 and rounds it to bf16 before the MMA.
 *
 * Conventions for every entry point:
 *   - All tensor pointers are DEVICE pointers owned by the caller; the library
 *     never allocates, frees or keeps them after the call returns.
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *     stream).  Work is enqueued asynchronously on it; nothing synchronises
 *     except mla_last_device_status().
 *   - Host-detectable argument errors return immediately (nothing enqueued).
 *   - Errors the GPU detects (a block index outside [0, num_blocks), a wait
 *     that exceeded its time limit) are recorded in a status word inside the
 *     workspace; the first error recorded is kept until cleared.
 *   - Supported shapes: d_qk 576, d_v 512, one latent KV head, 64-token
 *     blocks, M = s_q * h_q query rows per request with 1 <= M <= 1024, bf16
 *     q/out, fp32 lse; q, kv_cache and out 16-byte aligned;
 *     batch * ceil(M / 128) <= 16384.  A request with M > 128 is served as
 *     ceil(M / 128) row tiles of at most 128 rows, scheduled like separate
 *     requests that read the same pages (at about the same time, so that
 *     the second read of a page is likely to come from L2).
 */
#ifndef MLA_B200_H_
#define MLA_B200_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  MLA_OK = 0,
  MLA_ERR_INVALID_ARG = 1,     /* null pointer, bad size, misalignment, non-finite scale */
  MLA_ERR_UNSUPPORTED = 2,     /* shape outside the supported set, or no sm_100 device */
  MLA_ERR_WORKSPACE = 3,       /* workspace or schedule buffer too small */
  MLA_ERR_CUDA = 4,            /* a CUDA runtime/driver call or launch failed */
  MLA_ERR_TIMEOUT = 5,         /* device: a bounded wait gave up (kernel returned early) */
  MLA_ERR_BAD_BLOCK_INDEX = 6  /* device: block_table entry outside [0, num_blocks) */
} mla_status_t;

typedef enum { MLA_KV_BF16 = 0, MLA_KV_FP8_656 = 1 } mla_kv_format_t;

/* Human-readable name of a status code (static string, never NULL). */
const char* mla_status_string(mla_status_t status);

/* Number of CTA pairs ("SM parts") the decode kernel should use on `device`:
 * half the SM count (74 on a 148-SM B200).  Returns <= 0 if the device cannot
 * be queried. */
int mla_default_num_sm_parts(int device);

/* Bytes of the int32 schedule buffer `sched` for mla_get_metadata (0 for a
 * shape outside the supported set). */
size_t mla_metadata_size(int batch, int s_q, int h_q, int num_sm_parts);

/* Entries of the int32 `num_splits` array: batch * ceil(s_q * h_q / 128) + 1
 * (0 for a shape outside the supported set). */
int mla_num_splits_len(int batch, int s_q, int h_q);

/*
 * Split-KV schedule (the split-KV idea follows from the variable-length
 * batches the 8bitnewsroom page names as FlashMLA's target; the pages give
 * no algorithm, this one is our own).  Every request costs ceil(L/64) pages
 * plus a fixed per-request overhead; the concatenated cost line is cut into
 * num_sm_parts equal pieces, so a request may be split across CTA pairs.
 * When giving each CTA pair ceil(batch / num_sm_parts) consecutive whole
 * requests makes no pair's cost exceed the balanced cut by more than 16
 * pages, that is done instead and nothing is split (no partial outputs, no
 * combine work).
 *
 *   cache_seqlens  device int32 [batch], each >= 0
 *   s_q, h_q       query tokens and heads per request: they fix the row
 *                  tiles per request, R = ceil(s_q * h_q / 128)
 *   num_sm_parts   CTA pairs the decode launch will use (>= 1)
 *   sched          device int32 buffer of mla_metadata_size() bytes (output)
 *   num_splits     device int32 [batch * R + 1] (output): exclusive prefix
 *                  sum of the number of splits per row tile; row tile t of
 *                  request b (v = b * R + t) has num_splits[v+1] -
 *                  num_splits[v] splits.
 * The same `sched`/`num_splits` are valid for any decode call with the same
 * cache_seqlens, s_q * h_q row tiling and num_sm_parts.  One tiny kernel,
 * enqueued on `stream`.
 */
mla_status_t mla_get_metadata(const int32_t* cache_seqlens, int batch, int s_q, int h_q,
                              int num_sm_parts, int32_t* sched, int32_t* num_splits,
                              void* stream);

/* Bytes of workspace mla_decode_fwd needs: a status word plus fp32 partial
 * outputs and partial lse for split requests.  Zero-fill it once after
 * allocation (that clears the device status word). */
size_t mla_workspace_size(int batch, int s_q, int h_q, int num_sm_parts);

/*
 * MLA decode over a paged cache (the hot path).
 *
 *   q              device bf16 [batch, s_q, h_q, 576], row-major
 *   kv_cache       device, fmt-dependent (see above), [num_blocks, 64, ...]
 *   fmt            MLA_KV_BF16 or MLA_KV_FP8_656
 *   num_blocks     number of physical 64-token blocks in kv_cache (>= 1)
 *   block_table    device int32 [batch, max_pages]; only the first
 *                  ceil(L_b/64) entries of row b are read
 *   max_pages      row stride of block_table (>= 1)
 *   cache_seqlens  device int32 [batch]; L_b <= 64 * max_pages
 *   softmax_scale  finite multiplier of the logits (576^-0.5 in the configs)
 *   causal         non-zero: bottom-right causal mask among the s_q tokens
 *   sched, num_splits  from mla_get_metadata with the same num_sm_parts
 *   out            device bf16 [batch, s_q, h_q, 512] (output)
 *   lse            device fp32 [batch, s_q, h_q] (output)
 *   workspace      device buffer of >= mla_workspace_size() bytes
 * Enqueues the decode kernel and the split-KV combine kernel (whose blocks
 * exit at once when no request is split) on `stream`.  Both are launched
 * with programmatic dependent launch: their CTAs may start while the
 * previous kernel in `stream` is still running, and wait for it to complete
 * before they read or write any memory.  (Before that wait the decode CTAs
 * only issue L2 prefetch hints for q and block_table, which read no value.)
 * Tail slots of a request's last page
 * and blocks it does not reference may hold any bits (NaN/Inf included).
 * Device-detected errors (status word, see mla_last_device_status):
 *   a block_table entry outside [0, num_blocks)     MLA_ERR_BAD_BLOCK_INDEX
 *   sched made for another batch or num_sm_parts    MLA_ERR_INVALID_ARG
 *     (nothing is computed or written then)
 *   a wait that ran past its limit                  MLA_ERR_TIMEOUT
 */
mla_status_t mla_decode_fwd(const void* q, const void* kv_cache, mla_kv_format_t fmt,
                            int64_t num_blocks, const int32_t* block_table, int max_pages,
                            const int32_t* cache_seqlens, int batch, int s_q, int h_q,
                            float softmax_scale, int causal, const int32_t* sched,
                            const int32_t* num_splits, int num_sm_parts, void* out, float* lse,
                            void* workspace, size_t workspace_bytes, void* stream);

/*
 * Sparse decode over the 656-byte FP8 cache.  The menfem.com DeepSeek page
 * ("Key Contributions") names a sparse decode kernel over this cache format
 * (250 -> 410 TFLOPS on H800, up to 350 TFLOPS on B200) without defining
 * it; this library's reading:
 *
 *   For request b, query token i in [0, s_q) and head h, with
 *   L = cache_seqlens[b] and the list idx = indices[b, i, 0:topk]:
 *     the keys are K_{idx_k} for every entry with 0 <= idx_k < L (the same
 *     positions the dense decode reads through block_table); entries outside
 *     [0, L) are padding and are not keys; an entry listed twice is two
 *     terms.  There is no causal mask: the list decides what is visible.
 *     x_k = softmax_scale * q[b,i,h,:] . K_{idx_k}
 *     lse[b,i,h] = ln sum_k exp(x_k),  out[b,i,h,:] = sum_k exp(x_k - lse) V_{idx_k}
 *   A row with no valid entry gets out = 0 and lse = -inf.
 *
 *   q              device bf16 [batch, s_q, h_q, 576]; h_q <= 1024
 *   kv_cache       device uint8 [num_blocks, 64, 656], 16-byte aligned
 *   block_table    device int32 [batch, max_pages]
 *   cache_seqlens  device int32 [batch]
 *   indices        device int32 [batch, s_q, topk], 4-byte aligned
 *   topk           entries per list, 1 <= topk <= 2^24
 *   sched, num_splits  from mla_get_sparse_metadata (same batch, s_q, h_q,
 *                  topk, num_sm_parts): a schedule of batch * s_q units of
 *                  h_q rows, each of length topk
 *   out, lse       as mla_decode_fwd;  workspace >= mla_sparse_workspace_size()
 * Each CTA pair gathers the listed tokens of a 64-entry tile with TMA row
 * gathers (per CTA, its 256 latent bytes and bytes 496-655 of each token),
 * dequantises them like the dense FP8 decode and runs the same MMA and
 * softmax pipeline.  Device-
 * detected errors as mla_decode_fwd (a listed position whose page maps
 * outside [0, num_blocks): MLA_ERR_BAD_BLOCK_INDEX, that entry left out).
 */
int mla_sparse_num_splits_len(int batch, int s_q, int h_q);
size_t mla_sparse_metadata_size(int batch, int s_q, int h_q, int num_sm_parts);
size_t mla_sparse_workspace_size(int batch, int s_q, int h_q, int num_sm_parts);
mla_status_t mla_get_sparse_metadata(int batch, int s_q, int h_q, int topk, int num_sm_parts,
                                     int32_t* sched, int32_t* num_splits, void* stream);
mla_status_t mla_sparse_decode_fwd(const void* q, const void* kv_cache, int64_t num_blocks,
                                   const int32_t* block_table, int max_pages,
                                   const int32_t* cache_seqlens, const int32_t* indices, int topk,
                                   int batch, int s_q, int h_q, float softmax_scale,
                                   const int32_t* sched, const int32_t* num_splits, int num_sm_parts,
                                   void* out, float* lse, void* workspace, size_t workspace_bytes,
                                   void* stream);

/*
 * Cache append: write new tokens into the paged cache, the step that fills
 * what mla_decode_fwd reads.  The pages print only the FP8 token's size (656
 * bytes against 1,152 in BF16, RoPE slice kept in BF16: menfem.com DeepSeek
 * page, "Key Contributions") and name E4M3 (CUTLASS discussion page); the
 * quantisation below is this library's reading of that format.
 *
 *   kv_new         device bf16 [batch, s_new, 576], row-major, 16-byte aligned:
 *                  the new tokens' keys (512 latent + 64 RoPE), finite values
 *   batch, s_new   requests and new tokens per request (>= 1 each)
 *   cache_seqlens  device int32 [batch]: lengths AFTER the append (the same
 *                  array the following decode call takes).  New token t of
 *                  request b is token p = cache_seqlens[b] - s_new + t and is
 *                  written to slot p % 64 of block block_table[b, p / 64].
 *   block_table    device int32 [batch, max_pages]
 *   kv_cache       device, fmt-dependent (see above), [num_blocks, 64, ...],
 *                  16-byte aligned; only the slots of the new tokens change
 *   fmt            MLA_KV_BF16: the 1,152 bytes of each token are stored as
 *                  given.  MLA_KV_FP8_656: per 128-wide latent group g,
 *                  scale_g = amax_g / 448 and code = E4M3 (OCP, bias 7)
 *                  round-to-nearest-even of x / scale_g, saturated to +-448,
 *                  both divisions IEEE binary32; a group with amax_g = 0 gets
 *                  scale 0 and codes 0; the RoPE values are copied as bf16.
 *   workspace      device buffer whose first 4 bytes are a status word (the
 *                  decode workspace serves), >= 4 bytes, 4-byte aligned
 * One kernel (a warp per new token) enqueued on `stream`.  Device-detected
 * errors, recorded in the status word, with the token not written:
 *   p < 0 (cache_seqlens[b] < s_new)                 MLA_ERR_INVALID_ARG
 *   p / 64 >= max_pages, or a block index outside
 *   [0, num_blocks)                                  MLA_ERR_BAD_BLOCK_INDEX
 * Two new tokens that map to the same slot race; the result is one of them.
 */
mla_status_t mla_kv_append(const void* kv_new, int batch, int s_new, const int32_t* cache_seqlens,
                           const int32_t* block_table, int max_pages, void* kv_cache, mla_kv_format_t fmt,
                           int64_t num_blocks, void* workspace, size_t workspace_bytes, void* stream);

/* Synchronises `stream`, then returns the device-detected status recorded in
 * `workspace` (MLA_OK if none) or MLA_ERR_CUDA if the stream reports an error. */
mla_status_t mla_last_device_status(const void* workspace, void* stream);

/* Enqueues a reset of the workspace status word to MLA_OK on `stream`. */
mla_status_t mla_clear_device_status(void* workspace, void* stream);

/*
 * Diagnostics.  The pages have no counterpart of these calls.
 *
 * mla_set_wait_timeout_ns: every wait inside the decode kernel (for a page,
 * for the tensor cores, for the peer CTA) gives up after this many
 * nanoseconds; the kernel then records MLA_ERR_TIMEOUT in the status word,
 * drains its copies and tensor-core work, frees its tensor memory and exits,
 * leaving out/lse undefined.  The default is 2 s, far above any legitimate
 * wait; a smaller value lets a test or a watchdog see that path.  Applies to
 * decode calls enqueued after it returns, process-wide; 0 restores the
 * default.  Returns the previous value.
 */
uint64_t mla_set_wait_timeout_ns(uint64_t ns);

/*
 * mla_debug_set_trace_buffer: only a library built with MLA_TRACE defined
 * (build.py builds it as libmla_b200_trace.so) records per-tile timestamps of
 * the decode kernel: for the first 4 CTAs and their first 128 tiles, the SM
 * clock at fixed points of each warp role (layout in csrc/common.cuh), into
 * a caller-owned device buffer of mla_debug_trace_bytes() bytes, 8-byte
 * aligned.  NULL stops recording.  The product library returns
 * MLA_ERR_UNSUPPORTED and records nothing.
 */
size_t mla_debug_trace_bytes(void);
mla_status_t mla_debug_set_trace_buffer(void* buffer, size_t bytes);

/*
 * mla_debug_hold_at_tile: from the next decode call on (process-wide), the
 * thread of every CTA that issues the P*V tensor-core work waits, before the
 * tile it counts as number `tile` (from 0, over the CTA's whole run), until
 * the device int at `flag` becomes non-zero.  That wait is bounded like every
 * other one (mla_set_wait_timeout_ns).  With a flag that nothing sets, the
 * wait runs out while the pipeline is full, and the call ends through the
 * abort path: MLA_ERR_TIMEOUT in the status word, copies and tensor-core work
 * drained, tensor memory freed, the context still usable.  This is how the
 * tests exercise failure detection without faulting a GPU.  flag NULL or
 * tile < 0 turns the hold off (the default).  `flag` must be 4-byte aligned
 * and stay valid while decode calls that may hold on it run.
 */
mla_status_t mla_debug_hold_at_tile(const int* flag, int tile);

/*
 * Allocation-free decode.  The pages have no counterpart of this call: it is a
 * deployment aid of this library for callers that cannot allocate device
 * memory or pass a workspace, e.g. code running during CUDA graph capture,
 * engine plugins whose enqueue step may not allocate, or servers that have
 * already reserved all device memory for their own pool.
 *
 * Same arguments and results as mla_decode_fwd without the workspace: the
 * split-KV scratch (status word + partial results) lives in a static array
 * of MLA_NOALLOC_SCRATCH_BYTES inside the library, reserved on every GPU that
 * loads the library until the process exits.  The call allocates nothing.
 *   - Argument errors return the same codes as mla_decode_fwd, enqueuing
 *     nothing.  MLA_ERR_WORKSPACE, also with nothing enqueued, when the shape
 *     needs more scratch than the array holds, i.e. mla_workspace_size(batch,
 *     s_q, h_q, num_sm_parts) > MLA_NOALLOC_SCRATCH_BYTES (64 MiB: for 128
 *     query rows per request, batch + num_sm_parts <= 255).
 *   - The first call on a device (with that device current) looks up the
 *     array's device address; make that first call before any stream capture.
 *   - All calls share the one array and it keeps the previous call's contents;
 *     each call resets the status word on `stream` first.  Calls that can
 *     overlap on the GPU (other streams or host threads) race on the array.
 * Device-detected errors go to the status word inside the shared array;
 * mla_noalloc_last_device_status reads it (for the current device).
 */
#define MLA_NOALLOC_SCRATCH_BYTES (64u << 20)
mla_status_t mla_decode_fwd_noalloc(const void* q, const void* kv_cache, mla_kv_format_t fmt,
                                    int64_t num_blocks, const int32_t* block_table, int max_pages,
                                    const int32_t* cache_seqlens, int batch, int s_q, int h_q,
                                    float softmax_scale, int causal, const int32_t* sched,
                                    const int32_t* num_splits, int num_sm_parts, void* out,
                                    float* lse, void* stream);

/* Synchronises `stream`, then returns the device-detected status of the last
 * mla_decode_fwd_noalloc call on the current device (MLA_OK if none was
 * recorded).  The next call on the device clears it. */
mla_status_t mla_noalloc_last_device_status(void* stream);

#ifdef __cplusplus
}
#endif

#endif /* MLA_B200_H_ */

/*
 * libmla -- Multi-head Latent Attention decode over a paged KV cache, for NVIDIA B200 (sm_100a).
 *
 * The operation (FlashMLA pages: mha_fwd_kvcache_mla in the "flash_api.cpp" excerpt of the
 * mmssai.com page; get_mla_metadata / flash_mla_with_kvcache in the usage examples of the
 * kdjingpai.com, aiboss88.com and deepseekonline.chat pages; the FP8 token layout table
 * and the newer is_fp8 argument on the wmrh.cn page):
 *
 *   q        [batch, s_q, h_q, 576]            bf16   query rows (512 latent + 64 RoPE dims)
 *   kvcache  [num_blocks, 64, h_kv, 576]        bf16   paged latent cache, 64-token pages
 *            or [num_blocks, 64, 656]           u8     FP8 tokens: 512 e4m3 codes, 4 fp32
 *                                                      scales (one per 128 dims), 64 bf16 RoPE
 *   block_table [batch, max_blocks]             int32  page j of request b is block_table[b][j]
 *   cache_seqlens [batch]                       int32  tokens cached per request (L_b)
 *
 *   For request b, query position i and head h (h_kv = 1: every head reads the same cache):
 *     s_j  = softmax_scale * <q[b,i,h,:], K_b[j,:]>       over all 576 dims, j < L_b,
 *            and, if causal, j <= L_b - s_q + i          (the queries sit at the end of the cache)
 *     O[b,i,h,:] = sum_j softmax(s)_j * K_b[j, 0:512]     (V = first 512 dims of the cached vector)
 *     LSE[b,h,i] = log sum_j exp(s_j)                     (natural log; -inf if no key is visible)
 *
 *   out [batch, s_q, h_q, 512] bf16,  lse [batch, h_q, s_q] fp32.
 *
 * Conventions for every call
 *   - All pointers are DEVICE pointers unless stated otherwise; the caller owns every buffer.
 *   - Outside the serving session (mla_session_*), the library allocates no device memory and
 *     never synchronises the stream; calls are enqueued on `stream` (a cudaStream_t, NULL =
 *     legacy default stream) and return at once.
 *   - Return value: MLA_OK (0) or a negative MLA_ERR_* code.  Argument errors are detected on
 *     the host before anything is enqueued.  A CUDA launch failure returns MLA_ERR_CUDA.
 *   - Values inside device arrays (seqlens, block_table) are trusted: out-of-range page ids are
 *     not detected (the copy engine reads zeros for pages outside the cache).
 *   - Supported shapes: h_kv = 1, d_v = 512, head dim 576, page size 64, 1 <= s_q * h_q <= 4096.
 */
#ifndef MLA_H_
#define MLA_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define MLA_API __attribute__((visibility("default")))
#else
#define MLA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

#define MLA_OK 0
#define MLA_ERR_NULL_POINTER (-1)     /* a required pointer is NULL */
#define MLA_ERR_MISALIGNED (-2)       /* q, kvcache, out or workspace not 16-byte aligned; lse not 4-byte */
#define MLA_ERR_BAD_DIM (-3)          /* d_v != 512 */
#define MLA_ERR_BAD_HEADS (-4)        /* h_kv != 1, h_q < 1, or h_q % h_kv != 0 */
#define MLA_ERR_BAD_KV_DTYPE (-5)     /* kv_dtype not MLA_KV_BF16 / MLA_KV_FP8 */
#define MLA_ERR_WORKSPACE (-6)        /* workspace_bytes < mla_workspace_size(...) */
#define MLA_ERR_BAD_SHAPE (-7)        /* batch < 1, s_q < 1, num_blocks < 1, max_blocks < 1,
                                         rows out of range, or num_blocks * 64 >= 2^31 */
#define MLA_ERR_BAD_PARTS (-8)        /* num_sm_parts < 1 (pass the same value to
                                         mla_get_metadata and mla_decode_kvcache) */
#define MLA_ERR_NO_DEVICE (-9)        /* device query failed */
#define MLA_ERR_SCRATCH_LIMIT (-10)   /* mla_decode_kvcache_noalloc: the problem needs more than
                                         its 16 MiB built-in scratch array */
#define MLA_ERR_CUDA (-100)           /* a CUDA runtime / driver call failed */

#define MLA_KV_BF16 0                 /* kvcache bf16 [num_blocks, 64, 1, 576] */
#define MLA_KV_FP8 1                  /* kvcache u8   [num_blocks, 64, 656]    */

/* Device status bits written into the workspace by the kernels (sticky until reset). */
#define MLA_STATUS_WAIT_TIMEOUT 1     /* an internal pipeline wait ran past its bound (~1 s);
                                         the outputs of that call are undefined */
#define MLA_STATUS_BAD_METADATA 2     /* the tile metadata passed in was flagged by the scheduler
                                         as unbuildable (see mla_get_metadata); the call wrote
                                         O = 0 and LSE = -inf for every row */
#define MLA_STATUS_F16_RANGE 4        /* FP8 cache with more than 64 query rows per request (f16
                                         tensor-core operands): a value of q or of a RoPE dim of
                                         magnitude >= 65536, or a scale above 65504 / 448, left
                                         the f16 range; that call's outputs are unreliable */

/*
 * Number of scheduler parts ("SM parts") for a problem.  A chunk of pages is processed by
 * G SMs: G = 1 when rows_per_kv_head <= 64 (one CTA carries up to 64 query rows), otherwise
 * G = 2 * ceil(rows_per_kv_head / 128) (a pair of CTAs on the two SMs of a TPC carries 128
 * rows), so num_sm_parts = max(1, SM count of `device` / (h_kv * G)).  For example, on 148
 * SMs: 148 parts for 16 rows, 74 for 128, 37 for 192 or 256.
 *   rows_per_kv_head  s_q * h_q / h_kv
 * Returns the count (>= 1) or a negative MLA_ERR_* code.
 */
MLA_API int mla_num_sm_parts(int rows_per_kv_head, int h_kv, int device);

/*
 * Tile-scheduler metadata (get_mla_metadata): splits every request's 128-token blocks into
 * chunks and spreads them over num_sm_parts parts so that each part carries about the same
 * cost (blocks + a fixed cost of 2 blocks per chunk).  Run once per decode step; the result
 * is reused by every layer.
 *   cache_seqlens  device int32 [batch]
 *   tile_md        device int32 [num_sm_parts, 8] (written): per part
 *                  {begin_b, begin_block, end_b, end_block, first_split, 0, 0, 0}
 *   num_splits     device int32 [batch + 1] (written): prefix count of chunks per request
 * The total cost (sum over requests with tokens of ceil(L_b / 128) + 2) must stay below 2^31.
 * The lengths are device data, so this is checked on the device: a batch above it gets every
 * part empty with tile_md[p][5] = 1 and num_splits all 0, and a decode call given that
 * metadata raises MLA_STATUS_BAD_METADATA in its workspace status word.
 * Errors: MLA_ERR_NULL_POINTER, MLA_ERR_BAD_SHAPE (batch < 1), MLA_ERR_BAD_HEADS,
 *         MLA_ERR_BAD_PARTS, MLA_ERR_CUDA.
 */
MLA_API int mla_get_metadata(const int32_t* cache_seqlens, int batch, int rows_per_kv_head, int h_kv, int32_t* tile_md,
                     int num_sm_parts, int32_t* num_splits, void* stream);

/*
 * Bytes of device workspace mla_decode_kvcache needs: a 256-byte status header, then fp32
 * partial LSE [batch + num_sm_parts, rows] and partial O [batch + num_sm_parts, rows, 512]
 * for requests split over several parts.  Returns 0 for invalid arguments.
 */
MLA_API size_t mla_workspace_size(int batch, int num_sm_parts, int rows_per_kv_head, int h_kv);

/*
 * MLA decode (flash_mla_with_kvcache / mha_fwd_kvcache_mla): split-KV main kernel then the
 * LSE combine, both enqueued on `stream`.
 *   q              device bf16 [batch, s_q, h_q, 576], contiguous, 16-byte aligned
 *   kvcache        device, see kv_dtype; contiguous, 16-byte aligned
 *   num_blocks     physical pages in kvcache
 *   block_table    device int32 [batch, max_blocks], row-major
 *   cache_seqlens  device int32 [batch]
 *   h_kv           must be 1;  d_v must be 512
 *   tile_md, num_splits   from mla_get_metadata with the same cache_seqlens and num_sm_parts
 *   softmax_scale  multiplies q.k (e.g. 576^-0.5)
 *   causal         0 / 1
 *   kv_dtype       MLA_KV_BF16 or MLA_KV_FP8.  With MLA_KV_FP8 and more than 64 query rows per
 *                  request the products run on f16 tensor cores: q, the RoPE dims and every
 *                  code * scale must stay within the f16 range (|x| < 65504; scales up to
 *                  65504 / 448 = 146.2); a call that meets a value outside it raises
 *                  MLA_STATUS_F16_RANGE.  e4m3 NaN codes are not expected (a quantised cache
 *                  holds none)
 *   out            device bf16 [batch, s_q, h_q, 512] (written)
 *   lse            device fp32 [batch, h_q, s_q] (written)
 *   workspace      device scratch of >= mla_workspace_size(batch, num_sm_parts, s_q*h_q, h_kv) bytes,
 *                  16-byte aligned; its first word is the device status (MLA_STATUS_*)
 */
MLA_API int mla_decode_kvcache(const void* q, const void* kvcache, int64_t num_blocks, const int32_t* block_table,
                       int max_blocks, const int32_t* cache_seqlens, int batch, int s_q, int h_q, int h_kv,
                       int d_v, const int32_t* tile_md, int num_sm_parts, const int32_t* num_splits,
                       float softmax_scale, int causal, int kv_dtype, void* out, float* lse, void* workspace,
                       size_t workspace_bytes, void* stream);

/*
 * mla_decode_kvcache without a workspace argument, for callers that cannot allocate device
 * memory when they run decode: engines that reserve all device memory at start-up and forbid
 * later allocations, code running inside an allocator hook or driver callback where an
 * allocation would re-enter the allocator, or plain C programs that link no allocator.
 * (The FlashMLA pages have no counterpart of this call.)
 *
 * The workspace is a 16 MiB array inside this library, held by every GPU that loads it until
 * the process exits.  Problems with mla_workspace_size(...) > 16 MiB return
 * MLA_ERR_SCRATCH_LIMIT (e.g. batch 128 x 16 query rows fits, batch 128 x 128 rows does not).
 * The first call on a device (with that device current) looks the array's address up once;
 * make that first call before any stream capture.  All calls share the array and it keeps the
 * last call's contents: the status word is cleared at the start of each call (an async memset
 * on `stream`, no allocation), partial results are written before they are read.  Calls that
 * overlap on the GPU (other streams or host threads) race on the array.  No cudaMalloc,
 * cudaFree or allocating routine is called.  Other arguments and errors as mla_decode_kvcache.
 */
MLA_API int mla_decode_kvcache_noalloc(const void* q, const void* kvcache, int64_t num_blocks,
                                       const int32_t* block_table, int max_blocks, const int32_t* cache_seqlens,
                                       int batch, int s_q, int h_q, int h_kv, int d_v, const int32_t* tile_md,
                                       int num_sm_parts, const int32_t* num_splits, float softmax_scale, int causal,
                                       int kv_dtype, void* out, float* lse, void* stream);

/*
 * Device status word (MLA_STATUS_* bits) of the last mla_decode_kvcache_noalloc call on the
 * current device, which lives in that call's built-in array (callers of the no-alloc call have
 * no workspace of their own to read it from).  Waits on `stream` (enqueue it on the stream of
 * the decode call), copies the word into *status and, when `reset` is nonzero, clears it.
 * Like the decode call it allocates nothing; it shares the array with it, so read the status
 * before the next no-alloc call on the device clears it.  Errors: MLA_ERR_NULL_POINTER,
 * MLA_ERR_NO_DEVICE, MLA_ERR_CUDA.  (The FlashMLA pages have no counterpart of this call.)
 */
MLA_API int mla_noalloc_read_status(int reset, int* status, void* stream);

/*
 * Token-sparse decode (the `topk` argument of get_mla_metadata and the `indices` argument of
 * flash_mla_with_kvcache on the gitcode FlashMLA page, "解码阶段使用示例" / "稀疏解码场景").
 * The page names the arguments but not their shape; this library's reading:
 *   indices        device int32 [batch, s_q, topk], 4-byte aligned: query position i of
 *                  request b attends to the tokens at the logical cache positions
 *                  indices[b, i, :] (through block_table, as in dense decode).  An entry
 *                  outside [0, cache_seqlens[b]) is an empty slot; a position listed twice
 *                  counts twice.  No causal mask applies.  A query with no valid entry gets
 *                  O = 0 and LSE = -inf.
 * Every query position is scheduled as a request of topk tokens:
 *   mla_get_metadata_sparse  tile_md [num_sm_parts, 8] and num_splits [batch * s_q + 1] for
 *                            batch * s_q positions of topk tokens; num_sm_parts from
 *                            mla_num_sm_parts(h_q, h_kv).  MLA_ERR_BAD_SHAPE when
 *                            batch * s_q * (ceil(topk / 128) + 2) >= 2^31 (the scheduler's
 *                            cost sums are 32-bit)
 *   mla_decode_kvcache_sparse  as mla_decode_kvcache (bf16 cache only: MLA_ERR_BAD_KV_DTYPE
 *                            otherwise), with the workspace of
 *                            mla_workspace_size(batch * s_q, num_sm_parts, h_q, h_kv) bytes
 */
MLA_API int mla_get_metadata_sparse(int batch, int s_q, int topk, int h_q, int h_kv, int32_t* tile_md,
                                    int num_sm_parts, int32_t* num_splits, void* stream);

MLA_API int mla_decode_kvcache_sparse(const void* q, const void* kvcache, int64_t num_blocks,
                                      const int32_t* block_table, int max_blocks, const int32_t* cache_seqlens,
                                      int batch, int s_q, int h_q, int h_kv, int d_v, const int32_t* indices,
                                      int topk, const int32_t* tile_md, int num_sm_parts,
                                      const int32_t* num_splits, float softmax_scale, int kv_dtype, void* out,
                                      float* lse, void* workspace, size_t workspace_bytes, void* stream);

/*
 * Sparse prefill (flash_mla_sparse_fwd(q, kv, indices, sm_scale, d_v = 512) on the gitcode
 * FlashMLA page, "稀疏预填充使用"): every query token attends to the listed tokens of one
 * contiguous cache, with the reading of the token-sparse decode above.
 *   q        device bf16 [s_q, h_q, 576];   kv  device bf16 [s_kv, 1, 576] (16-byte aligned)
 *   indices  device int32 [s_q, 1, topk]: positions in [0, s_kv), others are empty slots
 *   tile_md, num_splits   from mla_get_metadata_sparse(1, s_q, topk, h_q, h_kv, ...)
 *   out      device bf16 [s_q, h_q, 512];  lse  device fp32 [h_q, s_q] (natural log)
 *   workspace  >= mla_workspace_size(s_q, num_sm_parts, h_q, h_kv) bytes
 */
MLA_API int mla_sparse_prefill(const void* q, const void* kv, int s_kv, const int32_t* indices, int s_q, int h_q,
                               int h_kv, int d_v, int topk, const int32_t* tile_md, int num_sm_parts,
                               const int32_t* num_splits, float softmax_scale, void* out, float* lse,
                               void* workspace, size_t workspace_bytes, void* stream);

/*
 * Serving session: decode steps whose inputs and outputs are HOST buffers (pinned memory lets
 * the copies run asynchronously), pipelined two steps deep.  The one part of the library that
 * allocates device memory and creates streams and events, all at mla_session_create: two sets
 * of staging buffers (q, block_table, cache_seqlens, indices, out, lse), the tile metadata,
 * the workspace, a copy-in and a copy-out stream.  The KV cache stays a device buffer of the
 * caller.
 *
 * mla_session_create  device, batch, s_q, h_q, h_kv (= 1), max_blocks (block-table width),
 *                     topk (0: dense decode; > 0: token-sparse decode, bf16 cache only, with
 *                     indices [batch, s_q, topk] per step), kv_dtype, num_sm_parts (from
 *                     mla_num_sm_parts(topk ? h_q : s_q * h_q, h_kv)).  *session receives the
 *                     handle.  Argument errors as mla_decode_kvcache; MLA_ERR_CUDA if an
 *                     allocation fails (nothing is left allocated).
 * mla_session_decode  one step with host buffers: q [batch, s_q, h_q, 576] bf16,
 *                     block_table [batch, max_blocks] and cache_seqlens [batch] int32, indices
 *                     [batch, s_q, topk] int32 (token-sparse sessions; NULL otherwise),
 *                     out [batch, s_q, h_q, 512] bf16 and lse [batch, h_q, s_q] fp32; kvcache
 *                     as in mla_decode_kvcache.  Enqueues the copy of the inputs into staging set
 *                     k % 2 (copy-in stream, after step k - 2 has read that set), the scheduler,
 *                     decode and combine on `stream` (after that copy, and after step k - 2's
 *                     results have been copied out), and the copy of out and lse into the host
 *                     buffers (copy-out stream).  So step k + 1's copy-in and step k - 1's
 *                     copy-out run while step k computes.  Returns at once; the host inputs
 *                     must stay unchanged until the step's copy-in has run.
 * mla_session_join    makes `stream` wait for the copy-out of every step enqueued so far (no
 *                     host wait: synchronise `stream` to read the host outputs); the next step's
 *                     copy-in is then ordered after the work enqueued on `stream` before it.
 *                     The first step after mla_session_create is ordered the same way.
 * mla_session_status  reads the session workspace's status word (MLA_STATUS_*) into *status
 *                     after waiting for the session's work; reset != 0 clears it.
 * mla_session_destroy waits for the session's work and frees everything it allocated.
 */
typedef struct mla_session mla_session;

MLA_API int mla_session_create(int device, int batch, int s_q, int h_q, int h_kv, int max_blocks, int topk,
                               int kv_dtype, int num_sm_parts, mla_session** session);

MLA_API int mla_session_decode(mla_session* session, const void* q_host, const void* kvcache, int64_t num_blocks,
                               const int32_t* block_table_host, const int32_t* cache_seqlens_host,
                               const int32_t* indices_host, float softmax_scale, int causal, void* out_host,
                               float* lse_host, void* stream);

MLA_API int mla_session_join(mla_session* session, void* stream);

MLA_API int mla_session_status(mla_session* session, int reset, int* status);

MLA_API int mla_session_destroy(mla_session* session);

/*
 * Fault injection for tests of the kernels' bounded waits (the pages have no counterpart; it
 * exists so that the time-out path can be exercised without faulting or hanging a GPU).  Arms
 * the next mla_decode_kvcache call made in this process, which then uses
 *   wait_limit_cycles  as the bound of every pipeline wait, in SM clock cycles (0: the default
 *                      bound of about one second), and
 *   withhold_fill      the index of a shared-memory slot fill (counted from 0 over the call's
 *                      CTA) that the copy producer skips (-1: none).  The slot's consumer then
 *                      waits in vain until the bound runs out, sets MLA_STATUS_WAIT_TIMEOUT,
 *                      and every role of the CTA unwinds (copies in flight are drained, tensor
 *                      memory is freed); the call's outputs are undefined.
 * Honoured by the single-CTA kernel, which runs bf16 caches with up to 64 query rows per
 * request (fill index counted over the CTA).  The next call takes and clears the setting
 * whichever kernel it runs.  Errors: MLA_ERR_BAD_SHAPE for a
 * negative limit or a fill index below -1.
 */
MLA_API int mla_fault_injection_arm(long long wait_limit_cycles, int withhold_fill);

/*
 * Reads the device status word of a workspace into *status (host pointer).  This call
 * synchronises `stream`.  reset != 0 clears the word afterwards (enqueued on `stream`).
 */
MLA_API int mla_read_status(void* workspace, int reset, int* status, void* stream);

/* Static description of an MLA_* code. Never NULL. */
MLA_API const char* mla_strerror(int code);

/* Library version, e.g. "0.1.0". */
MLA_API const char* mla_version(void);

#ifdef __cplusplus
}
#endif

#endif /* MLA_H_ */

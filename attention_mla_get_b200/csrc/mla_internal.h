// Internal declarations shared by the C-ABI layer (mla_api.cu) and the kernels.
// Nothing here is part of the public interface in include/mla.h.
#pragma once
#include <cstddef>
#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

namespace mla {

constexpr int kDqk = 576;          // 512 latent (NoPE) + 64 RoPE dims per cached token
constexpr int kDv = 512;           // V = first 512 dims of the cached vector
constexpr int kPage = 64;          // tokens per KV page
constexpr int kBlockTokens = 128;  // scheduling unit: two pages, one main-loop step
constexpr int kFixedSplitCost = 2; // scheduler: cost of opening a chunk, in blocks
constexpr int kMdInts = 8;         // ints per tile-scheduler metadata row
constexpr int kRowsPerCta = 64;    // query rows one CTA carries at most
constexpr int kFp8TokenBytes = 656;

// device status bits (sticky, in the first word of the workspace)
constexpr int kStatusWaitTimeout = 1;
constexpr int kStatusBadMetadata = 2;  // the tile scheduler flagged its metadata (see kMdOverflow)
constexpr int kStatusF16Range = 4;     // FP8 CTA pair: an operand left the f16 range
// tile_md[part][5]: nonzero when the scheduler could not build the metadata (the total cost of
// the batch does not fit its 32-bit prefix sums); every part is then empty
constexpr int kMdOverflow = 1;

struct DecodeParams {
  const int32_t* block_table;
  const int32_t* cache_seqlens;
  const int32_t* tile_md;
  const int32_t* num_splits;
  __nv_bfloat16* out;     // [b, s_q, h_q, 512]
  float* lse;             // [b, h_q, s_q]
  float* o_part;          // [max_splits, R, 512]
  float* lse_part;        // [max_splits, R]
  int* status;
  int max_blocks;
  int batch;
  int num_sm_parts;
  int s_q;
  int h_q;
  int rows;               // R = s_q * h_q / h_kv
  int row_groups;         // G = ceil(R / rows per CTA, or per CTA pair)
  int causal;
  float scale_log2;       // softmax_scale * log2(e)
  // token-sparse decode (topk > 0): the scheduler's "requests" are the batch * s_q query
  // positions (vq = s_q of them per request), each over topk listed cache positions
  const void* kv;         // the bf16 cache (read with per-token copies)
  const int32_t* indices; // [batch * s_q, topk] logical cache positions; others: empty slots
  int topk;
  int vq;
  int kv_len;             // sparse prefill: tokens of the one contiguous cache (cache_seqlens null)
  // fault injection for tests of the bounded waits (mla_fault_injection_arm; bf16 kernels up to
  // 64 rows): a shorter wait bound, and 1 + the index of a slot fill the producer skips
  long long wait_limit;   // 0: the default bound
  int withhold_fill1;     // 0: none
};

struct CombineParams {
  const int32_t* num_splits;
  const float* o_part;
  const float* lse_part;
  __nv_bfloat16* out;
  float* lse;
  int batch;
  int s_q;
  int h_q;
  int rows;
  int vq;  // token-sparse: query positions per request (batch counts positions), else 0
};

inline int row_groups_for(int rows) { return rows <= kRowsPerCta ? 1 : (rows + kRowsPerCta - 1) / kRowsPerCta; }

// Requests with more than 64 query rows run on CTA pairs of 128 rows each (mla_decode_pair.cu,
// bf16 or FP8 cache); a scheduler part then needs 2 SMs per 128-row group.
constexpr int kPairRows = 128;
inline bool use_pair_kernel(int rows, bool /*fp8*/) { return rows > kRowsPerCta; }
inline int sms_per_part(int rows) { return rows <= kRowsPerCta ? 1 : 2 * ((rows + kPairRows - 1) / kPairRows); }

// Output tensor maps of the decode kernels' epilogues (TMA stores of 128 dims x 32 rows, or 16
// rows for the 16-row kernel): o_part fp32 {512, rows, splits}, out bf16 {512, rows, batch}
struct OutMaps {
  CUtensorMap o_part;
  CUtensorMap out;
};

// launchers (return cudaError_t as int)
// cache_seqlens == nullptr: every one of the `batch` requests has uniform_len tokens
int launch_scheduler(const int32_t* cache_seqlens, int batch, int num_sm_parts, int32_t* tile_md,
                     int32_t* num_splits, cudaStream_t stream, int uniform_len = 0);
int launch_decode_bf16(const CUtensorMap& tm_q, const CUtensorMap& tm_kv, const OutMaps& om, const DecodeParams& p,
                       int rows_per_cta, cudaStream_t stream);
int launch_decode_fp8(const CUtensorMap& tm_q, const CUtensorMap& tm_codes, const CUtensorMap& tm_scale,
                      const CUtensorMap& tm_rope, const OutMaps& om, const DecodeParams& p, int rows_per_cta,
                      cudaStream_t stream);
int launch_decode_sparse_bf16(const CUtensorMap& tm_q, const OutMaps& om, const DecodeParams& p, int rows_per_cta,
                              cudaStream_t stream);
int launch_decode_pair_bf16(const CUtensorMap& tm_q, const CUtensorMap& tm_kv, const OutMaps& om,
                            const DecodeParams& p, cudaStream_t stream);
int launch_decode_pair_fp8(const CUtensorMap& tm_q, const CUtensorMap& tm_codes, const CUtensorMap& tm_scale,
                           const CUtensorMap& tm_rope, const OutMaps& om, const DecodeParams& p,
                           cudaStream_t stream);
int launch_decode_pair_sparse_bf16(const CUtensorMap& tm_q, const OutMaps& om, const DecodeParams& p,
                                   cudaStream_t stream);
int launch_combine(const CombineParams& p, cudaStream_t stream);

}  // namespace mla

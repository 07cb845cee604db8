// C-ABI of libmla (declared in include/mla.h): host-side argument checks, workspace
// partitioning, TMA descriptor encoding and the kernel launches.  No compute happens here.
#include <atomic>
#include <cstdio>
#include <cstring>

#include "mla.h"
#include "mla_internal.h"

namespace {

using mla::kDqk;
using mla::kDv;
using mla::kPage;

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(ptr);
  }
  return fn;
}

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

constexpr size_t kHeaderBytes = 256;
constexpr int kMaxRows = 4096;

struct WorkspaceLayout {
  size_t lse_off, o_off, total;
};

// The decode kernels' output maps (boxes of 128 dims x box_rows rows, no swizzle): o_part fp32
// {512, rows, batch + parts} in the workspace, out bf16 {512, rows, batch}.
static bool encode_out_maps(EncodeTiledFn encode, mla::OutMaps* om, float* o_part, void* out, int rows, int batch,
                            int parts, int box_rows) {
  const cuuint32_t box[3] = {128, static_cast<cuuint32_t>(box_rows), 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  {
    const cuuint64_t dims[3] = {static_cast<cuuint64_t>(kDv), static_cast<cuuint64_t>(rows),
                                static_cast<cuuint64_t>(batch) + static_cast<cuuint64_t>(parts)};
    const cuuint64_t strides[2] = {static_cast<cuuint64_t>(kDv) * 4, static_cast<cuuint64_t>(kDv) * 4 * rows};
    if (encode(&om->o_part, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, o_part, dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_NONE,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return false;
  }
  const cuuint64_t dims[3] = {static_cast<cuuint64_t>(kDv), static_cast<cuuint64_t>(rows),
                              static_cast<cuuint64_t>(batch)};
  const cuuint64_t strides[2] = {static_cast<cuuint64_t>(kDv) * 2, static_cast<cuuint64_t>(kDv) * 2 * rows};
  return encode(&om->out, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, out, dims, strides, box, estr,
                CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_NONE,
                CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

WorkspaceLayout workspace_layout(int batch, int parts, int rows) {
  const size_t splits = static_cast<size_t>(batch) + static_cast<size_t>(parts);
  WorkspaceLayout w;
  w.lse_off = kHeaderBytes;
  w.o_off = round_up(w.lse_off + splits * rows * sizeof(float), 256);
  w.total = w.o_off + splits * rows * kDv * sizeof(float);
  return w;
}

int rows_per_cta_for(int rows) { return rows <= 16 ? 16 : (rows <= 32 ? 32 : 64); }

// armed by mla_fault_injection_arm, taken (and cleared) by the next mla_decode_kvcache call
std::atomic<long long> g_fault_wait_limit{0};
std::atomic<int> g_fault_withhold1{0};

}  // namespace

extern "C" {

const char* mla_version(void) { return "0.1.0"; }

const char* mla_strerror(int code) {
  switch (code) {
    case MLA_OK: return "success";
    case MLA_ERR_NULL_POINTER: return "a required pointer is NULL";
    case MLA_ERR_MISALIGNED: return "q, kvcache, out and workspace must be 16-byte aligned, lse 4-byte aligned";
    case MLA_ERR_BAD_DIM: return "d_v must be 512 (V is the first 512 of the 576 cached dims)";
    case MLA_ERR_BAD_HEADS: return "h_kv must be 1, h_q >= 1 and h_q % h_kv == 0";
    case MLA_ERR_BAD_KV_DTYPE: return "kv_dtype must be MLA_KV_BF16 or MLA_KV_FP8";
    case MLA_ERR_WORKSPACE: return "workspace is smaller than mla_workspace_size()";
    case MLA_ERR_BAD_SHAPE: return "bad shape: batch, s_q, num_blocks, max_blocks must be >= 1, "
                                   "s_q*h_q <= 4096 and num_blocks*64 < 2^31";
    case MLA_ERR_BAD_PARTS: return "num_sm_parts must be >= 1";
    case MLA_ERR_NO_DEVICE: return "CUDA device query failed";
    case MLA_ERR_SCRATCH_LIMIT:
      return "the problem's workspace exceeds the 16 MiB built-in scratch of the no-alloc call";
    case MLA_ERR_CUDA: return "a CUDA call failed";
    default: return "unknown libmla error code";
  }
}

int mla_num_sm_parts(int rows_per_kv_head, int h_kv, int device) {
  if (h_kv != 1) return MLA_ERR_BAD_HEADS;
  if (rows_per_kv_head < 1 || rows_per_kv_head > kMaxRows) return MLA_ERR_BAD_SHAPE;
  int sms = 0;
  if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, device) != cudaSuccess || sms < 1)
    return MLA_ERR_NO_DEVICE;
  const int g = mla::sms_per_part(rows_per_kv_head);
  const int parts = sms / (h_kv * g);
  return parts < 1 ? 1 : parts;
}

size_t mla_workspace_size(int batch, int num_sm_parts, int rows_per_kv_head, int h_kv) {
  if (batch < 1 || num_sm_parts < 1 || h_kv != 1 || rows_per_kv_head < 1 || rows_per_kv_head > kMaxRows) return 0;
  return workspace_layout(batch, num_sm_parts, rows_per_kv_head).total;
}

int mla_get_metadata(const int32_t* cache_seqlens, int batch, int rows_per_kv_head, int h_kv, int32_t* tile_md,
                     int num_sm_parts, int32_t* num_splits, void* stream) {
  if (!cache_seqlens || !tile_md || !num_splits) return MLA_ERR_NULL_POINTER;
  if (batch < 1 || rows_per_kv_head < 1 || rows_per_kv_head > kMaxRows) return MLA_ERR_BAD_SHAPE;
  if (h_kv != 1) return MLA_ERR_BAD_HEADS;
  if (num_sm_parts < 1) return MLA_ERR_BAD_PARTS;
  const int e = mla::launch_scheduler(cache_seqlens, batch, num_sm_parts, tile_md, num_splits,
                                      static_cast<cudaStream_t>(stream));
  return e == 0 ? MLA_OK : MLA_ERR_CUDA;
}

int mla_decode_kvcache(const void* q, const void* kvcache, int64_t num_blocks, const int32_t* block_table,
                       int max_blocks, const int32_t* cache_seqlens, int batch, int s_q, int h_q, int h_kv,
                       int d_v, const int32_t* tile_md, int num_sm_parts, const int32_t* num_splits,
                       float softmax_scale, int causal, int kv_dtype, void* out, float* lse, void* workspace,
                       size_t workspace_bytes, void* stream) {
  // ---- argument checks (nothing is enqueued before they all pass) ----
  if (!q || !kvcache || !block_table || !cache_seqlens || !tile_md || !num_splits || !out || !lse || !workspace)
    return MLA_ERR_NULL_POINTER;
  if (!aligned(q, 16) || !aligned(kvcache, 16) || !aligned(out, 16) || !aligned(workspace, 16) || !aligned(lse, 4))
    return MLA_ERR_MISALIGNED;
  if (d_v != kDv) return MLA_ERR_BAD_DIM;
  if (h_kv != 1 || h_q < 1 || h_q % h_kv != 0) return MLA_ERR_BAD_HEADS;
  if (kv_dtype != MLA_KV_BF16 && kv_dtype != MLA_KV_FP8) return MLA_ERR_BAD_KV_DTYPE;
  if (batch < 1 || s_q < 1 || num_blocks < 1 || max_blocks < 1) return MLA_ERR_BAD_SHAPE;
  const long long rows_ll = static_cast<long long>(s_q) * h_q / h_kv;
  if (rows_ll > kMaxRows) return MLA_ERR_BAD_SHAPE;
  if (num_blocks * kPage >= (1ll << 31)) return MLA_ERR_BAD_SHAPE;
  if (num_sm_parts < 1) return MLA_ERR_BAD_PARTS;
  const int rows = static_cast<int>(rows_ll);
  const WorkspaceLayout wl = workspace_layout(batch, num_sm_parts, rows);
  if (workspace_bytes < wl.total) return MLA_ERR_WORKSPACE;

  EncodeTiledFn encode = encode_fn();
  if (!encode) return MLA_ERR_CUDA;
  const bool pair = mla::use_pair_kernel(rows, kv_dtype == MLA_KV_FP8);
  const int rg = pair ? mla::kRowsPerCta : rows_per_cta_for(rows);  // query rows of one Q box

  // q as a 3-D tensor {576 dims, rows, batch}; one box = 64 dims x rg rows of one request
  CUtensorMap tm_q, tm_kv, tm_scale, tm_rope;
  {
    cuuint64_t dims[3] = {static_cast<cuuint64_t>(kDqk), static_cast<cuuint64_t>(rows),
                          static_cast<cuuint64_t>(batch)};
    cuuint64_t strides[2] = {static_cast<cuuint64_t>(kDqk) * 2, static_cast<cuuint64_t>(kDqk) * 2 * rows};
    cuuint32_t box[3] = {64, static_cast<cuuint32_t>(rg), 1};
    cuuint32_t estr[3] = {1, 1, 1};
    if (encode(&tm_q, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(q), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return MLA_ERR_CUDA;
  }
  if (kv_dtype == MLA_KV_BF16) {
    // the cache as 2-D {576 dims, num_blocks * 64 tokens}; one box = 64 dims x one page
    cuuint64_t dims[2] = {static_cast<cuuint64_t>(kDqk), static_cast<cuuint64_t>(num_blocks) * kPage};
    cuuint64_t strides[1] = {static_cast<cuuint64_t>(kDqk) * 2};
    cuuint32_t box[2] = {64, 64};
    cuuint32_t estr[2] = {1, 1};
    if (encode(&tm_kv, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(kvcache), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return MLA_ERR_CUDA;
  } else {
    // FP8 tokens as a 2-D byte tensor {656 bytes, num_blocks * 64 tokens}, read three ways:
    // 128-byte columns of e4m3 codes, the 16 scale bytes at byte 512, and the 128 RoPE bytes
    // at byte 528 with the 128-byte swizzle the MMA operand layout uses.
    cuuint64_t dims[2] = {static_cast<cuuint64_t>(mla::kFp8TokenBytes), static_cast<cuuint64_t>(num_blocks) * kPage};
    cuuint64_t strides[1] = {static_cast<cuuint64_t>(mla::kFp8TokenBytes)};
    cuuint32_t estr[2] = {1, 1};
    cuuint32_t box_codes[2] = {128, 64}, box_scale[2] = {16, 64};
    if (encode(&tm_kv, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(kvcache), dims, strides, box_codes, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS ||
        encode(&tm_scale, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(kvcache), dims, strides, box_scale,
               estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS ||
        encode(&tm_rope, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(kvcache), dims, strides, box_codes,
               estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return MLA_ERR_CUDA;
  }

  uint8_t* ws = static_cast<uint8_t*>(workspace);
  mla::DecodeParams p{};
  p.block_table = block_table;
  p.cache_seqlens = cache_seqlens;
  p.tile_md = tile_md;
  p.num_splits = num_splits;
  p.out = static_cast<__nv_bfloat16*>(out);
  p.lse = lse;
  p.lse_part = reinterpret_cast<float*>(ws + wl.lse_off);
  p.o_part = reinterpret_cast<float*>(ws + wl.o_off);
  p.status = reinterpret_cast<int*>(ws);
  p.max_blocks = max_blocks;
  p.batch = batch;
  p.num_sm_parts = num_sm_parts;
  p.s_q = s_q;
  p.h_q = h_q;
  p.rows = rows;
  p.row_groups = pair ? (rows + mla::kPairRows - 1) / mla::kPairRows : (rows + rg - 1) / rg;
  p.causal = causal ? 1 : 0;
  p.scale_log2 = softmax_scale * 1.4426950408889634f;
  p.wait_limit = g_fault_wait_limit.exchange(0);
  p.withhold_fill1 = g_fault_withhold1.exchange(0);

  mla::OutMaps om;
  if (!encode_out_maps(encode, &om, p.o_part, out, rows, batch, num_sm_parts, rg == 16 ? 16 : 32))
    return MLA_ERR_CUDA;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  int e = kv_dtype == MLA_KV_BF16 ? (pair ? mla::launch_decode_pair_bf16(tm_q, tm_kv, om, p, st)
                                          : mla::launch_decode_bf16(tm_q, tm_kv, om, p, rg, st))
          : pair ? mla::launch_decode_pair_fp8(tm_q, tm_kv, tm_scale, tm_rope, om, p, st)
                 : mla::launch_decode_fp8(tm_q, tm_kv, tm_scale, tm_rope, om, p, rg, st);
  if (e != 0) return MLA_ERR_CUDA;

  mla::CombineParams cp{};
  cp.num_splits = num_splits;
  cp.o_part = p.o_part;
  cp.lse_part = p.lse_part;
  cp.out = p.out;
  cp.lse = lse;
  cp.batch = batch;
  cp.s_q = s_q;
  cp.h_q = h_q;
  cp.rows = rows;
  e = mla::launch_combine(cp, st);
  return e == 0 ? MLA_OK : MLA_ERR_CUDA;
}

int mla_get_metadata_sparse(int batch, int s_q, int topk, int h_q, int h_kv, int32_t* tile_md, int num_sm_parts,
                            int32_t* num_splits, void* stream) {
  if (!tile_md || !num_splits) return MLA_ERR_NULL_POINTER;
  if (batch < 1 || s_q < 1 || topk < 1 || h_q < 1 || h_q > kMaxRows) return MLA_ERR_BAD_SHAPE;
  if (static_cast<long long>(batch) * s_q >= (1ll << 30)) return MLA_ERR_BAD_SHAPE;
  // the scheduler's 32-bit prefix sums: total cost = positions * (blocks of topk + 2) < 2^31
  const long long blocks = (static_cast<long long>(topk) + mla::kBlockTokens - 1) / mla::kBlockTokens;
  const long long cost = static_cast<long long>(batch) * s_q * (blocks + mla::kFixedSplitCost);
  if (cost >= (1ll << 31)) return MLA_ERR_BAD_SHAPE;
  if (h_kv != 1) return MLA_ERR_BAD_HEADS;
  if (num_sm_parts < 1) return MLA_ERR_BAD_PARTS;
  const int e = mla::launch_scheduler(nullptr, batch * s_q, num_sm_parts, tile_md, num_splits,
                                      static_cast<cudaStream_t>(stream), topk);
  return e == 0 ? MLA_OK : MLA_ERR_CUDA;
}

int mla_decode_kvcache_sparse(const void* q, const void* kvcache, int64_t num_blocks, const int32_t* block_table,
                              int max_blocks, const int32_t* cache_seqlens, int batch, int s_q, int h_q, int h_kv,
                              int d_v, const int32_t* indices, int topk, const int32_t* tile_md, int num_sm_parts,
                              const int32_t* num_splits, float softmax_scale, int kv_dtype, void* out, float* lse,
                              void* workspace, size_t workspace_bytes, void* stream) {
  // ---- argument checks (nothing is enqueued before they all pass) ----
  if (!q || !kvcache || !block_table || !cache_seqlens || !indices || !tile_md || !num_splits || !out || !lse ||
      !workspace)
    return MLA_ERR_NULL_POINTER;
  if (!aligned(q, 16) || !aligned(kvcache, 16) || !aligned(out, 16) || !aligned(workspace, 16) || !aligned(lse, 4) ||
      !aligned(indices, 4))
    return MLA_ERR_MISALIGNED;
  if (d_v != kDv) return MLA_ERR_BAD_DIM;
  if (h_kv != 1 || h_q < 1) return MLA_ERR_BAD_HEADS;
  if (kv_dtype != MLA_KV_BF16) return MLA_ERR_BAD_KV_DTYPE;
  if (batch < 1 || s_q < 1 || topk < 1 || num_blocks < 1 || max_blocks < 1) return MLA_ERR_BAD_SHAPE;
  if (h_q > kMaxRows || static_cast<long long>(batch) * s_q >= (1ll << 30)) return MLA_ERR_BAD_SHAPE;
  if (static_cast<long long>(batch) * s_q * topk >= (1ll << 31)) return MLA_ERR_BAD_SHAPE;
  if (num_blocks * kPage >= (1ll << 31)) return MLA_ERR_BAD_SHAPE;
  if (num_sm_parts < 1) return MLA_ERR_BAD_PARTS;
  const int positions = batch * s_q;
  const WorkspaceLayout wl = workspace_layout(positions, num_sm_parts, h_q);
  if (workspace_bytes < wl.total) return MLA_ERR_WORKSPACE;

  EncodeTiledFn encode = encode_fn();
  if (!encode) return MLA_ERR_CUDA;
  const bool pair = mla::use_pair_kernel(h_q, false);  // more than 64 heads: CTA pairs of 128
  const int rg = pair ? mla::kRowsPerCta : rows_per_cta_for(h_q);
  // q as {576 dims, h_q heads, batch * s_q positions}; one box = 64 dims x rg heads of a position
  CUtensorMap tm_q;
  {
    cuuint64_t dims[3] = {static_cast<cuuint64_t>(kDqk), static_cast<cuuint64_t>(h_q),
                          static_cast<cuuint64_t>(positions)};
    cuuint64_t strides[2] = {static_cast<cuuint64_t>(kDqk) * 2, static_cast<cuuint64_t>(kDqk) * 2 * h_q};
    cuuint32_t box[3] = {64, static_cast<cuuint32_t>(rg), 1};
    cuuint32_t estr[3] = {1, 1, 1};
    if (encode(&tm_q, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(q), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return MLA_ERR_CUDA;
  }
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  mla::DecodeParams p{};
  p.block_table = block_table;
  p.cache_seqlens = cache_seqlens;
  p.tile_md = tile_md;
  p.num_splits = num_splits;
  p.out = static_cast<__nv_bfloat16*>(out);
  p.lse = lse;
  p.lse_part = reinterpret_cast<float*>(ws + wl.lse_off);
  p.o_part = reinterpret_cast<float*>(ws + wl.o_off);
  p.status = reinterpret_cast<int*>(ws);
  p.max_blocks = max_blocks;
  p.batch = positions;  // the scheduler's requests are the query positions
  p.num_sm_parts = num_sm_parts;
  p.s_q = s_q;
  p.h_q = h_q;
  p.rows = h_q;
  p.row_groups = pair ? (h_q + mla::kPairRows - 1) / mla::kPairRows : (h_q + rg - 1) / rg;
  p.causal = 0;
  p.scale_log2 = softmax_scale * 1.4426950408889634f;
  p.kv = kvcache;
  p.indices = indices;
  p.topk = topk;
  p.vq = s_q;
  mla::OutMaps om;
  if (!encode_out_maps(encode, &om, p.o_part, out, h_q, p.batch, num_sm_parts, rg == 16 ? 16 : 32))
    return MLA_ERR_CUDA;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  int e = pair ? mla::launch_decode_pair_sparse_bf16(tm_q, om, p, st)
               : mla::launch_decode_sparse_bf16(tm_q, om, p, rg, st);
  if (e != 0) return MLA_ERR_CUDA;
  mla::CombineParams cp{};
  cp.num_splits = num_splits;
  cp.o_part = p.o_part;
  cp.lse_part = p.lse_part;
  cp.out = p.out;
  cp.lse = lse;
  cp.batch = positions;
  cp.s_q = s_q;
  cp.h_q = h_q;
  cp.rows = h_q;
  cp.vq = s_q;
  e = mla::launch_combine(cp, st);
  return e == 0 ? MLA_OK : MLA_ERR_CUDA;
}

int mla_sparse_prefill(const void* q, const void* kv, int s_kv, const int32_t* indices, int s_q, int h_q, int h_kv,
                       int d_v, int topk, const int32_t* tile_md, int num_sm_parts, const int32_t* num_splits,
                       float softmax_scale, void* out, float* lse, void* workspace, size_t workspace_bytes,
                       void* stream) {
  if (!q || !kv || !indices || !tile_md || !num_splits || !out || !lse || !workspace) return MLA_ERR_NULL_POINTER;
  if (!aligned(q, 16) || !aligned(kv, 16) || !aligned(out, 16) || !aligned(workspace, 16) || !aligned(lse, 4) ||
      !aligned(indices, 4))
    return MLA_ERR_MISALIGNED;
  if (d_v != kDv) return MLA_ERR_BAD_DIM;
  if (h_kv != 1 || h_q < 1) return MLA_ERR_BAD_HEADS;
  if (s_kv < 1 || s_q < 1 || topk < 1 || h_q > kMaxRows || s_q >= (1 << 30)) return MLA_ERR_BAD_SHAPE;
  if (static_cast<long long>(s_q) * topk >= (1ll << 31)) return MLA_ERR_BAD_SHAPE;
  if (num_sm_parts < 1) return MLA_ERR_BAD_PARTS;
  const WorkspaceLayout wl = workspace_layout(s_q, num_sm_parts, h_q);
  if (workspace_bytes < wl.total) return MLA_ERR_WORKSPACE;
  EncodeTiledFn encode = encode_fn();
  if (!encode) return MLA_ERR_CUDA;
  const bool pair = mla::use_pair_kernel(h_q, false);  // more than 64 heads: CTA pairs of 128
  const int rg = pair ? mla::kRowsPerCta : rows_per_cta_for(h_q);
  CUtensorMap tm_q;  // {576 dims, h_q heads, s_q query tokens}
  {
    cuuint64_t dims[3] = {static_cast<cuuint64_t>(kDqk), static_cast<cuuint64_t>(h_q), static_cast<cuuint64_t>(s_q)};
    cuuint64_t strides[2] = {static_cast<cuuint64_t>(kDqk) * 2, static_cast<cuuint64_t>(kDqk) * 2 * h_q};
    cuuint32_t box[3] = {64, static_cast<cuuint32_t>(rg), 1};
    cuuint32_t estr[3] = {1, 1, 1};
    if (encode(&tm_q, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(q), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return MLA_ERR_CUDA;
  }
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  mla::DecodeParams p{};
  p.block_table = nullptr;  // the cache is contiguous: logical position = row
  p.cache_seqlens = nullptr;
  p.kv_len = s_kv;
  p.tile_md = tile_md;
  p.num_splits = num_splits;
  p.out = static_cast<__nv_bfloat16*>(out);
  p.lse = lse;
  p.lse_part = reinterpret_cast<float*>(ws + wl.lse_off);
  p.o_part = reinterpret_cast<float*>(ws + wl.o_off);
  p.status = reinterpret_cast<int*>(ws);
  p.batch = s_q;  // one request of s_q query positions
  p.num_sm_parts = num_sm_parts;
  p.s_q = s_q;
  p.h_q = h_q;
  p.rows = h_q;
  p.row_groups = pair ? (h_q + mla::kPairRows - 1) / mla::kPairRows : (h_q + rg - 1) / rg;
  p.causal = 0;
  p.scale_log2 = softmax_scale * 1.4426950408889634f;
  p.kv = kv;
  p.indices = indices;
  p.topk = topk;
  p.vq = s_q;
  mla::OutMaps om;
  if (!encode_out_maps(encode, &om, p.o_part, out, h_q, p.batch, num_sm_parts, rg == 16 ? 16 : 32))
    return MLA_ERR_CUDA;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  int e = pair ? mla::launch_decode_pair_sparse_bf16(tm_q, om, p, st)
               : mla::launch_decode_sparse_bf16(tm_q, om, p, rg, st);
  if (e != 0) return MLA_ERR_CUDA;
  mla::CombineParams cp{};
  cp.num_splits = num_splits;
  cp.o_part = p.o_part;
  cp.lse_part = p.lse_part;
  cp.out = p.out;
  cp.lse = lse;
  cp.batch = s_q;
  cp.s_q = s_q;
  cp.h_q = h_q;
  cp.rows = h_q;
  cp.vq = s_q;
  e = mla::launch_combine(cp, st);
  return e == 0 ? MLA_OK : MLA_ERR_CUDA;
}

int mla_fault_injection_arm(long long wait_limit_cycles, int withhold_fill) {
  if (wait_limit_cycles < 0 || withhold_fill < -1) return MLA_ERR_BAD_SHAPE;
  g_fault_wait_limit.store(wait_limit_cycles);
  g_fault_withhold1.store(withhold_fill + 1);
  return MLA_OK;
}

int mla_read_status(void* workspace, int reset, int* status, void* stream) {
  if (!workspace || !status) return MLA_ERR_NULL_POINTER;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  int v = 0;
  if (cudaMemcpyAsync(&v, workspace, sizeof(int), cudaMemcpyDeviceToHost, st) != cudaSuccess) return MLA_ERR_CUDA;
  if (cudaStreamSynchronize(st) != cudaSuccess) return MLA_ERR_CUDA;
  *status = v;
  if (reset && cudaMemsetAsync(workspace, 0, sizeof(int), st) != cudaSuccess) return MLA_ERR_CUDA;
  return MLA_OK;
}

}  // extern "C"

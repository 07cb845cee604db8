// mla_decode_kvcache_noalloc: the decode call for callers that cannot allocate device memory.
//
// mla_decode_kvcache needs a caller-provided workspace (a status word plus the fp32 partial
// results of requests that are split over several SM parts).  Some callers cannot obtain one
// at the point where they run decode: an engine that reserves all device memory at start-up
// and forbids later allocations, code that runs inside an allocator hook or a driver callback
// where calling an allocator would re-enter it, or a plain C host program that never links an
// allocator at all.  For them the workspace lives here, in a file-scope device array of a
// fixed size that every GPU loading this library holds until the process exits.
//
// Properties (also stated in include/mla.h):
//   - the array holds kNoAllocScratchBytes (16 MiB); problems whose workspace would be larger
//     are rejected with MLA_ERR_SCRATCH_LIMIT before anything is enqueued;
//   - on the first call on a device (with that device current) the array's device address is
//     looked up once with cudaGetSymbolAddress; make that first call before any stream capture;
//   - every call on a device shares the one array and leaves its contents behind; the device
//     status word is cleared (cudaMemsetAsync, no allocation) at the start of each call, the
//     partial results are always written before they are read;
//   - calls that overlap on the GPU (other streams, or other host threads) race on the array;
//   - mla_noalloc_read_status reads the status word back (the caller has no workspace pointer
//     to hand to mla_read_status);
//   - the cached address belongs to the device's current context: after cudaDeviceReset the
//     module is loaded again and the array may move, so do not call these entry points after
//     resetting a device in the same process.
// Nothing here calls cudaMalloc, cudaFree or any allocating routine.
#include <mutex>

#include "mla.h"
#include "mla_internal.h"

namespace {

constexpr size_t kNoAllocScratchBytes = size_t(16) << 20;
constexpr int kMaxDevices = 64;

__device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

std::mutex g_setup_mutex;
void* g_scratch_ptr[kMaxDevices] = {};

// Device address of g_noalloc_scratch on the current device (looked up on first use).
int scratch_for_current_device(void** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return MLA_ERR_NO_DEVICE;
  std::lock_guard<std::mutex> lock(g_setup_mutex);
  if (g_scratch_ptr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) return MLA_ERR_CUDA;
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return MLA_OK;
}

}  // namespace

extern "C" {

int mla_decode_kvcache_noalloc(const void* q, const void* kvcache, int64_t num_blocks, const int32_t* block_table,
                               int max_blocks, const int32_t* cache_seqlens, int batch, int s_q, int h_q, int h_kv,
                               int d_v, const int32_t* tile_md, int num_sm_parts, const int32_t* num_splits,
                               float softmax_scale, int causal, int kv_dtype, void* out, float* lse, void* stream) {
  // Argument checks first, with nothing enqueued: the regular entry point validates every
  // argument before it looks at the workspace size, so a zero-byte workspace makes it stop
  // with MLA_ERR_WORKSPACE exactly when all other arguments are valid.  The stand-in
  // workspace pointer below is only checked for alignment, never dereferenced.
  static const unsigned char kAligned[16] __attribute__((aligned(16))) = {};
  const int v = mla_decode_kvcache(q, kvcache, num_blocks, block_table, max_blocks, cache_seqlens, batch, s_q, h_q,
                                   h_kv, d_v, tile_md, num_sm_parts, num_splits, softmax_scale, causal, kv_dtype,
                                   out, lse, const_cast<unsigned char*>(kAligned), 0, stream);
  if (v != MLA_ERR_WORKSPACE) return v;
  const size_t need = mla_workspace_size(batch, num_sm_parts, s_q * h_q / h_kv, h_kv);
  if (need == 0 || need > kNoAllocScratchBytes) return MLA_ERR_SCRATCH_LIMIT;

  void* ws = nullptr;
  const int e = scratch_for_current_device(&ws);
  if (e != MLA_OK) return e;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (cudaMemsetAsync(ws, 0, sizeof(int), st) != cudaSuccess) return MLA_ERR_CUDA;  // status word
  return mla_decode_kvcache(q, kvcache, num_blocks, block_table, max_blocks, cache_seqlens, batch, s_q, h_q, h_kv,
                            d_v, tile_md, num_sm_parts, num_splits, softmax_scale, causal, kv_dtype, out, lse, ws,
                            kNoAllocScratchBytes, stream);
}

int mla_noalloc_read_status(int reset, int* status, void* stream) {
  if (!status) return MLA_ERR_NULL_POINTER;
  void* ws = nullptr;
  const int e = scratch_for_current_device(&ws);
  if (e != MLA_OK) return e;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  int v = 0;
  if (cudaMemcpyAsync(&v, ws, sizeof(int), cudaMemcpyDeviceToHost, st) != cudaSuccess) return MLA_ERR_CUDA;
  if (cudaStreamSynchronize(st) != cudaSuccess) return MLA_ERR_CUDA;
  *status = v;
  if (reset && cudaMemsetAsync(ws, 0, sizeof(int), st) != cudaSuccess) return MLA_ERR_CUDA;
  return MLA_OK;
}

}  // extern "C"

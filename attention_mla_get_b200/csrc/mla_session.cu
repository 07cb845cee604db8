// Serving session of include/mla.h: decode steps with host inputs and outputs, pipelined two
// steps deep over double-buffered device staging, a copy-in and a copy-out stream.  Host code
// only: each step is the scheduler, decode and combine of mla_api.cu, enqueued on the caller's
// stream between the two copies, ordered by events.
#include <cuda_runtime.h>

#include <cstdint>
#include <new>

#include "mla.h"

struct mla_session {
  int device = 0;
  int batch = 0, s_q = 0, h_q = 0, h_kv = 1, max_blocks = 0, topk = 0, kv_dtype = 0, parts = 0;
  size_t q_bytes = 0, bt_bytes = 0, sl_bytes = 0, idx_bytes = 0, out_bytes = 0, lse_bytes = 0, ws_bytes = 0;
  size_t md_bytes = 0, ns_bytes = 0;
  void* q[2] = {nullptr, nullptr};
  void* bt[2] = {nullptr, nullptr};
  void* sl[2] = {nullptr, nullptr};
  void* idx[2] = {nullptr, nullptr};
  void* out[2] = {nullptr, nullptr};
  void* lse[2] = {nullptr, nullptr};
  void* tile_md = nullptr;
  void* num_splits = nullptr;
  void* ws = nullptr;
  cudaStream_t s_in = nullptr, s_out = nullptr;
  cudaEvent_t in_ready[2] = {nullptr, nullptr};
  cudaEvent_t computed[2] = {nullptr, nullptr};
  cudaEvent_t out_read[2] = {nullptr, nullptr};
  cudaEvent_t begin = nullptr;
  long long steps = 0;  // steps enqueued
  bool fresh = true;    // the next copy-in is ordered after the caller's stream
};

namespace {

// restores the calling thread's current device on scope exit
struct DeviceGuard {
  int prev = -1;
  explicit DeviceGuard(int dev) {
    if (cudaGetDevice(&prev) != cudaSuccess) prev = -1;
    if (prev != dev) cudaSetDevice(dev);
  }
  ~DeviceGuard() {
    int cur = -1;
    if (prev >= 0 && cudaGetDevice(&cur) == cudaSuccess && cur != prev) cudaSetDevice(prev);
  }
};

void release(mla_session* s) {
  for (int i = 0; i < 2; ++i) {
    for (void* p : {s->q[i], s->bt[i], s->sl[i], s->idx[i], s->out[i], s->lse[i]})
      if (p) cudaFree(p);
    for (cudaEvent_t e : {s->in_ready[i], s->computed[i], s->out_read[i]})
      if (e) cudaEventDestroy(e);
  }
  if (s->tile_md) cudaFree(s->tile_md);
  if (s->num_splits) cudaFree(s->num_splits);
  if (s->ws) cudaFree(s->ws);
  if (s->begin) cudaEventDestroy(s->begin);
  if (s->s_in) cudaStreamDestroy(s->s_in);
  if (s->s_out) cudaStreamDestroy(s->s_out);
  delete s;
}

// waits for every device operation of the session (copies and the steps' kernels)
cudaError_t wait_all(mla_session* s) {
  cudaError_t e = cudaSuccess;
  for (int i = 0; i < 2; ++i) {
    if (s->steps > i) {
      const cudaError_t a = cudaEventSynchronize(s->computed[i]);
      const cudaError_t b = cudaEventSynchronize(s->out_read[i]);
      if (e == cudaSuccess) e = a != cudaSuccess ? a : b;
    }
  }
  const cudaError_t c = cudaStreamSynchronize(s->s_in);
  return e != cudaSuccess ? e : c;
}

}  // namespace

extern "C" {

MLA_API int mla_session_create(int device, int batch, int s_q, int h_q, int h_kv, int max_blocks, int topk,
                               int kv_dtype, int num_sm_parts, mla_session** session) {
  if (!session) return MLA_ERR_NULL_POINTER;
  *session = nullptr;
  if (h_kv != 1 || h_q < 1) return MLA_ERR_BAD_HEADS;
  if (kv_dtype != MLA_KV_BF16 && kv_dtype != MLA_KV_FP8) return MLA_ERR_BAD_KV_DTYPE;
  if (topk > 0 && kv_dtype != MLA_KV_BF16) return MLA_ERR_BAD_KV_DTYPE;
  if (batch < 1 || s_q < 1 || max_blocks < 1 || topk < 0) return MLA_ERR_BAD_SHAPE;
  const long long rows = static_cast<long long>(s_q) * h_q;
  if ((topk > 0 ? h_q : rows) > 4096) return MLA_ERR_BAD_SHAPE;
  if (static_cast<long long>(batch) * s_q >= (1ll << 30)) return MLA_ERR_BAD_SHAPE;
  if (num_sm_parts < 1) return MLA_ERR_BAD_PARTS;
  int ndev = 0;
  if (cudaGetDeviceCount(&ndev) != cudaSuccess || device < 0 || device >= ndev) return MLA_ERR_NO_DEVICE;
  DeviceGuard guard(device);

  mla_session* s = new (std::nothrow) mla_session();
  if (!s) return MLA_ERR_CUDA;
  s->device = device;
  s->batch = batch;
  s->s_q = s_q;
  s->h_q = h_q;
  s->h_kv = h_kv;
  s->max_blocks = max_blocks;
  s->topk = topk;
  s->kv_dtype = kv_dtype;
  s->parts = num_sm_parts;
  const size_t positions = static_cast<size_t>(batch) * s_q;
  s->q_bytes = positions * h_q * 576 * 2;
  s->bt_bytes = static_cast<size_t>(batch) * max_blocks * 4;
  s->sl_bytes = static_cast<size_t>(batch) * 4;
  s->idx_bytes = positions * static_cast<size_t>(topk) * 4;
  s->out_bytes = positions * h_q * 512 * 2;
  s->lse_bytes = positions * h_q * 4;
  s->md_bytes = static_cast<size_t>(num_sm_parts) * 8 * 4;
  s->ns_bytes = ((topk > 0 ? positions : static_cast<size_t>(batch)) + 1) * 4;
  s->ws_bytes = topk > 0 ? mla_workspace_size(static_cast<int>(positions), num_sm_parts, h_q, h_kv)
                         : mla_workspace_size(batch, num_sm_parts, static_cast<int>(rows), h_kv);

  bool ok = true;
  auto alloc = [&](void** p, size_t bytes) {
    if (ok && bytes > 0) ok = cudaMalloc(p, bytes) == cudaSuccess;
  };
  for (int i = 0; i < 2; ++i) {
    alloc(&s->q[i], s->q_bytes);
    alloc(&s->bt[i], s->bt_bytes);
    alloc(&s->sl[i], s->sl_bytes);
    alloc(&s->idx[i], s->idx_bytes);
    alloc(&s->out[i], s->out_bytes);
    alloc(&s->lse[i], s->lse_bytes);
    for (cudaEvent_t* e : {&s->in_ready[i], &s->computed[i], &s->out_read[i]})
      if (ok) ok = cudaEventCreateWithFlags(e, cudaEventDisableTiming) == cudaSuccess;
  }
  alloc(&s->tile_md, s->md_bytes);
  alloc(&s->num_splits, s->ns_bytes);
  alloc(&s->ws, s->ws_bytes);
  if (ok) ok = cudaMemset(s->ws, 0, s->ws_bytes) == cudaSuccess;
  if (ok) ok = cudaEventCreateWithFlags(&s->begin, cudaEventDisableTiming) == cudaSuccess;
  if (ok) ok = cudaStreamCreateWithFlags(&s->s_in, cudaStreamNonBlocking) == cudaSuccess;
  if (ok) ok = cudaStreamCreateWithFlags(&s->s_out, cudaStreamNonBlocking) == cudaSuccess;
  if (ok) ok = cudaDeviceSynchronize() == cudaSuccess;  // the zeroed workspace is in place
  if (!ok) {
    release(s);
    return MLA_ERR_CUDA;
  }
  *session = s;
  return MLA_OK;
}

MLA_API int mla_session_decode(mla_session* s, const void* q_host, const void* kvcache, int64_t num_blocks,
                               const int32_t* block_table_host, const int32_t* cache_seqlens_host,
                               const int32_t* indices_host, float softmax_scale, int causal, void* out_host,
                               float* lse_host, void* stream) {
  if (!s || !q_host || !kvcache || !block_table_host || !cache_seqlens_host || !out_host || !lse_host)
    return MLA_ERR_NULL_POINTER;
  if ((s->topk > 0) != (indices_host != nullptr)) return MLA_ERR_NULL_POINTER;
  DeviceGuard guard(s->device);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int b = static_cast<int>(s->steps & 1);
  bool ok = true;
  auto chk = [&](cudaError_t e) { ok = ok && e == cudaSuccess; };
  if (s->fresh) {
    // nothing of this step is copied before the work already enqueued on `stream`
    chk(cudaEventRecord(s->begin, st));
    chk(cudaStreamWaitEvent(s->s_in, s->begin, 0));
    s->fresh = false;
  }
  // copy-in, once step k - 2 has read staging set b
  if (s->steps >= 2) chk(cudaStreamWaitEvent(s->s_in, s->computed[b], 0));
  chk(cudaMemcpyAsync(s->q[b], q_host, s->q_bytes, cudaMemcpyHostToDevice, s->s_in));
  chk(cudaMemcpyAsync(s->bt[b], block_table_host, s->bt_bytes, cudaMemcpyHostToDevice, s->s_in));
  chk(cudaMemcpyAsync(s->sl[b], cache_seqlens_host, s->sl_bytes, cudaMemcpyHostToDevice, s->s_in));
  if (s->topk > 0) chk(cudaMemcpyAsync(s->idx[b], indices_host, s->idx_bytes, cudaMemcpyHostToDevice, s->s_in));
  chk(cudaEventRecord(s->in_ready[b], s->s_in));
  if (!ok) return MLA_ERR_CUDA;

  // the step on the caller's stream, once its inputs are in and step k - 2's outputs are out
  chk(cudaStreamWaitEvent(st, s->in_ready[b], 0));
  if (s->steps >= 2) chk(cudaStreamWaitEvent(st, s->out_read[b], 0));
  if (!ok) return MLA_ERR_CUDA;
  int32_t* md = static_cast<int32_t*>(s->tile_md);
  int32_t* ns = static_cast<int32_t*>(s->num_splits);
  int rc;
  if (s->topk > 0) {
    rc = mla_get_metadata_sparse(s->batch, s->s_q, s->topk, s->h_q, s->h_kv, md, s->parts, ns, stream);
    if (rc == MLA_OK)
      rc = mla_decode_kvcache_sparse(s->q[b], kvcache, num_blocks, static_cast<const int32_t*>(s->bt[b]),
                                     s->max_blocks, static_cast<const int32_t*>(s->sl[b]), s->batch, s->s_q, s->h_q,
                                     s->h_kv, 512, static_cast<const int32_t*>(s->idx[b]), s->topk, md, s->parts, ns,
                                     softmax_scale, s->kv_dtype, s->out[b], static_cast<float*>(s->lse[b]), s->ws,
                                     s->ws_bytes, stream);
  } else {
    const int rows = s->s_q * s->h_q;
    rc = mla_get_metadata(static_cast<const int32_t*>(s->sl[b]), s->batch, rows, s->h_kv, md, s->parts, ns, stream);
    if (rc == MLA_OK)
      rc = mla_decode_kvcache(s->q[b], kvcache, num_blocks, static_cast<const int32_t*>(s->bt[b]), s->max_blocks,
                              static_cast<const int32_t*>(s->sl[b]), s->batch, s->s_q, s->h_q, s->h_kv, 512, md,
                              s->parts, ns, softmax_scale, causal, s->kv_dtype, s->out[b],
                              static_cast<float*>(s->lse[b]), s->ws, s->ws_bytes, stream);
  }
  // the events are recorded whatever happened, so that the next step's waits stay well defined
  chk(cudaEventRecord(s->computed[b], st));
  chk(cudaStreamWaitEvent(s->s_out, s->computed[b], 0));
  chk(cudaMemcpyAsync(out_host, s->out[b], s->out_bytes, cudaMemcpyDeviceToHost, s->s_out));
  chk(cudaMemcpyAsync(lse_host, s->lse[b], s->lse_bytes, cudaMemcpyDeviceToHost, s->s_out));
  chk(cudaEventRecord(s->out_read[b], s->s_out));
  ++s->steps;
  if (rc != MLA_OK) return rc;
  return ok ? MLA_OK : MLA_ERR_CUDA;
}

MLA_API int mla_session_join(mla_session* s, void* stream) {
  if (!s) return MLA_ERR_NULL_POINTER;
  DeviceGuard guard(s->device);
  s->fresh = true;
  if (s->steps == 0) return MLA_OK;
  // copy-outs run in order on one stream: the last step's covers the earlier ones
  const int last = static_cast<int>((s->steps - 1) & 1);
  return cudaStreamWaitEvent(static_cast<cudaStream_t>(stream), s->out_read[last], 0) == cudaSuccess ? MLA_OK
                                                                                                       : MLA_ERR_CUDA;
}

MLA_API int mla_session_status(mla_session* s, int reset, int* status) {
  if (!s || !status) return MLA_ERR_NULL_POINTER;
  DeviceGuard guard(s->device);
  if (wait_all(s) != cudaSuccess) return MLA_ERR_CUDA;
  return mla_read_status(s->ws, reset, status, s->s_in);
}

MLA_API int mla_session_destroy(mla_session* s) {
  if (!s) return MLA_ERR_NULL_POINTER;
  DeviceGuard guard(s->device);
  const cudaError_t e = wait_all(s);
  release(s);
  return e == cudaSuccess ? MLA_OK : MLA_ERR_CUDA;
}

}  // extern "C"

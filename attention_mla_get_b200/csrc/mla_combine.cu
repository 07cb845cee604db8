// Split-KV combine (FlashMLA pages: the combine kernel that follows splitkv_mla and is
// overlapped with it by programmatic dependent launch, wmrh.cn page "计算流水线设计").
//
// For a request whose blocks were split over several SM parts, every split s wrote
//   O_s   = its own softmax-normalised output (fp32, [R, 512])
//   lse_s = log of its own softmax denominator plus its max (natural log)
// and the exact result is  LSE = log sum_s exp(lse_s),  O = sum_s exp(lse_s - LSE) * O_s.
// Requests with exactly one split were written directly by the main kernel; requests
// with none (cache length 0) get O = 0 and LSE = -inf here.
//
// One warp per output row, 16 dims per lane as four float4 loads, splits streamed in
// order.  The kernel is launched with the programmatic-stream-serialization attribute and
// blocks in griddepcontrol.wait until the main kernel's writes are visible.
#include <cuda_bf16.h>
#include <math_constants.h>

#include "mla_internal.h"
#include "mla_ptx.cuh"

namespace mla {

namespace {

constexpr int kCombineWarps = 8;

__global__ void __launch_bounds__(kCombineWarps * 32) mla_combine_kernel(const CombineParams p) {
  const int b = blockIdx.x;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int row = blockIdx.y * kCombineWarps + warp;
  pdl_wait_primary();
  const int s0 = p.num_splits[b];
  const int ns = p.num_splits[b + 1] - s0;
  if (ns == 1 || row >= p.rows) return;
  const int R = p.rows;
  const long long orow = static_cast<long long>(b) * R + row;
  // token-sparse: request b is query position (b / vq, b % vq) and its rows are the heads
  float* lse_out = p.vq > 0 ? p.lse + (static_cast<long long>(b / p.vq) * p.h_q + row) * p.vq + b % p.vq
                            : p.lse + (static_cast<long long>(b) * p.h_q + row % p.h_q) * p.s_q + row / p.h_q;
  __nv_bfloat16* out = p.out + orow * kDv;
  if (ns == 0) {
    for (int d = lane; d < kDv; d += 32) out[d] = __float2bfloat16_rn(0.f);
    if (lane == 0) *lse_out = -CUDART_INF_F;
    return;
  }
  float m = -CUDART_INF_F;
  for (int s = lane; s < ns; s += 32) m = fmaxf(m, p.lse_part[static_cast<long long>(s0 + s) * R + row]);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  float acc[16];
#pragma unroll
  for (int i = 0; i < 16; ++i) acc[i] = 0.f;
  if (m == -CUDART_INF_F) {
    // no split saw a visible key
    for (int d = lane; d < kDv; d += 32) out[d] = __float2bfloat16_rn(0.f);
    if (lane == 0) *lse_out = -CUDART_INF_F;
    return;
  }
  float sum = 0.f;
  for (int s = lane; s < ns; s += 32) sum += expf(p.lse_part[static_cast<long long>(s0 + s) * R + row] - m);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
  const float lse = m + logf(sum);
  // unrolled so that the loads of several splits are in flight together
#pragma unroll 4
  for (int s = 0; s < ns; ++s) {
    const float w = expf(p.lse_part[static_cast<long long>(s0 + s) * R + row] - lse);
    const float4* src = reinterpret_cast<const float4*>(p.o_part + (static_cast<long long>(s0 + s) * R + row) * kDv);
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const float4 v = src[k * 32 + lane];
      acc[4 * k + 0] += w * v.x;
      acc[4 * k + 1] += w * v.y;
      acc[4 * k + 2] += w * v.z;
      acc[4 * k + 3] += w * v.w;
    }
  }
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const int d = 4 * (k * 32 + lane);
    uint2 packed;
    packed.x = pack_bf16x2(acc[4 * k + 0], acc[4 * k + 1]);
    packed.y = pack_bf16x2(acc[4 * k + 2], acc[4 * k + 3]);
    *reinterpret_cast<uint2*>(out + d) = packed;
  }
  if (lane == 0) *lse_out = lse;
}

}  // namespace

int launch_combine(const CombineParams& p, cudaStream_t stream) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(p.batch, (p.rows + kCombineWarps - 1) / kCombineWarps, 1);
  cfg.blockDim = dim3(kCombineWarps * 32, 1, 1);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaError_t e = cudaLaunchKernelEx(&cfg, mla_combine_kernel, p);
  return static_cast<int>(e);
}

}  // namespace mla

// Tile scheduler (get_mla_metadata on the FlashMLA pages: tile_scheduler_metadata
// [num_sm_parts x TileSchedulerMetaDataSize] and num_splits [batch + 1], "flash_api.cpp"
// excerpt on the mmssai.com page; the scheduler balances requests and blocks over the
// SMs, wmrh.cn page "计算流水线设计").
//
// The rule is integer-only and runs in one thread: it is O(batch + num_sm_parts) work
// done once per decode step and reused by every layer.  It is:
//   n_b      = ceil(L_b / 128) blocks (0 for L_b <= 0)
//   T        = sum over n_b > 0 of (n_b + F),  F = kFixedSplitCost
//   payload  = ceil(T / P) + F
//   each part p, with budget = payload, takes chunks k = min(n_b - blk, budget - F)
//   while budget > F, paying F + k per chunk, the cursor (b, blk) moving forward
//   (skipping requests with n_b = 0).
//   row p = {begin_b, begin_blk, end_b, end_blk, first_split, 0, 0, 0}
//   num_splits[b+1] = num_splits[b] + chunks of b; a chunk's split index is
//   num_splits[b] + its ordinal within b.
#include "mla_internal.h"

namespace mla {

__device__ __forceinline__ int blocks_of(int L) { return L > 0 ? (L + kBlockTokens - 1) / kBlockTokens : 0; }

__global__ void __launch_bounds__(32) mla_tile_scheduler_kernel(const int32_t* __restrict__ seqlens, int batch,
                                                                int parts, int32_t* __restrict__ md,
                                                                int32_t* __restrict__ num_splits) {
  if (threadIdx.x != 0) return;
  const int F = kFixedSplitCost;
  long long T = 0;
  for (int b = 0; b < batch; ++b) {
    const int n = blocks_of(seqlens[b]);
    num_splits[b + 1] = 0;  // chunk counts first, prefix sums after the walk
    if (n > 0) T += n + F;
  }
  num_splits[0] = 0;
  const long long payload = (T + parts - 1) / parts + F;

  int b = 0;
  while (b < batch && blocks_of(seqlens[b]) == 0) ++b;
  int blk = 0;
  for (int p = 0; p < parts; ++p) {
    const int begin_b = b, begin_blk = blk;
    const int first_ordinal = b < batch ? num_splits[b + 1] : 0;
    long long budget = payload;
    while (budget > F && b < batch) {
      const int n = blocks_of(seqlens[b]);
      const long long room = budget - F;
      const int k = (n - blk) < room ? (n - blk) : static_cast<int>(room);
      num_splits[b + 1] += 1;
      budget -= F + k;
      blk += k;
      if (blk == n) {
        ++b;
        while (b < batch && blocks_of(seqlens[b]) == 0) ++b;
        blk = 0;
      }
    }
    int32_t* row = md + static_cast<long long>(p) * kMdInts;
    row[0] = begin_b;
    row[1] = begin_blk;
    row[2] = b;
    row[3] = blk;
    row[4] = first_ordinal;  // made absolute below
    row[5] = row[6] = row[7] = 0;
  }
  for (int i = 0; i < batch; ++i) num_splits[i + 1] += num_splits[i];
  for (int p = 0; p < parts; ++p) {
    int32_t* row = md + static_cast<long long>(p) * kMdInts;
    row[4] += num_splits[row[0]];
  }
}

int launch_scheduler(const int32_t* cache_seqlens, int batch, int num_sm_parts, int32_t* tile_md,
                     int32_t* num_splits, cudaStream_t stream) {
  mla_tile_scheduler_kernel<<<1, 32, 0, stream>>>(cache_seqlens, batch, num_sm_parts, tile_md, num_splits);
  return static_cast<int>(cudaGetLastError());
}

}  // namespace mla

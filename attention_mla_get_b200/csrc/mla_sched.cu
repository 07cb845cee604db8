// Tile scheduler (get_mla_metadata on the FlashMLA pages: tile_scheduler_metadata
// [num_sm_parts x TileSchedulerMetaDataSize] and num_splits [batch + 1], "flash_api.cpp"
// excerpt on the mmssai.com page; the scheduler balances requests and blocks over the
// SMs, wmrh.cn page "计算流水线设计").
//
// The rule (integer only):
//   n_b    = ceil(L_b / 128) blocks (0 for L_b <= 0)
//   cost   requests with n_b > 0 laid end to end, F + n_b units each (F = kFixedSplitCost);
//          C_b = start of request b, block j of request b sits at C_b + F + j, T = total
//   q      = ceil(T / P); part p owns the positions [p*q, (p+1)*q)
//   row p  = {begin_b, begin_blk, end_b, end_blk, first_split, 0, 0, 0} where begin / end are
//            the first block at a position >= p*q / >= (p+1)*q; (batch, 0) when there is none
//   chunks of b = (last owner part) - (first owner part) + 1 = floor((C_b+F+n_b-1)/q) - floor((C_b+F)/q) + 1
//   num_splits = prefix sum of chunks; first_split = num_splits[begin_b] + p - floor((C_b+F)/q)
// Every quantity is a closed form of prefix sums, so one CTA of 1024 threads computes the
// metadata in a few microseconds: a scan of costs, a binary search per part, a scan of
// chunk counts.  A batch whose total cost T does not fit in 31 bits gets empty parts flagged
// with kMdOverflow in column 5 (and no splits); the decode kernels report it as a status bit.
#include "mla_internal.h"
#include "mla_ptx.cuh"

namespace mla {

namespace {

constexpr int kSchedThreads = 1024;
constexpr int kSmemBatch = 8192;  // batches up to this size keep the prefix array in shared memory

__device__ __forceinline__ long long blocks_of(int L) { return L > 0 ? (L + kBlockTokens - 1) / kBlockTokens : 0; }

// Inclusive scan of v over the CTA (any multiple of 32 threads up to 1024); returns the
// thread's inclusive prefix, *total gets the sum.
__device__ long long block_scan(long long v, long long* warp_tot, long long* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const long long u = __shfl_up_sync(0xffffffffu, v, o);
    if (lane >= o) v += u;
  }
  if (lane == 31) warp_tot[warp] = v;
  __syncthreads();
  if (warp == 0) {
    long long w = lane < static_cast<int>(blockDim.x >> 5) ? warp_tot[lane] : 0;  // absent warps: 0
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const long long u = __shfl_up_sync(0xffffffffu, w, o);
      if (lane >= o) w += u;
    }
    warp_tot[lane] = w;  // inclusive over warps
  }
  __syncthreads();
  const long long before = warp == 0 ? 0 : warp_tot[warp - 1];
  const long long tot = warp_tot[31];
  __syncthreads();
  if (total) *total = tot;
  return v + before;
}

__global__ void __launch_bounds__(kSchedThreads)
    mla_tile_scheduler_kernel(const int32_t* __restrict__ seqlens, int uniform_len, int batch, int parts,
                              int32_t* __restrict__ md, int32_t* __restrict__ ns) {
  // seqlens == nullptr: every request has uniform_len tokens (token-sparse decode: the
  // requests are the query positions, each over its topk listed positions)
  __shared__ long long warp_tot[32];
  __shared__ int32_t s_cum[kSmemBatch + 1];  // C_{b+1}: binary searches stay on chip
  const long long F = kFixedSplitCost;
  const int tid = threadIdx.x;
  const bool on_chip = batch <= kSmemBatch;
  pdl_launch_dependents();  // the decode kernel's set-up may start now; it waits for this grid

  const int nthreads = static_cast<int>(blockDim.x);
  // pass 1: ns[b + 1] = C_{b+1} (inclusive prefix of costs), T
  long long carry = 0;
  long long n_first = 0;  // this thread's cost in the first tile (reused by pass 3 when it is the only one)
  for (int base = 0; base < batch; base += nthreads) {
    const int b = base + tid;
    const long long n = b < batch ? blocks_of(seqlens ? seqlens[b] : uniform_len) : 0;
    if (base == 0) n_first = n;
    long long tile_total;
    const long long incl = block_scan(n > 0 ? n + F : 0, warp_tot, &tile_total) + carry;
    if (b < batch) {
      ns[b + 1] = static_cast<int32_t>(incl);
      if (on_chip) s_cum[b + 1] = static_cast<int32_t>(incl);
    }
    carry += tile_total;
  }
  if (tid == 0) {
    ns[0] = 0;
    s_cum[0] = 0;
  }
  const long long T = carry;
  const long long q = T > 0 ? (T + parts - 1) / parts : 1;
  __syncthreads();
  if (T > 0x7fffffffll) {
    // the prefix sums above were stored as 32-bit values and wrapped: publish empty parts
    // flagged kMdOverflow (the decode kernels raise a status bit) and no splits at all
    for (int p = tid; p < parts; p += nthreads) {
      int32_t* row = md + static_cast<long long>(p) * kMdInts;
      row[0] = batch;
      row[1] = 0;
      row[2] = batch;
      row[3] = 0;
      row[4] = 0;
      row[5] = kMdOverflow;
      row[6] = row[7] = 0;
    }
    for (int b = tid; b <= batch; b += nthreads) ns[b] = 0;
    return;
  }

  // pass 2: per part, the first block at a position >= x (binary search on C_{b+1})
  const int32_t* cum = on_chip ? s_cum : ns;  // C_{b+1} at index b + 1
  auto find = [&](long long x, int& fb, int& fj) {
    int lo = 0, hi = batch;
    while (lo < hi) {
      const int mid = (lo + hi) >> 1;
      if (static_cast<long long>(cum[mid + 1]) > x) hi = mid;
      else lo = mid + 1;
    }
    fb = lo;
    if (lo >= batch) {
      fj = 0;
      return;
    }
    const long long cb = lo == 0 ? 0 : cum[lo];
    const long long j = x - (cb + F);
    fj = j > 0 ? static_cast<int>(j) : 0;
  };
  for (int p = tid; p < parts; p += nthreads) {
    int bb, bj, eb, ej;
    find(static_cast<long long>(p) * q, bb, bj);
    find(static_cast<long long>(p + 1) * q, eb, ej);
    int ordinal = 0;
    if ((bb != eb || bj != ej) && bb < batch) {
      const long long cb = bb == 0 ? 0 : cum[bb];
      ordinal = static_cast<int>(p - (cb + F) / q);
    }
    int32_t* row = md + static_cast<long long>(p) * kMdInts;
    row[0] = bb;
    row[1] = bj;
    row[2] = eb;
    row[3] = ej;
    row[4] = ordinal;  // made absolute in pass 4
    row[5] = row[6] = row[7] = 0;
  }
  __syncthreads();

  // pass 3: ns = prefix sum of chunk counts (costs are scanned again instead of read back,
  // because ns is overwritten here)
  carry = 0;
  long long chunk_carry = 0;
  for (int base = 0; base < batch; base += nthreads) {
    const int b = base + tid;
    const long long n = batch <= nthreads ? n_first : (b < batch ? blocks_of(seqlens ? seqlens[b] : uniform_len) : 0);
    long long tile_total;
    const long long incl = block_scan(n > 0 ? n + F : 0, warp_tot, &tile_total) + carry;
    const long long cb = incl - (n > 0 ? n + F : 0);
    const long long chunks = n > 0 ? (cb + F + n - 1) / q - (cb + F) / q + 1 : 0;
    long long chunk_total;
    const long long cincl = block_scan(chunks, warp_tot, &chunk_total) + chunk_carry;
    if (b < batch) ns[b + 1] = static_cast<int32_t>(cincl);
    carry += tile_total;
    chunk_carry += chunk_total;
  }
  __syncthreads();

  // pass 4: absolute split index of each part's first chunk
  for (int p = tid; p < parts; p += nthreads) {
    int32_t* row = md + static_cast<long long>(p) * kMdInts;
    row[4] += ns[row[0]];
  }
}

}  // namespace

int launch_scheduler(const int32_t* cache_seqlens, int batch, int num_sm_parts, int32_t* tile_md,
                     int32_t* num_splits, cudaStream_t stream, int uniform_len) {
  // one thread per request (and per part), in whole warps, at most kSchedThreads: small batches
  // take fewer, cheaper barriers
  const int want = batch > num_sm_parts ? batch : num_sm_parts;
  const int threads = want >= kSchedThreads ? kSchedThreads : (want < 32 ? 32 : (want + 31) / 32 * 32);
  mla_tile_scheduler_kernel<<<1, threads, 0, stream>>>(cache_seqlens, uniform_len, batch, num_sm_parts, tile_md,
                                                       num_splits);
  return static_cast<int>(cudaGetLastError());
}

}  // namespace mla

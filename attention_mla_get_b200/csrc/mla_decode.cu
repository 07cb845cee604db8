// Split-KV MLA decode main kernel for sm_100a (bf16 or FP8 paged KV cache).
//
// Problem (FlashMLA pages: mha_fwd_kvcache_mla / run_mha_fwd_splitkv_mla<bf16, 576> in the
// "flash_api.cpp" excerpt, mmssai.com page; 64-token pages addressed by block_table,
// kdjingpai.com page; query folding q.view(b, s_q, h_kv, ngroups, d).transpose(2, 3),
// deepseekonline.chat page): for each request, R = s_q*h_q query rows attend to one shared
// latent KV of 576 dims; V is the first 512 dims of the same cached vector.
//
// Design (B200-native, "swap-AB"): the KV tile is the large operand, so it is the M side
// of every tcgen05 MMA and the query rows are the N side:
//   S^T [128 tokens x RG rows]  = K_tile[128 x 576]  . Q^T[576 x RG]      (fp32 in TMEM)
//   O^T [512 dims  x RG rows] += V_tile^T[512 x 128] . P^T[128 x RG]      (fp32 in TMEM)
// One CTA carries RG = 16, 32 or 64 query rows (more rows per request run on the CTA pair of
// mla_decode_pair.cu), so O^T needs only 4*RG TMEM columns and the whole 512-dim output stays
// in TMEM.
// A step covers 128 tokens (two 64-token pages).  Pages are TMA-loaded through the block
// table in 64x64 boxes (the 9-boxes-per-page split on the wmrh.cn page, "内存访问优化策略")
// into 32 KB ring slots (128 tokens x 128 dims, 128-byte swizzle).  The same slot layout is
// read K-major by QK^T and MN-major (as V^T) by PV, so V is never transposed.
//
// Roles: warps 0-3 online softmax + epilogue (thread = token lane of S^T, then dim lane of
// O^T), warp 4 TMA producer (one lane), warp 5 MMA issuer and TMEM owner (the whole warp,
// converged, one elected lane issuing each MMA and commit), warps 6-13 (16- and 32-row tiles) or
// 6-9 (64-row tiles) FP8 dequant.
// Online softmax keeps a per-row running reference max (log2 units) and rescales O^T in
// TMEM only when a block max exceeds it by more than kTau (the running-max-and-scale idea
// of the wmrh.cn page, "跷跷板调度算法" paragraph); P^T is written to shared memory as
// bf16, the row sums use the unrounded fp32 P.
//
// Issue order.  The ring of slots is filled and consumed in one fixed order per chunk of n
// steps:  K(0) .. K(kLook),  then for t = 0 .. n-1:  V(t), K(t + kLook + 1).
// K(t) is five slots (dims 0-127, ..., 384-511, and the 64 RoPE dims); V(t) is four slots
// re-reading dims 0-511 of the same pages (an L2 hit).  QK(t) only needs K(t) and a free S^T
// buffer, so it runs kLook steps ahead of PV(t), which waits for softmax(t).  Softmax
// therefore always has kLook steps of MMA work to hide behind, the ring recycles at MMA
// speed, and the tensor core never idles on the softmax (kLook + 1 S^T buffers in TMEM).
//
// FP8 cache (656-byte tokens: 512 e4m3 codes, 4 fp32 scales, 64 bf16 RoPE dims; wmrh.cn
// page, "FP8 KV缓存内存效率" table): the producer TMA-loads raw code columns (128 dims x 64
// tokens) and the per-token scales into a raw ring; a dequant warpgroup writes code * scale as
// bf16 into the same swizzled slot ring the MMA reads (same order as above), and TMA-loads the
// RoPE dims straight into their slot with the 128-byte swizzle.  Tokens past the end of the
// request are written as zeros, so no tail fix-up is needed.
//
// Token-sparse decode (SPARSE, bf16): seven gather warps copy the listed tokens' rows into the
// slots with 16-byte cp.async (see the kernel's gather branch).  The epilogue writes each group
// of rows of O^T through the P^T buffers with a TMA tensor store, and the kernel is launched as
// a programmatic dependent of the tile scheduler (set-up first, then it waits for the metadata).
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <math_constants.h>

#include "mla_internal.h"
#include "mla_ptx.cuh"

namespace mla {

namespace {

constexpr float kTau = 8.0f;  // lazy-rescale threshold, log2 units (P <= 2^8)
constexpr float kLn2 = 0.69314718055994530942f;
constexpr int kLook = 1;           // QK runs this many steps ahead of PV (2 measured no faster)
constexpr int kNumS = kLook + 1;   // S^T buffers in TMEM
constexpr int kMaxSlots = 6;

template <int RG, bool FP8>
struct Cfg {
  // FP8: warps converting e4m3 codes to bf16 slots; 16- and 32-row tiles have the registers for
  // eight (two threads per token, one 64-dim atom column each), 64-row tiles keep four
  static constexpr int kDequantWarps = (FP8 && RG <= 32) ? 8 : 4;
  static constexpr int kThreads = FP8 ? 192 + 32 * kDequantWarps : 192;
  static constexpr int kSlotBytes = 32768;   // 128 tokens x 128 dims bf16
  static constexpr int kAtomColBytes = 16384;// 128 tokens x 64 dims (one swizzle column)
  static constexpr int kPageBoxBytes = 8192; // 64 tokens x 64 dims: one TMA box
  static constexpr int kQAtomBytes = RG * 128;
  static constexpr int kQBytes = 9 * kQAtomBytes;
  static constexpr int kPRowBytes = RG * 2;  // one token row of P^T (MN-major, rows contiguous)
  static constexpr int kPBytes = 128 * kPRowBytes;
  static constexpr int kNumP = (RG == 64) ? 1 : 2;
  static constexpr int kNumSlots = FP8 ? (RG == 64 ? 3 : 4) : (RG == 16 ? 6 : (RG == 64 ? 4 : 5));
  static constexpr int kNumRaw = FP8 ? 2 : 0;   // raw e4m3 code columns, 128 tokens x 128 bytes
  static constexpr int kRawBytes = 16384;
  static constexpr int kScaleBytes = 2048;       // 128 tokens x 4 fp32 scales
  static constexpr int kNumScale = FP8 ? kNumS : 0;
  static constexpr int kTmemCols = RG == 16 ? 128 : (RG == 32 ? 256 : 512);
  static constexpr int kOffQ = 0;
  static constexpr int kOffP = kOffQ + kQBytes;
  static constexpr int kOffSlots = kOffP + kNumP * kPBytes;
  static constexpr int kOffRaw = kOffSlots + kNumSlots * kSlotBytes;
  static constexpr int kOffScale = kOffRaw + kNumRaw * kRawBytes;
  static constexpr int kOffMisc = kOffScale + kNumScale * kScaleBytes;
  static constexpr int kMiscBytes = FP8 ? 3072 : 6656;  // bf16: + 7 x 512 B of token-sparse row tables
  static constexpr int kSmemBytes = kOffMisc + kMiscBytes + 1024;  // + alignment slack
  static constexpr uint32_t kPSwzMask = RG / 8 - 1;                // (row bytes / 16) - 1
  static constexpr uint32_t kPLayout = RG == 64 ? kSwizzle128 : (RG == 32 ? kSwizzle64 : kSwizzle32);
  static constexpr uint32_t kIdescQK = idesc_bf16(128, RG, false, false);
  static constexpr uint32_t kIdescPV = idesc_bf16(128, RG, true, true);
  static constexpr int kColO = 0;       // 4 blocks of RG columns: O^T dims 128j..128j+127
  static constexpr int kColS = 4 * RG;  // kNumS buffers of RG columns: S^T
  static constexpr int kNOut = RG == 64 ? 2 : 1;  // columns per lane after a warp reduce-scatter
  static_assert(kSmemBytes <= 232448, "shared memory budget");
  static_assert(kNumSlots <= kMaxSlots, "slot barriers");
  static_assert(kColS + kNumS * RG <= kTmemCols, "TMEM budget");
  static_assert(kQBytes % 1024 == 0 && kPBytes % 1024 == 0, "swizzle atoms need 1024-byte alignment");
};

// barrier indices in the misc area
enum : int {
  kBarSlotFull = 0,     // [kMaxSlots]
  kBarSlotEmpty = 6,    // [kMaxSlots]
  kBarSFull = 12,       // [kNumS]
  kBarSEmpty = 15,      // [kNumS]
  kBarPFull = 18,       // [2]
  kBarPEmpty = 20,      // [2]
  kBarQFull = 22,
  kBarQEmpty = 23,
  kBarOFull = 24,
  kBarOEmpty = 25,
  kBarDrain = 26,
  kBarRawFull = 27,     // [2]
  kBarRawEmpty = 29,    // [2]
  kBarScaleFull = 31,   // [kNumS]
  kBarScaleEmpty = 34,  // [kNumS]
  kNumBars = 37,
};

__device__ __forceinline__ int blocks_of(int L) { return L > 0 ? (L + kBlockTokens - 1) / kBlockTokens : 0; }

// Walks the chunks of one scheduler part: (request b, blocks [c0, c1), split index).
struct ChunkWalk {
  int b, blk, split, end_b, end_blk;
  __device__ ChunkWalk(const DecodeParams& p, int part) {
    const int32_t* md = p.tile_md + part * kMdInts;
    b = md[0];
    blk = md[1];
    end_b = md[2];
    end_blk = md[3];
    split = md[4];
  }
  __device__ bool next(const DecodeParams& p, int& cb, int& c0, int& c1, int& csplit) {
    while (b < end_b || (b == end_b && blk < end_blk)) {
      // token-sparse: every query position is a request of topk listed positions
      const int n = blocks_of(p.topk > 0 ? p.topk : p.cache_seqlens[b]);
      const int stop = (b == end_b) ? end_blk : n;
      cb = b;
      c0 = blk;
      c1 = stop;
      csplit = split;
      ++b;
      blk = 0;
      if (b <= p.batch) split = p.num_splits[b];
      if (stop > c0) return true;
    }
    return false;
  }
};

// The fixed fill / consume order of one chunk of n steps: K(0) .. K(kLook), then V(t),
// K(t + kLook + 1) for t = 0 .. n-1.  Entry e of the order is (is_v, step).
__device__ __forceinline__ int order_len(int n) { return 2 * n; }
__device__ __forceinline__ void order_at(int e, int n, bool& is_v, int& step) {
  const int head = min(kLook + 1, n);
  if (e < head) {
    is_v = false;
    step = e;
    return;
  }
  const int r = e - head;           // alternating V(t), K(t + kLook + 1) while K steps remain
  const int tail_k = n - head;      // K steps after the head
  if (r < 2 * tail_k) {
    is_v = (r & 1) == 0;
    step = is_v ? (r >> 1) : (r >> 1) + head;
  } else {
    is_v = true;
    step = tail_k + (r - 2 * tail_k);
  }
}
// Slot fills of the chunk that precede V(t) slot 0 (each K step is 5 slots, each V step 4).
__device__ __forceinline__ uint32_t slots_before_v(int t, int n) {
  return 5u * static_cast<uint32_t>(min(t + kLook + 1, n)) + 4u * static_cast<uint32_t>(t);
}

// Drain wait used only after an abort: bounded, does not look at the abort flag.
__device__ __forceinline__ void mbar_wait_drain(uint32_t bar, uint32_t parity) {
  const long long t0 = clock64();
  while (!mbar_try_wait(bar, parity)) {
    if (clock64() - t0 > kWaitLimitCycles) return;
  }
}

// Every lane polls the barrier itself and the outcome is warp-uniform (false on every lane if
// any gave up).  One polling lane plus a shuffle of the outcome measured slower.
__device__ __forceinline__ bool warp_all_wait(uint32_t bar, uint32_t parity, const WaitCtl& wc) {
  return __all_sync(0xffffffffu, mbar_wait(bar, parity, wc) ? 1 : 0) != 0;
}

// Warp reduce-scatter over the 32 token lanes of N column values.  Afterwards lane l holds
// the warp-wide reduction of column col_of(l, i) in v[i], i < max(1, N / 32).
template <int N, bool MAX>
__device__ __forceinline__ void reduce_scatter(float* v, int lane) {
#pragma unroll
  for (int r = 0; r < 5; ++r) {
    const int o = 16 >> r;
    const int n = N >> r;
    if (n > 1) {
      const bool upper = (lane & o) != 0;
#pragma unroll
      for (int i = 0; i < n / 2; ++i) {
        const float keep = upper ? v[i + n / 2] : v[i];
        const float send = upper ? v[i] : v[i + n / 2];
        const float recv = __shfl_xor_sync(0xffffffffu, send, o);
        v[i] = MAX ? fmaxf(keep, recv) : keep + recv;
      }
    } else {
      const float recv = __shfl_xor_sync(0xffffffffu, v[0], o);
      v[0] = MAX ? fmaxf(v[0], recv) : v[0] + recv;
    }
  }
}

template <int RG>
__device__ __forceinline__ int col_of(int lane, int i) {
  if constexpr (RG == 64) return 2 * lane + i;
  else if constexpr (RG == 32) return lane;
  else return lane >> 1;
}

__device__ __forceinline__ uint32_t e4m3x2_to_bf16x2(uint32_t two_codes, float scale) {
  uint32_t h;
  const unsigned short c = static_cast<unsigned short>(two_codes & 0xFFFFu);
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h) : "h"(c));
  const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&h));
  return pack_bf16x2(f.x * scale, f.y * scale);
}

// Pages of step `st` of a request: page A always exists, page B only if the request has it.
struct StepPages {
  int a, b;
  bool has_b;
};
__device__ __forceinline__ StepPages step_pages(const int32_t* bt, int st, int npages) {
  StepPages sp;
  sp.a = bt[2 * st];
  sp.has_b = 2 * st + 1 < npages;
  sp.b = sp.has_b ? bt[2 * st + 1] : 0;
  return sp;
}

// tm_kv is the bf16 cache (64x64 boxes) or, for FP8, the byte view of the cache with 128-byte
// code boxes; tm_scale (16-byte boxes at byte 512) and tm_rope (128-byte swizzled boxes at byte
// 528) are used by the FP8 path only.
// SPARSE (bf16 cache only): token-sparse decode.  A "request" b of the chunk walk is the query
// position (b / vq, b % vq) with topk listed cache positions; the producer warp copies the
// listed tokens' rows (16-byte cp.async per lane, zeros for empty slots) instead of TMA pages.
// token-sparse: warps 4 and 6-11 gather (warp 4 also loads Q)
constexpr int kGatherWarps = 7;
template <int RG, bool FP8, bool SPARSE>
constexpr int threads_of() { return SPARSE ? 384 : Cfg<RG, FP8>::kThreads; }

template <int RG, bool FP8, bool SPARSE = false>
__global__ void __launch_bounds__(threads_of<RG, FP8, SPARSE>(), 1)
    mla_decode_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_kv,
                      const __grid_constant__ CUtensorMap tm_scale, const __grid_constant__ CUtensorMap tm_rope,
                      const __grid_constant__ CUtensorMap tm_opart, const __grid_constant__ CUtensorMap tm_out,
                      const DecodeParams p) {
  using C = Cfg<RG, FP8>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  const uint32_t sQ = sbase + C::kOffQ;
  const uint32_t sP = sbase + C::kOffP;
  const uint32_t sSlots = sbase + C::kOffSlots;
  const uint32_t sRaw = sbase + C::kOffRaw;
  const uint32_t sScale = sbase + C::kOffScale;
  uint8_t* misc = smem + C::kOffMisc;
  const uint32_t sBars = smem_u32(misc);
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(misc + 512);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(misc + 516);
  float* red = reinterpret_cast<float*>(misc + 1024);       // [4][64]
  float* m_sm = reinterpret_cast<float*>(misc + 2048);      // [64]
  float* alpha_sm = reinterpret_cast<float*>(misc + 2304);  // [64]
  float* inv_sm = reinterpret_cast<float*>(misc + 2560);    // [64]
  int32_t* row_tabs = reinterpret_cast<int32_t*>(misc + 3072);  // SPARSE [7][128]: cache row per token slot
  static_assert(kNumBars * 8 <= 512, "barrier area");
  auto bar = [&](int i) -> uint32_t { return sBars + 8u * static_cast<uint32_t>(i); };

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int part = blockIdx.x;
  const int rg = blockIdx.y;  // row group
  const WaitCtl wc{abort_flag, p.status, kStatusWaitTimeout, p.wait_limit > 0 ? p.wait_limit : kWaitLimitCycles};

  if (threadIdx.x == 0) {
    for (int i = 0; i < kMaxSlots; ++i) {
      mbar_init(bar(kBarSlotFull + i), SPARSE ? 32 * kGatherWarps : 1);  // SPARSE: a cp.async arrival per lane
      mbar_init(bar(kBarSlotEmpty + i), 1);
    }
    for (int i = 0; i < kNumS; ++i) {
      mbar_init(bar(kBarSFull + i), 1);
      mbar_init(bar(kBarSEmpty + i), 4);
      mbar_init(bar(kBarScaleFull + i), 1);
      mbar_init(bar(kBarScaleEmpty + i), 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(bar(kBarPFull + i), 4);
      mbar_init(bar(kBarPEmpty + i), 1);
      mbar_init(bar(kBarRawFull + i), 1);
      mbar_init(bar(kBarRawEmpty + i), 1);
    }
    mbar_init(bar(kBarQFull), 1);
    mbar_init(bar(kBarQEmpty), 1);
    mbar_init(bar(kBarOFull), 1);
    mbar_init(bar(kBarOEmpty), 4);
    mbar_init(bar(kBarDrain), 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 4 && lane == 0) {
    tma_prefetch_desc(&tm_q);
    tma_prefetch_desc(&tm_kv);
    if (FP8) {
      tma_prefetch_desc(&tm_scale);
      tma_prefetch_desc(&tm_rope);
    }
  }
  if (warp == 5) {
    tmem_alloc(smem_u32(tmem_holder), C::kTmemCols);
    tmem_relinquish();
  }
  // Zero the ring once: a page half that is never loaded then holds finite values.
  for (int i = threadIdx.x; i < C::kNumSlots * C::kSlotBytes / 16; i += blockDim.x)
    st_shared_v4(sSlots + 16u * i, 0u, 0u, 0u, 0u);
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;

  pdl_launch_dependents();
  // launched as a programmatic dependent of the tile scheduler: the set-up above overlapped
  // it; its metadata is complete and visible from here on
  pdl_wait_primary();
  // metadata the scheduler could not build: its parts are empty, report it
  if (threadIdx.x == 0 && p.status && p.tile_md[part * kMdInts + 5] != 0) atomicOr(p.status, kStatusBadMetadata);

  if (SPARSE && (warp == 4 || warp >= 6)) {
    // ======================= gather producers (token-sparse) =======================
    // Seven warps fill every slot together (more copies in flight).  Each looks up the 128 listed
    // tokens of a step once per step group into its own row table (physical cache row, -1 for
    // an empty slot); every warp-wide cp.async then copies 16-byte chunks of two (or four) token
    // rows, so each instruction reads a few contiguous row segments, and warp gw issues every
    // seventh of them.  The slot's full barrier counts one arrival per lane of the seven warps,
    // made when that lane's copies landed.
    const int gw = warp == 4 ? 0 : warp - 5;
    int32_t* row_tab = row_tabs + 128 * gw;
    uint32_t g = 0;
    int q_fills = 0;
    bool ok = true;
    const char* kvb = static_cast<const char*>(p.kv);
    ChunkWalk walk(p, part);
    int b, c0, c1, split;
    while (ok && walk.next(p, b, c0, c1, split)) {
      const int breal = b / p.vq;
      // sparse prefill: one contiguous cache of kv_len tokens (no length array, no block table)
      const int L = p.cache_seqlens ? p.cache_seqlens[breal] : p.kv_len;
      const int32_t* bt = p.block_table ? p.block_table + static_cast<long long>(breal) * p.max_blocks : nullptr;
      const int32_t* ind = p.indices + static_cast<long long>(b) * p.topk;
      if (gw == 0) {
        if (lane == 0) {
          ok = mbar_wait(bar(kBarQEmpty), (q_fills & 1) ^ 1, wc);
          if (ok) {
            mbar_arrive_expect_tx(bar(kBarQFull), 9u * C::kQAtomBytes);
            for (int a = 0; a < 9; ++a)
              tma_load_3d(sQ + a * C::kQAtomBytes, &tm_q, 64 * a, rg * RG, b, bar(kBarQFull));
          }
        }
        ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
        if (!ok) break;
        ++q_fills;
      }
      const int n = c1 - c0;
      auto rows_of = [&](int t) {
        __syncwarp();  // the previous group's copies were all issued
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const int r = lane + 32 * k;
          const int pos = (c0 + t) * kBlockTokens + r;
          const int idx = pos < p.topk ? ind[pos] : -1;
          row_tab[r] = (idx >= 0 && idx < L) ? (bt ? bt[idx >> 6] * kPage + (idx & (kPage - 1)) : idx) : -1;
        }
        __syncwarp();
      };
      // natoms 64-dim columns from dims0: a row slice is 16 * natoms chunks of 16 bytes
      auto fill = [&](int dims0, int natoms) -> bool {
        const int s = static_cast<int>(g % C::kNumSlots);
        const uint32_t use = g / C::kNumSlots;
        if (!warp_all_wait(bar(kBarSlotEmpty + s), (use & 1u) ^ 1u, wc)) return false;
        const uint32_t dst = sSlots + static_cast<uint32_t>(s) * C::kSlotBytes;
        const int cpr = 8 * natoms;        // chunks per row slice
        const int rpi = 32 / cpr;          // rows per warp instruction
        const int sub = lane / cpr, c = lane % cpr;
        const uint32_t a = static_cast<uint32_t>(c >> 3), cc = static_cast<uint32_t>(c & 7);
        const char* src0 = kvb + (dims0 + 8 * c) * 2;
        for (int i = gw; i < kBlockTokens / rpi; i += kGatherWarps) {
          const uint32_t r = static_cast<uint32_t>(i * rpi + sub);
          const int row = row_tab[r];
          cp_async_16(dst + a * C::kAtomColBytes + r * 128u + ((cc ^ (r & 7u)) << 4),
                      src0 + (row >= 0 ? static_cast<long long>(row) * (kDqk * 2) : 0), row >= 0 ? 16u : 0u);
        }
        cp_async_arrive_noinc(bar(kBarSlotFull + s));
        ++g;
        return true;
      };
      for (int e = 0; ok && e < order_len(n); ++e) {
        bool is_v;
        int t;
        order_at(e, n, is_v, t);
        rows_of(t);
        for (int ks = 0; ok && ks < 4; ++ks) ok = fill(128 * ks, 2);
        if (ok && !is_v) ok = fill(kDv, 1);
      }
    }
    cp_async_wait_all();  // this lane's copies have landed before the CTA may exit
  } else if (warp == 4) {
    // ================================ TMA producer ================================
    if (lane == 0) {
      const uint64_t pol_stream = policy_evict_first();
      const uint64_t pol_keep = policy_evict_last();
      // dims < 512 are read again (V reload, other row groups): keep them in L2 until then
      const uint64_t pol_v = p.row_groups > 1 ? pol_keep : pol_stream;
      uint32_t g = 0;   // bf16 slot fills issued
      uint32_t gr = 0;  // FP8 raw fills issued
      uint32_t us = 0;  // FP8 scale fills issued
      int last_use[kMaxSlots];
      for (int i = 0; i < kMaxSlots; ++i) last_use[i] = -1;
      int last_raw[2] = {-1, -1}, last_scale[kNumS];
      for (int i = 0; i < kNumS; ++i) last_scale[i] = -1;
      int q_fills = 0;
      bool ok = true;
      ChunkWalk walk(p, part);
      int b, c0, c1, split;
      // one bf16 slot: natoms 64-dim columns starting at dims0, for the step's two pages
      auto fill = [&](int dims0, int natoms, const StepPages& sp, uint64_t pol) -> bool {
        const int s = static_cast<int>(g % C::kNumSlots);
        const uint32_t use = g / C::kNumSlots;
        if (g + 1 == static_cast<uint32_t>(p.withhold_fill1)) {
          // fault injection (tests only): this fill is never issued, so its consumer's bounded
          // wait runs out and the CTA unwinds
          ++g;
          return true;
        }
        if (!mbar_wait(bar(kBarSlotEmpty + s), (use & 1u) ^ 1u, wc)) return false;
        mbar_arrive_expect_tx(bar(kBarSlotFull + s),
                              static_cast<uint32_t>(natoms * (sp.has_b ? 2 : 1) * C::kPageBoxBytes));
        const uint32_t dst = sSlots + static_cast<uint32_t>(s) * C::kSlotBytes;
        for (int a = 0; a < natoms; ++a) {
          tma_load_2d(dst + a * C::kAtomColBytes, &tm_kv, dims0 + 64 * a, sp.a * kPage, bar(kBarSlotFull + s), pol);
          if (sp.has_b)
            tma_load_2d(dst + a * C::kAtomColBytes + C::kPageBoxBytes, &tm_kv, dims0 + 64 * a, sp.b * kPage,
                        bar(kBarSlotFull + s), pol);
        }
        last_use[s] = static_cast<int>(use);
        ++g;
        return true;
      };
      // FP8: one raw column of e4m3 codes (group grp = dims 128grp..128grp+127)
      auto fill_raw = [&](int grp, const StepPages& sp, uint64_t pol) -> bool {
        constexpr uint32_t kRaw = C::kNumRaw > 0 ? C::kNumRaw : 1;
        const int r = static_cast<int>(gr % kRaw);
        const uint32_t use = gr / kRaw;
        if (!mbar_wait(bar(kBarRawEmpty + r), (use & 1u) ^ 1u, wc)) return false;
        mbar_arrive_expect_tx(bar(kBarRawFull + r), (sp.has_b ? 2u : 1u) * 8192u);
        const uint32_t dst = sRaw + static_cast<uint32_t>(r) * C::kRawBytes;
        tma_load_2d(dst, &tm_kv, 128 * grp, sp.a * kPage, bar(kBarRawFull + r), pol);
        if (sp.has_b) tma_load_2d(dst + 8192, &tm_kv, 128 * grp, sp.b * kPage, bar(kBarRawFull + r), pol);
        last_raw[r] = static_cast<int>(use);
        ++gr;
        return true;
      };
      // FP8: the per-token scales of one step
      auto fill_scale = [&](const StepPages& sp) -> bool {
        const int sb = static_cast<int>(us % kNumS);
        const uint32_t use = us / kNumS;
        if (!mbar_wait(bar(kBarScaleEmpty + sb), (use & 1u) ^ 1u, wc)) return false;
        mbar_arrive_expect_tx(bar(kBarScaleFull + sb), (sp.has_b ? 2u : 1u) * 1024u);
        const uint32_t dst = sScale + static_cast<uint32_t>(sb) * C::kScaleBytes;
        tma_load_2d(dst, &tm_scale, kDv, sp.a * kPage, bar(kBarScaleFull + sb), pol_keep);
        if (sp.has_b) tma_load_2d(dst + 1024, &tm_scale, kDv, sp.b * kPage, bar(kBarScaleFull + sb), pol_keep);
        last_scale[sb] = static_cast<int>(use);
        ++us;
        return true;
      };
      while (ok && walk.next(p, b, c0, c1, split)) {
        const int L = p.cache_seqlens[b];
        const int npages = (L + kPage - 1) / kPage;
        const int32_t* bt = p.block_table + static_cast<long long>(b) * p.max_blocks;
        if (!mbar_wait(bar(kBarQEmpty), (q_fills & 1) ^ 1, wc)) break;
        mbar_arrive_expect_tx(bar(kBarQFull), 9u * C::kQAtomBytes);
        for (int a = 0; a < 9; ++a) tma_load_3d(sQ + a * C::kQAtomBytes, &tm_q, 64 * a, rg * RG, b, bar(kBarQFull));
        ++q_fills;
        const int n = c1 - c0;
        for (int e = 0; ok && e < order_len(n); ++e) {
          bool is_v;
          int t;
          order_at(e, n, is_v, t);
          const StepPages sp = step_pages(bt, c0 + t, npages);
          if constexpr (FP8) {
            if (!is_v) ok = fill_scale(sp);
            for (int grp = 0; ok && grp < 4; ++grp) ok = fill_raw(grp, sp, is_v ? pol_v : pol_keep);
          } else {
            for (int ks = 0; ok && ks < 4; ++ks) ok = fill(128 * ks, 2, sp, is_v ? pol_v : pol_keep);
            if (ok && !is_v) ok = fill(kDv, 1, sp, pol_stream);
          }
        }
      }
      if (*abort_flag) {
        // let every copy this warp started land before the CTA may exit
        for (int s = 0; s < C::kNumSlots; ++s)
          if (last_use[s] >= 0) mbar_wait_drain(bar(kBarSlotFull + s), static_cast<uint32_t>(last_use[s]) & 1u);
        for (int r = 0; r < 2; ++r)
          if (last_raw[r] >= 0) mbar_wait_drain(bar(kBarRawFull + r), static_cast<uint32_t>(last_raw[r]) & 1u);
        for (int r = 0; r < kNumS; ++r)
          if (last_scale[r] >= 0)
            mbar_wait_drain(bar(kBarScaleFull + r), static_cast<uint32_t>(last_scale[r]) & 1u);
        if (q_fills > 0) mbar_wait_drain(bar(kBarQFull), static_cast<uint32_t>(q_fills - 1) & 1u);
      }
    }
  } else if (warp == 5) {
    // ================================ MMA issuer ==================================
    // the whole warp runs the issue loop (waits seen by every lane, outcome warp-uniform); each
    // MMA and commit is issued by one elected lane
    {
      uint32_t g = 0;   // slot fills consumed
      uint32_t u = 0;   // steps whose QK was issued (S^T buffers)
      uint32_t up = 0;  // steps whose PV was issued (P buffers)
      int chunk = 0;
      bool ok = true;
      ChunkWalk walk(p, part);
      int b, c0, c1, split;
      auto next_slot = [&](uint32_t& s) -> bool {
        s = g % C::kNumSlots;
        if (!warp_all_wait(bar(kBarSlotFull + s), (g / C::kNumSlots) & 1u, wc)) return false;
        ++g;
        if (SPARSE) fence_proxy_async_smem();  // slots written by cp.async (generic proxy)
        tc_fence_after();
        return true;
      };
      auto do_qk = [&]() -> bool {
        const int sb = static_cast<int>(u % kNumS);
        if (!warp_all_wait(bar(kBarSEmpty + sb), ((u / kNumS) & 1u) ^ 1u, wc)) return false;
        tc_fence_after();
        const uint32_t d = tmem + C::kColS + sb * RG;
        for (int ks = 0; ks < 5; ++ks) {
          uint32_t s;
          if (!next_slot(s)) return false;
          const uint32_t kbase = sSlots + s * C::kSlotBytes;
          const int nk = ks < 4 ? 8 : 4;
          for (int kk = 0; kk < nk; ++kk) {
            const uint32_t a = kbase + (kk >> 2) * C::kAtomColBytes + (kk & 3) * 32;
            const uint32_t bq = sQ + (2 * ks + (kk >> 2)) * C::kQAtomBytes + (kk & 3) * 32;
            umma_bf16_warp(d, smem_desc(a, 16, 1024, kSwizzle128), smem_desc(bq, 16, 1024, kSwizzle128), C::kIdescQK,
                           (ks | kk) != 0 ? 1u : 0u);
          }
          umma_commit_warp(bar(kBarSlotEmpty + s));
        }
        umma_commit_warp(bar(kBarSFull + sb));
        ++u;
        return true;
      };
      auto do_pv = [&](bool first_of_chunk) -> bool {
        const int pb = static_cast<int>(up % C::kNumP);
        if (!warp_all_wait(bar(kBarPFull + pb), (up / C::kNumP) & 1u, wc)) return false;
        if (first_of_chunk && !warp_all_wait(bar(kBarOEmpty), (chunk & 1) ^ 1, wc)) return false;
        tc_fence_after();
        const uint32_t pbase = sP + static_cast<uint32_t>(pb) * C::kPBytes;
        for (int vs = 0; vs < 4; ++vs) {
          uint32_t s;
          if (!next_slot(s)) return false;
          const uint32_t d = tmem + C::kColO + vs * RG;
          const uint32_t vbase = sSlots + s * C::kSlotBytes;
#pragma unroll
          for (int kt = 0; kt < 8; ++kt) {
            const uint64_t adesc = smem_desc(vbase + kt * 2048, C::kAtomColBytes, 1024, kSwizzle128);
            const uint64_t bdesc = smem_desc(pbase + kt * 16 * C::kPRowBytes, 16 * 8 * C::kPRowBytes,
                                             8 * C::kPRowBytes, C::kPLayout);
            umma_bf16_warp(d, adesc, bdesc, C::kIdescPV, (first_of_chunk && kt == 0) ? 0u : 1u);
          }
          umma_commit_warp(bar(kBarSlotEmpty + s));
        }
        umma_commit_warp(bar(kBarPEmpty + pb));
        ++up;
        return true;
      };
      while (ok && walk.next(p, b, c0, c1, split)) {
        const int n = c1 - c0;
        if (!warp_all_wait(bar(kBarQFull), chunk & 1, wc)) break;
        for (int e = 0; ok && e < order_len(n); ++e) {
          bool is_v;
          int t;
          order_at(e, n, is_v, t);
          if (is_v) {
            ok = do_pv(t == 0);
          } else {
            ok = do_qk();
            if (ok && t == n - 1) umma_commit_warp(bar(kBarQEmpty));
          }
        }
        if (!ok) break;
        umma_commit_warp(bar(kBarOFull));
        ++chunk;
      }
      // every MMA this warp issued is complete before TMEM is released
      umma_commit_warp(bar(kBarDrain));
      mbar_wait_drain(bar(kBarDrain), 0);
    }
  } else if (warp < 4) {
    // ============================ softmax + epilogue ==============================
    const int tid = threadIdx.x;  // 0..127: token lane of S^T, dim lane of O^T
    const uint32_t lane_base = static_cast<uint32_t>(warp * 32) << 16;
    const float NEG_INF = -CUDART_INF_F;
    float m_ref = NEG_INF;  // thread c < RG: reference max of row c (log2 units)
    float lsum[C::kNOut];
#pragma unroll
    for (int i = 0; i < C::kNOut; ++i) lsum[i] = 0.f;
    uint32_t u = 0;
    uint32_t gchunk = 0;  // slot fills before the current chunk
    int chunk = 0;
    bool fail = false;
    const int R = p.rows;
    ChunkWalk walk(p, part);
    int b, c0, c1, split;
    while (walk.next(p, b, c0, c1, split)) {
      const int L = !SPARSE ? p.cache_seqlens[b] : (p.cache_seqlens ? p.cache_seqlens[b / p.vq] : p.kv_len);
      const int n = c1 - c0;
      const bool single = (p.num_splits[b + 1] - p.num_splits[b]) == 1;
      const int row0 = rg * RG;
      bool aborted = false;
      for (int t = 0; t < n; ++t) {
        const int t0 = (c0 + t) * kBlockTokens;
        const int j = t0 + tid;
        const int sb = static_cast<int>(u % kNumS);
        bool ok = warp_all_wait(bar(kBarSFull + sb), (u / kNumS) & 1u, wc);
        float x[RG];
        tc_fence_after();
#pragma unroll
        for (int c = 0; c < RG; c += 16) tmem_ld16(tmem + lane_base + C::kColS + sb * RG + c, x + c);
        tmem_wait_ld();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(kBarSEmpty + sb));
        // scale into log2 units and mask: key j is visible to row r iff j < L and, when causal,
        // j <= L - s_q + r / h_q (the query block sits at the end of the cache).  With
        // i0 = j - L + s_q that is r / h_q >= i0, i.e. r >= i0 * h_q, i.e. c >= cmin.
        int cmin = -(1 << 30);
        if constexpr (SPARSE) {
          // token-sparse: slot j of the list is a key iff it names a position in [0, L)
          const int idx = j < p.topk ? p.indices[static_cast<long long>(b) * p.topk + j] : -1;
          if (idx < 0 || idx >= L) cmin = 1 << 30;
        } else {
          if (p.causal) {
            const int i0 = j - L + p.s_q;
            if (i0 > 0) cmin = i0 * p.h_q - row0;
          }
          if (j >= L) cmin = 1 << 30;
        }
#pragma unroll
        for (int c = 0; c < RG; ++c) x[c] = (c >= cmin) ? x[c] * p.scale_log2 : NEG_INF;
        float v[RG];
#pragma unroll
        for (int c = 0; c < RG; ++c) v[c] = x[c];
        reduce_scatter<RG, true>(v, lane);
#pragma unroll
        for (int i = 0; i < C::kNOut; ++i) red[warp * 64 + col_of<RG>(lane, i)] = v[i];
        if (named_bar_any(1, 128, !ok || fail)) { aborted = true; break; }
        bool need = false;
        if (tid < RG) {
          const float bm = fmaxf(fmaxf(red[tid], red[64 + tid]), fmaxf(red[128 + tid], red[192 + tid]));
          float alpha = 1.f;
          float m_new = m_ref;
          if (bm > m_ref + kTau || (m_ref == NEG_INF && bm != NEG_INF)) {
            m_new = bm;
            alpha = (m_ref == NEG_INF) ? 0.f : ex2(m_ref - m_new);
          }
          need = (alpha != 1.f) && (t > 0);
          m_ref = m_new;
          m_sm[tid] = (m_new == NEG_INF) ? 0.f : m_new;
          alpha_sm[tid] = alpha;
        }
        const bool rescale = named_bar_any(1, 128, need);
#pragma unroll
        for (int c = 0; c < RG; c += 4) {
          const float4 m4 = *reinterpret_cast<const float4*>(m_sm + c);
          x[c + 0] = ex2(x[c + 0] - m4.x);
          x[c + 1] = ex2(x[c + 1] - m4.y);
          x[c + 2] = ex2(x[c + 2] - m4.z);
          x[c + 3] = ex2(x[c + 3] - m4.w);
        }
#pragma unroll
        for (int c = 0; c < RG; ++c) v[c] = x[c];
        reduce_scatter<RG, false>(v, lane);
#pragma unroll
        for (int i = 0; i < C::kNOut; ++i) lsum[i] = lsum[i] * alpha_sm[col_of<RG>(lane, i)] + v[i];
        // P^T row of this token (bf16), once PV(u - kNumP) has released the buffer
        const int pb = static_cast<int>(u % C::kNumP);
        if (u >= static_cast<uint32_t>(C::kNumP))
          ok &= warp_all_wait(bar(kBarPEmpty + pb), ((u - C::kNumP) / C::kNumP) & 1u, wc);
        {
          const uint32_t prow = static_cast<uint32_t>(tid) * C::kPRowBytes;
          const uint32_t pbase = sP + static_cast<uint32_t>(pb) * C::kPBytes;
#pragma unroll
          for (int q = 0; q < RG / 8; ++q) {
            uint32_t off = prow + 16u * q;
            off ^= ((off >> 7) & C::kPSwzMask) << 4;
            st_shared_v4(pbase + off, pack_bf16x2(x[8 * q + 0], x[8 * q + 1]), pack_bf16x2(x[8 * q + 2], x[8 * q + 3]),
                         pack_bf16x2(x[8 * q + 4], x[8 * q + 5]), pack_bf16x2(x[8 * q + 6], x[8 * q + 7]));
          }
        }
        if (rescale) {
          // O^T *= alpha per row, after PV(u - 1) has finished
          const uint32_t uq = u - 1;
          ok &= warp_all_wait(bar(kBarPEmpty + uq % C::kNumP), (uq / C::kNumP) & 1u, wc);
          tc_fence_after();
#pragma unroll
          for (int vs = 0; vs < 4; ++vs) {
#pragma unroll
            for (int c = 0; c < RG; c += 16) {
              float o[16];
              const uint32_t ta = tmem + lane_base + C::kColO + vs * RG + c;
              tmem_ld16(ta, o);
              tmem_wait_ld();
#pragma unroll
              for (int e = 0; e < 16; ++e) o[e] *= alpha_sm[c + e];
              tmem_st16(ta, o);
            }
          }
          tmem_wait_st();
        }
        if (!FP8 && !SPARSE && t0 + kBlockTokens > L) {
          // tail step: zero the V rows of tokens past the end (their cache slots may hold NaN,
          // and 0 * NaN would poison O)
          for (int vs = 0; vs < 4; ++vs) {
            const uint32_t gv = gchunk + slots_before_v(t, n) + vs;
            const uint32_t s = gv % C::kNumSlots;
            ok &= warp_all_wait(bar(kBarSlotFull + s), (gv / C::kNumSlots) & 1u, wc);
            if (j >= L) {
              const uint32_t rowaddr = sSlots + s * C::kSlotBytes + static_cast<uint32_t>(tid) * 128u;
#pragma unroll
              for (int a = 0; a < 2; ++a)
#pragma unroll
                for (int q = 0; q < 8; ++q) st_shared_v4(rowaddr + a * C::kAtomColBytes + 16u * q, 0u, 0u, 0u, 0u);
            }
          }
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(kBarPFull + pb));
        fail |= !ok;
        ++u;
      }
      if (aborted) break;
      // ------------------------------- epilogue ---------------------------------
#pragma unroll
      for (int i = 0; i < C::kNOut; ++i) red[warp * 64 + col_of<RG>(lane, i)] = lsum[i];
      if (named_bar_any(1, 128, fail)) break;
      if (tid < RG) {
        const float l = red[tid] + red[64 + tid] + red[128 + tid] + red[192 + tid];
        const int row = row0 + tid;
        const float lse_val = l > 0.f ? (m_ref + log2f(l)) * kLn2 : NEG_INF;
        inv_sm[tid] = l > 0.f ? 1.f / l : 0.f;
        if (row < R) {
          if (single) {
            if (SPARSE)  // query position (b / vq, b % vq), head row
              p.lse[(static_cast<long long>(b / p.vq) * p.h_q + row) * p.vq + b % p.vq] = lse_val;
            else
              p.lse[(static_cast<long long>(b) * p.h_q + row % p.h_q) * p.s_q + row / p.h_q] = lse_val;
          } else {
            p.lse_part[static_cast<long long>(split) * R + row] = lse_val;
          }
        }
        m_ref = NEG_INF;
      }
#pragma unroll
      for (int i = 0; i < C::kNOut; ++i) lsum[i] = 0.f;
      named_bar_sync(1, 128);
      const bool ok = warp_all_wait(bar(kBarOFull), chunk & 1, wc);
      fail |= !ok;
      tc_fence_after();
      {
        // O^T block vs (dims 128 vs + tid), columns = query rows.  Groups of kGR rows go out
        // through the P^T buffers (free once the chunk's last PV has completed): the softmax
        // warps write them as [row][128 dims], then one thread stores the group with a TMA
        // tensor store (rows past the request's end fall outside the map).  Plain stores from
        // these warps were slower.
        constexpr int kGR = (C::kNumP * C::kPBytes / 512) < RG ? (C::kNumP * C::kPBytes / 512) : RG;
        static_assert(kGR == (RG == 16 ? 16 : 32), "output map box rows");
        float* stage_f = reinterpret_cast<float*>(smem + C::kOffP);
        __nv_bfloat16* stage_h = reinterpret_cast<__nv_bfloat16*>(smem + C::kOffP);
        bool first = true;
#pragma unroll 1
        for (int vs = 0; vs < 4; ++vs) {
#pragma unroll 1
          for (int g0 = 0; g0 < RG; g0 += kGR) {
            if (!first) {
              // the previous group's store has read the buffers
              if (tid == 0) bulk_wait_read_all();
              named_bar_sync(1, 128);
            }
            first = false;
#pragma unroll
            for (int c = 0; c < kGR; c += 16) {
              float o[16];
              tmem_ld16(tmem + lane_base + C::kColO + vs * RG + g0 + c, o);
              tmem_wait_ld();
#pragma unroll
              for (int e = 0; e < 16; ++e) {
                const float val = o[e] * inv_sm[g0 + c + e];
                if (single)
                  stage_h[(c + e) * 128 + tid] = __float2bfloat16_rn(val);
                else
                  stage_f[(c + e) * 128 + tid] = val;
              }
            }
            fence_proxy_async_smem();
            named_bar_sync(1, 128);
            if (tid == 0) {
              if (single)
                tma_store_3d(&tm_out, sP, vs * 128, row0 + g0, b);
              else
                tma_store_3d(&tm_opart, sP, vs * 128, row0 + g0, split);
              bulk_commit();
            }
          }
        }
        // the buffers hold P^T again from the next step on
        if (tid == 0) bulk_wait_read_all();
        named_bar_sync(1, 128);
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(kBarOEmpty));
      gchunk += 9u * static_cast<uint32_t>(n);
      ++chunk;
    }
  }

  if constexpr (FP8) {
    if (warp >= 6) {
      // ============================ FP8 dequant warpgroup ==========================
      // Produces the bf16 slots in the order the MMA consumes them (see the file header); slot 4
      // of K(t) is the RoPE part, copied by TMA.
      const int dq = threadIdx.x - 192;             // dequant thread
      const int dt = dq & 127;                       // token lane within a step
      constexpr int kHalves = C::kDequantWarps / 4;  // threads per token, each on its own atom columns
      constexpr int kChunks = 8 / kHalves;           // 16-code chunks per thread and slot
      const int dh = dq >> 7;                        // this thread's share of the token's 128 dims
      const uint64_t pol_rope = p.row_groups > 1 ? policy_evict_last() : policy_evict_first();
      uint32_t gs = 0, gr = 0, us = 0;
      int last_rope[kMaxSlots];
      for (int i = 0; i < kMaxSlots; ++i) last_rope[i] = -1;
      bool ok = true, aborted = false;
      ChunkWalk walk(p, part);
      int b, c0, c1, split;
      // code * scale -> bf16 for 128 dims of this thread's token (zeros past the end)
      auto dequant_slot = [&](int grp, uint32_t sbuf, int t0, int L) -> bool {
        const uint32_t s = gs % C::kNumSlots;
        const uint32_t r = gr % C::kNumRaw;
        ok &= warp_all_wait(bar(kBarRawFull + r), (gr / C::kNumRaw) & 1u, wc);
        ok &= warp_all_wait(bar(kBarSlotEmpty + s), ((gs / C::kNumSlots) & 1u) ^ 1u, wc);
        const uint32_t dst = sSlots + s * C::kSlotBytes + static_cast<uint32_t>(dt) * 128u;
        const uint32_t swz = static_cast<uint32_t>(dt & 7);
        if (t0 + dt < L) {
          float scale;
          asm volatile("ld.shared.f32 %0, [%1];" : "=f"(scale)
                       : "r"(sScale + sbuf * C::kScaleBytes + static_cast<uint32_t>(dt) * 16u + 4u * grp));
          const uint32_t src = sRaw + r * C::kRawBytes + static_cast<uint32_t>(dt) * 128u;
#pragma unroll
          for (int c = 0; c < kChunks; ++c) {
            const uint32_t cc = static_cast<uint32_t>(dh * kChunks + ((c + dt) & (kChunks - 1)));
            uint32_t w0, w1, w2, w3;
            asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
                         : "=r"(w0), "=r"(w1), "=r"(w2), "=r"(w3) : "r"(src + 16u * cc));
            const uint32_t oc = 2u * cc;  // 16 codes -> output chunks oc, oc + 1 (8 dims each)
            const uint32_t base = dst + (oc >> 3) * C::kAtomColBytes;
            st_shared_v4(base + ((((oc & 7u) ^ swz)) << 4), e4m3x2_to_bf16x2(w0, scale),
                         e4m3x2_to_bf16x2(w0 >> 16, scale), e4m3x2_to_bf16x2(w1, scale),
                         e4m3x2_to_bf16x2(w1 >> 16, scale));
            st_shared_v4(base + ((((oc + 1u) & 7u) ^ swz) << 4), e4m3x2_to_bf16x2(w2, scale),
                         e4m3x2_to_bf16x2(w2 >> 16, scale), e4m3x2_to_bf16x2(w3, scale),
                         e4m3x2_to_bf16x2(w3 >> 16, scale));
          }
        } else {
#pragma unroll
          for (int a = 0; a < 2 / kHalves; ++a)
#pragma unroll
            for (int q = 0; q < 8; ++q)
              st_shared_v4(dst + (dh * (2 / kHalves) + a) * C::kAtomColBytes + 16u * q, 0u, 0u, 0u, 0u);
        }
        fence_proxy_async_smem();
        if (named_bar_any(2, 32 * C::kDequantWarps, !ok)) return false;
        if (dq == 0) {
          mbar_arrive(bar(kBarSlotFull + s));
          mbar_arrive(bar(kBarRawEmpty + r));
        }
        ++gs;
        ++gr;
        return true;
      };
      auto rope_slot = [&](const StepPages& sp) {
        const uint32_t s = gs % C::kNumSlots;
        const uint32_t use = gs / C::kNumSlots;
        if (dq == 0 && ok) {
          ok = mbar_wait(bar(kBarSlotEmpty + s), (use & 1u) ^ 1u, wc);
          if (ok) {
            mbar_arrive_expect_tx(bar(kBarSlotFull + s), (sp.has_b ? 2u : 1u) * C::kPageBoxBytes);
            const uint32_t dst = sSlots + s * C::kSlotBytes;
            tma_load_2d(dst, &tm_rope, kDv + 16, sp.a * kPage, bar(kBarSlotFull + s), pol_rope);
            if (sp.has_b)
              tma_load_2d(dst + C::kPageBoxBytes, &tm_rope, kDv + 16, sp.b * kPage, bar(kBarSlotFull + s), pol_rope);
            last_rope[s] = static_cast<int>(use);
          }
        }
        ++gs;
      };
      while (!aborted && walk.next(p, b, c0, c1, split)) {
        const int L = p.cache_seqlens[b];
        const int npages = (L + kPage - 1) / kPage;
        const int32_t* bt = p.block_table + static_cast<long long>(b) * p.max_blocks;
        const int n = c1 - c0;
        const uint32_t us0 = us;  // scale fill index of step 0 of this chunk
        for (int e = 0; !aborted && e < order_len(n); ++e) {
          bool is_v;
          int t;
          order_at(e, n, is_v, t);
          const int t0 = (c0 + t) * kBlockTokens;
          const uint32_t su = us0 + static_cast<uint32_t>(t);  // scale fill of step t
          if (!is_v) {
            ok &= warp_all_wait(bar(kBarScaleFull + su % kNumS), (su / kNumS) & 1u, wc);
            ++us;
          }
          for (int grp = 0; grp < 4 && !aborted; ++grp) aborted = !dequant_slot(grp, su % kNumS, t0, L);
          if (aborted) break;
          if (!is_v) {
            rope_slot(step_pages(bt, c0 + t, npages));
          } else if (dq == 0) {
            mbar_arrive(bar(kBarScaleEmpty + su % kNumS));  // the last use of step t's scales
          }
        }
      }
      if (dq == 0 && *abort_flag)
        for (int s = 0; s < C::kNumSlots; ++s)
          if (last_rope[s] >= 0) mbar_wait_drain(bar(kBarSlotFull + s), static_cast<uint32_t>(last_rope[s]) & 1u);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 5) {
    tc_fence_after();
    tmem_dealloc(tmem, C::kTmemCols);
  }
}

template <int RG, bool FP8, bool SPARSE = false>
int launch_impl(const CUtensorMap& tm_q, const CUtensorMap& tm_kv, const CUtensorMap& tm_scale,
                const CUtensorMap& tm_rope, const OutMaps& om, const DecodeParams& p, cudaStream_t stream) {
  using C = Cfg<RG, FP8>;
  auto kern = mla_decode_kernel<RG, FP8, SPARSE>;
  constexpr int kThreads = threads_of<RG, FP8, SPARSE>();
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemBytes);
  if (e != cudaSuccess) return static_cast<int>(e);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(p.num_sm_parts, p.row_groups, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = C::kSmemBytes;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;  // overlaps the scheduler's tail
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  e = cudaLaunchKernelEx(&cfg, kern, tm_q, tm_kv, tm_scale, tm_rope, om.o_part, om.out, p);
  return static_cast<int>(e);
}

}  // namespace

// bf16 cache, up to 64 query rows (16-, 32- or 64-row tiles)
int launch_decode_bf16(const CUtensorMap& tm_q, const CUtensorMap& tm_kv, const OutMaps& om, const DecodeParams& p,
                       int rows_per_cta, cudaStream_t stream) {
  switch (rows_per_cta) {
    case 16: return launch_impl<16, false>(tm_q, tm_kv, tm_kv, tm_kv, om, p, stream);
    case 32: return launch_impl<32, false>(tm_q, tm_kv, tm_kv, tm_kv, om, p, stream);
    case 64: return launch_impl<64, false>(tm_q, tm_kv, tm_kv, tm_kv, om, p, stream);
    default: return static_cast<int>(cudaErrorInvalidValue);
  }
}

int launch_decode_sparse_bf16(const CUtensorMap& tm_q, const OutMaps& om, const DecodeParams& p, int rows_per_cta,
                              cudaStream_t stream) {
  switch (rows_per_cta) {
    case 16: return launch_impl<16, false, true>(tm_q, tm_q, tm_q, tm_q, om, p, stream);
    case 32: return launch_impl<32, false, true>(tm_q, tm_q, tm_q, tm_q, om, p, stream);
    case 64: return launch_impl<64, false, true>(tm_q, tm_q, tm_q, tm_q, om, p, stream);
    default: return static_cast<int>(cudaErrorInvalidValue);
  }
}

int launch_decode_fp8(const CUtensorMap& tm_q, const CUtensorMap& tm_codes, const CUtensorMap& tm_scale,
                      const CUtensorMap& tm_rope, const OutMaps& om, const DecodeParams& p, int rows_per_cta,
                      cudaStream_t stream) {
  switch (rows_per_cta) {
    case 16: return launch_impl<16, true>(tm_q, tm_codes, tm_scale, tm_rope, om, p, stream);
    case 32: return launch_impl<32, true>(tm_q, tm_codes, tm_scale, tm_rope, om, p, stream);
    case 64: return launch_impl<64, true>(tm_q, tm_codes, tm_scale, tm_rope, om, p, stream);
    default: return static_cast<int>(cudaErrorInvalidValue);
  }
}

}  // namespace mla

// Split-KV MLA decode for up to 32 query rows per request (the memory-bound shapes: h_q 16 with
// s_q 1 or 2) on a cluster of two CTAs that split the cached dims between them.
//
// Problem as in mla_decode.cu (FlashMLA pages: mha_fwd_kvcache_mla in the "flash_api.cpp"
// excerpt, mmssai.com page; 64-token pages through block_table, kdjingpai.com page; V is the
// first 512 of the 576 cached dims).  With so few query rows the work is bound by HBM, and
// what limits a single CTA is how many bytes of KV it can keep in flight: QK^T needs all 576
// dims of a 128-token step (147 KB), PV needs its first 512 again after the softmax, and
// 227 KB of shared memory cannot hold a step for that long while the next ones stream in (the
// single-CTA kernel re-reads V from L2 instead, which doubles its shared-memory fills).
//
// Here the two CTAs of a cluster (two SMs) share every 128-token step: CTA c holds the latent
// dims 256c .. 256c+255 and the RoPE dims 512+32c .. 512+32c+31 of the step's tokens (72 KB),
// computes the partial scores S_c^T[128 tokens x RG rows] = K_c . Q_c^T over its 288 dims on
// its own tensor core, and sends them to the peer with st.async (8 KB per step for 16 rows).
// Each CTA adds the two partials in the same order (the sums are bit-identical in both), runs
// the same online softmax, and accumulates its own half of the output,
//   O_c^T[256 dims x RG] += V_c^T[256 x 128 tokens] . P^T,
// from the K slots it already holds: V is never loaded twice, so a step's 72 KB stays
// resident from its fill through QK^T, the exchange, the softmax and PV, and the ring of five
// 32 KB slots keeps 2.5 steps in flight per SM.  A cluster walks two adjacent scheduler parts
// one after the other, so num_sm_parts keeps its one-SM-per-part meaning.
//
// Roles per CTA: warps 0-3 softmax + epilogue (thread = token lane of S^T, then dim lane of
// O^T), warp 4 TMA producer, warp 5 MMA issuer and TMEM owner (both run converged on the whole
// warp, one elected lane issuing each copy, MMA and commit).  Issue order per chunk of n
// steps: QK(0), QK(1), PV(0), QK(2), PV(1), ..., PV(n-1) (two S^T buffers in TMEM).  MMAs are
// cta_group::1 (each CTA's tensor core works on its own dims); the only cross-CTA traffic is
// the score exchange and, on a time-out, the abort flag.
#include <cuda_bf16.h>
#include <math_constants.h>

#include "mla_internal.h"
#include "mla_ptx.cuh"

namespace mla {

namespace {

constexpr float kTau = 8.0f;  // lazy-rescale threshold, log2 units (P <= 2^8)
constexpr float kLn2 = 0.69314718055994530942f;
constexpr int kNumS = 2;       // S^T buffers in TMEM (QK runs one step ahead of PV)
constexpr int kNumX = 2;       // buffers for the peer's partial scores
constexpr int kNumP = 2;       // P^T buffers
constexpr int kRopeSlots = 3;  // ring of RoPE half slots (released right after QK)
constexpr int kThreads = 192;
constexpr int kSlotBytes = 32768;      // 128 tokens x 128 dims: two 64-dim swizzle atoms
constexpr int kAtomBytes = 16384;      // 128 tokens x 64 dims (128-byte rows)
constexpr int kBoxBytes = 8192;        // one page (64 tokens) x 64 dims: one TMA box
constexpr int kRopeSlotBytes = 8192;   // 128 tokens x 32 dims (64-byte rows, 64-byte swizzle)
constexpr int kRopeBoxBytes = 4096;    // one page x 32 dims
constexpr int kDimsPerCta = 256;       // latent dims per CTA (V and the NoPE part of K)
constexpr int kRopePerCta = 32;        // RoPE dims per CTA

template <int RG>
struct DsCfg {
  static_assert(RG == 16 || RG == 32, "rows per cluster");
  static constexpr int kNumSlots = RG == 16 ? 5 : 4;
  static constexpr int kQAtomBytes = RG * 128;  // RG rows x 64 dims
  static constexpr int kQRopeBytes = RG * 64;   // RG rows x 32 dims
  static constexpr int kQBytes = (4 * kQAtomBytes + kQRopeBytes + 1023) / 1024 * 1024;
  static constexpr int kPRowBytes = RG * 2;     // one token row of P^T
  static constexpr int kPBytes = 128 * kPRowBytes;
  static constexpr int kXBytes = 128 * RG * 4;  // fp32 partial S^T [token][row]
  static constexpr int kOffQ = 0;
  static constexpr int kOffP = kOffQ + kQBytes;
  static constexpr int kOffX = kOffP + kNumP * kPBytes;
  static constexpr int kOffSlots = kOffX + kNumX * kXBytes;
  static constexpr int kOffRope = kOffSlots + kNumSlots * kSlotBytes;
  static constexpr int kOffMisc = kOffRope + kRopeSlots * kRopeSlotBytes;
  static constexpr int kMiscBytes = 4096;
  static constexpr int kSmemBytes = kOffMisc + kMiscBytes + 1024;  // + alignment slack
  static constexpr uint32_t kPSwzMask = RG / 8 - 1;
  static constexpr uint32_t kPLayout = RG == 32 ? kSwizzle64 : kSwizzle32;
  static constexpr uint32_t kIdescQK = idesc_bf16(128, RG, false, false);
  static constexpr uint32_t kIdescPV = idesc_bf16(128, RG, true, true);
  static constexpr int kColO = 0;       // 2 blocks of RG columns: O^T dims 128j..128j+127 of this CTA's 256
  static constexpr int kColS = 2 * RG;  // kNumS buffers of RG columns: partial S^T
  static constexpr int kTmemCols = RG == 16 ? 64 : 128;
  static constexpr int kXChunks = RG / 4;  // 16-byte chunks of one token's partial scores
  static_assert(kSmemBytes <= 232448, "shared memory budget");
  static_assert(kOffSlots % 1024 == 0 && kOffRope % 1024 == 0, "swizzle atoms need 1024-byte alignment");
  static_assert((4 * kQAtomBytes) % 512 == 0 && kOffP % 512 == 0, "64-byte swizzle needs 512-byte alignment");
  static_assert(kColS + kNumS * RG <= kTmemCols, "TMEM budget");
  static_assert(kNumP * kPBytes == 512 * RG, "the epilogue stages RG rows x 128 fp32 dims in the P^T buffers");
};

// barrier indices in the misc area
enum : int {
  kBarSlotFull = 0,                     // [5]
  kBarSlotEmpty = kBarSlotFull + 5,     // [5]
  kBarRopeFull = kBarSlotEmpty + 5,     // [kRopeSlots]
  kBarRopeEmpty = kBarRopeFull + kRopeSlots,
  kBarSFull = kBarRopeEmpty + kRopeSlots,  // [kNumS]
  kBarSEmpty = kBarSFull + kNumS,
  kBarXFull = kBarSEmpty + kNumS,       // [kNumX] the peer's partial scores landed (st.async bytes)
  kBarPFull = kBarXFull + kNumX,        // [kNumP]
  kBarPEmpty = kBarPFull + kNumP,
  kBarQFull = kBarPEmpty + kNumP,
  kBarQEmpty,
  kBarOFull,
  kBarOEmpty,
  kBarDrain,
  kNumBars,
};
constexpr int kMiscHolder = 512;    // TMEM base address
constexpr int kMiscAbort = 516;     // abort flag (set by this CTA or its peer)
constexpr int kMiscPeerSent = 520;  // partials the peer sent (written by the peer before exit)
constexpr int kMiscRed = 1024;      // float [4 warps][32 rows]
constexpr int kMiscM = 1536;        // float [32]
constexpr int kMiscAlpha = 1664;    // float [32]
constexpr int kMiscInv = 1792;      // float [32]
static_assert(kNumBars * 8 <= kMiscHolder, "barrier area");

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
      const int n = blocks_of(p.cache_seqlens[b]);
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

// The chunks of the cluster's two scheduler parts (2c, then 2c + 1 when it exists).
struct DualWalk {
  ChunkWalk w0, w1;
  bool second, has_second;
  __device__ DualWalk(const DecodeParams& p, int part0, bool has1)
      : w0(p, part0), w1(p, has1 ? part0 + 1 : part0), second(false), has_second(has1) {}
  __device__ bool next(const DecodeParams& p, int& b, int& c0, int& c1, int& split) {
    if (!second) {
      if (w0.next(p, b, c0, c1, split)) return true;
      second = true;
      if (!has_second) return false;
    }
    return has_second && w1.next(p, b, c0, c1, split);
  }
};

// The fixed consume order of one chunk of n steps: QK(0), QK(1), then PV(t), QK(t + 2) for
// t = 0 .. n - 1.  Entry e is (is_pv, step).
__device__ __forceinline__ void order_at(int e, int n, bool& is_pv, int& step) {
  const int head = min(2, n);
  if (e < head) {
    is_pv = false;
    step = e;
    return;
  }
  const int r = e - head;
  const int tail_qk = n - head;
  if (r < 2 * tail_qk) {
    is_pv = (r & 1) == 0;
    step = is_pv ? (r >> 1) : (r >> 1) + head;
  } else {
    is_pv = true;
    step = tail_qk + (r - 2 * tail_qk);
  }
}

// Bounded waits.  On time-out: status bit, this CTA's and the peer's abort flags; every waiter
// of both CTAs then unwinds.
struct DsCtl {
  volatile int* abort_flag;
  uint32_t peer_abort;  // cluster address of the peer's abort flag
  int* status;
  long long limit;
};

static __device__ __noinline__ void ds_timeout(const DsCtl& c) {
  *c.abort_flag = 1;
  st_cluster_u32(c.peer_abort, 1u);
  if (c.status) atomicOr(c.status, kStatusWaitTimeout);
  __threadfence();
}

__device__ __forceinline__ bool dwait(uint32_t bar, uint32_t parity, const DsCtl& c) {
  if (mbar_try_wait(bar, parity)) return true;
  const long long t0 = clock64();
  while (true) {
    if (mbar_try_wait(bar, parity)) return true;
    if (*c.abort_flag) return false;
    if (clock64() - t0 > c.limit) {
      ds_timeout(c);
      return false;
    }
  }
}

// used only at exit: bounded, ignores the abort flag
__device__ __forceinline__ void drain_wait(uint32_t bar, uint32_t parity) {
  const long long t0 = clock64();
  while (!mbar_try_wait(bar, parity)) {
    if (clock64() - t0 > kWaitLimitCycles) return;
  }
}

// Every lane polls the barrier itself (it then reads what the phase guards); the outcome is
// warp-uniform.  One polling lane plus a shuffle of the outcome measured slower.
__device__ __forceinline__ bool warp_all_dwait(uint32_t bar, uint32_t parity, const DsCtl& c) {
  return __all_sync(0xffffffffu, dwait(bar, parity, c) ? 1 : 0) != 0;
}

// Warp reduce-scatter over the 32 token lanes of N column values; afterwards lane l holds the
// warp-wide reduction of column col_of(l) in v[0].
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
__device__ __forceinline__ int col_of(int lane) {
  if constexpr (RG == 32) return lane;
  else return lane >> 1;
}

// Position of 16-byte chunk k of token row i's partial scores (rows of RG floats): rotated so
// that the 32 lanes of a warp, one row each, touch distinct banks.
template <int RG>
__device__ __forceinline__ uint32_t xchunk(int i, int k) {
  constexpr int n = RG / 4;
  return static_cast<uint32_t>((k + (RG == 16 ? (i >> 1) : i)) & (n - 1));
}

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

template <int RG>
__global__ void __launch_bounds__(kThreads, 1)
    mla_decode_dsplit_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_q_rope,
                             const __grid_constant__ CUtensorMap tm_kv,
                             const __grid_constant__ CUtensorMap tm_kv_rope,
                             const __grid_constant__ CUtensorMap tm_opart, const __grid_constant__ CUtensorMap tm_out,
                             const DecodeParams p) {
  using C = DsCfg<RG>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  const uint32_t sQ = sbase + C::kOffQ;
  const uint32_t sP = sbase + C::kOffP;
  const uint32_t sX = sbase + C::kOffX;
  const uint32_t sSlots = sbase + C::kOffSlots;
  const uint32_t sRope = sbase + C::kOffRope;
  uint8_t* misc = smem + C::kOffMisc;
  const uint32_t sMisc = smem_u32(misc);
  const uint32_t sBars = sMisc;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(misc + kMiscHolder);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(misc + kMiscAbort);
  float* red = reinterpret_cast<float*>(misc + kMiscRed);
  float* m_sm = reinterpret_cast<float*>(misc + kMiscM);
  float* alpha_sm = reinterpret_cast<float*>(misc + kMiscAlpha);
  float* inv_sm = reinterpret_cast<float*>(misc + kMiscInv);
  auto bar = [&](int i) -> uint32_t { return sBars + 8u * static_cast<uint32_t>(i); };

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_cta_rank();
  const uint32_t peer = rank ^ 1u;
  const int part0 = 2 * static_cast<int>(blockIdx.x >> 1);
  const bool has1 = part0 + 1 < p.num_sm_parts;
  auto other = [&](uint32_t a) -> uint32_t { return map_to_cta(a, peer); };
  const DsCtl wc{abort_flag, other(sMisc + kMiscAbort), p.status, p.wait_limit > 0 ? p.wait_limit : kWaitLimitCycles};

  if (threadIdx.x == 0) {
    for (int i = 0; i < C::kNumSlots; ++i) {
      mbar_init(bar(kBarSlotFull + i), 1);
      mbar_init(bar(kBarSlotEmpty + i), 1);
    }
    for (int i = 0; i < kRopeSlots; ++i) {
      mbar_init(bar(kBarRopeFull + i), 1);
      mbar_init(bar(kBarRopeEmpty + i), 1);
    }
    for (int i = 0; i < kNumS; ++i) {
      mbar_init(bar(kBarSFull + i), 1);
      mbar_init(bar(kBarSEmpty + i), 4);
    }
    for (int i = 0; i < kNumX; ++i) mbar_init(bar(kBarXFull + i), 1);
    for (int i = 0; i < kNumP; ++i) {
      mbar_init(bar(kBarPFull + i), 4);
      mbar_init(bar(kBarPEmpty + i), 1);
    }
    mbar_init(bar(kBarQFull), 1);
    mbar_init(bar(kBarQEmpty), 1);
    mbar_init(bar(kBarOFull), 1);
    mbar_init(bar(kBarOEmpty), 4);
    mbar_init(bar(kBarDrain), 1);
    *abort_flag = 0;
    *reinterpret_cast<volatile uint32_t*>(misc + kMiscPeerSent) = 0;
    fence_barrier_init();
  }
  if (warp == 4 && lane == 0) {
    tma_prefetch_desc(&tm_q);
    tma_prefetch_desc(&tm_q_rope);
    tma_prefetch_desc(&tm_kv);
    tma_prefetch_desc(&tm_kv_rope);
  }
  if (warp == 5) {
    tmem_alloc(smem_u32(tmem_holder), C::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();  // both CTAs' barriers initialised before any remote store or arrive
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;

  pdl_launch_dependents();
  // launched as a programmatic dependent of the tile scheduler: the set-up above overlapped
  // it; its metadata is complete and visible from here on
  pdl_wait_primary();
  // metadata the scheduler could not build: its parts are empty, report it
  if (threadIdx.x == 0 && p.status &&
      (p.tile_md[part0 * kMdInts + 5] != 0 || (has1 && p.tile_md[(part0 + 1) * kMdInts + 5] != 0)))
    atomicOr(p.status, kStatusBadMetadata);

  uint32_t x_exp = 0;   // softmax thread 0: phases whose expected bytes it registered
  uint32_t x_sent = 0;  // softmax thread 0: partials sent to the peer
  uint32_t x_seen = 0;  // softmax thread 0: phases of the peer's partials observed complete

  if (warp == 4) {
    // ================================ TMA producer ================================
    // the whole warp runs the fill loop; one elected lane issues each copy and arrive
    {
      const uint64_t pol = policy_evict_first();  // every byte of the cache is read once
      uint32_t g = 0;   // slot fills issued
      uint32_t gr = 0;  // RoPE half-slot fills issued
      int last_use[5] = {-1, -1, -1, -1, -1};
      int last_rope[kRopeSlots] = {-1, -1, -1};
      int q_fills = 0;
      bool ok = true;
      DualWalk walk(p, part0, has1);
      int b, c0, c1, split;
      const int d0 = kDimsPerCta * static_cast<int>(rank);
      const int dr = kDv + kRopePerCta * static_cast<int>(rank);
      while (ok && walk.next(p, b, c0, c1, split)) {
        const int L = p.cache_seqlens[b];
        const int npages = (L + kPage - 1) / kPage;
        const int32_t* bt = p.block_table + static_cast<long long>(b) * p.max_blocks;
        if (!warp_all_dwait(bar(kBarQEmpty), (q_fills & 1) ^ 1, wc)) break;
        if (elect_one()) {
          mbar_arrive_expect_tx(bar(kBarQFull), 4u * C::kQAtomBytes + C::kQRopeBytes);
          for (int a = 0; a < 4; ++a) tma_load_3d(sQ + a * C::kQAtomBytes, &tm_q, d0 + 64 * a, 0, b, bar(kBarQFull));
          tma_load_3d(sQ + 4 * C::kQAtomBytes, &tm_q_rope, dr, 0, b, bar(kBarQFull));
        }
        ++q_fills;
        for (int t = 0; ok && t < c1 - c0; ++t) {
          const StepPages sp = step_pages(bt, c0 + t, npages);
          const uint32_t npg = sp.has_b ? 2u : 1u;
          {
            // this CTA's 32 RoPE dims of the step's tokens (QK^T only)
            const int r = static_cast<int>(gr % kRopeSlots);
            const uint32_t use = gr / kRopeSlots;
            if (!warp_all_dwait(bar(kBarRopeEmpty + r), (use & 1u) ^ 1u, wc)) { ok = false; break; }
            const uint32_t dst = sRope + static_cast<uint32_t>(r) * kRopeSlotBytes;
            if (elect_one()) {
              mbar_arrive_expect_tx(bar(kBarRopeFull + r), npg * kRopeBoxBytes);
              tma_load_2d(dst, &tm_kv_rope, dr, sp.a * kPage, bar(kBarRopeFull + r), pol);
              if (sp.has_b) tma_load_2d(dst + kRopeBoxBytes, &tm_kv_rope, dr, sp.b * kPage, bar(kBarRopeFull + r), pol);
            }
            last_rope[r] = static_cast<int>(use);
            ++gr;
          }
          for (int k = 0; ok && k < 2; ++k) {
            // slot k: this CTA's dims d0 + 128k .. d0 + 128k + 127 (two 64-dim atoms, two pages)
            const int s = static_cast<int>(g % C::kNumSlots);
            const uint32_t use = g / C::kNumSlots;
            if (rank == 0 && g + 1 == static_cast<uint32_t>(p.withhold_fill1)) {
              // fault injection (tests only): CTA 0 never issues this fill, so its MMA thread's
              // bounded wait runs out and both CTAs of the cluster unwind
              ++g;
              continue;
            }
            if (!warp_all_dwait(bar(kBarSlotEmpty + s), (use & 1u) ^ 1u, wc)) { ok = false; break; }
            const uint32_t dst = sSlots + static_cast<uint32_t>(s) * kSlotBytes;
            if (elect_one()) {
              mbar_arrive_expect_tx(bar(kBarSlotFull + s), 2u * npg * kBoxBytes);
              for (int a = 0; a < 2; ++a) {
                const int x = d0 + 128 * k + 64 * a;
                tma_load_2d(dst + a * kAtomBytes, &tm_kv, x, sp.a * kPage, bar(kBarSlotFull + s), pol);
                if (sp.has_b) tma_load_2d(dst + a * kAtomBytes + kBoxBytes, &tm_kv, x, sp.b * kPage, bar(kBarSlotFull + s), pol);
              }
            }
            last_use[s] = static_cast<int>(use);
            ++g;
          }
        }
      }
      if (*abort_flag) {
        // let every copy this warp started land before the CTA may exit
        for (int s = 0; s < C::kNumSlots; ++s)
          if (last_use[s] >= 0) drain_wait(bar(kBarSlotFull + s), static_cast<uint32_t>(last_use[s]) & 1u);
        for (int r = 0; r < kRopeSlots; ++r)
          if (last_rope[r] >= 0) drain_wait(bar(kBarRopeFull + r), static_cast<uint32_t>(last_rope[r]) & 1u);
        if (q_fills > 0) drain_wait(bar(kBarQFull), static_cast<uint32_t>(q_fills - 1) & 1u);
      }
    }
  } else if (warp == 5) {
    // ================================ MMA issuer ==================================
    // the whole warp runs the issue loop; every wait is observed by all lanes and its outcome made
    // warp-uniform, each MMA and commit is issued by one elected lane
    {
      uint32_t g = 0;   // slot fills consumed by QK
      uint32_t gr = 0;  // RoPE fills consumed
      uint32_t u = 0;   // steps whose QK was issued
      uint32_t up = 0;  // steps whose PV was issued
      uint32_t gchunk = 0;
      int chunk = 0;
      bool ok = true;
      DualWalk walk(p, part0, has1);
      int b, c0, c1, split;
      // shared-memory descriptors of the operands' first bytes; an operand at byte offset o from
      // there is the descriptor plus o >> 4 (the 14-bit start-address field, 16-byte units)
      const uint64_t kdesc0 = smem_desc(sSlots, 16, 1024, kSwizzle128);
      const uint64_t vdesc0 = smem_desc(sSlots, kAtomBytes, 1024, kSwizzle128);
      const uint64_t qdesc0 = smem_desc(sQ, 16, 1024, kSwizzle128);
      const uint64_t rdesc0 = smem_desc(sRope, 16, 512, kSwizzle64);
      const uint64_t qrdesc0 = smem_desc(sQ + 4 * C::kQAtomBytes, 16, 512, kSwizzle64);
      const uint64_t pdesc0 = smem_desc(sP, 16 * 8 * C::kPRowBytes, 8 * C::kPRowBytes, C::kPLayout);
      auto adv = [](uint64_t d, uint32_t bytes) -> uint64_t { return d + static_cast<uint64_t>(bytes >> 4); };
      while (ok && walk.next(p, b, c0, c1, split)) {
        const int n = c1 - c0;
        if (!warp_all_dwait(bar(kBarQFull), chunk & 1, wc)) break;
        tc_fence_after();
        for (int e = 0; ok && e < 2 * n; ++e) {
          bool is_pv;
          int t;
          order_at(e, n, is_pv, t);
          if (!is_pv) {
            // QK(t): partial S^T over this CTA's 288 dims into S buffer u % 2
            const int sb = static_cast<int>(u % kNumS);
            if (!warp_all_dwait(bar(kBarSEmpty + sb), ((u / kNumS) & 1u) ^ 1u, wc)) { ok = false; break; }
            const uint32_t d = tmem + C::kColS + sb * RG;
            const int r = static_cast<int>(gr % kRopeSlots);
            if (!warp_all_dwait(bar(kBarRopeFull + r), (gr / kRopeSlots) & 1u, wc)) { ok = false; break; }
            tc_fence_after();
            const uint64_t rdesc = adv(rdesc0, static_cast<uint32_t>(r) * kRopeSlotBytes);
#pragma unroll
            for (int kk = 0; kk < 2; ++kk)
              umma_bf16_warp(d, adv(rdesc, 32 * kk), adv(qrdesc0, 32 * kk), C::kIdescQK, kk != 0 ? 1u : 0u);
            umma_commit_warp(bar(kBarRopeEmpty + r));
            ++gr;
            for (int k = 0; ok && k < 2; ++k) {
              const uint32_t s = g % C::kNumSlots;
              if (!warp_all_dwait(bar(kBarSlotFull + s), (g / C::kNumSlots) & 1u, wc)) { ok = false; break; }
              tc_fence_after();
              ++g;
              const uint64_t kdesc = adv(kdesc0, s * kSlotBytes);
#pragma unroll
              for (int kk = 0; kk < 8; ++kk)
                umma_bf16_warp(d, adv(kdesc, (kk >> 2) * kAtomBytes + (kk & 3) * 32),
                          adv(qdesc0, (2 * k + (kk >> 2)) * C::kQAtomBytes + (kk & 3) * 32), C::kIdescQK, 1u);
            }
            if (!ok) break;
            umma_commit_warp(bar(kBarSFull + sb));
            ++u;
            if (t == n - 1) umma_commit_warp(bar(kBarQEmpty));
          } else {
            // PV(t): O_c^T += V_c^T . P^T from the two slots QK(t) read (kept since then)
            const int pb = static_cast<int>(up % kNumP);
            if (!warp_all_dwait(bar(kBarPFull + pb), (up / kNumP) & 1u, wc)) { ok = false; break; }
            if (t == 0 && !warp_all_dwait(bar(kBarOEmpty), (chunk & 1) ^ 1, wc)) { ok = false; break; }
            tc_fence_after();
            const uint64_t pdesc = adv(pdesc0, static_cast<uint32_t>(pb) * C::kPBytes);
            for (int k = 0; k < 2; ++k) {
              const uint32_t s = (gchunk + 2u * static_cast<uint32_t>(t) + static_cast<uint32_t>(k)) % C::kNumSlots;
              const uint64_t vdesc = adv(vdesc0, s * kSlotBytes);
              const uint32_t d = tmem + C::kColO + k * RG;
#pragma unroll
              for (int kt = 0; kt < 8; ++kt)
                umma_bf16_warp(d, adv(vdesc, kt * 2048), adv(pdesc, kt * 16 * C::kPRowBytes), C::kIdescPV,
                          (t == 0 && kt == 0) ? 0u : 1u);
              umma_commit_warp(bar(kBarSlotEmpty + s));
            }
            umma_commit_warp(bar(kBarPEmpty + pb));
            ++up;
          }
        }
        if (!ok) break;
        umma_commit_warp(bar(kBarOFull));
        gchunk += 2u * static_cast<uint32_t>(n);
        ++chunk;
      }
      // every MMA this warp issued is complete before TMEM is released
      umma_commit_warp(bar(kBarDrain));
      drain_wait(bar(kBarDrain), 0);
    }
  } else {
    // ============================ softmax + epilogue ==============================
    const int tid = threadIdx.x;  // 0..127: token lane of S^T, dim lane of O^T
    const uint32_t lane_base = static_cast<uint32_t>(warp * 32) << 16;
    const float NEG_INF = -CUDART_INF_F;
    const uint32_t peer_x = other(sX);
    float m_ref = NEG_INF;  // thread c < RG: reference max of row c (log2 units)
    float lsum = 0.f;       // lane's reduce-scatter column (col_of) of this warp's row sums
    uint32_t u = 0;
    uint32_t gchunk = 0;
    int chunk = 0;
    bool fail = false;
    const int R = p.rows;
    DualWalk walk(p, part0, has1);
    int b, c0, c1, split;
    while (walk.next(p, b, c0, c1, split)) {
      const int L = p.cache_seqlens[b];
      const int n = c1 - c0;
      const bool single = (p.num_splits[b + 1] - p.num_splits[b]) == 1;
      bool aborted = false;
      for (int t = 0; t < n; ++t) {
        const int t0 = (c0 + t) * kBlockTokens;
        const int j = t0 + tid;
        const int sb = static_cast<int>(u % kNumS);
        const int xb = static_cast<int>(u % kNumX);
        bool ok = warp_all_dwait(bar(kBarSFull + sb), (u / kNumS) & 1u, wc);
        float x[RG];
        tc_fence_after();
#pragma unroll
        for (int c = 0; c < RG; c += 16) tmem_ld16(tmem + lane_base + C::kColS + sb * RG + c, x + c);
        tmem_wait_ld();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(kBarSEmpty + sb));
        // exchange: this CTA's partial scores of token tid go to the peer (row tid of its
        // buffer xb); the peer's arrive here.  Both CTAs then hold own + peer in the same order.
        if (tid == 0) {
          mbar_arrive_expect_tx(bar(kBarXFull + xb), C::kXBytes);
          ++x_exp;
        }
        if (ok) {
          const uint32_t row = peer_x + static_cast<uint32_t>(xb * C::kXBytes + tid * RG * 4);
          const uint32_t xbar = other(bar(kBarXFull + xb));
#pragma unroll
          for (int k = 0; k < C::kXChunks; ++k)
            st_async_v4(row + 16u * xchunk<RG>(tid, k), __float_as_uint(x[4 * k]), __float_as_uint(x[4 * k + 1]),
                        __float_as_uint(x[4 * k + 2]), __float_as_uint(x[4 * k + 3]), xbar);
          if (tid == 0) ++x_sent;
        }
        ok &= warp_all_dwait(bar(kBarXFull + xb), (u / kNumX) & 1u, wc);
        if (tid == 0 && ok) ++x_seen;
        {
          const uint32_t row = sX + static_cast<uint32_t>(xb * C::kXBytes + tid * RG * 4);
#pragma unroll
          for (int k = 0; k < C::kXChunks; ++k) {
            float4 y;
            asm volatile("ld.shared.v4.f32 {%0, %1, %2, %3}, [%4];"
                         : "=f"(y.x), "=f"(y.y), "=f"(y.z), "=f"(y.w)
                         : "r"(row + 16u * xchunk<RG>(tid, k)));
            // own + peer in CTA 0, peer + own in CTA 1: the same sum
            x[4 * k + 0] += y.x;
            x[4 * k + 1] += y.y;
            x[4 * k + 2] += y.z;
            x[4 * k + 3] += y.w;
          }
        }
        // scale into log2 units and mask: key j is visible to row c iff j < L and, when causal,
        // j <= L - s_q + c / h_q (the query block sits at the end of the cache).  With
        // i0 = j - L + s_q that is c / h_q >= i0, i.e. c >= i0 * h_q.
        int cmin = -(1 << 30);
        if (p.causal) {
          const int i0 = j - L + p.s_q;
          if (i0 > 0) cmin = i0 * p.h_q;
        }
        if (j >= L) cmin = 1 << 30;
#pragma unroll
        for (int c = 0; c < RG; ++c) x[c] = (c >= cmin) ? x[c] * p.scale_log2 : NEG_INF;
        float v[RG];
#pragma unroll
        for (int c = 0; c < RG; ++c) v[c] = x[c];
        reduce_scatter<RG, true>(v, lane);
        red[warp * 32 + col_of<RG>(lane)] = v[0];
        if (named_bar_any(1, 128, !ok || fail)) { aborted = true; break; }
        bool need = false;
        if (tid < RG) {
          const float bm = fmaxf(fmaxf(red[tid], red[32 + tid]), fmaxf(red[64 + tid], red[96 + tid]));
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
        lsum = lsum * alpha_sm[col_of<RG>(lane)] + v[0];
        // P^T row of this token (bf16), once PV(u - kNumP) has released the buffer
        const int pb = static_cast<int>(u % kNumP);
        if (u >= static_cast<uint32_t>(kNumP))
          ok &= warp_all_dwait(bar(kBarPEmpty + pb), ((u - kNumP) / kNumP) & 1u, wc);
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
          ok &= warp_all_dwait(bar(kBarPEmpty + uq % kNumP), (uq / kNumP) & 1u, wc);
          tc_fence_after();
#pragma unroll
          for (int k = 0; k < 2; ++k) {
#pragma unroll
            for (int c = 0; c < RG; c += 16) {
              float o[16];
              const uint32_t ta = tmem + lane_base + C::kColO + k * RG + c;
              tmem_ld16(ta, o);
              tmem_wait_ld();
#pragma unroll
              for (int e = 0; e < 16; ++e) o[e] *= alpha_sm[c + e];
              tmem_st16(ta, o);
            }
          }
          tmem_wait_st();
        }
        if (t0 + kBlockTokens > L && j >= L) {
          // tail step: zero this CTA's V rows of tokens past the end (their cache slots may hold
          // NaN, and 0 * NaN would poison O).  QK(t) has read the slots (its S^T was waited for).
#pragma unroll
          for (int k = 0; k < 2; ++k) {
            const uint32_t s = (gchunk + 2u * static_cast<uint32_t>(t) + static_cast<uint32_t>(k)) % C::kNumSlots;
            const uint32_t rowaddr = sSlots + s * kSlotBytes + static_cast<uint32_t>(tid) * 128u;
#pragma unroll
            for (int a = 0; a < 2; ++a)
#pragma unroll
              for (int q = 0; q < 8; ++q) st_shared_v4(rowaddr + a * kAtomBytes + 16u * q, 0u, 0u, 0u, 0u);
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
      red[warp * 32 + col_of<RG>(lane)] = lsum;
      if (named_bar_any(1, 128, fail)) break;
      if (tid < RG) {
        const float l = red[tid] + red[32 + tid] + red[64 + tid] + red[96 + tid];
        const float lse_val = l > 0.f ? (m_ref + log2f(l)) * kLn2 : NEG_INF;
        inv_sm[tid] = l > 0.f ? 1.f / l : 0.f;
        if (rank == 0 && tid < R) {
          if (single)
            p.lse[(static_cast<long long>(b) * p.h_q + tid % p.h_q) * p.s_q + tid / p.h_q] = lse_val;
          else
            p.lse_part[static_cast<long long>(split) * R + tid] = lse_val;
        }
        m_ref = NEG_INF;
      }
      lsum = 0.f;
      named_bar_sync(1, 128);
      const bool ok = warp_all_dwait(bar(kBarOFull), chunk & 1, wc);
      fail |= !ok;
      tc_fence_after();
      {
        // O^T block k (this CTA's dims 256 rank + 128k + tid), columns = query rows: written
        // through the P^T buffers (free once the chunk's last PV has completed) as
        // [row][128 dims], then stored by one thread with a TMA tensor store (rows past the
        // request's end fall outside the map).
        float* stage_f = reinterpret_cast<float*>(smem + C::kOffP);
        __nv_bfloat16* stage_h = reinterpret_cast<__nv_bfloat16*>(smem + C::kOffP);
#pragma unroll 1
        for (int k = 0; k < 2; ++k) {
          if (k > 0) {
            // the previous block's store has read the buffers
            if (tid == 0) bulk_wait_read_all();
            named_bar_sync(1, 128);
          }
#pragma unroll
          for (int c = 0; c < RG; c += 16) {
            float o[16];
            tmem_ld16(tmem + lane_base + C::kColO + k * RG + c, o);
            tmem_wait_ld();
#pragma unroll
            for (int e = 0; e < 16; ++e) {
              const float val = o[e] * inv_sm[c + e];
              if (single)
                stage_h[(c + e) * 128 + tid] = __float2bfloat16_rn(val);
              else
                stage_f[(c + e) * 128 + tid] = val;
            }
          }
          fence_proxy_async_smem();
          named_bar_sync(1, 128);
          if (tid == 0) {
            const int dd = kDimsPerCta * static_cast<int>(rank) + 128 * k;
            if (single)
              tma_store_3d(&tm_out, sP, dd, 0, b);
            else
              tma_store_3d(&tm_opart, sP, dd, 0, split);
            bulk_commit();
          }
        }
        // the buffers hold P^T again from the next step on
        if (tid == 0) bulk_wait_read_all();
        named_bar_sync(1, 128);
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(kBarOEmpty));
      gchunk += 2u * static_cast<uint32_t>(n);
      ++chunk;
    }
    // the peer learns how many partials this CTA sent (read after the cluster barrier below)
    if (tid == 0) st_cluster_u32(other(sMisc + kMiscPeerSent), x_sent);
  }

  // ---------------------------------- exit ----------------------------------------
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();
  if (threadIdx.x == 0 && *abort_flag) {
    // After an abort the two CTAs may have stopped at different steps: let every partial the
    // peer sent land here before this CTA's shared memory goes away.  A phase this CTA never
    // reached still needs its expected-bytes arrival.
    const uint32_t peer_sent = *reinterpret_cast<volatile uint32_t*>(misc + kMiscPeerSent);
    for (uint32_t k = x_seen; k < peer_sent; ++k) {
      const int xb = static_cast<int>(k % kNumX);
      if (k >= x_exp) mbar_arrive_expect_tx(bar(kBarXFull + xb), C::kXBytes);
      drain_wait(bar(kBarXFull + xb), (k / kNumX) & 1u);
    }
  }
  __syncthreads();
  cluster_sync_all();
  if (warp == 5) {
    tc_fence_after();
    tmem_dealloc(tmem, C::kTmemCols);
  }
}

template <int RG>
int launch_dsplit_impl(const CUtensorMap& tm_q, const CUtensorMap& tm_q_rope, const CUtensorMap& tm_kv,
                       const CUtensorMap& tm_kv_rope, const OutMaps& om, const DecodeParams& p, cudaStream_t stream) {
  using C = DsCfg<RG>;
  auto kern = mla_decode_dsplit_kernel<RG>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemBytes);
  if (e != cudaSuccess) return static_cast<int>(e);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2 * ((p.num_sm_parts + 1) / 2), 1, 1);  // one cluster per two scheduler parts
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = C::kSmemBytes;
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;  // overlaps the scheduler's tail
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  e = cudaLaunchKernelEx(&cfg, kern, tm_q, tm_q_rope, tm_kv, tm_kv_rope, om.o_part, om.out, p);
  return static_cast<int>(e);
}

}  // namespace

int launch_decode_dsplit_bf16(const CUtensorMap& tm_q, const CUtensorMap& tm_q_rope, const CUtensorMap& tm_kv,
                              const CUtensorMap& tm_kv_rope, const OutMaps& om, const DecodeParams& p,
                              int rows_per_cluster, cudaStream_t stream) {
  switch (rows_per_cluster) {
    case 16: return launch_dsplit_impl<16>(tm_q, tm_q_rope, tm_kv, tm_kv_rope, om, p, stream);
    case 32: return launch_dsplit_impl<32>(tm_q, tm_q_rope, tm_kv, tm_kv_rope, om, p, stream);
    default: return static_cast<int>(cudaErrorInvalidValue);
  }
}

}  // namespace mla

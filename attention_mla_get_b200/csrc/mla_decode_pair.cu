// Split-KV MLA decode on CTA pairs (cta_group::2) for requests with more than 64 query rows:
// bf16 or FP8 paged KV cache, and token-sparse decode / sparse prefill (bf16).
//
// The problem is the one of mla_decode.cu (FlashMLA pages: mha_fwd_kvcache_mla on a paged
// latent cache of 576-dim tokens, V = the first 512 dims, 64-token pages addressed by
// block_table).  With many query rows per request (h_q = 128 query heads sharing one latent KV
// head, "MLA" on the deepseekonline.chat page) the work per cached token is large, so the
// kernel is bound by the tensor core, and what limits it is how many bytes the SMs must read
// per MMA.  A 2-SM pair handles 128 query rows and 256 tokens per step:
//
//   S^T [256 tokens x 128 rows]  = K[256 x 576] . Q^T[576 x 128]        M = 256, N = 128
//   O^T [512 dims  x 128 rows]  += V^T[512 x 256] . P^T[256 x 128]      2 x (M = 256, N = 128)
//
// Each MMA of the pair runs at the full per-SM rate (N = 128), each CTA keeps only its 64 rows
// of Q^T (N half) and of P^T, and each SM's tensor memory holds the pair's M half: S^T of its own
// 128 tokens and O^T of its own 256 output dims (dims 128c..128c+127 and 256+128c..256+128c+127
// on CTA c).  That is 2 x 128 + 2 x 128 of the 512 TMEM columns, so the whole 512 x 128 output
// of a 128-row group stays on chip.
//
// Data per step and CTA c: the 9 K boxes (64 dims x 128 tokens) of its own 128-token block for
// S^T, and the V boxes (its 256 dims x all 256 tokens) for O^T, read through the block table
// with 64-token TMA boxes (the 9-boxes-per-page split of the wmrh.cn page, "内存访问优化策略").
// Both CTAs' loads count their bytes on the leader's (rank 0) barrier (each CTA's producer runs
// on one lane); the leader's MMA warp issues the pair MMAs (converged, one elected lane per MMA
// and commit); tcgen05.commit multicasts completion to both CTAs.
//
// Online softmax (the running-max-and-rescale idea of the wmrh.cn page, "跷跷板调度算法"):
// CTA c sees only its own 128 tokens of S^T, so the per-row block maximum is exchanged through
// distributed shared memory every step, and both CTAs make the same rescale decisions.  Each
// CTA writes the bf16 P^T rows of its tokens into both CTAs' P^T halves (64 query rows each).
// Row sums are exchanged once per chunk.
//
// Ring: 32 KB stages (K stage = 128 tokens x 128 dims, V stage = two pages x 128 dims) and a
// separate slot for the 64 RoPE dims of a K step.  Order per chunk of n pair steps: K(0), K(1),
// then V(t), K(t + 2) for t = 0 .. n-1 (QK runs one step ahead of PV).  Tokens past the request
// or the chunk are masked in S^T; their V rows (stale ring contents or the cache's unused page
// tail) are zeroed by each CTA before PV reads them.
//
// FP8 cache (656-byte tokens: 512 e4m3 codes, 4 fp32 scales per 128 dims, 64 bf16 RoPE dims;
// the wmrh.cn page, "FP8 KV缓存内存效率" table): the producer TMA-loads raw code columns (128
// dims x 2 pages) with their scales into a raw ring of this CTA; four dequant warps write each
// stage of the same order as f16 (code * scale) into the 32 KB stages, with zeros for tokens
// outside the request, and convert the Q tile and each RoPE slot from bf16 to f16 in place.
// The MMAs then run on f16 operands: e4m3 codes are exact in f16, which also keeps 11
// mantissa bits of q, P and code * scale where bf16 keeps 8 (f16's range, |x| < 65504, holds
// for the scaled cache and the queries).
//
// Token-sparse (SPARSE): the steps run over 128-slot blocks of each query position's index
// list; a row-lookup warp and five gather warps copy the listed rows with 16-byte cp.async.
//
// Epilogue: each 32-row group of O^T goes from tensor memory through the P^T buffer to global
// memory with TMA tensor stores.  The kernel is launched as a programmatic dependent of the
// tile scheduler: its set-up overlaps the scheduler, and it waits for the metadata after it.
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <math_constants.h>

#include <type_traits>

#include "mla_internal.h"
#include "mla_ptx.cuh"

namespace mla {

namespace {

constexpr float kTau = 8.0f;  // lazy-rescale threshold, log2 units
constexpr float kLn2 = 0.69314718055994530942f;
// warps 0-7 softmax + epilogue, 8 producer, 9 MMA issuer / TMEM owner, 10-13 FP8 dequant
constexpr int kSoftmaxThreads = 256;
constexpr int kWarpProducer = 8;
constexpr int kWarpMma = 9;
constexpr int kWarpDequant = 10;
constexpr int kDequantThreads = 128;
constexpr int kRows = 128;        // query rows per pair
constexpr int kHalfRows = 64;     // query rows of Q^T / P^T held by each CTA
// The ring holds 32 KB stages of 8 MMAs each: every wait on a barrier in the MMA issue stream
// idles the tensor pipe for ~200 cycles, so stages must carry enough MMA work to amortise it.
constexpr int kSlotBytes = 32768;
constexpr int kHalfBytes = 16384;  // half a stage: 128 tokens x 64 dims, or one page x 128 dims
constexpr int kRopeBytes = 16384;  // the 64 RoPE dims of a K step: a ring of its own (one slot)
constexpr int kBoxBytes = 8192;    // 64 tokens x 64 dims bf16
constexpr int kKFills = 4;         // K stages per step (dims 0-511 in 128-dim blocks)
constexpr int kVFills = 4;         // V stages per step (2 dim blocks x 2 token blocks)
constexpr int kQBytes = 9 * kBoxBytes;          // 64 rows x 576 dims
constexpr int kPBytes = 256 * kHalfRows * 2;    // 256 tokens x 64 rows bf16
constexpr int kRawCodeBytes = 16384;  // FP8: 128 dims x 2 pages of e4m3 codes
constexpr int kRawScaleBytes = 2048;  // FP8: the 4 fp32 scales of those 128 tokens
constexpr int kRawBytes = kRawCodeBytes + kRawScaleBytes;
constexpr int kNumRaw = 2;
constexpr int kOffQ = 0;
constexpr int kOffP = kOffQ + kQBytes;
constexpr int kOffSlots = kOffP + kPBytes;
constexpr int kMiscBytes = 6144;
constexpr int kRowSlots = 4;  // token-sparse: ring of row tables (one per pair step)
constexpr int kTmemCols = 512;
constexpr int kColO = 0;      // O^T dim block m at columns 128m
constexpr int kColS = 256;    // S^T buffer sb at columns 256 + 128 sb

// f16 operands (FP8 cache): the A and B format fields of the instruction descriptor are 0
__host__ __device__ constexpr uint32_t idesc_f16(int M, int N, bool a_mn_major, bool b_mn_major) {
  return idesc_bf16(M, N, a_mn_major, b_mn_major) & ~((7u << 7) | (7u << 10));
}

template <bool FP8, bool SPARSE = false>
struct PairCfg {
  // FP8 and token-sparse: 16 warps (FP8: two idle) so that the compiler keeps every thread
  // within 128 registers, the per-SM-sub-partition share of 4 resident warps
  static constexpr int kThreads = (FP8 || SPARSE) ? 512 : 320;
  static constexpr int kNumSlots = FP8 ? 2 : 3;  // FP8 gives a stage to the raw ring
  static constexpr int kOffRaw = kOffSlots + kNumSlots * kSlotBytes;
  static constexpr int kOffRope = kOffRaw + (FP8 ? kNumRaw * kRawBytes : 0);
  static constexpr int kOffMisc = kOffRope + kRopeBytes;
  // token-sparse: + the ring of row tables, 1 KB per step (256 list slots)
  static constexpr int kMisc = kMiscBytes + (SPARSE ? kRowSlots * 1024 : 0);
  static constexpr int kSmemBytes = kOffMisc + kMisc + 1024;  // + alignment slack
  static constexpr uint32_t kIdescQK = FP8 ? idesc_f16(256, kRows, false, false) : idesc_bf16(256, kRows, false, false);
  static constexpr uint32_t kIdescPV = FP8 ? idesc_f16(256, kRows, true, true) : idesc_bf16(256, kRows, true, true);
  static_assert(kSmemBytes <= 232448, "shared memory budget");
  static_assert(kOffSlots % 1024 == 0 && kOffRope % 1024 == 0 && kOffRaw % 128 == 0,
                "swizzle atoms need 1024-byte alignment");
};
static_assert(kOffP % 1024 == 0, "swizzle atoms need 1024-byte alignment");
constexpr int kMaxSlots = 3;

// misc area: barriers, then scalars, then per-row scratch
enum : int {
  // [stages] leader: both producers, count 2 + bytes (FP8: every dequant warp of both CTAs)
  kBarSlotFull = 0,
  kBarSlotEmpty = kBarSlotFull + kMaxSlots,   // [stages] both: pair commit
  kBarZFull = kBarSlotEmpty + kMaxSlots,      // [stages] leader: both CTAs zeroed a tail V slot
  kBarZLocal = kBarZFull + kMaxSlots,         // [stages] both: this CTA's bytes of a tail V slot
  // leader: both producers, count 2 + bytes (FP8: this CTA's producer, count 1 + bytes)
  kBarRopeFull = kBarZLocal + kMaxSlots,
  kBarRopeEmpty = kBarRopeFull + 1,           // both: pair commit
  kBarSFull = kBarRopeEmpty + 1,              // [2] both: pair commit
  kBarSEmpty = kBarSFull + 2,                 // [2] leader: 16 softmax warps of the pair
  kBarPFull = kBarSEmpty + 2,                 // leader: the 8 warps that write P^T locally
  kBarPEmpty = kBarPFull + 1,                 // both: pair commit
  kBarQFull = kBarPEmpty + 1,                 // leader: both producers (FP8: this CTA's, count 1)
  kBarQEmpty = kBarQFull + 1,                 // both: pair commit
  kBarOFull = kBarQEmpty + 1,                 // both: pair commit
  kBarOEmpty = kBarOFull + 1,                 // leader: 16 epilogue warps
  kBarDrain = kBarOEmpty + 1,                 // leader: final commit
  kBarMaxFull = kBarDrain + 1,                // [2] both: 512 bytes of the peer's block maxima
  kBarLFull = kBarMaxFull + 2,                // both: 512 bytes of the peer's row sums
  kBarPRecv = kBarLFull + 1,                  // both: 16 KB of P^T rows from the peer
  kBarRawFull = kBarPRecv + 1,                // [2] FP8, both: this CTA's raw fill, count 1 + bytes
  kBarRawEmpty = kBarRawFull + kNumRaw,       // [2] FP8, both: this CTA's dequant warps
  kBarQReady = kBarRawEmpty + kNumRaw,        // FP8, leader: Q in f16 (every dequant warp, both CTAs)
  kBarRopeReady = kBarQReady + 1,             // FP8, leader: RoPE slot in f16 (as kBarQReady)
  // token-sparse, both: this CTA's gather warps' cp.async landed ([stages], then RoPE slot)
  kBarGather = kBarRopeReady + 1,
  kBarGatherRope = kBarGather + kMaxSlots,
  kBarRowFull = kBarGatherRope + 1,           // [row tables] token-sparse: the 32 lanes of the index warp
  kBarRowEmpty = kBarRowFull + kRowSlots,     // [row tables] token-sparse: every gather lane
  kNumBars = kBarRowEmpty + kRowSlots,
};
constexpr int kMiscHolder = 512;   // TMEM base address
constexpr int kMiscAbort = 516;    // abort flag
constexpr int kMiscPeerFills = 520;// follower's slot fills (written into the leader at exit)
constexpr int kMiscPeerQ = 524;    // follower's Q fills
constexpr int kMiscPeerRope = 528; // follower's RoPE fills
constexpr int kMiscRed = 1024;     // float [4 lane quadrants][128 rows]
constexpr int kMiscM = 3072;       // float [128]
constexpr int kMiscAlpha = 3584;   // float [128]
constexpr int kMiscInv = 4096;     // float [128]
constexpr int kMiscXMax = 4608;    // float [2][128]: the peer's block maxima
constexpr int kMiscXL = 5632;      // float [128]: the peer's row sums
constexpr int kMiscRowTab = 6144;  // token-sparse: int32 [row tables][256] cache rows of a step's slots
constexpr int kWarpIndex = 10;     // token-sparse: the warp that looks up the cache rows
constexpr int kGatherWarps = 5;    // token-sparse: warps 11-15 copy the listed tokens' rows
constexpr int kGatherThreads = 32 * kGatherWarps;
static_assert(kNumBars * 8 <= kMiscHolder, "barrier area");
static_assert(kMiscXL + 512 <= kMiscBytes, "misc area");

__device__ __forceinline__ int blocks_of(int L) { return L > 0 ? (L + kBlockTokens - 1) / kBlockTokens : 0; }

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

// Fill / consume order of a chunk of n pair steps: K(0), K(1), then V(t), K(t + 2).
__device__ __forceinline__ void order_at(int e, int n, bool& is_v, int& step) {
  const int head = min(2, n);
  if (e < head) {
    is_v = false;
    step = e;
    return;
  }
  const int r = e - head;
  const int tail_k = n - head;
  if (r < 2 * tail_k) {
    is_v = (r & 1) == 0;
    step = is_v ? (r >> 1) : (r >> 1) + head;
  } else {
    is_v = true;
    step = tail_k + (r - 2 * tail_k);
  }
}
// Slot fills of the chunk before the first V slot of step t.
__device__ __forceinline__ uint32_t fills_before_v(int t, int n) {
  return static_cast<uint32_t>(kKFills * min(t + 2, n) + kVFills * t);
}
// Step t of a chunk [c0, c1) reads tokens no request position covers (V rows must be zeroed).
__device__ __forceinline__ bool is_tail(int c0, int c1, int t, int L) {
  return (c0 + 2 * t + 1 >= c1) || ((c0 + 2 * t + 2) * kBlockTokens > L);
}

// Bounded waits.  On time-out: status bit, this CTA's and the peer's abort flags; every waiter
// of both CTAs then unwinds.
struct PairCtl {
  volatile int* abort_flag;
  uint32_t peer_abort;  // cluster address of the peer's abort flag
  int* status;
};

static __device__ __noinline__ void pair_timeout(const PairCtl& c) {
  *c.abort_flag = 1;
  st_cluster_u32(c.peer_abort, 1u);
  if (c.status) atomicOr(c.status, kStatusWaitTimeout);
  __threadfence();
}

__device__ __forceinline__ bool pwait(uint32_t bar, uint32_t parity, const PairCtl& c) {
  if (mbar_try_wait(bar, parity)) return true;
  const long long t0 = clock64();
  while (true) {
    if (mbar_try_wait(bar, parity)) return true;
    if (*c.abort_flag) return false;
    if (clock64() - t0 > kWaitLimitCycles) {
      pair_timeout(c);
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

// Warp waits: every lane polls the barrier itself (it then reads or overwrites what the phase
// guards) and the outcome is made warp-uniform; false on every lane if any gave up.  Polling on
// one lane and broadcasting the outcome with a shuffle measured 2-5 % slower per step.
__device__ __forceinline__ bool warp_all_wait(uint32_t bar, uint32_t parity, const PairCtl& c) {
  return __all_sync(0xffffffffu, pwait(bar, parity, c) ? 1 : 0) != 0;
}

// Warp reduce-scatter (sum) of 64 column values over the 32 token lanes: afterwards lane l
// holds the warp-wide sums of columns 2l and 2l + 1 in v[0], v[1].
__device__ __forceinline__ void reduce_scatter64_sum(float* v, int lane) {
#pragma unroll
  for (int r = 0; r < 5; ++r) {
    const int o = 16 >> r;
    const int n = 64 >> r;
    const bool upper = (lane & o) != 0;
#pragma unroll
    for (int i = 0; i < n / 2; ++i) {
      const float keep = upper ? v[i + n / 2] : v[i];
      const float send = upper ? v[i] : v[i + n / 2];
      v[i] = keep + __shfl_xor_sync(0xffffffffu, send, o);
    }
  }
}

// bf16 pair -> f16 pair (round to nearest even)
__device__ __forceinline__ uint32_t bf16x2_to_f16x2(uint32_t w) {
  return pack_f16x2(__uint_as_float(w << 16), __uint_as_float(w & 0xFFFF0000u));
}
// Two e4m3 codes (low 16 bits) -> f16 pair of code * scale.  The codes are exact in f16; with
// the scale an f16 normal number (scale2 = that f16 twice) the product is one f16 multiply.
__device__ __forceinline__ uint32_t e4m3x2_times_f16x2(uint32_t codes, uint32_t scale2) {
  uint32_t h, r;
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h) : "h"(static_cast<unsigned short>(codes & 0xFFFFu)));
  asm("mul.rn.f16x2 %0, %1, %2;" : "=r"(r) : "r"(h), "r"(scale2));
  return r;
}
// Largest scale for which 448 * scale (the largest e4m3 magnitude) is finite in f16.
constexpr float kF16MaxScale = 65504.0f / 448.0f;
// The same with the product formed in fp32 (scales outside the f16 normal range).
__device__ __forceinline__ uint32_t e4m3x2_times_f32(uint32_t codes, float scale) {
  uint32_t h;
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h) : "h"(static_cast<unsigned short>(codes & 0xFFFFu)));
  const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&h));
  return pack_f16x2(f.x * scale, f.y * scale);
}

// One token row of an FP8 stage: 128 e4m3 codes at `src` times `scale`, as f16 into the two
// 64-dim halves of a swizzled stage row (`dst`, halves `hstride` apart; row index `row`).  All
// eight 16-byte loads are issued before the first conversion, so their latencies overlap.
__device__ __forceinline__ void dequant_row(uint32_t src, uint32_t dst, uint32_t hstride, uint32_t row, float scale) {
  const uint32_t swz = row & 7u;
  uint32_t w[8][4];
#pragma unroll
  for (int c = 0; c < 8; ++c) {
    const uint32_t cc = (static_cast<uint32_t>(c) + row) & 7u;  // spread the banks
    asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];" : "=r"(w[c][0]), "=r"(w[c][1]), "=r"(w[c][2]), "=r"(w[c][3])
                 : "r"(src + 16u * cc));
  }
  if (scale >= 6.103515625e-05f && scale <= 146.0f) {  // f16 normal scale, |448 scale| < 65504
    const __half2 s2h = __float2half2_rn(scale);
    const uint32_t s2 = *reinterpret_cast<const uint32_t*>(&s2h);
#pragma unroll
    for (int c = 0; c < 8; ++c) {
      const uint32_t cc = (static_cast<uint32_t>(c) + row) & 7u;
      // codes 16cc .. 16cc + 15: dim half cc / 4, 16-byte chunks 2 (cc % 4) and + 1
      const uint32_t base = dst + (cc >> 2) * hstride;
      const uint32_t q0 = 2u * (cc & 3u);
      st_shared_v4(base + ((q0 ^ swz) << 4), e4m3x2_times_f16x2(w[c][0], s2), e4m3x2_times_f16x2(w[c][0] >> 16, s2),
                   e4m3x2_times_f16x2(w[c][1], s2), e4m3x2_times_f16x2(w[c][1] >> 16, s2));
      st_shared_v4(base + (((q0 + 1u) ^ swz) << 4), e4m3x2_times_f16x2(w[c][2], s2),
                   e4m3x2_times_f16x2(w[c][2] >> 16, s2), e4m3x2_times_f16x2(w[c][3], s2),
                   e4m3x2_times_f16x2(w[c][3] >> 16, s2));
    }
  } else {
#pragma unroll
    for (int c = 0; c < 8; ++c) {
      const uint32_t cc = (static_cast<uint32_t>(c) + row) & 7u;
      const uint32_t base = dst + (cc >> 2) * hstride;
      const uint32_t q0 = 2u * (cc & 3u);
      st_shared_v4(base + ((q0 ^ swz) << 4), e4m3x2_times_f32(w[c][0], scale), e4m3x2_times_f32(w[c][0] >> 16, scale),
                   e4m3x2_times_f32(w[c][1], scale), e4m3x2_times_f32(w[c][1] >> 16, scale));
      st_shared_v4(base + (((q0 + 1u) ^ swz) << 4), e4m3x2_times_f32(w[c][2], scale),
                   e4m3x2_times_f32(w[c][2] >> 16, scale), e4m3x2_times_f32(w[c][3], scale),
                   e4m3x2_times_f32(w[c][3] >> 16, scale));
    }
  }
}

// SPARSE (bf16 cache): token-sparse decode, every query position a request of topk listed
// cache positions (see mla_decode.cu): warp 10 looks up the cache rows of the listed positions
// ahead of time, warps 11-15 copy those rows into the stages with 16-byte cp.async and the
// producer thread forwards each stage's completion to the leader.
template <bool FP8, bool SPARSE = false>
__global__ void __launch_bounds__(PairCfg<FP8, SPARSE>::kThreads, 1)
    mla_decode_pair_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_kv,
                           const __grid_constant__ CUtensorMap tm_scale, const __grid_constant__ CUtensorMap tm_rope,
                           const __grid_constant__ CUtensorMap tm_opart, const __grid_constant__ CUtensorMap tm_out,
                           const DecodeParams p) {
  using C = PairCfg<FP8, SPARSE>;
  constexpr int kNumSlots = C::kNumSlots;
  constexpr uint32_t kIdescQK = C::kIdescQK;
  constexpr uint32_t kIdescPV = C::kIdescPV;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  const uint32_t sQ = sbase + kOffQ;
  const uint32_t sP = sbase + kOffP;
  const uint32_t sSlots = sbase + kOffSlots;
  const uint32_t sRope = sbase + C::kOffRope;
  const uint32_t sRaw = sbase + C::kOffRaw;
  uint8_t* misc = smem + C::kOffMisc;
  const uint32_t sMisc = smem_u32(misc);
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(misc + kMiscHolder);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(misc + kMiscAbort);
  float* red = reinterpret_cast<float*>(misc + kMiscRed);
  float* m_sm = reinterpret_cast<float*>(misc + kMiscM);
  float* alpha_sm = reinterpret_cast<float*>(misc + kMiscAlpha);
  float* inv_sm = reinterpret_cast<float*>(misc + kMiscInv);
  const float* xmax = reinterpret_cast<const float*>(misc + kMiscXMax);
  const float* xl = reinterpret_cast<const float*>(misc + kMiscXL);
  auto bar = [&](int i) -> uint32_t { return sMisc + 8u * static_cast<uint32_t>(i); };

  const uint32_t rank = cluster_cta_rank();
  const uint32_t peer = rank ^ 1u;
  const bool leader = rank == 0;
  auto lead = [&](uint32_t a) -> uint32_t { return map_to_cta(a, 0); };
  auto other = [&](uint32_t a) -> uint32_t { return map_to_cta(a, peer); };

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int part = blockIdx.x >> 1;
  const int rg = blockIdx.y;  // 128-row group
  const PairCtl wc{abort_flag, other(sMisc + kMiscAbort), p.status};

  if (threadIdx.x == 0) {
    for (int i = 0; i < kNumSlots; ++i) {
      mbar_init(bar(kBarSlotFull + i), FP8 ? 2 * kDequantThreads / 32 : 2);
      mbar_init(bar(kBarSlotEmpty + i), 1);
      mbar_init(bar(kBarZFull + i), 8);
      mbar_init(bar(kBarZLocal + i), 1);
    }
    mbar_init(bar(kBarRopeFull), FP8 ? 1 : 2);
    mbar_init(bar(kBarRopeEmpty), 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(bar(kBarSFull + i), 1);
      mbar_init(bar(kBarSEmpty + i), 16);
      mbar_init(bar(kBarMaxFull + i), 1);
    }
    mbar_init(bar(kBarPFull), 8);
    mbar_init(bar(kBarPRecv), 1);
    mbar_init(bar(kBarPEmpty), 1);
    mbar_init(bar(kBarQFull), FP8 ? 1 : 2);
    mbar_init(bar(kBarQEmpty), 1);
    mbar_init(bar(kBarOFull), 1);
    mbar_init(bar(kBarOEmpty), 16);
    mbar_init(bar(kBarDrain), 1);
    mbar_init(bar(kBarLFull), 1);
    for (int i = 0; i < kNumRaw; ++i) {
      mbar_init(bar(kBarRawFull + i), 1);
      mbar_init(bar(kBarRawEmpty + i), kDequantThreads / 32);
    }
    mbar_init(bar(kBarQReady), 2 * kDequantThreads / 32);
    mbar_init(bar(kBarRopeReady), 2 * kDequantThreads / 32);
    for (int i = 0; i < kMaxSlots; ++i) mbar_init(bar(kBarGather + i), kGatherThreads);  // cp.async arrivals
    mbar_init(bar(kBarGatherRope), kGatherThreads);
    for (int i = 0; i < kRowSlots; ++i) {
      mbar_init(bar(kBarRowFull + i), 32);
      mbar_init(bar(kBarRowEmpty + i), kGatherThreads);
    }
    *abort_flag = 0;
    *reinterpret_cast<uint32_t*>(misc + kMiscPeerFills) = 0;
    *reinterpret_cast<uint32_t*>(misc + kMiscPeerQ) = 0;
    *reinterpret_cast<uint32_t*>(misc + kMiscPeerRope) = 0;
    fence_barrier_init();
  }
  if (warp == kWarpProducer && lane == 0) {
    tma_prefetch_desc(&tm_q);
    tma_prefetch_desc(&tm_kv);
    if (FP8) {
      tma_prefetch_desc(&tm_scale);
      tma_prefetch_desc(&tm_rope);
    }
  }
  if (warp == kWarpMma) {
    tmem_alloc_pair(smem_u32(tmem_holder), kTmemCols);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();  // barriers of both CTAs initialised before any remote arrive
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;

  pdl_launch_dependents();
  // launched as a programmatic dependent of the tile scheduler: the set-up above overlapped
  // it; its metadata is complete and visible from here on
  pdl_wait_primary();
  // metadata the scheduler could not build: its parts are empty, report it
  if (threadIdx.x == 0 && p.status && p.tile_md[part * kMdInts + 5] != 0) atomicOr(p.status, kStatusBadMetadata);

  // state the exit sequence needs
  uint32_t fills = 0;  // producer: stage fills issued
  int q_fills = 0;     // producer: Q fills issued
  int rope_fills = 0;  // producer: RoPE slot fills issued

  if (warp == kWarpProducer) {
    // ================================ TMA producer ================================
    if (lane == 0) {
      const uint64_t pol_stream = policy_evict_first();
      const uint64_t pol_keep = policy_evict_last();
      const uint64_t pol_v = p.row_groups > 1 ? pol_keep : pol_stream;
      const uint64_t pol_rope = p.row_groups > 1 ? pol_keep : pol_stream;
      int last_use[kNumSlots];
      for (int i = 0; i < kNumSlots; ++i) last_use[i] = -1;
      uint32_t zl_uses = 0, zl_par = 0;  // slots with a tail fill; parity of their last one
      bool ok = true;
      ChunkWalk walk(p, part);
      int b, c0, c1, split;
      // One stage = four 64x64 boxes: box (x[i], y[i]) lands at +8 KB * i and is copied only if
      // valid[i] (a page of the request).  The bytes count on the leader's full barrier, except for the
      // V stages of a tail step: there they count on this CTA's own barrier, so that this CTA can
      // zero the rows of tokens outside the request once its copy has landed (its softmax warps
      // then arrive on the leader's ZFull).
      auto fill = [&](const int* x, const int* y, const bool* valid, uint64_t pol, bool tail) -> bool {
        const int s = static_cast<int>(fills % kNumSlots);
        const uint32_t use = fills / kNumSlots;
        if (!pwait(bar(kBarSlotEmpty + s), (use & 1u) ^ 1u, wc)) return false;
        const uint32_t full = lead(bar(kBarSlotFull + s));
        uint32_t bytes = 0;
#pragma unroll
        for (int i = 0; i < 4; ++i) bytes += valid[i] ? static_cast<uint32_t>(kBoxBytes) : 0u;
        uint32_t dbar = full;
        if (tail) {
          mbar_arrive_expect_tx_relaxed(full, 0u);
          mbar_arrive_expect_tx(bar(kBarZLocal + s), bytes);
          dbar = map_to_cta(bar(kBarZLocal + s), rank);
          zl_uses |= 1u << s;
          zl_par ^= 1u << s;
        } else {
          mbar_arrive_expect_tx_relaxed(full, bytes);
        }
        const uint32_t dst = sSlots + static_cast<uint32_t>(s) * kSlotBytes;
#pragma unroll
        for (int i = 0; i < 4; ++i)
          if (valid[i]) tma_load_2d_pair(dst + i * kBoxBytes, &tm_kv, x[i], y[i], dbar, pol);
        last_use[s] = static_cast<int>(use);
        ++fills;
        return true;
      };
      // FP8: one stage's raw data = the 128 code bytes at byte cx of two pages (py, valid pv) and
      // their scales, into this CTA's raw ring ([page][64 tokens][128 B] codes, then
      // [page][64 tokens][16 B] scales), counted on this CTA's own barrier.
      int last_raw[kNumRaw];
      for (int i = 0; i < kNumRaw; ++i) last_raw[i] = -1;
      auto fill_raw = [&](int cx, const int* py, const bool* pv, uint64_t pol) -> bool {
        const int r = static_cast<int>(fills % kNumRaw);
        const uint32_t use = fills / kNumRaw;
        if (!pwait(bar(kBarRawEmpty + r), (use & 1u) ^ 1u, wc)) return false;
        const uint32_t full = bar(kBarRawFull + r);
        const uint32_t np = (pv[0] ? 1u : 0u) + (pv[1] ? 1u : 0u);
        mbar_arrive_expect_tx(full, np * (kRawCodeBytes / 2 + kRawScaleBytes / 2));
        const uint32_t dst = sRaw + static_cast<uint32_t>(r) * kRawBytes;
#pragma unroll
        for (int q = 0; q < 2; ++q) {
          if (!pv[q]) continue;
          tma_load_2d(dst + q * (kRawCodeBytes / 2), &tm_kv, cx, py[q], full, pol);
          tma_load_2d(dst + kRawCodeBytes + q * (kRawScaleBytes / 2), &tm_scale, kDv, py[q], full, pol);
        }
        last_raw[r] = static_cast<int>(use);
        ++fills;
        return true;
      };
      while (ok && walk.next(p, b, c0, c1, split)) {
        const int L = SPARSE ? 0 : p.cache_seqlens[b];  // token-sparse: b is a query position
        const int npages = (L + kPage - 1) / kPage;
        const int32_t* bt = SPARSE ? nullptr : p.block_table + static_cast<long long>(b) * p.max_blocks;
        if (!pwait(bar(kBarQEmpty), (q_fills & 1) ^ 1, wc)) break;
        if (FP8) {
          // this CTA's copy; its dequant warps convert Q to f16 before the leader's MMA uses it
          mbar_arrive_expect_tx(bar(kBarQFull), static_cast<uint32_t>(kQBytes));
          for (int a = 0; a < 9; ++a)
            tma_load_3d(sQ + a * kBoxBytes, &tm_q, 64 * a, rg * kRows + static_cast<int>(rank) * kHalfRows, b,
                        bar(kBarQFull));
        } else {
          const uint32_t qfull = lead(bar(kBarQFull));
          mbar_arrive_expect_tx_relaxed(qfull, static_cast<uint32_t>(kQBytes));
          for (int a = 0; a < 9; ++a)
            tma_load_3d_pair(sQ + a * kBoxBytes, &tm_q, 64 * a, rg * kRows + static_cast<int>(rank) * kHalfRows, b,
                             qfull);
        }
        ++q_fills;
        const int n = (c1 - c0 + 1) / 2;
        if (SPARSE) {
          // token-sparse: this CTA's gather warps fill the stages; pass each one's completion on
          // to the leader's full barrier, in the fill order (their copies are generic-proxy
          // writes, hence the proxy fence before the arrive)
          auto forward = [&]() -> bool {
            const int s = static_cast<int>(fills % kNumSlots);
            const uint32_t use = fills / kNumSlots;
            if (!pwait(bar(kBarGather + s), use & 1u, wc)) return false;
            fence_proxy_async_smem();
            mbar_arrive_remote(lead(bar(kBarSlotFull + s)));
            last_use[s] = static_cast<int>(use);
            ++fills;
            return true;
          };
          for (int e = 0; ok && e < 2 * n; ++e) {
            bool is_v;
            int t;
            order_at(e, n, is_v, t);
            if (!is_v) {
              if (!pwait(bar(kBarGatherRope), static_cast<uint32_t>(rope_fills) & 1u, wc)) { ok = false; break; }
              fence_proxy_async_smem();
              mbar_arrive_remote(lead(bar(kBarRopeFull)));
              ++rope_fills;
            }
            for (int k = 0; ok && k < 4; ++k) ok = forward();
          }
        }
        for (int e = 0; ok && !SPARSE && e < 2 * n; ++e) {
          bool is_v;
          int t;
          order_at(e, n, is_v, t);
          if (!is_v) {
            // K(t): this CTA's own 128-token block (pages a, b), all 576 dims
            const int kb = c0 + 2 * t + static_cast<int>(rank);
            const bool va = kb < c1;
            const bool vb = va && (2 * kb + 1 < npages);
            const int ya = va ? bt[2 * kb] * kPage : 0;
            const int yb = vb ? bt[2 * kb + 1] * kPage : 0;
            {
              // the RoPE dims first: QK(t) starts with them
              const uint32_t use = static_cast<uint32_t>(rope_fills);
              if (!pwait(bar(kBarRopeEmpty), (use & 1u) ^ 1u, wc)) { ok = false; break; }
              const uint32_t rbytes = static_cast<uint32_t>(((va ? 1 : 0) + (vb ? 1 : 0)) * kBoxBytes);
              if (FP8) {
                // the bf16 RoPE bytes of the 656-byte tokens, into this CTA (converted to f16 there)
                mbar_arrive_expect_tx(bar(kBarRopeFull), rbytes);
                if (va) tma_load_2d(sRope, &tm_rope, kDv + 16, ya, bar(kBarRopeFull), pol_rope);
                if (vb) tma_load_2d(sRope + kBoxBytes, &tm_rope, kDv + 16, yb, bar(kBarRopeFull), pol_rope);
              } else {
                const uint32_t rfull = lead(bar(kBarRopeFull));
                mbar_arrive_expect_tx_relaxed(rfull, rbytes);
                if (va) tma_load_2d_pair(sRope, &tm_kv, kDv, ya, rfull, pol_rope);
                if (vb) tma_load_2d_pair(sRope + kBoxBytes, &tm_kv, kDv, yb, rfull, pol_rope);
              }
              ++rope_fills;
            }
            for (int j = 0; ok && j < kKFills; ++j) {
              // half h = dims 128j + 64h .. +63 of both pages (page a at +0, page b at +8 KB)
              if (FP8) {
                const int py[2] = {ya, yb};
                const bool pv[2] = {va, vb};
                ok = fill_raw(128 * j, py, pv, pol_keep);
              } else {
                const int x[4] = {128 * j, 128 * j, 128 * j + 64, 128 * j + 64};
                const int yy[4] = {ya, yb, ya, yb};
                const bool vv[4] = {va, vb, va, vb};
                ok = fill(x, yy, vv, pol_keep, false);
              }
            }
          } else {
            // V(t): this CTA's 256 output dims of the step's two token blocks; stage (m, blk) holds
            // dims 256m + 128 rank .. +127 of pages 2(c0 + 2t + blk) (+0) and +1 (+16 KB)
            const bool tail = is_tail(c0, c1, t, L);
            bool v[4];
            int y[4];
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              const int pg = 2 * (c0 + 2 * t) + q;
              v[q] = (c0 + 2 * t + (q >> 1) < c1) && pg < npages;
              y[q] = v[q] ? bt[pg] * kPage : 0;
            }
            for (int m = 0; ok && m < 2; ++m) {
              const int d = 256 * m + 128 * static_cast<int>(rank);
              for (int blk = 0; ok && blk < 2; ++blk) {
                if (FP8) {
                  const int py[2] = {y[2 * blk], y[2 * blk + 1]};
                  const bool pv[2] = {v[2 * blk], v[2 * blk + 1]};
                  ok = fill_raw(d, py, pv, pol_v);
                } else {
                  const int x[4] = {d, d + 64, d, d + 64};
                  const int yy[4] = {y[2 * blk], y[2 * blk], y[2 * blk + 1], y[2 * blk + 1]};
                  const bool vv[4] = {v[2 * blk], v[2 * blk], v[2 * blk + 1], v[2 * blk + 1]};
                  ok = fill(x, yy, vv, pol_v, tail);
                }
              }
            }
          }
        }
      }
      if (!*abort_flag) {
        // the last pair commits on this CTA's barriers have landed before it may exit
        for (int s = 0; s < kNumSlots; ++s)
          if (last_use[s] >= 0) drain_wait(bar(kBarSlotEmpty + s), static_cast<uint32_t>(last_use[s]) & 1u);
        if (q_fills > 0) drain_wait(bar(kBarQEmpty), static_cast<uint32_t>(q_fills - 1) & 1u);
        if (rope_fills > 0) drain_wait(bar(kBarRopeEmpty), static_cast<uint32_t>(rope_fills - 1) & 1u);
      } else if (FP8) {
        // every copy of an FP8 CTA counts on its own barriers: let the last ones land
        for (int r = 0; r < kNumRaw; ++r)
          if (last_raw[r] >= 0) drain_wait(bar(kBarRawFull + r), static_cast<uint32_t>(last_raw[r]) & 1u);
        if (q_fills > 0) drain_wait(bar(kBarQFull), static_cast<uint32_t>(q_fills - 1) & 1u);
        if (rope_fills > 0) drain_wait(bar(kBarRopeFull), static_cast<uint32_t>(rope_fills - 1) & 1u);
      } else {
        // copies of tail V slots count on this CTA's own barriers: let them land
        for (int s = 0; s < kNumSlots; ++s)
          if ((zl_uses >> s) & 1u) drain_wait(bar(kBarZLocal + s), ((zl_par >> s) & 1u) ^ 1u);
      }
      if (!FP8 && !leader) {
        st_cluster_u32(lead(sMisc + kMiscPeerFills), fills);
        st_cluster_u32(lead(sMisc + kMiscPeerQ), static_cast<uint32_t>(q_fills));
        st_cluster_u32(lead(sMisc + kMiscPeerRope), static_cast<uint32_t>(rope_fills));
      }
    }
  } else if (warp == kWarpMma) {
    // ================================ MMA issuer (leader) =========================
    // the leader's whole warp runs the issue loop (waits seen by every lane, outcome warp-uniform);
    // each MMA and commit is issued by one elected lane
    if (leader) {
      uint32_t u = 0;   // QK steps issued
      uint32_t up = 0;  // PV steps issued
      uint32_t rope_used = 0;
      uint32_t zpar = 0;
      int chunk = 0;
      bool ok = true;
      ChunkWalk walk(p, part);
      int b, c0, c1, split;
      uint32_t gs = 0, gph = 0;  // slot of the next fill to consume, and its phase parity
      auto next_slot = [&](uint32_t& s) -> bool {
        s = gs;
        if (!warp_all_wait(bar(kBarSlotFull + s), gph, wc)) return false;
        if (++gs == static_cast<uint32_t>(kNumSlots)) {
          gs = 0;
          gph ^= 1u;
        }
        return true;
      };
      // shared-memory descriptors of stage 0; stage s adds s * kSlotBytes >> 4
      const uint64_t kdesc0 = smem_desc(sSlots, 16, 1024, kSwizzle128);
      const uint64_t vdesc0 = smem_desc(sSlots, kBoxBytes, 1024, kSwizzle128);
      while (ok && walk.next(p, b, c0, c1, split)) {
        const int L = SPARSE ? 0 : p.cache_seqlens[b];
        const int n = (c1 - c0 + 1) / 2;
        // FP8: both CTAs' dequant warps have converted their Q halves to f16
        if (!warp_all_wait(bar(FP8 ? kBarQReady : kBarQFull), chunk & 1, wc)) break;
        for (int e = 0; ok && e < 2 * n; ++e) {
          bool is_v;
          int t;
          order_at(e, n, is_v, t);
          if (!is_v) {
            const int sb = static_cast<int>(u & 1u);
            // the softmax warps finished their tcgen05.ld of this buffer (wait::ld) before arriving
            if (!warp_all_wait(bar(kBarSEmpty + sb), ((u >> 1) & 1u) ^ 1u, wc)) { ok = false; break; }
            const uint32_t d = tmem + kColS + 128u * sb;
            // RoPE dims first (they have their own slot), then the four 128-dim K stages
            if (!warp_all_wait(bar(FP8 ? kBarRopeReady : kBarRopeFull), rope_used & 1u, wc)) { ok = false; break; }
            ++rope_used;
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
              umma_bf16_pair_warp(d, smem_desc(sRope + 32 * kk, 16, 1024, kSwizzle128),
                                  smem_desc(sQ + 8 * kBoxBytes + 32 * kk, 16, 1024, kSwizzle128), kIdescQK,
                                  kk != 0 ? 1u : 0u);
            umma_commit_pair_mc_warp(bar(kBarRopeEmpty), 0x3);
            for (int j = 0; ok && j < kKFills; ++j) {
              uint32_t s;
              if (!next_slot(s)) { ok = false; break; }
              // descriptors advance by (byte offset >> 4) in their start-address field
              const uint64_t a0 = kdesc0 + static_cast<uint64_t>(s * (kSlotBytes >> 4));
              const uint64_t b0 = smem_desc(sQ + 2 * j * kBoxBytes, 16, 1024, kSwizzle128);
#pragma unroll
              for (int kk = 0; kk < 8; ++kk)
                umma_bf16_pair_warp(d, a0 + static_cast<uint64_t>(((kk >> 2) * kHalfBytes + 32 * (kk & 3)) >> 4),
                                    b0 + static_cast<uint64_t>(((kk >> 2) * kBoxBytes + 32 * (kk & 3)) >> 4),
                                    kIdescQK, 1u);
              umma_commit_pair_mc_warp(bar(kBarSlotEmpty + s), 0x3);
            }
            if (!ok) break;
            umma_commit_pair_mc_warp(bar(kBarSFull + sb), 0x3);
            ++u;
            if (t == n - 1) umma_commit_pair_mc_warp(bar(kBarQEmpty), 0x3);
          } else {
            if (!warp_all_wait(bar(kBarPFull), up & 1u, wc)) { ok = false; break; }
            if (t == 0 && !warp_all_wait(bar(kBarOEmpty), (chunk & 1) ^ 1, wc)) { ok = false; break; }
            // orders PV after the softmax warps' rescale of O^T (tcgen05.st) -- once per step: a
            // tcgen05 fence in the issue stream drains the MMA pipe, so none sits before
            // operands that only TMA or shared-memory stores produced
            tc_fence_after();
            // FP8 stages hold zeros for tokens outside the request (written by the dequant warps)
            const bool tail = !FP8 && !SPARSE && is_tail(c0, c1, t, L);
            for (int m = 0; ok && m < 2; ++m) {
              for (int blk = 0; blk < 2; ++blk) {
                uint32_t s;
                if (!next_slot(s)) { ok = false; break; }
                if (tail) {
                  if (!warp_all_wait(bar(kBarZFull + s), (zpar >> s) & 1u, wc)) { ok = false; break; }
                  zpar ^= 1u << s;
                }
                // half h = page 2 blk + h of the step (64 tokens x 128 dims, 64-dim boxes 8 KB apart)
                const uint64_t a0 = vdesc0 + static_cast<uint64_t>(s * (kSlotBytes >> 4));
                const uint64_t b0 = smem_desc(sP + 128 * blk * 128, kBoxBytes, 1024, kSwizzle128);
#pragma unroll
                for (int kt = 0; kt < 8; ++kt)
                  umma_bf16_pair_warp(tmem + kColO + 128u * m,
                                      a0 + static_cast<uint64_t>(((kt >> 2) * kHalfBytes + 2048 * (kt & 3)) >> 4),
                                      b0 + static_cast<uint64_t>((16 * kt * 128) >> 4), kIdescPV,
                                      (t == 0 && blk == 0 && kt == 0) ? 0u : 1u);
                umma_commit_pair_mc_warp(bar(kBarSlotEmpty + s), 0x3);
              }
            }
            if (!ok) break;
            umma_commit_pair_mc_warp(bar(kBarPEmpty), 0x3);
            ++up;
          }
        }
        if (!ok) break;
        umma_commit_pair_mc_warp(bar(kBarOFull), 0x3);
        ++chunk;
      }
      // every pair MMA is complete before tensor memory is released
      umma_commit_pair_warp(bar(kBarDrain));
      drain_wait(bar(kBarDrain), 0);
    }
  } else if (SPARSE && warp == kWarpIndex) {
    // ======================= row lookups (token-sparse): one warp =======================
    // For every pair step, ahead of the gather warps, the cache rows of the 256 list slots of its
    // two blocks: lane l takes slots 4l .. 4l + 3 of each.  A slot names a key iff it is inside
    // the list and holds a position in [0, L); its row is then page(position / 64) * 64 +
    // position % 64 (or the position itself in a contiguous cache), else -1.
    int32_t* row_tab = reinterpret_cast<int32_t*>(misc + kMiscRowTab);
    uint32_t st = 0;
    bool ok = true;
    ChunkWalk walk(p, part);
    int b, c0, c1, split;
    while (ok && walk.next(p, b, c0, c1, split)) {
      const int breal = b / p.vq;
      const int L = p.cache_seqlens ? p.cache_seqlens[breal] : p.kv_len;
      const int32_t* bt = p.block_table ? p.block_table + static_cast<long long>(breal) * p.max_blocks : nullptr;
      const int32_t* ind = p.indices + static_cast<long long>(b) * p.topk;
      const int n = (c1 - c0 + 1) / 2;
      for (int t = 0; t < n; ++t, ++st) {
        if (!(ok = warp_all_wait(bar(kBarRowEmpty + st % kRowSlots), ((st / kRowSlots) & 1u) ^ 1u, wc))) break;
        int r[8];
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          const int kb = c0 + 2 * t + (q >> 2);
          const int pos = kb * kBlockTokens + 4 * lane + (q & 3);
          r[q] = (kb < c1 && pos < p.topk) ? ind[pos] : -1;
        }
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          const int idx = r[q];
          r[q] = (idx >= 0 && idx < L) ? (bt ? bt[idx >> 6] * kPage + (idx & (kPage - 1)) : idx) : -1;
        }
        int4* tab = reinterpret_cast<int4*>(row_tab + (st % kRowSlots) * 256 + 4 * lane);
        tab[0] = make_int4(r[0], r[1], r[2], r[3]);
        tab[32] = make_int4(r[4], r[5], r[6], r[7]);
        mbar_arrive(bar(kBarRowFull + st % kRowSlots));
      }
    }
  } else if (SPARSE && warp > kWarpIndex) {
    // ======================= gather warps (token-sparse, 11-15) ======================
    // They copy the stages in the fill order with 16-byte cp.async from the rows of the step's
    // table (two or four token rows per warp instruction, every fifth instruction per warp, zeros
    // for empty slots).  Each lane's arrival on the CTA's gather barrier completes a stage once
    // all its copies landed; the producer thread forwards that to the leader.
    const int gw = warp - kWarpIndex - 1;  // 0..4
    const int32_t* row_tab = reinterpret_cast<const int32_t*>(misc + kMiscRowTab);
    const char* kvb = static_cast<const char*>(p.kv);
    uint32_t g = 0, rf = 0;
    uint32_t steps = 0;  // row tables taken before this chunk
    bool ok = true;
    ChunkWalk walk(p, part);
    int b, c0, c1, split;
    // the 128 rows of table entries tab.. as natoms 64-dim columns from dims0: row i at
    // dst + (i / 64) * pstride + (i % 64) * 128, column a at + a * hstride
    // (all of this warp's table reads first, then its copies back to back)
    auto copy = [&](uint32_t dst, const int32_t* tab, int dims0, auto natoms_c, uint32_t pstride, uint32_t hstride) {
      constexpr int kCpr = 8 * decltype(natoms_c)::value, kRpi = 32 / kCpr, kInst = kBlockTokens / kRpi;
      constexpr int kPerWarp = (kInst + kGatherWarps - 1) / kGatherWarps;
      const int sub = lane / kCpr, c = lane % kCpr;
      const uint32_t a = static_cast<uint32_t>(c >> 3), cc = static_cast<uint32_t>(c & 7);
      const char* src0 = kvb + (dims0 + 8 * c) * 2;
      int row[kPerWarp];
#pragma unroll
      for (int k = 0; k < kPerWarp; ++k) {
        const int it = gw + k * kGatherWarps;
        row[k] = it < kInst ? tab[it * kRpi + sub] : -1;
      }
#pragma unroll
      for (int k = 0; k < kPerWarp; ++k) {
        const int it = gw + k * kGatherWarps;
        if (it < kInst) {
          const uint32_t i = static_cast<uint32_t>(it * kRpi + sub);
          cp_async_16(dst + (i >> 6) * pstride + (i & 63u) * 128u + a * hstride + ((cc ^ (i & 7u)) << 4),
                      src0 + (row[k] >= 0 ? static_cast<long long>(row[k]) * (kDqk * 2) : 0), row[k] >= 0 ? 16u : 0u);
        }
      }
    };
    auto stage = [&](const int32_t* tab, int dims0, uint32_t pstride, uint32_t hstride) -> bool {
      const uint32_t s = g % kNumSlots, use = g / kNumSlots;
      if (!warp_all_wait(bar(kBarSlotEmpty + s), (use & 1u) ^ 1u, wc)) return false;
      copy(sSlots + s * kSlotBytes, tab, dims0, std::integral_constant<int, 2>{}, pstride, hstride);
      cp_async_arrive_noinc(bar(kBarGather + s));
      ++g;
      return true;
    };
    while (ok && walk.next(p, b, c0, c1, split)) {
      const int n = (c1 - c0 + 1) / 2;
      for (int e = 0; ok && e < 2 * n; ++e) {
        bool is_v;
        int t;
        order_at(e, n, is_v, t);
        const uint32_t st = steps + static_cast<uint32_t>(t);
        const int32_t* tab = row_tab + (st % kRowSlots) * 256;  // [block a: 128][block b: 128]
        if (!is_v) {
          // K(t): this CTA's block c0 + 2t + rank; the step's table is new here.  Its RoPE dims
          // first ([page][64 rows][64 dims]), then K stage j: dims 128j.. as
          // [dim half][page][64 rows][64 dims]
          if (!(ok = warp_all_wait(bar(kBarRowFull + st % kRowSlots), (st / kRowSlots) & 1u, wc))) break;
          const int32_t* kt = tab + 128 * static_cast<int>(rank);
          if (!(ok = warp_all_wait(bar(kBarRopeEmpty), (rf & 1u) ^ 1u, wc))) break;
          copy(sRope, kt, kDv, std::integral_constant<int, 1>{}, kBoxBytes, 0);
          cp_async_arrive_noinc(bar(kBarGatherRope));
          ++rf;
          for (int j = 0; ok && j < kKFills; ++j) ok = stage(kt, 128 * j, kBoxBytes, kHalfBytes);
        } else {
          // V stage k = (m, blk): dims 256m + 128 rank.. of block blk as [page][dim half][64 rows]
          for (int k = 0; ok && k < kVFills; ++k)
            ok = stage(tab + 128 * (k & 1), 256 * (k >> 1) + 128 * static_cast<int>(rank), kHalfBytes, kBoxBytes);
          if (ok) mbar_arrive(bar(kBarRowEmpty + st % kRowSlots));  // this lane has read the table
        }
      }
      steps += static_cast<uint32_t>(n);
    }
    cp_async_wait_all();  // this lane's copies have landed before the CTA may exit
  } else if (FP8 && warp >= kWarpDequant) {
    // =========================== FP8 dequant (warps 10-13) ===========================
    // Thread dt owns token row dt % 64 of page dt / 64 of each stage.  Order: per chunk the Q
    // tile, then the stages in the fill order, each K step preceded by its RoPE slot.
    if (warp < kWarpDequant + kDequantThreads / 32) {
    const int dt = threadIdx.x - kWarpDequant * 32;  // 0..127
    uint32_t g = 0;   // stages written
    uint32_t gr = 0;  // raw fills consumed
    uint32_t qc = 0, rc = 0;
    int last_use[kMaxSlots];
    for (int i = 0; i < kMaxSlots; ++i) last_use[i] = -1;
    bool ok = true;
    // largest |bf16| bit pattern seen by to_f16 in each 16-bit half, and whether a scale let
    // code * scale leave the f16 range: reported as a status bit at the end
    uint32_t mag = 0;
    bool scale_range = false;
    // bf16 -> f16 in place over `bytes` of shared memory at `base`; the magnitudes of the first
    // `checked` 16-byte chunks enter the range check (RoPE slots: the rows of tokens that exist,
    // 8 chunks per token row; page tails hold undefined data that never reaches a result)
    auto to_f16 = [&](uint32_t base, int bytes, int checked) {
      for (int c = dt; c < bytes / 16; c += kDequantThreads) {
        uint32_t w0, w1, w2, w3;
        asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];" : "=r"(w0), "=r"(w1), "=r"(w2), "=r"(w3)
                     : "r"(base + 16u * c));
        if (c < checked) {
          mag = __vmaxu2(mag, __vmaxu2(w0 & 0x7FFF7FFFu, w1 & 0x7FFF7FFFu));
          mag = __vmaxu2(mag, __vmaxu2(w2 & 0x7FFF7FFFu, w3 & 0x7FFF7FFFu));
        }
        st_shared_v4(base + 16u * c, bf16x2_to_f16x2(w0), bf16x2_to_f16x2(w1), bf16x2_to_f16x2(w2),
                     bf16x2_to_f16x2(w3));
      }
    };
    // publish this warp's f16 data to the leader's MMA (each dequant warp of both CTAs arrives)
    auto publish = [&](int b) -> bool {
      fence_proxy_async_smem();
      __syncwarp();
      if (!ok) return false;
      if (lane == 0) mbar_arrive_remote(lead(bar(b)));
      return true;
    };
    // one stage: kind V (else K), token block tb of the step, scale group grp; page p of the
    // stage lands at +p * pstride, dim half h at +h * hstride
    auto stage = [&](int tb, int c1, int L, int grp, uint32_t pstride, uint32_t hstride) -> bool {
      const uint32_t s = g % kNumSlots;
      const uint32_t use = g / kNumSlots;
      const uint32_t r = gr % kNumRaw;
      ok &= warp_all_wait(bar(kBarRawFull + r), (gr / kNumRaw) & 1u, wc);
      ok &= warp_all_wait(bar(kBarSlotEmpty + s), (use & 1u) ^ 1u, wc);
      if (ok) {
        const uint32_t raw = sRaw + r * kRawBytes;
        const uint32_t pg = static_cast<uint32_t>(dt) >> 6, i = static_cast<uint32_t>(dt) & 63u;
        const uint32_t dst = sSlots + s * kSlotBytes + pg * pstride + i * 128u;
        const int tok = tb * kBlockTokens + dt;  // page pg, row i
        if (tb < c1 && tok < L) {
          float scale;
          asm volatile("ld.shared.f32 %0, [%1];" : "=f"(scale)
                       : "r"(raw + kRawCodeBytes + pg * (kRawScaleBytes / 2) + i * 16u + 4u * grp));
          // 448 * scale must stay within f16 (a quantiser's scale is max|x| / 448, so this is
          // exactly the condition that the largest value of the group fits)
          scale_range |= !(scale <= kF16MaxScale);
          dequant_row(raw + pg * (kRawCodeBytes / 2) + i * 128u, dst, hstride, i, scale);
        } else {
          // tokens outside the request or the chunk: zeros (masked in S^T, 0 rows of V)
#pragma unroll
          for (int h = 0; h < 2; ++h)
#pragma unroll
            for (int q = 0; q < 8; ++q) st_shared_v4(dst + h * hstride + 16u * q, 0u, 0u, 0u, 0u);
        }
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (!ok) return false;
      if (lane == 0) {
        mbar_arrive(bar(kBarRawEmpty + r));
        mbar_arrive_remote(lead(bar(kBarSlotFull + s)));
      }
      last_use[s] = static_cast<int>(use);
      ++g;
      ++gr;
      return true;
    };
    ChunkWalk walk(p, part);
    int b, c0, c1, split;
    while (ok && walk.next(p, b, c0, c1, split)) {
      const int L = p.cache_seqlens[b];
      const int n = (c1 - c0 + 1) / 2;
      ok &= warp_all_wait(bar(kBarQFull), qc & 1u, wc);
      if (ok) to_f16(sQ, kQBytes, kQBytes / 16);
      ++qc;
      if (!publish(kBarQReady)) break;
      for (int e = 0; ok && e < 2 * n; ++e) {
        bool is_v;
        int t;
        order_at(e, n, is_v, t);
        if (!is_v) {
          ok &= warp_all_wait(bar(kBarRopeFull), rc & 1u, wc);
          if (ok) {
            // this CTA's block of the step: its tokens below the chunk end and the request length
            const int tb = c0 + 2 * t + static_cast<int>(rank);
            const int valid = tb < c1 ? min(kBlockTokens, max(0, L - tb * kBlockTokens)) : 0;
            to_f16(sRope, kRopeBytes, valid * 8);
          }
          ++rc;
          if (!publish(kBarRopeReady)) { ok = false; break; }
          // K(t) stage j: dims 128j.. of this CTA's block; [dim half][page][64 tokens][64 dims]
          for (int j = 0; ok && j < kKFills; ++j)
            ok = stage(c0 + 2 * t + static_cast<int>(rank), c1, L, j, kBoxBytes, kHalfBytes);
        } else {
          // V(t) stage (m, blk): dims 256m + 128 rank.. of block c0 + 2t + blk; [page][dim half][..]
          for (int k = 0; ok && k < kVFills; ++k)
            ok = stage(c0 + 2 * t + (k & 1), c1, L, 2 * (k >> 1) + static_cast<int>(rank), kHalfBytes, kBoxBytes);
        }
      }
    }
    if (!*abort_flag && lane == 0)
      // the last pair commits on this CTA's stage barriers have landed before it may exit
      for (int s = 0; s < kNumSlots; ++s)
        if (last_use[s] >= 0) drain_wait(bar(kBarSlotEmpty + s), static_cast<uint32_t>(last_use[s]) & 1u);
    // a bf16 value of q or of a RoPE dim of magnitude >= 65536 (0x4780) is infinite in f16
    const bool range_bad = scale_range || (mag & 0xFFFFu) >= 0x4780u || (mag >> 16) >= 0x4780u;
    if (__any_sync(0xffffffffu, range_bad) && lane == 0 && p.status) atomicOr(p.status, kStatusF16Range);
    __syncwarp();
    }
  } else {
    // ============================ softmax + epilogue ==============================
    // Warp w reads TMEM lane quadrant qd = w % 4 (tokens 32qd..32qd+31 of this CTA's block, or
    // output dims of O^T) and column half h = w / 4 (query rows 64h..64h+63 of S^T; O^T block m = h).
    // Threads 0..127 also own one query row each for the running max and the row sums.
    const int tid = threadIdx.x;  // 0..255
    const int qd = warp & 3;
    const int h = warp >> 2;
    const int tl = 32 * qd + lane;  // token lane of S^T, dim lane of O^T
    const uint32_t lane_base = static_cast<uint32_t>(32 * qd) << 16;
    const float NEG_INF = -CUDART_INF_F;
    float m_ref = NEG_INF;  // row tid (tid < 128): reference max, log2 units
    float lsum[2] = {0.f, 0.f};
    uint32_t u = 0;
    uint32_t gchunk = 0;
    uint32_t zlpar = 0;  // parity of each slot's next ZLocal phase
    int chunk = 0;
    bool fail = false;
    const int R = p.rows;
    const int row0 = rg * kRows;
    ChunkWalk walk(p, part);
    int b, c0, c1, split;
    while (walk.next(p, b, c0, c1, split)) {
      // token-sparse: b is the query position (b / vq, b % vq) of a request of length L
      const int L = !SPARSE ? p.cache_seqlens[b] : (p.cache_seqlens ? p.cache_seqlens[b / p.vq] : p.kv_len);
      const int n = (c1 - c0 + 1) / 2;
      const bool single = (p.num_splits[b + 1] - p.num_splits[b]) == 1;
      bool aborted = false;
      for (int t = 0; t < n; ++t) {
        const int kb = c0 + 2 * t + static_cast<int>(rank);
        const int j = kb * kBlockTokens + tl;
        // token-sparse: the position in list slot j, read before the wait for S hides its latency
        const int sidx = (SPARSE && kb < c1 && j < p.topk) ? p.indices[static_cast<long long>(b) * p.topk + j] : -1;
        const int sb = static_cast<int>(u & 1u);
        bool ok = warp_all_wait(bar(kBarSFull + sb), (u >> 1) & 1u, wc);
        float x[64];
        tc_fence_after();
#pragma unroll
        for (int c = 0; c < 64; c += 16) tmem_ld16(tmem + lane_base + kColS + 128u * sb + 64u * h + c, x + c);
        tmem_wait_ld();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive_remote(lead(bar(kBarSEmpty + sb)));
        // key j is visible to row r iff j < L, its block is in this chunk and, when causal,
        // j <= L - s_q + r / h_q, i.e. r >= (j - L + s_q) * h_q
        int cmin = -(1 << 30);
        if constexpr (SPARSE) {
          // slot j of the list is a key iff it names a position in [0, L)
          if (sidx < 0 || sidx >= L) cmin = 1 << 30;
        } else {
          if (p.causal) {
            const int i0 = j - L + p.s_q;
            if (i0 > 0) cmin = i0 * p.h_q - row0 - 64 * h;
          }
          if (kb >= c1 || j >= L) cmin = 1 << 30;
        }
        // raw scores: the scale is applied in the exponent (ex2(S * scale - m)) and to the block
        // maxima; the mask pass runs only when one of the warp's tokens is masked
        if (__any_sync(0xffffffffu, cmin > -(1 << 30))) {
#pragma unroll
          for (int c = 0; c < 64; ++c) x[c] = (c >= cmin) ? x[c] : NEG_INF;
        }
        // column maxima over this warp's 32 tokens; lane l keeps columns l and 32 + l
        float k0 = NEG_INF, k1 = NEG_INF;
#pragma unroll
        for (int c = 0; c < 32; ++c) {
          const float m0 = warp_max_f32(x[c]);
          const float m1 = warp_max_f32(x[32 + c]);
          k0 = (lane == c) ? m0 : k0;
          k1 = (lane == c) ? m1 : k1;
        }
        red[qd * kRows + 64 * h + lane] = k0;
        red[qd * kRows + 64 * h + 32 + lane] = k1;
        if (named_bar_any(1, kSoftmaxThreads, !ok || fail)) { aborted = true; break; }
        bool need = false;
        if (tid < kRows) {
          // block max of row tid over this CTA's tokens, then over the pair's
          const float bm_own =
              fmaxf(fmaxf(red[tid], red[kRows + tid]), fmaxf(red[2 * kRows + tid], red[3 * kRows + tid])) *
              p.scale_log2;
          const uint32_t xb = u & 1u;
          st_async_f32(other(sMisc + kMiscXMax + 4u * (xb * kRows + tid)), bm_own, other(bar(kBarMaxFull + xb)));
          if (tid == 0) mbar_arrive_expect_tx(bar(kBarMaxFull + xb), 4u * kRows);
          ok &= pwait(bar(kBarMaxFull + xb), (u >> 1) & 1u, wc);
          const float bm = fmaxf(bm_own, xmax[xb * kRows + tid]);
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
        const bool rescale = named_bar_any(1, kSoftmaxThreads, need);
#pragma unroll
        for (int c = 0; c < 64; c += 4) {
          const float4 m4 = *reinterpret_cast<const float4*>(m_sm + 64 * h + c);
          x[c + 0] = ex2(fmaf(x[c + 0], p.scale_log2, -m4.x));
          x[c + 1] = ex2(fmaf(x[c + 1], p.scale_log2, -m4.y));
          x[c + 2] = ex2(fmaf(x[c + 2], p.scale_log2, -m4.z));
          x[c + 3] = ex2(fmaf(x[c + 3], p.scale_log2, -m4.w));
        }
        {
          float v[64];
#pragma unroll
          for (int c = 0; c < 64; ++c) v[c] = x[c];
          reduce_scatter64_sum(v, lane);  // lane l: columns 2l, 2l + 1
#pragma unroll
          for (int i = 0; i < 2; ++i) lsum[i] = lsum[i] * alpha_sm[64 * h + 2 * lane + i] + v[i];
        }
        // P^T of step u - 1 has been read (and O^T is final for it) once PEmpty flips
        if (u >= 1) ok &= warp_all_wait(bar(kBarPEmpty), (u - 1) & 1u, wc);
        if (rescale) {
          tc_fence_after();
#pragma unroll
          for (int c = 0; c < kRows; c += 16) {
            float o[16];
            const uint32_t ta = tmem + lane_base + kColO + 128u * h + c;
            tmem_ld16(ta, o);
            tmem_wait_ld();
#pragma unroll
            for (int e = 0; e < 16; ++e) o[e] *= alpha_sm[c + e];
            tmem_st16(ta, o);
          }
          tmem_wait_st();
        }
        // this token's P^T row for query rows 64h..64h+63 goes to CTA h's half of P^T
        const uint32_t T = rank * 128u + static_cast<uint32_t>(tl);
        const bool local = static_cast<uint32_t>(h) == rank;
#pragma unroll
        for (int q8 = 0; q8 < 8; ++q8) {
          const uint32_t off = T * 128u + ((static_cast<uint32_t>(q8) ^ (T & 7u)) << 4);
          const float* xs = x + 8 * q8;
          uint32_t w0, w1, w2, w3;
          if (FP8) {
            w0 = pack_f16x2(xs[0], xs[1]), w1 = pack_f16x2(xs[2], xs[3]);
            w2 = pack_f16x2(xs[4], xs[5]), w3 = pack_f16x2(xs[6], xs[7]);
          } else {
            w0 = pack_bf16x2(xs[0], xs[1]), w1 = pack_bf16x2(xs[2], xs[3]);
            w2 = pack_bf16x2(xs[4], xs[5]), w3 = pack_bf16x2(xs[6], xs[7]);
          }
          if (local) st_shared_v4(sP + off, w0, w1, w2, w3);
          else st_async_v4(other(sP + off), w0, w1, w2, w3, other(bar(kBarPRecv)));
        }
        if (local) {
          // this CTA's half of P^T: own rows written here, the peer's rows by st.async (PRecv)
          fence_proxy_async_smem();
          tc_fence_before();
          __syncwarp();
          if (lane == 0 && qd == 0) mbar_arrive_expect_tx(bar(kBarPRecv), 16384u);
          const bool okp = warp_all_wait(bar(kBarPRecv), u & 1u, wc);
          fence_proxy_async_smem();
          if (lane == 0) mbar_arrive_remote(lead(bar(kBarPFull)));
          ok &= okp;
        }
        if (!FP8 && !SPARSE && tid < kRows && is_tail(c0, c1, t, L)) {
          // Zero, in this CTA's V slots of the step, the rows of tokens outside the request or the
          // chunk (stale ring contents or the cache's unused page tail: 0 * NaN would poison O^T).
          // These slots count their bytes on this CTA's own barrier; both CTAs then arrive on the
          // leader's ZFull, which the MMA waits for before it reads the slot.
          const int r = tid & 63, h = tid >> 6;  // row r of page h of the stage's token block
          for (int k = 0; k < kVFills; ++k) {
            const uint32_t gv = gchunk + fills_before_v(t, n) + static_cast<uint32_t>(k);
            const uint32_t s = gv % kNumSlots;
            ok &= warp_all_wait(bar(kBarZLocal + s), (zlpar >> s) & 1u, wc);
            zlpar ^= 1u << s;
            const int blk = k & 1;  // stages go (m = 0, blk 0), (0, 1), (1, 0), (1, 1)
            const int jj = (c0 + 2 * t + blk) * kBlockTokens + 64 * h + r;
            if ((c0 + 2 * t + blk >= c1) || jj >= L) {
              const uint32_t row = sSlots + s * kSlotBytes + static_cast<uint32_t>(h * kHalfBytes + r * 128);
#pragma unroll
              for (int c = 0; c < 8; ++c) {
                st_shared_v4(row + 16u * c, 0u, 0u, 0u, 0u);
                st_shared_v4(row + kBoxBytes + 16u * c, 0u, 0u, 0u, 0u);
              }
            }
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive_remote(lead(bar(kBarZFull + s)));
          }
        }
        fail |= !ok;
        ++u;
      }
      if (aborted) break;
      // ------------------------------- epilogue ---------------------------------
#pragma unroll
      for (int i = 0; i < 2; ++i) red[qd * kRows + 64 * h + 2 * lane + i] = lsum[i];
      if (named_bar_any(1, kSoftmaxThreads, fail)) break;
      bool ok = true;
      if (tid < kRows) {
        const float l_own = red[tid] + red[kRows + tid] + red[2 * kRows + tid] + red[3 * kRows + tid];
        st_async_f32(other(sMisc + kMiscXL + 4u * tid), l_own, other(bar(kBarLFull)));
        if (tid == 0) mbar_arrive_expect_tx(bar(kBarLFull), 4u * kRows);
        ok = pwait(bar(kBarLFull), chunk & 1, wc);
        const float l = l_own + xl[tid];
        const int row = row0 + tid;
        const float lse_val = l > 0.f ? (m_ref + log2f(l)) * kLn2 : NEG_INF;
        inv_sm[tid] = l > 0.f ? 1.f / l : 0.f;
        if (leader && row < R) {
          if (single && SPARSE)  // query position (b / vq, b % vq), head row
            p.lse[(static_cast<long long>(b / p.vq) * p.h_q + row) * p.vq + b % p.vq] = lse_val;
          else if (single)
            p.lse[(static_cast<long long>(b) * p.h_q + row % p.h_q) * p.s_q + row / p.h_q] = lse_val;
          else
            p.lse_part[static_cast<long long>(split) * R + row] = lse_val;
        }
        m_ref = NEG_INF;
      }
      lsum[0] = lsum[1] = 0.f;
      named_bar_sync(1, kSoftmaxThreads);
      ok &= warp_all_wait(bar(kBarOFull), chunk & 1, wc);
      fail |= !ok;
      tc_fence_after();
      {
        // O^T block h of this CTA: dim = lane's output dim, columns = query rows.  The tensor
        // memory is released (OEmpty) as soon as the last load has landed.  Each group of 32
        // rows goes out through the P^T buffer (free once the chunk's last PV has completed):
        // the softmax warps write it as [dim half][32 rows][128 dims], then a TMA tensor store
        // per half writes it out (rows past the request's end fall outside the map).
        // Plain stores from these warps took several times longer (they queue behind the
        // traffic of the stage copies on the load/store path), and so did one bulk copy per row.
        const uint32_t sStage = sP;
        float* stage_f = reinterpret_cast<float*>(smem + kOffP);
        // thread 0 stores dim half 0, thread 32 (another warp) dim half 1; FP8: thread 0 both
        // (the second issuer's registers cost the FP8 kernel more than it gains)
        const int issuer = tid == 0 ? 0 : (!FP8 && tid == 32 ? 1 : -1);
        __nv_bfloat16* stage_h = reinterpret_cast<__nv_bfloat16*>(smem + kOffP);
#pragma unroll 1
        for (int c = 0; c < kRows; c += 32) {
          float o[32];
          tmem_ld16(tmem + lane_base + kColO + 128u * h + c, o);
          tmem_ld16(tmem + lane_base + kColO + 128u * h + c + 16, o + 16);
          tmem_wait_ld();
          if (c + 32 == kRows) {
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive_remote(lead(bar(kBarOEmpty)));
          }
          if (c > 0) {
            // the previous group's stores have read the buffer
            if (issuer >= 0) bulk_wait_read_all();
            named_bar_sync(1, kSoftmaxThreads);
          }
          // the rows' 1 / l four at a time (one 16-byte load, the same for every lane)
#pragma unroll
          for (int e = 0; e < 32; e += 4) {
            const float4 iv = *reinterpret_cast<const float4*>(inv_sm + c + e);
            const float v[4] = {o[e] * iv.x, o[e + 1] * iv.y, o[e + 2] * iv.z, o[e + 3] * iv.w};
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              const int k = h * 4096 + (e + j) * 128 + tl;
              if (single)
                stage_h[k] = __float2bfloat16_rn(v[j]);
              else
                stage_f[k] = v[j];
            }
          }
          fence_proxy_async_smem();
          named_bar_sync(1, kSoftmaxThreads);
          if (issuer >= 0) {
            for (int hh = issuer; hh < 2; hh += FP8 ? 1 : 2) {
              const int d0 = 256 * hh + 128 * static_cast<int>(rank);
              if (single)
                tma_store_3d(&tm_out, sStage + hh * 8192u, d0, row0 + c, b);
              else
                tma_store_3d(&tm_opart, sStage + hh * 16384u, d0, row0 + c, split);
            }
            bulk_commit();
          }
        }
        // the buffer is P^T again from the next step on (a softmax barrier comes first)
        if (issuer >= 0) bulk_wait_read_all();
      }
      gchunk += static_cast<uint32_t>(kKFills + kVFills) * static_cast<uint32_t>(n);
      ++chunk;
    }
    // the last PEmpty commit on this CTA's barrier has landed before it may exit
    if (!*abort_flag && u >= 1 && lane == 0) drain_wait(bar(kBarPEmpty), (u - 1) & 1u);
    __syncwarp();
  }

  // ---------------------------------- exit ----------------------------------------
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();
  if (!FP8 && leader && warp == kWarpProducer && lane == 0 && *abort_flag) {
    // After an abort, complete on behalf of the CTA that stopped first the fills the other one
    // issued, and wait for every copy still in flight into either CTA (the follower's copies
    // count their bytes here).  The two producers are at most one ring apart.
    const uint32_t gf = *reinterpret_cast<volatile uint32_t*>(misc + kMiscPeerFills);
    const uint32_t qf = *reinterpret_cast<volatile uint32_t*>(misc + kMiscPeerQ);
    const uint32_t gmax = max(fills, gf);
    for (uint32_t k = gmax > static_cast<uint32_t>(kNumSlots) ? gmax - kNumSlots : 0u; k < gmax; ++k) {
      const uint32_t s = k % kNumSlots;
      if (k >= fills) mbar_arrive(bar(kBarSlotFull + s));
      if (k >= gf) mbar_arrive(bar(kBarSlotFull + s));
      drain_wait(bar(kBarSlotFull + s), (k / kNumSlots) & 1u);
    }
    const uint32_t ql = static_cast<uint32_t>(q_fills);
    const uint32_t qmax = max(ql, qf);
    if (qmax > 0) {
      const uint32_t k = qmax - 1;
      if (k >= ql) mbar_arrive(bar(kBarQFull));
      if (k >= qf) mbar_arrive(bar(kBarQFull));
      drain_wait(bar(kBarQFull), k & 1u);
    }
    const uint32_t rf = *reinterpret_cast<volatile uint32_t*>(misc + kMiscPeerRope);
    const uint32_t rl = static_cast<uint32_t>(rope_fills);
    const uint32_t rmax = max(rl, rf);
    if (rmax > 0) {
      const uint32_t k = rmax - 1;
      if (k >= rl) mbar_arrive(bar(kBarRopeFull));
      if (k >= rf) mbar_arrive(bar(kBarRopeFull));
      drain_wait(bar(kBarRopeFull), k & 1u);
    }
  }
  __syncthreads();
  cluster_sync_all();
  if (warp == kWarpMma) {
    tc_fence_after();
    tmem_dealloc_pair(tmem, kTmemCols);
  }
}

}  // namespace

template <bool FP8, bool SPARSE = false>
int launch_pair(const CUtensorMap& tm_q, const CUtensorMap& tm_kv, const CUtensorMap& tm_scale,
                const CUtensorMap& tm_rope, const OutMaps& om, const DecodeParams& p, cudaStream_t stream) {
  using C = PairCfg<FP8, SPARSE>;
  auto kern = mla_decode_pair_kernel<FP8, SPARSE>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemBytes);
  if (e != cudaSuccess) return static_cast<int>(e);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2 * p.num_sm_parts, p.row_groups, 1);
  cfg.blockDim = dim3(C::kThreads, 1, 1);
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
  e = cudaLaunchKernelEx(&cfg, kern, tm_q, tm_kv, tm_scale, tm_rope, om.o_part, om.out, p);
  return static_cast<int>(e);
}

int launch_decode_pair_bf16(const CUtensorMap& tm_q, const CUtensorMap& tm_kv, const OutMaps& om,
                            const DecodeParams& p, cudaStream_t stream) {
  return launch_pair<false>(tm_q, tm_kv, tm_kv, tm_kv, om, p, stream);
}

int launch_decode_pair_fp8(const CUtensorMap& tm_q, const CUtensorMap& tm_codes, const CUtensorMap& tm_scale,
                           const CUtensorMap& tm_rope, const OutMaps& om, const DecodeParams& p,
                           cudaStream_t stream) {
  return launch_pair<true>(tm_q, tm_codes, tm_scale, tm_rope, om, p, stream);
}

int launch_decode_pair_sparse_bf16(const CUtensorMap& tm_q, const OutMaps& om, const DecodeParams& p,
                                   cudaStream_t stream) {
  return launch_pair<false, true>(tm_q, tm_q, tm_q, tm_q, om, p, stream);
}

}  // namespace mla

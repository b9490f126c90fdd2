// Absorbed MLA decode of query groups over the latent cache on tcgen05 tensor cores (sm_100a), one
// CTA pair per tile stream ("DeepSeek-V3.2-Exp - Absorb key weights", decode excerpt: scores =
// scale (q~ . c^KV_t + q^R . k^R_t), softmax over positions, ctx = sum alpha c^KV_t).  It serves
// mla_decode_absorb_multi: T new tokens per sequence, each token a query group over the rows it may
// see (t <= length - T + s), reading the shared cache rows of its sequence.
//
// Design (a thread-block cluster of 2 CTAs on two SMs; one wave of clusters):
// * Every MMA spans the pair (tcgen05 cta_group::2, M = 128 heads): CTA r supplies the query rows
//   of heads [64 r, 64 r + 64) and receives their results; the pair's tensor cores share the B
//   operand, so no partial score ever crosses between the CTAs.
// * A tile is 128 cached positions.  For the scores S = Q K^T (N = 128), CTA r loads the full
//   576-feature rows of positions [64 r, 64 r + 64) of the tile (8 latent slabs + 1 rotary slab of
//   64 positions x 64 features, 128-byte swizzle) and the hardware combines both halves of N.
// * For O += P V (N = 256 per instruction, two instructions cover the 512 latent features) the B
//   operand is split by columns: CTA r supplies latent features [128 c + 256 r, ...) of ALL 128
//   positions.  Its own positions' rows of those features are already in place (the latent slabs
//   of its half, reused as V exactly where the score MMA read them as K); the other 64 positions'
//   rows are brought from L2 (the peer just loaded them from HBM) into the slabs the score MMA no
//   longer needs.  HBM bytes stay at one read of the cache; 32 KB per tile and CTA come from L2.
// * TMEM (512 columns per CTA): O (64 heads x 512 features in the pair layout: 256 columns), one
//   score buffer of 64 columns, and query features [0, 384) as the A operand of the first 24 score
//   K-steps (192 columns, each head's row present in both lane halves).  A pair MMA of N = 128
//   reads its A operand from TMEM at well above the rate it reads it from shared memory, so only
//   query features [384, 576) come from shared memory.  The single score buffer costs little: the
//   softmax frees it as soon as it has read it, and the previous tile's P.V fills the gap.  P
//   (bf16) goes through shared memory.
// * Warp roles (per CTA): warp 0 TMA producer; warp 1 TMEM allocator and, in the even CTA, the
//   score-MMA issuer; warp 2 (even CTA) the P.V issuer; warp 3 the L2 reload of the peer rows;
//   warps 4..11 softmax (two per TMEM lane quadrant, 32 positions each), O rescale and epilogue.
// * Online softmax in base 2 with the scale folded in; the running maximum is raised (and O
//   rescaled in TMEM) only when it grows by more than 8.
// * Work split and split-KV merge as in the per-pair plan: sequences cut into chunks of tiles or
//   contiguous ranges over all tiles; the last cluster of a split sequence merges the partials in
//   the same launch (or every cluster merges a slice of the heads when there are many).
// * Every wait is bounded (global timer); on expiry the kernel records MLA_ERR_TIMEOUT and drains.
#include <cuda.h>
#include <cuda_bf16.h>
#include <math.h>
#include <string.h>

#include <atomic>
#include <chrono>

#include "common.cuh"
#include "kernels.h"
#include "sm100_ptx.cuh"
#include "tma_host.h"

namespace mla {
namespace decode_pair {

using namespace sm100;

constexpr int kNH = 128, kDC = 512, kDR = 64;
constexpr int kHeads = 64;                       // heads per CTA
constexpr int kTile = 128;                       // positions per pair tile
constexpr int kKeys = kTile / 2;                 // positions per CTA (the score MMA's N/2)
constexpr int kSlab = kKeys * 128;               // kKeys rows x 64 features (bf16), 128-byte rows
constexpr int kBox = 8192;                       // 64 rows x 64 features: query, P and output boxes
constexpr int kStageSlabs = 9;                   // 8 latent + 1 rotary
constexpr int kStageBytes = kStageSlabs * kSlab;
constexpr int kStages = 2;
constexpr int kKSteps = kTile / 16;              // P.V K-steps per tile
constexpr int kBlockSteps = kKeys / 16;          // P.V K-steps per CTA's block of positions
constexpr int kSCols = kKeys / 2;                // score columns per softmax thread
// (The pair MMA's N must be a multiple of 64 for the full rate: N = 96, 112 or 80 ran at less than
// half of it, so tiles of fewer positions, which would leave shared memory for a third stage, lose.)
constexpr int kQSlabs = 3;                       // query features 384..511 and the rotary 64
constexpr int kQTmemSteps = 24;                  // score K-steps whose query half comes from TMEM
constexpr int kQOff = kStages * kStageBytes;
constexpr int kPBytes = 2 * kBox;                // 64 heads x up to 128 positions (bf16), two K slabs
constexpr int kPOff = kQOff + kQSlabs * kBox;
constexpr int kSmemOff = kPOff + 2 * kPBytes;
constexpr int kMaxClusters = 160;                // partial-slot list capacity (2 slots per cluster)
constexpr int kMergeLastMax = 4;                 // up to this many partials the last cluster merges alone
constexpr int kProdWarp = 0, kQkWarp = 1, kPvWarp = 2, kReloadWarp = 3, kSmWarp0 = 4, kSmWarps = 8;
constexpr int kThreads = 32 * (kSmWarp0 + kSmWarps);
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColO = 0, kColS = 256, kColQ = 320;   // O 256, S 64, query features [0, 384) 192
constexpr float kRescaleThreshold = 8.0f;        // log2 units
constexpr uint64_t kWaitLimitNs = 1000000000ull;
constexpr int kPrefetch = 2;                     // L2 prefetch distance, tiles
constexpr uint32_t kFullBytes = 2u * kStageBytes;         // both CTAs' own-position rows
constexpr uint32_t kQBytes = 2u * kQSlabs * kBox;         // both CTAs' query slabs
constexpr uint32_t kReloadBytes = 4u * kSlab;              // the peer positions' rows of this CTA's half

struct Params {
  CUtensorMap tm_ckv;  // 3-D (d_c, n_max, B), box (64, 64, 1), 128-byte swizzle
  CUtensorMap tm_kr;   // 3-D (d_r, n_max, B), box (64, 64, 1), 128-byte swizzle
  CUtensorMap tm_q;    // 2-D (d_c, B * 128) rows of q~, box (64, 64), 128-byte swizzle
  CUtensorMap tm_qp;   // 2-D (d_r, B * 128) rows of q^R, box (64, 64), 128-byte swizzle
  CUtensorMap tm_ctx;  // 2-D (d_c, B * 128) rows of ctx, box (64, 64), 128-byte swizzle (stores)
  CUtensorMap tm_ws;   // 2-D (d_c, 2 n_clusters x 2 x 64) partial rows, box (64, 64), 128-byte swizzle
  const __nv_bfloat16* q_tilde;
  int64_t ldqt;
  const int32_t* lengths;       // [B / T] cached rows per cache sequence
  int B, n_max, n_clusters;     // B query rows groups (pseudo-sequences): T per cache sequence
  int slice_above;              // more partials than this: the sliced merge (needs every cluster resident)
  int T;                        // new tokens per cache sequence (1 for the one-token decode)
  float scale_log2;
  __nv_bfloat16* ctx;
  float* lse;
  __nv_bfloat16* ws_o;          // [2 n_clusters slots][2 CTAs][64 heads][512 features] bf16 partial
                                // contexts normalised by their own softmax sum
  float2* ws_ml;                // [2 n_clusters slots][2 CTAs][128] (running max in log2 units, sum)
  unsigned long long* ws_ctr;   // [B][2 CTAs] arrival counters: (epoch << 8) | arrivals
  unsigned long long* ws_ready; // [2 n_clusters slots][2 CTAs] partial published: the writer's epoch
  unsigned long long epoch;     // unique per launch, never 0, < 2^56
  int32_t* err;
};

struct Smem {
  uint64_t full[kStages], empty[kStages], qk_done[kStages], v_full[kStages];
  uint64_t s_full, s_empty, p_full[2], pv_done[2];
  uint64_t q_full, q_empty, o_free, drain;
  uint64_t last_bar, pub_bar, mrg_full, mrg_done;
  uint64_t red_bar[2][2];        // [score buffer][head group]: the four warps of a head group wrote red
  uint64_t lsum_bar[2];          // [head group]: the four warps of a head group wrote lsum
  uint64_t out_bar;              // every softmax warp staged (or stored) its output rows
  float red[2][4][kHeads];       // [score buffer][4 threads of a head][head] partial row max
  float lsum[4][kHeads];         // [4 threads of a head][head] partial softmax sum
  int16_t slots[kMaxClusters];   // partial slots of the sequence being merged
  uint32_t tmem_base;
  int abort;
  int lo, hi, b0, t_b0;  // tile range [lo, hi) in the global tile order, its first sequence and
                         // that sequence's first global tile
  int len0;              // length of sequence b0 (clamped), so the first segment needs no reload
  int chunk;             // > 0: chunked plan, every cluster holds <= chunk tiles of one sequence
  int item0, kb;         // chunked plan: first chunk of this cluster's sequence, its chunk count
  long long total;       // tiles of all sequences
  int bad;               // some length outside [1, n_max]
  int nslots, is_last;
};

__device__ __forceinline__ int clamp_len(int len, int n_max) { return len < 0 ? 0 : (len > n_max ? n_max : len); }
__device__ __forceinline__ int tiles_of(int len) { return (len + kTile - 1) / kTile; }
// Keys query group b attends (before clamping): token s of T new tokens of cache sequence b / T
// sees rows t <= lengths[b / T] - T + s, the causal rule among the new tokens.
__device__ __forceinline__ int raw_len(const Params& p, int b) {
  return p.T == 1 ? p.lengths[b] : p.lengths[b / p.T] - (p.T - 1 - b % p.T);
}
__device__ __forceinline__ int seq_tiles(const Params& p, int b) { return tiles_of(clamp_len(raw_len(p, b), p.n_max)); }

__device__ __forceinline__ int warp_sum_i(int v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}
__device__ __forceinline__ int warp_max_i(int v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = max(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

// bf16 halves of a packed pair, widened exactly to fp32 (low half = first element).
__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

__device__ __forceinline__ uint64_t policy_evict_normal() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_normal.b64 %0, 1.0;" : "=l"(p));
  return p;
}

// Contiguous tile range [lo, hi) of cluster c among n_clusters over all sequences' tiles.
__device__ __forceinline__ int range_lo(long long c, long long total, long long nc) { return (int)((c * total) / nc); }

// The cluster whose contiguous range holds global tile t (ranges of empty clusters are skipped).
__device__ __forceinline__ int cluster_of(long long t, long long total, long long nc) {
  long long c = (t * nc) / (total > 0 ? total : 1);
  if (c >= nc) c = nc - 1;
  while (c + 1 < nc && range_lo(c + 1, total, nc) <= t) ++c;
  while (c > 0 && range_lo(c, total, nc) > t) --c;
  return (int)c;
}

// Clamped lengths of the first 256 sequences stay in registers (lane l holds sequences l + 32 k);
// later ones are re-read from global memory.
constexpr int kPlanRegs = 8;
struct PlanTiles {
  int l[kPlanRegs];
  __device__ int len_at(const Params& p, int k, int lane) const {  // length of sequence 32 k + lane
    if (k < kPlanRegs) {
      int v = 0;
#pragma unroll
      for (int i = 0; i < kPlanRegs; ++i) v = (i == k) ? l[i] : v;
      return v;
    }
    const int b = 32 * k + lane;
    return b < p.B ? clamp_len(raw_len(p, b), p.n_max) : 0;
  }
  __device__ int at(const Params& p, int k, int lane) const { return tiles_of(len_at(p, k, lane)); }
};

// ceil(a / c) for 0 <= a, 1 <= c < 2^22, from a float reciprocal of c with one integer correction.
__device__ __forceinline__ int ceil_div_rc(int a, int c, float rc) {
  const int n = a + c - 1;
  int q = __float2int_rz((float)n * rc);
  if (q * c > n) --q;
  else if ((q + 1) * c <= n) ++q;
  return q;
}

// Chunks of the chunked plan with chunk size c: the sum over sequences of ceil(tiles / c).
__device__ int chunk_items(const Params& p, const PlanTiles& pt, int c, int lane) {
  int n = 0;
  const int nk = (p.B + 31) / 32;
  const float rc = 1.f / (float)c;
#pragma unroll
  for (int k = 0; k < kPlanRegs; ++k)
    if (k < nk) n += ceil_div_rc(tiles_of(pt.l[k]), c, rc);
  for (int k = kPlanRegs; k < nk; ++k) n += ceil_div_rc(pt.at(p, k, lane), c, rc);
  return warp_sum_i(n);
}

// One warp: the work split.  Chunked plan when every non-empty sequence can have clusters of its
// own and the smallest chunk that fits the clusters is within a quarter (or 4 tiles) of the
// balanced share; else equal contiguous ranges over the concatenated tiles of all sequences.
__device__ void plan_range(const Params& p, int c, Smem& sm, int lane) {
  PlanTiles pt;
  long long total = 0;
  int maxt = 0, mint = 1 << 30, nonempty = 0;
  bool bad = false;
  const int nk = (p.B + 31) / 32;
  for (int k = 0; k < nk; ++k) {
    const int b = 32 * k + lane;
    int t = 0, lc = 0;
    if (b < p.B) {
      const int len = raw_len(p, b);
      bad |= (len < 1 || len > p.n_max);
      lc = clamp_len(len, p.n_max);
      t = tiles_of(lc);
    }
#pragma unroll
    for (int i = 0; i < kPlanRegs; ++i)
      if (i == k) pt.l[i] = lc;
    maxt = max(maxt, t);
    if (t > 0) mint = min(mint, t);
    nonempty += t > 0 ? 1 : 0;
    total += t;
  }
#pragma unroll
  for (int i = 0; i < kPlanRegs; ++i)
    if (i >= nk) pt.l[i] = 0;
  maxt = warp_max_i(maxt);
  mint = -warp_max_i(-mint);
  nonempty = warp_sum_i(nonempty);
  {
    long long v = total;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    total = v;
  }
  const bool any_bad = __any_sync(0xffffffffu, bad);
  if (any_bad && lane == 0 && c == 0 && cluster_ctarank() == 0) raise_error(p.err, MLA_ERR_LENGTH);
  const long long nc = p.n_clusters;
  const int balanced = (int)((total + nc - 1) / nc);
  int chunk = 0;
  if (nonempty > 0 && nonempty <= nc) {
    int lo = max(1, min(balanced, maxt)), hi = maxt;
    if (mint == maxt) {
      const int q = (int)(nc / nonempty);
      lo = hi = (maxt + q - 1) / q;
    }
    while (lo < hi) {
      const int mid = (lo + hi) >> 1;
      if (chunk_items(p, pt, mid, lane) <= nc) hi = mid;
      else lo = mid + 1;
    }
    // One tile longer than the smallest fitting chunk: a split sequence's last chunk is then
    // shorter, so its cluster finishes first and publishes while the merging cluster still works.
    if (lo <= balanced + max(4, balanced / 4)) chunk = (lo > 1 && lo < maxt) ? lo + 1 : lo;
  }
  int lo = 0, hi = 0, first_b = p.B, t_first = 0, item0 = 0, kb = 0;
  if (chunk > 0) {
    int base_items = 0, base_tiles = 0;
    for (int k = 0; k < nk && first_b == p.B; ++k) {
      const int t = pt.at(p, k, lane);
      const int kc = (t + chunk - 1) / chunk;
      int ik = kc, it = t;  // inclusive prefix sums within the warp
      for (int o = 1; o < 32; o <<= 1) {
        const int vk = __shfl_up_sync(0xffffffffu, ik, o), vt = __shfl_up_sync(0xffffffffu, it, o);
        if (lane >= o) {
          ik += vk;
          it += vt;
        }
      }
      const unsigned m = __ballot_sync(0xffffffffu, kc > 0 && base_items + ik > c);
      if (m) {
        const int l0 = __ffs(m) - 1;
        const int kk = __shfl_sync(0xffffffffu, kc, l0), tt = __shfl_sync(0xffffffffu, t, l0);
        item0 = base_items + __shfl_sync(0xffffffffu, ik, l0) - kk;
        t_first = base_tiles + __shfl_sync(0xffffffffu, it, l0) - tt;
        first_b = 32 * k + l0;
        kb = kk;
        const int j = c - item0;
        lo = t_first + j * chunk;
        hi = t_first + min((j + 1) * chunk, tt);
      }
      base_items += __shfl_sync(0xffffffffu, ik, 31);
      base_tiles += __shfl_sync(0xffffffffu, it, 31);
    }
  } else {
    lo = range_lo(c, total, nc);
    hi = range_lo(c + 1, total, nc);
  }
  if (chunk == 0 && lo < hi) {
    int base = 0;  // tiles before batch b0
    for (int b0 = 0; b0 < p.B && first_b == p.B; b0 += 32) {
      const int b = b0 + lane;
      const int t = b < p.B ? seq_tiles(p, b) : 0;
      int inc = t;
      for (int o = 1; o < 32; o <<= 1) {
        const int v = __shfl_up_sync(0xffffffffu, inc, o);
        if (lane >= o) inc += v;
      }
      const bool hit = (b < p.B) && t > 0 && (base + inc > lo);
      const unsigned m = __ballot_sync(0xffffffffu, hit);
      if (m) {
        const int l0 = __ffs(m) - 1;
        first_b = b0 + l0;
        t_first = base + __shfl_sync(0xffffffffu, inc - t, l0);
      }
      base += __shfl_sync(0xffffffffu, inc, 31);
    }
  }
  // length of the first sequence, from the registers when it is among the first 256 (no second
  // round trip to global memory)
  int len0 = 0;
  if (first_b < p.B) len0 = __shfl_sync(0xffffffffu, pt.len_at(p, first_b >> 5, lane), first_b & 31);
  if (lane == 0) {
    sm.lo = lo;
    sm.hi = hi;
    sm.b0 = first_b;
    sm.t_b0 = t_first;
    sm.len0 = len0;
    sm.chunk = chunk;
    sm.item0 = item0;
    sm.kb = kb;
    sm.total = total;
    sm.bad = any_bad ? 1 : 0;
  }
}

// Walks the segments (sequence, first tile, end tile) of this cluster's range.
struct SegIter {
  int b, tb, t, hi, len0;
  bool first;
  const Params& p;
  __device__ SegIter(const Smem& sm, const Params& p_)
      : b(sm.b0), tb(sm.t_b0), t(sm.lo), hi(sm.hi), len0(sm.len0), first(true), p(p_) {}
  __device__ bool next(int& sb, int& begin, int& end, int& len, bool& whole, int& base) {
    while (t < hi && b < p.B) {
      len = first ? len0 : clamp_len(raw_len(p, b), p.n_max);
      first = false;
      const int nt = tiles_of(len);
      if (tb + nt <= t) {
        tb += nt;
        ++b;
        continue;
      }
      sb = b;
      base = tb;
      begin = t - tb;
      end = min(hi, tb + nt) - tb;
      whole = (begin == 0 && end == nt);
      t = tb + end;
      tb += nt;
      ++b;
      return true;
    }
    return false;
  }
};

// Partial slots of sequence b (first global tile `base`, nt tiles): slot 2c holds the partial of
// cluster c's first segment, slot 2c + 1 that of its last segment.
__device__ int list_slots(const Params& p, Smem& sm, int base, int nt) {
  int n = 0;
  if (sm.chunk > 0) {
    for (int k = 0; k < sm.kb && n < kMaxClusters; ++k) sm.slots[n++] = (int16_t)(2 * (sm.item0 + k));
  } else {
    const long long total = sm.total, nc = p.n_clusters;
    const int c0 = cluster_of(base, total, nc), c1 = cluster_of((long long)base + nt - 1, total, nc);
    for (int c = c0; c <= c1 && n < kMaxClusters; ++c) {
      const long long lo = range_lo(c, total, nc), hi = range_lo(c + 1, total, nc);
      if (hi > lo) sm.slots[n++] = (int16_t)(2 * c + (lo >= base ? 0 : 1));
    }
  }
  sm.nslots = n;
  return n;
}

// Counts this CTA's arrival for (sequence, CTA rank) and reports whether it was the last of
// `expected`.  The counter holds (epoch << 8) | arrivals; a value from another launch (another
// epoch, or the 0 the last arrival leaves behind) counts as no arrival, so the workspace needs no
// initialisation.
__device__ bool arrive_last(unsigned long long* ctr, unsigned long long epoch, int expected, int32_t* err) {
  unsigned long long cur = atomicCAS(ctr, 0ull, (epoch << 8) | 1ull);
  if (cur == 0ull || (cur >> 8) == epoch) {
    const unsigned long long now = cur == 0ull ? ((epoch << 8) | 1ull) : atomicAdd(ctr, 1ull) + 1ull;
    if ((int)(now & 255ull) < expected) return false;
    atomicExch(ctr, 0ull);
    return true;
  }
  for (int i = 0; i < 4096; ++i) {
    const unsigned long long base = (cur >> 8) == epoch ? cur : (epoch << 8);
    const unsigned long long next = base + 1;
    const unsigned long long prev = atomicCAS(ctr, cur, next);
    if (prev == cur) {
      if ((int)(next & 255ull) < expected) return false;
      atomicExch(ctr, 0ull);
      return true;
    }
    cur = prev;
  }
  raise_error(err, MLA_ERR_TIMEOUT);
  return false;
}

__device__ __forceinline__ void fail_timeout(Smem& sm, int32_t* err) {
  raise_error(err, MLA_ERR_TIMEOUT);
  sm.abort = 1;
}

__device__ __forceinline__ void st_release_gpu(unsigned long long* f, unsigned long long v) {
  asm volatile("st.release.gpu.global.u64 [%0], %1;" ::"l"(f), "l"(v) : "memory");
}

// Bounded wait until *f == want (acquire at GPU scope); false on abort or after kWaitLimitNs.
__device__ bool wait_flag(const unsigned long long* f, unsigned long long want, const volatile int* abort) {
  const uint64_t t0 = globaltimer();
  while (true) {
    unsigned long long v;
    asm volatile("ld.acquire.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(f) : "memory");
    if (v == want) return true;
    if (*abort) return false;
    if (globaltimer() - t0 > kWaitLimitNs) return false;
    __nanosleep(64);
  }
}

// Arrive on barrier `bar_local` of the even CTA (this CTA's own barrier when it is the even one).
__device__ __forceinline__ void arrive_leader(uint32_t bar_local, uint32_t rank) {
  if (rank == 0) mbar_arrive(bar_local);
  else mbar_arrive_remote_cta(mapa(bar_local, 0));
}

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
    decode_kernel(const __grid_constant__ Params p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  Smem& sm = *reinterpret_cast<Smem*>(smem + kSmemOff);
  volatile int* abort_flag = &sm.abort;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const bool leader = (rank == 0);
  const int cl = blockIdx.x >> 1;
  const uint32_t sbase = smem_u32(smem);

  // The up-projection launched after this kernel may start its weight loads on SMs this grid leaves
  // free; the threads that read the preceding kernel's output wait for it first (griddep_wait).
  griddep_launch_dependents();
  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(smem_u32(&sm.full[s]), 1);      // the even CTA's producer arrive.expect_tx + TMA bytes
      mbar_init(smem_u32(&sm.empty[s]), 1);     // P.V commit
      mbar_init(smem_u32(&sm.qk_done[s]), 1);   // score commit
      mbar_init(smem_u32(&sm.v_full[s]), 1);    // this CTA's reload: arrive.expect_tx + TMA bytes
    }
    mbar_init(smem_u32(&sm.s_full), 1);
    mbar_init(smem_u32(&sm.s_empty), 2 * kSmWarps);  // softmax warps of both CTAs
    for (int i = 0; i < 2; ++i) {
      mbar_init(smem_u32(&sm.p_full[i]), 2 * kSmWarps);
      mbar_init(smem_u32(&sm.pv_done[i]), 1);
    }
    mbar_init(smem_u32(&sm.q_full), 1 + 2 * kSmWarps);  // producer's expect_tx + both CTAs' TMEM query halves
    mbar_init(smem_u32(&sm.q_empty), 1);
    mbar_init(smem_u32(&sm.o_free), 2 * kSmWarps);
    mbar_init(smem_u32(&sm.drain), 2);                  // one commit from each MMA-issuing warp
    mbar_init(smem_u32(&sm.last_bar), 1);
    mbar_init(smem_u32(&sm.pub_bar), kSmWarps);
    mbar_init(smem_u32(&sm.mrg_full), 1);
    mbar_init(smem_u32(&sm.mrg_done), kSmWarps);
    mbar_init(smem_u32(&sm.out_bar), kSmWarps);
    for (int i = 0; i < 2; ++i) {
      mbar_init(smem_u32(&sm.red_bar[i][0]), 4);
      mbar_init(smem_u32(&sm.red_bar[i][1]), 4);
      mbar_init(smem_u32(&sm.lsum_bar[i]), 4);
    }
    sm.abort = 0;
    fence_mbar_init();
    prefetch_tensormap(&p.tm_ckv);
    prefetch_tensormap(&p.tm_kr);
    prefetch_tensormap(&p.tm_q);
    prefetch_tensormap(&p.tm_qp);
    prefetch_tensormap(&p.tm_ctx);
    prefetch_tensormap(&p.tm_ws);
  }
  if (warp == kProdWarp) plan_range(p, cl, sm, lane);
  if (warp == kQkWarp) {
    tmem_alloc_pair(smem_u32(&sm.tmem_base), kTmemCols);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  // Both CTAs' barriers and TMEM must exist before any cross-CTA arrive, TMA completion or MMA.
  cluster_sync();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;

  if (warp == kProdWarp) {
    // ------------------------------------------------------------------ TMA producer
    if (lane == 0) {
      const uint64_t pol = policy_evict_normal();
      const uint32_t full0 = mapa(smem_u32(&sm.full[0]), 0), qfull = mapa(smem_u32(&sm.q_full), 0);
      SegIter seg(sm, p);
      int b, begin, end, len, base;
      bool whole;
      uint32_t it = 0, nseg = 0;
      bool ok = true;
      while (ok && seg.next(b, begin, end, len, whole, base)) {
        // this CTA's 64 heads of the query, features 384..511 and the rotary 64, into shared memory;
        // the first segment's query is the preceding kernel's output, so its first cache tiles (no
        // dependency) are requested before waiting for that kernel
        auto load_q = [&]() {
          if (leader) mbar_arrive_expect_tx(smem_u32(&sm.q_full), kQBytes);
          const int qrow = b * kNH + kHeads * (int)rank;
#pragma unroll
          for (int j = 0; j < kQSlabs - 1; ++j)
            tma_load_2d_pair(sbase + kQOff + j * kBox, &p.tm_q, qfull, 2 * kQTmemSteps * 8 + 64 * j, qrow, pol);
          tma_load_2d_pair(sbase + kQOff + (kQSlabs - 1) * kBox, &p.tm_qp, qfull, 0, qrow, pol);
        };
        bool q_pending = true;
        if (nseg > 0) {
          if (!(mbar_test(smem_u32(&sm.q_empty), (nseg - 1) & 1u) ||
                mbar_wait(smem_u32(&sm.q_empty), (nseg - 1) & 1u, abort_flag, kWaitLimitNs))) {
            fail_timeout(sm, p.err);
            ok = false;
            break;
          }
          load_q();
          q_pending = false;
        }
        for (int i = begin; i < end && ok; ++i, ++it) {
          if (q_pending && i - begin == kStages) {
            griddep_wait();
            load_q();
            q_pending = false;
          }
          const uint32_t st = it % kStages, ph = (it / kStages) & 1u;
          const uint32_t eb = smem_u32(&sm.empty[st]);
          if (!(mbar_test(eb, ph ^ 1u) || mbar_wait(eb, ph ^ 1u, abort_flag, kWaitLimitNs))) {
            fail_timeout(sm, p.err);
            ok = false;
            break;
          }
          const uint32_t dst = sbase + st * kStageBytes;
          if (leader) mbar_arrive_expect_tx(smem_u32(&sm.full[st]), kFullBytes);
          const int y = i * kTile + kKeys * (int)rank, z = p.T == 1 ? b : b / p.T;
#pragma unroll
          for (int s2 = 0; s2 < 8; ++s2) tma_load_3d_pair(dst + s2 * kSlab, &p.tm_ckv, full0 + 8 * st, 64 * s2, y, z, pol);
          tma_load_3d_pair(dst + 8 * kSlab, &p.tm_kr, full0 + 8 * st, 0, y, z, pol);
          // this CTA's rows of the tile kPrefetch ahead go to L2 now: its shared-memory stage frees up
          // only after this tile's P.V, and the load then finds the rows in L2 instead of waiting on HBM.
          // (The first two tiles' prefetches are issued by the reload warp once the first tile has
          // landed: issued here, they would queue ahead of the other CTAs' first loads.)
          if (i >= begin + kStages && i + kPrefetch < end) {
            const int yp = (i + kPrefetch) * kTile + kKeys * (int)rank;
#pragma unroll
            for (int s = 0; s < 8; ++s) tma_prefetch_3d(&p.tm_ckv, 64 * s, yp, z);
            tma_prefetch_3d(&p.tm_kr, 0, yp, z);
          }
        }
        if (q_pending && ok) {
          griddep_wait();
          load_q();
        }
        ++nseg;
      }
      // every load issued must have landed before the CTA may exit: the last stages' P.V commits
      // (or a timeout) cover it
      for (uint32_t k = it > (uint32_t)kStages ? it - kStages : 0; k < it; ++k)
        mbar_wait(smem_u32(&sm.empty[k % kStages]), (k / kStages) & 1u, abort_flag, kWaitLimitNs);
    }
    __syncwarp();
    griddep_wait();
    // lengths outside [1, n_max] (an error already flagged): sequences left without tiles get a
    // zero context and lse = -inf from cluster 0, each CTA its 64 heads
    if (cl == 0 && sm.bad) {
      for (int b = 0; b < p.B; ++b) {
        if (seq_tiles(p, b) != 0) continue;
        for (int i = lane; i < kHeads * 64; i += 32)
          reinterpret_cast<uint4*>(p.ctx + ((int64_t)b * kNH + kHeads * rank + (i >> 6)) * kDC)[i & 63] =
              make_uint4(0, 0, 0, 0);
        if (p.lse != nullptr)
          for (int hh = lane; hh < kHeads; hh += 32) p.lse[(int64_t)b * kNH + kHeads * rank + hh] = -INFINITY;
      }
    }
  } else if (warp == kReloadWarp) {
    // ------------------------------------------------------------------ L2 reload of the peer rows
    // After the score MMA of tile t, slabs [4 (1 - r), 4 (1 - r) + 4) of the stage (this CTA's own
    // positions, latent features of the peer's half) are no longer needed here; they receive the
    // peer positions' rows of this CTA's half of the latent, the V operand of the other 64 positions.
    if (lane == 0) {
      const uint64_t pol = policy_evict_first();
      SegIter seg(sm, p);
      int b, begin, end, len, base;
      bool whole;
      uint32_t it = 0;
      bool ok = true;
      while (ok && seg.next(b, begin, end, len, whole, base)) {
        for (int i = begin; i < end && ok; ++i, ++it) {
          const uint32_t st = it % kStages, ph = (it / kStages) & 1u;
          const uint32_t qb = smem_u32(&sm.qk_done[st]);
          if (!(mbar_test(qb, ph) || mbar_wait(qb, ph, abort_flag, kWaitLimitNs))) {
            fail_timeout(sm, p.err);
            ok = false;
            break;
          }
          if (i == begin) {
            // the segment's first tile has landed: its next two tiles' rows go to L2 (see the producer)
            const int z = p.T == 1 ? b : b / p.T;
            for (int j = begin + kStages; j < begin + kStages + kPrefetch && j < end; ++j) {
              const int yp = j * kTile + kKeys * (int)rank;
#pragma unroll
              for (int s = 0; s < 8; ++s) tma_prefetch_3d(&p.tm_ckv, 64 * s, yp, z);
              tma_prefetch_3d(&p.tm_kr, 0, yp, z);
            }
          }
          const uint32_t vb = smem_u32(&sm.v_full[st]);
          mbar_arrive_expect_tx(vb, kReloadBytes);
          const uint32_t dst = sbase + st * kStageBytes + 4 * (1u - rank) * kSlab;
          const int y = i * kTile + kKeys * (int)(1u - rank), z = p.T == 1 ? b : b / p.T;
#pragma unroll
          for (int j = 0; j < 4; ++j) tma_load_3d(dst + j * kSlab, &p.tm_ckv, vb, 64 * (4 * (int)rank + j), y, z, pol);
          if (i == end - 1 && !whole) {
            // The segment's last tile is under way: count this cluster's arrival for the sequence now
            // (an atomic costs a microsecond when HBM is saturated; here it overlaps the tile's
            // softmax and P.V instead of delaying the epilogue).  With up to p.slice_above partials
            // (kMergeLastMax when the whole grid is resident, else any number) the last cluster to
            // arrive merges them all, so it must know; with more, every cluster merges a slice and
            // counts its arrival afterwards.  The epilogue of the previous segment has
            // finished reading the slot list (this segment's first score MMA needed its query).
            const int ns = list_slots(p, sm, base, tiles_of(len));
            sm.is_last = ns > p.slice_above ? 0 : (arrive_last(p.ws_ctr + 2 * (int64_t)b + rank, p.epoch, ns, p.err) ? 1 : 0);
            mbar_arrive(smem_u32(&sm.last_bar));
          }
        }
      }
      // the reloads must have landed before the CTA exits
      for (uint32_t k = it > (uint32_t)kStages ? it - kStages : 0; k < it; ++k)
        mbar_wait(smem_u32(&sm.v_full[k % kStages]), (k / kStages) & 1u, abort_flag, kWaitLimitNs);
    }
    __syncwarp();
  } else if (warp == kQkWarp || warp == kPvWarp) {
    // ------------------------------------------------------------------ MMA issuers (even CTA)
    const bool is_qk = (warp == kQkWarp);
    bool ok = true;
    if (leader) {
      const uint32_t idesc_qk = idesc_bf16_f32(128, kTile, 0, 0);
      const uint32_t idesc_pv = idesc_bf16_f32(128, 256, 0, 1);
      SegIter seg(sm, p);
      int b, begin, end, len, base;
      bool whole;
      uint32_t it = 0, nseg = 0;
      auto wait_or_fail = [&](uint32_t bar, uint32_t par, bool cl_scope) {
        if (!ok) return false;
        const bool mine = (!cl_scope && mbar_test(bar, par)) || mbar_wait(bar, par, abort_flag, kWaitLimitNs, cl_scope);
        if (!__all_sync(0xffffffffu, mine)) {
          if (lane == 0) fail_timeout(sm, p.err);
          ok = false;
        }
        return ok;
      };
      while (ok && seg.next(b, begin, end, len, whole, base)) {
        if (is_qk) {
          if (!wait_or_fail(smem_u32(&sm.q_full), nseg & 1u, true)) break;
          tc_fence_after();
          for (int i = begin; i < end && ok; ++i, ++it) {
            const uint32_t st = it % kStages, ph = (it / kStages) & 1u;
            if (!wait_or_fail(smem_u32(&sm.full[st]), ph, false)) break;
            // the single score buffer: every softmax warp of both CTAs has read S(it - 1)
            if (!wait_or_fail(smem_u32(&sm.s_empty), (it & 1u) ^ 1u, true)) break;
            tc_fence_after();
            const uint32_t stage = sbase + st * kStageBytes, q_s = sbase + kQOff;
            const uint32_t dS = tmem + kColS;
            // K-steps of latent slab s2 (16 features each); query features [0, 384) are in TMEM, the
            // rest in shared memory
            auto qk_slab = [&](int s2, bool first) {
              if (lane != 0) return;
#pragma unroll
              for (int kk = 0; kk < 4; ++kk) {
                const int k = 4 * s2 + kk;
                const uint64_t bd = smem_desc(stage + s2 * kSlab + kk * 32, 16, 1024, kSwizzle128);
                if (k < kQTmemSteps) {
                  mma_pair_ts(dS, tmem + kColQ + 8 * k, bd, idesc_qk, (first && kk == 0) ? 0u : 1u);
                } else {
                  const uint64_t ad = smem_desc(q_s + ((k - kQTmemSteps) >> 2) * kBox + kk * 32, 16, 1024, kSwizzle128);
                  mma_pair_ss(dS, ad, bd, idesc_qk, 1u);
                }
              }
            };
#pragma unroll 1
            for (int s2 = 0; s2 < kStageSlabs; ++s2) qk_slab(s2, s2 == 0);
            if (lane == 0) {
              mma_commit_pair(smem_u32(&sm.s_full), (uint16_t)3);
              mma_commit_pair(smem_u32(&sm.qk_done[st]), (uint16_t)3);
            }
            __syncwarp();
          }
          // every score MMA of this segment has been issued: the query may be replaced once they end
          if (lane == 0) mma_commit_pair(smem_u32(&sm.q_empty), (uint16_t)3);
          __syncwarp();
        } else {
          if (nseg > 0 && !wait_or_fail(smem_u32(&sm.o_free), (nseg - 1) & 1u, true)) break;
          for (int i = begin; i < end && ok; ++i, ++it) {
            const uint32_t st = it % kStages, sb = it & 1u;
            if (!wait_or_fail(smem_u32(&sm.p_full[sb]), (it >> 1) & 1u, true)) break;
            tc_fence_after();
            const int valid = len - i * kTile;
            const int kmax = valid >= kTile ? kKSteps : (valid + 15) >> 4;
            if (lane == 0) {
              const uint32_t stage = sbase + st * kStageBytes, pb = sbase + kPOff + sb * kPBytes;
#pragma unroll
              for (int c = 0; c < 2; ++c) {
#pragma unroll
                for (int k = 0; k < kKSteps; ++k) {
                  if (k < kmax) {
                    // A: P, 16 positions of the K-major P boxes; B: V rows of block k / kBlockSteps
                    // (the positions of CTA 0, then of CTA 1), this CTA's latent columns of chunk c
                    // (slabs 2 c, 2 c + 1 of each block: half A for c = 0, half B for c = 1)
                    const uint64_t ad = smem_desc(pb + (k >> 2) * kBox + (k & 3) * 32, 16, 1024, kSwizzle128);
                    const int blk = k / kBlockSteps, kr = k % kBlockSteps;
                    const uint64_t bd =
                        smem_desc(stage + (4 * blk + 2 * c) * kSlab + kr * 2048, kSlab, 1024, kSwizzle128);
                    mma_pair_ss(tmem + kColO + 128 * c, ad, bd, idesc_pv, (i == begin && k == 0) ? 0u : 1u);
                  }
                }
              }
              mma_commit_pair(smem_u32(&sm.empty[st]), (uint16_t)3);
              mma_commit_pair(smem_u32(&sm.pv_done[sb]), (uint16_t)3);
            }
            __syncwarp();
          }
        }
        ++nseg;
      }
      // drain the tensor pipe (both CTAs wait for these before releasing TMEM)
      if (lane == 0) mma_commit_pair(smem_u32(&sm.drain), (uint16_t)3);
      __syncwarp();
    }
    if (is_qk) mbar_wait(smem_u32(&sm.drain), 0, abort_flag, kWaitLimitNs);
  } else {
    // ------------------------------------------------------------------ softmax warps
    griddep_wait();  // they read the absorbed query and write the context / workspace
    const int sw = warp - kSmWarp0;
    const int q = warp & 3;                       // TMEM lane quadrant
    const int kh = q >> 1;                        // which 64 positions of a tile / which O columns
    const int grp = q & 1;                        // head group: heads 32 grp .. 32 grp + 31
    const int hl = 32 * grp + lane;               // local head (TMEM lane 32 q + lane)
    const int wsub = sw >> 2;                     // 32 of the quadrant's 64 score columns, 128 of its O columns
    const int quad4 = 2 * kh + wsub;              // index among the four threads of a head
    const int h = kHeads * (int)rank + hl;        // head
    const uint32_t lane_off = (uint32_t)(q * 32) << 16;
    const uint32_t tO = tmem + lane_off + kColO + 128 * wsub;
    SegIter seg(sm, p);
    int b, begin, end, len, base;
    bool whole;
    uint32_t it = 0, nseg = 0, npart = 0, nmrg = 0, nmd = 0, nout = 0;
    bool ok = true;
    bool first_seg = true;
    auto warp_arrive_leader = [&](uint32_t bar) {
      __syncwarp();
      if (lane == 0) arrive_leader(bar, rank);
    };
    auto wait_or_fail = [&](uint32_t bar, uint32_t par) {
      if (!ok) return false;
      const bool mine = mbar_test(bar, par) || mbar_wait(bar, par, abort_flag, kWaitLimitNs);
      if (!__all_sync(0xffffffffu, mine)) {
        if (lane == 0) fail_timeout(sm, p.err);
        ok = false;
      }
      return ok;
    };
    while (ok && seg.next(b, begin, end, len, whole, base)) {
      // ---- query features [192 wsub, 192 wsub + 192) of this head into TMEM (A operand of the
      // first 24 score K-steps); both lane halves hold every head of this CTA
      if (nseg > 0 && !wait_or_fail(smem_u32(&sm.q_empty), (nseg - 1) & 1u)) break;
      {
        const uint4* qt = reinterpret_cast<const uint4*>(p.q_tilde + ((int64_t)b * kNH + h) * p.ldqt + 192 * wsub);
#pragma unroll
        for (int cc = 0; cc < 3; ++cc) {
          uint32_t r[32];
#pragma unroll
          for (int v = 0; v < 8; ++v) {
            const uint4 u = __ldg(qt + 8 * cc + v);
            r[4 * v] = u.x; r[4 * v + 1] = u.y; r[4 * v + 2] = u.z; r[4 * v + 3] = u.w;
          }
          tmem_st32(tmem + lane_off + kColQ + 96 * wsub + 32 * cc, r);
        }
        tmem_st_wait();
        tc_fence_before();
        warp_arrive_leader(smem_u32(&sm.q_full));
      }
      float m_run = -INFINITY, l_run = 0.f;
      for (int i = begin; i < end && ok; ++i, ++it) {
        const bool first = (i == begin);
        const uint32_t sb = it & 1u, st = it % kStages;
        if (!wait_or_fail(smem_u32(&sm.s_full), it & 1u)) break;
        tc_fence_after();
        float sa[kSCols];
        {
          uint32_t r[32];
          tmem_ld32(tmem + lane_off + kColS + 32 * wsub, r);
          tmem_ld_wait();
#pragma unroll
          for (int k = 0; k < 32; ++k) sa[k] = __uint_as_float(r[k]);
        }
        tc_fence_before();
        warp_arrive_leader(smem_u32(&sm.s_empty));
        const int valid = len - i * kTile;                 // positions of this tile inside the sequence
        const int vmine = valid - kKeys * kh - kSCols * wsub;  // ... of this thread's columns
        if (vmine < kSCols) {
#pragma unroll
          for (int k = 0; k < kSCols; ++k)
            if (k >= vmine) sa[k] = -INFINITY;
        }
        float mx[4];
#pragma unroll
        for (int qq = 0; qq < 4; ++qq) mx[qq] = fmaxf(fmaxf(sa[qq], sa[qq + 4]), fmaxf(sa[qq + 8], sa[qq + 12]));
#pragma unroll
        for (int qq = 0; qq < 4; ++qq)
          mx[qq] = fmaxf(mx[qq], fmaxf(fmaxf(sa[qq + 16], sa[qq + 20]), fmaxf(sa[qq + 24], sa[qq + 28])));
        // rendezvous of the four warps holding heads 32 grp .. 32 grp + 31 (red[sb] is rewritten two
        // tiles later, after every one of them has passed the rendezvous of the tile in between)
        sm.red[sb][quad4][hl] = fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3]));
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(&sm.red_bar[sb][grp]));
        if (!wait_or_fail(smem_u32(&sm.red_bar[sb][grp]), (it >> 1) & 1u)) break;
        const float m_tile = fmaxf(fmaxf(sm.red[sb][0][hl], sm.red[sb][1][hl]), fmaxf(sm.red[sb][2][hl], sm.red[sb][3][hl])) *
                             p.scale_log2;
        const float m_new = fmaxf(m_run, m_tile);
        const bool need = first || (m_new > m_run + kRescaleThreshold);
        float corr = 1.f;
        if (need) {
          if (!first) corr = ex2f_approx(m_run - m_new);
          m_run = m_new;
        }
        l_run *= corr;
        uint32_t pk[kSCols / 2];
        float ls[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int k = 0; k < kSCols / 2; ++k) {
          const float p0 = ex2f_approx(fmaf(sa[2 * k], p.scale_log2, -m_run));
          const float p1 = ex2f_approx(fmaf(sa[2 * k + 1], p.scale_log2, -m_run));
          pk[k] = pack_bf16x2(p0, p1);
          ls[k & 3] += p0 + p1;
        }
        l_run += (ls[0] + ls[1]) + (ls[2] + ls[3]);
        // ---- the previous P.V must be complete before O is rescaled or its P buffer reused (the
        // first tile of a segment follows an epilogue that already waited for it)
        if (!first) {
          const uint32_t pp = it - 1;
          if (!wait_or_fail(smem_u32(&sm.pv_done[pp & 1u]), (pp >> 1) & 1u)) break;
          tc_fence_after();
          if (__any_sync(0xffffffffu, need)) {
#pragma unroll 1
            for (int c = 0; c < 4; ++c) {
              uint32_t r[32];
              tmem_ld32(tO + c * 32, r);
              tmem_ld_wait();
#pragma unroll
              for (int k = 0; k < 32; ++k) r[k] = __float_as_uint(__uint_as_float(r[k]) * corr);
              tmem_st32(tO + c * 32, r);
            }
            tmem_st_wait();
          }
        }
        // ---- the peer positions' rows of this CTA's latent half have landed; in the last tile of a
        // sequence, rows past its end that the P.V reads are zeroed (0 * garbage could be NaN)
        if (!wait_or_fail(smem_u32(&sm.v_full[st]), (it / kStages) & 1u)) break;
        if (valid < kTile) {
          const int kend = ((valid + 15) >> 4) << 4;       // the P.V reads positions < kend
          const int nz = kend - valid;
          uint8_t* stage = smem + st * kStageBytes;
          for (int idx = sw * 32 + lane; idx < nz * 32; idx += kSmWarps * 32) {
            const int key = valid + (idx >> 5), j = (idx >> 3) & 3, ch = idx & 7;
            *reinterpret_cast<uint4*>(stage + (4 * (key / kKeys) + j) * kSlab + (key % kKeys) * 128 + ch * 16) =
                make_uint4(0, 0, 0, 0);
          }
        }
        // ---- P (bf16) into shared memory: K-major, 128-byte swizzle, boxes of 64 positions; this
        // thread's positions kKeys kh + kSCols wsub .. are 16-byte chunks q0 .. of the tile's row
        {
          const int q0 = (kKeys * kh + kSCols * wsub) >> 3;
          const uint32_t prow = sbase + kPOff + sb * kPBytes + hl * 128;
#pragma unroll
          for (int j = 0; j < kSCols / 8; ++j) {
            const int q = q0 + j;
            st_shared_v4_b32(prow + (q >> 3) * kBox + (((q & 7) ^ (hl & 7)) << 4), pk[4 * j], pk[4 * j + 1],
                             pk[4 * j + 2], pk[4 * j + 3]);
          }
        }
        fence_proxy_async_smem();
        tc_fence_before();
        warp_arrive_leader(smem_u32(&sm.p_full[sb]));
      }
      if (!ok) break;
      // ---- epilogue: O (this head's features [256 kh + 128 wsub, + 128)) -> ctx, or a partial
      {
        const uint32_t pp = it - 1;
        if (!wait_or_fail(smem_u32(&sm.pv_done[pp & 1u]), (pp >> 1) & 1u)) break;
        tc_fence_after();
      }
      // (lsum is rewritten in the next segment's epilogue, after the four warps have met again in
      // that segment's first tile)
      sm.lsum[quad4][hl] = l_run;
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&sm.lsum_bar[grp]));
      if (!wait_or_fail(smem_u32(&sm.lsum_bar[grp]), nseg & 1u)) break;
      const float l_tot = (sm.lsum[0][hl] + sm.lsum[1][hl]) + (sm.lsum[2][hl] + sm.lsum[3][hl]);
      const int fo = 256 * kh + 128 * wsub;               // first output feature of this thread
      const bool head_writer = (quad4 == 0);
      // The range's last segment: its P.V products are complete and no further cache tile or query
      // lands in shared memory, so the stage area is free.  Output rows (this CTA's 64 heads x 512
      // features) then go out through it: each thread writes its 128 features into 128-byte-swizzled
      // boxes of 64 rows x 64 features (the second 64 KB of the stage area), and one thread stores the
      // eight boxes with TMA as whole lines.  (Stores of 16 bytes from each thread straight to its own
      // 1 KB row write partial sectors: 64 KB took several microseconds that way.)  The first 64 KB
      // receives another cluster's partial when two are merged.
      const bool last_seg = (base + end >= sm.hi);
      const uint32_t stg_out = sbase + 65536u;
      auto stage_addr = [&](uint32_t region, int f, int v) -> uint32_t {  // chunk v of features [f, f + 32)
        const int j = f >> 6, c = ((f & 63) >> 3) + v;
        return region + (uint32_t)(j * kBox + hl * 128 + ((c ^ (hl & 7)) << 4));
      };
      // 32 features (four 16-byte chunks) of this thread's row: into the staging boxes, or straight
      // to the global row when staging is not possible
      auto put32 = [&](bool staged, __nv_bfloat16* grow, int f, const uint32_t (&w)[16]) {
#pragma unroll
        for (int v = 0; v < 4; ++v) {
          if (staged) st_shared_v4_b32(stage_addr(stg_out, f, v), w[4 * v], w[4 * v + 1], w[4 * v + 2], w[4 * v + 3]);
          else reinterpret_cast<uint4*>(grow + f)[v] = make_uint4(w[4 * v], w[4 * v + 1], w[4 * v + 2], w[4 * v + 3]);
        }
      };
      // every softmax warp staged its rows (and made its other writes visible): one thread stores the
      // boxes to rows [row0, row0 + 64) of `map` and waits until they are written
      auto store_staged = [&](const CUtensorMap* map, int row0, bool wait_written) -> bool {
        fence_proxy_async_smem();
        if (wait_written) __threadfence();  // a partial's (m, l) stores precede its ready flag
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(&sm.out_bar));
        bool good = true;
        if (sw == 0 && lane == 0) {
          good = mbar_wait(smem_u32(&sm.out_bar), nout & 1u, abort_flag, kWaitLimitNs);
          if (good) {
#pragma unroll 1
            for (int j = 0; j < 8; ++j) tma_store_tile_2d(map, stg_out + j * kBox, 64 * j, row0);
            bulk_group_commit();
            // a published partial must be in global memory before its ready flag rises; the context
            // only needs its staging read before the CTA may exit
            if (wait_written) {
              bulk_group_wait_all();
              fence_proxy_async_global();
            } else {
              bulk_group_wait_read_all();
            }
          } else {
            fail_timeout(sm, p.err);
          }
        }
        ++nout;
        return __shfl_sync(0xffffffffu, good ? 1 : 0, 0) != 0;
      };
      __nv_bfloat16* ws_rows = p.ws_o;                     // [slot][rank][64 heads][512 features]
      auto ws_row = [&](int64_t slot, int head) { return ws_rows + ((slot * 2 + rank) * kHeads + head) * kDC; };
      auto ws_row0 = [&](int64_t slot) { return (int)((slot * 2 + rank) * kHeads); };
      auto ml_at = [&](int64_t slot, int head) { return p.ws_ml + (slot * 2 + rank) * kNH + head; };
      if (whole) {
        const float inv = 1.f / l_tot;
        __nv_bfloat16* out = p.ctx + ((int64_t)b * kNH + h) * kDC;
#pragma unroll 1
        for (int c = 0; c < 4; ++c) {
          uint32_t r[32];
          tmem_ld32(tO + c * 32, r);
          tmem_ld_wait();
          uint32_t w[16];
#pragma unroll
          for (int k = 0; k < 16; ++k)
            w[k] = pack_bf16x2(__uint_as_float(r[2 * k]) * inv, __uint_as_float(r[2 * k + 1]) * inv);
          put32(last_seg, out, fo + 32 * c, w);
        }
        if (head_writer && p.lse != nullptr)
          p.lse[(int64_t)b * kNH + h] = (m_run + log2f(l_tot)) * 0.69314718055994531f;
        if (last_seg && !store_staged(&p.tm_ctx, b * kNH + kHeads * (int)rank, false)) {
          ok = false;
          break;
        }
      } else {
        // ---- partial: the last of the sequence's clusters to arrive (per CTA rank) merges every
        // partial into ctx; the others publish (O, m, l) in their segment's slot and raise the slot's
        // ready flag.  The merger counts its arrival first, so every cluster it then waits for has
        // already arrived (it is running) and needs nothing from the merger.
        const int own = 2 * cl + (first_seg ? 0 : 1);
        // the reload warp counted this cluster's arrival during the segment's last tile
        if (!wait_or_fail(smem_u32(&sm.last_bar), npart & 1u)) break;
        ++npart;
        // A partial is this segment's context normalised by its own softmax sum, in bf16: plain rows of
        // 512 features per (slot, CTA rank, head).
        const float inv_own = 1.f / l_tot;
        if (!sm.is_last) {
          __nv_bfloat16* row = ws_row(own, hl);
#pragma unroll 1
          for (int c = 0; c < 4; ++c) {
            uint32_t r[32];
            tmem_ld32(tO + c * 32, r);
            tmem_ld_wait();
            uint32_t w[16];
#pragma unroll
            for (int k = 0; k < 16; ++k)
              w[k] = pack_bf16x2(__uint_as_float(r[2 * k]) * inv_own, __uint_as_float(r[2 * k + 1]) * inv_own);
            put32(last_seg, row, fo + 32 * c, w);
          }
          if (head_writer) *ml_at(own, hl) = make_float2(m_run, l_tot);
          // the rows (staged or stored) and (m, l) are written before the slot's ready flag rises
          bool good;
          if (last_seg) {
            good = store_staged(&p.tm_ws, ws_row0(own), true);
          } else {
            __threadfence();
            __syncwarp();
            if (lane == 0) mbar_arrive(smem_u32(&sm.out_bar));
            good = true;
            if (sw == 0 && lane == 0) good = mbar_wait(smem_u32(&sm.out_bar), nout & 1u, abort_flag, kWaitLimitNs);
            ++nout;
            good = __shfl_sync(0xffffffffu, good ? 1 : 0, 0) != 0;
          }
          if (!good) {
            if (lane == 0) fail_timeout(sm, p.err);
            ok = false;
            break;
          }
          if (sw == 0 && lane == 0) {
            __threadfence();
            st_release_gpu(p.ws_ready + 2 * (int64_t)own + rank, p.epoch);
          }
        }
        if (sm.nslots > p.slice_above) {
          // ---- sliced merge: every slot's partial is published; this CTA merges heads [h_lo, h_hi)
          // of its 64, one head per warp and two 16-byte chunks per lane (a warp reads and writes
          // 512 contiguous bytes per step), summing the slots in slot order.  The last cluster to
          // finish its slice resets the flags for the next launch.
          const int ns = sm.nslots;
          int okw = 1;
          if (lane == 0) {
            for (int k = 0; k < ns && okw; ++k)
              okw = wait_flag(p.ws_ready + 2 * (int64_t)sm.slots[k] + rank, p.epoch, abort_flag) ? 1 : 0;
            if (!okw) fail_timeout(sm, p.err);
          }
          if (!__shfl_sync(0xffffffffu, okw, 0)) {
            ok = false;
            break;
          }
          int pos = 0;
          for (int k = 0; k < ns; ++k)
            if (sm.slots[k] == own) pos = k;
          const int h_lo = pos * kHeads / ns, h_hi = (pos + 1) * kHeads / ns;
          for (int hh = h_lo + sw; hh < h_hi; hh += kSmWarps) {
            float M = -INFINITY;
#pragma unroll 4
            for (int k = 0; k < ns; ++k) M = fmaxf(M, __ldcg(ml_at(sm.slots[k], hh)).x);
            float L = 0.f;
#pragma unroll 4
            for (int k = 0; k < ns; ++k) {
              const float2 ml = __ldcg(ml_at(sm.slots[k], hh));
              L += ml.y * ex2f_approx(ml.x - M);
            }
            const float inv = 1.f / L;
#pragma unroll
            for (int half = 0; half < 2; ++half) {
              const int chunk = 32 * half + lane;
              float acc[8];
#pragma unroll
              for (int qq = 0; qq < 8; ++qq) acc[qq] = 0.f;
#pragma unroll 4
              for (int k = 0; k < ns; ++k) {
                const int64_t sl = sm.slots[k];
                const float2 ml = __ldcg(ml_at(sl, hh));
                const float w = ml.y * ex2f_approx(ml.x - M) * inv;
                const uint4 u = __ldcg(reinterpret_cast<const uint4*>(ws_row(sl, hh)) + chunk);
                const uint32_t uw[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
                for (int qq = 0; qq < 4; ++qq) {
                  acc[2 * qq] = fmaf(w, bf16_lo(uw[qq]), acc[2 * qq]);
                  acc[2 * qq + 1] = fmaf(w, bf16_hi(uw[qq]), acc[2 * qq + 1]);
                }
              }
              *reinterpret_cast<uint4*>(p.ctx + ((int64_t)b * kNH + kHeads * rank + hh) * kDC + 8 * chunk) =
                  make_uint4(pack_bf16x2(acc[0], acc[1]), pack_bf16x2(acc[2], acc[3]), pack_bf16x2(acc[4], acc[5]),
                             pack_bf16x2(acc[6], acc[7]));
            }
            if (lane == 0 && p.lse != nullptr)
              p.lse[(int64_t)b * kNH + kHeads * rank + hh] = (M + log2f(L)) * 0.69314718055994531f;
          }
          __syncwarp();
          if (lane == 0) mbar_arrive(smem_u32(&sm.mrg_done));
          if (sw == 0 && lane == 0) {
            if (mbar_wait(smem_u32(&sm.mrg_done), nmd & 1u, abort_flag, kWaitLimitNs)) {
              if (arrive_last(p.ws_ctr + 2 * (int64_t)b + rank, p.epoch, ns, p.err))
                for (int k = 0; k < ns; ++k) p.ws_ready[2 * (int64_t)sm.slots[k] + rank] = 0ull;
            } else {
              fail_timeout(sm, p.err);
            }
          }
          ++nmd;
        } else if (sm.is_last) {
          const int ns = sm.nslots;
          int okw = 1;
          if (lane == 0) {
            for (int k = 0; k < ns && okw; ++k)
              if (sm.slots[k] != own)
                okw = wait_flag(p.ws_ready + 2 * (int64_t)sm.slots[k] + rank, p.epoch, abort_flag) ? 1 : 0;
            if (!okw) fail_timeout(sm, p.err);
          }
          if (!__shfl_sync(0xffffffffu, okw, 0)) {
            ok = false;
            break;
          }
          // In the range's last segment up to three other partials are loaded by TMA into the free
          // stage area (partial k of the others at k x 64 KB, in the same swizzled boxes as the
          // staging), and with one other partial the output is staged behind it and stored by TMA.
          // More partials (the sliced merge turned off) are read through L2.
          const bool bulk = last_seg && ns <= kMergeLastMax;
          const bool staged = last_seg && ns == 2;
          // (m, l) of the k-th other partial: in shared memory after the bulk loads, else in L2
          const float2* ml_smem = reinterpret_cast<const float2*>(smem + 196608);
          if (bulk && sw == 0 && lane == 0) {
            fence_proxy_async_global();  // the partials were written through the generic or async proxy
            const uint32_t bar = smem_u32(&sm.mrg_full);
            mbar_arrive_expect_tx(bar, (uint32_t)(ns - 1) * (kHeads * kDC * 2 + kHeads * 8));
            int k = 0;
            for (int s2 = 0; s2 < ns; ++s2) {
              const int sl = sm.slots[s2];
              if (sl == own) continue;
#pragma unroll 1
              for (int j = 0; j < 8; ++j)
                tma_load_2d(sbase + (uint32_t)k * 65536u + j * kBox, &p.tm_ws, bar, 64 * j, ws_row0(sl), policy_evict_first());
              bulk_load_g2s(sbase + 196608u + (uint32_t)k * kHeads * 8, ml_at(sl, 0), kHeads * 8, bar);
              ++k;
            }
          }
          if (bulk && !wait_or_fail(smem_u32(&sm.mrg_full), nmrg & 1u)) break;
          if (bulk) ++nmrg;
          auto ml_of = [&](int s2) -> float2 {  // (m, l) of slot position s2
            const int sl = sm.slots[s2];
            if (sl == own) return make_float2(m_run, l_tot);
            if (!bulk) return __ldcg(ml_at(sl, hl));
            int k = 0;
            for (int q2 = 0; q2 < s2; ++q2) k += sm.slots[q2] != own ? 1 : 0;
            return ml_smem[k * kHeads + hl];
          };
          // Weights of the slots (each partial's softmax sum rescaled to the common maximum), then the
          // sum over the slots in slot order, this CTA's own partial normalised and rounded to bf16
          // like a published one, so the result does not depend on which cluster merges.  (The four
          // weights live in registers: an array indexed by the slot went to local memory, and each of
          // its reads cost a round trip to L2.)
          float M = -INFINITY;
          for (int s2 = 0; s2 < ns; ++s2) M = fmaxf(M, ml_of(s2).x);
          float w0 = 0.f, w1 = 0.f, w2 = 0.f, w3 = 0.f, inv = 0.f;
          float L;
          if (ns == 2) {
            // two terms, each rounded once, added once: the same sum in either arrival order
            const float2 m0 = ml_of(0), m1 = ml_of(1);
            const float a = m0.y * ex2f_approx(m0.x - M), c = m1.y * ex2f_approx(m1.x - M);
            L = a + c;
            w0 = a / L;
            w1 = c / L;
          } else {
            L = 0.f;
            for (int s2 = 0; s2 < ns; ++s2) {
              const float2 ml = ml_of(s2);
              L += ml.y * ex2f_approx(ml.x - M);
            }
            inv = 1.f / L;
            for (int s2 = 0; s2 < ns && s2 < 4; ++s2) {
              const float2 ml = ml_of(s2);
              const float w = ml.y * ex2f_approx(ml.x - M) * inv;
              w0 = s2 == 0 ? w : w0;
              w1 = s2 == 1 ? w : w1;
              w2 = s2 == 2 ? w : w2;
              w3 = s2 == 3 ? w : w3;
            }
          }
          __nv_bfloat16* dst = p.ctx + ((int64_t)b * kNH + h) * kDC;
          if (ns == 2) {
            // Two partials (the common case), in a compact loop: the merge runs once per launch, and
            // unrolled code that is not in the instruction cache cost microseconds to fetch.  Each
            // product is rounded on its own and the two are added once, so the sum is the same in
            // either slot order, whichever cluster merges.
            const bool own_first = (sm.slots[0] == own);
            const float w_own = own_first ? w0 : w1, w_oth = own_first ? w1 : w0;
            const uint32_t oth_base = sbase;  // the other partial's boxes (bulk) or its global row
            const __nv_bfloat16* oth_row = ws_row(own_first ? sm.slots[1] : sm.slots[0], hl);
#pragma unroll 1
            for (int c = 0; c < 4; ++c) {
              const int f = fo + 32 * c;
              uint32_t r[32];
              tmem_ld32(tO + c * 32, r);
              tmem_ld_wait();
              uint32_t wv[16];
#pragma unroll
              for (int v = 0; v < 4; ++v) {
                const uint4 u = bulk ? ld_shared_v4_b32(stage_addr(oth_base, f, v))
                                     : __ldcg(reinterpret_cast<const uint4*>(oth_row + f) + v);
                const uint32_t uw[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                  const uint32_t pr = pack_bf16x2(__uint_as_float(r[8 * v + 2 * q]) * inv_own,
                                                  __uint_as_float(r[8 * v + 2 * q + 1]) * inv_own);
                  const float lo = __fadd_rn(__fmul_rn(w_own, bf16_lo(pr)), __fmul_rn(w_oth, bf16_lo(uw[q])));
                  const float hi = __fadd_rn(__fmul_rn(w_own, bf16_hi(pr)), __fmul_rn(w_oth, bf16_hi(uw[q])));
                  wv[4 * v + q] = pack_bf16x2(lo, hi);
                }
              }
              put32(staged, dst, f, wv);
            }
          } else {
#pragma unroll 1
          for (int c = 0; c < 4; ++c) {
            const int f = fo + 32 * c;
            uint32_t r[32];
            tmem_ld32(tO + c * 32, r);
            tmem_ld_wait();
            float own_v[32];
#pragma unroll
            for (int k = 0; k < 16; ++k) {
              const uint32_t pr = pack_bf16x2(__uint_as_float(r[2 * k]) * inv_own, __uint_as_float(r[2 * k + 1]) * inv_own);
              own_v[2 * k] = bf16_lo(pr);
              own_v[2 * k + 1] = bf16_hi(pr);
            }
            float acc[32];
#pragma unroll
            for (int k = 0; k < 32; ++k) acc[k] = 0.f;
            int kb2 = 0;
            for (int s2 = 0; s2 < ns; ++s2) {
              const int sl = sm.slots[s2];
              float w = s2 == 0 ? w0 : (s2 == 1 ? w1 : (s2 == 2 ? w2 : w3));
              if (s2 >= 4) {  // beyond four slots the weight is formed here, from (m, l) in L2
                const float2 ml = ml_of(s2);
                w = ml.y * ex2f_approx(ml.x - M) * inv;
              }
              if (sl == own) {
                if (ns == 2) {
#pragma unroll
                  for (int k = 0; k < 32; ++k) acc[k] = __fadd_rn(acc[k], __fmul_rn(w, own_v[k]));
                } else {
#pragma unroll
                  for (int k = 0; k < 32; ++k) acc[k] = fmaf(w, own_v[k], acc[k]);
                }
              } else {
#pragma unroll
                for (int v = 0; v < 4; ++v) {
                  const uint4 u = bulk ? ld_shared_v4_b32(stage_addr(sbase + (uint32_t)kb2 * 65536u, f, v))
                                       : __ldcg(reinterpret_cast<const uint4*>(ws_row(sl, hl) + f) + v);
                  const uint32_t uw[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
                  for (int qq = 0; qq < 4; ++qq) {
                    if (ns == 2) {
                      acc[8 * v + 2 * qq] = __fadd_rn(acc[8 * v + 2 * qq], __fmul_rn(w, bf16_lo(uw[qq])));
                      acc[8 * v + 2 * qq + 1] = __fadd_rn(acc[8 * v + 2 * qq + 1], __fmul_rn(w, bf16_hi(uw[qq])));
                    } else {
                      acc[8 * v + 2 * qq] = fmaf(w, bf16_lo(uw[qq]), acc[8 * v + 2 * qq]);
                      acc[8 * v + 2 * qq + 1] = fmaf(w, bf16_hi(uw[qq]), acc[8 * v + 2 * qq + 1]);
                    }
                  }
                }
                ++kb2;
              }
            }
            uint32_t wv[16];
#pragma unroll
            for (int k = 0; k < 16; ++k) wv[k] = pack_bf16x2(acc[2 * k], acc[2 * k + 1]);
            put32(staged, dst, f, wv);
          }
          }
          if (head_writer && p.lse != nullptr)
            p.lse[(int64_t)b * kNH + h] = (M + log2f(L)) * 0.69314718055994531f;
          if (staged && !store_staged(&p.tm_ctx, b * kNH + kHeads * (int)rank, false)) {
            ok = false;
            break;
          }
          // the flags go back to zero for the next launch (a replayed graph reuses the epoch)
          if (sw == 0 && lane == 0)
            for (int s2 = 0; s2 < ns; ++s2)
              if (sm.slots[s2] != own) p.ws_ready[2 * (int64_t)sm.slots[s2] + rank] = 0ull;
        }
      }
      // O has been read: the next segment's first P.V may overwrite it
      tc_fence_before();
      warp_arrive_leader(smem_u32(&sm.o_free));
      first_seg = false;
      ++nseg;
    }
  }

  // ---------------------------------------------------------------------- teardown
  tc_fence_before();
  __syncthreads();
  cluster_sync();  // no MMA, TMA completion or remote arrive of either CTA is still in flight
  tc_fence_after();
  if (warp == kQkWarp) tmem_dealloc_pair(tmem, kTmemCols);
}

// ------------------------------------------------------------------------------------------
// Host side
// ------------------------------------------------------------------------------------------
bool make_map_3d(CUtensorMap* m, const void* base, uint64_t d0, uint64_t d1, uint64_t d2, uint64_t s1_bytes,
                 uint64_t s2_bytes, uint32_t box0, uint32_t box1, CUtensorMapSwizzle sw) {
  const uint64_t dims[3] = {d0, d1, d2};
  const uint64_t strides[2] = {s1_bytes, s2_bytes};
  const uint32_t box[3] = {box0, box1, 1};
  return make_tensor_map_bf16(m, base, 3, dims, strides, box, sw);
}

size_t smem_bytes() { return (size_t)kSmemOff + sizeof(Smem) + 1024; }
static_assert(kSmemOff + sizeof(Smem) + 1024 <= 232448, "dynamic shared memory above the 227 KB per-CTA limit");
static_assert(3 * 65536 <= kSmemOff, "three partials fit below the barriers for the bulk merge");

size_t ws_o_bytes(size_t nc) { return 2 * nc * 2 * (size_t)kHeads * kDC * sizeof(__nv_bfloat16); }
size_t ws_ml_bytes(size_t nc) { return 2 * nc * 2 * 128 * sizeof(float2); }
size_t ws_ready_bytes(size_t nc) { return 2 * nc * 2 * sizeof(unsigned long long); }
size_t ws_bytes(size_t nc, size_t B) {
  return ws_o_bytes(nc) + ws_ml_bytes(nc) + ws_ready_bytes(nc) + B * 2 * sizeof(unsigned long long) + 256;
}

unsigned long long next_epoch() {
  static std::atomic<unsigned long long> counter{
      (unsigned long long)std::chrono::steady_clock::now().time_since_epoch().count() * 0x9E3779B97F4A7C15ull};
  unsigned long long e = 0;
  while (e == 0) e = counter.fetch_add(1, std::memory_order_relaxed) & ((1ull << 56) - 1);
  return e;
}

int max_clusters() {
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int n = sms / 2 < kMaxClusters ? sms / 2 : kMaxClusters;
  return n > 0 ? n : 1;
}

// Clusters of the persistent grid: as many CTA pairs as can be resident at once, so that the grid is
// exactly one wave.  `one_wave` records whether the occupancy query confirmed that (when it fails the
// grid takes the upper bound and the sliced merge, which needs every cluster resident, is not used).
// Cached per device.
struct Wave {
  int clusters;
  bool one_wave;
};
Wave grid_wave() {
  static Wave cache[64] = {};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev >= 0 && dev < 64 && cache[dev].clusters > 0) return cache[dev];
  const int upper = max_clusters();
  Wave w{upper, false};
  if (cudaFuncSetAttribute(decode_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem_bytes()) ==
      cudaSuccess) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(2 * upper);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = smem_bytes();
    int active = 0;
    if (cudaOccupancyMaxActiveClusters(&active, decode_kernel, &cfg) == cudaSuccess && active > 0) {
      w.clusters = active < upper ? active : upper;
      w.one_wave = true;
    }
  }
  cudaGetLastError();
  if (dev >= 0 && dev < 64) cache[dev] = w;
  return w;
}

}  // namespace decode_pair

size_t decode_pair_workspace(int B) { return decode_pair::ws_bytes(decode_pair::max_clusters(), B > 0 ? B : 0); }

cudaError_t decode_pair_launch(const DecodeArgs& a, void* ws, cudaStream_t st) {
  using namespace decode_pair;
  const Wave wave = grid_wave();
  const int nc = wave.clusters;
  Params p;
  memset(&p, 0, sizeof(p));
  const int T = a.T > 0 ? a.T : 1;
  const int n_seq = a.B / T;  // cache sequences
  const uint64_t bstride_c = n_seq > 1 ? (uint64_t)a.ckv_b * 2 : (uint64_t)a.n_max * a.ckv_r * 2;
  const uint64_t bstride_r = n_seq > 1 ? (uint64_t)a.kr_b * 2 : (uint64_t)a.n_max * a.kr_r * 2;
  if (!make_map_3d(&p.tm_ckv, a.c_kv, kDC, a.n_max, n_seq, (uint64_t)a.ckv_r * 2, bstride_c, 64, kKeys,
                   CU_TENSOR_MAP_SWIZZLE_128B) ||
      !make_map_3d(&p.tm_kr, a.k_r, kDR, a.n_max, n_seq, (uint64_t)a.kr_r * 2, bstride_r, 64, kKeys,
                   CU_TENSOR_MAP_SWIZZLE_128B))
    return cudaErrorInvalidValue;
  {
    const uint64_t qd[2] = {(uint64_t)kDC, (uint64_t)a.B * kNH}, qs[1] = {(uint64_t)a.ldqt * 2};
    const uint64_t rd[2] = {(uint64_t)kDR, (uint64_t)a.B * kNH}, rs[1] = {(uint64_t)a.ldqp * 2};
    const uint32_t box[2] = {64, kHeads};
    if (!make_tensor_map_bf16(&p.tm_q, a.q_tilde, 2, qd, qs, box, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !make_tensor_map_bf16(&p.tm_qp, a.q_pe, 2, rd, rs, box, CU_TENSOR_MAP_SWIZZLE_128B))
      return cudaErrorInvalidValue;
    const uint64_t cd[2] = {(uint64_t)kDC, (uint64_t)a.B * kNH}, cs[1] = {(uint64_t)kDC * 2};
    const uint64_t wd[2] = {(uint64_t)kDC, (uint64_t)2 * nc * 2 * kHeads};
    if (!make_tensor_map_bf16(&p.tm_ctx, a.ctx, 2, cd, cs, box, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !make_tensor_map_bf16(&p.tm_ws, ws, 2, wd, cs, box, CU_TENSOR_MAP_SWIZZLE_128B))
      return cudaErrorInvalidValue;
  }
  p.q_tilde = static_cast<const __nv_bfloat16*>(a.q_tilde);
  p.ldqt = a.ldqt;
  p.lengths = a.lengths;
  p.B = a.B;
  p.T = T;
  p.n_max = a.n_max;
  p.n_clusters = nc;
  p.slice_above = sliced_merge_allowed(wave.one_wave) ? kMergeLastMax : 0x7fffffff;
  p.scale_log2 = a.scale * 1.4426950408889634f;
  p.ctx = static_cast<__nv_bfloat16*>(a.ctx);
  p.lse = a.lse;
  uint8_t* w = static_cast<uint8_t*>(ws);
  p.ws_o = reinterpret_cast<__nv_bfloat16*>(w);
  w += ws_o_bytes(nc);
  p.ws_ml = reinterpret_cast<float2*>(w);
  w += ws_ml_bytes(nc);
  p.ws_ready = reinterpret_cast<unsigned long long*>(w);
  w += ws_ready_bytes(nc);
  p.ws_ctr = reinterpret_cast<unsigned long long*>(w);
  p.epoch = next_epoch();
  p.err = a.err;

  const size_t smem = smem_bytes();
  cudaError_t e = cudaFuncSetAttribute(decode_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  return launch_pdl(decode_kernel, dim3(2 * nc), dim3(kThreads), smem, st, p);
}

}  // namespace mla

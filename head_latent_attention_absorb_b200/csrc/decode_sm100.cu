// Absorbed MLA decode on tcgen05 tensor cores (sm_100a): attention of one query token per
// sequence directly over the latent cache ("Absorb key weights", decode excerpt:
// scores = scale (q~ . c^KV_t + q^R . k^R_t), softmax over positions, ctx = sum alpha c^KV_t).
//
// Design (one CTA pair = one thread-block cluster of 2, 1 CTA per SM, one wave):
// * The 128 heads of one sequence are the M = 128 rows of every MMA.
// * TMEM (512 columns) cannot hold the fp32 context of 128 heads x 512 latent features plus a
//   score tile, so the pair splits the latent axis: CTA r owns latent features
//   [256 r, 256 r + 256) and rotary features [32 r, 32 r + 32).  Each CTA loads only its half of
//   every cached row (no byte is loaded twice), computes the PARTIAL score tile over its 288
//   features, and the two partials are exchanged through distributed shared memory as fp16 (bulk
//   copies completing on the receiver's mbarrier); both CTAs add the same two fp16 halves, so
//   their scores agree bit for bit and they run the identical online softmax.
// * Per 64-key tile: TMA brings the CTA's half rows (4 x 128-byte-swizzled slabs + a 64-byte-
//   swizzled rotary slab) into a 4-stage ring; S = Q K^T runs with Q held in TMEM (A operand)
//   and K in shared memory; P (bf16) is written to TMEM and O += P V reads V from the SAME
//   shared-memory tile (K-major for the scores, MN-major for the values).
// * Top-k decode: the tile's selected rows are gathered with per-lane cp.async into the layout the
//   TMA boxes would give, keys 0..31 by the producer and keys 32..63 by warp 15.
// * FP8 latent cache (decode_kernel<true>): E4M3 rows and per-128-feature fp32 scales land in two
//   raw slots behind a 3-stage bf16 ring; warp 15 and the P.V warp convert them into the stages'
//   bf16 layout on chip, and the rest of the kernel is unchanged.
// * Warp roles: warp 0 = TMA producer; warp 1 = TMEM allocator + score-MMA issuer; warp 2 =
//   P.V-MMA issuer (and, with the FP8 cache, converter of half of every tile); warps 3..6 =
//   exchange (read S from TMEM, round to fp16, stage, bulk-copy to the peer); warps 7..14 =
//   softmax (two per TMEM lane quadrant, 32 keys each, agreeing on the row maximum through shared
//   memory), O rescale and epilogue; warp 15 = second gatherer (top-k) or converter (FP8 cache).
//   512 threads x 128 registers fill the register file.
// * Online softmax in base 2 with the scale folded in; the running maximum is only raised (and
//   O rescaled in TMEM) when it grows by more than 8, so rescales are rare.
// * Work split: when every non-empty sequence can get its own clusters, each sequence is cut into
//   chunks of at most `chunk` tiles and cluster i takes chunk i (one sequence per cluster, so the
//   query is loaded once, by TMA, and no pipeline restart happens mid-kernel); otherwise the
//   concatenated tiles of all sequences are cut into equal contiguous ranges.  A cluster that
//   covers a whole sequence writes ctx directly; the others write bf16 partials (O normalised,
//   with its m and l) and the last cluster to finish a sequence (an arrival counter per sequence
//   and latent half, counted by the producer at the segment's last tile) merges two of them;
//   three or more are merged in head slices by all the sequence's clusters.  No second kernel.
// * Every wait is a bounded mbarrier wait (global timer); on expiry the kernel records
//   MLA_ERR_TIMEOUT, drains and returns.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp8.h>
#include <math.h>
#include <string.h>

#include <atomic>
#include <chrono>
#include <mutex>

#include "common.cuh"
#include "kernels.h"
#include "sm100_ptx.cuh"
#include "tma_host.h"

namespace mla {
namespace decode_tc {

using namespace sm100;

constexpr int kNH = 128, kDC = 512, kDR = 64;
constexpr int kTile = 64;                       // keys per tile
constexpr int kStages = 4;
constexpr int kSlabBytes = kTile * 128;         // 64 rows x 64 latent features (bf16)
constexpr int kLatBytes = 4 * kSlabBytes;       // 256 latent features
constexpr int kRopeBytes = kTile * 64;          // 64 rows x 32 rotary features
constexpr int kStageBytes = kLatBytes + kRopeBytes;
constexpr int kXBytes = kNH * kTile * 2;        // one partial-score exchange buffer (fp16)
constexpr int kQLatBytes = kNH * 256 * 2;       // this CTA's latent half of the query (128 heads)
constexpr int kQRopeBytes = kNH * 32 * 2;       // this CTA's rotary half of the query
static_assert(kQLatBytes == 4 * kXBytes, "the first query is staged in the four exchange buffers");
constexpr int kXOff = kStages * kStageBytes;    // shared-memory layout: stages | exchange | q rope | Smem
constexpr int kQRopeOff = kXOff + 4 * kXBytes;
constexpr int kSmemOff = kQRopeOff + kQRopeBytes;
// FP8 latent cache: three bf16 stages, and behind them two raw slots of one tile's e4m3 latent half
// (64 rows x 256 bytes) plus its scales (64 rows x 4 fp32), which the conversion warp turns into the
// stage's bf16 tile
constexpr int kStagesFp8 = 3;
constexpr int kRawOff = kStagesFp8 * kStageBytes;
constexpr int kRawLatBytes = kTile * 256;
constexpr int kRawSlotBytes = kRawLatBytes + kTile * 16;
static_assert(kRawOff + 2 * kRawSlotBytes <= kXOff, "FP8 raw slots overlap the exchange buffers");
constexpr int kMaxClusters = 160;               // partial-slot list capacity (2 slots per cluster)
constexpr int kMergeLastMax = 2;                // up to this many partials the last cluster merges alone
constexpr int kSoftmaxWarps = 8;                // two per TMEM lane quadrant
constexpr int kPvWarp = 2;                      // the warp that issues the P*V MMAs
constexpr int kAWarp0 = 3;                      // 4 exchange warps, one per TMEM lane quadrant
constexpr int kBWarp0 = 7;                      // 8 softmax warps
constexpr int kGatherWarp = kBWarp0 + kSoftmaxWarps;  // top-k decode: copies keys [32, 64) of each tile
constexpr int kThreads = 32 * (kGatherWarp + 1);  // 512 threads x 128 registers: the whole register file
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColO = 0, kColS = 256, kColP = 320, kColQ = 352;  // Q: 128 + 16 columns
constexpr float kRescaleThreshold = 8.0f;       // log2 units
constexpr uint64_t kWaitLimitNs = 1000000000ull;

struct Params {
  CUtensorMap tm_ckv;  // 3-D (d_c, n_max, B), box (64, 64, 1), 128-byte swizzle
  CUtensorMap tm_kr;   // 3-D (d_r, n_max, B), box (32, 64, 1), 64-byte swizzle
  CUtensorMap tm_q;    // 2-D (d_c, B * 128) rows of q~, box (64, 128), 128-byte swizzle
  CUtensorMap tm_qp;   // 2-D (d_r, B * 128) rows of q^R, box (32, 128), 64-byte swizzle
  const int32_t* topk_idx;  // [B][topk] positions attended (distinct), or null for the dense decode
  int topk;
  const __nv_bfloat16* c_kv_base;  // sparse: row r = sequence * n_max + position at c_kv_base + r * ckv_row
  const __nv_bfloat16* k_r_base;
  int64_t ckv_row, kr_row;
  const __nv_bfloat16* q_tilde;
  int64_t ldqt;
  const __nv_bfloat16* q_pe;
  int64_t ldqp;
  const int32_t* lengths;
  int B, n_max, n_clusters;
  int slice_above;  // more partials than this: the sliced merge (needs every cluster resident at once)
  float scale_log2;
  __nv_bfloat16* ctx;
  float* lse;
  float* ws_o;     // [2 n_clusters slots][2 halves][128 heads][256 features] bf16 partial contexts,
                   // each normalised by its own softmax sum (16-byte chunks rotated by head & 15)
  float2* ws_ml;   // [2 n_clusters slots][2 halves][128] (running max in log2 units, sum)
  unsigned long long* ws_ctr;  // [B][2 halves] arrival counters: (epoch << 8) | arrivals
  unsigned long long* ws_ready;  // [2 n_clusters slots][2 halves] partial published: the writer's epoch
  unsigned long long epoch;    // unique per launch, never 0, < 2^56
  int32_t* err;
  // FP8 latent cache (the kFp8 kernel): e4m3 latent rows and their per-128-feature fp32 scales
  CUtensorMap tm_c8;   // 3-D (512 bytes, n_max, B), box (256, 64, 1), no swizzle
  CUtensorMap tm_sc;   // 3-D (4 scales, n_max, B), box (4, 64, 1)
};

struct Smem {
  uint64_t full[kStages], empty[kStages];
  uint64_t q_tma, q_full, s_full, s_empty, p_full, pv_done, drain;
  uint64_t x_full[2], x_free[2];   // exchange buffers (double-buffered by tile parity)
  uint64_t own_ready[2], stg_free[2];  // this CTA's fp16 partial staged / read by the softmax warps
  uint64_t red_bar[2][4], sum_bar; // row-max rendezvous of the two warps of a lane quadrant / final sum
  uint64_t pub_bar, last_bar;      // partial published by all softmax warps / merge decision made
  uint64_t mrg_full;               // the other cluster's partial bulk-loaded for the merge
  uint64_t mrg_full2[2], mrg_empty2[2];  // streamed merge of several partials (double-buffered)
  uint64_t xch_drained;            // the peer has read every partial score this CTA sent
  uint64_t mrg_done;               // every softmax warp finished its share of a sliced merge
  uint64_t raw_full[2], raw_empty[2];  // FP8 cache: raw tile landed / converted
  float red[2][2][kNH];            // [tile parity][key half][head] partial row max
  float lsum[2][kNH];              // [key half][head] partial softmax sum
  int16_t slots[kMaxClusters];     // partial slots of the sequence being merged
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
  int q_seg;             // segments whose query the softmax warps have copied (so whose predecessor's
                         // epilogue is done with the slot list): a count, free of phase aliasing
};

__device__ __forceinline__ int clamp_len(int len, int n_max) { return len < 0 ? 0 : (len > n_max ? n_max : len); }
__device__ __forceinline__ int tiles_of(int len) { return (len + kTile - 1) / kTile; }

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

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// bf16 halves of a packed pair, widened exactly to fp32 (low half = first element).
__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

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

// Keys a sequence attends: its cached length (dense), or the top-k set size (sparse: every sequence
// attends exactly topk gathered positions, which must lie in [0, length)).
__device__ __forceinline__ int seq_len(const Params& p, int b) {
  return p.topk > 0 ? p.topk : clamp_len(p.lengths[b], p.n_max);
}
__device__ __forceinline__ int seq_tiles(const Params& p, int b) { return tiles_of(seq_len(p, b)); }

// Tile counts of the first 256 sequences stay in registers (lane l holds sequences l + 32 k);
// later ones are re-read from global memory.
constexpr int kPlanRegs = 8;
struct PlanTiles {
  int t[kPlanRegs];
  __device__ int at(const Params& p, int k, int lane) const {  // tiles of sequence 32 k + lane
    if (k < kPlanRegs) {
      int v = 0;
#pragma unroll
      for (int i = 0; i < kPlanRegs; ++i) v = (i == k) ? t[i] : v;
      return v;
    }
    const int b = 32 * k + lane;
    return b < p.B ? seq_tiles(p, b) : 0;
  }
};

// ceil(a / c) for 0 <= a, 1 <= c < 2^22, from a float reciprocal of c with one integer correction
// (the float quotient is within one of the exact one at these sizes).
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
    if (k < nk) n += ceil_div_rc(pt.t[k], c, rc);
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
    int t = 0;
    if (b < p.B) {
      const int len = p.lengths[b];
      bad |= (len < 1 || len > p.n_max);
      t = tiles_of(p.topk > 0 ? p.topk : clamp_len(len, p.n_max));
    }
#pragma unroll
    for (int i = 0; i < kPlanRegs; ++i)
      if (i == k) pt.t[i] = t;
    maxt = max(maxt, t);
    if (t > 0) mint = min(mint, t);
    nonempty += t > 0 ? 1 : 0;
    total += t;
  }
#pragma unroll
  for (int i = 0; i < kPlanRegs; ++i)
    if (i >= nk) pt.t[i] = 0;
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
    // chunk_items(maxt) = nonempty <= nc; below the balanced share it exceeds nc
    int lo = max(1, min(balanced, maxt)), hi = maxt;
    if (mint == maxt) {
      // every non-empty sequence has T = maxt tiles: at most q = nc / nonempty chunks each, so the
      // smallest fitting chunk is ceil(T / q)
      const int q = (int)(nc / nonempty);
      lo = hi = (maxt + q - 1) / q;
    }
    while (lo < hi) {
      const int mid = (lo + hi) >> 1;
      if (chunk_items(p, pt, mid, lane) <= nc) hi = mid;
      else lo = mid + 1;
    }
    // One tile longer than the smallest fitting chunk (never more chunks, since chunk_items only
    // falls as the chunk grows): a split sequence's last chunk is then shorter than the others, so
    // its cluster finishes first and publishes its partial while the merging cluster still works.
    if (lo <= balanced + max(4, balanced / 4)) chunk = (lo > 1 && lo < maxt) ? lo + 1 : lo;
  }
  int lo = 0, hi = 0, first_b = p.B, t_first = 0, item0 = 0, kb = 0;
  if (chunk > 0) {
    // cluster c takes chunk c: find its sequence by a scan of the chunk counts
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
      int inc = t;  // inclusive prefix within the warp
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
  // length of the first sequence, read once here so the first segment needs no reload
  const int len0 = (first_b < p.B) ? seq_len(p, first_b) : 0;
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

// Top-k decode: copies keys [32 h, 32 h + 32) of a gathered tile (lane l holds the cache row of key
// 32 h + l) with 16-byte cp.async into exactly the layout the TMA boxes would give: latent slab s,
// key k, chunk c at s * 8 KB + 128 k + 16 (c ^ (k & 7)); rotary key k, chunk c at
// 32 KB + 64 k + 16 (c ^ ((k >> 1) & 3)).  Eight lanes cover one 128-byte row, so every instruction
// reads four whole rows and hits distinct banks.  Each lane's copies then count once on `bar`.
__device__ __forceinline__ void gather_half(const Params& p, int row_of_lane, int h, uint32_t dst, uint32_t bar,
                                            uint32_t rank, int lane) {
#pragma unroll
  for (int g = 0; g < 8; ++g) {
    const int kl = 4 * g + (lane >> 3), ch = lane & 7, key = 32 * h + kl;
    const int r = __shfl_sync(0xffffffffu, row_of_lane, kl);
    const __nv_bfloat16* src = p.c_kv_base + (int64_t)r * p.ckv_row + 256 * rank + 8 * ch;
    const uint32_t d = dst + key * 128 + ((ch ^ (key & 7)) << 4);
#pragma unroll
    for (int sl = 0; sl < 4; ++sl) cp_async_16(d + sl * kSlabBytes, src + 64 * sl);
  }
#pragma unroll
  for (int g = 0; g < 4; ++g) {
    const int kl = 8 * g + (lane >> 2), ch = lane & 3, key = 32 * h + kl;
    const int r = __shfl_sync(0xffffffffu, row_of_lane, kl);
    const __nv_bfloat16* src = p.k_r_base + (int64_t)r * p.kr_row + 32 * rank + 8 * ch;
    cp_async_16(dst + kLatBytes + key * 64 + ((ch ^ ((key >> 1) & 3)) << 4), src);
  }
  cp_async_mbar_arrive(bar);
}

// FP8 latent cache: rows [r0, r1) of a raw tile (e4m3 latent half, 256 bytes per row, then the
// rows' 4 fp32 scales) written as bf16 into a stage in exactly the layout the TMA boxes of the bf16
// cache give: slab s, row r, 16-byte chunk c at s * 8 KB + 128 r + 16 (c ^ (r & 7)).  Lane l converts
// chunk l (features 8 l .. 8 l + 7 of this CTA's half); value = bf16(float(code) * scale of its
// 128-feature block), one fp32 product and one rounding.  The writes are made visible to the
// tensor cores (async proxy) before returning.
__device__ __forceinline__ void convert_fp8_rows(const uint8_t* raw, uint32_t stage, int r0, int r1, uint32_t rank,
                                                 int lane) {
  const int blk = 2 * (int)rank + (lane >> 4);
  const uint32_t dst = stage + (uint32_t)(lane >> 3) * kSlabBytes, chunk = (uint32_t)(lane & 7);
#pragma unroll 4
  for (int r = r0; r < r1; ++r) {
    const uint2 w = *reinterpret_cast<const uint2*>(raw + r * 256 + lane * 8);
    const float sc = reinterpret_cast<const float*>(raw + kRawLatBytes + r * 16)[blk];
    uint32_t o[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const uint32_t word = j < 2 ? w.x : w.y;
      const __half2_raw hr =
          __nv_cvt_fp8x2_to_halfraw2((__nv_fp8x2_storage_t)((word >> (16 * (j & 1))) & 0xffffu), __NV_E4M3);
      const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&hr));
      o[j] = pack_bf16x2(f.x * sc, f.y * sc);
    }
    st_shared_v4_b32(dst + r * 128 + ((chunk ^ (uint32_t)(r & 7)) << 4), o[0], o[1], o[2], o[3]);
  }
  fence_proxy_async_smem();
}

// Walks the segments (sequence, first tile, end tile) of this cluster's range.
struct SegIter {
  int b, tb, t, hi, len0;
  bool first;
  const int32_t* lengths;
  int n_max, B, topk;
  __device__ SegIter(const Smem& sm, const Params& p)
      : b(sm.b0), tb(sm.t_b0), t(sm.lo), hi(sm.hi), len0(sm.len0), first(true), lengths(p.lengths),
        n_max(p.n_max), B(p.B), topk(p.topk) {}
  // On success: sequence b, tiles [begin, end) of it, its length, whether the range holds all of it,
  // and the global index of its first tile.
  __device__ bool next(int& sb, int& begin, int& end, int& len, bool& whole, int& base) {
    while (t < hi && b < B) {
      len = first ? len0 : (topk > 0 ? topk : clamp_len(lengths[b], n_max));
      first = false;
      const int nt = tiles_of(len);
      if (tb + nt <= t) {  // sequence entirely before t (or empty)
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

// Counts this CTA's arrival for (sequence, latent half) and reports whether it was the last of
// `expected`.  The counter holds (epoch << 8) | arrivals; a value from another launch (another
// epoch, or the 0 the last arrival leaves behind) counts as no arrival, so the workspace needs no
// initialisation.  Every failed compare-and-swap means another CTA's arrival succeeded, so the
// loop ends after at most `expected` rounds; the bound is only a guard.
__device__ bool arrive_last(unsigned long long* ctr, unsigned long long epoch, int expected, int32_t* err) {
  // Fast path, one or two atomics: the counter is 0 (left so by the previous launch's last arrival)
  // or already tagged with this launch's epoch (then adding 1 keeps the tag: arrivals < 256).
  unsigned long long cur = atomicCAS(ctr, 0ull, (epoch << 8) | 1ull);
  if (cur == 0ull || (cur >> 8) == epoch) {
    const unsigned long long now = cur == 0ull ? ((epoch << 8) | 1ull) : atomicAdd(ctr, 1ull) + 1ull;
    if ((int)(now & 255ull) < expected) return false;
    atomicExch(ctr, 0ull);  // every arrival of this launch is in: leave the counter for the next one
    return true;
  }
  // a counter another launch left behind (it stopped early): tag it with a compare-and-swap loop
  for (int i = 0; i < 4096; ++i) {
    const unsigned long long base = (cur >> 8) == epoch ? cur : (epoch << 8);
    const unsigned long long next = base + 1;
    const unsigned long long prev = atomicCAS(ctr, cur, next);
    if (prev == cur) {
      if ((int)(next & 255ull) < expected) return false;
      atomicExch(ctr, 0ull);  // every arrival of this launch is in: leave the counter for the next one
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

template <bool kFp8>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
    decode_kernel(const __grid_constant__ Params p) {
  // stages of the ring: four bf16 tiles, or three for the FP8 cache (its raw slots take the fourth)
  constexpr int kNS = kFp8 ? kStagesFp8 : kStages;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* stages = smem;
  uint8_t* xbuf = smem + kXOff;        // 2 receive + 2 staging exchange buffers (first: the query)
  uint8_t* qrope = smem + kQRopeOff;    // rotary half of the first query
  Smem& sm = *reinterpret_cast<Smem*>(smem + kSmemOff);
  volatile int* abort_flag = &sm.abort;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank(), peer = rank ^ 1u;
  const int cl = blockIdx.x >> 1;

  // The next kernel (the up-projection) may start its weight loads on SMs this grid leaves free.
  // This kernel's own set-up and plan need nothing from the preceding kernel (the absorbed query);
  // the threads that read its output or write memory it may read wait for it first (griddep_wait).
  griddep_launch_dependents();
  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      // dense: the producer's arrive.expect_tx + the TMA bytes; sparse: one cp.async arrival per lane
      // of the two gathering warps
      // FP8 cache: the producer's arrive.expect_tx for the rotary slab + the two converting warps
      mbar_init(smem_u32(&sm.full[s]), kFp8 ? 3 : (p.topk > 0 ? 64 : 1));
      mbar_init(smem_u32(&sm.empty[s]), 1);
    }
    // softmax-side arrivals are one per softmax warp, after a __syncwarp
    mbar_init(smem_u32(&sm.q_tma), 1);
    mbar_init(smem_u32(&sm.q_full), kSoftmaxWarps);
    mbar_init(smem_u32(&sm.s_full), 1);
    mbar_init(smem_u32(&sm.s_empty), 4);  // the four exchange warps
    mbar_init(smem_u32(&sm.p_full), kSoftmaxWarps);
    mbar_init(smem_u32(&sm.pv_done), 1);
    mbar_init(smem_u32(&sm.drain), 2);  // one commit from each MMA-issuing thread
    for (int i = 0; i < 2; ++i) {
      mbar_init(smem_u32(&sm.x_full[i]), 1);  // 1 local arrive.expect_tx + the peer's st.async bytes
      // 1 remote arrive from the peer: first when the peer has copied its query out of its exchange
      // buffers, then each time it has read a partial this CTA sent
      mbar_init(smem_u32(&sm.x_free[i]), 1);
      mbar_init(smem_u32(&sm.own_ready[i]), 4);
      mbar_init(smem_u32(&sm.stg_free[i]), kSoftmaxWarps);
      for (int q = 0; q < 4; ++q) mbar_init(smem_u32(&sm.red_bar[i][q]), 2);
    }
    mbar_init(smem_u32(&sm.sum_bar), kSoftmaxWarps);
    mbar_init(smem_u32(&sm.pub_bar), kSoftmaxWarps);
    mbar_init(smem_u32(&sm.last_bar), 1);
    mbar_init(smem_u32(&sm.mrg_full), 1);
    mbar_init(smem_u32(&sm.xch_drained), 4);  // the four exchange warps
    mbar_init(smem_u32(&sm.mrg_done), kSoftmaxWarps);
    for (int i = 0; i < 2; ++i) {
      mbar_init(smem_u32(&sm.mrg_full2[i]), 1);
      mbar_init(smem_u32(&sm.mrg_empty2[i]), kSoftmaxWarps);
      mbar_init(smem_u32(&sm.raw_full[i]), 1);
      mbar_init(smem_u32(&sm.raw_empty[i]), 2);  // the two converting warps
    }
    sm.abort = 0;
    sm.q_seg = 0;
    fence_mbar_init();
    prefetch_tensormap(&p.tm_ckv);
    prefetch_tensormap(&p.tm_kr);
    prefetch_tensormap(&p.tm_q);
    prefetch_tensormap(&p.tm_qp);
    if (kFp8) {
      prefetch_tensormap(&p.tm_c8);
      prefetch_tensormap(&p.tm_sc);
    }
  }
  if (warp == 0) plan_range(p, cl, sm, lane);
  if (warp == 1) {
    tmem_alloc(smem_u32(&sm.tmem_base), kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  // The peer's barriers must be initialised before any remote arrive or copy: every warp arrives on
  // the cluster barrier now and waits before its first remote operation.  The producer only touches
  // this CTA's memory, so it starts loading before it waits.
  asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory");
  if (warp != 0 && warp != kGatherWarp) asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory");
  const uint32_t tmem = sm.tmem_base;

  if (warp == 0) {
    // ------------------------------------------------------------------ TMA producer
    // The whole warp walks the tiles (the control flow is the same in every lane).  Dense: lane 0
    // issues one 3-D TMA box per 64-feature slab.  Sparse: the warp loads the tile's 64 selected
    // positions (two per lane), checks them against the sequence length, and copies the rows with
    // per-lane 16-byte cp.async into the layout the TMA boxes would give.
    {
      const uint64_t pol = policy_evict_first();
      SegIter seg(sm, p);
      int b, begin, end, len, base;
      bool whole;
      uint32_t it = 0, nseg_p = 0;
      bool ok = true, q_issued = false;
      while (ok && seg.next(b, begin, end, len, whole, base)) {
        if (!q_issued) {
          griddep_wait();  // the absorbed query is the preceding kernel's output
          // the first sequence's query (this CTA's halves) goes in ahead of the cache tiles: latent
          // half into the four exchange buffers (free until the first exchange), rotary half apart
          if (lane == 0) {
            const uint32_t qb = smem_u32(&sm.q_tma);
            mbar_arrive_expect_tx(qb, kQLatBytes + kQRopeBytes);
#pragma unroll
            for (int j = 0; j < 4; ++j)
              tma_load_2d(smem_u32(xbuf + j * kXBytes), &p.tm_q, qb, 256 * (int)rank + 64 * j, b * kNH, pol);
            tma_load_2d(smem_u32(qrope), &p.tm_qp, qb, 32 * (int)rank, b * kNH, pol);
          }
          q_issued = true;
        }
        const int seq_len_b = p.topk > 0 ? clamp_len(p.lengths[b], p.n_max) : 0;
        // sparse: the positions of keys [0, 32) of tile i + 1 are loaded while tile i is issued
        // (one per lane), so no tile waits for its own index load
        int pos_next = 0;
        auto load_pos = [&](int i) {
          const int k = i * kTile + lane;
          return k < p.topk ? p.topk_idx[(int64_t)b * p.topk + k] : 0;
        };
        if (p.topk > 0) pos_next = load_pos(begin);
        for (int i = begin; i < end && ok; ++i, ++it) {
          const int pos_cur = pos_next;
          if (p.topk > 0 && i + 1 < end) pos_next = load_pos(i + 1);
          const uint32_t st = it % kNS, ph = (it / kNS) & 1u;
          if (!__all_sync(0xffffffffu, mbar_wait(smem_u32(&sm.empty[st]), ph ^ 1u, abort_flag, kWaitLimitNs))) {
            if (lane == 0) fail_timeout(sm, p.err);
            ok = false;
            break;
          }
          const uint32_t dst = smem_u32(stages + st * kStageBytes);
          const uint32_t bar = smem_u32(&sm.full[st]);
          if (kFp8) {
            // the rotary half straight into the stage; the e4m3 latent half and its scales into raw
            // slot it & 1 once the conversion warp has read that slot's previous tile
            int okr = 1;
            if (lane == 0) {
              mbar_arrive_expect_tx(bar, kRopeBytes);
              tma_load_3d(dst + kLatBytes, &p.tm_kr, bar, 32 * (int)rank, i * kTile, b, pol);
              const uint32_t rs = it & 1u, rb = smem_u32(&sm.raw_full[rs]);
              if (mbar_wait(smem_u32(&sm.raw_empty[rs]), ((it >> 1) & 1u) ^ 1u, abort_flag, kWaitLimitNs)) {
                const uint32_t raw = smem_u32(smem + kRawOff + rs * kRawSlotBytes);
                mbar_arrive_expect_tx(rb, kRawSlotBytes);
                tma_load_3d(raw, &p.tm_c8, rb, 256 * (int)rank, i * kTile, b, pol);
                tma_load_3d(raw + kRawLatBytes, &p.tm_sc, rb, 0, i * kTile, b, pol);
              } else {
                fail_timeout(sm, p.err);
                okr = 0;
              }
            }
            if (!__shfl_sync(0xffffffffu, okr, 0)) {
              ok = false;
              break;
            }
          } else if (p.topk == 0) {
            if (lane == 0) {
              mbar_arrive_expect_tx(bar, kStageBytes);
#pragma unroll
              for (int s = 0; s < 4; ++s)
                tma_load_3d(dst + s * kSlabBytes, &p.tm_ckv, bar, 256 * (int)rank + 64 * s, i * kTile, b, pol);
              tma_load_3d(dst + kLatBytes, &p.tm_kr, bar, 32 * (int)rank, i * kTile, b, pol);
            }
          } else {
            // rows of the 2-D caches: b * n_max + position; positions past the top-k set (the last
            // tile's tail, zeroed before use) and invalid ones (flagged) read position 0
            int pos = 0;
            if (i * kTile + lane < p.topk) {
              pos = pos_cur;
              if (pos < 0 || pos >= seq_len_b) {
                raise_error(p.err, MLA_ERR_INDEX);
                pos = 0;
              }
            }
            gather_half(p, b * p.n_max + pos, 0, dst, bar, rank, lane);
          }
          __syncwarp();
          if (i == end - 1 && !whole) {
            // The segment's last tile is on its way: count this cluster's arrival for the sequence
            // (per latent half) now.  An atomic takes about a microsecond while HBM is busy; here it
            // overlaps the last tiles' work instead of delaying the epilogue.  The epilogue reads the
            // decision (and the slot list) after waiting on last_bar.  A later segment's decision
            // waits until that segment's query is in (q_full), i.e. until the previous segment's
            // epilogue is done with the slot list.
            int okq = 1;
            if (lane == 0) {
              if (nseg_p > 0) {
                // (a count, not q_full's phase parity: after short whole segments the producer can be
                // two segments ahead, and a parity wait would pass on an older phase)
                const uint64_t t0 = globaltimer();
                while (*reinterpret_cast<volatile int*>(&sm.q_seg) < (int)nseg_p + 1) {
                  if (*abort_flag || globaltimer() - t0 > kWaitLimitNs) {
                    okq = 0;
                    break;
                  }
                  __nanosleep(32);
                }
                __threadfence_block();
              }
              if (okq) {
                const int ns = list_slots(p, sm, base, tiles_of(len));
                // up to p.slice_above partials (kMergeLastMax = 2 when the whole grid is resident,
                // else any number) the last cluster to arrive merges them all; with more, every
                // cluster publishes and then merges its own slice of the heads (with three or four
                // partials the slices run in parallel: top-k call 43.8 -> 41.0 us against one
                // merging cluster)
                sm.is_last = ns > p.slice_above ? 0 : (arrive_last(p.ws_ctr + 2 * (int64_t)b + rank, p.epoch, ns, p.err) ? 1 : 0);
                mbar_arrive(smem_u32(&sm.last_bar));
              } else {
                fail_timeout(sm, p.err);
              }
            }
            if (!__shfl_sync(0xffffffffu, okq, 0)) {
              ok = false;
              break;
            }
          }
        }
        ++nseg_p;
      }
      // drain: every load issued must have landed before the CTA may exit
      if (lane == 0) {
        const uint32_t first = it > (uint32_t)kNS ? it - kNS : 0;
        for (uint32_t k = first; k < it; ++k)
          mbar_wait(smem_u32(&sm.full[k % kNS]), (k / kNS) & 1u, abort_flag, kWaitLimitNs);
        if (q_issued) mbar_wait(smem_u32(&sm.q_tma), 0, abort_flag, kWaitLimitNs);
      }
    }
    __syncwarp();
    asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory");
    griddep_wait();
    // lengths outside [1, n_max] (an error already flagged): sequences left without tiles get a
    // zero context and lse = -inf from cluster 0, each CTA its latent half
    if (cl == 0 && sm.bad) {
      for (int b = 0; b < p.B; ++b) {
        if (seq_tiles(p, b) != 0) continue;
        for (int i = lane; i < kNH * 32; i += 32)
          reinterpret_cast<uint4*>(p.ctx + ((int64_t)b * kNH + (i >> 5)) * kDC + 256 * rank)[i & 31] =
              make_uint4(0, 0, 0, 0);
        if (rank == 0 && p.lse != nullptr)
          for (int hh = lane; hh < kNH; hh += 32) p.lse[(int64_t)b * kNH + hh] = -INFINITY;
      }
    }
  } else if (warp == 1 || warp == kPvWarp) {
    // ------------------------------------------------------------------ MMA issuers
    // Warp 1 issues S(t) = Q K(t)^T as soon as stage t has landed and the softmax has read
    // S(t-1); warp kPvWarp issues O += P(t) V(t) as soon as P(t) is in TMEM.  Two issuing threads
    // keep a score MMA from queueing behind a wait for P.
    const bool is_qk = (warp == 1);
    const uint32_t idesc_qk = idesc_bf16_f32(128, kTile, 0, 0);
    const uint32_t idesc_pv = idesc_bf16_f32(128, 256, 0, 1);
    const uint32_t tO = tmem + kColO, tS = tmem + kColS, tP = tmem + kColP, tQ = tmem + kColQ;
    SegIter seg(sm, p);
    int b, begin, end, len, base;
    bool whole;
    uint32_t it = 0, nseg = 0;  // it: global index of the next tile
    bool ok = true;
    // every lane waits; the warp proceeds only if all lanes saw the barrier complete, so the
    // warp stays converged for the .sync.aligned tcgen05 instructions even on a timeout
    auto wait_or_fail = [&](uint32_t bar, uint32_t par, bool cl_scope) {
      if (!ok) return false;
      const bool mine = mbar_wait(bar, par, abort_flag, kWaitLimitNs, cl_scope);
      if (!__all_sync(0xffffffffu, mine)) {
        if (lane == 0) fail_timeout(sm, p.err);
        ok = false;
      }
      return ok;
    };
    // S(t) = Q K(t)^T over this CTA's 288 features
    auto issue_qk = [&](uint32_t t, int tile_in_seq) {
      const uint32_t st = t % kNS;
      if (!wait_or_fail(smem_u32(&sm.full[st]), (t / kNS) & 1u, false)) return;
      if (p.topk > 0 || kFp8) fence_proxy_async_smem();  // rows written through the generic proxy
      const int valid = len - tile_in_seq * kTile;
      if (valid < kTile) {  // rows past the sequence end: zero them so 0 * garbage cannot occur
        uint8_t* sbase = stages + st * kStageBytes;
        const int nrow = kTile - valid;
        for (int idx = lane; idx < nrow * 36; idx += 32) {
          const int r = valid + idx / 36, ch = idx % 36;  // 32 latent chunks + 4 rotary chunks
          uint8_t* dst = ch < 32 ? sbase + (ch >> 3) * kSlabBytes + r * 128 + (ch & 7) * 16
                                 : sbase + kLatBytes + r * 64 + (ch - 32) * 16;
          *reinterpret_cast<uint4*>(dst) = make_uint4(0, 0, 0, 0);
        }
        fence_proxy_async_smem();
        __syncwarp();
      }
      if (!wait_or_fail(smem_u32(&sm.s_empty), (t & 1u) ^ 1u, false)) return;
      tc_fence_after();
      if (lane == 0) {
        const uint32_t base = smem_u32(stages + st * kStageBytes);
#pragma unroll
        for (int k = 0; k < 16; ++k) {
          const uint64_t bd = smem_desc(base + (k >> 2) * kSlabBytes + (k & 3) * 32, 16, 1024, kSwizzle128);
          mma_ts(tS, tQ + k * 8, bd, idesc_qk, k > 0 ? 1u : 0u);
        }
#pragma unroll
        for (int k = 0; k < 2; ++k) {
          const uint64_t bd = smem_desc(base + kLatBytes + k * 32, 16, 512, kSwizzle64);
          mma_ts(tS, tQ + 128 + k * 8, bd, idesc_qk, 1u);
        }
        mma_commit(smem_u32(&sm.s_full));
      }
      __syncwarp();
    };
    // FP8 cache: the P*V warp converts rows [32, 64) of every tile (the conversion warp rows
    // [0, 32)), two tiles ahead of the tile whose P it waits for next: tiles 0 and 1 before the
    // first P*V, tile t + 2 right after issuing P*V(t)
    const uint32_t ntiles_fp8 = sm.hi > sm.lo ? (uint32_t)(sm.hi - sm.lo) : 0u;
    auto convert_half = [&](uint32_t t) -> bool {
      const uint32_t st = t % kNS, rs = t & 1u;
      if (!wait_or_fail(smem_u32(&sm.raw_full[rs]), (t >> 1) & 1u, false)) return false;
      if (!wait_or_fail(smem_u32(&sm.empty[st]), ((t / kNS) & 1u) ^ 1u, false)) return false;
      convert_fp8_rows(smem + kRawOff + rs * kRawSlotBytes, smem_u32(stages + st * kStageBytes), kTile / 2, kTile, rank,
                       lane);
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(smem_u32(&sm.full[st]));
        mbar_arrive(smem_u32(&sm.raw_empty[rs]));
      }
      return true;
    };
    if (kFp8 && !is_qk)
      for (uint32_t t = 0; t < 2 && t < ntiles_fp8 && ok; ++t) ok = convert_half(t);
    // O += P(t) V(t) over this CTA's 256 latent features
    auto issue_pv = [&](uint32_t t, bool first_of_seg) {
      if (!wait_or_fail(smem_u32(&sm.p_full), t & 1u, false)) return;
      tc_fence_after();
      if (p.topk > 0 || kFp8) fence_proxy_async_smem();
      const uint32_t st = t % kNS;
      if (lane == 0) {
        const uint32_t base = smem_u32(stages + st * kStageBytes);
#pragma unroll
        for (int k = 0; k < kTile / 16; ++k) {
          const uint64_t bd = smem_desc(base + k * 2048, kSlabBytes, 1024, kSwizzle128);
          mma_ts(tO, tP + k * 8, bd, idesc_pv, (first_of_seg && k == 0) ? 0u : 1u);
        }
        mma_commit(smem_u32(&sm.empty[st]));
        mma_commit(smem_u32(&sm.pv_done));
      }
      __syncwarp();
    };
    while (ok && seg.next(b, begin, end, len, whole, base)) {
      if (is_qk) {
        if (!wait_or_fail(smem_u32(&sm.q_full), nseg & 1u, false)) break;
        tc_fence_after();
        for (int i = begin; i < end && ok; ++i) issue_qk(it++, i);
      } else {
        for (int i = begin; i < end && ok; ++i) {
          issue_pv(it++, i == begin);
          // FP8 cache: rows [32, 64) of the tile two ahead, while this warp would wait for P
          if (kFp8 && ok && it + 1 < ntiles_fp8) ok = convert_half(it + 1);
        }
      }
      ++nseg;
    }
    // drain the tensor pipe before the TMEM is released
    if (lane == 0) mma_commit(smem_u32(&sm.drain));
    __syncwarp();
    mbar_wait(smem_u32(&sm.drain), 0, abort_flag, kWaitLimitNs);
  } else if (warp >= kAWarp0 && warp < kAWarp0 + 4) {
    // ------------------------------------------------------------------ exchange warps (one per quadrant)
    // Phase A of every tile: read this CTA's partial S(t) (fp32, 288 features) from TMEM, round it
    // to fp16 into the staging buffer (the softmax warps read it from there) and bulk-copy the same
    // 4 KB block to the peer.  Both CTAs then add the same two fp16 halves, so their scores agree
    // bit for bit (relative rounding 2^-11 per half-score).
    const int quad = warp & 3;
    const uint32_t lane_off = (uint32_t)(quad * 32) << 16;
    const uint32_t tS = tmem + lane_off + kColS;
    const bool a_leader = (warp == kAWarp0 && lane == 0);
    const uint32_t xb = smem_u32(xbuf), xb_peer = mapa(xb, peer), stg = xb + 2 * kXBytes;
    const uint32_t blk = quad * 4096;                          // [quad][key half][32 rows][32 keys]
    const uint32_t swz = (lane >> 1) & 3;
    const uint32_t x_full_l0 = smem_u32(&sm.x_full[0]), x_full_r0 = mapa(x_full_l0, peer);
    bool ok = true;
    auto wait_or_fail = [&](uint32_t bar, uint32_t par, bool cl_scope) {
      if (!ok) return false;
      const bool mine = mbar_wait(bar, par, abort_flag, kWaitLimitNs, cl_scope);
      if (!__all_sync(0xffffffffu, mine)) {
        if (lane == 0) fail_timeout(sm, p.err);
        ok = false;
      }
      return ok;
    };
    const uint32_t ntiles = sm.hi > sm.lo ? (uint32_t)(sm.hi - sm.lo) : 0u;
    for (uint32_t t = 0; t < ntiles && ok; ++t) {
      const uint32_t xi = t & 1u, use = t >> 1;
      if (!wait_or_fail(smem_u32(&sm.s_full), t & 1u, false)) break;
      tc_fence_after();
      uint32_t h16[32];
      {
        uint32_t r[32];
        tmem_ld32(tS, r);
        tmem_ld_wait();
#pragma unroll
        for (int k = 0; k < 16; ++k) h16[k] = pack_f16x2(__uint_as_float(r[2 * k]), __uint_as_float(r[2 * k + 1]));
        tmem_ld32(tS + 32, r);
        tmem_ld_wait();
#pragma unroll
        for (int k = 0; k < 16; ++k) h16[16 + k] = pack_f16x2(__uint_as_float(r[2 * k]), __uint_as_float(r[2 * k + 1]));
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&sm.s_empty));
      // the peer's receive buffer xi is free once the peer has copied its query out (phase 0) and
      // read this CTA's tile t - 2 (phase use); staging xi once this CTA's softmax warps read it
      if (!wait_or_fail(smem_u32(&sm.x_free[xi]), use & 1u, true)) break;
      if (!wait_or_fail(smem_u32(&sm.stg_free[xi]), (use & 1u) ^ 1u, false)) break;
      // The softmax warps release staging xi only after they have waited for receive buffer xi of
      // tile t - 2, so that phase of x_full[xi] is complete and this tile's expected byte count
      // opens the next one (never two arrivals in one phase).
      if (a_leader) mbar_arrive_expect_tx(x_full_l0 + 8 * xi, kXBytes);
      const uint32_t row = stg + xi * kXBytes + blk + lane * 64;
#pragma unroll
      for (int hf = 0; hf < 2; ++hf)
#pragma unroll
        for (int j = 0; j < 4; ++j)
          st_shared_v4_b32(row + hf * 2048 + ((j ^ swz) << 4), h16[16 * hf + 4 * j], h16[16 * hf + 4 * j + 1],
                           h16[16 * hf + 4 * j + 2], h16[16 * hf + 4 * j + 3]);
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) {
        bulk_copy_to_peer(xb_peer + xi * kXBytes + blk, stg + xi * kXBytes + blk, 4096, x_full_r0 + 8 * xi);
        mbar_arrive(smem_u32(&sm.own_ready[xi]));
      }
    }
    // Once the peer has read the last two partials this CTA sent, no copy reads the staging buffers
    // any more and the exchange buffers may hold other data (the split-KV merge).  The peer's read
    // of tile t completes phase (t >> 1) + 1 of x_free[t & 1].
    for (uint32_t t = ntiles >= 2 ? ntiles - 2 : 0; t < ntiles && ok; ++t)
      wait_or_fail(smem_u32(&sm.x_free[t & 1u]), ((t >> 1) + 1u) & 1u, true);
    __syncwarp();
    if (lane == 0) mbar_arrive(smem_u32(&sm.xch_drained));
  } else if (kFp8 && warp == kGatherWarp) {
    // ------------------------------------------------------------------ FP8 cache: conversion warp
    // Every tile: wait for its raw slot (e4m3 latent half + scales) and for its stage, convert half
    // of its rows into the stage, then count on both (the P*V warp converts the other half).
    SegIter seg(sm, p);
    int b, begin, end, len, base;
    bool whole;
    uint32_t it = 0;
    bool ok = true;
    while (ok && seg.next(b, begin, end, len, whole, base)) {
      for (int i = begin; i < end && ok; ++i, ++it) {
        const uint32_t st = it % kNS, rs = it & 1u;
        const bool got = mbar_wait(smem_u32(&sm.raw_full[rs]), (it >> 1) & 1u, abort_flag, kWaitLimitNs) &&
                         mbar_wait(smem_u32(&sm.empty[st]), ((it / kNS) & 1u) ^ 1u, abort_flag, kWaitLimitNs);
        if (!__all_sync(0xffffffffu, got)) {
          if (lane == 0) fail_timeout(sm, p.err);
          ok = false;
          break;
        }
        // rows [0, 32); the P*V warp converts rows [32, 64) two tiles ahead
        convert_fp8_rows(smem + kRawOff + rs * kRawSlotBytes, smem_u32(stages + st * kStageBytes), 0, kTile / 2, rank,
                         lane);
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(smem_u32(&sm.full[st]));
          mbar_arrive(smem_u32(&sm.raw_empty[rs]));
        }
      }
    }
    __syncwarp();
    asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory");
  } else if (warp == kGatherWarp) {
    // ------------------------------------------------------------------ second gathering warp
    // Top-k decode only: keys [32, 64) of every tile, in step with the producer (same stage ring;
    // the stage's full barrier counts both warps' lanes).  Like the producer it touches only this
    // CTA's memory, so it waits on the cluster barrier at the end.
    if (p.topk > 0) {
      SegIter seg(sm, p);
      int b, begin, end, len, base;
      bool whole;
      uint32_t it = 0;
      bool ok = true, waited = false;
      while (ok && seg.next(b, begin, end, len, whole, base)) {
        if (!waited) {
          griddep_wait();  // the top-k indices may be the preceding kernel's output
          waited = true;
        }
        const int seq_len_b = clamp_len(p.lengths[b], p.n_max);
        auto load_pos = [&](int i) {
          const int k = i * kTile + 32 + lane;
          return k < p.topk ? p.topk_idx[(int64_t)b * p.topk + k] : 0;
        };
        int pos_next = load_pos(begin);
        for (int i = begin; i < end && ok; ++i, ++it) {
          const int pos_cur = pos_next;
          if (i + 1 < end) pos_next = load_pos(i + 1);
          const uint32_t st = it % kNS, ph = (it / kNS) & 1u;
          if (!__all_sync(0xffffffffu, mbar_wait(smem_u32(&sm.empty[st]), ph ^ 1u, abort_flag, kWaitLimitNs))) {
            if (lane == 0) fail_timeout(sm, p.err);
            ok = false;
            break;
          }
          int pos = 0;
          if (i * kTile + 32 + lane < p.topk) {
            pos = pos_cur;
            if (pos < 0 || pos >= seq_len_b) {
              raise_error(p.err, MLA_ERR_INDEX);
              pos = 0;
            }
          }
          gather_half(p, b * p.n_max + pos, 1, smem_u32(stages + st * kStageBytes), smem_u32(&sm.full[st]), rank, lane);
          __syncwarp();
        }
      }
    }
    __syncwarp();
    asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory");
  } else {
    // ------------------------------------------------------------------ softmax warps (kBWarp0..)
    griddep_wait();  // they read the absorbed query and write the context / workspace
    const int sw = warp - kBWarp0;
    const int half = sw >> 2;                        // which 32 keys of each tile
    const int quad = warp & 3;                       // TMEM lane quadrant of this warp
    const int h = quad * 32 + lane;                  // head == TMEM lane
    const uint32_t lane_off = (uint32_t)(quad * 32) << 16;
    const uint32_t tO = tmem + lane_off + kColO + 128 * half;   // this half's O columns
    const uint32_t tP = tmem + lane_off + kColP + 16 * half;
    const uint32_t tQ = tmem + lane_off + kColQ;
    const uint32_t xb = smem_u32(xbuf), stg = xb + 2 * kXBytes;
    const uint32_t row_off = quad * 4096 + half * 2048 + lane * 64;
    const uint32_t swz = (lane >> 1) & 3;
    const uint32_t x_full_l0 = smem_u32(&sm.x_full[0]);
    const uint32_t x_free_peer0 = mapa(smem_u32(&sm.x_free[0]), peer);
    auto warp_arrive = [&](uint32_t bar) {
      __syncwarp();
      if (lane == 0) mbar_arrive(bar);
    };
    // Staged stores, for the range's last segment (no cache tile lands in the stage buffers any more):
    // this warp's 32 heads x 16 chunks of 16 bytes go through shared memory (its 8 KB at
    // stages + 72 KB, past a bulk-loaded partial and its (m, l) pairs; chunk c of lane l's head at
    // l * 256 + 16 (c ^ (l & 15)), conflict-free both ways), then every store instruction writes two
    // whole 256-byte head rows instead of 32 scattered 16-byte pieces.
    const uint32_t stg_out = smem_u32(stages) + 73728u + (uint32_t)sw * 8192u;
    auto stage_chunk = [&](int c, uint32_t x, uint32_t y, uint32_t z, uint32_t w) {
      st_shared_v4_b32(stg_out + lane * 256 + ((c ^ (lane & 15)) << 4), x, y, z, w);
    };
    // dst(hl, cc): global address of chunk cc (of 16) of local head hl (head quad * 32 + hl)
    auto flush_staged = [&](auto dst) {
      __syncwarp();
#pragma unroll 4
      for (int i = 0; i < 16; ++i) {
        const int hl = 2 * i + (lane >> 4), cc = lane & 15;
        *dst(hl, cc) = ld_shared_v4_b32(stg_out + hl * 256 + ((cc ^ (hl & 15)) << 4));
      }
      __syncwarp();
    };
    SegIter seg(sm, p);
    int b, begin, end, len, base;
    bool whole;
    uint32_t tb = 0;           // global tile counter
    uint32_t nseg = 0, npart = 0, npub = 0, nmrg = 0, nmd = 0;
    bool ok = true;
    bool first_seg = true;     // the first segment of the range uses partial slot 2c, the last 2c + 1
    auto wait_or_fail = [&](uint32_t bar, uint32_t par, bool cl_scope) {
      if (!ok) return false;
      const bool mine = mbar_wait(bar, par, abort_flag, kWaitLimitNs, cl_scope);
      if (!__all_sync(0xffffffffu, mine)) {
        if (lane == 0) fail_timeout(sm, p.err);
        ok = false;
      }
      return ok;
    };
    while (ok && seg.next(b, begin, end, len, whole, base)) {
      // ---- this sequence's query half into TMEM (A operand of the score MMA)
      if (nseg == 0) {
        // staged by TMA: latent chunk c = box c of the exchange buffers (128-byte swizzle, 128-byte
        // rows), rotary half in its own buffer (64-byte swizzle, 64-byte rows)
        if (!wait_or_fail(smem_u32(&sm.q_tma), 0, false)) break;
#pragma unroll
        for (int cc = 0; cc < 2; ++cc) {
          const int c = 2 * half + cc;
          const uint32_t row = xb + c * kXBytes + h * 128;
          uint32_t r[32];
#pragma unroll
          for (int v = 0; v < 8; ++v) {
            const uint4 u = ld_shared_v4_b32(row + ((v ^ (h & 7)) << 4));
            r[4 * v] = u.x; r[4 * v + 1] = u.y; r[4 * v + 2] = u.z; r[4 * v + 3] = u.w;
          }
          tmem_st32(tQ + c * 32, r);
        }
        if (half == 1) {
          const uint32_t row = smem_u32(qrope) + h * 64;
          uint32_t r16[16];
#pragma unroll
          for (int v = 0; v < 4; ++v) {
            const uint4 u = ld_shared_v4_b32(row + ((v ^ ((h >> 1) & 3)) << 4));
            r16[4 * v] = u.x; r16[4 * v + 1] = u.y; r16[4 * v + 2] = u.z; r16[4 * v + 3] = u.w;
          }
          tmem_st16(tQ + 128, r16);
        }
        tmem_st_wait();
        tc_fence_before();
        warp_arrive(smem_u32(&sm.q_full));
        if (sw == 0 && lane == 0) {
          // every softmax warp has copied its rows out: the peer may now write this CTA's buffers
          if (mbar_wait(smem_u32(&sm.q_full), 0, abort_flag, kWaitLimitNs)) {
            mbar_arrive_remote(x_free_peer0);
            mbar_arrive_remote(x_free_peer0 + 8);
            __threadfence_block();
            *reinterpret_cast<volatile int*>(&sm.q_seg) = 1;
          } else {
            fail_timeout(sm, p.err);
          }
        }
      } else {
        const __nv_bfloat16* qt = p.q_tilde + ((int64_t)b * kNH + h) * p.ldqt + 256 * rank;
        const __nv_bfloat16* qp = p.q_pe + ((int64_t)b * kNH + h) * p.ldqp + 32 * rank;
#pragma unroll
        for (int cc = 0; cc < 2; ++cc) {
          const int c = 2 * half + cc;
          uint32_t r[32];
#pragma unroll
          for (int v = 0; v < 8; ++v) {
            const uint4 u = __ldg(reinterpret_cast<const uint4*>(qt + c * 64) + v);
            r[4 * v] = u.x; r[4 * v + 1] = u.y; r[4 * v + 2] = u.z; r[4 * v + 3] = u.w;
          }
          tmem_st32(tQ + c * 32, r);
        }
        if (half == 1) {
          uint32_t r16[16];
#pragma unroll
          for (int v = 0; v < 4; ++v) {
            const uint4 u = __ldg(reinterpret_cast<const uint4*>(qp) + v);
            r16[4 * v] = u.x; r16[4 * v + 1] = u.y; r16[4 * v + 2] = u.z; r16[4 * v + 3] = u.w;
          }
          tmem_st16(tQ + 128, r16);
        }
        tmem_st_wait();
        tc_fence_before();
        warp_arrive(smem_u32(&sm.q_full));
        if (sw == 0 && lane == 0) {
          // every softmax warp has finished the previous segment and copied this one's query
          if (mbar_wait(smem_u32(&sm.q_full), nseg & 1u, abort_flag, kWaitLimitNs)) {
            __threadfence_block();
            *reinterpret_cast<volatile int*>(&sm.q_seg) = (int)nseg + 1;
          } else {
            fail_timeout(sm, p.err);
          }
        }
      }
      float m_run = -INFINITY, l_run = 0.f;
      for (int i = begin; i < end && ok; ++i) {
        // ---- full scores of this tile: own fp16 partial (staging) + the peer's (receive buffer)
        const bool first = (i == begin);
        const uint32_t xi = tb & 1u, use = tb >> 1;
        if (!wait_or_fail(smem_u32(&sm.own_ready[xi]), use & 1u, false)) break;
        if (!wait_or_fail(x_full_l0 + 8 * xi, use & 1u, true)) break;
        float sa[32];
        {
          uint4 mine[4], theirs[4];
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            mine[j] = ld_shared_v4_b32(stg + xi * kXBytes + row_off + ((j ^ swz) << 4));
            theirs[j] = ld_shared_v4_b32(xb + xi * kXBytes + row_off + ((j ^ swz) << 4));
          }
          warp_arrive(smem_u32(&sm.stg_free[xi]));
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const uint32_t a4[4] = {mine[j].x, mine[j].y, mine[j].z, mine[j].w};
            const uint32_t b4[4] = {theirs[j].x, theirs[j].y, theirs[j].z, theirs[j].w};
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              const float2 s2 = unpack_f16x2(hadd2_u32(a4[q], b4[q]));
              sa[8 * j + 2 * q] = s2.x;
              sa[8 * j + 2 * q + 1] = s2.y;
            }
          }
        }
        const int valid = len - i * kTile - 32 * half;  // keys of this half inside the sequence
        if (valid < 32) {
#pragma unroll
          for (int k = 0; k < 32; ++k)
            if (k >= valid) sa[k] = -INFINITY;
        }
        float mx[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) mx[q] = fmaxf(fmaxf(sa[q], sa[q + 4]), fmaxf(sa[q + 8], sa[q + 12]));
#pragma unroll
        for (int q = 0; q < 4; ++q) mx[q] = fmaxf(mx[q], fmaxf(fmaxf(sa[q + 16], sa[q + 20]), fmaxf(sa[q + 24], sa[q + 28])));
        const float lmax = fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3]));
        if (sw == 0 && lane == 0) {
          // all eight softmax warps have read receive buffer xi: the peer may refill it
          if (mbar_wait(smem_u32(&sm.stg_free[xi]), use & 1u, abort_flag, kWaitLimitNs))
            mbar_arrive_remote_relaxed(x_free_peer0 + 8 * xi);
        }
        // rendezvous with the warp holding the other key half of the same heads
        sm.red[xi][half][h] = lmax;
        warp_arrive(smem_u32(&sm.red_bar[xi][quad]));
        if (!wait_or_fail(smem_u32(&sm.red_bar[xi][quad]), use & 1u, false)) break;
        const float m_tile = fmaxf(lmax, sm.red[xi][half ^ 1][h]) * p.scale_log2;
        const float m_new = fmaxf(m_run, m_tile);
        const bool need = first || (m_new > m_run + kRescaleThreshold);
        float corr = 1.f;
        if (need) {
          if (!first) corr = ex2(m_run - m_new);
          m_run = m_new;
        }
        l_run *= corr;
        uint32_t pk[16];
        float ls[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int k = 0; k < 16; ++k) {
          const float p0 = ex2(fmaf(sa[2 * k], p.scale_log2, -m_run));
          const float p1 = ex2(fmaf(sa[2 * k + 1], p.scale_log2, -m_run));
          pk[k] = pack_bf16x2(p0, p1);
          ls[k & 3] += p0 + p1;
        }
        l_run += (ls[0] + ls[1]) + (ls[2] + ls[3]);
        // ---- the previous P*V must be complete before O is rescaled or P is overwritten
        if (!first) {
          if (!wait_or_fail(smem_u32(&sm.pv_done), (tb - 1) & 1u, false)) break;
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
          }
        }
        tmem_st16(tP, pk);
        tmem_st_wait();
        tc_fence_before();
        warp_arrive(smem_u32(&sm.p_full));
        ++tb;
      }
      if (!ok) break;
      // ---- epilogue: O (this CTA's 256 latent features) -> ctx, or a partial for the combine
      if (!wait_or_fail(smem_u32(&sm.pv_done), (tb - 1) & 1u, false)) break;
      tc_fence_after();
      sm.lsum[half][h] = l_run;
      warp_arrive(smem_u32(&sm.sum_bar));
      if (!wait_or_fail(smem_u32(&sm.sum_bar), nseg & 1u, false)) break;
      const float l_tot = l_run + sm.lsum[half ^ 1][h];
      const bool staged = (base + end >= sm.hi);  // the range's last segment: stage buffers idle
      // ctx chunk cc of local head hl, this CTA's latent half and this warp's 128 features
      auto ctx_chunk = [&](int hl, int cc) {
        return reinterpret_cast<uint4*>(p.ctx + ((int64_t)b * kNH + quad * 32 + hl) * kDC + 256 * rank + 128 * half) + cc;
      };
      if (whole) {
        const float inv = 1.f / l_tot;
        __nv_bfloat16* out = p.ctx + ((int64_t)b * kNH + h) * kDC + 256 * rank + 128 * half;
#pragma unroll 1
        for (int c = 0; c < 4; ++c) {
          uint32_t r[32];
          tmem_ld32(tO + c * 32, r);
          tmem_ld_wait();
          uint32_t w[16];
#pragma unroll
          for (int k = 0; k < 16; ++k)
            w[k] = pack_bf16x2(__uint_as_float(r[2 * k]) * inv, __uint_as_float(r[2 * k + 1]) * inv);
          uint4* dst = reinterpret_cast<uint4*>(out + c * 32);
#pragma unroll
          for (int v = 0; v < 4; ++v) {
            if (staged) stage_chunk(4 * c + v, w[4 * v], w[4 * v + 1], w[4 * v + 2], w[4 * v + 3]);
            else dst[v] = make_uint4(w[4 * v], w[4 * v + 1], w[4 * v + 2], w[4 * v + 3]);
          }
        }
        if (staged) flush_staged(ctx_chunk);
        if (rank == 0 && half == 0 && p.lse != nullptr)
          p.lse[(int64_t)b * kNH + h] = (m_run + log2f(l_tot)) * 0.69314718055994531f;
      } else {
        // ---- partial: the last of the sequence's clusters to arrive (per latent half) merges every
        // partial into ctx; the others publish (O, m, l) in their segment's slot and then raise the
        // slot's ready flag.  Counting the arrival first (the producer does, at the segment's last
        // tile) means the merger never writes its own partial, and every cluster it then waits for
        // has already arrived (so it is running) and needs nothing from the merger, so the wait
        // ends.
        const int own = 2 * cl + (first_seg ? 0 : 1);
        // the producer counted the arrival when it issued the segment's last tile
        if (!wait_or_fail(smem_u32(&sm.last_bar), npart & 1u, false)) break;
        ++npart;
        // A partial is this segment's context normalised by its own softmax sum, in bf16: head-major
        // rows of 256 features (512 B) whose 16-byte chunks are rotated by (head & 15), so that eight
        // consecutive heads reading the same chunk hit eight distinct bank groups.  This warp holds
        // features [128 half, 128 half + 128) = chunks [16 half, 16 half + 16) of its head's row.
        const float inv_own = 1.f / l_tot;
        const int cswz = h & 15;
        if (!sm.is_last) {
          uint4* row = reinterpret_cast<uint4*>(p.ws_o) + (((int64_t)own * 2 + rank) * kNH + h) * 32;
#pragma unroll 1
          for (int c = 0; c < 4; ++c) {
            uint32_t r[32];
            tmem_ld32(tO + c * 32, r);
            tmem_ld_wait();
#pragma unroll
            for (int v = 0; v < 4; ++v) {
              const int chunk = 16 * half + 4 * c + v;
              const uint32_t x = pack_bf16x2(__uint_as_float(r[8 * v]) * inv_own, __uint_as_float(r[8 * v + 1]) * inv_own);
              const uint32_t y = pack_bf16x2(__uint_as_float(r[8 * v + 2]) * inv_own, __uint_as_float(r[8 * v + 3]) * inv_own);
              const uint32_t z = pack_bf16x2(__uint_as_float(r[8 * v + 4]) * inv_own, __uint_as_float(r[8 * v + 5]) * inv_own);
              const uint32_t w = pack_bf16x2(__uint_as_float(r[8 * v + 6]) * inv_own, __uint_as_float(r[8 * v + 7]) * inv_own);
              if (staged) stage_chunk(4 * c + v, x, y, z, w);
              else row[chunk ^ cswz] = make_uint4(x, y, z, w);
            }
          }
          if (staged)
            flush_staged([&](int hl, int cc) {
              const int hh = quad * 32 + hl;
              return reinterpret_cast<uint4*>(p.ws_o) + (((int64_t)own * 2 + rank) * kNH + hh) * 32 +
                     ((16 * half + cc) ^ (hh & 15));
            });
          if (half == 0) p.ws_ml[((int64_t)own * 2 + rank) * kNH + h] = make_float2(m_run, l_tot);
          __threadfence();
          warp_arrive(smem_u32(&sm.pub_bar));
          if (sw == 0 && lane == 0) {
            if (mbar_wait(smem_u32(&sm.pub_bar), npub & 1u, abort_flag, kWaitLimitNs)) {
              __threadfence();
              st_release_gpu(p.ws_ready + 2 * (int64_t)own + rank, p.epoch);
            } else {
              fail_timeout(sm, p.err);
            }
          }
          ++npub;
        }
        if (sm.nslots > p.slice_above) {
          // ---- sliced merge: every slot's partial is published (lane 0 of each warp polls the flags,
          // this cluster's own included); this CTA merges heads [h_lo, h_hi) of its latent half, one
          // head per warp and one 16-byte chunk per lane, summing the slots in slot order.  The last
          // cluster to finish its slice resets the flags for the next launch.
          const int ns = sm.nslots;
          int okw = 1;
          if (lane == 0) {
            for (int i = 0; i < ns && okw; ++i)
              okw = wait_flag(p.ws_ready + 2 * (int64_t)sm.slots[i] + rank, p.epoch, abort_flag) ? 1 : 0;
            if (!okw) fail_timeout(sm, p.err);
          }
          if (!__shfl_sync(0xffffffffu, okw, 0)) {
            ok = false;
            break;
          }
          int pos = 0;
          for (int i = 0; i < ns; ++i)
            if (sm.slots[i] == own) pos = i;
          const int h_lo = pos * kNH / ns, h_hi = (pos + 1) * kNH / ns;
          for (int hh = h_lo + sw; hh < h_hi; hh += kSoftmaxWarps) {
            const float2* mlp = p.ws_ml + rank * kNH + hh;  // + slot * 2 * kNH
            float M = -INFINITY;
#pragma unroll 4
            for (int i = 0; i < ns; ++i) M = fmaxf(M, __ldcg(mlp + (int64_t)sm.slots[i] * 2 * kNH).x);
            float L = 0.f;
#pragma unroll 4
            for (int i = 0; i < ns; ++i) {
              const float2 ml = __ldcg(mlp + (int64_t)sm.slots[i] * 2 * kNH);
              L += ml.y * ex2(ml.x - M);
            }
            const float inv = 1.f / L;
            float acc[8];
#pragma unroll
            for (int q = 0; q < 8; ++q) acc[q] = 0.f;
            const uint4* base4 = reinterpret_cast<const uint4*>(p.ws_o) + ((int64_t)rank * kNH + hh) * 32 + (lane ^ (hh & 15));
#pragma unroll 4
            for (int i = 0; i < ns; ++i) {
              const int64_t sl = sm.slots[i];
              const float2 ml = __ldcg(mlp + sl * 2 * kNH);
              const float w = ml.y * ex2(ml.x - M) * inv;
              const uint4 u = __ldcg(base4 + sl * 2 * kNH * 32);
              const uint32_t uw[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
              for (int q = 0; q < 4; ++q) {
                acc[2 * q] = fmaf(w, bf16_lo(uw[q]), acc[2 * q]);
                acc[2 * q + 1] = fmaf(w, bf16_hi(uw[q]), acc[2 * q + 1]);
              }
            }
            *reinterpret_cast<uint4*>(p.ctx + ((int64_t)b * kNH + hh) * kDC + 256 * rank + 8 * lane) =
                make_uint4(pack_bf16x2(acc[0], acc[1]), pack_bf16x2(acc[2], acc[3]), pack_bf16x2(acc[4], acc[5]),
                           pack_bf16x2(acc[6], acc[7]));
            if (rank == 0 && lane == 0 && p.lse != nullptr)
              p.lse[(int64_t)b * kNH + hh] = (M + log2f(L)) * 0.69314718055994531f;
          }
          warp_arrive(smem_u32(&sm.mrg_done));
          if (sw == 0 && lane == 0) {
            if (mbar_wait(smem_u32(&sm.mrg_done), nmd & 1u, abort_flag, kWaitLimitNs)) {
              if (arrive_last(p.ws_ctr + 2 * (int64_t)b + rank, p.epoch, ns, p.err))
                for (int i = 0; i < ns; ++i) p.ws_ready[2 * (int64_t)sm.slots[i] + rank] = 0ull;
            } else {
              fail_timeout(sm, p.err);
            }
          }
          ++nmd;
        } else if (sm.is_last) {
          const int ns = sm.nslots;
          // every other slot's partial has been published (lane 0 of each warp polls the flags)
          int okw = 1;
          if (lane == 0) {
            for (int i = 0; i < ns && okw; ++i)
              if (sm.slots[i] != own)
                okw = wait_flag(p.ws_ready + 2 * (int64_t)sm.slots[i] + rank, p.epoch, abort_flag) ? 1 : 0;
            if (!okw) fail_timeout(sm, p.err);
          }
          if (!__shfl_sync(0xffffffffu, okw, 0)) {
            ok = false;
            break;
          }
          // One other partial, and no further cache tiles will land in the stage buffers (this is the
          // range's last segment and all its P*V products are complete): bulk-load the other
          // partial (64 KB) into the stages.  Otherwise read the partials through L2.
          int other = -1;
          for (int i = 0; i < ns; ++i)
            if (sm.slots[i] != own) other = sm.slots[i];
          const bool bulk = (ns == 2) && (base + end >= sm.hi);
          if (ns > 2 && (ns - 1) * 65536 <= kSmemOff && base + end >= sm.hi) {
            // ---- up to three other partials, and no further cache tiles will land in the stage
            // buffers: all of them are bulk-loaded at once into the free stage / exchange buffers
            // (64 KB each) and merged in registers, in slot order with the arithmetic of the
            // streamed merge below (same result bit for bit); this CTA's own partial is read from
            // its O columns, normalised and rounded through bf16 like a published one.
            // a third partial goes into the exchange buffers: wait until they are quiet
            if (ns - 1 > 2 && !wait_or_fail(smem_u32(&sm.xch_drained), 0, false)) break;
            if (sw == 0 && lane == 0) {
              fence_proxy_async_global();  // the partials were written through the generic proxy
              const uint32_t bar = smem_u32(&sm.mrg_full);
              mbar_arrive_expect_tx(bar, (uint32_t)(ns - 1) * kNH * 512);
              int k = 0;
              for (int i = 0; i < ns; ++i) {
                const int sl = sm.slots[i];
                if (sl == own) continue;
                const uint8_t* src = reinterpret_cast<const uint8_t*>(p.ws_o) + ((int64_t)sl * 2 + rank) * kNH * 512;
                const uint32_t dst = smem_u32(smem) + (uint32_t)k * 65536u;
                bulk_load_g2s(dst, src, 32768, bar);
                bulk_load_g2s(dst + 32768, src + 32768, 32768, bar);
                ++k;
              }
            }
            float M = m_run;
            for (int i = 0; i < ns; ++i)
              if (sm.slots[i] != own) M = fmaxf(M, __ldcg(p.ws_ml + ((int64_t)sm.slots[i] * 2 + rank) * kNH + h).x);
            float L = 0.f;
            for (int i = 0; i < ns; ++i) {
              const int sl = sm.slots[i];
              const float2 ml = sl == own ? make_float2(m_run, l_tot) : __ldcg(p.ws_ml + ((int64_t)sl * 2 + rank) * kNH + h);
              L += ml.y * ex2(ml.x - M);
            }
            const float inv = 1.f / L;
            if (!wait_or_fail(smem_u32(&sm.mrg_full), nmrg & 1u, false)) break;
            ++nmrg;
            __nv_bfloat16* dst = p.ctx + ((int64_t)b * kNH + h) * kDC + 256 * rank + 128 * half;
#pragma unroll 1
            for (int c = 0; c < 4; ++c) {
              uint32_t r[32];
              tmem_ld32(tO + c * 32, r);
              tmem_ld_wait();
              uint32_t ow[16];
#pragma unroll
              for (int k = 0; k < 16; ++k)
                ow[k] = pack_bf16x2(__uint_as_float(r[2 * k]) * inv_own, __uint_as_float(r[2 * k + 1]) * inv_own);
              float acc[32];
#pragma unroll
              for (int q = 0; q < 32; ++q) acc[q] = 0.f;
              int k = 0;
              for (int i = 0; i < ns; ++i) {
                const int sl = sm.slots[i];
                uint32_t uw[16];
                float w;
                if (sl == own) {
                  w = l_tot * ex2(m_run - M) * inv;
#pragma unroll
                  for (int q = 0; q < 16; ++q) uw[q] = ow[q];
                } else {
                  const float2 ml = __ldcg(p.ws_ml + ((int64_t)sl * 2 + rank) * kNH + h);
                  w = ml.y * ex2(ml.x - M) * inv;
                  const uint4* srow = reinterpret_cast<const uint4*>(smem + (size_t)k * 65536) + h * 32;
#pragma unroll
                  for (int v = 0; v < 4; ++v) {
                    const uint4 u = srow[(16 * half + 4 * c + v) ^ cswz];
                    uw[4 * v] = u.x; uw[4 * v + 1] = u.y; uw[4 * v + 2] = u.z; uw[4 * v + 3] = u.w;
                  }
                  ++k;
                }
#pragma unroll
                for (int q = 0; q < 16; ++q) {
                  acc[2 * q] = fmaf(w, bf16_lo(uw[q]), acc[2 * q]);
                  acc[2 * q + 1] = fmaf(w, bf16_hi(uw[q]), acc[2 * q + 1]);
                }
              }
              uint4* d4 = reinterpret_cast<uint4*>(dst + c * 32);
#pragma unroll
              for (int v = 0; v < 4; ++v)
                d4[v] = make_uint4(pack_bf16x2(acc[8 * v], acc[8 * v + 1]), pack_bf16x2(acc[8 * v + 2], acc[8 * v + 3]),
                                   pack_bf16x2(acc[8 * v + 4], acc[8 * v + 5]), pack_bf16x2(acc[8 * v + 6], acc[8 * v + 7]));
            }
            if (rank == 0 && half == 0 && p.lse != nullptr)
              p.lse[(int64_t)b * kNH + h] = (M + log2f(L)) * 0.69314718055994531f;
            if (sw == 0 && lane == 0)
              for (int i = 0; i < ns; ++i)
                if (sm.slots[i] != own) p.ws_ready[2 * (int64_t)sm.slots[i] + rank] = 0ull;
          } else if (ns > 2 && base + end >= sm.hi) {
            // ---- several partials, and no further cache tiles will land in the stage buffers:
            // stream the other partials through two 64 KB stage buffers (bulk loads, one ahead),
            // accumulating in TMEM in slot order.  This CTA's own partial, normalised and rounded
            // to bf16 like a published one, is kept in the TMEM columns the scores, P and the query
            // used (free after the last tile); the O columns become the accumulator.
            int own_pos = 0;
            for (int i = 0; i < ns; ++i)
              if (sm.slots[i] == own) own_pos = i;
            const int n_other = ns - 1;
            const bool issuer = (sw == 0 && lane == 0);
            auto issue = [&](int k) {  // other partial k -> stage buffer k & 1
              const int sl = sm.slots[k < own_pos ? k : k + 1];
              const uint32_t buf = smem_u32(stages) + (k & 1) * 65536;
              const uint32_t bar = smem_u32(&sm.mrg_full2[k & 1]);
              mbar_arrive_expect_tx(bar, kNH * 512);
              const uint8_t* src = reinterpret_cast<const uint8_t*>(p.ws_o) + ((int64_t)sl * 2 + rank) * kNH * 512;
              bulk_load_g2s(buf, src, 32768, bar);
              bulk_load_g2s(buf + 32768, src + 32768, 32768, bar);
            };
            if (issuer) {
              fence_proxy_async_global();  // the partials were written through the generic proxy
              issue(0);
              if (n_other > 1) issue(1);
            }
            float M = m_run;
#pragma unroll 4
            for (int i = 0; i < ns; ++i)
              if (sm.slots[i] != own) M = fmaxf(M, __ldcg(p.ws_ml + ((int64_t)sm.slots[i] * 2 + rank) * kNH + h).x);
            float L = 0.f;
#pragma unroll 4
            for (int i = 0; i < ns; ++i) {
              const int sl = sm.slots[i];
              const float2 ml = sl == own ? make_float2(m_run, l_tot) : __ldcg(p.ws_ml + ((int64_t)sl * 2 + rank) * kNH + h);
              L += ml.y * ex2(ml.x - M);
            }
            const float inv = 1.f / L;
            const uint32_t tStash = tmem + lane_off + kColS + 64 * half;  // 64 columns of bf16 pairs
#pragma unroll 1
            for (int c = 0; c < 4; ++c) {
              uint32_t r[32], pr[16];
              tmem_ld32(tO + c * 32, r);
              tmem_ld_wait();
#pragma unroll
              for (int k = 0; k < 16; ++k)
                pr[k] = pack_bf16x2(__uint_as_float(r[2 * k]) * inv_own, __uint_as_float(r[2 * k + 1]) * inv_own);
              tmem_st16(tStash + 16 * c, pr);
            }
            tmem_st_wait();
            __nv_bfloat16* dst = p.ctx + ((int64_t)b * kNH + h) * kDC + 256 * rank + 128 * half;
            int k = 0;
            bool okm = true;
            for (int i = 0; i < ns && okm; ++i) {
              const int sl = sm.slots[i];
              const bool mine = (sl == own);
              float w;
              const uint4* srow = nullptr;
              if (mine) {
                w = l_tot * ex2(m_run - M) * inv;
              } else {
                if (!wait_or_fail(smem_u32(&sm.mrg_full2[k & 1]), (k >> 1) & 1u, false)) {
                  okm = false;
                  break;
                }
                const float2 ml = __ldcg(p.ws_ml + ((int64_t)sl * 2 + rank) * kNH + h);
                w = ml.y * ex2(ml.x - M) * inv;
                srow = reinterpret_cast<const uint4*>(stages + (k & 1) * 65536) + h * 32;
              }
              const bool last_slot = (i + 1 == ns);
#pragma unroll 1
              for (int c = 0; c < 4; ++c) {
                float acc[32];
                if (i == 0) {
#pragma unroll
                  for (int q = 0; q < 32; ++q) acc[q] = 0.f;
                } else {
                  uint32_t r[32];
                  tmem_ld32(tO + c * 32, r);
                  tmem_ld_wait();
#pragma unroll
                  for (int q = 0; q < 32; ++q) acc[q] = __uint_as_float(r[q]);
                }
                uint32_t uw[16];
                if (mine) {
                  tmem_ld16(tStash + 16 * c, uw);
                  tmem_ld_wait();
                } else {
#pragma unroll
                  for (int v = 0; v < 4; ++v) {
                    const uint4 u = srow[(16 * half + 4 * c + v) ^ cswz];
                    uw[4 * v] = u.x; uw[4 * v + 1] = u.y; uw[4 * v + 2] = u.z; uw[4 * v + 3] = u.w;
                  }
                }
#pragma unroll
                for (int q = 0; q < 16; ++q) {
                  acc[2 * q] = fmaf(w, bf16_lo(uw[q]), acc[2 * q]);
                  acc[2 * q + 1] = fmaf(w, bf16_hi(uw[q]), acc[2 * q + 1]);
                }
                if (last_slot) {
                  uint4* d4 = reinterpret_cast<uint4*>(dst + c * 32);
#pragma unroll
                  for (int v = 0; v < 4; ++v)
                    d4[v] = make_uint4(pack_bf16x2(acc[8 * v], acc[8 * v + 1]), pack_bf16x2(acc[8 * v + 2], acc[8 * v + 3]),
                                       pack_bf16x2(acc[8 * v + 4], acc[8 * v + 5]), pack_bf16x2(acc[8 * v + 6], acc[8 * v + 7]));
                } else {
                  uint32_t r[32];
#pragma unroll
                  for (int q = 0; q < 32; ++q) r[q] = __float_as_uint(acc[q]);
                  tmem_st32(tO + c * 32, r);
                }
              }
              tmem_st_wait();
              if (!mine) {
                // this warp is done with stage buffer k & 1; once all are, it takes partial k + 2
                __syncwarp();
                if (lane == 0) mbar_arrive(smem_u32(&sm.mrg_empty2[k & 1]));
                if (issuer && k + 2 < n_other) {
                  if (mbar_wait(smem_u32(&sm.mrg_empty2[k & 1]), (k >> 1) & 1u, abort_flag, kWaitLimitNs)) issue(k + 2);
                  else fail_timeout(sm, p.err);
                }
                ++k;
              }
            }
            if (!okm) {
              ok = false;
              break;
            }
            if (rank == 0 && half == 0 && p.lse != nullptr)
              p.lse[(int64_t)b * kNH + h] = (M + log2f(L)) * 0.69314718055994531f;
            if (sw == 0 && lane == 0)
              for (int i = 0; i < ns; ++i)
                if (sm.slots[i] != own) p.ws_ready[2 * (int64_t)sm.slots[i] + rank] = 0ull;
          } else {
          if (bulk) {
            if (sw == 0 && lane == 0) {
              fence_proxy_async_global();  // the partial was written through the generic proxy
              const uint32_t bar = smem_u32(&sm.mrg_full);
              mbar_arrive_expect_tx(bar, kNH * 512 + kNH * 8);
              const uint8_t* src = reinterpret_cast<const uint8_t*>(p.ws_o) + ((int64_t)other * 2 + rank) * kNH * 512;
#pragma unroll
              for (int q = 0; q < 2; ++q) bulk_load_g2s(smem_u32(stages) + q * 32768, src + q * 32768, 32768, bar);
              // and its (m, l) pairs, right after the partial
              bulk_load_g2s(smem_u32(stages) + kNH * 512, p.ws_ml + ((int64_t)other * 2 + rank) * kNH, kNH * 8, bar);
            }
            if (!wait_or_fail(smem_u32(&sm.mrg_full), nmrg & 1u, false)) break;
            ++nmrg;
          }
          // Weights of the slots (the softmax sums rescaled to the common maximum), then the sum over
          // the slots in slot order, this CTA's own partial rounded to bf16 like the others: the
          // result does not depend on which cluster arrived last.
          float M, L, w_own = 0.f, w_other = 0.f;
          if (bulk) {
            const float2 ml = reinterpret_cast<const float2*>(stages + kNH * 512)[h];
            M = fmaxf(m_run, ml.x);
            // the same sum in either arrival order: two rounded terms, added once
            const float a = l_tot * ex2(m_run - M), c = ml.y * ex2(ml.x - M);
            L = a + c;
            w_own = a / L;
            w_other = c / L;
          } else {
            M = -INFINITY;
            for (int i = 0; i < ns; ++i) {
              const int sl = sm.slots[i];
              M = fmaxf(M, sl == own ? m_run : __ldcg(p.ws_ml + ((int64_t)sl * 2 + rank) * kNH + h).x);
            }
            L = 0.f;
            for (int i = 0; i < ns; ++i) {
              const int sl = sm.slots[i];
              const float2 ml = sl == own ? make_float2(m_run, l_tot) : __ldcg(p.ws_ml + ((int64_t)sl * 2 + rank) * kNH + h);
              L += ml.y * ex2(ml.x - M);
            }
          }
          const float inv = 1.f / L;
          const uint4* srow = reinterpret_cast<const uint4*>(stages) + h * 32;
          __nv_bfloat16* dst = p.ctx + ((int64_t)b * kNH + h) * kDC + 256 * rank + 128 * half;
#pragma unroll 1
          for (int c = 0; c < 4; ++c) {
            uint32_t r[32];
            tmem_ld32(tO + c * 32, r);
            tmem_ld_wait();
            float own_v[32];  // own partial, normalised and rounded through bf16 like a published one
#pragma unroll
            for (int k = 0; k < 16; ++k) {
              const uint32_t pr = pack_bf16x2(__uint_as_float(r[2 * k]) * inv_own, __uint_as_float(r[2 * k + 1]) * inv_own);
              own_v[2 * k] = bf16_lo(pr);
              own_v[2 * k + 1] = bf16_hi(pr);
            }
            float acc[32];
            if (bulk) {
              // two slots: a sum of two rounded products is the same in either order
#pragma unroll
              for (int v = 0; v < 4; ++v) {
                const uint4 u = srow[(16 * half + 4 * c + v) ^ cswz];
                const uint32_t uw[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                  // both products rounded on their own (no fused multiply-add), so the sum is the
                  // same whichever of the two clusters merges
                  acc[8 * v + 2 * q] = __fadd_rn(__fmul_rn(w_own, own_v[8 * v + 2 * q]), __fmul_rn(w_other, bf16_lo(uw[q])));
                  acc[8 * v + 2 * q + 1] =
                      __fadd_rn(__fmul_rn(w_own, own_v[8 * v + 2 * q + 1]), __fmul_rn(w_other, bf16_hi(uw[q])));
                }
              }
            } else {
#pragma unroll
              for (int k = 0; k < 32; ++k) acc[k] = 0.f;
              for (int i = 0; i < ns; ++i) {
                const int sl = sm.slots[i];
                if (sl == own) {
                  const float w = l_tot * ex2(m_run - M) * inv;
#pragma unroll
                  for (int k = 0; k < 32; ++k) acc[k] = fmaf(w, own_v[k], acc[k]);
                } else {
                  const float2 ml = __ldcg(p.ws_ml + ((int64_t)sl * 2 + rank) * kNH + h);
                  const float w = ml.y * ex2(ml.x - M) * inv;
                  const uint4* grow = reinterpret_cast<const uint4*>(p.ws_o) + (((int64_t)sl * 2 + rank) * kNH + h) * 32;
#pragma unroll
                  for (int v = 0; v < 4; ++v) {
                    const uint4 u = __ldcg(grow + ((16 * half + 4 * c + v) ^ cswz));
                    const uint32_t uw[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                      acc[8 * v + 2 * q] = fmaf(w, bf16_lo(uw[q]), acc[8 * v + 2 * q]);
                      acc[8 * v + 2 * q + 1] = fmaf(w, bf16_hi(uw[q]), acc[8 * v + 2 * q + 1]);
                    }
                  }
                }
              }
            }
            uint4* d4 = reinterpret_cast<uint4*>(dst + c * 32);
#pragma unroll
            for (int v = 0; v < 4; ++v) {
              const uint32_t x = pack_bf16x2(acc[8 * v], acc[8 * v + 1]), y = pack_bf16x2(acc[8 * v + 2], acc[8 * v + 3]);
              const uint32_t z = pack_bf16x2(acc[8 * v + 4], acc[8 * v + 5]), w = pack_bf16x2(acc[8 * v + 6], acc[8 * v + 7]);
              if (bulk) stage_chunk(4 * c + v, x, y, z, w);  // (bulk: the range's last segment)
              else d4[v] = make_uint4(x, y, z, w);
            }
          }
          if (bulk) flush_staged(ctx_chunk);
          if (rank == 0 && half == 0 && p.lse != nullptr)
            p.lse[(int64_t)b * kNH + h] = (M + log2f(L)) * 0.69314718055994531f;
          // the flags go back to zero for the next launch (which may reuse this launch's epoch when
          // it replays a captured graph)
          if (sw == 0 && lane == 0)
            for (int i = 0; i < ns; ++i)
              if (sm.slots[i] != own) p.ws_ready[2 * (int64_t)sm.slots[i] + rank] = 0ull;
          }
        }
      }
      first_seg = false;
      ++nseg;
    }
  }

  // ---------------------------------------------------------------------- teardown
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, kTmemCols);
  cluster_sync();  // neither CTA leaves while the peer may still touch its shared memory
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

// Workspace layout for n_clusters clusters and B sequences: partial O, partial (m, l), counters.
size_t ws_o_bytes(size_t nc) { return 2 * nc * 2 * 128 * 256 * sizeof(__nv_bfloat16); }
size_t ws_ml_bytes(size_t nc) { return 2 * nc * 2 * 128 * sizeof(float2); }
size_t ws_ready_bytes(size_t nc) { return 2 * nc * 2 * sizeof(unsigned long long); }
size_t ws_bytes(size_t nc, size_t B) {
  return ws_o_bytes(nc) + ws_ml_bytes(nc) + ws_ready_bytes(nc) + B * 2 * sizeof(unsigned long long) + 256;
}

// A launch identifier for the arrival counters: unique within the process (a 56-bit counter
// started from the clock), never 0.
unsigned long long next_epoch() {
  static std::atomic<unsigned long long> counter{
      (unsigned long long)std::chrono::steady_clock::now().time_since_epoch().count() * 0x9E3779B97F4A7C15ull};
  unsigned long long e = 0;
  while (e == 0) e = counter.fetch_add(1, std::memory_order_relaxed) & ((1ull << 56) - 1);
  return e;
}

// Upper bound of clusters: one CTA pair per two SMs (sizes the workspace).
int max_clusters() {
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int n = sms / 2 < kMaxClusters ? sms / 2 : kMaxClusters;
  return n > 0 ? n : 1;
}

// Clusters of the persistent grid: as many CTA pairs as can be resident at once (GPCs with an odd
// number of free SMs cannot host a full pair), so that the grid is exactly one wave.  `one_wave`
// records whether the occupancy query confirmed that (when it fails the grid takes the upper bound
// and the sliced merge, which needs every cluster resident, is not used).  Cached per device.
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
  if (cudaFuncSetAttribute(decode_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem_bytes()) ==
      cudaSuccess) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(2 * upper);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = smem_bytes();
    int active = 0;
    if (cudaOccupancyMaxActiveClusters(&active, decode_kernel<false>, &cfg) == cudaSuccess && active > 0) {
      w.clusters = active < upper ? active : upper;
      w.one_wave = true;
    }
  }
  cudaGetLastError();  // a failed query leaves no sticky state
  if (dev >= 0 && dev < 64) cache[dev] = w;
  return w;
}

}  // namespace decode_tc

size_t decode_tc_workspace(int B) { return decode_tc::ws_bytes(decode_tc::max_clusters(), B > 0 ? B : 0); }

cudaError_t decode_tc_launch(const DecodeArgs& a, void* ws, cudaStream_t st) {
  using namespace decode_tc;
  const Wave wave = grid_wave();
  const int nc = wave.clusters;
  Params p;
  memset(&p, 0, sizeof(p));
  const uint64_t bstride_c = a.B > 1 ? (uint64_t)a.ckv_b * 2 : (uint64_t)a.n_max * a.ckv_r * 2;
  const uint64_t bstride_r = a.B > 1 ? (uint64_t)a.kr_b * 2 : (uint64_t)a.n_max * a.kr_r * 2;
  // (the FP8 cache has no bf16 latent rows: its map is made below)
  if ((a.c8 == nullptr && !make_map_3d(&p.tm_ckv, a.c_kv, kDC, a.n_max, a.B, (uint64_t)a.ckv_r * 2, bstride_c, 64,
                                       kTile, CU_TENSOR_MAP_SWIZZLE_128B)) ||
      !make_map_3d(&p.tm_kr, a.k_r, kDR, a.n_max, a.B, (uint64_t)a.kr_r * 2, bstride_r, 32, kTile,
                   CU_TENSOR_MAP_SWIZZLE_64B))
    return cudaErrorInvalidValue;
  {
    const uint64_t qd[2] = {(uint64_t)kDC, (uint64_t)a.B * kNH}, qs[1] = {(uint64_t)a.ldqt * 2};
    const uint64_t rd[2] = {(uint64_t)kDR, (uint64_t)a.B * kNH}, rs[1] = {(uint64_t)a.ldqp * 2};
    const uint32_t qbox[2] = {64, kNH}, rbox[2] = {32, kNH};
    if (!make_tensor_map_bf16(&p.tm_q, a.q_tilde, 2, qd, qs, qbox, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !make_tensor_map_bf16(&p.tm_qp, a.q_pe, 2, rd, rs, rbox, CU_TENSOR_MAP_SWIZZLE_64B))
      return cudaErrorInvalidValue;
  }
  if (a.topk > 0) {
    // sparse: rows of the caches addressed as sequence * n_max + position (their batch stride is
    // n_max rows; the caller checked)
    p.topk_idx = a.topk_idx;
    p.topk = a.topk;
    p.c_kv_base = static_cast<const __nv_bfloat16*>(a.c_kv);
    p.k_r_base = static_cast<const __nv_bfloat16*>(a.k_r);
    p.ckv_row = a.ckv_r;
    p.kr_row = a.kr_r;
  }
  p.q_tilde = static_cast<const __nv_bfloat16*>(a.q_tilde);
  p.ldqt = a.ldqt;
  p.q_pe = static_cast<const __nv_bfloat16*>(a.q_pe);
  p.ldqp = a.ldqp;
  p.lengths = a.lengths;
  p.B = a.B;
  p.n_max = a.n_max;
  p.n_clusters = nc;
  p.slice_above = sliced_merge_allowed(wave.one_wave) ? kMergeLastMax : 0x7fffffff;
  p.scale_log2 = a.scale * 1.4426950408889634f;
  p.ctx = static_cast<__nv_bfloat16*>(a.ctx);
  p.lse = a.lse;
  uint8_t* w = static_cast<uint8_t*>(ws);
  p.ws_o = reinterpret_cast<float*>(w);
  w += ws_o_bytes(nc);
  p.ws_ml = reinterpret_cast<float2*>(w);
  w += ws_ml_bytes(nc);
  p.ws_ready = reinterpret_cast<unsigned long long*>(w);
  w += ws_ready_bytes(nc);
  p.ws_ctr = reinterpret_cast<unsigned long long*>(w);
  p.epoch = next_epoch();
  p.err = a.err;

  const size_t smem = smem_bytes();
  if (a.c8 != nullptr) {
    // FP8 latent cache: e4m3 rows (byte strides) and fp32 scales (4 per row), one tile's rows per box
    const uint64_t cb = a.B > 1 ? (uint64_t)a.c8_b : (uint64_t)a.n_max * a.c8_r;
    const uint64_t sb = a.B > 1 ? (uint64_t)a.sc_b * 4 : (uint64_t)a.n_max * a.sc_r * 4;
    const uint64_t d8[3] = {(uint64_t)kDC, (uint64_t)a.n_max, (uint64_t)a.B}, s8[2] = {(uint64_t)a.c8_r, cb};
    const uint64_t ds[3] = {4, (uint64_t)a.n_max, (uint64_t)a.B}, ss[2] = {(uint64_t)a.sc_r * 4, sb};
    const uint32_t b8[3] = {256, kTile, 1}, bs[3] = {4, kTile, 1};
    if (!make_tensor_map(&p.tm_c8, CU_TENSOR_MAP_DATA_TYPE_UINT8, a.c8, 3, d8, s8, b8, CU_TENSOR_MAP_SWIZZLE_NONE) ||
        !make_tensor_map(&p.tm_sc, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, a.kv_scale, 3, ds, ss, bs,
                         CU_TENSOR_MAP_SWIZZLE_NONE))
      return cudaErrorInvalidValue;
    cudaError_t e = cudaFuncSetAttribute(decode_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    return launch_pdl(decode_kernel<true>, dim3(2 * nc), dim3(kThreads), smem, st, p);
  }
  cudaError_t e = cudaFuncSetAttribute(decode_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  return launch_pdl(decode_kernel<false>, dim3(2 * nc), dim3(kThreads), smem, st, p);
}

// ------------------------------------------------------------------------------------------
// Built-in scratch of mla_decode_absorb_static
// ------------------------------------------------------------------------------------------
// Some callers cannot allocate device memory when they run a decode: a plugin or engine host
// whose enqueue callback may not call cudaMalloc (it would synchronise or break the host's memory
// budget), or a caller that only holds pointers handed to it by someone else.  For them the split-KV scratch lives in this
// file-scope array, which every GPU that loads the library holds until the process exits.
// Sized for 74 clusters (one CTA pair per two SMs of a 148-SM B200) and up to 4096 sequences:
// 74 x 2 partial slots of 128 heads x 512 bf16 features, their (m, l) pairs and ready flags, and
// two arrival counters per sequence, about 18.9 MiB.
namespace {
constexpr size_t kStaticMaxClusters = 74;
constexpr size_t kStaticMaxBatch = 4096;
constexpr size_t kStaticScratchBytes = 2 * kStaticMaxClusters * 2 * 128 * 256 * sizeof(__nv_bfloat16) +
                                       2 * kStaticMaxClusters * 2 * 128 * sizeof(float2) +
                                       2 * kStaticMaxClusters * 2 * sizeof(unsigned long long) +
                                       kStaticMaxBatch * 2 * sizeof(unsigned long long) + 256;
static __device__ __align__(256) unsigned char g_decode_scratch[kStaticScratchBytes];
}  // namespace

size_t decode_static_scratch_bytes() { return kStaticScratchBytes; }

// Device address of the array on the current device.  Host code may not use the array's name as a
// device pointer (it is a host-side stand-in), so the address is looked up once per device, with
// that device current, and cached.
cudaError_t decode_static_scratch(void** out) {
  static std::mutex mu;
  static void* addr[64] = {nullptr};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(mu);
  if (addr[dev] == nullptr) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_decode_scratch);
    if (e != cudaSuccess) return e;
    addr[dev] = p;
  }
  *out = addr[dev];
  return cudaSuccess;
}

}  // namespace mla

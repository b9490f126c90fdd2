// Absorbed MLA decode on tcgen05 tensor cores (sm_100a): attention of one query token per
// sequence directly over the latent cache ("Absorb key weights", decode excerpt:
// scores = scale (q~ . c^KV_t + q^R . k^R_t), softmax over positions, ctx = sum alpha c^KV_t).
//
// Design (one CTA pair = one thread-block cluster of 2 per work range, 1 CTA per SM):
// * The 128 heads of one sequence are the M = 128 rows of every MMA.
// * TMEM (512 columns) cannot hold the fp32 context of 128 heads x 512 latent features plus a
//   score tile, so the pair splits the latent axis: CTA r owns latent features
//   [256 r, 256 r + 256) and rotary features [32 r, 32 r + 32).  Each CTA loads only its half of
//   every cached row (no byte is loaded twice), computes the PARTIAL score tile over its 288
//   features, and the two partials are exchanged through distributed shared memory (st.async,
//   completion counted on the receiver's mbarrier), so both CTAs hold identical full scores and
//   run the identical online softmax.
// * Per 64-key tile: TMA brings the CTA's half rows (4 x 128-byte-swizzled slabs + a 64-byte-
//   swizzled rotary slab) into a 4-stage ring; S = Q K^T runs with Q held in TMEM (A operand)
//   and K in shared memory; P (bf16) is written to TMEM and O += P V reads V from the SAME
//   shared-memory tile (K-major for the scores, MN-major for the values).
// * Softmax: 8 warps, two per TMEM lane quadrant; the two warps of a quadrant split each tile's
//   64 keys (32 each) and agree on the row maximum through shared memory.  The per-tile work is
//   software-pipelined: phase A(t) reads S(t) from TMEM and ships the partial to the peer,
//   phase B(t) adds the peer's partial and does the softmax; the order A(t+1), B(t) keeps one
//   exchange in flight while the previous tile is normalised, and lets the score MMA of tile
//   t+1 run while the softmax of tile t-1 is still busy.
// * Online softmax in base 2 with the scale folded in; the running maximum is only raised (and
//   O rescaled in TMEM) when it grows by more than 8, so rescales are rare.
// * Split-KV: the sequence axis of all sequences is cut into equal contiguous tile ranges, one
//   per cluster (balanced for ragged lengths); a range that covers a whole sequence writes ctx
//   directly, the others write fp32 partials (O, m, l) and a combine kernel merges them.
// * Warp roles: warp 0 = TMA producer, warp 1 = TMEM allocator + MMA issuer, warps 2..9 =
//   softmax, exchange, rescale and epilogue.
// * Every wait is a bounded mbarrier wait (global timer); on expiry the kernel records
//   MLA_ERR_TIMEOUT, drains and returns.
#include <cuda.h>
#include <cuda_bf16.h>
#include <math.h>
#include <string.h>

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
constexpr int kSoftmaxWarps = 8;                // two per TMEM lane quadrant
constexpr int kPvWarp = 2;                      // the warp that issues the P*V MMAs
constexpr int kAWarp0 = 3;                      // 4 exchange warps, one per TMEM lane quadrant
constexpr int kBWarp0 = 7;                      // 8 softmax warps
constexpr int kThreads = 32 * (kBWarp0 + kSoftmaxWarps);
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColO = 0, kColS = 256, kColP = 320, kColQ = 352;  // Q: 128 + 16 columns
constexpr float kRescaleThreshold = 8.0f;       // log2 units
constexpr uint64_t kWaitLimitNs = 1000000000ull;

struct Params {
  CUtensorMap tm_ckv;  // 3-D (d_c, n_max, B), box (64, 64, 1), 128-byte swizzle
  CUtensorMap tm_kr;   // 3-D (d_r, n_max, B), box (32, 64, 1), 64-byte swizzle
  const __nv_bfloat16* q_tilde;
  int64_t ldqt;
  const __nv_bfloat16* q_pe;
  int64_t ldqp;
  const int32_t* lengths;
  int B, n_max, n_clusters;
  float scale_log2;
  __nv_bfloat16* ctx;
  float* lse;
  float* ws_o;     // [2 n_clusters slots][2 halves][128][256] fp32, unnormalised
  float2* ws_ml;   // [2 n_clusters slots][128] (running max in log2 units, sum)
  int32_t* ws_plan;  // [n_clusters] first sequence of each cluster's range
  int32_t* err;
};

struct Smem {
  uint64_t full[kStages], empty[kStages];
  uint64_t q_full, s_full, s_empty, p_full, pv_done, drain;
  uint64_t x_full[2], x_free[2];   // exchange buffers (double-buffered by tile parity)
  uint64_t own_ready[2], stg_free[2];  // this CTA's fp16 partial staged / read by the softmax warps
  uint64_t red_bar[2][4], sum_bar; // row-max rendezvous of the two warps of a lane quadrant / final sum
  float red[2][2][kNH];            // [tile parity][key half][head] partial row max
  float lsum[2][kNH];              // [key half][head] partial softmax sum
  uint32_t tmem_base;
  int abort;
  int lo, hi, b0, t_b0;
};

__device__ __forceinline__ int clamp_len(int len, int n_max) { return len < 0 ? 0 : (len > n_max ? n_max : len); }
__device__ __forceinline__ int tiles_of(int len) { return (len + kTile - 1) / kTile; }

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Contiguous tile range [lo, hi) of cluster c among n_clusters over all sequences' tiles.
__device__ __forceinline__ int range_lo(long long c, long long total, long long nc) { return (int)((c * total) / nc); }

// One warp: total tiles, this cluster's range, and the first sequence of the range.
__device__ void plan_range(const Params& p, int c, Smem& sm, int lane) {
  long long total = 0;
  bool bad = false;
  for (int b0 = 0; b0 < p.B; b0 += 32) {
    const int b = b0 + lane;
    int t = 0;
    if (b < p.B) {
      const int len = p.lengths[b];
      bad |= (len < 1 || len > p.n_max);
      t = tiles_of(clamp_len(len, p.n_max));
    }
    for (int o = 16; o > 0; o >>= 1) t += __shfl_xor_sync(0xffffffffu, t, o);
    total += t;
  }
  if (__any_sync(0xffffffffu, bad) && lane == 0 && c == 0 && cluster_ctarank() == 0) raise_error(p.err, MLA_ERR_LENGTH);
  const int lo = range_lo(c, total, p.n_clusters), hi = range_lo(c + 1, total, p.n_clusters);
  int first_b = p.B, t_first = 0;
  if (lo < hi) {
    int base = 0;  // tiles before batch b0
    for (int b0 = 0; b0 < p.B && first_b == p.B; b0 += 32) {
      const int b = b0 + lane;
      const int t = b < p.B ? tiles_of(clamp_len(p.lengths[b], p.n_max)) : 0;
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
  if (lane == 0) {
    sm.lo = lo;
    sm.hi = hi;
    sm.b0 = first_b;
    sm.t_b0 = t_first;
  }
}

// Walks the segments (sequence, first tile, end tile) of this cluster's range.
struct SegIter {
  int b, tb, t, hi;
  const int32_t* lengths;
  int n_max, B;
  __device__ SegIter(const Smem& sm, const Params& p) : b(sm.b0), tb(sm.t_b0), t(sm.lo), hi(sm.hi),
                                                        lengths(p.lengths), n_max(p.n_max), B(p.B) {}
  // On success: sequence b, tiles [begin, end) of it, its length, whether the range holds all of it.
  __device__ bool next(int& sb, int& begin, int& end, int& len, bool& whole) {
    while (t < hi && b < B) {
      len = clamp_len(lengths[b], n_max);
      const int nt = tiles_of(len);
      if (tb + nt <= t) {  // sequence entirely before t (or empty)
        tb += nt;
        ++b;
        continue;
      }
      sb = b;
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

__device__ __forceinline__ void fail_timeout(Smem& sm, int32_t* err) {
  raise_error(err, MLA_ERR_TIMEOUT);
  sm.abort = 1;
}

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
    decode_kernel(const __grid_constant__ Params p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* stages = smem;
  uint8_t* xbuf = smem + kStages * kStageBytes;  // 2 receive + 2 staging exchange buffers
  Smem& sm = *reinterpret_cast<Smem*>(smem + kStages * kStageBytes + 4 * kXBytes);
  volatile int* abort_flag = &sm.abort;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank(), peer = rank ^ 1u;
  const int cl = blockIdx.x >> 1;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(smem_u32(&sm.full[s]), 1);
      mbar_init(smem_u32(&sm.empty[s]), 1);
    }
    // softmax-side arrivals are one per softmax warp, after a __syncwarp
    mbar_init(smem_u32(&sm.q_full), kSoftmaxWarps);
    mbar_init(smem_u32(&sm.s_full), 1);
    mbar_init(smem_u32(&sm.s_empty), 4);  // the four exchange warps
    mbar_init(smem_u32(&sm.p_full), kSoftmaxWarps);
    mbar_init(smem_u32(&sm.pv_done), 1);
    mbar_init(smem_u32(&sm.drain), 2);  // one commit from each MMA-issuing thread
    for (int i = 0; i < 2; ++i) {
      mbar_init(smem_u32(&sm.x_full[i]), 1);  // 1 local arrive.expect_tx + the peer's st.async bytes
      mbar_init(smem_u32(&sm.x_free[i]), 1);  // 1 remote arrive from the peer
      mbar_init(smem_u32(&sm.own_ready[i]), 4);
      mbar_init(smem_u32(&sm.stg_free[i]), kSoftmaxWarps);
      for (int q = 0; q < 4; ++q) mbar_init(smem_u32(&sm.red_bar[i][q]), 2);
    }
    mbar_init(smem_u32(&sm.sum_bar), kSoftmaxWarps);
    sm.abort = 0;
    fence_mbar_init();
    prefetch_tensormap(&p.tm_ckv);
    prefetch_tensormap(&p.tm_kr);
  }
  if (warp == 0) plan_range(p, cl, sm, lane);
  if (warp == 1) {
    tmem_alloc(smem_u32(&sm.tmem_base), kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  cluster_sync();  // the peer's barriers are initialised before any remote arrive
  const uint32_t tmem = sm.tmem_base;
  if (threadIdx.x == 0 && rank == 0) p.ws_plan[cl] = sm.b0;

  if (warp == 0) {
    // ------------------------------------------------------------------ TMA producer
    if (lane == 0) {
      const uint64_t pol = policy_evict_first();
      SegIter seg(sm, p);
      int b, begin, end, len;
      bool whole;
      uint32_t it = 0;
      bool ok = true;
      while (ok && seg.next(b, begin, end, len, whole)) {
        for (int i = begin; i < end && ok; ++i, ++it) {
          const uint32_t st = it % kStages, ph = (it / kStages) & 1u;
          if (!mbar_wait(smem_u32(&sm.empty[st]), ph ^ 1u, abort_flag, kWaitLimitNs)) {
            fail_timeout(sm, p.err);
            ok = false;
            break;
          }
          const uint32_t dst = smem_u32(stages + st * kStageBytes);
          const uint32_t bar = smem_u32(&sm.full[st]);
          mbar_arrive_expect_tx(bar, kStageBytes);
#pragma unroll
          for (int s = 0; s < 4; ++s)
            tma_load_3d(dst + s * kSlabBytes, &p.tm_ckv, bar, 256 * (int)rank + 64 * s, i * kTile, b, pol);
          tma_load_3d(dst + kLatBytes, &p.tm_kr, bar, 32 * (int)rank, i * kTile, b, pol);
        }
      }
      // drain: every load issued must have landed before the CTA may exit
      const uint32_t first = it > (uint32_t)kStages ? it - kStages : 0;
      for (uint32_t k = first; k < it; ++k)
        mbar_wait(smem_u32(&sm.full[k % kStages]), (k / kStages) & 1u, abort_flag, kWaitLimitNs);
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
    int b, begin, end, len;
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
      const uint32_t st = t % kStages;
      if (!wait_or_fail(smem_u32(&sm.full[st]), (t / kStages) & 1u, false)) return;
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
    // O += P(t) V(t) over this CTA's 256 latent features
    auto issue_pv = [&](uint32_t t, bool first_of_seg) {
      if (!wait_or_fail(smem_u32(&sm.p_full), t & 1u, false)) return;
      tc_fence_after();
      const uint32_t st = t % kStages;
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
    while (ok && seg.next(b, begin, end, len, whole)) {
      if (is_qk) {
        if (!wait_or_fail(smem_u32(&sm.q_full), nseg & 1u, false)) break;
        tc_fence_after();
        for (int i = begin; i < end && ok; ++i) issue_qk(it++, i);
      } else {
        for (int i = begin; i < end && ok; ++i) issue_pv(it++, i == begin);
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
      // staging xi is free once the peer consumed tile t - 2 (so its copy is done) and this CTA's
      // softmax warps have read it
      if (!wait_or_fail(smem_u32(&sm.x_free[xi]), (use & 1u) ^ 1u, true)) break;
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
  } else {
    // ------------------------------------------------------------------ softmax warps (kBWarp0..)
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
    SegIter seg(sm, p);
    int b, begin, end, len;
    bool whole;
    uint32_t tb = 0;           // global tile counter
    uint32_t nseg = 0;
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
    while (ok && seg.next(b, begin, end, len, whole)) {
      // ---- this sequence's query half into TMEM (A operand of the score MMA)
      {
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
          for (int v = 0; v < 4; ++v) dst[v] = make_uint4(w[4 * v], w[4 * v + 1], w[4 * v + 2], w[4 * v + 3]);
        }
        if (rank == 0 && half == 0 && p.lse != nullptr)
          p.lse[(int64_t)b * kNH + h] = (m_run + log2f(l_tot)) * 0.69314718055994531f;
      } else {
        const int slot = 2 * cl + (first_seg ? 0 : 1);
        float* out = p.ws_o + (((int64_t)slot * 2 + rank) * kNH + h) * 256 + 128 * half;
#pragma unroll 1
        for (int c = 0; c < 4; ++c) {
          uint32_t r[32];
          tmem_ld32(tO + c * 32, r);
          tmem_ld_wait();
          uint4* dst = reinterpret_cast<uint4*>(out + c * 32);
#pragma unroll
          for (int v = 0; v < 8; ++v) dst[v] = make_uint4(r[4 * v], r[4 * v + 1], r[4 * v + 2], r[4 * v + 3]);
        }
        if (rank == 0 && half == 0) p.ws_ml[(int64_t)slot * kNH + h] = make_float2(m_run, l_tot);
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
// Combine: merge the fp32 partials of sequences whose tiles span several clusters
// ------------------------------------------------------------------------------------------
__global__ void __launch_bounds__(256) combine_kernel(const __grid_constant__ Params p) {
  const int b = blockIdx.x;
  const int h0 = blockIdx.y * 8;
  __shared__ int s_info[4];  // c_lo, c_hi, tiles of b, total tiles
  if (threadIdx.x < 32) {
    const int lane = threadIdx.x;
    long long total = 0, before = 0;
    for (int b0 = 0; b0 < p.B; b0 += 32) {
      const int bb = b0 + lane;
      int t = bb < p.B ? tiles_of(clamp_len(p.lengths[bb], p.n_max)) : 0;
      int tb = bb < b ? t : 0;
      for (int o = 16; o > 0; o >>= 1) {
        t += __shfl_xor_sync(0xffffffffu, t, o);
        tb += __shfl_xor_sync(0xffffffffu, tb, o);
      }
      total += t;
      before += tb;
    }
    if (lane == 0) {
      const int nt = tiles_of(clamp_len(p.lengths[b], p.n_max));
      const long long nc = p.n_clusters;
      auto cluster_of = [&](long long t) {
        long long c = (t * nc) / (total > 0 ? total : 1);
        while (c + 1 < nc && range_lo(c + 1, total, nc) <= t) ++c;
        while (c > 0 && range_lo(c, total, nc) > t) --c;
        return (int)c;
      };
      s_info[2] = nt;
      s_info[3] = (int)total;
      s_info[0] = nt > 0 ? cluster_of(before) : 0;
      s_info[1] = nt > 0 ? cluster_of(before + nt - 1) : 0;
    }
  }
  __syncthreads();
  const int c_lo = s_info[0], c_hi = s_info[1], nt = s_info[2];
  if (nt == 0) {  // empty sequence: zero context, lse = -inf
    for (int i = threadIdx.x; i < 8 * kDC; i += blockDim.x)
      p.ctx[((int64_t)b * kNH + h0 + i / kDC) * kDC + i % kDC] = __float2bfloat16_rn(0.f);
    if (p.lse && threadIdx.x < 8) p.lse[(int64_t)b * kNH + h0 + threadIdx.x] = -INFINITY;
    return;
  }
  if (c_lo == c_hi) return;  // one cluster held the whole sequence and wrote ctx itself
  // ---- the partial slots of this sequence, resolved once (clusters with an empty range hold none)
  constexpr int kMaxSlots = 256;
  __shared__ int s_slot[kMaxSlots];
  __shared__ int s_nslot;
  __shared__ float s_w[8][kMaxSlots];  // per head: e^{m_s - M} / L, the weight of partial s
  if (threadIdx.x == 0) {
    const long long total = s_info[3], nc = p.n_clusters;
    int ns = 0;
    long long lo = range_lo(c_lo, total, nc);
    for (int c = c_lo; c <= c_hi && ns < kMaxSlots; ++c) {
      const long long hi = range_lo(c + 1, total, nc);
      if (hi > lo) s_slot[ns++] = 2 * c + (p.ws_plan[c] == b ? 0 : 1);
      lo = hi;
    }
    s_nslot = ns;
  }
  __syncthreads();
  const int ns = s_nslot;
  {  // one warp per head: running-max merge of (m_s, l_s)
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, hh = h0 + warp;
    float M = -INFINITY;
    for (int s = lane; s < ns; s += 32) M = fmaxf(M, p.ws_ml[(int64_t)s_slot[s] * kNH + hh].x);
    M = warp_max(M);
    float L = 0.f;
    for (int s = lane; s < ns; s += 32) {
      const float2 ml = p.ws_ml[(int64_t)s_slot[s] * kNH + hh];
      const float w = ex2(ml.x - M);
      s_w[warp][s] = w;
      L += w * ml.y;
    }
    L = warp_sum(L);
    const float inv = 1.f / L;
    for (int s = lane; s < ns; s += 32) s_w[warp][s] *= inv;
    if (lane == 0 && p.lse) p.lse[(int64_t)b * kNH + hh] = (M + log2f(L)) * 0.69314718055994531f;
  }
  __syncthreads();
  for (int i = threadIdx.x; i < 8 * (kDC / 4); i += blockDim.x) {
    const int hl = i / (kDC / 4), hh = h0 + hl, d = (i % (kDC / 4)) * 4;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int s = 0; s < ns; ++s) {
      const float w = s_w[hl][s];
      const float4 o = *reinterpret_cast<const float4*>(
          p.ws_o + (((int64_t)s_slot[s] * 2 + (d >> 8)) * kNH + hh) * 256 + (d & 255));
      acc.x += w * o.x; acc.y += w * o.y; acc.z += w * o.z; acc.w += w * o.w;
    }
    __nv_bfloat16* out = p.ctx + ((int64_t)b * kNH + hh) * kDC + d;
    *reinterpret_cast<uint2*>(out) = make_uint2(pack_bf16x2(acc.x, acc.y), pack_bf16x2(acc.z, acc.w));
  }
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

size_t smem_bytes() { return (size_t)kStages * kStageBytes + 4 * kXBytes + sizeof(Smem) + 1024; }

// Upper bound of clusters: one CTA pair per two SMs (sizes the workspace).
int max_clusters() {
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  return sms / 2 > 0 ? sms / 2 : 1;
}

// Clusters that can be resident at once (GPCs with an odd number of free SMs cannot host a full
// pair), so that the persistent grid is exactly one wave.  Cached per device.
int num_clusters() {
  static int cache[64] = {0};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev >= 0 && dev < 64 && cache[dev] > 0) return cache[dev];
  const int upper = max_clusters();
  int n = upper;
  if (cudaFuncSetAttribute(decode_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem_bytes()) ==
      cudaSuccess) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(2 * upper);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = smem_bytes();
    int active = 0;
    if (cudaOccupancyMaxActiveClusters(&active, decode_kernel, &cfg) == cudaSuccess && active > 0 && active < n)
      n = active;
  }
  cudaGetLastError();  // a failed query leaves no sticky state; keep the upper bound
  if (dev >= 0 && dev < 64) cache[dev] = n;
  return n;
}

}  // namespace decode_tc

size_t decode_tc_workspace(int B) {
  (void)B;
  const size_t nc = decode_tc::max_clusters();
  return 2 * nc * (2 * 128 * 256 * sizeof(float)) + 2 * nc * 128 * sizeof(float2) + nc * sizeof(int32_t) + 1024;
}

cudaError_t decode_tc_launch(const DecodeArgs& a, void* ws, cudaStream_t st) {
  using namespace decode_tc;
  const int nc = num_clusters();
  Params p;
  memset(&p, 0, sizeof(p));
  const uint64_t bstride_c = a.B > 1 ? (uint64_t)a.ckv_b * 2 : (uint64_t)a.n_max * a.ckv_r * 2;
  const uint64_t bstride_r = a.B > 1 ? (uint64_t)a.kr_b * 2 : (uint64_t)a.n_max * a.kr_r * 2;
  if (!make_map_3d(&p.tm_ckv, a.c_kv, kDC, a.n_max, a.B, (uint64_t)a.ckv_r * 2, bstride_c, 64, kTile,
                   CU_TENSOR_MAP_SWIZZLE_128B) ||
      !make_map_3d(&p.tm_kr, a.k_r, kDR, a.n_max, a.B, (uint64_t)a.kr_r * 2, bstride_r, 32, kTile,
                   CU_TENSOR_MAP_SWIZZLE_64B))
    return cudaErrorInvalidValue;
  p.q_tilde = static_cast<const __nv_bfloat16*>(a.q_tilde);
  p.ldqt = a.ldqt;
  p.q_pe = static_cast<const __nv_bfloat16*>(a.q_pe);
  p.ldqp = a.ldqp;
  p.lengths = a.lengths;
  p.B = a.B;
  p.n_max = a.n_max;
  p.n_clusters = nc;
  p.scale_log2 = a.scale * 1.4426950408889634f;
  p.ctx = static_cast<__nv_bfloat16*>(a.ctx);
  p.lse = a.lse;
  uint8_t* w = static_cast<uint8_t*>(ws);
  p.ws_o = reinterpret_cast<float*>(w);
  w += 2 * (size_t)nc * (2 * 128 * 256 * sizeof(float));
  p.ws_ml = reinterpret_cast<float2*>(w);
  w += 2 * (size_t)nc * 128 * sizeof(float2);
  p.ws_plan = reinterpret_cast<int32_t*>(w);
  p.err = a.err;

  const size_t smem = smem_bytes();
  cudaError_t e = cudaFuncSetAttribute(decode_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  decode_kernel<<<2 * nc, kThreads, smem, st>>>(p);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  combine_kernel<<<dim3(a.B, kNH / 8), 256, 0, st>>>(p);
  return cudaGetLastError();
}

// ------------------------------------------------------------------------------------------
// Built-in scratch of mla_decode_absorb_static
// ------------------------------------------------------------------------------------------
// Some callers cannot allocate device memory when they run a decode: a plugin or engine host
// whose enqueue callback may not call cudaMalloc (it would synchronise or break the host's memory
// budget), code issuing work while a stream is being captured into a CUDA graph, or a caller that
// only holds pointers handed to it by someone else.  For them the split-KV scratch lives in this
// file-scope array, which every GPU that loads the library holds until the process exits.
// Sized for 74 clusters (one CTA pair per two SMs of a 148-SM B200): 74 x 2 partial slots of
// 128 heads x 512 fp32 features, their (m, l) pairs and the per-cluster plan, about 37.1 MiB.
namespace {
constexpr size_t kStaticMaxClusters = 74;
constexpr size_t kStaticScratchBytes = 2 * kStaticMaxClusters * (2 * 128 * 256 * sizeof(float)) +
                                       2 * kStaticMaxClusters * 128 * sizeof(float2) +
                                       kStaticMaxClusters * sizeof(int32_t) + 1024;
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

// Naive-path prefill on tcgen05 tensor cores (sm_100a), bf16 in / fp32 accumulation, for the
// DeepSeek-V3 dimensions (128 heads, d_c = 512, d_h = d_v = 128, d_R = 64).
//
// Expansion ("Naive path": the key/value up-projection wkv_b applied to every cached latent row):
//   kv[r, n] = sum_c c_KV[r, c] W_kv_b[n, c]      r = (sequence, position), n = (head, k_nope | v)
// a plain GEMM of M = B S rows, N = 128 * 256 = 32768 columns, K = 512.
//
// Design: one persistent CTA per SM walks 128 x 256 output tiles.  Warp 0 streams 64-wide K slabs
// of both operands with TMA (128-byte swizzle) through a 3-stage ring; warp 1 issues the MMAs
// (M = 128, N = 256, K = 16) into one of two TMEM accumulators (256 columns each), so the next
// tile's MMAs run while warps 2-5 drain the previous accumulator: TMEM -> registers -> bf16 ->
// a swizzled shared-memory tile -> TMA stores.  Every wait is bounded (global timer) and reports
// MLA_ERR_TIMEOUT.
#include <cuda.h>
#include <cuda_bf16.h>
#include <string.h>

#include "common.cuh"
#include "kernels.h"
#include "sm100_ptx.cuh"
#include "tma_host.h"

namespace mla {
namespace prefill_tc {

using namespace sm100;

constexpr int BM = 128, BN = 256, BK = 64;
constexpr int kStages = 3;
constexpr int kABytes = BM * BK * 2;              // 16 KB: 128 rows x 64 features
constexpr int kBBytes = BN * BK * 2;              // 32 KB: 256 rows x 64 features
constexpr int kStageBytes = kABytes + kBBytes;
constexpr int kOutBoxBytes = BM * 128;            // one 128-row x 64-column bf16 store box
constexpr int kOutOff = kStages * kStageBytes;    // shared-memory layout: stages | output tile | barriers
constexpr int kBarOff = kOutOff + 4 * kOutBoxBytes;
constexpr int kThreads = 192;                     // warp 0 loads, warp 1 MMAs, warps 2-5 epilogue
constexpr uint64_t kWaitLimitNs = 1000000000ull;

struct Params {
  CUtensorMap tm_a;    // 2-D (K, M): latent rows, box (64, 128), 128-byte swizzle
  CUtensorMap tm_b;    // 2-D (K, N): wkv_b rows, box (64, 256), 128-byte swizzle
  CUtensorMap tm_out;  // 2-D (N, M): expanded rows, box (64, 128), 128-byte swizzle (stores)
  int m_tiles, n_tiles, k_slabs;
  int32_t* err;
};

struct Bars {
  uint64_t full[kStages], empty[kStages];
  uint64_t acc_full[2], acc_empty[2];
  uint32_t tmem_base;
  int abort;
};

__device__ __forceinline__ void tma_store_2d(const CUtensorMap* map, uint32_t src, int x, int y) {
  asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%2, %3}], [%1];" ::"l"(
                   reinterpret_cast<uint64_t>(map)),
               "r"(src), "r"(x), "r"(y)
               : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait_read0() { asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait0() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

__global__ void __launch_bounds__(kThreads, 1) expand_kernel(const __grid_constant__ Params p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  Bars& bs = *reinterpret_cast<Bars*>(smem + kBarOff);
  volatile int* abort_flag = &bs.abort;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n_total = p.m_tiles * p.n_tiles;

  griddep_launch_dependents();
  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(smem_u32(&bs.full[s]), 1);
      mbar_init(smem_u32(&bs.empty[s]), 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(smem_u32(&bs.acc_full[a]), 1);
      mbar_init(smem_u32(&bs.acc_empty[a]), 4);
    }
    bs.abort = 0;
    fence_mbar_init();
    prefetch_tensormap(&p.tm_a);
    prefetch_tensormap(&p.tm_b);
    prefetch_tensormap(&p.tm_out);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(&bs.tmem_base), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bs.tmem_base;

  if (warp == 0) {
    // ---------------------------------------------------------------- TMA producer
    if (lane == 0) {
      griddep_wait();  // the latent rows may come from the preceding kernel
      const uint64_t pol = policy_evict_last();  // both operands are re-read by other tiles
      uint32_t it = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < n_total && ok; t += gridDim.x) {
        const int mt = t % p.m_tiles, nt = t / p.m_tiles;
        for (int kc = 0; kc < p.k_slabs; ++kc, ++it) {
          const uint32_t st = it % kStages, ph = (it / kStages) & 1u;
          if (!mbar_wait(smem_u32(&bs.empty[st]), ph ^ 1u, abort_flag, kWaitLimitNs)) {
            raise_error(p.err, MLA_ERR_TIMEOUT);
            bs.abort = 1;
            ok = false;
            break;
          }
          const uint32_t dst = smem_u32(smem + st * kStageBytes);
          const uint32_t bar = smem_u32(&bs.full[st]);
          mbar_arrive_expect_tx(bar, kStageBytes);
          tma_load_2d(dst, &p.tm_a, bar, BK * kc, BM * mt, pol);
          tma_load_2d(dst + kABytes, &p.tm_b, bar, BK * kc, BN * nt, pol);
        }
      }
      // every load issued has landed before the CTA may exit
      const uint32_t first = it > (uint32_t)kStages ? it - kStages : 0;
      for (uint32_t k = first; k < it; ++k)
        mbar_wait(smem_u32(&bs.full[k % kStages]), (k / kStages) & 1u, abort_flag, kWaitLimitNs);
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA issuer
    const uint32_t idesc = idesc_bf16_f32(BM, BN, 0, 0);
    uint32_t it = 0, i = 0;
    bool ok = true;
    auto wait_all = [&](uint32_t bar, uint32_t par) {
      const bool mine = mbar_wait(bar, par, abort_flag, kWaitLimitNs);
      if (!__all_sync(0xffffffffu, mine)) {
        if (lane == 0) {
          raise_error(p.err, MLA_ERR_TIMEOUT);
          bs.abort = 1;
        }
        ok = false;
      }
      return ok;
    };
    for (int t = blockIdx.x; t < n_total && ok; t += gridDim.x, ++i) {
      const uint32_t a = i & 1u;
      if (!wait_all(smem_u32(&bs.acc_empty[a]), ((i >> 1) & 1u) ^ 1u)) break;
      tc_fence_after();
      const uint32_t tacc = tmem + 256 * a;
      for (int kc = 0; kc < p.k_slabs && ok; ++kc, ++it) {
        const uint32_t st = it % kStages;
        if (!wait_all(smem_u32(&bs.full[st]), (it / kStages) & 1u)) break;
        tc_fence_after();
        if (lane == 0) {
          const uint32_t abase = smem_u32(smem + st * kStageBytes), bbase = abase + kABytes;
#pragma unroll
          for (int k = 0; k < BK / 16; ++k)
            mma_ss(tacc, smem_desc(abase + 32 * k, 16, 1024, kSwizzle128), smem_desc(bbase + 32 * k, 16, 1024, kSwizzle128),
                   idesc, (kc | k) ? 1u : 0u);
          mma_commit(smem_u32(&bs.empty[st]));
        }
        __syncwarp();
      }
      if (lane == 0) mma_commit(smem_u32(&bs.acc_full[a]));
      __syncwarp();
    }
  } else {
    // ---------------------------------------------------------------- epilogue (warps 2-5)
    const int quad = warp & 3;
    const int r = 32 * quad + lane;  // accumulator row of this thread
    const uint32_t lane_off = (uint32_t)(32 * quad) << 16;
    const uint32_t obase = smem_u32(smem + kOutOff);
    const bool leader = (warp == 2 && lane == 0);
    griddep_wait();  // the expanded rows may still be read by the preceding kernel
    uint32_t i = 0;
    for (int t = blockIdx.x; t < n_total; t += gridDim.x, ++i) {
      const int mt = t % p.m_tiles, nt = t / p.m_tiles;
      const uint32_t a = i & 1u;
      const bool mine = mbar_wait(smem_u32(&bs.acc_full[a]), (i >> 1) & 1u, abort_flag, kWaitLimitNs);
      if (!__all_sync(0xffffffffu, mine)) {
        if (lane == 0) {
          raise_error(p.err, MLA_ERR_TIMEOUT);
          bs.abort = 1;
        }
        break;
      }
      tc_fence_after();
      // the previous tile's stores have read the output tile
      if (leader) bulk_wait_read0();
      named_bar_sync(1, 128);
#pragma unroll 1
      for (int bx = 0; bx < 4; ++bx) {
        uint32_t v[64];
        {
          uint32_t r0[32], r1[32];
          tmem_ld32(tmem + lane_off + 256 * a + 64 * bx, r0);
          tmem_ld32(tmem + lane_off + 256 * a + 64 * bx + 32, r1);
          tmem_ld_wait();
#pragma unroll
          for (int k = 0; k < 32; ++k) {
            v[k] = r0[k];
            v[32 + k] = r1[k];
          }
        }
        const uint32_t row = obase + bx * kOutBoxBytes + r * 128;
#pragma unroll
        for (int j = 0; j < 8; ++j)
          st_shared_v4_b32(row + ((j ^ (r & 7)) << 4),
                           pack_bf16x2(__uint_as_float(v[8 * j]), __uint_as_float(v[8 * j + 1])),
                           pack_bf16x2(__uint_as_float(v[8 * j + 2]), __uint_as_float(v[8 * j + 3])),
                           pack_bf16x2(__uint_as_float(v[8 * j + 4]), __uint_as_float(v[8 * j + 5])),
                           pack_bf16x2(__uint_as_float(v[8 * j + 6]), __uint_as_float(v[8 * j + 7])));
      }
      // the accumulator may take the next tile; the tile goes out with TMA stores
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&bs.acc_empty[a]));
      fence_proxy_async_smem();
      named_bar_sync(1, 128);
      if (leader) {
#pragma unroll
        for (int bx = 0; bx < 4; ++bx) tma_store_2d(&p.tm_out, obase + bx * kOutBoxBytes, BN * nt + 64 * bx, BM * mt);
        bulk_commit();
      }
    }
    if (leader) bulk_wait0();  // every store complete before the CTA exits
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, 512);
}

size_t smem_bytes() { return (size_t)kBarOff + sizeof(Bars) + 1024; }
static_assert(kBarOff + sizeof(Bars) + 1024 <= 232448, "dynamic shared memory above the 227 KB per-CTA limit");

// ------------------------------------------------------------------------------------------
// Causal attention of the naive path ("Naive path": k = [k_nope; k_R broadcast], scores
// q . k / sqrt(192), softmax over positions t <= s, output sum_t alpha_t v_t), per (sequence,
// head, mirrored pair of 128-query tiles):
//   * Q (128 x 192) is TMA-loaded once and read from shared memory by the score MMAs;
//   * K tiles (128 keys: k_nope from the expanded rows, k_R shared by the heads) and V tiles stream
//     through two 2-stage TMA rings (a K stage is released by its score MMA, a V stage by its P.V);
//   * S goes to one of three TMEM buffers; the softmax (4 warps, one query row per thread) takes the
//     row maximum, then writes P = 2^(s - m) as bf16 over the same columns, and P.V reads it from
//     TMEM (A operand) while the next S is computed into another buffer;
//   * online softmax in base 2, the running maximum raised (and O rescaled) only when it grows by
//     more than 8.
// ------------------------------------------------------------------------------------------
constexpr int AT_TILE = 128;                      // queries per query tile, keys per key tile
constexpr int AT_SLAB = AT_TILE * 128;            // 128 rows x 64 bf16 (128-byte swizzle)
constexpr int AT_QOFF = 0;                        // Q: 3 slabs (q_nope 0-63, 64-127, q_pe)
constexpr int AT_STAGES = 2;                      // K and V rings of two stages each
constexpr int AT_K0 = 3 * AT_SLAB;                // K stage: k_nope 0-63, 64-127, k_R
constexpr int AT_KBYTES = 3 * AT_SLAB;
constexpr int AT_V0 = AT_K0 + AT_STAGES * AT_KBYTES;  // V stage: v 0-63, 64-127
constexpr int AT_VBYTES = 2 * AT_SLAB;
constexpr int AT_BAROFF = AT_V0 + AT_STAGES * AT_VBYTES;
constexpr int AT_THREADS = 192;                   // warp 0 loads, warp 1 MMAs, warps 2-5 softmax
constexpr int AT_SBUF = 3;                        // score buffers in TMEM
constexpr uint32_t AT_COL_S = 0, AT_COL_O = 384;  // S 3 x 128 columns, O 128

struct AttnParams {
  CUtensorMap tm_q;   // 4-D (192, H, S, B) query rows, box (64, 1, 128, 1)
  CUtensorMap tm_kv;  // 4-D (256, H, S, B) expanded rows (k_nope | v), box (64, 1, 128, 1)
  CUtensorMap tm_kr;  // 3-D (64, S, B) shared rotary keys, box (64, 128, 1)
  __nv_bfloat16* out; // [B][S][H][128]
  int B, S, H, n_qt, causal;
  float scale_log2;
  int32_t* err;
  // sparse variant: each query row's selected key positions (already cut to t <= s) as a bitmap,
  // and per (sequence, query tile) the compact list of key tiles any of its rows selects
  const uint32_t* bitmap;   // [B][S][row_words]
  int row_words;            // 4 * n_qt (128 bits per key tile)
  const int32_t* tile_list; // [B][n_qt][n_qt]
  const int32_t* tile_count;// [B][n_qt]
};

struct AttnBars {
  uint64_t q_tma, q_free, kfull[AT_STAGES], kempty[AT_STAGES], vfull[AT_STAGES], vempty[AT_STAGES];
  uint64_t s_full[AT_SBUF], p_full[AT_SBUF], pv_done[AT_SBUF];
  uint32_t tmem_base;
  int abort;
};

// Non-blocking check of an mbarrier phase: when the phase has already completed it answers
// without the suspend-and-wake of try_wait.
__device__ __forceinline__ bool mbar_test_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}

template <bool kSparse>
__global__ void __launch_bounds__(AT_THREADS, 1) attn_kernel(const __grid_constant__ AttnParams p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  AttnBars& bs = *reinterpret_cast<AttnBars*>(smem + AT_BAROFF);
  volatile int* abort_flag = &bs.abort;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // A CTA takes a mirrored pair of query tiles of one (sequence, head), the longest causal rows
  // first and then the shortest (n_qt + 1 key tiles together, the same for every pair), so the
  // grid is balanced and half as large; the second tile's query load and first score MMAs overlap
  // the first's tail.  The pairs of one (sequence, head) are consecutive blocks: blocks that run
  // together share that head's K/V tiles in L2.
  const int n_pairs = (p.n_qt + 1) / 2;
  const int idx = blockIdx.x;
  const int pi = idx % n_pairs, h = (idx / n_pairs) % p.H, b = idx / (n_pairs * p.H);
  const int n_items = (p.n_qt - 1 - pi != pi) ? 2 : 1;
  auto item_qt = [&](int it) { return it == 0 ? p.n_qt - 1 - pi : pi; };
  // key tiles attended by query tile `it`, and the j-th of them
  auto item_nkv = [&](int it) {
    if (kSparse) return p.tile_count[b * p.n_qt + item_qt(it)];
    return p.causal ? item_qt(it) + 1 : p.n_qt;
  };
  auto key_tile = [&](int it, int j) {
    return kSparse ? p.tile_list[((int64_t)b * p.n_qt + item_qt(it)) * p.n_qt + j] : j;
  };

  griddep_launch_dependents();
  if (threadIdx.x == 0) {
    mbar_init(smem_u32(&bs.q_tma), 1);
    mbar_init(smem_u32(&bs.q_free), 1);
    for (int i = 0; i < AT_STAGES; ++i) {
      mbar_init(smem_u32(&bs.kfull[i]), 1);
      mbar_init(smem_u32(&bs.kempty[i]), 1);
      mbar_init(smem_u32(&bs.vfull[i]), 1);
      mbar_init(smem_u32(&bs.vempty[i]), 1);
    }
    for (int i = 0; i < AT_SBUF; ++i) {
      mbar_init(smem_u32(&bs.s_full[i]), 1);
      mbar_init(smem_u32(&bs.p_full[i]), 4);
      mbar_init(smem_u32(&bs.pv_done[i]), 1);
    }
    bs.abort = 0;
    fence_mbar_init();
    prefetch_tensormap(&p.tm_q);
    prefetch_tensormap(&p.tm_kv);
    prefetch_tensormap(&p.tm_kr);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(&bs.tmem_base), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bs.tmem_base;
  auto fail = [&]() {
    raise_error(p.err, MLA_ERR_TIMEOUT);
    bs.abort = 1;
  };

  if (warp == 0) {
    // ---------------------------------------------------------------- TMA producer
    // Key tiles g = 0 .. G-1 of both query tiles in one sequence (global tile counter g).  K and V
    // go through separate rings: a K stage is free once its score MMA has read it, a V stage once
    // its P.V has, so the next key tile's load is not held behind the current softmax.  K runs one
    // tile ahead of V in issue order.  The second query tile's rows replace the first's in shared
    // memory once every score MMA of the first has completed.
    if (lane == 0) {
      griddep_wait();  // the expanded rows come from the preceding kernel
      const uint64_t pol = policy_evict_last();
      const uint32_t qb = smem_u32(&bs.q_tma);
      const int n_kv0 = item_nkv(0);
      const int G = n_kv0 + (n_items > 1 ? item_nkv(1) : 0);
      auto key_row = [&](int g) { return AT_TILE * (g < n_kv0 ? key_tile(0, g) : key_tile(1, g - n_kv0)); };
      bool ok = true;
      int nk = 0, nv = 0;  // K and V tiles issued
      mbar_arrive_expect_tx(qb, 3 * AT_SLAB);
      for (int sl = 0; sl < 3; ++sl)
        tma_load_4d(smem_u32(smem + AT_QOFF + sl * AT_SLAB), &p.tm_q, qb, 64 * sl, h, AT_TILE * item_qt(0), b, pol);
      for (int s = 0; s <= G && ok; ++s) {
        if (s < G) {
          const int g = s;
          const uint32_t st = g % AT_STAGES, ph = (g / AT_STAGES) & 1u;
          if (!mbar_wait(smem_u32(&bs.kempty[st]), ph ^ 1u, abort_flag, kWaitLimitNs)) {
            fail();
            ok = false;
            break;
          }
          const uint32_t dst = smem_u32(smem + AT_K0 + st * AT_KBYTES);
          const uint32_t bar = smem_u32(&bs.kfull[st]);
          mbar_arrive_expect_tx(bar, AT_KBYTES);
          tma_load_4d(dst, &p.tm_kv, bar, 0, h, key_row(g), b, pol);             // k_nope 0-63
          tma_load_4d(dst + AT_SLAB, &p.tm_kv, bar, 64, h, key_row(g), b, pol);  // k_nope 64-127
          tma_load_3d(dst + 2 * AT_SLAB, &p.tm_kr, bar, 0, key_row(g), b, pol);  // k_R
          ++nk;
          if (g == n_kv0) {  // second query tile: its rows, once the first's score MMAs are done
            if (!mbar_wait(smem_u32(&bs.q_free), 0u, abort_flag, kWaitLimitNs)) {
              fail();
              ok = false;
              break;
            }
            mbar_arrive_expect_tx(qb, 3 * AT_SLAB);
            for (int sl = 0; sl < 3; ++sl)
              tma_load_4d(smem_u32(smem + AT_QOFF + sl * AT_SLAB), &p.tm_q, qb, 64 * sl, h, AT_TILE * item_qt(1), b, pol);
          }
        }
        if (s >= 1) {
          const int g = s - 1;
          const uint32_t st = g % AT_STAGES, ph = (g / AT_STAGES) & 1u;
          if (!mbar_wait(smem_u32(&bs.vempty[st]), ph ^ 1u, abort_flag, kWaitLimitNs)) {
            fail();
            ok = false;
            break;
          }
          const uint32_t dst = smem_u32(smem + AT_V0 + st * AT_VBYTES);
          const uint32_t bar = smem_u32(&bs.vfull[st]);
          mbar_arrive_expect_tx(bar, AT_VBYTES);
          tma_load_4d(dst, &p.tm_kv, bar, 128, h, key_row(g), b, pol);            // v 0-63
          tma_load_4d(dst + AT_SLAB, &p.tm_kv, bar, 192, h, key_row(g), b, pol);  // v 64-127
          ++nv;
        }
      }
      // drain: every load issued must have landed before the CTA may exit
      for (int k = nk > AT_STAGES ? nk - AT_STAGES : 0; k < nk; ++k)
        mbar_wait(smem_u32(&bs.kfull[k % AT_STAGES]), (k / AT_STAGES) & 1u, abort_flag, kWaitLimitNs);
      for (int k = nv > AT_STAGES ? nv - AT_STAGES : 0; k < nv; ++k)
        mbar_wait(smem_u32(&bs.vfull[k % AT_STAGES]), (k / AT_STAGES) & 1u, abort_flag, kWaitLimitNs);
      mbar_wait(qb, (uint32_t)(n_items - 1) & 1u, abort_flag, kWaitLimitNs);
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA issuer
    const uint32_t idesc_qk = idesc_bf16_f32(128, AT_TILE, 0, 0);
    const uint32_t idesc_pv = idesc_bf16_f32(128, 128, 0, 1);
    bool ok = true;
    auto wait_all = [&](uint32_t bar, uint32_t par) {
      if (!ok) return false;
      const bool mine = mbar_test_wait(bar, par) || mbar_wait(bar, par, abort_flag, kWaitLimitNs);
      if (!__all_sync(0xffffffffu, mine)) {
        if (lane == 0) fail();
        ok = false;
      }
      return ok;
    };
    // O += P(g) V(g); `first`: the query tile's first key tile (O starts from it)
    auto issue_pv = [&](int g, bool first) {
      if (!wait_all(smem_u32(&bs.p_full[g % AT_SBUF]), (g / AT_SBUF) & 1u)) return;
      if (!wait_all(smem_u32(&bs.vfull[g % AT_STAGES]), (g / AT_STAGES) & 1u)) return;
      tc_fence_after();
      if (lane == 0) {
        const uint32_t vb = smem_u32(smem + AT_V0 + (g % AT_STAGES) * AT_VBYTES);
        const uint32_t tP = tmem + AT_COL_S + 128 * (g % AT_SBUF);
#pragma unroll
        for (int k = 0; k < AT_TILE / 16; ++k)
          mma_ts(tmem + AT_COL_O, tP + 8 * k, smem_desc(vb + 2048 * k, AT_SLAB, 1024, kSwizzle128), idesc_pv,
                 (!first || k > 0) ? 1u : 0u);
        mma_commit(smem_u32(&bs.vempty[g % AT_STAGES]));
        mma_commit(smem_u32(&bs.pv_done[g % AT_SBUF]));
      }
      __syncwarp();
    };
    int g = 0;
    for (int it = 0; it < n_items && ok; ++it) {
      const int n_kv = item_nkv(it);
      if (!wait_all(smem_u32(&bs.q_tma), (uint32_t)it & 1u)) break;  // this query tile's rows landed
      tc_fence_after();
      for (int j = 0; j < n_kv && ok; ++j, ++g) {
        // S(g) = Q K(g)^T into buffer g % 3, free once P.V(g - 3) has read the P it held: with three
        // buffers that product was issued a whole tile earlier, so the score MMA does not wait
        // for the tensor pipe to drain
        if (!wait_all(smem_u32(&bs.kfull[g % AT_STAGES]), (g / AT_STAGES) & 1u)) break;
        if (g >= AT_SBUF && !wait_all(smem_u32(&bs.pv_done[g % AT_SBUF]), ((g - AT_SBUF) / AT_SBUF) & 1u)) break;
        tc_fence_after();
        if (lane == 0) {
          const uint32_t kb = smem_u32(smem + AT_K0 + (g % AT_STAGES) * AT_KBYTES);
          const uint32_t tS = tmem + AT_COL_S + 128 * (g % AT_SBUF);
          const uint32_t qs = smem_u32(smem + AT_QOFF);
#pragma unroll
          for (int k = 0; k < 12; ++k)  // 8 K-steps of q_nope . k_nope, 4 of q_pe . k_R
            mma_ss(tS, smem_desc(qs + (k >> 2) * AT_SLAB + 32 * (k & 3), 16, 1024, kSwizzle128),
                   smem_desc(kb + (k >> 2) * AT_SLAB + 32 * (k & 3), 16, 1024, kSwizzle128), idesc_qk, k > 0 ? 1u : 0u);
          mma_commit(smem_u32(&bs.s_full[g % AT_SBUF]));
          mma_commit(smem_u32(&bs.kempty[g % AT_STAGES]));
          if (j == n_kv - 1 && it + 1 < n_items) mma_commit(smem_u32(&bs.q_free));  // query rows reusable
        }
        __syncwarp();
        if (j >= 1) issue_pv(g - 1, j == 1);  // P.V of the previous tile behind this tile's scores
      }
      if (ok && n_kv > 0) issue_pv(g - 1, n_kv == 1);
    }
  } else {
    // ---------------------------------------------------------------- softmax (warps 2-5)
    const int quad = warp & 3;
    const int r = 32 * quad + lane;               // query row of this thread within the tile
    const uint32_t lane_off = (uint32_t)(32 * quad) << 16;
    const uint32_t tO = tmem + lane_off + AT_COL_O;
    bool ok = true;
    auto wait_all = [&](uint32_t bar, uint32_t par) {
      if (!ok) return false;
      const bool mine = mbar_test_wait(bar, par) || mbar_wait(bar, par, abort_flag, kWaitLimitNs);
      if (!__all_sync(0xffffffffu, mine)) {
        if (lane == 0) fail();
        ok = false;
      }
      return ok;
    };
    int g = 0;
    for (int it = 0; it < n_items && ok; ++it) {
      const int qt = item_qt(it), n_kv = item_nkv(it);
      const int q_pos = AT_TILE * qt + r;         // this row's position in the sequence
      float m_run = -INFINITY, l_run = 0.f;
      for (int j = 0; j < n_kv && ok; ++j, ++g) {
        if (!wait_all(smem_u32(&bs.s_full[g % AT_SBUF]), (g / AT_SBUF) & 1u)) break;
        tc_fence_after();
        const uint32_t tS = tmem + lane_off + AT_COL_S + 128 * (g % AT_SBUF);
        const int key0 = AT_TILE * key_tile(it, j);
        // keys of this tile this row may attend: below the sequence length and (causal) <= q_pos
        const int lim = p.causal ? min(p.S - 1, q_pos) : p.S - 1;
        const int nvalid = lim - key0 + 1;  // keys 0 .. nvalid-1 of the tile are valid
        // the whole score row in registers: four loads, one wait (the row is read from TMEM once)
        uint32_t sv[4][32];
#pragma unroll
        for (int c = 0; c < 4; ++c) tmem_ld32(tS + 32 * c, sv[c]);
        tmem_ld_wait();
        // masked keys (past the row's causal limit or the sequence end; only the diagonal and the
        // last tile have any) become -inf: they leave the maximum alone and 2^-inf = 0
        if (kSparse) {
          // the row's selected keys of this tile: 128 bits (causal and length already applied);
          // rows past the sequence end select nothing
          uint4 bits = make_uint4(0u, 0u, 0u, 0u);
          if (q_pos < p.S)
            bits = *reinterpret_cast<const uint4*>(p.bitmap + ((int64_t)b * p.S + q_pos) * p.row_words + (key0 >> 5));
          const uint32_t bw[4] = {bits.x, bits.y, bits.z, bits.w};
#pragma unroll
          for (int c = 0; c < 4; ++c)
#pragma unroll
            for (int k = 0; k < 32; ++k)
              sv[c][k] = (bw[c] >> k) & 1u ? sv[c][k] : 0xff800000u;
        } else if (nvalid < AT_TILE) {
#pragma unroll
          for (int c = 0; c < 4; ++c)
#pragma unroll
            for (int k = 0; k < 32; ++k)
              sv[c][k] = 32 * c + k < nvalid ? sv[c][k] : 0xff800000u;
        }
        // row maximum and (below) row sum as eight and four independent chains, so the one warp
        // on each sub-partition is not stalled on a 128-long dependency chain
        float mxv[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) mxv[k] = __uint_as_float(sv[0][k]);
#pragma unroll
        for (int i = 8; i < AT_TILE; ++i) mxv[i & 7] = fmaxf(mxv[i & 7], __uint_as_float(sv[i >> 5][i & 31]));
        const float mx = fmaxf(fmaxf(fmaxf(mxv[0], mxv[1]), fmaxf(mxv[2], mxv[3])),
                               fmaxf(fmaxf(mxv[4], mxv[5]), fmaxf(mxv[6], mxv[7])));
        const float m_new = fmaxf(m_run, mx * p.scale_log2);
        const bool need = m_new > m_run + 8.0f;  // true on the first tile (m_run = -inf)
        if (j > 0 && __any_sync(0xffffffffu, need)) {
          // O holds P.V of the earlier tiles relative to the old maximum: rescale it once the
          // last of those products has landed
          if (!wait_all(smem_u32(&bs.pv_done[(g - 1) % AT_SBUF]), ((g - 1) / AT_SBUF) & 1u)) break;
          tc_fence_after();
          const float corr = need ? ex2f_approx(m_run - m_new) : 1.f;
#pragma unroll 1
          for (int c = 0; c < 4; ++c) {
            uint32_t v[32];
            tmem_ld32(tO + 32 * c, v);
            tmem_ld_wait();
#pragma unroll
            for (int k = 0; k < 32; ++k) v[k] = __float_as_uint(__uint_as_float(v[k]) * corr);
            tmem_st32(tO + 32 * c, v);
          }
        }
        if (need) {
          l_run = (m_run == -INFINITY) ? 0.f : l_run * ex2f_approx(m_run - m_new);
          m_run = m_new;
        }
        // P = 2^(s scale_log2 - m) in bf16, written over the scores it came from (chunk c of P takes
        // columns [16c, 16c + 16); the whole row is already in registers)
        // a sparse row with no selected key so far keeps m = -inf: its scores are all -inf, so any
        // finite reference gives P = 0 (a -inf reference would give 2^NaN)
        const float m_ref = (kSparse && m_run == -INFINITY) ? 0.f : m_run;
        float lsv[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          uint32_t pk[16];
#pragma unroll
          for (int k = 0; k < 16; ++k) {
            const float p0 = ex2f_approx(fmaf(__uint_as_float(sv[c][2 * k]), p.scale_log2, -m_ref));
            const float p1 = ex2f_approx(fmaf(__uint_as_float(sv[c][2 * k + 1]), p.scale_log2, -m_ref));
            lsv[k & 3] += p0 + p1;
            pk[k] = pack_bf16x2(p0, p1);
          }
          tmem_st16(tS + 16 * c, pk);
        }
        l_run += (lsv[0] + lsv[1]) + (lsv[2] + lsv[3]);
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(&bs.p_full[g % AT_SBUF]));
      }
      if (!ok) break;
      // ---- epilogue of this query tile: O / l -> out, once its last P.V (and so every earlier one)
      // has completed
      if (n_kv >= 1 && wait_all(smem_u32(&bs.pv_done[(g - 1) % AT_SBUF]), ((g - 1) / AT_SBUF) & 1u)) {
        tc_fence_after();
        // a sparse row that selected no visible key has no softmax: it is written as zeros and flagged
        const bool empty_row = kSparse && !(l_run > 0.f);
        if (empty_row && q_pos < p.S) raise_error(p.err, MLA_ERR_INDEX);
        const float inv = empty_row ? 0.f : 1.f / l_run;
#pragma unroll 1
        for (int c = 0; c < 4; ++c) {
          uint32_t v[32];
          tmem_ld32(tO + 32 * c, v);
          tmem_ld_wait();
          if (q_pos < p.S) {
            uint4* dst = reinterpret_cast<uint4*>(p.out + (((int64_t)b * p.S + q_pos) * p.H + h) * 128 + 32 * c);
#pragma unroll
            for (int w = 0; w < 4; ++w)
              dst[w] = make_uint4(pack_bf16x2(__uint_as_float(v[8 * w]) * inv, __uint_as_float(v[8 * w + 1]) * inv),
                                  pack_bf16x2(__uint_as_float(v[8 * w + 2]) * inv, __uint_as_float(v[8 * w + 3]) * inv),
                                  pack_bf16x2(__uint_as_float(v[8 * w + 4]) * inv, __uint_as_float(v[8 * w + 5]) * inv),
                                  pack_bf16x2(__uint_as_float(v[8 * w + 6]) * inv, __uint_as_float(v[8 * w + 7]) * inv));
          }
        }
        // the next query tile's first P.V overwrites O: its P is written only after this read
        tc_fence_before();
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, 512);
}

size_t attn_smem_bytes() { return (size_t)AT_BAROFF + sizeof(AttnBars) + 1024; }

// ---- sparse prefill: each query row's top-k set -> bitmap rows and per-query-tile key-tile lists ----
// One CTA per (row s, sequence b): the row's selected positions t <= s as bits (a set: repeats
// merge), written out as 4 words per key tile, and the key tiles holding any selected position
// marked for the row's query tile.  `activity` must be zero on entry.
__global__ void __launch_bounds__(128) sparse_rows_kernel(const int32_t* __restrict__ topk, int k, int S, int n_qt,
                                                         uint32_t* __restrict__ bitmap, int32_t* __restrict__ activity,
                                                         int32_t* err) {
  extern __shared__ uint32_t bits[];  // 4 * n_qt words
  const int s = blockIdx.x, b = blockIdx.y;
  const int words = 4 * n_qt;
  for (int w = threadIdx.x; w < words; w += blockDim.x) bits[w] = 0u;
  __syncthreads();
  const int32_t* row = topk + ((int64_t)b * S + s) * k;
  for (int i = threadIdx.x; i < k; i += blockDim.x) {
    const int t = row[i];
    if (t < 0 || t >= S) {
      raise_error(err, MLA_ERR_INDEX);
      continue;
    }
    if (t > s) continue;  // the causal mask removes it
    atomicOr(&bits[t >> 5], 1u << (t & 31));
  }
  __syncthreads();
  uint32_t* dst = bitmap + ((int64_t)b * S + s) * words;
  for (int w = threadIdx.x; w < words; w += blockDim.x) dst[w] = bits[w];
  const int qt = s / AT_TILE;
  for (int kt = threadIdx.x; kt < n_qt; kt += blockDim.x)
    if (bits[4 * kt] | bits[4 * kt + 1] | bits[4 * kt + 2] | bits[4 * kt + 3])
      activity[((int64_t)b * n_qt + qt) * n_qt + kt] = 1;  // every writer stores the same 1
}

// One warp per (query tile, sequence): the active key tiles in increasing order, and their count.
__global__ void __launch_bounds__(32) sparse_lists_kernel(const int32_t* __restrict__ activity, int n_qt,
                                                         int32_t* __restrict__ tile_list,
                                                         int32_t* __restrict__ tile_count) {
  const int qt = blockIdx.x, b = blockIdx.y, lane = threadIdx.x;
  const int32_t* act = activity + ((int64_t)b * n_qt + qt) * n_qt;
  int32_t* list = tile_list + ((int64_t)b * n_qt + qt) * n_qt;
  int count = 0;
  for (int base = 0; base < n_qt; base += 32) {
    const int kt = base + lane;
    const bool on = kt < n_qt && act[kt] != 0;
    const unsigned m = __ballot_sync(0xffffffffu, on);
    if (on) list[count + __popc(m & ((1u << lane) - 1u))] = kt;
    count += __popc(m);
  }
  // a query tile none of whose rows selected a visible key still runs one key tile, its diagonal,
  // with every score masked: its rows end as empty rows (zeros, flagged), and every role of the
  // attention kernel sees at least one key tile per query tile
  if (count == 0) {
    if (lane == 0) list[0] = qt;
    count = 1;
  }
  if (lane == 0) tile_count[b * n_qt + qt] = count;
}
static_assert(AT_BAROFF + sizeof(AttnBars) + 1024 <= 232448, "dynamic shared memory above the 227 KB per-CTA limit");
}  // namespace prefill_tc

// kv[B*S, n_h*(d_h+d_v)] = c_kv[B*S, d_c] * w_kv_b^T, bf16, DeepSeek dimensions.
cudaError_t expand_tc_launch(const PrefillArgs& a, cudaStream_t st) {
  using namespace prefill_tc;
  Params p;
  memset(&p, 0, sizeof(p));
  const uint64_t M = (uint64_t)a.B * a.S, N = (uint64_t)a.n_h * (a.d_h + a.d_v), K = (uint64_t)a.d_c;
  {
    const uint64_t dims[2] = {K, M}, strides[1] = {(uint64_t)a.ckv_r * 2};
    const uint32_t box[2] = {BK, BM};
    if (!make_tensor_map_bf16(&p.tm_a, a.c_kv, 2, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B))
      return cudaErrorInvalidValue;
  }
  {
    const uint64_t dims[2] = {K, N}, strides[1] = {K * 2};
    const uint32_t box[2] = {BK, BN};
    if (!make_tensor_map_bf16(&p.tm_b, a.w, 2, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B))
      return cudaErrorInvalidValue;
  }
  {
    const uint64_t dims[2] = {N, M}, strides[1] = {N * 2};
    const uint32_t box[2] = {64, BM};
    if (!make_tensor_map_bf16(&p.tm_out, a.kv, 2, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B))
      return cudaErrorInvalidValue;
  }
  p.m_tiles = (int)((M + BM - 1) / BM);
  p.n_tiles = (int)(N / BN);
  p.k_slabs = (int)(K / BK);
  p.err = nullptr;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int total = p.m_tiles * p.n_tiles;
  const int grid = total < sms ? total : sms;
  const size_t smem = smem_bytes();
  cudaError_t e = cudaFuncSetAttribute(expand_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  return launch_pdl(expand_kernel, dim3(grid), dim3(kThreads), smem, st, p);
}

namespace prefill_tc {
static bool attn_params(const PrefillArgs& a, AttnParams& p) {
  memset(&p, 0, sizeof(p));
  const uint64_t H = (uint64_t)a.n_h, S = (uint64_t)a.S, B = (uint64_t)a.B;
  const uint64_t dq = (uint64_t)(a.d_h + a.d_r), dkv = (uint64_t)(a.d_h + a.d_v);
  {
    const uint64_t dims[4] = {dq, H, S, B}, strides[3] = {dq * 2, H * dq * 2, S * H * dq * 2};
    const uint32_t box[4] = {64, 1, AT_TILE, 1};
    if (!make_tensor_map_bf16(&p.tm_q, a.q, 4, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B)) return false;
  }
  {
    const uint64_t dims[4] = {dkv, H, S, B}, strides[3] = {dkv * 2, H * dkv * 2, S * H * dkv * 2};
    const uint32_t box[4] = {64, 1, AT_TILE, 1};
    if (!make_tensor_map_bf16(&p.tm_kv, a.kv, 4, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B)) return false;
  }
  {
    const uint64_t dims[3] = {(uint64_t)a.d_r, S, B}, strides[2] = {(uint64_t)a.kr_r * 2, S * (uint64_t)a.kr_r * 2};
    const uint32_t box[3] = {64, AT_TILE, 1};
    if (!make_tensor_map_bf16(&p.tm_kr, a.k_r, 3, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B)) return false;
  }
  p.out = static_cast<__nv_bfloat16*>(a.out);
  p.B = a.B;
  p.S = a.S;
  p.H = a.n_h;
  p.n_qt = (a.S + AT_TILE - 1) / AT_TILE;
  p.causal = a.causal;
  p.scale_log2 = a.scale * 1.4426950408889634f;
  p.err = nullptr;
  return true;
}

template <bool kSparse>
static cudaError_t attn_launch(const AttnParams& p, int B, int H, cudaStream_t st) {
  const size_t smem = attn_smem_bytes();
  cudaError_t e = cudaFuncSetAttribute(attn_kernel<kSparse>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  return launch_pdl(attn_kernel<kSparse>, dim3((unsigned)((p.n_qt + 1) / 2 * B * H)), dim3(AT_THREADS), smem, st,
                    p);
}
}  // namespace prefill_tc

// Causal (or full) attention of the naive path over the expanded rows in a.kv, bf16, DeepSeek dims.
cudaError_t attn_tc_launch(const PrefillArgs& a, cudaStream_t st) {
  using namespace prefill_tc;
  AttnParams p;
  if (!attn_params(a, p)) return cudaErrorInvalidValue;
  return attn_launch<false>(p, a.B, a.n_h, st);
}

size_t sparse_prefill_scratch_bytes(int B, int S) {
  const int n_qt = (S + prefill_tc::AT_TILE - 1) / prefill_tc::AT_TILE;
  auto up = [](size_t x) { return (x + 255) & ~(size_t)255; };
  return up((size_t)B * S * 4 * n_qt * 4) + 2 * up((size_t)B * n_qt * n_qt * 4) + up((size_t)B * n_qt * 4);
}

// The masks of the sparse prefill (bitmap rows, key-tile lists) into `scratch`; launched before the
// expansion, so they are complete before the attention starts.
cudaError_t sparse_masks_launch(const PrefillArgs& a, const int32_t* topk, int k, void* scratch, int32_t* err,
                                cudaStream_t st) {
  using namespace prefill_tc;
  const int n_qt = (a.S + AT_TILE - 1) / AT_TILE;
  auto up = [](size_t x) { return (x + 255) & ~(size_t)255; };
  uint8_t* base = static_cast<uint8_t*>(scratch);
  uint32_t* bitmap = reinterpret_cast<uint32_t*>(base);
  int32_t* activity = reinterpret_cast<int32_t*>(base + up((size_t)a.B * a.S * 4 * n_qt * 4));
  int32_t* list = activity + up((size_t)a.B * n_qt * n_qt * 4) / 4;
  int32_t* count = list + up((size_t)a.B * n_qt * n_qt * 4) / 4;
  cudaError_t e = cudaMemsetAsync(activity, 0, (size_t)a.B * n_qt * n_qt * 4, st);
  if (e != cudaSuccess) return e;
  sparse_rows_kernel<<<dim3(a.S, a.B), 128, (size_t)16 * n_qt, st>>>(topk, k, a.S, n_qt, bitmap, activity, err);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  sparse_lists_kernel<<<dim3(n_qt, a.B), 32, 0, st>>>(activity, n_qt, list, count);
  return cudaGetLastError();
}

// Attention of the sparse prefill: each query row attends its selected positions t <= s.
cudaError_t attn_sparse_tc_launch(const PrefillArgs& a, const void* scratch, int32_t* err, cudaStream_t st) {
  using namespace prefill_tc;
  AttnParams p;
  if (!attn_params(a, p)) return cudaErrorInvalidValue;
  const int n_qt = p.n_qt;
  auto up = [](size_t x) { return (x + 255) & ~(size_t)255; };
  const uint8_t* base = static_cast<const uint8_t*>(scratch);
  p.bitmap = reinterpret_cast<const uint32_t*>(base);
  p.row_words = 4 * n_qt;
  const int32_t* activity = reinterpret_cast<const int32_t*>(base + up((size_t)a.B * a.S * 4 * n_qt * 4));
  p.tile_list = activity + up((size_t)a.B * n_qt * n_qt * 4) / 4;
  p.tile_count = p.tile_list + up((size_t)a.B * n_qt * n_qt * 4) / 4;
  p.causal = 1;
  p.err = err;
  return attn_launch<true>(p, a.B, a.n_h, st);
}

}  // namespace mla

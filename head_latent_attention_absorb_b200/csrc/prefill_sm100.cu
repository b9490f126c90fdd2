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

}  // namespace mla

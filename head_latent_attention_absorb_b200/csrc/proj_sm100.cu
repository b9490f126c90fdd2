// The two per-head projections of the absorbed decode on tcgen05 tensor cores (bf16 in, fp32
// accumulation in TMEM), for the DeepSeek-V3 dimensions (128 heads, d_h = d_v = 128, d_c = 512):
//
//   absorb_q  q~[b,h,c] = sum_d q_nope[b,h,d] W^UK_h[d,c]   ("Absorb key weights", first einsum)
//   out_up    o[b,h,d]  = sum_c ctx[b,h,c]    W^UV_h[d,c]   ("Absorb key weights", last einsum)
//
// Both are a batch of 128 small GEMMs whose cost is reading W (8.4M bf16 weights, 16.8 MB, per
// projection); each is run "swap-AB" so that the 128 rows of one head's weight block are the MMA's
// M = 128 and the batch is N (padded to a multiple of 16, at most 256 per CTA):
//   absorb_q: D[c, b] = W^UK_h^T[c, d] q_nope_h^T[d, b]   A = W^UK_h read MN-major, K = 128
//   out_up:   D[d, b] = W^UV_h[d, c]   ctx_h^T[c, b]      A = W^UV_h read K-major,  K = 512
// One CTA computes the tiles of one (head, batch block) and kMB 128-row blocks (two for absorb_q,
// whose four latent blocks of a head share the activations): TMA brings the W blocks and the
// activations (K split in 64-wide chunks, one mbarrier each, so MMAs start on the first chunk),
// one thread issues the MMAs into one TMEM accumulator per block, and four warps per block read
// them back.  Fewer, larger CTAs start sooner (the launch of 512 small ones took ~2 us).
#include <cuda.h>
#include <cuda_bf16.h>
#include <string.h>

#include "common.cuh"
#include "kernels.h"
#include "sm100_ptx.cuh"
#include "tma_host.h"

namespace mla {
namespace proj_tc {

using namespace sm100;

constexpr int kNH = 128, kDC = 512, kDH = 128, kRowsPerHead = 256;
constexpr uint64_t kWaitLimitNs = 1000000000ull;

struct Params {
  CUtensorMap tm_w;    // 2-D (512 latent, 32768 rows), box (64, 64 or 128), 128-byte swizzle
  CUtensorMap tm_act;  // 3-D (K features, 128 heads, B), box (64, 1, n_tile), 128-byte swizzle
  __nv_bfloat16* out;  // absorb_q: [B][128][512]; out_up: [B][128][128]
  int B, n_tile;       // n_tile: batch rows per CTA (multiple of 16, <= 256)
  int32_t* err;
};

template <bool kAbsorb>
struct Shape {
  static constexpr int kChunks = kAbsorb ? kDH / 64 : kDC / 64;       // 64-wide K chunks
  static constexpr int kAChunkBytes = 128 * 64 * 2;                   // 128 M rows x 64 K
  static constexpr int kMB = kAbsorb ? 2 : 1;                         // 128-row blocks per CTA
  static constexpr int kThreads = 128 * kMB;                          // four epilogue warps per block
};

__device__ __forceinline__ uint32_t tmem_cols_for(int n) { return n <= 32 ? 32 : (n <= 64 ? 64 : (n <= 128 ? 128 : 256)); }

template <bool kAbsorb>
__global__ void __launch_bounds__(Shape<kAbsorb>::kThreads) proj_kernel(const __grid_constant__ Params p) {
  using S = Shape<kAbsorb>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* a_s = smem;                                          // [kMB][kChunks] x 16 KB
  uint8_t* b_s = smem + S::kMB * S::kChunks * S::kAChunkBytes;  // kChunks x (n_tile x 128 B)
  __shared__ uint64_t full[S::kChunks];
  __shared__ uint64_t done;
  __shared__ uint32_t tmem_base;
  __shared__ int abort_flag;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int h = blockIdx.y;
  const int m0 = kAbsorb ? blockIdx.x * 128 * S::kMB : 0;  // first latent feature (absorb_q) of this CTA
  const int b0 = blockIdx.z * p.n_tile;
  const int n = p.n_tile;
  const uint32_t ncols = tmem_cols_for(n);
  const uint32_t b_chunk_bytes = (uint32_t)n * 128;

  griddep_launch_dependents();  // the next kernel may run its independent prologue
  if (threadIdx.x == 0) {
    for (int j = 0; j < S::kChunks; ++j) mbar_init(smem_u32(&full[j]), 1);
    mbar_init(smem_u32(&done), 1);
    abort_flag = 0;
    fence_mbar_init();
    prefetch_tensormap(&p.tm_w);
    prefetch_tensormap(&p.tm_act);
  }
  if (warp == 0) {
    tmem_alloc(smem_u32(&tmem_base), ncols * S::kMB);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base;

  if (threadIdx.x == 0) {
    // ---- loads: K chunk j = features [64 j, 64 j + 64) of the contraction
    const uint64_t pol_w = policy_evict_first(), pol_a = policy_evict_last();
    // the weights are no kernel's output: load them before waiting for the preceding kernel
    for (int j = 0; j < S::kChunks; ++j) {
      const uint32_t bar = smem_u32(&full[j]);
      mbar_arrive_expect_tx(bar, S::kMB * S::kAChunkBytes + b_chunk_bytes);
      const uint32_t a_dst = smem_u32(a_s + j * S::kAChunkBytes);
      if (kAbsorb) {
        // W^UK_h rows d in [64 j, 64 j + 64), latent columns [m0 + 128 mb, + 128) as two 64-column
        // boxes per block: MN-major A (M = latent feature contiguous), one 8 KB box per 64 M values
#pragma unroll
        for (int mb = 0; mb < S::kMB; ++mb) {
          const uint32_t d = a_dst + mb * S::kChunks * S::kAChunkBytes;
          tma_load_2d(d, &p.tm_w, bar, m0 + 128 * mb, h * kRowsPerHead + 64 * j, pol_w);
          tma_load_2d(d + 8192, &p.tm_w, bar, m0 + 128 * mb + 64, h * kRowsPerHead + 64 * j, pol_w);
        }
      } else {
        // W^UV_h rows d in [0, 128), latent columns [64 j, 64 j + 64): K-major A
        tma_load_2d(a_dst, &p.tm_w, bar, 64 * j, h * kRowsPerHead + kDH, pol_w);
      }
    }
    // the activations (and the output this kernel overwrites) belong to the preceding kernels
    griddep_wait();
    for (int j = 0; j < S::kChunks; ++j)
      tma_load_3d(smem_u32(b_s + j * b_chunk_bytes), &p.tm_act, smem_u32(&full[j]), 64 * j, h, b0, pol_a);
    // ---- MMAs: D[128 x n] (+)= A_j B_j^T over the chunks as they land
    const uint32_t idesc = idesc_bf16_f32(128, (uint32_t)n, kAbsorb ? 1u : 0u, 0u);
    bool ok = true;
    for (int j = 0; j < S::kChunks && ok; ++j) {
      if (!mbar_wait(smem_u32(&full[j]), 0, &abort_flag, kWaitLimitNs)) {
        raise_error(p.err, MLA_ERR_TIMEOUT);
        ok = false;
        break;
      }
      tc_fence_after();
      const uint32_t b_base = smem_u32(b_s + j * b_chunk_bytes);
#pragma unroll
      for (int mb = 0; mb < S::kMB; ++mb) {
        const uint32_t a_base = smem_u32(a_s + (mb * S::kChunks + j) * S::kAChunkBytes);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
          const uint64_t ad = kAbsorb ? smem_desc(a_base + kk * 2048, 8192, 1024, kSwizzle128)   // 16 K rows
                                      : smem_desc(a_base + kk * 32, 16, 1024, kSwizzle128);      // 16 K columns
          const uint64_t bd = smem_desc(b_base + kk * 32, 16, 1024, kSwizzle128);
          mma_ss(tmem + mb * ncols, ad, bd, idesc, (j | kk) ? 1u : 0u);
        }
      }
    }
    mma_commit(smem_u32(&done));
    if (!ok) abort_flag = 1;
  }
  __syncwarp();

  // ---- epilogue: lane i of warp w holds row 32 (w % 4) + i of block w / 4 of D (a latent /
  // value feature)
  griddep_wait();  // every thread that writes the output waits for the preceding kernel
  const bool ok = mbar_wait(smem_u32(&done), 0, &abort_flag, kWaitLimitNs);
  if (__all_sync(0xffffffffu, ok)) {
    tc_fence_after();
    const int mb = warp >> 2, quad = warp & 3;
    const int row = 32 * quad + lane;
    const uint32_t taddr = tmem + ((uint32_t)(32 * quad) << 16) + mb * ncols;
    const int out_w = kAbsorb ? kDC : kDH;
    __nv_bfloat16* out = p.out + (int64_t)h * out_w + m0 + 128 * mb + row;
    for (int c0 = 0; c0 < n; c0 += 16) {
      uint32_t r[16];
      tmem_ld16(taddr + c0, r);
      tmem_ld_wait();
#pragma unroll
      for (int k = 0; k < 16; ++k) {
        const int b = b0 + c0 + k;
        if (b < p.B) out[(int64_t)b * kNH * out_w] = __float2bfloat16_rn(__uint_as_float(r[k]));
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_dealloc(tmem, ncols * S::kMB);
}

size_t smem_bytes(bool absorb, int n_tile) {
  const int chunks = absorb ? kDH / 64 : kDC / 64, mbs = absorb ? Shape<true>::kMB : 1;
  return (size_t)chunks * (mbs * 128 * 64 * 2 + n_tile * 128) + 1024;
}
static_assert((kDC / 64) * (128 * 64 * 2 + 96 * 128) + 1024 <= 232448, "out_up tile above 227 KB of shared memory");
static_assert((kDH / 64) * (2 * 128 * 64 * 2 + 256 * 128) + 1024 <= 232448, "absorb_q tile above 227 KB");

// Batch rows per CTA: the whole batch up to the most that fits (one CTA per head and row block),
// else that many per CTA.  absorb_q holds 2 x 2 weight chunks, so 256 rows fit; out_up holds all 8
// chunks of its K = 512, and 8 x (16 KB + 128 B per row) stays within 227 KB only up to 96 rows.
int n_tile_for(bool absorb, int B) {
  const int cap = absorb ? 256 : 96;
  const int n = ((B + 15) / 16) * 16;
  return n > cap ? cap : n;
}

template <bool kAbsorb>
cudaError_t launch(int B, const void* act, int64_t ld_head, const void* w, void* out, int32_t* err, cudaStream_t st) {
  Params p;
  memset(&p, 0, sizeof(p));
  const int n_tile = n_tile_for(kAbsorb, B);
  const int kfeat = kAbsorb ? kDH : kDC;
  {
    const uint64_t dims[2] = {(uint64_t)kDC, (uint64_t)kNH * kRowsPerHead};
    const uint64_t strides[1] = {(uint64_t)kDC * 2};
    const uint32_t box[2] = {64, kAbsorb ? 64u : 128u};
    if (!make_tensor_map_bf16(&p.tm_w, w, 2, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B))
      return cudaErrorInvalidValue;
  }
  {
    const uint64_t dims[3] = {(uint64_t)kfeat, (uint64_t)kNH, (uint64_t)B};
    const uint64_t strides[2] = {(uint64_t)ld_head * 2, (uint64_t)ld_head * kNH * 2};
    const uint32_t box[3] = {64, 1, (uint32_t)n_tile};
    if (!make_tensor_map_bf16(&p.tm_act, act, 3, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B))
      return cudaErrorInvalidValue;
  }
  p.out = static_cast<__nv_bfloat16*>(out);
  p.B = B;
  p.n_tile = n_tile;
  p.err = err;
  const size_t smem = smem_bytes(kAbsorb, n_tile);
  cudaError_t e = cudaFuncSetAttribute(proj_kernel<kAbsorb>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const dim3 grid(kAbsorb ? kDC / 128 / Shape<kAbsorb>::kMB : 1, kNH, (B + n_tile - 1) / n_tile);
  return launch_pdl(proj_kernel<kAbsorb>, grid, dim3(Shape<kAbsorb>::kThreads), smem, st, p);
}

}  // namespace proj_tc

cudaError_t absorb_q_tc_launch(int B, const void* q_nope, int64_t ldq, const void* w, void* q_tilde, cudaStream_t st) {
  return proj_tc::launch<true>(B, q_nope, ldq, w, q_tilde, nullptr, st);
}

cudaError_t out_up_tc_launch(int B, const void* ctx, const void* w, void* out, cudaStream_t st) {
  return proj_tc::launch<false>(B, ctx, 512, w, out, nullptr, st);
}

}  // namespace mla

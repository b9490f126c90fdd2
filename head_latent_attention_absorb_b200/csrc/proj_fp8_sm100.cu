// The two per-head projections with an FP8 (e4m3) wkv_b and one fp32 scale per 128 x 128 block
// ("Key-value down-projection", linear excerpt: FP8 weights carry one float32 scale per 128 x 128
// block; "Value up-projection": the decode uses the dequantised matrix).  The weight is read from
// HBM as FP8 (half the bytes of the bf16 path) and dequantised on chip: each 8 KB e4m3 box lands in
// the upper half of the 16 KB bf16 operand buffer it becomes; every thread loads its share into
// registers, the CTA meets, and every thread writes its values times the block's scale, rounded to
// bf16, in the 128-byte-swizzled layout a bf16 TMA box would have.  The MMAs, activations and
// epilogue are those of the bf16 projections (swap-AB: the head's 128 weight rows are M, the batch
// is N).
//   absorb_q  q~[b,h,c] = sum_d q_nope[b,h,d] W^UK_h[d,c]    A = W^UK_h read MN-major, K = 128
//   out_up    o[b,h,d]  = sum_c ctx[b,h,c]    W^UV_h[d,c]    A = W^UV_h read K-major,  K = 512
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp8.h>
#include <string.h>

#include "common.cuh"
#include "kernels.h"
#include "sm100_ptx.cuh"
#include "tma_host.h"

namespace mla {
namespace proj_fp8 {

using namespace sm100;

constexpr int kNH = 128, kDC = 512, kDH = 128, kRowsPerHead = 256;
constexpr uint64_t kWaitLimitNs = 1000000000ull;

struct Params {
  CUtensorMap tm_w;     // 2-D uint8 (512 latent, 32768 rows), no swizzle; box (128, 64) absorb / (64, 128) out_up
  CUtensorMap tm_act;   // 3-D bf16 (K features, 128 heads, B), box (64, 1, n_tile), 128-byte swizzle
  const float* scale;   // [256 row blocks][4 column blocks]
  __nv_bfloat16* out;
  int B, n_tile;
  int32_t* err;
};

template <bool kAbsorb>
struct Shape {
  static constexpr int kChunks = kAbsorb ? kDH / 64 : kDC / 64;
  static constexpr int kAChunkBytes = 128 * 64 * 2;  // one bf16 operand buffer (16 KB)
  static constexpr int kMB = kAbsorb ? 2 : 1;
  static constexpr int kThreads = 128 * kMB;
  // per 64-wide K chunk: kMB x 1024 bf16 16-byte chunks to write, 8 per thread
  static_assert(kMB * 1024 == 8 * kThreads, "eight dequantised chunks per thread");
};

__device__ __forceinline__ uint32_t tmem_cols_for(int n) { return n <= 32 ? 32 : (n <= 64 ? 64 : (n <= 128 ? 128 : 256)); }

// 8 e4m3 values (little-endian in two words) times `s`, rounded to 8 bf16 (one 16-byte chunk)
__device__ __forceinline__ uint4 dequant8(uint2 v, float s) {
  uint32_t out[4];
  const uint32_t w[2] = {v.x, v.y};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const __nv_fp8x2_storage_t pair = (__nv_fp8x2_storage_t)((w[i >> 1] >> (16 * (i & 1))) & 0xffffu);
    const __half2 h = __half2(__nv_cvt_fp8x2_to_halfraw2(pair, __NV_E4M3));
    const float2 f = __half22float2(h);
    const __nv_bfloat162 b = __floats2bfloat162_rn(f.x * s, f.y * s);
    out[i] = *reinterpret_cast<const uint32_t*>(&b);
  }
  return make_uint4(out[0], out[1], out[2], out[3]);
}

template <bool kAbsorb>
__global__ void __launch_bounds__(Shape<kAbsorb>::kThreads) proj_fp8_kernel(const __grid_constant__ Params p) {
  using S = Shape<kAbsorb>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* a_s = smem;                                          // [kMB][kChunks] x 16 KB (bf16 operands)
  uint8_t* b_s = smem + S::kMB * S::kChunks * S::kAChunkBytes;  // kChunks x (n_tile x 128 B)
  __shared__ uint64_t wfull[S::kChunks], afull[S::kChunks];
  __shared__ uint64_t done;
  __shared__ uint32_t tmem_base;
  __shared__ int abort_flag;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int h = blockIdx.y;
  const int m0 = kAbsorb ? blockIdx.x * 128 * S::kMB : 0;
  const int b0 = blockIdx.z * p.n_tile;
  const int n = p.n_tile;
  const uint32_t ncols = tmem_cols_for(n);
  const uint32_t b_chunk_bytes = (uint32_t)n * 128;

  griddep_launch_dependents();
  if (threadIdx.x == 0) {
    for (int j = 0; j < S::kChunks; ++j) {
      mbar_init(smem_u32(&wfull[j]), 1);
      mbar_init(smem_u32(&afull[j]), 1);
    }
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
    // FP8 boxes into the upper half of each bf16 operand buffer; the weights are no kernel's output
    const uint64_t pol_w = policy_evict_first(), pol_a = policy_evict_last();
    for (int j = 0; j < S::kChunks; ++j) {
      const uint32_t bar = smem_u32(&wfull[j]);
      mbar_arrive_expect_tx(bar, S::kMB * 8192);
#pragma unroll
      for (int mb = 0; mb < S::kMB; ++mb) {
        const uint32_t dst = smem_u32(a_s + (mb * S::kChunks + j) * S::kAChunkBytes + 8192);
        if (kAbsorb)  // W^UK_h rows d in [64 j, +64), latent columns [m0 + 128 mb, +128): 64 rows x 128 B
          tma_load_2d(dst, &p.tm_w, bar, m0 + 128 * mb, h * kRowsPerHead + 64 * j, pol_w);
        else          // W^UV_h rows d in [0, 128), latent columns [64 j, +64): 128 rows x 64 B
          tma_load_2d(dst, &p.tm_w, bar, 64 * j, h * kRowsPerHead + kDH, pol_w);
      }
    }
    griddep_wait();  // the activations belong to the preceding kernels
    for (int j = 0; j < S::kChunks; ++j) {
      mbar_arrive_expect_tx(smem_u32(&afull[j]), b_chunk_bytes);
      tma_load_3d(smem_u32(b_s + j * b_chunk_bytes), &p.tm_act, smem_u32(&afull[j]), 64 * j, h, b0, pol_a);
    }
  }

  const uint32_t idesc = idesc_bf16_f32(128, (uint32_t)n, kAbsorb ? 1u : 0u, 0u);
  bool ok = true;
  for (int j = 0; j < S::kChunks; ++j) {
    // every thread: this chunk's FP8 boxes have landed (one decision for the whole CTA)
    const bool landed = mbar_wait(smem_u32(&wfull[j]), 0, &abort_flag, kWaitLimitNs);
    if (!__syncthreads_and(landed)) {
      if (threadIdx.x == 0) raise_error(p.err, MLA_ERR_TIMEOUT);
      ok = false;
      break;
    }
    // item i of this thread: 16-byte bf16 chunk q of row r of block mb (absorb: of one of two
    // 64-column boxes); its 8 e4m3 sources sit in the same buffer's upper half
    uint2 src[8];
    uint32_t dst[8];
    float sc[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int item = threadIdx.x + i * S::kThreads;   // < kMB * 1024
      const int mb = item >> 10, rem = item & 1023;
      const uint32_t buf = smem_u32(a_s + (mb * S::kChunks + j) * S::kAChunkBytes);
      if (kAbsorb) {
        // 2 boxes x 64 rows x 8 chunks: box k holds latent columns 64 k .. 64 k + 63 of the block
        const int k = rem >> 9, r = (rem >> 3) & 63, q = rem & 7;
        src[i] = *reinterpret_cast<const uint2*>(a_s + (mb * S::kChunks + j) * S::kAChunkBytes + 8192 + r * 128 +
                                                 64 * k + 8 * q);
        dst[i] = buf + k * 8192 + r * 128 + ((q ^ (r & 7)) << 4);
        sc[i] = p.scale[(2 * h) * 4 + (m0 + 128 * mb) / 128];
      } else {
        // 128 rows x 8 chunks: row r = value feature d, chunk q = latent columns 64 j + 8 q ..
        const int r = rem >> 3, q = rem & 7;
        src[i] = *reinterpret_cast<const uint2*>(a_s + (mb * S::kChunks + j) * S::kAChunkBytes + 8192 + r * 64 + 8 * q);
        dst[i] = buf + r * 128 + ((q ^ (r & 7)) << 4);
        sc[i] = p.scale[(2 * h + 1) * 4 + j / 2];
      }
    }
    __syncthreads();  // every FP8 source of this chunk is in registers before any bf16 write over it
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const uint4 v = dequant8(src[i], sc[i]);
      st_shared_v4_b32(dst[i], v.x, v.y, v.z, v.w);
    }
    fence_proxy_async_smem();  // generic-proxy writes, read next by the tensor core
    __syncthreads();
    if (threadIdx.x == 0) {
      if (!mbar_wait(smem_u32(&afull[j]), 0, &abort_flag, kWaitLimitNs)) {
        raise_error(p.err, MLA_ERR_TIMEOUT);
        abort_flag = 1;
      } else {
        tc_fence_after();
        const uint32_t b_base = smem_u32(b_s + j * b_chunk_bytes);
#pragma unroll
        for (int mb = 0; mb < S::kMB; ++mb) {
          const uint32_t a_base = smem_u32(a_s + (mb * S::kChunks + j) * S::kAChunkBytes);
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            const uint64_t ad = kAbsorb ? smem_desc(a_base + kk * 2048, 8192, 1024, kSwizzle128)
                                        : smem_desc(a_base + kk * 32, 16, 1024, kSwizzle128);
            const uint64_t bd = smem_desc(b_base + kk * 32, 16, 1024, kSwizzle128);
            mma_ss(tmem + mb * ncols, ad, bd, idesc, (j | kk) ? 1u : 0u);
          }
        }
      }
    }
  }
  if (threadIdx.x == 0) mma_commit(smem_u32(&done));
  __syncwarp();

  griddep_wait();  // every thread that writes the output waits for the preceding kernel
  const bool fin = ok && mbar_wait(smem_u32(&done), 0, &abort_flag, kWaitLimitNs) && !abort_flag;
  if (__all_sync(0xffffffffu, fin)) {
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

int n_tile_for(bool absorb, int B) {
  const int cap = absorb ? 256 : 96;
  const int n = ((B + 15) / 16) * 16;
  return n > cap ? cap : n;
}

inline bool make_tensor_map_u8(CUtensorMap* m, const void* base, const uint64_t* dims, const uint64_t* strides,
                               const uint32_t* box) {
  EncodeTiledFn enc = encode_tiled_fn();
  if (!enc) return false;
  cuuint64_t d[2] = {dims[0], dims[1]}, s[1] = {strides[0]};
  cuuint32_t b[2] = {box[0], box[1]}, e[2] = {1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), d, s, b, e, CU_TENSOR_MAP_INTERLEAVE_NONE,
             CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <bool kAbsorb>
cudaError_t launch(int B, const void* act, int64_t ld_head, const void* w, const float* scale, void* out,
                   int32_t* err, cudaStream_t st) {
  Params p;
  memset(&p, 0, sizeof(p));
  const int n_tile = n_tile_for(kAbsorb, B);
  const int kfeat = kAbsorb ? kDH : kDC;
  {
    const uint64_t dims[2] = {(uint64_t)kDC, (uint64_t)kNH * kRowsPerHead};
    const uint64_t strides[1] = {(uint64_t)kDC};
    const uint32_t box[2] = {kAbsorb ? 128u : 64u, kAbsorb ? 64u : 128u};
    if (!make_tensor_map_u8(&p.tm_w, w, dims, strides, box)) return cudaErrorInvalidValue;
  }
  {
    const uint64_t dims[3] = {(uint64_t)kfeat, (uint64_t)kNH, (uint64_t)B};
    const uint64_t strides[2] = {(uint64_t)ld_head * 2, (uint64_t)ld_head * kNH * 2};
    const uint32_t box[3] = {64, 1, (uint32_t)n_tile};
    if (!make_tensor_map_bf16(&p.tm_act, act, 3, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B))
      return cudaErrorInvalidValue;
  }
  p.scale = scale;
  p.out = static_cast<__nv_bfloat16*>(out);
  p.B = B;
  p.n_tile = n_tile;
  p.err = err;
  const size_t smem = smem_bytes(kAbsorb, n_tile);
  cudaError_t e = cudaFuncSetAttribute(proj_fp8_kernel<kAbsorb>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)smem);
  if (e != cudaSuccess) return e;
  const dim3 grid(kAbsorb ? kDC / 128 / Shape<kAbsorb>::kMB : 1, kNH, (B + n_tile - 1) / n_tile);
  return launch_pdl(proj_fp8_kernel<kAbsorb>, grid, dim3(Shape<kAbsorb>::kThreads), smem, st, p);
}

}  // namespace proj_fp8

cudaError_t absorb_q_fp8_tc_launch(int B, const void* q_nope, int64_t ldq, const void* w_fp8, const float* scale,
                                   void* q_tilde, int32_t* err, cudaStream_t st) {
  return proj_fp8::launch<true>(B, q_nope, ldq, w_fp8, scale, q_tilde, err, st);
}

cudaError_t out_up_fp8_tc_launch(int B, const void* ctx, const void* w_fp8, const float* scale, void* out,
                                 int32_t* err, cudaStream_t st) {
  return proj_fp8::launch<false>(B, ctx, 512, w_fp8, scale, out, err, st);
}

}  // namespace mla

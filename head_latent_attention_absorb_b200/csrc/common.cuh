// Shared helpers of the MLA CUDA library: element conversion, warp reductions, the device error
// flag and the argument blocks handed from the C-ABI layer to the kernel launchers.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>
#include <stdlib.h>

#include "mla_api.h"

namespace mla {

__device__ __forceinline__ float to_f32(float x) { return x; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 x) { return __bfloat162float(x); }

template <typename T> __device__ __forceinline__ T from_f32(float x);
template <> __device__ __forceinline__ float from_f32<float>(float x) { return x; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float x) {
  return __float2bfloat16_rn(x);
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

// First error wins: a later error never overwrites an earlier one.
__device__ __forceinline__ void raise_error(int32_t* flag, int32_t code) {
  if (flag != nullptr) atomicCAS(flag, 0, code);
}

// Whether a persistent decode launch may use the sliced merge, in which every cluster holding a
// piece of a sequence waits for all the others' partials.  That wait needs every cluster of the
// launch resident at once.  The launcher passes `one_wave` = the occupancy query confirmed that the
// whole grid fits on the GPU in one wave; MLA_DECODE_SLICED_MERGE=0 in the environment turns the
// sliced merge off as well, for GPUs whose SMs another context may hold for the length of a launch
// (MPS clients, another process's long-running kernel).  Without it the last cluster to arrive
// merges every partial, which waits only on clusters that have already run.
inline bool sliced_merge_allowed(bool one_wave) {
  const char* e = getenv("MLA_DECODE_SLICED_MERGE");
  return one_wave && !(e != nullptr && e[0] == '0' && e[1] == '\0');
}

// Validated arguments of one decode call (pointers already checked on the host).
struct DecodeArgs {
  int n_h, d_c, d_r, B, n_max, topk;
  int T = 1;  // new tokens per cache sequence: B query groups over B / T cache sequences
  const void* q_tilde; int64_t ldqt;
  const void* q_pe;    int64_t ldqp;
  const void* c_kv;    int64_t ckv_b, ckv_r;
  const void* k_r;     int64_t kr_b, kr_r;
  const int32_t* lengths;
  const int32_t* topk_idx;
  float scale;
  void* ctx;
  float* lse;
  int32_t* err;
  // FP8 latent cache (mla_decode_absorb_fp8kv): e4m3 rows replace c_kv; strides in bytes for c8 and
  // in floats for kv_scale (one fp32 scale per 128 latent features of a row)
  const void* c8 = nullptr;        int64_t c8_b = 0, c8_r = 0;
  const float* kv_scale = nullptr; int64_t sc_b = 0, sc_r = 0;
};

struct PrefillArgs {
  int n_h, d_c, d_r, d_h, d_v, B, S, causal;
  const void* q;
  const void* c_kv; int64_t ckv_r;
  const void* k_r;  int64_t kr_r;
  const void* w;
  float scale;
  void* out;
  void* kv;  // expanded [B, S, n_h, d_h + d_v] in the input dtype
};

// Validated arguments of one cache append (one new token per sequence).
struct AppendArgs {
  int d_c, d_r, B, n_max;
  const void* kv_a; int64_t lda;  // [B, d_c + d_r] rows: latent first, rotary key last
  const float* gain;              // [d_c] RMSNorm gain, or nullptr for ones
  float eps, rope_base;
  const int32_t* positions;       // [B] cache row (= position) of each new token
  void* c_kv; int64_t ckv_b, ckv_r;
  void* k_r;  int64_t kr_b, kr_r;
  int32_t* err;
};

// Launch with programmatic stream serialization: the kernel may start while the preceding kernel
// in the stream is still running, and synchronises with it through griddepcontrol.wait before it
// touches that kernel's data (every kernel of this library does).
template <typename... Args>
inline cudaError_t launch_pdl(void (*kernel)(Args...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                              Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, args...);
}

}  // namespace mla

// Cache append: the new token's joint down-projection row -> one latent row and one rotary row
// of the caches ("Key-value down-projection", mla-kv excerpt: split into the kv_lora_rank latent
// and the qk_rope_head_dim rotary key, RMSNorm on the latent, rotary embedding on the key;
// "Key-value latent RMSNorm": one gain per feature, computed in float32).
//
// One CTA per sequence.  The row is a few KB, so the kernel is bound by launch latency, not by
// bandwidth: it reads the row once from global memory, reduces the latent's sum of squares in
// fp32 across the block, and writes both cache rows.  The rotary angle pos * base^(-2i/d_r) is
// formed and reduced in fp64: at positions of 64K an fp32 product would be off by ~4e-3 rad.
#include <math.h>

#include "common.cuh"
#include "kernels.h"
#include "sm100_ptx.cuh"

namespace mla {
namespace {

constexpr int kAppendThreads = 128;

template <typename T>
__global__ void __launch_bounds__(kAppendThreads) cache_append_kernel(AppendArgs a) {
  __shared__ float part[kAppendThreads / 32];
  const int b = blockIdx.x;
  const int pos = a.positions[b];
  if (pos < 0 || pos >= a.n_max) {  // the row would land outside the cache: report, write nothing
    if (threadIdx.x == 0) raise_error(a.err, MLA_ERR_INDEX);
    return;
  }
  const T* row = static_cast<const T*>(a.kv_a) + (int64_t)b * a.lda;

  // RMSNorm of the latent: x / sqrt(mean(x^2) + eps), then the per-feature gain
  float ss = 0.f;
  for (int i = threadIdx.x; i < a.d_c; i += kAppendThreads) {
    const float x = to_f32(row[i]);
    ss = fmaf(x, x, ss);
  }
  ss = warp_sum(ss);
  if ((threadIdx.x & 31) == 0) part[threadIdx.x >> 5] = ss;
  __syncthreads();
  float tot = 0.f;
#pragma unroll
  for (int w = 0; w < kAppendThreads / 32; ++w) tot += part[w];
  const float inv_rms = rsqrtf(tot / (float)a.d_c + a.eps);
  T* c_dst = static_cast<T*>(a.c_kv) + (int64_t)b * a.ckv_b + (int64_t)pos * a.ckv_r;
  for (int i = threadIdx.x; i < a.d_c; i += kAppendThreads) {
    const float g = a.gain != nullptr ? a.gain[i] : 1.f;
    c_dst[i] = from_f32<T>(g * (to_f32(row[i]) * inv_rms));
  }

  // rotary key: pair (x[2i], x[2i+1]) rotated by pos * base^(-2i/d_r), i.e. multiplied as the
  // complex number x[2i] + j x[2i+1] by exp(j angle)
  T* k_dst = static_cast<T*>(a.k_r) + (int64_t)b * a.kr_b + (int64_t)pos * a.kr_r;
  const T* k_src = row + a.d_c;
  const double log_base = log((double)a.rope_base);
  for (int i = threadIdx.x; i < a.d_r / 2; i += kAppendThreads) {
    const double angle = (double)pos * exp(-(2.0 * i / a.d_r) * log_base);
    double s, c;
    sincos(angle, &s, &c);
    const float cf = (float)c, sf = (float)s;
    const float x0 = to_f32(k_src[2 * i]), x1 = to_f32(k_src[2 * i + 1]);
    k_dst[2 * i] = from_f32<T>(x0 * cf - x1 * sf);
    k_dst[2 * i + 1] = from_f32<T>(x0 * sf + x1 * cf);
  }
}

}  // namespace

template <typename T>
cudaError_t cache_append_launch(const AppendArgs& a, cudaStream_t st) {
  cache_append_kernel<T><<<a.B, kAppendThreads, 0, st>>>(a);
  return cudaGetLastError();
}

template cudaError_t cache_append_launch<float>(const AppendArgs&, cudaStream_t);
template cudaError_t cache_append_launch<__nv_bfloat16>(const AppendArgs&, cudaStream_t);

}  // namespace mla

// ------------------------------------------------------------------------------------------
// Top-k index validation (opt-in, outside the decode): the decode's gather reads each listed row
// once, so a repeated index would count twice where the pages' scatter mask counts it once
// ("Absorb key weights", decode excerpt: 0 scattered into a -inf row is a set).  One CTA per
// sequence marks its indices in a shared-memory bitmap of the cache length; an index outside
// [0, length) or one already marked raises MLA_ERR_INDEX.  Every bitmap access is behind the range
// check, so no index can reach outside the bitmap.
// ------------------------------------------------------------------------------------------
namespace mla {
namespace {

constexpr int kCheckThreads = 256;

__global__ void __launch_bounds__(kCheckThreads) check_topk_kernel(const int32_t* __restrict__ idx, int topk,
                                                                   const int32_t* __restrict__ lengths, int n_max,
                                                                   int32_t* err) {
  extern __shared__ uint32_t seen[];  // ceil(n_max / 32) words
  const int b = blockIdx.x;
  const int words = (n_max + 31) >> 5;
  for (int w = threadIdx.x; w < words; w += kCheckThreads) seen[w] = 0u;
  __syncthreads();
  const int len = lengths != nullptr ? lengths[b] : n_max;
  if (len < 1 || len > n_max) {
    if (threadIdx.x == 0) raise_error(err, MLA_ERR_LENGTH);
    return;
  }
  const int32_t* row = idx + (int64_t)b * topk;
  for (int i = threadIdx.x; i < topk; i += kCheckThreads) {
    const int t = row[i];
    if (t < 0 || t >= len) {
      raise_error(err, MLA_ERR_INDEX);
      continue;
    }
    const uint32_t bit = 1u << (t & 31);
    if (atomicOr(&seen[t >> 5], bit) & bit) raise_error(err, MLA_ERR_INDEX);  // listed twice
  }
}

}  // namespace

// The bounded wait every kernel uses, made to run out: an mbarrier expecting one arrival that never
// comes.  The wait gives up after limit_ns of global time and the flag records MLA_ERR_TIMEOUT.
__global__ void __launch_bounds__(32) wait_timeout_kernel(uint64_t limit_ns, int32_t* err) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    sm100::mbar_init(sm100::smem_u32(&bar), 1);
    abort_flag = 0;
    sm100::fence_mbar_init();
  }
  __syncwarp();
  const bool done = sm100::mbar_wait(sm100::smem_u32(&bar), 0, &abort_flag, limit_ns);
  if (threadIdx.x == 0 && !done) raise_error(err, MLA_ERR_TIMEOUT);
}

cudaError_t wait_timeout_launch(uint64_t limit_ns, int32_t* err, cudaStream_t st) {
  wait_timeout_kernel<<<1, 32, 0, st>>>(limit_ns, err);
  return cudaGetLastError();
}

size_t check_topk_smem_bytes(int n_max) { return (size_t)((n_max + 31) / 32) * sizeof(uint32_t); }

cudaError_t check_topk_launch(int B, const int32_t* idx, int topk, const int32_t* lengths, int n_max, int32_t* err,
                              cudaStream_t st) {
  const size_t smem = check_topk_smem_bytes(n_max);
  if (smem > 48 * 1024) {
    const cudaError_t e = cudaFuncSetAttribute(check_topk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                               (int)smem);
    if (e != cudaSuccess) return e;
  }
  check_topk_kernel<<<B, kCheckThreads, smem, st>>>(idx, topk, lengths, n_max, err);
  return cudaGetLastError();
}

}  // namespace mla

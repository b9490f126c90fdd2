// CUDA-core (SIMT) kernels of the four MLA operations, generic in the head dimensions.
// They carry the fp32 element type (no tensor cores, so no TF32 rounding) for any dimensions
// the C-ABI accepts.  The bf16 tensor-core kernels live in the *_sm100.cu files.
//
// Operations ("Absorb key weights", decode excerpt; "Value up-projection", prefill excerpt):
//   absorb_q   q~[b,h,c] = sum_d q_nope[b,h,d] W^UK_h[d,c]
//   decode     split-KV online softmax over scale (q~ . c_t + q_pe . k^R_t), ctx = sum alpha c_t
//   combine    merge of split partials (m, l, O): ctx = sum e^{m_s-M} O_s / sum e^{m_s-M} l_s
//   out_up     o[b,h,d] = sum_c ctx[b,h,c] W^UV_h[d,c]
//   prefill    wkv_b expansion GEMM, then causal attention with k = [k_nope; k^R]
#include <math.h>

#include "common.cuh"
#include "kernels.h"

namespace mla {

namespace {

constexpr int kBatchChunk = 16;

// ----------------------------------------------------------------------------------------
// absorb_q: one thread per latent column c of one head; W^UK_h streamed once per batch chunk
// ----------------------------------------------------------------------------------------
template <typename T>
__global__ void absorb_q_simt(int n_h, int d_c, int d_h, int d_v, int B, const T* __restrict__ q,
                              int64_t ldq, const T* __restrict__ w, T* __restrict__ qt) {
  extern __shared__ float qs[];  // [kBatchChunk][d_h]
  const int h = blockIdx.x;
  const int c = blockIdx.y * blockDim.x + threadIdx.x;
  const int b0 = blockIdx.z * kBatchChunk;
  const int nb = min(kBatchChunk, B - b0);
  for (int i = threadIdx.x; i < nb * d_h; i += blockDim.x) {
    const int j = i / d_h, d = i % d_h;
    qs[i] = to_f32(q[((int64_t)(b0 + j) * n_h + h) * ldq + d]);
  }
  __syncthreads();
  if (c >= d_c) return;
  float acc[kBatchChunk];
#pragma unroll
  for (int j = 0; j < kBatchChunk; ++j) acc[j] = 0.f;
  const T* wk = w + (int64_t)h * (d_h + d_v) * d_c + c;
  for (int d = 0; d < d_h; ++d) {
    const float wv = to_f32(wk[(int64_t)d * d_c]);
#pragma unroll
    for (int j = 0; j < kBatchChunk; ++j) acc[j] = fmaf(qs[j * d_h + d], wv, acc[j]);
  }
  for (int j = 0; j < nb; ++j) qt[((int64_t)(b0 + j) * n_h + h) * d_c + c] = from_f32<T>(acc[j]);
}

// ----------------------------------------------------------------------------------------
// out_up: one warp per output feature d of one head; lanes stride over the latent axis
// ----------------------------------------------------------------------------------------
template <typename T>
__global__ void out_up_simt(int n_h, int d_c, int d_h, int d_v, int B, const T* __restrict__ ctx,
                            const T* __restrict__ w, T* __restrict__ out) {
  extern __shared__ float cs[];  // [kBatchChunk][d_c]
  const int h = blockIdx.x;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int d = blockIdx.y * (blockDim.x >> 5) + warp;
  const int b0 = blockIdx.z * kBatchChunk;
  const int nb = min(kBatchChunk, B - b0);
  for (int i = threadIdx.x; i < nb * d_c; i += blockDim.x) {
    const int j = i / d_c, c = i % d_c;
    cs[i] = to_f32(ctx[((int64_t)(b0 + j) * n_h + h) * d_c + c]);
  }
  __syncthreads();
  if (d >= d_v) return;
  float acc[kBatchChunk];
#pragma unroll
  for (int j = 0; j < kBatchChunk; ++j) acc[j] = 0.f;
  const T* wv = w + ((int64_t)h * (d_h + d_v) + d_h + d) * d_c;
  for (int c = lane; c < d_c; c += 32) {
    const float x = to_f32(wv[c]);
#pragma unroll
    for (int j = 0; j < kBatchChunk; ++j) acc[j] = fmaf(cs[j * d_c + c], x, acc[j]);
  }
#pragma unroll
  for (int j = 0; j < kBatchChunk; ++j) acc[j] = warp_sum(acc[j]);
  if (lane == 0)
    for (int j = 0; j < nb; ++j) out[((int64_t)(b0 + j) * n_h + h) * d_v + d] = from_f32<T>(acc[j]);
}

// ----------------------------------------------------------------------------------------
// decode: one warp per (head, query group, split); lanes own latent columns lane + 32 i.
// kMulti: several new tokens per sequence, each with its own top-k set: query group b is token
// b % T of cache sequence b / T, and it sees the cached rows t <= length - T + (b % T) of its set
// (the prefill's causal rule applied after the set, as in the sparse prefill).
// ----------------------------------------------------------------------------------------
template <typename T, int NC, int NR, bool kMulti>
__global__ void decode_simt(DecodeArgs a, int n_splits, float* __restrict__ ws_o,
                            float2* __restrict__ ws_ml) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int h = blockIdx.x * (blockDim.x >> 5) + warp;
  const int b = blockIdx.y, split = blockIdx.z;
  if (h >= a.n_h) return;
  const int seq = kMulti ? b / a.T : b;  // cache sequence of this query group
  int len = a.lengths[seq];
  bool bad_len = false;
  if (len < (kMulti ? a.T : 1) || len > a.n_max) {
    if (lane == 0 && h == 0 && split == 0) raise_error(a.err, MLA_ERR_LENGTH);
    len = len < 0 ? 0 : (len > a.n_max ? a.n_max : len);
    bad_len = kMulti;  // several tokens: the sequence's tokens get ctx = 0 and lse = -inf
  }
  const int last = kMulti ? len - a.T + b % a.T : len - 1;  // the last row this query sees
  const int n_keys_cap = a.topk_idx ? a.topk : a.n_max;
  const int n_keys = a.topk_idx ? a.topk : len;
  const int chunk = (n_keys_cap + n_splits - 1) / n_splits;
  const int j0 = split * chunk;
  const int j1 = bad_len ? j0 : min(j0 + chunk, n_keys);

  const T* qt = static_cast<const T*>(a.q_tilde) + ((int64_t)b * a.n_h + h) * a.ldqt;
  const T* qp = static_cast<const T*>(a.q_pe) + ((int64_t)b * a.n_h + h) * a.ldqp;
  float q[NC], qr[NR], acc[NC];
#pragma unroll
  for (int i = 0; i < NC; ++i) {
    const int c = lane + 32 * i;
    q[i] = c < a.d_c ? to_f32(qt[c]) : 0.f;
    acc[i] = 0.f;
  }
#pragma unroll
  for (int i = 0; i < NR; ++i) {
    const int r = lane + 32 * i;
    qr[i] = r < a.d_r ? to_f32(qp[r]) : 0.f;
  }
  const T* cb = static_cast<const T*>(a.c_kv) + (int64_t)seq * a.ckv_b;
  const T* rb = static_cast<const T*>(a.k_r) + (int64_t)seq * a.kr_b;
  float m = -INFINITY, l = 0.f;
  for (int j = j0; j < j1; ++j) {
    int t = j;
    if (a.topk_idx) {
      t = a.topk_idx[(int64_t)b * a.topk + j];
      if (t < 0 || t >= len) {
        if (lane == 0 && h == 0) raise_error(a.err, MLA_ERR_INDEX);
        continue;
      }
      if (kMulti && t > last) continue;  // a later new token's row: removed by the causal rule
    }
    const T* crow = cb + (int64_t)t * a.ckv_r;
    const T* rrow = rb + (int64_t)t * a.kr_r;
    float cv[NC];
    float dot = 0.f;
#pragma unroll
    for (int i = 0; i < NC; ++i) {
      const int c = lane + 32 * i;
      cv[i] = c < a.d_c ? to_f32(crow[c]) : 0.f;
      dot = fmaf(q[i], cv[i], dot);
    }
#pragma unroll
    for (int i = 0; i < NR; ++i) {
      const int r = lane + 32 * i;
      if (r < a.d_r) dot = fmaf(qr[i], to_f32(rrow[r]), dot);
    }
    const float s = warp_sum(dot) * a.scale;
    const float m_new = fmaxf(m, s);
    const float corr = expf(m - m_new);
    const float p = expf(s - m_new);
    l = fmaf(l, corr, p);
#pragma unroll
    for (int i = 0; i < NC; ++i) acc[i] = fmaf(acc[i], corr, p * cv[i]);
    m = m_new;
  }
  if (n_splits == 1) {
    T* out = static_cast<T*>(a.ctx) + ((int64_t)b * a.n_h + h) * a.d_c;
    const float inv = l > 0.f ? 1.f / l : 0.f;
#pragma unroll
    for (int i = 0; i < NC; ++i) {
      const int c = lane + 32 * i;
      if (c < a.d_c) out[c] = from_f32<T>(acc[i] * inv);
    }
    if (a.lse && lane == 0) a.lse[(int64_t)b * a.n_h + h] = l > 0.f ? m + logf(l) : -INFINITY;
  } else {
    const int64_t row = ((int64_t)split * a.B + b) * a.n_h + h;
    float* o = ws_o + row * a.d_c;
#pragma unroll
    for (int i = 0; i < NC; ++i) {
      const int c = lane + 32 * i;
      if (c < a.d_c) o[c] = acc[i];
    }
    if (lane == 0) ws_ml[row] = make_float2(m, l);
  }
}

template <typename T>
__global__ void combine_simt(DecodeArgs a, int n_splits, const float* __restrict__ ws_o,
                             const float2* __restrict__ ws_ml) {
  const int h = blockIdx.x, b = blockIdx.y;
  float M = -INFINITY;
  for (int s = 0; s < n_splits; ++s) M = fmaxf(M, ws_ml[((int64_t)s * a.B + b) * a.n_h + h].x);
  float L = 0.f;
  for (int s = 0; s < n_splits; ++s) {
    const float2 ml = ws_ml[((int64_t)s * a.B + b) * a.n_h + h];
    if (ml.y > 0.f) L += ml.y * expf(ml.x - M);
  }
  const float inv = L > 0.f ? 1.f / L : 0.f;
  T* out = static_cast<T*>(a.ctx) + ((int64_t)b * a.n_h + h) * a.d_c;
  for (int c = threadIdx.x; c < a.d_c; c += blockDim.x) {
    float acc = 0.f;
    for (int s = 0; s < n_splits; ++s) {
      const int64_t row = ((int64_t)s * a.B + b) * a.n_h + h;
      const float2 ml = ws_ml[row];
      if (ml.y > 0.f) acc = fmaf(expf(ml.x - M), ws_o[row * a.d_c + c], acc);
    }
    out[c] = from_f32<T>(acc * inv);
  }
  if (a.lse && threadIdx.x == 0) a.lse[(int64_t)b * a.n_h + h] = L > 0.f ? M + logf(L) : -INFINITY;
}

// ----------------------------------------------------------------------------------------
// prefill: expansion GEMM kv = c_kv W^T (64x64 tiles), then one warp per (query, head)
// ----------------------------------------------------------------------------------------
template <typename T>
__global__ void expand_simt(int M, int N, int K, const T* __restrict__ A, int64_t lda,
                            const T* __restrict__ W, T* __restrict__ C) {
  __shared__ float As[16][64 + 1];
  __shared__ float Ws[16][64 + 1];
  const int tx = threadIdx.x % 16, ty = threadIdx.x / 16;  // 256 threads, 4x4 outputs each
  const int m0 = blockIdx.y * 64, n0 = blockIdx.x * 64;
  float acc[4][4] = {};
  for (int k0 = 0; k0 < K; k0 += 16) {
    for (int i = threadIdx.x; i < 64 * 16; i += 256) {
      const int r = i / 16, k = i % 16;
      As[k][r] = (m0 + r < M && k0 + k < K) ? to_f32(A[(int64_t)(m0 + r) * lda + k0 + k]) : 0.f;
      Ws[k][r] = (n0 + r < N && k0 + k < K) ? to_f32(W[(int64_t)(n0 + r) * K + k0 + k]) : 0.f;
    }
    __syncthreads();
#pragma unroll
    for (int k = 0; k < 16; ++k) {
      float av[4], wv[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) { av[i] = As[k][ty * 4 + i]; wv[i] = Ws[k][tx * 4 + i]; }
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(av[i], wv[j], acc[i][j]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int m = m0 + ty * 4 + i, n = n0 + tx * 4 + j;
      if (m < M && n < N) C[(int64_t)m * N + n] = from_f32<T>(acc[i][j]);
    }
}

template <typename T, int ND, int NR, int NV>
__global__ void prefill_attn_simt(PrefillArgs a) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int h = blockIdx.x * (blockDim.x >> 5) + warp;
  const int s = blockIdx.y, b = blockIdx.z;
  if (h >= a.n_h) return;
  const int dqk = a.d_h + a.d_r, dkv = a.d_h + a.d_v;
  const T* qrow = static_cast<const T*>(a.q) + (((int64_t)b * a.S + s) * a.n_h + h) * dqk;
  float qn[ND], qr[NR], acc[NV];
#pragma unroll
  for (int i = 0; i < ND; ++i) { const int d = lane + 32 * i; qn[i] = d < a.d_h ? to_f32(qrow[d]) : 0.f; }
#pragma unroll
  for (int i = 0; i < NR; ++i) { const int r = lane + 32 * i; qr[i] = r < a.d_r ? to_f32(qrow[a.d_h + r]) : 0.f; }
#pragma unroll
  for (int i = 0; i < NV; ++i) acc[i] = 0.f;
  const T* kv = static_cast<const T*>(a.kv);
  const T* kr = static_cast<const T*>(a.k_r);
  const int t_end = a.causal ? s + 1 : a.S;
  float m = -INFINITY, l = 0.f;
  for (int t = 0; t < t_end; ++t) {
    const T* krow = kv + (((int64_t)b * a.S + t) * a.n_h + h) * dkv;
    const T* rrow = kr + ((int64_t)b * a.S + t) * a.kr_r;
    float dot = 0.f;
#pragma unroll
    for (int i = 0; i < ND; ++i) { const int d = lane + 32 * i; if (d < a.d_h) dot = fmaf(qn[i], to_f32(krow[d]), dot); }
#pragma unroll
    for (int i = 0; i < NR; ++i) { const int r = lane + 32 * i; if (r < a.d_r) dot = fmaf(qr[i], to_f32(rrow[r]), dot); }
    const float sc = warp_sum(dot) * a.scale;
    const float m_new = fmaxf(m, sc);
    const float corr = expf(m - m_new);
    const float p = expf(sc - m_new);
    l = fmaf(l, corr, p);
#pragma unroll
    for (int i = 0; i < NV; ++i) {
      const int d = lane + 32 * i;
      const float v = d < a.d_v ? to_f32(krow[a.d_h + d]) : 0.f;
      acc[i] = fmaf(acc[i], corr, p * v);
    }
    m = m_new;
  }
  T* orow = static_cast<T*>(a.out) + (((int64_t)b * a.S + s) * a.n_h + h) * a.d_v;
  const float inv = 1.f / l;
#pragma unroll
  for (int i = 0; i < NV; ++i) { const int d = lane + 32 * i; if (d < a.d_v) orow[d] = from_f32<T>(acc[i] * inv); }
}

inline cudaError_t launch_check() { return cudaGetLastError(); }

}  // namespace

// ------------------------------------------------------------------------------------------
// Host launchers
// ------------------------------------------------------------------------------------------

template <typename T>
cudaError_t absorb_q_simt_launch(int n_h, int d_c, int d_h, int d_v, int B, const void* q, int64_t ldq,
                                 const void* w, void* qt, cudaStream_t st) {
  dim3 grid(n_h, (d_c + 127) / 128, (B + kBatchChunk - 1) / kBatchChunk);
  const size_t smem = sizeof(float) * kBatchChunk * d_h;
  absorb_q_simt<T><<<grid, 128, smem, st>>>(n_h, d_c, d_h, d_v, B, static_cast<const T*>(q), ldq,
                                            static_cast<const T*>(w), static_cast<T*>(qt));
  return launch_check();
}

template <typename T>
cudaError_t out_up_simt_launch(int n_h, int d_c, int d_h, int d_v, int B, const void* ctx, const void* w,
                               void* out, cudaStream_t st) {
  dim3 grid(n_h, (d_v + 7) / 8, (B + kBatchChunk - 1) / kBatchChunk);
  const size_t smem = sizeof(float) * kBatchChunk * d_c;
  if (smem > 48 * 1024)
    cudaFuncSetAttribute(out_up_simt<T>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  out_up_simt<T><<<grid, 256, smem, st>>>(n_h, d_c, d_h, d_v, B, static_cast<const T*>(ctx),
                                          static_cast<const T*>(w), static_cast<T*>(out));
  return launch_check();
}

int decode_simt_splits(int B, int n_keys_cap) {
  // enough (head-group, sequence, split) blocks to cover the GPU a few times over
  int s = (n_keys_cap + 255) / 256;
  const int want = (4 * 148 + B - 1) / B;
  if (s > want) s = want;
  if (s > 64) s = 64;
  return s < 1 ? 1 : s;
}

size_t decode_simt_workspace(int n_h, int d_c, int B, int n_keys_cap) {
  const int s = decode_simt_splits(B, n_keys_cap);
  if (s == 1) return 256;
  return (size_t)s * B * n_h * (d_c * sizeof(float) + sizeof(float2)) + 256;
}

template <typename T, bool kMulti>
void decode_simt_dispatch(const DecodeArgs& a, dim3 grid, int splits, float* ws_o, float2* ws_ml, cudaStream_t st) {
  if (a.d_c <= 64 && a.d_r <= 32)
    decode_simt<T, 2, 1, kMulti><<<grid, 128, 0, st>>>(a, splits, ws_o, ws_ml);
  else if (a.d_c <= 512 && a.d_r <= 64)
    decode_simt<T, 16, 2, kMulti><<<grid, 128, 0, st>>>(a, splits, ws_o, ws_ml);
  else
    decode_simt<T, 32, 4, kMulti><<<grid, 128, 0, st>>>(a, splits, ws_o, ws_ml);
}

// a.B query groups; a.T > 1 (with a top-k set) is the several-token decode over a.B / a.T sequences
template <typename T>
cudaError_t decode_simt_launch(const DecodeArgs& a, void* ws, cudaStream_t st) {
  const int n_keys_cap = a.topk_idx ? a.topk : a.n_max;
  const int splits = decode_simt_splits(a.B, n_keys_cap);
  float* ws_o = static_cast<float*>(ws);
  float2* ws_ml = reinterpret_cast<float2*>(ws_o + (size_t)splits * a.B * a.n_h * a.d_c);
  dim3 grid((a.n_h + 3) / 4, a.B, splits);
  if (a.T > 1 && a.topk_idx)
    decode_simt_dispatch<T, true>(a, grid, splits, ws_o, ws_ml, st);
  else
    decode_simt_dispatch<T, false>(a, grid, splits, ws_o, ws_ml, st);
  cudaError_t e = launch_check();
  if (e != cudaSuccess || splits == 1) return e;
  combine_simt<T><<<dim3(a.n_h, a.B), 128, 0, st>>>(a, splits, ws_o, ws_ml);
  return launch_check();
}

template <typename T>
cudaError_t prefill_attn_simt_launch(const PrefillArgs& a, cudaStream_t st) {
  dim3 grid((a.n_h + 3) / 4, a.S, a.B);
  if (a.d_h <= 32 && a.d_r <= 32 && a.d_v <= 32)
    prefill_attn_simt<T, 1, 1, 1><<<grid, 128, 0, st>>>(a);
  else
    prefill_attn_simt<T, 8, 4, 8><<<grid, 128, 0, st>>>(a);
  return launch_check();
}

template <typename T>
cudaError_t prefill_simt_launch(const PrefillArgs& a, cudaStream_t st) {
  const int M = a.B * a.S, N = a.n_h * (a.d_h + a.d_v), K = a.d_c;
  // the expansion reads c_kv rows with their own stride; rows of different sequences are
  // contiguous in the flattened [B*S] row index because c_kv row (b,s) is at (b*S + s)*stride
  expand_simt<T><<<dim3((N + 63) / 64, (M + 63) / 64), 256, 0, st>>>(
      M, N, K, static_cast<const T*>(a.c_kv), a.ckv_r, static_cast<const T*>(a.w), static_cast<T*>(a.kv));
  cudaError_t e = launch_check();
  if (e != cudaSuccess) return e;
  dim3 grid((a.n_h + 3) / 4, a.S, a.B);
  if (a.d_h <= 32 && a.d_r <= 32 && a.d_v <= 32)
    prefill_attn_simt<T, 1, 1, 1><<<grid, 128, 0, st>>>(a);
  else
    prefill_attn_simt<T, 8, 4, 8><<<grid, 128, 0, st>>>(a);
  return launch_check();
}

#define MLA_INSTANTIATE(T)                                                                            \
  template cudaError_t absorb_q_simt_launch<T>(int, int, int, int, int, const void*, int64_t, const void*, \
                                               void*, cudaStream_t);                                  \
  template cudaError_t out_up_simt_launch<T>(int, int, int, int, int, const void*, const void*, void*,    \
                                             cudaStream_t);                                           \
  template cudaError_t decode_simt_launch<T>(const DecodeArgs&, void*, cudaStream_t);                  \
  template cudaError_t prefill_simt_launch<T>(const PrefillArgs&, cudaStream_t);                    \
  template cudaError_t prefill_attn_simt_launch<T>(const PrefillArgs&, cudaStream_t);

MLA_INSTANTIATE(float)
MLA_INSTANTIATE(__nv_bfloat16)

}  // namespace mla

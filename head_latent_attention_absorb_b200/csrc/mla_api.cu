// C-ABI entry points of libmla_b200.so: host-side validation, then dispatch to the kernels.
// Every check that can be made on the host is made here, before anything is launched.
#include <stdarg.h>
#include <stdio.h>
#include <string.h>

#include "common.cuh"
#include "kernels.h"
#include "mla_api.h"

namespace {

thread_local char g_msg[512] = "";

mla_status fail(mla_status s, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_msg, sizeof(g_msg), fmt, ap);
  va_end(ap);
  return s;
}

mla_status cuda_status(cudaError_t e, const char* where) {
  if (e == cudaSuccess) return MLA_OK;
  return fail(MLA_ERR_CUDA, "%s: %s", where, cudaGetErrorString(e));
}

bool is_deepseek(const mla_dims& d) {
  return d.n_h == 128 && d.d_c == 512 && d.d_r == 64 && d.d_h == 128 && d.d_v == 128;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

mla_status check_dims(const mla_dims& d, mla_dtype dt) {
  if (d.n_h <= 0 || d.d_c <= 0 || d.d_r <= 0 || d.d_h <= 0 || d.d_v <= 0)
    return fail(MLA_ERR_INVALID_ARG, "dimensions must be positive (n_h=%d d_c=%d d_r=%d d_h=%d d_v=%d)",
                d.n_h, d.d_c, d.d_r, d.d_h, d.d_v);
  if (dt == MLA_BF16) {
    if (!is_deepseek(d))
      return fail(MLA_ERR_UNSUPPORTED, "bf16 kernels need n_h=128 d_c=512 d_r=64 d_h=d_v=128");
    return MLA_OK;
  }
  if (dt == MLA_F32) {
    if (d.n_h > 1024 || d.d_c > 1024 || d.d_r > 128 || d.d_h > 256 || d.d_v > 256)
      return fail(MLA_ERR_UNSUPPORTED, "fp32 kernels accept n_h, d_c <= 1024, d_r <= 128, d_h, d_v <= 256");
    return MLA_OK;
  }
  return fail(MLA_ERR_INVALID_ARG, "unknown dtype %d", (int)dt);
}

// bf16 operands feed 16-byte vector loads and TMA: pointers 16-byte aligned, strides 8-element multiples
mla_status check_bf16_ptr(mla_dtype dt, const void* p, const char* name) {
  if (dt == MLA_BF16 && !aligned16(p)) return fail(MLA_ERR_INVALID_ARG, "%s must be 16-byte aligned", name);
  return MLA_OK;
}
mla_status check_bf16_stride(mla_dtype dt, int64_t s, const char* name) {
  if (dt == MLA_BF16 && (s % 8) != 0) return fail(MLA_ERR_INVALID_ARG, "%s must be a multiple of 8 elements", name);
  return MLA_OK;
}

#define MLA_TRY(x)                   \
  do {                               \
    mla_status _s = (x);             \
    if (_s != MLA_OK) return _s;     \
  } while (0)

}  // namespace

extern "C" {

int32_t mla_abi_version(void) { return MLA_ABI_VERSION; }

const char* mla_status_string(mla_status s) {
  switch (s) {
    case MLA_OK: return "MLA_OK";
    case MLA_ERR_INVALID_ARG: return "MLA_ERR_INVALID_ARG: invalid argument";
    case MLA_ERR_UNSUPPORTED: return "MLA_ERR_UNSUPPORTED: no kernel for these dimensions / dtype";
    case MLA_ERR_CUDA: return "MLA_ERR_CUDA: CUDA runtime error";
    case MLA_ERR_INDEX: return "MLA_ERR_INDEX: top-k index outside [0, length)";
    case MLA_ERR_TIMEOUT: return "MLA_ERR_TIMEOUT: bounded wait in a kernel ran out";
    case MLA_ERR_WORKSPACE: return "MLA_ERR_WORKSPACE: workspace missing or too small";
    case MLA_ERR_LENGTH: return "MLA_ERR_LENGTH: sequence length outside [1, n_max]";
  }
  return "unknown mla_status";
}

const char* mla_last_error_message(void) { return g_msg; }

mla_status mla_absorb_q(mla_dims dims, mla_dtype dtype, int32_t B, const void* q_nope, int64_t ldq,
                        const void* w_kv_b, void* q_tilde, void* stream) {
  g_msg[0] = 0;
  MLA_TRY(check_dims(dims, dtype));
  if (B <= 0) return fail(MLA_ERR_INVALID_ARG, "B must be positive");
  if (!q_nope || !w_kv_b || !q_tilde) return fail(MLA_ERR_INVALID_ARG, "NULL pointer");
  if (ldq < dims.d_h) return fail(MLA_ERR_INVALID_ARG, "ldq < d_h");
  MLA_TRY(check_bf16_ptr(dtype, q_nope, "q_nope"));
  MLA_TRY(check_bf16_ptr(dtype, w_kv_b, "w_kv_b"));
  MLA_TRY(check_bf16_ptr(dtype, q_tilde, "q_tilde"));
  MLA_TRY(check_bf16_stride(dtype, ldq, "ldq"));
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  cudaError_t e;
  if (dtype == MLA_BF16)
    e = mla::absorb_q_tc_launch(B, q_nope, ldq, w_kv_b, q_tilde, st);
  else
    e = mla::absorb_q_simt_launch<float>(dims.n_h, dims.d_c, dims.d_h, dims.d_v, B, q_nope, ldq, w_kv_b, q_tilde, st);
  return cuda_status(e, "mla_absorb_q launch");
}

size_t mla_decode_workspace_size(mla_dims dims, mla_dtype dtype, int32_t B, int32_t n_max, int32_t topk) {
  if (check_dims(dims, dtype) != MLA_OK || B <= 0 || n_max <= 0 || topk < 0) return 0;
  // bf16 runs the tensor-core kernel (the sparse variant falls back to the CUDA-core kernel for a
  // cache whose batch stride is not n_max rows: size for both); fp32 the CUDA-core kernels
  if (dtype == MLA_BF16 && topk == 0) return mla::decode_tc_workspace(B);
  const int cap = topk > 0 ? topk : n_max;
  const size_t simt = mla::decode_simt_workspace(dims.n_h, dims.d_c, B, cap);
  if (dtype == MLA_BF16) {
    const size_t tc = mla::decode_tc_workspace(B);
    return tc > simt ? tc : simt;
  }
  return simt;
}

int32_t mla_decode_num_launches(mla_dims dims, mla_dtype dtype, int32_t B, int32_t n_max, int32_t topk) {
  if (check_dims(dims, dtype) != MLA_OK || B <= 0 || n_max <= 0 || topk < 0) return 0;
  const int cap = topk > 0 ? topk : n_max;
  if (dtype == MLA_BF16) return 1;  // tensor-core decode, partials merged in-kernel
  return mla::decode_simt_splits(B, cap) > 1 ? 2 : 1;
}

mla_status mla_decode_absorb(mla_dims dims, mla_dtype dtype, int32_t B, const void* q_tilde, int64_t ldqt,
                             const void* q_pe, int64_t ldqp, const void* c_kv, int64_t ckv_bstride,
                             int64_t ckv_rstride, const void* k_r, int64_t kr_bstride, int64_t kr_rstride,
                             int32_t n_max, const int32_t* lengths, const int32_t* topk_idx, int32_t topk,
                             float scale, void* ctx_out, float* lse_out, void* workspace, size_t ws_bytes,
                             int32_t* dev_err, void* stream) {
  g_msg[0] = 0;
  MLA_TRY(check_dims(dims, dtype));
  if (B <= 0 || n_max <= 0) return fail(MLA_ERR_INVALID_ARG, "B and n_max must be positive");
  if (!q_tilde || !q_pe || !c_kv || !k_r || !lengths || !ctx_out)
    return fail(MLA_ERR_INVALID_ARG, "NULL pointer");
  if (topk_idx && (topk < 1 || topk > n_max)) return fail(MLA_ERR_INVALID_ARG, "topk must lie in [1, n_max]");
  if (ldqt < dims.d_c || ldqp < dims.d_r) return fail(MLA_ERR_INVALID_ARG, "query row stride too small");
  if (ckv_rstride < dims.d_c || kr_rstride < dims.d_r || ckv_bstride < 0 || kr_bstride < 0)
    return fail(MLA_ERR_INVALID_ARG, "cache stride too small");
  if (!(scale > 0.f) || scale != scale) return fail(MLA_ERR_INVALID_ARG, "scale must be positive");
  MLA_TRY(check_bf16_ptr(dtype, q_tilde, "q_tilde"));
  MLA_TRY(check_bf16_ptr(dtype, q_pe, "q_pe"));
  MLA_TRY(check_bf16_ptr(dtype, c_kv, "c_kv"));
  MLA_TRY(check_bf16_ptr(dtype, k_r, "k_r"));
  MLA_TRY(check_bf16_ptr(dtype, ctx_out, "ctx_out"));
  MLA_TRY(check_bf16_stride(dtype, ldqt, "ldqt"));
  MLA_TRY(check_bf16_stride(dtype, ldqp, "ldqp"));
  MLA_TRY(check_bf16_stride(dtype, ckv_bstride, "ckv_bstride"));
  MLA_TRY(check_bf16_stride(dtype, ckv_rstride, "ckv_rstride"));
  MLA_TRY(check_bf16_stride(dtype, kr_bstride, "kr_bstride"));
  MLA_TRY(check_bf16_stride(dtype, kr_rstride, "kr_rstride"));
  if (dtype == MLA_BF16 && !topk_idx && (int64_t)B * ((n_max + 63) / 64) >= ((int64_t)1 << 31))
    return fail(MLA_ERR_UNSUPPORTED, "B * ceil(n_max / 64) must stay below 2^31");
  const size_t need = mla_decode_workspace_size(dims, dtype, B, n_max, topk_idx ? topk : 0);
  if (!workspace || ws_bytes < need)
    return fail(MLA_ERR_WORKSPACE, "workspace needs %zu bytes, got %zu", need, workspace ? ws_bytes : (size_t)0);
  if (!aligned16(workspace)) return fail(MLA_ERR_INVALID_ARG, "workspace must be 16-byte aligned");

  mla::DecodeArgs a;
  a.n_h = dims.n_h; a.d_c = dims.d_c; a.d_r = dims.d_r; a.B = B; a.n_max = n_max;
  a.topk = topk_idx ? topk : 0;
  a.q_tilde = q_tilde; a.ldqt = ldqt; a.q_pe = q_pe; a.ldqp = ldqp;
  a.c_kv = c_kv; a.ckv_b = ckv_bstride; a.ckv_r = ckv_rstride;
  a.k_r = k_r; a.kr_b = kr_bstride; a.kr_r = kr_rstride;
  a.lengths = lengths; a.topk_idx = topk_idx; a.scale = scale;
  a.ctx = ctx_out; a.lse = lse_out; a.err = dev_err;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  cudaError_t e;
  // the sparse tensor-core path gathers rows of the caches viewed as 2-D (B * n_max rows)
  const bool packed = (B == 1 || (ckv_bstride == (int64_t)n_max * ckv_rstride && kr_bstride == (int64_t)n_max * kr_rstride)) &&
                      (int64_t)B * n_max < ((int64_t)1 << 31);
  if (dtype == MLA_BF16 && (!topk_idx || packed))
    e = mla::decode_tc_launch(a, workspace, st);
  else if (dtype == MLA_BF16)
    e = mla::decode_simt_launch<__nv_bfloat16>(a, workspace, st);
  else
    e = mla::decode_simt_launch<float>(a, workspace, st);
  return cuda_status(e, "mla_decode_absorb launch");
}

mla_status mla_decode_absorb_fp8kv(mla_dims dims, int32_t B, const void* q_tilde, int64_t ldqt, const void* q_pe,
                                   int64_t ldqp, const void* c8, int64_t c8_bstride, int64_t c8_rstride,
                                   const float* kv_scale, int64_t sc_bstride, int64_t sc_rstride, const void* k_r,
                                   int64_t kr_bstride, int64_t kr_rstride, int32_t n_max, const int32_t* lengths,
                                   float scale, void* ctx_out, float* lse_out, void* workspace, size_t ws_bytes,
                                   int32_t* dev_err, void* stream) {
  g_msg[0] = 0;
  const mla_dtype dtype = MLA_BF16;
  MLA_TRY(check_dims(dims, dtype));
  if (B <= 0 || n_max <= 0) return fail(MLA_ERR_INVALID_ARG, "B and n_max must be positive");
  if (!q_tilde || !q_pe || !c8 || !kv_scale || !k_r || !lengths || !ctx_out)
    return fail(MLA_ERR_INVALID_ARG, "NULL pointer");
  if (ldqt < dims.d_c || ldqp < dims.d_r) return fail(MLA_ERR_INVALID_ARG, "query row stride too small");
  if (c8_rstride < dims.d_c || kr_rstride < dims.d_r || sc_rstride < dims.d_c / 128 || c8_bstride < 0 ||
      sc_bstride < 0 || kr_bstride < 0)
    return fail(MLA_ERR_INVALID_ARG, "cache stride too small");
  if ((c8_rstride % 16) || (c8_bstride % 16) || (sc_rstride % 4) || (sc_bstride % 4))
    return fail(MLA_ERR_INVALID_ARG, "c8 strides must be multiples of 16 bytes, kv_scale strides of 4 floats");
  if (!(scale > 0.f) || scale != scale) return fail(MLA_ERR_INVALID_ARG, "scale must be positive");
  MLA_TRY(check_bf16_ptr(dtype, q_tilde, "q_tilde"));
  MLA_TRY(check_bf16_ptr(dtype, q_pe, "q_pe"));
  MLA_TRY(check_bf16_ptr(dtype, c8, "c8"));
  MLA_TRY(check_bf16_ptr(dtype, kv_scale, "kv_scale"));
  MLA_TRY(check_bf16_ptr(dtype, k_r, "k_r"));
  MLA_TRY(check_bf16_ptr(dtype, ctx_out, "ctx_out"));
  MLA_TRY(check_bf16_stride(dtype, ldqt, "ldqt"));
  MLA_TRY(check_bf16_stride(dtype, ldqp, "ldqp"));
  MLA_TRY(check_bf16_stride(dtype, kr_bstride, "kr_bstride"));
  MLA_TRY(check_bf16_stride(dtype, kr_rstride, "kr_rstride"));
  if ((int64_t)B * ((n_max + 63) / 64) >= ((int64_t)1 << 31))
    return fail(MLA_ERR_UNSUPPORTED, "B * ceil(n_max / 64) must stay below 2^31");
  const size_t need = mla_decode_workspace_size(dims, dtype, B, n_max, 0);
  if (!workspace || ws_bytes < need)
    return fail(MLA_ERR_WORKSPACE, "workspace needs %zu bytes, got %zu", need, workspace ? ws_bytes : (size_t)0);
  if (!aligned16(workspace)) return fail(MLA_ERR_INVALID_ARG, "workspace must be 16-byte aligned");
  mla::DecodeArgs a;
  a.n_h = dims.n_h; a.d_c = dims.d_c; a.d_r = dims.d_r; a.B = B; a.n_max = n_max;
  a.topk = 0;
  a.q_tilde = q_tilde; a.ldqt = ldqt; a.q_pe = q_pe; a.ldqp = ldqp;
  a.c_kv = c8; a.ckv_b = 0; a.ckv_r = 0;
  a.k_r = k_r; a.kr_b = kr_bstride; a.kr_r = kr_rstride;
  a.lengths = lengths; a.topk_idx = nullptr; a.scale = scale;
  a.ctx = ctx_out; a.lse = lse_out; a.err = dev_err;
  a.c8 = c8; a.c8_b = c8_bstride; a.c8_r = c8_rstride;
  a.kv_scale = kv_scale; a.sc_b = sc_bstride; a.sc_r = sc_rstride;
  return cuda_status(mla::decode_tc_launch(a, workspace, static_cast<cudaStream_t>(stream)),
                     "mla_decode_absorb_fp8kv launch");
}

mla_status mla_decode_absorb_multi(mla_dims dims, mla_dtype dtype, int32_t B, int32_t T, const void* q_tilde,
                                   int64_t ldqt, const void* q_pe, int64_t ldqp, const void* c_kv,
                                   int64_t ckv_bstride, int64_t ckv_rstride, const void* k_r, int64_t kr_bstride,
                                   int64_t kr_rstride, int32_t n_max, const int32_t* lengths, float scale,
                                   void* ctx_out, float* lse_out, void* workspace, size_t ws_bytes,
                                   int32_t* dev_err, void* stream) {
  g_msg[0] = 0;
  if (T == 1)
    return mla_decode_absorb(dims, dtype, B, q_tilde, ldqt, q_pe, ldqp, c_kv, ckv_bstride, ckv_rstride, k_r,
                             kr_bstride, kr_rstride, n_max, lengths, nullptr, 0, scale, ctx_out, lse_out,
                             workspace, ws_bytes, dev_err, stream);
  MLA_TRY(check_dims(dims, dtype));
  if (dtype != MLA_BF16) return fail(MLA_ERR_UNSUPPORTED, "several tokens per sequence: bf16 only");
  if (B <= 0 || T < 1 || n_max <= 0 || T > n_max) return fail(MLA_ERR_INVALID_ARG, "need B > 0 and 1 <= T <= n_max");
  if ((int64_t)B * T * dims.n_h >= ((int64_t)1 << 31)) return fail(MLA_ERR_UNSUPPORTED, "B * T * n_h too large");
  if (!q_tilde || !q_pe || !c_kv || !k_r || !lengths || !ctx_out) return fail(MLA_ERR_INVALID_ARG, "NULL pointer");
  if (ldqt < dims.d_c || ldqp < dims.d_r) return fail(MLA_ERR_INVALID_ARG, "query row stride too small");
  if (ckv_rstride < dims.d_c || kr_rstride < dims.d_r || ckv_bstride < 0 || kr_bstride < 0)
    return fail(MLA_ERR_INVALID_ARG, "cache stride too small");
  if (!(scale > 0.f) || scale != scale) return fail(MLA_ERR_INVALID_ARG, "scale must be positive");
  MLA_TRY(check_bf16_ptr(dtype, q_tilde, "q_tilde"));
  MLA_TRY(check_bf16_ptr(dtype, q_pe, "q_pe"));
  MLA_TRY(check_bf16_ptr(dtype, c_kv, "c_kv"));
  MLA_TRY(check_bf16_ptr(dtype, k_r, "k_r"));
  MLA_TRY(check_bf16_ptr(dtype, ctx_out, "ctx_out"));
  MLA_TRY(check_bf16_stride(dtype, ldqt, "ldqt"));
  MLA_TRY(check_bf16_stride(dtype, ldqp, "ldqp"));
  MLA_TRY(check_bf16_stride(dtype, ckv_bstride, "ckv_bstride"));
  MLA_TRY(check_bf16_stride(dtype, ckv_rstride, "ckv_rstride"));
  MLA_TRY(check_bf16_stride(dtype, kr_bstride, "kr_bstride"));
  MLA_TRY(check_bf16_stride(dtype, kr_rstride, "kr_rstride"));
  const int32_t BT = B * T;
  if ((int64_t)BT * ((n_max + 63) / 64) >= ((int64_t)1 << 31))
    return fail(MLA_ERR_UNSUPPORTED, "B * T * ceil(n_max / 64) must stay below 2^31");
  const size_t need = mla_decode_workspace_size(dims, dtype, BT, n_max, 0);
  if (!workspace || ws_bytes < need)
    return fail(MLA_ERR_WORKSPACE, "workspace needs %zu bytes, got %zu", need, workspace ? ws_bytes : (size_t)0);
  if (!aligned16(workspace)) return fail(MLA_ERR_INVALID_ARG, "workspace must be 16-byte aligned");
  mla::DecodeArgs a;
  a.n_h = dims.n_h; a.d_c = dims.d_c; a.d_r = dims.d_r; a.B = BT; a.T = T; a.n_max = n_max;
  a.topk = 0;
  a.q_tilde = q_tilde; a.ldqt = ldqt; a.q_pe = q_pe; a.ldqp = ldqp;
  a.c_kv = c_kv; a.ckv_b = ckv_bstride; a.ckv_r = ckv_rstride;
  a.k_r = k_r; a.kr_b = kr_bstride; a.kr_r = kr_rstride;
  a.lengths = lengths; a.topk_idx = nullptr; a.scale = scale;
  a.ctx = ctx_out; a.lse = lse_out; a.err = dev_err;
  return cuda_status(mla::decode_pair_launch(a, workspace, static_cast<cudaStream_t>(stream)),
                     "mla_decode_absorb_multi launch");
}

mla_status mla_decode_absorb_multi_topk(mla_dims dims, mla_dtype dtype, int32_t B, int32_t T, const void* q_tilde,
                                        int64_t ldqt, const void* q_pe, int64_t ldqp, const void* c_kv,
                                        int64_t ckv_bstride, int64_t ckv_rstride, const void* k_r,
                                        int64_t kr_bstride, int64_t kr_rstride, int32_t n_max,
                                        const int32_t* lengths, const int32_t* topk_idx, int32_t topk, float scale,
                                        void* ctx_out, float* lse_out, void* workspace, size_t ws_bytes,
                                        int32_t* dev_err, void* stream) {
  g_msg[0] = 0;
  if (!topk_idx) return fail(MLA_ERR_INVALID_ARG, "NULL top-k index array");
  if (T == 1)
    return mla_decode_absorb(dims, dtype, B, q_tilde, ldqt, q_pe, ldqp, c_kv, ckv_bstride, ckv_rstride, k_r,
                             kr_bstride, kr_rstride, n_max, lengths, topk_idx, topk, scale, ctx_out, lse_out,
                             workspace, ws_bytes, dev_err, stream);
  MLA_TRY(check_dims(dims, dtype));
  if (B <= 0 || T < 1 || n_max <= 0 || T > n_max) return fail(MLA_ERR_INVALID_ARG, "need B > 0 and 1 <= T <= n_max");
  if (topk < 1 || topk > n_max) return fail(MLA_ERR_INVALID_ARG, "topk must lie in [1, n_max]");
  if ((int64_t)B * T * dims.n_h >= ((int64_t)1 << 31) || (int64_t)B * T > 65535)
    return fail(MLA_ERR_UNSUPPORTED, "B * T query groups too many");
  if (!q_tilde || !q_pe || !c_kv || !k_r || !lengths || !ctx_out) return fail(MLA_ERR_INVALID_ARG, "NULL pointer");
  if (ldqt < dims.d_c || ldqp < dims.d_r) return fail(MLA_ERR_INVALID_ARG, "query row stride too small");
  if (ckv_rstride < dims.d_c || kr_rstride < dims.d_r || ckv_bstride < 0 || kr_bstride < 0)
    return fail(MLA_ERR_INVALID_ARG, "cache stride too small");
  if (!(scale > 0.f) || scale != scale) return fail(MLA_ERR_INVALID_ARG, "scale must be positive");
  MLA_TRY(check_bf16_ptr(dtype, q_tilde, "q_tilde"));
  MLA_TRY(check_bf16_ptr(dtype, q_pe, "q_pe"));
  MLA_TRY(check_bf16_ptr(dtype, c_kv, "c_kv"));
  MLA_TRY(check_bf16_ptr(dtype, k_r, "k_r"));
  MLA_TRY(check_bf16_ptr(dtype, ctx_out, "ctx_out"));
  const int32_t BT = B * T;
  const size_t need = mla_decode_workspace_size(dims, dtype, BT, n_max, topk);
  if (!workspace || ws_bytes < need)
    return fail(MLA_ERR_WORKSPACE, "workspace needs %zu bytes, got %zu", need, workspace ? ws_bytes : (size_t)0);
  if (!aligned16(workspace)) return fail(MLA_ERR_INVALID_ARG, "workspace must be 16-byte aligned");
  mla::DecodeArgs a;
  a.n_h = dims.n_h; a.d_c = dims.d_c; a.d_r = dims.d_r; a.B = BT; a.T = T; a.n_max = n_max;
  a.topk = topk;
  a.q_tilde = q_tilde; a.ldqt = ldqt; a.q_pe = q_pe; a.ldqp = ldqp;
  a.c_kv = c_kv; a.ckv_b = ckv_bstride; a.ckv_r = ckv_rstride;
  a.k_r = k_r; a.kr_b = kr_bstride; a.kr_r = kr_rstride;
  a.lengths = lengths; a.topk_idx = topk_idx; a.scale = scale;
  a.ctx = ctx_out; a.lse = lse_out; a.err = dev_err;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const cudaError_t e = dtype == MLA_BF16 ? mla::decode_simt_launch<__nv_bfloat16>(a, workspace, st)
                                          : mla::decode_simt_launch<float>(a, workspace, st);
  return cuda_status(e, "mla_decode_absorb_multi_topk launch");
}

mla_status mla_decode_absorb_static(mla_dims dims, mla_dtype dtype, int32_t B, const void* q_tilde, int64_t ldqt,
                                    const void* q_pe, int64_t ldqp, const void* c_kv, int64_t ckv_bstride,
                                    int64_t ckv_rstride, const void* k_r, int64_t kr_bstride, int64_t kr_rstride,
                                    int32_t n_max, const int32_t* lengths, float scale, void* ctx_out,
                                    float* lse_out, int32_t* dev_err, void* stream) {
  g_msg[0] = 0;
  if (dtype != MLA_BF16)
    return fail(MLA_ERR_UNSUPPORTED, "mla_decode_absorb_static covers the bf16 dense decode only");
  MLA_TRY(check_dims(dims, dtype));
  if (B <= 0 || n_max <= 0) return fail(MLA_ERR_INVALID_ARG, "B and n_max must be positive");
  const size_t need = mla_decode_workspace_size(dims, dtype, B, n_max, 0);
  const size_t have = mla::decode_static_scratch_bytes();
  if (need > have)
    return fail(MLA_ERR_WORKSPACE,
                "mla_decode_absorb_static: this call needs %zu bytes of split-KV scratch, the built-in "
                "scratch holds %zu (it is sized for up to 148 SMs and 4096 sequences)", need, have);
  void* scratch = nullptr;
  MLA_TRY(cuda_status(mla::decode_static_scratch(&scratch), "mla_decode_absorb_static scratch set-up"));
  return mla_decode_absorb(dims, dtype, B, q_tilde, ldqt, q_pe, ldqp, c_kv, ckv_bstride, ckv_rstride, k_r,
                           kr_bstride, kr_rstride, n_max, lengths, nullptr, 0, scale, ctx_out, lse_out, scratch,
                           have, dev_err, stream);
}

mla_status mla_out_up(mla_dims dims, mla_dtype dtype, int32_t B, const void* ctx, const void* w_kv_b, void* out,
                      void* stream) {
  g_msg[0] = 0;
  MLA_TRY(check_dims(dims, dtype));
  if (B <= 0) return fail(MLA_ERR_INVALID_ARG, "B must be positive");
  if (!ctx || !w_kv_b || !out) return fail(MLA_ERR_INVALID_ARG, "NULL pointer");
  MLA_TRY(check_bf16_ptr(dtype, ctx, "ctx"));
  MLA_TRY(check_bf16_ptr(dtype, w_kv_b, "w_kv_b"));
  MLA_TRY(check_bf16_ptr(dtype, out, "out"));
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  cudaError_t e;
  if (dtype == MLA_BF16)
    e = mla::out_up_tc_launch(B, ctx, w_kv_b, out, st);
  else
    e = mla::out_up_simt_launch<float>(dims.n_h, dims.d_c, dims.d_h, dims.d_v, B, ctx, w_kv_b, out, st);
  return cuda_status(e, "mla_out_up launch");
}

mla_status mla_absorb_q_fp8(mla_dims dims, int32_t B, const void* q_nope, int64_t ldq, const void* w_fp8,
                            const float* w_scale, void* q_tilde, int32_t* dev_err, void* stream) {
  g_msg[0] = 0;
  MLA_TRY(check_dims(dims, MLA_BF16));
  if (B <= 0) return fail(MLA_ERR_INVALID_ARG, "B must be positive");
  if (!q_nope || !w_fp8 || !w_scale || !q_tilde) return fail(MLA_ERR_INVALID_ARG, "NULL pointer");
  if (ldq < dims.d_h) return fail(MLA_ERR_INVALID_ARG, "ldq smaller than d_h");
  MLA_TRY(check_bf16_ptr(MLA_BF16, q_nope, "q_nope"));
  MLA_TRY(check_bf16_ptr(MLA_BF16, w_fp8, "w_fp8"));
  MLA_TRY(check_bf16_ptr(MLA_BF16, q_tilde, "q_tilde"));
  MLA_TRY(check_bf16_stride(MLA_BF16, ldq, "ldq"));
  return cuda_status(mla::absorb_q_fp8_tc_launch(B, q_nope, ldq, w_fp8, w_scale, q_tilde, dev_err,
                                                 static_cast<cudaStream_t>(stream)),
                     "mla_absorb_q_fp8 launch");
}

mla_status mla_out_up_fp8(mla_dims dims, int32_t B, const void* ctx, const void* w_fp8, const float* w_scale,
                          void* out, int32_t* dev_err, void* stream) {
  g_msg[0] = 0;
  MLA_TRY(check_dims(dims, MLA_BF16));
  if (B <= 0) return fail(MLA_ERR_INVALID_ARG, "B must be positive");
  if (!ctx || !w_fp8 || !w_scale || !out) return fail(MLA_ERR_INVALID_ARG, "NULL pointer");
  MLA_TRY(check_bf16_ptr(MLA_BF16, ctx, "ctx"));
  MLA_TRY(check_bf16_ptr(MLA_BF16, w_fp8, "w_fp8"));
  MLA_TRY(check_bf16_ptr(MLA_BF16, out, "out"));
  return cuda_status(mla::out_up_fp8_tc_launch(B, ctx, w_fp8, w_scale, out, dev_err, static_cast<cudaStream_t>(stream)),
                     "mla_out_up_fp8 launch");
}

size_t mla_prefill_workspace_size(mla_dims dims, mla_dtype dtype, int32_t B, int32_t S) {
  if (check_dims(dims, dtype) != MLA_OK || B <= 0 || S <= 0) return 0;
  const size_t es = dtype == MLA_BF16 ? 2 : 4;
  return (size_t)B * S * dims.n_h * (dims.d_h + dims.d_v) * es;
}

mla_status mla_prefill_naive(mla_dims dims, mla_dtype dtype, int32_t B, int32_t S, const void* q, const void* c_kv,
                             int64_t ckv_rstride, const void* k_r, int64_t kr_rstride, const void* w_kv_b,
                             float scale, int32_t causal, void* out, void* workspace, size_t ws_bytes,
                             void* stream) {
  g_msg[0] = 0;
  MLA_TRY(check_dims(dims, dtype));
  if (B <= 0 || S <= 0) return fail(MLA_ERR_INVALID_ARG, "B and S must be positive");
  if (!q || !c_kv || !k_r || !w_kv_b || !out) return fail(MLA_ERR_INVALID_ARG, "NULL pointer");
  if (ckv_rstride < dims.d_c || kr_rstride < dims.d_r) return fail(MLA_ERR_INVALID_ARG, "row stride too small");
  if (!(scale > 0.f)) return fail(MLA_ERR_INVALID_ARG, "scale must be positive");
  MLA_TRY(check_bf16_ptr(dtype, q, "q"));
  MLA_TRY(check_bf16_ptr(dtype, c_kv, "c_kv"));
  MLA_TRY(check_bf16_ptr(dtype, k_r, "k_r"));
  MLA_TRY(check_bf16_ptr(dtype, w_kv_b, "w_kv_b"));
  MLA_TRY(check_bf16_ptr(dtype, out, "out"));
  MLA_TRY(check_bf16_stride(dtype, ckv_rstride, "ckv_rstride"));
  MLA_TRY(check_bf16_stride(dtype, kr_rstride, "kr_rstride"));
  const size_t need = mla_prefill_workspace_size(dims, dtype, B, S);
  if (!workspace || ws_bytes < need)
    return fail(MLA_ERR_WORKSPACE, "workspace needs %zu bytes, got %zu", need, workspace ? ws_bytes : (size_t)0);
  if (!aligned16(workspace)) return fail(MLA_ERR_INVALID_ARG, "workspace must be 16-byte aligned");
  mla::PrefillArgs a;
  a.n_h = dims.n_h; a.d_c = dims.d_c; a.d_r = dims.d_r; a.d_h = dims.d_h; a.d_v = dims.d_v;
  a.B = B; a.S = S; a.causal = causal ? 1 : 0;
  a.q = q; a.c_kv = c_kv; a.ckv_r = ckv_rstride; a.k_r = k_r; a.kr_r = kr_rstride; a.w = w_kv_b;
  a.scale = scale; a.out = out; a.kv = workspace;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  cudaError_t e;
  if (dtype == MLA_BF16) {
    // tensor-core expansion (needs 16-byte-aligned rows for its TMA maps), then the attention
    e = mla::expand_tc_launch(a, st);
    if (e == cudaSuccess) e = mla::attn_tc_launch(a, st);
  } else {
    e = mla::prefill_simt_launch<float>(a, st);
  }
  return cuda_status(e, "mla_prefill_naive launch");
}

mla_status mla_cache_append(mla_dims dims, mla_dtype dtype, int32_t B, const void* kv_a, int64_t lda,
                            const float* gain, float eps, float rope_base, const int32_t* positions, int32_t n_max,
                            void* c_kv, int64_t ckv_bstride, int64_t ckv_rstride, void* k_r, int64_t kr_bstride,
                            int64_t kr_rstride, int32_t* dev_err, void* stream) {
  g_msg[0] = 0;
  MLA_TRY(check_dims(dims, dtype));
  if (B <= 0 || n_max <= 0) return fail(MLA_ERR_INVALID_ARG, "B and n_max must be positive");
  if (!kv_a || !positions || !c_kv || !k_r) return fail(MLA_ERR_INVALID_ARG, "NULL pointer");
  if (dims.d_r % 2 != 0) return fail(MLA_ERR_INVALID_ARG, "d_r must be even (rotary pairs)");
  if (lda < (int64_t)dims.d_c + dims.d_r) return fail(MLA_ERR_INVALID_ARG, "lda smaller than d_c + d_r");
  if (ckv_rstride < dims.d_c || kr_rstride < dims.d_r) return fail(MLA_ERR_INVALID_ARG, "row stride too small");
  if (ckv_bstride < (int64_t)n_max * ckv_rstride || kr_bstride < (int64_t)n_max * kr_rstride)
    return fail(MLA_ERR_INVALID_ARG, "batch stride smaller than n_max rows");
  if (!(eps >= 0.f) || !(eps < 1e30f)) return fail(MLA_ERR_INVALID_ARG, "eps must be finite and >= 0");
  if (!(rope_base > 0.f) || !(rope_base < 1e30f)) return fail(MLA_ERR_INVALID_ARG, "rope_base must be finite and > 0");
  MLA_TRY(check_bf16_ptr(dtype, kv_a, "kv_a"));
  MLA_TRY(check_bf16_ptr(dtype, c_kv, "c_kv"));
  MLA_TRY(check_bf16_ptr(dtype, k_r, "k_r"));
  MLA_TRY(check_bf16_stride(dtype, lda, "lda"));
  MLA_TRY(check_bf16_stride(dtype, ckv_rstride, "ckv_rstride"));
  MLA_TRY(check_bf16_stride(dtype, kr_rstride, "kr_rstride"));
  MLA_TRY(check_bf16_stride(dtype, ckv_bstride, "ckv_bstride"));
  MLA_TRY(check_bf16_stride(dtype, kr_bstride, "kr_bstride"));
  mla::AppendArgs a;
  a.d_c = dims.d_c; a.d_r = dims.d_r; a.B = B; a.n_max = n_max;
  a.kv_a = kv_a; a.lda = lda; a.gain = gain; a.eps = eps; a.rope_base = rope_base; a.positions = positions;
  a.c_kv = c_kv; a.ckv_b = ckv_bstride; a.ckv_r = ckv_rstride;
  a.k_r = k_r; a.kr_b = kr_bstride; a.kr_r = kr_rstride;
  a.err = dev_err;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const cudaError_t e = dtype == MLA_BF16 ? mla::cache_append_launch<__nv_bfloat16>(a, st)
                                          : mla::cache_append_launch<float>(a, st);
  return cuda_status(e, "mla_cache_append launch");
}

mla_status mla_check_topk(int32_t B, const int32_t* topk_idx, int32_t topk, const int32_t* lengths, int32_t n_max,
                          int32_t* dev_err, void* stream) {
  g_msg[0] = 0;
  if (B <= 0 || topk <= 0 || n_max <= 0) return fail(MLA_ERR_INVALID_ARG, "B, topk and n_max must be positive");
  if (!topk_idx || !dev_err) return fail(MLA_ERR_INVALID_ARG, "NULL pointer");
  if (mla::check_topk_smem_bytes(n_max) > 232448)
    return fail(MLA_ERR_UNSUPPORTED, "n_max %d: the position bitmap exceeds shared memory", n_max);
  return cuda_status(mla::check_topk_launch(B, topk_idx, topk, lengths, n_max, dev_err,
                                            static_cast<cudaStream_t>(stream)),
                     "mla_check_topk launch");
}

size_t mla_prefill_sparse_workspace_size(mla_dims dims, mla_dtype dtype, int32_t B, int32_t S) {
  const size_t dense = mla_prefill_workspace_size(dims, dtype, B, S);
  if (dense == 0 || dtype != MLA_BF16) return 0;
  return ((dense + 255) & ~(size_t)255) + mla::sparse_prefill_scratch_bytes(B, S);
}

mla_status mla_prefill_sparse(mla_dims dims, mla_dtype dtype, int32_t B, int32_t S, const void* q, const void* c_kv,
                              int64_t ckv_rstride, const void* k_r, int64_t kr_rstride, const void* w_kv_b,
                              float scale, const int32_t* topk_idx, int32_t topk, void* out, void* workspace,
                              size_t ws_bytes, int32_t* dev_err, void* stream) {
  g_msg[0] = 0;
  MLA_TRY(check_dims(dims, dtype));
  if (dtype != MLA_BF16) return fail(MLA_ERR_UNSUPPORTED, "mla_prefill_sparse covers bf16 only");
  if (B <= 0 || S <= 0 || topk <= 0) return fail(MLA_ERR_INVALID_ARG, "B, S and topk must be positive");
  if (!q || !c_kv || !k_r || !w_kv_b || !out || !topk_idx) return fail(MLA_ERR_INVALID_ARG, "NULL pointer");
  if (ckv_rstride < dims.d_c || kr_rstride < dims.d_r) return fail(MLA_ERR_INVALID_ARG, "row stride too small");
  if (!(scale > 0.f)) return fail(MLA_ERR_INVALID_ARG, "scale must be positive");
  MLA_TRY(check_bf16_ptr(dtype, q, "q"));
  MLA_TRY(check_bf16_ptr(dtype, c_kv, "c_kv"));
  MLA_TRY(check_bf16_ptr(dtype, k_r, "k_r"));
  MLA_TRY(check_bf16_ptr(dtype, w_kv_b, "w_kv_b"));
  MLA_TRY(check_bf16_ptr(dtype, out, "out"));
  MLA_TRY(check_bf16_stride(dtype, ckv_rstride, "ckv_rstride"));
  MLA_TRY(check_bf16_stride(dtype, kr_rstride, "kr_rstride"));
  const size_t need = mla_prefill_sparse_workspace_size(dims, dtype, B, S);
  if (!workspace || ws_bytes < need)
    return fail(MLA_ERR_WORKSPACE, "workspace needs %zu bytes, got %zu", need, workspace ? ws_bytes : (size_t)0);
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
    return fail(MLA_ERR_INVALID_ARG, "workspace must be 256-byte aligned");
  if ((size_t)16 * ((S + 127) / 128) > 48 * 1024) return fail(MLA_ERR_UNSUPPORTED, "S too long for the row bitmap");
  mla::PrefillArgs a;
  a.n_h = dims.n_h; a.d_c = dims.d_c; a.d_r = dims.d_r; a.d_h = dims.d_h; a.d_v = dims.d_v;
  a.B = B; a.S = S; a.causal = 1;
  a.q = q; a.c_kv = c_kv; a.ckv_r = ckv_rstride; a.k_r = k_r; a.kr_r = kr_rstride; a.w = w_kv_b;
  a.scale = scale; a.out = out; a.kv = workspace;
  void* scratch = static_cast<uint8_t*>(workspace) + ((mla_prefill_workspace_size(dims, dtype, B, S) + 255) & ~(size_t)255);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  cudaError_t e = mla::sparse_masks_launch(a, topk_idx, topk, scratch, dev_err, st);
  if (e == cudaSuccess) e = mla::expand_tc_launch(a, st);
  if (e == cudaSuccess) e = mla::attn_sparse_tc_launch(a, scratch, dev_err, st);
  return cuda_status(e, "mla_prefill_sparse launch");
}

mla_status mla_selftest_wait_timeout(uint64_t limit_ns, int32_t* dev_err, void* stream) {
  g_msg[0] = 0;
  if (!dev_err) return fail(MLA_ERR_INVALID_ARG, "NULL pointer");
  if (limit_ns < 1000 || limit_ns > 1000000000ull) return fail(MLA_ERR_INVALID_ARG, "limit_ns outside [1 us, 1 s]");
  return cuda_status(mla::wait_timeout_launch(limit_ns, dev_err, static_cast<cudaStream_t>(stream)),
                     "mla_selftest_wait_timeout launch");
}

mla_status mla_clear_device_error(int32_t* dev_err, void* stream) {
  g_msg[0] = 0;
  if (!dev_err) return fail(MLA_ERR_INVALID_ARG, "NULL pointer");
  return cuda_status(cudaMemsetAsync(dev_err, 0, sizeof(int32_t), static_cast<cudaStream_t>(stream)),
                     "mla_clear_device_error");
}

mla_status mla_get_device_error(const int32_t* dev_err, int32_t* host_out) {
  g_msg[0] = 0;
  if (!dev_err || !host_out) return fail(MLA_ERR_INVALID_ARG, "NULL pointer");
  MLA_TRY(cuda_status(cudaDeviceSynchronize(), "mla_get_device_error sync"));
  return cuda_status(cudaMemcpy(host_out, dev_err, sizeof(int32_t), cudaMemcpyDeviceToHost),
                     "mla_get_device_error copy");
}

}  // extern "C"

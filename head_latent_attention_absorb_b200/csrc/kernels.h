// Kernel launchers behind the C-ABI (internal to libmla_b200.so).
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "common.cuh"

namespace mla {

// ---- CUDA-core kernels, any dimensions (fp32 element type) -------------------------------
template <typename T>
cudaError_t absorb_q_simt_launch(int n_h, int d_c, int d_h, int d_v, int B, const void* q, int64_t ldq,
                                 const void* w, void* qt, cudaStream_t st);
template <typename T>
cudaError_t out_up_simt_launch(int n_h, int d_c, int d_h, int d_v, int B, const void* ctx, const void* w,
                               void* out, cudaStream_t st);
template <typename T>
cudaError_t decode_simt_launch(const DecodeArgs& a, void* ws, cudaStream_t st);
template <typename T>
cudaError_t prefill_simt_launch(const PrefillArgs& a, cudaStream_t st);

int decode_simt_splits(int B, int n_keys_cap);

// ---- cache append (any dimensions; float or __nv_bfloat16) ---------------------------------
template <typename T>
cudaError_t cache_append_launch(const AppendArgs& a, cudaStream_t st);

// ---- top-k index validation (range and distinctness per sequence) --------------------------
size_t check_topk_smem_bytes(int n_max);
cudaError_t wait_timeout_launch(uint64_t limit_ns, int32_t* err, cudaStream_t st);
cudaError_t check_topk_launch(int B, const int32_t* idx, int topk, const int32_t* lengths, int n_max, int32_t* err,
                              cudaStream_t st);

// ---- tcgen05 kernels (bf16, DeepSeek-V3 dimensions) ------------------------------------------
size_t decode_tc_workspace(int B);
size_t decode_pair_workspace(int B);
cudaError_t decode_pair_launch(const DecodeArgs& a, void* ws, cudaStream_t st);
cudaError_t decode_tc_launch(const DecodeArgs& a, void* ws, cudaStream_t st);
cudaError_t absorb_q_tc_launch(int B, const void* q_nope, int64_t ldq, const void* w, void* q_tilde, cudaStream_t st);
cudaError_t out_up_tc_launch(int B, const void* ctx, const void* w, void* out, cudaStream_t st);
cudaError_t absorb_q_fp8_tc_launch(int B, const void* q_nope, int64_t ldq, const void* w_fp8, const float* scale,
                                   void* q_tilde, int32_t* err, cudaStream_t st);
cudaError_t out_up_fp8_tc_launch(int B, const void* ctx, const void* w_fp8, const float* scale, void* out,
                                 int32_t* err, cudaStream_t st);
cudaError_t expand_tc_launch(const PrefillArgs& a, cudaStream_t st);
cudaError_t attn_tc_launch(const PrefillArgs& a, cudaStream_t st);
size_t sparse_prefill_scratch_bytes(int B, int S);
cudaError_t sparse_masks_launch(const PrefillArgs& a, const int32_t* topk, int k, void* scratch, int32_t* err,
                                cudaStream_t st);
cudaError_t attn_sparse_tc_launch(const PrefillArgs& a, const void* scratch, int32_t* err, cudaStream_t st);
template <typename T>
cudaError_t prefill_attn_simt_launch(const PrefillArgs& a, cudaStream_t st);
size_t decode_static_scratch_bytes();
cudaError_t decode_static_scratch(void** out);
size_t decode_simt_workspace(int n_h, int d_c, int B, int n_keys_cap);

}  // namespace mla

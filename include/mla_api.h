/*
 * mla_api.h - C ABI of libmla_b200.so: multi-head latent attention (MLA) for NVIDIA B200 (sm_100a).
 *
 * The operations are the steps of DeepSeek-V3 / V3.2 MLA as the pages state them:
 *   mla_absorb_q       q~_i = (W^UK_i)^T q^C_i                       ("Absorb key weights", first einsum)
 *   mla_decode_absorb  softmax over cached positions of
 *                      scale (q~ . c^KV_t + q^R . k^R_t), weighted sum of c^KV_t
 *                                                                    ("Absorb key weights", decode excerpt)
 *   mla_out_up         o_i = W^UV_i ctx_i                            ("Absorb key weights", last einsum)
 *   mla_prefill_naive  wkv_b expansion, k = [k_nope; k^R], causal attention
 *                                                                    ("Value up-projection", prefill excerpt;
 *                                                                     "KV Reconstruction", "Naive path")
 *   mla_cache_append   the new token's latent (RMSNorm) and rotary key (RoPE) into the caches
 *                                                                    ("Key-value down-projection", mla-kv
 *                                                                     excerpt; "Key-value latent RMSNorm")
 *   mla_prefill_sparse the V3.2 prefill: each query row attends its top-k positions t <= s
 *                                                                    ("Value up-projection", MHA-prefill excerpt)
 *   mla_absorb_q_fp8, mla_out_up_fp8  the projections with an FP8 wkv_b and its 128 x 128 block scales
 *                                                                    ("Key-value down-projection", linear excerpt)
 * plus one opt-in check of the sparse decode's precondition:
 *   mla_check_topk     top-k indices in range and distinct per sequence (the mask is a set)
 *
 * Conventions shared by every call
 * --------------------------------
 * - Every data pointer is a DEVICE pointer owned by the caller; the library allocates nothing,
 *   keeps no pointer after a call returns and never synchronises the stream (except the two
 *   calls documented as blocking).  `stream` is a cudaStream_t (NULL = legacy default stream).
 * - Element type: MLA_BF16 (bf16 storage, fp32 accumulation) or MLA_F32 (fp32 throughout,
 *   no TF32).  Integer tensors are int32.  Strides are in ELEMENTS.
 * - W_kv_b is the fused up-projection ("KV Reconstruction", "How it works" and "Official code"):
 *   row-major [n_h * (d_h + d_v), d_c]; rows [i(d_h+d_v), i(d_h+d_v)+d_h) of head i are W^UK_i,
 *   the next d_v rows are W^UV_i ("Value up-projection", "Explanation").
 * - MLA_BF16 runs the tcgen05 tensor-core kernels, specialised for the DeepSeek-V3 dimensions
 *   n_h=128, d_c=512, d_r=64, d_h=d_v=128; other bf16 dimensions return MLA_ERR_UNSUPPORTED.
 *   bf16 pointers must be 16-byte aligned and row strides multiples of 8 elements.
 *   MLA_F32 accepts any dimensions with n_h <= 1024, d_c <= 1024, d_r <= 128, d_h, d_v <= 256.
 * - Host-checkable errors (NULL pointer, bad size, alignment, workspace too small) return at
 *   once and launch nothing.  Data-dependent errors found by a kernel (a length outside
 *   [1, n_max], a top-k index outside [0, length)) are written to the optional device flag
 *   `dev_err` (first error wins) and the offending row is skipped; kernels never trap.
 */
#ifndef MLA_API_H
#define MLA_API_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define MLA_ABI_VERSION 1

typedef enum {
  MLA_OK = 0,
  MLA_ERR_INVALID_ARG = 1,  /* NULL pointer, non-positive size, misaligned pointer or stride  */
  MLA_ERR_UNSUPPORTED = 2,  /* dimensions / dtype combination without a kernel               */
  MLA_ERR_CUDA = 3,         /* a CUDA runtime call failed (see mla_last_error_message)       */
  MLA_ERR_INDEX = 4,        /* device flag: a top-k index outside [0, length), or an append
                               position outside [0, n_max)                                    */
  MLA_ERR_TIMEOUT = 5,      /* device flag: a bounded wait inside a kernel ran out           */
  MLA_ERR_WORKSPACE = 6,    /* workspace NULL or smaller than the matching *_workspace_size  */
  MLA_ERR_LENGTH = 7        /* device flag: a sequence length outside [1, n_max]             */
} mla_status;

typedef enum { MLA_F32 = 0, MLA_BF16 = 1 } mla_dtype;

/* Head count and widths ("Key-value latent", MLA-init excerpt): n_h heads, latent d_c
 * (kv_lora_rank), rotary width d_r (qk_rope_head_dim), content key width d_h
 * (qk_nope_head_dim), value width d_v (v_head_dim).  DeepSeek-V3: {128, 512, 64, 128, 128}. */
typedef struct {
  int32_t n_h, d_c, d_r, d_h, d_v;
} mla_dims;

/* ABI version of the loaded library (MLA_ABI_VERSION when the header matches). */
int32_t mla_abi_version(void);

/* Static text for a status code; never NULL. */
const char* mla_status_string(mla_status s);

/* Details of the last host-side error raised on the calling thread ("" if none). */
const char* mla_last_error_message(void);

/*
 * mla_absorb_q - fold W^UK into each head's content query ("Absorb key weights": 128 content
 * features become 512 latent features; "KV Reconstruction", "Absorb path").
 *   q_nope   [B, n_h, d_h], element (b,h,d) at q_nope[(b*n_h + h)*ldq + d]   (ldq >= d_h)
 *   w_kv_b   [n_h*(d_h+d_v), d_c] row-major (only the W^UK rows are read)
 *   q_tilde  [B, n_h, d_c] contiguous output, q_tilde[b,h,c] = sum_d q_nope[b,h,d] W^UK_h[d,c]
 * Asynchronous on `stream`.
 */
mla_status mla_absorb_q(mla_dims dims, mla_dtype dtype, int32_t B,
                        const void* q_nope, int64_t ldq, const void* w_kv_b,
                        void* q_tilde, void* stream);

/*
 * mla_decode_workspace_size - bytes of scratch mla_decode_absorb needs for this shape on the
 * current device (split-KV partial results and the split plan).  An upper bound for any
 * lengths <= n_max; 0 never means "no workspace needed" for B > 0.
 */
size_t mla_decode_workspace_size(mla_dims dims, mla_dtype dtype, int32_t B, int32_t n_max, int32_t topk);

/*
 * mla_decode_num_launches - how many kernels one mla_decode_absorb call with these sizes
 * launches on the current device: 1 for bf16 (partials merged inside the kernel); for fp32 the
 * split-KV plan decides whether a combine pass runs.  (A bf16 top-k call over a cache whose batch
 * stride is not n_max rows runs the CUDA-core path, which this count does not cover.)
 * 0 for arguments mla_decode_absorb would reject.
 */
int32_t mla_decode_num_launches(mla_dims dims, mla_dtype dtype, int32_t B, int32_t n_max, int32_t topk);

/*
 * mla_decode_absorb - attention of one query token per sequence over its latent cache
 * ("Absorb key weights", decode excerpt; "KV Reconstruction", "Absorb path").
 *   For sequence b with length L_b = lengths[b] and every head h:
 *     s_t   = scale * (q_tilde[b,h,:] . c_kv[b,t,:] + q_pe[b,h,:] . k_r[b,t,:])
 *     kept positions: t in [0, L_b), or, when topk_idx != NULL, the set {topk_idx[b, j]} (the
 *     -inf scatter mask of the V3.2 sparse variant; indices must be distinct, in [0, L_b))
 *     ctx[b,h,:] = sum_t softmax(s)_t c_kv[b,t,:],   lse[b,h] = log sum_t exp(s_t)
 *   q_tilde  [B, n_h, d_c], element (b,h,c) at q_tilde[(b*n_h + h)*ldqt + c]
 *   q_pe     [B, n_h, d_r], element (b,h,r) at q_pe[(b*n_h + h)*ldqp + r]
 *   c_kv     row t of sequence b at c_kv + b*ckv_bstride + t*ckv_rstride (d_c elements)
 *   k_r      row t of sequence b at k_r + b*kr_bstride + t*kr_rstride (d_r elements)
 *            (a packed [B, n_max, d_c + d_r] cache is c_kv = base, k_r = base + d_c, both
 *             row strides d_c + d_r)
 *   n_max    cache capacity per sequence; lengths (device, int32 [B]) must lie in [1, n_max]
 *   topk_idx NULL (dense) or device int32 [B, topk]; 1 <= topk <= n_max
 *   scale    softmax scale, (d_h + d_r)^-0.5 for DeepSeek ("Key-value latent", MLA-init)
 *   ctx_out  [B, n_h, d_c] contiguous, dtype as the inputs
 *   lse_out  NULL or float [B, n_h] (natural log)
 *   workspace/ws_bytes  device scratch of at least mla_decode_workspace_size() bytes; its
 *            contents need no initialisation and are garbage afterwards
 *   dev_err  NULL or a device int32 flag; MLA_ERR_LENGTH / MLA_ERR_INDEX are stored there
 * Asynchronous on `stream`.
 * Accuracy (bf16): the two CTAs of a pair each compute half of every score (288 of the 576
 *   features, before the scale) and exchange it as fp16: a half-score beyond +-65504 saturates, and
 *   each is rounded to 2^-11 of its magnitude, an error of about |half-score| * scale * 2^-11 in the
 *   exponent of its softmax weight.  At DeepSeek magnitudes (RMS-normalised latent rows, scores of
 *   a few tens) that is ~1e-3 relative, inside bf16; half-scores of several hundred exceed it.
 *   The fp32 path and mla_decode_absorb_multi keep the scores in fp32.
 * Residency: the kernel is one persistent wave of CTA pairs sized by the occupancy query.  When a
 *   sequence is split into more than two pieces, every cluster holding a piece waits for all the
 *   others (the sliced merge), which needs every cluster resident at once.  The launcher uses that
 *   merge only when the occupancy query confirmed the wave; setting MLA_DECODE_SLICED_MERGE=0 in
 *   the environment turns it off (for GPUs shared with MPS clients or other processes' persistent
 *   kernels).  Without it the last piece to finish merges all the others.  A wait that runs out
 *   (SMs held by another context for longer than the limit) stores MLA_ERR_TIMEOUT in dev_err.
 */
mla_status mla_decode_absorb(mla_dims dims, mla_dtype dtype, int32_t B,
                             const void* q_tilde, int64_t ldqt, const void* q_pe, int64_t ldqp,
                             const void* c_kv, int64_t ckv_bstride, int64_t ckv_rstride,
                             const void* k_r, int64_t kr_bstride, int64_t kr_rstride,
                             int32_t n_max, const int32_t* lengths,
                             const int32_t* topk_idx, int32_t topk,
                             float scale, void* ctx_out, float* lse_out,
                             void* workspace, size_t ws_bytes, int32_t* dev_err, void* stream);

/*
 * mla_decode_absorb_fp8kv - mla_decode_absorb over an FP8 latent cache (dense, one token per
 * sequence).  The latent rows are stored as FP8 E4M3 codes with one fp32 scale per 128 latent
 * features of each row (the 128-wide blocks of the FP8 weights, "Key-value down-projection",
 * linear excerpt, applied per cached token: a reading, the pages keep the cache in bf16); the
 * rotary key stays bf16.  The kernel dequantises on chip, c_kv[t, f] = bf16(float(e4m3(c8[t, f])) *
 * kv_scale[t, f / 128]) with one fp32 product and one round-to-nearest-even, and then computes
 * exactly what mla_decode_absorb computes on that bf16 cache (bit-identical results).
 *   c8        row t of sequence b: d_c codes at (uint8*)c8 + b*c8_bstride + t*c8_rstride (BYTES;
 *             both multiples of 16)
 *   kv_scale  row t of sequence b: d_c / 128 floats at kv_scale + b*sc_bstride + t*sc_rstride
 *             (FLOATS; both multiples of 4)
 *   k_r       bf16 rotary rows as in mla_decode_absorb
 *   A packed 656-byte row [512 codes | 4 scales | 64 bf16 rotary features] is c8 = base,
 *   kv_scale = base + 512, k_r = base + 528, row strides 656, 164 and 328.
 *   Other arguments as in mla_decode_absorb (bf16 DeepSeek dimensions only; workspace as
 *   mla_decode_workspace_size(dims, MLA_BF16, B, n_max, 0)).  Asynchronous on `stream`.
 */
mla_status mla_decode_absorb_fp8kv(mla_dims dims, int32_t B, const void* q_tilde, int64_t ldqt, const void* q_pe,
                                   int64_t ldqp, const void* c8, int64_t c8_bstride, int64_t c8_rstride,
                                   const float* kv_scale, int64_t sc_bstride, int64_t sc_rstride, const void* k_r,
                                   int64_t kr_bstride, int64_t kr_rstride, int32_t n_max, const int32_t* lengths,
                                   float scale, void* ctx_out, float* lse_out, void* workspace, size_t ws_bytes,
                                   int32_t* dev_err, void* stream);

/*
 * mla_decode_absorb_multi - mla_decode_absorb for T new tokens per sequence ("DeepSeek-V3.2-Exp -
 * Absorb key weights", decode excerpt: the queries are [batch, s, heads, features] with s = T, e.g.
 * speculative tokens).  The T tokens of sequence b are the last T of its lengths[b] cached rows;
 * token s (0-based) attends rows t <= lengths[b] - T + s, the causal rule of the prefill excerpt
 * ("Value up-projection", MHA-prefill excerpt), so T = 1 is mla_decode_absorb.
 *   q_tilde, q_pe, ctx_out, lse_out  [B * T, n_h, .] with row (b * T + s, h), strides as in
 *                                    mla_decode_absorb (query rows (b * T + s) * n_h + h)
 *   c_kv, k_r                        [B, n_max, .] caches as in mla_decode_absorb
 *   lengths                          DEVICE int32 [B], each in [T, n_max]; a shorter or longer one
 *                                    sets MLA_ERR_LENGTH in dev_err and its tokens get ctx = 0,
 *                                    lse = -inf
 *   workspace                        mla_decode_workspace_size(dims, dtype, B * T, n_max, 0) bytes
 * bf16 DeepSeek dimensions only; a top-k set per token is mla_decode_absorb_multi_topk.  Each token
 * runs as its own query group over the shared cache rows of its sequence.  Asynchronous on `stream`.
 * Residency and MLA_DECODE_SLICED_MERGE as for mla_decode_absorb.
 */
mla_status mla_decode_absorb_multi(mla_dims dims, mla_dtype dtype, int32_t B, int32_t T,
                                   const void* q_tilde, int64_t ldqt, const void* q_pe, int64_t ldqp,
                                   const void* c_kv, int64_t ckv_bstride, int64_t ckv_rstride,
                                   const void* k_r, int64_t kr_bstride, int64_t kr_rstride,
                                   int32_t n_max, const int32_t* lengths, float scale, void* ctx_out,
                                   float* lse_out, void* workspace, size_t ws_bytes, int32_t* dev_err,
                                   void* stream);

/*
 * mla_decode_absorb_multi_topk - mla_decode_absorb_multi with a top-k set per new token (the V3.2
 * decode excerpt's index mask, one set per query as in the sparse prefill, "Value up-projection",
 * MHA-prefill excerpt, `index_mask += mask`): token s of sequence b attends the positions of its
 * set that the causal rule keeps, t <= lengths[b] - T + s; later positions in a set are removed by
 * that rule, not flagged.
 *   topk_idx  DEVICE int32 [B, T, topk] contiguous (row b * T + s is token s of sequence b);
 *             1 <= topk <= n_max; indices distinct per row (the set precondition of the gather
 *             decode); an index outside [0, lengths[b]) sets MLA_ERR_INDEX and is skipped
 *   lengths   DEVICE int32 [B] in [T, n_max]; another length sets MLA_ERR_LENGTH and the
 *             sequence's tokens get ctx = 0, lse = -inf
 *   workspace mla_decode_workspace_size(dims, dtype, B * T, n_max, topk) bytes
 *   Other arguments as in mla_decode_absorb_multi; bf16 (DeepSeek dimensions) or fp32.  T = 1 is
 *   mla_decode_absorb with topk_idx.  B * T <= 65535.
 * For T > 1 the CUDA-core kernel runs (one warp per head and query, split over the set, with a
 * merge pass when split): a query that selects no visible row gets ctx = 0 and lse = -inf.
 * Asynchronous on `stream`.
 */
mla_status mla_decode_absorb_multi_topk(mla_dims dims, mla_dtype dtype, int32_t B, int32_t T,
                                        const void* q_tilde, int64_t ldqt, const void* q_pe, int64_t ldqp,
                                        const void* c_kv, int64_t ckv_bstride, int64_t ckv_rstride,
                                        const void* k_r, int64_t kr_bstride, int64_t kr_rstride,
                                        int32_t n_max, const int32_t* lengths, const int32_t* topk_idx,
                                        int32_t topk, float scale, void* ctx_out, float* lse_out,
                                        void* workspace, size_t ws_bytes, int32_t* dev_err, void* stream);

/*
 * mla_decode_absorb_static - mla_decode_absorb for the bf16 dense decode (no top-k) WITHOUT a
 * caller-supplied workspace.  The pages have no counterpart: this is a deployment convenience.
 *   For callers that cannot allocate device memory around a decode call: a plugin or engine host
 *   whose enqueue path may not call cudaMalloc (an allocation there can synchronise the device or
 *   break the host's own memory budget), or a caller that only holds pointers handed to it by
 *   someone else and owns no allocator.  The split-KV scratch is
 *   a file-scope device array of 19,769,920 bytes (about 18.9 MiB: 74 clusters x 2 bf16 partial
 *   slots), held by every GPU that loads the library until the process exits.
 *   Arguments and results are those of mla_decode_absorb with topk_idx = NULL and without
 *   workspace / ws_bytes.  dtype must be MLA_BF16 (else MLA_ERR_UNSUPPORTED); a device that would
 *   need more scratch than the array holds (more than 148 SMs) gets MLA_ERR_WORKSPACE.
 *   The first call on a device looks up the array's device address (cudaGetSymbolAddress, with
 *   that device current) and caches it; make that first call before any stream capture begins.
 *   Every call shares the one array and it keeps the last call's contents; nothing in it needs to
 *   start at zero (each byte a call reads was written earlier in the same call, and its arrival
 *   counters and partial-ready flags carry a per-launch tag), but calls whose
 *   work overlaps on the GPU (different streams, or different host threads) race on it: serialise
 *   them.  No allocation of any kind happens inside this call.  Asynchronous on `stream`.
 */
mla_status mla_decode_absorb_static(mla_dims dims, mla_dtype dtype, int32_t B,
                                    const void* q_tilde, int64_t ldqt, const void* q_pe, int64_t ldqp,
                                    const void* c_kv, int64_t ckv_bstride, int64_t ckv_rstride,
                                    const void* k_r, int64_t kr_bstride, int64_t kr_rstride,
                                    int32_t n_max, const int32_t* lengths, float scale,
                                    void* ctx_out, float* lse_out, int32_t* dev_err, void* stream);

/*
 * mla_out_up - map the latent context back up through W^UV ("Absorb key weights", last einsum;
 * "KV Reconstruction", "Absorb path": W^UV applied after the weighted sum).
 *   ctx  [B, n_h, d_c] contiguous;  out [B, n_h, d_v] contiguous,
 *   out[b,h,d] = sum_c ctx[b,h,c] W^UV_h[d,c]   (only the W^UV rows of w_kv_b are read)
 * Asynchronous on `stream`.
 */
mla_status mla_out_up(mla_dims dims, mla_dtype dtype, int32_t B,
                      const void* ctx, const void* w_kv_b, void* out, void* stream);

/*
 * mla_absorb_q_fp8 / mla_out_up_fp8 - mla_absorb_q and mla_out_up with an FP8 wkv_b ("Key-value
 * down-projection", linear excerpt: an FP8 weight carries one float32 scale per 128 x 128 block;
 * the decode uses the dequantised matrix, "Value up-projection").
 *   w_fp8    e4m3 [n_h*(d_h+d_v), d_c] row-major, 16-byte aligned
 *   w_scale  DEVICE fp32 [ceil(n_h*(d_h+d_v)/128), ceil(d_c/128)] row-major: the weight is
 *            w[i, j] = w_fp8[i, j] * w_scale[i / 128, j / 128]
 *   The weight is read as FP8 and dequantised on chip to bf16 (each value times its block's scale,
 *   rounded to nearest), so the result equals mla_absorb_q / mla_out_up given that bf16 weight.
 *   bf16 activations and outputs, DeepSeek dimensions only.  Asynchronous on `stream`.
 */
mla_status mla_absorb_q_fp8(mla_dims dims, int32_t B, const void* q_nope, int64_t ldq, const void* w_fp8,
                            const float* w_scale, void* q_tilde, int32_t* dev_err, void* stream);
mla_status mla_out_up_fp8(mla_dims dims, int32_t B, const void* ctx, const void* w_fp8, const float* w_scale,
                          void* out, int32_t* dev_err, void* stream);

/*
 * mla_prefill_workspace_size - bytes of scratch mla_prefill_naive needs: the expanded
 * [B, S, n_h, d_h + d_v] keys/values in the input dtype.
 */
size_t mla_prefill_workspace_size(mla_dims dims, mla_dtype dtype, int32_t B, int32_t S);

/*
 * mla_prefill_naive - the naive path over a whole sequence ("Value up-projection", prefill
 * excerpt; "KV Reconstruction", "Naive path"):
 *   kv[b,s,h,:] = W_kv_b c_kv[b,s,:]  viewed as [d_h | d_v] -> k_nope, v
 *   k[b,t,h,:]  = [k_nope[b,t,h,:]; k_r[b,t,:]]        (k_r shared by all heads)
 *   out[b,s,h,:] = sum_t softmax_t(scale q[b,s,h,:] . k[b,t,h,:] + mask) v[b,t,h,:]
 *   mask: causal != 0 keeps t <= s (the additive causal mask); causal == 0 keeps every t.
 *   q     [B, S, n_h, d_h + d_r] contiguous (content part first, rotary part last)
 *   c_kv  row s of sequence b at c_kv + (b*S + s)*ckv_rstride;  k_r likewise with kr_rstride
 *   out   [B, S, n_h, d_v] contiguous
 *   workspace/ws_bytes  at least mla_prefill_workspace_size() bytes (holds the expansion)
 * Asynchronous on `stream`.
 */
mla_status mla_prefill_naive(mla_dims dims, mla_dtype dtype, int32_t B, int32_t S,
                             const void* q, const void* c_kv, int64_t ckv_rstride,
                             const void* k_r, int64_t kr_rstride, const void* w_kv_b,
                             float scale, int32_t causal, void* out,
                             void* workspace, size_t ws_bytes, void* stream);

/*
 * mla_cache_append - write one new token per sequence into the latent and rotary caches, the
 * step that precedes the decode ("Key-value down-projection", mla-kv excerpt: the joint
 * down-projection is split into the latent and the rotary key, the latent goes through kv_norm
 * and the key through the rotary embedding; "Key-value latent RMSNorm": fp32, one gain per
 * feature, eps inside the square root).  The pages do not show the cache write or the rotary
 * convention; the reading taken here is the decode's: row t of both caches holds position t.
 *   kv_a       new rows, element (b, j) at kv_a[b*lda + j]; j < d_c latent, d_c <= j < d_c+d_r rotary
 *   gain       DEVICE fp32 [d_c] RMSNorm gain, or NULL for ones
 *   positions  DEVICE int32 [B]: position p_b of each new token = the cache row it is written to
 *   c_kv       c_kv[b*ckv_bstride + p_b*ckv_rstride + c] = gain[c] * x_c / sqrt(mean_c(x_c^2) + eps),
 *              x = kv_a[b, 0:d_c] in fp32
 *   k_r        pair i of k_r[b*kr_bstride + p_b*kr_rstride + :] = (y[2i] + j y[2i+1]) exp(j p_b base^(-2i/d_r)),
 *              y = kv_a[b, d_c:d_c+d_r]: interleaved pairs, base = rope_base (10000 in DeepSeek-V3)
 *   Every other cache row is left as it was.  d_r must be even; eps >= 0; rope_base > 0.
 *   Device flag: a position outside [0, n_max) sets MLA_ERR_INDEX and that sequence writes nothing.
 * Asynchronous on `stream`.
 */
mla_status mla_cache_append(mla_dims dims, mla_dtype dtype, int32_t B,
                            const void* kv_a, int64_t lda, const float* gain, float eps, float rope_base,
                            const int32_t* positions, int32_t n_max,
                            void* c_kv, int64_t ckv_bstride, int64_t ckv_rstride,
                            void* k_r, int64_t kr_bstride, int64_t kr_rstride,
                            int32_t* dev_err, void* stream);

/*
 * mla_check_topk - opt-in validation of a top-k index array before a sparse decode.  The pages'
 * mask ("Absorb key weights", decode excerpt) scatters 0 into a -inf row, so the selected
 * positions form a set; the gather kernels read each listed row once, so distinct indices are
 * their precondition.  This call checks it on the device, per sequence b:
 *   topk_idx  DEVICE int32 [B, topk] contiguous
 *   lengths   DEVICE int32 [B], or NULL for n_max everywhere
 *   an index outside [0, lengths[b]) or listed twice in its row sets MLA_ERR_INDEX; a length
 *   outside [1, n_max] sets MLA_ERR_LENGTH.  Nothing else is written.
 *   n_max up to 1,859,584 (a bitmap of the positions in shared memory); larger returns
 *   MLA_ERR_UNSUPPORTED.
 * Asynchronous on `stream`; read the flag with mla_get_device_error.
 */
mla_status mla_check_topk(int32_t B, const int32_t* topk_idx, int32_t topk, const int32_t* lengths, int32_t n_max,
                          int32_t* dev_err, void* stream);

/*
 * mla_prefill_sparse_workspace_size - bytes of scratch mla_prefill_sparse needs: the expansion of
 * mla_prefill_workspace_size plus the per-row selection bitmaps and per-query-tile key-tile lists.
 */
size_t mla_prefill_sparse_workspace_size(mla_dims dims, mla_dtype dtype, int32_t B, int32_t S);

/*
 * mla_prefill_sparse - the V3.2 sparse prefill ("Value up-projection", MHA-prefill excerpt: a -inf
 * row with 0 scattered at each query row's top-k positions, plus the causal mask, added to the
 * scores): as mla_prefill_naive with causal = 1, except that query row s attends only the
 * positions t <= s listed in its row of topk_idx (a set: repeats count once).
 *   topk_idx  DEVICE int32 [B, S, topk] contiguous; an index outside [0, S) sets MLA_ERR_INDEX and
 *             is ignored; indices past the row (t > s) are removed by the causal mask
 *   a row whose set holds no t <= s has no softmax: it is written as zeros and MLA_ERR_INDEX is set
 *   bf16 DeepSeek dimensions only (MLA_ERR_UNSUPPORTED otherwise).
 * Asynchronous on `stream`.
 */
mla_status mla_prefill_sparse(mla_dims dims, mla_dtype dtype, int32_t B, int32_t S,
                              const void* q, const void* c_kv, int64_t ckv_rstride,
                              const void* k_r, int64_t kr_rstride, const void* w_kv_b,
                              float scale, const int32_t* topk_idx, int32_t topk, void* out,
                              void* workspace, size_t ws_bytes, int32_t* dev_err, void* stream);

/*
 * mla_selftest_wait_timeout - failure detection without a fault: one CTA waits on an mbarrier that
 * nothing arrives on, with the bounded wait every kernel of the library uses; after limit_ns
 * (1 us .. 1 s) of global time it gives up and sets MLA_ERR_TIMEOUT in dev_err.  The context stays
 * usable.  Asynchronous on `stream`.
 */
mla_status mla_selftest_wait_timeout(uint64_t limit_ns, int32_t* dev_err, void* stream);

/* Zero the device flag (asynchronous on `stream`). */
mla_status mla_clear_device_error(int32_t* dev_err, void* stream);

/* BLOCKING: wait for all work on the current device, then copy the device flag to *host_out. */
mla_status mla_get_device_error(const int32_t* dev_err, int32_t* host_out);

#ifdef __cplusplus
}
#endif

#endif /* MLA_API_H */

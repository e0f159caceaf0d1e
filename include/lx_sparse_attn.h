/*
 * lx_sparse_attn.h -- dynamic block-sparse, low-precision self-attention for
 * long-sequence video DiTs, for NVIDIA B200 (sm_100a).
 *
 * What it computes (the method LightX2V calls Dynamic Sparse SageAttention):
 *  - "600倍加速，720p视频实时生成！单卡也能带的动14B模型", §动态稀疏量化注意力:
 *    the importance of attention tiles is estimated from block-level means of
 *    Q and K, key blocks are chosen at run time, only the activated tiles are
 *    computed and a chosen block stays dense inside (typical sparsity 80-90%).
 *  - same page, §高效推理算子: about 10% of the blocks are kept and the
 *    arithmetic is Q/K INT8 with V FP8.
 *  - "Run Wan2.2-A14B on One RTX 5090: 720p Video in 3.8s", §3 Dynamic sparse
 *    attention: the same in English (top 10-20% of blocks, dense inside).
 * The pages fix no block size, score, selection rule or scale granularity;
 * this library's fixed reading is: 64-token blocks (nB = ceil(L/64), the last
 * block may be partial), score s[i][j] = mean(Q_i) . mean(K_j) / sqrt(D),
 * keep k = clamp(ceil(keep*nB - 1e-6), 1, nB) key blocks per query block with
 * ties to the lower index, INT8 Q/K with one absmax/127 scale per (b,h,block),
 * FP8 E4M3 V with one absmax/448 scale per (b,h,channel), and in INT8/FP8
 * mode P quantised to E4M3 (scale 448) against the running row max, one
 * 64-key block at a time in ascending key-block order.
 *
 * Conventions for every entry point:
 *  - All tensors are device memory owned by the caller; the library allocates
 *    no memory and keeps no state besides one status word per device.
 *  - Q, K, V, O are bf16 [B,H,L,D] with element strides sB, sH, sL (the stride
 *    of D is 1); D is 64 or 128; base pointers and every stride in bytes must
 *    be multiples of 16.
 *  - Argument errors are detected on the host before any launch and return a
 *    negative status; nothing is launched then.  Launches are asynchronous on
 *    `stream`; a launch failure returns LX_ERR_CUDA.  Errors found on the device
 *    (a bounded wait that ran out, a malformed plan) are recorded in the status
 *    word and reported by lx_last_device_status().
 *  - Calls are stream-ordered and never synchronise, except
 *    lx_last_device_status().
 */
#ifndef LX_SPARSE_ATTN_H
#define LX_SPARSE_ATTN_H

#include <stddef.h>
#include <stdint.h>
#include <cuda_runtime_api.h>

#ifdef __cplusplus
extern "C" {
#endif

#define LX_BLOCK 64

typedef enum lx_status {
  LX_OK = 0,
  LX_ERR_INVALID = -1,     /* bad pointer, shape, stride or keep */
  LX_ERR_UNSUPPORTED = -2, /* D not in {64,128}, or nB beyond the planner limit */
  LX_ERR_ALIGN = -3,       /* a pointer or byte stride not a multiple of 16 */
  LX_ERR_WORKSPACE = -4,   /* workspace null or smaller than the size query says */
  LX_ERR_CUDA = -5,        /* a CUDA call or launch failed */
  LX_ERR_TIMEOUT = -6,     /* device: a bounded wait ran out (kernel gave up cleanly) */
  LX_ERR_PLAN = -7         /* device: a plan row not strictly ascending / out of range, or non-finite scores */
} lx_status;

typedef enum lx_mode { LX_MODE_BF16 = 0, LX_MODE_INT8FP8 = 1 } lx_mode;

/* A bf16 [B,H,L,D] tensor view; strides in elements, stride of D is 1. */
typedef struct lx_bhld {
  void* data;
  int64_t B, H, L, D;
  int64_t sB, sH, sL;
} lx_bhld;

/* A block plan.  idx: int32 [B,H,nB,k], each row the kept key-block ids in
 * strictly ascending order.  mask: uint32 [B,H,nB,ceil(nB/32)], bit (j%32) of
 * word j/32 set iff key block j is kept; may be NULL.  Plain caller-owned data:
 * a caller may build or edit a plan by hand. */
typedef struct lx_plan {
  int32_t* idx;
  uint32_t* mask;
  int64_t B, H, L, nB, k;
  int32_t block; /* always LX_BLOCK */
} lx_plan;

/* Sizes of a plan.  k = clamp(ceil(keep*nB - 1e-6), 1, nB) with nB = ceil(L/64);
 * idx_bytes / mask_bytes size the plan arrays; ws_bytes sizes the workspace of
 * lx_sparse_attn_plan: two fp32 [B,H,nB,D] block-mean arrays followed by the
 * fp32 [B,H,nB,ldS] score matrix (ldS = nB rounded up to a multiple of 32), each
 * rounded up to 256 bytes.
 * keep must lie in (0, 1].  Any output pointer may be NULL. */
lx_status lx_plan_size(int64_t B, int64_t H, int64_t L, int64_t D, double keep, int64_t* k, size_t* idx_bytes,
                       size_t* mask_bytes, size_t* ws_bytes);

/* Step a1 -- block means ("600倍加速…", §动态稀疏量化注意力: "块级均值").
 * mq, mk: fp32 [B,H,nB,D] contiguous outputs, mean over the valid tokens of
 * each 64-token block (the last block divides by its own token count). */
lx_status lx_pool_means(const lx_bhld* Q, const lx_bhld* K, float* mq, float* mk, cudaStream_t stream);

/* Step a2 -- score and select.  From the block means (layout as above) writes
 * plan->idx (and plan->mask when not NULL): per query block the k key blocks
 * with the largest mean(Q_i).mean(K_j)/sqrt(D), ties to the lower index,
 * ascending.  plan->idx/mask must be set by the caller; the call fills
 * plan->B, H, L, nB, k and block.  nB must not exceed 2176 (L <= 139264).
 * ws: scratch for the fp32 [B,H,nB,ldS] score matrix (ldS = nB rounded up to a
 * multiple of 32), at least 4*B*H*nB*ldS bytes (rounded up to 256), 16-byte
 * aligned (LX_ERR_WORKSPACE /
 * LX_ERR_ALIGN otherwise).  The scores are computed on the tensor cores in
 * three tf32 products (high.high + high.low + low.high of each fp32 mean), which
 * keeps them within about 1e-6 relative of the fp32 dot products. */
lx_status lx_score_topk(const float* mq, const float* mk, int64_t B, int64_t H, int64_t L, int64_t D, double keep,
                        lx_plan* plan, void* ws, size_t ws_bytes, cudaStream_t stream);

/* Steps a1 + a2 -- the planner.  ws: at least ws_bytes of lx_plan_size. */
lx_status lx_sparse_attn_plan(const lx_bhld* Q, const lx_bhld* K, double keep, lx_plan* plan, void* ws,
                              size_t ws_bytes, cudaStream_t stream);

/* Step a3 -- INT8 Q and K ("600倍加速…", §高效推理算子: "Q/K INT8").
 * qc, kc: int8 [B,H,L,D] contiguous codes; qs, ks: fp32 [B,H,nB] scales.
 * scale = absmax/127 over the block's valid tokens and all D channels (1 for
 * an all-zero block); code = clamp(rint_even(fl32(x * fl32(127/absmax))), +-127). */
lx_status lx_quantize_qk(const lx_bhld* Q, const lx_bhld* K, int8_t* qc, float* qs, int8_t* kc, float* ks,
                         cudaStream_t stream);

/* Steps a1 + a3 in one read of Q and K: the block means of lx_pool_means and
 * the codes and scales of lx_quantize_qk, bit-identical to those two calls
 * (all three run one kernel).  Arguments, layouts and errors as there; every
 * output pointer must be non-NULL and 16-byte aligned. */
lx_status lx_pool_quantize_qk(const lx_bhld* Q, const lx_bhld* K, float* mq, float* mk, int8_t* qc, float* qs,
                              int8_t* kc, float* ks, cudaStream_t stream);

/* Step f1 -- the fused Q/K prologue ("600倍加速…", §高效推理算子, last
 * paragraph: 3D RoPE and RMSNorm as fused kernels, fewer round trips through
 * memory).  The pages give no formula; this library's reading, per tensor:
 *   y = rope(x / sqrt(mean_c x_c^2 + eps) * w[h, c])
 * (RMSNorm over each head's D channels, weights fp32 [H, D]), where the
 * token at raster index n of the (T, Hh, W) grid (W fastest) has position
 * (t, h, w) = (n / (Hh W), (n / W) mod Hh, n mod W); the head dimension is cut
 * into the t, h and w parts of dt, dh and dw channels (even, in that order,
 * summing to D; the default reading is D - 4 floor(D/6), 2 floor(D/6),
 * 2 floor(D/6)), and pair i of a part of m channels turns by
 * pos * theta^(-2i/m): (a, b) -> (a cos - b sin, a sin + b cos).
 * The prologue's output is bf16(y); the block means and INT8 codes/scales are
 * those of that bf16 tensor, bit-identical to lx_pool_quantize_qk run on it. */
typedef struct lx_rope3d {
  int64_t T, Hh, W;   /* token grid; T*Hh*W >= L */
  int32_t dt, dh, dw; /* channels of the t, h and w parts */
  double theta;       /* base, > 0 (10000 in the default reading) */
} lx_rope3d;

/* Bytes of the (cos, sin) table of lx_rope3d_table: 8 * (T dt + Hh dh + W dw) / 2. */
lx_status lx_rope3d_table_size(const lx_rope3d* rope, int64_t D, size_t* bytes);

/* Fills `table` (device, 16-byte aligned) with fp32 (cos, sin) pairs, the
 * angles and their sine and cosine taken in fp64: the t part (T positions x
 * dt/2 pairs), then the h part, then the w part.  It depends on the grid and
 * D only, so one table serves every call of that shape. */
lx_status lx_rope3d_table(const lx_rope3d* rope, int64_t D, float* table, cudaStream_t stream);

/* The prologue of Q and K in one read of each.  wq, wk: fp32 [H, D]; table:
 * from lx_rope3d_table; eps >= 0.  Yq, Yk: bf16 outputs (both or neither may
 * be NULL), same shape as Q.  mq, mk: block means fp32 [B,H,nB,D] (required).
 * qc, qs, kc, ks: INT8 codes and scales as for lx_quantize_qk (all four or
 * none may be NULL).  L must not exceed T*Hh*W.  All pointers 16-byte
 * aligned. */
lx_status lx_qk_prologue(const lx_bhld* Q, const lx_bhld* K, const float* wq, const float* wk, float eps,
                         const lx_rope3d* rope, const float* table, const lx_bhld* Yq, const lx_bhld* Yk, float* mq,
                         float* mk, int8_t* qc, float* qs, int8_t* kc, float* ks, cudaStream_t stream);

/* K smoothing -- a variant, not on the pages (the SageAttention family, which
 * the pages name, subtracts K's mean before quantising).  Subtracting one
 * vector m from every key shifts each score row by the constant q.m, which the
 * softmax removes; quantising K - m shrinks the INT8 error when K has large
 * channel offsets.  Reading: m = the per-(b, h, channel) mean of K over all L
 * tokens, taken in fp64 and rounded to fp32 once.
 * lx_k_channel_mean: km fp32 [B,H,D]; ws: scratch of lx_k_channel_mean_ws_size
 * bytes (8 * B * H * ceil(L/512) * D), 16-byte aligned.  The sums run in a
 * fixed order, so km is reproducible bit for bit.
 * lx_quantize_qk_smooth: Q's codes as lx_quantize_qk; K's codes and scales are
 * those of fl32(K - km) by the same rule.  The attention takes them unchanged
 * (lx_attn_int8fp8). */
lx_status lx_k_channel_mean_ws_size(const lx_bhld* K, size_t* bytes);
lx_status lx_k_channel_mean(const lx_bhld* K, void* ws, size_t ws_bytes, float* km, cudaStream_t stream);
lx_status lx_quantize_qk_smooth(const lx_bhld* Q, const lx_bhld* K, const float* km, int8_t* qc, float* qs, int8_t* kc,
                                float* ks, cudaStream_t stream);
/* The same codes plus the block means of Q and K (of the unshifted K, which
 * rank the key blocks alike) in one read, as lx_pool_quantize_qk. */
lx_status lx_pool_quantize_qk_smooth(const lx_bhld* Q, const lx_bhld* K, const float* km, float* mq, float* mk,
                                     int8_t* qc, float* qs, int8_t* kc, float* ks, cudaStream_t stream);

/* Light-Ulysses exchange (multi-GPU sequence parallelism, "600倍加速…",
 * §多卡路径: the sequence is split over the GPUs and an all-to-all moves the
 * data between the sequence and head dimensions; FP8 payloads, Q/K/V fused in
 * one payload, the exchange run per head chunk).  Reading: rank r holds tokens
 * [r Lr, (r+1) Lr) of all H heads before the exchange, heads [r Hr, (r+1) Hr)
 * (Hr = H / N) of all L = N Lr tokens after it.  One FP8 scale per (token,
 * head, tensor) row of D values: s = absmax/448 (1 for an all-zero row), code
 * = E4M3_rn_satfinite(fl32(x * fl32(448/absmax))); the receiver writes
 * bf16(fl32(decode(code) * s)).  The collective itself is the caller's: one
 * all-to-all with equal splits over a payload of N segments; these calls
 * build and read the payload.
 *
 * Payload: N segments of seg bytes (lx_ulysses_segment_bytes), segment n for
 * (pack) or from (unpack) rank n.  A segment holds the codes, uint8
 * [B][hc][Lr][X][D] (X = 3 tensors q, k, v for the Q/K/V payload, X = 1 for
 * the output payload), then, from byte offset roundup16(B hc Lr X D), the
 * scales, fp32 [B][hc][Lr][X]; seg = that offset + roundup16(4 B hc Lr X).
 *
 * lx_ulysses_segment_bytes: seg for the given sizes (tensors = X = 3 or 1);
 * LX_ERR_INVALID for sizes below 1, D other than 64 or 128, or another X.
 * lx_ulysses_pack_qkv: q, k, v this rank's shard viewed as [B, H, Lr, D] (any
 * strides, e.g. the [B, Lr, H, D] layout); segment n carries heads
 * n Hr + h0 .. n Hr + h0 + hc - 1 of the shard.
 * lx_ulysses_unpack_qkv: the received Q/K/V payload (segment n from rank n,
 * hc = q's head count, Lr = L / N) into q, k, v [B, hc, L, D] (token n Lr + t
 * from rank n).
 * lx_ulysses_pack_o: the attention output o [B, hc, L, D] of those heads;
 * segment n holds rank n's tokens (Lr = L / N).
 * lx_ulysses_unpack_o: the received output payload into this rank's shard
 * out [B, H, Lr, D] (any strides), heads n Hr + h0 .. n Hr + h0 + hc - 1 from
 * segment n.  The payload pointer 16-byte aligned (LX_ERR_ALIGN otherwise);
 * shapes as stated (LX_ERR_INVALID otherwise); the payload is the caller's
 * device memory, N seg bytes. */
lx_status lx_ulysses_segment_bytes(int64_t B, int64_t hc, int64_t Lr, int64_t D, int64_t tensors, size_t* seg_bytes);
lx_status lx_ulysses_pack_qkv(const lx_bhld* q, const lx_bhld* k, const lx_bhld* v, int64_t N, int64_t h0, int64_t hc,
                              uint8_t* payload, cudaStream_t stream);
lx_status lx_ulysses_unpack_qkv(const uint8_t* payload, int64_t N, const lx_bhld* q, const lx_bhld* k,
                                const lx_bhld* v, cudaStream_t stream);
lx_status lx_ulysses_pack_o(const lx_bhld* o, int64_t N, uint8_t* payload, cudaStream_t stream);
lx_status lx_ulysses_unpack_o(const uint8_t* payload, int64_t N, int64_t h0, int64_t hc, const lx_bhld* out,
                              cudaStream_t stream);

/* Step a3 -- FP8 E4M3 V ("600倍加速…", §高效推理算子: "V FP8").
 * vc: uint8 [B,H,L,D] contiguous E4M3 codes; vs: fp32 [B,H,D] scales =
 * absmax over all L tokens / 448 (1 for an all-zero channel);
 * code = E4M3_rn_satfinite(fl32(v * fl32(448/absmax))).
 * amax_ws: caller scratch of B*H*D uint32 (zeroed by the call). */
lx_status lx_quantize_v(const lx_bhld* V, uint8_t* vc, float* vs, uint32_t* amax_ws, cudaStream_t stream);

/* Largest B*H*D that lx_quantize_v_noalloc accepts (its built-in scratch holds
 * this many uint32 words, 256 KiB per device). */
#define LX_NOALLOC_AMAX_MAX 65536

/* lx_quantize_v without a caller-supplied scratch buffer.  The paper has no
 * counterpart to this call: it exists for callers that cannot hand over device
 * scratch, e.g. plain C hosts without a device allocator of their own, where a
 * cudaMalloc/cudaFree pair per call would synchronise the device, or callers
 * whose device memory is fully budgeted up front.  It computes exactly what
 * lx_quantize_v computes (same codes and scales, bit for bit) and allocates
 * nothing.
 *
 * Scratch: a per-device array of LX_NOALLOC_AMAX_MAX uint32 words built into
 * this library.  The call zeroes the first B*H*D words on `stream` before use,
 * so nothing has to be cleared beforehand.  Because the array is shared, calls
 * that may overlap on the same device (two streams, two host threads without
 * ordering) race on it and may produce wrong scales; serialise them, or use
 * lx_quantize_v with a buffer per stream.
 *
 * First-call setup: the first call on each device looks up the array's device
 * address (cudaGetSymbolAddress, with that device current, guarded by a host
 * mutex) and caches it together with the device's current context; later
 * calls in the same context only read the cache.  After a cudaDeviceReset the
 * device has a new context, and the next call looks the address up again.
 * The lookup may load the library's device code, so make the first call on a
 * device (and the first after a reset) before any stream capture begins.
 *
 * Errors: LX_ERR_WORKSPACE when B*H*D > LX_NOALLOC_AMAX_MAX (nothing is
 * launched); LX_ERR_CUDA when the lookup fails; otherwise as lx_quantize_v. */
lx_status lx_quantize_v_noalloc(const lx_bhld* V, uint8_t* vc, float* vs, cudaStream_t stream);

/* Step a4 -- attention over the kept blocks in BF16 (tcgen05 kind::f16).
 * O[t] = sum_u softmax_u(q_t.k_u/sqrt(D)) v_u over the valid keys u of the
 * kept blocks of t's query block ("600倍加速…", §动态稀疏量化注意力). */
lx_status lx_attn_bf16(const lx_bhld* Q, const lx_bhld* K, const lx_bhld* V, const lx_plan* plan, const lx_bhld* O,
                       cudaStream_t stream);

/* Step a4 -- attention over the kept blocks from quantised operands
 * (tcgen05 kind::i8 for QK^T, kind::f8f6f4 for PV).  qc, kc, vc, qs, ks, vs as
 * written by lx_quantize_qk / lx_quantize_v for tensors of shape
 * [B,H,L,D] = O's shape.  P follows the E4M3 protocol stated at the top. */
lx_status lx_attn_int8fp8(const int8_t* qc, const float* qs, const int8_t* kc, const float* ks, const uint8_t* vc,
                          const float* vs, const lx_plan* plan, const lx_bhld* O, cudaStream_t stream);

/* Workspace of lx_sparse_attn_fwd: 0 for BF16; for INT8/FP8 the int8 Q/K codes,
 * E4M3 V codes, their scales and the V absmax scratch (each 256-byte aligned). */
lx_status lx_fwd_workspace_size(const lx_bhld* Q, lx_mode mode, size_t* bytes);

/* Steps a3 + a4: O = sparse attention of (Q, K, V) under `plan` in `mode`. */
lx_status lx_sparse_attn_fwd(const lx_bhld* Q, const lx_bhld* K, const lx_bhld* V, const lx_plan* plan, lx_mode mode,
                             const lx_bhld* O, void* ws, size_t ws_bytes, cudaStream_t stream);

/* Steps a1-a4 in one call: plan (written to *plan, whose idx/mask the caller
 * sets as for lx_score_topk) and forward.  INT8/FP8 mode reads Q and K once
 * for the block means and the INT8 codes (lx_pool_quantize_qk), so the result
 * equals lx_sparse_attn_plan followed by lx_sparse_attn_fwd bit for bit with
 * one pass over Q and K fewer.  ws: lx_sparse_attn_ws_size bytes, 256-byte
 * aligned (the planner's workspace, rounded to 256, then the forward's). */
lx_status lx_sparse_attn_ws_size(const lx_bhld* Q, double keep, lx_mode mode, size_t* bytes);
lx_status lx_sparse_attn(const lx_bhld* Q, const lx_bhld* K, const lx_bhld* V, double keep, lx_mode mode,
                         lx_plan* plan, const lx_bhld* O, void* ws, size_t ws_bytes, cudaStream_t stream);

/* ---------------------------------------------------------------- NVFP4
 * "Run Wan2.2-A14B on One RTX 5090: 720p Video in 3.8s", §2 (NVFP4
 * quantization-aware training): NVFP4 = E2M1 values, one E4M3 scale per 16
 * consecutive elements, one FP32 scale per tensor; the linear layers run a
 * block-scaled GEMM of NVFP4 activations by NVFP4 weights with FP32
 * accumulation, BF16 output and the column bias fused in the epilogue.
 *
 * Scale rule (this library's reading; the pages give only the format), in fp32:
 *   g   = amax / 2688 (1 for an all-zero tensor),  ig6 = 1 / (6 g)
 *   s   = E4M3_rn_satfinite(amax_block * ig6),  inv = 1 / (s g)  (0 when s = 0)
 *   code = E2M1_rn_satfinite(x * inv) (ties to even; a zero result is +0)
 * each product and reciprocal rounded to fp32 once.
 *
 * Layouts (device memory, dense):
 *   codes  uint8 [R][K/2]: element 2i in the low nibble of byte i of the row;
 *   scales uint8, tiled for the tensor core: rows padded to a multiple of 128
 *          (padding scales are 0); the E4M3 scale of row r, 16-element block j
 *          sits at byte (t*KS + ks)*512 + l*16 + c*4 + jj with t = r/128,
 *          l = r%32, c = (r%128)/32, ks = j/4, jj = j%4, KS = K/64.
 *   global scale: one fp32 in device memory. */

/* Bytes of the code and scale buffers of an [R, K] tensor (K % 64 == 0). */
lx_status lx_nvfp4_sizes(int64_t R, int64_t K, size_t* code_bytes, size_t* sf_bytes);

/* Quantise bf16 x [R, K] (row stride ldx elements, ldx % 8 == 0, K % 64 == 0,
 * 16-byte aligned) to NVFP4.  compute_gscale != 0: *gscale (device fp32) is
 * computed from x and written (an amax pass, then the quantiser); 0: *gscale
 * is read as given and must be a positive finite fp32.  codes / sf: buffers of lx_nvfp4_sizes bytes, 16-byte
 * aligned, owned by the caller.  Finite inputs only. */
lx_status lx_nvfp4_quantize(const void* x, int64_t R, int64_t K, int64_t ldx, int compute_gscale, float* gscale,
                            uint8_t* codes, uint8_t* sf, cudaStream_t stream);

/* Y[m, n] = bf16(fl32(acc[m, n] * fl32(gx * gw)) + bias[n]), acc = the fp32
 * tensor-core sum over k of x[m, k] w[n, k] (each the E2M1 value times its E4M3
 * block scale): X = (xc, xsf, gx) [M, K], W = (wc, wsf, gw) [N, K] as written by
 * lx_nvfp4_quantize; bias fp32 [N] or NULL; y bf16 [M, N] with row stride ldy
 * (ldy % 8 == 0, 16-byte aligned).  N % 128 == 0, K % 256 == 0; M is any
 * count >= 1; M and N below 2^31 - 256, K up to 2^30 (else LX_ERR_UNSUPPORTED).
 * One persistent CTA per SM walks the 128 x 256 output tiles.  A wait that
 * runs out sets the device status to LX_ERR_TIMEOUT (see lx_last_device_status). */
lx_status lx_nvfp4_gemm(const uint8_t* xc, const uint8_t* xsf, const float* gx, const uint8_t* wc,
                        const uint8_t* wsf, const float* gw, const float* bias, int64_t M, int64_t N, int64_t K,
                        void* y, int64_t ldy, cudaStream_t stream);

/* Synchronises `stream`, returns and clears the device status word of the
 * current device: LX_OK, LX_ERR_TIMEOUT, LX_ERR_PLAN, or LX_ERR_CUDA when the
 * stream itself reports an error. */
lx_status lx_last_device_status(cudaStream_t stream);

/* Launches one kernel that waits on a barrier nothing completes, giving up
 * after limit_ns; the failure path of every bounded wait, for tests. */
lx_status lx_debug_wait_timeout(uint64_t limit_ns, cudaStream_t stream);

const char* lx_status_string(lx_status status);

#ifdef __cplusplus
}
#endif
#endif /* LX_SPARSE_ATTN_H */

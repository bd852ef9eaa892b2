/*
 * attn.h -- C ABI of the B200 (sm_100a) exact attention library.
 *
 * The operation is exact scaled-dot-product attention (the forward pass, and
 * its gradients in attn_bwd):
 *
 *     O = softmax(scale * Q K^T + mask) V,     LSE = logsumexp(scale * Q K^T + mask)
 *
 * as stated in "Flash Attention in a production Stable-Diffusion service"
 * (xxmr.cn/news/81028), section 2.3 (QK^T, divide by sqrt(d_k), add attn_mask,
 * softmax over the last axis, multiply by V; dropout is zero at inference) and
 * computed tile by tile with an online softmax as in "FlashAttention technical
 * analysis" (jsqmd.com/news/722897), section 2.2.  The N x N score matrix never
 * reaches device memory; the only extra output is the per-row log-sum-exp that
 * a recomputing backward pass needs (same page, section 3.3).
 *
 * Conventions shared by every entry point:
 *   - Pointers named "device" must point to device memory of the current CUDA
 *     device; the library neither allocates, frees nor retains them.  Calls are
 *     asynchronous on the given stream: buffers must stay alive until the
 *     stream has passed the call.
 *   - `stream` is a cudaStream_t passed as void* (NULL = the legacy default stream).
 *   - Every function returns an attn_status_t and never prints, exits or traps.
 *     Host-side argument errors are reported synchronously; faults detected
 *     inside a kernel (an expired bounded wait) are recorded on the device and
 *     reported by attn_check_device_status().
 */
#ifndef ATTN_H_
#define ATTN_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum attn_status_t {
    ATTN_OK = 0,
    ATTN_ERR_INVALID_ARG = 1,  /* null pointer, non-positive size, Hq % Hkv != 0, bad scale ... */
    ATTN_ERR_UNSUPPORTED = 2,  /* head dim other than 64 / 128, or no sm_100 device */
    ATTN_ERR_ALIGNMENT = 3,    /* a tensor base is not 16-byte aligned */
    ATTN_ERR_CUDA = 4,         /* a CUDA runtime / driver call failed; see attn_last_cuda_error() */
    ATTN_ERR_TIMEOUT = 5,      /* a bounded wait inside a kernel expired (asynchronous) */
    ATTN_ERR_DEVICE = 6,       /* another device-side consistency check failed (asynchronous) */
    ATTN_ERR_SCRATCH = 7       /* attn_fwd_splitkv_noalloc: the call needs more than
                                  ATTN_NOALLOC_SCRATCH_BYTES of scratch */
} attn_status_t;

/*
 * attn_fwd -- exact attention forward pass.
 *
 * Layout ([batch, heads, seq, head_dim], the layout the Stable-Diffusion page,
 * section 3.1, passes to scaled_dot_product_attention), all contiguous:
 *   q    device bf16 [B, Hq,  Nq, d]
 *   k    device bf16 [B, Hkv, Nk, d]
 *   v    device bf16 [B, Hkv, Nk, d]
 *   out  device bf16 [B, Hq,  Nq, d]    (written; rounded to nearest even)
 *   lse  device fp32 [B, Hq,  Nq] or NULL (written: natural-log log-sum-exp of
 *        the scaled, masked scores of each query row; -inf for a row that has
 *        no unmasked key, whose output row is then 0)
 * Sizes: B, Hq, Hkv, Nq, Nk >= 1; Hq % Hkv == 0 (query head h reads K/V head
 * h / (Hq / Hkv)); d in {64, 128}.  Every base pointer 16-byte aligned.
 * scale: multiplies Q K^T; 0 selects 1/sqrt(d) (flash_attn_func's
 * softmax_scale=None on the ChatGLM2 page, jsqmd.com/news/348824); negative,
 * infinite or NaN scales are rejected.
 * is_causal: non-zero masks key j for query i when j > i (top-left alignment,
 * the convention of scaled_dot_product_attention's is_causal).
 * key_lens: device int32 [B] or NULL.  Keys j >= key_lens[b] of batch b are
 *   masked (padding); 0 <= key_lens[b] <= Nk is the caller's contract.
 * additive_mask: device fp32 or NULL, added to the scaled scores
 *   (s = scale * q.k + mask, the order of section 2.3 of the Stable-Diffusion
 *   page); -inf entries mask a key.  Element (b, h, i, j) is read at
 *   additive_mask[b*mask_strides[0] + h*mask_strides[1] + i*mask_strides[2] + j];
 *   a stride of 0 broadcasts that axis; mask_strides (host, 3 x int64) NULL
 *   means dense [B, Hq, Nq, Nk].  key_lens and additive_mask may not both be
 *   given.  Mask values must not be +inf or NaN.
 * Masked keys get probability exactly 0.  Q, K and V must be finite everywhere,
 * padding included (0 * inf is NaN inside the matrix units).
 * Errors: ATTN_ERR_INVALID_ARG, ATTN_ERR_UNSUPPORTED, ATTN_ERR_ALIGNMENT,
 * ATTN_ERR_CUDA (launch failure); kernel-side faults via attn_check_device_status.
 */
attn_status_t attn_fwd(const void *q, const void *k, const void *v, void *out, float *lse,
                       int B, int Hq, int Hkv, int Nq, int Nk, int d,
                       float scale, int is_causal,
                       const int32_t *key_lens,
                       const float *additive_mask, const int64_t *mask_strides,
                       void *stream);

/*
 * Score and mask variants for attn_fwd_mod.
 *
 * softcap > 0 replaces the scaled score x = scale * q.k by softcap * tanh(x /
 * softcap) before the softmax: the score_mod example ("soft-capping with
 * tanh", cap 30) of the PyTorch attention article (atyun.com/61003.html).
 * 0 disables it.
 *
 * mask2d_kind treats the tokens as a row-major grid with grid_w tokens per
 * row, token n at (n / grid_w, n % grid_w):
 *   ATTN_MASK2D_NEIGHBORHOOD: query i sees key j iff |r_i - r_j| < size and
 *     |c_i - c_j| < size -- the mask_mod example ("neighbourhood masking",
 *     grid 56 wide, size 5) of the same article;
 *   ATTN_MASK2D_WINDOW: the grid is cut into non-overlapping size x size
 *     windows displaced by `shift` tokens in both directions (0 = plain,
 *     size / 2 = shifted; border windows are partial, no cyclic wrap); query i
 *     sees key j iff both lie in the same window -- the window attention of
 *     "Flash Attention in a production Stable-Diffusion service"
 *     (xxmr.cn/news/81028), section 3.2.
 * Key blocks that no query of a work unit may see are skipped, as causal
 * attention skips the blocks above the diagonal.
 */
enum {
    ATTN_MASK2D_NONE = 0,
    ATTN_MASK2D_NEIGHBORHOOD = 1,
    ATTN_MASK2D_WINDOW = 2
};

typedef struct attn_score_mod_t {
    float softcap;   /* >= 0, finite; 0 = off */
    int mask2d_kind; /* ATTN_MASK2D_* */
    int grid_w;      /* tokens per grid row, >= 1 (2-D masks only) */
    int size;        /* neighbourhood radius or window side, >= 1 (2-D masks only) */
    int shift;       /* window displacement, >= 0 (windows only) */
} attn_score_mod_t;

/*
 * attn_fwd_mod -- attn_fwd with the variants of `mod` (host pointer, read
 * during the call only).  Soft-capping and 2-D masks combine with each other,
 * with is_causal and with key_lens (all masks intersect); an additive mask is
 * not accepted here.  With softcap = 0 and no 2-D mask it computes exactly
 * what attn_fwd computes.
 * Errors: as attn_fwd; ATTN_ERR_INVALID_ARG also for mod == NULL, a negative
 * or non-finite softcap, an unknown kind, or grid_w / size < 1 or shift < 0
 * with a 2-D mask.
 */
attn_status_t attn_fwd_mod(const void *q, const void *k, const void *v, void *out, float *lse,
                           int B, int Hq, int Hkv, int Nq, int Nk, int d,
                           float scale, int is_causal,
                           const int32_t *key_lens,
                           const attn_score_mod_t *mod,
                           void *stream);

/*
 * attn_splitkv_plan -- how attn_fwd_splitkv would split the keys, and the
 * workspace it then needs.  Host-only arithmetic (no CUDA call) when
 * sm_count > 0; sm_count == 0 queries the current device's SM count.
 *   n_splits: 0 = choose automatically; k > 0 = at most k ranges.
 *   n_splits_out (host, may be NULL): key ranges planned.
 *   workspace_bytes (host, may be NULL): bytes of device workspace needed
 *     (0 when the call writes out directly).
 * Decoding shapes -- (Hq / Hkv) * Nq <= 16 query rows per K/V head and not
 * causal -- run on the decode kernel: ranges of 32-key chunks; the automatic
 * count is the first minimiser of ceil(B * Hkv * n / SMs) * (chunks per range
 * + 15) over counts n that the equal cut realises exactly, with at least 6
 * chunks per range; its partial results always go through the workspace.  Other shapes run on the tile kernel:
 * ranges of 128-key blocks, the automatic choice minimising (waves of units
 * over the SMs) x (key blocks per range + 2), and one range writes out
 * directly.  The plan does not depend on an additive mask: with a mask, a
 * decoding shape runs the tile kernel with at most the planned ranges.
 * Errors: ATTN_ERR_INVALID_ARG for non-positive sizes, Hq % Hkv != 0 or
 * negative counts, ATTN_ERR_UNSUPPORTED for d not in {64, 128}.
 */
attn_status_t attn_splitkv_plan(int B, int Hq, int Hkv, int Nq, int Nk, int d, int is_causal, int n_splits,
                                int sm_count, int *n_splits_out, size_t *workspace_bytes);

/*
 * attn_fwd_splitkv -- attn_fwd with the keys of every (batch, head) cut into
 * ranges that run as separate work units, then merged: the decoding-phase
 * scheme that "FlashAttention technical analysis" (jsqmd.com/news/722897),
 * section 5.2, names FlashDecoding.  It serves short query blocks (Nq of 1 to
 * a few hundred) over long key sequences, where B * Hq alone leaves SMs idle.
 *
 * Range s gives O_s (its rows normalised by the range's own row sum) and
 * LSE_s; the merge is exact: with M = max_s LSE_s and w_s = exp(LSE_s - M),
 * O = sum_s w_s O_s / sum_s w_s and LSE = M + ln(sum_s w_s).  A range with no
 * unmasked key of a row has LSE_s = -inf and weight 0.
 *
 * Arguments as attn_fwd, plus:
 *   n_splits: 0 = automatic (attn_splitkv_plan), k > 0 = at most k ranges.
 *   workspace: device, 256-byte aligned, at least the bytes attn_splitkv_plan
 *     reports for the same sizes, is_causal and n_splits (may be NULL when
 *     that is 0).  The library
 *     writes it before reading it (nothing needs to start at zero); its
 *     contents after the call are unspecified.  Two calls in flight at once
 *     must not share a workspace.
 * Two kernels run on `stream`: the attention kernel -- the decode kernel
 * (CUDA cores; every query row of a K/V head shares each K/V chunk, read from
 * HBM once) or the tile kernel -- with partials to the workspace, then the
 * merge (out, lse); a tile-kernel call with one range writes out directly.
 * Errors: as attn_fwd; ATTN_ERR_INVALID_ARG also for n_splits < 0 or a
 * missing / short workspace, ATTN_ERR_ALIGNMENT for a misaligned workspace.
 */
attn_status_t attn_fwd_splitkv(const void *q, const void *k, const void *v, void *out, float *lse,
                               int B, int Hq, int Hkv, int Nq, int Nk, int d,
                               float scale, int is_causal,
                               const int32_t *key_lens,
                               const float *additive_mask, const int64_t *mask_strides,
                               int n_splits, void *workspace, size_t workspace_bytes,
                               void *stream);

/*
 * attn_fwd_splitkv_noalloc -- attn_fwd_splitkv with the workspace taken from a
 * fixed buffer inside the library instead of from the caller.  The pages have
 * no counterpart: it exists for callers that cannot hand over device memory
 * per call -- plain C hosts that only receive tensor pointers from another
 * framework and own no device allocator; servers that have reserved all of
 * the GPU's memory up front (for example for a key/value cache) so that a
 * new allocation would fail; and decode loops that must not call
 * cudaMalloc / cudaFree, which may synchronise the whole device and so stall
 * the other streams.
 *
 * The buffer is a statically sized device array of
 * ATTN_NOALLOC_SCRATCH_BYTES (16 MiB) per device, part of the library's
 * device image; nothing is allocated by this call or by the library.  A call
 * whose split plan (attn_splitkv_plan with the same sizes and n_splits) needs
 * more than that returns ATTN_ERR_SCRATCH before launching anything; a plan
 * of one range needs none.  Nothing in the buffer has to start at zero: the
 * attention kernel writes every partial result before the merge reads it.
 *
 * The first call on a device does one-time set-up with that device current
 * (kernel attributes and the buffer's device address); make it before any
 * stream capture.  Calls that overlap in time on one device -- on different
 * streams, or from different host threads -- share the buffer and race:
 * order them on one stream or synchronise between them.
 *
 * Arguments and results as attn_fwd_splitkv without workspace and
 * workspace_bytes.  Errors: as attn_fwd_splitkv, plus ATTN_ERR_SCRATCH.  All
 * argument checks run before the first-call set-up, so a rejected call does
 * no set-up.
 */
#define ATTN_NOALLOC_SCRATCH_BYTES (16u << 20)
attn_status_t attn_fwd_splitkv_noalloc(const void *q, const void *k, const void *v, void *out, float *lse,
                                       int B, int Hq, int Hkv, int Nq, int Nk, int d,
                                       float scale, int is_causal,
                                       const int32_t *key_lens,
                                       const float *additive_mask, const int64_t *mask_strides,
                                       int n_splits, void *stream);

/*
 * attn_fwd_fp8 -- attn_fwd on FP8 E4M3 inputs with one fp32 scale factor per
 * 128-row block of every head; the output stays bf16.
 *
 * "FlashAttention technical analysis" (jsqmd.com/news/722897), sections 4.2
 * and 6.3: Q, K and V enter the tensor cores as FP8, each block of rows with
 * its own scale factor, and the softmax and the accumulators stay in higher
 * precision.  The value computed is attn_fwd's on the dequantized inputs
 *   Q[b,h,i,:] = q_scale[b,h,i/128] * e4m3(q8[b,h,i,:])   (likewise K, V),
 * i.e. softmax(scale * Q K^T) V with per-row LSE.  Both products run on FP8
 * tensor cores with fp32 accumulation; the block scales of Q and K scale each
 * score block, and the probabilities enter the second product as E4M3 after
 * being multiplied by v_scale(block) / max(v_scale of the head), the largest
 * V scale being applied to the output once.  Rounding P to E4M3 (3 mantissa
 * bits) bounds the error of an output element by about 2^-4 times
 * sum_j P_ij |V_jc|, plus subnormal and bf16 output rounding.
 *
 * Layout, all device, contiguous:
 *   q8   uint8 E4M3 [B, Hq, Nq, d]      k8, v8   uint8 E4M3 [B, Hkv, Nk, d]
 *   q_scale fp32 [B, Hq, ceil(Nq/128)]   k_scale, v_scale fp32 [B, Hkv, ceil(Nk/128)]
 *   out  bf16 [B, Hq, Nq, d]             lse  fp32 [B, Hq, Nq] or NULL
 * Every scale must be positive and finite; the codes 0x7F and 0xFF (NaN) must
 * not occur.  The kernel does not check either (a violation gives undefined
 * values, never a fault).  q8, k8, v8 and out 16-byte aligned, scales and lse
 * 4-byte aligned.  d must be 128.  scale, is_causal, key_lens: as attn_fwd;
 * additive masks and split-KV are not offered on this path.
 * Errors: as attn_fwd; ATTN_ERR_UNSUPPORTED for d != 128.
 */
attn_status_t attn_fwd_fp8(const void *q8, const void *k8, const void *v8,
                           const float *q_scale, const float *k_scale, const float *v_scale,
                           void *out, float *lse,
                           int B, int Hq, int Hkv, int Nq, int Nk, int d,
                           float scale, int is_causal, const int32_t *key_lens, void *stream);

/*
 * attn_quantize_e4m3_blocks -- the FP8 inputs of attn_fwd_fp8 from a bf16
 * tensor, on the device: block quantisation with one fp32 scale factor per
 * 128-row block of every head ("FlashAttention technical analysis",
 * jsqmd.com/news/722897, section 4.2: FP8 with block quantisation; section
 * 6.3: each block keeps its own scale factor).  For each block, in fp32:
 *   amax = max |x| over its rows (fewer than 128 in a head's last block),
 *   scale = amax / 448 (1 when amax = 0), the largest finite E4M3 value 448,
 *   code = E4M3 of min(max(x / scale, -448), 448),
 * the division and the E4M3 conversion both rounding to nearest even.
 *   x       device bf16 [heads, N, d], 16-byte aligned (heads = B * H)
 *   codes   device uint8 [heads, N, d], 16-byte aligned (written)
 *   scales  device fp32 [heads, ceil(N / 128)], 4-byte aligned (written)
 * x must be finite.  d in {64, 128} (attn_fwd_fp8 takes d = 128).  One kernel
 * on `stream`, reading x once.
 * Errors: ATTN_ERR_INVALID_ARG (NULL pointer, non-positive size, more than
 * 2^31 - 1 blocks), ATTN_ERR_UNSUPPORTED (d), ATTN_ERR_ALIGNMENT, ATTN_ERR_CUDA.
 */
attn_status_t attn_quantize_e4m3_blocks(const void *x, void *codes, float *scales, int heads, int N, int d,
                                        void *stream);

/*
 * attn_bwd_plan -- device workspace bytes attn_bwd needs (host-only).  The
 * workspace holds two fp32 values per query row (D = rowsum(dO * O) and the
 * base-2 LSE), rows padded to a multiple of 128 per head.
 * Errors: ATTN_ERR_INVALID_ARG for non-positive sizes or a NULL output.
 */
attn_status_t attn_bwd_plan(int B, int Hq, int Nq, size_t *workspace_bytes);

/*
 * attn_bwd -- gradients of attn_fwd: given the forward inputs, its outputs O
 * and LSE, and dO = dLoss/dO, writes dQ, dK, dV.
 *
 * "FlashAttention technical analysis" (jsqmd.com/news/722897), section 3.3:
 * the forward keeps only per-row statistics; the backward recomputes each
 * block of P = exp(scale * Q K^T - LSE) and never stores an N x N matrix.
 * dV = P^T dO, dS = P o (dO V^T - D) with D_i = sum_t dO_it O_it,
 * dQ = scale dS K, dK = scale dS^T Q.  Grouped heads: dK and dV of a K/V head
 * sum the contributions of all query heads that read it.
 *
 * Layout as attn_fwd, all device, contiguous, 16-byte-aligned bases:
 *   q, out, dout, dq   bf16 [B, Hq, Nq, d]     (dq written)
 *   k, v, dk, dv       bf16 [B, Hkv, Nk, d]    (dk, dv written)
 *   lse                fp32 [B, Hq, Nq], as written by attn_fwd for the same inputs
 * scale, is_causal, key_lens: as attn_fwd (additive masks and the score
 * variants: attn_bwd_ex).  Rows of dq with no visible key and keys no query sees get 0.
 * workspace: device, 256-byte aligned, >= attn_bwd_plan bytes; scratch whose
 * contents need not be initialised; calls in flight at once must not share it.
 * Three kernels run on `stream` (row statistics, dK/dV, dQ).
 * Errors: as attn_fwd; ATTN_ERR_INVALID_ARG also for a NULL or short workspace.
 */
attn_status_t attn_bwd(const void *q, const void *k, const void *v, const void *out, const float *lse,
                       const void *dout, void *dq, void *dk, void *dv,
                       int B, int Hq, int Hkv, int Nq, int Nk, int d,
                       float scale, int is_causal, const int32_t *key_lens,
                       void *workspace, size_t workspace_bytes, void *stream);

/*
 * attn_bwd_ex -- attn_bwd for the forward's score and mask variants: the
 * gradients of attn_fwd with an additive mask, or of attn_fwd_mod with
 * soft-capping and / or a 2-D neighbourhood or window mask (`out` and `lse`
 * must come from that forward call with the same options).  With the score
 * s = c(x) + mask, x = scale * q.k, c(x) = softcap * tanh(x / softcap) (else
 * c(x) = x): P = exp(s - LSE), dS = P o (dP - D) as in attn_bwd, and the
 * gradient with respect to x is dS * c'(x), c'(x) = 1 - tanh^2(x / softcap),
 * from which dQ = scale dX K and dK = scale dX^T Q; keys a 2-D mask hides get
 * P = 0 (their blocks are computed, not skipped).  The additive mask gets no
 * gradient.  With all variants off it computes exactly what attn_bwd computes.
 *   additive_mask, mask_strides: as attn_fwd (fp32 device, NULL = none);
 *   mod: host pointer or NULL, as attn_fwd_mod.
 * An additive mask does not combine with key_lens or with `mod`
 * (ATTN_ERR_INVALID_ARG / ATTN_ERR_UNSUPPORTED, as in the forward).
 * Errors: as attn_bwd, plus those of attn_fwd_mod's `mod` checks.
 */
attn_status_t attn_bwd_ex(const void *q, const void *k, const void *v, const void *out, const float *lse,
                          const void *dout, void *dq, void *dk, void *dv,
                          int B, int Hq, int Hkv, int Nq, int Nk, int d,
                          float scale, int is_causal, const int32_t *key_lens,
                          const float *additive_mask, const int64_t *mask_strides,
                          const attn_score_mod_t *mod,
                          void *workspace, size_t workspace_bytes, void *stream);

/*
 * attn_check_device_status -- synchronise `stream`, then read and clear the
 * device-side error word of the current device.  Returns ATTN_OK,
 * ATTN_ERR_TIMEOUT, ATTN_ERR_DEVICE, or ATTN_ERR_CUDA if the synchronisation
 * itself failed.  `info` (host, may be NULL) receives the raw error word
 * (bits 0-7: code, bits 8-15: kernel role, bits 16-31: wait site).
 */
attn_status_t attn_check_device_status(void *stream, uint32_t *info);

/*
 * attn_set_wait_timeout_ns -- upper bound (nanoseconds, wall clock on the
 * device) of every wait inside the library's kernels; default 2e9.  After it
 * expires the waiting role records ATTN_ERR_TIMEOUT, stops its work, and the
 * block releases its tensor memory and returns.  0 restores the default.
 */
attn_status_t attn_set_wait_timeout_ns(uint64_t ns);

/*
 * attn_selftest_timeout -- launches a one-warp kernel that waits, with the
 * current bound, on a barrier nothing ever arrives at, so that the bounded
 * wait must expire and record ATTN_ERR_TIMEOUT.  Used by the failure tests;
 * it touches no caller memory.  Asynchronous on `stream`.
 */
attn_status_t attn_selftest_timeout(void *stream);

/*
 * attn_selftest_exp2_poly -- y[i] = 2^x[i] by the polynomial exponential that
 * the FP8 forward pass runs on the FMA pipe for one pair of probabilities in
 * four (x = n + f with n the nearest integer, 2^f from a cubic fitted for least
 * maximum relative error on |f| <= 1/2; 0 for x < -125).  Exposed so that its
 * accuracy can be tested against 2^x; not part of the attention computation.
 *   x, y: device fp32 [n], 4-byte aligned; n >= 0.  Asynchronous on `stream`.
 * Errors: ATTN_ERR_INVALID_ARG (n < 0, or a NULL pointer with n > 0),
 * ATTN_ERR_ALIGNMENT, ATTN_ERR_UNSUPPORTED / ATTN_ERR_CUDA as attn_fwd.
 */
attn_status_t attn_selftest_exp2_poly(const float *x, float *y, int n, void *stream);

/* Text for a status code (static storage). */
const char *attn_status_string(int status);

/* The cudaError_t kept from the last call that returned ATTN_ERR_CUDA (0 if none). */
int attn_last_cuda_error(void);

/* Library version: major * 10000 + minor * 100 + patch. */
int attn_version(void);

#ifdef __cplusplus
}
#endif

#endif /* ATTN_H_ */

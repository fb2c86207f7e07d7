/*
 * attn_bwd.h -- C ABI of the backward of the B200 (sm_100a) fused attention
 * declared in attn_fwd.h: the gradients dQ, dK, dV of
 * O = softmax(scale Q K^T + mask) V given the incoming gradient dO.
 *
 * The attention weights are recomputed from the forward's saved row
 * log-sum-exp instead of being stored (the FlashAttention recompute of the
 * bjdmk.com.cn survey page, section 5.1; forward intermediates reused by the
 * backward, intelliparadigm.com AVO page, section 3.2 item 3):
 *
 *     S  = scale Q K^T, masked as the forward (causal bottom-right, window)
 *     P  = exp(S - LSE)                       (LSE from the forward)
 *     dV = P^T dO
 *     dP = dO V^T,   D_i = sum_c dO[i][c] O[i][c],   dS = P * (dP - D)
 *     dQ = scale dS K,   dK = scale dS^T Q
 *
 * Grouped-query / multi-query attention: dK and dV of key/value head g sum
 * the contributions of every query head of its group (h / (h_q / h_kv) == g).
 * Keys that no query sees (under a sliding window with s_q < s_k, those
 * before the first query's window) carry no weight: their dK and dV are
 * written as zeros.
 *
 * Numerics: S and dP accumulate in FP32 on the tensor cores; P and dS are
 * rounded to BF16 before the products that use them; dQ, dK, dV accumulate
 * in FP32 and are written as BF16 (round to nearest even).  Every output
 * element is written once by one CTA (no atomics), so results are
 * bit-for-bit reproducible.
 */
#ifndef SDPA10_ATTN_BWD_H
#define SDPA10_ATTN_BWD_H

#include "attn_fwd.h"

#ifdef __cplusplus
extern "C" {
#endif

/*
 * Bytes of device workspace attn_bwd needs: two FP32 rows per query row of
 * every head, padded to a multiple of 128 rows (D = rowsum(dO * O) and the
 * negated base-2 LSE).  0 for non-positive sizes.
 */
size_t attn_bwd_workspace_bytes(int batch, int h_q, int s_q);

/*
 * attn_bwd -- gradients of attn_fwd / attn_fwd_window.
 *
 *   q, k, v   device, bf16, attn_fwd's layouts (read)
 *   o         device, bf16 [batch, s_q, h_q, d]: the forward's output (read)
 *   dout      device, bf16 [batch, s_q, h_q, d]: dL/dO (read)
 *   lse       device, fp32 [batch, h_q, s_q]: the forward's LSE (read)
 *   dq        device, bf16 [batch, s_q, h_q,  d] (written)
 *   dk, dv    device, bf16 [batch, s_k, h_kv, d] (written)
 *   batch, h_q, h_kv, s_q, s_k, d, causal, scale
 *             as attn_fwd (d must be 128); the same values the forward
 *             was called with
 *   window_left  -1 for none, else the forward's sliding window (requires
 *             causal = 1), as attn_fwd_window
 *   workspace device buffer of at least attn_bwd_workspace_bytes(batch,
 *             h_q, s_q) bytes, 256-byte aligned, owned by the caller and
 *             overwritten
 *   stream    CUDA stream (NULL: the legacy default stream)
 *
 * Three launches on `stream` (row statistics, dK/dV, dQ); asynchronous; the
 * call allocates nothing.  Outputs must not overlap the inputs or each
 * other.  q, k, v, o, dout, dq, dk, dv must be 16-byte aligned, lse 4-byte.
 *
 * Errors: ATTN_ERR_INVALID for null pointers, unsupported or inconsistent
 * sizes (as attn_fwd), window_left < -1 or a window without causal, or a
 * workspace smaller than attn_bwd_workspace_bytes; ATTN_ERR_ALIGN for
 * misaligned buffers; ATTN_ERR_UNSUPPORTED as attn_fwd (d != 128, causal
 * with s_q > s_k, ...).  These are detected before any launch, and then
 * nothing is written.  ATTN_ERR_CUDA if a launch fails (outputs and
 * workspace then hold unspecified values).  As for the forward, a device
 * wait that gives up makes the kernels exit early and the next attn_status
 * call report ATTN_ERR_TIMEOUT.
 */
int attn_bwd(const void* q, const void* k, const void* v, const void* o, const void* dout,
             const float* lse, void* dq, void* dk, void* dv, int batch, int h_q, int h_kv,
             int s_q, int s_k, int d, int causal, int window_left, float scale, void* workspace,
             size_t workspace_bytes, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* SDPA10_ATTN_BWD_H */

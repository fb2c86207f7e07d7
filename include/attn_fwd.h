/*
 * attn_fwd.h -- C ABI of the B200 (sm_100a) fused scaled dot-product
 * attention forward.
 *
 * The operation (rkmt.cn "GPU attention operator optimisation" page,
 * section 1; the three steps of the bjdmk.com.cn survey page, section 1):
 *
 *     S   = scale * Q K^T                  (per batch and query head)
 *     S   = S with S[i][j] = -inf for j > i + (s_k - s_q)
 *           (causal mode only, s_q <= s_k: the mask of the
 *           intelliparadigm.com AVO page, section 2.2, aligned to the
 *           bottom-right corner; j > i when s_q == s_k)
 *     O   = softmax_rows(S) V
 *     LSE = log(sum_j exp(S[i][j]))        (natural log, per query row)
 *
 * Grouped-query / multi-query attention (rkmt.cn page, section 3.2): query
 * head h reads key/value head h / (h_q / h_kv); h_kv == h_q is plain
 * multi-head attention, h_kv == 1 is multi-query attention.
 *
 * Numerics: Q, K, V are BF16; Q K^T and P V accumulate in FP32 on the tensor
 * cores; the softmax runs in FP32 (the precision split of the bjdmk.com.cn
 * page, section 3); the probabilities P are rounded to BF16 before the P V
 * product; O is written as BF16 (round to nearest even), LSE as FP32.
 * Inputs containing NaN or Inf give unspecified results (not checked).
 *
 * Every function returns an attn_status_t code.  On any error nothing is
 * written to o or lse.
 *
 * Device: every call launches on the calling thread's current CUDA device
 * (cudaGetDevice).  Device buffers must be allocations on that device and
 * `stream` one of its streams; the library does not look up where a pointer
 * lives, so a buffer of another device is not detected.  The Python binding
 * checks that the tensors of a call share one device and makes it current.
 */
#ifndef SDPA10_ATTN_FWD_H
#define SDPA10_ATTN_FWD_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    ATTN_OK = 0,
    ATTN_ERR_INVALID = 1,     /* null pointer, dimension <= 0, h_q % h_kv != 0,
                                 non-finite scale, causal not 0 or 1, size
                                 beyond the kernel's 32-bit tile indexing,
                                 workspace too small */
    ATTN_ERR_UNSUPPORTED = 2, /* d != 128, or causal with s_q > s_k */
    ATTN_ERR_ALIGN = 3,       /* a q/k/v/o pointer not 16-byte aligned (TMA),
                                 or lse not 4-byte aligned */
    ATTN_ERR_CUDA = 4,        /* a CUDA runtime/driver call failed (no device,
                                 launch failure, ...) */
    ATTN_ERR_TIMEOUT = 5,     /* a kernel gave up a bounded wait (reported by
                                 attn_status) */
    ATTN_ERR_TOO_LARGE = 6    /* attn_fwd_host_static: the problem does not fit
                                 the library's static device staging area */
} attn_status_t;

/*
 * attn_fwd -- launch the fused forward on `stream` (a cudaStream_t; NULL is
 * the legacy default stream) and return without synchronising.
 *
 *   q    device, bf16 [batch, s_q, h_q,  d] contiguous (read)
 *   k    device, bf16 [batch, s_k, h_kv, d] contiguous (read)
 *   v    device, bf16 [batch, s_k, h_kv, d] contiguous (read)
 *   o    device, bf16 [batch, s_q, h_q,  d] contiguous (written)
 *   lse  device, fp32 [batch, h_q, s_q]     contiguous (written)
 *   d     must be 128
 *   causal  0: full attention; 1: key j is visible to query i iff
 *           j <= i + (s_k - s_q) -- the mask aligned to the bottom-right
 *           corner, so the last query sees every key (j <= i when
 *           s_q == s_k); requires s_q <= s_k
 *   scale   multiplies Q K^T before the softmax (usually 1/sqrt(d)); any
 *           finite value, including 0 (uniform weights over the visible
 *           keys) and negative values
 *
 * The caller owns every buffer; the call allocates nothing.  o and lse must
 * not overlap the inputs.  q/k/v/o must be 16-byte aligned, lse 4-byte
 * aligned.  The kernel's device-side waits are bounded: if one gives up, the
 * kernel exits early (o/lse then hold unspecified values) and the next
 * attn_status call reports ATTN_ERR_TIMEOUT.
 */
int attn_fwd(const void* q, const void* k, const void* v, void* o, float* lse,
             int batch, int h_q, int h_kv, int s_q, int s_k, int d,
             int causal, float scale, void* stream);

/*
 * attn_fwd_window -- causal attention with a sliding window (the local
 * window variant of the bjdmk.com.cn survey page, section 2.1): query row i
 * sees keys i + (s_k - s_q) - window_left .. i + (s_k - s_q), the
 * window_left keys before its diagonal and the diagonal key itself.
 * Arguments, layouts and errors as attn_fwd with causal = 1, plus:
 *
 *   window_left  >= 0 (ATTN_ERR_INVALID otherwise); 0 leaves each row only
 *                its diagonal key; >= s_k is the plain causal mask
 *
 * Key blocks wholly outside a query block's window are skipped, so the work
 * grows with window_left, not with s_k.  One launch; asynchronous; allocates
 * nothing.
 */
int attn_fwd_window(const void* q, const void* k, const void* v, void* o, float* lse,
                    int batch, int h_q, int h_kv, int s_q, int s_k, int d,
                    int window_left, float scale, void* stream);

/*
 * attn_fwd_varlen -- a packed batch of sequences of different lengths
 * (the dynamic sequence-length support of the intelliparadigm.com AVO page,
 * section 6): sequence b holds query rows cu_seqlens_q[b] ..
 * cu_seqlens_q[b+1] - 1 and keys cu_seqlens_k[b] .. cu_seqlens_k[b+1] - 1
 * of the packed tensors, and each sequence is its own attention problem
 * (no query sees another sequence's keys; the causal mask and window are
 * those of attn_fwd / attn_fwd_window with that sequence's s_q and s_k).
 *
 *   q    device, bf16 [total_q, h_q,  d] contiguous (read)
 *   k    device, bf16 [total_k, h_kv, d] contiguous (read)
 *   v    device, bf16 [total_k, h_kv, d] contiguous (read)
 *   o    device, bf16 [total_q, h_q,  d] contiguous (written)
 *   lse  device, fp32 [h_q, total_q]     contiguous (written)
 *   cu_seqlens_q, cu_seqlens_k  device, int32 [batch + 1], non-decreasing,
 *        starting at 0 and ending at total_q / total_k (4-byte aligned)
 *   max_seqlen_q, max_seqlen_k  upper bounds of the sequences' lengths (the
 *        launch has work items for max_seqlen_q rows per sequence)
 *   causal, window_left  as attn_fwd / attn_fwd_window (window_left = -1:
 *        none; a window needs causal = 1); causal needs s_q <= s_k per
 *        sequence.  In a sequence with more query rows than keys the first
 *        s_q - s_k rows see no key: where such a row shares a 128-row block
 *        with a row that sees keys it gets O = 0, LSE = -inf, but blocks
 *        in which no row sees a key are not written at all
 *
 * The host cannot read cu_seqlens: sequences that break the rules above
 * give unspecified values, but every access stays inside the packed
 * tensors.  One launch; asynchronous; allocates nothing.
 */
int attn_fwd_varlen(const void* q, const void* k, const void* v, void* o, float* lse,
                    const int* cu_seqlens_q, const int* cu_seqlens_k, int batch,
                    int max_seqlen_q, int max_seqlen_k, int total_q, int total_k,
                    int h_q, int h_kv, int d, int causal, int window_left, float scale,
                    void* stream);

/*
 * attn_fwd_fp8 -- the forward on FP8 E4M3 inputs with per-tensor scales
 * (the FP8-GEMM / FP32-softmax precision split of the bjdmk.com.cn survey
 * page, section 3, and the rkmt.cn page, section 3.1.1): the inputs stand for
 * Q = q_scale * q, K = k_scale * k, V = v_scale * v, and the result is
 * attn_fwd's on those values:
 *
 *   q, k, v   device, E4M3 bytes ("e4m3fn": no infinities) in attn_fwd's
 *             layouts, one byte per element, 16-byte aligned
 *   o, lse    as attn_fwd (BF16 O, FP32 natural-log LSE)
 *   q_scale, k_scale, v_scale  finite per-tensor scales (ATTN_ERR_INVALID
 *             otherwise)
 *
 * Q K^T and P V run on the tensor core in FP8 (kind::f8f6f4) with FP32
 * accumulation; the softmax is FP32; the weights P are rounded to E4M3
 * (stored as 2^6 P so the bulk of a row stays in E4M3's normal range).
 * Arguments and errors otherwise as attn_fwd.  One launch; asynchronous;
 * allocates nothing.
 */
int attn_fwd_fp8(const void* q, const void* k, const void* v, void* o, float* lse,
                 int batch, int h_q, int h_kv, int s_q, int s_k, int d, int causal,
                 float scale, float q_scale, float k_scale, float v_scale, void* stream);

/*
 * attn_fwd_host -- the same forward on HOST buffers: copies q, k, v to the
 * device, runs the forward, copies o and lse back, and returns without
 * synchronising (the caller synchronises `stream` before reading o/lse;
 * pinned host memory makes the copies asynchronous).
 *
 *   q, k, v, o, lse   host pointers with the layouts of attn_fwd
 *   workspace         device buffer of at least
 *                     attn_fwd_host_workspace_bytes(...) bytes, 256-byte
 *                     aligned, owned by the caller
 *
 * Problems with at least two key/value heads and 32 MiB or more of inputs
 * run in up to 8 groups of key/value heads (with their query heads, each
 * group at least 16 MiB of inputs): a group's rows are copied in with strided
 * copies on a host-to-device stream, its forward runs on `stream`, and its
 * O and LSE go back on a device-to-host stream, so the copies of one group
 * overlap the kernel of another.  The two copy streams and their events
 * belong to the library (created on the first such call on each device).
 * Ordering is that of `stream`: the call starts after the work already
 * queued on it, and it waits for the call's last copy out, so synchronising
 * `stream` covers everything.  Results are bit-identical to attn_fwd's.
 *
 * Errors: as attn_fwd, plus ATTN_ERR_INVALID for a null or too small
 * workspace and ATTN_ERR_ALIGN for a workspace not 256-byte aligned, all
 * found before anything is queued.  ATTN_ERR_CUDA from a copy or launch that
 * fails to be queued part way through: o and lse are then unspecified, and
 * copies of earlier groups may still be running on the library's streams
 * when the call returns, so synchronise the device (not only `stream`)
 * before reusing or freeing the buffers.
 */
int attn_fwd_host(const void* q, const void* k, const void* v, void* o, float* lse,
                  int batch, int h_q, int h_kv, int s_q, int s_k, int d,
                  int causal, float scale, void* workspace, size_t workspace_bytes,
                  void* stream);

/* Device workspace bytes attn_fwd_host needs for these sizes (0 on bad sizes). */
size_t attn_fwd_host_workspace_bytes(int batch, int h_q, int h_kv, int s_q, int s_k, int d);

/*
 * attn_fwd_host_static -- attn_fwd_host for callers that cannot allocate
 * device memory: instead of a caller-provided workspace it stages q, k, v, o
 * and lse in a device array that the library itself declares at file scope
 * (ATTN_STATIC_STAGING_BYTES, held on every GPU that loads the library until
 * the process exits).  It calls no cudaMalloc/cudaFree or other allocating
 * routine, and creates no streams or events: its copies in, forward and
 * copies out run in order on `stream` alone (not grouped and overlapped as
 * in attn_fwd_host).  The paper has no counterpart to this entry point: it
 * is a deployment convenience of this library.
 *
 * Who needs it: code that may not allocate on the device at call time -- a
 * plugin handed only host arrays by an application that owns all device
 * memory (for example through a framework's caching allocator that must stay
 * the only allocator), or a caller that cannot afford the device-wide
 * synchronisation a cudaMalloc/cudaFree can imply.
 *
 *   q, k, v, o, lse   host pointers, layouts of attn_fwd (pinned memory makes
 *                     the copies asynchronous)
 *   returns           ATTN_ERR_TOO_LARGE, before any CUDA call, when
 *                     attn_fwd_host_workspace_bytes(...) exceeds
 *                     ATTN_STATIC_STAGING_BYTES; otherwise as attn_fwd_host
 *
 * The first call on a device looks up the staging array's device address
 * (cudaGetSymbolAddress, with that device current); make that first call
 * before any stream capture.  Every call on a device shares the one staging
 * array and it keeps the last call's contents; nothing in it needs to start
 * at zero (each call overwrites the inputs and the kernel writes every output
 * element).  Calls whose GPU work overlaps -- on different streams, or from
 * different host threads -- race on the array: serialise them.
 */
#define ATTN_STATIC_STAGING_BYTES ((size_t)32 << 20)
int attn_fwd_host_static(const void* q, const void* k, const void* v, void* o, float* lse,
                         int batch, int h_q, int h_kv, int s_q, int s_k, int d,
                         int causal, float scale, void* stream);

/*
 * Split-KV forward (split the key sequence into ranges, then merge).
 *
 * The same result as attn_fwd, computed as one work item per (query-block
 * pair, key range) and then merged: for a key set split into ranges r, with
 * O_r the softmax-weighted average of V over range r and LSE_r the
 * log-sum-exp of that range's scaled scores,
 *     LSE = log sum_r exp(LSE_r),    O = sum_r exp(LSE_r - LSE) O_r
 * (the rkmt.cn GPU attention operator page's "local attention, then global
 * reduction", section 3.1.1, applied to whole key ranges).  It pays off when
 * batch * h_q * ceil(s_q / 256) work items leave most SMs idle, e.g. few
 * query rows over a long key sequence.
 *
 * attn_fwd_num_splits -- the key-range count this library would pick on the
 * current device: 1 when the pairs already fill the SMs, else about
 * #SMs / pairs, at most ceil(s_k / 128).  0 on invalid sizes.
 */
int attn_fwd_num_splits(int batch, int h_q, int h_kv, int s_q, int s_k, int d, int causal);

/* Device workspace bytes attn_fwd_split needs for num_splits ranges
 * (num_splits * batch * h_q * s_q * (128 + 1) FP32 values, rounded; 0 on bad
 * sizes). */
size_t attn_fwd_split_workspace_bytes(int batch, int h_q, int s_q, int num_splits);

/*
 * attn_fwd_split -- attn_fwd through num_splits key ranges (>= 1; more than
 * ceil(s_k / 128) is reduced to that, and the ranges are ceil(n_kb / n)
 * key blocks of 128 each, the last one shorter).  Arguments, layouts and
 * errors as attn_fwd, plus:
 *
 *   workspace  device buffer of at least
 *              attn_fwd_split_workspace_bytes(batch, h_q, s_q, num_splits)
 *              bytes, 256-byte aligned, owned by the caller (per-range
 *              partials: FP32 O_r [n][batch][h_q][s_q][128], then FP32 LSE_r
 *              [n][batch][h_q][s_q]); ATTN_ERR_INVALID if smaller or null,
 *              ATTN_ERR_ALIGN if misaligned.
 *
 * Two launches on `stream` (the forward writing partials, then the merge);
 * asynchronous; allocates nothing.  Results agree with attn_fwd within
 * rounding (bit for bit when num_splits is 1).
 */
int attn_fwd_split(const void* q, const void* k, const void* v, void* o, float* lse,
                   int batch, int h_q, int h_kv, int s_q, int s_k, int d, int causal,
                   float scale, int num_splits, void* workspace, size_t workspace_bytes,
                   void* stream);

/*
 * attn_fwd_partials -- the partial of one key range: the forward over the
 * keys given, written unmerged for attn_merge_partials.  What a rank of a
 * key-sequence (context-parallel) split computes on its own key shard before
 * the partials are gathered.  Arguments and errors as attn_fwd, except:
 *
 *   o_part    device, fp32 [batch, h_q, s_q, d] (written): softmax over these
 *             keys times V, already divided by the range's row sum; 16-byte
 *             aligned
 *   lse_part  device, fp32 [batch, h_q, s_q] (written): natural-log
 *             log-sum-exp of the range's scaled scores
 *
 * With causal = 1 the mask is attn_fwd's, aligned to the bottom-right corner
 * of THIS call's keys (s_q <= s_k); a shard of a longer key sequence whose
 * keys do not end at the diagonal needs attn_fwd_partials_shard.
 *
 * One launch; asynchronous; allocates nothing.
 */
int attn_fwd_partials(const void* q, const void* k, const void* v, float* o_part,
                      float* lse_part, int batch, int h_q, int h_kv, int s_q, int s_k, int d,
                      int causal, float scale, void* stream);

/*
 * attn_fwd_partials_shard -- attn_fwd_partials for a key shard that need not
 * end at the causal diagonal of the whole problem: what one rank of a
 * key-sequence (context-parallel) split computes when the rank holds keys
 * [k0, k0 + s_k) of S_k keys in all.  Arguments, layouts and errors as
 * attn_fwd_partials, plus:
 *
 *   diag_offset  causal = 1: query row i sees key j of this call iff
 *                j <= i + diag_offset.  With the queries as the last s_q of
 *                the whole key sequence (the bottom-right mask of attn_fwd),
 *                a shard at global key k0 takes diag_offset = S_k - s_q - k0.
 *                Negative and large values are allowed (|diag_offset| <=
 *                2^30); ignored when causal = 0.  s_q > s_k is allowed.
 *
 * A row that sees none of the shard's keys gets O_r = 0 and LSE_r = -inf (no
 * weight in attn_merge_partials).  One launch, or two when some rows see no
 * key at all (a fill of those rows, then the forward); asynchronous;
 * allocates nothing.
 */
int attn_fwd_partials_shard(const void* q, const void* k, const void* v, float* o_part,
                            float* lse_part, int batch, int h_q, int h_kv, int s_q, int s_k,
                            int d, int causal, int diag_offset, float scale, void* stream);

/*
 * attn_merge_partials -- the merge step alone, for partials computed
 * elsewhere (for example over key ranges held by different GPUs and gathered
 * onto this one):
 *
 *   o_parts    device, fp32 [n_parts, batch, h_q, s_q, d], each part already
 *              normalised over its own keys (16-byte aligned)
 *   lse_parts  device, fp32 [n_parts, batch, h_q, s_q], natural log; a part
 *              with no keys for a row carries -inf there (weight 0; its O
 *              values for that row are not read)
 *   o          device, bf16 [batch, s_q, h_q, d] (written, 16-byte aligned)
 *   lse        device, fp32 [batch, h_q, s_q] (written)
 *   d          must be 128
 *
 * A row whose parts are all -inf gets O = 0 and LSE = -inf.  One launch on
 * `stream`; asynchronous; allocates nothing.  ATTN_ERR_INVALID on a null
 * pointer or a count <= 0, ATTN_ERR_UNSUPPORTED if d != 128, ATTN_ERR_ALIGN
 * on misaligned buffers.
 */
int attn_merge_partials(const float* o_parts, const float* lse_parts, int n_parts, int batch,
                        int h_q, int s_q, int d, void* o, float* lse, void* stream);

/*
 * attn_status -- synchronise `stream`, then read and clear the calling
 * device's kernel status word.  Returns ATTN_OK, ATTN_ERR_TIMEOUT if a kernel
 * launched since the last call gave up a bounded wait, or ATTN_ERR_CUDA if
 * the synchronisation itself failed.
 */
int attn_status(void* stream);

/* Static, human-readable text for a status code. */
const char* attn_strerror(int code);

/*
 * attn_set_wait_timeout_ns -- bound (nanoseconds) on every device-side wait
 * of kernels launched afterwards by this process (default 2e9 = 2 s;
 * 0 restores the default).
 */
int attn_set_wait_timeout_ns(uint64_t ns);

/*
 * attn_selftest_wait_timeout -- launch one CTA that waits on a barrier
 * nothing ever arrives on, bounded by `timeout_ns`; the wait gives up, the
 * kernel sets the status word and exits.  A following attn_status returns
 * ATTN_ERR_TIMEOUT.  Exercises the bounded-wait path without faulting.
 */
int attn_selftest_wait_timeout(uint64_t timeout_ns, void* stream);

/* Number of kernel launches the last forward call made (1; 2 for
 * attn_fwd_split: forward + merge; 1 or 2 for attn_fwd_partials_shard). */
int attn_last_launch_count(void);

#ifdef __cplusplus
}
#endif

#endif /* SDPA10_ATTN_FWD_H */

// attn_common.cuh -- constants, launch parameters and the bounded mbarrier
// waits shared by the attention kernels.
#pragma once

#include <cuda_bf16.h>
#include <math_constants.h>

#include "sm100_ptx.cuh"

namespace sdpa10 {

constexpr int kHeadDim = 128;
constexpr int kBlockM = 128;                        // query rows per tile
constexpr int kBlockN = 128;                        // keys per key/value tile
constexpr int kTileBytes = kBlockM * kHeadDim * 2;  // 32 KiB: one Q, K or V tile
constexpr int kHalfTileBytes = kTileBytes / 2;      // one 64-column (128-byte row) half
constexpr int kTmemCols = 512;
constexpr unsigned kStatusTimeout = 1u;

// Rescale the running output only when the row maximum grows by more than
// this many powers of two; otherwise keep the stale maximum (probabilities
// then stay below 2^8, well inside FP32 and BF16 range, and the final O / l
// and LSE are unchanged).
constexpr float kRescaleThresholdLog2 = 8.0f;

// Division by a divisor fixed for the launch, without the hardware's
// float-reciprocal integer division (whose conversions share the XU pipe
// with the softmax's ex2): q = (umulhi(n, m) + n) >> s with s = ceil(log2 d)
// and m = floor(2^32 (2^s - d) / d) + 1 (Granlund and Montgomery, "Division
// by invariant integers using multiplication", 1994); exact for
// 0 <= n < 2^31 and 1 <= d < 2^31.
struct FastDiv {
    uint32_t d, m, s;
    __host__ __device__ static FastDiv make(uint32_t d) {
        uint32_t s = 0;
        while ((1ull << s) < d) ++s;
        const uint64_t m = ((1ull << 32) * ((1ull << s) - d)) / d + 1;
        return FastDiv{d, static_cast<uint32_t>(m), s};
    }
    __device__ __forceinline__ int div(int n) const {
        const uint32_t u = static_cast<uint32_t>(n);
        return static_cast<int>((__umulhi(u, m) + u) >> s);
    }
};

struct FwdParams {
    int batch, h_q, h_kv, s_q, s_k;
    int group;    // h_q / h_kv
    int n_qb;     // ceil(s_q / 128)
    int n_kb;     // ceil(s_k / 128)
    int n_pairs;  // ceil(n_qb / 2): CTA tiles per (batch, head)
    int causal;
    int causal_offset;      // causal row i sees keys 0 .. i + causal_offset: s_k - s_q,
                            // or a key shard's diagonal (may be negative)
    int num_tiles;          // work items: pairs x n_splits
    int units_per_section;  // (batch, kv head) units whose K/V share L2 at once
    int n_splits;           // key ranges per pair (1: the whole key sequence)
    int kb_per_split;       // key blocks per range
    // Work-item decoding (see PairCursor::decode): sections of
    // units_per_section (batch, kv head) units, the last one holding
    // last_units; the divisors the decoding needs.
    int last_section, last_units;
    FastDiv div_splits;     // n_splits
    FastDiv div_section;    // units_per_section * group * n_pairs
    FastDiv div_rank;       // units_per_section * group
    FastDiv div_rank_last;  // last_units * group
    FastDiv div_group;      // group
    FastDiv div_h_kv;       // h_kv
    // |scale| * log2(e) (at least 1e-30, see below).  A negative scale is
    // carried by the sign of the scores themselves: the Q K^T instruction
    // descriptor negates A, so the tensor core produces -Q K^T and the
    // softmax always works with a positive factor.  Scale 0 runs with the
    // factor 1e-30: every exponent is then below 2^-90 and every weight
    // rounds to exactly 1 in FP32, the uniform softmax, while masked
    // scores (-inf) still give weight 0 (0 * -inf would be NaN).
    float scale_log2;
    uint32_t idesc_qk;      // instruction descriptor of S = (+/-) Q K^T
    __nv_bfloat16* o;
    float* lse;
    // Split-KV partials (null unless n_splits > 1 or a split launch): per key
    // range r, O_r = softmax over that range times V, FP32
    // [n_splits][batch][h_q][s_q][128], and LSE_r [n_splits][batch][h_q][s_q].
    float* o_part;
    float* lse_part;
    unsigned long long timeout_ns;
    unsigned int* status;
    int window_left;  // sliding window (windowed kernel only): keys before the diagonal
    // Packed variable-length batch (varlen kernel only): sequence b holds
    // packed query rows cu_q[b] .. cu_q[b+1] - 1 and keys cu_k[b] ..
    // cu_k[b+1] - 1; O is [total_q][h_q][128], LSE [h_q][total_q].
    const int* cu_q;
    const int* cu_k;
    int total_q;
    float v_scale;  // FP8 kernel only: V = v_scale * E4M3 values (1 otherwise)
};

// ------------------------------------------------------------------ waits
struct WaitCtx {
    volatile int* abort_flag;  // shared memory, per CTA
    unsigned int* status;      // global, per device
    unsigned long long timeout_ns;
};

// Slow path of a bounded mbarrier wait.  Gives up when the CTA's abort flag
// is raised (if honoured) or the time limit passes; a timeout raises the
// abort flag and sets the status word.
__device__ __forceinline__ bool wait_slow(uint32_t bar, uint32_t parity, WaitCtx w,
                                       bool honour_abort) {
    // Each probe may sleep up to kSuspendNs in hardware (woken as soon as
    // the phase completes); the abort flag and the time limit are checked
    // after every probe, so the wait stays bounded.
    constexpr uint32_t kSuspendNs = 20000;
    const uint64_t t0 = ptx::globaltimer_ns();
    for (uint32_t i = 1;; ++i) {
        if (ptx::mbar_try_wait_sleep(bar, parity, kSuspendNs)) return true;
        if (honour_abort && *w.abort_flag) return false;
        if (ptx::globaltimer_ns() - t0 > w.timeout_ns || i > (1u << 28)) {
            *w.abort_flag = 1;
            atomicOr(w.status, kStatusTimeout);
            return false;
        }
    }
}

__device__ __forceinline__ bool wait_bar(uint32_t bar, uint32_t parity, const WaitCtx& w) {
    if (ptx::mbar_try_wait(bar, parity)) return true;
    return wait_slow(bar, parity, w, true);
}


// Warp-uniform wait: every lane waits, and the warp proceeds only if all did.
__device__ __forceinline__ bool wait_bar_warp(uint32_t bar, uint32_t parity, const WaitCtx& w) {
    const bool ok = wait_bar(bar, parity, w);
    return __all_sync(0xffffffffu, ok);
}

// Waits on a barrier nothing arrives on; the bounded wait must give up,
// set the status word and let the kernel return.
__global__ void wait_timeout_selftest_kernel(unsigned int* status, unsigned long long timeout_ns) {
    __shared__ __align__(8) uint64_t bar_storage;
    __shared__ int abort_storage;
    const uint32_t b = ptx::smem_u32(&bar_storage);
    if (threadIdx.x == 0) {
        ptx::mbar_init(b, 1);
        abort_storage = 0;
        ptx::fence_mbar_init();
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        const WaitCtx w{&abort_storage, status, timeout_ns};
        wait_bar(b, 0, w);
    }
    __syncthreads();
}

}  // namespace sdpa10

// attn_merge.cuh -- combine per-key-range attention partials into O and LSE.
//
// Softmax over a key set split into ranges r: with O_r the softmax-weighted
// average of V over range r and LSE_r the log-sum-exp of the range's scaled
// scores, the whole set gives
//     LSE = log sum_r exp(LSE_r)      O = sum_r exp(LSE_r - LSE) O_r,
// the "local attention, then global reduction" merge of the rkmt.cn page
// (section 3.1.1) applied to whole key ranges.  This is memory-bound work:
// one warp per output row reads the row's partials (512 bytes each, 16 bytes
// per lane) and writes 256 bytes of BF16 O and one FP32 LSE.
#pragma once

#include <cuda_bf16.h>
#include <math_constants.h>

#include <cstddef>

namespace sdpa10 {

struct MergeParams {
    const float* o_part;    // [n_parts][rows][128] FP32, rows = batch * h_q * s_q
    const float* lse_part;  // [n_parts][rows], natural log
    int n_parts;
    int batch, h_q, s_q;
    // Key ranges of keys_per_part keys each, over s_k keys: range r holds
    // keys [r * keys_per_part, (r + 1) * keys_per_part).  A range that holds
    // no key of the row (past s_k, or past row + causal_offset under the
    // causal mask) is not read.  keys_per_part = 0: every part is read for every row (a part
    // with LSE = -inf then carries no weight).
    int keys_per_part, s_k, causal;
    int causal_offset;  // s_k - s_q: causal row i sees keys 0 .. i + causal_offset
    __nv_bfloat16* o;  // [batch][s_q][h_q][128]
    float* lse;        // [batch][h_q][s_q]
};

constexpr int kMergeThreads = 256;
constexpr int kMergeBatch = 8;  // partials whose loads are in flight together

__global__ void __launch_bounds__(kMergeThreads) attn_merge_kernel(const MergeParams m) {
    const int lane = threadIdx.x & 31;
    const size_t rows = static_cast<size_t>(m.batch) * m.h_q * m.s_q;
    const size_t warps = static_cast<size_t>(gridDim.x) * (kMergeThreads / 32);
    for (size_t r = blockIdx.x * static_cast<size_t>(kMergeThreads / 32) + (threadIdx.x >> 5);
         r < rows; r += warps) {
        const int i = static_cast<int>(r % m.s_q);
        const size_t bh = r / m.s_q;
        const int h = static_cast<int>(bh % m.h_q);
        const int b = static_cast<int>(bh / m.h_q);
        int nv = m.n_parts;
        if (m.keys_per_part > 0) {
            nv = min(nv, (m.s_k + m.keys_per_part - 1) / m.keys_per_part);
            if (m.causal) nv = min(nv, (i + m.causal_offset) / m.keys_per_part + 1);
        }
        // The loads of kMergeBatch partials are issued before any of them
        // is combined (the row's partials are independent loads; walking
        // them one by one left the kernel latency-bound).  The sums run in
        // partial order, as the definition's left-to-right sum.
        float mx = -CUDART_INF_F;
        for (int s0 = 0; s0 < nv; s0 += kMergeBatch) {
            float l[kMergeBatch];
#pragma unroll
            for (int k = 0; k < kMergeBatch; ++k)
                l[k] = s0 + k < nv ? m.lse_part[static_cast<size_t>(s0 + k) * rows + r]
                                   : -CUDART_INF_F;
#pragma unroll
            for (int k = 0; k < kMergeBatch; ++k) mx = fmaxf(mx, l[k]);
        }
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
        float wsum = 0.f;
        if (mx != -CUDART_INF_F) {
            for (int s0 = 0; s0 < nv; s0 += kMergeBatch) {
                float l[kMergeBatch];
                float4 v[kMergeBatch];
#pragma unroll
                for (int k = 0; k < kMergeBatch; ++k) {
                    const size_t idx = static_cast<size_t>(s0 + k) * rows + r;
                    l[k] = s0 + k < nv ? m.lse_part[idx] : -CUDART_INF_F;
                    // A part with no keys for the row (-inf) is not read.
                    v[k] = l[k] != -CUDART_INF_F
                               ? reinterpret_cast<const float4*>(m.o_part + idx * 128)[lane]
                               : make_float4(0.f, 0.f, 0.f, 0.f);
                }
#pragma unroll
                for (int k = 0; k < kMergeBatch; ++k) {
                    if (l[k] == -CUDART_INF_F) continue;
                    const float w = expf(l[k] - mx);
                    wsum += w;
                    acc.x += w * v[k].x;
                    acc.y += w * v[k].y;
                    acc.z += w * v[k].z;
                    acc.w += w * v[k].w;
                }
            }
        }
        const float inv = wsum > 0.f ? 1.f / wsum : 0.f;
        const __nv_bfloat162 lo = __floats2bfloat162_rn(acc.x * inv, acc.y * inv);
        const __nv_bfloat162 hi = __floats2bfloat162_rn(acc.z * inv, acc.w * inv);
        uint2 packed;
        packed.x = *reinterpret_cast<const uint32_t*>(&lo);
        packed.y = *reinterpret_cast<const uint32_t*>(&hi);
        reinterpret_cast<uint2*>(m.o + ((static_cast<size_t>(b) * m.s_q + i) * m.h_q + h) * 128)[lane] =
            packed;
        if (lane == 0) m.lse[r] = wsum > 0.f ? mx + logf(wsum) : -CUDART_INF_F;
    }
}

}  // namespace sdpa10

namespace sdpa10 {

// Partials of a key shard under the causal mask: query rows 0 .. n_empty - 1
// see none of the shard's keys.  The forward skips their blocks when whole
// blocks are empty, so this writes their partial (O = 0, LSE = -inf: no
// weight in a merge).  One warp per row, 16 bytes per lane; memory-bound.
__global__ void __launch_bounds__(kMergeThreads)
    attn_fill_empty_rows_kernel(float* o_part, float* lse_part, int batch, int h_q, int s_q,
                                int n_empty) {
    const int lane = threadIdx.x & 31;
    const size_t rows = static_cast<size_t>(batch) * h_q * n_empty;
    const size_t warps = static_cast<size_t>(gridDim.x) * (kMergeThreads / 32);
    for (size_t r = blockIdx.x * static_cast<size_t>(kMergeThreads / 32) + (threadIdx.x >> 5);
         r < rows; r += warps) {
        const size_t bh = r / n_empty;
        const size_t row = bh * s_q + (r - bh * n_empty);  // [batch][h_q][s_q] row index
        reinterpret_cast<float4*>(o_part + row * 128)[lane] = make_float4(0.f, 0.f, 0.f, 0.f);
        if (lane == 0) lse_part[row] = -CUDART_INF_F;
    }
}

}  // namespace sdpa10

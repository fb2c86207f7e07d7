// attn_bwd_kernel.cuh -- backward of the fused attention forward for B200
// (sm_100a): dQ, dK, dV from Q, K, V, the forward's O and LSE, and dO.
//
// The backward recomputes the attention weights from the forward's saved
// row statistics instead of storing them (the FlashAttention recompute the
// bjdmk.com.cn survey page describes, section 5.1; the AVO page's reuse of
// forward intermediates, section 3.2):
//     P_ij = 2^(S_ij c - L_i),  S = Q K^T,  c = scale log2(e),  L = LSE log2(e)
//     D_i  = sum_c dO_ic O_ic  (= sum_j P_ij dP_ij)
//     dP   = dO V^T,   dS = P * (dP - D)
//     dQ   = scale dS K,   dK = scale dS^T Q,   dV = P^T dO
//
// Three launches:
//   attn_bwd_prep_kernel  -- D and -L per query row (memory-bound), written
//                            to a padded workspace (padding rows: -L = -inf,
//                            D = 0, so they carry weight 0);
//   attn_bwd_dq_kernel    -- one CTA item per 128-row query block
//                            (persistent): Q and dO stay in shared memory,
//                            K/V tiles stream through a two-slot ring; per
//                            key block S and dP on the tensor core (TMEM),
//                            dS by two warpgroups (each 64 of the block's
//                            keys, thread = row), written to TMEM in BF16;
//                            dQ += dS K on the tensor core reads it there as
//                            the A operand;
//   attn_bwd_dkdv_kernel  -- one CTA item per 128-key block of a key/value
//                            head: K and V stay in shared memory, 128-row
//                            Q / dO tiles of every query head of the group
//                            stream through two-slot rings; S^T = K Q^T and
//                            dP^T = V dO^T on the tensor core (TMEM), P^T
//                            and dS^T by two warpgroups (each 64 of the
//                            step's queries, thread = key), written back to
//                            TMEM in BF16 over the columns they came from;
//                            dV += P^T dO and dK += dS^T Q read them there
//                            as the A operand.
// Both main kernels issue only N = 128 products: on B200 a 128 x 64 x 16
// tcgen05.mma takes 55 cycles against 64 for 128 x 128 x 16, so 64-wide
// steps run the tensor core at about half rate.
// Splitting dQ from dK/dV costs a second Q K^T and dO V^T but needs no
// atomics: every output element is written once, by one CTA, and the result
// is bit-for-bit reproducible.
#pragma once

#include <type_traits>

#include "attn_common.cuh"

namespace sdpa10 {
namespace bwd {

struct BwdParams {
    int batch, h_q, h_kv, s_q, s_k;
    int group;             // h_q / h_kv
    int n_qb;              // ceil(s_q / 128)   (dQ kernel)
    int n_kb;              // ceil(s_k / 128)
    int s_q_pad;           // row stride of the L / D workspace: n_qb * 128
    int causal;
    int causal_offset;     // s_k - s_q
    int window_left;       // -1: none
    int num_items;
    // Items are grouped in sections of `section` heads ((batch, query head)
    // for dQ, (batch, key/value head) for dK/dV): inside a section the order
    // is longest first, then head, so the CTAs running at one time share the
    // few heads whose streamed tiles stay in L2.  section = all heads when
    // the launch has too few items to balance per section.
    int section;
    FastDiv div_n_qb;      // n_qb
    FastDiv div_n_kb;      // n_kb
    FastDiv div_h_q;       // h_q
    FastDiv div_h_kv;      // h_kv
    float scale;           // dQ, dK factor
    float scale_log2;      // scale * log2(e)
    const float* NL;       // [batch][h_q][s_q_pad]  -LSE * log2(e) (-inf padding)
    const float* D;        // [batch][h_q][s_q_pad]  rowsum(dO * O) (0 padding)
    __nv_bfloat16* dk;     // [batch][s_k][h_kv][128] outputs of the dK/dV kernel
    __nv_bfloat16* dv;
    unsigned long long timeout_ns;
    unsigned int* status;
};

// ------------------------------------------------------------------ prep
// One warp per query row: D = sum_c dO[c] O[c] (BF16 in, FP32 sum) and
// -L = -LSE * log2(e) (stored negated so the exponent 2^(S c - L) is one
// fused multiply-add); the rows s_q .. s_q_pad - 1 of each head get
// -L = -inf and D = 0.
struct PrepParams {
    const __nv_bfloat16* o;
    const __nv_bfloat16* dout;
    const float* lse;
    float* NL;
    float* D;
    int batch, h_q, s_q, s_q_pad;
};

constexpr int kPrepThreads = 256;

__global__ void __launch_bounds__(kPrepThreads) attn_bwd_prep_kernel(const PrepParams a) {
    const int lane = threadIdx.x & 31;
    const size_t rows = static_cast<size_t>(a.batch) * a.h_q * a.s_q_pad;
    const size_t warps = static_cast<size_t>(gridDim.x) * (kPrepThreads / 32);
    for (size_t r = blockIdx.x * static_cast<size_t>(kPrepThreads / 32) + (threadIdx.x >> 5);
         r < rows; r += warps) {
        const size_t bh = r / a.s_q_pad;
        const int i = static_cast<int>(r - bh * a.s_q_pad);
        if (i >= a.s_q) {
            if (lane == 0) {
                a.NL[r] = -CUDART_INF_F;
                a.D[r] = 0.f;
            }
            continue;
        }
        const int h = static_cast<int>(bh % a.h_q);
        const size_t b = bh / a.h_q;
        const size_t off = ((b * a.s_q + i) * a.h_q + h) * kHeadDim + lane * 4;
        const uint2 ov = *reinterpret_cast<const uint2*>(a.o + off);
        const uint2 dv = *reinterpret_cast<const uint2*>(a.dout + off);
        const __nv_bfloat162* o2 = reinterpret_cast<const __nv_bfloat162*>(&ov);
        const __nv_bfloat162* d2 = reinterpret_cast<const __nv_bfloat162*>(&dv);
        float acc = 0.f;
#pragma unroll
        for (int k = 0; k < 2; ++k) {
            const float2 of = __bfloat1622float2(o2[k]);
            const float2 df = __bfloat1622float2(d2[k]);
            acc = fmaf(of.x, df.x, acc);
            acc = fmaf(of.y, df.y, acc);
        }
#pragma unroll
        for (int sh = 16; sh > 0; sh >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, sh);
        if (lane == 0) {
            a.D[r] = acc;
            a.NL[r] = a.lse[bh * a.s_q + i] * -1.4426950408889634f;
        }
    }
}

// ------------------------------------------------------------------ dQ kernel
namespace dq {

// Two compute warpgroups (warps 0-3 and 4-7) split each 128-key step by
// columns: warpgroup w takes keys 64w .. 64w + 63 of every row, so each row's
// exponentials and dS run on two warps per SM sub-partition; warp 8 is the
// TMA producer and warp 9 the MMA issuer.
constexpr int kThreads = 320;
constexpr int kLoadWarp = 8;
constexpr int kMmaWarp = 9;

struct Smem {
    static constexpr int kQ = 0;                       // Q tile  (A of S = Q K^T)
    static constexpr int kDO = kTileBytes;             // dO tile (A of dP = dO V^T)
    static constexpr int kOut = 2 * kTileBytes;        // dQ staging for the TMA store
    static constexpr int kK = 3 * kTileBytes;          // K ring (2)
    static constexpr int kV = 5 * kTileBytes;          // V ring (2)
    static constexpr int kBars = 7 * kTileBytes;
    static constexpr int bQFull = 0, bQEmpty = 1, bKFull = 2, bKEmpty = 4, bVFull = 6,
                         bVEmpty = 8, bSFull = 10, bSFree = 11, bPFull = 12, bPFree = 13,
                         bDsFull = 14, bDsFree = 15, bDqFull = 16, bDqFree = 17,
                         bStaged = 18, bStored = 19, bDrain = 20, kNumBars = 21;
    static constexpr int kTmemSlot = kBars + kNumBars * 8;
    static constexpr int kAbort = kTmemSlot + 4;
    static constexpr int kBytes = kAbort + 4;
    static constexpr int kAlloc = kBytes + 1024;
};
constexpr int kStages = 2;

// Item t -> (batch, query head, query block): by section of heads, then
// query block descending (longest causal work first), then head.
struct Cursor {
    int round, t;
    int b, h, g, qb, n;  // n: key blocks visited
    int kb_lo;           // first key block (sliding window)
    __device__ __forceinline__ void decode(const BwdParams& p) {
        // Once per item: plain divisions are fine.
        const int bh_count = p.batch * p.h_q;
        const int per_sec = p.section * p.n_qb;
        const int sec = t / per_sec;
        const int in_sec = min(p.section, bh_count - sec * p.section);  // heads in this section
        const int r = t - sec * per_sec;
        const int rank = r / in_sec;
        const int bh = sec * p.section + (r - rank * in_sec);
        qb = p.n_qb - 1 - rank;
        b = p.div_h_q.div(bh);
        h = bh - b * p.h_q;
        g = h / p.group;
        const int last_row = min(qb * kBlockM + kBlockM - 1, p.s_q - 1);
        int hi = p.n_kb;
        if (p.causal) hi = min(hi, ((last_row + p.causal_offset) >> 7) + 1);
        kb_lo = 0;
        if (p.window_left >= 0)
            kb_lo = max(0, (qb * kBlockM + p.causal_offset - p.window_left) >> 7);
        n = max(0, hi - kb_lo);
    }
    __device__ __forceinline__ void settle(const BwdParams& p) {
        for (;; ++round) {
            const int c = static_cast<int>(blockIdx.x), G = static_cast<int>(gridDim.x);
            t = round * G + ((round & 1) ? G - 1 - c : c);
            if (t >= p.num_items) return;
            decode(p);
            if (n > 0) return;
        }
    }
    __device__ __forceinline__ void start(const BwdParams& p) { round = 0; settle(p); }
    __device__ __forceinline__ void next(const BwdParams& p) { ++round; settle(p); }
    __device__ __forceinline__ bool valid(const BwdParams& p) const { return t < p.num_items; }
};

__global__ void __launch_bounds__(kThreads, 1)
    attn_bwd_dq_kernel(const __grid_constant__ CUtensorMap tm_q,
                       const __grid_constant__ CUtensorMap tm_k,
                       const __grid_constant__ CUtensorMap tm_v,
                       const __grid_constant__ CUtensorMap tm_do,
                       const __grid_constant__ CUtensorMap tm_dq,
                       const __grid_constant__ BwdParams p) {
    using L = Smem;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    const uint32_t sbase = ptx::smem_u32(smem);
    const uint32_t bars = sbase + L::kBars;
    auto bar = [&](int i) -> uint32_t { return bars + 8u * static_cast<uint32_t>(i); };
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kAbort);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kTmemSlot);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        ptx::mbar_init(bar(L::bQFull), 1);
        ptx::mbar_init(bar(L::bQEmpty), 1);
        for (int i = 0; i < kStages; ++i) {
            ptx::mbar_init(bar(L::bKFull + i), 1);
            ptx::mbar_init(bar(L::bKEmpty + i), 1);
            ptx::mbar_init(bar(L::bVFull + i), 1);
            ptx::mbar_init(bar(L::bVEmpty + i), 1);
        }
        ptx::mbar_init(bar(L::bSFull), 1);
        ptx::mbar_init(bar(L::bSFree), 8);  // both compute warpgroups, 4 warps each
        ptx::mbar_init(bar(L::bPFull), 1);   // dP in TMEM
        ptx::mbar_init(bar(L::bPFree), 8);
        ptx::mbar_init(bar(L::bDsFull), 8);
        ptx::mbar_init(bar(L::bDsFree), 1);
        ptx::mbar_init(bar(L::bDqFull), 1);
        ptx::mbar_init(bar(L::bDqFree), 8);
        ptx::mbar_init(bar(L::bStaged), 8);
        ptx::mbar_init(bar(L::bStored), 1);
        ptx::mbar_init(bar(L::bDrain), 1);
        *abort_flag = 0;
        ptx::fence_mbar_init();
    }
    if (warp == kLoadWarp && lane == 0) {
        ptx::prefetch_tmap(&tm_q);
        ptx::prefetch_tmap(&tm_k);
        ptx::prefetch_tmap(&tm_v);
        ptx::prefetch_tmap(&tm_do);
        ptx::prefetch_tmap(&tm_dq);
    }
    if (warp == kMmaWarp) {
        ptx::tmem_alloc(ptx::smem_u32(tmem_slot), kTmemCols);
        ptx::tmem_relinquish();
    }
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    const uint32_t tmem = *tmem_slot;  // S | dP | dQ | dS at columns 0, 128, 256, 384
    const WaitCtx wc{abort_flag, p.status, p.timeout_ns};

    if (warp == kLoadWarp) {
        // ============================================================ producer
        if (lane == 0) {
            const uint64_t pol_kv = ptx::policy_evict_last();
            const uint64_t pol_q = ptx::policy_evict_first();
            uint32_t k_loads = 0, v_loads = 0, q_loads = 0;
            bool ok = true;
            auto tile = [&](const CUtensorMap* tm, uint32_t dst, uint32_t full, int c1, int row,
                            int bb, uint64_t pol) {
                ptx::tma_load_4d(dst, tm, full, 0, c1, row, bb, pol);
                ptx::tma_load_4d(dst + kHalfTileBytes, tm, full, 64, c1, row, bb, pol);
            };
            Cursor c;
            for (c.start(p); ok && c.valid(p); c.next(p)) {
                if (!(ok = wait_bar(bar(L::bQEmpty), (q_loads & 1) ^ 1, wc))) break;
                ptx::mbar_arrive_expect_tx(bar(L::bQFull), 2 * kTileBytes);
                tile(&tm_q, sbase + L::kQ, bar(L::bQFull), c.h, c.qb * kBlockM, c.b, pol_q);
                tile(&tm_do, sbase + L::kDO, bar(L::bQFull), c.h, c.qb * kBlockM, c.b, pol_q);
                ++q_loads;
                for (int j = 0; j < c.n && ok; ++j) {
                    const int key0 = (c.kb_lo + j) * kBlockN;
                    const int ks = k_loads % kStages, vs = v_loads % kStages;
                    if (!(ok = wait_bar(bar(L::bKEmpty + ks), ((k_loads / kStages) & 1) ^ 1, wc)))
                        break;
                    ptx::mbar_arrive_expect_tx(bar(L::bKFull + ks), kTileBytes);
                    tile(&tm_k, sbase + L::kK + ks * kTileBytes, bar(L::bKFull + ks), c.g, key0,
                         c.b, pol_kv);
                    ++k_loads;
                    if (!(ok = wait_bar(bar(L::bVEmpty + vs), ((v_loads / kStages) & 1) ^ 1, wc)))
                        break;
                    ptx::mbar_arrive_expect_tx(bar(L::bVFull + vs), kTileBytes);
                    tile(&tm_v, sbase + L::kV + vs * kTileBytes, bar(L::bVFull + vs), c.g, key0,
                         c.b, pol_kv);
                    ++v_loads;
                }
            }
            // Drain: every issued copy lands before the CTA may exit.
            for (int i = 0; i < kStages && i < static_cast<int>(k_loads); ++i) {
                const uint32_t f = k_loads - 1 - i;
                wait_slow(bar(L::bKFull + f % kStages), (f / kStages) & 1, wc, false);
            }
            for (int i = 0; i < kStages && i < static_cast<int>(v_loads); ++i) {
                const uint32_t f = v_loads - 1 - i;
                wait_slow(bar(L::bVFull + f % kStages), (f / kStages) & 1, wc, false);
            }
            if (q_loads > 0) wait_slow(bar(L::bQFull), (q_loads - 1) & 1, wc, false);
        }
        __syncwarp();
    } else if (warp == kMmaWarp) {
        // ============================================================ MMA issuer
        // The whole warp runs the issue loop; one elected lane issues.
        {
            constexpr uint32_t kIdS = idesc_bf16_f32(kBlockM, kBlockN, 0, 0);    // Q K^T, dO V^T
            constexpr uint32_t kIdDq = idesc_bf16_f32(kBlockM, kHeadDim, 0, 1);  // dS K (K MN-major)
            const uint32_t q_lo = desc_lo_sw128(sbase + L::kQ, 16);
            const uint32_t do_lo = desc_lo_sw128(sbase + L::kDO, 16);
            const uint32_t k_lo = desc_lo_sw128(sbase + L::kK, 16);
            const uint32_t kmn_lo = desc_lo_sw128(sbase + L::kK, kHalfTileBytes);
            const uint32_t v_lo = desc_lo_sw128(sbase + L::kV, 16);
            // TMEM: S | dP | dQ | dS (BF16, the A operand of dQ += dS K) at
            // columns 0, 128, 256, 384.
            const uint32_t s_tm = tmem, dp_tm = tmem + 128, dq_tm = tmem + 256, ds_tm = tmem + 384;
            uint32_t k_used = 0, v_used = 0, items = 0, steps = 0;
            bool ok = true;
            // K-major operands: 8 K-steps of 16 BF16 (32 bytes) inside a
            // 64-column half; the second half is 16 KiB on.
            auto gemm_kmajor = [&](uint32_t d_tm, uint32_t a_lo, uint32_t b_lo) {
#pragma unroll
                for (int k = 0; k < kHeadDim / 16; ++k) {
                    const uint32_t off = ((k >> 2) * kHalfTileBytes + (k & 3) * 32) >> 4;
                    ptx::mma_ss_warp(d_tm, desc_from_lo(a_lo + off), desc_from_lo(b_lo + off), kIdS,
                                k > 0 ? 1u : 0u);
                }
            };
            // Per item: S(0), dP(0), then per key block j: S(j+1), dQ(j),
            // dP(j+1) -- the next scores run under this block's exponentials
            // and dQ(j) runs while the compute warps start on block j + 1.
            auto scores = [&](uint32_t gs) -> bool {
                const uint32_t ks = k_used % kStages;
                if (!wait_bar_warp(bar(L::bKFull + ks), (k_used / kStages) & 1, wc)) return false;
                if (gs > 0 && !wait_bar_warp(bar(L::bSFree), (gs - 1) & 1, wc)) return false;
                ptx::tc_fence_after();
                gemm_kmajor(s_tm, q_lo, k_lo + ((ks * kTileBytes) >> 4));
                ptx::mma_commit_warp(bar(L::bSFull));
                ++k_used;  // K(j) stays in its slot until dQ(j) has read it
                return true;
            };
            auto dprobs = [&](uint32_t gs) -> bool {
                const uint32_t vs = v_used % kStages;
                if (!wait_bar_warp(bar(L::bVFull + vs), (v_used / kStages) & 1, wc)) return false;
                if (gs > 0 && !wait_bar_warp(bar(L::bPFree), (gs - 1) & 1, wc)) return false;
                ptx::tc_fence_after();
                gemm_kmajor(dp_tm, do_lo, v_lo + ((vs * kTileBytes) >> 4));
                ptx::mma_commit_warp(bar(L::bPFull));
                ptx::mma_commit_warp(bar(L::bVEmpty + vs));
                ++v_used;
                return true;
            };
            uint32_t k_freed = 0;  // K tiles released after their dQ
            Cursor c;
            for (c.start(p); ok && c.valid(p); c.next(p)) {
                if (!(ok = wait_bar_warp(bar(L::bQFull), items & 1, wc))) break;
                // dQ of the previous item must have been read out of TMEM.
                if (items > 0 && !(ok = wait_bar_warp(bar(L::bDqFree), (items - 1) & 1, wc))) break;
                ++items;
                if (!(ok = scores(steps) && dprobs(steps))) break;
                for (int j = 0; j < c.n && ok; ++j) {
                    const uint32_t gs = steps + j;
                    if (j + 1 < c.n && !(ok = scores(gs + 1))) break;
                    // dQ += dS K once dS is in TMEM.
                    if (!(ok = wait_bar_warp(bar(L::bDsFull), gs & 1, wc))) break;
                    ptx::tc_fence_after();
                    const uint32_t ks = k_freed % kStages;
                    const uint32_t kb = kmn_lo + ((ks * kTileBytes) >> 4);
#pragma unroll
                    for (int k = 0; k < kBlockN / 16; ++k) {
                        // A = dS from TMEM: 16 keys = 8 packed columns per
                        // step (keys 0-63 written by warpgroup 0, 64-127 by
                        // warpgroup 1); B = K, MN-major (head dim contiguous):
                        // 16 keys = 2 KiB per step.
                        ptx::mma_ts_warp(dq_tm, ds_tm + 8 * k,
                                         desc_from_lo(kb + ((k * 2048) >> 4)), kIdDq,
                                         (j > 0 || k > 0) ? 1u : 0u);
                    }
                    ptx::mma_commit_warp(bar(L::bDsFree));
                    ptx::mma_commit_warp(bar(L::bKEmpty + ks));
                    ++k_freed;
                    if (j + 1 < c.n && !(ok = dprobs(gs + 1))) break;
                }
                if (!ok) break;
                steps += c.n;
                ptx::mma_commit_warp(bar(L::bQEmpty));
                ptx::mma_commit_warp(bar(L::bDqFull));
            }
            ptx::mma_commit_warp(bar(L::bDrain));
            wait_slow(bar(L::bDrain), 0, wc, false);
        }
        __syncwarp();
    } else {
        // ============================================================ compute
        // Warpgroup `half` = warp / 4 takes columns 64 half .. 64 half + 63 of S, dP, dS
        // and dQ; thread r owns query row r of the block (TMEM lane r).
        const int half = warp >> 2;
        const int r = (warp & 3) * 32 + lane;
        const uint32_t lane_base = static_cast<uint32_t>((warp & 3) * 32) << 16;
        const uint32_t s_tm = tmem + lane_base + 64 * half,
                       dp_tm = tmem + lane_base + 128 + 64 * half,
                       dq_tm = tmem + lane_base + 256 + 64 * half,
                       ds_tm = tmem + lane_base + 384 + 32 * half;
        // This row's half of the dQ staging tile: the tile's 64-column half
        // `half` (16 KiB), chunk k of the half at ((k ^ (r % 8)) * 16).
        const uint32_t out_row =
            sbase + L::kOut + half * kHalfTileBytes + (r >> 3) * 1024 + (r & 7) * 128;
        const uint32_t xr = static_cast<uint32_t>(r & 7);
        const float c2 = p.scale_log2;
        const uint64_t c2c2 = ptx::f2_pack(c2, c2);
        uint32_t items = 0, steps = 0;
        Cursor c;
        for (c.start(p); c.valid(p); c.next(p)) {
            const int row = c.qb * kBlockM + r;
            const size_t stat = (static_cast<size_t>(c.b) * p.h_q + c.h) * p.s_q_pad + row;
            const float NLr = p.NL[stat];  // -inf past s_q: P = 0
            const float Dr = p.D[stat];
            const uint64_t nl2 = ptx::f2_pack(NLr, NLr), nd2 = ptx::f2_pack(-Dr, -Dr);
            for (int j = 0; j < c.n; ++j, ++steps) {
                const int kv0 = (c.kb_lo + j) * kBlockN + 64 * half;  // this half's first key
                // Visible keys of this row inside the block: [lo, hi).
                int hi = min(64, p.s_k - kv0);
                if (p.causal) hi = min(hi, row + p.causal_offset - kv0 + 1);
                int lo = 0;
                if (p.window_left >= 0) lo = row + p.causal_offset - p.window_left - kv0;
                float pr[64];
                if (!wait_bar_warp(bar(L::bSFull), steps & 1, wc)) return;
                ptx::tc_fence_after();
#pragma unroll
                for (int q = 0; q < 2; ++q) {
                    uint32_t sr[32];
                    ptx::tmem_ld32(s_tm + q * 32, sr);
                    ptx::tmem_wait_ld();
#pragma unroll
                    for (int k = 0; k < 32; ++k) pr[q * 32 + k] = __uint_as_float(sr[k]);
                }
                ptx::tc_fence_before();
                __syncwarp();
                if (lane == 0) ptx::mbar_arrive(bar(L::bSFree));
                // P = 2^(S c - L), pairs of columns in packed FP32; the mask
                // is applied only where some row of the warp needs it (the
                // diagonal and ragged blocks).
                auto exps = [&](auto mask_tag) {
                    constexpr bool kMask = decltype(mask_tag)::value;
#pragma unroll
                    for (int k = 0; k < 64; k += 2) {
                        float x0, x1;
                        ptx::f2_unpack(ptx::f2_fma(ptx::f2_pack(pr[k], pr[k + 1]), c2c2, nl2), x0, x1);
                        x0 = ptx::ex2(x0);
                        x1 = ptx::ex2(x1);
                        if (kMask) {
                            x0 = (k >= lo && k < hi) ? x0 : 0.f;
                            x1 = (k + 1 >= lo && k + 1 < hi) ? x1 : 0.f;
                        }
                        pr[k] = x0;
                        pr[k + 1] = x1;
                    }
                };
                if (__any_sync(0xffffffffu, lo > 0 || hi < 64))
                    exps(std::true_type{});
                else
                    exps(std::false_type{});
                // dS = P (dP - D) -> BF16 pairs, into this warpgroup's 32
                // TMEM columns of dS (its 64 keys, the A operand of dQ).
                if (!wait_bar_warp(bar(L::bPFull), steps & 1, wc)) return;
                if (steps > 0 && !wait_bar_warp(bar(L::bDsFree), (steps - 1) & 1, wc)) return;
                ptx::tc_fence_after();
                uint32_t ds[32];
#pragma unroll
                for (int q = 0; q < 2; ++q) {
                    uint32_t dr[32];
                    ptx::tmem_ld32(dp_tm + q * 32, dr);
                    ptx::tmem_wait_ld();
#pragma unroll
                    for (int k = 0; k < 16; ++k) {
                        const uint64_t t = ptx::f2_add(
                            ptx::f2_pack(__uint_as_float(dr[2 * k]), __uint_as_float(dr[2 * k + 1])), nd2);
                        float a, b2;
                        ptx::f2_unpack(ptx::f2_mul(ptx::f2_pack(pr[q * 32 + 2 * k], pr[q * 32 + 2 * k + 1]), t),
                                       a, b2);
                        ds[q * 16 + k] = ptx::pack_bf16x2(a, b2);
                    }
                }
                ptx::tmem_st32(ds_tm, ds);
                ptx::tmem_wait_st();
                ptx::tc_fence_before();
                __syncwarp();
                if (lane == 0) {
                    ptx::mbar_arrive(bar(L::bPFree));
                    ptx::mbar_arrive(bar(L::bDsFull));
                }
            }
            // Epilogue: dQ * scale -> BF16 rows, each warpgroup its 64
            // columns, staged in its half of the staging tile and stored
            // with TMA.
            if (!wait_bar_warp(bar(L::bDqFull), items & 1, wc)) return;
            ptx::tc_fence_after();
#pragma unroll
            for (int q = 0; q < 2; ++q) {
                uint32_t v[32];
                ptx::tmem_ld32(dq_tm + q * 32, v);
                ptx::tmem_wait_ld();
                uint32_t w[16];
#pragma unroll
                for (int k = 0; k < 16; ++k)
                    w[k] = ptx::pack_bf16x2(__uint_as_float(v[2 * k]) * p.scale,
                                            __uint_as_float(v[2 * k + 1]) * p.scale);
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    const int cc = 4 * q + k;
                    ptx::st_shared_v4(out_row + ((cc ^ xr) << 4), w[4 * k], w[4 * k + 1],
                                      w[4 * k + 2], w[4 * k + 3]);
                }
            }
            ptx::tc_fence_before();
            ptx::fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) {
                ptx::mbar_arrive(bar(L::bDqFree));
                ptx::mbar_arrive(bar(L::bStaged));
            }
            if (warp == 0 && lane == 0) {
                if (!wait_bar(bar(L::bStaged), items & 1, wc)) return;
                ptx::tma_store_4d(&tm_dq, sbase + L::kOut, 0, c.h, c.qb * kBlockM, c.b);
                ptx::tma_store_4d(&tm_dq, sbase + L::kOut + kHalfTileBytes, 64, c.h,
                                  c.qb * kBlockM, c.b);
                ptx::bulk_commit_group();
                ptx::bulk_wait_group_read0();
                ptx::mbar_arrive(bar(L::bStored));
            }
            // The staging tile is rewritten by the next item only after TMA
            // has read the staged rows.
            if (!wait_bar_warp(bar(L::bStored), items & 1, wc)) return;
            ++items;
        }
        if (warp == 0 && lane == 0) ptx::bulk_wait_group0();
    }

    ptx::tc_fence_before();
    __syncthreads();
    if (warp == kMmaWarp) {
        ptx::tc_fence_after();
        ptx::tmem_dealloc(tmem, kTmemCols);
    }
}

}  // namespace dq
}  // namespace bwd
}  // namespace sdpa10

namespace sdpa10 {
namespace bwd {
namespace dkdv {

// Two compute warpgroups split every 128-query step by columns: warpgroup w
// takes queries 64w .. 64w + 63 of the step for all 128 keys of the block
// (thread = key = TMEM lane).  Warp 8 is the TMA producer, warp 9 the MMA
// issuer.
constexpr int kThreads = 320;
constexpr int kLoadWarp = 8;
constexpr int kMmaWarp = 9;
constexpr int kStages = 2;  // slots of the Q ring and of the dO ring

struct Smem {
    static constexpr int kK = 0;                             // K tile (A of S^T = K Q^T)
    static constexpr int kV = kTileBytes;                    // V tile (A of dP^T = V dO^T)
    static constexpr int kQ = 2 * kTileBytes;                // ring of Q tiles (128 rows)
    static constexpr int kDO = kQ + kStages * kTileBytes;    // ring of dO tiles
    static constexpr int kLD = kDO + kStages * kTileBytes;   // per Q slot: -L[128], D[128]
    static constexpr int kLDSlot = 2 * kBlockM * 4;
    static constexpr int kBars = kLD + kStages * kLDSlot;
    static constexpr int bKFull = 0, bKEmpty = 1, bVFull = 2, bVEmpty = 3, bQFull = 4,
                         bQEmpty = bQFull + kStages, bOFull = bQEmpty + kStages,
                         bOEmpty = bOFull + kStages, bSFull = bOEmpty + kStages,
                         bPFull = bSFull + 1, bPTFull = bPFull + 1, bDSTFull = bPTFull + 1,
                         bAccFull = bDSTFull + 1, bAccFree = bAccFull + 1, bDrain = bAccFree + 1,
                         kNumBars = bDrain + 1;
    static constexpr int kTmemSlot = kBars + kNumBars * 8;
    static constexpr int kAbort = kTmemSlot + 4;
    static constexpr int kBytes = kAbort + 4;
    static constexpr int kAlloc = kBytes + 1024;
};
static_assert(Smem::kAlloc <= 232448, "dK/dV shared memory exceeds the per-CTA limit");

// TMEM columns: S^T at 0 (P^T in BF16 over its first half of each
// warpgroup's 64 columns), dP^T at 128 (dS^T likewise), dV at 256, dK at 384.
constexpr uint32_t kTmS = 0, kTmDP = 128, kTmDV = 256, kTmDK = 384;

// Item t -> (key block, batch, key/value head): by section of heads, then
// key block ascending (under the causal mask the first key blocks are seen
// by the most query rows: longest first), then head.  The item walks the
// query heads of the group and, for each, the 128-row query blocks that see
// the key block.
struct Cursor {
    int round, t;
    int b, g, kb;
    int qlo, nq;  // query blocks qlo .. qlo + nq - 1 per head
    __device__ __forceinline__ void decode(const BwdParams& p) {
        const int bg_count = p.batch * p.h_kv;
        const int per_sec = p.section * p.n_kb;
        const int sec = t / per_sec;
        const int in_sec = min(p.section, bg_count - sec * p.section);
        const int r = t - sec * per_sec;
        kb = r / in_sec;
        const int bg = sec * p.section + (r - kb * in_sec);
        b = p.div_h_kv.div(bg);
        g = bg - b * p.h_kv;
        int lo = 0, hi = p.n_qb;
        if (p.causal) {
            // Query i sees key 128 kb (the block's first key) iff
            // i >= 128 kb - causal_offset: floor division by 128.
            lo = max(0, (kb * kBlockN - p.causal_offset) >> 7);
        }
        if (p.window_left >= 0) {
            // Query i still sees the block's last key iff
            // i <= 128 kb + 127 + window_left - causal_offset.
            const int last = kb * kBlockN + kBlockN - 1 + p.window_left - p.causal_offset;
            hi = min(hi, (last >> 7) + 1);
        }
        qlo = lo;
        nq = max(0, hi - lo);
    }
    __device__ __forceinline__ void settle(const BwdParams& p) {
        for (;; ++round) {
            const int c = static_cast<int>(blockIdx.x), G = static_cast<int>(gridDim.x);
            t = round * G + ((round & 1) ? G - 1 - c : c);
            if (t >= p.num_items) return;
            decode(p);
            if (nq > 0) return;
        }
    }
    __device__ __forceinline__ void start(const BwdParams& p) { round = 0; settle(p); }
    __device__ __forceinline__ void next(const BwdParams& p) { ++round; settle(p); }
    __device__ __forceinline__ bool valid(const BwdParams& p) const { return t < p.num_items; }
    __device__ __forceinline__ int steps(const BwdParams& p) const { return p.group * nq; }
    // Query head and query block of step s.
    __device__ __forceinline__ void step(const BwdParams& p, int s, int& h, int& qb) const {
        const int hl = s / nq;
        qb = qlo + (s - hl * nq);
        h = g * p.group + hl;
    }
};

// A key block that no query sees has no item in the main loop (nq = 0):
// under a sliding window with s_q < s_k the keys before the first query's
// window are such blocks.  Their dK and dV rows are zero (no weight reaches
// them).  The CTAs share the items by a grid stride (each item t is
// visited by CTA t mod gridDim.x alone) and write the rows of those with
// nq = 0; the main loop never touches these rows.
__device__ __noinline__ void zero_unseen_key_blocks(const BwdParams& p) {
    constexpr int kPieces = kHeadDim * 2 / 16;  // 16-byte pieces of one row
    Cursor c;
    for (int t = static_cast<int>(blockIdx.x); t < p.num_items;
         t += static_cast<int>(gridDim.x)) {
        c.t = t;
        c.decode(p);
        if (c.nq > 0) continue;
        const int r0 = c.kb * kBlockN;
        const int rows = min(kBlockN, p.s_k - r0);
        for (int i = static_cast<int>(threadIdx.x); i < rows * kPieces;
             i += static_cast<int>(blockDim.x)) {
            const int row = r0 + i / kPieces;
            const size_t e = ((static_cast<size_t>(c.b) * p.s_k + row) * p.h_kv + c.g) * kHeadDim +
                             static_cast<size_t>(i % kPieces) * 8;
            *reinterpret_cast<uint4*>(p.dk + e) = make_uint4(0u, 0u, 0u, 0u);
            *reinterpret_cast<uint4*>(p.dv + e) = make_uint4(0u, 0u, 0u, 0u);
        }
    }
}

__global__ void __launch_bounds__(kThreads, 1)
    attn_bwd_dkdv_kernel(const __grid_constant__ CUtensorMap tm_q,
                         const __grid_constant__ CUtensorMap tm_k,
                         const __grid_constant__ CUtensorMap tm_v,
                         const __grid_constant__ CUtensorMap tm_do,
                         const __grid_constant__ BwdParams p) {
    using L = Smem;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    const uint32_t sbase = ptx::smem_u32(smem);
    const uint32_t bars = sbase + L::kBars;
    auto bar = [&](int i) -> uint32_t { return bars + 8u * static_cast<uint32_t>(i); };
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kAbort);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kTmemSlot);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    if (p.window_left >= 0) zero_unseen_key_blocks(p);
    if (threadIdx.x == 0) {
        ptx::mbar_init(bar(L::bKFull), 1);
        ptx::mbar_init(bar(L::bKEmpty), 1);
        ptx::mbar_init(bar(L::bVFull), 1);
        ptx::mbar_init(bar(L::bVEmpty), 1);
        for (int i = 0; i < kStages; ++i) {
            ptx::mbar_init(bar(L::bQFull + i), 1);
            ptx::mbar_init(bar(L::bQEmpty + i), 1);
            ptx::mbar_init(bar(L::bOFull + i), 1);
            ptx::mbar_init(bar(L::bOEmpty + i), 1);
        }
        ptx::mbar_init(bar(L::bSFull), 1);
        ptx::mbar_init(bar(L::bPFull), 1);
        ptx::mbar_init(bar(L::bPTFull), 8);   // every compute warp has written P^T
        ptx::mbar_init(bar(L::bDSTFull), 8);  // ... dS^T
        ptx::mbar_init(bar(L::bAccFull), 1);
        ptx::mbar_init(bar(L::bAccFree), 8);  // every compute warp has read dV / dK
        ptx::mbar_init(bar(L::bDrain), 1);
        *abort_flag = 0;
        ptx::fence_mbar_init();
    }
    if (warp == kLoadWarp && lane == 0) {
        ptx::prefetch_tmap(&tm_q);
        ptx::prefetch_tmap(&tm_k);
        ptx::prefetch_tmap(&tm_v);
        ptx::prefetch_tmap(&tm_do);
    }
    if (warp == kMmaWarp) {
        ptx::tmem_alloc(ptx::smem_u32(tmem_slot), kTmemCols);
        ptx::tmem_relinquish();
    }
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const WaitCtx wc{abort_flag, p.status, p.timeout_ns};
    auto q_addr = [&](uint32_t u) { return sbase + L::kQ + (u % kStages) * kTileBytes; };
    auto do_addr = [&](uint32_t u) { return sbase + L::kDO + (u % kStages) * kTileBytes; };

    if (warp == kLoadWarp) {
        // ============================================================ producer
        // Per item: K, Q of its first step, V, dO of its first step, then Q
        // and dO of the following steps; K (V) of the next item is loaded as
        // soon as the last S^T (dP^T) of this one has been read.
        if (lane == 0) {
            const uint64_t pol_kv = ptx::policy_evict_first();
            const uint64_t pol_q = ptx::policy_evict_last();
            uint32_t items = 0, loads = 0;
            bool ok = true;
            auto load_q = [&](const Cursor& c, int s) -> bool {
                int h, qb;
                c.step(p, s, h, qb);
                const uint32_t slot = loads % kStages;
                if (!wait_bar(bar(L::bQEmpty + slot), ((loads / kStages) & 1) ^ 1, wc)) return false;
                const uint32_t full = bar(L::bQFull + slot);
                ptx::mbar_arrive_expect_tx(full, kTileBytes + L::kLDSlot);
#pragma unroll
                for (int half = 0; half < 2; ++half)
                    ptx::tma_load_4d(q_addr(loads) + half * kHalfTileBytes, &tm_q, full, 64 * half,
                                     h, qb * kBlockM, c.b, pol_q);
                const size_t stat =
                    (static_cast<size_t>(c.b) * p.h_q + h) * p.s_q_pad + qb * kBlockM;
                const uint32_t ld = sbase + L::kLD + slot * L::kLDSlot;
                ptx::bulk_load(ld, p.NL + stat, kBlockM * 4, full);
                ptx::bulk_load(ld + kBlockM * 4, p.D + stat, kBlockM * 4, full);
                return true;
            };
            auto load_do = [&](const Cursor& c, int s) -> bool {
                int h, qb;
                c.step(p, s, h, qb);
                const uint32_t slot = loads % kStages;
                if (!wait_bar(bar(L::bOEmpty + slot), ((loads / kStages) & 1) ^ 1, wc)) return false;
                const uint32_t full = bar(L::bOFull + slot);
                ptx::mbar_arrive_expect_tx(full, kTileBytes);
#pragma unroll
                for (int half = 0; half < 2; ++half)
                    ptx::tma_load_4d(do_addr(loads) + half * kHalfTileBytes, &tm_do, full,
                                     64 * half, h, qb * kBlockM, c.b, pol_q);
                return true;
            };
            Cursor c;
            for (c.start(p); ok && c.valid(p); c.next(p)) {
                const uint32_t ph = (items & 1) ^ 1;
                if (!(ok = wait_bar(bar(L::bKEmpty), ph, wc))) break;
                ptx::mbar_arrive_expect_tx(bar(L::bKFull), kTileBytes);
#pragma unroll
                for (int half = 0; half < 2; ++half)
                    ptx::tma_load_4d(sbase + L::kK + half * kHalfTileBytes, &tm_k, bar(L::bKFull),
                                     64 * half, c.g, c.kb * kBlockN, c.b, pol_kv);
                if (!(ok = load_q(c, 0))) break;
                if (!(ok = wait_bar(bar(L::bVEmpty), ph, wc))) break;
                ptx::mbar_arrive_expect_tx(bar(L::bVFull), kTileBytes);
#pragma unroll
                for (int half = 0; half < 2; ++half)
                    ptx::tma_load_4d(sbase + L::kV + half * kHalfTileBytes, &tm_v, bar(L::bVFull),
                                     64 * half, c.g, c.kb * kBlockN, c.b, pol_kv);
                if (!(ok = load_do(c, 0))) break;
                ++loads;
                ++items;
                const int n = c.steps(p);
                for (int s = 1; s < n && ok; ++s) {
                    if (!(ok = load_q(c, s))) break;
                    if (!(ok = load_do(c, s))) break;
                    ++loads;
                }
            }
            // Let every issued copy land before the CTA can exit.
            if (items > 0) {
                wait_slow(bar(L::bKFull), (items - 1) & 1, wc, false);
                wait_slow(bar(L::bVFull), (items - 1) & 1, wc, false);
            }
            for (int i = 0; i < kStages && i < static_cast<int>(loads); ++i) {
                const uint32_t f = loads - 1 - i;
                wait_slow(bar(L::bQFull + f % kStages), (f / kStages) & 1, wc, false);
                wait_slow(bar(L::bOFull + f % kStages), (f / kStages) & 1, wc, false);
            }
        }
        __syncwarp();
    } else if (warp == kMmaWarp) {
        // ============================================================ MMA issuer
        // The whole warp runs the issue loop; one elected lane issues.
        {
            constexpr uint32_t kIdS = idesc_bf16_f32(kBlockN, kBlockM, 0, 0);     // K Q^T, V dO^T
            constexpr uint32_t kIdAcc = idesc_bf16_f32(kBlockN, kHeadDim, 0, 1);  // P^T dO, dS^T Q
            const uint32_t k_lo = desc_lo_sw128(sbase + L::kK, 16);
            const uint32_t v_lo = desc_lo_sw128(sbase + L::kV, 16);
            // X^T = A B^T with A the [128 x 128] K or V tile and B the
            // 128-row Q or dO tile, both K-major: 8 K-steps of 16.
            auto gemm_t = [&](uint32_t d_tm, uint32_t a_lo, uint32_t b_addr) {
                const uint32_t b_lo = desc_lo_sw128(b_addr, 16);
#pragma unroll
                for (int k = 0; k < kHeadDim / 16; ++k) {
                    const uint32_t o = ((k >> 2) * kHalfTileBytes + (k & 3) * 32) >> 4;
                    ptx::mma_ss_warp(d_tm, desc_from_lo(a_lo + o), desc_from_lo(b_lo + o), kIdS,
                                k > 0 ? 1u : 0u);
                }
            };
            // Acc += A B with A = P^T or dS^T [128 keys x 128 queries] in
            // TMEM (queries 0-63 packed in the columns at a_tm, queries
            // 64-127 at a_tm + 64) and B the 128-row Q or dO tile read
            // MN-major: 16 queries = 2 KiB per K-step, head-dim halves 16 KiB
            // apart.
            auto gemm_acc = [&](uint32_t d_tm, uint32_t a_tm, uint32_t b_addr, bool acc) {
                const uint32_t b_lo = desc_lo_sw128(b_addr, kHalfTileBytes);
#pragma unroll
                for (int k = 0; k < kBlockM / 16; ++k)
                    ptx::mma_ts_warp(d_tm, a_tm + (k >> 2) * 64 + (k & 3) * 8,
                                desc_from_lo(b_lo + ((k * 2048) >> 4)), kIdAcc,
                                (acc || k > 0) ? 1u : 0u);
            };
            uint32_t gs = 0, items = 0, kv = 0;
            bool ok = true;
            Cursor c;
            c.start(p);
            // S^T(gs) once K and Q are in; dP^T(gs) once V and dO are in.  A
            // new item's first S^T / dP^T also waits for its K / V; the last
            // S^T / dP^T of an item releases K / V for the next one.
            auto issue_s = [&](uint32_t u, bool first, bool last) -> bool {
                if (first && !wait_bar_warp(bar(L::bKFull), kv & 1, wc)) return false;
                if (!wait_bar_warp(bar(L::bQFull + u % kStages), (u / kStages) & 1, wc)) return false;
                ptx::tc_fence_after();
                gemm_t(tmem + kTmS, k_lo, q_addr(u));
                ptx::mma_commit_warp(bar(L::bSFull));
                if (last) ptx::mma_commit_warp(bar(L::bKEmpty));
                return true;
            };
            auto issue_dp = [&](uint32_t u, bool first, bool last) -> bool {
                if (first && !wait_bar_warp(bar(L::bVFull), kv & 1, wc)) return false;
                if (!wait_bar_warp(bar(L::bOFull + u % kStages), (u / kStages) & 1, wc)) return false;
                ptx::tc_fence_after();
                gemm_t(tmem + kTmDP, v_lo, do_addr(u));
                ptx::mma_commit_warp(bar(L::bPFull));
                if (last) ptx::mma_commit_warp(bar(L::bVEmpty));
                return true;
            };
            if (c.valid(p)) {
                int n = c.steps(p), s = 0;
                ok = issue_s(0, true, n == 1) && issue_dp(0, true, n == 1);
                ++kv;
                while (ok) {
                    // Step gs (step s of n of the current item).  P^T(gs) in
                    // TMEM over S^T: dV += P^T dO.
                    if (!(ok = wait_bar_warp(bar(L::bPTFull), gs & 1, wc))) break;
                    if (s == 0 && items > 0 && !(ok = wait_bar_warp(bar(L::bAccFree), (items - 1) & 1, wc)))
                        break;
                    ptx::tc_fence_after();
                    gemm_acc(tmem + kTmDV, tmem + kTmS, do_addr(gs), s > 0);
                    ptx::mma_commit_warp(bar(L::bOEmpty + gs % kStages));
                    // The next step's S^T overwrites P^T(gs) only after the
                    // dV products above (the tensor core runs in issue order).
                    Cursor cn = c;
                    int sn = s + 1, nn = n;
                    if (sn == n) {
                        cn.next(p);
                        sn = 0;
                        nn = cn.valid(p) ? cn.steps(p) : 0;
                    }
                    const bool more = cn.valid(p);
                    if (more && !(ok = issue_s(gs + 1, sn == 0, sn == nn - 1))) break;
                    // dS^T(gs) in TMEM over dP^T: dK += dS^T Q.
                    if (!(ok = wait_bar_warp(bar(L::bDSTFull), gs & 1, wc))) break;
                    ptx::tc_fence_after();
                    gemm_acc(tmem + kTmDK, tmem + kTmDP, q_addr(gs), s > 0);
                    ptx::mma_commit_warp(bar(L::bQEmpty + gs % kStages));
                    if (s == n - 1) {
                        ptx::mma_commit_warp(bar(L::bAccFull));
                        ++items;
                    }
                    if (more && !(ok = issue_dp(gs + 1, sn == 0, sn == nn - 1))) break;
                    if (!more) break;
                    if (sn == 0) ++kv;
                    c = cn;
                    s = sn;
                    n = nn;
                    ++gs;
                }
            }
            ptx::mma_commit_warp(bar(L::bDrain));
            wait_slow(bar(L::bDrain), 0, wc, false);
        }
        __syncwarp();
    } else {
        // ============================================================ compute
        // Warpgroup w = warp / 4 takes query columns 64w .. 64w + 63 of each
        // step; thread r owns key row r of the block (TMEM lane r).
        const int w = warp >> 2;
        const int r = (warp & 3) * 32 + lane;
        const uint32_t lane_base = static_cast<uint32_t>((warp & 3) * 32) << 16;
        const uint32_t s_tm = tmem + lane_base + kTmS + 64 * w;
        const uint32_t dp_tm = tmem + lane_base + kTmDP + 64 * w;
        const uint32_t acc_tm = tmem + lane_base + (w ? kTmDK : kTmDV);
        __nv_bfloat16* const out = w ? p.dk : p.dv;
        const float f = w ? p.scale : 1.f;
        const float c2 = p.scale_log2;
        const uint64_t c2c2 = ptx::f2_pack(c2, c2), neg1 = ptx::f2_pack(-1.f, -1.f);
        uint32_t gs = 0, items = 0;
        Cursor c;
        for (c.start(p); c.valid(p); c.next(p)) {
            const int n = c.steps(p);
            const int key = c.kb * kBlockN + r;
            for (int s = 0; s < n; ++s, ++gs) {
                int h, qb;
                c.step(p, s, h, qb);
                // Visible columns j (query qb*128 + 64w + j) of this key row:
                // lo <= j <= hi.
                const int q0 = qb * kBlockM + 64 * w;
                int lo = 0, hi = 63;
                if (p.causal) lo = key - p.causal_offset - q0;
                if (p.window_left >= 0) hi = min(hi, key + p.window_left - p.causal_offset - q0);
                const uint32_t slot = gs % kStages;
                const uint32_t sL = sbase + L::kLD + slot * L::kLDSlot + 4 * 64 * w;
                const uint32_t sD = sL + kBlockM * 4;
                float pt[64];
                // -L and D arrive with the step's Q tile; that slot is refilled
                // only after this step's dK products, which wait for dS^T.
                if (!wait_bar_warp(bar(L::bQFull + slot), (gs / kStages) & 1, wc)) return;
                if (!wait_bar_warp(bar(L::bSFull), gs & 1, wc)) return;
                ptx::tc_fence_after();
                {
                    uint32_t s0[32], s1[32];
                    ptx::tmem_ld32(s_tm, s0);
                    ptx::tmem_ld32(s_tm + 32, s1);
                    ptx::tmem_wait_ld();
#pragma unroll
                    for (int k = 0; k < 32; ++k) {
                        pt[k] = __uint_as_float(s0[k]);
                        pt[32 + k] = __uint_as_float(s1[k]);
                    }
                }
                // P^T = 2^(S^T c - L), pairs of columns in packed FP32; the
                // mask is applied only where some key row of the warp needs
                // it (the diagonal steps of a causal or windowed launch).
                auto exps = [&](auto mask_tag) {
                    constexpr bool kMask = decltype(mask_tag)::value;
#pragma unroll
                    for (int k4 = 0; k4 < 16; ++k4) {
                        const float4 l4 = ptx::ld_shared_f4(sL + 16 * k4);  // -L, same address: broadcast
#pragma unroll
                        for (int e = 0; e < 2; ++e) {
                            const int k = 4 * k4 + 2 * e;
                            float x0, x1;
                            ptx::f2_unpack(ptx::f2_fma(ptx::f2_pack(pt[k], pt[k + 1]), c2c2,
                                                       e ? ptx::f2_pack(l4.z, l4.w) : ptx::f2_pack(l4.x, l4.y)),
                                           x0, x1);
                            x0 = ptx::ex2(x0);
                            x1 = ptx::ex2(x1);
                            if (kMask) {
                                x0 = (k >= lo && k <= hi) ? x0 : 0.f;
                                x1 = (k + 1 >= lo && k + 1 <= hi) ? x1 : 0.f;
                            }
                            pt[k] = x0;
                            pt[k + 1] = x1;
                        }
                    }
                };
                if (__any_sync(0xffffffffu, lo > 0 || hi < 63))
                    exps(std::true_type{});
                else
                    exps(std::false_type{});
                // P^T in BF16 over the first 32 of this warpgroup's S^T
                // columns (read above by this thread only).
                {
                    uint32_t pk[32];
#pragma unroll
                    for (int j = 0; j < 32; ++j) pk[j] = ptx::pack_bf16x2(pt[2 * j], pt[2 * j + 1]);
                    ptx::tmem_st32(s_tm, pk);
                    ptx::tmem_wait_st();
                }
                ptx::tc_fence_before();
                __syncwarp();
                if (lane == 0) ptx::mbar_arrive(bar(L::bPTFull));
                // dS^T = P^T (dP^T - D), BF16 over the first 32 of this
                // warpgroup's dP^T columns.
                if (!wait_bar_warp(bar(L::bPFull), gs & 1, wc)) return;
                ptx::tc_fence_after();
#pragma unroll
                for (int q = 0; q < 2; ++q) {
                    uint32_t dr[32];
                    ptx::tmem_ld32(dp_tm + q * 32, dr);
                    ptx::tmem_wait_ld();
#pragma unroll
                    for (int k4 = 0; k4 < 8; ++k4) {
                        const float4 d4 = ptx::ld_shared_f4(sD + 4 * (q * 32 + 4 * k4));
#pragma unroll
                        for (int e = 0; e < 2; ++e) {
                            const int k = 4 * k4 + 2 * e;
                            // (dP - D) by one packed FMA, then times P.
                            const uint64_t t = ptx::f2_fma(
                                e ? ptx::f2_pack(d4.z, d4.w) : ptx::f2_pack(d4.x, d4.y), neg1,
                                ptx::f2_pack(__uint_as_float(dr[k]), __uint_as_float(dr[k + 1])));
                            float a, b2;
                            ptx::f2_unpack(ptx::f2_mul(ptx::f2_pack(pt[q * 32 + k], pt[q * 32 + k + 1]), t),
                                           a, b2);
                            pt[q * 32 + k] = a;
                            pt[q * 32 + k + 1] = b2;
                        }
                    }
                }
                {
                    uint32_t pk[32];
#pragma unroll
                    for (int j = 0; j < 32; ++j) pk[j] = ptx::pack_bf16x2(pt[2 * j], pt[2 * j + 1]);
                    ptx::tmem_st32(dp_tm, pk);
                    ptx::tmem_wait_st();
                }
                ptx::tc_fence_before();
                __syncwarp();
                if (lane == 0) ptx::mbar_arrive(bar(L::bDSTFull));
            }
            // Epilogue: warpgroup 0 writes dV, warpgroup 1 dK * scale; each
            // thread stores its key row (256 contiguous bytes) directly.
            if (!wait_bar_warp(bar(L::bAccFull), items & 1, wc)) return;
            ptx::tc_fence_after();
            __nv_bfloat16* row =
                out + ((static_cast<size_t>(c.b) * p.s_k + key) * p.h_kv + c.g) * kHeadDim;
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                uint32_t v[32];
                ptx::tmem_ld32(acc_tm + q * 32, v);
                ptx::tmem_wait_ld();
                if (key < p.s_k) {
#pragma unroll
                    for (int k = 0; k < 4; ++k) {
                        uint4 u;
                        u.x = ptx::pack_bf16x2(__uint_as_float(v[8 * k]) * f, __uint_as_float(v[8 * k + 1]) * f);
                        u.y = ptx::pack_bf16x2(__uint_as_float(v[8 * k + 2]) * f, __uint_as_float(v[8 * k + 3]) * f);
                        u.z = ptx::pack_bf16x2(__uint_as_float(v[8 * k + 4]) * f, __uint_as_float(v[8 * k + 5]) * f);
                        u.w = ptx::pack_bf16x2(__uint_as_float(v[8 * k + 6]) * f, __uint_as_float(v[8 * k + 7]) * f);
                        *reinterpret_cast<uint4*>(row + q * 32 + 8 * k) = u;
                    }
                }
            }
            ptx::tc_fence_before();
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive(bar(L::bAccFree));
            ++items;
        }
    }

    ptx::tc_fence_before();
    __syncthreads();
    if (warp == kMmaWarp) {
        ptx::tc_fence_after();
        ptx::tmem_dealloc(tmem, kTmemCols);
    }
}

}  // namespace dkdv
}  // namespace bwd
}  // namespace sdpa10

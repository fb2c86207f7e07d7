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
//   attn_bwd_prep_kernel  -- D and L per query row (memory-bound), written
//                            to a padded workspace (padding rows: L = +inf,
//                            D = 0, so they carry weight 0);
//   attn_bwd_dq_kernel    -- one CTA item per 128-row query block
//                            (persistent): Q and dO stay in shared memory,
//                            K/V tiles stream through a two-slot ring; per
//                            key block S and dP on the tensor core (TMEM),
//                            dS by two warpgroups (each 64 of the block's
//                            keys, thread = row), dQ += dS K on the tensor
//                            core;
//   attn_bwd_dkdv_kernel  -- one CTA item per 128-key block of a key/value
//                            head: K and V stay in shared memory, 64-row
//                            Q/dO tiles of every query head of the group
//                            stream through a three-slot ring; S^T = K Q^T
//                            and dP^T = V dO^T on the tensor core, P^T and
//                            dS^T by one of two warpgroups (alternate steps,
//                            thread = key), dV += P^T dO and dK += dS^T Q.
// In the dK/dV kernel one warpgroup's exponentials run while the other's
// products are on the tensor core.  (The same split for dQ, with 64-key
// steps, measured slower on B200 than this single-warpgroup dQ kernel with
// 128-key steps, which already overlaps S(j+1) with block j's softmax.)
// Splitting dQ from dK/dV costs a second Q K^T and dO V^T but needs no
// atomics: every output element is written once, by one CTA, and the result
// is bit-for-bit reproducible.
#pragma once

#include "attn_common.cuh"

namespace sdpa10 {
namespace bwd {

constexpr int kBlockQ = 64;             // query rows per dK/dV step
constexpr int kQTile64Bytes = kBlockQ * kHeadDim * 2;  // 16 KiB: 64 rows x 128
constexpr int kHalf64Bytes = kQTile64Bytes / 2;         // one 64-column half

struct BwdParams {
    int batch, h_q, h_kv, s_q, s_k;
    int group;             // h_q / h_kv
    int n_qb;              // ceil(s_q / 128)   (dQ kernel)
    int n_kb;              // ceil(s_k / 128)
    int n_qb64;            // ceil(s_q / 64)    (dK/dV kernel)
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
    const float* L;        // [batch][h_q][s_q_pad]  LSE * log2(e) (+inf padding)
    const float* D;        // [batch][h_q][s_q_pad]  rowsum(dO * O) (0 padding)
    unsigned long long timeout_ns;
    unsigned int* status;
};

// ------------------------------------------------------------------ prep
// One warp per query row: D = sum_c dO[c] O[c] (BF16 in, FP32 sum) and
// L = LSE * log2(e); the rows s_q .. s_q_pad - 1 of each head get L = +inf
// and D = 0.
struct PrepParams {
    const __nv_bfloat16* o;
    const __nv_bfloat16* dout;
    const float* lse;
    float* L;
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
                a.L[r] = CUDART_INF_F;
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
            a.L[r] = a.lse[bh * a.s_q + i] * 1.4426950408889634f;
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
    static constexpr int kDS = 2 * kTileBytes;         // dS (A of dQ += dS K); O staging
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
    const uint32_t tmem = *tmem_slot;  // S | dP | dQ at columns 0, 128, 256
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
        if (lane == 0) {
            constexpr uint32_t kIdS = idesc_bf16_f32(kBlockM, kBlockN, 0, 0);    // Q K^T, dO V^T
            constexpr uint32_t kIdDq = idesc_bf16_f32(kBlockM, kHeadDim, 0, 1);  // dS K (K MN-major)
            const uint32_t q_lo = desc_lo_sw128(sbase + L::kQ, 16);
            const uint32_t do_lo = desc_lo_sw128(sbase + L::kDO, 16);
            const uint32_t ds_lo = desc_lo_sw128(sbase + L::kDS, 16);
            const uint32_t k_lo = desc_lo_sw128(sbase + L::kK, 16);
            const uint32_t kmn_lo = desc_lo_sw128(sbase + L::kK, kHalfTileBytes);
            const uint32_t v_lo = desc_lo_sw128(sbase + L::kV, 16);
            const uint32_t s_tm = tmem, dp_tm = tmem + 128, dq_tm = tmem + 256;
            uint32_t k_used = 0, v_used = 0, items = 0, steps = 0;
            bool ok = true;
            // K-major operands: 8 K-steps of 16 BF16 (32 bytes) inside a
            // 64-column half; the second half is 16 KiB on.
            auto gemm_kmajor = [&](uint32_t d_tm, uint32_t a_lo, uint32_t b_lo) {
#pragma unroll
                for (int k = 0; k < kHeadDim / 16; ++k) {
                    const uint32_t off = ((k >> 2) * kHalfTileBytes + (k & 3) * 32) >> 4;
                    ptx::mma_ss(d_tm, desc_from_lo(a_lo + off), desc_from_lo(b_lo + off), kIdS,
                                k > 0 ? 1u : 0u);
                }
            };
            // Per item: S(0), dP(0), then per key block j: S(j+1), dQ(j),
            // dP(j+1) -- the next scores run under this block's exponentials
            // and dQ(j) runs while the compute warps start on block j + 1.
            auto scores = [&](uint32_t gs) -> bool {
                const uint32_t ks = k_used % kStages;
                if (!wait_bar(bar(L::bKFull + ks), (k_used / kStages) & 1, wc)) return false;
                if (gs > 0 && !wait_bar(bar(L::bSFree), (gs - 1) & 1, wc)) return false;
                ptx::tc_fence_after();
                gemm_kmajor(s_tm, q_lo, k_lo + ((ks * kTileBytes) >> 4));
                ptx::mma_commit(bar(L::bSFull));
                ++k_used;  // K(j) stays in its slot until dQ(j) has read it
                return true;
            };
            auto dprobs = [&](uint32_t gs) -> bool {
                const uint32_t vs = v_used % kStages;
                if (!wait_bar(bar(L::bVFull + vs), (v_used / kStages) & 1, wc)) return false;
                if (gs > 0 && !wait_bar(bar(L::bPFree), (gs - 1) & 1, wc)) return false;
                ptx::tc_fence_after();
                gemm_kmajor(dp_tm, do_lo, v_lo + ((vs * kTileBytes) >> 4));
                ptx::mma_commit(bar(L::bPFull));
                ptx::mma_commit(bar(L::bVEmpty + vs));
                ++v_used;
                return true;
            };
            uint32_t k_freed = 0;  // K tiles released after their dQ
            Cursor c;
            for (c.start(p); ok && c.valid(p); c.next(p)) {
                if (!(ok = wait_bar(bar(L::bQFull), items & 1, wc))) break;
                // dQ of the previous item must have been read out of TMEM.
                if (items > 0 && !(ok = wait_bar(bar(L::bDqFree), (items - 1) & 1, wc))) break;
                ++items;
                if (!(ok = scores(steps) && dprobs(steps))) break;
                for (int j = 0; j < c.n && ok; ++j) {
                    const uint32_t gs = steps + j;
                    if (j + 1 < c.n && !(ok = scores(gs + 1))) break;
                    // dQ += dS K once dS is in shared memory.
                    if (!(ok = wait_bar(bar(L::bDsFull), gs & 1, wc))) break;
                    ptx::tc_fence_after();
                    const uint32_t ks = k_freed % kStages;
                    const uint32_t kb = kmn_lo + ((ks * kTileBytes) >> 4);
#pragma unroll
                    for (int k = 0; k < kBlockN / 16; ++k) {
                        // A = dS (K-major like Q); B = K, MN-major (head dim
                        // contiguous): 16 keys = 2 KiB per step.
                        const uint32_t off = ((k >> 2) * kHalfTileBytes + (k & 3) * 32) >> 4;
                        ptx::mma_ss(dq_tm, desc_from_lo(ds_lo + off),
                                    desc_from_lo(kb + ((k * 2048) >> 4)), kIdDq,
                                    (j > 0 || k > 0) ? 1u : 0u);
                    }
                    ptx::mma_commit(bar(L::bDsFree));
                    ptx::mma_commit(bar(L::bKEmpty + ks));
                    ++k_freed;
                    if (j + 1 < c.n && !(ok = dprobs(gs + 1))) break;
                }
                if (!ok) break;
                steps += c.n;
                ptx::mma_commit(bar(L::bQEmpty));
                ptx::mma_commit(bar(L::bDqFull));
            }
            ptx::mma_commit(bar(L::bDrain));
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
                       dq_tm = tmem + lane_base + 256 + 64 * half;
        // This row's half of the dS tile: the tile's 64-column half `half`
        // (16 KiB), chunk k of the half at ((k ^ (r % 8)) * 16).
        const uint32_t ds_row =
            sbase + L::kDS + half * kHalfTileBytes + (r >> 3) * 1024 + (r & 7) * 128;
        const uint32_t xr = static_cast<uint32_t>(r & 7);
        const float c2 = p.scale_log2;
        uint32_t items = 0, steps = 0;
        Cursor c;
        for (c.start(p); c.valid(p); c.next(p)) {
            const int row = c.qb * kBlockM + r;
            const size_t stat = (static_cast<size_t>(c.b) * p.h_q + c.h) * p.s_q_pad + row;
            const float Lr = p.L[stat];  // +inf past s_q: P = 0
            const float Dr = p.D[stat];
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
#pragma unroll
                for (int k = 0; k < 64; ++k) {
                    const float x = ptx::ex2(fmaf(pr[k], c2, -Lr));
                    pr[k] = (k >= lo && k < hi) ? x : 0.f;
                }
                // dS = P (dP - D) -> BF16, into this warpgroup's half of the
                // dS tile (K-major, 128-byte swizzle).
                if (!wait_bar_warp(bar(L::bPFull), steps & 1, wc)) return;
                if (steps > 0 && !wait_bar_warp(bar(L::bDsFree), (steps - 1) & 1, wc)) return;
                ptx::tc_fence_after();
#pragma unroll
                for (int q = 0; q < 2; ++q) {
                    uint32_t dr[32];
                    ptx::tmem_ld32(dp_tm + q * 32, dr);
                    ptx::tmem_wait_ld();
                    uint32_t w[16];
#pragma unroll
                    for (int k = 0; k < 16; ++k) {
                        const float a = pr[q * 32 + 2 * k] * (__uint_as_float(dr[2 * k]) - Dr);
                        const float b2 = pr[q * 32 + 2 * k + 1] * (__uint_as_float(dr[2 * k + 1]) - Dr);
                        w[k] = ptx::pack_bf16x2(a, b2);
                    }
#pragma unroll
                    for (int k = 0; k < 4; ++k) {
                        const int cc = 4 * q + k;  // chunk within this half
                        ptx::st_shared_v4(ds_row + ((cc ^ xr) << 4), w[4 * k], w[4 * k + 1],
                                          w[4 * k + 2], w[4 * k + 3]);
                    }
                }
                ptx::tc_fence_before();
                ptx::fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) {
                    ptx::mbar_arrive(bar(L::bPFree));
                    ptx::mbar_arrive(bar(L::bDsFull));
                }
            }
            // Epilogue: dQ * scale -> BF16 rows, each warpgroup its 64
            // columns, staged in its half of the dS tile (free once the last
            // dQ MMA has completed) and stored with TMA.
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
                    ptx::st_shared_v4(ds_row + ((cc ^ xr) << 4), w[4 * k], w[4 * k + 1],
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
                ptx::tma_store_4d(&tm_dq, sbase + L::kDS, 0, c.h, c.qb * kBlockM, c.b);
                ptx::tma_store_4d(&tm_dq, sbase + L::kDS + kHalfTileBytes, 64, c.h,
                                  c.qb * kBlockM, c.b);
                ptx::bulk_commit_group();
                ptx::bulk_wait_group_read0();
                ptx::mbar_arrive(bar(L::bStored));
            }
            // The dS tile is rewritten by the next item only after TMA has
            // read the staged rows.
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

// Two compute warpgroups take alternate 64-row steps (warps 0-3 the even
// global steps, warps 4-7 the odd ones), so one warpgroup's exponentials and
// dS^T run while the other's tiles are on the tensor core; warp 8 is the
// TMA producer and warp 9 the MMA issuer.
constexpr int kThreads = 320;
constexpr int kLoadWarp = 8;
constexpr int kMmaWarp = 9;
constexpr int kQDStages = 3;

struct Smem {
    static constexpr int kK = 0;                              // K tile (A of S^T = K Q^T)
    static constexpr int kV = kTileBytes;                     // V tile (A of dP^T = V dO^T)
    static constexpr int kQD = 2 * kTileBytes;                // ring of 3 x (Q 64 rows, dO 64 rows)
    static constexpr int kQDSlot = 2 * kQTile64Bytes;         // 32 KiB per slot
    // Per warpgroup w: P^T_w then dS^T_w ([128 keys x 64], 16 KiB each),
    // 32 KiB contiguous; at the end of an item warpgroup 0 stages dV and
    // warpgroup 1 stages dK there for the TMA store.
    static constexpr int kWG = kQD + kQDStages * kQDSlot;
    static constexpr int kWGBytes = 2 * kQTile64Bytes;
    static constexpr int kLD = kWG + 2 * kWGBytes;            // ring of 3 x (L[64], D[64])
    static constexpr int kBars = kLD + kQDStages * 512;
    static constexpr int bKVFull = 0, bKVEmpty = 1, bQDFull = 2, bQDEmpty = 2 + kQDStages,
                         bSFull = 2 + 2 * kQDStages,       // [2] per warpgroup from here on
                         bSFree = bSFull + 2, bPFull = bSFree + 2, bPFree = bPFull + 2,
                         bPTFull = bPFree + 2, bPTFree = bPTFull + 2, bDSTFull = bPTFree + 2,
                         bDSTFree = bDSTFull + 2, bStaged = bDSTFree + 2, bStored = bStaged + 2,
                         bAccFull = bStored + 2, bAccFree = bAccFull + 1, bDrain = bAccFree + 1,
                         kNumBars = bDrain + 1;
    static constexpr int kTmemSlot = kBars + kNumBars * 8;
    static constexpr int kAbort = kTmemSlot + 4;
    static constexpr int kBytes = kAbort + 4;
    static constexpr int kAlloc = kBytes + 1024;
};
static_assert(Smem::kAlloc <= 232448, "dK/dV shared memory exceeds the per-CTA limit");

// Item t -> (key block, batch, key/value head): by section of heads, then
// key block ascending (under the causal mask the first key blocks are seen
// by the most query rows: longest first), then head.  The item walks the query heads of
// the group and, for each, the 64-row query blocks that see the key block.
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
        int lo = 0, hi = p.n_qb64;
        if (p.causal) {
            // Query i sees key 128 kb (the block's first key) iff
            // i >= 128 kb - causal_offset: floor division by 64.
            lo = max(0, (kb * kBlockN - p.causal_offset) >> 6);
        }
        if (p.window_left >= 0) {
            // Query i still sees the block's last key iff
            // i <= 128 kb + 127 + window_left - causal_offset.
            const int last = kb * kBlockN + kBlockN - 1 + p.window_left - p.causal_offset;
            hi = min(hi, (last >> 6) + 1);
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
};

__global__ void __launch_bounds__(kThreads, 1)
    attn_bwd_dkdv_kernel(const __grid_constant__ CUtensorMap tm_q64,
                         const __grid_constant__ CUtensorMap tm_k,
                         const __grid_constant__ CUtensorMap tm_v,
                         const __grid_constant__ CUtensorMap tm_do64,
                         const __grid_constant__ CUtensorMap tm_dk,
                         const __grid_constant__ CUtensorMap tm_dv,
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
        ptx::mbar_init(bar(L::bKVFull), 1);
        ptx::mbar_init(bar(L::bKVEmpty), 1);
        for (int i = 0; i < kQDStages; ++i) {
            ptx::mbar_init(bar(L::bQDFull + i), 1);
            ptx::mbar_init(bar(L::bQDEmpty + i), 1);
        }
        for (int w = 0; w < 2; ++w) {
            ptx::mbar_init(bar(L::bSFull + w), 1);
            ptx::mbar_init(bar(L::bSFree + w), 4);
            ptx::mbar_init(bar(L::bPFull + w), 1);
            ptx::mbar_init(bar(L::bPFree + w), 4);
            ptx::mbar_init(bar(L::bPTFull + w), 4);
            ptx::mbar_init(bar(L::bPTFree + w), 1);
            ptx::mbar_init(bar(L::bDSTFull + w), 4);
            ptx::mbar_init(bar(L::bDSTFree + w), 1);
            ptx::mbar_init(bar(L::bStaged + w), 4);
            ptx::mbar_init(bar(L::bStored + w), 1);
        }
        ptx::mbar_init(bar(L::bAccFull), 1);
        ptx::mbar_init(bar(L::bAccFree), 8);  // both warpgroups have read dV / dK
        ptx::mbar_init(bar(L::bDrain), 1);
        *abort_flag = 0;
        ptx::fence_mbar_init();
    }
    if (warp == kLoadWarp && lane == 0) {
        ptx::prefetch_tmap(&tm_q64);
        ptx::prefetch_tmap(&tm_k);
        ptx::prefetch_tmap(&tm_v);
        ptx::prefetch_tmap(&tm_do64);
        ptx::prefetch_tmap(&tm_dk);
        ptx::prefetch_tmap(&tm_dv);
    }
    if (warp == kMmaWarp) {
        ptx::tmem_alloc(ptx::smem_u32(tmem_slot), kTmemCols);
        ptx::tmem_relinquish();
    }
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    // TMEM: S^T_0 | S^T_1 | dP^T_0 | dP^T_1 (64 columns each) | dV | dK at
    // columns 0, 64, 128, 192, 256, 384.
    const uint32_t tmem = *tmem_slot;
    const WaitCtx wc{abort_flag, p.status, p.timeout_ns};
    auto qd_addr = [&](uint32_t u) { return sbase + L::kQD + (u % kQDStages) * L::kQDSlot; };

    if (warp == kLoadWarp) {
        // ============================================================ producer
        if (lane == 0) {
            const uint64_t pol_kv = ptx::policy_evict_first();
            const uint64_t pol_q = ptx::policy_evict_last();
            uint32_t kv_loads = 0, qd_loads = 0;
            bool ok = true;
            Cursor c;
            for (c.start(p); ok && c.valid(p); c.next(p)) {
                if (!(ok = wait_bar(bar(L::bKVEmpty), (kv_loads & 1) ^ 1, wc))) break;
                ptx::mbar_arrive_expect_tx(bar(L::bKVFull), 2 * kTileBytes);
#pragma unroll
                for (int half = 0; half < 2; ++half) {
                    ptx::tma_load_4d(sbase + L::kK + half * kHalfTileBytes, &tm_k, bar(L::bKVFull),
                                     64 * half, c.g, c.kb * kBlockN, c.b, pol_kv);
                    ptx::tma_load_4d(sbase + L::kV + half * kHalfTileBytes, &tm_v, bar(L::bKVFull),
                                     64 * half, c.g, c.kb * kBlockN, c.b, pol_kv);
                }
                ++kv_loads;
                const int n = c.steps(p);
                for (int s = 0; s < n && ok; ++s) {
                    const int hl = s / c.nq;
                    const int qb = c.qlo + (s - hl * c.nq);
                    const int h = c.g * p.group + hl;
                    const uint32_t slot = qd_loads % kQDStages;
                    if (!(ok = wait_bar(bar(L::bQDEmpty + slot),
                                        ((qd_loads / kQDStages) & 1) ^ 1, wc)))
                        break;
                    const uint32_t full = bar(L::bQDFull + slot);
                    const uint32_t dst = qd_addr(qd_loads);
                    ptx::mbar_arrive_expect_tx(full, 2 * kQTile64Bytes + 512);
#pragma unroll
                    for (int half = 0; half < 2; ++half) {
                        ptx::tma_load_4d(dst + half * kHalf64Bytes, &tm_q64, full, 64 * half, h,
                                         qb * kBlockQ, c.b, pol_q);
                        ptx::tma_load_4d(dst + kQTile64Bytes + half * kHalf64Bytes, &tm_do64, full,
                                         64 * half, h, qb * kBlockQ, c.b, pol_q);
                    }
                    const size_t stat =
                        (static_cast<size_t>(c.b) * p.h_q + h) * p.s_q_pad + qb * kBlockQ;
                    ptx::bulk_load(sbase + L::kLD + slot * 512, p.L + stat, 256, full);
                    ptx::bulk_load(sbase + L::kLD + slot * 512 + 256, p.D + stat, 256, full);
                    ++qd_loads;
                }
            }
            if (kv_loads > 0) wait_slow(bar(L::bKVFull), (kv_loads - 1) & 1, wc, false);
            for (int i = 0; i < kQDStages && i < static_cast<int>(qd_loads); ++i) {
                const uint32_t f = qd_loads - 1 - i;
                wait_slow(bar(L::bQDFull + f % kQDStages), (f / kQDStages) & 1, wc, false);
            }
        }
        __syncwarp();
    } else if (warp == kMmaWarp) {
        // ============================================================ MMA issuer
        if (lane == 0) {
            constexpr uint32_t kIdS = idesc_bf16_f32(kBlockN, kBlockQ, 0, 0);   // K Q^T, V dO^T
            constexpr uint32_t kIdAcc = idesc_bf16_f32(kBlockN, kHeadDim, 0, 1);  // P^T dO, dS^T Q
            const uint32_t k_lo = desc_lo_sw128(sbase + L::kK, 16);
            const uint32_t v_lo = desc_lo_sw128(sbase + L::kV, 16);
            const uint32_t dv_tm = tmem + 256, dk_tm = tmem + 384;
            uint32_t items = 0, gs0 = 0;
            bool ok = true;
            // X^T = A B^T with A a [128 x 128] K-major tile (K or V) and B a
            // 64-row K-major tile (Q or dO): 8 K-steps; the 64-row tile's
            // second 64-column half is 8 KiB on.
            auto gemm_t = [&](uint32_t d_tm, uint32_t a_lo, uint32_t b_lo) {
#pragma unroll
                for (int k = 0; k < kHeadDim / 16; ++k) {
                    const uint32_t oa = ((k >> 2) * kHalfTileBytes + (k & 3) * 32) >> 4;
                    const uint32_t ob = ((k >> 2) * kHalf64Bytes + (k & 3) * 32) >> 4;
                    ptx::mma_ss(d_tm, desc_from_lo(a_lo + oa), desc_from_lo(b_lo + ob), kIdS,
                                k > 0 ? 1u : 0u);
                }
            };
            // Acc += A B with A a [128 x 64] K-major tile (P^T or dS^T, one
            // 64-column half) and B the 64-row tile read MN-major (head dim
            // contiguous, halves 8 KiB apart): 4 K-steps of 16 rows = 2 KiB.
            auto gemm_acc = [&](uint32_t d_tm, uint32_t a_lo, uint32_t b_addr, bool acc) {
                const uint32_t b_lo = desc_lo_sw128(b_addr, kHalf64Bytes);
#pragma unroll
                for (int k = 0; k < kBlockQ / 16; ++k)
                    ptx::mma_ss(d_tm, desc_from_lo(a_lo + ((k * 32) >> 4)),
                                desc_from_lo(b_lo + ((k * 2048) >> 4)), kIdAcc,
                                (acc || k > 0) ? 1u : 0u);
            };
            // S^T and dP^T of global step gs into warpgroup (gs & 1)'s
            // columns once that warpgroup has read its previous ones.
            auto scores = [&](uint32_t gs) -> bool {
                const uint32_t w = gs & 1, i = gs >> 1;
                if (!wait_bar(bar(L::bQDFull + gs % kQDStages), (gs / kQDStages) & 1, wc))
                    return false;
                if (i > 0 && !wait_bar(bar(L::bSFree + w), (i - 1) & 1, wc)) return false;
                ptx::tc_fence_after();
                gemm_t(tmem + 64 * w, k_lo, desc_lo_sw128(qd_addr(gs), 16));
                ptx::mma_commit(bar(L::bSFull + w));
                if (i > 0 && !wait_bar(bar(L::bPFree + w), (i - 1) & 1, wc)) return false;
                ptx::tc_fence_after();
                gemm_t(tmem + 128 + 64 * w, v_lo, desc_lo_sw128(qd_addr(gs) + kQTile64Bytes, 16));
                ptx::mma_commit(bar(L::bPFull + w));
                return true;
            };
            Cursor c;
            for (c.start(p); ok && c.valid(p); c.next(p)) {
                const int n = c.steps(p);
                if (!(ok = wait_bar(bar(L::bKVFull), items & 1, wc))) break;
                // Per item: S^T, dP^T of its first two steps, then per step
                // s: dV(s), dK(s), then S^T, dP^T of step s + 2 (same
                // warpgroup) -- the other warpgroup's step s + 1 runs on the
                // tensor core while this one's exponentials run.
                if (!(ok = scores(gs0))) break;
                if (n > 1 && !(ok = scores(gs0 + 1))) break;
                // dV / dK of the previous item must have been read out.
                if (items > 0 && !(ok = wait_bar(bar(L::bAccFree), (items - 1) & 1, wc))) break;
                ++items;
                for (int s = 0; s < n && ok; ++s) {
                    const uint32_t gs = gs0 + s, w = gs & 1, i = gs >> 1;
                    const uint32_t pt_lo = desc_lo_sw128(sbase + L::kWG + w * L::kWGBytes, 16);
                    const uint32_t dst_lo =
                        desc_lo_sw128(sbase + L::kWG + w * L::kWGBytes + kQTile64Bytes, 16);
                    if (!(ok = wait_bar(bar(L::bPTFull + w), i & 1, wc))) break;
                    ptx::tc_fence_after();
                    gemm_acc(dv_tm, pt_lo, qd_addr(gs) + kQTile64Bytes, s > 0);
                    ptx::mma_commit(bar(L::bPTFree + w));
                    if (!(ok = wait_bar(bar(L::bDSTFull + w), i & 1, wc))) break;
                    ptx::tc_fence_after();
                    gemm_acc(dk_tm, dst_lo, qd_addr(gs), s > 0);
                    ptx::mma_commit(bar(L::bDSTFree + w));
                    ptx::mma_commit(bar(L::bQDEmpty + gs % kQDStages));
                    if (s + 2 < n && !(ok = scores(gs + 2))) break;
                }
                if (!ok) break;
                gs0 += n;
                ptx::mma_commit(bar(L::bKVEmpty));
                ptx::mma_commit(bar(L::bAccFull));
            }
            ptx::mma_commit(bar(L::bDrain));
            wait_slow(bar(L::bDrain), 0, wc, false);
        }
        __syncwarp();
    } else {
        // ============================================================ compute
        // Warpgroup w = warp / 4; thread r owns key row r of the block (TMEM
        // lane r) and takes the global steps gs with gs % 2 == w.
        const int w = warp >> 2;
        const int r = (warp & 3) * 32 + lane;
        const uint32_t lane_base = static_cast<uint32_t>((warp & 3) * 32) << 16;
        const uint32_t s_tm = tmem + lane_base + 64 * w, dp_tm = tmem + lane_base + 128 + 64 * w;
        const uint32_t acc_tm = tmem + lane_base + (w ? 384 : 256);  // dK (w 1) or dV (w 0)
        // Row r of a [128 x 64] K-major tile: 8 chunks of 16 bytes, chunk cc
        // at (r / 8) * 1024 + (r % 8) * 128 + ((cc ^ (r % 8)) * 16).
        const uint32_t xr = static_cast<uint32_t>(r & 7);
        const uint32_t wg_base = sbase + L::kWG + w * L::kWGBytes;
        const uint32_t row_off = (r >> 3) * 1024 + (r & 7) * 128;
        const uint32_t pt_row = wg_base + row_off;
        const uint32_t dst_row = wg_base + kQTile64Bytes + row_off;
        const uint32_t st_row = wg_base + row_off;  // [128 x 128] staging, halves 16 KiB apart
        const float c2 = p.scale_log2;
        uint32_t items = 0, gs0 = 0, mine = 0;  // mine: steps this warpgroup has done
        Cursor c;
        for (c.start(p); c.valid(p); c.next(p)) {
            const int n = c.steps(p);
            const int key = c.kb * kBlockN + r;
            for (int s = (gs0 & 1) == static_cast<uint32_t>(w) ? 0 : 1; s < n; s += 2, ++mine) {
                const uint32_t gs = gs0 + s;
                const int hl = s / c.nq;
                const int qb = c.qlo + (s - hl * c.nq);
                // Visible query columns of this key row: [lo, hi].
                int lo = 0, hi = kBlockQ - 1;
                if (p.causal) lo = key - p.causal_offset - qb * kBlockQ;
                if (p.window_left >= 0)
                    hi = min(hi, key + p.window_left - p.causal_offset - qb * kBlockQ);
                const uint32_t slot = gs % kQDStages;
                const uint32_t sL = sbase + L::kLD + slot * 512;  // L[64], then D[64]
                const uint32_t sD = sL + 256;
                float pt[64];
                // L and D of this step's rows arrive with its Q / dO tiles
                // (the slot is refilled only after this step's dK MMA, which
                // waits for this warpgroup).
                if (!wait_bar_warp(bar(L::bQDFull + slot), (gs / kQDStages) & 1, wc)) return;
                if (!wait_bar_warp(bar(L::bSFull + w), mine & 1, wc)) return;
                ptx::tc_fence_after();
#pragma unroll
                for (int q = 0; q < 2; ++q) {
                    uint32_t sr[32];
                    ptx::tmem_ld32(s_tm + q * 32, sr);
                    ptx::tmem_wait_ld();
#pragma unroll
                    for (int k = 0; k < 32; ++k) pt[q * 32 + k] = __uint_as_float(sr[k]);
                }
                ptx::tc_fence_before();
                __syncwarp();
                if (lane == 0) ptx::mbar_arrive(bar(L::bSFree + w));
#pragma unroll
                for (int k4 = 0; k4 < 16; ++k4) {
                    const float4 l4 = ptx::ld_shared_f4(sL + 16 * k4);  // same address: broadcast
                    const float lv[4] = {l4.x, l4.y, l4.z, l4.w};
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const int k = 4 * k4 + e;
                        const float x = ptx::ex2(fmaf(pt[k], c2, -lv[e]));
                        pt[k] = (k >= lo && k <= hi) ? x : 0.f;
                    }
                }
                // P^T -> BF16 into this warpgroup's tile once its last dV
                // MMA has read it.
                if (mine > 0 && !wait_bar_warp(bar(L::bPTFree + w), (mine - 1) & 1, wc)) return;
#pragma unroll
                for (int cc = 0; cc < 8; ++cc)
                    ptx::st_shared_v4(pt_row + ((cc ^ xr) << 4),
                                      ptx::pack_bf16x2(pt[8 * cc], pt[8 * cc + 1]),
                                      ptx::pack_bf16x2(pt[8 * cc + 2], pt[8 * cc + 3]),
                                      ptx::pack_bf16x2(pt[8 * cc + 4], pt[8 * cc + 5]),
                                      ptx::pack_bf16x2(pt[8 * cc + 6], pt[8 * cc + 7]));
                ptx::fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) ptx::mbar_arrive(bar(L::bPTFull + w));
                // dS^T = P^T (dP^T - D) -> BF16.
                if (!wait_bar_warp(bar(L::bPFull + w), mine & 1, wc)) return;
                if (mine > 0 && !wait_bar_warp(bar(L::bDSTFree + w), (mine - 1) & 1, wc)) return;
                ptx::tc_fence_after();
#pragma unroll
                for (int q = 0; q < 2; ++q) {
                    uint32_t dr[32];
                    ptx::tmem_ld32(dp_tm + q * 32, dr);
                    ptx::tmem_wait_ld();
#pragma unroll
                    for (int k4 = 0; k4 < 8; ++k4) {
                        const float4 d4 = ptx::ld_shared_f4(sD + 4 * (q * 32 + 4 * k4));
                        const float dv4[4] = {d4.x, d4.y, d4.z, d4.w};
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const int k = 4 * k4 + e;
                            pt[q * 32 + k] = pt[q * 32 + k] * (__uint_as_float(dr[k]) - dv4[e]);
                        }
                    }
                }
                ptx::tc_fence_before();
                __syncwarp();
                if (lane == 0) ptx::mbar_arrive(bar(L::bPFree + w));
#pragma unroll
                for (int cc = 0; cc < 8; ++cc)
                    ptx::st_shared_v4(dst_row + ((cc ^ xr) << 4),
                                      ptx::pack_bf16x2(pt[8 * cc], pt[8 * cc + 1]),
                                      ptx::pack_bf16x2(pt[8 * cc + 2], pt[8 * cc + 3]),
                                      ptx::pack_bf16x2(pt[8 * cc + 4], pt[8 * cc + 5]),
                                      ptx::pack_bf16x2(pt[8 * cc + 6], pt[8 * cc + 7]));
                ptx::fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) ptx::mbar_arrive(bar(L::bDSTFull + w));
            }
            gs0 += n;
            // Epilogue: warpgroup 0 writes dV, warpgroup 1 dK * scale, as
            // BF16 rows staged in its own 32 KiB (its P^T and dS^T tiles, free
            // once every MMA of the item has completed) and stored with TMA
            // (rows past s_k are clipped by the tensor map).
            if (!wait_bar_warp(bar(L::bAccFull), items & 1, wc)) return;
            ptx::tc_fence_after();
            const float f = w ? p.scale : 1.f;
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                uint32_t v[32];
                ptx::tmem_ld32(acc_tm + q * 32, v);
                ptx::tmem_wait_ld();
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    const int cc = 4 * q + k;
                    ptx::st_shared_v4(
                        st_row + (cc >> 3) * kQTile64Bytes + (((cc & 7) ^ xr) << 4),
                        ptx::pack_bf16x2(__uint_as_float(v[8 * k]) * f, __uint_as_float(v[8 * k + 1]) * f),
                        ptx::pack_bf16x2(__uint_as_float(v[8 * k + 2]) * f, __uint_as_float(v[8 * k + 3]) * f),
                        ptx::pack_bf16x2(__uint_as_float(v[8 * k + 4]) * f, __uint_as_float(v[8 * k + 5]) * f),
                        ptx::pack_bf16x2(__uint_as_float(v[8 * k + 6]) * f, __uint_as_float(v[8 * k + 7]) * f));
                }
            }
            ptx::tc_fence_before();
            ptx::fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) {
                ptx::mbar_arrive(bar(L::bAccFree));
                ptx::mbar_arrive(bar(L::bStaged + w));
            }
            if (r == 0) {
                if (!wait_bar(bar(L::bStaged + w), items & 1, wc)) return;
                const CUtensorMap* tm = w ? &tm_dk : &tm_dv;
                ptx::tma_store_4d(tm, wg_base, 0, c.g, c.kb * kBlockN, c.b);
                ptx::tma_store_4d(tm, wg_base + kQTile64Bytes, 64, c.g, c.kb * kBlockN, c.b);
                ptx::bulk_commit_group();
                ptx::bulk_wait_group_read0();
                ptx::mbar_arrive(bar(L::bStored + w));
            }
            // This warpgroup's tiles are rewritten by its next step only
            // after TMA has read the staged rows.
            if (!wait_bar_warp(bar(L::bStored + w), items & 1, wc)) return;
            ++items;
        }
        if (r == 0) ptx::bulk_wait_group0();
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

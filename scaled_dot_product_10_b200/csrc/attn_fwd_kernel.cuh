// attn_fwd_kernel.cuh -- fused scaled dot-product attention forward for
// B200 (sm_100a): TMA -> shared-memory ring -> tcgen05.mma into Tensor
// Memory -> FP32 online softmax -> tcgen05.mma with P read from Tensor
// Memory -> BF16 O and FP32 LSE.
//
// What is computed is the SDPA definition softmax(Q K^T * scale) V (rkmt.cn
// "GPU attention operator optimisation" page, section 1), evaluated the way
// the pages' FlashAttention discussion describes: key/value blocks are
// streamed through on-chip memory and S is never written to HBM
// (bjdmk.com.cn page, section 5.1), and each block's local softmax is merged
// into a running result ("local attention then global reduction", rkmt.cn
// page, section 3.1.1).  The merge is the exact online-softmax rescaling:
// with a running row maximum m and sum l,
//     m' = max(m, max_j s_j),  l' = l * 2^((m - m') c) + sum_j 2^(s_j c - m' c),
//     O' = O * 2^((m - m') c) + P V,      c = scale * log2(e),
// which equals the definition exactly in exact arithmetic.  The scale is
// folded into the exponent (the AVO page, section 3.1, fuses the scale into
// the QK^T stage) and the mask is applied while the scores are in registers
// (AVO page, section 2.2).
//
// Warp roles of one CTA (192 threads):
//   warps 0-3  softmax / correction / epilogue; thread t owns query row t
//              of the tile, i.e. Tensor Memory lane t
//   warp  4    TMA producer (one elected lane)
//   warp  5    tcgen05.mma issuer (one elected lane) and TMEM allocator
// Tensor Memory (512 columns): S/P double buffer at columns 0 and 128
// (P is written as packed BF16 over the first 64 columns of its S), O at 256.
// Shared memory: two Q tiles (so the next tile's Q loads early) and a ring of
// KV_STAGES key/value tiles, all 128 rows x 128 BF16 in the 128-byte swizzle
// that TMA writes and tcgen05 descriptors read.
//
// Every wait is bounded (the per-CTA abort flag plus a global-timer limit);
// a wait that gives up sets the device status word, and the CTA drains its
// in-flight copies and MMAs, frees Tensor Memory and exits.
#pragma once

#include <cuda_bf16.h>
#include <math_constants.h>

#include "sm100_ptx.cuh"

namespace sdpa10 {

constexpr int kHeadDim = 128;
constexpr int kBlockM = 128;  // query rows per tile
constexpr int kBlockN = 128;  // keys per key/value tile
constexpr int kTileBytes = kBlockM * kHeadDim * 2;  // 32 KiB: one Q, K or V tile
constexpr int kHalfTileBytes = kTileBytes / 2;      // one 64-column (128-byte row) half
constexpr int kTmemCols = 512;
constexpr unsigned kStatusTimeout = 1u;

// Rescale the running output only when the row maximum grows by more than
// this many powers of two; otherwise keep the stale maximum (the
// probabilities then stay below 2^8, well inside FP32 and BF16 range, and
// the final O / l and LSE are unchanged).
constexpr float kRescaleThresholdLog2 = 8.0f;

struct FwdParams {
    int batch, h_q, h_kv, s_q, s_k;
    int group;  // h_q / h_kv
    int n_qb;   // ceil(s_q / 128)
    int n_kb;   // ceil(s_k / 128)
    int causal;
    int num_tiles;
    int units_per_section;  // (batch, kv head) units whose K/V share L2 at once
    float scale_log2;       // scale * log2(e)
    __nv_bfloat16* o;
    float* lse;
    unsigned long long timeout_ns;
    unsigned int* status;
};

// ------------------------------------------------------------------ schedule
// Tile t -> (batch, query head, query block).  Tiles are grouped in
// sections of `units_per_section` (batch, kv head) units so the K/V of a
// section stay resident in L2 while its tiles run; inside a section the
// order is query block descending (longest causal work first), then unit,
// then the query heads of the unit's group (adjacent heads share K/V).
struct TileCursor {
    int t;   // tile index
    int it;  // key/value block within the tile
    int b, h, g, qb, n_kv;

    __device__ __forceinline__ void decode(const FwdParams& p) {
        const int tiles_per_unit = p.group * p.n_qb;
        const int units_total = p.batch * p.h_kv;
        const int G = p.units_per_section;
        const int sec = t / (G * tiles_per_unit);
        const int r = t - sec * G * tiles_per_unit;
        const int Gs = min(G, units_total - sec * G);
        const int qb_rank = r / (Gs * p.group);
        const int rem = r - qb_rank * Gs * p.group;
        const int unit = sec * G + rem / p.group;
        const int h_local = rem - (rem / p.group) * p.group;
        qb = p.n_qb - 1 - qb_rank;
        b = unit / p.h_kv;
        g = unit - b * p.h_kv;
        h = g * p.group + h_local;
        // Causal (s_q == s_k): rows of block qb see keys up to the block's
        // last row, i.e. key blocks 0..qb.
        n_kv = p.causal ? min(p.n_kb, qb + 1) : p.n_kb;
    }
    __device__ __forceinline__ void start(const FwdParams& p) {
        t = blockIdx.x;
        it = 0;
        if (t < p.num_tiles) decode(p);
    }
    __device__ __forceinline__ bool valid(const FwdParams& p) const { return t < p.num_tiles; }
    // Step to the next (tile, key block) pair of this CTA.  Returns true when
    // the step started a new tile.
    __device__ __forceinline__ bool advance(const FwdParams& p) {
        if (++it < n_kv) return false;
        it = 0;
        t += gridDim.x;
        if (t < p.num_tiles) decode(p);
        return true;
    }
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
__device__ __noinline__ bool wait_slow(uint32_t bar, uint32_t parity, WaitCtx w,
                                       bool honour_abort) {
    const uint64_t t0 = ptx::globaltimer_ns();
    for (uint32_t i = 1;; ++i) {
        if (ptx::mbar_try_wait(bar, parity)) return true;
        if ((i & 31u) == 0) {
            if (honour_abort && *w.abort_flag) return false;
            if (ptx::globaltimer_ns() - t0 > w.timeout_ns || i > (1u << 28)) {
                *w.abort_flag = 1;
                atomicOr(w.status, kStatusTimeout);
                return false;
            }
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

// ------------------------------------------------------------------ layout
template <int KV_STAGES>
struct SmemLayout {
    static constexpr int kQ = 0;                                    // 2 Q tiles
    static constexpr int kKV = 2 * kTileBytes;                      // ring
    static constexpr int kBars = kKV + KV_STAGES * kTileBytes;      // mbarriers
    // barrier indices
    static constexpr int bQFull = 0, bQEmpty = 2, bKVFull = 4, bKVEmpty = 4 + KV_STAGES,
                         bSFull = 4 + 2 * KV_STAGES, bPFull = bSFull + 2, bOFull = bPFull + 2,
                         bOEmpty = bOFull + 1, bDrain = bOEmpty + 1, kNumBars = bDrain + 1;
    static constexpr int kTmemSlot = kBars + kNumBars * 8;
    static constexpr int kAbort = kTmemSlot + 4;
    static constexpr int kBytes = kAbort + 4;
    static constexpr int kAlloc = kBytes + 1024;  // slack for 1024-byte alignment
};

// ------------------------------------------------------------------ kernel
template <int KV_STAGES>
__global__ void __launch_bounds__(192, 1)
    attn_fwd_sm100_kernel(const __grid_constant__ CUtensorMap tm_q,
                          const __grid_constant__ CUtensorMap tm_k,
                          const __grid_constant__ CUtensorMap tm_v, const FwdParams p) {
    using L = SmemLayout<KV_STAGES>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    const uint32_t sbase = ptx::smem_u32(smem);
    const uint32_t sQ = sbase + L::kQ;
    const uint32_t sKV = sbase + L::kKV;
    const uint32_t bars = sbase + L::kBars;
    auto bar = [&](int i) -> uint32_t { return bars + 8u * static_cast<uint32_t>(i); };
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kAbort);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kTmemSlot);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int i = 0; i < 2; ++i) {
            ptx::mbar_init(bar(L::bQFull + i), 1);
            ptx::mbar_init(bar(L::bQEmpty + i), 1);
            ptx::mbar_init(bar(L::bSFull + i), 1);
            ptx::mbar_init(bar(L::bPFull + i), 4);
        }
        for (int i = 0; i < KV_STAGES; ++i) {
            ptx::mbar_init(bar(L::bKVFull + i), 1);
            ptx::mbar_init(bar(L::bKVEmpty + i), 1);
        }
        ptx::mbar_init(bar(L::bOFull), 1);
        ptx::mbar_init(bar(L::bOEmpty), 4);
        ptx::mbar_init(bar(L::bDrain), 1);
        *abort_flag = 0;
        ptx::fence_mbar_init();
    }
    if (warp == 4 && lane == 0) {
        ptx::prefetch_tmap(&tm_q);
        ptx::prefetch_tmap(&tm_k);
        ptx::prefetch_tmap(&tm_v);
    }
    if (warp == 5) {
        ptx::tmem_alloc(ptx::smem_u32(tmem_slot), kTmemCols);
        ptx::tmem_relinquish();
    }
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const WaitCtx wc{abort_flag, p.status, p.timeout_ns};

    if (warp == 4) {
        // ============================================================ producer
        if (lane == 0) {
            const uint64_t pol_kv = ptx::policy_evict_last();
            const uint64_t pol_q = ptx::policy_evict_first();
            uint32_t fills = 0;   // key/value tiles issued
            int q_loads = 0;      // Q tiles issued
            bool ok = true;
            auto load_q = [&](const TileCursor& c) -> bool {
                const int buf = q_loads & 1;
                if (!wait_bar(bar(L::bQEmpty + buf), ((q_loads >> 1) & 1) ^ 1, wc)) return false;
                const uint32_t dst = sQ + buf * kTileBytes;
                ptx::mbar_arrive_expect_tx(bar(L::bQFull + buf), kTileBytes);
                ptx::tma_load_4d(dst, &tm_q, bar(L::bQFull + buf), 0, c.h, c.qb * kBlockM, c.b,
                                 pol_q);
                ptx::tma_load_4d(dst + kHalfTileBytes, &tm_q, bar(L::bQFull + buf), 64, c.h,
                                 c.qb * kBlockM, c.b, pol_q);
                ++q_loads;
                return true;
            };
            auto load_kv = [&](const CUtensorMap* tm, const TileCursor& c) -> bool {
                const int slot = fills % KV_STAGES;
                if (!wait_bar(bar(L::bKVEmpty + slot), ((fills / KV_STAGES) & 1) ^ 1, wc))
                    return false;
                const uint32_t dst = sKV + slot * kTileBytes;
                ptx::mbar_arrive_expect_tx(bar(L::bKVFull + slot), kTileBytes);
                ptx::tma_load_4d(dst, tm, bar(L::bKVFull + slot), 0, c.g, c.it * kBlockN, c.b,
                                 pol_kv);
                ptx::tma_load_4d(dst + kHalfTileBytes, tm, bar(L::bKVFull + slot), 64, c.g,
                                 c.it * kBlockN, c.b, pol_kv);
                ++fills;
                return true;
            };
            // Issue order = the MMA warp's consumption order:
            // K(0), then for each step G: K(G+1), V(G).
            TileCursor c;
            c.start(p);
            if (c.valid(p)) {
                ok = load_q(c) && load_kv(&tm_k, c);
                while (ok) {
                    TileCursor nx = c;
                    const bool new_tile = nx.advance(p);
                    const bool has_next = nx.valid(p);
                    if (has_next) {
                        if (new_tile && !(ok = load_q(nx))) break;
                        if (!(ok = load_kv(&tm_k, nx))) break;
                    }
                    if (!(ok = load_kv(&tm_v, c))) break;
                    if (!has_next) break;
                    c = nx;
                }
            }
            // Drain: every issued copy must land before the CTA may exit.
            for (int i = 0; i < KV_STAGES && i < static_cast<int>(fills); ++i) {
                const uint32_t f = fills - 1 - i;
                wait_slow(bar(L::bKVFull + f % KV_STAGES), (f / KV_STAGES) & 1, wc, false);
            }
            for (int i = 0; i < 2 && i < q_loads; ++i) {
                const int ql = q_loads - 1 - i;
                wait_slow(bar(L::bQFull + (ql & 1)), (ql >> 1) & 1, wc, false);
            }
        }
        __syncwarp();
    } else if (warp == 5) {
        // ============================================================ MMA issuer
        if (lane == 0) {
            constexpr uint32_t kIdescQK = idesc_bf16_f32(kBlockM, kBlockN, 0, 0);
            constexpr uint32_t kIdescPV = idesc_bf16_f32(kBlockM, kHeadDim, 0, 1);
            uint32_t fills = 0;  // key/value tiles consumed
            auto issue_s = [&](const TileCursor& c, int lt, uint32_t G) -> bool {
                const int qbuf = lt & 1;
                if (c.it == 0 && !wait_bar(bar(L::bQFull + qbuf), (lt >> 1) & 1, wc)) return false;
                const int slot = fills % KV_STAGES;
                if (!wait_bar(bar(L::bKVFull + slot), (fills / KV_STAGES) & 1, wc)) return false;
                ptx::tc_fence_after();
                const uint32_t d_tmem = tmem + (G & 1) * 128;
                const uint32_t qa = sQ + qbuf * kTileBytes;
                const uint32_t ka = sKV + slot * kTileBytes;
#pragma unroll
                for (int k = 0; k < kHeadDim / 16; ++k) {
                    // K-major, 128-byte swizzle: 16 BF16 (32 bytes) per step
                    // inside a 64-column half; the second half is 16 KiB on.
                    const uint32_t off = (k >> 2) * kHalfTileBytes + (k & 3) * 32;
                    ptx::mma_ss(d_tmem, smem_desc_sw128(qa + off, 16, 1024),
                                smem_desc_sw128(ka + off, 16, 1024), kIdescQK, k > 0 ? 1u : 0u);
                }
                ptx::mma_commit(bar(L::bSFull + (G & 1)));
                ptx::mma_commit(bar(L::bKVEmpty + slot));
                if (c.it == c.n_kv - 1) ptx::mma_commit(bar(L::bQEmpty + qbuf));
                ++fills;
                return true;
            };
            auto issue_pv = [&](const TileCursor& c, int lt, uint32_t G) -> bool {
                if (!wait_bar(bar(L::bPFull + (G & 1)), (G >> 1) & 1, wc)) return false;
                if (c.it == 0 && lt > 0 && !wait_bar(bar(L::bOEmpty), (lt - 1) & 1, wc))
                    return false;
                const int slot = fills % KV_STAGES;
                if (!wait_bar(bar(L::bKVFull + slot), (fills / KV_STAGES) & 1, wc)) return false;
                ptx::tc_fence_after();
                const uint32_t p_tmem = tmem + (G & 1) * 128;
                const uint32_t va = sKV + slot * kTileBytes;
#pragma unroll
                for (int k = 0; k < kBlockN / 16; ++k) {
                    // A = P from TMEM: 16 keys = 8 packed columns per step.
                    // B = V, MN-major (head dim contiguous): 16 keys = two
                    // 8-row swizzle atoms = 2 KiB per step; the two 64-wide
                    // head-dim halves are 16 KiB apart (leading offset).
                    ptx::mma_ts(tmem + 256, p_tmem + k * 8,
                                smem_desc_sw128(va + k * 2048, kHalfTileBytes, 1024), kIdescPV,
                                (c.it > 0 || k > 0) ? 1u : 0u);
                }
                ptx::mma_commit(bar(L::bOFull));
                ptx::mma_commit(bar(L::bKVEmpty + slot));
                ++fills;
                return true;
            };
            TileCursor c;
            c.start(p);
            if (c.valid(p) && issue_s(c, 0, 0)) {
                int lt = 0;
                uint32_t G = 0;
                for (;;) {
                    TileCursor nx = c;
                    const bool new_tile = nx.advance(p);
                    const bool has_next = nx.valid(p);
                    const int lt_next = lt + (new_tile ? 1 : 0);
                    if (has_next && !issue_s(nx, lt_next, G + 1)) break;
                    if (!issue_pv(c, lt, G)) break;
                    ++G;
                    if (!has_next) break;
                    c = nx;
                    lt = lt_next;
                }
            }
            // Drain: all issued MMAs complete before Tensor Memory is freed.
            ptx::mma_commit(bar(L::bDrain));
            wait_slow(bar(L::bDrain), 0, wc, false);
        }
        __syncwarp();
    } else {
        // ============================================================ softmax
        const int r = threadIdx.x;  // row within the tile == TMEM lane
        const uint32_t lane_base = static_cast<uint32_t>(warp * 32) << 16;
        const float c2 = p.scale_log2;
        TileCursor c;
        c.start(p);
        uint32_t G = 0;
        float m_run = -CUDART_INF_F;  // running maximum (raw score units)
        float l_run = 0.f;            // running sum, relative to m_run
        while (c.valid(p)) {
            if (!wait_bar_warp(bar(L::bSFull + (G & 1)), (G >> 1) & 1, wc)) break;
            ptx::tc_fence_after();
            const uint32_t s_tmem = tmem + lane_base + (G & 1) * 128;
            uint32_t sr[4][32];
#pragma unroll
            for (int q = 0; q < 4; ++q) ptx::tmem_ld32(s_tmem + q * 32, sr[q]);
            ptx::tmem_wait_ld();
            float s[128];
#pragma unroll
            for (int j = 0; j < 128; ++j) s[j] = __uint_as_float(sr[j >> 5][j & 31]);

            const int row = c.qb * kBlockM + r;
            const int kv0 = c.it * kBlockN;
            const bool diag = p.causal && (kv0 + kBlockN - 1 > c.qb * kBlockM);
            if (diag || kv0 + kBlockN > p.s_k) {
                const int lim_tail = p.s_k - kv0;                // keys >= s_k
                const int lim_causal = p.causal ? row - kv0 + 1 : kBlockN;  // keys > row
                const int lim = min(lim_tail, lim_causal);
#pragma unroll
                for (int j = 0; j < 128; ++j)
                    if (j >= lim) s[j] = -CUDART_INF_F;
            }
            float mx = s[0];
#pragma unroll
            for (int j = 1; j < 128; ++j) mx = fmaxf(mx, s[j]);

            float alpha = 1.f;
            bool rescale = false;
            if (m_run == -CUDART_INF_F) {
                m_run = mx;
            } else if ((mx - m_run) * c2 > kRescaleThresholdLog2) {
                alpha = ptx::ex2((m_run - mx) * c2);
                m_run = mx;
                rescale = true;
            }
            const float m_ref = (m_run == -CUDART_INF_F) ? 0.f : m_run;
            const float neg_mc = -m_ref * c2;
            float sum = 0.f;
            uint32_t pk[64];
#pragma unroll
            for (int j = 0; j < 64; ++j) {
                const float p0 = ptx::ex2(fmaf(s[2 * j], c2, neg_mc));
                const float p1 = ptx::ex2(fmaf(s[2 * j + 1], c2, neg_mc));
                sum += p0 + p1;
                pk[j] = ptx::pack_bf16x2(p0, p1);
            }
            l_run = l_run * alpha + sum;

            // Correction: O *= alpha once the previous P V has landed.
            if (c.it > 0 && __any_sync(0xffffffffu, rescale)) {
                if (!wait_bar_warp(bar(L::bOFull), (G - 1) & 1, wc)) break;
                ptx::tc_fence_after();
                const uint32_t o_tmem = tmem + lane_base + 256;
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    uint32_t ov[32];
                    ptx::tmem_ld32(o_tmem + q * 32, ov);
                    ptx::tmem_wait_ld();
#pragma unroll
                    for (int j = 0; j < 32; ++j)
                        ov[j] = __float_as_uint(__uint_as_float(ov[j]) * alpha);
                    ptx::tmem_st32(o_tmem + q * 32, ov);
                }
                ptx::tmem_wait_st();
            }
            // P (BF16) over the first 64 columns of this S buffer.
            {
                uint32_t lo[32], hi[32];
#pragma unroll
                for (int j = 0; j < 32; ++j) {
                    lo[j] = pk[j];
                    hi[j] = pk[32 + j];
                }
                ptx::tmem_st32(s_tmem, lo);
                ptx::tmem_st32(s_tmem + 32, hi);
                ptx::tmem_wait_st();
            }
            ptx::tc_fence_before();
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive(bar(L::bPFull + (G & 1)));

            if (c.it == c.n_kv - 1) {
                // Epilogue: O / l -> BF16 rows, LSE in natural log.
                if (!wait_bar_warp(bar(L::bOFull), G & 1, wc)) break;
                ptx::tc_fence_after();
                const uint32_t o_tmem = tmem + lane_base + 256;
                const float inv_l = 1.f / l_run;
                uint4* orow = reinterpret_cast<uint4*>(
                    p.o + ((static_cast<size_t>(c.b) * p.s_q + row) * p.h_q + c.h) * kHeadDim);
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    uint32_t ov[32];
                    ptx::tmem_ld32(o_tmem + q * 32, ov);
                    ptx::tmem_wait_ld();
                    if (row < p.s_q) {
#pragma unroll
                        for (int j = 0; j < 4; ++j) {
                            uint4 w;
                            w.x = ptx::pack_bf16x2(__uint_as_float(ov[8 * j + 0]) * inv_l,
                                                   __uint_as_float(ov[8 * j + 1]) * inv_l);
                            w.y = ptx::pack_bf16x2(__uint_as_float(ov[8 * j + 2]) * inv_l,
                                                   __uint_as_float(ov[8 * j + 3]) * inv_l);
                            w.z = ptx::pack_bf16x2(__uint_as_float(ov[8 * j + 4]) * inv_l,
                                                   __uint_as_float(ov[8 * j + 5]) * inv_l);
                            w.w = ptx::pack_bf16x2(__uint_as_float(ov[8 * j + 6]) * inv_l,
                                                   __uint_as_float(ov[8 * j + 7]) * inv_l);
                            orow[q * 4 + j] = w;
                        }
                    }
                }
                ptx::tc_fence_before();
                __syncwarp();
                if (lane == 0) ptx::mbar_arrive(bar(L::bOEmpty));
                if (row < p.s_q) {
                    p.lse[(static_cast<size_t>(c.b) * p.h_q + c.h) * p.s_q + row] =
                        (m_ref * c2 + __log2f(l_run)) * 0.69314718055994531f;
                }
                m_run = -CUDART_INF_F;
                l_run = 0.f;
            }
            ++G;
            c.advance(p);
        }
    }

    ptx::tc_fence_before();
    __syncthreads();
    if (warp == 5) {
        ptx::tc_fence_after();
        ptx::tmem_dealloc(tmem, kTmemCols);
    }
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

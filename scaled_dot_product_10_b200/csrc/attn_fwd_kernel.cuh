// attn_fwd_kernel.cuh -- fused scaled dot-product attention forward for
// B200 (sm_100a): TMA -> shared memory -> tcgen05.mma into Tensor Memory ->
// FP32 online softmax -> P (BF16) in shared memory -> tcgen05.mma -> BF16 O
// and FP32 LSE.
//
// What is computed is the SDPA definition softmax(Q K^T * scale) V (rkmt.cn
// "GPU attention operator optimisation" page, section 1), evaluated the way
// the pages' FlashAttention discussion describes: key/value blocks stream
// through on-chip memory and S is never written to HBM (bjdmk.com.cn page,
// section 5.1), and each block's local softmax is merged into a running
// result ("local attention then global reduction", rkmt.cn page,
// section 3.1.1).  The merge is the exact online-softmax rescaling: with a
// running row maximum m and sum l,
//     m' = max(m, max_j s_j),  l' = l * 2^((m - m') c) + sum_j 2^(s_j c - m' c),
//     O' = O * 2^((m - m') c) + P V,      c = scale * log2(e),
// which equals the definition exactly in exact arithmetic.  The scale is
// folded into the exponent (the AVO page, section 3.1, fuses the scale into
// the QK^T stage) and the mask is applied while the scores sit in registers
// (AVO page, section 2.2).
//
// One CTA step ("pair") covers two adjacent 128-row query blocks of one
// (batch, head) that share every K/V tile.  Warp roles (384 threads):
//   warps 0-3  softmax warpgroup 0: query block 2p   (TMEM lanes = rows)
//   warps 4-7  softmax warpgroup 1: query block 2p+1
//              each also rescales its O when needed and writes its O/LSE
//   warp  8    tcgen05.mma issuer for query block 0 (one lane); TMEM allocator
//   warp  9    TMA producer (one lane)
//   warp 10    tcgen05.mma issuer for query block 1 (one lane)
//   warp 11    idle (completes the control warpgroup for setmaxnreg)
// Tensor Memory (512 columns): S0 | S1 | O0 | O1 at columns 0, 128, 256, 384.
// P_i goes to shared memory (in the layout the MMA reads), so a softmax
// warpgroup hands S_i back as soon as it has loaded the scores: the next
// Q K^T of the block then runs while the current exponentials are computed,
// and the two warpgroups work continuously instead of waiting on their
// block's P V -> Q K^T chain.  Each block has its own issuing lane, so one
// block's events never wait behind the other's; a K or V slot is released
// when both issuers are done with it.
// The two warpgroups take turns on the exponential unit: their exponential
// phases run in a fixed global order (per pair, per key block: block 0, then
// block 1), passed on through a "turn" mbarrier, so one warpgroup's loads,
// row max and waits overlap the other's exponentials instead of both
// warpgroups doing the same phase at the same time.
// Shared memory: Q0, Q1, P0, P1 (32 KiB each), a ring of kKStages K tiles and
// a ring of kVStages V tiles (32 KiB each), all in the 128-byte swizzle that
// TMA writes and tcgen05 reads.  K and V have separate rings: K(j+1) is used
// early in step j (right after the softmax frees S) and released soon after,
// while V(j) is held until the end of step j's softmax, so V gets the
// deeper ring.
//
// Every wait is bounded (per-CTA abort flag plus a global-timer limit); a
// wait that gives up sets the device status word, and the CTA drains its
// in-flight copies and MMAs, frees Tensor Memory and exits.
#pragma once

#include "attn_common.cuh"

namespace sdpa10 {

constexpr int kThreads = 384;
constexpr int kMmaWarp0 = 8;   // issues query block 0's MMAs, allocates TMEM
constexpr int kLoadWarp = 9;
constexpr int kMmaWarp1 = 10;  // issues query block 1's MMAs
// A warpgroup passes the exponential turn on after 12 of its 16 P chunks:
// the next warpgroup's wake-up then overlaps the tail of the loop (measured
// best among hand-off points 6..16 on B200).
constexpr int kTurnChunk = 12;
// Register split (per thread): launched at 65536 / 384 -> 168; the control
// warpgroup (two MMA issuers, TMA, one idle warp) drops to 72 so each softmax
// warpgroup can rise to 216: 2 * 128 * 216 + 128 * 72 = 384 * 168.
constexpr uint32_t kRegsSoftmax = 216;
constexpr uint32_t kRegsControl = 72;

// ------------------------------------------------------------------ schedule
// Items are dealt to the G = gridDim.x persistent CTAs in rounds of G, in a
// snake order: in round k CTA c takes item kG + c when k is even and
// kG + G - 1 - c when k is odd.  Items run longest first (below), so a CTA
// that took a long item in one round takes a short one in the next and the
// causal work per CTA evens out (a plain grid stride gives CTA 0 the longest
// item of every round).
// Work item t -> (pair, key range): pair u = t / n_splits, key range
// t % n_splits (the ranges of one pair are adjacent, so they share its Q
// tiles in L2).  Pair u -> (batch, query head, first query block): pairs are
// grouped in sections of `units_per_section` (batch, kv head) units so the
// K/V of a section stay resident in L2 while its pairs run; inside a section
// the order is pair descending (longest causal work first), then unit, then
// the query heads of the unit's group (adjacent heads share K/V).  Items
// whose key range no row of the pair may see (causal) are skipped by every
// role alike.
//
// With a sliding window (kWindow) the two query blocks of a pair see
// different key intervals: iteration t of the pair's K/V stream is key block
// kb0 + t; block 0 visits iterations 0 .. n[0] - 1 and block 1 iterations
// st1 .. st1 + n[1] - 1 (its window starts st1 key blocks later).
//
// In a packed variable-length batch (kVarlen) "batch" b is sequence b: its
// query rows are cu_q[b] .. cu_q[b+1] - 1 and its keys cu_k[b] .. cu_k[b+1]
// - 1 of the packed tensors, and the pairs past its own length have no work.
template <bool kWindow, bool kVarlen>
struct PairCursor {
    int round;  // rounds of gridDim.x items dealt so far
    int t;
    int b, h, g, qb0;
    int split, kb0;  // key range of the item: key blocks kb0 .. kb0 + n[i] - 1
    int n[2];        // key/value blocks each query block of the pair visits (0: none)
    int st1;         // kWindow: first iteration of block 1 (0 otherwise)
    // kVarlen: the sequence's first packed query row and key, its lengths
    // and its causal offset s_k - s_q.
    int q_row0, k_row0, s_q, s_k, off;

    __device__ __forceinline__ void decode(const FwdParams& p) {
        const int u = p.div_splits.div(t);
        split = t - u * p.n_splits;
        kb0 = split * p.kb_per_split;
        int kb_end = min(p.n_kb, kb0 + p.kb_per_split);
        const int G = p.units_per_section;
        const int sec = p.div_section.div(u);
        const int r = u - sec * G * p.group * p.n_pairs;
        const bool last = sec == p.last_section;
        const int Gs = last ? p.last_units : G;
        const int rank = last ? p.div_rank_last.div(r) : p.div_rank.div(r);
        const int rem = r - rank * Gs * p.group;
        const int unit_in_sec = p.div_group.div(rem);
        const int unit = sec * G + unit_in_sec;
        const int h_local = rem - unit_in_sec * p.group;
        const int pair = p.n_pairs - 1 - rank;
        b = p.div_h_kv.div(unit);
        g = unit - b * p.h_kv;
        h = g * p.group + h_local;
        qb0 = 2 * pair;
        int sq = p.s_q, nqb = p.n_qb, coff = p.causal_offset;
        if constexpr (kVarlen) {
            // No key ranges here (kb0 = 0): the sequence's own extents.
            q_row0 = __ldg(p.cu_q + b);
            s_q = __ldg(p.cu_q + b + 1) - q_row0;
            k_row0 = __ldg(p.cu_k + b);
            s_k = __ldg(p.cu_k + b + 1) - k_row0;
            off = s_k - s_q;
            sq = s_q;
            nqb = max(0, (s_q + kBlockM - 1) >> 7);
            coff = off;
            kb_end = max(0, (s_k + kBlockN - 1) >> 7);
        }
        // Causal: the last row of block qb, min(128 qb + 127, s_q - 1), sees
        // keys up to row + causal_offset (s_k - s_q, or a key shard's own
        // diagonal, which may be negative: floor division by the shift).
        static_assert(kBlockN == 128, "the shift below divides by kBlockN");
        const int last0 = (min(qb0 * kBlockM + kBlockM - 1, sq - 1) + coff) >> 7;
        const int last1 = (min(qb0 * kBlockM + 2 * kBlockM - 1, sq - 1) + coff) >> 7;
        const int vis0 = p.causal ? min(kb_end, last0 + 1) : kb_end;
        const int vis1 = (qb0 + 1 < nqb) ? (p.causal ? min(kb_end, last1 + 1) : kb_end) : 0;
        n[0] = max(0, vis0 - kb0);
        n[1] = max(0, vis1 - kb0);
        if constexpr (kVarlen) {
            if (qb0 >= nqb) n[0] = 0;  // the pair lies past this sequence
        }
        if constexpr (kWindow) {
            // Causal with a window of window_left keys before the diagonal
            // (no key ranges): row r sees keys r + causal_offset -
            // window_left .. r + causal_offset, so a block starts at the key
            // block of its first row's lower bound.
            const int lo0 = max(0, (qb0 * kBlockM + coff - p.window_left) >> 7);
            const int lo1 = max(0, ((qb0 + 1) * kBlockM + coff - p.window_left) >> 7);
            kb0 = lo0;
            n[0] = max(0, vis0 - lo0);
            st1 = lo1 - lo0;
            n[1] = (qb0 + 1 < nqb) ? max(0, vis1 - lo1) : 0;
            if constexpr (kVarlen) {
                if (qb0 >= nqb) n[0] = 0;
            }
        } else {
            st1 = 0;
        }
    }
    // This CTA's item of the current round, moving on past items with no
    // work.  Positions only grow from round to round, so the first one past
    // the last item ends the walk.
    __device__ __forceinline__ void settle(const FwdParams& p) {
        for (;; ++round) {
            const int c = static_cast<int>(blockIdx.x);
            const int g = static_cast<int>(gridDim.x);
            t = round * g + ((round & 1) ? g - 1 - c : c);
            if (t >= p.num_tiles) return;
            decode(p);
            if (n[0] > 0 || n[1] > 0) return;
        }
    }
    __device__ __forceinline__ void start(const FwdParams& p) {
        round = 0;
        settle(p);
    }
    __device__ __forceinline__ void next(const FwdParams& p) {
        ++round;
        settle(p);
    }
    __device__ __forceinline__ bool valid(const FwdParams& p) const { return t < p.num_tiles; }
    __device__ __forceinline__ int iters() const {
        if constexpr (kWindow) return max(n[0], st1 + n[1]);
        return max(n[0], n[1]);
    }
    // Iterations both blocks visit, [common_begin, common_end) (may be empty).
    __device__ __forceinline__ int common_begin() const { return st1; }
    __device__ __forceinline__ int common_end() const { return min(n[0], st1 + n[1]); }
};

// ------------------------------------------------------------------ layout
// BF16: 32 KiB Q/K/V/P tiles, a K ring of 1 and a V ring of 2, O staged in
// the block's P tile.  FP8 (E4M3): 16 KiB tiles (a 128-byte row is one
// swizzle atom), deeper rings, and a BF16 O staging tile per block.
template <bool kFp8>
struct SmemLayoutT {
    static constexpr int kTile = kFp8 ? kTileBytes / 2 : kTileBytes;
    static constexpr int kKStages = kFp8 ? 2 : 1;  // K tiles in flight
    static constexpr int kVStages = kFp8 ? 3 : 2;  // V tiles in flight
    static constexpr int kQ = 0;                              // Q0, Q1
    static constexpr int kP = 2 * kTile;                      // P0, P1
    static constexpr int kK = 4 * kTile;                      // K ring
    static constexpr int kV = kK + kKStages * kTile;          // V ring
    static constexpr int kO = kV + kVStages * kTile;          // FP8: O staging (2 x 32 KiB)
    static constexpr int kBars = kO + (kFp8 ? 2 * kTileBytes : 0);  // mbarriers
    static constexpr int bQFull = 0, bQEmpty = 2, bKFull = 4, bKEmpty = 4 + kKStages,
                         bVFull = 4 + 2 * kKStages, bVEmpty = bVFull + kVStages,
                         bSFull = bVEmpty + kVStages,
                         bSFree = bSFull + 2, bPFull = bSFree + 2, bOFull = bPFull + 2,
                         bOEmpty = bOFull + 2, bTurn = bOEmpty + 2, bDrain = bTurn + 1,
                         bOStaged = bDrain + 2, bOStored = bOStaged + 2,
                         kNumBars = bOStored + 2;
    static constexpr int kTmemSlot = kBars + kNumBars * 8;
    // Leading offset of the V descriptor (MN-major): the second 64-column
    // head-dim half for BF16; FP8 rows are one atom wide, so it is not used.
    static constexpr uint32_t kFp8Lbo = kFp8 ? kTile : kHalfTileBytes;
    static constexpr int kAbort = kTmemSlot + 4;
    static constexpr int kBytes = kAbort + 4;
    static constexpr int kAlloc = kBytes + 1024;  // slack for 1024-byte alignment
};
using SmemLayout = SmemLayoutT<false>;

// FP8 P: the lazy rescale threshold is 2^2 and the weights are stored as
// 2^6 * P, so a row's weights span up to 2^8 at the top and keep E4M3's
// normal range (down to 2^-6, i.e. P >= 2^-12) for the bulk of the mass;
// the 2^6 cancels in O / l and is taken out of the LSE.
constexpr float kFp8RescaleThresholdLog2 = 2.0f;
constexpr float kFp8PBiasLog2 = 6.0f;

// ------------------------------------------------------------------ exponentials
// P = 2^(s c - m c) for one 128-key row on the MUFU ex2 unit: FP32 row sum
// returned in two accumulators, BF16 P written to this row of the
// shared-memory P tile (16-byte chunk cc at row_base + (cc / 8) * 16 KiB +
// ((cc % 8) ^ xor) * 16).  When `pass_turn` is set the warp arrives on the
// turn barrier after kTurnChunk chunks.
template <bool kFp8>
__device__ __forceinline__ void exp_row(const float (&s)[128], uint64_t c2x2, uint64_t nmc2,
                                        uint32_t p_row, uint32_t p_xor, float& sum_a,
                                        float& sum_b, bool pass_turn, uint32_t turn, int lane) {
    uint64_t sum2a = ptx::f2_pack(0.f, 0.f), sum2b = sum2a;
    uint32_t w8[4];  // FP8: two 8-key groups make one 16-byte chunk
#pragma unroll
    for (int cc = 0; cc < 16; ++cc) {
        uint32_t w[4];
        float pv[8];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            const int e0 = 8 * cc + 2 * k;
            const uint64_t x = ptx::f2_fma(ptx::f2_pack(s[e0], s[e0 + 1]), c2x2, nmc2);
            float x0, x1;
            ptx::f2_unpack(x, x0, x1);
            const float p0 = ptx::ex2(x0), p1 = ptx::ex2(x1);
            const uint64_t e = ptx::f2_pack(p0, p1);
            if (k & 1) sum2b = ptx::f2_add(sum2b, e);
            else sum2a = ptx::f2_add(sum2a, e);
            if constexpr (kFp8) {
                pv[2 * k] = p0;
                pv[2 * k + 1] = p1;
            } else {
                w[k] = ptx::pack_bf16x2(p0, p1);
            }
        }
        if constexpr (kFp8) {
            // Row of 128 E4M3 weights = one 128-byte swizzle atom row:
            // 16-byte chunk c (keys 16c .. 16c + 15) at ((c ^ xor) * 16).
            w8[2 * (cc & 1)] = ptx::pack_e4m3x4(pv[0], pv[1], pv[2], pv[3]);
            w8[2 * (cc & 1) + 1] = ptx::pack_e4m3x4(pv[4], pv[5], pv[6], pv[7]);
            if (cc & 1)
                ptx::st_shared_v4(p_row + ((((cc >> 1) & 7) ^ p_xor) << 4), w8[0], w8[1], w8[2],
                                  w8[3]);
        } else {
            ptx::st_shared_v4(p_row + (cc >> 3) * kHalfTileBytes + (((cc & 7) ^ p_xor) << 4),
                              w[0], w[1], w[2], w[3]);
        }
        if (cc == kTurnChunk - 1 && pass_turn) {
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive(turn);
        }
    }
    float a0, a1, b0, b1;
    ptx::f2_unpack(sum2a, a0, a1);
    ptx::f2_unpack(sum2b, b0, b1);
    sum_a += a0 + a1;
    sum_b += b0 + b1;
}

// ------------------------------------------------------------------ softmax
// One softmax warpgroup: thread r owns query row r of its block (TMEM lane r).
template <bool kWindow, bool kVarlen, bool kFp8>
__device__ __forceinline__ void softmax_role(const FwdParams& p, const CUtensorMap* tm_o,
                                             const WaitCtx& wc, uint32_t tmem, uint32_t sP,
                                             uint32_t sO, uint32_t bars, int wg, int warp_in_wg,
                                             int lane) {
    using L = SmemLayoutT<kFp8>;
    auto bar = [&](int i) -> uint32_t { return bars + 8u * static_cast<uint32_t>(i); };
    const int r = warp_in_wg * 32 + lane;
    const uint32_t lane_base = static_cast<uint32_t>(warp_in_wg * 32) << 16;
    const uint32_t s_tmem = tmem + lane_base + wg * 128;
    const uint32_t o_tmem = tmem + lane_base + 256 + wg * 128;
    const uint32_t b_sfull = bar(L::bSFull + wg), b_sfree = bar(L::bSFree + wg);
    const uint32_t b_pfull = bar(L::bPFull + wg);
    const uint32_t b_ofull = bar(L::bOFull + wg), b_oempty = bar(L::bOEmpty + wg);
    const uint32_t b_ostaged = bar(L::bOStaged + wg), b_ostored = bar(L::bOStored + wg);
    // This row of P in shared memory (K-major, 128-byte swizzle, two 64-key
    // halves 16 KiB apart): 16-byte chunk c of the row lands at
    // row_base + (c / 8) * 16 KiB + ((c % 8) ^ (r % 8)) * 16.
    const uint32_t p_row = sP + wg * L::kTile + (r >> 3) * 1024 + (r & 7) * 128;
    const uint32_t p_xor = static_cast<uint32_t>(r & 7);
    // The BF16 O tile of this block is staged at o_tile before its TMA store
    // (the block's P tile for BF16 inputs).
    const uint32_t o_tile = (kFp8 ? sO : sP) + wg * kTileBytes;
    const uint32_t o_row = o_tile + (r >> 3) * 1024 + (r & 7) * 128;
    constexpr float kThreshold = kFp8 ? kFp8RescaleThresholdLog2 : kRescaleThresholdLog2;
    const float c2 = p.scale_log2;
    const uint64_t c2x2 = ptx::f2_pack(c2, c2);

    const uint32_t b_turn = bar(L::bTurn);
    // Exponential turns strictly alternate: at key block j < min(n0, n1) of
    // a pair, block 0 takes turn 2K and block 1 turn 2K + 1 (K counts such
    // rounds over all pairs); a block's key blocks past that run without a
    // turn.  Each wait then finds the turn barrier at most one phase short,
    // which its single parity bit can tell apart.
    uint32_t cnt = 0;     // S blocks this warpgroup has processed (all pairs)
    uint32_t stored = 0;  // O tiles this warpgroup has stored through TMA
    uint32_t rounds = 0;  // alternation rounds before this pair
    PairCursor<kWindow, kVarlen> c;
    c.start(p);
    for (; c.valid(p); c.next(p)) {
        const int n = c.n[wg];
        int n_turns, t0 = 0, cb = 0;
        if constexpr (kWindow) {
            // Turns over the iterations both blocks visit; this block's
            // local step j is iteration t0 + j.
            cb = c.common_begin();
            n_turns = max(0, c.common_end() - cb);
            t0 = wg ? c.st1 : 0;
        } else {
            n_turns = min(c.n[0], c.n[1]);
        }
        const uint32_t round0 = rounds;
        rounds += static_cast<uint32_t>(n_turns);
        if (n == 0) continue;
        const int qb = c.qb0 + wg;
        const int row = qb * kBlockM + r;
        float m_run = -CUDART_INF_F;  // running maximum (raw score units)
        float l_run = 0.f;            // running sum, relative to m_run
        for (int j = 0; j < n; ++j, ++cnt) {
            if (!wait_bar_warp(b_sfull, cnt & 1, wc)) return;
            ptx::tc_fence_after();
            float s[128];
            {
                uint32_t sr[4][32];
#pragma unroll
                for (int q = 0; q < 4; ++q) ptx::tmem_ld32(s_tmem + q * 32, sr[q]);
                ptx::tmem_wait_ld();
#pragma unroll
                for (int k = 0; k < 128; ++k) s[k] = __uint_as_float(sr[k >> 5][k & 31]);
            }
            // The scores are in registers: S_i may take the next Q K^T.
            ptx::tc_fence_before();
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive(b_sfree);

            const int kv0 = (c.kb0 + t0 + j) * kBlockN;
            int seq_k = p.s_k, coff = p.causal_offset;
            if constexpr (kVarlen) {
                seq_k = c.s_k;
                coff = c.off;
            }
            const bool diag = p.causal && (kv0 + kBlockN - 1 > qb * kBlockM + coff);
            bool masked = diag || kv0 + kBlockN > seq_k;
            if constexpr (kWindow) {
                // keys before the last row's window start
                masked = masked || kv0 < qb * kBlockM + kBlockM - 1 + coff - p.window_left;
            }
            if (masked) {
                const int lim_tail = seq_k - kv0;                           // keys >= s_k
                // keys past row + s_k - s_q
                const int lim_causal = p.causal ? row + coff - kv0 + 1 : kBlockN;
                const int lim = min(lim_tail, lim_causal);
                if constexpr (kWindow) {
                    // and keys before row + s_k - s_q - window_left
                    const int lo = row + coff - p.window_left - kv0;
#pragma unroll
                    for (int k = 0; k < 128; ++k)
                        if (k >= lim || k < lo) s[k] = -CUDART_INF_F;
                } else {
#pragma unroll
                    for (int k = 0; k < 128; ++k)
                        if (k >= lim) s[k] = -CUDART_INF_F;
                }
            }
            float mx;
            {
                // Eight independent 3-input-max chains, then combine.
                float m8[8];
#pragma unroll
                for (int k = 0; k < 8; ++k) m8[k] = fmaxf(s[2 * k], s[2 * k + 1]);
#pragma unroll
                for (int k = 16; k < 128; k += 16) {
#pragma unroll
                    for (int t = 0; t < 8; ++t) m8[t] = ptx::max3(m8[t], s[k + 2 * t], s[k + 2 * t + 1]);
                }
                mx = ptx::max3(ptx::max3(m8[0], m8[1], m8[2]), ptx::max3(m8[3], m8[4], m8[5]),
                               fmaxf(m8[6], m8[7]));
            }
            float alpha = 1.f;
            bool rescale = false;
            if (m_run == -CUDART_INF_F) {
                m_run = mx;
            } else if ((mx - m_run) * c2 > kThreshold) {
                alpha = ptx::ex2((m_run - mx) * c2);
                m_run = mx;
                rescale = true;
            }
            const float m_ref = (m_run == -CUDART_INF_F) ? 0.f : m_run;
            float neg_mc = -m_ref * c2;
            if constexpr (kFp8) neg_mc += kFp8PBiasLog2;  // weights stored as 2^6 P

            // The previous P V of this block must be done before its P
            // buffer is rewritten (and before O is rescaled).
            if (cnt > 0 && !wait_bar_warp(b_ofull, (cnt - 1) & 1, wc)) return;
            if (j > 0 && __any_sync(0xffffffffu, rescale)) {
                // Correction: O *= alpha.
                ptx::tc_fence_after();
                const uint64_t a2 = ptx::f2_pack(alpha, alpha);
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    uint32_t ov[32];
                    ptx::tmem_ld32(o_tmem + q * 32, ov);
                    ptx::tmem_wait_ld();
#pragma unroll
                    for (int k = 0; k < 16; ++k) {
                        uint64_t v = ptx::f2_mul(ptx::f2_pack(__uint_as_float(ov[2 * k]),
                                                              __uint_as_float(ov[2 * k + 1])),
                                                 a2);
                        float lo, hi;
                        ptx::f2_unpack(v, lo, hi);
                        ov[2 * k] = __float_as_uint(lo);
                        ov[2 * k + 1] = __float_as_uint(hi);
                    }
                    ptx::tmem_st32(o_tmem + q * 32, ov);
                }
                ptx::tmem_wait_st();
                ptx::tc_fence_before();
            }

            // Our turn on the exponential unit: wait for turn m - 1.
            bool turn;
            uint32_t m;
            if constexpr (kWindow) {
                const int tc = t0 + j - cb;  // position in the common interval
                turn = tc >= 0 && tc < n_turns;
                m = 2 * (round0 + tc) + wg;
            } else {
                turn = j < n_turns;
                m = 2 * (round0 + j) + wg;
            }
            if (turn && m > 0 && !wait_bar_warp(b_turn, (m - 1) & 1, wc)) return;
            float sum_a = 0.f, sum_b = 0.f;
            exp_row<kFp8>(s, c2x2, ptx::f2_pack(neg_mc, neg_mc), p_row, p_xor, sum_a, sum_b, turn,
                          b_turn, lane);
            // Make P visible to the tensor core (async proxy) and hand it over.
            ptx::fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive(b_pfull);
            l_run = l_run * alpha + (sum_a + sum_b);

            if (j == n - 1) {
                // Epilogue: O / l -> BF16 rows (or FP32 partial rows of a key
                // range), LSE in natural log.
                if (!wait_bar_warp(b_ofull, cnt & 1, wc)) return;
                ptx::tc_fence_after();
                float inv_l = 1.f / l_run;
                if constexpr (kVarlen) {
                    // A causal row of a sequence with fewer keys than
                    // queries may see no key: O = 0 (LSE = -inf).
                    inv_l = l_run > 0.f ? inv_l : 0.f;
                }
                if constexpr (kFp8) inv_l *= p.v_scale;  // V = v_scale * E4M3 values
                const uint64_t il2 = ptx::f2_pack(inv_l, inv_l);
                float log2_l = __log2f(l_run);
                if constexpr (kFp8) log2_l -= kFp8PBiasLog2;
                const float lse_row = (m_ref * c2 + log2_l) * 0.69314718055994531f;
                const size_t row_id = (static_cast<size_t>(c.b) * p.h_q + c.h) * p.s_q + row;
                if (p.o_part != nullptr) {
                    // A row of a key shard may see none of its keys (l = 0):
                    // O = 0 and LSE = -inf, so a merge gives it no weight.
                    const float inv_lp = l_run > 0.f ? inv_l : 0.f;
                    const uint64_t il2p = ptx::f2_pack(inv_lp, inv_lp);
                    const size_t part =
                        static_cast<size_t>(c.split) * p.batch * p.h_q * p.s_q + row_id;
                    float4* frow = reinterpret_cast<float4*>(p.o_part + part * kHeadDim);
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        uint32_t ov[32];
                        ptx::tmem_ld32(o_tmem + q * 32, ov);
                        ptx::tmem_wait_ld();
                        if (row < p.s_q) {
#pragma unroll
                            for (int k = 0; k < 8; ++k) {
                                float a0, a1, b0, b1;
                                ptx::f2_unpack(ptx::f2_mul(ptx::f2_pack(__uint_as_float(ov[4 * k]),
                                                                        __uint_as_float(ov[4 * k + 1])),
                                                           il2p),
                                               a0, a1);
                                ptx::f2_unpack(ptx::f2_mul(ptx::f2_pack(__uint_as_float(ov[4 * k + 2]),
                                                                        __uint_as_float(ov[4 * k + 3])),
                                                           il2p),
                                               b0, b1);
                                frow[q * 8 + k] = make_float4(a0, a1, b0, b1);
                            }
                        }
                    }
                    ptx::tc_fence_before();
                    __syncwarp();
                    if (lane == 0) ptx::mbar_arrive(b_oempty);
                    if (row < p.s_q) p.lse_part[part] = lse_row;
                } else {
                    // BF16 O rows go to this block's P buffer (free: the last
                    // P V has completed) in the tile layout TMA reads, and
                    // one thread stores the tile with two TMA copies (rows
                    // past s_q are clipped by the tensor map).  In a packed
                    // batch a sequence's last, partial tile is written row
                    // by row instead (a tile store would overwrite the next
                    // sequence's rows); every row stays inside the packed
                    // tensor even if cu_seqlens are inconsistent.
                    bool tma_tile = true;
                    bool row_ok = true;
                    __nv_bfloat16* orow = nullptr;
                    if constexpr (kVarlen) {
                        tma_tile = (qb + 1) * kBlockM <= c.s_q &&
                                   c.q_row0 + (qb + 1) * kBlockM <= p.total_q;
                        row_ok = row < c.s_q && c.q_row0 + row < p.total_q;
                        orow = p.o + (static_cast<size_t>(c.q_row0 + row) * p.h_q + c.h) * kHeadDim;
                    }
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        uint32_t ov[32];
                        ptx::tmem_ld32(o_tmem + q * 32, ov);
                        ptx::tmem_wait_ld();
                        uint32_t w[16];
#pragma unroll
                        for (int k = 0; k < 16; ++k) {
                            const uint64_t v = ptx::f2_mul(
                                ptx::f2_pack(__uint_as_float(ov[2 * k]), __uint_as_float(ov[2 * k + 1])),
                                il2);
                            float lo, hi;
                            ptx::f2_unpack(v, lo, hi);
                            w[k] = ptx::pack_bf16x2(lo, hi);
                        }
                        if (tma_tile) {
#pragma unroll
                            for (int k = 0; k < 4; ++k) {
                                const int cc = 4 * q + k;
                                ptx::st_shared_v4(
                                    o_row + (cc >> 3) * kHalfTileBytes + (((cc & 7) ^ p_xor) << 4),
                                    w[4 * k], w[4 * k + 1], w[4 * k + 2], w[4 * k + 3]);
                            }
                        } else if (row_ok) {
#pragma unroll
                            for (int k = 0; k < 4; ++k)
                                reinterpret_cast<uint4*>(orow)[4 * q + k] =
                                    make_uint4(w[4 * k], w[4 * k + 1], w[4 * k + 2], w[4 * k + 3]);
                        }
                    }
                    ptx::tc_fence_before();
                    __syncwarp();
                    if (lane == 0) ptx::mbar_arrive(b_oempty);
                    // Rows staged (all four warps) -> thread 0 stores the tile
                    // and waits until TMA has read it -> the P buffer is free.
                    ptx::fence_proxy_async_smem();
                    __syncwarp();
                    if (lane == 0) ptx::mbar_arrive(b_ostaged);
                    if (r == 0) {
                        if (!wait_bar(b_ostaged, stored & 1, wc)) return;
                        if (tma_tile) {
                            const uint32_t tile = o_tile;
                            int row0 = qb * kBlockM, bc = c.b;
                            if constexpr (kVarlen) {
                                row0 += c.q_row0;  // packed rows, batch extent 1
                                bc = 0;
                            }
                            ptx::tma_store_4d(tm_o, tile, 0, c.h, row0, bc);
                            ptx::tma_store_4d(tm_o, tile + kHalfTileBytes, 64, c.h, row0, bc);
                            ptx::bulk_commit_group();
                            ptx::bulk_wait_group_read0();
                        }
                        ptx::mbar_arrive(b_ostored);
                    }
                    if (!wait_bar_warp(b_ostored, stored & 1, wc)) return;
                    ++stored;
                    if constexpr (kVarlen) {
                        // LSE [h_q][total_q]
                        if (row_ok)
                            p.lse[static_cast<size_t>(c.h) * p.total_q + c.q_row0 + row] = lse_row;
                    } else {
                        if (row < p.s_q) p.lse[row_id] = lse_row;
                    }
                }
            }
        }
    }
    if (r == 0) ptx::bulk_wait_group0();  // the last O tile has reached global memory
}

// ------------------------------------------------------------------ kernel
template <bool kWindow, bool kVarlen, bool kFp8 = false>
__global__ void __launch_bounds__(kThreads, 1)
    attn_fwd_sm100_kernel(const __grid_constant__ CUtensorMap tm_q,
                          const __grid_constant__ CUtensorMap tm_k,
                          const __grid_constant__ CUtensorMap tm_v,
                          const __grid_constant__ CUtensorMap tm_o,
                          const __grid_constant__ FwdParams p) {
    using L = SmemLayoutT<kFp8>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    const uint32_t sbase = ptx::smem_u32(smem);
    const uint32_t sQ = sbase + L::kQ;
    const uint32_t sP = sbase + L::kP;
    const uint32_t sK = sbase + L::kK;
    const uint32_t sV = sbase + L::kV;
    const uint32_t sO = sbase + L::kO;
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
            ptx::mbar_init(bar(L::bSFree + i), 4);
            ptx::mbar_init(bar(L::bPFull + i), 4);
            ptx::mbar_init(bar(L::bOFull + i), 1);
            ptx::mbar_init(bar(L::bOEmpty + i), 4);
            ptx::mbar_init(bar(L::bOStaged + i), 4);  // the 4 warps' rows are staged
            ptx::mbar_init(bar(L::bOStored + i), 1);  // TMA has read the staged tile
        }
        for (int i = 0; i < L::kKStages; ++i) {
            ptx::mbar_init(bar(L::bKFull + i), 1);
            ptx::mbar_init(bar(L::bKEmpty + i), 2);  // one arrival per MMA issuer
        }
        for (int i = 0; i < L::kVStages; ++i) {
            ptx::mbar_init(bar(L::bVFull + i), 1);
            ptx::mbar_init(bar(L::bVEmpty + i), 2);
        }
        ptx::mbar_init(bar(L::bDrain + 1), 1);
        ptx::mbar_init(bar(L::bTurn), 4);  // the 4 warps of the finishing warpgroup
        ptx::mbar_init(bar(L::bDrain), 1);
        *abort_flag = 0;
        ptx::fence_mbar_init();
    }
    if (warp == kLoadWarp && lane == 0) {
        ptx::prefetch_tmap(&tm_q);
        ptx::prefetch_tmap(&tm_k);
        ptx::prefetch_tmap(&tm_v);
        ptx::prefetch_tmap(&tm_o);
    }
    if (warp == kMmaWarp0) {
        ptx::tmem_alloc(ptx::smem_u32(tmem_slot), kTmemCols);
        ptx::tmem_relinquish();
    }
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const WaitCtx wc{abort_flag, p.status, p.timeout_ns};

    if (warp == kLoadWarp) {
        // ============================================================ producer
        ptx::reg_dealloc<kRegsControl>();
        if (lane == 0) {
            const uint64_t pol_kv = ptx::policy_evict_last();
            const uint64_t pol_q = ptx::policy_evict_first();
            uint32_t k_loads = 0, v_loads = 0;  // K / V tiles issued
            uint32_t q_loads[2] = {0, 0};
            bool ok = true;
            auto load_tile = [&](const CUtensorMap* tm, uint32_t dst, uint32_t full,
                                 const PairCursor<kWindow, kVarlen>& c,
                                 int j) {
                ptx::mbar_arrive_expect_tx(full, L::kTile);
                int key0 = (c.kb0 + j) * kBlockN, bc = c.b;
                if constexpr (kVarlen) {
                    key0 += c.k_row0;  // packed keys, batch extent 1
                    bc = 0;
                }
                ptx::tma_load_4d(dst, tm, full, 0, c.g, key0, bc, pol_kv);
                if constexpr (!kFp8)
                    ptx::tma_load_4d(dst + kHalfTileBytes, tm, full, 64, c.g, key0, bc, pol_kv);
            };
            auto load_k = [&](const PairCursor<kWindow, kVarlen>& c, int j) -> bool {
                const int slot = k_loads % L::kKStages;
                if (!wait_bar(bar(L::bKEmpty + slot), ((k_loads / L::kKStages) & 1) ^ 1, wc))
                    return false;
                load_tile(&tm_k, sK + slot * L::kTile, bar(L::bKFull + slot), c, j);
                ++k_loads;
                return true;
            };
            auto load_v = [&](const PairCursor<kWindow, kVarlen>& c, int j) -> bool {
                const int slot = v_loads % L::kVStages;
                if (!wait_bar(bar(L::bVEmpty + slot), ((v_loads / L::kVStages) & 1) ^ 1, wc))
                    return false;
                load_tile(&tm_v, sV + slot * L::kTile, bar(L::bVFull + slot), c, j);
                ++v_loads;
                return true;
            };
            PairCursor<kWindow, kVarlen> c;
            c.start(p);
            for (; ok && c.valid(p); c.next(p)) {
#pragma unroll
                for (int i = 0; i < 2; ++i) {
                    if (!ok || c.n[i] == 0) continue;
                    if (!wait_bar(bar(L::bQEmpty + i), (q_loads[i] & 1) ^ 1, wc)) {
                        ok = false;
                        continue;
                    }
                    const uint32_t dst = sQ + i * L::kTile;
                    int row0 = (c.qb0 + i) * kBlockM, bc = c.b;
                    if constexpr (kVarlen) {
                        row0 += c.q_row0;
                        bc = 0;
                    }
                    ptx::mbar_arrive_expect_tx(bar(L::bQFull + i), L::kTile);
                    ptx::tma_load_4d(dst, &tm_q, bar(L::bQFull + i), 0, c.h, row0, bc, pol_q);
                    if constexpr (!kFp8)
                        ptx::tma_load_4d(dst + kHalfTileBytes, &tm_q, bar(L::bQFull + i), 64, c.h,
                                         row0, bc, pol_q);
                    ++q_loads[i];
                }
                // Issue order = the MMA warp's consumption order:
                // K0, then for each step j: K(j+1), V(j).
                const int n = c.iters();
                if (ok) ok = load_k(c, 0);
                for (int j = 0; j < n && ok; ++j) {
                    if (j + 1 < n) ok = load_k(c, j + 1);
                    if (ok) ok = load_v(c, j);
                }
            }
            // Drain: every issued copy must land before the CTA may exit.
            for (int i = 0; i < L::kKStages && i < static_cast<int>(k_loads); ++i) {
                const uint32_t f = k_loads - 1 - i;
                wait_slow(bar(L::bKFull + f % L::kKStages), (f / L::kKStages) & 1, wc, false);
            }
            for (int i = 0; i < L::kVStages && i < static_cast<int>(v_loads); ++i) {
                const uint32_t f = v_loads - 1 - i;
                wait_slow(bar(L::bVFull + f % L::kVStages), (f / L::kVStages) & 1, wc, false);
            }
#pragma unroll
            for (int i = 0; i < 2; ++i)
                if (q_loads[i] > 0)
                    wait_slow(bar(L::bQFull + i), (q_loads[i] - 1) & 1, wc, false);
        }
        __syncwarp();
    } else if (warp == kMmaWarp0 || warp == kMmaWarp1) {
        // ============================================================ MMA issuers
        ptx::reg_dealloc<kRegsControl>();
        if (lane == 0) {
            const int i = (warp == kMmaWarp0) ? 0 : 1;  // query block this lane serves
            const uint32_t idesc_qk = p.idesc_qk;
            constexpr uint32_t kIdescPV = idesc_bf16_f32(kBlockM, kHeadDim, 0, 1);
            uint32_t k_used = 0, v_used = 0;  // K / V tiles passed (used or skipped)
            uint32_t started = 0;             // pairs in which query block i was active
            uint32_t s_cnt = 0, pv_cnt = 0;   // Q K^T / P V groups issued
            bool ok = true;
            // Descriptor low words (start address >> 4 | leading offset).
            const uint32_t q_lo = desc_lo_sw128(sQ + i * L::kTile, 16);
            const uint32_t p_lo = desc_lo_sw128(sP + i * L::kTile, 16);
            const uint32_t k_lo = desc_lo_sw128(sK, 16);
            const uint32_t v_lo = desc_lo_sw128(sV, L::kFp8Lbo);
            const uint32_t s_tm = tmem + i * 128, o_tm = tmem + 256 + i * 128;
            auto wait_k = [&]() -> bool {
                return wait_bar(bar(L::bKFull + k_used % L::kKStages), (k_used / L::kKStages) & 1,
                                wc);
            };
            auto wait_v = [&]() -> bool {
                return wait_bar(bar(L::bVFull + v_used % L::kVStages), (v_used / L::kVStages) & 1,
                                wc);
            };
            // A tile this block does not use: once it has landed (so the slot's
            // previous use is released), give up this issuer's share of it.
            auto skip_k = [&]() -> bool {
                if (!wait_k()) return false;
                ptx::mbar_arrive(bar(L::bKEmpty + k_used % L::kKStages));
                ++k_used;
                return true;
            };
            auto skip_v = [&]() -> bool {
                if (!wait_v()) return false;
                ptx::mbar_arrive(bar(L::bVEmpty + v_used % L::kVStages));
                ++v_used;
                return true;
            };
            // S_i = Q_i K^T once warpgroup i has read its previous S.
            auto qk = [&](bool last_of_pair) -> bool {
                if (!wait_k()) return false;
                if (s_cnt > 0 && !wait_bar(bar(L::bSFree + i), (s_cnt - 1) & 1, wc)) return false;
                ptx::tc_fence_after();
                const uint32_t ka = k_lo + (((k_used % L::kKStages) * L::kTile) >> 4);
                if constexpr (kFp8) {
                    // K-major, 128-byte swizzle: 32 E4M3 (32 bytes) per step;
                    // a 128-element row is one swizzle atom.
#pragma unroll
                    for (int k = 0; k < kHeadDim / 32; ++k)
                        ptx::mma_ss_f8(s_tm, desc_from_lo(q_lo + 2 * k), desc_from_lo(ka + 2 * k),
                                       idesc_qk, k > 0 ? 1u : 0u);
                } else {
#pragma unroll
                    for (int k = 0; k < kHeadDim / 16; ++k) {
                        // K-major, 128-byte swizzle: 16 BF16 (32 bytes) per step
                        // inside a 64-column half; the second half is 16 KiB on.
                        const uint32_t off = ((k >> 2) * kHalfTileBytes + (k & 3) * 32) >> 4;
                        ptx::mma_ss(s_tm, desc_from_lo(q_lo + off), desc_from_lo(ka + off),
                                    idesc_qk, k > 0 ? 1u : 0u);
                    }
                }
                ptx::mma_commit(bar(L::bSFull + i));
                if (last_of_pair) ptx::mma_commit(bar(L::bQEmpty + i));
                ptx::mma_commit(bar(L::bKEmpty + k_used % L::kKStages));
                ++k_used;
                ++s_cnt;
                return true;
            };
            // O_i += P_i V once P_i is in shared memory.
            auto pv = [&](bool acc) -> bool {
                if (!wait_v()) return false;
                if (!wait_bar(bar(L::bPFull + i), pv_cnt & 1, wc)) return false;
                ptx::tc_fence_after();
                const uint32_t va = v_lo + (((v_used % L::kVStages) * L::kTile) >> 4);
                if constexpr (kFp8) {
                    // A = P (E4M3, K-major like Q): 32 keys (32 bytes) per
                    // step; B = V, MN-major (head dim contiguous, one
                    // 128-byte atom wide): 32 keys = 32 rows = 4 KiB per step.
                    constexpr uint32_t kIdescPV8 = idesc_e4m3_f32(kBlockM, kHeadDim, 0, 1);
#pragma unroll
                    for (int k = 0; k < kBlockN / 32; ++k)
                        ptx::mma_ss_f8(o_tm, desc_from_lo(p_lo + 2 * k),
                                       desc_from_lo(va + ((k * 4096) >> 4)), kIdescPV8,
                                       (acc || k > 0) ? 1u : 0u);
                } else {
#pragma unroll
                    for (int k = 0; k < kBlockN / 16; ++k) {
                        // A = P (K-major like Q); B = V, MN-major (head dim
                        // contiguous): 16 keys = two 8-row swizzle atoms = 2 KiB
                        // per step; the two 64-wide head-dim halves are 16 KiB apart.
                        const uint32_t off = ((k >> 2) * kHalfTileBytes + (k & 3) * 32) >> 4;
                        ptx::mma_ss(o_tm, desc_from_lo(p_lo + off),
                                    desc_from_lo(va + ((k * 2048) >> 4)), kIdescPV,
                                    (acc || k > 0) ? 1u : 0u);
                    }
                }
                ptx::mma_commit(bar(L::bOFull + i));
                ptx::mma_commit(bar(L::bVEmpty + v_used % L::kVStages));
                ++v_used;
                ++pv_cnt;
                return true;
            };
            PairCursor<kWindow, kVarlen> c;
            c.start(p);
            for (; ok && c.valid(p); c.next(p)) {
                const int n = c.iters();
                const int ni = c.n[i];
                if constexpr (kWindow) {
                    // Block i visits iterations [st, st + ni) of the pair's
                    // K/V stream; other tiles are passed on.  Tile order (the
                    // producer's): K(0), then per step j: K(j+1), V(j).
                    const int st = i ? c.st1 : 0;
                    auto in_range = [&](int t) { return ni > 0 && t >= st && t < st + ni; };
                    auto scores = [&](int t) -> bool {
                        if (!in_range(t)) return skip_k();
                        if (t == st) {
                            if (!wait_bar(bar(L::bQFull + i), started & 1, wc)) return false;
                            ++started;
                        }
                        return qk(t == st + ni - 1);
                    };
                    if (!(ok = scores(0))) break;
                    for (int j = 0; j < n && ok; ++j) {
                        if (j + 1 < n && !(ok = scores(j + 1))) break;
                        if (in_range(j)) {
                            if (j == st && started > 1 &&
                                !(ok = wait_bar(bar(L::bOEmpty + i), started & 1, wc)))
                                break;
                            ok = pv(j > st);
                        } else {
                            ok = skip_v();
                        }
                    }
                    continue;
                }
                // Tile order (the producer's): K0, then per step j: K(j+1), V(j).
                if (ni > 0) {
                    if (!(ok = wait_bar(bar(L::bQFull + i), started & 1, wc))) break;
                    ++started;
                    if (!(ok = qk(ni == 1))) break;
                } else if (!(ok = skip_k())) {
                    break;
                }
                for (int j = 0; j < n && ok; ++j) {
                    // Next scores first: they are what the softmax waits for.
                    if (j + 1 < n) ok = (j + 1 < ni) ? qk(j + 2 == ni) : skip_k();
                    if (!ok) break;
                    if (j < ni) {
                        // O_i is free once the previous pair's epilogue read it.
                        if (j == 0 && started > 1 &&
                            !(ok = wait_bar(bar(L::bOEmpty + i), started & 1, wc)))
                            break;
                        ok = pv(j > 0);
                    } else {
                        ok = skip_v();
                    }
                }
            }
            // Drain: all issued MMAs complete before Tensor Memory is freed.
            ptx::mma_commit(bar(L::bDrain + i));
            wait_slow(bar(L::bDrain + i), 0, wc, false);
        }
        __syncwarp();
    } else if (warp < 8) {
        ptx::reg_alloc<kRegsSoftmax>();
        softmax_role<kWindow, kVarlen, kFp8>(p, &tm_o, wc, tmem, sP, sO, bars, warp >> 2, warp & 3,
                                             lane);
    } else {
        ptx::reg_dealloc<kRegsControl>();  // idle warps of the control warpgroup
    }

    ptx::tc_fence_before();
    __syncthreads();
    if (warp == kMmaWarp0) {
        ptx::tc_fence_after();
        ptx::tmem_dealloc(tmem, kTmemCols);
    }
}

}  // namespace sdpa10

// attn_api.cu -- the C ABI declared in include/attn_fwd.h: argument
// validation (no CUDA call on an invalid argument), TMA descriptor encoding,
// the persistent launch, and the per-device status word.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstdlib>
#include <mutex>
#include <vector>

#include "attn_bwd_kernel.cuh"
#include "attn_fwd.h"
#include "attn_fwd_kernel.cuh"
#include "attn_merge.cuh"

namespace {

using namespace sdpa10;

using Layout = SmemLayout;
constexpr unsigned long long kDefaultTimeoutNs = 2000000000ull;
// Bytes of K/V that the tiles running at one time should share through L2
// (non-causal launches).  Measured on B200 with 16, 32, 48 and 96 MB and one
// section: 16 MB was fastest for every MHA workload (8K and 16K 10-11 %
// faster than 48 MB), and no size mattered for the 2K GQA workload.
constexpr size_t kL2SectionBytes = 16ull << 20;
// Causal launches of short rows: sections of this much K/V when the deal
// stays within kCausalSectionBalance of even (see launch_fwd).
constexpr size_t kCausalSectionBytes = 8ull << 20;
constexpr double kCausalSectionBalance = 1.06;
constexpr int kMaxDevices = 64;

// Per-device status word: bit 0 = a bounded wait gave up.
__device__ unsigned int g_status_word;

struct DeviceState {
    bool ready = false;
    int num_sms = 0;
    unsigned int* status = nullptr;  // device address of g_status_word
};

std::mutex g_mutex;
DeviceState g_dev[kMaxDevices];
PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
unsigned long long g_timeout_ns = kDefaultTimeoutNs;
int g_last_launches = 0;

int init_device(int dev, DeviceState** out) {
    if (dev < 0 || dev >= kMaxDevices) return ATTN_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_mutex);
    DeviceState& st = g_dev[dev];
    if (!st.ready) {
        if (!g_encode) {
            void* fn = nullptr;
            cudaDriverEntryPointQueryResult q;
            if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) !=
                    cudaSuccess ||
                q != cudaDriverEntryPointSuccess || fn == nullptr)
                return ATTN_ERR_CUDA;
            g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
        }
        int sms = 0;
        if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
            return ATTN_ERR_CUDA;
        const auto smem = cudaFuncAttributeMaxDynamicSharedMemorySize;
        if (cudaFuncSetAttribute(attn_fwd_sm100_kernel<false, false>, smem, Layout::kAlloc) !=
                cudaSuccess ||
            cudaFuncSetAttribute(attn_fwd_sm100_kernel<true, false>, smem, Layout::kAlloc) !=
                cudaSuccess ||
            cudaFuncSetAttribute(attn_fwd_sm100_kernel<false, true>, smem, Layout::kAlloc) !=
                cudaSuccess ||
            cudaFuncSetAttribute(attn_fwd_sm100_kernel<true, true>, smem, Layout::kAlloc) !=
                cudaSuccess ||
            cudaFuncSetAttribute(attn_fwd_sm100_kernel<false, false, true>, smem,
                                 SmemLayoutT<true>::kAlloc) != cudaSuccess ||
            cudaFuncSetAttribute(bwd::dq::attn_bwd_dq_kernel, smem, bwd::dq::Smem::kAlloc) !=
                cudaSuccess ||
            cudaFuncSetAttribute(bwd::dkdv::attn_bwd_dkdv_kernel, smem,
                                 bwd::dkdv::Smem::kAlloc) != cudaSuccess)
            return ATTN_ERR_CUDA;
        void* sp = nullptr;
        if (cudaGetSymbolAddress(&sp, g_status_word) != cudaSuccess) return ATTN_ERR_CUDA;
        st.num_sms = sms;
        st.status = static_cast<unsigned int*>(sp);
        st.ready = true;
    }
    *out = &st;
    return ATTN_OK;
}

// Encoded tensor maps of recent calls, per host thread: a map depends only
// on its base address, shape, element type and box, so a call that repeats
// a tensor (the usual case in a loop) reuses it instead of encoding it again
// on the launch path.
struct MapKey {
    const void* base;
    int heads, seq, batch, box_rows, fp8;
    bool operator==(const MapKey& o) const {
        return base == o.base && heads == o.heads && seq == o.seq && batch == o.batch &&
               box_rows == o.box_rows && fp8 == o.fp8;
    }
};
constexpr int kMapCacheSize = 16;
struct MapCache {
    MapKey key[kMapCacheSize];
    CUtensorMap map[kMapCacheSize];
    int used = 0, next = 0;
};
thread_local MapCache g_map_cache;

bool cached_map(CUtensorMap* m, const MapKey& k, bool (*encode)(CUtensorMap*, const MapKey&)) {
    MapCache& c = g_map_cache;
    for (int i = 0; i < c.used; ++i)
        if (c.key[i] == k) {
            *m = c.map[i];
            return true;
        }
    if (!encode(m, k)) return false;
    c.key[c.next] = k;
    c.map[c.next] = *m;
    c.next = (c.next + 1) % kMapCacheSize;
    if (c.used < kMapCacheSize) ++c.used;
    return true;
}

// [batch, seq, heads, 128] BF16 as a 4-D tensor map {d, heads, seq, batch},
// box {64, 1, box_rows, 1} (one 128-byte swizzled half of a box_rows-row
// tile; 128 rows unless given).
bool encode_map_bf16(CUtensorMap* m, const MapKey& k) {
    const void* base = k.base;
    const int heads = k.heads, seq = k.seq, batch = k.batch;
    const unsigned box_rows = static_cast<unsigned>(k.box_rows);
    cuuint64_t dims[4] = {static_cast<cuuint64_t>(kHeadDim), static_cast<cuuint64_t>(heads),
                          static_cast<cuuint64_t>(seq), static_cast<cuuint64_t>(batch)};
    cuuint64_t strides[3] = {static_cast<cuuint64_t>(kHeadDim) * 2,
                             static_cast<cuuint64_t>(heads) * kHeadDim * 2,
                             static_cast<cuuint64_t>(seq) * heads * kHeadDim * 2};
    cuuint32_t box[4] = {64, 1, box_rows, 1};
    cuuint32_t estr[4] = {1, 1, 1, 1};
    CUresult r = g_encode(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims,
                          strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                          CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// [batch, seq, heads, 128] FP8 (one byte per element) as a 4-D tensor map,
// box {128, 1, 128, 1}: a 128-row tile whose 128-byte rows are one swizzle
// atom each.
bool encode_map_e4m3(CUtensorMap* m, const MapKey& k) {
    const void* base = k.base;
    const int heads = k.heads, seq = k.seq, batch = k.batch;
    cuuint64_t dims[4] = {static_cast<cuuint64_t>(kHeadDim), static_cast<cuuint64_t>(heads),
                          static_cast<cuuint64_t>(seq), static_cast<cuuint64_t>(batch)};
    cuuint64_t strides[3] = {static_cast<cuuint64_t>(kHeadDim),
                             static_cast<cuuint64_t>(heads) * kHeadDim,
                             static_cast<cuuint64_t>(seq) * heads * kHeadDim};
    cuuint32_t box[4] = {128, 1, 128, 1};
    cuuint32_t estr[4] = {1, 1, 1, 1};
    CUresult r = g_encode(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 4, const_cast<void*>(base), dims,
                          strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                          CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

bool encode_map(CUtensorMap* m, const void* base, int heads, int seq, int batch,
                int box_rows = 128) {
    return cached_map(m, MapKey{base, heads, seq, batch, box_rows, 0}, encode_map_bf16);
}

bool encode_map_fp8(CUtensorMap* m, const void* base, int heads, int seq, int batch) {
    return cached_map(m, MapKey{base, heads, seq, batch, 128, 1}, encode_map_e4m3);
}

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

int validate_sizes(int batch, int h_q, int h_kv, int s_q, int s_k, int d) {
    if (batch <= 0 || h_q <= 0 || h_kv <= 0 || s_q <= 0 || s_k <= 0 || d <= 0)
        return ATTN_ERR_INVALID;
    if (h_q % h_kv != 0) return ATTN_ERR_INVALID;
    if (d != kHeadDim) return ATTN_ERR_UNSUPPORTED;
    const long long n_qb = (s_q + kBlockM - 1) / kBlockM;
    if (static_cast<long long>(batch) * h_q * n_qb > 0x7fffffffLL) return ATTN_ERR_INVALID;
    return ATTN_OK;
}

int validate(const void* q, const void* k, const void* v, const void* o, const float* lse,
             int batch, int h_q, int h_kv, int s_q, int s_k, int d, int causal, float scale) {
    if (!q || !k || !v || !o || !lse) return ATTN_ERR_INVALID;
    int rc = validate_sizes(batch, h_q, h_kv, s_q, s_k, d);
    if (rc != ATTN_OK) return rc;
    if (!std::isfinite(scale)) return ATTN_ERR_INVALID;
    if (causal != 0 && causal != 1) return ATTN_ERR_INVALID;
    if (causal && s_q > s_k) return ATTN_ERR_UNSUPPORTED;  // a row would see no key
    if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(o, 16) ||
        !aligned(lse, 4))
        return ATTN_ERR_ALIGN;
    return ATTN_OK;
}

size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// Effective key ranges for a requested count: ceil(n_kb / n) key blocks per
// range, and as many ranges as that takes.
void split_shape(int s_k, int num_splits, int* n_splits, int* kb_per_split) {
    const int n_kb = (s_k + kBlockN - 1) / kBlockN;
    const int n = num_splits < 1 ? 1 : (num_splits > n_kb ? n_kb : num_splits);
    *kb_per_split = (n_kb + n - 1) / n;
    *n_splits = (n_kb + *kb_per_split - 1) / *kb_per_split;
}

size_t split_workspace_bytes(int batch, int h_q, int s_q, int n_splits) {
    const size_t rows = static_cast<size_t>(batch) * h_q * s_q;
    return round_up(static_cast<size_t>(n_splits) * rows * kHeadDim * 4, 256) +
           static_cast<size_t>(n_splits) * rows * 4;
}

// Busiest CTA over the mean, in a model of the persistent kernel's causal
// schedule: items in the kernel's order (sections of units_per_section
// (batch, kv head) units; pair descending inside a section, then unit, then
// the unit's query heads), dealt in the snake order to `grid` CTAs.  An
// item costs the key blocks its two query blocks visit plus 8 (the pair
// boundary: O store, next Q load), in half-step units.
double causal_deal_balance(int batch, int h_q, int h_kv, int n_qb, int s_q, int causal_offset,
                           int units_per_section, int grid) {
    const int group = h_q / h_kv;
    const int n_pairs = (n_qb + 1) / 2;
    const int units = batch * h_kv;
    std::vector<double> load(static_cast<size_t>(grid), 0.0);
    long long t = 0;
    double total = 0.0;
    for (int sec0 = 0; sec0 < units; sec0 += units_per_section) {
        const int in_sec = std::min(units_per_section, units - sec0);
        for (int pair = n_pairs - 1; pair >= 0; --pair) {
            const int qb0 = 2 * pair;
            const int last0 = std::min(qb0 * kBlockM + kBlockM - 1, s_q - 1) + causal_offset;
            const int last1 = std::min(qb0 * kBlockM + 2 * kBlockM - 1, s_q - 1) + causal_offset;
            const int n0 = last0 / kBlockN + 1;
            const int n1 = qb0 + 1 < n_qb ? last1 / kBlockN + 1 : 0;
            const double w = n0 + n1 + 8;
            for (int u = 0; u < in_sec * group; ++u, ++t) {
                const long long k = t / grid, pos = t % grid;
                load[static_cast<size_t>((k & 1) ? grid - 1 - pos : pos)] += w;
                total += w;
            }
        }
    }
    const double mx = *std::max_element(load.begin(), load.end());
    return mx / (total / grid);
}

// A packed variable-length batch: device cu_seqlens and the packed extents.
struct Varlen {
    const int* cu_q;
    const int* cu_k;
    int total_q, total_k;
    int max_s_q, max_s_k;
};

// The forward launch shared by every forward entry point (arguments already
// validated).  o_part / lse_part null: O and LSE directly.  varlen non-null:
// a packed batch (batch = number of sequences; s_q, s_k unused).
int launch_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int batch,
               int h_q, int h_kv, int s_q, int s_k, int causal, int causal_offset, float scale,
               int n_splits, int kb_per_split, float* o_part, float* lse_part, void* stream,
               int window_left = -1, const Varlen* varlen = nullptr,
               const float* fp8_scales = nullptr) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return ATTN_ERR_CUDA;
    DeviceState* st = nullptr;
    const int rc = init_device(dev, &st);
    if (rc != ATTN_OK) return rc;

    // Packed tensors are one batch of total rows; the cursor adds each
    // sequence's first row.
    const int map_b = varlen ? 1 : batch;
    const int map_sq = varlen ? varlen->total_q : s_q;
    const int map_sk = varlen ? varlen->total_k : s_k;
    if (varlen) {
        s_q = varlen->max_s_q;
        s_k = varlen->max_s_k;
    }
    CUtensorMap tq, tk, tv, to;
    if (fp8_scales) {
        if (!encode_map_fp8(&tq, q, h_q, map_sq, map_b) ||
            !encode_map_fp8(&tk, k, h_kv, map_sk, map_b) ||
            !encode_map_fp8(&tv, v, h_kv, map_sk, map_b))
            return ATTN_ERR_CUDA;
    } else if (!encode_map(&tq, q, h_q, map_sq, map_b) ||
               !encode_map(&tk, k, h_kv, map_sk, map_b) ||
               !encode_map(&tv, v, h_kv, map_sk, map_b)) {
        return ATTN_ERR_CUDA;
    }
    // O is stored through a tensor map of the same shape as Q's (unused when
    // the launch writes FP32 partials instead).
    if (o != nullptr) {
        if (!encode_map(&to, o, h_q, map_sq, map_b)) return ATTN_ERR_CUDA;
    } else {
        to = tq;
    }

    FwdParams p{};
    p.batch = batch;
    p.h_q = h_q;
    p.h_kv = h_kv;
    p.s_q = s_q;
    p.s_k = s_k;
    p.group = h_q / h_kv;
    p.n_qb = (s_q + kBlockM - 1) / kBlockM;
    p.n_kb = (s_k + kBlockN - 1) / kBlockN;
    p.causal = causal;
    p.causal_offset = causal_offset;
    p.n_pairs = (p.n_qb + 1) / 2;
    p.n_splits = n_splits;
    p.kb_per_split = kb_per_split;
    p.num_tiles = batch * h_q * p.n_pairs * n_splits;
    const size_t unit_bytes = 2ull * s_k * kHeadDim * 2;  // K and V of one (batch, kv head)
    const size_t per_sec = kL2SectionBytes / (unit_bytes ? unit_bytes : 1);
    const int units_total = batch * h_kv;
    // Non-causal items are all alike: L2 sections keep the K/V of the units
    // in flight resident.  Causal items differ in length: one section puts
    // every item in one longest-first order, which the snake deal evens out
    // across the CTAs (the CTAs on one head then start their key streams
    // together and share them through L2).  For short rows (at most 64 key
    // blocks) the K/V locality of 8 MB sections is worth more (measured on
    // B200: 4K causal 7.8 % faster, 8K 2 %), provided those sections still
    // deal evenly; rows of 128 key blocks and more were fastest with one
    // section at every section size tried (8-48 MB).
    const int grid_est = std::min(p.num_tiles, st->num_sms);
    int ups = static_cast<int>(per_sec < 1 ? 1 : (per_sec > (size_t)units_total ? units_total : per_sec));
    if (causal) {
        const size_t per8 = kCausalSectionBytes / (unit_bytes ? unit_bytes : 1);
        const int u8 = static_cast<int>(per8 < 1 ? 1 : (per8 > (size_t)units_total ? units_total : per8));
        ups = units_total;
        if (!varlen && n_splits == 1 && p.n_kb <= 64 && u8 < units_total &&
            p.num_tiles <= (1 << 20)) {
            // The model runs once per shape (calls repeat with one shape).
            struct Key {
                int batch, h_q, h_kv, s_q, s_k, grid;
                bool operator==(const Key& o) const {
                    return batch == o.batch && h_q == o.h_q && h_kv == o.h_kv && s_q == o.s_q &&
                           s_k == o.s_k && grid == o.grid;
                }
            };
            thread_local Key last_key{0, 0, 0, 0, 0, 0};
            thread_local bool last_use = false;
            const Key key{batch, h_q, h_kv, s_q, s_k, grid_est};
            if (!(key == last_key)) {
                last_use = causal_deal_balance(batch, h_q, h_kv, p.n_qb, s_q, p.causal_offset, u8,
                                               grid_est) <= kCausalSectionBalance;
                last_key = key;
            }
            if (last_use) ups = u8;
        }
    }
    p.units_per_section = ups;
    p.last_section = (units_total - 1) / p.units_per_section;
    p.last_units = units_total - p.last_section * p.units_per_section;
    p.div_splits = FastDiv::make(static_cast<uint32_t>(n_splits));
    p.div_section = FastDiv::make(static_cast<uint32_t>(p.units_per_section) * p.group * p.n_pairs);
    p.div_rank = FastDiv::make(static_cast<uint32_t>(p.units_per_section) * p.group);
    p.div_rank_last = FastDiv::make(static_cast<uint32_t>(p.last_units) * p.group);
    p.div_group = FastDiv::make(static_cast<uint32_t>(p.group));
    p.div_h_kv = FastDiv::make(static_cast<uint32_t>(h_kv));
    // The kernel exponentiates 2^((s - m) c) with c > 0: a negative scale
    // negates the scores on the tensor core instead (see FwdParams).  FP8
    // inputs fold the Q and K scales into c and the V scale into 1 / l.
    double eff = static_cast<double>(scale);
    if (fp8_scales) eff *= static_cast<double>(fp8_scales[0]) * fp8_scales[1];
    const double c = std::fabs(eff) * 1.4426950408889634;
    p.scale_log2 = static_cast<float>(c < 1e-30 ? 1e-30 : c);
    p.idesc_qk = (fp8_scales ? idesc_e4m3_f32(kBlockM, kBlockN, 0, 0)
                             : idesc_bf16_f32(kBlockM, kBlockN, 0, 0)) |
                 (eff < 0.0 ? kIdescNegateA : 0u);
    p.v_scale = fp8_scales ? fp8_scales[2] : 1.f;
    p.o = static_cast<__nv_bfloat16*>(o);
    p.lse = lse;
    p.o_part = o_part;
    p.lse_part = lse_part;
    p.timeout_ns = g_timeout_ns;
    p.status = st->status;

    p.window_left = window_left;
    if (varlen) {
        p.cu_q = varlen->cu_q;
        p.cu_k = varlen->cu_k;
        p.total_q = varlen->total_q;
    }

    const int grid = p.num_tiles < st->num_sms ? p.num_tiles : st->num_sms;
    const cudaStream_t cs = static_cast<cudaStream_t>(stream);
    const bool win = window_left >= 0;
    if (fp8_scales)
        attn_fwd_sm100_kernel<false, false, true>
            <<<grid, kThreads, SmemLayoutT<true>::kAlloc, cs>>>(tq, tk, tv, to, p);
    else if (!varlen && !win)
        attn_fwd_sm100_kernel<false, false><<<grid, kThreads, Layout::kAlloc, cs>>>(tq, tk, tv, to, p);
    else if (!varlen)
        attn_fwd_sm100_kernel<true, false><<<grid, kThreads, Layout::kAlloc, cs>>>(tq, tk, tv, to, p);
    else if (!win)
        attn_fwd_sm100_kernel<false, true><<<grid, kThreads, Layout::kAlloc, cs>>>(tq, tk, tv, to, p);
    else
        attn_fwd_sm100_kernel<true, true><<<grid, kThreads, Layout::kAlloc, cs>>>(tq, tk, tv, to, p);
    g_last_launches = 1;
    if (cudaGetLastError() != cudaSuccess) return ATTN_ERR_CUDA;
    return ATTN_OK;
}

int launch_merge(const float* o_part, const float* lse_part, int n_parts, int batch, int h_q,
                 int s_q, int keys_per_part, int s_k, int causal, void* o, float* lse,
                 void* stream) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return ATTN_ERR_CUDA;
    DeviceState* st = nullptr;
    const int rc = init_device(dev, &st);
    if (rc != ATTN_OK) return rc;
    MergeParams m{};
    m.o_part = o_part;
    m.lse_part = lse_part;
    m.n_parts = n_parts;
    m.batch = batch;
    m.h_q = h_q;
    m.s_q = s_q;
    m.keys_per_part = keys_per_part;
    m.s_k = s_k;
    m.causal = causal;
    m.causal_offset = s_k - s_q;
    m.o = static_cast<__nv_bfloat16*>(o);
    m.lse = lse;
    const size_t rows = static_cast<size_t>(batch) * h_q * s_q;
    const size_t per_block = kMergeThreads / 32;
    size_t blocks = (rows + per_block - 1) / per_block;
    const size_t cap = static_cast<size_t>(st->num_sms) * 8;
    if (blocks > cap) blocks = cap;
    attn_merge_kernel<<<static_cast<unsigned>(blocks), kMergeThreads, 0,
                        static_cast<cudaStream_t>(stream)>>>(m);
    if (cudaGetLastError() != cudaSuccess) return ATTN_ERR_CUDA;
    return ATTN_OK;
}

}  // namespace

extern "C" int attn_fwd(const void* q, const void* k, const void* v, void* o, float* lse,
                        int batch, int h_q, int h_kv, int s_q, int s_k, int d, int causal,
                        float scale, void* stream) {
    const int rc = validate(q, k, v, o, lse, batch, h_q, h_kv, s_q, s_k, d, causal, scale);
    if (rc != ATTN_OK) return rc;
    const int n_kb = (s_k + kBlockN - 1) / kBlockN;
    return launch_fwd(q, k, v, o, lse, batch, h_q, h_kv, s_q, s_k, causal, s_k - s_q, scale, 1,
                      n_kb, nullptr, nullptr, stream);
}

extern "C" int attn_fwd_window(const void* q, const void* k, const void* v, void* o, float* lse,
                               int batch, int h_q, int h_kv, int s_q, int s_k, int d,
                               int window_left, float scale, void* stream) {
    const int rc = validate(q, k, v, o, lse, batch, h_q, h_kv, s_q, s_k, d, 1, scale);
    if (rc != ATTN_OK) return rc;
    if (window_left < 0) return ATTN_ERR_INVALID;
    const int n_kb = (s_k + kBlockN - 1) / kBlockN;
    // A window of s_k keys or more is the plain causal mask.
    const int w = window_left >= s_k ? -1 : window_left;
    return launch_fwd(q, k, v, o, lse, batch, h_q, h_kv, s_q, s_k, 1, s_k - s_q, scale, 1, n_kb,
                      nullptr, nullptr, stream, w);
}

extern "C" int attn_fwd_varlen(const void* q, const void* k, const void* v, void* o, float* lse,
                               const int* cu_seqlens_q, const int* cu_seqlens_k, int batch,
                               int max_seqlen_q, int max_seqlen_k, int total_q, int total_k,
                               int h_q, int h_kv, int d, int causal, int window_left,
                               float scale, void* stream) {
    if (!cu_seqlens_q || !cu_seqlens_k) return ATTN_ERR_INVALID;
    // The packed tensors are validated as one batch of total rows.
    int rc = validate(q, k, v, o, lse, 1, h_q, h_kv, total_q, total_k, d, 0, scale);
    if (rc != ATTN_OK) return rc;
    if (batch <= 0 || max_seqlen_q <= 0 || max_seqlen_k <= 0) return ATTN_ERR_INVALID;
    if (causal != 0 && causal != 1) return ATTN_ERR_INVALID;
    if (window_left < -1 || (window_left >= 0 && !causal)) return ATTN_ERR_INVALID;
    if (!aligned(cu_seqlens_q, 4) || !aligned(cu_seqlens_k, 4)) return ATTN_ERR_ALIGN;
    const long long n_qb = (max_seqlen_q + kBlockM - 1) / kBlockM;
    if (static_cast<long long>(batch) * h_q * ((n_qb + 1) / 2) > 0x7fffffffLL)
        return ATTN_ERR_INVALID;
    Varlen vl{cu_seqlens_q, cu_seqlens_k, total_q, total_k, max_seqlen_q, max_seqlen_k};
    const int n_kb = (max_seqlen_k + kBlockN - 1) / kBlockN;
    const int w = (window_left >= max_seqlen_k) ? -1 : window_left;
    return launch_fwd(q, k, v, o, lse, batch, h_q, h_kv, max_seqlen_q, max_seqlen_k, causal, 0,
                      scale, 1, n_kb, nullptr, nullptr, stream, w, &vl);
}

extern "C" size_t attn_bwd_workspace_bytes(int batch, int h_q, int s_q) {
    if (batch <= 0 || h_q <= 0 || s_q <= 0) return 0;
    const size_t pad = static_cast<size_t>((s_q + kBlockM - 1) / kBlockM) * kBlockM;
    return 2 * static_cast<size_t>(batch) * h_q * pad * sizeof(float);
}

extern "C" int attn_bwd(const void* q, const void* k, const void* v, const void* o,
                        const void* dout, const float* lse, void* dq, void* dk, void* dv,
                        int batch, int h_q, int h_kv, int s_q, int s_k, int d, int causal,
                        int window_left, float scale, void* workspace, size_t workspace_bytes,
                        void* stream) {
    int rc = validate(q, k, v, o, lse, batch, h_q, h_kv, s_q, s_k, d, causal, scale);
    if (rc != ATTN_OK) return rc;
    if (!dout || !dq || !dk || !dv || !workspace) return ATTN_ERR_INVALID;
    if (window_left < -1 || (window_left >= 0 && !causal)) return ATTN_ERR_INVALID;
    if (!aligned(dout, 16) || !aligned(dq, 16) || !aligned(dk, 16) || !aligned(dv, 16) ||
        !aligned(workspace, 256))
        return ATTN_ERR_ALIGN;
    if (workspace_bytes < attn_bwd_workspace_bytes(batch, h_q, s_q)) return ATTN_ERR_INVALID;
    const long long n_qb = (s_q + kBlockM - 1) / kBlockM;
    const long long n_kb = (s_k + kBlockN - 1) / kBlockN;
    if (static_cast<long long>(batch) * h_q * n_qb > 0x7fffffffLL ||
        static_cast<long long>(batch) * h_kv * n_kb > 0x7fffffffLL)
        return ATTN_ERR_INVALID;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return ATTN_ERR_CUDA;
    DeviceState* st = nullptr;
    rc = init_device(dev, &st);
    if (rc != ATTN_OK) return rc;
    const cudaStream_t cs = static_cast<cudaStream_t>(stream);

    bwd::BwdParams p{};
    p.batch = batch;
    p.h_q = h_q;
    p.h_kv = h_kv;
    p.s_q = s_q;
    p.s_k = s_k;
    p.group = h_q / h_kv;
    p.n_qb = static_cast<int>(n_qb);
    p.n_kb = static_cast<int>(n_kb);
    p.s_q_pad = p.n_qb * kBlockM;
    p.causal = causal;
    p.causal_offset = s_k - s_q;
    p.window_left = (window_left >= s_k) ? -1 : window_left;
    p.div_h_q = FastDiv::make(static_cast<uint32_t>(h_q));
    p.div_h_kv = FastDiv::make(static_cast<uint32_t>(h_kv));
    p.scale = scale;
    p.scale_log2 = static_cast<float>(static_cast<double>(scale) * 1.4426950408889634);
    float* Lw = static_cast<float*>(workspace);
    float* Dw = Lw + static_cast<size_t>(batch) * h_q * p.s_q_pad;
    p.NL = Lw;
    p.D = Dw;
    p.dk = static_cast<__nv_bfloat16*>(dk);
    p.dv = static_cast<__nv_bfloat16*>(dv);
    p.timeout_ns = g_timeout_ns;
    p.status = st->status;

    // 1. D = rowsum(dO * O) and -L = -LSE log2(e), padded per head.
    bwd::PrepParams a{static_cast<const __nv_bfloat16*>(o), static_cast<const __nv_bfloat16*>(dout),
                      lse, Lw, Dw, batch, h_q, s_q, p.s_q_pad};
    const size_t rows = static_cast<size_t>(batch) * h_q * p.s_q_pad;
    size_t blocks = (rows + bwd::kPrepThreads / 32 - 1) / (bwd::kPrepThreads / 32);
    const size_t cap = static_cast<size_t>(st->num_sms) * 16;
    if (blocks > cap) blocks = cap;
    bwd::attn_bwd_prep_kernel<<<static_cast<unsigned>(blocks), bwd::kPrepThreads, 0, cs>>>(a);
    if (cudaGetLastError() != cudaSuccess) return ATTN_ERR_CUDA;

    CUtensorMap tq, tk, tv, tdo, tdq;
    if (!encode_map(&tq, q, h_q, s_q, batch) || !encode_map(&tk, k, h_kv, s_k, batch) ||
        !encode_map(&tv, v, h_kv, s_k, batch) || !encode_map(&tdo, dout, h_q, s_q, batch) ||
        !encode_map(&tdq, dq, h_q, s_q, batch))
        return ATTN_ERR_CUDA;

    // Sections of 4 heads keep the streamed tiles of the heads in flight in
    // L2; launches with few items (at most 4 rounds of SMs) use one section
    // so their longest-first order can balance the CTAs.
    constexpr int kHeadsPerSection = 4;
    const int rounds4 = 4 * st->num_sms;

    // 2. dK, dV: one item per (key block, batch, key/value head).
    p.num_items = batch * h_kv * p.n_kb;
    p.section = p.num_items <= rounds4 ? batch * h_kv : kHeadsPerSection;
    if (p.section > batch * h_kv) p.section = batch * h_kv;
    int grid = p.num_items < st->num_sms ? p.num_items : st->num_sms;
    bwd::dkdv::attn_bwd_dkdv_kernel<<<grid, bwd::dkdv::kThreads, bwd::dkdv::Smem::kAlloc, cs>>>(
        tq, tk, tv, tdo, p);
    if (cudaGetLastError() != cudaSuccess) return ATTN_ERR_CUDA;

    // 3. dQ: one item per (query block, batch, query head).
    p.num_items = batch * h_q * p.n_qb;
    p.section = p.num_items <= rounds4 ? batch * h_q : kHeadsPerSection;
    if (p.section > batch * h_q) p.section = batch * h_q;
    grid = p.num_items < st->num_sms ? p.num_items : st->num_sms;
    bwd::dq::attn_bwd_dq_kernel<<<grid, bwd::dq::kThreads, bwd::dq::Smem::kAlloc, cs>>>(
        tq, tk, tv, tdo, tdq, p);
    if (cudaGetLastError() != cudaSuccess) return ATTN_ERR_CUDA;
    g_last_launches = 3;
    return ATTN_OK;
}

extern "C" int attn_fwd_fp8(const void* q, const void* k, const void* v, void* o, float* lse,
                            int batch, int h_q, int h_kv, int s_q, int s_k, int d, int causal,
                            float scale, float q_scale, float k_scale, float v_scale,
                            void* stream) {
    const int rc = validate(q, k, v, o, lse, batch, h_q, h_kv, s_q, s_k, d, causal, scale);
    if (rc != ATTN_OK) return rc;
    if (!std::isfinite(q_scale) || !std::isfinite(k_scale) || !std::isfinite(v_scale))
        return ATTN_ERR_INVALID;
    const float scales[3] = {q_scale, k_scale, v_scale};
    const int n_kb = (s_k + kBlockN - 1) / kBlockN;
    return launch_fwd(q, k, v, o, lse, batch, h_q, h_kv, s_q, s_k, causal, s_k - s_q, scale, 1,
                      n_kb, nullptr, nullptr, stream, -1, nullptr, scales);
}

extern "C" int attn_fwd_num_splits(int batch, int h_q, int h_kv, int s_q, int s_k, int d,
                                   int causal) {
    if (validate_sizes(batch, h_q, h_kv, s_q, s_k, d) != ATTN_OK) return 0;
    if (causal != 0 && causal != 1) return 0;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 0;
    DeviceState* st = nullptr;
    if (init_device(dev, &st) != ATTN_OK) return 0;
    const long long pairs = static_cast<long long>(batch) * h_q * ((s_q + 2 * kBlockM - 1) / (2 * kBlockM));
    const int n_kb = (s_k + kBlockN - 1) / kBlockN;
    if (pairs >= st->num_sms) return 1;
    long long n = st->num_sms / pairs;
    if (n > n_kb) n = n_kb;
    int n_splits = 1, kb = 1;
    split_shape(s_k, static_cast<int>(n < 1 ? 1 : n), &n_splits, &kb);
    return n_splits;
}

extern "C" size_t attn_fwd_split_workspace_bytes(int batch, int h_q, int s_q, int num_splits) {
    if (batch <= 0 || h_q <= 0 || s_q <= 0 || num_splits <= 0) return 0;
    return split_workspace_bytes(batch, h_q, s_q, num_splits);
}

extern "C" int attn_fwd_split(const void* q, const void* k, const void* v, void* o, float* lse,
                              int batch, int h_q, int h_kv, int s_q, int s_k, int d, int causal,
                              float scale, int num_splits, void* workspace,
                              size_t workspace_bytes, void* stream) {
    int rc = validate(q, k, v, o, lse, batch, h_q, h_kv, s_q, s_k, d, causal, scale);
    if (rc != ATTN_OK) return rc;
    if (num_splits < 1 || !workspace) return ATTN_ERR_INVALID;
    if (!aligned(workspace, 256)) return ATTN_ERR_ALIGN;
    int n_splits = 1, kb_per_split = 1;
    split_shape(s_k, num_splits, &n_splits, &kb_per_split);
    const long long n_qb = (s_q + kBlockM - 1) / kBlockM;
    if (static_cast<long long>(batch) * h_q * ((n_qb + 1) / 2) * n_splits > 0x7fffffffLL)
        return ATTN_ERR_INVALID;
    if (workspace_bytes < split_workspace_bytes(batch, h_q, s_q, n_splits)) return ATTN_ERR_INVALID;
    const size_t rows = static_cast<size_t>(batch) * h_q * s_q;
    float* o_part = static_cast<float*>(workspace);
    float* lse_part = reinterpret_cast<float*>(static_cast<char*>(workspace) +
                                               round_up(static_cast<size_t>(n_splits) * rows *
                                                            kHeadDim * 4,
                                                        256));
    rc = launch_fwd(q, k, v, o, lse, batch, h_q, h_kv, s_q, s_k, causal, s_k - s_q, scale,
                    n_splits, kb_per_split, o_part, lse_part, stream);
    if (rc != ATTN_OK) return rc;
    rc = launch_merge(o_part, lse_part, n_splits, batch, h_q, s_q, kb_per_split * kBlockN, s_k,
                      causal, o, lse, stream);
    g_last_launches = 2;
    return rc;
}

extern "C" int attn_fwd_partials(const void* q, const void* k, const void* v, float* o_part,
                                 float* lse_part, int batch, int h_q, int h_kv, int s_q, int s_k,
                                 int d, int causal, float scale, void* stream) {
    const int rc = validate(q, k, v, o_part, lse_part, batch, h_q, h_kv, s_q, s_k, d, causal,
                            scale);
    if (rc != ATTN_OK) return rc;
    const int n_kb = (s_k + kBlockN - 1) / kBlockN;
    return launch_fwd(q, k, v, nullptr, nullptr, batch, h_q, h_kv, s_q, s_k, causal, s_k - s_q,
                      scale, 1, n_kb, o_part, lse_part, stream);
}

extern "C" int attn_fwd_partials_shard(const void* q, const void* k, const void* v,
                                       float* o_part, float* lse_part, int batch, int h_q,
                                       int h_kv, int s_q, int s_k, int d, int causal,
                                       int diag_offset, float scale, void* stream) {
    if (!q || !k || !v || !o_part || !lse_part) return ATTN_ERR_INVALID;
    int rc = validate_sizes(batch, h_q, h_kv, s_q, s_k, d);
    if (rc != ATTN_OK) return rc;
    if (!std::isfinite(scale) || (causal != 0 && causal != 1)) return ATTN_ERR_INVALID;
    // Row + diagonal must stay inside 32-bit arithmetic in the kernel.
    if (diag_offset < -(1 << 30) || diag_offset > (1 << 30)) return ATTN_ERR_INVALID;
    if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(o_part, 16) ||
        !aligned(lse_part, 4))
        return ATTN_ERR_ALIGN;
    const int diag = causal ? diag_offset : s_k - s_q;
    // Causal rows 0 .. -diag - 1 see no key of the shard: their partial is
    // written by a fill launch first (the forward skips wholly empty blocks).
    const long long n_empty = causal ? (diag < 0 ? (-static_cast<long long>(diag) < s_q
                                                         ? -static_cast<long long>(diag)
                                                         : s_q)
                                                  : 0)
                                     : 0;
    int launches = 0;
    if (n_empty > 0) {
        int dev = 0;
        if (cudaGetDevice(&dev) != cudaSuccess) return ATTN_ERR_CUDA;
        DeviceState* st = nullptr;
        rc = init_device(dev, &st);
        if (rc != ATTN_OK) return rc;
        const size_t rows = static_cast<size_t>(batch) * h_q * n_empty;
        size_t blocks = (rows + kMergeThreads / 32 - 1) / (kMergeThreads / 32);
        const size_t cap = static_cast<size_t>(st->num_sms) * 8;
        if (blocks > cap) blocks = cap;
        attn_fill_empty_rows_kernel<<<static_cast<unsigned>(blocks), kMergeThreads, 0,
                                      static_cast<cudaStream_t>(stream)>>>(
            o_part, lse_part, batch, h_q, s_q, static_cast<int>(n_empty));
        if (cudaGetLastError() != cudaSuccess) return ATTN_ERR_CUDA;
        ++launches;
    }
    if (n_empty < s_q) {
        const int n_kb = (s_k + kBlockN - 1) / kBlockN;
        rc = launch_fwd(q, k, v, nullptr, nullptr, batch, h_q, h_kv, s_q, s_k, causal, diag,
                        scale, 1, n_kb, o_part, lse_part, stream);
        if (rc != ATTN_OK) return rc;
        ++launches;
    }
    g_last_launches = launches;
    return ATTN_OK;
}

extern "C" int attn_merge_partials(const float* o_parts, const float* lse_parts, int n_parts,
                                   int batch, int h_q, int s_q, int d, void* o, float* lse,
                                   void* stream) {
    if (!o_parts || !lse_parts || !o || !lse) return ATTN_ERR_INVALID;
    if (n_parts <= 0 || batch <= 0 || h_q <= 0 || s_q <= 0 || d <= 0) return ATTN_ERR_INVALID;
    if (d != kHeadDim) return ATTN_ERR_UNSUPPORTED;
    if (!aligned(o_parts, 16) || !aligned(o, 16) || !aligned(lse_parts, 4) || !aligned(lse, 4))
        return ATTN_ERR_ALIGN;
    const int rc = launch_merge(o_parts, lse_parts, n_parts, batch, h_q, s_q, 0, 0, 0, o, lse,
                                stream);
    g_last_launches = 1;
    return rc;
}

extern "C" size_t attn_fwd_host_workspace_bytes(int batch, int h_q, int h_kv, int s_q, int s_k,
                                                int d) {
    if (validate_sizes(batch, h_q, h_kv, s_q, s_k, d) != ATTN_OK) return 0;
    const size_t qb = static_cast<size_t>(batch) * s_q * h_q * d * 2;
    const size_t kb = static_cast<size_t>(batch) * s_k * h_kv * d * 2;
    const size_t lb = static_cast<size_t>(batch) * h_q * s_q * 4;
    return round_up(qb, 256) * 2 + round_up(kb, 256) * 2 + round_up(lb, 256);
}

// The host-buffer forward is pipelined: the problem is cut into up to
// kHostChunks groups of key/value heads (each with its query heads), each
// group a compact sub-problem in the workspace.  A group's inputs are copied
// in with strided 2-D copies on an H2D stream, its forward runs on the
// caller's stream once they have landed, and its O and LSE go back on a D2H
// stream, so the copies of one group overlap the kernel of another.  Events
// order the three streams; the caller's stream finally waits for the last
// copy out, so synchronising it covers the whole call.
constexpr int kHostChunks = 8;
constexpr size_t kHostChunkMinBytes = size_t(16) << 20;  // smaller groups: fewer chunks

struct HostPipe {
    bool ready = false;
    cudaStream_t h2d = nullptr, d2h = nullptr;
    cudaEvent_t start = nullptr, done = nullptr;
    cudaEvent_t in[kHostChunks] = {}, comp[kHostChunks] = {};
    std::mutex mu;  // one call's enqueue sequence at a time per device
};
HostPipe g_pipe[kMaxDevices];

int host_pipe(int dev, HostPipe** out) {
    HostPipe& hp = g_pipe[dev];
    if (!hp.ready) {
        const unsigned fl = cudaEventDisableTiming;
        if (cudaStreamCreateWithFlags(&hp.h2d, cudaStreamNonBlocking) != cudaSuccess ||
            cudaStreamCreateWithFlags(&hp.d2h, cudaStreamNonBlocking) != cudaSuccess ||
            cudaEventCreateWithFlags(&hp.start, fl) != cudaSuccess ||
            cudaEventCreateWithFlags(&hp.done, fl) != cudaSuccess)
            return ATTN_ERR_CUDA;
        for (int c = 0; c < kHostChunks; ++c)
            if (cudaEventCreateWithFlags(&hp.in[c], fl) != cudaSuccess ||
                cudaEventCreateWithFlags(&hp.comp[c], fl) != cudaSuccess)
                return ATTN_ERR_CUDA;
        hp.ready = true;
    }
    *out = &hp;
    return ATTN_OK;
}

// Strided copy of `rows` rows of `width` bytes (a plain copy when the rows
// are contiguous on both sides).
cudaError_t copy_rows(void* dst, size_t dpitch, const void* src, size_t spitch, size_t width,
                      size_t rows, cudaMemcpyKind kind, cudaStream_t s) {
    if (dpitch == width && spitch == width)
        return cudaMemcpyAsync(dst, src, width * rows, kind, s);
    return cudaMemcpy2DAsync(dst, dpitch, src, spitch, width, rows, kind, s);
}

// The host-buffer forward: pipelined on the library's streams, or (for the
// allocation-free entry, which creates no streams or events) copy in, run
// and copy out in order on the caller's stream alone.
int host_forward(const void* q, const void* k, const void* v, void* o, float* lse, int batch,
                 int h_q, int h_kv, int s_q, int s_k, int d, int causal, float scale,
                 void* workspace, size_t workspace_bytes, void* stream, bool pipelined) {
    int rc = validate(q, k, v, o, lse, batch, h_q, h_kv, s_q, s_k, d, causal, scale);
    if (rc != ATTN_OK) return rc;
    if (!workspace) return ATTN_ERR_INVALID;
    if (!aligned(workspace, 256)) return ATTN_ERR_ALIGN;
    const size_t need = attn_fwd_host_workspace_bytes(batch, h_q, h_kv, s_q, s_k, d);
    if (workspace_bytes < need) return ATTN_ERR_INVALID;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return ATTN_ERR_CUDA;
    DeviceState* st = nullptr;
    rc = init_device(dev, &st);
    if (rc != ATTN_OK) return rc;
    const cudaStream_t s = static_cast<cudaStream_t>(stream);
    HostPipe* hp = nullptr;
    if (pipelined) {
        std::lock_guard<std::mutex> lock(g_mutex);  // creation only: attn_fwd takes it too
        rc = host_pipe(dev, &hp);
        if (rc != ATTN_OK) return rc;
    }
    std::unique_lock<std::mutex> pipe_lock;
    if (hp) pipe_lock = std::unique_lock<std::mutex>(hp->mu);
    const cudaStream_t s_in = hp ? hp->h2d : s, s_out = hp ? hp->d2h : s;

    const size_t row = static_cast<size_t>(d) * 2;  // bytes of one head's row
    const size_t qb = static_cast<size_t>(batch) * s_q * h_q * row;
    const size_t kb = static_cast<size_t>(batch) * s_k * h_kv * row;
    int nc = !hp ? 1 : (h_kv < kHostChunks ? h_kv : kHostChunks);
    while (nc > 1 && (qb + 2 * kb) / nc < kHostChunkMinBytes) --nc;
    const int group = h_q / h_kv;
    // Workspace: per group q | k | v | o (compact [b, s, heads, d]; every
    // size a multiple of 256 bytes), then all groups' LSE [b, heads, s_q].
    char* w = static_cast<char*>(workspace);
    float* lse_all = reinterpret_cast<float*>(w + 2 * qb + 2 * kb);
    if (hp && (cudaEventRecord(hp->start, s) != cudaSuccess ||
               cudaStreamWaitEvent(hp->h2d, hp->start, 0) != cudaSuccess))
        return ATTN_ERR_CUDA;
    size_t off = 0, loff = 0;
    int g0 = 0;
    for (int c = 0; c < nc; ++c) {
        const int gc = h_kv / nc + (c < h_kv % nc ? 1 : 0);
        const int hq0 = g0 * group, hqc = gc * group;
        const size_t qc = static_cast<size_t>(batch) * s_q * hqc * row;
        const size_t kc = static_cast<size_t>(batch) * s_k * gc * row;
        char* dq = w + off;
        char* dk = dq + qc;
        char* dv = dk + kc;
        char* d_o = dv + kc;
        float* dl = lse_all + loff;
        off += 2 * qc + 2 * kc;
        loff += static_cast<size_t>(batch) * hqc * s_q;
        const size_t q_rows = static_cast<size_t>(batch) * s_q;
        const size_t k_rows = static_cast<size_t>(batch) * s_k;
        const char* qh = static_cast<const char*>(q) + hq0 * row;
        const char* kh = static_cast<const char*>(k) + g0 * row;
        const char* vh = static_cast<const char*>(v) + g0 * row;
        if (copy_rows(dq, hqc * row, qh, h_q * row, hqc * row, q_rows, cudaMemcpyHostToDevice,
                      s_in) != cudaSuccess ||
            copy_rows(dk, gc * row, kh, h_kv * row, gc * row, k_rows, cudaMemcpyHostToDevice,
                      s_in) != cudaSuccess ||
            copy_rows(dv, gc * row, vh, h_kv * row, gc * row, k_rows, cudaMemcpyHostToDevice,
                      s_in) != cudaSuccess)
            return ATTN_ERR_CUDA;
        if (hp && (cudaEventRecord(hp->in[c], hp->h2d) != cudaSuccess ||
                   cudaStreamWaitEvent(s, hp->in[c], 0) != cudaSuccess))
            return ATTN_ERR_CUDA;
        rc = attn_fwd(dq, dk, dv, d_o, dl, batch, hqc, gc, s_q, s_k, d, causal, scale, stream);
        if (rc != ATTN_OK) return rc;
        char* oh = static_cast<char*>(o) + hq0 * row;
        char* lh = reinterpret_cast<char*>(lse) + static_cast<size_t>(hq0) * s_q * 4;
        const size_t lw = static_cast<size_t>(hqc) * s_q * 4;
        if (hp && (cudaEventRecord(hp->comp[c], s) != cudaSuccess ||
                   cudaStreamWaitEvent(hp->d2h, hp->comp[c], 0) != cudaSuccess))
            return ATTN_ERR_CUDA;
        if (copy_rows(oh, h_q * row, d_o, hqc * row, hqc * row, q_rows, cudaMemcpyDeviceToHost,
                      s_out) != cudaSuccess ||
            copy_rows(lh, static_cast<size_t>(h_q) * s_q * 4, dl, lw, lw, batch,
                      cudaMemcpyDeviceToHost, s_out) != cudaSuccess)
            return ATTN_ERR_CUDA;
        g0 += gc;
    }
    if (hp && (cudaEventRecord(hp->done, hp->d2h) != cudaSuccess ||
               cudaStreamWaitEvent(s, hp->done, 0) != cudaSuccess))
        return ATTN_ERR_CUDA;
    g_last_launches = nc;
    return ATTN_OK;
}

extern "C" int attn_fwd_host(const void* q, const void* k, const void* v, void* o, float* lse,
                             int batch, int h_q, int h_kv, int s_q, int s_k, int d, int causal,
                             float scale, void* workspace, size_t workspace_bytes, void* stream) {
    return host_forward(q, k, v, o, lse, batch, h_q, h_kv, s_q, s_k, d, causal, scale, workspace,
                        workspace_bytes, stream, true);
}

extern "C" int attn_status(void* stream) {
    if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess)
        return ATTN_ERR_CUDA;
    unsigned int word = 0;
    if (cudaMemcpyFromSymbol(&word, g_status_word, sizeof(word)) != cudaSuccess)
        return ATTN_ERR_CUDA;
    if (word != 0) {
        const unsigned int zero = 0;
        if (cudaMemcpyToSymbol(g_status_word, &zero, sizeof(zero)) != cudaSuccess)
            return ATTN_ERR_CUDA;
        return ATTN_ERR_TIMEOUT;
    }
    return ATTN_OK;
}

extern "C" const char* attn_strerror(int code) {
    switch (code) {
        case ATTN_OK: return "success";
        case ATTN_ERR_INVALID: return "invalid argument";
        case ATTN_ERR_UNSUPPORTED: return "unsupported configuration (d must be 128; causal needs s_q <= s_k)";
        case ATTN_ERR_ALIGN: return "misaligned pointer (q/k/v/o need 16 bytes, lse 4 bytes)";
        case ATTN_ERR_CUDA: return "CUDA runtime or driver error";
        case ATTN_ERR_TIMEOUT: return "a kernel gave up a bounded device-side wait";
        case ATTN_ERR_TOO_LARGE: return "problem larger than the static device staging area (ATTN_STATIC_STAGING_BYTES)";
        default: return "unknown status code";
    }
}

extern "C" int attn_set_wait_timeout_ns(uint64_t ns) {
    g_timeout_ns = ns ? static_cast<unsigned long long>(ns) : kDefaultTimeoutNs;
    return ATTN_OK;
}

extern "C" int attn_selftest_wait_timeout(uint64_t timeout_ns, void* stream) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return ATTN_ERR_CUDA;
    DeviceState* st = nullptr;
    int rc = init_device(dev, &st);
    if (rc != ATTN_OK) return rc;
    wait_timeout_selftest_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(
        st->status, static_cast<unsigned long long>(timeout_ns));
    if (cudaGetLastError() != cudaSuccess) return ATTN_ERR_CUDA;
    return ATTN_OK;
}

extern "C" int attn_last_launch_count(void) { return g_last_launches; }

// ---------------------------------------------------------------------------
// attn_fwd_host_static: the host-buffer entry point with its device staging in
// a file-scope array, for callers that cannot allocate device memory.  Host
// code must not pass the array's name to a kernel or a copy: on the host it is
// only a stand-in symbol.  Its device address is looked up once per device.
namespace {

static __device__ __align__(256) unsigned char g_static_staging[ATTN_STATIC_STAGING_BYTES];

std::mutex g_static_mutex;
void* g_static_staging_ptr[kMaxDevices] = {};

}  // namespace

extern "C" int attn_fwd_host_static(const void* q, const void* k, const void* v, void* o,
                                    float* lse, int batch, int h_q, int h_kv, int s_q, int s_k,
                                    int d, int causal, float scale, void* stream) {
    int rc = validate(q, k, v, o, lse, batch, h_q, h_kv, s_q, s_k, d, causal, scale);
    if (rc != ATTN_OK) return rc;
    const size_t need = attn_fwd_host_workspace_bytes(batch, h_q, h_kv, s_q, s_k, d);
    if (need > ATTN_STATIC_STAGING_BYTES) return ATTN_ERR_TOO_LARGE;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return ATTN_ERR_CUDA;
    void* staging = nullptr;
    {
        std::lock_guard<std::mutex> lock(g_static_mutex);
        if (!g_static_staging_ptr[dev]) {
            // Set-up, once per device, with that device current.
            void* ptr = nullptr;
            if (cudaGetSymbolAddress(&ptr, g_static_staging) != cudaSuccess || !ptr)
                return ATTN_ERR_CUDA;
            g_static_staging_ptr[dev] = ptr;
        }
        staging = g_static_staging_ptr[dev];
    }
    return host_forward(q, k, v, o, lse, batch, h_q, h_kv, s_q, s_k, d, causal, scale, staging,
                        ATTN_STATIC_STAGING_BYTES, stream, false);
}

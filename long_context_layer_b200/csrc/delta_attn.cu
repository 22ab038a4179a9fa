// DELTA decode attention stack for B200 (sm_100a): kernels and the C ABI of include/delta_attn.h.
//
// Method: "DELTA: Dynamic Layer-Aware Token Attention for Efficient Long-Context Reasoning",
// ai.info summary, section "Methodology in Plain English".  Initial layers run full attention,
// delta-layers run full attention and score 16-token KV pages, sparse layers attend only to
// the selected pages; the paged KV cache is kept in full.
//
// Kernels (all launched on the caller's stream with programmatic dependent launch, none
// synchronises the host):
//   kv_append_kernel,     the current token's k, v into its page slot: one (sequence, KV head)
//   kv_append_layers_     per CTA (and per layer), 16-byte vector copies.
//     kernel
//   decode_mma_kernel     bf16 split-KV online-softmax decode on the tensor cores (mma.sync,
//                         decode_mma.cuh).  Grid (split, KV head, sequence) in thread-block
//                         clusters; each warp streams whole pages (K and V of one KV head) into
//                         its own shared-memory ring with 2-D TMA tensor copies.  Delta-layers
//                         also write each (head, page)'s log2-sum-exp and each split's per-head
//                         state; sparse layers walk the selected page list.  Splits merge by
//                         pushing their partials into the owning CTA of the cluster (st.async
//                         on its mbarrier); several clusters of one unit meet in the workspace,
//                         merged by whichever CTA arrives last (an atomic ticket; no CTA waits).
//   decode_kernel         the fp32 counterpart on the CUDA cores (decode_simt.cuh), same merge.
//   score_select_kernel   one thread-block cluster per sequence (select.cuh): page score = sum
//                         over heads of 2^(lse_hp - c_h), c_h from the splits' states; the k-th
//                         largest candidate by a bucket histogram and an exact in-bucket rank
//                         (one CTA) or an MSB-first radix select (cluster); lower-index tie-break,
//                         union with sink and recency pages, ascending compaction.
//   layer_shift_kernel    1 - cos between two layers' page-score vectors (calibration metric).
//
// Logits are carried in base 2 (q is pre-scaled by sm_scale*log2(e)) so every exponential is
// one exp2.  No floating-point atomics are used: results are deterministic run to run.

#include "delta_attn.h"

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>

#include <mutex>

#include "common.cuh"
#include "decode_simt.cuh"
#include "decode_mma.cuh"
#include "select.cuh"

namespace delta {

// ------------------------------------------------------------------ host side
constexpr int kMmaStages = 3;      // tensor-core kernel: stages per warp (8 KB each for D = 128), 2 CTAs/SM
constexpr int kMmaWideWarps = 8;   // when a cluster per unit fits one CTA per SM: 8-warp CTAs
constexpr int kMmaShortWarps = 6;  // short page lists: 6 warps with 2 stages each (same shared memory)
constexpr int kMmaShortStages = 2;
enum : int { kVarNarrow = 0, kVarWide = 1, kVarShort = 2 };   // tensor-core kernel variants
constexpr int variant_threads(int v) { return 32 * (v == kVarWide ? kMmaWideWarps : v == kVarShort ? kMmaShortWarps : kWarps); }

struct WsLayout {
    size_t err, tickets, seq_tickets, part_ml, part_o, page_lse, split_ml, score_acc, keys, logits,
        total;
};

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

int elem_bytes(int dtype) { return dtype == DELTA_BF16 ? 2 : 4; }

int current_device() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return -1;
    return dev;
}

// Guards the per-device caches below (SM count, kernel attributes, cluster occupancy, the tensor-map
// encoder and the scratch array's address): first calls from several host threads may race.
std::recursive_mutex& cache_mutex() {
    static std::recursive_mutex mu;
    return mu;
}

int device_sm_count() {
    static int cache[64] = {0};
    std::lock_guard<std::recursive_mutex> lock(cache_mutex());
    const int dev = current_device();
    if (dev < 0) return 148;
    if (cache[dev] == 0) {
        int sms = 0;
        if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || sms <= 0) sms = 148;
        cache[dev] = sms;
    }
    return cache[dev];
}

// Stages of the CUDA-core kernel (fp32): about 24 KB of pages in flight per warp.
constexpr int simt_stages(int ebytes, int D) {
    return (24 * 1024) / (2 * kPage * D * ebytes) < 2   ? 2
           : (24 * 1024) / (2 * kPage * D * ebytes) > 4 ? 4
                                                        : (24 * 1024) / (2 * kPage * D * ebytes);
}

// Dynamic shared memory of the decode kernel that serves (dtype, D).
size_t decode_smem_bytes(int dtype, int D) {
    if (dtype == DELTA_BF16)
        return D == 128 ? MmaSmem<128, kMmaStages>::kBytes : MmaSmem<64, kMmaStages>::kBytes;
    return D == 128 ? DecodeSmem<float, 128, simt_stages(4, 128)>::kBytes : DecodeSmem<float, 64, simt_stages(4, 64)>::kBytes;
}

int ctas_per_sm(int dtype, int D) {
    const size_t per_sm = 233472;  // shared memory per SM on B200
    int c = int(per_sm / (decode_smem_bytes(dtype, D) + 1024));
    return c < 1 ? 1 : (c > 8 ? 8 : c);
}

// Split plan: about one full wave of CTAs over the GPU, at least one page per warp.  Up to 16
// splits form one thread-block cluster; more are grouped into clusters whose partials meet in the
// workspace.
struct SplitPlan {
    int cluster, clusters;
    int variant;   // kVarNarrow: 4-warp CTAs, 3 stages, two per SM; kVarWide: one 8-warp CTA per SM;
                   // kVarShort: 6-warp CTAs, 2 stages, two per SM (tensor-core kernel)
    int splits() const { return cluster * clusters; }
};

// Split-plan constants (compile-time; a sweep rebuilds the library with -D overrides).
#ifndef DELTA_CTAS_PER_SM
#define DELTA_CTAS_PER_SM 0          // 0: as many CTAs per SM as shared memory allows
#endif
#ifndef DELTA_MAX_SPLITS
#define DELTA_MAX_SPLITS 0           // 0: no cap beyond kMaxSplits
#endif
#ifndef DELTA_MAX_WIDE_SPLITS
#define DELTA_MAX_WIDE_SPLITS 0      // 0: no extra cap on 8-warp plans
#endif
#ifndef DELTA_MAX_NARROW_SPLITS
#define DELTA_MAX_NARROW_SPLITS 0    // 0: no extra cap on 4- and 6-warp plans
#endif
#ifndef DELTA_WIDE
#define DELTA_WIDE 1                 // 0: never use 8-warp CTAs
#endif
#ifndef DELTA_PAGES_PER_CLUSTER
#define DELTA_PAGES_PER_CLUSTER 256  // pages each cluster must get before a unit uses several
#endif
#ifndef DELTA_ONE_CLUSTER_PAGES
#define DELTA_ONE_CLUSTER_PAGES 512  // up to this many pages per unit, one cluster
#endif

int split_target_per_sm(int dtype, int D) {
    return DELTA_CTAS_PER_SM > 0 ? DELTA_CTAS_PER_SM : ctas_per_sm(dtype, D);
}

// About one wave of CTAs, at least one page per warp.  The splits of one (sequence, KV head) form
// clusters of at most 16 CTAs that merge through distributed shared memory; only long page lists
// (fit_plan) make several clusters meet in the workspace.
// The plan of one variant.
SplitPlan plan_variant(int dtype, int D, int batch, int Hkv, int items, int variant) {
    if (items <= 0) return {1, 1, kVarNarrow};
    const bool wide = variant == kVarWide;
    const int sms = device_sm_count();
    const int units = batch * Hkv;
    const int warps = variant_threads(variant) / 32;
    const int slots = wide ? sms : sms * split_target_per_sm(dtype, D);
    int s = slots / (units > 0 ? units : 1);
    // at least one page per warp; 4- and 6-warp tensor-core CTAs take at least 2 * warps - 1
    // (two pages for all warps but one): of the plans that give no warp more than one two-page
    // loop iteration, that one measured fastest on the 8k sparse layers (81 pages)
    const int per_cta = (!wide && dtype == DELTA_BF16) ? 2 * warps - 1 : warps;
    const int cap = (items + per_cta - 1) / per_cta;
    if (s > cap) s = cap;
    if (s > kMaxSplits) s = kMaxSplits;
    if (DELTA_MAX_SPLITS > 0 && s > DELTA_MAX_SPLITS) s = DELTA_MAX_SPLITS;
    if (wide && DELTA_MAX_WIDE_SPLITS > 0 && s > DELTA_MAX_WIDE_SPLITS) s = DELTA_MAX_WIDE_SPLITS;
    if (!wide && DELTA_MAX_NARROW_SPLITS > 0 && s > DELTA_MAX_NARROW_SPLITS) s = DELTA_MAX_NARROW_SPLITS;
    if (s < 1) s = 1;
    SplitPlan pl;
    pl.cluster = s < 16 ? s : 16;
    pl.clusters = s / pl.cluster;
    pl.variant = variant;
    return pl;
}

// delta_fused: a delta-layer that scores and selects its pages inside the decode (HEAD_SUM).
SplitPlan plan_splits(int dtype, int D, int batch, int Hkv, int items, bool delta_fused = false) {
    // One 8-warp CTA per SM, each warp streaming half the pages of a 4-warp CTA's warp (the per-warp
    // chain of dependent MMAs, exponentials and shuffles, not the memory system, bounds such layers):
    //  - few (sequence, KV head) units, so that a full cluster per unit fits one CTA per SM, and at
    //    least two pages per warp of such a cluster (short lists of such batches, sparse layers, keep
    //    smaller CTAs, two per SM, so the next layer's CTAs find room beside them and start early);
    //  - mid-size batches, where a 16-CTA cluster per unit would not fit but every unit still gets
    //    at least four SMs, for every layer kind (measured: the 8-sequence 16k-32k stack's step
    //    640 -> 551 us and the 4-sequence 64k stack's 1296 -> 1239 us, every layer kind faster,
    //    against 4- and 6-warp CTAs two per SM).
    const int64_t units = int64_t(batch) * Hkv;
    const int sms = device_sm_count();
    const bool few_units = units * 16 <= sms && items >= 16 * kMmaWideWarps * 2;
    const bool mid_units = units * 16 > sms && units * 4 <= sms;
    const bool wide = DELTA_WIDE && dtype == DELTA_BF16 && (few_units || mid_units);
    if (wide) return plan_variant(dtype, D, batch, Hkv, items, kVarWide);
    // 6 warps with 2 stages each (the same shared memory and pages in flight as 4 warps x 3 stages,
    // spread over more warps) for three kinds of list:
    //  - lists that 4-warp CTAs would cover with at most two pages per warp (a sparse layer of a
    //    small batch), so more warps share the few pages;
    //  - short lists (sparse layers, at most kShortListPages) that still give a 4-warp CTA at least
    //    kShortLongCta pages (a sparse layer of a large batch): each warp streams fewer pages, so the
    //    slowest warp, which ends the layer, finishes sooner (measured: 29.0 instead of 30.1 us per
    //    sparse layer of the 16-sequence 16k stack with 81 pages per CTA; slower at 32 pages per CTA
    //    on the 4-sequence 64k stack, 17.2 instead of 16.0 us);
    //  - delta-layers of large batches (at most two splits per unit, at least 64 pages per CTA): the
    //    page terms add work to every page, which more warps share (measured: 167 instead of 171 us
    //    per delta-layer of the 16-sequence 16k stack; at nine splits per unit, the 64k stack's, the
    //    6-warp plan ran slower, 204 instead of 178 us).
    //  Other long lists (full layers) keep 3 stages per warp.
    constexpr int kShortListPages = 512, kShortLongCta = 48;
    const SplitPlan narrow = plan_variant(dtype, D, batch, Hkv, items, kVarNarrow);
    const int per_cta = (items + narrow.splits() - 1) / narrow.splits();
    const bool short_list = per_cta <= 2 * kWarps || (items <= kShortListPages && per_cta >= kShortLongCta);
    const bool delta_large_batch = delta_fused && narrow.splits() <= 2 && per_cta >= 64;
    if (dtype == DELTA_BF16 && (short_list || delta_large_batch))
        return plan_variant(dtype, D, batch, Hkv, items, kVarShort);
    return narrow;
}

// Most splits any launch on page lists of at most max_pages can get (workspace bound): both
// variants' split counts grow with the page count.
int max_splits_for(int dtype, int D, int batch, int Hkv, int max_pages) {
    // (a short-list plan never has more splits than the 4-warp plan of the same list)
    const int a = plan_variant(dtype, D, batch, Hkv, max_pages, kVarNarrow).splits();
    const int b = plan_variant(dtype, D, batch, Hkv, max_pages, kVarWide).splits();
    return a > b ? a : b;
}

// with_logits: room for per-token logits of every query head (delta-layers scoring with HEAD_MAX)
WsLayout ws_layout(const delta_desc* d, int batch, int max_pages, bool with_logits = false) {
    WsLayout w{};
    // room for as many cluster partials as there are splits (fit_plan never exceeds a plan's)
    const int S = max_splits_for(d->dtype, d->head_dim, batch, d->num_kv_heads, max_pages);
    const size_t rows = size_t(batch) * d->num_q_heads;
    size_t off = 0;
    // the counters (error word, tickets) come first: they are the part that must start at zero
    w.err = off;          off += align256(64);
    w.tickets = off;      off += align256(size_t(batch) * d->num_kv_heads * sizeof(int));
    w.seq_tickets = off;  off += align256(size_t(batch) * sizeof(int));
    w.part_ml = off;      off += align256(rows * S * sizeof(float2));
    w.part_o = off;       off += align256(rows * S * d->head_dim * sizeof(float));
    w.page_lse = off;     off += align256(rows * size_t(max_pages) * sizeof(float));
    w.split_ml = off;     off += align256(rows * S * sizeof(float2));
    w.score_acc = off;    off += align256(size_t(batch) * size_t(max_pages) * sizeof(unsigned long long));
    w.keys = off;         off += align256(size_t(batch) * size_t(max_pages) * sizeof(uint32_t));
    w.logits = off;       off += with_logits ? align256(rows * size_t(max_pages) * kPage * sizeof(float)) : 0;
    w.total = off;
    return w;
}

delta_status check_desc(const delta_desc* d) {
    if (d == nullptr) return DELTA_ERR_INVALID_ARG;
    if (d->num_q_heads <= 0 || d->num_kv_heads <= 0 || d->head_dim <= 0 || d->page_size <= 0 ||
        d->num_phys_pages < 0)
        return DELTA_ERR_INVALID_ARG;
    if (d->num_q_heads % d->num_kv_heads != 0) return DELTA_ERR_INVALID_ARG;
    if (d->dtype != DELTA_F32 && d->dtype != DELTA_BF16) return DELTA_ERR_INVALID_ARG;
    if (!(d->sm_scale >= 0.f) || isinf(d->sm_scale)) return DELTA_ERR_INVALID_ARG;
    if (d->page_size != kPage) return DELTA_ERR_UNSUPPORTED;
    if (d->head_dim != 64 && d->head_dim != 128) return DELTA_ERR_UNSUPPORTED;
    if (d->num_q_heads / d->num_kv_heads > kMaxGroup) return DELTA_ERR_UNSUPPORTED;
    if (d->num_kv_heads > 64) return DELTA_ERR_UNSUPPORTED;
    // rows of the pool viewed as a [pages * Hkv * 16, D] matrix must fit a 32-bit TMA coordinate
    if (d->num_phys_pages * d->num_kv_heads * kPage > int64_t(INT32_MAX)) return DELTA_ERR_UNSUPPORTED;
    return DELTA_OK;
}

delta_status check_pt(const delta_page_table* pt) {
    if (pt == nullptr || pt->batch < 0) return DELTA_ERR_INVALID_ARG;
    if (pt->batch == 0) return DELTA_OK;
    if (pt->page_indptr == nullptr || pt->page_indices == nullptr || pt->kv_len == nullptr) return DELTA_ERR_INVALID_ARG;
    if (pt->max_pages_per_seq <= 0) return DELTA_ERR_INVALID_ARG;
    if (pt->batch > 65535) return DELTA_ERR_UNSUPPORTED;
    return DELTA_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

delta_status launch_status() { return cudaPeekAtLastError() == cudaSuccess ? DELTA_OK : DELTA_ERR_CUDA; }

// ---- tensor maps (driver entry point resolved through the runtime; no libcuda link needed)
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    std::lock_guard<std::recursive_mutex> lock(cache_mutex());
    if (fn == nullptr) {
        void* ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(ptr);
    }
    return fn;
}

// A bf16 pool [pages][Hkv][16][D] seen as a [pages*Hkv*16, D] matrix, 16-row x 64-column boxes,
// 128-byte swizzle (what the ldmatrix addressing of the tensor-core kernel assumes).
bool make_pool_map(CUtensorMap* map, const void* pool, const delta_desc* d) {
    EncodeTiledFn enc = encode_fn();
    if (enc == nullptr) return false;
    const cuuint64_t dims[2] = {cuuint64_t(d->head_dim), cuuint64_t(d->num_phys_pages) * d->num_kv_heads * kPage};
    const cuuint64_t strides[1] = {cuuint64_t(d->head_dim) * 2};
    const cuuint32_t box[2] = {64, kPage};
    const cuuint32_t estr[2] = {1, 1};
    return enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(pool), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// ---- kernel selection and cluster occupancy
template <int D, int G>
const void* mma_ptr(int variant, size_t* smem) {
    if (variant == kVarWide) {
        *smem = MmaSmem<D, kMmaStages, kMmaWideWarps>::kBytes;
        return reinterpret_cast<const void*>(decode_mma_kernel<D, G, kMmaStages, kMmaWideWarps>);
    }
    if (variant == kVarShort) {
        *smem = MmaSmem<D, kMmaShortStages, kMmaShortWarps>::kBytes;
        return reinterpret_cast<const void*>(decode_mma_kernel<D, G, kMmaShortStages, kMmaShortWarps>);
    }
    *smem = MmaSmem<D, kMmaStages>::kBytes;
    return reinterpret_cast<const void*>(decode_mma_kernel<D, G, kMmaStages, kWarps>);
}
template <int D, int G>
const void* simt_ptr(size_t* smem) {
    constexpr int STAGES = simt_stages(4, D);
    *smem = DecodeSmem<float, D, STAGES>::kBytes;
    return reinterpret_cast<const void*>(decode_kernel<float, D, G, STAGES>);
}
#define DELTA_G_PTR(G, CALL)  \
    switch (G) {               \
        case 1: return CALL(1); \
        case 2: return CALL(2); \
        case 3: return CALL(3); \
        case 4: return CALL(4); \
        case 5: return CALL(5); \
        case 6: return CALL(6); \
        case 7: return CALL(7); \
        case 8: return CALL(8); \
        default: return nullptr; \
    }
const void* decode_ptr(int dtype, int D, int G, int variant, size_t* smem) {
    if (dtype == DELTA_BF16) {
        if (D == 128) {
#define CALL(g) mma_ptr<128, g>(variant, smem)
            DELTA_G_PTR(G, CALL)
#undef CALL
        }
#define CALL(g) mma_ptr<64, g>(variant, smem)
        DELTA_G_PTR(G, CALL)
#undef CALL
    }
    if (D == 128) {
#define CALL(g) simt_ptr<128, g>(smem)
        DELTA_G_PTR(G, CALL)
#undef CALL
    }
#define CALL(g) simt_ptr<64, g>(smem)
    DELTA_G_PTR(G, CALL)
#undef CALL
}

// One-time per-device attributes of a decode kernel (shared-memory limit, cluster sizes > 8).
bool configure_kernel(const void* func, size_t smem) {
    constexpr int kSlots = 256;
    static const void* done_fn[64][kSlots];
    std::lock_guard<std::recursive_mutex> lock(cache_mutex());
    const int dev = current_device();
    if (dev < 0) return false;
    int i = 0;
    for (; i < kSlots && done_fn[dev][i] != nullptr; ++i)
        if (done_fn[dev][i] == func) return true;
    if (cudaFuncSetAttribute(func, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem)) != cudaSuccess ||
        cudaFuncSetAttribute(func, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) != cudaSuccess)
        return false;
    if (i < kSlots) done_fn[dev][i] = func;
    return true;
}

// Clusters of `cluster` CTAs of this kernel that can be resident at once (cached per device).
int max_active_clusters(const void* func, size_t smem, int cluster, int threads) {
    constexpr int kSlots = 512;
    struct Entry { const void* fn; int cluster; int n; };
    static Entry cache[64][kSlots];
    std::lock_guard<std::recursive_mutex> lock(cache_mutex());
    const int dev = current_device();
    if (dev < 0) return 1;
    int i = 0;
    for (; i < kSlots && cache[dev][i].fn != nullptr; ++i)
        if (cache[dev][i].fn == func && cache[dev][i].cluster == cluster) return cache[dev][i].n;
    if (!configure_kernel(func, smem)) return 1;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(cluster, 1, 1);
    cfg.blockDim = dim3(threads);
    cfg.dynamicSmemBytes = smem;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = cluster;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, func, &cfg) != cudaSuccess || n < 1) {
        cudaGetLastError();
        n = 1;
    }
    if (i < kSlots) cache[dev][i] = {func, cluster, n};
    return n;
}

// Fit a split plan to the clusters that can be resident at once.  Among cluster sizes C <= the
// plan's, pick the (C, clusters) pair with the most CTAs (C * clusters <= the plan's splits) whose
// units * clusters all fit in one wave; ties go to the larger cluster (fewer cross-cluster
// partials).  Long sequences thus keep ~one wave of CTAs even where large clusters do not pack
// into the GPCs.
// one_cluster_per_unit: delta-layers that select their pages at the end of the decode keep every
// (sequence, KV head) unit in one cluster, so each CTA gets the unit's per-head normalisers from the
// cluster merge (a unit spread over several clusters needs a second arrival stage).
SplitPlan fit_plan(SplitPlan pl, int dtype, int D, int G, int units, int items, bool one_cluster_per_unit = false) {
    const int s = pl.splits();
    // Clusters meet through the workspace only when each gets at least 256 pages (and the unit has
    // more than 512): below that the cross-cluster merge costs more than the extra CTAs gain.
    // Up to 512 pages per (sequence, KV head) one cluster is faster (measured on the 8k stack).
    constexpr int per_cluster = DELTA_PAGES_PER_CLUSTER, one_cluster = DELTA_ONE_CLUSTER_PAGES;
    const int max_clusters =
        (one_cluster_per_unit || items <= one_cluster || items / per_cluster < 1) ? 1 : items / per_cluster;
    SplitPlan best = pl;
    int best_ctas = -1;
    for (int c = pl.cluster; c >= 1; --c) {
        SplitPlan cand = pl;
        cand.cluster = c;
        cand.clusters = s / c < max_clusters ? s / c : max_clusters;
        if (cand.clusters < 1) continue;
        size_t smem = 0;
        const void* fn = decode_ptr(dtype, D, G, cand.variant, &smem);
        if (fn == nullptr) return pl;
        const int maxc = max_active_clusters(fn, smem, c, dtype == DELTA_BF16 ? variant_threads(cand.variant) : kThreads);
        if (int64_t(units) * cand.clusters > maxc) {
            cand.clusters = maxc / units;
            if (cand.clusters < 1) continue;
        }
        const int ctas = c * cand.clusters;
        if (ctas > best_ctas) {
            best = cand;
            best_ctas = ctas;
        }
    }
    if (best_ctas < 0) {   // more units than resident clusters even at size 1: several waves
        best.cluster = 1;
        best.clusters = 1;
        best.variant = kVarNarrow;
    }
    return best;
}

// Launch with programmatic dependent launch: the kernel may be scheduled while the previous
// kernel of the stream drains; it waits for it in pdl_wait() before touching global memory.
template <typename K, typename... Args>
delta_status launch_pdl(K kern, dim3 grid, dim3 block, size_t smem, cudaStream_t st, Args... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaLaunchKernelEx(&cfg, kern, args...) != cudaSuccess) return DELTA_ERR_CUDA;
    return launch_status();
}

// Launch a decode kernel as clusters of `cluster` CTAs along the split dimension.
template <typename K, typename... Args>
delta_status launch_clustered(K kern, size_t smem, int threads, const DecodeParams& prm, int cluster, int batch,
                              int Hkv, cudaStream_t st, Args... args) {
    if (!configure_kernel(reinterpret_cast<const void*>(kern), smem)) return DELTA_ERR_CUDA;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(prm.num_splits, Hkv, batch);
    cfg.blockDim = dim3(threads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = cluster;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    if (cudaLaunchKernelEx(&cfg, kern, prm, args...) != cudaSuccess) return DELTA_ERR_CUDA;
    return launch_status();
}

template <typename T, int D, int G>
delta_status launch_simt_g(const DecodeParams& prm, int cluster, int batch, int Hkv, cudaStream_t st) {
    constexpr int STAGES = simt_stages(int(sizeof(T)), D);
    return launch_clustered(decode_kernel<T, D, G, STAGES>, DecodeSmem<T, D, STAGES>::kBytes, kThreads, prm, cluster,
                            batch, Hkv, st);
}

template <int D, int G>
delta_status launch_mma_g(const DecodeParams& prm, const CUtensorMap& mk, const CUtensorMap& mv, int cluster,
                          int variant, int batch, int Hkv, cudaStream_t st) {
    if (variant == kVarWide)
        return launch_clustered(decode_mma_kernel<D, G, kMmaStages, kMmaWideWarps>,
                                MmaSmem<D, kMmaStages, kMmaWideWarps>::kBytes, kMmaWideWarps * 32, prm, cluster, batch,
                                Hkv, st, mk, mv);
    if (variant == kVarShort)
        return launch_clustered(decode_mma_kernel<D, G, kMmaShortStages, kMmaShortWarps>,
                                MmaSmem<D, kMmaShortStages, kMmaShortWarps>::kBytes, kMmaShortWarps * 32, prm, cluster,
                                batch, Hkv, st, mk, mv);
    return launch_clustered(decode_mma_kernel<D, G, kMmaStages, kWarps>, MmaSmem<D, kMmaStages>::kBytes, kThreads, prm,
                            cluster, batch, Hkv, st, mk, mv);
}

#define DELTA_G_SWITCH(G, CALL) \
    switch (G) {                  \
        case 1: return CALL(1);   \
        case 2: return CALL(2);   \
        case 3: return CALL(3);   \
        case 4: return CALL(4);   \
        case 5: return CALL(5);   \
        case 6: return CALL(6);   \
        case 7: return CALL(7);   \
        case 8: return CALL(8);   \
        default: return DELTA_ERR_UNSUPPORTED; \
    }

delta_status launch_decode(const delta_desc* d, const DecodeParams& prm, int cluster, int variant, int batch,
                           cudaStream_t st) {
    const int Hkv = d->num_kv_heads, G = d->num_q_heads / Hkv;
    if (d->dtype == DELTA_BF16) {
        CUtensorMap mk, mv;
        if (!make_pool_map(&mk, prm.k_pool, d) || !make_pool_map(&mv, prm.v_pool, d)) return DELTA_ERR_CUDA;
        if (d->head_dim == 128) {
#define CALL(g) launch_mma_g<128, g>(prm, mk, mv, cluster, variant, batch, Hkv, st)
            DELTA_G_SWITCH(G, CALL)
#undef CALL
        } else {
#define CALL(g) launch_mma_g<64, g>(prm, mk, mv, cluster, variant, batch, Hkv, st)
            DELTA_G_SWITCH(G, CALL)
#undef CALL
        }
    }
    if (d->head_dim == 128) {
#define CALL(g) launch_simt_g<float, 128, g>(prm, cluster, batch, Hkv, st)
        DELTA_G_SWITCH(G, CALL)
#undef CALL
    }
#define CALL(g) launch_simt_g<float, 64, g>(prm, cluster, batch, Hkv, st)
    DELTA_G_SWITCH(G, CALL)
#undef CALL
}

// Shared driver of the three attention entry points.
delta_status run_attention(int mode, const delta_desc* d, const delta_page_table* pt, const delta_select_params* sp,
                           const int32_t* sel_cnt_in, const int32_t* sel_pages_in, int32_t sel_stride_in,
                           const void* q, const void* k_pool, const void* v_pool, void* o, int32_t* sel_cnt_out,
                           int32_t* sel_pages_out, int32_t sel_stride_out, float* page_scores, void* ws,
                           size_t ws_bytes, void* stream, bool settled = false) {
    delta_status s = check_desc(d);
    if (s != DELTA_OK) return s;
    s = check_pt(pt);
    if (s != DELTA_OK) return s;
    if (mode == kModeDelta) {
        if (sp == nullptr) return DELTA_ERR_INVALID_ARG;
        if (sp->budget_pages < 0 || sp->sink_tokens < 0 || sp->recency_tokens < 0) return DELTA_ERR_INVALID_ARG;
        if (sp->reduce != DELTA_HEAD_SUM && sp->reduce != DELTA_HEAD_MAX) return DELTA_ERR_INVALID_ARG;
        if (d->num_q_heads > kMaxQHeadsSelect) return DELTA_ERR_UNSUPPORTED;
    }
    if (pt->batch == 0) return DELTA_OK;
    if (q == nullptr || k_pool == nullptr || v_pool == nullptr || o == nullptr) return DELTA_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k_pool) || !aligned16(v_pool) || !aligned16(o)) return DELTA_ERR_INVALID_ARG;
    if (mode == kModeDelta) {
        if (sel_cnt_out == nullptr || sel_pages_out == nullptr) return DELTA_ERR_INVALID_ARG;
        if (sel_stride_out < delta_sel_capacity(sp, d->page_size)) return DELTA_ERR_INVALID_ARG;
        if (pt->max_pages_per_seq > kMaxSelectPages) return DELTA_ERR_UNSUPPORTED;
    }
    if (mode == kModeSparse) {
        if (sel_cnt_in == nullptr || sel_pages_in == nullptr || sel_stride_in <= 0) return DELTA_ERR_INVALID_ARG;
    }
    if (ws == nullptr || (reinterpret_cast<uintptr_t>(ws) & 255u) != 0) return DELTA_ERR_WORKSPACE;
    const bool head_max = mode == kModeDelta && sp->reduce == DELTA_HEAD_MAX;
    const WsLayout L = ws_layout(d, pt->batch, pt->max_pages_per_seq, head_max);
    if (ws_bytes < L.total) return DELTA_ERR_WORKSPACE;

    const int D = d->head_dim, Hq = d->num_q_heads, Hkv = d->num_kv_heads;
    int items = pt->max_pages_per_seq;
    if (mode == kModeSparse && sel_stride_in < items) items = sel_stride_in;
    const SplitPlan plan = fit_plan(plan_splits(d->dtype, D, pt->batch, Hkv, items, mode == kModeDelta && !head_max), d->dtype, D, Hq / Hkv,
                                    pt->batch * Hkv, items, mode == kModeDelta && !head_max);
    // the in-kernel selection forms each unit's normalisers from its one cluster's merge
    if (mode == kModeDelta && !head_max && plan.clusters != 1) return DELTA_ERR_UNSUPPORTED;
    const int S = plan.splits();
    unsigned char* base = static_cast<unsigned char*>(ws);

    DecodeParams prm{};
    prm.q = q;
    prm.k_pool = k_pool;
    prm.v_pool = v_pool;
    prm.indptr = pt->page_indptr;
    prm.indices = pt->page_indices;
    prm.kv_len = pt->kv_len;
    prm.sel_cnt = sel_cnt_in;
    prm.sel_pages = sel_pages_in;
    prm.sel_stride = sel_stride_in;
    prm.num_q_heads = Hq;
    prm.num_kv_heads = Hkv;
    prm.items_per_split = (items + S - 1) / S;
    prm.num_splits = S;
    prm.max_pages = pt->max_pages_per_seq;
    prm.num_phys_pages = d->num_phys_pages;
    const float scale = d->sm_scale > 0.f ? d->sm_scale : 1.0f / sqrtf(float(D));
    prm.qscale = scale * 1.4426950408889634f;
    prm.mode = mode;
    prm.part_ml = reinterpret_cast<float2*>(base + L.part_ml);
    prm.part_o = reinterpret_cast<float*>(base + L.part_o);
    prm.page_lse = reinterpret_cast<float*>(base + L.page_lse);
    prm.split_ml = mode == kModeDelta ? reinterpret_cast<float2*>(base + L.split_ml) : nullptr;
    prm.err = reinterpret_cast<int*>(base + L.err);
    prm.o = o;
    prm.num_clusters = plan.clusters;
    prm.logits = head_max ? reinterpret_cast<float*>(base + L.logits) : nullptr;
    prm.tickets = reinterpret_cast<int*>(base + L.tickets);
    prm.settled = (mode == kModeSparse && settled) ? 1 : 0;
    // delta-layers scoring with HEAD_SUM select their pages at the end of the decode kernel
    prm.fuse_select = (mode == kModeDelta && !head_max) ? 1 : 0;
    if (prm.fuse_select) {
        prm.budget_pages = sp->budget_pages;
        prm.sink_tokens = sp->sink_tokens;
        prm.recency_tokens = sp->recency_tokens;
        prm.sel_cnt_out = sel_cnt_out;
        prm.sel_pages_out = sel_pages_out;
        prm.sel_stride_out = sel_stride_out;
        prm.page_scores = page_scores;
        prm.score_acc = reinterpret_cast<unsigned long long*>(base + L.score_acc);
        prm.keys = reinterpret_cast<uint32_t*>(base + L.keys);
        prm.seq_tickets = reinterpret_cast<int*>(base + L.seq_tickets);
    }

    cudaStream_t st = static_cast<cudaStream_t>(stream);
    s = launch_decode(d, prm, plan.cluster, plan.variant, pt->batch, st);
    if (s != DELTA_OK || mode != kModeDelta || prm.fuse_select) return s;

    SelectParams sp2{};
    sp2.indptr = pt->page_indptr;
    sp2.kv_len = pt->kv_len;
    sp2.page_lse = prm.page_lse;
    sp2.split_ml = prm.split_ml;
    sp2.num_splits = S;
    sp2.num_q_heads = Hq;
    sp2.max_pages = pt->max_pages_per_seq;
    sp2.budget_pages = sp->budget_pages;
    sp2.sink_tokens = sp->sink_tokens;
    sp2.recency_tokens = sp->recency_tokens;
    sp2.sel_cnt = sel_cnt_out;
    sp2.sel_pages = sel_pages_out;
    sp2.sel_stride = sel_stride_out;
    sp2.page_scores = page_scores;
    sp2.logits = prm.logits;
    sp2.err = prm.err;
    // one cluster of C CTAs per sequence, about 16K page terms per CTA; HEAD_MAX scores every
    // token of every head (a warp per page), so there a CTA takes about one page per warp
    const int maxp = pt->max_pages_per_seq;
    int C = head_max ? (maxp + kSelectThreads / 32 - 1) / (kSelectThreads / 32)
                     : int((int64_t(Hq) * maxp + 16383) / 16384);
    C = C < 1 ? 1 : (C > 16 ? 16 : C);
    const int chunk = (maxp + C - 1) / C;
    const SelectSmem SL{chunk, C};
    // C >= Hq * maxp / 16384 (or 16) keeps a CTA's pages at 16384 or fewer
    if (chunk > kMaxSelectChunk) return DELTA_ERR_UNSUPPORTED;
    const size_t smem_max = SelectSmem{kMaxSelectChunk, 16}.bytes();
    if (!configure_kernel(reinterpret_cast<const void*>(score_select_kernel), smem_max)) return DELTA_ERR_CUDA;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(C, pt->batch);
    cfg.blockDim = dim3(kSelectThreads);
    cfg.dynamicSmemBytes = SL.bytes();
    cfg.stream = st;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = C;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    if (cudaLaunchKernelEx(&cfg, score_select_kernel, sp2, chunk) != cudaSuccess) return DELTA_ERR_CUDA;
    return launch_status();
}

// ------------------------------------------------------------------ allocation-free variant
// Scratch of delta_full_attn_noalloc: a fixed array in the library's own device memory, so the
// call needs no workspace from the caller.  Every GPU that loads the library holds it until the
// process exits.
constexpr size_t kStaticScratchBytes = size_t(8) << 20;   // 8 MiB
static __device__ __align__(256) unsigned char g_noalloc_scratch[kStaticScratchBytes];

// Device address of the scratch array on the current device, looked up once per device.  In
// host code the array's name only stands for the symbol; the kernel must get this address.
unsigned char* noalloc_scratch() {
    static unsigned char* addr[64] = {nullptr};
    std::lock_guard<std::recursive_mutex> lock(cache_mutex());
    const int dev = current_device();
    if (dev < 0) return nullptr;
    if (addr[dev] == nullptr) {
        void* ptr = nullptr;
        if (cudaGetSymbolAddress(&ptr, g_noalloc_scratch) != cudaSuccess || ptr == nullptr) return nullptr;
        addr[dev] = static_cast<unsigned char*>(ptr);
    }
    return addr[dev];
}

}  // namespace delta

using namespace delta;

// ================================================================== C ABI
extern "C" {

size_t delta_workspace_size(const delta_desc* desc, int32_t batch, int32_t max_pages_per_seq) {
    if (check_desc(desc) != DELTA_OK || batch < 0 || max_pages_per_seq < 0) return 0;
    return ws_layout(desc, batch, max_pages_per_seq).total;
}

size_t delta_workspace_size_reduce(const delta_desc* desc, int32_t batch, int32_t max_pages_per_seq, int32_t reduce) {
    if (check_desc(desc) != DELTA_OK || batch < 0 || max_pages_per_seq < 0) return 0;
    if (reduce != DELTA_HEAD_SUM && reduce != DELTA_HEAD_MAX) return 0;
    return ws_layout(desc, batch, max_pages_per_seq, reduce == DELTA_HEAD_MAX).total;
}

delta_status delta_workspace_init(void* workspace, size_t ws_bytes, void* stream) {
    if (workspace == nullptr) return DELTA_ERR_INVALID_ARG;
    if (cudaMemsetAsync(workspace, 0, ws_bytes, static_cast<cudaStream_t>(stream)) != cudaSuccess) return DELTA_ERR_CUDA;
    return DELTA_OK;
}

int32_t delta_sel_capacity(const delta_select_params* sp, int32_t page_size) {
    if (sp == nullptr || page_size <= 0 || sp->budget_pages < 0 || sp->sink_tokens < 0 || sp->recency_tokens < 0)
        return -1;
    const int32_t sink = (sp->sink_tokens + page_size - 1) / page_size;
    const int32_t rec = sp->recency_tokens > 0 ? (sp->recency_tokens + page_size - 1) / page_size + 1 : 0;
    return sp->budget_pages + sink + rec;
}

delta_status delta_kv_append(const delta_desc* desc, const delta_page_table* pt, const void* k_new,
                             const void* v_new, void* k_pool, void* v_pool, void* stream) {
    delta_status s = check_desc(desc);
    if (s != DELTA_OK) return s;
    s = check_pt(pt);
    if (s != DELTA_OK) return s;
    if (pt->batch == 0) return DELTA_OK;
    if (k_new == nullptr || v_new == nullptr || k_pool == nullptr || v_pool == nullptr) return DELTA_ERR_INVALID_ARG;
    if (!aligned16(k_new) || !aligned16(v_new) || !aligned16(k_pool) || !aligned16(v_pool)) return DELTA_ERR_INVALID_ARG;
    // kv_append has no workspace to flag errors in: an out-of-range page is skipped, and the
    // attention call that follows on the same page table flags it.
    const int row_vecs = desc->head_dim * elem_bytes(desc->dtype) / 16;
    return launch_pdl(kv_append_kernel, dim3(pt->batch, desc->num_kv_heads), dim3(32), 0,
                      static_cast<cudaStream_t>(stream), static_cast<const uint4*>(k_new),
                      static_cast<const uint4*>(v_new), static_cast<uint4*>(k_pool), static_cast<uint4*>(v_pool),
                      pt->page_indptr, pt->page_indices, pt->kv_len, desc->num_kv_heads, row_vecs,
                      desc->num_phys_pages);
}

delta_status delta_kv_append_layers(const delta_desc* desc, const delta_page_table* pt, int32_t num_layers,
                                    const void* const* k_new, const void* const* v_new, void* const* k_pools,
                                    void* const* v_pools, void* stream) {
    delta_status s = check_desc(desc);
    if (s != DELTA_OK) return s;
    s = check_pt(pt);
    if (s != DELTA_OK) return s;
    if (num_layers < 0 || num_layers > kMaxAppendLayers) return num_layers < 0 ? DELTA_ERR_INVALID_ARG : DELTA_ERR_UNSUPPORTED;
    if (pt->batch == 0 || num_layers == 0) return DELTA_OK;
    if (k_new == nullptr || v_new == nullptr || k_pools == nullptr || v_pools == nullptr) return DELTA_ERR_INVALID_ARG;
    AppendLayers a = {};
    for (int l = 0; l < num_layers; ++l) {
        if (k_new[l] == nullptr || v_new[l] == nullptr || k_pools[l] == nullptr || v_pools[l] == nullptr)
            return DELTA_ERR_INVALID_ARG;
        if (!aligned16(k_new[l]) || !aligned16(v_new[l]) || !aligned16(k_pools[l]) || !aligned16(v_pools[l]))
            return DELTA_ERR_INVALID_ARG;
        a.k_new[l] = static_cast<const uint4*>(k_new[l]);
        a.v_new[l] = static_cast<const uint4*>(v_new[l]);
        a.k_pool[l] = static_cast<uint4*>(k_pools[l]);
        a.v_pool[l] = static_cast<uint4*>(v_pools[l]);
    }
    const int row_vecs = desc->head_dim * elem_bytes(desc->dtype) / 16;
    return launch_pdl(kv_append_layers_kernel, dim3(pt->batch, desc->num_kv_heads, num_layers), dim3(32), 0,
                      static_cast<cudaStream_t>(stream), a, pt->page_indptr, pt->page_indices, pt->kv_len,
                      desc->num_kv_heads, row_vecs, desc->num_phys_pages);
}

delta_status delta_full_attn(const delta_desc* desc, const delta_page_table* pt, const void* q, const void* k_pool,
                             const void* v_pool, void* o, void* workspace, size_t ws_bytes, void* stream) {
    return run_attention(kModeFull, desc, pt, nullptr, nullptr, nullptr, 0, q, k_pool, v_pool, o, nullptr, nullptr, 0,
                         nullptr, workspace, ws_bytes, stream);
}

delta_status delta_full_attn_noalloc(const delta_desc* desc, const delta_page_table* pt, const void* q,
                                     const void* k_pool, const void* v_pool, void* o, void* stream) {
    delta_status s = check_desc(desc);
    if (s != DELTA_OK) return s;
    s = check_pt(pt);
    if (s != DELTA_OK) return s;
    if (pt->batch == 0) return DELTA_OK;
    const WsLayout L = ws_layout(desc, pt->batch, pt->max_pages_per_seq);
    if (L.total > kStaticScratchBytes) return DELTA_ERR_UNSUPPORTED;   // shape needs more scratch than the array holds
    unsigned char* ws = noalloc_scratch();
    if (ws == nullptr) return DELTA_ERR_CUDA;
    // the error word and the split-arrival tickets must start at zero; the rest is overwritten
    if (cudaMemsetAsync(ws, 0, L.part_ml, static_cast<cudaStream_t>(stream)) != cudaSuccess) return DELTA_ERR_CUDA;
    return run_attention(kModeFull, desc, pt, nullptr, nullptr, nullptr, 0, q, k_pool, v_pool, o, nullptr, nullptr, 0,
                         nullptr, ws, kStaticScratchBytes, stream);
}

delta_status delta_select_attn(const delta_desc* desc, const delta_page_table* pt, const delta_select_params* sp,
                               const void* q, const void* k_pool, const void* v_pool, void* o, int32_t* sel_cnt,
                               int32_t* sel_pages, int32_t sel_stride, float* page_scores, void* workspace,
                               size_t ws_bytes, void* stream) {
    return run_attention(kModeDelta, desc, pt, sp, nullptr, nullptr, 0, q, k_pool, v_pool, o, sel_cnt, sel_pages,
                         sel_stride, page_scores, workspace, ws_bytes, stream);
}

delta_status delta_sparse_attn(const delta_desc* desc, const delta_page_table* pt, const int32_t* sel_cnt,
                               const int32_t* sel_pages, int32_t sel_stride, const void* q, const void* k_pool,
                               const void* v_pool, void* o, void* workspace, size_t ws_bytes, void* stream) {
    return run_attention(kModeSparse, desc, pt, nullptr, sel_cnt, sel_pages, sel_stride, q, k_pool, v_pool, o, nullptr,
                         nullptr, 0, nullptr, workspace, ws_bytes, stream);
}

delta_status delta_sparse_attn_settled(const delta_desc* desc, const delta_page_table* pt, const int32_t* sel_cnt,
                                       const int32_t* sel_pages, int32_t sel_stride, const void* q,
                                       const void* k_pool, const void* v_pool, void* o, void* workspace,
                                       size_t ws_bytes, void* stream) {
    return run_attention(kModeSparse, desc, pt, nullptr, sel_cnt, sel_pages, sel_stride, q, k_pool, v_pool, o, nullptr,
                         nullptr, 0, nullptr, workspace, ws_bytes, stream, true);
}

delta_status delta_layer_shift(const delta_page_table* pt, const float* scores_a, const float* scores_b,
                               float* shift_out, void* stream) {
    delta_status s = check_pt(pt);
    if (s != DELTA_OK) return s;
    if (pt->batch == 0) return DELTA_OK;
    if (scores_a == nullptr || scores_b == nullptr || shift_out == nullptr) return DELTA_ERR_INVALID_ARG;
    return launch_pdl(layer_shift_kernel, dim3(pt->batch), dim3(kShiftThreads), 0, static_cast<cudaStream_t>(stream),
                      scores_a, scores_b, pt->page_indptr, pt->kv_len, pt->max_pages_per_seq, shift_out);
}

delta_status delta_choose_layers(const float* shift, int32_t num_layers, int32_t count, int32_t first,
                                 int32_t min_gap, int32_t* out_layers, int32_t* out_count) {
    if (shift == nullptr || out_layers == nullptr || out_count == nullptr) return DELTA_ERR_INVALID_ARG;
    if (num_layers <= 0 || num_layers > 4096 || first < 0 || first >= num_layers || min_gap < 0)
        return DELTA_ERR_INVALID_ARG;
    for (int32_t l = 0; l < num_layers; ++l)
        if (!(shift[l] == shift[l])) return DELTA_ERR_INVALID_ARG;   // NaN has no order
    int32_t n = 0;
    out_layers[n++] = first;
    // candidates after `first` by decreasing shift, equal shifts lower layer first; a candidate is
    // kept when at least min_gap layers away from every kept layer
    bool used[4096] = {false};
    while (n < count) {
        int32_t best = -1;
        for (int32_t l = first + 1; l < num_layers; ++l) {
            if (used[l]) continue;
            if (best < 0 || shift[l] > shift[best]) best = l;
        }
        if (best < 0) break;
        used[best] = true;
        bool far = true;
        for (int32_t i = 0; i < n; ++i) {
            const int32_t d = best > out_layers[i] ? best - out_layers[i] : out_layers[i] - best;
            if (d < min_gap) far = false;
        }
        if (far) out_layers[n++] = best;
    }
    for (int32_t i = 1; i < n; ++i)   // ascending
        for (int32_t j = i; j > 0 && out_layers[j - 1] > out_layers[j]; --j) {
            const int32_t t = out_layers[j];
            out_layers[j] = out_layers[j - 1];
            out_layers[j - 1] = t;
        }
    *out_count = n;
    return DELTA_OK;
}

delta_status delta_read_device_error(void* workspace, int32_t* flags_out, void* stream) {
    if (workspace == nullptr) return DELTA_ERR_INVALID_ARG;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    int32_t h = 0;
    if (cudaMemcpyAsync(&h, workspace, sizeof(int32_t), cudaMemcpyDeviceToHost, st) != cudaSuccess) return DELTA_ERR_CUDA;
    if (cudaMemsetAsync(workspace, 0, sizeof(int32_t), st) != cudaSuccess) return DELTA_ERR_CUDA;
    if (cudaStreamSynchronize(st) != cudaSuccess) return DELTA_ERR_CUDA;
    if (flags_out != nullptr) *flags_out = h;
    return h ? DELTA_ERR_BOUNDS : DELTA_OK;
}

const char* delta_status_string(delta_status s) {
    switch (s) {
        case DELTA_OK: return "ok";
        case DELTA_ERR_INVALID_ARG: return "invalid argument";
        case DELTA_ERR_UNSUPPORTED: return "unsupported shape or mode";
        case DELTA_ERR_WORKSPACE: return "workspace missing, misaligned or too small";
        case DELTA_ERR_CUDA: return "CUDA launch or runtime error";
        case DELTA_ERR_BOUNDS: return "device-side bounds check failed";
        default: return "unknown status";
    }
}

}  // extern "C"

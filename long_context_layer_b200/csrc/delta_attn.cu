// DELTA decode attention stack for B200 (sm_100a): kernels and the C ABI of include/delta_attn.h.
//
// Method: "DELTA: Dynamic Layer-Aware Token Attention for Efficient Long-Context Reasoning",
// ai.info summary, section "Methodology in Plain English".  Initial layers run full attention,
// delta-layers run full attention and score 16-token KV pages, sparse layers attend only to
// the selected pages; the paged KV cache is kept in full.
//
// Kernels (all launched on the caller's stream, none synchronises the host):
//   kv_append_kernel      one (sequence, KV head) per CTA, 16-byte vector copies.
//   decode_kernel         split-KV online-softmax decode.  Grid (split, KV head, sequence).
//                         Each of the 4 warps streams whole pages (K and V of one KV head,
//                         2*16*D elements) from HBM into its own shared-memory ring with
//                         1-D TMA bulk copies (cp.async.bulk + mbarrier transaction counts)
//                         and packs the G query heads of the group against them: a half-warp
//                         owns 8 tokens of a page, a lane owns D/16 dimensions; partial dot
//                         products are reduce-scattered across the half-warp so each lane
//                         ends with one (token, head) logit.  The delta variant also writes
//                         each page's (max logit, sum exp) per query head.  The sparse
//                         variant walks the selected page list instead of 0..N-1.
//                         The split partials of a (sequence, KV head) are merged by whichever
//                         of its CTAs arrives last (an atomic ticket; no CTA ever waits), which
//                         writes o and, for delta-layers, each head's (max, sum-exp) pair.
//   score_select_kernel   one CTA per sequence: page score = sum over heads of
//                         2^(m_hp - M_h) l_hp / L_h, then an MSB-first 4x8-bit radix select of
//                         the k-th largest candidate score with shared-memory histograms,
//                         lower-index tie-break by a block prefix scan, union with sink and
//                         recency pages, ascending compaction.
//
// Logits are carried in base 2 (q is pre-scaled by sm_scale*log2(e)) so every exponential is
// one exp2.  No floating-point atomics are used: results are deterministic run to run.

#include "delta_attn.h"

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>

#include "common.cuh"
#include "decode_simt.cuh"
#include "decode_mma.cuh"
#include "select.cuh"

namespace delta {

// ------------------------------------------------------------------ host side
constexpr int kMmaStages = 3;      // tensor-core kernel: stages per warp (8 KB each for D = 128)
constexpr int kMaxQHeadsSelect = 256;

struct WsLayout {
    size_t err, tickets, part_ml, part_o, page_ml, total;
};

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

int elem_bytes(int dtype) { return dtype == DELTA_BF16 ? 2 : 4; }

int current_device() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return -1;
    return dev;
}

int device_sm_count() {
    static int cache[64] = {0};
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

// Split count: one full wave of CTAs over the GPU, at least 4 pages per CTA (one per warp).
int num_splits_for(int dtype, int D, int batch, int Hkv, int items) {
    if (items <= 0) return 1;
    const int slots = device_sm_count() * ctas_per_sm(dtype, D);
    const int units = batch * Hkv;
    int s = slots / (units > 0 ? units : 1);
    const int cap = (items + kWarps - 1) / kWarps;
    if (s > cap) s = cap;
    if (s > kMaxSplits) s = kMaxSplits;
    if (s < 1) s = 1;
    const int ips = (items + s - 1) / s;
    return (items + ips - 1) / ips;
}

WsLayout ws_layout(const delta_desc* d, int batch, int max_pages) {
    WsLayout w{};
    const int S = num_splits_for(d->dtype, d->head_dim, batch, d->num_kv_heads, max_pages);
    const size_t rows = size_t(batch) * d->num_q_heads;
    size_t off = 0;
    w.err = off;        off += align256(64);
    w.tickets = off;    off += align256(size_t(batch) * d->num_kv_heads * sizeof(int));
    w.part_ml = off;    off += align256(rows * S * sizeof(float2));
    w.part_o = off;     off += align256(rows * S * d->head_dim * sizeof(float));
    w.page_ml = off;    off += align256(rows * size_t(max_pages) * sizeof(float2));
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

// Raise a kernel's dynamic shared-memory limit once per device.
template <typename K>
bool set_smem_once(K kern, size_t bytes, int* configured) {
    const int dev = current_device();
    if (dev < 0) return false;
    if (!configured[dev]) {
        if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, int(bytes)) != cudaSuccess)
            return false;
        configured[dev] = 1;
    }
    return true;
}

// ---- tensor maps (driver entry point resolved through the runtime; no libcuda link needed)
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
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

template <typename T, int D, int G>
delta_status launch_simt_g(const DecodeParams& prm, int batch, int Hkv, cudaStream_t st) {
    constexpr int STAGES = simt_stages(int(sizeof(T)), D);
    using Sm = DecodeSmem<T, D, STAGES>;
    auto kern = decode_kernel<T, D, G, STAGES>;
    static int configured[64] = {0};
    if (!set_smem_once(kern, Sm::kBytes, configured)) return DELTA_ERR_CUDA;
    kern<<<dim3(prm.num_splits, Hkv, batch), kThreads, Sm::kBytes, st>>>(prm);
    return launch_status();
}

template <int D, int G>
delta_status launch_mma_g(const DecodeParams& prm, const CUtensorMap& mk, const CUtensorMap& mv, int batch, int Hkv,
                          cudaStream_t st) {
    using Sm = MmaSmem<D, kMmaStages>;
    auto kern = decode_mma_kernel<D, G, kMmaStages>;
    static int configured[64] = {0};
    if (!set_smem_once(kern, Sm::kBytes, configured)) return DELTA_ERR_CUDA;
    kern<<<dim3(prm.num_splits, Hkv, batch), kThreads, Sm::kBytes, st>>>(prm, mk, mv);
    return launch_status();
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

delta_status launch_decode(const delta_desc* d, const DecodeParams& prm, int batch, cudaStream_t st) {
    const int Hkv = d->num_kv_heads, G = d->num_q_heads / Hkv;
    if (d->dtype == DELTA_BF16) {
        CUtensorMap mk, mv;
        if (!make_pool_map(&mk, prm.k_pool, d) || !make_pool_map(&mv, prm.v_pool, d)) return DELTA_ERR_CUDA;
        if (d->head_dim == 128) {
#define CALL(g) launch_mma_g<128, g>(prm, mk, mv, batch, Hkv, st)
            DELTA_G_SWITCH(G, CALL)
#undef CALL
        } else {
#define CALL(g) launch_mma_g<64, g>(prm, mk, mv, batch, Hkv, st)
            DELTA_G_SWITCH(G, CALL)
#undef CALL
        }
    }
    if (d->head_dim == 128) {
#define CALL(g) launch_simt_g<float, 128, g>(prm, batch, Hkv, st)
        DELTA_G_SWITCH(G, CALL)
#undef CALL
    }
#define CALL(g) launch_simt_g<float, 64, g>(prm, batch, Hkv, st)
    DELTA_G_SWITCH(G, CALL)
#undef CALL
}

// Shared driver of the three attention entry points.
delta_status run_attention(int mode, const delta_desc* d, const delta_page_table* pt, const delta_select_params* sp,
                           const int32_t* sel_cnt_in, const int32_t* sel_pages_in, int32_t sel_stride_in,
                           const void* q, const void* k_pool, const void* v_pool, void* o, int32_t* sel_cnt_out,
                           int32_t* sel_pages_out, int32_t sel_stride_out, float* page_scores, void* ws,
                           size_t ws_bytes, void* stream) {
    delta_status s = check_desc(d);
    if (s != DELTA_OK) return s;
    s = check_pt(pt);
    if (s != DELTA_OK) return s;
    if (mode == kModeDelta) {
        if (sp == nullptr) return DELTA_ERR_INVALID_ARG;
        if (sp->budget_pages < 0 || sp->sink_tokens < 0 || sp->recency_tokens < 0) return DELTA_ERR_INVALID_ARG;
        if (sp->reduce != DELTA_HEAD_SUM) return sp->reduce == DELTA_HEAD_MAX ? DELTA_ERR_UNSUPPORTED : DELTA_ERR_INVALID_ARG;
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
    const WsLayout L = ws_layout(d, pt->batch, pt->max_pages_per_seq);
    if (ws_bytes < L.total) return DELTA_ERR_WORKSPACE;

    const int D = d->head_dim, Hq = d->num_q_heads, Hkv = d->num_kv_heads;
    int items = pt->max_pages_per_seq;
    if (mode == kModeSparse && sel_stride_in < items) items = sel_stride_in;
    const int S = num_splits_for(d->dtype, D, pt->batch, Hkv, items);
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
    prm.page_ml = reinterpret_cast<float2*>(base + L.page_ml);
    prm.err = reinterpret_cast<int*>(base + L.err);
    prm.o = o;
    prm.lse = nullptr;
    prm.tickets = reinterpret_cast<int*>(base + L.tickets);

    cudaStream_t st = static_cast<cudaStream_t>(stream);
    s = launch_decode(d, prm, pt->batch, st);
    if (s != DELTA_OK || mode != kModeDelta) return s;

    SelectParams sp2{};
    sp2.indptr = pt->page_indptr;
    sp2.kv_len = pt->kv_len;
    sp2.page_ml = prm.page_ml;
    sp2.num_q_heads = Hq;
    sp2.max_pages = pt->max_pages_per_seq;
    sp2.budget_pages = sp->budget_pages;
    sp2.sink_tokens = sp->sink_tokens;
    sp2.recency_tokens = sp->recency_tokens;
    sp2.sel_cnt = sel_cnt_out;
    sp2.sel_pages = sel_pages_out;
    sp2.sel_stride = sel_stride_out;
    sp2.page_scores = page_scores;
    sp2.err = prm.err;
    static int configured[64] = {0};
    if (!set_smem_once(score_select_kernel, size_t(kMaxSelectPages) * sizeof(uint32_t), configured))
        return DELTA_ERR_CUDA;
    score_select_kernel<<<pt->batch, kSelectThreads, size_t(pt->max_pages_per_seq) * sizeof(uint32_t), st>>>(sp2);
    return launch_status();
}

}  // namespace delta

using namespace delta;

// ================================================================== C ABI
extern "C" {

size_t delta_workspace_size(const delta_desc* desc, int32_t batch, int32_t max_pages_per_seq) {
    if (check_desc(desc) != DELTA_OK || batch < 0 || max_pages_per_seq < 0) return 0;
    return ws_layout(desc, batch, max_pages_per_seq).total;
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
    kv_append_kernel<<<dim3(pt->batch, desc->num_kv_heads), 32, 0, static_cast<cudaStream_t>(stream)>>>(
        static_cast<const uint4*>(k_new), static_cast<const uint4*>(v_new), static_cast<uint4*>(k_pool),
        static_cast<uint4*>(v_pool), pt->page_indptr, pt->page_indices, pt->kv_len, desc->num_kv_heads, row_vecs,
        desc->num_phys_pages);
    return launch_status();
}

delta_status delta_full_attn(const delta_desc* desc, const delta_page_table* pt, const void* q, const void* k_pool,
                             const void* v_pool, void* o, void* workspace, size_t ws_bytes, void* stream) {
    return run_attention(kModeFull, desc, pt, nullptr, nullptr, nullptr, 0, q, k_pool, v_pool, o, nullptr, nullptr, 0,
                         nullptr, workspace, ws_bytes, stream);
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

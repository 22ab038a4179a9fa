// Shared device helpers of the DELTA decode kernels (included by delta_attn.cu only).
#pragma once

#include <cooperative_groups.h>
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>

namespace delta {


constexpr int kPage = 16;
constexpr int kWarps = 4;
constexpr int kThreads = kWarps * 32;
constexpr int kMaxGroup = 8;
constexpr int kMaxSelectPages = 32768;
constexpr int kMaxSelectChunk = 16384;   // pages one CTA of the selection cluster owns at most
constexpr int kSelectThreads = 1024;
constexpr int kMaxQHeadsSelect = 256;   // query heads a delta-layer selection supports
constexpr int kMaxSplits = 512;   // the merge stages G*S*12 bytes of split weights in shared memory
constexpr uint32_t kWaitLimit = 1u << 24;   // try_wait polls before a stage wait gives up

enum : int { kErrPage = 1, kErrLen = 2, kErrSel = 4, kErrTimeout = 8 };
enum : int { kModeFull = 0, kModeDelta = 1, kModeSparse = 2 };

// ------------------------------------------------------------------ PTX helpers
__device__ __forceinline__ uint32_t smem_addr(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(bar)), "r"(count) : "memory");
}
__device__ __forceinline__ void fence_mbar_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
__device__ __forceinline__ void fence_proxy_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
__device__ __forceinline__ void mbar_expect_tx(uint64_t* bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_addr(bar)), "r"(bytes)
                 : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_addr(bar)) : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n selp.u32 %0, 1, 0, p;\n}"
        : "=r"(ok)
        : "r"(smem_addr(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}
// Bounded wait: false after kWaitLimit unsuccessful polls (each poll may suspend briefly).
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity) {
    for (uint32_t i = 0; i < kWaitLimit; ++i)
        if (mbar_try_wait(bar, parity)) return true;
    return false;
}
__device__ __forceinline__ uint64_t evict_first_policy() {
    uint64_t pol;
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
    return pol;
}
// 1-D TMA bulk copy global -> shared, completion counted on an mbarrier; KV is read once per
// layer, so it is marked evict-first in L2.
__device__ __forceinline__ void bulk_load(void* dst, const void* src, uint32_t bytes, uint64_t* bar,
                                          uint64_t policy) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint [%0], [%1], %2, [%3], %4;" ::
            "r"(smem_addr(dst)),
        "l"(src), "r"(bytes), "r"(smem_addr(bar)), "l"(policy)
        : "memory");
}

// Bulk prefetch of a global range into L2 (no shared-memory destination, no completion).
// Distributed shared memory: the cluster address of a shared variable in CTA `rank`, and an
// asynchronous 8- or 16-byte store into it whose arrival is counted (in bytes) on that CTA's mbarrier.
__device__ __forceinline__ uint32_t cluster_addr(const void* p, uint32_t rank) {
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(smem_addr(p)), "r"(rank));
    return r;
}
__device__ __forceinline__ void st_async(uint32_t dst, float4 v, uint32_t bar) {
    asm volatile("st.async.shared::cluster.mbarrier::complete_tx::bytes.v4.f32 [%0], {%1, %2, %3, %4}, [%5];" ::"r"(dst),
                 "f"(v.x), "f"(v.y), "f"(v.z), "f"(v.w), "r"(bar)
                 : "memory");
}
__device__ __forceinline__ void st_async(uint32_t dst, float2 v, uint32_t bar) {
    asm volatile("st.async.shared::cluster.mbarrier::complete_tx::bytes.v2.f32 [%0], {%1, %2}, [%3];" ::"r"(dst),
                 "f"(v.x), "f"(v.y), "r"(bar)
                 : "memory");
}
__device__ __forceinline__ void cluster_arrive_relaxed() {
    asm volatile("barrier.cluster.arrive.relaxed.aligned;" ::: "memory");
}
__device__ __forceinline__ void cluster_wait() { asm volatile("barrier.cluster.wait.aligned;" ::: "memory"); }

__device__ __forceinline__ void prefetch_l2(const void* src, uint32_t bytes) {
    asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(src), "r"(bytes) : "memory");
}

__device__ __forceinline__ float exp2_approx(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}
__device__ __forceinline__ float log2_approx(float x) {
    float y;
    asm("lg2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// ------------------------------------------------------------------ element access
template <typename T>
struct Elem;
template <>
struct Elem<float> {
    static __device__ __forceinline__ float to_f(float x) { return x; }
    static __device__ __forceinline__ float from_f(float x) { return x; }
};
template <>
struct Elem<__nv_bfloat16> {
    static __device__ __forceinline__ float to_f(__nv_bfloat16 x) { return __bfloat162float(x); }
    static __device__ __forceinline__ __nv_bfloat16 from_f(float x) { return __float2bfloat16_rn(x); }
};

__device__ __forceinline__ void unpack_bf16x2(uint32_t w, float& lo, float& hi) {
    lo = __uint_as_float(w << 16);
    hi = __uint_as_float(w & 0xffff0000u);
}

// Load N consecutive elements (16-byte aligned) as floats.
template <typename T, int N>
__device__ __forceinline__ void load_row(const T* p, float (&x)[N]);

template <>
__device__ __forceinline__ void load_row<__nv_bfloat16, 8>(const __nv_bfloat16* p, float (&x)[8]) {
    uint4 w = *reinterpret_cast<const uint4*>(p);
    unpack_bf16x2(w.x, x[0], x[1]);
    unpack_bf16x2(w.y, x[2], x[3]);
    unpack_bf16x2(w.z, x[4], x[5]);
    unpack_bf16x2(w.w, x[6], x[7]);
}
template <>
__device__ __forceinline__ void load_row<__nv_bfloat16, 4>(const __nv_bfloat16* p, float (&x)[4]) {
    uint2 w = *reinterpret_cast<const uint2*>(p);
    unpack_bf16x2(w.x, x[0], x[1]);
    unpack_bf16x2(w.y, x[2], x[3]);
}
template <>
__device__ __forceinline__ void load_row<float, 8>(const float* p, float (&x)[8]) {
    float4 a = reinterpret_cast<const float4*>(p)[0];
    float4 b = reinterpret_cast<const float4*>(p)[1];
    x[0] = a.x; x[1] = a.y; x[2] = a.z; x[3] = a.w;
    x[4] = b.x; x[5] = b.y; x[6] = b.z; x[7] = b.w;
}
template <>
__device__ __forceinline__ void load_row<float, 4>(const float* p, float (&x)[4]) {
    float4 a = *reinterpret_cast<const float4*>(p);
    x[0] = a.x; x[1] = a.y; x[2] = a.z; x[3] = a.w;
}

// Order-preserving 32-bit key of a float (larger float, larger key).
__device__ __forceinline__ uint32_t order_key(float f) {
    const uint32_t u = __float_as_uint(f);
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

__host__ __device__ constexpr int pad_group(int g) { return g <= 1 ? 1 : g <= 2 ? 2 : g <= 4 ? 4 : 8; }

// ------------------------------------------------------------------ decode kernel
struct DecodeParams {
    const void* q;
    const void* k_pool;
    const void* v_pool;
    const int32_t* indptr;
    const int32_t* indices;
    const int32_t* kv_len;
    const int32_t* sel_cnt;
    const int32_t* sel_pages;
    int32_t sel_stride;
    int32_t num_q_heads;
    int32_t num_kv_heads;
    int32_t items_per_split;
    int32_t num_splits;
    int32_t max_pages;
    int64_t num_phys_pages;
    float qscale;  // sm_scale * log2(e)
    int32_t mode;
    float2* part_ml;  // [B][Hq][S]  (max, sum) of each split, base-2 logits
    float* part_o;    // [B][Hq][S][D] unnormalised outputs of each split
    float* page_lse;  // [B][Hq][max_pages] per-page log2-sum-exp of base-2 logits (delta-layers)
    float2* split_ml; // [B][Hq][S] (max, sum) of each split CTA's own pages (delta-layers)
    void* o;          // [B][Hq][D] output
    int32_t num_clusters;   // clusters along the split dimension (num_splits = cluster size * this)
    // sparse layers: the selection, pools and page table were final before the previous kernel
    // of the stream began, so they are read (and the pages loaded) before waiting on it
    int32_t settled;
    float* logits;          // [B][Hq][max_pages*16] base-2 logits (delta-layers in HEAD_MAX mode), else null
    int* tickets;     // [B][Hkv] arrival counters of the split CTAs, zero between launches
    int* err;
    // Delta-layers scoring with HEAD_SUM: the page selection runs at the end of the decode kernel
    // (select_tail.cuh) instead of in a separate launch.
    int32_t fuse_select;
    int32_t budget_pages, sink_tokens, recency_tokens;
    int32_t* sel_cnt_out;     // [B]
    int32_t* sel_pages_out;   // [B][sel_stride_out]
    int32_t sel_stride_out;
    float* page_scores;       // [B][max_pages] or null
    unsigned long long* score_acc;   // [B][max_pages] page scores in 2^-55 fixed point, summed over the
                                     // KV heads by integer atomics; zero between launches
    uint32_t* keys;           // [B][max_pages] order keys of the page scores (when shared memory is short)
    int* seq_tickets;         // [B] units of a sequence that finished, zero between launches
};



// ------------------------------------------------------------------ programmatic dependent launch
// Wait until the grids this one depends on have completed and their writes are visible.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
// Let the next kernel in the stream be scheduled (its CTAs still wait in pdl_wait()).
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

// ------------------------------------------------------------------ page lists
// Logical and physical page of the pages a warp streams, fetched by all 32 lanes at once (one
// page per lane, so the two dependent loads are paid once per 32 pages) and kept one chunk of
// 32 pages ahead of use.  Pages that must be skipped get phys = -1 (and raise an error flag).
struct WarpPages {
    int lp_a, ph_a;   // chunk `cur`
    int lp_b, ph_b;   // chunk `cur + 1`
    int cur;
};

struct SeqExtent {
    int n;                  // tokens (clamped)
    int N;                  // pages
    int pbeg;               // first entry of the sequence in page_indices
    int count;              // items to attend: N, or the selection length
};

// QUIET: a speculative lookup (before the wait, for an L2 prefetch only) that raises no flags.
// W: warps of the CTA (warp w streams items i0 + w, i0 + w + W, ...).
template <bool QUIET = false, int W = kWarps, typename P>
__device__ __forceinline__ void fetch_pages(const P& p, const SeqExtent& ex, int b, int i0, int warp, int nk, int kbase,
                                            int lane, int& lp, int& ph) {
    const int k = kbase + lane;
    lp = -1;
    ph = -1;
    if (k >= nk) return;
    const int i = i0 + warp + k * W;
    // the selection is read from L2 (another kernel of the step wrote it; no stale L1 line)
    lp = (p.mode == kModeSparse) ? __ldcg(p.sel_pages + size_t(b) * p.sel_stride + i) : i;
    if (lp < 0 || lp >= ex.N) {
        if (!QUIET) atomicOr(p.err, kErrSel);
        lp = -1;
        return;
    }
    const int64_t x = p.indices[ex.pbeg + lp];
    if (x < 0 || x >= p.num_phys_pages) {
        if (!QUIET) atomicOr(p.err, kErrPage);
        return;
    }
    ph = int(x);
}

template <int W = kWarps, typename P>
__device__ __forceinline__ void pages_init(WarpPages& w, const P& p, const SeqExtent& ex, int b, int i0, int warp,
                                           int nk, int lane) {
    w.cur = 0;
    fetch_pages<false, W>(p, ex, b, i0, warp, nk, 0, lane, w.lp_a, w.ph_a);
    fetch_pages<false, W>(p, ex, b, i0, warp, nk, 32, lane, w.lp_b, w.ph_b);
}

// Called by all lanes at the top of iteration k (uniform).
template <int W = kWarps, typename P>
__device__ __forceinline__ void pages_advance(WarpPages& w, const P& p, const SeqExtent& ex, int b, int i0, int warp,
                                              int nk, int lane, int k) {
    if (k > 0 && (k & 31) == 0) {
        w.cur = k >> 5;
        w.lp_a = w.lp_b;
        w.ph_a = w.ph_b;
        fetch_pages<false, W>(p, ex, b, i0, warp, nk, (w.cur + 1) * 32, lane, w.lp_b, w.ph_b);
    }
}

// Page k of the warp (all lanes call; k must lie in chunk cur or cur + 1).
__device__ __forceinline__ void pages_get(const WarpPages& w, int k, int& lp, int& ph) {
    const bool a = (k >> 5) == w.cur;
    lp = __shfl_sync(0xffffffffu, a ? w.lp_a : w.lp_b, k & 31);
    ph = __shfl_sync(0xffffffffu, a ? w.ph_a : w.ph_b, k & 31);
}

// Tokens and pages of sequence b, validated against the page table (bad values clamped and
// flagged).  Reads only the page table and kv_len, which are inputs of the whole step.
template <typename P>
__device__ __forceinline__ SeqExtent seq_extent(const P& p, int b) {
    SeqExtent ex;
    int n = p.kv_len[b];
    ex.pbeg = p.indptr[b];
    const int npg = p.indptr[b + 1] - ex.pbeg;
    if (n < 0) n = 0;
    if (n > npg * kPage || n > p.max_pages * kPage) {
        if (threadIdx.x == 0) atomicOr(p.err, kErrLen);
        n = min(max(npg, 0), p.max_pages) * kPage;
    }
    ex.n = n;
    ex.N = (n + kPage - 1) / kPage;
    ex.count = ex.N;
    return ex;
}

// Sparse layers: the number of selected pages (an output of the delta-layer: read after the wait).
template <typename P>
__device__ __forceinline__ void seq_count(const P& p, int b, SeqExtent& ex) {
    if (p.mode != kModeSparse) return;
    const int scnt = __ldcg(p.sel_cnt + b);
    const int cap = min(p.sel_stride, p.items_per_split * p.num_splits);
    ex.count = scnt;
    if (scnt < 0 || scnt > cap) {
        if (threadIdx.x == 0) atomicOr(p.err, kErrSel);
        ex.count = min(max(scnt, 0), cap);
    }
}

// Floats of the dedicated receive area of the cluster merge (never aliased with pipeline stages,
// so other CTAs of the cluster may push into it while this CTA is still streaming pages).  Its
// first 16 bytes hold the mbarrier that counts the bytes pushed into it.
template <int D>
constexpr int recv_floats() { return 4 + kMaxGroup * D + 16 * 4 + 16 * kMaxGroup * 4 + kMaxGroup * 2; }

// Per-CTA states [C][G][4] inside a cluster's merge receive area (after its barrier and the C slices).
template <int D, int G>
__device__ __forceinline__ const float* merge_recv_states(const float* recv, int C) {
    const int chunk = (((G * D + C - 1) / C) + 3) & ~3;
    return recv + 4 + C * chunk;
}

// Kernel prologue of the cluster merge, all threads, before the wait for the previous kernel:
// thread 0 initialises this CTA's receive barrier, then one cluster barrier makes every CTA's
// initialisation visible before any CTA can signal it (the CTAs of a cluster start together, so
// this costs nothing while the previous kernel is still running).
__device__ __forceinline__ void merge_prologue(float* recv) {
    if (threadIdx.x == 0) {
        mbar_init(reinterpret_cast<uint64_t*>(recv), 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    __syncwarp();
    cluster_arrive_relaxed();
    cluster_wait();
}

// Part rr's records: outputs mo[rr * ostride + h * OROW + d], states ml[rr * mstride + 2 * h] (max,
// sum) of base-2 logits; dml (delta-layers, same strides as ml) holds the states over the exact
// fp32 page terms when those differ from ml.
template <typename T, int D, int G, int NPART, int NTHR = kThreads, int OROW = D>
__device__ __forceinline__ void merge_epilogue(const DecodeParams& p, unsigned char* smem, const float* mo,
                                               const float* mml, float* recv, int b, int g, int ostride,
                                               int mstride, const float* dml = nullptr) {
    namespace cg = cooperative_groups;
    cg::cluster_group cluster = cg::this_cluster();
    const int C = int(cluster.num_blocks());
    const int rank = int(cluster.block_rank());
    const int cidx = blockIdx.x / C;
    const int nC = p.num_clusters;
    const int Hq = p.num_q_heads;
    const int h0 = g * G;
    const int tid = threadIdx.x, nthr = blockDim.x;
    const int warp = tid >> 5, lane = tid & 31;
    T* out = reinterpret_cast<T*>(p.o);

    // 1. this CTA's NPART states -> one state, pushed straight into the shared memory of the
    //    cluster CTA that owns each output element with asynchronous remote stores; each owner
    //    waits on its own barrier for the bytes of all C CTAs (no cluster-wide barrier, no round
    //    trip).  Every thread combines the parts' states it needs itself (no barrier).  Slices
    //    are multiples of 4 elements so every push is one 16-byte store.
    const int total = G * D;
    const int chunk = (((total + C - 1) / C) + 3) & ~3;
    uint64_t* rbar = reinterpret_cast<uint64_t*>(recv);
    recv += 4;
    // [C][G][4]: each CTA's (max, sum) per head, and on delta-layers also the state over the exact
    // fp32 page terms, from which every CTA forms the page scores' per-head normalisers itself
    float* recv_ml = recv + C * chunk;
    const bool delta = p.mode == kModeDelta;
    const int e0 = rank * chunk, e1 = min(e0 + chunk, total);                      // this CTA's slice
    if (tid == 0)
        mbar_expect_tx(rbar, uint32_t(C) * (uint32_t(max(e1 - e0, 0)) * 4u + uint32_t(G) * (delta ? 16u : 8u)));
    auto part_max = [&](const float* ml, int h) {
        float M = -INFINITY;
#pragma unroll
        for (int rr = 0; rr < NPART; ++rr) M = fmaxf(M, ml[rr * mstride + 2 * h]);
        return M;
    };
    auto part_sum = [&](const float* ml, int h, float M) {
        const float mu = (M == -INFINITY) ? 0.f : M;
        float L = 0.f;
#pragma unroll
        for (int rr = 0; rr < NPART; ++rr) L = fmaf(exp2_approx(ml[rr * mstride + 2 * h] - mu), ml[rr * mstride + 2 * h + 1], L);
        return L;
    };
    if (tid < C * G) {   // this CTA's (max, sum) of head h to cluster rank j
        const int j = tid / G, h = tid % G;
        const float M = part_max(mml, h);
        const float L = part_sum(mml, h, M);
        float Md = M, Ld = L;
        if (dml != nullptr) {
            Md = part_max(dml, h);
            Ld = part_sum(dml, h, Md);
        }
        if (delta)
            st_async(cluster_addr(recv_ml + (rank * G + h) * 4, j), make_float4(M, L, Md, Ld), cluster_addr(rbar, j));
        else
            st_async(cluster_addr(recv_ml + (rank * G + h) * 4, j), make_float2(M, L), cluster_addr(rbar, j));
        if (j == 0 && p.split_ml != nullptr)   // the selection combines its per-head totals from these
            p.split_ml[(size_t(b) * Hq + h0 + h) * p.num_splits + blockIdx.x] = make_float2(Md, Ld);
    }
    for (int q4 = tid; q4 * 4 < total; q4 += nthr) {
        const int idx = q4 * 4, h = idx / D, d = idx % D;    // D is a multiple of 4: one head per group
        const float M = part_max(mml, h);
        const float mu = (M == -INFINITY) ? 0.f : M;
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
        for (int rr = 0; rr < NPART; ++rr) {
            const float w = exp2_approx(mml[rr * mstride + 2 * h] - mu);
            const float4 v = *reinterpret_cast<const float4*>(&mo[rr * ostride + h * OROW + d]);
            acc.x = fmaf(w, v.x, acc.x);
            acc.y = fmaf(w, v.y, acc.y);
            acc.z = fmaf(w, v.z, acc.z);
            acc.w = fmaf(w, v.w, acc.w);
        }
        const int owner = idx / chunk;
        st_async(cluster_addr(recv + rank * chunk + (idx - owner * chunk), owner), acc, cluster_addr(rbar, owner));
    }
    // all C CTAs' bytes have landed (bounded wait; a timeout is flagged and the merge goes on)
    if (!mbar_wait(rbar, 0) && tid == 0) atomicOr(p.err, kErrTimeout);

    // 2. each CTA merges the C states of its slice from its own shared memory
    for (int e = e0 + tid; e < e1; e += nthr) {
        const int h = e / D, d = e % D;
        float M = -INFINITY;
        for (int j = 0; j < C; ++j) M = fmaxf(M, recv_ml[(j * G + h) * 4]);
        const float mu = (M == -INFINITY) ? 0.f : M;
        float L = 0.f, acc = 0.f;
        for (int j = 0; j < C; ++j) {
            const float w = exp2_approx(recv_ml[(j * G + h) * 4] - mu);
            L = fmaf(w, recv_ml[(j * G + h) * 4 + 1], L);
            acc = fmaf(w, recv[j * chunk + (e - e0)], acc);
        }
        if (nC == 1) {
            out[(size_t(b) * Hq + h0 + h) * D + d] = Elem<T>::from_f(M == -INFINITY ? 0.f : __fdividef(acc, L));
        } else {
            const size_t row = (size_t(b) * Hq + h0 + h) * nC + cidx;
            p.part_o[row * D + d] = acc;
            if (d == 0) p.part_ml[row] = make_float2(M, L);
        }
    }
    if (nC == 1) return;

    // 3. the last CTA of (b, g) to arrive merges the nC cluster partials
    __shared__ int s_last;
    __threadfence();
    __syncthreads();
    if (tid == 0) {
        const int t = atomicAdd(&p.tickets[b * p.num_kv_heads + g], 1);
        s_last = (t == C * nC - 1);
        if (s_last) p.tickets[b * p.num_kv_heads + g] = 0;   // ready for the next launch
    }
    __syncthreads();
    if (!s_last) return;
    __threadfence();
    float* sml = reinterpret_cast<float*>(smem);          // [G][nC] maxima, then weights
    float* sl = sml + G * nC;                              // [G][nC] sums
    float* sML = sl + G * nC;                              // [G][2]
    for (int idx = tid; idx < G * nC; idx += nthr) {
        const float2 ml = __ldcg(&p.part_ml[(size_t(b) * Hq + h0) * nC + idx]);
        sml[idx] = ml.x;
        sl[idx] = ml.y;
    }
    __syncthreads();
    for (int h = warp; h < G; h += nthr / 32) {
        float M = -INFINITY;
        for (int c = lane; c < nC; c += 32) M = fmaxf(M, sml[h * nC + c]);
#pragma unroll
        for (int o2 = 16; o2 >= 1; o2 >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o2));
        const float mu = (M == -INFINITY) ? 0.f : M;
        float Ls = 0.f;
        for (int c = lane; c < nC; c += 32) Ls += exp2_approx(sml[h * nC + c] - mu) * sl[h * nC + c];
#pragma unroll
        for (int o2 = 16; o2 >= 1; o2 >>= 1) Ls += __shfl_xor_sync(0xffffffffu, Ls, o2);
        if (lane == 0) { sML[2 * h] = M; sML[2 * h + 1] = Ls; }
    }
    __syncthreads();
    for (int idx = tid; idx < G * nC; idx += nthr) {
        const int h = idx / nC;
        const float M = sML[2 * h], Ls = sML[2 * h + 1];
        sml[idx] = (M == -INFINITY) ? 0.f : exp2_approx(sml[idx] - M) / Ls;
    }
    __syncthreads();
    constexpr int J = (G * D + NTHR - 1) / NTHR;   // outputs per thread
    float a[J];
#pragma unroll
    for (int j = 0; j < J; ++j) a[j] = 0.f;
#pragma unroll 2
    for (int c = 0; c < nC; ++c) {
#pragma unroll
        for (int j = 0; j < J; ++j) {
            const int idx = tid + j * NTHR;
            if (idx < G * D) {
                const int h = idx / D, d = idx % D;
                a[j] = fmaf(sml[h * nC + c], __ldcg(p.part_o + ((size_t(b) * Hq + h0 + h) * nC + c) * D + d), a[j]);
            }
        }
    }
#pragma unroll
    for (int j = 0; j < J; ++j) {
        const int idx = tid + j * NTHR;
        if (idx < G * D) out[(size_t(b) * Hq + h0 + idx / D) * D + idx % D] = Elem<T>::from_f(a[j]);
    }
}

}  // namespace delta

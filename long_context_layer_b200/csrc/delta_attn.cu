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

namespace {

constexpr int kPage = 16;
constexpr int kWarps = 4;
constexpr int kThreads = kWarps * 32;
constexpr int kMaxGroup = 8;
constexpr int kMaxSelectPages = 32768;
constexpr int kSelectThreads = 1024;
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

__device__ __forceinline__ float exp2_approx(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
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
    float2* page_ml;  // [B][Hq][max_pages] per-page (max, sum) for delta-layers
    void* o;          // [B][Hq][D] output
    float2* lse;      // [B][Hq] (max, sum) over the whole context, delta-layers only (else null)
    int* tickets;     // [B][Hkv] arrival counters of the split CTAs, zero between launches
    int* err;
};

template <typename T, int D, int STAGES>
struct DecodeSmem {
    static constexpr uint32_t kChunk = kPage * D * sizeof(T);                    // one K or V page
    static constexpr size_t kStages = size_t(kWarps) * STAGES * 2 * kChunk;
    static constexpr size_t kBars = size_t(kWarps) * STAGES * sizeof(uint64_t);
    static constexpr size_t kPbuf = size_t(kWarps) * 2 * 8 * kMaxGroup * sizeof(float);
    static constexpr size_t kAbuf = size_t(kWarps) * 2 * kMaxGroup * sizeof(float);
    static constexpr size_t kMerge = size_t(kWarps) * 2 * kMaxGroup * (D + 2) * sizeof(float);
    static constexpr size_t kMain = kStages > kMerge ? kStages : kMerge;
    static constexpr size_t kBytes = kMain + kBars + kPbuf + kAbuf;
};

template <typename T, int D, int G, int STAGES>
__global__ void __launch_bounds__(kThreads) decode_kernel(const DecodeParams p) {
    using S = DecodeSmem<T, D, STAGES>;
    constexpr int DS = D / 16;          // dimensions per lane
    constexpr int GP = pad_group(G);    // group padded to a power of two
    constexpr int PE = kPage * D;       // elements of one K or V page

    extern __shared__ __align__(128) unsigned char smem[];
    T* stages = reinterpret_cast<T*>(smem);
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + S::kMain);
    float* pbuf = reinterpret_cast<float*>(smem + S::kMain + S::kBars);
    float* abuf = pbuf + kWarps * 2 * 8 * kMaxGroup;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int half = lane >> 4, hl = lane & 15;
    const int b = blockIdx.z, g = blockIdx.y, split = blockIdx.x;
    const int Hq = p.num_q_heads;
    const int h0 = g * G;

    // ---- sequence extent (validated; bad values are clamped and flagged)
    int n = p.kv_len[b];
    const int pbeg = p.indptr[b];
    const int npg = p.indptr[b + 1] - pbeg;
    if (n < 0) n = 0;
    if (n > npg * kPage || n > p.max_pages * kPage) {   // beyond the sequence's pages or the stated bound
        if (threadIdx.x == 0) atomicOr(p.err, kErrLen);
        n = min(max(npg, 0), p.max_pages) * kPage;
    }
    const int N = (n + kPage - 1) / kPage;
    int count = N;
    if (p.mode == kModeSparse) {
        count = p.sel_cnt[b];
        if (count < 0 || count > p.sel_stride || count > p.items_per_split * p.num_splits) {
            if (threadIdx.x == 0) atomicOr(p.err, kErrSel);
            count = min(max(count, 0), min(p.sel_stride, p.items_per_split * p.num_splits));
        }
    }
    const int i0 = split * p.items_per_split;
    const int i1 = min(i0 + p.items_per_split, count);
    const int nk = (i1 - i0 > warp) ? (i1 - i0 - warp + kWarps - 1) / kWarps : 0;  // pages of this warp

    // ---- queries of the group, pre-scaled into base-2 logits
    float q[G][DS];
    {
        const T* qp = reinterpret_cast<const T*>(p.q) + (size_t(b) * Hq + h0) * D + hl * DS;
#pragma unroll
        for (int h = 0; h < G; ++h) {
            load_row<T, DS>(qp + size_t(h) * D, q[h]);
#pragma unroll
            for (int d = 0; d < DS; ++d) q[h][d] *= p.qscale;
        }
    }

    uint64_t* wbar = bars + warp * STAGES;
    T* wst = stages + size_t(warp) * STAGES * 2 * PE;
    if (lane == 0) {
#pragma unroll
        for (int s = 0; s < STAGES; ++s) mbar_init(&wbar[s], 1);
        fence_mbar_init();
    }
    __syncwarp();

    const T* kpool = reinterpret_cast<const T*>(p.k_pool);
    const T* vpool = reinterpret_cast<const T*>(p.v_pool);
    const uint64_t policy = evict_first_policy();

    // logical page of the warp's k-th item and its physical page; false if it must be skipped
    auto resolve = [&](int k, int& lp, int64_t& phys) -> bool {
        const int i = i0 + warp + k * kWarps;
        lp = (p.mode == kModeSparse) ? p.sel_pages[size_t(b) * p.sel_stride + i] : i;
        if (lp < 0 || lp >= N) return false;
        phys = p.indices[pbeg + lp];
        return phys >= 0 && phys < p.num_phys_pages;
    };
    auto issue = [&](int k) {  // lane 0 only
        int lp;
        int64_t phys;
        const int s = k % STAGES;
        if (resolve(k, lp, phys)) {
            T* dst = wst + size_t(s) * 2 * PE;
            const size_t off = (size_t(phys) * p.num_kv_heads + g) * PE;
            mbar_expect_tx(&wbar[s], 2 * S::kChunk);
            bulk_load(dst, kpool + off, S::kChunk, &wbar[s], policy);
            bulk_load(dst + PE, vpool + off, S::kChunk, &wbar[s], policy);
        } else {
            atomicOr(p.err, (lp < 0 || lp >= N) ? kErrSel : kErrPage);
            mbar_arrive(&wbar[s]);  // completes the phase with no data; consumers skip the page
        }
    };

    if (lane == 0)
        for (int k = 0; k < min(STAGES, nk); ++k) issue(k);

    float m_run = -INFINITY, l_run = 0.f;  // running state of head (hl & (GP-1)) of this half
    float o[G][DS];
#pragma unroll
    for (int h = 0; h < G; ++h)
#pragma unroll
        for (int d = 0; d < DS; ++d) o[h][d] = 0.f;

    float* wp = pbuf + (warp * 2 + half) * 8 * kMaxGroup;   // [8 tokens][8 heads]
    float* wa = abuf + (warp * 2 + half) * kMaxGroup;
    bool failed = false;
    int consumed = 0;

    for (int k = 0; k < nk; ++k) {
        const int s = k % STAGES;
        if (!mbar_wait(&wbar[s], (k / STAGES) & 1)) {
            if (lane == 0) atomicOr(p.err, kErrTimeout);
            failed = true;
            break;
        }
        consumed = k + 1;
        int lp;
        int64_t phys;
        if (resolve(k, lp, phys)) {
            const T* Ks = wst + size_t(s) * 2 * PE;
            const T* Vs = Ks + PE;
            const int tv = min(kPage, n - lp * kPage);     // valid tokens of this page
            float sc[8];
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                const int t = half * 8 + j;
                float kx[DS];
                load_row<T, DS>(Ks + t * D + hl * DS, kx);
                float v[GP];
#pragma unroll
                for (int h = 0; h < GP; ++h) {
                    float acc = 0.f;
                    if (h < G) {
#pragma unroll
                        for (int d = 0; d < DS; ++d) acc = fmaf(q[h < G ? h : 0][d], kx[d], acc);
                    }
                    v[h] = acc;
                }
                // reduce-scatter across the 16 lanes of the half-warp: lane keeps head (hl & (GP-1))
#pragma unroll
                for (int m = GP / 2; m >= 1; m >>= 1) {
                    const bool upper = (hl & m) != 0;
#pragma unroll
                    for (int i = 0; i < m; ++i) {
                        const float send = upper ? v[i] : v[i + m];
                        const float keep = upper ? v[i + m] : v[i];
                        v[i] = keep + __shfl_xor_sync(0xffffffffu, send, m);
                    }
                }
#pragma unroll
                for (int m = GP; m < 16; m <<= 1) v[0] += __shfl_xor_sync(0xffffffffu, v[0], m);
                sc[j] = (t < tv) ? v[0] : -INFINITY;
            }
            float mb = sc[0];
#pragma unroll
            for (int j = 1; j < 8; ++j) mb = fmaxf(mb, sc[j]);
            if (p.mode == kModeDelta) {
                const float mp = fmaxf(mb, __shfl_xor_sync(0xffffffffu, mb, 16));
                float e = 0.f;
#pragma unroll
                for (int j = 0; j < 8; ++j) e += exp2_approx(sc[j] - mp);
                e += __shfl_xor_sync(0xffffffffu, e, 16);
                if (half == 0 && hl < G)
                    p.page_ml[(size_t(b) * Hq + h0 + hl) * p.max_pages + lp] = make_float2(mp, e);
            }
            const float m_new = fmaxf(m_run, mb);
            const float mu = (m_new == -INFINITY) ? 0.f : m_new;
            const float alpha = exp2_approx(m_run - mu);
            float lsum = 0.f;
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                const float pj = exp2_approx(sc[j] - mu);
                lsum += pj;
                if (hl < G) wp[j * kMaxGroup + hl] = pj;
            }
            l_run = l_run * alpha + lsum;
            m_run = m_new;
            if (hl < G) wa[hl] = alpha;
            __syncwarp();
            float al[G];
#pragma unroll
            for (int h = 0; h < G; ++h) al[h] = wa[h];
#pragma unroll
            for (int h = 0; h < G; ++h)
#pragma unroll
                for (int d = 0; d < DS; ++d) o[h][d] *= al[h];
            const int jmax = min(8, tv - half * 8);
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                if (j < jmax) {
                    const int t = half * 8 + j;
                    float vx[DS];
                    load_row<T, DS>(Vs + t * D + hl * DS, vx);
                    float pj[G];
#pragma unroll
                    for (int h = 0; h < G; ++h) pj[h] = wp[j * kMaxGroup + h];
#pragma unroll
                    for (int h = 0; h < G; ++h)
#pragma unroll
                        for (int d = 0; d < DS; ++d) o[h][d] = fmaf(pj[h], vx[d], o[h][d]);
                }
            }
        }
        __syncwarp();
        if (lane == 0 && k + STAGES < nk) issue(k + STAGES);
    }
    if (failed) {
        // drain this warp's copies still in flight (bounded) before shared memory is released
        for (int k = consumed + 1; k < min(consumed + STAGES, nk); ++k) mbar_wait(&wbar[k % STAGES], (k / STAGES) & 1);
    }

    // ---- merge the 8 partial states (4 warps x 2 half-warps) of this CTA
    __syncthreads();
    float* mo = reinterpret_cast<float*>(smem);                 // [8][G][D]
    float* mml = mo + kWarps * 2 * kMaxGroup * D;              // [8][G][2]
    const int r = warp * 2 + half;
#pragma unroll
    for (int h = 0; h < G; ++h)
#pragma unroll
        for (int d = 0; d < DS; ++d) mo[(r * kMaxGroup + h) * D + hl * DS + d] = o[h][d];
    if (hl < G) {
        mml[(r * kMaxGroup + hl) * 2 + 0] = m_run;
        mml[(r * kMaxGroup + hl) * 2 + 1] = l_run;
    }
    __syncthreads();
    const int S_ = p.num_splits;
    for (int idx = threadIdx.x; idx < G * D; idx += kThreads) {
        const int h = idx / D, d = idx % D;
        float M = -INFINITY;
#pragma unroll
        for (int rr = 0; rr < kWarps * 2; ++rr) M = fmaxf(M, mml[(rr * kMaxGroup + h) * 2]);
        const float mu = (M == -INFINITY) ? 0.f : M;
        float L = 0.f, acc = 0.f;
#pragma unroll
        for (int rr = 0; rr < kWarps * 2; ++rr) {
            const float w = exp2_approx(mml[(rr * kMaxGroup + h) * 2] - mu);
            L = fmaf(w, mml[(rr * kMaxGroup + h) * 2 + 1], L);
            acc = fmaf(w, mo[(rr * kMaxGroup + h) * D + d], acc);
        }
        const size_t row = (size_t(b) * Hq + h0 + h) * S_ + split;
        p.part_o[row * D + d] = acc;
        if (d == 0) p.part_ml[row] = make_float2(M, L);
    }

    // ---- the last CTA of (b, g) to finish merges the splits; nobody waits for anybody
    __shared__ int s_last;
    __threadfence();
    __syncthreads();
    if (threadIdx.x == 0) {
        const int t = atomicAdd(&p.tickets[b * p.num_kv_heads + g], 1);
        s_last = (t == S_ - 1);
        if (s_last) p.tickets[b * p.num_kv_heads + g] = 0;   // ready for the next launch
    }
    __syncthreads();
    if (!s_last) return;
    __threadfence();
    T* out = reinterpret_cast<T*>(p.o);
    for (int idx = threadIdx.x; idx < G * D; idx += kThreads) {
        const int h = idx / D, d = idx % D;
        const size_t row = (size_t(b) * Hq + h0 + h) * S_;
        float M = -INFINITY;
        for (int s2 = 0; s2 < S_; ++s2) M = fmaxf(M, __ldcg(&p.part_ml[row + s2]).x);
        float res = 0.f, L = 0.f;
        if (M != -INFINITY) {
            float acc = 0.f;
            for (int s2 = 0; s2 < S_; ++s2) {
                const float2 ml = __ldcg(&p.part_ml[row + s2]);
                const float w = exp2_approx(ml.x - M);
                L = fmaf(w, ml.y, L);
                acc = fmaf(w, __ldcg(&p.part_o[(row + s2) * D + d]), acc);
            }
            res = acc / L;
        }
        out[(size_t(b) * Hq + h0 + h) * D + d] = Elem<T>::from_f(res);
        if (p.lse != nullptr && d == 0) p.lse[size_t(b) * Hq + h0 + h] = make_float2(M, L);
    }
}

// ------------------------------------------------------------------ score + select kernel
struct SelectParams {
    const int32_t* indptr;
    const int32_t* kv_len;
    const float2* page_ml;  // [B][Hq][max_pages]
    const float2* lse;      // [B][Hq]
    int32_t num_q_heads;
    int32_t max_pages;
    int32_t budget_pages, sink_tokens, recency_tokens;
    int32_t* sel_cnt;
    int32_t* sel_pages;
    int32_t sel_stride;
    float* page_scores;
    int* err;
};

__device__ __forceinline__ uint32_t order_key(float f) {
    const uint32_t u = __float_as_uint(f);
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// Exclusive block-wide prefix sum of one value per thread (blockDim.x == kSelectThreads).
__device__ __forceinline__ int block_exclusive_scan(int x, int* warp_sums, int& total) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    int incl = x;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
    }
    if (lane == 31) warp_sums[warp] = incl;
    __syncthreads();
    if (warp == 0) {
        int w = (lane < kSelectThreads / 32) ? warp_sums[lane] : 0;
        int wi = w;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, wi, o);
            if (lane >= o) wi += y;
        }
        warp_sums[lane] = wi - w;           // exclusive prefix of warp totals
        if (lane == 31) warp_sums[32] = wi;  // block total
    }
    __syncthreads();
    const int res = warp_sums[warp] + incl - x;
    total = warp_sums[32];
    __syncthreads();
    return res;
}

__global__ void __launch_bounds__(kSelectThreads) score_select_kernel(const SelectParams p) {
    extern __shared__ uint32_t keys[];  // [max_pages]
    __shared__ uint32_t hist[256];
    __shared__ int warp_sums[33];
    __shared__ uint32_t s_digit, s_above;

    const int b = blockIdx.x, tid = threadIdx.x;
    int n = p.kv_len[b];
    const int npg = p.indptr[b + 1] - p.indptr[b];
    if (n < 0) n = 0;
    if (n > npg * kPage) n = max(npg, 0) * kPage;   // flagged by the decode kernel
    const int N = min((n + kPage - 1) / kPage, p.max_pages);
    const int Hq = p.num_q_heads;
    const int sinkP = (min(p.sink_tokens, n) + kPage - 1) / kPage;
    const int recStart = (p.recency_tokens > 0) ? max(n - p.recency_tokens, 0) / kPage : N;

    // 1. page scores: S_j = sum_h 2^(m_hj - M_h) * l_hj / L_h
    for (int j = tid; j < N; j += kSelectThreads) {
        float sc = 0.f;
        for (int h = 0; h < Hq; ++h) {
            const float2 ml = p.page_ml[(size_t(b) * Hq + h) * p.max_pages + j];
            const float2 tot = p.lse[size_t(b) * Hq + h];
            sc += exp2_approx(ml.x - tot.x) * ml.y / tot.y;
        }
        keys[j] = order_key(sc);
        if (p.page_scores != nullptr) p.page_scores[size_t(b) * p.max_pages + j] = sc;
    }
    __syncthreads();

    auto forced = [&](int j) { return j < sinkP || j >= recStart; };
    // 2. number of candidates (pages neither sink nor recency)
    int my_c = 0;
    for (int j = tid; j < N; j += kSelectThreads) my_c += forced(j) ? 0 : 1;
    int ncand;
    block_exclusive_scan(my_c, warp_sums, ncand);
    const int k = p.budget_pages;

    // 3. radix select of the k-th largest candidate key (only when candidates exceed k)
    uint32_t T = 0, need_eq = 0;
    bool take_all = ncand <= k;
    if (!take_all && k > 0) {
        uint32_t prefix = 0, mask = 0, kk = k;
        for (int shift = 24; shift >= 0; shift -= 8) {
            for (int i = tid; i < 256; i += kSelectThreads) hist[i] = 0;
            __syncthreads();
            for (int j = tid; j < N; j += kSelectThreads) {
                const uint32_t key = keys[j];
                if (!forced(j) && (key & mask) == prefix) atomicAdd(&hist[(key >> shift) & 255u], 1u);
            }
            __syncthreads();
            if (tid < 32) {
                // lane covers digits 255-8*lane .. 248-8*lane (descending)
                uint32_t c[8], sum = 0;
#pragma unroll
                for (int i = 0; i < 8; ++i) { c[i] = hist[255 - 8 * tid - i]; sum += c[i]; }
                uint32_t incl = sum;
#pragma unroll
                for (int o = 1; o < 32; o <<= 1) {
                    const uint32_t y = __shfl_up_sync(0xffffffffu, incl, o);
                    if (tid >= o) incl += y;
                }
                const uint32_t excl = incl - sum;
                if (excl < kk && kk <= incl) {
                    uint32_t above = excl;
#pragma unroll
                    for (int i = 0; i < 8; ++i) {
                        if (above + c[i] >= kk) { s_digit = 255 - 8 * tid - i; s_above = above; break; }
                        above += c[i];
                    }
                }
            }
            __syncthreads();
            prefix |= s_digit << shift;
            mask |= 0xffu << shift;
            kk -= s_above;
            __syncthreads();
        }
        T = prefix;
        need_eq = kk;  // how many of the keys equal to T are taken (lowest page indices first)
    }

    // 4. rank of each T-valued candidate among equals, then the ascending compaction
    const int chunk = (N + kSelectThreads - 1) / kSelectThreads;
    const int jb = tid * chunk, je = min(jb + chunk, N);
    int eq_cnt = 0;
    if (!take_all && k > 0)
        for (int j = jb; j < je; ++j) eq_cnt += (!forced(j) && keys[j] == T) ? 1 : 0;
    int eq_tot;
    int eq_rank = block_exclusive_scan(eq_cnt, warp_sums, eq_tot);
    auto selected = [&](int j, int& eq_seen) -> bool {
        if (forced(j)) return true;
        if (take_all) return true;
        if (k <= 0) return false;
        const uint32_t key = keys[j];
        if (key > T) return true;
        if (key == T) return (uint32_t)(eq_rank + eq_seen++) < need_eq;
        return false;
    };
    int cnt = 0, seen = 0;
    for (int j = jb; j < je; ++j) cnt += selected(j, seen) ? 1 : 0;
    int total;
    int pos = block_exclusive_scan(cnt, warp_sums, total);
    seen = 0;
    for (int j = jb; j < je; ++j) {
        if (selected(j, seen)) {
            if (pos < p.sel_stride) p.sel_pages[size_t(b) * p.sel_stride + pos] = j;
            ++pos;
        }
    }
    if (tid == 0) p.sel_cnt[b] = min(total, p.sel_stride);
}

// ------------------------------------------------------------------ kv append kernel
__global__ void kv_append_kernel(const uint4* __restrict__ k_new, const uint4* __restrict__ v_new,
                                 uint4* __restrict__ k_pool, uint4* __restrict__ v_pool,
                                 const int32_t* __restrict__ indptr, const int32_t* __restrict__ indices,
                                 const int32_t* __restrict__ kv_len, int Hkv, int row_vecs,
                                 int64_t num_phys_pages) {
    const int b = blockIdx.x, g = blockIdx.y;
    const int n = kv_len[b];
    if (n <= 0) return;
    const int pos = n - 1;
    const int lp = pos / kPage, slot = pos % kPage;
    const int pbeg = indptr[b], npg = indptr[b + 1] - pbeg;
    if (lp >= npg) return;                       // flagged by the attention call
    const int64_t phys = indices[pbeg + lp];
    if (phys < 0 || phys >= num_phys_pages) return;
    const size_t src = (size_t(b) * Hkv + g) * row_vecs;
    const size_t dst = ((size_t(phys) * Hkv + g) * kPage + slot) * row_vecs;
    for (int i = threadIdx.x; i < row_vecs; i += blockDim.x) {
        k_pool[dst + i] = k_new[src + i];
        v_pool[dst + i] = v_new[src + i];
    }
}

// ------------------------------------------------------------------ host side
struct WsLayout {
    size_t err, tickets, part_ml, part_o, lse, page_ml, total;
};

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

int elem_bytes(int dtype) { return dtype == DELTA_BF16 ? 2 : 4; }

int device_sm_count() {
    static int cache[64] = {0};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
    if (cache[dev] == 0) {
        int sms = 0;
        if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || sms <= 0) sms = 148;
        cache[dev] = sms;
    }
    return cache[dev];
}

// CTAs of the decode kernel resident per SM, from its shared-memory footprint (the kernel is
// written so registers never limit it below this).
int stages_for(int dtype, int D) {
    const int stage = 2 * kPage * D * elem_bytes(dtype);
    int s = (24 * 1024) / stage;
    return s < 2 ? 2 : (s > 4 ? 4 : s);
}
size_t decode_smem_bytes(int dtype, int D) {
    const size_t chunk = size_t(kPage) * D * elem_bytes(dtype);
    const size_t st = size_t(kWarps) * stages_for(dtype, D) * 2 * chunk;
    const size_t merge = size_t(kWarps) * 2 * kMaxGroup * (D + 2) * sizeof(float);
    return (st > merge ? st : merge) + size_t(kWarps) * stages_for(dtype, D) * 8 +
           size_t(kWarps) * 2 * 8 * kMaxGroup * 4 + size_t(kWarps) * 2 * kMaxGroup * 4;
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
    w.lse = off;        off += align256(rows * sizeof(float2));
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
    if (d->num_kv_heads > 65535) return DELTA_ERR_UNSUPPORTED;
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

delta_status launch_status() {
    return cudaPeekAtLastError() == cudaSuccess ? DELTA_OK : DELTA_ERR_CUDA;
}

template <typename T, int D, int G>
delta_status launch_decode_g(const DecodeParams& prm, int batch, int Hkv, cudaStream_t st) {
    constexpr int STAGES = (24 * 1024) / (2 * kPage * D * int(sizeof(T))) < 2   ? 2
                           : (24 * 1024) / (2 * kPage * D * int(sizeof(T))) > 4 ? 4
                                                                                 : (24 * 1024) / (2 * kPage * D * int(sizeof(T)));
    using Sm = DecodeSmem<T, D, STAGES>;
    auto kern = decode_kernel<T, D, G, STAGES>;
    static int configured[64] = {0};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev >= 0 && dev < 64 && !configured[dev]) {
        if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, int(Sm::kBytes)) != cudaSuccess)
            return DELTA_ERR_CUDA;
        configured[dev] = 1;
    }
    dim3 grid(prm.num_splits, Hkv, batch);
    kern<<<grid, kThreads, Sm::kBytes, st>>>(prm);
    return launch_status();
}

template <typename T, int D>
delta_status launch_decode_d(int G, const DecodeParams& prm, int batch, int Hkv, cudaStream_t st) {
    switch (G) {
        case 1: return launch_decode_g<T, D, 1>(prm, batch, Hkv, st);
        case 2: return launch_decode_g<T, D, 2>(prm, batch, Hkv, st);
        case 3: return launch_decode_g<T, D, 3>(prm, batch, Hkv, st);
        case 4: return launch_decode_g<T, D, 4>(prm, batch, Hkv, st);
        case 5: return launch_decode_g<T, D, 5>(prm, batch, Hkv, st);
        case 6: return launch_decode_g<T, D, 6>(prm, batch, Hkv, st);
        case 7: return launch_decode_g<T, D, 7>(prm, batch, Hkv, st);
        case 8: return launch_decode_g<T, D, 8>(prm, batch, Hkv, st);
        default: return DELTA_ERR_UNSUPPORTED;
    }
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

    const int D = d->head_dim, Hq = d->num_q_heads, Hkv = d->num_kv_heads, G = Hq / Hkv;
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
    prm.lse = (mode == kModeDelta) ? reinterpret_cast<float2*>(base + L.lse) : nullptr;
    prm.tickets = reinterpret_cast<int*>(base + L.tickets);

    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (d->dtype == DELTA_BF16) {
        s = (D == 128) ? launch_decode_d<__nv_bfloat16, 128>(G, prm, pt->batch, Hkv, st)
                       : launch_decode_d<__nv_bfloat16, 64>(G, prm, pt->batch, Hkv, st);
    } else {
        s = (D == 128) ? launch_decode_d<float, 128>(G, prm, pt->batch, Hkv, st)
                       : launch_decode_d<float, 64>(G, prm, pt->batch, Hkv, st);
    }
    if (s != DELTA_OK) return s;

    float2* lse = prm.lse;

    if (mode == kModeDelta) {
        SelectParams sp2{};
        sp2.indptr = pt->page_indptr;
        sp2.kv_len = pt->kv_len;
        sp2.page_ml = prm.page_ml;
        sp2.lse = lse;
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
        const size_t smem = size_t(pt->max_pages_per_seq) * sizeof(uint32_t);
        static int configured[64] = {0};
        int dev = 0;
        cudaGetDevice(&dev);
        if (dev >= 0 && dev < 64 && !configured[dev]) {
            if (cudaFuncSetAttribute(score_select_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     kMaxSelectPages * int(sizeof(uint32_t))) != cudaSuccess)
                return DELTA_ERR_CUDA;
            configured[dev] = 1;
        }
        score_select_kernel<<<pt->batch, kSelectThreads, smem, st>>>(sp2);
        s = launch_status();
    }
    return s;
}

}  // namespace

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

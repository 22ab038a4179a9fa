// Shared device helpers of the DELTA decode kernels (included by delta_attn.cu only).
#pragma once

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
constexpr int kSelectThreads = 1024;
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


// Epilogue shared by the decode kernels.  mo [NPART][kMaxGroup][D] and mml [NPART][kMaxGroup][2]
// (in shared memory) hold NPART partial states (base-2 max, sum, unnormalised output) of the
// G query heads of this CTA.  They are merged into this split's partial in global memory; the
// last CTA of (b, g) to arrive then merges all splits and writes o (and lse for delta-layers).
template <typename T, int D, int G, int NPART>
__device__ __forceinline__ void split_epilogue(const DecodeParams& p, unsigned char* smem, const float* mo,
                                               const float* mml, int b, int g, int split) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int Hq = p.num_q_heads;
    const int h0 = g * G;
    const int S_ = p.num_splits;
    for (int idx = threadIdx.x; idx < G * D; idx += kThreads) {
        const int h = idx / D, d = idx % D;
        float M = -INFINITY;
#pragma unroll
        for (int rr = 0; rr < NPART; ++rr) M = fmaxf(M, mml[(rr * kMaxGroup + h) * 2]);
        const float mu = (M == -INFINITY) ? 0.f : M;
        float L = 0.f, acc = 0.f;
#pragma unroll
        for (int rr = 0; rr < NPART; ++rr) {
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
    // Split weights w[h][s] = 2^(m_s - M_h) / L_h staged in shared memory, then every output
    // element sums its S partials with independent (unrolled) loads.
    float* sml = reinterpret_cast<float*>(smem);          // [G][S] (max) then weights
    float* sl = sml + G * S_;                              // [G][S] (sum)
    float* sML = sl + G * S_;                              // [G][2] (M, L)
    for (int idx = threadIdx.x; idx < G * S_; idx += kThreads) {
        const int h = idx / S_, s2 = idx % S_;
        const float2 ml = __ldcg(&p.part_ml[(size_t(b) * Hq + h0 + h) * S_ + s2]);
        sml[idx] = ml.x;
        sl[idx] = ml.y;
    }
    __syncthreads();
    for (int h = warp; h < G; h += kWarps) {
        float M = -INFINITY;
        for (int s2 = lane; s2 < S_; s2 += 32) M = fmaxf(M, sml[h * S_ + s2]);
#pragma unroll
        for (int o2 = 16; o2 >= 1; o2 >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o2));
        const float mu = (M == -INFINITY) ? 0.f : M;
        float Ls = 0.f;
        for (int s2 = lane; s2 < S_; s2 += 32) Ls += exp2_approx(sml[h * S_ + s2] - mu) * sl[h * S_ + s2];
#pragma unroll
        for (int o2 = 16; o2 >= 1; o2 >>= 1) Ls += __shfl_xor_sync(0xffffffffu, Ls, o2);
        if (lane == 0) { sML[2 * h] = M; sML[2 * h + 1] = Ls; }
    }
    __syncthreads();
    for (int idx = threadIdx.x; idx < G * S_; idx += kThreads) {
        const int h = idx / S_;
        const float M = sML[2 * h], Ls = sML[2 * h + 1];
        sml[idx] = (M == -INFINITY) ? 0.f : exp2_approx(sml[idx] - M) / Ls;
    }
    __syncthreads();
    T* out = reinterpret_cast<T*>(p.o);
    for (int idx = threadIdx.x; idx < G * D; idx += kThreads) {
        const int h = idx / D, d = idx % D;
        const float* po = p.part_o + (size_t(b) * Hq + h0 + h) * S_ * D + d;
        const float* w = sml + h * S_;
        float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
        int s2 = 0;
        for (; s2 + 4 <= S_; s2 += 4) {
            a0 = fmaf(w[s2 + 0], __ldcg(po + size_t(s2 + 0) * D), a0);
            a1 = fmaf(w[s2 + 1], __ldcg(po + size_t(s2 + 1) * D), a1);
            a2 = fmaf(w[s2 + 2], __ldcg(po + size_t(s2 + 2) * D), a2);
            a3 = fmaf(w[s2 + 3], __ldcg(po + size_t(s2 + 3) * D), a3);
        }
        for (; s2 < S_; ++s2) a0 = fmaf(w[s2], __ldcg(po + size_t(s2) * D), a0);
        out[(size_t(b) * Hq + h0 + h) * D + d] = Elem<T>::from_f((a0 + a1) + (a2 + a3));
        if (p.lse != nullptr && d == 0) p.lse[size_t(b) * Hq + h0 + h] = make_float2(sML[2 * h], sML[2 * h + 1]);
    }
}

}  // namespace delta

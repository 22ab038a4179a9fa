// Page-score + top-k selection kernel and the KV append kernel (included by delta_attn.cu only).
#pragma once

#include "common.cuh"

namespace delta {

// ------------------------------------------------------------------ score + select kernel
struct SelectParams {
    const int32_t* indptr;
    const int32_t* kv_len;
    const float2* page_ml;  // [B][Hq][max_pages]
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
    __shared__ uint32_t hist[512];   // radix histogram; first reused for per-head totals
    __shared__ int warp_sums[33];
    __shared__ uint32_t s_digit, s_above;

    const int b = blockIdx.x, tid = threadIdx.x;
    pdl_wait();
    pdl_trigger();
    int n = p.kv_len[b];
    const int npg = p.indptr[b + 1] - p.indptr[b];
    if (n < 0) n = 0;
    if (n > npg * kPage) n = max(npg, 0) * kPage;   // flagged by the decode kernel
    const int N = min((n + kPage - 1) / kPage, p.max_pages);
    const int Hq = p.num_q_heads;
    const int sinkP = (min(p.sink_tokens, n) + kPage - 1) / kPage;
    const int recStart = (p.recency_tokens > 0) ? max(n - p.recency_tokens, 0) / kPage : N;

    // 1. per-head totals over the page partials: M_h = max_j m_hj, Z_h = sum_j 2^(m_hj - M_h) l_hj
    //    (one warp per head, lanes stride over pages with an online max/sum, then a warp merge)
    float* headM = reinterpret_cast<float*>(hist);          // reuse: Hq <= 256 floats each
    float* headZ = headM + 256;
    const int warp = tid >> 5, lane = tid & 31;
    for (int h = warp; h < Hq; h += kSelectThreads / 32) {
        const float2* pm = p.page_ml + (size_t(b) * Hq + h) * p.max_pages;
        float M = -INFINITY, Z = 0.f;
        for (int j = lane; j < N; j += 32) {
            const float2 ml = pm[j];
            const float Mn = fmaxf(M, ml.x);
            Z = Z * exp2_approx(M - Mn) + ml.y * exp2_approx(ml.x - Mn);
            M = Mn;
        }
#pragma unroll
        for (int o = 16; o >= 1; o >>= 1) {
            const float Mo = __shfl_xor_sync(0xffffffffu, M, o), Zo = __shfl_xor_sync(0xffffffffu, Z, o);
            const float Mn = fmaxf(M, Mo);
            const float mu = (Mn == -INFINITY) ? 0.f : Mn;
            Z = Z * exp2_approx(M - mu) + Zo * exp2_approx(Mo - mu);
            M = Mn;
        }
        if (lane == 0) { headM[h] = M; headZ[h] = Z; }
    }
    __syncthreads();
    // 2. page scores S_j = sum_h 2^(m_hj - M_h) * l_hj / Z_h
    for (int j = tid; j < N; j += kSelectThreads) {
        float sc = 0.f;
        for (int h = 0; h < Hq; ++h) {
            const float2 ml = p.page_ml[(size_t(b) * Hq + h) * p.max_pages + j];
            sc += exp2_approx(ml.x - headM[h]) * ml.y / headZ[h];
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

// ------------------------------------------------------------------ kv append kernels
// Copy one token row (row_vecs 16-byte vectors) of KV head g of sequence b into slot
// (kv_len-1) % 16 of logical page (kv_len-1) / 16.  Out-of-range pages are skipped (the attention
// call that follows on the same page table flags them).
__device__ __forceinline__ void append_row(const uint4* __restrict__ k_new, const uint4* __restrict__ v_new,
                                           uint4* __restrict__ k_pool, uint4* __restrict__ v_pool,
                                           const int32_t* __restrict__ indptr, const int32_t* __restrict__ indices,
                                           const int32_t* __restrict__ kv_len, int Hkv, int row_vecs,
                                           int64_t num_phys_pages, int b, int g) {
    const int n = kv_len[b];
    if (n <= 0) return;
    const int pos = n - 1;
    const int lp = pos / kPage, slot = pos % kPage;
    const int pbeg = indptr[b], npg = indptr[b + 1] - pbeg;
    if (lp >= npg) return;
    const int64_t phys = indices[pbeg + lp];
    if (phys < 0 || phys >= num_phys_pages) return;
    const size_t src = (size_t(b) * Hkv + g) * row_vecs;
    const size_t dst = ((size_t(phys) * Hkv + g) * kPage + slot) * row_vecs;
    for (int i = threadIdx.x; i < row_vecs; i += blockDim.x) {
        k_pool[dst + i] = k_new[src + i];
        v_pool[dst + i] = v_new[src + i];
    }
}

__global__ void kv_append_kernel(const uint4* __restrict__ k_new, const uint4* __restrict__ v_new,
                                 uint4* __restrict__ k_pool, uint4* __restrict__ v_pool,
                                 const int32_t* __restrict__ indptr, const int32_t* __restrict__ indices,
                                 const int32_t* __restrict__ kv_len, int Hkv, int row_vecs,
                                 int64_t num_phys_pages) {
    pdl_wait();
    pdl_trigger();
    append_row(k_new, v_new, k_pool, v_pool, indptr, indices, kv_len, Hkv, row_vecs, num_phys_pages, blockIdx.x,
               blockIdx.y);
}

constexpr int kMaxAppendLayers = 64;
struct AppendLayers {
    const uint4* k_new[kMaxAppendLayers];
    const uint4* v_new[kMaxAppendLayers];
    uint4* k_pool[kMaxAppendLayers];
    uint4* v_pool[kMaxAppendLayers];
};

// Every layer of a decode step in one launch: grid (batch, KV heads, layers).
__global__ void kv_append_layers_kernel(const __grid_constant__ AppendLayers a, const int32_t* __restrict__ indptr,
                                        const int32_t* __restrict__ indices, const int32_t* __restrict__ kv_len,
                                        int Hkv, int row_vecs, int64_t num_phys_pages) {
    pdl_wait();
    pdl_trigger();
    const int l = blockIdx.z;
    append_row(a.k_new[l], a.v_new[l], a.k_pool[l], a.v_pool[l], indptr, indices, kv_len, Hkv, row_vecs,
               num_phys_pages, blockIdx.x, blockIdx.y);
}

}  // namespace delta

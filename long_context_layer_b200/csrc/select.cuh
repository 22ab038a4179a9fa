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
    const float* logits;   // [B][Hq][max_pages*16] base-2 logits: HEAD_MAX scoring when non-null
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

// Shared-memory plan of the selection cluster (dynamic): keys of this CTA's pages, per-head
// partial totals received from every CTA, double-buffered histograms received from every CTA.
struct SelectSmem {
    int chunk, C, Hq;
    __host__ __device__ size_t keys() const { return 0; }
    __host__ __device__ size_t mz() const { return (size_t(chunk) * 4 + 15) & ~size_t(15); }
    __host__ __device__ size_t hist() const { return mz() + size_t(C) * Hq * 8; }
    __host__ __device__ size_t counts() const { return hist() + size_t(2) * C * 256 * 4; }
    __host__ __device__ size_t bytes() const { return counts() + size_t(C) * 8; }
};

// One thread-block cluster per sequence; CTA r of C owns pages [r*chunk, (r+1)*chunk).
// 1. per-head totals over the page partials, M_h = max_j m_hj and Z_h = sum_j 2^(m_hj - M_h) l_hj
//    (each CTA over its pages, exchanged through distributed shared memory);
// 2. page scores S_j = sum_h 2^(m_hj - M_h) l_hj / Z_h -> order-preserving keys;
// 3. MSB-first 4 x 8-bit radix select of the k-th largest candidate key (histograms summed over
//    the cluster), candidates being the pages neither sink nor recency;
// 4. ascending compaction of sink U recency U {key > T} U {the first (k - #greater) keys == T in
//    page order} with cluster-wide offsets.
// Every exchange pushes into the other CTAs' shared memory and is followed by one cluster barrier,
// so no CTA reads remote memory after the last barrier.
__global__ void __launch_bounds__(kSelectThreads) score_select_kernel(const SelectParams p, int chunk) {
    namespace cg = cooperative_groups;
    cg::cluster_group cluster = cg::this_cluster();
    const int C = int(cluster.num_blocks()), rank = int(cluster.block_rank());
    auto cluster_barrier = [&]() {
        if (C > 1) cluster.sync();
        else __syncthreads();
    };
    extern __shared__ __align__(16) unsigned char sm[];
    const int Hq = p.num_q_heads;
    const SelectSmem L{chunk, C, Hq};
    uint32_t* keys = reinterpret_cast<uint32_t*>(sm + L.keys());
    float2* recv_mz = reinterpret_cast<float2*>(sm + L.mz());        // [C][Hq]
    uint32_t* recv_hist = reinterpret_cast<uint32_t*>(sm + L.hist());  // [2][C][256]
    int2* recv_cnt = reinterpret_cast<int2*>(sm + L.counts());         // [C]
    __shared__ float headM[kMaxQHeadsSelect], headZ[kMaxQHeadsSelect];
    __shared__ uint32_t hist[256];
    __shared__ int warp_sums[33];
    __shared__ uint32_t s_digit, s_above;

    const int b = blockIdx.y, tid = threadIdx.x;
    const int warp = tid >> 5, lane = tid & 31;
    pdl_wait();
    pdl_trigger();
    int n = p.kv_len[b];
    const int npg = p.indptr[b + 1] - p.indptr[b];
    if (n < 0) n = 0;
    if (n > npg * kPage) n = max(npg, 0) * kPage;   // flagged by the decode kernel
    const int N = min((n + kPage - 1) / kPage, p.max_pages);
    const int j0 = min(rank * chunk, N), j1 = min(j0 + chunk, N);   // this CTA's pages
    const int nloc = j1 - j0;
    const int sinkP = min((min(p.sink_tokens, n) + kPage - 1) / kPage, N);
    const int recStart = (p.recency_tokens > 0) ? min(max(n - p.recency_tokens, 0) / kPage, N) : N;
    auto forced = [&](int j) { return j < sinkP || j >= recStart; };
    const int ncand = max(recStart - sinkP, 0);
    const int k = p.budget_pages;
    const bool take_all = ncand <= k;

    // 1. per-head partial totals over this CTA's pages (a warp per head), pushed to every CTA
    for (int h = warp; h < Hq; h += kSelectThreads / 32) {
        const float2* pm = p.page_ml + (size_t(b) * Hq + h) * p.max_pages;
        float M = -INFINITY, Z = 0.f;
        // sixteen independent loads in flight per lane, then an online (max, sum) update
        for (int base = j0; base < j1; base += 32 * 16) {
            float2 v[16];
#pragma unroll
            for (int u = 0; u < 16; ++u) {
                const int j = base + lane + 32 * u;
                v[u] = (j < j1) ? pm[j] : make_float2(-INFINITY, 0.f);
            }
#pragma unroll
            for (int u = 0; u < 16; ++u) {
                const float Mn = fmaxf(M, v[u].x);
                const float mu = (Mn == -INFINITY) ? 0.f : Mn;
                Z = Z * exp2_approx(M - mu) + v[u].y * exp2_approx(v[u].x - mu);
                M = Mn;
            }
        }
#pragma unroll
        for (int o = 16; o >= 1; o >>= 1) {
            const float Mo = __shfl_xor_sync(0xffffffffu, M, o), Zo = __shfl_xor_sync(0xffffffffu, Z, o);
            const float Mn = fmaxf(M, Mo);
            const float mu = (Mn == -INFINITY) ? 0.f : Mn;
            Z = Z * exp2_approx(M - mu) + Zo * exp2_approx(Mo - mu);
            M = Mn;
        }
        if (lane < C) cluster.map_shared_rank(recv_mz, lane)[rank * Hq + h] = make_float2(M, Z);
    }
    cluster_barrier();
    for (int h = tid; h < Hq; h += kSelectThreads) {
        float M = -INFINITY, Z = 0.f;
        for (int j = 0; j < C; ++j) {
            const float2 v = recv_mz[j * Hq + h];
            const float Mn = fmaxf(M, v.x);
            const float mu = (Mn == -INFINITY) ? 0.f : Mn;
            Z = Z * exp2_approx(M - mu) + v.y * exp2_approx(v.x - mu);
            M = Mn;
        }
        headM[h] = M;
        headZ[h] = 1.f / Z;   // stored as the reciprocal: the score pass multiplies
    }
    __syncthreads();

    // 2. page scores of this CTA's pages
    if (p.logits != nullptr) {
        // HEAD_MAX: S_j = sum over the page's tokens t < n of max_h 2^(s_ht - M_h) / Z_h.  A warp per
        // page, lanes over heads, each lane holding the page's 16 token maxima of its heads.
        const size_t hs = size_t(p.max_pages) * kPage;
        for (int j = j0 + warp; j < j1; j += kSelectThreads / 32) {
            float mx[kPage];
#pragma unroll
            for (int t = 0; t < kPage; ++t) mx[t] = 0.f;
            for (int h = lane; h < Hq; h += 32) {
                const float4* lg = reinterpret_cast<const float4*>(p.logits + (size_t(b) * Hq + h) * hs + size_t(j) * kPage);
                const float inv = headZ[h];
#pragma unroll
                for (int q4 = 0; q4 < kPage / 4; ++q4) {
                    const float4 v = lg[q4];
                    mx[4 * q4 + 0] = fmaxf(mx[4 * q4 + 0], exp2_approx(v.x - headM[h]) * inv);
                    mx[4 * q4 + 1] = fmaxf(mx[4 * q4 + 1], exp2_approx(v.y - headM[h]) * inv);
                    mx[4 * q4 + 2] = fmaxf(mx[4 * q4 + 2], exp2_approx(v.z - headM[h]) * inv);
                    mx[4 * q4 + 3] = fmaxf(mx[4 * q4 + 3], exp2_approx(v.w - headM[h]) * inv);
                }
            }
            float sc = 0.f;
#pragma unroll
            for (int t = 0; t < kPage; ++t) {
                float v = mx[t];
#pragma unroll
                for (int o = 16; o >= 1; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
                if (j * kPage + t < n) sc += v;
            }
            if (lane == 0) {
                keys[j - j0] = order_key(sc);
                if (p.page_scores != nullptr) p.page_scores[size_t(b) * p.max_pages + j] = sc;
            }
        }
    } else {
        // HEAD_SUM: two threads per page, each summing every other head with up to sixteen
        // independent loads in flight, so a page's partials arrive in one round
        const int sub = tid & 1;
        for (int base = j0; base < j1; base += kSelectThreads / 2) {   // uniform trip count
            const int j = base + (tid >> 1);
            const bool active = j < j1;
            const float2* pm = p.page_ml + size_t(b) * Hq * p.max_pages + (active ? j : j0);
            float sc = 0.f;
            for (int hb = 0; hb < Hq; hb += 32) {
                float2 v[16];
#pragma unroll
                for (int u = 0; u < 16; ++u) {
                    const int h = hb + sub + 2 * u;
                    v[u] = (active && h < Hq) ? pm[size_t(h) * p.max_pages] : make_float2(-INFINITY, 0.f);
                }
#pragma unroll
                for (int u = 0; u < 16; ++u) {
                    const int h = hb + sub + 2 * u;
                    if (h < Hq) sc += exp2_approx(v[u].x - headM[h]) * v[u].y * headZ[h];
                }
            }
            sc += __shfl_xor_sync(0xffffffffu, sc, 1);
            if (active && sub == 0) {
                keys[j - j0] = order_key(sc);
                if (p.page_scores != nullptr) p.page_scores[size_t(b) * p.max_pages + j] = sc;
            }
        }
    }
    __syncthreads();

    // 3. radix select of the k-th largest candidate key over the whole cluster
    uint32_t T = 0, need_eq = 0;
    if (!take_all && k > 0) {
        uint32_t prefix = 0, mask = 0, kk = k;
        for (int pass = 0, shift = 24; shift >= 0; ++pass, shift -= 8) {
            for (int i = tid; i < 256; i += kSelectThreads) hist[i] = 0;
            __syncthreads();
            for (int j = j0 + tid; j < j1; j += kSelectThreads) {
                const uint32_t key = keys[j - j0];
                if (!forced(j) && (key & mask) == prefix) atomicAdd(&hist[(key >> shift) & 255u], 1u);
            }
            __syncthreads();
            if (C > 1) {   // sum the histograms of the cluster (one CTA: already the total)
                uint32_t* rh = recv_hist + (pass & 1) * C * 256;
                for (int i = tid; i < C * 256; i += kSelectThreads) {
                    const int j = i >> 8, bin = i & 255;
                    cluster.map_shared_rank(rh, j)[rank * 256 + bin] = hist[bin];
                }
                cluster_barrier();
                if (tid < 256) {
                    uint32_t t = 0;
                    for (int j = 0; j < C; ++j) t += rh[j * 256 + tid];
                    hist[tid] = t;
                }
                __syncthreads();
            }
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
        need_eq = kk;   // how many of the keys equal to T are taken (lowest page indices first)
    }

    // 4. cluster-wide offsets, then the ascending compaction of this CTA's pages
    const int per = (nloc + kSelectThreads - 1) / kSelectThreads;
    const int jb = j0 + tid * per, je = min(jb + per, j1);
    const bool radix = !take_all && k > 0;
    int eq_cnt = 0, gtf_cnt = 0;
    for (int j = jb; j < je; ++j) {
        if (forced(j)) { ++gtf_cnt; continue; }
        if (take_all) { ++gtf_cnt; continue; }
        if (!radix) continue;
        const uint32_t key = keys[j - j0];
        if (key > T) ++gtf_cnt;
        else if (key == T) ++eq_cnt;
    }
    int eq_tot_loc, gtf_tot_loc;
    const int eq_rank_loc = block_exclusive_scan(eq_cnt, warp_sums, eq_tot_loc);
    block_exclusive_scan(gtf_cnt, warp_sums, gtf_tot_loc);
    if (tid < C) cluster.map_shared_rank(recv_cnt, tid)[rank] = make_int2(eq_tot_loc, gtf_tot_loc);
    cluster_barrier();
    int eq_cum = 0, eq_before = 0, sel_before = 0, total = 0;
    for (int j = 0; j < C; ++j) {
        const int2 v = recv_cnt[j];
        const int taken = min(max(int(need_eq) - eq_cum, 0), v.x);   // T-valued pages of CTA j that are kept
        if (j < rank) {
            sel_before += v.y + taken;
            eq_before += v.x;
        }
        total += v.y + taken;
        eq_cum += v.x;
    }
    auto selected = [&](int j, int& eq_seen) -> bool {
        if (forced(j) || take_all) return true;
        if (!radix) return false;
        const uint32_t key = keys[j - j0];
        if (key > T) return true;
        if (key == T) return uint32_t(eq_before + eq_rank_loc + eq_seen++) < need_eq;
        return false;
    };
    int cnt = 0, seen = 0;
    for (int j = jb; j < je; ++j) cnt += selected(j, seen) ? 1 : 0;
    int local_total;
    int pos = sel_before + block_exclusive_scan(cnt, warp_sums, local_total);
    seen = 0;
    for (int j = jb; j < je; ++j) {
        if (selected(j, seen)) {
            if (pos < p.sel_stride) p.sel_pages[size_t(b) * p.sel_stride + pos] = j;
            ++pos;
        }
    }
    if (rank == 0 && tid == 0) p.sel_cnt[b] = min(total, p.sel_stride);
}

// ------------------------------------------------------------------ layer-shift metric
// 1 - cos(S_a[b], S_b[b]) over the pages j < ceil(kv_len[b]/16) of two layers' page scores, one
// CTA per sequence (fixed-order reduction: deterministic).  A zero vector gives 1.
constexpr int kShiftThreads = 256;
__global__ void __launch_bounds__(kShiftThreads) layer_shift_kernel(const float* __restrict__ sa,
                                                                  const float* __restrict__ sb,
                                                                  const int32_t* __restrict__ indptr,
                                                                  const int32_t* __restrict__ kv_len, int max_pages,
                                                                  float* __restrict__ out) {
    __shared__ float red[3][kShiftThreads / 32];
    pdl_wait();
    pdl_trigger();
    const int b = blockIdx.x, tid = threadIdx.x;
    int n = kv_len[b];
    const int npg = indptr[b + 1] - indptr[b];
    n = min(max(n, 0), max(npg, 0) * kPage);
    const int N = min((n + kPage - 1) / kPage, max_pages);
    float ab = 0.f, aa = 0.f, bb = 0.f;
    for (int j = tid; j < N; j += kShiftThreads) {
        const float x = sa[size_t(b) * max_pages + j], y = sb[size_t(b) * max_pages + j];
        ab = fmaf(x, y, ab);
        aa = fmaf(x, x, aa);
        bb = fmaf(y, y, bb);
    }
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) {
        ab += __shfl_xor_sync(0xffffffffu, ab, o);
        aa += __shfl_xor_sync(0xffffffffu, aa, o);
        bb += __shfl_xor_sync(0xffffffffu, bb, o);
    }
    if ((tid & 31) == 0) { red[0][tid >> 5] = ab; red[1][tid >> 5] = aa; red[2][tid >> 5] = bb; }
    __syncthreads();
    if (tid == 0) {
        float s0 = 0.f, s1 = 0.f, s2 = 0.f;
        for (int w = 0; w < kShiftThreads / 32; ++w) { s0 += red[0][w]; s1 += red[1][w]; s2 += red[2][w]; }
        out[b] = (s1 > 0.f && s2 > 0.f) ? 1.f - s0 / (sqrtf(s1) * sqrtf(s2)) : 1.f;
    }
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

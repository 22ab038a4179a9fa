// Page-score + top-k selection kernel and the KV append kernel (included by delta_attn.cu only).
#pragma once

#include "common.cuh"

namespace delta {

// ------------------------------------------------------------------ score + select kernel
struct SelectParams {
    const int32_t* indptr;
    const int32_t* kv_len;
    const float* page_lse;   // [B][Hq][max_pages] log2-sum-exp of each page's base-2 logits
    const float2* split_ml;  // [B][Hq][num_splits] (max, sum) of each decode split
    int32_t num_splits;
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
    return res;   // warp_sums is not written again: no trailing barrier
}

// Shared-memory plan of the selection cluster (dynamic): keys of this CTA's pages, the keys of the
// threshold bucket (one-CTA path), double-buffered histograms and the compaction counts received
// from every CTA.
struct SelectSmem {
    int chunk, C;
    __host__ __device__ size_t keys() const { return 0; }
    __host__ __device__ size_t list() const { return (size_t(chunk) * 4 + 15) & ~size_t(15); }
    __host__ __device__ size_t hist() const { return list() + ((size_t(chunk) * 4 + 15) & ~size_t(15)); }
    __host__ __device__ size_t counts() const { return hist() + size_t(2) * C * 256 * 4; }
    __host__ __device__ size_t bytes() const { return counts() + size_t(C) * 8; }
};

// One thread-block cluster per sequence; CTA r of C owns pages [r*chunk, (r+1)*chunk).
// 1. per-head normalisers c_h = log2 sum_j 2^(lse_hj), combined from the decode splits' (max, sum)
//    states (a few per head, so every CTA does all heads and nothing is exchanged);
// 2. page scores S_j = sum_h 2^(lse_hj - c_h) -> order-preserving keys;
// 3. the k-th largest candidate key T (candidates: pages neither sink nor recency).  One CTA:
//    a 256-bucket histogram over [min, max] of the keys, then the exact rank inside the bucket
//    holding the k-th; a cluster: MSB-first 4 x 8-bit radix select with histograms summed over
//    the cluster;
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
    const SelectSmem L{chunk, C};
    uint32_t* keys = reinterpret_cast<uint32_t*>(sm + L.keys());
    uint32_t* blist = reinterpret_cast<uint32_t*>(sm + L.list());
    uint32_t* recv_hist = reinterpret_cast<uint32_t*>(sm + L.hist());  // [2][C][256]
    int2* recv_cnt = reinterpret_cast<int2*>(sm + L.counts());         // [C]
    __shared__ float headC[kMaxQHeadsSelect];
    __shared__ uint32_t hist[2][256];
    __shared__ int warp_sums[33];
    __shared__ uint32_t s_digit[2], s_above[2];
    __shared__ uint32_t s_kmin[32], s_kmax[32], s_T, s_need;
    __shared__ int s_m;

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

    const int sub = tid & 1;

    // 1. per-head normaliser from the splits' states, a warp per head: the maximum first, then the
    //    rescaled sum, so the exponentials are independent (no serial online update); four states
    //    per lane and round, no exponential for an empty slot
    for (int h = warp; h < Hq; h += kSelectThreads / 32) {
        const float2* ps = p.split_ml + (size_t(b) * Hq + h) * p.num_splits;
        float M = -INFINITY, Z = 0.f;
        for (int base = 0; base < p.num_splits; base += 32 * 4) {
            float2 v[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const int s = base + lane + 32 * u;
                v[u] = (s < p.num_splits) ? ps[s] : make_float2(-INFINITY, 0.f);
            }
            float Mr = fmaxf(fmaxf(v[0].x, v[1].x), fmaxf(v[2].x, v[3].x));
#pragma unroll
            for (int o = 16; o >= 1; o >>= 1) Mr = fmaxf(Mr, __shfl_xor_sync(0xffffffffu, Mr, o));
            const float Mn = fmaxf(M, Mr);
            const float mu = (Mn == -INFINITY) ? 0.f : Mn;
            float z = 0.f;
#pragma unroll
            for (int u = 0; u < 4; ++u)
                if (v[u].y > 0.f) z = fmaf(v[u].y, exp2_approx(v[u].x - mu), z);
#pragma unroll
            for (int o = 16; o >= 1; o >>= 1) z += __shfl_xor_sync(0xffffffffu, z, o);
            Z = Z * exp2_approx(M - mu) + z;
            M = Mn;
        }
        // no token of the head: every page term is 2^(-inf) = 0
        if (lane == 0) headC[h] = (Z > 0.f) ? M + log2_approx(Z) : INFINITY;
    }
    if (tid < 256) hist[0][tid] = 0;
    __syncthreads();

    // 2. page scores of this CTA's pages
    uint32_t kmin_loc = 0xffffffffu, kmax_loc = 0u;
    auto put_key = [&](int j, float sc) {
        const uint32_t key = order_key(sc);
        keys[j - j0] = key;
        if (!forced(j)) {
            kmin_loc = min(kmin_loc, key);
            kmax_loc = max(kmax_loc, key);
        }
        if (p.page_scores != nullptr) p.page_scores[size_t(b) * p.max_pages + j] = sc;
    };
    if (p.logits != nullptr) {
        // HEAD_MAX: S_j = sum over the page's tokens t < n of max_h 2^(s_ht - c_h).  A warp per
        // page, lanes over heads, each lane holding the page's 16 token maxima of its heads.
        const size_t hs = size_t(p.max_pages) * kPage;
        for (int j = j0 + warp; j < j1; j += kSelectThreads / 32) {
            float mx[kPage];
#pragma unroll
            for (int t = 0; t < kPage; ++t) mx[t] = 0.f;
            for (int h = lane; h < Hq; h += 32) {
                const float4* lg = reinterpret_cast<const float4*>(p.logits + (size_t(b) * Hq + h) * hs + size_t(j) * kPage);
                const float c = headC[h];
#pragma unroll
                for (int q4 = 0; q4 < kPage / 4; ++q4) {
                    const float4 v = lg[q4];
                    mx[4 * q4 + 0] = fmaxf(mx[4 * q4 + 0], exp2_approx(v.x - c));
                    mx[4 * q4 + 1] = fmaxf(mx[4 * q4 + 1], exp2_approx(v.y - c));
                    mx[4 * q4 + 2] = fmaxf(mx[4 * q4 + 2], exp2_approx(v.z - c));
                    mx[4 * q4 + 3] = fmaxf(mx[4 * q4 + 3], exp2_approx(v.w - c));
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
            if (lane == 0) put_key(j, sc);
        }
    } else {
        // HEAD_SUM: two threads per page, each summing every other head with up to sixteen
        // independent loads in flight, so a page's terms arrive in one round
        for (int base = j0; base < j1; base += kSelectThreads / 2) {   // uniform trip count
            const int j = base + (tid >> 1);
            const bool active = j < j1;
            const float* pl = p.page_lse + size_t(b) * Hq * p.max_pages + (active ? j : j0);
            float sc = 0.f;
            for (int hb = 0; hb < Hq; hb += 32) {
                float v[16];
#pragma unroll
                for (int u = 0; u < 16; ++u) {
                    const int h = hb + sub + 2 * u;
                    v[u] = (active && h < Hq) ? pl[size_t(h) * p.max_pages] : -INFINITY;
                }
#pragma unroll
                for (int u = 0; u < 16; ++u) {
                    const int h = hb + sub + 2 * u;
                    if (h < Hq) sc += exp2_approx(v[u] - headC[h]);
                }
            }
            sc += __shfl_xor_sync(0xffffffffu, sc, 1);
            if (active && sub == 0) put_key(j, sc);
        }
    }
    // range of the candidate keys (the one-CTA threshold search buckets it), per warp here and
    // over the CTA after the barrier
    kmin_loc = __reduce_min_sync(0xffffffffu, kmin_loc);
    kmax_loc = __reduce_max_sync(0xffffffffu, kmax_loc);
    if (lane == 0) {
        s_kmin[warp] = kmin_loc;
        s_kmax[warp] = kmax_loc;
    }
    if (tid == 0) s_m = 0;
    __syncthreads();

    // 3. radix select of the k-th largest candidate key over the whole cluster.  Histograms and
    //    the chosen digit are double-buffered, so a pass needs two block barriers.
    uint32_t T = 0, need_eq = 0;
    if (!take_all && k > 0 && C == 1) {
        // one CTA: bucket b(key) = (key - kmin) >> sh in [0, 255] (monotone in the key)
        // every warp combines the 32 per-warp values itself: one load per lane, not 64 per thread
        const uint32_t kmin = __reduce_min_sync(0xffffffffu, s_kmin[lane]);
        const uint32_t kmax = __reduce_max_sync(0xffffffffu, s_kmax[lane]);
        const uint32_t span = kmax - kmin;   // ncand > k >= 1 candidates: kmin <= kmax
        const int sh = max(0, 24 - __clz(span));
        for (int j = j0 + tid; j < j1; j += kSelectThreads)
            if (!forced(j)) atomicAdd(&hist[0][(keys[j - j0] - kmin) >> sh], 1u);
        __syncthreads();
        if (tid < 32) {   // the bucket holding the k-th largest, and the keys in higher buckets
            uint32_t c[8], sum = 0;
#pragma unroll
            for (int i = 0; i < 8; ++i) { c[i] = hist[0][255 - 8 * tid - i]; sum += c[i]; }
            uint32_t incl = sum;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const uint32_t y = __shfl_up_sync(0xffffffffu, incl, o);
                if (tid >= o) incl += y;
            }
            const uint32_t excl = incl - sum;
            if (excl < uint32_t(k) && uint32_t(k) <= incl) {
                uint32_t above = excl;
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    if (above + c[i] >= uint32_t(k)) { s_digit[0] = 255 - 8 * tid - i; s_above[0] = above; break; }
                    above += c[i];
                }
            }
        }
        __syncthreads();
        const uint32_t tb = s_digit[0];
        const int kk = k - int(s_above[0]);   // rank of T inside its bucket, 1-based
        // gather the bucket's keys (warp-aggregated slots; uniform trip count for the ballot)
        for (int base = j0; base < j1; base += kSelectThreads) {
            const int j = base + tid;
            const bool in = j < j1 && !forced(j) && ((keys[j - j0] - kmin) >> sh) == tb;
            const uint32_t bal = __ballot_sync(0xffffffffu, in);
            int slot = 0;
            if (lane == 0 && bal != 0u) slot = atomicAdd(&s_m, __popc(bal));
            slot = __shfl_sync(0xffffffffu, slot, 0);
            if (in) blist[slot + __popc(bal & ((1u << lane) - 1u))] = keys[j - j0];
        }
        __syncthreads();
        // T = the key v of the bucket with #(> v) < kk <= #(>= v); every holder of v writes the same
        const int m = s_m;
        for (int i = tid; i < m; i += kSelectThreads) {
            const uint32_t v = blist[i];
            int gt = 0, ge = 0;
            for (int t = 0; t < m; ++t) {
                const uint32_t w = blist[t];
                gt += w > v ? 1 : 0;
                ge += w >= v ? 1 : 0;
            }
            if (gt < kk && kk <= ge) {
                s_T = v;
                s_need = uint32_t(kk - gt);
            }
        }
        __syncthreads();
        T = s_T;
        need_eq = s_need;   // how many of the keys equal to T are taken (lowest page indices first)
    } else if (!take_all && k > 0) {
        uint32_t prefix = 0, mask = 0, kk = k;
        for (int pass = 0, shift = 24; shift >= 0; ++pass, shift -= 8) {
            const int cur = pass & 1;
            // warp-aggregated: the leading digits of most keys agree, so lanes with equal digits
            // add once (uniform trip count for the warp-wide match)
            for (int base = j0; base < j1; base += kSelectThreads) {
                const int j = base + tid;
                uint32_t dig = 0xffffffffu;
                if (j < j1 && !forced(j)) {
                    const uint32_t key = keys[j - j0];
                    if ((key & mask) == prefix) dig = (key >> shift) & 255u;
                }
                const uint32_t peers = __match_any_sync(0xffffffffu, dig);
                if (dig != 0xffffffffu && lane == __ffs(peers) - 1) atomicAdd(&hist[cur][dig], uint32_t(__popc(peers)));
            }
            if (tid < 256) hist[cur ^ 1][tid] = 0;   // the next pass's buffer (last read two barriers ago)
            __syncthreads();
            if (C > 1) {   // sum the histograms of the cluster (one CTA: already the total)
                uint32_t* rh = recv_hist + cur * C * 256;
                for (int i = tid; i < C * 256; i += kSelectThreads) {
                    const int j = i >> 8, bin = i & 255;
                    cluster.map_shared_rank(rh, j)[rank * 256 + bin] = hist[cur][bin];
                }
                cluster_barrier();
                if (tid < 256) {
                    uint32_t t = 0;
                    for (int j = 0; j < C; ++j) t += rh[j * 256 + tid];
                    hist[cur][tid] = t;
                }
                __syncthreads();
            }
            if (tid < 32) {
                // lane covers digits 255-8*lane .. 248-8*lane (descending)
                uint32_t c[8], sum = 0;
#pragma unroll
                for (int i = 0; i < 8; ++i) { c[i] = hist[cur][255 - 8 * tid - i]; sum += c[i]; }
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
                        if (above + c[i] >= kk) { s_digit[cur] = 255 - 8 * tid - i; s_above[cur] = above; break; }
                        above += c[i];
                    }
                }
            }
            __syncthreads();
            prefix |= s_digit[cur] << shift;
            mask |= 0xffu << shift;
            kk -= s_above[cur];
        }
        T = prefix;
        need_eq = kk;   // how many of the keys equal to T are taken (lowest page indices first)
    }

    // 4. cluster-wide offsets, then the ascending compaction of this CTA's pages.  Pages equal to T
    //    are taken in page order, so the taken ones before a thread follow from the equal ones
    //    before it: one (packed) scan gives every thread its output position.
    const int per = (nloc + kSelectThreads - 1) / kSelectThreads;
    const int jb = j0 + tid * per, je = min(jb + per, j1);
    const bool radix = !take_all && k > 0;
    int eq_cnt = 0, gtf_cnt = 0;
    for (int j = jb; j < je; ++j) {
        if (forced(j) || take_all) { ++gtf_cnt; continue; }
        if (!radix) continue;
        const uint32_t key = keys[j - j0];
        if (key > T) ++gtf_cnt;
        else if (key == T) ++eq_cnt;
    }
    int tot_loc;   // both counts fit 15 bits: a CTA owns at most 16384 pages
    const int packed = block_exclusive_scan(eq_cnt | (gtf_cnt << 16), warp_sums, tot_loc);
    const int eq_rank_loc = packed & 0xffff, gtf_rank_loc = packed >> 16;
    const int eq_tot_loc = tot_loc & 0xffff, gtf_tot_loc = tot_loc >> 16;
    int eq_cum = 0, eq_before = 0, sel_before = 0, total = 0;
    if (C == 1) {   // one CTA: its own totals
        total = gtf_tot_loc + min(int(need_eq), eq_tot_loc);
    } else {
        if (tid < C) cluster.map_shared_rank(recv_cnt, tid)[rank] = make_int2(eq_tot_loc, gtf_tot_loc);
        cluster_barrier();
    }
    for (int j = 0; j < C && C > 1; ++j) {
        const int2 v = recv_cnt[j];
        const int taken = min(max(int(need_eq) - eq_cum, 0), v.x);   // T-valued pages of CTA j that are kept
        if (j < rank) {
            sel_before += v.y + taken;
            eq_before += v.x;
        }
        total += v.y + taken;
        eq_cum += v.x;
    }
    const int eq_left = max(int(need_eq) - eq_before, 0);            // T-valued pages this CTA may still take
    int pos = sel_before + gtf_rank_loc + min(eq_left, eq_rank_loc);
    int eq_seen = eq_rank_loc;
    for (int j = jb; j < je; ++j) {
        bool take;
        if (forced(j) || take_all) {
            take = true;
        } else if (!radix) {
            take = false;
        } else {
            const uint32_t key = keys[j - j0];
            take = key > T || (key == T && eq_seen++ < eq_left);
        }
        if (take) {
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

// Page scoring and selection at the end of the delta-layer decode kernel (HEAD_SUM scoring;
// included by the decode kernels only).
//
// DELTA's delta-layers rank the KV pages by the attention they receive and keep the sink pages,
// the recency window and the best-scoring remaining pages ("DELTA: Dynamic Layer-Aware Token
// Attention", ai.info summary, "Methodology in Plain English" and "Main Findings" bullet 5).
// The score of page j is S_j = sum over query heads h of sum over the page's tokens of p[h][t]
// = sum_h 2^(lse_hj - c_h), with lse_hj the log2-sum-exp of head h's base-2 logits on page j
// (written by the decode loop) and c_h that head's log2-sum-exp over the whole context.
//
// No CTA waits for another.  Delta-layer plans keep each (sequence, KV head) unit in one cluster,
// so the output merge has already given every CTA every split's state of the unit's heads: each CTA
// forms c_h itself and adds its own pages' share of the scores (the sum over the unit's G heads)
// into per-page 2^-55 fixed-point accumulators with integer atomics (integer addition is
// associative, so the sums do not depend on the order of arrival), then takes one ticket on its
// sequence.  The last CTA of the sequence reads the sums, finds the k-th largest candidate score by
// an adaptive-range radix select and writes the ascending selection.
#pragma once

#include "common.cuh"

namespace delta {

constexpr int kTailList = 128;              // keys the final rank step compares pairwise, at most
// Fixed-point unit of the score accumulators: 2^-55.  A page score is at most H_q <= 256 = 2^8
// (delta-layers are limited to 256 query heads), so every sum stays below 2^63; scores resolve down
// to 2^-55 (about 2.8e-17), below which a page scores 0 and ties go to the lower page index.
constexpr float kFixScale = 36028797018963968.f;   // 2^55
constexpr float kFixInv = 2.7755575615628914e-17f;  // 2^-55

// What the sequence's last CTA needs (passed by value to the non-inlined final stage).
struct SelectFinal {
    unsigned long long* score_acc;   // [B][max_pages]
    uint32_t* keys;                  // [B][max_pages]
    float* page_scores;              // [B][max_pages] or null
    int32_t* sel_cnt;
    int32_t* sel_pages;
    int32_t sel_stride, max_pages, budget_pages, sink_tokens, recency_tokens;
};

// Takes a ticket on `counter`; true in every thread of the CTA that arrives `expected`-th (which
// also resets the counter for the next launch).  The CTA's earlier global writes and reductions
// are visible to that CTA first: the block barrier orders every thread's accesses before thread
// 0's fence and atomic, and the last CTA's thread 0 fences again before the barrier that releases
// its threads.
__device__ __forceinline__ bool arrive_last(int* counter, int expected, uint32_t* s_flag) {
    __syncthreads();
    if (threadIdx.x == 0) {
        __threadfence();
        const int t = atomicAdd(counter, 1);
        const uint32_t last = (t == expected - 1) ? 1u : 0u;
        if (last) {
            *counter = 0;
            __threadfence();
        }
        *s_flag = last;
    }
    __syncthreads();
    return *s_flag != 0u;
}

// Delta-layers, one cluster per unit: this CTA's page terms lse_hj for its first 2 NTHR pages,
// loaded right after the loop (its warps wrote them before the preceding block barrier) so that
// their latency overlaps the output merge.
template <int NTHR, int G>
__device__ __forceinline__ void select_preload(const DecodeParams& p, int b, int g, int N, float (&pre)[2][G]) {
    const size_t maxp = size_t(p.max_pages);
    const float* pl = p.page_lse + (size_t(b) * p.num_q_heads + g * G) * maxp;
    const int i0 = blockIdx.x * p.items_per_split, i1 = min(i0 + p.items_per_split, N);
#pragma unroll
    for (int i = 0; i < 2; ++i)
#pragma unroll
        for (int h = 0; h < G; ++h) {
            const int j = i0 + int(threadIdx.x) + i * NTHR;
            pre[i][h] = (j < i1) ? pl[size_t(h) * maxp + j] : -INFINITY;
        }
}

// Steps of the sequence's last CTA: page scores and their order keys, the threshold key T and the
// number of keys equal to T to take, then the ascending compaction.  smem: free_bytes of idle
// shared memory (16-byte aligned).
template <int NTHR>
__device__ __noinline__ void select_final(const SelectFinal a, unsigned char* smem, size_t free_bytes, int b, int n,
                                          int N) {
    constexpr int W = NTHR / 32;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const size_t maxp = size_t(a.max_pages);
    uint32_t* hist = reinterpret_cast<uint32_t*>(smem);      // [W][256] one histogram per warp
    uint32_t* list = hist + W * 256;                          // [kTailList]
    uint32_t* s_u = list + kTailList;                         // [8] broadcasts
    uint32_t* s_wmin = s_u + 8;                               // [W]
    uint32_t* s_wmax = s_wmin + W;                            // [W]
    uint32_t* s_wt = s_wmax + W;                              // [W] taken pages per warp segment
    uint32_t* s_we = s_wt + W;                                // [W] pages equal to T per warp segment
    constexpr size_t kScratch = ((W * 256 + kTailList + 8 + 4 * W) * 4 + 15) & ~size_t(15);
    const int key_cap = int((free_bytes - kScratch) / 4);
    uint32_t* keys = (N <= key_cap) ? reinterpret_cast<uint32_t*>(smem + kScratch) : a.keys + size_t(b) * maxp;

    // 1. page scores from the accumulators (which go back to zero for the next launch), order keys,
    //    candidate key range (candidates: pages neither sink nor recency); sixteen loads in flight
    const int sinkP = min((min(a.sink_tokens, n) + kPage - 1) / kPage, N);
    const int recStart = (a.recency_tokens > 0) ? min(max(n - a.recency_tokens, 0) / kPage, N) : N;
    const int k = a.budget_pages;
    const bool take_all = max(recStart - sinkP, 0) <= k;
    const bool radix = !take_all && k > 0;
    unsigned long long* acc = a.score_acc + size_t(b) * maxp;
    uint32_t kmin = 0xffffffffu, kmax = 0u;
    for (int jb = tid; jb < N; jb += 16 * NTHR) {
        unsigned long long v[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            const int j = jb + i * NTHR;
            v[i] = (j < N) ? __ldcg(acc + j) : 0ull;
        }
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            const int j = jb + i * NTHR;
            if (j >= N) break;   // small contexts: most slots are empty
            acc[j] = 0ull;
            const float sc = __ull2float_rn(v[i]) * kFixInv;
            if (a.page_scores != nullptr) a.page_scores[size_t(b) * maxp + j] = sc;
            const uint32_t key = order_key(sc);
            keys[j] = key;
            if (j >= sinkP && j < recStart) {
                kmin = min(kmin, key);
                kmax = max(kmax, key);
            }
        }
    }
    kmin = __reduce_min_sync(0xffffffffu, kmin);
    kmax = __reduce_max_sync(0xffffffffu, kmax);
    if (lane == 0) {
        s_wmin[warp] = kmin;
        s_wmax[warp] = kmax;
    }
    __syncthreads();

    // 2. threshold T and the number of keys equal to T to take (lowest page index first).  Each
    //    pass buckets the keys of [lo, lo + span] into 256 buckets of width 2^sh, finds the bucket
    //    holding the kk-th largest and narrows the range to it (span shrinks by 2^8 a pass, so at
    //    most four passes); once the bucket holds at most kTailList keys they are ranked exactly.
    uint32_t T = 0, need = 0;
    if (radix) {
        uint32_t lo = 0xffffffffu, hi = 0u;
        for (int w = 0; w < W; ++w) {
            lo = min(lo, s_wmin[w]);
            hi = max(hi, s_wmax[w]);
        }
        uint32_t span = hi - lo;   // more than k >= 1 candidates: lo <= hi
        uint32_t kk = uint32_t(k);
        bool exact = false;
        for (;;) {
            const int sh = max(0, 24 - __clz(span));   // (span >> sh) <= 255
            for (int i = tid; i < W * 256; i += NTHR) hist[i] = 0u;
            __syncthreads();
            // per-warp histograms: same-bucket atomics contend only inside a warp; eight keys per thread
            // are loaded before their atomics so the loads overlap
            for (int j0 = sinkP + tid; j0 < recStart; j0 += 8 * NTHR) {
                uint32_t kv[8];
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    const int j = j0 + i * NTHR;
                    kv[i] = (j < recStart) ? keys[j] : 0u;
                }
#pragma unroll
                for (int i = 0; i < 8; ++i)
                    if (j0 + i * NTHR < recStart && kv[i] >= lo && kv[i] - lo <= span)
                        atomicAdd(&hist[warp * 256 + ((kv[i] - lo) >> sh)], 1u);
            }
            __syncthreads();
            for (int i = tid; i < 256; i += NTHR) {
                uint32_t c = 0;
                for (int w = 0; w < W; ++w) c += hist[w * 256 + i];
                hist[i] = c;   // warp 0's row becomes the total (each thread only reads its own column)
            }
            __syncthreads();
            if (warp == 0) {   // lane covers buckets 255-8*lane .. 248-8*lane (descending)
                uint32_t c[8], sum = 0;
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    c[i] = hist[255 - 8 * lane - i];
                    sum += c[i];
                }
                uint32_t incl = sum;
#pragma unroll
                for (int o = 1; o < 32; o <<= 1) {
                    const uint32_t y = __shfl_up_sync(0xffffffffu, incl, o);
                    if (lane >= o) incl += y;
                }
                const uint32_t excl = incl - sum;
                if (excl < kk && kk <= incl) {
                    uint32_t above = excl;
#pragma unroll
                    for (int i = 0; i < 8; ++i) {
                        if (above + c[i] >= kk) {
                            s_u[1] = uint32_t(255 - 8 * lane - i);
                            s_u[2] = above;
                            s_u[3] = c[i];
                            break;
                        }
                        above += c[i];
                    }
                }
            }
            __syncthreads();
            const uint32_t tb = s_u[1], cnt = s_u[3];
            kk -= s_u[2];
            lo += tb << sh;
            if (sh == 0) {   // the bucket is one key value
                exact = true;
                break;
            }
            span = min(span - (tb << sh), (1u << sh) - 1u);
            if (cnt <= uint32_t(kTailList)) break;
        }
        if (exact) {
            T = lo;
            need = kk;
        } else {
            // gather the bucket's keys (at most kTailList) and rank them exactly
            if (tid == 0) s_u[4] = 0;
            __syncthreads();
            // four groups of NTHR keys per step (uniform trip count for the ballots): loads first, then
            // one slot reservation per warp for all four groups
            for (int base = sinkP; base < recStart; base += 4 * NTHR) {
                uint32_t kv[4], bal[4];
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const int j = base + u * NTHR + tid;
                    kv[u] = (j < recStart) ? keys[j] : 0u;
                }
                uint32_t cnt = 0;
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const int j = base + u * NTHR + tid;
                    bal[u] = __ballot_sync(0xffffffffu, (j < recStart) & (kv[u] >= lo) & (kv[u] - lo <= span));
                    cnt += __popc(bal[u]);
                }
                uint32_t slot = 0;
                if (lane == 0 && cnt != 0u) slot = atomicAdd(&s_u[4], cnt);
                slot = __shfl_sync(0xffffffffu, slot, 0);
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    if ((bal[u] >> lane) & 1u) list[slot + __popc(bal[u] & ((1u << lane) - 1u))] = kv[u];
                    slot += __popc(bal[u]);
                }
            }
            __syncthreads();
            const int m = int(s_u[4]);
            // T = the key v with #(> v) < kk <= #(>= v); every holder of v writes the same values
            for (int i = tid; i < m; i += NTHR) {
                const uint32_t v = list[i];
                uint32_t gt = 0, ge = 0;
                for (int t = 0; t < m; ++t) {
                    const uint32_t w = list[t];
                    gt += w > v ? 1u : 0u;
                    ge += w >= v ? 1u : 0u;
                }
                if (gt < kk && kk <= ge) {
                    s_u[5] = v;
                    s_u[6] = kk - gt;
                }
            }
            __syncthreads();
            T = s_u[5];
            need = s_u[6];
        }
    }

    // 3. ascending compaction of sink U recency U {key > T} U {the first `need` keys == T}: warp w owns
    //    a contiguous segment of pages and walks it 32 pages at a time (lane = page); ballots give the
    //    ranks inside the warp, one exchange of the warps' totals gives the segments' offsets
    const int seg = (((N + W - 1) / W) + 31) & ~31;
    const int s0 = min(warp * seg, N), s1 = min(s0 + seg, N);
    const uint32_t below = (1u << lane) - 1u;
    // four groups of 32 pages per step, branch-free: the key loads first, then the flags (a page is
    // taken if forced or above T; equal to T is decided by rank)
    auto classify4 = [&](int c, bool (&tk)[4], bool (&eq)[4]) {
        uint32_t kv[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const int j = c + 32 * u + lane;
            kv[u] = (j < s1) ? keys[j] : 0u;
        }
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const int j = c + 32 * u + lane;
            const bool inr = j < s1;
            const bool forced = take_all | (j < sinkP) | (j >= recStart);
            tk[u] = inr & (forced | (radix & (kv[u] > T)));
            eq[u] = inr & !forced & radix & (kv[u] == T);
        }
    };
    uint32_t ct = 0, ce = 0;
    for (int c = s0; c < s1; c += 128) {
        bool tk[4], eq[4];
        classify4(c, tk, eq);
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            ct += __popc(__ballot_sync(0xffffffffu, tk[u]));
            ce += __popc(__ballot_sync(0xffffffffu, eq[u]));
        }
    }
    if (lane == 0) {
        s_wt[warp] = ct;
        s_we[warp] = ce;
    }
    __syncthreads();
    uint32_t take_before = 0, eq_before = 0, take_tot = 0, eq_tot = 0;
    for (int w = 0; w < W; ++w) {
        if (w < warp) {
            take_before += s_wt[w];
            eq_before += s_we[w];
        }
        take_tot += s_wt[w];
        eq_tot += s_we[w];
    }
    uint32_t pos = take_before + min(need, eq_before), eq_seen = eq_before;
    int32_t* out = a.sel_pages + size_t(b) * a.sel_stride;
    for (int c = s0; c < s1; c += 128) {
        bool tk[4], eq[4];
        uint32_t beq[4];
        classify4(c, tk, eq);
#pragma unroll
        for (int u = 0; u < 4; ++u) beq[u] = __ballot_sync(0xffffffffu, eq[u]);
#pragma unroll
        for (int u = 0; u < 4; ++u) {   // in page order: the ranks carry from group to group
            const bool take = tk[u] || (eq[u] && eq_seen + __popc(beq[u] & below) < need);
            const uint32_t bt = __ballot_sync(0xffffffffu, take);
            if (take) {
                const uint32_t at = pos + __popc(bt & below);
                if (at < uint32_t(a.sel_stride)) out[at] = c + 32 * u + lane;
            }
            pos += __popc(bt);
            eq_seen += __popc(beq[u]);
        }
    }
    if (tid == 0) a.sel_cnt[b] = int(min(take_tot + min(need, eq_tot), uint32_t(a.sel_stride)));
}

// Every thread of the CTA calls this after the output merge.  smem: the kernel's page-stage area,
// idle by now (free_bytes long, 16-byte aligned); recv: the merge's receive area; n, N: the
// sequence's tokens and pages; pre: select_preload's terms.
template <int NTHR, int G, int D>
__device__ __forceinline__ void select_tail(const DecodeParams& p, unsigned char* smem, size_t free_bytes,
                                            const float* recv, int b, int g, int n, int N,
                                            const float (&pre)[2][G]) {
    const int tid = threadIdx.x;
    const int Hq = p.num_q_heads, Hkv = p.num_kv_heads, S = p.num_splits, h0 = g * G;
    const size_t maxp = size_t(p.max_pages);
    float* s_c = reinterpret_cast<float*>(smem);               // [kMaxGroup] per-head normalisers
    uint32_t* s_flag = reinterpret_cast<uint32_t*>(s_c + kMaxGroup);
    const float* pl = p.page_lse + (size_t(b) * Hq + h0) * maxp;
    unsigned long long* acc = p.score_acc + size_t(b) * maxp;
    // adds the unit's share of page j's score (the sum over its G heads of 2^(lse_hj - c_h))
    auto add_share = [&](int j, const float (&v)[G]) {
        float sc = 0.f;
#pragma unroll
        for (int h = 0; h < G; ++h) sc += exp2_approx(v[h] - s_c[h]);
        atomicAdd(acc + j, __float2ull_rn(sc * kFixScale));
    };
    // pages [j0, j1), four per thread at a time (4 G independent loads in flight)
    auto shares = [&](int j0, int j1) {
        for (int jb = j0 + tid; jb < j1; jb += 4 * NTHR) {
            float v[4][G];
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int h = 0; h < G; ++h) {
                    const int j = jb + i * NTHR;
                    v[i][h] = (j < j1) ? __ldcg(pl + size_t(h) * maxp + j) : -INFINITY;
                }
#pragma unroll
            for (int i = 0; i < 4; ++i)
                if (jb + i * NTHR < j1) add_share(jb + i * NTHR, v[i]);
        }
    };
    // c_h = log2 of the sum over states of l * 2^m (no token of the head: +inf, every term 0)
    auto norm = [](float M, float Z) { return (Z > 0.f) ? M + log2_approx(Z) : INFINITY; };

    // Delta-layer plans keep each unit in one cluster (fit_plan), so every state of the unit is in
    // this CTA's receive area: c_h here, then this CTA's pages
    const int C = S;
    const float* st = merge_recv_states<D, G>(recv, C);   // [C][G][4]: (m, l) then the fp32-term (m, l)
    __syncthreads();   // no thread still reads the merge records in the stage area
    if (tid < G) {
        float M = -INFINITY;
        for (int j = 0; j < C; ++j) M = fmaxf(M, st[(j * G + tid) * 4 + 2]);
        const float mu = (M == -INFINITY) ? 0.f : M;
        float Z = 0.f;
        for (int j = 0; j < C; ++j) {
            const float l = st[(j * G + tid) * 4 + 3];
            if (l > 0.f) Z = fmaf(l, exp2_approx(st[(j * G + tid) * 4 + 2] - mu), Z);
        }
        s_c[tid] = norm(M, Z);
    }
    __syncthreads();
    const int i0 = blockIdx.x * p.items_per_split, i1 = min(i0 + p.items_per_split, N);
#pragma unroll
    for (int i = 0; i < 2; ++i)   // the preloaded pages
        if (i0 + tid + i * NTHR < i1) add_share(i0 + tid + i * NTHR, pre[i]);
    shares(i0 + 2 * NTHR, i1);
    if (!arrive_last(p.seq_tickets + b, Hkv * S, s_flag)) return;
    SelectFinal a;
    a.score_acc = p.score_acc;
    a.keys = p.keys;
    a.page_scores = p.page_scores;
    a.sel_cnt = p.sel_cnt_out;
    a.sel_pages = p.sel_pages_out;
    a.sel_stride = p.sel_stride_out;
    a.max_pages = p.max_pages;
    a.budget_pages = p.budget_pages;
    a.sink_tokens = p.sink_tokens;
    a.recency_tokens = p.recency_tokens;
    __syncthreads();   // s_c and s_flag are about to be overwritten by the final stage's scratch
    select_final<NTHR>(a, smem, free_bytes, b, n, N);
}

}  // namespace delta

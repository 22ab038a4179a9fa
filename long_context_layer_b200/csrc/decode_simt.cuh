// CUDA-core split-KV decode kernel (fp32 storage; included by delta_attn.cu only).
#pragma once

#include "common.cuh"
#include "select_tail.cuh"

namespace delta {

template <typename T, int D, int STAGES>
struct DecodeSmem {
    static constexpr uint32_t kChunk = kPage * D * sizeof(T);                    // one K or V page
    static constexpr size_t kStages = size_t(kWarps) * STAGES * 2 * kChunk;
    static constexpr size_t kBars = size_t(kWarps) * STAGES * sizeof(uint64_t);
    static constexpr size_t kPbuf = size_t(kWarps) * 2 * 8 * kMaxGroup * sizeof(float);
    static constexpr size_t kAbuf = size_t(kWarps) * 2 * kMaxGroup * sizeof(float);
    static constexpr size_t kMerge = size_t(kWarps * 2 + 1) * kMaxGroup * (D + 2) * sizeof(float);
    static constexpr size_t kMain = kStages > kMerge ? kStages : kMerge;
    static constexpr size_t kRecv = size_t(recv_floats<D>()) * sizeof(float);
    static constexpr size_t kBytes = kMain + kBars + kPbuf + kAbuf + kRecv;
};

template <typename T, int D, int G, int STAGES>
__global__ void __launch_bounds__(kThreads, 1) decode_kernel(const DecodeParams p) {
    using S = DecodeSmem<T, D, STAGES>;
    constexpr int DS = D / 16;          // dimensions per lane
    constexpr int GP = pad_group(G);    // group padded to a power of two
    constexpr int PE = kPage * D;       // elements of one K or V page

    extern __shared__ __align__(128) unsigned char smem[];
    T* stages = reinterpret_cast<T*>(smem);
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + S::kMain);
    float* pbuf = reinterpret_cast<float*>(smem + S::kMain + S::kBars);
    float* abuf = pbuf + kWarps * 2 * 8 * kMaxGroup;
    float* recv = reinterpret_cast<float*>(smem + S::kMain + S::kBars + S::kPbuf + S::kAbuf);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int half = lane >> 4, hl = lane & 15;
    const int b = blockIdx.z, g = blockIdx.y, split = blockIdx.x;
    const int Hq = p.num_q_heads;
    const int h0 = g * G;

    uint64_t* wbar = bars + warp * STAGES;
    T* wst = stages + size_t(warp) * STAGES * 2 * PE;
    if (lane == 0) {
#pragma unroll
        for (int s = 0; s < STAGES; ++s) mbar_init(&wbar[s], 1);
        fence_mbar_init();
    }
    __syncwarp();
    merge_prologue(recv);
    // The page table and kv_len are inputs of the whole step (no kernel of the stream writes them),
    // so full and delta layers resolve their pages before waiting for the previous kernel; a sparse
    // layer's page list is the output of the delta-layer: read after the wait unless the caller
    // states it settled.
    SeqExtent ex = seq_extent(p, b);
    int i0 = 0, nk = 0;
    WarpPages pages;
    auto setup = [&]() {
        seq_count(p, b, ex);
        i0 = split * p.items_per_split;
        const int i1 = min(i0 + p.items_per_split, ex.count);
        nk = (i1 - i0 > warp) ? (i1 - i0 - warp + kWarps - 1) / kWarps : 0;   // pages of this warp
        pages_init(pages, p, ex, b, i0, warp, nk, lane);
    };
    const T* kpool = reinterpret_cast<const T*>(p.k_pool);
    const T* vpool = reinterpret_cast<const T*>(p.v_pool);
    const uint64_t policy = evict_first_policy();

    // all lanes call (the page id is shuffled out of the prefetched list); lane 0 issues
    auto issue = [&](int k) {
        int lp, ph;
        pages_get(pages, k, lp, ph);
        if (lane != 0) return;
        const int s = k % STAGES;
        if (ph >= 0) {
            T* dst = wst + size_t(s) * 2 * PE;
            const size_t off = (size_t(ph) * p.num_kv_heads + g) * PE;
            mbar_expect_tx(&wbar[s], 2 * S::kChunk);
            bulk_load(dst, kpool + off, S::kChunk, &wbar[s], policy);
            bulk_load(dst + PE, vpool + off, S::kChunk, &wbar[s], policy);
        } else {
            mbar_arrive(&wbar[s]);  // completes the phase with no data; consumers skip the page
        }
    };

    // Before waiting for the previous kernel: full and delta layers (and sparse layers whose
    // selection the caller states settled) know their pages, so the first stages' copies start
    // now, except the page holding the appended token, which the previous kernel may still write
    // (settled inputs: that one too); q goes to L2.
    const bool known = p.mode != kModeSparse || p.settled;
    uint32_t early = 0;   // bit k: page k's copy was issued before the wait
    if (known) {
        setup();
        for (int k = 0; k < min(STAGES, nk); ++k) {
            int lp, ph;
            pages_get(pages, k, lp, ph);
            if (ph >= 0 && (lp != ex.N - 1 || p.settled)) {
                issue(k);
                early |= 1u << k;
            }
        }
    }
    if (threadIdx.x == 0) prefetch_l2(reinterpret_cast<const T*>(p.q) + (size_t(b) * Hq + h0) * D, G * D * sizeof(T));
    pdl_wait();      // q, the appended token and a selection written by earlier kernels
    pdl_trigger();
    if (!known) setup();
    const int n = ex.n;

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

    for (int k = 0; k < min(STAGES, nk); ++k)
        if (!((early >> k) & 1u)) issue(k);

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
        pages_advance(pages, p, ex, b, i0, warp, nk, lane, k);
        const int s = k % STAGES;
        if (!mbar_wait(&wbar[s], (k / STAGES) & 1)) {
            if (lane == 0) atomicOr(p.err, kErrTimeout);
            failed = true;
            break;
        }
        consumed = k + 1;
        int lp, ph;
        pages_get(pages, k, lp, ph);
        if (ph >= 0) {
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
                    p.page_lse[(size_t(b) * Hq + h0 + hl) * p.max_pages + lp] = mp + log2_approx(e);
                if (p.logits != nullptr && hl < G) {   // per-token logits (HEAD_MAX scoring)
                    float* lg = p.logits + ((size_t(b) * Hq + h0 + hl) * p.max_pages + lp) * kPage + half * 8;
#pragma unroll
                    for (int j = 0; j < 8; ++j) lg[j] = sc[j];
                }
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
        if (k + STAGES < nk) issue(k + STAGES);
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
    float pre[2][G];   // delta-layers: this CTA's page terms, loaded before the merge
    if (p.fuse_select) select_preload<kThreads, G>(p, b, g, ex.N, pre);
    merge_epilogue<T, D, G, kWarps * 2>(p, smem, mo, mml, recv, b, g, kMaxGroup * D, kMaxGroup * 2);
    // delta-layers scoring with HEAD_SUM: page scores and the selection, in the stage area
    if (p.fuse_select) select_tail<kThreads, G, D>(p, smem, S::kMain, recv, b, g, ex.n, ex.N, pre);
}

}  // namespace delta

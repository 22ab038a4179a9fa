// Tensor-core split-KV decode kernel for bf16 storage (included by delta_attn.cu only).
//
// One CTA = (split, KV head, sequence); each of its WARPS warps (4, 6 or 8) streams whole pages.  A page of one
// KV head (16 tokens x D) of K and of V arrives in the warp's shared-memory stage through 2-D
// TMA tensor copies (cp.async.bulk.tensor, 64-column boxes, 128-byte swizzle) completing on an
// mbarrier.  Per page:
//   S^T[16 tok x 8 heads] = K[16 x D] . Q^T[D x 8]      D/16 mma.m16n8k16 (bf16 in, fp32 acc),
//                                                        K fragments by ldmatrix from the
//                                                        swizzled tile, Q fragments in registers;
//   online softmax per head (base-2 logits; the G <= 8 query heads are the MMA's N columns);
//   P^T fragments = movmatrix.trans of the bf16-rounded probabilities;
//   O^T[D x 8] += V^T[D x 16 tok] . P^T[16 tok x 8]      D/16 mma.m16n8k16, V fragments by
//                                                        ldmatrix.trans.
// The softmax normaliser is accumulated from the same bf16-rounded probabilities the PV product
// uses, so every output is a true weighted mean of the values.
#pragma once

#include "common.cuh"
#include "select_tail.cuh"

namespace delta {

__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, int x, int y, uint64_t* bar,
                                            uint64_t policy) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes.L2::cache_hint"
        " [%0], [%1, {%2, %3}], [%4], %5;" ::"r"(smem_addr(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(smem_addr(bar)), "l"(policy)
        : "memory");
}

__device__ __forceinline__ void ldmatrix_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(addr));
}
__device__ __forceinline__ void ldmatrix_x4_trans(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                                  uint32_t& r3) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(addr));
}
__device__ __forceinline__ void mma_bf16_16816(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                               uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
        "{%0, %1, %2, %3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}
__device__ __forceinline__ uint32_t movmatrix_trans(uint32_t x) {
    uint32_t y;
    asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;" : "=r"(y) : "r"(x));
    return y;
}
__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&v);
}

// Shared-memory plan of the tensor-core kernel.
template <int D, int STAGES, int WARPS = kWarps>
struct MmaSmem {
    static constexpr int kBoxes = D / 64;                     // 64-column (128-byte) boxes per row
    static constexpr uint32_t kBox = 16 * 128;                // one box: 16 rows x 128 bytes
    static constexpr uint32_t kPage = 2 * kBoxes * kBox;      // K and V of one page, one KV head
    static constexpr size_t kStages = size_t(WARPS) * STAGES * kPage;
    // each warp's merge record ([8][D] outputs, two [8][2] states) reuses its own stages
    static_assert(size_t(STAGES) * kPage >= (size_t(kMaxGroup) * (D + 4) + 4 * kMaxGroup) * sizeof(float), "merge record");
    static constexpr size_t kMain = kStages;
    static constexpr size_t kBars = size_t(WARPS) * STAGES * sizeof(uint64_t);
    static constexpr size_t kRecv = size_t(recv_floats<D>()) * sizeof(float);
    static constexpr size_t kBytes = 1024 /* alignment slack */ + kMain + kBars + kRecv;
};

template <int D, int G, int STAGES, int WARPS>
__global__ void __launch_bounds__(WARPS * 32, 1) decode_mma_kernel(const DecodeParams p,
                                                              const __grid_constant__ CUtensorMap tmap_k,
                                                              const __grid_constant__ CUtensorMap tmap_v) {
    using S = MmaSmem<D, STAGES, WARPS>;
    constexpr int KS = D / 16;   // k-steps of the QK product = M-tiles of the PV product
    extern __shared__ unsigned char smem_raw[];
    unsigned char* smem =
        smem_raw + ((1024 - (static_cast<uint32_t>(__cvta_generic_to_shared(smem_raw)) & 1023)) & 1023);
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + S::kMain);
    float* recv = reinterpret_cast<float*>(smem + S::kMain + S::kBars);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g4 = lane >> 2, t4 = lane & 3;
    const int b = blockIdx.z, g = blockIdx.y, split = blockIdx.x;
    const int Hq = p.num_q_heads;
    const int h0 = g * G;

    uint64_t* wbar = bars + warp * STAGES;
    unsigned char* wst = smem + size_t(warp) * STAGES * S::kPage;
    if (lane == 0) {
#pragma unroll
        for (int s = 0; s < STAGES; ++s) mbar_init(&wbar[s], 1);
        fence_mbar_init();
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmap_k)) : "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmap_v)) : "memory");
    }
    __syncwarp();
    merge_prologue(recv);
    // The page table and kv_len are inputs of the whole step (no kernel of the stream writes them),
    // so full and delta layers resolve their pages before waiting for the previous kernel; a
    // sparse layer's page list is the output of the delta-layer: read before the wait when the
    // caller states it settled, else speculated on before the wait and checked after it.
    SeqExtent ex = seq_extent(p, b);
    int i0 = 0, nk = 0;
    WarpPages pages;
    auto setup = [&]() {
        seq_count(p, b, ex);
        i0 = split * p.items_per_split;
        const int i1 = min(i0 + p.items_per_split, ex.count);
        nk = (i1 - i0 > warp) ? (i1 - i0 - warp + WARPS - 1) / WARPS : 0;   // pages of this warp
        pages_init<WARPS>(pages, p, ex, b, i0, warp, nk, lane);
    };
    const uint64_t policy = evict_first_policy();
    // TMA of one page (K and V of KV head g) into stage k % STAGES; lane 0 only.
    auto load_page = [&](int k, int ph) {
        const int s = k % STAGES;
        unsigned char* dst = wst + size_t(s) * S::kPage;
        const int y = (ph * p.num_kv_heads + g) * kPage;   // row of (page, KV head g)
        mbar_expect_tx(&wbar[s], S::kPage);
#pragma unroll
        for (int nb = 0; nb < S::kBoxes; ++nb) {
            tma_load_2d(dst + nb * S::kBox, &tmap_k, nb * 64, y, &wbar[s], policy);
            tma_load_2d(dst + (S::kBoxes + nb) * S::kBox, &tmap_v, nb * 64, y, &wbar[s], policy);
        }
    };

    // ---- First pipeline stage, before the wait.  The previous kernel may still be running, so
    // only data no earlier kernel of the step changes is loaded now: pool pages other than the
    // sequence's last one (the appended token's page is loaded after the wait).  Full and delta
    // layers know their pages; sparse layers speculate that the selection is already final (it
    // is for every sparse layer but the first after a delta-layer) and check it after the wait.
    if (threadIdx.x == 0)
        prefetch_l2(reinterpret_cast<const __nv_bfloat16*>(p.q) + (size_t(b) * Hq + h0) * D, G * D * 2);
    uint32_t early = 0;       // bit k: page k's load was issued before the wait
    uint32_t spec_used = 0;   // bit s: stage s spent its first phase on a discarded speculative load
    WarpPages spec;
    int nk_spec = 0;
    if (p.mode != kModeSparse || p.settled) {
        setup();   // a settled selection is final: read (and checked) now
    } else {
        const int cap = min(p.sel_stride, p.items_per_split * p.num_splits);
        const int scnt = min(max(__ldcg(p.sel_cnt + b), 0), cap);
        const int si0 = split * p.items_per_split;
        const int si1 = min(si0 + p.items_per_split, scnt);
        nk_spec = (si1 - si0 > warp) ? (si1 - si0 - warp + WARPS - 1) / WARPS : 0;
        spec.cur = 0;
        fetch_pages<true, WARPS>(p, ex, b, si0, warp, nk_spec, 0, lane, spec.lp_a, spec.ph_a);
        spec.lp_b = spec.ph_b = -1;
    }
    {
        const bool speculative = p.mode == kModeSparse && !p.settled;
        const WarpPages& pre = speculative ? spec : pages;
        const int npre = min(STAGES, speculative ? nk_spec : nk);
        for (int k = 0; k < npre; ++k) {
            int lp, ph;
            pages_get(pre, k, lp, ph);
            // the appended token's page too once the inputs are settled
            if (ph >= 0 && (lp != ex.N - 1 || p.settled)) {
                if (lane == 0) load_page(k, ph);
                early |= 1u << k;
            }
        }
    }
    pdl_wait();      // q, the appended token, and a selection written by the previous kernel
    pdl_trigger();

    // ---- Q^T fragments (B operand of the QK product): head g4 of the group, dims k*16 + 2*t4 (+8);
    // issued first so their latency overlaps the selection check below
    uint32_t qb[KS][2];
    {
        const __nv_bfloat16* qp = reinterpret_cast<const __nv_bfloat16*>(p.q) + (size_t(b) * Hq + h0 + g4) * D;
#pragma unroll
        for (int k = 0; k < KS; ++k) {
            if (g4 < G) {
                qb[k][0] = *reinterpret_cast<const uint32_t*>(qp + k * 16 + 2 * t4);
                qb[k][1] = *reinterpret_cast<const uint32_t*>(qp + k * 16 + 8 + 2 * t4);
            } else {
                qb[k][0] = qb[k][1] = 0u;
            }
        }
    }

    if (p.mode == kModeSparse && !p.settled) {
        // The selection's entries at the speculated positions are loaded together with its count
        // (one round trip); they are the real ones whenever the count is the speculated one.
        const int lp_real =
            (lane < nk_spec) ? __ldcg(p.sel_pages + size_t(b) * p.sel_stride + split * p.items_per_split + warp +
                                      lane * WARPS)
                             : -1;
        seq_count(p, b, ex);
        i0 = split * p.items_per_split;
        const int i1 = min(i0 + p.items_per_split, ex.count);
        nk = (i1 - i0 > warp) ? (i1 - i0 - warp + WARPS - 1) / WARPS : 0;
        // The speculation holds if the selection's logical pages of this warp's first chunk are the
        // ones guessed (the page table does not change within the step) and were all valid.
        const bool all_same = __all_sync(0xffffffffu, lane >= nk || (lp_real == spec.lp_a && spec.ph_a >= 0)) &&
                              nk == nk_spec;
        if (all_same) {
            pages = spec;
            fetch_pages<false, WARPS>(p, ex, b, i0, warp, nk, 32, lane, pages.lp_b, pages.ph_b);
        } else {
            pages_init<WARPS>(pages, p, ex, b, i0, warp, nk, lane);
            // keep an early load only if it is exactly the selection's page; otherwise drain all
            bool same = nk == nk_spec;
            for (int k = 0; k < min(STAGES, nk_spec); ++k) {
                if (!((early >> k) & 1u)) continue;
                int lp0, ph0, lp1, ph1;
                pages_get(spec, k, lp0, ph0);
                pages_get(pages, k, lp1, ph1);
                same = same && lp0 == lp1 && ph0 == ph1;
            }
            if (!same) {
                // drain the speculative loads (bounded wait); those stages start their real use one
                // phase later
                for (int k = 0; k < min(STAGES, nk_spec); ++k)
                    if ((early >> k) & 1u) {
                        if (!mbar_wait(&wbar[k % STAGES], 0) && lane == 0) atomicOr(p.err, kErrTimeout);
                        spec_used |= 1u << (k % STAGES);
                    }
                early = 0;
            }
        }
    }

    // all lanes call (the page id is shuffled out of the prefetched list); lane 0 issues
    auto issue = [&](int k) {
        int lp, ph;
        pages_get(pages, k, lp, ph);
        if (lane != 0) return;
        if (ph >= 0) load_page(k, ph);
        else mbar_arrive(&wbar[k % STAGES]);   // completes the phase with no data; the page is skipped
    };
    for (int k = 0; k < min(STAGES, nk); ++k)
        if (!((early >> k) & 1u)) issue(k);
    // phase parity of the stage holding page k
    auto parity = [&](int k) -> uint32_t { return ((k / STAGES) + ((spec_used >> (k % STAGES)) & 1u)) & 1u; };

    float m_run[2] = {-INFINITY, -INFINITY}, l_run[2] = {0.f, 0.f};   // heads 2*t4, 2*t4+1
    // delta-layers: the sum of the unrounded fp32 terms 2^(s - m_run) (l_run sums the bf16-rounded
    // probabilities that also weight V), so the selection's normalisers match its page terms; its
    // maximum is m_run
    float dl_run[2] = {0.f, 0.f};
    float acc[KS][4];
#pragma unroll
    for (int mt = 0; mt < KS; ++mt) acc[mt][0] = acc[mt][1] = acc[mt][2] = acc[mt][3] = 0.f;

    // per-lane ldmatrix row/chunk roles (see the fragment layouts of mma.m16n8k16)
    const int lj = lane >> 3;
    const int k_row = (lane & 7) + ((lj & 1) << 3);     // K: token row of this lane's address
    const int k_sub = lj >> 1;                          // K: which 8-column half of the k-step
    const int v_row = (lane & 7) + ((lj >> 1) << 3);    // V: token row
    const int v_sub = lj & 1;                           // V: which 8-column half of the M-tile
    bool failed = false;
    int consumed = 0;

    // S^T (16 tokens x 8 heads) of the page in stage s; masked tokens get -inf.  Two accumulator
    // chains (even / odd k-steps) halve the dependent MMA chain.
    auto qk_page = [&](int s, int tv, float (&sc)[4]) {
        const uint32_t kbase = smem_addr(wst + size_t(s) * S::kPage);
        float c0[4] = {0.f, 0.f, 0.f, 0.f}, c1[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int kk = 0; kk < KS; ++kk) {
            const int chunk = kk * 2 + k_sub;               // 16-byte chunk of the row (0..D/8-1)
            const uint32_t addr = kbase + (chunk >> 3) * S::kBox + k_row * 128 + (((chunk & 7) ^ (k_row & 7)) << 4);
            uint32_t a0, a1, a2, a3;
            ldmatrix_x4(addr, a0, a1, a2, a3);
            if (kk & 1) mma_bf16_16816(c1, a0, a1, a2, a3, qb[kk][0], qb[kk][1]);
            else mma_bf16_16816(c0, a0, a1, a2, a3, qb[kk][0], qb[kk][1]);
        }
        // base-2 logits; tokens g4 and g4+8, heads 2*t4 and 2*t4+1
        const bool ok0 = g4 < tv, ok1 = g4 + 8 < tv;
        sc[0] = ok0 ? (c0[0] + c1[0]) * p.qscale : -INFINITY;
        sc[1] = ok0 ? (c0[1] + c1[1]) * p.qscale : -INFINITY;
        sc[2] = ok1 ? (c0[2] + c1[2]) * p.qscale : -INFINITY;
        sc[3] = ok1 ? (c0[3] + c1[3]) * p.qscale : -INFINITY;
    };
    // Delta-layers: each page's log2-sum-exp per head, from the same unrounded terms 2^(s - m) the
    // online softmax forms (m: the running maximum over both pages), summed over the page's 16
    // tokens (the g4 lanes), and the fp32-term running sum.  p*: a lane's terms of page A / B
    // (tokens g4, g4 + 8; heads 2 t4, 2 t4 + 1); al: the softmax's rescale factors.
    auto page_partials = [&](const float (&pa)[4], const float (&pb)[4], float mn0, float mn1, float al0, float al1,
                             bool vA, bool vB, int lpA, int lpB) {
        float ea0 = pa[0] + pa[2], ea1 = pa[1] + pa[3], eb0 = pb[0] + pb[2], eb1 = pb[1] + pb[3];
#pragma unroll
        for (int o = 4; o < 32; o <<= 1) {
            ea0 += __shfl_xor_sync(0xffffffffu, ea0, o);
            ea1 += __shfl_xor_sync(0xffffffffu, ea1, o);
            eb0 += __shfl_xor_sync(0xffffffffu, eb0, o);
            eb1 += __shfl_xor_sync(0xffffffffu, eb1, o);
        }
        dl_run[0] = dl_run[0] * al0 + (ea0 + eb0);
        dl_run[1] = dl_run[1] * al1 + (ea1 + eb1);
        const int hA = 2 * t4, hB = 2 * t4 + 1;
        if (g4 == 0) {
            float* row = p.page_lse + (size_t(b) * Hq + h0) * p.max_pages;
            if (vA && hA < G) row[size_t(hA) * p.max_pages + lpA] = mn0 + log2_approx(ea0);
            if (vA && hB < G) row[size_t(hB) * p.max_pages + lpA] = mn1 + log2_approx(ea1);
            if (vB && hA < G) row[size_t(hA) * p.max_pages + lpB] = mn0 + log2_approx(eb0);
            if (vB && hB < G) row[size_t(hB) * p.max_pages + lpB] = mn1 + log2_approx(eb1);
        }
    };
    // HEAD_MAX scoring: every head's per-token logits (tokens g4, g4 + 8; heads 2 t4, 2 t4 + 1)
    auto store_logits = [&](const float (&sc)[4], int lp) {
        float* lg = p.logits + (size_t(b) * Hq + h0) * (size_t(p.max_pages) * kPage) + size_t(lp) * kPage;
        const size_t hs = size_t(p.max_pages) * kPage;
        if (2 * t4 < G) { lg[2 * t4 * hs + g4] = sc[0]; lg[2 * t4 * hs + g4 + 8] = sc[2]; }
        if (2 * t4 + 1 < G) { lg[(2 * t4 + 1) * hs + g4] = sc[1]; lg[(2 * t4 + 1) * hs + g4 + 8] = sc[3]; }
    };
    // tokens past the end of the context: zero their V rows (they may hold non-finite bytes)
    auto zero_tail = [&](int s, int tv) {
        uint4* vz = reinterpret_cast<uint4*>(wst + size_t(s) * S::kPage + S::kBoxes * S::kBox);
        const int per_box = (kPage - tv) * 8;
        for (int c = lane; c < S::kBoxes * per_box; c += 32) {
            const int box = c / per_box, rem = c % per_box;
            vz[box * (S::kBox / 16) + (tv + rem / 8) * 8 + (rem % 8)] = make_uint4(0, 0, 0, 0);
        }
        __syncwarp();
    };
    // O^T += V^T . P^T for the page in stage s
    auto pv_page = [&](int s, uint32_t pb0, uint32_t pb1) {
        const uint32_t vbase = smem_addr(wst + size_t(s) * S::kPage) + S::kBoxes * S::kBox;
#pragma unroll
        for (int mt = 0; mt < KS; ++mt) {
            const int chunk = mt * 2 + v_sub;
            const uint32_t addr = vbase + (chunk >> 3) * S::kBox + v_row * 128 + (((chunk & 7) ^ (v_row & 7)) << 4);
            uint32_t a0, a1, a2, a3;
            ldmatrix_x4_trans(addr, a0, a1, a2, a3);
            mma_bf16_16816(acc[mt], a0, a1, a2, a3, pb0, pb1);
        }
    };

    // Pages are taken two at a time: their QK products, one softmax update and their PV
    // products are independent chains the scheduler interleaves.
    for (int k = 0; k < nk; k += 2) {
        pages_advance<WARPS>(pages, p, ex, b, i0, warp, nk, lane, k);
        const bool two = k + 1 < nk;
        const int sA = k % STAGES, sB = (k + 1) % STAGES;
        if (!mbar_wait(&wbar[sA], parity(k)) || (two && !mbar_wait(&wbar[sB], parity(k + 1)))) {
            if (lane == 0) atomicOr(p.err, kErrTimeout);
            failed = true;
            break;
        }
        consumed = k + (two ? 2 : 1);
        int lpA, phA, lpB = -1, phB = -1;
        pages_get(pages, k, lpA, phA);
        if (two) pages_get(pages, k + 1, lpB, phB);
        const bool vA = phA >= 0, vB = phB >= 0;
        const int tvA = vA ? min(kPage, ex.n - lpA * kPage) : 0;
        const int tvB = vB ? min(kPage, ex.n - lpB * kPage) : 0;
        float scA[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
        float scB[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
        if (vA) qk_page(sA, tvA, scA);
        if (vB) qk_page(sB, tvB, scB);
        bool zeroed = false;
        if (vA || vB) {
            if (p.logits != nullptr) {
                if (vA) store_logits(scA, lpA);
                if (vB) store_logits(scB, lpB);
            }
            float mx0 = fmaxf(fmaxf(scA[0], scA[2]), fmaxf(scB[0], scB[2]));
            float mx1 = fmaxf(fmaxf(scA[1], scA[3]), fmaxf(scB[1], scB[3]));
#pragma unroll
            for (int o = 4; o < 32; o <<= 1) {
                mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, o));
                mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, o));
            }
            const float mn0 = fmaxf(m_run[0], mx0), mn1 = fmaxf(m_run[1], mx1);   // finite: a valid token exists
            const float al0 = exp2_approx(m_run[0] - mn0), al1 = exp2_approx(m_run[1] - mn1);
            const float pa[4] = {exp2_approx(scA[0] - mn0), exp2_approx(scA[1] - mn1), exp2_approx(scA[2] - mn0),
                                 exp2_approx(scA[3] - mn1)};
            const float pb[4] = {exp2_approx(scB[0] - mn0), exp2_approx(scB[1] - mn1), exp2_approx(scB[2] - mn0),
                                 exp2_approx(scB[3] - mn1)};
            if (p.mode == kModeDelta) page_partials(pa, pb, mn0, mn1, al0, al1, vA, vB, lpA, lpB);
            const uint32_t xa0 = pack_bf16(pa[0], pa[1]);
            const uint32_t xa1 = pack_bf16(pa[2], pa[3]);
            const uint32_t xb0 = pack_bf16(pb[0], pb[1]);
            const uint32_t xb1 = pack_bf16(pb[2], pb[3]);
            float p0, p1, p2, p3, q0, q1, q2, q3;
            unpack_bf16x2(xa0, p0, p1);
            unpack_bf16x2(xa1, p2, p3);
            unpack_bf16x2(xb0, q0, q1);
            unpack_bf16x2(xb1, q2, q3);
            float rs0 = (p0 + p2) + (q0 + q2), rs1 = (p1 + p3) + (q1 + q3);
#pragma unroll
            for (int o = 4; o < 32; o <<= 1) {
                rs0 += __shfl_xor_sync(0xffffffffu, rs0, o);
                rs1 += __shfl_xor_sync(0xffffffffu, rs1, o);
            }
            l_run[0] = l_run[0] * al0 + rs0;
            l_run[1] = l_run[1] * al1 + rs1;
            m_run[0] = mn0;
            m_run[1] = mn1;
#pragma unroll
            for (int mt = 0; mt < KS; ++mt) {
                acc[mt][0] *= al0;
                acc[mt][1] *= al1;
                acc[mt][2] *= al0;
                acc[mt][3] *= al1;
            }
            if (vA && tvA < kPage) { zero_tail(sA, tvA); zeroed = true; }
            if (vB && tvB < kPage) { zero_tail(sB, tvB); zeroed = true; }
            if (vA) pv_page(sA, movmatrix_trans(xa0), movmatrix_trans(xa1));
            if (vB) pv_page(sB, movmatrix_trans(xb0), movmatrix_trans(xb1));
        }
        __syncwarp();
        if (zeroed && lane == 0) fence_proxy_async_smem();
        if (k + STAGES < nk) issue(k + STAGES);
        if (two && k + 1 + STAGES < nk) issue(k + 1 + STAGES);
    }
    if (failed) {
        // drain this warp's copies still in flight (bounded) before shared memory is released
        for (int k = consumed + 1; k < min(consumed + STAGES, nk); ++k) mbar_wait(&wbar[k % STAGES], parity(k));
    }

    // ---- this warp's state into its own stage area (all of its copies have landed and no other
    // warp touches that area), one barrier, then the merge of the CTA's warps and of the splits
    __syncwarp();
    // rows padded by 4 floats: the four lanes of a column group (t4) store to different banks
    constexpr int kRow = D + 4;
    float* po = reinterpret_cast<float*>(wst);           // [8][D + 4] outputs
    float* pml = po + kMaxGroup * kRow;                   // [8][2] (max, sum)
    float* pdl = pml + kMaxGroup * 2;                     // [8][2] delta-layers: over the fp32 page terms
#pragma unroll
    for (int mt = 0; mt < KS; ++mt) {
        const int d = mt * 16 + g4;
        po[(2 * t4) * kRow + d] = acc[mt][0];
        po[(2 * t4 + 1) * kRow + d] = acc[mt][1];
        po[(2 * t4) * kRow + d + 8] = acc[mt][2];
        po[(2 * t4 + 1) * kRow + d + 8] = acc[mt][3];
    }
    if (g4 == 0) {
        pml[(2 * t4) * 2 + 0] = m_run[0];
        pml[(2 * t4) * 2 + 1] = l_run[0];
        pml[(2 * t4 + 1) * 2 + 0] = m_run[1];
        pml[(2 * t4 + 1) * 2 + 1] = l_run[1];
        if (p.mode == kModeDelta) {
            pdl[(2 * t4) * 2 + 0] = m_run[0];
            pdl[(2 * t4) * 2 + 1] = dl_run[0];
            pdl[(2 * t4 + 1) * 2 + 0] = m_run[1];
            pdl[(2 * t4 + 1) * 2 + 1] = dl_run[1];
        }
    }
    __syncthreads();
    constexpr int kPart = STAGES * int(S::kPage) / 4;     // floats between two warps' records
    const float* mo0 = reinterpret_cast<const float*>(smem);
    float pre[2][G];   // delta-layers: this CTA's page terms, loaded before the merge
    if (p.fuse_select) select_preload<WARPS * 32, G>(p, b, g, ex.N, pre);
    merge_epilogue<__nv_bfloat16, D, G, WARPS, WARPS * 32, kRow>(
        p, smem, mo0, mo0 + kMaxGroup * kRow, recv, b, g, kPart, kPart,
        (p.mode == kModeDelta) ? mo0 + kMaxGroup * kRow + kMaxGroup * 2 : nullptr);
    // delta-layers scoring with HEAD_SUM: page scores and the selection, in the stage area
    if (p.fuse_select) select_tail<WARPS * 32, G, D>(p, smem, S::kStages, recv, b, g, ex.n, ex.N, pre);
}

}  // namespace delta

// Tensor-core split-KV decode kernel for bf16 storage (included by delta_attn.cu only).
//
// One CTA = (split, KV head, sequence); each of its 4 warps streams whole pages.  A page of one
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
template <int D, int STAGES>
struct MmaSmem {
    static constexpr int kBoxes = D / 64;                     // 64-column (128-byte) boxes per row
    static constexpr uint32_t kBox = 16 * 128;                // one box: 16 rows x 128 bytes
    static constexpr uint32_t kPage = 2 * kBoxes * kBox;      // K and V of one page, one KV head
    static constexpr size_t kStages = size_t(kWarps) * STAGES * kPage;
    static constexpr size_t kMerge = size_t(kWarps) * kMaxGroup * (D + 2) * sizeof(float);
    static constexpr size_t kLast = size_t(kMaxGroup) * kMaxSplits * 3 * sizeof(float) + 64;
    static constexpr size_t kMain0 = kStages > kMerge ? kStages : kMerge;
    static constexpr size_t kMain = kMain0 > kLast ? kMain0 : kLast;
    static constexpr size_t kBars = size_t(kWarps) * STAGES * sizeof(uint64_t);
    static constexpr size_t kMeta = size_t(kWarps) * STAGES * sizeof(int2);
    static constexpr size_t kBytes = 1024 /* alignment slack */ + kMain + kBars + kMeta;
};

template <int D, int G, int STAGES>
__global__ void __launch_bounds__(kThreads) decode_mma_kernel(const DecodeParams p,
                                                              const __grid_constant__ CUtensorMap tmap_k,
                                                              const __grid_constant__ CUtensorMap tmap_v) {
    using S = MmaSmem<D, STAGES>;
    constexpr int KS = D / 16;   // k-steps of the QK product = M-tiles of the PV product
    extern __shared__ unsigned char smem_raw[];
    unsigned char* smem =
        smem_raw + ((1024 - (static_cast<uint32_t>(__cvta_generic_to_shared(smem_raw)) & 1023)) & 1023);
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + S::kMain);
    int2* meta = reinterpret_cast<int2*>(smem + S::kMain + S::kBars);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g4 = lane >> 2, t4 = lane & 3;
    const int b = blockIdx.z, g = blockIdx.y, split = blockIdx.x;
    const int Hq = p.num_q_heads;
    const int h0 = g * G;

    // ---- sequence extent (validated; bad values are clamped and flagged)
    int n = p.kv_len[b];
    const int pbeg = p.indptr[b];
    const int npg = p.indptr[b + 1] - pbeg;
    if (n < 0) n = 0;
    if (n > npg * kPage || n > p.max_pages * kPage) {
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
    const int nk = (i1 - i0 > warp) ? (i1 - i0 - warp + kWarps - 1) / kWarps : 0;

    // ---- Q^T fragments (B operand of the QK product): head g4 of the group, dims k*16 + 2*t4 (+8)
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

    uint64_t* wbar = bars + warp * STAGES;
    int2* wmeta = meta + warp * STAGES;
    unsigned char* wst = smem + size_t(warp) * STAGES * S::kPage;
    if (lane == 0) {
#pragma unroll
        for (int s = 0; s < STAGES; ++s) mbar_init(&wbar[s], 1);
        fence_mbar_init();
    }
    __syncwarp();
    const uint64_t policy = evict_first_policy();
    const int row_base_g = g * kPage;   // row of (page, g) = (phys * Hkv + g) * 16

    auto issue = [&](int k) {   // lane 0 only
        const int s = k % STAGES;
        const int i = i0 + warp + k * kWarps;
        const int lp = (p.mode == kModeSparse) ? p.sel_pages[size_t(b) * p.sel_stride + i] : i;
        int valid = 0;
        int64_t phys = -1;
        if (lp >= 0 && lp < N) {
            phys = p.indices[pbeg + lp];
            valid = (phys >= 0 && phys < p.num_phys_pages) ? 1 : 0;
            if (!valid) atomicOr(p.err, kErrPage);
        } else {
            atomicOr(p.err, kErrSel);
        }
        wmeta[s] = make_int2(lp, valid);
        if (valid) {
            unsigned char* dst = wst + size_t(s) * S::kPage;
            const int y = int(phys) * p.num_kv_heads * kPage + row_base_g;
            mbar_expect_tx(&wbar[s], S::kPage);
#pragma unroll
            for (int nb = 0; nb < S::kBoxes; ++nb) {
                tma_load_2d(dst + nb * S::kBox, &tmap_k, nb * 64, y, &wbar[s], policy);
                tma_load_2d(dst + (S::kBoxes + nb) * S::kBox, &tmap_v, nb * 64, y, &wbar[s], policy);
            }
        } else {
            mbar_arrive(&wbar[s]);
        }
    };
    if (lane == 0)
        for (int k = 0; k < min(STAGES, nk); ++k) issue(k);

    float m_run[2] = {-INFINITY, -INFINITY}, l_run[2] = {0.f, 0.f};   // heads 2*t4, 2*t4+1
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

    for (int k = 0; k < nk; ++k) {
        const int s = k % STAGES;
        if (!mbar_wait(&wbar[s], (k / STAGES) & 1)) {
            if (lane == 0) atomicOr(p.err, kErrTimeout);
            failed = true;
            break;
        }
        consumed = k + 1;
        const int2 mt_ = wmeta[s];
        bool zeroed = false;
        if (mt_.y) {
            const int lp = mt_.x;
            const int tv = min(kPage, n - lp * kPage);
            const uint32_t kbase = smem_addr(wst + size_t(s) * S::kPage);
            const uint32_t vbase = kbase + S::kBoxes * S::kBox;
            // S^T = K . Q^T
            float sc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int kk = 0; kk < KS; ++kk) {
                const int chunk = kk * 2 + k_sub;               // 16-byte chunk of the row (0..D/8-1)
                const uint32_t addr = kbase + (chunk >> 3) * S::kBox + k_row * 128 + (((chunk & 7) ^ (k_row & 7)) << 4);
                uint32_t a0, a1, a2, a3;
                ldmatrix_x4(addr, a0, a1, a2, a3);
                mma_bf16_16816(sc, a0, a1, a2, a3, qb[kk][0], qb[kk][1]);
            }
            // base-2 logits; tokens g4 and g4+8, heads 2*t4 and 2*t4+1
            const bool ok0 = g4 < tv, ok1 = g4 + 8 < tv;
            sc[0] = ok0 ? sc[0] * p.qscale : -INFINITY;
            sc[1] = ok0 ? sc[1] * p.qscale : -INFINITY;
            sc[2] = ok1 ? sc[2] * p.qscale : -INFINITY;
            sc[3] = ok1 ? sc[3] * p.qscale : -INFINITY;
            float mx0 = fmaxf(sc[0], sc[2]), mx1 = fmaxf(sc[1], sc[3]);
#pragma unroll
            for (int o = 4; o < 32; o <<= 1) {
                mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, o));
                mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, o));
            }
            const float mn0 = fmaxf(m_run[0], mx0), mn1 = fmaxf(m_run[1], mx1);   // mx is finite: tv >= 1
            const float al0 = exp2_approx(m_run[0] - mn0), al1 = exp2_approx(m_run[1] - mn1);
            const uint32_t x0 = pack_bf16(exp2_approx(sc[0] - mn0), exp2_approx(sc[1] - mn1));
            const uint32_t x1 = pack_bf16(exp2_approx(sc[2] - mn0), exp2_approx(sc[3] - mn1));
            float p0, p1, p2, p3;
            unpack_bf16x2(x0, p0, p1);
            unpack_bf16x2(x1, p2, p3);
            float rs0 = p0 + p2, rs1 = p1 + p3;
#pragma unroll
            for (int o = 4; o < 32; o <<= 1) {
                rs0 += __shfl_xor_sync(0xffffffffu, rs0, o);
                rs1 += __shfl_xor_sync(0xffffffffu, rs1, o);
            }
            if (p.mode == kModeDelta) {
                // page partials from the unrounded probabilities: max logit and sum of 2^(s - max)
                float e0 = exp2_approx(sc[0] - mx0) + exp2_approx(sc[2] - mx0);
                float e1 = exp2_approx(sc[1] - mx1) + exp2_approx(sc[3] - mx1);
#pragma unroll
                for (int o = 4; o < 32; o <<= 1) {
                    e0 += __shfl_xor_sync(0xffffffffu, e0, o);
                    e1 += __shfl_xor_sync(0xffffffffu, e1, o);
                }
                const int hA = 2 * t4, hB = 2 * t4 + 1;
                if (g4 == 0 && hA < G)
                    p.page_ml[(size_t(b) * Hq + h0 + hA) * p.max_pages + lp] = make_float2(mx0, e0);
                if (g4 == 0 && hB < G)
                    p.page_ml[(size_t(b) * Hq + h0 + hB) * p.max_pages + lp] = make_float2(mx1, e1);
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
            const uint32_t pb0 = movmatrix_trans(x0), pb1 = movmatrix_trans(x1);
            if (tv < kPage) {
                // tokens past the end of the context: zero their V rows (they may hold non-finite bytes)
                uint4* vz = reinterpret_cast<uint4*>(wst + size_t(s) * S::kPage + S::kBoxes * S::kBox);
                const int nchunks = S::kBoxes * (kPage - tv) * 8;
                for (int c = lane; c < nchunks; c += 32) {
                    const int box = c / ((kPage - tv) * 8), rem = c % ((kPage - tv) * 8);
                    vz[box * (S::kBox / 16) + (tv + rem / 8) * 8 + (rem % 8)] = make_uint4(0, 0, 0, 0);
                }
                __syncwarp();
                zeroed = true;
            }
            // O^T += V^T . P^T
#pragma unroll
            for (int mt = 0; mt < KS; ++mt) {
                const int chunk = mt * 2 + v_sub;
                const uint32_t addr = vbase + (chunk >> 3) * S::kBox + v_row * 128 + (((chunk & 7) ^ (v_row & 7)) << 4);
                uint32_t a0, a1, a2, a3;
                ldmatrix_x4_trans(addr, a0, a1, a2, a3);
                mma_bf16_16816(acc[mt], a0, a1, a2, a3, pb0, pb1);
            }
        }
        __syncwarp();
        if (lane == 0 && k + STAGES < nk) {
            if (zeroed) fence_proxy_async_smem();
            issue(k + STAGES);
        }
    }
    if (failed) {
        for (int k = consumed + 1; k < min(consumed + STAGES, nk); ++k) mbar_wait(&wbar[k % STAGES], (k / STAGES) & 1);
    }

    // ---- merge the 4 warps' states of this CTA, then the splits
    __syncthreads();
    float* mo = reinterpret_cast<float*>(smem);          // [4][8][D]
    float* mml = mo + kWarps * kMaxGroup * D;            // [4][8][2]
#pragma unroll
    for (int mt = 0; mt < KS; ++mt) {
        const int d = mt * 16 + g4;
        mo[(warp * kMaxGroup + 2 * t4) * D + d] = acc[mt][0];
        mo[(warp * kMaxGroup + 2 * t4 + 1) * D + d] = acc[mt][1];
        mo[(warp * kMaxGroup + 2 * t4) * D + d + 8] = acc[mt][2];
        mo[(warp * kMaxGroup + 2 * t4 + 1) * D + d + 8] = acc[mt][3];
    }
    if (g4 == 0) {
        mml[(warp * kMaxGroup + 2 * t4) * 2 + 0] = m_run[0];
        mml[(warp * kMaxGroup + 2 * t4) * 2 + 1] = l_run[0];
        mml[(warp * kMaxGroup + 2 * t4 + 1) * 2 + 0] = m_run[1];
        mml[(warp * kMaxGroup + 2 * t4 + 1) * 2 + 1] = l_run[1];
    }
    __syncthreads();
    split_epilogue<__nv_bfloat16, D, G, kWarps>(p, smem, mo, mml, b, g, split);
}

}  // namespace delta

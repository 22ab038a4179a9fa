// Device-side fill of paged K/V pools with the counter-based generator of synth/rng.py.
//
// Holds no attention arithmetic.  Every element it writes equals, bit for bit, the host
// generator's value at the same (tensor, layer, b, kv head, position, dim) counter:
// splitmix64 finaliser of key + (counter+1)*0x9E3779B97F4A7C15, Irwin-Hall sum of the four
// 16-bit fields, one round-to-nearest single multiply, and (bf16 pools) round-to-nearest-even
// onto the upper 16 bits.
#include <cuda_runtime.h>
#include <stdint.h>

namespace {

__device__ __forceinline__ uint64_t mix64(uint64_t z) {
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
    return z ^ (z >> 31);
}

__global__ void fill_kernel(void* pool, int is_bf16, int64_t num_phys_pages, int Hkv, int D,
                            const int32_t* __restrict__ indptr, const int32_t* __restrict__ indices,
                            const int32_t* __restrict__ fill_len, uint64_t key, uint64_t hi_bits,
                            float scale) {
    const int lp = blockIdx.x, g = blockIdx.y, b = blockIdx.z;
    const int pbeg = indptr[b], npg = indptr[b + 1] - pbeg;
    if (lp >= npg) return;
    const int64_t phys = indices[pbeg + lp];
    if (phys < 0 || phys >= num_phys_pages) return;
    const int n = fill_len[b];
    // counter = hi(tensor, layer, b, g) << 28 | pos << 8 | d
    const uint64_t hi = ((hi_bits << 6 | uint64_t(b)) << 6 | uint64_t(g)) << 28;
    const size_t base = (size_t(phys) * Hkv + g) * 16 * size_t(D);
    for (int e = threadIdx.x; e < 16 * D; e += blockDim.x) {
        const int t = e / D, d = e % D;
        const int pos = lp * 16 + t;
        if (pos >= n) continue;
        const uint64_t c = hi | (uint64_t(pos) << 8) | uint64_t(d);
        const uint64_t r = mix64(key + (c + 1ull) * 0x9E3779B97F4A7C15ull);
        const int64_t s = int64_t(r & 0xFFFF) + int64_t((r >> 16) & 0xFFFF) + int64_t((r >> 32) & 0xFFFF) +
                          int64_t(r >> 48);
        const float x = __fmul_rn(float(s - 131070), scale);
        if (is_bf16) {
            uint32_t u = __float_as_uint(x);
            u = u + 0x7FFFu + ((u >> 16) & 1u);
            reinterpret_cast<uint16_t*>(pool)[base + e] = uint16_t(u >> 16);
        } else {
            reinterpret_cast<float*>(pool)[base + e] = x;
        }
    }
}

// out[l][b][g][d] = generator value of (tensor, l, b, g, pos[b], d) for layers 0..L-1: the token
// each sequence appends at this decode step.
__global__ void fill_tokens_kernel(void* out, int is_bf16, int Hkv, int D, const int32_t* __restrict__ pos,
                                   uint64_t key, int tensor, float scale) {
    const int l = blockIdx.x, b = blockIdx.y, B = gridDim.y;
    const int p = pos[b];
    for (int e = threadIdx.x; e < Hkv * D; e += blockDim.x) {
        const int g = e / D, d = e % D;
        const uint64_t hi = ((((uint64_t(tensor) << 6) | uint64_t(l)) << 6 | uint64_t(b)) << 6 | uint64_t(g)) << 28;
        const uint64_t c = hi | (uint64_t(p) << 8) | uint64_t(d);
        const uint64_t r = mix64(key + (c + 1ull) * 0x9E3779B97F4A7C15ull);
        const int64_t s = int64_t(r & 0xFFFF) + int64_t((r >> 16) & 0xFFFF) + int64_t((r >> 32) & 0xFFFF) +
                          int64_t(r >> 48);
        const float x = __fmul_rn(float(s - 131070), scale);
        const size_t o = ((size_t(l) * B + b) * Hkv + g) * D + d;
        if (is_bf16) {
            uint32_t u = __float_as_uint(x);
            u = u + 0x7FFFu + ((u >> 16) & 1u);
            reinterpret_cast<uint16_t*>(out)[o] = uint16_t(u >> 16);
        } else {
            reinterpret_cast<float*>(out)[o] = x;
        }
    }
}

}  // namespace

extern "C" int synth_fill_tokens(void* out, int is_bf16, int L, int B, int Hkv, int D, const int32_t* pos,
                                 uint64_t key, int tensor, float scale, void* stream) {
    if (out == nullptr || pos == nullptr || L <= 0 || L > 64 || B <= 0 || B > 64 || Hkv <= 0 || Hkv > 64 || D <= 0 ||
        D > 256 || tensor < 0 || tensor > 3)
        return 1;
    fill_tokens_kernel<<<dim3(L, B), 256, 0, static_cast<cudaStream_t>(stream)>>>(out, is_bf16, Hkv, D, pos, key,
                                                                                  tensor, scale);
    return cudaPeekAtLastError() == cudaSuccess ? 0 : 2;
}

extern "C" int synth_fill_kv(void* pool, int is_bf16, int64_t num_phys_pages, int Hkv, int D,
                             const int32_t* indptr, const int32_t* indices, const int32_t* fill_len,
                             int batch, int max_pages, uint64_t key, int tensor, int layer, float scale,
                             void* stream) {
    if (pool == nullptr || batch <= 0 || max_pages <= 0 || D <= 0 || D > 256 || Hkv <= 0 || Hkv > 64 ||
        batch > 64 || layer < 0 || layer >= 64 || tensor < 0 || tensor > 3)
        return 1;
    const uint64_t hi_bits = (uint64_t(tensor) << 6) | uint64_t(layer);
    fill_kernel<<<dim3(max_pages, Hkv, batch), 256, 0, static_cast<cudaStream_t>(stream)>>>(
        pool, is_bf16, num_phys_pages, Hkv, D, indptr, indices, fill_len, key, hi_bits, scale);
    return cudaPeekAtLastError() == cudaSuccess ? 0 : 2;
}

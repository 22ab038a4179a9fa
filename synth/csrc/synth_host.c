/* Host-side (CPU) copy of the counter-based generator of synth/rng.py, in plain C so that large
 * blocks of synthetic K/V values can be regenerated quickly on the host.
 *
 * Holds no attention arithmetic.  Element (tensor, layer, b, head, pos, d) has the counter
 *   hi(tensor, layer, b, head) << 28 | pos << 8 | d
 * and the value float32(S - 131070) * scale, S the sum of the four 16-bit fields of the
 * splitmix64 finaliser (Steele, Lea, Flood, OOPSLA 2014) of key + (counter + 1) * 0x9E3779B97F4A7C15,
 * optionally rounded to bfloat16 (nearest-even) and returned widened to float32.  It must equal
 * rng.normal_block (and round_to_dtype) bit for bit; tests/test_synth.py checks that.
 */
#include <stdint.h>
#include <string.h>

static inline uint64_t mix64(uint64_t z) {
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
    return z ^ (z >> 31);
}

/* out[i][d] for i < npos, d < dim: the generator value at (tensor, layer, b, head, pos[i], d). */
int synth_host_normal_block(uint64_t key, int tensor, int layer, int b, int head, const int64_t* pos, int64_t npos,
                            int dim, float scale, int round_bf16, float* out) {
    if (pos == 0 || out == 0 || dim <= 0 || dim > 256 || tensor < 0 || tensor > 3 || layer < 0 || layer >= 64 ||
        b < 0 || b >= 64 || head < 0 || head >= 64 || npos < 0)
        return 1;
    const uint64_t hi = ((((uint64_t)tensor << 6 | (uint64_t)layer) << 6 | (uint64_t)b) << 6 | (uint64_t)head) << 28;
    for (int64_t i = 0; i < npos; ++i) {
        const uint64_t p = (uint64_t)pos[i];
        if (p >= (1u << 20)) return 2;
        float* row = out + i * (int64_t)dim;
        for (int d = 0; d < dim; ++d) {
            const uint64_t c = hi | (p << 8) | (uint64_t)d;
            const uint64_t r = mix64(key + (c + 1ull) * 0x9E3779B97F4A7C15ull);
            const int64_t s = (int64_t)(r & 0xFFFF) + (int64_t)((r >> 16) & 0xFFFF) + (int64_t)((r >> 32) & 0xFFFF) +
                              (int64_t)(r >> 48);
            float x = (float)(s - 131070) * scale;   /* one IEEE single multiply, nearest */
            if (round_bf16) {
                uint32_t u;
                memcpy(&u, &x, 4);
                u = (u + 0x7FFFu + ((u >> 16) & 1u)) & 0xFFFF0000u;
                memcpy(&x, &u, 4);
            }
            row[d] = x;
        }
    }
    return 0;
}

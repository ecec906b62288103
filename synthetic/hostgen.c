/* Host C twin of the numpy generator in synthetic/__init__.py (same words,
 * same Irwin-Hall deviates, same roundings), for large tensors.  No NVFP4
 * arithmetic here.  Built with -ffp-contract=off. */
#include <stdint.h>
#include <string.h>

static const uint64_t G = 0x9E3779B97F4A7C15ull;

static uint64_t mix(uint64_t z) {
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
    return z ^ (z >> 31);
}

uint64_t hg_key(uint64_t seed, uint64_t stream) { return mix(mix(seed + G) + (stream + 1) * G); }

void hg_normal_bf16(uint64_t seed, uint64_t stream, int64_t start, int64_t count, double sigma, int scale,
                    uint16_t *out) {
    const uint64_t key = hg_key(seed, stream);
    #pragma omp parallel for schedule(static)
    for (int64_t j = 0; j < count; ++j) {
        const uint64_t base = 3ull * (uint64_t)(start + j);
        int64_t s = 0;
        for (int w = 0; w < 3; ++w) {
            uint64_t x = mix(key + (base + w + 1) * G);
            s += (int64_t)(x & 0xFFFF) + (int64_t)((x >> 16) & 0xFFFF) + (int64_t)((x >> 32) & 0xFFFF) +
                 (int64_t)(x >> 48);
        }
        double z = (double)(s - 393210) / 65536.0;
        if (scale) z = z * sigma;
        float f = (float)z;
        uint32_t b;
        memcpy(&b, &f, 4);
        out[j] = (uint16_t)((b + 0x7FFFu + ((b >> 16) & 1u)) >> 16);
    }
}

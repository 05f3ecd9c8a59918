/*
 * Seeded synthetic inputs for prefill KV-cache eviction workloads.
 *
 * This file only draws random numbers and shapes them into bf16 tensors. It holds
 * none of the eviction method's arithmetic (no attention logits, softmax, scores,
 * selection or gather); both the CUDA path's tests and the CPU oracle consume its
 * output as plain input data.
 *
 * Generator: a counter-based hash. Element e of stream s under seed S is the
 * splitmix64 finaliser (Steele, Lea, Flood, "Fast splittable pseudorandom number
 * generators", OOPSLA 2014) applied to a key built from (S, s, e). The 64 output bits
 * give two uniforms in (0,1), turned into one standard normal by the Box-Muller
 * transform (cosine branch). Values are rounded to bf16 with round-to-nearest-even.
 */
#include <math.h>
#include <stdint.h>
#include <string.h>

static inline uint64_t mix64(uint64_t z) {
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ULL;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBULL;
    return z ^ (z >> 31);
}

static inline uint64_t draw(uint64_t seed, uint64_t stream, uint64_t e) {
    uint64_t key = mix64(seed * 0x9E3779B97F4A7C15ULL + 0x632BE59BD9B4E019ULL) ^
                   mix64(stream * 0xD1B54A32D192ED03ULL + 0x8CB92BA72F3D8DD7ULL);
    return mix64(key + (e + 1) * 0x9E3779B97F4A7C15ULL);
}

static inline double normal_of(uint64_t bits) {
    const double inv32 = 1.0 / 4294967296.0;
    double u1 = ((double)(bits >> 32) + 0.5) * inv32;
    double u2 = ((double)(bits & 0xFFFFFFFFULL) + 0.5) * inv32;
    return sqrt(-2.0 * log(u1)) * cos(6.283185307179586476925286766559 * u2);
}

/* float64 -> float32 (RNE, by the C cast) -> bf16 bits (RNE). */
static inline uint16_t to_bf16(double x) {
    float f = (float)x;
    uint32_t u;
    memcpy(&u, &f, 4);
    if ((u & 0x7F800000u) == 0x7F800000u) return (uint16_t)(u >> 16); /* inf/nan: truncate */
    u += 0x7FFFu + ((u >> 16) & 1u);
    return (uint16_t)(u >> 16);
}

/* Raw 64-bit draws, exposed so tests can check the generator against its definition. */
void synth_draw_u64(uint64_t seed, uint64_t stream, uint64_t first, int64_t n, uint64_t* out) {
    for (int64_t i = 0; i < n; ++i) out[i] = draw(seed, stream, first + (uint64_t)i);
}

/*
 * Fill out[r*d + c] (r < rows, c < d) with bf16 of
 *     z(seed, stream, r*d + c) * scale[(r / rows_per_head) * d + c]
 * (scale may be NULL for 1.0). When rope_base > 0, the pair (c, c + d/2), c < d/2, of
 * every row is then rotated by the angle pos * rope_base^(-2c/d), pos = r % rows_per_head
 * (rotate-half pairing). All arithmetic in double; one rounding to bf16 at the end.
 */
void synth_normal_bf16(uint16_t* out, int64_t rows, int32_t d, uint64_t seed, uint64_t stream,
                       int64_t rows_per_head, const float* scale, double rope_base) {
    const int32_t half = d / 2;
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < rows; ++r) {
        double row[1024];
        const int64_t head = r / rows_per_head;
        const int64_t pos = r % rows_per_head;
        for (int32_t c = 0; c < d; ++c) {
            double z = normal_of(draw(seed, stream, (uint64_t)(r * d + c)));
            if (scale) z *= (double)scale[head * d + c];
            row[c] = z;
        }
        if (rope_base > 0.0) {
            for (int32_t c = 0; c < half; ++c) {
                double theta = (double)pos * pow(rope_base, -2.0 * (double)c / (double)d);
                double cs = cos(theta), sn = sin(theta);
                double x1 = row[c], x2 = row[c + half];
                row[c] = x1 * cs - x2 * sn;
                row[c + half] = x1 * sn + x2 * cs;
            }
        }
        for (int32_t c = 0; c < d; ++c) out[r * d + c] = to_bf16(row[c]);
    }
}

/* Round float64 values to bf16 bits (RNE); used for planted rows. */
void synth_round_bf16(const double* x, int64_t n, uint16_t* out) {
    for (int64_t i = 0; i < n; ++i) out[i] = to_bf16(x[i]);
}

/*
 * synth_gen.c -- seeded random inputs (no arithmetic of the method lives here).
 *
 * SplitMix64 (Steele, Lea, Flood, OOPSLA 2014) used counter-style: value i of the stream with key
 * `key` is mix(key + (i + 1) * GAMMA).  Uniforms take the top 53 bits.  Normals: Box-Muller in fp64
 * on uniforms 2i (radius) and 2i+1 (angle).  OpenMP splits the index range; every value depends
 * only on (key, i), so the output does not depend on the thread count.
 */
#include <math.h>
#include <stdint.h>

#define GAMMA 0x9E3779B97F4A7C15ull

static inline uint64_t mix(uint64_t z)
{
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
    return z ^ (z >> 31);
}

static inline double unif(uint64_t key, int64_t i)
{
    return (double)(mix(key + (uint64_t)(i + 1) * GAMMA) >> 11) * (1.0 / 9007199254740992.0);
}

void syn_u64(uint64_t key, int64_t start, int64_t n, uint64_t* out)
{
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; i++) out[i] = mix(key + (uint64_t)(start + i + 1) * GAMMA);
}

void syn_uniform(uint64_t key, int64_t n, double* out)
{
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; i++) out[i] = unif(key, i);
}

static inline double box_muller(uint64_t key, int64_t i)
{
    double u0 = unif(key, 2 * i), u1 = unif(key, 2 * i + 1);
    return sqrt(-2.0 * log1p(-u0)) * cos(6.283185307179586 * u1);
}

void syn_normal(uint64_t key, int64_t n, double* out)
{
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; i++) out[i] = box_muller(key, i);
}

/* fp32 weights: N(0, std^2), each entry times `mul` where the outlier uniform is below p. */
void syn_weights(uint64_t key_normal, uint64_t key_outlier, int64_t n, double std, double p, float mul,
                 float* out)
{
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; i++) {
        float v = (float)(box_muller(key_normal, i) * std);
        if (p > 0.0 && unif(key_outlier, i) < p) v *= mul;
        out[i] = v;
    }
}

/* fp32 standard normals scaled by `scale`. */
void syn_normal_f32(uint64_t key, int64_t n, double scale, float* out)
{
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; i++) out[i] = (float)(box_muller(key, i) * scale);
}

/* fp32 Student-t with 3 degrees of freedom: Z / sqrt(chi2_3 / 3), chi2_3 from three more normals. */
void syn_student_t3_f32(uint64_t kz, uint64_t k0, uint64_t k1, uint64_t k2, int64_t n, float* out)
{
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; i++) {
        double a = box_muller(k0, i), b = box_muller(k1, i), c = box_muller(k2, i);
        out[i] = (float)(box_muller(kz, i) / sqrt((a * a + b * b + c * c) / 3.0));
    }
}

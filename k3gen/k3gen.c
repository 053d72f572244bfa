/*
 * k3gen: seeded synthetic inputs for the MXFP4 routed-expert MoE layer.
 *
 * This module only draws numbers and lays bytes out; it holds none of the
 * layer's arithmetic (no E2M1/E8M0 decode, no matvec, no softmax).  Both the
 * fp64 oracle and the CUDA path take their inputs from here.
 *
 * Generator: a counter-based SplitMix64 (Steele, Lea and Flood, "Fast
 * splittable pseudorandom number generators", OOPSLA 2014).  For a (seed,
 * stream) pair the base state is
 *     base = mix64(seed ^ mix64(stream * C1 + C2))
 * and the i-th 64-bit draw is the i-th output of SplitMix64 started at base:
 *     draw(i) = mix64(base + (i + 1) * GAMMA)
 * so any element can be produced independently of the others (OpenMP-safe).
 *
 * Streams: 0 = hidden states x, 1 = router weights, 2 = router bias,
 *          3 = expert nibble bytes, 4 = expert E8M0 scale bytes,
 *          5 = shared-expert weights, 6 = Zipf rank permutation.
 */
#include <math.h>
#include <stdint.h>
#include <string.h>

#define GAMMA 0x9E3779B97F4A7C15ULL
#define C1 0xD1B54A32D192ED03ULL
#define C2 0x8CB92BA72F3D8DD7ULL

static inline uint64_t mix64(uint64_t z) {
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ULL;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBULL;
    return z ^ (z >> 31);
}

uint64_t k3gen_base(uint64_t seed, uint64_t stream) {
    return mix64(seed ^ mix64(stream * C1 + C2));
}

static inline uint64_t draw(uint64_t base, uint64_t i) {
    return mix64(base + (i + 1) * GAMMA);
}

uint64_t k3gen_draw(uint64_t seed, uint64_t stream, uint64_t i) {
    return draw(k3gen_base(seed, stream), i);
}

/* uniform in [0,1) with 53 random bits */
static inline double unif(uint64_t base, uint64_t i) {
    return (double)(draw(base, i) >> 11) * 0x1.0p-53;
}

/* standard normal number i of a stream: Box-Muller on draws 2i and 2i+1 */
static inline double normal_at(uint64_t base, uint64_t i) {
    double u1 = (double)((draw(base, 2 * i) >> 11) + 1) * 0x1.0p-53; /* (0,1] */
    double u2 = unif(base, 2 * i + 1);
    return sqrt(-2.0 * log(u1)) * cos(6.283185307179586476925286766559 * u2);
}

double k3gen_normal(uint64_t seed, uint64_t stream, uint64_t i) {
    return normal_at(k3gen_base(seed, stream), i);
}

/* round a double to bfloat16 bits, nearest-even, in one step (normal range) */
uint16_t k3gen_bf16_bits(double v) {
    if (v == 0.0 || isnan(v) || isinf(v)) {
        float f = (float)v;
        uint32_t b;
        memcpy(&b, &f, 4);
        return (uint16_t)(b >> 16);
    }
    int e;
    double m = frexp(fabs(v), &e);           /* m in [0.5, 1) */
    double r = nearbyint(ldexp(m, 8));       /* 8 significant bits, ties to even */
    float f = (float)ldexp(r, e - 8);        /* exact in float */
    uint32_t b;
    memcpy(&b, &f, 4);
    uint16_t h = (uint16_t)(b >> 16);
    if (v < 0) h |= 0x8000u;
    return h;
}

void k3gen_normal_bf16(uint64_t seed, uint64_t stream, uint64_t offset, uint64_t n,
                       double scale, uint16_t *out) {
    uint64_t base = k3gen_base(seed, stream);
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < (int64_t)n; ++i)
        out[i] = k3gen_bf16_bits(scale * normal_at(base, offset + (uint64_t)i));
}

void k3gen_normal_f32(uint64_t seed, uint64_t stream, uint64_t offset, uint64_t n,
                      double scale, float *out) {
    uint64_t base = k3gen_base(seed, stream);
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < (int64_t)n; ++i)
        out[i] = (float)(scale * normal_at(base, offset + (uint64_t)i));
}

/* byte j of the stream = byte (j & 7) of draw(j >> 3), little-endian */
void k3gen_uniform_bytes(uint64_t seed, uint64_t stream, uint64_t offset, uint64_t n,
                         uint8_t *out) {
    uint64_t base = k3gen_base(seed, stream);
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < (int64_t)n; ++i) {
        uint64_t j = offset + (uint64_t)i;
        out[i] = (uint8_t)(draw(base, j >> 3) >> (8 * (j & 7)));
    }
}

/* lo + floor(count * hi32(draw(j)) / 2^32): integers uniform in [lo, lo+count) */
void k3gen_uniform_range_u8(uint64_t seed, uint64_t stream, uint64_t offset, uint64_t n,
                            uint32_t lo, uint32_t count, uint8_t *out) {
    uint64_t base = k3gen_base(seed, stream);
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < (int64_t)n; ++i) {
        uint64_t hi = draw(base, offset + (uint64_t)i) >> 32;
        out[i] = (uint8_t)(lo + ((hi * count) >> 32));
    }
}

/*
 * Zipf prior on the router: a seeded permutation (Fisher-Yates, draws from
 * `stream`) gives each expert a rank r in 1..E; bias[e] = -s * ln(r_e), so the
 * softmax prior of expert e is proportional to r_e^(-s).
 */
int k3gen_zipf_bias(uint64_t seed, uint64_t stream, int32_t E, double s, float *out,
                    int32_t *rank_out) {
    uint64_t base = k3gen_base(seed, stream);
    int32_t perm[8192];
    if (E < 1 || E > 8192) return -1;
    for (int32_t i = 0; i < E; ++i) perm[i] = i;
    uint64_t c = 0;
    for (int32_t i = E - 1; i >= 1; --i) {
        uint64_t hi = draw(base, c++) >> 32;
        int32_t j = (int32_t)((hi * (uint64_t)(i + 1)) >> 32);
        int32_t t = perm[i];
        perm[i] = perm[j];
        perm[j] = t;
    }
    for (int32_t i = 0; i < E; ++i) {
        int32_t e = perm[i];
        int32_t r = i + 1;
        out[e] = (float)(-s * log((double)r));
        if (rank_out) rank_out[e] = r;
    }
    return 0;
}

/*
 * One routed expert's blob, planes in the order
 *   [W_g nibbles | W_g scales | W_u nibbles | W_u scales | W_d nibbles | W_d scales]
 * W_g, W_u are [ff rows][d cols], W_d is [d rows][ff cols]; a nibble plane has
 * rows*cols/2 bytes, a scale plane rows*cols/32 bytes.  Nibble bytes are
 * uniform 0..255 (two uniform nibbles), scale bytes uniform in
 * [scale_lo, scale_lo + scale_count).  Matrix m of expert e draws from
 * counter offset ((e*3 + m) << 36) in streams 3 (nibbles) and 4 (scales).
 */
uint64_t k3gen_blob_bytes(int64_t d, int64_t ff) { return (uint64_t)(3 * d * ff * 17 / 32); }

void k3gen_expert_blob(uint64_t seed, int64_t e, int64_t d, int64_t ff, uint32_t scale_lo,
                       uint32_t scale_count, uint8_t *out) {
    uint64_t mat = (uint64_t)d * (uint64_t)ff;
    uint8_t *p = out;
    for (int m = 0; m < 3; ++m) {
        uint64_t off = ((uint64_t)(e * 3 + m)) << 36;
        k3gen_uniform_bytes(seed, 3, off, mat / 2, p);
        p += mat / 2;
        k3gen_uniform_range_u8(seed, 4, off, mat / 32, scale_lo, scale_count, p);
        p += mat / 32;
    }
}

/*
 * Shared expert, bf16: W_g,s and W_u,s [ff_s][d], W_d,s [d][ff_s], entries
 * bf16(sigma * N(0,1)); matrix m draws stream 5 from offset (m << 40).
 */
void k3gen_shared(uint64_t seed, int64_t d, int64_t ffs, double sigma, uint16_t *wg,
                  uint16_t *wu, uint16_t *wd) {
    uint64_t n = (uint64_t)d * (uint64_t)ffs;
    k3gen_normal_bf16(seed, 5, 0ull << 40, n, sigma, wg);
    k3gen_normal_bf16(seed, 5, 1ull << 40, n, sigma, wu);
    k3gen_normal_bf16(seed, 5, 2ull << 40, n, sigma, wd);
}

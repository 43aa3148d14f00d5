/*
 * Seeded synthetic inputs for the packed MiniMax-H3 attention call.
 *
 * This module holds the input recipe only: counter-based random numbers,
 * the per-frame cluster means and bf16 rounding.  It contains none of the
 * attention method's arithmetic, and both the oracle-side tests and the GPU
 * path draw their inputs from it.
 *
 * Counter-based generator: every element is a pure function of
 * (seed, tensor id, head, row, column), so any sampled row can be
 * regenerated without producing the whole tensor.
 *   h = mix(mix(mix(mix(seed ^ SALT[tensor]) + head) + row) + col)
 * where mix() is the splitmix64 finaliser (Steele, Lea, Flood,
 * "Fast splittable pseudorandom number generators", OOPSLA 2014).
 * A standard normal is formed from the two 32-bit halves of h with the
 * Box-Muller transform (Box & Muller 1958) in double precision.
 *
 * Cluster means: for every (head, segment, latent frame) with a frame id
 * >= 0, g ~ N(0, I_d) is drawn with tensor id CLUSTER and counter
 * (head, segment * 65536 + frame, column); c = norm * g / |g|.  The same c
 * is added to the Q and the K rows of that frame; V gets no mean.
 *
 * Rounding: value (double) -> float (round to nearest even) -> bf16
 * (round to nearest even on the float bits).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

static const uint64_t SALT[4] = {
    0x51ULL * 0x9E3779B97F4A7C15ULL,  /* Q */
    0x4BULL * 0x9E3779B97F4A7C15ULL,  /* K */
    0x56ULL * 0x9E3779B97F4A7C15ULL,  /* V */
    0x43ULL * 0x9E3779B97F4A7C15ULL,  /* cluster means */
};

static inline uint64_t mix64(uint64_t z) {
    z += 0x9E3779B97F4A7C15ULL;
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ULL;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBULL;
    return z ^ (z >> 31);
}

static inline uint64_t counter_hash(uint64_t seed, int tensor, uint64_t a,
                                    uint64_t b, uint64_t c) {
    uint64_t z = mix64(seed ^ SALT[tensor]);
    z = mix64(z + a);
    z = mix64(z + b);
    return mix64(z + c);
}

static inline double normal_from_hash(uint64_t h) {
    const double two32 = 4294967296.0;
    double u1 = ((double)(uint32_t)(h >> 32) + 0.5) / two32; /* (0,1) */
    double u2 = (double)(uint32_t)h / two32;                  /* [0,1) */
    return sqrt(-2.0 * log(u1)) * cos(6.283185307179586476925 * u2);
}

/* float -> bf16 bits, round to nearest even (finite inputs only). */
static inline uint16_t bf16_rne(float f) {
    uint32_t u;
    memcpy(&u, &f, 4);
    uint32_t lsb = (u >> 16) & 1u;
    u += 0x7FFFu + lsb;
    return (uint16_t)(u >> 16);
}

/* One standard normal for element (tensor, head, row, col). */
double gen_normal(uint64_t seed, int tensor, int head, int64_t row, int col) {
    return normal_from_hash(counter_hash(seed, tensor, (uint64_t)head,
                                         (uint64_t)row, (uint64_t)col));
}

/* Cluster mean vector c (length d) of (head, segment, frame). */
void gen_cluster(uint64_t seed, int head, int segment, int frame, int d,
                 double norm, double *c) {
    double ss = 0.0;
    uint64_t key = (uint64_t)segment * 65536ULL + (uint64_t)frame;
    for (int j = 0; j < d; ++j) {
        c[j] = normal_from_hash(counter_hash(seed, 3, (uint64_t)head, key,
                                             (uint64_t)j));
        ss += c[j] * c[j];
    }
    double s = norm / sqrt(ss);
    for (int j = 0; j < d; ++j) c[j] *= s;
}

/*
 * Fill out[(h - h0)][(r - row0)][:] (bf16 bits) for heads [h0, h0 + nh) and
 * rows [row0, row0 + nrows) of tensor `tensor` (0 Q, 1 K, 2 V).
 * seg[S] and frame[S] describe every row of the sequence (frame < 0: no
 * cluster mean).  cluster_norm <= 0 disables the means.  Cluster means are
 * applied to Q and K only.
 */
void gen_tensor(uint64_t seed, int tensor, int S, int d, const uint8_t *seg,
                const int32_t *frame, double cluster_norm, int h0, int nh,
                int64_t row0, int64_t nrows, uint16_t *out) {
    int use_cluster = (cluster_norm > 0.0) && (tensor == 0 || tensor == 1);
    int64_t total = (int64_t)nh * nrows;
#pragma omp parallel
    {
        double *c = (double *)malloc(sizeof(double) * (size_t)d);
        int c_head = -1, c_seg = -1, c_frame = -1;
#pragma omp for schedule(static)
        for (int64_t t = 0; t < total; ++t) {
            int h = h0 + (int)(t / nrows);
            int64_t r = row0 + t % nrows;
            uint16_t *dst = out + (size_t)t * (size_t)d;
            int has_c = 0;
            if (use_cluster && r < S && frame[r] >= 0) {
                if (h != c_head || seg[r] != c_seg || frame[r] != c_frame) {
                    gen_cluster(seed, h, seg[r], frame[r], d, cluster_norm, c);
                    c_head = h;
                    c_seg = seg[r];
                    c_frame = frame[r];
                }
                has_c = 1;
            }
            for (int j = 0; j < d; ++j) {
                double z = gen_normal(seed, tensor, h, r, j);
                if (has_c) z += c[j];
                dst[j] = bf16_rne((float)z);
            }
        }
        free(c);
    }
}

int gen_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

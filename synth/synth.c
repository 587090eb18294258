/*
 * Seeded synthetic inputs for NABLA-style block-sparse attention on 3D video
 * token grids.
 *
 * This file generates input data only: it holds none of the method's
 * arithmetic (no pooling, softmax, selection or attention).  Both the fp64
 * oracle and the CUDA path are fed from it.
 *
 * Random numbers: a counter-based SplitMix64 stream (Steele, Lea and Flood,
 * "Fast splittable pseudorandom number generators", OOPSLA 2014; the 64-bit
 * finaliser constants are the ones Vigna published for splitmix64.c).  Output
 * i of a generator seeded with `key` is mix(key + (i+1)*gamma), so every
 * element can be drawn independently of thread count.  Gaussians come from
 * the Box-Muller transform in fp64.
 *
 * Layouts: Q, K, V are [B, H, S, d] row-major; tokens are ordered tile-major
 * (64-token tiles of 4x4x4 in (t, h, w) raster order over the tile grid, and
 * (t, h, w) raster order inside a tile).  Values are rounded to bf16 with
 * round-to-nearest-even after a round-to-nearest conversion to fp32.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define SM_GAMMA 0x9E3779B97F4A7C15ULL

static inline uint64_t sm_mix(uint64_t z) {
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ULL;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBULL;
    return z ^ (z >> 31);
}

/* Output number i (0-based) of a SplitMix64 generator whose state starts at key. */
uint64_t synth_splitmix64_at(uint64_t key, uint64_t i) {
    return sm_mix(key + (i + 1) * SM_GAMMA);
}

/* Stream key of one tensor: output `tensor_id` of the generator seeded with `seed`. */
uint64_t synth_tensor_key(uint64_t seed, int tensor_id) {
    return synth_splitmix64_at(seed, (uint64_t)tensor_id);
}

/* Uniform in the open interval (0, 1): the top 53 bits, centred in their cell. */
static inline double sm_uniform(uint64_t key, uint64_t i) {
    return ((double)(synth_splitmix64_at(key, i) >> 11) + 0.5) * 0x1.0p-53;
}

double synth_uniform_at(uint64_t key, uint64_t i) { return sm_uniform(key, i); }

/* Standard normal for flat element index `flat`: elements 2k and 2k+1 share
 * the Box-Muller pair built from uniforms 2k and 2k+1 (cos for even, sin for odd). */
static inline double sm_normal(uint64_t key, uint64_t flat) {
    uint64_t k = flat >> 1;
    double u1 = sm_uniform(key, 2 * k);
    double u2 = sm_uniform(key, 2 * k + 1);
    double r = sqrt(-2.0 * log(u1));
    double th = 6.283185307179586476925286766559 * u2;
    return (flat & 1) ? r * sin(th) : r * cos(th);
}

double synth_normal_at(uint64_t key, uint64_t flat) { return sm_normal(key, flat); }

uint16_t synth_f64_to_bf16(double x) {
    float f = (float)x;
    uint32_t u;
    memcpy(&u, &f, 4);
    if ((u & 0x7F800000u) == 0x7F800000u) return (uint16_t)(u >> 16); /* inf/nan: truncate */
    u += 0x7FFFu + ((u >> 16) & 1u);
    return (uint16_t)(u >> 16);
}

/* Token coordinates (t, h, w) of token s in tile-major order on a tile grid
 * of Tt x Th x Tw tiles, each tile 4 x 4 x 4 tokens. */
void synth_token_coords(int64_t s, int Tt, int Th, int Tw, int* t, int* h, int* w) {
    (void)Tt;
    int64_t tile = s / 64, u = s % 64;
    int tw = (int)(tile % Tw), th = (int)((tile / Tw) % Th), tt = (int)(tile / ((int64_t)Tw * Th));
    int uw = (int)(u % 4), uh = (int)((u / 4) % 4), ut = (int)(u / 16);
    *t = 4 * tt + ut;
    *h = 4 * th + uh;
    *w = 4 * tw + uw;
}

/* 3D sinusoidal embedding of dim d at token coordinates (t, h, w).
 * Channel pair i (channels 2i, 2i+1) belongs to axis a = i mod 3 (t, h, w),
 * frequency index k = i div 3, and n_a = number of pairs on axis a;
 * omega = 10000^(-k / n_a); channel 2i = sin(pos_a * omega), 2i+1 = cos(...). */
void synth_embedding(int d, int t, int h, int w, double* e) {
    int npairs = d / 2;
    int pos[3] = {t, h, w};
    for (int i = 0; i < npairs; ++i) {
        int a = i % 3, k = i / 3;
        int n_a = (npairs - a + 2) / 3;
        double omega = pow(10000.0, -(double)k / (double)n_a);
        double arg = (double)pos[a] * omega;
        e[2 * i] = sin(arg);
        e[2 * i + 1] = cos(arg);
    }
}

/* Fill one [B, H, S, d] bf16 tensor: x = pos_weight * e(t,h,w) + noise_weight * z,
 * z ~ N(0,1) from stream `tensor_id` (0 = Q, 1 = K, 2 = V by convention).
 * pos_weight == 0 skips the embedding (the grid arguments are then unused). */
int synth_fill_tensor(uint16_t* out, int tensor_id, uint64_t seed, int B, int H, int64_t S, int d,
                      int Tt, int Th, int Tw, double pos_weight, double noise_weight) {
    if (!out || B <= 0 || H <= 0 || S <= 0 || d <= 0 || (d & 1)) return -1;
    int use_emb = pos_weight != 0.0;
    if (use_emb && (S % 64 != 0 || (int64_t)Tt * Th * Tw * 64 != S)) return -2;
    uint64_t key = synth_tensor_key(seed, tensor_id);
    /* Embedding table per (axis coordinate, channel): e depends on one axis per channel. */
    int maxpos = use_emb ? 4 * (Tt > Th ? (Tt > Tw ? Tt : Tw) : (Th > Tw ? Th : Tw)) : 1;
    double* table = (double*)malloc(sizeof(double) * (size_t)maxpos * d);
    if (!table) return -3;
    if (use_emb) {
        double* e = (double*)malloc(sizeof(double) * d);
        for (int p = 0; p < maxpos; ++p) {
            synth_embedding(d, p, p, p, e);
            memcpy(table + (size_t)p * d, e, sizeof(double) * d);
        }
        free(e);
    }
    int64_t rows = (int64_t)B * H * S;
#pragma omp parallel for schedule(static)
    for (int64_t row = 0; row < rows; ++row) {
        int64_t s = row % S;
        int crd[3] = {0, 0, 0};
        if (use_emb) synth_token_coords(s, Tt, Th, Tw, &crd[0], &crd[1], &crd[2]);
        uint64_t base = (uint64_t)row * (uint64_t)d;
        for (int c = 0; c < d; c += 2) {
            /* one Box-Muller pair serves channels c and c+1 */
            uint64_t k = (base + (uint64_t)c) >> 1;
            double u1 = sm_uniform(key, 2 * k), u2 = sm_uniform(key, 2 * k + 1);
            double r = sqrt(-2.0 * log(u1));
            double th = 6.283185307179586476925286766559 * u2;
            double z0 = r * cos(th), z1 = r * sin(th);
            double e0 = 0.0, e1 = 0.0;
            if (use_emb) {
                int a = (c / 2) % 3;
                e0 = table[(size_t)crd[a] * d + c];
                e1 = table[(size_t)crd[a] * d + c + 1];
            }
            out[base + c] = synth_f64_to_bf16(pos_weight * e0 + noise_weight * z0);
            out[base + c + 1] = synth_f64_to_bf16(pos_weight * e1 + noise_weight * z1);
        }
    }
    free(table);
    return 0;
}

/* Per-head static block masks, i.i.d. Bernoulli(p) per (bh, r, c) entry from
 * stream `tensor_id`, with the diagonal block forced on when force_diag != 0.
 * out is [BH, nb, nb] uint8 (1 = keep). */
int synth_fill_bernoulli_mask(uint8_t* out, int tensor_id, uint64_t seed, int64_t BH, int nb,
                              double p, int force_diag) {
    if (!out || BH <= 0 || nb <= 0) return -1;
    uint64_t key = synth_tensor_key(seed, tensor_id);
    int64_t rows = BH * nb;
#pragma omp parallel for schedule(static)
    for (int64_t row = 0; row < rows; ++row) {
        int r = (int)(row % nb);
        for (int c = 0; c < nb; ++c) {
            uint64_t flat = (uint64_t)row * (uint64_t)nb + (uint64_t)c;
            uint8_t keep = sm_uniform(key, flat) < p;
            if (force_diag && r == c) keep = 1;
            out[flat] = keep;
        }
    }
    return 0;
}

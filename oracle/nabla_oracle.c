/*
 * fp64 CPU oracle for NABLA block-mask building and masked softmax attention.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the tests, the package's smoke check and the
 * bench's CPU-baseline leg may load this library.  It shares no code with the
 * CUDA path: plain loops, fp64 throughout, no blocking or fusion beyond what the
 * definitions state.  Inputs are bf16 bit patterns (uint16), widened exactly.
 *
 * Sources (page titles and sections):
 *  - "NABLA: Neighborhood Adaptive Block-Level Attention" (machine review on
 *    pith.science), "What carries the argument" and "Core claim": Algorithm 1
 *    average-pools Q and K over N-token blocks, takes a softmax over the S/N x
 *    S/N reduced map, sorts each row, forms the cumulative sum and keeps the
 *    smallest prefix of sorted entries whose mass reaches 1 - thr; the mask is
 *    optionally OR-ed with a sliding-tile (STA) mask.  Referee report, minor
 *    comment 2: sort and cumsum run along the key-block axis and "reorder"
 *    returns the flags to block order.
 *  - "Fast Video Generation with Sliding Tile Attention" (blog notes): queries
 *    of one tile attend to the key tiles in a common local window, with the
 *    tile equal to the attention block.
 *  - FlashAttention abstract: attention is exact softmax(QK^T) V; the block
 *    sparse extension computes it over the kept blocks only.
 *
 * Readings where the pages are silent (each is listed in the design notes):
 *  - block size N = 64 (one 4x4x4 tile); the reduced map is scaled by 1/sqrt(d);
 *  - ties in the sorted row go to the lower block index;
 *  - keep sorted position k iff k == 0 or the exclusive prefix sum E_k < 1-thr
 *    (so the argmax is always kept), and thr <= 0 keeps every block;
 *  - the STA window is clipped at the grid edge (no shifted centre);
 *  - LSE is the natural log of sum exp(scale * q.k) over kept keys; a row with
 *    no kept key has O = 0 and LSE = -inf.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORACLE_BLOCK 64

static double bf16_to_f64(uint16_t b) {
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, 4);
    return (double)f;
}

/* Block mean-pool (Algorithm 1, reshape to [.., S/N, N, d] and average over N).
 * x: [BH, S, d] bf16 bits; out: [BH, S/64, d]. */
void oracle_pool(const uint16_t* x, int64_t BH, int64_t S, int d, double* out) {
    int64_t nb = S / ORACLE_BLOCK;
#pragma omp parallel for schedule(static)
    for (int64_t br = 0; br < BH * nb; ++br) {
        int64_t bh = br / nb, r = br % nb;
        for (int c = 0; c < d; ++c) {
            double s = 0.0;
            for (int t = 0; t < ORACLE_BLOCK; ++t)
                s += bf16_to_f64(x[((bh * S) + r * ORACLE_BLOCK + t) * d + c]);
            out[br * d + c] = s / ORACLE_BLOCK;
        }
    }
}

/* Reduced map of one head: L[r][c] = qbar_r . kbar_c / sqrt(d). */
void oracle_logits(const double* qbar, const double* kbar, int nb, int d, double* L) {
    double inv = 1.0 / sqrt((double)d);
    for (int r = 0; r < nb; ++r)
        for (int c = 0; c < nb; ++c) {
            double s = 0.0;
            for (int k = 0; k < d; ++k) s += qbar[(int64_t)r * d + k] * kbar[(int64_t)c * d + k];
            L[(int64_t)r * nb + c] = s * inv;
        }
}

/* Row softmax with the maximum subtracted first. */
void oracle_softmax_row(const double* L, int n, double* P) {
    double m = -INFINITY;
    for (int c = 0; c < n; ++c) m = L[c] > m ? L[c] : m;
    double z = 0.0;
    for (int c = 0; c < n; ++c) z += exp(L[c] - m);
    for (int c = 0; c < n; ++c) P[c] = exp(L[c] - m) / z;
}

typedef struct { double p; int idx; } pv_t;

/* Descending probability; equal probabilities go to the lower block index. */
static int cmp_desc(const void* a, const void* b) {
    const pv_t* x = (const pv_t*)a;
    const pv_t* y = (const pv_t*)b;
    if (x->p > y->p) return -1;
    if (x->p < y->p) return 1;
    return (x->idx > y->idx) - (x->idx < y->idx);
}

/* CDF binarisation of one softmax row (Algorithm 1: sort, cumsum, threshold at
 * 1 - thr, reorder).  keep[c] is set to 0/1 for c in [0, n).  Returns the kept
 * count.  diag (may be NULL) receives, for the last kept sorted position k*:
 *   diag[0] = E_{k*}   (exclusive prefix sum before k*),
 *   diag[1] = E_{k*+1} (inclusive sum through k*),
 *   diag[2] = p at k*,  diag[3] = p at k*+1 (or -1 when k* is the last). */
int oracle_row_select(const double* p, int n, double thr, uint8_t* keep, double* diag) {
    pv_t* v = (pv_t*)malloc(sizeof(pv_t) * (size_t)n);
    for (int c = 0; c < n; ++c) { v[c].p = p[c]; v[c].idx = c; keep[c] = 0; }
    qsort(v, (size_t)n, sizeof(pv_t), cmp_desc);
    double target = 1.0 - thr;
    double E = 0.0, E_star = 0.0;
    int kstar = 0, count = 0;
    for (int k = 0; k < n; ++k) {
        int take = (thr <= 0.0) || k == 0 || E < target;
        if (!take) break;
        keep[v[k].idx] = 1;   /* "reorder": the flag goes back to the block's own index */
        ++count;
        kstar = k;
        E_star = E;
        E += v[k].p;
    }
    if (diag) {
        diag[0] = E_star;
        diag[1] = E_star + v[kstar].p;
        diag[2] = v[kstar].p;
        diag[3] = (kstar + 1 < n) ? v[kstar + 1].p : -1.0;
    }
    free(v);
    return count;
}

/* Fixed-budget baseline (NABLA review, "What carries the argument": Appendix C
 * compares the mass rule with keeping a fixed Top-k of blocks per row): keep
 * the k entries that come first in the descending order (ties: lower block
 * index).  Returns the kept count, min(k, n). */
int oracle_row_select_topk(const double* p, int n, int k, uint8_t* keep, double* diag) {
    pv_t* v = (pv_t*)malloc(sizeof(pv_t) * (size_t)n);
    for (int c = 0; c < n; ++c) { v[c].p = p[c]; v[c].idx = c; keep[c] = 0; }
    qsort(v, (size_t)n, sizeof(pv_t), cmp_desc);
    int count = 0;
    for (int j = 0; j < n && j < k; ++j) { keep[v[j].idx] = 1; ++count; }
    if (diag) {   /* no mass cut; probabilities at the last kept and first dropped position */
        diag[0] = diag[1] = -1.0;
        diag[2] = v[count - 1].p;
        diag[3] = (count < n) ? v[count].p : -1.0;
    }
    free(v);
    return count;
}

/* OR the sliding-tile window of query tile r into one mask row (tile
 * coordinates; the window is clipped to the grid). */
void oracle_sta_or(uint8_t* row, int r, int Tt, int Th, int Tw, int wt, int wh, int ww) {
    int rt = r / (Th * Tw), rh = (r / Tw) % Th, rw = r % Tw;
    for (int c = 0; c < Tt * Th * Tw; ++c) {
        int ct = c / (Th * Tw), ch = (c / Tw) % Th, cw = c % Tw;
        if (abs(ct - rt) <= wt && abs(ch - rh) <= wh && abs(cw - rw) <= ww) row[c] = 1;
    }
}

/* Full mask builder: q, k [BH, S, d] bf16 bits -> mask [BH, nb, nb] uint8.
 * topk > 0 selects the fixed top-k rule in place of the mass rule.
 * diag (may be NULL): [BH, nb, 4] as in oracle_row_select (before the STA OR).
 * adaptive_counts (may be NULL): [BH, nb] kept count before the STA OR. */
void oracle_build_mask(const uint16_t* q, const uint16_t* k, int64_t BH, int64_t S, int d,
                       int Tt, int Th, int Tw, double thr, int topk, int use_sta, int wt, int wh,
                       int ww, uint8_t* mask, double* diag, int32_t* adaptive_counts) {
    int nb = (int)(S / ORACLE_BLOCK);
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t bh = 0; bh < BH; ++bh) {
        double* qbar = (double*)malloc(sizeof(double) * (size_t)nb * d);
        double* kbar = (double*)malloc(sizeof(double) * (size_t)nb * d);
        double* L = (double*)malloc(sizeof(double) * (size_t)nb * nb);
        double* P = (double*)malloc(sizeof(double) * (size_t)nb);
        oracle_pool(q + bh * S * d, 1, S, d, qbar);
        oracle_pool(k + bh * S * d, 1, S, d, kbar);
        oracle_logits(qbar, kbar, nb, d, L);
        for (int r = 0; r < nb; ++r) {
            uint8_t* row = mask + (bh * nb + r) * (int64_t)nb;
            oracle_softmax_row(L + (int64_t)r * nb, nb, P);
            int cnt;
            if (topk > 0) {
                cnt = oracle_row_select_topk(P, nb, topk, row, diag ? diag + (bh * nb + r) * 4 : NULL);
            } else {
                cnt = oracle_row_select(P, nb, thr, row, diag ? diag + (bh * nb + r) * 4 : NULL);
            }
            if (adaptive_counts) adaptive_counts[bh * nb + r] = cnt;
            if (use_sta) oracle_sta_or(row, r, Tt, Th, Tw, wt, wh, ww);
        }
        free(qbar); free(kbar); free(L); free(P);
    }
}

/* Masked softmax attention for a list of query rows.
 * q, k, v: [BH, S, d] bf16 bits; mask: [BH, nb, nb] uint8 (block keep flags).
 * rows: global row ids bh*S + i.  O: [nrows, d]; LSE: [nrows] (natural log).
 * s_ij = scale * q_i . k_j over keys j in kept blocks of row i's block. */
void oracle_masked_attention(const uint16_t* q, const uint16_t* k, const uint16_t* v,
                             int64_t BH, int64_t S, int d, const uint8_t* mask, double scale,
                             int64_t nrows, const int64_t* rows, double* O, double* LSE) {
    int64_t nb = S / ORACLE_BLOCK;
    (void)BH;
#pragma omp parallel for schedule(dynamic, 4)
    for (int64_t n = 0; n < nrows; ++n) {
        int64_t g = rows[n], bh = g / S, i = g % S, r = i / ORACLE_BLOCK;
        const uint8_t* mrow = mask + (bh * nb + r) * nb;
        double* qi = (double*)malloc(sizeof(double) * d);
        double* acc = (double*)calloc((size_t)d, sizeof(double));
        double* s = (double*)malloc(sizeof(double) * (size_t)S);
        for (int c = 0; c < d; ++c) qi[c] = bf16_to_f64(q[(bh * S + i) * d + c]);
        double m = -INFINITY;
        int64_t nk = 0;
        for (int64_t cb = 0; cb < nb; ++cb) {
            if (!mrow[cb]) continue;
            for (int64_t j = cb * ORACLE_BLOCK; j < (cb + 1) * ORACLE_BLOCK; ++j) {
                double dot = 0.0;
                for (int c = 0; c < d; ++c) dot += qi[c] * bf16_to_f64(k[(bh * S + j) * d + c]);
                s[j] = scale * dot;
                if (s[j] > m) m = s[j];
                ++nk;
            }
        }
        if (nk == 0) {
            for (int c = 0; c < d; ++c) O[n * d + c] = 0.0;
            LSE[n] = -INFINITY;
        } else {
            double l = 0.0;
            for (int64_t cb = 0; cb < nb; ++cb) {
                if (!mrow[cb]) continue;
                for (int64_t j = cb * ORACLE_BLOCK; j < (cb + 1) * ORACLE_BLOCK; ++j) {
                    double w = exp(s[j] - m);
                    l += w;
                    for (int c = 0; c < d; ++c) acc[c] += w * bf16_to_f64(v[(bh * S + j) * d + c]);
                }
            }
            for (int c = 0; c < d; ++c) O[n * d + c] = acc[c] / l;
            LSE[n] = m + log(l);
        }
        free(qi); free(acc); free(s);
    }
}

/* Dense softmax attention (every key of the head) for the self-checks. */
void oracle_dense_attention(const uint16_t* q, const uint16_t* k, const uint16_t* v, int64_t BH,
                            int64_t S, int d, double scale, int64_t nrows, const int64_t* rows,
                            double* O, double* LSE) {
    (void)BH;
#pragma omp parallel for schedule(dynamic, 4)
    for (int64_t n = 0; n < nrows; ++n) {
        int64_t g = rows[n], bh = g / S, i = g % S;
        double* s = (double*)malloc(sizeof(double) * (size_t)S);
        double m = -INFINITY;
        for (int64_t j = 0; j < S; ++j) {
            double dot = 0.0;
            for (int c = 0; c < d; ++c)
                dot += bf16_to_f64(q[(bh * S + i) * d + c]) * bf16_to_f64(k[(bh * S + j) * d + c]);
            s[j] = scale * dot;
            if (s[j] > m) m = s[j];
        }
        double l = 0.0;
        for (int c = 0; c < d; ++c) O[n * d + c] = 0.0;
        for (int64_t j = 0; j < S; ++j) {
            double w = exp(s[j] - m);
            l += w;
            for (int c = 0; c < d; ++c) O[n * d + c] += w * bf16_to_f64(v[(bh * S + j) * d + c]);
        }
        for (int c = 0; c < d; ++c) O[n * d + c] /= l;
        LSE[n] = m + log(l);
        free(s);
    }
}

/* Token reordering (NABLA review, Figure 4: neighbouring tokens are gathered
 * so that each attention block is one spatial-temporal patch; here the patch
 * is the 4x4x4 tile).  For every token (t, h, w) of the 4Tt x 4Th x 4Tw grid:
 * raster position (t*H + h)*W + w, tile-major position
 * ((t/4*Th + h/4)*Tw + w/4)*64 + ((t%4)*4 + h%4)*4 + w%4.
 * to_tile_major = 1 moves raster rows to tile-major rows, 0 the reverse.
 * src, dst: [BH, S, d] 16-bit rows (copied bit for bit). */
void oracle_reorder(const uint16_t* src, uint16_t* dst, int64_t BH, int Tt, int Th, int Tw, int d,
                    int to_tile_major) {
    const int64_t T = 4 * (int64_t)Tt, H = 4 * (int64_t)Th, W = 4 * (int64_t)Tw;
    const int64_t S = T * H * W;
    for (int64_t bh = 0; bh < BH; ++bh)
        for (int64_t t = 0; t < T; ++t)
            for (int64_t h = 0; h < H; ++h)
                for (int64_t w = 0; w < W; ++w) {
                    int64_t raster = (t * H + h) * W + w;
                    int64_t tile = ((t / 4) * Th + h / 4) * Tw + w / 4;
                    int64_t major = tile * 64 + ((t % 4) * 4 + h % 4) * 4 + w % 4;
                    int64_t from = to_tile_major ? raster : major;
                    int64_t to = to_tile_major ? major : raster;
                    memcpy(dst + (bh * S + to) * d, src + (bh * S + from) * d,
                           (size_t)d * sizeof(uint16_t));
                }
}

/* Block attention energy ("Accelerating Text-to-Video Generation with
 * Calibrated Sparse Attention", section 2 "Methodologie: CalibAtt", A "Offline
 * Kalibratie": the energy, i.e. summed attention scores,
 * of each block; NABLA review, major comment 1: the true attention mass of an
 * N x N block).  For each listed (r, c):
 *   E[r][c] = (1/64) sum_{i in block r} sum_{j in block c} exp(scale q_i.k_j - lse_i)
 * mask [BH, nb, nb] uint8 marks the listed blocks; lse [BH*S] is given (a row
 * with a non-finite lse contributes nothing).  The block rows evaluated are
 * rows[0..nrows) (global ids bh*nb + r), or every row when rows is NULL;
 * energy [nrows, nb] is written in full, 0 where unlisted; block_mass (may be
 * NULL) [nrows] = sum_c E[r][c]. */
void oracle_block_energy(const uint16_t* q, const uint16_t* k, const double* lse, int64_t BH,
                         int64_t S, int d, const uint8_t* mask, double scale, int64_t nrows,
                         const int64_t* rows, double* energy, double* block_mass) {
    const int64_t nb = S / ORACLE_BLOCK;
    if (rows == NULL) nrows = BH * nb;
#pragma omp parallel for schedule(dynamic)
    for (int64_t n = 0; n < nrows; ++n) {
        int64_t br = rows ? rows[n] : n;
        int64_t bh = br / nb, r = br % nb;
        double total = 0.0;
        for (int64_t c = 0; c < nb; ++c) {
            double e = 0.0;
            if (mask[br * nb + c]) {
                for (int64_t i = r * ORACLE_BLOCK; i < (r + 1) * ORACLE_BLOCK; ++i) {
                    double li = lse[bh * S + i];
                    if (!isfinite(li)) continue;
                    for (int64_t j = c * ORACLE_BLOCK; j < (c + 1) * ORACLE_BLOCK; ++j) {
                        double dot = 0.0;
                        for (int t = 0; t < d; ++t)
                            dot += bf16_to_f64(q[(bh * S + i) * d + t]) *
                                   bf16_to_f64(k[(bh * S + j) * d + t]);
                        e += exp(scale * dot - li);
                    }
                }
                e /= ORACLE_BLOCK;
            }
            energy[n * nb + c] = e;
            total += e;
        }
        if (block_mass) block_mass[n] = total;
    }
}

/* One calibration run (CalibAtt, Methodology A, "threshold" step): each energy
 * row, normalised by its sum, goes through the same minimal-prefix rule as the
 * NABLA mask with thr = eps; votes[r][c] += 1 for every kept block.  A row
 * whose energy sums to zero keeps nothing; negative or NaN energies count as
 * zero. */
void oracle_calib_accumulate(const double* energy, int64_t nrows, int nb, double eps,
                             int32_t* votes) {
#pragma omp parallel for schedule(static)
    for (int64_t g = 0; g < nrows; ++g) {
        double* p = (double*)malloc(sizeof(double) * (size_t)nb);
        uint8_t* keep = (uint8_t*)malloc((size_t)nb);
        double z = 0.0;
        for (int c = 0; c < nb; ++c) {
            double e = energy[g * nb + c];
            p[c] = e > 0.0 ? e : 0.0;
            z += p[c];
        }
        if (z > 0.0) {
            for (int c = 0; c < nb; ++c) p[c] /= z;
            oracle_row_select(p, nb, eps, keep, NULL);
            for (int c = 0; c < nb; ++c) votes[g * nb + c] += keep[c];
        }
        free(p);
        free(keep);
    }
}

/* Aggregation over the calibration runs (CalibAtt, Methodology A: blocks that
 * the runs consistently miss are skipped): mask = votes >= min_votes. */
void oracle_calib_finalize(const int32_t* votes, int64_t n, int32_t min_votes, uint8_t* mask) {
    for (int64_t i = 0; i < n; ++i) mask[i] = votes[i] >= min_votes ? 1 : 0;
}

/* Row statistics of block-masked attention for query row i of head bh:
 * lse = ln sum_j exp(scale q_i.k_j) over kept keys (-inf when none) and
 * D = dO_i . O_i with O_i the exact fp64 attention output (0 when none). */
static void attn_row_stats(const uint16_t* q, const uint16_t* k, const uint16_t* v,
                           const uint16_t* dO, int64_t bh, int64_t S, int d, const uint8_t* mask,
                           double scale, int64_t i, double* lse_out, double* D_out) {
    const int64_t nb = S / ORACLE_BLOCK;
    const uint8_t* mrow = mask + (bh * nb + i / ORACLE_BLOCK) * nb;
    double m = -INFINITY;
    for (int64_t j = 0; j < S; ++j) {
        if (!mrow[j / ORACLE_BLOCK]) continue;
        double dot = 0.0;
        for (int c = 0; c < d; ++c)
            dot += bf16_to_f64(q[(bh * S + i) * d + c]) * bf16_to_f64(k[(bh * S + j) * d + c]);
        if (scale * dot > m) m = scale * dot;
    }
    if (m == -INFINITY) { *lse_out = -INFINITY; *D_out = 0.0; return; }
    double l = 0.0, D = 0.0;
    for (int64_t j = 0; j < S; ++j) {
        if (!mrow[j / ORACLE_BLOCK]) continue;
        double dot = 0.0, dv = 0.0;
        for (int c = 0; c < d; ++c) {
            dot += bf16_to_f64(q[(bh * S + i) * d + c]) * bf16_to_f64(k[(bh * S + j) * d + c]);
            dv += bf16_to_f64(dO[(bh * S + i) * d + c]) * bf16_to_f64(v[(bh * S + j) * d + c]);
        }
        double w = exp(scale * dot - m);
        l += w;
        D += w * dv;   /* sum_j p_ij (dO_i . v_j) = dO_i . O_i, up to the 1/l below */
    }
    *lse_out = m + log(l);
    *D_out = D / l;
}

/* Backward of block-masked softmax attention (FlashAttention's backward: the
 * probabilities are recomputed from the forward's log-sum-exp; the mask is
 * the one the forward used).  For kept (i, j), p_ij = exp(scale q_i.k_j -
 * lse_i), dP_ij = dO_i.v_j, dS_ij = p_ij (dP_ij - D_i) with D_i = dO_i.O_i:
 *   dQ_i = scale sum_j dS_ij k_j,  dK_j = scale sum_i dS_ij q_i,  dV_j = sum_i p_ij dO_i.
 * qrows (nq global row ids bh*S + i; NULL = every row) select the dQ rows,
 * krows (nk ids bh*S + j; NULL = every key) the dK, dV rows; outputs fp64
 * [nq, d] and [nk, d].  Inputs q, k, v, dO are bf16 bits [BH, S, d]. */
void oracle_attention_bwd(const uint16_t* q, const uint16_t* k, const uint16_t* v,
                          const uint16_t* dO, int64_t BH, int64_t S, int d, const uint8_t* mask,
                          double scale, int64_t nq, const int64_t* qrows, double* dQ, int64_t nk,
                          const int64_t* krows, double* dK, double* dV) {
    const int64_t nb = S / ORACLE_BLOCK;
    if (qrows == NULL) nq = BH * S;
    if (krows == NULL) nk = BH * S;
#pragma omp parallel for schedule(dynamic)
    for (int64_t n = 0; n < nq; ++n) {
        const int64_t g = qrows ? qrows[n] : n, bh = g / S, i = g % S;
        double lse, D;
        attn_row_stats(q, k, v, dO, bh, S, d, mask, scale, i, &lse, &D);
        for (int c = 0; c < d; ++c) dQ[n * d + c] = 0.0;
        if (lse == -INFINITY) continue;
        const uint8_t* mrow = mask + (bh * nb + i / ORACLE_BLOCK) * nb;
        for (int64_t j = 0; j < S; ++j) {
            if (!mrow[j / ORACLE_BLOCK]) continue;
            double dot = 0.0, dp = 0.0;
            for (int c = 0; c < d; ++c) {
                dot += bf16_to_f64(q[(bh * S + i) * d + c]) * bf16_to_f64(k[(bh * S + j) * d + c]);
                dp += bf16_to_f64(dO[(bh * S + i) * d + c]) * bf16_to_f64(v[(bh * S + j) * d + c]);
            }
            double p = exp(scale * dot - lse);
            double ds = p * (dp - D);
            for (int c = 0; c < d; ++c) dQ[n * d + c] += scale * ds * bf16_to_f64(k[(bh * S + j) * d + c]);
        }
    }
    if (nk == 0) return;
    /* row statistics of every query row of every head */
    double* lse_all = (double*)malloc(sizeof(double) * (size_t)(BH * S));
    double* D_all = (double*)malloc(sizeof(double) * (size_t)(BH * S));
#pragma omp parallel for schedule(dynamic)
    for (int64_t g = 0; g < BH * S; ++g)
        attn_row_stats(q, k, v, dO, g / S, S, d, mask, scale, g % S, &lse_all[g], &D_all[g]);
#pragma omp parallel for schedule(dynamic)
    for (int64_t n = 0; n < nk; ++n) {
        const int64_t g = krows ? krows[n] : n, bh = g / S, j = g % S;
        for (int c = 0; c < d; ++c) { dK[n * d + c] = 0.0; dV[n * d + c] = 0.0; }
        for (int64_t i = 0; i < S; ++i) {
            if (!mask[(bh * nb + i / ORACLE_BLOCK) * nb + j / ORACLE_BLOCK]) continue;
            const double lse = lse_all[bh * S + i];
            double dot = 0.0, dp = 0.0;
            for (int c = 0; c < d; ++c) {
                dot += bf16_to_f64(q[(bh * S + i) * d + c]) * bf16_to_f64(k[(bh * S + j) * d + c]);
                dp += bf16_to_f64(dO[(bh * S + i) * d + c]) * bf16_to_f64(v[(bh * S + j) * d + c]);
            }
            double p = exp(scale * dot - lse);
            double ds = p * (dp - D_all[bh * S + i]);
            for (int c = 0; c < d; ++c) {
                dK[n * d + c] += scale * ds * bf16_to_f64(q[(bh * S + i) * d + c]);
                dV[n * d + c] += p * bf16_to_f64(dO[(bh * S + i) * d + c]);
            }
        }
    }
    free(lse_all);
    free(D_all);
}

/* XAttention antidiagonal block scores ("XAttention: Block Sparse Attention
 * with Antidiagonal Scoring" notes: blocks are scored along antidiagonals and
 * selected by a threshold).  Reading (the notes give no formula): stride St
 * divides 64; strided query row i and key row j of a head stand for the St x St
 * sub-block of Q K^T at rows i*St.., columns j*St..; their score is the mean of
 * that sub-block's antidiagonal,
 *   a_ij = (1/St) sum_{s<St} q_{i*St + St-1-s} . k_{j*St + s} / sqrt(d),
 * p_i = softmax over all strided keys j of a_i, and the block score of query
 * block r and key block c is the mean over r's 64/St strided rows of the mass
 * p puts on c's 64/St strided keys (so each row of scores sums to 1).
 * rows (nrows global block-row ids bh*nb + r; NULL = every row) select the
 * rows computed; scores [nrows, nb]. */
void oracle_xattn_scores(const uint16_t* q, const uint16_t* k, int64_t BH, int64_t S, int d,
                         int St, int64_t nrows, const int64_t* rows, double* scores) {
    const int64_t nb = S / ORACLE_BLOCK, L = S / St, per = ORACLE_BLOCK / St;
    const double scale = 1.0 / (St * sqrt((double)d));
    if (rows == NULL) nrows = BH * nb;
#pragma omp parallel for schedule(dynamic)
    for (int64_t n = 0; n < nrows; ++n) {
        const int64_t g = rows ? rows[n] : n, bh = g / nb, r = g % nb;
        double* a = (double*)malloc(sizeof(double) * (size_t)L);
        for (int64_t c = 0; c < nb; ++c) scores[n * nb + c] = 0.0;
        for (int64_t ii = 0; ii < per; ++ii) {
            const int64_t i = r * per + ii;
            double m = -INFINITY;
            for (int64_t j = 0; j < L; ++j) {
                double acc = 0.0;
                for (int s = 0; s < St; ++s) {
                    const uint16_t* qr = q + (bh * S + i * St + St - 1 - s) * d;
                    const uint16_t* kr = k + (bh * S + j * St + s) * d;
                    for (int t = 0; t < d; ++t) acc += bf16_to_f64(qr[t]) * bf16_to_f64(kr[t]);
                }
                a[j] = scale * acc;
                if (a[j] > m) m = a[j];
            }
            double z = 0.0;
            for (int64_t j = 0; j < L; ++j) z += exp(a[j] - m);
            for (int64_t j = 0; j < L; ++j) scores[n * nb + j / per] += exp(a[j] - m) / z / per;
        }
        free(a);
    }
}

/* Threads OpenMP will use (for reporting the CPU baseline's core count). */
int oracle_max_threads(void) {
#ifdef _OPENMP
    extern int omp_get_max_threads(void);
    return omp_get_max_threads();
#else
    return 1;
#endif
}

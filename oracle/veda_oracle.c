/*
 * veda_oracle.c -- plain, slow fp64 CPU oracle for Veda's inference hot path.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test suite, the package smoke check and
 * the benchmark's CPU-baseline leg may load or run this code.  It shares no
 * code, header, table or helper with the CUDA path, and it never reads a value
 * that the CUDA path produced except where a caller hands it an index list to
 * re-run attention on (the same mask on both sides).
 *
 * Source: "Veda: Scalable Video Diffusion via Distilled Sparse Attention"
 * (project page).  Every function below cites the section it follows.
 *
 * Readings where the page is silent (each one is listed in the design notes):
 *   - tokens are laid out in raster (t, y, x) order: n = (t*Hs + y)*Ws + x;
 *   - tiles of head h are the boxes of shape (p_t, p_h, p_w)_h in raster order
 *     of the tile grid, and the rows inside a tile are in raster order too;
 *   - TripPool statistics are per channel over the tile's tokens;
 *   - the three statistics are projected by the same head-specific d x d
 *     matrix (W_q on the query side, W_k on the key side), and the tile score
 *     is the sum of the three inner products;
 *   - Top-k keeps the k highest scores, ties going to the lower tile index;
 *   - attention is softmax(scale * q.k) over every key of the selected tiles.
 *
 * Parity pins: see tests/test_oracle_pins.py.  Every function here is pinned
 * (brute force on tiny grids, closed forms and invariants).
 *
 * Inputs are raw bf16 bit patterns (uint16); they are widened to fp64 exactly.
 * Outputs are fp64.  All loops are plain nested loops; OpenMP only spreads
 * independent (batch, head, tile) units over cores.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#ifdef _OPENMP
#include <omp.h>
#endif

/* bf16 -> fp64, exact: a bf16 value is the top half of an fp32 value. */
static double bf16_to_f64(uint16_t bits) {
    uint32_t u = ((uint32_t)bits) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

int oracle_num_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

void oracle_set_num_threads(int n) {
#ifdef _OPENMP
    if (n > 0) omp_set_num_threads(n);
#else
    (void)n;
#endif
}

/* Token index of grid point (t, y, x): raster order. */
static int64_t token_index(int64_t Hs, int64_t Ws, int64_t t, int64_t y, int64_t x) {
    return (t * Hs + y) * Ws + x;
}

/*
 * Token of row r of tile j for a head with tile shape (pt, ph, pw).
 * Head-Conditioned Tile Geometry (Principle 02): the tile is a pt x ph x pw
 * box of the T x Hs x Ws grid.  Tiles are numbered in raster order of the
 * (T/pt, Hs/ph, Ws/pw) tile grid; rows inside the tile in raster order.
 */
static int64_t tile_row_token(int64_t Hs, int64_t Ws, int64_t pt, int64_t ph, int64_t pw,
                              int64_t j, int64_t r) {
    int64_t nh = Hs / ph, nw = Ws / pw;
    int64_t a = j / (nh * nw);
    int64_t b = (j / nw) % nh;
    int64_t c = j % nw;
    int64_t lt = r / (ph * pw);
    int64_t lh = (r / pw) % ph;
    int64_t lw = r % pw;
    return token_index(Hs, Ws, a * pt + lt, b * ph + lh, c * pw + lw);
}

/* Fills tokens[j*Bt + r] with the token of row r of tile j (head shape given). */
void oracle_tile_tokens(int64_t T, int64_t Hs, int64_t Ws, int32_t pt, int32_t ph, int32_t pw,
                        int64_t* tokens) {
    int64_t Bt = (int64_t)pt * ph * pw;
    int64_t nT = (T / pt) * (Hs / ph) * (Ws / pw);
    for (int64_t j = 0; j < nT; ++j)
        for (int64_t r = 0; r < Bt; ++r)
            tokens[j * Bt + r] = tile_row_token(Hs, Ws, pt, ph, pw, j, r);
}

/*
 * TripPool (Attention Structure Distillation, "Estimator"; Theoretical
 * Rationale 2, "Tile Statistics"): for every tile and channel, the average,
 * the maximum and the minimum of X over the tile's tokens.
 *   X     : [B, H, N, d] bf16 bits, N = T*Hs*Ws
 *   shapes: [H][3] (pt, ph, pw), pt*ph*pw equal for every head
 *   stats : [B, H, nT, 3, d] fp64, statistic order (avg, max, min)
 */
void oracle_tripool(int64_t B, int64_t H, int64_t d, int64_t T, int64_t Hs, int64_t Ws,
                    const int32_t* shapes, const uint16_t* X, double* stats) {
    int64_t N = T * Hs * Ws;
    int64_t pt0 = shapes[0], ph0 = shapes[1], pw0 = shapes[2];
    int64_t nT = N / (pt0 * ph0 * pw0);
    int64_t units = B * H * nT;
#pragma omp parallel for schedule(dynamic, 16)
    for (int64_t u = 0; u < units; ++u) {
        int64_t j = u % nT;
        int64_t h = (u / nT) % H;
        int64_t b = u / (nT * H);
        int64_t pt = shapes[3 * h], ph = shapes[3 * h + 1], pw = shapes[3 * h + 2];
        int64_t Bt = pt * ph * pw;
        const uint16_t* Xh = X + (b * H + h) * N * d;
        double* out = stats + ((b * H + h) * nT + j) * 3 * d;
        for (int64_t c = 0; c < d; ++c) {
            double sum = 0.0, mx = -INFINITY, mn = INFINITY;
            for (int64_t r = 0; r < Bt; ++r) {
                int64_t n = tile_row_token(Hs, Ws, pt, ph, pw, j, r);
                double v = bf16_to_f64(Xh[n * d + c]);
                sum += v;
                if (v > mx) mx = v;
                if (v < mn) mn = v;
            }
            out[0 * d + c] = sum / (double)Bt;
            out[1 * d + c] = mx;
            out[2 * d + c] = mn;
        }
    }
}

/*
 * Head-specific projection (Attention Structure Distillation, "Estimator":
 * head-specific Q/K projections of the tile statistics).  Each statistic row
 * vector s (length d) becomes s . W[h] (W[h] is d x d, row index = input
 * channel, column index = output channel).
 *   stats: [B, H, nT, 3, d] fp64;  W: [H, d, d] fp32;  out: same shape as stats.
 */
void oracle_project(int64_t B, int64_t H, int64_t nT, int64_t d,
                    const double* stats, const float* W, double* out) {
    int64_t rows = B * H * nT * 3;
#pragma omp parallel for schedule(static)
    for (int64_t row = 0; row < rows; ++row) {
        int64_t h = (row / (3 * nT)) % H;
        const double* s = stats + row * d;
        const float* Wh = W + h * d * d;
        double* o = out + row * d;
        for (int64_t co = 0; co < d; ++co) {
            double acc = 0.0;
            for (int64_t ci = 0; ci < d; ++ci) acc += s[ci] * (double)Wh[ci * d + co];
            o[co] = acc;
        }
    }
}

/*
 * Tile score (Attention Structure Distillation, "Estimator"; Theoretical
 * Rationale 4: the estimator's scores over key tiles, before Top-k):
 *   S[i, j] = sum over s in {avg, max, min} of <q~_{i,s}, k~_{j,s}>.
 *   qt, kt: [B, H, nT, 3, d] projected statistics;  S: [B, H, nT, nT] fp64.
 */
void oracle_score(int64_t B, int64_t H, int64_t nT, int64_t d,
                  const double* qt, const double* kt, double* S) {
    int64_t rows = B * H * nT;
#pragma omp parallel for schedule(static)
    for (int64_t row = 0; row < rows; ++row) {
        int64_t bh = row / nT;
        const double* q = qt + row * 3 * d;
        for (int64_t j = 0; j < nT; ++j) {
            const double* kk = kt + (bh * nT + j) * 3 * d;
            double acc = 0.0;
            for (int64_t s = 0; s < 3; ++s)
                for (int64_t c = 0; c < d; ++c) acc += q[s * d + c] * kk[s * d + c];
            S[row * nT + j] = acc;
        }
    }
}

typedef struct {
    double v;
    int64_t j;
} scored_tile;

/* Total order of the selection: higher score first, then lower tile index. */
static int scored_tile_cmp(const void* pa, const void* pb) {
    const scored_tile* a = (const scored_tile*)pa;
    const scored_tile* b = (const scored_tile*)pb;
    if (a->v > b->v) return -1;
    if (a->v < b->v) return 1;
    if (a->j < b->j) return -1;
    if (a->j > b->j) return 1;
    return 0;
}

static int int32_cmp(const void* pa, const void* pb) {
    int32_t a = *(const int32_t*)pa, b = *(const int32_t*)pb;
    return (a > b) - (a < b);
}

/*
 * Head-aware Top-k (Attention Structure Distillation, "Execution"): per
 * query-tile row keep the k highest-scoring key tiles; ties go to the lower
 * tile index (fp64 comparison, so -0.0 and +0.0 tie).  Emits the 0/1 mask and
 * the ascending index list.
 *   S: [rows, nT] fp64;  mask: [rows, nT] (may be NULL);  idx: [rows, k].
 */
void oracle_topk(int64_t rows, int64_t nT, int64_t k, const double* S,
                 uint8_t* mask, int32_t* idx) {
#pragma omp parallel
    {
        scored_tile* buf = (scored_tile*)malloc(sizeof(scored_tile) * (size_t)nT);
#pragma omp for schedule(static)
        for (int64_t row = 0; row < rows; ++row) {
            for (int64_t j = 0; j < nT; ++j) {
                buf[j].v = S[row * nT + j];
                buf[j].j = j;
            }
            qsort(buf, (size_t)nT, sizeof(scored_tile), scored_tile_cmp);
            int32_t* out = idx + row * k;
            for (int64_t t = 0; t < k; ++t) out[t] = (int32_t)buf[t].j;
            qsort(out, (size_t)k, sizeof(int32_t), int32_cmp);
            if (mask) {
                memset(mask + row * nT, 0, (size_t)nT);
                for (int64_t t = 0; t < k; ++t) mask[row * nT + out[t]] = 1;
            }
        }
        free(buf);
    }
}

/*
 * Tile-skipping attention (Attention Structure Distillation, "Execution";
 * Theoretical Rationale 1, "Softmax Geometry": the kept keys are renormalised
 * among themselves).  For every query token of tile i of unit (b, h, i):
 *   O = softmax(scale * q . k over all keys of the selected tiles) . V
 *   lse = ln sum exp(scale * q . k) over the same keys.
 * Units are given as triples (b, h, i); outputs are per unit, row r of the
 * unit being row r of tile i (token given by oracle_tile_tokens).
 *   Q, K, V: [B, H, N, d] bf16 bits;  idx: [B, H, nT, k] int32
 *   O_out: [nunits, Bt, d] fp64;  lse_out: [nunits, Bt] fp64 (may be NULL)
 */
void oracle_sparse_attention(int64_t B, int64_t H, int64_t d, int64_t T, int64_t Hs, int64_t Ws,
                             const int32_t* shapes, int64_t k, double scale,
                             const uint16_t* Q, const uint16_t* K, const uint16_t* V,
                             const int32_t* idx, int64_t nunits, const int64_t* units,
                             double* O_out, double* lse_out) {
    int64_t N = T * Hs * Ws;
    int64_t Bt = (int64_t)shapes[0] * shapes[1] * shapes[2];
    int64_t nT = N / Bt;
    int64_t nkeys = k * Bt;
    /* one work item per (unit, query row) */
    int64_t items = nunits * Bt;
#pragma omp parallel
    {
        double* logit = (double*)malloc(sizeof(double) * (size_t)nkeys);
        int64_t* key_tok = (int64_t*)malloc(sizeof(int64_t) * (size_t)nkeys);
        double* q = (double*)malloc(sizeof(double) * (size_t)d);
#pragma omp for schedule(dynamic, 8)
        for (int64_t it = 0; it < items; ++it) {
            int64_t u = it / Bt, r = it % Bt;
            int64_t b = units[3 * u], h = units[3 * u + 1], i = units[3 * u + 2];
            int64_t pt = shapes[3 * h], ph = shapes[3 * h + 1], pw = shapes[3 * h + 2];
            const uint16_t* Qh = Q + (b * H + h) * N * d;
            const uint16_t* Kh = K + (b * H + h) * N * d;
            const uint16_t* Vh = V + (b * H + h) * N * d;
            const int32_t* sel = idx + ((b * H + h) * nT + i) * k;
            int64_t qn = tile_row_token(Hs, Ws, pt, ph, pw, i, r);
            for (int64_t c = 0; c < d; ++c) q[c] = bf16_to_f64(Qh[qn * d + c]);
            double mx = -INFINITY;
            for (int64_t t = 0; t < k; ++t)
                for (int64_t rr = 0; rr < Bt; ++rr) {
                    int64_t kn = tile_row_token(Hs, Ws, pt, ph, pw, sel[t], rr);
                    double dot = 0.0;
                    for (int64_t c = 0; c < d; ++c) dot += q[c] * bf16_to_f64(Kh[kn * d + c]);
                    double z = scale * dot;
                    logit[t * Bt + rr] = z;
                    key_tok[t * Bt + rr] = kn;
                    if (z > mx) mx = z;
                }
            double denom = 0.0;
            for (int64_t e = 0; e < nkeys; ++e) {
                logit[e] = exp(logit[e] - mx);
                denom += logit[e];
            }
            double* o = O_out + (u * Bt + r) * d;
            for (int64_t c = 0; c < d; ++c) o[c] = 0.0;
            for (int64_t e = 0; e < nkeys; ++e) {
                double p = logit[e] / denom;
                const uint16_t* vrow = Vh + key_tok[e] * d;
                for (int64_t c = 0; c < d; ++c) o[c] += p * bf16_to_f64(vrow[c]);
            }
            if (lse_out) lse_out[u * Bt + r] = mx + log(denom);
        }
        free(logit);
        free(key_tok);
        free(q);
    }
}

/*
 * Max-pooled full-attention teacher (Attention Structure Distillation,
 * "Teacher"; Empirical Study 02, "Controlled Mask Intervention": the oracle
 * mask max-pools the full attention map).  With P = softmax(scale * Q K^T)
 * over all N keys, teacher[i, j] = max over query tokens of tile i and key
 * tokens of tile j of P.  Also returns the dense lse per token.
 *   teacher: [B, H, nT, nT] fp64;  lse_dense: [B, H, N] fp64 (may be NULL)
 * Cost is O(B*H*N^2*d): small grids only.
 */
void oracle_teacher(int64_t B, int64_t H, int64_t d, int64_t T, int64_t Hs, int64_t Ws,
                    const int32_t* shapes, double scale,
                    const uint16_t* Q, const uint16_t* K,
                    double* teacher, double* lse_dense) {
    int64_t N = T * Hs * Ws;
    int64_t Bt = (int64_t)shapes[0] * shapes[1] * shapes[2];
    int64_t nT = N / Bt;
    int64_t units = B * H * nT;
#pragma omp parallel
    {
        double* logit = (double*)malloc(sizeof(double) * (size_t)N);
        double* q = (double*)malloc(sizeof(double) * (size_t)d);
        int64_t* key_tile = (int64_t*)malloc(sizeof(int64_t) * (size_t)N);
#pragma omp for schedule(dynamic, 1)
        for (int64_t u = 0; u < units; ++u) {
            int64_t i = u % nT, h = (u / nT) % H, b = u / (nT * H);
            int64_t pt = shapes[3 * h], ph = shapes[3 * h + 1], pw = shapes[3 * h + 2];
            const uint16_t* Qh = Q + (b * H + h) * N * d;
            const uint16_t* Kh = K + (b * H + h) * N * d;
            double* trow = teacher + ((b * H + h) * nT + i) * nT;
            for (int64_t j = 0; j < nT; ++j) {
                trow[j] = 0.0;
                for (int64_t rr = 0; rr < Bt; ++rr)
                    key_tile[tile_row_token(Hs, Ws, pt, ph, pw, j, rr)] = j;
            }
            for (int64_t r = 0; r < Bt; ++r) {
                int64_t qn = tile_row_token(Hs, Ws, pt, ph, pw, i, r);
                for (int64_t c = 0; c < d; ++c) q[c] = bf16_to_f64(Qh[qn * d + c]);
                double mx = -INFINITY;
                for (int64_t n = 0; n < N; ++n) {
                    double dot = 0.0;
                    for (int64_t c = 0; c < d; ++c) dot += q[c] * bf16_to_f64(Kh[n * d + c]);
                    logit[n] = scale * dot;
                    if (logit[n] > mx) mx = logit[n];
                }
                double denom = 0.0;
                for (int64_t n = 0; n < N; ++n) denom += exp(logit[n] - mx);
                for (int64_t n = 0; n < N; ++n) {
                    double p = exp(logit[n] - mx) / denom;
                    int64_t j = key_tile[n];
                    if (p > trow[j]) trow[j] = p;
                }
                if (lse_dense) lse_dense[(b * H + h) * N + qn] = mx + log(denom);
            }
        }
        free(logit);
        free(q);
        free(key_tile);
    }
}

/*
 * Tile recall (Empirical Study 02, "Controlled Mask Intervention": the share
 * of oracle-selected tiles that a predicted mask recovers).  Per row, the
 * number of reference tiles that also appear in the predicted row, divided by
 * k; returns the mean over rows.
 *   pred, ref: [rows, k] tile indices;  per_row: [rows] (may be NULL)
 */
double oracle_tile_recall(int64_t rows, int64_t k, const int32_t* pred, const int32_t* ref,
                          double* per_row) {
    double total = 0.0;
    for (int64_t row = 0; row < rows; ++row) {
        int64_t hits = 0;
        for (int64_t a = 0; a < k; ++a) {
            int found = 0;
            for (int64_t b = 0; b < k; ++b)
                if (pred[row * k + b] == ref[row * k + a]) found = 1;
            hits += found;
        }
        if (per_row) per_row[row] = (double)hits / (double)k;
        total += (double)hits;
    }
    return total / ((double)rows * (double)k);
}

/*
 * KL structure distillation (Principle 01, "Full-Attention Structure
 * Distillation"; Theoretical Rationale 4, "Distillation Objective": row-wise
 * KL between the teacher's tile distribution and the estimator's soft
 * distribution over key tiles).  Readings: the target row is the teacher row
 * divided by its sum; the prediction is softmax(S / tau); the loss is the mean
 * of the row divergences over all B*H*nT rows.
 *   statsQ, statsK: [B, H, nT, 3, d];  Wq, Wk: [H, d, d] fp32
 *   teacher: [B, H, nT, nT];  dWq, dWk: [H, d, d] (may be NULL)
 * Returns the loss.  The gradient follows the chain rule through
 * S = sum_s (statsQ_s Wq) . (statsK_s Wk):
 *   dS = (pred - tgt) / (tau R);  dq~ = dS k~;  dk~ = dS^T q~;
 *   dWq = sum stats_Q^T dq~;  dWk = sum stats_K^T dk~.
 */
double oracle_distill_kl(int64_t B, int64_t H, int64_t nT, int64_t d,
                         const double* statsQ, const double* statsK, const float* Wq,
                         const float* Wk, const double* teacher, double tau,
                         double* dWq, double* dWk) {
    int64_t n3 = B * H * nT * 3 * d;
    double* qt = (double*)malloc(sizeof(double) * (size_t)n3);
    double* kt = (double*)malloc(sizeof(double) * (size_t)n3);
    double* S = (double*)malloc(sizeof(double) * (size_t)(B * H * nT * nT));
    double* G = (double*)malloc(sizeof(double) * (size_t)(B * H * nT * nT));
    oracle_project(B, H, nT, d, statsQ, Wq, qt);
    oracle_project(B, H, nT, d, statsK, Wk, kt);
    oracle_score(B, H, nT, d, qt, kt, S);
    int64_t R = B * H * nT;
    double total = 0.0;
    for (int64_t row = 0; row < R; ++row) {
        const double* s = S + row * nT;
        const double* t = teacher + row * nT;
        double mx = -INFINITY, tsum = 0.0;
        for (int64_t j = 0; j < nT; ++j) {
            if (s[j] / tau > mx) mx = s[j] / tau;
            tsum += t[j];
        }
        double se = 0.0;
        for (int64_t j = 0; j < nT; ++j) se += exp(s[j] / tau - mx);
        double lse = mx + log(se);
        double kl = 0.0;
        for (int64_t j = 0; j < nT; ++j) {
            double logp = s[j] / tau - lse;
            double tg = t[j] / tsum;
            if (tg > 0.0) kl += tg * (log(tg) - logp);
            G[row * nT + j] = (exp(logp) - tg) / (tau * (double)R);
        }
        total += kl;
    }
    if (dWq && dWk) {
        for (int64_t e = 0; e < H * d * d; ++e) {
            dWq[e] = 0.0;
            dWk[e] = 0.0;
        }
        double* dq = (double*)malloc(sizeof(double) * (size_t)(3 * d));
        double* dk = (double*)malloc(sizeof(double) * (size_t)(3 * d));
        for (int64_t b = 0; b < B; ++b)
            for (int64_t h = 0; h < H; ++h) {
                int64_t bh = b * H + h;
                for (int64_t i = 0; i < nT; ++i) {
                    /* dq~_i = sum_j G[i,j] k~_j ;  dk~_i = sum_j G[j,i] q~_j */
                    for (int64_t c = 0; c < 3 * d; ++c) {
                        dq[c] = 0.0;
                        dk[c] = 0.0;
                    }
                    for (int64_t j = 0; j < nT; ++j) {
                        double gij = G[(bh * nT + i) * nT + j];
                        double gji = G[(bh * nT + j) * nT + i];
                        for (int64_t c = 0; c < 3 * d; ++c) {
                            dq[c] += gij * kt[(bh * nT + j) * 3 * d + c];
                            dk[c] += gji * qt[(bh * nT + j) * 3 * d + c];
                        }
                    }
                    for (int64_t s3 = 0; s3 < 3; ++s3) {
                        const double* sq = statsQ + ((bh * nT + i) * 3 + s3) * d;
                        const double* sk = statsK + ((bh * nT + i) * 3 + s3) * d;
                        for (int64_t ci = 0; ci < d; ++ci)
                            for (int64_t co = 0; co < d; ++co) {
                                dWq[(h * d + ci) * d + co] += sq[ci] * dq[s3 * d + co];
                                dWk[(h * d + ci) * d + co] += sk[ci] * dk[s3 * d + co];
                            }
                    }
                }
            }
        free(dq);
        free(dk);
    }
    free(qt);
    free(kt);
    free(S);
    free(G);
    return total / (double)R;
}

/* ----------------------------------------------------------- fp8 weights
 * fp8 estimator weights.  News page ("Veda from ByteDance, HKU and USTC: an
 * open method that speeds up video generation fivefold", "Why this matters
 * for users"): the predictor is distributed in fp8 at half the size of the
 * bf16 file with almost the same tile recall.  The page names no encoding or
 * scaling; the reading taken here is the OCP FP8 E4M3 format ("e4m3fn": 1
 * sign bit, 4 exponent bits with bias 7, 3 mantissa bits, no infinities; the
 * all-ones exponent with all-ones mantissa is NaN, so the largest finite
 * value is 1.75 * 2^8 = 448; exponent field 0 holds the subnormals
 * m/8 * 2^-6) with one scale per head, s = amax / 448, W ~= s * e4m3(W / s),
 * rounding to the nearest code, ties to the even code, saturating at +-448.
 * The scale and W / s are fp32 operations (the quantiser's decisions are
 * taken on fp32 values); the dequantised weight is the fp32 product
 * e4m3 * s, the weight the fp32 estimator then computes with.
 */
double oracle_e4m3_decode(int32_t code)
{
    const int sign = (code >> 7) & 1, e = (code >> 3) & 15, m = code & 7;
    double v;
    if (e == 15 && m == 7) return NAN;
    if (e == 0)
        v = ldexp((double)m / 8.0, -6);
    else
        v = ldexp(1.0 + (double)m / 8.0, e - 7);
    return sign ? -v : v;
}

/* Nearest e4m3 code of an fp32 value: ties to the even code, saturating. */
int32_t oracle_e4m3_encode(float x)
{
    if (isnan(x)) return 0x7F;
    const int32_t sign = signbit(x) ? 0x80 : 0;
    const double a = fabs((double)x);
    if (a >= 448.0) return sign | 126;
    /* codes 0..126 are the non-negative finite values in increasing order:
       find the largest code whose value is <= a */
    int32_t lo = 0, hi = 126;
    while (lo < hi) {
        const int32_t mid = (lo + hi + 1) / 2;
        if (oracle_e4m3_decode(mid) <= a)
            lo = mid;
        else
            hi = mid - 1;
    }
    const double dlo = a - oracle_e4m3_decode(lo);      /* exact in fp64 */
    const double dhi = oracle_e4m3_decode(lo + 1) - a;
    int32_t code;
    if (dlo < dhi)
        code = lo;
    else if (dlo > dhi)
        code = lo + 1;
    else
        code = (lo & 1) ? lo + 1 : lo;
    return sign | code;
}

/* W: fp32 [H][n]; codes: uint8 [H][n]; scale: fp32 [H]. */
void oracle_quantize_e4m3(int64_t H, int64_t n, const float* W, uint8_t* codes, float* scale)
{
    for (int64_t h = 0; h < H; ++h) {
        float amax = 0.0f;
        for (int64_t i = 0; i < n; ++i) {
            const float a = fabsf(W[h * n + i]);
            if (a > amax) amax = a;
        }
        const float s = amax > 0.0f ? amax / 448.0f : 1.0f;
        scale[h] = s;
        for (int64_t i = 0; i < n; ++i) {
            const float y = W[h * n + i] / s;
            codes[h * n + i] = (uint8_t)oracle_e4m3_encode(y);
        }
    }
}

/* W[h][i] = fp32(e4m3(codes[h][i]) * scale[h]). */
void oracle_dequantize_e4m3(int64_t H, int64_t n, const uint8_t* codes, const float* scale,
                            float* W)
{
    for (int64_t h = 0; h < H; ++h)
        for (int64_t i = 0; i < n; ++i) {
            const float v = (float)oracle_e4m3_decode(codes[h * n + i]);
            W[h * n + i] = v * scale[h];
        }
}

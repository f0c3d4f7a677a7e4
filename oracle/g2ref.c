/*
 * g2ref.c -- fp64 CPU oracle for the Gemma 2 per-layer attention forward
 * and its gradients.
 *
 * TEST INFRASTRUCTURE (see g2ref.h): loaded only by the tests, the smoke
 * check and the benchmark's CPU-baseline leg. Plain loops, no blocking, no
 * fusion: one query row at a time, in the order of the Gemma 2 card's
 * per-layer attention pseudo-code ("Method" section): scale the queries,
 * score every key, soft-cap, mask, softmax, mix the values.
 */
#include "g2ref.h"

#include <math.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* bf16 is the upper half of an IEEE binary32; widening is exact. */
static double widen(uint16_t bits) {
    uint32_t u = (uint32_t)bits << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

static int check_args(int64_t B, int64_t T, int64_t S, int64_t H, int64_t Hkv, int64_t d,
                      int64_t q_offset, double softcap, int64_t window) {
    if (B <= 0 || T <= 0 || S <= 0 || H <= 0 || Hkv <= 0 || d <= 0) return -1;
    if (H % Hkv != 0) return -1;
    if (q_offset < 0 || window < 0 || softcap < 0) return -1;
    return 0;
}

/* Mask of the card's pseudo-code: causal, and for a local layer also within
 * the window. The window keeps the key at distance 0 (the query itself) and
 * the window-1 keys before it: "Gemma 2 Guide" code builds the local mask with
 * tril(diagonal=-W) and the card's paper-vs-code notes state the lower bound
 * as "position greater than pos - W". */
static int visible(int64_t p, int64_t j, int64_t window) {
    if (j > p) return 0;
    if (window > 0 && p - j >= window) return 0;
    return 1;
}

/* The KV head that query head h shares: the card's "every two query heads
 * share one" read as consecutive heads (h / group). */
static int64_t kv_head(int64_t h, int64_t H, int64_t Hkv) { return h / (H / Hkv); }

/* queries = queries * query_scale (the card's pseudo-code scales the query
 * row before the dot products). */
static void scaled_query(const uint16_t* qrow, int64_t d, double query_scale, double* qs) {
    for (int64_t c = 0; c < d; ++c) qs[c] = query_scale * widen(qrow[c]);
}

/* Capped logit of key j for the (already scaled) query qs.
 * Soft-cap formula: "Gemma 2 Guide", section 1, cap_val * tanh(logits / cap_val),
 * with cap_val = 50 for attention; the card applies it to every logit before
 * the mask. softcap == 0 means the cap is switched off. */
static double capped_logit(const double* qs, const uint16_t* krow, int64_t d, double softcap) {
    double x = 0.0;
    for (int64_t c = 0; c < d; ++c) x += qs[c] * widen(krow[c]);
    if (softcap > 0.0) x = softcap * tanh(x / softcap);
    return x;
}

/* One query row (b, i, h): fills s[0..S) with the masked capped logits and,
 * when out_row/lse are given, the mixed values and the log-sum-exp. */
static void one_row(const uint16_t* q, const uint16_t* k, const uint16_t* v,
                    int64_t b, int64_t i, int64_t h,
                    int64_t T, int64_t S, int64_t H, int64_t Hkv, int64_t d,
                    int64_t q_offset, double query_scale, double softcap, int64_t window,
                    double* qs, double* s, double* w, double* out_row, double* lse) {
    const int64_t g = kv_head(h, H, Hkv);
    const int64_t p = i + q_offset;
    scaled_query(q + ((b * T + i) * H + h) * d, d, query_scale, qs);

    /* logits -> soft-cap -> where(mask, logits, -inf) */
    for (int64_t j = 0; j < S; ++j) {
        const uint16_t* krow = k + ((b * S + j) * Hkv + g) * d;
        double sj = capped_logit(qs, krow, d, softcap);
        s[j] = visible(p, j, window) ? sj : -INFINITY;
    }

    /* softmax over keys */
    double m = -INFINITY;
    for (int64_t j = 0; j < S; ++j)
        if (s[j] > m) m = s[j];
    double l = 0.0;
    for (int64_t j = 0; j < S; ++j) {
        w[j] = (s[j] == -INFINITY) ? 0.0 : exp(s[j] - m);
        l += w[j];
    }
    for (int64_t j = 0; j < S; ++j) w[j] /= l;

    /* mix the values */
    if (out_row) {
        for (int64_t c = 0; c < d; ++c) out_row[c] = 0.0;
        for (int64_t j = 0; j < S; ++j) {
            if (w[j] == 0.0) continue; /* masked: weight exactly 0 */
            const uint16_t* vrow = v + ((b * S + j) * Hkv + g) * d;
            for (int64_t c = 0; c < d; ++c) out_row[c] += w[j] * widen(vrow[c]);
        }
    }
    if (lse) *lse = m + log(l);
}

int g2ref_attn(const uint16_t* q, const uint16_t* k, const uint16_t* v,
               double* out, double* lse,
               int64_t B, int64_t T, int64_t S, int64_t H, int64_t Hkv, int64_t d,
               int64_t q_offset, double query_scale, double softcap, int64_t window) {
    if (check_args(B, T, S, H, Hkv, d, q_offset, softcap, window)) return -1;
    const int64_t nrows = B * T * H;
    int err = 0;
#pragma omp parallel
    {
        double* qs = (double*)malloc(sizeof(double) * (size_t)d);
        double* s = (double*)malloc(sizeof(double) * (size_t)S);
        double* w = (double*)malloc(sizeof(double) * (size_t)S);
        if (!qs || !s || !w) {
#pragma omp atomic write
            err = 1;
        } else {
#pragma omp for schedule(dynamic, 4)
            for (int64_t r = 0; r < nrows; ++r) {
                const int64_t b = r / (T * H);
                const int64_t i = (r / H) % T;
                const int64_t h = r % H;
                one_row(q, k, v, b, i, h, T, S, H, Hkv, d, q_offset, query_scale, softcap,
                        window, qs, s, w, out + ((b * T + i) * H + h) * d,
                        lse + (b * H + h) * T + i);
            }
        }
        free(qs);
        free(s);
        free(w);
    }
    return err ? -1 : 0;
}

int g2ref_attn_rows(const uint16_t* q, const uint16_t* k, const uint16_t* v,
                    double* out, double* lse, const int64_t* rows, int64_t n,
                    int64_t B, int64_t T, int64_t S, int64_t H, int64_t Hkv, int64_t d,
                    int64_t q_offset, double query_scale, double softcap, int64_t window) {
    if (check_args(B, T, S, H, Hkv, d, q_offset, softcap, window)) return -1;
    for (int64_t r = 0; r < n; ++r) {
        const int64_t b = rows[3 * r], i = rows[3 * r + 1], h = rows[3 * r + 2];
        if (b < 0 || b >= B || i < 0 || i >= T || h < 0 || h >= H) return -1;
    }
    int err = 0;
#pragma omp parallel
    {
        double* qs = (double*)malloc(sizeof(double) * (size_t)d);
        double* s = (double*)malloc(sizeof(double) * (size_t)S);
        double* w = (double*)malloc(sizeof(double) * (size_t)S);
        if (!qs || !s || !w) {
#pragma omp atomic write
            err = 1;
        } else {
#pragma omp for schedule(dynamic, 1)
            for (int64_t r = 0; r < n; ++r) {
                one_row(q, k, v, rows[3 * r], rows[3 * r + 1], rows[3 * r + 2], T, S, H, Hkv,
                        d, q_offset, query_scale, softcap, window, qs, s, w, out + r * d,
                        lse + r);
            }
        }
        free(qs);
        free(s);
        free(w);
    }
    return err ? -1 : 0;
}

int g2ref_row_detail(const uint16_t* q, const uint16_t* k,
                     double* s, double* w, int64_t b, int64_t i, int64_t h,
                     int64_t B, int64_t T, int64_t S, int64_t H, int64_t Hkv, int64_t d,
                     int64_t q_offset, double query_scale, double softcap, int64_t window) {
    if (check_args(B, T, S, H, Hkv, d, q_offset, softcap, window)) return -1;
    if (b < 0 || b >= B || i < 0 || i >= T || h < 0 || h >= H) return -1;
    double* qs = (double*)malloc(sizeof(double) * (size_t)d);
    if (!qs) return -1;
    one_row(q, k, NULL, b, i, h, T, S, H, Hkv, d, q_offset, query_scale, softcap, window, qs,
            s, w, NULL, NULL);
    free(qs);
    return 0;
}

/* Backward of one query row (b, i, h) whose forward (qs, w) one_row has just
 * formed: dw_j = dout . v_j, D = sum_j w_j dw_j, then for every visible key
 * ds_j = w_j (dw_j - D) and dx_j = ds_j (1 - tanh^2(x_j / C)). Adds the row's
 * dq (dqrow), and its terms of dk and dv (rows of the (b, g) slices, when
 * given). Returns D. x holds S doubles of scratch. */
static double row_backward(const uint16_t* k, const uint16_t* v, const uint16_t* dout,
                           int64_t b, int64_t i, int64_t h, int64_t T, int64_t S, int64_t H,
                           int64_t Hkv, int64_t d, double query_scale, double softcap,
                           const double* qs, const double* w, double* x, double* dqrow,
                           double* dk, double* dv) {
    const int64_t g = kv_head(h, H, Hkv);
    const uint16_t* dorow = dout + ((b * T + i) * H + h) * d;
    /* dw_j = dout . v_j, and D = sum_j w_j dw_j */
    double D = 0.0;
    for (int64_t j = 0; j < S; ++j) {
        x[j] = 0.0;
        if (w[j] == 0.0) continue;
        const uint16_t* vj = v + ((b * S + j) * Hkv + g) * d;
        double dw = 0.0;
        for (int64_t c = 0; c < d; ++c) dw += widen(dorow[c]) * widen(vj[c]);
        x[j] = dw; /* holds dw_j until ds_j is formed */
        D += w[j] * dw;
    }
    if (!dqrow && !dk && !dv) return D;
    for (int64_t j = 0; j < S; ++j) {
        if (w[j] == 0.0) continue;
        const uint16_t* krow = k + ((b * S + j) * Hkv + g) * d;
        /* softmax: ds_j = w_j (dw_j - D) */
        double dx = w[j] * (x[j] - D);
        /* cap: d(C tanh(x/C))/dx = 1 - tanh^2(x/C), with x the scaled logit */
        if (softcap > 0.0) {
            double xl = 0.0;
            for (int64_t c = 0; c < d; ++c) xl += qs[c] * widen(krow[c]);
            const double t = tanh(xl / softcap);
            dx *= 1.0 - t * t;
        }
        /* x = (query_scale q) . k */
        if (dqrow)
            for (int64_t c = 0; c < d; ++c) dqrow[c] += query_scale * dx * widen(krow[c]);
        if (dk) {
            double* dkrow = dk + ((b * S + j) * Hkv + g) * d;
            for (int64_t c = 0; c < d; ++c) dkrow[c] += dx * qs[c];
        }
        if (dv) {
            double* dvrow = dv + ((b * S + j) * Hkv + g) * d;
            for (int64_t c = 0; c < d; ++c) dvrow[c] += w[j] * widen(dorow[c]);
        }
    }
    return D;
}

/* Gradients (see g2ref.h). Each (b, g) owns dk[b,:,g,:] and dv[b,:,g,:] and
 * the dq rows of its heads, so the parallel loop runs over (b, g). */
int g2ref_attn_bwd(const uint16_t* q, const uint16_t* k, const uint16_t* v,
                   const uint16_t* dout, double* dq, double* dk, double* dv,
                   int64_t B, int64_t T, int64_t S, int64_t H, int64_t Hkv, int64_t d,
                   int64_t q_offset, double query_scale, double softcap, int64_t window) {
    if (check_args(B, T, S, H, Hkv, d, q_offset, softcap, window)) return -1;
    const int64_t group = H / Hkv;
    memset(dq, 0, sizeof(double) * (size_t)(B * T * H * d));
    memset(dk, 0, sizeof(double) * (size_t)(B * S * Hkv * d));
    memset(dv, 0, sizeof(double) * (size_t)(B * S * Hkv * d));
    int err = 0;
#pragma omp parallel
    {
        double* qs = (double*)malloc(sizeof(double) * (size_t)d);
        double* s = (double*)malloc(sizeof(double) * (size_t)S);
        double* w = (double*)malloc(sizeof(double) * (size_t)S);
        double* x = (double*)malloc(sizeof(double) * (size_t)S);
        if (!qs || !s || !w || !x) {
#pragma omp atomic write
            err = 1;
        } else {
#pragma omp for schedule(dynamic, 1)
            for (int64_t bg = 0; bg < B * Hkv; ++bg) {
                const int64_t b = bg / Hkv, g = bg % Hkv;
                for (int64_t h = g * group; h < (g + 1) * group; ++h) {
                    for (int64_t i = 0; i < T; ++i) {
                        /* forward of this row: s, w (and qs = query_scale * q) */
                        one_row(q, k, v, b, i, h, T, S, H, Hkv, d, q_offset, query_scale,
                                softcap, window, qs, s, w, NULL, NULL);
                        row_backward(k, v, dout, b, i, h, T, S, H, Hkv, d, query_scale,
                                     softcap, qs, w, x, dq + ((b * T + i) * H + h) * d, dk, dv);
                    }
                }
            }
        }
        free(qs);
        free(s);
        free(w);
        free(x);
    }
    return err ? -1 : 0;
}

/* Gradients at chosen query rows and chosen keys (see g2ref.h), for layers
 * too large for g2ref_attn_bwd. The same chain rule as above, in two passes:
 * first every row that a chosen key can reach gets its softmax statistics
 * (lse and D = sum_j w_j dw_j, by one_row and the same dw loop); then each
 * chosen key sums its terms over those rows, each weight recovered from the
 * row's lse as w = exp(s - lse). dq rows are formed exactly as above. */
int g2ref_attn_bwd_sampled(const uint16_t* q, const uint16_t* k, const uint16_t* v,
                           const uint16_t* dout, const int64_t* qrows, int64_t nq,
                           const int64_t* keys, int64_t nk, double* dq, double* dk, double* dv,
                           int64_t B, int64_t T, int64_t S, int64_t H, int64_t Hkv, int64_t d,
                           int64_t q_offset, double query_scale, double softcap,
                           int64_t window) {
    if (check_args(B, T, S, H, Hkv, d, q_offset, softcap, window)) return -1;
    const int64_t group = H / Hkv;
    for (int64_t r = 0; r < nq; ++r) {
        const int64_t b = qrows[3 * r], i = qrows[3 * r + 1], h = qrows[3 * r + 2];
        if (b < 0 || b >= B || i < 0 || i >= T || h < 0 || h >= H) return -1;
    }
    for (int64_t r = 0; r < nk; ++r) {
        const int64_t b = keys[3 * r], j = keys[3 * r + 1], g = keys[3 * r + 2];
        if (b < 0 || b >= B || j < 0 || j >= S || g < 0 || g >= Hkv) return -1;
    }
    /* which (b, g) have a chosen key: only their rows need statistics */
    unsigned char* need = (unsigned char*)calloc((size_t)(B * Hkv), 1);
    double* row_lse = (double*)malloc(sizeof(double) * (size_t)(B * T * H));
    double* row_D = (double*)malloc(sizeof(double) * (size_t)(B * T * H));
    if (!need || !row_lse || !row_D) {
        free(need);
        free(row_lse);
        free(row_D);
        return -1;
    }
    for (int64_t r = 0; r < nk; ++r) need[keys[3 * r] * Hkv + keys[3 * r + 2]] = 1;
    int err = 0;
#pragma omp parallel
    {
        double* qs = (double*)malloc(sizeof(double) * (size_t)d);
        double* s = (double*)malloc(sizeof(double) * (size_t)S);
        double* w = (double*)malloc(sizeof(double) * (size_t)S);
        double* x = (double*)malloc(sizeof(double) * (size_t)S);
        if (!qs || !s || !w || !x) {
#pragma omp atomic write
            err = 1;
        } else {
            /* pass 1a: dq of the chosen rows, as in g2ref_attn_bwd */
#pragma omp for schedule(dynamic, 1)
            for (int64_t r = 0; r < nq; ++r) {
                const int64_t b = qrows[3 * r], i = qrows[3 * r + 1], h = qrows[3 * r + 2];
                one_row(q, k, v, b, i, h, T, S, H, Hkv, d, q_offset, query_scale, softcap,
                        window, qs, s, w, NULL, NULL);
                double* dqrow = dq + r * d;
                for (int64_t c = 0; c < d; ++c) dqrow[c] = 0.0;
                row_backward(k, v, dout, b, i, h, T, S, H, Hkv, d, query_scale, softcap, qs, w,
                             x, dqrow, NULL, NULL);
            }
            /* pass 1b: lse and D of every row of a (b, g) that has a chosen key */
#pragma omp for schedule(dynamic, 4)
            for (int64_t r = 0; r < B * T * H; ++r) {
                const int64_t b = r / (T * H);
                const int64_t i = (r / H) % T;
                const int64_t h = r % H;
                if (!need[b * Hkv + kv_head(h, H, Hkv)]) continue;
                double lse;
                one_row(q, k, v, b, i, h, T, S, H, Hkv, d, q_offset, query_scale, softcap,
                        window, qs, s, w, NULL, &lse);
                row_lse[(b * H + h) * T + i] = lse;
                row_D[(b * H + h) * T + i] = row_backward(k, v, dout, b, i, h, T, S, H, Hkv, d,
                                                          query_scale, softcap, qs, w, x, NULL,
                                                          NULL, NULL);
            }
            /* pass 2: dk and dv of each chosen key, summed over the rows of
             * both heads of its group that see it */
#pragma omp for schedule(dynamic, 1)
            for (int64_t r = 0; r < nk; ++r) {
                const int64_t b = keys[3 * r], j = keys[3 * r + 1], g = keys[3 * r + 2];
                const uint16_t* krow = k + ((b * S + j) * Hkv + g) * d;
                const uint16_t* vj = v + ((b * S + j) * Hkv + g) * d;
                double* dkrow = dk + r * d;
                double* dvrow = dv + r * d;
                for (int64_t c = 0; c < d; ++c) dkrow[c] = dvrow[c] = 0.0;
                for (int64_t h = g * group; h < (g + 1) * group; ++h) {
                    for (int64_t i = 0; i < T; ++i) {
                        if (!visible(i + q_offset, j, window)) continue;
                        const uint16_t* dorow = dout + ((b * T + i) * H + h) * d;
                        scaled_query(q + ((b * T + i) * H + h) * d, d, query_scale, qs);
                        /* x = (query_scale q) . k, the capped logit and its weight */
                        double xl = 0.0;
                        for (int64_t c = 0; c < d; ++c) xl += qs[c] * widen(krow[c]);
                        double sl = xl, cap_grad = 1.0;
                        if (softcap > 0.0) {
                            const double th = tanh(xl / softcap);
                            sl = softcap * th;
                            cap_grad = 1.0 - th * th;
                        }
                        const double wl = exp(sl - row_lse[(b * H + h) * T + i]);
                        double dw = 0.0;
                        for (int64_t c = 0; c < d; ++c) dw += widen(dorow[c]) * widen(vj[c]);
                        const double dx = wl * (dw - row_D[(b * H + h) * T + i]) * cap_grad;
                        for (int64_t c = 0; c < d; ++c) {
                            dkrow[c] += dx * qs[c];
                            dvrow[c] += wl * widen(dorow[c]);
                        }
                    }
                }
            }
        }
        free(qs);
        free(s);
        free(w);
        free(x);
    }
    free(need);
    free(row_lse);
    free(row_D);
    return err ? -1 : 0;
}

void g2ref_set_threads(int n) {
#ifdef _OPENMP
    if (n > 0) omp_set_num_threads(n);
#else
    (void)n;
#endif
}

int g2ref_max_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

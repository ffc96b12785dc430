/*
 * Oracle for causal grouped-query attention with rotary embeddings, forward
 * and backward, in plain fp64 C.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path links, loads or
 * calls this file; only the test suite, the smoke check and the benchmark's
 * CPU-baseline leg do.  It shares no source, header, table or helper with the
 * CUDA library and it never sees a value produced by it.
 *
 * What it computes (the plain definition, no tiling, no online softmax, the
 * full T x T score matrix of every head is materialised):
 *
 *   - Rotary position embedding on queries and keys, not on values
 *     ("NanoEuler" write-up, aimsg.uk, section 2 "Model components", RoPE
 *     bullet; agentlenshq.com summary, "Technical specification" list;
 *     "Tiny Hackable CUDA LM", aimsg.uk, section 1 "Architecture", RoPE
 *     bullet).  The pages fix neither base, pairing nor origin; this oracle
 *     rotates the interleaved pairs (x[2i], x[2i+1]) by the angle
 *     t * base^(-2i/D), with t = 0 .. T-1 the position in the sequence.
 *     base <= 0 switches the rotation off.
 *   - Scaled dot-product scores with scale 1/sqrt(D) and a causal mask
 *     (key j visible to query i iff j <= i) ("Tiny Hackable CUDA LM",
 *     section 1, causal attention and scaled dot-product bullets).
 *   - Softmax over each row, output O = P V, and the row log-sum-exp
 *     LSE_i = ln sum_j exp(s_ij) that the tiled forward keeps so that no
 *     T x T matrix stays in memory ("NanoEuler" write-up, section 4 "GPU
 *     version" bullet on FlashAttention).
 *   - Grouped-query attention: query head h reads key/value head
 *     g = floor(h / G), G = Hq / Hkv ("NanoEuler" write-up, section 2, GQA
 *     bullet; agentlenshq.com model-configuration table, 12/4 and 4/2 heads).
 *   - No bias and no additive mask other than the causal one ("NanoEuler"
 *     write-up, section 2, no-bias bullet).
 *   - Backward by the chain rule of the definition above, for an upstream
 *     gradient dO of O ("NanoEuler" write-up, section 3: every analytic
 *     gradient is hand-written and checked against double-precision central
 *     differences, which the tests here repeat on this oracle).
 *
 * Layouts: Q, O, dO, dQ are [B][T][Hq][D]; K, V, dK, dV are [B][T][Hkv][D];
 * LSE and Dvec are [B][Hq][T].  All row-major, contiguous, double.
 *
 * Parallelism: OpenMP over independent (batch, head) or (batch, kv-head)
 * units only; the arithmetic inside a unit is sequential.
 */
#include <math.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define ORACLE_OK 0
#define ORACLE_ERR_ARG 1
#define ORACLE_ERR_NOMEM 2

static int check_shape(int B, int T, int Hq, int Hkv, int D) {
    if (B < 0 || T < 0 || Hq < 1 || Hkv < 1 || D < 2 || (D % 2) != 0) return 0;
    if (Hq % Hkv != 0) return 0;
    return 1;
}

/* Rotation angle of pair i at position t: t * base^(-2i/D). */
static double rope_angle(int t, int i, int D, double base) {
    return (double)t * pow(base, -2.0 * (double)i / (double)D);
}

/* out = R_t x for one head vector of length D (interleaved pairs). */
static void rope_rotate(const double* x, double* out, int t, int D, double base) {
    if (base <= 0.0) {
        for (int d = 0; d < D; ++d) out[d] = x[d];
        return;
    }
    for (int i = 0; i < D / 2; ++i) {
        double a = rope_angle(t, i, D, base);
        double c = cos(a), s = sin(a);
        double x0 = x[2 * i], x1 = x[2 * i + 1];
        out[2 * i] = x0 * c - x1 * s;
        out[2 * i + 1] = x0 * s + x1 * c;
    }
}

/* out = R_t^T y (the transpose, i.e. inverse, rotation). */
static void rope_rotate_transpose(const double* y, double* out, int t, int D, double base) {
    if (base <= 0.0) {
        for (int d = 0; d < D; ++d) out[d] = y[d];
        return;
    }
    for (int i = 0; i < D / 2; ++i) {
        double a = rope_angle(t, i, D, base);
        double c = cos(a), s = sin(a);
        double y0 = y[2 * i], y1 = y[2 * i + 1];
        out[2 * i] = y0 * c + y1 * s;
        out[2 * i + 1] = -y0 * s + y1 * c;
    }
}

void oracle_set_threads(int n) {
#ifdef _OPENMP
    if (n > 0) omp_set_num_threads(n);
#else
    (void)n;
#endif
}

int oracle_get_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* Applies R_t to every head vector of X [B][T][H][D]. */
int oracle_rope(const double* X, double* Y, int B, int T, int H, int D, double base) {
    if (B < 0 || T < 0 || H < 1 || D < 2 || D % 2) return ORACLE_ERR_ARG;
    for (long bt = 0; bt < (long)B * T; ++bt) {
        int t = (int)(bt % T);
        for (int h = 0; h < H; ++h) {
            const double* x = X + (bt * H + h) * D;
            rope_rotate(x, Y + (bt * H + h) * D, t, D, base);
        }
    }
    return ORACLE_OK;
}

/*
 * Scores and probabilities of one (b, h): S[i][j] = scale * q'_i . k'_j,
 * masked to -inf for j > i when causal; P = row softmax of S; LSE per row.
 * Qr: [T][D] rotated queries of head h, Kr: [T][D] rotated keys of head g.
 */
static void head_probs(const double* Qr, const double* Kr, int T, int D, int causal,
                       double* P, double* lse) {
    const double scale = 1.0 / sqrt((double)D);
    for (int i = 0; i < T; ++i) {
        double* prow = P + (long)i * T;
        double m = -INFINITY;
        for (int j = 0; j < T; ++j) {
            if (causal && j > i) {
                prow[j] = -INFINITY;
                continue;
            }
            double acc = 0.0;
            for (int d = 0; d < D; ++d) acc += Qr[(long)i * D + d] * Kr[(long)j * D + d];
            prow[j] = scale * acc;
            if (prow[j] > m) m = prow[j];
        }
        double sum = 0.0;
        for (int j = 0; j < T; ++j) sum += (prow[j] == -INFINITY) ? 0.0 : exp(prow[j] - m);
        double L = m + log(sum);
        lse[i] = L;
        for (int j = 0; j < T; ++j) prow[j] = (prow[j] == -INFINITY) ? 0.0 : exp(prow[j] - L);
    }
}

/* Gathers head h of X [B][T][H][D] at batch b into out [T][D], rotated or not. */
static void gather_head(const double* X, double* out, int b, int h, int T, int H, int D,
                        double base, int rotate) {
    for (int t = 0; t < T; ++t) {
        const double* x = X + (((long)b * T + t) * H + h) * D;
        if (rotate)
            rope_rotate(x, out + (long)t * D, t, D, base);
        else
            memcpy(out + (long)t * D, x, sizeof(double) * D);
    }
}

/*
 * Forward: O [B][T][Hq][D] and LSE [B][Hq][T] (LSE may be NULL).
 */
int oracle_attn_fwd(const double* Q, const double* K, const double* V, double* O, double* LSE,
                    int B, int T, int Hq, int Hkv, int D, double base, int causal) {
    if (!check_shape(B, T, Hq, Hkv, D)) return ORACLE_ERR_ARG;
    if (B == 0 || T == 0) return ORACLE_OK;
    const int G = Hq / Hkv;
    int err = 0;
#pragma omp parallel for schedule(dynamic, 1)
    for (long bh = 0; bh < (long)B * Hq; ++bh) {
        int b = (int)(bh / Hq), h = (int)(bh % Hq), g = h / G;
        double* Qr = malloc(sizeof(double) * (size_t)T * D);
        double* Kr = malloc(sizeof(double) * (size_t)T * D);
        double* Vg = malloc(sizeof(double) * (size_t)T * D);
        double* P = malloc(sizeof(double) * (size_t)T * T);
        double* lse = malloc(sizeof(double) * (size_t)T);
        if (!Qr || !Kr || !Vg || !P || !lse) {
#pragma omp atomic write
            err = 1;
        } else {
            gather_head(Q, Qr, b, h, T, Hq, D, base, 1);
            gather_head(K, Kr, b, g, T, Hkv, D, base, 1);
            gather_head(V, Vg, b, g, T, Hkv, D, base, 0);
            head_probs(Qr, Kr, T, D, causal, P, lse);
            for (int i = 0; i < T; ++i) {
                double* o = O + (((long)b * T + i) * Hq + h) * D;
                for (int d = 0; d < D; ++d) o[d] = 0.0;
                for (int j = 0; j < T; ++j) {
                    double p = P[(long)i * T + j];
                    if (p == 0.0) continue;
                    for (int d = 0; d < D; ++d) o[d] += p * Vg[(long)j * D + d];
                }
                if (LSE) LSE[((long)b * Hq + h) * T + i] = lse[i];
            }
        }
        free(Qr); free(Kr); free(Vg); free(P); free(lse);
    }
    return err ? ORACLE_ERR_NOMEM : ORACLE_OK;
}

/*
 * Row-softmax probabilities of one (b, h) as a dense [T][T] matrix, for the
 * row-sum and shape checks.
 */
int oracle_attn_probs(const double* Q, const double* K, double* P, int B, int T, int Hq,
                      int Hkv, int D, double base, int causal, int b, int h) {
    if (!check_shape(B, T, Hq, Hkv, D) || b < 0 || b >= B || h < 0 || h >= Hq) return ORACLE_ERR_ARG;
    const int G = Hq / Hkv;
    double* Qr = malloc(sizeof(double) * (size_t)T * D);
    double* Kr = malloc(sizeof(double) * (size_t)T * D);
    double* lse = malloc(sizeof(double) * (size_t)T);
    if (!Qr || !Kr || !lse) { free(Qr); free(Kr); free(lse); return ORACLE_ERR_NOMEM; }
    gather_head(Q, Qr, b, h, T, Hq, D, base, 1);
    gather_head(K, Kr, b, h / G, T, Hkv, D, base, 1);
    head_probs(Qr, Kr, T, D, causal, P, lse);
    free(Qr); free(Kr); free(lse);
    return ORACLE_OK;
}

/*
 * Backward for upstream gradient dO: dQ [B][T][Hq][D], dK and dV
 * [B][T][Hkv][D].  Optionally returns O, LSE and the row term
 * Dvec_i = sum_j P_ij dP_ij (any of them may be NULL).
 *
 * Chain rule of the forward definition, per (b, h), g = floor(h/G):
 *   dV_g     += P^T dO
 *   dP        = dO V_g^T
 *   dS_ij     = P_ij (dP_ij - sum_k P_ik dP_ik)
 *   dQ'       = scale dS K'_g,        dQ = R^T dQ'   (per position)
 *   dK'_g    += scale dS^T Q'_h,      dK = R^T dK'
 * The sum over the G query heads of a group is taken inside one parallel
 * unit (b, g), so the accumulation needs no atomics.
 */
int oracle_attn_bwd(const double* Q, const double* K, const double* V, const double* dO,
                    double* dQ, double* dK, double* dV, double* O, double* LSE, double* Dvec,
                    int B, int T, int Hq, int Hkv, int D, double base, int causal) {
    if (!check_shape(B, T, Hq, Hkv, D)) return ORACLE_ERR_ARG;
    if (B == 0 || T == 0) return ORACLE_OK;
    const int G = Hq / Hkv;
    const double scale = 1.0 / sqrt((double)D);
    int err = 0;
#pragma omp parallel for schedule(dynamic, 1)
    for (long bg = 0; bg < (long)B * Hkv; ++bg) {
        int b = (int)(bg / Hkv), g = (int)(bg % Hkv);
        size_t td = (size_t)T * D;
        double* Qr = malloc(sizeof(double) * td);
        double* Kr = malloc(sizeof(double) * td);
        double* Vg = malloc(sizeof(double) * td);
        double* dOh = malloc(sizeof(double) * td);
        double* dKr = calloc(td, sizeof(double));
        double* dVg = calloc(td, sizeof(double));
        double* dQr = malloc(sizeof(double) * td);
        double* P = malloc(sizeof(double) * (size_t)T * T);
        double* dS = malloc(sizeof(double) * (size_t)T * T);
        double* lse = malloc(sizeof(double) * (size_t)T);
        double* tmp = malloc(sizeof(double) * (size_t)D);
        if (!Qr || !Kr || !Vg || !dOh || !dKr || !dVg || !dQr || !P || !dS || !lse || !tmp) {
#pragma omp atomic write
            err = 1;
            goto done;
        }
        gather_head(K, Kr, b, g, T, Hkv, D, base, 1);
        gather_head(V, Vg, b, g, T, Hkv, D, base, 0);
        for (int hh = 0; hh < G; ++hh) {
            int h = g * G + hh;
            gather_head(Q, Qr, b, h, T, Hq, D, base, 1);
            gather_head(dO, dOh, b, h, T, Hq, D, base, 0);
            head_probs(Qr, Kr, T, D, causal, P, lse);
            for (int i = 0; i < T; ++i) {
                const double* prow = P + (long)i * T;
                double* dsrow = dS + (long)i * T;
                const double* doi = dOh + (long)i * D;
                double rowdot = 0.0;
                for (int j = 0; j < T; ++j) {
                    double dp = 0.0;
                    for (int d = 0; d < D; ++d) dp += doi[d] * Vg[(long)j * D + d];
                    dsrow[j] = dp; /* dP for now */
                    rowdot += prow[j] * dp;
                }
                for (int j = 0; j < T; ++j) dsrow[j] = prow[j] * (dsrow[j] - rowdot);
                if (Dvec) Dvec[((long)b * Hq + h) * T + i] = rowdot;
                if (LSE) LSE[((long)b * Hq + h) * T + i] = lse[i];
                if (O) {
                    double* o = O + (((long)b * T + i) * Hq + h) * D;
                    for (int d = 0; d < D; ++d) o[d] = 0.0;
                    for (int j = 0; j < T; ++j)
                        for (int d = 0; d < D; ++d) o[d] += prow[j] * Vg[(long)j * D + d];
                }
            }
            /* dV_g += P^T dO ; dK'_g += scale dS^T Q' ; dQ' = scale dS K' */
            for (int i = 0; i < T; ++i) {
                const double* prow = P + (long)i * T;
                const double* dsrow = dS + (long)i * T;
                for (int j = 0; j < T; ++j) {
                    double p = prow[j], ds = dsrow[j];
                    for (int d = 0; d < D; ++d) {
                        dVg[(long)j * D + d] += p * dOh[(long)i * D + d];
                        dKr[(long)j * D + d] += scale * ds * Qr[(long)i * D + d];
                    }
                }
                double* dq = dQr + (long)i * D;
                for (int d = 0; d < D; ++d) dq[d] = 0.0;
                for (int j = 0; j < T; ++j) {
                    double ds = dsrow[j];
                    for (int d = 0; d < D; ++d) dq[d] += scale * ds * Kr[(long)j * D + d];
                }
                rope_rotate_transpose(dq, tmp, i, D, base);
                memcpy(dQ + (((long)b * T + i) * Hq + h) * D, tmp, sizeof(double) * D);
            }
        }
        for (int j = 0; j < T; ++j) {
            rope_rotate_transpose(dKr + (long)j * D, tmp, j, D, base);
            memcpy(dK + (((long)b * T + j) * Hkv + g) * D, tmp, sizeof(double) * D);
            memcpy(dV + (((long)b * T + j) * Hkv + g) * D, dVg + (long)j * D, sizeof(double) * D);
        }
    done:
        free(Qr); free(Kr); free(Vg); free(dOh); free(dKr); free(dVg); free(dQr);
        free(P); free(dS); free(lse); free(tmp);
    }
    return err ? ORACLE_ERR_NOMEM : ORACLE_OK;
}

/*
 * Decode attention over a key/value cache: one new query per sequence
 * attends to the cached positions 0 .. len_b - 1, the last of which is its
 * own (the generation path of the same causal attention: "NanoEuler"
 * write-up, aimsg.uk, section 1, head-0 generation; the scores, softmax and
 * GQA head map as in oracle_attn_fwd).
 *
 *   Q   [B][Hq][D]     un-rotated query of the token at position len_b - 1
 *   Kc  [B][Tc][Hkv][D] cached keys, already rotated at their positions
 *   Vc  [B][Tc][Hkv][D] cached values
 *   lens[B]            valid cache length, 0 <= len_b <= Tc
 *   O   [B][Hq][D], LSE [B][Hq]
 *
 * q' = R_{len_b - 1} q; s_j = q' . k_j / sqrt(D) for j < len_b;
 * LSE = ln sum_j exp(s_j); O = sum_j exp(s_j - LSE) v_j.  An empty cache
 * (len_b = 0) gives O = 0 and LSE = -inf.
 */
int oracle_attn_decode(const double* Q, const double* Kc, const double* Vc, const int* lens, double* O,
                       double* LSE, int B, int Tc, int Hq, int Hkv, int D, double rope_base) {
    if (!check_shape(B, Tc, Hq, Hkv, D)) return ORACLE_ERR_ARG;
    for (int b = 0; b < B; ++b)
        if (lens[b] < 0 || lens[b] > Tc) return ORACLE_ERR_ARG;
    const int G = Hq / Hkv;
    const double scale = 1.0 / sqrt((double)D);
    int err = 0;
#pragma omp parallel for schedule(dynamic) reduction(| : err)
    for (long bh = 0; bh < (long)B * Hq; ++bh) {
        const int b = (int)(bh / Hq), h = (int)(bh % Hq), g = h / G, len = lens[b];
        double* o = O + bh * D;
        double* qr = (double*)malloc(sizeof(double) * D);
        double* s = (double*)malloc(sizeof(double) * (len > 0 ? len : 1));
        if (!qr || !s) {
            err |= 1;
            free(qr);
            free(s);
            continue;
        }
        for (int d = 0; d < D; ++d) o[d] = 0.0;
        if (len == 0) {
            LSE[bh] = -INFINITY;
        } else {
            rope_rotate(Q + bh * D, qr, len - 1, D, rope_base);
            double m = -INFINITY;
            for (int j = 0; j < len; ++j) {
                const double* k = Kc + (((long)b * Tc + j) * Hkv + g) * D;
                double acc = 0.0;
                for (int d = 0; d < D; ++d) acc += qr[d] * k[d];
                s[j] = scale * acc;
                if (s[j] > m) m = s[j];
            }
            double l = 0.0;
            for (int j = 0; j < len; ++j) l += exp(s[j] - m);
            const double lse = m + log(l);
            for (int j = 0; j < len; ++j) {
                const double p = exp(s[j] - lse);
                const double* v = Vc + (((long)b * Tc + j) * Hkv + g) * D;
                for (int d = 0; d < D; ++d) o[d] += p * v[d];
            }
            LSE[bh] = lse;
        }
        free(qr);
        free(s);
    }
    return err ? ORACLE_ERR_NOMEM : ORACLE_OK;
}

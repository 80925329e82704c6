/*
 * hlta_oracle.c -- plain fp64 CPU oracle of the Hybrid Linear Temporal
 * Attention forward pass (Kairos, arXiv 2606.16533, section 2.2).
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path links, loads or calls
 * this file: only the tests, the package's smoke check and the benchmark's CPU
 * baseline do.  It shares no code with the CUDA library.
 *
 * Everything is computed in double precision.  Inputs arrive either as float32
 * arrays or as bf16 bit patterns (uint16); both hold exact values that are
 * widened to double before use.
 *
 * Layouts (row-major):
 *   q, k : [B, L, H, d_k]      v, out : [B, L, H, d_v]
 *   alpha, beta : [B, L, H] float32
 *   S : [B, H, d_v, d_k] double (S maps keys to values: v ~ S k)
 *
 * Functions and the passages they follow:
 *   oracle_attention  -- section 2.2.2, Eq. (7) (SWA) and Eq. (8) (DSWA), with
 *                        the causal window and residue-class dilation readings
 *                        documented beside each predicate below.
 *   oracle_attention_centred -- the same with the centred window Eq. (7) prints
 *                        (the diffusion in-clip reading) and, optionally, rotary
 *                        position embedding on q and k (the pages name RoPE on the
 *                        sliding-window blocks; the rotation below is a reading).
 *   oracle_gdn        -- section 2.2.1, steps 2-4 (Eq. (2)-(6)) and the output
 *                        o_t = S_t q_t.
 *   oracle_gdn_chunked-- the same recurrence regrouped into chunks (a
 *                        derivation from Eq. (6), not on the pages); used only to
 *                        show that the chunk form computes the recurrence.
 *   oracle_attention_backward, oracle_gdn_backward -- reverse-mode derivatives
 *                        of the two forward definitions (the chain rule applied
 *                        to them step by step; the pages print no backward).
 *
 * Parity pins for every function live in tests/test_oracle.py.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#ifdef _OPENMP
#include <omp.h>
#endif

/* dtype codes of input tensors */
#define ORC_F32 0
#define ORC_BF16 1

static inline double load_elem(const void *p, int dt, size_t i) {
    if (dt == ORC_BF16) {
        uint32_t u = ((uint32_t)((const uint16_t *)p)[i]) << 16;
        float f;
        memcpy(&f, &u, sizeof f);
        return (double)f;
    }
    return (double)((const float *)p)[i];
}

/* ------------------------------------------------------------------------ */
/* Attention masks (section 2.2.2).                                          */
/* ------------------------------------------------------------------------ */

/* SWA, Eq. (7), causal reading: query i sees the w most recent keys including
 * itself, i - w < j <= i.  (The equation prints a centred window; the layer
 * built here is causal.) */
static inline int swa_in_window(long i, long j, long w) {
    return j <= i && j > i - w;
}

/* DSWA, Eq. (8): SWA applied after rearranging (B, F*P, D) -> (B*d, F/d*P, D).
 * Reading: frames are split into d residue classes f mod d; within one class
 * the frames f = g, g+d, g+2d, ... are concatenated in order, so token
 * t = f*P + s sits at rearranged position r(t) = floor(f/d)*P + s.  Query i
 * sees key j iff both are in the same class and 0 <= r(i) - r(j) < w. */
static inline long rearranged_pos(long t, long P, long dil) {
    long f = t / P, s = t % P;
    return (f / dil) * P + s;
}

static inline int dswa_in_window(long i, long j, long P, long dil, long w) {
    long fi = i / P, fj = j / P;
    if ((fi - fj) % dil != 0) return 0;
    long dr = rearranged_pos(i, P, dil) - rearranged_pos(j, P, dil);
    return dr >= 0 && dr < w;
}

/* Centred reading of Eq. (7): key j is admitted iff |i - j| <= floor(w/2) (for
 * DSWA: in the same residue class and |r(i) - r(j)| <= floor(w/2)). */
static inline int swa_in_centred(long i, long j, long w) {
    long d = i - j;
    return (d < 0 ? -d : d) <= w / 2;
}

static inline int dswa_in_centred(long i, long j, long P, long dil, long w) {
    long fi = i / P, fj = j / P;
    if ((fi - fj) % dil != 0) return 0;
    long dr = rearranged_pos(i, P, dil) - rearranged_pos(j, P, dil);
    return (dr < 0 ? -dr : dr) <= w / 2;
}

/* Rotary position embedding (reading): for token position t and channel pair
 * (2m, 2m+1), m < d/2, rotate (x_2m, x_2m+1) by the angle t * base^(-2m/d). */
static void rope_rotate(double *x, int d, long t, double base) {
    for (int m = 0; 2 * m + 1 < d; ++m) {
        double theta = (double)t * pow(base, -2.0 * m / (double)d);
        double c = cos(theta), sn = sin(theta);
        double a = x[2 * m], b = x[2 * m + 1];
        x[2 * m] = a * c - b * sn;
        x[2 * m + 1] = a * sn + b * c;
    }
}

/*
 * oracle_attention: softmax attention rows under the SWA (kind 0) or DSWA
 * (kind 1) mask.
 *
 *   logits_j = q_i . k_j / sqrt(d_k) over every key j the mask admits;
 *   p = softmax(logits) (max-subtracted, fp64 sums);  o_i = sum_j p_j v_j.
 *
 * rows: nrows row ids, id = (b*L + t)*H + h, or NULL for all B*L*H rows in
 * that order.  out: [nrows, d_v] doubles.
 * span: keys are examined over j in [max(0, i - span), i]; pass span < 0 to
 * examine every j <= i.  The predicate alone decides membership, so any span
 * at least as large as the farthest admitted key gives the same result.
 * Returns 0, or -1 on bad arguments.
 */
static int attention_core(int kind, int centred, double rope_base, int B, int L, int H, int d_k,
                          int d_v, int P, int dil, int w, const void *q, const void *k, const void *v,
                          int dt, long nrows, const long long *rows, long span, double *out) {
    if (B <= 0 || L <= 0 || H <= 0 || d_k <= 0 || d_v <= 0 || P <= 0 || dil <= 0 || w <= 0)
        return -1;
    if (kind != 0 && kind != 1) return -1;
    if (rope_base < 0.0 || (rope_base > 0.0 && d_k % 2 != 0)) return -1;
    const double scale = 1.0 / sqrt((double)d_k);

#pragma omp parallel
    {
        double *logit = (double *)malloc(sizeof(double) * (size_t)L);
        double *qi = (double *)malloc(sizeof(double) * (size_t)d_k);
        double *kj = (double *)malloc(sizeof(double) * (size_t)d_k);
#pragma omp for schedule(dynamic, 16)
        for (long r = 0; r < nrows; ++r) {
            long long id = rows ? rows[r] : (long long)r;
            long h = (long)(id % H);
            long t = (long)((id / H) % L);
            long b = (long)(id / ((long long)H * L));
            size_t qoff = (((size_t)b * L + t) * H + h) * d_k;
            for (int c = 0; c < d_k; ++c) qi[c] = load_elem(q, dt, qoff + c);
            if (rope_base > 0.0) rope_rotate(qi, d_k, t, rope_base);
            long lo = (span < 0 || t - span < 0) ? 0 : t - span;
            long hi = !centred ? t : ((span < 0 || t + span > L - 1) ? L - 1 : t + span);
            double m = -INFINITY;
            for (long j = lo; j <= hi; ++j) {
                int in;
                if (centred)
                    in = kind == 0 ? swa_in_centred(t, j, w) : dswa_in_centred(t, j, P, dil, w);
                else
                    in = kind == 0 ? swa_in_window(t, j, w) : dswa_in_window(t, j, P, dil, w);
                if (!in) {
                    logit[j] = NAN; /* marks a masked key */
                    continue;
                }
                size_t koff = (((size_t)b * L + j) * H + h) * d_k;
                for (int c = 0; c < d_k; ++c) kj[c] = load_elem(k, dt, koff + c);
                if (rope_base > 0.0) rope_rotate(kj, d_k, j, rope_base);
                double s = 0.0;
                for (int c = 0; c < d_k; ++c) s += qi[c] * kj[c];
                s *= scale;
                logit[j] = s;
                if (s > m) m = s;
            }
            double *o = out + (size_t)r * d_v;
            for (int c = 0; c < d_v; ++c) o[c] = 0.0;
            double denom = 0.0;
            for (long j = lo; j <= hi; ++j) {
                if (isnan(logit[j])) continue;
                double p = exp(logit[j] - m);
                denom += p;
                size_t voff = (((size_t)b * L + j) * H + h) * d_v;
                for (int c = 0; c < d_v; ++c) o[c] += p * load_elem(v, dt, voff + c);
            }
            for (int c = 0; c < d_v; ++c) o[c] /= denom;
        }
        free(logit);
        free(qi);
        free(kj);
    }
    return 0;
}

int oracle_attention(int kind, int B, int L, int H, int d_k, int d_v, int P, int dil, int w,
                     const void *q, const void *k, const void *v, int dt, long nrows,
                     const long long *rows, long span, double *out) {
    return attention_core(kind, 0, 0.0, B, L, H, d_k, d_v, P, dil, w, q, k, v, dt, nrows, rows, span,
                          out);
}

/*
 * oracle_attention_centred: as oracle_attention with the centred window
 * (|r(i) - r(j)| <= floor(w/2), see the predicates above) and, when
 * rope_base > 0, q and k rotated by rope_rotate at their token positions before
 * the dot product.  span bounds |i - j| from above (< 0: every key).
 */
int oracle_attention_centred(int kind, double rope_base, int B, int L, int H, int d_k, int d_v, int P,
                             int dil, int w, const void *q, const void *k, const void *v, int dt,
                             long nrows, const long long *rows, long span, double *out) {
    return attention_core(kind, 1, rope_base, B, L, H, d_k, d_v, P, dil, w, q, k, v, dt, nrows, rows,
                          span, out);
}

/* ------------------------------------------------------------------------ */
/* Gated delta memory (section 2.2.1).                                       */
/* ------------------------------------------------------------------------ */

/*
 * oracle_gdn: the token-by-token recurrence for every (b, h).
 *
 * variant 0 (the layer built here): retrieval reads the decayed state,
 *     v_old = (alpha_t S_{t-1}) k_t                       (Eq. 2 on alpha*S)
 *     v_new = beta_t v_t + (1 - beta_t) v_old             (Eq. 2)
 *     S_t   = alpha_t S_{t-1} - v_old k_t^T + v_new k_t^T (Eq. 5)
 *   which equals alpha_t S_{t-1} (I - beta_t k_t k_t^T) + beta_t v_t k_t^T.
 * variant 1 (the equations as printed): v_old = S_{t-1} k_t, then Eq. (2) and
 *   Eq. (5), i.e. Eq. (6): S_t = alpha_t S_{t-1} + beta_t (v_t - v_old) k_t^T.
 * matrix_form != 0 evaluates variant 0 as the explicit product
 *   alpha_t S_{t-1} (I - beta_t k_t k_t^T) + beta_t v_t k_t^T
 * (d_k x d_k matrix products), for the self-consistency pin.
 *
 * Output (step 4): o_t = S_t q_t, from the updated state.
 * S0: [B,H,d_v,d_k] or NULL (zero state).  S_out: final state or NULL.
 * out: [B,L,H,d_v] or NULL.  Returns 0, or -1 on bad arguments.
 */
int oracle_gdn(int B, int L, int H, int d_k, int d_v, const void *q, const void *k,
               const void *v, int dt, const float *alpha, const float *beta,
               const double *S0, double *S_out, double *out, int variant, int matrix_form) {
    if (B <= 0 || L < 0 || H <= 0 || d_k <= 0 || d_v <= 0) return -1;
    if (variant != 0 && variant != 1) return -1;
    if (matrix_form && variant != 0) return -1;

#pragma omp parallel for collapse(2) schedule(static)
    for (int b = 0; b < B; ++b) {
        for (int h = 0; h < H; ++h) {
            size_t sd = (size_t)d_v * d_k;
            double *S = (double *)malloc(sizeof(double) * sd);
            double *kt = (double *)malloc(sizeof(double) * d_k);
            double *qt = (double *)malloc(sizeof(double) * d_k);
            double *vt = (double *)malloc(sizeof(double) * d_v);
            double *vold = (double *)malloc(sizeof(double) * d_v);
            double *G = matrix_form ? (double *)malloc(sizeof(double) * (size_t)d_k * d_k) : NULL;
            double *T = matrix_form ? (double *)malloc(sizeof(double) * sd) : NULL;
            if (S0)
                memcpy(S, S0 + ((size_t)b * H + h) * sd, sizeof(double) * sd);
            else
                memset(S, 0, sizeof(double) * sd);

            for (int t = 0; t < L; ++t) {
                size_t row = ((size_t)b * L + t) * H + h;
                double a = (double)alpha[row], be = (double)beta[row];
                for (int c = 0; c < d_k; ++c) {
                    kt[c] = load_elem(k, dt, row * d_k + c);
                    qt[c] = load_elem(q, dt, row * d_k + c);
                }
                for (int c = 0; c < d_v; ++c) vt[c] = load_elem(v, dt, row * d_v + c);

                if (matrix_form) {
                    /* G = I - beta k k^T ; T = S G ; S = alpha T + beta v k^T */
                    for (int i = 0; i < d_k; ++i)
                        for (int j = 0; j < d_k; ++j)
                            G[(size_t)i * d_k + j] = (i == j ? 1.0 : 0.0) - be * kt[i] * kt[j];
                    for (int i = 0; i < d_v; ++i)
                        for (int j = 0; j < d_k; ++j) {
                            double s = 0.0;
                            for (int c = 0; c < d_k; ++c) s += S[(size_t)i * d_k + c] * G[(size_t)c * d_k + j];
                            T[(size_t)i * d_k + j] = s;
                        }
                    for (int i = 0; i < d_v; ++i)
                        for (int j = 0; j < d_k; ++j)
                            S[(size_t)i * d_k + j] = a * T[(size_t)i * d_k + j] + be * vt[i] * kt[j];
                } else {
                    /* retrieval: v_old = S' k with S' = alpha S (variant 0) or S (variant 1) */
                    double ret_scale = variant == 0 ? a : 1.0;
                    for (int i = 0; i < d_v; ++i) {
                        double s = 0.0;
                        for (int c = 0; c < d_k; ++c) s += S[(size_t)i * d_k + c] * kt[c];
                        vold[i] = ret_scale * s;
                    }
                    for (int i = 0; i < d_v; ++i) {
                        double vnew = be * vt[i] + (1.0 - be) * vold[i];
                        for (int c = 0; c < d_k; ++c) {
                            double *sij = &S[(size_t)i * d_k + c];
                            /* decay, remove the old association, write the new one */
                            *sij = a * (*sij) - vold[i] * kt[c] + vnew * kt[c];
                        }
                    }
                }
                if (out) {
                    double *o = out + row * d_v;
                    for (int i = 0; i < d_v; ++i) {
                        double s = 0.0;
                        for (int c = 0; c < d_k; ++c) s += S[(size_t)i * d_k + c] * qt[c];
                        o[i] = s;
                    }
                }
            }
            if (S_out) memcpy(S_out + ((size_t)b * H + h) * sd, S, sizeof(double) * sd);
            free(S);
            free(kt);
            free(qt);
            free(vt);
            free(vold);
            free(G);
            free(T);
        }
    }
    return 0;
}

/*
 * oracle_gdn_chunked: variant 0 of oracle_gdn regrouped into chunks of C
 * tokens.  Not on the pages; derived from the recurrence as follows.  Write
 * S_t = alpha_t S_{t-1} + u_t k_t^T with u_t = beta_t (v_t - alpha_t S_{t-1} k_t).
 * Inside a chunk with start state S0 and decay ratios g(t,s) = prod_{s<r<=t}
 * alpha_r (g(t,s) = exp(l_t - l_s), l = running sum of log alpha, l_0 = 0 at the
 * chunk start, positions numbered from 1):
 *   S_t = g(t,0) S0 + sum_{s<=t} g(t,s) u_s k_s^T
 *   u_t + beta_t sum_{s<t} g(t,s) (k_t . k_s) u_s = beta_t v_t - beta_t g(t,0) S0 k_t
 *   o_t = g(t,0) S0 q_t + sum_{s<=t} g(t,s) (q_t . k_s) u_s
 *   S_C = g(C,0) S0 + sum_s g(C,s) u_s k_s^T.
 * The unit-lower-triangular system for u is solved by forward substitution.
 * Same arguments as oracle_gdn (variant 0 only).
 */
int oracle_gdn_chunked(int B, int L, int H, int d_k, int d_v, const void *q, const void *k,
                       const void *v, int dt, const float *alpha, const float *beta,
                       const double *S0, double *S_out, double *out, int C) {
    if (B <= 0 || L < 0 || H <= 0 || d_k <= 0 || d_v <= 0 || C <= 0) return -1;

#pragma omp parallel for collapse(2) schedule(static)
    for (int b = 0; b < B; ++b) {
        for (int h = 0; h < H; ++h) {
            size_t sd = (size_t)d_v * d_k;
            double *S = (double *)malloc(sizeof(double) * sd);
            double *Kc = (double *)malloc(sizeof(double) * (size_t)C * d_k);
            double *Qc = (double *)malloc(sizeof(double) * (size_t)C * d_k);
            double *Vc = (double *)malloc(sizeof(double) * (size_t)C * d_v);
            double *U = (double *)malloc(sizeof(double) * (size_t)C * d_v);
            double *ell = (double *)malloc(sizeof(double) * (size_t)(C + 1));
            double *bt = (double *)malloc(sizeof(double) * (size_t)C);
            double *Snew = (double *)malloc(sizeof(double) * sd);
            if (S0)
                memcpy(S, S0 + ((size_t)b * H + h) * sd, sizeof(double) * sd);
            else
                memset(S, 0, sizeof(double) * sd);

            for (int t0 = 0; t0 < L; t0 += C) {
                int n = (L - t0 < C) ? L - t0 : C;
                ell[0] = 0.0;
                for (int i = 0; i < n; ++i) {
                    size_t row = ((size_t)b * L + t0 + i) * H + h;
                    ell[i + 1] = ell[i] + log((double)alpha[row]);
                    bt[i] = (double)beta[row];
                    for (int c = 0; c < d_k; ++c) {
                        Kc[(size_t)i * d_k + c] = load_elem(k, dt, row * d_k + c);
                        Qc[(size_t)i * d_k + c] = load_elem(q, dt, row * d_k + c);
                    }
                    for (int c = 0; c < d_v; ++c) Vc[(size_t)i * d_v + c] = load_elem(v, dt, row * d_v + c);
                }
                /* forward substitution for u (rows of U) */
                for (int i = 0; i < n; ++i) {
                    double g0 = exp(ell[i + 1]);
                    for (int c = 0; c < d_v; ++c) {
                        double sk = 0.0;
                        for (int e = 0; e < d_k; ++e) sk += S[(size_t)c * d_k + e] * Kc[(size_t)i * d_k + e];
                        U[(size_t)i * d_v + c] = bt[i] * Vc[(size_t)i * d_v + c] - bt[i] * g0 * sk;
                    }
                    for (int s = 0; s < i; ++s) {
                        double kk = 0.0;
                        for (int e = 0; e < d_k; ++e) kk += Kc[(size_t)i * d_k + e] * Kc[(size_t)s * d_k + e];
                        double a_is = bt[i] * exp(ell[i + 1] - ell[s + 1]) * kk;
                        for (int c = 0; c < d_v; ++c) U[(size_t)i * d_v + c] -= a_is * U[(size_t)s * d_v + c];
                    }
                }
                /* outputs */
                if (out) {
                    for (int i = 0; i < n; ++i) {
                        size_t row = ((size_t)b * L + t0 + i) * H + h;
                        double g0 = exp(ell[i + 1]);
                        double *o = out + row * d_v;
                        for (int c = 0; c < d_v; ++c) {
                            double sq = 0.0;
                            for (int e = 0; e < d_k; ++e) sq += S[(size_t)c * d_k + e] * Qc[(size_t)i * d_k + e];
                            o[c] = g0 * sq;
                        }
                        for (int s = 0; s <= i; ++s) {
                            double qk = 0.0;
                            for (int e = 0; e < d_k; ++e) qk += Qc[(size_t)i * d_k + e] * Kc[(size_t)s * d_k + e];
                            double coef = exp(ell[i + 1] - ell[s + 1]) * qk;
                            for (int c = 0; c < d_v; ++c) o[c] += coef * U[(size_t)s * d_v + c];
                        }
                    }
                }
                /* state at the chunk end */
                double gC = exp(ell[n]);
                for (int c = 0; c < d_v; ++c)
                    for (int e = 0; e < d_k; ++e) {
                        double s = gC * S[(size_t)c * d_k + e];
                        for (int i = 0; i < n; ++i)
                            s += exp(ell[n] - ell[i + 1]) * U[(size_t)i * d_v + c] * Kc[(size_t)i * d_k + e];
                        Snew[(size_t)c * d_k + e] = s;
                    }
                memcpy(S, Snew, sizeof(double) * sd);
            }
            if (S_out) memcpy(S_out + ((size_t)b * H + h) * sd, S, sizeof(double) * sd);
            free(S);
            free(Kc);
            free(Qc);
            free(Vc);
            free(U);
            free(ell);
            free(bt);
            free(Snew);
        }
    }
    return 0;
}

/* Number of threads the OpenMP runtime will use (1 without OpenMP). */
int oracle_num_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* ------------------------------------------------------------------------ */
/* Backward pass (reverse-mode derivatives of the functions above).         */
/* The pages train the layer but print no backward formulas; the ones below */
/* are the chain rule applied to the forward definitions, step by step.     */
/* ------------------------------------------------------------------------ */

/* Transpose of rope_rotate: maps the gradient of the rotated vector to the
 * gradient of the unrotated one (rotation by -theta). */
static void rope_unrotate(double *g, int d, long t, double base) {
    for (int m = 0; 2 * m + 1 < d; ++m) {
        double theta = (double)t * pow(base, -2.0 * m / (double)d);
        double c = cos(theta), sn = sin(theta);
        double a = g[2 * m], b = g[2 * m + 1];
        g[2 * m] = a * c + b * sn;
        g[2 * m + 1] = -a * sn + b * c;
    }
}

/*
 * oracle_attention_backward: derivatives of the attention rows of
 * attention_core (same kind / centred / rope_base / window arguments) with
 * respect to q, k and v, given dO = dLoss/dO for every row [B,L,H,d_v].
 * For query i with admitted keys J(i), logits s_j = q_i.k_j / sqrt(d_k) and
 * p = softmax(s):
 *   dv_j += p_j dO_i
 *   dp_j  = dO_i . v_j,   ds_j = p_j (dp_j - sum_m p_m dp_m)
 *   dq_i += sum_j ds_j k_j / sqrt(d_k),   dk_j += ds_j q_i / sqrt(d_k)
 * With rotary embedding q, k above are the rotated vectors and the results are
 * mapped back through the transposed rotation.
 * dq, dk: [B,L,H,d_k], dv: [B,L,H,d_v] doubles, overwritten.  Every key is
 * examined (no span bound).  Returns 0, or -1 on bad arguments.
 */
int oracle_attention_backward(int kind, int centred, double rope_base, int B, int L, int H, int d_k,
                              int d_v, int P, int dil, int w, const void *q, const void *k,
                              const void *v, int dt, const double *dO, double *dq, double *dk,
                              double *dv) {
    if (B <= 0 || L <= 0 || H <= 0 || d_k <= 0 || d_v <= 0 || P <= 0 || dil <= 0 || w <= 0)
        return -1;
    if (kind != 0 && kind != 1) return -1;
    if (rope_base < 0.0 || (rope_base > 0.0 && (d_k % 2 != 0 || !centred))) return -1;
    const double scale = 1.0 / sqrt((double)d_k);
    memset(dq, 0, sizeof(double) * (size_t)B * L * H * d_k);
    memset(dk, 0, sizeof(double) * (size_t)B * L * H * d_k);
    memset(dv, 0, sizeof(double) * (size_t)B * L * H * d_v);

    /* keys accumulate over queries, so one thread owns one (b, h) */
#pragma omp parallel for collapse(2) schedule(dynamic, 1)
    for (int b = 0; b < B; ++b) {
        for (int h = 0; h < H; ++h) {
            double *Qr = (double *)malloc(sizeof(double) * (size_t)L * d_k);
            double *Kr = (double *)malloc(sizeof(double) * (size_t)L * d_k);
            double *dQr = (double *)calloc((size_t)L * d_k, sizeof(double));
            double *dKr = (double *)calloc((size_t)L * d_k, sizeof(double));
            double *p = (double *)malloc(sizeof(double) * (size_t)L);
            double *dp = (double *)malloc(sizeof(double) * (size_t)L);
            for (long t = 0; t < L; ++t) {
                size_t off = (((size_t)b * L + t) * H + h) * d_k;
                for (int c = 0; c < d_k; ++c) {
                    Qr[(size_t)t * d_k + c] = load_elem(q, dt, off + c);
                    Kr[(size_t)t * d_k + c] = load_elem(k, dt, off + c);
                }
                if (rope_base > 0.0) {
                    rope_rotate(Qr + (size_t)t * d_k, d_k, t, rope_base);
                    rope_rotate(Kr + (size_t)t * d_k, d_k, t, rope_base);
                }
            }
            for (long i = 0; i < L; ++i) {
                const double *qi = Qr + (size_t)i * d_k;
                const double *dOi = dO + (((size_t)b * L + i) * H + h) * d_v;
                double m = -INFINITY;
                for (long j = 0; j < L; ++j) {
                    int in;
                    if (centred)
                        in = kind == 0 ? swa_in_centred(i, j, w) : dswa_in_centred(i, j, P, dil, w);
                    else
                        in = kind == 0 ? swa_in_window(i, j, w) : dswa_in_window(i, j, P, dil, w);
                    if (!in) {
                        p[j] = NAN;
                        continue;
                    }
                    double s = 0.0;
                    for (int c = 0; c < d_k; ++c) s += qi[c] * Kr[(size_t)j * d_k + c];
                    p[j] = s * scale;
                    if (p[j] > m) m = p[j];
                }
                double denom = 0.0;
                for (long j = 0; j < L; ++j)
                    if (!isnan(p[j])) {
                        p[j] = exp(p[j] - m);
                        denom += p[j];
                    }
                double pdp = 0.0;
                for (long j = 0; j < L; ++j) {
                    if (isnan(p[j])) continue;
                    p[j] /= denom;
                    size_t voff = (((size_t)b * L + j) * H + h) * d_v;
                    double s = 0.0;
                    for (int c = 0; c < d_v; ++c) s += dOi[c] * load_elem(v, dt, voff + c);
                    dp[j] = s;
                    pdp += p[j] * s;
                }
                for (long j = 0; j < L; ++j) {
                    if (isnan(p[j])) continue;
                    double ds = p[j] * (dp[j] - pdp) * scale;
                    for (int c = 0; c < d_k; ++c) {
                        dQr[(size_t)i * d_k + c] += ds * Kr[(size_t)j * d_k + c];
                        dKr[(size_t)j * d_k + c] += ds * qi[c];
                    }
                    double *dvj = dv + (((size_t)b * L + j) * H + h) * d_v;
                    for (int c = 0; c < d_v; ++c) dvj[c] += p[j] * dOi[c];
                }
            }
            for (long t = 0; t < L; ++t) {
                if (rope_base > 0.0) {
                    rope_unrotate(dQr + (size_t)t * d_k, d_k, t, rope_base);
                    rope_unrotate(dKr + (size_t)t * d_k, d_k, t, rope_base);
                }
                size_t off = (((size_t)b * L + t) * H + h) * d_k;
                memcpy(dq + off, dQr + (size_t)t * d_k, sizeof(double) * d_k);
                memcpy(dk + off, dKr + (size_t)t * d_k, sizeof(double) * d_k);
            }
            free(Qr);
            free(Kr);
            free(dQr);
            free(dKr);
            free(p);
            free(dp);
        }
    }
    return 0;
}

/* One step of the recurrence in the form oracle_gdn_backward uses:
 * Sn = alpha Sp + u k^T, u = beta (v - rho Sp k), rho = alpha (variant 0) or 1. */
static void gdn_step(const double *Sp, double *Sn, const double *kt, const double *vt, double a,
                     double be, int variant, int d_k, int d_v) {
    const double rho = variant == 0 ? a : 1.0;
    for (int e = 0; e < d_v; ++e) {
        double s = 0.0;
        for (int c = 0; c < d_k; ++c) s += Sp[(size_t)e * d_k + c] * kt[c];
        const double u = be * (vt[e] - rho * s);
        for (int c = 0; c < d_k; ++c) Sn[(size_t)e * d_k + c] = a * Sp[(size_t)e * d_k + c] + u * kt[c];
    }
}

/*
 * oracle_gdn_backward: derivatives of oracle_gdn (variant 0 or 1) with respect
 * to q, k, v, alpha, beta and the initial state, given dO [B,L,H,d_v] and
 * dS_final [B,H,d_v,d_k] (NULL: zero), the gradient of the final state.
 *
 * Both variants write the update as S_t = alpha_t S_{t-1} + u_t k_t^T with the
 * retrieval r_t = S_{t-1} k_t and u_t = beta_t (v_t - rho_t r_t), rho_t = alpha_t
 * (variant 0) or 1 (variant 1).  Walking t = L-1 .. 0 with G the gradient of
 * S_t (G starts at dS_final):
 *   G    += dO_t q_t^T;          dq_t = S_t^T dO_t
 *   du    = G k_t;               dv_t = beta_t du;   dbeta_t = du . (v_t - rho_t r_t)
 *   dr    = -beta_t rho_t du;    dalpha_t = <G, S_{t-1}> (+ -beta_t du . r_t, variant 0)
 *   dk_t  = G^T u_t + S_{t-1}^T dr
 *   G    <- alpha_t G + dr k_t^T  (the gradient of S_{t-1})
 * and dS0 = G at the end.  S_{t-1} is needed in reverse order: the states at
 * every 64th step are kept from a first forward sweep, and the states inside
 * one such segment are recomputed from its first state by the same recurrence.
 * Outputs (doubles, overwritten): dq, dk [B,L,H,d_k], dv [B,L,H,d_v], dalpha,
 * dbeta [B,L,H], dS0 [B,H,d_v,d_k] or NULL.  Returns 0, or -1 on bad arguments.
 */
int oracle_gdn_backward(int B, int L, int H, int d_k, int d_v, const void *q, const void *k,
                        const void *v, int dt, const float *alpha, const float *beta,
                        const double *S0, const double *dO, const double *dS_final, double *dq,
                        double *dk, double *dv, double *dalpha, double *dbeta, double *dS0,
                        int variant) {
    if (B <= 0 || L < 0 || H <= 0 || d_k <= 0 || d_v <= 0) return -1;
    if (variant != 0 && variant != 1) return -1;
    const int SEG = 64;
    const int nseg = (L + SEG - 1) / SEG;

#pragma omp parallel for collapse(2) schedule(dynamic, 1)
    for (int b = 0; b < B; ++b) {
        for (int h = 0; h < H; ++h) {
            const size_t sd = (size_t)d_v * d_k;
            /* ckpt[g]: state before segment g; seg[i]: state after step g*SEG + i */
            double *ckpt = (double *)malloc(sizeof(double) * sd * (size_t)(nseg > 0 ? nseg : 1));
            double *seg = (double *)malloc(sizeof(double) * sd * (size_t)(SEG + 1));
            double *G = (double *)malloc(sizeof(double) * sd);
            double *kt = (double *)malloc(sizeof(double) * d_k);
            double *qt = (double *)malloc(sizeof(double) * d_k);
            double *vt = (double *)malloc(sizeof(double) * d_v);
            double *r = (double *)malloc(sizeof(double) * d_v);
            double *u = (double *)malloc(sizeof(double) * d_v);
            double *du = (double *)malloc(sizeof(double) * d_v);
            double *dr = (double *)malloc(sizeof(double) * d_v);

#define LOAD_TOKEN(t)                                                              \
    do {                                                                           \
        size_t row_ = ((size_t)b * L + (t)) * H + h;                               \
        for (int c = 0; c < d_k; ++c) {                                            \
            kt[c] = load_elem(k, dt, row_ * d_k + c);                              \
            qt[c] = load_elem(q, dt, row_ * d_k + c);                              \
        }                                                                          \
        for (int c = 0; c < d_v; ++c) vt[c] = load_elem(v, dt, row_ * d_v + c);    \
    } while (0)
            /* forward sweep: checkpoints */
            double *S = seg; /* scratch state */
            if (S0)
                memcpy(S, S0 + ((size_t)b * H + h) * sd, sizeof(double) * sd);
            else
                memset(S, 0, sizeof(double) * sd);
            for (int t = 0; t < L; ++t) {
                if (t % SEG == 0) memcpy(ckpt + (size_t)(t / SEG) * sd, S, sizeof(double) * sd);
                size_t row = ((size_t)b * L + t) * H + h;
                LOAD_TOKEN(t);
                double *Sn = seg + sd;
                gdn_step(S, Sn, kt, vt, (double)alpha[row], (double)beta[row], variant, d_k, d_v);
                memcpy(S, Sn, sizeof(double) * sd);
            }
            if (dS_final)
                memcpy(G, dS_final + ((size_t)b * H + h) * sd, sizeof(double) * sd);
            else
                memset(G, 0, sizeof(double) * sd);

            for (int g = nseg - 1; g >= 0; --g) {
                int t0 = g * SEG, n = (L - t0 < SEG) ? L - t0 : SEG;
                /* recompute the segment's states: seg[0] = before, seg[i+1] = after step t0+i */
                memcpy(seg, ckpt + (size_t)g * sd, sizeof(double) * sd);
                for (int i = 0; i < n; ++i) {
                    size_t row = ((size_t)b * L + t0 + i) * H + h;
                    LOAD_TOKEN(t0 + i);
                    gdn_step(seg + (size_t)i * sd, seg + (size_t)(i + 1) * sd, kt, vt, (double)alpha[row],
                             (double)beta[row], variant, d_k, d_v);
                }
                for (int i = n - 1; i >= 0; --i) {
                    int t = t0 + i;
                    size_t row = ((size_t)b * L + t) * H + h;
                    const double a = (double)alpha[row], be = (double)beta[row];
                    const double rho = variant == 0 ? a : 1.0;
                    const double *Sp = seg + (size_t)i * sd, *St = seg + (size_t)(i + 1) * sd;
                    LOAD_TOKEN(t);
                    const double *dOt = dO + row * d_v;
                    /* r and u of this step, from S_{t-1} */
                    for (int e = 0; e < d_v; ++e) {
                        double s = 0.0;
                        for (int c = 0; c < d_k; ++c) s += Sp[(size_t)e * d_k + c] * kt[c];
                        r[e] = s;
                        u[e] = be * (vt[e] - rho * s);
                    }
                    /* output o_t = S_t q_t: dq_t = S_t^T dO_t; G += dO_t q_t^T */
                    for (int c = 0; c < d_k; ++c) {
                        double s = 0.0;
                        for (int e = 0; e < d_v; ++e) s += St[(size_t)e * d_k + c] * dOt[e];
                        dq[row * d_k + c] = s;
                    }
                    for (int e = 0; e < d_v; ++e)
                        for (int c = 0; c < d_k; ++c) G[(size_t)e * d_k + c] += dOt[e] * qt[c];
                    /* S_t = alpha S_{t-1} + u k^T */
                    double dbe = 0.0, dal = 0.0, ur = 0.0;
                    for (int e = 0; e < d_v; ++e) {
                        double s = 0.0;
                        for (int c = 0; c < d_k; ++c) s += G[(size_t)e * d_k + c] * kt[c];
                        du[e] = s;
                        dv[row * d_v + e] = be * s;
                        dbe += s * (vt[e] - rho * r[e]);
                        ur += s * r[e];
                        dr[e] = -be * rho * s;
                    }
                    for (size_t x = 0; x < sd; ++x) dal += G[x] * Sp[x];
                    if (variant == 0) dal += -be * ur;
                    dalpha[row] = dal;
                    dbeta[row] = dbe;
                    for (int c = 0; c < d_k; ++c) {
                        double s = 0.0;
                        for (int e = 0; e < d_v; ++e)
                            s += G[(size_t)e * d_k + c] * u[e] + Sp[(size_t)e * d_k + c] * dr[e];
                        dk[row * d_k + c] = s;
                    }
                    /* gradient of S_{t-1} */
                    for (int e = 0; e < d_v; ++e)
                        for (int c = 0; c < d_k; ++c)
                            G[(size_t)e * d_k + c] = a * G[(size_t)e * d_k + c] + dr[e] * kt[c];
                }
            }
#undef LOAD_TOKEN
            if (dS0) memcpy(dS0 + ((size_t)b * H + h) * sd, G, sizeof(double) * sd);
            free(ckpt);
            free(seg);
            free(G);
            free(kt);
            free(qt);
            free(vt);
            free(r);
            free(u);
            free(du);
            free(dr);
        }
    }
    return 0;
}

/*
 * ORACLE — test infrastructure only. Only the tests, the smoke check and the
 * benchmark's CPU-baseline leg may load this code; the product path never does.
 *
 * fp32 canonical block selector: the single-precision arithmetic, in a fixed
 * order, in which the selection decision (an integer result decided by floating
 * point) is taken. Each statement below is one IEEE-754 binary32 operation with
 * round-to-nearest-even; fmaf() is the correctly rounded fused multiply-add of
 * C99 (F.10.10.1). Compile with -ffp-contract=off so that no other operation is
 * fused.
 *
 * What it computes (COBS: Cumulant Order Block Sparse Attention, gist.science
 * explainer of arXiv 2607.09052, §2.2 "Die Kumulanten-Expansion" and §2.3
 * "Second-Order Scoring"; the per-channel variance form of the covariance term):
 *
 *   summaries  mu_{b,c}   = (1/L) sum_r k_{bL+r,c}
 *              var_{b,c}  = (1/L) sum_r (k_{bL+r,c} - mu_{b,c})^2
 *   group query  Qsum_c = sum_{h in g} q_{h,c},  Q2_c = sum_{h in g} q_{h,c}^2
 *   score      S_{g,b} = (sum_c Qsum_c mu_{b,c}) * isd + c2 * (sum_c Q2_c var_{b,c})
 *              with isd = RN(1/sqrt(d)), c2 = RN(alpha / (2 d)),
 *   which equals sum_{h in g} [ q_h.mu_b / sqrt(d) + alpha/2 * sum_c q_{h,c}^2 var_{b,c} / d ].
 *
 * Order: every sum over rows or heads runs over its index in ascending order starting from +0.
 * The two channel sums of a score (sum_c Qsum_c mu_c and sum_c Q2_c var_c) each run as four
 * interleaved partial chains, chain j taking the channels c = j (mod 4) in ascending order from
 * +0 with one fmaf per term, and are combined as (s_0 + s_1) + (s_2 + s_3). (The pages fix no
 * order; this one keeps the dependency chains short and matches four consecutive channels per
 * 16-byte load.)
 */


#include <math.h>
#include <stddef.h>
#include <stdint.h>

/* sum_c x_c y_c in the canonical four-chain order (d a multiple of 4). */
static float dot4(const float* x, const float* y, int d) {
    float s0 = 0.0f, s1 = 0.0f, s2 = 0.0f, s3 = 0.0f;
    for (int c = 0; c < d; c += 4) {
        s0 = fmaf(x[c + 0], y[c + 0], s0);
        s1 = fmaf(x[c + 1], y[c + 1], s1);
        s2 = fmaf(x[c + 2], y[c + 2], s2);
        s3 = fmaf(x[c + 3], y[c + 3], s3);
    }
    return (s0 + s1) + (s2 + s3);
}

/*
 * K: [T][d] float32 rows (exact bf16 or fp32 values). Writes out[j][0][c] = mu,
 * out[j][1][c] = var for the complete blocks j < T / L.
 */
void cobs_oracle_summaries_f32(const float* K, int64_t T, int d, int L, float* out) {
    const int64_t nB = T / L;
    const float invL = 1.0f / (float)L; /* exact: L is a power of two */
    for (int64_t j = 0; j < nB; ++j) {
        for (int c = 0; c < d; ++c) {
            float s = 0.0f;
            for (int r = 0; r < L; ++r) s = s + K[(j * L + r) * d + c];
            const float mu = s * invL;
            float a = 0.0f;
            for (int r = 0; r < L; ++r) {
                const float t = K[(j * L + r) * d + c] - mu;
                a = fmaf(t, t, a);
            }
            out[(j * 2 + 0) * d + c] = mu;
            out[(j * 2 + 1) * d + c] = a * invL;
        }
    }
}

/* q: [G][d] query heads of one group. Writes qsum[d], q2[d]. */
void cobs_oracle_group_query_f32(const float* q, int G, int d, float* qsum, float* q2) {
    for (int c = 0; c < d; ++c) {
        float s = 0.0f, s2 = 0.0f;
        for (int h = 0; h < G; ++h) {
            const float x = q[h * d + c];
            s = s + x;
            s2 = fmaf(x, x, s2);
        }
        qsum[c] = s;
        q2[c] = s2;
    }
}

/* Score constants: isd = RN32(1/sqrt(d)) (via double), c2 = RN32(alpha * 0.5 / d). */
void cobs_oracle_score_constants(int d, float alpha, float* isd, float* c2) {
    *isd = (float)(1.0 / sqrt((double)d));
    *c2 = (float)((double)alpha * 0.5 / (double)d);
}

/*
 * Scores of nq group queries against blocks [0, nb) of one unit.
 * qsum, q2: [nq][d]; summ: [nb][2][d]; S: [nq][nb].
 */
void cobs_oracle_scores_f32(const float* qsum, const float* q2, const float* summ, int64_t nq,
                            int64_t nb, int d, float isd, float c2, float* S) {
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < nq; ++i) {
        const float* qs = qsum + i * d;
        const float* qq = q2 + i * d;
        for (int64_t b = 0; b < nb; ++b) {
            const float* mu = summ + (b * 2 + 0) * d;
            const float* var = summ + (b * 2 + 1) * d;
            const float a = dot4(qs, mu, d);
            const float v = dot4(qq, var, d);
            S[i * nb + b] = fmaf(c2, v, a * isd);
        }
    }
}

/*
 * Isotropic scalar variant (one second-order scalar per block). COBS §2.2/§2.3 compress the
 * block covariance Sigma_b; the skill card's "Pitfalls" asks for one or two scalars per block.
 * Taking Sigma_b ~ sigma2_b I with sigma2_b = tr(Sigma_b) / d (the mean per-channel
 * variance) gives 1/2 q^T Sigma_b q = 1/2 sigma2_b |q|^2, so per block
 *   summary   mu_{b,c} (as above) and sigma2_b = (1/d) sum_c var_{b,c}
 *   score     S_{g,b} = (sum_c Qsum_c mu_{b,c}) * isd + c2 * (Q2tot * sigma2_b),
 *             Q2tot = sum_c Q2_c  (= sum_{h in g} |q_h|^2).
 * Canonical order: var_{b,c} as in cobs_oracle_summaries_f32; sigma2_b = (adds over c
 * ascending from +0) * (1/d) (exact scaling, d a power of two); Q2tot = adds over c
 * ascending from +0; S = fma(c2, Q2tot * sigma2_b, a * isd) with a as above (four chains).
 */

/* summ: [nb][2][d] (mean, per-channel variance, as written above). out: [nb][d + 1] (mean, sigma2). */
void cobs_oracle_iso_summaries_f32(const float* summ, int64_t nb, int d, float* out) {
    const float invd = 1.0f / (float)d; /* exact: d is a power of two */
    for (int64_t b = 0; b < nb; ++b) {
        float s = 0.0f;
        for (int c = 0; c < d; ++c) {
            out[b * (d + 1) + c] = summ[(b * 2 + 0) * d + c];
            s = s + summ[(b * 2 + 1) * d + c];
        }
        out[b * (d + 1) + d] = s * invd;
    }
}

/* qsum, q2: [nq][d]; summ_iso: [nb][d + 1]; S: [nq][nb]. */
void cobs_oracle_iso_scores_f32(const float* qsum, const float* q2, const float* summ_iso, int64_t nq,
                                int64_t nb, int d, float isd, float c2, float* S) {
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < nq; ++i) {
        const float* qs = qsum + i * d;
        const float* qq = q2 + i * d;
        float q2tot = 0.0f;
        for (int c = 0; c < d; ++c) q2tot = q2tot + qq[c];
        for (int64_t b = 0; b < nb; ++b) {
            const float* mu = summ_iso + b * (d + 1);
            const float a = dot4(qs, mu, d);
            const float v = q2tot * mu[d];
            S[i * nb + b] = fmaf(c2, v, a * isd);
        }
    }
}

/*
 * Low-rank variant. COBS §2.2/§2.3 keep the block covariance Sigma_b in compressed form, first
 * of all as its leading eigenpairs (lambda_j, u_j), j < r: 1/2 q^T Sigma_b q ~ 1/2 sum_j
 * lambda_j (q . u_j)^2. Per block the summary holds the mean mu_b, the r unit vectors u_j and
 * the r values lambda_j; the score of a GQA group (the sum of its heads' scores) is
 *   S_{g,b} = (sum_c Qsum_c mu_c) * isd + c2 * sum_j lambda_j * (sum_{h in g} (q_h . u_j)^2).
 *
 * The eigenpairs come from a fixed, deterministic float32 solver whose every operation this
 * file fixes (the GPU runs the same steps in the same order, so both produce the same bits):
 *   Y[r][c] = k_{r,c} - mu_c                       (rows r < L of the block, channels c < d)
 *   V = V0 (d x R), V0[c][j] = +-1 by a fixed bit pattern of (c, j)
 *   repeat LR_ITERS times:
 *     T[r][j] = dot4_c(Y[r][.], V[.][j])            (four-chain order over c, as the scores)
 *     W[c][j] = dot4_r(Y[.][c], T[.][j])            (four-chain order over r)
 *     modified Gram-Schmidt over j ascending:
 *       for i < j: p = wdot(W[.][i], W[.][j]); W[c][j] = fmaf(-p, W[c][i], W[c][j])
 *       n = sqrtf(wdot(W[.][j], W[.][j])); W[c][j] = W[c][j] / n   (n == 0: the column is 0)
 *     V = W
 *   T = Y V; lambda_j = dot4_r(T[.][j], T[.][j]) * (1/L)
 *   order the pairs by lambda descending (ties: lower j first)
 * wdot is the "32-lane" order: partial p_l = sum over c = l, l + 32, ... (ascending, fmaf),
 * l < 32, then five butterfly levels p_l = p_l + p_{l xor o}, o = 16, 8, 4, 2, 1; the result
 * is p_0. sqrtf and the division are correctly rounded (IEEE).
 * The fixed iteration count makes the result a deterministic function of the block; for
 * well-separated leading eigenvalues it converges to the leading eigenpairs.
 */
#define LR_ITERS 24
#define LR_MAXR 8

static float wdot32(const float* x, const float* y, int d, int stride_x, int stride_y) {
    float p[32];
    for (int l = 0; l < 32; ++l) {
        float s = 0.0f;
        for (int c = l; c < d; c += 32) s = fmaf(x[(size_t)c * stride_x], y[(size_t)c * stride_y], s);
        p[l] = s;
    }
    for (int o = 16; o > 0; o >>= 1) {
        float q[32];
        for (int l = 0; l < 32; ++l) q[l] = p[l] + p[l ^ o];
        for (int l = 0; l < 32; ++l) p[l] = q[l];
    }
    return p[0];
}

/* four-chain dot with strides (n a multiple of 4) */
static float dot4s(const float* x, const float* y, int n, int sx, int sy) {
    float s0 = 0.0f, s1 = 0.0f, s2 = 0.0f, s3 = 0.0f;
    for (int i = 0; i < n; i += 4) {
        s0 = fmaf(x[(size_t)(i + 0) * sx], y[(size_t)(i + 0) * sy], s0);
        s1 = fmaf(x[(size_t)(i + 1) * sx], y[(size_t)(i + 1) * sy], s1);
        s2 = fmaf(x[(size_t)(i + 2) * sx], y[(size_t)(i + 2) * sy], s2);
        s3 = fmaf(x[(size_t)(i + 3) * sx], y[(size_t)(i + 3) * sy], s3);
    }
    return (s0 + s1) + (s2 + s3);
}

/* The fixed start V0[c][j]: +1 or -1 by bit 11 of (c * 2654435761 + (j + 1) * 40503) (32-bit). */
static float lr_v0(int c, int j) {
    const uint32_t h = (uint32_t)c * 2654435761u + (uint32_t)(j + 1) * 40503u;
    return ((h >> 11) & 1u) ? 1.0f : -1.0f;
}

/*
 * K: [T][d] float32 rows; mu: [nb][d] canonical block means (cobs_oracle_summaries_f32);
 * out_u: [nb][R][d] eigenvectors, out_l: [nb][R] eigenvalues (descending).
 */
void cobs_oracle_lowrank_f32(const float* K, const float* mu, int64_t nb, int d, int L, int R, float* out_u,
                             float* out_l) {
#pragma omp parallel for schedule(static)
    for (int64_t b = 0; b < nb; ++b) {
        float Y[64 * 128], V[128 * LR_MAXR], W[128 * LR_MAXR], T[64 * LR_MAXR], lam[LR_MAXR];
        const float* m = mu + b * d;
        for (int r = 0; r < L; ++r)
            for (int c = 0; c < d; ++c) Y[r * d + c] = K[(b * L + r) * (int64_t)d + c] - m[c];
        for (int c = 0; c < d; ++c)
            for (int j = 0; j < R; ++j) V[c * R + j] = lr_v0(c, j);
        for (int it = 0; it <= LR_ITERS; ++it) {
            for (int r = 0; r < L; ++r)
                for (int j = 0; j < R; ++j) T[r * R + j] = dot4s(Y + r * d, V + j, d, 1, R);
            if (it == LR_ITERS) break;
            for (int c = 0; c < d; ++c)
                for (int j = 0; j < R; ++j) W[c * R + j] = dot4s(Y + c, T + j, L, d, R);
            for (int j = 0; j < R; ++j) {
                for (int i = 0; i < j; ++i) {
                    const float p = wdot32(W + i, W + j, d, R, R);
                    for (int c = 0; c < d; ++c) W[c * R + j] = fmaf(-p, W[c * R + i], W[c * R + j]);
                }
                const float n = sqrtf(wdot32(W + j, W + j, d, R, R));
                for (int c = 0; c < d; ++c) W[c * R + j] = n > 0.0f ? W[c * R + j] / n : 0.0f;
            }
            for (int e = 0; e < d * R; ++e) V[e] = W[e];
        }
        for (int j = 0; j < R; ++j) lam[j] = dot4s(T + j, T + j, L, R, R) * (1.0f / (float)L);
        /* order by lambda descending, ties by j (stable selection) */
        int ord[LR_MAXR];
        for (int j = 0; j < R; ++j) ord[j] = j;
        for (int a = 0; a < R; ++a)
            for (int z = a + 1; z < R; ++z)
                if (lam[ord[z]] > lam[ord[a]] || (lam[ord[z]] == lam[ord[a]] && ord[z] < ord[a])) {
                    const int t = ord[a]; ord[a] = ord[z]; ord[z] = t;
                }
        for (int j = 0; j < R; ++j) {
            out_l[b * R + j] = lam[ord[j]];
            for (int c = 0; c < d; ++c) out_u[(b * R + j) * d + c] = V[c * R + ord[j]];
        }
    }
}

/*
 * Low-rank group scores. q: [G][d] the group's query heads (exact float32 values); qsum: [d]
 * (cobs_oracle_group_query_f32); mu: [nb][d]; u: [nb][R][d]; lam: [nb][R]; S: [nb].
 *   a = dot4(qsum, mu_b); for j: e_j = sum over h ascending of fmaf(p, p, .) with p = dot4(q_h, u_j);
 *   v = sum over j ascending of fmaf(lam_j, e_j, .); S = fmaf(c2, v, a * isd).
 */
void cobs_oracle_lowrank_scores_f32(const float* q, const float* qsum, int G, const float* mu, const float* u,
                                    const float* lam, int64_t nb, int d, int R, float isd, float c2, float* S) {
    for (int64_t b = 0; b < nb; ++b) {
        const float a = dot4s(qsum, mu + b * d, d, 1, 1);
        float v = 0.0f;
        for (int j = 0; j < R; ++j) {
            float e = 0.0f;
            for (int h = 0; h < G; ++h) {
                const float p = dot4s(q + h * d, u + (b * R + j) * d, d, 1, 1);
                e = fmaf(p, p, e);
            }
            v = fmaf(lam[b * R + j], e, v);
        }
        S[b] = fmaf(c2, v, a * isd);
    }
}

/*
 * FP4 variant of the low-rank summaries (COBS §2.3: the eigenvectors stored in FP4, E2M1, and
 * the mean in BF16). From the canonical float32 mean and eigenvectors above:
 *   mean:  mu'_c = RN_bf16(mu_c)  (round to nearest, ties to even, as a float32 value)
 *   vector j: a = max_c |u_c|; s = a / 6 (float32 division); code_c = E2M1(u_c / s), u'_c = (+-m) * s
 *     where E2M1 rounds |x| to the nearest of the magnitudes m = 0, 0.5, 1, 1.5, 2, 3, 4, 6 (ties to
 *     the even magnitude index, |x| > 6 saturates to 6) and keeps the sign (a zero magnitude has
 *     code 0); s = 0 gives code 0 everywhere.
 * The eigenvalues stay float32; the score is the low-rank score of (mu', u', lambda).
 */
static const float kE2M1[8] = {0.0f, 0.5f, 1.0f, 1.5f, 2.0f, 3.0f, 4.0f, 6.0f};

int cobs_oracle_e2m1_code(float x) {
    const float a = fabsf(x);
    int best = 0;
    float bd = a;  /* distance to magnitude 0 */
    for (int i = 1; i < 8; ++i) {
        const float dist = fabsf(a - kE2M1[i]);
        if (dist < bd || (dist == bd && (i & 1) == 0)) {
            best = i;
            bd = dist;
        }
    }
    if (a > 6.0f) best = 7;
    if (best == 0) return 0;
    return (x < 0.0f ? 8 : 0) | best;
}

float cobs_oracle_bf16_rn(float x) {
    union { float f; uint32_t u; } v;
    v.f = x;
    v.u = (v.u + 0x7FFFu + ((v.u >> 16) & 1u)) & 0xFFFF0000u;
    return v.f;
}

/* The E2M1 form of n vectors of len numbers each (the rule above, one scale per vector):
 * x [n][len] -> codes [n][len] (0..15), scales [n], xq [n][len] (the dequantized values). */
void cobs_oracle_fp4_vectors(const float* x, int64_t n, int len, uint8_t* codes, float* scales, float* xq) {
    for (int64_t r = 0; r < n; ++r) {
        const float* v = x + r * len;
        float a = 0.0f;
        for (int c = 0; c < len; ++c) a = fmaxf(a, fabsf(v[c]));
        const float s = a / 6.0f;
        scales[r] = s;
        for (int c = 0; c < len; ++c) {
            const int code = s > 0.0f ? cobs_oracle_e2m1_code(v[c] / s) : 0;
            codes[r * len + c] = (uint8_t)code;
            const float m = (code & 8) ? -kE2M1[code & 7] : kE2M1[code & 7];
            xq[r * len + c] = m * s;
        }
    }
}

/* mu: [nb][d] -> mu_q [nb][d]; u: [nb][R][d] -> codes [nb][R][d] (0..15), scales [nb][R], u_q [nb][R][d]. */
void cobs_oracle_lowrank_fp4_f32(const float* mu, const float* u, int64_t nb, int d, int R, float* mu_q,
                                 uint8_t* codes, float* scales, float* u_q) {
    for (int64_t b = 0; b < nb; ++b)
        for (int c = 0; c < d; ++c) mu_q[b * d + c] = cobs_oracle_bf16_rn(mu[b * d + c]);
    cobs_oracle_fp4_vectors(u, nb * R, d, codes, scales, u_q);
}

/*
 * Query-subspace variant (COBS §2.3: the eigenvectors kept as coordinates in a query subspace of
 * dimension s < d, r d -> r s numbers per block). P: [d][s] with orthonormal columns, the
 * caller's estimate of the subspace the queries live in (from their second moment). Per block the
 * summary keeps mu (d), u~_j = P^T u_j (s numbers) and lambda_j; a query head is projected the
 * same way, q~ = P^T q, and the covariance term uses (q~ . u~_j) in place of (q . u_j):
 *   x~_i = four-chain sum over c of P[c][i] x_c            (i < s)
 *   S = fmaf(c2, sum_j fmaf(lambda_j, e_j, .), a * isd), e_j = sum_h fmaf(p, p, .),
 *   p = four-chain sum over i of q~_{h,i} u~_{j,i},  a = four-chain sum over c of Qsum_c mu_c.
 */
/* out[n][s] = P^T x_n for n rows x [n][d] */
void cobs_oracle_subspace_project(const float* P, const float* x, int64_t n, int d, int s, float* out) {
    for (int64_t r = 0; r < n; ++r)
        for (int i = 0; i < s; ++i) out[r * s + i] = dot4s(P + i, x + r * d, d, s, 1);
}

/*
 * Query subspace with FP4 coordinates and a BF16 mean (COBS §2.3 applies the three compressions
 * together; §4.1 reports this form as "Subspace, r=4, FP4"): the subspace summaries above, then
 *   mean: mu'_c = RN_bf16(mu_c);  projected vector j: the E2M1 rule above over its s coordinates
 *   (a = max_i |u~_{j,i}|, scale a / 6), u~'_{j,i} = (+-m) * scale;  lambda_j stays float32.
 * The score is the subspace score of (mu', u~', lambda).
 * mu: [nb][d] -> mu_q; ut: [nb][R][s] -> codes [nb][R][s], scales [nb][R], ut_q [nb][R][s].
 */
void cobs_oracle_subspace_fp4_f32(const float* mu, const float* ut, int64_t nb, int d, int s, int R, float* mu_q,
                                  uint8_t* codes, float* scales, float* ut_q) {
    for (int64_t b = 0; b < nb; ++b)
        for (int c = 0; c < d; ++c) mu_q[b * d + c] = cobs_oracle_bf16_rn(mu[b * d + c]);
    cobs_oracle_fp4_vectors(ut, nb * R, s, codes, scales, ut_q);
}

/* q: [G][d]; qsum: [d]; mu: [nb][d]; ut: [nb][R][s]; lam: [nb][R]; P: [d][s]; S: [nb] */
void cobs_oracle_subspace_scores(const float* q, const float* qsum, int G, const float* mu, const float* ut,
                                 const float* lam, int64_t nb, int d, int s, int R, const float* P, float isd,
                                 float c2, float* S) {
    float qt[16 * 128];
    cobs_oracle_subspace_project(P, q, G, d, s, qt);
    for (int64_t b = 0; b < nb; ++b) {
        const float a = dot4s(qsum, mu + b * d, d, 1, 1);
        float v = 0.0f;
        for (int j = 0; j < R; ++j) {
            float e = 0.0f;
            for (int h = 0; h < G; ++h) {
                const float p = dot4s(qt + h * s, ut + (b * R + j) * (int64_t)s, s, 1, 1);
                e = fmaf(p, p, e);
            }
            v = fmaf(lam[b * R + j], e, v);
        }
        S[b] = fmaf(c2, v, a * isd);
    }
}

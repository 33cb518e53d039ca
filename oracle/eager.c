/*
 * oracle/eager.c -- fp64 per-token eager recurrence for SSM-layer decode.
 *
 * TEST INFRASTRUCTURE ONLY.  This is the CPU oracle the CUDA path is checked
 * against; it shares no code, header, table or helper with the CUDA library and
 * must never be linked into, loaded by or called from the product path.  Only
 * tests/, the smoke check and the benchmark's CPU-baseline leg may use it.
 *
 * What it computes (the plain definition, written out; no blocking, fusion or
 * reordering beyond the loop over independent (sequence, head) pairs):
 *
 *  Mamba-2 layer, per (b, h), group g = h / (H / G)  ("ReplaySSM" reports,
 *  blog.thibaultmonteiro.fr, section "La fiche qu'on reecrit": every token reads
 *  the state, applies a decay and a rank-1 update, computes the output, writes
 *  the state back; the recurrence itself is the standard Mamba-2 one):
 *      a_t = exp(dt_t * A_h)
 *      S_t = a_t S_{t-1} + (s_t x_t) B_t^T      s_t = dt_t if dt_scales_input else 1
 *      y_t = S_t C_t + D_h x_t                  (output from the updated state:
 *                                                datadaily.news, "Comment fonctionnent
 *                                                reellement les modeles a espace d'etats")
 *
 *  Gated DeltaNet layer, per (b, h) (same section: a delta-rule correction with an
 *  update of the same form):
 *      S_t = alpha_t S_{t-1} (I - beta_t k_t k_t^T) + beta_t v_t k_t^T
 *      o_t = S_t q_t
 *    applied to each row s of S (S is d_v x d_k, row-major, d_k contiguous):
 *      s <- alpha (s - beta (s . k) k) + beta v[row] k
 *
 *  Kimi Delta Attention layer, per (b, h) (named with Mamba-2 and GDN on the same
 *  page, section "Des couches rapides sur le papier", and covered by the same
 *  argument in "La fiche qu'on reecrit"; the pages give no formula, so this is the
 *  plainest reading: GDN with the scalar gate replaced by a gate per key channel,
 *  applied before the delta-rule correction):
 *      S_t = S_{t-1} Diag(alpha_t) (I - beta_t k_t k_t^T) + beta_t v_t k_t^T
 *      o_t = S_t q_t
 *    applied to each row s of S:  u = alpha (.) s;  s <- u - beta (u . k) k + beta v[row] k
 *
 * Layouts (all row-major, float64):
 *   S[B][H][P][N];  Mamba-2: x[B][H][P], dt[B][H], Bm[B][G][N], Cm[B][G][N], y[B][H][P]
 *   GDN (P = d_v, N = d_k): q[B][H][N], k[B][H][N], v[B][H][P], alpha[B][H], beta[B][H], o[B][H][P]
 *   KDA: as GDN with alpha[B][H][N]
 */
#include <math.h>
#include <stdint.h>
#ifdef _OPENMP
#include <omp.h>
#endif

int oracle_max_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

void oracle_set_threads(int n)
{
#ifdef _OPENMP
    if (n > 0) omp_set_num_threads(n);
#else
    (void)n;
#endif
}

void oracle_mamba2_eager_step(int64_t Bn, int64_t H, int64_t P, int64_t N, int64_t G,
                              const double *A, const double *D, int dt_scales_input,
                              double *S, const double *x, const double *dt,
                              const double *Bm, const double *Cm, double *y)
{
    const int64_t heads_per_group = H / G;
#pragma omp parallel for collapse(2) schedule(static)
    for (int64_t b = 0; b < Bn; ++b) {
        for (int64_t h = 0; h < H; ++h) {
            const int64_t g = h / heads_per_group;
            const double dth = dt[b * H + h];
            const double a = exp(dth * A[h]);
            const double s_in = dt_scales_input ? dth : 1.0;
            double *Sbh = S + (b * H + h) * P * N;
            const double *xbh = x + (b * H + h) * P;
            const double *Bv = Bm + (b * G + g) * N;
            const double *Cv = Cm + (b * G + g) * N;
            for (int64_t p = 0; p < P; ++p) {
                double acc = 0.0;
                for (int64_t n = 0; n < N; ++n) {
                    double s = a * Sbh[p * N + n] + (s_in * xbh[p]) * Bv[n];
                    Sbh[p * N + n] = s;
                    acc += s * Cv[n];
                }
                y[(b * H + h) * P + p] = acc + D[h] * xbh[p];
            }
        }
    }
}

void oracle_gdn_eager_step(int64_t Bn, int64_t H, int64_t P, int64_t N, double *S,
                           const double *q, const double *k, const double *v,
                           const double *alpha, const double *beta, double *o)
{
#pragma omp parallel for collapse(2) schedule(static)
    for (int64_t b = 0; b < Bn; ++b) {
        for (int64_t h = 0; h < H; ++h) {
            const double al = alpha[b * H + h];
            const double be = beta[b * H + h];
            double *Sbh = S + (b * H + h) * P * N;
            const double *qv = q + (b * H + h) * N;
            const double *kv = k + (b * H + h) * N;
            const double *vv = v + (b * H + h) * P;
            for (int64_t r = 0; r < P; ++r) {
                double *row = Sbh + r * N;
                double sk = 0.0;
                for (int64_t n = 0; n < N; ++n) sk += row[n] * kv[n];
                double acc = 0.0;
                for (int64_t n = 0; n < N; ++n) {
                    double s = al * (row[n] - be * sk * kv[n]) + be * vv[r] * kv[n];
                    row[n] = s;
                    acc += s * qv[n];
                }
                o[(b * H + h) * P + r] = acc;
            }
        }
    }
}

void oracle_kda_eager_step(int64_t Bn, int64_t H, int64_t P, int64_t N, double *S,
                           const double *q, const double *k, const double *v,
                           const double *alpha, const double *beta, double *o)
{
#pragma omp parallel for collapse(2) schedule(static)
    for (int64_t b = 0; b < Bn; ++b) {
        for (int64_t h = 0; h < H; ++h) {
            const double *al = alpha + (b * H + h) * N;
            const double be = beta[b * H + h];
            double *Sbh = S + (b * H + h) * P * N;
            const double *qv = q + (b * H + h) * N;
            const double *kv = k + (b * H + h) * N;
            const double *vv = v + (b * H + h) * P;
            for (int64_t r = 0; r < P; ++r) {
                double *row = Sbh + r * N;
                double uk = 0.0;
                for (int64_t n = 0; n < N; ++n) {
                    row[n] = al[n] * row[n];  /* u = alpha (.) s */
                    uk += row[n] * kv[n];
                }
                double acc = 0.0;
                for (int64_t n = 0; n < N; ++n) {
                    double s = row[n] - be * uk * kv[n] + be * vv[r] * kv[n];
                    row[n] = s;
                    acc += s * qv[n];
                }
                o[(b * H + h) * P + r] = acc;
            }
        }
    }
}

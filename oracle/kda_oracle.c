/*
 * kda_oracle.c -- fp64 CPU oracle of the KDA layer-half decode step.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the tests, the package's smoke check and the
 * benchmark's CPU-baseline leg may load this library.  It shares no code,
 * header, table or helper with the CUDA library: the two meet only through the
 * seeded input bytes.
 *
 * What it computes (one decode token per sequence, every quantity in fp64):
 *
 *   x       <- bf16 hidden state, widened exactly
 *   W       <- decode(E4M3 code) * fp32 block scale, one scale per 128 x 128
 *              block (Kiln, "How was Kiln measured": FP8 weights with
 *              128 x 128 block scales)
 *   q, k, v  = W_q x, W_k x, W_v x           (per head slices of dk, dk, dv)
 *   beta_h   = sigmoid(W_b x)_h              (one gate per head)
 *   alpha    = exp(-softplus(W_a_up (W_a_down x)))   (one decay per key channel)
 *   k^_h     = k_h / ||k_h||_2               (a zero k_h maps to 0)
 *   S'_h     = (I - beta_h k^ k^T) diag(alpha_h) S_h + beta_h k^ v_h^T
 *              with S_h in R^{dk x dv}, updated in place
 *   o_h      = S'_h^T q_h
 *   out      = W_o concat_h(o_h)
 *
 * The pages name the layer ("KDA (linear attention)", TrnRT story) and its
 * fixed-size recurrent state updated in place per sequence (TrnRT listing,
 * "The interesting bit"; Kiln, "The decode kernels, and why they are opt-in")
 * but print no equations; the gated delta rule above is the workload
 * definition the decode benchmark states, read with S in the dk x dv layout it
 * names (so that beta = 1 and a unit k give S'^T k = v).
 *
 * Two forms of the state update are provided: the literal one that builds the
 * dk x dk matrix (I - beta k^ k^T) diag(alpha) and multiplies, and the rank-1
 * form  S~ = diag(alpha) S,  w = S~^T k^,  S' = S~ + k^ (beta (v - w))^T.
 * All reductions run sequentially in index order; OpenMP only splits
 * independent rows / heads, so results do not depend on the thread count.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#ifdef _OPENMP
#include <omp.h>
#endif

#define KDA_ORACLE_BLOCK 128

/* ---------------------------------------------------------------- scalars */

/* FP8 E4M3 ("fn" variant: exponent bias 7, no infinities, S.1111.111 is NaN).
 * normal   (e >= 1): (-1)^s * 2^(e-7) * (1 + m/8)
 * subnormal (e = 0): (-1)^s * 2^(-6)  * (m/8)                                 */
double kda_oracle_e4m3_decode(unsigned int code)
{
    unsigned int s = (code >> 7) & 1u, e = (code >> 3) & 15u, m = code & 7u;
    double mag;
    if (e == 15u && m == 7u) return NAN;
    if (e == 0u) mag = ldexp((double)m / 8.0, -6);
    else mag = ldexp(1.0 + (double)m / 8.0, (int)e - 7);
    return s ? -mag : mag;
}

/* bf16 -> fp64: the 16 bits are the top half of an IEEE binary32. */
double kda_oracle_bf16_to_f64(uint16_t b)
{
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

double kda_oracle_sigmoid(double a) { return 1.0 / (1.0 + exp(-a)); }

/* softplus(z) = log(1 + e^z); for z > 0 written as z + log1p(e^-z) so that
 * e^z never overflows. */
double kda_oracle_softplus(double z)
{
    return z > 0.0 ? z + log1p(exp(-z)) : log1p(exp(z));
}

/* alpha = exp(-softplus(z)) in (0, 1]. */
double kda_oracle_alpha(double z) { return exp(-kda_oracle_softplus(z)); }

/* ---------------------------------------------------------------- weights */

/* W[i][j] = decode(code[i][j]) * scale[i/128][j/128]; row-major [rows, cols]. */
void kda_oracle_dequant_fp8(const uint8_t *codes, const float *scales, int rows, int cols, double *w)
{
    int nbc = (cols + KDA_ORACLE_BLOCK - 1) / KDA_ORACLE_BLOCK;
#pragma omp parallel for schedule(static)
    for (int i = 0; i < rows; ++i)
        for (int j = 0; j < cols; ++j) {
            double s = (double)scales[(size_t)(i / KDA_ORACLE_BLOCK) * nbc + j / KDA_ORACLE_BLOCK];
            w[(size_t)i * cols + j] = kda_oracle_e4m3_decode(codes[(size_t)i * cols + j]) * s;
        }
}

void kda_oracle_widen_bf16(const uint16_t *b, size_t n, double *w)
{
#pragma omp parallel for schedule(static)
    for (size_t i = 0; i < n; ++i) w[i] = kda_oracle_bf16_to_f64(b[i]);
}

/* y[n] = sum_k W[n][k] x[k], k ascending. */
static void matvec(const double *W, const double *x, int rows, int cols, double *y)
{
#pragma omp parallel for schedule(static)
    for (int n = 0; n < rows; ++n) {
        const double *w = W + (size_t)n * cols;
        double acc = 0.0;
        for (int k = 0; k < cols; ++k) acc += w[k] * x[k];
        y[n] = acc;
    }
}

/* ---------------------------------------------------------------- model */

typedef struct kda_oracle_dims {
    int batch, hidden, num_heads, head_dk, head_dv, alpha_rank;
} kda_oracle_dims;

/* Dequantised fp64 copies of every weight, made once per model. */
typedef struct kda_oracle_model {
    kda_oracle_dims d;
    double *wq, *wk, *wv, *wo, *wa_down, *wa_up, *wb;
} kda_oracle_model;

kda_oracle_model *kda_oracle_model_new(const kda_oracle_dims *d,
                                       const uint8_t *wq, const float *sq,
                                       const uint8_t *wk, const float *sk,
                                       const uint8_t *wv, const float *sv,
                                       const uint8_t *wo, const float *so,
                                       const uint16_t *wa_down, const uint16_t *wa_up, const uint16_t *wb)
{
    kda_oracle_model *m = (kda_oracle_model *)calloc(1, sizeof *m);
    if (!m) return NULL;
    m->d = *d;
    size_t H = (size_t)d->hidden, Dk = (size_t)d->num_heads * d->head_dk, Dv = (size_t)d->num_heads * d->head_dv;
    size_t r = (size_t)d->alpha_rank, nh = (size_t)d->num_heads;
    m->wq = (double *)malloc(Dk * H * sizeof(double));
    m->wk = (double *)malloc(Dk * H * sizeof(double));
    m->wv = (double *)malloc(Dv * H * sizeof(double));
    m->wo = (double *)malloc(H * Dv * sizeof(double));
    m->wa_down = (double *)malloc(r * H * sizeof(double));
    m->wa_up = (double *)malloc(Dk * r * sizeof(double));
    m->wb = (double *)malloc(nh * H * sizeof(double));
    if (!m->wq || !m->wk || !m->wv || !m->wo || !m->wa_down || !m->wa_up || !m->wb) {
        free(m->wq); free(m->wk); free(m->wv); free(m->wo); free(m->wa_down); free(m->wa_up); free(m->wb);
        free(m);
        return NULL;
    }
    kda_oracle_dequant_fp8(wq, sq, (int)Dk, (int)H, m->wq);
    kda_oracle_dequant_fp8(wk, sk, (int)Dk, (int)H, m->wk);
    kda_oracle_dequant_fp8(wv, sv, (int)Dv, (int)H, m->wv);
    kda_oracle_dequant_fp8(wo, so, (int)H, (int)Dv, m->wo);
    kda_oracle_widen_bf16(wa_down, r * H, m->wa_down);
    kda_oracle_widen_bf16(wa_up, Dk * r, m->wa_up);
    kda_oracle_widen_bf16(wb, nh * H, m->wb);
    return m;
}

void kda_oracle_model_free(kda_oracle_model *m)
{
    if (!m) return;
    free(m->wq); free(m->wk); free(m->wv); free(m->wo); free(m->wa_down); free(m->wa_up); free(m->wb);
    free(m);
}

/* Literal form for one head: M = (I - beta k^ k^T) diag(alpha) (dk x dk),
 * S' = M S + beta k^ v^T. */
static void state_update_literal(int dk, int dv, const double *kh, const double *v, double beta,
                                 const double *alpha, double *S, double *M, double *Snew)
{
    for (int i = 0; i < dk; ++i)
        for (int j = 0; j < dk; ++j)
            M[(size_t)i * dk + j] = ((i == j ? 1.0 : 0.0) - beta * kh[i] * kh[j]) * alpha[j];
    for (int i = 0; i < dk; ++i)
        for (int j = 0; j < dv; ++j) {
            double acc = 0.0;
            for (int l = 0; l < dk; ++l) acc += M[(size_t)i * dk + l] * S[(size_t)l * dv + j];
            Snew[(size_t)i * dv + j] = acc + beta * kh[i] * v[j];
        }
    memcpy(S, Snew, (size_t)dk * dv * sizeof(double));
}

/* Rank-1 form for one head: S~ = diag(alpha) S, w = S~^T k^, u = beta (v - w),
 * S' = S~ + k^ u^T. */
static void state_update_rank1(int dk, int dv, const double *kh, const double *v, double beta,
                               const double *alpha, double *S, double *w)
{
    for (int i = 0; i < dk; ++i)
        for (int j = 0; j < dv; ++j) S[(size_t)i * dv + j] *= alpha[i];
    for (int j = 0; j < dv; ++j) {
        double acc = 0.0;
        for (int i = 0; i < dk; ++i) acc += kh[i] * S[(size_t)i * dv + j];
        w[j] = acc;
    }
    for (int j = 0; j < dv; ++j) w[j] = beta * (v[j] - w[j]);
    for (int i = 0; i < dk; ++i)
        for (int j = 0; j < dv; ++j) S[(size_t)i * dv + j] += kh[i] * w[j];
}

/*
 * One decode step for every sequence of the batch.
 *   x_bf16  [B, H] bf16 bits
 *   state   [B, nh, dk, dv] fp64, updated in place
 *   out     [B, H] fp64
 *   literal 1: dk x dk matrix form, 0: rank-1 form
 *   dbg     optional (may be NULL): per sequence, concatenated
 *           q [nh*dk], k^ [nh*dk], v [nh*dv], beta [nh], alpha [nh*dk],
 *           o [nh*dv], t = W_a_down x [r], k (unnormalised) [nh*dk]
 * Returns 0, or -1 on allocation failure.
 */
int kda_oracle_step(const kda_oracle_model *m, const uint16_t *x_bf16, double *state, double *out,
                    int literal, double *dbg)
{
    const kda_oracle_dims *d = &m->d;
    const int B = d->batch, H = d->hidden, nh = d->num_heads, dk = d->head_dk, dv = d->head_dv, r = d->alpha_rank;
    const int Dk = nh * dk, Dv = nh * dv;
    double *x = (double *)malloc((size_t)H * sizeof(double));
    double *q = (double *)malloc((size_t)Dk * sizeof(double));
    double *k = (double *)malloc((size_t)Dk * sizeof(double));
    double *kraw = (double *)malloc((size_t)Dk * sizeof(double));
    double *v = (double *)malloc((size_t)Dv * sizeof(double));
    double *t = (double *)malloc((size_t)r * sizeof(double));
    double *z = (double *)malloc((size_t)Dk * sizeof(double));
    double *bl = (double *)malloc((size_t)nh * sizeof(double));
    double *beta = (double *)malloc((size_t)nh * sizeof(double));
    double *alpha = (double *)malloc((size_t)Dk * sizeof(double));
    double *o = (double *)malloc((size_t)Dv * sizeof(double));
    int rc = 0;
    if (!x || !q || !k || !kraw || !v || !t || !z || !bl || !beta || !alpha || !o) { rc = -1; goto done; }

    for (int b = 0; b < B; ++b) {
        for (int i = 0; i < H; ++i) x[i] = kda_oracle_bf16_to_f64(x_bf16[(size_t)b * H + i]);
        /* projections */
        matvec(m->wq, x, Dk, H, q);
        matvec(m->wk, x, Dk, H, k);
        matvec(m->wv, x, Dv, H, v);
        matvec(m->wb, x, nh, H, bl);
        matvec(m->wa_down, x, r, H, t);
        matvec(m->wa_up, t, Dk, r, z);
        memcpy(kraw, k, (size_t)Dk * sizeof(double));
        /* gates and key normalisation */
        for (int h = 0; h < nh; ++h) beta[h] = kda_oracle_sigmoid(bl[h]);
        for (int i = 0; i < Dk; ++i) alpha[i] = kda_oracle_alpha(z[i]);
        for (int h = 0; h < nh; ++h) {
            double ss = 0.0;
            for (int i = 0; i < dk; ++i) ss += k[h * dk + i] * k[h * dk + i];
            double nrm = sqrt(ss);
            for (int i = 0; i < dk; ++i) k[h * dk + i] = nrm > 0.0 ? k[h * dk + i] / nrm : 0.0;
        }
        /* state update and readout, per head */
        int fail = 0;
#pragma omp parallel
        {
            double *M = NULL, *Snew = NULL, *w = NULL;
            if (literal) {
                M = (double *)malloc((size_t)dk * dk * sizeof(double));
                Snew = (double *)malloc((size_t)dk * dv * sizeof(double));
            } else {
                w = (double *)malloc((size_t)dv * sizeof(double));
            }
            if ((literal && (!M || !Snew)) || (!literal && !w)) {
#pragma omp atomic write
                fail = 1;
            } else {
#pragma omp for schedule(static)
                for (int h = 0; h < nh; ++h) {
                    double *S = state + ((size_t)b * nh + h) * (size_t)dk * dv;
                    const double *kh = k + (size_t)h * dk, *vh = v + (size_t)h * dv, *al = alpha + (size_t)h * dk;
                    if (literal) state_update_literal(dk, dv, kh, vh, beta[h], al, S, M, Snew);
                    else state_update_rank1(dk, dv, kh, vh, beta[h], al, S, w);
                    const double *qh = q + (size_t)h * dk;
                    for (int j = 0; j < dv; ++j) {
                        double acc = 0.0;
                        for (int i = 0; i < dk; ++i) acc += S[(size_t)i * dv + j] * qh[i];
                        o[(size_t)h * dv + j] = acc;
                    }
                }
            }
            free(M); free(Snew); free(w);
        }
        if (fail) { rc = -1; goto done; }
        /* output projection */
        matvec(m->wo, o, H, Dv, out + (size_t)b * H);
        if (dbg) {
            double *p = dbg + (size_t)b * (size_t)(4 * Dk + 2 * Dv + nh + r);
            memcpy(p, q, (size_t)Dk * sizeof(double)); p += Dk;
            memcpy(p, k, (size_t)Dk * sizeof(double)); p += Dk;
            memcpy(p, v, (size_t)Dv * sizeof(double)); p += Dv;
            memcpy(p, beta, (size_t)nh * sizeof(double)); p += nh;
            memcpy(p, alpha, (size_t)Dk * sizeof(double)); p += Dk;
            memcpy(p, o, (size_t)Dv * sizeof(double)); p += Dv;
            memcpy(p, t, (size_t)r * sizeof(double)); p += r;
            memcpy(p, kraw, (size_t)Dk * sizeof(double));
        }
    }
done:
    free(x); free(q); free(k); free(kraw); free(v); free(t); free(z); free(bl); free(beta); free(alpha); free(o);
    return rc;
}

int kda_oracle_num_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

void kda_oracle_set_num_threads(int n)
{
#ifdef _OPENMP
    if (n > 0) omp_set_num_threads(n);
#else
    (void)n;
#endif
}

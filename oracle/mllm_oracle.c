/*
 * mllm_oracle.c -- plain, slow CPU oracle for the MaskLLM per-block N:M mask sampler.
 *
 * TEST INFRASTRUCTURE. Only the test suite, the package smoke check and the benchmark's
 * CPU-baseline leg load this library. The CUDA library never calls it, and the two share
 * no code, header, table or constant generator: every table below is built here, from
 * its definition, at load time.
 *
 * What it follows (the pages are the text of web pages summarising arXiv 2409.17481,
 * "MaskLLM: Learnable Semi-Structured Sparsity for Large Language Models"):
 *   - candidate set S_{2:4} and its order ........ paper-graph-ui summary, s.3.2, Eq.2 listing
 *   - Gumbel noise g = -log(-log eps) ............ s.3.4 "Step 1: Gumbel Max", Eq.5
 *   - soft index softmax((kappa*pi + g)/tau) ..... s.3.4 Eq.6 and the logit parameterisation
 *   - soft mask M = sum_i y_i S_i ................ s.3.4 "Step 3", Eq.7 (worked example)
 *   - regulariser L_LM - lambda sum ||W.M||^2 .... s.3.4 "Sparse Weight Regularization", Eq.8
 *   - gradient to the logits, weights frozen ..... s.3.2 "Frozen LLM Backbone"; s.3.4 Alg.1 step 2
 *   - AdamW on the logits (lr, wd 0.1) ........... s.3.4 "Optimizer and training length", Table 7
 *   - prior similarity and prior init ............ s.3.4 "Mask Prior", Eq.9 and Eq.10
 *   - hard mask k = argmax pi .................... s.3.2 "Information flow at inference"; Alg.1 step 3
 *
 * Precision. Everything is IEEE double except two quantities whose bits the specification
 * fixes at fp32, because the soft mask amplifies their rounding by kappa/tau (up to 1e4):
 *   (1) the Gumbel noise g, a random number: Philox4x32-10 (Salmon et al., SC'11, "Parallel
 *       random numbers: as easy as 1, 2, 3") -> 21-bit field k -> eps = (2k+1) 2^-22 ->
 *       t = -nlog(eps) -> g = -nlog(t), with nlog the fp32 table-driven logarithm below
 *       (the method of P.T.P. Tang, "Table-driven implementation of the logarithm function
 *       in IEEE floating-point arithmetic", ACM TOMS 16(4), 1990: a table indexed by the
 *       binary exponent and a 7-bit mantissa prefix, and a degree-3 Taylor remainder);
 *   (2) the perturbed logit w = fma(kappa, pi, g), one fp32 rounding.
 * The flag `round_w = 0` evaluates w = kappa*pi + g in double instead (used only by the
 * finite-difference and autograd pins, where a rounding step would be a staircase).
 *
 * Build: gcc -O2 -std=c11 -ffp-contract=off -fno-fast-math -fPIC -shared -lm.
 */
#define _DEFAULT_SOURCE
#include <math.h>
#include <stdint.h>
#include <string.h>

#define ORC_OK 0
#define ORC_ERR 1

/* ------------------------------------------------------------------------------------ */
/* Candidate set S_{N:M}                                                                 */
/* ------------------------------------------------------------------------------------ */

/* 2:4 rows exactly as listed on the page (s.3.2, Eq.2): [1,1,0,0], [1,0,1,0], [1,0,0,1],
 * [0,1,0,1], [0,1,1,0], [0,0,1,1]. This order is not lexicographic. */
static const uint8_t S24[6][4] = {
    {1, 1, 0, 0}, {1, 0, 1, 0}, {1, 0, 0, 1}, {0, 1, 0, 1}, {0, 1, 1, 0}, {0, 0, 1, 1}};

/* 4:8: the pages list no order; all 4-subsets of {0..7} in lexicographic order of their
 * ascending index tuples, (0,1,2,3), (0,1,2,4), ..., (4,5,6,7). Built at load time. */
static uint8_t S48[70][8];

static int num_candidates(int n, int m) {
    if (n == 2 && m == 4) return 6;
    if (n == 4 && m == 8) return 70;
    return 0;
}

static const uint8_t *cand_row(int n, int m, int i) {
    (void)n;
    return (m == 4) ? S24[i] : S48[i];
}

static void build_s48(void) {
    int r = 0;
    for (int a = 0; a < 8; a++)
        for (int b = a + 1; b < 8; b++)
            for (int c = b + 1; c < 8; c++)
                for (int d = c + 1; d < 8; d++) {
                    memset(S48[r], 0, 8);
                    S48[r][a] = S48[r][b] = S48[r][c] = S48[r][d] = 1;
                    r++;
                }
}

/* ------------------------------------------------------------------------------------ */
/* Philox4x32-10 (Salmon, Moraes, Dror, Shaw, SC'11), the published round and key schedule */
/* ------------------------------------------------------------------------------------ */

static void philox4x32_10(const uint32_t ctr_in[4], const uint32_t key_in[2], uint32_t out[4]) {
    const uint32_t MUL0 = 0xD2511F53u, MUL1 = 0xCD9E8D57u; /* round multipliers */
    const uint32_t BUMP0 = 0x9E3779B9u, BUMP1 = 0xBB67AE85u; /* Weyl key increments */
    uint32_t x0 = ctr_in[0], x1 = ctr_in[1], x2 = ctr_in[2], x3 = ctr_in[3];
    uint32_t k0 = key_in[0], k1 = key_in[1];
    for (int round = 0; round < 10; round++) {
        if (round > 0) {
            k0 += BUMP0;
            k1 += BUMP1;
        }
        uint64_t p0 = (uint64_t)MUL0 * (uint64_t)x0;
        uint64_t p1 = (uint64_t)MUL1 * (uint64_t)x2;
        uint32_t hi0 = (uint32_t)(p0 >> 32), lo0 = (uint32_t)p0;
        uint32_t hi1 = (uint32_t)(p1 >> 32), lo1 = (uint32_t)p1;
        uint32_t y0 = hi1 ^ x1 ^ k0;
        uint32_t y1 = lo1;
        uint32_t y2 = hi0 ^ x3 ^ k1;
        uint32_t y3 = lo0;
        x0 = y0; x1 = y1; x2 = y2; x3 = y3;
    }
    out[0] = x0; out[1] = x1; out[2] = x2; out[3] = x3;
}

void orc_philox4x32_10(const uint32_t *ctr, const uint32_t *key, uint32_t *out) {
    philox4x32_10(ctr, key, out);
}

/* The four output words form one 128-bit little-endian integer (word 0 lowest). Field f,
 * f = 0..5, is bits [21f, 21f+21) of it. */
static uint32_t field21(const uint32_t x[4], int f) {
    int lo = 21 * f;
    uint32_t v = 0;
    for (int b = 0; b < 21; b++) {
        int bit = lo + b;
        uint32_t word = x[bit / 32];
        v |= ((word >> (bit % 32)) & 1u) << b;
    }
    return v;
}

/* Random words for (seed, block gid, step, group): counter (gid lo, gid hi, step, group),
 * key (seed lo, seed hi). step 0xFFFFFFFF is reserved for the logit initialisation. */
static void block_words(uint64_t seed, uint64_t gid, uint32_t step, uint32_t group, uint32_t out[4]) {
    uint32_t ctr[4] = {(uint32_t)gid, (uint32_t)(gid >> 32), step, group};
    uint32_t key[2] = {(uint32_t)seed, (uint32_t)(seed >> 32)};
    philox4x32_10(ctr, key, out);
}

/* 21-bit field for candidate c of a block: group c/6, field c%6. */
static uint32_t candidate_field(uint64_t seed, uint64_t gid, uint32_t step, int c) {
    uint32_t w[4];
    block_words(seed, gid, step, (uint32_t)(c / 6), w);
    return field21(w, c % 6);
}

#define INIT_STEP 0xFFFFFFFFu

/* ------------------------------------------------------------------------------------ */
/* nlog: the fp32 logarithm that defines the noise bits (Tang 1990 table-driven method)   */
/* ------------------------------------------------------------------------------------ */
/* x = 2^e * mm with mm within 2^-8 of a breakpoint F_j. j is the 7-bit mantissa prefix of
 * x rounded to nearest; prefixes j >= 64 (mantissa >= 1.5) move to the next binade, so
 * F_j = 1 + j/128 for j < 64 and (1 + j/128)/2 for j >= 64, both in [0.75, 1.5).
 * c_j = fl32(1/F_j). With r = fma(mm, c_j, -1), |r| < 2^-8,
 *   ln x = e ln2 - ln c_j + ln(1 + r),  ln(1 + r) = r - r^2/2 + r^3/3 + O(r^4),
 * and T[e][j] = fl32(e ln2 - ln c_j) (evaluated in double, rounded once) carries the first
 * two terms. The noise only ever takes logarithms of x in [2^-22, 16) (eps >= 2^-22 and
 * t = -ln eps <= 15.25), so e runs over [-22, 4]: 27 rows of 128 entries. Outside that
 * domain nlog is not defined (this implementation returns NaN). */
#define NLOG_EMIN (-22)
#define NLOG_EMAX 4
#define NLOG_ROWS (NLOG_EMAX - NLOG_EMIN + 1)
static float NLOG_C[128], NLOG_T[NLOG_ROWS][128];
static float ONE_THIRD;

static void build_nlog(void) {
    for (int j = 0; j < 128; j++) {
        double F = (j < 64) ? (1.0 + j / 128.0) : (1.0 + j / 128.0) / 2.0;
        NLOG_C[j] = (float)(1.0 / F);
    }
    for (int e = NLOG_EMIN; e <= NLOG_EMAX; e++)
        for (int j = 0; j < 128; j++)
            NLOG_T[e - NLOG_EMIN][j] = (float)((double)e * M_LN2 - log((double)NLOG_C[j]));
    ONE_THIRD = (float)(1.0 / 3.0);
}

static float nlog(float x) {
    uint32_t b;
    memcpy(&b, &x, 4);
    uint32_t ib = b + 0x8000u;                 /* round the mantissa at its 7-bit prefix */
    uint32_t j = (ib >> 16) & 0x7Fu;
    int32_t e = (int32_t)(ib >> 23) - 127 + (int32_t)(j >> 6);
    if (!(x > 0.0f) || e < NLOG_EMIN || e > NLOG_EMAX) return NAN;
    uint32_t mb = b - ((uint32_t)e << 23);     /* mm = x * 2^-e, exact */
    float mm;
    memcpy(&mm, &mb, 4);
    float r = fmaf(mm, NLOG_C[j], -1.0f);
    float q = fmaf(r, ONE_THIRD, -0.5f);
    float rq = r * q;
    float p = fmaf(rq, r, r);                  /* r - r^2/2 + r^3/3 */
    return NLOG_T[e - NLOG_EMIN][j] + p;
}

float orc_nlog(float x) { return nlog(x); }

void orc_nlog_array(int64_t n, const float *x, float *out) {
    for (int64_t i = 0; i < n; i++) out[i] = nlog(x[i]);
}

/* c [128], T [27 * 128] (row e - NLOG_EMIN), consts[0] = fl32(1/3), consts[1..2] = e range. */
void orc_nlog_table(float *c, float *T, float *consts) {
    for (int j = 0; j < 128; j++) c[j] = NLOG_C[j];
    for (int r = 0; r < NLOG_ROWS; r++)
        for (int j = 0; j < 128; j++) T[r * 128 + j] = NLOG_T[r][j];
    consts[0] = ONE_THIRD;
    consts[1] = (float)NLOG_EMIN;
    consts[2] = (float)NLOG_EMAX;
}

/* eps = (2k+1) 2^-22, exact in fp32, strictly inside (0, 1). */
static float uniform_from_field(uint32_t k) { return (float)(2u * k + 1u) * 0x1p-22f; }

/* Gumbel noise, Eq.5: g = -log(-log eps). */
static float gumbel_from_field(uint32_t k) {
    float eps = uniform_from_field(k);
    float t = -nlog(eps);
    return -nlog(t);
}

/* ------------------------------------------------------------------------------------ */
/* Exported helpers                                                                       */
/* ------------------------------------------------------------------------------------ */

int orc_num_candidates(int n, int m) { return num_candidates(n, m); }

int orc_candidates(int n, int m, uint8_t *rows) {
    int C = num_candidates(n, m);
    if (!C) return ORC_ERR;
    for (int i = 0; i < C; i++) memcpy(rows + (size_t)i * m, cand_row(n, m, i), (size_t)m);
    return ORC_OK;
}

void orc_fields21(const uint32_t *x, uint32_t *f) {
    for (int i = 0; i < 6; i++) f[i] = field21(x, i);
}

/* Uniforms eps and noise g for nb blocks and all C candidates of each. */
int orc_noise(int n, int m, uint64_t seed, uint32_t step, int64_t nb, const uint64_t *gid,
              float *eps_out, float *g_out) {
    int C = num_candidates(n, m);
    if (!C) return ORC_ERR;
    for (int64_t b = 0; b < nb; b++)
        for (int c = 0; c < C; c++) {
            uint32_t k = candidate_field(seed, gid[b], step, c);
            if (eps_out) eps_out[b * C + c] = uniform_from_field(k);
            if (g_out) g_out[b * C + c] = gumbel_from_field(k);
        }
    return ORC_OK;
}

/* Eq.7 on its own: M_j = sum_i y_i S_ij. */
int orc_soft_mask(int n, int m, int64_t nb, const double *y, double *msoft) {
    int C = num_candidates(n, m);
    if (!C) return ORC_ERR;
    for (int64_t b = 0; b < nb; b++)
        for (int j = 0; j < m; j++) {
            double s = 0.0;
            for (int i = 0; i < C; i++)
                if (cand_row(n, m, i)[j]) s += y[b * C + i];
            msoft[b * m + j] = s;
        }
    return ORC_OK;
}

/* ------------------------------------------------------------------------------------ */
/* Forward: Eq.5-Eq.8 for one block                                                       */
/* ------------------------------------------------------------------------------------ */

/* Soft index and soft mask of one block.
 *   w_i = fma(kappa, pi_i, g_i) in fp32 (round_w = 1) or kappa*pi_i + g_i in double;
 *   y_i = exp((w_i - max w)/tau) / sum_k exp((w_k - max w)/tau)           (Eq.6)
 *   M_j = sum_{i: S_ij = 1} y_i                                            (Eq.7)
 *   Mc_j = sum_{i: S_ij = 0} y_i, which is 1 - M_j because sum_i y_i = 1, formed as a sum
 *   so that it keeps its relative accuracy when M_j is within rounding of 1. */
static void block_soft(int n, int m, int C, const float *pi, uint64_t gid, float kappa, float tau,
                       uint64_t seed, uint32_t step, int noise_on, int round_w,
                       double *y, double *msoft, double *mcomp) {
    double w[70];
    for (int i = 0; i < C; i++) {
        float g = noise_on ? gumbel_from_field(candidate_field(seed, gid, step, i)) : 0.0f;
        if (round_w)
            w[i] = (double)fmaf(kappa, pi[i], g);
        else
            w[i] = (double)kappa * (double)pi[i] + (double)g;
    }
    double wmax = -INFINITY;
    for (int i = 0; i < C; i++) if (w[i] > wmax) wmax = w[i];
    double inv_tau = 1.0 / (double)tau, sum = 0.0;
    for (int i = 0; i < C; i++) { y[i] = exp((w[i] - wmax) * inv_tau); sum += y[i]; }
    for (int i = 0; i < C; i++) y[i] /= sum;
    for (int j = 0; j < m; j++) {
        double s1 = 0.0, s0 = 0.0;
        for (int i = 0; i < C; i++) {
            if (cand_row(n, m, i)[j]) s1 += y[i]; else s0 += y[i];
        }
        msoft[j] = s1;
        mcomp[j] = s0;
    }
}

/* Forward over nb blocks. W is [nb, M] (exact values of the stored weights), pi is
 * [nb, C] fp32, gid[b] the global block id. Outputs (each nullable): y [nb, C], msoft and
 * mcomp [nb, M], x = W * msoft unrounded [nb, M]; reg_out = sum over the blocks of
 * ||W . M||^2 (Eq.8 without lambda), accumulated in block order. */
int orc_sample_fwd(int n, int m, int64_t nb, const double *W, const float *pi, const uint64_t *gid,
                   float kappa, float tau, uint64_t seed, uint32_t step, int noise_on, int round_w,
                   double *y_out, double *msoft_out, double *mcomp_out, double *x_out,
                   double *reg_out) {
    int C = num_candidates(n, m);
    if (!C || !(tau > 0.0f)) return ORC_ERR;
    double reg = 0.0;
    for (int64_t b = 0; b < nb; b++) {
        double y[70], ms[8], mc[8];
        block_soft(n, m, C, pi + b * C, gid[b], kappa, tau, seed, step, noise_on, round_w, y, ms, mc);
        for (int j = 0; j < m; j++) {
            double xj = W[b * m + j] * ms[j];
            if (x_out) x_out[b * m + j] = xj;
            reg += xj * xj;
            if (msoft_out) msoft_out[b * m + j] = ms[j];
            if (mcomp_out) mcomp_out[b * m + j] = mc[j];
        }
        if (y_out) for (int i = 0; i < C; i++) y_out[b * C + i] = y[i];
    }
    if (reg_out) *reg_out = reg;
    return ORC_OK;
}

/* ------------------------------------------------------------------------------------ */
/* Backward to the logits (weights frozen)                                               */
/* ------------------------------------------------------------------------------------ */
/* Loss L = <G, X> - lambda ||X||^2 with X = W . M, G = dL_LM/dX given (Eq.8, Alg.1 step 2).
 *   u_j  = dL/dM_j = G_j W_j - 2 lambda W_j^2 M_j
 *   a_i  = dL/dy_i = sum_j S_ij u_j                                        (through Eq.7)
 *   dL/dz_i = y_i (a_i - sum_k y_k a_k)                    (softmax Jacobian of Eq.6)
 *           = y_i sum_j (S_ij - M_j) u_j                   (since sum_k y_k S_kj = M_j)
 *   dL/dpi_i = (kappa/tau) dL/dz_i                         (z_i = (kappa pi_i + g_i)/tau)
 * For S_ij = 1 the factor S_ij - M_j = 1 - M_j is taken as Mc_j (the same number, formed
 * without cancellation). scale_out[i] = (kappa/tau) y_i sum_j |S_ij - M_j| |u_j| is the
 * magnitude of the summands of each gradient, the yardstick for its rounding error. */
int orc_sample_bwd(int n, int m, int64_t nb, const double *W, const double *G, const float *pi,
                   const uint64_t *gid, float kappa, float tau, float lambda, uint64_t seed,
                   uint32_t step, int noise_on, int round_w, double *grad_out, double *scale_out) {
    int C = num_candidates(n, m);
    if (!C || !(tau > 0.0f)) return ORC_ERR;
    double c = (double)kappa / (double)tau;
    for (int64_t b = 0; b < nb; b++) {
        double y[70], ms[8], mc[8], u[8];
        block_soft(n, m, C, pi + b * C, gid[b], kappa, tau, seed, step, noise_on, round_w, y, ms, mc);
        for (int j = 0; j < m; j++) {
            double wj = W[b * m + j];
            u[j] = G[b * m + j] * wj - 2.0 * (double)lambda * wj * wj * ms[j];
        }
        for (int i = 0; i < C; i++) {
            const uint8_t *row = cand_row(n, m, i);
            double d = 0.0, mag = 0.0;
            for (int j = 0; j < m; j++) {
                double coef = row[j] ? mc[j] : -ms[j];
                d += coef * u[j];
                mag += fabs(coef) * fabs(u[j]);
            }
            grad_out[b * C + i] = c * y[i] * d;
            if (scale_out) scale_out[b * C + i] = c * y[i] * mag;
        }
    }
    return ORC_OK;
}

/* ------------------------------------------------------------------------------------ */
/* AdamW (decoupled weight decay, Loshchilov & Hutter; PyTorch's AdamW step order)        */
/* ------------------------------------------------------------------------------------ */
/* t is the 1-based step count used in the bias corrections. */
void orc_adamw(int64_t n, const double *param, const double *m_in, const double *v_in,
               const double *grad, double lr, double beta1, double beta2, double eps, double wd,
               int64_t t, double *param_out, double *m_out, double *v_out) {
    double bc1 = 1.0 - pow(beta1, (double)t);
    double bc2 = 1.0 - pow(beta2, (double)t);
    for (int64_t i = 0; i < n; i++) {
        double p = param[i] * (1.0 - lr * wd);
        double mm = beta1 * m_in[i] + (1.0 - beta1) * grad[i];
        double vv = beta2 * v_in[i] + (1.0 - beta2) * grad[i] * grad[i];
        double denom = sqrt(vv) / sqrt(bc2) + eps;
        p -= (lr / bc1) * mm / denom;
        param_out[i] = p;
        m_out[i] = mm;
        v_out[i] = vv;
    }
}

/* ------------------------------------------------------------------------------------ */
/* Mask prior (Eq.9, Eq.10) from the magnitude one-shot pruner                           */
/* ------------------------------------------------------------------------------------ */

/* Ordering used for "largest |w|": NaN ranks below every number; equal magnitudes rank
 * the lower position first. Returns 1 if position a ranks above position b. */
static int ranks_above(double wa, int a, double wb, int b) {
    double ma = fabs(wa), mb = fabs(wb);
    int na = isnan(ma), nbn = isnan(mb);
    if (na != nbn) return nbn;          /* the number ranks above the NaN */
    if (!na && ma != mb) return ma > mb;
    return a < b;
}

/* Magnitude prior M0: keep the N positions of largest |w| (each position's rank is the
 * number of positions ranking above it; keep ranks < N). */
static void magnitude_prior(int n, int m, const double *w, uint8_t *m0) {
    for (int j = 0; j < m; j++) {
        int rank = 0;
        for (int k = 0; k < m; k++)
            if (k != j && ranks_above(w[k], k, w[j], j)) rank++;
        m0[j] = (uint8_t)(rank < n);
    }
}

/* Box-Muller pairs from the reserved init domain: candidates (2p, 2p+1) take radius
 * sqrt(-2 ln u_2p) and angle 2 pi u_(2p+1), where u_c = (2k+1) 2^-22 for candidate c's field. */
static void init_normals(int C, uint64_t seed, uint64_t gid, double *nrm) {
    for (int p = 0; 2 * p < C; p++) {
        double u1 = (double)uniform_from_field(candidate_field(seed, gid, INIT_STEP, 2 * p));
        double u2 = (double)uniform_from_field(candidate_field(seed, gid, INIT_STEP, 2 * p + 1));
        double r = sqrt(-2.0 * log(u1));
        double th = 2.0 * M_PI * u2;
        nrm[2 * p] = r * cos(th);
        if (2 * p + 1 < C) nrm[2 * p + 1] = r * sin(th);
    }
}

/* Prior initialisation for nb blocks (W [nb, M] values, gid per block).
 *   M0 = magnitude prior of the block
 *   sim_i = M0 . S_i - (1/|S|) sum_k M0 . S_k                              (Eq.9)
 *   pi0_i = init_std * n_i, n_i ~ N(0,1)                     (Table 7: N(0, 0.01) init)
 *   pi_i  = pi0_i + alpha * sigma(pi0) * sim_i, sigma = population std over i (Eq.10)
 * init_std == 0 selects a deterministic mode (not on the pages): pi_i = alpha * sim_i.
 * Outputs: pi_out [nb, C]; prior_idx_out [nb] (index of the candidate equal to M0);
 * sim_out [nb, C] (nullable). */
int orc_prior_init(int n, int m, int64_t nb, const double *W, const uint64_t *gid, double alpha,
                   double init_std, uint64_t seed, double *pi_out, int32_t *prior_idx_out,
                   double *sim_out) {
    int C = num_candidates(n, m);
    if (!C) return ORC_ERR;
    for (int64_t b = 0; b < nb; b++) {
        uint8_t m0[8];
        magnitude_prior(n, m, W + b * m, m0);
        double ip[70], mean_ip = 0.0;
        int32_t pidx = -1;
        for (int i = 0; i < C; i++) {
            const uint8_t *row = cand_row(n, m, i);
            int s = 0, same = 1;
            for (int j = 0; j < m; j++) { s += row[j] * m0[j]; if (row[j] != m0[j]) same = 0; }
            ip[i] = (double)s;
            mean_ip += ip[i];
            if (same) pidx = i;
        }
        mean_ip /= (double)C;
        double sim[70];
        for (int i = 0; i < C; i++) sim[i] = ip[i] - mean_ip;
        if (init_std == 0.0) {
            for (int i = 0; i < C; i++) pi_out[b * C + i] = alpha * sim[i];
        } else {
            double nrm[70], pi0[70], mu = 0.0, var = 0.0;
            init_normals(C, seed, gid[b], nrm);
            for (int i = 0; i < C; i++) { pi0[i] = init_std * nrm[i]; mu += pi0[i]; }
            mu /= (double)C;
            for (int i = 0; i < C; i++) var += (pi0[i] - mu) * (pi0[i] - mu);
            double sigma = sqrt(var / (double)C);
            for (int i = 0; i < C; i++) pi_out[b * C + i] = pi0[i] + alpha * sigma * sim[i];
        }
        if (prior_idx_out) prior_idx_out[b] = pidx;
        if (sim_out) for (int i = 0; i < C; i++) sim_out[b * C + i] = sim[i];
    }
    return ORC_OK;
}

/* Prior initialisation from a given prior mask per block (the transfer prior: s.3.4 "Mask
 * Prior" takes M0 from any one-shot method or from a previous MaskLLM run, Table 5).
 * M0 of block b = S_{prior_idx[b]}; an index >= C means the block has no prior: sim = 0, so
 * pi = pi0 (or 0 in the deterministic mode). Otherwise exactly orc_prior_init with that M0. */
int orc_prior_init_from_index(int n, int m, int64_t nb, const uint64_t *gid, const int32_t *prior_idx,
                              double alpha, double init_std, uint64_t seed, double *pi_out,
                              double *sim_out) {
    int C = num_candidates(n, m);
    if (!C) return ORC_ERR;
    for (int64_t b = 0; b < nb; b++) {
        double sim[70];
        int32_t k = prior_idx[b];
        if (k < 0 || k >= C) {
            for (int i = 0; i < C; i++) sim[i] = 0.0;
        } else {
            const uint8_t *m0 = cand_row(n, m, k);
            double ip[70], mean_ip = 0.0;
            for (int i = 0; i < C; i++) {
                const uint8_t *row = cand_row(n, m, i);
                int sacc = 0;
                for (int j = 0; j < m; j++) sacc += row[j] * m0[j];
                ip[i] = (double)sacc;
                mean_ip += ip[i];
            }
            mean_ip /= (double)C;
            for (int i = 0; i < C; i++) sim[i] = ip[i] - mean_ip;
        }
        if (init_std == 0.0) {
            for (int i = 0; i < C; i++) pi_out[b * C + i] = alpha * sim[i];
        } else {
            double nrm[70], pi0[70], mu = 0.0, var = 0.0;
            init_normals(C, seed, gid[b], nrm);
            for (int i = 0; i < C; i++) { pi0[i] = init_std * nrm[i]; mu += pi0[i]; }
            mu /= (double)C;
            for (int i = 0; i < C; i++) var += (pi0[i] - mu) * (pi0[i] - mu);
            double sigma = sqrt(var / (double)C);
            for (int i = 0; i < C; i++) pi_out[b * C + i] = pi0[i] + alpha * sigma * sim[i];
        }
        if (sim_out) for (int i = 0; i < C; i++) sim_out[b * C + i] = sim[i];
    }
    return ORC_OK;
}

/* ------------------------------------------------------------------------------------ */
/* Hard mask and compressed export                                                       */
/* ------------------------------------------------------------------------------------ */

/* First index of the largest logit; NaN never wins; all-NaN gives 0. */
static int argmax_first(const float *pi, int C) {
    int k = -1;
    for (int i = 0; i < C; i++) {
        if (isnan(pi[i])) continue;
        if (k < 0 || pi[i] > pi[k]) k = i;
    }
    return k < 0 ? 0 : k;
}

int orc_argmax(int64_t nb, int C, const float *pi, int32_t *k_out) {
    for (int64_t b = 0; b < nb; b++) k_out[b] = argmax_first(pi + b * C, C);
    return ORC_OK;
}

/* Hard extraction and packing of one matrix, row-major [rows, cols], blocks of M along cols.
 *   k = argmax pi (Alg.1 step 3), kept positions p_0 < ... < p_{N-1} of S_k;
 *   values[r, q*N + t] = W[r, q*M + p_t], copied bit for bit (elem_bytes 2 or 4);
 *   2:4 metadata: nibble p_0 | p_1 << 2 for block q of row r, in bits [4(q%8), 4(q%8)+4)
 *     of uint32 word q/8 of the row; a row has ceil((cols/4)/8) words, unused bits zero;
 *   4:8 metadata: one uint16 per block, p_0 | p_1 << 3 | p_2 << 6 | p_3 << 9;
 *   cand_idx[block] = k (nullable). */
int orc_hard_pack(int n, int m, int64_t rows, int64_t cols, int elem_bytes, const void *W,
                  const float *pi, void *values, void *meta, uint8_t *cand_idx) {
    int C = num_candidates(n, m);
    if (!C || cols % m || (elem_bytes != 2 && elem_bytes != 4)) return ORC_ERR;
    int64_t bpr = cols / m;
    int64_t words = (bpr + 7) / 8;
    const uint8_t *src = (const uint8_t *)W;
    uint8_t *dst = (uint8_t *)values;
    if (m == 4) memset(meta, 0, (size_t)(rows * words * 4));
    for (int64_t r = 0; r < rows; r++)
        for (int64_t q = 0; q < bpr; q++) {
            int64_t blk = r * bpr + q;
            int k = argmax_first(pi + blk * C, C);
            const uint8_t *row = cand_row(n, m, k);
            int pos[4], t = 0;
            for (int j = 0; j < m; j++) if (row[j]) pos[t++] = j;
            for (t = 0; t < n; t++) {
                int64_t s_off = (r * cols + q * m + pos[t]) * elem_bytes;
                int64_t d_off = (r * (cols / m * n) + q * n + t) * elem_bytes;
                memcpy(dst + d_off, src + s_off, (size_t)elem_bytes);
            }
            if (m == 4) {
                uint32_t nib = (uint32_t)(pos[0] | (pos[1] << 2));
                uint32_t *mw = (uint32_t *)meta + r * words + q / 8;
                *mw |= nib << (4 * (q % 8));
            } else {
                uint16_t code = (uint16_t)(pos[0] | (pos[1] << 3) | (pos[2] << 6) | (pos[3] << 9));
                ((uint16_t *)meta)[blk] = code;
            }
            if (cand_idx) cand_idx[blk] = (uint8_t)k;
        }
    return ORC_OK;
}

/* ------------------------------------------------------------------------------------ */
/* Diagnostics of the learned masks (s.3.4 Figs. 5, 6, 8) and a candidate-index codec     */
/* ------------------------------------------------------------------------------------ */

/* Number of blocks whose hard mask (candidate index) differs between a and b: the mask
 * difference between two masks (Fig. 8) or between adjacent steps (Fig. 5a). */
int64_t orc_mask_diff(int64_t n, const uint8_t *a, const uint8_t *b) {
    int64_t d = 0;
    for (int64_t i = 0; i < n; i++) d += (a[i] != b[i]);
    return d;
}

/* Mask statistics over nb blocks (W [nb, M] values, pi [nb, C]):
 *   out[0] = sum over blocks of max_i p_i with p = softmax(kappa pi) (mean max probability,
 *            Fig. 5b, is out[0] / nb);
 *   out[1] = sum of |W_j| over the positions the hard mask (argmax pi) keeps;
 *   out[2] = sum of |W_j| over the positions the magnitude mask (top-N |W|) keeps
 *            (out[1] / out[2] is the relative L1 norm of the kept weights, Fig. 6);
 *   out[3] = number of blocks whose hard mask equals the magnitude mask. */
int orc_mask_stats(int n, int m, int64_t nb, const double *W, const float *pi, double kappa, double *out) {
    int C = num_candidates(n, m);
    if (!C) return ORC_ERR;
    double s_maxp = 0.0, s_l1 = 0.0, s_l1_mag = 0.0, same = 0.0;
    for (int64_t b = 0; b < nb; b++) {
        const float *p = pi + b * C;
        const double *w = W + b * m;
        int k = argmax_first(p, C);
        double mx = -INFINITY, sum = 0.0;
        for (int i = 0; i < C; i++) if ((double)kappa * p[i] > mx) mx = (double)kappa * p[i];
        for (int i = 0; i < C; i++) sum += exp((double)kappa * p[i] - mx);
        s_maxp += 1.0 / sum;
        uint8_t m0[8];
        magnitude_prior(n, m, w, m0);
        const uint8_t *row = cand_row(n, m, k);
        int eq = 1;
        for (int j = 0; j < m; j++) {
            if (row[j]) s_l1 += fabs(w[j]);
            if (m0[j]) s_l1_mag += fabs(w[j]);
            if (row[j] != m0[j]) eq = 0;
        }
        same += eq;
    }
    out[0] = s_maxp; out[1] = s_l1; out[2] = s_l1_mag; out[3] = same;
    return ORC_OK;
}

/* Candidate-index codec: D = 12 indices per uint32 for 2:4 (6^12 < 2^32, 0.667 bits per
 * weight against log2(6)/4 = 0.646, the page's 0.65 bits/param) and D = 5 per uint32 for 4:8
 * (70^5 < 2^32, 0.8 bits per weight). Word w = sum_{t<D} idx[wD + t] C^t (missing tail
 * indices count as 0). */
int orc_encode_candidates(int n, int m, int64_t nb, const uint8_t *idx, uint32_t *out) {
    int C = num_candidates(n, m);
    if (!C) return ORC_ERR;
    int D = (m == 4) ? 12 : 5;
    int64_t words = (nb + D - 1) / D;
    for (int64_t wi = 0; wi < words; wi++) {
        uint64_t v = 0, p = 1;
        for (int t = 0; t < D; t++) {
            int64_t i = wi * D + t;
            if (i < nb) v += (uint64_t)idx[i] * p;
            p *= (uint64_t)C;
        }
        out[wi] = (uint32_t)v;
    }
    return ORC_OK;
}

int orc_decode_candidates(int n, int m, int64_t nb, const uint32_t *in, uint8_t *idx) {
    int C = num_candidates(n, m);
    if (!C) return ORC_ERR;
    int D = (m == 4) ? 12 : 5;
    for (int64_t i = 0; i < nb; i++) {
        uint64_t v = in[i / D];
        for (int t = 0; t < (int)(i % D); t++) v /= (uint64_t)C;
        idx[i] = (uint8_t)(v % (uint64_t)C);
    }
    return ORC_OK;
}

/* ------------------------------------------------------------------------------------ */
/* Deployment: the product with the hard-masked weight (s.3.2 "Information flow at       */
/* inference": the learned mask is applied once and the sparse network is served)        */
/* ------------------------------------------------------------------------------------ */

static double bf16_to_double(uint16_t h) {
    uint32_t bits = (uint32_t)h << 16;
    float f;
    memcpy(&f, &bits, 4);
    return (double)f;
}

/* y = x W*^T for a matrix W* = W (.) M* given in orc_hard_pack's compressed form (bf16
 * values, 2:4 nibble or 4:8 uint16 metadata), and activations x [tokens, cols] in bf16:
 *   y[t*rows + r] = sum over blocks q of row r, over kept slots i < N,
 *                   values[r, qN + i] * x[t, qM + p_i],
 * p_i the i-th kept position decoded from the metadata. Every term is an exact product of
 * two bf16 numbers; the sum runs in double in the order written. */
int orc_sparse_linear(int n, int m, int64_t rows, int64_t cols, const uint16_t *values, const void *meta,
                      int64_t tokens, const uint16_t *x, double *y) {
    if (!num_candidates(n, m) || cols % m || rows < 0 || tokens < 0) return ORC_ERR;
    int64_t bpr = cols / m, words = (bpr + 7) / 8;
    for (int64_t t = 0; t < tokens; t++)
        for (int64_t r = 0; r < rows; r++) {
            double acc = 0.0;
            for (int64_t q = 0; q < bpr; q++) {
                int pos[4];
                if (m == 4) {
                    uint32_t w = ((const uint32_t *)meta)[r * words + q / 8];
                    uint32_t nib = (w >> (4 * (q % 8))) & 0xFu;
                    pos[0] = (int)(nib & 3u);
                    pos[1] = (int)(nib >> 2);
                } else {
                    uint32_t code = ((const uint16_t *)meta)[r * bpr + q];
                    for (int i = 0; i < 4; i++) pos[i] = (int)((code >> (3 * i)) & 7u);
                }
                for (int i = 0; i < n; i++)
                    acc += bf16_to_double(values[r * bpr * n + q * n + i]) *
                           bf16_to_double(x[t * cols + q * m + pos[i]]);
            }
            y[t * rows + r] = acc;
        }
    return ORC_OK;
}

/* ------------------------------------------------------------------------------------ */
/* Rounding of the soft-masked weights to their storage type                             */
/* ------------------------------------------------------------------------------------ */

/* Round each double to bfloat16 (8 significant bits, fp32 exponent range), to nearest,
 * ties to even, with gradual underflow below 2^-126; returns the bf16 bit patterns. */
void orc_round_bf16(int64_t n, const double *in, uint16_t *out) {
    for (int64_t i = 0; i < n; i++) {
        double v = in[i];
        double a = fabs(v), q;
        if (a == 0.0 || isnan(v)) {
            q = a;
        } else {
            int e;
            frexp(a, &e);                               /* a = f 2^e, f in [0.5, 1) */
            int qexp = (e - 1 >= -126) ? (e - 1 - 7) : (-126 - 7); /* quantum exponent */
            q = ldexp(nearbyint(ldexp(a, -qexp)), qexp);  /* ties-to-even rounding mode */
        }
        float f = (float)copysign(q, v);                /* exact: q has <= 8 significant bits */
        uint32_t bits;
        memcpy(&bits, &f, 4);
        if (isnan(v)) bits = 0x7FC00000u;
        out[i] = (uint16_t)(bits >> 16);
    }
}

__attribute__((constructor)) static void orc_init(void) {
    build_s48();
    build_nlog();
}

/*
 * FluxBin oracle: plain, slow, fp64 CPU reference.  TEST INFRASTRUCTURE ONLY.
 *
 * Only the tests, the package smoke check and the benchmark's CPU-baseline
 * leg may load this code.  The product path (the CUDA library) shares no
 * code, header, table or helper with it.
 *
 * What it computes (FluxBin, "FluxBin: Flexible LUT-based Ultra-low-bit LLM
 * Inference by Algorithm-Kernel Synergy", source-linked summary):
 *
 *   Section 3 "Quantization": the weight matrix is a sum over decomposition
 *   orders k of row-scaled, column-scaled +-1 bases,
 *       W = sum_k diag(r_k) B_k diag(c_k).
 *   Section 3 "Salient-Aware Hybrid Bases" and "Virtual Columnar Mapping":
 *   a salient refinement with its own bases and scales is added on a chosen
 *   set S of columns; the dense salient sub-matrix is only a re-layout, so
 *   its column t is scattered back to the true column S[t].
 *   Appendix C.2: row scales may be block-wise (one per row per G-column
 *   block); the salient branch may likewise carry one row scale per block
 *   of s salient columns.
 *
 *   y[b] = W x[b], every value widened exactly from fp16 to fp64.
 *
 * The LUT functions follow the method's own steps (Section 3 "LUT-Based GEMV
 * Kernel", Appendix C.1, and the LUT Tensor Core notes, Section 2.2 "LUT-based
 * mpGEMM" and Section 3.1.2 "table symmetrisation"): for every activation
 * sub-vector v of length mu the table holds all 2^mu signed partial sums
 *   T[p] = sum_t (2 bit_t(p) - 1) v_t,
 * the column scale is fused into v (v = c (.) x), and a row's result is the
 * sum of the table entries that its sign patterns select, times the row scale.
 *
 * Readings where the pages are silent:
 *   bit value 1 means +1, 0 means -1; bit t of a pattern is column j*mu + t;
 *   the symmetric half table keeps the entries whose top bit (t = mu-1) is 0.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

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

/* Row scale of global base k for row i and column j.
 * G == 0: r is [Kb][M]; G > 0: r is [Kb][ceil(N/G)][M]. */
static double row_scale(const double* r, int64_t M, int64_t N, int G, int k, int64_t i, int64_t j) {
    if (G <= 0) return r[(int64_t)k * M + i];
    int64_t ng = (N + G - 1) / G;
    return r[((int64_t)k * ng + j / G) * M + i];
}

/*
 * The definition: for every requested row i, rebuild row i of W in fp64,
 *   W[i][j] = sum_k r_k(i, j) B_k[i][j] c_k[j]
 *           + sum_s sum_{t : S[t] = j} rs_s(i, t) Bs_s[i][t] cs_s[t],
 * and return y[b][row] = sum_j W[i][j] x[b][j].
 *
 *   signs     int8 [Kb][M][N]   (+1 / -1; 0 is accepted and contributes 0)
 *   r         [Kb][M] or [Kb][ceil(N/G)][M]
 *   c         [Kb][N]
 *   sal_signs int8 [Ks][M][n_sal]
 *   rs        [Ks][M] or [Ks][ceil(n_sal/Gs)][M]
 *   cs        [Ks][n_sal]
 *   sal_idx   [n_sal]  true column of salient column t (any order)
 *   x         [B][N]
 *   rows      [nrows]  row indices to evaluate
 *   y         [B][nrows]
 */
/* Row i of W in fp64 (w has N entries). */
static void rebuild_row(int64_t M, int64_t N, int Kb, int G,
                        const int8_t* signs, const double* r, const double* c,
                        int Ks, int64_t n_sal, int Gs,
                        const int8_t* sal_signs, const double* rs, const double* cs,
                        const int32_t* sal_idx, int64_t i, double* w) {
    for (int64_t j = 0; j < N; ++j) w[j] = 0.0;
    for (int k = 0; k < Kb; ++k) {
        const int8_t* s = signs + ((int64_t)k * M + i) * N;
        for (int64_t j = 0; j < N; ++j)
            w[j] += row_scale(r, M, N, G, k, i, j) * (double)s[j] * c[(int64_t)k * N + j];
    }
    for (int k = 0; k < Ks; ++k) {
        const int8_t* s = sal_signs + ((int64_t)k * M + i) * n_sal;
        for (int64_t t = 0; t < n_sal; ++t)
            w[sal_idx[t]] += row_scale(rs, M, n_sal, Gs, k, i, t) * (double)s[t] * cs[(int64_t)k * n_sal + t];
    }
}

/* y[b] = w . x[b] for one rebuilt row. */
static void dot_row(int64_t N, const double* w, int B, const double* x, int64_t nrows, int64_t q, double* y) {
    for (int b = 0; b < B; ++b) {
        const double* xb = x + (int64_t)b * N;
        double acc = 0.0;
        for (int64_t j = 0; j < N; ++j) acc += w[j] * xb[j];
        y[(int64_t)b * nrows + q] = acc;
    }
}

void oracle_linear_rows(int64_t M, int64_t N, int Kb, int G,
                        const int8_t* signs, const double* r, const double* c,
                        int Ks, int64_t n_sal, int Gs,
                        const int8_t* sal_signs, const double* rs, const double* cs,
                        const int32_t* sal_idx,
                        int B, const double* x,
                        int64_t nrows, const int64_t* rows, double* y) {
    #pragma omp parallel
    {
        double* w = (double*)malloc(sizeof(double) * (size_t)(N > 0 ? N : 1));
        #pragma omp for schedule(static)
        for (int64_t q = 0; q < nrows; ++q) {
            rebuild_row(M, N, Kb, G, signs, r, c, Ks, n_sal, Gs, sal_signs, rs, cs, sal_idx, rows[q], w);
            dot_row(N, w, B, x, nrows, q, y);
        }
        free(w);
    }
}

/* The two halves of oracle_linear_rows, timed apart by the CPU baseline:
 * the requested rows of W rebuilt in fp64 (W [nrows][N]) ... */
void oracle_rebuild_rows(int64_t M, int64_t N, int Kb, int G,
                         const int8_t* signs, const double* r, const double* c,
                         int Ks, int64_t n_sal, int Gs,
                         const int8_t* sal_signs, const double* rs, const double* cs,
                         const int32_t* sal_idx,
                         int64_t nrows, const int64_t* rows, double* W) {
    #pragma omp parallel for schedule(static)
    for (int64_t q = 0; q < nrows; ++q)
        rebuild_row(M, N, Kb, G, signs, r, c, Ks, n_sal, Gs, sal_signs, rs, cs, sal_idx, rows[q], W + q * N);
}

/* ... and the GEMV on those rebuilt rows: y[b][q] = W[q] . x[b]. */
void oracle_gemv_rows(int64_t N, int64_t nrows, const double* W, int B, const double* x, double* y) {
    #pragma omp parallel for schedule(static)
    for (int64_t q = 0; q < nrows; ++q) dot_row(N, W + q * N, B, x, nrows, q, y);
}

/* All 2^mu signed partial sums of one sub-vector: T[p] = sum_t (2 bit_t(p) - 1) v_t. */
void oracle_lut_table(const double* v, int mu, double* T) {
    int64_t E = (int64_t)1 << mu;
    for (int64_t p = 0; p < E; ++p) {
        double acc = 0.0;
        for (int t = 0; t < mu; ++t) acc += (((p >> t) & 1) ? v[t] : -v[t]);
        T[p] = acc;
    }
}

/* Symmetric half table: the 2^(mu-1) entries whose top bit is 0. */
void oracle_lut_table_sym(const double* v, int mu, double* Th) {
    int64_t E = (int64_t)1 << (mu - 1);
    for (int64_t p = 0; p < E; ++p) {
        double acc = 0.0;
        for (int t = 0; t < mu; ++t) acc += (((p >> t) & 1) ? v[t] : -v[t]);
        Th[p] = acc;
    }
}

/* Full-table value from the half table: T[p] = -T[~p] when the top bit of p is set. */
double oracle_lut_lookup_sym(const double* Th, int mu, int64_t p) {
    int64_t mask = ((int64_t)1 << mu) - 1;
    if ((p >> (mu - 1)) & 1) return -Th[(~p) & mask];
    return Th[p];
}

/*
 * Table quantisation (LUT Tensor Core notes, Section 3.1.3: the precomputed
 * table entries are stored in a lower precision than the activations).
 *
 * oracle_round_fp16: the IEEE binary16 value nearest to v (ties to the even
 * significand), from the format's definition: 10 fraction bits, exponents
 * -14 .. 15, subnormal spacing 2^-24, values at or beyond 65520 overflow.
 */
/*
 * The element-wise operator taken to precede a layer when the table
 * precompute is fused into it (LUT Tensor Core notes, Section 3.1.1): the RMS
 * normalisation of a LLaMA-style block,
 *     x[n] = h[n] * gamma[n] / sqrt(mean_m(h[m]^2) + eps),
 * the definition written out in fp64 (no rounding of x).
 */
void oracle_rmsnorm(int64_t N, const double* h, const double* gamma, double eps, double* x) {
    double ss = 0.0;
    for (int64_t n = 0; n < N; ++n) ss += h[n] * h[n];
    const double rms = sqrt(ss / (double)N + eps);
    for (int64_t n = 0; n < N; ++n) x[n] = h[n] * gamma[n] / rms;
}

double oracle_round_fp16(double v) {
    if (v != v) return v;
    double a = fabs(v);
    if (a >= 65520.0) return v > 0 ? INFINITY : -INFINITY;
    int e;
    (void)frexp(a, &e);                   /* a = f * 2^e, 0.5 <= f < 1 */
    int ex = e - 1;                       /* a in [2^ex, 2^(ex+1)) */
    if (ex < -14) ex = -14;               /* subnormals share the spacing of the smallest binade */
    double ulp = ldexp(1.0, ex - 10);
    double q = a / ulp;                   /* exact: a power-of-two scaling */
    double r = floor(q);
    double frac = q - r;
    if (frac > 0.5 || (frac == 0.5 && fmod(r, 2.0) != 0.0)) r += 1.0;
    return copysign(r * ulp, v);
}

/*
 * INT8 table with one scale per table: s = max_p |T[p]| / 127 and every
 * entry replaced by s * q, q the integer nearest to T[p] / s (ties to even),
 * |q| <= 127.  An all-zero table stays zero.  Returns s.
 */
double oracle_quantize_table_int8(double* T, int64_t E) {
    double m = 0.0;
    for (int64_t p = 0; p < E; ++p)
        if (fabs(T[p]) > m) m = fabs(T[p]);
    if (m == 0.0) return 0.0;
    double s = m / 127.0;
    for (int64_t p = 0; p < E; ++p) {
        double q = T[p] / s, r = floor(q), frac = q - r;
        if (frac > 0.5 || (frac == 0.5 && fmod(r, 2.0) != 0.0)) r += 1.0;
        if (r > 127.0) r = 127.0;
        if (r < -127.0) r = -127.0;
        T[p] = r * s;
    }
    return s;
}

/* Applies table quantisation mode tq (0: none, 1: fp16 entries, 2: INT8 per table). */
static void quantize_table(double* T, int64_t E, int tq) {
    if (tq == 1) {
        for (int64_t p = 0; p < E; ++p) T[p] = oracle_round_fp16(T[p]);
    } else if (tq == 2) {
        (void)oracle_quantize_table_int8(T, E);
    }
}

/*
 * One branch in LUT form, for every requested row:
 *   acc_k,g(i) = sum over sub-vectors j of the block g of T_{k,j}[pattern of B_k[i][j*mu .. j*mu+mu-1]]
 *   y(i)      += sum_{k,g} r_k(i, g) acc_k,g(i)
 * with v_{k,j,t} = c_k[j*mu+t] * x[col(j*mu+t)] (0 beyond ncols), col = gather or identity.
 * The row-scale block (G columns) must hold whole sub-vectors (G % mu == 0).
 * Adds into y[b][nrows] (caller zeroes it).
 */
static void lut_branch_rows(int64_t M, int64_t ncols, int64_t N, int nb, int mu, int G,
                            const int8_t* signs, const double* r, const double* c,
                            const int32_t* gather, int B, const double* x,
                            int64_t nrows, const int64_t* rows, int sym, int tq, double* y) {
    int64_t nsub = (ncols + mu - 1) / mu;
    int64_t E = (int64_t)1 << mu;
    int64_t Estore = sym ? (E >> 1) : E;
    double* tab = (double*)malloc(sizeof(double) * (size_t)(nb * nsub * Estore + 1));
    double v[16];
    for (int b = 0; b < B; ++b) {
        const double* xb = x + (int64_t)b * N;
        /* LUT building with scale fusion: one table per base and sub-vector. */
        for (int k = 0; k < nb; ++k)
            for (int64_t j = 0; j < nsub; ++j) {
                for (int t = 0; t < mu; ++t) {
                    int64_t n = j * mu + t;
                    v[t] = (n < ncols) ? c[(int64_t)k * ncols + n] * xb[gather ? gather[n] : n] : 0.0;
                }
                double* T = tab + ((int64_t)k * nsub + j) * Estore;
                if (sym) oracle_lut_table_sym(v, mu, T); else oracle_lut_table(v, mu, T);
                quantize_table(T, Estore, tq);
            }
        /* Lookup and accumulate; the row scale multiplies the accumulated sum. */
        for (int64_t q = 0; q < nrows; ++q) {
            int64_t i = rows[q];
            double out = 0.0;
            for (int k = 0; k < nb; ++k) {
                const int8_t* s = signs + ((int64_t)k * M + i) * ncols;
                double acc = 0.0;
                int64_t gcur = -1;
                for (int64_t j = 0; j < nsub; ++j) {
                    int64_t p = 0;
                    for (int t = 0; t < mu; ++t) {
                        int64_t n = j * mu + t;
                        int bit = (n < ncols) ? (s[n] > 0) : 0;
                        p |= (int64_t)bit << t;
                    }
                    const double* T = tab + ((int64_t)k * nsub + j) * Estore;
                    double tv = sym ? oracle_lut_lookup_sym(T, mu, p) : T[p];
                    if (G > 0) {
                        int64_t g = (j * mu) / G;
                        if (g != gcur) {
                            if (gcur >= 0) out += row_scale(r, M, ncols, G, k, i, gcur * G) * acc;
                            acc = 0.0;
                            gcur = g;
                        }
                    }
                    acc += tv;
                }
                if (G > 0) {
                    if (gcur >= 0) out += row_scale(r, M, ncols, G, k, i, gcur * G) * acc;
                } else {
                    out += r[(int64_t)k * M + i] * acc;
                }
            }
            y[(int64_t)b * nrows + q] += out;
        }
    }
    free(tab);
}

/*
 * The full layer in LUT form: the global branch over the N input columns,
 * plus the salient branch over its dense n_sal columns whose activations and
 * scales are gathered through sal_idx (Virtual Columnar Mapping).
 * sym != 0 uses the symmetric half tables; tq quantises every table after it
 * is built (0: none, 1: fp16 entries, 2: INT8 with a per-table scale).  Signs must be +-1 here (a zero
 * has no bit pattern).  Block sizes G and Gs must be multiples of mu.
 * Returns 0, or -1 if a block size does not hold whole sub-vectors.
 */
int oracle_lut_linear_rows(int64_t M, int64_t N, int Kb, int G,
                           const int8_t* signs, const double* r, const double* c,
                           int Ks, int64_t n_sal, int Gs,
                           const int8_t* sal_signs, const double* rs, const double* cs,
                           const int32_t* sal_idx, int mu, int sym, int tq,
                           int B, const double* x,
                           int64_t nrows, const int64_t* rows, double* y) {
    if ((G > 0 && G % mu) || (Gs > 0 && Gs % mu) || mu < 1 || mu > 16 || tq < 0 || tq > 2) return -1;
    memset(y, 0, sizeof(double) * (size_t)(B * nrows));
    lut_branch_rows(M, N, N, Kb, mu, G, signs, r, c, NULL, B, x, nrows, rows, sym, tq, y);
    if (Ks > 0 && n_sal > 0)
        lut_branch_rows(M, n_sal, N, Ks, mu, Gs, sal_signs, rs, cs, sal_idx, B, x, nrows, rows, sym, tq, y);
    return 0;
}

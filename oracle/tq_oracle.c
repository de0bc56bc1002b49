/*
 * tq_oracle.c -- plain, slow CPU oracle for TurboQuant KV-vector compression.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check and the CPU-baseline
 * leg of the benchmark may load this library.  It shares no code, header, table
 * or constant with the CUDA library: everything here is written out again from
 * the method's definition, in double precision, one vector / one token at a time.
 *
 * Sources (web pages about the turboquant-pytorch / turboquant-py implementations
 * of Google's TurboQuant):
 *   [P2] "turboquant-pytorch" skill page (atskills.one), sections "What It Does",
 *        "Algorithm Details: Why Random Rotation? / Why QJL for Keys but Not Values?"
 *   [P3] "turboquant-pytorch" skill page (nav.superapi.store), sections
 *        主要能力 (two stages), 核心 API (build_lloyd_max_codebook, TurboQuantMSE,
 *        TurboQuantProd, TurboQuantKVCache, compressors), 常见使用模式 (usage
 *        patterns), 算法细节 (algorithm details), 限制与注意事项 (caveats)
 *   [P5] "TurboQuant er nå tilgjengelig som Python-bibliotek" (jansverre.net),
 *        sections "Hva er TurboQuant, kort fortalt?" and "Hva gjør Python-implementasjonen?"
 *
 * Readings taken where the pages are silent (each is also listed in the design notes):
 *   - rotation convention y = R u (R applied from the left to the unit vector);
 *   - code of a coordinate = number of interior boundaries strictly below it, so a
 *     value equal to a boundary goes to the lower cell;  the decision is taken on the
 *     fp32-rounded rotated value against fp32-rounded boundaries (the precision the
 *     GPU kernels decide in);
 *   - keys spend (bits-1) bits on the MSE stage and 1 bit per projection on QJL;
 *   - QJL residual in the original space, r = u - R^T c[idx];  sign(0) -> bit 1;
 *   - inner-product estimate <q,u> ~ <q, R^T c[idx]> + rho*sqrt(pi/2)/m * <S q, sign(S r)>,
 *     scaled by the stored key norm;  norms are used after fp16 rounding (what is stored);
 *   - attention: softmax(scale * score) over all tokens, no mask, GQA head h reads KV
 *     head h / (Hq/Hkv);
 *   - packed layout: per 32-coordinate group g, word g*beta+p holds bit p of the
 *     codes of coordinates 32g..32g+31 at bit positions 0..31 (planar); sign word g
 *     bit l = [p_{32g+l} >= 0].
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#ifdef _OPENMP
#include <omp.h>
#endif

#define ORA_PI 3.14159265358979323846

/* ------------------------------------------------------------------ fp16 */

/* IEEE binary16, round-to-nearest-even from a double. */
uint16_t ora_f64_to_f16(double v)
{
    uint16_t sign = 0;
    if (signbit(v)) { sign = 0x8000; v = -v; }
    if (isnan(v)) return (uint16_t)(sign | 0x7e00);
    if (isinf(v)) return (uint16_t)(sign | 0x7c00);
    /* largest finite half is 65504; values >= 65520 round to infinity */
    if (v >= 65520.0) return (uint16_t)(sign | 0x7c00);
    if (v < ldexp(1.0, -14)) {
        /* subnormal range: units of 2^-24 */
        double q = v * ldexp(1.0, 24);
        double f = floor(q);
        double rem = q - f;
        uint32_t m = (uint32_t)f;
        if (rem > 0.5 || (rem == 0.5 && (m & 1u))) m += 1;
        return (uint16_t)(sign | m); /* m == 1024 becomes the smallest normal, which is correct */
    }
    int e;
    double fr = frexp(v, &e); /* v = fr * 2^e, fr in [0.5, 1) */
    /* v = 1.mant * 2^(e-1); 10 fraction bits */
    double q = fr * 2048.0; /* in [1024, 2048) */
    double f = floor(q);
    double rem = q - f;
    uint32_t m = (uint32_t)f;
    if (rem > 0.5 || (rem == 0.5 && (m & 1u))) m += 1;
    int exp_h = e - 1 + 15;
    if (m == 2048) { m = 1024; exp_h += 1; }
    if (exp_h >= 31) return (uint16_t)(sign | 0x7c00);
    return (uint16_t)(sign | ((uint32_t)exp_h << 10) | (m - 1024));
}

double ora_f16_to_f64(uint16_t h)
{
    int s = (h >> 15) & 1;
    int e = (h >> 10) & 31;
    int m = h & 1023;
    double v;
    if (e == 0) v = ldexp((double)m, -24);
    else if (e == 31) v = m ? NAN : INFINITY;
    else v = ldexp((double)(m + 1024), e - 25);
    return s ? -v : v;
}

/* --------------------------------------------------------- Lloyd-Max codebook */

static double std_pdf(double t) { return exp(-0.5 * t * t) / sqrt(2.0 * ORA_PI); }
/* upper tail Q(t) = P(Z > t) */
static double std_upper(double t) { return 0.5 * erfc(t / sqrt(2.0)); }

/*
 * Lloyd-Max scalar quantizer for one coordinate of a randomly rotated unit vector,
 * whose law the pages give as N(0, 1/dim) ([P2] "Why Random Rotation?", [P3] 算法细节;
 * build_lloyd_max_codebook(dim, bits) -> (boundaries, centroids) in [P3] 核心 API).
 *
 * Lloyd's two conditions, alternated until nothing moves:
 *   boundary_k = (c_k + c_{k+1}) / 2                                  (nearest neighbour)
 *   c_k        = E[Z | b_{k-1} < Z < b_k]
 *              = (pdf(b_{k-1}) - pdf(b_k)) / (P(Z > b_{k-1}) - P(Z > b_k))  (centroid)
 * in standard-normal units, with b_{-1} = -inf and b_{K-1} = +inf; then everything is
 * scaled by sigma = 1/sqrt(dim).  The conditional mean of the Gaussian has this closed
 * form, so no numerical integration is needed.
 *
 * bounds: K-1 interior boundaries (ascending), cents: K centroids (ascending).
 * Returns the number of iterations, or -1 on bad arguments / no convergence.
 */
int ora_codebook(int dim, int bits, double *bounds, double *cents)
{
    if (dim <= 0 || bits < 1 || bits > 8) return -1;
    const int K = 1 << bits;
    double *c = (double *)malloc(sizeof(double) * K);
    double *b = (double *)malloc(sizeof(double) * (K + 1));
    for (int k = 0; k < K; ++k) c[k] = -3.0 + 6.0 * (k + 0.5) / K;
    int it;
    const int max_it = 200000;
    for (it = 1; it <= max_it; ++it) {
        b[0] = -INFINITY;
        b[K] = INFINITY;
        for (int k = 1; k < K; ++k) b[k] = 0.5 * (c[k - 1] + c[k]);
        double delta = 0.0;
        for (int k = 0; k < K; ++k) {
            double lo = b[k], hi = b[k + 1];
            double plo = isinf(lo) ? 0.0 : std_pdf(lo);
            double phi_ = isinf(hi) ? 0.0 : std_pdf(hi);
            /* P(lo < Z < hi) from upper tails, accurate in both tails via symmetry */
            double mass;
            if (lo >= 0.0) {
                mass = std_upper(lo) - (isinf(hi) ? 0.0 : std_upper(hi));
            } else if (hi <= 0.0) {
                mass = std_upper(-hi) - (isinf(lo) ? 0.0 : std_upper(-lo));
            } else {
                mass = 1.0 - (isinf(lo) ? 0.0 : std_upper(-lo)) - (isinf(hi) ? 0.0 : std_upper(hi));
            }
            double nc = (plo - phi_) / mass;
            double dd = fabs(nc - c[k]);
            if (dd > delta) delta = dd;
            c[k] = nc;
        }
        if (delta < 1e-15) break;
    }
    if (it > max_it) { free(c); free(b); return -1; }
    /* the law is symmetric: make the codebook exactly antisymmetric */
    for (int k = 0; k < K / 2; ++k) {
        double a = 0.5 * (c[K - 1 - k] - c[k]);
        c[k] = -a;
        c[K - 1 - k] = a;
    }
    const double sigma = 1.0 / sqrt((double)dim);
    for (int k = 0; k < K; ++k) cents[k] = c[k] * sigma;
    for (int k = 1; k < K; ++k) bounds[k - 1] = 0.5 * (c[k - 1] + c[k]) * sigma;
    bounds[K / 2 - 1] = 0.0;
    free(c);
    free(b);
    return it;
}

/*
 * Lloyd-Max quantizer for the exact law of one coordinate of a uniformly random unit vector
 * in R^dim, which [P5] "Hva er TurboQuant, kort fortalt?" describes as a concentrated Beta law:
 * y = 2 B - 1 with B ~ Beta((dim-1)/2, (dim-1)/2), i.e. density proportional to
 * (1 - y^2)^((dim-3)/2) on (-1, 1).  (N(0, 1/dim) is its large-dim limit.)
 *
 * The same two conditions as above, alternated until nothing moves:
 *   boundary_k = (c_k + c_{k+1}) / 2,   c_k = E[y | b_{k-1} < y < b_k]   (b_{-1} = -1, b_{K-1} = 1)
 * The conditional mean is (int y f) / (int f) over the cell.  With y = sin(theta) both integrals
 * become integrals of smooth functions of theta, int cos^(dim-2) and int sin cos^(dim-2), taken
 * by composite 16-point Gauss-Legendre quadrature on panels no wider than 1/(2 sqrt(dim)).
 * Returns the number of iterations, or -1 on bad arguments / no convergence.
 */
static double gl_x[16], gl_w[16];
static int gl_ready = 0;

static void gauss_legendre16(void)
{
    /* nodes: roots of P_16 by Newton's method; weights 2 / ((1 - x^2) P_16'(x)^2) */
    const int n = 16;
    for (int i = 0; i < n / 2; ++i) {
        double z = cos(ORA_PI * (i + 0.75) / (n + 0.5)), dp = 0.0;
        for (int it = 0; it < 100; ++it) {
            double p0 = 1.0, p1 = z;
            for (int k = 2; k <= n; ++k) {
                const double p2 = ((2.0 * k - 1.0) * z * p1 - (k - 1.0) * p0) / k;
                p0 = p1;
                p1 = p2;
            }
            dp = n * (z * p1 - p0) / (z * z - 1.0);
            const double dz = p1 / dp;
            z -= dz;
            if (fabs(dz) < 1e-16) break;
        }
        gl_x[i] = -z;
        gl_x[n - 1 - i] = z;
        gl_w[i] = gl_w[n - 1 - i] = 2.0 / ((1.0 - z * z) * dp * dp);
    }
    gl_ready = 1;
}

/* mass and first moment of the law over (lo, hi), up to the common normalising constant */
static void beta_cell(int dim, double lo, double hi, double *mass, double *moment)
{
    const double t0 = asin(lo), t1 = asin(hi);
    double hmax = 0.5 / sqrt((double)dim);
    if (hmax > 0.05) hmax = 0.05;
    int panels = (int)ceil((t1 - t0) / hmax);
    if (panels < 1) panels = 1;
    const double h = (t1 - t0) / panels;
    double m0 = 0.0, m1 = 0.0;
    for (int p = 0; p < panels; ++p) {
        const double mid = t0 + (p + 0.5) * h;
        for (int i = 0; i < 16; ++i) {
            const double th = mid + 0.5 * h * gl_x[i];
            const double w = 0.5 * h * gl_w[i] * pow(cos(th), dim - 2);
            m0 += w;
            m1 += w * sin(th);
        }
    }
    *mass = m0;
    *moment = m1;
}

int ora_codebook_beta(int dim, int bits, double *bounds, double *cents)
{
    if (dim < 2 || bits < 1 || bits > 8) return -1;
    if (!gl_ready) gauss_legendre16();
    const int K = 1 << bits;
    double *c = (double *)malloc(sizeof(double) * K);
    double *b = (double *)malloc(sizeof(double) * (K + 1));
    double spread = 3.0 / sqrt((double)dim);
    if (spread > 0.9) spread = 0.9;
    for (int k = 0; k < K; ++k) c[k] = spread * (-1.0 + (2.0 * k + 1.0) / K);
    const double tol = 1e-14 / sqrt((double)dim);
    int it;
    const int max_it = 200000;
    for (it = 1; it <= max_it; ++it) {
        b[0] = -1.0;
        b[K] = 1.0;
        for (int k = 1; k < K; ++k) b[k] = 0.5 * (c[k - 1] + c[k]);
        double delta = 0.0;
        for (int k = 0; k < K; ++k) {
            double m0, m1;
            beta_cell(dim, b[k], b[k + 1], &m0, &m1);
            const double nc = m1 / m0;
            const double dd = fabs(nc - c[k]);
            if (dd > delta) delta = dd;
            c[k] = nc;
        }
        if (delta < tol) break;
    }
    if (it > max_it) { free(c); free(b); return -1; }
    /* the law is symmetric: make the codebook exactly antisymmetric */
    for (int k = 0; k < K / 2; ++k) {
        double a = 0.5 * (c[K - 1 - k] - c[k]);
        c[k] = -a;
        c[K - 1 - k] = a;
    }
    for (int k = 0; k < K; ++k) cents[k] = c[k];
    for (int k = 1; k < K; ++k) bounds[k - 1] = 0.5 * (c[k - 1] + c[k]);
    bounds[K / 2 - 1] = 0.0;
    free(c);
    free(b);
    return it;
}

/* law 0: N(0, 1/dim) (ora_codebook); law 1: the exact Beta law (ora_codebook_beta) */
int ora_codebook_law(int dim, int bits, int law, double *bounds, double *cents)
{
    if (law == 0) return ora_codebook(dim, bits, bounds, cents);
    if (law == 1) return ora_codebook_beta(dim, bits, bounds, cents);
    return -1;
}

/* fp32-rounded codebook of either law */
int ora_codebook_law_f32(int dim, int bits, int law, float *bounds, float *cents)
{
    const int K = 1 << bits;
    double cb[256], cc[256];
    int it = ora_codebook_law(dim, bits, law, cb, cc);
    if (it < 0) return it;
    for (int k = 0; k < K - 1; ++k) bounds[k] = (float)cb[k];
    for (int k = 0; k < K; ++k) cents[k] = (float)cc[k];
    return it;
}

/* fp32-rounded codebook: the values the quantizer decides against and dequantizes to. */
int ora_codebook_f32(int dim, int bits, float *bounds, float *cents)
{
    const int K = 1 << bits;
    double cb[256], cc[256];
    int it = ora_codebook(dim, bits, cb, cc);
    if (it < 0) return it;
    for (int k = 0; k < K - 1; ++k) bounds[k] = (float)cb[k];
    for (int k = 0; k < K; ++k) cents[k] = (float)cc[k];
    return it;
}

/* ------------------------------------------------------------ packed layout */

static void pack_codes(const int *idx, int dim, int beta, uint32_t *words)
{
    const int groups = dim / 32;
    memset(words, 0, sizeof(uint32_t) * (size_t)groups * beta);
    for (int j = 0; j < dim; ++j) {
        int g = j / 32, l = j % 32;
        for (int p = 0; p < beta; ++p)
            if ((idx[j] >> p) & 1) words[g * beta + p] |= (1u << l);
    }
}

static void unpack_codes(const uint32_t *words, int dim, int beta, int *idx)
{
    for (int j = 0; j < dim; ++j) {
        int g = j / 32, l = j % 32, v = 0;
        for (int p = 0; p < beta; ++p) v |= (int)((words[g * beta + p] >> l) & 1u) << p;
        idx[j] = v;
    }
}

/* exported for the round-trip pin */
void ora_pack_codes(const int32_t *idx, int dim, int beta, uint32_t *words)
{
    int *tmp = (int *)malloc(sizeof(int) * dim);
    for (int j = 0; j < dim; ++j) tmp[j] = idx[j];
    pack_codes(tmp, dim, beta, words);
    free(tmp);
}

void ora_unpack_codes(const uint32_t *words, int dim, int beta, int32_t *idx)
{
    int *tmp = (int *)malloc(sizeof(int) * dim);
    unpack_codes(words, dim, beta, tmp);
    for (int j = 0; j < dim; ++j) idx[j] = tmp[j];
    free(tmp);
}

/* ------------------------------------------------------------- compression */

/*
 * Compress n vectors (TurboQuantMSE.quantize for values, TurboQuantProd.compress for keys;
 * [P3] 核心 API and 常见使用模式, [P2] "What It Does", [P5] TurboQuantProd description).
 *
 * For each vector x (dim coordinates):
 *   1. n = ||x||, u = x / n             (inputs are normalised first: [P3] 限制与注意事项)
 *   2. y = R u                          (stage 1: random orthogonal rotation)
 *   3. idx_j = #{k : boundary_k < y_j}  (Lloyd-Max scalar quantization per coordinate)
 *   4. codes = planar bit-pack of idx
 * keys additionally (stage 2, QJL on the residual):
 *   5. x_hat = R^T c[idx]               (the MSE dequantization)
 *   6. r = u - x_hat, rho = ||r||
 *   7. p = S r, sign bit_i = [p_i >= 0]
 *
 * is_key: 1 for keys (beta = bits-1 MSE bits + signs), 0 for values (beta = bits).
 * x: n*dim values, fp16 bits (x_is_f16 = 1) or fp32.  R: dim*dim fp32, S: m*dim fp32.
 * codes: n * beta*dim/32 words; signs: n * m/32 words (keys); norm, rnorm: fp16 bits.
 * y32_out (optional, n*dim): the fp32-rounded rotated coordinates the codes were decided on.
 * p32_out (optional, n*m): the fp32-rounded projections the signs were decided on.
 */
int ora_compress(int is_key, int dim, int bits, int m, const float *R, const float *S,
                 const void *x, int x_is_f16, int64_t n, uint32_t *codes, uint32_t *signs,
                 uint16_t *norm, uint16_t *rnorm, float *y32_out, float *p32_out, int law)
{
    const int beta = is_key ? bits - 1 : bits;
    if (dim <= 0 || dim % 32 || beta < 1 || beta > 8) return -1;
    if (is_key && (m <= 0 || m % 32)) return -1;
    const int K = 1 << beta;
    float cb32[256], cc32[256];
    if (ora_codebook_law_f32(dim, beta, law, cb32, cc32) < 0) return -1;
    const int wpv = beta * dim / 32;

#pragma omp parallel
    {
        double *u = (double *)malloc(sizeof(double) * dim);
        double *y = (double *)malloc(sizeof(double) * dim);
        double *xh = (double *)malloc(sizeof(double) * dim);
        int *idx = (int *)malloc(sizeof(int) * dim);
#pragma omp for schedule(static)
        for (int64_t v = 0; v < n; ++v) {
            /* 1. norm and unit vector */
            double ss = 0.0;
            for (int j = 0; j < dim; ++j) {
                double xv = x_is_f16 ? ora_f16_to_f64(((const uint16_t *)x)[v * dim + j])
                                     : (double)((const float *)x)[v * dim + j];
                u[j] = xv;
                ss += xv * xv;
            }
            double nv = sqrt(ss);
            for (int j = 0; j < dim; ++j) u[j] = (nv > 0.0) ? u[j] / nv : 0.0;
            norm[v] = ora_f64_to_f16(nv);
            /* 2. rotate: y = R u */
            for (int i = 0; i < dim; ++i) {
                double acc = 0.0;
                for (int j = 0; j < dim; ++j) acc += (double)R[(size_t)i * dim + j] * u[j];
                y[i] = acc;
            }
            /* 3. quantize each coordinate against the fp32 boundaries */
            for (int i = 0; i < dim; ++i) {
                float y32 = (float)y[i];
                if (y32_out) y32_out[v * dim + i] = y32;
                int c = 0;
                for (int k = 0; k < K - 1; ++k)
                    if (cb32[k] < y32) ++c;
                idx[i] = c;
            }
            /* 4. pack */
            pack_codes(idx, dim, beta, codes + v * wpv);
            if (!is_key) continue;
            /* 5. dequantize: x_hat = R^T c[idx] */
            for (int j = 0; j < dim; ++j) {
                double acc = 0.0;
                for (int i = 0; i < dim; ++i) acc += (double)R[(size_t)i * dim + j] * (double)cc32[idx[i]];
                xh[j] = acc;
            }
            /* 6. residual and its norm */
            double rr = 0.0;
            for (int j = 0; j < dim; ++j) {
                xh[j] = u[j] - xh[j]; /* xh now holds r */
                rr += xh[j] * xh[j];
            }
            rnorm[v] = ora_f64_to_f16(sqrt(rr));
            /* 7. QJL: signs of S r */
            uint32_t *sw = signs + v * (m / 32);
            memset(sw, 0, sizeof(uint32_t) * (m / 32));
            for (int i = 0; i < m; ++i) {
                double acc = 0.0;
                for (int j = 0; j < dim; ++j) acc += (double)S[(size_t)i * dim + j] * xh[j];
                float p32 = (float)acc;
                if (p32_out) p32_out[v * m + i] = p32;
                if (p32 >= 0.0f) sw[i / 32] |= 1u << (i % 32);
            }
        }
        free(u);
        free(y);
        free(xh);
        free(idx);
    }
    return 0;
}

/* ------------------------------------------------------ dequantization helper */

/* x_hat = norm * R^T c[idx] for one packed vector (original space). */
static void dequant_one(int dim, int beta, const float *R, const float *cc32, const uint32_t *words,
                        double scale, int *idx, double *out)
{
    unpack_codes(words, dim, beta, idx);
    /* out[j] = scale * sum_i R[i][j] c[idx_i], summed over i in ascending order (rows of R are
       walked in memory order; every out[j] sees the same sequence of additions as a column walk) */
    for (int j = 0; j < dim; ++j) out[j] = 0.0;
    for (int i = 0; i < dim; ++i) {
        const double ci = (double)cc32[idx[i]];
        const float *Ri = R + (size_t)i * dim;
        for (int j = 0; j < dim; ++j) out[j] += (double)Ri[j] * ci;
    }
    for (int j = 0; j < dim; ++j) out[j] *= scale;
}

/* Dequantize n packed vectors to the original space (TurboQuantMSE.dequantize). */
int ora_dequantize(int dim, int beta, const float *R, const uint32_t *codes, const uint16_t *norm,
                   int64_t n, double *out, int law)
{
    float cb32[256], cc32[256];
    if (ora_codebook_law_f32(dim, beta, law, cb32, cc32) < 0) return -1;
    const int wpv = beta * dim / 32;
#pragma omp parallel
    {
        int *idx = (int *)malloc(sizeof(int) * dim);
#pragma omp for schedule(static)
        for (int64_t v = 0; v < n; ++v)
            dequant_one(dim, beta, R, cc32, codes + v * wpv, ora_f16_to_f64(norm[v]), idx,
                        out + v * dim);
        free(idx);
    }
    return 0;
}

/* ------------------------------------------------------------------ scoring */

/*
 * Asymmetric inner-product estimate of <q, k> from a packed key
 * (TurboQuantProd.inner_product / asymmetric_attention_scores; [P3] 核心 API and
 * 常见使用模式 "asymmetric_attention_scores ... directly from the compressed keys"):
 *   s = ||k|| * ( <q, R^T c[idx]> + rho * sqrt(pi/2)/m * <S q, 2*bit - 1> )
 * The sqrt(pi/2)/m factor is what makes the 1-bit sign sketch unbiased
 * ([P2] "QJL residual correction ... makes inner product estimates unbiased"):
 * for s ~ N(0, I), E[(s.q) sign(s.r)] = sqrt(2/pi) <q, r> / ||r||.
 *
 * q: [B, Hq, Nq, dim] fp32.  Keys: [B, Hkv, T] records.  scores: [B, Hq, Nq, T] doubles.
 */
int ora_scores(int dim, int bits, int m, const float *R, const float *S, const float *q, int B, int Hq,
               int Hkv, int Nq, int64_t T, const uint32_t *kcodes, const uint32_t *ksigns,
               const uint16_t *knorm, const uint16_t *krnorm, double *scores, int law)
{
    const int beta = bits - 1;
    if (Hkv <= 0 || Hq % Hkv) return -1;
    const int G = Hq / Hkv;
    float cb32[256], cc32[256];
    if (ora_codebook_law_f32(dim, beta, law, cb32, cc32) < 0) return -1;
    const int wpk = beta * dim / 32, spk = m / 32;
    const double qjl = sqrt(ORA_PI / 2.0) / (double)m;
    const int64_t slices = (int64_t)B * Hkv;
    for (int64_t sl = 0; sl < slices; ++sl) {
        const int b = (int)(sl / Hkv), kv = (int)(sl % Hkv);
        /* S q for every query row that reads this KV head */
        double *sq = (double *)malloc(sizeof(double) * (size_t)G * Nq * m);
        for (int g = 0; g < G; ++g)
            for (int i = 0; i < Nq; ++i) {
                const float *qr = q + (((size_t)b * Hq + kv * G + g) * Nq + i) * dim;
                for (int a = 0; a < m; ++a) {
                    double acc = 0.0;
                    for (int j = 0; j < dim; ++j) acc += (double)S[(size_t)a * dim + j] * (double)qr[j];
                    sq[((size_t)g * Nq + i) * m + a] = acc;
                }
            }
#pragma omp parallel
        {
            int *idx = (int *)malloc(sizeof(int) * dim);
            double *xh = (double *)malloc(sizeof(double) * dim);
#pragma omp for schedule(static)
            for (int64_t t = 0; t < T; ++t) {
                const int64_t rec = sl * T + t;
                /* MSE part: dequantize the unit key and take the plain dot product */
                dequant_one(dim, beta, R, cc32, kcodes + rec * wpk, 1.0, idx, xh);
                const double nk = ora_f16_to_f64(knorm[rec]);
                const double rho = ora_f16_to_f64(krnorm[rec]);
                const uint32_t *sw = ksigns + rec * spk;
                for (int g = 0; g < G; ++g)
                    for (int i = 0; i < Nq; ++i) {
                        const float *qr = q + (((size_t)b * Hq + kv * G + g) * Nq + i) * dim;
                        double d1 = 0.0;
                        for (int j = 0; j < dim; ++j) d1 += (double)qr[j] * xh[j];
                        const double *sqr = sq + ((size_t)g * Nq + i) * m;
                        double d2 = 0.0;
                        for (int a = 0; a < m; ++a) {
                            double sgn = ((sw[a / 32] >> (a % 32)) & 1u) ? 1.0 : -1.0;
                            d2 += sqr[a] * sgn;
                        }
                        scores[(((size_t)b * Hq + kv * G + g) * Nq + i) * T + t] =
                            nk * (d1 + rho * qjl * d2);
                    }
            }
            free(idx);
            free(xh);
        }
        free(sq);
    }
    return 0;
}

/* ---------------------------------------------------------------- attention */

/*
 * Attention over a compressed cache ([P3] 常见使用模式: asymmetric scores from the
 * compressed keys, softmax, weighted sum over the decompressed values; values are
 * stage-1 (MSE) only, [P2] "Why QJL for Keys but Not Values?").
 *   a_t = exp(scale*s_t - max) / sum_u exp(scale*s_u - max)
 *   o   = sum_t a_t * ||v_t|| * R^T c[idx_t]
 * q: [B, Hq, Nq, dim]; out: [B, Hq, Nq, dim] doubles.
 */
int ora_attend(int dim, int bits, int m, const float *R, const float *S, const float *q, int B, int Hq,
               int Hkv, int Nq, int64_t T, const uint32_t *kcodes, const uint32_t *ksigns,
               const uint16_t *knorm, const uint16_t *krnorm, const uint32_t *vcodes,
               const uint16_t *vnorm, double scale, double *out, int law)
{
    if (Hkv <= 0 || Hq % Hkv || T <= 0) return -1;
    const int G = Hq / Hkv;
    const int vbeta = bits;
    float cb32[256], cc32[256];
    if (ora_codebook_law_f32(dim, vbeta, law, cb32, cc32) < 0) return -1;
    const int wpv = vbeta * dim / 32;
    double *sc = (double *)malloc(sizeof(double) * (size_t)B * Hq * Nq * T);
    if (!sc) return -1;
    int rc = ora_scores(dim, bits, m, R, S, q, B, Hq, Hkv, Nq, T, kcodes, ksigns, knorm, krnorm, sc, law);
    if (rc) { free(sc); return rc; }
    const int64_t rows = (int64_t)B * Hq * Nq;
    /* dequantized values of one KV slice, shared by the G heads that read it */
    for (int64_t sl = 0; sl < (int64_t)B * Hkv; ++sl) {
        const int b = (int)(sl / Hkv), kv = (int)(sl % Hkv);
        double *vh = (double *)malloc(sizeof(double) * (size_t)T * dim);
#pragma omp parallel
        {
            int *idx = (int *)malloc(sizeof(int) * dim);
#pragma omp for schedule(static)
            for (int64_t t = 0; t < T; ++t)
                dequant_one(dim, vbeta, R, cc32, vcodes + (sl * T + t) * wpv,
                            ora_f16_to_f64(vnorm[sl * T + t]), idx, vh + (size_t)t * dim);
            free(idx);
        }
#pragma omp parallel for schedule(static)
        for (int gi = 0; gi < G * Nq; ++gi) {
            const int g = gi / Nq, i = gi % Nq;
            const int64_t row = ((int64_t)b * Hq + kv * G + g) * Nq + i;
            const double *s = sc + row * T;
            double mx = -INFINITY;
            for (int64_t t = 0; t < T; ++t)
                if (scale * s[t] > mx) mx = scale * s[t];
            double den = 0.0;
            for (int64_t t = 0; t < T; ++t) den += exp(scale * s[t] - mx);
            double *o = out + row * dim;
            for (int j = 0; j < dim; ++j) o[j] = 0.0;
            for (int64_t t = 0; t < T; ++t) {
                const double a = exp(scale * s[t] - mx) / den;
                for (int j = 0; j < dim; ++j) o[j] += a * vh[(size_t)t * dim + j];
            }
        }
        free(vh);
    }
    (void)rows;
    free(sc);
    return 0;
}

/* ------------------------------------------------------------------ top-k */

typedef struct { double s; int64_t i; } ora_pair;

static int pair_cmp(const void *a, const void *b)
{
    const ora_pair *x = (const ora_pair *)a, *y = (const ora_pair *)b;
    if (x->s > y->s) return -1;
    if (x->s < y->s) return 1;
    return (x->i < y->i) ? -1 : (x->i > y->i);
}

/*
 * Nearest-neighbour search by estimated inner product ([P5] TurboQuantProd for vector
 * databases): the k largest scores of each row, descending, ties to the smaller index.
 */
int ora_topk(const double *scores, int64_t rows, int64_t T, int k, int64_t *idx, double *val)
{
    if (k <= 0 || k > T) return -1;
#pragma omp parallel
    {
        ora_pair *buf = (ora_pair *)malloc(sizeof(ora_pair) * (size_t)T);
#pragma omp for schedule(static)
        for (int64_t r = 0; r < rows; ++r) {
            for (int64_t t = 0; t < T; ++t) { buf[t].s = scores[r * T + t]; buf[t].i = t; }
            qsort(buf, (size_t)T, sizeof(ora_pair), pair_cmp);
            for (int j = 0; j < k; ++j) { idx[r * k + j] = buf[j].i; val[r * k + j] = buf[j].s; }
        }
        free(buf);
    }
    return 0;
}

/* ---------------------------------------------------------- size accounting */

/*
 * Nominal compressed KV-cache size in bytes ([P3] 常见使用模式 "估算内存节省": from
 * layers, KV heads, sequence length, head_dim and bits; [P2] size table 289 -> 76/58/40 MB):
 * b bits per coordinate for both K and V plus three 16-bit scalars per token-head
 * (key norm, residual norm, value norm).  fp16 baseline: 2 bytes per coordinate, K and V.
 */
double ora_nominal_bytes(int layers, int kv_heads, int64_t seq, int dim, int bits)
{
    double per = 2.0 * ceil((double)dim * bits / 8.0) + 6.0;
    return (double)layers * kv_heads * (double)seq * per;
}

double ora_fp16_bytes(int layers, int kv_heads, int64_t seq, int dim)
{
    return (double)layers * kv_heads * (double)seq * 2.0 * dim * 2.0;
}

int ora_num_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

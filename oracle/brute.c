/*
 * Scalar brute-force oracle of the vision-to-language bridge.
 * TEST INFRASTRUCTURE ONLY: loaded by the tests to cross-check the numpy oracle
 * on tiny grids; never linked into or called by the CUDA library.
 *
 * Everything is a direct index formula evaluated one element at a time, in
 * double precision, so that it shares no reshape/transpose logic with the
 * numpy oracle:
 *   - space-to-depth with high-end zero pad and channel-outermost order
 *     c*k*k + dy*k + dx  ("port DeepSeek-VL2", Projector steps 1-2);
 *   - optional pre-merge LayerNorm per patch (biased variance);
 *   - Linear -> exact-erf GELU -> Linear, weights stored (out, in)
 *     ("port DeepSeek-VL2", Projector step 3);
 *   - the row index of every merged token, newline and separator inside an
 *     image's assembled block for tile tag "2D"
 *     ("port DeepSeek-VL2", Tile-sequence assembly).
 */
#include <math.h>
#include <stdint.h>

/* Nearest bf16 value of x, ties to even. A value with 2^e <= |x| < 2^(e+1)
 * keeps 8 significant bits, so its bf16 spacing is 2^(e-7); below 2^-126 the
 * spacing stays 2^-133. */
double brute_round_bf16(double x)
{
    if (x == 0.0 || !isfinite(x)) return x;
    int e = ilogb(fabs(x));
    if (e < -126) e = -126;
    double ulp = ldexp(1.0, e - 7);
    double q = x / ulp;             /* exact: ulp is a power of two */
    double f = floor(q);
    double r = q - f;
    if (r > 0.5 || (r == 0.5 && fmod(f, 2.0) != 0.0)) f += 1.0;
    return f * ulp;
}

double brute_gelu(double x) { return 0.5 * x * (1.0 + erf(x / sqrt(2.0))); }

/* Merged A operand of token (i, j) of one view: a[c*k*k + dy*k + dx] is patch
 * (k*i+dy, k*j+dx), channel c, after the optional LayerNorm and bf16 rounding,
 * or 0 where that patch lies in the high-end pad. feat is (h*w, C) row-major. */
void brute_token_a(const double* feat, int h, int w, int C, int k, int i, int j,
                   int has_ln, const double* gamma, const double* beta, double eps,
                   int quantise, double* a)
{
    for (int dy = 0; dy < k; ++dy)
        for (int dx = 0; dx < k; ++dx) {
            int r = k * i + dy, s = k * j + dx;
            const double* x = feat + ((long)r * w + s) * C;
            double mu = 0.0, var = 0.0;
            if (r < h && s < w && has_ln) {
                for (int c = 0; c < C; ++c) mu += x[c];
                mu /= C;
                for (int c = 0; c < C; ++c) var += (x[c] - mu) * (x[c] - mu);
                var /= C;
            }
            for (int c = 0; c < C; ++c) {
                double v = 0.0;
                if (r < h && s < w) {
                    v = x[c];
                    if (has_ln) v = (v - mu) / sqrt(var + eps) * gamma[c] + beta[c];
                    if (quantise) v = brute_round_bf16(v);
                }
                a[c * k * k + dy * k + dx] = v;
            }
        }
}

/* Projected row of token (i, j): y[n] = b2[n] + sum_m W2[n][m] g[m],
 * g[m] = GELU(b1[m] + sum_q W1[m][q] a[q]) (rounded to bf16 when quantise). */
void brute_token_y(const double* feat, int h, int w, int C, int k, int i, int j,
                   int has_ln, const double* gamma, const double* beta, double eps,
                   const double* W1, const double* b1, int N1,
                   const double* W2, const double* b2, int N2,
                   int quantise, double* scratch_a, double* scratch_g, double* y)
{
    int K1 = k * k * C;
    brute_token_a(feat, h, w, C, k, i, j, has_ln, gamma, beta, eps, quantise, scratch_a);
    for (int m = 0; m < N1; ++m) {
        double acc = b1[m];
        for (int q = 0; q < K1; ++q) acc += W1[(long)m * K1 + q] * scratch_a[q];
        double g = brute_gelu(acc);
        scratch_g[m] = quantise ? brute_round_bf16(g) : g;
    }
    for (int n = 0; n < N2; ++n) {
        double acc = b2[n];
        for (int m = 0; m < N1; ++m) acc += W2[(long)n * N1 + m] * scratch_g[m];
        y[n] = acc;
    }
}

/* Row of merged token (i, j) of view v inside its image's assembled block.
 * tiled == 0: the view's own row-major order, i*w' + j.
 * tiled != 0 (global view first): the global view is v == 0 with one newline
 * closing each of its h' rows; one separator follows; local tile v-1 sits at
 * tile row ty = (v-1) / tw, tile column tx = (v-1) % tw of a (th*h') x (tw*w')
 * canvas whose rows also end in a newline. */
long brute_row_of_token(int tiled, int v, int i, int j, int hp, int wp, int tw)
{
    if (!tiled) return (long)i * wp + j;
    if (v == 0) return (long)i * (wp + 1) + j;
    long base = (long)hp * (wp + 1) + 1;
    int t = v - 1, ty = t / tw, tx = t % tw;
    long row = (long)ty * hp + i, col = (long)tx * wp + j;
    return base + row * ((long)tw * wp + 1) + col;
}

/* Row of the n-th newline of a tiled image (n < h' + th*h'). */
long brute_row_of_newline(int n, int hp, int wp, int tw)
{
    if (n < hp) return (long)n * (wp + 1) + wp;
    long base = (long)hp * (wp + 1) + 1;
    long r = n - hp;
    return base + r * ((long)tw * wp + 1) + (long)tw * wp;
}

/* Row of the view separator of a tiled image. */
long brute_row_of_separator(int hp, int wp) { return (long)hp * (wp + 1); }

/* One dense layer of a token: y[n] = b[n] + sum_q W[n][q] x[q] (W stored (out, in)),
 * then GELU when gelu != 0, then bf16 rounding when quantise != 0. */
void brute_dense(const double* x, int K, const double* W, const double* b, int N, int gelu, int quantise, double* y)
{
    for (int n = 0; n < N; ++n) {
        double acc = b[n];
        for (int q = 0; q < K; ++q) acc += W[(long)n * K + q] * x[q];
        if (gelu) acc = brute_gelu(acc);
        y[n] = quantise ? brute_round_bf16(acc) : acc;
    }
}

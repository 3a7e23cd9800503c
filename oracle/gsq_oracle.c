/*
 * gsq_oracle.c -- the oracle: a plain, slow CPU implementation of one GSQ
 * Gumbel-Softmax layer-reconstruction step, used only as test
 * infrastructure (parity reference and timed CPU baseline).  It shares no
 * code, header, table or constant generator with the CUDA library.
 *
 * What it computes (GSQ paper, arXiv 2604.18556; method as summarised on
 * agihunt.info, method and optimisation paragraphs, and atlas.scime.ai,
 * Approach):
 *   - each weight coordinate owns logits over the levels of a symmetric,
 *     zero-point-free, group-wise scalar grid with one scale per group of 128;
 *   - Gumbel noise is added, a tempered softmax gives a soft weighted sum of
 *     grid points (2-bit: 4 levels, 4 logits; ternary: a mask choice times a
 *     sign choice; 3 bits and up: 5 logits for shifts -2..+2 around the
 *     initial level);
 *   - the objective is the output reconstruction error on calibration data;
 *   - logits and scales are trained with Lion; annealing the temperature
 *     collapses the soft choice to a hard one (argmax), which is packed.
 * Where the pages leave a step open the plainest reading is taken; each such
 * reading is listed in the design notes.
 *
 * Precision: fp64 everywhere, except where floating point decides an integer
 * (round-to-nearest init level, sign inside Lion) or defines stored fp32
 * state: there the library's fp32 order is followed so both sides take the
 * same decision.
 *
 * Parity unpinned: the multi-step trajectory as a whole (the pages print no
 * worked example); its pieces are pinned individually by the CPU tests.
 */
#include "gsq_oracle.h"

#include <math.h>
#include <stdlib.h>
#include <string.h>

/* ------------------------------------------------------------------ grids */

int gsqo_num_logits(int mode) {
    switch (mode) {
    case GSQO_GRID_2BIT: return 4;
    case GSQO_GRID_TERNARY: return 4;      /* mask pair + sign pair */
    case GSQO_GRID_3BIT_LOCAL: return 5;   /* shifts -2..+2 */
    default: return -1;
    }
}

int gsqo_num_levels(int mode) {
    switch (mode) {
    case GSQO_GRID_2BIT: return 4;
    case GSQO_GRID_TERNARY: return 3;
    case GSQO_GRID_3BIT_LOCAL: return 8;
    default: return -1;
    }
}

/* Symmetric grids with no zero-point: 2-bit {-1.5,-0.5,0.5,1.5},
 * ternary {-1,0,1}, 3-bit {-3.5..3.5} in unit steps. */
double gsqo_level_value(int mode, int j) {
    switch (mode) {
    case GSQO_GRID_2BIT: return (double)j - 1.5;
    case GSQO_GRID_TERNARY: return (double)j - 1.0;
    case GSQO_GRID_3BIT_LOCAL: return (double)j - 3.5;
    default: return 0.0;
    }
}

static double grid_max(int mode) {
    return gsqo_level_value(mode, gsqo_num_levels(mode) - 1);
}

/* ----------------------------------------------------------------- Philox */

/* Philox4x32 (SC'11, section 4): two 32x32->64 multiplications per round,
 * the high halves xored with the other counter words and the round key,
 * the key bumped by the Weyl constants between rounds; 10 rounds. */
void gsqo_philox4x32_10(const uint32_t ctr[4], const uint32_t key[2],
                        uint32_t out[4]) {
    const uint64_t M0 = 0xD2511F53u, M1 = 0xCD9E8D57u;
    const uint32_t W0 = 0x9E3779B9u, W1 = 0xBB67AE85u;
    uint32_t c0 = ctr[0], c1 = ctr[1], c2 = ctr[2], c3 = ctr[3];
    uint32_t k0 = key[0], k1 = key[1];
    for (int r = 0; r < 10; ++r) {
        if (r > 0) {
            k0 += W0;
            k1 += W1;
        }
        uint64_t p0 = M0 * (uint64_t)c0;
        uint64_t p1 = M1 * (uint64_t)c2;
        uint32_t hi0 = (uint32_t)(p0 >> 32), lo0 = (uint32_t)p0;
        uint32_t hi1 = (uint32_t)(p1 >> 32), lo1 = (uint32_t)p1;
        uint32_t n0 = hi1 ^ c1 ^ k0;
        uint32_t n1 = lo1;
        uint32_t n2 = hi0 ^ c3 ^ k1;
        uint32_t n3 = lo0;
        c0 = n0; c1 = n1; c2 = n2; c3 = n3;
    }
    out[0] = c0; out[1] = c1; out[2] = c2; out[3] = c3;
}

/* The top 23 bits, centred in their cell: u = (m + 1/2) 2^-23 with
 * m = x >> 9.  m + 1/2 has at most 24 significant bits, so u is exact in
 * fp32 and lies in [2^-24, 1 - 2^-24], never 0 or 1. */
float gsqo_u01(uint32_t x) {
    double u = ((double)(x >> 9) + 0.5) * (1.0 / 8388608.0);
    return (float)u;
}

/* Counter layout: ctr = (low word, high word, step t, block), key = (seed
 * low word, seed high word).  Words used per coordinate:
 *   2-bit       block 0 of the coordinate, words 0..3  -> logits 0..3
 *   ternary     block 0 words 0,1   -> mask (zero, nonzero)
 *               block 0 words 2,3   -> sign (minus, plus)
 *   3-bit local block 0 words 0..3 -> shifts -2..+1, and for shift +2 word
 *               coord % 4 of block 1 of the aligned quad's first coordinate
 *               coord - coord % 4 (the quad's four coordinates take the four
 *               words of one block-1 draw). */
static void coord_words(int mode, uint64_t seed, uint32_t t, uint64_t coord,
                        uint32_t* w) {
    uint32_t key[2] = {(uint32_t)seed, (uint32_t)(seed >> 32)};
    uint32_t ctr[4] = {(uint32_t)coord, (uint32_t)(coord >> 32), t, 0u};
    gsqo_philox4x32_10(ctr, key, w);
    if (mode == GSQO_GRID_3BIT_LOCAL) {
        uint32_t out[4];
        uint64_t q = coord - coord % 4;
        uint32_t ctr1[4] = {(uint32_t)q, (uint32_t)(q >> 32), t, 1u};
        gsqo_philox4x32_10(ctr1, key, out);
        w[4] = out[coord % 4];
    }
}

static void coord_uniforms(int mode, uint64_t seed, uint32_t t, uint64_t coord,
                           float* u) {
    uint32_t w[5];
    coord_words(mode, seed, t, coord, w);
    for (int j = 0; j < gsqo_num_logits(mode); ++j) u[j] = gsqo_u01(w[j]);
}

void gsqo_uniforms(int mode, uint64_t seed, uint32_t t, uint64_t coord0,
                   int64_t count, float* out) {
    int L = gsqo_num_logits(mode);
    for (int64_t i = 0; i < count; ++i) {
        float u[5];
        coord_uniforms(mode, seed, t, coord0 + (uint64_t)i, u);
        for (int j = 0; j < L; ++j) out[i * L + j] = u[j];
    }
}

/* ---------------------------------------------------------------- rounding */

/* round x to a multiple of 2^(e-p) where 2^e <= |x| < 2^(e+1), e clamped
 * below at emin (subnormals), ties to even */
static double round_sig(double x, int p, int emin) {
    if (x == 0.0 || isnan(x) || isinf(x)) return x;
    int e = ilogb(x);
    if (e < emin) e = emin;
    double q = ldexp(1.0, e - p);
    return nearbyint(x / q) * q; /* x/q exact: power-of-two scaling */
}

double gsqo_bf16_round(double x) {
    double r = round_sig(x, 7, -126); /* 8 significant bits */
    if (fabs(r) > 3.3895313892515355e38) r = copysign(INFINITY, x);
    return r;
}

double gsqo_f16_round(double x) {
    double r = round_sig(x, 10, -14); /* 11 significant bits */
    if (fabs(r) > 65504.0) r = copysign(INFINITY, x);
    return r;
}

uint16_t gsqo_f16_bits(double x) {
    double r = gsqo_f16_round(x);
    uint16_t sign = signbit(r) ? 0x8000u : 0u;
    double a = fabs(r);
    if (isnan(r)) return 0x7E00u;
    if (isinf(a)) return (uint16_t)(sign | 0x7C00u);
    if (a == 0.0) return sign;
    int e = ilogb(a);
    if (e < -14) { /* subnormal: a = m * 2^-24 */
        return (uint16_t)(sign | (uint16_t)(a * 16777216.0));
    }
    uint16_t mant = (uint16_t)((ldexp(a, -e) - 1.0) * 1024.0);
    return (uint16_t)(sign | (uint16_t)((e + 15) << 10) | mant);
}

/* -------------------------------------------------------------------- init */

/* Round-to-nearest level of q = w/s under the grid, first index on ties.
 * Taken in fp32, the precision of the library's init kernel, because this
 * floating-point comparison decides an integer. */
static int rtn_level(int mode, float q) {
    int nl = gsqo_num_levels(mode);
    int best = 0;
    float bestd = fabsf(q - (float)gsqo_level_value(mode, 0));
    for (int j = 1; j < nl; ++j) {
        float d = fabsf(q - (float)gsqo_level_value(mode, j));
        if (d < bestd) {
            bestd = d;
            best = j;
        }
    }
    return best;
}

int gsqo_init(int mode, int64_t N, int64_t K, int group, const float* W,
              const int8_t* init_idx, float* s, int8_t* i0, float* logits,
              float* mom, float* ms) {
    int L = gsqo_num_logits(mode);
    if (L < 0 || group <= 0 || K % group != 0 || N <= 0 || K <= 0) return -1;
    int64_t G = K / group;
    int64_t NK = N * K;
    float cmax = (float)grid_max(mode);
    for (int64_t n = 0; n < N; ++n) {
        for (int64_t g = 0; g < G; ++g) {
            /* per-group scale: absmax / largest grid magnitude (fp32) */
            float amax = 0.0f;
            for (int64_t k = g * group; k < (g + 1) * group; ++k) {
                float a = fabsf(W[n * K + k]);
                if (a > amax) amax = a;
            }
            float sg = amax / cmax;
            s[n * G + g] = sg;
            ms[n * G + g] = 0.0f;
            for (int64_t k = g * group; k < (g + 1) * group; ++k) {
                int64_t c = n * K + k;
                float w = W[c];
                int lev;
                if (init_idx) {
                    lev = init_idx[c];
                } else {
                    float q = (sg > 0.0f) ? w / sg : 0.0f;
                    lev = rtn_level(mode, q);
                }
                i0[c] = (int8_t)lev;
                for (int p = 0; p < L; ++p) {
                    logits[p * NK + c] = 0.0f;
                    mom[p * NK + c] = 0.0f;
                }
                if (mode == GSQO_GRID_2BIT) {
                    logits[lev * NK + c] = 2.0f;
                } else if (mode == GSQO_GRID_3BIT_LOCAL) {
                    logits[2 * NK + c] = 2.0f; /* shift 0 */
                } else {
                    /* ternary: mask pair (zero, nonzero), sign pair (-, +) */
                    int nonzero = (lev != 1);
                    logits[(nonzero ? 1 : 0) * NK + c] = 2.0f;
                    int plus = (lev == 2) || (lev == 1 && !(w < 0.0f));
                    logits[(plus ? 3 : 2) * NK + c] = 2.0f;
                }
            }
        }
    }
    return 0;
}

void gsqo_reference_output(int64_t N, int64_t K, int64_t T, const float* W,
                           const float* X, double* Yref) {
    #pragma omp parallel for schedule(static)
    for (int64_t t = 0; t < T; ++t) {
        for (int64_t n = 0; n < N; ++n) {
            double acc = 0.0;
            for (int64_t k = 0; k < K; ++k)
                acc += gsqo_bf16_round(X[t * K + k]) * (double)W[n * K + k];
            Yref[t * N + n] = acc;
        }
    }
}

/* ------------------------------------------------------------ soft weight */

/* candidate unit values c'_k of each logit of a categorical mode */
static void candidates(int mode, int lev0, double* c) {
    if (mode == GSQO_GRID_2BIT) {
        for (int k = 0; k < 4; ++k) c[k] = gsqo_level_value(mode, k);
    } else { /* 3-bit local shift: level clamp(i0 + d, 0, 7), d = -2..2 */
        for (int k = 0; k < 5; ++k) {
            int j = lev0 + k - 2;
            if (j < 0) j = 0;
            if (j > 7) j = 7;
            c[k] = gsqo_level_value(mode, j);
        }
    }
}

static void softmax(const double* z, int n, double* y) {
    double zmax = z[0];
    for (int k = 1; k < n; ++k) if (z[k] > zmax) zmax = z[k];
    double sum = 0.0;
    for (int k = 0; k < n; ++k) {
        y[k] = exp(z[k] - zmax);
        sum += y[k];
    }
    for (int k = 0; k < n; ++k) y[k] /= sum;
}

/* Probabilities and unit value of one coordinate.  y holds L entries:
 * categorical: softmax over all logits; ternary: (p0, p1, q-, q+). */
static double coord_soft(int mode, const double* l, const double* g,
                         double tau, int lev0, double* y) {
    int L = gsqo_num_logits(mode);
    double z[5];
    for (int k = 0; k < L; ++k) z[k] = (l[k] + g[k]) / tau;
    if (mode == GSQO_GRID_TERNARY) {
        softmax(z, 2, y);         /* mask: zero, nonzero */
        softmax(z + 2, 2, y + 2); /* sign: minus, plus */
        return y[1] * (y[3] - y[2]);
    }
    softmax(z, L, y);
    double c[5];
    candidates(mode, lev0, c);
    double v = 0.0;
    for (int k = 0; k < L; ++k) v += y[k] * c[k];
    return v;
}

static void coord_noise(int mode, int noise_on, uint64_t seed, uint32_t t,
                        uint64_t coord, double* g) {
    int L = gsqo_num_logits(mode);
    if (!noise_on) {
        for (int k = 0; k < L; ++k) g[k] = 0.0;
        return;
    }
    float u[5];
    coord_uniforms(mode, seed, t, coord, u);
    for (int k = 0; k < L; ++k) g[k] = -log(-log((double)u[k])); /* Gumbel(0,1) */
}

void gsqo_soft_weight(int mode, int64_t row0, int64_t N, int64_t K, int group,
                      const float* logits, const float* s, const int8_t* i0,
                      uint64_t seed, uint32_t t, float tau, int noise_on,
                      double* y, double* v, double* w, float* w_bf16) {
    int L = gsqo_num_logits(mode);
    int64_t G = K / group, NK = N * K;
    #pragma omp parallel for schedule(static)
    for (int64_t n = 0; n < N; ++n) {
        for (int64_t k = 0; k < K; ++k) {
            int64_t c = n * K + k;
            double l[5], g[5], yy[5];
            for (int p = 0; p < L; ++p) l[p] = logits[p * NK + c];
            coord_noise(mode, noise_on, seed, t, (uint64_t)((row0 + n) * K + k), g);
            double vv = coord_soft(mode, l, g, (double)tau, i0 ? i0[c] : 0, yy);
            double ww = (double)s[n * G + k / group] * vv;
            if (y) for (int p = 0; p < L; ++p) y[p * NK + c] = yy[p];
            if (v) v[c] = vv;
            if (w) w[c] = ww;
            if (w_bf16) w_bf16[c] = (float)gsqo_bf16_round(ww);
        }
    }
}

/* ---------------------------------------------------------------- GEMMs */

void gsqo_gemm_abt(int64_t M, int64_t N, int64_t Kc, const float* A,
                   const float* B, double* C) {
    #pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < M; ++i)
        for (int64_t j = 0; j < N; ++j) {
            double acc = 0.0;
            for (int64_t k = 0; k < Kc; ++k)
                acc += (double)A[i * Kc + k] * (double)B[j * Kc + k];
            C[i * N + j] = acc;
        }
}

double gsqo_forward(int64_t N, int64_t K, int64_t T, const float* X,
                    const float* Wb, const double* Yref, float* dY) {
    /* per-token partial sums, then one sequential sum: deterministic */
    double* part = (double*)malloc((size_t)T * sizeof(double));
    #pragma omp parallel for schedule(static)
    for (int64_t t = 0; t < T; ++t) {
        double row = 0.0;
        for (int64_t n = 0; n < N; ++n) {
            double acc = 0.0;
            for (int64_t k = 0; k < K; ++k)
                acc += gsqo_bf16_round(X[t * K + k]) * (double)Wb[n * K + k];
            double e = acc - Yref[t * N + n];
            row += e * e;
            if (dY) dY[t * N + n] = (float)gsqo_bf16_round(2.0 * e);
        }
        part[t] = row;
    }
    double loss = 0.0;
    for (int64_t t = 0; t < T; ++t) loss += part[t];
    free(part);
    return loss;
}

void gsqo_weight_grad(int64_t N, int64_t K, int64_t T, const float* dY,
                      const float* X, float* dW) {
    #pragma omp parallel
    {
        double* acc = (double*)malloc((size_t)K * sizeof(double));
        #pragma omp for schedule(static)
        for (int64_t n = 0; n < N; ++n) {
            for (int64_t k = 0; k < K; ++k) acc[k] = 0.0;
            for (int64_t t = 0; t < T; ++t) {
                double d = dY[t * N + n];
                for (int64_t k = 0; k < K; ++k)
                    acc[k] += d * gsqo_bf16_round(X[t * K + k]);
            }
            for (int64_t k = 0; k < K; ++k) dW[n * K + k] = (float)acc[k];
        }
        free(acc);
    }
}

/* ------------------------------------------------------------- gradients */

/* A5 gradients.  With a = s_g * dw / tau (d loss / d v = s_g * dw and
 * d z / d l = 1 / tau):
 *   categorical  dl_k = a * y_k * sum_j y_j (c_k - c_j)   (= a y_k (c_k - v))
 *   ternary      v = p1 (q+ - q-):  dl_mask1 = a (q+ - q-) p1 p0 = -dl_mask0,
 *                dl_sign+ = a * 2 p1 q+ q- = -dl_sign-
 *   scale        ds_g = sum over the group of dw * v                      */
void gsqo_backward(int mode, int64_t N, int64_t K, int group, const double* y,
                   const double* v, const float* s, const int8_t* i0,
                   const float* dW, float tau, float* dl, float* ds) {
    int L = gsqo_num_logits(mode);
    int64_t G = K / group, NK = N * K;
    #pragma omp parallel for schedule(static)
    for (int64_t n = 0; n < N; ++n) {
        for (int64_t g = 0; g < G; ++g) {
            double sg = s[n * G + g];
            double dsg = 0.0;
            for (int64_t k = g * group; k < (g + 1) * group; ++k) {
                int64_t c = n * K + k;
                double dw = dW[c];
                double a = sg * dw / (double)tau;
                double yy[5];
                for (int p = 0; p < L; ++p) yy[p] = y[p * NK + c];
                if (mode == GSQO_GRID_TERNARY) {
                    double p0 = yy[0], p1 = yy[1], qm = yy[2], qp = yy[3];
                    double gm = a * (qp - qm) * p1 * p0; /* d v / d z_mask1 */
                    double gs = a * 2.0 * p1 * qp * qm;  /* d v / d z_sign+ */
                    dl[0 * NK + c] = (float)(-gm);
                    dl[1 * NK + c] = (float)gm;
                    dl[2 * NK + c] = (float)(-gs);
                    dl[3 * NK + c] = (float)gs;
                } else {
                    double cand[5];
                    candidates(mode, i0 ? i0[c] : 0, cand);
                    for (int p = 0; p < L; ++p) {
                        double acc = 0.0;
                        for (int j = 0; j < L; ++j) acc += yy[j] * (cand[p] - cand[j]);
                        dl[p * NK + c] = (float)(a * yy[p] * acc);
                    }
                }
                dsg += dw * v[c]; /* d loss / d s = sum dw * v */
            }
            ds[n * G + g] = (float)dsg;
        }
    }
}

/* ------------------------------------------------------------------ Lion */

/* Lion: c = b1*m + (1-b1)*g; theta -= lr*sign(c); m = b2*m + (1-b2)*g.
 * fp32 state; the two blends as single fused multiply-adds, (1-b) in fp32. */
void gsqo_lion(int64_t n, float* theta, float* mom, const float* grad,
               float lr, float beta1, float beta2) {
    float omb1 = 1.0f - beta1, omb2 = 1.0f - beta2;
    for (int64_t i = 0; i < n; ++i) {
        float g = grad[i];
        float m = mom[i];
        float c = fmaf(beta1, m, omb1 * g);
        float sg = (c > 0.0f) ? 1.0f : ((c < 0.0f) ? -1.0f : 0.0f);
        theta[i] = theta[i] - lr * sg;
        mom[i] = fmaf(beta2, m, omb2 * g);
    }
}

/* ------------------------------------------------------------------ step */

int gsqo_backward_lion(int mode, int64_t row0, int64_t N, int64_t K, int group,
                       float* logits, float* mom, float* s, float* ms,
                       const int8_t* i0, const float* dW, uint64_t seed,
                       uint32_t t, float tau, float lr, float beta1,
                       float beta2, int noise_on, float* dl_dump,
                       float* ds_dump) {
    int L = gsqo_num_logits(mode);
    if (L < 0 || K % group != 0) return -1;
    int64_t NK = N * K, G = K / group;
    double* y = (double*)malloc((size_t)(L * NK) * sizeof(double));
    double* v = (double*)malloc((size_t)NK * sizeof(double));
    float* dl = (float*)malloc((size_t)(L * NK) * sizeof(float));
    float* ds = (float*)malloc((size_t)(N * G) * sizeof(float));
    if (!y || !v || !dl || !ds) {
        free(y); free(v); free(dl); free(ds);
        return -3;
    }
    /* same noise (step t) and pre-update parameters as the forward pass */
    gsqo_soft_weight(mode, row0, N, K, group, logits, s, i0, seed, t, tau,
                     noise_on, y, v, NULL, NULL);
    gsqo_backward(mode, N, K, group, y, v, s, i0, dW, tau, dl, ds);
    if (dl_dump) memcpy(dl_dump, dl, (size_t)(L * NK) * sizeof(float));
    if (ds_dump) memcpy(ds_dump, ds, (size_t)(N * G) * sizeof(float));
    gsqo_lion(L * NK, logits, mom, dl, lr, beta1, beta2);
    gsqo_lion(N * G, s, ms, ds, lr, beta1, beta2);
    free(y); free(v); free(dl); free(ds);
    return 0;
}

int gsqo_step(int mode, int64_t row0, int64_t N, int64_t K, int64_t T,
              int group, float* logits, float* mom, float* s, float* ms,
              const int8_t* i0, const float* X, const double* Yref,
              uint64_t seed, uint32_t t, float tau, float lr, float beta1,
              float beta2, int noise_on, double* loss, double* w_dump,
              float* dY_dump, float* dW_dump, float* dl_dump, float* ds_dump) {
    int L = gsqo_num_logits(mode);
    if (L < 0 || K % group != 0 || !(tau > 0.0f)) return -1;
    int64_t NK = N * K;
    double* w = (double*)malloc((size_t)NK * sizeof(double));
    float* wb = (float*)malloc((size_t)NK * sizeof(float));
    float* dY = (float*)malloc((size_t)(T * N) * sizeof(float));
    float* dW = (float*)malloc((size_t)NK * sizeof(float));
    if (!w || !wb || !dY || !dW) {
        free(w); free(wb); free(dY); free(dW);
        return -3;
    }
    /* A1+A2: soft weight with this step's noise */
    gsqo_soft_weight(mode, row0, N, K, group, logits, s, i0, seed, t, tau,
                     noise_on, NULL, NULL, w, wb);
    /* A3: reconstruction loss and its output gradient */
    double l = gsqo_forward(N, K, T, X, wb, Yref, dY);
    /* A4: weight gradient */
    gsqo_weight_grad(N, K, T, dY, X, dW);
    /* A5: logits and scale gradients, then Lion */
    int rc = gsqo_backward_lion(mode, row0, N, K, group, logits, mom, s, ms, i0,
                                dW, seed, t, tau, lr, beta1, beta2, noise_on,
                                dl_dump, ds_dump);
    if (loss) *loss = l;
    if (w_dump) memcpy(w_dump, w, (size_t)NK * sizeof(double));
    if (dY_dump) memcpy(dY_dump, dY, (size_t)(T * N) * sizeof(float));
    if (dW_dump) memcpy(dW_dump, dW, (size_t)NK * sizeof(float));
    free(w); free(wb); free(dY); free(dW);
    return rc;
}

/* --------------------------------------------- bf16 logit / momentum state */

/* Stochastic rounding of an fp32 value to bf16 with a 9-bit threshold r:
 * r << 7 is added to the fp32 bit pattern and the low 16 bits are dropped,
 * so the magnitude rounds up with probability (low 16 bits) / 2^16, to 2^-9
 * of a bf16 unit.  Exactly representable values are returned unchanged. */
float gsqo_bf16_sr(float x, uint32_t r9) {
    uint32_t b;
    memcpy(&b, &x, sizeof(b));
    b += (r9 & 0x1FFu) << 7;
    b &= 0xFFFF0000u;
    float y;
    memcpy(&y, &b, sizeof(y));
    return y;
}

/* After the fp32 Lion update of step t: logits to bf16 by stochastic
 * rounding, the threshold of logit p of a coordinate being the low 9 bits of
 * the Philox word that gives that coordinate and logit its noise at step
 * t + 1 (the words of coord_uniforms); momenta to the nearest bf16 (ties to
 * even).  Rows row0.. of the layer (global coordinate (row0 + n) K + k). */
void gsqo_state16_store(int mode, int64_t row0, int64_t N, int64_t K,
                        uint64_t seed, uint32_t t_next, float* logits,
                        float* mom) {
    const int L = gsqo_num_logits(mode);
    const int64_t NK = N * K;
    for (int64_t i = 0; i < NK; ++i) {
        const uint64_t coord = (uint64_t)(row0 * K + i);
        uint32_t w[5];
        coord_words(mode, seed, t_next, coord, w);
        for (int p = 0; p < L; ++p) {
            logits[p * NK + i] = gsqo_bf16_sr(logits[p * NK + i], w[p]);
            mom[p * NK + i] = (float)gsqo_bf16_round((double)mom[p * NK + i]);
        }
    }
}

/* ---------------------------------------------------------- harden, pack */

static int argmax_first(const float* l, int n) {
    int best = 0;
    for (int k = 1; k < n; ++k)
        if (l[k] > l[best]) best = k;
    return best;
}

void gsqo_harden(int mode, int64_t N, int64_t K, const float* logits,
                 const int8_t* i0, uint8_t* level) {
    int L = gsqo_num_logits(mode);
    int64_t NK = N * K;
    for (int64_t c = 0; c < NK; ++c) {
        float l[5];
        for (int p = 0; p < L; ++p) l[p] = logits[p * NK + c];
        int lev;
        if (mode == GSQO_GRID_2BIT) {
            lev = argmax_first(l, 4);
        } else if (mode == GSQO_GRID_3BIT_LOCAL) {
            lev = i0[c] + argmax_first(l, 5) - 2;
            if (lev < 0) lev = 0;
            if (lev > 7) lev = 7;
        } else {
            int nonzero = argmax_first(l, 2);      /* 0: zero, 1: nonzero */
            int plus = argmax_first(l + 2, 2);     /* 0: minus, 1: plus */
            lev = nonzero ? (plus ? 2 : 0) : 1;    /* level index of {-1,0,1} */
        }
        level[c] = (uint8_t)lev;
    }
}

static int code_bits(int mode) { return mode == GSQO_GRID_3BIT_LOCAL ? 3 : 2; }

int64_t gsqo_packed_words_per_row(int mode, int64_t K) {
    return (K * code_bits(mode) + 31) / 32;
}

/* LSB-first bitstream per row: code j of a row occupies bits
 * [j*b, j*b + b) of the row's little-endian stream of 32-bit words. */
void gsqo_pack(int mode, int64_t N, int64_t K, const uint8_t* level,
               uint32_t* packed) {
    int b = code_bits(mode);
    int64_t wpr = gsqo_packed_words_per_row(mode, K);
    memset(packed, 0, (size_t)(N * wpr) * sizeof(uint32_t));
    for (int64_t n = 0; n < N; ++n)
        for (int64_t k = 0; k < K; ++k)
            for (int i = 0; i < b; ++i) {
                int64_t bit = k * b + i;
                if ((level[n * K + k] >> i) & 1u)
                    packed[n * wpr + bit / 32] |= (1u << (bit % 32));
            }
}

void gsqo_unpack(int mode, int64_t N, int64_t K, const uint32_t* packed,
                 uint8_t* level) {
    int b = code_bits(mode);
    int64_t wpr = gsqo_packed_words_per_row(mode, K);
    for (int64_t n = 0; n < N; ++n)
        for (int64_t k = 0; k < K; ++k) {
            unsigned v = 0;
            for (int i = 0; i < b; ++i) {
                int64_t bit = k * b + i;
                v |= ((packed[n * wpr + bit / 32] >> (bit % 32)) & 1u) << i;
            }
            level[n * K + k] = (uint8_t)v;
        }
}

/* ----------------------------------------------------- scale-only step */

/* Scale-only training (agihunt.info summary, optimisation paragraph: the
 * 2-bit models get one more round that changes only the group scales),
 * restated for the layer objective: the assignments stay at the hard choice
 * of the current logits (gsqo_harden), the weight is w = bf16(s_g c_level),
 * and only s moves:
 *   ds_g = sum over the group of dW_i c_level(i)   (fp64 sum, in k order)
 * followed by Lion on s with its momentum ms.  Given dW. */
void gsqo_scale_backward_lion(int mode, int64_t N, int64_t K, int group,
                              const float* logits, const int8_t* i0, float* s,
                              float* ms, const float* dW, float lr, float beta1,
                              float beta2, float* ds_dump) {
    int64_t NK = N * K, G = K / group;
    uint8_t* lev = (uint8_t*)malloc((size_t)NK);
    float* ds = (float*)malloc((size_t)(N * G) * sizeof(float));
    gsqo_harden(mode, N, K, logits, i0, lev);
    for (int64_t n = 0; n < N; ++n)
        for (int64_t g = 0; g < G; ++g) {
            double acc = 0.0;
            for (int64_t k = g * group; k < (g + 1) * group; ++k)
                acc += (double)dW[n * K + k] * gsqo_level_value(mode, lev[n * K + k]);
            ds[n * G + g] = (float)acc;
        }
    if (ds_dump) memcpy(ds_dump, ds, (size_t)(N * G) * sizeof(float));
    gsqo_lion(N * G, s, ms, ds, lr, beta1, beta2);
    free(lev);
    free(ds);
}

/* One scale-only step: hard weight, loss and output gradient (gsqo_forward),
 * weight gradient (gsqo_weight_grad), then gsqo_scale_backward_lion. */
int gsqo_scale_step(int mode, int64_t N, int64_t K, int64_t T, int group,
                    const float* logits, const int8_t* i0, float* s, float* ms,
                    const float* X, const double* Yref, float lr, float beta1,
                    float beta2, double* loss, float* w_dump, float* dW_dump,
                    float* ds_dump) {
    if (gsqo_num_logits(mode) < 0 || K % group != 0) return -1;
    int64_t NK = N * K, G = K / group;
    uint8_t* lev = (uint8_t*)malloc((size_t)NK);
    float* wq = (float*)malloc((size_t)NK * sizeof(float));
    float* dY = (float*)malloc((size_t)(T * N) * sizeof(float));
    float* dW = (float*)malloc((size_t)NK * sizeof(float));
    if (!lev || !wq || !dY || !dW) {
        free(lev); free(wq); free(dY); free(dW);
        return -3;
    }
    gsqo_harden(mode, N, K, logits, i0, lev);
    for (int64_t c = 0; c < NK; ++c) {
        int64_t n = c / K, k = c % K;
        double w = (double)s[n * G + k / group] * gsqo_level_value(mode, lev[c]);
        wq[c] = (float)gsqo_bf16_round(w);
    }
    double l = gsqo_forward(N, K, T, X, wq, Yref, dY);
    gsqo_weight_grad(N, K, T, dY, X, dW);
    gsqo_scale_backward_lion(mode, N, K, group, logits, i0, s, ms, dW, lr, beta1,
                             beta2, ds_dump);
    if (loss) *loss = l;
    if (w_dump) memcpy(w_dump, wq, (size_t)NK * sizeof(float));
    if (dW_dump) memcpy(dW_dump, dW, (size_t)NK * sizeof(float));
    free(lev); free(wq); free(dY); free(dW);
    return 0;
}

/* ------------------------------------------------------------ recon error */

void gsqo_recon_error(int gmode, int emode, int64_t N, int64_t K, int64_t T,
                      int group, const float* logits, const float* s,
                      const int8_t* i0, const float* X, const double* Yref,
                      float tau, double* abs_err, double* rel_err) {
    int64_t NK = N * K, G = K / group;
    float* wq = (float*)malloc((size_t)NK * sizeof(float));
    if (emode == 0) {
        uint8_t* lev = (uint8_t*)malloc((size_t)NK);
        gsqo_harden(gmode, N, K, logits, i0, lev);
        for (int64_t c = 0; c < NK; ++c) {
            int64_t n = c / K, k = c % K;
            double w = (double)s[n * G + k / group] * gsqo_level_value(gmode, lev[c]);
            wq[c] = (float)gsqo_bf16_round(w);
        }
        free(lev);
    } else {
        gsqo_soft_weight(gmode, 0, N, K, group, logits, s, i0, 0, 0, tau, 0,
                         NULL, NULL, NULL, wq);
    }
    double e2 = gsqo_forward(N, K, T, X, wq, Yref, NULL);
    double y2 = 0.0;
    for (int64_t i = 0; i < T * N; ++i) y2 += Yref[i] * Yref[i];
    *abs_err = e2;
    *rel_err = (y2 > 0.0) ? e2 / y2 : 0.0;
    free(wq);
}

/* --------------------------------------------------- SwiGLU MLP stage */

static double sigmoid(double x) { return 1.0 / (1.0 + exp(-x)); }

/* The block's MLP stage (agihunt.info summary, optimisation paragraph: the
 * MLP is trained on the block output after the attention stages): one
 * forward and backward pass of the SwiGLU MLP against the fixed target R. */
double gsqo_mlp_forward_backward(int64_t T, int64_t H, int64_t F,
                                 const float* Xn, const double* R,
                                 const float* Wg, const float* Wu,
                                 const float* Wd, int round, float* dWg,
                                 float* dWu, float* dWd) {
    double* a = (double*)malloc((size_t)(T * F) * sizeof(double));
    double* b = (double*)malloc((size_t)(T * F) * sizeof(double));
    double* h = (double*)malloc((size_t)(T * F) * sizeof(double));
    double* dp = (double*)malloc((size_t)(T * H) * sizeof(double));
    double* da = (double*)malloc((size_t)(T * F) * sizeof(double));
    double* db = (double*)malloc((size_t)(T * F) * sizeof(double));
    double* part = (double*)malloc((size_t)T * sizeof(double));
    /* a, b, h */
    #pragma omp parallel for schedule(static)
    for (int64_t t = 0; t < T; ++t)
        for (int64_t f = 0; f < F; ++f) {
            double sa = 0.0, sb = 0.0;
            for (int64_t k = 0; k < H; ++k) {
                double x = round ? gsqo_bf16_round(Xn[t * H + k]) : (double)Xn[t * H + k];
                sa += x * Wg[f * H + k];
                sb += x * Wu[f * H + k];
            }
            a[t * F + f] = sa;
            b[t * F + f] = sb;
            double hv = sa * sigmoid(sa) * sb; /* silu(a) * b */
            h[t * F + f] = round ? gsqo_bf16_round(hv) : hv;
        }
    /* pred, E, loss, dpred = 2E */
    #pragma omp parallel for schedule(static)
    for (int64_t t = 0; t < T; ++t) {
        double row = 0.0;
        for (int64_t n = 0; n < H; ++n) {
            double acc = 0.0;
            for (int64_t f = 0; f < F; ++f) acc += h[t * F + f] * Wd[n * F + f];
            double e = acc - R[t * H + n];
            row += e * e;
            dp[t * H + n] = round ? gsqo_bf16_round(2.0 * e) : 2.0 * e;
        }
        part[t] = row;
    }
    double loss = 0.0;
    for (int64_t t = 0; t < T; ++t) loss += part[t];
    /* dh = dpred Wd; da = dh b silu'(a); db = dh silu(a) */
    #pragma omp parallel for schedule(static)
    for (int64_t t = 0; t < T; ++t)
        for (int64_t f = 0; f < F; ++f) {
            double dh = 0.0;
            for (int64_t n = 0; n < H; ++n) dh += dp[t * H + n] * Wd[n * F + f];
            double av = a[t * F + f], sg = sigmoid(av);
            double dsilu = sg * (1.0 + av * (1.0 - sg));
            double gav = dh * b[t * F + f] * dsilu;
            double gbv = dh * av * sg;
            da[t * F + f] = round ? gsqo_bf16_round(gav) : gav;
            db[t * F + f] = round ? gsqo_bf16_round(gbv) : gbv;
        }
    /* weight gradients */
    if (dWd) {
        #pragma omp parallel for schedule(static)
        for (int64_t n = 0; n < H; ++n)
            for (int64_t f = 0; f < F; ++f) {
                double acc = 0.0;
                for (int64_t t = 0; t < T; ++t) acc += dp[t * H + n] * h[t * F + f];
                dWd[n * F + f] = (float)acc;
            }
    }
    if (dWg || dWu) {
        #pragma omp parallel for schedule(static)
        for (int64_t f = 0; f < F; ++f)
            for (int64_t k = 0; k < H; ++k) {
                double ag = 0.0, au = 0.0;
                for (int64_t t = 0; t < T; ++t) {
                    double x = round ? gsqo_bf16_round(Xn[t * H + k]) : (double)Xn[t * H + k];
                    ag += da[t * F + f] * x;
                    au += db[t * F + f] * x;
                }
                if (dWg) dWg[f * H + k] = (float)ag;
                if (dWu) dWu[f * H + k] = (float)au;
            }
    }
    free(a); free(b); free(h); free(dp); free(da); free(db); free(part);
    return loss;
}

/* ------------------------------------------- attention V/O joint stage */

/* The block's value/output stage (agihunt.info summary, optimisation
 * paragraph: Q and K first, then V and O jointly): the attention
 * probabilities come from the frozen query/key weights and stay fixed. */
void gsqo_attn_probs(int64_t nseq, int64_t S, int64_t nh, int64_t nkv,
                     int64_t d, double theta, const float* Xa, const float* Wq,
                     const float* Wk, int round, float* P) {
    const int64_t H = nh * d, Hk = nkv * d, T = nseq * S, half = d / 2;
    const int64_t grp = nh / nkv;
    double* Q = (double*)malloc((size_t)(T * H) * sizeof(double));
    double* K = (double*)malloc((size_t)(T * Hk) * sizeof(double));
    /* projections */
    #pragma omp parallel for schedule(static)
    for (int64_t t = 0; t < T; ++t) {
        for (int64_t j = 0; j < H; ++j) {
            double acc = 0.0;
            for (int64_t k = 0; k < H; ++k)
                acc += (round ? gsqo_bf16_round(Xa[t * H + k]) : (double)Xa[t * H + k]) * Wq[j * H + k];
            Q[t * H + j] = acc;
        }
        for (int64_t j = 0; j < Hk; ++j) {
            double acc = 0.0;
            for (int64_t k = 0; k < H; ++k)
                acc += (round ? gsqo_bf16_round(Xa[t * H + k]) : (double)Xa[t * H + k]) * Wk[j * H + k];
            K[t * Hk + j] = acc;
        }
    }
    /* rotary embedding at the position within the sequence */
    #pragma omp parallel for schedule(static)
    for (int64_t t = 0; t < T; ++t) {
        const double p = (double)(t % S);
        for (int64_t i = 0; i < half; ++i) {
            const double ang = p * pow(theta, -2.0 * (double)i / (double)d);
            const double cs = cos(ang), sn = sin(ang);
            for (int64_t h = 0; h < nh; ++h) {
                double* x = Q + t * H + h * d;
                const double a = x[i], b = x[i + half];
                x[i] = a * cs - b * sn;
                x[i + half] = b * cs + a * sn;
            }
            for (int64_t g = 0; g < nkv; ++g) {
                double* x = K + t * Hk + g * d;
                const double a = x[i], b = x[i + half];
                x[i] = a * cs - b * sn;
                x[i + half] = b * cs + a * sn;
            }
        }
        if (round) {
            for (int64_t j = 0; j < H; ++j) Q[t * H + j] = gsqo_bf16_round(Q[t * H + j]);
            for (int64_t j = 0; j < Hk; ++j) K[t * Hk + j] = gsqo_bf16_round(K[t * Hk + j]);
        }
    }
    /* causal softmax of the scaled scores */
    const double scale = 1.0 / sqrt((double)d);
    #pragma omp parallel for collapse(2) schedule(static)
    for (int64_t s = 0; s < nseq; ++s)
        for (int64_t h = 0; h < nh; ++h) {
            const int64_t g = h / grp;
            double* row = (double*)malloc((size_t)S * sizeof(double));
            for (int64_t q = 0; q < S; ++q) {
                const double* qv = Q + (s * S + q) * H + h * d;
                double mx = -INFINITY;
                for (int64_t k = 0; k <= q; ++k) {
                    const double* kv = K + (s * S + k) * Hk + g * d;
                    double acc = 0.0;
                    for (int64_t j = 0; j < d; ++j) acc += qv[j] * kv[j];
                    row[k] = acc * scale;
                    if (row[k] > mx) mx = row[k];
                }
                double sum = 0.0;
                for (int64_t k = 0; k <= q; ++k) {
                    row[k] = exp(row[k] - mx);
                    sum += row[k];
                }
                float* out = P + ((s * nh + h) * S + q) * S;
                for (int64_t k = 0; k < S; ++k) {
                    const double pv = k <= q ? row[k] / sum : 0.0;
                    out[k] = (float)(round ? gsqo_bf16_round(pv) : pv);
                }
            }
            free(row);
        }
    free(Q);
    free(K);
}

double gsqo_attn_vo_forward_backward(int64_t nseq, int64_t S, int64_t nh,
                                     int64_t nkv, int64_t d, const float* Xa,
                                     const float* P, const double* R,
                                     const float* Wv, const float* Wo,
                                     int round, float* dWv, float* dWo) {
    const int64_t H = nh * d, Hk = nkv * d, T = nseq * S, grp = nh / nkv;
#define RB(x) (round ? gsqo_bf16_round(x) : (x))
    double* V = (double*)malloc((size_t)(T * Hk) * sizeof(double));
    double* o = (double*)malloc((size_t)(T * H) * sizeof(double));
    double* dp = (double*)malloc((size_t)(T * H) * sizeof(double));
    double* dO = (double*)malloc((size_t)(T * H) * sizeof(double));
    double* dV = (double*)malloc((size_t)(T * Hk) * sizeof(double));
    double* part = (double*)malloc((size_t)T * sizeof(double));
    /* V = Xa Wv^T */
    #pragma omp parallel for schedule(static)
    for (int64_t t = 0; t < T; ++t)
        for (int64_t j = 0; j < Hk; ++j) {
            double acc = 0.0;
            for (int64_t k = 0; k < H; ++k) acc += RB((double)Xa[t * H + k]) * Wv[j * H + k];
            V[t * Hk + j] = RB(acc);
        }
    /* o_(s,h) = P_(s,h) V_(s,g) */
    #pragma omp parallel for collapse(2) schedule(static)
    for (int64_t s = 0; s < nseq; ++s)
        for (int64_t h = 0; h < nh; ++h) {
            const int64_t g = h / grp;
            for (int64_t q = 0; q < S; ++q)
                for (int64_t j = 0; j < d; ++j) {
                    double acc = 0.0;
                    for (int64_t k = 0; k < S; ++k)
                        acc += (double)P[((s * nh + h) * S + q) * S + k] * V[(s * S + k) * Hk + g * d + j];
                    o[(s * S + q) * H + h * d + j] = RB(acc);
                }
        }
    /* pred = o Wo^T, loss, dp = 2E */
    #pragma omp parallel for schedule(static)
    for (int64_t t = 0; t < T; ++t) {
        double row = 0.0;
        for (int64_t n = 0; n < H; ++n) {
            double acc = 0.0;
            for (int64_t k = 0; k < H; ++k) acc += o[t * H + k] * Wo[n * H + k];
            const double e = acc - R[t * H + n];
            row += e * e;
            dp[t * H + n] = RB(2.0 * e);
        }
        part[t] = row;
    }
    double loss = 0.0;
    for (int64_t t = 0; t < T; ++t) loss += part[t];
    /* dWo = dp^T o; do = dp Wo */
    if (dWo) {
        #pragma omp parallel for schedule(static)
        for (int64_t n = 0; n < H; ++n)
            for (int64_t k = 0; k < H; ++k) {
                double acc = 0.0;
                for (int64_t t = 0; t < T; ++t) acc += dp[t * H + n] * o[t * H + k];
                dWo[n * H + k] = (float)acc;
            }
    }
    #pragma omp parallel for schedule(static)
    for (int64_t t = 0; t < T; ++t)
        for (int64_t k = 0; k < H; ++k) {
            double acc = 0.0;
            for (int64_t n = 0; n < H; ++n) acc += dp[t * H + n] * Wo[n * H + k];
            dO[t * H + k] = RB(acc);
        }
    /* dV_(s,g) = sum over the group's heads of P_(s,h)^T do_(s,h) */
    #pragma omp parallel for collapse(2) schedule(static)
    for (int64_t s = 0; s < nseq; ++s)
        for (int64_t g = 0; g < nkv; ++g)
            for (int64_t k = 0; k < S; ++k)
                for (int64_t j = 0; j < d; ++j) {
                    double acc = 0.0;
                    for (int64_t h = g * grp; h < (g + 1) * grp; ++h)
                        for (int64_t q = 0; q < S; ++q)
                            acc += (double)P[((s * nh + h) * S + q) * S + k] * dO[(s * S + q) * H + h * d + j];
                    dV[(s * S + k) * Hk + g * d + j] = RB(acc);
                }
    /* dWv = dV^T Xa */
    if (dWv) {
        #pragma omp parallel for schedule(static)
        for (int64_t j = 0; j < Hk; ++j)
            for (int64_t k = 0; k < H; ++k) {
                double acc = 0.0;
                for (int64_t t = 0; t < T; ++t) acc += dV[t * Hk + j] * RB((double)Xa[t * H + k]);
                dWv[j * H + k] = (float)acc;
            }
    }
#undef RB
    free(V); free(o); free(dp); free(dO); free(dV); free(part);
    return loss;
}

/* One query row of the attention probabilities, for sampled checks. */
static void rotated_projection(const float* Xa, const float* W, int64_t H,
                               int64_t t, int64_t S, int64_t col0, int64_t d,
                               double theta, int round, double* out) {
    const int64_t half = d / 2;
    for (int64_t j = 0; j < d; ++j) {
        double acc = 0.0;
        for (int64_t k = 0; k < H; ++k)
            acc += (round ? gsqo_bf16_round(Xa[t * H + k]) : (double)Xa[t * H + k]) *
                   W[(col0 + j) * H + k];
        out[j] = acc;
    }
    const double p = (double)(t % S);
    for (int64_t i = 0; i < half; ++i) {
        const double ang = p * pow(theta, -2.0 * (double)i / (double)d);
        const double cs = cos(ang), sn = sin(ang);
        const double a = out[i], b = out[i + half];
        out[i] = a * cs - b * sn;
        out[i + half] = b * cs + a * sn;
    }
    if (round)
        for (int64_t j = 0; j < d; ++j) out[j] = gsqo_bf16_round(out[j]);
}

void gsqo_attn_prob_row(int64_t nseq, int64_t S, int64_t nh, int64_t nkv,
                        int64_t d, double theta, const float* Xa,
                        const float* Wq, const float* Wk, int round, int64_t s,
                        int64_t h, int64_t q, float* row) {
    (void)nseq;
    const int64_t H = nh * d, g = h / (nh / nkv);
    double* qv = (double*)malloc((size_t)d * sizeof(double));
    double* sc = (double*)malloc((size_t)S * sizeof(double));
    rotated_projection(Xa, Wq, H, s * S + q, S, h * d, d, theta, round, qv);
    const double scale = 1.0 / sqrt((double)d);
    #pragma omp parallel for schedule(static)
    for (int64_t k = 0; k <= q; ++k) {
        double kv[256];
        rotated_projection(Xa, Wk, H, s * S + k, S, g * d, d, theta, round, kv);
        double acc = 0.0;
        for (int64_t j = 0; j < d; ++j) acc += qv[j] * kv[j];
        sc[k] = acc * scale;
    }
    double mx = -INFINITY, sum = 0.0;
    for (int64_t k = 0; k <= q; ++k) if (sc[k] > mx) mx = sc[k];
    for (int64_t k = 0; k <= q; ++k) { sc[k] = exp(sc[k] - mx); sum += sc[k]; }
    for (int64_t k = 0; k < S; ++k) {
        const double pv = k <= q ? sc[k] / sum : 0.0;
        row[k] = (float)(round ? gsqo_bf16_round(pv) : pv);
    }
    free(qv);
    free(sc);
}

/*
 * mh3a_oracle.c -- plain, slow fp64 CPU oracle of the MiniMax-H3 audio-VAE BigVGAN decode.
 *
 * TEST INFRASTRUCTURE ONLY (see mh3a_oracle.h).  Written from the pages' description of the
 * method, one definition per function, with no blocking, fusion or reordering beyond what
 * each definition states.  Every step is pinned by tests/test_oracle_*.py against closed
 * forms, brute-force definitions and independent library routines.
 *
 * Readings taken where the pages are silent (each also listed in the design notes):
 *  R1  AMP residual block body: for each dilation d, x <- x + conv_k,1(act(conv_k,d(act(x)))),
 *      two weight-normed convs per dilation, "same" padding d(k-1)/2.  Source: [P3] module
 *      summary, bullet "Decoder" ("AMP residual blocks with SnakeBeta behind alias-free
 *      Kaiser-window up/down sampling") -- the block body itself is not printed.
 *  R2  Anti-aliased activation: ratio 2, K = 12 taps, cutoff 0.5/2, half-width 0.6/2, one
 *      filter shared by the upsampler and the decimator.  Upsampler: replicate-pad K/2-1
 *      samples each side, stride-2 transposed conv with the taps, gain 2, crop
 *      (K/2-1)*2 + (K-2)/2 samples from the left and (K/2-1)*2 + (K-1)/2 from the right.
 *      Decimator: replicate-pad K/2-1 left and K/2 right, stride-2 conv with the taps.
 *  R3  SnakeBeta with linear-scale parameters: y = x + sin^2(alpha x) / (beta + 1e-9).
 *  R4  Weight norm over every axis but the first of the stored tensor (conv [O,I,K]: per
 *      output channel; transposed conv [I,O,K]: per input channel).
 *  R5  conv_pre and conv_post kernel size 7 (padding 3 preserves length only for k = 7).
 */
#include "mh3a_oracle.h"

#include <math.h>
#include <omp.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#ifndef M_PI
#define M_PI 3.14159265358979323846
#endif

/* ------------------------------------------------------------------------------------------ */
/* Kaiser-sinc low-pass: [P3] `kaiser_sinc_filter1d(cutoff, half_width, kernel_size)`.          */
/* ------------------------------------------------------------------------------------------ */

double orc_bessel_i0(double x) {
    /* I0(x) = sum_k ((x/2)^(2k)) / (k!)^2 */
    double q = 0.25 * x * x, term = 1.0, sum = 1.0;
    for (int k = 1; k < 500; ++k) {
        term *= q / ((double)k * (double)k);
        sum += term;
        if (term < 1e-18 * sum) break;
    }
    return sum;
}

void orc_kaiser_sinc_filter(double cutoff, double half_width, int K, double* taps,
                            double* atten, double* beta_out) {
    const int half = K / 2;
    /* Kaiser's attenuation estimate with transition width 4*half_width, then his beta rule. */
    const double A = 2.285 * (half - 1) * M_PI * (4.0 * half_width) + 7.95;
    double beta;
    if (A > 50.0)
        beta = 0.1102 * (A - 8.7);
    else if (A >= 21.0)
        beta = 0.5842 * pow(A - 21.0, 0.4) + 0.07886 * (A - 21.0);
    else
        beta = 0.0;
    const double i0b = orc_bessel_i0(beta);
    double sum = 0.0;
    for (int n = 0; n < K; ++n) {
        /* symmetric (non-periodic) Kaiser window of length K */
        double r = (K > 1) ? (2.0 * n / (double)(K - 1) - 1.0) : 0.0;
        double wn = orc_bessel_i0(beta * sqrt(fmax(0.0, 1.0 - r * r))) / i0b;
        /* filter time axis: half-integer for even K, integer for odd K */
        double t = (K % 2 == 0) ? ((double)(n - half) + 0.5) : (double)(n - half);
        double arg = 2.0 * cutoff * t;
        double sinc = (arg == 0.0) ? 1.0 : sin(M_PI * arg) / (M_PI * arg);
        taps[n] = 2.0 * cutoff * wn * sinc;
        sum += taps[n];
    }
    for (int n = 0; n < K; ++n) taps[n] /= sum;
    if (atten) *atten = A;
    if (beta_out) *beta_out = beta;
}

/* ------------------------------------------------------------------------------------------ */
/* Weight norm: [P3] `_wn_weight(weight_v, weight_g)`, reading R4.                              */
/* ------------------------------------------------------------------------------------------ */

void orc_weight_norm(const float* v, const float* g, long long dim0, long long rest, double* w) {
    for (long long i = 0; i < dim0; ++i) {
        double ss = 0.0;
        for (long long r = 0; r < rest; ++r) ss += (double)v[i * rest + r] * (double)v[i * rest + r];
        const double scale = (double)g[i] / sqrt(ss);
        for (long long r = 0; r < rest; ++r) w[i * rest + r] = scale * (double)v[i * rest + r];
    }
}

/* ------------------------------------------------------------------------------------------ */
/* Convolutions ([P3] `_conv1d`, `_conv_transpose1d`), by their definitions.                   */
/* ------------------------------------------------------------------------------------------ */

void orc_conv1d(const double* x, int Cin, int Lin, const double* w, int Cout, int K,
                const double* bias, int stride, int pad, int dil, double* y, int Lout) {
    const int TB = 1024; /* time block: only splits the parallel work, not the sums */
    const int nblk = (Lout + TB - 1) / TB;
#pragma omp parallel for collapse(2) schedule(dynamic)
    for (int o = 0; o < Cout; ++o) {
        for (int blk = 0; blk < nblk; ++blk) {
            const int t0 = blk * TB;
            const int t1 = (t0 + TB < Lout) ? t0 + TB : Lout;
            double* yo = y + (long long)o * Lout;
            for (int t = t0; t < t1; ++t) yo[t] = bias ? bias[o] : 0.0;
            for (int c = 0; c < Cin; ++c) {
                const double* xc = x + (long long)c * Lin;
                for (int j = 0; j < K; ++j) {
                    const double wv = w[((long long)o * Cin + c) * K + j];
                    const int off = j * dil - pad;
                    /* the t for which the tap lands inside [0, Lin); outside it reads zero */
                    int lo = t0, hi = t1;
                    while (lo < hi && lo * stride + off < 0) ++lo;
                    while (hi > lo && (hi - 1) * stride + off >= Lin) --hi;
                    if (stride == 1) {
                        const double* xs = xc + off;
                        for (int t = lo; t < hi; ++t) yo[t] += wv * xs[t];
                    } else {
                        for (int t = lo; t < hi; ++t) yo[t] += wv * xc[t * stride + off];
                    }
                }
            }
        }
    }
}

void orc_conv_transpose1d(const double* x, int Cin, int Lin, const double* w, int Cout, int K,
                          const double* bias, int stride, int pad, double* y, int Lout) {
#pragma omp parallel for schedule(dynamic)
    for (int o = 0; o < Cout; ++o) {
        double* yo = y + (long long)o * Lout;
        for (int t = 0; t < Lout; ++t) yo[t] = bias ? bias[o] : 0.0;
        for (int c = 0; c < Cin; ++c) {
            const double* xc = x + (long long)c * Lin;
            for (int i = 0; i < Lin; ++i) {
                for (int j = 0; j < K; ++j) {
                    const int t = i * stride - pad + j;
                    if (t >= 0 && t < Lout) yo[t] += xc[i] * w[((long long)c * Cout + o) * K + j];
                }
            }
        }
    }
}

/* ------------------------------------------------------------------------------------------ */
/* SnakeBeta and the anti-aliased activation ([P3] `_activation1d`), readings R2, R3.          */
/* ------------------------------------------------------------------------------------------ */

void orc_snake_beta(const double* x, long long n, double alpha, double beta, double* y) {
    const double inv = 1.0 / (beta + 1e-9);
    for (long long i = 0; i < n; ++i) {
        const double s = sin(alpha * x[i]);
        y[i] = x[i] + inv * s * s;
    }
}

static int clampi(int v, int lo, int hi) { return v < lo ? lo : (v > hi ? hi : v); }

void orc_upsample2(const double* x, int L, const double* taps, int K, double* u) {
    const int ratio = 2;
    const int pad = K / ratio - 1;                                  /* replicate pad */
    const int crop_l = pad * ratio + (K - ratio) / 2;
    const int Lp = L + 2 * pad;
    const int Lfull = (Lp - 1) * ratio + K;                         /* transposed-conv length */
    double* full = (double*)calloc((size_t)Lfull, sizeof(double));
    for (int i = 0; i < Lp; ++i) {
        const double xi = x[clampi(i - pad, 0, L - 1)];
        for (int j = 0; j < K; ++j) full[i * ratio + j] += xi * taps[j];
    }
    for (int n = 0; n < ratio * L; ++n) u[n] = (double)ratio * full[crop_l + n];
    free(full);
}

void orc_downsample2(const double* s, int L2, const double* taps, int K, double* y) {
    const int ratio = 2;
    const int pad_l = K / 2 - ((K % 2 == 0) ? 1 : 0);
    const int Lout = L2 / ratio;
    for (int t = 0; t < Lout; ++t) {
        double acc = 0.0;
        for (int j = 0; j < K; ++j) acc += taps[j] * s[clampi(t * ratio + j - pad_l, 0, L2 - 1)];
        y[t] = acc;
    }
}

void orc_activation1d(const double* x, int L, double alpha, double beta, const double* taps,
                      int K, double* y) {
    double* u = (double*)malloc(sizeof(double) * 2 * (size_t)L);
    orc_upsample2(x, L, taps, K, u);
    orc_snake_beta(u, 2LL * L, alpha, beta, u);
    orc_downsample2(u, 2 * L, taps, K, y);
    free(u);
}

/* Activation over [C, L] with per-channel alpha/beta (fp32 parameters). */
static void act_channels(const double* x, int C, int L, const float* alpha, const float* beta,
                         const double* taps, int K, double* y) {
#pragma omp parallel for schedule(dynamic)
    for (int c = 0; c < C; ++c)
        orc_activation1d(x + (long long)c * L, L, (double)alpha[c], (double)beta[c], taps, K,
                         y + (long long)c * L);
}

/* ------------------------------------------------------------------------------------------ */
/* Weight table lookup and the decode ([P3] `MLXMiniMaxH3AudioVAE.decode`).                     */
/* ------------------------------------------------------------------------------------------ */

int orc_num_threads(void) { return omp_get_max_threads(); }

void orc_default_config(orc_config* cfg) {
    static const int rates[7] = {5, 5, 2, 2, 2, 2, 2};
    static const int kernels[7] = {9, 9, 4, 4, 4, 4, 4};
    memset(cfg, 0, sizeof(*cfg));
    cfg->latent_channels = 32;
    cfg->latent_dim = 2048;
    cfg->decoder_dim = 1024;
    cfg->n_stages = 7;
    for (int i = 0; i < 7; ++i) { cfg->rates[i] = rates[i]; cfg->kernels[i] = kernels[i]; }
    cfg->n_resblocks = 3;
    cfg->rb_kernels[0] = 3; cfg->rb_kernels[1] = 7; cfg->rb_kernels[2] = 11;
    cfg->n_dilations = 3;
    for (int j = 0; j < 3; ++j) {
        cfg->rb_dilations[j][0] = 1; cfg->rb_dilations[j][1] = 3; cfg->rb_dilations[j][2] = 5;
    }
    cfg->clamp = 1;
}

static const orc_tensor* find(const orc_tensor* w, int nw, const char* name) {
    for (int i = 0; i < nw; ++i)
        if (w[i].name && strcmp(w[i].name, name) == 0) return &w[i];
    return NULL;
}

static long long numel(const orc_tensor* t) {
    long long n = 1;
    for (int d = 0; d < t->ndim; ++d) n *= t->shape[d];
    return n;
}

/* Widened copy of a plain tensor; NULL when absent. */
static double* load_plain(const orc_tensor* w, int nw, const char* name, long long expect, int* err) {
    const orc_tensor* t = find(w, nw, name);
    if (!t) return NULL;
    if (numel(t) != expect) { *err = ORC_ERR_SHAPE; return NULL; }
    double* d = (double*)malloc(sizeof(double) * (size_t)expect);
    for (long long i = 0; i < expect; ++i) d[i] = (double)t->data[i];
    return d;
}

/* Weight-normed kernel `<prefix>.weight_v` / `<prefix>.weight_g` folded to fp64. */
static double* load_wn(const orc_tensor* w, int nw, const char* prefix, long long d0, long long d1,
                       long long k, int* err) {
    char nv[320], ng[320];
    snprintf(nv, sizeof nv, "%s.weight_v", prefix);
    snprintf(ng, sizeof ng, "%s.weight_g", prefix);
    const orc_tensor* v = find(w, nw, nv);
    const orc_tensor* g = find(w, nw, ng);
    if (!v || !g) { *err = ORC_ERR_MISSING; return NULL; }
    if (v->ndim != 3 || v->shape[0] != d0 || v->shape[1] != d1 || v->shape[2] != k ||
        numel(g) != d0) { *err = ORC_ERR_SHAPE; return NULL; }
    double* out = (double*)malloc(sizeof(double) * (size_t)(d0 * d1 * k));
    orc_weight_norm(v->data, g->data, d0, d1 * k, out);
    return out;
}

static double* load_bias(const orc_tensor* w, int nw, const char* prefix, long long n, int required,
                         int* err) {
    char nb[320];
    snprintf(nb, sizeof nb, "%s.bias", prefix);
    double* b = load_plain(w, nw, nb, n, err);
    if (!b && required && *err == ORC_OK) *err = ORC_ERR_MISSING;
    return b;
}

static void filter_taps(double* taps, int K) {
    /* ratio 2: cutoff 0.5/2, half-width 0.6/2 (reading R2); stored as fp32 buffers */
    orc_kaiser_sinc_filter(0.5 / 2.0, 0.6 / 2.0, K, taps, NULL, NULL);
    for (int i = 0; i < K; ++i) taps[i] = (double)(float)taps[i];
}

/* The AMP stage for one batch item: mean over resblocks j of the residual chain. */
static int amp_stage_item(const orc_config* cfg, const orc_tensor* w, int nw, int stage,
                          const double* h, int C, int L, double* out) {
    enum { KF = 12 };
    double taps[KF];
    filter_taps(taps, KF);
    int err = ORC_OK;
    const long long CL = (long long)C * L;
    double* x = (double*)malloc(sizeof(double) * (size_t)CL);
    double* a = (double*)malloc(sizeof(double) * (size_t)CL);
    double* t = (double*)malloc(sizeof(double) * (size_t)CL);
    for (long long i = 0; i < CL; ++i) out[i] = 0.0;
    for (int j = 0; j < cfg->n_resblocks && err == ORC_OK; ++j) {
        const int k = cfg->rb_kernels[j];
        const int rb = stage * cfg->n_resblocks + j;
        memcpy(x, h, sizeof(double) * (size_t)CL);
        for (int m = 0; m < cfg->n_dilations && err == ORC_OK; ++m) {
            const int d = cfg->rb_dilations[j][m];
            char p[256];
            const orc_tensor *a1, *b1, *a2, *b2;
            snprintf(p, sizeof p, "decoder.resblocks.%d.activations.%d.act.alpha", rb, 2 * m);
            a1 = find(w, nw, p);
            snprintf(p, sizeof p, "decoder.resblocks.%d.activations.%d.act.beta", rb, 2 * m);
            b1 = find(w, nw, p);
            snprintf(p, sizeof p, "decoder.resblocks.%d.activations.%d.act.alpha", rb, 2 * m + 1);
            a2 = find(w, nw, p);
            snprintf(p, sizeof p, "decoder.resblocks.%d.activations.%d.act.beta", rb, 2 * m + 1);
            b2 = find(w, nw, p);
            if (!a1 || !b1 || !a2 || !b2) { err = ORC_ERR_MISSING; break; }
            if (numel(a1) != C || numel(b1) != C || numel(a2) != C || numel(b2) != C) {
                err = ORC_ERR_SHAPE; break;
            }
            snprintf(p, sizeof p, "decoder.resblocks.%d.convs1.%d", rb, m);
            double* w1 = load_wn(w, nw, p, C, C, k, &err);
            double* bias1 = load_bias(w, nw, p, C, 1, &err);
            snprintf(p, sizeof p, "decoder.resblocks.%d.convs2.%d", rb, m);
            double* w2 = load_wn(w, nw, p, C, C, k, &err);
            double* bias2 = load_bias(w, nw, p, C, 1, &err);
            if (err == ORC_OK) {
                act_channels(x, C, L, a1->data, b1->data, taps, KF, a);
                orc_conv1d(a, C, L, w1, C, k, bias1, 1, d * (k - 1) / 2, d, t, L);
                act_channels(t, C, L, a2->data, b2->data, taps, KF, a);
                orc_conv1d(a, C, L, w2, C, k, bias2, 1, (k - 1) / 2, 1, t, L);
                for (long long i = 0; i < CL; ++i) x[i] += t[i];
            }
            free(w1); free(bias1); free(w2); free(bias2);
        }
        for (long long i = 0; i < CL; ++i) out[i] += x[i];
    }
    for (long long i = 0; i < CL; ++i) out[i] /= (double)cfg->n_resblocks;
    free(x); free(a); free(t);
    return err;
}

static int stage_channels(const orc_config* cfg, int stage) {
    return cfg->decoder_dim >> (stage + 1);
}

int orc_amp_stage_f64(const orc_config* cfg, const orc_tensor* w, int nw, int stage,
                      const double* x, int B, int L, double* out) {
    if (!cfg || !w || !x || !out || B < 1 || L < 1 || stage < 0 || stage >= cfg->n_stages)
        return ORC_ERR_ARG;
    const int C = stage_channels(cfg, stage);
    for (int b = 0; b < B; ++b) {
        int err = amp_stage_item(cfg, w, nw, stage, x + (long long)b * C * L, C, L,
                                 out + (long long)b * C * L);
        if (err) return err;
    }
    return ORC_OK;
}

int orc_amp_stage(const orc_config* cfg, const orc_tensor* w, int nw, int stage,
                  const float* x, int B, int L, double* out) {
    if (!cfg || !x || stage < 0 || stage >= cfg->n_stages || B < 1 || L < 1) return ORC_ERR_ARG;
    const long long n = (long long)B * stage_channels(cfg, stage) * L;
    double* xd = (double*)malloc(sizeof(double) * (size_t)n);
    for (long long i = 0; i < n; ++i) xd[i] = (double)x[i];
    int err = orc_amp_stage_f64(cfg, w, nw, stage, xd, B, L, out);
    free(xd);
    return err;
}

/* One batch item of the decode; z is [latent_channels, N] fp64, y is [hop * N]. */
static int decode_item(const orc_config* cfg, const orc_tensor* w, int nw, const double* z, int N,
                       double* y) {
    int err = ORC_OK;
    const int Cz = cfg->latent_channels, D = cfg->latent_dim, C0 = cfg->decoder_dim;
    /* dec_in_proj: 1x1 conv with bias */
    const orc_tensor* wi = find(w, nw, "dec_in_proj.weight");
    if (!wi) return ORC_ERR_MISSING;
    if (numel(wi) != (long long)D * Cz) return ORC_ERR_SHAPE;
    double* w_in = load_plain(w, nw, "dec_in_proj.weight", (long long)D * Cz, &err);
    double* b_in = load_bias(w, nw, "dec_in_proj", D, 1, &err);
    if (err) { free(w_in); free(b_in); return err; }
    double* h0 = (double*)malloc(sizeof(double) * (size_t)D * N);
    orc_conv1d(z, Cz, N, w_in, D, 1, b_in, 1, 0, 1, h0, N);
    free(w_in); free(b_in);

    /* conv_pre: weight-normed conv, padding 3 (kernel 7, reading R5) */
    const orc_tensor* vpre = find(w, nw, "decoder.conv_pre.weight_v");
    if (!vpre) { free(h0); return ORC_ERR_MISSING; }
    const int kpre = (int)vpre->shape[2];
    double* w_pre = load_wn(w, nw, "decoder.conv_pre", C0, D, kpre, &err);
    double* b_pre = load_bias(w, nw, "decoder.conv_pre", C0, 1, &err);
    if (err) { free(h0); free(w_pre); free(b_pre); return err; }
    double* h = (double*)malloc(sizeof(double) * (size_t)C0 * N);
    orc_conv1d(h0, D, N, w_pre, C0, kpre, b_pre, 1, 3, 1, h, N);
    free(h0); free(w_pre); free(b_pre);

    int C = C0, L = N;
    for (int i = 0; i < cfg->n_stages; ++i) {
        const int r = cfg->rates[i], K = cfg->kernels[i];
        const int Co = C / 2, Lo = L * r;
        char p[64];
        snprintf(p, sizeof p, "decoder.ups.%d.0", i);
        double* wu = load_wn(w, nw, p, C, Co, K, &err);
        double* bu = load_bias(w, nw, p, Co, 1, &err);
        if (err) { free(h); free(wu); free(bu); return err; }
        double* hu = (double*)malloc(sizeof(double) * (size_t)Co * Lo);
        orc_conv_transpose1d(h, C, L, wu, Co, K, bu, r, (K - r) / 2, hu, Lo);
        free(h); free(wu); free(bu);
        h = (double*)malloc(sizeof(double) * (size_t)Co * Lo);
        err = amp_stage_item(cfg, w, nw, i, hu, Co, Lo, h);
        free(hu);
        if (err) { free(h); return err; }
        C = Co; L = Lo;
    }

    /* activation_post, conv_post (bias optional), clamp */
    const orc_tensor* ap = find(w, nw, "decoder.activation_post.act.alpha");
    const orc_tensor* bp = find(w, nw, "decoder.activation_post.act.beta");
    if (!ap || !bp) { free(h); return ORC_ERR_MISSING; }
    if (numel(ap) != C || numel(bp) != C) { free(h); return ORC_ERR_SHAPE; }
    enum { KF = 12 };
    double taps[KF];
    filter_taps(taps, KF);
    double* a = (double*)malloc(sizeof(double) * (size_t)C * L);
    act_channels(h, C, L, ap->data, bp->data, taps, KF, a);
    free(h);
    const orc_tensor* vpost = find(w, nw, "decoder.conv_post.weight_v");
    if (!vpost) { free(a); return ORC_ERR_MISSING; }
    const int kpost = (int)vpost->shape[2];
    double* w_post = load_wn(w, nw, "decoder.conv_post", 1, C, kpost, &err);
    double* b_post = load_bias(w, nw, "decoder.conv_post", 1, 0, &err);
    if (err) { free(a); free(w_post); free(b_post); return err; }
    orc_conv1d(a, C, L, w_post, 1, kpost, b_post, 1, 3, 1, y, L);
    free(a); free(w_post); free(b_post);
    if (cfg->clamp)
        for (int t = 0; t < L; ++t) {
            /* NaN propagates; +-1 inclusive */
            if (y[t] < -1.0) y[t] = -1.0;
            else if (y[t] > 1.0) y[t] = 1.0;
        }
    return ORC_OK;
}

int orc_decode(const orc_config* cfg, const orc_tensor* w, int nw, const float* latents,
               int B, int N, double* out) {
    if (!cfg || !w || !latents || !out || B < 1 || N < 1) return ORC_ERR_ARG;
    long long hop = 1;
    for (int i = 0; i < cfg->n_stages; ++i) hop *= cfg->rates[i];
    const int Cz = cfg->latent_channels;
    double* z = (double*)malloc(sizeof(double) * (size_t)Cz * N);
    for (int b = 0; b < B; ++b) {
        for (int c = 0; c < Cz; ++c)
            for (int n = 0; n < N; ++n) {
                double v = (double)latents[((long long)b * Cz + c) * N + n];
                /* [P4]: denormalise z = x * std_c + mean_c */
                if (cfg->latents_std) v *= (double)cfg->latents_std[c];
                if (cfg->latents_mean) v += (double)cfg->latents_mean[c];
                z[(long long)c * N + n] = v;
            }
        int err = decode_item(cfg, w, nw, z, N, out + (long long)b * hop * N);
        if (err) { free(z); return err; }
    }
    free(z);
    return ORC_OK;
}

/*
 * mh3a_oracle.h -- plain, slow CPU oracle of the MiniMax-H3 audio-VAE BigVGAN decode.
 *
 * TEST INFRASTRUCTURE ONLY.  Only tests/, __graft_entry__.smoke() and the CPU-baseline /
 * reference legs of bench.py may load this library.  The CUDA library never includes,
 * links or calls anything here, and this file includes nothing from it.
 *
 * Every floating-point step runs in double (fp64): fp32 weights and inputs are widened on
 * entry, all intermediate tensors are fp64, and results are returned in fp64.  Each batch
 * item is processed on its own, and every output element is produced by exactly one
 * thread in a fixed order, so results do not depend on the OpenMP thread count.
 *
 * Sources (web pages; cited by title and section):
 *   [P1] diffusers "AutoencoderKLMiniMaxH3Audio" API page: constructor parameters,
 *        `decode` section (latents [B,32,N] -> waveform [B,1,800N] clamped to [-1,1]).
 *   [P3] FastVideo "minimax_h3_audio_vae" (MLX runtime) page: `MLXMiniMaxH3AudioVAE.decode`
 *        and `kaiser_sinc_filter1d`; module summary bullet "Decoder".
 *   [P4] diffusers "AutoencoderKLMiniMaxH3" page: per-channel latent (de)normalisation bullet.
 */
#ifndef MH3A_ORACLE_H
#define MH3A_ORACLE_H

#ifdef __cplusplus
extern "C" {
#endif

/* A named fp32 tensor from the caller's weight table (host memory). */
typedef struct {
    const char* name;
    const float* data;
    int ndim;
    long long shape[3];
} orc_tensor;

/* Architecture ([P1] constructor parameters) plus oracle switches. */
typedef struct {
    int latent_channels;        /* 32 */
    int latent_dim;             /* 2048 */
    int decoder_dim;            /* 1024, halved per upsampling stage */
    int n_stages;               /* len(decoder_rates) = 7 */
    int rates[8];               /* (5,5,2,2,2,2,2) */
    int kernels[8];             /* (9,9,4,4,4,4,4) */
    int n_resblocks;            /* len(resblock_kernel_sizes) = 3 */
    int rb_kernels[4];          /* (3,7,11) */
    int n_dilations;            /* 3 */
    int rb_dilations[4][4];     /* ((1,3,5),(1,3,5),(1,3,5)) */
    int clamp;                  /* 1: clamp the waveform to [-1,1] ([P3] decode, last line) */
    const float* latents_mean;  /* [latent_channels] or NULL ([P4] denormalisation) */
    const float* latents_std;   /* [latent_channels] or NULL */
} orc_config;

/* Return codes. */
enum { ORC_OK = 0, ORC_ERR_ARG = 1, ORC_ERR_MISSING = 2, ORC_ERR_SHAPE = 3, ORC_ERR_ALLOC = 4 };

/* Kaiser-windowed sinc low-pass, [P3] `kaiser_sinc_filter1d`, evaluated in fp64.
 * taps[K] receives the normalised taps; *atten and *beta (may be NULL) the Kaiser design values. */
void orc_kaiser_sinc_filter(double cutoff, double half_width, int K, double* taps,
                            double* atten, double* beta);

/* Zeroth-order modified Bessel function of the first kind (power series). */
double orc_bessel_i0(double x);

/* Weight norm w = g * v / ||v||, the norm over every axis but the first of the stored
 * tensor ([P3] `_wn_weight(weight_v, weight_g)`).  v is [dim0, rest], g is [dim0]. */
void orc_weight_norm(const float* v, const float* g, long long dim0, long long rest, double* w);

/* Zero-padded conv1d: y[o,t] = b[o] + sum_{c,j} w[o,c,j] x[c, t*stride + j*dil - pad].
 * x [Cin,Lin], w [Cout,Cin,K], bias [Cout] or NULL, y [Cout,Lout],
 * Lout = (Lin + 2 pad - dil (K-1) - 1) / stride + 1. */
void orc_conv1d(const double* x, int Cin, int Lin, const double* w, int Cout, int K,
                const double* bias, int stride, int pad, int dil, double* y, int Lout);

/* Transposed conv1d by its scatter definition: y[o, i*stride - pad + j] += x[c,i] w[c,o,j].
 * x [Cin,Lin], w [Cin,Cout,K], y [Cout,Lout] with Lout = (Lin-1) stride - 2 pad + K. */
void orc_conv_transpose1d(const double* x, int Cin, int Lin, const double* w, int Cout, int K,
                          const double* bias, int stride, int pad, double* y, int Lout);

/* SnakeBeta y = x + sin^2(alpha x) / (beta + 1e-9), elementwise for one channel. */
void orc_snake_beta(const double* x, long long n, double alpha, double beta, double* y);

/* Anti-aliased activation on one channel of length L: 2x Kaiser-sinc upsample (replicate
 * padded) -> SnakeBeta -> 2x low-pass decimation (replicate padded).  taps[K] are the
 * shared filter taps as stored (fp32 values widened to fp64). */
void orc_upsample2(const double* x, int L, const double* taps, int K, double* u /*[2L]*/);
void orc_downsample2(const double* s, int L2, const double* taps, int K, double* y /*[L2/2]*/);
void orc_activation1d(const double* x, int L, double alpha, double beta, const double* taps,
                      int K, double* y);

/* Number of OpenMP threads the oracle's parallel loops use. */
int orc_num_threads(void);

/* Default architecture ([P1] constructor defaults) with clamp on and no denormalisation. */
void orc_default_config(orc_config* cfg);

/* Full decode ([P3] `MLXMiniMaxH3AudioVAE.decode`): latents [B, latent_channels, N] fp32 ->
 * out [B, 1, N * prod(rates)] fp64. */
int orc_decode(const orc_config* cfg, const orc_tensor* w, int nw, const float* latents,
               int B, int N, double* out);

/* One AMP stage (the averaged parallel residual blocks after upsampling stage `stage`):
 * x [B, C, L] fp32 with C = decoder_dim / 2^(stage+1) -> out [B, C, L] fp64. */
int orc_amp_stage(const orc_config* cfg, const orc_tensor* w, int nw, int stage,
                  const float* x, int B, int L, double* out);

/* Same, but starting from an fp64 input (used by the decode and by tests). */
int orc_amp_stage_f64(const orc_config* cfg, const orc_tensor* w, int nw, int stage,
                      const double* x, int B, int L, double* out);

#ifdef __cplusplus
}
#endif
#endif

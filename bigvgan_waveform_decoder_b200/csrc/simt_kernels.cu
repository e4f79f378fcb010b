// simt_kernels.cu -- fp32 CUDA-core kernels of the decode.
//
// k_conv_simt: one stride-1 convolution (dilated, "same" padded) whose input optionally goes
// through the anti-aliased SnakeBeta first, computed in shared memory as the conv's prologue:
//   a = down2(snake(up2(x)))      (FastVideo "minimax_h3_audio_vae" page, `_activation1d`;
//                                  filter from `kaiser_sinc_filter1d`)
//   y[o,t] = bias[o] + sum_{c,j} w[o,c,j] a[c, t + j*dil - pad]  (+ residual)
// The up-sampler replicate-pads its input by 5 samples, runs a stride-2 transposed conv with
// the 12 taps at gain 2 and crops 15 samples per side; in polyphase form that is
//   u[2m]   = sum_q 2 f[2q+1] x[m+2-q],   u[2m+1] = sum_q 2 f[2q] x[m+3-q],   q = 0..5,
// with x indices clamped to [0, L).  SnakeBeta: s = u + sin^2(alpha u) / (beta + 1e-9).  The
// decimator replicate-pads s by 5 (left) / 6 (right) and takes a[t] = sum_j f[j] s[2t+j-5]
// with the index clamped to [0, 2L).  The conv zero-pads a outside [0, L).
//
// Up to four independent jobs (the parallel residual blocks of one AMP stage, which share
// shapes but not kernels or weights) run in one launch, one per blockIdx.z.
//
// k_convT_simt: transposed conv (upsampling stage) in polyphase form: output t = r*u + phi
// only meets taps j = (phi + pad) mod r + r*m, so no zero is ever inserted or multiplied.
#include "mh3a_internal.cuh"
#include "tc_ptx.cuh"

namespace mh3a {
namespace {

constexpr int CK = 8;  // input channels staged per chunk

__device__ __forceinline__ int clampi(int v, int lo, int hi) { return v < lo ? lo : (v > hi ? hi : v); }

// sin^2(alpha * u).  The phase is carried as v + e with v = fl(alpha u) and e = alpha u - v
// (exact, from one fma), so no rounding of the product reaches the sine.  sin^2 has period
// pi: the phase is reduced to r = v - k pi + e, k = rint(v / pi), by the Cody-Waite method
// (pi split into fp32(pi) and the fp32 remainder; each k * part is subtracted inside one fma).
// sin(r) on [-pi/2, pi/2] is its Taylor series through r^13 (truncation error below
// (pi/2)^15 / 15! < 7e-10), evaluated by Horner's rule in r^2.
__device__ __forceinline__ float sin_sq(float alpha, float u) {
    const float kInvPi = 0.318309886183790671538f;
    const float kPiHi = 3.14159274101257324219f;      // fp32(pi)
    const float kPiLo = -8.74227800037248297e-08f;    // pi - fp32(pi)
    const float v = alpha * u;
    const float e = fmaf(alpha, u, -v);
    const float k = rintf(v * kInvPi);
    float r = fmaf(-k, kPiHi, v);
    r = fmaf(-k, kPiLo, r) + e;
    const float r2 = r * r;
    float p = 1.0f / 6227020800.0f;                   //  1/13!
    p = fmaf(p, r2, -1.0f / 39916800.0f);             // -1/11!
    p = fmaf(p, r2, 1.0f / 362880.0f);                //  1/9!
    p = fmaf(p, r2, -1.0f / 5040.0f);                 // -1/7!
    p = fmaf(p, r2, 1.0f / 120.0f);                   //  1/5!
    p = fmaf(p, r2, -1.0f / 6.0f);                    // -1/3!
    const float s = fmaf(r * r2, p, r);
    return s * s;
}

__device__ __forceinline__ float load_in(const float* x0, const float* x1, const float* x2, long long i,
                                         bool mean3) {
    if (mean3) return (__ldg(x0 + i) + __ldg(x1 + i) + __ldg(x2 + i)) / 3.0f;
    return __ldg(x0 + i);
}

template <int K, int CO_T, int RO, int RT, int TX>
__device__ __forceinline__ void fma_chunk(float (&acc)[RO][RT], const float* __restrict__ as, int AWs,
                                          const float* __restrict__ ws, int Ks, int dil, int ty, int tx) {
#pragma unroll
    for (int c = 0; c < CK; ++c) {
#pragma unroll
        for (int j = 0; j < K; ++j) {
            float wv[RO], av[RT];
#pragma unroll
            for (int r = 0; r < RO; ++r) wv[r] = ws[(c * Ks + j) * CO_T + ty * RO + r];
#pragma unroll
            for (int i = 0; i < RT; ++i) av[i] = as[c * AWs + tx + i * TX + j * dil];
#pragma unroll
            for (int r = 0; r < RO; ++r)
#pragma unroll
                for (int i = 0; i < RT; ++i) acc[r][i] = fmaf(wv[r], av[i], acc[r][i]);
        }
    }
}

template <int CO_T, int RO, int RT, int TX>
__device__ __forceinline__ void fma_chunk_dyn(float (&acc)[RO][RT], const float* __restrict__ as, int AWs,
                                              const float* __restrict__ ws, int K, int dil, int ty, int tx) {
    for (int c = 0; c < CK; ++c) {
        for (int j = 0; j < K; ++j) {
            float wv[RO], av[RT];
#pragma unroll
            for (int r = 0; r < RO; ++r) wv[r] = ws[(c * K + j) * CO_T + ty * RO + r];
#pragma unroll
            for (int i = 0; i < RT; ++i) av[i] = as[c * AWs + tx + i * TX + j * dil];
#pragma unroll
            for (int r = 0; r < RO; ++r)
#pragma unroll
                for (int i = 0; i < RT; ++i) acc[r][i] = fmaf(wv[r], av[i], acc[r][i]);
        }
    }
}

// Shared-memory plan (floats): xs[CK][XW] | sw[CK][SW] | as[CK][AWs] | ws[CK][Kmax][CO_T]
struct SmemPlan {
    int XW, SW, AWs, Kmax;
};

template <int CO_T, int T_T, int RO, int RT, bool ACT, bool MEAN3>
__global__ void __launch_bounds__((CO_T / RO) * (T_T / RT))
k_conv_simt(const ConvParams p, const SmemPlan sp) {
    constexpr int TX = T_T / RT;
    constexpr int NT = (CO_T / RO) * TX;
    extern __shared__ float smem[];
    float* xs = smem;
    float* sw = xs + (ACT ? CK * sp.XW : 0);
    float* as = sw + (ACT ? CK * sp.SW : 0);
    float* ws = as + CK * sp.AWs;

    const ConvJob& J = p.job[blockIdx.z];
    const int K = J.K, dil = J.dil, pad = J.pad;
    const int L = p.L, Cin = p.Cin, Cout = p.Cout;
    const int b = blockIdx.x / p.tiles_t;
    const int t0 = (blockIdx.x % p.tiles_t) * T_T;
    const int o0 = blockIdx.y * CO_T;
    const int tid = threadIdx.x;
    const int ty = tid / TX, tx = tid % TX;
    const int AW = T_T + (K - 1) * dil;   // conv input window
    const int a_start = t0 - pad;
    const int xs_start = a_start - 6;     // x window for the activation
    const int XW = AW + 12;
    const int n_start = 2 * a_start - 5;  // 2x-rate window for the decimator
    const int SW = 2 * AW + 10;
    const long long in_base = (long long)b * Cin * L;

    // Two-level summation: each chunk of CK input channels accumulates into a fresh fp32
    // partial, which is folded into a Kahan-compensated running total, so the rounding error
    // grows with the chunk length rather than with Cin * K (2048 * 7 terms for conv_pre).
    float acc[RO][RT], tot[RO][RT], cmp[RO][RT];
#pragma unroll
    for (int r = 0; r < RO; ++r)
#pragma unroll
        for (int i = 0; i < RT; ++i) tot[r][i] = cmp[r][i] = 0.f;

    for (int c0 = 0; c0 < Cin; c0 += CK) {
#pragma unroll
        for (int r = 0; r < RO; ++r)
#pragma unroll
            for (int i = 0; i < RT; ++i) acc[r][i] = 0.f;
        if (ACT) {
            // The 8 warps of the block own the 8 channels of the chunk (NT == 32 * CK), so the
            // three steps below touch only their own warp's rows and need no block barrier.
            const int c = tid >> 5, lane = tid & 31;
            float* xrow = xs + c * sp.XW;
            float* srow = sw + c * sp.SW;
            const bool live = c0 + c < Cin;
            // 1. raw input window, replicate-clamped at the sequence ends
            for (int q = lane; q < XW; q += 32)
                xrow[q] = live ? load_in(J.x0, J.x1, J.x2,
                                         in_base + (long long)(c0 + c) * L + clampi(xs_start + q, 0, L - 1), MEAN3)
                               : 0.f;
            __syncwarp();
            // 2. SnakeBeta of the 2x upsampled signal over the decimator's window.  A lane takes
            //    one input position m and forms both phases n = 2m, 2m+1 from x[m-3 .. m+3];
            //    positions past either end repeat the end sample (replicate padding).
            {
                const float al = live ? __ldg(J.alpha + c0 + c) : 0.f;
                const float ib = live ? __ldg(J.inv_beta + c0 + c) : 0.f;
                const float* xr0 = xrow - xs_start;
                const int m_lo = n_start >> 1, m_hi = (n_start + SW - 1) >> 1;
                for (int m = m_lo + lane; m <= m_hi; m += 32) {
                    const int mc = clampi(m, 0, L - 1);
                    float xv[7];
#pragma unroll
                    for (int k = 0; k < 7; ++k) xv[k] = xr0[mc + k - 3];
                    float ue = 0.f, uo = 0.f;
#pragma unroll
                    for (int k = 0; k < 6; ++k) {
                        ue = fmaf(p.filt.up[2 * k + 1], xv[5 - k], ue);
                        uo = fmaf(p.filt.up[2 * k], xv[6 - k], uo);
                    }
                    const float se = fmaf(sin_sq(al, ue), ib, ue);
                    const float so = fmaf(sin_sq(al, uo), ib, uo);
                    const int ie = 2 * m - n_start;
                    if (ie >= 0 && ie < SW) srow[ie] = (m > L - 1) ? so : se;
                    if (ie + 1 >= 0 && ie + 1 < SW) srow[ie + 1] = (m < 0) ? se : so;
                }
            }
            __syncwarp();
            // 3. decimate into the conv window (zero outside the sequence)
            for (int q = lane; q < AW; q += 32) {
                const int g = a_start + q;
                float a = 0.f;
                if (g >= 0 && g < L) {
                    const float2* sr = reinterpret_cast<const float2*>(srow + 2 * q);
#pragma unroll
                    for (int j = 0; j < kFilterTaps / 2; ++j) {
                        const float2 v = sr[j];
                        a = fmaf(p.filt.down[2 * j], v.x, a);
                        a = fmaf(p.filt.down[2 * j + 1], v.y, a);
                    }
                }
                as[c * sp.AWs + q] = a;
            }
        } else {
            for (int i = tid; i < CK * AW; i += NT) {
                const int c = i / AW, q = i - c * AW;
                const int g = a_start + q;
                float v = 0.f;
                if (c0 + c < Cin && g >= 0 && g < L)
                    v = load_in(J.x0, J.x1, J.x2, in_base + (long long)(c0 + c) * L + g, MEAN3);
                as[c * sp.AWs + q] = v;
            }
        }
        // weights of this chunk: ws[c][j][o] = w[c0+c][j][o0+o]
        for (int i = tid; i < CK * K * CO_T; i += NT) {
            const int o = i % CO_T, cj = i / CO_T;
            const int c = cj / K;
            float v = 0.f;
            if (c0 + c < Cin && o0 + o < Cout) v = __ldg(J.w + ((long long)(c0 + c) * K + (cj - c * K)) * Cout + o0 + o);
            ws[cj * CO_T + o] = v;
        }
        __syncthreads();
        switch (K) {
            case 1: fma_chunk<1, CO_T, RO, RT, TX>(acc, as, sp.AWs, ws, 1, dil, ty, tx); break;
            case 3: fma_chunk<3, CO_T, RO, RT, TX>(acc, as, sp.AWs, ws, 3, dil, ty, tx); break;
            case 7: fma_chunk<7, CO_T, RO, RT, TX>(acc, as, sp.AWs, ws, 7, dil, ty, tx); break;
            case 11: fma_chunk<11, CO_T, RO, RT, TX>(acc, as, sp.AWs, ws, 11, dil, ty, tx); break;
            default: fma_chunk_dyn<CO_T, RO, RT, TX>(acc, as, sp.AWs, ws, K, dil, ty, tx); break;
        }
#pragma unroll
        for (int r = 0; r < RO; ++r)
#pragma unroll
            for (int i = 0; i < RT; ++i) {
                const float y = acc[r][i] - cmp[r][i];
                const float t = tot[r][i] + y;
                cmp[r][i] = (t - tot[r][i]) - y;
                tot[r][i] = t;
            }
        __syncthreads();
    }

    const long long out_base = (long long)b * Cout * L;
#pragma unroll
    for (int r = 0; r < RO; ++r) {
        const int o = o0 + ty * RO + r;
        if (o >= Cout) continue;
        const float bo = J.bias ? __ldg(J.bias + o) : 0.f;
#pragma unroll
        for (int i = 0; i < RT; ++i) {
            const int t = t0 + tx + i * TX;
            if (t >= L) continue;
            const long long idx = out_base + (long long)o * L + t;
            float y = (tot[r][i] - cmp[r][i]) + bo;
            if (J.res) y += J.res[idx];
            if (p.clamp) y = (y < -1.f) ? -1.f : ((y > 1.f) ? 1.f : y);  // NaN passes through
            J.out[idx] = y;
        }
    }
}

// Transposed conv, polyphase.  The tile covers T = r * U outputs starting at t0 = tile * r * U;
// thread (ty, tx) owns outputs t = t0 + r * (tx + i * TX) + phi for every phase phi < r, so all
// lanes of a warp share phi and read the same weights.
template <int CO_T, int RO, int RT, int TX, int RMAX, bool MEAN3>
__global__ void __launch_bounds__((CO_T / RO) * TX)
k_convT_simt(const ConvTParams p) {
    constexpr int NT = (CO_T / RO) * TX;
    constexpr int U = TX * RT;
    extern __shared__ float smem[];
    const int r = p.r, K = p.K, pad = p.pad;
    const int Lout = p.Lin * r;
    const int nmax = (K + r - 1) / r;                   // taps per phase (at most)
    const int b = blockIdx.x / p.tiles_t;
    const int tile = blockIdx.x % p.tiles_t;
    const int t0 = tile * r * U;
    const int u0 = t0 / r;
    const int i_lo = u0 - nmax;                          // lowest input index touched
    const int IW = U + nmax + (r - 1 + pad) / r + 2;     // input window length
    float* xs = smem;                                    // [CK][IW]
    float* ws = xs + CK * IW;                            // [CK][K][CO_T]
    const int o0 = blockIdx.y * CO_T;
    const int tid = threadIdx.x, ty = tid / TX, tx = tid % TX;
    const long long in_base = (long long)b * p.Cin * p.Lin;

    // two-level summation: per-chunk fp32 partials folded into a running total
    float acc[RMAX][RO][RT], tot[RMAX][RO][RT];
#pragma unroll
    for (int f = 0; f < RMAX; ++f)
#pragma unroll
        for (int q = 0; q < RO; ++q)
#pragma unroll
            for (int i = 0; i < RT; ++i) tot[f][q][i] = 0.f;

    for (int c0 = 0; c0 < p.Cin; c0 += CK) {
#pragma unroll
        for (int f = 0; f < RMAX; ++f)
#pragma unroll
            for (int q = 0; q < RO; ++q)
#pragma unroll
                for (int i = 0; i < RT; ++i) acc[f][q][i] = 0.f;
        for (int i = tid; i < CK * IW; i += NT) {
            const int c = i / IW, q = i - c * IW;
            const int g = i_lo + q;
            float v = 0.f;
            if (c0 + c < p.Cin && g >= 0 && g < p.Lin)
                v = load_in(p.x0, p.x1, p.x2, in_base + (long long)(c0 + c) * p.Lin + g, MEAN3);
            xs[i] = v;
        }
        for (int i = tid; i < CK * K * CO_T; i += NT) {
            const int o = i % CO_T, cj = i / CO_T, c = cj / K;
            float v = 0.f;
            if (c0 + c < p.Cin && o0 + o < p.Cout)
                v = __ldg(p.w + ((long long)(c0 + c) * K + (cj - c * K)) * p.Cout + o0 + o);
            ws[i] = v;
        }
        __syncthreads();
#pragma unroll
        for (int phi = 0; phi < RMAX; ++phi) {
            if (phi >= r) break;
            const int j0 = (phi + pad) % r;
            const int base = (phi + pad) / r;            // input offset of tap j0
            for (int c = 0; c < CK; ++c) {
                for (int m = 0; m < nmax; ++m) {
                    const int j = j0 + m * r;
                    if (j >= K) break;
                    float wv[RO];
#pragma unroll
                    for (int q = 0; q < RO; ++q) wv[q] = ws[(c * K + j) * CO_T + ty * RO + q];
#pragma unroll
                    for (int i = 0; i < RT; ++i) {
                        // input index u0 + tx + i*TX + base - m, relative to i_lo
                        const float xv = xs[c * IW + (tx + i * TX + base - m + nmax)];
#pragma unroll
                        for (int q = 0; q < RO; ++q) acc[phi][q][i] = fmaf(wv[q], xv, acc[phi][q][i]);
                    }
                }
            }
        }
#pragma unroll
        for (int f = 0; f < RMAX; ++f)
#pragma unroll
            for (int q = 0; q < RO; ++q)
#pragma unroll
                for (int i = 0; i < RT; ++i) tot[f][q][i] += acc[f][q][i];
        __syncthreads();
    }
    const long long out_base = (long long)b * p.Cout * Lout;
#pragma unroll
    for (int phi = 0; phi < RMAX; ++phi) {
        if (phi >= r) break;
#pragma unroll
        for (int q = 0; q < RO; ++q) {
            const int o = o0 + ty * RO + q;
            if (o >= p.Cout) continue;
            const float bo = __ldg(p.bias + o);
#pragma unroll
            for (int i = 0; i < RT; ++i) {
                const int t = t0 + r * (tx + i * TX) + phi;
                if (t < Lout) p.out[out_base + (long long)o * Lout + t] = tot[phi][q][i] + bo;
            }
        }
    }
}

__global__ void k_mean3(const Mean3Params p) {
    const long long n4 = p.vec4 ? p.n / 4 : 0;
    const long long stride = (long long)gridDim.x * blockDim.x;
    for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < n4; i += stride) {
        const float4 a = __ldg(reinterpret_cast<const float4*>(p.x0) + i);
        const float4 b = __ldg(reinterpret_cast<const float4*>(p.x1) + i);
        const float4 c = __ldg(reinterpret_cast<const float4*>(p.x2) + i);
        float4 y;
        y.x = (a.x + b.x + c.x) / 3.0f;
        y.y = (a.y + b.y + c.y) / 3.0f;
        y.z = (a.z + b.z + c.z) / 3.0f;
        y.w = (a.w + b.w + c.w) / 3.0f;
        reinterpret_cast<float4*>(p.out)[i] = y;
    }
    for (long long i = 4 * n4 + blockIdx.x * (long long)blockDim.x + threadIdx.x; i < p.n; i += stride)
        p.out[i] = (p.x0[i] + p.x1[i] + p.x2[i]) / 3.0f;
}

template <int CO_T, int T_T, int RO, int RT, bool ACT, bool MEAN3>
int launch_conv_cfg(const ConvParams& p0, int njobs, cudaStream_t s) {
    ConvParams p = p0;
    p.tiles_t = (p.L + T_T - 1) / T_T;
    int span = 0, kmax = 1;
    for (int j = 0; j < njobs; ++j) {
        span = span > (p.job[j].K - 1) * p.job[j].dil ? span : (p.job[j].K - 1) * p.job[j].dil;
        kmax = kmax > p.job[j].K ? kmax : p.job[j].K;
    }
    SmemPlan sp;
    sp.AWs = T_T + span;
    sp.XW = sp.AWs + 12;
    sp.SW = 2 * sp.AWs + 10;
    sp.Kmax = kmax;
    size_t floats = (size_t)CK * sp.AWs + (size_t)CK * kmax * CO_T;
    if (ACT) floats += (size_t)CK * (sp.XW + sp.SW);
    const size_t bytes = floats * sizeof(float);
    auto kern = k_conv_simt<CO_T, T_T, RO, RT, ACT, MEAN3>;
    if (bytes > 48 * 1024) {
        if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes) != cudaSuccess)
            return -1;
    }
    dim3 grid(p.tiles_t * p.B, (p.Cout + CO_T - 1) / CO_T, njobs);
    kern<<<grid, (CO_T / RO) * (T_T / RT), bytes, s>>>(p, sp);
    return cudaPeekAtLastError() == cudaSuccess ? 1 : -1;
}

template <bool ACT, bool MEAN3>
int launch_conv_dispatch(const ConvParams& p, int njobs, cudaStream_t s) {
    if (p.Cout >= 64) return launch_conv_cfg<64, 64, 4, 4, ACT, MEAN3>(p, njobs, s);
    if (p.Cout >= 32) return launch_conv_cfg<32, 128, 4, 4, ACT, MEAN3>(p, njobs, s);
    if (p.Cout >= 16) return launch_conv_cfg<16, 256, 4, 4, ACT, MEAN3>(p, njobs, s);
    if (p.Cout >= 2) return launch_conv_cfg<8, 256, 2, 4, ACT, MEAN3>(p, njobs, s);
    return launch_conv_cfg<1, 256, 1, 1, ACT, MEAN3>(p, njobs, s);
}

template <int CO_T, int RO, int RT, int TX, int RMAX, bool MEAN3>
int launch_convT_cfg(const ConvTParams& p0, cudaStream_t s) {
    ConvTParams p = p0;
    constexpr int U = TX * RT;
    const int Lout = p.Lin * p.r;
    p.tiles_t = (Lout + p.r * U - 1) / (p.r * U);
    const int nmax = (p.K + p.r - 1) / p.r;
    const int IW = U + nmax + (p.r - 1 + p.pad) / p.r + 2;
    const size_t bytes = ((size_t)CK * IW + (size_t)CK * p.K * CO_T) * sizeof(float);
    auto kern = k_convT_simt<CO_T, RO, RT, TX, RMAX, MEAN3>;
    if (bytes > 48 * 1024) {
        if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes) != cudaSuccess)
            return -1;
    }
    dim3 grid(p.tiles_t * p.B, (p.Cout + CO_T - 1) / CO_T, 1);
    kern<<<grid, (CO_T / RO) * TX, bytes, s>>>(p);
    return cudaPeekAtLastError() == cudaSuccess ? 1 : -1;
}

}  // namespace

int launch_conv_simt(const ConvParams& p, int njobs, bool act, bool mean3, cudaStream_t s) {
    if (act) return mean3 ? launch_conv_dispatch<true, true>(p, njobs, s) : launch_conv_dispatch<true, false>(p, njobs, s);
    return mean3 ? launch_conv_dispatch<false, true>(p, njobs, s) : launch_conv_dispatch<false, false>(p, njobs, s);
}

template <int RMAX>
int launch_convT_rate(const ConvTParams& p, bool mean3, cudaStream_t s) {
    if (p.Cout >= 32) {
        return mean3 ? launch_convT_cfg<32, 4, 2, 32, RMAX, true>(p, s)
                     : launch_convT_cfg<32, 4, 2, 32, RMAX, false>(p, s);
    }
    return mean3 ? launch_convT_cfg<8, 1, 2, 32, RMAX, true>(p, s) : launch_convT_cfg<8, 1, 2, 32, RMAX, false>(p, s);
}

int launch_convT_simt(const ConvTParams& p, bool mean3, cudaStream_t s) {
    if (p.r < 1 || p.r > 8) return -1;
    if (p.r <= 2) return launch_convT_rate<2>(p, mean3, s);
    if (p.r <= 5) return launch_convT_rate<5>(p, mean3, s);
    return launch_convT_rate<8>(p, mean3, s);
}

// Pointwise (k = 1) conv with few input channels (dec_in_proj, 32 -> 2048): one thread per time
// sample holds the Cin inputs in registers and sweeps 16 output channels whose weights sit in
// shared memory (every lane reads the same weight: a broadcast).
constexpr int kPwCin = 64;
constexpr int kPwOut = 16;
constexpr int kPwThreads = 128;

__global__ void __launch_bounds__(kPwThreads) k_conv1x1(const ConvParams p) {
    __shared__ float ws[kPwCin][kPwOut];
    const ConvJob& J = p.job[0];
    const int L = p.L, Cin = p.Cin, Cout = p.Cout;
    const int tiles = (L + kPwThreads - 1) / kPwThreads;
    const int b = blockIdx.x / tiles;
    const int t = (blockIdx.x % tiles) * kPwThreads + threadIdx.x;
    const int o0 = blockIdx.y * kPwOut;
    // weights [Cin, 1, Cout]: every copy in flight at once
    for (int i = threadIdx.x; i < Cin * kPwOut; i += kPwThreads) {
        const int c = i / kPwOut, o = i % kPwOut;
        if (o0 + o < Cout) ptx::cp_async4(&ws[c][o], J.w + (size_t)c * Cout + o0 + o);
        else ws[c][o] = 0.f;
    }
    ptx::cp_async_commit();
    ptx::cp_async_wait_all();
    __syncthreads();
    if (t >= L) return;
    float z[kPwCin];
#pragma unroll
    for (int c = 0; c < kPwCin; ++c) z[c] = (c < Cin) ? __ldg(J.x0 + ((long long)b * Cin + c) * L + t) : 0.f;
    for (int o = 0; o < kPwOut && o0 + o < Cout; ++o) {
        float acc = 0.f;
#pragma unroll
        for (int c = 0; c < kPwCin; ++c)
            if (c < Cin) acc = fmaf(ws[c][o], z[c], acc);
        J.out[((long long)b * Cout + o0 + o) * L + t] = acc + __ldg(J.bias + o0 + o);
    }
}

int launch_conv1x1(const ConvParams& p, cudaStream_t s) {
    const ConvJob& J = p.job[0];
    if (J.K != 1 || J.pad != 0 || p.Cin < 1 || p.Cin > kPwCin || p.L < 1 || !J.bias) return -1;
    dim3 grid(((p.L + kPwThreads - 1) / kPwThreads) * p.B, (p.Cout + kPwOut - 1) / kPwOut);
    k_conv1x1<<<grid, kPwThreads, 0, s>>>(p);
    return cudaPeekAtLastError() == cudaSuccess ? 1 : -1;
}

int launch_mean3(const Mean3Params& p, cudaStream_t s) {
    const int threads = 256;
    long long blocks = (p.n / 4 + threads - 1) / threads;
    if (blocks < 1) blocks = 1;
    if (blocks > 148 * 16) blocks = 148 * 16;
    k_mean3<<<(unsigned)blocks, threads, 0, s>>>(p);
    return cudaPeekAtLastError() == cudaSuccess ? 1 : -1;
}

}  // namespace mh3a

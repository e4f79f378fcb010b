// act_math.cuh -- the anti-aliased SnakeBeta of one channel, register-blocked per lane (the
// standalone activation kernel), and the sine of SnakeBeta that the producer warps of the fused
// tensor-core AMP kernel share with it.
//
//   a = down2(snake(up2(x)))      (FastVideo "minimax_h3_audio_vae" page, `_activation1d`;
//                                  filter from `kaiser_sinc_filter1d`)
// up2: replicate-pad 5, stride-2 transposed conv with the 12 taps at gain 2, crop 15 per side;
// in polyphase form u[2m] = sum_q 2 f[2q+1] x[m+2-q], u[2m+1] = sum_q 2 f[2q] x[m+3-q];
// snake: s = u + sin^2(alpha u) / (beta + 1e-9); down2: a[t] = sum_j f[j] s[2t+j-5] with s
// replicate-padded (index clamped to [0, 2L)).
//
// A warp computes 32 RUN consecutive outputs of one channel, rows [tw, tw + 32 RUN): lane l owns
// rows tw + RUN l + [0, RUN).  It forms the 2 RUN SnakeBeta values at the 2x rate that belong to
// its rows in registers, receives the 5 + 5 halo values from its neighbour lanes by warp
// shuffles (the two values outside the warp's run come from lanes 0-9, one each), and decimates
// in registers.  The input window x[tw - 8, tw + 32 RUN + 8) sits in shared memory with 4 floats
// of padding after every 16 (skew), so that lanes reading their runs hit distinct banks.
#pragma once

#include <cuda_bf16.h>

#include "mh3a_internal.cuh"

namespace mh3a {
namespace actm {

__device__ __forceinline__ int clampi(int v, int lo, int hi) { return v < lo ? lo : (v > hi ? hi : v); }
__device__ __forceinline__ int skew(int i) { return i + ((i >> 4) << 2); }
// skewed size of a window of n floats
__host__ __device__ constexpr int skewed(int n) { return n + n / 16 * 4 + 4; }

// sin^2(alpha u) with the hardware sine.  Its argument error grows with |alpha u| as the fp32
// rounding of the product alpha u itself does (about |alpha u| 2^-24), so reducing the phase
// modulo pi first would not make the result more accurate.  Relative to the SnakeBeta output
// (of magnitude about |u|) both stay far below the 3xBF16 operand error (2^-17); the parity
// tests bound the end-to-end effect.
__device__ __forceinline__ float sin_sq_fast(float alpha, float u) {
    const float s = __sinf(alpha * u);
    return s * s;
}

// Two fp32 values -> packed bf16x2 (round to nearest even), first value in the low half.
__device__ __forceinline__ uint32_t pack2(float first, float second) {
    const __nv_bfloat162 v = __floats2bfloat162_rn(first, second);
    return *reinterpret_cast<const uint32_t*>(&v);
}

// Head/tail split of two values: heads packed in *h, tails (v - head) packed in *l.
__device__ __forceinline__ void split2(float a, float b, uint32_t* h, uint32_t* l) {
    const uint32_t hp = pack2(a, b);
    const float ha = __uint_as_float(hp << 16), hb = __uint_as_float(hp & 0xFFFF0000u);
    *h = hp;
    *l = pack2(a - ha, b - hb);
}

// SnakeBeta value j of a lane's window, n = 2 (tw + q0) - 5 + j, from xv[k] = x[tw + q0 - 8 + k]
// (j even: odd phase n = 2m + 1; j odd: even phase n = 2m).
template <int J>
__device__ __forceinline__ float snake_at(const ActFilter& f, const float* xv, float al, float ib) {
    float u = 0.f;
    if (J % 2 == 0) {
#pragma unroll
        for (int k = 0; k < 6; ++k) u = fmaf(f.up[2 * k], xv[8 + J / 2 - k], u);
    } else {
#pragma unroll
        for (int k = 0; k < 6; ++k) u = fmaf(f.up[2 * k + 1], xv[8 + (J - 1) / 2 - k], u);
    }
    return fmaf(sin_sq_fast(al, u), ib, u);
}

template <int J0, int J1>
__device__ __forceinline__ void snake_range(const ActFilter& f, const float* xv, float al, float ib, float* s) {
    if constexpr (J0 < J1) {
        s[J0] = snake_at<J0>(f, xv, al, ib);
        snake_range<J0 + 1, J1>(f, xv, al, ib, s);
    }
}

// SnakeBeta values J and J + 1 (J even) as one packed pair: the two upsampled values, then
// alpha u, sin, its square and the final fma as fp32x2 operations where the hardware has them.
template <int J>
__device__ __forceinline__ void snake_pair(const ActFilter& f, const float* xv, float2 al2, float2 ib2, float* s) {
    static_assert(J % 2 == 0, "pairs start on even indices");
    // J even reads the odd phase taps f[2k], J + 1 the even phase taps f[2k + 1], both at the
    // same input sample: one packed fma per tap pair
    float2 u2 = make_float2(0.f, 0.f);
#pragma unroll
    for (int k = 0; k < 6; ++k) {
        const float xk = xv[8 + J / 2 - k];
        u2 = __ffma2_rn(make_float2(f.up[2 * k], f.up[2 * k + 1]), make_float2(xk, xk), u2);
    }
    const float2 t2 = __fmul2_rn(al2, u2);
    const float2 sn = make_float2(__sinf(t2.x), __sinf(t2.y));
    const float2 r2 = __ffma2_rn(__fmul2_rn(sn, sn), ib2, u2);
    s[J] = r2.x;
    s[J + 1] = r2.y;
}

template <int J0, int J1>
__device__ __forceinline__ void snake_pairs(const ActFilter& f, const float* xv, float2 al2, float2 ib2, float* s) {
    if constexpr (J0 < J1) {
        snake_pair<J0>(f, xv, al2, ib2, s);
        snake_pairs<J0 + 2, J1>(f, xv, al2, ib2, s);
    }
}

// Outputs a[k] = act(x)[tw + RUN lane + k] of one channel (RUN even).  xs: the skewed window,
// logical index i <-> x[tw - 8 + i], at least 32 RUN + 16 floats, staged with the sequence's
// replicate padding when EDGE.  EDGE also substitutes the end values for SnakeBeta positions
// outside [0, 2L); rows outside [0, L) are the caller's to discard.  Called by all 32 lanes.
template <int RUN, bool EDGE>
__device__ __forceinline__ void act_lane(const ActFilter& f, const float* xs, float al, float ib, int tw, int L,
                                         float (&a)[RUN]) {
    static_assert(RUN % 2 == 0, "lane runs start on 8-byte boundaries");
    constexpr int NS = 2 * RUN + 10;                          // SnakeBeta values a lane reads
    constexpr int NXV = (RUN % 4 == 0) ? (RUN + 11 + 3) / 4 * 4 : (RUN + 11 + 1) / 2 * 2;
    const int lane = threadIdx.x & 31;
    const int q0 = RUN * lane;
    float xv[NXV];
    if constexpr (RUN % 4 == 0) {
#pragma unroll
        for (int k = 0; k < NXV / 4; ++k) {
            const float4 v = *reinterpret_cast<const float4*>(xs + skew(q0 + 4 * k));
            xv[4 * k] = v.x;
            xv[4 * k + 1] = v.y;
            xv[4 * k + 2] = v.z;
            xv[4 * k + 3] = v.w;
        }
    } else {
#pragma unroll
        for (int k = 0; k < NXV / 2; ++k) {
            const float2 v = *reinterpret_cast<const float2*>(xs + skew(q0 + 2 * k));
            xv[2 * k] = v.x;
            xv[2 * k + 1] = v.y;
        }
    }
    float s[NS];
    // the lane's own 2 RUN values, s[5 .. 2 RUN + 4]: the interior pairs (s[2m], s[2m + 1]) go
    // through SnakeBeta as packed fp32x2 operations (the same rounding as the scalar form)
    s[5] = snake_at<5>(f, xv, al, ib);
    snake_pairs<6, 2 * RUN + 4>(f, xv, make_float2(al, al), make_float2(ib, ib), s);
    s[2 * RUN + 4] = snake_at<2 * RUN + 4>(f, xv, al, ib);
    // The 5 values left of lane 0's run and right of lane 31's run: lanes 0-4 and 5-9 form one
    // each (value j of lane 0's window, resp. j = 2 RUN + 5 .. 2 RUN + 9 of lane 31's).
    float hv = 0.f;
    if (lane < 10) {
        const int j = (lane < 5) ? lane : lane + 2 * RUN;
        const int i0 = ((lane < 5) ? 0 : RUN * 31) + 8 + (j >> 1);
        const int par = j & 1;
        float u = 0.f;
#pragma unroll
        for (int k = 0; k < 6; ++k) u = fmaf(f.up[2 * k + par], xs[skew(i0 - k)], u);
        hv = fmaf(sin_sq_fast(al, u), ib, u);
    }
#pragma unroll
    for (int j = 0; j < 5; ++j) {
        const float from_left = __shfl_up_sync(0xffffffffu, s[j + 2 * RUN], 1);
        const float from_right = __shfl_down_sync(0xffffffffu, s[j + 5], 1);
        const float h = __shfl_sync(0xffffffffu, hv, (lane == 31) ? j + 5 : j);
        s[j] = (lane == 0) ? h : from_left;
        s[j + 5 + 2 * RUN] = (lane == 31) ? h : from_right;
    }
    if (EDGE) {
        // replicate padding at the 2x rate: n < 0 takes s(0), n > 2L - 1 takes s(2L - 1)
        const int n0 = 2 * (tw + q0) - 5;
        const int j0 = -n0, je = 2 * L - 1 - n0;
        float sf = s[0], sl = s[NS - 1];
#pragma unroll
        for (int j = 0; j < NS; ++j) {
            sf = (j == j0) ? s[j] : sf;
            sl = (j == je) ? s[j] : sl;
        }
#pragma unroll
        for (int j = 0; j < NS; ++j) s[j] = (j < j0) ? sf : ((j > je) ? sl : s[j]);
    }
    // decimation: even and odd taps as the two halves of packed fp32x2 FMAs on the pairs
    // (s[2m], s[2m + 1]), then one add
#pragma unroll
    for (int i = 0; i < RUN; ++i) {
        float2 v = make_float2(0.f, 0.f);
#pragma unroll
        for (int q = 0; q < kFilterTaps / 2; ++q)
            v = __ffma2_rn(make_float2(f.down[2 * q], f.down[2 * q + 1]), make_float2(s[2 * i + 2 * q], s[2 * i + 2 * q + 1]), v);
        a[i] = v.x + v.y;
    }
}

}  // namespace actm
}  // namespace mh3a

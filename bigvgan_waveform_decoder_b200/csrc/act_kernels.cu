// act_kernels.cu -- the anti-aliased SnakeBeta of the AMP residual blocks as a standalone
// CUDA-core kernel that writes the tensor-core A operand (3xBF16 head and tail) to memory.
//
//   a = down2(snake(up2(x)))      (FastVideo "minimax_h3_audio_vae" page, `_activation1d`;
//                                  filter from `kaiser_sinc_filter1d`)
// up2: replicate-pad 5, stride-2 transposed conv with the 12 taps at gain 2, crop 15 per side;
// in polyphase form u[2m] = sum_q 2 f[2q+1] x[m+2-q], u[2m+1] = sum_q 2 f[2q] x[m+3-q];
// snake: s = u + sin^2(alpha u) / (beta + 1e-9); down2: a[t] = sum_j f[j] s[2t+j-5] with s
// replicate-padded (index clamped to [0, 2L)).
//
// Output layout (per batch item b and channel group g of 8): rows of 16 bytes, one row per time
// sample, holding the 8 channels' bf16 values -- the no-swizzle K-major core-matrix layout the
// tensor-core kernel copies straight into shared memory.  Rows [-pad_l, 0) and [L, L + pad_r)
// are written as zeros: they are the conv's zero padding, so the GEMM never special-cases the
// sequence ends.  Heads and tails go to separate arrays.
#include <cuda_bf16.h>

#include "act_kernels.cuh"

namespace mh3a {
namespace {

constexpr int TT = 384;       // output rows per block (static shared memory stays under 48 KB)
constexpr int NT_ACT = 256;   // threads per block (8 warps: one per channel of the group)

__device__ __forceinline__ int clampi(int v, int lo, int hi) { return v < lo ? lo : (v > hi ? hi : v); }

// sin^2(alpha u): Cody-Waite reduction modulo pi, then the hardware sine on [-pi/2, pi/2]
// (absolute error near 2^-21, far below the 3xBF16 operand error).
// The nearest integer k = rint(v / pi) is formed by adding and subtracting 1.5 * 2^23 in
// round-to-nearest fp32 arithmetic, exact for |v / pi| < 2^22.
__device__ __forceinline__ float sin_sq_fast(float alpha, float u) {
    const float kInvPi = 0.318309886183790671538f;
    const float kPiHi = 3.14159274101257324219f;
    const float kPiLo = -8.74227800037248297e-08f;
    const float kRound = 12582912.0f;  // 1.5 * 2^23
    const float v = alpha * u;
    const float k = __fsub_rn(__fmaf_rn(v, kInvPi, kRound), kRound);
    float r = fmaf(-k, kPiHi, v);
    r = fmaf(-k, kPiLo, r);
    const float s = __sinf(r);
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

// grid: x = row tiles over [-pad_l, L + pad_r), y = B * C / 8 (item, group), z = job
__global__ void __launch_bounds__(NT_ACT) k_act_split(const ActParams p) {
    __shared__ float xs[8][TT + 16];
    __shared__ __align__(16) float sw[8][2 * TT + 12];
    const ActJob& J = p.job[blockIdx.z];
    const int C = p.C, L = p.L;
    const int ngroups = C / 8;
    const int b = blockIdx.y / ngroups, g = blockIdx.y % ngroups;
    const int t0 = -p.pad_l + blockIdx.x * TT;           // first output row of the tile
    const int rows = min(TT, L + p.pad_r - t0);
    const int tid = threadIdx.x, c = tid >> 5, lane = tid & 31;
    const long long Lpad = (long long)L + p.pad_l + p.pad_r;
    uint4* ohi = reinterpret_cast<uint4*>(J.a_hi) + ((long long)b * ngroups + g) * Lpad + p.pad_l;
    uint4* olo = reinterpret_cast<uint4*>(J.a_lo) + ((long long)b * ngroups + g) * Lpad + p.pad_l;

    const bool any_inside = t0 < L && t0 + rows > 0;
    if (any_inside) {
        const int xs_start = t0 - 6;
        const int XW = rows + 12;
        const float* xrow = J.x + ((long long)b * C + g * 8 + c) * L;
        for (int q = lane; q < XW; q += 32) xs[c][q] = __ldg(xrow + clampi(xs_start + q, 0, L - 1));
        __syncwarp();
        // SnakeBeta at the 2x rate over n in [2 t0 - 5, 2 (t0 + rows) + 5): a lane takes one
        // input position m and forms both phases; positions past either end repeat the end.
        const float al = __ldg(J.alpha + g * 8 + c), ib = __ldg(J.inv_beta + g * 8 + c);
        const int n_start = 2 * t0 - 5, SW = 2 * rows + 10;
        const float* xr0 = &xs[c][0] - xs_start;
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
            const float se = fmaf(sin_sq_fast(al, ue), ib, ue);
            const float so = fmaf(sin_sq_fast(al, uo), ib, uo);
            const int ie = 2 * m - n_start;
            if (ie >= 0 && ie < SW) sw[c][ie] = (m > L - 1) ? so : se;
            if (ie + 1 >= 0 && ie + 1 < SW) sw[c][ie + 1] = (m < 0) ? se : so;
        }
    }
    __syncthreads();
    // decimate, zero outside [0, L), split into head and tail, one 16-byte row per thread
    for (int q = tid; q < rows; q += NT_ACT) {
        const int t = t0 + q;
        float a[8];
        if (t >= 0 && t < L) {
#pragma unroll
            for (int cc = 0; cc < 8; ++cc) {
                const float2* sr = reinterpret_cast<const float2*>(&sw[cc][2 * q]);
                float v = 0.f;
#pragma unroll
                for (int j = 0; j < kFilterTaps / 2; ++j) {
                    const float2 s2 = sr[j];
                    v = fmaf(p.filt.down[2 * j], s2.x, v);
                    v = fmaf(p.filt.down[2 * j + 1], s2.y, v);
                }
                a[cc] = v;
            }
        } else {
#pragma unroll
            for (int cc = 0; cc < 8; ++cc) a[cc] = 0.f;
        }
        uint4 hv, lv;
        split2(a[0], a[1], &hv.x, &lv.x);
        split2(a[2], a[3], &hv.y, &lv.y);
        split2(a[4], a[5], &hv.z, &lv.z);
        split2(a[6], a[7], &hv.w, &lv.w);
        ohi[t] = hv;
        olo[t] = lv;
    }
}

}  // namespace

int launch_act_split(const ActParams& p, int njobs, cudaStream_t s) {
    if (p.C % 8 != 0 || p.L < 1 || p.pad_l < 0 || p.pad_r < 0) return -1;
    const int total = p.L + p.pad_l + p.pad_r;
    dim3 grid((total + TT - 1) / TT, p.B * (p.C / 8), njobs);
    k_act_split<<<grid, NT_ACT, 0, s>>>(p);
    return cudaPeekAtLastError() == cudaSuccess ? 1 : -1;
}

}  // namespace mh3a

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
        // u at both phases of position mc from x[mc-3 .. mc+3] (xv[k] = x[mc + k - 3 + off])
        auto up2 = [&](const float* xv, int off, float& ue, float& uo) {
            ue = 0.f;
            uo = 0.f;
#pragma unroll
            for (int k = 0; k < 6; ++k) {
                ue = fmaf(p.filt.up[2 * k + 1], xv[off + 5 - k], ue);
                uo = fmaf(p.filt.up[2 * k], xv[off + 6 - k], uo);
            }
        };
        // A lane takes two consecutive input positions; inside the sequence they share eight
        // inputs x[m0-3 .. m0+4].  At the ends each position is clamped on its own.
        for (int m0 = m_lo + 2 * lane; m0 <= m_hi; m0 += 64) {
            float ue[2], uo[2];
            if (m0 >= 0 && m0 + 1 <= L - 1) {
                float xv[8];
#pragma unroll
                for (int k = 0; k < 8; ++k) xv[k] = xr0[m0 + k - 3];
                up2(xv, 0, ue[0], uo[0]);
                up2(xv, 1, ue[1], uo[1]);
            } else {
#pragma unroll
                for (int i = 0; i < 2; ++i) {
                    const int mc = clampi(m0 + i, 0, L - 1);
                    float xv[7];
#pragma unroll
                    for (int k = 0; k < 7; ++k) xv[k] = xr0[mc + k - 3];
                    up2(xv, 0, ue[i], uo[i]);
                }
            }
#pragma unroll
            for (int i = 0; i < 2; ++i) {
                const int m = m0 + i;
                if (m > m_hi) break;
                const float se = fmaf(sin_sq_fast(al, ue[i]), ib, ue[i]);
                const float so = fmaf(sin_sq_fast(al, uo[i]), ib, uo[i]);
                const int ie = 2 * m - n_start;
                if (ie >= 0 && ie < SW) sw[c][ie] = (m > L - 1) ? so : se;
                if (ie + 1 >= 0 && ie + 1 < SW) sw[c][ie + 1] = (m < 0) ? se : so;
            }
        }
    }
    __syncthreads();
    // decimate, zero outside [0, L), split into head and tail: 2 rows x 4 channels per item
    const int npairs = (rows + 1) >> 1;
    for (int it = tid; it < 2 * npairs; it += NT_ACT) {
        const int rp = it >> 1, hf = it & 1;
        const int q0 = 2 * rp;
        float a0[4], a1[4];
        if (any_inside) {
#pragma unroll
            for (int cc = 0; cc < 4; ++cc) {
                const float2* sr = reinterpret_cast<const float2*>(&sw[4 * hf + cc][2 * q0]);
                float s[14];
#pragma unroll
                for (int j = 0; j < 7; ++j) {
                    const float2 s2 = sr[j];
                    s[2 * j] = s2.x;
                    s[2 * j + 1] = s2.y;
                }
                float v0 = 0.f, v1 = 0.f;
#pragma unroll
                for (int j = 0; j < kFilterTaps; ++j) {
                    v0 = fmaf(p.filt.down[j], s[j], v0);
                    v1 = fmaf(p.filt.down[j], s[j + 2], v1);
                }
                a0[cc] = v0;
                a1[cc] = v1;
            }
        }
#pragma unroll
        for (int r = 0; r < 2; ++r) {
            const int q = q0 + r;
            if (q >= rows) break;
            const int t = t0 + q;
            const bool in = t >= 0 && t < L;
            float v[4];
#pragma unroll
            for (int cc = 0; cc < 4; ++cc) v[cc] = in ? (r == 0 ? a0[cc] : a1[cc]) : 0.f;
            uint2 hv, lv;
            split2(v[0], v[1], &hv.x, &lv.x);
            split2(v[2], v[3], &hv.y, &lv.y);
            reinterpret_cast<uint2*>(ohi + t)[hf] = hv;
            reinterpret_cast<uint2*>(olo + t)[hf] = lv;
        }
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

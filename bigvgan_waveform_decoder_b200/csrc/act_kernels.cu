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
//
// A block covers TT = 512 output rows of one channel group.  Every lane owns 16 consecutive
// outputs of one channel, forms the 32 SnakeBeta values at the 2x rate that belong to them in
// registers, receives the 5 + 5 halo values from its neighbour lanes by warp shuffles, and
// decimates in registers; a shared-memory transpose then packs rows of 8 channels.  Tiles that
// touch a sequence end clamp the input index and substitute the end values at the 2x rate
// (the replicate paddings); tiles wholly outside the sequence only write zero rows.
#include <cuda_bf16.h>

#include "act_kernels.cuh"
#include "tc_ptx.cuh"

namespace mh3a {
namespace {

constexpr int TT = 512;                   // output rows per block
constexpr int RUN = 16;                   // outputs per lane (TT = 32 RUN)
constexpr int NT_ACT = 256;               // threads per block (8 warps: one per channel)
constexpr int NS = 2 * RUN + 10;          // SnakeBeta values one lane's decimation reads
// Shared layout: per channel a window of x and a row of outputs, each with 4 floats
// of padding after every 16 so that lanes reading 16-float runs hit distinct banks.
constexpr int XF = TT + 16;               // x[t0 - 8, t0 + TT + 8)
constexpr int XF_P = XF + XF / 16 * 4;
constexpr int TF_P = TT + TT / 16 * 4;
constexpr int SMEM_FLOATS = 8 * (XF_P + TF_P);

__device__ __forceinline__ int clampi(int v, int lo, int hi) { return v < lo ? lo : (v > hi ? hi : v); }
__device__ __forceinline__ int skew(int i) { return i + ((i >> 4) << 2); }

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


// SnakeBeta value j of a lane's window, n = 2 (t0 + q0) - 5 + j, from xv[k] = x[t0 + q0 - 8 + k]
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

// One tile: rows [t0, t0 + TT).  EDGE = false requires 8 <= t0 and t0 + TT + 8 <= L, so that
// neither the input window nor the 2x-rate SnakeBeta window reaches past a sequence end.  EDGE
// tiles clamp the input index (the replicate padding of x), replace SnakeBeta values outside
// [0, 2L) by the end values (the replicate padding at the 2x rate), and write zero rows
// outside [0, L).
template <bool EDGE>
__device__ __forceinline__ void act_tile(const ActParams& p, const ActJob& J, float* buf, int b, int g, int t0,
                                         int rows, uint4* ohi, uint4* olo) {
    const int L = p.L;
    const int tid = threadIdx.x, c = tid >> 5, lane = tid & 31;
    float* xs = buf + c * XF_P;
    float* T = buf + 8 * XF_P;   // [8][TF_P] outputs, skewed
    const float* xrow = J.x + ((long long)b * p.C + g * 8 + c) * L;
    // all of the window's loads in flight at once (asynchronous copies straight to shared);
    // skew(lane + 32 k) = skew(lane) + 40 k
    {
        float* dst = xs + skew(lane);
#pragma unroll
        for (int k = 0; k < (XF + 31) / 32; ++k) {
            const int i = lane + 32 * k;
            if (i < XF) {
                int src = t0 - 8 + i;
                if (EDGE) src = clampi(src, 0, L - 1);
                ptx::cp_async4(dst + 40 * k, xrow + src);
            }
        }
    }
    ptx::cp_async_commit();
    ptx::cp_async_wait_all();
    __syncwarp();
    const float al = __ldg(J.alpha + g * 8 + c), ib = __ldg(J.inv_beta + g * 8 + c);
    const int q0 = RUN * lane;
    float xv[32];
#pragma unroll
    for (int k = 0; k < 8; ++k) {
        const float4 v = *reinterpret_cast<const float4*>(xs + skew(q0 + 4 * k));
        xv[4 * k] = v.x;
        xv[4 * k + 1] = v.y;
        xv[4 * k + 2] = v.z;
        xv[4 * k + 3] = v.w;
    }
    float s[NS];
    snake_range<5, 5 + 2 * RUN>(p.filt, xv, al, ib, s);     // the lane's own 2 RUN values
    // The 5 values left of lane 0's run and right of lane 31's run: lanes 0-4 and 5-9 form one
    // each (value j of lane 0's window, resp. j = 37 .. 41 of lane 31's), from the same taps.
    float hv = 0.f;
    if (lane < 10) {
        const int j = (lane < 5) ? lane : lane + 2 * RUN;
        const int i0 = ((lane < 5) ? 0 : RUN * 31) + 8 + (j >> 1);
        const int par = j & 1;
        float u = 0.f;
#pragma unroll
        for (int k = 0; k < 6; ++k) u = fmaf(p.filt.up[2 * k + par], xs[skew(i0 - k)], u);
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
        const int n0 = 2 * (t0 + q0) - 5;
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
    float a[RUN];
#pragma unroll
    for (int i = 0; i < RUN; ++i) {
        float v = 0.f;
#pragma unroll
        for (int j = 0; j < kFilterTaps; ++j) v = fmaf(p.filt.down[j], s[2 * i + j], v);
        a[i] = v;
    }
    float* trow = T + c * TF_P;
#pragma unroll
    for (int k = 0; k < RUN / 4; ++k)
        *reinterpret_cast<float4*>(trow + skew(q0 + 4 * k)) = make_float4(a[4 * k], a[4 * k + 1], a[4 * k + 2], a[4 * k + 3]);
    __syncthreads();
    // rows of 8 channels: skew(q + 256) = skew(q) + 320
#pragma unroll
    for (int r = 0; r < TT / NT_ACT; ++r) {
        const int q = tid + r * NT_ACT;
        if (EDGE && q >= rows) break;
        const int qs = skew(tid) + r * (NT_ACT + NT_ACT / 4);
        const int t = t0 + q;
        float v[8];
#pragma unroll
        for (int cc = 0; cc < 8; ++cc) v[cc] = T[cc * TF_P + qs];
        if (EDGE && (t < 0 || t >= L)) {
#pragma unroll
            for (int cc = 0; cc < 8; ++cc) v[cc] = 0.f;
        }
        uint4 hv4, lv4;
        split2(v[0], v[1], &hv4.x, &lv4.x);
        split2(v[2], v[3], &hv4.y, &lv4.y);
        split2(v[4], v[5], &hv4.z, &lv4.z);
        split2(v[6], v[7], &hv4.w, &lv4.w);
        ohi[t] = hv4;
        olo[t] = lv4;
    }
}

// grid: x = row tiles over [-pad_l, L + pad_r), y = B * C / 8 (item, group), z = job
__global__ void __launch_bounds__(NT_ACT) k_act_split(const ActParams p) {
    __shared__ __align__(16) float buf[SMEM_FLOATS];
    const ActJob& J = p.job[blockIdx.z];
    const int L = p.L;
    const int ngroups = p.C / 8;
    const int b = blockIdx.y / ngroups, g = blockIdx.y % ngroups;
    const int t0 = -p.pad_l + blockIdx.x * TT;           // first output row of the tile
    const int rows = min(TT, L + p.pad_r - t0);
    const long long Lpad = (long long)L + p.pad_l + p.pad_r;
    uint4* ohi = reinterpret_cast<uint4*>(J.a_hi) + ((long long)b * ngroups + g) * Lpad + p.pad_l;
    uint4* olo = reinterpret_cast<uint4*>(J.a_lo) + ((long long)b * ngroups + g) * Lpad + p.pad_l;
    if (t0 >= 8 && t0 + TT + 8 <= L) {
        act_tile<false>(p, J, buf, b, g, t0, TT, ohi, olo);
    } else if (t0 < L && t0 + rows > 0) {
        act_tile<true>(p, J, buf, b, g, t0, rows, ohi, olo);
    } else {
        // rows entirely outside [0, L): zeros (the conv's padding)
        const uint4 z = make_uint4(0u, 0u, 0u, 0u);
        for (int q = threadIdx.x; q < rows; q += NT_ACT) {
            ohi[t0 + q] = z;
            olo[t0 + q] = z;
        }
    }
}

// Plain head/tail split (no activation) into the same row layout, of x0 or of the mean
// (x0 + x1 + x2) / 3 of three block outputs.  grid: x = row tiles of NT_ACT, y = B * C / 8.
__global__ void __launch_bounds__(NT_ACT) k_split_rows(const SplitParams p) {
    const int L = p.L, ngroups = p.C / 8;
    const int b = blockIdx.y / ngroups, g = blockIdx.y % ngroups;
    const int t = -p.pad_l + blockIdx.x * NT_ACT + threadIdx.x;
    if (t >= L + p.pad_r) return;
    const long long Lpad = (long long)L + p.pad_l + p.pad_r;
    const long long row = ((long long)b * ngroups + g) * Lpad + p.pad_l + t;
    float v[8];
    if (t >= 0 && t < L) {
        const long long base = ((long long)b * p.C + g * 8) * L + t;
#pragma unroll
        for (int c = 0; c < 8; ++c) {
            const long long i = base + (long long)c * L;
            v[c] = p.x1 ? (__ldg(p.x0 + i) + __ldg(p.x1 + i) + __ldg(p.x2 + i)) / 3.0f : __ldg(p.x0 + i);
        }
    } else {
#pragma unroll
        for (int c = 0; c < 8; ++c) v[c] = 0.f;
    }
    uint4 hv, lv;
    split2(v[0], v[1], &hv.x, &lv.x);
    split2(v[2], v[3], &hv.y, &lv.y);
    split2(v[4], v[5], &hv.z, &lv.z);
    split2(v[6], v[7], &hv.w, &lv.w);
    reinterpret_cast<uint4*>(p.a_hi)[row] = hv;
    reinterpret_cast<uint4*>(p.a_lo)[row] = lv;
}

}  // namespace

int launch_split_rows(const SplitParams& p, cudaStream_t s) {
    if (p.C % 8 != 0 || p.L < 1 || p.pad_l < 0 || p.pad_r < 0 || !p.x0) return -1;
    if ((p.x1 == nullptr) != (p.x2 == nullptr)) return -1;
    const int total = p.L + p.pad_l + p.pad_r;
    dim3 grid((total + NT_ACT - 1) / NT_ACT, p.B * (p.C / 8));
    k_split_rows<<<grid, NT_ACT, 0, s>>>(p);
    return cudaPeekAtLastError() == cudaSuccess ? 1 : -1;
}

int launch_act_split(const ActParams& p, int njobs, cudaStream_t s) {
    if (p.C % 8 != 0 || p.L < 1 || p.pad_l < 0 || p.pad_r < 0) return -1;
    const int total = p.L + p.pad_l + p.pad_r;
    dim3 grid((total + TT - 1) / TT, p.B * (p.C / 8), njobs);
    k_act_split<<<grid, NT_ACT, 0, s>>>(p);
    return cudaPeekAtLastError() == cudaSuccess ? 1 : -1;
}

}  // namespace mh3a

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
#include "act_math.cuh"
#include "tc_ptx.cuh"

namespace mh3a {
namespace {

constexpr int TT = 512;                   // output rows per block
constexpr int RUN = 16;                   // outputs per lane (TT = 32 RUN)
constexpr int NT_ACT = 256;               // threads per block (8 warps: one per channel)
// Shared layout: per channel a window of x and a row of outputs, each with 4 floats
// of padding after every 16 so that lanes reading 16-float runs hit distinct banks.
constexpr int XF = TT + 16;               // x[t0 - 8, t0 + TT + 8)
constexpr int XF_P = XF + XF / 16 * 4;
constexpr int TF_P = TT + TT / 16 * 4;
constexpr int SMEM_FLOATS = 8 * (XF_P + TF_P);

using actm::clampi;
using actm::skew;
using actm::split2;

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
    // all of the window's loads in flight at once (asynchronous copies straight to shared)
    if (!EDGE && (reinterpret_cast<uintptr_t>(xrow + t0 - 8) & 15) == 0) {
        // 16-byte copies (the window starts on a 16-byte boundary; a skewed group of 4 floats
        // stays contiguous and 16-byte aligned in shared memory).  Piece k of a lane is float
        // 4 lane + 128 k of the window, at skew(4 lane) + 160 k in shared memory.
        float* dst = xs + skew(4 * lane);
        const float* src = xrow + t0 - 8 + 4 * lane;
#pragma unroll
        for (int k = 0; k < (XF / 4 + 31) / 32; ++k) {
            if (4 * lane + 128 * k < XF) ptx::cp_async16(dst + 160 * k, src + 128 * k);
        }
    } else {
        // skew(lane + 32 k) = skew(lane) + 40 k
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
    float a[RUN];
    actm::act_lane<RUN, EDGE>(p.filt, xs, al, ib, t0, L, a);
    float* trow = T + c * TF_P;
#pragma unroll
    for (int k = 0; k < RUN / 4; ++k)
        *reinterpret_cast<float4*>(trow + skew(q0 + 4 * k)) = make_float4(a[4 * k], a[4 * k + 1], a[4 * k + 2], a[4 * k + 3]);
    __syncthreads();
    // rows of 8 channels: skew(q + 256) = skew(q) + 320
    ohi += t0 + tid;
    olo += t0 + tid;
    const int qs0 = skew(tid);
#pragma unroll
    for (int r = 0; r < TT / NT_ACT; ++r) {
        const int q = tid + r * NT_ACT;
        if (EDGE && q >= rows) break;
        const int qs = qs0 + r * (NT_ACT + NT_ACT / 4);
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
        ohi[r * NT_ACT] = hv4;
        olo[r * NT_ACT] = lv4;
    }
}

// grid: x = row tiles over [-pad_l, L + pad_r), y = B * C / 8 (item, group), z = job.  With the
// packed fp32x2 SnakeBeta and decimation, four blocks per SM at 64 registers (no spills) issue
// slightly better than five at 48 (which spill a few registers to L1).
__global__ void __launch_bounds__(NT_ACT, 4) k_act_split(const ActParams p) {
    ptx::grid_dep_wait();     // launched as a programmatic dependent (see launch_dependent)
    ptx::grid_dep_launch();
    __shared__ __align__(16) float buf[SMEM_FLOATS];
    const ActJob& J = p.job[blockIdx.z];
    const int L = p.L;
    const int ngroups = p.C / 8;
    // channel groups per item are a power of two at every stage width: shift and mask
    const int b = p.g_log2 >= 0 ? (int)(blockIdx.y >> p.g_log2) : (int)blockIdx.y / ngroups;
    const int g = (int)blockIdx.y - b * ngroups;
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

// Input value of channel row `ci` (index into [B, C, L]) in the form the split takes.  The
// inputs (conv_pre's partial outputs, a stage's block outputs) are read here for the last time,
// so the loads are streaming (evict-first): measured 5 us less per decode over the seven splits.
__device__ __forceinline__ float split_in(const SplitParams& p, long long ci) {
    if (p.x3) return ((__ldcs(p.x0 + ci) + __ldcs(p.x1 + ci)) + __ldcs(p.x2 + ci)) + __ldcs(p.x3 + ci);
    if (p.x1) return (__ldcs(p.x0 + ci) + __ldcs(p.x1 + ci) + __ldcs(p.x2 + ci)) * (1.0f / 3.0f);
    return __ldcs(p.x0 + ci);
}

__device__ __forceinline__ float2 split_in2(const SplitParams& p, long long ci) {
    const float2 a = __ldcs(reinterpret_cast<const float2*>(p.x0 + ci));
    if (!p.x1) return a;
    const float2 b = __ldcs(reinterpret_cast<const float2*>(p.x1 + ci));
    const float2 c = __ldcs(reinterpret_cast<const float2*>(p.x2 + ci));
    if (p.x3) {
        const float2 d = __ldcs(reinterpret_cast<const float2*>(p.x3 + ci));
        return make_float2(((a.x + b.x) + c.x) + d.x, ((a.y + b.y) + c.y) + d.y);
    }
    return make_float2((a.x + b.x + c.x) * (1.0f / 3.0f), (a.y + b.y + c.y) * (1.0f / 3.0f));
}

__device__ __forceinline__ void store_row(const SplitParams& p, long long row, const float (&v)[8]) {
    uint4 hv, lv;
    split2(v[0], v[1], &hv.x, &lv.x);
    split2(v[2], v[3], &hv.y, &lv.y);
    split2(v[4], v[5], &hv.z, &lv.z);
    split2(v[6], v[7], &hv.w, &lv.w);
    reinterpret_cast<uint4*>(p.a_hi)[row] = hv;
    reinterpret_cast<uint4*>(p.a_lo)[row] = lv;
}

// Plain head/tail split (no activation) into the same row layout, of x0, of the mean
// (x0 + x1 + x2) / 3 of three block outputs, or of the sum of four partial outputs.  grid: x =
// tiles of 2 NT_ACT rows (two adjacent rows per thread, read as float2 where both lie inside an
// even-length sequence), y = B * C / 8.
__global__ void __launch_bounds__(NT_ACT) k_split_rows(const SplitParams p) {
    ptx::grid_dep_wait();     // launched as a programmatic dependent (see launch_dependent)
    ptx::grid_dep_launch();
    const int L = p.L, ngroups = p.C / 8;
    const int b = blockIdx.y / ngroups, g = blockIdx.y % ngroups;
    const int t = -p.pad_l + 2 * (blockIdx.x * NT_ACT + threadIdx.x);   // the thread's first row
    if (t >= L + p.pad_r) return;
    const long long Lpad = (long long)L + p.pad_l + p.pad_r;
    const long long row = ((long long)b * ngroups + g) * Lpad + p.pad_l + t;
    const long long base = ((long long)b * p.C + g * 8) * L;
    const bool second = t + 1 < L + p.pad_r;
    float v0[8], v1[8];
    const uintptr_t align = reinterpret_cast<uintptr_t>(p.x0) | reinterpret_cast<uintptr_t>(p.x1) |
                            reinterpret_cast<uintptr_t>(p.x2) | reinterpret_cast<uintptr_t>(p.x3);
    if ((L % 2 == 0) && (p.pad_l % 2 == 0) && (align & 7) == 0 && t >= 0 && t + 1 < L) {
#pragma unroll
        for (int c = 0; c < 8; ++c) {
            const float2 v = split_in2(p, base + (long long)c * L + t);
            v0[c] = v.x;
            v1[c] = v.y;
        }
    } else {
#pragma unroll
        for (int c = 0; c < 8; ++c) {
            v0[c] = (t >= 0 && t < L) ? split_in(p, base + (long long)c * L + t) : 0.f;
            v1[c] = (t + 1 >= 0 && t + 1 < L) ? split_in(p, base + (long long)c * L + t + 1) : 0.f;
        }
    }
    store_row(p, row, v0);
    if (second) store_row(p, row + 1, v1);
}

// grid: x = row tiles of NT_ACT, y = B * C / 8.  The group's 8 x Cz weights and 8 biases sit in
// shared memory (read back as broadcasts); every thread forms one row of 8 channels.
__global__ void __launch_bounds__(NT_ACT) k_proj_split(const ProjSplitParams p) {
    ptx::grid_dep_wait();     // launched as a programmatic dependent (see launch_dependent)
    ptx::grid_dep_launch();
    __shared__ __align__(16) float ws[kProjMaxCz][8];
    __shared__ float bs[8];
    const int L = p.L, ngroups = p.C / 8, Cz = p.Cz;
    const int b = blockIdx.y / ngroups, g = blockIdx.y % ngroups;
    for (int i = threadIdx.x; i < Cz * 8; i += NT_ACT) ws[i >> 3][i & 7] = __ldg(p.w + (size_t)(i >> 3) * p.C + g * 8 + (i & 7));
    if (threadIdx.x < 8) bs[threadIdx.x] = __ldg(p.bias + g * 8 + threadIdx.x);
    __syncthreads();
    const int t = -p.pad_l + blockIdx.x * NT_ACT + threadIdx.x;
    if (t >= L + p.pad_r) return;
    const long long Lpad = (long long)L + p.pad_l + p.pad_r;
    const long long row = ((long long)b * ngroups + g) * Lpad + p.pad_l + t;
    float v[8];
    if (t >= 0 && t < L) {
#pragma unroll
        for (int o = 0; o < 8; ++o) v[o] = bs[o];
        const float* zc = p.z + (long long)b * Cz * L + t;
        for (int k = 0; k < Cz; ++k) {
            const float zk = __ldg(zc + (long long)k * L);
            const float4 w0 = *reinterpret_cast<const float4*>(&ws[k][0]);
            const float4 w1 = *reinterpret_cast<const float4*>(&ws[k][4]);
            v[0] = fmaf(w0.x, zk, v[0]);
            v[1] = fmaf(w0.y, zk, v[1]);
            v[2] = fmaf(w0.z, zk, v[2]);
            v[3] = fmaf(w0.w, zk, v[3]);
            v[4] = fmaf(w1.x, zk, v[4]);
            v[5] = fmaf(w1.y, zk, v[5]);
            v[6] = fmaf(w1.z, zk, v[6]);
            v[7] = fmaf(w1.w, zk, v[7]);
        }
    } else {
#pragma unroll
        for (int o = 0; o < 8; ++o) v[o] = 0.f;   // the conv's zero padding
    }
    uint4 hv, lv;
    split2(v[0], v[1], &hv.x, &lv.x);
    split2(v[2], v[3], &hv.y, &lv.y);
    split2(v[4], v[5], &hv.z, &lv.z);
    split2(v[6], v[7], &hv.w, &lv.w);
    reinterpret_cast<uint4*>(p.a_hi)[row] = hv;
    reinterpret_cast<uint4*>(p.a_lo)[row] = lv;
}

// grid: x = output tiles of TT - (K - 1) samples, y = B.  Warp c stages the mean input window of
// channel c, forms its 512 activation values of rows [t0 - pad, t0 - pad + 512) with the same
// lane routine as k_act_split, and parks them in shared memory (zero outside [0, L): the conv's
// padding); then every thread forms up to two outputs from the 8 x K window.  The three block
// outputs' windows arrive as asynchronous copies, all in flight at once (a load loop waited for
// each round of loads: 41 -> 35 us per launch at B = 2, L = 320000); blocks 1 and 2 land in a
// staging area that the activation rows reuse afterwards.
constexpr int POST_STAGE = 2 * 8 * XF;   // floats: the windows of blocks 1 and 2, unskewed
static_assert(POST_STAGE >= 8 * TT, "the activation rows fit in the staging area");
constexpr int POST_SMEM = (8 * XF_P + POST_STAGE + 8 * kPostMaxK) * 4;   // bytes (dynamic)
__global__ void __launch_bounds__(NT_ACT) k_post_act(const PostParams p) {
    ptx::grid_dep_wait();     // launched as a programmatic dependent (see launch_dependent)
    ptx::grid_dep_launch();
    extern __shared__ __align__(16) float post_smem[];
    float* xsb = post_smem;                          // [8][XF_P] skewed mean windows
    float* stage = xsb + 8 * XF_P;                   // [2][8][XF], then [8][TT] activation rows
    float* wsh = stage + POST_STAGE;                 // [8 * K] conv_post weights
    float (*arow)[TT] = reinterpret_cast<float (*)[TT]>(stage);
    const int L = p.L, K = p.K, TO = TT - (K - 1);
    const int b = blockIdx.y;
    const int t0 = blockIdx.x * TO;
    const int tw = t0 - p.pad;                      // first activation row of the block
    const int tid = threadIdx.x, c = tid >> 5, lane = tid & 31;
    for (int i = tid; i < 8 * K; i += NT_ACT) wsh[i] = __ldg(p.w + i);
    float* xs = xsb + c * XF_P;
    float* w1 = stage + c * XF;
    float* w2 = stage + (8 + c) * XF;
    const long long rb = ((long long)b * 8 + c) * L;
    const bool edge = !(tw >= 8 && tw + TT + 8 <= L);
    // the three block outputs over x[tw - 8, tw + TT + 8), replicate-clamped at the ends, then
    // their mean into the skewed window
#pragma unroll
    for (int k = 0; k < (XF + 31) / 32; ++k) {
        const int i = lane + 32 * k;
        if (i < XF) {
            const long long g = rb + clampi(tw - 8 + i, 0, L - 1);
            ptx::cp_async4(xs + skew(i), p.x0 + g);
            ptx::cp_async4(w1 + i, p.x1 + g);
            ptx::cp_async4(w2 + i, p.x2 + g);
        }
    }
    ptx::cp_async_commit();
    ptx::cp_async_wait_all();
    __syncwarp();
    for (int i = lane; i < XF; i += 32) xs[skew(i)] = (xs[skew(i)] + w1[i] + w2[i]) / 3.0f;
    __syncthreads();   // every warp is done with the staging area before it holds activation rows
    const float al = __ldg(p.alpha + c), ib = __ldg(p.inv_beta + c);
    float a[RUN];
    if (edge) actm::act_lane<RUN, true>(p.filt, xs, al, ib, tw, L, a);
    else actm::act_lane<RUN, false>(p.filt, xs, al, ib, tw, L, a);
#pragma unroll
    for (int k = 0; k < RUN; ++k) {
        const int t = tw + RUN * lane + k;
        arow[c][RUN * lane + k] = (t >= 0 && t < L) ? a[k] : 0.f;
    }
    __syncthreads();
    const float bo = p.bias ? __ldg(p.bias) : 0.f;
    if (K == 7) {
        // two adjacent outputs per thread share 8 window values per channel
        const int q = 2 * tid;
        if (q < TO && t0 + q < L) {
            float y0 = 0.f, y1 = 0.f;
#pragma unroll
            for (int cc = 0; cc < 8; ++cc) {
                float xa[8];
#pragma unroll
                for (int j = 0; j < 8; j += 2) {
                    const float2 v = *reinterpret_cast<const float2*>(&arow[cc][q + j]);
                    xa[j] = v.x;
                    xa[j + 1] = v.y;
                }
#pragma unroll
                for (int j = 0; j < 7; ++j) {
                    const float wv = wsh[cc * 7 + j];
                    y0 = fmaf(wv, xa[j], y0);
                    y1 = fmaf(wv, xa[j + 1], y1);
                }
            }
            y0 += bo;
            y1 += bo;
            if (p.clamp) {   // NaN passes through
                y0 = (y0 < -1.f) ? -1.f : ((y0 > 1.f) ? 1.f : y0);
                y1 = (y1 < -1.f) ? -1.f : ((y1 > 1.f) ? 1.f : y1);
            }
            // one 8-byte store per pair where aligned (full 256-byte warp stores, which also
            // suits an output in mapped host memory)
            float* o = p.out + (long long)b * L + t0 + q;
            const bool pair = q + 1 < TO && t0 + q + 1 < L;
            if (pair && (reinterpret_cast<uintptr_t>(o) & 7) == 0) {
                *reinterpret_cast<float2*>(o) = make_float2(y0, y1);
            } else {
                o[0] = y0;
                if (pair) o[1] = y1;
            }
        }
    } else {
        for (int q = tid; q < TO; q += NT_ACT) {
            const int t = t0 + q;
            if (t >= L) break;
            float y = 0.f;
            for (int cc = 0; cc < 8; ++cc)
                for (int j = 0; j < K; ++j) y = fmaf(wsh[cc * K + j], arow[cc][q + j], y);
            y += bo;
            if (p.clamp) y = (y < -1.f) ? -1.f : ((y > 1.f) ? 1.f : y);   // NaN passes through
            p.out[(long long)b * L + t] = y;
        }
    }
}

}  // namespace

int launch_post_act(const PostParams& p, cudaStream_t s) {
    if (p.L < 1 || p.B < 1 || p.K < 1 || p.K > kPostMaxK || p.pad < 0 || p.pad > p.K - 1 || !p.x0 || !p.x1 ||
        !p.x2 || !p.w || !p.out)
        return -1;
    const int TO = TT - (p.K - 1);
    dim3 grid((p.L + TO - 1) / TO, p.B);
    if (cudaFuncSetAttribute(k_post_act, cudaFuncAttributeMaxDynamicSharedMemorySize, POST_SMEM) != cudaSuccess)
        return -1;
    return launch_dependent(k_post_act, grid, dim3(NT_ACT), POST_SMEM, s, p) == cudaSuccess ? 1 : -1;
}

int launch_proj_split(const ProjSplitParams& p, cudaStream_t s) {
    if (p.C % 8 != 0 || p.L < 1 || p.pad_l < 0 || p.pad_r < 0 || p.Cz < 1 || p.Cz > kProjMaxCz || !p.z || !p.w ||
        !p.bias)
        return -1;
    const int total = p.L + p.pad_l + p.pad_r;
    dim3 grid((total + NT_ACT - 1) / NT_ACT, p.B * (p.C / 8));
    return launch_dependent(k_proj_split, grid, dim3(NT_ACT), 0, s, p) == cudaSuccess ? 1 : -1;
}

int launch_split_rows(const SplitParams& p, cudaStream_t s) {
    if (p.C % 8 != 0 || p.L < 1 || p.pad_l < 0 || p.pad_r < 0 || !p.x0) return -1;
    if ((p.x1 == nullptr) != (p.x2 == nullptr) || (p.x3 && !p.x1)) return -1;
    const int total = p.L + p.pad_l + p.pad_r;
    dim3 grid((total + 2 * NT_ACT - 1) / (2 * NT_ACT), p.B * (p.C / 8));
    return launch_dependent(k_split_rows, grid, dim3(NT_ACT), 0, s, p) == cudaSuccess ? 1 : -1;
}

int launch_act_split(const ActParams& p, int njobs, cudaStream_t s) {
    if (p.C % 8 != 0 || p.L < 1 || p.pad_l < 0 || p.pad_r < 0) return -1;
    const int total = p.L + p.pad_l + p.pad_r;
    ActParams q = p;
    const int ng = p.C / 8;
    q.g_log2 = (ng & (ng - 1)) == 0 ? __builtin_ctz((unsigned)ng) : -1;
    dim3 grid((total + TT - 1) / TT, p.B * ng, njobs);
    return launch_dependent(k_act_split, grid, dim3(NT_ACT), 0, s, q) == cudaSuccess ? 1 : -1;
}

}  // namespace mh3a

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
        // stays contiguous and 16-byte aligned in shared memory)
#pragma unroll
        for (int k = 0; k < (XF / 4 + 31) / 32; ++k) {
            const int i = 4 * (lane + 32 * k);
            if (i < XF) ptx::cp_async16(xs + skew(i), xrow + t0 - 8 + i);
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

// Plain head/tail split (no activation) into the same row layout, of x0, of the mean
// (x0 + x1 + x2) / 3 of three block outputs, or of the sum of four partial outputs.  grid: x = row tiles of NT_ACT, y = B * C / 8.
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
            if (p.x3) v[c] = ((__ldg(p.x0 + i) + __ldg(p.x1 + i)) + __ldg(p.x2 + i)) + __ldg(p.x3 + i);
            else if (p.x1) v[c] = (__ldg(p.x0 + i) + __ldg(p.x1 + i) + __ldg(p.x2 + i)) / 3.0f;
            else v[c] = __ldg(p.x0 + i);
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
    if ((p.x1 == nullptr) != (p.x2 == nullptr) || (p.x3 && !p.x1)) return -1;
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

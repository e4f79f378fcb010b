// tc_kernels.cu -- tensor-core (tcgen05 / TMEM) path of the AMP-stage convolutions.
//
// One launch runs one conv layer of every residual block of an AMP stage (blockIdx.z = block,
// heaviest kernel first).  For block j the layer is
//   y[o, t] = bias[o] + sum_{c, tap} W[o, c, tap] * a[c, t + tap*dil - pad]  (+ residual[o, t])
//   a = down2(snake(up2(x)))   -- the anti-aliased SnakeBeta of the FastVideo
//                                 "minimax_h3_audio_vae" page's `_activation1d`
// as an implicit GEMM D[t, o] = sum_k A[t, k] B[o, k] with M = time (128-row accumulators in
// tensor memory, MT of them per CTA), N = output channels (NT per CTA), K = input channels x
// taps.
//
// Precision (3xBF16): every fp32 operand is split into a bf16 head h = bf16(v) and a bf16
// tail l = bf16(v - h); the product is accumulated as A_h B_h + A_h B_l + A_l B_h in fp32.
//
// Shared-memory operands use the no-swizzle K-major canonical layout: core matrices of 8 rows
// x 16 bytes (8 bf16 along K).  The activation window is stored with ALL its rows 16 bytes
// apart inside each 8-channel group, so the operand for tap `tap` is the same window started
// `tap * dil` rows later: only the descriptor start address moves, and no data is copied per
// tap.  Weights are pre-split and pre-laid-out at create time in exactly that layout, one
// contiguous block per (output tile, 32-channel chunk, tap), so one 1-D bulk copy stages it.
//
// Warp roles: warp 0 -- TMEM allocation and the MMA issuer (one thread); warp 1 -- weight
// bulk copies (one thread); warps 2..9 -- activation producers, then the epilogue (TMEM ->
// registers -> bias + residual -> coalesced fp32 stores along time).  Every mbarrier wait is
// bounded; a timeout raises the error flag, and the kernel drains and returns.
#include <cuda_bf16.h>

#include <algorithm>
#include <cstring>

#include "tc_kernels.cuh"
#include "tc_ptx.cuh"

namespace mh3a {
namespace {

constexpr int KC = 32;              // input channels per chunk (4 groups of 8)
constexpr int KG = KC / 8;          // channel groups per chunk
constexpr int NPROD = 512;          // producer / epilogue threads (warps 2..17)
constexpr int NTHREADS = NPROD + 64;
constexpr int NSA = 2;              // activation pipeline depth
constexpr int NSB = 3;              // weight pipeline depth
constexpr uint64_t kWaitLimit = 1000000000ull;  // ns; legitimate waits last milliseconds

struct TcJob {
    const float* x;
    const uint16_t* w;   // pre-split operand blocks
    const float* bias;
    const float* alpha;
    const float* inv_beta;
    const float* res;
    float* out;
    int K, dil, pad;
};

struct TcParams {
    TcJob job[MH3A_MAX_RESBLOCKS];
    int C, L, B, tiles_t;
    ActFilter filt;
    int* err;
};

struct TcPlan {
    int RS;         // activation rows per channel group (max over jobs)
    int XWs, SWs;   // staging strides (floats)
    int SA, SB;     // bytes per activation / weight pipeline stage
    int offB, offX, offBar;
    int smem;
};

__device__ __forceinline__ int clampi(int v, int lo, int hi) { return v < lo ? lo : (v > hi ? hi : v); }

// sin^2(alpha u) for the tensor-core path: Cody-Waite reduction modulo pi, then the hardware
// sine on [-pi/2, pi/2] (absolute error near 2^-21, far below the 3xBF16 operand error).
__device__ __forceinline__ float sin_sq_fast(float alpha, float u) {
    const float kInvPi = 0.318309886183790671538f;
    const float kPiHi = 3.14159274101257324219f;
    const float kPiLo = -8.74227800037248297e-08f;
    const float v = alpha * u;
    const float k = rintf(v * kInvPi);
    float r = fmaf(-k, kPiHi, v);
    r = fmaf(-k, kPiLo, r);
    const float s = __sinf(r);
    return s * s;
}

__device__ __forceinline__ void prod_sync() { asm volatile("bar.sync 1, %0;" ::"n"(NPROD) : "memory"); }

__device__ __forceinline__ uint32_t pack_bf16(float lo_elem, float hi_elem) {
    const uint32_t a = __bfloat16_as_ushort(__float2bfloat16_rn(lo_elem));
    const uint32_t b = __bfloat16_as_ushort(__float2bfloat16_rn(hi_elem));
    return a | (b << 16);
}

__device__ __forceinline__ float bf16_round(float v) { return __bfloat162float(__float2bfloat16_rn(v)); }

// Accumulation: the tensor core rounds its fp32 accumulator toward zero at every instruction,
// so a long K loop into one accumulator builds a bias of about (instructions) x 2^-24
// relative.  Each M tile therefore owns NACC accumulators of NT columns: head x head products
// rotate over the first NACC-1 by chunk, and the small cross terms (head x tail, tail x head)
// go to the last one; the epilogue adds them in fp32 with round-to-nearest.
template <int MT, int NT, int NACC>
__global__ void __launch_bounds__(NTHREADS, 1) k_amp_conv_tc(const TcParams p, const TcPlan pl) {
    extern __shared__ __align__(1024) uint8_t smem[];
    constexpr int NHH = NACC - 1;
    constexpr int USED = MT * NT * NACC;
    static_assert(NACC >= 2 && USED <= 512, "tensor memory holds 512 columns");
    constexpr int NCOLS = (USED <= 32) ? 32 : (USED <= 64) ? 64 : (USED <= 128) ? 128 : (USED <= 256) ? 256 : 512;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const TcJob& J = p.job[blockIdx.z];
    const int K = J.K, dil = J.dil, pad = J.pad;
    const int C = p.C, L = p.L;
    const int b = blockIdx.x / p.tiles_t;
    const int t0 = (blockIdx.x % p.tiles_t) * (128 * MT);
    const int o_tile = blockIdx.y;
    const int o0 = o_tile * NT;
    const int nchunks = C / KC;
    const int ROWS = 128 * MT + (K - 1) * dil;
    const int RS = pl.RS;

    uint8_t* As = smem;                        // [NSA][2][KG][RS][16 B]
    uint8_t* Bs = smem + pl.offB;              // [NSB][2][KG][NT][16 B]
    float* xs = reinterpret_cast<float*>(smem + pl.offX);  // [2][8][XWs] (double buffer)
    float* sw = xs + 2 * 8 * pl.XWs;                        // [8][SWs]
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + pl.offBar);
    uint64_t* a_full = bars;
    uint64_t* a_empty = bars + NSA;
    uint64_t* b_full = bars + 2 * NSA;
    uint64_t* b_empty = bars + 2 * NSA + NSB;
    uint64_t* acc_full = bars + 2 * NSA + 2 * NSB;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * NSA + 2 * NSB + 1);
    // abort_flag: any role gave up; prod_go: the producers' shared decision, written only by
    // producer thread 0 before a producer barrier so that all producers branch alike.
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
    volatile int* prod_go = abort_flag + 1;

    if (threadIdx.x == 0) {
        for (int s = 0; s < NSA; ++s) {
            ptx::mbar_init(&a_full[s], 1);
            ptx::mbar_init(&a_empty[s], 1);
        }
        for (int s = 0; s < NSB; ++s) {
            ptx::mbar_init(&b_full[s], 1);
            ptx::mbar_init(&b_empty[s], 1);
        }
        ptx::mbar_init(acc_full, 1);
        // once a launch has failed, every later block skips its work (the host reads the flag)
        *abort_flag = (*reinterpret_cast<volatile int*>(p.err) != 0) ? 1 : 0;
        *prod_go = 0;
        ptx::fence_mbar_init();
    }
    if (warp == 0) {
        ptx::tmem_alloc(tmem_slot, NCOLS);
        ptx::tmem_relinquish();
    }
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == 0) {
        // ---------------------------------------------------------------- MMA issuer
        if (lane == 0) {
            const uint32_t idesc = ptx::idesc_bf16(128, NT);
            const uint32_t a_smem = ptx::smem_u32(As), b_smem = ptx::smem_u32(Bs);
            const bool skip = *abort_flag != 0;
            bool ok = !skip;
            int u = 0;
            for (int chunk = 0; chunk < nchunks && ok; ++chunk) {
                const int sa = chunk % NSA;
                if (!ptx::mbar_wait(&a_full[sa], (chunk / NSA) & 1, kWaitLimit)) { ok = false; break; }
                ptx::tc_fence_after();
                const uint32_t a_hi = a_smem + sa * pl.SA;
                const uint32_t a_lo = a_hi + KG * RS * 16;
                for (int tap = 0; tap < K; ++tap, ++u) {
                    const int sb = u % NSB;
                    if (!ptx::mbar_wait(&b_full[sb], (u / NSB) & 1, kWaitLimit)) { ok = false; break; }
                    ptx::tc_fence_after();
                    const uint32_t b_hi = b_smem + sb * pl.SB;
                    const uint32_t b_lo = b_hi + KG * NT * 16;
#pragma unroll
                    for (int kk = 0; kk < KG / 2; ++kk) {
                        const uint32_t boff = (uint32_t)(2 * kk) * NT * 16;
                        const uint64_t bh = ptx::smem_desc(b_hi + boff, NT * 16, 128);
                        const uint64_t bl = ptx::smem_desc(b_lo + boff, NT * 16, 128);
#pragma unroll
                        for (int mt = 0; mt < MT; ++mt) {
                            const uint32_t aoff = (uint32_t)(2 * kk) * RS * 16 + (uint32_t)(mt * 128 + tap * dil) * 16;
                            const uint64_t ah = ptx::smem_desc(a_hi + aoff, RS * 16, 128);
                            const uint64_t al = ptx::smem_desc(a_lo + aoff, RS * 16, 128);
                            const uint32_t dh = tmem + (uint32_t)((mt * NACC + chunk % NHH) * NT);
                            const uint32_t dx = tmem + (uint32_t)((mt * NACC + NHH) * NT);
                            const uint32_t acc_h = (chunk >= NHH || tap > 0 || kk > 0) ? 1u : 0u;
                            const uint32_t acc_x = (chunk > 0 || tap > 0 || kk > 0) ? 1u : 0u;
                            ptx::mma_bf16(dh, ah, bh, idesc, acc_h);
                            ptx::mma_bf16(dx, ah, bl, idesc, acc_x);
                            ptx::mma_bf16(dx, al, bh, idesc, 1u);
                        }
                    }
                    ptx::mma_commit(&b_empty[sb]);
                }
                if (ok) ptx::mma_commit(&a_empty[sa]);
            }
            if (!ok) {
                *abort_flag = 1;
                if (!skip) atomicExch(p.err, 1);
            }
            // always signal the epilogue (an empty commit arrives at once)
            ptx::mma_commit(acc_full);
        }
        __syncwarp();
    } else if (warp == 1) {
        // ---------------------------------------------------------------- weight loader
        if (lane == 0) {
            const int units = nchunks * K;
            const size_t unit_elems = (size_t)2 * KG * NT * 8;
            const uint16_t* wsrc = J.w + (size_t)o_tile * units * unit_elems;
            int issued = 0;
            for (int u = 0; u < units; ++u) {
                const int sb = u % NSB;
                if (*abort_flag || !ptx::mbar_wait(&b_empty[sb], ((u / NSB) & 1) ^ 1, kWaitLimit)) {
                    *abort_flag = 1;
                    atomicExch(p.err, 2);
                    break;
                }
                ptx::mbar_arrive_expect_tx(&b_full[sb], (uint32_t)pl.SB);
                ptx::bulk_g2s(Bs + (size_t)sb * pl.SB, wsrc + (size_t)u * unit_elems, (uint32_t)pl.SB, &b_full[sb]);
                issued = u + 1;
            }
            if (*abort_flag) {
                // let the copies already in flight land before the CTA can exit
                for (int u = (issued > NSB ? issued - NSB : 0); u < issued; ++u)
                    ptx::mbar_wait(&b_full[u % NSB], (u / NSB) & 1, kWaitLimit);
            }
        }
        __syncwarp();
    } else {
        // ---------------------------------------------------------------- activation producers
        // Work is done one group of 8 input channels at a time.  Warp pair (2c, 2c+1) owns
        // channel c of the group; its 64 lanes stride over positions.  The next group's input
        // window is prefetched with cp.async into the other half of a double buffer while the
        // current group is being processed.
        const int ptid = threadIdx.x - 64;
        const int pw = ptid >> 5;                  // producer warp 0..15
        const int ch = pw >> 1;                    // channel within the group
        const int lane64 = ((pw & 1) << 5) | lane; // position stride index 0..63
        const int a_start = t0 - pad;
        const int xs_start = a_start - 6;
        const int n_start = 2 * a_start - 5;
        const int XW = ROWS + 12, SW = 2 * ROWS + 10;
        const long long xbase = (long long)b * C * L;
        const int gtotal = nchunks * KG;
        // x window of group gi (channels gi*8 .. gi*8+7), replicate-clamped at the sequence ends
        auto prefetch = [&](int gi) {
            float* dst = xs + (size_t)(gi & 1) * 8 * pl.XWs + ch * pl.XWs;
            const float* src = J.x + xbase + (long long)(gi * 8 + ch) * L;
            for (int q = lane64; q < XW; q += 64) ptx::cp_async4(dst + q, src + clampi(xs_start + q, 0, L - 1));
            ptx::cp_async_commit();
        };
        prefetch(0);
        for (int gi = 0; gi < gtotal; ++gi) {
            const int chunk = gi / KG, g = gi - chunk * KG;
            const int sa = chunk % NSA;
            if (g == 0) {
                if (ptid == 0) {
                    bool go = *abort_flag == 0;
                    if (go && !ptx::mbar_wait(&a_empty[sa], ((chunk / NSA) & 1) ^ 1, kWaitLimit)) {
                        go = false;
                        *abort_flag = 1;
                        atomicExch(p.err, 3);
                    }
                    *prod_go = go ? 1 : 0;
                }
            }
            ptx::cp_async_wait_all();
            prod_sync();   // x window of this group landed; the previous group's decimation is done
            if (g == 0 && *prod_go == 0) break;
            // ---- SnakeBeta of the 2x upsampled signal, one channel per warp pair
            {
                const float* xr0 = xs + (size_t)(gi & 1) * 8 * pl.XWs + ch * pl.XWs - xs_start;
                float* srow = sw + ch * pl.SWs;
                const float al = __ldg(J.alpha + gi * 8 + ch), ib = __ldg(J.inv_beta + gi * 8 + ch);
                for (int q = lane64; q < SW; q += 64) {
                    const int n = clampi(n_start + q, 0, 2 * L - 1);
                    const float* xr = xr0 + (n >> 1);
                    float u = 0.f;
                    if ((n & 1) == 0) {
#pragma unroll
                        for (int k = 0; k < 6; ++k) u = fmaf(p.filt.up[2 * k + 1], xr[2 - k], u);
                    } else {
#pragma unroll
                        for (int k = 0; k < 6; ++k) u = fmaf(p.filt.up[2 * k], xr[3 - k], u);
                    }
                    srow[q] = fmaf(sin_sq_fast(al, u), ib, u);
                }
            }
            if (gi + 1 < gtotal) prefetch(gi + 1);
            prod_sync();   // all 8 snake rows ready
            // ---- decimate into the A operand: 2 rows x 4 channels per thread
            {
                uint8_t* a_hi = As + (size_t)sa * pl.SA + (size_t)g * RS * 16;
                uint8_t* a_lo = a_hi + (size_t)KG * RS * 16;
                const int npairs = (ROWS + 1) >> 1;
                for (int it = ptid; it < 2 * npairs; it += NPROD) {
                    const int rp = it >> 1, chh = it & 1;
                    const int q0 = 2 * rp;
                    float a0[4], a1[4];
#pragma unroll
                    for (int c = 0; c < 4; ++c) {
                        const float2* sr = reinterpret_cast<const float2*>(sw + (4 * chh + c) * pl.SWs + 2 * q0);
                        float s[14];
#pragma unroll
                        for (int j = 0; j < 7; ++j) {
                            const float2 v2 = sr[j];
                            s[2 * j] = v2.x;
                            s[2 * j + 1] = v2.y;
                        }
                        float v0 = 0.f, v1 = 0.f;
#pragma unroll
                        for (int j = 0; j < kFilterTaps; ++j) {
                            v0 = fmaf(p.filt.down[j], s[j], v0);
                            v1 = fmaf(p.filt.down[j], s[j + 2], v1);
                        }
                        a0[c] = v0;
                        a1[c] = v1;
                    }
                    const int gp0 = a_start + q0;
                    const bool in0 = gp0 >= 0 && gp0 < L, in1 = gp0 + 1 >= 0 && gp0 + 1 < L;
#pragma unroll
                    for (int r = 0; r < 2; ++r) {
                        if (q0 + r >= ROWS) break;
                        float* a = r == 0 ? a0 : a1;
                        const bool in = r == 0 ? in0 : in1;
                        float h[4], l[4];
#pragma unroll
                        for (int c = 0; c < 4; ++c) {
                            const float v = in ? a[c] : 0.f;
                            h[c] = bf16_round(v);
                            l[c] = v - h[c];
                        }
                        uint2 hv, lv;
                        hv.x = pack_bf16(h[0], h[1]);
                        hv.y = pack_bf16(h[2], h[3]);
                        lv.x = pack_bf16(l[0], l[1]);
                        lv.y = pack_bf16(l[2], l[3]);
                        const size_t off = (size_t)(q0 + r) * 16 + chh * 8;
                        *reinterpret_cast<uint2*>(a_hi + off) = hv;
                        *reinterpret_cast<uint2*>(a_lo + off) = lv;
                    }
                }
            }
            if (g == KG - 1) {
                ptx::fence_proxy_async_smem();
                prod_sync();
                if (ptid == 0) ptx::mbar_arrive(&a_full[sa]);
            }
        }
        ptx::cp_async_wait_all();

        // ---------------------------------------------------------------- epilogue
        if (ptid == 0) {
            bool go = ptx::mbar_wait(acc_full, 0, kWaitLimit);
            if (!go) atomicExch(p.err, 4);
            go = go && *abort_flag == 0;
            if (!go) *abort_flag = 1;
            *prod_go = go ? 1 : 0;
        }
        prod_sync();
        const bool epi_go = *prod_go != 0;   // identical in every producer thread
        ptx::tc_fence_after();
        const int q4 = warp & 3;                   // TMEM lane quarter this warp may access
        const int part = (warp - 2) >> 2;          // which quarter of the columns (0..3)
        constexpr int CPP = (NT / 4 >= 16) ? NT / 4 : 16;
        const long long obase = (long long)b * C * L;
        if (epi_go && part * CPP < NT) {
#pragma unroll
            for (int mt = 0; mt < MT; ++mt) {
                const int t = t0 + mt * 128 + q4 * 32 + lane;
                for (int cb = part * CPP; cb < part * CPP + CPP && cb < NT; cb += 16) {
                    float v[16], w[16];
                    const uint32_t lane_addr = tmem + ((uint32_t)(q4 * 32) << 16);
                    ptx::tmem_ld16(lane_addr + (uint32_t)(mt * NACC * NT + cb), v);
#pragma unroll
                    for (int a = 1; a < NACC; ++a) {
                        ptx::tmem_ld16(lane_addr + (uint32_t)((mt * NACC + a) * NT + cb), w);
#pragma unroll
                        for (int i = 0; i < 16; ++i) v[i] += w[i];
                    }
                    if (t < L) {
#pragma unroll
                        for (int i = 0; i < 16; ++i) {
                            const int o = o0 + cb + i;
                            const long long idx = obase + (long long)o * L + t;
                            float y = v[i] + __ldg(J.bias + o);
                            if (J.res) y += J.res[idx];
                            J.out[idx] = y;
                        }
                    }
                }
            }
        }
    }
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    if (warp == 0) ptx::tmem_dealloc(tmem, NCOLS);
}

// ----------------------------------------------------------------------------------------------
// host side
// ----------------------------------------------------------------------------------------------

uint16_t bf16_bits_rn(float v) {
    uint32_t u;
    std::memcpy(&u, &v, 4);
    u += 0x7FFFu + ((u >> 16) & 1u);
    return (uint16_t)(u >> 16);
}

float bf16_value(uint16_t h) {
    const uint32_t u = (uint32_t)h << 16;
    float v;
    std::memcpy(&v, &u, 4);
    return v;
}

int ntile_for(int C) { return C >= 256 ? 256 : C; }

template <int MT, int NT>
TcPlan make_plan(const TcParams& p, int njobs) {
    int span = 0;
    for (int j = 0; j < njobs; ++j) span = std::max(span, (p.job[j].K - 1) * p.job[j].dil);
    TcPlan pl{};
    pl.RS = 128 * MT + span;
    pl.XWs = pl.RS + 12;
    pl.SWs = 2 * pl.RS + 12;  // even (8-byte rows) with room for the last row pair's reads
    pl.SA = 2 * KG * pl.RS * 16;
    pl.SB = 2 * KG * NT * 16;
    pl.offB = NSA * pl.SA;
    pl.offX = pl.offB + NSB * pl.SB;
    const int stage_bytes = 8 * (2 * pl.XWs + pl.SWs) * 4;
    pl.offBar = (pl.offX + stage_bytes + 15) / 16 * 16;
    pl.smem = pl.offBar + 8 * (2 * NSA + 2 * NSB + 1) + 16;
    return pl;
}

template <int MT, int NT, int NACC>
int launch_tc(const TcParams& p0, int njobs, cudaStream_t s) {
    TcParams p = p0;
    if (NACC - 1 > p.C / KC) return -1;  // every head accumulator must receive a chunk
    p.tiles_t = (p.L + 128 * MT - 1) / (128 * MT);
    const TcPlan pl = make_plan<MT, NT>(p, njobs);
    if (pl.smem > 227 * 1024) return -1;
    auto kern = k_amp_conv_tc<MT, NT, NACC>;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, pl.smem) != cudaSuccess) return -1;
    dim3 grid(p.tiles_t * p.B, p.C / NT, njobs);
    kern<<<grid, NTHREADS, pl.smem, s>>>(p, pl);
    return cudaPeekAtLastError() == cudaSuccess ? 1 : -1;
}

// Tile shape per width: MT x 128 time rows, NT output channels, NACC accumulators per M tile
// (MT * NT * NACC <= 512 tensor-memory columns).
int dispatch_tc(const TcParams& p, int njobs, cudaStream_t s) {
    switch (p.C) {
        case 512: return launch_tc<1, 256, 2>(p, njobs, s);
        case 256: return launch_tc<1, 256, 2>(p, njobs, s);
        case 128: return launch_tc<2, 128, 2>(p, njobs, s);
        case 64: return launch_tc<2, 64, 3>(p, njobs, s);
        case 32: return launch_tc<2, 32, 2>(p, njobs, s);
        default: return -1;
    }
}

}  // namespace

bool tc_stage_supported(int C, const mh3a_config& c) {
    if (C != 512 && C != 256 && C != 128 && C != 64 && C != 32) return false;
    if (c.n_resblocks != 3) return false;
    for (int j = 0; j < c.n_resblocks; ++j)
        for (int m = 0; m < c.n_dilations; ++m) {
            // the activation window must fit the shared-memory plan
            if ((c.rb_kernels[j] - 1) * c.rb_dilations[j][m] > 64) return false;
        }
    return true;
}

// Operand blocks: [o_tile][chunk][tap][part (head, tail)][group][row o][8 channels] as bf16.
void prepare_tc_conv(const std::vector<float>& w, int C, int k, TcConv* out) {
    const int NT = ntile_for(C);
    const int ntiles = C / NT, nchunks = C / KC;
    const size_t n = (size_t)C * C * k * 2;  // bf16 elements (head + tail)
    std::vector<uint16_t> buf(n);
    size_t pos = 0;
    for (int ot = 0; ot < ntiles; ++ot)
        for (int ch = 0; ch < nchunks; ++ch)
            for (int tap = 0; tap < k; ++tap)
                for (int part = 0; part < 2; ++part)
                    for (int g = 0; g < KG; ++g)
                        for (int o = 0; o < NT; ++o)
                            for (int e = 0; e < 8; ++e) {
                                const int oo = ot * NT + o, cc = ch * KC + g * 8 + e;
                                const float v = w[((size_t)oo * C + cc) * k + tap];
                                const uint16_t hb = bf16_bits_rn(v);
                                buf[pos++] = part == 0 ? hb : bf16_bits_rn(v - bf16_value(hb));
                            }
    out->staging.assign(n / 2, 0.f);
    std::memcpy(out->staging.data(), buf.data(), n * sizeof(uint16_t));
    out->cout = C;
    out->cin = C;
    out->k = k;
}

void prepare_tc_pre(const std::vector<float>&, int, int, int, TcStageWeights*) {}

void tc_finalize(TcStageWeights* w) {
    for (auto& a : w->conv)
        for (auto& b : a)
            for (auto& c : b) std::vector<float>().swap(c.staging);
    std::vector<float>().swap(w->pre.staging);
}

int launch_conv_tc(const ConvParams& cp, int njobs, const TcStageWeights& w, int m, int half, cudaStream_t s,
                   int* err) {
    TcParams p{};
    p.C = cp.Cin;
    p.L = cp.L;
    p.B = cp.B;
    p.filt = cp.filt;
    p.err = err;
    // heaviest kernel first (blockIdx.z = 0), so the longest blocks start earliest
    int order[MH3A_MAX_RESBLOCKS];
    for (int j = 0; j < njobs; ++j) order[j] = j;
    std::sort(order, order + njobs, [&](int a, int b) { return cp.job[a].K > cp.job[b].K; });
    for (int z = 0; z < njobs; ++z) {
        const int j = order[z];
        const ConvJob& J = cp.job[j];
        const TcConv& tw = w.conv[j][m][half];
        if (!tw.dev) return -1;
        TcJob& T = p.job[z];
        T.x = J.x0;
        T.w = reinterpret_cast<const uint16_t*>(tw.dev);
        T.bias = J.bias;
        T.alpha = J.alpha;
        T.inv_beta = J.inv_beta;
        T.res = J.res;
        T.out = J.out;
        T.K = J.K;
        T.dil = J.dil;
        T.pad = J.pad;
    }
    return dispatch_tc(p, njobs, s);
}

int launch_conv_pre_tc(const ConvParams&, const TcStageWeights&, cudaStream_t) { return -1; }

}  // namespace mh3a

// tc_kernels.cu -- tensor-core (tcgen05 / TMEM) convolutions of the decode, as implicit GEMMs
// D[row, o] = sum_k A[row, k] B[o, k] with M = time rows (128-row accumulators in tensor
// memory), N = output channels and K = input channels x taps.
//
//  k_gemm_ps   the persistent GEMM that runs every tensor-core conv of a decode: the AMP
//              residual-block convs (the anti-aliased SnakeBeta of the FastVideo
//              "minimax_h3_audio_vae" page's `_activation1d` already written as the A operand
//              by the activation kernel), conv_pre, and the weight-normed transposed convs
//              (`ups.i.0`) in polyphase form: output t = r u + phi only meets taps
//              j = (phi + pad) mod r + r m, which read input u + (phi + pad - j) / r, so no zero
//              is ever inserted or multiplied.  Its design notes precede the kernel.
//  k_conv_tc   a fused AMP layer (activation computed by 16 producer warps into the A operand
//              in shared memory) for the allocation-free stage entry point, which has no
//              operand arrays.
//
// Precision (3xBF16): every fp32 operand is split into a bf16 head h = bf16(v) and a bf16
// tail l = bf16(v - h); the product is accumulated as A_h B_h + A_h B_l + A_l B_h in fp32.
//
// Accumulation: the tensor core rounds its fp32 accumulator toward zero at every instruction,
// so a long K loop into one accumulator builds a bias of about (instructions) x 2^-24
// relative.  k_gemm_ps bounds every accumulator to one pass of at most 16 K-steps and adds the
// passes in fp32 registers with round-to-nearest; k_conv_tc gives each M tile NACC
// accumulators (head x head products rotating over the first NACC-1 by chunk, the cross terms
// in the last) and adds them in the epilogue.
//
// Shared-memory operands use the no-swizzle K-major canonical layout: core matrices of 8 rows
// x 16 bytes (8 bf16 along K).  The input window is stored with ALL its rows 16 bytes apart
// inside each 8-channel group, so the operand of any tap is the same window started a few rows
// later: only the descriptor start address moves.  Weights are pre-split and pre-laid-out at
// create time in that layout, one contiguous block per (output tile, K chunk, tap or tap pair),
// so 1-D bulk copies stage them.  Every mbarrier wait is bounded; a timeout raises the error
// flag, and the kernel drains and returns.
#include <cuda_bf16.h>

#include <algorithm>
#include <cstring>

#include "act_math.cuh"
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
    const float* x0;     // the layer input [B, Cin, L]
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
    int Cin, Cout;
    int L;               // sequence length (input = output)
    int B, tiles_t;
    ActFilter filt;
    int* err;
};

struct TcPlan {
    int RS;         // window rows per channel group (max over jobs)
    int XWs, SWs;   // staging strides (floats)
    int SA, SB;     // bytes per activation / weight pipeline stage
    int offB, offX, offBar;
    int smem;
};

__device__ __forceinline__ int clampi(int v, int lo, int hi) { return v < lo ? lo : (v > hi ? hi : v); }

// Narrow output tiles (NT <= 64) of plain convs take the two-MMA form of the 3xBF16 K-step:
//   D[0, 2 NT) += A_h [B_h | B_l]      (head x head and head x tail side by side in N)
//   D[NT, 2 NT) += A_l B_h             (tail x head into the cross columns)
// so the activation operand is read twice per K-step instead of three times (the MMA of a
// narrow tile is bound by reading that operand from shared memory).  Their weight blocks store
// each core column's head rows directly followed by its tail rows.
__host__ __device__ constexpr bool interleaved_b(int NT, int R) { return R == 1 && NT <= 64; }

// Upsampler rates whose taps are grouped by input row offset (one MMA over all phases per
// group).  At rate 2 a group holds at most two taps, so the zero rows would cost what the wider
// MMA saves.
__host__ __device__ constexpr bool convt_grouped(int R) { return R > 2; }

__device__ __forceinline__ void prod_sync() { asm volatile("bar.sync 1, %0;" ::"n"(NPROD) : "memory"); }

__device__ __forceinline__ uint32_t pack_bf16(float lo_elem, float hi_elem) {
    const uint32_t a = __bfloat16_as_ushort(__float2bfloat16_rn(lo_elem));
    const uint32_t b = __bfloat16_as_ushort(__float2bfloat16_rn(hi_elem));
    return a | (b << 16);
}

__device__ __forceinline__ float bf16_round(float v) { return __bfloat162float(__float2bfloat16_rn(v)); }

// Fused AMP layer.  Warp roles: warp 0 -- TMEM allocation and the MMA issuer (one thread);
// warp 1 -- weight bulk copies (one thread); warps 2..17 -- input producers (cp.async prefetch
// of the next 8-channel window, SnakeBeta at the 2x rate, decimation into the A operand), then
// the epilogue (TMEM -> registers -> bias + residual -> fp32 stores along time).
template <int MT, int NT, int NACC>
__global__ void __launch_bounds__(NTHREADS, 1) k_conv_tc(const TcParams p, const TcPlan pl) {
    extern __shared__ __align__(1024) uint8_t smem[];
    constexpr int NHH = NACC - 1;
    constexpr int USED = MT * NT * NACC;
    static_assert(NACC >= 2 && USED <= 512, "tensor memory holds 512 columns");
    constexpr int NCOLS = (USED <= 32) ? 32 : (USED <= 64) ? 64 : (USED <= 128) ? 128 : (USED <= 256) ? 256 : 512;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const TcJob& J = p.job[blockIdx.z];
    const int K = J.K, dil = J.dil, pad = J.pad;
    const int Cin = p.Cin, Cout = p.Cout, L = p.L;
    const int b = blockIdx.x / p.tiles_t;
    const int t0 = (blockIdx.x % p.tiles_t) * (128 * MT);
    const int o_tile = blockIdx.y;
    const int o0 = o_tile * NT;
    const int nchunks = Cin / KC;
    const int span = (K - 1) * dil;
    const int ROWS = 128 * MT + span;
    const int RS = pl.RS;

    uint8_t* As = smem;                        // [NSA][2][KG][RS][16 B]
    uint8_t* Bs = smem + pl.offB;              // [NSB][2][KG][NT][16 B]
    float* xs = reinterpret_cast<float*>(smem + pl.offX);  // [2][8][XWs] (double buffer)
    float* sw = xs + 2 * 8 * pl.XWs;                        // [8][SWs] SnakeBeta rows
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
                    const int shift = tap * dil;
                    const bool first = tap == 0;
                    // weight blocks: [part][core col][row] or, for narrow tiles,
                    // [core col][part][row] (interleaved_b)
                    constexpr bool ILV = interleaved_b(NT, 1);
                    constexpr uint32_t b_lbo = (ILV ? 2 * NT : NT) * 16;
                    const uint32_t b_hi = b_smem + sb * pl.SB;
                    const uint32_t b_lo = ILV ? b_hi + NT * 16 : b_hi + KG * NT * 16;
#pragma unroll
                    for (int kk = 0; kk < KG / 2; ++kk) {
                        const uint32_t boff = (uint32_t)(2 * kk) * (b_lbo);
                        const uint64_t bh = ptx::smem_desc(b_hi + boff, b_lbo, 128);
                        const uint64_t bl = ptx::smem_desc(b_lo + boff, b_lbo, 128);
#pragma unroll
                        for (int mt = 0; mt < MT; ++mt) {
                            const uint32_t aoff = (uint32_t)(2 * kk) * RS * 16 + (uint32_t)(mt * 128 + shift) * 16;
                            const uint64_t ah = ptx::smem_desc(a_hi + aoff, RS * 16, 128);
                            const uint64_t al = ptx::smem_desc(a_lo + aoff, RS * 16, 128);
                            const int accbase = mt * NACC;
                            const uint32_t dh = tmem + (uint32_t)((accbase + chunk % NHH) * NT);
                            const uint32_t dx = tmem + (uint32_t)((accbase + NHH) * NT);
                            const uint32_t acc_h = (chunk >= NHH || !first || kk > 0) ? 1u : 0u;
                            const uint32_t acc_x = (chunk > 0 || !first || kk > 0) ? 1u : 0u;
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
        // ---------------------------------------------------------------- input producers
        // Work is done one group of 8 input channels at a time.  Warp pair (2c, 2c+1) owns
        // channel c of the group; its 64 lanes stride over positions.  The next group's input
        // window is prefetched with cp.async into the other half of a double buffer while the
        // current group is being processed.
        const int ptid = threadIdx.x - 64;
        const int pw = ptid >> 5;                  // producer warp 0..15
        const int ch = pw >> 1;                    // channel within the group
        const int lane64 = ((pw & 1) << 5) | lane; // position stride index 0..63
        const int a_start = t0 - pad;            // first window row
        const int xs_start = a_start - 6;        // first staged sample
        const int n_start = 2 * a_start - 5;
        const int XW = ROWS + 12;
        const int SW = 2 * ROWS + 10;
        const long long xbase = (long long)b * Cin * L;
        const int gtotal = nchunks * KG;
        auto prefetch = [&](int gi) {
            const float* src = J.x0 + xbase + (long long)(gi * 8 + ch) * L;
            float* dst = xs + ((size_t)(gi & 1) * 8 + ch) * pl.XWs;
            for (int q = lane64; q < XW; q += 64) ptx::cp_async4(dst + q, src + clampi(xs_start + q, 0, L - 1));
            ptx::cp_async_commit();
        };
        prefetch(0);
        for (int gi = 0; gi < gtotal; ++gi) {
            const int chunk = gi / KG, g = gi - chunk * KG;
            const int sa = chunk % NSA;
            if (g == 0 && ptid == 0) {
                bool go = *abort_flag == 0;
                if (go && !ptx::mbar_wait(&a_empty[sa], ((chunk / NSA) & 1) ^ 1, kWaitLimit)) {
                    go = false;
                    *abort_flag = 1;
                    atomicExch(p.err, 3);
                }
                *prod_go = go ? 1 : 0;
            }
            ptx::cp_async_wait_all();
            prod_sync();   // this group's window landed; the previous group's stores are done
            if (g == 0 && *prod_go == 0) break;
            uint8_t* a_hi = As + (size_t)sa * pl.SA + (size_t)g * RS * 16;
            uint8_t* a_lo = a_hi + (size_t)KG * RS * 16;
            const float* xg = xs + (size_t)(gi & 1) * 8 * pl.XWs;
            {
                // ---- SnakeBeta of the 2x upsampled signal, one channel per warp pair.  A lane
                // takes one input position m and forms both phases n = 2m (taps 1,3,..,11 on
                // x[m+2..m-3]) and n = 2m+1 (taps 0,2,..,10 on x[m+3..m-2]) from the same seven
                // inputs; positions past either end repeat the end sample (replicate padding).
                {
                    const float* xr0 = xg + ch * pl.XWs - xs_start;
                    float* srow = sw + ch * pl.SWs;
                    const float al = __ldg(J.alpha + gi * 8 + ch), ib = __ldg(J.inv_beta + gi * 8 + ch);
                    const int m_lo = n_start >> 1, m_hi = (n_start + SW - 1) >> 1;
                    for (int m = m_lo + lane64; m <= m_hi; m += 64) {
                        const int mc = clampi(m, 0, L - 1);
                        const float* xr = xr0 + mc;
                        float xv[7];
#pragma unroll
                        for (int k = 0; k < 7; ++k) xv[k] = xr[k - 3];   // x[mc-3 .. mc+3]
                        float ue = 0.f, uo = 0.f;
#pragma unroll
                        for (int k = 0; k < 6; ++k) {
                            ue = fmaf(p.filt.up[2 * k + 1], xv[5 - k], ue);
                            uo = fmaf(p.filt.up[2 * k], xv[6 - k], uo);
                        }
                        const float se = fmaf(actm::sin_sq_fast(al, ue), ib, ue);
                        const float so = fmaf(actm::sin_sq_fast(al, uo), ib, uo);
                        const int ie = 2 * m - n_start;
                        const float ve = (m > L - 1) ? so : se;
                        const float vo = (m < 0) ? se : so;
                        if (ie >= 0 && ie < SW) srow[ie] = ve;
                        if (ie + 1 >= 0 && ie + 1 < SW) srow[ie + 1] = vo;
                    }
                }
                if (gi + 1 < gtotal) prefetch(gi + 1);
                prod_sync();   // all 8 snake rows ready
                // ---- decimate into the A operand: 2 rows x 2 channels per thread
                const int npairs = (ROWS + 1) >> 1;
                for (int it = ptid; it < 4 * npairs; it += NPROD) {
                    const int rp = it >> 2, cq = it & 3;   // row pair, channel pair
                    const int q0 = 2 * rp;
                    float a0[2], a1[2];
#pragma unroll
                    for (int c = 0; c < 2; ++c) {
                        const float2* sr = reinterpret_cast<const float2*>(sw + (2 * cq + c) * pl.SWs + 2 * q0);
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
#pragma unroll
                    for (int rr = 0; rr < 2; ++rr) {
                        const int q = q0 + rr;
                        if (q >= ROWS) break;
                        const bool in = a_start + q >= 0 && a_start + q < L;   // conv zero padding
                        float h[2], l[2];
#pragma unroll
                        for (int c = 0; c < 2; ++c) {
                            const float v = in ? (rr == 0 ? a0[c] : a1[c]) : 0.f;
                            h[c] = bf16_round(v);
                            l[c] = v - h[c];
                        }
                        const size_t off = (size_t)q * 16 + cq * 4;
                        *reinterpret_cast<uint32_t*>(a_hi + off) = pack_bf16(h[0], h[1]);
                        *reinterpret_cast<uint32_t*>(a_lo + off) = pack_bf16(l[0], l[1]);
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
        const long long obase = (long long)b * Cout * L;
        if (epi_go && part * CPP < NT) {
            const uint32_t lane_addr = tmem + ((uint32_t)(q4 * 32) << 16);
#pragma unroll
            for (int mt = 0; mt < MT; ++mt) {
                const int t = t0 + mt * 128 + q4 * 32 + lane;
                for (int cb = part * CPP; cb < part * CPP + CPP && cb < NT; cb += 16) {
                    float v[16], w[16];
                    const int accbase = mt * NACC;
                    ptx::tmem_ld16(lane_addr + (uint32_t)(accbase * NT + cb), v);
#pragma unroll
                    for (int a = 1; a < NACC; ++a) {
                        ptx::tmem_ld16(lane_addr + (uint32_t)((accbase + a) * NT + cb), w);
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
// GEMM operands for the persistent kernel below: the activation (or plain split) has already
// been written to memory as the A operand (rows of 8 bf16 channels, heads and tails in separate
// arrays, with the conv's zero padding materialised), so both operands arrive by 1-D bulk
// copies.
// ----------------------------------------------------------------------------------------------

struct GemmJob {
    const uint8_t* a_hi;   // [B, Cin/8, Lpad] rows of 16 bytes
    const uint8_t* a_lo;
    const uint16_t* w;     // pre-split operand blocks
    const float* bias;
    const float* res;
    float* out;
    int K, dil, pad;
    int g0;               // first 8-channel group of the job's input-channel slice
    int span;             // window rows a tile reads beyond its 128 MT output rows
    // polyphase transposed conv (R > 1): window row offset and output phase of every tap
    int8_t tap_row[16];
    int8_t tap_phase[16];
};

struct GemmParams {
    GemmJob job[MH3A_MAX_RESBLOCKS];
    int Cin, Cout, L, B, tiles_t;
    int a_groups;         // 8-channel groups per item in the A arrays (Cin / 8 unless split)
    int pad_l;            // zero rows before the sequence in the A arrays
    long long Lpad;       // rows per (item, channel group) in the A arrays
    int tpu;              // tap units per weight bulk copy (set by the launcher)
    int* err;
    int* sched;           // [next tile, CTAs done]: zero before a launch, left zero after it
    // Fused input split of the next upsampler (R == 1, three jobs = the stage's residual blocks;
    // ms_hi null: off).  See mean_split_rows.
    uint8_t* ms_hi;       // [B, Cout/8, ms_Lpad] rows of 16 bytes (heads), pad ms_padl rows
    uint8_t* ms_lo;       // tails
    long long ms_Lpad;
    int ms_padl;
    int ms_blk[MH3A_MAX_RESBLOCKS];   // residual block of job z
    int ms_z[3];                      // job of block j
    const float* ms_x[3];             // the blocks' outputs, in block order
};

// ----------------------------------------------------------------------------------------------
// persistent AMP GEMM: one CTA per SM walks a list of output tiles (job, item, 128 MT time rows,
// NT output channels).  The tile's K loop is cut into passes of at most 16 MMA K-steps; each
// pass accumulates head x head and both cross products into one of two TMEM buffers, and the
// epilogue warps fold the finished buffer into fp32 registers (round to nearest) while the
// tensor core fills the other.  A pass therefore holds at most 48 truncating accumulations,
// the epilogue of one tile overlaps the MMAs of the next, and A / B stream through rings of
// bulk copies that run several stages ahead.
// ----------------------------------------------------------------------------------------------
// EW epilogue warps (EW / 4 per TMEM lane quarter) after warp 0 (MMA) and warp 1 (loader).
constexpr int ps_threads(int EW) { return 64 + 32 * EW; }
constexpr int PS_MAXS = 8;                              // ring stages (max)
constexpr int PS_TQ = 16;                               // tile-index queue entries
constexpr int PS_BAR_BYTES = 8 * (4 * PS_MAXS + 5 + PS_TQ) + 8 + 4 * PS_TQ;   // barriers, flags, queue
constexpr int PS_BUFCOLS = 256;                         // TMEM columns per accumulator buffer (max)

struct PsPlan {
    int RS;             // window rows per channel group (max over jobs)
    int SA, SB;         // bytes per A / B ring stage
    int nsa, nsb;       // ring depths
    int offB, offBar;
    int smem;
};

struct PsSched {
    int ntiles, n_ot, per_job;   // tiles in all, output-channel tiles, tiles per job
    int pu;                      // tap units per pass
};

// Tile k of the launch (jobs sorted by cost, heaviest first).
struct PsTile {
    int z, b, t0, ot;
};

template <int MT>
__device__ __forceinline__ PsTile ps_tile(const GemmParams& p, const PsSched& sc, int k) {
    PsTile T;
    T.z = k / sc.per_job;
    int r = k - T.z * sc.per_job;
    const int per_b = p.tiles_t * sc.n_ot;
    T.b = r / per_b;
    r -= T.b * per_b;
    const int tt = r / sc.n_ot;
    T.ot = r - tt * sc.n_ot;
    T.t0 = tt * 128 * MT;
    return T;
}


// Residual group g (channels GW g .. GW g + GW - 1 of a warp's columns) of one row, rp = the row's
// first column; channels past Cout (16-wide tiles only) read nothing.
template <int NT, int GW>
__device__ __forceinline__ void load_res_group(float (&rq)[GW], const float* rp, int g, long long Lout, int o_base,
                                               int Cout) {
#pragma unroll
    for (int c = 0; c < GW; ++c) {
        const int cc = GW * g + c;
        rq[c] = (NT > 16 || o_base + cc < Cout) ? __ldg(rp + (long long)cc * Lout) : 0.f;
    }
}

// acc[GW g + c] += rq[c] with a run-time g: one compile-time branch per group keeps every
// accumulator index a constant (and the accumulators in registers).  The adds are volatile asm
// so that they stay ahead of the tensor-memory loads that follow them, which would otherwise
// need registers while rq is still live.
template <int CW, int GW, int N>
__device__ __forceinline__ void add_res_group(float (&acc)[N], const float (&rq)[GW], int g) {
#pragma unroll
    for (int gg = 0; gg < CW / GW; ++gg) {
        if (gg == g) {
#pragma unroll
            for (int c = 0; c < GW; ++c) asm volatile("add.rn.f32 %0, %0, %1;" : "+f"(acc[GW * gg + c]) : "f"(rq[c]));
        }
    }
}

// The fused input split of the next upsampler.  In the last layer of an AMP stage the three
// jobs are the residual blocks; the scheduler then hands out units of three tiles -- the same
// item, rows and channels for blocks 0, 1 and 2, in that order -- so that one CTA, and in it
// the same epilogue thread, stores all three outputs of each of its rows and columns.  At the
// block-2 tile that thread forms the stage output -- the mean ((x0 + x1) + x2) / 3 in block
// order, the arithmetic of the standalone split (k_split_rows), from its own two earlier stores
// and its registers -- and writes it as head/tail rows of 8 channels into the upsampler's A
// operand.  The threads that hold the sequence's first and last rows also zero the kMsZeroRows
// rows before and after it, which the upsampler's window reads (its taps reach one row to
// either side).
constexpr int kMsZeroRows = 8;
// Epilogue warps of at most this many columns run it (the 16- to 64-channel stages); wider
// warps would spill (their stage keeps the standalone split).
constexpr int kMsMaxCW = 32;

template <int CW>
__device__ __forceinline__ void mean_split_rows(const GemmParams& p, int b, int t, int o_base, long long idx0,
                                                const float (&acc)[CW]) {
    const int L = p.L, ngroups = p.Cout / 8;
    uint4* hi = reinterpret_cast<uint4*>(p.ms_hi);
    uint4* lo = reinterpret_cast<uint4*>(p.ms_lo);
    const uint4 zero = make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
    for (int gq = 0; gq < CW / 8; ++gq) {
        const int g = o_base / 8 + gq;
        if (g >= ngroups) continue;   // 16-wide tiles past Cout
        const long long rbase = ((long long)b * ngroups + g) * p.ms_Lpad + p.ms_padl;
        if (t < L) {
            float v[8];
#pragma unroll
            for (int c = 0; c < 8; ++c) {
                const long long off = idx0 + (long long)(gq * 8 + c) * L;
                const float x0 = __ldcg(p.ms_x[0] + off), x1 = __ldcg(p.ms_x[1] + off);
                v[c] = (x0 + x1 + acc[gq * 8 + c]) * (1.0f / 3.0f);
            }
            uint4 hv, lv;
            actm::split2(v[0], v[1], &hv.x, &lv.x);
            actm::split2(v[2], v[3], &hv.y, &lv.y);
            actm::split2(v[4], v[5], &hv.z, &lv.z);
            actm::split2(v[6], v[7], &hv.w, &lv.w);
            hi[rbase + t] = hv;
            lo[rbase + t] = lv;
        }
        if (t == 0)
            for (int r = 1; r <= kMsZeroRows; ++r) {
                hi[rbase - r] = zero;
                lo[rbase - r] = zero;
            }
        if (t == L - 1)
            for (int r = 0; r < kMsZeroRows; ++r) {
                hi[rbase + L + r] = zero;
                lo[rbase + L + r] = zero;
            }
    }
}

// KGT = 8-channel groups per K chunk (4: 32 input channels; 2: 16).  KGT = 1 serves 8-channel
// layers: one MMA K-step of 16 then covers the same 8 channels at two consecutive taps -- the
// second core matrix along K is the window shifted by `dil` rows, i.e. the A descriptor's
// leading-byte offset is dil * 16 -- and the weight block of a unit holds that tap pair (a
// zero block stands in for the tap past the last one).
// R > 1: the polyphase transposed conv (upsampler).  Rows are input samples u; tap j reads the
// window at row offset tap_row[j] and accumulates into the region of its output phase
// tap_phase[j]; the epilogue writes phase phi of row u to output sample R u + phi.  With
// GRP (R > 2) a unit is instead a group of taps sharing one row offset: its weight block holds
// all R phases (zero rows where the group has no tap), so one MMA of N = R NT covers every
// phase region and the group's first unit initialises all of them.  A pass is
// then one whole chunk, so that the first tap of every phase (j < R) starts its region.
// Accumulator columns per M tile, TMEM columns per buffer, and CTAs per SM.  A GEMM with 8
// epilogue warps whose accumulators take at most 128 columns per buffer (the 16- and 32-channel
// AMP convs, the rate-2 upsamplers) runs two CTAs per SM: their double buffers fill the 512
// TMEM columns exactly, their threads the register file, and each takes at most half the
// shared memory (so no third CTA, of this launch or the next, can wait on tensor memory).
// Measured per launch against one CTA per SM: AMP 32 channels 48.1 -> 41.9 us, 16 channels
// 49.9 -> 45.0 us (with 16 epilogue warps there); upsamplers 2-6 56 -> 50, 40 -> 38, 36 -> 34,
// 21 -> 18, 25 -> 19 us.
__host__ __device__ constexpr int ps_rstr(int NT, int R) { return interleaved_b(NT, R) ? 2 * NT : R * NT; }
__host__ __device__ constexpr int ps_ctas(int MT, int NT, int EW, int R) {
    return (EW == 8 && MT * ps_rstr(NT, R) <= 128) ? 2 : 1;
}
__host__ __device__ constexpr int ps_bufcols(int MT, int NT, int EW, int R) {
    return ps_ctas(MT, NT, EW, R) == 2 ? 128 : PS_BUFCOLS;
}

template <int MT, int NT, int KGT, int EW, int R>
__global__ void __launch_bounds__(ps_threads(EW), ps_ctas(MT, NT, EW, R))
    k_gemm_ps(const GemmParams p, const PsSched sc, const PsPlan pl) {
    extern __shared__ __align__(1024) uint8_t smem[];
    ptx::grid_dep_wait();   // launched as a programmatic dependent (see launch_dependent)
    constexpr bool ILV = interleaved_b(NT, R);            // two-MMA K-steps, head | cross columns
    constexpr int RSTR = ILV ? 2 * NT : R * NT;            // accumulator columns per M tile
    constexpr int BUFC = ps_bufcols(MT, NT, EW, R);        // TMEM columns per accumulator buffer
    static_assert(MT * RSTR <= BUFC, "one accumulator buffer holds MT x RSTR columns");
    static_assert(R == 1 || KGT >= 2, "the upsampler uses 16- or 32-channel chunks");
    static_assert(KGT == 1 || KGT == 2 || KGT == 4, "channel groups per chunk");
    static_assert(EW == 8 || EW == 16, "epilogue warps");
    static_assert((4 * MT * NT / EW) % 16 == 0 && 4 * MT * NT / EW <= NT, "epilogue column split");
    constexpr int BG = (KGT == 1) ? 2 : KGT;
    constexpr bool GRP = convt_grouped(R);                 // units are row-offset groups
    constexpr int BROWS = GRP ? R * NT : NT;                // B rows per core column of a unit
    constexpr int TAPB = 2 * BG * BROWS * 16;
    constexpr int CW = 4 * MT * NT / EW;                // accumulator columns per epilogue warp
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int Cin = p.Cin, Cout = p.Cout, L = p.L;
    const int nchunks = Cin / (8 * KGT);
    const int TPU = p.tpu, PU = sc.pu;
    const int RS = pl.RS, nsa = pl.nsa, nsb = pl.nsb;

    uint8_t* As = smem;
    uint8_t* Bs = smem + pl.offB;
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + pl.offBar);
    uint64_t* a_full = bars;
    uint64_t* a_empty = bars + PS_MAXS;
    uint64_t* b_full = bars + 2 * PS_MAXS;
    uint64_t* b_empty = bars + 3 * PS_MAXS;
    uint64_t* acc_full = bars + 4 * PS_MAXS;
    uint64_t* acc_empty = acc_full + 2;
    uint64_t* done_bar = acc_full + 4;
    uint64_t* tile_full = done_bar + 1;                  // [PS_TQ] a tile index was queued
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(tile_full + PS_TQ);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
    volatile int* tile_q = abort_flag + 1;               // [PS_TQ] tile indices, -1 = no more
    float* bias_s = reinterpret_cast<float*>(smem + pl.offBar + PS_BAR_BYTES);   // [EW][CW] per warp

    if (threadIdx.x == 0) {
        for (int s = 0; s < nsa; ++s) {
            ptx::mbar_init(&a_full[s], 1);
            ptx::mbar_init(&a_empty[s], 1);
        }
        for (int s = 0; s < nsb; ++s) {
            ptx::mbar_init(&b_full[s], 1);
            ptx::mbar_init(&b_empty[s], 1);
        }
        for (int s = 0; s < 2; ++s) {
            ptx::mbar_init(&acc_full[s], 1);
            ptx::mbar_init(&acc_empty[s], EW);
        }
        ptx::mbar_init(done_bar, 1);
        for (int q = 0; q < PS_TQ; ++q) ptx::mbar_init(&tile_full[q], 1);
        *abort_flag = (*reinterpret_cast<volatile int*>(p.err) != 0) ? 1 : 0;
        ptx::fence_mbar_init();
    }
    if (warp == 0) {
        ptx::tmem_alloc(tmem_slot, 2 * BUFC);
        ptx::tmem_relinquish();
    }
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == 0) {
        // ---------------------------------------------------------------- MMA issuer
        // The whole warp walks the loop in lock step, so that every descriptor and address is
        // warp-uniform; one elected lane issues each group of three MMAs and each commit.
        // Descriptors are built once per ring slot and advanced by adding 16-byte offsets to
        // their low word (the start-address field).
        constexpr uint32_t idesc = ptx::idesc_bf16(128, BROWS);
        constexpr uint32_t idesc_2n = ptx::idesc_bf16(128, ILV ? 2 * NT : NT);
        constexpr uint32_t b_lbo = (ILV ? 2 * NT : BROWS) * 16;   // bytes between core columns
        constexpr int KK = (KGT == 1) ? 1 : KGT / 2;   // K-steps per tap unit
        const uint32_t a_smem = ptx::smem_u32(As), b_smem = ptx::smem_u32(Bs);
        bool ok = *abort_flag == 0;
        int sa = 0, sb = 0, buf = 0;
        uint32_t pa = 0, pb = 0, pacc = 0;   // phase bits of the slots in use
        for (int i = 0; ok; ++i) {
            if (!__all_sync(0xffffffffu, ptx::mbar_wait(&tile_full[i % PS_TQ], (i / PS_TQ) & 1, kWaitLimit))) {
                ok = false;
                break;
            }
            const int k = tile_q[i % PS_TQ];
            if (k < 0) break;
            const PsTile T = ps_tile<MT>(p, sc, k);
            const GemmJob& J = p.job[T.z];
            const int K = J.K, dil = J.dil;
            const int KU = (KGT == 1) ? (K + 1) / 2 : K;
            const uint32_t step = (uint32_t)((KGT == 1 ? 2 : 1) * dil);   // window rows per unit
            const uint32_t a_lbo = (KGT == 1) ? (uint32_t)dil * 16 : (uint32_t)RS * 16;
            for (int chunk = 0; chunk < nchunks && ok; ++chunk) {
                if (!__all_sync(0xffffffffu, ptx::mbar_wait(&a_full[sa], pa, kWaitLimit))) { ok = false; break; }
                ptx::tc_fence_after();
                const uint32_t ah0 = ptx::desc_lo(a_smem + sa * pl.SA, a_lbo);
                int ucopy = 0, upass = 0;
                uint32_t bh0 = 0, ashift = 0;
                for (int unit = 0; unit < KU; ++unit, ashift += step) {
                    if (ucopy == 0) {
                        if (!__all_sync(0xffffffffu, ptx::mbar_wait(&b_full[sb], pb, kWaitLimit))) { ok = false; break; }
                        ptx::tc_fence_after();
                        bh0 = ptx::desc_lo(b_smem + sb * pl.SB, b_lbo);
                    }
                    if (upass == 0) {
                        if (!__all_sync(0xffffffffu, ptx::mbar_wait(&acc_empty[buf], pacc ^ 1, kWaitLimit))) { ok = false; break; }
                        ptx::tc_fence_after();
                    }
                    // KGT >= 2: unit = tap, K-steps over channel-group pairs.  KGT == 1: unit =
                    // tap pair, one K-step whose two core-matrix columns are taps 2u and 2u+1.
                    const uint32_t bh = bh0 + (uint32_t)ucopy * (TAPB >> 4);
                    uint32_t dbase = tmem + (uint32_t)(buf * BUFC);
                    uint32_t arow = ashift;
                    bool first = upass == 0;
                    if (GRP) {
                        arow = (uint32_t)J.tap_row[unit];
                        first = unit == 0;
                    } else if (R > 1) {
                        arow = (uint32_t)J.tap_row[unit];
                        dbase += (uint32_t)(J.tap_phase[unit] * NT);
                        first = unit < R;
                    }
#pragma unroll
                    for (int kk = 0; kk < KK; ++kk) {
#pragma unroll
                        for (int mt = 0; mt < MT; ++mt) {
                            const uint32_t a = ah0 + arow + (uint32_t)(2 * kk * RS + mt * 128);
                            const uint32_t d = dbase + (uint32_t)(mt * RSTR);
                            const uint32_t acc = (first && kk == 0) ? 0u : 1u;
                            if (ILV) {
                                // core columns 2kk, 2kk+1 hold [heads | tails] of NT rows each
                                const uint32_t bk = bh + (uint32_t)(2 * kk * 2 * NT);
                                ptx::mma2_bf16_elect(d, d + (uint32_t)NT, ptx::desc64(a),
                                                     ptx::desc64(a + (uint32_t)(KGT * RS)), ptx::desc64(bk), idesc_2n,
                                                     idesc, acc);
                            } else {
                                const uint32_t bhk = bh + (uint32_t)(2 * kk * BROWS);
                                const uint32_t blk = bhk + (uint32_t)(BG * BROWS);
                                ptx::mma3_bf16_elect(d, ptx::desc64(a), ptx::desc64(a + (uint32_t)(KGT * RS)),
                                                     ptx::desc64(bhk), ptx::desc64(blk), idesc, acc);
                            }
                        }
                    }
                    ++ucopy;
                    ++upass;
                    if (ucopy == TPU || unit == KU - 1) {
                        ptx::mma_commit_elect(&b_empty[sb]);
                        ucopy = 0;
                        if (++sb == nsb) { sb = 0; pb ^= 1; }
                    }
                    if (upass == PU || unit == KU - 1) {
                        ptx::mma_commit_elect(&acc_full[buf]);
                        upass = 0;
                        buf ^= 1;
                        if (buf == 0) pacc ^= 1;
                    }
                }
                if (!ok) break;
                ptx::mma_commit_elect(&a_empty[sa]);
                if (++sa == nsa) { sa = 0; pa ^= 1; }
                if (*abort_flag) ok = false;
                ok = __all_sync(0xffffffffu, ok);
            }
        }
        if (!ok && lane == 0) {
            *abort_flag = 1;
            atomicExch(p.err, 5);
        }
        // every MMA issued has completed before the CTA releases its tensor memory
        ptx::mma_commit_elect(done_bar);
        ptx::mbar_wait(done_bar, 0, kWaitLimit);
        __syncwarp();
    } else if (warp == 1) {
        // ---------------------------------------------------------------- A and B loader
        if (lane == 0) {
            const size_t unit_elems = (size_t)2 * BG * BROWS * 8;
            bool ok = *abort_flag == 0;
            int ia = 0, ib = 0;
            bool drained = false;   // the scheduler handed this CTA its end marker
            int unit = 0;
            for (int i = 0; ok; ++i) {
                // dynamic schedule: tiles go out heaviest job first, each to the CTA that asks
                // next; with the fused split, units of the three blocks' tiles in block order
                int k;
                if (R == 1 && p.ms_hi != nullptr) {
                    if (i % 3 == 0) unit = atomicAdd(p.sched, 1);
                    k = unit < sc.per_job ? p.ms_z[i % 3] * sc.per_job + unit : -1;
                } else {
                    k = atomicAdd(p.sched, 1);
                    if (k >= sc.ntiles) k = -1;
                }
                tile_q[i % PS_TQ] = k;
                ptx::mbar_arrive(&tile_full[i % PS_TQ]);
                if (k < 0) {
                    drained = true;
                    break;
                }
                const PsTile T = ps_tile<MT>(p, sc, k);
                const GemmJob& J = p.job[T.z];
                const int K = J.K;
                const int KU = (KGT == 1) ? (K + 1) / 2 : K;
                const int NUC = (KU + TPU - 1) / TPU;
                const int ROWS = 128 * MT + J.span;
                const uint32_t a_bytes = (uint32_t)(2 * KGT * ROWS * 16);
                const long long row0 = p.pad_l + T.t0 - J.pad;   // first window row in the A arrays
                const uint16_t* wsrc = J.w + (size_t)T.ot * nchunks * KU * unit_elems;
                for (int chunk = 0; chunk < nchunks && ok; ++chunk) {
                    const int sa = ia % nsa;
                    if (!ptx::mbar_wait(&a_empty[sa], ((ia / nsa) & 1) ^ 1, kWaitLimit)) { ok = false; break; }
                    ptx::mbar_arrive_expect_tx(&a_full[sa], a_bytes);
                    for (int part = 0; part < 2; ++part) {
                        const uint8_t* base = part == 0 ? J.a_hi : J.a_lo;
                        for (int g = 0; g < KGT; ++g) {
                            const long long grp = (long long)T.b * p.a_groups + J.g0 + chunk * KGT + g;
                            ptx::bulk_g2s(As + (size_t)sa * pl.SA + ((size_t)(part * KGT + g) * RS) * 16,
                                          base + (grp * p.Lpad + row0) * 16, (uint32_t)(ROWS * 16), &a_full[sa]);
                        }
                    }
                    ++ia;
                    for (int uc = 0; uc < NUC; ++uc) {
                        const int sb = ib % nsb;
                        if (!ptx::mbar_wait(&b_empty[sb], ((ib / nsb) & 1) ^ 1, kWaitLimit)) { ok = false; break; }
                        // tap units [uc * TPU, min(KU, (uc + 1) * TPU)) are contiguous in the packing
                        const int nunits = min(KU, (uc + 1) * TPU) - uc * TPU;
                        const uint32_t bytes = (uint32_t)(nunits * TAPB);
                        ptx::mbar_arrive_expect_tx(&b_full[sb], bytes);
                        ptx::bulk_g2s(Bs + (size_t)sb * pl.SB,
                                      wsrc + ((size_t)chunk * KU + (size_t)uc * TPU) * unit_elems, bytes, &b_full[sb]);
                        ++ib;
                    }
                    if (*abort_flag) ok = false;
                }
            }
            if (!ok) {
                *abort_flag = 1;
                atomicExch(p.err, 6);
            }
            // the last CTA to drain the schedule resets it for the next launch
            if (drained && atomicAdd(p.sched + 1, 1) == (int)gridDim.x - 1) {
                atomicExch(p.sched, 0);
                atomicExch(p.sched + 1, 0);
            }
            // let the copies still in flight land before the CTA can exit
            for (int c = (ia > nsa ? ia - nsa : 0); c < ia; ++c)
                ptx::mbar_wait(&a_full[c % nsa], (c / nsa) & 1, kWaitLimit);
            for (int v = (ib > nsb ? ib - nsb : 0); v < ib; ++v)
                ptx::mbar_wait(&b_full[v % nsb], (v / nsb) & 1, kWaitLimit);
        }
        __syncwarp();
    } else {
        // ---------------------------------------------------------------- epilogue (warps 2 .. EW+1)
        const int e = warp - 2;
        const int q4 = warp & 3;               // TMEM lane quarter this warp may access
        const int col0 = (e >> 2) * CW;        // first channel column of this warp ([mt][NT] order)
        const int mt = col0 / NT, oc0 = col0 % NT;
        // regions [mt][phase][NT]: this warp's columns of phase phi start at + phi * NT
        const uint32_t lane_addr = tmem + ((uint32_t)(q4 * 32) << 16) + (uint32_t)(mt * RSTR + oc0);
        const long long Lout = (long long)L * R;
        bool ok = *abort_flag == 0;
        int ip = 0;
        for (int i = 0; ok; ++i) {
            if (!ptx::mbar_wait(&tile_full[i % PS_TQ], (i / PS_TQ) & 1, kWaitLimit)) {
                ok = false;
                break;
            }
            const int k = tile_q[i % PS_TQ];
            if (k < 0) break;
            const PsTile T = ps_tile<MT>(p, sc, k);
            const GemmJob& J = p.job[T.z];
            const int KU = (KGT == 1) ? (J.K + 1) / 2 : J.K;
            const int npass = nchunks * ((KU + PU - 1) / PU);
            const int t = T.t0 + mt * 128 + q4 * 32 + lane;   // the row (input sample when R > 1)
            const int o_base = T.ot * NT + oc0;
            const long long idx0 = ((long long)T.b * Cout + o_base) * Lout + (long long)R * t;
            // The accumulator starts from bias + residual.  Wide warps (CW >= 64) stream the
            // residual in, 16 channels per pass, each group loaded after one pass's drain and
            // added at the next: read at the tile's start, those reads would queue behind the
            // tensor core's operand traffic while the MMA warp waits for the first drain.
            // Narrow warps read their few residual values at the tile's start.  The bias slice
            // goes through shared memory (CW / 32 loads per lane, then broadcasts).
            constexpr bool kSpread = R == 1 && CW >= 64;
            constexpr int GW = 16;                            // residual group width
            constexpr int G = CW / GW;                        // residual groups per warp
            const bool has_res = R == 1 && J.res != nullptr && t < L;
            const float* rp = has_res ? J.res + idx0 : nullptr;
            float* bsl = bias_s + (warp - 2) * CW;
            for (int c = lane; c < CW; c += 32) bsl[c] = (J.bias && o_base + c < Cout) ? __ldg(J.bias + o_base + c) : 0.f;
            __syncwarp();
            float acc[R * CW];
#pragma unroll
            for (int c = 0; c < CW; ++c) acc[c] = 0.f;
            // 16-column warps keep the residual apart and add it after the last pass, so that
            // the first drain does not wait for the loads
            constexpr bool kLate = R == 1 && CW == 16;
            float rl[kLate ? CW : 1];
            if constexpr (kLate) {
                if (has_res) {
#pragma unroll
                    for (int c = 0; c < CW; ++c) rl[c] = (NT > 16 || o_base + c < Cout) ? __ldg(rp + (long long)c * Lout) : 0.f;
                }
            }
            if (!kLate && !kSpread && has_res) {
                if (NT > 16 || o_base + CW <= Cout) {
#pragma unroll
                    for (int c = 0; c < CW; ++c) acc[c] = __ldg(rp + (long long)c * Lout);
                } else {   // only 16-wide tiles pad past Cout
#pragma unroll
                    for (int c = 0; c < CW; ++c)
                        if (o_base + c < Cout) acc[c] = __ldg(rp + (long long)c * Lout);
                }
            }
#pragma unroll
            for (int cb = 0; cb < CW; cb += 4) {
                const float4 b4 = *reinterpret_cast<const float4*>(bsl + cb);
                acc[cb] += b4.x;
                acc[cb + 1] += b4.y;
                acc[cb + 2] += b4.z;
                acc[cb + 3] += b4.w;
            }
#pragma unroll
            for (int ph = 1; ph < R; ++ph)
#pragma unroll
                for (int c = 0; c < CW; ++c) acc[ph * CW + c] = acc[c];
            float rq[kSpread ? GW : 1];
            for (int ps = 0; ps < npass; ++ps, ++ip) {
                const int buf = ip & 1;
                if (!ptx::mbar_wait(&acc_full[buf], (ip >> 1) & 1, kWaitLimit)) { ok = false; break; }
                ptx::tc_fence_after();
                // the group loaded after the previous pass (added before the drain, so that its
                // registers are free again during the drain)
                if constexpr (kSpread)
                    if (has_res && ps >= 1 && ps <= G) add_res_group<CW, GW>(acc, rq, ps - 1);
#pragma unroll
                for (int ph = 0; ph < R; ++ph) {
                    if constexpr (kSpread) {
                        // 8 columns at a time: the residual group holds 16 registers here
#pragma unroll
                        for (int cb = 0; cb < CW; cb += 8) {
                            float v[8];
                            ptx::tmem_ld8(lane_addr + (uint32_t)(buf * BUFC + ph * NT + cb), v);
#pragma unroll
                            for (int c = 0; c < 8; ++c) acc[ph * CW + cb + c] += v[c];
                        }
                    } else {
#pragma unroll
                        for (int cb = 0; cb < CW; cb += 16) {
                            float v[16];
                            ptx::tmem_ld16(lane_addr + (uint32_t)(buf * BUFC + ph * NT + cb), v);
                            if (ILV) {
                                float x[16];
                                ptx::tmem_ld16(lane_addr + (uint32_t)(buf * BUFC + NT + cb), x);
#pragma unroll
                                for (int c = 0; c < 16; ++c) v[c] += x[c];
                            }
#pragma unroll
                            for (int c = 0; c < 16; ++c) acc[ph * CW + cb + c] += v[c];
                        }
                    }
                }
                ptx::tc_fence_before();
                __syncwarp();
                if (lane == 0) ptx::mbar_arrive(&acc_empty[buf]);
                if constexpr (kSpread)
                    if (has_res && ps < G) load_res_group<NT, GW>(rq, rp, ps, Lout, o_base, Cout);
            }
            if constexpr (kSpread) {
                if (has_res && ok && npass <= G) {
                    // fewer passes than groups: the last loaded group and the ones never loaded
                    if (npass >= 1) add_res_group<CW, GW>(acc, rq, npass - 1);
                    for (int g = npass; g < G; ++g) {
                        load_res_group<NT, GW>(rq, rp, g, Lout, o_base, Cout);
                        add_res_group<CW, GW>(acc, rq, g);
                    }
                }
            }
            if (!ok || *abort_flag) {
                ok = false;
                break;
            }
            if constexpr (kLate) {
                if (has_res) {
#pragma unroll
                    for (int c = 0; c < CW; ++c) acc[c] += rl[c];
                }
            }
            if (t < L) {
#pragma unroll
                for (int c = 0; c < CW; ++c) {
                    if (NT <= 16 && o_base + c >= Cout) continue;   // channels past Cout pad the tile
#pragma unroll
                    for (int ph = 0; ph < R; ++ph) J.out[idx0 + (long long)c * Lout + ph] = acc[ph * CW + c];
                }
            }
            if constexpr (R == 1 && CW <= kMsMaxCW) {
                // the block-2 tile of a unit: this thread stored blocks 0 and 1 of these rows
                // and columns in the unit's two previous tiles
                if (p.ms_hi != nullptr && p.ms_blk[T.z] == 2) mean_split_rows<CW>(p, T.b, t, o_base, idx0, acc);
            }
            __syncwarp();   // the bias slice is rewritten for the next tile
        }
        if (!ok) {
            *abort_flag = 1;
            atomicExch(p.err, 7);
        }
    }
    ptx::grid_dep_launch();   // every role is done: the next grid may be scheduled
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    if (warp == 0) ptx::tmem_dealloc(tmem, 2 * BUFC);
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

// Output-channel tile of each layer kind (the weight blocks are laid out for it).
int ntile_amp(int C) { return C >= 256 ? 256 : (C >= 128 ? 128 : (C >= 64 ? 64 : C)); }
int ntile_pre(int) { return 256; }
int ntile_convt(int Cout, int r) {
    if (r > 2) return Cout >= 32 ? 32 : Cout;
    return Cout >= 64 ? 64 : (Cout > 16 ? Cout : 16);   // narrow outputs padded to 16 columns
}

// 8-channel groups per K chunk of an upsampler: 32-channel chunks, or one 16-channel chunk.
int kgt_convt(int Cin) { return Cin % 32 == 0 ? 4 : (Cin == 16 ? 2 : 0); }

template <int MT, int NT>
TcPlan make_plan(const TcParams& p, int njobs) {
    int span = 0;
    for (int j = 0; j < njobs; ++j) span = std::max(span, (p.job[j].K - 1) * p.job[j].dil);
    TcPlan pl{};
    pl.RS = 128 * MT + span;
    pl.XWs = pl.RS + 12;
    pl.SWs = 2 * pl.RS + 12;   // even (8-byte rows), room for the last pair
    pl.SA = 2 * KG * pl.RS * 16;
    pl.SB = 2 * KG * NT * 16;
    pl.offB = NSA * pl.SA;
    pl.offX = pl.offB + NSB * pl.SB;
    const int stage_bytes = (2 * 8 * pl.XWs + 8 * pl.SWs) * 4;
    pl.offBar = (pl.offX + stage_bytes + 15) / 16 * 16;
    pl.smem = pl.offBar + 8 * (2 * NSA + 2 * NSB + 1) + 16;
    return pl;
}

template <int MT, int NT, int NACC>
int launch_tc(const TcParams& p0, int njobs, cudaStream_t s) {
    TcParams p = p0;
    if (NACC - 1 > p.Cin / KC) return -1;  // every head accumulator must receive a chunk
    if (p.Cin % KC != 0 || p.Cout % NT != 0) return -1;
    p.tiles_t = (p.L + 128 * MT - 1) / (128 * MT);
    const TcPlan pl = make_plan<MT, NT>(p, njobs);
    if (pl.smem > 227 * 1024) return -1;
    auto kern = k_conv_tc<MT, NT, NACC>;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, pl.smem) != cudaSuccess) return -1;
    dim3 grid(p.tiles_t * p.B, p.Cout / NT, njobs);
    kern<<<grid, NTHREADS, pl.smem, s>>>(p, pl);
    return cudaPeekAtLastError() == cudaSuccess ? 1 : -1;
}

// Fused AMP kernel (allocation-free stage entry point): MT x 128 time rows, NT output channels,
// NACC accumulators per M tile (MT * NT * NACC <= 512 tensor-memory columns).  NT follows the
// weight packing shared with the persistent GEMM, so the two widest stages get 256-column tiles
// and a single head accumulator (stage-0 relative error about 4e-5, against 1e-5 with three).
int dispatch_amp(const TcParams& p, int njobs, cudaStream_t s) {
    switch (p.Cin) {
        case 512: return launch_tc<1, 256, 2>(p, njobs, s);
        case 256: return launch_tc<1, 256, 2>(p, njobs, s);
        case 128: return launch_tc<1, 128, 4>(p, njobs, s);
        case 64: return launch_tc<2, 64, 3>(p, njobs, s);
        case 32: return launch_tc<2, 32, 2>(p, njobs, s);
        default: return -1;
    }
}

int sm_count() {
    static int cache[64] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 0;
    if (cache[dev] == 0) {
        int n = 0;
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
        cache[dev] = n;
    }
    return cache[dev];
}

// Every job must carry K, pad (window rows before a tile's first output row) and span (window
// rows past its last); R > 1 jobs also their tap tables.
template <int MT, int NT, int KGT, int EW, int R>
int launch_gemm_ps(const GemmParams& p0, int njobs, cudaStream_t s) {
    GemmParams p = p0;
    const int kc = 8 * KGT;
    if (p.Cin % kc != 0 || njobs < 1 || !p.sched || !p.err) return -1;
    if (NT > 16 && p.Cout % NT != 0) return -1;   // the epilogue pads channels past Cout only in 16-wide tiles
    if (p.a_groups == 0) p.a_groups = p.Cin / 8;
    p.tiles_t = (p.L + 128 * MT - 1) / (128 * MT);
    int span = 0, kumax = 1;
    for (int j = 0; j < njobs; ++j) {
        const GemmJob& J = p.job[j];
        if (J.pad < 0 || J.span < 0 || J.K < 1 || (R > 1 && J.K > 16)) return -1;
        span = std::max(span, J.span);
        kumax = std::max(kumax, KGT == 1 ? (J.K + 1) / 2 : J.K);
        // every window row the tiles touch must exist in the A arrays
        if (p.pad_l < J.pad ||
            p.Lpad < (long long)p.pad_l - J.pad + (long long)p.tiles_t * 128 * MT + J.span)
            return -1;
        if (R > 1)
            for (int k = 0; k < J.K; ++k)
                if (J.tap_row[k] < 0 || J.tap_row[k] > J.span ||
                    (!convt_grouped(R) && (J.tap_phase[k] < 0 || J.tap_phase[k] >= R)))
                    return -1;
    }
    constexpr int TAPB = 2 * (KGT == 1 ? 2 : KGT) * (convt_grouped(R) ? R * NT : NT) * 16;
    // Weight copies of about 16 KB; the AMP convs of 32 to 128 channels and the upsamplers take
    // up to 64 KB per copy, which halves or quarters the ring's per-copy commits and waits
    // (measured per launch: 128 channels 82 -> 77 us, 64 channels 58 -> 55 us, 32 channels
    // 51 -> 49 us; upsamplers 1024 -> 512 channels 66.5 -> 60.5 us, 512 -> 256 70.7 -> 64.5 us,
    // 256 -> 128 60.4 -> 58.3 us; 32 KB copies gained only the last).  The widest AMP tiles and
    // the narrow 2-group chunks stay at 16 KB, where larger copies measured slower or equal.
    constexpr int CTAS = ps_ctas(MT, NT, EW, R);
    const int wbytes = (CTAS == 1 && (R > 1 || (KGT == 4 && NT <= 128))) ? 65536 : 16384;
    p.tpu = std::max(1, std::min(kumax, wbytes / TAPB));
    PsSched sc{};
    sc.n_ot = (p.Cout + NT - 1) / NT;
    sc.per_job = p.B * p.tiles_t * sc.n_ot;
    sc.ntiles = njobs * sc.per_job;
    if (p.ms_hi) {
        // the fused split: the three residual blocks of an AMP layer, one counter per (tile of
        // a job, epilogue warp), whole 8-channel groups, warps narrow enough to run it
        if (R != 1 || njobs != 3 || 4 * MT * NT / EW > kMsMaxCW || !p.ms_lo || p.Cout % 8 != 0 ||
            p.ms_padl < kMsZeroRows || p.ms_Lpad < (long long)p.ms_padl + p.L + kMsZeroRows)
            return -1;
        int seen = 0;
        for (int z = 0; z < 3; ++z) {
            if (p.ms_blk[z] < 0 || p.ms_blk[z] > 2 || !p.ms_x[z]) return -1;
            seen |= 1 << p.ms_blk[z];
            p.ms_z[p.ms_blk[z]] = z;
        }
        if (seen != 7) return -1;
    }
    // Passes of 8 MMA K-steps (4 taps of 32 channels) at the widest tiles; 16 K-steps (8 taps)
    // for the 32- to 128-channel convs and 16 taps of the 16-channel chunks, where fewer
    // accumulator drains measured 1-3 us per launch faster; the upsampler's pass is one whole
    // chunk.  A pass holds at most 48 truncating accumulations per accumulator column.
    sc.pu = (R > 1) ? 64 : (KGT == 4) ? ((NT <= 128) ? 8 : 4) : 16;
    PsPlan pl{};
    pl.RS = 128 * MT + span;
    pl.SA = 2 * KGT * pl.RS * 16;
    pl.SB = p.tpu * TAPB;
    constexpr int kBarBytes = PS_BAR_BYTES + 4 * EW * 4 * MT * NT / EW;   // + the epilogue's bias slices
    constexpr int kBudget = (CTAS == 2 ? 113 * 1024 : 227 * 1024) - kBarBytes - 64;
    pl.nsa = (4 * pl.SA <= kBudget / 2) ? 4 : 3;
    if (pl.nsa * pl.SA + 2 * pl.SB > kBudget) pl.nsa = 2;
    pl.nsb = std::min(PS_MAXS, (kBudget - pl.nsa * pl.SA) / pl.SB);
    if (pl.nsb < 2) return -1;
    pl.offB = pl.nsa * pl.SA;
    pl.offBar = (pl.offB + pl.nsb * pl.SB + 15) / 16 * 16;
    pl.smem = pl.offBar + kBarBytes;
    // One CTA per SM takes at least half the SM's shared memory, so that a second CTA never
    // waits on the first's tensor memory; two take at most half each.
    const int smem_req = CTAS == 2 ? pl.smem : std::max(pl.smem, 116 * 1024);
    if (smem_req > (CTAS == 2 ? 113 : 227) * 1024) return -1;
    const int nsm = sm_count();
    if (nsm <= 0) return -1;
    auto kern = k_gemm_ps<MT, NT, KGT, EW, R>;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem_req) != cudaSuccess) return -1;
    const int grid = std::min(sc.ntiles, CTAS * nsm);
    return launch_dependent(kern, dim3(grid), dim3(ps_threads(EW)), smem_req, s, p, sc, pl) == cudaSuccess ? 1 : -1;
}

int dispatch_gemm(const GemmParams& p, int njobs, cudaStream_t s) {
    switch (p.Cin) {
        case 512: return launch_gemm_ps<1, 256, 4, 8, 1>(p, njobs, s);
        case 256: return launch_gemm_ps<1, 256, 4, 8, 1>(p, njobs, s);
        case 128: return launch_gemm_ps<2, 128, 4, 8, 1>(p, njobs, s);
        case 64: return launch_gemm_ps<2, 64, 4, 16, 1>(p, njobs, s);
        // two CTAs per SM at 32 and 16 channels (see ps_ctas)
        case 32: return launch_gemm_ps<2, 32, 4, 8, 1>(p, njobs, s);
        case 16: return launch_gemm_ps<2, 16, 2, 8, 1>(p, njobs, s);
        case 8: return launch_gemm_ps<4, 16, 1, 16, 1>(p, njobs, s);
        default: return -1;
    }
}

// Weight-block layout of the AMP convolutions by width: output tile NT and 8-channel groups
// per K chunk (1 = tap-pair units for 8-channel layers).
void amp_layout(int C, int* NT, int* KGT) {
    if (C >= 32) {
        *NT = ntile_amp(C);
        *KGT = 4;
    } else if (C == 16) {
        *NT = 16;
        *KGT = 2;
    } else {
        *NT = 16;
        *KGT = 1;
    }
}

// Operand blocks: [o_tile][chunk][unit][part (head, tail)][core column][row o][8 channels] as
// bf16, from weights given as w(o, c, tap).  For KGT >= 2 a unit is one tap and the core
// columns are the chunk's channel groups; for KGT == 1 a unit is a tap pair and the two core
// columns are its taps (zero past the last tap).  Rows o >= Cout are zero.
template <class W>
void pack_blocks(W w, int Cout, int Cin, int K, int NT, int KGT, bool interleave, TcConv* out) {
    const int kc = 8 * KGT;
    const int ntiles = (Cout + NT - 1) / NT, nchunks = Cin / kc;
    const int KU = (KGT == 1) ? (K + 1) / 2 : K;
    const int BG = (KGT == 1) ? 2 : KGT;
    const size_t n = (size_t)ntiles * nchunks * KU * 2 * BG * NT * 8;  // bf16 elements
    std::vector<uint16_t> buf(n);
    size_t pos = 0;
    // interleave: [core col][part] (the head rows of a core column directly followed by its tail
    // rows); otherwise [part][core col]
    for (int ot = 0; ot < ntiles; ++ot)
        for (int chk = 0; chk < nchunks; ++chk)
            for (int unit = 0; unit < KU; ++unit)
                for (int outer = 0; outer < (interleave ? BG : 2); ++outer)
                    for (int inner = 0; inner < (interleave ? 2 : BG); ++inner)
                        for (int o = 0; o < NT; ++o)
                            for (int e = 0; e < 8; ++e) {
                                const int part = interleave ? inner : outer;
                                const int col = interleave ? outer : inner;
                                const int oo = ot * NT + o;
                                const int tap = (KGT == 1) ? 2 * unit + col : unit;
                                const int cc = chk * kc + ((KGT == 1) ? 0 : col * 8) + e;
                                const float v = (oo < Cout && tap < K) ? w(oo, cc, tap) : 0.f;
                                const uint16_t hb = bf16_bits_rn(v);
                                buf[pos++] = part == 0 ? hb : bf16_bits_rn(v - bf16_value(hb));
                            }
    out->staging.assign((n + 1) / 2, 0.f);
    std::memcpy(out->staging.data(), buf.data(), n * sizeof(uint16_t));
    out->cout = Cout;
    out->cin = Cin;
    out->k = K;
}

// Row-offset groups of a polyphase transposed conv (rate r <= 8, K <= 16 taps, padding pad):
// tap j serves output phase (j - pad) mod r and reads input row u + (phase + pad - j) / r, so
// two taps of one phase never share a row offset.  Groups are the distinct offsets in
// increasing order; tap[g][phase] is the group's tap of that phase, or -1.
struct ConvtGroups {
    int n = 0;
    int shift[16];
    int tap[16][8];
};

ConvtGroups convt_groups(int K, int r, int pad) {
    ConvtGroups G;
    int sh[16];
    for (int j = 0; j < K; ++j) {
        const int phase = ((j - pad) % r + r) % r;
        sh[j] = (phase + pad - j) / r;   // exact: phase + pad - j is a multiple of r
    }
    for (int v = -16; v <= 16; ++v) {
        bool any = false;
        for (int j = 0; j < K; ++j) any = any || sh[j] == v;
        if (!any) continue;
        G.shift[G.n] = v;
        for (int ph = 0; ph < 8; ++ph) G.tap[G.n][ph] = -1;
        for (int j = 0; j < K; ++j)
            if (sh[j] == v) G.tap[G.n][((j - pad) % r + r) % r] = j;
        ++G.n;
    }
    return G;
}

// Upsampler operand blocks with grouped units: [o_tile][chunk][group][part][core col]
// [phase][row o][8 channels], the rows of a phase without a tap in the group zero.
void pack_convt_grouped(const std::vector<float>& w_iok, int Cin, int Cout, int K, int r, int NT, int KGT,
                        TcConv* out) {
    const ConvtGroups G = convt_groups(K, r, (K - r) / 2);
    const int kc = 8 * KGT, ntiles = (Cout + NT - 1) / NT, nchunks = Cin / kc;
    const size_t n = (size_t)ntiles * nchunks * G.n * 2 * KGT * r * NT * 8;
    std::vector<uint16_t> buf(n);
    size_t pos = 0;
    for (int ot = 0; ot < ntiles; ++ot)
        for (int chk = 0; chk < nchunks; ++chk)
            for (int g = 0; g < G.n; ++g)
                for (int part = 0; part < 2; ++part)
                    for (int col = 0; col < KGT; ++col)
                        for (int ph = 0; ph < r; ++ph)
                            for (int o = 0; o < NT; ++o)
                                for (int e = 0; e < 8; ++e) {
                                    const int oo = ot * NT + o, cc = chk * kc + col * 8 + e, tap = G.tap[g][ph];
                                    const float v = (tap >= 0 && oo < Cout) ? w_iok[((size_t)cc * Cout + oo) * K + tap] : 0.f;
                                    const uint16_t hb = bf16_bits_rn(v);
                                    buf[pos++] = part == 0 ? hb : bf16_bits_rn(v - bf16_value(hb));
                                }
    out->staging.assign((n + 1) / 2, 0.f);
    std::memcpy(out->staging.data(), buf.data(), n * sizeof(uint16_t));
    out->cout = Cout;
    out->cin = Cin;
    out->k = K;
}

TcJob make_job(const ConvJob& J, const TcConv& tw) {
    TcJob T{};
    T.x0 = J.x0;
    T.w = reinterpret_cast<const uint16_t*>(tw.dev);
    T.bias = J.bias;
    T.alpha = J.alpha;
    T.inv_beta = J.inv_beta;
    T.res = J.res;
    T.out = J.out;
    T.K = J.K;
    T.dil = J.dil;
    T.pad = J.pad;
    return T;
}

}  // namespace

// The 32- and 16-channel stages: their last layers have 626 units of three tiles at the bench
// workload (B = 2), and the fused split saves its launch (ups5 35.8 -> 20.5 us, ups6 37.9 -> 24.6)
// for 7-10 us more in the layer (with two CTAs per SM: stages 4-5 and upsamplers 5-6 872 us
// against 887 us with the standalone split).  At 64 channels the 314 units leave a heavy last
// wave on 148 SMs (amp3 +22 us against ups4 -13 us), so that stage keeps the standalone split.
bool amp_gemm_split_fusable(int C) { return C == 32 || C == 16; }

bool tc_stage_supported(int C, const mh3a_config& c) {
    if (C != 512 && C != 256 && C != 128 && C != 64 && C != 32 && C != 16 && C != 8) return false;
    if (c.n_resblocks != 3) return false;
    for (int j = 0; j < c.n_resblocks; ++j)
        for (int m = 0; m < c.n_dilations; ++m) {
            // the activation window must fit the shared-memory plan
            if ((c.rb_kernels[j] - 1) * c.rb_dilations[j][m] > 64) return false;
        }
    return true;
}

bool tc_pre_supported(int Cout, int Cin, int k) {
    return Cout % 256 == 0 && Cin % (32 * kPreSplit) == 0 && k <= 15;
}

bool tc_convt_supported(int Cin, int Cout, int r, int K) {
    const int kgt = kgt_convt(Cin);
    if (kgt == 0) return false;
    if (r != 5 && r != 2) return false;
    if (K > 16 || K < r) return false;
    const int NT = ntile_convt(Cout, r);
    if (NT < 16 || NT % 16 != 0 || (Cout % NT != 0 && Cout > NT)) return false;
    if (r == 5 && (NT != 32 || kgt != 4)) return false;
    if (kgt == 2 && NT != 16) return false;
    return true;
}

void prepare_tc_conv(const std::vector<float>& w, int C, int k, TcConv* out) {
    int NT, KGT;
    amp_layout(C, &NT, &KGT);
    pack_blocks([&](int o, int c, int tap) { return w[((size_t)o * C + c) * k + tap]; }, C, C, k, NT, KGT,
                interleaved_b(NT, 1), out);
}

void prepare_tc_pre(const std::vector<float>& w, int O, int I, int k, TcStageWeights* out) {
    const int Is = I / kPreSplit;   // input channels per slice
    for (int sl = 0; sl < kPreSplit; ++sl)
        pack_blocks([&](int o, int c, int tap) { return w[((size_t)o * I + sl * Is + c) * k + tap]; }, O, Is, k,
                    ntile_pre(O), 4, interleaved_b(ntile_pre(O), 1), &out->pre[sl]);
}

void prepare_tc_convt(const std::vector<float>& w_iok, int Cin, int Cout, int K, int r, TcConv* out) {
    if (convt_grouped(r)) {
        pack_convt_grouped(w_iok, Cin, Cout, K, r, ntile_convt(Cout, r), kgt_convt(Cin), out);
        return;
    }
    pack_blocks([&](int o, int c, int tap) { return w_iok[((size_t)c * Cout + o) * K + tap]; }, Cout, Cin, K,
                ntile_convt(Cout, r), kgt_convt(Cin), interleaved_b(ntile_convt(Cout, r), r), out);
}

void tc_finalize(TcStageWeights* w) {
    for (auto& a : w->conv)
        for (auto& b : a)
            for (auto& c : b) std::vector<float>().swap(c.staging);
    for (auto& c : w->pre) std::vector<float>().swap(c.staging);
    std::vector<float>().swap(w->ups.staging);
}

int launch_conv_tc(const ConvParams& cp, int njobs, const TcStageWeights& w, int m, int half, cudaStream_t s,
                   int* err) {
    TcParams p{};
    p.Cin = cp.Cin;
    p.Cout = cp.Cout;
    p.L = cp.L;
    p.B = cp.B;
    p.filt = cp.filt;
    p.err = err;
    // heaviest kernel first (blockIdx.z = 0), so the longest blocks start earliest
    int order[MH3A_MAX_RESBLOCKS];
    for (int j = 0; j < njobs; ++j) order[j] = j;
    std::sort(order, order + njobs, [&](int a, int b) { return cp.job[a].K > cp.job[b].K; });
    for (int z = 0; z < njobs; ++z) {
        const TcConv& tw = w.conv[order[z]][m][half];
        if (!tw.dev) return -1;
        p.job[z] = make_job(cp.job[order[z]], tw);
    }
    return dispatch_amp(p, njobs, s);
}

int launch_amp_gemm_tc(const ConvParams& cp, int njobs, const TcStageWeights& w, int m, int half,
                       const void* const* a_hi, const void* const* a_lo, int pad_l, long long Lpad,
                       cudaStream_t s, int* err, int* sched, const MeanSplitTarget* ms) {
    GemmParams p{};
    if (ms) {
        p.ms_hi = static_cast<uint8_t*>(ms->a_hi);
        p.ms_lo = static_cast<uint8_t*>(ms->a_lo);
        p.ms_Lpad = ms->Lpad;
        p.ms_padl = ms->pad_l;
        if (njobs != 3) return -1;
        for (int j = 0; j < 3; ++j) p.ms_x[j] = cp.job[j].out;
    }
    p.sched = sched;
    p.Cin = cp.Cin;
    p.Cout = cp.Cout;
    p.L = cp.L;
    p.B = cp.B;
    p.pad_l = pad_l;
    p.Lpad = Lpad;
    p.err = err;
    // heaviest kernel first (blockIdx.z = 0), so the longest blocks start earliest
    int order[MH3A_MAX_RESBLOCKS];
    for (int j = 0; j < njobs; ++j) order[j] = j;
    std::sort(order, order + njobs, [&](int a, int b) { return cp.job[a].K > cp.job[b].K; });
    for (int z = 0; z < njobs; ++z) {
        const int j = order[z];
        const TcConv& tw = w.conv[j][m][half];
        if (!tw.dev) return -1;
        p.ms_blk[z] = j;
        GemmJob& G = p.job[z];
        G.a_hi = static_cast<const uint8_t*>(a_hi[j]);
        G.a_lo = static_cast<const uint8_t*>(a_lo[j]);
        G.w = reinterpret_cast<const uint16_t*>(tw.dev);
        G.bias = cp.job[j].bias;
        G.res = cp.job[j].res;
        G.out = cp.job[j].out;
        G.K = cp.job[j].K;
        G.dil = cp.job[j].dil;
        G.pad = cp.job[j].pad;
        int NT, KGT;
        amp_layout(cp.Cin, &NT, &KGT);
        // KGT == 1 pairs taps: the phantom tap after the last one reads `dil` more rows
        G.span = (G.K - 1) * G.dil + (KGT == 1 ? G.dil : 0);
    }
    return dispatch_gemm(p, njobs, s);
}


int launch_conv_pre_gemm(const ConvParams& cp, const TcStageWeights& w, const void* a_hi, const void* a_lo,
                         int pad_l, long long Lpad, float* const* part, cudaStream_t s, int* err, int* sched) {
    if (cp.Cout % ntile_pre(cp.Cout) != 0 || cp.Cin % (32 * kPreSplit) != 0) return -1;
    GemmParams p{};
    p.sched = sched;
    p.Cin = cp.Cin / kPreSplit;       // the K range of one job
    p.a_groups = cp.Cin / 8;
    p.Cout = cp.Cout;
    p.L = cp.L;
    p.B = cp.B;
    p.pad_l = pad_l;
    p.Lpad = Lpad;
    p.err = err;
    for (int sl = 0; sl < kPreSplit; ++sl) {
        if (!w.pre[sl].dev || !part[sl]) return -1;
        GemmJob& G = p.job[sl];
        G.a_hi = static_cast<const uint8_t*>(a_hi);
        G.a_lo = static_cast<const uint8_t*>(a_lo);
        G.w = reinterpret_cast<const uint16_t*>(w.pre[sl].dev);
        G.bias = sl == 0 ? cp.job[0].bias : nullptr;
        G.res = nullptr;
        G.out = part[sl];
        G.K = cp.job[0].K;
        G.dil = cp.job[0].dil;
        G.pad = cp.job[0].pad;
        G.g0 = sl * (p.Cin / 8);
        G.span = (G.K - 1) * G.dil;
    }
    return launch_gemm_ps<1, 256, 4, 8, 1>(p, kPreSplit, s);
}

int launch_convT_gemm(const ConvTParams& q, const TcStageWeights& w, const void* a_hi, const void* a_lo,
                      int pad_l, long long Lpad, cudaStream_t s, int* err, int* sched) {
    if (!w.ups.dev || q.K > 16 || q.K < q.r) return -1;
    GemmParams p{};
    p.sched = sched;
    p.Cin = q.Cin;
    p.Cout = q.Cout;
    p.L = q.Lin;
    p.B = q.B;
    p.pad_l = pad_l;
    p.Lpad = Lpad;
    p.err = err;
    GemmJob& G = p.job[0];
    // tap j serves output phase phi = (j - pad) mod r and reads input row u + (phi + pad - j) / r
    int sh[16], smin = 1 << 20, smax = -(1 << 20);
    for (int j = 0; j < q.K; ++j) {
        const int phase = ((j - q.pad) % q.r + q.r) % q.r;
        sh[j] = (phase + q.pad - j) / q.r;   // exact: phase + pad - j is a multiple of r
        G.tap_phase[j] = (int8_t)phase;
        smin = std::min(smin, sh[j]);
        smax = std::max(smax, sh[j]);
    }
    for (int j = 0; j < q.K; ++j) G.tap_row[j] = (int8_t)(sh[j] - smin);
    G.K = q.K;
    if (convt_grouped(q.r)) {
        // units are the row-offset groups, in the packer's order
        const ConvtGroups CG = convt_groups(q.K, q.r, q.pad);
        for (int g = 0; g < CG.n; ++g) G.tap_row[g] = (int8_t)(CG.shift[g] - smin);
        G.K = CG.n;
    }
    G.a_hi = static_cast<const uint8_t*>(a_hi);
    G.a_lo = static_cast<const uint8_t*>(a_lo);
    G.w = reinterpret_cast<const uint16_t*>(w.ups.dev);
    G.bias = q.bias;
    G.res = nullptr;
    G.out = q.out;
    G.dil = 1;
    G.pad = -smin;
    G.span = smax - smin;
    const int NT = ntile_convt(q.Cout, q.r);
    if (kgt_convt(q.Cin) == 2) return (q.r == 2 && NT == 16) ? launch_gemm_ps<2, 16, 2, 8, 2>(p, 1, s) : -1;
    if (q.r == 5 && NT == 32) return launch_gemm_ps<1, 32, 4, 8, 5>(p, 1, s);
    if (q.r == 2) {
        switch (NT) {
            // 128-row tiles at 64 output channels: upsamplers 2 and 3 have 158-160 tiles of 256
            // rows at the bench workload, 1.08 waves on 148 SMs; 128-row tiles measured 58.3 ->
            // 56.4 and 42.0 -> 40.0 us per launch
            case 64: return launch_gemm_ps<1, 64, 4, 8, 2>(p, 1, s);
            case 32: return launch_gemm_ps<2, 32, 4, 8, 2>(p, 1, s);
            case 16: return launch_gemm_ps<2, 16, 4, 8, 2>(p, 1, s);
            default: return -1;
        }
    }
    return -1;
}


}  // namespace mh3a

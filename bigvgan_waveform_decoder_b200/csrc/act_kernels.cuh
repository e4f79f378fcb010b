// act_kernels.cuh -- standalone anti-aliased SnakeBeta producing the tensor-core A operand.
#pragma once

#include "mh3a_internal.cuh"

namespace mh3a {

struct ActJob {
    const float* x;         // [B, C, L] fp32
    const float* alpha;     // [C]
    const float* inv_beta;  // [C]
    void* a_hi;             // [B, C/8, pad_l + L + pad_r] rows of 8 bf16 (heads)
    void* a_lo;             // same shape (tails)
};

struct ActParams {
    ActJob job[MH3A_MAX_RESBLOCKS];
    int C, L, B;
    int pad_l, pad_r;       // zero rows before / after the sequence in the output
    int g_log2;             // log2(C / 8) when C / 8 is a power of two, else -1 (set by the launcher)
    ActFilter filt;
};

struct SplitParams {
    const float* x0;        // [B, C, L] fp32
    const float* x1;        // with x2: split the mean (x0 + x1 + x2) / 3 instead (else null)
    const float* x2;
    const float* x3;        // with x1, x2: split the sum ((x0 + x1) + x2) + x3 instead (else null)
    void* a_hi;             // [B, C/8, pad_l + L + pad_r] rows of 8 bf16 (heads)
    void* a_lo;             // same shape (tails)
    int C, L, B;
    int pad_l, pad_r;       // zero rows before / after the sequence in the output
};

// Head/tail split without activation (the A operand of conv_pre and of the upsamplers).
int launch_split_rows(const SplitParams& p, cudaStream_t s);

// One launch for `njobs` activations of the same shape (blockIdx.z = job).  Returns the number
// of kernels launched or -1.
int launch_act_split(const ActParams& p, int njobs, cudaStream_t s);

// dec_in_proj (a 1x1 conv, Cz -> C) fused into the head/tail split of its output, which is
// conv_pre's A operand: h[c, t] = bias[c] + sum_k w[k, c] z[k, t], written as rows of 8
// channels like launch_split_rows (h itself is never stored).
struct ProjSplitParams {
    const float* z;         // [B, Cz, L] latents
    const float* w;         // [Cz, C] folded 1x1 weights
    const float* bias;      // [C]
    void* a_hi;             // [B, C/8, pad_l + L + pad_r] rows of 8 bf16 (heads)
    void* a_lo;             // same shape (tails)
    int Cz, C, L, B;
    int pad_l, pad_r;
};
constexpr int kProjMaxCz = 64;   // latent channels the fused projection accepts
int launch_proj_split(const ProjSplitParams& p, cudaStream_t s);

// The decoder's tail in one kernel: the mean of the last stage's three block outputs, the
// anti-aliased SnakeBeta (activation_post), the K-tap conv_post to one channel, its bias and
// the clamp to [-1, 1].  Exactly 8 input channels (one warp each).
struct PostParams {
    const float* x0;        // [B, 8, L] block outputs
    const float* x1;
    const float* x2;
    const float* alpha;     // [8]
    const float* inv_beta;  // [8]
    const float* w;         // [8, K] folded conv_post weights
    const float* bias;      // [1] or null
    float* out;             // [B, 1, L]
    int L, B, K, pad;
    int clamp;              // 1: clamp to [-1, 1] (NaN passes through)
    ActFilter filt;
};
constexpr int kPostMaxK = 15;
int launch_post_act(const PostParams& p, cudaStream_t s);

}  // namespace mh3a

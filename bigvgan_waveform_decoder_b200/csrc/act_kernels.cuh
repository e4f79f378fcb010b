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


}  // namespace mh3a

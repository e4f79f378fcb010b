// tc_kernels.cuh -- tensor-core (tcgen05) convolution path: weight preparation and launchers.
#pragma once

#include <vector>

#include "mh3a_internal.cuh"

namespace mh3a {

// One convolution's operand copy for the tensor cores: bf16 head and tail of every folded
// fp32 weight, laid out exactly as the kernel stages it in shared memory.
struct TcConv {
    std::vector<float> staging;  // host words (bf16 pairs) before the device copy
    float* dev = nullptr;        // device copy inside the weight arena
    int cout = 0, cin = 0, k = 0;
};

struct TcStageWeights {
    TcConv conv[MH3A_MAX_RESBLOCKS][MH3A_MAX_DILATIONS][2];
    TcConv pre;
};

// True when the AMP convolutions of a stage with C channels run on the tensor cores.
bool tc_stage_supported(int C, const mh3a_config& c);

void prepare_tc_conv(const std::vector<float>& w_oik, int C, int k, TcConv* out);
void prepare_tc_pre(const std::vector<float>& w_oik, int O, int I, int k, TcStageWeights* out);

template <class AddFn>
void tc_register(TcStageWeights* w, AddFn add) {
    for (auto& a : w->conv)
        for (auto& b : a)
            for (auto& c : b)
                if (!c.staging.empty()) add(c.staging, &c.dev);
    if (!w->pre.staging.empty()) add(w->pre.staging, &w->pre.dev);
}

// Drop host staging once the device copy exists.
void tc_finalize(TcStageWeights* w);

// Launch one AMP conv layer (dilation index m, half 0 = dilated conv, 1 = k x 1 conv) for all
// residual blocks on the tensor cores.  Returns the number of kernels launched or -1.
// `err` is a device int the kernel sets (non-zero) if one of its bounded waits times out.
int launch_conv_tc(const ConvParams& p, int njobs, const TcStageWeights& w, int m, int half,
                   cudaStream_t s, int* err);
int launch_conv_pre_tc(const ConvParams& p, const TcStageWeights& w, cudaStream_t s);

}  // namespace mh3a

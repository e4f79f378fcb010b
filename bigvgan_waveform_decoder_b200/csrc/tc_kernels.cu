// tc_kernels.cu -- tensor-core (tcgen05) convolution path.
#include "tc_kernels.cuh"

namespace mh3a {

bool tc_stage_supported(int, const mh3a_config&) { return false; }

void prepare_tc_conv(const std::vector<float>&, int, int, TcConv*) {}
void prepare_tc_pre(const std::vector<float>&, int, int, int, TcStageWeights*) {}

void tc_finalize(TcStageWeights* w) {
    for (auto& a : w->conv)
        for (auto& b : a)
            for (auto& c : b) std::vector<float>().swap(c.staging);
    std::vector<float>().swap(w->pre.staging);
}

int launch_conv_tc(const ConvParams&, int, const TcStageWeights&, int, int, cudaStream_t) { return -1; }
int launch_conv_pre_tc(const ConvParams&, const TcStageWeights&, cudaStream_t) { return -1; }

}  // namespace mh3a

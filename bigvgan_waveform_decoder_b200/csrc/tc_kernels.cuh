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

// conv_pre is split along its input channels into kPreSplit slices (jobs of one launch, each
// writing a partial output that the next layer's input split sums).
constexpr int kPreSplit = 4;
static_assert(kPreSplit <= MH3A_MAX_RESBLOCKS, "one GEMM job per slice");

struct TcStageWeights {
    TcConv conv[MH3A_MAX_RESBLOCKS][MH3A_MAX_DILATIONS][2];  // AMP convs of the stage
    TcConv ups;                                             // the stage's transposed conv
    TcConv pre[kPreSplit];                                  // conv_pre slices (stage 0 only)
};

// Which layers run on the tensor cores.
bool tc_stage_supported(int C, const mh3a_config& c);           // AMP convs, C channels
bool tc_pre_supported(int Cout, int Cin, int k);                 // conv_pre
bool tc_convt_supported(int Cin, int Cout, int r, int K);        // transposed conv

// Weight packing from folded fp32 weights: conv weights are [O, I, K], transposed-conv
// weights [I, O, K].
void prepare_tc_conv(const std::vector<float>& w_oik, int C, int k, TcConv* out);
void prepare_tc_pre(const std::vector<float>& w_oik, int O, int I, int k, TcStageWeights* out);
void prepare_tc_convt(const std::vector<float>& w_iok, int Cin, int Cout, int K, int r, TcConv* out);

template <class AddFn>
void tc_register(TcStageWeights* w, AddFn add) {
    for (auto& a : w->conv)
        for (auto& b : a)
            for (auto& c : b)
                if (!c.staging.empty()) add(c.staging, &c.dev);
    if (!w->ups.staging.empty()) add(w->ups.staging, &w->ups.dev);
    for (auto& c : w->pre)
        if (!c.staging.empty()) add(c.staging, &c.dev);
}

// The narrow AMP stages (8 and 16 channels) as one fused kernel per stage (amp_fused.cu): each
// CTA runs all layers of one residual block over a window of rows, intermediates on chip.
bool fused_stage_supported(int C, const mh3a_config& c);
// One layer's weights ([O, I, K] folded fp32) in the fused kernel's K-step layout.
void prepare_fused_conv(const std::vector<float>& w_oik, int C, int K, TcConv* out);
// `layers[l]` (l = 0 .. nlayers-1, two per dilation: the dilated conv, then the k x 1 conv)
// describe the stage's layers for all `njobs` residual blocks as the per-layer launches would
// (weights, biases, activations, dilations); the stage input is x and block j's output goes to
// layers[nlayers-1].job[j].out.  Weights come from w.conv[j][l / 2][l % 2] (prepare_fused_conv).
int launch_amp_fused(const ConvParams* layers, int nlayers, int njobs, const TcStageWeights& w, const float* x,
                     cudaStream_t s, int* err);

// Drop host staging once the device copy exists.
void tc_finalize(TcStageWeights* w);

// Launchers; each returns the number of kernels launched or -1.  `err` is a device int the
// kernels set (non-zero) if one of their bounded waits times out.
// One AMP conv layer (dilation index m, half 0 = dilated conv, 1 = k x 1 conv) for all
// residual blocks:
int launch_conv_tc(const ConvParams& p, int njobs, const TcStageWeights& w, int m, int half,
                   cudaStream_t s, int* err);
// The same layer as a pure GEMM whose A operand (the activation, heads and tails) has been
// written by launch_act_split into a_hi[j] / a_lo[j] with pad_l zero rows before the sequence
// and Lpad rows per (item, channel group).  `sched` points to two device ints, zero before the
// launch (the kernel leaves them zero when it completes): the dynamic tile scheduler's state.
// With `ms` (the last layer of a stage whose next upsampler runs on the tensor cores; three
// residual blocks), the kernel also writes the stage output -- the mean of the blocks' outputs
// -- as that upsampler's head/tail rows (the standalone split's arithmetic, bit for bit), with
// the zero rows its window reads next to the sequence.
// Whether the AMP GEMM at C channels takes a MeanSplitTarget (the 16- and 32-channel stages;
// the kernel itself accepts epilogue warps of at most 32 columns).
bool amp_gemm_split_fusable(int C);
struct MeanSplitTarget {
    void* a_hi;           // [B, C/8, Lpad] rows of 8 bf16 heads; must not be an operand of this launch
    void* a_lo;           // tails
    int pad_l;            // rows before the sequence (at least 8)
    long long Lpad;       // rows per (item, channel group), at least pad_l + L + 8
};
int launch_amp_gemm_tc(const ConvParams& p, int njobs, const TcStageWeights& w, int m, int half,
                       const void* const* a_hi, const void* const* a_lo, int pad_l, long long Lpad,
                       cudaStream_t s, int* err, int* sched, const MeanSplitTarget* ms = nullptr);

// conv_pre and the upsamplers on the persistent GEMM, reading their input as pre-split rows
// (launch_split_rows) with pad_l zero rows before the sequence and Lpad rows per channel group.
// conv_pre writes kPreSplit partial outputs: part[0] = cp.job[0].out (with the bias), part[s]
// for s >= 1 (input-channel slice s, no bias); their sum is the conv's output.
int launch_conv_pre_gemm(const ConvParams& cp, const TcStageWeights& w, const void* a_hi, const void* a_lo,
                         int pad_l, long long Lpad, float* const* part, cudaStream_t s, int* err, int* sched);
int launch_convT_gemm(const ConvTParams& q, const TcStageWeights& w, const void* a_hi, const void* a_lo,
                      int pad_l, long long Lpad, cudaStream_t s, int* err, int* sched);

}  // namespace mh3a

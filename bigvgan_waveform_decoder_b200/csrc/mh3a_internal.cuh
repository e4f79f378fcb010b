// mh3a_internal.cuh -- types shared by the library's translation units (not part of the ABI).
#pragma once

#include <cuda_runtime.h>
#include <cstdint>
#include <string>
#include <utility>

#include "mh3a.h"  // include/ is on the include path

namespace mh3a {

// Text returned by mh3a_last_error() on the calling host thread.
void set_last_error(const std::string& what);

constexpr int kFilterTaps = 12;  // activation filter length (ratio 2: 6 * ratio)

// Launch with programmatic dependent launch allowed: the grid may be scheduled while the
// previous kernel of the stream is still finishing.  Every kernel launched this way executes
// griddepcontrol.wait (ptx::grid_dep_wait) before it reads or writes global memory, which
// waits for the preceding grid to complete and its writes to be visible, so stream order of the
// data is kept; only the launch and the block scheduling overlap the predecessor's tail.
template <typename... KArgs, typename... Args>
cudaError_t launch_dependent(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                             Args&&... args) {
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
}

// Anti-aliased SnakeBeta filter taps: f (decimator) and 2 f (upsampler, gain = ratio).
struct ActFilter {
    float down[kFilterTaps];
    float up[kFilterTaps];
};

// One stride-1 convolution over [B, Cin, L] -> [B, Cout, L] with an optional anti-aliased
// SnakeBeta applied to its input and an optional residual added to its output.
struct ConvJob {
    const float* x0;     // input [B, Cin, L]
    const float* x1;     // when non-null with x2: the input is (x0 + x1 + x2) / 3
    const float* x2;
    const float* w;      // [Cin, K, Cout] (fp32, weight norm folded)
    const float* bias;   // [Cout] or null
    const float* alpha;  // [Cin] SnakeBeta alpha of the input activation (ACT kernels)
    const float* inv_beta;  // [Cin] 1 / (beta + 1e-9)
    const float* res;    // residual [B, Cout, L] or null (may alias out)
    float* out;          // [B, Cout, L]
    int K, dil, pad;
};

struct ConvParams {
    ConvJob job[MH3A_MAX_RESBLOCKS];
    int Cin, Cout, L, B;
    int tiles_t;         // time tiles per batch item
    int clamp;           // clamp the output to [-1, 1] (NaN passes through)
    ActFilter filt;
};

// Transposed conv: x [B, Cin, Lin] (or the mean of three buffers) -> [B, Cout, Lin * r].
struct ConvTParams {
    const float* x0;
    const float* x1;
    const float* x2;
    const float* w;      // [Cin, K, Cout]
    const float* bias;   // [Cout]
    float* out;
    int Cin, Cout, Lin, B, r, K, pad;
    int tiles_t;
};

struct Mean3Params {
    const float* x0;
    const float* x1;
    const float* x2;
    float* out;
    long long n;
    int vec4;            // all four pointers are 16-byte aligned
};

// Device weights of one convolution (fp32, weight norm folded, [Cin, K, Cout]).
struct DevConv {
    float* w = nullptr;
    float* b = nullptr;
    int cin = 0, cout = 0, k = 0;
};

// Per-activation parameters on the device.
struct DevAct {
    float* alpha = nullptr;
    float* inv_beta = nullptr;
};

// Launchers (simt_kernels.cu).  Each returns the number of kernels launched (>= 0) or -1.
int launch_conv_simt(const ConvParams& p, int njobs, bool act, bool mean3, cudaStream_t s);
int launch_convT_simt(const ConvTParams& p, bool mean3, cudaStream_t s);
int launch_mean3(const Mean3Params& p, cudaStream_t s);
// k = 1 conv with at most 64 input channels (the input projection); -1 if the shape does not fit.
int launch_conv1x1(const ConvParams& p, cudaStream_t s);

}  // namespace mh3a

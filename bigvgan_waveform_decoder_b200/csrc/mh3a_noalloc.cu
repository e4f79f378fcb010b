// mh3a_noalloc.cu -- mh3a_amp_stage_static: the AMP-stage entry point for callers that cannot
// allocate device memory while they run.
//
// The six intermediate buffers of an AMP stage (the running sum and the intermediate of each
// of the three residual blocks) live in one file-scope device array instead of the handle's
// workspace.  The CUDA runtime places that array in device memory when it loads this
// library's code onto a GPU, and every GPU that loads it keeps it until the process exits;
// the call itself never allocates.
#include <mutex>
#include <string>

#include "mh3a_internal.cuh"

namespace mh3a {
void set_last_error(const std::string& msg);
int handle_device(const mh3a_handle* h);
int handle_stage_channels(const mh3a_handle* h, int stage);
bool handle_stage_valid(const mh3a_handle* h, int stage);
int handle_n_resblocks(const mh3a_handle* h);
mh3a_status amp_stage_into(mh3a_handle* h, const float* x, int B, int L, int stage, float* out,
                           float* const* X, float* const* T, cudaStream_t s);
}  // namespace mh3a

namespace {

constexpr long long kScratchFloats = MH3A_STATIC_SCRATCH_BYTES / 4;
constexpr int kBuffers = 6;  // X[0..2], T[0..2]
// Each buffer starts on a 256-byte boundary.
constexpr long long kBufferFloats = (kScratchFloats / kBuffers) / 64 * 64;
static_assert(kBufferFloats == MH3A_STATIC_SCRATCH_MAX_ELEMS, "header limit out of date");

// Host code must never use this name as a device address: it is a host-side stand-in.
// Its device address comes from cudaGetSymbolAddress, once per device.
static __device__ __align__(256) float g_scratch[kScratchFloats];

std::mutex g_mu;
constexpr int kMaxDevices = 64;
float* g_scratch_dev[kMaxDevices] = {};

// Device address of g_scratch on the current device (looked up on first use per device).
mh3a_status scratch_address(int dev, float** out) {
    std::lock_guard<std::mutex> lock(g_mu);
    if (!g_scratch_dev[dev]) {
        void* p = nullptr;
        const cudaError_t e = cudaGetSymbolAddress(&p, g_scratch);
        if (e != cudaSuccess || !p) {
            mh3a::set_last_error(std::string("cudaGetSymbolAddress(static scratch): ") + cudaGetErrorString(e));
            return MH3A_ERR_CUDA;
        }
        g_scratch_dev[dev] = static_cast<float*>(p);
    }
    *out = g_scratch_dev[dev];
    return MH3A_OK;
}

}  // namespace

extern "C" MH3A_API mh3a_status mh3a_amp_stage_static(mh3a_handle* h, const float* x, int B, int L, int stage,
                                                      float* out, void* stream) {
    if (!h || !x || !out) return MH3A_ERR_INVALID_ARG;
    if (!mh3a::handle_stage_valid(h, stage)) return MH3A_ERR_INVALID_ARG;
    if (B < 1 || L < 1) return MH3A_ERR_SHAPE;
    if (mh3a::handle_n_resblocks(h) != 3) return MH3A_ERR_UNSUPPORTED;
    const long long n = (long long)B * mh3a::handle_stage_channels(h, stage) * L;
    if (n > kBufferFloats) {
        mh3a::set_last_error("mh3a_amp_stage_static: B*C*L = " + std::to_string(n) +
                             " exceeds the static scratch limit of " + std::to_string(kBufferFloats) +
                             " elements per buffer");
        return MH3A_ERR_SHAPE;
    }
    int dev = -1;
    const cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) {
        mh3a::set_last_error(std::string("cudaGetDevice: ") + cudaGetErrorString(e));
        return MH3A_ERR_CUDA;
    }
    if (dev != mh3a::handle_device(h)) {
        mh3a::set_last_error("mh3a_amp_stage_static: the current device is not the handle's device");
        return MH3A_ERR_INVALID_ARG;
    }
    if (dev < 0 || dev >= kMaxDevices) return MH3A_ERR_UNSUPPORTED;
    float* base = nullptr;
    mh3a_status st = scratch_address(dev, &base);
    if (st) return st;
    float* X[3] = {base, base + kBufferFloats, base + 2 * kBufferFloats};
    float* T[3] = {base + 3 * kBufferFloats, base + 4 * kBufferFloats, base + 5 * kBufferFloats};
    // Every buffer element the stage reads is written earlier in the same call, so nothing
    // left over from a previous call needs clearing.
    return mh3a::amp_stage_into(h, x, B, L, stage, out, X, T, (cudaStream_t)stream);
}

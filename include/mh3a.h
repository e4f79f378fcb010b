/*
 * mh3a.h -- C ABI of the B200 (sm_100a) BigVGAN waveform decoder of the MiniMax-H3 audio VAE.
 *
 * The library turns latents [B, 32, N] into a mono 32 kHz waveform [B, 1, 800 N] clamped to
 * [-1, 1] (diffusers "AutoencoderKLMiniMaxH3Audio" page, `decode` section).  Stereo is carried
 * as two batch items that decode independently (same page, introduction).  The network is the
 * one the FastVideo "minimax_h3_audio_vae" page's `MLXMiniMaxH3AudioVAE.decode` evaluates:
 * a 1x1 input projection, a weight-normed conv, seven weight-normed transposed-conv upsampling
 * stages each followed by the average of three AMP residual blocks, a final anti-aliased
 * SnakeBeta, a weight-normed output conv and the clamp.
 *
 * Conventions for every entry point:
 *   - Tensors are fp32, channel-first and time-contiguous: [B, C, T] row-major.
 *   - Pointers documented as "device" must point to memory of the handle's device; pointers
 *     documented as "host" to ordinary or pinned host memory.  The caller owns all of them;
 *     the library never frees or retains a caller pointer past the call.
 *   - `stream` is a cudaStream_t passed as void* (NULL = the legacy default stream).  Device
 *     work is enqueued on it asynchronously; the call returns before the work finishes unless
 *     stated otherwise.
 *   - Every entry point returns an mh3a_status.  Argument, shape and configuration errors are
 *     detected on the host before any work is enqueued and leave outputs untouched.  Launch
 *     failures are reported as MH3A_ERR_CUDA (the CUDA error text is available from
 *     mh3a_last_error()).  No C++ exception crosses this boundary.
 *   - A handle owns one workspace, so calls on one handle must not overlap in time (on
 *     different streams or host threads).  Different handles are independent.
 */
#ifndef MH3A_H
#define MH3A_H

#if defined(__GNUC__)
#define MH3A_API __attribute__((visibility("default")))
#else
#define MH3A_API
#endif

#include <stddef.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    MH3A_OK = 0,
    MH3A_ERR_INVALID_ARG = 1,    /* NULL pointer, negative size, out-of-range index       */
    MH3A_ERR_CONFIG = 2,         /* architecture the library cannot run (see mh3a_create) */
    MH3A_ERR_SHAPE = 3,          /* B / N / L beyond the handle's limits, weight shapes   */
    MH3A_ERR_MISSING_WEIGHT = 4, /* a required tensor is absent from the weight table     */
    MH3A_ERR_ALLOC = 5,          /* device or host allocation failed                      */
    MH3A_ERR_CUDA = 6,           /* a CUDA runtime call or kernel launch failed           */
    MH3A_ERR_UNSUPPORTED = 7     /* valid request this build does not implement           */
} mh3a_status;

/* Arithmetic of the convolutions (activations are always computed in fp32).
 *   MH3A_FP32     fp32 operands, fp32 accumulation, CUDA cores.
 *   MH3A_BF16X3   tensor cores (tcgen05): each fp32 operand is split into a bf16 head and a
 *                 bf16 tail, and the product is formed as head*head + head*tail + tail*head
 *                 with fp32 accumulation in tensor memory (about 16 significant bits per
 *                 operand).  In this mode every convolution of the default architecture runs
 *                 on the tensor cores -- conv_pre, the seven upsamplers and the AMP convs of
 *                 all seven stages, 512 down to 8 channels -- and mh3a_decode and
 *                 mh3a_amp_stage launch the same kernels for a stage.  Only the 1x1 input
 *                 projection and the 8 -> 1 output conv are fp32 CUDA-core arithmetic. */
typedef enum { MH3A_FP32 = 0, MH3A_BF16X3 = 1 } mh3a_precision;

#define MH3A_FLAG_NO_CLAMP 1u /* return the waveform before the final clamp (testing)   */

#define MH3A_MAX_STAGES 8
#define MH3A_MAX_RESBLOCKS 4
#define MH3A_MAX_DILATIONS 4

/* Architecture and run-time limits.  Defaults (mh3a_default_config) are the constructor
 * defaults of the diffusers "AutoencoderKLMiniMaxH3Audio" page. */
typedef struct {
    int latent_channels;                      /* 32                                       */
    int latent_dim;                           /* 2048                                     */
    int decoder_dim;                          /* 1024, halved by every upsampling stage   */
    int n_stages;                             /* 7                                        */
    int rates[MH3A_MAX_STAGES];               /* (5,5,2,2,2,2,2); product = hop = 800     */
    int kernels[MH3A_MAX_STAGES];             /* (9,9,4,4,4,4,4)                          */
    int n_resblocks;                          /* 3                                        */
    int rb_kernels[MH3A_MAX_RESBLOCKS];       /* (3,7,11)                                 */
    int n_dilations;                          /* 3                                        */
    int rb_dilations[MH3A_MAX_RESBLOCKS][MH3A_MAX_DILATIONS]; /* ((1,3,5) x 3)            */
    int sampling_rate;                        /* 32000 (informational)                    */
    int precision;                            /* mh3a_precision                           */
    unsigned flags;                           /* MH3A_FLAG_*                              */
    /* Per-channel latent statistics (host, [latent_channels]) or NULL.  When given, decode
     * first denormalises z = x * std_c + mean_c (diffusers "AutoencoderKLMiniMaxH3" page,
     * latent normalisation bullet); the library folds this into the input projection. */
    const float* latents_mean;
    const float* latents_std;
    int max_batch;                            /* workspace sizing: largest B              */
    int max_frames;                           /* workspace sizing: largest N (latents)    */
} mh3a_config;

/* One named host tensor of the weight table.  Names are the checkpoint keys the MLX page's
 * decode reads: "dec_in_proj.weight|bias", "decoder.conv_pre.weight_v|weight_g|bias",
 * "decoder.ups.{i}.0.weight_v|weight_g|bias", "decoder.resblocks.{n}.convs1.{m}.weight_v|
 * weight_g|bias", "decoder.resblocks.{n}.convs2.{m}.…", "decoder.resblocks.{n}.activations.
 * {a}.act.alpha|beta" (a = 2m before convs1.m, 2m+1 before convs2.m),
 * "decoder.activation_post.act.alpha|beta", "decoder.conv_post.weight_v|weight_g[|bias]".
 * Transposed-conv weights are stored [in, out, k]; all other conv weights [out, in, k];
 * weight_g is [dim0, 1, 1] and normalises over every axis but the first. */
typedef struct {
    const char* name;
    const float* host_data;
    int ndim;
    long long shape[3];
} mh3a_tensor;

typedef struct mh3a_handle mh3a_handle;

/* Fill *cfg with the default architecture, precision MH3A_BF16X3, no flags, no latent
 * statistics, max_batch 2, max_frames 400. */
MH3A_API void mh3a_default_config(mh3a_config* cfg);

/* Fill *cfg from a released component's config.json: the diffusers
 * "AutoencoderKLMiniMaxH3Audio" constructor arguments, which the FastVideo
 * "minimax_h3_audio_vae" page's `MiniMaxH3AudioVAEConfigView.from_vae_dir` reads from the
 * component directory.  Starts from mh3a_default_config and takes latent_channels, latent_dim,
 * decoder_dim, decoder_rates, decoder_kernel_sizes, resblock_kernel_sizes,
 * resblock_dilation_sizes, sampling_rate and latents_mean / latents_std (null or a list of
 * latent_channels numbers); every other key is skipped.  A list that changes a count
 * (decoder_rates, resblock_kernel_sizes) needs its companion list (decoder_kernel_sizes,
 * resblock_dilation_sizes).  Statistics are written to the caller's host arrays latents_mean /
 * latents_std (cap floats each; NULL is allowed when the file has none) and cfg->latents_mean /
 * latents_std point at them, so those arrays must outlive the mh3a_create that uses *cfg.
 * Precision, flags and workspace limits keep their defaults for the caller to set.  The values
 * themselves are checked by mh3a_create.
 * Errors: MH3A_ERR_INVALID_ARG (NULL path/cfg, negative cap, unreadable file, malformed JSON,
 * a field of the wrong type), MH3A_ERR_CONFIG (more stages, blocks or dilations than the MAX_*
 * limits; list lengths that disagree), MH3A_ERR_SHAPE (a statistics list not of latent_channels
 * values, or no caller array large enough).  The reason is in mh3a_last_error(); on error *cfg
 * is left unchanged. */
MH3A_API mh3a_status mh3a_config_from_json(const char* path, mh3a_config* cfg, float* latents_mean,
                                           float* latents_std, int cap);

/* Build a decoder on the current CUDA device.  Copies the weight table to device memory,
 * folds every weight norm w = g * v / ||v|| (MLX page `_wn_weight`) and the optional latent
 * denormalisation into the weights, builds the Kaiser-sinc activation filter (MLX page
 * `kaiser_sinc_filter1d`, cutoff 0.25, half-width 0.3, 12 taps) and allocates the workspace for
 * max_batch x max_frames.  Blocks until the copies are done.  The host tensors may be freed
 * after the call.
 * Errors: MH3A_ERR_INVALID_ARG (NULL cfg/weights/out), MH3A_ERR_CONFIG (the product of the
 * rates is not 800, the hop of the encoder the decoder inverts; some K_i - r_i is odd or
 * negative, so a stage would not output exactly r_i samples per input; decoder_dim is not
 * divisible by 2^n_stages; more stages/blocks/dilations than the MAX_* limits; an even
 * residual-block kernel; unknown precision; non-positive max_batch or max_frames), MH3A_ERR_MISSING_WEIGHT, MH3A_ERR_SHAPE (a tensor's shape disagrees with the
 * architecture), MH3A_ERR_ALLOC, MH3A_ERR_CUDA.  On error *out is set to NULL. */
MH3A_API mh3a_status mh3a_create(const mh3a_config* cfg, const mh3a_tensor* weights, int n_weights,
                        mh3a_handle** out);

/* Device-memory provider for mh3a_create_with_allocator.  alloc(bytes, user) returns device
 * memory of the current device, 256-byte aligned, or NULL on failure; release(ptr, user) gives
 * back a pointer alloc returned.  Both are called only from mh3a_create_with_allocator (two
 * allocations: the folded weights and the workspace) and from mh3a_destroy, on the calling host
 * thread. */
typedef struct {
    void* (*alloc)(size_t bytes, void* user);
    void (*release)(void* ptr, void* user);
    void* user;
} mh3a_allocator;

/* mh3a_create with the handle's device memory taken from `allocator` instead of cudaMalloc
 * (the pages have no counterpart): for hosts whose device memory is owned by another framework's
 * allocator or pool.  allocator == NULL is mh3a_create.  A NULL alloc or release is
 * MH3A_ERR_INVALID_ARG.  If an allocation fails (NULL, or a pointer that is not 256-byte
 * aligned), the call returns MH3A_ERR_ALLOC, after giving back through `release` every
 * allocation it had obtained, and sets *out to NULL; both allocations are made before any data
 * is copied to the device.  The allocator must outlive the handle: mh3a_destroy releases
 * through it. */
MH3A_API mh3a_status mh3a_create_with_allocator(const mh3a_config* cfg, const mh3a_tensor* weights,
                                                int n_weights, const mh3a_allocator* allocator,
                                                mh3a_handle** out);

/* Build a decoder from the audio VAE component's checkpoint file, the single safetensors file
 * the FastVideo "minimax_h3_audio_vae" page loads (`mlx_h3_audio_vae_from_dir`,
 * `mlx_h3_audio_vae_from_file`: `diffusion_pytorch_model.safetensors`).  `path` is a host
 * NUL-terminated file name.  Format: an 8-byte little-endian header length n, a JSON header of n
 * bytes mapping tensor names to {"dtype", "shape", "data_offsets": [begin, end]} (plus an
 * optional "__metadata__" object), then the data section.  Of the file, only tensors named
 * "dec_in_proj.*" and "decoder.*" (the decode path) are read; every other entry (the encoder's,
 * the latent statistics' projections) is parsed and skipped.  Those tensors must be stored as
 * "F32" (the page requires fp32 storage) with 1 to 3 dimensions; "dec_in_proj.weight",
 * "decoder.conv_pre.weight_v" and "decoder.conv_post.weight_v" must be present (the page's
 * required decode keys).  The released activation filter buffers ("*.upsample.filter",
 * "*.downsample.lowpass.filter") are not read: the library builds the same Kaiser-sinc filter.
 * The tensors are then passed, under their file names, to mh3a_create_with_allocator
 * (`allocator` may be NULL: cudaMalloc), whose checks apply unchanged.  The file is read with
 * host buffers that are released before the call returns.
 * Errors: MH3A_ERR_INVALID_ARG (NULL cfg/path/out; the file cannot be opened or read; a header
 * length out of range; malformed header JSON; data offsets outside the data section or
 * disagreeing with the shape), MH3A_ERR_UNSUPPORTED (a decode tensor not stored as F32, or with
 * more than 3 dimensions), MH3A_ERR_MISSING_WEIGHT (a required key absent; others as reported by
 * mh3a_create), MH3A_ERR_ALLOC (a host buffer), and every error of mh3a_create.  The reason is in
 * mh3a_last_error().  On error *out is set to NULL. */
MH3A_API mh3a_status mh3a_create_from_safetensors(const mh3a_config* cfg, const char* path,
                                                  const mh3a_allocator* allocator, mh3a_handle** out);

/* Decode latents (device, [B, latent_channels, N]) into a waveform (device, [B, 1, hop*N]),
 * clamped to [-1, 1] unless MH3A_FLAG_NO_CLAMP was configured.  `out` must not overlap
 * `latents`.  1 <= B <= max_batch, 1 <= N <= max_frames, else MH3A_ERR_SHAPE. */
MH3A_API mh3a_status mh3a_decode(mh3a_handle* h, const float* latents, int B, int N, float* out,
                        void* stream);

/* The same decode from and to HOST memory: copies the latents in, decodes, and delivers the
 * waveform to `out_host`, all on `stream`, and waits for the stream before returning.  When
 * `out_host` is page-locked memory that the current device can address (cudaHostAlloc /
 * cudaMallocHost memory, e.g. a pinned torch tensor, under unified addressing), the decode's
 * last kernel stores the waveform into it directly, so the transfer overlaps that kernel;
 * other host memory receives a device-to-host copy after the decode.  Pinned host buffers
 * give the fastest transfers.  Same shape limits as mh3a_decode. */
MH3A_API mh3a_status mh3a_decode_host(mh3a_handle* h, const float* latents_host, int B, int N,
                             float* out_host, void* stream);

/* One AMP stage (MLX page `decode`, the averaged `_amp_block` outputs of upsampling stage
 * `stage`): x (device, [B, C, L]) -> out (device, [B, C, L]) with C = decoder_dim /
 * 2^(stage+1).  `out` must not overlap `x`.  B * L must not exceed the workspace, i.e.
 * B * L <= max_batch * max_frames * (product of rates[0..stage]); else MH3A_ERR_SHAPE. */
MH3A_API mh3a_status mh3a_amp_stage(mh3a_handle* h, const float* x, int B, int L, int stage, float* out,
                           void* stream);

/* Allocation-free variant of mh3a_amp_stage.  The pages have no counterpart: this entry point
 * exists for callers that cannot allocate device memory at the time they run a stage -- a
 * real-time audio thread that must never block in the driver's allocator, or a host whose
 * device memory belongs to another framework's fixed budget.  Such a caller creates the handle
 * once at start-up (it may pass max_batch = max_frames = 1 to keep the handle's own workspace
 * small) and then runs stages through this call, which allocates nothing.
 *
 * Arguments and status codes are those of mh3a_amp_stage.  The results agree with
 * mh3a_amp_stage's within the parity tolerance of the handle's precision, and are identical to
 * them bit for bit where this call runs the same kernel: at a stage that the decode runs as one
 * fused kernel (8 channels in MH3A_BF16X3 mode), which needs no scratch beyond the block
 * outputs.  At the other stages the decode's tensor-core path stages the activation through
 * operand arrays in the workspace; this call instead runs a layer kernel that computes the
 * activation inside the conv (32 channels and wider) or the fp32 CUDA-core kernels (narrower),
 * so its low-order bits differ.  The six intermediate
 * [B, C, L] buffers of the stage live in one fixed array of MH3A_STATIC_SCRATCH_BYTES in the
 * library's device image: the CUDA runtime places it when it loads the library's code onto a
 * GPU, and every GPU that loads the library holds it until the process exits.  B * C * L must
 * not exceed MH3A_STATIC_SCRATCH_MAX_ELEMS, else MH3A_ERR_SHAPE (the limit and the requested
 * size are in mh3a_last_error()).  The current device must be the handle's device, else
 * MH3A_ERR_INVALID_ARG.  The first call on each device looks up the array's device address
 * (cudaGetSymbolAddress) and caches it; make that first call before any stream capture.  All
 * calls on one device share the array and each call leaves its contents behind: calls that
 * overlap in time on the GPU (other streams, threads or handles) race and corrupt each other's
 * results, so serialise them. */
#define MH3A_STATIC_SCRATCH_BYTES (64ll << 20)
#define MH3A_STATIC_SCRATCH_MAX_ELEMS 2796160ll /* per buffer: (64 MiB / 4 / 6) rounded to 64 */
MH3A_API mh3a_status mh3a_amp_stage_static(mh3a_handle* h, const float* x, int B, int L, int stage,
                                           float* out, void* stream);

/* Graph replay of decodes.  With graph mode on, the second mh3a_decode (or mh3a_decode_host)
 * for a given (B, N, latents pointer, output pointer) captures the decode's kernel launches on
 * the caller's stream into a CUDA graph and instantiates it; that call and every later one with
 * the same four values launch the instantiated graph.  The first call for a key launches
 * directly, so a caller that passes new buffers every time never pays for a capture.  A replay
 * performs exactly the launches of a direct decode (identical results; mh3a_launch_count grows
 * by the same amount) with less launch overhead.  The graph holds the two pointers: refilling
 * the same input buffer and calling again is the intended use.  Up to 4 graphs are kept per
 * handle (the least recently used one is replaced, after a device synchronisation).  Decodes
 * on the legacy default stream (NULL) or the per-thread default stream, on a stream the caller
 * is capturing, or with mh3a_set_profiling / mh3a_set_kernel_profiling active launch directly.
 * Disabling (enable = 0) synchronises the device and releases every graph.  Capture or
 * instantiation errors return MH3A_ERR_CUDA (mh3a_last_error says which) and leave the stream
 * usable.  Default: off. */
MH3A_API mh3a_status mh3a_set_graph_mode(mh3a_handle* h, int enable);

/* Per-segment device timing.  When enabled, each decode records CUDA events between its
 * segments (input projection, conv_pre, then per stage: upsampling, AMP stage; then the output
 * activation+conv); mh3a_segment_times waits for the last decode and writes up to `cap`
 * durations in milliseconds, returning the number of segments through *count. */
MH3A_API mh3a_status mh3a_set_profiling(mh3a_handle* h, int enable);
MH3A_API mh3a_status mh3a_segment_times(mh3a_handle* h, float* ms, int cap, int* count);

/* Per-kernel device timing of one tensor-core AMP stage.  After
 * mh3a_set_kernel_profiling(h, stage), each decode records CUDA events around that stage's six
 * activation launches and six GEMM launches (stage -1: none; each event record costs a few
 * microseconds of stream time, so only one stage is instrumented).  mh3a_stage_kernel_times
 * waits for the last decode and writes the summed durations (milliseconds) of the stage's
 * activation launches to *act_ms and of its GEMM launches to *gemm_ms.  MH3A_ERR_INVALID_ARG
 * for a NULL argument or an out-of-range stage; MH3A_ERR_UNSUPPORTED if the last decode did not
 * record that stage (another stage selected, or the stage not on the tensor cores). */
MH3A_API mh3a_status mh3a_set_kernel_profiling(mh3a_handle* h, int stage);
MH3A_API mh3a_status mh3a_stage_kernel_times(mh3a_handle* h, int stage, float* act_ms, float* gemm_ms);

/* 1 if the AMP convolutions of `stage` run on the tensor cores for this handle, 0 if on the
 * fp32 CUDA cores, -1 for a NULL handle or an out-of-range stage. */
MH3A_API int mh3a_stage_uses_tensor_cores(const mh3a_handle* h, int stage);

/* Same question per timing segment, numbered as in mh3a_segment_times: 0 input projection,
 * 1 conv_pre, 2 + 2i upsampling stage i, 3 + 2i AMP stage i, 2 + 2 n_stages output conv.
 * Returns 1, 0, or -1 for a NULL handle or an out-of-range segment. */
MH3A_API int mh3a_segment_uses_tensor_cores(const mh3a_handle* h, int segment);

/* Waits for the device, then reports whether any tensor-core kernel of this handle gave up
 * one of its bounded pipeline waits since the last check (MH3A_ERR_CUDA, with the reason in
 * mh3a_last_error(); the outputs of that call are invalid) and clears the flag.  Such a
 * timeout is a defect, never an expected outcome: every wait in those kernels has an
 * iteration limit so that a defect ends the kernel instead of hanging the GPU. */
MH3A_API mh3a_status mh3a_check_device_error(mh3a_handle* h);

/* Number of kernels this handle has launched since creation (all entry points). */
MH3A_API long long mh3a_launch_count(const mh3a_handle* h);

/* Bytes of device memory the handle owns (weights + workspace). */
MH3A_API long long mh3a_device_bytes(const mh3a_handle* h);

/* Release the handle's device memory.  NULL is ignored.  Waits for the handle's work. */
MH3A_API void mh3a_destroy(mh3a_handle* h);

/* Static description of a status code. */
MH3A_API const char* mh3a_status_string(mh3a_status s);

/* Text of the last CUDA error seen by the calling host thread ("" if none). */
MH3A_API const char* mh3a_last_error(void);

#ifdef __cplusplus
}
#endif
#endif /* MH3A_H */

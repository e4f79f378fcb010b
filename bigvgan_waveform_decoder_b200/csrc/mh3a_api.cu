// mh3a_api.cu -- the C ABI (include/mh3a.h): configuration checks, weight folding at create
// time, workspace management and the launch sequence of the decode.
//
// Decode (FastVideo "minimax_h3_audio_vae" page, `MLXMiniMaxH3AudioVAE.decode`):
//   h = conv1x1(z) (dec_in_proj)  ->  h = conv_k7(h) (conv_pre, weight-normed, padding 3)
//   for each stage i: h = convT(h; r_i, K_i, padding (K_i - r_i)/2)   (ups.i.0)
//                     h = mean_j AMP_j(h)                           (resblocks 3i + j)
//   h = act(h) (activation_post)  ->  y = conv_k7(h) (conv_post)  ->  clamp(y, -1, 1)
// AMP_j(x): for each dilation d: x = x + conv_k,1(act(conv_k,d(act(x)))), k = rb_kernels[j].
#include <cmath>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <string>
#include <vector>

#include "mh3a_internal.cuh"
#include "act_kernels.cuh"
#include "tc_kernels.cuh"

using namespace mh3a;

namespace {

thread_local std::string g_last_error;

mh3a_status cuda_fail(cudaError_t e, const char* what) {
    g_last_error = std::string(what) + ": " + cudaGetErrorString(e);
    return MH3A_ERR_CUDA;
}

#define CK_CUDA(call, what)                                  \
    do {                                                     \
        cudaError_t e_ = (call);                             \
        if (e_ != cudaSuccess) return cuda_fail(e_, what);   \
    } while (0)

constexpr int kMaxSegments = 2 + 2 * MH3A_MAX_STAGES + 1;

// Zero rows around each (item, channel group) of the tensor-core A operands: before the
// sequence at least the largest conv padding, after it the largest tile overhang (2 x 128
// rows) plus that padding.
constexpr int kApadL = 32;
constexpr int kMsSlot = 3;   // the A operand pair the fused upsampler input split writes
constexpr int kApadR = 4 * 128 + 32;

// Kaiser-windowed sinc low-pass of the activation (FastVideo "minimax_h3_audio_vae" page,
// `kaiser_sinc_filter1d`): Kaiser's estimate A = 2.285 (K/2 - 1) pi (4 hw) + 7.95 of the stop-band
// attenuation, his rule for the window shape beta(A), a symmetric Kaiser window over K points,
// a sinc of cutoff fc on the half-integer (even K) grid, and unit DC gain.
double bessel0(double x) {
    // I0(x) = sum_n ((x/2)^n / n!)^2
    double half = 0.5 * x, term = 1.0, total = 1.0;
    for (int n = 1; n < 300 && term > 1e-20 * total; ++n) {
        term *= (half / n) * (half / n);
        total += term;
    }
    return total;
}

void build_filter(ActFilter* f) {
    const int K = kFilterTaps;
    const double fc = 0.5 / 2.0, hw = 0.6 / 2.0;  // ratio 2
    const double A = 2.285 * (K / 2 - 1) * M_PI * (4.0 * hw) + 7.95;
    const double beta = (A > 50.0) ? 0.1102 * (A - 8.7)
                      : (A >= 21.0) ? 0.5842 * std::pow(A - 21.0, 0.4) + 0.07886 * (A - 21.0)
                                    : 0.0;
    double h[K], total = 0.0;
    for (int n = 0; n < K; ++n) {
        const double pos = (n - (K - 1) / 2.0) / ((K - 1) / 2.0);  // -1 .. 1
        const double win = bessel0(beta * std::sqrt(std::max(0.0, 1.0 - pos * pos))) / bessel0(beta);
        const double t = n - K / 2 + ((K % 2 == 0) ? 0.5 : 0.0);
        const double x = 2.0 * fc * t;
        const double sinc = (x == 0.0) ? 1.0 : std::sin(M_PI * x) / (M_PI * x);
        h[n] = 2.0 * fc * win * sinc;
        total += h[n];
    }
    for (int n = 0; n < K; ++n) {
        f->down[n] = (float)(h[n] / total);
        f->up[n] = 2.0f * f->down[n];  // upsampler gain = ratio
    }
}

struct Lookup {
    const mh3a_tensor* w;
    int n;
    const mh3a_tensor* find(const std::string& name) const {
        for (int i = 0; i < n; ++i)
            if (w[i].name && name == w[i].name) return &w[i];
        return nullptr;
    }
};

long long numel(const mh3a_tensor* t) {
    long long n = 1;
    for (int d = 0; d < t->ndim; ++d) n *= t->shape[d];
    return n;
}

}  // namespace

struct mh3a_handle {
    mh3a_config cfg{};
    int device = 0;
    int hop = 1;
    ActFilter filt{};
    // fp32 weights (weight norm folded), [Cin, K, Cout]
    DevConv in_proj, pre, ups[MH3A_MAX_STAGES], post;
    DevConv rb1[MH3A_MAX_STAGES][MH3A_MAX_RESBLOCKS][MH3A_MAX_DILATIONS];
    DevConv rb2[MH3A_MAX_STAGES][MH3A_MAX_RESBLOCKS][MH3A_MAX_DILATIONS];
    DevAct act1[MH3A_MAX_STAGES][MH3A_MAX_RESBLOCKS][MH3A_MAX_DILATIONS];
    DevAct act2[MH3A_MAX_STAGES][MH3A_MAX_RESBLOCKS][MH3A_MAX_DILATIONS];
    DevAct act_post;
    TcStageWeights tc[MH3A_MAX_STAGES];   // tensor-core operand copies (BF16X3)
    bool stage_tc[MH3A_MAX_STAGES] = {};
    bool stage_fused[MH3A_MAX_STAGES] = {};   // narrow stages: one fused kernel per stage
    bool pre_tc = false;                  // conv_pre on the tensor cores
    bool ups_tc[MH3A_MAX_STAGES] = {};    // transposed convs on the tensor cores
    mh3a_allocator alloc{};               // caller's device allocator (alloc == NULL: cudaMalloc)
    char* warena = nullptr;
    size_t wbytes = 0;
    // workspace
    char* arena = nullptr;
    size_t abytes = 0;
    long long stage_cap = 0;   // floats per stage buffer
    float* buf_in = nullptr;   // [B, latent_dim, N]
    float* buf_pre = nullptr;  // [B, decoder_dim, N]
    float* pre_part[4] = {};   // conv_pre's partial outputs on the tensor-core path
    float* H = nullptr;
    float* X[MH3A_MAX_RESBLOCKS] = {};
    float* T[MH3A_MAX_RESBLOCKS] = {};
    void* A_hi[MH3A_MAX_RESBLOCKS] = {};   // tensor-core A operands (activations, bf16 heads)
    void* A_lo[MH3A_MAX_RESBLOCKS] = {};   //   and tails, with zero padding rows
    long long a_cap = 0;                   // bf16 elements per A array
    // The fused upsampler input split (three residual blocks): the last AMP layer of a 16- or
    // 32-channel stage writes the next upsampler's operand into A_hi/A_lo[3] (no operand of that
    // layer).
    bool ms_on = false;
    float* lat_io = nullptr;   // host-API staging
    float* wav_io = nullptr;
    int* dev_err = nullptr;    // 64 ints: [0] set by a tensor-core kernel whose bounded wait timed
                               // out; [16..17] the persistent GEMM's tile scheduler
    // profiling
    bool profiling = false;
    cudaEvent_t ev[kMaxSegments + 1] = {};
    int nseg = 0;
    // kernel profiling of one AMP stage: events before the activation, between it and the
    // GEMM, and after the GEMM of each of its 6 layers
    int kprof_stage = -1;
    cudaEvent_t kev[6][3] = {};
    bool kev_made = false;
    int kev_rec = -1;                       // the stage the last decode recorded
    bool kev_fused = false;                 // it was a fused stage: one launch, kev[0][0..1]
    long long launches = 0;
    // graph replay (mh3a_set_graph_mode): one captured decode per (B, N, input, output)
    struct GraphEntry {
        int B = 0, N = 0;
        const float* in = nullptr;
        float* out = nullptr;
        cudaGraphExec_t exec = nullptr;
        long long launches = 0;          // kernels one replay launches
        unsigned long long used = 0;     // last use, for replacement
    };
    static constexpr int kGraphSlots = 4;
    bool graph_mode = false;
    GraphEntry graphs[kGraphSlots];
    // keys decoded once without a graph: a key is captured on its second use, so callers that
    // pass fresh buffers every time never pay for a capture
    static constexpr int kSeenSlots = 8;
    GraphEntry seen[kSeenSlots];
    unsigned long long graph_tick = 0;
};

namespace {

int stage_channels(const mh3a_config& c, int i) { return c.decoder_dim >> (i + 1); }

mh3a_status validate(const mh3a_config& c) {
    if (c.n_stages < 1 || c.n_stages > MH3A_MAX_STAGES) return MH3A_ERR_CONFIG;
    if (c.n_resblocks < 1 || c.n_resblocks > MH3A_MAX_RESBLOCKS) return MH3A_ERR_CONFIG;
    if (c.n_dilations < 1 || c.n_dilations > MH3A_MAX_DILATIONS) return MH3A_ERR_CONFIG;
    if (c.latent_channels < 1 || c.latent_dim < 1 || c.decoder_dim < 1) return MH3A_ERR_CONFIG;
    long long hop = 1;
    for (int i = 0; i < c.n_stages; ++i) {
        const int r = c.rates[i], K = c.kernels[i];
        if (r < 1 || r > 8 || K < r || (K - r) % 2 != 0) return MH3A_ERR_CONFIG;
        hop *= r;
    }
    if (hop != 800) return MH3A_ERR_CONFIG;
    if (c.decoder_dim % (1 << c.n_stages) != 0) return MH3A_ERR_CONFIG;
    for (int j = 0; j < c.n_resblocks; ++j) {
        const int k = c.rb_kernels[j];
        if (k < 1 || k % 2 == 0 || k > 31) return MH3A_ERR_CONFIG;
        for (int m = 0; m < c.n_dilations; ++m)
            if (c.rb_dilations[j][m] < 1 || c.rb_dilations[j][m] > 16) return MH3A_ERR_CONFIG;
    }
    if (c.precision != MH3A_FP32 && c.precision != MH3A_BF16X3) return MH3A_ERR_CONFIG;
    if (c.max_batch < 1 || c.max_frames < 1) return MH3A_ERR_CONFIG;
    return MH3A_OK;
}

// Device memory of a handle: from the caller's allocator when one was given, else cudaMalloc.
bool dev_alloc(mh3a_handle* h, size_t bytes, char** out) {
    *out = nullptr;
    if (h->alloc.alloc) {
        void* p = h->alloc.alloc(bytes, h->alloc.user);
        if (!p || (reinterpret_cast<uintptr_t>(p) & 255) != 0) {
            if (p) h->alloc.release(p, h->alloc.user);   // misaligned: not usable
            return false;
        }
        *out = static_cast<char*>(p);
        return true;
    }
    void* p = nullptr;
    if (cudaMalloc(&p, bytes) != cudaSuccess) {
        cudaGetLastError();   // the failed allocation is reported as MH3A_ERR_ALLOC, not left pending
        return false;
    }
    *out = static_cast<char*>(p);
    return true;
}

void dev_free(mh3a_handle* h, char* p) {
    if (!p) return;
    if (h->alloc.alloc) h->alloc.release(p, h->alloc.user);
    else cudaFree(p);
}

// Host staging of the folded weights before one device copy.
struct HostArena {
    std::vector<float> data;
    struct Fix { float** dst; size_t off; };
    std::vector<Fix> fix;
    size_t add(const std::vector<float>& v, float** dst) {
        size_t off = data.size();
        data.insert(data.end(), v.begin(), v.end());
        data.resize((data.size() + 63) & ~size_t(63), 0.f);  // 256-byte alignment of the next
        fix.push_back({dst, off});
        return off;
    }
};

// Weight-normed conv [O, I, K] -> folded, transposed to [I, K, O].
mh3a_status fold_conv(const Lookup& lk, const std::string& prefix, int O, int I, int K, bool bias_required,
                      HostArena& ha, DevConv* dc, std::vector<float>* folded_oik = nullptr) {
    const mh3a_tensor* v = lk.find(prefix + ".weight_v");
    const mh3a_tensor* g = lk.find(prefix + ".weight_g");
    if (!v || !g) return MH3A_ERR_MISSING_WEIGHT;
    if (!v->host_data || !g->host_data) return MH3A_ERR_INVALID_ARG;
    if (v->ndim != 3 || v->shape[0] != O || v->shape[1] != I || v->shape[2] != K || numel(g) != O)
        return MH3A_ERR_SHAPE;
    std::vector<float> w((size_t)I * K * O);
    if (folded_oik) folded_oik->assign((size_t)O * I * K, 0.f);
    for (int o = 0; o < O; ++o) {
        const float* vo = v->host_data + (size_t)o * I * K;
        double ss = 0.0;
        for (long long q = 0; q < (long long)I * K; ++q) ss += (double)vo[q] * vo[q];
        const double sc = (double)g->host_data[o] / std::sqrt(ss);
        for (int c = 0; c < I; ++c)
            for (int j = 0; j < K; ++j) {
                const float val = (float)(sc * vo[(size_t)c * K + j]);
                w[((size_t)c * K + j) * O + o] = val;
                if (folded_oik) (*folded_oik)[((size_t)o * I + c) * K + j] = val;
            }
    }
    ha.add(w, &dc->w);
    const mh3a_tensor* b = lk.find(prefix + ".bias");
    if (b) {
        if (numel(b) != O) return MH3A_ERR_SHAPE;
        ha.add(std::vector<float>(b->host_data, b->host_data + O), &dc->b);
    } else if (bias_required) {
        return MH3A_ERR_MISSING_WEIGHT;
    } else {
        ha.add(std::vector<float>(O, 0.f), &dc->b);
    }
    dc->cin = I;
    dc->cout = O;
    dc->k = K;
    return MH3A_OK;
}

// Weight-normed transposed conv [I, O, K] (norm per input channel) -> [I, K, O].
mh3a_status fold_convT(const Lookup& lk, const std::string& prefix, int I, int O, int K, HostArena& ha,
                       DevConv* dc, std::vector<float>* folded_iok = nullptr) {
    const mh3a_tensor* v = lk.find(prefix + ".weight_v");
    const mh3a_tensor* g = lk.find(prefix + ".weight_g");
    const mh3a_tensor* b = lk.find(prefix + ".bias");
    if (!v || !g || !b) return MH3A_ERR_MISSING_WEIGHT;
    if (v->ndim != 3 || v->shape[0] != I || v->shape[1] != O || v->shape[2] != K || numel(g) != I ||
        numel(b) != O)
        return MH3A_ERR_SHAPE;
    std::vector<float> w((size_t)I * K * O);
    if (folded_iok) folded_iok->assign((size_t)I * O * K, 0.f);
    for (int c = 0; c < I; ++c) {
        const float* vc = v->host_data + (size_t)c * O * K;
        double ss = 0.0;
        for (long long q = 0; q < (long long)O * K; ++q) ss += (double)vc[q] * vc[q];
        const double sc = (double)g->host_data[c] / std::sqrt(ss);
        for (int o = 0; o < O; ++o)
            for (int j = 0; j < K; ++j) {
                const float val = (float)(sc * vc[(size_t)o * K + j]);
                w[((size_t)c * K + j) * O + o] = val;
                if (folded_iok) (*folded_iok)[((size_t)c * O + o) * K + j] = val;
            }
    }
    ha.add(w, &dc->w);
    ha.add(std::vector<float>(b->host_data, b->host_data + O), &dc->b);
    dc->cin = I;
    dc->cout = O;
    dc->k = K;
    return MH3A_OK;
}

mh3a_status load_act(const Lookup& lk, const std::string& prefix, int C, HostArena& ha, DevAct* da) {
    const mh3a_tensor* a = lk.find(prefix + ".alpha");
    const mh3a_tensor* b = lk.find(prefix + ".beta");
    if (!a || !b) return MH3A_ERR_MISSING_WEIGHT;
    if (numel(a) != C || numel(b) != C) return MH3A_ERR_SHAPE;
    std::vector<float> ib(C);
    for (int c = 0; c < C; ++c) ib[c] = (float)(1.0 / ((double)b->host_data[c] + 1e-9));
    ha.add(std::vector<float>(a->host_data, a->host_data + C), &da->alpha);
    ha.add(ib, &da->inv_beta);
    return MH3A_OK;
}

mh3a_status record(mh3a_handle* h, cudaStream_t s) {
    if (!h->profiling) return MH3A_OK;
    if (h->nseg > kMaxSegments) return MH3A_OK;
    CK_CUDA(cudaEventRecord(h->ev[h->nseg], s), "cudaEventRecord");
    h->nseg++;
    return MH3A_OK;
}

mh3a_status counted(mh3a_handle* h, int n) {
    if (n < 0) {
        const cudaError_t e = cudaGetLastError();
        if (e != cudaSuccess) return cuda_fail(e, "kernel launch");
        g_last_error = "a launcher refused its arguments (no kernel was launched)";
        return MH3A_ERR_UNSUPPORTED;
    }
    h->launches += n;
    return MH3A_OK;
}

// The six residual-chain launches of one AMP stage: input h (B, C, L); the per-block running
// sums end in h->X[j].  Every launch covers all residual blocks (blockIdx.z).
mh3a_status run_amp(mh3a_handle* h, int stage, const float* in, int B, int L, cudaStream_t s,
                    const MeanSplitTarget* ms = nullptr) {
    const mh3a_config& c = h->cfg;
    const int C = stage_channels(c, stage);
    const int nrb = c.n_resblocks;
    ConvParams layers[2 * MH3A_MAX_DILATIONS];
    for (int m = 0; m < c.n_dilations; ++m) {
        for (int half = 0; half < 2; ++half) {
            ConvParams p{};
            p.Cin = C;
            p.Cout = C;
            p.L = L;
            p.B = B;
            p.clamp = 0;
            p.filt = h->filt;
            for (int j = 0; j < nrb; ++j) {
                const int k = c.rb_kernels[j];
                const int d = (half == 0) ? c.rb_dilations[j][m] : 1;
                ConvJob& J = p.job[j];
                const DevConv& dc = (half == 0) ? h->rb1[stage][j][m] : h->rb2[stage][j][m];
                const DevAct& da = (half == 0) ? h->act1[stage][j][m] : h->act2[stage][j][m];
                J.x0 = (half == 0) ? (m == 0 ? in : h->X[j]) : h->T[j];
                J.w = dc.w;
                J.bias = dc.b;
                J.alpha = da.alpha;
                J.inv_beta = da.inv_beta;
                J.res = (half == 0) ? nullptr : (m == 0 ? in : h->X[j]);
                J.out = (half == 0) ? h->T[j] : h->X[j];
                J.K = k;
                J.dil = d;
                J.pad = d * (k - 1) / 2;
            }
            if (h->stage_fused[stage]) {
                layers[2 * m + half] = p;   // launched below, all layers at once
                continue;
            }
            int n;
            if (h->stage_tc[stage]) {
                // activation once per layer into the A operand, then the tensor-core GEMM
                if ((long long)B * C * ((long long)L + kApadL + kApadR) > h->a_cap) {
                    g_last_error = "batch too large for the tensor-core operand buffers (B > max_batch)";
                    return MH3A_ERR_SHAPE;
                }
                ActParams ap{};
                ap.C = C;
                ap.L = L;
                ap.B = B;
                ap.pad_l = kApadL;
                ap.pad_r = kApadR;
                ap.filt = h->filt;
                for (int j = 0; j < nrb; ++j) {
                    ap.job[j].x = p.job[j].x0;
                    ap.job[j].alpha = p.job[j].alpha;
                    ap.job[j].inv_beta = p.job[j].inv_beta;
                    ap.job[j].a_hi = h->A_hi[j];
                    ap.job[j].a_lo = h->A_lo[j];
                }
                const bool kprof = h->kprof_stage == stage && h->kev_made;
                const int li = 2 * m + half;
                if (kprof) CK_CUDA(cudaEventRecord(h->kev[li][0], s), "cudaEventRecord");
                mh3a_status st = counted(h, launch_act_split(ap, nrb, s));
                if (st) return st;
                if (kprof) CK_CUDA(cudaEventRecord(h->kev[li][1], s), "cudaEventRecord");
                const long long Lpad = (long long)L + kApadL + kApadR;
                const bool last = m == c.n_dilations - 1 && half == 1;
                n = launch_amp_gemm_tc(p, nrb, h->tc[stage], m, half, h->A_hi, h->A_lo, kApadL, Lpad, s, h->dev_err,
                                       h->dev_err + 16, last ? ms : nullptr);
                if (kprof && n > 0) {
                    CK_CUDA(cudaEventRecord(h->kev[li][2], s), "cudaEventRecord");
                    if (li == 5) {
                        h->kev_rec = stage;
                        h->kev_fused = false;
                    }
                }
            } else {
                n = launch_conv_simt(p, nrb, /*act=*/true, /*mean3=*/false, s);
            }
            mh3a_status st = counted(h, n);
            if (st) return st;
        }
    }
    if (h->stage_fused[stage]) {
        const bool kprof = h->kprof_stage == stage && h->kev_made;
        if (kprof) CK_CUDA(cudaEventRecord(h->kev[0][0], s), "cudaEventRecord");
        mh3a_status st = counted(h, launch_amp_fused(layers, 2 * c.n_dilations, nrb, h->tc[stage], in, s, h->dev_err));
        if (st) return st;
        if (kprof) {
            CK_CUDA(cudaEventRecord(h->kev[0][1], s), "cudaEventRecord");
            h->kev_rec = stage;
            h->kev_fused = true;
        }
    }
    return MH3A_OK;
}

// The kPreSplit partial outputs of the tensor-core conv_pre: buf_pre (with the bias), then three
// stage buffers that are free until the first AMP stage (sized for decoder_dim x N at create).
float* const* pre_parts(mh3a_handle* h) {
    static_assert(kPreSplit == 4, "four partial buffers");
    h->pre_part[0] = h->buf_pre;
    h->pre_part[1] = h->H;
    h->pre_part[2] = h->X[0];
    h->pre_part[3] = h->T[0];
    return h->pre_part;
}

// Head/tail rows of x0 (or of the mean of x0, x1, x2, or of the sum of x0 .. x3) into the first
// A operand pair.
mh3a_status split_to_a(mh3a_handle* h, const float* x0, const float* x1, const float* x2, int C, int L, int B,
                       cudaStream_t s, const float* x3 = nullptr) {
    if ((long long)B * C * ((long long)L + kApadL + kApadR) > h->a_cap) {
        g_last_error = "batch too large for the tensor-core operand buffers (B > max_batch)";
        return MH3A_ERR_SHAPE;
    }
    SplitParams sp{};
    sp.x0 = x0;
    sp.x1 = x1;
    sp.x2 = x2;
    sp.x3 = x3;
    sp.a_hi = h->A_hi[0];
    sp.a_lo = h->A_lo[0];
    sp.C = C;
    sp.L = L;
    sp.B = B;
    sp.pad_l = kApadL;
    sp.pad_r = kApadR;
    return counted(h, launch_split_rows(sp, s));
}

mh3a_status run_decode(mh3a_handle* h, const float* lat, int B, int N, float* out, cudaStream_t s) {
    const mh3a_config& c = h->cfg;
    h->nseg = 0;
    mh3a_status st = record(h, s);
    if (st) return st;
    const bool fused_proj = h->pre_tc && c.latent_channels <= kProjMaxCz;
    // dec_in_proj (denormalisation folded in)
    {
        ConvParams p{};
        p.Cin = c.latent_channels;
        p.Cout = c.latent_dim;
        p.L = N;
        p.B = B;
        p.job[0].x0 = lat;
        p.job[0].w = h->in_proj.w;
        p.job[0].bias = h->in_proj.b;
        p.job[0].out = h->buf_in;
        p.job[0].K = 1;
        p.job[0].dil = 1;
        p.job[0].pad = 0;
        if (fused_proj) {
            // the projection goes straight into conv_pre's head/tail operand rows
            if ((long long)B * c.latent_dim * ((long long)N + kApadL + kApadR) > h->a_cap) {
                g_last_error = "batch too large for the tensor-core operand buffers (B > max_batch)";
                return MH3A_ERR_SHAPE;
            }
            ProjSplitParams pp{};
            pp.z = lat;
            pp.w = h->in_proj.w;
            pp.bias = h->in_proj.b;
            pp.a_hi = h->A_hi[0];
            pp.a_lo = h->A_lo[0];
            pp.Cz = c.latent_channels;
            pp.C = c.latent_dim;
            pp.L = N;
            pp.B = B;
            pp.pad_l = kApadL;
            pp.pad_r = kApadR;
            if ((st = counted(h, launch_proj_split(pp, s)))) return st;
        } else {
            if ((st = counted(h, launch_conv1x1(p, s)))) return st;
        }
        if ((st = record(h, s))) return st;
    }
    // conv_pre
    {
        ConvParams p{};
        p.Cin = c.latent_dim;
        p.Cout = c.decoder_dim;
        p.L = N;
        p.B = B;
        p.job[0].x0 = h->buf_in;
        p.job[0].w = h->pre.w;
        p.job[0].bias = h->pre.b;
        p.job[0].out = h->buf_pre;
        p.job[0].K = h->pre.k;
        p.job[0].dil = 1;
        p.job[0].pad = 3;
        int n;
        if (h->pre_tc) {
            // the input as head/tail rows (already written by the fused projection, or split
            // here), then the persistent tensor-core GEMM
            if (!fused_proj && (st = split_to_a(h, h->buf_in, nullptr, nullptr, c.latent_dim, N, B, s))) return st;
            n = launch_conv_pre_gemm(p, h->tc[0], h->A_hi[0], h->A_lo[0], kApadL, (long long)N + kApadL + kApadR,
                                     pre_parts(h), s, h->dev_err, h->dev_err + 16);
        } else {
            n = launch_conv_simt(p, 1, false, false, s);
        }
        if ((st = counted(h, n))) return st;
        if ((st = record(h, s))) return st;
    }
    int C = c.decoder_dim, L = N;
    bool ms_done = false;
    for (int i = 0; i < c.n_stages; ++i) {
        ConvTParams q{};
        const bool mean3 = (i > 0);
        q.x0 = (i == 0) ? h->buf_pre : h->X[0];
        q.x1 = mean3 ? h->X[1] : nullptr;
        q.x2 = mean3 ? h->X[2] : nullptr;
        q.w = h->ups[i].w;
        q.bias = h->ups[i].b;
        q.out = h->H;
        q.Cin = C;
        q.Cout = C / 2;
        q.Lin = L;
        q.B = B;
        q.r = c.rates[i];
        q.K = c.kernels[i];
        q.pad = (q.K - q.r) / 2;
        if (mean3 && c.n_resblocks != 3) {
            // the fused mean reads exactly three block outputs; otherwise reduce explicitly
            return MH3A_ERR_UNSUPPORTED;
        }
        int nl;
        if (i > 0 && ms_done) {
            // the previous stage's last layer wrote this upsampler's operand rows
            nl = launch_convT_gemm(q, h->tc[i], h->A_hi[kMsSlot], h->A_lo[kMsSlot], kApadL,
                                   (long long)L + kApadL + kApadR, s, h->dev_err, h->dev_err + 16);
        } else if (i == 0 && h->pre_tc) {
            // conv_pre left its output as partial sums over input-channel slices
            float* const* part = pre_parts(h);
            if (!h->ups_tc[i]) return MH3A_ERR_UNSUPPORTED;
            if ((st = split_to_a(h, part[0], part[1], part[2], C, L, B, s, part[3]))) return st;
            nl = launch_convT_gemm(q, h->tc[i], h->A_hi[0], h->A_lo[0], kApadL, (long long)L + kApadL + kApadR, s,
                                   h->dev_err, h->dev_err + 16);
        } else if (h->ups_tc[i]) {
            if ((st = split_to_a(h, q.x0, q.x1, q.x2, C, L, B, s))) return st;
            nl = launch_convT_gemm(q, h->tc[i], h->A_hi[0], h->A_lo[0], kApadL, (long long)L + kApadL + kApadR, s,
                                   h->dev_err, h->dev_err + 16);
        } else {
            nl = launch_convT_simt(q, mean3, s);
        }
        if ((st = counted(h, nl))) return st;
        if ((st = record(h, s))) return st;
        C /= 2;
        L *= c.rates[i];
        // the stage's last layer also forms the next upsampler's operand where it can
        ms_done = h->ms_on && i + 1 < c.n_stages && h->stage_tc[i] && !h->stage_fused[i] && h->ups_tc[i + 1] &&
                  amp_gemm_split_fusable(C) && (long long)B * C * ((long long)L + kApadL + kApadR) <= h->a_cap;
        MeanSplitTarget mst{h->A_hi[kMsSlot], h->A_lo[kMsSlot], kApadL, (long long)L + kApadL + kApadR};
        if ((st = run_amp(h, i, h->H, B, L, s, ms_done ? &mst : nullptr))) return st;
        if ((st = record(h, s))) return st;
    }
    // activation_post + conv_post + clamp, reading the mean of the last stage's blocks
    {
        ConvParams p{};
        p.Cin = C;
        p.Cout = 1;
        p.L = L;
        p.B = B;
        p.clamp = (c.flags & MH3A_FLAG_NO_CLAMP) ? 0 : 1;
        p.filt = h->filt;
        p.job[0].x0 = h->X[0];
        p.job[0].x1 = h->X[1];
        p.job[0].x2 = h->X[2];
        p.job[0].w = h->post.w;
        p.job[0].bias = h->post.b;
        p.job[0].alpha = h->act_post.alpha;
        p.job[0].inv_beta = h->act_post.inv_beta;
        p.job[0].out = out;
        p.job[0].K = h->post.k;
        p.job[0].dil = 1;
        p.job[0].pad = 3;
        if (c.precision == MH3A_BF16X3 && C == 8 && c.n_resblocks == 3) {
            PostParams pp{};
            pp.x0 = h->X[0];
            pp.x1 = h->X[1];
            pp.x2 = h->X[2];
            pp.alpha = h->act_post.alpha;
            pp.inv_beta = h->act_post.inv_beta;
            pp.w = h->post.w;
            pp.bias = h->post.b;
            pp.out = out;
            pp.L = L;
            pp.B = B;
            pp.K = h->post.k;
            pp.pad = 3;
            pp.clamp = p.clamp;
            pp.filt = h->filt;
            if ((st = counted(h, launch_post_act(pp, s)))) return st;
        } else {
            if ((st = counted(h, launch_conv_simt(p, 1, true, true, s)))) return st;
        }
        if ((st = record(h, s))) return st;
    }
    return MH3A_OK;
}

}  // namespace

namespace mh3a {

void set_last_error(const std::string& msg) { g_last_error = msg; }

int handle_device(const mh3a_handle* h) { return h->device; }

int handle_stage_channels(const mh3a_handle* h, int stage) { return stage_channels(h->cfg, stage); }

bool handle_stage_valid(const mh3a_handle* h, int stage) { return stage >= 0 && stage < h->cfg.n_stages; }

int handle_n_resblocks(const mh3a_handle* h) { return h->cfg.n_resblocks; }

// One AMP stage with caller-provided block buffers X[j] (running sums) and T[j]
// (intermediates), each of at least B * C * L floats, then the mean of the blocks into `out`.
mh3a_status amp_stage_into(mh3a_handle* h, const float* x, int B, int L, int stage, float* out,
                           float* const* X, float* const* T, cudaStream_t s) {
    const mh3a_config& c = h->cfg;
    const int C = stage_channels(c, stage);
    const int nrb = c.n_resblocks;
    ConvParams layers[2 * MH3A_MAX_DILATIONS];
    for (int m = 0; m < c.n_dilations; ++m) {
        for (int half = 0; half < 2; ++half) {
            ConvParams p{};
            p.Cin = C;
            p.Cout = C;
            p.L = L;
            p.B = B;
            p.clamp = 0;
            p.filt = h->filt;
            for (int j = 0; j < nrb; ++j) {
                const int k = c.rb_kernels[j];
                const int d = (half == 0) ? c.rb_dilations[j][m] : 1;
                ConvJob& J = p.job[j];
                const DevConv& dc = (half == 0) ? h->rb1[stage][j][m] : h->rb2[stage][j][m];
                const DevAct& da = (half == 0) ? h->act1[stage][j][m] : h->act2[stage][j][m];
                J.x0 = (half == 0) ? (m == 0 ? x : X[j]) : T[j];
                J.w = dc.w;
                J.bias = dc.b;
                J.alpha = da.alpha;
                J.inv_beta = da.inv_beta;
                J.res = (half == 0) ? nullptr : (m == 0 ? x : X[j]);
                J.out = (half == 0) ? T[j] : X[j];
                J.K = k;
                J.dil = d;
                J.pad = d * (k - 1) / 2;
            }
            if (h->stage_fused[stage]) {
                layers[2 * m + half] = p;   // the fused stage kernel, launched below
                continue;
            }
            // the fused tensor-core layer kernel (activation computed in its own producer warps)
            // needs no operand buffers beyond X and T; it serves widths of 32 channels and more
            const int n = (h->stage_tc[stage] && C >= 32)
                              ? launch_conv_tc(p, nrb, h->tc[stage], m, half, s, h->dev_err)
                              : launch_conv_simt(p, nrb, /*act=*/true, /*mean3=*/false, s);
            mh3a_status st = counted(h, n);
            if (st) return st;
        }
    }
    if (h->stage_fused[stage]) {
        // the kernel mh3a_amp_stage and the decode run for this stage: it needs no scratch but
        // the block outputs X
        mh3a_status st = counted(h, launch_amp_fused(layers, 2 * c.n_dilations, nrb, h->tc[stage], x, s, h->dev_err));
        if (st) return st;
    }
    Mean3Params mp{X[0], X[1], X[2], out, (long long)B * C * L, 0};
    mp.vec4 = ((reinterpret_cast<uintptr_t>(out) | reinterpret_cast<uintptr_t>(X[0]) |
                reinterpret_cast<uintptr_t>(X[1]) | reinterpret_cast<uintptr_t>(X[2])) & 15) == 0;
    return counted(h, launch_mean3(mp, s));
}

}  // namespace mh3a

extern "C" {

void mh3a_default_config(mh3a_config* c) {
    if (!c) return;
    std::memset(c, 0, sizeof(*c));
    c->latent_channels = 32;
    c->latent_dim = 2048;
    c->decoder_dim = 1024;
    c->n_stages = 7;
    const int rates[7] = {5, 5, 2, 2, 2, 2, 2}, kernels[7] = {9, 9, 4, 4, 4, 4, 4};
    for (int i = 0; i < 7; ++i) {
        c->rates[i] = rates[i];
        c->kernels[i] = kernels[i];
    }
    c->n_resblocks = 3;
    c->rb_kernels[0] = 3;
    c->rb_kernels[1] = 7;
    c->rb_kernels[2] = 11;
    c->n_dilations = 3;
    for (int j = 0; j < 3; ++j) {
        c->rb_dilations[j][0] = 1;
        c->rb_dilations[j][1] = 3;
        c->rb_dilations[j][2] = 5;
    }
    c->sampling_rate = 32000;
    c->precision = MH3A_BF16X3;
    c->flags = 0;
    c->max_batch = 2;
    c->max_frames = 400;
}

const char* mh3a_status_string(mh3a_status s) {
    switch (s) {
        case MH3A_OK: return "ok";
        case MH3A_ERR_INVALID_ARG: return "invalid argument";
        case MH3A_ERR_CONFIG: return "unsupported configuration";
        case MH3A_ERR_SHAPE: return "shape mismatch";
        case MH3A_ERR_MISSING_WEIGHT: return "missing weight";
        case MH3A_ERR_ALLOC: return "allocation failed";
        case MH3A_ERR_CUDA: return "CUDA error";
        case MH3A_ERR_UNSUPPORTED: return "unsupported request";
    }
    return "unknown status";
}

const char* mh3a_last_error(void) { return g_last_error.c_str(); }

void mh3a_destroy(mh3a_handle* h) {
    if (!h) return;
    int prev = 0;
    cudaGetDevice(&prev);
    cudaSetDevice(h->device);
    cudaDeviceSynchronize();
    for (auto& g : h->graphs)
        if (g.exec) cudaGraphExecDestroy(g.exec);
    for (auto& e : h->ev)
        if (e) cudaEventDestroy(e);
    for (auto& li : h->kev)
        for (auto& e : li)
            if (e) cudaEventDestroy(e);
    dev_free(h, h->warena);
    dev_free(h, h->arena);
    cudaSetDevice(prev);
    delete h;
}

mh3a_status mh3a_create(const mh3a_config* cfg, const mh3a_tensor* weights, int n_weights, mh3a_handle** out) {
    return mh3a_create_with_allocator(cfg, weights, n_weights, nullptr, out);
}

mh3a_status mh3a_create_with_allocator(const mh3a_config* cfg, const mh3a_tensor* weights, int n_weights,
                                       const mh3a_allocator* allocator, mh3a_handle** out) {
    if (out) *out = nullptr;
    if (!cfg || !weights || !out || n_weights < 1) return MH3A_ERR_INVALID_ARG;
    if (allocator && (!allocator->alloc || !allocator->release)) return MH3A_ERR_INVALID_ARG;
    mh3a_status st = validate(*cfg);
    if (st) return st;
    mh3a_handle* h = new (std::nothrow) mh3a_handle();
    if (!h) return MH3A_ERR_ALLOC;
    if (allocator) h->alloc = *allocator;
    h->cfg = *cfg;
    h->cfg.latents_mean = nullptr;  // folded below; the caller's arrays are not retained
    h->cfg.latents_std = nullptr;
    cudaGetDevice(&h->device);
    build_filter(&h->filt);
    const mh3a_config& c = h->cfg;
    for (int i = 0; i < c.n_stages; ++i) h->hop *= c.rates[i];

    Lookup lk{weights, n_weights};
    HostArena ha;
    auto fail = [&](mh3a_status s) {
        mh3a_destroy(h);
        return s;
    };
    // dec_in_proj with the optional denormalisation z = x * std + mean folded in:
    //   W'[o, c] = W[o, c] std_c,   b'[o] = b[o] + sum_c W[o, c] mean_c
    {
        const mh3a_tensor* w = lk.find("dec_in_proj.weight");
        const mh3a_tensor* b = lk.find("dec_in_proj.bias");
        if (!w || !b) return fail(MH3A_ERR_MISSING_WEIGHT);
        const int O = c.latent_dim, I = c.latent_channels;
        if (numel(w) != (long long)O * I || numel(b) != O) return fail(MH3A_ERR_SHAPE);
        std::vector<float> wt((size_t)I * O), bt(O);
        for (int o = 0; o < O; ++o) {
            double bo = b->host_data[o];
            for (int ci = 0; ci < I; ++ci) {
                const double wv = w->host_data[(size_t)o * I + ci];
                const double sd = cfg->latents_std ? cfg->latents_std[ci] : 1.0;
                const double mu = cfg->latents_mean ? cfg->latents_mean[ci] : 0.0;
                wt[(size_t)ci * O + o] = (float)(wv * sd);
                bo += wv * mu;
            }
            bt[o] = (float)bo;
        }
        ha.add(wt, &h->in_proj.w);
        ha.add(bt, &h->in_proj.b);
        h->in_proj.cin = I;
        h->in_proj.cout = O;
        h->in_proj.k = 1;
    }
    {
        const mh3a_tensor* v = lk.find("decoder.conv_pre.weight_v");
        if (!v) return fail(MH3A_ERR_MISSING_WEIGHT);
        if (v->ndim != 3 || v->shape[2] != 7) return fail(MH3A_ERR_SHAPE);
        std::vector<float> oik;
        // the tensor-core conv_pre leaves partial sums that only the tensor-core upsampler's
        // input split reduces
        h->pre_tc = c.precision == MH3A_BF16X3 && tc_pre_supported(c.decoder_dim, c.latent_dim, 7) &&
                    c.n_stages >= 1 && tc_convt_supported(c.decoder_dim, c.decoder_dim / 2, c.rates[0], c.kernels[0]);
        if ((st = fold_conv(lk, "decoder.conv_pre", c.decoder_dim, c.latent_dim, 7, true, ha, &h->pre,
                            h->pre_tc ? &oik : nullptr)))
            return fail(st);
        if (h->pre_tc) prepare_tc_pre(oik, c.decoder_dim, c.latent_dim, 7, &h->tc[0]);
    }
    int C = c.decoder_dim;
    char buf[160];
    for (int i = 0; i < c.n_stages; ++i) {
        const int Co = C / 2;
        std::snprintf(buf, sizeof buf, "decoder.ups.%d.0", i);
        h->ups_tc[i] = c.precision == MH3A_BF16X3 && (i == 0 || c.n_resblocks == 3) &&
                       tc_convt_supported(C, Co, c.rates[i], c.kernels[i]);
        std::vector<float> iok;
        if ((st = fold_convT(lk, buf, C, Co, c.kernels[i], ha, &h->ups[i], h->ups_tc[i] ? &iok : nullptr)))
            return fail(st);
        if (h->ups_tc[i]) prepare_tc_convt(iok, C, Co, c.kernels[i], c.rates[i], &h->tc[i].ups);
        h->stage_tc[i] = (c.precision == MH3A_BF16X3) && tc_stage_supported(Co, c);
        h->stage_fused[i] = h->stage_tc[i] && fused_stage_supported(Co, c);
        for (int j = 0; j < c.n_resblocks; ++j) {
            const int k = c.rb_kernels[j];
            const int rb = i * c.n_resblocks + j;
            for (int m = 0; m < c.n_dilations; ++m) {
                std::vector<float> oik1, oik2;
                const bool tc = h->stage_tc[i];
                std::snprintf(buf, sizeof buf, "decoder.resblocks.%d.convs1.%d", rb, m);
                if ((st = fold_conv(lk, buf, Co, Co, k, true, ha, &h->rb1[i][j][m], tc ? &oik1 : nullptr)))
                    return fail(st);
                std::snprintf(buf, sizeof buf, "decoder.resblocks.%d.convs2.%d", rb, m);
                if ((st = fold_conv(lk, buf, Co, Co, k, true, ha, &h->rb2[i][j][m], tc ? &oik2 : nullptr)))
                    return fail(st);
                if (tc && h->stage_fused[i]) {
                    prepare_fused_conv(oik1, Co, k, &h->tc[i].conv[j][m][0]);
                    prepare_fused_conv(oik2, Co, k, &h->tc[i].conv[j][m][1]);
                } else if (tc) {
                    prepare_tc_conv(oik1, Co, k, &h->tc[i].conv[j][m][0]);
                    prepare_tc_conv(oik2, Co, k, &h->tc[i].conv[j][m][1]);
                }
                std::snprintf(buf, sizeof buf, "decoder.resblocks.%d.activations.%d.act", rb, 2 * m);
                if ((st = load_act(lk, buf, Co, ha, &h->act1[i][j][m]))) return fail(st);
                std::snprintf(buf, sizeof buf, "decoder.resblocks.%d.activations.%d.act", rb, 2 * m + 1);
                if ((st = load_act(lk, buf, Co, ha, &h->act2[i][j][m]))) return fail(st);
            }
        }
        C = Co;
    }
    if ((st = load_act(lk, "decoder.activation_post.act", C, ha, &h->act_post))) return fail(st);
    {
        const mh3a_tensor* v = lk.find("decoder.conv_post.weight_v");
        if (!v) return fail(MH3A_ERR_MISSING_WEIGHT);
        if (v->ndim != 3 || v->shape[2] != 7) return fail(MH3A_ERR_SHAPE);
        if ((st = fold_conv(lk, "decoder.conv_post", 1, C, 7, false, ha, &h->post))) return fail(st);
    }
    // tensor-core operand copies go into the same arena
    for (int i = 0; i < c.n_stages; ++i) tc_register(&h->tc[i], [&](const std::vector<float>& v, float** d) { ha.add(v, d); });

    h->wbytes = ha.data.size() * sizeof(float);

    // workspace: stage buffers sized for the widest stage at max_batch x max_frames
    long long cap = 0, len = 1;
    for (int i = 0; i < c.n_stages; ++i) {
        len *= c.rates[i];
        const long long v = (long long)stage_channels(c, i) * len;
        cap = cap > v ? cap : v;
    }
    const long long BN = (long long)c.max_batch * c.max_frames;
    h->stage_cap = ((cap * BN + 63) / 64) * 64;
    if (h->pre_tc)   // three stage buffers also hold conv_pre's partial outputs
        h->stage_cap = std::max(h->stage_cap, (((long long)c.decoder_dim * BN + 63) / 64) * 64);
    auto rnd = [](long long n) { return ((n + 63) / 64) * 64; };
    const long long n_in = rnd((long long)c.latent_dim * BN), n_pre = rnd((long long)c.decoder_dim * BN);
    const long long n_lat = rnd((long long)c.latent_channels * BN), n_wav = rnd((long long)h->hop * BN);
    const long long nbuf = 1 + 2 * c.n_resblocks;
    // tensor-core A operands: per block, heads and tails of B x C x (L + padding rows) bf16, for
    // every layer that reads them (AMP convs, conv_pre, upsamplers)
    {
        long long need = 0, Lin = c.max_frames;
        const long long pads = kApadL + kApadR;
        if (h->pre_tc) need = std::max(need, (long long)c.latent_dim * (c.max_frames + pads));
        int Cin = c.decoder_dim;
        for (int i = 0; i < c.n_stages; ++i) {
            if (h->ups_tc[i]) need = std::max(need, (long long)Cin * (Lin + pads));
            Lin *= c.rates[i];
            Cin /= 2;
            if (h->stage_tc[i] && !h->stage_fused[i]) need = std::max(need, (long long)Cin * (Lin + pads));
        }
        h->a_cap = need * c.max_batch;
    }
    const long long n_a = rnd((h->a_cap + 1) / 2);   // floats per head or tail array
    // the fused upsampler input split writes a fourth operand pair
    h->ms_on = c.n_resblocks == 3 && n_a > 0;
    if (h->ms_on) {
        bool any = false;
        int Cs = c.decoder_dim;
        for (int i = 0; i + 1 < c.n_stages; ++i) {
            Cs /= 2;
            any = any || (h->stage_tc[i] && !h->stage_fused[i] && h->ups_tc[i + 1] && amp_gemm_split_fusable(Cs));
        }
        h->ms_on = any;
    }
    const int n_pairs = c.n_resblocks + (h->ms_on ? 1 : 0);
    const long long total = n_in + n_pre + nbuf * h->stage_cap + n_lat + n_wav + 64 + 2 * n_pairs * n_a;
    h->abytes = (size_t)total * sizeof(float);
    // both device allocations before any device work, so that a failed one leaves nothing behind
    // but what fail() releases
    if (!dev_alloc(h, h->wbytes, &h->warena)) {
        g_last_error = "device allocation of the weights failed";
        return fail(MH3A_ERR_ALLOC);
    }
    if (!dev_alloc(h, h->abytes, &h->arena)) {
        g_last_error = "device allocation of the workspace failed";
        return fail(MH3A_ERR_ALLOC);
    }
    // one device copy of every folded weight
    if (cudaMemcpy(h->warena, ha.data.data(), h->wbytes, cudaMemcpyHostToDevice) != cudaSuccess)
        return fail(cuda_fail(cudaGetLastError(), "weight upload"));
    for (auto& f : ha.fix) *f.dst = reinterpret_cast<float*>(h->warena) + f.off;
    for (int i = 0; i < c.n_stages; ++i) tc_finalize(&h->tc[i]);
    float* p = reinterpret_cast<float*>(h->arena);
    h->buf_in = p; p += n_in;
    h->buf_pre = p; p += n_pre;
    h->H = p; p += h->stage_cap;
    for (int j = 0; j < c.n_resblocks; ++j) { h->X[j] = p; p += h->stage_cap; }
    for (int j = 0; j < c.n_resblocks; ++j) { h->T[j] = p; p += h->stage_cap; }
    h->lat_io = p; p += n_lat;
    h->wav_io = p; p += n_wav;
    for (int j = 0; j < n_pairs && n_a > 0; ++j) {
        h->A_hi[j] = p; p += n_a;
        h->A_lo[j] = p; p += n_a;
    }
    h->dev_err = reinterpret_cast<int*>(p);
    if (cudaMemset(h->dev_err, 0, 64 * sizeof(float)) != cudaSuccess)
        return fail(cuda_fail(cudaGetLastError(), "cudaMemset"));
    for (auto& e : h->ev)
        if (cudaEventCreate(&e) != cudaSuccess) return fail(cuda_fail(cudaGetLastError(), "cudaEventCreate"));
    if (cudaDeviceSynchronize() != cudaSuccess) return fail(cuda_fail(cudaGetLastError(), "create"));
    *out = h;
    return MH3A_OK;
}

namespace {

// A decode through the graph cache: the first call for a (B, N, input, output) captures the
// decode's launches on `s` and instantiates them; every call launches the instantiated graph.
// Streams that cannot be captured (the legacy default stream) and streams the caller is already
// capturing run the launches directly.
mh3a_status decode_dispatch(mh3a_handle* h, const float* in, int B, int N, float* out, cudaStream_t s) {
    const bool special = s == nullptr || s == cudaStreamLegacy || s == cudaStreamPerThread;
    if (!h->graph_mode || h->profiling || h->kprof_stage >= 0 || special) return run_decode(h, in, B, N, out, s);
    cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
    CK_CUDA(cudaStreamIsCapturing(s, &cs), "cudaStreamIsCapturing");
    if (cs != cudaStreamCaptureStatusNone) return run_decode(h, in, B, N, out, s);
    mh3a_handle::GraphEntry* e = nullptr;
    for (auto& g : h->graphs)
        if (g.exec && g.B == B && g.N == N && g.in == in && g.out == out) e = &g;
    if (!e) {
        // first use of this key: remember it and launch directly
        mh3a_handle::GraphEntry* k = nullptr;
        for (auto& g : h->seen)
            if (g.used && g.B == B && g.N == N && g.in == in && g.out == out) k = &g;
        if (!k) {
            k = &h->seen[0];
            for (auto& g : h->seen) {
                if (!g.used) { k = &g; break; }
                if (g.used < k->used) k = &g;
            }
            k->B = B;
            k->N = N;
            k->in = in;
            k->out = out;
            k->used = ++h->graph_tick;
            return run_decode(h, in, B, N, out, s);
        }
        *k = mh3a_handle::GraphEntry{};   // second use: captured below
    }
    if (!e) {
        // a free slot, else the least recently used one
        e = &h->graphs[0];
        for (auto& g : h->graphs) {
            if (!g.exec) { e = &g; break; }
            if (g.used < e->used) e = &g;
        }
        if (e->exec) {
            // its last replay may still be running on some stream
            CK_CUDA(cudaDeviceSynchronize(), "cudaDeviceSynchronize");
            CK_CUDA(cudaGraphExecDestroy(e->exec), "cudaGraphExecDestroy");
            *e = mh3a_handle::GraphEntry{};
        }
        CK_CUDA(cudaStreamBeginCapture(s, cudaStreamCaptureModeThreadLocal), "cudaStreamBeginCapture");
        const long long l0 = h->launches;
        const mh3a_status st = run_decode(h, in, B, N, out, s);
        cudaGraph_t graph = nullptr;
        const cudaError_t ce = cudaStreamEndCapture(s, &graph);
        const long long nl = h->launches - l0;
        h->launches = l0;   // the capture itself launched nothing
        if (st != MH3A_OK || ce != cudaSuccess) {
            if (graph) cudaGraphDestroy(graph);
            return st != MH3A_OK ? st : cuda_fail(ce, "cudaStreamEndCapture");
        }
        cudaGraphExec_t exec = nullptr;
        const cudaError_t ie = cudaGraphInstantiate(&exec, graph, 0);
        cudaGraphDestroy(graph);
        if (ie != cudaSuccess) return cuda_fail(ie, "cudaGraphInstantiate");
        e->B = B;
        e->N = N;
        e->in = in;
        e->out = out;
        e->exec = exec;
        e->launches = nl;
    }
    e->used = ++h->graph_tick;
    CK_CUDA(cudaGraphLaunch(e->exec, s), "cudaGraphLaunch");
    h->launches += e->launches;
    return MH3A_OK;
}

}  // namespace

mh3a_status mh3a_set_graph_mode(mh3a_handle* h, int enable) {
    if (!h) return MH3A_ERR_INVALID_ARG;
    if (!enable) {
        CK_CUDA(cudaDeviceSynchronize(), "cudaDeviceSynchronize");   // no replay still running
        for (auto& g : h->graphs) {
            if (g.exec) {
                CK_CUDA(cudaGraphExecDestroy(g.exec), "cudaGraphExecDestroy");
            }
            g = mh3a_handle::GraphEntry{};
        }
        for (auto& g : h->seen) g = mh3a_handle::GraphEntry{};
    }
    h->graph_mode = enable != 0;
    return MH3A_OK;
}

mh3a_status mh3a_decode(mh3a_handle* h, const float* latents, int B, int N, float* out, void* stream) {
    if (!h || !latents || !out) return MH3A_ERR_INVALID_ARG;
    if (B < 1 || N < 1 || B > h->cfg.max_batch || N > h->cfg.max_frames) return MH3A_ERR_SHAPE;
    return decode_dispatch(h, latents, B, N, out, (cudaStream_t)stream);
}

mh3a_status mh3a_decode_host(mh3a_handle* h, const float* latents_host, int B, int N, float* out_host,
                             void* stream) {
    if (!h || !latents_host || !out_host) return MH3A_ERR_INVALID_ARG;
    if (B < 1 || N < 1 || B > h->cfg.max_batch || N > h->cfg.max_frames) return MH3A_ERR_SHAPE;
    cudaStream_t s = (cudaStream_t)stream;
    const size_t in_bytes = (size_t)B * h->cfg.latent_channels * N * sizeof(float);
    const size_t out_bytes = (size_t)B * h->hop * N * sizeof(float);
    // A pinned output buffer that the current device can address (page-locked memory from
    // cudaHostAlloc / cudaMallocHost is mapped into the device's address space under unified
    // addressing) is written by the decode's last kernel directly: the waveform crosses the bus
    // while that kernel runs instead of in a copy after it.  Any other host memory gets the
    // device waveform buffer and a copy.
    float* out_mapped = nullptr;
    cudaPointerAttributes pa{};
    if (cudaPointerGetAttributes(&pa, out_host) == cudaSuccess) {
        if (pa.type == cudaMemoryTypeHost && pa.devicePointer) out_mapped = static_cast<float*>(pa.devicePointer);
    } else {
        (void)cudaGetLastError();   // not a pointer the runtime knows: plain host memory
    }
    CK_CUDA(cudaMemcpyAsync(h->lat_io, latents_host, in_bytes, cudaMemcpyHostToDevice, s), "latents upload");
    mh3a_status st = decode_dispatch(h, h->lat_io, B, N, out_mapped ? out_mapped : h->wav_io, s);
    if (st) return st;
    if (!out_mapped)
        CK_CUDA(cudaMemcpyAsync(out_host, h->wav_io, out_bytes, cudaMemcpyDeviceToHost, s), "waveform download");
    CK_CUDA(cudaStreamSynchronize(s), "cudaStreamSynchronize");
    return MH3A_OK;
}

mh3a_status mh3a_amp_stage(mh3a_handle* h, const float* x, int B, int L, int stage, float* out, void* stream) {
    if (!h || !x || !out) return MH3A_ERR_INVALID_ARG;
    if (stage < 0 || stage >= h->cfg.n_stages) return MH3A_ERR_INVALID_ARG;
    if (B < 1 || L < 1) return MH3A_ERR_SHAPE;
    const int C = stage_channels(h->cfg, stage);
    if ((long long)B * C * L > h->stage_cap) return MH3A_ERR_SHAPE;
    if (h->cfg.n_resblocks != 3) return MH3A_ERR_UNSUPPORTED;
    cudaStream_t s = (cudaStream_t)stream;
    mh3a_status st = run_amp(h, stage, x, B, L, s);
    if (st) return st;
    Mean3Params mp{h->X[0], h->X[1], h->X[2], out, (long long)B * C * L, 0};
    mp.vec4 = ((reinterpret_cast<uintptr_t>(out) | reinterpret_cast<uintptr_t>(h->X[0]) |
                reinterpret_cast<uintptr_t>(h->X[1]) | reinterpret_cast<uintptr_t>(h->X[2])) & 15) == 0;
    return counted(h, launch_mean3(mp, s));
}

mh3a_status mh3a_set_profiling(mh3a_handle* h, int enable) {
    if (!h) return MH3A_ERR_INVALID_ARG;
    h->profiling = enable != 0;
    return MH3A_OK;
}

mh3a_status mh3a_set_kernel_profiling(mh3a_handle* h, int stage) {
    if (!h || stage < -1 || stage >= h->cfg.n_stages) return MH3A_ERR_INVALID_ARG;
    if (stage >= 0 && !h->kev_made) {
        int prev = 0;
        cudaGetDevice(&prev);
        cudaSetDevice(h->device);
        cudaError_t e_ = cudaSuccess;
        for (auto& li : h->kev)
            for (auto& e : li)
                if (e_ == cudaSuccess) e_ = cudaEventCreate(&e);
        cudaSetDevice(prev);
        if (e_ != cudaSuccess) return cuda_fail(e_, "cudaEventCreate");
        h->kev_made = true;
    }
    h->kprof_stage = stage;
    h->kev_rec = -1;
    return MH3A_OK;
}

mh3a_status mh3a_stage_kernel_times(mh3a_handle* h, int stage, float* act_ms, float* gemm_ms) {
    if (!h || !act_ms || !gemm_ms || stage < 0 || stage >= h->cfg.n_stages) return MH3A_ERR_INVALID_ARG;
    *act_ms = 0.f;
    *gemm_ms = 0.f;
    if (!h->kev_made || h->kev_rec != stage) return MH3A_ERR_UNSUPPORTED;
    if (h->kev_fused) {
        // one fused launch does the whole stage: its time is reported as the GEMM time
        CK_CUDA(cudaEventSynchronize(h->kev[0][1]), "cudaEventSynchronize");
        CK_CUDA(cudaEventElapsedTime(gemm_ms, h->kev[0][0], h->kev[0][1]), "cudaEventElapsedTime");
        return MH3A_OK;
    }
    CK_CUDA(cudaEventSynchronize(h->kev[5][2]), "cudaEventSynchronize");
    for (int li = 0; li < 6; ++li) {
        float a = 0.f, g = 0.f;
        CK_CUDA(cudaEventElapsedTime(&a, h->kev[li][0], h->kev[li][1]), "cudaEventElapsedTime");
        CK_CUDA(cudaEventElapsedTime(&g, h->kev[li][1], h->kev[li][2]), "cudaEventElapsedTime");
        *act_ms += a;
        *gemm_ms += g;
    }
    return MH3A_OK;
}

mh3a_status mh3a_segment_times(mh3a_handle* h, float* ms, int cap, int* count) {
    if (!h || !ms || !count || cap < 0) return MH3A_ERR_INVALID_ARG;
    *count = 0;
    if (h->nseg < 2) return MH3A_OK;
    CK_CUDA(cudaEventSynchronize(h->ev[h->nseg - 1]), "cudaEventSynchronize");
    const int n = h->nseg - 1;
    for (int i = 0; i < n && i < cap; ++i) {
        float t = 0.f;
        CK_CUDA(cudaEventElapsedTime(&t, h->ev[i], h->ev[i + 1]), "cudaEventElapsedTime");
        ms[i] = t;
    }
    *count = n < cap ? n : cap;
    return MH3A_OK;
}

long long mh3a_launch_count(const mh3a_handle* h) { return h ? h->launches : -1; }

int mh3a_stage_uses_tensor_cores(const mh3a_handle* h, int stage) {
    if (!h || stage < 0 || stage >= h->cfg.n_stages) return -1;
    return h->stage_tc[stage] ? 1 : 0;
}

int mh3a_segment_uses_tensor_cores(const mh3a_handle* h, int segment) {
    if (!h) return -1;
    const int n = 2 + 2 * h->cfg.n_stages + 1;
    if (segment < 0 || segment >= n) return -1;
    if (segment == 0 || segment == n - 1) return 0;   // input projection, output conv
    if (segment == 1) return h->pre_tc ? 1 : 0;
    const int i = (segment - 2) / 2;
    return ((segment - 2) % 2 == 0 ? h->ups_tc[i] : h->stage_tc[i]) ? 1 : 0;
}

mh3a_status mh3a_check_device_error(mh3a_handle* h) {
    if (!h) return MH3A_ERR_INVALID_ARG;
    int flag = 0;
    CK_CUDA(cudaMemcpy(&flag, h->dev_err, sizeof(int), cudaMemcpyDeviceToHost), "read device error flag");
    if (flag == 0) return MH3A_OK;
    // the flag and the tile scheduler's counters (stale after an aborted launch)
    CK_CUDA(cudaMemset(h->dev_err, 0, 64 * sizeof(int)), "clear device error flag");
    g_last_error = "a tensor-core kernel gave up waiting on its pipeline (code " + std::to_string(flag) +
                   "); its outputs are invalid";
    return MH3A_ERR_CUDA;
}

long long mh3a_device_bytes(const mh3a_handle* h) { return h ? (long long)(h->wbytes + h->abytes) : -1; }

}  // extern "C"

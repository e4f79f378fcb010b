// mh3a_config_json.cu -- mh3a_config_from_json: the architecture of a released audio VAE
// component from its config.json.
//
// The FastVideo "minimax_h3_audio_vae" page builds its configuration view from the component
// directory (`MiniMaxH3AudioVAEConfigView.from_vae_dir`); the view's fields are the diffusers
// "AutoencoderKLMiniMaxH3Audio" constructor arguments, whose defaults mirror the released
// config.json.  The decoder needs latent_channels, latent_dim, decoder_dim, decoder_rates,
// decoder_kernel_sizes, resblock_kernel_sizes, resblock_dilation_sizes, sampling_rate and the
// optional per-channel latents_mean / latents_std; every other key (the encoder's, attention
// heads, the diffusers bookkeeping keys) is skipped.
#include <cstdio>
#include <string>
#include <vector>

#include "json_reader.cuh"
#include "mh3a_internal.cuh"

namespace {

constexpr long long kMaxConfigBytes = 16ll << 20;

mh3a_status bad(const std::string& path, const std::string& why, mh3a_status st = MH3A_ERR_INVALID_ARG) {
    mh3a::set_last_error(path + ": " + why);
    return st;
}

struct Cfg : mh3a::Json {
    bool positive(int& out) {
        long long v;
        if (!uint(v)) return false;
        if (v < 1 || v > (1 << 30)) return fail("expected a positive integer");
        out = (int)v;
        return true;
    }
    // null (-> present = false) or an array of numbers
    bool floats(std::vector<double>& out, bool& present) {
        out.clear();
        present = false;
        if (null_lit()) return true;
        if (!lit('[')) return fail("expected null or an array of numbers");
        present = true;
        if (lit(']')) return true;
        for (;;) {
            double v;
            if (!number(v)) return false;
            out.push_back(v);
            if (lit(']')) return true;
            if (!lit(',')) return fail("expected ',' or ']'");
        }
    }
    bool int_rows(std::vector<std::vector<long long>>& out) {
        out.clear();
        if (!lit('[')) return fail("expected an array of arrays");
        if (lit(']')) return true;
        for (;;) {
            std::vector<long long> row;
            if (!int_array(row)) return false;
            out.push_back(std::move(row));
            if (lit(']')) return true;
            if (!lit(',')) return fail("expected ',' or ']'");
        }
    }
};

}  // namespace

mh3a_status mh3a_config_from_json(const char* path, mh3a_config* cfg, float* latents_mean, float* latents_std,
                                  int cap) {
    if (!path || !cfg || cap < 0) return MH3A_ERR_INVALID_ARG;
    const std::string P(path);
    FILE* f = std::fopen(path, "rb");
    if (!f) return bad(P, "cannot open the file");
    std::string text;
    char buf[1 << 16];
    size_t got;
    while ((got = std::fread(buf, 1, sizeof buf, f)) > 0) {
        text.append(buf, got);
        if ((long long)text.size() > kMaxConfigBytes) {
            std::fclose(f);
            return bad(P, "larger than 16 MiB");
        }
    }
    const bool read_err = std::ferror(f) != 0;
    std::fclose(f);
    if (read_err) return bad(P, "cannot read the file");

    mh3a_config c;
    mh3a_default_config(&c);
    std::vector<long long> rates, kernels, rb_kernels;
    std::vector<std::vector<long long>> dil;
    std::vector<double> mean, stdv;
    bool have_rates = false, have_kernels = false, have_rbk = false, have_dil = false;
    bool have_mean = false, have_std = false;
    Cfg J;
    J.p = text.data();
    J.e = text.data() + text.size();
    bool ok = J.lit('{');
    if (!ok) J.fail("the file is not a JSON object");
    if (ok && !J.lit('}')) {
        for (;;) {
            std::string k;
            if (!J.str(k) || !J.lit(':')) {
                ok = J.fail("bad object member");
                break;
            }
            if (k == "latent_channels") ok = J.positive(c.latent_channels);
            else if (k == "latent_dim") ok = J.positive(c.latent_dim);
            else if (k == "decoder_dim") ok = J.positive(c.decoder_dim);
            else if (k == "sampling_rate") ok = J.positive(c.sampling_rate);
            else if (k == "decoder_rates") ok = have_rates = J.int_array(rates);
            else if (k == "decoder_kernel_sizes") ok = have_kernels = J.int_array(kernels);
            else if (k == "resblock_kernel_sizes") ok = have_rbk = J.int_array(rb_kernels);
            else if (k == "resblock_dilation_sizes") ok = have_dil = J.int_rows(dil);
            else if (k == "latents_mean") ok = J.floats(mean, have_mean);
            else if (k == "latents_std") ok = J.floats(stdv, have_std);
            else ok = J.skip(1);
            if (!ok) break;
            if (J.lit('}')) break;
            if (!J.lit(',')) {
                ok = J.fail("expected ',' between members");
                break;
            }
        }
    }
    if (ok) {
        J.ws();
        if (J.p != J.e) ok = J.fail("text after the object");
    }
    if (!ok) return bad(P, "malformed config: " + J.err);

    // the list-valued fields, each against the defaults of the other when only one is given
    if (have_rates) {
        if (rates.empty() || (int)rates.size() > MH3A_MAX_STAGES)
            return bad(P, "decoder_rates: 1 to " + std::to_string(MH3A_MAX_STAGES) + " stages supported", MH3A_ERR_CONFIG);
        c.n_stages = (int)rates.size();
        for (int i = 0; i < c.n_stages; ++i) c.rates[i] = (int)rates[i];
    }
    if (have_kernels) {
        if ((int)kernels.size() != c.n_stages)
            return bad(P, "decoder_kernel_sizes has " + std::to_string(kernels.size()) + " entries for " +
                              std::to_string(c.n_stages) + " stages",
                       MH3A_ERR_CONFIG);
        for (int i = 0; i < c.n_stages; ++i) c.kernels[i] = (int)kernels[i];
    } else if (have_rates && c.n_stages != 7) {
        return bad(P, "decoder_rates changes the stage count but decoder_kernel_sizes is absent", MH3A_ERR_CONFIG);
    }
    if (have_rbk) {
        if (rb_kernels.empty() || (int)rb_kernels.size() > MH3A_MAX_RESBLOCKS)
            return bad(P, "resblock_kernel_sizes: 1 to " + std::to_string(MH3A_MAX_RESBLOCKS) + " blocks supported",
                       MH3A_ERR_CONFIG);
        c.n_resblocks = (int)rb_kernels.size();
        for (int j = 0; j < c.n_resblocks; ++j) c.rb_kernels[j] = (int)rb_kernels[j];
    }
    if (have_dil) {
        if ((int)dil.size() != c.n_resblocks)
            return bad(P, "resblock_dilation_sizes has " + std::to_string(dil.size()) + " rows for " +
                              std::to_string(c.n_resblocks) + " residual blocks",
                       MH3A_ERR_CONFIG);
        const size_t nd = dil[0].size();
        if (nd == 0 || (int)nd > MH3A_MAX_DILATIONS)
            return bad(P, "resblock_dilation_sizes: 1 to " + std::to_string(MH3A_MAX_DILATIONS) + " dilations supported",
                       MH3A_ERR_CONFIG);
        for (const auto& row : dil)
            if (row.size() != nd) return bad(P, "resblock_dilation_sizes rows differ in length", MH3A_ERR_CONFIG);
        c.n_dilations = (int)nd;
        for (int j = 0; j < c.n_resblocks; ++j)
            for (int m = 0; m < c.n_dilations; ++m) c.rb_dilations[j][m] = (int)dil[j][m];
    } else if (have_rbk && c.n_resblocks != 3) {
        return bad(P, "resblock_kernel_sizes changes the block count but resblock_dilation_sizes is absent",
                   MH3A_ERR_CONFIG);
    }
    c.latents_mean = nullptr;
    c.latents_std = nullptr;
    const struct {
        bool present;
        const std::vector<double>* v;
        float* dst;
        const float** field;
        const char* name;
    } stats[2] = {{have_mean, &mean, latents_mean, &c.latents_mean, "latents_mean"},
                  {have_std, &stdv, latents_std, &c.latents_std, "latents_std"}};
    for (const auto& s : stats) {
        if (!s.present) continue;
        if ((int)s.v->size() != c.latent_channels)
            return bad(P, std::string(s.name) + " has " + std::to_string(s.v->size()) + " values for " +
                              std::to_string(c.latent_channels) + " latent channels",
                       MH3A_ERR_SHAPE);
        if (!s.dst || (int)s.v->size() > cap)
            return bad(P, std::string(s.name) + ": no caller buffer of " + std::to_string(s.v->size()) + " floats",
                       MH3A_ERR_SHAPE);
        for (size_t i = 0; i < s.v->size(); ++i) s.dst[i] = (float)(*s.v)[i];
        *s.field = s.dst;
    }
    *cfg = c;
    return MH3A_OK;
}

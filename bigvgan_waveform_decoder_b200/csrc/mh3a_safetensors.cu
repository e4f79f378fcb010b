// mh3a_safetensors.cu -- mh3a_create_from_safetensors: a decoder built straight from the audio
// VAE component's checkpoint file.
//
// The FastVideo "minimax_h3_audio_vae" page (`mlx_h3_audio_vae_from_dir`,
// `mlx_h3_audio_vae_from_file`) loads the released weights from one file,
// `diffusion_pytorch_model.safetensors`, keeps the tensors whose names start with the decode
// prefixes "dec_in_proj." and "decoder." (plus encoder prefixes this library does not run),
// requires "dec_in_proj.weight", "decoder.conv_pre.weight_v" and "decoder.conv_post.weight_v",
// and insists on fp32 storage.  This file reads that format:
//
//   bytes [0, 8)            header length n, unsigned 64-bit little endian
//   bytes [8, 8 + n)        JSON object: name -> {"dtype": "F32", "shape": [..],
//                           "data_offsets": [begin, end]}, plus an optional "__metadata__"
//                           object of strings
//   bytes [8 + n, size)     the tensor data; a tensor's bytes are [begin, end) of this section
//
// Only the decode tensors are read; every other entry is parsed and skipped.  The tensors are
// copied into host buffers and handed to mh3a_create_with_allocator as a weight table, so all
// shape and completeness checks of the architecture stay in one place.
#include <cstdint>
#include <cstdio>
#include <cstring>
#include <string>
#include <vector>

#include "json_reader.cuh"
#include "mh3a_internal.cuh"

namespace {

constexpr unsigned long long kMaxHeader = 100ull << 20;   // the format caps the header at 100 MB

struct Entry {
    std::string name, dtype;
    std::vector<long long> shape;
    long long begin = -1, end = -1;
};

// The safetensors header: name -> tensor entry, plus "__metadata__".
struct StHeader : mh3a::Json {
    bool entry(Entry& t) {
        if (!lit('{')) return fail("a tensor entry is not an object");
        bool have_dtype = false, have_shape = false, have_offsets = false;
        if (!lit('}')) {
            for (;;) {
                std::string k;
                if (!str(k) || !lit(':')) return fail("bad tensor field");
                if (k == "dtype") {
                    if (!str(t.dtype)) return false;
                    have_dtype = true;
                } else if (k == "shape") {
                    if (!int_array(t.shape)) return false;
                    have_shape = true;
                } else if (k == "data_offsets") {
                    std::vector<long long> o;
                    if (!int_array(o)) return false;
                    if (o.size() != 2) return fail("data_offsets must hold two integers");
                    t.begin = o[0];
                    t.end = o[1];
                    have_offsets = true;
                } else if (!skip(1)) {
                    return false;
                }
                if (lit('}')) break;
                if (!lit(',')) return fail("expected ',' in a tensor entry");
            }
        }
        if (!have_dtype || !have_shape || !have_offsets) return fail("a tensor entry lacks dtype, shape or data_offsets");
        return true;
    }
    bool header(std::vector<Entry>& out) {
        if (!lit('{')) return fail("the header is not a JSON object");
        if (lit('}')) {
            ws();
            return p == e ? true : fail("text after the header object");
        }
        for (;;) {
            Entry t;
            if (!str(t.name) || !lit(':')) return fail("bad header member");
            if (t.name == "__metadata__") {
                if (!skip(1)) return false;
            } else {
                if (!entry(t)) return false;
                out.push_back(std::move(t));
            }
            if (lit('}')) break;
            if (!lit(',')) return fail("expected ',' between header members");
        }
        ws();
        return p == e ? true : fail("text after the header object");
    }
};

bool decode_tensor(const std::string& n) {
    return n.compare(0, 12, "dec_in_proj.") == 0 || n.compare(0, 8, "decoder.") == 0;
}

mh3a_status bad(const std::string& path, const std::string& why, mh3a_status st = MH3A_ERR_INVALID_ARG) {
    mh3a::set_last_error(path + ": " + why);
    return st;
}

struct File {
    FILE* f = nullptr;
    ~File() {
        if (f) std::fclose(f);
    }
};

}  // namespace

mh3a_status mh3a_create_from_safetensors(const mh3a_config* cfg, const char* path, const mh3a_allocator* allocator,
                                         mh3a_handle** out) {
    if (out) *out = nullptr;
    if (!cfg || !path || !out) return MH3A_ERR_INVALID_ARG;
    const std::string P(path);
    File F;
    F.f = std::fopen(path, "rb");
    if (!F.f) return bad(P, "cannot open the file");
    if (fseeko(F.f, 0, SEEK_END) != 0) return bad(P, "cannot seek");
    const long long size = (long long)ftello(F.f);
    if (size < 8 || fseeko(F.f, 0, SEEK_SET) != 0) return bad(P, "shorter than the 8-byte header length");
    unsigned char lenb[8];
    if (std::fread(lenb, 1, 8, F.f) != 8) return bad(P, "cannot read the header length");
    unsigned long long n = 0;
    for (int i = 7; i >= 0; --i) n = (n << 8) | lenb[i];
    if (n == 0 || n > kMaxHeader || (long long)n > size - 8) return bad(P, "header length out of range");
    std::string text((size_t)n, '\0');
    if (std::fread(&text[0], 1, (size_t)n, F.f) != (size_t)n) return bad(P, "cannot read the header");
    std::vector<Entry> all;
    StHeader J;
    J.p = text.data();
    J.e = text.data() + text.size();
    if (!J.header(all)) return bad(P, "malformed header: " + J.err);
    const long long data0 = 8 + (long long)n, data_bytes = size - data0;

    // the decode tensors: F32, at most 3 dims, offsets inside the data section and matching the
    // shape
    std::vector<const Entry*> use;
    for (const Entry& t : all) {
        if (t.begin < 0 || t.end < t.begin || t.end > data_bytes)
            return bad(P, "tensor '" + t.name + "': data_offsets outside the data section");
        if (!decode_tensor(t.name)) continue;
        if (t.dtype != "F32")
            return bad(P, "tensor '" + t.name + "' is stored as " + t.dtype + "; the decoder takes fp32 storage only",
                       MH3A_ERR_UNSUPPORTED);
        if (t.shape.empty() || t.shape.size() > 3)
            return bad(P, "tensor '" + t.name + "' has " + std::to_string(t.shape.size()) + " dims (1 to 3 supported)",
                       MH3A_ERR_UNSUPPORTED);
        long long elems = 1;
        for (long long d : t.shape) {
            if (d < 1 || elems > (1ll << 40) / d) return bad(P, "tensor '" + t.name + "': bad shape");
            elems *= d;
        }
        if (t.end - t.begin != 4 * elems) return bad(P, "tensor '" + t.name + "': byte count disagrees with its shape");
        use.push_back(&t);
    }
    static const char* const required[] = {"dec_in_proj.weight", "decoder.conv_pre.weight_v",
                                           "decoder.conv_post.weight_v"};
    for (const char* r : required) {
        bool found = false;
        for (const Entry* t : use) found = found || t->name == r;
        if (!found) return bad(P, std::string("required tensor '") + r + "' is missing", MH3A_ERR_MISSING_WEIGHT);
    }

    // read them (little-endian fp32, the format's byte order) and build the weight table
    std::vector<std::vector<float>> data(use.size());
    std::vector<mh3a_tensor> table(use.size());
    for (size_t i = 0; i < use.size(); ++i) {
        const Entry& t = *use[i];
        const size_t elems = (size_t)((t.end - t.begin) / 4);
        try {
            data[i].resize(elems);
        } catch (...) {
            return bad(P, "host allocation for tensor '" + t.name + "' failed", MH3A_ERR_ALLOC);
        }
        if (fseeko(F.f, (off_t)(data0 + t.begin), SEEK_SET) != 0 ||
            std::fread(data[i].data(), 4, elems, F.f) != elems)
            return bad(P, "cannot read tensor '" + t.name + "'");
        mh3a_tensor& m = table[i];
        m.name = t.name.c_str();
        m.host_data = data[i].data();
        m.ndim = (int)t.shape.size();
        for (int d = 0; d < 3; ++d) m.shape[d] = d < m.ndim ? t.shape[d] : 1;
    }
    std::fclose(F.f);
    F.f = nullptr;
    return mh3a_create_with_allocator(cfg, table.data(), (int)table.size(), allocator, out);
}

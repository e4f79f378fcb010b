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

#include "mh3a_internal.cuh"

namespace {

constexpr unsigned long long kMaxHeader = 100ull << 20;   // the format caps the header at 100 MB
constexpr int kMaxDepth = 64;                             // nesting limit of skipped JSON values

struct Entry {
    std::string name, dtype;
    std::vector<long long> shape;
    long long begin = -1, end = -1;
};

// A small JSON reader for the header: objects, arrays, strings (with escapes), integers and the
// literals; fractions and exponents are accepted only inside skipped values.
struct Json {
    const char* p;
    const char* e;
    std::string err;

    bool fail(const char* what) {
        if (err.empty()) err = what;
        return false;
    }
    void ws() {
        while (p < e && (*p == ' ' || *p == '\t' || *p == '\n' || *p == '\r')) ++p;
    }
    bool lit(char c) {
        ws();
        if (p < e && *p == c) {
            ++p;
            return true;
        }
        return false;
    }
    static int hexv(char c) {
        if (c >= '0' && c <= '9') return c - '0';
        if (c >= 'a' && c <= 'f') return c - 'a' + 10;
        if (c >= 'A' && c <= 'F') return c - 'A' + 10;
        return -1;
    }
    static void utf8(std::string& out, unsigned cp) {
        if (cp < 0x80) {
            out += (char)cp;
        } else if (cp < 0x800) {
            out += (char)(0xC0 | (cp >> 6));
            out += (char)(0x80 | (cp & 0x3F));
        } else if (cp < 0x10000) {
            out += (char)(0xE0 | (cp >> 12));
            out += (char)(0x80 | ((cp >> 6) & 0x3F));
            out += (char)(0x80 | (cp & 0x3F));
        } else {
            out += (char)(0xF0 | (cp >> 18));
            out += (char)(0x80 | ((cp >> 12) & 0x3F));
            out += (char)(0x80 | ((cp >> 6) & 0x3F));
            out += (char)(0x80 | (cp & 0x3F));
        }
    }
    bool str(std::string& out) {
        out.clear();
        if (!lit('"')) return fail("expected a string");
        while (p < e && *p != '"') {
            const unsigned char c = (unsigned char)*p++;
            if (c < 0x20) return fail("control character in a string");
            if (c != '\\') {
                out += (char)c;
                continue;
            }
            if (p >= e) return fail("unterminated escape");
            const char x = *p++;
            switch (x) {
                case '"': out += '"'; break;
                case '\\': out += '\\'; break;
                case '/': out += '/'; break;
                case 'b': out += '\b'; break;
                case 'f': out += '\f'; break;
                case 'n': out += '\n'; break;
                case 'r': out += '\r'; break;
                case 't': out += '\t'; break;
                case 'u': {
                    if (e - p < 4) return fail("short \\u escape");
                    unsigned cp = 0;
                    for (int i = 0; i < 4; ++i) {
                        const int v = hexv(p[i]);
                        if (v < 0) return fail("bad \\u escape");
                        cp = cp * 16 + (unsigned)v;
                    }
                    p += 4;
                    if (cp >= 0xD800 && cp < 0xDC00) {   // a surrogate pair
                        if (e - p < 6 || p[0] != '\\' || p[1] != 'u') return fail("lone surrogate");
                        unsigned lo = 0;
                        for (int i = 0; i < 4; ++i) {
                            const int v = hexv(p[2 + i]);
                            if (v < 0) return fail("bad \\u escape");
                            lo = lo * 16 + (unsigned)v;
                        }
                        if (lo < 0xDC00 || lo >= 0xE000) return fail("lone surrogate");
                        p += 6;
                        cp = 0x10000 + ((cp - 0xD800) << 10) + (lo - 0xDC00);
                    }
                    utf8(out, cp);
                    break;
                }
                default: return fail("bad escape");
            }
        }
        if (p >= e) return fail("unterminated string");
        ++p;
        return true;
    }
    // A non-negative integer that fits in 63 bits.
    bool uint(long long& v) {
        ws();
        if (p >= e || *p < '0' || *p > '9') return fail("expected a non-negative integer");
        v = 0;
        while (p < e && *p >= '0' && *p <= '9') {
            if (v > (INT64_MAX - 9) / 10) return fail("integer too large");
            v = v * 10 + (*p++ - '0');
        }
        if (p < e && (*p == '.' || *p == 'e' || *p == 'E')) return fail("expected an integer");
        return true;
    }
    bool int_array(std::vector<long long>& out) {
        out.clear();
        if (!lit('[')) return fail("expected an array");
        if (lit(']')) return true;
        for (;;) {
            long long v;
            if (!uint(v)) return false;
            out.push_back(v);
            if (lit(']')) return true;
            if (!lit(',')) return fail("expected ',' or ']'");
        }
    }
    bool skip(int depth) {
        if (depth > kMaxDepth) return fail("nesting too deep");
        ws();
        if (p >= e) return fail("unexpected end");
        if (*p == '"') {
            std::string s;
            return str(s);
        }
        if (*p == '{' || *p == '[') {
            const char close = (*p == '{') ? '}' : ']';
            const bool obj = *p == '{';
            ++p;
            if (lit(close)) return true;
            for (;;) {
                if (obj) {
                    std::string k;
                    if (!str(k) || !lit(':')) return fail("bad object member");
                }
                if (!skip(depth + 1)) return false;
                if (lit(close)) return true;
                if (!lit(',')) return fail("expected ',' in a container");
            }
        }
        static const char* const lits[] = {"true", "false", "null"};
        for (const char* l : lits) {
            const size_t n = std::strlen(l);
            if ((size_t)(e - p) >= n && std::memcmp(p, l, n) == 0) {
                p += n;
                return true;
            }
        }
        // a number
        const char* s = p;
        if (p < e && *p == '-') ++p;
        while (p < e && ((*p >= '0' && *p <= '9') || *p == '.' || *p == 'e' || *p == 'E' || *p == '+' || *p == '-'))
            ++p;
        return p > s ? true : fail("unexpected character");
    }
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
    Json J{text.data(), text.data() + text.size(), {}};
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

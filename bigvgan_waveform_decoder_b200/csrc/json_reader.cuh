// json_reader.cuh -- a small JSON reader for the host-side file formats the library reads
// (the safetensors header, the component's config.json): objects, arrays, strings with
// escapes, integers, numbers and the literals.  Values it is not asked for are skipped with a
// nesting limit.  A reader holds only its position in one text.
#pragma once

#include <cstdint>
#include <cstdlib>
#include <cstring>
#include <string>
#include <vector>

namespace mh3a {

constexpr int kJsonMaxDepth = 64;   // nesting limit of skipped values

struct Json {
    const char* p = nullptr;   // next character
    const char* e = nullptr;   // end of the text
    std::string err;           // the first error

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
    // Any JSON number, as a double.
    bool number(double& v) {
        ws();
        const char* s = p;
        if (p < e && *p == '-') ++p;
        if (p >= e || *p < '0' || *p > '9') return fail("expected a number");
        while (p < e && ((*p >= '0' && *p <= '9') || *p == '.' || *p == 'e' || *p == 'E' || *p == '+' || *p == '-'))
            ++p;
        const std::string tok(s, p);
        char* endp = nullptr;
        v = std::strtod(tok.c_str(), &endp);
        if (!endp || *endp != '\0') return fail("malformed number");
        return true;
    }
    // The literal null (consumed when present).
    bool null_lit() {
        ws();
        if (e - p >= 4 && std::memcmp(p, "null", 4) == 0) {
            p += 4;
            return true;
        }
        return false;
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
        if (depth > kJsonMaxDepth) return fail("nesting too deep");
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
};

}  // namespace mh3a

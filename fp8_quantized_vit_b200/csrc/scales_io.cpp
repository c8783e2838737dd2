// Static per-layer scale file (vLLM "FP8 ViT Encoder Attention", "Scale File
// Format" and "Calibrate-Once, Reuse Workflow"):
//   { "visual.blocks.0.attn.attn": {"q": 224.0, "k": 198.0, "v": 210.0}, ... }
// with q_scale / k_scale / v_scale accepted as aliases.  The numbers are in
// the amax domain: the calibration pass saves margin (default 1.5) x the
// observed amax, and the descale is value / 448.
//
// A small recursive-descent JSON reader: objects, arrays, strings with
// escapes, numbers, true/false/null.  Only the layout above is interpreted;
// other members are parsed and ignored.
#include <cerrno>
#include <cmath>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <string>

#include "fp8vit.h"

namespace {

struct Reader {
    const char* p;
    const char* end;
    bool ok = true;

    void ws() {
        while (p < end && (*p == ' ' || *p == '\t' || *p == '\n' || *p == '\r')) ++p;
    }
    bool eat(char c) {
        ws();
        if (p < end && *p == c) {
            ++p;
            return true;
        }
        return false;
    }
    bool string(std::string* out) {
        ws();
        if (p >= end || *p != '"') return ok = false;
        ++p;
        std::string s;
        while (p < end && *p != '"') {
            char c = *p++;
            if (c == '\\') {
                if (p >= end) return ok = false;
                char e = *p++;
                switch (e) {
                    case '"': s += '"'; break;
                    case '\\': s += '\\'; break;
                    case '/': s += '/'; break;
                    case 'b': s += '\b'; break;
                    case 'f': s += '\f'; break;
                    case 'n': s += '\n'; break;
                    case 'r': s += '\r'; break;
                    case 't': s += '\t'; break;
                    case 'u': {
                        if (end - p < 4) return ok = false;
                        unsigned v = 0;
                        for (int i = 0; i < 4; ++i) {
                            char h = *p++;
                            v <<= 4;
                            if (h >= '0' && h <= '9') v |= (unsigned)(h - '0');
                            else if (h >= 'a' && h <= 'f') v |= (unsigned)(h - 'a' + 10);
                            else if (h >= 'A' && h <= 'F') v |= (unsigned)(h - 'A' + 10);
                            else return ok = false;
                        }
                        if (v < 0x80) s += (char)v;
                        else if (v < 0x800) {
                            s += (char)(0xC0 | (v >> 6));
                            s += (char)(0x80 | (v & 0x3F));
                        } else {
                            s += (char)(0xE0 | (v >> 12));
                            s += (char)(0x80 | ((v >> 6) & 0x3F));
                            s += (char)(0x80 | (v & 0x3F));
                        }
                        break;
                    }
                    default: return ok = false;
                }
            } else {
                if ((unsigned char)c < 0x20) return ok = false;
                s += c;
            }
        }
        if (p >= end) return ok = false;
        ++p;  // closing quote
        if (out) *out = s;
        return true;
    }
    bool number(double* out) {
        ws();
        const char* s = p;
        if (p < end && (*p == '-' || *p == '+')) ++p;
        while (p < end && ((*p >= '0' && *p <= '9') || *p == '.' || *p == 'e' || *p == 'E' ||
                           *p == '-' || *p == '+'))
            ++p;
        if (p == s) return ok = false;
        std::string tok(s, p);
        char* q = nullptr;
        errno = 0;
        double v = std::strtod(tok.c_str(), &q);
        if (q == tok.c_str() || *q != '\0' || !std::isfinite(v)) return ok = false;
        if (out) *out = v;
        return true;
    }
    bool literal(const char* w) {
        ws();
        size_t n = std::strlen(w);
        if ((size_t)(end - p) < n || std::strncmp(p, w, n) != 0) return ok = false;
        p += n;
        return true;
    }
    // Parse and discard any JSON value.
    bool skip_value(int depth = 0) {
        if (depth > 64) return ok = false;
        ws();
        if (p >= end) return ok = false;
        char c = *p;
        if (c == '{') {
            ++p;
            if (eat('}')) return true;
            do {
                if (!string(nullptr) || !eat(':') || !skip_value(depth + 1)) return ok = false;
            } while (eat(','));
            return eat('}') || (ok = false);
        }
        if (c == '[') {
            ++p;
            if (eat(']')) return true;
            do {
                if (!skip_value(depth + 1)) return ok = false;
            } while (eat(','));
            return eat(']') || (ok = false);
        }
        if (c == '"') return string(nullptr);
        if (c == 't') return literal("true");
        if (c == 'f') return literal("false");
        if (c == 'n') return literal("null");
        return number(nullptr);
    }
};

// Parse one layer object {"q": .., "k": .., "v": ..} (aliases allowed).
fp8vit_status parse_layer(Reader& r, float out[3]) {
    if (!r.eat('{')) return FP8VIT_EPARSE;
    bool have[3] = {false, false, false};
    double val[3] = {0, 0, 0};
    static const char* names[3][2] = {{"q", "q_scale"}, {"k", "k_scale"}, {"v", "v_scale"}};
    if (!r.eat('}')) {
        do {
            std::string key;
            if (!r.string(&key) || !r.eat(':')) return FP8VIT_EPARSE;
            int which = -1;
            for (int t = 0; t < 3; ++t)
                if (key == names[t][0] || key == names[t][1]) which = t;
            if (which < 0) {
                if (!r.skip_value()) return FP8VIT_EPARSE;
                continue;
            }
            double v;
            if (!r.number(&v)) return FP8VIT_EPARSE;
            // an amax-domain value: non-negative and finite as the fp32 it is used as
            if (!(v >= 0.0) || !std::isfinite((float)v)) return FP8VIT_EPARSE;
            if (have[which] && (float)val[which] != (float)v) return FP8VIT_EPARSE;
            have[which] = true;
            val[which] = v;
        } while (r.eat(','));
        if (!r.eat('}')) return FP8VIT_EPARSE;
    }
    for (int t = 0; t < 3; ++t) {
        if (!have[t]) return FP8VIT_EPARSE;
        out[t] = (float)val[t];
    }
    return FP8VIT_OK;
}

bool read_file(const char* path, std::string* out) {
    FILE* f = std::fopen(path, "rb");
    if (!f) return false;
    char buf[65536];
    size_t n;
    while ((n = std::fread(buf, 1, sizeof buf, f)) > 0) out->append(buf, n);
    bool err = std::ferror(f) != 0;
    std::fclose(f);
    return !err;
}

void write_json_string(FILE* f, const char* s) {
    std::fputc('"', f);
    for (const unsigned char* c = (const unsigned char*)s; *c; ++c) {
        if (*c == '"' || *c == '\\') std::fprintf(f, "\\%c", *c);
        else if (*c < 0x20) std::fprintf(f, "\\u%04x", *c);
        else std::fputc(*c, f);
    }
    std::fputc('"', f);
}

}  // namespace

extern "C" {

fp8vit_status fp8_static_scales_load(const char* path, const char* layer, float out_qkv[3]) {
    if (!path || !layer || !out_qkv) return FP8VIT_EINVAL;
    std::string text;
    if (!read_file(path, &text)) return FP8VIT_EIO;
    Reader r{text.data(), text.data() + text.size()};
    if (!r.eat('{')) return FP8VIT_EPARSE;
    bool found = false;
    float vals[3] = {0, 0, 0};
    if (!r.eat('}')) {
        do {
            std::string name;
            if (!r.string(&name) || !r.eat(':')) return FP8VIT_EPARSE;
            float tmp[3];
            fp8vit_status s = parse_layer(r, tmp);
            if (s != FP8VIT_OK) return s;
            if (name == layer) {
                if (found && (tmp[0] != vals[0] || tmp[1] != vals[1] || tmp[2] != vals[2]))
                    return FP8VIT_EPARSE;
                found = true;
                for (int t = 0; t < 3; ++t) vals[t] = tmp[t];
            }
        } while (r.eat(','));
        if (!r.eat('}')) return FP8VIT_EPARSE;
    }
    r.ws();
    if (r.p != r.end) return FP8VIT_EPARSE;
    if (!found) return FP8VIT_ENOTFOUND;
    for (int t = 0; t < 3; ++t) out_qkv[t] = vals[t];
    return FP8VIT_OK;
}

fp8vit_status fp8_static_scales_save(const char* path, int32_t n_layers,
                                     const char* const* layers, const float* qkv_amax,
                                     float margin) {
    if (!path || n_layers < 0 || (n_layers > 0 && (!layers || !qkv_amax))) return FP8VIT_EINVAL;
    if (!(margin > 0.0f) || !std::isfinite(margin)) return FP8VIT_EINVAL;
    for (int32_t i = 0; i < n_layers; ++i)
        if (!layers[i]) return FP8VIT_EINVAL;
    FILE* f = std::fopen(path, "wb");
    if (!f) return FP8VIT_EIO;
    std::fputs("{\n", f);
    static const char* keys[3] = {"q", "k", "v"};
    for (int32_t i = 0; i < n_layers; ++i) {
        std::fputs("    ", f);
        write_json_string(f, layers[i]);
        std::fputs(": {", f);
        for (int t = 0; t < 3; ++t) {
            volatile float prod = margin * qkv_amax[3 * i + t];  // fp32 product
            std::fprintf(f, "\"%s\": %.9g%s", keys[t], (double)prod, t < 2 ? ", " : "");
        }
        std::fprintf(f, "}%s\n", i + 1 < n_layers ? "," : "");
    }
    std::fputs("}\n", f);
    bool err = std::ferror(f) != 0;
    if (std::fclose(f) != 0 || err) return FP8VIT_EIO;
    return FP8VIT_OK;
}

}  // extern "C"

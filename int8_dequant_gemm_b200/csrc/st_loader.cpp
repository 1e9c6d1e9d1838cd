// Reader of quantized checkpoints in the plain safetensors container; the
// weight format follows from the tensors' dtypes.
//
// Container (the standard safetensors layout, which both quantized cards use
// with nothing of their own added): an 8-byte little-endian header length
// n, n bytes of JSON mapping each tensor name to {"dtype", "shape",
// "data_offsets": [begin, end]} (plus an optional "__metadata__" object of
// strings), then the tensors' bytes; offsets count from the end of the
// header.
//
// Formats ("Quantization format" on the int4 and int8 cards, "FP8 Format" on
// the FP8 card):
//   q4    <name>          U8  [N, K/2]        packed codes, low nibble = even k
//         <name>.q4_scale F16 [N, K/32, 2]    (scale, min) per group of 32
//                             (also accepted: [N, K/16], the same bytes)
//   q8    <name>          I8  [N, K]          codes
//         <name>.q_scale  F32 [N] or [N, 1]   per-row scale
//   e4m3  <name>          F8_E4M3 [N, K]      float8_e4m3fn weights
// Any other combination is reported as unsupported.  The file is mapped
// read-only; a weight's pointers stay valid until rt_st_close.
#include <fcntl.h>
#include <sys/mman.h>
#include <sys/stat.h>
#include <unistd.h>

#include <cstdint>
#include <cstring>
#include <map>
#include <new>
#include <string>
#include <vector>

#include "../../include/rtq.h"

namespace {

struct TensorInfo {
    std::string dtype;
    std::vector<int64_t> shape;
    uint64_t begin = 0, end = 0;
};

// Minimal JSON reader for the safetensors header: objects, arrays, strings,
// non-negative integers; true/false/null and other numbers are skipped.
class Json {
  public:
    Json(const char *p, size_t n) : p_(p), e_(p + n) {}

    bool parse_header(std::map<std::string, TensorInfo> &out) {
        ws();
        if (!eat('{')) return false;
        ws();
        if (eat('}')) return done();
        while (true) {
            std::string key;
            ws();
            if (!string(key)) return false;
            ws();
            if (!eat(':')) return false;
            ws();
            if (key == "__metadata__") {
                if (!skip_value()) return false;
            } else {
                TensorInfo t;
                if (!tensor(t) || out.count(key)) return false;
                out.emplace(key, t);
            }
            ws();
            if (eat(',')) continue;
            if (eat('}')) return done();
            return false;
        }
    }

  private:
    const char *p_, *e_;

    bool done() {
        ws();
        return p_ == e_;
    }
    void ws() {
        while (p_ < e_ && (*p_ == ' ' || *p_ == '\t' || *p_ == '\n' || *p_ == '\r')) ++p_;
    }
    bool eat(char c) {
        if (p_ < e_ && *p_ == c) {
            ++p_;
            return true;
        }
        return false;
    }
    bool string(std::string &s) {
        if (!eat('"')) return false;
        while (p_ < e_ && *p_ != '"') {
            char c = *p_++;
            if (c == '\\') {
                if (p_ >= e_) return false;
                const char x = *p_++;
                switch (x) {
                    case '"': c = '"'; break;
                    case '\\': c = '\\'; break;
                    case '/': c = '/'; break;
                    case 'b': c = '\b'; break;
                    case 'f': c = '\f'; break;
                    case 'n': c = '\n'; break;
                    case 'r': c = '\r'; break;
                    case 't': c = '\t'; break;
                    case 'u': {
                        // keep the escape verbatim (names of interest are ASCII)
                        if (e_ - p_ < 4) return false;
                        s += "\\u";
                        s.append(p_, 4);
                        p_ += 4;
                        continue;
                    }
                    default: return false;
                }
            } else if (static_cast<unsigned char>(c) < 0x20) {
                return false;
            }
            s += c;
        }
        return eat('"');
    }
    bool integer(uint64_t &v) {
        if (p_ >= e_ || *p_ < '0' || *p_ > '9') return false;
        v = 0;
        while (p_ < e_ && *p_ >= '0' && *p_ <= '9') {
            const uint64_t d = static_cast<uint64_t>(*p_++ - '0');
            if (v > (UINT64_MAX - d) / 10) return false;
            v = v * 10 + d;
        }
        return true;
    }
    bool int_array(std::vector<int64_t> &a) {
        if (!eat('[')) return false;
        ws();
        if (eat(']')) return true;
        while (true) {
            ws();
            uint64_t v;
            if (!integer(v) || v > static_cast<uint64_t>(INT64_MAX)) return false;
            a.push_back(static_cast<int64_t>(v));
            ws();
            if (eat(',')) continue;
            return eat(']');
        }
    }
    bool tensor(TensorInfo &t) {
        if (!eat('{')) return false;
        bool has_dtype = false, has_shape = false, has_off = false;
        while (true) {
            ws();
            std::string key;
            if (!string(key)) return false;
            ws();
            if (!eat(':')) return false;
            ws();
            if (key == "dtype") {
                if (!string(t.dtype)) return false;
                has_dtype = true;
            } else if (key == "shape") {
                if (!int_array(t.shape)) return false;
                has_shape = true;
            } else if (key == "data_offsets") {
                std::vector<int64_t> o;
                if (!int_array(o) || o.size() != 2 || o[1] < o[0]) return false;
                t.begin = static_cast<uint64_t>(o[0]);
                t.end = static_cast<uint64_t>(o[1]);
                has_off = true;
            } else if (!skip_value()) {
                return false;
            }
            ws();
            if (eat(',')) continue;
            if (!eat('}')) return false;
            return has_dtype && has_shape && has_off;
        }
    }
    bool skip_value(int depth = 0) {
        if (depth > 32) return false;
        ws();
        if (p_ >= e_) return false;
        if (*p_ == '"') {
            std::string s;
            return string(s);
        }
        if (*p_ == '{' || *p_ == '[') {
            const char close = *p_ == '{' ? '}' : ']';
            const bool obj = *p_ == '{';
            ++p_;
            ws();
            if (eat(close)) return true;
            while (true) {
                ws();
                if (obj) {
                    std::string k;
                    if (!string(k)) return false;
                    ws();
                    if (!eat(':')) return false;
                }
                if (!skip_value(depth + 1)) return false;
                ws();
                if (eat(',')) continue;
                return eat(close);
            }
        }
        // number, true, false, null
        const char *q = p_;
        while (p_ < e_ && std::strchr("+-.0123456789eEtruefalsn", *p_)) ++p_;
        return p_ > q;
    }
};

int64_t dtype_size(const std::string &d) {
    if (d == "U8" || d == "I8" || d == "F8_E4M3" || d == "F8_E5M2" || d == "BOOL") return 1;
    if (d == "F16" || d == "BF16" || d == "I16" || d == "U16") return 2;
    if (d == "F32" || d == "I32" || d == "U32") return 4;
    if (d == "F64" || d == "I64" || d == "U64") return 8;
    return 0;
}

}  // namespace

struct rt_st_file {
    void *map = nullptr;
    size_t size = 0;
    const uint8_t *data = nullptr;   // first byte after the header
    size_t data_size = 0;
    std::map<std::string, TensorInfo> tensors;
};

namespace {

rt_status parse(rt_st_file *f) {
    if (f->size < 8) return RT_ERR_FORMAT;
    const uint8_t *b = static_cast<const uint8_t *>(f->map);
    uint64_t n = 0;
    for (int i = 7; i >= 0; --i) n = (n << 8) | b[i];
    if (n == 0 || n > f->size - 8 || n > (uint64_t(100) << 20)) return RT_ERR_FORMAT;
    Json j(reinterpret_cast<const char *>(b + 8), static_cast<size_t>(n));
    if (!j.parse_header(f->tensors)) return RT_ERR_FORMAT;
    f->data = b + 8 + n;
    f->data_size = f->size - 8 - n;
    for (const auto &kv : f->tensors) {
        const TensorInfo &t = kv.second;
        const int64_t es = dtype_size(t.dtype);
        if (es == 0 || t.end > f->data_size) return RT_ERR_FORMAT;
        int64_t count = 1;
        for (int64_t d : t.shape) {
            if (d < 0 || (d > 0 && count > INT64_MAX / d)) return RT_ERR_FORMAT;
            count *= d;
        }
        if (count > INT64_MAX / es || static_cast<uint64_t>(count * es) != t.end - t.begin)
            return RT_ERR_FORMAT;
    }
    return RT_OK;
}

const TensorInfo *find(const rt_st_file *f, const std::string &name) {
    auto it = f->tensors.find(name);
    return it == f->tensors.end() ? nullptr : &it->second;
}

int64_t elements(const TensorInfo &t) {
    int64_t c = 1;
    for (int64_t d : t.shape) c *= d;
    return c;
}

}  // namespace

extern "C" {

rt_status rt_st_open(const char *path, rt_st_file **out) {
    if (!path || !out) return RT_ERR_INVALID_ARG;
    *out = nullptr;
    const int fd = open(path, O_RDONLY);
    if (fd < 0) return RT_ERR_IO;
    struct stat st;
    if (fstat(fd, &st) != 0 || st.st_size < 8) {
        close(fd);
        return st.st_size < 8 ? RT_ERR_FORMAT : RT_ERR_IO;
    }
    void *m = mmap(nullptr, static_cast<size_t>(st.st_size), PROT_READ, MAP_PRIVATE, fd, 0);
    close(fd);
    if (m == MAP_FAILED) return RT_ERR_IO;
    rt_st_file *f = new (std::nothrow) rt_st_file;
    if (!f) {
        munmap(m, static_cast<size_t>(st.st_size));
        return RT_ERR_IO;
    }
    f->map = m;
    f->size = static_cast<size_t>(st.st_size);
    const rt_status s = parse(f);
    if (s != RT_OK) {
        rt_st_close(f);
        return s;
    }
    *out = f;
    return RT_OK;
}

void rt_st_close(rt_st_file *f) {
    if (!f) return;
    if (f->map) munmap(f->map, f->size);
    delete f;
}

int64_t rt_st_count(const rt_st_file *f) {
    return f ? static_cast<int64_t>(f->tensors.size()) : -1;
}

rt_status rt_st_weight_find(const rt_st_file *f, const char *name, rt_st_weight *out) {
    if (!f || !name || !out) return RT_ERR_INVALID_ARG;
    std::memset(out, 0, sizeof *out);
    const TensorInfo *w = find(f, name);
    if (!w) return RT_ERR_NOT_FOUND;
    const std::string base(name);
    if (w->shape.size() != 2 || w->shape[0] < 1 || w->shape[1] < 1)
        return RT_ERR_UNSUPPORTED_SHAPE;
    const int64_t N = w->shape[0], C = w->shape[1];
    const TensorInfo *s = nullptr;
    if (w->dtype == "U8") {
        // q4: codes [N, K/2] + (scale, min) pairs [N, K/32, 2] in fp16
        s = find(f, base + ".q4_scale");
        if (!s) return RT_ERR_NOT_FOUND;
        const int64_t K = 2 * C;
        if (s->dtype != "F16" || K % 32 != 0) return RT_ERR_FORMAT;
        const bool shape_ok = (s->shape.size() == 3 && s->shape[0] == N &&
                               s->shape[1] == K / 32 && s->shape[2] == 2) ||
                              (s->shape.size() == 2 && s->shape[0] == N &&
                               s->shape[1] == K / 16);
        if (!shape_ok) return RT_ERR_FORMAT;
        out->fmt = RT_FMT_Q4;
        out->K = K;
    } else if (w->dtype == "I8") {
        s = find(f, base + ".q_scale");
        if (!s) return RT_ERR_NOT_FOUND;
        if (s->dtype != "F32" || elements(*s) != N ||
            !(s->shape.size() == 1 || (s->shape.size() == 2 && s->shape[1] == 1)))
            return RT_ERR_FORMAT;
        out->fmt = RT_FMT_Q8;
        out->K = C;
    } else if (w->dtype == "F8_E4M3") {
        out->fmt = RT_FMT_E4M3;
        out->K = C;
    } else {
        return RT_ERR_FORMAT;
    }
    out->N = N;
    out->codes = f->data + w->begin;
    out->code_bytes = static_cast<int64_t>(w->end - w->begin);
    if (s) {
        out->scales = f->data + s->begin;
        out->scale_bytes = static_cast<int64_t>(s->end - s->begin);
    }
    return RT_OK;
}

}  // extern "C"

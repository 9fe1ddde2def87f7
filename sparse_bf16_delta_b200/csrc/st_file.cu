// st_file.cu -- the delta file: one delta (offsets, indices, values) as a
// safetensors file, "Shipping a Trillion Parameters With a Hub Bucket: Delta
// Weight Sync in TRL", §4.1 (wire format: per changed parameter an int32
// "{name}.indices" and a bf16 "{name}.values" entry, string metadata sparse /
// model_version / sparsity / changed_params) and §4.3 (the receiver applies
// the parameters that changed_params lists).
//
// Host code only.  The JSON header is built and parsed on the CPU; the data
// never passes through a host-side repack: the writer lays the file out as
// [8-byte length][header][all indices][all values], which is the encode's
// two device arrays as they stand, so a file is two cudaMemcpyAsync from the
// device into the caller's (pinned) buffer.  The reader takes any safetensors
// layout and coalesces the per-parameter ranges that are adjacent in both the
// file and the dws layout into one copy each (two copies for a file this
// writer made).
#include <cuda_runtime.h>

#include <algorithm>
#include <charconv>
#include <clocale>
#include <cstdio>
#include <cstring>
#include <locale.h>
#include <new>
#include <string>
#include <string_view>
#include <unordered_map>
#include <unordered_set>
#include <utility>
#include <vector>

#include "dws_internal.cuh"

namespace {

dws_status_t from_cuda(cudaError_t e) { return e == cudaSuccess ? DWS_OK : DWS_ERR_CUDA; }

// ---- UTF-8 --------------------------------------------------------------

// Strict UTF-8: shortest forms only, no surrogate code points, <= U+10FFFF.
bool valid_utf8(const unsigned char *s, size_t n) {
    size_t i = 0;
    while (i < n) {
        unsigned c = s[i];
        if (c < 0x80) {
            ++i;
            continue;
        }
        int len;
        unsigned cp, least;
        if ((c & 0xE0u) == 0xC0u) {
            len = 2, cp = c & 0x1Fu, least = 0x80;
        } else if ((c & 0xF0u) == 0xE0u) {
            len = 3, cp = c & 0x0Fu, least = 0x800;
        } else if ((c & 0xF8u) == 0xF0u) {
            len = 4, cp = c & 0x07u, least = 0x10000;
        } else {
            return false;
        }
        if (n - i < static_cast<size_t>(len)) return false;
        for (int k = 1; k < len; ++k) {
            unsigned d = s[i + k];
            if ((d & 0xC0u) != 0x80u) return false;
            cp = (cp << 6) | (d & 0x3Fu);
        }
        if (cp < least || cp > 0x10FFFF || (cp >= 0xD800 && cp <= 0xDFFF)) return false;
        i += len;
    }
    return true;
}

// Any code point below 0x110000 as UTF-8; a lone surrogate (which a JSON
// \u escape can name) gets its 3-byte form, which is not valid UTF-8 and so
// never equals a parameter name.
void put_utf8(std::string &out, unsigned cp) {
    if (cp < 0x80) {
        out += static_cast<char>(cp);
    } else if (cp < 0x800) {
        out += static_cast<char>(0xC0 | (cp >> 6));
        out += static_cast<char>(0x80 | (cp & 0x3F));
    } else if (cp < 0x10000) {
        out += static_cast<char>(0xE0 | (cp >> 12));
        out += static_cast<char>(0x80 | ((cp >> 6) & 0x3F));
        out += static_cast<char>(0x80 | (cp & 0x3F));
    } else {
        out += static_cast<char>(0xF0 | (cp >> 18));
        out += static_cast<char>(0x80 | ((cp >> 12) & 0x3F));
        out += static_cast<char>(0x80 | ((cp >> 6) & 0x3F));
        out += static_cast<char>(0x80 | (cp & 0x3F));
    }
}

// ---- JSON writing ---------------------------------------------------------

// A JSON string literal: quote, backslash and the C0 controls escaped (the
// short forms \b \f \n \r \t where JSON has them, else \u00xx), every other
// byte as it is (UTF-8 stays raw).
void put_json_string(std::string &out, std::string_view s) {
    out += '"';
    size_t i = 0;
    while (i < s.size()) {
        // the run of bytes that need no escape goes in at once
        size_t j = i;
        while (j < s.size() && s[j] != '"' && s[j] != '\\' && static_cast<unsigned char>(s[j]) >= 0x20) ++j;
        out.append(s.data() + i, j - i);
        if (j == s.size()) break;
        const unsigned char c = static_cast<unsigned char>(s[j]);
        i = j + 1;
        switch (c) {
        case '"': out += "\\\""; break;
        case '\\': out += "\\\\"; break;
        case '\b': out += "\\b"; break;
        case '\f': out += "\\f"; break;
        case '\n': out += "\\n"; break;
        case '\r': out += "\\r"; break;
        case '\t': out += "\\t"; break;
        default: {  // the other C0 controls
            static const char hex[] = "0123456789abcdef";
            out += "\\u00";
            out += hex[c >> 4];
            out += hex[c & 15];
        }
        }
    }
    out += '"';
}

void put_int(std::string &out, long long v) {
    char buf[24];
    const std::to_chars_result r = std::to_chars(buf, buf + sizeof buf, v);
    out.append(buf, static_cast<size_t>(r.ptr - buf));
}

// x with 6 decimals, '.' as the separator whatever the process locale.
std::string fixed6(double x) {
    static locale_t c_locale = newlocale(LC_ALL_MASK, "C", static_cast<locale_t>(0));
    locale_t prev = c_locale ? uselocale(c_locale) : static_cast<locale_t>(0);
    char buf[64];
    std::snprintf(buf, sizeof buf, "%.6f", x);
    if (c_locale) uselocale(prev);
    return buf;
}

// ---- JSON reading ---------------------------------------------------------

// A parsed JSON document, held flat so that a header of tens of thousands of
// entries costs a few allocations, not one per value: the nodes in one array,
// the children of each array or object as one contiguous run of node indices
// (with the keys of an object's children beside them), every decoded string
// in one arena.
struct JNode {
    enum Kind : unsigned char { kNull, kBool, kNum, kStr, kArr, kObj };
    Kind kind = kNull;
    bool is_count = false;         // kNum: a plain integer >= 0 (or -0) within 64 bits
    unsigned long long count = 0;  // kNum: its value when is_count
    size_t a = 0, n = 0;           // kStr: arena offset and length; kArr/kObj: first child slot, children
};

struct JDoc {
    static constexpr size_t npos = ~size_t(0);
    std::vector<JNode> nodes;
    std::vector<size_t> kids;                          // child node index per slot
    std::vector<std::pair<size_t, size_t>> keys;       // key (arena offset, length) per slot
    std::string arena;

    std::string_view str(size_t node) const {
        return std::string_view(arena.data() + nodes[node].a, nodes[node].n);
    }
    std::string_view key(size_t slot) const {
        return std::string_view(arena.data() + keys[slot].first, keys[slot].second);
    }
    // The value under key k of object `obj` (linear: for the small objects).
    size_t get(size_t obj, std::string_view k) const {
        const JNode &o = nodes[obj];
        for (size_t s = o.a; s < o.a + o.n; ++s)
            if (key(s) == k) return kids[s];
        return npos;
    }
    JNode::Kind kind(size_t node) const { return node == npos ? JNode::kNull : nodes[node].kind; }
};

// Recursive-descent parser of RFC 8259 JSON over [p, e) into a JDoc; no
// extensions (no NaN/Infinity, no comments, no trailing commas), objects with
// a repeated key are refused, nesting deeper than kMaxDepth is refused.
class JsonParser {
  public:
    JsonParser(const char *p, const char *e, JDoc &doc) : p_(p), e_(e), d_(doc) {
        // a first guess from the text's size, capped: a larger document grows
        const size_t bytes = static_cast<size_t>(e - p);
        d_.nodes.reserve(std::min<size_t>(bytes / 16 + 4, size_t(1) << 20));
        d_.arena.reserve(std::min<size_t>(bytes / 2 + 16, size_t(64) << 20));
    }

    bool document(size_t *root) {
        ws();
        if (!value(root, 0)) return false;
        ws();
        return p_ == e_;
    }

  private:
    static constexpr int kMaxDepth = 512;
    const char *p_;
    const char *e_;
    JDoc &d_;
    std::vector<size_t> stack_kids_;                     // children of the open containers
    std::vector<std::pair<size_t, size_t>> stack_keys_;  // and their keys

    void ws() {
        while (p_ < e_ && (*p_ == ' ' || *p_ == '\t' || *p_ == '\n' || *p_ == '\r')) ++p_;
    }

    bool word(const char *w) {
        size_t n = std::strlen(w);
        if (static_cast<size_t>(e_ - p_) < n || std::memcmp(p_, w, n) != 0) return false;
        p_ += n;
        return true;
    }

    size_t add(JNode::Kind k) {
        JNode nd;
        nd.kind = k;
        d_.nodes.push_back(nd);
        return d_.nodes.size() - 1;
    }

    bool value(size_t *out, int depth) {
        if (depth > kMaxDepth || p_ >= e_) return false;
        switch (*p_) {
        case '{': return container(out, depth, true);
        case '[': return container(out, depth, false);
        case '"': {
            size_t off = 0, len = 0;
            if (!string(&off, &len)) return false;
            *out = add(JNode::kStr);
            d_.nodes[*out].a = off;
            d_.nodes[*out].n = len;
            return true;
        }
        case 't': *out = add(JNode::kBool); return word("true");
        case 'f': *out = add(JNode::kBool); return word("false");
        case 'n': *out = add(JNode::kNull); return word("null");
        default: *out = add(JNode::kNum); return number(&d_.nodes[*out]);
        }
    }

    // An object (with keys) or an array: children collected on the stack,
    // then moved to one run of slots when the container closes.
    bool container(size_t *out, int depth, bool is_obj) {
        const size_t node = add(is_obj ? JNode::kObj : JNode::kArr);
        *out = node;
        const size_t base = stack_kids_.size();
        const char close = is_obj ? '}' : ']';
        ++p_;
        ws();
        if (p_ < e_ && *p_ == close) {
            ++p_;
        } else {
            for (;;) {
                ws();
                std::pair<size_t, size_t> k(0, 0);
                if (is_obj) {
                    if (p_ >= e_ || *p_ != '"') return false;
                    if (!string(&k.first, &k.second)) return false;
                    ws();
                    if (p_ >= e_ || *p_ != ':') return false;
                    ++p_;
                    ws();
                }
                size_t child = 0;
                if (!value(&child, depth + 1)) return false;
                stack_kids_.push_back(child);
                stack_keys_.push_back(k);
                ws();
                if (p_ >= e_) return false;
                if (*p_ == ',') {
                    ++p_;
                    continue;
                }
                if (*p_ != close) return false;
                ++p_;
                break;
            }
        }
        const size_t n = stack_kids_.size() - base;
        d_.nodes[node].a = d_.kids.size();
        d_.nodes[node].n = n;
        d_.kids.insert(d_.kids.end(), stack_kids_.begin() + base, stack_kids_.end());
        d_.keys.insert(d_.keys.end(), stack_keys_.begin() + base, stack_keys_.end());
        stack_kids_.resize(base);
        stack_keys_.resize(base);
        if (!is_obj || n < 2) return true;
        // no key twice (the arena is not growing while this runs)
        const size_t first = d_.nodes[node].a;
        if (n <= 16) {
            for (size_t i = first; i < first + n; ++i)
                for (size_t j = i + 1; j < first + n; ++j)
                    if (d_.key(i) == d_.key(j)) return false;
            return true;
        }
        std::unordered_set<std::string_view> seen;
        seen.reserve(n);
        for (size_t i = first; i < first + n; ++i)
            if (!seen.insert(d_.key(i)).second) return false;
        return true;
    }

    bool hex4(unsigned &cp) {
        if (e_ - p_ < 4) return false;
        cp = 0;
        for (int k = 0; k < 4; ++k) {
            char c = *p_++;
            unsigned d;
            if (c >= '0' && c <= '9') d = c - '0';
            else if (c >= 'a' && c <= 'f') d = c - 'a' + 10;
            else if (c >= 'A' && c <= 'F') d = c - 'A' + 10;
            else return false;
            cp = (cp << 4) | d;
        }
        return true;
    }

    // A string literal, decoded into the arena at [*off, *off + *len).
    bool string(size_t *off, size_t *len) {
        std::string &out = d_.arena;
        *off = out.size();
        ++p_;  // the opening quote
        for (;;) {
            // the run of plain bytes up to the next quote, escape or control
            const char *q = p_;
            while (q < e_ && *q != '"' && *q != '\\' && static_cast<unsigned char>(*q) >= 0x20) ++q;
            out.append(p_, static_cast<size_t>(q - p_));
            p_ = q;
            if (p_ >= e_) return false;
            unsigned char c = static_cast<unsigned char>(*p_++);
            if (c == '"') {
                *len = out.size() - *off;
                return true;
            }
            if (c < 0x20) return false;
            // c == '\\'
            if (p_ >= e_) return false;
            switch (*p_++) {
            case '"': out += '"'; break;
            case '\\': out += '\\'; break;
            case '/': out += '/'; break;
            case 'b': out += '\b'; break;
            case 'f': out += '\f'; break;
            case 'n': out += '\n'; break;
            case 'r': out += '\r'; break;
            case 't': out += '\t'; break;
            case 'u': {
                unsigned cp;
                if (!hex4(cp)) return false;
                // A high surrogate followed by an escaped low one is one
                // code point; otherwise each escape stands alone.
                if (cp >= 0xD800 && cp < 0xDC00 && e_ - p_ >= 2 && p_[0] == '\\' && p_[1] == 'u') {
                    const char *back = p_;
                    p_ += 2;
                    unsigned lo;
                    if (!hex4(lo)) return false;
                    if (lo >= 0xDC00 && lo < 0xE000)
                        cp = 0x10000 + ((cp - 0xD800) << 10) + (lo - 0xDC00);
                    else
                        p_ = back;
                }
                put_utf8(out, cp);
                break;
            }
            default: return false;
            }
        }
    }

    static bool digit(char c) { return c >= '0' && c <= '9'; }

    bool number(JNode *v) {
        bool neg = false, plain = true, fits = true;
        unsigned long long u = 0;
        if (p_ < e_ && *p_ == '-') {
            neg = true;
            ++p_;
        }
        if (p_ >= e_ || !digit(*p_)) return false;
        if (*p_ == '0') {
            ++p_;
        } else {
            while (p_ < e_ && digit(*p_)) {
                unsigned d = *p_++ - '0';
                if (u > (~0ull - d) / 10) fits = false;
                u = u * 10 + d;
            }
        }
        if (p_ < e_ && *p_ == '.') {
            plain = false;
            ++p_;
            if (p_ >= e_ || !digit(*p_)) return false;
            while (p_ < e_ && digit(*p_)) ++p_;
        }
        if (p_ < e_ && (*p_ == 'e' || *p_ == 'E')) {
            plain = false;
            ++p_;
            if (p_ < e_ && (*p_ == '+' || *p_ == '-')) ++p_;
            if (p_ >= e_ || !digit(*p_)) return false;
            while (p_ < e_ && digit(*p_)) ++p_;
        }
        v->is_count = plain && fits && (!neg || u == 0);
        v->count = v->is_count ? u : 0;
        return true;
    }
};

// A decimal integer string ("-"? digits) that fits in 64 bits.
bool parse_version(std::string_view s, long long *out) {
    size_t i = 0;
    bool neg = false;
    if (i < s.size() && s[i] == '-') neg = true, ++i;
    if (i == s.size()) return false;
    unsigned long long u = 0, limit = neg ? (1ull << 63) : (1ull << 63) - 1;
    for (; i < s.size(); ++i) {
        if (s[i] < '0' || s[i] > '9') return false;
        unsigned d = s[i] - '0';
        if (u > (limit - d) / 10) return false;
        u = u * 10 + d;
    }
    *out = neg ? static_cast<long long>(0ull - u) : static_cast<long long>(u);
    return true;
}

bool ends_with(std::string_view s, std::string_view tail) {
    return s.size() >= tail.size() && s.compare(s.size() - tail.size(), tail.size(), tail) == 0;
}

// Checks the table's names: present, valid UTF-8, pairwise distinct.
dws_status_t check_names(const char *const *names, int32_t T,
                         std::vector<std::string_view> *views) {
    if (names == nullptr && T > 0) return DWS_ERR_INVALID;
    views->resize(T);
    std::unordered_set<std::string_view> seen;
    seen.reserve(T);
    for (int32_t t = 0; t < T; ++t) {
        if (names[t] == nullptr) return DWS_ERR_INVALID;
        std::string_view n(names[t]);
        if (!valid_utf8(reinterpret_cast<const unsigned char *>(n.data()), n.size()))
            return DWS_ERR_INVALID;
        if (!seen.insert(n).second) return DWS_ERR_INVALID;
        (*views)[t] = n;
    }
    return DWS_OK;
}

// One tensor entry {"dtype": dtype, "shape": [n], "data_offsets": [a, b]}
// whose range lies in the data and holds n elements of elem bytes.
bool tensor_entry(const JDoc &doc, size_t e, const char *dtype, unsigned long long elem,
                  unsigned long long data_bytes, unsigned long long *n,
                  unsigned long long *begin) {
    if (doc.kind(e) != JNode::kObj) return false;
    const size_t dt = doc.get(e, "dtype");
    const size_t shape = doc.get(e, "shape");
    const size_t span = doc.get(e, "data_offsets");
    if (doc.kind(dt) != JNode::kStr || doc.str(dt) != dtype) return false;
    if (doc.kind(shape) != JNode::kArr || doc.nodes[shape].n != 1) return false;
    if (doc.kind(span) != JNode::kArr || doc.nodes[span].n != 2) return false;
    const JNode &c0 = doc.nodes[doc.kids[doc.nodes[shape].a]];
    const JNode &a0 = doc.nodes[doc.kids[doc.nodes[span].a]];
    const JNode &b0 = doc.nodes[doc.kids[doc.nodes[span].a + 1]];
    if (c0.kind != JNode::kNum || !c0.is_count || a0.kind != JNode::kNum || !a0.is_count ||
        b0.kind != JNode::kNum || !b0.is_count)
        return false;
    const unsigned long long a = a0.count, b = b0.count, c = c0.count;
    if (a > b || b > data_bytes) return false;
    if (c > (b - a) / elem || c * elem != b - a) return false;
    *n = c;
    *begin = a;
    return true;
}

// The 8-byte length and the padded JSON header of the delta file of
// (offsets, names); *nnz receives offsets[T].
dws_status_t build_header(const dws_plan_t *plan, const char *const *names,
                          const int64_t *offsets, int64_t model_version, std::string *out,
                          long long *nnz_out) {
    int32_t T = 0;
    const long long *numel = nullptr;
    if (!dws::plan_numels(plan, &T, &numel) || offsets == nullptr) return DWS_ERR_INVALID;
    std::vector<std::string_view> name;
    dws_status_t st = check_names(names, T, &name);
    if (st != DWS_OK) return st;
    if (offsets[0] != 0) return DWS_ERR_BAD_DELTA;
    long long total = 0;
    for (int32_t t = 0; t < T; ++t) {
        long long c = offsets[t + 1] - offsets[t];
        if (offsets[t + 1] < offsets[t] || c > numel[t]) return DWS_ERR_BAD_DELTA;
        total += numel[t];
    }
    const long long nnz = offsets[T];

    size_t name_bytes = 0;
    for (int32_t t = 0; t < T; ++t) name_bytes += name[t].size();
    std::string changed = "[";
    changed.reserve(name_bytes + 3 * static_cast<size_t>(T) + 2);
    for (int32_t t = 0; t < T; ++t) {
        if (offsets[t + 1] == offsets[t]) continue;
        if (changed.size() > 1) changed += ',';
        put_json_string(changed, name[t]);
    }
    changed += ']';

    std::string h(8, '\0');
    h.reserve(256 + 2 * changed.size() + 2 * name_bytes + 160 * static_cast<size_t>(T));
    h += "{\"__metadata__\":{\"sparse\":\"True\",\"model_version\":\"";
    put_int(h, model_version);
    h += "\",\"sparsity\":\"";
    h += fixed6(total > 0 ? 1.0 - static_cast<double>(nnz) / static_cast<double>(total) : 1.0);
    h += "\",\"changed_params\":";
    put_json_string(h, changed);
    h += '}';
    std::string key;
    for (int32_t t = 0; t < T; ++t) {
        const long long a = offsets[t], b = offsets[t + 1];
        if (a == b) continue;
        key.assign(name[t]);
        key += ".indices";
        h += ',';
        put_json_string(h, key);
        h += ":{\"dtype\":\"I32\",\"shape\":[";
        put_int(h, b - a);
        h += "],\"data_offsets\":[";
        put_int(h, 4 * a);
        h += ',';
        put_int(h, 4 * b);
        h += "]}";
        key.assign(name[t]);
        key += ".values";
        h += ',';
        put_json_string(h, key);
        h += ":{\"dtype\":\"BF16\",\"shape\":[";
        put_int(h, b - a);
        h += "],\"data_offsets\":[";
        put_int(h, 4 * nnz + 2 * a);
        h += ',';
        put_int(h, 4 * nnz + 2 * b);
        h += "]}";
    }
    h += '}';
    h.append((8 - h.size() % 8) % 8, ' ');
    const unsigned long long json_bytes = h.size() - 8;
    for (int k = 0; k < 8; ++k) h[k] = static_cast<char>((json_bytes >> (8 * k)) & 0xFF);
    *out = std::move(h);
    *nnz_out = nnz;
    return DWS_OK;
}

dws_status_t st_delta_header(const dws_plan_t *plan, const char *const *names,
                             const int64_t *offsets, int64_t model_version, uint8_t *out,
                             int64_t capacity, int64_t *header_bytes) {
    if (header_bytes == nullptr || capacity < 0) return DWS_ERR_INVALID;
    std::string h;
    long long nnz = 0;
    dws_status_t st = build_header(plan, names, offsets, model_version, &h, &nnz);
    if (st != DWS_OK) return st;
    *header_bytes = static_cast<int64_t>(h.size());
    if (out == nullptr) return DWS_OK;
    if (capacity < static_cast<int64_t>(h.size())) return DWS_ERR_CAPACITY;
    std::memcpy(out, h.data(), h.size());
    return DWS_OK;
}

dws_status_t st_delta_write(const dws_plan_t *plan, const char *const *names,
                            const int64_t *offsets, int64_t model_version,
                            const int32_t *indices, const uint16_t *values, uint8_t *file,
                            int64_t capacity, int64_t *file_bytes, dws_stream_t stream) {
    if (file_bytes == nullptr || capacity < 0) return DWS_ERR_INVALID;
    std::string h;
    long long nnz = 0;
    dws_status_t st = build_header(plan, names, offsets, model_version, &h, &nnz);
    if (st != DWS_OK) return st;
    const long long need = static_cast<long long>(h.size()) + 6 * nnz;
    *file_bytes = need;
    if (file == nullptr) return DWS_OK;
    if (nnz > 0 && (indices == nullptr || values == nullptr)) return DWS_ERR_INVALID;
    if (capacity < need) return DWS_ERR_CAPACITY;
    std::memcpy(file, h.data(), h.size());
    if (nnz == 0) return DWS_OK;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    uint8_t *body = file + h.size();
    cudaError_t e = cudaMemcpyAsync(body, indices, 4 * nnz, cudaMemcpyDefault, s);
    if (e == cudaSuccess) e = cudaMemcpyAsync(body + 4 * nnz, values, 2 * nnz, cudaMemcpyDefault, s);
    return from_cuda(e);
}

dws_status_t st_delta_read(const dws_plan_t *plan, const char *const *names,
                           const uint8_t *file, int64_t file_size, int64_t *offsets_host,
                           int64_t *offsets, int32_t *indices, uint16_t *values,
                           int64_t capacity, int64_t *nnz_out, int64_t *model_version,
                           dws_stream_t stream) {
    int32_t T = 0;
    const long long *numel = nullptr;
    if (!dws::plan_numels(plan, &T, &numel) || offsets_host == nullptr || offsets == nullptr ||
        nnz_out == nullptr || capacity < 0 || file_size < 0 || (file == nullptr && file_size > 0))
        return DWS_ERR_INVALID;
    std::vector<std::string_view> name;
    dws_status_t st = check_names(names, T, &name);
    if (st != DWS_OK) return st;

    // The container: length prefix, UTF-8 JSON header, data.
    if (file_size < 8) return DWS_ERR_BAD_DELTA;
    unsigned long long hl = 0;
    for (int k = 0; k < 8; ++k) hl |= static_cast<unsigned long long>(file[k]) << (8 * k);
    if (hl > static_cast<unsigned long long>(file_size - 8)) return DWS_ERR_BAD_DELTA;
    const char *hdr = reinterpret_cast<const char *>(file + 8);
    if (!valid_utf8(file + 8, hl)) return DWS_ERR_BAD_DELTA;
    JDoc doc;
    size_t root = 0;
    if (!JsonParser(hdr, hdr + hl, doc).document(&root) || doc.kind(root) != JNode::kObj)
        return DWS_ERR_BAD_DELTA;
    const uint8_t *data = file + 8 + hl;
    const unsigned long long data_bytes = static_cast<unsigned long long>(file_size - 8) - hl;

    // Metadata: a delta (sparse "True"), its version, the list it applies.
    const size_t meta = doc.get(root, "__metadata__");
    if (doc.kind(meta) != JNode::kObj) return DWS_ERR_BAD_DELTA;
    const size_t sparse = doc.get(meta, "sparse");
    const size_t ver = doc.get(meta, "model_version");
    const size_t listed = doc.get(meta, "changed_params");
    if (doc.kind(sparse) != JNode::kStr || doc.str(sparse) != "True") return DWS_ERR_BAD_DELTA;
    long long version = 0;
    if (doc.kind(ver) != JNode::kStr || !parse_version(doc.str(ver), &version))
        return DWS_ERR_BAD_DELTA;
    if (doc.kind(listed) != JNode::kStr) return DWS_ERR_BAD_DELTA;
    const std::string_view listed_text = doc.str(listed);
    JDoc ldoc;
    size_t lroot = 0;
    if (!JsonParser(listed_text.data(), listed_text.data() + listed_text.size(), ldoc).document(&lroot) ||
        ldoc.kind(lroot) != JNode::kArr)
        return DWS_ERR_BAD_DELTA;
    std::unordered_map<std::string_view, int32_t> slot;
    slot.reserve(T);
    for (int32_t t = 0; t < T; ++t) slot.emplace(name[t], t);
    const JNode &lnode = ldoc.nodes[lroot];
    std::vector<std::string_view> list;  // the listed names, in their order
    list.reserve(lnode.n);
    std::unordered_set<std::string_view> changed;
    changed.reserve(lnode.n);
    for (size_t s = lnode.a; s < lnode.a + lnode.n; ++s) {
        const size_t c = ldoc.kids[s];
        if (ldoc.kind(c) != JNode::kStr) return DWS_ERR_BAD_DELTA;
        const std::string_view n = ldoc.str(c);
        if (!changed.insert(n).second) return DWS_ERR_BAD_DELTA;
        if (slot.find(n) == slot.end()) return DWS_ERR_BAD_DELTA;
        list.push_back(n);
    }

    // Every tensor entry belongs to a listed parameter.
    const JNode &rnode = doc.nodes[root];
    std::unordered_map<std::string_view, size_t> entry;
    entry.reserve(rnode.n);
    for (size_t s = rnode.a; s < rnode.a + rnode.n; ++s) {
        const std::string_view k = doc.key(s);
        if (k == "__metadata__") continue;
        std::string_view base;
        if (ends_with(k, ".indices")) base = k.substr(0, k.size() - 8);
        else if (ends_with(k, ".values")) base = k.substr(0, k.size() - 7);
        else return DWS_ERR_BAD_DELTA;
        if (changed.find(base) == changed.end()) return DWS_ERR_BAD_DELTA;
        entry.emplace(k, doc.kids[s]);
    }

    // Each listed parameter: its two entries, equal lengths.
    struct Part { unsigned long long n = 0, ib = 0, vb = 0; bool present = false; };
    std::vector<Part> part(T);
    std::string key;
    for (const std::string_view n : list) {
        const int32_t t = slot.find(n)->second;
        Part &p = part[t];
        unsigned long long nv = 0;
        key.assign(n);
        key += ".indices";
        auto it = entry.find(key);
        if (it == entry.end() || !tensor_entry(doc, it->second, "I32", 4, data_bytes, &p.n, &p.ib))
            return DWS_ERR_BAD_DELTA;
        key.assign(n);
        key += ".values";
        it = entry.find(key);
        if (it == entry.end() || !tensor_entry(doc, it->second, "BF16", 2, data_bytes, &nv, &p.vb))
            return DWS_ERR_BAD_DELTA;
        if (nv != p.n) return DWS_ERR_BAD_DELTA;
        // each changed element at most once: no more entries than elements
        // (the writer's bound as well)
        if (p.n > static_cast<unsigned long long>(numel[t])) return DWS_ERR_BAD_DELTA;
        p.present = true;
    }

    offsets_host[0] = 0;
    for (int32_t t = 0; t < T; ++t)
        offsets_host[t + 1] = offsets_host[t] + static_cast<long long>(part[t].n);
    const long long nnz = offsets_host[T];
    *nnz_out = nnz;
    if (model_version != nullptr) *model_version = version;
    if (nnz > capacity) return DWS_ERR_CAPACITY;
    if (nnz > 0 && (indices == nullptr || values == nullptr)) return DWS_ERR_INVALID;

    // Copies: the dws layout is contiguous in table order; a run of tensors
    // whose file ranges follow one another is one copy.
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    cudaError_t e = cudaMemcpyAsync(offsets, offsets_host, 8 * (static_cast<size_t>(T) + 1),
                                    cudaMemcpyDefault, s);
    for (int pass = 0; pass < 2 && e == cudaSuccess; ++pass) {
        const size_t elem = pass == 0 ? 4 : 2;
        uint8_t *dst = pass == 0 ? reinterpret_cast<uint8_t *>(indices)
                                 : reinterpret_cast<uint8_t *>(values);
        long long run_dst = 0;
        unsigned long long run_src = 0, run_len = 0;
        for (int32_t t = 0; t <= T && e == cudaSuccess; ++t) {
            const bool last = t == T;
            unsigned long long src = 0, len = 0;
            if (!last) {
                if (part[t].n == 0) continue;
                src = pass == 0 ? part[t].ib : part[t].vb;
                len = part[t].n * elem;
                if (run_len > 0 && src == run_src + run_len) {
                    run_len += len;
                    continue;
                }
            }
            if (run_len > 0)
                e = cudaMemcpyAsync(dst + run_dst * elem, data + run_src, run_len,
                                    cudaMemcpyDefault, s);
            if (!last) {
                run_dst = offsets_host[t];
                run_src = src;
                run_len = len;
            }
        }
    }
    return from_cuda(e);
}

}  // namespace

// The exported entry points: a host allocation that fails (a header larger
// than the memory at hand) is reported as DWS_ERR_INVALID instead of an
// exception crossing the C boundary.
extern "C" {

dws_status_t dws_st_delta_header(const dws_plan_t *plan, const char *const *names,
                                 const int64_t *offsets, int64_t model_version, uint8_t *out,
                                 int64_t capacity, int64_t *header_bytes) {
    try {
        return st_delta_header(plan, names, offsets, model_version, out, capacity, header_bytes);
    } catch (const std::bad_alloc &) {
        return DWS_ERR_INVALID;
    }
}

dws_status_t dws_st_delta_write(const dws_plan_t *plan, const char *const *names,
                                const int64_t *offsets, int64_t model_version,
                                const int32_t *indices, const uint16_t *values, uint8_t *file,
                                int64_t capacity, int64_t *file_bytes, dws_stream_t stream) {
    try {
        return st_delta_write(plan, names, offsets, model_version, indices, values, file, capacity,
                              file_bytes, stream);
    } catch (const std::bad_alloc &) {
        return DWS_ERR_INVALID;
    }
}

dws_status_t dws_st_delta_read(const dws_plan_t *plan, const char *const *names,
                               const uint8_t *file, int64_t file_size, int64_t *offsets_host,
                               int64_t *offsets, int32_t *indices, uint16_t *values,
                               int64_t capacity, int64_t *nnz_out, int64_t *model_version,
                               dws_stream_t stream) {
    try {
        return st_delta_read(plan, names, file, file_size, offsets_host, offsets, indices, values,
                             capacity, nnz_out, model_version, stream);
    } catch (const std::bad_alloc &) {
        return DWS_ERR_INVALID;
    }
}

}  // extern "C"

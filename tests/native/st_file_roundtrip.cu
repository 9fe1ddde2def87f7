// Round trip of the delta file through libdws's host code with the copies
// made real on the CPU: this file supplies cudaMemcpyAsync as a plain memcpy
// (host buffers only) and the plan's element counts, and is linked with
// csrc/st_file.cu alone (no CUDA runtime) by tests/test_st_file_fuzz.py.
// For random deltas it writes the file with dws_st_delta_write and reads it
// back with dws_st_delta_read, and it reads files laid out per parameter in a
// shuffled order (every parameter's data its own range, as a library writer
// would place it), checking offsets, indices and values exactly.  Exits
// non-zero on the first mismatch.  Built with the host compiler alone, so the
// stub below is declared with the C types the runtime's symbol has.
#include <algorithm>
#include <cstdint>
#include <cstdio>
#include <cstring>
#include <random>
#include <string>
#include <vector>

#include "dws.h"

extern "C" int cudaMemcpyAsync(void *dst, const void *src, size_t count, int /*kind*/,
                               void * /*stream*/) {
    std::memmove(dst, src, count);
    return 0;  // cudaSuccess
}

// nvcc registers each file's (here empty) device image at start-up; without the
// CUDA runtime those calls land in these no-ops.
extern "C" void **__cudaRegisterFatBinary(void *) {
    static void *handle = nullptr;
    return &handle;
}
extern "C" void __cudaRegisterFatBinaryEnd(void **) {}
extern "C" void __cudaUnregisterFatBinary(void **) {}

namespace dws {
static std::vector<long long> g_numel;
bool plan_numels(const dws_plan_t *plan, int32_t *T, const long long **numels) {
    if (plan == nullptr) return false;
    *T = static_cast<int32_t>(g_numel.size());
    *numels = g_numel.data();
    return true;
}
}  // namespace dws

namespace {

int fail(const char *what, int it) {
    std::printf("FAIL %s at case %d\n", what, it);
    return 1;
}

std::string jstr(const std::string &s) {  // names here hold no character that needs escaping
    return "\"" + s + "\"";
}

}  // namespace

int main(int argc, char **argv) {
    std::mt19937_64 rng(argc > 1 ? std::strtoull(argv[1], nullptr, 10) : 1);
    const dws_plan_t *plan = reinterpret_cast<const dws_plan_t *>(0x1);
    int checked = 0;
    for (int it = 0; it < 300; ++it) {
        const int T = 1 + static_cast<int>(rng() % 40);
        dws::g_numel.assign(T, 0);
        std::vector<std::string> names(T);
        std::vector<const char *> np(T);
        std::vector<int64_t> off(T + 1, 0);
        std::vector<int32_t> idx;
        std::vector<uint16_t> val;
        for (int t = 0; t < T; ++t) {
            const long long n = static_cast<long long>(rng() % 5000);
            dws::g_numel[t] = n;
            names[t] = "layer." + std::to_string(t) + (rng() % 3 ? ".weight" : ".bias");
            np[t] = names[t].c_str();
            const long long c = (n > 0 && rng() % 3) ? static_cast<long long>(rng() % (n + 1)) : 0;
            std::vector<int32_t> pick;
            for (long long i = 0; i < n && static_cast<long long>(pick.size()) < c; ++i)
                if (static_cast<long long>(rng() % n) < c) pick.push_back(static_cast<int32_t>(i));
            for (int32_t i : pick) {
                idx.push_back(i);
                val.push_back(static_cast<uint16_t>(rng()));
            }
            off[t + 1] = off[t] + static_cast<int64_t>(pick.size());
        }
        const int64_t nnz = off[T];
        const int64_t version = static_cast<int64_t>(rng() % 100000) - 50000;

        // 1. this writer's layout, both directions through libdws
        int64_t fbytes = 0;
        if (dws_st_delta_write(plan, np.data(), off.data(), version, idx.data(), val.data(), nullptr,
                               0, &fbytes, nullptr) != DWS_OK)
            return fail("size query", it);
        std::vector<uint8_t> file(static_cast<size_t>(fbytes));
        if (dws_st_delta_write(plan, np.data(), off.data(), version, idx.data(), val.data(),
                               file.data(), fbytes, &fbytes, nullptr) != DWS_OK)
            return fail("write", it);
        for (int layout = 0; layout < 2; ++layout) {
            if (layout == 1) {
                // 2. per-parameter ranges in a shuffled order, keys shuffled too
                std::vector<int> order;
                for (int t = 0; t < T; ++t)
                    if (off[t + 1] > off[t]) order.push_back(t);
                std::shuffle(order.begin(), order.end(), rng);
                std::vector<uint8_t> data;
                std::vector<std::string> ents;
                std::string changed = "[";
                for (int t = 0; t < T; ++t)
                    if (off[t + 1] > off[t]) changed += (changed.size() > 1 ? "," : "") + std::string("\\\"") + names[t] + "\\\"";
                changed += "]";
                for (int t : order) {
                    const int64_t n = off[t + 1] - off[t];
                    const size_t a = data.size();
                    data.insert(data.end(), reinterpret_cast<const uint8_t *>(val.data() + off[t]),
                                reinterpret_cast<const uint8_t *>(val.data() + off[t + 1]));
                    ents.push_back(jstr(names[t] + ".values") + ":{\"dtype\":\"BF16\",\"shape\":[" +
                                   std::to_string(n) + "],\"data_offsets\":[" + std::to_string(a) + "," +
                                   std::to_string(data.size()) + "]}");
                    const size_t b = data.size();
                    data.insert(data.end(), reinterpret_cast<const uint8_t *>(idx.data() + off[t]),
                                reinterpret_cast<const uint8_t *>(idx.data() + off[t + 1]));
                    ents.push_back(jstr(names[t] + ".indices") + ":{\"dtype\":\"I32\",\"shape\":[" +
                                   std::to_string(n) + "],\"data_offsets\":[" + std::to_string(b) + "," +
                                   std::to_string(data.size()) + "]}");
                }
                std::shuffle(ents.begin(), ents.end(), rng);
                std::string h = "{";
                for (const std::string &e : ents) h += e + ",";
                h += "\"__metadata__\":{\"changed_params\":\"" + changed + "\",\"model_version\":\"" +
                     std::to_string(version) + "\",\"sparse\":\"True\"}}";
                file.assign(8, 0);
                for (int k = 0; k < 8; ++k) file[k] = static_cast<uint8_t>(static_cast<uint64_t>(h.size()) >> (8 * k));
                file.insert(file.end(), h.begin(), h.end());
                file.insert(file.end(), data.begin(), data.end());
            }
            std::vector<int64_t> oh(T + 1, -1), od(T + 1, -1);
            std::vector<int32_t> ri(static_cast<size_t>(nnz) + 1, -1);
            std::vector<uint16_t> rv(static_cast<size_t>(nnz) + 1, 0xffff);
            int64_t got = -1, ver = 0;
            const dws_status_t st = dws_st_delta_read(plan, np.data(), file.data(),
                                                      static_cast<int64_t>(file.size()), oh.data(),
                                                      od.data(), ri.data(), rv.data(), nnz, &got, &ver,
                                                      nullptr);
            if (st != DWS_OK) return fail(layout ? "read (shuffled)" : "read", it);
            if (got != nnz || ver != version) return fail("nnz or version", it);
            if (oh != off || od != off) return fail("offsets", it);
            if (!std::equal(idx.begin(), idx.end(), ri.begin()) || ri[nnz] != -1)
                return fail("indices", it);
            if (!std::equal(val.begin(), val.end(), rv.begin()) || rv[nnz] != 0xffff)
                return fail("values", it);
            ++checked;
        }
    }
    std::printf("round trips %d\n", checked);
    return 0;
}

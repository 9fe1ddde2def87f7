// Memory-safety fuzz of the delta-file host code (csrc/st_file.cu), built with
// AddressSanitizer and UndefinedBehaviorSanitizer by tests/test_st_file_fuzz.py.
// Seeds are delta files written by dws_st_delta_header over a 4-tensor table;
// each iteration flips, inserts or deletes header bytes (or the length prefix,
// or truncates) and parses the result with dws_st_delta_read at capacity 0,
// whose only possible copy is the offsets array into host memory.  No device
// memory is touched.  Every call must return a status; deep nesting must be
// refused.  The plan is a stand-in: plan_numels below answers for any non-null
// plan pointer.
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <string>
#include <vector>
#include <random>
#include "dws.h"
namespace dws {
static long long g_numel[4] = {5, 3, 70000, 1};
bool plan_numels(const dws_plan_t *plan, int32_t *T, const long long **numels) {
    if (!plan) return false;
    *T = 4; *numels = g_numel; return true;
}
}
int main(int argc, char **argv) {
    const char *names[4] = {"w", "a\"b", "\xc3\xbc", "x.y"};
    const dws_plan_t *plan = reinterpret_cast<const dws_plan_t *>(0x1);
    std::vector<std::vector<uint8_t>> seeds;
    std::mt19937_64 rng(argc > 1 ? atoi(argv[1]) : 1);
    for (int s = 0; s < 6; ++s) {
        int64_t off[5] = {0, 0, 0, 0, 0};
        for (int t = 0; t < 4; ++t) off[t + 1] = off[t] + (int64_t)(rng() % (dws::g_numel[t] < 2 ? dws::g_numel[t] + 1 : 3));
        int64_t hb = 0;
        if (dws_st_delta_header(plan, names, off, (int64_t)rng() % 1000, nullptr, 0, &hb) != DWS_OK) return 2;
        std::vector<uint8_t> f(hb + 6 * off[4]);
        if (dws_st_delta_header(plan, names, off, 7, f.data(), hb, &hb) != DWS_OK) return 3;
        for (size_t i = hb; i < f.size(); ++i) f[i] = (uint8_t)rng();
        seeds.push_back(f);
    }
    const char alphabet[] = "{}[]\":,\\0123456789-.eEtfnrulas \t\n\x80\xc3\xbc\xff";
    long accepted = 0, refused = 0, other = 0;
    std::vector<int64_t> oh(5), sink(5);
    const long iters = argc > 2 ? atol(argv[2]) : 300000;
    for (long it = 0; it < iters; ++it) {
        std::vector<uint8_t> f = seeds[rng() % seeds.size()];
        int nm = 1 + (int)(rng() % 4);
        for (int m = 0; m < nm && f.size() > 8; ++m) {
            size_t pos = 8 + rng() % (f.size() - 8);
            int r = (int)(rng() % 10);
            if (r < 6) f[pos] = (uint8_t)alphabet[rng() % (sizeof(alphabet) - 1)];
            else if (r < 8) f.insert(f.begin() + pos, (uint8_t)alphabet[rng() % (sizeof(alphabet) - 1)]);
            else f.erase(f.begin() + pos);
        }
        if (rng() % 8 == 0) {  // a random length prefix
            uint64_t hl = rng() % (f.size() + 16);
            for (int k = 0; k < 8; ++k) f[k] = (uint8_t)(hl >> (8 * k));
        }
        if (rng() % 50 == 0) f.resize(rng() % (f.size() + 1));
        int64_t nnz = -1, ver = 0;
        dws_status_t st = dws_st_delta_read(plan, names, f.empty() ? nullptr : f.data(), (int64_t)f.size(),
                                            oh.data(), sink.data(), nullptr, nullptr, 0, &nnz, &ver, nullptr);
        if (st == DWS_ERR_BAD_DELTA) ++refused;
        else if (st == DWS_ERR_CAPACITY || st == DWS_OK || st == DWS_ERR_CUDA) ++accepted;
        else ++other;
    }
    // deep nesting and long strings
    std::string deep = "{\"__metadata__\":{\"sparse\":\"True\",\"model_version\":\"1\",\"changed_params\":\"[]\",\"d\":";
    for (int i = 0; i < 100000; ++i) deep += "[";
    std::vector<uint8_t> f(8 + deep.size());
    for (int k = 0; k < 8; ++k) f[k] = (uint8_t)((uint64_t)deep.size() >> (8 * k));
    memcpy(f.data() + 8, deep.data(), deep.size());
    int64_t nnz = 0;
    dws_status_t st = dws_st_delta_read(plan, names, f.data(), (int64_t)f.size(), oh.data(), sink.data(),
                                        nullptr, nullptr, 0, &nnz, nullptr, nullptr);
    printf("accepted %ld refused %ld other %ld deep %d\n", accepted, refused, other, (int)st);
    return other == 0 && st == DWS_ERR_BAD_DELTA ? 0 : 1;
}

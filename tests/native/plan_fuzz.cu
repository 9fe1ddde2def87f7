// Memory-safety and consistency fuzz of libdws's host code for plans and
// argument checks (csrc/dws_abi.cu), built with AddressSanitizer and
// UndefinedBehaviorSanitizer by tests/test_host_fuzz.py together with every
// other source of the library.  Only calls that return before any CUDA call
// are made: plan creation and queries, the delta-file header, and entry points
// given arguments that the host refuses (no workspace, a misaligned or short
// one, negative sizes).  Exits non-zero on the first inconsistency.
#include <cstdint>
#include <cstdio>
#include <cstdlib>
#include <random>
#include <string>
#include <vector>

#include "dws.h"

namespace {

int fail(const char *what, long it) {
    std::printf("FAIL %s at iteration %ld\n", what, it);
    return 1;
}

}  // namespace

int main(int argc, char **argv) {
    std::mt19937_64 rng(argc > 1 ? std::strtoull(argv[1], nullptr, 10) : 1);
    const long iters = argc > 2 ? std::atol(argv[2]) : 2000;
    const int64_t tile = dws_tile_elems();
    long made = 0, refused = 0;
    for (long it = 0; it < iters; ++it) {
        const int32_t T = static_cast<int32_t>(1 + rng() % (it % 50 == 0 ? 20000 : 300));
        std::vector<int64_t> numel(T);
        bool valid = true;
        for (int32_t t = 0; t < T; ++t) {
            const uint64_t r = rng() % 100;
            int64_t n;
            if (r < 20) n = 0;
            else if (r < 40) n = static_cast<int64_t>(rng() % 70000);
            else if (r < 60) n = tile * static_cast<int64_t>(rng() % 4) + static_cast<int64_t>(rng() % 3) - 1;
            else if (r < 99) n = static_cast<int64_t>(rng() % (1u << 24));
            else n = (rng() % 2) ? -1 - static_cast<int64_t>(rng() % 5) : (int64_t(1) << 31) + static_cast<int64_t>(rng() % 5);
            if (n < 0 && r < 60) n = 0;
            if (n < 0 || n > INT32_MAX) valid = false;
            numel[t] = n;
        }
        if (it % 7 == 3) numel[rng() % T] = INT32_MAX;
        dws_plan_t *p = nullptr;
        const int32_t elem = (it % 97 == 5) ? 4 : 2;
        const dws_status_t st = dws_plan_create(numel.data(), T, elem, &p);
        if (elem != 2) {
            if (st != DWS_ERR_UNSUPPORTED || p != nullptr) return fail("elem_size", it);
            ++refused;
            continue;
        }
        if (!valid) {
            if (st != DWS_ERR_INVALID || p != nullptr) return fail("invalid numel accepted", it);
            ++refused;
            continue;
        }
        if (st != DWS_OK || p == nullptr) return fail("valid plan refused", it);
        ++made;
        int64_t N = 0, tiles = 0;
        for (int32_t t = 0; t < T; ++t) {
            N += numel[t];
            tiles += numel[t] == 0 ? 1 : (numel[t] + tile - 1) / tile;
        }
        if (dws_plan_num_tensors(p) != T || dws_plan_num_elements(p) != N ||
            dws_plan_num_tiles(p) != tiles)
            return fail("plan queries", it);
        const size_t ws = dws_plan_workspace_bytes(p);
        if (ws < static_cast<size_t>(68 * tiles) || ws > static_cast<size_t>(256 + 16 * T + 16 + 72 * tiles + 4096))
            return fail("workspace size", it);
        for (int k = 0; k < 8; ++k) {
            const int32_t t = static_cast<int32_t>(rng() % T);
            if (dws_pos_width(p, t) != (numel[t] <= 65536 ? 2 : 4)) return fail("pos_width", it);
        }
        if (dws_pos_width(p, -1) != 0 || dws_pos_width(p, T) != 0) return fail("pos_width range", it);

        // refused on the host: no workspace, misaligned, too small, negative sizes
        void *fake = reinterpret_cast<void *>(0x100000);
        const void *const *tbl = reinterpret_cast<const void *const *>(fake);
        void *const *snaps = reinterpret_cast<void *const *>(fake);
        if (dws_encode(p, tbl, tbl, static_cast<int64_t *>(fake), static_cast<int32_t *>(fake),
                       static_cast<uint16_t *>(fake), 10, nullptr, ws, nullptr) != DWS_ERR_INVALID)
            return fail("encode null workspace", it);
        if (dws_encode(p, tbl, tbl, static_cast<int64_t *>(fake), static_cast<int32_t *>(fake),
                       static_cast<uint16_t *>(fake), 10, static_cast<char *>(fake) + 8, ws,
                       nullptr) != DWS_ERR_WORKSPACE)
            return fail("encode misaligned workspace", it);
        if (dws_encode(p, tbl, tbl, static_cast<int64_t *>(fake), static_cast<int32_t *>(fake),
                       static_cast<uint16_t *>(fake), 10, fake, ws - 1, nullptr) != DWS_ERR_WORKSPACE)
            return fail("encode short workspace", it);
        if (dws_encode(p, tbl, tbl, static_cast<int64_t *>(fake), static_cast<int32_t *>(fake),
                       static_cast<uint16_t *>(fake), -1, fake, ws, nullptr) != DWS_ERR_INVALID)
            return fail("encode negative capacity", it);
        if (dws_apply(p, snaps, static_cast<int64_t *>(fake), static_cast<int32_t *>(fake),
                      static_cast<uint16_t *>(fake), -3, fake, ws, nullptr) != DWS_ERR_INVALID)
            return fail("apply negative count", it);

        // the delta file's header for random valid counts and names
        std::vector<int64_t> off(T + 1, 0);
        std::vector<std::string> names(T);
        std::vector<const char *> np(T);
        for (int32_t t = 0; t < T; ++t) {
            const int64_t c = numel[t] == 0 ? 0 : static_cast<int64_t>(rng() % (numel[t] + 1));
            off[t + 1] = off[t] + (rng() % 3 == 0 ? c : 0);
            names[t] = "p" + std::to_string(t) + (rng() % 5 == 0 ? "\"\\\n\x01\xc3\xa9" : "");
            np[t] = names[t].c_str();
        }
        int64_t hb = 0;
        if (dws_st_delta_header(p, np.data(), off.data(), static_cast<int64_t>(rng()), nullptr, 0, &hb) !=
                DWS_OK ||
            hb < 8 || hb % 8 != 0)
            return fail("delta header", it);
        std::vector<uint8_t> buf(static_cast<size_t>(hb));
        int64_t hb2 = 0;
        if (dws_st_delta_header(p, np.data(), off.data(), 7, buf.data(), hb, &hb2) != DWS_OK)
            return fail("delta header write", it);
        if (T > 1) {  // a repeated name is refused
            np[1] = np[0];
            if (dws_st_delta_header(p, np.data(), off.data(), 7, nullptr, 0, &hb2) != DWS_ERR_INVALID)
                return fail("repeated name", it);
        }
        dws_plan_destroy(p);
    }
    std::printf("plans %ld refused %ld\n", made, refused);
    return made > 0 && refused > 0 ? 0 : 1;
}

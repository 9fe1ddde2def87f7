// chain.cu -- replay of a chain of deltas onto an anchor snapshot, in place
// ("Delta Weight Sync in TRL" §4.1: an anchor every N syncs, sparse deltas in
// between; a new replica takes the latest anchor and replays the deltas after
// it, the later delta winning where two touch the same element).
//
// Two kernels per pass over the snapshot:
//
//   chain_index_kernel  reads every entry of every delta once (coalesced
//     16-byte loads), checks it (index inside its tensor, strictly above the
//     entry before it in its tensor's segment) and writes the chain's tile
//     index: for tile g and delta k, the first entry of k at or past the start
//     of g, mod 2^32.  A failed check sets the workspace's delta flag, and the
//     replay kernel then writes nothing: a chain with a bad entry anywhere is
//     not applied at all.
//
//   chain_tile_kernel  one CTA per tile: the tile index gives each delta's
//     entries of the tile; every entry raises its element's tag in shared
//     memory to (k + 1) << 16 | value with atomicMax, so the latest delta
//     wins whatever the thread order; then the tagged elements are stored
//     (DWS_CHAIN_SCATTER: untouched sectors are not moved), or the whole tile,
//     read in first, is written back (DWS_CHAIN_TILE_MERGE: whole-sector
//     writes).  A tile no delta touches is not moved in either mode.
#include <cuda_runtime.h>

#include "dws_internal.cuh"

namespace dws {
namespace {

// ---------------------------------------------------------------------------
// Tile index and validation
// ---------------------------------------------------------------------------
constexpr int kIdxThreads = 256;
constexpr int kIdxPerThread = 16;
constexpr int kIdxChunk = kIdxThreads * kIdxPerThread;  // entries per block step

struct IndexParams {
    WsView ws;
    DeltaRef d[DWS_MAX_CHAIN];
    int K;
    int write;                 // write the tile index (else only check)
    uint32_t *index;           // [(ntiles + 1) * kChainGroup]
};

// index rows (lo, hi] of column `col` get `v`; the warp's lanes with long
// runs fill them together, the others alone.  Every lane of the warp calls
// it (warp-wide primitives); rows outside [0, nrows] are never written.
__device__ __forceinline__ void fill_rows(uint32_t *index, int col, long long lo, long long hi,
                                          uint32_t v, int lane, long long nrows) {
    if (lo < -1) lo = -1;
    if (hi > nrows) hi = nrows;
    const bool big = hi - lo > 32;
    unsigned int m = __ballot_sync(0xffffffffu, big);
    if (!big) {
        for (long long g = lo + 1; g <= hi; ++g) index[g * kChainGroup + col] = v;
    }
    while (m != 0u) {
        const int l = __ffs(m) - 1;
        m &= m - 1;
        const long long a = __shfl_sync(0xffffffffu, lo, l);
        const long long b = __shfl_sync(0xffffffffu, hi, l);
        const uint32_t w = __shfl_sync(0xffffffffu, v, l);
        for (long long g = a + 1 + lane; g <= b; g += 32) index[g * kChainGroup + col] = w;
    }
}

// Tile of entry j (index i, tensor t), or -2 if i is outside the tensor.
__device__ __forceinline__ long long entry_tile(const IndexParams &p, int t, int i) {
    return (i >= 0 && static_cast<long long>(i) < p.ws.numel[t]) ? p.ws.first_tile[t] + (i >> kTileShift) : -2;
}

// Block (x, k): entries [x * kIdxChunk, (x + 1) * kIdxChunk) of delta k,
// 16 consecutive ones per thread.  Each thread checks its run (strictly
// ascending, inside its tensor) and writes the index rows that start at its
// entries: entry j starts rows (tile of entry j-1, tile of entry j], the last
// entry also rows (its tile, ntiles] (at n).
__global__ void __launch_bounds__(kIdxThreads, 4) chain_index_kernel(IndexParams p) {
    __shared__ int s_t[2];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int k = blockIdx.y;
    const DeltaRef d = p.d[k];
    const int T = p.ws.num_tensors;
    const long long ntiles = p.ws.num_tiles;
    if (!ws_matches(p.ws)) return;
    if (ld_relaxed_gpu_u32(&p.ws.hdr->delta_bad) != 0u) return;  // offsets failed: nothing else
    const long long n = d.offsets[T];
    const long long base = static_cast<long long>(blockIdx.x) * kIdxChunk;
    if (n == 0) {  // no entry: every row points at entry 0
        if (p.write && blockIdx.x == 0 && warp == 0) fill_rows(p.index, k, -1, ntiles, 0u, lane, ntiles);
        return;
    }
    if (base >= n) return;  // uniform
    const long long last = (base + kIdxChunk < n ? base + kIdxChunk : n) - 1;
    if (warp < 2) {  // tensors of the block's first and last entries
        const int t = warp_tensor_of_entry(d.offsets, T, warp == 0 ? base : last);
        if (lane == 0) s_t[warp] = t;
    }
    // this thread's entries and the one before them, in flight meanwhile
    const long long j0 = base + static_cast<long long>(tid) * kIdxPerThread;
    const bool live0 = j0 <= last;
    const int nlive = !live0 ? 0 : static_cast<int>(last - j0 + 1 < kIdxPerThread ? last - j0 + 1 : kIdxPerThread);
    int x[kIdxPerThread];
    if (nlive == kIdxPerThread && (reinterpret_cast<uintptr_t>(d.indices) & 15u) == 0) {
#pragma unroll
        for (int v = 0; v < kIdxPerThread / 4; ++v) {
            const int4 a = __ldg(reinterpret_cast<const int4 *>(d.indices + j0) + v);
            x[4 * v] = a.x; x[4 * v + 1] = a.y; x[4 * v + 2] = a.z; x[4 * v + 3] = a.w;
        }
    } else {
#pragma unroll
        for (int q = 0; q < kIdxPerThread; ++q) x[q] = (q < nlive) ? __ldg(d.indices + j0 + q) : 0;
    }
    const int prev = (live0 && j0 > 0) ? __ldg(d.indices + j0 - 1) : 0;
    __syncthreads();
    const int t0 = s_t[0], t1 = s_t[1];

    bool bad = false;
    long long bad_j = 0;
    long long glast = -2;  // tile of this thread's last entry
    // The path is chosen per warp (both call warp-wide primitives): the fast
    // one only if every lane's run qualifies.
    const bool fast_lane = live0 && nlive == kIdxPerThread &&
                           (t0 == t1 || d.offsets[t0 + 1] > j0 + kIdxPerThread - 1) && d.offsets[t0] <= j0;
    if (__all_sync(0xffffffffu, fast_lane)) {
        // Common case, 32-bit: the run lies in tensor t0.  It must ascend
        // strictly (one compare per entry); then it is in range if its ends
        // are.  The run's first entry may open t0's segment: no order check
        // then, and its predecessor (another tensor's) bounds its rows.
        const int t = t0;
        const int nm = static_cast<int>(p.ws.numel[t]);
        const long long ft = p.ws.first_tile[t];
        const bool opens = d.offsets[t] == j0;
        bool viol = !opens && !(prev < x[0]);
#pragma unroll
        for (int q = 1; q < kIdxPerThread; ++q) viol |= !(x[q - 1] < x[q]);
        const bool ok = !viol && x[0] >= 0 && x[kIdxPerThread - 1] < nm;
        if (!ok) {
            // rare: the first offending entry (unrolled: x stays in registers)
            unsigned int badm = 0;
#pragma unroll
            for (int q = 0; q < kIdxPerThread; ++q) {
                const int pv = q == 0 ? prev : x[q - 1];
                const bool e_ok = x[q] >= 0 && x[q] < nm && ((q == 0 && opens) || pv < x[q]);
                badm |= e_ok ? 0u : (1u << q);
            }
            bad = true;
            bad_j = j0 + (badm ? __ffs(badm) - 1 : 0);
        }
        glast = ok ? ft + (x[kIdxPerThread - 1] >> kTileShift) : -2;
        if (p.write) {
            // the tile of the entry before the run: this tensor's, or, when
            // the run opens the segment, found by a search (once per tensor)
            long long gprev = -1;
            if (j0 > 0) {
                if (!opens) {
                    gprev = ft + (prev >> kTileShift);
                } else {
                    int lo = 0, hi = t;  // the tensor of entry j0 - 1
                    while (lo < hi) {
                        const int mid = (lo + hi + 1) >> 1;
                        if (d.offsets[mid] <= j0 - 1) lo = mid;
                        else hi = mid - 1;
                    }
                    gprev = entry_tile(p, lo, prev);
                }
            }
            // Rows (tile of entry q-1, tile of entry q] start at entry q, and
            // after the delta's last entry rows (its tile, ntiles] at n.  Each
            // lane writes its own short runs of rows (one row, usually);
            // runs longer than 32 rows (sparse deltas) are written by the
            // whole warp afterwards.  Bit 16 of `bigm` is the tail.
            unsigned int bigm = 0;
            const bool tail = ok && j0 + kIdxPerThread - 1 == n - 1;
            if (ok && gprev >= -1) {
                const long long g0 = ft + (x[0] >> kTileShift);
                if (g0 > gprev) {
                    if (g0 - gprev <= 32) {
                        for (long long g = gprev + 1; g <= g0; ++g)
                            p.index[g * kChainGroup + k] = static_cast<uint32_t>(j0);
                    } else {
                        bigm |= 1u;
                    }
                }
                int tp = x[0] >> kTileShift;
#pragma unroll
                for (int q = 1; q < kIdxPerThread; ++q) {
                    const int tl = x[q] >> kTileShift;
                    if (tl != tp) {
                        if (tl - tp <= 32) {
                            for (long long g = ft + tp + 1; g <= ft + tl; ++g)
                                p.index[g * kChainGroup + k] = static_cast<uint32_t>(j0 + q);
                        } else {
                            bigm |= 1u << q;
                        }
                    }
                    tp = tl;
                }
                if (tail) {
                    if (ntiles - glast <= 32) {
                        for (long long g = glast + 1; g <= ntiles; ++g)
                            p.index[g * kChainGroup + k] = static_cast<uint32_t>(n);
                    } else {
                        bigm |= 1u << 16;
                    }
                }
            }
            while (__any_sync(0xffffffffu, bigm != 0u)) {
                // one long run per lane per round, the warp writing together
                long long lo = 0, hi = 0;
                uint32_t v = 0;
                if (bigm != 0u) {
                    const int q = __ffs(bigm) - 1;
                    bigm &= bigm - 1;
                    if (q == 16) {
                        lo = glast;
                        hi = ntiles;
                        v = static_cast<uint32_t>(n);
                    } else {
                        int xi = 0, xp = 0;
#pragma unroll
                        for (int r = 0; r < kIdxPerThread; ++r) {
                            if (r == q) xi = x[r];
                            if (r == q - 1) xp = x[r];
                        }
                        hi = ft + (xi >> kTileShift);
                        lo = (q == 0) ? gprev : ft + (xp >> kTileShift);
                        v = static_cast<uint32_t>(j0 + q);
                    }
                }
                fill_rows(p.index, k, lo, hi, v, lane, ntiles);
            }
        }
    } else {
        // General case (a run across tensors, a short run, or a block that
        // the search placed oddly): every entry's tensor is walked.
        long long g[kIdxPerThread];
        unsigned int okm = 0;  // bit q: entry q in range and ordered
        long long gprev0 = -1;  // tile of the entry before the run
        int tq = t0;
        if (live0) {
            int lo = t0, hi = t1;  // the tensor of entry j0
            while (lo < hi) {
                const int mid = (lo + hi + 1) >> 1;
                if (d.offsets[mid] <= j0) lo = mid;
                else hi = mid - 1;
            }
            tq = lo;
            if (j0 > 0) {
                int tp = tq;
                if (d.offsets[tq] > j0 - 1 || d.offsets[tq] == j0) {
                    int a = 0, b = tq;  // the tensor of entry j0 - 1
                    while (a < b) {
                        const int mid = (a + b + 1) >> 1;
                        if (d.offsets[mid] <= j0 - 1) a = mid;
                        else b = mid - 1;
                    }
                    tp = a;
                }
                gprev0 = entry_tile(p, tp, prev);
            }
        }
        int pv = prev;
#pragma unroll
        for (int q = 0; q < kIdxPerThread; ++q) {
            const long long j = j0 + q;
            g[q] = -2;
            if (q < nlive) {
                while (d.offsets[tq + 1] <= j) ++tq;  // empty tensors are skipped too
                const int i = x[q];
                const bool ord = j == d.offsets[tq] || pv < i;
                g[q] = entry_tile(p, tq, i);
                okm |= (g[q] >= 0 && ord) ? (1u << q) : 0u;
            }
            pv = x[q];
        }
        const unsigned int livem = (1u << nlive) - 1u;
        const unsigned int badm = livem & ~okm;
        if (badm != 0u) {
            bad = true;
            bad_j = j0 + (__ffs(badm) - 1);
        }
#pragma unroll
        for (int r = 0; r < kIdxPerThread; ++r)
            if (r == nlive - 1) glast = g[r];
        if (p.write) {
            unsigned int bnd = 0;
            long long gp = gprev0;
#pragma unroll
            for (int q = 0; q < kIdxPerThread; ++q) {
                if (((livem >> q) & 1u) && g[q] >= 0 && gp >= -1 && g[q] > gp) bnd |= 1u << q;
                if ((livem >> q) & 1u) gp = g[q];
            }
            const bool tail = nlive > 0 && j0 + nlive - 1 == n - 1 && glast >= 0;
            unsigned int any_q = __reduce_or_sync(0xffffffffu, bnd);
            while (any_q != 0u) {
                const int q = __ffs(any_q) - 1;
                any_q &= any_q - 1;
                long long lo = gprev0, gq = 0;
#pragma unroll
                for (int r = 0; r < kIdxPerThread; ++r) {
                    if (r < q && ((livem >> r) & 1u)) lo = g[r];
                    if (r == q) gq = g[r];
                }
                const bool mine = (bnd >> q) & 1u;
                fill_rows(p.index, k, mine ? lo : 0, mine ? gq : 0, static_cast<uint32_t>(j0 + q), lane, ntiles);
            }
            if (__any_sync(0xffffffffu, tail))
                fill_rows(p.index, k, tail ? glast : 0, tail ? ntiles : 0, static_cast<uint32_t>(n), lane, ntiles);
        }
    }
    if (bad) {
        atomicOr(&p.ws.hdr->delta_bad, 1u);
        record_error(p.ws.hdr, DWS_ERR_BAD_DELTA, bad_j);
    }
}

// ---------------------------------------------------------------------------
// Per-tile replay: one CTA per tile
// ---------------------------------------------------------------------------
constexpr int kTileThreads = 256;
constexpr int kTileWarps = kTileThreads / 32;
constexpr int kItemEntries = 128;                         // 4 consecutive entries per lane
constexpr int kTileItems = 3;                             // items per warp per round
constexpr int kTileRoundItems = kTileWarps * kTileItems;  // items per round
constexpr int kTileMinBlocks = 6;

struct TileParams {
    WsView ws;
    uint16_t *const *snap_ptrs;
    const uint32_t *index;
    int K;
    DeltaRef d[kChainGroup];
};

struct TileShared {
    // Delta k's entries of the tile are base + [lo, hi), base = the first
    // entry rounded down to a multiple of 4, so that items start aligned;
    // lim = entries from base to the end of the delta's arrays.
    const int *ip[kChainGroup];
    const uint16_t *vp[kChainGroup];
    int lo[kChainGroup];
    int hi[kChainGroup];
    long long lim[kChainGroup];
    int vec[kChainGroup];                       // 16-byte loads allowed (aligned arrays)
    int C[kChainGroup + 1];                     // items of the deltas before k
    uint16_t *dst;                              // tile start in the snapshot (null: skip)
    int local;                                  // tile start within its tensor
    int count;                                  // elements of the tile
};

__device__ __forceinline__ int int4_at(const int4 &v, int e) {
    return e == 0 ? v.x : (e == 1 ? v.y : (e == 2 ? v.z : v.w));
}
__device__ __forceinline__ uint32_t u16x4_at(const uint2 &v, int e) {
    const uint32_t w = e < 2 ? v.x : v.y;
    return (e & 1) ? (w >> 16) : (w & 0xffffu);
}

// Round r of this warp's items: item i = r * kTileRoundItems + warp + q *
// kTileWarps covers entries base + 128 c + [0, 128) of delta k (c = i -
// C[k]); lane l takes the 4 entries from base + 128 c + 4 l.  kq[q] = k
// (warp-uniform; -1: no such item); vm[q] bit e: entry e is the tile's.
// Every load of the round is in flight at once.
__device__ __forceinline__ void tile_load_round(const TileShared &sm, int K, int r, int4 (&ix)[kTileItems],
                                                uint2 (&vx)[kTileItems], int (&kq)[kTileItems],
                                                unsigned int (&vm)[kTileItems]) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int i0 = r * kTileRoundItems + warp;
    const int items = sm.C[K];
    int k = 0;
    while (k + 1 < K && sm.C[k + 1] <= i0) ++k;
#pragma unroll
    for (int q = 0; q < kTileItems; ++q) {
        const int i = i0 + q * kTileWarps;
        kq[q] = -1;
        vm[q] = 0u;
        if (i < items) {  // warp-uniform
            while (k + 1 < K && sm.C[k + 1] <= i) ++k;
            kq[q] = k;
            const int o = (i - sm.C[k]) * kItemEntries + 4 * lane;
            const int lo = sm.lo[k], hi = sm.hi[k];
            unsigned int m = 0u;
#pragma unroll
            for (int e = 0; e < 4; ++e) m |= (o + e >= lo && o + e < hi) ? (1u << e) : 0u;
            vm[q] = m;
            if (m == 0xfu && sm.vec[k] && o + 3 < sm.lim[k]) {
                ix[q] = __ldg(reinterpret_cast<const int4 *>(sm.ip[k] + o));
                vx[q] = __ldg(reinterpret_cast<const uint2 *>(sm.vp[k] + o));
            } else if (m != 0u) {
                int xs[4] = {0, 0, 0, 0};
                uint32_t vs[4] = {0u, 0u, 0u, 0u};
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    if ((m >> e) & 1u) {
                        xs[e] = __ldg(sm.ip[k] + o + e);
                        vs[e] = __ldg(sm.vp[k] + o + e);
                    }
                }
                ix[q] = make_int4(xs[0], xs[1], xs[2], xs[3]);
                vx[q] = make_uint2(vs[0] | (vs[1] << 16), vs[2] | (vs[3] << 16));
            }
        }
    }
}

// One CTA replays every delta of the group onto one tile.  Each element has
// a 32-bit tag in shared memory; every entry of delta k raises its element's
// tag to (k + 1) << 16 | value with atomicMax, so that whatever the thread
// order the tag ends with the latest delta's value, and no entry is read
// twice.  Then one coalesced pass writes the tile:
//   scatter (kMerge false): tags start at 0, and only tagged elements are
//     stored to the snapshot (untouched sectors are not moved);
//   merge (kMerge true): tags start as the tile's own values (version 0),
//     and the whole tile is written back (whole-sector writes).
// Warp 0 first turns the tile's two index rows into per-delta entry ranges;
// the work is cut into items of 128 entries of one delta (4 per lane, 16-byte
// loads when the arrays allow).  A tile no delta touches is not moved.
template <bool kMerge>
__global__ void __launch_bounds__(kTileThreads, kTileMinBlocks) chain_tile_kernel(TileParams p) {
    __shared__ TileShared sm;
    __shared__ __align__(16) uint32_t s_tag[kTileElems];
    const int tid = threadIdx.x, lane = tid & 31;
    const long long g = blockIdx.x;
    const int K = p.K;

    if constexpr (!kMerge) {
#pragma unroll
        for (int q = 0; q < kTileElems / 4 / kTileThreads; ++q)
            reinterpret_cast<uint4 *>(s_tag)[tid + q * kTileThreads] = make_uint4(0u, 0u, 0u, 0u);
    }
    if (tid < 32) {
        // The rows are requested before the header is checked: the workspace
        // size was checked on the host, so every address here is inside it.
        const int t = p.ws.tile_tensor[g];
        uint32_t ra = 0, rb = 0;
        if (lane < K) {
            ra = p.index[g * kChainGroup + lane];
            rb = p.index[(g + 1) * kChainGroup + lane];
        }
        const WsHeader *h = p.ws.hdr;
        bool ok = h->magic == kWsMagic && h->fingerprint == p.ws.fingerprint &&
                  h->num_tiles == p.ws.num_tiles && h->num_tensors == p.ws.num_tensors;
        if (!ok && lane == 0) record_error(p.ws.hdr, DWS_ERR_WORKSPACE, 0);
        ok = ok && ld_relaxed_gpu_u32(&h->delta_bad) == 0u;
        if (ok && (t < 0 || t >= p.ws.num_tensors)) {
            if (lane == 0) record_error(p.ws.hdr, DWS_ERR_WORKSPACE, g);
            ok = false;
        }
        long long s = 0;
        int n = 0;
        if (ok && lane < K) {
            const DeltaRef d = p.d[lane];
            const long long lo = d.offsets[t];
            s = lo + static_cast<long long>(ra - static_cast<uint32_t>(lo));
            long long e = lo + static_cast<long long>(rb - static_cast<uint32_t>(lo));
            // kept inside the delta's arrays and one tile's worth
            s = s < 0 ? 0 : (s > d.count ? d.count : s);
            e = e > d.count ? d.count : e;
            e = e - s > kTileElems ? s + kTileElems : e;
            n = e > s ? static_cast<int>(e - s) : 0;
            const long long base = s & ~3LL;
            sm.ip[lane] = d.indices + base;
            sm.vp[lane] = d.values + base;
            sm.lo[lane] = static_cast<int>(s - base);
            sm.hi[lane] = static_cast<int>(s - base) + n;
            sm.lim[lane] = d.count - base;
            sm.vec[lane] = ((reinterpret_cast<uintptr_t>(d.indices) & 15u) == 0 &&
                            (reinterpret_cast<uintptr_t>(d.values) & 7u) == 0) ? 1 : 0;
        }
        // items of delta k: ceil(hi / 128), none if it has no entry here
        int pre = n > 0 ? (static_cast<int>(s & 3LL) + n + kItemEntries - 1) / kItemEntries : 0;
#pragma unroll
        for (int o = 1; o < kChainGroup; o <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, pre, o);
            if (lane >= o) pre += y;
        }
        if (lane < K) sm.C[lane + 1] = pre;
        if (lane == 0) {
            sm.C[0] = 0;
            uint16_t *dst = nullptr;
            int local = 0, count = 0;
            if (ok) {
                const long long ls = (g - p.ws.first_tile[t]) << kTileShift;
                const long long rest = p.ws.numel[t] - ls;
                count = static_cast<int>(rest < kTileElems ? (rest > 0 ? rest : 0) : kTileElems);
                local = static_cast<int>(ls);
                dst = p.snap_ptrs[t];
                if (count > 0 && (dst == nullptr || (reinterpret_cast<uintptr_t>(dst) & 1u))) {
                    record_error(p.ws.hdr, DWS_ERR_INVALID, t);
                    dst = nullptr;
                }
                if (dst != nullptr) dst += ls;
            }
            sm.dst = dst;
            sm.local = local;
            sm.count = count;
        }
    }
    __syncthreads();
    uint16_t *const dst = sm.dst;
    const int items = sm.C[K];
    if (dst == nullptr || items == 0) return;  // uniform
    const int local = sm.local, count = sm.count;
    const bool vec = count == kTileElems && (reinterpret_cast<uintptr_t>(dst) & 15u) == 0;

    const int rounds = (items + kTileRoundItems - 1) / kTileRoundItems;
    int4 ix[kTileItems];
    uint2 vx[kTileItems];
    int kq[kTileItems];
    unsigned int vm[kTileItems];
    tile_load_round(sm, K, 0, ix, vx, kq, vm);
    if constexpr (kMerge) {
        // tags <- the tile's values (version 0), while the entries arrive
        if (vec) {
            uint4 t4[kTileElems / 8 / kTileThreads];
#pragma unroll
            for (int q = 0; q < kTileElems / 8 / kTileThreads; ++q)
                t4[q] = ld_stream_v4(reinterpret_cast<const uint4 *>(dst) + tid + q * kTileThreads);
#pragma unroll
            for (int q = 0; q < kTileElems / 8 / kTileThreads; ++q) {
                uint4 *o = reinterpret_cast<uint4 *>(s_tag + (tid + q * kTileThreads) * 8);
                o[0] = make_uint4(t4[q].x & 0xffffu, t4[q].x >> 16, t4[q].y & 0xffffu, t4[q].y >> 16);
                o[1] = make_uint4(t4[q].z & 0xffffu, t4[q].z >> 16, t4[q].w & 0xffffu, t4[q].w >> 16);
            }
        } else {
            for (int i = tid; i < kTileElems; i += kTileThreads) s_tag[i] = i < count ? dst[i] : 0u;
        }
    }
    __syncthreads();  // tags initialised
    for (int r = 0; r < rounds; ++r) {
        if (r > 0) tile_load_round(sm, K, r, ix, vx, kq, vm);
#pragma unroll
        for (int q = 0; q < kTileItems; ++q) {
            const uint32_t ver = static_cast<uint32_t>(kq[q] + 1) << 16;
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                if ((vm[q] >> e) & 1u) {
                    // position within the tile; checked entries never fall outside
                    const uint32_t pos = static_cast<uint32_t>(int4_at(ix[q], e) - local);
                    if (pos < static_cast<uint32_t>(count)) atomicMax(&s_tag[pos], ver | u16x4_at(vx[q], e));
                    else record_error(p.ws.hdr, DWS_ERR_WORKSPACE, g);
                }
            }
        }
    }
    __syncthreads();
    if constexpr (kMerge) {
        if (vec) {
#pragma unroll
            for (int q = 0; q < kTileElems / 8 / kTileThreads; ++q) {
                const uint4 *t = reinterpret_cast<const uint4 *>(s_tag + (tid + q * kTileThreads) * 8);
                const uint4 a = t[0], b = t[1];
                st_stream_v4(reinterpret_cast<uint4 *>(dst) + tid + q * kTileThreads,
                             make_uint4((a.x & 0xffffu) | (a.y << 16), (a.z & 0xffffu) | (a.w << 16),
                                        (b.x & 0xffffu) | (b.y << 16), (b.z & 0xffffu) | (b.w << 16)));
            }
        } else {
            for (int i = tid; i < count; i += kTileThreads) dst[i] = static_cast<uint16_t>(s_tag[i]);
        }
    } else {
        // 4 consecutive elements per thread, a warp 128: the tagged ones are
        // stored, as one 8-byte store when all four are and it is aligned
        const bool al8 = (reinterpret_cast<uintptr_t>(dst) & 7u) == 0;
#pragma unroll 2
        for (int q = 0; q < kTileElems / 4 / kTileThreads; ++q) {
            const int e0 = (tid + q * kTileThreads) * 4;
            const uint4 t = reinterpret_cast<const uint4 *>(s_tag)[tid + q * kTileThreads];
            const bool h0 = t.x >> 16, h1 = t.y >> 16, h2 = t.z >> 16, h3 = t.w >> 16;
            if (h0 && h1 && h2 && h3 && al8) {
                *reinterpret_cast<uint2 *>(dst + e0) =
                    make_uint2((t.x & 0xffffu) | (t.y << 16), (t.z & 0xffffu) | (t.w << 16));
            } else {
                if (h0) dst[e0] = static_cast<uint16_t>(t.x);
                if (h1) dst[e0 + 1] = static_cast<uint16_t>(t.y);
                if (h2) dst[e0 + 2] = static_cast<uint16_t>(t.z);
                if (h3) dst[e0 + 3] = static_cast<uint16_t>(t.w);
            }
        }
    }
}

}  // namespace

cudaError_t launch_apply_chain(const WsView &ws, uint16_t *const *snap_ptrs, const DeltaRef *deltas,
                               int K, bool merge, cudaStream_t s) {
    cudaError_t e = launch_delta_check(ws, deltas, K, s);  // offsets of every delta
    if (e != cudaSuccess) return e;
    uint32_t *index = reinterpret_cast<uint32_t *>(ws.tile_status);

    // Index-pass grid: one block per kIdxChunk entries of every delta.
    auto index_grid = [&](const DeltaRef *ds, int nk, IndexParams &) -> long long {
        long long max_n = 1;
        for (int k = 0; k < nk; ++k) max_n = ds[k].count > max_n ? ds[k].count : max_n;
        return (max_n + kIdxChunk - 1) / kIdxChunk;
    };
    IndexParams ip;
    ip.ws = ws;
    ip.index = index;
    if (K > kChainGroup) {  // every delta checked before the first pass writes
        ip.K = K;
        ip.write = 0;
        for (int k = 0; k < K; ++k) ip.d[k] = deltas[k];
        const long long bx = index_grid(deltas, K, ip);
        if (bx > 0x7fffffffLL) return cudaErrorInvalidValue;
        chain_index_kernel<<<dim3(static_cast<unsigned int>(bx), K), kIdxThreads, 0, s>>>(ip);
        e = launched();
        if (e != cudaSuccess) return e;
    }
    for (int k0 = 0; k0 < K; k0 += kChainGroup) {
        const int kg = (K - k0 < kChainGroup) ? K - k0 : kChainGroup;
        ip.K = kg;
        ip.write = 1;
        for (int k = 0; k < kg; ++k) ip.d[k] = deltas[k0 + k];
        const long long gx = index_grid(deltas + k0, kg, ip);
        if (gx > 0x7fffffffLL) return cudaErrorInvalidValue;
        chain_index_kernel<<<dim3(static_cast<unsigned int>(gx), kg), kIdxThreads, 0, s>>>(ip);
        e = launched();
        if (e != cudaSuccess) return e;
        TileParams tp;
        tp.ws = ws;
        tp.snap_ptrs = snap_ptrs;
        tp.index = index;
        tp.K = kg;
        for (int k = 0; k < kg; ++k) tp.d[k] = deltas[k0 + k];
        if (ws.num_tiles > 0x7fffffffLL) return cudaErrorInvalidValue;
        if (ws.num_tiles > 0) {
            const unsigned int grid = static_cast<unsigned int>(ws.num_tiles);
            if (merge) chain_tile_kernel<true><<<grid, kTileThreads, 0, s>>>(tp);
            else chain_tile_kernel<false><<<grid, kTileThreads, 0, s>>>(tp);
        }
        e = launched();
        if (e != cudaSuccess) return e;
    }
    return cudaSuccess;
}

}  // namespace dws

// chain.cu -- replay of a chain of deltas onto an anchor snapshot, in place
// ("Delta Weight Sync in TRL" §4.1: an anchor every N syncs, sparse deltas in
// between; a new replica takes the latest anchor and replays the deltas after
// it, the later delta winning where two touch the same element).
//
// Three kernels per pass over the snapshot:
//
//   chain_index_kernel  reads every entry of every delta once (coalesced
//     16-byte loads), checks it (index inside its tensor, strictly above the
//     entry before it in its tensor's segment) and writes the chain's tile
//     index: for tile g and delta k, the first entry of k at or past the start
//     of g, mod 2^32.  A failed check sets the workspace's delta flag, and the
//     replay kernels then write nothing: a chain with a bad entry anywhere is
//     not applied at all.
//
//   chain_merge_kernel  (DWS_CHAIN_TILE_MERGE) CTAs over contiguous ranges of
//     tiles; per tile each thread owns 32 elements and each warp a share of
//     the tile's entries (exactly the tile's, from the tile index), all
//     loaded one tile ahead into registers with plain vector loads; every
//     entry raises its element's tag in shared memory to (k + 1) << 16 |
//     value with atomicMax (the latest delta wins whatever the thread order),
//     then each thread merges its 32 elements and writes them back.  A tile
//     no delta touches is neither read nor written.
//
//   chain_scatter_kernel  (DWS_CHAIN_SCATTER) per window of 32 tiles the
//     deltas are replayed from the last to the first, an element being
//     stored only if its written-bit in shared memory is clear, so every
//     element is written once, by the latest delta that names it; untouched
//     32-byte sectors are not moved at all.  The tile index gives each
//     window's stretch of every delta.
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
            int pv = prev;  // rare: locate the first offending entry
            for (int q = 0; q < kIdxPerThread; ++q) {
                if (!(x[q] >= 0 && x[q] < nm && ((q == 0 && opens) || pv < x[q]))) {
                    bad = true;
                    bad_j = j0 + q;
                    break;
                }
                pv = x[q];
            }
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

// The first entry of delta `d` at or past the start of tile g (in tensor t),
// from the tile index: the only value in [offsets[t], offsets[t+1]] with
// these low 32 bits (a tensor has fewer than 2^31 entries).
__device__ __forceinline__ long long index_entry(const DeltaRef &d, const uint32_t *index, long long g,
                                                 int col, int t) {
    const long long lo = d.offsets[t];
    return lo + static_cast<long long>(index[g * kChainGroup + col] - static_cast<uint32_t>(lo));
}

// ---------------------------------------------------------------------------
// Tile merge (register streaming)
// ---------------------------------------------------------------------------
// Each CTA walks a contiguous range of tiles.  Per tile, thread t owns the
// 32 elements [32 t, 32 t + 32) (four 16-byte vectors) and each warp a share
// of the tile's entries, in work items of 32 entries of one delta (the tile
// index gives every delta's range).  While tile i is merged, the loads of
// tile i+1 -- its 32 elements per thread and its entries -- are in flight in
// registers.  Merge: every entry raises its element's tag in shared memory to
// (k + 1) << 16 | value (atomicMax: the latest delta wins whatever the thread
// order); then each thread takes the tags of its elements, clears them, and
// writes its 32 merged elements back with 16-byte stores.  A tile no delta
// touches is neither read nor written; a tile whose elements cannot move as
// whole 16-byte vectors (an unaligned tensor, a tensor's short last tile)
// gets its tagged values stored one by one.
constexpr int kMThreads = 256;
constexpr int kMWarps = kMThreads / 32;
constexpr int kMPer = kTileElems / kMThreads;  // 32 elements per thread
constexpr int kMVec = kMPer / 8;               // 4 vectors of 8 elements
constexpr int kMPre = 10;                      // entry items per warp held in registers

struct MergeParams {
    WsView ws;
    uint16_t *const *snap_ptrs;
    const uint32_t *index;
    long long tiles_per_cta;
    int K;
    DeltaRef d[kChainGroup];
};

struct MergeSmem {
    uint32_t tag[kTileElems];
    const int *idx[kChainGroup];
    const uint16_t *val[kChainGroup];
    long long cnt[kChainGroup];
};

// One tile as a warp sees it.  Lane k < K: delta k's first entry of the tile
// (s), its entries (n) and the exclusive prefix of the items (c0, items of 32
// entries of one delta, in delta order).
struct TileView {
    uint16_t *ptr;  // the tile's first element (null: untouched)
    int local_start;
    int count;      // elements
    bool vec;       // whole 16-byte vectors: aligned pointer and a full tile
    long long s;
    int n;
    int c0;
    int items;      // the tile's items
};

// This thread's loads of one tile, in flight: its 32 elements and its warp's
// first kMPre items (item w + kMWarps * r is this warp's r-th): the entry's
// index and its tag (k + 1) << 16 | value (0: no entry).
struct TileLoads {
    uint4 e[kMVec];
    int ix[kMPre];
    uint32_t tg[kMPre];
};

// The delta (lane) an item belongs to: items are in delta order.
__device__ __forceinline__ int item_delta(int item, int c0, int n_items, int K) {
    const int lane = threadIdx.x & 31;
    const bool before = lane < K && c0 + n_items <= item;  // delta `lane` ends at or before item
    return __popc(__ballot_sync(0xffffffffu, before));
}

// Warp-wide: the view of tile i (tensor t, its first tile `first`, numel,
// pointer), from the index rows of tiles i and i+1 (lane k: delta k).
__device__ __forceinline__ void tile_view(const MergeParams &p, long long i, long long first, long long numel,
                                          uint16_t *tptr, uint32_t row_i, uint32_t row_next, long long &cursor,
                                          TileView &v) {
    const int lane = threadIdx.x & 31;
    const long long ls = (i - first) << kTileShift;
    const long long rest = numel - ls;
    v.local_start = static_cast<int>(ls);
    v.count = static_cast<int>(rest < kTileElems ? (rest > 0 ? rest : 0) : kTileElems);
    v.s = cursor;
    v.n = lane < p.K ? static_cast<int>(row_next - row_i) : 0;
    if (lane < p.K) cursor += v.n;
    const int ni = (v.n + 31) >> 5;
    int incl = ni;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int x = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += x;
    }
    v.c0 = incl - ni;
    v.items = __shfl_sync(0xffffffffu, incl, 31);
    const bool touched = v.items > 0 && v.count > 0 && tptr != nullptr &&
                         (reinterpret_cast<uintptr_t>(tptr) & 1u) == 0;
    v.ptr = touched ? tptr + ls : nullptr;
    v.vec = touched && v.count == kTileElems && (reinterpret_cast<uintptr_t>(tptr) & 15u) == 0;
}

// Issues this thread's loads of tile v (elements when v.vec; the warp's first
// kMPre items).
__device__ __forceinline__ void tile_issue(const MergeParams &p, const MergeSmem &sm, const TileView &v,
                                           TileLoads &L) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    if (v.vec) {
        const uint4 *src = reinterpret_cast<const uint4 *>(v.ptr + threadIdx.x * kMPer);
#pragma unroll
        for (int q = 0; q < kMVec; ++q) L.e[q] = ld_stream_v4(src + q);
    }
#pragma unroll
    for (int r = 0; r < kMPre; ++r) {
        const int item = warp + r * kMWarps;
        L.ix[r] = 0;
        L.tg[r] = 0u;
        if (item < v.items) {  // uniform per warp
            const int k = item_delta(item, v.c0, (v.n + 31) >> 5, p.K);
            const int c0 = __shfl_sync(0xffffffffu, v.c0, k);
            const int n = __shfl_sync(0xffffffffu, v.n, k);
            const long long s = __shfl_sync(0xffffffffu, v.s, k);
            const int el = ((item - c0) << 5) + lane;
            const long long j = s + el;
            if (el < n && j >= 0 && j < sm.cnt[k]) {  // (the index keeps it inside; the check is cheap)
                L.ix[r] = __ldg(sm.idx[k] + j);
                L.tg[r] = (static_cast<uint32_t>(k + 1) << 16) | __ldg(sm.val[k] + j);
            }
        }
    }
}

// Tags one entry: the element at (index - local_start) of the tile gets the
// entry's tag unless a later delta's is there.
__device__ __forceinline__ void tag_entry(MergeSmem &sm, const MergeParams &p, const TileView &v, int index,
                                          uint32_t tag) {
    const int pos = index - v.local_start;  // in [0, count): the index pass's ranges
    if (static_cast<unsigned>(pos) < static_cast<unsigned>(v.count))
        atomicMax(&sm.tag[pos], tag);
    else
        record_error(p.ws.hdr, DWS_ERR_WORKSPACE, pos);  // never expected
}

__global__ void __launch_bounds__(kMThreads, 2) chain_merge_kernel(MergeParams p) {
    extern __shared__ __align__(128) unsigned char merge_smem_raw[];
    MergeSmem &sm = *reinterpret_cast<MergeSmem *>(merge_smem_raw);
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;

    if (!ws_matches(p.ws)) return;
    if (ld_relaxed_gpu_u32(&p.ws.hdr->delta_bad) != 0u) return;
    const long long tb = static_cast<long long>(blockIdx.x) * p.tiles_per_cta;
    long long te = tb + p.tiles_per_cta;
    if (te > p.ws.num_tiles) te = p.ws.num_tiles;
    if (tb >= te) return;

    for (int e = tid; e < kTileElems; e += kMThreads) sm.tag[e] = 0u;
    if (tid < p.K) {
        sm.idx[tid] = p.d[tid].indices;
        sm.val[tid] = p.d[tid].values;
        sm.cnt[tid] = p.d[tid].count;
    }
    // every warp keeps its own copy of the walk: tensor, cursors, index rows
    int t = p.ws.tile_tensor[tb];
    long long first = p.ws.first_tile[t], next = p.ws.first_tile[t + 1], numel = p.ws.numel[t];
    uint16_t *tptr = p.snap_ptrs[t];
    long long cursor = 0;  // lane k: delta k's first entry of the next tile to view
    // lane k: index rows of tiles i+1 and i+2 (row i+3 is loaded one tile ahead)
    uint32_t row0 = 0, row1 = 0, row2 = 0;
    const long long nrows = p.ws.num_tiles;
    if (lane < p.K) {
        cursor = index_entry(p.d[lane], p.index, tb, lane, t);
        row0 = p.index[tb * kChainGroup + lane];
        row1 = p.index[(tb + 1) * kChainGroup + lane];
        if (tb + 2 <= nrows) row2 = p.index[(tb + 2) * kChainGroup + lane];
    }
    __syncthreads();

    TileView va, vb;
    TileLoads la, lb;
    tile_view(p, tb, first, numel, tptr, row0, row1, cursor, va);
    tile_issue(p, sm, va, la);

    // One tile: view and start loading tile i + 1 into (nv, nl), then merge
    // tile i from (cv, cl).  Called with the two buffers swapped on
    // alternate tiles, so that no register holding a load in flight is
    // copied (a copy would wait for the load).
    auto step = [&](long long i, const TileView &cv, const TileLoads &cl, TileView &nv, TileLoads &nl) {
        nv.items = 0;
        nv.ptr = nullptr;
        if (i + 1 < te) {
            while (i + 1 >= next) {  // uniform: the next tensor
                ++t;
                first = p.ws.first_tile[t];
                next = p.ws.first_tile[t + 1];
                numel = p.ws.numel[t];
                tptr = p.snap_ptrs[t];
            }
            const uint32_t row3 = (lane < p.K && i + 3 <= nrows) ? p.index[(i + 3) * kChainGroup + lane] : 0u;
            tile_view(p, i + 1, first, numel, tptr, row1, row2, cursor, nv);
            tile_issue(p, sm, nv, nl);
            row1 = row2;
            row2 = row3;
        }
        if (cv.ptr == nullptr) return;  // uniform: untouched
        // tag tile i's entries: the items held, then the rest
#pragma unroll
        for (int r = 0; r < kMPre; ++r)
            if (cl.tg[r] != 0u) tag_entry(sm, p, cv, cl.ix[r], cl.tg[r]);
        for (int item = warp + kMPre * kMWarps; item < cv.items; item += kMWarps) {
            const int k = item_delta(item, cv.c0, (cv.n + 31) >> 5, p.K);
            const int c0 = __shfl_sync(0xffffffffu, cv.c0, k);
            const int n = __shfl_sync(0xffffffffu, cv.n, k);
            const long long s = __shfl_sync(0xffffffffu, cv.s, k);
            const int el = ((item - c0) << 5) + lane;
            const long long j = s + el;
            if (el < n && j >= 0 && j < sm.cnt[k])
                tag_entry(sm, p, cv, __ldg(sm.idx[k] + j),
                          (static_cast<uint32_t>(k + 1) << 16) | __ldg(sm.val[k] + j));
        }
        __syncthreads();
        // merge this thread's 32 elements, clear their tags
        const int e0 = tid * kMPer;
        if (cv.vec) {
            uint4 *dst = reinterpret_cast<uint4 *>(cv.ptr + e0);
#pragma unroll
            for (int q = 0; q < kMVec; ++q) {
                uint32_t w[4] = {cl.e[q].x, cl.e[q].y, cl.e[q].z, cl.e[q].w};
                const uint4 ta = *reinterpret_cast<const uint4 *>(&sm.tag[e0 + 8 * q]);
                const uint4 tc = *reinterpret_cast<const uint4 *>(&sm.tag[e0 + 8 * q + 4]);
                const uint32_t tg[8] = {ta.x, ta.y, ta.z, ta.w, tc.x, tc.y, tc.z, tc.w};
                if ((ta.x | ta.y | ta.z | ta.w | tc.x | tc.y | tc.z | tc.w) != 0u) {
#pragma unroll
                    for (int h = 0; h < 8; ++h) {
                        if (tg[h]) {
                            const uint32_t sh = (h & 1) * 16;
                            w[h >> 1] = (w[h >> 1] & ~(0xffffu << sh)) | ((tg[h] & 0xffffu) << sh);
                        }
                    }
                    *reinterpret_cast<uint4 *>(&sm.tag[e0 + 8 * q]) = make_uint4(0u, 0u, 0u, 0u);
                    *reinterpret_cast<uint4 *>(&sm.tag[e0 + 8 * q + 4]) = make_uint4(0u, 0u, 0u, 0u);
                }
                st_stream_v4(dst + q, make_uint4(w[0], w[1], w[2], w[3]));
            }
        } else {
#pragma unroll 4
            for (int h = 0; h < kMPer; ++h) {
                const int e = e0 + h;
                const uint32_t tg = sm.tag[e];
                if (tg) {
                    sm.tag[e] = 0u;
                    if (e < cv.count) cv.ptr[e] = static_cast<uint16_t>(tg & 0xffffu);
                }
            }
        }
        __syncthreads();  // tags clear before the next tile's entries
    };
    for (long long i = tb; i < te; i += 2) {
        step(i, va, la, vb, lb);
        if (i + 1 < te) step(i + 1, vb, lb, va, la);
    }
}

// ---------------------------------------------------------------------------
// Reverse-order scatter over windows, with a written-bitmap
// ---------------------------------------------------------------------------
constexpr int kScatThreads = 1024;
constexpr int kScatWarps = kScatThreads / 32;
constexpr int kWinTiles = 32;
constexpr int kWinElems = kWinTiles * kTileElems;
constexpr int kScatDepth = 4;

struct ScatParams {
    WsView ws;
    uint16_t *const *snap_ptrs;
    const uint32_t *index;
    long long tiles_per_cta;
    int K;
    DeltaRef d[kChainGroup];
};

struct ScatSmem {
    uint32_t written[kWinElems / 32];
    long long cur[kChainGroup];      // per delta: first entry of the current window
    long long len[kChainGroup];      // per delta: entries of the current window
    long long base[kWinTiles];       // per window tensor: (first_tile - window start) * tile
    long long numel[kWinTiles];
    uint16_t *ptr[kWinTiles];
    long long offs[2][kWinTiles + 1];  // a delta's offsets of the window tensors (by parity)
};

__global__ void __launch_bounds__(kScatThreads, 1) chain_scatter_kernel(ScatParams p) {
    extern __shared__ __align__(128) unsigned char scat_smem_raw[];
    ScatSmem &sm = *reinterpret_cast<ScatSmem *>(scat_smem_raw);
    const int tid = threadIdx.x;
    const int lane = tid & 31;
    const int warp = tid >> 5;

    if (!ws_matches(p.ws)) return;
    if (ld_relaxed_gpu_u32(&p.ws.hdr->delta_bad) != 0u) return;
    const long long tb = static_cast<long long>(blockIdx.x) * p.tiles_per_cta;
    long long te = tb + p.tiles_per_cta;
    if (te > p.ws.num_tiles) te = p.ws.num_tiles;
    if (tb >= te) return;

    if (tid < p.K) sm.cur[tid] = index_entry(p.d[tid], p.index, tb, tid, p.ws.tile_tensor[tb]);

    for (long long a = tb; a < te; a += kWinTiles) {
        const long long b = (a + kWinTiles < te) ? a + kWinTiles : te;
        const int win_words = static_cast<int>(b - a) * (kTileElems / 32);
        const int t_lo = p.ws.tile_tensor[a];
        const int nt = p.ws.tile_tensor[b - 1] - t_lo + 1;  // <= b - a: every tensor owns a tile
        if (t_lo < 0 || nt < 1 || nt > kWinTiles || t_lo + nt > p.ws.num_tensors) {
            if (tid == 0) record_error(p.ws.hdr, DWS_ERR_WORKSPACE, a);
            return;  // uniform: every thread read the same table entries
        }
        __syncthreads();  // the previous window is complete
        if (p.K > 1)
            for (int w = tid; w < win_words; w += kScatThreads) sm.written[w] = 0u;
        if (tid < nt) {
            const int t = t_lo + tid;
            const long long n = p.ws.numel[t];
            uint16_t *ptr = p.snap_ptrs[t];
            if (n > 0 && (ptr == nullptr || (reinterpret_cast<uintptr_t>(ptr) & 1u))) {
                record_error(p.ws.hdr, DWS_ERR_INVALID, t);
                ptr = nullptr;
            }
            sm.base[tid] = (p.ws.first_tile[t] - a) << kTileShift;
            sm.numel[tid] = n;
            sm.ptr[tid] = ptr;
        }
        if (tid < p.K) {
            const int tn = b < p.ws.num_tiles ? p.ws.tile_tensor[b] : p.ws.num_tensors - 1;
            sm.len[tid] = index_entry(p.d[tid], p.index, b, tid, tn) - sm.cur[tid];
        }
        constexpr long long kStride = 32LL * kScatWarps;
        if (tid <= nt) sm.offs[(p.K - 1) & 1][tid] = p.d[p.K - 1].offsets[t_lo + tid];
        __syncthreads();

        int ix[kScatDepth];
        uint16_t vx[kScatDepth];
        bool prefetched = false;  // the phase's first chunks already requested (uniform)
        for (int k = p.K - 1; k >= 0; --k) {
            const DeltaRef d = p.d[k];
            const int ph = k & 1;
            const long long *offs = sm.offs[ph];
            // the window's stretch of delta k, kept inside its arrays
            const long long j0 = sm.cur[k] < 0 ? 0 : (sm.cur[k] > d.count ? d.count : sm.cur[k]);
            const long long nl = sm.len[k] < 0 ? 0 : (j0 + sm.len[k] > d.count ? d.count - j0 : sm.len[k]);
            const int n = static_cast<int>(nl < kWinElems ? nl : kWinElems);  // one window of one delta
            const int *pi = d.indices + j0;
            const uint16_t *pv = d.values + j0;
            int r = 32 * warp + lane;  // this lane's entry of the current chunk
            if (!prefetched) {
#pragma unroll
                for (int q = 0; q < kScatDepth; ++q) {
                    if (r + q * kStride < n) {
                        ix[q] = __ldg(pi + r + q * kStride);
                        vx[q] = __ldg(pv + r + q * kStride);
                    }
                }
            }
            // The warp's current tensor (its chunks only move forward) and
            // that tensor's constants: segment end relative to j0, window
            // offset, size, pointer.
            int tw = 0;
            while (tw + 1 < nt && offs[tw + 1] <= j0 + r - lane) ++tw;
            long long seg_hi = offs[tw + 1] - j0;
            int off_c = static_cast<int>(-sm.base[tw]);
            uint16_t *ptr_c = sm.ptr[tw];
            for (bool more = r - lane < n; more;) {
#pragma unroll
                for (int q = 0; q < kScatDepth; ++q) {
                    const int cs = r - lane;
                    if (cs >= n) {  // the whole chunk is past the stretch (uniform)
                        more = false;
                        break;
                    }
                    const int idx = ix[q];
                    const uint16_t val = vx[q];
                    if (r + kScatDepth * kStride < n) {
                        ix[q] = __ldg(pi + r + kScatDepth * kStride);
                        vx[q] = __ldg(pv + r + kScatDepth * kStride);
                    }
                    const bool valid = r < n;
                    if (cs >= seg_hi) {  // uniform: move to the chunk's first tensor
                        while (tw + 1 < nt && offs[tw + 1] <= j0 + cs) ++tw;
                        seg_hi = offs[tw + 1] - j0;
                        off_c = static_cast<int>(-sm.base[tw]);
                        ptr_c = sm.ptr[tw];
                    }
                    const int cl = (cs + 31 < n) ? cs + 31 : n - 1;
                    uint32_t rel = 0;  // element within the window
                    uint16_t *dst = ptr_c;
                    if (cl < seg_hi) {
                        // The chunk lies in one tensor (checked entries:
                        // 0 <= idx - off_c < window length).
                        rel = static_cast<uint32_t>(idx - off_c);
                    } else if (valid) {
                        const long long j = j0 + r;
                        int tl = tw;
                        while (tl + 1 < nt && offs[tl + 1] <= j) ++tl;
                        rel = static_cast<uint32_t>(sm.base[tl] + idx);
                        dst = sm.ptr[tl];
                    }
                    if (valid && rel >= static_cast<uint32_t>(kWinElems)) {  // never expected
                        record_error(p.ws.hdr, DWS_ERR_WORKSPACE, j0 + r);
                        rel = 0;
                        dst = nullptr;
                    }
                    bool store = valid;
                    if (p.K > 1) {  // uniform: a single delta needs no written-bits
                        const uint32_t word = rel >> 5;
                        const uint32_t bit = 1u << (rel & 31u);
                        if (valid) store = (sm.written[word] & bit) == 0u;
                        // Mark this delta's elements: one OR per lane, or two
                        // for a run of 32 consecutive elements (a clustered
                        // change), where per-lane ORs would all hit one word.
                        const uint32_t r0 = __shfl_sync(0xffffffffu, rel, 0);
                        const uint32_t r31 = __shfl_sync(0xffffffffu, rel, 31);
                        bool marked = false;
                        if (r31 - r0 == 31u && cs + 31 < n) {  // uniform; entries ascend
                            if (lane == 0) atomicOr(&sm.written[r0 >> 5], ~0u << (r0 & 31u));
                            if (lane == 31 && (r31 & 31u) != 31u)
                                atomicOr(&sm.written[r31 >> 5], (2u << (r31 & 31u)) - 1u);
                            marked = true;
                        }
                        if (!marked && valid) atomicOr(&sm.written[word], bit);
                    }
                    if (store && dst != nullptr) dst[idx] = val;
                    r += kStride;
                }
            }
            // This warp is done with delta k.  While the others finish,
            // request the next (earlier) delta's offsets and first chunks.
            prefetched = false;
            if (k > 0) {
                const DeltaRef dn = p.d[k - 1];
                if (tid <= nt) sm.offs[ph ^ 1][tid] = dn.offsets[t_lo + tid];
                const long long jn = sm.cur[k - 1] < 0 ? 0 : (sm.cur[k - 1] > dn.count ? dn.count : sm.cur[k - 1]);
                const long long nn0 = sm.len[k - 1] < 0 ? 0 : (jn + sm.len[k - 1] > dn.count ? dn.count - jn : sm.len[k - 1]);
                const long long nn = nn0 < kWinElems ? nn0 : kWinElems;
                const int rn = 32 * warp + lane;
#pragma unroll
                for (int q = 0; q < kScatDepth; ++q) {
                    if (rn + q * kStride < nn) {
                        ix[q] = __ldg(dn.indices + jn + rn + q * kStride);
                        vx[q] = __ldg(dn.values + jn + rn + q * kStride);
                    }
                }
                prefetched = true;
            }
            __syncthreads();  // every entry of this delta stored before the next (earlier) one
        }
        if (tid < p.K) sm.cur[tid] += sm.len[tid];
    }
}

}  // namespace

cudaError_t chain_set_attributes() {
    cudaError_t e = cudaFuncSetAttribute(chain_merge_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(sizeof(MergeSmem)));
    if (e != cudaSuccess) return e;
    return cudaFuncSetAttribute(chain_scatter_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                static_cast<int>(sizeof(ScatSmem)));
}

cudaError_t chain_occupancy(int *ctas_per_sm) {
    return cudaOccupancyMaxActiveBlocksPerMultiprocessor(ctas_per_sm, chain_merge_kernel, kMThreads,
                                                         sizeof(MergeSmem));
}

cudaError_t index_occupancy(int *ctas_per_sm) {
    return cudaOccupancyMaxActiveBlocksPerMultiprocessor(ctas_per_sm, chain_index_kernel, kIdxThreads, 0);
}

cudaError_t scatter_occupancy(int *ctas_per_sm) {
    return cudaOccupancyMaxActiveBlocksPerMultiprocessor(ctas_per_sm, chain_scatter_kernel,
                                                         kScatThreads, sizeof(ScatSmem));
}

cudaError_t launch_apply_chain(const WsView &ws, uint16_t *const *snap_ptrs, const DeltaRef *deltas,
                               int K, bool merge, cudaStream_t s) {
    DeviceInfo di;
    cudaError_t e = device_info(&di);
    if (e != cudaSuccess) return e;
    e = launch_delta_check(ws, deltas, K, s);  // offsets of every delta
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
        if (merge) {
            MergeParams mp;
            mp.ws = ws;
            mp.snap_ptrs = snap_ptrs;
            mp.index = index;
            mp.K = kg;
            for (int k = 0; k < kg; ++k) mp.d[k] = deltas[k0 + k];
            long long grid = static_cast<long long>(di.sm_count) * di.chain_ctas_per_sm;
            if (grid > ws.num_tiles) grid = ws.num_tiles;
            if (grid < 1) grid = 1;
            mp.tiles_per_cta = (ws.num_tiles + grid - 1) / grid;
            grid = (ws.num_tiles + mp.tiles_per_cta - 1) / mp.tiles_per_cta;
            chain_merge_kernel<<<static_cast<unsigned int>(grid), kMThreads, sizeof(MergeSmem), s>>>(mp);
        } else {
            ScatParams sp;
            sp.ws = ws;
            sp.snap_ptrs = snap_ptrs;
            sp.index = index;
            sp.K = kg;
            for (int k = 0; k < kg; ++k) sp.d[k] = deltas[k0 + k];
            long long grid = static_cast<long long>(di.sm_count) * di.scatter_ctas_per_sm;
            const long long windows = (ws.num_tiles + kWinTiles - 1) / kWinTiles;
            if (grid > windows) grid = windows;
            if (grid < 1) grid = 1;
            // whole windows per CTA, so that only the last window of the plan is short
            const long long win_per_cta = (windows + grid - 1) / grid;
            sp.tiles_per_cta = win_per_cta * kWinTiles;
            grid = (ws.num_tiles + sp.tiles_per_cta - 1) / sp.tiles_per_cta;
            chain_scatter_kernel<<<static_cast<unsigned int>(grid), kScatThreads, sizeof(ScatSmem), s>>>(sp);
        }
        e = launched();
        if (e != cudaSuccess) return e;
    }
    return cudaSuccess;
}

}  // namespace dws

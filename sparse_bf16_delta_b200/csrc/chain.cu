// chain.cu -- replay of a chain of deltas onto an anchor snapshot, in place
// ("Delta Weight Sync in TRL" §4.1: an anchor every N syncs, sparse deltas in
// between; a new replica takes the latest anchor and replays the deltas after
// it, the later delta winning where two touch the same element).
//
// Three kernels per pass over the snapshot (up to 16 deltas a pass):
//
//   chain_index_kernel  reads every entry of every delta once (coalesced
//     16-byte loads), checks it (index inside its tensor, strictly above the
//     entry before it in its tensor's segment) and writes the chain's tile
//     index: for tile g and delta k, the first entry of k at or past the start
//     of g, mod 2^32 -- the rows inside each tensor's segment.  A failed check
//     sets the workspace's delta flag, and the replay kernel then writes
//     nothing: a chain with a bad entry anywhere is not applied at all.
//
//   chain_index_ends_kernel  one thread per tensor and delta: the index rows
//     of the tensor's tiles before its first entry and after its last.
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
// Row g of the tile index, column k: the first entry of delta k at or past
// the start of tile g (mod 2^32); row ntiles: the delta's entry count n.
// With every entry valid the tiles of the entries never decrease, and
//   rows of tensor t's tiles up to the tile of its first entry a: a,
//   rows (tile of j-1, tile of j] for j inside t's segment: j,
//   rows after the tile of t's last entry b-1, to t's last tile: b,
//   all of t's rows when its segment is empty: a.
// chain_index_ends_kernel writes the first, third and fourth kind (one
// thread per tensor and delta), chain_index_kernel the second while it checks
// every entry, so that no thread needs the tile of an entry of another tensor.
constexpr int kIdxThreads = 256;
constexpr int kIdxPerThread = 16;
constexpr int kIdxChunk = kIdxThreads * kIdxPerThread;  // entries per block
constexpr int kEndsThreads = 256;

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

__device__ __forceinline__ bool header_ok(const WsView &ws) {
    const WsHeader *h = ws.hdr;
    return h->magic == kWsMagic && h->fingerprint == ws.fingerprint && h->num_tiles == ws.num_tiles &&
           h->num_tensors == ws.num_tensors;
}

// Thread (t, k): the rows of tensor t's tiles before and after its segment
// of delta k (the whole tensor if the segment is empty), and row ntiles.
__global__ void __launch_bounds__(kEndsThreads) chain_index_ends_kernel(IndexParams p) {
    const int lane = threadIdx.x & 31;
    const int k = blockIdx.y;
    const int T = p.ws.num_tensors;
    const long long t = static_cast<long long>(blockIdx.x) * kEndsThreads + threadIdx.x;
    if (!header_ok(p.ws) || ld_relaxed_gpu_u32(&p.ws.hdr->delta_bad) != 0u) return;  // uniform
    const DeltaRef d = p.d[k];
    const long long ntiles = p.ws.num_tiles;
    if (t == 0) p.index[ntiles * kChainGroup + k] = static_cast<uint32_t>(d.offsets[T]);
    long long lo1 = 0, hi1 = 0, lo2 = 0, hi2 = 0;  // rows (lo, hi]
    uint32_t v1 = 0, v2 = 0;
    if (t < T) {
        const long long a = d.offsets[t], b = d.offsets[t + 1];
        const long long f0 = p.ws.first_tile[t], f1 = p.ws.first_tile[t + 1];
        if (a >= b) {
            lo1 = f0 - 1;
            hi1 = f1 - 1;
            v1 = static_cast<uint32_t>(a);
        } else {
            // a bad index is flagged by the entry pass; here it only must
            // not move the rows outside the tensor's own
            long long ga = f0 + (static_cast<long long>(d.indices[a]) >> kTileShift);
            long long gb = f0 + (static_cast<long long>(d.indices[b - 1]) >> kTileShift);
            ga = ga < f0 - 1 ? f0 - 1 : (ga > f1 - 1 ? f1 - 1 : ga);
            gb = gb < f0 - 1 ? f0 - 1 : (gb > f1 - 1 ? f1 - 1 : gb);
            lo1 = f0 - 1;
            hi1 = ga;
            v1 = static_cast<uint32_t>(a);
            lo2 = gb;
            hi2 = f1 - 1;
            v2 = static_cast<uint32_t>(b);
        }
    }
    fill_rows(p.index, k, lo1, hi1, v1, lane, ntiles - 1);
    fill_rows(p.index, k, lo2, hi2, v2, lane, ntiles - 1);
}

// Per delta, one level-by-level 32-way search over the offsets for the
// tensor holding entry j (a non-empty one: the last t with offsets[t] <= j).
// Lane 0 returns it with that tensor's segment [a, b), size and first tile,
// read in the search's last level (lane c reads its candidate's).
struct TensorMeta {
    int t;
    long long a, b, numel, first_tile;
};
__device__ __forceinline__ TensorMeta warp_tensor_meta(const WsView &ws, const long long *offsets, int T,
                                                       long long j) {
    const int lane = threadIdx.x & 31;
    int lo = 0, hi = T - 1;  // the answer lies in [lo, hi]
    while (true) {
        const int span = hi - lo + 1;
        const int step = (span + 31) / 32;
        const int t = lo + lane * step;
        const bool in = t <= hi;
        const long long ot = in ? __ldg(offsets + t) : 0;
        long long ob = 0, nm = 0, ft = 0;
        if (step == 1 && in) {  // last level: the candidates' metadata too
            ob = __ldg(offsets + t + 1);
            nm = __ldg(ws.numel + t);
            ft = __ldg(ws.first_tile + t);
        }
        const unsigned int bl = __ballot_sync(0xffffffffu, in && ot <= j);  // a prefix of lanes
        const int c = bl ? __popc(bl) : 1;
        if (step == 1) {
            TensorMeta m;
            m.t = lo + c - 1;
            m.a = __shfl_sync(0xffffffffu, ot, c - 1);
            m.b = __shfl_sync(0xffffffffu, ob, c - 1);
            m.numel = __shfl_sync(0xffffffffu, nm, c - 1);
            m.first_tile = __shfl_sync(0xffffffffu, ft, c - 1);
            return m;
        }
        const int nlo = lo + (c - 1) * step;
        const int nhi = lo + c * step - 1;
        lo = nlo;
        hi = nhi < hi ? nhi : hi;
    }
}

// The rare paths of the index pass are kept out of line, so that the hot
// one stays small in the instruction cache; they reload the thread's entries
// (cache hits) instead of keeping them in registers.

// The tensor holding entry j (a non-empty segment), searched in [lo, hi].
__device__ __forceinline__ int tensor_in(const long long *offsets, int lo, int hi, long long j) {
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (offsets[mid] <= j) lo = mid;
        else hi = mid - 1;
    }
    return lo;
}

// A run across tensors, a short run, or one outside the block's first
// tensor: every entry's tensor is walked.  Checks entries [j0, j0 + nlive),
// writes the short gaps of rows (when `write`), sets bit q of *bigm for a
// long one; returns the first offending entry, or -1.
__device__ __noinline__ long long index_run_general(DeltaRef d, const long long *numel, const long long *first_tile,
                                                    uint32_t *index, int T, int k, long long j0, int nlive,
                                                    int t0, int t1, int write, unsigned int *bigm) {
    int tq = tensor_in(d.offsets, t0, t1 > t0 ? t1 : t0, j0);
    long long a = d.offsets[tq], b = d.offsets[tq + 1];
    long long nm = numel[tq], ft = first_tile[tq];
    int pv = j0 > 0 ? d.indices[j0 - 1] : 0;
    for (int q = 0; q < nlive; ++q) {
        const long long j = j0 + q;
        while (j >= b && tq + 1 < T) {  // the next non-empty segment holding j
            ++tq;
            a = d.offsets[tq];
            b = d.offsets[tq + 1];
            nm = numel[tq];
            ft = first_tile[tq];
        }
        const int i = d.indices[j];
        const bool opens = j == a;
        if (!(i >= 0 && i < nm && (opens || pv < i))) return j;
        if (!opens && write) {
            const int tp = pv >> kTileShift, tl = i >> kTileShift;
            if (tl - tp > 32) {
                *bigm |= 1u << q;
            } else {
                for (int g = tp + 1; g <= tl; ++g) index[(ft + g) * kChainGroup + k] = static_cast<uint32_t>(j);
            }
        }
        pv = i;
    }
    return -1;
}

// The first offending entry of a run that lies in one tensor (numel nm,
// opening its segment or not).
__device__ __noinline__ long long index_first_bad(const int *indices, long long j0, int nm, bool opens) {
    int pv = j0 > 0 ? indices[j0 - 1] : 0;
    for (int q = 0; q < kIdxPerThread; ++q) {
        const int i = indices[j0 + q];
        if (!(i >= 0 && i < nm && ((q == 0 && opens) || pv < i))) return j0 + q;
        pv = i;
    }
    return j0;
}

// The rows a checked run inside one tensor starts: bit q of `bnd` marks an
// entry j0 + q in a later tile than the entry before it (both in this
// tensor).  Short gaps are written here, long ones returned as a mask.  Out
// of line, and only the marked entries are reread: at the densities of the
// workloads a run crosses a tile about once in twenty.
__device__ __noinline__ unsigned int index_run_rows(const int *indices, uint32_t *index, int k, long long j0,
                                                    long long ft, unsigned int bnd) {
    unsigned int bigm = 0;
    while (bnd != 0u) {
        const int q = __ffs(bnd) - 1;
        bnd &= bnd - 1;
        const int tp = indices[j0 + q - 1] >> kTileShift, tl = indices[j0 + q] >> kTileShift;
        if (tl - tp <= 32) {
            for (int g = tp + 1; g <= tl; ++g) index[(ft + g) * kChainGroup + k] = static_cast<uint32_t>(j0 + q);
        } else {
            bigm |= 1u << q;
        }
    }
    return bigm;
}

// Long gaps (more than 32 rows, sparse deltas): for each q, the lanes with
// one at entry q write them together.  Every lane of the warp calls it.
__device__ __noinline__ void index_long_gaps(DeltaRef d, const long long *first_tile, uint32_t *index, int k,
                                             long long j0, unsigned int bigm, int t0, int t1, long long nrows) {
    const int lane = threadIdx.x & 31;
    for (int q = 0; q < kIdxPerThread; ++q) {
        const bool mine = (bigm >> q) & 1u;
        if (!__any_sync(0xffffffffu, mine)) continue;
        long long lo = 0, hi = 0;
        if (mine) {  // rows (tile of entry q-1, tile of entry q], both in one tensor
            const long long j = j0 + q;
            const long long ft = first_tile[tensor_in(d.offsets, t0, t1 > t0 ? t1 : t0, j)];
            lo = ft + (d.indices[j - 1] >> kTileShift);
            hi = ft + (d.indices[j] >> kTileShift);
        }
        fill_rows(index, k, lo, hi, static_cast<uint32_t>(j0 + q), lane, nrows);
    }
}

// Block (x, k): entries [x * kIdxChunk, (x + 1) * kIdxChunk) of delta k, 16
// consecutive ones per thread.  Every entry is checked (inside its tensor,
// strictly above the entry before it in its tensor's segment) and, when the
// index is written, entry j inside a segment writes rows (tile of j-1, tile
// of j].  The header, the entries and the first level of the searches for
// the tensors of the block's first and last entries are all requested at
// once; the first tensor's metadata arrives with the search's last level.
__global__ void __launch_bounds__(kIdxThreads, 6) chain_index_kernel(IndexParams p) {
    __shared__ TensorMeta s_m0;
    __shared__ int s_t1;
    __shared__ int s_ok;
    __shared__ long long s_n;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int k = blockIdx.y;
    const DeltaRef d = p.d[k];
    const int T = p.ws.num_tensors;
    const long long ntiles = p.ws.num_tiles;
    const long long base = static_cast<long long>(blockIdx.x) * kIdxChunk;
    if (base >= d.count) return;  // uniform: past this delta's arrays
    // the last entry the arrays hold in this block (the true last is <= it)
    const long long last_a = (base + kIdxChunk < d.count ? base + kIdxChunk : d.count) - 1;

    if (warp == 0) {
        s_m0 = warp_tensor_meta(p.ws, d.offsets, T, base);
    } else if (warp == 1) {
        int lo = 0, hi = T - 1;  // tensor of last_a (an upper bound for the block's tensors)
        while (true) {
            const int span = hi - lo + 1;
            const int step = (span + 31) / 32;
            const int t = lo + lane * step;
            const bool le = (t <= hi) && (__ldg(d.offsets + t) <= last_a);
            const unsigned int bl = __ballot_sync(0xffffffffu, le);
            const int c = bl ? __popc(bl) : 1;
            if (step == 1) {
                if (lane == 0) s_t1 = lo + c - 1;
                break;
            }
            const int nlo = lo + (c - 1) * step, nhi = lo + c * step - 1;
            lo = nlo;
            hi = nhi < hi ? nhi : hi;
        }
    } else if (tid == 64) {
        s_ok = header_ok(p.ws) && ld_relaxed_gpu_u32(&p.ws.hdr->delta_bad) == 0u;
        s_n = d.offsets[T];
    }
    // this thread's entries and the one before them, in flight meanwhile
    const long long j0 = base + static_cast<long long>(tid) * kIdxPerThread;
    const int nload = j0 > last_a ? 0 : static_cast<int>(last_a - j0 + 1 < kIdxPerThread ? last_a - j0 + 1 : kIdxPerThread);
    int x[kIdxPerThread];
    if (nload == kIdxPerThread && (reinterpret_cast<uintptr_t>(d.indices) & 15u) == 0) {
#pragma unroll
        for (int v = 0; v < kIdxPerThread / 4; ++v) {
            const int4 a4 = __ldg(reinterpret_cast<const int4 *>(d.indices + j0) + v);
            x[4 * v] = a4.x; x[4 * v + 1] = a4.y; x[4 * v + 2] = a4.z; x[4 * v + 3] = a4.w;
        }
    } else {
#pragma unroll
        for (int q = 0; q < kIdxPerThread; ++q) x[q] = (q < nload) ? __ldg(d.indices + j0 + q) : 0;
    }
    const int prev = (nload > 0 && j0 > 0) ? __ldg(d.indices + j0 - 1) : 0;
    __syncthreads();
    if (!s_ok) {
        if (tid == 0 && !header_ok(p.ws)) record_error(p.ws.hdr, DWS_ERR_WORKSPACE, 0);
        return;  // uniform: a foreign workspace, or the offsets failed
    }
    const long long n = s_n;
    if (base >= n) return;  // uniform
    const TensorMeta m0 = s_m0;
    const int t1 = s_t1;
    const long long last = (base + kIdxChunk < n ? base + kIdxChunk : n) - 1;
    const int nlive = j0 > last ? 0 : static_cast<int>(last - j0 + 1 < kIdxPerThread ? last - j0 + 1 : kIdxPerThread);

    long long bad_j = -1;
    unsigned int bigm = 0;  // bit q: a long gap of rows ends at entry q
    if (nlive == kIdxPerThread && m0.a <= j0 && j0 + kIdxPerThread - 1 < m0.b) {
        // Common case, 32-bit: the run lies in tensor m0.t.  It must ascend
        // strictly (one compare per entry); then it is in range if its ends
        // are.  A run that opens the segment has no order check on its first
        // entry and writes no rows for it (the ends kernel does).
        const int nm = static_cast<int>(m0.numel);
        const bool opens = m0.a == j0;
        bool viol = !opens && !(prev < x[0]);
#pragma unroll
        for (int q = 1; q < kIdxPerThread; ++q) viol |= !(x[q - 1] < x[q]);
        if (viol || x[0] < 0 || x[kIdxPerThread - 1] >= nm) {
            bad_j = index_first_bad(d.indices, j0, nm, opens);
        } else if (p.write) {
            // any tile change in the run (or from the entry before it)?
            const int tp = opens ? (x[0] >> kTileShift) : (prev >> kTileShift);
            if ((x[kIdxPerThread - 1] >> kTileShift) != tp) {
                unsigned int bnd = (x[0] >> kTileShift) != tp ? 1u : 0u;
#pragma unroll
                for (int q = 1; q < kIdxPerThread; ++q)
                    bnd |= ((x[q] >> kTileShift) != (x[q - 1] >> kTileShift)) ? (1u << q) : 0u;
                bigm = index_run_rows(d.indices, p.index, k, j0, m0.first_tile, bnd);
            }
        }
    } else if (nlive > 0) {
        bad_j = index_run_general(d, p.ws.numel, p.ws.first_tile, p.index, T, k, j0, nlive, m0.t, t1, p.write,
                                  &bigm);
    }
    if (bad_j >= 0) bigm = 0;
    if (__any_sync(0xffffffffu, bigm != 0u))
        index_long_gaps(d, p.ws.first_tile, p.index, k, j0, bigm, m0.t, t1, ntiles - 1);
    if (bad_j >= 0) {
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
constexpr int kTileItems = 2;                             // items per warp per round
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
    int vlim[kChainGroup];                      // 16-byte loads at offsets below this (aligned
                                                // arrays, 4 entries inside them)
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

// A warp's position in the tile's item list: item i of delta k covers
// entries base + 128 (i - C[k]) + [0, 128); the delta's constants are kept in
// registers and reread only when the warp moves on to the next delta.
struct ItemCursor {
    int k, ck, cn;  // delta, C[k], C[k + 1]
    int lo, hi, vlim;
    const int *ip;
    const uint16_t *vp;
};

__device__ __forceinline__ void cursor_load(const TileShared &sm, ItemCursor &c) {
    c.ck = sm.C[c.k];
    c.cn = sm.C[c.k + 1];
    c.lo = sm.lo[c.k];
    c.hi = sm.hi[c.k];
    c.vlim = sm.vlim[c.k];
    c.ip = sm.ip[c.k];
    c.vp = sm.vp[c.k];
}

// Items i0 .. i0 + kTileItems - 1 of this warp (those below iend; the warp
// takes its items in order): lane l takes the 4 entries from base + 128 c +
// 4 l.  kq[q] = k (warp-uniform; -1: no such item); vm[q] bit e: entry e is
// the tile's.  Every load of the round is in flight at once.
__device__ __forceinline__ void tile_load_round(const TileShared &sm, int K, ItemCursor &c, int i0, int iend,
                                                int4 (&ix)[kTileItems], uint2 (&vx)[kTileItems],
                                                int (&kq)[kTileItems], unsigned int (&vm)[kTileItems]) {
    const int lane = threadIdx.x & 31;
#pragma unroll
    for (int q = 0; q < kTileItems; ++q) {
        const int i = i0 + q;
        kq[q] = -1;
        vm[q] = 0u;
        if (i < iend) {  // warp-uniform
            if (i >= c.cn) {  // the next delta with items (C[K] > i, so k stays below K)
                do {
                    ++c.k;
                } while (c.k + 1 < K && sm.C[c.k + 1] <= i);
                cursor_load(sm, c);
            }
            kq[q] = c.k;
            const int o = (i - c.ck) * kItemEntries + 4 * lane;
            unsigned int m = 0xfu;
            if (o < c.lo || o + 4 > c.hi) {  // an item's ends only
                m = 0u;
#pragma unroll
                for (int e = 0; e < 4; ++e) m |= (o + e >= c.lo && o + e < c.hi) ? (1u << e) : 0u;
            }
            vm[q] = m;
            if (o < c.vlim) {  // entries outside [lo, hi) are loaded and not used
                ix[q] = __ldg(reinterpret_cast<const int4 *>(c.ip + o));
                vx[q] = __ldg(reinterpret_cast<const uint2 *>(c.vp + o));
            } else if (m != 0u) {
                int xs[4] = {0, 0, 0, 0};
                uint32_t vs[4] = {0u, 0u, 0u, 0u};
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    if ((m >> e) & 1u) {
                        xs[e] = __ldg(c.ip + o + e);
                        vs[e] = __ldg(c.vp + o + e);
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
            const bool vec = (reinterpret_cast<uintptr_t>(d.indices) & 15u) == 0 &&
                             (reinterpret_cast<uintptr_t>(d.values) & 7u) == 0;
            const long long room = d.count - base - 3;  // offsets o with o + 3 inside the arrays
            sm.vlim[lane] = !vec ? 0 : static_cast<int>(room < (1LL << 30) ? (room > 0 ? room : 0) : (1LL << 30));
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

    // this warp's items: a contiguous range, in rounds of kTileItems
    const int warp = tid >> 5;
    const int per = (items + kTileWarps - 1) / kTileWarps;
    const int ib = warp * per < items ? warp * per : items;
    const int ie = ib + per < items ? ib + per : items;
    ItemCursor cur;
    cur.k = 0;
    cursor_load(sm, cur);
    int4 ix[kTileItems];
    uint2 vx[kTileItems];
    int kq[kTileItems];
    unsigned int vm[kTileItems];
    tile_load_round(sm, K, cur, ib, ie, ix, vx, kq, vm);
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
    if constexpr (kMerge) __syncthreads();  // tags initialised (the scatter's were zeroed before the first barrier)
    bool outside = false;  // an entry outside the tile: never, for checked entries
    for (int i0 = ib; i0 < ie; i0 += kTileItems) {
        if (i0 > ib) tile_load_round(sm, K, cur, i0, ie, ix, vx, kq, vm);
#pragma unroll
        for (int q = 0; q < kTileItems; ++q) {
            if (kq[q] < 0) continue;  // warp-uniform
            const uint32_t ver = static_cast<uint32_t>(kq[q] + 1) << 16;
            const unsigned int m = vm[q];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const uint32_t pos = static_cast<uint32_t>(int4_at(ix[q], e) - local);
                const bool use = (m == 0xfu) || ((m >> e) & 1u);
                const bool in = pos < static_cast<uint32_t>(count);
                if (use && in) atomicMax(&s_tag[pos], ver | u16x4_at(vx[q], e));
                outside |= use && !in;
            }
        }
    }
    if (outside) record_error(p.ws.hdr, DWS_ERR_WORKSPACE, g);
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
        const long long ex = (static_cast<long long>(ws.num_tensors) + kEndsThreads - 1) / kEndsThreads;
        chain_index_ends_kernel<<<dim3(static_cast<unsigned int>(ex), kg), kEndsThreads, 0, s>>>(ip);
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
